"""Wave-index sparse decode attention and segmented k-means index build for
NVIDIA B200 (sm_100a).

A thin ctypes binding over libwi.so (include/wi.h).  Every step of the path
runs in the library's CUDA kernels; this module only allocates tensors with
torch, marshals pointers and sizes, and turns status codes into exceptions.
There is no CPU fallback: importing fails loudly when libwi.so is missing.

Method: "RetroInfer: A Vector Storage Engine for Scalable Long-Context LLM
Inference" (technical summary), section 2.A Wave Index (steady, retrieval and
estimation zones; segmented clustering); build/decode split and paged layout
after the Vortex summary, sections 2.A and 2.B.
"""
from __future__ import annotations

import ctypes as C
import math
import os
from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwi.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing; build it with "
        "`python retrieval_sparse_attention_wave_b200/build.py` (needs nvcc)")
_lib = C.CDLL(LIB_PATH)

# ---------------------------------------------------------------- C types

WI_OK, WI_ERR_INVALID_ARG, WI_ERR_UNSUPPORTED, WI_ERR_WORKSPACE, WI_ERR_CUDA, \
    WI_ERR_DEVICE_CHECK = range(6)
WI_F32, WI_BF16 = 0, 1
WI_MAX_BATCH = 256
WI_MAX_SEG_LEN = 16384
WI_MAX_STEADY = 8192
WI_DEV_BAD_PAGE, WI_DEV_BAD_SLOT, WI_DEV_BAD_CLUSTER, WI_DEV_BAD_HIST = 0x1, 0x2, 0x4, 0x8
WI_DEV_TIMEOUT, WI_DEV_CANCELLATION = 0x10, 0x20
WI_TOPK_EXACT, WI_TOPK_SAMPLED = 0, 1

EXPORTED = [
    "wi_index_clusters", "wi_build_workspace_size", "wi_build_workspace_layout",
    "wi_build_index", "wi_build_blocks",
    "wi_extend_index",
    "wi_kmeans_assign",
    "wi_decode_workspace_size", "wi_decode_workspace_layout", "wi_decode", "wi_decode_host",
    "wi_decode_stage_count", "wi_decode_stage_name", "wi_read_device_status",
    "wi_status_string", "wi_last_error_string", "wi_decode_noalloc",
]


class WiKVCache(C.Structure):
    _fields_ = [("dtype", C.c_int), ("batch", C.c_int32), ("n_kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("page_size", C.c_int32), ("n_pages", C.c_int64),
                ("k_pool", C.c_void_p), ("v_pool", C.c_void_p), ("block_table", C.c_void_p),
                ("max_pages", C.c_int32), ("seq_lens", C.POINTER(C.c_int32))]


class WiIndex(C.Structure):
    _fields_ = [("dtype", C.c_int), ("batch", C.c_int32), ("n_kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("page_size", C.c_int32), ("seg_len", C.c_int32),
                ("cluster_size", C.c_int32), ("seq_lens", C.POINTER(C.c_int32)),
                ("centroids", C.c_void_p), ("value_sums", C.c_void_p), ("offsets", C.c_void_p),
                ("perm", C.c_void_p), ("invperm", C.c_void_p), ("labels", C.c_void_p),
                ("k_pool", C.c_void_p),
                ("v_pool", C.c_void_p), ("n_pages", C.c_int64), ("block_table", C.c_void_p),
                ("max_pages", C.c_int32)]


class WiDecodeParams(C.Structure):
    _fields_ = [("n_q_heads", C.c_int32), ("n_sink", C.c_int32), ("window", C.c_int32),
                ("topk_clusters", C.c_int32), ("topk_fraction", C.c_double),
                ("stage_events", C.POINTER(C.c_void_p)), ("exact_only", C.c_int32),
                ("topk_mode", C.c_int32), ("seed", C.c_uint32), ("scores_out", C.c_void_p)]


class WiBuildLayout(C.Structure):
    _fields_ = [("total_bytes", C.c_size_t), ("status", C.c_size_t),
                ("centroids_f32", C.c_size_t), ("assign", C.c_size_t)]


class WiDecodeLayout(C.Structure):
    _fields_ = [("total_bytes", C.c_size_t), ("status", C.c_size_t), ("records", C.c_size_t),
                ("selected", C.c_size_t), ("unit_info", C.c_size_t),
                ("n_scan_ctas", C.c_int32), ("n_gather_ctas", C.c_int32),
                ("info_ints", C.c_int32)]


_P = C.c_void_p
_sig = {
    "wi_index_clusters": (C.c_int, [C.c_int32, C.POINTER(C.c_int32), C.c_int32, C.c_int32,
                                    C.POINTER(C.c_int32), C.POINTER(C.c_int64)]),
    "wi_build_workspace_size": (C.c_int, [C.POINTER(WiKVCache), C.c_int32, C.c_int32,
                                          C.POINTER(C.c_size_t)]),
    "wi_build_workspace_layout": (C.c_int, [C.POINTER(WiKVCache), C.c_int32, C.c_int32,
                                            C.POINTER(WiBuildLayout)]),
    "wi_build_index": (C.c_int, [C.POINTER(WiKVCache), C.c_int32, C.c_int32, C.c_int32,
                                 C.POINTER(WiIndex), _P, C.c_size_t, _P]),
    "wi_build_blocks": (C.c_int, [C.POINTER(WiKVCache), C.c_int32, C.c_int32,
                                  C.POINTER(WiIndex), _P, C.c_size_t, _P]),
    "wi_extend_index": (C.c_int, [C.POINTER(WiIndex), C.POINTER(WiKVCache), C.c_int32,
                                  C.POINTER(WiIndex), _P, C.c_size_t, _P]),
    "wi_kmeans_assign": (C.c_int, [C.POINTER(WiKVCache), C.c_int32, C.c_int32, _P, _P, _P,
                                   C.c_size_t, _P]),
    "wi_decode_workspace_size": (C.c_int, [C.POINTER(WiIndex), C.POINTER(WiDecodeParams),
                                           C.POINTER(C.c_size_t)]),
    "wi_decode_workspace_layout": (C.c_int, [C.POINTER(WiIndex), C.POINTER(WiDecodeParams),
                                             C.POINTER(WiDecodeLayout)]),
    "wi_decode": (C.c_int, [_P, C.POINTER(WiIndex), C.POINTER(WiDecodeParams), _P, _P, _P,
                            C.c_size_t, _P]),
    "wi_decode_host": (C.c_int, [_P, C.POINTER(WiIndex), C.POINTER(WiDecodeParams), _P, _P, _P,
                                 C.c_size_t, _P]),
    "wi_decode_noalloc": (C.c_int, [_P, C.POINTER(WiIndex), C.POINTER(WiDecodeParams), _P, _P,
                                    _P]),
    "wi_decode_stage_count": (C.c_int32, []),
    "wi_decode_stage_name": (C.c_char_p, [C.c_int32]),
    "wi_read_device_status": (C.c_int, [_P, _P, C.POINTER(C.c_uint32), C.c_int]),
    "wi_status_string": (C.c_char_p, [C.c_int]),
    "wi_last_error_string": (C.c_char_p, []),
}
for _name, (_res, _args) in _sig.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class WaveIndexError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.wi_status_string(status).decode()
        if status == WI_ERR_CUDA:
            msg += ": " + _lib.wi_last_error_string().decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


def _check(status: int, where: str):
    if status != WI_OK:
        raise WaveIndexError(status, where)


def lib() -> C.CDLL:
    return _lib


# ---------------------------------------------------------------- helpers

def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return WI_BF16
    if dt == torch.float32:
        return WI_F32
    raise ValueError(f"unsupported KV dtype {dt}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream_ptr(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _i32_array(xs: Sequence[int]):
    arr = (C.c_int32 * len(xs))(*[int(x) for x in xs])
    return arr


def clusters_per_sequence(seq_lens: Sequence[int], seg_len: int, cluster_size: int) -> List[int]:
    """NC_b = sum over segments of ceil(len/cluster_size) (library's own count)."""
    n = len(seq_lens)
    out = (C.c_int32 * n)()
    tot = C.c_int64()
    _check(_lib.wi_index_clusters(n, _i32_array(seq_lens), seg_len, cluster_size, out,
                                  C.byref(tot)), "wi_index_clusters")
    return list(out)


def pages_for(T: int, page_size: int) -> int:
    return (T + page_size - 1) // page_size


def contiguous_block_table(seq_lens: Sequence[int], page_size: int, device) -> torch.Tensor:
    """Block table giving each sequence its own consecutive run of pages."""
    need = [pages_for(T, page_size) for T in seq_lens]
    bt = torch.full((len(seq_lens), max(need)), -1, dtype=torch.int32)
    at = 0
    for b, n in enumerate(need):
        bt[b, :n] = torch.arange(at, at + n, dtype=torch.int32)
        at += n
    return bt.to(device)


# ---------------------------------------------------------------- KV cache

@dataclass
class KVCache:
    """Paged KV cache in original token order.

    k_pool, v_pool: [n_pages][n_kv_heads][page_size][head_dim] (bf16 or fp32, on the GPU)
    block_table: [batch][max_pages] int32 on the GPU; seq_lens: host list.
    """
    k_pool: torch.Tensor
    v_pool: torch.Tensor
    block_table: torch.Tensor
    seq_lens: List[int]

    def __post_init__(self):
        self._seq = _i32_array(self.seq_lens)

    @property
    def n_kv_heads(self) -> int:
        return self.k_pool.shape[1]

    @property
    def page_size(self) -> int:
        return self.k_pool.shape[2]

    @property
    def head_dim(self) -> int:
        return self.k_pool.shape[3]

    def c_struct(self) -> WiKVCache:
        s = WiKVCache()
        s.dtype = _dtype_code(self.k_pool.dtype)
        s.batch = len(self.seq_lens)
        s.n_kv_heads = self.n_kv_heads
        s.head_dim = self.head_dim
        s.page_size = self.page_size
        s.n_pages = self.k_pool.shape[0]
        s.k_pool = self.k_pool.data_ptr()
        s.v_pool = self.v_pool.data_ptr()
        s.block_table = self.block_table.data_ptr()
        s.max_pages = self.block_table.shape[1]
        s.seq_lens = C.cast(self._seq, C.POINTER(C.c_int32))
        return s


# ---------------------------------------------------------------- the index

class WaveIndex:
    """Caller-owned buffers of one batch's wave index (see include/wi.h)."""

    def __init__(self, seq_lens, n_kv_heads, head_dim, dtype, page_size, seg_len, cluster_size,
                 device, block_table: Optional[torch.Tensor] = None,
                 n_pages: Optional[int] = None, pools=None):
        self.seq_lens = [int(t) for t in seq_lens]
        self.n_kv_heads, self.head_dim, self.dtype = n_kv_heads, head_dim, dtype
        self.page_size, self.seg_len, self.cluster_size = page_size, seg_len, cluster_size
        self.nc = clusters_per_sequence(self.seq_lens, seg_len, cluster_size)
        H, B = n_kv_heads, len(self.seq_lens)
        ncl, ntok = H * sum(self.nc), H * sum(self.seq_lens)
        dev = torch.device(device)
        self.centroids = torch.zeros(ncl, head_dim, dtype=dtype, device=dev)
        self.value_sums = torch.zeros(ncl, head_dim, dtype=dtype, device=dev)
        self.offsets = torch.zeros(H * (sum(self.nc) + B), dtype=torch.int32, device=dev)
        self.perm = torch.zeros(ntok, dtype=torch.int32, device=dev)
        self.invperm = torch.zeros(ntok, dtype=torch.int32, device=dev)
        self.labels = torch.zeros(ntok, dtype=torch.int32, device=dev)
        if block_table is None:
            block_table = contiguous_block_table(self.seq_lens, page_size, dev)
        if n_pages is None:
            n_pages = int(block_table.max().item()) + 1
        self.block_table = block_table.to(device=dev, dtype=torch.int32).contiguous()
        if pools is not None:   # another index's permuted pools (an extension)
            self.k_pool, self.v_pool = pools
        else:
            self.k_pool = torch.zeros(n_pages, H, page_size, head_dim, dtype=dtype, device=dev)
            self.v_pool = torch.zeros_like(self.k_pool)
        self._seq = _i32_array(self.seq_lens)

    # unit (b, h) views ------------------------------------------------------
    def cl_row(self, b: int, h: int) -> int:
        return self.n_kv_heads * sum(self.nc[:b]) + h * self.nc[b]

    def off_row(self, b: int, h: int) -> int:
        return self.n_kv_heads * (sum(self.nc[:b]) + b) + h * (self.nc[b] + 1)

    def tok_row(self, b: int, h: int) -> int:
        return self.n_kv_heads * sum(self.seq_lens[:b]) + h * self.seq_lens[b]

    def c_struct(self) -> WiIndex:
        # the marshalled struct is kept while the buffers it points at are
        # the same (a decode per layer and step marshals the same index)
        bufs = (self.centroids, self.value_sums, self.offsets, self.perm, self.invperm,
                self.labels, self.k_pool, self.v_pool, self.block_table)
        sig = tuple(t.data_ptr() for t in bufs) + (self.k_pool.shape[0], self.block_table.shape[1])
        if getattr(self, "_cs_sig", None) == sig:
            return self._cs
        s = WiIndex()
        s.dtype = _dtype_code(self.dtype)
        s.batch = len(self.seq_lens)
        s.n_kv_heads = self.n_kv_heads
        s.head_dim = self.head_dim
        s.page_size = self.page_size
        s.seg_len = self.seg_len
        s.cluster_size = self.cluster_size
        s.seq_lens = C.cast(self._seq, C.POINTER(C.c_int32))
        s.centroids = self.centroids.data_ptr()
        s.value_sums = self.value_sums.data_ptr()
        s.offsets = self.offsets.data_ptr()
        s.perm = self.perm.data_ptr()
        s.invperm = self.invperm.data_ptr()
        s.labels = self.labels.data_ptr()
        s.k_pool = self.k_pool.data_ptr()
        s.v_pool = self.v_pool.data_ptr()
        s.n_pages = self.k_pool.shape[0]
        s.block_table = self.block_table.data_ptr()
        s.max_pages = self.block_table.shape[1]
        self._cs, self._cs_sig = s, sig
        return s


# ---------------------------------------------------------------- build

def build_workspace_bytes(kv: KVCache, seg_len: int, cluster_size: int) -> int:
    n = C.c_size_t()
    s = kv.c_struct()
    _check(_lib.wi_build_workspace_size(C.byref(s), seg_len, cluster_size, C.byref(n)),
           "wi_build_workspace_size")
    return n.value


def build_layout(kv: KVCache, seg_len: int, cluster_size: int) -> WiBuildLayout:
    lay = WiBuildLayout()
    s = kv.c_struct()
    _check(_lib.wi_build_workspace_layout(C.byref(s), seg_len, cluster_size, C.byref(lay)),
           "wi_build_workspace_layout")
    return lay


def build_state(kv: KVCache, index: "WaveIndex"):
    """The fp32 working centroids [Hkv * sum NC_b][d] and the int32 assignment
    [Hkv * sum T_b] a build left in its workspace (views into it)."""
    lay = build_layout(kv, index.seg_len, index.cluster_size)
    ws = index._build_ws
    ncl = index.n_kv_heads * sum(index.nc)
    ntok = index.n_kv_heads * sum(index.seq_lens)
    cent = ws[lay.centroids_f32:lay.centroids_f32 + ncl * index.head_dim * 4].view(torch.float32)
    asg = ws[lay.assign:lay.assign + ntok * 4].view(torch.int32)
    return cent.view(ncl, index.head_dim), asg


def workspace(nbytes: int, device) -> torch.Tensor:
    """A zeroed, 256-byte aligned workspace tensor (torch allocations are)."""
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)


def build_index(kv: KVCache, seg_len: int, cluster_size: int, iters: int,
                out: Optional[WaveIndex] = None, ws: Optional[torch.Tensor] = None,
                block_table: Optional[torch.Tensor] = None, n_pages: Optional[int] = None,
                stream=None) -> WaveIndex:
    """Segmented k-means index build into caller-owned (or newly allocated) buffers."""
    if out is None:
        out = WaveIndex(kv.seq_lens, kv.n_kv_heads, kv.head_dim, kv.k_pool.dtype, kv.page_size,
                        seg_len, cluster_size, kv.k_pool.device, block_table, n_pages)
    need = build_workspace_bytes(kv, seg_len, cluster_size)
    if ws is None:
        ws = workspace(need, kv.k_pool.device)
    s, o = kv.c_struct(), out.c_struct()
    _check(_lib.wi_build_index(C.byref(s), seg_len, cluster_size, iters, C.byref(o),
                               _ptr(ws), ws.numel(), _stream_ptr(stream)), "wi_build_index")
    out._build_ws = ws
    return out


def build_blocks(kv: KVCache, seg_len: int, block_size: int, out: Optional[WaveIndex] = None,
                 ws: Optional[torch.Tensor] = None, block_table: Optional[torch.Tensor] = None,
                 n_pages: Optional[int] = None, stream=None) -> WaveIndex:
    """Index of position-contiguous blocks of block_size tokens (block
    centroids and value sums; perm is the identity), laid out like a k-means
    index with cluster_size = block_size."""
    if out is None:
        out = WaveIndex(kv.seq_lens, kv.n_kv_heads, kv.head_dim, kv.k_pool.dtype, kv.page_size,
                        seg_len, block_size, kv.k_pool.device, block_table, n_pages)
    need = build_workspace_bytes(kv, seg_len, block_size)
    if ws is None:
        ws = workspace(need, kv.k_pool.device)
    s, o = kv.c_struct(), out.c_struct()
    _check(_lib.wi_build_blocks(C.byref(s), seg_len, block_size, C.byref(o), _ptr(ws), ws.numel(),
                                _stream_ptr(stream)), "wi_build_blocks")
    out._build_ws = ws
    return out


def extend_index(old: WaveIndex, kv: KVCache, iters: int, ws: Optional[torch.Tensor] = None,
                 stream=None) -> WaveIndex:
    """The index of the longer sequences in `kv`, grown from `old` segment by
    segment (new centroid / value-sum / offset / perm / invperm / label
    buffers; `old`'s permuted pools and block table are kept, so the block
    table must already map pages for the new slots)."""
    out = WaveIndex(kv.seq_lens, old.n_kv_heads, old.head_dim, old.dtype, old.page_size,
                    old.seg_len, old.cluster_size, old.k_pool.device, old.block_table,
                    old.k_pool.shape[0], pools=(old.k_pool, old.v_pool))
    need = build_workspace_bytes(kv, old.seg_len, old.cluster_size)
    if ws is None:
        ws = workspace(need, kv.k_pool.device)
    o_old, s, o = old.c_struct(), kv.c_struct(), out.c_struct()
    _check(_lib.wi_extend_index(C.byref(o_old), C.byref(s), iters, C.byref(o), _ptr(ws),
                                ws.numel(), _stream_ptr(stream)), "wi_extend_index")
    out._build_ws = ws
    return out


def kmeans_assign(kv: KVCache, seg_len: int, cluster_size: int, centroids: torch.Tensor,
                  ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One assignment step against caller-given fp32 centroids
    ([Hkv * sum NC_b][d], unit-major).  Returns int32 [Hkv * sum T_b]."""
    assert centroids.dtype == torch.float32 and centroids.is_contiguous()
    H = kv.n_kv_heads
    assign = torch.full((H * sum(kv.seq_lens),), -1, dtype=torch.int32,
                        device=kv.k_pool.device)
    need = build_workspace_bytes(kv, seg_len, cluster_size)
    if ws is None:
        ws = workspace(need, kv.k_pool.device)
    s = kv.c_struct()
    _check(_lib.wi_kmeans_assign(C.byref(s), seg_len, cluster_size, _ptr(centroids),
                                 _ptr(assign), _ptr(ws), ws.numel(), _stream_ptr(stream)),
           "wi_kmeans_assign")
    return assign


# ---------------------------------------------------------------- decode

@dataclass
class DecodeParams:
    n_q_heads: int
    n_sink: int = 4
    window: int = 64
    topk_clusters: int = -1
    topk_fraction: float = 0.018
    exact_only: bool = False     # no estimation zone (block top-k workload)
    sampled: bool = False        # stochastic radix top-k (threshold bin sampled)
    seed: int = 0                # draws of the sampled selection
    scores_out: Optional[torch.Tensor] = None   # float [Hkv * sum NC_b][G], filled if given

    def c_struct(self, events=None) -> WiDecodeParams:
        sig = (self.n_q_heads, self.n_sink, self.window, self.topk_clusters, self.topk_fraction,
               self.exact_only, self.sampled, self.seed)
        plain = events is None and self.scores_out is None
        if plain and getattr(self, "_cs_sig", None) == sig:
            return self._cs
        p = WiDecodeParams()
        p.n_q_heads, p.n_sink, p.window = self.n_q_heads, self.n_sink, self.window
        p.topk_clusters, p.topk_fraction = self.topk_clusters, self.topk_fraction
        p.exact_only = 1 if self.exact_only else 0
        p.topk_mode = WI_TOPK_SAMPLED if self.sampled else WI_TOPK_EXACT
        p.seed = int(self.seed) & 0xFFFFFFFF
        if self.scores_out is not None:
            assert self.scores_out.dtype == torch.float32 and self.scores_out.is_contiguous()
            p.scores_out = self.scores_out.data_ptr()
        if events is not None:
            for e in events:
                if not e.cuda_event:      # torch creates the CUDA event on first record
                    e.record()
            arr = (C.c_void_p * len(events))(*[e.cuda_event for e in events])
            p.stage_events = C.cast(arr, C.POINTER(C.c_void_p))
            p._keep = arr
        if plain:
            self._cs, self._cs_sig = p, sig
        return p


def decode_layout(index: WaveIndex, params: DecodeParams) -> WiDecodeLayout:
    lay = WiDecodeLayout()
    ix, p = index.c_struct(), params.c_struct()
    _check(_lib.wi_decode_workspace_layout(C.byref(ix), C.byref(p), C.byref(lay)),
           "wi_decode_workspace_layout")
    return lay


def decode_workspace(index: WaveIndex, params: DecodeParams) -> torch.Tensor:
    return workspace(decode_layout(index, params).total_bytes, index.centroids.device)


def stage_names() -> List[str]:
    return [_lib.wi_decode_stage_name(i).decode() for i in range(_lib.wi_decode_stage_count())]


def decode(q: torch.Tensor, index: WaveIndex, params: DecodeParams,
           out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
           ws: Optional[torch.Tensor] = None, stream=None, stage_events=None):
    """One decode step: q [B][Hq][d] (KV dtype, on the GPU) -> out [B][Hq][d] fp32, lse [B][Hq]."""
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = decode_workspace(index, params)
    ix, p = index.c_struct(), params.c_struct(stage_events)
    _check(_lib.wi_decode(_ptr(q), C.byref(ix), C.byref(p), _ptr(out), _ptr(lse), _ptr(ws),
                          ws.numel(), _stream_ptr(stream)), "wi_decode")
    return out, lse


def decode_host(q_host: torch.Tensor, index: WaveIndex, params: DecodeParams,
                out_host: torch.Tensor, lse_host: Optional[torch.Tensor], ws: torch.Tensor,
                stream=None):
    """Decode from host q into host out/lse (copies on the stream; pin the
    host tensors for asynchronous copies).  Does not synchronise."""
    ix, p = index.c_struct(), params.c_struct()
    _check(_lib.wi_decode_host(_ptr(q_host), C.byref(ix), C.byref(p), _ptr(out_host),
                               _ptr(lse_host), _ptr(ws), ws.numel(), _stream_ptr(stream)),
           "wi_decode_host")


NOALLOC_SCRATCH_MIB = 32


def decode_noalloc(q: torch.Tensor, index: WaveIndex, params: DecodeParams,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   stream=None):
    """Decode with the library's fixed device scratch instead of a workspace.

    For callers that cannot allocate device memory where they decode (inside a
    stream capture, under a fixed memory arena, or from a runtime without an
    allocator).  Pass preallocated out / lse to allocate nothing at all.  Calls
    share one scratch array: do not overlap them on the GPU.  The first call on
    a device looks up the scratch address; make it before any stream capture.
    """
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    ix, p = index.c_struct(), params.c_struct()
    _check(_lib.wi_decode_noalloc(_ptr(q), C.byref(ix), C.byref(p), _ptr(out), _ptr(lse),
                                  _stream_ptr(stream)), "wi_decode_noalloc")
    return out, lse


def read_device_status(ws: torch.Tensor, stream=None, clear: bool = True) -> int:
    """Synchronise and return the WI_DEV_* bits set by kernels in this workspace."""
    flags = C.c_uint32()
    st = _lib.wi_read_device_status(_ptr(ws), _stream_ptr(stream), C.byref(flags), int(clear))
    if st not in (WI_OK, WI_ERR_DEVICE_CHECK):
        _check(st, "wi_read_device_status")
    return flags.value


# ---------------------------------------------------------------- workspace views

def unit_info(ws: torch.Tensor, layout: WiDecodeLayout, n_units: int) -> torch.Tensor:
    """Per-unit record from a decode workspace (int32 [U][info_ints]):
    {sel_count, thr_key, thr_idx, sel_tokens, steady, n_affected, dense,
    candidates, full_rows, partial_rows, non_candidates, no_estimate, mode,
    threshold_bin, draw_hi, draw_lo}."""
    n = layout.info_ints
    return ws[layout.unit_info:layout.unit_info + n_units * n * 4].view(torch.int32).view(n_units, n)


def selected_clusters(ws: torch.Tensor, layout: WiDecodeLayout, index: WaveIndex,
                      b: int, h: int, count: int) -> torch.Tensor:
    """The retrieved clusters of unit (b, h), ascending: the first `count`
    entries of the unit's rows of the workspace's selection list (rows laid
    out like the centroids)."""
    row = index.cl_row(b, h)
    if count < 0 or count > index.nc[b]:
        raise RuntimeError(f"selection count {count} outside [0, {index.nc[b]}]")
    ids = ws[layout.selected:].view(torch.int32)[row:row + count].clone()
    if count > 1 and not bool(torch.all(ids[1:] > ids[:-1])):
        raise RuntimeError("selection list is not ascending")
    return ids


def selection_keys(ws: torch.Tensor, layout: WiDecodeLayout, index: WaveIndex,
                   b: int, h: int) -> torch.Tensor:
    """The order-preserving selection keys of unit (b, h)'s clusters (uint32
    values in an int64 tensor; 0 = not a candidate)."""
    row = index.cl_row(b, h)
    n = index.nc[b]
    rec = ws[layout.records:].view(torch.int32)[2 * row:2 * (row + n)].view(n, 2)
    return rec[:, 0].to(torch.int64) & 0xFFFFFFFF


def scores_buffer(index: WaveIndex, n_q_heads: int) -> torch.Tensor:
    """A float [Hkv * sum NC_b][G] buffer for DecodeParams.scores_out."""
    G = n_q_heads // index.n_kv_heads
    return torch.zeros(index.n_kv_heads * sum(index.nc), G, dtype=torch.float32,
                       device=index.centroids.device)


def centroid_scores(scores: torch.Tensor, index: WaveIndex, b: int, h: int) -> torch.Tensor:
    """fp32 scores [NC_b][G] of unit (b, h) from a scores_out buffer."""
    row = index.cl_row(b, h)
    return scores[row:row + index.nc[b]]

// C ABI of libwi.so: argument validation, launch plans, workspace layout.
// Every argument error is detected here, on the host, before any CUDA call.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <map>
#include <tuple>
#include <vector>
#include <algorithm>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "wi.h"
#include "wi_common.cuh"
#include "wi_plan.h"

namespace wi {
namespace {

thread_local char g_last_error[256] = "";

wi_status cuda_fail(cudaError_t e) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return WI_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
int ilog2(int x) { int r = 0; while ((1 << r) < x) ++r; return r; }
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

int64_t clusters_of(int64_t T, int S, int cs) {
  const int64_t full = T / S, rem = T % S;
  return full * (S / cs) + cdiv(rem, cs);
}

int esize(wi_dtype d) { return d == WI_BF16 ? 2 : 4; }

// Common geometry checks for a paged pool description.
wi_status check_common(wi_dtype dtype, int batch, int hkv, int d, int page, int64_t n_pages,
                       const void* kp, const void* vp, const int32_t* bt, int max_pages,
                       const int32_t* seq_lens) {
  if (dtype != WI_F32 && dtype != WI_BF16) return WI_ERR_INVALID_ARG;
  if (batch < 1 || hkv < 1 || d < 1 || page < 1 || n_pages < 1 || max_pages < 1)
    return WI_ERR_INVALID_ARG;
  if (batch > kMaxBatch) return WI_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return WI_ERR_UNSUPPORTED;
  if (!pow2(page) || page > 1024) return WI_ERR_INVALID_ARG;
  if (!kp || !vp || !bt || !seq_lens) return WI_ERR_INVALID_ARG;
  if (!aligned(kp, 16) || !aligned(vp, 16) || !aligned(bt, 4)) return WI_ERR_INVALID_ARG;
  int64_t tot = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t T = seq_lens[b];
    if (T < 1) return WI_ERR_INVALID_ARG;
    if (cdiv(T, page) > max_pages) return WI_ERR_INVALID_ARG;
    tot += T;
  }
  if (tot * hkv > INT32_MAX) return WI_ERR_UNSUPPORTED;
  return WI_OK;
}

wi_status check_seg(int S, int cs) {
  if (S < 1 || cs < 1 || S % cs != 0) return WI_ERR_INVALID_ARG;
  if (S > WI_MAX_SEG_LEN) return WI_ERR_UNSUPPORTED;
  return WI_OK;
}

void fill_geo(Geo& g, int batch, int hkv, int d, const int32_t* seq_lens, int S, int cs) {
  std::memset(&g, 0, sizeof(g));
  g.batch = batch; g.hkv = hkv; g.d = d;
  for (int b = 0; b < batch; ++b) {
    g.tok_base[b + 1] = g.tok_base[b] + seq_lens[b];
    g.cl_base[b + 1] = g.cl_base[b] + (int32_t)clusters_of(seq_lens[b], S, cs);
  }
}

int64_t n_steady(int64_t T, int64_t n_sink, int64_t window) {
  const int64_t ns = std::min(n_sink, T);
  const int64_t ws = std::max(T - window, ns);
  return ns + (T - ws);
}


// Chunk map of the scan: CTA that takes chunk k of n over N CTAs

// The scan CTAs' chunk runs (pl.k0s).  The last `late` CTAs are launched
// beside the steady kernel's U CTAs and start once those have left their
// SMs: they take a share of weight 3 against 5 (when there are chunks enough
// for every CTA to keep one).  With up to 32 units (and no more units than
// CTAs) the runs are unit-aligned: unit u gets c_u CTAs of its own, its
// chunks split over them by weight, and the c_u are moved one at a time
// from the unit that loses least to the unit with the latest predicted
// finish (a CTA's predicted finish, in chunk times: its share of its unit's
// chunks, plus 3 for a late CTA) while the latest finish drops, so no CTA
// ends one unit and starts another in the middle of its run.  Otherwise CTA
// s takes chunks [n W(s) / W(N), n W(s + 1) / W(N)), W the prefix of the
// weights.  The runs are kept by geometry.
void balance_scan(DecodePlan& pl) {
  const int n = pl.n_chunks, N = pl.n_scan, H = pl.geo.hkv, B = pl.geo.batch;
  pl.k0s[0] = 0;
  for (int s = 1; s <= kNumSMs; ++s) pl.k0s[s] = n;
  if (n <= 0) return;
  const int late = n >= 2 * N ? std::min(pl.U, N / 4) : 0;
  auto weighted = [&]() {
    const int a = N - late;
    auto ws = [&](int s) -> uint64_t { return s <= a ? 5ull * s : 5ull * a + 3ull * (uint64_t)(s - a); };
    for (int s = 0; s <= N; ++s) pl.k0s[s] = (int32_t)((uint64_t)n * ws(s) / ws(N));
  };
  std::vector<int> uf, um;   // the units with chunks: first chunk, chunks
  for (int b = 0; b < B; ++b) {
    const int per = (pl.ch_base[b + 1] - pl.ch_base[b]) / H;
    for (int h = 0; h < H && per > 0; ++h) {
      uf.push_back(pl.ch_base[b] + h * per);
      um.push_back(per);
    }
  }
  const int Uu = (int)uf.size();
  if (Uu == 0 || Uu > 32 || Uu > N) {
    weighted();
    return;
  }
  using Key = std::tuple<std::vector<int32_t>, int, int, int>;
  static std::mutex mu;
  static std::map<Key, std::vector<int32_t>> memo;
  Key key{std::vector<int32_t>(pl.ch_base, pl.ch_base + B + 1), H, N, late};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = memo.find(key);
    if (it != memo.end()) {
      std::copy(it->second.begin(), it->second.end(), pl.k0s);
      return;
    }
  }
  // CTAs per unit, first in proportion to its chunks
  std::vector<int> c(Uu);
  int sum = 0;
  for (int i = 0; i < Uu; ++i) {
    c[i] = std::max(1, (int)std::lround((double)N * um[i] / n));
    sum += c[i];
  }
  while (sum > N) {
    int i = 0;
    for (int j = 1; j < Uu; ++j) if (c[j] > c[i]) i = j;
    --c[i];
    --sum;
  }
  while (sum < N) {
    int i = 0;
    for (int j = 1; j < Uu; ++j) if ((double)um[j] / c[j] > (double)um[i] / c[i]) i = j;
    ++c[i];
    ++sum;
  }
  // each unit's late CTAs (the last `late` of all), its predicted finish,
  // and whether every CTA keeps a chunk
  std::vector<double> cost(Uu);
  auto evaluate = [&](const std::vector<int>& cc, double* worst) {
    int F = 0;
    *worst = 0.0;
    bool ok = true;
    for (int i = 0; i < Uu; ++i) {
      const int nl = std::max(0, std::min(F + cc[i], N) - std::max(F, N - late));
      const int nn = cc[i] - nl;
      const double W = 5.0 * nn + 3.0 * nl;
      double r = 0.0;
      if (nn > 0) r = um[i] * 5.0 / W;
      if (nl > 0) r = std::max(r, 3.0 + um[i] * 3.0 / W);
      cost[i] = r;
      *worst = std::max(*worst, r);
      if (cc[i] > um[i] || (nl > 0 && um[i] * 3.0 / W < 1.0) || (nn > 0 && um[i] * 5.0 / W < 1.0))
        ok = false;
      F += cc[i];
    }
    return ok;
  };
  double worst;
  if (!evaluate(c, &worst)) {
    weighted();
    return;
  }
  for (int it = 0; it < 8 * N; ++it) {
    int imax = 0;
    for (int i = 1; i < Uu; ++i) if (cost[i] > cost[imax]) imax = i;
    double best = worst;
    int bj = -1;
    for (int j = 0; j < Uu; ++j) {
      if (j == imax || c[j] <= 1) continue;
      std::vector<int> c2 = c;
      --c2[j];
      ++c2[imax];
      double w2;
      if (evaluate(c2, &w2) && w2 < best - 1e-9) {
        best = w2;
        bj = j;
      }
    }
    if (bj < 0) break;
    --c[bj];
    ++c[imax];
    evaluate(c, &worst);
  }
  std::vector<int32_t> tab(N + 1);
  int s = 0;
  for (int i = 0; i < Uu; ++i) {
    const int F = s;
    uint64_t W = 0;
    for (int j = 0; j < c[i]; ++j) W += F + j >= N - late ? 3 : 5;
    uint64_t acc = 0;
    for (int j = 0; j < c[i]; ++j) {
      tab[s++] = uf[i] + (int32_t)((uint64_t)um[i] * acc / W);
      acc += F + j >= N - late ? 3 : 5;
    }
  }
  tab[N] = n;
  bool ok = s == N && tab[0] == 0;
  for (int t = 0; t < N && ok; ++t) ok = tab[t] < tab[t + 1];
  if (!ok) {
    weighted();
    return;
  }
  std::copy(tab.begin(), tab.end(), pl.k0s);
  std::lock_guard<std::mutex> lock(mu);
  if (memo.size() >= 256) memo.clear();
  memo[key] = tab;
}

wi_status make_decode_plan(const wi_index* ix, const wi_decode_params* p, DecodePlan& pl) {
  if (!ix || !p) return WI_ERR_INVALID_ARG;
  wi_status st = check_common(ix->dtype, ix->batch, ix->n_kv_heads, ix->head_dim, ix->page_size,
                              ix->n_pages, ix->k_pool, ix->v_pool, ix->block_table,
                              ix->max_pages, ix->seq_lens);
  if (st != WI_OK) return st;
  if ((st = check_seg(ix->seg_len, ix->cluster_size)) != WI_OK) return st;
  if (!ix->centroids || !ix->value_sums || !ix->offsets || !ix->perm || !ix->invperm ||
      !ix->labels)
    return WI_ERR_INVALID_ARG;
  if (!aligned(ix->centroids, 16) || !aligned(ix->value_sums, 16) || !aligned(ix->offsets, 4) ||
      !aligned(ix->perm, 4) || !aligned(ix->invperm, 4) || !aligned(ix->labels, 4))
    return WI_ERR_INVALID_ARG;
  if (p->n_q_heads < 1 || p->n_q_heads % ix->n_kv_heads != 0) return WI_ERR_INVALID_ARG;
  if (ix->n_pages * ix->n_kv_heads * ix->page_size >= INT32_MAX) return WI_ERR_UNSUPPORTED;
  const int G = p->n_q_heads / ix->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return WI_ERR_UNSUPPORTED;
  if (p->n_sink < 0 || p->window < 0) return WI_ERR_INVALID_ARG;
  if (p->topk_clusters < 0 && !(p->topk_fraction >= 0.0 && p->topk_fraction <= 1.0))
    return WI_ERR_INVALID_ARG;
  if (p->topk_mode != WI_TOPK_EXACT && p->topk_mode != WI_TOPK_SAMPLED) return WI_ERR_INVALID_ARG;
  if (p->scores_out && !aligned(p->scores_out, 4)) return WI_ERR_INVALID_ARG;

  std::memset(&pl, 0, sizeof(pl));
  fill_geo(pl.geo, ix->batch, ix->n_kv_heads, ix->head_dim, ix->seq_lens, ix->seg_len,
           ix->cluster_size);
  const int B = ix->batch, H = ix->n_kv_heads;
  pl.dtype = ix->dtype; pl.D = ix->head_dim; pl.G = G; pl.Hq = p->n_q_heads;
  pl.U = B * H;
  pl.n_sink = p->n_sink; pl.window = p->window;
  pl.topk_clusters = p->topk_clusters; pl.topk_fraction = p->topk_fraction;
  pl.exact_only = p->exact_only != 0;
  pl.mode = p->topk_mode;
  pl.seed = p->seed;
  pl.scale = 1.0f / std::sqrt((float)ix->head_dim);

  int max_nc = 0, cap = 1;
  bool dense[kMaxBatch];
  int nst[kMaxBatch];
  for (int b = 0; b < B; ++b) {
    const int T = ix->seq_lens[b];
    max_nc = std::max(max_nc, pl.geo.NC(b));
    const int64_t n = n_steady(T, p->n_sink, p->window);
    dense[b] = n >= T;
    nst[b] = (int)std::min<int64_t>(n, T);
    if (!dense[b]) {   // not attended densely: its steady list is kept
      if (n > WI_MAX_STEADY) return WI_ERR_UNSUPPORTED;
      cap = std::max<int>(cap, (int)n);
    }
  }
  pl.max_nc = max_nc;
  pl.cap = cap;
  pl.ncl = (int64_t)pl.geo.cl_base[B] * H;
  pl.ntok = (int64_t)pl.geo.tok_base[B] * H;

  // scan: chunks of kTileRows clusters of every unit that is not dense,
  // contiguous runs of them per CTA, one CTA per SM at most
  pl.ch_base[0] = 0;
  for (int b = 0; b < B; ++b) {
    const int nch = dense[b] ? 0 : (int)cdiv(pl.geo.NC(b), kTileRows);
    pl.ch_base[b + 1] = pl.ch_base[b] + H * nch;
  }
  pl.n_chunks = pl.ch_base[B];
  pl.n_scan = std::max(1, std::min(pl.n_chunks, kNumSMs));
  balance_scan(pl);
  const ChunkMap cm = chunk_map(pl);
  pl.p1max = 1;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H && cm.per_unit(b) > 0; ++h) pl.p1max = std::max(pl.p1max, cm.parts(b, h));
  // units a scan CTA touches (it runs the tails of those it finishes last)
  for (int sc = 0; sc < pl.n_scan && pl.n_chunks > 0; ++sc) {
    const int k0 = cm.k0(sc), k1 = cm.k0(sc + 1);
    int touched = 0;
    for (int k = k0; k < k1;) {
      const int b = cm.seq_of(k), per = cm.per_unit(b);
      const int h = (k - cm.ch_base[b]) / per;
      if (++touched > kMaxTailsPerCta) return WI_ERR_UNSUPPORTED;
      k = std::min(k1, cm.first(b, h) + per);   // past the unit's last chunk in this CTA's range
    }
  }
  // ring slots: tile(s) plus the side area (offsets box, queries); about
  // 144 KB of them, 2 to 4
  const size_t slot = decode_scan_slot_bytes(pl.dtype, pl.D, G, pl.exact_only);
  pl.slots = (int)std::max<size_t>(2, std::min<size_t>(4, (size_t)147456 / slot));
  if (decode_scan_smem(pl.dtype, pl.D, G, pl.slots, pl.exact_only) > 227 * 1024)
    return WI_ERR_UNSUPPORTED;
  if (decode_gather_smem(pl.dtype, pl.D, G) > 227 * 1024) return WI_ERR_UNSUPPORTED;
  if (decode_steady_smem(cap) > 96 * 1024) return WI_ERR_UNSUPPORTED;

  // gather: per sequence, CTAs for the rows the unit is expected to hold
  // (retrieved tokens at cluster_size each, steady tokens, and the rows taken
  // out of the estimate), kGatherTiles tiles each; they loop over more
  const int rpb = kGatherTiles * kTileRows;
  pl.n2_base[0] = 0;
  pl.n2max = 1;
  for (int b = 0; b < B; ++b) {
    const int T = ix->seq_lens[b], NC = pl.geo.NC(b);
    int64_t rows;
    if (dense[b]) {
      rows = T;
    } else {
      const int64_t kr = p->topk_clusters >= 0 ? p->topk_clusters
                                               : (int64_t)std::ceil(p->topk_fraction * (double)NC);
      const int64_t k = std::min<int64_t>(std::max<int64_t>(kr, 0), NC);
      rows = std::min<int64_t>(k * ix->cluster_size, T) + nst[b];
      if (!pl.exact_only) rows += k + nst[b];
    }
    // half as many again as expected: the clusters a query retrieves run
    // larger than the average cluster (a third larger at the 131072-token
    // workload), and a CTA that loops over a second block holds up the
    // unit's merge
    rows += rows / 2;
    const int n2 = (int)std::max<int64_t>(1, std::min<int64_t>(cdiv(rows, rpb), kMaxGatherPerUnit));
    pl.n2_base[b + 1] = pl.n2_base[b] + H * n2;
    pl.n2max = std::max(pl.n2max, n2);
  }
  pl.n_gather = pl.n2_base[B];

  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t r = o; o = align_up(o + bytes, 256); return r; };
  const size_t PS = (size_t)G * (pl.D + 4) * 4;   // one part: G heads of {m, l, -, -, o[D]}
  pl.off_status = take(256);
  pl.off_cnt1 = take((size_t)pl.U * 4);
  pl.off_cnt2 = take((size_t)pl.U * 4);
  pl.off_hist = take((size_t)pl.U * kHistBins * 4);   // zeroed after use by the tails
  pl.off_rec = take((size_t)pl.ncl * 8);
  pl.off_info = take((size_t)pl.U * kInfoInts * 4);
  pl.off_st_slot = take((size_t)pl.U * cap * 4);
  pl.off_pc = take((size_t)pl.U * cap * 8);
  pl.off_nonc = take((size_t)pl.U * cap * 8);
  pl.off_sel = take((size_t)pl.ncl * 4);
  pl.off_tok = take((size_t)pl.ntok * 4);
  pl.off_selinfo = take((size_t)pl.ncl * 16);
  pl.off_est = take(pl.exact_only ? 0 : (size_t)pl.U * pl.p1max * PS);
  pl.off_gat = take((size_t)pl.U * pl.n2max * PS);
  const size_t nq = (size_t)B * p->n_q_heads;
  pl.off_q = take(nq * pl.D * esize(ix->dtype));
  pl.off_out = take(nq * pl.D * 4);
  pl.off_lse = take(nq * 4);
  pl.total = o;
  return WI_OK;
}

wi_status check_ws(const void* ws, size_t have, size_t need) {
  if (!ws || !aligned(ws, 256) || have < need) return WI_ERR_WORKSPACE;
  return WI_OK;
}

wi_status make_build_plan(const wi_kv_cache* kv, int S, int cs, BuildPlan& pl) {
  if (!kv) return WI_ERR_INVALID_ARG;
  wi_status st = check_common(kv->dtype, kv->batch, kv->n_kv_heads, kv->head_dim, kv->page_size,
                              kv->n_pages, kv->k_pool, kv->v_pool, kv->block_table,
                              kv->max_pages, kv->seq_lens);
  if (st != WI_OK) return st;
  if ((st = check_seg(S, cs)) != WI_OK) return st;
  std::memset(&pl, 0, sizeof(pl));
  fill_geo(pl.geo, kv->batch, kv->n_kv_heads, kv->head_dim, kv->seq_lens, S, cs);
  pl.dtype = kv->dtype; pl.D = kv->head_dim; pl.U = kv->batch * kv->n_kv_heads;
  pl.S = S; pl.cs = cs;
  int max_nseg = 0;
  for (int b = 0; b < kv->batch; ++b) max_nseg = std::max<int>(max_nseg, (int)cdiv(kv->seq_lens[b], S));
  pl.max_nseg = max_nseg;
  pl.nseg_grid = max_nseg;   // every segment from the first (sf zero)
  pl.max_ncl_seg = S / cs;
  pl.update_smem = (size_t)(2 * pl.max_ncl_seg + 1 + 32) * 4 + (size_t)S * 2 * 2;
  const int64_t ncl = (int64_t)pl.geo.cl_base[kv->batch] * kv->n_kv_heads;
  const int64_t ntok = (int64_t)pl.geo.tok_base[kv->batch] * kv->n_kv_heads;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t r = o; o = align_up(o + bytes, 256); return r; };
  pl.off_status = take(256);
  pl.off_cent32 = take((size_t)ncl * pl.D * 4);
  pl.off_assign = take((size_t)ntok * 4);
  // bf16 keys: per (unit, segment), the two bf16 terms of each chunk of
  // 128 centroids as operand tiles, and the centroids' squared norms
  pl.nch = (int)cdiv(pl.max_ncl_seg, 128);
  const size_t nchunks = (size_t)pl.U * max_nseg * pl.nch;
  if (pl.dtype == WI_BF16) {
    pl.off_cimg = take(nchunks * 2 * 128 * pl.D * 2);
    pl.off_cn2 = take(nchunks * 128 * 4);
  }
  pl.total = o;
  return WI_OK;
}

Pool make_pool(const void* base, const int32_t* bt, int64_t n_pages, int max_pages, int page) {
  return Pool{base, bt, n_pages, max_pages, ilog2(page)};
}

// Host-buffer decodes replayed from CUDA graphs: the copy of q in, the
// decode's kernels and the copies of out and lse back, captured once a call
// with the same key (every pointer, size and option the launches bake in)
// is seen a second time, then launched as one graph.  A call on the legacy
// default stream, on a stream that is being captured, with pageable host
// buffers or with stage events or score output enqueues its work directly.
struct HostGraphs {
  std::mutex mu;
  struct Entry {
    cudaGraphExec_t exec;
    uint64_t used;
  };
  std::map<std::vector<int64_t>, Entry> graphs;
  std::map<std::vector<int64_t>, int> seen;
  uint64_t tick = 0;
};
HostGraphs& host_graphs() {
  static HostGraphs* g = new HostGraphs;   // (left to the process's exit)
  return *g;
}
constexpr size_t kMaxHostGraphs = 16;

// The device address of a pinned, device-mapped host buffer, else null.
void* mapped_device_ptr(const void* ptr) {
  if (!ptr) return nullptr;
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, ptr) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

bool host_pinned(const void* ptr) {
  if (!ptr) return true;
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, ptr) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeHost;
}

// The current context's id (unique for the process's life, so a graph of a
// context that a device reset destroyed is never handed to its successor);
// 0 when it cannot be read (the call then enqueues its work directly).
unsigned long long current_context_id() {
  static std::once_flag once;
  static PFN_cuCtxGetCurrent_v4000 get_ctx = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_ctx = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_ctx || !get_id || get_ctx(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

std::vector<int64_t> host_graph_key(unsigned long long ctx_id, const wi_index* ix,
                                    const wi_decode_params* p, const void* ws, size_t ws_bytes,
                                    const void* q_host, const float* out_host, const float* lse_host) {
  auto ptr = [](const void* x) { return (int64_t)reinterpret_cast<intptr_t>(x); };
  double frac = p->topk_fraction;
  int64_t frac_bits = 0;
  std::memcpy(&frac_bits, &frac, sizeof(frac_bits));
  std::vector<int64_t> k = {(int64_t)ctx_id, ptr(ws), (int64_t)ws_bytes, ptr(q_host), ptr(out_host),
                            ptr(lse_host), ix->dtype, ix->batch, ix->n_kv_heads, ix->head_dim,
                            ix->page_size, ix->seg_len, ix->cluster_size, ptr(ix->centroids),
                            ptr(ix->value_sums), ptr(ix->offsets), ptr(ix->perm), ptr(ix->invperm),
                            ptr(ix->labels), ptr(ix->k_pool), ptr(ix->v_pool), ix->n_pages,
                            ptr(ix->block_table), ix->max_pages, p->n_q_heads, p->n_sink, p->window,
                            p->topk_clusters, frac_bits, p->exact_only, p->topk_mode, p->seed};
  for (int b = 0; b < ix->batch; ++b) k.push_back(ix->seq_lens[b]);
  return k;
}

wi_status decode_impl(const void* q, const wi_index* ix, const wi_decode_params* p, float* out,
                      float* lse, void* ws, size_t ws_bytes, cudaStream_t s, const void* q_host,
                      float* out_host, float* lse_host) {
  DecodePlan pl;
  wi_status st = make_decode_plan(ix, p, pl);
  if (st != WI_OK) return st;
  const bool host = q_host != nullptr || out_host != nullptr;
  if (host) {
    if (!q_host || !out_host) return WI_ERR_INVALID_ARG;
  } else {
    if (!q || !out || !aligned(q, 16) || !aligned(out, 4) || (lse && !aligned(lse, 4)))
      return WI_ERR_INVALID_ARG;
  }
  if ((st = check_ws(ws, ws_bytes, pl.total)) != WI_OK) return st;
  unsigned char* w = static_cast<unsigned char*>(ws);
  const size_t nq = (size_t)ix->batch * p->n_q_heads;
  // out and lse: written by the kernels straight into the caller's host
  // buffers when both are pinned and device-mapped, else into the
  // workspace and copied back
  bool direct_out = false;
  bool outs_pinned = false;   // out_host and lse_host (if given) pinned and mapped
  if (host) {
    q = w + pl.off_q;
    float* out_dev = static_cast<float*>(mapped_device_ptr(out_host));
    float* lse_dev = static_cast<float*>(mapped_device_ptr(lse_host));
    direct_out = out_dev && (!lse_host || lse_dev);
    outs_pinned = direct_out;
    if (direct_out) {
      out = out_dev;
      lse = lse_dev;
    } else {
      out = reinterpret_cast<float*>(w + pl.off_out);
      lse = lse_host ? reinterpret_cast<float*>(w + pl.off_lse) : nullptr;
    }
  }
  DecodeArgs a{};
  a.q = q;
  a.centroids = ix->centroids;
  a.value_sums = ix->value_sums;
  a.offsets = ix->offsets;
  a.perm = ix->perm;
  a.invperm = ix->invperm;
  a.labels = ix->labels;
  a.kp = make_pool(ix->k_pool, ix->block_table, ix->n_pages, ix->max_pages, ix->page_size);
  a.vp = make_pool(ix->v_pool, ix->block_table, ix->n_pages, ix->max_pages, ix->page_size);
  a.out = out;
  a.lse = lse;
  a.ws = w;
  a.stage_events = reinterpret_cast<cudaEvent_t*>(p->stage_events);
  a.scores_out = p->scores_out;
  // the call's work on the stream: copies of the host buffers around the kernels
  auto enqueue = [&]() -> cudaError_t {
    cudaError_t e = cudaSuccess;
    if (host)
      e = cudaMemcpyAsync(const_cast<void*>(q), q_host, nq * pl.D * esize(ix->dtype),
                          cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = launch_decode(pl, a, s);
    if (e == cudaSuccess && host && !direct_out) {
      e = cudaMemcpyAsync(out_host, out, nq * pl.D * 4, cudaMemcpyDeviceToHost, s);
      if (e == cudaSuccess && lse_host)
        e = cudaMemcpyAsync(lse_host, lse, nq * 4, cudaMemcpyDeviceToHost, s);
    }
    return e;
  };
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  const bool graphable = host && s != nullptr && s != cudaStreamLegacy && !p->stage_events &&
                         !p->scores_out && cudaStreamIsCapturing(s, &cap) == cudaSuccess &&
                         cap == cudaStreamCaptureStatusNone && host_pinned(q_host) && outs_pinned;
  const unsigned long long ctx_id = graphable ? current_context_id() : 0;
  if (graphable && ctx_id != 0) {
    HostGraphs& hg = host_graphs();
    std::vector<int64_t> key = host_graph_key(ctx_id, ix, p, ws, ws_bytes, q_host, out_host, lse_host);
    key.push_back(direct_out ? 1 : 0);
    cudaGraphExec_t exec = nullptr;
    bool capture = false;
    {
      std::lock_guard<std::mutex> lock(hg.mu);
      auto it = hg.graphs.find(key);
      if (it != hg.graphs.end()) {
        exec = it->second.exec;
        it->second.used = ++hg.tick;
      } else {
        if (hg.seen.size() >= 1024) hg.seen.clear();
        capture = ++hg.seen[key] >= 2;
      }
    }
    if (!exec && capture) {
      cudaGraph_t graph = nullptr;
      cudaError_t e = cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal);
      if (e == cudaSuccess) {
        const cudaError_t e1 = enqueue();
        e = cudaStreamEndCapture(s, &graph);
        if (e == cudaSuccess) e = e1;
      }
      if (e == cudaSuccess && graph) e = cudaGraphInstantiate(&exec, graph, 0);
      if (graph) cudaGraphDestroy(graph);
      if (e != cudaSuccess) {
        cudaGetLastError();
        exec = nullptr;   // (this call enqueues its work directly)
      } else {
        std::lock_guard<std::mutex> lock(hg.mu);
        if (hg.graphs.size() >= kMaxHostGraphs) {   // the least recently used leaves
          auto lru = hg.graphs.begin();
          for (auto it = hg.graphs.begin(); it != hg.graphs.end(); ++it)
            if (it->second.used < lru->second.used) lru = it;
          cudaGraphExecDestroy(lru->second.exec);
          hg.graphs.erase(lru);
        }
        hg.graphs[key] = HostGraphs::Entry{exec, ++hg.tick};
      }
    }
    if (exec) {
      const cudaError_t e = cudaGraphLaunch(exec, s);
      return e == cudaSuccess ? WI_OK : cuda_fail(e);
    }
  }
  const cudaError_t e = enqueue();
  return e == cudaSuccess ? WI_OK : cuda_fail(e);
}

}  // namespace

// Total workspace bytes of a decode call and the length of its leading
// region that must be zero when a call starts (status word, merge counters,
// selection histogram).  Host only.
wi_status decode_workspace_extent(const wi_index* idx, const wi_decode_params* p, size_t* total,
                                  size_t* zero_prefix) {
  DecodePlan pl;
  const wi_status st = make_decode_plan(idx, p, pl);
  if (st != WI_OK) return st;
  *total = pl.total;
  *zero_prefix = pl.off_rec;
  return WI_OK;
}

}  // namespace wi

namespace wi {
namespace {
// Checks of an index that a build writes, against the KV cache it is built from.
wi_status check_build_out(const wi_kv_cache* kv, int32_t seg_len, int32_t cluster_size,
                          const wi_index* out) {
  if (!out) return WI_ERR_INVALID_ARG;
  wi_status st;
  if (out->dtype != kv->dtype || out->batch != kv->batch || out->n_kv_heads != kv->n_kv_heads ||
      out->head_dim != kv->head_dim || out->page_size != kv->page_size ||
      out->seg_len != seg_len || out->cluster_size != cluster_size || !out->seq_lens)
    return WI_ERR_INVALID_ARG;
  for (int b = 0; b < kv->batch; ++b)
    if (out->seq_lens[b] != kv->seq_lens[b]) return WI_ERR_INVALID_ARG;
  st = check_common(out->dtype, out->batch, out->n_kv_heads, out->head_dim, out->page_size,
                    out->n_pages, out->k_pool, out->v_pool, out->block_table, out->max_pages,
                    out->seq_lens);
  if (st != WI_OK) return st;
  if (!out->centroids || !out->value_sums || !out->offsets || !out->perm || !out->invperm ||
      !out->labels)
    return WI_ERR_INVALID_ARG;
  if (!aligned(out->centroids, 16) || !aligned(out->value_sums, 16) || !aligned(out->offsets, 4) ||
      !aligned(out->perm, 4) || !aligned(out->invperm, 4) || !aligned(out->labels, 4))
    return WI_ERR_INVALID_ARG;
  if (out->k_pool == kv->k_pool || out->v_pool == kv->v_pool || out->k_pool == kv->v_pool ||
      out->v_pool == kv->k_pool)
    return WI_ERR_INVALID_ARG;
  return WI_OK;
}

BuildArgs build_args(const wi_kv_cache* kv, const wi_index* out, void* ws) {
  BuildArgs a{};
  a.kin = make_pool(kv->k_pool, kv->block_table, kv->n_pages, kv->max_pages, kv->page_size);
  a.vin = make_pool(kv->v_pool, kv->block_table, kv->n_pages, kv->max_pages, kv->page_size);
  a.centroids = out->centroids;
  a.value_sums = out->value_sums;
  a.offsets = out->offsets;
  a.perm = out->perm;
  a.invperm = out->invperm;
  a.labels = out->labels;
  a.kout = out->k_pool;
  a.vout = out->v_pool;
  a.bt_out = out->block_table;
  a.n_pages_out = out->n_pages;
  a.max_pages_out = out->max_pages;
  a.page_shift_out = ilog2(out->page_size);
  a.ws = static_cast<unsigned char*>(ws);
  return a;
}
}  // namespace
}  // namespace wi

using namespace wi;

extern "C" {

wi_status wi_index_clusters(int32_t batch, const int32_t* seq_lens, int32_t seg_len,
                            int32_t cluster_size, int32_t* nc_out, int64_t* nc_total) {
  if (batch < 1 || !seq_lens || !nc_total) return WI_ERR_INVALID_ARG;
  wi_status st = check_seg(seg_len, cluster_size);
  if (st != WI_OK) return st;
  int64_t tot = 0;
  for (int b = 0; b < batch; ++b) {
    if (seq_lens[b] < 1) return WI_ERR_INVALID_ARG;
    const int64_t nc = clusters_of(seq_lens[b], seg_len, cluster_size);
    if (nc_out) nc_out[b] = (int32_t)nc;
    tot += nc;
  }
  *nc_total = tot;
  return WI_OK;
}

wi_status wi_build_workspace_size(const wi_kv_cache* kv, int32_t seg_len, int32_t cluster_size,
                                  size_t* bytes) {
  if (!bytes) return WI_ERR_INVALID_ARG;
  BuildPlan pl;
  wi_status st = make_build_plan(kv, seg_len, cluster_size, pl);
  if (st != WI_OK) return st;
  *bytes = pl.total;
  return WI_OK;
}


wi_status wi_build_workspace_layout(const wi_kv_cache* kv, int32_t seg_len,
                                    int32_t cluster_size, wi_build_layout* layout) {
  if (!layout) return WI_ERR_INVALID_ARG;
  BuildPlan pl;
  wi_status st = make_build_plan(kv, seg_len, cluster_size, pl);
  if (st != WI_OK) return st;
  layout->total_bytes = pl.total;
  layout->status = pl.off_status;
  layout->centroids_f32 = pl.off_cent32;
  layout->assign = pl.off_assign;
  return WI_OK;
}

wi_status wi_build_index(const wi_kv_cache* kv, int32_t seg_len, int32_t cluster_size,
                         int32_t iters, const wi_index* out, void* ws, size_t ws_bytes,
                         wi_stream_t stream) {
  BuildPlan pl;
  wi_status st = make_build_plan(kv, seg_len, cluster_size, pl);
  if (st != WI_OK) return st;
  if (iters < 1) return WI_ERR_INVALID_ARG;
  if ((st = check_build_out(kv, seg_len, cluster_size, out)) != WI_OK) return st;
  pl.iters = iters;
  if ((st = check_ws(ws, ws_bytes, pl.total)) != WI_OK) return st;
  const BuildArgs a = build_args(kv, out, ws);
  const cudaError_t e = launch_build(pl, a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WI_OK : cuda_fail(e);
}

wi_status wi_build_blocks(const wi_kv_cache* kv, int32_t seg_len, int32_t block_size,
                          const wi_index* out, void* ws, size_t ws_bytes, wi_stream_t stream) {
  BuildPlan pl;
  wi_status st = make_build_plan(kv, seg_len, block_size, pl);
  if (st != WI_OK) return st;
  if ((st = check_build_out(kv, seg_len, block_size, out)) != WI_OK) return st;
  pl.iters = 1;
  if ((st = check_ws(ws, ws_bytes, pl.total)) != WI_OK) return st;
  const BuildArgs a = build_args(kv, out, ws);
  const cudaError_t e = launch_blocks(pl, a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WI_OK : cuda_fail(e);
}

wi_status wi_extend_index(const wi_index* old_ix, const wi_kv_cache* kv, int32_t iters,
                          const wi_index* out, void* ws, size_t ws_bytes, wi_stream_t stream) {
  if (!old_ix || !kv || !out) return WI_ERR_INVALID_ARG;
  const int32_t S = out->seg_len, cs = out->cluster_size;
  BuildPlan pl;
  wi_status st = make_build_plan(kv, S, cs, pl);
  if (st != WI_OK) return st;
  if (iters < 1) return WI_ERR_INVALID_ARG;
  if ((st = check_build_out(kv, S, cs, out)) != WI_OK) return st;
  // the old index: same geometry, no sequence longer than now
  if (old_ix->dtype != kv->dtype || old_ix->batch != kv->batch ||
      old_ix->n_kv_heads != kv->n_kv_heads || old_ix->head_dim != kv->head_dim ||
      old_ix->page_size != kv->page_size || old_ix->seg_len != S || old_ix->cluster_size != cs ||
      !old_ix->seq_lens || !old_ix->centroids || !old_ix->value_sums || !old_ix->offsets ||
      !old_ix->perm || !old_ix->invperm || !old_ix->labels)
    return WI_ERR_INVALID_ARG;
  if (!aligned(old_ix->centroids, 16) || !aligned(old_ix->value_sums, 16))
    return WI_ERR_INVALID_ARG;
  if (old_ix->centroids == out->centroids || old_ix->value_sums == out->value_sums ||
      old_ix->offsets == out->offsets || old_ix->perm == out->perm ||
      old_ix->invperm == out->invperm || old_ix->labels == out->labels)
    return WI_ERR_INVALID_ARG;
  for (int b = 0; b < kv->batch; ++b)
    if (old_ix->seq_lens[b] < 1 || old_ix->seq_lens[b] > kv->seq_lens[b]) return WI_ERR_INVALID_ARG;
  ExtendCopy c{};
  fill_geo(c.gold, old_ix->batch, old_ix->n_kv_heads, old_ix->head_dim, old_ix->seq_lens, S, cs);
  c.centroids = old_ix->centroids;
  c.value_sums = old_ix->value_sums;
  c.offsets = old_ix->offsets;
  c.perm = old_ix->perm;
  c.invperm = old_ix->invperm;
  c.labels = old_ix->labels;
  // whole segments of the old index are kept; from its first incomplete one
  // (or the first new one) on, segments are clustered anew
  int nseg_grid = 0;
  for (int b = 0; b < kv->batch; ++b) {
    pl.sf.s0[b] = old_ix->seq_lens[b] / S;
    nseg_grid = std::max<int>(nseg_grid, (int)cdiv(kv->seq_lens[b], S) - pl.sf.s0[b]);
  }
  pl.nseg_grid = nseg_grid;
  pl.iters = iters;
  if ((st = check_ws(ws, ws_bytes, pl.total)) != WI_OK) return st;
  const BuildArgs a = build_args(kv, out, ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_extend_copy(pl, c, a, s);
  if (e == cudaSuccess) e = launch_build(pl, a, s);
  return e == cudaSuccess ? WI_OK : cuda_fail(e);
}

wi_status wi_kmeans_assign(const wi_kv_cache* kv, int32_t seg_len, int32_t cluster_size,
                           const float* centroids, int32_t* assign, void* ws, size_t ws_bytes,
                           wi_stream_t stream) {
  BuildPlan pl;
  wi_status st = make_build_plan(kv, seg_len, cluster_size, pl);
  if (st != WI_OK) return st;
  if (!centroids || !assign || !aligned(centroids, 16) || !aligned(assign, 4))
    return WI_ERR_INVALID_ARG;
  if ((st = check_ws(ws, ws_bytes, pl.total)) != WI_OK) return st;
  BuildArgs a{};
  a.kin = make_pool(kv->k_pool, kv->block_table, kv->n_pages, kv->max_pages, kv->page_size);
  a.vin = make_pool(kv->v_pool, kv->block_table, kv->n_pages, kv->max_pages, kv->page_size);
  a.ws = static_cast<unsigned char*>(ws);
  const cudaError_t e =
      launch_assign_only(pl, a, centroids, assign, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WI_OK : cuda_fail(e);
}

wi_status wi_decode_workspace_size(const wi_index* idx, const wi_decode_params* p, size_t* bytes) {
  if (!bytes) return WI_ERR_INVALID_ARG;
  DecodePlan pl;
  const wi_status st = make_decode_plan(idx, p, pl);
  if (st != WI_OK) return st;
  *bytes = pl.total;
  return WI_OK;
}

wi_status wi_decode_workspace_layout(const wi_index* idx, const wi_decode_params* p,
                                     wi_decode_layout* layout) {
  if (!layout) return WI_ERR_INVALID_ARG;
  DecodePlan pl;
  const wi_status st = make_decode_plan(idx, p, pl);
  if (st != WI_OK) return st;
  layout->total_bytes = pl.total;
  layout->status = pl.off_status;
  layout->records = pl.off_rec;
  layout->selected = pl.off_sel;
  layout->unit_info = pl.off_info;
  layout->n_scan_ctas = pl.n_scan;
  layout->n_gather_ctas = pl.n_gather;
  layout->info_ints = kInfoInts;
  return WI_OK;
}

wi_status wi_decode(const void* q, const wi_index* idx, const wi_decode_params* p, float* out,
                    float* lse, void* ws, size_t ws_bytes, wi_stream_t stream) {
  return decode_impl(q, idx, p, out, lse, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream),
                     nullptr, nullptr, nullptr);
}

wi_status wi_decode_host(const void* q_host, const wi_index* idx, const wi_decode_params* p,
                         float* out_host, float* lse_host, void* ws, size_t ws_bytes,
                         wi_stream_t stream) {
  if (!q_host || !out_host) return WI_ERR_INVALID_ARG;
  return decode_impl(nullptr, idx, p, nullptr, nullptr, ws, ws_bytes,
                     reinterpret_cast<cudaStream_t>(stream), q_host, out_host, lse_host);
}

int32_t wi_decode_stage_count(void) { return kDecodeStages; }

const char* wi_decode_stage_name(int32_t i) {
  return (i >= 0 && i < kDecodeStages) ? kDecodeStageNames[i] : nullptr;
}

wi_status wi_read_device_status(const void* ws, wi_stream_t stream, uint32_t* flags, int clear) {
  if (!ws || !flags || !aligned(ws, 256)) return WI_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  uint32_t v = 0;
  e = cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  if (clear && v) {
    e = cudaMemsetAsync(const_cast<void*>(ws), 0, sizeof(v), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  *flags = v;
  return v ? WI_ERR_DEVICE_CHECK : WI_OK;
}

const char* wi_status_string(wi_status s) {
  switch (s) {
    case WI_OK: return "ok";
    case WI_ERR_INVALID_ARG: return "invalid argument";
    case WI_ERR_UNSUPPORTED: return "unsupported configuration";
    case WI_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case WI_ERR_CUDA: return "CUDA error";
    case WI_ERR_DEVICE_CHECK: return "device-side index check failed";
  }
  return "unknown status";
}

const char* wi_last_error_string(void) { return g_last_error; }

}  // extern "C"

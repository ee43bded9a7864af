// Decode-step kernels of the wave index (sm_100a).
//
// One decode step is the query-dependent phase of the method (RetroInfer
// technical summary, section 2.A, items 1-3; Vortex summary, section 2.A
// forward_indexer).  Three launches, chained with programmatic dependent
// launch so each one's prologue overlaps the previous one's tail:
//
//  K_A score    q . centroid / sqrt(d) for every cluster and q head, the
//               group-max selection key and its first radix digit's
//               histogram (item 2, the index lookup).  U extra CTAs resolve
//               the steady zone (item 1): sink and window positions -> slots
//               -> clusters, run-length encoded, and the steady members'
//               value sums dV.  bf16 with d = 128: centroid tiles by 2-D
//               tensor copies, scores on mma.sync.  Other shapes: FFMA over
//               16-byte cp.async tiles, with every cluster's estimation term
//               folded in during the same pass over the value sums.
//  K_B topk     exact radix select of the k best candidate clusters per KV
//               head (a threshold key and id), ties to the lower id (Vortex
//               2.C Top-K).
//  K_C attend   range CTAs pick their range's retrieved clusters against the
//               threshold, resolve the tokens' pool rows and run exact
//               attention over them (items 1 and 2) together with the
//               range's estimation zone (item 3); steady CTAs attend the
//               steady zone; the last CTA of each unit merges every part by
//               log-sum-exp.
//
// The score and estimation contractions have M = G <= 8 rows: on the tensor
// cores the heads are padded to the 16 rows of an m16n8k16 tile; on the CUDA
// cores every row is spread over LPR = d*sizeof(T)/16 lanes.
#include <cfloat>
#include <climits>
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <type_traits>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "wi_common.cuh"
#include "wi_plan.h"

namespace wi {

const char* const kDecodeStageNames[kDecodeStages] = {"score", "topk", "attend"};

namespace {

template <typename T, int D>
struct RowShape {
  static constexpr int EPL = Elem<T>::kPerVec;  // elements per lane (one 16-B vector)
  static constexpr int LPR = D / EPL;           // lanes per row
  static constexpr int RPW = 32 / LPR;          // rows per warp step
  static constexpr int ROWB = D * (int)sizeof(T);
  static constexpr int TILE = 16384 / ROWB;     // rows per 16 KB shared-memory tile
};

// G consecutive floats of shared memory (16-byte aligned rows when G >= 4)
template <int G>
__device__ __forceinline__ void load_row(const float* p, float (&v)[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int g = 0; g < G; g += 4) {
      const float4 x = *reinterpret_cast<const float4*>(p + g);
      v[g] = x.x; v[g + 1] = x.y; v[g + 2] = x.z; v[g + 3] = x.w;
    }
  } else if constexpr (G == 2) {
    const float2 x = *reinterpret_cast<const float2*>(p);
    v[0] = x.x; v[1] = x.y;
  } else {
#pragma unroll
    for (int g = 0; g < G; ++g) v[g] = p[g];
  }
}

template <int G>
__device__ __forceinline__ void store_row(float* p, const float (&v)[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int g = 0; g < G; g += 4)
      *reinterpret_cast<float4*>(p + g) = make_float4(v[g], v[g + 1], v[g + 2], v[g + 3]);
  } else if constexpr (G == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  } else {
#pragma unroll
    for (int g = 0; g < G; ++g) p[g] = v[g];
  }
}

template <typename T, int D, int G>
__device__ __forceinline__ void load_q(const T* q, int n_q_heads, int b, int h, int sub, float scale,
                                       float (&qv)[G][Elem<T>::kPerVec]) {
  constexpr int EPL = Elem<T>::kPerVec;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const T* qp = q + ((int64_t)b * n_q_heads + (int64_t)h * G + g) * D + sub * EPL;
    const uint4 raw = *reinterpret_cast<const uint4*>(qp);
    Elem<T>::unpack(raw, qv[g]);
#pragma unroll
    for (int e = 0; e < EPL; ++e) qv[g][e] *= scale;
  }
}

struct SteadyArgs {
  const int32_t* invperm;
  const int32_t* labels;
  const int32_t* offsets;
  Pool vp;
  int n_sink, window, cap, sort_pow2;
  int32_t *st_slot, *st_cl, *aff_cl, *aff_start, *nonc, *info;
  float* dv;       // [U][cap][D] fp32: sum of the steady members' values per affected cluster
  int32_t* aff_of; // [U][max_nc]: affected cluster j: (j+1) | (its steady members << 16),
                   // or -(j+1) when none of its members is left (not a candidate)
  int max_nc;
};

constexpr int kSteadyRank = 256;   // steady lists up to this size are rank-sorted in one step
constexpr int kSteadyStage = 128;  // ... and up to this size their value rows are staged

// Steady zone of unit u: positions -> (slot, cluster) through invperm and
// labels (one round of independent loads), sorted by slot (which also
// groups them by cluster, clusters being slot ranges), run-length encoded
// into (affected cluster, first steady index); the affected clusters left
// without a non-steady member are listed (they are not candidates), and the
// value rows of each affected cluster's steady members are summed in slot
// order (dV).  `sh` is the CTA's dynamic shared memory (>= 64 KB).
template <typename T, int D>
__device__ void steady_role(const Geo& geo, int u, const SteadyArgs& a, uint32_t* status,
                            unsigned char* sh) {
  const int b = u / geo.hkv, h = u - b * geo.hkv;
  const int Tb = geo.T(b), NC = geo.NC(b);
  const int ns = min(a.n_sink, Tb);
  const int wstart = max(Tb - a.window, ns);
  const int n_st = ns + (Tb - wstart);
  int32_t* I = a.info + (int64_t)u * kInfoInts;
  int32_t* nonc = a.nonc + (int64_t)u * (a.cap + 1);
  if (n_st >= Tb) {  // all steady: attended densely, nothing retrieved or estimated
    if (threadIdx.x == 0) { I[4] = Tb; I[5] = 0; I[6] = 1; nonc[0] = 0; }
    return;
  }
  const int tid = threadIdx.x;
  int npow = 1;
  while (npow < n_st) npow <<= 1;
  npow = min(npow, a.sort_pow2);
  unsigned long long* srt = reinterpret_cast<unsigned long long*>(sh);   // [npow] sorted keys
  __shared__ int s_naff, s_nnc;
  const int32_t* inv = a.invperm + geo.tok_row(b, h);
  const int32_t* lab = a.labels + geo.tok_row(b, h);
  auto key_of = [&](int i) -> unsigned long long {
    const int pos = i < ns ? i : wstart + (i - ns);
    int s = __ldg(inv + pos), c = __ldg(lab + pos);
    if (s < 0 || s >= Tb) { flag_error(status, WI_DEV_BAD_SLOT); s = 0x7fffffff; }
    if (c < 0 || c >= NC) { flag_error(status, WI_DEV_BAD_CLUSTER); c = 0; }
    return ((unsigned long long)(uint32_t)s << 32) | (uint32_t)c;
  };
  const bool rank_sort = n_st <= kSteadyRank && n_st <= (int)blockDim.x;
  if (rank_sort) {
    // rank sort: one key per thread, rank = smaller keys + equal keys before it
    unsigned long long* raw = srt + npow;
    const unsigned long long k = tid < n_st ? key_of(tid) : 0ull;
    if (tid < n_st) raw[tid] = k;
    __syncthreads();
    if (tid < n_st) {
      int r = 0;
      for (int j = 0; j < n_st; ++j) {
        const unsigned long long x = raw[j];
        r += (x < k) || (x == k && j < tid);
      }
      srt[r] = k;
    }
    __syncthreads();
  } else {
    for (int i = tid; i < npow; i += blockDim.x) srt[i] = i < n_st ? key_of(i) : ~0ull;
    __syncthreads();
    for (int k = 2; k <= npow; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < npow; i += blockDim.x) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const bool up = (i & k) == 0;
            const unsigned long long x = srt[i], y = srt[ixj];
            if ((x > y) == up) { srt[i] = y; srt[ixj] = x; }
          }
        }
        __syncthreads();
      }
    }
  }
  int32_t* slots = a.st_slot + (int64_t)u * a.cap;
  int32_t* cls = a.st_cl + (int64_t)u * a.cap;
  for (int i = tid; i < n_st; i += blockDim.x) {
    slots[i] = (int32_t)(srt[i] >> 32);
    cls[i] = (int32_t)(srt[i] & 0xffffffffu);
  }
  // run heads -> affected clusters (shared copies beside the global lists)
  int32_t* s_acl = reinterpret_cast<int32_t*>(srt + (rank_sort ? 2 : 1) * npow);  // [n_st]
  int32_t* s_ast = s_acl + n_st;                                      // [n_st + 1]
  if (tid < 32) {
    const int lane = tid;
    int32_t* acl = a.aff_cl + (int64_t)u * a.cap;
    int32_t* ast = a.aff_start + (int64_t)u * (a.cap + 1);
    int n_aff = 0;
    for (int base = 0; base < n_st; base += 32) {
      const int i = base + lane;
      const int c = i < n_st ? (int)(srt[i] & 0xffffffffu) : -1;
      const bool head = i < n_st && (i == 0 || (int)(srt[i - 1] & 0xffffffffu) != c);
      const unsigned bal = __ballot_sync(0xffffffffu, head);
      if (head) {
        const int r = n_aff + __popc(bal & ((1u << lane) - 1u));
        acl[r] = c; ast[r] = i;
        s_acl[r] = c; s_ast[r] = i;
      }
      n_aff += __popc(bal);
    }
    if (lane == 0) {
      ast[n_aff] = n_st;
      s_ast[n_aff] = n_st;
      I[4] = n_st; I[5] = n_aff; I[6] = 0;
      s_naff = n_aff;
      s_nnc = 0;
    }
  }
  __syncthreads();
  const int n_aff = s_naff;
  constexpr int EPL = Elem<T>::kPerVec, LPR = D / EPL, GPB = kStreamThreads / LPR;
  constexpr int ROWB = D * (int)sizeof(T);
  const bool staged = n_st <= kSteadyStage;
  int64_t* s_ro = reinterpret_cast<int64_t*>(s_ast + n_st + 2);        // [n_st] (8-byte aligned below)
  s_ro = reinterpret_cast<int64_t*>((reinterpret_cast<uintptr_t>(s_ro) + 15) & ~uintptr_t(15));
  T* s_rows = reinterpret_cast<T*>(s_ro + kSteadyStage);              // [n_st][D]
  // one round: the member counts of the affected clusters and the pool rows
  // of the steady slots
  const int32_t* off = a.offsets + geo.off_row(b, h);
  for (int i = tid; i < n_st; i += blockDim.x) {
    if (i < n_aff) {
      const int c = s_acl[i];
      const int full = __ldg(off + c + 1) - __ldg(off + c);
      const bool none_left = full - (s_ast[i + 1] - s_ast[i]) <= 0;
      if (none_left) nonc[1 + atomicAdd(&s_nnc, 1)] = c;
      a.aff_of[(int64_t)u * a.max_nc + c] =
          none_left ? -(i + 1) : (i + 1) | ((s_ast[i + 1] - s_ast[i]) << 16);
    }
    if (staged) s_ro[i] = pool_row(a.vp, geo.hkv, D, b, h, (int)(srt[i] >> 32), status);
  }
  __syncthreads();
  if (tid == 0) nonc[0] = s_nnc;
  const int lane = tid & 31, sub = lane % LPR, grp = tid / LPR;
  const T* vb = reinterpret_cast<const T*>(a.vp.base);
  if (staged) {
    for (int k = tid; k < n_st * LPR; k += blockDim.x) {
      const int i = k / LPR, ch = k - i * LPR;
      if (s_ro[i] >= 0) cp_async16(s_rows + i * D + ch * EPL, vb + s_ro[i] + ch * EPL);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
  }
  // dV: one group of LPR lanes per affected cluster, members in slot order
  for (int j = grp; j < n_aff; j += GPB) {
    float acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
    for (int i = s_ast[j]; i < s_ast[j + 1]; ++i) {
      float x[EPL];
      if (staged) {
        if (s_ro[i] < 0) continue;
        Elem<T>::unpack(*reinterpret_cast<const uint4*>(s_rows + i * D + sub * EPL), x);
      } else {
        const int64_t ro = pool_row(a.vp, geo.hkv, D, b, h, (int)(srt[i] >> 32), status);
        if (ro < 0) continue;
        Elem<T>::unpack(ld_stream(vb + ro + sub * EPL), x);
      }
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[e] += x[e];
    }
    float* dst = a.dv + ((int64_t)u * a.cap + j) * D + sub * EPL;
#pragma unroll
    for (int e = 0; e < EPL; ++e) dst[e] = acc[e];
  }
  (void)ROWB;
}

// -------------------------------------------------------- K_A score + estimate
// Each CTA takes a chunk of CROWS clusters of one unit: 32 KB of centroid
// rows and the same clusters' 32 KB of value-sum rows, staged in shared
// memory by 16-byte cp.async in four groups (centroid tiles first).  It
// scores the chunk, writes the per-head scores and the group-max keys, adds
// the keys' top 11 bits to the unit's selection histogram (the first radix
// digit of the top-k), and folds ALL the chunk's clusters into one softmax
// part per q head: m = max s, l = sum cnt e^(s-m), o = sum e^(s-m) Vsum.
// The retrieved clusters, the clusters left without a non-steady member and
// the steady members of the other affected clusters are taken back out in
// K_C: the estimation zone is a sum over clusters, so "all minus those" is
// the same sum, and since a cluster's estimated mass never exceeds the exact
// mass of its own tokens (Jensen), the cancellation costs at most a few fp32
// ulps of the merged output.  This way the value sums stream in the same
// pass as the centroids instead of after the selection.
constexpr int kHistBins = 2048;
constexpr int kHistShift = 21;

template <int D>
struct Part {  // one softmax part of one (unit, q head): {m, l, -, -, o[D]}
  static constexpr int kStride = D + 4;
  static constexpr int kO = 4;
};

// part.o[g][e] = sum over the CTA of acc (+ extra[g][e] * fac[g] when extra;
// fac null: 1)
template <int G, int EPL, int LPR, int D>
__device__ __forceinline__ void reduce_and_store(float (&acc)[G][EPL], float* s_red, int warp,
                                                 int sub, int rsub, float* part,
                                                 const float* extra = nullptr,
                                                 const float* fac = nullptr) {
  constexpr int NW = kStreamThreads / 32;
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL; ++e)
#pragma unroll
      for (int o = LPR; o < 32; o <<= 1) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], o);
  if (rsub == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EPL; ++e) s_red[(warp * G + g) * D + sub * EPL + e] = acc[g][e];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
    const int g = i / D, e = i - g * D;
    float v = extra ? extra[g * D + e] * (fac ? fac[g] : 1.f) : 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += s_red[(w * G + g) * D + e];
    part[g * Part<D>::kStride + Part<D>::kO + e] = v;
  }
}

// (m, l, o) = (-inf, 0, 0) for each of G heads, PS floats apart
__device__ __forceinline__ void empty_part(float* part, int G, int PS) {
  for (int i = threadIdx.x; i < G * PS; i += blockDim.x) part[i] = (i % PS) == 0 ? -INFINITY : 0.f;
}

// Shared-memory layout of a K_A stream CTA (bytes).
template <typename T, int D, int G>
struct ScoreSmem {
  static constexpr int ROWB = D * (int)sizeof(T);
  static constexpr int CROWS = kScoreChunkBytes / ROWB;          // clusters per chunk
  static constexpr int TR = 16384 / ROWB;                         // rows per 16 KB tile
  static constexpr size_t kRing = 4 * 16384;                      // 4 tiles in flight
  static constexpr size_t kRed = (size_t)(kStreamThreads / 32) * G * D * 4;
  static constexpr size_t kHist = (size_t)kHistBins / 2 * 4;
  static constexpr size_t kOff = (size_t)2 * (CROWS + 4) * 4;    // offsets, double-buffered
  static constexpr size_t kW = (size_t)CROWS * G * 4;
  static constexpr size_t kQ = (size_t)2 * G * D * sizeof(T);    // q, double-buffered
  static constexpr size_t oRed = kRing, oHist = oRed + kRed, oOff = oHist + kHist,
                          oW = oOff + kOff, oQ = oW + kW, kTotal = oQ + kQ;
};

// K_A.  blockIdx.x < U: the steady role of unit blockIdx.x.  The other
// n_stream CTAs are persistent: CTA s takes chunks [s n / n_stream,
// (s+1) n / n_stream) of the n = U * n_chunks chunks (unit-major) and streams
// each chunk's two centroid tiles and two value-sum tiles through a ring of
// four 16 KB slots (one cp.async group per tile; a slot is refilled with the
// tile four places ahead as soon as it is consumed, so the next chunk loads
// while this one computes).  The chunk's offsets and q ride in the group of
// its first tile.
template <typename T, int D, int G>
__global__ void __launch_bounds__(kStreamThreads, G >= 8 ? 1 : 2)
wave_score_kernel(const Geo geo, const T* __restrict__ q, int n_q_heads, const T* __restrict__ cent,
                  const T* __restrict__ vsum, const int32_t* __restrict__ offsets,
                  float* __restrict__ scores, uint32_t* __restrict__ keys,
                  int32_t* __restrict__ hist_g, float* __restrict__ est_parts, float scale,
                  int n_chunks, int n_stream, const SteadyArgs sa, uint32_t* status) {
  using RS = RowShape<T, D>;
  using SM = ScoreSmem<T, D, G>;
  constexpr int EPL = RS::EPL, LPR = RS::LPR, RPW = RS::RPW, TR = RS::TILE;
  constexpr int NW = kStreamThreads / 32;
  constexpr int CROWS = SM::CROWS;
  constexpr int PS = Part<D>::kStride;
  constexpr int ITR = TR / (NW * RPW);
  static_assert(G <= LPR && G <= NW, "group larger than lanes per row or warps");
  static_assert(CROWS == 2 * TR, "two tiles per matrix per chunk");
  extern __shared__ __align__(16) unsigned char sh_dyn[];
  __shared__ float s_m[G], s_l[G];
  pdl_launch_dependents();
  const int U = geo.batch * geo.hkv;
  if ((int)blockIdx.x < U) {
    steady_role<T, D>(geo, blockIdx.x, sa, status, sh_dyn);
    return;
  }
  const int sidx = blockIdx.x - U;
  const int n_tot = U * n_chunks;
  const int k0 = (int)((int64_t)sidx * n_tot / n_stream);
  const int k1 = (int)((int64_t)(sidx + 1) * n_tot / n_stream);
  const int nk = k1 - k0;
  T* ring = reinterpret_cast<T*>(sh_dyn);
  float* s_red = reinterpret_cast<float*>(sh_dyn + SM::oRed);
  uint32_t* hist = reinterpret_cast<uint32_t*>(sh_dyn + SM::oHist);
  int* s_offb = reinterpret_cast<int*>(sh_dyn + SM::oOff);
  float* s_w = reinterpret_cast<float*>(sh_dyn + SM::oW);
  T* s_q = reinterpret_cast<T*>(sh_dyn + SM::oQ);
  __shared__ __align__(8) uint64_t s_bar[4];         // one per ring slot
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane % LPR, rsub = lane / LPR;
  const int j = sub / (LPR / G);
  struct Chunk { int u, b, h, c0, nrows; int64_t row0; };
  auto chunk = [&](int k) -> Chunk {
    Chunk c;
    c.u = k / n_chunks;
    c.b = c.u / geo.hkv;
    c.h = c.u - c.b * geo.hkv;
    c.c0 = (k - c.u * n_chunks) * CROWS;
    c.nrows = max(0, min(geo.NC(c.b) - c.c0, CROWS));
    c.row0 = geo.cl_row(c.b, c.h);
    return c;
  };
  // thread 0: tile i of this CTA (chunk i / 4; centroid rows 0..TR-1,
  // TR..2TR-1, then value-sum rows likewise) into ring slot i % 4 as one bulk
  // copy completing on the slot's barrier (a plain arrive for an empty tile)
  auto issue_tile = [&](int i) {
    if (i >= 4 * nk) return;
    const int part = i & 3;
    const Chunk c = chunk(k0 + (i >> 2));
    const int r0 = (part & 1) * TR, nr = min(TR, c.nrows - r0);
    uint64_t* bar = &s_bar[i & 3];
    if (nr <= 0) { mbar_arrive(bar); return; }
    const T* src = (part < 2 ? cent : vsum) + (c.row0 + c.c0 + r0) * D;
    fence_proxy_async();
    mbar_arrive_expect(bar, (uint32_t)(nr * SM::ROWB));
    bulk_load(ring + (size_t)(i & 3) * TR * D, src, (uint32_t)(nr * SM::ROWB), bar);
  };
  // all threads: chunk kk's offsets and q (double-buffered), one cp.async group
  auto issue_meta = [&](int kk) {
    if (kk < nk) {
      const Chunk c = chunk(k0 + kk);
      if (c.nrows > 0) {
        int* so = s_offb + (kk & 1) * (CROWS + 4);
        const int32_t* off = offsets + geo.off_row(c.b, c.h) + c.c0;
        for (int x = tid; x <= c.nrows; x += blockDim.x) cp_async4(so + x, off + x);
        T* sq = s_q + (size_t)(kk & 1) * G * D;
        const T* qs = q + ((int64_t)c.b * n_q_heads + (int64_t)c.h * G) * D;
        for (int x = tid; x < G * LPR; x += blockDim.x) cp_async16(sq + x * EPL, qs + x * EPL);
      }
    }
    cp_async_commit();
  };
  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) mbar_init(&s_bar[i], 1);
    mbar_init_fence();
  }
  for (int i = tid; i < kHistBins / 2; i += blockDim.x) hist[i] = 0u;
  __syncthreads();
  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) issue_tile(i);
  }
  issue_meta(0);
  issue_meta(1);

  for (int kk = 0; kk < nk; ++kk) {
    const Chunk c = chunk(k0 + kk);
    float* part = est_parts + ((int64_t)(k0 + kk)) * G * PS;   // [u][chunk] = k
    const int* s_off = s_offb + (kk & 1) * (CROWS + 4);
    const uint32_t par = kk & 1;                                 // each slot: one phase per chunk
    cp_async_wait<1>();  // this chunk's offsets and q (the next chunk's may be in flight)
    __syncthreads();
    float qv[G][EPL];
    if (c.nrows > 0) {
      const T* sq = s_q + (size_t)(kk & 1) * G * D;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        Elem<T>::unpack(*reinterpret_cast<const uint4*>(sq + g * D + sub * EPL), qv[g]);
#pragma unroll
        for (int e = 0; e < EPL; ++e) qv[g][e] *= scale;
      }
    }
    // ---- scores over the two centroid tiles
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      mbar_wait(&s_bar[(4 * kk + t) & 3], par, status);
      const T* tile = ring + (size_t)((4 * kk + t) & 3) * TR * D;
      if (c.nrows > t * TR) {
#pragma unroll
        for (int it = 0; it < ITR; ++it) {
          const int rl = (it * NW + warp) * RPW + rsub;
          const int r = t * TR + rl;
          const bool ok = r < c.nrows;
          float x[EPL];
          if (ok) {
            Elem<T>::unpack(*reinterpret_cast<const uint4*>(tile + rl * D + sub * EPL), x);
          } else {
#pragma unroll
            for (int e = 0; e < EPL; ++e) x[e] = 0.f;
          }
          float acc[G];
          dot_g<G, EPL>(qv, x, acc);
          group_reduce_multi<G, LPR>(acc, lane);
          float m = acc[0];
#pragma unroll
          for (int o = LPR / 2; o >= LPR / G; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          if (ok) {
            if (sub % (LPR / G) == 0) {
              scores[(c.row0 + c.c0 + r) * G + j] = acc[0];
              s_w[r * G + j] = acc[0];
            }
            if (sub == 0) {
              const uint32_t key = (s_off[r + 1] - s_off[r]) > 0 ? ordered_key(m) : 0u;
              keys[c.row0 + c.c0 + r] = key;
              if (key) atomicAdd(&hist[key >> (kHistShift + 1)], 1u << (16 * ((key >> kHistShift) & 1u)));
            }
          }
        }
      }
      __syncthreads();
      if (tid == 0) issue_tile(4 * kk + t + 4);
    }
    if (c.nrows == 0) {
      // past this sequence's clusters: an empty part; consume the value-sum tiles
      empty_part(part, G, PS);
#pragma unroll
      for (int t = 2; t < 4; ++t) {
        mbar_wait(&s_bar[(4 * kk + t) & 3], par, status);
        __syncthreads();
        if (tid == 0) issue_tile(4 * kk + t + 4);
      }
      issue_meta(kk + 2);
      continue;
    }
    // ---- histogram flush (two 16-bit counts per word), chunk statistics
    {
      int* hg = hist_g + (int64_t)c.u * kHistBins;
      for (int i = tid; i < kHistBins / 2; i += blockDim.x) {
        const uint32_t w = hist[i];
        if (w) {
          if (w & 0xffffu) atomicAdd(hg + 2 * i, (int)(w & 0xffffu));
          if (w >> 16) atomicAdd(hg + 2 * i + 1, (int)(w >> 16));
          hist[i] = 0u;
        }
      }
    }
    if (warp < G) {  // warp g: head g's max, weights and denominator
      float m = -INFINITY;
      for (int r = lane; r < c.nrows; r += 32) m = fmaxf(m, s_w[r * G + warp]);
      m = warp_max(m);
      float l = 0.f;
      for (int r = lane; r < c.nrows; r += 32) {
        const int cnt = s_off[r + 1] - s_off[r];
        const float w = cnt > 0 ? __expf(s_w[r * G + warp] - m) : 0.f;
        s_w[r * G + warp] = w;
        l += (float)cnt * w;
      }
      l = warp_sum(l);
      if (lane == 0) { s_m[warp] = m; s_l[warp] = l; }
    }
    __syncthreads();
    // ---- weighted value sums over the two value-sum tiles
    float acc[G][EPL];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
#pragma unroll
    for (int t = 2; t < 4; ++t) {
      mbar_wait(&s_bar[(4 * kk + t) & 3], par, status);
      const T* tile = ring + (size_t)((4 * kk + t) & 3) * TR * D;
#pragma unroll
      for (int it = 0; it < ITR; ++it) {
        const int rl = (it * NW + warp) * RPW + rsub;
        const int r = (t - 2) * TR + rl;
        if (r < c.nrows) {
          float x[EPL];
          Elem<T>::unpack(*reinterpret_cast<const uint4*>(tile + rl * D + sub * EPL), x);
          float wv[G];
          load_row<G>(s_w + r * G, wv);
          axpy_g<G, EPL>(wv, x, acc);
        }
      }
      __syncthreads();
      if (tid == 0) issue_tile(4 * kk + t + 4);
    }
    reduce_and_store<G, EPL, LPR, D>(acc, s_red, warp, sub, rsub, part);
    if (tid < G) { part[tid * PS] = s_m[tid]; part[tid * PS + 1] = s_l[tid]; }
    issue_meta(kk + 2);
  }
  cp_async_wait<0>();
  // every tile issued was waited for above; should a bounded wait have given
  // up, wait (bounded again) for each slot's last copy before leaving
  if (nk > 0) {
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) mbar_wait(&s_bar[sl], (uint32_t)((nk - 1) & 1), status);
  }
}

// K_A on the tensor cores (bf16, d = 128): the centroids alone.  Same
// chunking as wave_score_kernel (128 clusters per chunk); a chunk's two
// centroid tiles stream through a ring of NS 16 KB slots filled by 2-D tensor
// copies (two 64-column boxes per tile, 128-byte swizzle, so ldmatrix is
// conflict-free); scores S^T[g][r] = sum_d q[g][d] c[r][d] on mma.sync
// m16n8k16 (A = q with the heads padded to 16 rows, B = centroid rows),
// scaled by 1/sqrt(d) after.  The value sums are read by the attend
// kernel's range CTAs, which estimate their own clusters.
template <int G>
struct MmaSmem {
  static constexpr int D = 128, CROWS = kScoreChunkBytes / (D * 2), TR = 64;
  static constexpr int kSlots = 6;                     // tiles in flight per CTA
  static constexpr size_t kRing = (size_t)kSlots * 16384;
  static constexpr size_t kHist = (size_t)kHistBins / 2 * 4;
  static constexpr size_t kOff = (size_t)2 * (CROWS + 4) * 4;
  static constexpr size_t kQ = (size_t)2 * G * D * 2;
  static constexpr size_t oHist = kRing, oOff = oHist + kHist, oQ = oOff + kOff,
                          kTotal = oQ + kQ + 1024;   // + 1 KB to align the ring to 1024 B
};

template <int G>
__global__ void __launch_bounds__(kStreamThreads, 2)
wave_score_mma_kernel(const Geo geo, const __nv_bfloat16* __restrict__ q, int n_q_heads,
                      const __grid_constant__ CUtensorMap tm_cent,
                      const int32_t* __restrict__ offsets, float* __restrict__ scores,
                      uint32_t* __restrict__ keys, int32_t* __restrict__ hist_g, float scale,
                      int n_chunks, int n_stream, const SteadyArgs sa, uint32_t* status) {
  using T = __nv_bfloat16;
  using SM = MmaSmem<G>;
  constexpr int D = SM::D, CROWS = SM::CROWS, TR = SM::TR, NS = SM::kSlots;
  static_assert(G <= 8, "at most 8 query heads per KV head (MMA rows 0..7)");
  extern __shared__ __align__(16) unsigned char sh_raw[];
  __shared__ __align__(8) uint64_t s_bar[SM::kSlots];
  pdl_launch_dependents();
  const int U = geo.batch * geo.hkv;
  if ((int)blockIdx.x < U) {
    steady_role<T, D>(geo, blockIdx.x, sa, status, sh_raw);
    return;
  }
  unsigned char* sh = align_smem_1024(sh_raw);
  unsigned char* ring = sh;
  uint32_t* hist = reinterpret_cast<uint32_t*>(sh + SM::oHist);
  int* s_offb = reinterpret_cast<int*>(sh + SM::oOff);
  T* s_q = reinterpret_cast<T*>(sh + SM::oQ);
  const int sidx = blockIdx.x - U;
  const int n_tot = U * n_chunks;
  const int k0 = (int)((int64_t)sidx * n_tot / n_stream);
  const int k1 = (int)((int64_t)(sidx + 1) * n_tot / n_stream);
  const int nk = k1 - k0;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;    // MMA fragment row (head) and column pair
  struct Chunk { int u, b, h, c0, nrows; int64_t row0; };
  auto chunk = [&](int k) -> Chunk {
    Chunk c;
    c.u = k / n_chunks;
    c.b = c.u / geo.hkv;
    c.h = c.u - c.b * geo.hkv;
    c.c0 = (k - c.u * n_chunks) * CROWS;
    c.nrows = max(0, min(geo.NC(c.b) - c.c0, CROWS));
    c.row0 = geo.cl_row(c.b, c.h);
    return c;
  };
  // thread 0: tile i (chunk i / 2, centroid rows (i % 2) * TR ..) into slot i % NS
  auto issue_tile = [&](int i) {
    if (i >= 2 * nk) return;
    const Chunk c = chunk(k0 + (i >> 1));
    const int r0 = (i & 1) * TR;
    uint64_t* bar = &s_bar[i % NS];
    if (c.nrows - r0 <= 0) { mbar_arrive(bar); return; }
    unsigned char* dst = ring + (size_t)(i % NS) * 16384;
    const int y = (int)(c.row0 + c.c0 + r0);
    if (i >= NS) fence_proxy_async();   // the slot was read by the generic proxy
    mbar_arrive_expect(bar, 16384u);
    tensor_load_2d(dst, &tm_cent, 0, y, bar);
    tensor_load_2d(dst + 8192, &tm_cent, 64, y, bar);
  };
  auto issue_meta = [&](int kk) {   // all threads: chunk kk's offsets and q
    if (kk < nk) {
      const Chunk c = chunk(k0 + kk);
      if (c.nrows > 0) {
        int* so = s_offb + (kk & 1) * (CROWS + 4);
        const int32_t* off = offsets + geo.off_row(c.b, c.h) + c.c0;
        for (int x = tid; x <= c.nrows; x += blockDim.x) cp_async4(so + x, off + x);
        T* sq = s_q + (size_t)(kk & 1) * G * D;
        const T* qs = q + ((int64_t)c.b * n_q_heads + (int64_t)c.h * G) * D;
        for (int x = tid; x < G * D / 8; x += blockDim.x) cp_async16(sq + x * 8, qs + x * 8);
      }
    }
    cp_async_commit();
  };
  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < NS; ++i) mbar_init(&s_bar[i], 1);
    mbar_init_fence();
  }
  for (int i = tid; i < kHistBins / 2; i += blockDim.x) hist[i] = 0u;
  issue_meta(0);   // the small loads first, ahead of the tiles
  issue_meta(1);
  __syncthreads();
  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < NS; ++i) issue_tile(i);
  }
  // tile i sits in slot i % NS and completes phase (i / NS) & 1 of its barrier
  auto tile_wait = [&](int i) { mbar_wait(&s_bar[i % NS], (uint32_t)((i / NS) & 1), status); };

  int since_flush = 0;
  for (int kk = 0; kk < nk; ++kk) {
    const Chunk c = chunk(k0 + kk);
    const int* s_off = s_offb + (kk & 1) * (CROWS + 4);
    cp_async_wait<1>();
    __syncthreads();
    // q as A fragments (rows = heads; heads >= G and rows 8..15 are zero)
    uint32_t qa0[D / 16], qa2[D / 16];
    {
      const uint32_t* qw = reinterpret_cast<const uint32_t*>(s_q + (size_t)(kk & 1) * G * D + (g < G ? g : 0) * D);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        qa0[ks] = (g < G && c.nrows > 0) ? qw[8 * ks + tq] : 0u;
        qa2[ks] = (g < G && c.nrows > 0) ? qw[8 * ks + 4 + tq] : 0u;
      }
    }
    // scores: warp w takes the tile's rows 8w .. 8w + 7
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      tile_wait(2 * kk + t);
      const unsigned char* slot = ring + (size_t)((2 * kk + t) % NS) * 16384;
      if (c.nrows > t * TR) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const int n0 = 8 * warp;
#pragma unroll
        for (int ks = 0; ks < D / 16; ks += 2) {
          const int ch = 2 * ks + (lane >> 3);                     // 16-byte column chunk
          uint32_t bm[4];
          ldsm_x4(bm, slot + (ch >> 3) * 8192 + swz128(n0 + (lane & 7), ch & 7));
          mma_bf16(acc, qa0[ks], qa2[ks], bm[0], bm[1]);
          mma_bf16(acc, qa0[ks + 1], qa2[ks + 1], bm[2], bm[3]);
        }
        const int rl = t * TR + n0 + 2 * tq;                       // rows rl, rl + 1 of the chunk
        const float s0 = acc[0] * scale, s1 = acc[1] * scale;
        const bool ok0 = rl < c.nrows, ok1 = rl + 1 < c.nrows;
        if (g < G) {
          if (ok0) scores[(c.row0 + c.c0 + rl) * G + g] = s0;
          if (ok1) scores[(c.row0 + c.c0 + rl + 1) * G + g] = s1;
        }
        float m0 = g < G ? s0 : -INFINITY, m1 = g < G ? s1 : -INFINITY;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
          m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
        }
        if (g == 0) {
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int r = rl + k;
            if (r < c.nrows) {
              const uint32_t key = (s_off[r + 1] - s_off[r]) > 0 ? ordered_key(k ? m1 : m0) : 0u;
              keys[c.row0 + c.c0 + r] = key;
              if (key) atomicAdd(&hist[key >> (kHistShift + 1)], 1u << (16 * ((key >> kHistShift) & 1u)));
            }
          }
        }
      }
      __syncthreads();
      if (tid == 0) issue_tile(2 * kk + t + NS);
    }
    // histogram flush (two 16-bit counts per word) when the next chunk is
    // another unit's, after the last chunk, or before a count could reach
    // 2^16; a barrier waits for the round trip of global atomics issued
    // before it, so they are issued as rarely as possible
    ++since_flush;
    if (kk == nk - 1 || chunk(k0 + kk + 1).u != c.u || since_flush == 256) {
      int* hg = hist_g + (int64_t)c.u * kHistBins;
      for (int i = tid; i < kHistBins / 2; i += blockDim.x) {
        const uint32_t w = hist[i];
        if (w) {
          if (w & 0xffffu) atomicAdd(hg + 2 * i, (int)(w & 0xffffu));
          if (w >> 16) atomicAdd(hg + 2 * i + 1, (int)(w >> 16));
          hist[i] = 0u;
        }
      }
      since_flush = 0;
    }
    issue_meta(kk + 2);
  }
  cp_async_wait<0>();
  // the last tile of each slot (waited above; again, bounded, in case a wait gave up)
  for (int i = max(0, 2 * nk - NS); i < 2 * nk; ++i) tile_wait(i);
}

// ----------------------------------------------------------------- K_B topk
// One CTA per unit finds the selection threshold: the k-th best candidate
// key kstar and the largest id thr taken at that key, so that cluster c is
// retrieved iff key_c > kstar or (key_c == kstar and c <= thr) (Vortex 2.C
// Top-K: exact, ties to the lower id).  Every global read is issued in one
// round at the start (unit record, first-digit histogram, non-candidate
// list, and the keys, kTopkPerLane per thread, lane-interleaved so each warp
// load is one 128-byte line); then
//  1. the first radix digit's histogram comes from K_A (zeroed after use, so
//     the workspace is clean for the next call), minus the non-candidates; a
//     histogram whose total disagrees with the candidate count is flagged
//     and the select falls back to a full radix select over all keys;
//  2. the keys of the threshold bin (1-2% of them) get a second 11-bit digit
//     histogram, and the few keys of its threshold bin are ranked exactly by
//     (key desc, id asc).
// The retrieved clusters themselves are picked by the attend kernel's CTAs,
// each over its own range of cluster ids.
constexpr int kTopkPerLane = 16;
constexpr int kTopkRound = kTopkThreads * kTopkPerLane;   // 8192 ids per round
constexpr int kTopkCand = 1024;
constexpr int kTopkCand2 = 256;

// Fold CTAs of the attend kernel (CUDA-core path, where K_A writes one
// estimation part per 32 KB chunk): each log-sum-exp combines kFold
// consecutive chunk parts into one part of the unit's final merge, so the
// merge reads a few parts instead of one per chunk.  All loads of a fold are
// issued before the first use.
struct FoldArgs {
  const float* est_parts;   // [U][n_chunks][G][D+4]
  int n_chunks;
  float* partials;          // [U][n_parts][G][D+4]
  int n_parts, first;       // this kernel writes parts first .. first + n_fold - 1
  int G, D;
};

__device__ void fold_role(const FoldArgs& f, int u, int j) {
  const int PS = f.D + 4;
  const int p0 = j * kFold, np = min(kFold, f.n_chunks - p0);
  const float* in = f.est_parts + ((int64_t)u * f.n_chunks + p0) * f.G * PS;
  float* out = f.partials + ((int64_t)u * f.n_parts + f.first + j) * f.G * PS;
  for (int i = threadIdx.x; i < f.G * f.D; i += blockDim.x) {
    const int g = i / f.D, e = i - g * f.D;
    float mp[kFold], lp[kFold], op[kFold];
#pragma unroll
    for (int p = 0; p < kFold; ++p) {
      const float* pp = in + ((int64_t)p * f.G + g) * PS;
      mp[p] = p < np ? __ldcg(pp) : -INFINITY;
      lp[p] = p < np ? __ldcg(pp + 1) : 0.f;
      op[p] = p < np ? __ldcg(pp + 4 + e) : 0.f;
    }
    float M = -INFINITY;
#pragma unroll
    for (int p = 0; p < kFold; ++p) M = fmaxf(M, mp[p]);
    float l = 0.f, o = 0.f;
#pragma unroll
    for (int p = 0; p < kFold; ++p) {
      const float w = mp[p] == -INFINITY ? 0.f : expf(mp[p] - M);
      l += w * lp[p];
      o += w * op[p];
    }
    out[g * PS + 4 + e] = o;
    if (e == 0) { out[g * PS] = M; out[g * PS + 1] = l; }
  }
}

struct TopkArgs {
  const uint32_t* keys;
  int32_t* hist_g;
  const int32_t* nonc;       // [U][cap+1]: count, then the non-candidate clusters
  int cap;
  int topk_clusters;
  double topk_fraction;
  int32_t* info;
};

__global__ void __launch_bounds__(kTopkThreads)
wave_topk_kernel(const Geo geo, const TopkArgs A, uint32_t* status) {
  // dynamic shared: excluded bitmask [ceil(NCmax/32)] | non-candidates [cap+1]
  extern __shared__ __align__(16) int32_t sdyn[];
  __shared__ __align__(16) int hist[kHistBins];
  __shared__ unsigned long long cand[kTopkCand];
  __shared__ unsigned long long cand2[kTopkCand2];
  __shared__ int scan_sh[64];
  __shared__ int s_info[kInfoInts];
  __shared__ int s_ctl[8];
  pdl_launch_dependents();
  constexpr int PT = kTopkPerLane;
  constexpr int NW = kTopkThreads / 32;
  const int tid = threadIdx.x, nt = kTopkThreads, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int u = blockIdx.x, b = u / geo.hkv, h = u - b * geo.hkv;
  const int NC = geo.NC(b);
  const int nmask = (NC + 31) >> 5;
  const int cap = A.cap;
  uint32_t* sx = reinterpret_cast<uint32_t*>(sdyn);
  int32_t* snc = sdyn + nmask;
  for (int i = tid; i < nmask; i += nt) sx[i] = 0u;
  if (tid == 0) { s_ctl[0] = 0; s_ctl[5] = 0; }
  int32_t* I = A.info + (int64_t)u * kInfoInts;
  const int64_t row0 = geo.cl_row(b, h);
  int* hg = A.hist_g + (int64_t)u * kHistBins;
  const int k_req = A.topk_clusters >= 0 ? A.topk_clusters
                                         : (int)ceil(A.topk_fraction * (double)NC);
  const uint32_t* kk = A.keys + row0;
  const int n_rounds = (NC + kTopkRound - 1) / kTopkRound;
  const int wbase = warp * (kTopkRound / NW);       // warp's offset inside a round
  uint32_t kr[PT];
  auto cid = [&](int r, int i) { return r * kTopkRound + wbase + i * 32 + lane; };
  auto load_round = [&](int r) {
#pragma unroll
    for (int i = 0; i < PT; ++i) {
      const int c = cid(r, i);
      kr[i] = c < NC ? kk[c] : 0u;
    }
  };
  auto masked = [&](int c) -> bool { return ((sx[c >> 5] >> (c & 31)) & 1u) != 0u; };
  auto mask_round = [&](int r) {
#pragma unroll
    for (int i = 0; i < PT; ++i) {
      const int c = cid(r, i);
      if (c < NC && masked(c)) kr[i] = 0u;
    }
  };

  pdl_wait();
  // ---- the one round of loads
  if (tid < kInfoInts) cp_async4(&s_info[tid], I + tid);
  for (int i = tid; i < kHistBins / 4; i += nt) cp_async16(&hist[4 * i], hg + 4 * i);
  for (int i = tid; i <= cap; i += nt) cp_async4(snc + i, A.nonc + (int64_t)u * (cap + 1) + i);
  cp_async_commit();
  load_round(0);
  cp_async_wait<0>();
  __syncthreads();
  if (s_info[6]) {  // dense unit: every token is attended, nothing is selected
    for (int i = tid; i < kHistBins; i += nt) hg[i] = 0;   // clean for the next call
    if (tid == 0) { I[0] = 0; I[1] = (int32_t)0xFFFFFFFFu; I[2] = -1; I[7] = 0; }
    return;
  }
  // clusters left without a non-steady member are not candidates
  const int n_nonc = min(max(snc[0], 0), cap);
  for (int j = tid; j < n_nonc; j += nt) {
    const int c = snc[1 + j];
    if (c >= 0 && c < NC) {
      atomicOr(&sx[c >> 5], 1u << (c & 31));
      if (c >= kTopkRound) {  // beyond the registers' round: read its key
        const uint32_t key = kk[c];
        if (key) atomicSub(&hist[key >> kHistShift], 1);
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < PT; ++i) {
    const int c = cid(0, i);
    if (c < NC && masked(c)) {
      if (kr[i]) atomicSub(&hist[kr[i] >> kHistShift], 1);
      kr[i] = 0u;
    }
  }
  __syncthreads();

  // bin holding the krem-th largest of the histogram (bins scanned
  // downwards); *above: the count in the bins above it; *total: all
  auto first_digit = [&](int krem, int* above, int* total) -> int {
    // thread t owns bins 2047-4t .. 2044-4t (descending)
    int c4[4], s4 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) { c4[i] = hist[kHistBins - 1 - 4 * tid - i]; s4 += c4[i]; }
    int tot;
    const int incl = block_inclusive_scan(s4, scan_sh, &tot);
    if (krem < 0) krem = min(max(k_req, 0), tot);   // the first digit: k clamped to the total
    int acc = incl - s4;
    if (tid == 0) { s_ctl[1] = -1; s_ctl[2] = 0; }
    __syncthreads();
    if (krem > 0 && acc < krem && incl >= krem) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (acc + c4[i] >= krem) { s_ctl[1] = kHistBins - 1 - 4 * tid - i; s_ctl[2] = acc; break; }
        acc += c4[i];
      }
    }
    __syncthreads();
    *above = s_ctl[2];
    if (total) *total = tot;
    return s_ctl[1];
  };
  // ballot-aggregated append of x to list[cap_] through counter *ctr
  auto append = [&](bool in, unsigned long long x, unsigned long long* list, int cap_, int* ctr) {
    const unsigned bal = __ballot_sync(0xffffffffu, in);
    if (bal) {
      int base = 0;
      if (lane == __ffs(bal) - 1) base = atomicAdd(ctr, __popc(bal));
      base = __shfl_sync(0xffffffffu, base, __ffs(bal) - 1);
      const int slot = base + __popc(bal & lt);
      if (in && slot < cap_) list[slot] = x;
    }
  };
  int above1 = 0, hist_total = 0;
  int bin1 = first_digit(-1, &above1, &hist_total);
  if (min(max(k_req, 0), hist_total) >= hist_total) bin1 = -1;   // all or none: no threshold bin

  // pass A: candidate count, and the keys of the threshold bin
  int mine = 0;
  for (int r = 0; r < n_rounds; ++r) {
    if (r > 0) { load_round(r); mask_round(r); }
    // the round's threshold-bin members: counted per thread, placed by one
    // warp prefix and one shared-memory atomic per warp (the list is a set:
    // its order does not matter)
    int nm = 0;
#pragma unroll
    for (int i = 0; i < PT; ++i) {
      mine += kr[i] != 0u;
      nm += kr[i] != 0u && (int)(kr[i] >> kHistShift) == bin1;
    }
    int incl = nm;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int wb = 0;
    if (lane == 31 && incl > 0) wb = atomicAdd(&s_ctl[0], incl);
    int pos = __shfl_sync(0xffffffffu, wb, 31) + incl - nm;
    if (nm > 0) {
#pragma unroll
      for (int i = 0; i < PT; ++i) {
        if (kr[i] != 0u && (int)(kr[i] >> kHistShift) == bin1) {
          if (pos < kTopkCand)
            cand[pos] = ((unsigned long long)kr[i] << 32) | (0xFFFFFFFFu - (uint32_t)cid(r, i));
          ++pos;
        }
      }
    }
  }
  int ncand;
  block_inclusive_scan(mine, scan_sh, &ncand);
  const int nbin = s_ctl[0];
  const bool hist_ok = ncand == hist_total;
  if (!hist_ok && tid == 0) flag_error(status, WI_DEV_BAD_HIST);
  const int ksel = min(max(k_req, 0), ncand);
  uint32_t kstar = 0;
  int thr = 0;
  bool found = false;
  if (ksel == 0) { kstar = 0xFFFFFFFFu; thr = -1; found = true; }
  else if (ksel == ncand) { kstar = 1u; thr = NC; found = true; }
  else if (hist_ok && nbin <= kTopkCand) {
    // second digit (key bits 20..10) over the threshold bin's members
    int krem = ksel - above1;
    for (int i = tid; i < kHistBins; i += nt) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < nbin; i += nt)
      atomicAdd(&hist[(int)(cand[i] >> 42) & (kHistBins - 1)], 1);
    __syncthreads();
    int above2;
    const int bin2 = first_digit(krem, &above2, nullptr);
    krem -= above2;
    for (int i0 = 0; i0 < nbin; i0 += nt) {
      const int i = i0 + tid;
      const unsigned long long x = i < nbin ? cand[i] : 0ull;
      append(i < nbin && ((int)(x >> 42) & (kHistBins - 1)) == bin2, x, cand2, kTopkCand2,
             &s_ctl[5]);
    }
    __syncthreads();
    const int n2 = s_ctl[5];
    if (n2 <= kTopkCand2) {
      // the krem-th largest of bin2's members by (key, -id)
      for (int i = tid; i < n2; i += nt) {
        const unsigned long long x = cand2[i];
        int rank = 0;
        for (int j = 0; j < n2; ++j) rank += cand2[j] > x;
        if (rank == krem - 1) { s_ctl[3] = (int)(x >> 32); s_ctl[4] = (int)(0xFFFFFFFFu - (uint32_t)x); }
      }
      __syncthreads();
      kstar = (uint32_t)s_ctl[3];
      thr = s_ctl[4];
      found = true;
    }
  }
  if (!found) {
    // fallback: a full radix select over all keys (stale histogram or a
    // crowded threshold bin), 11 + 11 + 10 bit digits
    auto cand_key = [&](int c) -> uint32_t { return masked(c) ? 0u : kk[c]; };
    uint32_t prefix = 0, pmask = 0;
    int krem = ksel;
    for (int pass = 0; pass < 3; ++pass) {
      const int bits = pass == 2 ? 10 : 11;
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const int nbins = 1 << bits;
      for (int i = tid; i < kHistBins; i += nt) hist[i] = 0;
      __syncthreads();
      for (int c = tid; c < NC; c += nt) {
        const uint32_t key = cand_key(c);
        if (key != 0u && (key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & (nbins - 1)], 1);
      }
      __syncthreads();
      int ab;
      const int d = first_digit(krem, &ab, nullptr) & (nbins - 1);
      krem -= ab;
      prefix |= (uint32_t)d << shift;
      pmask |= (uint32_t)(nbins - 1) << shift;
      __syncthreads();
    }
    kstar = prefix;
    // the krem-th key equal to kstar in ascending id order
    if (tid == 0) s_ctl[4] = -1;
    __syncthreads();
    int run = 0;
    for (int base = 0; base < NC && s_ctl[4] < 0; base += nt) {
      const int c = base + tid;
      const int f = (c < NC && cand_key(c) == kstar) ? 1 : 0;
      int tot;
      const int incl = block_inclusive_scan(f, scan_sh, &tot);
      if (f && run + incl == krem) s_ctl[4] = c;
      run += tot;
      __syncthreads();
    }
    thr = s_ctl[4];
  }
  if (tid == 0) { I[0] = ksel; I[1] = (int32_t)kstar; I[2] = thr; I[7] = ncand; }
  for (int i = tid; i < kHistBins; i += nt) hg[i] = 0;   // clean for the next call
}

// ----------------------------------------------------------------- K_C attend
// range CTAs (kRangeW cluster ids each): pick the retrieved clusters of the
// range against K_B's threshold, write the range's words of the unit's
// selection bitmap, resolve their tokens' pool rows (skipping steady members)
// and run exact attention over them.  The estimation zone of the range goes
// into the same part:
//  - tensor-core path (bf16, d = 128): the range's value sums (64 KB) are
//    brought into shared memory by 2-D tensor copies issued before the
//    grid-dependency wait, so they land while the top-k runs; after the
//    picks, o_e = sum over the zone of e^(s - m_e) Vsum on mma.sync and
//    l_e = sum of (cnt - steady members) e^(s - m_e); the steady members'
//    value sums dV of the zone's affected clusters are taken back out;
//  - CUDA-core path: K_A's chunk parts counted every cluster, so the range
//    CTA takes back out what the zone leaves out: every retrieved cluster and
//    every cluster left without a non-steady member in full (cnt, Vsum), and
//    the steady members (their count, dV) of the other affected clusters;
//    fold CTAs combine K_A's chunk parts into a few merge parts;
// steady CTAs (two tiles of steady slots each): exact attention over the
// steady zone;
// the last CTA of each unit merges the parts by log-sum-exp.
constexpr int kRangeW = kRangeClusters;    // clusters per range CTA, one per thread
static_assert(kRangeW == kStreamThreads, "one cluster per thread");
constexpr int kCorrRows = 32;              // correction rows staged per pass
constexpr int kRowCap = 512;               // tokens resolved per pass of a range CTA
constexpr int kBtStage = 2 * kRangeW;      // block-table entries a range CTA stages

struct AttendArgs {
  const uint32_t* keys;
  const float* scores;
  const int32_t* info;
  int32_t* aff_of;           // [U][max_nc]: (j+1) | (steady members << 16) affected,
                             // -(j+1) non-candidate; reset here
  int max_nc;
  const int32_t* aff_start;  // [U][cap+1]
  const int32_t* st_slot;    // [U][cap]
  const float* dv;           // [U][cap][D]
  int cap;
  const int32_t* perm;       // slot -> position
  int n_sink, window;
  uint32_t* sel;             // [U][sel_words]: selection bitmap (bit c: cluster c retrieved)
  int sel_words;
  const float* est_parts;    // [U][n_chunks][G][D+4], folded by the fold CTAs
  int n_chunks;
  int n_rng, n_sc, n_fold, n_parts;
  float* partials;
  int32_t* counters;
  float* out;
  float* lse;
  float scale;
  int exact_only;            // no estimation zone: retrieved clusters and steady zone only
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kStreamThreads, G * Elem<T>::kPerVec >= 64 ? 1 : 2)
wave_attend_kernel(const Geo geo, const T* __restrict__ q, int n_q_heads, const Pool kp,
                   const Pool vp, const T* __restrict__ vsum,
                   const int32_t* __restrict__ offsets, const AttendArgs A,
                   const __grid_constant__ CUtensorMap tm_vsum, uint32_t* status) {
  using RS = RowShape<T, D>;
  constexpr int EPL = RS::EPL, LPR = RS::LPR, RPW = RS::RPW, TR = RS::TILE;
  constexpr int NW = kStreamThreads / 32;
  constexpr int PS = Part<D>::kStride;
  static_assert(TR % (NW * RPW) == 0, "tile must be a multiple of rows per CTA step");
  static_assert(2 * TR <= kStreamThreads, "one thread per token of a chunk");
  extern __shared__ __align__(16) unsigned char sh_raw[];
  // dynamic, from the first 1024-byte boundary (the tensor copies' swizzle
  // repeats every 1024 bytes of address): [ring 64 KB: K x2, V x2 tiles, or
  // the range's value sums; the cross-warp reduction and the merge reuse it]
  // [correction rows kCorrRows x D fp32] [merge factors]
  unsigned char* sh = align_smem_1024(sh_raw);
  T* ring = reinterpret_cast<T*>(sh);
  float* s_red = reinterpret_cast<float*>(sh);
  unsigned char* s_crow = sh + 4 * 16384;
  float* s_f = reinterpret_cast<float*>(s_crow + kCorrRows * D * 4);
  __shared__ int32_t s_row[kRowCap];                 // pool rows of the tokens (-1 = skip)
  __shared__ __align__(16) float s_sc[TR][G];
  __shared__ int s_pkc[kRangeW], s_pkt[kRangeW], s_pko[kRangeW];   // picked: id, token start, slot start
  __shared__ int s_cec[kRangeW], s_cew[kRangeW];                   // correction: row selector, count
  __shared__ int scan_sh[64];
  __shared__ int s_info[kInfoInts], s_last;
  __shared__ float s_m[G], s_l[G];
  // tensor-core exact attention (bf16, d = 128): tile weights, per-warp tile
  // max / sum, the exact part's output and running (m, l)
  constexpr bool kMma = std::is_same_v<T, __nv_bfloat16> && D == 128;
  __shared__ int32_t s_bt[kMma ? kBtStage : 1];      // block-table window of a range CTA
  __shared__ __align__(16) float s_ces[kMma ? 1 : kRangeW * G];   // correction: scores -> weights
  // MMA A operands in bf16, high terms in rows 0..7 (head g = row g), low
  // terms in rows 8..15, rows of heads >= G zero; padded rows (144 / 528
  // bytes) keep ldmatrix conflict-free: a tile's weights, and a range CTA's
  // estimation weights
  __shared__ __align__(16) __nv_bfloat16 s_P[kMma ? 16 : 1][kMma ? 72 : 1];
  __shared__ __align__(16) __nv_bfloat16 s_W[kMma ? 16 : 1][kMma ? kRangeW + 8 : 1];
  __shared__ float s_wmax[NW][G], s_wsum[NW][G];
  __shared__ __align__(16) float s_o[kMma ? G * D : 1];
  __shared__ float s_em[G], s_el[G], s_f1[G];
  __shared__ __align__(8) uint64_t s_vbar;          // the range's value sums have landed

  const int u = blockIdx.y, b = u / geo.hkv, h = u - b * geo.hkv;
  const int NC = geo.NC(b), Tb = geo.T(b);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tid = threadIdx.x;
  const int sub = lane % LPR, rsub = lane / LPR;
  const int jh = sub / (LPR / G);
  const int64_t row0 = geo.cl_row(b, h);
  const int32_t* off = offsets + geo.off_row(b, h);
  const bool role_range = (int)blockIdx.x < A.n_rng;
  const bool role_fold = (int)blockIdx.x >= A.n_rng + A.n_sc;
  float* part = A.partials + ((int64_t)u * A.n_parts + blockIdx.x) * G * PS;
  const int ns = min(A.n_sink, Tb), wstart = max(Tb - A.window, ns);

  float qv[G][EPL];
  load_q<T, D, G>(q, n_q_heads, b, h, sub, A.scale, qv);
  float acc[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
  float m_run[G], l_run[G];
#pragma unroll
  for (int g = 0; g < G; ++g) { m_run[g] = -INFINITY; l_run[g] = 0.f; }
  // MMA-path state: this lane's head gm = lane / 4 (valid below G), its
  // column pair tq, q as A fragments, running (mr, lr) of head gm, and the
  // output columns 16 warp .. 16 warp + 15 of head gm: in oacc[nt][0..1]
  // the products of the weights' high bf16 terms (A rows 0..7), in
  // oacc[nt][2..3] those of their low terms (A rows 8..15), summed at the end
  const int gm = lane >> 2, tq = lane & 3;
  uint32_t qa0[kMma ? 8 : 1], qa2[kMma ? 8 : 1];
  float mr = -INFINITY, lr = 0.f;
  float oacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  // range CTAs of the MMA path: their clusters' offsets and first page,
  // read before the grid-dependency wait (index data: written before this
  // call, never by the decode's kernels)
  int r_o0 = 0, r_o1 = 0, r_lp0 = -1;
  if constexpr (kMma) {
    const uint32_t* qw = reinterpret_cast<const uint32_t*>(
        q + ((int64_t)b * n_q_heads + (int64_t)h * G + (gm < G ? gm : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qa0[ks] = gm < G ? qw[8 * ks + tq] : 0u;
      qa2[ks] = gm < G ? qw[8 * ks + 4 + tq] : 0u;
    }
    if (role_range && !A.exact_only) {
      // the range's 256 value-sum rows (index data, independent of the
      // previous kernels): four 64-row tiles, each two 64-column boxes, fill
      // the ring (rows past the last cluster row are zero-filled)
      if (tid == 0) {
        mbar_init(&s_vbar, 1);
        mbar_init_fence();
        mbar_arrive_expect(&s_vbar, 4u * 16384u);
        const int y0 = (int)(row0 + (int64_t)blockIdx.x * kRangeW);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          tensor_load_2d(sh + t * 16384, &tm_vsum, 0, y0 + 64 * t, &s_vbar);
          tensor_load_2d(sh + t * 16384 + 8192, &tm_vsum, 64, y0 + 64 * t, &s_vbar);
        }
      }
    } else {
      // rows no copy writes keep finite contents (zero weight times a finite row)
      for (int i = tid; i < 4 * 16384 / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(sh)[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (role_range) {
      const int c0 = (int)blockIdx.x * kRangeW;
      if (c0 + tid < NC) {
        r_o0 = __ldg(off + c0 + tid);
        r_o1 = __ldg(off + c0 + tid + 1);
      }
      r_lp0 = c0 < NC ? __ldg(off + c0) >> kp.page_shift : -1;
      // the block-table entries of the range's pages, in flight until the
      // exact part resolves its rows
      if (r_lp0 >= 0) {
        for (int i = tid; i < kBtStage; i += blockDim.x)
          if (r_lp0 + i < kp.max_pages) cp_async4(&s_bt[i], kp.bt + (int64_t)b * kp.max_pages + r_lp0 + i);
        cp_async_commit();
      }
    }
    // the A operands' rows that no head writes stay zero
    for (int i = tid; i < (int)(sizeof(s_P) / 16); i += blockDim.x)
      reinterpret_cast<uint4*>(&s_P[0][0])[i] = make_uint4(0u, 0u, 0u, 0u);
    if (role_range)
      for (int i = tid; i < (int)(sizeof(s_W) / 16); i += blockDim.x)
        reinterpret_cast<uint4*>(&s_W[0][0])[i] = make_uint4(0u, 0u, 0u, 0u);
  }

  // exact attention over the tokens in s_row[0 .. n) (pool rows, -1 = skip):
  // tiles of TR tokens stream through two ring slots (K and V tiles each),
  // tile t + 2 issued as soon as tile t is consumed; online softmax carried
  // in m_run / l_run / acc
  // MMA path, tiles of 64 tokens: tile t's K rows into ring slot
  // kv_slot(t), its V rows into the next slot (slots 2, 3 for even tiles,
  // 0, 1 for odd ones), each 16 KB slot two 128-byte-swizzled halves of 64
  // rows; one cp.async group per tile
  auto kv_slot = [](int t) { return 2 * ((t + 1) & 1); };
  auto issue_kv = [&](int t, int n) {
    const unsigned char* kb8 = reinterpret_cast<const unsigned char*>(kp.base);
    const unsigned char* vb8 = reinterpret_cast<const unsigned char*>(vp.base);
    unsigned char* r8 = reinterpret_cast<unsigned char*>(ring);
    if (t < (n + 63) / 64) {
      unsigned char* ks_ = r8 + (size_t)kv_slot(t) * 16384;
      unsigned char* vs_ = ks_ + 16384;
      for (int i = tid; i < 64 * 16; i += blockDim.x) {
        const int r = i >> 4, ch = i & 15;
        const int rr = t * 64 + r;
        const int32_t ri = rr < n ? s_row[rr] : -1;
        if (ri >= 0) {
          const int o = (ch >> 3) * 8192 + swz128(r, ch & 7);
          cp_async16(ks_ + o, kb8 + (int64_t)ri * 256 + ch * 16);
          cp_async16(vs_ + o, vb8 + (int64_t)ri * 256 + ch * 16);
        }
      }
    }
    cp_async_commit();
  };
  // exact attention over the tokens of s_row[0 .. n) on the tensor cores;
  // tiles 0 .. issued - 1 were issued by the caller
  auto attend_tokens_mma = [&](int n, int issued) {
    unsigned char* r8 = reinterpret_cast<unsigned char*>(ring);
    const int ntile = (n + 63) / 64;
    auto issue = [&](int t) { issue_kv(t, n); };
    for (int t = issued; t < 2; ++t) issue(t);
    for (int t = 0; t < ntile; ++t) {
      cp_async_wait<1>();
      __syncthreads();
      const unsigned char* ks_ = r8 + (size_t)kv_slot(t) * 16384;
      const unsigned char* vs_ = ks_ + 16384;
      // scores of rows 8 warp .. 8 warp + 7
      float sacc[4] = {0.f, 0.f, 0.f, 0.f};
      const int n0 = 8 * warp;
#pragma unroll
      for (int ks = 0; ks < 8; ks += 2) {
        const int ch = 2 * ks + (lane >> 3);
        uint32_t bm[4];
        ldsm_x4(bm, ks_ + (ch >> 3) * 8192 + swz128(n0 + (lane & 7), ch & 7));
        mma_bf16(sacc, qa0[ks], qa2[ks], bm[0], bm[1]);
        mma_bf16(sacc, qa0[ks + 1], qa2[ks + 1], bm[2], bm[3]);
      }
      const int r0 = n0 + 2 * tq;
      const bool v0 = t * 64 + r0 < n && s_row[t * 64 + r0] >= 0;
      const bool v1 = t * 64 + r0 + 1 < n && s_row[t * 64 + r0 + 1] >= 0;
      const float sc0 = v0 ? sacc[0] * A.scale : -INFINITY;
      const float sc1 = v1 ? sacc[1] * A.scale : -INFINITY;
      float mx = fmaxf(sc0, sc1);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      if (tq == 0 && gm < G) s_wmax[warp][gm] = mx;
      __syncthreads();
      float mt = -INFINITY;
      if (gm < G) {
#pragma unroll
        for (int w = 0; w < NW; ++w) mt = fmaxf(mt, s_wmax[w][gm]);
      }
      const float mnew = fmaxf(mr, mt);
      const float corr = mnew == -INFINITY ? 1.f : __expf(mr - mnew);
      const float p0 = sc0 == -INFINITY ? 0.f : __expf(sc0 - mnew);
      const float p1 = sc1 == -INFINITY ? 0.f : __expf(sc1 - mnew);
      if (gm < G) {
        uint32_t hi, lo;
        split_bf16(p0, p1, hi, lo);
        *reinterpret_cast<uint32_t*>(&s_P[gm][r0]) = hi;
        *reinterpret_cast<uint32_t*>(&s_P[8 + gm][r0]) = lo;
      }
      float ps = p0 + p1;
      ps += __shfl_xor_sync(0xffffffffu, ps, 1);
      ps += __shfl_xor_sync(0xffffffffu, ps, 2);
      if (tq == 0 && gm < G) s_wsum[warp][gm] = ps;
      __syncthreads();
      float lt = 0.f;
      if (gm < G) {
#pragma unroll
        for (int w = 0; w < NW; ++w) lt += s_wsum[w][gm];
      }
      lr = lr * corr + lt;
      mr = mnew;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[nt][e] *= corr;
      // P V for output columns 16 warp .. 16 warp + 15 (one MMA takes both
      // bf16 terms of the weights: high in rows 0..7, low in rows 8..15)
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t a[4];
        ldsm_x4(a, &s_P[(lane & 7) + 8 * ((lane >> 3) & 1)][16 * ks + 8 * (lane >> 4)]);
        const int row = 16 * ks + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int ch = 2 * warp + (lane >> 4);
        uint32_t bm[4];
        ldsm_x4_t(bm, vs_ + (ch >> 3) * 8192 + swz128(row, ch & 7));
        mma_bf16_4(oacc[0], a[0], a[1], a[2], a[3], bm[0], bm[1]);
        mma_bf16_4(oacc[1], a[0], a[1], a[2], a[3], bm[2], bm[3]);
      }
      __syncthreads();  // slots, s_P and the per-warp stats are read before reuse
      issue(t + 2);
    }
    cp_async_wait<0>();
  };

  auto attend_tokens = [&](int n, int issued) {
    if constexpr (kMma) { attend_tokens_mma(n, issued); return; }
    const T* kbase = reinterpret_cast<const T*>(kp.base);
    const T* vbase = reinterpret_cast<const T*>(vp.base);
    const int ntile = (n + TR - 1) / TR;
    auto issue = [&](int t) {
      if (t < ntile) {
        T* kt = ring + (size_t)(t & 1) * TR * D;
        T* vt = ring + (size_t)(2 + (t & 1)) * TR * D;
        for (int i = tid; i < TR * LPR; i += blockDim.x) {
          const int r = i / LPR, ch = i - r * LPR;
          const int rr = t * TR + r;
          const int32_t ri = rr < n ? s_row[rr] : -1;
          if (ri >= 0) {
            cp_async16(kt + r * D + ch * EPL, kbase + (int64_t)ri * D + ch * EPL);
            cp_async16(vt + r * D + ch * EPL, vbase + (int64_t)ri * D + ch * EPL);
          }
        }
      }
      cp_async_commit();
    };
    issue(0);
    issue(1);
    constexpr int ITR = TR / (NW * RPW);   // row steps of a warp per tile
    static_assert(TR % 32 == 0, "tile rows a multiple of the warp size");
    for (int t = 0; t < ntile; ++t) {
      cp_async_wait<1>();
      __syncthreads();
      const T* kt = ring + (size_t)(t & 1) * TR * D;
      const T* vt = ring + (size_t)(2 + (t & 1)) * TR * D;
      // scores: the warp's ITR row steps are independent (unrolled)
#pragma unroll
      for (int it = 0; it < ITR; ++it) {
        const int r = (it * NW + warp) * RPW + rsub;
        const int rr = t * TR + r;
        const bool ok = rr < n && s_row[rr] >= 0;
        float x[EPL];
        if (ok) {
          Elem<T>::unpack(*reinterpret_cast<const uint4*>(kt + r * D + sub * EPL), x);
        } else {
#pragma unroll
          for (int e = 0; e < EPL; ++e) x[e] = 0.f;
        }
        float a[G];
        dot_g<G, EPL>(qv, x, a);
        group_reduce_multi<G, LPR>(a, lane);
        if (sub % (LPR / G) == 0) s_sc[r][jh] = ok ? a[0] : -INFINITY;
      }
      __syncthreads();
      // softmax statistics of the tile for all heads at once (each warp
      // redundantly, no barrier): lane holds rows lane, lane + 32, ...
      float sv[TR / 32][G];
#pragma unroll
      for (int k = 0; k < TR / 32; ++k) load_row<G>(&s_sc[lane + 32 * k][0], sv[k]);
      float mt[G], ps[G], corr[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        mt[g] = sv[0][g];
#pragma unroll
        for (int k = 1; k < TR / 32; ++k) mt[g] = fmaxf(mt[g], sv[k][g]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int g = 0; g < G; ++g) mt[g] = fmaxf(mt[g], __shfl_xor_sync(0xffffffffu, mt[g], o));
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float mnew = fmaxf(m_run[g], mt[g]);
        corr[g] = mnew == -INFINITY ? 1.f : __expf(m_run[g] - mnew);
        m_run[g] = mnew;
        ps[g] = 0.f;
#pragma unroll
        for (int k = 0; k < TR / 32; ++k) {
          sv[k][g] = sv[k][g] == -INFINITY ? 0.f : __expf(sv[k][g] - mnew);
          ps[g] += sv[k][g];
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int g = 0; g < G; ++g) ps[g] += __shfl_xor_sync(0xffffffffu, ps[g], o);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        l_run[g] = l_run[g] * corr[g] + ps[g];
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[g][e] *= corr[g];
      }
      __syncthreads();  // every warp has read the scores
      if (warp == 0) {  // the weights e^(s - m) replace the scores
#pragma unroll
        for (int k = 0; k < TR / 32; ++k) store_row<G>(&s_sc[lane + 32 * k][0], sv[k]);
      }
      __syncthreads();
#pragma unroll
      for (int it = 0; it < ITR; ++it) {
        const int r = (it * NW + warp) * RPW + rsub;
        const int rr = t * TR + r;
        if (!(rr < n && s_row[rr] >= 0)) continue;
        float x[EPL];
        Elem<T>::unpack(*reinterpret_cast<const uint4*>(vt + r * D + sub * EPL), x);
        float pw[G];
        load_row<G>(&s_sc[r][0], pw);
        axpy_g<G, EPL>(pw, x, acc);
      }
      __syncthreads();  // slot t & 1 and s_sc are read before they are refilled
      issue(t + 2);
    }
    cp_async_wait<0>();
  };

  // MMA path: the exact part's output and (m, l) into shared memory, (m, l)
  // into every thread's m_run / l_run
  auto exact_to_shared = [&]() {
    if constexpr (kMma) {
      if (gm < G) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int d = 16 * warp + 8 * nt + 2 * tq;
          *reinterpret_cast<float2*>(&s_o[gm * D + d]) =
              make_float2(oacc[nt][0] + oacc[nt][2], oacc[nt][1] + oacc[nt][3]);
        }
        if (warp == 0 && tq == 0) { s_em[gm] = mr; s_el[gm] = lr; }
      }
      __syncthreads();
#pragma unroll
      for (int g = 0; g < G; ++g) { m_run[g] = s_em[g]; l_run[g] = s_el[g]; }
    }
  };

  // exact attention over the picked clusters' tokens (lists s_pkc / s_pkt /
  // s_pko of n_pk clusters, n_tk tokens), kRowCap tokens per pass; each
  // thread resolves two tokens with their loads (position, page) in flight
  // together; an affected cluster's steady members are skipped.  Pages
  // lp0 .. lp0 + kBtStage - 1 of the block table are read from s_bt when
  // lp0 >= 0 (staged by the caller), the others from global memory.
  auto exact_over_picked = [&](int n_pk, int n_tk, bool dense, int lp0, auto&& first_pass) {
    const int32_t* pm = A.perm + geo.tok_row(b, h);
    for (int p0 = 0; p0 < n_tk; p0 += kRowCap) {
      const int np_ = min(kRowCap, n_tk - p0);
      int slot2[2], cl2[2];
      bool st2[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int t = p0 + tid + k * kStreamThreads;
        slot2[k] = -1;
        cl2[k] = 0;
        st2[k] = false;
        if (t < p0 + np_) {
          int lo = 0, hi = n_pk - 1;  // largest i with s_pkt[i] <= t
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_pkt[mid] <= t) lo = mid; else hi = mid - 1;
          }
          slot2[k] = s_pko[lo] + (t - s_pkt[lo]);
          cl2[k] = s_pkc[lo];
        }
      }
      int pos2[2];
#pragma unroll
      for (int k = 0; k < 2; ++k)   // an affected cluster's tokens: steady?
        pos2[k] = (slot2[k] >= 0 && cl2[k] < 0 && !dense) ? __ldg(pm + slot2[k]) : -1;
      int32_t ro2[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        int64_t ro = -1;
        if (slot2[k] >= 0) {
          const int li = (slot2[k] >> kp.page_shift) - lp0;
          ro = lp0 >= 0 && li >= 0 && li < kBtStage
                   ? pool_row_pg(kp, geo.hkv, 1, h, slot2[k], s_bt[li], status)
                   : pool_row(kp, geo.hkv, 1, b, h, slot2[k], status);
        }
        ro2[k] = (int32_t)ro;
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int t = tid + k * kStreamThreads;
        if (t < np_) {
          st2[k] = pos2[k] >= 0 && (pos2[k] < ns || pos2[k] >= wstart);
          s_row[t] = st2[k] ? -1 : ro2[k];
        }
      }
      __syncthreads();
      // first_pass(np_) may issue the first tiles itself; it returns how many
      attend_tokens(np_, p0 == 0 ? first_pass(np_) : 0);
      __syncthreads();
    }
  };

  bool acc_used = !kMma;   // the CUDA-core accumulators hold part of the output
  pdl_wait();
  if (role_fold) {
    FoldArgs fa{A.est_parts, A.n_chunks, A.partials, A.n_parts, A.n_rng + A.n_sc, G, D};
    fold_role(fa, u, (int)blockIdx.x - A.n_rng - A.n_sc);
  } else if (role_range) {
   if constexpr (kMma) {
    // ------------------------------------ range CTA, tensor-core estimate
    const int c = (int)blockIdx.x * kRangeW + tid;
    const bool inr = c < NC;
    uint32_t key = 0u;
    int af = 0;
    const int o0 = r_o0, o1 = r_o1, lp0 = r_lp0;
    float scv[G];
#pragma unroll
    for (int g = 0; g < G; ++g) scv[g] = 0.f;
    int32_t* afp = A.aff_of + (int64_t)u * A.max_nc + c;
    if (inr) {
      key = A.keys[row0 + c];
      af = *afp;
#pragma unroll
      for (int g = 0; g < G; ++g) scv[g] = A.scores[(row0 + c) * G + g];
    }
    if (tid < kInfoInts) s_info[tid] = A.info[(int64_t)u * kInfoInts + tid];
    __syncthreads();
    if (af != 0) *afp = 0;  // consumed: clean for the next call
    const bool dense = s_info[6] != 0;
    const bool est = !A.exact_only && !dense && s_info[0] < s_info[7] && NC > 0;
    const uint32_t kstar = (uint32_t)s_info[1];
    const int thr = s_info[2];
    const int cnt = o1 - o0;
    const bool pk = inr && cnt > 0 &&
                    (dense || (key != 0u && af >= 0 && (key > kstar || (key == kstar && c <= thr))));
    // estimation zone: a candidate (it keeps a non-steady member) that is not
    // retrieved; an affected one's steady members come back out (ce)
    const bool ez = est && inr && cnt > 0 && !pk && af >= 0;
    const bool ce = ez && af > 0;
    const int dcnt = ce ? af >> 16 : 0;       // its steady members
#pragma unroll
    for (int g = 0; g < G; ++g) {   // per head: the zone's score max, per warp
      const float mx = warp_max(ez ? scv[g] : -INFINITY);
      if (lane == 0) s_wmax[warp][g] = mx;
    }
    int2 tot;
    const int2 incl = block_inclusive_scan2(make_int2((pk ? 1 : 0) | ((ce ? 1 : 0) << 16), pk ? cnt : 0),
                                            scan_sh, &tot);
    const int n_pk = tot.x & 0xffff, n_ce = tot.x >> 16, n_tk = tot.y;
    if (pk) {
      const int i = (incl.x & 0xffff) - 1;
      s_pkc[i] = af > 0 ? ~c : c;             // marked when it has steady members
      s_pkt[i] = incl.y - cnt;
      s_pko[i] = o0;
    }
    if (ce) {
      const int i = (incl.x >> 16) - 1;
      s_cec[i] = (af & 0xffff) - 1;           // its affected-list entry (dV row)
      s_cew[i] = tid;                         // its weights' column
    }
    // weights w = e^(s - m_e) of the zone (zero elsewhere) by head, as two
    // bf16 terms (the value the tensor cores use, also for the denominator
    // terms (cnt - steady members) w and the dV correction)
    float me0 = -INFINITY;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float me = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) me = fmaxf(me, s_wmax[w][g]);
      if (g == 0) me0 = me;
      const float wgt = ez ? __expf(scv[g] - me) : 0.f;
      const __nv_bfloat16 whi = __float2bfloat16_rn(wgt);
      const __nv_bfloat16 wlo = __float2bfloat16_rn(wgt - __bfloat162float(whi));
      s_W[g][tid] = whi;
      s_W[8 + g][tid] = wlo;
      const float lz = warp_sum((__bfloat162float(whi) + __bfloat162float(wlo)) * (float)(cnt - dcnt));
      if (lane == 0) s_wsum[warp][g] = lz;
    }
    // the range's words of the selection bitmap (no atomics: a barrier after
    // a global atomic would wait for its round trip)
    {
      const uint32_t bits = __ballot_sync(0xffffffffu, pk && !dense);
      if (lane == 0) A.sel[(int64_t)u * A.sel_words + blockIdx.x * (kRangeW / 32) + warp] = bits;
    }
    __syncthreads();
    // this lane's head gm: the zone's (m_e, l_e)
    float me_r = -INFINITY, le_r = 0.f;
    if (gm < G) {
#pragma unroll
      for (int w = 0; w < NW; ++w) { me_r = fmaxf(me_r, s_wmax[w][gm]); le_r += s_wsum[w][gm]; }
    }
    // dV rows of the zone's affected clusters, kCorrRows per pass: the first
    // pass in flight with the exact part's tiles (its group completes first)
    constexpr int CHF = D * 4 / 16;
    auto issue_dv = [&](int p0) {
      const int np_ = min(kCorrRows, n_ce - p0);
      for (int k = tid; k < np_ * CHF; k += blockDim.x) {
        const int i = k / CHF, ch = k - i * CHF;
        cp_async16(s_crow + (size_t)i * D * 4 + ch * 16,
                   reinterpret_cast<const unsigned char*>(A.dv + ((int64_t)u * A.cap + s_cec[p0 + i]) * D) +
                       ch * 16);
      }
      cp_async_commit();
    };
    if (n_ce > 0) issue_dv(0);
    // o_e = W Vsum on the tensor cores: A = the weights split into two bf16
    // terms (high in rows 0..7, low in rows 8..15, heads below G), B = the
    // value-sum rows of the ring (ldmatrix.trans); warp w owns output columns
    // 16 w .. 16 w + 15.  k-steps 8..15 (ring slots 2, 3) run first, so the
    // exact part's first tile can load into those slots while k-steps 0..7
    // run; its second tile follows into slots 0, 1.
    auto est_steps = [&](float (&oe)[2][4], int ks0, int ks1) {
      const unsigned char* r8 = sh;
#pragma unroll 4
      for (int ks = ks0; ks < ks1; ++ks) {
        uint32_t a[4];
        ldsm_x4(a, &s_W[(lane & 7) + 8 * ((lane >> 3) & 1)][16 * ks + 8 * (lane >> 4)]);
        const unsigned char* tile = r8 + (size_t)(ks >> 2) * 16384;
        const int row = 16 * (ks & 3) + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int ch = 2 * warp + (lane >> 4);
        uint32_t bm[4];
        ldsm_x4_t(bm, tile + (ch >> 3) * 8192 + swz128(row, ch & 7));
        mma_bf16_4(oe[0], a[0], a[1], a[2], a[3], bm[0], bm[1]);
        mma_bf16_4(oe[1], a[0], a[1], a[2], a[3], bm[2], bm[3]);
      }
    };
    auto estimate = [&](int np_) -> int {
      float oe[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      if (!A.exact_only) mbar_wait(&s_vbar, 0, status);   // (no copies without a zone)
      if (me0 != -INFINITY) est_steps(oe, kRangeW / 32, kRangeW / 16);
      __syncthreads();              // slots 2, 3 are read
      issue_kv(0, np_);
      if (me0 != -INFINITY) est_steps(oe, 0, kRangeW / 32);
      if (gm < G) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int d = 16 * warp + 8 * nt + 2 * tq;
          *reinterpret_cast<float2*>(&s_o[gm * D + d]) =
              make_float2(oe[nt][0] + oe[nt][2], oe[nt][1] + oe[nt][3]);
        }
      }
      __syncthreads();              // slots 0, 1 are read
      issue_kv(1, np_);
      return 2;
    };
    // the exact part, the estimate folded into its first pass
    if (lp0 >= 0) cp_async_wait_dyn(n_ce > 0 ? 1 : 0);   // the block-table window
    __syncthreads();
    exact_over_picked(n_pk, n_tk, dense, lp0, estimate);
    if (n_tk == 0) estimate(0);
    // exact and zone parts of head gm at a common max, into s_o
    if (gm < G) {
      const float M = fmaxf(mr, me_r);
      const float fx = mr == -INFINITY ? 0.f : expf(mr - M);
      const float fe = me_r == -INFINITY ? 0.f : expf(me_r - M);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int d = 16 * warp + 8 * nt + 2 * tq;
        float2* op = reinterpret_cast<float2*>(&s_o[gm * D + d]);
        const float2 e = *op;
        *op = make_float2((oacc[nt][0] + oacc[nt][2]) * fx + e.x * fe,
                          (oacc[nt][1] + oacc[nt][3]) * fx + e.y * fe);
      }
      if (warp == 0 && tq == 0) { s_em[gm] = M; s_el[gm] = lr * fx + le_r * fe; s_f1[gm] = fe; }
    }
    // the steady members' dV, weighted like their clusters, come back out
    float cacc[G][EPL];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EPL; ++e) cacc[g][e] = 0.f;
    for (int p0 = 0; p0 < n_ce; p0 += kCorrRows) {
      const int np_ = min(kCorrRows, n_ce - p0);
      if (p0 > 0) issue_dv(p0);
      cp_async_wait<0>();
      __syncthreads();
      for (int rb = warp * RPW; rb < np_; rb += NW * RPW) {
        const int i = rb + rsub;
        if (i >= np_) continue;
        const float* fr = reinterpret_cast<const float*>(s_crow + (size_t)i * D * 4) + sub * EPL;
        float x[EPL];
#pragma unroll
        for (int e4 = 0; e4 < EPL; e4 += 4) {
          const float4 v = *reinterpret_cast<const float4*>(fr + e4);
          x[e4] = v.x; x[e4 + 1] = v.y; x[e4 + 2] = v.z; x[e4 + 3] = v.w;
        }
        float wv[G];
#pragma unroll
        for (int g = 0; g < G; ++g)
          wv[g] = __bfloat162float(s_W[g][s_cew[p0 + i]]) + __bfloat162float(s_W[8 + g][s_cew[p0 + i]]);
        axpy_g<G, EPL>(wv, x, cacc);
      }
      __syncthreads();
    }
    __syncthreads();   // s_em / s_el / s_f1 are written
    if (tid == 0) part[2] = dense ? 0.f : (float)n_tk;   // retrieved tokens, summed by the merge
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m_run[g] = s_em[g];
      l_run[g] = s_el[g];
      const float fe = s_f1[g];
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[g][e] = -cacc[g][e] * fe;
    }
    acc_used = n_ce > 0;
   } else {
    // ------------------------------------------------- range CTA, CUDA cores
    const int c = (int)blockIdx.x * kRangeW + tid;
    const bool inr = c < NC;
    // one round: unit record, and this thread's cluster: key, affected
    // index, offsets, scores
    uint32_t key = 0u;
    int af = 0, o0 = 0, o1 = 0;
    float scv[G];
#pragma unroll
    for (int g = 0; g < G; ++g) scv[g] = 0.f;
    int32_t* afp = A.aff_of + (int64_t)u * A.max_nc + c;
    if (inr) {
      key = A.keys[row0 + c];
      af = *afp;
      o0 = __ldg(off + c);
      o1 = __ldg(off + c + 1);
#pragma unroll
      for (int g = 0; g < G; ++g) scv[g] = A.scores[(row0 + c) * G + g];
    }
    if (tid < kInfoInts) s_info[tid] = A.info[(int64_t)u * kInfoInts + tid];
    __syncthreads();
    if (af != 0) *afp = 0;  // consumed: clean for the next call
    const bool dense = s_info[6] != 0;
    const bool est = !A.exact_only && !dense && s_info[0] < s_info[7] && NC > 0;
    const uint32_t kstar = (uint32_t)s_info[1];
    const int thr = s_info[2];
    const int cnt = o1 - o0;
    const bool pk = inr && cnt > 0 &&
                    (dense || (key != 0u && af >= 0 && (key > kstar || (key == kstar && c <= thr))));
    int cw = 0, csel = 0;  // correction: count, row selector
    if (est && inr && cnt > 0) {
      if (pk || af < 0) { cw = cnt; csel = c; }
      else if (af > 0 && key != 0u) { cw = af >> 16; csel = ~((af & 0xffff) - 1); }
    }
    int2 tot;
    const int2 incl = block_inclusive_scan2(make_int2((pk ? 1 : 0) | ((cw != 0 ? 1 : 0) << 16), pk ? cnt : 0),
                                            scan_sh, &tot);
    const int n_pk = tot.x & 0xffff, n_ce = tot.x >> 16, n_tk = tot.y;
    if (pk) {
      const int i = (incl.x & 0xffff) - 1;
      s_pkc[i] = af > 0 ? ~c : c;             // marked when it has steady members
      s_pkt[i] = incl.y - cnt;
      s_pko[i] = o0;
    }
    if (cw != 0) {
      const int i = (incl.x >> 16) - 1;
      s_cec[i] = csel;
      s_cew[i] = cw;
#pragma unroll
      for (int g = 0; g < G; ++g) s_ces[i * G + g] = scv[g];
    }
    {
      const uint32_t bits = __ballot_sync(0xffffffffu, pk && !dense);
      if (lane == 0) A.sel[(int64_t)u * A.sel_words + blockIdx.x * (kRangeW / 32) + warp] = bits;
    }
    if (tid == 0) part[2] = dense ? 0.f : (float)n_tk;   // retrieved tokens, summed by the merge
    __syncthreads();
    // exact part: the picked clusters' tokens, kRowCap per pass; each
    // thread resolves two tokens with their loads (position, page) in flight
    // together
    // correction rows, first kCorrRows of them: staged now, in flight with the
    // exact part's tiles (their group completes before the first tile's)
    constexpr int CHF = D * 4 / 16, CHT = RS::ROWB / 16;
    auto issue_corr = [&](int p0) {
      const int np_ = min(kCorrRows, n_ce - p0);
      for (int k = tid; k < np_ * CHF; k += blockDim.x) {
        const int i = k / CHF, ch = k - i * CHF;
        const int sel_ = s_cec[p0 + i];
        unsigned char* slot = s_crow + (size_t)i * D * 4;
        if (sel_ >= 0) {
          if (ch < CHT)
            cp_async16(slot + ch * 16, reinterpret_cast<const unsigned char*>(vsum + (row0 + sel_) * D) + ch * 16);
        } else {
          cp_async16(slot + ch * 16,
                     reinterpret_cast<const unsigned char*>(A.dv + ((int64_t)u * A.cap + ~sel_) * D) + ch * 16);
        }
      }
      cp_async_commit();
    };
    if (n_ce > 0) issue_corr(0);
    exact_over_picked(n_pk, n_tk, dense, -1, [](int) { return 0; });
    exact_to_shared();
    // correction part: -(cnt e^(s - mc) , e^(s - mc) row), kCorrRows rows per pass
    float mc[G], lc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) { mc[g] = -INFINITY; lc[g] = 0.f; }
    float cacc[G][EPL];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EPL; ++e) cacc[g][e] = 0.f;
    if (n_ce > 0) {
      if (warp < G) {   // per head: max, weights and denominator over the entries
        float m = -INFINITY;
        for (int i = lane; i < n_ce; i += 32) m = fmaxf(m, s_ces[i * G + warp]);
        m = warp_max(m);
        float l = 0.f;
        for (int i = lane; i < n_ce; i += 32) {
          const float w = __expf(s_ces[i * G + warp] - m);
          s_ces[i * G + warp] = w;
          l += (float)s_cew[i] * w;
        }
        l = warp_sum(l);
        if (lane == 0) { s_m[warp] = m; s_l[warp] = l; }
      }
      __syncthreads();
#pragma unroll
      for (int g = 0; g < G; ++g) { mc[g] = s_m[g]; lc[g] = s_l[g]; }
      for (int p0 = 0; p0 < n_ce; p0 += kCorrRows) {
        const int np_ = min(kCorrRows, n_ce - p0);
        if (p0 > 0) issue_corr(p0);
        cp_async_wait<0>();
        __syncthreads();
        for (int rb = warp * RPW; rb < np_; rb += NW * RPW) {
          const int i = rb + rsub;
          if (i >= np_) continue;
          const unsigned char* slot = s_crow + (size_t)i * D * 4;
          float x[EPL];
          if (s_cec[p0 + i] >= 0) {
            Elem<T>::unpack(*reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(slot) + sub * EPL), x);
          } else {
            const float* fr = reinterpret_cast<const float*>(slot) + sub * EPL;
#pragma unroll
            for (int e4 = 0; e4 < EPL; e4 += 4) {
              const float4 v = *reinterpret_cast<const float4*>(fr + e4);
              x[e4] = v.x; x[e4 + 1] = v.y; x[e4 + 2] = v.z; x[e4 + 3] = v.w;
            }
          }
          float wv[G];
#pragma unroll
          for (int g = 0; g < G; ++g) wv[g] = s_ces[(p0 + i) * G + g];
          axpy_g<G, EPL>(wv, x, cacc);
        }
        __syncthreads();
      }
    }
    // one part: exact minus correction at a common max
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float M = fmaxf(m_run[g], mc[g]);
      const float f1 = m_run[g] == -INFINITY ? 0.f : expf(m_run[g] - M);
      const float f2 = mc[g] == -INFINITY ? 0.f : expf(mc[g] - M);
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[g][e] = acc[g][e] * f1 - cacc[g][e] * f2;
      l_run[g] = l_run[g] * f1 - lc[g] * f2;
      m_run[g] = M;
      if (tid == 0) s_f1[g] = f1;
    }
   }
  } else {
    // --------------------------------------------------------- steady CTA
    // steady slots j0 .. j0 + 2 TR - 1 of the unit's (slot-sorted) steady list
    const int j0 = ((int)blockIdx.x - A.n_rng) * 2 * TR;
    if (tid < kInfoInts) s_info[tid] = A.info[(int64_t)u * kInfoInts + tid];
    int32_t sl = -1;
    if (tid < 2 * TR && j0 + tid < A.cap) sl = A.st_slot[(int64_t)u * A.cap + j0 + tid];
    __syncthreads();
    const int n_here = max(0, min(2 * TR, (s_info[6] ? 0 : s_info[4]) - j0));
    if (tid < 2 * TR) s_row[tid] = tid < n_here ? (int32_t)pool_row(kp, geo.hkv, 1, b, h, sl, status) : -1;
    __syncthreads();
    if (n_here > 0) attend_tokens(n_here, 0);
    exact_to_shared();
  }
  if (!role_fold) {
    __syncthreads();
    if (acc_used) {
      reduce_and_store<G, EPL, LPR, D>(acc, s_red, warp, sub, rsub, part, kMma ? s_o : nullptr);
    } else if constexpr (kMma) {   // nothing in acc: the part's output is s_o
      for (int i = tid; i < G * D; i += blockDim.x) {
        const int g = i / D;
        part[g * PS + Part<D>::kO + (i - g * D)] = s_o[i];
      }
    }
    if (tid == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) { part[g * PS] = m_run[g]; part[g * PS + 1] = l_run[g]; }
    }
  }

  // ---------------------------------------- last CTA of the unit merges
  // (thread 0's acquire-release add orders the CTA's part writes, which the
  // barrier ordered before it, ahead of the count; the last arrival acquires
  // every other CTA's parts)
  __syncthreads();
  if (tid == 0) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(A.counters + u) : "memory");
    s_last = old == A.n_rng + A.n_sc + A.n_fold - 1;
  }
  __syncthreads();
  if (!s_last) return;
  // parts: [range CTAs | steady CTAs | folded estimation parts]; a unit with
  // nothing estimated (dense, or every candidate retrieved) merges the
  // first two groups alone
  const int32_t* I = A.info + (int64_t)u * kInfoInts;
  const int np = A.n_fold == 0 || (!A.exact_only && !I[6] && I[0] < I[7] && NC > 0)
                     ? A.n_parts : A.n_rng + A.n_sc;
  // the parts stream through the ring and the correction rows (contiguous)
  // in batches: one cp.async round per batch, the first batch issued
  // together with the loads of every part's (m, l)
  constexpr int PFL = G * PS;                       // floats per part
  const int bcap = max(1, (int)((4 * 16384 + kCorrRows * D * 4) / (PFL * 4)));
  float* stage = reinterpret_cast<float*>(sh);
  float* f = s_f;                                   // [np][G] rescale factors
  float* lp = s_f + A.n_parts * G;                  // [np][G] part denominators
  const float* pbase = A.partials + (int64_t)u * A.n_parts * PFL;
  auto stage_batch = [&](int p0) {
    const int nb = min(bcap, np - p0);
    const float4* src = reinterpret_cast<const float4*>(pbase + (int64_t)p0 * PFL);
    for (int i = tid; i < nb * PFL / 4; i += blockDim.x)
      cp_async16(reinterpret_cast<float4*>(stage) + i, src + i);
    cp_async_commit();
  };
  stage_batch(0);
  for (int i = tid; i < np * G; i += blockDim.x) {
    f[i] = __ldcg(pbase + (int64_t)i * PS);
    lp[i] = __ldcg(pbase + (int64_t)i * PS + 1);
  }
  if (warp == NW - 1) {   // the unit's retrieved tokens: the range parts' counts
    int st = 0;
    for (int p = lane; p < A.n_rng; p += 32) st += (int)__ldcg(pbase + (int64_t)p * PFL + 2);
    st = warp_sum_int(st);
    if (lane == 0) const_cast<int32_t*>(I)[3] = st;
  }
  __syncthreads();
  if (warp < G) {
    float M = -INFINITY;
    for (int p = lane; p < np; p += 32) M = fmaxf(M, f[p * G + warp]);
    M = warp_max(M);
    float l = 0.f;
    for (int p = lane; p < np; p += 32) {
      const float mp = f[p * G + warp];
      l += mp == -INFINITY ? 0.f : expf(mp - M) * lp[p * G + warp];
    }
    l = warp_sum(l);
    if (lane == 0) { s_m[warp] = M; s_l[warp] = l; }
  }
  __syncthreads();
  for (int i = tid; i < np * G; i += blockDim.x) {
    const float mp = f[i];
    f[i] = mp == -INFINITY ? 0.f : expf(mp - s_m[i % G]);
  }
  // each thread: output pairs tid, tid + 256, ... of the G x D block, the
  // parts taken two at a time into two accumulators (independent chains)
  constexpr int OPT = (G * D / 2 + kStreamThreads - 1) / kStreamThreads;
  float2 o[OPT];
#pragma unroll
  for (int k = 0; k < OPT; ++k) o[k] = make_float2(0.f, 0.f);
  for (int p0 = 0; p0 < np; p0 += bcap) {
    if (p0 > 0) {
      __syncthreads();  // the previous batch is consumed
      stage_batch(p0);
    }
    cp_async_wait<0>();
    __syncthreads();
    const int nb = min(bcap, np - p0);
#pragma unroll
    for (int k = 0; k < OPT; ++k) {
      const int i = 2 * (tid + k * kStreamThreads);
      if (i < G * D) {
        const int g = i / D, e = i - g * D;
        const float* sp = stage + g * PS + Part<D>::kO + e;
        const float* fp = f + p0 * G + g;
        float2 a0 = o[k], a1 = make_float2(0.f, 0.f);
        int p = 0;
#pragma unroll 4
        for (; p + 1 < nb; p += 2) {
          const float2 v0 = *reinterpret_cast<const float2*>(sp + p * PFL);
          const float2 v1 = *reinterpret_cast<const float2*>(sp + (p + 1) * PFL);
          const float w0 = fp[p * G], w1 = fp[(p + 1) * G];
          a0.x += w0 * v0.x; a0.y += w0 * v0.y;
          a1.x += w1 * v1.x; a1.y += w1 * v1.y;
        }
        if (p < nb) {
          const float2 v0 = *reinterpret_cast<const float2*>(sp + p * PFL);
          const float w0 = fp[p * G];
          a0.x += w0 * v0.x; a0.y += w0 * v0.y;
        }
        o[k] = make_float2(a0.x + a1.x, a0.y + a1.y);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < OPT; ++k) {
    const int i = 2 * (tid + k * kStreamThreads);
    if (i < G * D) {
      const int g = i / D, e = i - g * D;
      const float l = s_l[g];
      const int64_t qh = (int64_t)b * n_q_heads + (int64_t)h * G + g;
      A.out[qh * D + e] = l > 0.f ? o[k].x / l : 0.f;   // (out is only 4-byte aligned)
      A.out[qh * D + e + 1] = l > 0.f ? o[k].y / l : 0.f;
      if (e == 0 && A.lse != nullptr) A.lse[qh] = l > 0.f ? s_m[g] + logf(l) : -INFINITY;
    }
  }
  if (tid == 0) A.counters[u] = 0;
}

template <typename F>
cudaError_t with_types(int dtype, int D, int G, F&& f) {
  auto byG = [&]<typename T, int DD>() -> cudaError_t {
    switch (G) {
      case 1: return f.template operator()<T, DD, 1>();
      case 2: return f.template operator()<T, DD, 2>();
      case 4: return f.template operator()<T, DD, 4>();
      case 8: return f.template operator()<T, DD, 8>();
    }
    return cudaErrorInvalidValue;
  };
  if (dtype == WI_BF16) {
    if (D == 128) return byG.template operator()<__nv_bfloat16, 128>();
    if (D == 64) return byG.template operator()<__nv_bfloat16, 64>();
  } else {
    if (D == 128) return byG.template operator()<float, 128>();
    if (D == 64) return byG.template operator()<float, 64>();
  }
  return cudaErrorInvalidValue;
}

template <typename Kern, typename... Args>
cudaError_t launch_ex(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                      Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace

size_t decode_attend_smem(int dtype, int D, int G, int n_parts) {
  (void)dtype;
  // 1024-byte alignment | ring (also the merge staging) | correction rows |
  // merge factors and denominators
  return 1024 + 4 * 16384 + (size_t)kCorrRows * D * 4 + 2 * (size_t)n_parts * G * 4;
}

size_t decode_topk_smem(int max_nc, int cap) {
  return ((size_t)(max_nc + 31) / 32 + (size_t)cap + 1) * sizeof(int32_t);
}

size_t decode_score_smem(int dtype, int D, int G, int sort_pow2, int cap) {
  const int rowb = D * (dtype == WI_BF16 ? 2 : 4);
  // stream CTA: ring | reduction | histogram | offsets | weights | q
  const size_t chunk = 4 * 16384 + (size_t)(kStreamThreads / 32) * G * D * 4 +
                       (size_t)kHistBins / 2 * 4 + (size_t)2 * (kScoreChunkBytes / rowb + 4) * 4 +
                       (size_t)(kScoreChunkBytes / rowb) * G * 4 +
                       (size_t)2 * G * D * (dtype == WI_BF16 ? 2 : 4);
  // steady role: sort keys (twice for the rank sort) | affected lists |
  // staged pool rows (offsets + rows, lists of up to kSteadyStage)
  const size_t steady = (size_t)8 * sort_pow2 * (sort_pow2 <= kSteadyRank ? 2 : 1) +
                        (size_t)4 * (2 * cap + 2) + 16 + (size_t)8 * kSteadyStage +
                        (size_t)std::min(cap, kSteadyStage) * rowb;
  return std::max(chunk, steady);
}

namespace {

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library); null when unavailable
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// rows x 128 bf16 matrix, boxes of 64 rows x 64 columns, 128-byte swizzle
bool encode_rows128(CUtensorMap* tm, const void* base, int64_t rows) {
  auto fn = encode_fn();
  if (!fn || rows <= 0) return false;
  const cuuint64_t dims[2] = {128, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {128 * 2};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Dynamic shared memory limit, and the full shared-memory carveout for every
// decode kernel: kernels that run back to back (or overlap under
// programmatic dependent launch) then never need the SM's L1 / shared split
// reconfigured between them.
template <typename Kern>
void set_smem(Kern kern, size_t bytes) {
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                       (int)cudaSharedmemCarveoutMaxShared);
}

int sm_count() {
  int dev = 0, n = kNumSMs;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace

cudaError_t launch_decode(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  unsigned char* ws = a.ws;
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + p.off_status);
  float* scores = reinterpret_cast<float*>(ws + p.off_scores);
  uint32_t* keys = reinterpret_cast<uint32_t*>(ws + p.off_keys);
  uint32_t* sel = reinterpret_cast<uint32_t*>(ws + p.off_sel);
  int32_t* info = reinterpret_cast<int32_t*>(ws + p.off_info);
  int32_t* counters = reinterpret_cast<int32_t*>(ws + p.off_counters);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + p.off_hist);
  int32_t* aff_of = reinterpret_cast<int32_t*>(ws + p.off_aff_of);
  int32_t* st_slot = reinterpret_cast<int32_t*>(ws + p.off_st_slot);
  int32_t* st_cl = reinterpret_cast<int32_t*>(ws + p.off_st_cl);
  int32_t* aff_cl = reinterpret_cast<int32_t*>(ws + p.off_aff_cl);
  int32_t* aff_start = reinterpret_cast<int32_t*>(ws + p.off_aff_start);
  float* partials = reinterpret_cast<float*>(ws + p.off_partials);
  float* est_parts = reinterpret_cast<float*>(ws + p.off_est);
  float* dv = reinterpret_cast<float*>(ws + p.off_dv);
  int32_t* nonc = reinterpret_cast<int32_t*>(ws + p.off_nonc);
  cudaEvent_t* ev = a.stage_events;
  const bool pdl = ev == nullptr;  // stage timing serialises the launches
  auto mark = [&](int i) { if (ev) cudaEventRecord(ev[i], s); };

  return with_types(p.dtype, p.D, p.G, [&]<typename T, int D, int G>() -> cudaError_t {
    const T* q = reinterpret_cast<const T*>(a.q);
    SteadyArgs sa{a.invperm, a.labels, a.offsets, a.vp, p.n_sink, p.window, p.cap, p.sort_pow2,
                  st_slot, st_cl, aff_cl, aff_start, nonc, info, dv, aff_of, p.max_nc};
    cudaError_t e;
    mark(0);
    const size_t steady_smem = decode_score_smem(p.dtype, D, G, p.sort_pow2, p.cap);
    const int n_tot = p.U * p.n_score_blocks;
    e = cudaErrorInvalidValue;
    // tensor-core path (bf16, d = 128): K_A scores only; the attend kernel's
    // range CTAs estimate from the value sums through their own tensor map
    CUtensorMap tm_vsum;
    std::memset(&tm_vsum, 0, sizeof(tm_vsum));
    bool done = false;
    if constexpr (std::is_same_v<T, __nv_bfloat16> && D == 128) {
      CUtensorMap tmc;
      if (!encode_rows128(&tmc, a.centroids, p.ncl) || !encode_rows128(&tm_vsum, a.value_sums, p.ncl))
        return cudaErrorInvalidValue;
      const size_t smem = std::max(MmaSmem<G>::kTotal, steady_smem);
      set_smem(wave_score_mma_kernel<G>, smem);
      int per_sm = 0;
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, wave_score_mma_kernel<G>,
                                                    kStreamThreads, smem);
      const int n_stream = std::max(1, std::min(n_tot, std::max(1, per_sm) * sm_count() - p.U));
      e = launch_ex(wave_score_mma_kernel<G>, dim3(p.U + n_stream), dim3(kStreamThreads), smem, s,
                    false, p.geo, q, p.Hq, tmc, a.offsets, scores, keys, hist, p.scale,
                    p.n_score_blocks, n_stream, sa, status);
      done = true;
    }
    if (!done) {
      const size_t score_smem = steady_smem;
      set_smem(wave_score_kernel<T, D, G>, score_smem);
      int per_sm = 0;
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, wave_score_kernel<T, D, G>,
                                                    kStreamThreads, score_smem);
      const int n_stream = std::max(1, std::min(n_tot, std::max(1, per_sm) * sm_count() - p.U));
      e = launch_ex(wave_score_kernel<T, D, G>, dim3(p.U + n_stream), dim3(kStreamThreads),
                    score_smem, s, false, p.geo, q, p.Hq, reinterpret_cast<const T*>(a.centroids),
                    reinterpret_cast<const T*>(a.value_sums), a.offsets, scores, keys, hist,
                    est_parts, p.scale, p.n_score_blocks, n_stream, sa, status);
    }
    if (e != cudaSuccess) return e;
    mark(1);
    const size_t topk_smem = decode_topk_smem(p.max_nc, p.cap);
    set_smem(wave_topk_kernel, topk_smem);
    TopkArgs ta{keys, hist, nonc, p.cap, p.topk_clusters, p.topk_fraction, info};
    e = launch_ex(wave_topk_kernel, dim3(p.U), dim3(kTopkThreads), topk_smem, s, pdl, p.geo, ta,
                  status);
    if (e != cudaSuccess) return e;
    mark(2);
    AttendArgs A{keys, scores, info, aff_of, p.max_nc, aff_start, st_slot, dv, p.cap, a.perm,
                 p.n_sink, p.window, sel, p.sel_words, est_parts, p.n_score_blocks, p.n_rng, p.n_sc,
                 p.n_fold, p.n_parts, partials, counters, a.out, a.lse, p.scale, p.exact_only};
    const size_t smem = decode_attend_smem(p.dtype, D, G, p.n_parts);
    set_smem(wave_attend_kernel<T, D, G>, smem);
    e = launch_ex(wave_attend_kernel<T, D, G>, dim3(p.n_rng + p.n_sc + p.n_fold, p.U), dim3(kStreamThreads),
                  smem, s, pdl, p.geo, q, p.Hq, a.kp, a.vp,
                  reinterpret_cast<const T*>(a.value_sums), a.offsets, A, tm_vsum, status);
    if (e != cudaSuccess) return e;
    mark(3);
    return cudaGetLastError();
  });
}

}  // namespace wi

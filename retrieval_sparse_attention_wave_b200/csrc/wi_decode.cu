// Decode-step kernels of the wave index (sm_100a).
//
// One decode step is the query-dependent phase of the method (RetroInfer
// technical summary, section 2.A, items 1-3; Vortex summary, section 2.A
// forward_indexer).  Three launches, chained with programmatic dependent
// launch so each one's prologue overlaps the previous one's tail:
//
//  K_A score    q . centroid / sqrt(d) for every cluster and q head, and the
//               group-max selection key (item 2, the index lookup).  U extra
//               CTAs resolve the steady zone (item 1): sink and window
//               positions -> slots -> clusters, run-length encoded.
//  K_B topk     exact radix select (11+11+10-bit digits) of the k best
//               candidate clusters per KV head, ties to the lower id (Vortex
//               2.C Top-K), and the gather plan (slot starts, token prefix,
//               split boundaries).
//  K_C attend + estimate
//               attend CTAs: gather the retrieved clusters' rows and the
//               steady rows from the cluster-permuted paged layout into
//               shared memory (16-byte cp.async) and run split-K exact
//               attention (items 1 and 2);
//               estimate CTAs: prefetch their value-sum rows into a shared
//               memory ring before waiting on K_B, then add every other
//               candidate cluster as cnt' * e^s with value sum Vsum'
//               (item 3 Estimation Zone);
//               the last CTA of each unit merges all parts by log-sum-exp.
//
// The score / estimate GEMVs have M = G <= 8 rows, so they run on the CUDA
// cores (FFMA); every row is spread over LPR = d*sizeof(T)/16 lanes.
#include <cfloat>
#include <climits>
#include <algorithm>
#include <cmath>

#include "wi_common.cuh"
#include "wi_plan.h"

namespace wi {

const char* const kDecodeStageNames[kDecodeStages] = {"score_estimate", "topk", "attend"};

namespace {

template <typename T, int D>
struct RowShape {
  static constexpr int EPL = Elem<T>::kPerVec;  // elements per lane (one 16-B vector)
  static constexpr int LPR = D / EPL;           // lanes per row
  static constexpr int RPW = 32 / LPR;          // rows per warp step
  static constexpr int ROWB = D * (int)sizeof(T);
  static constexpr int TILE = 16384 / ROWB;     // rows per 16 KB shared-memory tile
};

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

// Binary search in a sorted shared-memory array: index of x or -1.
__device__ __forceinline__ int find_sorted(const int32_t* a, int n, int x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < x) lo = mid + 1; else hi = mid;
  }
  return (lo < n && a[lo] == x) ? lo : -1;
}

struct SteadyArgs {
  const int32_t* invperm;
  const int32_t* labels;
  const int32_t* offsets;
  Pool vp;
  int n_sink, window, cap, sort_pow2;
  int32_t *st_slot, *st_cl, *aff_cl, *aff_start, *nonc, *info;
  float* dv;  // [U][cap][D] fp32: sum of the steady members' values per affected cluster
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
      if (full - (s_ast[i + 1] - s_ast[i]) <= 0) nonc[1 + atomicAdd(&s_nnc, 1)] = c;
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

template <int G, int EPL, int LPR, int D>
__device__ __forceinline__ void reduce_and_store(float (&acc)[G][EPL], float* s_red, int warp,
                                                 int sub, int rsub, float* part) {
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
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += s_red[(w * G + g) * D + e];
    part[g * Part<D>::kStride + Part<D>::kO + e] = v;
  }
}

// (m, l, o) = (-inf, 0, 0) for each of G heads, PS floats apart
__device__ __forceinline__ void empty_part(float* part, int G, int PS) {
  for (int i = threadIdx.x; i < G * PS; i += blockDim.x) part[i] = (i % PS) == 0 ? -INFINITY : 0.f;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kStreamThreads, G >= 8 ? 2 : 3)
wave_score_kernel(const Geo geo, const T* __restrict__ q, int n_q_heads, const T* __restrict__ cent,
                  const T* __restrict__ vsum, const int32_t* __restrict__ offsets,
                  float* __restrict__ scores, uint32_t* __restrict__ keys,
                  int32_t* __restrict__ hist_g, float* __restrict__ est_parts, float scale,
                  int n_score_blocks, const SteadyArgs sa, uint32_t* status) {
  using RS = RowShape<T, D>;
  constexpr int EPL = RS::EPL, LPR = RS::LPR, RPW = RS::RPW, TR = RS::TILE;
  constexpr int NW = kStreamThreads / 32;
  constexpr int CROWS = kScoreChunkBytes / RS::ROWB;  // clusters per CTA
  constexpr int NT = CROWS / TR;                      // 16 KB tiles per matrix
  constexpr int PS = Part<D>::kStride;
  static_assert(G <= LPR && G <= NW, "group larger than lanes per row or warps");
  static_assert(NT == 2, "two tiles per matrix");
  extern __shared__ __align__(16) unsigned char sh_dyn[];
  __shared__ float s_m[G], s_l[G];
  pdl_launch_dependents();
  const int u = blockIdx.y;
  if (blockIdx.x == n_score_blocks) {
    steady_role<T, D>(geo, u, sa, status, sh_dyn);
    return;
  }
  const int b = u / geo.hkv, h = u - b * geo.hkv;
  const int NC = geo.NC(b);
  const int c0 = blockIdx.x * CROWS;
  float* part = est_parts + ((int64_t)u * n_score_blocks + blockIdx.x) * G * PS;
  const int tid = threadIdx.x;
  if (c0 >= NC) {  // past this sequence's clusters: an empty part
    empty_part(part, G, PS);
    return;
  }
  const int nrows = min(NC - c0, CROWS);
  // shared: centroid rows [CROWS][D] | value-sum rows [CROWS][D] | histogram,
  //         two 16-bit counts per word [kHistBins/2] | offsets [CROWS+1 (+3)]
  //         | scores, then weights [CROWS][G]
  T* crow = reinterpret_cast<T*>(sh_dyn);
  T* vrow = crow + CROWS * D;
  uint32_t* hist = reinterpret_cast<uint32_t*>(vrow + CROWS * D);
  int* s_off = reinterpret_cast<int*>(hist + kHistBins / 2);
  float* s_w = reinterpret_cast<float*>(s_off + CROWS + 4);
  const int lane = tid & 31, warp = tid >> 5;
  const int sub = lane % LPR, rsub = lane / LPR;
  const int64_t row0 = geo.cl_row(b, h);
#pragma unroll
  for (int t = 0; t < 2 * NT; ++t) {
    const T* src = (t < NT ? cent : vsum) + (row0 + c0) * D;
    T* dst = t < NT ? crow : vrow;
    const int r0 = (t % NT) * TR, nr = min(TR, nrows - r0);
    for (int i = tid; i < nr * LPR; i += blockDim.x)
      cp_async16(dst + (r0 * LPR + i) * EPL, src + (r0 * LPR + i) * EPL);
    cp_async_commit();
  }
  const int32_t* off = offsets + geo.off_row(b, h) + c0;
  for (int i = tid; i <= nrows; i += blockDim.x) s_off[i] = __ldg(off + i);
  for (int i = tid; i < kHistBins / 2; i += blockDim.x) hist[i] = 0u;
  float qv[G][EPL];
  load_q<T, D, G>(q, n_q_heads, b, h, sub, scale, qv);
  const int j = sub / (LPR / G);
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    cp_async_wait_dyn(2 * NT - 1 - t);  // centroid tile t has landed
    __syncthreads();
    const int r1 = min(nrows, (t + 1) * TR);
    for (int rb = t * TR + warp * RPW; rb < r1; rb += NW * RPW) {
      const int r = rb + rsub;
      const bool ok = r < r1;
      float x[EPL];
      if (ok) {
        Elem<T>::unpack(*reinterpret_cast<const uint4*>(crow + r * D + sub * EPL), x);
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
          scores[(row0 + c0 + r) * G + j] = acc[0];
          s_w[r * G + j] = acc[0];
        }
        if (sub == 0) {
          const uint32_t key = (s_off[r + 1] - s_off[r]) > 0 ? ordered_key(m) : 0u;
          keys[row0 + c0 + r] = key;
          if (key) atomicAdd(&hist[key >> (kHistShift + 1)], 1u << (16 * ((key >> kHistShift) & 1u)));
        }
      }
    }
  }
  __syncthreads();
  {
    int* hg = hist_g + (int64_t)u * kHistBins;
    for (int i = tid; i < kHistBins / 2; i += blockDim.x) {
      const uint32_t w = hist[i];
      if (w & 0xffffu) atomicAdd(hg + 2 * i, (int)(w & 0xffffu));
      if (w >> 16) atomicAdd(hg + 2 * i + 1, (int)(w >> 16));
    }
  }
  // the chunk's max, weights and denominator per head (warp g: head g)
  if (warp < G) {
    float m = -INFINITY;
    for (int r = lane; r < nrows; r += 32) m = fmaxf(m, s_w[r * G + warp]);
    m = warp_max(m);
    float l = 0.f;
    for (int r = lane; r < nrows; r += 32) {
      const int cnt = s_off[r + 1] - s_off[r];
      const float w = cnt > 0 ? __expf(s_w[r * G + warp] - m) : 0.f;
      s_w[r * G + warp] = w;
      l += (float)cnt * w;
    }
    l = warp_sum(l);
    if (lane == 0) { s_m[warp] = m; s_l[warp] = l; }
  }
  __syncthreads();
  float acc[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    cp_async_wait_dyn(NT - 1 - t);  // value-sum tile t has landed
    __syncthreads();
    const int r1 = min(nrows, (t + 1) * TR);
    for (int rb = t * TR + warp * RPW; rb < r1; rb += NW * RPW) {
      const int r = rb + rsub;
      if (r < r1) {
        float x[EPL];
        Elem<T>::unpack(*reinterpret_cast<const uint4*>(vrow + r * D + sub * EPL), x);
        float wv[G];
#pragma unroll
        for (int g = 0; g < G; ++g) wv[g] = s_w[r * G + g];
        axpy_g<G, EPL>(wv, x, acc);
      }
    }
  }
  // the cross-warp reduction reuses the centroid rows (<= 32 KB, read long ago)
  reduce_and_store<G, EPL, LPR, D>(acc, reinterpret_cast<float*>(sh_dyn), warp, sub, rsub, part);
  if (tid < G) { part[tid * PS] = s_m[tid]; part[tid * PS + 1] = s_l[tid]; }
}

// ----------------------------------------------------------------- K_B topk
// One CTA per unit.  Every global read it needs is issued in one round at
// the start (unit record, first-digit histogram, non-candidate, steady and
// affected lists, the sequence's block-table row, and the first kTopkRound
// keys and offsets into registers, 16 consecutive cluster ids per thread);
// all later steps work in shared memory and registers:
//  1. the first radix digit's histogram comes from K_A (zeroed after use, so
//     the workspace is clean for the next call), minus the non-candidates; a
//     histogram whose total disagrees with the candidate count is flagged
//     and the select falls back to a full radix select over all keys;
//  2. the keys of the threshold bin (1-2% of them) get a second 11-bit digit
//     histogram, and the few keys of its threshold bin are ranked exactly by
//     (key desc, id asc) (Vortex 2.C Top-K: exact, ties to the lower id);
//  3. one block scan orders the selection: each thread writes its selected
//     clusters (ascending ids) with their token starts; then each warp
//     expands its threads' selected clusters into the gather list (pool rows
//     of their tokens, -1 for steady members), and the steady slots' rows
//     follow.
constexpr int kTopkPerLane = 16;
constexpr int kTopkRound = kTopkThreads * kTopkPerLane;   // 8192 ids per round
constexpr int kTopkCand = 1024;
constexpr int kTopkCand2 = 256;

// Fold CTAs of K_B (blockIdx.x >= 1, beside the unit's top-k CTA): each
// log-sum-exp combines kFold consecutive chunk parts of K_A into one part of
// the unit's final merge, so the merge reads a few parts instead of one per
// 32 KB chunk.  All loads of a fold are issued before the first use.
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
  const int32_t* offsets;
  int32_t* hist_g;
  const int32_t* nonc;       // [U][cap+1]: count, then the non-candidate clusters
  const int32_t* st_slot;    // [U][cap]: steady slots, ascending
  const int32_t* aff_cl;     // [U][cap]: affected clusters, ascending
  const int32_t* aff_start;  // [U][cap+1]: their first steady index
  int cap;
  int topk_clusters;
  double topk_fraction;
  int32_t *sel, *sel_tok, *info;
  Pool kp;
  int32_t* gather;
  int64_t gather_stride;
  int bt_cap;                // block-table entries staged in shared memory
};

__global__ void __launch_bounds__(kTopkThreads)
wave_topk_kernel(const Geo geo, const TopkArgs A, const FoldArgs fa, uint32_t* status) {
  // dynamic shared: excluded bitmask [ceil(NCmax/32)] | non-candidates [cap+1]
  //   | steady slots [cap] | affected clusters [cap] | their starts [cap+1]
  //   | block-table row [bt_cap]
  extern __shared__ __align__(16) int32_t sdyn[];
  __shared__ __align__(16) int hist[kHistBins];
  __shared__ unsigned long long cand[kTopkCand];
  __shared__ unsigned long long cand2[kTopkCand2];
  __shared__ int scan_sh[64];
  __shared__ int s_info[kInfoInts];
  __shared__ int s_ctl[8];
  pdl_launch_dependents();
  if (blockIdx.x > 0) {
    pdl_wait();
    fold_role(fa, blockIdx.y, blockIdx.x - 1);
    return;
  }
  constexpr int PT = kTopkPerLane;
  const int tid = threadIdx.x, nt = kTopkThreads, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int u = blockIdx.y, b = u / geo.hkv, h = u - b * geo.hkv;
  const int NC = geo.NC(b), Tb = geo.T(b);
  const int nmask = (NC + 31) >> 5;
  const int cap = A.cap;
  uint32_t* sx = reinterpret_cast<uint32_t*>(sdyn);
  int32_t* snc = sdyn + nmask;
  int32_t* ss = snc + cap + 1;
  int32_t* sacl = ss + cap;
  int32_t* sast = sacl + cap;
  int32_t* sbt = sast + cap + 1;
  const int page_shift = A.kp.page_shift;
  const int n_bt = (Tb + (1 << page_shift) - 1) >> page_shift;
  const bool bt_sh = n_bt <= A.bt_cap && n_bt <= A.kp.max_pages;
  for (int i = tid; i < nmask; i += nt) sx[i] = 0u;
  if (tid == 0) { s_ctl[0] = 0; s_ctl[5] = 0; }
  int32_t* I = A.info + (int64_t)u * kInfoInts;
  const int64_t row0 = geo.cl_row(b, h);
  int32_t* pre = A.sel_tok + row0 + u;
  int* hg = A.hist_g + (int64_t)u * kHistBins;
  const int k_req = A.topk_clusters >= 0 ? A.topk_clusters
                                         : (int)ceil(A.topk_fraction * (double)NC);
  const uint32_t* kk = A.keys + row0;
  const int32_t* off = A.offsets + geo.off_row(b, h);
  int32_t* gat = A.gather + (int64_t)u * A.gather_stride;
  const int n_rounds = (NC + kTopkRound - 1) / kTopkRound;
  uint32_t kr[PT];
  int ofs[PT + 1];
  auto cid = [&](int r, int i) { return r * kTopkRound + tid * PT + i; };
  auto load_round = [&](int r) {                    // raw keys and offsets of round r
#pragma unroll
    for (int i = 0; i < PT; ++i) {
      const int c = cid(r, i);
      kr[i] = c < NC ? kk[c] : 0u;
      ofs[i] = c <= NC ? __ldg(off + c) : 0;
    }
    const int c = cid(r, PT);
    ofs[PT] = c <= NC ? __ldg(off + c) : 0;
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
  for (int i = tid; i <= cap; i += nt) {
    cp_async4(snc + i, A.nonc + (int64_t)u * (cap + 1) + i);
    cp_async4(sast + i, A.aff_start + (int64_t)u * (cap + 1) + i);
    if (i < cap) {
      cp_async4(ss + i, A.st_slot + (int64_t)u * cap + i);
      cp_async4(sacl + i, A.aff_cl + (int64_t)u * cap + i);
    }
  }
  if (bt_sh)
    for (int i = tid; i < n_bt; i += nt) cp_async4(sbt + i, A.kp.bt + (int64_t)b * A.kp.max_pages + i);
  cp_async_commit();
  load_round(0);
  cp_async_wait<0>();
  __syncthreads();
  for (int i = tid; i < kHistBins; i += nt) hg[i] = 0;   // clean for the next call
  const int n_st = s_info[4];
  const int dense = s_info[6];
  const int n_aff = dense ? 0 : min(max(s_info[5], 0), cap);
  auto row_of = [&](int slot) -> int32_t {
    if (bt_sh) {
      const int lp = slot >> page_shift;
      const int pg = (slot >= 0 && lp < n_bt) ? sbt[lp] : -1;
      if (pg < 0 || (int64_t)pg >= A.kp.n_pages) {
        flag_error(status, slot < 0 || lp >= n_bt ? WI_DEV_BAD_SLOT : WI_DEV_BAD_PAGE);
        return -1;
      }
      return (((int32_t)pg * geo.hkv + h) << page_shift) + (slot & ((1 << page_shift) - 1));
    }
    const int64_t ro = pool_row(A.kp, geo.hkv, 1, b, h, slot, status);
    return ro < 0 ? -1 : (int32_t)ro;
  };
  if (dense) {  // the attend CTAs take all slots in order
    for (int t = tid; t < Tb; t += nt) gat[t] = row_of(t);
    if (tid == 0) {
      I[0] = 0; I[1] = (int32_t)0xFFFFFFFFu; I[2] = -1; I[3] = 0; I[7] = 0;
      pre[0] = 0;
    }
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

  // histogram total -> threshold bin of the first digit (valid if consistent)
  int hs = 0;
  for (int i = tid; i < kHistBins; i += nt) hs += hist[i];
  int hist_total;
  block_inclusive_scan(hs, scan_sh, &hist_total);
  int ksel = min(max(k_req, 0), hist_total);
  // bin holding the krem-th largest of the histogram (bins scanned downwards);
  // *above: count in the bins above it
  auto first_digit = [&](int krem, int* above) -> int {
    // thread t owns bins 2047-4t .. 2044-4t (descending)
    int c4[4], s4 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) { c4[i] = hist[kHistBins - 1 - 4 * tid - i]; s4 += c4[i]; }
    int tot;
    const int incl = block_inclusive_scan(s4, scan_sh, &tot);
    int acc = incl - s4;
    if (acc < krem && incl >= krem) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (acc + c4[i] >= krem) { s_ctl[1] = kHistBins - 1 - 4 * tid - i; s_ctl[2] = acc; break; }
        acc += c4[i];
      }
    }
    __syncthreads();
    *above = s_ctl[2];
    return s_ctl[1];
  };
  int bin1 = -1, above1 = 0;
  if (ksel > 0 && ksel < hist_total) bin1 = first_digit(ksel, &above1);
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

  // pass A: candidate count, and the keys of the threshold bin
  int mine = 0;
  for (int r = 0; r < n_rounds; ++r) {
    if (r > 0) { load_round(r); mask_round(r); }
#pragma unroll
    for (int i = 0; i < PT; ++i) {
      const uint32_t key = kr[i];
      mine += key != 0u;
      append(key != 0u && (int)(key >> kHistShift) == bin1,
             ((unsigned long long)key << 32) | (0xFFFFFFFFu - (uint32_t)cid(r, i)), cand, kTopkCand,
             &s_ctl[0]);
    }
  }
  int ncand;
  block_inclusive_scan(mine, scan_sh, &ncand);
  const int nbin = s_ctl[0];
  const bool hist_ok = ncand == hist_total;
  if (!hist_ok && tid == 0) flag_error(status, WI_DEV_BAD_HIST);
  ksel = min(max(k_req, 0), ncand);
  uint32_t kstar;
  int thr;
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
    const int bin2 = first_digit(krem, &above2);
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
      const int d = first_digit(krem, &ab) & (nbins - 1);
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
  auto picked = [&](int c, uint32_t key) -> bool {  // key: candidate key or 0
    return key != 0u && (key > kstar || (key == kstar && c <= thr));
  };

  // ordered compaction and gather list, round by round
  int sel_run = 0, tok_run = 0;   // totals of earlier rounds
  for (int r = 0; r < n_rounds; ++r) {
    if (n_rounds > 1) { load_round(r); mask_round(r); }
    int cnt = 0, tk = 0;
#pragma unroll
    for (int i = 0; i < PT; ++i) {
      const bool p = picked(cid(r, i), kr[i]);
      cnt += p;
      tk += p ? ofs[i + 1] - ofs[i] : 0;
    }
    int2 tot;
    const int2 incl = block_inclusive_scan2(make_int2(cnt, tk), scan_sh, &tot);
    int si = sel_run + incl.x - cnt, st = tok_run + incl.y - tk;
    // this thread's selected clusters: list entries, and per cluster the
    // token start and the range of its steady members (affected clusters)
    unsigned pmask = 0u;
    int tst[PT], aj[PT];
#pragma unroll
    for (int i = 0; i < PT; ++i) {
      const int c = cid(r, i);
      tst[i] = st;
      aj[i] = -1;
      if (picked(c, kr[i])) {
        pmask |= 1u << i;
        A.sel[row0 + si] = c;
        pre[si] = st;
        aj[i] = n_aff ? find_sorted(sacl, n_aff, c) : -1;
        ++si;
        st += ofs[i + 1] - ofs[i];
      }
    }
    // the warp expands its lanes' selected clusters, one cluster at a time
#pragma unroll
    for (int i = 0; i < PT; ++i) {
      unsigned bal = __ballot_sync(0xffffffffu, (pmask >> i) & 1u);
      while (bal) {
        const int src = __ffs(bal) - 1;
        bal &= bal - 1u;
        const int o0 = __shfl_sync(0xffffffffu, ofs[i], src);
        const int n = __shfl_sync(0xffffffffu, ofs[i + 1], src) - o0;
        const int t0 = __shfl_sync(0xffffffffu, tst[i], src);
        const int j = __shfl_sync(0xffffffffu, aj[i], src);
        const int s0 = j >= 0 ? sast[j] : 0, s1 = j >= 0 ? sast[j + 1] : 0;
        for (int t = lane; t < n; t += 32) {
          const int slot = o0 + t;
          bool steady = false;
          for (int k = s0; k < s1; ++k) steady |= ss[k] == slot;
          gat[t0 + t] = steady ? -1 : row_of(slot);
        }
      }
    }
    sel_run += tot.x;
    tok_run += tot.y;
  }
  const int total_tok = tok_run;
  for (int j = tid; j < n_st; j += nt) gat[total_tok + j] = row_of(ss[j]);
  if (tid == 0) {
    pre[ksel] = total_tok;
    I[0] = ksel; I[1] = (int32_t)kstar; I[2] = thr; I[3] = total_tok; I[7] = ncand;
  }
}

// --------------------------------------------------- K_C attend + correct
// attend CTAs: split-K exact attention over the gather list (retrieved
// clusters' non-steady rows, then the steady rows);
// correction CTAs: the part -(what K_A's chunk parts counted that the
// estimation zone leaves out), kNegChunk clusters per CTA, their rows staged
// in shared memory by one round of cp.async;
// the last CTA of each unit merges the attend parts, the correction parts and
// K_B's folded estimation parts by log-sum-exp.
constexpr int kNegChunk = kNegRows;

struct AttendArgs {
  const int32_t *gather, *aff_cl, *aff_start, *sel;
  const float* dv;
  int64_t gather_stride;
  const int32_t* info;
  const float* scores;
  const uint32_t* keys;
  int cap, n_splits, n_neg, n_parts, wcap;
  float* partials;
  int32_t* counters;
  float* out;
  float* lse;
  float scale;
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kStreamThreads)
wave_attend_estimate_kernel(const Geo geo, const T* __restrict__ q, int n_q_heads, const Pool kp,
                            const Pool vp, const T* __restrict__ vsum,
                            const int32_t* __restrict__ offsets, const AttendArgs A,
                            uint32_t* status) {
  using RS = RowShape<T, D>;
  constexpr int EPL = RS::EPL, LPR = RS::LPR, RPW = RS::RPW, TR = RS::TILE;
  constexpr int NW = kStreamThreads / 32;
  static_assert(TR % (NW * RPW) == 0, "tile must be a multiple of rows per CTA step");
  static_assert(kNegChunk * D * 4 <= 4 * 16384, "correction rows must fit the ring");
  extern __shared__ __align__(16) unsigned char sh[];
  // shared layout: [ring 64 KB: attend K x2, V x2 tiles | correction rows,
  //                 kNegChunk slots of D fp32; the final cross-warp reduction
  //                 and the merge reuse it] [s_w wcap*G f32] [s_cnt, s_ent kNegChunk i32]
  T* ring = reinterpret_cast<T*>(sh);
  float* s_red = reinterpret_cast<float*>(sh);
  float* s_w = reinterpret_cast<float*>(sh + 4 * 16384);
  int* s_cnt = reinterpret_cast<int*>(s_w + A.wcap * G);
  int* s_ent = s_cnt + kNegChunk;
  __shared__ int64_t s_row[2][TR];
  __shared__ float s_sc[TR][G];
  __shared__ int s_last;
  __shared__ float s_m[G], s_l[G], s_part[NW][G];
  __shared__ int s_info[kInfoInts];

  const int u = blockIdx.y, b = u / geo.hkv, h = u - b * geo.hkv;
  const int NC = geo.NC(b);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tid = threadIdx.x;
  const int sub = lane % LPR, rsub = lane / LPR;
  const int jh = sub / (LPR / G);
  const int64_t row0 = geo.cl_row(b, h);
  const int32_t* off = offsets + geo.off_row(b, h);
  const bool role_neg = (int)blockIdx.x >= A.n_splits;
  constexpr int PS = Part<D>::kStride;
  float* part = A.partials + ((int64_t)u * A.n_parts + blockIdx.x) * G * PS;

  float acc[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;

  if (role_neg) {
    // ---------------------------------------------------------- correction
    // entries e0 .. e0+ne-1 of [retrieved clusters (ascending) | affected
    // clusters]: a retrieved cluster or an affected one left without a
    // non-steady member counts in full (cnt, Vsum); another affected one
    // that is estimated counts its steady members (their count, dV); an
    // affected one that is also retrieved was counted with the retrieved.
    pdl_wait();
    if (tid < kInfoInts) s_info[tid] = A.info[(int64_t)u * kInfoInts + tid];
    __syncthreads();
    const int ksel = s_info[0];
    const int n_aff = min(A.cap, s_info[5]);
    const bool est = !s_info[6] && ksel < s_info[7] && NC > 0;
    const int e0 = (blockIdx.x - A.n_splits) * kNegChunk;
    const int ne = est ? max(0, min(kNegChunk, ksel + n_aff - e0)) : 0;
    const uint32_t kstar = (uint32_t)s_info[1];
    const int thr = s_info[2];
    float m_loc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) m_loc[g] = -INFINITY;
    for (int i = tid; i < ne; i += blockDim.x) {
      const int e = e0 + i;
      int c, cnt, ent;
      if (e < ksel) {
        c = min(max(A.sel[row0 + e], 0), NC - 1);
        cnt = __ldg(off + c + 1) - __ldg(off + c);
        ent = c;
      } else {
        const int jj = e - ksel;
        c = min(max(A.aff_cl[(int64_t)u * A.cap + jj], 0), NC - 1);
        const int32_t* as = A.aff_start + (int64_t)u * (A.cap + 1) + jj;
        const int dc = as[1] - as[0];
        const int full = __ldg(off + c + 1) - __ldg(off + c);
        const uint32_t key = A.keys[row0 + c];
        if (full - dc <= 0) { cnt = full; ent = c; }
        else if (key > kstar || (key == kstar && c <= thr)) { cnt = 0; ent = c; }
        else { cnt = dc; ent = ~jj; }
      }
      s_cnt[i] = cnt;
      s_ent[i] = ent;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float v = cnt > 0 ? A.scores[(row0 + c) * G + g] : -INFINITY;
        s_w[i * G + g] = v;
        m_loc[g] = fmaxf(m_loc[g], v);
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float v = warp_max(m_loc[g]);
      if (lane == 0) s_part[warp][g] = v;
    }
    __syncthreads();
    // stage the rows: slot i holds D fp32 (dV) or D elements of T (Vsum)
    constexpr int CHF = D * 4 / 16, CHT = RS::ROWB / 16;
    for (int k = tid; k < ne * CHF; k += blockDim.x) {
      const int i = k / CHF, ch = k - i * CHF;
      if (s_cnt[i] <= 0) continue;
      const int ent = s_ent[i];
      unsigned char* slot = sh + (size_t)i * D * 4;
      if (ent >= 0) {
        if (ch < CHT)
          cp_async16(slot + ch * 16, reinterpret_cast<const unsigned char*>(vsum + (row0 + ent) * D) + ch * 16);
      } else {
        cp_async16(slot + ch * 16,
                   reinterpret_cast<const unsigned char*>(A.dv + ((int64_t)u * A.cap + ~ent) * D) + ch * 16);
      }
    }
    cp_async_commit();
    if (tid < G) {
      float v = -INFINITY;
      for (int w = 0; w < NW; ++w) v = fmaxf(v, s_part[w][tid]);
      s_m[tid] = v;
    }
    __syncthreads();
    float l_loc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) l_loc[g] = 0.f;
    for (int i = tid; i < ne; i += blockDim.x) {
      const int cnt = s_cnt[i];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float w = cnt > 0 ? __expf(s_w[i * G + g] - s_m[g]) : 0.f;
        s_w[i * G + g] = w;
        l_loc[g] += (float)cnt * w;
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float v = warp_sum(l_loc[g]);
      if (lane == 0) s_part[warp][g] = v;
    }
    cp_async_wait<0>();
    __syncthreads();
    if (tid < G) {
      float v = 0.f;
      for (int w = 0; w < NW; ++w) v += s_part[w][tid];
      s_l[tid] = v;
    }
    for (int rb = warp * RPW; rb < ne; rb += NW * RPW) {
      const int i = rb + rsub;
      if (i >= ne || s_cnt[i] <= 0) continue;
      const unsigned char* slot = sh + (size_t)i * D * 4;
      float x[EPL];
      if (s_ent[i] >= 0) {
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
      for (int g = 0; g < G; ++g) wv[g] = -s_w[i * G + g];
      axpy_g<G, EPL>(wv, x, acc);
    }
    __syncthreads();  // the staged rows are read before the reduction reuses them
    reduce_and_store<G, EPL, LPR, D>(acc, s_red, warp, sub, rsub, part);
    if (tid < G) { part[tid * PS] = s_m[tid]; part[tid * PS + 1] = -s_l[tid]; }
  } else {
    // -------------------------------------------------------------- attend
    // chunks of 2 TR tokens of the unit's gather list: chunk x, then (when
    // the clusters hold more tokens than the plan expected) x + n_splits,
    // x + 2 n_splits, ...; the first chunk's list entries are read in the
    // same round as the unit record, then the K and V rows of both tiles of
    // a chunk are issued together
    float qv[G][EPL];
    load_q<T, D, G>(q, n_q_heads, b, h, sub, A.scale, qv);
    pdl_wait();
    const int32_t* gat = A.gather + (int64_t)u * A.gather_stride;
    int32_t ge = -1;
    {
      const int t = (int)blockIdx.x * 2 * TR + tid;
      if (tid < 2 * TR && t < A.gather_stride) ge = gat[t];  // valid below n_tok
    }
    if (tid < kInfoInts) s_info[tid] = A.info[(int64_t)u * kInfoInts + tid];
    __syncthreads();
    const int n_tok = (s_info[6] ? 0 : s_info[3]) + s_info[4];
    T* const kt0 = ring;
    T* const vt0 = ring + (size_t)2 * TR * D;
    const T* kbase = reinterpret_cast<const T*>(kp.base);
    const T* vbase = reinterpret_cast<const T*>(vp.base);
    float m_run[G], l_run[G];
#pragma unroll
    for (int g = 0; g < G; ++g) { m_run[g] = -INFINITY; l_run[g] = 0.f; }
    for (int ck = blockIdx.x; ck * 2 * TR < n_tok; ck += A.n_splits) {
      const int t0 = ck * 2 * TR;
      if (ck != (int)blockIdx.x) ge = (tid < 2 * TR && t0 + tid < n_tok) ? gat[t0 + tid] : -1;
      if (tid < 2 * TR) s_row[tid / TR][tid % TR] = (t0 + tid < n_tok && ge >= 0) ? (int64_t)ge * D : -1;
      __syncthreads();
      const int ntile = (min(2 * TR, n_tok - t0) + TR - 1) / TR;
      for (int bi = 0; bi < ntile; ++bi) {
        T* kt = kt0 + (size_t)bi * TR * D;
        T* vt = vt0 + (size_t)bi * TR * D;
        for (int i = tid; i < TR * LPR; i += blockDim.x) {
          const int r = i / LPR, ch = i - r * LPR;
          const int64_t ro = s_row[bi][r];
          if (ro >= 0) {
            cp_async16(kt + r * D + ch * EPL, kbase + ro + ch * EPL);
            cp_async16(vt + r * D + ch * EPL, vbase + ro + ch * EPL);
          }
        }
        cp_async_commit();
      }
      for (int bi = 0; bi < ntile; ++bi) {
        if (bi == 0 && ntile > 1) cp_async_wait<1>(); else cp_async_wait<0>();
        __syncthreads();
        const T* kt = kt0 + (size_t)bi * TR * D;
        const T* vt = vt0 + (size_t)bi * TR * D;
        for (int rb = warp * RPW; rb < TR; rb += NW * RPW) {
          const int r = rb + rsub;
          const int64_t ro = s_row[bi][r];
          float x[EPL];
          if (ro >= 0) {
            const uint4 raw = *reinterpret_cast<const uint4*>(kt + r * D + sub * EPL);
            Elem<T>::unpack(raw, x);
          } else {
#pragma unroll
            for (int e = 0; e < EPL; ++e) x[e] = 0.f;
          }
          float a[G];
          dot_g<G, EPL>(qv, x, a);
          group_reduce_multi<G, LPR>(a, lane);
          if (sub % (LPR / G) == 0) s_sc[r][jh] = ro >= 0 ? a[0] : -INFINITY;
        }
        __syncthreads();
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float mt = -INFINITY;
          for (int r = lane; r < TR; r += 32) mt = fmaxf(mt, s_sc[r][g]);
          mt = warp_max(mt);
          const float mnew = fmaxf(m_run[g], mt);
          const float corr = mnew == -INFINITY ? 1.f : __expf(m_run[g] - mnew);
          float ps = 0.f;
          for (int r = lane; r < TR; r += 32) {
            const float sv = s_sc[r][g];
            ps += sv == -INFINITY ? 0.f : __expf(sv - mnew);
          }
          ps = warp_sum(ps);
          l_run[g] = l_run[g] * corr + ps;
          m_run[g] = mnew;
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[g][e] *= corr;
        }
        for (int rb = warp * RPW; rb < TR; rb += NW * RPW) {
          const int r = rb + rsub;
          if (s_row[bi][r] < 0) continue;
          const uint4 raw = *reinterpret_cast<const uint4*>(vt + r * D + sub * EPL);
          float x[EPL];
          Elem<T>::unpack(raw, x);
          float pw[G];
#pragma unroll
          for (int g = 0; g < G; ++g) pw[g] = __expf(s_sc[r][g] - m_run[g]);
          axpy_g<G, EPL>(pw, x, acc);
        }
      }
      __syncthreads();  // this chunk's tiles and rows are read before the next chunk reuses them
    }
    reduce_and_store<G, EPL, LPR, D>(acc, s_red, warp, sub, rsub, part);
    if (tid == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) { part[g * PS] = m_run[g]; part[g * PS + 1] = l_run[g]; }
    }
  }

  // ---------------------------------------- last CTA of the unit merges
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(A.counters + u, 1) == A.n_splits + A.n_neg - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // parts: [attend splits | corrections | folded estimation parts]; a unit
  // with nothing estimated (dense, or every candidate retrieved) merges the
  // attend parts alone
  const int32_t* I = A.info + (int64_t)u * kInfoInts;
  const int np = (!I[6] && I[0] < I[7] && NC > 0) ? A.n_parts : A.n_splits;
  // one round of loads: every part's (m, l) into shared memory, and this
  // thread's first MB parts of its float4 output chunk into registers
  constexpr int NCH = G * D / 4;                  // float4 chunks of one part's outputs
  constexpr int PP = kStreamThreads / NCH > 0 ? kStreamThreads / NCH : 1;
  constexpr int MB = 16;
  float* f = s_w;                                   // [np][G] rescale factors
  float* lp = reinterpret_cast<float*>(ring);       // [np][G] part denominators
  const float* pbase = A.partials + (int64_t)u * A.n_parts * G * PS;
  const int ch0 = tid % NCH, g0 = (ch0 * 4) / D, e0 = (ch0 * 4) - g0 * D;
  const int pb = tid / NCH;
  float4 v[MB];
#pragma unroll
  for (int k = 0; k < MB; ++k) {
    const int p = pb + k * PP;
    v[k] = (tid < NCH * PP && p < np)
               ? __ldcg(reinterpret_cast<const float4*>(pbase + ((int64_t)p * G + g0) * PS + Part<D>::kO + e0))
               : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int i = tid; i < np * G; i += blockDim.x) {
    f[i] = __ldcg(pbase + (int64_t)i * PS);
    lp[i] = __ldcg(pbase + (int64_t)i * PS + 1);
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
  __syncthreads();
  {
    // thread t sums float4 chunk (t % NCH) over parts p = t / NCH, t / NCH + PP, ...
    float4* red4 = reinterpret_cast<float4*>(lp + ((np * G + 3) & ~3));
    for (int ch = ch0; ch < NCH; ch += kStreamThreads) {
      const int g = (ch * 4) / D, e = (ch * 4) - g * D;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (ch == ch0) {
#pragma unroll
        for (int k = 0; k < MB; ++k) {
          const int p = pb + k * PP;
          const float w = p < np ? f[p * G + g] : 0.f;
          o.x += w * v[k].x; o.y += w * v[k].y; o.z += w * v[k].z; o.w += w * v[k].w;
        }
      }
      for (int p = (ch == ch0 ? pb + MB * PP : pb); p < np; p += PP) {
        const float4 x = __ldcg(reinterpret_cast<const float4*>(pbase + ((int64_t)p * G + g) * PS + Part<D>::kO + e));
        const float w = f[p * G + g];
        o.x += w * x.x; o.y += w * x.y; o.z += w * x.z; o.w += w * x.w;
      }
      if (tid < NCH * PP) red4[tid] = o;
    }
    __syncthreads();
    for (int ch = tid; ch < NCH; ch += blockDim.x) {
      float4 o = red4[ch];
      for (int k = 1; k < PP; ++k) {
        const float4 v = red4[ch + k * NCH];
        o.x += v.x; o.y += v.y; o.z += v.z; o.w += v.w;
      }
      const int g = (ch * 4) / D, e = (ch * 4) - g * D;
      const float l = s_l[g];
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int64_t qh = (int64_t)b * n_q_heads + (int64_t)h * G + g;
      *reinterpret_cast<float4*>(A.out + qh * D + e) =
          make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
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

size_t decode_attend_smem(int dtype, int D, int G, int wcap) {
  (void)dtype; (void)D;
  const size_t ring = 4 * 16384;  // also holds the correction rows and the reductions
  return ring + (size_t)wcap * G * 4 + 2 * (size_t)kNegChunk * 4;
}

size_t decode_topk_smem(int max_nc, int cap, int bt_cap) {
  return ((size_t)(max_nc + 31) / 32 + 4 * (size_t)cap + 2 + (size_t)bt_cap) * sizeof(int32_t);
}

size_t decode_score_smem(int dtype, int D, int sort_pow2, int cap) {
  const int rowb = D * (dtype == WI_BF16 ? 2 : 4);
  const int crows = kScoreChunkBytes / rowb;
  const size_t chunk = 2 * (size_t)kScoreChunkBytes + (size_t)kHistBins / 2 * 4 +
                       (size_t)(crows + 4) * 4 + (size_t)crows * 8 * 4;
  // steady role: sort keys (twice for the rank sort) | affected lists |
  // staged pool rows (offsets + rows, lists of up to kSteadyStage)
  const size_t steady = (size_t)8 * sort_pow2 * (sort_pow2 <= kSteadyRank ? 2 : 1) +
                        (size_t)4 * (2 * cap + 2) + 16 + (size_t)8 * kSteadyStage +
                        (size_t)std::min(cap, kSteadyStage) * rowb;
  return std::max(chunk, steady);
}

cudaError_t launch_decode(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  unsigned char* ws = a.ws;
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + p.off_status);
  float* scores = reinterpret_cast<float*>(ws + p.off_scores);
  uint32_t* keys = reinterpret_cast<uint32_t*>(ws + p.off_keys);
  int32_t* sel = reinterpret_cast<int32_t*>(ws + p.off_sel);
  int32_t* seltok = reinterpret_cast<int32_t*>(ws + p.off_seltok);
  int32_t* info = reinterpret_cast<int32_t*>(ws + p.off_info);
  int32_t* counters = reinterpret_cast<int32_t*>(ws + p.off_counters);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + p.off_hist);
  int32_t* st_slot = reinterpret_cast<int32_t*>(ws + p.off_st_slot);
  int32_t* st_cl = reinterpret_cast<int32_t*>(ws + p.off_st_cl);
  int32_t* aff_cl = reinterpret_cast<int32_t*>(ws + p.off_aff_cl);
  int32_t* aff_start = reinterpret_cast<int32_t*>(ws + p.off_aff_start);
  float* partials = reinterpret_cast<float*>(ws + p.off_partials);
  float* est_parts = reinterpret_cast<float*>(ws + p.off_est);
  int32_t* gather = reinterpret_cast<int32_t*>(ws + p.off_gather);
  float* dv = reinterpret_cast<float*>(ws + p.off_dv);
  int32_t* nonc = reinterpret_cast<int32_t*>(ws + p.off_nonc);
  cudaEvent_t* ev = a.stage_events;
  const bool pdl = ev == nullptr;  // stage timing serialises the launches
  auto mark = [&](int i) { if (ev) cudaEventRecord(ev[i], s); };

  return with_types(p.dtype, p.D, p.G, [&]<typename T, int D, int G>() -> cudaError_t {
    const T* q = reinterpret_cast<const T*>(a.q);
    SteadyArgs sa{a.invperm, a.labels, a.offsets, a.vp, p.n_sink, p.window, p.cap, p.sort_pow2,
                  st_slot, st_cl, aff_cl, aff_start, nonc, info, dv};
    cudaError_t e;
    mark(0);
    const size_t score_smem = decode_score_smem(p.dtype, D, p.sort_pow2, p.cap);
    cudaFuncSetAttribute(wave_score_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)score_smem);
    e = launch_ex(wave_score_kernel<T, D, G>, dim3(p.n_score_blocks + 1, p.U),
                  dim3(kStreamThreads), score_smem, s, false, p.geo, q, p.Hq,
                  reinterpret_cast<const T*>(a.centroids), reinterpret_cast<const T*>(a.value_sums),
                  a.offsets, scores, keys, hist, est_parts, p.scale, p.n_score_blocks, sa, status);
    if (e != cudaSuccess) return e;
    mark(1);
    const size_t topk_smem = decode_topk_smem(p.max_nc, p.cap, p.bt_cap);
    cudaFuncSetAttribute(wave_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)topk_smem);
    FoldArgs fa{est_parts, p.n_score_blocks, partials, p.n_parts, p.n_splits + p.n_neg, G, D};
    TopkArgs ta{keys, a.offsets, hist, nonc, st_slot, aff_cl, aff_start, p.cap, p.topk_clusters,
                p.topk_fraction, sel, seltok, info, a.kp, gather, (int64_t)p.gather_stride, p.bt_cap};
    e = launch_ex(wave_topk_kernel, dim3(1 + p.n_fold, p.U), dim3(kTopkThreads), topk_smem, s,
                  pdl, p.geo, ta, fa, status);
    if (e != cudaSuccess) return e;
    mark(2);
    AttendArgs A{gather, aff_cl, aff_start, sel, dv, (int64_t)p.gather_stride, info, scores,
                 keys, p.cap, p.n_splits, p.n_neg, p.n_parts, p.wcap, partials, counters,
                 a.out, a.lse, p.scale};
    const size_t smem = decode_attend_smem(p.dtype, D, G, p.wcap);
    cudaFuncSetAttribute(wave_attend_estimate_kernel<T, D, G>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    e = launch_ex(wave_attend_estimate_kernel<T, D, G>, dim3(p.n_splits + p.n_neg, p.U),
                  dim3(kStreamThreads), smem, s, pdl, p.geo, q, p.Hq, a.kp, a.vp,
                  reinterpret_cast<const T*>(a.value_sums), a.offsets, A, status);
    if (e != cudaSuccess) return e;
    mark(3);
    return cudaGetLastError();
  });
}

}  // namespace wi

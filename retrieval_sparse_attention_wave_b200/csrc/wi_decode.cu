// Decode-step kernels of the wave index (sm_100a).
//
// One decode step is the query-dependent phase of the method
// (RetroInfer technical summary, section 2.A, items 1-3; Vortex summary,
// section 2.A forward_indexer):
//   steady    resolve the steady zone (sinks + recent window) to slots and
//             clusters (query-independent; item 1 Steady Zone)
//   score     q . centroid / sqrt(d) for every cluster, per q head, and the
//             group-max selection key (item 2, the index lookup)
//   topk      exact radix select of the k best candidate clusters per KV head
//             (item 2; Vortex 2.C Top-K), ties to the lower cluster id
//   attend    gather the retrieved clusters' rows plus the steady rows from the
//             cluster-permuted paged layout and run split-K exact attention
//             (items 1 and 2)
//   estimate  every other candidate cluster as cnt' * e^s with value sum
//             Vsum' (item 3 Estimation Zone)
//   merge     log-sum-exp combine of all partial softmax parts
// All streaming kernels read 16-byte vectors with the row of one cluster or
// token spread over LPR = d*sizeof(T)/16 lanes; the score / estimate GEMVs
// have M = G <= 8 rows, so they run on the CUDA cores (FFMA), not tensor cores.
#include <cfloat>
#include <climits>
#include <cmath>

#include "wi_common.cuh"
#include "wi_plan.h"

namespace wi {

const char* const kDecodeStageNames[kDecodeStages] = {"steady", "score", "topk",
                                                      "attend", "estimate", "merge"};

namespace {

template <typename T, int D>
struct RowShape {
  static constexpr int EPL = Elem<T>::kPerVec;  // elements per lane (one 16-B vector)
  static constexpr int LPR = D / EPL;           // lanes per row
  static constexpr int RPW = 32 / LPR;          // rows per warp step
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

// ------------------------------------------------------------------ steady
// One CTA per unit.  Maps the steady positions to slots (invperm), sorts the
// slots (bitonic, shared memory), finds each slot's cluster (binary search in
// offsets) and run-length encodes the clusters ("affected" clusters with
// their steady-member ranges).
__global__ void __launch_bounds__(kStreamThreads)
wave_steady_kernel(const Geo geo, const int32_t* __restrict__ invperm,
                   const int32_t* __restrict__ offsets, int n_sink, int window, int cap,
                   int sort_pow2, int32_t* __restrict__ st_slot, int32_t* __restrict__ st_cl,
                   int32_t* __restrict__ aff_cl, int32_t* __restrict__ aff_start,
                   int32_t* __restrict__ info, uint32_t* status) {
  extern __shared__ int32_t sh_sort[];
  const int u = blockIdx.x, b = u / geo.hkv, h = u - b * geo.hkv;
  const int T = geo.T(b), NC = geo.NC(b);
  const int ns = min(n_sink, T);
  const int wstart = max(T - window, ns);
  const int n_st = ns + (T - wstart);
  int32_t* I = info + (int64_t)u * kInfoInts;
  if (n_st >= T) {  // all steady: attended densely, nothing retrieved or estimated
    if (threadIdx.x == 0) { I[4] = T; I[5] = 0; I[6] = 1; }
    return;
  }
  int npow = 1;
  while (npow < n_st) npow <<= 1;
  if (npow > sort_pow2) npow = sort_pow2;  // host guarantees n_st <= cap <= sort_pow2
  const int32_t* inv = invperm + geo.tok_row(b, h);
  for (int i = threadIdx.x; i < npow; i += blockDim.x) {
    int32_t s = INT_MAX;
    if (i < n_st) {
      const int pos = i < ns ? i : wstart + (i - ns);
      s = inv[pos];
      if (s < 0 || s >= T) { flag_error(status, WI_DEV_BAD_SLOT); s = INT_MAX; }
    }
    sh_sort[i] = s;
  }
  __syncthreads();
  for (int k = 2; k <= npow; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < npow; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const bool up = (i & k) == 0;
          const int32_t a = sh_sort[i], c = sh_sort[ixj];
          if ((a > c) == up) { sh_sort[i] = c; sh_sort[ixj] = a; }
        }
      }
      __syncthreads();
    }
  }
  const int32_t* off = offsets + geo.off_row(b, h);
  int32_t* slots = st_slot + (int64_t)u * cap;
  int32_t* cls = st_cl + (int64_t)u * cap;
  for (int i = threadIdx.x; i < n_st; i += blockDim.x) {
    const int32_t s = sh_sort[i];
    // largest c with off[c] <= s
    int lo = 0, hi = NC;  // answer in [0, NC)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (off[mid] <= s) lo = mid; else hi = mid - 1;
    }
    if (s != INT_MAX && (off[lo] > s || off[lo + 1] <= s)) flag_error(status, WI_DEV_BAD_CLUSTER);
    slots[i] = s;
    cls[i] = lo;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int32_t* acl = aff_cl + (int64_t)u * cap;
    int32_t* ast = aff_start + (int64_t)u * (cap + 1);
    int n_aff = 0;
    for (int base = 0; base < n_st; base += 32) {
      const int i = base + lane;
      const int c = i < n_st ? cls[i] : -1;
      const bool head = i < n_st && (i == 0 || cls[i - 1] != c);
      const unsigned bal = __ballot_sync(0xffffffffu, head);
      if (head) {
        const int r = __popc(bal & ((1u << lane) - 1u));
        acl[n_aff + r] = c;
        ast[n_aff + r] = i;
      }
      n_aff += __popc(bal);
    }
    if (lane == 0) {
      ast[n_aff] = n_st;
      I[4] = n_st; I[5] = n_aff; I[6] = 0;
    }
  }
}

// ------------------------------------------------------------------- score
template <typename T, int D, int G>
__global__ void __launch_bounds__(kStreamThreads)
wave_score_kernel(const Geo geo, const T* __restrict__ q, int n_q_heads, const T* __restrict__ cent,
                  const int32_t* __restrict__ offsets, float* __restrict__ scores,
                  uint32_t* __restrict__ keys, float scale, int chunk) {
  using RS = RowShape<T, D>;
  constexpr int EPL = RS::EPL, LPR = RS::LPR, RPW = RS::RPW, UNR = 4;
  constexpr int NW = kStreamThreads / 32;
  static_assert(G <= LPR, "group larger than lanes per row");
  const int u = blockIdx.y, b = u / geo.hkv, h = u - b * geo.hkv;
  const int NC = geo.NC(b);
  const int c0 = blockIdx.x * chunk;
  if (c0 >= NC) return;
  const int c1 = min(NC, c0 + chunk);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % LPR, rsub = lane / LPR;
  float qv[G][EPL];
  load_q<T, D, G>(q, n_q_heads, b, h, sub, scale, qv);
  const int64_t row0 = geo.cl_row(b, h);
  const T* cb = cent + row0 * D + sub * EPL;
  const int32_t* off = offsets + geo.off_row(b, h);
  const int j = sub / (LPR / G);
  for (int base = c0 + warp * RPW * UNR; base < c1; base += NW * RPW * UNR) {
    uint4 raw[UNR];
#pragma unroll
    for (int i = 0; i < UNR; ++i) {
      const int c = base + i * RPW + rsub;
      raw[i] = c < c1 ? ld_stream(cb + (int64_t)c * D) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < UNR; ++i) {
      const int c = base + i * RPW + rsub;
      float x[EPL];
      Elem<T>::unpack(raw[i], x);
      float acc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        acc[g] = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[g] = fmaf(qv[g][e], x[e], acc[g]);
      }
      group_reduce_multi<G, LPR>(acc, lane);
      float m = acc[0];
#pragma unroll
      for (int o = LPR / 2; o >= LPR / G; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (c < c1) {
        if (sub % (LPR / G) == 0) scores[(row0 + c) * G + j] = acc[0];
        if (sub == 0) {
          const int cnt = off[c + 1] - off[c];
          keys[row0 + c] = cnt > 0 ? ordered_key(m) : 0u;
        }
      }
    }
  }
}

// -------------------------------------------------------------------- topk
// One CTA per unit: drop clusters with no non-steady member, then an exact
// 4-pass MSB radix select (8-bit digits) of the k-th largest key, then an
// ordered compaction of the selected ids and a prefix sum of their sizes.
__global__ void __launch_bounds__(kTopkThreads)
wave_topk_kernel(const Geo geo, uint32_t* __restrict__ keys, const int32_t* __restrict__ offsets,
                 const int32_t* __restrict__ aff_cl, const int32_t* __restrict__ aff_start, int cap,
                 int topk_clusters, double topk_fraction, int32_t* __restrict__ sel,
                 int32_t* __restrict__ sel_tok, int32_t* __restrict__ info) {
  __shared__ int hist[256];
  __shared__ int scan_sh[32];
  __shared__ int bcast[4];
  const int u = blockIdx.x, b = u / geo.hkv, h = u - b * geo.hkv;
  const int NC = geo.NC(b);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* I = info + (int64_t)u * kInfoInts;
  const int64_t row0 = geo.cl_row(b, h);
  int32_t* pre = sel_tok + row0 + u;
  const int k_req = topk_clusters >= 0 ? topk_clusters
                                       : (int)ceil(topk_fraction * (double)NC);
  if (I[6]) {  // dense unit
    if (tid == 0) {
      I[0] = 0; I[1] = (int32_t)0xFFFFFFFFu; I[2] = -1; I[3] = 0; I[7] = k_req;
      pre[0] = 0;
    }
    return;
  }
  uint32_t* kk = keys + row0;
  const int32_t* off = offsets + geo.off_row(b, h);
  const int n_aff = I[5];
  for (int jj = tid; jj < n_aff; jj += blockDim.x) {
    const int c = aff_cl[(int64_t)u * cap + jj];
    const int dc = aff_start[(int64_t)u * (cap + 1) + jj + 1] - aff_start[(int64_t)u * (cap + 1) + jj];
    if (c >= 0 && c < NC && off[c + 1] - off[c] - dc <= 0) kk[c] = 0u;
  }
  __syncthreads();

  uint32_t prefix = 0, pmask = 0;
  int krem = 0, ncand = 0, ksel = 0;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    int mine = 0;
    for (int c = tid; c < NC; c += blockDim.x) {
      const uint32_t key = kk[c];
      if (key == 0u) continue;
      ++mine;
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    if (pass == 0) {
      int tot;
      block_inclusive_scan(mine, scan_sh, &tot);
      ncand = tot;
      ksel = min(max(k_req, 0), ncand);
      krem = ksel;
      if (ksel == 0 || ksel == ncand) break;
    } else {
      __syncthreads();
    }
    if (warp == 0) {
      int cnt[8], sum = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) { cnt[t] = hist[255 - 8 * lane - t]; sum += cnt[t]; }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, incl >= krem);
      const int first = __ffs(bal) - 1;
      if (lane == first) {
        int acc = incl - sum;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (acc + cnt[t] >= krem) { bcast[0] = 255 - 8 * lane - t; bcast[1] = acc; break; }
          acc += cnt[t];
        }
      }
    }
    __syncthreads();
    krem -= bcast[1];
    prefix |= (uint32_t)bcast[0] << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }

  uint32_t kstar;
  int thr;
  if (ksel == 0) {
    kstar = 0xFFFFFFFFu; thr = -1;
  } else if (ksel == ncand) {
    kstar = 1u; thr = NC;
  } else {
    kstar = prefix;
    // index of the krem-th key equal to kstar, in ascending cluster id
    int running = 0;
    if (tid == 0) bcast[2] = -1;
    __syncthreads();
    for (int base = 0; base < NC; base += blockDim.x) {
      const int c = base + tid;
      const int f = (c < NC && kk[c] == kstar) ? 1 : 0;
      int tot;
      const int incl = block_inclusive_scan(f, scan_sh, &tot);
      if (f && running + incl == krem) bcast[2] = c;
      running += tot;
      __syncthreads();
      if (bcast[2] >= 0) break;
    }
    thr = bcast[2];
  }
  // ordered compaction of the selection
  int running = 0;
  for (int base = 0; base < NC; base += blockDim.x) {
    const int c = base + tid;
    int f = 0;
    if (c < NC) {
      const uint32_t key = kk[c];
      f = key != 0u && (key > kstar || (key == kstar && c <= thr));
    }
    int tot;
    const int incl = block_inclusive_scan(f, scan_sh, &tot);
    if (f) sel[row0 + running + incl - 1] = c;
    running += tot;
  }
  __syncthreads();
  // token prefix over the selected clusters (all slots, steady ones included)
  int tok = 0;
  for (int base = 0; base < ksel; base += blockDim.x) {
    const int i = base + tid;
    int cnt = 0;
    if (i < ksel) {
      const int c = sel[row0 + i];
      cnt = (c >= 0 && c < NC) ? off[c + 1] - off[c] : 0;
    }
    int tot;
    const int incl = block_inclusive_scan(cnt, scan_sh, &tot);
    if (i < ksel) pre[i + 1] = tok + incl;
    tok += tot;
  }
  if (tid == 0) {
    pre[0] = 0;
    I[0] = ksel; I[1] = (int32_t)kstar; I[2] = thr; I[3] = tok; I[7] = k_req;
  }
}

// ------------------------------------------------------------------ attend
// Split-K exact attention over the retrieved clusters' non-steady rows
// followed by the steady rows.  CTA (split, unit) takes an equal share of
// the unit's token list; the list is resolved tile by tile through the
// prefix sums of the selected cluster sizes.
template <typename T, int D, int G>
__global__ void __launch_bounds__(kStreamThreads)
wave_attend_kernel(const Geo geo, const T* __restrict__ q, int n_q_heads, const Pool kp,
                   const Pool vp, const int32_t* __restrict__ perm,
                   const int32_t* __restrict__ offsets, const int32_t* __restrict__ sel,
                   const int32_t* __restrict__ sel_tok, const int32_t* __restrict__ st_slot,
                   const int32_t* __restrict__ info, int n_sink, int window, int cap,
                   int n_splits, int n_parts, float* __restrict__ partials, float scale,
                   uint32_t* status) {
  using RS = RowShape<T, D>;
  constexpr int EPL = RS::EPL, LPR = RS::LPR, RPW = RS::RPW;
  constexpr int NW = kStreamThreads / 32;
  constexpr int TILE = kAttendTile;
  static_assert(TILE % (NW * RPW) == 0, "tile must be a multiple of rows per CTA step");
  __shared__ int64_t s_row[TILE];
  __shared__ float s_sc[TILE][G];
  __shared__ int s_pre[TILE + 2];
  __shared__ int s_coff[TILE + 1];
  __shared__ int s_cursor;
  __shared__ float s_red[NW][G][D];

  const int u = blockIdx.y, b = u / geo.hkv, h = u - b * geo.hkv;
  const int Tb = geo.T(b), NC = geo.NC(b);
  const int ns = min(n_sink, Tb);
  const int wstart = max(Tb - window, ns);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tid = threadIdx.x;
  const int sub = lane % LPR, rsub = lane / LPR;
  const int32_t* I = info + (int64_t)u * kInfoInts;
  const int dense = I[6];
  const int ksel = dense ? 0 : I[0];
  const int nsel_tok = dense ? 0 : I[3];
  const int n_st = I[4];
  const int n_tok = nsel_tok + n_st;
  const int per = (n_tok + n_splits - 1) / n_splits;
  const int t0 = blockIdx.x * per;
  const int t1 = min(n_tok, t0 + per);

  float qv[G][EPL];
  load_q<T, D, G>(q, n_q_heads, b, h, sub, scale, qv);
  const int64_t row0 = geo.cl_row(b, h);
  const int32_t* pre = sel_tok + row0 + u;
  const int32_t* selu = sel + row0;
  const int32_t* off = offsets + geo.off_row(b, h);
  const int32_t* permu = perm + geo.tok_row(b, h);
  const T* kbase = reinterpret_cast<const T*>(kp.base) + sub * EPL;
  const T* vbase = reinterpret_cast<const T*>(vp.base) + sub * EPL;
  const int jh = sub / (LPR / G);

  float m_run[G], l_run[G], acc[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -INFINITY; l_run[g] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
  }

  if (tid == 0) {
    int cur = ksel;
    if (t0 < nsel_tok) {  // largest i < ksel with pre[i] <= t0
      int lo = 0, hi = ksel - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= t0) lo = mid; else hi = mid - 1;
      }
      cur = lo;
    }
    s_cursor = cur;
  }
  __syncthreads();

  for (int tb = t0; tb < t1; tb += TILE) {
    const int n = min(TILE, t1 - tb);
    const int cur = s_cursor;
    if (tb < nsel_tok) {
      for (int i = tid; i < TILE + 2; i += blockDim.x) {
        const int idx = cur + i;
        s_pre[i] = idx <= ksel ? pre[idx] : INT_MAX;
      }
      for (int i = tid; i < TILE + 1; i += blockDim.x) {
        const int idx = cur + i;
        int o = 0;
        if (idx < ksel) {
          const int c = selu[idx];
          if (c >= 0 && c < NC) o = off[c]; else flag_error(status, WI_DEV_BAD_CLUSTER);
        }
        s_coff[i] = o;
      }
    }
    __syncthreads();
    if (tid < TILE) {
      int64_t rowoff = -1;
      if (tid < n) {
        const int tok = tb + tid;
        int slot;
        bool valid = true;
        if (tok < nsel_tok) {
          int lo = 0, hi = TILE;  // largest i with s_pre[i] <= tok
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_pre[mid] <= tok) lo = mid; else hi = mid - 1;
          }
          slot = s_coff[lo] + (tok - s_pre[lo]);
          if (slot < 0 || slot >= Tb) {
            flag_error(status, WI_DEV_BAD_SLOT);
            valid = false;
          } else {
            const int pos = permu[slot];
            valid = !(pos < ns || pos >= wstart);
          }
          if (tid == n - 1) s_cursor = cur + lo;
        } else {
          const int js = tok - nsel_tok;
          slot = dense ? js : st_slot[(int64_t)u * cap + js];
        }
        if (valid) rowoff = pool_row(kp, geo.hkv, D, b, h, slot, status);
      }
      s_row[tid] = rowoff;
    }
    __syncthreads();
    // scores of the tile
#pragma unroll
    for (int rb = warp * RPW; rb < TILE; rb += NW * RPW) {
      const int r = rb + rsub;
      const int64_t ro = s_row[r];
      const uint4 raw = ro >= 0 ? ld_stream(kbase + ro) : make_uint4(0, 0, 0, 0);
      float x[EPL];
      Elem<T>::unpack(raw, x);
      float a[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        a[g] = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) a[g] = fmaf(qv[g][e], x[e], a[g]);
      }
      group_reduce_multi<G, LPR>(a, lane);
      if (sub % (LPR / G) == 0) s_sc[r][jh] = ro >= 0 ? a[0] : -INFINITY;
    }
    __syncthreads();
    // running max / sum update (identical in every warp)
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mt = -INFINITY;
      for (int r = lane; r < TILE; r += 32) mt = fmaxf(mt, s_sc[r][g]);
      mt = warp_max(mt);
      const float mnew = fmaxf(m_run[g], mt);
      const float corr = mnew == -INFINITY ? 1.f : __expf(m_run[g] - mnew);
      float ps = 0.f;
      for (int r = lane; r < TILE; r += 32) {
        const float sv = s_sc[r][g];
        ps += sv == -INFINITY ? 0.f : __expf(sv - mnew);
      }
      ps = warp_sum(ps);
      l_run[g] = l_run[g] * corr + ps;
      m_run[g] = mnew;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[g][e] *= corr;
    }
    // weighted value sum
#pragma unroll
    for (int rb = warp * RPW; rb < TILE; rb += NW * RPW) {
      const int r = rb + rsub;
      const int64_t ro = s_row[r];
      const uint4 raw = ro >= 0 ? ld_stream(vbase + ro) : make_uint4(0, 0, 0, 0);
      float x[EPL];
      Elem<T>::unpack(raw, x);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float sv = s_sc[r][g];
        const float p = sv == -INFINITY ? 0.f : __expf(sv - m_run[g]);
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[g][e] = fmaf(p, x[e], acc[g][e]);
      }
    }
    __syncthreads();
  }
  // reduce the value accumulators over row groups and warps
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
      for (int e = 0; e < EPL; ++e) s_red[warp][g][sub * EPL + e] = acc[g][e];
  }
  __syncthreads();
  float* part = partials + ((int64_t)u * n_parts + blockIdx.x) * G * (D + 2);
  for (int i = tid; i < G * D; i += blockDim.x) {
    const int g = i / D, e = i - g * D;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += s_red[w][g][e];
    part[g * (D + 2) + 2 + e] = v;
  }
  if (tid == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) { part[g * (D + 2)] = m_run[g]; part[g * (D + 2) + 1] = l_run[g]; }
  }
}

// ---------------------------------------------------------------- estimate
// CTA (chunk, unit) estimates the candidate clusters of its chunk that were
// not retrieved: weights w = e^(s - m) from the stored scores, denominator
// sum cnt' * w, numerator sum w * Vsum, then minus w * v for each steady
// member of an affected cluster (Vsum' = Vsum - sum of steady values).
template <typename T, int D, int G>
__global__ void __launch_bounds__(kStreamThreads)
wave_estimate_kernel(const Geo geo, const T* __restrict__ vsum, const int32_t* __restrict__ offsets,
                     const float* __restrict__ scores, const uint32_t* __restrict__ keys,
                     const int32_t* __restrict__ info, const int32_t* __restrict__ aff_cl,
                     const int32_t* __restrict__ aff_start, const int32_t* __restrict__ st_slot,
                     const int32_t* __restrict__ st_cl, const Pool vp, int cap, int echunk,
                     int n_splits, int n_parts, float* __restrict__ partials, uint32_t* status) {
  using RS = RowShape<T, D>;
  constexpr int EPL = RS::EPL, LPR = RS::LPR, RPW = RS::RPW, UNR = 4;
  constexpr int NW = kStreamThreads / 32;
  extern __shared__ float sh_est[];
  float* s_w = sh_est;                                   // [echunk][G]
  int* s_cnt = reinterpret_cast<int*>(sh_est + echunk * G);  // [echunk]
  __shared__ float s_red[NW][G][D];
  __shared__ float s_part[NW][G];
  __shared__ float s_m[G], s_l[G];
  __shared__ int s_arange[2];

  const int u = blockIdx.y, b = u / geo.hkv, h = u - b * geo.hkv;
  const int NC = geo.NC(b);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tid = threadIdx.x;
  const int sub = lane % LPR, rsub = lane / LPR;
  const int32_t* I = info + (int64_t)u * kInfoInts;
  const int c0 = blockIdx.x * echunk;
  const int c1 = min(NC, c0 + echunk);
  float* part = partials + ((int64_t)u * n_parts + n_splits + blockIdx.x) * G * (D + 2);
  if (I[6] || c0 >= NC) {
    for (int i = tid; i < G * (D + 2); i += blockDim.x) {
      const int e = i % (D + 2);
      part[i] = e == 0 ? -INFINITY : 0.f;
    }
    return;
  }
  const uint32_t kstar = (uint32_t)I[1];
  const int thr = I[2];
  const int n_aff = I[5];
  const int64_t row0 = geo.cl_row(b, h);
  const int32_t* off = offsets + geo.off_row(b, h);
  const int32_t* acl = aff_cl + (int64_t)u * cap;
  const int32_t* ast = aff_start + (int64_t)u * (cap + 1);
  if (tid < 2) {  // affected clusters inside [c0, c1): lower_bound of c0 and c1
    const int key = tid == 0 ? c0 : c1;
    int lo = 0, hi = n_aff;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (acl[mid] < key) lo = mid + 1; else hi = mid;
    }
    s_arange[tid] = lo;
  }
  __syncthreads();
  const int a0 = s_arange[0], a1 = s_arange[1];

  // phase 1: contribution mask, reduced counts, scores
  float mloc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) mloc[g] = -INFINITY;
  for (int i = tid; i < c1 - c0; i += blockDim.x) {
    const int c = c0 + i;
    const uint32_t key = keys[row0 + c];
    const bool picked = key > kstar || (key == kstar && c <= thr);
    int cntp = off[c + 1] - off[c];
    bool contrib = key != 0u && !picked;
    if (contrib && a1 > a0) {
      int lo = a0, hi = a1;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (acl[mid] < c) lo = mid + 1; else hi = mid;
      }
      if (lo < a1 && acl[lo] == c) cntp -= ast[lo + 1] - ast[lo];
    }
    contrib = contrib && cntp > 0;
    s_cnt[i] = contrib ? cntp : 0;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float sv = contrib ? scores[(row0 + c) * G + g] : -INFINITY;
      s_w[i * G + g] = sv;
      mloc[g] = fmaxf(mloc[g], sv);
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float v = warp_max(mloc[g]);
    if (lane == 0) s_part[warp][g] = v;
  }
  __syncthreads();
  if (tid < G) {
    float v = -INFINITY;
    for (int w = 0; w < NW; ++w) v = fmaxf(v, s_part[w][tid]);
    s_m[tid] = v;
  }
  __syncthreads();
  // phase 2: weights and denominator
  float lloc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) lloc[g] = 0.f;
  for (int i = tid; i < c1 - c0; i += blockDim.x) {
    const int cnt = s_cnt[i];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float w = cnt > 0 ? __expf(s_w[i * G + g] - s_m[g]) : 0.f;
      s_w[i * G + g] = w;
      lloc[g] += (float)cnt * w;
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float v = warp_sum(lloc[g]);
    if (lane == 0) s_part[warp][g] = v;
  }
  __syncthreads();
  if (tid < G) {
    float v = 0.f;
    for (int w = 0; w < NW; ++w) v += s_part[w][tid];
    s_l[tid] = v;
  }
  // phase 3: numerator over the value sums
  float acc[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
  const T* vb = vsum + row0 * D + sub * EPL;
  for (int base = c0 + warp * RPW * UNR; base < c1; base += NW * RPW * UNR) {
    uint4 raw[UNR];
#pragma unroll
    for (int i = 0; i < UNR; ++i) {
      const int c = base + i * RPW + rsub;
      raw[i] = (c < c1 && s_cnt[c - c0] > 0) ? ld_stream(vb + (int64_t)c * D)
                                             : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < UNR; ++i) {
      const int c = base + i * RPW + rsub;
      if (c < c1 && s_cnt[c - c0] > 0) {
        float x[EPL];
        Elem<T>::unpack(raw[i], x);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float w = s_w[(c - c0) * G + g];
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[g][e] = fmaf(w, x[e], acc[g][e]);
        }
      }
    }
  }
  // phase 4: remove the steady members of estimated clusters
  if (a1 > a0) {
    const int s_begin = ast[a0], s_end = ast[a1];
    const int32_t* slots = st_slot + (int64_t)u * cap;
    const int32_t* cls = st_cl + (int64_t)u * cap;
    const T* vpb = reinterpret_cast<const T*>(vp.base) + sub * EPL;
    for (int base = s_begin + warp * RPW; base < s_end; base += NW * RPW) {
      const int i = base + rsub;
      bool ok = false;
      int64_t ro = -1;
      int ci = 0;
      if (i < s_end) {
        ci = cls[i] - c0;
        ok = ci >= 0 && ci < c1 - c0 && s_cnt[ci] > 0;
        if (ok) {
          ro = pool_row(vp, geo.hkv, D, b, h, slots[i], status);
          ok = ro >= 0;
        }
      }
      if (ok) {
        const uint4 raw = ld_stream(vpb + ro);
        float x[EPL];
        Elem<T>::unpack(raw, x);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float w = s_w[ci * G + g];
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[g][e] = fmaf(-w, x[e], acc[g][e]);
        }
      }
    }
  }
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
      for (int e = 0; e < EPL; ++e) s_red[warp][g][sub * EPL + e] = acc[g][e];
  }
  __syncthreads();
  for (int i = tid; i < G * D; i += blockDim.x) {
    const int g = i / D, e = i - g * D;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += s_red[w][g][e];
    part[g * (D + 2) + 2 + e] = v;
  }
  if (tid < G) {
    part[tid * (D + 2)] = s_m[tid];
    part[tid * (D + 2) + 1] = s_l[tid];
  }
}

// ------------------------------------------------------------------- merge
// One CTA per (unit, q head): log-sum-exp combine of all parts.
template <int D, int G>
__global__ void __launch_bounds__(128)
wave_merge_kernel(const Geo geo, const float* __restrict__ partials, int n_parts, int n_q_heads,
                  float* __restrict__ out, float* __restrict__ lse) {
  const int u = blockIdx.x / G, g = blockIdx.x % G;
  const int b = u / geo.hkv, h = u - b * geo.hkv;
  const float* base = partials + ((int64_t)u * n_parts * G + g) * (D + 2);
  const int64_t stride = (int64_t)G * (D + 2);
  float M = -INFINITY;
  for (int p = 0; p < n_parts; ++p) M = fmaxf(M, base[p * stride]);
  float l = 0.f;
  float o[(D + 127) / 128];
#pragma unroll
  for (int i = 0; i < (D + 127) / 128; ++i) o[i] = 0.f;
  for (int p = 0; p < n_parts; ++p) {
    const float mp = base[p * stride];
    const float f = mp == -INFINITY ? 0.f : expf(mp - M);
    l += f * base[p * stride + 1];
#pragma unroll
    for (int i = 0; i < (D + 127) / 128; ++i) {
      const int e = threadIdx.x + 128 * i;
      if (e < D) o[i] += f * base[p * stride + 2 + e];
    }
  }
  const int64_t qh = (int64_t)b * n_q_heads + (int64_t)h * G + g;
#pragma unroll
  for (int i = 0; i < (D + 127) / 128; ++i) {
    const int e = threadIdx.x + 128 * i;
    if (e < D) out[qh * D + e] = l > 0.f ? o[i] / l : 0.f;
  }
  if (lse != nullptr && threadIdx.x == 0) lse[qh] = l > 0.f ? M + logf(l) : -INFINITY;
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

}  // namespace

cudaError_t launch_decode(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  unsigned char* ws = a.ws;
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + p.off_status);
  float* scores = reinterpret_cast<float*>(ws + p.off_scores);
  uint32_t* keys = reinterpret_cast<uint32_t*>(ws + p.off_keys);
  int32_t* sel = reinterpret_cast<int32_t*>(ws + p.off_sel);
  int32_t* seltok = reinterpret_cast<int32_t*>(ws + p.off_seltok);
  int32_t* info = reinterpret_cast<int32_t*>(ws + p.off_info);
  int32_t* st_slot = reinterpret_cast<int32_t*>(ws + p.off_st_slot);
  int32_t* st_cl = reinterpret_cast<int32_t*>(ws + p.off_st_cl);
  int32_t* aff_cl = reinterpret_cast<int32_t*>(ws + p.off_aff_cl);
  int32_t* aff_start = reinterpret_cast<int32_t*>(ws + p.off_aff_start);
  float* partials = reinterpret_cast<float*>(ws + p.off_partials);
  cudaEvent_t* ev = a.stage_events;
  auto mark = [&](int i) { if (ev) cudaEventRecord(ev[i], s); };

  return with_types(p.dtype, p.D, p.G, [&]<typename T, int D, int G>() -> cudaError_t {
    const T* q = reinterpret_cast<const T*>(a.q);
    mark(0);
    wave_steady_kernel<<<p.U, kStreamThreads, p.sort_pow2 * sizeof(int32_t), s>>>(
        p.geo, a.invperm, a.offsets, p.n_sink, p.window, p.cap, p.sort_pow2, st_slot, st_cl,
        aff_cl, aff_start, info, status);
    mark(1);
    wave_score_kernel<T, D, G><<<dim3(p.n_score_blocks, p.U), kStreamThreads, 0, s>>>(
        p.geo, q, p.Hq, reinterpret_cast<const T*>(a.centroids), a.offsets, scores, keys,
        p.scale, p.score_chunk);
    mark(2);
    wave_topk_kernel<<<p.U, kTopkThreads, 0, s>>>(p.geo, keys, a.offsets, aff_cl, aff_start,
                                                  p.cap, p.topk_clusters, p.topk_fraction, sel,
                                                  seltok, info);
    mark(3);
    wave_attend_kernel<T, D, G><<<dim3(p.n_splits, p.U), kStreamThreads, 0, s>>>(
        p.geo, q, p.Hq, a.kp, a.vp, a.perm, a.offsets, sel, seltok, st_slot, info, p.n_sink,
        p.window, p.cap, p.n_splits, p.n_parts, partials, p.scale, status);
    mark(4);
    const size_t est_smem = (size_t)p.echunk * (G + 1) * sizeof(float);
    cudaFuncSetAttribute(wave_estimate_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)est_smem);
    wave_estimate_kernel<T, D, G><<<dim3(p.n_est, p.U), kStreamThreads, est_smem, s>>>(
        p.geo, reinterpret_cast<const T*>(a.value_sums), a.offsets, scores, keys, info, aff_cl,
        aff_start, st_slot, st_cl, a.vp, p.cap, p.echunk, p.n_splits, p.n_parts, partials,
        status);
    mark(5);
    wave_merge_kernel<D, G><<<p.U * G, 128, 0, s>>>(p.geo, partials, p.n_parts, p.Hq, a.out,
                                                    a.lse);
    mark(6);
    return cudaGetLastError();
  });
}

}  // namespace wi

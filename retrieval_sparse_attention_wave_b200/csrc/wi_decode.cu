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

const char* const kDecodeStageNames[kDecodeStages] = {"score", "topk", "attend_estimate"};

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
  Pool vp;
  int n_sink, window, cap, sort_pow2;
  int32_t *st_slot, *st_cl, *aff_cl, *aff_start, *info;
  float* dv;  // [U][cap][D] fp32: sum of the steady members' values per affected cluster
};

// Steady zone of unit u: positions -> (slot, cluster) through invperm and
// labels (one round of independent loads), sorted by slot (which also
// groups them by cluster, clusters being slot ranges), then run-length
// encoded into (affected cluster, first steady index), and the value rows
// of each affected cluster's steady members summed in slot order (dV).
template <typename T, int D>
__device__ void steady_role(const Geo& geo, int u, const SteadyArgs& a, uint32_t* status,
                            unsigned long long* sh_sort) {
  const int b = u / geo.hkv, h = u - b * geo.hkv;
  const int Tb = geo.T(b), NC = geo.NC(b);
  const int ns = min(a.n_sink, Tb);
  const int wstart = max(Tb - a.window, ns);
  const int n_st = ns + (Tb - wstart);
  int32_t* I = a.info + (int64_t)u * kInfoInts;
  if (n_st >= Tb) {  // all steady: attended densely, nothing retrieved or estimated
    if (threadIdx.x == 0) { I[4] = Tb; I[5] = 0; I[6] = 1; }
    return;
  }
  int npow = 1;
  while (npow < n_st) npow <<= 1;
  npow = min(npow, a.sort_pow2);
  const int32_t* inv = a.invperm + geo.tok_row(b, h);
  const int32_t* lab = a.labels + geo.tok_row(b, h);
  for (int i = threadIdx.x; i < npow; i += blockDim.x) {
    unsigned long long kv = ~0ull;
    if (i < n_st) {
      const int pos = i < ns ? i : wstart + (i - ns);
      int s = __ldg(inv + pos), c = __ldg(lab + pos);
      if (s < 0 || s >= Tb) { flag_error(status, WI_DEV_BAD_SLOT); s = 0x7fffffff; }
      if (c < 0 || c >= NC) { flag_error(status, WI_DEV_BAD_CLUSTER); c = 0; }
      kv = ((unsigned long long)(uint32_t)s << 32) | (uint32_t)c;
    }
    sh_sort[i] = kv;
  }
  __syncthreads();
  for (int k = 2; k <= npow; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < npow; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const bool up = (i & k) == 0;
          const unsigned long long x = sh_sort[i], y = sh_sort[ixj];
          if ((x > y) == up) { sh_sort[i] = y; sh_sort[ixj] = x; }
        }
      }
      __syncthreads();
    }
  }
  int32_t* slots = a.st_slot + (int64_t)u * a.cap;
  int32_t* cls = a.st_cl + (int64_t)u * a.cap;
  for (int i = threadIdx.x; i < n_st; i += blockDim.x) {
    slots[i] = (int32_t)(sh_sort[i] >> 32);
    cls[i] = (int32_t)(sh_sort[i] & 0xffffffffu);
  }
  __shared__ int s_naff;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int32_t* acl = a.aff_cl + (int64_t)u * a.cap;
    int32_t* ast = a.aff_start + (int64_t)u * (a.cap + 1);
    int n_aff = 0;
    for (int base = 0; base < n_st; base += 32) {
      const int i = base + lane;
      const int c = i < n_st ? (int)(sh_sort[i] & 0xffffffffu) : -1;
      const bool head = i < n_st && (i == 0 || (int)(sh_sort[i - 1] & 0xffffffffu) != c);
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
      s_naff = n_aff;
    }
  }
  __syncthreads();
  // dV: one group of LPR lanes per affected cluster, members in slot order
  constexpr int EPL = Elem<T>::kPerVec, LPR = D / EPL, GPB = kStreamThreads / LPR;
  const int lane = threadIdx.x & 31, sub = lane % LPR, grp = threadIdx.x / LPR;
  const int n_aff = s_naff;
  const int32_t* ast = a.aff_start + (int64_t)u * (a.cap + 1);
  const T* vb = reinterpret_cast<const T*>(a.vp.base) + sub * EPL;
  for (int j = grp; j < n_aff; j += GPB) {
    float acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
    int i0 = 0, i1 = 0;  // steady index range of cluster j (recomputed from the sorted list)
    {
      // the j-th run head: count heads until j (runs are short; ast was written above)
      i0 = ast[j];
      i1 = ast[j + 1];
    }
    for (int i = i0; i < i1; ++i) {
      const int slot = (int)(sh_sort[i] >> 32);
      const int64_t ro = pool_row(a.vp, geo.hkv, D, b, h, slot, status);
      if (ro >= 0) {
        float x[EPL];
        Elem<T>::unpack(ld_stream(vb + ro), x);
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] += x[e];
      }
    }
    float* dst = a.dv + ((int64_t)u * a.cap + j) * D + sub * EPL;
#pragma unroll
    for (int e = 0; e < EPL; ++e) dst[e] = acc[e];
  }
}

// ---------------------------------------------------------------- K_A score
// Each CTA stages its chunk of centroid rows (64 KB) in shared memory with
// 16-byte cp.async, scores it, writes the per-head scores and the
// order-preserving group-max keys, and adds its keys' top 11 bits to the
// unit's selection histogram (the first radix digit of the top-k).
constexpr int kHistBins = 2048;
constexpr int kHistShift = 21;

template <typename T, int D, int G>
__global__ void __launch_bounds__(kStreamThreads)
wave_score_kernel(const Geo geo, const T* __restrict__ q, int n_q_heads, const T* __restrict__ cent,
                  const int32_t* __restrict__ offsets, float* __restrict__ scores,
                  uint32_t* __restrict__ keys, int32_t* __restrict__ hist_g, float scale,
                  int n_score_blocks, const SteadyArgs sa, uint32_t* status) {
  using RS = RowShape<T, D>;
  constexpr int EPL = RS::EPL, LPR = RS::LPR, RPW = RS::RPW;
  constexpr int NW = kStreamThreads / 32;
  constexpr int CROWS = 65536 / RS::ROWB;   // rows per CTA
  static_assert(G <= LPR, "group larger than lanes per row");
  extern __shared__ __align__(16) unsigned char sh_dyn[];
  pdl_launch_dependents();
  const int u = blockIdx.y;
  if (blockIdx.x == n_score_blocks) {
    steady_role<T, D>(geo, u, sa, status, reinterpret_cast<unsigned long long*>(sh_dyn));
    return;
  }
  const int b = u / geo.hkv, h = u - b * geo.hkv;
  const int NC = geo.NC(b);
  const int c0 = blockIdx.x * CROWS;
  if (c0 >= NC) return;
  const int c1 = min(NC, c0 + CROWS);
  const int nrows = c1 - c0;
  T* rows = reinterpret_cast<T*>(sh_dyn);
  int* hist = reinterpret_cast<int*>(sh_dyn + 65536);
  int* s_off = hist + kHistBins;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tid = threadIdx.x;
  const int sub = lane % LPR, rsub = lane / LPR;
  const int64_t row0 = geo.cl_row(b, h);
  const T* src = cent + (row0 + c0) * D;
  constexpr int TR = RS::TILE, NT = CROWS / TR;  // 4 tiles of 16 KB, one cp.async group each
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int r0 = t * TR, nr = min(TR, nrows - r0);
    for (int i = tid; i < nr * LPR; i += blockDim.x)
      cp_async16(rows + (r0 * LPR + i) * EPL, src + (r0 * LPR + i) * EPL);
    cp_async_commit();
  }
  const int32_t* off = offsets + geo.off_row(b, h) + c0;
  for (int i = tid; i <= nrows; i += blockDim.x) s_off[i] = __ldg(off + i);
  for (int i = tid; i < kHistBins; i += blockDim.x) hist[i] = 0;
  float qv[G][EPL];
  load_q<T, D, G>(q, n_q_heads, b, h, sub, scale, qv);
  const int j = sub / (LPR / G);
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    cp_async_wait_dyn(NT - 1 - t);  // tile t has landed; later tiles still in flight
    __syncthreads();
    const int r1 = min(nrows, (t + 1) * TR);
    for (int rb = t * TR + warp * RPW; rb < r1; rb += NW * RPW) {
      const int r = rb + rsub;
      const bool ok = r < r1;
      float x[EPL];
      if (ok) {
        Elem<T>::unpack(*reinterpret_cast<const uint4*>(rows + r * D + sub * EPL), x);
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
        if (sub % (LPR / G) == 0) scores[(row0 + c0 + r) * G + j] = acc[0];
        if (sub == 0) {
          const uint32_t key = (s_off[r + 1] - s_off[r]) > 0 ? ordered_key(m) : 0u;
          keys[row0 + c0 + r] = key;
          if (key) atomicAdd(&hist[key >> kHistShift], 1);
        }
      }
    }
  }
  __syncthreads();
  int* hg = hist_g + (int64_t)u * kHistBins;
  for (int i = tid; i < kHistBins; i += blockDim.x)
    if (hist[i]) atomicAdd(hg + i, hist[i]);
}

// ----------------------------------------------------------------- K_B topk
// One CTA per unit.  Keys are walked in rounds of kTopkThreads*16: warp w
// owns a contiguous id range of 512 per round, lane-interleaved (coalesced
// loads, ballot-based ranking, no shared-memory bank conflicts).
//  1. the first radix digit's histogram comes from K_A (zeroed after use, so
//     the workspace is clean for the next call; a histogram whose total
//     disagrees with the candidate count is rebuilt and flagged);
//  2. the keys in the threshold bin (1-2% of them) are gathered and ranked
//     exactly by (key desc, id asc); more than kTopkCand of them fall back
//     to two further radix digits over all keys;
//  3. an ordered compaction writes the selection, its slot starts, the token
//     prefix, the split starts and the gather list (pool rows of the
//     retrieved clusters' tokens, -1 for their steady members).
constexpr int kTopkPerLane = 16;
constexpr int kTopkRound = kTopkThreads * kTopkPerLane;   // 8192 ids per round
constexpr int kTopkCand = 1024;

__global__ void __launch_bounds__(kTopkThreads)
wave_topk_kernel(const Geo geo, const uint32_t* __restrict__ keys,
                 const int32_t* __restrict__ offsets, int32_t* __restrict__ hist_g,
                 const int32_t* __restrict__ aff_cl, const int32_t* __restrict__ aff_start, int cap,
                 int topk_clusters, double topk_fraction, int n_splits,
                 int32_t* __restrict__ sel, int32_t* __restrict__ sel_slot0,
                 int32_t* __restrict__ sel_tok, int32_t* __restrict__ split_first,
                 int32_t* __restrict__ info, const int32_t* __restrict__ st_slot, const Pool kp,
                 int32_t* __restrict__ gather, int64_t gather_stride, uint32_t* status) {
  // dynamic shared: excluded bitmask [ceil(NCmax/32)] | steady slots [cap]
  //                 | affected list [cap] | round list (token start, slot start) [2 * kTopkRound + 2]
  extern __shared__ int32_t sdyn[];
  __shared__ int hist[kHistBins];
  __shared__ unsigned long long cand[kTopkCand];
  __shared__ int scan_sh[64];
  __shared__ int s_info[kInfoInts];
  __shared__ int s_w[2][32];
  __shared__ int s_ctl[8];
  pdl_launch_dependents();
  const int tid = threadIdx.x, nt = kTopkThreads, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = kTopkThreads / 32;
  const unsigned lt = (1u << lane) - 1u;
  const int u = blockIdx.x, b = u / geo.hkv, h = u - b * geo.hkv;
  const int NC = geo.NC(b), Tb = geo.T(b);
  const int nmask = (NC + 31) >> 5;
  uint32_t* sx = reinterpret_cast<uint32_t*>(sdyn);
  int32_t* ss = sdyn + nmask;
  int32_t* sa = ss + cap;
  int32_t* lst = sa + cap;                         // [kTopkRound + 1] token starts
  int32_t* lso = lst + kTopkRound + 1;             // [kTopkRound] slot starts
  for (int i = tid; i < nmask; i += nt) sx[i] = 0u;
  if (tid == 0) s_ctl[0] = 0;
  pdl_wait();
  int32_t* I = info + (int64_t)u * kInfoInts;
  const int64_t row0 = geo.cl_row(b, h);
  int32_t* pre = sel_tok + row0 + u;
  int32_t* split = split_first + (int64_t)u * (n_splits + 1);
  int* hg = hist_g + (int64_t)u * kHistBins;
  const int k_req = topk_clusters >= 0 ? topk_clusters : (int)ceil(topk_fraction * (double)NC);
  const uint32_t* kk = keys + row0;
  const int32_t* off = offsets + geo.off_row(b, h);
  int32_t* gat = gather + (int64_t)u * gather_stride;
  // one round of independent loads
  if (tid < kInfoInts) s_info[tid] = I[tid];
  for (int i = tid; i < kHistBins; i += nt) { hist[i] = hg[i]; hg[i] = 0; }
  for (int i = tid; i < cap; i += nt) {
    sa[i] = aff_cl[(int64_t)u * cap + i];
    ss[i] = st_slot[(int64_t)u * cap + i];
  }
  __syncthreads();
  const int n_st = s_info[4];
  const int dense = s_info[6];
  const int n_aff = dense ? 0 : min(cap, s_info[5]);
  auto row_of = [&](int slot) -> int32_t {
    const int64_t ro = pool_row(kp, geo.hkv, 1, b, h, slot, status);
    return ro < 0 ? -1 : (int32_t)ro;
  };
  if (dense) {  // the attend CTAs take all slots in order
    for (int t = tid; t < Tb; t += nt) gat[t] = row_of(t);
    if (tid == 0) {
      I[0] = 0; I[1] = (int32_t)0xFFFFFFFFu; I[2] = -1; I[3] = 0; I[7] = k_req;
      pre[0] = 0;
    }
    for (int j = tid; j <= n_splits; j += nt) split[j] = 0;
    return;
  }
  // clusters left without a non-steady member are not candidates
  for (int j = tid; j < n_aff; j += nt) {
    const int c = sa[j];
    const int dc = aff_start[(int64_t)u * (cap + 1) + j + 1] - aff_start[(int64_t)u * (cap + 1) + j];
    if (c >= 0 && c < NC && __ldg(off + c + 1) - __ldg(off + c) - dc <= 0) {
      atomicOr(&sx[c >> 5], 1u << (c & 31));
      const uint32_t key = kk[c];
      if (key) atomicSub(&hist[key >> kHistShift], 1);
    }
  }
  __syncthreads();
  auto cand_key = [&](int c, uint32_t key) -> uint32_t {
    return ((sx[c >> 5] >> (c & 31)) & 1u) ? 0u : key;
  };
  const int n_rounds = (NC + kTopkRound - 1) / kTopkRound;
  const int wbase = warp * (kTopkRound / NW);       // warp's offset inside a round

  // histogram total -> threshold bin of the first digit (valid if consistent)
  int hs = 0;
  for (int i = tid; i < kHistBins; i += nt) hs += hist[i];
  int hist_total;
  block_inclusive_scan(hs, scan_sh, &hist_total);
  int ksel = min(max(k_req, 0), hist_total);
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

  // the round's keys / offsets in registers: all loads issued before any use
  uint32_t kr[kTopkPerLane];
  int o0r[kTopkPerLane], o1r[kTopkPerLane];
  auto load_round = [&](int r, bool with_off) {
#pragma unroll
    for (int i = 0; i < kTopkPerLane; ++i) {
      const int c = r * kTopkRound + wbase + i * 32 + lane;
      kr[i] = c < NC ? kk[c] : 0u;
      if (with_off) {
        o0r[i] = c < NC ? __ldg(off + c) : 0;
        o1r[i] = c < NC ? __ldg(off + c + 1) : 0;
      }
    }
#pragma unroll
    for (int i = 0; i < kTopkPerLane; ++i) {
      const int c = r * kTopkRound + wbase + i * 32 + lane;
      kr[i] = c < NC ? cand_key(c, kr[i]) : 0u;
    }
  };
  // pass A: candidate count, and the keys of the threshold bin
  int mine = 0;
  for (int r = 0; r < n_rounds; ++r) {
    load_round(r, true);
#pragma unroll
    for (int i = 0; i < kTopkPerLane; ++i) {
      const uint32_t key = kr[i];
      if (key == 0u) continue;
      ++mine;
      if ((int)(key >> kHistShift) == bin1) {
        const int c = r * kTopkRound + wbase + i * 32 + lane;
        const int slot = atomicAdd(&s_ctl[0], 1);
        if (slot < kTopkCand)
          cand[slot] = ((unsigned long long)key << 32) | (0xFFFFFFFFu - (uint32_t)c);
      }
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
  if (ksel == 0) { kstar = 0xFFFFFFFFu; thr = -1; }
  else if (ksel == ncand) { kstar = 1u; thr = NC; }
  else if (hist_ok && nbin <= kTopkCand) {
    // exact rank inside the threshold bin: the (ksel - above1)-th largest
    const int want = ksel - above1 - 1;
    for (int i = tid; i < nbin; i += nt) {
      const unsigned long long x = cand[i];
      int rank = 0;
      for (int j = 0; j < nbin; ++j) rank += cand[j] > x;
      if (rank == want) { s_ctl[3] = (int)(x >> 32); s_ctl[4] = (int)(0xFFFFFFFFu - (uint32_t)x); }
    }
    __syncthreads();
    kstar = (uint32_t)s_ctl[3];
    thr = s_ctl[4];
  } else {
    // fallback: a full radix select over all keys (stale histogram or a
    // crowded threshold bin), 11 + 11 + 10 bit digits
    uint32_t prefix = 0, pmask = 0;
    int krem = ksel;
    for (int pass = 0; pass < 3; ++pass) {
      const int bits = pass == 2 ? 10 : 11;
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const int nbins = 1 << bits;
      for (int i = tid; i < kHistBins; i += nt) hist[i] = 0;
      __syncthreads();
      for (int c = tid; c < NC; c += nt) {
        const uint32_t key = cand_key(c, kk[c]);
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
      const int f = (c < NC && cand_key(c, kk[c]) == kstar) ? 1 : 0;
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

  // pass B: ordered compaction, round by round
  int sel_run = 0, tok_run = 0;   // totals of earlier rounds
  int total_tok = 0;
  {  // token total first: the split length depends on it
    int tk = 0;
    for (int r = 0; r < n_rounds; ++r) {
      if (n_rounds > 1) load_round(r, true);
#pragma unroll
      for (int i = 0; i < kTopkPerLane; ++i) {
        const int c = r * kTopkRound + wbase + i * 32 + lane;
        if (picked(c, kr[i])) tk += o1r[i] - o0r[i];
      }
    }
    block_inclusive_scan(tk, scan_sh, &total_tok);
  }
  const int n_tok = total_tok + n_st;
  const int split_len = (n_tok + n_splits - 1) / n_splits;
  for (int r = 0; r < n_rounds; ++r) {
    if (n_rounds > 1) load_round(r, true);
    int cnt = 0, tk = 0;
#pragma unroll
    for (int i = 0; i < kTopkPerLane; ++i) {
      const int c = r * kTopkRound + wbase + i * 32 + lane;
      const bool p = picked(c, kr[i]);
      cnt += __popc(__ballot_sync(0xffffffffu, p));
      tk += p ? o1r[i] - o0r[i] : 0;
    }
    tk = warp_sum_int(tk);
    if (lane == 0) { s_w[0][warp] = cnt; s_w[1][warp] = tk; }
    __syncthreads();
    int sb = sel_run, tb = tok_run, rs = 0, rt = 0;
    for (int w = 0; w < NW; ++w) {
      if (w < warp) { sb += s_w[0][w]; tb += s_w[1][w]; }
      rs += s_w[0][w]; rt += s_w[1][w];
    }
    // write this warp's selection in id order
#pragma unroll
    for (int i = 0; i < kTopkPerLane; ++i) {
      const int c = r * kTopkRound + wbase + i * 32 + lane;
      const bool p = picked(c, kr[i]);
      const int o0 = o0r[i];
      const int n = p ? o1r[i] - o0 : 0;
      const unsigned bs = __ballot_sync(0xffffffffu, p);
      int incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (p) {
        const int si = sb + __popc(bs & lt), st = tb + incl - n;
        sel[row0 + si] = c;
        sel_slot0[row0 + si] = o0;
        pre[si] = st;
        lst[si - sel_run] = st;
        lso[si - sel_run] = o0;
        if (split_len > 0)  // splits whose first token falls inside this cluster start at it
          for (int j = (st + split_len - 1) / split_len; j * split_len < st + n && j < n_splits; ++j)
            split[j] = si;
      }
      sb += __popc(bs);
      tb += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (tid == 0) lst[rs] = tok_run + rt;
    __syncthreads();
    // gather list: the round's tokens expanded CTA-wide
    for (int qq = tok_run + tid; qq < tok_run + rt; qq += nt) {
      int lo = 0, hi = rs - 1;  // largest k with lst[k] <= qq
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (lst[mid] <= qq) lo = mid; else hi = mid - 1;
      }
      const int slot = lso[lo] + (qq - lst[lo]);
      gat[qq] = find_sorted(ss, n_st, slot) >= 0 ? -1 : row_of(slot);
    }
    sel_run += rs;
    tok_run += rt;
    __syncthreads();
  }
  for (int j = tid; j < n_st; j += nt) gat[total_tok + j] = row_of(ss[j]);
  if (tid == 0) {
    pre[ksel] = total_tok;
    const int j0 = split_len > 0 ? (total_tok + split_len - 1) / split_len : 0;
    for (int j = j0; j <= n_splits; ++j) split[j] = ksel;
    I[0] = ksel; I[1] = (int32_t)kstar; I[2] = thr; I[3] = total_tok; I[7] = k_req;
  }
}

// -------------------------------------------------- K_C attend + estimate
struct AttendArgs {
  const int32_t *gather, *aff_cl, *aff_start;
  const float* dv;
  int64_t gather_stride;
  const int32_t* info;
  const float* scores;
  const uint32_t* keys;
  int n_sink, window, cap, n_splits, n_est, echunk, n_parts, wcap;
  float* partials;
  int32_t* counters;
  float* out;
  float* lse;
  float scale;
};

// A softmax part of one (unit, q head): {m, l, -, -, o[D]}; o starts 16-byte aligned.
template <int D>
struct Part {
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

template <typename T, int D, int G>
__global__ void __launch_bounds__(kStreamThreads)
wave_attend_estimate_kernel(const Geo geo, const T* __restrict__ q, int n_q_heads, const Pool kp,
                            const Pool vp, const T* __restrict__ vsum,
                            const int32_t* __restrict__ offsets, const AttendArgs A,
                            uint32_t* status) {
  using RS = RowShape<T, D>;
  constexpr int EPL = RS::EPL, LPR = RS::LPR, RPW = RS::RPW, TR = RS::TILE;
  constexpr int NW = kStreamThreads / 32;
  constexpr int NST = 4;                    // estimate ring stages (TR rows each)
  static_assert(TR % (NW * RPW) == 0, "tile must be a multiple of rows per CTA step");
  extern __shared__ __align__(16) unsigned char sh[];
  // shared layout: [ring: 4 tiles of TR rows (attend: K x2, V x2); the final
  //                 cross-warp reduction reuses it] [s_w wcap*G f32]
  //                [s_cnt echunk i32] [steady / affected lists 2*cap+2 i32]
  T* ring = reinterpret_cast<T*>(sh);
  float* s_red = reinterpret_cast<float*>(sh);
  float* s_w = reinterpret_cast<float*>(sh + NST * TR * RS::ROWB);
  int* s_cnt = reinterpret_cast<int*>(s_w + A.wcap * G);
  int32_t* s_list = s_cnt + A.echunk;
  __shared__ int64_t s_row[2][TR];
  __shared__ float s_sc[TR][G];
  __shared__ int s_last;
  __shared__ float s_m[G], s_l[G], s_part[NW][G];
  __shared__ int s_info[kInfoInts];

  const int u = blockIdx.y, b = u / geo.hkv, h = u - b * geo.hkv;
  const int Tb = geo.T(b), NC = geo.NC(b);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tid = threadIdx.x;
  const int sub = lane % LPR, rsub = lane / LPR;
  const int jh = sub / (LPR / G);
  const int64_t row0 = geo.cl_row(b, h);
  const int32_t* off = offsets + geo.off_row(b, h);
  const bool role_est = (int)blockIdx.x >= A.n_splits;
  constexpr int PS = Part<D>::kStride;
  float* part = A.partials + ((int64_t)u * A.n_parts + blockIdx.x) * G * PS;

  float acc[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;

  if (role_est) {
    // ------------------------------------------------------------ estimate
    const int c0 = (blockIdx.x - A.n_splits) * A.echunk;
    const int c1 = min(NC, c0 + A.echunk);
    const int ntile = c0 < c1 ? (c1 - c0 + TR - 1) / TR : 0;
    const T* vrow = vsum + row0 * D;
    auto issue = [&](int t) {
      if (t < ntile) {
        T* dst = ring + (size_t)(t % NST) * TR * D;
        const int r0 = c0 + t * TR, nr = min(TR, c1 - r0);
        for (int i = tid; i < nr * LPR; i += blockDim.x) {
          const int r = i / LPR, ch = i - r * LPR;
          cp_async16(dst + r * D + ch * EPL, vrow + (int64_t)(r0 + r) * D + ch * EPL);
        }
      }
      cp_async_commit();
    };
#pragma unroll
    for (int t = 0; t < NST; ++t) issue(t);  // value sums do not depend on the selection
    pdl_wait();
    // one round of independent loads: unit record, affected list, and the
    // chunk's keys, offsets and scores (kept in registers across the barrier)
    constexpr int EPT = 2;                       // clusters per thread (echunk <= 512)
    const int32_t* I = A.info + (int64_t)u * kInfoInts;
    if (tid < kInfoInts) s_info[tid] = I[tid];
    int32_t* s_acl = s_list;
    int32_t* s_ast = s_list + A.cap;
    for (int i = tid; i < A.cap; i += blockDim.x) {
      s_acl[i] = A.aff_cl[(int64_t)u * A.cap + i];
      s_ast[i] = A.aff_start[(int64_t)u * (A.cap + 1) + i];
    }
    if (tid == 0) s_ast[A.cap] = A.aff_start[(int64_t)u * (A.cap + 1) + A.cap];
    uint32_t kv[EPT];
    int cv[EPT];
    float sv[EPT][G];
#pragma unroll
    for (int k = 0; k < EPT; ++k) {
      const int c = c0 + tid + k * kStreamThreads;
      kv[k] = 0u; cv[k] = 0;
      if (c < c1) {
        kv[k] = A.keys[row0 + c];
        cv[k] = __ldg(off + c + 1) - __ldg(off + c);
      }
#pragma unroll
      for (int g = 0; g < G; ++g) sv[k][g] = c < c1 ? A.scores[(row0 + c) * G + g] : -INFINITY;
    }
    __syncthreads();
    const bool skip = s_info[6] || c0 >= c1;
    const int n_aff = s_info[6] ? 0 : min(A.cap, s_info[5]);
    if (!skip) {
      const uint32_t kstar = (uint32_t)s_info[1];
      const int thr = s_info[2];
      float m_loc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) m_loc[g] = -INFINITY;
#pragma unroll
      for (int k = 0; k < EPT; ++k) {
        const int i = tid + k * kStreamThreads;
        if (i >= c1 - c0) continue;
        const int c = c0 + i;
        const uint32_t key = kv[k];
        const bool picked = key > kstar || (key == kstar && c <= thr);
        int cntp = cv[k];
        bool contrib = key != 0u && !picked;
        if (contrib && n_aff > 0) {
          const int f = find_sorted(s_acl, n_aff, c);
          if (f >= 0) cntp -= s_ast[f + 1] - s_ast[f];
        }
        contrib = contrib && cntp > 0;
        s_cnt[i] = contrib ? cntp : 0;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float v = contrib ? sv[k][g] : -INFINITY;
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
      if (tid < G) {
        float v = -INFINITY;
        for (int w = 0; w < NW; ++w) v = fmaxf(v, s_part[w][tid]);
        s_m[tid] = v;
      }
      __syncthreads();
      float l_loc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) l_loc[g] = 0.f;
      for (int i = tid; i < c1 - c0; i += blockDim.x) {
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
      __syncthreads();
      if (tid < G) {
        float v = 0.f;
        for (int w = 0; w < NW; ++w) v += s_part[w][tid];
        s_l[tid] = v;
      }
    }
    // stream the value sums through the ring
    for (int t = 0; t < ntile; ++t) {
      cp_async_wait<NST - 1>();
      __syncthreads();
      if (!skip) {
        const T* tile = ring + (size_t)(t % NST) * TR * D;
        const int r0 = t * TR, nr = min(TR, c1 - c0 - r0);
        for (int rb = warp * RPW; rb < nr; rb += NW * RPW) {
          const int r = rb + rsub;
          if (r < nr && s_cnt[r0 + r] > 0) {
            const uint4 raw = *reinterpret_cast<const uint4*>(tile + r * D + sub * EPL);
            float x[EPL];
            Elem<T>::unpack(raw, x);
            float wv[G];
#pragma unroll
            for (int g = 0; g < G; ++g) wv[g] = s_w[(r0 + r) * G + g];
            axpy_g<G, EPL>(wv, x, acc);
          }
        }
      }
      __syncthreads();
      issue(t + NST);
    }
    cp_async_wait<0>();
    if (!skip) {
      // Vsum' = Vsum - (values of the cluster's steady members)
      int a0, a1;
      {  // affected clusters inside [c0, c1)
        int lo = 0, hi = n_aff;
        while (lo < hi) { const int mid = (lo + hi) >> 1; if (s_acl[mid] < c0) lo = mid + 1; else hi = mid; }
        a0 = lo;
        hi = n_aff;
        while (lo < hi) { const int mid = (lo + hi) >> 1; if (s_acl[mid] < c1) lo = mid + 1; else hi = mid; }
        a1 = lo;
      }
      // each affected cluster of the chunk that is estimated: subtract w * dV
      for (int base = a0 + warp * RPW; base < a1; base += NW * RPW) {
        const int j = base + rsub;
        if (j >= a1) continue;
        const int ci = s_acl[j] - c0;
        if (ci < 0 || ci >= c1 - c0 || s_cnt[ci] <= 0) continue;
        const float* dvr = A.dv + ((int64_t)u * A.cap + j) * D + sub * EPL;
        float x[EPL];
#pragma unroll
        for (int e4 = 0; e4 < EPL; e4 += 4) {
          const float4 v = *reinterpret_cast<const float4*>(dvr + e4);
          x[e4] = v.x; x[e4 + 1] = v.y; x[e4 + 2] = v.z; x[e4 + 3] = v.w;
        }
        float wv[G];
#pragma unroll
        for (int g = 0; g < G; ++g) wv[g] = -s_w[ci * G + g];
        axpy_g<G, EPL>(wv, x, acc);
      }
      reduce_and_store<G, EPL, LPR, D>(acc, s_red, warp, sub, rsub, part);
      if (tid < G) { part[tid * PS] = s_m[tid]; part[tid * PS + 1] = s_l[tid]; }
    } else {
      for (int i = tid; i < G * PS; i += blockDim.x) part[i] = (i % PS) == 0 ? -INFINITY : 0.f;
    }
  } else {
    // -------------------------------------------------------------- attend
    float qv[G][EPL];
    load_q<T, D, G>(q, n_q_heads, b, h, sub, A.scale, qv);
    pdl_wait();
    const int32_t* I = A.info + (int64_t)u * kInfoInts;
    const int dense = I[6];
    const int n_tok = (dense ? 0 : I[3]) + I[4];
    const int per = (n_tok + A.n_splits - 1) / A.n_splits;
    const int t0 = min(n_tok, (int)blockIdx.x * per);
    const int t1 = min(n_tok, t0 + per);
    const int32_t* gat = A.gather + (int64_t)u * A.gather_stride;
    T* const kt0 = ring;
    T* const vt0 = ring + (size_t)2 * TR * D;
    const T* kbase = reinterpret_cast<const T*>(kp.base);
    const T* vbase = reinterpret_cast<const T*>(vp.base);
    const int ntile = t0 < t1 ? (t1 - t0 + TR - 1) / TR : 0;

    // tile t: pool rows from the gather list, then 16-byte copies of K and V
    auto stage = [&](int t) {
      const int bi = t & 1;
      const int tb = t0 + t * TR, n = min(TR, t1 - tb);
      if (tid < TR) {
        const int32_t ri = tid < n ? gat[tb + tid] : -1;
        s_row[bi][tid] = ri >= 0 ? (int64_t)ri * D : -1;
      }
      __syncthreads();
      T* kt = kt0 + (size_t)bi * TR * D;
      T* vt = vt0 + (size_t)bi * TR * D;
      for (int i = tid; i < n * LPR; i += blockDim.x) {
        const int r = i / LPR, ch = i - r * LPR;
        const int64_t ro = s_row[bi][r];
        if (ro >= 0) {
          cp_async16(kt + r * D + ch * EPL, kbase + ro + ch * EPL);
          cp_async16(vt + r * D + ch * EPL, vbase + ro + ch * EPL);
        }
      }
      cp_async_commit();
    };

    float m_run[G], l_run[G];
#pragma unroll
    for (int g = 0; g < G; ++g) { m_run[g] = -INFINITY; l_run[g] = 0.f; }
    if (ntile > 0) stage(0);
    for (int t = 0; t < ntile; ++t) {
      const int bi = t & 1;
      if (t + 1 < ntile) { stage(t + 1); cp_async_wait<1>(); } else { cp_async_wait<0>(); }
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
      __syncthreads();
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
  if (tid == 0) s_last = atomicAdd(A.counters + u, 1) == A.n_parts - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // stage every part's (m, l) in shared memory with one round of loads
  float* f = s_w;                                   // [n_parts][G] rescale factors
  float* lp = reinterpret_cast<float*>(ring);       // [n_parts][G] part denominators
  const float* pbase = A.partials + (int64_t)u * A.n_parts * G * PS;
  for (int i = tid; i < A.n_parts * G; i += blockDim.x) {
    f[i] = __ldcg(pbase + (int64_t)i * PS);
    lp[i] = __ldcg(pbase + (int64_t)i * PS + 1);
  }
  __syncthreads();
  if (warp < G) {
    float M = -INFINITY;
    for (int p = lane; p < A.n_parts; p += 32) M = fmaxf(M, f[p * G + warp]);
    M = warp_max(M);
    float l = 0.f;
    for (int p = lane; p < A.n_parts; p += 32) {
      const float mp = f[p * G + warp];
      l += mp == -INFINITY ? 0.f : expf(mp - M) * lp[p * G + warp];
    }
    l = warp_sum(l);
    if (lane == 0) { s_m[warp] = M; s_l[warp] = l; }
  }
  __syncthreads();
  for (int i = tid; i < A.n_parts * G; i += blockDim.x) {
    const float mp = f[i];
    f[i] = mp == -INFINITY ? 0.f : expf(mp - s_m[i % G]);
  }
  __syncthreads();
  {
    // thread t sums float4 chunk (t % NCH) over parts p = t / NCH, t / NCH + PP, ...
    constexpr int NCH = G * D / 4;                  // float4 chunks of one part's outputs
    constexpr int PP = kStreamThreads / NCH > 0 ? kStreamThreads / NCH : 1;
    float4* red4 = reinterpret_cast<float4*>(lp + ((A.n_parts * G + 3) & ~3));
    for (int ch = tid % NCH; ch < NCH; ch += kStreamThreads) {
      const int g = (ch * 4) / D, e = (ch * 4) - g * D;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      int p = tid / NCH;
      for (; p + 3 * PP < A.n_parts; p += 4 * PP) {  // four independent loads in flight
        float4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          v[k] = __ldcg(reinterpret_cast<const float4*>(pbase + ((int64_t)(p + k * PP) * G + g) * PS + Part<D>::kO + e));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float w = f[(p + k * PP) * G + g];
          o.x += w * v[k].x; o.y += w * v[k].y; o.z += w * v[k].z; o.w += w * v[k].w;
        }
      }
      for (; p < A.n_parts; p += PP) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(pbase + ((int64_t)p * G + g) * PS + Part<D>::kO + e));
        const float w = f[p * G + g];
        o.x += w * v.x; o.y += w * v.y; o.z += w * v.z; o.w += w * v.w;
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

size_t decode_attend_smem(int dtype, int D, int G, int wcap, int echunk, int cap) {
  (void)dtype;
  const size_t ring = 4 * 16384;  // also holds the NW*G*D fp32 reduction (<= 32 KB)
  return ring + (size_t)wcap * G * 4 + (size_t)echunk * 4 + (size_t)(2 * cap + 2) * 4;
}

cudaError_t launch_decode(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
  unsigned char* ws = a.ws;
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + p.off_status);
  float* scores = reinterpret_cast<float*>(ws + p.off_scores);
  uint32_t* keys = reinterpret_cast<uint32_t*>(ws + p.off_keys);
  int32_t* sel = reinterpret_cast<int32_t*>(ws + p.off_sel);
  int32_t* sel_slot0 = reinterpret_cast<int32_t*>(ws + p.off_sel_slot0);
  int32_t* seltok = reinterpret_cast<int32_t*>(ws + p.off_seltok);
  int32_t* split_first = reinterpret_cast<int32_t*>(ws + p.off_split);
  int32_t* info = reinterpret_cast<int32_t*>(ws + p.off_info);
  int32_t* counters = reinterpret_cast<int32_t*>(ws + p.off_counters);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + p.off_hist);
  int32_t* st_slot = reinterpret_cast<int32_t*>(ws + p.off_st_slot);
  int32_t* st_cl = reinterpret_cast<int32_t*>(ws + p.off_st_cl);
  int32_t* aff_cl = reinterpret_cast<int32_t*>(ws + p.off_aff_cl);
  int32_t* aff_start = reinterpret_cast<int32_t*>(ws + p.off_aff_start);
  float* partials = reinterpret_cast<float*>(ws + p.off_partials);
  int32_t* gather = reinterpret_cast<int32_t*>(ws + p.off_gather);
  float* dv = reinterpret_cast<float*>(ws + p.off_dv);
  cudaEvent_t* ev = a.stage_events;
  const bool pdl = ev == nullptr;  // stage timing serialises the launches
  auto mark = [&](int i) { if (ev) cudaEventRecord(ev[i], s); };

  return with_types(p.dtype, p.D, p.G, [&]<typename T, int D, int G>() -> cudaError_t {
    const T* q = reinterpret_cast<const T*>(a.q);
    SteadyArgs sa{a.invperm, a.labels, a.vp, p.n_sink, p.window, p.cap, p.sort_pow2, st_slot,
                  st_cl, aff_cl, aff_start, info, dv};
    cudaError_t e;
    mark(0);
    const size_t score_smem = std::max<size_t>(65536 + (kHistBins + 1) * 4 +
                                                   (size_t)(65536 / (D * sizeof(T)) + 1) * 4,
                                               (size_t)p.sort_pow2 * 8);
    cudaFuncSetAttribute(wave_score_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)score_smem);
    e = launch_ex(wave_score_kernel<T, D, G>, dim3(p.n_score_blocks + 1, p.U),
                  dim3(kStreamThreads), score_smem, s, false, p.geo, q, p.Hq,
                  reinterpret_cast<const T*>(a.centroids), a.offsets, scores, keys, hist, p.scale,
                  p.n_score_blocks, sa, status);
    if (e != cudaSuccess) return e;
    mark(1);
    const size_t topk_smem = ((size_t)(p.max_nc + 31) / 32 + 2 * (size_t)p.cap +
                              2 * (size_t)kTopkRound + 2) * sizeof(int32_t);
    cudaFuncSetAttribute(wave_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)topk_smem);
    e = launch_ex(wave_topk_kernel, dim3(p.U), dim3(kTopkThreads), topk_smem, s, pdl, p.geo,
                  (const uint32_t*)keys, a.offsets, hist, (const int32_t*)aff_cl,
                  (const int32_t*)aff_start, p.cap, p.topk_clusters, p.topk_fraction, p.n_splits,
                  sel, sel_slot0, seltok, split_first, info, (const int32_t*)st_slot, a.kp, gather,
                  (int64_t)p.gather_stride, status);
    if (e != cudaSuccess) return e;
    mark(2);
    AttendArgs A{gather, aff_cl, aff_start, dv, (int64_t)p.gather_stride, info, scores, keys,
                 p.n_sink, p.window, p.cap, p.n_splits, p.n_est, p.echunk, p.n_parts, p.wcap,
                 partials, counters, a.out, a.lse, p.scale};
    const size_t smem = decode_attend_smem(p.dtype, D, G, p.wcap, p.echunk, p.cap);
    cudaFuncSetAttribute(wave_attend_estimate_kernel<T, D, G>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    e = launch_ex(wave_attend_estimate_kernel<T, D, G>, dim3(p.n_splits + p.n_est, p.U),
                  dim3(kStreamThreads), smem, s, pdl, p.geo, q, p.Hq, a.kp, a.vp,
                  reinterpret_cast<const T*>(a.value_sums), a.offsets, A, status);
    if (e != cudaSuccess) return e;
    mark(3);
    return cudaGetLastError();
  });
}

}  // namespace wi

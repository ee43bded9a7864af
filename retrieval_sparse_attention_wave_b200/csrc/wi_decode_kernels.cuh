#pragma once
// Decode-step kernels of the wave index (sm_100a), included by the
// per-type translation units that instantiate them.
//
// One decode step is the query-dependent phase of the method (RetroInfer
// technical summary, section 2.A, items 1-3; Vortex summary, section 2.A
// forward_indexer).  Three launches, chained with programmatic dependent
// launch:
//
//  K0 steady   one CTA per unit resolves the steady zone (item 1): sink and
//              window positions -> slots and clusters, sorted by slot; the
//              clusters left without a non-steady token (not candidates) and
//              the steady tokens of the other affected clusters.  It runs
//              beside K1, whose tails are the first to need it.
//  K1 scan     persistent CTAs stream every cluster's centroid and value-sum
//              rows once, in tiles of 64 rows brought in by 2-D tensor copies
//              (one producer warp, a ring of slots, one mbarrier pair per
//              slot).  Eight consumer warps take 8 rows each: the scores
//              q . centroid / sqrt(d) of the group's heads (mma.sync, or
//              packed FMA for fp32), the group-max selection key and its
//              first radix digit, and ALL the clusters' estimation terms
//              (item 3) folded into one running softmax part per warp.  The
//              last CTA to finish a unit runs the unit's exact top-k (item
//              2; Vortex 2.C Top-K) in its tail and writes the rows the
//              gather reads.
//  K2 gather   token-balanced CTAs gather the retrieved clusters' token rows
//              and the steady rows through the block table (one bulk copy a
//              row) and attend them exactly (items 1 and 2); the same pass
//              takes back out of the
//              estimate what the estimation zone does not hold (the
//              retrieved clusters, the clusters left without a candidate
//              token, and the steady tokens of the other affected clusters).
//              The last CTA of each unit merges every part by log-sum-exp.
//
// The estimation zone is computed as "every cluster minus what the zone
// leaves out": the same sum over clusters, streamed in the same pass as the
// centroids instead of after the selection.  A cluster's estimated mass never
// exceeds the exact mass of its own tokens (Jensen), and those tokens are in
// the exact part, so the cancellation costs at most a few fp32 ulps of the
// merged output's denominator.
#include <cfloat>
#include <climits>
#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>
#include <type_traits>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "wi_common.cuh"
#include "wi_plan.h"

namespace wi {

namespace {

constexpr int kHistShift = 21;    // first radix digit: key bits 31..21
constexpr float kCancelRatio = 16.f;   // taken-out mass / merged denominator flagged above this
constexpr int kPartStride = 4;    // a softmax part of one head: {m, l, ln, -, o[D]}

// ------------------------------------------------------------------ tiles
// A tile holds kTileRows rows of D elements as NB = D * sizeof(T) / 128
// boxes of [kTileRows][128 bytes], each 128-byte swizzled: 16-byte chunk c
// of row r sits at r * 128 + ((c ^ (r & 7)) << 4) of its box.  That is the
// layout a SWIZZLE_128B tensor copy of a {128-byte, 64-row} box writes (the
// scan's tiles); ldmatrix reads it without bank conflicts.  The gather's
// tiles hold whole rows instead (PadTile below).
template <typename T, int D>
struct TileShape {
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int NB = kRowBytes / 128;
  static constexpr int kBoxBytes = kTileRows * 128;
  static constexpr int kBytes = NB * kBoxBytes;
  static constexpr int kChunks = kRowBytes / 16;
  static_assert(kRowBytes % 128 == 0, "rows of a multiple of 128 bytes");
};

// byte offset of 16-byte chunk c of row r in a tile
__device__ __forceinline__ int tile_off(int r, int c) {
  return (c >> 3) * (kTileRows * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

// Tile layouts the accumulators read: the scan's (the swizzled boxes above,
// as its tensor copies write them) and the gather's (whole rows of RB bytes,
// RB + 16 apart, as its row copies write them: the pad puts the same 16-byte
// chunk of eight consecutive rows in eight distinct groups of four banks).
struct SwzTile {
  __device__ static __forceinline__ int off(int r, int c) { return tile_off(r, c); }
};
template <int RB>
struct PadTile {
  static constexpr int kStride = RB + 16;
  static constexpr int kBytes = kTileRows * kStride;
  __device__ static __forceinline__ int off(int r, int c) { return r * kStride + c * 16; }
};

// Multipliers of the 8 rows a warp takes in one step: the row's weight in the
// numerator (wo) and in the denominator (wl); invalid rows take no part.
struct RowMult {
  float wo, wl;
  int valid;
};

// ------------------------------------------------- warp softmax accumulators
// One warp folds rows (a key row and a value row each, with multipliers wo
// and wl) into a running softmax part of the G query heads:
//   m = max score, l = sum wl e^(s - m), o = sum wo e^(s - m) value.
// Scores s = q_g . key / sqrt(d).

// bf16: tensor cores.  Scores on m16n8k16 (A = q, heads in rows 0..7; B = 8
// key rows by ldmatrix); the weights' two bf16 terms (w = hi + lo to about
// 2^-17) go in rows 0..7 and 8..15 of one m16n8k8 A operand, built in
// registers from the score fragments; B = value rows by ldmatrix.trans.
template <int D, int G>
struct MmaAcc {
  static_assert(G <= 8, "at most 8 query heads per KV head (MMA rows 0..7)");
  uint32_t qa0[D / 16], qa2[D / 16];
  float m, l;          // head lane / 4: running max, this lane's share of the sum
  float ln;            // this lane's share of the rows with negative weight, as magnitudes
  float o[D / 8][4];   // [n-tile][hi pair, lo pair] of output columns 8j + 2(lane % 4)

  __device__ __forceinline__ void load_q(const __nv_bfloat16* q_group) {
    const int lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    const uint32_t* qw = reinterpret_cast<const uint32_t*>(q_group + (g < G ? g : 0) * D);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qa0[ks] = g < G ? qw[8 * ks + tq] : 0u;
      qa2[ks] = g < G ? qw[8 * ks + 4 + tq] : 0u;
    }
  }
  __device__ __forceinline__ void reset() {
    m = -INFINITY;
    l = 0.f;
    ln = 0.f;
#pragma unroll
    for (int j = 0; j < D / 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[j][e] = 0.f;
  }
  // scores of rows r0 + 2t, r0 + 2t + 1 (t = lane % 4) for head lane / 4
  template <class Lay = SwzTile>
  __device__ __forceinline__ void scores(const unsigned char* ktile, int r0, float scale,
                                         float& s0, float& s1) const {
    const int lane = threadIdx.x & 31;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < D / 16; ks += 2) {
      uint32_t b[4];
      ldsm_x4(b, ktile + Lay::off(r0 + (lane & 7), 2 * ks + (lane >> 3)));
      mma_bf16(acc, qa0[ks], qa2[ks], b[0], b[1]);
      mma_bf16(acc, qa0[ks + 1], qa2[ks + 1], b[2], b[3]);
    }
    s0 = acc[0] * scale;
    s1 = acc[1] * scale;
  }
  // fold the warp's 8 rows r0 .. r0 + 7: s0 / s1 their scores (as above),
  // rm the rows' multipliers
  template <class Lay = SwzTile>
  __device__ __forceinline__ void fold(const unsigned char* vtile, int r0, float s0, float s1,
                                       const RowMult* rm) {
    const int lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    const RowMult m0 = rm[2 * tq], m1 = rm[2 * tq + 1];
    const float x0 = (g < G && m0.valid) ? s0 : -INFINITY;
    const float x1 = (g < G && m1.valid) ? s1 : -INFINITY;
    float mx = fmaxf(x0, x1);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mnew = fmaxf(m, mx);
    const float corr = mnew == -INFINITY ? 1.f : __expf(m - mnew);
    const float p0 = x0 == -INFINITY ? 0.f : __expf(x0 - mnew);
    const float p1 = x1 == -INFINITY ? 0.f : __expf(x1 - mnew);
    l = l * corr + m0.wl * p0 + m1.wl * p1;
    ln = ln * corr + fmaxf(-m0.wl, 0.f) * p0 + fmaxf(-m1.wl, 0.f) * p1;
    m = mnew;
    uint32_t hi, lo;
    split_bf16(m0.wo * p0, m1.wo * p1, hi, lo);
#pragma unroll
    for (int j = 0; j < D / 8; j += 4) {
      uint32_t b[4];
      ldsm_x4_t(b, vtile + Lay::off(r0 + (lane & 7), j + (lane >> 3)));
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int e = 0; e < 4; ++e) o[j + i][e] *= corr;
        mma_bf16_k8(o[j + i], hi, lo, b[i]);
      }
    }
  }
  // this warp's part -> comb [G][D + 4] = {m, l, ln, -, o[D]} per head
  __device__ __forceinline__ void to_smem(float* comb) const {
    const int lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    float ls = l, lns = ln;
    ls += __shfl_xor_sync(0xffffffffu, ls, 1);
    ls += __shfl_xor_sync(0xffffffffu, ls, 2);
    lns += __shfl_xor_sync(0xffffffffu, lns, 1);
    lns += __shfl_xor_sync(0xffffffffu, lns, 2);
    if (g < G) {
      float* row = comb + g * (D + kPartStride);
#pragma unroll
      for (int j = 0; j < D / 8; ++j)
        *reinterpret_cast<float2*>(row + kPartStride + 8 * j + 2 * tq) =
            make_float2(o[j][0] + o[j][2], o[j][1] + o[j][3]);
      if (tq == 0) { row[0] = m; row[1] = ls; row[2] = lns; }
    }
  }
};

// fp32: packed FMA.  Lane l reads 16-byte chunk l % LPR of row l / LPR (+ RPW
// per step); dot products are summed over the LPR lanes of a row.
template <int D, int G>
struct FmaAcc {
  static constexpr int LPR = D / 4, RPW = 32 / LPR, NST = 8 / RPW;
  static_assert(G <= LPR, "group larger than lanes per row");
  float qv[G][4];
  float m[G], l[G], ln[G];
  float o[G][4];

  __device__ __forceinline__ void load_q(const float* q_group, float scale) {
    const int sub = (threadIdx.x & 31) % LPR;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float4 v = reinterpret_cast<const float4*>(q_group + g * D)[sub];
      qv[g][0] = v.x * scale; qv[g][1] = v.y * scale; qv[g][2] = v.z * scale; qv[g][3] = v.w * scale;
    }
  }
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
      ln[g] = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) o[g][e] = 0.f;
    }
  }
  template <class Lay>
  __device__ __forceinline__ static float4 chunk(const unsigned char* tile, int r, int c) {
    return *reinterpret_cast<const float4*>(tile + Lay::off(r, c));
  }
  // scores of the warp's 8 rows into s [8][G] (shared memory of this warp)
  template <class Lay = SwzTile>
  __device__ __forceinline__ void scores(const unsigned char* ktile, int r0, float* s) const {
    const int lane = threadIdx.x & 31, sub = lane % LPR, rs = lane / LPR;
    const int j = sub / (LPR / G);
#pragma unroll
    for (int i = 0; i < NST; ++i) {
      const int r = RPW * i + rs;
      const float4 x = chunk<Lay>(ktile, r0 + r, sub);
      float a[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float2 t = __ffma2_rn(make_float2(qv[g][0], qv[g][1]), make_float2(x.x, x.y),
                              make_float2(0.f, 0.f));
        t = __ffma2_rn(make_float2(qv[g][2], qv[g][3]), make_float2(x.z, x.w), t);
        a[g] = t.x + t.y;
      }
      group_reduce_multi<G, LPR>(a, lane);
      if (sub % (LPR / G) == 0) s[r * G + j] = a[0];
    }
    __syncwarp();
  }
  template <class Lay = SwzTile>
  __device__ __forceinline__ void fold(const unsigned char* vtile, int r0, const float* s,
                                       const RowMult* rm) {
    const int lane = threadIdx.x & 31, sub = lane % LPR, rs = lane / LPR;
    float p[8][G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mx = -INFINITY;
#pragma unroll
      for (int r = 0; r < 8; ++r) mx = rm[r].valid ? fmaxf(mx, s[r * G + g]) : mx;
      const float mnew = fmaxf(m[g], mx);
      const float corr = mnew == -INFINITY ? 1.f : __expf(m[g] - mnew);
      float ls = 0.f, lns = 0.f;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        p[r][g] = rm[r].valid ? __expf(s[r * G + g] - mnew) : 0.f;
        ls += rm[r].wl * p[r][g];
        lns += fmaxf(-rm[r].wl, 0.f) * p[r][g];
      }
      l[g] = l[g] * corr + ls;
      ln[g] = ln[g] * corr + lns;
      m[g] = mnew;
#pragma unroll
      for (int e = 0; e < 4; ++e) o[g][e] *= corr;
    }
#pragma unroll
    for (int i = 0; i < NST; ++i) {
      const int r = RPW * i + rs;
      const float4 x = chunk<Lay>(vtile, r0 + r, sub);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float w = rm[r].wo * p[r][g];
        float2 a = __ffma2_rn(make_float2(w, w), make_float2(x.x, x.y), make_float2(o[g][0], o[g][1]));
        float2 b = __ffma2_rn(make_float2(w, w), make_float2(x.z, x.w), make_float2(o[g][2], o[g][3]));
        o[g][0] = a.x; o[g][1] = a.y; o[g][2] = b.x; o[g][3] = b.y;
      }
    }
    __syncwarp();
  }
  __device__ __forceinline__ void to_smem(float* comb) {
    const int lane = threadIdx.x & 31, sub = lane % LPR, rs = lane / LPR;
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int ofs = LPR; ofs < 32; ofs <<= 1) o[g][e] += __shfl_xor_sync(0xffffffffu, o[g][e], ofs);
    if (rs == 0) {   // rows of D + 4 floats: 8-byte aligned pairs
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float2* p = reinterpret_cast<float2*>(comb + g * (D + kPartStride) + kPartStride + 4 * sub);
        p[0] = make_float2(o[g][0], o[g][1]);
        p[1] = make_float2(o[g][2], o[g][3]);
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        comb[g * (D + kPartStride)] = m[g];
        comb[g * (D + kPartStride) + 1] = l[g];
        comb[g * (D + kPartStride) + 2] = ln[g];
      }
    }
  }
};

// Combine the per-warp parts comb [kConsumerWarps][G][D + 4] into one part
// [G][D + 4] at `part` (threads 0 .. kConsumers - 1).
template <int D, int G>
__device__ __forceinline__ void combine_warps(float* comb, float* part, int tid, float* pre = nullptr) {
  constexpr int RS = D + kPartStride;
  // each head's maximum, denominators and the warps' factors (kept in each
  // row's spare word 3) by one thread per head; `pre` (shared memory, the
  // same rows), when given, is one more part to fold in
  if (tid < G) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, comb[(w * G + tid) * RS]);
    if (pre) M = fmaxf(M, pre[tid * RS]);
    float L = 0.f, LN = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      float* row = comb + (w * G + tid) * RS;
      const float f = row[0] == -INFINITY ? 0.f : __expf(row[0] - M);
      row[3] = f;
      L += f * row[1];
      LN += f * row[2];
    }
    if (pre) {
      float* row = pre + tid * RS;
      const float f = row[0] == -INFINITY ? 0.f : __expf(row[0] - M);
      row[3] = f;
      L += f * row[1];
      LN += f * row[2];
    }
    part[tid * RS] = M;
    part[tid * RS + 1] = L;
    part[tid * RS + 2] = LN;
  }
  named_sync(1, kConsumers);   // the consumer threads (all of the gather's)
  for (int i = tid; i < G * D; i += kConsumers) {
    const int g = i / D, e = i - g * D;
    float O = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float* row = comb + (w * G + g) * RS;
      O += row[3] * row[kPartStride + e];
    }
    if (pre) O += pre[g * RS + 3] * pre[g * RS + kPartStride + e];
    part[g * RS + kPartStride + e] = O;
  }
}

// combine_warps by one warp: lane l takes columns 4 l .. 4 l + 3 of every
// head, each lane computing the heads' maxima and the warps' factors itself
// (broadcast reads).
template <int D, int G>
__device__ __forceinline__ void combine_warps_1w(const float* comb, float* part, int lane) {
  static_assert(D <= 128, "4 columns per lane");
  constexpr int RS = D + kPartStride;
  const int c = 4 * lane;
#pragma unroll 1
  for (int g = 0; g < G; ++g) {
    float mw[kConsumerWarps];
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      mw[w] = comb[(w * G + g) * RS];
      M = fmaxf(M, mw[w]);
    }
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.f, LN = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float* row = comb + (w * G + g) * RS;
      const float f = mw[w] == -INFINITY ? 0.f : __expf(mw[w] - M);
      L = fmaf(f, row[1], L);
      LN = fmaf(f, row[2], LN);
      if (c < D) {
        const float4 x = *reinterpret_cast<const float4*>(row + kPartStride + c);
        o.x = fmaf(f, x.x, o.x);
        o.y = fmaf(f, x.y, o.y);
        o.z = fmaf(f, x.z, o.z);
        o.w = fmaf(f, x.w, o.w);
      }
    }
    if (c < D) *reinterpret_cast<float4*>(part + g * RS + kPartStride + c) = o;
    if (lane == 0) {
      part[g * RS] = M;
      part[g * RS + 1] = L;
      part[g * RS + 2] = LN;
    }
  }
}

// ------------------------------------------------------------- K0 steady
struct SteadyArgs {
  const int32_t* invperm;
  const int32_t* labels;
  const int32_t* offsets;
  int n_sink, window, cap;
  int32_t* info;     // [U][kInfoInts]
  int32_t* st_slot;  // [U][cap] steady slots, ascending
  int2* pc;          // [U][cap] (slot, cluster) of steady tokens of candidate clusters
  int2* nonc;        // [U][cap] (cluster, count) of clusters without a non-steady token
  int32_t* hist;     // [U][kHistBins] the scan's first-digit histograms, cleared here
  int32_t* cnt1;     // [U] the scan's arrivals, cleared here
  int32_t* cnt2;     // [U] the gather's arrivals, cleared here
};

__global__ void __launch_bounds__(256)
wave_steady_kernel(const Geo geo, const SteadyArgs a, uint32_t* status) {
  extern __shared__ __align__(16) unsigned long long srt[];   // [npow] sort keys
  __shared__ int s_runs, s_nonc, s_pc;
  pdl_launch_dependents();
  const int u = blockIdx.x, b = u / geo.hkv, h = u - b * geo.hkv;
  const int Tb = geo.T(b), NC = geo.NC(b);
  const int ns = min(a.n_sink, Tb);
  const int wstart = max(Tb - a.window, ns);
  const int n_st = ns + (Tb - wstart);
  const int tid = threadIdx.x, lane = tid & 31;
  int32_t* I = a.info + (int64_t)u * kInfoInts;
  // this call's counters start from zero whatever an earlier call left (the
  // scan and the gather touch them only after this kernel has finished)
  for (int i = tid; i < kHistBins / 4; i += blockDim.x)
    reinterpret_cast<int4*>(a.hist + (int64_t)u * kHistBins)[i] = make_int4(0, 0, 0, 0);
  if (tid == 0) { a.cnt1[u] = 0; a.cnt2[u] = 0; }
  if (n_st >= Tb) {   // all steady: attended densely, nothing retrieved or estimated
    if (tid < kInfoInts) {
      int v = 0;
      if (tid == kSteady) v = Tb;
      if (tid == kDense || tid == kNoEstimate) v = 1;
      if (tid == kThrKey || tid == kThrIdx) v = -1;
      I[tid] = v;
    }
    return;
  }
  int npow = 1;
  while (npow < n_st) npow <<= 1;
  const int32_t* inv = a.invperm + geo.tok_row(b, h);
  const int32_t* lab = a.labels + geo.tok_row(b, h);
  for (int i = tid; i < npow; i += blockDim.x) {
    unsigned long long k = ~0ull;
    if (i < n_st) {
      const int pos = i < ns ? i : wstart + (i - ns);
      int s = __ldg(inv + pos), c = __ldg(lab + pos);
      if (s < 0 || s >= Tb) { flag_error(status, WI_DEV_BAD_SLOT); s = Tb; }
      if (c < 0 || c >= NC) { flag_error(status, WI_DEV_BAD_CLUSTER); c = 0; }
      k = ((unsigned long long)(uint32_t)s << 32) | (uint32_t)c;
    }
    srt[i] = k;
  }
  __syncthreads();
  if (n_st <= (int)blockDim.x) {
    // short lists (the usual 68): each key's rank among all, one step
    const unsigned long long mine = tid < n_st ? srt[tid] : 0ull;
    int rank = 0;
    if (tid < n_st)
      for (int j = 0; j < n_st; ++j) {
        const unsigned long long x = srt[j];
        rank += x < mine || (x == mine && j < tid);   // equal keys only on a bad slot
      }
    __syncthreads();
    if (tid < n_st) srt[rank] = mine;
    __syncthreads();
  } else {
  // bitonic sort by slot (clusters are slot ranges, so this groups them too)
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
  for (int i = tid; i < n_st; i += blockDim.x) slots[i] = (int32_t)(srt[i] >> 32);
  // runs of one cluster (clusters are slot ranges, so a cluster's steady
  // tokens are consecutive): a run's cluster is a candidate iff it keeps a
  // non-steady member.  Each run's head marks its members (bit 31 of the
  // key's cluster word, free since cluster ids are below 2^31).
  const int32_t* off = a.offsets + geo.off_row(b, h);
  auto cl_of = [&](int i) { return (int)(srt[i] & 0x7fffffffu); };
  for (int i = tid; i < n_st; i += blockDim.x) {
    const int c = cl_of(i);
    if (i == 0 || cl_of(i - 1) != c) {
      int e = i + 1;
      while (e < n_st && cl_of(e) == c) ++e;
      const int full = __ldg(off + c + 1) - __ldg(off + c);
      if (full - (e - i) > 0)
        for (int m = i; m < e; ++m) srt[m] |= 0x80000000ull;
    }
  }
  __syncthreads();
  // in order (warp 0): the non-candidates (cluster, count) and the steady
  // tokens of candidate clusters (slot, cluster), which the gather takes out
  // of the estimate unless their cluster is retrieved
  int2* pc = a.pc + (int64_t)u * a.cap;
  int2* nonc = a.nonc + (int64_t)u * a.cap;
  if (tid < 32) {
    const unsigned lt = (1u << lane) - 1u;
    int n_runs = 0, n_nc = 0, n_pc = 0;
    for (int base = 0; base < n_st; base += 32) {
      const int i = base + lane;
      const bool in = i < n_st;
      const int c = in ? cl_of(i) : -1;
      const bool head = in && (i == 0 || cl_of(i - 1) != c);
      const bool cand = in && (srt[i] & 0x80000000ull) != 0ull;
      const unsigned bh = __ballot_sync(0xffffffffu, head);
      const unsigned bn = __ballot_sync(0xffffffffu, head && !cand);
      const unsigned bp = __ballot_sync(0xffffffffu, cand);
      if (head && !cand)
        nonc[n_nc + __popc(bn & lt)] = make_int2(c, __ldg(off + c + 1) - __ldg(off + c));
      if (cand) pc[n_pc + __popc(bp & lt)] = make_int2((int)(srt[i] >> 32), c);
      n_runs += __popc(bh);
      n_nc += __popc(bn);
      n_pc += __popc(bp);
    }
    if (lane == 0) { s_runs = n_runs; s_nonc = n_nc; s_pc = n_pc; }
  }
  __syncthreads();
  if (tid == 0) {
    I[kSteady] = n_st;
    I[kAffected] = s_runs;
    I[kDense] = 0;
    I[kPartRows] = s_pc;
    I[kNonCand] = s_nonc;
  }
}

// --------------------------------------------------------------- K1 scan
struct ScanArgs {
  const void* q;
  int Hq;
  uint2* rec;            // [ncl] {selection key (0: not a candidate), first slot}
  int32_t* hist;         // [U][kHistBins] first-digit histogram (zero between calls)
  int32_t* cnt1;         // [U] arrivals (zero between calls)
  float* est;            // [U][p1max][G][D + 4] estimation parts
  int p1max;
  float* scores_out;     // optional [ncl][G]
  float scale;
  int exact_only;
  // tail
  int32_t* info;
  const int2* nonc;
  int32_t* sel;          // [ncl] retrieved ids, ascending (unit rows as the centroids)
  int4* selinfo;         // [ncl] retrieved {id, first slot, count, first token row}
  int32_t* blkf;         // [ntok] per block of kGatherRows token rows: its first retrieved
                         // cluster (unit rows as perm)
  int cap;
  int topk_clusters;
  double topk_fraction;
  int mode;
  uint32_t seed;
  int slots;
  int mid_ok;      // a second part buffer fits: a CTA whose chunks span units hands its
                   // first unit's arrival to the producer warp
};

// A chunk's offsets arrive as one 1-D tensor box of kOffBox int32 that starts
// at the entry of the chunk's first cluster rounded down to a multiple of 4
// (16 bytes): the chunk's kTileRows + 1 entries sit at box index
// (first entry) % 4.
constexpr int kOffBox = 72;
constexpr int kOffArea = 512;   // bytes of a slot's side area before its queries

// Position of a scan chunk: its unit and first cluster.  Consecutive chunks
// of one unit advance by kTileRows clusters; the kernel parameters are read
// again only when a chunk starts another unit.
struct ChunkPos {
  int k;            // chunk index
  int b, h, u;
  int c0, nrows;    // first cluster in the unit, rows in the chunk
  int NC;           // clusters of the unit
  int kend;         // one past the unit's last chunk
  int64_t row0;     // centroid row of the unit's cluster 0
  int64_t orow;     // offsets entry of the unit's cluster 0
};
__device__ __forceinline__ void chunk_seek(ChunkPos& p, const Geo& geo, const ChunkMap& cm, int k) {
  p.k = k;
  p.b = cm.seq_of(k);
  const int per = cm.per_unit(p.b);
  const int rel = k - cm.ch_base[p.b];
  p.h = rel / per;
  p.c0 = (rel - p.h * per) * kTileRows;
  p.u = p.b * geo.hkv + p.h;
  p.NC = geo.NC(p.b);
  p.kend = cm.ch_base[p.b] + (p.h + 1) * per;
  p.row0 = geo.cl_row(p.b, p.h);
  p.orow = geo.off_row(p.b, p.h);
  p.nrows = min(kTileRows, p.NC - p.c0);
}
__device__ __forceinline__ void chunk_next(ChunkPos& p, const Geo& geo, const ChunkMap& cm) {
  if (p.k + 1 < p.kend) {
    ++p.k;
    p.c0 += kTileRows;
    p.nrows = min(kTileRows, p.NC - p.c0);
  } else {
    chunk_seek(p, geo, cm, p.k + 1);
  }
}

constexpr int kTailSteps = 32;                       // records per consumer lane and round
constexpr int kTailRound = kConsumers * kTailSteps;  // 8192 records per round
constexpr int kTailDraws = 256;                      // threshold bins ranked member by member
static_assert(kTailDraws % 16 == 0 && kTailDraws <= kConsumers, "the rank rounds read 16 values; a thread per value");
// a round of records (and the next one) staged in shared memory, one pad
// record per 32 (the ring, once the chunks are done)
constexpr size_t kTailStage = ((size_t)(kTailRound + kTailRound / 32 + 2) * 8 + 1023) / 1024 * 1024;
// the ring keeps the slots' side areas (tensor-copy destinations) 128-byte
// aligned and the tiles 1024-byte aligned
static_assert(kTailStage % 1024 == 0, "record stage must keep the ring 1024-byte aligned");

// Shared memory of a scan CTA (bytes, after 1024-byte alignment): the ring of
// tiles (also the tail's record stage), each slot's side area (offsets box,
// the unit's queries), and a union of the per-warp softmax parts and the
// tail's work areas.
template <typename T, int D, int G>
struct ScanSmem {
  using TS = TileShape<T, D>;
  static constexpr size_t kQBytes = (size_t)G * D * sizeof(T);
  static constexpr size_t kSide = kOffArea + (kQBytes + 127) / 128 * 128;
  static_assert(kSide % 128 == 0 && TS::kBytes % 1024 == 0, "slot areas keep tensor-copy alignment");
  static constexpr size_t kComb = (size_t)kConsumerWarps * G * (D + kPartStride) * 4;
  // tail: histogram, threshold-bin members, their draws, scan scratch and
  // control words
  static constexpr size_t kTailHist = 0;
  static constexpr size_t kTailCandOff = kTailHist + (size_t)kHistBins * 4;
  static constexpr size_t kTailDrawOff = kTailCandOff + (size_t)kTailCand * 8;
  static constexpr size_t kTailShOff = kTailDrawOff + (size_t)kTailDraws * 8;
  static constexpr size_t kTail = kTailShOff + 512;
  static constexpr size_t kHist16 = (size_t)kHistBins / 2 * 4;
  static constexpr size_t kRows = (size_t)kConsumerWarps * 8 * sizeof(RowMult);
  static constexpr size_t kSc = (size_t)kConsumerWarps * 8 * G * 4;
  __host__ __device__ static size_t tile_bytes(int exact_only) { return (size_t)TS::kBytes * (exact_only ? 1 : 2); }
  __host__ __device__ static size_t ring_bytes(int slots, int exact_only) {
    const size_t r = slots * tile_bytes(exact_only);
    return r > kTailStage ? r : kTailStage;
  }
  __host__ __device__ static size_t side_bytes(int slots) { return slots * kSide; }
  // (mid: room for a second unit's warp parts, see ScanArgs::mid_ok)
  __host__ __device__ static size_t total(int slots, int exact_only, int mid = 0) {
    return 1024 + ring_bytes(slots, exact_only) + side_bytes(slots) + kTail + (mid ? 2 : 1) * kComb +
           kHist16 + kRows + kSc;
  }
};

// SplitMix64 (Steele, Lea and Flood 2014): the draw of the sampled selection.
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Block-wide helpers over the kConsumers consumer threads (named barrier 1).
__device__ __forceinline__ void csync() { named_sync(1, kConsumers); }

// inclusive scan of x over the consumers; *total the sum.  sh: 32 ints.
__device__ __forceinline__ int cscan(int x, int* sh, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[w] = x;
  csync();
  if (w == 0) {
    int s = lane < kConsumerWarps ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kConsumerWarps) sh[lane] = s;
  }
  csync();
  const int r = x + (w > 0 ? sh[w - 1] : 0);
  *total = sh[kConsumerWarps - 1];
  csync();
  return r;
}

// Exclusive prefix over the consumer warps of a warp-uniform pair of values;
// *total the sums.  sh: 16 ints.
__device__ __forceinline__ int2 wscan2(int2 v, int* sh, int2* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (lane == 0) { sh[w] = v.x; sh[8 + w] = v.y; }
  csync();
  int2 base = make_int2(0, 0), t = make_int2(0, 0);
#pragma unroll
  for (int i = 0; i < kConsumerWarps; ++i) {
    const int a = sh[i], c = sh[8 + i];
    if (i < w) { base.x += a; base.y += c; }
    t.x += a;
    t.y += c;
  }
  csync();
  *total = t;
  return base;
}

// Whether cluster c (selection key `key`, 0 for a non-candidate) is
// retrieved, given the unit's threshold: exact mode, key > kstar or key ==
// kstar and c <= thr; sampled mode, a key above the threshold bin, or in it
// with (SplitMix64(seed 2^32 + c), c) <= (hstar, thr).
struct Threshold {
  uint32_t kstar;
  int thr;
  int sampled, bin1;
  uint64_t hstar;
  uint32_t seed;
  __device__ __forceinline__ bool picked(uint32_t key, uint32_t c) const {
    if (key == 0u) return false;
    if (sampled) {
      const int bn = (int)(key >> kHistShift);
      if (bn != bin1) return bn > bin1;
      const uint64_t d = splitmix64(((uint64_t)seed << 32) | (uint64_t)c);
      return d < hstar || (d == hstar && (int)c <= thr);
    }
    return key > kstar || (key == kstar && (int)c <= thr);
  }
};

// Bin of a histogram (bins scanned downwards) that holds the krem-th largest
// element; *above: the count in the bins above it.  nb bins (<= 2048), each
// consumer owns nb / kConsumers consecutive bins from the top.
__device__ __forceinline__ int select_bin(const int* hist, int nb, int krem, int* above, int* sh,
                                          int* s_ctl) {
  const int tid = threadIdx.x;
  const int per = nb / kConsumers;
  int c[8], s = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = i < per ? hist[nb - 1 - per * tid - i] : 0;
    s += c[i];
  }
  int tot;
  const int incl = cscan(s, sh, &tot);
  if (tid == 0) { s_ctl[0] = -1; s_ctl[1] = 0; }
  csync();
  int acc = incl - s;
  if (acc < krem && incl >= krem) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i < per && acc + c[i] >= krem) { s_ctl[0] = nb - 1 - per * tid - i; s_ctl[1] = acc; break; }
      acc += c[i];
    }
  }
  csync();
  *above = s_ctl[1];
  const int r = s_ctl[0];
  csync();
  return r;
}

// The unit's geometry, passed to the tail as scalars (the 2 KB Geo would be
// copied to local memory for a call).
struct TailUnit {
  int u, NC, Tb;
  int64_t row0, trow;
};

// Records of a round as staged in shared memory: record i (round-relative)
// at i + i / 32, so consumer thread t reads its 32 consecutive records
// 32 t .. 32 t + 31 without bank conflicts.
__device__ __forceinline__ int rpad(int i) { return i + (i >> 5); }

// Stage round r of a unit's records in shared memory (record r kTailRound +
// i; past the unit: key 0, first slot T_b; and the record after the round,
// for the last count).  Loads of 8 records per thread are in flight at once.
__device__ __forceinline__ void stage_round(const uint2* rec, int NC, int Tb, int r, uint2* stage) {
  const int tid = threadIdx.x;
  const int c0 = r * kTailRound;
  // (every thread's loads in flight together: one round trip)
  uint2 v[kTailSteps];
#pragma unroll
  for (int q = 0; q < kTailSteps; ++q) {
    const int c = c0 + tid + q * kConsumers;
    v[q] = c < NC ? __ldcg(rec + c) : make_uint2(0u, (uint32_t)Tb);
  }
  csync();   // the previous round's readers are done
#pragma unroll
  for (int q = 0; q < kTailSteps; ++q) stage[rpad(tid + q * kConsumers)] = v[q];
  if (tid == 0)
    stage[rpad(kTailRound)] =
        make_uint2(0u, c0 + kTailRound < NC ? __ldcg(&rec[c0 + kTailRound].y) : (uint32_t)Tb);
  csync();
}

// Exclusive prefix over the consumer threads of a pair of values (thread
// order); *total the sums.  sh: 16 ints.
__device__ __forceinline__ int2 cscan2_excl(int2 v, int* sh, int2* total) {
  const int lane = threadIdx.x & 31;
  int2 x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ya = __shfl_up_sync(0xffffffffu, x.x, o);
    const int yb = __shfl_up_sync(0xffffffffu, x.y, o);
    if (lane >= o) { x.x += ya; x.y += yb; }
  }
  const int2 wtot = make_int2(__shfl_sync(0xffffffffu, x.x, 31), __shfl_sync(0xffffffffu, x.y, 31));
  const int2 wb = wscan2(wtot, sh, total);
  return make_int2(wb.x + x.x - v.x, wb.y + x.y - v.y);
}

// The tail of unit u (by the last scan CTA to finish it): the exact top-k
// threshold (kstar, thr) -- cluster c is retrieved iff its key > kstar, or
// key == kstar and c <= thr (lower id first on equal keys) -- or, in the
// sampled mode, every key above the threshold bin plus the threshold bin's
// members with the smallest (SplitMix64(seed 2^32 + c), c) draws; then the
// retrieved ids, their token slots and the clusters whose estimate the
// gather takes back out.
//
// A round of kTailRound records at a time is staged in shared memory, and
// consumer thread t walks records 32 t .. 32 t + 31, so thread order is id
// order: every pass is one short loop per thread and one block-wide prefix
// sum.  The tail runs once per unit on one CTA: its cost is its chains of
// dependent shuffles and shared loads and the fetch of its instructions, so
// its loops stay rolled and its code small.
__device__ __forceinline__ void scan_tail(const TailUnit tu, const ScanArgs& A, unsigned char* sh,
                                          unsigned char* stage_bytes, size_t cand_off,
                                          size_t draw_off, size_t sh_off, uint32_t* status) {
  const int u = tu.u, NC = tu.NC, Tb = tu.Tb;
  const int tid = threadIdx.x;
  int* s_hist = reinterpret_cast<int*>(sh);                                         // [2048]
  unsigned long long* s_cand = reinterpret_cast<unsigned long long*>(sh + cand_off); // [kTailCand]
  unsigned long long* s_draw = reinterpret_cast<unsigned long long*>(sh + draw_off); // [kTailDraws]
  int* s_sh = reinterpret_cast<int*>(sh + sh_off);                                   // [64]
  int* s_ctl = s_sh + 64;                                                             // [16]
  uint2* stage = reinterpret_cast<uint2*>(stage_bytes);
  uint2* rec = A.rec + tu.row0;
  int32_t* I = A.info + (int64_t)u * kInfoInts;
  int32_t* hg = A.hist + (int64_t)u * kHistBins;
  const int2* nonc = A.nonc + (int64_t)u * A.cap;
  const int n_rounds = (NC + kTailRound - 1) / kTailRound;
  auto draw = [&](uint32_t c) { return splitmix64(((uint64_t)A.seed << 32) | (uint64_t)c); };
  int loaded = -1;
  auto get_round = [&](int r) {
    if (loaded != r) {
      stage_round(rec, NC, Tb, r, stage);
      loaded = r;
    }
  };
  // this thread's record j of the staged round
  auto key_of = [&](int j) { return stage[rpad(kTailSteps * tid + j)].x; };

  auto id_of = [&](int r, int j) { return (uint32_t)(r * kTailRound + kTailSteps * tid + j); };

  pdl_wait();   // the steady kernel's lists
  // ---- the histogram, the non-candidate count and round 0 in one round trip
  const int4 h0 = __ldcg(reinterpret_cast<const int4*>(hg) + tid);
  const int4 h1 = __ldcg(reinterpret_cast<const int4*>(hg) + kConsumers + tid);
  const int n_nonc = __ldcg(I + kNonCand);
  const int nc_first = tid < A.cap ? __ldcg(&nonc[tid].x) : -1;   // (read before the count is known)
  get_round(0);
  reinterpret_cast<int4*>(s_hist)[tid] = h0;
  reinterpret_cast<int4*>(s_hist)[kConsumers + tid] = h1;
  csync();
  // the clusters left without a non-steady token are not candidates: their
  // keys leave the histogram and become 0 in the records (and in the staged
  // round 0)
  if (n_nonc > 0) {
    for (int j = tid; j < n_nonc; j += kConsumers) {
      const int c = j == tid ? nc_first : __ldcg(&nonc[j].x);
      if (c >= 0 && c < NC) {
        const uint32_t key = c < kTailRound ? stage[rpad(c)].x : __ldcg(&rec[c].x);
        if (key) {
          atomicSub(&s_hist[key >> kHistShift], 1);
          if (c < kTailRound) stage[rpad(c)].x = 0u;
          __stcg(&rec[c].x, 0u);
        }
      }
    }
    csync();   // the cleared keys and counts are visible to every thread
  }
  // ---- candidates: the histogram's total (the steady kernel cleared it, and
  // the threshold bin's member count is checked against it below), and a
  // prefix over its bins from the top down (thread t: bins 2047 - 8 t ..
  // 2040 - 8 t), from which the threshold bin is read once k is known
  constexpr int kBpt = kHistBins / kConsumers;
  int hc[kBpt], hs = 0;
#pragma unroll
  for (int i = 0; i < kBpt; ++i) {
    hc[i] = s_hist[kHistBins - 1 - kBpt * tid - i];
    hs += hc[i];
  }
  int n_cand;
  const int h_incl = cscan(hs, s_sh, &n_cand);
  const int k_req = A.topk_clusters >= 0 ? A.topk_clusters
                                         : (int)ceil(A.topk_fraction * (double)NC);
  const int k = min(max(k_req, 0), n_cand);
  uint32_t kstar = 0xFFFFFFFFu;   // nothing retrieved
  int thr = -1;
  int bin1 = -1;
  uint64_t hstar = 0;
  // a single round: this thread's records above the threshold bin and in it
  // (masks), and the tokens above it, from the member pass
  uint32_t am = 0u, bm1 = 0u;
  int atok = 0;

  // the kth (1-based) record in id order that satisfies pred(key, id)
  auto ordered_pick = [&](auto&& pred, int kth) -> int {
    if (tid == 0) s_ctl[2] = -1;
    int run = 0;
    for (int r = 0; r < n_rounds; ++r) {
      get_round(r);
      uint32_t m = 0u;
#pragma unroll 4
      for (int j = 0; j < kTailSteps; ++j) m |= pred(key_of(j), id_of(r, j)) ? 1u << j : 0u;
      int2 t2;
      const int before = run + cscan2_excl(make_int2(__popc(m), 0), s_sh, &t2).x;
      if (before < kth && before + __popc(m) >= kth) {
        for (int n = kth - before; n > 1; --n) m &= m - 1u;   // drop the first n - 1 set bits
        s_ctl[2] = (int)id_of(r, __ffs(m) - 1);
      }
      run += t2.x;
    }
    csync();
    const int id = s_ctl[2];
    csync();
    return id;
  };

  if (k == n_cand && k > 0) {
    kstar = 1u;
    thr = INT_MAX;
  } else if (k > 0) {
    // the bin holding the k-th largest key: exactly one thread's bins do
    {
      int acc = h_incl - hs;
      if (acc < k && h_incl >= k) {
#pragma unroll
        for (int i = 0; i < kBpt; ++i) {
          if (acc + hc[i] >= k) {
            s_ctl[0] = kHistBins - 1 - kBpt * tid - i;
            s_ctl[1] = acc;
            break;
          }
          acc += hc[i];
        }
      }
    }
    csync();
    bin1 = s_ctl[0];
    const int above = s_ctl[1];
    int krem = k - above;
    const int nb1 = s_hist[bin1];
    csync();   // read by all before the radix passes reuse the histogram
    // the threshold bin's members (key, id) when they fit; otherwise each
    // refinement pass reads the records again
    const bool fits = nb1 <= kTailCand;
    if (fits || n_rounds == 1) {
      int run = 0;
      const int rb = kTailSteps * tid;
      for (int r = 0; r < n_rounds; ++r) {
        get_round(r);
        uint32_t m = 0u;
        uint2 x = stage[rpad(rb)];   // each record read once: the next one's first slot ends it
#pragma unroll 4
        for (int j = 0; j < kTailSteps; ++j) {
          const uint2 xn = stage[rpad(rb + j + 1)];
          const int bn = (int)(x.x >> kHistShift);
          const bool in = x.x != 0u && bn == bin1, up = x.x != 0u && bn > bin1;
          m |= (uint32_t)in << j;
          am |= (uint32_t)up << j;
          atok += up ? (int)(xn.y - x.y) : 0;
          x = xn;
        }
        bm1 = m;
        int2 t2;
        int pos = run + cscan2_excl(make_int2(__popc(m), 0), s_sh, &t2).x;
        if (fits) {
          while (m) {
            const int j = __ffs(m) - 1;
            m &= m - 1u;
            const uint2 x = stage[rpad(rb + j)];
            if (pos < kTailCand) s_cand[pos] = ((unsigned long long)x.x << 32) | id_of(r, j);
            ++pos;
          }
        }
        run += t2.x;
      }
      // the members counted must be the histogram's (its bins were cleared by
      // the steady kernel; a mismatch says the workspace was disturbed)
      if (tid == 0 && run != nb1) flag_error(status, WI_DEV_BAD_HIST);
      csync();
    }
    auto cand_key = [&](int i) { return (uint32_t)(s_cand[i] >> 32); };
    auto cand_id = [&](int i) { return (uint32_t)s_cand[i]; };
    // a radix pass over the members (or, when they did not fit, over the
    // records of the threshold bin): count(x) takes each one's value
    auto over_members = [&](auto&& count) {
      if (fits) {
        for (int i = tid; i < nb1; i += kConsumers) count(cand_key(i), cand_id(i));
      } else {
        for (int r = 0; r < n_rounds; ++r) {
          get_round(r);
#pragma unroll 4
          for (int j = 0; j < kTailSteps; ++j)
            if (key_of(j) != 0u && (int)(key_of(j) >> kHistShift) == bin1) count(key_of(j), id_of(r, j));
        }
      }
    };
    if (A.mode == 1) {
      // sampled: the krem members of the threshold bin with the smallest
      // (draw, id)
      if (fits && nb1 <= kTailDraws) {
        if (tid < nb1) s_draw[tid] = draw(cand_id(tid));
        if (tid == 0) s_ctl[2] = -1;
        csync();
        if (tid < nb1) {
          const uint64_t dm = s_draw[tid];
          const uint32_t im = cand_id(tid);
          int rank = 0;
#pragma unroll 8
          for (int j = 0; j < nb1; ++j) {
            const uint64_t dj = s_draw[j];
            rank += dj < dm || (dj == dm && cand_id(j) < im);
          }
          if (rank == krem - 1) {
            s_ctl[2] = (int)im;
            s_ctl[3] = (int)(uint32_t)(dm >> 32);
            s_ctl[4] = (int)(uint32_t)dm;
          }
        }
        csync();
        thr = s_ctl[2];
        hstar = ((uint64_t)(uint32_t)s_ctl[3] << 32) | (uint32_t)s_ctl[4];
        csync();
      } else {
        // an exact radix select of the 64-bit draws (11/11/11/11/10/10-bit
        // digits, smallest first), then the ties in id order
        uint64_t prefix = 0, pmask = 0;
        int kr = krem;
#pragma unroll 1
        for (int pass = 0; pass < 6; ++pass) {
          const int sh_ = pass < 4 ? 53 - 11 * pass : (pass == 4 ? 10 : 0);
          const int nb = pass < 4 ? 2048 : 1024;
          for (int i = tid; i < kHistBins; i += kConsumers) s_hist[i] = 0;
          csync();
          over_members([&](uint32_t, uint32_t id) {
            const uint64_t d = draw(id);
            if ((d & pmask) == prefix)
              atomicAdd(&s_hist[(nb - 1) - (int)((d >> sh_) & (uint64_t)(nb - 1))], 1);
          });
          csync();
          // the histogram is filled reversed, so select_bin's largest bin is
          // the smallest digit
          int ab;
          const int dd = (nb - 1) - select_bin(s_hist, nb, kr, &ab, s_sh, s_ctl);
          kr -= ab;
          prefix |= (uint64_t)dd << sh_;
          pmask |= (uint64_t)(nb - 1) << sh_;
        }
        hstar = prefix;
        if (fits) {
          // the kr-th smallest id among the members drawing hstar
          if (tid == 0) s_ctl[2] = -1;
          csync();
          for (int i = tid; i < nb1; i += kConsumers) {
            const uint32_t ci = cand_id(i);
            if (draw(ci) != hstar) continue;
            int rank = 0;
            for (int j = 0; j < nb1; ++j) {
              const uint32_t cj = cand_id(j);
              rank += cj < ci && draw(cj) == hstar;
            }
            if (rank == kr - 1) s_ctl[2] = (int)ci;
          }
          csync();
          thr = s_ctl[2];
          csync();
        } else {
          thr = ordered_pick([&](uint32_t key, uint32_t id) {
            return key != 0u && (int)(key >> kHistShift) == bin1 && draw(id) == hstar;
          }, kr);
        }
      }
    } else {
      // exact: the krem-th largest (key, -id) of the threshold bin
      if (fits && nb1 <= kTailDraws) {
        // (key, -id) as one 64-bit value (key high, the id's complement low):
        // a member's rank is the count of larger values, one comparison each
        // Padded with zeros (below every member, whose key is nonzero) to a
        // multiple of 16, read 16 values a round with all loads in flight.
        unsigned long long* s_kv = s_draw;
        const int nbp = (nb1 + 15) & ~15;   // <= kTailDraws, a multiple of 16
        if (tid < nb1) {
          const unsigned long long cm_ = s_cand[tid];
          s_kv[tid] = (cm_ & 0xFFFFFFFF00000000ull) | (uint32_t)~(uint32_t)cm_;
        } else if (tid < nbp) {
          s_kv[tid] = 0ull;
        }
        if (tid == 0) s_ctl[2] = -1;
        csync();
        if (tid < nb1) {
          const unsigned long long me = s_kv[tid];
          int rank = 0;
#pragma unroll 1
          for (int j = 0; j < nbp; j += 16) {
            ulonglong2 v[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) v[t] = *reinterpret_cast<const ulonglong2*>(s_kv + j + 2 * t);
#pragma unroll
            for (int t = 0; t < 8; ++t) rank += (v[t].x > me) + (v[t].y > me);
          }
          if (rank == krem - 1) {
            s_ctl[2] = (int)~(uint32_t)me;
            s_ctl[3] = (int)(uint32_t)(me >> 32);
          }
        }
        csync();
        thr = s_ctl[2];
        kstar = (uint32_t)s_ctl[3];
        csync();
      } else {
        // refine by the key's bits 20..10, then 9..0, then the ties in id order
        uint32_t prefix = (uint32_t)bin1 << kHistShift, pmask = 0xFFE00000u;
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
          const int sh_ = pass == 0 ? 10 : 0;
          const int nb = pass == 0 ? 2048 : 1024;
          for (int i = tid; i < kHistBins; i += kConsumers) s_hist[i] = 0;
          csync();
          over_members([&](uint32_t key, uint32_t) {
            if ((key & pmask) == prefix) atomicAdd(&s_hist[(key >> sh_) & (nb - 1)], 1);
          });
          csync();
          int ab;
          const int dd = select_bin(s_hist, nb, krem, &ab, s_sh, s_ctl);
          krem -= ab;
          prefix |= (uint32_t)dd << sh_;
          pmask |= (uint32_t)(nb - 1) << sh_;
        }
        kstar = prefix;
        if (fits) {
          if (tid == 0) s_ctl[2] = -1;
          csync();
          for (int i = tid; i < nb1; i += kConsumers) {
            if (cand_key(i) != kstar) continue;
            const uint32_t ci = cand_id(i);
            int rank = 0;
            for (int j = 0; j < nb1; ++j) rank += cand_key(j) == kstar && cand_id(j) < ci;
            if (rank == krem - 1) s_ctl[2] = (int)ci;
          }
          csync();
          thr = s_ctl[2];
          csync();
        } else {
          thr = ordered_pick([&](uint32_t key, uint32_t) { return key == kstar; }, krem);
        }
      }
    }
  }
  // ---- emit, in id order: the retrieved clusters {id, first slot, count,
  // first token row} (the gather's token rows are theirs, concatenated; the
  // clusters taken back out of the estimate are they and the
  // non-candidates), and for every block of kGatherRows token rows the first
  // retrieved cluster that overlaps it
  const bool sampled = A.mode == 1 && k > 0 && k < n_cand;
  const Threshold th{kstar, thr, sampled ? 1 : 0, bin1, hstar, A.seed};
  const bool no_est = A.exact_only || k == n_cand;
  int32_t* sel = A.sel + tu.row0;
  int4* selinfo = A.selinfo + tu.row0;
  int32_t* blkf = A.blkf + tu.trow;
  int n_sel = 0, n_tok = 0;
  if (k > 0) {
    for (int r = 0; r < n_rounds; ++r) {
      get_round(r);
      // (the mode test out of the loop; each record's count without a
      // branch, from its first slot and the next record's)
      uint32_t pm = 0u;
      int pt = 0;
      const int rb = kTailSteps * tid;
      if (n_rounds == 1 && bin1 >= 0) {
        // a single round: the records above the threshold bin, and the bin's
        // members that the threshold keeps (masks from the member pass)
        pm = am;
        pt = atok;
        uint32_t mm = bm1;
        while (mm) {
          const int j = __ffs(mm) - 1;
          mm &= mm - 1u;
          const uint2 x = stage[rpad(rb + j)];
          if (th.picked(x.x, id_of(r, j))) {
            pm |= 1u << j;
            pt += (int)(stage[rpad(rb + j + 1)].y - x.y);
          }
        }
      } else if (!th.sampled) {
#pragma unroll 4
        for (int j = 0; j < kTailSteps; ++j) {
          const uint2 x = stage[rpad(rb + j)];
          const uint32_t nx = stage[rpad(rb + j + 1)].y;
          const bool p = x.x != 0u && (x.x > th.kstar || (x.x == th.kstar && (int)id_of(r, j) <= th.thr));
          pm |= (uint32_t)p << j;
          pt += p ? (int)(nx - x.y) : 0;
        }
      } else {
#pragma unroll 4
        for (int j = 0; j < kTailSteps; ++j) {
          const uint2 x = stage[rpad(rb + j)];
          const uint32_t nx = stage[rpad(rb + j + 1)].y;
          const bool p = th.picked(x.x, id_of(r, j));
          pm |= (uint32_t)p << j;
          pt += p ? (int)(nx - x.y) : 0;
        }
      }
      int2 tot;
      const int2 ex = cscan2_excl(make_int2(__popc(pm), pt), s_sh, &tot);
      int e = n_sel + ex.x, tpos = n_tok + ex.y;
      while (pm) {
        const int j = __ffs(pm) - 1;
        pm &= pm - 1u;
        const uint2 x = stage[rpad(rb + j)];
        const int cnt = (int)(stage[rpad(rb + j + 1)].y - x.y);
        const int id = (int)id_of(r, j);
        sel[e] = id;
        selinfo[e] = make_int4(id, (int)x.y, cnt, tpos);
        for (int bk = (tpos + kGatherRows - 1) / kGatherRows; bk * kGatherRows < tpos + cnt; ++bk)
          blkf[bk] = e;
        ++e;
        tpos += cnt;
      }
      n_sel += tot.x;
      n_tok += tot.y;
    }
  }
  const int n_full = no_est ? 0 : n_sel + n_nonc;
  if (tid == 0) {
    I[kSelCount] = n_sel;
    I[kThrKey] = (int32_t)kstar;
    I[kThrIdx] = thr;
    I[kSelTokens] = n_tok;
    I[kCandidates] = n_cand;
    I[kFullRows] = n_full;
    I[kNoEstimate] = no_est ? 1 : 0;
    I[kMode] = sampled ? 1 : 0;
    I[kSampBin] = bin1;
    I[kSampHash] = (int32_t)(uint32_t)(hstar >> 32);
    I[kSampHashLo] = (int32_t)(uint32_t)hstar;
    A.cnt1[u] = 0;   // clean for the next call
  }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kScanThreads, 1)
wave_scan_kernel(const __grid_constant__ Geo geo, const __grid_constant__ ChunkMap cm,
                 const __grid_constant__ ScanArgs A,
                 const __grid_constant__ CUtensorMap tm_cent,
                 const __grid_constant__ CUtensorMap tm_vsum,
                 const __grid_constant__ CUtensorMap tm_off, uint32_t* status) {
  using TS = TileShape<T, D>;
  using SM = ScanSmem<T, D, G>;
  constexpr bool kMma = std::is_same_v<T, __nv_bfloat16>;
  constexpr int kBoxCols = 128 / (int)sizeof(T);
  extern __shared__ __align__(16) unsigned char sh_raw[];
  __shared__ __align__(8) uint64_t s_full[4], s_empty[4];
  __shared__ int s_ntails;
  __shared__ int s_tails[kMaxTailsPerCta];   // units whose last arrival was this CTA's
  __shared__ float* s_last_part;             // the CTA's last unit's estimation part
  __shared__ int32_t s_k0s[kNumSMs + 1];     // the scan CTAs' first chunks
  // the hand-off of the first unit's arrival to the producer warp, when the
  // CTA's chunks span more than one unit
  __shared__ __align__(8) uint64_t s_mid_full, s_mid_done;
  __shared__ float* s_mid_part;
  __shared__ int s_mid_u, s_mid_parts;
  pdl_launch_dependents();
  unsigned char* sh = align_smem_1024(sh_raw);
  const int slots = A.slots;
  const size_t tile_bytes = SM::tile_bytes(A.exact_only);
  unsigned char* ring = sh;
  unsigned char* side0 = ring + SM::ring_bytes(slots, A.exact_only);
  unsigned char* s_tail = side0 + SM::side_bytes(slots);
  float* comb = reinterpret_cast<float*>(s_tail + SM::kTail);   // per-warp softmax parts
  float* comb2 = comb + SM::kComb / 4;                          // (of the first of two units)
  uint32_t* hist16 = reinterpret_cast<uint32_t*>(reinterpret_cast<unsigned char*>(comb) +
                                                 SM::kComb * (A.mid_ok ? 2 : 1));
  RowMult* s_rows = reinterpret_cast<RowMult*>(reinterpret_cast<unsigned char*>(hist16) + SM::kHist16);
  float* s_sc = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(s_rows) + SM::kRows);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = blockIdx.x;
  const int k0 = cm.n_chunks > 0 ? cm.k0(s) : 0, k1 = cm.n_chunks > 0 ? cm.k0(s + 1) : 0;
  const int nk = k1 - k0;
  // chunks of the CTA's first unit; `mid`: more follow (the first unit's
  // arrival is then the producer warp's)
  int n1 = 0;
  if (nk > 0) {
    ChunkPos p1;
    chunk_seek(p1, geo, cm, k0);
    n1 = min(nk, p1.kend - p1.k);
  }
  const bool mid = A.mid_ok && n1 < nk;
  if (tid == 0) {
    for (int i = 0; i < slots; ++i) { mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], kConsumerWarps); }
    mbar_init(&s_mid_full, 1);
    mbar_init(&s_mid_done, 1);
    mbar_init_fence();
  }
  for (int i = tid; i < kHistBins / 2; i += blockDim.x) hist16[i] = 0u;
  for (int i = tid; i <= cm.n_scan; i += blockDim.x) s_k0s[i] = cm.k0s[i];
  if (tid == 0) s_ntails = 0;
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---- producer: chunk i into slot i % slots once the slot is free: its
    // key (and value-sum) tile, its offsets box, and the unit's queries when
    // the chunk starts a unit
    if (lane == 0 && nk > 0) {
      // the first unit's arrival, once the consumers have flushed its
      // histogram counts (they hand it over on s_mid_full)
      auto mid_arrival = [&]() {
        mbar_wait(&s_mid_full, 0u, status);
        fence_acq_rel_gpu();
        const int old = atomicAdd(A.cnt1 + s_mid_u, 1);
        if (old == s_mid_parts - 1) {
          fence_acq_rel_gpu();
          s_tails[atomicAdd(&s_ntails, 1)] = s_mid_u;
        }
        mbar_arrive(&s_mid_done);
      };
      const int i_mid = n1 - 1 + slots;   // the first issue that needs the first unit's last slot
      ChunkPos p;
      chunk_seek(p, geo, cm, k0);
      int prev_u = -1;
      for (int i = 0; i < nk; ++i) {
        const int sl = i % slots;
        if (i >= slots) mbar_wait(&s_empty[sl], (uint32_t)((i / slots - 1) & 1), status);
        if (mid && i == i_mid) mid_arrival();
        if (i > 0) chunk_next(p, geo, cm);
        const bool new_u = p.u != prev_u;
        prev_u = p.u;
        const int y = (int)(p.row0 + p.c0);
        unsigned char* dst = ring + sl * tile_bytes;
        unsigned char* side = side0 + sl * SM::kSide;
        const uint32_t bytes = (uint32_t)tile_bytes + kOffBox * 4 + (new_u ? (uint32_t)SM::kQBytes : 0u);
        mbar_arrive_expect(&s_full[sl], bytes);
#pragma unroll
        for (int nb = 0; nb < TS::NB; ++nb)
          tensor_load_2d(dst + nb * TS::kBoxBytes, &tm_cent, nb * kBoxCols, y, &s_full[sl]);
        if (!A.exact_only) {
#pragma unroll
          for (int nb = 0; nb < TS::NB; ++nb)
            tensor_load_2d(dst + TS::kBytes + nb * TS::kBoxBytes, &tm_vsum, nb * kBoxCols, y,
                           &s_full[sl]);
        }
        tensor_load_1d(side, &tm_off, (int)((p.orow + p.c0) & ~(int64_t)3), &s_full[sl]);
        if (new_u) {
          const unsigned char* qsrc = reinterpret_cast<const unsigned char*>(A.q) +
                                      ((int64_t)p.b * A.Hq + (int64_t)p.h * G) * D * (int64_t)sizeof(T);
          bulk_load(side + kOffArea, qsrc, (uint32_t)SM::kQBytes, &s_full[sl]);
        }
      }
      if (mid && i_mid >= nk) mid_arrival();
      // every copy issued has landed before the CTA may leave (bounded)
      for (int i = max(0, nk - slots); i < nk; ++i)
        mbar_wait(&s_full[i % slots], (uint32_t)((i / slots) & 1), status);
    }
    // the CTA's last estimation part, combined while the consumers run the
    // tails (barrier 2: the consumers' warp parts are in shared memory)
    if (!A.exact_only && nk > 0) {
      __syncwarp();
      named_sync(2, kScanThreads);
      combine_warps_1w<D, G>(comb, s_last_part, lane);
      if (mid) combine_warps_1w<D, G>(comb2, s_mid_part, lane);
    }
    pdl_wait();
    return;
  }

  // ---- consumers: an outer loop over the units of the CTA's range, a
  // tight inner loop over a unit's chunks (slot and phase kept as counters)
  MmaAcc<D, G> macc;
  FmaAcc<D, G> facc;
  const int g = lane >> 2, tq = lane & 3;
  int since_flush = 0;
  RowMult* rm = s_rows + warp * 8;
  float* sc = s_sc + warp * 8 * G;
  const int r0 = 8 * warp;   // the warp's rows of every chunk
  int sl = 0;
  uint32_t ph = 0u;
  for (int i = 0; i < nk;) {
    ChunkPos c;
    chunk_seek(c, geo, cm, k0 + i);
    const int n_here = min(nk - i, c.kend - c.k);   // the unit's chunks in this CTA
    // this CTA's part index among the unit's scan CTAs, and their number
    const int cf = ChunkMap::cta_in(s_k0s, cm.n_scan, c.kend - cm.per_unit(c.b));
    const int u_slot = s - cf;
    const int u_parts = ChunkMap::cta_in(s_k0s, cm.n_scan, c.kend - 1) - cf + 1;
    for (int ii = 0; ii < n_here; ++ii) {
      const unsigned char* ktile = ring + sl * tile_bytes;
      const unsigned char* vtile = ktile + TS::kBytes;
      const unsigned char* side = side0 + sl * SM::kSide;
      __syncwarp();   // the previous chunk's row data is read
      mbar_wait(&s_full[sl], ph, status);
      if (ii == 0) {
        const T* qs = reinterpret_cast<const T*>(side + kOffArea);
        if constexpr (kMma) { macc.load_q(qs); macc.reset(); }
        else { facc.load_q(qs, A.scale); facc.reset(); }
      }
      // rows r0 .. r0 + 7: counts and first slots from the chunk's offsets
      const int32_t* offs = reinterpret_cast<const int32_t*>(side) + (int)((c.orow + c.c0) & 3);
      const int off_l = lane <= 8 ? offs[r0 + lane] : 0;
      {
        const int o_next = __shfl_down_sync(0xffffffffu, off_l, 1);
        if (lane < 8) {
          const int cnt = o_next - off_l;
          const bool ok = r0 + lane < c.nrows && cnt > 0;
          rm[lane] = RowMult{1.f, (float)cnt, ok ? 1 : 0};
        }
        __syncwarp();
      }
      // scores, keys, estimation
      float key_s[2] = {-INFINITY, -INFINITY};   // group max of rows 2tq, 2tq+1 (MMA) / lane's row (FMA)
      if constexpr (kMma) {
        float s0, s1;
        macc.scores(ktile, r0, A.scale, s0, s1);
        if (A.scores_out && g < G) {
          const int cl = c.c0 + r0 + 2 * tq;
          if (cl < c.c0 + c.nrows) A.scores_out[(c.row0 + cl) * G + g] = s0;
          if (cl + 1 < c.c0 + c.nrows) A.scores_out[(c.row0 + cl + 1) * G + g] = s1;
        }
        float m0 = g < G ? s0 : -INFINITY, m1 = g < G ? s1 : -INFINITY;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
          m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
        }
        key_s[0] = m0;
        key_s[1] = m1;
        if (!A.exact_only) macc.fold(vtile, r0, s0, s1, rm);
      } else {
        facc.scores(ktile, r0, sc);
        if (lane < 8) {
          float mx = -INFINITY;
#pragma unroll
          for (int gg = 0; gg < G; ++gg) mx = fmaxf(mx, sc[lane * G + gg]);
          key_s[0] = mx;
          if (A.scores_out) {
            const int cl = c.c0 + r0 + lane;
            if (cl < c.c0 + c.nrows)
              for (int gg = 0; gg < G; ++gg) A.scores_out[(c.row0 + cl) * G + gg] = sc[lane * G + gg];
          }
        }
        if (!A.exact_only) facc.fold(vtile, r0, sc, rm);
      }
      // the slot's last reads are done: release it to the producer
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[sl]);
      if (++sl == slots) { sl = 0; ph ^= 1u; }
      // the records {key, first slot} of the warp's 8 rows (lanes 0..7, one
      // 64-byte store) and the first digit's histogram
      {
        float kv = key_s[0];
        if constexpr (kMma) {
          // MMA lane t (t < 4) holds the keys of rows 2t and 2t + 1
          const float ka = __shfl_sync(0xffffffffu, key_s[0], (lane >> 1) & 3);
          const float kb = __shfl_sync(0xffffffffu, key_s[1], (lane >> 1) & 3);
          kv = (lane & 1) ? kb : ka;
        }
        if (lane < 8 && r0 + lane < c.nrows) {
          const uint32_t key = rm[lane].valid ? ordered_key(kv) : 0u;
          A.rec[c.row0 + c.c0 + r0 + lane] = make_uint2(key, (uint32_t)off_l);
          if (key) atomicAdd(&hist16[key >> (kHistShift + 1)], 1u << (16 * ((key >> kHistShift) & 1u)));
        }
      }
      since_flush += kTileRows;
      if (since_flush >= 65536 - kTileRows && ii + 1 < n_here) {
        // 16-bit counters near overflow inside a long unit: flush them now
        pdl_wait();   // (the steady kernel has cleared the histograms)
        csync();
        int32_t* hg = A.hist + (int64_t)c.u * kHistBins;
        for (int wd = tid; wd < kHistBins / 2; wd += kConsumers) {
          const uint32_t v = hist16[wd];
          if (v) {
            if (v & 0xffffu) atomicAdd(hg + 2 * wd, (int)(v & 0xffffu));
            if (v >> 16) atomicAdd(hg + 2 * wd + 1, (int)(v >> 16));
            hist16[wd] = 0u;
          }
        }
        since_flush = 0;
        csync();
      }
      c.c0 += kTileRows;
      c.nrows = min(kTileRows, c.NC - c.c0);
    }
    i += n_here;
    // ---- end of the CTA's part of the unit: histogram, arrival, part
    pdl_wait();   // the steady kernel has cleared the histograms and counters
    csync();
    {
      int32_t* hg = A.hist + (int64_t)c.u * kHistBins;
      for (int wd = tid; wd < kHistBins / 2; wd += kConsumers) {
        const uint32_t v = hist16[wd];
        if (v) {
          if (v & 0xffffu) atomicAdd(hg + 2 * wd, (int)(v & 0xffffu));
          if (v >> 16) atomicAdd(hg + 2 * wd + 1, (int)(v >> 16));
          hist16[wd] = 0u;
        }
      }
      since_flush = 0;
    }
    // every thread's records and histogram counts are written before the
    // barrier; one fenced arrival publishes them (a cumulative fence)
    csync();   // (and the words are clear before the next unit counts into them)
    float* const part = A.est + ((int64_t)c.u * A.p1max + u_slot) * G * (D + kPartStride);
    if (mid && i == n1) {
      // the first of several units: its warps' parts wait in comb2 and the
      // producer warp arrives for it (and combines the parts at the end)
      if (!A.exact_only) {
        if constexpr (kMma) macc.to_smem(comb2 + warp * G * (D + kPartStride));
        else facc.to_smem(comb2 + warp * G * (D + kPartStride));
      }
      csync();
      if (tid == 0) {
        s_mid_part = part;
        s_mid_u = c.u;
        s_mid_parts = u_parts;
        mbar_arrive(&s_mid_full);
      }
      continue;
    }
    if (tid == 0) {
      fence_acq_rel_gpu();
      const int old = atomicAdd(A.cnt1 + c.u, 1);
      if (old == u_parts - 1) {
        fence_acq_rel_gpu();
        s_tails[atomicAdd(&s_ntails, 1)] = c.u;
      }
    }
    // the estimation part is the gather's, read once the scan has completed:
    // the warps' parts are combined after the arrival, the CTA's last unit's
    // by the producer warp while the consumers run the tails
    if (!A.exact_only) {
      if constexpr (kMma) macc.to_smem(comb + warp * G * (D + kPartStride));
      else facc.to_smem(comb + warp * G * (D + kPartStride));
      csync();
      if (i < nk) {
        combine_warps<D, G>(comb, part, tid);
        csync();   // the parts are read before the next unit writes them
      } else {
        if (tid == 0) s_last_part = part;
        named_arrive(2, kScanThreads);   // the producer warp combines it
      }
    }
  }
  // ---- the tails of the units this CTA finished last (after the loop, so
  // the accumulators are dead and the tail has the registers)
  if (mid) mbar_wait(&s_mid_done, 0u, status);   // the producer's arrival for the first unit
  csync();
  const int nt = s_ntails;
  for (int t = 0; t < nt; ++t) {
    const int u = s_tails[t], b = u / geo.hkv, h = u - b * geo.hkv;
    const TailUnit tu{u, geo.NC(b), geo.T(b), geo.cl_row(b, h), geo.tok_row(b, h)};
    scan_tail(tu, A, s_tail, ring, SM::kTailCandOff, SM::kTailDrawOff, SM::kTailShOff, status);
    csync();
  }
  pdl_wait();
}

// ------------------------------------------------------------- K2 gather
struct GatherArgs {
  const void* q;
  int Hq;
  Pool kp, vp;
  const void* centroids;
  const void* value_sums;
  const int32_t* perm;
  const uint2* rec;
  const int32_t* info;
  const int32_t* st_slot;
  const int2* pc;
  const int4* selinfo;   // retrieved {id, first slot, count, first token row}
  const int32_t* blkf;   // per block of token rows: its first retrieved cluster
  const int2* nonc;      // (cluster, count) of the non-candidates
  int cap;
  int n_sink, window;
  float* est;
  int p1max;
  float* gat;            // [U][n2max][G][D + 4]
  int n2max;
  int32_t* cnt2;         // [U] arrivals (zero between calls)
  float* out;
  float* lse;
  float scale;
  uint32_t seed;
  int32_t n2_base[kMaxBatch + 1];
};

enum RowKind { kRowNone = 0, kRowToken = 1, kRowSteady = 2, kRowFull = 3, kRowPart = 4 };

template <typename T, int D, int G>
struct GatherSmem {
  using TS = TileShape<T, D>;
  using GT = PadTile<TS::kRowBytes>;   // the gather's tile layout
  static constexpr int kRowsPerBlock = kGatherTiles * kTileRows;
  static constexpr size_t kTiles = (size_t)2 * kGatherTiles * GT::kBytes;   // K and V
  static constexpr size_t kMeta = (size_t)kRowsPerBlock * (8 + 8 + 4 + 4);
  static constexpr size_t kComb = (size_t)kConsumerWarps * G * (D + kPartStride) * 4;
  static constexpr size_t kRows = (size_t)kConsumerWarps * 8 * sizeof(RowMult);
  static constexpr size_t kSc = (size_t)kConsumerWarps * 8 * G * 4;
  static constexpr size_t kMergeParts = kMaxGatherPerUnit;   // parts a unit's merge reads
  static constexpr size_t kMerge = (kMergeParts * G * 3 * 4 + (size_t)G * 8 + 15) / 16 * 16;
  static constexpr size_t kPart = (size_t)G * (D + kPartStride) * 4;   // s_part, s_pre
  static constexpr size_t kTotal = 1024 + kTiles + kMeta + kComb + kRows + kSc + kMerge +
                                   2 * kPart + (size_t)G * 8;
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kGatherThreads, 2)
wave_gather_kernel(const __grid_constant__ Geo geo, const __grid_constant__ ChunkMap cm,
                   const __grid_constant__ GatherArgs A, uint32_t* status) {
  using TS = TileShape<T, D>;
  using SM = GatherSmem<T, D, G>;
  using GT = typename SM::GT;
  constexpr bool kMma = std::is_same_v<T, __nv_bfloat16>;
  constexpr int RPB = SM::kRowsPerBlock;
  static_assert(kGatherThreads == 2 * RPB, "one thread per row of K and of V");
  extern __shared__ __align__(16) unsigned char sh_raw[];
  __shared__ int s_rec[kInfoInts];
  __shared__ int s_last;
  __shared__ int s_bf[2];                  // first retrieved clusters of the CTA's first block and the next
  __shared__ int s_slot[kGatherRows];      // token slots of the block's token rows
  __shared__ __align__(8) uint64_t s_gbar; // the block's row copies
  unsigned char* sh = align_smem_1024(sh_raw);
  unsigned char* tiles = sh;                                   // [K t0][K t1][V t0][V t1]
  const unsigned char** s_kp = reinterpret_cast<const unsigned char**>(tiles + SM::kTiles);
  const unsigned char** s_vp = s_kp + RPB;
  int* s_kind = reinterpret_cast<int*>(s_vp + RPB);
  int* s_aux = s_kind + RPB;
  float* comb = reinterpret_cast<float*>(s_aux + RPB);
  RowMult* s_rows = reinterpret_cast<RowMult*>(reinterpret_cast<unsigned char*>(comb) + SM::kComb);
  float* s_sc = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(s_rows) + SM::kRows);
  float* s_merge = s_sc + kConsumerWarps * 8 * G;
  float* s_part = s_merge + SM::kMerge / 4;                  // [G][D + 4] this CTA's part
  float* s_pre = s_part + SM::kPart / 4;                     // [G][D + 4] a prefetched scan part
  float* s_fac = s_pre + SM::kPart / 4;                      // [G][2] fold factors
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // CTA -> (sequence b, KV head h, index j of the unit's n2 CTAs)
  int b = 0;
  {
    int lo = 0, hi = geo.batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (A.n2_base[mid] <= (int)blockIdx.x) lo = mid; else hi = mid - 1;
    }
    b = lo;
  }
  const int n2 = (A.n2_base[b + 1] - A.n2_base[b]) / geo.hkv;
  const int rel = (int)blockIdx.x - A.n2_base[b];
  // index j of the unit's CTAs major: the CTAs that launch first (one per SM)
  // are the ones whose blocks are full
  const int j = rel / geo.hkv, h = rel - j * geo.hkv;
  const int u = b * geo.hkv + h;
  const int Tb = geo.T(b);
  const int ns = min(A.n_sink, Tb), wstart = max(Tb - A.window, ns);
  const int64_t row0 = geo.cl_row(b, h), trow = geo.tok_row(b, h);
  const T* qg = reinterpret_cast<const T*>(A.q) + ((int64_t)b * A.Hq + (int64_t)h * G) * D;
  MmaAcc<D, G> macc;
  FmaAcc<D, G> facc;
  if constexpr (kMma) { macc.load_q(qg); macc.reset(); }
  else { facc.load_q(qg, A.scale); facc.reset(); }
  // while the scan finishes: the sequence's block table into L2 (by the
  // first CTA of each sequence; the token rows' page lookups hit it there)
  if (rel == 0)
    for (int i = 32 * tid; i < A.kp.max_pages; i += 32 * kGatherThreads)
      prefetch_l2(A.kp.bt + (int64_t)b * A.kp.max_pages + i);

  // the scan's parts of the unit: the scan CTAs whose chunks meet its own
  const int u_first = cm.first(b, h), u_end = u_first + cm.per_unit(b);
  const int np_scan = __syncthreads_count(tid < cm.n_scan && cm.k0s[tid] < u_end &&
                                          cm.k0s[tid + 1] > u_first);

  if (tid == 0) {
    mbar_init(&s_gbar, 1);
    mbar_init_fence();
  }
  uint32_t gphase = 0u;

  pdl_wait();   // the scan's and the steady kernel's results
  // the unit's record, and (speculatively) where the first block's token
  // rows start among the retrieved clusters
  if (tid < kInfoInts) s_rec[tid] = __ldcg(A.info + (int64_t)u * kInfoInts + tid);
  if (tid == 32 || tid == 33) {
    const int bk = j + tid - 32;
    s_bf[tid - 32] = bk < Tb ? __ldcg(A.blkf + trow + bk) : 0;
  }
  __syncthreads();
  const bool dense = s_rec[kDense] != 0, no_est = s_rec[kNoEstimate] != 0;
  // the scan's estimation parts this CTA folds into its own (p = j, j + n2,
  // ...): the first one's copies go out now, to land during the gather
  const int np1 = no_est ? 0 : np_scan;
  if (np1 > j) {
    const float* src = A.est + ((int64_t)u * A.p1max + j) * G * (D + kPartStride);
    for (int x = tid; x < G * (D + kPartStride) / 4; x += blockDim.x)
      cp_async16(s_pre + 4 * x, src + 4 * x);
    cp_async_commit();
  }
  const int n_sel = dense ? 0 : s_rec[kSelCount];
  const int n_tok = dense ? 0 : s_rec[kSelTokens];
  const int n_st = s_rec[kSteady];
  const int n_full = (dense || no_est) ? 0 : s_rec[kFullRows];
  const int n_pc = (dense || no_est) ? 0 : s_rec[kPartRows];
  const int R = n_tok + n_st + n_full + n_pc;
  const Threshold th{(uint32_t)s_rec[kThrKey], s_rec[kThrIdx], s_rec[kMode], s_rec[kSampBin],
                     ((uint64_t)(uint32_t)s_rec[kSampHash] << 32) | (uint32_t)s_rec[kSampHashLo],
                     A.seed};
  const unsigned char* kpool = reinterpret_cast<const unsigned char*>(A.kp.base);
  const unsigned char* vpool = reinterpret_cast<const unsigned char*>(A.vp.base);
  const unsigned char* cent = reinterpret_cast<const unsigned char*>(A.centroids);
  const unsigned char* vsum = reinterpret_cast<const unsigned char*>(A.value_sums);
  constexpr int RB = TS::kRowBytes;

  for (int blk = j; blk * RPB < R; blk += n2) {
    const int rb = blk * RPB;
    // ---- the block's token rows: the slots of the retrieved clusters that
    // overlap it (at most RPB + 1 of them), filled in by their records
    if (rb < n_tok) {
      int s_lo = blk == j ? s_bf[0] : __ldcg(A.blkf + trow + blk);
      int s_hi = rb + RPB >= n_tok ? n_sel - 1
                                   : (blk == j ? s_bf[1] : __ldcg(A.blkf + trow + blk + 1));
      if (s_lo < 0 || s_hi >= n_sel || s_hi < s_lo || s_hi - s_lo > RPB) {
        if (tid == 0) flag_error(status, WI_DEV_BAD_CLUSTER);
        s_lo = 0;
        s_hi = -1;
      }
      if (tid < RPB) s_slot[tid] = -1;
      __syncthreads();
      for (int e = tid; e <= s_hi - s_lo; e += blockDim.x) {
        const int4 si = __ldcg(A.selinfo + row0 + s_lo + e);   // {id, first slot, count, first row}
        const int r0 = max(si.w, rb), r1 = min(min(si.w + si.z, rb + RPB), n_tok);
        for (int r = r0; r < r1; ++r) s_slot[r - rb] = si.y + (r - si.w);
      }
      __syncthreads();
    }
    // ---- resolve the block's rows: kind, key and value row addresses (the
    // token rows' positions and the partial rows' cluster keys, which only
    // the attention needs, are loaded once the rows' copies are out)
    int kind = kRowNone, aux = 0;
    const int32_t* auxp = nullptr;
    int auxc = -1;
    if (tid < RPB) {
      const int r = rb + tid;
      const unsigned char* kr = nullptr;
      const unsigned char* vr = nullptr;
      int slot = -1, c = -1;
      if (r < R) {
        if (dense) {
          slot = r; kind = kRowSteady;
        } else if (r < n_tok) {
          slot = s_slot[tid];
          kind = kRowToken;
        } else if (r < n_tok + n_st) {
          slot = __ldcg(A.st_slot + (int64_t)u * A.cap + (r - n_tok));
          kind = kRowSteady;
        } else if (r < n_tok + n_st + n_full) {
          const int f = r - n_tok - n_st;   // retrieved clusters, then the non-candidates
          if (f < n_sel) {
            const int4 si = __ldcg(A.selinfo + row0 + f);
            c = si.x; aux = si.z;
          } else {
            const int2 nc = __ldcg(A.nonc + (int64_t)u * A.cap + (f - n_sel));
            c = nc.x; aux = nc.y;
          }
          kind = kRowFull;
        } else {
          const int2 p = __ldcg(A.pc + (int64_t)u * A.cap + (r - n_tok - n_st - n_full));
          slot = p.x; c = p.y; kind = kRowPart;
        }
      }
      if (kind == kRowFull || kind == kRowPart) {
        if (c < 0 || c >= geo.NC(b)) { flag_error(status, WI_DEV_BAD_CLUSTER); kind = kRowNone; }
        else kr = cent + (row0 + c) * RB;
      }
      if (kind == kRowFull) vr = vsum + (row0 + c) * RB;
      if (kind == kRowToken || kind == kRowSteady || kind == kRowPart) {
        const int64_t ro = pool_row(A.kp, geo.hkv, D, b, h, slot, status);
        if (ro < 0) {
          kind = kRowNone;
        } else {
          if (kind != kRowPart) kr = kpool + ro * (int64_t)sizeof(T);
          vr = vpool + ro * (int64_t)sizeof(T);
          if (kind == kRowToken) {
            if (slot >= Tb) { flag_error(status, WI_DEV_BAD_SLOT); kind = kRowNone; }
            else auxp = A.perm + trow + slot;
          } else if (kind == kRowPart) {
            auxp = reinterpret_cast<const int32_t*>(&A.rec[row0 + c].x);
            auxc = c;
          }
        }
      }
      s_kind[tid] = kind;
      s_aux[tid] = aux;
      s_kp[tid] = kind == kRowNone ? nullptr : kr;
      s_vp[tid] = kind == kRowNone ? nullptr : vr;
    }
    const int nrows = __syncthreads_count(tid < RPB && kind != kRowNone);
    // ---- gather: each key and value row by one bulk copy (thread t: row
    // t % RPB of K or V), all completing on one barrier; rows past the
    // block's are zero
    if (tid == 0) mbar_arrive_expect(&s_gbar, (uint32_t)(2 * nrows * TS::kRowBytes));
    {
      const int mat = tid / RPB, rr = tid - mat * RPB;
      const unsigned char* src = mat == 0 ? s_kp[rr] : s_vp[rr];
      unsigned char* dst = tiles + (size_t)(mat * kGatherTiles + rr / kTileRows) * GT::kBytes +
                           GT::off(rr % kTileRows, 0);
      if (src) {
        bulk_load(dst, src, TS::kRowBytes, &s_gbar);
      } else {
#pragma unroll
        for (int ch = 0; ch < TS::kChunks; ++ch)
          reinterpret_cast<uint4*>(dst)[ch] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    if (kind == kRowToken) {
      s_aux[tid] = __ldg(auxp);   // the token's position in the sequence
    } else if (kind == kRowPart) {
      // a partial row's cluster is taken out of the estimate only when it
      // is not retrieved
      s_aux[tid] = th.picked(__ldcg(reinterpret_cast<const uint32_t*>(auxp)), (uint32_t)auxc) ? 1 : 0;
    }
    mbar_wait(&s_gbar, gphase, status);
    gphase ^= 1u;
    __syncthreads();   // (the zero rows)
    // ---- attend: warp w takes rows 8w .. 8w + 7 of each tile
#pragma unroll 1
    for (int t = 0; t < kGatherTiles; ++t) {
      const int lr = t * kTileRows + 8 * warp;    // block-local row of the warp's first
      RowMult* rm = s_rows + warp * 8;
      if (lane < 8) {
        const int q = lr + lane;
        const int kind = s_kind[q];
        RowMult m{0.f, 0.f, 0};
        if (kind == kRowToken) {
          const int pos = s_aux[q];
          const bool st = pos < ns || pos >= wstart;
          m = st ? RowMult{0.f, 0.f, 0} : RowMult{1.f, 1.f, 1};
        } else if (kind == kRowSteady) {
          m = RowMult{1.f, 1.f, 1};
        } else if (kind == kRowFull) {
          m = RowMult{-1.f, -(float)s_aux[q], 1};
        } else if (kind == kRowPart) {
          m = s_aux[q] ? RowMult{0.f, 0.f, 0} : RowMult{-1.f, -1.f, 1};
        }
        rm[lane] = m;
      }
      __syncwarp();
      const unsigned char* kt = tiles + (size_t)t * GT::kBytes;
      const unsigned char* vt = tiles + (size_t)(kGatherTiles + t) * GT::kBytes;
      if constexpr (kMma) {
        float s0, s1;
        macc.template scores<GT>(kt, 8 * warp, A.scale, s0, s1);
        macc.template fold<GT>(vt, 8 * warp, s0, s1, rm);
      } else {
        float* sc = s_sc + warp * 8 * G;
        facc.template scores<GT>(kt, 8 * warp, sc);
        facc.template fold<GT>(vt, 8 * warp, sc, rm);
      }
      __syncwarp();
    }
    fence_proxy_async();   // the tiles' reads and zero rows before the next block's copies
    __syncthreads();       // tiles and row data are read before the next block
  }
  // ---- this CTA's part (its rows, plus its share of the scan's estimation
  // parts: p = j, j + n2, ...), then the unit's merge by its last CTA
  if constexpr (kMma) macc.to_smem(comb + warp * G * (D + kPartStride));
  else facc.to_smem(comb + warp * G * (D + kPartStride));
  const bool has_pre = np1 > j;               // the scan part prefetched into s_pre
  const bool extra = j + n2 < np1;            // more scan parts than the unit's CTAs
  if (has_pre) cp_async_wait<0>();
  __syncthreads();
  float* part = A.gat + ((int64_t)u * A.n2max + j) * G * (D + kPartStride);
  // the warps' parts and the prefetched scan part in one combine, straight
  // into the published part (through s_part when more scan parts follow)
  combine_warps<D, G>(comb, extra ? s_part : part, tid, has_pre ? s_pre : nullptr);
  auto fold_part = [&](const float* src) {   // s_part <- s_part (+) src (shared or global)
    if (tid < G) {
      const float ma = s_part[tid * (D + kPartStride)], mb = src[tid * (D + kPartStride)];
      const float M = fmaxf(ma, mb);
      const float fa = ma == -INFINITY ? 0.f : expf(ma - M);
      const float fb = mb == -INFINITY ? 0.f : expf(mb - M);
      s_fac[2 * tid] = fa;
      s_fac[2 * tid + 1] = fb;
      float* row = s_part + tid * (D + kPartStride);
      row[0] = M;
      row[1] = row[1] * fa + src[tid * (D + kPartStride) + 1] * fb;
      row[2] = row[2] * fa + src[tid * (D + kPartStride) + 2] * fb;
    }
    __syncthreads();
    for (int i = tid; i < G * D; i += blockDim.x) {
      const int gg = i / D, e = i - gg * D;
      float* o = s_part + gg * (D + kPartStride) + kPartStride + e;
      *o = *o * s_fac[2 * gg] + src[gg * (D + kPartStride) + kPartStride + e] * s_fac[2 * gg + 1];
    }
    __syncthreads();
  };
  if (extra) {
    __syncthreads();
    for (int p = j + n2; p < np1; p += n2)
      fold_part(A.est + ((int64_t)u * A.p1max + p) * G * (D + kPartStride));
    for (int i = tid; i < G * (D + kPartStride); i += blockDim.x) part[i] = s_part[i];
  }
  // every thread's part is written before the barrier; one fenced arrival
  // publishes it (a cumulative fence)
  __syncthreads();
  if (tid == 0) {
    fence_acq_rel_gpu();
    const int old = atomicAdd(A.cnt2 + u, 1);
    if (old == n2 - 1) fence_acq_rel_gpu();
    s_last = old == n2 - 1;
  }
  __syncthreads();
  if (!s_last) return;
  // the merge of the unit's n2 parts.  Every part's (m, l, ln) is loaded
  // first; then each thread's share of the parts' outputs (a 16-byte column,
  // the threads forming kS slices of the parts) is loaded straight into
  // registers, landing while the heads' maxima and the parts' factors form
  const int np = n2;
  auto part_ptr = [&](int p) -> const float* {
    return A.gat + ((int64_t)u * A.n2max + p) * G * (D + kPartStride);
  };
  constexpr int C4 = G * D / 4;                     // 16-byte columns of a part's outputs
  static_assert(kGatherThreads % C4 == 0, "the columns tile the CTA");
  constexpr int kS = kGatherThreads / C4;           // part slices
  constexpr int kB = 16;                            // parts a thread holds in registers
  constexpr int kF = (kMaxGatherPerUnit * G + kGatherThreads - 1) / kGatherThreads;
  const int c4 = tid % C4, sl = tid / C4;
  const int gq = c4 / (D / 4), e4 = c4 - gq * (D / 4);   // the column's head and offset
  const int64_t qh = (int64_t)b * A.Hq + (int64_t)h * G + gq;
  float* outp = A.out + qh * D + 4 * e4;
  float* lsep = A.lse;
  asm volatile("" : "+l"(outp), "+l"(lsep));   // the parameters are read now, off the tail
  auto col = [&](int p) {
    return __ldcg(reinterpret_cast<const float4*>(part_ptr(p) + gq * (D + kPartStride) + kPartStride) + e4);
  };
  float4 fm[kF];
#pragma unroll
  for (int k = 0; k < kF; ++k) {
    const int x = tid + k * kGatherThreads;
    if (x < np * G)
      fm[k] = __ldcg(reinterpret_cast<const float4*>(part_ptr(x / G) + (x % G) * (D + kPartStride)));
  }
  float4 ov[kB];
#pragma unroll
  for (int i = 0; i < kB; ++i)
    if (sl + i * kS < np) ov[i] = col(sl + i * kS);
  float* s_f = s_merge;                             // [kMergeParts][G] (m then factor, l, ln)
  float* s_M = s_merge + SM::kMergeParts * G * 3;   // [G] max, [G] denominator
  float* s_L = s_M + G;
#pragma unroll
  for (int k = 0; k < kF; ++k) {
    const int x = tid + k * kGatherThreads;
    if (x < np * G) {
      s_f[3 * x] = fm[k].x;
      s_f[3 * x + 1] = fm[k].y;
      s_f[3 * x + 2] = fm[k].z;
    }
  }
  __syncthreads();
  if (warp < G) {   // warp g: head g's max, the parts' factors, the denominator
    float M = -INFINITY;
    for (int p = lane; p < np; p += 32) M = fmaxf(M, s_f[3 * (p * G + warp)]);
    M = warp_max(M);
    float L = 0.f, LN = 0.f;
    for (int p = lane; p < np; p += 32) {
      const float mp = s_f[3 * (p * G + warp)];
      const float f = mp == -INFINITY ? 0.f : expf(mp - M);
      L += f * s_f[3 * (p * G + warp) + 1];
      LN += f * s_f[3 * (p * G + warp) + 2];
      s_f[3 * (p * G + warp)] = f;
    }
    L = warp_sum(L);
    LN = warp_sum(LN);
    if (lane == 0) {
      s_M[warp] = M;
      s_L[warp] = L;
      // the estimate is "every cluster minus what the zone leaves out": the
      // mass taken back out stays within the merged denominator when every
      // centroid is the mean of its members (Jensen); far above it, the
      // difference has lost its precision, and the call says so
      if (LN > kCancelRatio * fmaxf(L, 0.f)) flag_error(status, WI_DEV_CANCELLATION);
    }
  }
  __syncthreads();
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  auto fold = [&](int p0) {
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int p = p0 + sl + i * kS;
      if (p < np) {
        const float f = s_f[3 * (p * G + gq)];
        o.x += f * ov[i].x;
        o.y += f * ov[i].y;
        o.z += f * ov[i].z;
        o.w += f * ov[i].w;
      }
    }
  };
  fold(0);
  for (int p0 = kB * kS; p0 < np; p0 += kB * kS) {   // parts beyond the registers' batch
#pragma unroll
    for (int i = 0; i < kB; ++i)
      if (p0 + sl + i * kS < np) ov[i] = col(p0 + sl + i * kS);
    fold(p0);
  }
  if constexpr (kS > 1) {   // the slices' sums (the tile area is free by now)
    float4* red = reinterpret_cast<float4*>(tiles);
    if (sl > 0) red[(sl - 1) * C4 + c4] = o;
    __syncthreads();
    if (sl == 0)
#pragma unroll
      for (int k = 1; k < kS; ++k) {
        const float4 r = red[(k - 1) * C4 + c4];
        o.x += r.x;
        o.y += r.y;
        o.z += r.z;
        o.w += r.w;
      }
  }
  if (sl == 0) {
    const float L = s_L[gq];
    const float4 r = make_float4(L > 0.f ? o.x / L : 0.f, L > 0.f ? o.y / L : 0.f, L > 0.f ? o.z / L : 0.f,
                                 L > 0.f ? o.w / L : 0.f);
    // one 16-byte store where the output allows it (whole lines, also when
    // the output is the caller's mapped host buffer)
    if ((reinterpret_cast<uintptr_t>(outp) & 15) == 0) {
      *reinterpret_cast<float4*>(outp) = r;
    } else {
      outp[0] = r.x;
      outp[1] = r.y;
      outp[2] = r.z;
      outp[3] = r.w;
    }
    if (e4 == 0 && lsep) lsep[qh] = L > 0.f ? s_M[gq] + logf(L) : -INFINITY;
  }
  if (tid == 0) A.cnt2[u] = 0;   // clean for the next call
}

}  // namespace
}  // namespace wi


namespace wi {
namespace {

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

// rows x D matrix of bf16 or fp32, boxes of 64 rows x 128 bytes, 128-byte swizzle
bool encode_rows(CUtensorMap* tm, const void* base, int64_t rows, int D, int dtype) {
  auto fn = encode_fn();
  if (!fn || rows <= 0) return false;
  const int es = dtype == WI_BF16 ? 2 : 4;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * es};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / es), (cuuint32_t)kTileRows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(tm, dtype == WI_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
            2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// the offsets array as a 1-D int32 tensor, boxes of kOffBox entries
bool encode_offsets(CUtensorMap* tm, const int32_t* base, int64_t n) {
  auto fn = encode_fn();
  if (!fn || n <= 0) return false;
  const cuuint64_t dims[1] = {(cuuint64_t)n};
  const cuuint64_t strides[1] = {4};   // unused for one dimension
  const cuuint32_t box[1] = {(cuuint32_t)kOffBox};
  const cuuint32_t estr[1] = {1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_INT32, 1, const_cast<int32_t*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Dynamic shared memory limit, and the full shared-memory carveout for every
// decode kernel (kernels that overlap under programmatic dependent launch
// then never need the SM's L1 / shared split reconfigured between them).
// The attributes are set once per device and kernel, raised when a call
// needs more (each setting is a driver call on the decode's launch path).
template <typename Kern>
void set_smem(Kern kern, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, size_t> done;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  size_t& have = done[{dev, reinterpret_cast<const void*>(kern)}];
  if (have >= bytes && have != 0) return;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                       (int)cudaSharedmemCarveoutMaxShared);
  have = bytes;
}

// Tensor maps of recent calls' buffers, by (device, base, extent, row size,
// type); a map describes the buffer only, so a hit is always valid.
struct MapKey {
  int dev, dtype, D;
  const void* base;
  int64_t n;
  bool operator<(const MapKey& o) const {
    return std::tie(dev, dtype, D, base, n) < std::tie(o.dev, o.dtype, o.D, o.base, o.n);
  }
};
template <typename Encode>
bool cached_map(CUtensorMap* tm, const MapKey& key, Encode&& encode) {
  static std::mutex mu;
  static std::map<MapKey, CUtensorMap> maps;
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = maps.find(key);
    if (it != maps.end()) { *tm = it->second; return true; }
  }
  if (!encode(tm)) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (maps.size() >= 64) maps.clear();
  maps[key] = *tm;
  return true;
}

int pow2_at_least(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

}  // namespace

// K1 and K2 of one decode for key type T, head size D and group size G (the
// steady kernel, which does not depend on them, is launched by the caller).
template <typename T, int D, int G>
cudaError_t launch_decode_typed(const DecodePlan& p, const DecodeArgs& a, const ChunkMap& cm,
                                cudaStream_t s) {
  unsigned char* ws = a.ws;
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + p.off_status);
  cudaEvent_t* ev = a.stage_events;
  const bool pdl = ev == nullptr;
  auto mark = [&](int i) { if (ev) cudaEventRecord(ev[i], s); };
  int32_t* info = reinterpret_cast<int32_t*>(ws + p.off_info);
  int32_t* st_slot = reinterpret_cast<int32_t*>(ws + p.off_st_slot);
  int2* pc = reinterpret_cast<int2*>(ws + p.off_pc);
  int2* nonc = reinterpret_cast<int2*>(ws + p.off_nonc);
  // K1: scan + tails
  CUtensorMap tmc, tmv, tmo;
  std::memset(&tmc, 0, sizeof(tmc));
  std::memset(&tmv, 0, sizeof(tmv));
  std::memset(&tmo, 0, sizeof(tmo));
  const int64_t n_off = ((int64_t)p.geo.cl_base[p.geo.batch] + p.geo.batch) * p.geo.hkv;
  int dev = 0;
  cudaGetDevice(&dev);
  auto rows_map = [&](CUtensorMap* tm, const void* base) {
    return cached_map(tm, MapKey{dev, p.dtype, D, base, p.ncl},
                      [&](CUtensorMap* t) { return encode_rows(t, base, p.ncl, D, p.dtype); });
  };
  if (!rows_map(&tmc, a.centroids) || !rows_map(&tmv, a.value_sums) ||
      !cached_map(&tmo, MapKey{dev, -1, 0, a.offsets, n_off},
                  [&](CUtensorMap* t) { return encode_offsets(t, a.offsets, n_off); }))
    return cudaErrorInvalidValue;
  ScanArgs A{};
  A.q = a.q;
  A.Hq = p.Hq;
  A.rec = reinterpret_cast<uint2*>(ws + p.off_rec);
  A.hist = reinterpret_cast<int32_t*>(ws + p.off_hist);
  A.cnt1 = reinterpret_cast<int32_t*>(ws + p.off_cnt1);
  A.est = reinterpret_cast<float*>(ws + p.off_est);
  A.p1max = std::max(1, p.p1max);
  A.scores_out = a.scores_out;
  A.scale = p.scale;
  A.exact_only = p.exact_only;
  A.info = info;
  A.nonc = nonc;
  A.sel = reinterpret_cast<int32_t*>(ws + p.off_sel);
  A.blkf = reinterpret_cast<int32_t*>(ws + p.off_tok);
  A.selinfo = reinterpret_cast<int4*>(ws + p.off_selinfo);
  A.cap = p.cap;
  A.topk_clusters = p.topk_clusters;
  A.topk_fraction = p.topk_fraction;
  A.mode = p.mode;
  A.seed = p.seed;
  A.slots = p.slots;
  A.mid_ok = ScanSmem<T, D, G>::total(p.slots, p.exact_only, 1) <= (size_t)227 * 1024 ? 1 : 0;
  const size_t scan_smem = ScanSmem<T, D, G>::total(p.slots, p.exact_only, A.mid_ok);
  set_smem(wave_scan_kernel<T, D, G>, scan_smem);
  mark(1);
  cudaError_t e1 = launch_ex(wave_scan_kernel<T, D, G>, dim3(std::max(1, p.n_scan)),
                             dim3(kScanThreads), scan_smem, s, pdl, p.geo, cm, A, tmc, tmv,
                             tmo, status);
  if (e1 != cudaSuccess) return e1;
  // K2: gather, exact attention, estimate corrections, merge
  GatherArgs B{};
  B.q = a.q;
  B.Hq = p.Hq;
  B.kp = a.kp;
  B.vp = a.vp;
  B.centroids = a.centroids;
  B.value_sums = a.value_sums;
  B.perm = a.perm;
  B.rec = A.rec;
  B.info = info;
  B.st_slot = st_slot;
  B.pc = pc;
  B.blkf = A.blkf;
  B.selinfo = A.selinfo;
  B.nonc = nonc;
  B.cap = p.cap;
  B.n_sink = p.n_sink;
  B.window = p.window;
  B.est = A.est;
  B.p1max = A.p1max;
  B.gat = reinterpret_cast<float*>(ws + p.off_gat);
  B.n2max = p.n2max;
  B.cnt2 = reinterpret_cast<int32_t*>(ws + p.off_cnt2);
  B.out = a.out;
  B.lse = a.lse;
  B.scale = p.scale;
  B.seed = p.seed;
  std::memcpy(B.n2_base, p.n2_base, sizeof(B.n2_base));
  const size_t g_smem = GatherSmem<T, D, G>::kTotal;
  set_smem(wave_gather_kernel<T, D, G>, g_smem);
  mark(2);
  cudaError_t e2 = launch_ex(wave_gather_kernel<T, D, G>, dim3(p.n_gather), dim3(kGatherThreads),
                             g_smem, s, pdl, p.geo, cm, B, status);
  if (e2 != cudaSuccess) return e2;
  mark(3);
  return cudaGetLastError();
}

#define WI_DECODE_INSTANTIATE(T, D)                                                          \
  template cudaError_t launch_decode_typed<T, D, 1>(const DecodePlan&, const DecodeArgs&,    \
                                                    const ChunkMap&, cudaStream_t);          \
  template cudaError_t launch_decode_typed<T, D, 2>(const DecodePlan&, const DecodeArgs&,    \
                                                    const ChunkMap&, cudaStream_t);          \
  template cudaError_t launch_decode_typed<T, D, 4>(const DecodePlan&, const DecodeArgs&,    \
                                                    const ChunkMap&, cudaStream_t);          \
  template cudaError_t launch_decode_typed<T, D, 8>(const DecodePlan&, const DecodeArgs&,    \
                                                    const ChunkMap&, cudaStream_t);

#define WI_DECODE_EXTERN(T, D)                                                               \
  extern template cudaError_t launch_decode_typed<T, D, 1>(const DecodePlan&, const DecodeArgs&, \
                                                           const ChunkMap&, cudaStream_t);       \
  extern template cudaError_t launch_decode_typed<T, D, 2>(const DecodePlan&, const DecodeArgs&, \
                                                           const ChunkMap&, cudaStream_t);       \
  extern template cudaError_t launch_decode_typed<T, D, 4>(const DecodePlan&, const DecodeArgs&, \
                                                           const ChunkMap&, cudaStream_t);       \
  extern template cudaError_t launch_decode_typed<T, D, 8>(const DecodePlan&, const DecodeArgs&, \
                                                           const ChunkMap&, cudaStream_t);

}  // namespace wi

// Index-build kernels of the wave index (sm_100a): segmented k-means and the
// cluster-permuted paged KV scatter (RetroInfer technical summary, section
// 2.A, Segmented Clustering paragraph and item 2 Retrieval Zone; Vortex
// summary, section 2.A forward_cache).
//
//   init    centroid j of a segment = key at segment position j*cs
//   assign  argmin_j sum_e (k_e - c_je)^2 in fp32 (direct form, no
//           ||k||^2 - 2k.c + ||c||^2 cancellation), ties to the lower j;
//           fp32 keys: 64 tokens x 64 centroids per tile, 4x4 outputs per
//           thread; bf16 keys: k.c on the tcgen05 tensor cores, the direct
//           form wherever the two best are too close to call
//   update  per (unit, segment): stable counting sort of the tokens by
//           cluster, fp64 sums in ascending position, mean = sum / count;
//           on the last round it also writes offsets, perm, invperm, labels, the
//           rounded centroids and value sums, and copies the K/V rows to the
//           permuted pools (one pass over K and V).
#include <cfloat>
#include <climits>
#include <type_traits>

#include "wi_common.cuh"
#include "wi_plan.h"
#include "wi_umma.cuh"

namespace wi {
namespace {

template <typename T, int D>
struct BRow {
  static constexpr int EPL = Elem<T>::kPerVec;
  static constexpr int LPR = D / EPL;
  static constexpr int RPW = 32 / LPR;
};

// ------------------------------------------------------------------- init
template <typename T, int D>
__global__ void __launch_bounds__(kStreamThreads)
kmeans_init_kernel(const Geo geo, const Pool kin, int S, int cs, const SegFrom sf,
                   float* __restrict__ cent32, uint32_t* status) {
  using R = BRow<T, D>;
  const int u = blockIdx.y, b = u / geo.hkv, h = u - b * geo.hkv;
  const int T_ = geo.T(b);
  const int seg = sf.s0[b] + (int)blockIdx.x, start = seg * S;
  if (start >= T_) return;
  const int len = min(S, T_ - start);
  const int ncl = (len + cs - 1) / cs;
  const int64_t crow = geo.cl_row(b, h) + (int64_t)seg * (S / cs);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % R::LPR, rsub = lane / R::LPR;
  const int groups = (blockDim.x >> 5) * R::RPW;
  for (int j = warp * R::RPW + rsub; j < ncl; j += groups) {
    const int64_t ro = pool_row(kin, geo.hkv, D, b, h, start + j * cs, status);
    float x[R::EPL];
    if (ro >= 0) {
      const uint4 raw = ld_stream(reinterpret_cast<const T*>(kin.base) + ro + sub * R::EPL);
      Elem<T>::unpack(raw, x);
    } else {
#pragma unroll
      for (int e = 0; e < R::EPL; ++e) x[e] = 0.f;
    }
    float* dst = cent32 + (crow + j) * D + sub * R::EPL;
#pragma unroll
    for (int e = 0; e < R::EPL; ++e) dst[e] = x[e];
  }
}

// ----------------------------------------------------------------- assign
constexpr int kTok = 64, kCen = 64, kPad = 4;

template <typename T, int D>
__global__ void __launch_bounds__(256)
kmeans_assign_kernel(const Geo geo, const Pool kin, int S, int cs, const SegFrom sf,
                     const float* __restrict__ cent32, int32_t* __restrict__ assign,
                     uint32_t* status) {
  using R = BRow<T, D>;
  extern __shared__ float4 sh_assign4[];
  float* sk = reinterpret_cast<float*>(sh_assign4);      // [D][kTok + kPad]
  float* sc = sk + D * (kTok + kPad);                    // [D][kCen + kPad]
  const int u = blockIdx.z, b = u / geo.hkv, h = u - b * geo.hkv;
  const int T_ = geo.T(b);
  const int seg = sf.s0[b] + (int)blockIdx.y, start = seg * S;
  if (start >= T_) return;
  const int len = min(S, T_ - start);
  const int t0 = blockIdx.x * kTok;
  if (t0 >= len) return;
  const int ntok = min(kTok, len - t0);
  const int ncl = (len + cs - 1) / cs;
  const int64_t crow = geo.cl_row(b, h) + (int64_t)seg * (S / cs);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tx = tid & 15, ty = tid >> 4;
  const int sub = lane % R::LPR, rsub = lane / R::LPR;
  constexpr int LD = kTok + kPad;

  // keys of the tile, transposed into shared memory as fp32
  for (int r = warp * R::RPW + rsub; r < kTok; r += 8 * R::RPW) {
    float x[R::EPL];
#pragma unroll
    for (int e = 0; e < R::EPL; ++e) x[e] = 0.f;
    if (r < ntok) {
      const int64_t ro = pool_row(kin, geo.hkv, D, b, h, start + t0 + r, status);
      if (ro >= 0) {
        const uint4 raw = ld_stream(reinterpret_cast<const T*>(kin.base) + ro + sub * R::EPL);
        Elem<T>::unpack(raw, x);
      }
    }
#pragma unroll
    for (int e = 0; e < R::EPL; ++e) sk[(sub * R::EPL + e) * LD + r] = x[e];
  }

  float best[4];
  int besti[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) { best[i] = INFINITY; besti[i] = 0; }

  for (int cb = 0; cb < ncl; cb += kCen) {
    __syncthreads();
    // centroid tile, transposed (fp32 rows of D floats, 4 per lane per step)
    for (int idx = tid; idx < kCen * (D / 4); idx += blockDim.x) {
      const int j = idx / (D / 4), e4 = idx - j * (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (cb + j < ncl) v = *reinterpret_cast<const float4*>(cent32 + (crow + cb + j) * D + e4 * 4);
      sc[(e4 * 4 + 0) * LD + j] = v.x;
      sc[(e4 * 4 + 1) * LD + j] = v.y;
      sc[(e4 * 4 + 2) * LD + j] = v.z;
      sc[(e4 * 4 + 3) * LD + j] = v.w;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
    for (int e = 0; e < D; ++e) {
      const float4 a = *reinterpret_cast<const float4*>(sk + e * LD + ty * 4);
      const float4 c = *reinterpret_cast<const float4*>(sc + e * LD + tx * 4);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float df = av[i] - cv[j];
          acc[i][j] = fmaf(df, df, acc[i][j]);
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int cj = cb + tx * 4 + j;
      if (cj < ncl) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (acc[i][j] < best[i]) { best[i] = acc[i][j]; besti[i] = cj; }
      }
    }
  }
  // reduce over the 16 threads that share the same tokens (same ty)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best[i], o);
      const int oi = __shfl_xor_sync(0xffffffffu, besti[i], o);
      if (ob < best[i] || (ob == best[i] && oi < besti[i])) { best[i] = ob; besti[i] = oi; }
    }
  }
  if (tx == 0) {
    int32_t* dst = assign + geo.tok_row(b, h) + start + t0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (ty * 4 + i < ntok) dst[ty * 4 + i] = besti[i];
  }
}

// --------------------------------------------- assign on the tensor cores
// bf16 keys are exact in bf16, so ||k - c||^2 = ||c||^2 - 2 k.c + ||k||^2
// can take k.c from the tensor cores: the fp32 centroid c is split into two
// bf16 terms c1 + c2 (c1 = bf16(c), c2 = bf16(c - c1); the rest is below
// 2^-18 |c| elementwise) and k.c1 + k.c2 is accumulated in fp32 by tcgen05
// MMAs in tensor memory (the products of two bf16 values are exact in fp32).
//
// kmeans_split_kernel writes, once per round, every segment's centroids as
// the two terms' operand tiles (kUCen centroids x D, the MMA's K-major
// 128-byte-swizzled layout, one tile per (chunk of kUCen centroids, term);
// zero rows pad a segment's last chunk) and their ||c||^2 in fp32.
// kmeans_assign_umma_kernel takes kUTok tokens of a segment (the MMA's M)
// against every chunk of its centroids (the MMA's N): one warp streams the
// chunks' term tiles into a ring of shared-memory stages with bulk copies,
// one thread issues the MMAs (A = the keys, staged once; B = a term tile;
// both terms of a chunk accumulate into the chunk's kUCen columns of tensor
// memory, kUSlots chunks in flight), and four warps read each finished chunk
// back, one token row per thread, keeping each token's two smallest
// approximate distances a = ||c||^2 - 2 k.c.  Two CTAs share an SM, so one's
// loads and read-back overlap the other's MMAs.
//
// The decision is the direct form's: the FMA kernel above computes
// d = sum_e (k_e - c_e)^2 in fp32 (ascending e, fused multiply-add), and a
// token whose two best approximate distances are more than delta apart takes
// the best, since both |a - ||k - c||^2 + ||k||^2| errors are below
// delta / 2 (see the bound below); any other token (ties included)
// re-evaluates the direct form over all the segment's centroids, with the
// same arithmetic and the same tie rule (lower index), so the assignment
// equals the direct form's.
//
// Error bound, with |k.c| <= |k||c| <= (|k|^2 + |c|^2) / 2: the direct form
// sums D <= 128 terms, error <= 128 * 2^-24 * d <= 2^-16 (|k|^2 + |c|^2).
// The tensor-core sum adds 2 D <= 256 exact products, in whatever order,
// each addition within 2^-23 relative even if the accumulator truncates, so
// 2 k.c is off by at most 2 * 256 * 2^-23 (|k|^2 + |c|^2) / 2 =
// 2^-15 (|k|^2 + |c|^2); the split leaves 2 * 2^-18 |k||c| <=
// 2^-18 (|k|^2 + |c|^2); ||c||^2 in fp32 adds 128 * 2^-24 |c|^2: together
// below 2^-13 (|k|^2 + |c|^2).  delta = 2^-12 (|k|^2 + max |c|^2) leaves a
// factor of two.
constexpr int kUTok = 128;      // tokens per CTA: the MMA's M, one tensor-memory lane each
constexpr int kUCen = 128;      // centroids per chunk: the MMA's N
constexpr int kUTerms = 2;      // bf16 terms per centroid
constexpr int kUStages = 2;     // term tiles in flight
constexpr int kUSlots = 2;      // chunks accumulating at once: kUSlots * kUCen columns
constexpr int kUThreads = 192;  // warps 0..3 read the accumulators, 4 loads, 5 issues the MMAs

// byte offset of 16-byte chunk c of row r in a K-major, 128-byte-swizzled
// operand tile of `rows` rows: K blocks of 64 bf16, each rows x 128 bytes
__host__ __device__ __forceinline__ int mtile_off(int rows, int r, int c) {
  return (c >> 3) * (rows * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

// first chunk of (unit u, segment seg) among the operand tiles and norms
__host__ __device__ __forceinline__ int64_t cimg_chunk0(int u, int seg, int max_nseg, int nch) {
  return ((int64_t)u * max_nseg + seg) * nch;
}

template <int D>
__global__ void __launch_bounds__(256)
kmeans_split_kernel(const Geo geo, int S, int cs, const SegFrom sf, int max_nseg, int nch,
                    const float* __restrict__ cent32, unsigned char* __restrict__ cimg,
                    float* __restrict__ cn2) {
  constexpr int CH = D / 8;                 // 16-byte chunks of a bf16 row
  constexpr int CPB = 256 / CH;             // centroids per block
  static_assert(kUCen % CPB == 0, "blocks tile a chunk");
  constexpr size_t kTile = (size_t)kUCen * D * 2;
  const int u = blockIdx.z, b = u / geo.hkv, h = u - b * geo.hkv;
  const int T_ = geo.T(b);
  const int seg = sf.s0[b] + (int)blockIdx.y, start = seg * S;
  if (start >= T_) return;
  const int len = min(S, T_ - start);
  const int ncl = (len + cs - 1) / cs;
  const int j = blockIdx.x * CPB + (int)threadIdx.x / CH, c8 = (int)threadIdx.x % CH;
  const int64_t crow = geo.cl_row(b, h) + (int64_t)seg * (S / cs);
  float v[8];
  if (j < ncl) {
    const float4 lo = *reinterpret_cast<const float4*>(cent32 + (crow + j) * D + c8 * 8);
    const float4 hi = *reinterpret_cast<const float4*>(cent32 + (crow + j) * D + c8 * 8 + 4);
    v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
    v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = 0.f;
  }
  uint32_t w[kUTerms][4];
#pragma unroll
  for (int e = 0; e < 8; e += 2) split_bf16(v[e], v[e + 1], w[0][e / 2], w[1][e / 2]);
  const int64_t ch0 = cimg_chunk0(u, seg, max_nseg, nch);
  unsigned char* tiles = cimg + (ch0 + j / kUCen) * kUTerms * kTile;
#pragma unroll
  for (int t = 0; t < kUTerms; ++t)
    *reinterpret_cast<uint4*>(tiles + t * kTile + mtile_off(kUCen, j % kUCen, c8)) =
        make_uint4(w[t][0], w[t][1], w[t][2], w[t][3]);
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
#pragma unroll
  for (int o = 1; o < CH; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (c8 == 0) cn2[ch0 * kUCen + j] = ss;
}

template <int D>
__global__ void __launch_bounds__(kUThreads, 2)
kmeans_assign_umma_kernel(const Geo geo, const Pool kin, int S, int cs, const SegFrom sf,
                          int max_nseg, int nch, const unsigned char* __restrict__ cimg,
                          const float* __restrict__ cn2, const float* __restrict__ cent32,
                          int32_t* __restrict__ assign, uint32_t* status) {
  using T = __nv_bfloat16;
  constexpr int CH = D / 8;                                // 16-byte chunks per bf16 row
  constexpr uint32_t kTile = (uint32_t)kUCen * D * 2;      // a term tile (and the key tile)
  static_assert(kUTok == kUCen, "A and B tiles share their K-block stride");
  constexpr uint32_t kKBlock = (uint32_t)kUCen * 128;      // bytes between K blocks of 64 bf16
  constexpr uint32_t kIdesc = umma_idesc_bf16_f32<kUTok, kUCen>();
  constexpr int kRowsPerPass = kUThreads / CH;             // key rows staged per pass
  constexpr int kPasses = (kUTok + kRowsPerPass - 1) / kRowsPerPass;
  extern __shared__ unsigned char sh_umma_raw[];
  unsigned char* sk = align_smem_1024(sh_umma_raw);        // keys [kUTok][D], swizzled
  unsigned char* stg = sk + kTile;                         // kUStages term tiles
  __shared__ __align__(8) uint64_t s_full[kUStages], s_empty[kUStages];
  __shared__ __align__(8) uint64_t s_accf[kUSlots], s_acce[kUSlots], s_done;
  __shared__ __align__(16) float s_cn2[kUSlots][kUCen];   // the chunks' ||c||^2 (+inf past the segment)
  __shared__ uint32_t s_tmem;
  __shared__ float s_cmax2;
  __shared__ int s_namb;
  __shared__ int s_amb[kUTok];
  const int u = blockIdx.z, b = u / geo.hkv, h = u - b * geo.hkv;
  const int T_ = geo.T(b);
  const int seg = sf.s0[b] + (int)blockIdx.y, start = seg * S;
  if (start >= T_) return;
  const int len = min(S, T_ - start);
  const int t0 = blockIdx.x * kUTok;
  if (t0 >= len) return;
  const int ntok = min(kUTok, len - t0);
  const int ncl = (len + cs - 1) / cs;
  const int nchs = (ncl + kUCen - 1) / kUCen;              // this segment's chunks
  const int nst = kUTerms * nchs;                          // term tiles
  const int64_t crow = geo.cl_row(b, h) + (int64_t)seg * (S / cs);
  const int64_t ch0 = cimg_chunk0(u, seg, max_nseg, nch);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t ncols = nchs == 1 ? (uint32_t)kUCen : (uint32_t)(kUSlots * kUCen);

  if (tid == 0) {
    for (int i = 0; i < kUStages; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 1);
    }
    for (int i = 0; i < kUSlots; ++i) {
      mbar_init(&s_accf[i], 1);
      mbar_init(&s_acce[i], 4);
    }
    mbar_init(&s_done, 1);
    mbar_init_fence();
    s_cmax2 = 0.f;
    s_namb = 0;
  }
  if (warp == 5) tmem_alloc(&s_tmem, ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  // the first term tiles go out before the keys are staged
  const int npre = min(nst, kUStages);
  if (warp == 4 && lane == 0)
    for (int i = 0; i < npre; ++i) {
      mbar_arrive_expect(&s_full[i], kTile);
      bulk_load(stg + (size_t)i * kTile, cimg + (size_t)(ch0 * kUTerms + i) * kTile, kTile, &s_full[i]);
    }
  // the keys (zero rows past the segment), every row's page looked up
  // before any copy is issued; read by the MMAs through the async proxy
  {
    const int c = tid % CH;
    int64_t ro[kPasses];
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      const int r = tid / CH + p * kRowsPerPass;
      ro[p] = r < ntok ? pool_row(kin, geo.hkv, D, b, h, start + t0 + r, status) : -1;
    }
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      const int r = tid / CH + p * kRowsPerPass;
      if (r < kUTok) {
        unsigned char* dst = sk + mtile_off(kUTok, r, c);
        if (ro[p] >= 0) cp_async16(dst, reinterpret_cast<const T*>(kin.base) + ro[p] + c * 8);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    cp_async_commit();
    float m = 0.f;   // the largest ||c||^2 of the segment (norms are >= 0)
    for (int j = tid; j < ncl; j += kUThreads) m = fmaxf(m, __ldg(cn2 + ch0 * kUCen + j));
    atomicMax(reinterpret_cast<int*>(&s_cmax2), __float_as_int(m));
    cp_async_wait<0>();
  }
  fence_proxy_async();
  __syncthreads();

  if (warp == 4) {
    // ---- loads: term tile i = kUTerms c + t of chunk c into stage i % kUStages
    if (lane == 0) {
      int issued = npre;
      for (int i = npre; i < nst; ++i) {
        const int s = i % kUStages;
        if (!mbar_wait(&s_empty[s], (uint32_t)((i / kUStages) - 1) & 1u, status)) break;
        mbar_arrive_expect(&s_full[s], kTile);
        bulk_load(stg + (size_t)s * kTile, cimg + (size_t)(ch0 * kUTerms + i) * kTile, kTile, &s_full[s]);
        issued = i + 1;
      }
      // no copy is left in flight when the CTA ends
      for (int i = max(0, issued - kUStages); i < issued; ++i)
        mbar_wait(&s_full[i % kUStages], (uint32_t)(i / kUStages) & 1u, status);
    }
  } else if (warp == 5) {
    // ---- MMAs: chunk c into columns (c % kUSlots) kUCen .., once the
    // accumulators read back from them are free
    if (lane == 0) {
      const uint32_t a0 = smem_addr(sk);
      for (int c = 0; c < nchs; ++c) {
        const int slot = c % kUSlots;
        if (c >= kUSlots && !mbar_wait(&s_acce[slot], (uint32_t)((c / kUSlots) - 1) & 1u, status)) break;
        tc_fence_after();
        bool ok = true;
        for (int t = 0; t < kUTerms && ok; ++t) {
          const int i = kUTerms * c + t, s = i % kUStages;
          ok = mbar_wait(&s_full[s], (uint32_t)(i / kUStages) & 1u, status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t b0 = smem_addr(stg + (size_t)s * kTile);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {   // K = 16 per MMA: 32 bytes of each row
            const uint32_t ko = (uint32_t)(k >> 2) * kKBlock + (uint32_t)(k & 3) * 32u;
            umma_bf16(tmem + (uint32_t)(slot * kUCen), umma_desc_sw128(a0 + ko),
                      umma_desc_sw128(b0 + ko), kIdesc, (t | k) != 0);
          }
          umma_commit(&s_empty[s]);   // the stage is free once these MMAs are done
        }
        if (!ok) break;
        umma_commit(&s_accf[slot]);
      }
      // every MMA issued has completed before the columns are released
      umma_commit(&s_done);
      mbar_wait(&s_done, 0u, status);
    }
  } else {
    // ---- accumulators: token row r = 32 warp + lane, lane r of tensor memory
    const int r = 32 * warp + lane;
    float xn2 = 0.f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      float xv[8];
      Elem<T>::unpack(*reinterpret_cast<const uint4*>(sk + mtile_off(kUTok, r, c)), xv);
#pragma unroll
      for (int e = 0; e < 8; ++e) xn2 = fmaf(xv[e], xv[e], xn2);
    }
    // b1 <= b2: the two smallest a, i1: the index of b1 (equal values make
    // b2 == b1 and send the token to the direct form)
    float b1 = INFINITY, b2 = INFINITY;
    int i1 = 0;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
    for (int c = 0; c < nchs; ++c) {
      const int slot = c % kUSlots;
      {
        const int j = c * kUCen + r;
        s_cn2[slot][r] = j < ncl ? __ldg(cn2 + ch0 * kUCen + j) : INFINITY;
      }
      named_sync(1, 128);   // the chunk's norms (every reader of chunk c - kUSlots is past it)
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&s_accf[slot], (uint32_t)(c / kUSlots) & 1u, status));
      tc_fence_after();
      if (ok) {
#pragma unroll
        for (int q = 0; q < kUCen / 32; ++q) {
          float v[32];
          tmem_ld32(lane_base + (uint32_t)(slot * kUCen + 32 * q), v);
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 n4 = *reinterpret_cast<const float4*>(&s_cn2[slot][32 * q + 4 * e4]);
            const float nn[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float a = fmaf(-2.f, v[4 * e4 + e], nn[e]);
              i1 = a < b1 ? c * kUCen + 32 * q + 4 * e4 + e : i1;
              b2 = fminf(b2, fmaxf(b1, a));
              b1 = fminf(b1, a);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_acce[slot]);
    }
    int32_t* dst = assign + geo.tok_row(b, h) + start + t0;
    if (r < ntok) {
      const float delta = ldexpf(xn2 + s_cmax2, -12);
      if (b2 - b1 > delta) dst[r] = i1;
      else s_amb[atomicAdd(&s_namb, 1)] = r;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
  // near the decision boundary: the direct form over every centroid, as the
  // FMA kernel computes it (fp32, ascending e, lower index on ties)
  int32_t* dst = assign + geo.tok_row(b, h) + start + t0;
  const int namb = s_namb;
  for (int a = warp; a < namb; a += kUThreads / 32) {
    const int r = s_amb[a];
    float best = INFINITY;
    int bi = 0;
    for (int j = lane; j < ncl; j += 32) {
      const float* c = cent32 + (crow + j) * D;
      float acc = 0.f;
#pragma unroll 4
      for (int c8 = 0; c8 < CH; ++c8) {
        float xv[8];
        Elem<T>::unpack(*reinterpret_cast<const uint4*>(sk + mtile_off(kUTok, r, c8)), xv);
        const float4 lo = *reinterpret_cast<const float4*>(c + c8 * 8);
        const float4 hi = *reinterpret_cast<const float4*>(c + c8 * 8 + 4);
        const float cv[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float df = xv[e] - cv[e];
          acc = fmaf(df, df, acc);
        }
      }
      if (acc < best) { best = acc; bi = j; }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob < best || (ob == best && oi < bi)) { best = ob; bi = oi; }
    }
    if (lane == 0) dst[r] = bi;
  }
}

// ----------------------------------------------------------------- update
constexpr int kUpdThreads = 512;
constexpr int kUpdBatch = 8;   // cluster members whose rows are in flight together

struct FinalOut {
  void* centroids;
  void* value_sums;
  int32_t* offsets;
  int32_t* perm;
  int32_t* invperm;
  int32_t* labels;
  void* kout;
  void* vout;
  Pool pout;   // block table / geometry of the permuted pools
  Pool vin;
  int enabled;
};

template <typename T, int D>
__global__ void __launch_bounds__(kUpdThreads)
kmeans_update_kernel(const Geo geo, const Pool kin, int S, int cs, const SegFrom sf,
                     float* __restrict__ cent32, const int32_t* __restrict__ assign,
                     const FinalOut fo, uint32_t* status) {
  using R = BRow<T, D>;
  extern __shared__ int32_t sh_upd[];
  const int u = blockIdx.y, b = u / geo.hkv, h = u - b * geo.hkv;
  const int T_ = geo.T(b);
  const int seg = sf.s0[b] + (int)blockIdx.x, start = seg * S;
  if (start >= T_) return;
  const int len = min(S, T_ - start);
  const int ncl = (len + cs - 1) / cs;
  const int ncl_max = (S + cs - 1) / cs;
  int32_t* s_cur = sh_upd;                                      // [ncl_max] cursor
  int32_t* s_start = s_cur + ncl_max;                           // [ncl_max + 1]
  int32_t* s_scan = s_start + ncl_max + 1;                      // [32]
  uint16_t* s_asg = reinterpret_cast<uint16_t*>(s_scan + 32);   // [S]
  uint16_t* s_mem = s_asg + S;                                  // [S]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int64_t trow = geo.tok_row(b, h);
  const int64_t crow = geo.cl_row(b, h) + (int64_t)seg * (S / cs);

  for (int j = tid; j < ncl; j += blockDim.x) s_cur[j] = 0;
  __syncthreads();
  for (int i = tid; i < len; i += blockDim.x) {
    int a = assign[trow + start + i];
    if (a < 0 || a >= ncl) { flag_error(status, WI_DEV_BAD_CLUSTER); a = 0; }
    s_asg[i] = (uint16_t)a;
    atomicAdd(&s_cur[a], 1);
  }
  __syncthreads();
  // exclusive scan of the counts
  int run = 0;
  for (int base = 0; base < ncl; base += blockDim.x) {
    const int j = base + tid;
    const int c = j < ncl ? s_cur[j] : 0;
    int tot;
    const int incl = block_inclusive_scan(c, s_scan, &tot);
    if (j < ncl) s_start[j] = run + incl - c;
    run += tot;
  }
  if (tid == 0) s_start[ncl] = len;
  __syncthreads();
  for (int j = tid; j < ncl; j += blockDim.x) s_cur[j] = s_start[j];
  __syncthreads();
  // stable scatter: tokens in ascending order, warps in turn within a round
  for (int base = 0; base < len; base += blockDim.x) {
    const int t = base + tid;
    const unsigned act = __ballot_sync(0xffffffffu, t < len);
    for (int w = 0; w < nw; ++w) {
      if (warp == w && t < len) {
        const int bin = s_asg[t];
        const unsigned peers = __match_any_sync(act, bin);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        const int leader = __ffs(peers) - 1;
        int pos = 0;
        if (lane == leader) { pos = s_cur[bin]; s_cur[bin] = pos + __popc(peers); }
        pos = __shfl_sync(peers, pos, leader);
        s_mem[pos + rank] = (uint16_t)t;
      }
      __syncthreads();
    }
  }
  // means (fixed ascending-position order per cluster), final layout
  const int sub = lane % R::LPR, rsub = lane / R::LPR;
  const int groups = nw * R::RPW;
  const T* kb = reinterpret_cast<const T*>(kin.base) + sub * R::EPL;
  for (int j = warp * R::RPW + rsub; j < ncl; j += groups) {
    const int m0 = s_start[j], m1 = s_start[j + 1];
    // member sums in fp64: the stored mean / sum is then the correctly rounded
    // value of the exact one (the fp32 working centroid too)
    double ks[R::EPL], vs[R::EPL];
#pragma unroll
    for (int e = 0; e < R::EPL; ++e) { ks[e] = 0.0; vs[e] = 0.0; }
    // kUpdBatch members at a time: their pages looked up and their rows
    // loaded together, then summed in ascending position order
    for (int mb = m0; mb < m1; mb += kUpdBatch) {
      int p[kUpdBatch];
      int64_t ro[kUpdBatch];
      uint4 kraw[kUpdBatch];
#pragma unroll
      for (int q = 0; q < kUpdBatch; ++q) {
        p[q] = mb + q < m1 ? start + s_mem[mb + q] : -1;
        ro[q] = p[q] >= 0 ? pool_row(kin, geo.hkv, D, b, h, p[q], status) : -1;
      }
#pragma unroll
      for (int q = 0; q < kUpdBatch; ++q) kraw[q] = ro[q] >= 0 ? ld_stream(kb + ro[q]) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int q = 0; q < kUpdBatch; ++q) {
        if (ro[q] < 0) continue;
        float x[R::EPL];
        Elem<T>::unpack(kraw[q], x);
#pragma unroll
        for (int e = 0; e < R::EPL; ++e) ks[e] += (double)x[e];
      }
      if (fo.enabled) {
        int64_t vo[kUpdBatch], oo[kUpdBatch];
        uint4 vraw[kUpdBatch];
#pragma unroll
        for (int q = 0; q < kUpdBatch; ++q) {
          vo[q] = ro[q] >= 0 ? pool_row(fo.vin, geo.hkv, D, b, h, p[q], status) : -1;
          oo[q] = ro[q] >= 0 ? pool_row(fo.pout, geo.hkv, D, b, h, start + mb + q, status) : -1;
        }
#pragma unroll
        for (int q = 0; q < kUpdBatch; ++q)
          vraw[q] = vo[q] >= 0 ? ld_stream(reinterpret_cast<const T*>(fo.vin.base) + vo[q] + sub * R::EPL)
                               : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int q = 0; q < kUpdBatch; ++q) {
          if (ro[q] < 0) continue;
          const int slot = start + mb + q;
          float x[R::EPL];
          Elem<T>::unpack(vraw[q], x);
#pragma unroll
          for (int e = 0; e < R::EPL; ++e) vs[e] += (double)x[e];
          if (oo[q] >= 0) {
            *reinterpret_cast<uint4*>(reinterpret_cast<T*>(fo.kout) + oo[q] + sub * R::EPL) = kraw[q];
            *reinterpret_cast<uint4*>(reinterpret_cast<T*>(fo.vout) + oo[q] + sub * R::EPL) = vraw[q];
          }
          if (sub == 0) {
            fo.perm[trow + slot] = p[q];
            fo.invperm[trow + p[q]] = slot;
            fo.labels[trow + p[q]] = seg * (S / cs) + j;
          }
        }
      }
    }
    const int cnt = m1 - m0;
    float* c32 = cent32 + (crow + j) * D + sub * R::EPL;
    double mean[R::EPL];
#pragma unroll
    for (int e = 0; e < R::EPL; ++e) mean[e] = cnt > 0 ? ks[e] / (double)cnt : (double)c32[e];
    if (cnt > 0) {
#pragma unroll
      for (int e = 0; e < R::EPL; ++e) c32[e] = __double2float_rn(mean[e]);
    }
    if (fo.enabled) {
      T* cdst = reinterpret_cast<T*>(fo.centroids) + (crow + j) * D + sub * R::EPL;
      T* vdst = reinterpret_cast<T*>(fo.value_sums) + (crow + j) * D + sub * R::EPL;
#pragma unroll
      for (int e = 0; e < R::EPL; ++e) {
        store_elem(cdst + e, mean[e]);
        store_elem(vdst + e, vs[e]);
      }
      if (sub == 0) fo.offsets[geo.off_row(b, h) + seg * (S / cs) + j] = start + m0;
    }
  }
  if (fo.enabled && tid == 0 && start + len == T_) fo.offsets[geo.off_row(b, h) + geo.NC(b)] = T_;
}

// ------------------------------------------------------- position blocks
// The block index's assignment: token t of a segment belongs to block
// t / block_size of that segment (cs plays the block size).
__global__ void __launch_bounds__(kStreamThreads)
block_assign_kernel(const Geo geo, int S, int cs, int32_t* __restrict__ assign) {
  const int u = blockIdx.y, b = u / geo.hkv, h = u - b * geo.hkv;
  const int T_ = geo.T(b);
  const int64_t trow = geo.tok_row(b, h);
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T_; t += gridDim.x * blockDim.x)
    assign[trow + t] = (t % S) / cs;
}

// ----------------------------------------------------------- extension copy
// Unit blockIdx.y: the first s0 * S / cs clusters (centroid and value-sum
// rows, their offsets and the offset after them) and the first s0 * S tokens
// (perm, invperm, labels) of the old index, moved to the unit's rows of the
// new index.  Those segments are whole in both, so their slots, clusters and
// labels keep their numbers.
template <typename T, int D>
__global__ void __launch_bounds__(kStreamThreads)
extend_copy_kernel(const Geo gnew, const Geo gold, int S, int cs, const SegFrom sf,
                   const ExtendCopy c, void* __restrict__ centroids, void* __restrict__ value_sums,
                   int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
                   int32_t* __restrict__ invperm, int32_t* __restrict__ labels) {
  const int u = blockIdx.y, b = u / gnew.hkv, h = u - b * gnew.hkv;
  const int ncc = sf.s0[b] * (S / cs);          // clusters kept
  const int ntc = sf.s0[b] * S;                 // tokens kept
  constexpr int V = 16 / (int)sizeof(T);        // elements per 16-byte vector
  const int64_t ro = gold.cl_row(b, h) * D, rn = gnew.cl_row(b, h) * D;
  const int nvec = ncc * D / V;
  const int stride = gridDim.x * blockDim.x;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += stride) {
    reinterpret_cast<uint4*>(static_cast<T*>(centroids) + rn)[i] =
        reinterpret_cast<const uint4*>(static_cast<const T*>(c.centroids) + ro)[i];
    reinterpret_cast<uint4*>(static_cast<T*>(value_sums) + rn)[i] =
        reinterpret_cast<const uint4*>(static_cast<const T*>(c.value_sums) + ro)[i];
  }
  const int64_t oo = gold.off_row(b, h), on = gnew.off_row(b, h);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= ncc; i += stride)
    offsets[on + i] = c.offsets[oo + i];
  const int64_t to = gold.tok_row(b, h), tn = gnew.tok_row(b, h);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < ntc; i += stride) {
    perm[tn + i] = c.perm[to + i];
    invperm[tn + i] = c.invperm[to + i];
    labels[tn + i] = c.labels[to + i];
  }
}

template <typename F>
cudaError_t with_build_types(int dtype, int D, F&& f) {
  if (dtype == WI_BF16) {
    if (D == 128) return f.template operator()<__nv_bfloat16, 128>();
    if (D == 64) return f.template operator()<__nv_bfloat16, 64>();
  } else {
    if (D == 128) return f.template operator()<float, 128>();
    if (D == 64) return f.template operator()<float, 64>();
  }
  return cudaErrorInvalidValue;
}

size_t assign_smem(int D) { return (size_t)D * ((kTok + kPad) + (kCen + kPad)) * sizeof(float); }
size_t assign_umma_smem(int D) { return 1024 + (size_t)(1 + kUStages) * kUCen * D * 2; }

// One assignment pass over every unit's segments: the tensor-core kernels
// for bf16 keys (the centroids' operand tiles, then the assignment), the
// fp32 direct form otherwise.
template <typename T, int D>
cudaError_t launch_assign(const BuildPlan& p, const Pool& kin, const float* cent32,
                          int32_t* assign, unsigned char* ws, uint32_t* status, cudaStream_t s) {
  if constexpr (std::is_same_v<T, __nv_bfloat16>) {
    unsigned char* cimg = ws + p.off_cimg;
    float* cn2 = reinterpret_cast<float*>(ws + p.off_cn2);
    kmeans_split_kernel<D><<<dim3(p.nch * kUCen / (256 / (D / 8)), p.nseg_grid, p.U), 256, 0, s>>>(
        p.geo, p.S, p.cs, p.sf, p.max_nseg, p.nch, cent32, cimg, cn2);
    const size_t smem = assign_umma_smem(D);
    cudaFuncSetAttribute(kmeans_assign_umma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    const dim3 grid((p.S + kUTok - 1) / kUTok, p.nseg_grid, p.U);
    kmeans_assign_umma_kernel<D><<<grid, kUThreads, smem, s>>>(
        p.geo, kin, p.S, p.cs, p.sf, p.max_nseg, p.nch, cimg, cn2, cent32, assign, status);
  } else {
    const size_t smem = assign_smem(D);
    cudaFuncSetAttribute(kmeans_assign_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    const dim3 grid((p.S + kTok - 1) / kTok, p.nseg_grid, p.U);
    kmeans_assign_kernel<T, D><<<grid, 256, smem, s>>>(p.geo, kin, p.S, p.cs, p.sf, cent32,
                                                       assign, status);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_assign_only(const BuildPlan& p, const BuildArgs& a, const float* cent32,
                               int32_t* assign, cudaStream_t s) {
  uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + p.off_status);
  return with_build_types(p.dtype, p.D, [&]<typename T, int D>() -> cudaError_t {
    return launch_assign<T, D>(p, a.kin, cent32, assign, a.ws, status, s);
  });
}

cudaError_t launch_build(const BuildPlan& p, const BuildArgs& a, cudaStream_t s) {
  uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + p.off_status);
  float* cent32 = reinterpret_cast<float*>(a.ws + p.off_cent32);
  int32_t* assign = reinterpret_cast<int32_t*>(a.ws + p.off_assign);
  return with_build_types(p.dtype, p.D, [&]<typename T, int D>() -> cudaError_t {
    cudaFuncSetAttribute(kmeans_update_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)p.update_smem);
    if (p.nseg_grid < 1) return cudaSuccess;   // nothing new to cluster
    kmeans_init_kernel<T, D><<<dim3(p.nseg_grid, p.U), kStreamThreads, 0, s>>>(
        p.geo, a.kin, p.S, p.cs, p.sf, cent32, status);
    FinalOut none{};
    none.enabled = 0;
    FinalOut fin{};
    fin.centroids = a.centroids;
    fin.value_sums = a.value_sums;
    fin.offsets = a.offsets;
    fin.perm = a.perm;
    fin.invperm = a.invperm;
    fin.labels = a.labels;
    fin.kout = a.kout;
    fin.vout = a.vout;
    fin.pout = Pool{a.kout, a.bt_out, a.n_pages_out, a.max_pages_out, a.page_shift_out};
    fin.vin = a.vin;
    fin.enabled = 1;
    for (int it = 0; it < p.iters; ++it) {
      const cudaError_t ea = launch_assign<T, D>(p, a.kin, cent32, assign, a.ws, status, s);
      if (ea != cudaSuccess) return ea;
      kmeans_update_kernel<T, D><<<dim3(p.nseg_grid, p.U), kUpdThreads, p.update_smem, s>>>(
          p.geo, a.kin, p.S, p.cs, p.sf, cent32, assign, it == p.iters - 1 ? fin : none, status);
    }
    return cudaGetLastError();
  });
}

cudaError_t launch_blocks(const BuildPlan& p, const BuildArgs& a, cudaStream_t s) {
  uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + p.off_status);
  float* cent32 = reinterpret_cast<float*>(a.ws + p.off_cent32);
  int32_t* assign = reinterpret_cast<int32_t*>(a.ws + p.off_assign);
  return with_build_types(p.dtype, p.D, [&]<typename T, int D>() -> cudaError_t {
    cudaFuncSetAttribute(kmeans_update_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)p.update_smem);
    block_assign_kernel<<<dim3(64, p.U), kStreamThreads, 0, s>>>(p.geo, p.S, p.cs, assign);
    FinalOut fin{};
    fin.centroids = a.centroids;
    fin.value_sums = a.value_sums;
    fin.offsets = a.offsets;
    fin.perm = a.perm;
    fin.invperm = a.invperm;
    fin.labels = a.labels;
    fin.kout = a.kout;
    fin.vout = a.vout;
    fin.pout = Pool{a.kout, a.bt_out, a.n_pages_out, a.max_pages_out, a.page_shift_out};
    fin.vin = a.vin;
    fin.enabled = 1;
    kmeans_update_kernel<T, D><<<dim3(p.nseg_grid, p.U), kUpdThreads, p.update_smem, s>>>(
        p.geo, a.kin, p.S, p.cs, p.sf, cent32, assign, fin, status);
    return cudaGetLastError();
  });
}

cudaError_t launch_extend_copy(const BuildPlan& p, const ExtendCopy& c, const BuildArgs& a,
                               cudaStream_t s) {
  return with_build_types(p.dtype, p.D, [&]<typename T, int D>() -> cudaError_t {
    extend_copy_kernel<T, D><<<dim3(16, p.U), kStreamThreads, 0, s>>>(
        p.geo, c.gold, p.S, p.cs, p.sf, c, a.centroids, a.value_sums, a.offsets, a.perm,
        a.invperm, a.labels);
    return cudaGetLastError();
  });
}

}  // namespace wi

// Shared device helpers for the wave-index kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "wi.h"

namespace wi {

constexpr int kMaxBatch = WI_MAX_BATCH;
constexpr int kWarp = 32;

// Ragged per-call geometry, passed to kernels by value (about 2 KB).
struct Geo {
  int32_t batch, hkv, d;
  int32_t tok_base[kMaxBatch + 1];  // prefix sums of T_b
  int32_t cl_base[kMaxBatch + 1];   // prefix sums of NC_b

  __host__ __device__ __forceinline__ int T(int b) const { return tok_base[b + 1] - tok_base[b]; }
  __host__ __device__ __forceinline__ int NC(int b) const { return cl_base[b + 1] - cl_base[b]; }
  // first cluster row of unit (b,h) in centroid / score / key arrays
  __host__ __device__ __forceinline__ int64_t cl_row(int b, int h) const {
    return (int64_t)cl_base[b] * hkv + (int64_t)h * NC(b);
  }
  // first entry of unit (b,h) in the offsets array (NC_b + 1 entries per unit)
  __host__ __device__ __forceinline__ int64_t off_row(int b, int h) const {
    return ((int64_t)cl_base[b] + b) * hkv + (int64_t)h * (NC(b) + 1);
  }
  // first entry of unit (b,h) in token-indexed arrays (perm, invperm, assign)
  __host__ __device__ __forceinline__ int64_t tok_row(int b, int h) const {
    return (int64_t)tok_base[b] * hkv + (int64_t)h * T(b);
  }
};

// A paged pool [n_pages][hkv][page][d] addressed through a block table.
struct Pool {
  const void* base;
  const int32_t* bt;
  int64_t n_pages;
  int32_t max_pages;
  int32_t page_shift;  // log2(page_size)
};

// Status word in the first bytes of every workspace.
__device__ __forceinline__ void flag_error(uint32_t* status, uint32_t bit) {
  atomicOr(status, bit);
}

// Element offset of row `slot` of unit (b,h) in a pool, or -1 (and a status
// bit) when the block table points outside the pool.
__device__ __forceinline__ int64_t pool_row(const Pool& p, int hkv, int d, int b, int h, int slot,
                                            uint32_t* status) {
  const int lp = slot >> p.page_shift;
  if (slot < 0 || lp >= p.max_pages) {
    flag_error(status, WI_DEV_BAD_SLOT);
    return -1;
  }
  const int pg = __ldg(p.bt + (int64_t)b * p.max_pages + lp);
  if (pg < 0 || (int64_t)pg >= p.n_pages) {
    flag_error(status, WI_DEV_BAD_PAGE);
    return -1;
  }
  const int row = slot & ((1 << p.page_shift) - 1);
  return ((((int64_t)pg * hkv + h) << p.page_shift) + row) * d;
}

// pool_row with the page lookup supplied: `pg` is the block-table entry of
// the slot's logical page (read earlier, e.g. staged in shared memory)
__device__ __forceinline__ int64_t pool_row_pg(const Pool& p, int hkv, int d, int h, int slot, int pg,
                                               uint32_t* status) {
  const int lp = slot >> p.page_shift;
  if (slot < 0 || lp >= p.max_pages) {
    flag_error(status, WI_DEV_BAD_SLOT);
    return -1;
  }
  if (pg < 0 || (int64_t)pg >= p.n_pages) {
    flag_error(status, WI_DEV_BAD_PAGE);
    return -1;
  }
  const int row = slot & ((1 << p.page_shift) - 1);
  return ((((int64_t)pg * hkv + h) << p.page_shift) + row) * d;
}

// Hint: bring the 128-byte line holding ptr into L2.
__device__ __forceinline__ void prefetch_l2(const void* ptr) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}

// 16-byte streaming load (read-only path, no L1 allocation).
__device__ __forceinline__ uint4 ld_stream(const void* ptr) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr));
  return r;
}

// Element traits: how a 16-byte vector unpacks into floats.
template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kPerVec = 4;
  __device__ __forceinline__ static void unpack(const uint4& v, float* x) {
    x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static float from_float(float f) { return f; }
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  __device__ __forceinline__ static void unpack(const uint4& v, float* x) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

__device__ __forceinline__ void store_elem(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
// Round-to-nearest-even from double straight to the storage type (no double rounding).
__device__ __forceinline__ void store_elem(float* p, double v) { *p = __double2float_rn(v); }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, double v) { *p = __double2bfloat16(v); }

// Order-preserving map of a float to uint32 (larger float -> larger key).
// Key 0 is reserved for "not a candidate".
__device__ __forceinline__ uint32_t ordered_key(float f) {
  const uint32_t u = __float_as_uint(f);
  const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return k == 0u ? 1u : k;
}

// Sum N values across groups of L consecutive lanes (N <= L, both powers of
// two) with log2(L) shuffle rounds and N-1+log2(L/N) shuffles in total: each
// round halves the values a lane keeps (it keeps the half selected by its
// lane bit and receives the partner's copy of that half).  Afterwards v[0] of
// every lane holds the group's full sum of value index j = (lane % L) / (L / N).
template <int N, int O>
struct GroupReduce {
  __device__ __forceinline__ static void run(float* v, int lane) {
    if constexpr (O >= 1) {
      const bool hi = (lane & O) != 0;
      if constexpr (N > 1) {
#pragma unroll
        for (int i = 0; i < N / 2; ++i) {
          const float keep = hi ? v[i + N / 2] : v[i];
          const float send = hi ? v[i] : v[i + N / 2];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
        }
        GroupReduce<N / 2, O / 2>::run(v, lane);
      } else {
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
        GroupReduce<1, O / 2>::run(v, lane);
      }
    }
  }
};

template <int N, int L>
__device__ __forceinline__ void group_reduce_multi(float (&v)[N], int lane) {
  static_assert(N >= 1 && N <= L && L <= 32, "bad reduce shape");
  GroupReduce<N, L / 2>::run(v, lane);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Named barrier `id` over the first `n` threads of the CTA (a multiple of 32);
// id 0 is __syncthreads' barrier.
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Release / acquire fence at GPU scope: the writes this thread has made or
// observed (a CTA barrier before it included) are visible GPU-wide before
// its later writes (a counter it then increments); for the thread that
// reads the last increment, the others' published writes are visible after
// it.
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Arrive at named barrier `id` (n threads in all) without waiting.
__device__ __forceinline__ void named_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Loads of data other CTAs of the same grid wrote (L2, bypassing L1).
__device__ __forceinline__ int ldcg_i32(const int32_t* p) { return __ldcg(p); }
__device__ __forceinline__ uint32_t ldcg_u32(const uint32_t* p) { return __ldcg(p); }

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue now / wait until the previous kernel's results are visible.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// 16-byte asynchronous global -> shared copy (L2 only) and its group fences.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
// 4-byte asynchronous copy (any 4-byte aligned address), cached at all levels.
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// The first 1024-byte boundary at or after p, a shared-memory pointer: the
// offset is added to p itself (not computed through an integer round trip),
// so the compiler keeps the shared address space and emits shared-memory
// instructions for every access through the result.
__device__ __forceinline__ unsigned char* align_smem_1024(unsigned char* p) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// ---- bulk (TMA) copies into shared memory, completed on an mbarrier
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
// make initialised barriers visible to the async proxy
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// arrive once and expect `bytes` of transactions in the current phase
__device__ __forceinline__ void mbar_arrive_expect(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
constexpr uint32_t kSpinLimit = 1u << 22;   // try_wait rounds before a wait gives up
// wait for phase `parity` of the barrier to complete; false (and a status
// bit) when the bounded wait gives up
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    if (ok) return true;
  }
  atomicOr(status, 0x10u);  // WI_DEV_TIMEOUT
  return false;
}
// generic-proxy accesses of shared memory before async-proxy writes to it
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// 2-D tiled bulk copy through a tensor map (box at element coordinates
// x = column, y = row; x * element size must be a multiple of 16 bytes)
__device__ __forceinline__ void tensor_load_2d(void* smem, const void* tmap, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(smem)), "l"(tmap), "r"(x), "r"(y),
      "r"(smem_addr(bar)) : "memory");
}

// 1-D tiled bulk copy through a tensor map (box at element coordinate x;
// x * element size a multiple of 16 bytes)
__device__ __forceinline__ void tensor_load_1d(void* smem, const void* tmap, int x, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.1d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2}], [%3];" ::"r"(smem_addr(smem)), "l"(tmap), "r"(x), "r"(smem_addr(bar))
      : "memory");
}

// ---- warp-level bf16 tensor-core fragments (m16n8k16, fp32 accumulate)
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* smem) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_addr(smem)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* smem) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_addr(smem)));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t (&r)[2], const void* smem) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1]) : "r"(smem_addr(smem)));
}
// d += a * b with a = {a0, 0, a2, 0} (rows 8..15 of A are zero)
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9},"
      " {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
// d += a * b with all four A registers: a0 / a2 rows 0..7, a1 / a3 rows
// 8..15 (k 0..7 / 8..15 of each)
__device__ __forceinline__ void mma_bf16_4(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                           uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9},"
      " {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// d += a * b, m16n8k8 (bf16 in, fp32 accumulate): a0 rows 0..7 and a1 rows
// 8..15 of A (k 2t, 2t+1 of thread t % 4), b0 the k-pair of column t / 4
__device__ __forceinline__ void mma_bf16_k8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6},"
      " {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}
// two floats as a bf16 pair (round to nearest even), low element first
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// w = hi + lo as two bf16 pairs (the split keeps ~16 bits of w)
__device__ __forceinline__ void split_bf16(float w0, float w1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(w0, w1);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(w0 - hf.x, w1 - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}
// byte offset of (row r, 16-byte chunk c) in a 128-byte-swizzled box of
// 128-byte rows (the layout a SWIZZLE_128B tensor copy writes)
__device__ __forceinline__ int swz128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

// bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
__device__ __forceinline__ void bulk_load(void* smem, const void* gmem, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(smem)), "l"(gmem), "r"(bytes), "r"(smem_addr(bar)) : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Wait until at most n of this thread's cp.async groups are pending (n <= 7).
__device__ __forceinline__ void cp_async_wait_dyn(int n) {
  switch (n) {
    case 0: cp_async_wait<0>(); break;
    case 1: cp_async_wait<1>(); break;
    case 2: cp_async_wait<2>(); break;
    case 3: cp_async_wait<3>(); break;
    case 4: cp_async_wait<4>(); break;
    case 5: cp_async_wait<5>(); break;
    case 6: cp_async_wait<6>(); break;
    default: cp_async_wait<7>(); break;
  }
}

// Dot products of one 16-byte vector (EPL elements, already fp32) with G
// query slices, two lanes of packed fp32 FMA (sm_100 FFMA2) at a time.
template <int G, int EPL>
__device__ __forceinline__ void dot_g(const float (&qv)[G][EPL], const float (&x)[EPL],
                                      float (&acc)[G]) {
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float2 a = make_float2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < EPL; e += 2)
      a = __ffma2_rn(make_float2(qv[g][e], qv[g][e + 1]), make_float2(x[e], x[e + 1]), a);
    acc[g] = a.x + a.y;
  }
}

// acc[g][e] += w[g] * x[e] with packed fp32 FMA.
template <int G, int EPL>
__device__ __forceinline__ void axpy_g(const float (&w)[G], const float (&x)[EPL],
                                       float (&acc)[G][EPL]) {
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL; e += 2) {
      const float2 r = __ffma2_rn(make_float2(w[g], w[g]), make_float2(x[e], x[e + 1]),
                                  make_float2(acc[g][e], acc[g][e + 1]));
      acc[g][e] = r.x;
      acc[g][e + 1] = r.y;
    }
}

// Inclusive scan of two ints per thread over the block (as block_inclusive_scan).
// `sh` needs 64 ints.
__device__ __forceinline__ int2 block_inclusive_scan2(int2 x, int* sh, int2* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ya = __shfl_up_sync(0xffffffffu, x.x, o);
    const int yb = __shfl_up_sync(0xffffffffu, x.y, o);
    if (lane >= o) { x.x += ya; x.y += yb; }
  }
  if (lane == 31) { sh[w] = x.x; sh[32 + w] = x.y; }
  __syncthreads();
  if (w == 0) {
    int a = lane < nw ? sh[lane] : 0, c = lane < nw ? sh[32 + lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, a, o);
      const int yc = __shfl_up_sync(0xffffffffu, c, o);
      if (lane >= o) { a += ya; c += yc; }
    }
    sh[lane] = a; sh[32 + lane] = c;
  }
  __syncthreads();
  const int2 r = make_int2(x.x + (w > 0 ? sh[w - 1] : 0), x.y + (w > 0 ? sh[32 + w - 1] : 0));
  *total = make_int2(sh[nw - 1], sh[32 + nw - 1]);
  __syncthreads();
  return r;
}

// Inclusive scan of one int per thread over the block (blockDim.x multiple of
// 32, <= 1024).  `sh` needs 32 ints.  Returns the inclusive prefix; *total
// receives the block sum.  Contains __syncthreads.
__device__ __forceinline__ int block_inclusive_scan(int x, int* sh, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = lane < nw ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    sh[lane] = s;
  }
  __syncthreads();
  const int r = x + (w > 0 ? sh[w - 1] : 0);
  *total = sh[nw - 1];
  __syncthreads();
  return r;
}

}  // namespace wi

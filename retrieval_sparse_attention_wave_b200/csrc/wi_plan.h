// Host-side launch plans for the wave-index kernels: the geometry of one call,
// the launch shapes, and where each workspace region lives.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cstring>

#include "wi_common.cuh"

namespace wi {

constexpr int kStreamThreads = 256;   // build kernels: 8 warps
constexpr int kNumSMs = 148;          // B200

// Decode kernels.  A tile is 64 rows (centroid / value-sum rows in the scan,
// gathered key / value rows in the gather); each of 8 consumer warps takes 8.
constexpr int kTileRows = 64;
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = 32 * kConsumerWarps;   // 256 consumer threads
constexpr int kScanThreads = kConsumers + 32;     // + one producer warp
constexpr int kGatherThreads = kConsumers;
constexpr int kGatherTiles = 2;                   // tiles per gather block (128 rows)
constexpr int kGatherRows = kGatherTiles * kTileRows;   // rows per gather block
constexpr int kInfoInts = 16;                     // per-unit record (see wi_decode_layout)
constexpr int kHistBins = 2048;                   // first radix digit: key bits 31..21
constexpr int kTailCand = 1024;                   // threshold-bin members refined in shared memory
constexpr int kMaxGatherPerUnit = 64;             // gather CTAs per unit (they loop beyond)
constexpr int kMaxTailsPerCta = 64;               // units one scan CTA may touch

// The scan's work: the clusters of every unit that is not attended densely,
// in chunks of kTileRows; sequence b's units own ch_base[b + 1] - ch_base[b]
// chunks (Hkv units of equal count).  Scan CTA s takes the chunks
// [k0s[s], k0s[s + 1]): contiguous runs in order, at least one chunk each,
// sized on the host (balance_scan in the plan).
struct ChunkMap {
  int32_t ch_base[kMaxBatch + 1];
  int n_chunks, n_scan, batch, hkv;
  int32_t k0s[kNumSMs + 1];
  __host__ __device__ __forceinline__ int k0(int s) const { return k0s[s]; }
  // the CTA of chunk k in a table of first chunks (the last s with tab[s] <= k)
  __host__ __device__ __forceinline__ static int cta_in(const int32_t* tab, int n_scan, int k) {
    int lo = 0, hi = n_scan - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tab[mid] <= k) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
  __host__ __device__ __forceinline__ int cta_of(int k) const { return cta_in(k0s, n_scan, k); }
  __host__ __device__ __forceinline__ int seq_of(int k) const {
    int lo = 0, hi = batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (ch_base[mid] <= k) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
  __host__ __device__ __forceinline__ int per_unit(int b) const {
    return (int)((uint32_t)(ch_base[b + 1] - ch_base[b]) / (uint32_t)hkv);
  }
  __host__ __device__ __forceinline__ int first(int b, int h) const { return ch_base[b] + h * per_unit(b); }
  // scan parts (CTAs) of unit (b, h): the CTAs of its first and last chunk and between
  __host__ __device__ __forceinline__ int parts(int b, int h) const {
    const int n = per_unit(b);
    return n == 0 ? 0 : cta_of(first(b, h) + n - 1) - cta_of(first(b, h)) + 1;
  }
};

// Per-unit record fields (int32 [U][kInfoInts]).
enum UnitField {
  kSelCount = 0,   // retrieved clusters (tail)
  kThrKey = 1,     // k-th key, 0xFFFFFFFF when nothing is retrieved (tail)
  kThrIdx = 2,     // largest id taken at the k-th key (tail)
  kSelTokens = 3,  // token rows of the retrieved clusters (tail)
  kSteady = 4,     // steady slots (steady kernel; T_b for a dense unit)
  kAffected = 5,   // clusters holding a steady token (steady kernel)
  kDense = 6,      // 1: attended densely (steady kernel)
  kCandidates = 7, // candidate clusters (tail)
  kFullRows = 8,   // clusters whose estimate is taken back out (tail)
  kPartRows = 9,   // steady tokens of candidate clusters (steady kernel)
  kNonCand = 10,   // clusters left without a non-steady token (steady kernel)
  kNoEstimate = 11,// 1: the estimation zone is empty (tail)
  kMode = 12,      // selection mode (0 exact, 1 sampled threshold bin)
  kSampBin = 13,   // sampled mode: the threshold bin
  kSampHash = 14,  // sampled mode: high 32 bits of the last draw taken ...
  kSampHashLo = 15 // ... and its low 32 bits (the id is kThrIdx)
};

struct DecodePlan {
  int exact_only;          // no estimation zone (block top-k workload)
  int mode;                // 0 exact top-k, 1 sampled threshold bin
  uint32_t seed;           // draws of the sampled mode
  Geo geo;
  int dtype, D, G, Hq, U;
  int n_sink, window, topk_clusters;
  double topk_fraction;
  float scale;             // 1/sqrt(d)
  int max_nc;
  int cap;                 // steady slots per unit (>= 1)
  int64_t ncl;             // centroid rows of the index (Hkv * sum NC_b)
  int64_t ntok;            // token rows of the index (Hkv * sum T_b)
  // scan (K1): chunks of kTileRows clusters of the units that are not dense
  int32_t ch_base[kMaxBatch + 1];   // chunk prefix over sequences (Hkv chunks-per-unit each)
  int n_chunks, n_scan, p1max;      // total chunks, scan CTAs, parts per unit at most
  int32_t k0s[kNumSMs + 1];         // first chunk of each scan CTA (ChunkMap)
  int slots;                        // ring slots per scan CTA
  // gather (K2): per sequence n2_b CTAs per unit
  int32_t n2_base[kMaxBatch + 1];   // CTA prefix over sequences (Hkv * n2_b each)
  int n_gather, n2max;
  // workspace byte offsets; [0, off_rec) must be zero before the first call
  size_t off_status, off_cnt1, off_cnt2, off_hist;
  size_t off_rec, off_info, off_st_slot, off_pc, off_nonc, off_sel, off_tok, off_selinfo;
  size_t off_est, off_gat, off_q, off_out, off_lse;
  size_t total;
};

// The scan's chunk map of a plan.
inline ChunkMap chunk_map(const DecodePlan& p) {
  ChunkMap cm;
  std::memcpy(cm.ch_base, p.ch_base, sizeof(cm.ch_base));
  cm.n_chunks = p.n_chunks;
  cm.n_scan = p.n_scan > 0 ? p.n_scan : 1;
  cm.batch = p.geo.batch;
  cm.hkv = p.geo.hkv;
  std::memcpy(cm.k0s, p.k0s, sizeof(cm.k0s));
  return cm;
}
// First segment each sequence's build kernels process (all zero for a full
// build; an index extension starts at the old index's first incomplete one).
struct SegFrom {
  int32_t s0[kMaxBatch];
};

struct BuildPlan {
  Geo geo;
  int dtype, D, U, S, cs, iters;
  int max_nseg, max_ncl_seg;
  SegFrom sf;              // first segment per sequence
  int nseg_grid;           // max over sequences of (segments - first segment)
  size_t update_smem;
  int nch;                 // chunks of 128 centroids per segment (tensor-core assignment)
  size_t off_status, off_cent32, off_assign;
  size_t off_cimg, off_cn2;  // bf16 keys: the centroids' operand tiles and squared norms
  size_t total;
};

// Pointers of one decode call.
struct DecodeArgs {
  const void* q;
  const void* centroids;
  const void* value_sums;
  const int32_t* offsets;
  const int32_t* perm;
  const int32_t* invperm;
  const int32_t* labels;
  Pool kp, vp;
  float* out;
  float* lse;
  unsigned char* ws;
  cudaEvent_t* stage_events;
  float* scores_out;       // optional [ncl][G] per-head centroid scores
};

struct BuildArgs {
  Pool kin, vin;
  // outputs (index); null pointers for the assign-only entry
  void* centroids;
  void* value_sums;
  int32_t* offsets;
  int32_t* perm;
  int32_t* invperm;
  int32_t* labels;
  void* kout;
  void* vout;
  const int32_t* bt_out;
  int64_t n_pages_out;
  int32_t max_pages_out;
  int32_t page_shift_out;
  unsigned char* ws;
};

constexpr int kDecodeStages = 3;
extern const char* const kDecodeStageNames[kDecodeStages];

cudaError_t launch_decode(const DecodePlan& p, const DecodeArgs& a, cudaStream_t s);
wi_status decode_workspace_extent(const wi_index* idx, const wi_decode_params* p, size_t* total,
                                  size_t* zero_prefix);
// shared memory of the decode kernels (host plan checks)
size_t decode_scan_smem(int dtype, int D, int G, int slots, int exact_only);
size_t decode_gather_smem(int dtype, int D, int G);
size_t decode_steady_smem(int cap);
size_t decode_scan_slot_bytes(int dtype, int D, int G, int exact_only);
cudaError_t launch_build(const BuildPlan& p, const BuildArgs& a, cudaStream_t s);
// Position-block index: each token's cluster is its block inside its segment,
// then one finalizing update pass.
cudaError_t launch_blocks(const BuildPlan& p, const BuildArgs& a, cudaStream_t s);
// Copy the part of an old index that an extension keeps (segments below
// p.sf.s0[b]) into the new index's buffers: centroid and value-sum rows,
// offsets, perm, invperm and labels.
struct ExtendCopy {
  Geo gold;
  const void* centroids;
  const void* value_sums;
  const int32_t* offsets;
  const int32_t* perm;
  const int32_t* invperm;
  const int32_t* labels;
};
cudaError_t launch_extend_copy(const BuildPlan& p, const ExtendCopy& c, const BuildArgs& a,
                               cudaStream_t s);
cudaError_t launch_assign_only(const BuildPlan& p, const BuildArgs& a, const float* cent32,
                               int32_t* assign, cudaStream_t s);

}  // namespace wi

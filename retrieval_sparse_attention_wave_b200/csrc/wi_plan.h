// Host-side launch plans for the wave-index kernels: the geometry of one call,
// the launch shapes, and where each workspace region lives.
#pragma once

#include <cstddef>
#include <cstdint>

#include "wi_common.cuh"

namespace wi {

constexpr int kStreamThreads = 256;   // streaming kernels: 8 warps
constexpr int kTopkThreads = 512;     // one CTA per unit
constexpr int kAttendTile = 64;       // tokens per exact-attention tile
constexpr int kInfoInts = 8;          // per-unit info record (see wi_decode_layout)
constexpr int kNumSMs = 148;          // B200
constexpr int kScoreChunkBytes = 32768;  // centroid bytes (and as many value-sum bytes) per score CTA
constexpr int kFold = 16;             // score-chunk parts folded into one by an attend fold CTA
constexpr int kRangeClusters = 256;   // cluster ids per attend range CTA (one per thread)

struct DecodePlan {
  int exact_only;          // no estimation zone (block top-k workload)
  Geo geo;
  int dtype, D, G, Hq, U;
  int n_sink, window, topk_clusters;
  double topk_fraction;
  int max_nc;
  int64_t ncl;               // centroid rows of the index (Hkv * sum NC_b)
  int seg_len, seg_clusters;  // segment length and clusters per full segment
  int score_chunk, n_score_blocks;   // clusters per score CTA, score CTAs per unit
  int cap;                 // steady-list capacity per unit (>= 1)
  int sort_pow2;           // shared-memory sort size for the steady list
  int n_rng;               // attend range CTAs per unit (kRangeW cluster ids each)
  int n_sc;                // attend steady CTAs per unit (two tiles of steady slots each)
  int n_fold;              // fold CTAs per unit (kFold score parts each)
  int n_parts;             // n_rng + n_sc + n_fold softmax parts per (unit, head)
  float scale;             // 1/sqrt(d)
  // workspace byte offsets; [0, off_scores) must be zero before the first call
  size_t off_status, off_counters, off_hist, off_aff_of;
  size_t off_scores, off_keys, off_sel, off_info;
  int sel_words;           // selection bitmap words per unit (kRangeClusters / 32 per range CTA)
  size_t off_st_slot, off_st_cl, off_aff_cl, off_aff_start, off_partials;
  size_t off_dv, off_est, off_nonc;
  size_t off_q, off_out, off_lse;
  size_t total;
};

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
  size_t off_status, off_cent32, off_assign;
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
size_t decode_attend_smem(int dtype, int D, int G, int n_parts);
size_t decode_score_smem(int dtype, int D, int G, int sort_pow2, int cap);
size_t decode_topk_smem(int max_nc, int cap);
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

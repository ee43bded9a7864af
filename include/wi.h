/*
 * wi.h - wave-index sparse decode attention and segmented k-means index build
 *        for NVIDIA B200 (sm_100a).  C ABI of libwi.so.
 *
 * The method is the "wave index" of
 *   "RetroInfer: A Vector Storage Engine for Scalable Long-Context LLM
 *    Inference" (technical summary), section 2.A Wave Index:
 *   item 1 Steady Zone      - sink tokens and the most recent tokens are
 *                             always attended exactly;
 *   item 2 Retrieval Zone   - the clusters most similar to the query are
 *                             fetched and attended exactly;
 *   item 3 Estimation Zone  - every other cluster contributes through its
 *                             centroid, counted once per member token;
 *   Segmented Clustering    - the index is built at prefill by clustering
 *                             each segment of the sequence separately.
 * The split into a query-independent build and a query-dependent decode,
 * and the paged ragged layout (batch, index pointers, ragged index
 * structures), follow "Vortex - Servizio di Attention Sparsa Efficiente e
 * Programmabile per Agenti AI", sections 2.A (forward_cache /
 * forward_indexer; GeMM, Softmax, Top-K, Gather) and 2.B (vTensor).
 *
 * Conventions for every entry point:
 *  - Ownership: the caller allocates and owns every buffer.  The library
 *    never allocates device or pinned memory and keeps no state between
 *    calls (apart from a thread-local copy of the last CUDA error string).
 *  - Asynchrony: work is enqueued on `stream`; no call synchronises the
 *    host except wi_read_device_status.  Calls may be captured in a CUDA
 *    graph.
 *  - Errors: argument errors are detected on the host and returned before
 *    any CUDA call (so they are safe to test without a GPU).  A failed
 *    launch returns WI_ERR_CUDA.  Kernels bounds-check every page, slot and
 *    cluster index they dereference; on a violation they skip the access
 *    and set a bit in the workspace status word (wi_read_device_status).
 *  - Pointers: device pointers must be 16-byte aligned; workspaces 256-byte
 *    aligned.  "host" marks arguments read on the host during the call.
 *  - Workspace: the first 256 bytes of a workspace hold the device status
 *    word.  Zero them once when the workspace is first allocated; the
 *    library leaves them unchanged except for setting error bits.
 *
 * Notation: B batch, T_b tokens of sequence b, Hq query heads, Hkv KV heads,
 * G = Hq/Hkv (q head h reads KV head h/G), d head_dim, P page_size,
 * S seg_len, cs cluster_size, NC_b = sum over segments of ceil(len/cs).
 * A "unit" is one (sequence b, KV head h) pair, u = b*Hkv + h.
 */
#ifndef WI_H
#define WI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / cudaEvent_t; NULL stream = legacy default. */
typedef struct CUstream_st *wi_stream_t;
typedef struct CUevent_st *wi_event_t;

typedef enum wi_status {
  WI_OK = 0,
  WI_ERR_INVALID_ARG = 1,   /* bad pointer, size or geometry; nothing launched */
  WI_ERR_UNSUPPORTED = 2,   /* valid, but outside the built kernels or limits  */
  WI_ERR_WORKSPACE = 3,     /* workspace missing, too small or misaligned      */
  WI_ERR_CUDA = 4,          /* a CUDA call failed (wi_last_error_string)       */
  WI_ERR_DEVICE_CHECK = 5   /* a kernel met an out-of-range index and skipped it */
} wi_status;

typedef enum wi_dtype { WI_F32 = 0, WI_BF16 = 1 } wi_dtype;

#define WI_MAX_BATCH 256      /* sequences per call                            */
#define WI_MAX_SEG_LEN 16384  /* tokens per segment                            */
#define WI_MAX_STEADY 8192    /* steady tokens per sequence unless it is all steady */

/* Device status bits (wi_read_device_status). */
#define WI_DEV_BAD_PAGE    0x1u  /* block-table entry outside [0, n_pages)      */
#define WI_DEV_BAD_SLOT    0x2u  /* perm / invperm value outside [0, T_b)       */
#define WI_DEV_BAD_CLUSTER 0x4u  /* offsets not monotone or cluster out of range */
#define WI_DEV_BAD_HIST    0x8u  /* stale selection histogram (workspace reused
                                    after a failed call); recomputed, result valid */
#define WI_DEV_TIMEOUT     0x10u /* a bounded wait for an asynchronous copy gave
                                    up; the call's results are not valid        */
#define WI_DEV_CANCELLATION 0x20u /* the estimate taken back out (retrieved and
                                    non-candidate clusters, steady tokens) was
                                    more than 16x the output's softmax
                                    denominator, so the estimation zone lost its
                                    precision: the index's centroids are not the
                                    means of their members (every index the
                                    build calls write is); results not valid    */

/*
 * Paged KV cache in original token order (the build input).
 * Token t of sequence b, KV head h lives at
 *   pool[block_table[b*max_pages + t/P]][h][t%P][0..d)
 * Rows are d contiguous elements of `dtype`.
 */
typedef struct wi_kv_cache {
  wi_dtype dtype;              /* WI_F32 or WI_BF16                             */
  int32_t batch;               /* 1..WI_MAX_BATCH                               */
  int32_t n_kv_heads;          /* >= 1                                          */
  int32_t head_dim;            /* 64 or 128                                     */
  int32_t page_size;           /* power of two, 1..1024                         */
  int64_t n_pages;             /* pages in k_pool / v_pool                      */
  const void *k_pool;          /* device [n_pages][Hkv][P][d]                   */
  const void *v_pool;          /* device [n_pages][Hkv][P][d]                   */
  const int32_t *block_table;  /* device [batch][max_pages]                     */
  int32_t max_pages;           /* >= ceil(T_b/P) for every b                    */
  const int32_t *seq_lens;     /* host [batch], T_b >= 1                        */
} wi_kv_cache;

/*
 * The wave index of a batch (all buffers caller-allocated, device unless
 * marked host).  Cluster-indexed arrays are unit-major: unit u = (b, h)
 * starts at row  cl_row(b,h) = Hkv*C_b + h*NC_b  where C_b = sum_{b'<b} NC_b'.
 * Token-indexed arrays start at  tok_row(b,h) = Hkv*S_b + h*T_b  where
 * S_b = sum_{b'<b} T_b'.  offsets start at  Hkv*(C_b + b) + h*(NC_b + 1).
 *
 * Slot s of unit (b,h) is the s-th row of the cluster-permuted layout:
 * clusters in order, members of a cluster in ascending original position.
 * Segment g occupies slots [g*S, g*S + len_g), the same as its positions.
 */
typedef struct wi_index {
  wi_dtype dtype;              /* KV dtype; centroids and value sums use it too */
  int32_t batch, n_kv_heads, head_dim, page_size, seg_len, cluster_size;
  const int32_t *seq_lens;     /* host [batch]                                  */
  void *centroids;             /* [Hkv*sum NC_b][d]  mean key of each cluster   */
  void *value_sums;            /* [Hkv*sum NC_b][d]  sum of member values       */
  int32_t *offsets;            /* [Hkv*(sum NC_b + batch)]  slot range per cluster,
                                  NC_b+1 entries per unit, last = T_b           */
  int32_t *perm;               /* [Hkv*sum T_b]  slot -> original position      */
  int32_t *invperm;            /* [Hkv*sum T_b]  original position -> slot      */
  int32_t *labels;             /* [Hkv*sum T_b]  original position -> cluster id
                                  (0..NC_b-1, unit-local)                       */
  void *k_pool;                /* [n_pages][Hkv][P][d]  keys in slot order      */
  void *v_pool;                /* [n_pages][Hkv][P][d]  values in slot order    */
  int64_t n_pages;
  const int32_t *block_table;  /* [batch][max_pages]  pages of the permuted pools */
  int32_t max_pages;
} wi_index;

/* Retrieval-zone selection modes (wi_decode_params.topk_mode). */
#define WI_TOPK_EXACT   0  /* the k best candidates, lower id first on equal scores */
#define WI_TOPK_SAMPLED 1  /* Vortex 2.C stochastic radix top-k: see below          */

/* Decode options (query-dependent phase). */
typedef struct wi_decode_params {
  int32_t n_q_heads;           /* Hq, a multiple of Hkv with G in {1,2,4,8}     */
  int32_t n_sink;              /* steady zone: first n_sink positions (>= 0)    */
  int32_t window;              /* steady zone: last `window` positions (>= 0)   */
  int32_t topk_clusters;       /* >= 0: clusters retrieved per unit;
                                  < 0: ceil(topk_fraction * NC_b) (in double)   */
  double topk_fraction;        /* in [0, 1], used when topk_clusters < 0        */
  wi_event_t *stage_events;    /* optional: wi_decode_stage_count()+1 events,
                                  recorded before each stage and after the last */
  int32_t exact_only;          /* nonzero: no estimation zone; the output is
                                  attention over the retrieved clusters and the
                                  steady zone only (the block top-k workload of
                                  Vortex 2.A on a wi_build_blocks index)        */
  int32_t topk_mode;           /* WI_TOPK_EXACT or WI_TOPK_SAMPLED.  Sampled
                                  (Vortex 2.C, early termination by sampling):
                                  the selection keys are ranked by the top 11
                                  bits of the fp32 group-max score's
                                  order-preserving key; every candidate in a bin
                                  above the bin of the k-th key is retrieved,
                                  and the rest are drawn from that bin without
                                  replacement: cluster c draws
                                  SplitMix64(seed * 2^32 + c) and the smallest
                                  (draw, c) win                                 */
  uint32_t seed;               /* draws of WI_TOPK_SAMPLED                      */
  float *scores_out;           /* optional device float [Hkv*sum NC_b][G]: each
                                  cluster's score q_g . centroid / sqrt(d) per
                                  query head (rows laid out like the centroids;
                                  units attended densely are not written).  It
                                  costs 4 G bytes of writes per cluster.        */
} wi_decode_params;

/* Byte offsets of the decode workspace regions (for inspection and tests). */
typedef struct wi_decode_layout {
  size_t total_bytes;
  size_t status;       /* uint32 status word (offset 0)                           */
  size_t records;      /* uint32 pairs [Hkv*sum NC_b]: {selection key of the
                          group-max score (order-preserving; 0 = not a
                          candidate), the cluster's first slot}                  */
  size_t selected;     /* int32 [Hkv*sum NC_b], rows laid out like the centroids:
                          the first sel_count entries of a unit's rows are its
                          retrieved cluster ids, ascending                        */
  size_t unit_info;    /* int32 [B*Hkv][info_ints]: {sel_count, thr_key, thr_idx,
                          sel_tokens, steady, n_affected, dense, candidates,
                          full_rows, partial_rows, non_candidates, no_estimate,
                          mode, threshold_bin, draw_hi, draw_lo}                  */
  int32_t n_scan_ctas;   /* streaming CTAs of the scan kernel                     */
  int32_t n_gather_ctas; /* CTAs of the gather kernel                             */
  int32_t info_ints;     /* ints per unit record                                  */
} wi_decode_layout;

/* ------------------------------------------------------------------ sizes */

/* Clusters of each sequence: nc_out[b] = sum over segments of
 * ceil(len/cluster_size) (nullable); *nc_total = sum_b NC_b.  Host only. */
wi_status wi_index_clusters(int32_t batch, const int32_t *seq_lens, int32_t seg_len,
                            int32_t cluster_size, int32_t *nc_out, int64_t *nc_total);

/* ------------------------------------------------------------------ build */

/* Workspace bytes wi_build_index and wi_kmeans_assign need.  Host only. */
wi_status wi_build_workspace_size(const wi_kv_cache *kv, int32_t seg_len,
                                  int32_t cluster_size, size_t *bytes);

/* Byte offsets of the build workspace regions (for inspection and tests).
 * After wi_build_index with `iters` = r, the region at centroids_f32 holds
 * the fp32 working centroids after round r's update (float [Hkv*sum NC_b][d],
 * laid out like wi_index.centroids: the correctly rounded means of round r's
 * assignment, or the previous value for an empty cluster), and the region at
 * `assign` holds round r's assignment (int32 [Hkv*sum T_b], segment-local
 * cluster index of each original position, token-indexed like
 * wi_index.perm).  RetroInfer 2.A, Segmented Clustering.  Host only. */
typedef struct wi_build_layout {
  size_t total_bytes;
  size_t status;          /* uint32 status word (offset 0)                     */
  size_t centroids_f32;
  size_t assign;
} wi_build_layout;
wi_status wi_build_workspace_layout(const wi_kv_cache *kv, int32_t seg_len,
                                    int32_t cluster_size, wi_build_layout *layout);

/*
 * Build the wave index (RetroInfer 2.A, Segmented Clustering; Vortex 2.A
 * forward_cache).  For every unit and every segment of seg_len tokens (the
 * last may be shorter): ceil(len/cs) centroids start as the keys at segment
 * positions 0, cs, 2cs, ...; then `iters` rounds of
 *   assign: each key to the centroid at least squared Euclidean distance
 *           (fp32, direct form sum (k-c)^2; ties to the lower index),
 *   update: each centroid to the mean of its members (fp64 sum in
 *           ascending position, kept as fp32 for the next assignment); an
 *           empty cluster keeps its centroid.
 * Then writes `out`: centroids (the final means) and value sums rounded to
 * the KV dtype (round-to-nearest-even), offsets, perm, invperm, labels, and the K/V
 * rows scattered into out->k_pool/v_pool in slot order through
 * out->block_table.  Requires seg_len % cluster_size == 0, seg_len <=
 * WI_MAX_SEG_LEN, iters >= 1, and `out` geometry equal to `kv`'s.
 * The output pools must not alias the input pools.
 */
wi_status wi_build_index(const wi_kv_cache *kv, int32_t seg_len, int32_t cluster_size,
                         int32_t iters, const wi_index *out, void *ws, size_t ws_bytes,
                         wi_stream_t stream);

/*
 * Build an index of position-contiguous blocks (Vortex summary, section 2.A:
 * forward_cache builds block centroids; forward_indexer then selects the
 * top-k blocks and attends).  Inside each segment of seg_len positions,
 * block j holds positions j*block_size .. (j+1)*block_size - 1 (the last one
 * may be shorter); its centroid is the mean key and its value sum the sum of
 * its values, both rounded to the KV dtype; perm is the identity and the K/V
 * rows are copied to out's pools in position order.  `out` is laid out like
 * any index, with cluster_size = block_size.  Decode it with
 * wi_decode_params.exact_only set for the block top-k workload (or without,
 * to estimate the unselected blocks).  Same workspace as wi_build_index and
 * the same argument errors (block_size in the cluster_size role).
 */
wi_status wi_build_blocks(const wi_kv_cache *kv, int32_t seg_len, int32_t block_size,
                          const wi_index *out, void *ws, size_t ws_bytes, wi_stream_t stream);

/*
 * Extend a built index to longer sequences (RetroInfer 2.A, Segmented
 * Clustering: the index is a sequence of independently clustered segments,
 * so tokens appended while decoding join it segment by segment).
 *
 * old_ix  an index built (or extended) for lengths T_b = old_ix->seq_lens[b].
 * kv      the KV cache in original token order, now of lengths
 *         T'_b = kv->seq_lens[b] >= T_b.  Only positions from
 *         s0_b = floor(T_b / seg_len) * seg_len on are read.
 * out     the index for T'_b, with the seg_len and cluster_size of old_ix.
 *         Its centroid, value-sum, offset, perm, invperm and label buffers
 *         are new, sized for T'_b, and must not be old_ix's.  Its permuted
 *         pools and block table must already hold old_ix's permuted rows for
 *         every slot below s0_b (normally old_ix's own pools, with the block
 *         table extended by pages for the new slots): those rows are not
 *         read or written.
 *
 * The whole segments below s0_b are copied from old_ix. From s0_b on,
 * segments are clustered anew and scattered: a partial last segment of
 * old_ix is redone together with its new tokens. The result equals
 * wi_build_index on the extended sequences with the same iters, bit for
 * bit. Once its slots from s0_b on are rewritten, old_ix no longer matches
 * a shared pool. Workspace: wi_build_workspace_size for kv.
 *
 * Errors are those of wi_build_index, plus WI_ERR_INVALID_ARG when old_ix's
 * geometry differs from out's, when some T'_b < T_b, or when out reuses
 * one of old_ix's index buffers.
 */
wi_status wi_extend_index(const wi_index *old_ix, const wi_kv_cache *kv, int32_t iters,
                          const wi_index *out, void *ws, size_t ws_bytes, wi_stream_t stream);

/*
 * One k-means assignment step with caller-given fp32 centroids
 * (RetroInfer 2.A, Segmented Clustering), the kernel wi_build_index uses.
 * centroids: device float [Hkv*sum NC_b][d] laid out like wi_index.centroids.
 * assign:    device int32 [Hkv*sum T_b], token-indexed like wi_index.perm;
 *            receives the segment-local cluster index of each token.
 */
wi_status wi_kmeans_assign(const wi_kv_cache *kv, int32_t seg_len, int32_t cluster_size,
                           const float *centroids, int32_t *assign, void *ws, size_t ws_bytes,
                           wi_stream_t stream);

/* ----------------------------------------------------------------- decode */

/* Workspace bytes and region offsets for wi_decode / wi_decode_host. */
wi_status wi_decode_workspace_size(const wi_index *idx, const wi_decode_params *p,
                                   size_t *bytes);
wi_status wi_decode_workspace_layout(const wi_index *idx, const wi_decode_params *p,
                                     wi_decode_layout *layout);

/*
 * One decode step over the wave index (RetroInfer 2.A items 1-3; Vortex 2.A
 * forward_indexer).  For each unit (b,h), with its G query heads:
 *  (a) s[g][c] = q_g . centroid_c / sqrt(d) for every cluster c;
 *  (b) retrieval: the k clusters with the largest max_g s[g][c] among
 *      candidates (clusters with at least one non-steady member), lower id
 *      first on ties, k clamped to the candidate count;
 *  (c) exact attention over the steady zone (positions [0, n_sink) and
 *      [T_b - window, T_b)) plus the non-steady members of the retrieved
 *      clusters, read from the permuted paged layout;
 *  (d) estimation: every other candidate c adds cnt'_c * e^{s[g][c]} to the
 *      softmax denominator and e^{s[g][c]} * Vsum'_c to the numerator, where
 *      cnt' and Vsum' exclude the cluster's steady members;
 *  (e) log-sum-exp merge of the parts.
 * q:   device [B][Hq][d] in the KV dtype.
 * out: device float [B][Hq][d];  lse: device float [B][Hq] or NULL
 *      (natural log of the softmax denominator).
 * A sequence whose steady zone covers all of it is attended exactly (dense).
 * Non-dense sequences need n_steady <= WI_MAX_STEADY (else WI_ERR_UNSUPPORTED).
 */
wi_status wi_decode(const void *q, const wi_index *idx, const wi_decode_params *p,
                    float *out, float *lse, void *ws, size_t ws_bytes, wi_stream_t stream);

/*
 * wi_decode with host buffers: copies q (host [B][Hq][d], KV dtype) into the
 * workspace, decodes, and copies out (host float [B][Hq][d]) and lse (host
 * float [B][Hq], nullable) back, all on `stream`.  When out (and lse, if
 * given) are pinned, device-mapped host memory (as cudaHostAlloc returns on
 * a unified-address system), the kernels write them directly through their
 * device addresses instead, and they are complete once the stream passes
 * the call.  The host buffers must stay valid until the stream has passed
 * the call; use pinned memory for asynchronous copies.  Needs the workspace size wi_decode_workspace_size
 * reports (it includes the staging area).
 * With pinned host buffers on a stream other than the legacy default one,
 * and no stage events or score output, the second call with the same
 * pointers, sizes and options captures the call's copies and kernels into a
 * CUDA graph, and later such calls launch that graph (the library keeps the
 * 16 most recently used, keyed by the current CUDA context's unique id, so a
 * device reset never reuses one); the result is the same.  A call on a
 * stream that is being captured enqueues its work into that capture instead.
 */
wi_status wi_decode_host(const void *q_host, const wi_index *idx, const wi_decode_params *p,
                         float *out_host, float *lse_host, void *ws, size_t ws_bytes,
                         wi_stream_t stream);

/*
 * wi_decode with no allocation and no caller workspace.  The method has no
 * counterpart of this call; it exists for callers that cannot allocate device
 * memory where they decode: code inside a CUDA stream capture (cudaMalloc
 * cannot be captured), serving loops whose device memory is all owned by a
 * fixed arena, and C callers embedded in runtimes without a device allocator.
 *
 * The workspace is a fixed array of WI_NOALLOC_SCRATCH_MIB MiB in the
 * library's device memory, held by every GPU that loads the library until
 * the process exits.  A decode whose workspace (wi_decode_workspace_size)
 * exceeds it returns WI_ERR_WORKSPACE before touching the GPU.  Each call
 * clears the part of the scratch that must start at zero, then runs exactly
 * what wi_decode runs.  All calls share the one array, so calls that overlap
 * on the GPU (other streams, other host threads) race; serialise them.  The
 * first call on a device looks up the array's device address, so make it
 * before any stream capture on that device.  Device-side index checks still
 * skip bad accesses, but their status bits are not readable through this
 * entry point.  The address is cached per CUDA context: after a device reset
 * the new context looks it up again on its first call.  Argument errors
 * (null or misaligned q / out / lse, bad index or parameters) are returned
 * before any CUDA call.  q, out, lse: as for wi_decode.
 */
#define WI_NOALLOC_SCRATCH_MIB 32
wi_status wi_decode_noalloc(const void *q, const wi_index *idx, const wi_decode_params *p,
                            float *out, float *lse, wi_stream_t stream);

/* Number of kernels one wi_decode call launches, and its stage names. */
int32_t wi_decode_stage_count(void);
const char *wi_decode_stage_name(int32_t i);

/* --------------------------------------------------------------- status */

/*
 * Synchronise `stream`, read the status word of workspace `ws` into *flags
 * (WI_DEV_* bits), and clear it if `clear` is non-zero.  Returns
 * WI_ERR_DEVICE_CHECK when a bit is set, WI_OK otherwise.
 */
wi_status wi_read_device_status(const void *ws, wi_stream_t stream, uint32_t *flags, int clear);

const char *wi_status_string(wi_status s);
const char *wi_last_error_string(void);   /* thread-local, last CUDA failure */

#ifdef __cplusplus
}
#endif
#endif /* WI_H */

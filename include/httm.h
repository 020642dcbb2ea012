/*
 * httm.h -- C ABI of a B200 (sm_100a) implementation of HTTM's head-wise
 * temporal token merging around one VGGT-style global-attention layer.
 *
 * Method: "HTTM: Head-wise Temporal Token Merging for Faster VGGT"
 * (papernotes.org note, CVPR 2026).  The layer merges each head's Q/K/V
 * tokens before the attention kernel and unmerges after it (overall
 * framework); merging is per head (key design 1), only inside temporal
 * blocks of n_s patches x n_t frames (key design 2), and a global top-d%
 * query outlier filter restores badly merged queries (key design 3).
 *
 * Conventions shared by every entry point
 *  - Tensors are row-major [h, N, d_head] with N = T * P and token
 *    n = t * P + p (p in raster order on the patch grid); element type bf16
 *    (HTTM_BF16) or fp32 (HTTM_F32).  All tensor pointers are DEVICE
 *    pointers, 16-byte aligned, owned by the caller.
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy
 *    default stream.  Entry points that take a stream only enqueue work on
 *    it: they never synchronise and never copy to the host, unless stated.
 *  - Host-detectable errors return a status synchronously and enqueue
 *    nothing.  Errors the device detects (an injected plan that is not a
 *    valid plan, an index out of bounds, a bounded wait that ran out) set
 *    bits of a status word kept in the workspace; the kernels skip the bad
 *    access instead of trapping.  Each forward call clears the word when it
 *    starts; httm_get_device_status() reads it.
 *  - Nothing throws across this boundary.  The library allocates no device
 *    memory except the small block table owned by a plan (and, for an
 *    HTTM_PARTITION plan, its token classes and block lists).
 *  - A plan is not thread-safe: calls on one plan from several host threads
 *    must not overlap (the caller serialises them, or gives each thread a
 *    plan of its own; plans are cheap).  Calls on different plans may run
 *    concurrently from any threads.
 */
#ifndef HTTM_H_
#define HTTM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HTTM_OK = 0,
  HTTM_ERR_ARG = 1,              /* null pointer, bad size or field */
  HTTM_ERR_UNSUPPORTED = 2,      /* valid request this build does not handle */
  HTTM_ERR_INFEASIBLE_RATIO = 3, /* r_b exceeds the sources of some block */
  HTTM_ERR_WORKSPACE = 4,        /* workspace smaller than httm_workspace_bytes() */
  HTTM_ERR_ALIGN = 5,            /* a pointer is not 16-byte aligned */
  HTTM_ERR_CUDA = 6,             /* a CUDA runtime call failed */
  HTTM_ERR_TIMEOUT = 7,          /* device: a bounded wait ran out */
  HTTM_ERR_DEVICE_BOUNDS = 8,    /* device: an index was out of bounds / plan invalid */
  HTTM_ERR_EXCHANGE = 9,         /* the caller's collective (httm_exchange) reported a failure */
} httm_status;

typedef enum { HTTM_BF16 = 0, HTTM_F32 = 1 } httm_dtype;

typedef enum {
  HTTM_HEADWISE_TEMPORAL = 0, /* HTTM: per-head plans inside temporal blocks */
  HTTM_HEAD_UNIFORM = 1,      /* one plan per block from the head-mean cosine, used by all heads */
  HTTM_CONTIGUOUS = 2,        /* per-head plans inside runs of contig_block tokens, no reorder */
  HTTM_DENSE = 3,             /* no merging: plain softmax attention over all N tokens */
  HTTM_PARTITION = 4,         /* HTTM blocks with LiteVGGT's destination rule (httm_plan_partition) */
} httm_mode;

/* Device status word bits (httm_get_device_status). */
#define HTTM_DEV_BAD_PLAN 0x1u    /* an injected plan broke a rule; see httm_forward_with_plan */
#define HTTM_DEV_BOUNDS 0x2u      /* an index fell outside its buffer */
#define HTTM_DEV_TIMEOUT 0x4u     /* a bounded device wait ran out */

/*
 * Layer configuration (plain data).  The knobs are those of the HTTM note's
 * training-strategy section: n_s spatial tokens x n_t frames per block,
 * a query merge ratio, a key/value merge ratio and an outlier ratio.
 *  h, T, P, d_head   heads (<= 64), frames, patch tokens per frame, channels
 *                    per head; d_head in {16, 64}.  The tensor-core kernels
 *                    serve bf16 with d_head = 64; other shapes run on
 *                    CUDA-core kernels (a correctness path for small cases).
 *                    HTTM_PARTITION needs bf16 with d_head = 64.
 *  n_s, n_t          block = n_s consecutive patches (raster) x n_t frames;
 *                    the last region / temporal group may be partial.
 *  contig_block      block length of HTTM_CONTIGUOUS (ignored otherwise).
 *  q_dst_stride      the in-block tokens i with i % stride == 0 are the
 *  kv_dst_stride     destinations, the others sources (>= 2).
 *  q_merge_pct       r: floor(pct * n_b / 100) sources of each block merge.
 *  kv_merge_pct
 *  outlier_pct       d: floor(pct * h * N / 100) queries restored (capped at
 *                    the number of merged queries).
 *  softmax_scale     0 selects 1 / sqrt(d_head).
 */
typedef struct {
  int32_t h, T, P, d_head;
  int32_t dtype; /* httm_dtype */
  int32_t mode;  /* httm_mode */
  int32_t n_s, n_t, contig_block;
  int32_t q_dst_stride, kv_dst_stride;
  int32_t q_merge_pct, kv_merge_pct, outlier_pct;
  float softmax_scale;
} httm_cfg;

typedef struct httm_plan_s* httm_plan_t;

/* Static sizes of a plan (all per head unless stated). */
typedef struct {
  int64_t N;              /* tokens */
  int32_t n_blocks;       /* merge blocks per head */
  int32_t q_slots;        /* regular query slots R_q = sum_b (n_b - r_b^Q) */
  int32_t kv_slots;       /* key/value slots L_k = sum_b (n_b - r_b^KV) */
  int64_t k_out_max;      /* floor(outlier_pct * H * N / 100): outlier budget of all H heads of
                             the layer (H = h, or h * shards after httm_plan_shard) */
  int64_t q_rows_alloc;   /* rows of the shortened-query buffer (all heads, padded) */
  int64_t ws_q_tilde;     /* workspace byte offsets of the shortened tensors: */
  int64_t ws_k_tilde;     /*   Q~ rows [q_rows_alloc, d] (regular slots of head hh at */
  int64_t ws_v_tilde;     /*   hh * q_slots, then per-head outlier runs), K~/V~ [h, L_k, d], */
  int64_t ws_o_tilde;     /*   O~ laid out like Q~; element type = the input dtype */
  int64_t ws_n_out;       /* int32 [h]: outliers per head after a forward */
  int64_t ws_out_base;    /* int32 [h]: first row of each head's outlier run in Q~ */
  int64_t workspace_bytes;
} httm_plan_info;

/*
 * httm_plan: validate `cfg` and build the static block table (key design 2:
 * temporal reordering into blocks of n_s x n_t) on the host; no device call.
 * Returns HTTM_ERR_ARG for a bad field, HTTM_ERR_UNSUPPORTED for shapes this
 * build has no kernel for (d_head not 16/64, a block over 8192 tokens, more
 * than 64 heads), HTTM_ERR_INFEASIBLE_RATIO when r_b exceeds the sources of
 * some block.  The first httm_forward* / httm_reorder call uploads the
 * table to the then-current device (a synchronous copy; make that first call
 * outside any stream capture) and binds the plan to that device: calls from
 * another device return HTTM_ERR_ARG.  That call also creates, except for
 * HTTM_DENSE, one non-blocking CUDA stream and two events, which the plan
 * owns with the table until httm_plan_destroy().
 */
httm_status httm_plan(const httm_cfg* cfg, httm_plan_t* out);
void httm_plan_destroy(httm_plan_t plan);
httm_status httm_get_plan_info(httm_plan_t plan, httm_plan_info* info);

/* Device workspace bytes httm_forward* needs (caller allocates, >= 256-B aligned). */
size_t httm_workspace_bytes(httm_plan_t plan);

/*
 * httm_forward: the merged global-attention layer (overall framework of the
 * HTTM note): per head and block, bipartite cosine matching of sources to
 * destinations, top-r mean merging of Q and of K with V following K's plan
 * (key design 1); the global query outlier filter and restore (key design
 * 3); softmax(Q~ K~^T * scale) V~ on the shortened sequences; unmerge, which
 * copies each merged token's output back to its members and undoes the
 * reorder.  Q, K, V: [h, N, d] inputs; out: [h, N, d] output (same dtype).
 * HTTM_DENSE computes plain attention of Q, K, V.  Asynchronous on `stream`;
 * the workspace must not be shared by calls that overlap on the GPU.
 * Bit-deterministic for identical inputs.  Unless stage timing is on, the
 * key branch (matching, planning and gathering K/V) runs on the plan's own
 * stream, forked from `stream` by an event at the call's start and joined
 * back before attention, so the call stays ordered on `stream` and records
 * into a CUDA graph captured on it; calls on one plan enqueued on several
 * streams share that stream, which only serialises their key branches.
 */
httm_status httm_forward(httm_plan_t plan, const void* Q, const void* K, const void* V,
                         void* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Debug exports (all optional DEVICE pointers; NULL skips the export).
 * Per-token arrays are [h, N] in original token order.
 */
typedef struct {
  int32_t* q_best;    /* original index of the destination each query source chose; -1 on destinations */
  float* q_score;     /* its cosine (fp32); 0 on destinations */
  uint8_t* q_merged;  /* 1 if the source merged */
  int32_t* k_best;    /* the same for the key plan (values follow it) */
  float* k_score;
  uint8_t* k_merged;
  int32_t* q_slot;    /* final query slot: regular slot, or q_slots + rank for an outlier */
  int32_t* k_slot;    /* key/value slot */
  float* dev;         /* deviation ||q_n - q~||_2 of eligible queries, 0 otherwise */
  uint8_t* outlier;   /* the mask M_o */
  float* q_means;     /* [h, q_slots, d] fp32 query means before the filter */
  float* q_restored;  /* [h, q_slots, d] fp32 query means after the restore */
  float* k_means;     /* [h, kv_slots, d] fp32 */
  float* v_means;     /* [h, kv_slots, d] fp32 */
} httm_debug;

httm_status httm_forward_debug(httm_plan_t plan, const void* Q, const void* K, const void* V,
                               void* out, void* workspace, size_t workspace_bytes,
                               const httm_debug* dbg, void* stream);

/*
 * A merge plan supplied by the caller (device pointers, [h, N], original
 * order), which replaces the one the layer would compute, so that merging,
 * the filter, attention and unmerge can be checked on a given plan.
 *  q_best/k_best   for each source: original index of its destination (the
 *                  destination must lie in the same block); ignored on
 *                  destinations.
 *  q_merged/k_merged  1 if the source merges; exactly r_b per block.
 *  outlier         optional M_o (NULL: computed).  Only queries in groups of
 *                  >= 2 tokens may be set, at most k_out_max in all.
 * A plan breaking a rule sets HTTM_DEV_BAD_PLAN (the output is then undefined).
 * In HTTM_HEAD_UNIFORM mode the per-head arrays are used as given.
 */
typedef struct {
  const int32_t* q_best;
  const uint8_t* q_merged;
  const int32_t* k_best;
  const uint8_t* k_merged;
  const uint8_t* outlier;
} httm_merge_plan;

httm_status httm_forward_with_plan(httm_plan_t plan, const void* Q, const void* K, const void* V,
                                   void* out, void* workspace, size_t workspace_bytes,
                                   const httm_merge_plan* injected, const httm_debug* dbg,
                                   void* stream);

/*
 * httm_forward_reuse: the layer on new Q, K, V with the merge indices of an
 * earlier call kept.  The LiteVGGT note (key design 3, cross-layer cached
 * merging) computes the merge indices once every few layers and lets the
 * layers in between reuse them, since token similarity changes little from
 * one layer to the next.  Here the reused state is both plans' member lists
 * (which sources merged into which destination, per head and block) left in
 * `workspace` by the last httm_forward / httm_forward_debug /
 * httm_forward_with_plan call on the same plan and workspace; matching and
 * top-r selection are skipped.  Group means of Q, K and V, the query
 * deviations, the outlier filter and restore, attention and unmerge are all
 * recomputed from the new inputs.  The call is otherwise httm_forward's
 * (same arguments, asynchronous on `stream`).
 * Errors: HTTM_ERR_ARG in HTTM_DENSE mode.  If the workspace does not hold
 * member lists written by this plan (no earlier call, another plan's call
 * since, or a call whose planning failed), the device sets HTTM_DEV_BAD_PLAN
 * and the output is undefined; httm_get_device_status() reports it.
 */
httm_status httm_forward_reuse(httm_plan_t plan, const void* Q, const void* K, const void* V,
                               void* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Head sharding (one layer over several GPUs).  Every step of the layer is
 * per head except one: the outlier filter's budget, the top-d% of the
 * deviations of ALL heads' queries (key design 3: the filter is global
 * across heads, ties broken by the flat index h * N + n).  A layer of
 * H = h * shards heads can therefore run as `shards` plans of h heads each,
 * one per GPU, shard s holding heads [s * h, s * h + h) of Q, K, V and out,
 * if the shards sum five small integer buffers between the filter's steps:
 * the eligible-query count (4 B), the three radix histograms (8, 8 and
 * 4 KB), and the per-shard counts of keys equal to the threshold (256 B).  The selection, and so the mask, is
 * then exactly that of the unsharded layer.
 *
 * httm_exchange: the caller's collective.  allreduce_sum must sum `count`
 * elements of `elem_bytes` bytes (4: uint32, 8: uint64) at the DEVICE
 * address `buf` over all shards, in place, ordered on `stream` (work
 * enqueued on `stream` after it returns sees the sums), e.g. an NCCL
 * all-reduce; return 0 on success.  The library calls it from the thread
 * that called httm_forward_sharded, the same number of times in the same
 * order on every shard; `user` is passed through.
 */
typedef struct {
  int32_t (*allreduce_sum)(void* buf, int64_t count, int32_t elem_bytes, void* stream, void* user);
  void* user;
} httm_exchange;

/*
 * httm_plan_shard: make `plan` (cfg.h = heads per shard) shard `shard` of
 * `shards` of a head-sharded layer.  Changes the outlier budget to
 * floor(d% * h * shards * N / 100) and so httm_workspace_bytes(); call it
 * before the plan's first forward.  Errors: HTTM_ERR_ARG (shards < 1 or
 * above 64, shard outside [0, shards), or the plan has already run);
 * HTTM_ERR_UNSUPPORTED for HTTM_HEAD_UNIFORM with shards > 1 (its plan
 * averages the cosines of all heads).
 */
httm_status httm_plan_shard(httm_plan_t plan, int32_t shard, int32_t shards);

/*
 * httm_forward_sharded: httm_forward (or, with a non-null dbg,
 * httm_forward_debug) for one shard of a head-sharded layer, calling
 * ex->allreduce_sum five times on `stream` (never in HTTM_DENSE mode).  ex may be NULL
 * only for a single-shard plan.  A sharded plan runs only through this
 * call: httm_forward, httm_forward_debug, httm_forward_with_plan and
 * httm_forward_reuse return HTTM_ERR_ARG on it.  HTTM_ERR_EXCHANGE if a
 * collective failed (the work already enqueued stays enqueued; the output
 * is undefined).
 */
httm_status httm_forward_sharded(httm_plan_t plan, const void* Q, const void* K, const void* V, void* out,
                                 void* workspace, size_t workspace_bytes, const httm_exchange* ex,
                                 const httm_debug* dbg, void* stream);

/*
 * httm_plan_partition: LiteVGGT's token partition as the destination rule
 * of an HTTM_PARTITION plan ("LiteVGGT: Boosting Vanilla VGGT via
 * Geometry-aware Cached Token Merging", key designs 1-2).  `score` is a
 * DEVICE array [T, P] fp32, one geometric-importance score per token
 * (shared by the heads; the note derives it from image gradients and local
 * variance -- here the caller supplies it).  Per frame the
 * floor(ga_pct * P / 100) highest scores are geometry-aware (GA) tokens that
 * never merge (score ties: lower patch index first); the first frame's
 * other tokens are all destinations; in every later frame the lowest-
 * scoring non-GA token of each 2x2 cell of the grid x grid patch grid (P =
 * grid^2; cells from even rows and columns, 2x1 / 1x2 / 1x1 on an odd edge;
 * ties: lower patch index) is a destination; the other tokens are sources.
 * Merging stays per head inside the plan's temporal blocks (n_s x n_t): a
 * block's destinations are the destination-class tokens in it, every source
 * merges into its most similar one (cosine, ties to the lowest destination
 * in block order), GA tokens (and the sources of a block without
 * destinations) stay single.  Q and K use the same classes; V follows K.
 * The plan's q/kv strides and merge ratios are ignored in this mode.
 * The classes and per-block lists are computed on the device; the call then
 * SYNCHRONISES `stream` to read the per-block counts (2 ints a block) and
 * resizes the plan: call httm_get_plan_info / httm_workspace_bytes again
 * afterwards.  It may be called again with a new score (the plan then
 * holds the new partition).  roles_out (optional DEVICE [T, P] u8) receives
 * the classes: 0 source, 1 destination, 2 GA.  The first call binds the plan
 * to the current device and allocates its class / list arrays (N bytes +
 * 8 N bytes, owned by the plan).  Errors: HTTM_ERR_ARG (not an
 * HTTM_PARTITION plan, null score, ga_pct outside [0, 100], P not a square);
 * HTTM_ERR_UNSUPPORTED (P > 16384, or a block with more than 1280
 * destinations).  Forward calls on an HTTM_PARTITION plan return
 * HTTM_ERR_ARG until it has been partitioned; httm_forward_with_plan and
 * httm_plan_shard do not support this mode (HTTM_ERR_UNSUPPORTED).
 */
httm_status httm_plan_partition(httm_plan_t plan, const float* score, int32_t ga_pct, uint8_t* roles_out,
                                void* stream);

/*
 * httm_reorder: temporal reordering (key design 2).  inverse = 0: X in
 * original order [h, N, d] -> Xb in block order (block after block, each
 * block frame-major: the n_s-patch region of frame t0, then of t0 + 1, ...).
 * inverse = 1: the inverse permutation.  X and Xb must not overlap.
 */
httm_status httm_reorder(httm_plan_t plan, const void* X, void* Xb, int inverse, void* stream);

/*
 * httm_set_wait_budget: the bound, in nanoseconds, of every device-side wait
 * of the later forward calls on `plan` (default 2e9: 2 s).  A wait that runs
 * out sets HTTM_DEV_TIMEOUT in the status word; its CTA stops its work,
 * waits (with a fixed 2 s bound) for the tensor-core operations it issued,
 * frees its tensor memory and exits, and the call's output is undefined.
 * The context stays usable.  0 makes every wait that is not already
 * complete run out at once: a failure-detection check, not a setting for
 * real work.  Host only; returns HTTM_ERR_ARG for a null plan.  Not from the
 * pages (bounded waits are this library's own safeguard).
 */
httm_status httm_set_wait_budget(httm_plan_t plan, uint64_t nanoseconds);

/*
 * httm_set_fused_unmerge: with enable != 0, later forward calls on `plan`
 * that run the tensor-core attention (bf16, d_head = 64, merged modes) write
 * each attention output row straight to the tokens it stands for -- the
 * non-outlier members of its slot, or the outlier itself -- from the
 * attention epilogue, and launch no separate unmerge kernel (HTTM note, key
 * designs 1-2: unmerge copies a merged token's output back to its members
 * in the original order).  The output is bit-identical to the default path;
 * the O~ rows in the workspace are then not written.  Default 0: the
 * attention writes O~ and an unmerge kernel copies it out (measured faster
 * on B200: the scattered row writes lengthen every attention wave's tail).
 * Host only; HTTM_ERR_ARG for a null plan.
 */
httm_status httm_set_fused_unmerge(httm_plan_t plan, int enable);

/*
 * Synchronises `stream`, then reads the device status word of `workspace`
 * into *status (0 = clean; HTTM_DEV_* bits otherwise) and clears it.
 * Returns HTTM_ERR_DEVICE_BOUNDS / HTTM_ERR_TIMEOUT when bits were set.
 */
httm_status httm_get_device_status(httm_plan_t plan, void* workspace, void* stream,
                                   uint32_t* status);

/* Kernel launches the last httm_forward* call on this plan enqueued. */
int32_t httm_forward_launches(httm_plan_t plan);

/*
 * Stage timing.  While enabled, every httm_forward* call on the plan
 * records a CUDA event pair around each stage on its stream (no host
 * synchronisation).  httm_profile_read() synchronises on those events, adds
 * their elapsed times per stage into ms[HTTM_NUM_STAGES] (milliseconds) and
 * the number of timed launches into launches[HTTM_NUM_STAGES], then forgets
 * them.  Either output may be NULL.  Host-side only; the plan owns the events.
 * While enabled, every stage runs on `stream` alone, one after another.
 */
typedef enum {
  HTTM_STAGE_MATCH = 0,     /* bipartite cosine matching (key design 1) */
  HTTM_STAGE_MERGE = 1,     /* top-r select, group means, query deviation */
  HTTM_STAGE_OUTLIER = 2,   /* global top-d% select and restore (key design 3) */
  HTTM_STAGE_ATTENTION = 3, /* softmax(Q~ K~^T * scale) V~ */
  HTTM_STAGE_UNMERGE = 4,   /* copy-back in original order */
  HTTM_STAGE_OTHER = 5,     /* state reset, plan import, debug export */
  HTTM_NUM_STAGES = 6
} httm_stage;

httm_status httm_profile_enable(httm_plan_t plan, int enable);
httm_status httm_profile_read(httm_plan_t plan, float* ms, int32_t* launches);

/*
 * httm_select_outliers_noalloc: the global outlier selection of the filter
 * stage, for callers that cannot allocate device memory -- code running
 * inside a host application or inference runtime that hands it only input
 * and output buffers and owns every allocation itself, or a latency-critical
 * loop where a cudaMalloc could synchronise the device or fail under memory
 * pressure.  The HTTM note has no counterpart of this entry point; it exists
 * for those callers only.
 *
 * It allocates nothing: no cudaMalloc/cudaFree and no allocating library
 * routine.  Its scratch (selection histograms, per-chunk counts, counters,
 * about 157 KB) is a fixed array inside the library that every GPU which
 * loads the library holds until the process exits.  Every call on a device
 * shares that one array, and each call clears what must start at zero, so
 * consecutive calls are independent -- but calls that overlap on the GPU
 * (different streams, or different host threads, at the same time) race and
 * give undefined results.  The first call on each device looks up the
 * array's device address (a host-side set-up step, done once per device and
 * CUDA context: after a device reset the next call looks it up again in the
 * new context); make that first call before any stream capture.  A CUDA
 * error that an earlier, unrelated call left pending makes this call return
 * HTTM_ERR_CUDA without enqueuing anything and without clearing that error.
 *
 * Inputs (device): dev [h, N] fp32, each query's deviation from its merged
 * token (finite, >= 0 where eligible); eligible [h, N] u8, nonzero for
 * queries in a merged group of >= 2 tokens.  It selects
 * k = min(floor(outlier_pct * h * N / 100), #eligible) eligible queries with
 * the largest deviation, ties to the lower flat index h * N + n -- the same
 * mask httm_forward_debug exports -- and writes mask [h, N] u8 (1 = outlier)
 * and n_out [h] int32 (outliers per head).  Limits: h <= 64 and
 * h * N <= 33,554,432 tokens; larger sizes return HTTM_ERR_UNSUPPORTED and
 * enqueue nothing.  Asynchronous on `stream`.
 */
httm_status httm_select_outliers_noalloc(const float* dev, const uint8_t* eligible, int32_t h, int32_t N,
                                         int32_t outlier_pct, uint8_t* mask, int32_t* n_out, void* stream);

const char* httm_status_str(httm_status s);

/*
 * After a call returned HTTM_ERR_CUDA: which launch or runtime call of the
 * library failed and the CUDA error it met ("<call>: <error name> (<error
 * string>)"), for the calling host thread; "" if none has failed on this
 * thread.  The string stays valid until the thread's next call of this
 * function.
 */
const char* httm_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* HTTM_H_ */

// Host-side launchers of the kernels (internal; the public ABI is httm.h).
#pragma once
#include <cuda_runtime.h>

#include "internal.h"

namespace httm {

// Debug export destinations (device pointers, any may be null).
struct Debug {
  int32_t* q_best; float* q_score; uint8_t* q_merged;
  int32_t* k_best; float* k_score; uint8_t* k_merged;
  int32_t* q_slot; int32_t* k_slot;
  float* dev; uint8_t* outlier;
  float* q_means; float* q_restored; float* k_means; float* v_means;
};

struct Inject {
  const int32_t* q_best; const uint8_t* q_merged;
  const int32_t* k_best; const uint8_t* k_merged;
  const uint8_t* outlier;
};

// Clears the per-call state; `keep_stamp` keeps the record of which plan
// wrote the workspace's member lists (calls that reuse them).
cudaError_t launch_zero_state(const Dims& dims, const Buffers& buf, bool keep_stamp, cudaStream_t s);

cudaError_t launch_match_simt(const Dims& dims, bool fp32, const BlockDesc* blocks,
                              const int4* items, int n_items, const void* Q, const void* K,
                              const Buffers& buf, cudaStream_t s);

// Tensor-core matching (bf16, d = 64, head-wise plans).  Returns
// cudaErrorNotSupported when the shape is not covered.
cudaError_t launch_match_tc(const Dims& dims, const BlockDesc* blocks, const int4* items,
                            int n_items, const void* Q, const void* K, const Buffers& buf,
                            cudaStream_t s);

cudaError_t launch_import_plan(const Dims& dims, const BlockDesc* blocks, const Inject& inj,
                               const Buffers& buf, cudaStream_t s);

// Merge planning then the mean-merging gathers; `tensors` 3: Q and K (the
// planning of both in one launch, then the Q gather and the K/V gather),
// 1: Q only, 2: K (and V) only.  With `reuse`, only the gathers, on the
// member lists an earlier call left in the workspace.
cudaError_t launch_merge(const Dims& dims, bool fp32, const BlockDesc* blocks, bool injected, bool reuse,
                         const void* Q, const void* K, const void* V, const Buffers& buf,
                         const Debug& dbg, cudaStream_t s, int tensors = 3);

cudaError_t launch_outlier(const Dims& dims, bool fp32, const void* Q, bool mask_injected,
                           const Buffers& buf, cudaStream_t s);
// The same filter in steps, for a head-sharded layer whose shards sum the
// eligible count and each radix histogram between steps (and, after the
// count step, the per-shard counts of keys equal to the threshold):
// histogram pass 2 or 3, then count, then scan + emit.
cudaError_t launch_outlier_pass(const Dims& dims, const Buffers& buf, int pass, cudaStream_t s);
cudaError_t launch_outlier_count(const Dims& dims, bool mask_injected, const Buffers& buf, cudaStream_t s);
cudaError_t launch_outlier_emit(const Dims& dims, bool fp32, const void* Q, bool mask_injected,
                                const Buffers& buf, cudaStream_t s);

cudaError_t launch_restore(const Dims& dims, bool fp32, const BlockDesc* blocks, const void* Q,
                           const Buffers& buf, const Debug& dbg, cudaStream_t s);

cudaError_t launch_dense_items(const Dims& dims, const Buffers& buf, cudaStream_t s);

// softmax(Q K^T * scale) V over the work items in buf.items.  q/o rows are
// indexed by the items; head hh's keys/values are rows [hh * Lk, hh * Lk + Lk).
cudaError_t launch_attention(const Dims& dims, bool fp32, const void* q, const void* k,
                             const void* v, void* o, int Lk, const Buffers& buf, cudaStream_t s);

cudaError_t launch_unmerge(const Dims& dims, bool fp32, const Buffers& buf, void* out,
                           cudaStream_t s);

cudaError_t launch_reorder(const Dims& dims, bool fp32, const BlockDesc* blocks, const void* X,
                           void* Xb, bool inverse, cudaStream_t s);

// HTTM_PARTITION: token classes from the score [T, P] (ga_k GA tokens per
// frame), then every block's destination / other lists, each token's
// ordinal in its list and per block (destinations, sources) in counts.
cudaError_t launch_partition(const Dims& dims, int T, int grid, int ga_k, const float* score, const BlockDesc* blocks,
                             uint8_t* roles, int32_t* lists, int32_t* ord, int32_t* counts, cudaStream_t s);

cudaError_t launch_export(const Dims& dims, const BlockDesc* blocks, const Buffers& buf,
                          const Debug& dbg, cudaStream_t s);

}  // namespace httm

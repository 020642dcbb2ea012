// Internal structures shared by the host planner and the kernels.
//
// Token n = t * P + p of head hh lives at row hh * N + n of a [h, N, d]
// tensor.  Merge blocks follow key design 2 of the HTTM note ("temporal
// reordering + in-block merging"): block b covers the patches
// [p0, p0 + s) of frames [t0, t0 + t_g); in-block index i = tau * s + sigma
// maps to token base + tau * P + sigma with base = t0 * P + p0.  The
// contiguous variant is one frame-less run: s = n_b, t_g = 1.
#pragma once
#include <cstddef>
#include <cstdint>

namespace httm {

struct BlockDesc {
  int32_t base;        // original index of in-block token 0
  int32_t s;           // tokens per frame slice (s_j), n_b for contiguous blocks
  int32_t n_b;         // tokens in the block
  int32_t tok_off;     // offset of the block in block order (sum of earlier n_b)
  int32_t q_ndst, q_r, q_src_off, q_slot_off;   // query plan: dsts, merged, offsets
  int32_t k_ndst, k_r, k_src_off, k_slot_off;   // key plan (values follow it)
};

// Everything a kernel needs to know about the layer; passed by value.
struct Dims {
  int32_t h, N, P, d;
  int32_t mode;                  // httm_mode
  int32_t n_s, n_t, R, contig;   // token -> block mapping
  int32_t nblk;
  int32_t q_stride, kv_stride;
  int32_t q_src, k_src;          // sources per head, all blocks
  int32_t q_slots, k_slots;      // regular query slots / key-value slots per head
  int32_t max_ndst, max_nsrc, max_nb;
  int64_t k_out_max;
  int64_t out_base;              // first row of the outlier region in Q~ / O~
  int64_t q_rows_alloc;
  int32_t nchunk_per_head;       // chunks of the outlier scan per head
  int32_t max_items;             // attention work items (upper bound)
  float scale;
  uint32_t plan_id;              // stamps a workspace whose member lists this plan wrote
  uint64_t wait_budget_ns;       // bound of a device wait (httm_set_wait_budget; default 2 s)
  int32_t shard, shards;         // head sharding: this shard holds heads [shard h, shard h + h) of h shards
  // HTTM_PARTITION (LiteVGGT's destination rule): per token its class and its
  // ordinal in its block's list; per block, at its tok_off, the in-block
  // indices of its destinations (ascending) then of the others (ascending).
  // Null in the other modes, whose destinations are the i % stride == 0.
  const uint8_t* proles;
  const int32_t* plists;
  const int32_t* pord;
};

constexpr uint8_t kRoleSrc = 0, kRoleDst = 1, kRoleGA = 2;   // token classes of HTTM_PARTITION

constexpr int kChunk = 4096;       // keys per chunk of the outlier compaction
constexpr int kHistBins = 2048;    // radix digit of the outlier select (11 bits)
constexpr int kMaxShards = 64;     // head shards of one layer (httm_plan_shard)
constexpr int kAttnRows = 256;     // query rows per attention work item (two 128-row tiles)
constexpr int kMaxAttnParts = 256; // partial results of the last wave's split items (<= one per SM)
constexpr int kBigSlot = 32;       // slots with more members are summed by a whole CTA (listed, then a kernel of their own)
constexpr int kAttnPartStride = 68; // floats per partial row: O (64), row sum, max in use, 2 unused (16-byte rows)
static_assert(kAttnPartStride * 4 % 16 == 0, "partial rows are read and written as float4");

// Capacity of the list of big query slots: members of the slots of one head
// are distinct tokens, so a head has at most N / (kBigSlot + 1) of them.
constexpr size_t big_list_cap(int h, int N) { return (size_t)h * ((size_t)N / (kBigSlot + 1) + 1); }

// Device-side state at the head of the workspace.
struct DevState {
  uint32_t status;               // HTTM_DEV_* bits (sticky until read)
  uint32_t n_eligible;           // queries in groups of >= 2 tokens
  uint32_t n_items;              // live attention work items
  uint32_t plan_stamp;           // plan_id of the member lists held (0: none)
  uint32_t sel[8];               // outlier select: threshold key, eq budget, total
  uint32_t wait_site;            // first bounded wait that ran out: barrier offset | parity << 20 | 1 << 31
  uint32_t wait_cta;             // ... its CTA index
  uint32_t wait_grid;            // ... and the grid size of its launch (tells the kernels apart)
  uint32_t n_big;                // query slots listed in Buffers::q_big
  uint32_t n_kbig;               // key slots listed in Buffers::k_big
  uint64_t wait_ns;              // this call's wait bound (from Dims::wait_budget_ns)
};

struct Workspace {
  size_t state, hist, chunk, n_out, out_base, items;
  size_t q_best, q_score, q_merged, k_best, k_score, k_merged;
  size_t q_slot, q_orank, o_tok, keys, mask, q_members, q_gstart, q_gcount, k_members, k_gstart, k_gcount, q_big, k_big;
  size_t q_tilde, k_tilde, v_tilde, o_tilde;
  size_t attn_part;
  size_t total;
};

struct Debug;  // mirrors httm_debug

// Pointers into one forward's workspace, resolved on the host.
struct Buffers {
  DevState* state;
  uint32_t* hist;          // [3][kHistBins], then [kMaxShards]: keys equal to the threshold per shard
  uint32_t* chunk;         // [nchunk][4]: gt, eq, take, out_before
  int32_t* n_out;          // [h]
  int32_t* out_base;       // [h]
  int4* items;             // [max_items]: head, q_row0, n_rows, unused
  int32_t* q_best; float* q_score; uint8_t* q_merged;
  int32_t* k_best; float* k_score; uint8_t* k_merged;
  int32_t* q_slot;         // [h, N]: regular query slot of every token (kept across calls)
  int32_t* q_orank;        // [h, N]: rank of an outlier within its head (valid where mask is set)
  int32_t* o_tok;          // [q_rows_alloc - out_base]: token (within its head) of each outlier row of Q~
  uint32_t* keys;          // [h, N]: eligible ? bits(dev) + 1 : 0
  uint8_t* mask;           // [h, N]
  int32_t* q_members;      // [h, N]: tokens in slot order (block after block)
  int32_t* q_gstart;       // [h, q_slots]: first member position of each slot
  int32_t* q_gcount;       // [h, q_slots]: members of each slot
  int32_t* k_members;      // the same for the key plan (values follow it)
  int32_t* k_gstart;
  int32_t* k_gcount;
  int32_t* q_big;          // [big_list_cap]: the query slots of more than kBigSlot members, any order
  int32_t* k_big;          // the same for the key slots
  void* q_tilde; void* k_tilde; void* v_tilde; void* o_tilde;
  float* attn_part;        // [kMaxAttnParts][kAttnRows][kAttnPartStride]: partial attention of split items
};

}  // namespace httm

// Host side of the C ABI: validation, the static block table (key design 2
// of the HTTM note: blocks of n_s patches x n_t frames), the workspace layout
// and the launch sequence of one merged global-attention layer.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/httm.h"
#include "internal.h"
#include "launch.h"

using namespace httm;

struct httm_plan_s {
  httm_cfg cfg;
  Dims dims;
  bool fp32;
  int device = -1;
  std::vector<BlockDesc> blocks_h;
  BlockDesc* blocks_d = nullptr;
  int4* match_items_d = nullptr;
  int n_match_items = 0;
  int4* tc_items_d = nullptr;   // tensor-core matching: (tensor + 2 * head, block, first source, sources)
  int n_tc_items = 0;
  int n_tc_q = 0;               // the query items come first in tc_items
  // the key branch of a forward (matching, planning and gathering K/V) runs
  // on this stream, beside the query branch on the caller's stream
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  std::vector<int4> tc_items_h;
  Workspace ws;
  int launches = 0;
  std::vector<int4> items_h;
  // stage timing
  bool profile = false;
  bool fused_unmerge = false;   // httm_set_fused_unmerge
  // HTTM_PARTITION: token classes, block lists, list ordinals, per-block counts
  bool partitioned = false;
  uint8_t* roles_d = nullptr;
  int32_t* lists_d = nullptr;
  int32_t* ord_d = nullptr;
  int32_t* counts_d = nullptr;
  struct Rec { int stage; int n; cudaEvent_t a, b; };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
};

namespace {
cudaEvent_t pool_event(httm_plan_s* p) {
  if (!p->pool.empty()) {
    cudaEvent_t e = p->pool.back();
    p->pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Brackets the launches of one stage with an event pair when profiling.
struct StageTimer {
  httm_plan_s* p;
  cudaStream_t s;
  int stage, n;
  cudaEvent_t a = nullptr;
  StageTimer(httm_plan_s* p_, cudaStream_t s_, int stage_, int n_) : p(p_), s(s_), stage(stage_), n(n_) {
    if (p->profile && (a = pool_event(p)) != nullptr) cudaEventRecord(a, s);
  }
  ~StageTimer() {
    if (!a) return;
    cudaEvent_t b = pool_event(p);
    if (!b) {
      p->pool.push_back(a);
      return;
    }
    cudaEventRecord(b, s);
    p->recs.push_back({stage, n, a, b});
  }
};
}  // namespace

namespace httm {
cudaError_t launch_attention_simt(const Dims& dims, bool fp32, const void* q, const void* k, const void* v,
                                  void* o, int Lk, const Buffers& buf, cudaStream_t s);
bool attention_tc_supported(const Dims& dims, bool fp32);
cudaError_t launch_attention_tc(const Dims& dims, const void* q, const void* k, const void* v, void* o,
                                int Lk, const Buffers& buf, cudaStream_t s, void* unmerge_out);
bool match_tc_supported(const Dims& dims, bool fp32);
}  // namespace httm

namespace {

// The last CUDA error a call of this library met on this thread, for
// httm_last_cuda_error().
thread_local cudaError_t t_last_err = cudaSuccess;
thread_local const char* t_last_where = "";

httm_status cuda_fail(cudaError_t e, const char* where) {
  t_last_err = e;
  t_last_where = where;
  return HTTM_ERR_CUDA;
}

// HTTM_SYNC_CHECK=1 in the environment: synchronise the stream after every
// launch, so that a fault is attributed to the kernel that raised it (a
// debugging aid; it serialises the forward).
bool sync_check() {
  static const bool on = [] {
    const char* v = getenv("HTTM_SYNC_CHECK");
    return v && v[0] == '1';
  }();
  return on;
}

cudaError_t checked(cudaError_t e, cudaStream_t s) {
  if (e != cudaSuccess || !sync_check()) return e;
  (void)s;
  const cudaError_t e2 = cudaDeviceSynchronize();    // every stream of the call (the key branch too)
  return e2 != cudaSuccess ? e2 : cudaGetLastError();
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

Workspace layout(const Dims& d, bool fp32) {
  Workspace w{};
  const size_t es = fp32 ? 4 : 2;
  const size_t hN = (size_t)d.h * d.N;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  w.state = take(sizeof(DevState));
  w.hist = take((3ull * kHistBins + kMaxShards) * 4);
  w.chunk = take((size_t)d.h * d.nchunk_per_head * 16);
  w.n_out = take((size_t)d.h * 4);
  w.out_base = take((size_t)d.h * 4);
  w.items = take((size_t)d.max_items * 16);
  w.q_best = take((size_t)d.h * d.q_src * 4);
  w.q_score = take((size_t)d.h * d.q_src * 4);
  w.q_merged = take((size_t)d.h * d.q_src);
  w.k_best = take((size_t)d.h * d.k_src * 4);
  w.k_score = take((size_t)d.h * d.k_src * 4);
  w.k_merged = take((size_t)d.h * d.k_src);
  w.q_slot = take(hN * 4);
  w.q_orank = take(hN * 4);
  w.o_tok = take((size_t)(d.q_rows_alloc - d.out_base) * 4);
  w.keys = take(hN * 4);
  w.mask = take(hN);
  w.q_members = take(hN * 4);
  w.q_gstart = take((size_t)d.h * d.q_slots * 4);
  w.q_gcount = take((size_t)d.h * d.q_slots * 4);
  w.k_members = take(hN * 4);
  w.k_gstart = take((size_t)d.h * d.k_slots * 4);
  w.k_gcount = take((size_t)d.h * d.k_slots * 4);
  w.q_big = take(big_list_cap(d.h, d.N) * 4);
  w.k_big = take(big_list_cap(d.h, d.N) * 4);
  w.q_tilde = take((size_t)d.q_rows_alloc * d.d * es);
  w.k_tilde = take((size_t)d.h * d.k_slots * d.d * es);
  w.v_tilde = take((size_t)d.h * d.k_slots * d.d * es);
  w.o_tilde = take((size_t)d.q_rows_alloc * d.d * es);
  w.attn_part = take((size_t)kMaxAttnParts * kAttnRows * kAttnPartStride * 4);
  w.total = off;
  return w;
}

Buffers resolve(const Workspace& w, void* base) {
  char* p = static_cast<char*>(base);
  Buffers b{};
  b.state = reinterpret_cast<DevState*>(p + w.state);
  b.hist = reinterpret_cast<uint32_t*>(p + w.hist);
  b.chunk = reinterpret_cast<uint32_t*>(p + w.chunk);
  b.n_out = reinterpret_cast<int32_t*>(p + w.n_out);
  b.out_base = reinterpret_cast<int32_t*>(p + w.out_base);
  b.items = reinterpret_cast<int4*>(p + w.items);
  b.q_best = reinterpret_cast<int32_t*>(p + w.q_best);
  b.q_score = reinterpret_cast<float*>(p + w.q_score);
  b.q_merged = reinterpret_cast<uint8_t*>(p + w.q_merged);
  b.k_best = reinterpret_cast<int32_t*>(p + w.k_best);
  b.k_score = reinterpret_cast<float*>(p + w.k_score);
  b.k_merged = reinterpret_cast<uint8_t*>(p + w.k_merged);
  b.q_slot = reinterpret_cast<int32_t*>(p + w.q_slot);
  b.q_orank = reinterpret_cast<int32_t*>(p + w.q_orank);
  b.o_tok = reinterpret_cast<int32_t*>(p + w.o_tok);
  b.keys = reinterpret_cast<uint32_t*>(p + w.keys);
  b.mask = reinterpret_cast<uint8_t*>(p + w.mask);
  b.q_members = reinterpret_cast<int32_t*>(p + w.q_members);
  b.q_gstart = reinterpret_cast<int32_t*>(p + w.q_gstart);
  b.q_gcount = reinterpret_cast<int32_t*>(p + w.q_gcount);
  b.k_members = reinterpret_cast<int32_t*>(p + w.k_members);
  b.k_gstart = reinterpret_cast<int32_t*>(p + w.k_gstart);
  b.k_gcount = reinterpret_cast<int32_t*>(p + w.k_gcount);
  b.q_big = reinterpret_cast<int32_t*>(p + w.q_big);
  b.k_big = reinterpret_cast<int32_t*>(p + w.k_big);
  b.q_tilde = p + w.q_tilde;
  b.k_tilde = p + w.k_tilde;
  b.v_tilde = p + w.v_tilde;
  b.o_tilde = p + w.o_tilde;
  b.attn_part = reinterpret_cast<float*>(p + w.attn_part);
  return b;
}

// The outlier budget of the whole layer (all shards' heads) and the
// outlier rows, work items and workspace it needs: one shard may receive
// every outlier of the layer.
void size_outliers(Dims& d, int outlier_pct) {
  const long long heads = (long long)d.h * d.shards;
  d.k_out_max = ((long long)outlier_pct * heads * d.N) / 100;
  d.out_base = (long long)align_up((size_t)d.h * d.q_slots, kAttnRows);
  d.q_rows_alloc = d.out_base + d.k_out_max + (long long)kAttnRows * (d.h + 1);
  d.max_items = (int32_t)(d.h * ((d.q_slots + kAttnRows - 1) / kAttnRows) + (d.k_out_max + kAttnRows - 1) / kAttnRows +
                          d.h);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The first call that needs the device uploads the block table and the
// matching work list to the current device (synchronously) and binds the
// plan to that device; later calls must come from the same device.
httm_status check_device(httm_plan_s* plan) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return HTTM_ERR_CUDA;
  if (plan->device < 0) {
    if (plan->dims.mode != HTTM_DENSE) {
      const size_t nb = plan->blocks_h.size() * sizeof(BlockDesc);
      const size_t ni = std::max<size_t>(1, plan->items_h.size()) * sizeof(int4);
      const size_t nt = std::max<size_t>(1, plan->tc_items_h.size()) * sizeof(int4);
      if (cudaMalloc(&plan->blocks_d, nb) != cudaSuccess ||
          cudaMemcpy(plan->blocks_d, plan->blocks_h.data(), nb, cudaMemcpyHostToDevice) != cudaSuccess ||
          cudaMalloc(&plan->match_items_d, ni) != cudaSuccess ||
          (!plan->items_h.empty() &&
           cudaMemcpy(plan->match_items_d, plan->items_h.data(), plan->items_h.size() * sizeof(int4),
                      cudaMemcpyHostToDevice) != cudaSuccess) ||
          cudaMalloc(&plan->tc_items_d, nt) != cudaSuccess ||
          (!plan->tc_items_h.empty() &&
           cudaMemcpy(plan->tc_items_d, plan->tc_items_h.data(), plan->tc_items_h.size() * sizeof(int4),
                      cudaMemcpyHostToDevice) != cudaSuccess)) {
        if (plan->blocks_d) cudaFree(plan->blocks_d);
        if (plan->match_items_d) cudaFree(plan->match_items_d);
        if (plan->tc_items_d) cudaFree(plan->tc_items_d);
        plan->blocks_d = nullptr;
        plan->match_items_d = nullptr;
        plan->tc_items_d = nullptr;
        return HTTM_ERR_CUDA;
      }
    }
    if (plan->dims.mode != HTTM_DENSE &&
        (cudaStreamCreateWithFlags(&plan->side, cudaStreamNonBlocking) != cudaSuccess ||
         cudaEventCreateWithFlags(&plan->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
         cudaEventCreateWithFlags(&plan->ev_join, cudaEventDisableTiming) != cudaSuccess)) {
      if (plan->side) cudaStreamDestroy(plan->side);
      if (plan->ev_fork) cudaEventDestroy(plan->ev_fork);
      if (plan->ev_join) cudaEventDestroy(plan->ev_join);
      plan->side = nullptr;
      plan->ev_fork = plan->ev_join = nullptr;
      return HTTM_ERR_CUDA;
    }
    plan->device = dev;
  }
  return dev == plan->device ? HTTM_OK : HTTM_ERR_ARG;
}

#define HTTM_LAUNCH(expr)                             \
  do {                                                \
    cudaError_t e_ = checked((expr), s);              \
    ++launches;                                       \
    if (e_ != cudaSuccess) return cuda_fail(e_, #expr); \
  } while (0)

// The attention stage: the tensor-core kernel plus the merge of the last
// wave's split items (two launches, timed as one stage), or the CUDA-core
// kernel.  With `unmerge_out` (a merged layer on the tensor-core path) the
// tensor-core kernels write every output row straight to the tokens it
// stands for in unmerge_out and *fused is set: no unmerge launch follows.
// Adds its launches to *launches.
httm_status attention(const httm_plan_s* plan, const void* q, const void* k, const void* v, void* o, int Lk,
                      const Buffers& buf, cudaStream_t s, int* launches, void* unmerge_out = nullptr,
                      bool* fused = nullptr) {
  cudaError_t e;
  if (fused) *fused = false;
  if (attention_tc_supported(plan->dims, plan->fp32)) {
    e = launch_attention_tc(plan->dims, q, k, v, o, Lk, buf, s, unmerge_out);
    *launches += 2;
    if (fused) *fused = unmerge_out != nullptr;
  } else {
    e = launch_attention_simt(plan->dims, plan->fp32, q, k, v, o, Lk, buf, s);
    *launches += 1;
  }
  e = checked(e, s);
  return e == cudaSuccess ? HTTM_OK : cuda_fail(e, "attention");
}

// The outlier filter and its restore.  With a collective (a head-sharded
// layer), the shards sum the eligible count and the first histogram (both
// built by the query gather), each later histogram, and the per-shard counts
// of keys equal to the threshold, between the steps.
httm_status filter_stage(const httm_plan_s* plan, const void* Q, bool mask_inj, const Buffers& buf, const Debug& dd,
                         cudaStream_t s, const httm_exchange* ex, int* launches) {
  const Dims& dims = plan->dims;
  const bool fp32 = plan->fp32;
  if (!ex) {
    if (cudaError_t e_ = checked(launch_outlier(dims, fp32, Q, mask_inj, buf, s), s); e_ != cudaSuccess) return cuda_fail(e_, "launch_outlier");
    *launches += mask_inj ? 3 : 5;  // two histogram passes, count, scan, emit
  } else {
    auto sum = [&](void* p, int64_t n, int32_t eb) { return ex->allreduce_sum(p, n, eb, s, ex->user) == 0; };
    if (!sum(&buf.state->n_eligible, 1, 4) || !sum(buf.hist, kHistBins, 4)) return HTTM_ERR_EXCHANGE;
    for (int pass = 2; pass <= 3; ++pass) {
      if (cudaError_t e_ = checked(launch_outlier_pass(dims, buf, pass, s), s); e_ != cudaSuccess) return cuda_fail(e_, "launch_outlier_pass");
      ++*launches;
      if (!sum(buf.hist + (pass - 1) * kHistBins, pass == 2 ? kHistBins : 1024, 4)) return HTTM_ERR_EXCHANGE;
    }
    if (cudaError_t e_ = checked(launch_outlier_count(dims, false, buf, s), s); e_ != cudaSuccess) return cuda_fail(e_, "launch_outlier_count");
    ++*launches;
    if (!sum(buf.hist + 3 * kHistBins, kMaxShards, 4)) return HTTM_ERR_EXCHANGE;
    if (cudaError_t e_ = checked(launch_outlier_emit(dims, fp32, Q, false, buf, s), s); e_ != cudaSuccess) return cuda_fail(e_, "launch_outlier_emit");
    *launches += 2;  // scan, emit
  }
  if (cudaError_t e_ = checked(launch_restore(dims, fp32, plan->blocks_d, Q, buf, dd, s), s); e_ != cudaSuccess) return cuda_fail(e_, "launch_restore");
  *launches += 2;  // the restore, then its big slots
  return HTTM_OK;
}

httm_status forward_impl(httm_plan_s* plan, const void* Q, const void* K, const void* V, void* out, void* ws,
                         size_t ws_bytes, const httm_merge_plan* inj, const httm_debug* dbg, void* stream,
                         bool reuse = false, bool sharded_call = false, const httm_exchange* ex = nullptr) {
  if (!plan || !Q || !K || !V || !out || !ws) return HTTM_ERR_ARG;
  if (plan->dims.shards > 1 && (!sharded_call || !ex)) return HTTM_ERR_ARG;
  if (ex && !ex->allreduce_sum) return HTTM_ERR_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out)) return HTTM_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return HTTM_ERR_ALIGN;
  if (reuse && (inj || plan->dims.mode == HTTM_DENSE)) return HTTM_ERR_ARG;
  if (plan->dims.mode == HTTM_PARTITION && !plan->partitioned) return HTTM_ERR_ARG;
  if (plan->dims.mode == HTTM_PARTITION && inj) return HTTM_ERR_UNSUPPORTED;
  if (ws_bytes < plan->ws.total) return HTTM_ERR_WORKSPACE;
  if (inj) {
    const bool any = inj->q_best || inj->q_merged || inj->k_best || inj->k_merged;
    const bool all = inj->q_best && inj->q_merged && inj->k_best && inj->k_merged;
    if (any && !all) return HTTM_ERR_ARG;
    if (plan->dims.mode == HTTM_DENSE) return HTTM_ERR_ARG;
  }
  httm_status st = check_device(plan);
  if (st != HTTM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Dims& dims = plan->dims;
  const bool fp32 = plan->fp32;
  Buffers buf = resolve(plan->ws, ws);
  Debug dd{};
  if (dbg) {
    dd = Debug{dbg->q_best, dbg->q_score, dbg->q_merged, dbg->k_best, dbg->k_score, dbg->k_merged,
               dbg->q_slot, dbg->k_slot, dbg->dev, dbg->outlier, dbg->q_means, dbg->q_restored,
               dbg->k_means, dbg->v_means};
  }
  int launches = 0;
  {
    StageTimer t(plan, s, HTTM_STAGE_OTHER, dims.mode == HTTM_DENSE ? 2 : 1);
    HTTM_LAUNCH(launch_zero_state(dims, buf, reuse, s));
    if (dims.mode == HTTM_DENSE) HTTM_LAUNCH(launch_dense_items(dims, buf, s));
  }
  if (dims.mode == HTTM_DENSE) {
    StageTimer t(plan, s, HTTM_STAGE_ATTENTION, 1);
    st = attention(plan, Q, K, V, out, dims.N, buf, s, &launches);
    plan->launches = launches;
    return st;
  }
  const bool plan_inj = inj && inj->q_best;
  const bool mask_inj = inj && inj->outlier;
  if (plan_inj || mask_inj) {
    StageTimer t(plan, s, HTTM_STAGE_OTHER, 1);
    Inject ii{inj->q_best, inj->q_merged, inj->k_best, inj->k_merged, inj->outlier};
    HTTM_LAUNCH(launch_import_plan(dims, plan->blocks_d, ii, buf, s));
  }
  // Without stage timing, the key branch (matching, planning and the K/V
  // gather) runs on the plan's side stream beside the query branch
  // (matching, planning, the query gather and the outlier filter), joined
  // before attention: the branches share no buffer, and the small,
  // latency-bound kernels of one overlap the other's.  With stage timing
  // everything runs in order on `s`, so that each stage can be timed.
  if (!plan->profile && plan->side && match_tc_supported(dims, fp32)) {
    cudaStream_t s2 = plan->side;
    if (cudaEventRecord(plan->ev_fork, s) != cudaSuccess || cudaStreamWaitEvent(s2, plan->ev_fork, 0) != cudaSuccess)
      return HTTM_ERR_CUDA;
    if (!plan_inj && !reuse) {
      if (plan->n_tc_q > 0)
        HTTM_LAUNCH(launch_match_tc(dims, plan->blocks_d, plan->tc_items_d, plan->n_tc_q, Q, K, buf, s));
      if (plan->n_tc_items > plan->n_tc_q)
        HTTM_LAUNCH(launch_match_tc(dims, plan->blocks_d, plan->tc_items_d + plan->n_tc_q,
                                    plan->n_tc_items - plan->n_tc_q, Q, K, buf, s2));
    }
    HTTM_LAUNCH(launch_merge(dims, fp32, plan->blocks_d, plan_inj, reuse, Q, K, V, buf, dd, s, 1));
    HTTM_LAUNCH(launch_merge(dims, fp32, plan->blocks_d, plan_inj, reuse, Q, K, V, buf, dd, s2, 2));
    launches += reuse ? 2 : 4;  // the big-slot kernels after both gathers, and (unless reused) both plannings
    if ((st = filter_stage(plan, Q, mask_inj, buf, dd, s, ex, &launches)) != HTTM_OK) return st;
    if (cudaEventRecord(plan->ev_join, s2) != cudaSuccess || cudaStreamWaitEvent(s, plan->ev_join, 0) != cudaSuccess)
      return HTTM_ERR_CUDA;
    bool fused = false;
    st = attention(plan, buf.q_tilde, buf.k_tilde, buf.v_tilde, buf.o_tilde, dims.k_slots, buf, s, &launches,
                   plan->fused_unmerge ? out : nullptr, &fused);
    if (st != HTTM_OK) return st;
    if (!fused) HTTM_LAUNCH(launch_unmerge(dims, fp32, buf, out, s));
    if (dbg) HTTM_LAUNCH(launch_export(dims, plan->blocks_d, buf, dd, s));
    plan->launches = launches;
    return HTTM_OK;
  }
  if (!plan_inj && !reuse) {
    StageTimer t(plan, s, HTTM_STAGE_MATCH, 1);
    cudaError_t e = cudaErrorNotSupported;
    if (match_tc_supported(dims, fp32))
      e = launch_match_tc(dims, plan->blocks_d, plan->tc_items_d, plan->n_tc_items, Q, K, buf, s);
    else
      e = launch_match_simt(dims, fp32, plan->blocks_d, plan->match_items_d, plan->n_match_items, Q, K, buf, s);
    ++launches;
    e = checked(e, s);
    if (e != cudaSuccess) return cuda_fail(e, "matching");
  }
  {
    StageTimer t(plan, s, HTTM_STAGE_MERGE, reuse ? 4 : 5);
    HTTM_LAUNCH(launch_merge(dims, fp32, plan->blocks_d, plan_inj, reuse, Q, K, V, buf, dd, s));
    launches += reuse ? 3 : 4;  // planning (unless reused), then each gather and its big-slot kernel
  }
  {
    const int before = launches;
    StageTimer t(plan, s, HTTM_STAGE_OUTLIER, 0);
    if ((st = filter_stage(plan, Q, mask_inj, buf, dd, s, ex, &launches)) != HTTM_OK) return st;
    t.n = launches - before;
  }
  bool fused = false;
  {
    // with the unmerge fused into the attention epilogue, its time (and its
    // writes of the output) fall in this stage
    StageTimer t(plan, s, HTTM_STAGE_ATTENTION, 1);
    st = attention(plan, buf.q_tilde, buf.k_tilde, buf.v_tilde, buf.o_tilde, dims.k_slots, buf, s, &launches,
                   plan->fused_unmerge ? out : nullptr, &fused);
    if (st != HTTM_OK) return st;
  }
  if (!fused) {
    StageTimer t(plan, s, HTTM_STAGE_UNMERGE, 1);
    HTTM_LAUNCH(launch_unmerge(dims, fp32, buf, out, s));
  }
  if (dbg) {
    StageTimer t(plan, s, HTTM_STAGE_OTHER, 1);
    HTTM_LAUNCH(launch_export(dims, plan->blocks_d, buf, dd, s));
  }
  plan->launches = launches;
  return HTTM_OK;
}

// From each block's destination / merge counts (q_ndst, k_ndst, q_r, k_r):
// the source and slot offsets, the plan's sizes and outlier budget, and the
// matching work lists (CUDA-core: 128-source tiles of every (tensor, block);
// tensor cores: one CTA per (tensor, head, block), a block split in runs of
// whole 128-source tiles when that gives too few CTAs; costliest first).
void finish_blocks(httm_plan_s* p) {
  const httm_cfg& c = p->cfg;
  Dims& d = p->dims;
  std::vector<BlockDesc>& B = p->blocks_h;
  int qs = 0, ks = 0, qsl = 0, ksl = 0;
  d.max_ndst = d.max_nsrc = d.max_nb = 0;
  for (BlockDesc& b : B) {
    b.q_src_off = qs;
    b.k_src_off = ks;
    b.q_slot_off = qsl;
    b.k_slot_off = ksl;
    qs += b.n_b - b.q_ndst;
    ks += b.n_b - b.k_ndst;
    qsl += b.n_b - b.q_r;
    ksl += b.n_b - b.k_r;
    d.max_ndst = std::max(d.max_ndst, std::max(b.q_ndst, b.k_ndst));
    d.max_nsrc = std::max(d.max_nsrc, std::max(b.n_b - b.q_ndst, b.n_b - b.k_ndst));
    d.max_nb = std::max(d.max_nb, b.n_b);
  }
  d.q_src = qs;
  d.k_src = ks;
  d.q_slots = qsl;
  d.k_slots = ksl;
  size_outliers(d, c.outlier_pct);
  std::vector<int4> items;
  for (int t = 0; t < 2; ++t)
    for (int bi = 0; bi < d.nblk; ++bi) {
      const BlockDesc& b = B[bi];
      const int ns = b.n_b - (t == 0 ? b.q_ndst : b.k_ndst);
      for (int s0 = 0; s0 < ns; s0 += 128) items.push_back(make_int4(t, bi, s0, std::min(128, ns - s0)));
    }
  std::stable_sort(items.begin(), items.end(), [&](const int4& a, const int4& b) {
    const int ca = a.x == 0 ? B[a.y].q_ndst : B[a.y].k_ndst;
    const int cb = b.x == 0 ? B[b.y].q_ndst : B[b.y].k_ndst;
    return ca > cb;
  });
  p->n_match_items = (int)items.size();
  p->items_h = std::move(items);
  // (head-uniform: one item list for all heads, item.x = tensor; a block
  // without destinations, possible under HTTM_PARTITION, needs no matching)
  std::vector<int4> tci;
  const int hs = c.mode == HTTM_HEAD_UNIFORM ? 1 : c.h;
  const int parts_want = std::max(1, (4 * 148 + 2 * d.nblk * hs - 1) / (2 * d.nblk * hs));
  for (int hh = 0; hh < hs; ++hh)
    for (int t = 0; t < 2; ++t)
      for (int bi = 0; bi < d.nblk; ++bi) {
        const BlockDesc& b = B[bi];
        const int nd = t == 0 ? b.q_ndst : b.k_ndst;
        if (nd == 0) continue;
        const int ns = b.n_b - nd;
        const int tiles = (ns + 127) / 128;
        const int parts = std::max(1, std::min(parts_want, tiles));
        const int per = (tiles + parts - 1) / parts;
        for (int t0 = 0; t0 < tiles; t0 += per) {
          const int s0 = t0 * 128, n = std::min(per * 128, ns - s0);
          tci.push_back(make_int4(t + 2 * hh, bi, s0, n));
        }
      }
  // query items first, then key items; each costliest first
  std::stable_sort(tci.begin(), tci.end(), [&](const int4& a, const int4& b) {
    if ((a.x & 1) != (b.x & 1)) return (a.x & 1) < (b.x & 1);
    const long long ca = (long long)((a.x & 1) == 0 ? B[a.y].q_ndst : B[a.y].k_ndst) * a.w;
    const long long cb = (long long)((b.x & 1) == 0 ? B[b.y].q_ndst : B[b.y].k_ndst) * b.w;
    return ca > cb;
  });
  p->n_tc_q = (int)std::count_if(tci.begin(), tci.end(), [](const int4& a) { return (a.x & 1) == 0; });
  p->n_tc_items = (int)tci.size();
  p->tc_items_h = std::move(tci);
}

}  // namespace

extern "C" {

const char* httm_status_str(httm_status s) {
  switch (s) {
    case HTTM_OK: return "ok";
    case HTTM_ERR_ARG: return "invalid argument";
    case HTTM_ERR_UNSUPPORTED: return "unsupported configuration";
    case HTTM_ERR_INFEASIBLE_RATIO: return "merge ratio exceeds the sources of a block";
    case HTTM_ERR_WORKSPACE: return "workspace too small";
    case HTTM_ERR_ALIGN: return "pointer not aligned";
    case HTTM_ERR_CUDA: return "CUDA runtime error";
    case HTTM_ERR_TIMEOUT: return "device wait timed out";
    case HTTM_ERR_DEVICE_BOUNDS: return "device bounds / plan check failed";
    case HTTM_ERR_EXCHANGE: return "the caller's collective failed";
  }
  return "unknown status";
}

httm_status httm_plan(const httm_cfg* cfg, httm_plan_t* out) {
  if (!cfg || !out) return HTTM_ERR_ARG;
  *out = nullptr;
  const httm_cfg c = *cfg;
  if (c.h < 1 || c.h > 64 || c.T < 1 || c.P < 1) return HTTM_ERR_ARG;
  if (c.dtype != HTTM_BF16 && c.dtype != HTTM_F32) return HTTM_ERR_ARG;
  if (c.mode < HTTM_HEADWISE_TEMPORAL || c.mode > HTTM_PARTITION) return HTTM_ERR_ARG;
  if (c.mode == HTTM_PARTITION && (c.dtype != HTTM_BF16 || c.d_head != 64)) return HTTM_ERR_UNSUPPORTED;
  if (c.d_head != 16 && c.d_head != 64) return HTTM_ERR_UNSUPPORTED;
  if (c.softmax_scale < 0.f) return HTTM_ERR_ARG;
  const long long N = (long long)c.T * c.P;
  if (N > (1ll << 30) || (long long)c.h * N > (1ll << 31) - 1) return HTTM_ERR_UNSUPPORTED;
  if (c.mode != HTTM_DENSE) {
    if (c.mode != HTTM_PARTITION) {          // the partition fixes destinations and merges itself
      if (c.q_dst_stride < 2 || c.kv_dst_stride < 2) return HTTM_ERR_ARG;
      if (c.q_merge_pct < 0 || c.q_merge_pct > 100 || c.kv_merge_pct < 0 || c.kv_merge_pct > 100) return HTTM_ERR_ARG;
    }
    if (c.outlier_pct < 0 || c.outlier_pct > 100) return HTTM_ERR_ARG;
    if (c.mode == HTTM_CONTIGUOUS ? c.contig_block < 1 : (c.n_s < 1 || c.n_t < 1)) return HTTM_ERR_ARG;
  }
  httm_plan_s* p = new (std::nothrow) httm_plan_s();
  if (!p) return HTTM_ERR_ARG;
  static std::atomic<uint32_t> next_id{1};
  p->cfg = c;
  p->fp32 = c.dtype == HTTM_F32;
  Dims& d = p->dims;
  d = Dims{};
  d.h = c.h;
  d.N = (int32_t)N;
  d.P = c.P;
  d.d = c.d_head;
  d.mode = c.mode;
  d.n_s = c.n_s;
  d.n_t = c.n_t;
  d.contig = c.contig_block;
  d.q_stride = c.q_dst_stride;
  d.kv_stride = c.kv_dst_stride;
  d.scale = c.softmax_scale > 0.f ? c.softmax_scale : 1.0f / sqrtf((float)c.d_head);
  d.plan_id = next_id.fetch_add(1);
  if (d.plan_id == 0) d.plan_id = next_id.fetch_add(1);
  d.wait_budget_ns = 2000000000ull;
  d.shard = 0;
  d.shards = 1;
  d.nchunk_per_head = (int32_t)((N + kChunk - 1) / kChunk);
  if (c.mode == HTTM_DENSE) {
    d.max_items = (int32_t)(c.h * ((N + kAttnRows - 1) / kAttnRows));
  } else {
    std::vector<BlockDesc>& B = p->blocks_h;
    auto add = [&](int base, int s, int n_b) {
      BlockDesc b{};
      b.base = base;
      b.s = s;
      b.n_b = n_b;
      B.push_back(b);
    };
    if (c.mode == HTTM_CONTIGUOUS) {
      for (long long s0 = 0; s0 < N; s0 += c.contig_block) {
        const int nb = (int)std::min<long long>(c.contig_block, N - s0);
        add((int)s0, nb, nb);
      }
      d.R = 0;
    } else {
      const int G = (c.T + c.n_t - 1) / c.n_t;
      const int R = (c.P + c.n_s - 1) / c.n_s;
      d.R = R;
      for (int g = 0; g < G; ++g) {
        const int t0 = g * c.n_t, tg = std::min(c.n_t, c.T - t0);
        for (int j = 0; j < R; ++j) {
          const int p0 = j * c.n_s, sj = std::min(c.n_s, c.P - p0);
          add(t0 * c.P + p0, sj, tg * sj);
        }
      }
    }
    int tok = 0;
    for (BlockDesc& b : B) {
      if (b.n_b > 8192) {
        delete p;
        return HTTM_ERR_UNSUPPORTED;
      }
      b.tok_off = tok;
      tok += b.n_b;
      if (c.mode == HTTM_PARTITION) continue;     // destinations come from httm_plan_partition
      b.q_ndst = (b.n_b + c.q_dst_stride - 1) / c.q_dst_stride;
      b.k_ndst = (b.n_b + c.kv_dst_stride - 1) / c.kv_dst_stride;
      b.q_r = (int)(((long long)c.q_merge_pct * b.n_b) / 100);
      b.k_r = (int)(((long long)c.kv_merge_pct * b.n_b) / 100);
      if (b.q_r > b.n_b - b.q_ndst || b.k_r > b.n_b - b.k_ndst) {
        delete p;
        return HTTM_ERR_INFEASIBLE_RATIO;
      }
    }
    d.nblk = (int32_t)B.size();
    if (c.mode != HTTM_PARTITION) finish_blocks(p);
  }
  p->ws = layout(d, p->fp32);
  *out = p;
  return HTTM_OK;
}

void httm_plan_destroy(httm_plan_t plan) {
  if (!plan) return;
  for (auto& r : plan->recs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (cudaEvent_t e : plan->pool) cudaEventDestroy(e);
  if (plan->blocks_d) cudaFree(plan->blocks_d);
  if (plan->match_items_d) cudaFree(plan->match_items_d);
  if (plan->tc_items_d) cudaFree(plan->tc_items_d);
  if (plan->roles_d) cudaFree(plan->roles_d);
  if (plan->lists_d) cudaFree(plan->lists_d);
  if (plan->ord_d) cudaFree(plan->ord_d);
  if (plan->counts_d) cudaFree(plan->counts_d);
  if (plan->side) cudaStreamDestroy(plan->side);
  if (plan->ev_fork) cudaEventDestroy(plan->ev_fork);
  if (plan->ev_join) cudaEventDestroy(plan->ev_join);
  delete plan;
}

size_t httm_workspace_bytes(httm_plan_t plan) { return plan ? plan->ws.total : 0; }

httm_status httm_get_plan_info(httm_plan_t plan, httm_plan_info* info) {
  if (!plan || !info) return HTTM_ERR_ARG;
  const Dims& d = plan->dims;
  info->N = d.N;
  info->n_blocks = d.nblk;
  info->q_slots = d.q_slots;
  info->kv_slots = d.k_slots;
  info->k_out_max = d.k_out_max;
  info->q_rows_alloc = d.q_rows_alloc;
  info->ws_q_tilde = (int64_t)plan->ws.q_tilde;
  info->ws_k_tilde = (int64_t)plan->ws.k_tilde;
  info->ws_v_tilde = (int64_t)plan->ws.v_tilde;
  info->ws_o_tilde = (int64_t)plan->ws.o_tilde;
  info->ws_n_out = (int64_t)plan->ws.n_out;
  info->ws_out_base = (int64_t)plan->ws.out_base;
  info->workspace_bytes = (int64_t)plan->ws.total;
  return HTTM_OK;
}

httm_status httm_forward(httm_plan_t plan, const void* Q, const void* K, const void* V, void* out, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return forward_impl(plan, Q, K, V, out, workspace, workspace_bytes, nullptr, nullptr, stream);
}

httm_status httm_forward_debug(httm_plan_t plan, const void* Q, const void* K, const void* V, void* out,
                               void* workspace, size_t workspace_bytes, const httm_debug* dbg, void* stream) {
  if (!dbg) return HTTM_ERR_ARG;
  return forward_impl(plan, Q, K, V, out, workspace, workspace_bytes, nullptr, dbg, stream);
}

httm_status httm_forward_with_plan(httm_plan_t plan, const void* Q, const void* K, const void* V, void* out,
                                   void* workspace, size_t workspace_bytes, const httm_merge_plan* injected,
                                   const httm_debug* dbg, void* stream) {
  if (!injected) return HTTM_ERR_ARG;
  return forward_impl(plan, Q, K, V, out, workspace, workspace_bytes, injected, dbg, stream);
}

httm_status httm_forward_reuse(httm_plan_t plan, const void* Q, const void* K, const void* V, void* out,
                               void* workspace, size_t workspace_bytes, void* stream) {
  return forward_impl(plan, Q, K, V, out, workspace, workspace_bytes, nullptr, nullptr, stream, true);
}

httm_status httm_plan_shard(httm_plan_t plan, int32_t shard, int32_t shards) {
  if (!plan || shards < 1 || shards > kMaxShards || shard < 0 || shard >= shards || plan->device >= 0)
    return HTTM_ERR_ARG;
  if (plan->dims.mode == HTTM_HEAD_UNIFORM && shards > 1) return HTTM_ERR_UNSUPPORTED;
  if (plan->dims.mode == HTTM_PARTITION) return HTTM_ERR_UNSUPPORTED;
  Dims d = plan->dims;
  d.shard = shard;
  d.shards = shards;
  if (d.mode != HTTM_DENSE) {
    size_outliers(d, plan->cfg.outlier_pct);
    if (d.k_out_max > (1ll << 31) - 1 || d.q_rows_alloc > (1ll << 31) - 1) return HTTM_ERR_UNSUPPORTED;
  }
  plan->dims = d;
  plan->ws = layout(d, plan->fp32);
  return HTTM_OK;
}

httm_status httm_forward_sharded(httm_plan_t plan, const void* Q, const void* K, const void* V, void* out,
                                 void* workspace, size_t workspace_bytes, const httm_exchange* ex,
                                 const httm_debug* dbg, void* stream) {
  return forward_impl(plan, Q, K, V, out, workspace, workspace_bytes, nullptr, dbg, stream, false, true, ex);
}

httm_status httm_plan_partition(httm_plan_t plan, const float* score, int32_t ga_pct, uint8_t* roles_out,
                                void* stream) {
  if (!plan || !score || plan->dims.mode != HTTM_PARTITION || ga_pct < 0 || ga_pct > 100) return HTTM_ERR_ARG;
  const httm_cfg& c = plan->cfg;
  int grid = 0;
  while ((grid + 1) * (grid + 1) <= c.P) ++grid;
  if (grid * grid != c.P) return HTTM_ERR_ARG;
  if (c.P > 16384) return HTTM_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return HTTM_ERR_CUDA;
  if (plan->device >= 0 && plan->device != dev) return HTTM_ERR_ARG;
  Dims& d = plan->dims;
  const size_t N = (size_t)d.N;
  const size_t nb = plan->blocks_h.size();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!plan->roles_d) {
    if (cudaMalloc(&plan->roles_d, N) != cudaSuccess || cudaMalloc(&plan->lists_d, N * 4) != cudaSuccess ||
        cudaMalloc(&plan->ord_d, N * 4) != cudaSuccess || cudaMalloc(&plan->counts_d, nb * 8) != cudaSuccess ||
        (!plan->blocks_d && cudaMalloc(&plan->blocks_d, nb * sizeof(BlockDesc)) != cudaSuccess))
      return HTTM_ERR_CUDA;
  }
  // the block geometry (base, s, n_b, tok_off) is all the lists kernel reads
  if (cudaMemcpy(plan->blocks_d, plan->blocks_h.data(), nb * sizeof(BlockDesc), cudaMemcpyHostToDevice) != cudaSuccess)
    return HTTM_ERR_CUDA;
  const int ga_k = (int)(((long long)ga_pct * c.P) / 100);
  if (cudaError_t e = launch_partition(d, c.T, grid, ga_k, score, plan->blocks_d, plan->roles_d, plan->lists_d,
                                       plan->ord_d, plan->counts_d, s);
      e != cudaSuccess)
    return cuda_fail(e, "launch_partition");
  if (roles_out && cudaMemcpyAsync(roles_out, plan->roles_d, N, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return HTTM_ERR_CUDA;
  std::vector<int32_t> counts(2 * nb);
  if (cudaError_t e = cudaStreamSynchronize(s); e != cudaSuccess) return cuda_fail(e, "launch_partition (sync)");
  if (cudaMemcpy(counts.data(), plan->counts_d, nb * 8, cudaMemcpyDeviceToHost) != cudaSuccess) return HTTM_ERR_CUDA;
  // every source merges into its best destination, if its block has one
  for (size_t i = 0; i < nb; ++i) {
    BlockDesc& b = plan->blocks_h[i];
    const int n_dst = counts[2 * i], n_src = counts[2 * i + 1];
    if (n_dst < 0 || n_src < 0 || n_dst + n_src > b.n_b) return HTTM_ERR_DEVICE_BOUNDS;
    b.q_ndst = b.k_ndst = n_dst;
    b.q_r = b.k_r = n_dst > 0 ? n_src : 0;
  }
  finish_blocks(plan);
  if (d.max_ndst > 1280) return HTTM_ERR_UNSUPPORTED;   // the matching kernel stages <= 1280 destination rows
  d.proles = plan->roles_d;
  d.plists = plan->lists_d;
  d.pord = plan->ord_d;
  // upload the sized block table and the matching work list
  const size_t nt = std::max<size_t>(1, plan->tc_items_h.size()) * sizeof(int4);
  if (plan->tc_items_d) cudaFree(plan->tc_items_d);
  plan->tc_items_d = nullptr;
  if (cudaMemcpy(plan->blocks_d, plan->blocks_h.data(), nb * sizeof(BlockDesc), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMalloc(&plan->tc_items_d, nt) != cudaSuccess ||
      (!plan->tc_items_h.empty() &&
       cudaMemcpy(plan->tc_items_d, plan->tc_items_h.data(), plan->tc_items_h.size() * sizeof(int4),
                  cudaMemcpyHostToDevice) != cudaSuccess))
    return HTTM_ERR_CUDA;
  if (plan->device < 0) {
    if (cudaStreamCreateWithFlags(&plan->side, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&plan->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&plan->ev_join, cudaEventDisableTiming) != cudaSuccess)
      return HTTM_ERR_CUDA;
    // the CUDA-core matching list is not used in this mode; a one-entry buffer keeps the invariants
    if (cudaMalloc(&plan->match_items_d, sizeof(int4)) != cudaSuccess) return HTTM_ERR_CUDA;
    plan->device = dev;
  }
  plan->ws = layout(d, plan->fp32);
  plan->partitioned = true;
  return HTTM_OK;
}

httm_status httm_reorder(httm_plan_t plan, const void* X, void* Xb, int inverse, void* stream) {
  if (!plan || !X || !Xb) return HTTM_ERR_ARG;
  if (plan->dims.mode == HTTM_DENSE) return HTTM_ERR_ARG;
  if (!aligned16(X) || !aligned16(Xb)) return HTTM_ERR_ALIGN;
  httm_status st = check_device(plan);
  if (st != HTTM_OK) return st;
  cudaError_t e = launch_reorder(plan->dims, plan->fp32, plan->blocks_d, X, Xb, inverse != 0,
                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HTTM_OK : HTTM_ERR_CUDA;
}

httm_status httm_get_device_status(httm_plan_t plan, void* workspace, void* stream, uint32_t* status) {
  if (!plan || !workspace || !status) return HTTM_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return HTTM_ERR_CUDA;
  DevState* st = reinterpret_cast<DevState*>(static_cast<char*>(workspace) + plan->ws.state);
  uint32_t v = 0;
  if (cudaMemcpy(&v, &st->status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return HTTM_ERR_CUDA;
  if (v && cudaMemset(&st->status, 0, 4) != cudaSuccess) return HTTM_ERR_CUDA;
  *status = v;
  if (v & HTTM_DEV_TIMEOUT) return HTTM_ERR_TIMEOUT;
  if (v) return HTTM_ERR_DEVICE_BOUNDS;
  return HTTM_OK;
}

int32_t httm_forward_launches(httm_plan_t plan) { return plan ? plan->launches : -1; }

const char* httm_last_cuda_error(void) {
  static thread_local char msg[256];
  if (t_last_err == cudaSuccess) return "";
  snprintf(msg, sizeof(msg), "%s: %s (%s)", t_last_where, cudaGetErrorName(t_last_err), cudaGetErrorString(t_last_err));
  return msg;
}

httm_status httm_set_wait_budget(httm_plan_t plan, uint64_t nanoseconds) {
  if (!plan) return HTTM_ERR_ARG;
  plan->dims.wait_budget_ns = nanoseconds;
  return HTTM_OK;
}

httm_status httm_set_fused_unmerge(httm_plan_t plan, int enable) {
  if (!plan) return HTTM_ERR_ARG;
  plan->fused_unmerge = enable != 0;
  return HTTM_OK;
}

httm_status httm_profile_enable(httm_plan_t plan, int enable) {
  if (!plan) return HTTM_ERR_ARG;
  plan->profile = enable != 0;
  return HTTM_OK;
}

httm_status httm_profile_read(httm_plan_t plan, float* ms, int32_t* launches) {
  if (!plan) return HTTM_ERR_ARG;
  if (ms)
    for (int i = 0; i < HTTM_NUM_STAGES; ++i) ms[i] = 0.f;
  if (launches)
    for (int i = 0; i < HTTM_NUM_STAGES; ++i) launches[i] = 0;
  httm_status st = HTTM_OK;
  for (auto& r : plan->recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      st = HTTM_ERR_CUDA;
    if (ms) ms[r.stage] += t;
    if (launches) launches[r.stage] += r.n;
    plan->pool.push_back(r.a);
    plan->pool.push_back(r.b);
  }
  plan->recs.clear();
  return st;
}

}  // extern "C"

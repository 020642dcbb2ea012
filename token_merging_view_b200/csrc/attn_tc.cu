// softmax(Q~ K~^T * scale) V~ on tensor cores (tcgen05 + TMEM + TMA), bf16,
// d_head = 64.
//
// "HTTM: Head-wise Temporal Token Merging for Faster VGGT", overall framework
// and training-strategy section: after merging, attention runs per head on
// the shortened Q~/K~/V~ in bf16 with a FlashAttention-style kernel.  The
// same kernel is the library's dense attention (HTTM_DENSE).
//
// One CTA per work item: up to 256 query rows of one head, as two 128-row
// tiles t = 0, 1.  12 warps = 3 warpgroups:
//   warp 0      TMA producer: both Q tiles once, then K/V tiles of 128 keys
//               into a 4-stage shared-memory ring;
//   warp 1      one thread issues tcgen05.mma:
//                 S = Q_t K_j^T     (M=128, N=128, K=64; A, B in shared memory)
//                 O_t += P V_j      (M=128, N=64, K=128; A = P in TMEM)
//               in the order  PV(0,j), QK(1,j+1), PV(1,j), QK(0,j+2);
//   warps 2, 3  idle;
//   warps 4..7  softmax of tile 0, warps 8..11 softmax of tile 1: one query
//               row per thread (TMEM lane = row).
// Registers: launched at 168 per thread (384 x 168 = 64,512); warpgroup 0
// gives part of its share back (setmaxnreg to 88) and the softmax warpgroups
// take it (208): 128 x 88 + 256 x 208 = 64,512.
// TMEM (512 columns): a ring of three 128-column S buffers [0, 384) -- the
// i-th S product, i = 2j + t, goes to buffer i % 3, and the softmax writes
// that tile's P (bf16 pairs, 64 columns) over the first half of the same
// buffer once S is in registers -- then O_0 [384, 448) and O_1 [448, 512).
// Tensor-core operations complete in issue order: S product i + 3 reuses a
// buffer only after the PV that read P from it, and a softmax sees S for
// (0, j+1) before it finishes (0, j).  A softmax arrives for step j only
// once PV(t, j-1) has completed (and rescales O_t only then).  Two warpgroups keep two softmax warps per SM
// sub-partition busy on the exp unit while the tensor core alternates
// between the tiles.
//
// Softmax: base-2 max, updated lazily -- the exponentials of a tile are taken
// against the max in use, and O_t and the row sum are rescaled (and the tile
// redone) only when they sum above 2^16, i.e. when some score lies more than
// 16 log2 units above that max; P stays below 2^16 and most tiles never touch
// O_t nor compute a max.  Sums use split accumulators for instruction-level
// parallelism.  Every wait is bounded
// (WaitClock: 2 s of global time and 1 s of cycles at the top clock): a wait
// that runs out sets HTTM_DEV_TIMEOUT, the CTA drains its MMAs, frees TMEM
// and exits.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace httm {
namespace {

using namespace tc;

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kD = 64;
constexpr int kStages = 4;
constexpr int kThreads = 384;
constexpr uint32_t kTile = kBN * kD * 2;   // 16 KB: 128 rows x 64 bf16
constexpr uint32_t kColO = 384;             // O_t at kColO + 64 t; S ring buffers at 0, 128, 256

constexpr int kListCap = 8;                 // output tokens of a query row kept in shared memory

struct AttnSmem {
  uint8_t q[2][kTile];
  uint8_t k[kStages][kTile];
  uint8_t v[kStages][kTile];
  int lst_tok[kAttnRows][kListCap];         // fused unmerge: the tokens each query row's output goes to
  int lst_n[kAttnRows];                     // ... how many (more than kListCap: walk the member list)
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[3], p_full[2], o_done[2];
  uint64_t lists_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Fused unmerge: where the rows of O~ go.  out == null: the kernel writes
// the O~ rows and a separate unmerge kernel copies them out.  Otherwise
// every output row is written straight to the tokens it stands for in
// out [h, N, 64] -- the non-outlier members of a regular slot, or the
// outlier itself (HTTM note, key designs 1-2: unmerge copies a merged
// token's output back to each member, in the original order) -- and O~ is
// not written.
struct Scatter {
  __nv_bfloat16* out;
  int N;
  long long out_base;                       // first outlier row of Q~
};

// The tokens whose output is row gr of O~ (head hh), in member order;
// calls put(tok) for each.  Members that are outliers take their own row.
template <class F>
__device__ __forceinline__ void row_targets(const Buffers& buf, const Scatter& sc, int hh, long long gr, F&& put) {
  const size_t tb = (size_t)hh * sc.N;
  if (gr >= sc.out_base) {
    const int tok = buf.o_tok[gr - sc.out_base];
    if (tok >= 0 && tok < sc.N) put(tok);
    else set_status(buf.state, HTTM_DEV_BOUNDS);
    return;
  }
  const int c = buf.q_gcount[gr], gs = buf.q_gstart[gr];
  if (c < 0 || gs < 0 || gs + c > sc.N) {
    set_status(buf.state, HTTM_DEV_BOUNDS);
    return;
  }
  for (int j = 0; j < c; ++j) {
    const int tok = buf.q_members[tb + gs + j];
    if (tok < 0 || tok >= sc.N) {
      set_status(buf.state, HTTM_DEV_BOUNDS);
      continue;
    }
    if (buf.mask[tb + tok] == 0) put(tok);
  }
}

__device__ __forceinline__ void put_row(const Scatter& sc, int hh, int tok, const uint32_t (&packed)[32]) {
  uint4* dst = reinterpret_cast<uint4*>(sc.out + ((size_t)hh * sc.N + tok) * kD);
#pragma unroll
  for (int v = 0; v < 8; ++v)
    dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
}
constexpr size_t kSmemBytes = sizeof(AttnSmem) + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

// Bounded wait that ignores the abort flag (used to drain in-flight MMAs).
__device__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  const WaitClock clk;                                // the fixed 2 s bound, whatever the call's budget
  while (!mbar_try_wait(bar, parity))
    if (clk.expired()) return false;
  return true;
}

// The last, partial wave of work items is split along the keys: with n items
// and S SMs, the r = n mod S items of the last wave each become p CTAs
// (p = min(4, S / r, key tiles)) over consecutive key-tile ranges, so that
// the wave fills more SMs; each part writes O (unnormalised, fp32), its row
// sums and maxima to the partial area, and attn_combine_kernel merges them.
struct SplitPlan {
  int n_full, r, p;   // items [0, n_full) whole; items [n_full, n_full + r) in p parts
};
__device__ __forceinline__ SplitPlan split_plan(int n, int S, int n_kv) {
  const int r = S > 0 ? n % S : 0;
  int p = r > 0 ? min(4, S / r) : 1;
  p = min(p, n_kv);
  if (p <= 1) return SplitPlan{n, 0, 1};
  return SplitPlan{n - r, r, p};
}

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, __nv_bfloat16* __restrict__ O, int Lk, float scale_log2,
               int n_sm, Buffers buf, Scatter sc) {
  const int n_kv_all = (Lk + kBN - 1) / kBN;
  const SplitPlan sp = split_plan((int)buf.state->n_items, n_sm, n_kv_all);
  const int n_cta = sp.n_full + sp.r * sp.p;
  if ((int)blockIdx.x >= n_cta) return;
  if (cta_plan_failed(buf.state)) return;
  // this CTA's item and key tiles [j0, j0 + n_kv); part >= 0 for a split item
  int item = blockIdx.x, part = -1, j0 = 0, n_kv = n_kv_all;
  if ((int)blockIdx.x >= sp.n_full) {
    const int k = blockIdx.x - sp.n_full;
    item = sp.n_full + k / sp.p;
    part = k;                                        // index of the partial result
    const int q = k % sp.p;
    j0 = q * n_kv_all / sp.p;
    n_kv = (q + 1) * n_kv_all / sp.p - j0;
  }
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int4 it = buf.items[item];
  const int hh = it.x, q_row0 = it.y, n_rows = it.z;
  const int kv_row0 = hh * Lk + j0 * kBN;            // first key row of this CTA's range
  DevState* st = buf.state;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int i = 0; i < 3; ++i) mbar_init(&sm.s_full[i], 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.p_full[t], 128);
      mbar_init(&sm.o_done[t], 1);
    }
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.lists_full, 64);
    sm.abort = 0;
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(&sm.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 88;" ::: "memory");
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ producer
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      mbar_arrive_expect_tx(&sm.q_full, 2 * kTile);
      tma_load_2d(sm.q[0], &tq, &sm.q_full, 0, q_row0);
      tma_load_2d(sm.q[1], &tq, &sm.q_full, 0, q_row0 + kBM);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !mbar_wait(&sm.kv_empty[s], ((j / kStages) - 1) & 1, abort, st)) break;
        mbar_arrive_expect_tx(&sm.kv_full[s], 2 * kTile);
        tma_load_2d(sm.k[s], &tk, &sm.kv_full[s], 0, kv_row0 + j * kBN);
        tma_load_2d(sm.v[s], &tv, &sm.kv_full[s], 0, kv_row0 + j * kBN);
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ MMA issue
      constexpr uint32_t id_s = idesc_bf16(kBM, kBN, false, false);
      constexpr uint32_t id_o = idesc_bf16(kBM, kD, false, true);
      // S product i = 2j + t into ring buffer i % 3
      auto issue_qk = [&](int t, int j) {
        const uint32_t q_addr = smem_u32(sm.q[t]);
        const uint32_t k_addr = smem_u32(sm.k[j % kStages]);
        const int bsel = (2 * j + t) % 3;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          umma_bf16(tmem + bsel * kBN, sw128_desc(q_addr + kk * 32, 1024), sw128_desc(k_addr + kk * 32, 1024),
                    id_s, kk > 0);
        umma_commit(&sm.s_full[bsel]);
      };
      auto issue_pv = [&](int t, int j) {
        const uint32_t v_addr = smem_u32(sm.v[j % kStages]);
        const uint32_t p_col = (uint32_t)((2 * j + t) % 3) * kBN;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          umma_bf16_ts(tmem + kColO + t * kD, tmem + p_col + kk * 8, sw128_desc(v_addr + kk * 16 * 128, 1024), id_o,
                       (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&sm.o_done[t]);
      };
      bool ok = mbar_wait(&sm.q_full, 0, abort, st) && mbar_wait(&sm.kv_full[0], 0, abort, st);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        issue_qk(1, 0);
        if (n_kv > 1) {
          ok = mbar_wait(&sm.kv_full[1 % kStages], (1 / kStages) & 1, abort, st);
          if (ok) issue_qk(0, 1);
        }
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        if (!mbar_wait(&sm.p_full[0], j & 1, abort, st)) break;
        tc_fence_after();
        issue_pv(0, j);
        if (j + 1 < n_kv) issue_qk(1, j + 1);          // K_{j+1} arrived before QK(0, j+1)
        if (!mbar_wait(&sm.p_full[1], j & 1, abort, st)) break;
        tc_fence_after();
        issue_pv(1, j);
        umma_commit(&sm.kv_empty[j % kStages]);
        if (j + 2 < n_kv) {
          if (!mbar_wait(&sm.kv_full[(j + 2) % kStages], ((j + 2) / kStages) & 1, abort, st)) break;
          tc_fence_after();
          issue_qk(0, j + 2);
        }
      }
      // every MMA issued above completes before TMEM is released
      umma_commit(&sm.drain);
      drain_wait(&sm.drain, 0);
    } else if ((warp == 2 || warp == 3) && sc.out != nullptr && part < 0) {
      // ---------------------------------------------------- unmerge targets
      // while the main loop runs: each query row's output tokens into
      // shared memory (the epilogue then writes without a global lookup)
      for (int r = threadIdx.x - 64; r < kAttnRows; r += 64) {
        int n = 0;
        if (r < n_rows)
          row_targets(buf, sc, hh, (long long)q_row0 + r, [&](int tok) {
            if (n < kListCap) sm.lst_tok[r][n] = tok;
            ++n;
          });
        sm.lst_n[r] = n;
      }
      mbar_arrive(&sm.lists_full);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 208;" ::: "memory");
    // -------------------------------------------------------------- softmax
    const int t = (warp - 4) >> 2;                      // query tile of this warpgroup
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;                // row inside the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t to = tmem + lane_off + kColO + t * kD;    // this row of O_t
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int qi = 2 * j + t, bsel = qi % 3;              // S product index and its ring buffer
      const uint32_t ts = tmem + lane_off + bsel * kBN;    // this row of S, then of P
      // waits are made warp-uniform: tcgen05.ld/st below need every lane
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[bsel], (qi / 3) & 1, abort, st))) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(ts + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      const int valid = Lk - (j0 + j) * kBN;
      if (valid < kBN) {
#pragma unroll
        for (int i = 0; i < kBN; ++i)
          if (i >= valid) sr[i] = __float_as_uint(-INFINITY);
      }
      // p = 2^(s * c - m) with the max m in use: the affine part and the row
      // sums on packed fp32 pairs, the exponentials on the exp unit.  A row
      // whose exponentials sum above 2^16 has a score more than 16 (log2
      // units) above m -- always so on the first tile, where m = -inf --
      // and makes the warp rescale O and the sum to the row's new max and
      // redo the tile.  Otherwise P stays below 2^16 and O_t is untouched.
      const unsigned long long cc = f2_pack(scale_log2, scale_log2);
      const bool live_row = t * kBM + row < n_rows;
      bool pv_done = j == 0;                              // PV(t, j-1) seen complete
      float rsum = 0.f;
      for (int pass = 0; pass < 2; ++pass) {
        const unsigned long long mm = f2_pack(-m_used, -m_used);
        unsigned long long rs[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) rs[a] = 0ull;         // (0.f, 0.f)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float s0 = __uint_as_float(sr[c * 64 + 2 * i]), s1 = __uint_as_float(sr[c * 64 + 2 * i + 1]);
            const unsigned long long xp = f2_fma(f2_pack(s0, s1), cc, mm);
            float x0, x1;
            f2_unpack(xp, x0, x1);
            const float p0 = ex2(x0), p1 = ex2(x1);
            rs[i & 3] = f2_add(rs[i & 3], f2_pack(p0, p1));
            pk[i] = pack_bf16(p0, p1);
          }
          tmem_st32(ts + c * 32, pk);
        }
        float r0, r1, r2, r3, r4, r5, r6, r7;
        f2_unpack(rs[0], r0, r1);
        f2_unpack(rs[1], r2, r3);
        f2_unpack(rs[2], r4, r5);
        f2_unpack(rs[3], r6, r7);
        rsum = ((r0 + r1) + (r2 + r3)) + ((r4 + r5) + (r6 + r7));
        if (pass == 1) break;
        // rows past the item's end (padding, or the next head's rows) hold
        // whatever the buffer holds: they never ask for a redo, so that the
        // live rows' results do not depend on them.  NaN sums (the first
        // tile's masked tail) count as large.
        const bool need = live_row && !(rsum <= 65536.f);
        if (!__any_sync(0xffffffffu, need)) break;
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < 64; ++i)
          mx[i & 3] = max3(mx[i & 3], __uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]));
        const float mts = max3(mx[0], mx[1], fmaxf(mx[2], mx[3])) * scale_log2;
        const float m_new = fmaxf(m_used, mts);
        const float alpha = ex2(m_used - m_new);
        if (j > 0) {
          if (!pv_done && !__all_sync(0xffffffffu, mbar_wait(&sm.o_done[t], (j - 1) & 1, abort, st))) {
            ok = false;
            break;
          }
          pv_done = true;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t o[32];
            tmem_ld32(to + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(to + c * 32, o);
          }
        }
        l *= alpha;
        m_used = m_new;
      }
      if (!ok) break;
      l += rsum;
      // No arrival for step j before PV(t, j-1) has completed.  Parity waits
      // are exact only while a barrier is at most one phase from the one
      // awaited: this keeps o_done within one phase of every later wait on
      // it (the rescale's, the next step's, the final one -- a two-tile item
      // could otherwise see "phase 1 done" before PV(t, 0) finished), and
      // since PV(t, j-1) follows the close of p_full's phase j-1, no warp can
      // arrive for step j while a slower warp of its warpgroup has not yet
      // arrived for step j-1 (p_full counts arrivals, not steps).
      if (!pv_done && !__all_sync(0xffffffffu, mbar_wait(&sm.o_done[t], (j - 1) & 1, abort, st))) {
        ok = false;
        break;
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[t]);
    }
    const bool done = ok && __all_sync(0xffffffffu, mbar_wait(&sm.o_done[t], (n_kv - 1) & 1, abort, st));
    if (done && part >= 0) {
      // a part of a split item: O unnormalised, the row sum and the max in
      // use, for attn_combine_kernel
      tc_fence_after();
      const int r = t * kBM + row;
      float* dst = buf.attn_part + ((size_t)part * kAttnRows + r) * kAttnPartStride;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        tmem_ld32(to + c * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int v = 0; v < 8; ++v)
          reinterpret_cast<float4*>(dst)[c * 8 + v] =
              make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]), __uint_as_float(o[4 * v + 2]),
                          __uint_as_float(o[4 * v + 3]));
      }
      dst[kD] = l;
      dst[kD + 1] = m_used;
    } else if (done) {
      tc_fence_after();
      const float inv = 1.f / l;
      uint32_t packed[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        tmem_ld32(to + c * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          packed[c * 16 + i] = pack_bf16(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
      }
      const int r = t * kBM + row;
      if (sc.out != nullptr) {
        // fused unmerge: the row goes to each token it stands for
        if (__all_sync(0xffffffffu, mbar_wait(&sm.lists_full, 0, abort, st)) && r < n_rows) {
          const int n = sm.lst_n[r];
          if (n <= kListCap) {
            for (int j = 0; j < n; ++j) put_row(sc, hh, sm.lst_tok[r][j], packed);
          } else {
            row_targets(buf, sc, hh, (long long)q_row0 + r, [&](int tok) { put_row(sc, hh, tok, packed); });
          }
        }
      } else if (r < n_rows) {
        uint4* dst = reinterpret_cast<uint4*>(O + ((size_t)q_row0 + r) * kD);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    if (*abort) {
      // let TMA copies still in flight land before the shared memory goes away
      for (int i = 0; i < 200; ++i) __nanosleep(1000);
    }
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the parts of each split item (see split_plan): with M the largest
// max in use, O = sum_p O_p 2^(m_p - M) / sum_p l_p 2^(m_p - M), in part
// order; rows past the item's end are left alone.
__global__ void __launch_bounds__(kAttnRows)
attn_combine_kernel(__nv_bfloat16* __restrict__ O, int Lk, int n_sm, Buffers buf, Scatter sc) {
  if (plan_failed(buf.state)) return;
  const SplitPlan sp = split_plan((int)buf.state->n_items, n_sm, (Lk + kBN - 1) / kBN);
  for (int i = blockIdx.x; i < sp.r; i += gridDim.x) {
    const int4 it = buf.items[sp.n_full + i];
    for (int r = threadIdx.x; r < it.z; r += blockDim.x) {
      const float* src[4];
      float w[4], mx = -INFINITY, l = 0.f;
      for (int q = 0; q < sp.p; ++q) {
        src[q] = buf.attn_part + ((size_t)(i * sp.p + q) * kAttnRows + r) * kAttnPartStride;
        mx = fmaxf(mx, src[q][kD + 1]);
      }
      for (int q = 0; q < sp.p; ++q) {
        w[q] = ex2(src[q][kD + 1] - mx);
        l = fmaf(src[q][kD], w[q], l);
      }
      const float inv = 1.f / l;
      uint32_t packed[32];
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        float a[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] = 0.f;
        for (int q = 0; q < sp.p; ++q) {
          const float4 x0 = reinterpret_cast<const float4*>(src[q])[2 * v];
          const float4 x1 = reinterpret_cast<const float4*>(src[q])[2 * v + 1];
          a[0] = fmaf(x0.x, w[q], a[0]); a[1] = fmaf(x0.y, w[q], a[1]);
          a[2] = fmaf(x0.z, w[q], a[2]); a[3] = fmaf(x0.w, w[q], a[3]);
          a[4] = fmaf(x1.x, w[q], a[4]); a[5] = fmaf(x1.y, w[q], a[5]);
          a[6] = fmaf(x1.z, w[q], a[6]); a[7] = fmaf(x1.w, w[q], a[7]);
        }
        packed[4 * v] = pack_bf16(a[0] * inv, a[1] * inv);
        packed[4 * v + 1] = pack_bf16(a[2] * inv, a[3] * inv);
        packed[4 * v + 2] = pack_bf16(a[4] * inv, a[5] * inv);
        packed[4 * v + 3] = pack_bf16(a[6] * inv, a[7] * inv);
      }
      if (sc.out != nullptr) {
        row_targets(buf, sc, it.x, (long long)it.y + r, [&](int tok) { put_row(sc, it.x, tok, packed); });
      } else {
        uint4* dst = reinterpret_cast<uint4*>(O + ((size_t)it.y + r) * kD);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
      }
    }
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [rows, 64] bf16 row-major, 128-row x 64-column boxes, 128-byte swizzle;
// rows past the end read as zero.
bool map_rows64(CUtensorMap* m, const void* base, uint64_t rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  cuuint32_t box[2] = {(cuuint32_t)kD, 128};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tma_encode_available() { return encode_fn() != nullptr; }

bool attention_tc_supported(const Dims& dims, bool fp32) {
  return !fp32 && dims.d == kD && tma_encode_available();
}

cudaError_t launch_attention_tc(const Dims& dims, const void* q, const void* k, const void* v, void* o, int Lk,
                                const Buffers& buf, cudaStream_t s, void* unmerge_out) {
  CUtensorMap tq, tk, tv;
  const uint64_t q_rows = dims.mode == HTTM_DENSE ? (uint64_t)dims.h * dims.N : (uint64_t)dims.q_rows_alloc;
  const uint64_t kv_rows = (uint64_t)dims.h * Lk;
  if (!map_rows64(&tq, q, q_rows) || !map_rows64(&tk, k, kv_rows) || !map_rows64(&tv, v, kv_rows))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const float scale_log2 = dims.scale * 1.4426950408889634f;
  static int n_sm_cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidValue;
  int& n_sm = n_sm_cached[dev & 63];
  if (n_sm == 0 && cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaErrorInvalidValue;
  const int S = std::min(n_sm, kMaxAttnParts);
  // up to S extra CTAs for the split parts of the last wave
  const Scatter sc{static_cast<__nv_bfloat16*>(unmerge_out), dims.N, dims.out_base};
  attn_tc_kernel<<<dims.max_items + S, kThreads, kSmemBytes, s>>>(tq, tk, tv, static_cast<__nv_bfloat16*>(o), Lk,
                                                                  scale_log2, S, buf, sc);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_combine_kernel<<<S, kAttnRows, 0, s>>>(static_cast<__nv_bfloat16*>(o), Lk, S, buf, sc);
  return cudaGetLastError();
}

}  // namespace httm

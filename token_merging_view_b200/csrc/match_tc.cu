// Bipartite cosine matching on tensor cores (tcgen05 + TMEM), bf16, d = 64.
//
// "HTTM: Head-wise Temporal Token Merging for Faster VGGT", key design 1:
// per head, Sim = RowNorm(S) . RowNorm(D)^T and every source keeps only its
// most similar destination; key design 2: only inside a block.  Here the
// block's raw source/destination rows feed the MMA (bf16 products are exact,
// sums are fp32), and the normalisation moves to the epilogue:
// argmax_t dot(s, t) / ||t||, score = that / ||s||, so the n_src x n_dst
// similarity matrix never leaves the SM.
//
// One CTA per (tensor, head, block, run of 128-source tiles), 17 warps:
//   warps 0..15 gather rows with cp.async into the 128-byte-swizzled operand
//               layout (all destinations of the block once, then source tiles
//               double-buffered), compute norms, and run the epilogue: warp w
//               reads TMEM lanes 32*(w%4).. (one source row per thread) and the
//               32-column groups g = w/4, w/4 + 4, ... of each chunk, one
//               group's load at a time (a second group in registers spills);
//               running (max, first index).
//               Four warps per TMEM lane quarter keep the argmax, the bound of
//               this kernel (half a packed multiply, a compare and two
//               selects per score),
//               issuing while others wait on TMEM or the MMA;
//   warp 16     allocates TMEM and one thread issues tcgen05.mma: for each
//               source tile, destination chunks of <= 256 columns into two
//               TMEM buffers of 256 fp32 columns.
// Ties keep the lowest destination (strict '>' in ascending column order;
// of the four column parts the lowest index wins equal values).  Every wait
// is bounded.
#include "common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace httm {
namespace {

using namespace tc;

constexpr int kEpiThreads = 512;
constexpr int kParts = kEpiThreads / 128;  // epilogue warps per TMEM lane quarter
constexpr int kThreads = kEpiThreads + 32;
constexpr int kMaxDst = 1280;          // destination rows a block may have on this path
constexpr int kChunkCols = 256;
constexpr uint32_t kRowsTile = 128;
constexpr uint32_t kTileBytes = kRowsTile * 128;

struct MatchSmem {
  uint8_t dst[kMaxDst * 128];          // K-major SW128, 160 KB
  uint8_t src[2][kTileBytes];
  float inv_d[kMaxDst];
  float best_v[kParts][128];
  int best_i[kParts][128];
  uint64_t src_ready[2], full[2], empty[2], drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = sizeof(MatchSmem) + 1024;

__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk) {
  return (row >> 3) * 1024u + (row & 7u) * 128u + ((chunk ^ (row & 7u)) << 4);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const uint32_t n = valid ? 16u : 0u;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory"); }

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  const WaitClock clk;                                // the fixed 2 s bound, whatever the call's budget
  while (!mbar_try_wait(bar, parity))
    if (clk.expired()) return false;
  return true;
}

// item: tensor (0 = Q, 1 = K) + 2 * head, block, first source ordinal, sources
__global__ void __launch_bounds__(kThreads, 1)
match_tc_kernel(Dims dims, const BlockDesc* __restrict__ blocks, const int4* __restrict__ items,
                const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K, Buffers buf) {
  extern __shared__ uint8_t smem_raw[];
  MatchSmem& sm = *reinterpret_cast<MatchSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int4 it = items[blockIdx.x];
  const int hh = it.x >> 1;
  const bool is_q = (it.x & 1) == 0;
  const BlockDesc b = blocks[it.y];
  const int stride = is_q ? dims.q_stride : dims.kv_stride;
  const int ndst = is_q ? b.q_ndst : b.k_ndst;
  const int ndst_pad = (ndst + 63) & ~63;
  const int nchunk = (ndst_pad + kChunkCols - 1) / kChunkCols;
  const int src0 = it.z, nsrc = it.w;
  const int ntile = (nsrc + kRowsTile - 1) / kRowsTile;
  const __nv_bfloat16* Xh = (is_q ? Q : K) + (size_t)hh * dims.N * 64;
  const size_t out_base = (size_t)hh * (is_q ? dims.q_src : dims.k_src) + (is_q ? b.q_src_off : b.k_src_off);
  int32_t* best_out = (is_q ? buf.q_best : buf.k_best) + out_base;
  float* score_out = (is_q ? buf.q_score : buf.k_score) + out_base;
  DevState* st = buf.state;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.src_ready[i], kEpiThreads);
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], kEpiThreads);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    mbar_fence_init();
  }
  if (warp == kEpiThreads / 32) tmem_alloc(&sm.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp == kEpiThreads / 32) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issue
      uint32_t gc = 0;
      bool ok = true;
      const uint32_t dst_addr = smem_u32(sm.dst);
      for (int t = 0; ok && t < ntile; ++t) {
        if (!mbar_wait(&sm.src_ready[t & 1], (t >> 1) & 1, abort, st)) break;
        tc_fence_after();
        const uint32_t src_addr = smem_u32(sm.src[t & 1]);
        for (int c = 0; c < nchunk; ++c, ++gc) {
          const uint32_t bb = gc & 1;
          if (gc >= 2 && !mbar_wait(&sm.empty[bb], ((gc - 2) >> 1) & 1, abort, st)) { ok = false; break; }
          tc_fence_after();
          const int width = min(kChunkCols, ndst_pad - c * kChunkCols);
          const uint32_t idesc = idesc_bf16(128, width, false, false);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem + bb * kChunkCols, sw128_desc(src_addr + kk * 32, 1024),
                      sw128_desc(dst_addr + c * kChunkCols * 128 + kk * 32, 1024), idesc, kk > 0);
          umma_commit(&sm.full[bb]);
        }
      }
      umma_commit(&sm.drain);
      drain_wait(&sm.drain, 0);
    }
  } else {
    // ------------------------------------------------------ gather + epilogue
    const uint32_t dst_addr = smem_u32(sm.dst);
    // destinations (rows padded with zeros to a multiple of 64)
    // in-block indices: i % stride == 0 are the destinations; under
    // HTTM_PARTITION the block's lists name them (destinations, then the rest)
    const int32_t* bl = dims.plists ? dims.plists + b.tok_off : nullptr;
    for (int e = tid; e < ndst_pad * 8; e += kEpiThreads) {
      const int r = e >> 3, ch = e & 7;
      const bool valid = r < ndst;
      const int tok = valid ? block_token(b, bl ? bl[r] : r * stride, dims.P) : b.base;
      cp_async16(dst_addr + swz(r, ch), Xh + (size_t)tok * 64 + ch * 8, valid);
    }
    auto load_tile = [&](int t) {
      const uint32_t base = smem_u32(sm.src[t & 1]);
      for (int e = tid; e < (int)kRowsTile * 8; e += kEpiThreads) {
        const int r = e >> 3, ch = e & 7;
        const int k = src0 + t * kRowsTile + r;
        const bool valid = t * (int)kRowsTile + r < nsrc;
        const int tok = valid ? block_token(b, bl ? bl[ndst + k] : src_index(k, stride), dims.P) : b.base;
        cp_async16(base + swz(r, ch), Xh + (size_t)tok * 64 + ch * 8, valid);
      }
    };
    load_tile(0);
    cp_async_commit();
    const int quarter = warp & 3, part = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    // Abort handling: a failed wait clears `ok` (warp-uniform) and sets the
    // CTA's abort flag; the warp then skips its work but still reaches every
    // named barrier, so no warp waits on one that another warp has left.
    uint32_t gc = 0;
    bool ok = true;
    for (int t = 0; t < ntile; ++t) {
      if (t + 1 < ntile) {
        load_tile(t + 1);
        cp_async_commit();
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      fence_async_smem();
      epi_sync();
      if (t == 0) {
        // destination inverse norms (fp32, fixed order)
        for (int r = tid; r < ndst_pad; r += kEpiThreads) {
          float ss = 0.f;
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 w = *reinterpret_cast<const uint4*>(sm.dst + swz(r, ch));
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float lo = __uint_as_float(ws[q] << 16), hi = __uint_as_float(ws[q] & 0xffff0000u);
              ss = fmaf(lo, lo, ss);
              ss = fmaf(hi, hi, ss);
            }
          }
          sm.inv_d[r] = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
        }
        epi_sync();
      }
      mbar_arrive(&sm.src_ready[t & 1]);
      // this row's inverse norm (used by the warps of column part 0, which
      // write the row's result)
      float inv_s = 0.f;
      if (part == 0) {
        float ss = 0.f;
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 w = *reinterpret_cast<const uint4*>(sm.src[t & 1] + swz(row, ch));
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float lo = __uint_as_float(ws[q] << 16), hi = __uint_as_float(ws[q] & 0xffff0000u);
            ss = fmaf(lo, lo, ss);
            ss = fmaf(hi, hi, ss);
          }
        }
        inv_s = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
      }
      // four running (max, first index) pairs, one per column position mod 4
      // (independent chains), merged below: larger value, lower index
      float bv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      int bx[4] = {0x7fffffff, 0x7fffffff, 0x7fffffff, 0x7fffffff};
      for (int c = 0; c < nchunk; ++c, ++gc) {
        const uint32_t bb = gc & 1;
        if (ok && !__all_sync(0xffffffffu, mbar_wait(&sm.full[bb], (gc >> 1) & 1, abort, st))) {
          ok = false;
          *abort = 1;
        }
        if (!ok) continue;
        tc_fence_after();
        const int width = min(kChunkCols, ndst_pad - c * kChunkCols);   // multiple of 64
        auto scan = [&](const uint32_t (&r)[32], int cb) {
          if (cb + 32 <= ndst) {
            const float4* invp = reinterpret_cast<const float4*>(sm.inv_d + cb);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 iv = invp[q];
              // the scaling on packed pairs: one instruction for two scores, the same products
              float v0, v1, v2, v3;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1])), f2_pack(iv.x, iv.y)),
                        v0, v1);
              f2_unpack(f2_mul(f2_pack(__uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3])),
                               f2_pack(iv.z, iv.w)),
                        v2, v3);
              if (v0 > bv[0]) { bv[0] = v0; bx[0] = cb + 4 * q; }
              if (v1 > bv[1]) { bv[1] = v1; bx[1] = cb + 4 * q + 1; }
              if (v2 > bv[2]) { bv[2] = v2; bx[2] = cb + 4 * q + 2; }
              if (v3 > bv[3]) { bv[3] = v3; bx[3] = cb + 4 * q + 3; }
            }
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              if (cb + q < ndst) {
                const float v = __uint_as_float(r[q]) * sm.inv_d[cb + q];
                if (v > bv[q & 3]) { bv[q & 3] = v; bx[q & 3] = cb + q; }
              }
            }
          }
        };
        // this warp's groups: columns [32 g, 32 g + 32) for g = part, part + kParts (chunks of <= 256)
        const int g0 = part * 32, g1 = (part + kParts) * 32;
        uint32_t r0[32];
        if (g0 < width) {
          tmem_ld32(tmem + lane_off + bb * kChunkCols + g0, r0);
          tmem_wait_ld();
          scan(r0, c * kChunkCols + g0);
        }
        if (g1 < width) {
          tmem_ld32(tmem + lane_off + bb * kChunkCols + g1, r0);
          tmem_wait_ld();
          scan(r0, c * kChunkCols + g1);
        }
        tc_fence_before();
        mbar_arrive(&sm.empty[bb]);
      }
      float best = bv[0];
      int bi = bx[0];
#pragma unroll
      for (int j = 1; j < 4; ++j)
        if (bv[j] > best || (bv[j] == best && bx[j] < bi)) {
          best = bv[j];
          bi = bx[j];
        }
      sm.best_v[part][row] = best;
      sm.best_i[part][row] = bi;
      epi_sync();
      if (part == 0 && ok) {
        const int k = t * kRowsTile + row;
        if (k < nsrc) {
          // the column parts of one row: larger value, lower index on ties
          float v = sm.best_v[0][row];
          int i = sm.best_i[0][row];
#pragma unroll
          for (int p = 1; p < kParts; ++p) {
            const float v1 = sm.best_v[p][row];
            const int i1 = sm.best_i[p][row];
            if (v1 > v || (v1 == v && i1 < i)) {
              v = v1;
              i = i1;
            }
          }
          best_out[src0 + k] = i;
          score_out[src0 + k] = v * inv_s;
        }
      }
      epi_sync();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kEpiThreads / 32) {          // the warp that allocated
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


// Head-uniform variant (one plan per block for every head, ToMe / FastVGGT
// style; HTTM note, background section): the score of a (source,
// destination) pair is the mean over heads of the per-head cosines,
// c(s, t) = (1/h) sum_h dot_h(s, t) / (||s_h|| ||t_h||).  The per-head dot
// products come from the tensor core on the raw bf16 rows (exact products,
// fp32 sums) and the per-head norms are applied in the epilogue, so nothing
// is rounded to bf16 after normalising.  Per (source tile of 128 rows,
// destination chunk of <= 256 columns) the CTA steps through the heads: the
// head's source and destination rows are staged in shared memory (double
// buffered, cp.async), one thread issues S_h = X_s,h X_d,h^T (K = 64) into
// one of two TMEM buffers, and 16 epilogue warps add S_h * inv_s,h *
// inv_t,h into register accumulators (a thread: one row, 64 columns); after
// the last head they take the argmax (strict '>' in ascending column order,
// lowest index across the four column parts on ties) and keep a running
// best over the chunks.  The plan is written for every head.
constexpr int kUChunk = 256;

struct UniformSmem {
  uint8_t src[2][kRowsTile * 128];            // staged source rows of one head (K-major SW128)
  uint8_t dst[2][kUChunk * 128];              // staged destination rows of one head
  float inv_s[2][kRowsTile];
  float inv_t[2][kUChunk];
  float best_v[kParts][128];
  int best_i[kParts][128];
  uint64_t ready[2], full[2], empty[2], drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kUSmemBytes = sizeof(UniformSmem) + 1024;

// item: tensor (0 = Q, 1 = K), block, first source ordinal, sources
__global__ void __launch_bounds__(kThreads, 1)
match_uniform_tc_kernel(Dims dims, const BlockDesc* __restrict__ blocks, const int4* __restrict__ items,
                        const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K, Buffers buf) {
  extern __shared__ uint8_t smem_raw[];
  UniformSmem& sm = *reinterpret_cast<UniformSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int4 it = items[blockIdx.x];
  const bool is_q = it.x == 0;
  const BlockDesc b = blocks[it.y];
  const int H = dims.h;
  const int stride = is_q ? dims.q_stride : dims.kv_stride;
  const int ndst = is_q ? b.q_ndst : b.k_ndst;
  const int ndst_pad = (ndst + 63) & ~63;
  const int nchunk = (ndst_pad + kUChunk - 1) / kUChunk;
  const int src0 = it.z, nsrc = it.w;
  const int ntile = (nsrc + kRowsTile - 1) / kRowsTile;
  const int nstep = ntile * nchunk * H;
  const __nv_bfloat16* X = is_q ? Q : K;
  const int src_off = is_q ? b.q_src_off : b.k_src_off;
  const int nsrc_head = is_q ? dims.q_src : dims.k_src;
  int32_t* best_out = is_q ? buf.q_best : buf.k_best;
  float* score_out = is_q ? buf.q_score : buf.k_score;
  DevState* st = buf.state;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.ready[i], kEpiThreads);
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], kEpiThreads);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    mbar_fence_init();
  }
  if (warp == kEpiThreads / 32) tmem_alloc(&sm.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp == kEpiThreads / 32) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issue
      for (int s = 0; s < nstep; ++s) {
        const int bb = s & 1;
        if (!mbar_wait(&sm.ready[bb], (s >> 1) & 1, abort, st)) break;
        if (s >= 2 && !mbar_wait(&sm.empty[bb], ((s - 2) >> 1) & 1, abort, st)) break;
        tc_fence_after();
        const int c = (s / H) % nchunk;
        const int width = min(kUChunk, ndst_pad - c * kUChunk);
        const uint32_t idesc = idesc_bf16(128, width, false, false);
        const uint32_t sa = smem_u32(sm.src[bb]), da = smem_u32(sm.dst[bb]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tmem + bb * kUChunk, sw128_desc(sa + kk * 32, 1024), sw128_desc(da + kk * 32, 1024), idesc,
                    kk > 0);
        umma_commit(&sm.full[bb]);
      }
      umma_commit(&sm.drain);
      drain_wait(&sm.drain, 0);
    }
  } else {
    // ------------------------------------------------------ gather + epilogue
    // stage step s: head h's source tile and destination chunk
    auto load_step = [&](int s) {
      const int bb = s & 1;
      const int h = s % H, c = (s / H) % nchunk, t = s / (H * nchunk);
      const __nv_bfloat16* Xh = X + (size_t)h * dims.N * 64;
      const uint32_t sb = smem_u32(sm.src[bb]), db = smem_u32(sm.dst[bb]);
      for (int e = tid; e < (int)kRowsTile * 8; e += kEpiThreads) {
        const int r = e >> 3, ch = e & 7;
        const int k = src0 + t * kRowsTile + r;
        const bool valid = t * (int)kRowsTile + r < nsrc;
        const int tok = valid ? block_token(b, src_index(k, stride), dims.P) : b.base;
        cp_async16(sb + swz(r, ch), Xh + (size_t)tok * 64 + ch * 8, valid);
      }
      for (int e = tid; e < kUChunk * 8; e += kEpiThreads) {
        const int r = e >> 3, ch = e & 7;
        const int m = c * kUChunk + r;
        const bool valid = m < ndst;
        const int tok = valid ? block_token(b, m * stride, dims.P) : b.base;
        cp_async16(db + swz(r, ch), Xh + (size_t)tok * 64 + ch * 8, valid);
      }
    };
    auto row_inv = [](const uint8_t* base, int r) {
      float ss = 0.f;
      for (int ch = 0; ch < 8; ++ch) {
        const uint4 w = *reinterpret_cast<const uint4*>(base + swz(r, ch));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float lo = __uint_as_float(ws[q] << 16), hi = __uint_as_float(ws[q] & 0xffff0000u);
          ss = fmaf(lo, lo, ss);
          ss = fmaf(hi, hi, ss);
        }
      }
      return ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
    };
    const int quarter = warp & 3, part = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    float acc[64];
    float bv = -INFINITY;
    int bx = 0x7fffffff;
    load_step(0);
    cp_async_commit();
    for (int s = 0; s < nstep; ++s) {
      const int bb = s & 1;
      const int h = s % H, c = (s / H) % nchunk, t = s / (H * nchunk);
      if (s + 1 < nstep) {
        load_step(s + 1);           // its buffers were last read by step s - 1, complete below
        cp_async_commit();
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      fence_async_smem();
      epi_sync();
      if (tid < kRowsTile) sm.inv_s[bb][tid] = row_inv(sm.src[bb], tid);
      else if (tid < kRowsTile + kUChunk) sm.inv_t[bb][tid - kRowsTile] = row_inv(sm.dst[bb], tid - kRowsTile);
      epi_sync();
      mbar_arrive(&sm.ready[bb]);
      if (h == 0) {
#pragma unroll
        for (int e = 0; e < 64; ++e) acc[e] = 0.f;
      }
      const int width = min(kUChunk, ndst_pad - c * kUChunk);
      if (ok && !__all_sync(0xffffffffu, mbar_wait(&sm.full[bb], (s >> 1) & 1, abort, st))) {
        ok = false;
        *abort = 1;
      }
      if (ok) {
        tc_fence_after();
        const int g0 = part * 64;
        if (g0 < width) {
          const float is = sm.inv_s[bb][row];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t r0[32];
            tmem_ld32(tmem + lane_off + bb * kUChunk + g0 + half * 32, r0);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e)
              acc[half * 32 + e] = fmaf(__uint_as_float(r0[e]) * is, sm.inv_t[bb][g0 + half * 32 + e], acc[half * 32 + e]);
          }
        }
        tc_fence_before();
      }
      mbar_arrive(&sm.empty[bb]);
      if (h == H - 1) {
        // the chunk's mean cosines: this part's argmax joins the running best
        const float inv_h = 1.f / (float)H;
        const int cb = c * kUChunk + part * 64;
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const float v = acc[e] * inv_h;
          if (cb + e < ndst && v > bv) {
            bv = v;
            bx = cb + e;
          }
        }
        if (c == nchunk - 1) {
          // the tile is done: combine the four column parts of each row
          sm.best_v[part][row] = bv;
          sm.best_i[part][row] = bx;
          epi_sync();
          if (part == 0 && ok) {
            const int k = t * kRowsTile + row;
            if (k < nsrc) {
              float v = sm.best_v[0][row];
              int i = sm.best_i[0][row];
#pragma unroll
              for (int p = 1; p < kParts; ++p) {
                const float v1 = sm.best_v[p][row];
                const int i1 = sm.best_i[p][row];
                if (v1 > v || (v1 == v && i1 < i)) {
                  v = v1;
                  i = i1;
                }
              }
              for (int hh = 0; hh < H; ++hh) {
                best_out[(size_t)hh * nsrc_head + src_off + src0 + k] = i;
                score_out[(size_t)hh * nsrc_head + src_off + src0 + k] = v;
              }
            }
          }
          epi_sync();
          bv = -INFINITY;
          bx = 0x7fffffff;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kEpiThreads / 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool tma_encode_available();

bool match_tc_supported(const Dims& dims, bool fp32) {
  return !fp32 && dims.d == 64 && dims.max_ndst <= kMaxDst;
}

cudaError_t launch_match_tc(const Dims& dims, const BlockDesc* blocks, const int4* items, int n_items,
                            const void* Q, const void* K, const Buffers& buf, cudaStream_t s) {
  if (n_items == 0) return cudaSuccess;
  if (dims.mode == HTTM_HEAD_UNIFORM) {
    cudaError_t e = cudaFuncSetAttribute(match_uniform_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kUSmemBytes);
    if (e != cudaSuccess) return e;
    match_uniform_tc_kernel<<<n_items, kThreads, kUSmemBytes, s>>>(
        dims, blocks, items, static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K), buf);
    return cudaGetLastError();
  }
  cudaError_t e = cudaFuncSetAttribute(match_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  match_tc_kernel<<<n_items, kThreads, kSmemBytes, s>>>(
      dims, blocks, items, static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K), buf);
  return cudaGetLastError();
}

}  // namespace httm

// LiteVGGT's token partition as the destination rule inside HTTM's blocks.
//
// "LiteVGGT: Boosting Vanilla VGGT via Geometry-aware Cached Token Merging",
// key designs 1-2: every token carries a geometric importance score (here an
// input, one float per token shared by the heads); per frame the top ga% by
// score are geometry-aware (GA) tokens and never merge; the first frame's
// other tokens are all destinations; in every later frame the lowest-scoring
// non-GA token of each 2x2 cell of the patch grid is a destination; the rest
// are sources, each merging into its most similar destination.  The
// matching stays inside HTTM's temporal blocks and per head ("HTTM:
// Head-wise Temporal Token Merging for Faster VGGT", key designs 1-2), so a
// block's destinations are the destination-class tokens that fall in it.
//
// Readings where the note is silent: GA count floor(ga% * P / 100) per frame;
// score ties go to the lower patch index (GA: higher score first; a cell's
// destination: lower score first); cells start at even rows and columns
// (2x1, 1x2 or 1x1 on an odd edge); first-frame GA tokens stay GA.
//
// roles_kernel: one CTA per frame.  A patch's rank is the number of patches
// with a higher score, or an equal score and a lower index -- exact, no
// float arithmetic -- and rank < k makes it GA.  Then one thread per cell
// picks the cell's lowest-scoring non-GA patch.
// lists_kernel: one CTA per block.  Walking the block's in-block indices in
// order, an exclusive scan splits them into the ascending destination list
// and the ascending list of the others (sources and GA), which the matching
// and planning kernels read in place of the i % stride rule; each token's
// ordinal in its list and the block's counts are written too.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace httm {
namespace {

constexpr int kRoleThreads = 512;
constexpr int kListThreads = 256;

__global__ void __launch_bounds__(kRoleThreads)
roles_kernel(const float* __restrict__ score, int P, int grid, int ga_k, uint8_t* __restrict__ roles) {
  extern __shared__ float s_score[];                 // [P]
  const int t = blockIdx.x;
  const float* sc = score + (size_t)t * P;
  uint8_t* rl = roles + (size_t)t * P;
  for (int p = threadIdx.x; p < P; p += blockDim.x) s_score[p] = sc[p];
  __syncthreads();
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    const float v = s_score[p];
    int rank = 0;
    for (int q = 0; q < P; ++q) {
      const float w = s_score[q];
      rank += (w > v) || (w == v && q < p);
    }
    const bool ga = rank < ga_k;
    rl[p] = ga ? kRoleGA : (t == 0 ? kRoleDst : kRoleSrc);
  }
  if (t == 0) return;
  __syncthreads();
  const int cw = (grid + 1) / 2;
  for (int c = threadIdx.x; c < cw * cw; c += blockDim.x) {
    const int cy = c / cw, cx = c - cy * cw;
    int best = -1;
    float bv = 0.f;
    for (int dy = 0; dy < 2; ++dy)
      for (int dx = 0; dx < 2; ++dx) {
        const int py = 2 * cy + dy, px = 2 * cx + dx;
        if (py >= grid || px >= grid) continue;
        const int p = py * grid + px;
        if (rl[p] == kRoleGA) continue;
        const float v = s_score[p];
        if (best < 0 || v < bv || (v == bv && p < best)) {
          best = p;
          bv = v;
        }
      }
    if (best >= 0) rl[best] = kRoleDst;
  }
}

// counts[2 b] = destinations of block b, counts[2 b + 1] = sources (the
// source class; GA tokens are neither)
__global__ void __launch_bounds__(kListThreads)
lists_kernel(const BlockDesc* __restrict__ blocks, int P, const uint8_t* __restrict__ roles, int32_t* __restrict__ lists,
             int32_t* __restrict__ ord, int32_t* __restrict__ counts) {
  __shared__ uint32_t tmp[40];
  __shared__ uint32_t s_ndst;
  const BlockDesc b = blocks[blockIdx.x];
  // pass 1: destinations and sources of the block
  uint32_t nd = 0, ns = 0;
  for (int i = threadIdx.x; i < b.n_b; i += blockDim.x) {
    const uint8_t r = roles[block_token(b, i, P)];
    nd += r == kRoleDst;
    ns += r == kRoleSrc;
  }
  uint32_t tot;
  block_excl_scan(nd, tmp, &tot);
  const uint32_t ndst = tot;
  block_excl_scan(ns, tmp, &tot);
  if (threadIdx.x == 0) {
    s_ndst = ndst;
    counts[2 * blockIdx.x] = (int32_t)ndst;
    counts[2 * blockIdx.x + 1] = (int32_t)tot;
  }
  __syncthreads();
  // pass 2: in-block order, chunk by chunk: destinations first, then the rest
  int32_t* L = lists + b.tok_off;
  uint32_t dst_before = 0;
  for (int i0 = 0; i0 < b.n_b; i0 += blockDim.x) {
    const int i = i0 + threadIdx.x;
    const bool live = i < b.n_b;
    const int n = live ? block_token(b, i, P) : 0;
    const bool is_dst = live && roles[n] == kRoleDst;
    uint32_t chunk_dst;
    const uint32_t before = block_excl_scan(is_dst ? 1u : 0u, tmp, &chunk_dst) + dst_before;
    if (live) {
      if (is_dst) {
        L[before] = i;
        ord[n] = (int32_t)before;
      } else {
        const uint32_t o = (uint32_t)i - before;     // earlier non-destinations of the block
        L[s_ndst + o] = i;
        ord[n] = (int32_t)o;
      }
    }
    dst_before += chunk_dst;
  }
}

}  // namespace

cudaError_t launch_partition(const Dims& dims, int T, int grid, int ga_k, const float* score, const BlockDesc* blocks,
                             uint8_t* roles, int32_t* lists, int32_t* ord, int32_t* counts, cudaStream_t s) {
  const size_t smem = (size_t)dims.P * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(roles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  roles_kernel<<<T, kRoleThreads, smem, s>>>(score, dims.P, grid, ga_k, roles);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  lists_kernel<<<dims.nblk, kListThreads, 0, s>>>(blocks, dims.P, roles, lists, ord, counts);
  return cudaGetLastError();
}

}  // namespace httm

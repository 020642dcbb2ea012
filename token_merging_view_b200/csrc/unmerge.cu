// Unmerge and temporal (inverse) reordering: pure data movement.
//
// "HTTM: Head-wise Temporal Token Merging for Faster VGGT": unmerge copies
// each merged token's attention output back to every original token it
// stands for (key design 1), and the output is put back in the input order
// (key design 2: unmerge inside the block, then undo the reorder).  Here
// both happen in one gather: out[hh, n] = O~[row of slot(hh, n)], so the
// block order never materialises.
//
// Rows move as 16-byte vectors; a row of d_head elements is
// d_head * sizeof(T) / 16 consecutive lanes, so reads of O~ rows and writes
// of out rows are coalesced within a row.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace httm {
namespace {

constexpr int kUnmergeU = 4;        // tokens per row group and step

// One head per blockIdx.y; each warp copies U consecutive groups of
// 32 / VEC rows (one row per VEC lanes), so the slot lookups of all of them,
// then their row loads, are in flight together.
template <int VEC>
__global__ void __launch_bounds__(256)
unmerge_kernel(Dims dims, const uint4* __restrict__ Ot, uint4* __restrict__ out, Buffers buf) {
  constexpr int RPW = 32 / VEC, U = kUnmergeU;
  if (plan_failed(buf.state)) return;
  const int hh = blockIdx.y;
  const int lane = threadIdx.x & 31, rg = lane / VEC, v = lane % VEC;
  const size_t tokbase = (size_t)hh * dims.N;
  const long long ob = buf.out_base[hh];
  const int t0 = (blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * RPW * U;
  size_t row[U];
  bool ok[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int n = t0 + u * RPW + rg;
    ok[u] = n < dims.N;
    row[u] = 0;
    if (ok[u]) {
      const size_t tok = tokbase + n;
      const int32_t rs = buf.q_slot[tok], ro = buf.q_orank[tok];
      const long long r = buf.mask[tok] ? ob + ro : (long long)hh * dims.q_slots + rs;
      if ((buf.mask[tok] ? (ro < 0) : (rs < 0 || rs >= dims.q_slots)) || r < 0 || r >= dims.q_rows_alloc) {
        set_status(buf.state, HTTM_DEV_BOUNDS);
        ok[u] = false;
      } else {
        row[u] = (size_t)r;
      }
    }
  }
  uint4 x[U];
#pragma unroll
  for (int u = 0; u < U; ++u)
    if (ok[u]) x[u] = __ldg(Ot + row[u] * VEC + v);
#pragma unroll
  for (int u = 0; u < U; ++u)
    if (ok[u]) out[(tokbase + t0 + u * RPW + rg) * VEC + v] = x[u];
}

template <int VEC>
__global__ void __launch_bounds__(256)
reorder_kernel(Dims dims, const BlockDesc* __restrict__ blocks, const uint4* __restrict__ X, uint4* __restrict__ Xb,
               int inverse) {
  const BlockDesc b = blocks[blockIdx.x];
  const int hh = blockIdx.y;
  const size_t hb = (size_t)hh * dims.N;
  for (int e = threadIdx.x; e < b.n_b * VEC; e += blockDim.x) {
    const int i = e / VEC, v = e - (e / VEC) * VEC;
    const size_t n = hb + block_token(b, i, dims.P);
    const size_t q = hb + b.tok_off + i;
    if (!inverse) Xb[q * VEC + v] = __ldg(X + n * VEC + v);
    else Xb[n * VEC + v] = __ldg(X + q * VEC + v);
  }
}

}  // namespace

cudaError_t launch_unmerge(const Dims& dims, bool fp32, const Buffers& buf, void* out, cudaStream_t s) {
  const int row_bytes = dims.d * (fp32 ? 4 : 2);
  const int vec = row_bytes / 16;
  const int per_cta = 8 * (32 / vec) * kUnmergeU;   // tokens per CTA of 8 warps
  const dim3 grid((unsigned)((dims.N + per_cta - 1) / per_cta), (unsigned)dims.h);
  switch (vec) {
    case 2: unmerge_kernel<2><<<grid, 256, 0, s>>>(dims, (const uint4*)buf.o_tilde, (uint4*)out, buf); break;
    case 4: unmerge_kernel<4><<<grid, 256, 0, s>>>(dims, (const uint4*)buf.o_tilde, (uint4*)out, buf); break;
    case 8: unmerge_kernel<8><<<grid, 256, 0, s>>>(dims, (const uint4*)buf.o_tilde, (uint4*)out, buf); break;
    case 16: unmerge_kernel<16><<<grid, 256, 0, s>>>(dims, (const uint4*)buf.o_tilde, (uint4*)out, buf); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_reorder(const Dims& dims, bool fp32, const BlockDesc* blocks, const void* X, void* Xb,
                           bool inverse, cudaStream_t s) {
  const int row_bytes = dims.d * (fp32 ? 4 : 2);
  dim3 grid(dims.nblk, dims.h);
  const int inv = inverse ? 1 : 0;
  switch (row_bytes / 16) {
    case 2: reorder_kernel<2><<<grid, 256, 0, s>>>(dims, blocks, (const uint4*)X, (uint4*)Xb, inv); break;
    case 4: reorder_kernel<4><<<grid, 256, 0, s>>>(dims, blocks, (const uint4*)X, (uint4*)Xb, inv); break;
    case 8: reorder_kernel<8><<<grid, 256, 0, s>>>(dims, blocks, (const uint4*)X, (uint4*)Xb, inv); break;
    case 16: reorder_kernel<16><<<grid, 256, 0, s>>>(dims, blocks, (const uint4*)X, (uint4*)Xb, inv); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace httm

// Unmerge and temporal (inverse) reordering: pure data movement.
//
// "HTTM: Head-wise Temporal Token Merging for Faster VGGT": unmerge copies
// each merged token's attention output back to every original token it
// stands for (key design 1), and the output is put back in the input order
// (key design 2: unmerge inside the block, then undo the reorder).  Here
// both happen in one gather: out[hh, n] = O~[row of slot(hh, n)], so the
// block order never materialises.
//
// Each 16-byte vector is one thread's work; a row of d_head elements is
// d_head * sizeof(T) / 16 consecutive threads, so reads of O~ rows and
// writes of out rows are coalesced within a row.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace httm {
namespace {

template <int VEC>
__global__ void __launch_bounds__(256)
unmerge_kernel(Dims dims, const uint4* __restrict__ Ot, uint4* __restrict__ out, Buffers buf) {
  if (plan_failed(buf.state)) return;
  const size_t total = (size_t)dims.h * dims.N * VEC;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const size_t tok = i / VEC;
    const int v = (int)(i - tok * VEC);
    const int hh = (int)(tok / dims.N);
    const int32_t s = buf.mask[tok] ? dims.q_slots + buf.q_orank[tok] : buf.q_slot[tok];
    size_t row;
    if (s < dims.q_slots) row = (size_t)hh * dims.q_slots + s;
    else row = (size_t)buf.out_base[hh] + (s - dims.q_slots);
    if (s < 0 || row >= (size_t)dims.q_rows_alloc) {
      set_status(buf.state, HTTM_DEV_BOUNDS);
      continue;
    }
    out[i] = __ldg(Ot + row * VEC + v);
  }
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
  const size_t total = (size_t)dims.h * dims.N * (row_bytes / 16);
  const int grid = (int)std::max<size_t>(1, std::min<size_t>((total + 255) / 256, 148 * 8));
  switch (row_bytes / 16) {
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

// softmax(Q~ K~^T * scale) V~ on the shortened sequences, CUDA-core version.
//
// "HTTM: Head-wise Temporal Token Merging for Faster VGGT", overall
// framework: attention runs on the merged Q~/K~/V~ of each head.  This
// kernel is the fp32 path (and the d_head = 16 path); bf16 with d_head = 64
// runs on the tensor-core kernel in attn_tc.cu.
//
// One thread per query row; keys/values are staged in shared memory in
// tiles of kKeys; the softmax is the usual running-max form in base 2,
// with exp2 of (score * scale * log2(e) - running max).
#include "common.cuh"
#include "launch.h"

namespace httm {
namespace {

constexpr int kKeys = 32;

template <class T, int D>
__global__ void __launch_bounds__(kAttnRows)
attn_simt_kernel(Dims dims, const T* __restrict__ Qb, const T* __restrict__ Kb, const T* __restrict__ Vb,
                 T* __restrict__ Ob, int Lk, Buffers buf) {
  __shared__ float ks[kKeys][D];
  __shared__ float vs[kKeys][D];
  if (blockIdx.x >= buf.state->n_items || cta_plan_failed(buf.state)) return;
  const int4 it = buf.items[blockIdx.x];
  const int hh = it.x;
  const bool live = (int)threadIdx.x < it.z;
  const size_t row = (size_t)it.y + threadIdx.x;
  const float sl2 = dims.scale * 1.4426950408889634f;
  float q[D], o[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    q[c] = live ? to_f(Qb[row * D + c]) * sl2 : 0.f;
    o[c] = 0.f;
  }
  float mrun = -INFINITY, l = 0.f;
  const T* Kh = Kb + (size_t)hh * Lk * D;
  const T* Vh = Vb + (size_t)hh * Lk * D;
  for (int j0 = 0; j0 < Lk; j0 += kKeys) {
    const int nj = min(kKeys, Lk - j0);
    for (int e = threadIdx.x; e < kKeys * D; e += blockDim.x) {
      const int j = e / D, c = e - j * D;
      ks[j][c] = j < nj ? to_f(Kh[(size_t)(j0 + j) * D + c]) : 0.f;
      vs[j][c] = j < nj ? to_f(Vh[(size_t)(j0 + j) * D + c]) : 0.f;
    }
    __syncthreads();
    float s[kKeys];
    float mt = mrun;
#pragma unroll
    for (int j = 0; j < kKeys; ++j) {
      float a = 0.f;
#pragma unroll
      for (int c = 0; c < D; ++c) a = fmaf(q[c], ks[j][c], a);
      s[j] = j < nj ? a : -INFINITY;
      mt = fmaxf(mt, s[j]);
    }
    const float alpha = exp2f(mrun - mt);
    l *= alpha;
#pragma unroll
    for (int c = 0; c < D; ++c) o[c] *= alpha;
#pragma unroll
    for (int j = 0; j < kKeys; ++j) {
      const float p = exp2f(s[j] - mt);
      l += p;
#pragma unroll
      for (int c = 0; c < D; ++c) o[c] = fmaf(p, vs[j][c], o[c]);
    }
    mrun = mt;
    __syncthreads();
  }
  if (live) {
    const float inv = 1.f / l;
#pragma unroll
    for (int c = 0; c < D; ++c) Ob[row * D + c] = from_f<T>(o[c] * inv);
  }
}

template <class T, int D>
cudaError_t launch_t(const Dims& dims, const void* q, const void* k, const void* v, void* o, int Lk,
                     const Buffers& buf, cudaStream_t s) {
  attn_simt_kernel<T, D><<<dims.max_items, kAttnRows, 0, s>>>(dims, (const T*)q, (const T*)k, (const T*)v,
                                                              (T*)o, Lk, buf);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_simt(const Dims& dims, bool fp32, const void* q, const void* k, const void* v,
                                  void* o, int Lk, const Buffers& buf, cudaStream_t s) {
  if (fp32) {
    if (dims.d == 16) return launch_t<float, 16>(dims, q, k, v, o, Lk, buf, s);
    return launch_t<float, 64>(dims, q, k, v, o, Lk, buf, s);
  }
  if (dims.d == 16) return launch_t<__nv_bfloat16, 16>(dims, q, k, v, o, Lk, buf, s);
  return launch_t<__nv_bfloat16, 64>(dims, q, k, v, o, Lk, buf, s);
}

}  // namespace httm

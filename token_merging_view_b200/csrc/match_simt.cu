// Bipartite cosine matching inside a merge block, CUDA-core version.
//
// "HTTM: Head-wise Temporal Token Merging for Faster VGGT", key design 1:
// Sim = RowNorm(S) . RowNorm(D)^T per head, and every source keeps only its
// most similar destination.  This kernel serves the fp32 path and the
// head-uniform variant (one plan per block from the head-mean cosine); the
// bf16 head-wise path uses the tensor-core kernel in match_tc.cu.
//
// Numerics: norms and dot products accumulate in fp32 in a fixed order.  The
// argmax compares dot * (1 / ||d||) over destinations in ascending order with
// a strict '>', so ties keep the lowest destination; score = that value times
// 1 / ||s||.  A zero row has inverse norm 0, hence cosine 0.
#include "common.cuh"
#include "launch.h"

namespace httm {
namespace {

constexpr int kThreads = 128;   // one source row per thread
constexpr int kDstChunk = 32;   // destinations staged per step

template <class T, int D>
__device__ __forceinline__ float load_row_norm(const T* row, float (&x)[D]) {
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < D; ++c) {
    x[c] = to_f(row[c]);
    ss = fmaf(x[c], x[c], ss);
  }
  return ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
}

// Stage destinations [c0, c0 + kDstChunk) of (head hh, block b) as fp32 rows
// plus their inverse norms.
template <class T, int D>
__device__ __forceinline__ void stage_dst(const T* Xh, const BlockDesc& b, int P, int stride,
                                          int ndst, int c0, float (*sm)[D + 1], float* sinv) {
  for (int e = threadIdx.x; e < kDstChunk * D; e += blockDim.x) {
    int j = e / D, c = e - j * D;
    int m = c0 + j;
    float v = 0.f;
    if (m < ndst) v = to_f(Xh[(size_t)block_token(b, m * stride, P) * D + c]);
    sm[j][c] = v;
  }
  __syncthreads();
  if (threadIdx.x < kDstChunk) {
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < D; ++c) ss = fmaf(sm[threadIdx.x][c], sm[threadIdx.x][c], ss);
    sinv[threadIdx.x] = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
  }
  __syncthreads();
}

template <class T, int D, bool UNIFORM>
__global__ void __launch_bounds__(kThreads)
match_simt_kernel(Dims dims, const BlockDesc* __restrict__ blocks, const int4* __restrict__ items,
                  const T* __restrict__ Q, const T* __restrict__ K, Buffers buf) {
  __shared__ float sm[kDstChunk][D + 1];
  __shared__ float sinv[kDstChunk];
  const int4 it = items[blockIdx.x];           // tensor, block, first source, sources
  const bool is_q = it.x == 0;
  const BlockDesc b = blocks[it.y];
  const int stride = is_q ? dims.q_stride : dims.kv_stride;
  const int ndst = is_q ? b.q_ndst : b.k_ndst;
  const int src_off = is_q ? b.q_src_off : b.k_src_off;
  const int nsrc_head = is_q ? dims.q_src : dims.k_src;
  const T* X = is_q ? Q : K;
  int32_t* best_out = is_q ? buf.q_best : buf.k_best;
  float* score_out = is_q ? buf.q_score : buf.k_score;
  const int k = it.z + threadIdx.x;
  const bool live = threadIdx.x < it.w;
  const int src_tok = live ? block_token(b, src_index(k, stride), dims.P) : b.base;

  float best = -INFINITY, score = 0.f;
  int bi = 0;
  if (!UNIFORM) {
    const int hh = blockIdx.y;
    const T* Xh = X + (size_t)hh * dims.N * D;
    float x[D];
    const float inv_s = load_row_norm<T, D>(Xh + (size_t)src_tok * D, x);
    for (int c0 = 0; c0 < ndst; c0 += kDstChunk) {
      stage_dst<T, D>(Xh, b, dims.P, stride, ndst, c0, sm, sinv);
      const int nj = min(kDstChunk, ndst - c0);
      for (int j = 0; j < nj; ++j) {
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < D; ++c) dot = fmaf(x[c], sm[j][c], dot);
        const float v = dot * sinv[j];
        if (v > best) { best = v; bi = c0 + j; }
      }
      __syncthreads();
    }
    score = best * inv_s;
    if (live) {
      best_out[(size_t)hh * nsrc_head + src_off + k] = bi;
      score_out[(size_t)hh * nsrc_head + src_off + k] = score;
    }
  } else {
    // Head-uniform: c_bar(s, t) = (1/h) sum_h cos_h(s, t), one plan for all heads.
    for (int c0 = 0; c0 < ndst; c0 += kDstChunk) {
      float acc[kDstChunk];
#pragma unroll
      for (int j = 0; j < kDstChunk; ++j) acc[j] = 0.f;
      for (int hh = 0; hh < dims.h; ++hh) {
        const T* Xh = X + (size_t)hh * dims.N * D;
        float x[D];
        const float inv_s = load_row_norm<T, D>(Xh + (size_t)src_tok * D, x);
        stage_dst<T, D>(Xh, b, dims.P, stride, ndst, c0, sm, sinv);
#pragma unroll
        for (int j = 0; j < kDstChunk; ++j) {
          float dot = 0.f;
#pragma unroll
          for (int c = 0; c < D; ++c) dot = fmaf(x[c], sm[j][c], dot);
          acc[j] += dot * inv_s * sinv[j];
        }
        __syncthreads();
      }
      const int nj = min(kDstChunk, ndst - c0);
#pragma unroll
      for (int j = 0; j < kDstChunk; ++j) {
        const float v = acc[j] / (float)dims.h;
        if (j < nj && v > best) { best = v; bi = c0 + j; }
      }
    }
    score = best;
    if (live) {
      for (int hh = 0; hh < dims.h; ++hh) {
        best_out[(size_t)hh * nsrc_head + src_off + k] = bi;
        score_out[(size_t)hh * nsrc_head + src_off + k] = score;
      }
    }
  }
}

template <class T, int D>
cudaError_t launch_match_simt_t(const Dims& dims, const BlockDesc* blocks, const int4* items,
                                int n_items, const void* Q, const void* K, const Buffers& buf,
                                cudaStream_t stream) {
  if (n_items == 0) return cudaSuccess;
  if (dims.mode == HTTM_HEAD_UNIFORM) {
    match_simt_kernel<T, D, true><<<dim3(n_items, 1), kThreads, 0, stream>>>(
        dims, blocks, items, (const T*)Q, (const T*)K, buf);
  } else {
    match_simt_kernel<T, D, false><<<dim3(n_items, dims.h), kThreads, 0, stream>>>(
        dims, blocks, items, (const T*)Q, (const T*)K, buf);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_match_simt(const Dims& dims, bool fp32, const BlockDesc* blocks,
                              const int4* items, int n_items, const void* Q, const void* K,
                              const Buffers& buf, cudaStream_t stream) {
  if (fp32) {
    if (dims.d == 16) return launch_match_simt_t<float, 16>(dims, blocks, items, n_items, Q, K, buf, stream);
    return launch_match_simt_t<float, 64>(dims, blocks, items, n_items, Q, K, buf, stream);
  }
  if (dims.d == 16) return launch_match_simt_t<__nv_bfloat16, 16>(dims, blocks, items, n_items, Q, K, buf, stream);
  return launch_match_simt_t<__nv_bfloat16, 64>(dims, blocks, items, n_items, Q, K, buf, stream);
}

}  // namespace httm

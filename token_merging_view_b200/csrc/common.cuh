// Device helpers shared by the kernels (element access, block addressing,
// status reporting, warp/block reductions).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/httm.h"
#include "internal.h"

namespace httm {

template <class T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <class T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ void set_status(DevState* st, uint32_t bit) {
  atomicOr(&st->status, bit);
}

// Once a plan check has failed, the later stages of that forward do nothing
// (the output is undefined, and no kernel reads through a broken index).
__device__ __forceinline__ bool plan_failed(const DevState* st) {
  return (*(volatile const uint32_t*)&st->status & HTTM_DEV_BAD_PLAN) != 0u;
}

// The same, read once per CTA so that every thread of the CTA agrees (a
// kernel that may itself set the bit must not let its threads diverge
// around a later __syncthreads).
__device__ __forceinline__ bool cta_plan_failed(const DevState* st) {
  __shared__ int s_failed;
  if (threadIdx.x == 0) s_failed = plan_failed(st) ? 1 : 0;
  __syncthreads();
  return s_failed != 0;
}

// Original token index of in-block index i.
__device__ __forceinline__ int32_t block_token(const BlockDesc& b, int32_t i, int32_t P) {
  int32_t tau = i / b.s;
  return b.base + tau * P + (i - tau * b.s);
}

// (block, in-block index) of original token n.
__device__ __forceinline__ void token_block(const Dims& D, int32_t n, int32_t& blk, int32_t& i) {
  if (D.mode == HTTM_CONTIGUOUS) {
    blk = n / D.contig;
    i = n - blk * D.contig;
    return;
  }
  int32_t t = n / D.P, p = n - (n / D.P) * D.P;
  int32_t g = t / D.n_t, j = p / D.n_s;
  int32_t s = min(D.n_s, D.P - j * D.n_s);
  blk = g * D.R + j;
  i = (t - g * D.n_t) * s + (p - j * D.n_s);
}

// In-block index of source ordinal k and destination ordinal m.
__device__ __forceinline__ int32_t src_index(int32_t k, int32_t stride) {
  return (k / (stride - 1)) * stride + (k % (stride - 1)) + 1;
}
__device__ __forceinline__ int32_t src_ordinal(int32_t i, int32_t stride) {
  return (i / stride) * (stride - 1) + (i % stride) - 1;
}

// Order-preserving map of a float to an unsigned key (larger float, larger key).
__device__ __forceinline__ uint32_t float_order(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// Exclusive scan over the whole thread block (blockDim.x a multiple of 32,
// at most 1024).  `tmp` holds >= 33 words of shared memory.  Returns the
// exclusive prefix of v; *total receives the block sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* tmp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  uint32_t inc = warp_incl_scan(v);
  if (lane == 31) tmp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < nw ? tmp[lane] : 0u;
    uint32_t wi = warp_incl_scan(w);
    if (lane < nw) tmp[lane] = wi - w;
    if (lane == 31) tmp[32] = wi;
  }
  __syncthreads();
  uint32_t r = inc - v + tmp[warp];
  *total = tmp[32];
  __syncthreads();
  return r;
}

// One full warp: the bin holding the k-th largest element (k >= 1) of a
// histogram hist[0, nb), scanned from the top bin down, and k minus the
// number of elements in higher bins.  Every lane gets the result.
__device__ __forceinline__ void warp_select_bin(const uint32_t* hist, int nb, uint32_t k, int* bin, uint32_t* krem) {
  const int lane = threadIdx.x & 31;
  uint32_t above = 0;
  for (int top = nb - 1; top >= 0; top -= 32) {
    const int bb = top - lane;
    const uint32_t c = bb >= 0 ? hist[bb] : 0u;
    const uint32_t inc = warp_incl_scan(c);
    const uint32_t tot = __shfl_sync(0xffffffffu, inc, 31);
    if (above + tot >= k) {
      const unsigned ballot = __ballot_sync(0xffffffffu, above + inc >= k);
      const int l = __ffs(ballot) - 1;
      *bin = top - l;
      *krem = k - (above + __shfl_sync(0xffffffffu, inc, l) - __shfl_sync(0xffffffffu, c, l));
      return;
    }
    above += tot;
  }
  *bin = 0;
  *krem = 0;
}

// Bitonic sort (ascending) of n = 2^k 64-bit keys in shared memory by the
// whole thread block.
__device__ __forceinline__ void block_bitonic_sort(unsigned long long* a, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < (n >> 1); t += blockDim.x) {
        int lo = 2 * t - (t & (stride - 1));
        int hi = lo + stride;
        bool up = ((lo & size) == 0);
        unsigned long long x = a[lo], y = a[hi];
        if ((x > y) == up) {
          a[lo] = y;
          a[hi] = x;
        }
      }
      __syncthreads();
    }
  }
}

}  // namespace httm

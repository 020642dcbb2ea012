// Rows of a [rows, D] tensor moved as 16-byte chunks spread over a warp,
// with fp32 arithmetic on them (sums, squared distances) shared by the
// merging, restore and outlier kernels.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

#include "tc_ptx.cuh"

namespace httm {

// A row as 16-byte chunks spread over a warp: CPR chunks per row, RPI rows
// per warp-wide access, EPC elements per chunk.
template <class T, int D>
struct Chunk {
  static constexpr int EPC = 16 / (int)sizeof(T);
  static constexpr int CPR = D / EPC;
  static constexpr int RPI = 32 / CPR;
  static_assert(CPR >= 1 && CPR <= 32 && 32 % CPR == 0, "row must split into 16-byte chunks over a warp");
  __device__ static uint4 load(const T* row, int ch) { return __ldg(reinterpret_cast<const uint4*>(row) + ch); }
  __device__ static void unpack(const uint4& w, float (&v)[EPC]) {
    if constexpr (sizeof(T) == 2) {
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[2 * q] = __uint_as_float(ws[q] << 16);
        v[2 * q + 1] = __uint_as_float(ws[q] & 0xffff0000u);
      }
    } else {
      v[0] = __uint_as_float(w.x); v[1] = __uint_as_float(w.y);
      v[2] = __uint_as_float(w.z); v[3] = __uint_as_float(w.w);
    }
  }
  // acc += row, element by element (pairs of fp32 lanes per instruction:
  // the same sums as one add per element)
  __device__ static void add(float (&acc)[EPC], const uint4& w) {
    float v[EPC];
    unpack(w, v);
#pragma unroll
    for (int e = 0; e < EPC; e += 2) {
      float a0, a1;
      tc::f2_unpack(tc::f2_add(tc::f2_pack(acc[e], acc[e + 1]), tc::f2_pack(v[e], v[e + 1])), a0, a1);
      acc[e] = a0;
      acc[e + 1] = a1;
    }
  }
  // sum over the chunk of (row - mean)^2: even and odd elements in two
  // fp32 lanes, added at the end
  __device__ static float sq_dist(const uint4& w, const float (&mean)[EPC]) {
    float v[EPC];
    unpack(w, v);
    const unsigned long long m1 = tc::f2_pack(-1.f, -1.f);
    unsigned long long ss = 0ull;                      // (0.f, 0.f)
#pragma unroll
    for (int e = 0; e < EPC; e += 2) {
      const unsigned long long d = tc::f2_fma(tc::f2_pack(mean[e], mean[e + 1]), m1, tc::f2_pack(v[e], v[e + 1]));
      ss = tc::f2_fma(d, d, ss);
    }
    float s0, s1;
    tc::f2_unpack(ss, s0, s1);
    return s0 + s1;
  }
  // Sum over the RPI lanes holding the same chunk of different rows; every
  // lane gets the same bits (the butterfly is symmetric).
  __device__ static float across_rows(float v) {
#pragma unroll
    for (int o = CPR; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
  }
  // Sum over the CPR lanes holding one row.
  __device__ static float within_row(float v) {
#pragma unroll
    for (int o = 1; o < CPR; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
  }
  __device__ static void store(T* row, int ch, const float (&v)[EPC]) {
    uint4 w;
    if constexpr (sizeof(T) == 2) {
      uint32_t ws[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
        ws[q] = *reinterpret_cast<const uint32_t*>(&p);
      }
      w = make_uint4(ws[0], ws[1], ws[2], ws[3]);
    } else {
      w = make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]));
    }
    reinterpret_cast<uint4*>(row)[ch] = w;
  }
  __device__ static void store_raw(T* row, int ch, const uint4& w) { reinterpret_cast<uint4*>(row)[ch] = w; }
  __device__ static void store_f32(float* row, int ch, const float (&v)[EPC]) {
#pragma unroll
    for (int e = 0; e < EPC; ++e) row[ch * EPC + e] = v[e];
  }
  __device__ static void store_raw_f32(float* row, int ch, const uint4& w) {
    float v[EPC];
    unpack(w, v);
    store_f32(row, ch, v);
  }
};

}  // namespace httm

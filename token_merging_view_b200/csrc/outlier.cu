// Cross-head adaptive outlier filter, the global selection part.
//
// "HTTM: Head-wise Temporal Token Merging for Faster VGGT", key design 3:
// the deviations of all heads' queries compete for one budget: the top-d%
// form the mask M_o in {0,1}^{h x N}.  Here the budget is
// k = min(floor(d% * h * N / 100), #eligible) and the order is
// (deviation desc, flat index h * N + n asc).
//
// Each query carries a 32-bit key = bits(dev) + 1 if it sits in a group of
// >= 2 tokens, else 0 (dev >= 0, so float bits order like the values).  The
// k-th largest key T is found by a three-digit radix select (11 + 11 + 10
// bits); the first digit's histogram is built by the query merge kernel.
// Then keys > T are outliers, plus the first (k - #{key > T}) keys equal to
// T in flat-index order, found with chunk counts and a scan.  Every step is
// its own launch (no grid-wide barrier, no spin wait), and every count is an
// integer, so the mask is deterministic.
//
// Head sharding: the histograms count this shard's heads only; the caller's
// collective sums them over the shards between the steps, so every shard
// finds the same T and budget.  Keys equal to T are taken in flat-index
// order over the whole layer: each shard counts its own, and the shards
// before it (lower heads) take theirs first.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace httm {
namespace {

__device__ __forceinline__ uint32_t k_total(const Dims& dims, const Buffers& buf) {
  const unsigned long long e = buf.state->n_eligible;
  return (uint32_t)min((unsigned long long)dims.k_out_max, e);
}

// Selected digits of the passes done so far (computed by warp 0 of each CTA).
struct Sel {
  int b1, b2, b3;
  uint32_t k1, k2, k3;
};

// The bin holding the k-th largest key of hist[0, nb) by the whole block
// (each thread owns nb / blockDim.x consecutive bins from the top; one block
// scan finds the owner), and k minus the keys in higher bins.
__device__ void block_select(const uint32_t* hist, int nb, uint32_t k, uint32_t* tmp, int* bin, uint32_t* krem) {
  const int per = nb / blockDim.x;
  const int top = nb - 1 - threadIdx.x * per;
  if (threadIdx.x == 0) {   // k above the histogram's total: bin 0 (the owner, if any, writes after the scan)
    *bin = 0;
    *krem = 0;
  }
  uint32_t s = 0;
  for (int i = 0; i < per; ++i) s += __ldcg(hist + top - i);   // built by other CTAs: read at L2
  uint32_t tot;
  uint32_t above = block_excl_scan(s, tmp, &tot);
  if (above < k && k <= above + s) {
    for (int i = 0; i < per; ++i) {
      const uint32_t c = __ldcg(hist + top - i);
      if (k <= above + c) {
        *bin = top - i;
        *krem = k - above;
        break;
      }
      above += c;
    }
  }
  __syncthreads();
}

// Selected digits of the passes done so far, by every thread of the block
// (blockDim.x = 1024).
__device__ void select_digits(const Buffers& buf, uint32_t k, int passes, Sel* s, uint32_t* tmp) {
  block_select(buf.hist, kHistBins, k, tmp, &s->b1, &s->k1);
  if (passes >= 2) block_select(buf.hist + kHistBins, kHistBins, s->k1, tmp, &s->b2, &s->k2);
  if (passes >= 3) block_select(buf.hist + 2 * kHistBins, 1024, s->k2, tmp, &s->b3, &s->k3);
}

// Histogram of the next digit among keys whose higher digits were selected.
__global__ void __launch_bounds__(1024) hist_pass_kernel(Dims dims, Buffers buf, int pass) {
  __shared__ uint32_t sh[kHistBins];
  __shared__ Sel sel;
  __shared__ uint32_t tmp[40];
  if (cta_plan_failed(buf.state)) return;
  const uint32_t k = k_total(dims, buf);
  if (k == 0) return;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0u;
  select_digits(buf, k, pass - 1, &sel, tmp);
  const size_t total = (size_t)dims.h * dims.N;
  const uint32_t pre = pass == 2 ? (uint32_t)sel.b1 : ((uint32_t)sel.b1 << 11) | (uint32_t)sel.b2;
  const int shift = pass == 2 ? 21 : 10;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const uint32_t key = buf.keys[i];
    if ((key >> shift) == pre) atomicAdd(&sh[pass == 2 ? (key >> 10) & 2047u : key & 1023u], 1u);
  }
  __syncthreads();
  uint32_t* gh = buf.hist + (pass - 1) * kHistBins;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (sh[i]) atomicAdd(&gh[i], sh[i]);
}

// Per chunk of kChunk consecutive queries of one head: #{key > T}, #{key == T}.
__global__ void __launch_bounds__(1024) out_count_kernel(Dims dims, Buffers buf, int mask_injected) {
  __shared__ Sel sel;
  __shared__ uint32_t tmp[40];
  if (cta_plan_failed(buf.state)) return;
  const int c = blockIdx.x;
  const int hh = c / dims.nchunk_per_head, cc = c - hh * dims.nchunk_per_head;
  const int lo = cc * kChunk, hi = min(dims.N, lo + kChunk);
  const size_t base = (size_t)hh * dims.N;
  uint32_t gt = 0, eq = 0, T = 0xffffffffu, need = 0;
  const uint32_t k = k_total(dims, buf);
  if (!mask_injected) {
    if (k > 0) {
      select_digits(buf, k, 3, &sel, tmp);
      T = ((uint32_t)sel.b1 << 21) | ((uint32_t)sel.b2 << 10) | (uint32_t)sel.b3;
      need = sel.k3;
      for (int n = lo + threadIdx.x; n < hi; n += blockDim.x) {
        const uint32_t key = buf.keys[base + n];
        gt += key > T;
        eq += key == T;
      }
    }
  } else {
    for (int n = lo + threadIdx.x; n < hi; n += blockDim.x) {
      if (buf.mask[base + n]) {
        ++gt;
        if (buf.keys[base + n] == 0u) set_status(buf.state, HTTM_DEV_BAD_PLAN);
      }
    }
  }
  uint32_t tot;
  block_excl_scan(gt, tmp, &tot);
  gt = tot;
  block_excl_scan(eq, tmp, &tot);
  eq = tot;
  if (threadIdx.x == 0) {
    buf.chunk[4 * c + 0] = gt;
    buf.chunk[4 * c + 1] = eq;
    if (eq) atomicAdd(&buf.hist[3 * kHistBins + dims.shard], eq);   // this shard's keys equal to T
    if (c == 0) {
      buf.state->sel[0] = T;
      buf.state->sel[1] = need;
      buf.state->sel[2] = k;
    }
  }
}

// One CTA: which equal keys are taken, outlier offsets per chunk and head,
// the outlier row ranges, and the attention work list.
__global__ void __launch_bounds__(1024) out_scan_kernel(Dims dims, Buffers buf) {
  __shared__ uint32_t tmp[40];
  __shared__ int tile_off[65];
  if (cta_plan_failed(buf.state)) return;
  const int tid = threadIdx.x;
  const int cph = dims.nchunk_per_head;
  const int nchunk = dims.h * cph;
  // Equal keys are taken in flat-index order over all heads of the layer:
  // the shards before this one (lower heads) take theirs first.
  const uint32_t* eq_shard = buf.hist + 3 * kHistBins;
  uint32_t before = 0;
  for (int r = 0; r < dims.shard; ++r) before += eq_shard[r];
  const uint32_t need_all = buf.state->sel[1];
  const uint32_t need = need_all > before ? min(need_all - before, eq_shard[dims.shard]) : 0u;
  uint32_t carry = 0;
  for (int base = 0; base < nchunk; base += blockDim.x) {
    const int c = base + tid;
    const uint32_t eq = c < nchunk ? buf.chunk[4 * c + 1] : 0u;
    uint32_t tot;
    const uint32_t ex = block_excl_scan(eq, tmp, &tot) + carry;
    if (c < nchunk) {
      const uint32_t take = need > ex ? min(need - ex, eq) : 0u;
      buf.chunk[4 * c + 2] = take;
      buf.chunk[4 * c + 3] = buf.chunk[4 * c + 0] + take;
    }
    carry += tot;
  }
  __syncthreads();
  for (int hh = 0; hh < dims.h; ++hh) {
    uint32_t run = 0;
    for (int base = 0; base < cph; base += blockDim.x) {
      const int c = hh * cph + base + tid;
      const bool in = base + tid < cph;
      const uint32_t v = in ? buf.chunk[4 * c + 3] : 0u;
      uint32_t tot;
      const uint32_t ex = block_excl_scan(v, tmp, &tot) + run;
      if (in) buf.chunk[4 * c + 3] = ex;
      run += tot;
    }
    if (tid == 0) buf.n_out[hh] = (int32_t)run;
    __syncthreads();
  }
  if (tid == 0) {
    unsigned long long total = 0;
    for (int hh = 0; hh < dims.h; ++hh) total += (uint32_t)buf.n_out[hh];
    if (total > (unsigned long long)dims.k_out_max) {
      set_status(buf.state, HTTM_DEV_BAD_PLAN);
      for (int hh = 0; hh < dims.h; ++hh) buf.n_out[hh] = 0;
      total = 0;
    }
    long long row = dims.out_base;
    int tiles = 0;
    for (int hh = 0; hh < dims.h; ++hh) {
      buf.out_base[hh] = (int32_t)row;
      row += ((buf.n_out[hh] + kAttnRows - 1) / kAttnRows) * kAttnRows;
      tile_off[hh] = tiles;
      tiles += (buf.n_out[hh] + kAttnRows - 1) / kAttnRows;
    }
    tile_off[dims.h] = tiles;
    buf.state->sel[3] = (uint32_t)total;
  }
  __syncthreads();
  // head after head: its regular slot tiles, then its outlier tiles, so
  // that the CTAs reading one head's K~/V~ run close together in time and
  // find them in L2
  const int tq = (dims.q_slots + kAttnRows - 1) / kAttnRows;
  for (int i = tid; i < dims.h * tq; i += blockDim.x) {
    const int hh = i / tq, t = i - hh * tq;
    buf.items[hh * tq + tile_off[hh] + t] =
        make_int4(hh, hh * dims.q_slots + t * kAttnRows, min(kAttnRows, dims.q_slots - t * kAttnRows), 0);
  }
  for (int hh = 0; hh < dims.h; ++hh) {
    const int nt = tile_off[hh + 1] - tile_off[hh];
    for (int t = tid; t < nt; t += blockDim.x)
      buf.items[(hh + 1) * tq + tile_off[hh] + t] =
          make_int4(hh, buf.out_base[hh] + t * kAttnRows, min(kAttnRows, buf.n_out[hh] - t * kAttnRows), 0);
  }
  if (tid == 0) buf.state->n_items = (uint32_t)(dims.h * tq + tile_off[dims.h]);
}

// Per chunk: decide each query, write M_o, give outliers their ranks (the
// slots after the head's regular ones) and copy each outlier's own row into
// its slot of Q~.
template <class T, int D>
__global__ void __launch_bounds__(1024)
out_emit_kernel(Dims dims, const T* __restrict__ Q, Buffers buf, int mask_injected) {
  __shared__ uint32_t tmp[40];
  __shared__ int32_t list[kChunk];                     // this chunk's outliers in rank order
  constexpr int PER = kChunk / 1024;
  if (cta_plan_failed(buf.state)) return;
  const int c = blockIdx.x;
  const int hh = c / dims.nchunk_per_head, cc = c - hh * dims.nchunk_per_head;
  const int lo = cc * kChunk, hi = min(dims.N, lo + kChunk);
  const size_t base = (size_t)hh * dims.N;
  const uint32_t total_out = buf.state->sel[3];
  if (total_out == 0) {
    for (int n = lo + threadIdx.x; n < hi; n += blockDim.x) buf.mask[base + n] = 0;
    return;
  }
  const uint32_t Tk = buf.state->sel[0];
  const uint32_t take = buf.chunk[4 * c + 2];
  const uint32_t obefore = buf.chunk[4 * c + 3];
  const int n0 = lo + threadIdx.x * PER;
  bool gt[PER], eq[PER];
  uint32_t neq = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int n = n0 + j;
    gt[j] = eq[j] = false;
    if (n < hi) {
      if (mask_injected) {
        gt[j] = buf.mask[base + n] != 0;
      } else {
        const uint32_t key = buf.keys[base + n];
        gt[j] = key > Tk;
        eq[j] = key == Tk;
      }
    }
    neq += eq[j];
  }
  uint32_t tot;
  uint32_t eq_rank = block_excl_scan(neq, tmp, &tot);
  bool out[PER];
  uint32_t nout = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    out[j] = gt[j] || (eq[j] && eq_rank < take);
    eq_rank += eq[j];
    nout += out[j];
  }
  uint32_t rank = obefore + block_excl_scan(nout, tmp, &tot);
  const uint32_t cnt = tot;                            // outliers of this chunk, ranks obefore + [0, cnt)
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int n = n0 + j;
    if (n >= hi) continue;
    buf.mask[base + n] = out[j] ? 1 : 0;
    if (out[j]) {
      buf.q_orank[base + n] = (int32_t)rank;
      buf.o_tok[(size_t)buf.out_base[hh] + rank - dims.out_base] = n;
      list[rank - obefore] = n;
      ++rank;
    }
  }
  __syncthreads();
  // each outlier's own row into its slot of Q~, 16-byte vectors spread over
  // the threads (consecutive threads: consecutive parts of one row, then of
  // the next outlier's row)
  constexpr int VEC = (int)(D * sizeof(T) / 16);
  const uint4* Qh = reinterpret_cast<const uint4*>(Q + base * D);
  uint4* Qt = reinterpret_cast<uint4*>(reinterpret_cast<T*>(buf.q_tilde) + ((size_t)buf.out_base[hh] + obefore) * D);
  for (uint32_t e = threadIdx.x; e < cnt * VEC; e += blockDim.x) {
    const uint32_t i = e / VEC, v = e - i * VEC;
    Qt[e] = __ldg(Qh + (size_t)list[i] * VEC + v);
  }
}

__global__ void dense_items_kernel(Dims dims, Buffers buf) {
  const int tq = (dims.N + kAttnRows - 1) / kAttnRows;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < dims.h * tq; i += gridDim.x * blockDim.x) {
    const int hh = i / tq, t = i - hh * tq;
    buf.items[i] = make_int4(hh, hh * dims.N + t * kAttnRows, min(kAttnRows, dims.N - t * kAttnRows), 0);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) buf.state->n_items = (uint32_t)(dims.h * tq);
}

}  // namespace

cudaError_t launch_outlier_pass(const Dims& dims, const Buffers& buf, int pass, cudaStream_t s) {
  const size_t total = (size_t)dims.h * dims.N;
  const int hgrid = (int)std::max<size_t>(1, std::min<size_t>((total + 4095) / 4096, 148 * 2));
  hist_pass_kernel<<<hgrid, 1024, 0, s>>>(dims, buf, pass);
  return cudaGetLastError();
}

cudaError_t launch_outlier_count(const Dims& dims, bool mask_injected, const Buffers& buf, cudaStream_t s) {
  out_count_kernel<<<dims.h * dims.nchunk_per_head, 1024, 0, s>>>(dims, buf, mask_injected ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_outlier(const Dims& dims, bool fp32, const void* Q, bool mask_injected,
                           const Buffers& buf, cudaStream_t s) {
  cudaError_t e;
  if (!mask_injected) {
    if ((e = launch_outlier_pass(dims, buf, 2, s)) != cudaSuccess) return e;
    if ((e = launch_outlier_pass(dims, buf, 3, s)) != cudaSuccess) return e;
  }
  if ((e = launch_outlier_count(dims, mask_injected, buf, s)) != cudaSuccess) return e;
  return launch_outlier_emit(dims, fp32, Q, mask_injected, buf, s);
}

cudaError_t launch_outlier_emit(const Dims& dims, bool fp32, const void* Q, bool mask_injected,
                                const Buffers& buf, cudaStream_t s) {
  const int nchunk = dims.h * dims.nchunk_per_head;
  out_scan_kernel<<<1, 1024, 0, s>>>(dims, buf);
  const int mi = mask_injected ? 1 : 0;
  if (fp32) {
    if (dims.d == 16) out_emit_kernel<float, 16><<<nchunk, 1024, 0, s>>>(dims, (const float*)Q, buf, mi);
    else out_emit_kernel<float, 64><<<nchunk, 1024, 0, s>>>(dims, (const float*)Q, buf, mi);
  } else {
    if (dims.d == 16) out_emit_kernel<__nv_bfloat16, 16><<<nchunk, 1024, 0, s>>>(dims, (const __nv_bfloat16*)Q, buf, mi);
    else out_emit_kernel<__nv_bfloat16, 64><<<nchunk, 1024, 0, s>>>(dims, (const __nv_bfloat16*)Q, buf, mi);
  }
  return cudaGetLastError();
}

cudaError_t launch_dense_items(const Dims& dims, const Buffers& buf, cudaStream_t s) {
  dense_items_kernel<<<148, 256, 0, s>>>(dims, buf);
  return cudaGetLastError();
}

}  // namespace httm

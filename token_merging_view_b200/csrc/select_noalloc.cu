// Allocation-free variant of the global outlier selection.
//
// Same selection as the forward's filter stage ("HTTM: Head-wise Temporal
// Token Merging for Faster VGGT", key design 3, the cross-head adaptive
// outlier filter): among the queries flagged eligible, the
// k = min(floor(pct * h * N / 100), #eligible) with the largest deviation,
// ties by ascending flat index h * N + n.  It differs in
// where its scratch (radix histograms, per-chunk counts, counters) lives:
// not in a caller workspace but in g_select_scratch below, a file-scope
// device array of fixed size, so a call allocates nothing at all.
//
// Host code never hands the array's name to a kernel: in host code that
// name is only a stand-in, not a device address.  The device address comes
// from cudaGetSymbolAddress, taken once per device with that device current,
// and is passed to every kernel as a pointer.
#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace httm {
namespace {

constexpr long long kNaMaxTokens = 1ll << 25;   // h * N limit (33,554,432)
constexpr int kNaMaxHeads = 64;
constexpr int kNaMaxChunks = (int)(kNaMaxTokens / kChunk) + kNaMaxHeads;

struct NaScratch {
  uint32_t n_eligible, k, T, need, total, pad[11];
  uint32_t hist[3][kHistBins];
  uint32_t chunk[kNaMaxChunks][4];     // gt, eq, take, outliers before (within head)
};

// Shared by every call on this device; keeps the last call's contents.
static __device__ __align__(256) unsigned char g_select_scratch[sizeof(NaScratch)];

__device__ __forceinline__ uint32_t na_key(const float* dev, const uint8_t* elig, size_t i) {
  return elig[i] ? __float_as_uint(dev[i]) + 1u : 0u;
}

struct NaSel {
  int b[3];
  uint32_t k[3];
};

__device__ void na_digits(const NaScratch* s, int passes, NaSel* out) {
  if ((threadIdx.x >> 5) != 0) return;
  warp_select_bin(s->hist[0], kHistBins, s->k, &out->b[0], &out->k[0]);
  if (passes >= 2) warp_select_bin(s->hist[1], kHistBins, out->k[0], &out->b[1], &out->k[1]);
  if (passes >= 3) warp_select_bin(s->hist[2], 1024, out->k[1], &out->b[2], &out->k[2]);
}

__global__ void na_zero_kernel(NaScratch* s) {
  uint32_t* p = &s->n_eligible;
  for (int i = threadIdx.x; i < 16 + 3 * kHistBins; i += blockDim.x) p[i] = 0u;
}

// First digit histogram and the eligible count.
__global__ void __launch_bounds__(1024) na_hist1_kernel(const float* dev, const uint8_t* elig, size_t total,
                                                        NaScratch* s) {
  __shared__ uint32_t sh[kHistBins];
  __shared__ uint32_t se;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0u;
  if (threadIdx.x == 0) se = 0u;
  __syncthreads();
  uint32_t ne = 0;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const uint32_t key = na_key(dev, elig, i);
    if (key) {
      atomicAdd(&sh[key >> 21], 1u);
      ++ne;
    }
  }
  ne = __reduce_add_sync(0xffffffffu, ne);
  if ((threadIdx.x & 31) == 0 && ne) atomicAdd(&se, ne);
  __syncthreads();
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (sh[i]) atomicAdd(&s->hist[0][i], sh[i]);
  if (threadIdx.x == 0 && se) atomicAdd(&s->n_eligible, se);
}

__global__ void na_budget_kernel(NaScratch* s, long long k_max) {
  s->k = (uint32_t)min((unsigned long long)k_max, (unsigned long long)s->n_eligible);
}

__global__ void __launch_bounds__(1024) na_hist_kernel(const float* dev, const uint8_t* elig, size_t total,
                                                       NaScratch* s, int pass) {
  __shared__ uint32_t sh[kHistBins];
  __shared__ NaSel sel;
  if (s->k == 0) return;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0u;
  na_digits(s, pass - 1, &sel);
  __syncthreads();
  const uint32_t pre = pass == 2 ? (uint32_t)sel.b[0] : ((uint32_t)sel.b[0] << 11) | (uint32_t)sel.b[1];
  const int shift = pass == 2 ? 21 : 10;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const uint32_t key = na_key(dev, elig, i);
    if ((key >> shift) == pre) atomicAdd(&sh[pass == 2 ? (key >> 10) & 2047u : key & 1023u], 1u);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (sh[i]) atomicAdd(&s->hist[pass - 1][i], sh[i]);
}

__global__ void __launch_bounds__(1024) na_count_kernel(const float* dev, const uint8_t* elig, int N, int cph,
                                                        NaScratch* s) {
  __shared__ NaSel sel;
  __shared__ uint32_t tmp[40];
  const int c = blockIdx.x;
  const int hh = c / cph, cc = c - hh * cph;
  const int lo = cc * kChunk, hi = min(N, lo + kChunk);
  const size_t base = (size_t)hh * N;
  uint32_t gt = 0, eq = 0, T = 0xffffffffu, need = 0;
  if (s->k > 0) {
    na_digits(s, 3, &sel);
    __syncthreads();
    T = ((uint32_t)sel.b[0] << 21) | ((uint32_t)sel.b[1] << 10) | (uint32_t)sel.b[2];
    need = sel.k[2];
    for (int n = lo + threadIdx.x; n < hi; n += blockDim.x) {
      const uint32_t key = na_key(dev, elig, base + n);
      gt += key > T;
      eq += key == T;
    }
  }
  uint32_t tot;
  block_excl_scan(gt, tmp, &tot);
  gt = tot;
  block_excl_scan(eq, tmp, &tot);
  eq = tot;
  if (threadIdx.x == 0) {
    s->chunk[c][0] = gt;
    s->chunk[c][1] = eq;
    if (c == 0) {
      s->T = T;
      s->need = need;
    }
  }
}

__global__ void __launch_bounds__(1024) na_scan_kernel(int h, int cph, NaScratch* s, int32_t* n_out) {
  __shared__ uint32_t tmp[40];
  const int tid = threadIdx.x;
  const int nchunk = h * cph;
  const uint32_t need = s->need;
  uint32_t carry = 0;
  for (int base = 0; base < nchunk; base += blockDim.x) {
    const int c = base + tid;
    const uint32_t eq = c < nchunk ? s->chunk[c][1] : 0u;
    uint32_t tot;
    const uint32_t ex = block_excl_scan(eq, tmp, &tot) + carry;
    if (c < nchunk) {
      const uint32_t take = need > ex ? min(need - ex, eq) : 0u;
      s->chunk[c][2] = take;
      s->chunk[c][3] = s->chunk[c][0] + take;
    }
    carry += tot;
  }
  __syncthreads();
  uint32_t all = 0;
  for (int hh = 0; hh < h; ++hh) {
    uint32_t run = 0;
    for (int base = 0; base < cph; base += blockDim.x) {
      const int c = hh * cph + base + tid;
      const bool in = base + tid < cph;
      const uint32_t v = in ? s->chunk[c][3] : 0u;
      uint32_t tot;
      const uint32_t ex = block_excl_scan(v, tmp, &tot) + run;
      if (in) s->chunk[c][3] = ex;
      run += tot;
    }
    if (tid == 0) n_out[hh] = (int32_t)run;
    all += run;
  }
  if (tid == 0) s->total = all;
}

__global__ void __launch_bounds__(1024) na_emit_kernel(const float* dev, const uint8_t* elig, int N, int cph,
                                                       const NaScratch* s, uint8_t* mask) {
  __shared__ uint32_t tmp[40];
  constexpr int PER = kChunk / 1024;
  const int c = blockIdx.x;
  const int hh = c / cph, cc = c - hh * cph;
  const int lo = cc * kChunk, hi = min(N, lo + kChunk);
  const size_t base = (size_t)hh * N;
  if (s->total == 0) {
    for (int n = lo + threadIdx.x; n < hi; n += blockDim.x) mask[base + n] = 0;
    return;
  }
  const uint32_t T = s->T, take = s->chunk[c][2];
  const int n0 = lo + threadIdx.x * PER;
  bool gt[PER], eq[PER];
  uint32_t neq = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int n = n0 + j;
    const uint32_t key = n < hi ? na_key(dev, elig, base + n) : 0u;
    gt[j] = n < hi && key > T;
    eq[j] = n < hi && key == T;
    neq += eq[j];
  }
  uint32_t tot;
  uint32_t eq_rank = block_excl_scan(neq, tmp, &tot);
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int n = n0 + j;
    const bool out = gt[j] || (eq[j] && eq_rank < take);
    eq_rank += eq[j];
    if (n < hi) mask[base + n] = out ? 1 : 0;
  }
}

std::mutex g_setup_mu;
// Per device: the device address of g_select_scratch and the context it was
// taken in.  A device reset (cudaDeviceReset) destroys the primary context
// and reloads the module in the next one, which may place the array
// elsewhere, so the address is looked up again whenever the device's current
// context is not the one it was taken in.
struct ScratchAddr {
  void* ptr = nullptr;
  void* ctx = nullptr;
};
std::vector<ScratchAddr> g_scratch;

typedef int (*CtxGetCurrentFn)(void**);   // cuCtxGetCurrent (CUresult is an int enum)

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// With the device current: the array's device address in the current
// context (looked up once per device and context).  If no context is current
// yet, the lookup itself initialises the device's primary context.
httm_status scratch_address(NaScratch** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return HTTM_ERR_CUDA;
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return HTTM_ERR_CUDA;
  void* ctx = nullptr;
  if (get(&ctx) != 0) return HTTM_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if ((int)g_scratch.size() <= dev) g_scratch.resize(dev + 1);
  ScratchAddr& a = g_scratch[dev];
  if (!a.ptr || ctx == nullptr || a.ctx != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || p == nullptr) return HTTM_ERR_CUDA;
    if (get(&ctx) != 0 || ctx == nullptr) return HTTM_ERR_CUDA;
    a.ptr = p;
    a.ctx = ctx;
  }
  *out = static_cast<NaScratch*>(a.ptr);
  return HTTM_OK;
}

}  // namespace
}  // namespace httm

using namespace httm;

extern "C" httm_status httm_select_outliers_noalloc(const float* dev, const uint8_t* eligible, int32_t h,
                                                    int32_t N, int32_t outlier_pct, uint8_t* mask,
                                                    int32_t* n_out, void* stream) {
  if (!dev || !eligible || !mask || !n_out) return HTTM_ERR_ARG;
  if (h < 1 || N < 1 || outlier_pct < 0 || outlier_pct > 100) return HTTM_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(dev) & 3u) || (reinterpret_cast<uintptr_t>(n_out) & 3u)) return HTTM_ERR_ALIGN;
  if (h > kNaMaxHeads || (long long)h * N > kNaMaxTokens) return HTTM_ERR_UNSUPPORTED;
  // an error another call left pending is not this call's: leave it for its
  // owner to read, and enqueue nothing
  if (cudaPeekAtLastError() != cudaSuccess) return HTTM_ERR_CUDA;
  NaScratch* s = nullptr;
  httm_status st = scratch_address(&s);
  if (st != HTTM_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const size_t total = (size_t)h * N;
  const int cph = (N + kChunk - 1) / kChunk;
  const int nchunk = h * cph;
  const int grid = (int)std::max<size_t>(1, std::min<size_t>((total + 4095) / 4096, 148 * 2));
  const long long k_max = ((long long)outlier_pct * h * N) / 100;
  na_zero_kernel<<<1, 1024, 0, cs>>>(s);
  na_hist1_kernel<<<grid, 1024, 0, cs>>>(dev, eligible, total, s);
  na_budget_kernel<<<1, 1, 0, cs>>>(s, k_max);
  na_hist_kernel<<<grid, 1024, 0, cs>>>(dev, eligible, total, s, 2);
  na_hist_kernel<<<grid, 1024, 0, cs>>>(dev, eligible, total, s, 3);
  na_count_kernel<<<nchunk, 1024, 0, cs>>>(dev, eligible, N, cph, s);
  na_scan_kernel<<<1, 1024, 0, cs>>>(h, cph, s, n_out);
  na_emit_kernel<<<nchunk, 1024, 0, cs>>>(dev, eligible, N, cph, s, mask);
  return cudaGetLastError() == cudaSuccess ? HTTM_OK : HTTM_ERR_CUDA;
}

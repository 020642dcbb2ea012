// Top-r mean merging inside a block, the query deviation, the restore step
// of the outlier filter, and plan import/export.
//
// "HTTM: Head-wise Temporal Token Merging for Faster VGGT":
//  key design 1 -- the top-r sources by match score merge into their best
//    destination; a merged token is the mean of its members; Q and K merge
//    independently and V follows K's plan;
//  key design 3 -- each query's L2 deviation from its merged token (0 if it
//    was not merged) feeds a global top-d% filter; each outlier is
//    subtracted from its merged token and kept as a token of its own.
//
// One CTA per (block, head).  The top-r choice is a bitonic sort of
// (~order(score), source ordinal), so ties go to the lower in-block index;
// the groups come from a second sort of (best destination, source ordinal),
// which lists every group's members in ascending order.  Sums accumulate in
// fp32 in member order (destination first), or for a slot of more than
// kBigSlot members in a fixed split over a CTA's row groups, so results are
// bit-reproducible.
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "rows.cuh"
#include "tc_ptx.cuh"

namespace httm {
namespace {

constexpr int kMergeThreads = 256;
static_assert(kMergeThreads == 256, "the planning kernel clears and selects 256 radix bins, one per thread");

template <int E>
__device__ __forceinline__ void store_f32(float* row, int lane, int D, const float (&v)[E]) {
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (lane * E + e < D) row[lane * E + e] = v[e];
}

// Exclusive scan of in[0, n) into out[0, n) by the whole block.
__device__ void block_scan_array(const int32_t* in, int32_t* out, int n, uint32_t* tmp) {
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int lo = min(n, (int)threadIdx.x * per), hi = min(n, lo + per);
  uint32_t s = 0;
  for (int i = lo; i < hi; ++i) s += in[i];
  uint32_t tot;
  uint32_t run = block_excl_scan(s, tmp, &tot);
  for (int i = lo; i < hi; ++i) {
    out[i] = run;
    run += in[i];
  }
  __syncthreads();
}

// The bin holding the k-th largest element (k >= 1) of hist[0, nb) and k
// minus the elements in higher bins, by the whole thread block: each thread
// owns nb / blockDim.x consecutive bins from the top, one block scan finds
// the owner.  Results land in *bin / *krem (shared memory).
__device__ void block_select_bin(const uint32_t* hist, int nb, uint32_t k, uint32_t* tmp, int* bin, uint32_t* krem) {
  const int per = nb / blockDim.x;
  const int top = nb - 1 - threadIdx.x * per;
  uint32_t s = 0;
  for (int i = 0; i < per; ++i) s += hist[top - i];
  uint32_t tot;
  uint32_t above = block_excl_scan(s, tmp, &tot);
  if (above < k && k <= above + s) {
    for (int i = 0; i < per; ++i) {
      const uint32_t c = hist[top - i];
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

// Quotient of n by d for n, d < 2^16 as a multiply-high by ceil(2^32 / d):
// exact because n * d < 2^32 keeps the error of the product below 1 / d.
struct SmallDiv {
  unsigned long long m;
  __device__ explicit SmallDiv(uint32_t d) : m(0xFFFFFFFFull / d + 1ull) {}
  __device__ uint32_t div(uint32_t n) const { return (uint32_t)(((unsigned long long)n * m) >> 32); }
};

// Merge planning, one CTA per (block, head, tensor): which sources merge
// (top-r), their groups, and the member lists (CSR) the gather kernel reads.
// Members of a destination group: the destination, then its merged sources
// by ascending in-block index; kept sources follow as singletons.  Every
// token of the block is the member of exactly one slot.  Every phase is
// spread evenly over the threads: the top-r threshold by a 4-digit radix
// select (8-bit digits), group sizes by shared-memory counting, each merged
// source's place in its group by counting the group's smaller ordinals (or,
// when a group exceeds 64 members, by ranks taken in source order), and
// the member list written position by position (a binary search over the
// group starts finds each position's group).
__global__ void __launch_bounds__(kMergeThreads)
plan_kernel(Dims dims, const BlockDesc* __restrict__ blocks, Buffers buf, Debug dbg, int injected, int cap,
            int tensor0) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* key = reinterpret_cast<uint32_t*>(smem);        // [cap] ordered score bits
  int32_t* bst = reinterpret_cast<int32_t*>(key + cap);      // [cap] destination of each source
  int32_t* mem = bst + cap;                                  // [cap] merged by group, then kept
  int32_t* aux = mem + cap;                                  // [cap] merged, unordered within a group
  int32_t* cm = aux + cap;                                   // [max_ndst] merged sources per destination
  int32_t* gsm = cm + dims.max_ndst;                         // [max_ndst] exclusive scan of cm
  int32_t* cur = gsm + dims.max_ndst;                        // [max_ndst] placement cursors
  uint32_t* rh = reinterpret_cast<uint32_t*>(cur + dims.max_ndst);  // [256] radix select
  uint32_t* tmp = rh + 256;                                  // [64]
  uint8_t* mf = reinterpret_cast<uint8_t*>(tmp + 64);        // [cap] merged flag
  __shared__ int s_bad;
  __shared__ int s_bin;
  __shared__ uint32_t s_krem;

  const bool is_q = blockIdx.z + tensor0 == 0;         // z-th tensor from tensor0 (0 = Q, 1 = K)
  const int tid = threadIdx.x, bd = blockDim.x;
  const int hh = blockIdx.y;
  const BlockDesc b = blocks[blockIdx.x];
  const int stride = is_q ? dims.q_stride : dims.kv_stride;
  const int ndst = is_q ? b.q_ndst : b.k_ndst;
  const int r = is_q ? b.q_r : b.k_r;
  const int nsrc = b.n_b - ndst;
  const size_t sbase = (size_t)hh * (is_q ? dims.q_src : dims.k_src) + (is_q ? b.q_src_off : b.k_src_off);
  const int32_t* best = (is_q ? buf.q_best : buf.k_best) + sbase;
  const float* score = (is_q ? buf.q_score : buf.k_score) + sbase;
  uint8_t* merged = (is_q ? buf.q_merged : buf.k_merged) + sbase;
  const int slot_off = is_q ? b.q_slot_off : b.k_slot_off;
  const int nslots = is_q ? dims.q_slots : dims.k_slots;
  const size_t tokbase = (size_t)hh * dims.N;
  int32_t* members = (is_q ? buf.q_members : buf.k_members) + tokbase;
  int32_t* gstart = (is_q ? buf.q_gstart : buf.k_gstart) + (size_t)hh * nslots;
  int32_t* gcount = (is_q ? buf.q_gcount : buf.k_gcount) + (size_t)hh * nslots;
  // thread-contiguous source ranges for the order-dependent scans
  const int per = (nsrc + bd - 1) / bd;
  const int lo = min(nsrc, tid * per), hi = min(nsrc, lo + per);

  if (cta_plan_failed(buf.state)) return;
  if (tid == 0) s_bad = 0;
  for (int m = tid; m < ndst; m += bd) cm[m] = 0;
  for (int k = tid; k < nsrc; k += bd) {
    bst[k] = best[k];
    if (!injected) key[k] = float_order(score[k]);
  }
  __syncthreads();

  // HTTM_PARTITION: the block's lists give the in-block index of
  // destination a (bl[a]) and of source ordinal k (bl[ndst + k])
  const int32_t* bl = dims.plists ? dims.plists + b.tok_off : nullptr;

  // 1. top-r: the r sources with the largest (score, -ordinal) merge.  The
  //    r-th largest ordered score T comes from the radix select; all keys
  //    above T merge, and of the keys equal to T the lowest ordinals.
  //    HTTM_PARTITION: every source-class token merges (r of them when the
  //    block has destinations, else none); GA tokens stay single.
  if (bl && !injected) {
    uint32_t cnt = 0;
    for (int k = lo; k < hi; ++k) {
      const bool m = r > 0 && dims.proles[block_token(b, bl[ndst + k], dims.P)] == kRoleSrc;
      mf[k] = m ? 1 : 0;
      merged[k] = m ? 1 : 0;
      cnt += m;
    }
    uint32_t tot;
    block_excl_scan(cnt, tmp, &tot);
    if (tid == 0 && tot != (uint32_t)r) s_bad = 1;
  } else if (!injected) {
    uint32_t T = 0, need = 0;
    if (r > 0) {
      uint32_t prefix = 0, krem = (uint32_t)r;
#pragma unroll 1
      for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        rh[tid] = 0;                                     // blockDim.x == 256 bins
        __syncthreads();
        for (int k = tid; k < nsrc; k += bd) {
          const uint32_t kk = key[k];
          if (pass == 0 || (kk >> (shift + 8)) == prefix) atomicAdd(&rh[(kk >> shift) & 255u], 1u);
        }
        __syncthreads();
        block_select_bin(rh, 256, krem, tmp, &s_bin, &s_krem);
        prefix = (prefix << 8) | (uint32_t)s_bin;
        krem = s_krem;
      }
      T = prefix;
      need = krem;
    }
    uint32_t neq = 0;
    for (int k = lo; k < hi; ++k) neq += r > 0 && key[k] == T;
    uint32_t tot;
    uint32_t eq_before = block_excl_scan(neq, tmp, &tot);
    for (int k = lo; k < hi; ++k) {
      bool m = false;
      if (r > 0) {
        const uint32_t kk = key[k];
        m = kk > T || (kk == T && eq_before < need);
        eq_before += kk == T;
      }
      mf[k] = m ? 1 : 0;
      merged[k] = m ? 1 : 0;
    }
  } else {
    uint32_t c = 0;
    for (int k = tid; k < nsrc; k += bd) {
      mf[k] = merged[k] != 0;
      c += mf[k];
    }
    uint32_t tot;
    block_excl_scan(c, tmp, &tot);
    if (tid == 0 && tot != (uint32_t)r) s_bad = 1;
  }
  __syncthreads();

  // 2. groups: merged sources per destination (counting), then placement
  //    (in any order: atomics), then each merged source's place in its group
  //    from the number of the group's smaller ordinals.
  for (int k = tid; k < nsrc; k += bd) {
    if (mf[k]) {
      const int m = bst[k];
      if (m < 0 || m >= ndst) s_bad = 1;
      else atomicAdd(&cm[m], 1);
    }
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) set_status(buf.state, HTTM_DEV_BAD_PLAN);
    return;
  }
  block_scan_array(cm, gsm, ndst, tmp);
  // the largest group decides how merged sources find their place: by
  // counting the group's smaller ordinals (cheap for the usual few members),
  // or, past 64 members (near-identical tokens put most of a block in one
  // group), in source order, warp after warp, ranked within a warp by
  // __match_any_sync -- the same ascending order without the c^2 cost
  int cmax_local = 0;
  for (int m = tid; m < ndst; m += bd) cmax_local = max(cmax_local, cm[m]);
  cmax_local = __reduce_max_sync(0xffffffffu, cmax_local);
  if ((tid & 31) == 0) tmp[tid >> 5] = (uint32_t)cmax_local;
  __syncthreads();
  int cmax_all = 0;
  for (int w = 0; w < (bd >> 5); ++w) cmax_all = max(cmax_all, (int)tmp[w]);
  const bool big_groups = cmax_all > 64;
  for (int m = tid; m < ndst; m += bd) cur[m] = gsm[m];
  __syncthreads();
  if (big_groups) {
    const unsigned lt = (1u << (tid & 31)) - 1u;
    for (int c0 = 0; c0 < nsrc; c0 += bd) {
      const int k = c0 + tid;
      const int m = (k < nsrc && mf[k]) ? bst[k] : -1;
      const unsigned same = __match_any_sync(0xffffffffu, m);
      const int rank = __popc(same & lt), cnt = __popc(same);
      for (int w = 0; w < (bd >> 5); ++w) {
        if ((tid >> 5) == w) {
          const int base = m >= 0 ? cur[m] : 0;
          __syncwarp();
          if (m >= 0) {
            mem[base + rank] = k;
            if (rank == 0) cur[m] = base + cnt;
          }
        }
        __syncthreads();
      }
    }
  } else {
    for (int k = tid; k < nsrc; k += bd)
      if (mf[k]) aux[atomicAdd(&cur[bst[k]], 1)] = k;
  }
  {
    // kept sources in ascending ordinal after the r merged ones
    uint32_t nm = 0;
    for (int k = lo; k < hi; ++k) nm += mf[k];
    uint32_t tot;
    uint32_t before = block_excl_scan(nm, tmp, &tot);
    for (int k = lo; k < hi; ++k) {
      if (mf[k]) ++before;
      else mem[r + (k - (int)before)] = k;
    }
  }
  __syncthreads();
  if (!big_groups) {
    for (int p = tid; p < r; p += bd) {
      const int v = aux[p];
      const int m = bst[v], s0 = gsm[m], c = cm[m];
      int rank = 0;
      for (int j = 0; j < c; ++j) rank += aux[s0 + j] < v;
      mem[s0 + rank] = v;
    }
  }
  __syncthreads();

  // 3. member lists (tokens), slot starts and counts, the query slot map.
  //    Group m holds positions [gsm[m] + m, gsm[m + 1] + m + 1); pm maps
  //    each of those positions to m (key and bst are free by now and hold
  //    2 * cap >= n_b entries).
  int32_t* pm = reinterpret_cast<int32_t*>(key);
  for (int m = tid; m < ndst; m += bd) {
    const int p0 = gsm[m] + m, c = cm[m] + 1;
    gstart[slot_off + m] = b.tok_off + p0;
    gcount[slot_off + m] = c;
    for (int j = 0; j < c; ++j) pm[p0 + j] = m;
    if (c > kBigSlot) {                              // a big slot: listed for the CTA-wide kernels
      const uint32_t k = atomicAdd(is_q ? &buf.state->n_big : &buf.state->n_kbig, 1u);
      if (k < big_list_cap(dims.h, dims.N)) (is_q ? buf.q_big : buf.k_big)[k] = hh * nslots + slot_off + m;
    }
  }
  for (int p = tid; p < nsrc - r; p += bd) {
    gstart[slot_off + ndst + p] = b.tok_off + ndst + r + p;
    gcount[slot_off + ndst + p] = 1;
  }
  __syncthreads();
  const SmallDiv by_s(b.s), by_gap(stride - 1);
  for (int q = tid; q < b.n_b; q += bd) {
    int idx, slot;
    if (q < ndst + r) {
      const int a = pm[q], j = q - (gsm[a] + a);
      if (j == 0) {
        idx = bl ? bl[a] : a * stride;
      } else {
        const int k = mem[gsm[a] + j - 1], g = (int)by_gap.div(k);
        idx = bl ? bl[ndst + k] : g * stride + (k - g * (stride - 1)) + 1;   // in-block index of source ordinal k
      }
      slot = slot_off + a;
    } else {
      const int p = q - ndst - r, k = mem[r + p], g = (int)by_gap.div(k);
      idx = bl ? bl[ndst + k] : g * stride + (k - g * (stride - 1)) + 1;
      slot = slot_off + ndst + p;
    }
    const int tau = (int)by_s.div(idx);
    const int tok = b.base + tau * dims.P + (idx - tau * b.s);
    members[b.tok_off + q] = tok;
    if (is_q) buf.q_slot[tokbase + tok] = slot;
    else if (dbg.k_slot) dbg.k_slot[tokbase + tok] = slot;
  }
}

// Slots with more than kBigSlot members -- a destination that drew most of
// its block, as near-identical tokens make it -- are not left to one row
// group, whose member loop would take c / kU dependent steps: the row-group
// kernels list them, and a kernel launched after them gives each listed slot
// a whole CTA.  Row group g of the CTA's RG adds the members g, g + RG,
// g + 2 RG, ... in that order, and the partial rows are then added in
// row-group order, element by element: a fixed order, so the result is
// reproducible (and the same wherever a slot is summed this way).

template <class T, int D>
struct SlotCta {
  using Ch = Chunk<T, D>;
  static constexpr int RG = (256 / 32) * Ch::RPI;   // row groups of a 256-thread CTA
};

// sum[t * D + e] = sum over the members q < c of mem with use(q, tok) of row
// tok of tensor t (NT tensors), by all 256 threads of the CTA.  part holds
// NT * RG * D floats and sum NT * D (shared memory); the sums are visible to
// every thread on return.
template <class T, int D, int NT, class Use>
__device__ void cta_slot_sum(const T* const (&X)[NT], const int32_t* mem, int c, Use use, float* part, float* sum) {
  using Ch = Chunk<T, D>;
  constexpr int CPR = Ch::CPR, EPC = Ch::EPC, RG = SlotCta<T, D>::RG, kU = 4;
  const int lane = threadIdx.x & 31;
  const int g = (int)(threadIdx.x >> 5) * Ch::RPI + lane / CPR, ch = lane % CPR;
  float acc[NT][EPC];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[t][e] = 0.f;
  for (int q0 = g; q0 < c; q0 += kU * RG) {
    uint4 x[NT][kU];
    bool on[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int q = q0 + u * RG;
      on[u] = false;
      if (q < c) {
        const int tok = mem[q];
        on[u] = use(q, tok);
        if (on[u])
#pragma unroll
          for (int t = 0; t < NT; ++t) x[t][u] = Ch::load(X[t] + (size_t)tok * D, ch);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (on[u])
#pragma unroll
        for (int t = 0; t < NT; ++t) Ch::add(acc[t], x[t][u]);
  }
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int e = 0; e < EPC; ++e) part[(t * RG + g) * D + ch * EPC + e] = acc[t][e];
  __syncthreads();
  for (int i = threadIdx.x; i < NT * D; i += blockDim.x) {
    const int t = i / D, e = i - t * D;
    float v = 0.f;
    for (int r = 0; r < RG; ++r) v += part[(t * RG + r) * D + e];
    sum[i] = v;
  }
  __syncthreads();
}

// Mean merging (key design 1), flat over every (head, slot).  Rows are read
// as 16-byte chunks, lane l owning chunk l % CPR; each of the RPI row groups
// of a warp (CPR lanes) takes its own slot, fetches up to kU member rows
// before summing them in member order, and meanwhile already fetches the
// (start, count) and first member indices of its next slot, so the CSR
// lookups overlap the row loads.  Queries also get each member's deviation
// from the mean (key design 3), kept as a 32-bit key (bits(dev) + 1 for
// members of groups of >= 2, else 0), and the first radix digit of those
// keys is histogrammed for the global outlier select.  A slot of more than
// kBigSlot members (the planning lists them in Buffers::q_big / k_big) is
// left to big_gather_kernel.
template <class T, int D, bool IS_Q>
__global__ void __launch_bounds__(256, 4)
gather_kernel(Dims dims, const T* __restrict__ X, const T* __restrict__ V, Buffers buf, Debug dbg, int reuse) {
  using Ch = Chunk<T, D>;
  constexpr int CPR = Ch::CPR, RPI = Ch::RPI, EPC = Ch::EPC, kU = 4;
  __shared__ uint32_t hist[IS_Q ? kHistBins : 1];
  __shared__ uint32_t s_elig;
  // member lists from an earlier call must carry this plan's stamp
  if (reuse && threadIdx.x == 0 && *(volatile uint32_t*)&buf.state->plan_stamp != dims.plan_id)
    set_status(buf.state, HTTM_DEV_BAD_PLAN);
  if (cta_plan_failed(buf.state)) return;
  if (!reuse && IS_Q && blockIdx.x == 0 && threadIdx.x == 0) buf.state->plan_stamp = dims.plan_id;
  const int tid = threadIdx.x, lane = tid & 31;
  const int rg = lane / CPR, ch = lane % CPR;
  if (IS_Q) {
    for (int i = tid; i < kHistBins; i += blockDim.x) hist[i] = 0;
    if (tid == 0) s_elig = 0;
    __syncthreads();
  }
  // (head, slot) pairs are numbered gsl = head * nslots + slot; the plan
  // limits h * N to 2^31 - 1, so 32-bit indices suffice
  const int nslots = IS_Q ? dims.q_slots : dims.k_slots;
  const int total = dims.h * nslots;
  const int32_t* members = IS_Q ? buf.q_members : buf.k_members;
  const int32_t* gstart = IS_Q ? buf.q_gstart : buf.k_gstart;
  const int32_t* gcount = IS_Q ? buf.q_gcount : buf.k_gcount;
  T* Xt = reinterpret_cast<T*>(IS_Q ? buf.q_tilde : buf.k_tilde);
  T* Vt = reinterpret_cast<T*>(buf.v_tilde);
  float* dmean = IS_Q ? dbg.q_means : dbg.k_means;
  uint32_t elig = 0;
  const int step = gridDim.x * (blockDim.x >> 5) * RPI;
  int g0 = (blockIdx.x * (blockDim.x >> 5) + (tid >> 5)) * RPI;
  // the slot this row group handles next: count, start, first member tokens
  auto fetch = [&](int gsl, int& c, int& gs, int (&tk)[kU]) {
    c = 0;
    gs = 0;
    if (gsl < total) {
      c = gcount[gsl];
      gs = gstart[gsl];
      if (c > kBigSlot) c = 0;                     // big_gather_kernel's (the planning listed it)
      const size_t tb = (size_t)(gsl / nslots) * dims.N;
#pragma unroll
      for (int u = 0; u < kU; ++u) tk[u] = u < c ? members[tb + gs + u] : 0;
    }
  };
  int c, gs, tk[kU];
  fetch(g0 + rg, c, gs, tk);
  for (; g0 < total; g0 += step) {
    const int gsl = g0 + rg;
    const int hh = gsl < total ? (int)(gsl / nslots) : 0;
    const size_t tokbase = (size_t)hh * dims.N;
    const T* Xh = X + tokbase * D;
    const T* Vh = IS_Q ? nullptr : V + tokbase * D;
    const int cmax = __reduce_max_sync(0xffffffffu, c);
    float acc[EPC], accv[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] = accv[e] = 0.f;
    uint4 xk[kU];
    int tk0[kU];
    // first batch: member indices are already here
    {
      uint4 x[kU], xv[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        tk0[u] = tk[u];
        if (u < c) {
          x[u] = Ch::load(Xh + (size_t)tk[u] * D, ch);
          if (!IS_Q) xv[u] = Ch::load(Vh + (size_t)tk[u] * D, ch);
        }
      }
      const int c_cur = c, gs_cur = gs;
      fetch(g0 + step + rg, c, gs, tk);         // next slot, while these rows arrive
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        if (u < c_cur) {
          Ch::add(acc, x[u]);
          if (!IS_Q) Ch::add(accv, xv[u]);
        }
        xk[u] = x[u];
      }
      // members beyond the first batch (large groups)
      for (int q0 = kU; q0 < cmax; q0 += kU) {
        int tq[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          tq[u] = q0 + u < c_cur ? members[tokbase + gs_cur + q0 + u] : 0;
          if (q0 + u < c_cur) {
            x[u] = Ch::load(Xh + (size_t)tq[u] * D, ch);
            if (!IS_Q) xv[u] = Ch::load(Vh + (size_t)tq[u] * D, ch);
          }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          if (q0 + u < c_cur) {
            Ch::add(acc, x[u]);
            if (!IS_Q) Ch::add(accv, xv[u]);
          }
        }
      }
      const bool live = gsl < total && c_cur > 0;
      if (live) {
        const float inv = 1.f / (float)c_cur;
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
          acc[e] *= inv;
          accv[e] *= inv;
        }
        const size_t row = (size_t)gsl;       // = head * nslots + slot
        Ch::store(Xt + row * D, ch, acc);
        if (dmean) Ch::store_f32(dmean + row * D, ch, acc);
        if (!IS_Q) {
          Ch::store(Vt + row * D, ch, accv);
          if (dbg.v_means) Ch::store_f32(dbg.v_means + row * D, ch, accv);
        }
      }
      if (IS_Q) {
        for (int q0 = 0; q0 < cmax; q0 += kU) {
          if constexpr (CPR == 8 && kU == 4) {
            // four members at once: each lane's partial sums of squares,
            // then a reduce-scatter over the row's 8 lanes (xor 4, 2, 1)
            // that leaves member m's sum in lanes 2m' (m = 2 bit2 + bit1 of
            // the lane), whose even lanes then write the four keys together
            int tok[kU];
            float s4[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
              const int q = q0 + u;
              const bool mine = q < c_cur;
              tok[u] = q0 == 0 ? tk0[u] : (mine ? members[tokbase + gs_cur + q] : 0);
              uint4 xr = xk[u];
              if (q0 > 0 && mine) xr = Ch::load(Xh + (size_t)tok[u] * D, ch);
              s4[u] = mine && c_cur >= 2 ? Ch::sq_dist(xr, acc) : 0.f;
            }
            const bool b2 = (ch & 4) != 0, b1 = (ch & 2) != 0;
            float k0 = b2 ? s4[2] : s4[0], k1 = b2 ? s4[3] : s4[1];
            k0 += __shfl_xor_sync(0xffffffffu, b2 ? s4[0] : s4[2], 4);
            k1 += __shfl_xor_sync(0xffffffffu, b2 ? s4[1] : s4[3], 4);
            float ss = b1 ? k1 : k0;
            ss += __shfl_xor_sync(0xffffffffu, b1 ? k0 : k1, 2);
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            const int m = (b2 ? 2 : 0) + (b1 ? 1 : 0);
            if ((ch & 1) == 0 && q0 + m < c_cur) {
              const int tm = m == 0 ? tok[0] : m == 1 ? tok[1] : m == 2 ? tok[2] : tok[3];
              const uint32_t key = c_cur >= 2 ? __float_as_uint(sqrtf(ss)) + 1u : 0u;
              buf.keys[tokbase + tm] = key;
              if (key) {
                atomicAdd(&hist[key >> 21], 1u);
                ++elig;
              }
            }
          } else {
#pragma unroll
            for (int u = 0; u < kU; ++u) {
              const int q = q0 + u;
              const bool mine = q < c_cur;
              const int tok = q0 == 0 ? tk0[u] : (mine ? members[tokbase + gs_cur + q] : 0);
              uint4 xr = xk[u];
              if (q0 > 0 && mine) xr = Ch::load(Xh + (size_t)tok * D, ch);
              const float ss = Ch::within_row(mine && c_cur >= 2 ? Ch::sq_dist(xr, acc) : 0.f);
              if (mine && ch == 0) {
                const uint32_t key = c_cur >= 2 ? __float_as_uint(sqrtf(ss)) + 1u : 0u;
                buf.keys[tokbase + tok] = key;
                if (key) {
                  atomicAdd(&hist[key >> 21], 1u);
                  ++elig;
                }
              }
            }
          }
        }
      }
    }
  }
  if (IS_Q) {
    if (elig) atomicAdd(&s_elig, elig);
    __syncthreads();
    for (int i = tid; i < kHistBins; i += blockDim.x)
      if (hist[i]) atomicAdd(&buf.hist[i], hist[i]);
    if (tid == 0 && s_elig) atomicAdd(&buf.state->n_eligible, s_elig);
  }
}

// The slots the gather listed as big (more than kBigSlot members), one at a
// time per CTA: the mean by cta_slot_sum and, for queries, every member's
// deviation key and its first radix digit, as in gather_kernel.
template <class T, int D, bool IS_Q>
__global__ void __launch_bounds__(256)
big_gather_kernel(Dims dims, const T* __restrict__ X, const T* __restrict__ V, Buffers buf, Debug dbg) {
  using Ch = Chunk<T, D>;
  constexpr int CPR = Ch::CPR, RPI = Ch::RPI, EPC = Ch::EPC, NT = IS_Q ? 1 : 2, RG = SlotCta<T, D>::RG, kU = 4;
  const uint32_t listed = *(volatile const uint32_t*)(IS_Q ? &buf.state->n_big : &buf.state->n_kbig);
  const int nbig = (int)min(listed, (uint32_t)big_list_cap(dims.h, dims.N));
  if ((int)blockIdx.x >= nbig) return;
  if (cta_plan_failed(buf.state)) return;
  __shared__ uint32_t hist[IS_Q ? kHistBins : 1];
  __shared__ uint32_t s_elig;
  __shared__ float s_part[NT * RG * D], s_sum[NT * D];
  const int tid = threadIdx.x, lane = tid & 31;
  const int ch = lane % CPR, g = (tid >> 5) * RPI + lane / CPR;
  if (IS_Q) {
    for (int i = tid; i < kHistBins; i += blockDim.x) hist[i] = 0;
    if (tid == 0) s_elig = 0;
    __syncthreads();
  }
  const int nslots = IS_Q ? dims.q_slots : dims.k_slots;
  const int total = dims.h * nslots;
  const int32_t* list = IS_Q ? buf.q_big : buf.k_big;
  const int32_t* members = IS_Q ? buf.q_members : buf.k_members;
  const int32_t* gstart = IS_Q ? buf.q_gstart : buf.k_gstart;
  const int32_t* gcount = IS_Q ? buf.q_gcount : buf.k_gcount;
  T* Xt = reinterpret_cast<T*>(IS_Q ? buf.q_tilde : buf.k_tilde);
  T* Vt = reinterpret_cast<T*>(buf.v_tilde);
  float* dmean = IS_Q ? dbg.q_means : dbg.k_means;
  uint32_t elig = 0;
  for (int i = blockIdx.x; i < nbig; i += gridDim.x) {
    const int gsl = list[i];
    if (gsl < 0 || gsl >= total) {
      if (tid == 0) set_status(buf.state, HTTM_DEV_BOUNDS);
      continue;
    }
    const size_t tokbase = (size_t)(gsl / nslots) * dims.N;
    const int c = gcount[gsl];
    const int32_t* mem = members + tokbase + gstart[gsl];
    if constexpr (IS_Q) {
      const T* const src[1] = {X + tokbase * D};
      cta_slot_sum<T, D, 1>(src, mem, c, [](int, int) { return true; }, s_part, s_sum);
    } else {
      const T* const src[2] = {X + tokbase * D, V + tokbase * D};
      cta_slot_sum<T, D, 2>(src, mem, c, [](int, int) { return true; }, s_part, s_sum);
    }
    const float inv = 1.f / (float)c;
    float mean[EPC], meanv[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) {
      mean[e] = s_sum[ch * EPC + e] * inv;
      meanv[e] = s_sum[(NT - 1) * D + ch * EPC + e] * inv;
    }
    if (g == 0) {
      Ch::store(Xt + (size_t)gsl * D, ch, mean);
      if (dmean) Ch::store_f32(dmean + (size_t)gsl * D, ch, mean);
      if (!IS_Q) {
        Ch::store(Vt + (size_t)gsl * D, ch, meanv);
        if (dbg.v_means) Ch::store_f32(dbg.v_means + (size_t)gsl * D, ch, meanv);
      }
    }
    if (IS_Q) {
      // every member's deviation from the mean (c > kBigSlot >= 2: all eligible)
      const T* Xh = X + tokbase * D;
      for (int q0 = 0; q0 < c; q0 += kU * RG) {
        uint4 x[kU];
        int tok[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int q = q0 + u * RG + g;
          tok[u] = q < c ? mem[q] : -1;
          if (tok[u] >= 0) x[u] = Ch::load(Xh + (size_t)tok[u] * D, ch);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const float ss = Ch::within_row(tok[u] >= 0 ? Ch::sq_dist(x[u], mean) : 0.f);
          if (tok[u] >= 0 && ch == 0) {
            const uint32_t key = __float_as_uint(sqrtf(ss)) + 1u;
            buf.keys[tokbase + tok[u]] = key;
            atomicAdd(&hist[key >> 21], 1u);
            ++elig;
          }
        }
      }
    }
    __syncthreads();                                   // s_sum is the next slot's
  }
  if (IS_Q) {
    if (elig) atomicAdd(&s_elig, elig);
    __syncthreads();
    for (int i = tid; i < kHistBins; i += blockDim.x)
      if (hist[i]) atomicAdd(&buf.hist[i], hist[i]);
    if (tid == 0 && s_elig) atomicAdd(&buf.state->n_eligible, s_elig);
  }
}

// Restore (key design 3), flat over every (head, query slot): a slot holding
// outliers becomes the mean of its remaining members (in member order); a
// slot whose members are all outliers is drained (zeros; no token reads it).
template <class T, int D>
__global__ void __launch_bounds__(256)
restore_kernel(Dims dims, const T* __restrict__ Q, Buffers buf, Debug dbg) {
  using Ch = Chunk<T, D>;
  constexpr int CPR = Ch::CPR, RPI = Ch::RPI, EPC = Ch::EPC, kU = 4;
  if (plan_failed(buf.state)) return;
  if (buf.state->sel[3] == 0 && dbg.q_restored == nullptr) return;  // no outlier anywhere
  const int lane = threadIdx.x & 31;
  const int rg = lane / CPR, ch = lane % CPR;
  const int total = dims.h * dims.q_slots;          // h * N < 2^31 (plan limit)
  T* Qt = reinterpret_cast<T*>(buf.q_tilde);
  const int nwarp_total = gridDim.x * (blockDim.x >> 5);
  for (int g0 = (blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * RPI; g0 < total; g0 += nwarp_total * RPI) {
    const int gsl = g0 + rg;
    const bool live = gsl < total;
    const int hh = live ? gsl / dims.q_slots : 0;
    const size_t tokbase = (size_t)hh * dims.N;
    int c = live ? buf.q_gcount[gsl] : 0;
    const int gs = live ? buf.q_gstart[gsl] : 0;
    if (c < 0 || gs < 0 || gs + c > dims.N) {
      if (ch == 0) set_status(buf.state, HTTM_DEV_BOUNDS);
      c = 0;
    }
    if (c > kBigSlot) c = 0;                           // restore_big_kernel takes it
    // outliers among the members (the lanes of the row group share them out)
    int nout = 0;
    if (c >= 2) {
      for (int q = ch; q < c; q += CPR) {
        const int tok = buf.q_members[tokbase + gs + q];
        nout += (tok >= 0 && tok < dims.N) ? (buf.mask[tokbase + tok] != 0) : 0;
      }
    }
#pragma unroll
    for (int o = 1; o < CPR; o <<= 1) nout += __shfl_xor_sync(0xffffffffu, nout, o);
    const bool work = live && (nout > 0 || (dbg.q_restored != nullptr && c >= 1));
    const int cw = work ? c : 0;
    const int cmax = __reduce_max_sync(0xffffffffu, cw);
    if (cmax == 0) continue;
    float acc[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
    for (int q0 = 0; q0 < cmax; q0 += kU) {
      uint4 x[kU];
      bool use[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        use[u] = false;
        if (q0 + u < cw) {
          const int tok = buf.q_members[tokbase + gs + q0 + u];
          use[u] = tok >= 0 && tok < dims.N && buf.mask[tokbase + tok] == 0;
          if (use[u]) x[u] = Ch::load(Q + (tokbase + tok) * D, ch);
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (use[u]) Ch::add(acc, x[u]);
    }
    if (!work) continue;
    const int remain = c - nout;
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] = remain ? acc[e] / (float)remain : 0.f;
    if (nout > 0) Ch::store(Qt + (size_t)gsl * D, ch, acc);
    if (dbg.q_restored) {
      float o[EPC];
#pragma unroll
      for (int e = 0; e < EPC; ++e) o[e] = remain ? acc[e] : __int_as_float(0x7fc00000);
      Ch::store_f32(dbg.q_restored + (size_t)gsl * D, ch, o);
    }
  }
}

// Restore (key design 3) driven by the outliers: one row group per outlier
// row of Q~ (rows [out_base, q_rows_alloc), head after head, with padding
// between heads).  Of the outliers in one slot, the first in member order
// recomputes the slot's mean from the remaining members -- the same members
// in the same order, added the same way as the flat kernel above, so both
// give the same bits; a slot whose members are all outliers is drained.
// Big slots are restore_big_kernel's, after either kernel.
template <class T, int D>
__global__ void __launch_bounds__(256)
restore_out_kernel(Dims dims, const T* __restrict__ Q, Buffers buf) {
  using Ch = Chunk<T, D>;
  constexpr int CPR = Ch::CPR, RPI = Ch::RPI, EPC = Ch::EPC, kU = 4;
  __shared__ int s_base[64], s_nout[64];
  if (plan_failed(buf.state)) return;
  if (buf.state->sel[3] == 0) return;                 // no outlier anywhere
  for (int i = threadIdx.x; i < dims.h; i += blockDim.x) {
    s_base[i] = (int)(buf.out_base[i] - dims.out_base);
    s_nout[i] = buf.n_out[i];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int rg = lane / CPR, ch = lane % CPR;
  const int span = (int)(dims.q_rows_alloc - dims.out_base);
  T* Qt = reinterpret_cast<T*>(buf.q_tilde);
  const int nwarp_total = gridDim.x * (blockDim.x >> 5);
  for (int r0 = (blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * RPI; r0 < span; r0 += nwarp_total * RPI) {
    const int row = r0 + rg;
    int hh = -1;
    if (row < span) {
      for (int x = 0; x < dims.h; ++x)                 // row bases increase with the head
        if (s_base[x] <= row) hh = x;
      if (hh >= 0 && row - s_base[hh] >= s_nout[hh]) hh = -1;   // padding
    }
    int c = 0, gs = 0, gsl = 0, tok = -1;
    size_t tokbase = 0;
    if (hh >= 0) {
      tokbase = (size_t)hh * dims.N;
      tok = buf.o_tok[row];
      const int sl = (tok >= 0 && tok < dims.N) ? buf.q_slot[tokbase + tok] : -1;
      if (sl >= 0 && sl < dims.q_slots) {
        gsl = hh * dims.q_slots + sl;
        c = buf.q_gcount[gsl];
        gs = buf.q_gstart[gsl];
      }
      if (c < 0 || gs < 0 || gs + c > dims.N || sl < 0 || sl >= dims.q_slots) {
        if (ch == 0) set_status(buf.state, HTTM_DEV_BOUNDS);
        c = 0;
      }
      if (c > kBigSlot) c = 0;                         // restore_big_kernel takes it
    }
    // outliers among the members, and the first of them in member order
    int nout = 0, first = 0x7fffffff;
    for (int q = ch; q < c; q += CPR) {
      const int m = buf.q_members[tokbase + gs + q];
      const bool o = (m >= 0 && m < dims.N) && buf.mask[tokbase + m] != 0;
      nout += o;
      if (o && q < first) first = q;
    }
#pragma unroll
    for (int o = 1; o < CPR; o <<= 1) {
      nout += __shfl_xor_sync(0xffffffffu, nout, o);
      first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
    }
    const bool lead = c > 0 && first < c && buf.q_members[tokbase + gs + first] == tok;
    const int cw = lead ? c : 0;
    const int cmax = __reduce_max_sync(0xffffffffu, cw);
    if (cmax == 0) continue;
    float acc[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
    for (int q0 = 0; q0 < cmax; q0 += kU) {
      uint4 x[kU];
      bool use[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        use[u] = false;
        if (q0 + u < cw) {
          const int m = buf.q_members[tokbase + gs + q0 + u];
          use[u] = m >= 0 && m < dims.N && buf.mask[tokbase + m] == 0;
          if (use[u]) x[u] = Ch::load(Q + (tokbase + m) * D, ch);
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (use[u]) Ch::add(acc, x[u]);
    }
    if (!lead) continue;
    const int remain = c - nout;
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] = remain ? acc[e] / (float)remain : 0.f;
    Ch::store(Qt + (size_t)gsl * D, ch, acc);
  }
}

// The big query slots (more than kBigSlot members; the query gather listed
// them), one at a time per CTA: the outliers among the members, then the sum
// of the others as cta_slot_sum adds them, divided by their count -- the
// slot's new row when it holds outliers.  dbg_rows (the fp32 export, or null)
// gets that mean for every big slot (NaN where every member is an outlier).
template <class T, int D>
__global__ void __launch_bounds__(256)
restore_big_kernel(Dims dims, const T* __restrict__ Q, Buffers buf, float* dbg_rows) {
  using Ch = Chunk<T, D>;
  constexpr int CPR = Ch::CPR, EPC = Ch::EPC, RG = SlotCta<T, D>::RG;
  const uint32_t listed = *(volatile const uint32_t*)&buf.state->n_big;
  const int nbig = (int)min(listed, (uint32_t)big_list_cap(dims.h, dims.N));
  if ((int)blockIdx.x >= nbig) return;
  if (cta_plan_failed(buf.state)) return;
  if (buf.state->sel[3] == 0 && dbg_rows == nullptr) return;     // no outlier anywhere
  __shared__ float s_part[RG * D], s_sum[D];
  const int lane = threadIdx.x & 31, ch = lane % CPR;
  const int g = (int)(threadIdx.x >> 5) * Ch::RPI + lane / CPR;
  T* Qt = reinterpret_cast<T*>(buf.q_tilde);
  const int total = dims.h * dims.q_slots;
  for (int i = blockIdx.x; i < nbig; i += gridDim.x) {
    const int gsl = buf.q_big[i];
    int c = 0, gs = 0, hh = 0;
    if (gsl >= 0 && gsl < total) {
      hh = gsl / dims.q_slots;
      c = buf.q_gcount[gsl];
      gs = buf.q_gstart[gsl];
    }
    if (gsl < 0 || gsl >= total || c < 0 || gs < 0 || gs + c > dims.N) {
      if (threadIdx.x == 0) set_status(buf.state, HTTM_DEV_BOUNDS);
      c = 0;
    }
    const size_t tokbase = (size_t)hh * dims.N;
    const int32_t* mem = buf.q_members + tokbase + gs;
    int nout = 0;
    for (int q0 = 0; q0 < c; q0 += blockDim.x) {
      const int q = q0 + threadIdx.x;
      bool o = false;
      if (q < c) {
        const int tok = mem[q];
        o = tok >= 0 && tok < dims.N && buf.mask[tokbase + tok] != 0;
      }
      nout += __syncthreads_count(o);
    }
    if (c == 0 || (nout == 0 && dbg_rows == nullptr)) continue;
    const T* const src[1] = {Q + tokbase * D};
    cta_slot_sum<T, D, 1>(
        src, mem, c,
        [&](int, int tok) { return tok >= 0 && tok < dims.N && buf.mask[tokbase + tok] == 0; }, s_part, s_sum);
    const int remain = c - nout;
    if (g == 0) {
      float acc[EPC];
#pragma unroll
      for (int e = 0; e < EPC; ++e) acc[e] = remain ? s_sum[ch * EPC + e] / (float)remain : 0.f;
      if (nout > 0) Ch::store(Qt + (size_t)gsl * D, ch, acc);
      if (dbg_rows) {
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc[e] = remain ? acc[e] : __int_as_float(0x7fc00000);
        Ch::store_f32(dbg_rows + (size_t)gsl * D, ch, acc);
      }
    }
    __syncthreads();                                   // s_sum is the next slot's
  }
}

// Injected plan -> internal source-order arrays, with validation.
__global__ void import_kernel(Dims dims, const BlockDesc* __restrict__ blocks, Inject inj, Buffers buf) {
  const size_t total = 2ull * dims.h * dims.N;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int tensor = (int)(idx / ((size_t)dims.h * dims.N));
    const size_t rem = idx - (size_t)tensor * dims.h * dims.N;
    const int hh = (int)(rem / dims.N);
    const int n = (int)(rem - (size_t)hh * dims.N);
    if (tensor == 0 && inj.outlier) buf.mask[rem] = inj.outlier[rem] ? 1 : 0;
    if (inj.q_best == nullptr) continue;
    const int stride = tensor == 0 ? dims.q_stride : dims.kv_stride;
    int blk, i;
    token_block(dims, n, blk, i);
    if (i % stride == 0) continue;
    const BlockDesc b = blocks[blk];
    const int k = src_ordinal(i, stride);
    const int32_t* ib = tensor == 0 ? inj.q_best : inj.k_best;
    const uint8_t* im = tensor == 0 ? inj.q_merged : inj.k_merged;
    const int nd = ib[rem];
    int m = 0;
    const bool mg = im[rem] != 0;
    if (mg) {
      bool ok = nd >= 0 && nd < dims.N;
      if (ok) {
        int blk2, i2;
        token_block(dims, nd, blk2, i2);
        ok = blk2 == blk && i2 % stride == 0;
        if (ok) m = i2 / stride;
      }
      if (!ok) set_status(buf.state, HTTM_DEV_BAD_PLAN);
    }
    const size_t si = (size_t)hh * (tensor == 0 ? dims.q_src : dims.k_src) +
                      (tensor == 0 ? b.q_src_off : b.k_src_off) + k;
    (tensor == 0 ? buf.q_best : buf.k_best)[si] = m;
    (tensor == 0 ? buf.q_merged : buf.k_merged)[si] = mg ? 1 : 0;
    (tensor == 0 ? buf.q_score : buf.k_score)[si] = 0.f;
  }
}

// Internal arrays -> the [h, N] original-order debug exports.
__global__ void export_kernel(Dims dims, const BlockDesc* __restrict__ blocks, Buffers buf, Debug dbg) {
  if (plan_failed(buf.state)) return;
  const size_t total = (size_t)dims.h * dims.N;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int hh = (int)(idx / dims.N);
    const int n = (int)(idx - (size_t)hh * dims.N);
    int blk, i;
    token_block(dims, n, blk, i);
    const BlockDesc b = blocks[blk];
#pragma unroll
    for (int tensor = 0; tensor < 2; ++tensor) {
      int32_t* ob = tensor == 0 ? dbg.q_best : dbg.k_best;
      float* os = tensor == 0 ? dbg.q_score : dbg.k_score;
      uint8_t* om = tensor == 0 ? dbg.q_merged : dbg.k_merged;
      if (!ob && !os && !om) continue;
      const int stride = tensor == 0 ? dims.q_stride : dims.kv_stride;
      int bt = -1, mg = 0;
      float sc = 0.f;
      // HTTM_PARTITION: a token's class says whether it is a destination,
      // its ordinal places it in its list; a block without destinations
      // has no match (best -1)
      const bool part = dims.plists != nullptr;
      const bool is_dst = part ? dims.proles[n] == kRoleDst : i % stride == 0;
      const int ndst = tensor == 0 ? b.q_ndst : b.k_ndst;
      if (!is_dst && (!part || ndst > 0)) {
        const size_t si = (size_t)hh * (tensor == 0 ? dims.q_src : dims.k_src) +
                          (tensor == 0 ? b.q_src_off : b.k_src_off) + (part ? dims.pord[n] : src_ordinal(i, stride));
        const int m = (tensor == 0 ? buf.q_best : buf.k_best)[si];
        bt = block_token(b, part ? dims.plists[b.tok_off + m] : m * stride, dims.P);
        sc = (tensor == 0 ? buf.q_score : buf.k_score)[si];
        mg = (tensor == 0 ? buf.q_merged : buf.k_merged)[si];
      }
      if (ob) ob[idx] = bt;
      if (os) os[idx] = sc;
      if (om) om[idx] = (uint8_t)mg;
    }
    if (dbg.q_slot) dbg.q_slot[idx] = buf.mask[idx] ? dims.q_slots + buf.q_orank[idx] : buf.q_slot[idx];
    if (dbg.dev) {
      const uint32_t key = buf.keys[idx];
      dbg.dev[idx] = key ? __uint_as_float(key - 1u) : 0.f;
    }
    if (dbg.outlier) dbg.outlier[idx] = buf.mask[idx];
  }
}

__global__ void zero_state_kernel(Buffers buf, int keep_stamp, unsigned long long wait_ns) {
  for (int i = threadIdx.x; i < 3 * kHistBins + kMaxShards; i += blockDim.x) buf.hist[i] = 0u;
  if (threadIdx.x == 0) {
    if (!keep_stamp) buf.state->plan_stamp = 0u;   // rewritten once this call's planning has succeeded
    buf.state->status = 0u;
    buf.state->n_eligible = 0u;
    buf.state->n_items = 0u;
    buf.state->wait_site = 0u;
    buf.state->wait_cta = 0u;
    buf.state->wait_grid = 0u;
    if (!keep_stamp) {                             // the big-slot lists go with the member lists
      buf.state->n_big = 0u;
      buf.state->n_kbig = 0u;
    }
    buf.state->wait_ns = wait_ns;
  }
  if (threadIdx.x < 8) buf.state->sel[threadIdx.x] = 0u;
}

// CTAs of 8 warps for `units` warp-sized pieces of work, at most `per_sm`
// per SM (the gathers run four per SM at their register bound; each warp
// then takes several slots in turn, so that its prefetches pay).
int gather_grid(long long units, int per_sm = 8) {
  return (int)std::max<long long>(1, std::min<long long>((units + 7) / 8, 148LL * per_sm));
}

template <class T, int D>
cudaError_t launch_merge_t(const Dims& dims, const BlockDesc* blocks, bool injected, bool reuse, const void* Q,
                           const void* K, const void* V, const Buffers& buf, const Debug& dbg, cudaStream_t s,
                           int tensors) {
  const bool do_q = (tensors & 1) != 0, do_k = (tensors & 2) != 0;
  if (!reuse) {
    // cap sources per block, and 2 * cap >= n_b for the position map
    const int cap = (std::max(dims.max_nsrc, (dims.max_nb + 1) / 2) + kMergeThreads - 1) / kMergeThreads * kMergeThreads;
    const size_t smem = (size_t)cap * 17 + 3ull * dims.max_ndst * 4 + 256 * 4 + 64 * 4;
    cudaError_t e = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    plan_kernel<<<dim3(dims.nblk, dims.h, (do_q && do_k) ? 2 : 1), kMergeThreads, smem, s>>>(
        dims, blocks, buf, dbg, injected ? 1 : 0, cap, do_q ? 0 : 1);
  }
  constexpr int RPI = Chunk<T, D>::RPI;
  // resident warps handle several slots each, so that prefetching pays
  // the big slots' kernels: as many CTAs as the lists could need, at most
  // two per SM; CTAs past the listed count return at once
  const int big_grid = (int)std::min<size_t>(2 * 148, big_list_cap(dims.h, dims.N));
  if (do_q) {
    gather_kernel<T, D, true><<<gather_grid((long long)dims.h * dims.q_slots / (4 * RPI) + 1, 4), 256, 0, s>>>(
        dims, (const T*)Q, nullptr, buf, dbg, reuse ? 1 : 0);
    big_gather_kernel<T, D, true><<<big_grid, 256, 0, s>>>(dims, (const T*)Q, nullptr, buf, dbg);
  }
  if (do_k) {
    gather_kernel<T, D, false><<<gather_grid((long long)dims.h * dims.k_slots / (4 * RPI) + 1, 4), 256, 0, s>>>(
        dims, (const T*)K, (const T*)V, buf, dbg, reuse ? 1 : 0);
    big_gather_kernel<T, D, false><<<big_grid, 256, 0, s>>>(dims, (const T*)K, (const T*)V, buf, dbg);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_zero_state(const Dims& dims, const Buffers& buf, bool keep_stamp, cudaStream_t s) {
  zero_state_kernel<<<1, 1024, 0, s>>>(buf, keep_stamp ? 1 : 0, (unsigned long long)dims.wait_budget_ns);
  return cudaGetLastError();
}

cudaError_t launch_merge(const Dims& dims, bool fp32, const BlockDesc* blocks, bool injected, bool reuse,
                         const void* Q, const void* K, const void* V, const Buffers& buf, const Debug& dbg,
                         cudaStream_t s, int tensors) {
  if (fp32) {
    if (dims.d == 16) return launch_merge_t<float, 16>(dims, blocks, injected, reuse, Q, K, V, buf, dbg, s, tensors);
    return launch_merge_t<float, 64>(dims, blocks, injected, reuse, Q, K, V, buf, dbg, s, tensors);
  }
  if (dims.d == 16)
    return launch_merge_t<__nv_bfloat16, 16>(dims, blocks, injected, reuse, Q, K, V, buf, dbg, s, tensors);
  return launch_merge_t<__nv_bfloat16, 64>(dims, blocks, injected, reuse, Q, K, V, buf, dbg, s, tensors);
}

cudaError_t launch_restore(const Dims& dims, bool fp32, const BlockDesc*, const void* Q, const Buffers& buf,
                           const Debug& dbg, cudaStream_t s) {
  // the fp32 export needs every slot's restored mean: the flat kernel;
  // otherwise only the slots holding outliers change
  const bool flat = dbg.q_restored != nullptr;
  const long long units = flat ? (long long)dims.h * dims.q_slots : dims.q_rows_alloc - dims.out_base;
  const int big_grid = (int)std::min<size_t>(2 * 148, big_list_cap(dims.h, dims.N));
#define HTTM_RESTORE(T, DD)                                                                                  \
  do {                                                                                                       \
    const int grid = gather_grid(units / Chunk<T, DD>::RPI + 1);                                             \
    if (flat) restore_kernel<T, DD><<<grid, 256, 0, s>>>(dims, (const T*)Q, buf, dbg);                       \
    else restore_out_kernel<T, DD><<<grid, 256, 0, s>>>(dims, (const T*)Q, buf);                             \
    restore_big_kernel<T, DD><<<big_grid, 256, 0, s>>>(dims, (const T*)Q, buf, flat ? dbg.q_restored : nullptr); \
  } while (0)
  if (fp32) {
    if (dims.d == 16) HTTM_RESTORE(float, 16);
    else HTTM_RESTORE(float, 64);
  } else {
    if (dims.d == 16) HTTM_RESTORE(__nv_bfloat16, 16);
    else HTTM_RESTORE(__nv_bfloat16, 64);
  }
#undef HTTM_RESTORE
  return cudaGetLastError();
}

cudaError_t launch_import_plan(const Dims& dims, const BlockDesc* blocks, const Inject& inj,
                               const Buffers& buf, cudaStream_t s) {
  const size_t total = 2ull * dims.h * dims.N;
  const int grid = (int)std::min<size_t>((total + 255) / 256, 148 * 16);
  import_kernel<<<grid, 256, 0, s>>>(dims, blocks, inj, buf);
  return cudaGetLastError();
}

cudaError_t launch_export(const Dims& dims, const BlockDesc* blocks, const Buffers& buf, const Debug& dbg,
                          cudaStream_t s) {
  const size_t total = (size_t)dims.h * dims.N;
  const int grid = (int)std::min<size_t>((total + 255) / 256, 148 * 16);
  export_kernel<<<grid, 256, 0, s>>>(dims, blocks, buf, dbg);
  return cudaGetLastError();
}

}  // namespace httm

// Row-wise Top-K selection (ADIndex, arXiv 2611.12956v1, §3 Eq. (2), and the bank Top-P
// of Eq. (13)) as an exact radix select.
//
// Each CTA owns one row (or one segment of a row, for the first stage of a split select).
// Scores are mapped to order-preserving 32-bit keys; the K-th largest key is found digit by
// digit (12 + 12 + 8 bits) with shared-memory histograms, and a last pass writes every
// element above the threshold plus the lowest-indexed elements equal to it, in index order,
// using block-wide prefix sums (warp shuffles) for the output slots. -inf marks a masked
// (invisible) key and NaN is treated the same way: neither is ever selected. Rows with fewer
// than K valid elements return all of them, padded with index -1 and score -inf.
#include <cooperative_groups.h>

#include <algorithm>
#include <cfloat>
#include <cstdint>
#include <type_traits>

#include "adx_internal.h"
#include "sm100_ptx.cuh"

namespace adx {

namespace cg = cooperative_groups;

namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kBins = 4096;

__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ bool is_valid(float v) { return !(v != v) && v != -INFINITY; }

// Inclusive prefix sum over the block (all threads participate); also returns the total.
__device__ __forceinline__ uint32_t block_inclusive_scan(uint32_t x, uint32_t* warp_tot,
                                                         uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = lane < kSelWarps ? warp_tot[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < kSelWarps) warp_tot[lane] = t;  // inclusive warp prefix
  }
  __syncthreads();
  const uint32_t before = warp == 0 ? 0u : warp_tot[warp - 1];
  total = warp_tot[kSelWarps - 1];
  __syncthreads();  // warp_tot may be reused right after
  return x + before;
}

// The fp32 value of an order-preserving key (inverse of order_key).
__device__ __forceinline__ float key_value_long(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Position of element id through the row's map (per element, or per block of 2^shift).
__device__ __forceinline__ int32_t map_id(const int32_t* map, int32_t id, int shift) {
  if (map == nullptr || id < 0) return id;
  if (shift == 0) return map[id];
  return (map[id >> shift] << shift) + (id & ((1 << shift) - 1));
}

struct RowInfo {
  int64_t lo, hi;  // element range of this CTA
};

__device__ __forceinline__ int64_t row_length(const SelectArgs& a, int r) {
  int64_t n;
  if (a.len_mode == 0) {
    n = a.len_fixed;
  } else if (a.len_mode == 1) {
    n = a.pos_base + static_cast<int64_t>(r) * a.pos_step + 1;
  } else if (a.len_mode == 2) {
    n = a.seq_len[r / a.rows_per_batch];
  } else {
    n = (static_cast<int64_t>(a.row_pos[r]) + 1 + a.len_off) * (a.len_mul > 1 ? a.len_mul : 1);
  }
  if (n > a.len_cap) n = a.len_cap;
  return n < 0 ? 0 : n;
}

// Multi-pass radix select of one row (or row segment) streamed from global memory: three
// digit passes (12 + 12 + 8 bits) over the row, then an ordered output pass. hist holds kBins
// words, warp_tot 32, sh two; all in shared memory, all threads of the CTA take part.
__device__ void radix_row(const SelectArgs& a, int r, int seg, uint32_t* hist, uint32_t* warp_tot,
                          uint32_t* sh) {
  uint32_t& sh_bin = sh[0];
  uint32_t& sh_above = sh[1];
  const int64_t n = row_length(a, r);
  const int64_t lo = static_cast<int64_t>(seg) * a.seg_len;
  const int64_t hi = a.n_seg == 1 ? n : min(n, lo + a.seg_len);
  const float* vals = a.vals + static_cast<int64_t>(r) * a.ld;
  const int32_t* in_idx = a.in_idx ? a.in_idx + static_cast<int64_t>(r) * a.ld : nullptr;
  const int32_t* map =
      a.idx_map ? a.idx_map + static_cast<int64_t>(r / a.rows_per_batch) * a.map_stride : nullptr;
  const int64_t out_base = (static_cast<int64_t>(r) * a.n_seg + seg) * a.out_ld;
  const int K = a.K;

  // ---- radix passes: find the K-th largest key digit by digit -------------------------
  // After the passes: elements whose top (32 - shift) key bits are > prefix are selected;
  // those equal to prefix are selected while their tie rank is < need.
  uint32_t prefix = 0;
  int shift = 32;            // number of low key bits not yet resolved
  uint32_t need = K;
  bool take_all = false;
  const int widths[3] = {12, 12, 8};
  for (int p = 0; p < 3; ++p) {
    const int wbits = widths[p];
    const int nb = 1 << wbits;
    const int nshift = shift - wbits;
    for (int i = threadIdx.x; i < nb; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int64_t base = lo; base < hi; base += kSelThreads) {
      const int64_t i = base + threadIdx.x;
      const float v = i < hi ? vals[i] : -INFINITY;
      const uint32_t u = order_key(v);
      if (is_valid(v) && (shift >= 32 || (u >> shift) == prefix))
        atomicAdd(&hist[(u >> nshift) & (nb - 1)], 1u);
    }
    __syncthreads();
    // thread t owns the bins nb-1-(t*bpt) .. nb-(t+1)*bpt, i.e. thread 0 the highest ones
    const int bpt = nb >= kSelThreads ? nb / kSelThreads : 1;
    const bool owner = threadIdx.x * bpt < nb;
    uint32_t mine = 0;
    if (owner)
      for (int j = 0; j < bpt; ++j) mine += hist[nb - 1 - (threadIdx.x * bpt + j)];
    uint32_t total;
    const uint32_t incl = block_inclusive_scan(mine, warp_tot, total);
    if (p == 0 && total <= static_cast<uint32_t>(K)) {
      take_all = true;  // every valid element is selected
      break;
    }
    const uint32_t excl = incl - mine;
    if (owner && excl < need && need <= incl) {
      uint32_t above = excl;
      for (int j = 0; j < bpt; ++j) {
        const int bin = nb - 1 - (threadIdx.x * bpt + j);
        const uint32_t h = hist[bin];
        if (above + h >= need) {
          sh_bin = static_cast<uint32_t>(bin);
          sh_above = above;
          break;
        }
        above += h;
      }
    }
    __syncthreads();
    const uint32_t bin = sh_bin;
    need -= sh_above;
    const uint32_t in_bin = hist[bin];
    prefix = (shift < 32 ? (prefix << wbits) : 0u) | bin;
    shift = nshift;
    __syncthreads();
    if (in_bin == need) break;  // the whole bin is taken: no further digits needed
  }

  // ---- output pass, in index order ----------------------------------------------------
  uint32_t eq_carry = 0, sel_carry = 0;
  constexpr int V = 4;
  for (int64_t base = lo; base < hi; base += static_cast<int64_t>(kSelThreads) * V) {
    float v[V];
    uint32_t gt_mask = 0, eq_mask = 0;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int64_t i = base + threadIdx.x * V + j;
      v[j] = i < hi ? vals[i] : -INFINITY;
      if (!is_valid(v[j])) continue;
      if (take_all) {
        gt_mask |= 1u << j;
        continue;
      }
      const uint32_t top = order_key(v[j]) >> shift;
      if (top > prefix) gt_mask |= 1u << j;
      else if (top == prefix) eq_mask |= 1u << j;
    }
    uint32_t eq_tot;
    const uint32_t n_eq = __popc(eq_mask);
    const uint32_t eq_excl = block_inclusive_scan(n_eq, warp_tot, eq_tot) - n_eq + eq_carry;
    uint32_t sel_mask = gt_mask;
    uint32_t rank = eq_excl;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      if (eq_mask & (1u << j)) {
        if (rank < need) sel_mask |= 1u << j;
        ++rank;
      }
    }
    uint32_t sel_tot;
    const uint32_t n_sel = __popc(sel_mask);
    uint32_t slot = block_inclusive_scan(n_sel, warp_tot, sel_tot) - n_sel + sel_carry;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      if (sel_mask & (1u << j)) {
        const int64_t i = base + threadIdx.x * V + j;
        int32_t id = in_idx ? in_idx[i] : static_cast<int32_t>(i);
        id = map_id(map, id, a.map_shift);
        if (slot < static_cast<uint32_t>(K)) {
          a.out_idx[out_base + slot] = id;
          if (a.out_val) a.out_val[out_base + slot] = v[j];
        }
        ++slot;
      }
    }
    eq_carry += eq_tot;
    sel_carry += sel_tot;
  }
  for (int64_t j = sel_carry + threadIdx.x; j < K; j += kSelThreads) {
    a.out_idx[out_base + j] = -1;
    if (a.out_val) a.out_val[out_base + j] = -INFINITY;
  }
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(const SelectArgs a) {
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t sh[2];
  const int seg = blockIdx.x % a.n_seg;
  const int r = blockIdx.x / a.n_seg;
  if (r >= a.rows) return;
  radix_row(a, r, seg, hist, warp_tot, sh);
}

// ---------------------------------------------------------------------------------------
// Register-resident select: each thread holds a contiguous run of ITEMS elements of its
// CTA's part of the row, so global memory is read once; the digit passes work on registers
// and one block-wide scan of (above, equal) counts gives every thread its output slots in
// index order. The CTA size (and digit width) is chosen per row-length class, so short rows
// of a causal prefix do not pay for long ones.
//
// CLUSTER: one thread-block cluster per row, for few long rows. The row is cut into one
// contiguous slice per CTA of the cluster; the valid-key range, the digit histograms and the
// per-CTA output counts are combined through distributed shared memory, so every CTA of the
// cluster takes the same decisions and writes its own share of the output slots. Histograms
// alternate between two buffers: a CTA clears a buffer only after a cluster barrier that every
// other CTA reaches after its last read of that buffer, so one barrier per digit suffices.
// All CTAs of a cluster compute the same row length, key range and bins, so they pass the
// same cluster barriers.
// ---------------------------------------------------------------------------------------
constexpr int kRegItems = 32;      // elements per thread of the row-per-CTA classes
constexpr int kWideItems = 36;     // ... of the 256-thread class for rows just above 8192
constexpr int kClusterItems = 36;  // elements per thread of the cluster class
constexpr int kClusterThreads = 512;
constexpr int kClusterMaxCtas = 8;  // portable cluster size

template <int THREADS>
__device__ __forceinline__ unsigned long long block_exclusive_scan64(unsigned long long x,
                                                                    unsigned long long* warp_tot,
                                                                    unsigned long long& total) {
  constexpr int NW = THREADS / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  unsigned long long before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const unsigned long long v = warp_tot[w];
    if (w < warp) before += v;
    tot += v;
  }
  total = tot;
  __syncthreads();
  return before + incl - x;
}

// Outputs of a row are staged in shared memory (up to this K) and written with coalesced
// stores; per-thread runs of slots would otherwise scatter every store instruction.
constexpr int kStageMaxK = 4096;
// When at most kGatherMax keys remain in the threshold bin they are gathered into shared
// memory and the selection finishes there: by counting (each key's rank among them) up to
// kCountMax keys, by 8-bit digit passes over the gathered keys beyond that.
constexpr int kCountMax = 128;
constexpr int kGatherMax = 2048;

template <int ITEMS>
using ItemMask = typename std::conditional<(ITEMS > 32), unsigned long long, uint32_t>::type;

__device__ __forceinline__ int lowest_set_bit(uint32_t m) { return __ffs(m) - 1; }
__device__ __forceinline__ int lowest_set_bit(unsigned long long m) { return __ffsll(m) - 1; }

template <int THREADS, int DIGIT, int ITEMS, bool CLUSTER>
__global__ void __launch_bounds__(THREADS, 1024 / THREADS)
select_reg_kernel(const SelectArgs a, int row0) {
  constexpr int NW = THREADS / 32;
  constexpr int NB = 1 << DIGIT;
  constexpr int NH = CLUSTER ? 2 : 1;  // histogram buffers
  using Mask = ItemMask<ITEMS>;
  extern __shared__ __align__(16) uint8_t stage_smem[];
  __shared__ __align__(16) uint32_t hist[NH][NB];
  __shared__ unsigned long long warp_tot64[NW];
  __shared__ uint32_t red_min[NW], red_max[NW], red_cnt[NW];
  __shared__ uint32_t sh_bin, sh_above, sh_inbin;
  __shared__ uint32_t cl_red[3];         // this CTA's (min, max, count) of valid keys
  __shared__ unsigned long long cl_tots[kClusterMaxCtas];  // CTA c's packed (above, equal) counts
  __shared__ uint32_t cl_part[NH][CLUSTER ? THREADS : 1];  // per-thread bin-range counts
  __shared__ uint32_t sh_ccount, sh_theta, sh_needt;
  __shared__ uint32_t c_key[kGatherMax];               // this CTA's keys of the threshold bin
  __shared__ uint32_t c_off[kClusterMaxCtas + 1];       // where each CTA's keys go in c_all
  __shared__ uint32_t h_small[256];                     // digit histogram of gathered keys

  int r, seg = 0, nparts = 1, part = 0;
  if constexpr (CLUSTER) {
    nparts = static_cast<int>(cg::this_cluster().num_blocks());
    part = static_cast<int>(cg::this_cluster().block_rank());
    r = row0 + static_cast<int>(blockIdx.x) / nparts;  // cluster c covers CTAs c*nparts ..
  } else {
    seg = blockIdx.x % a.n_seg;
    r = row0 + static_cast<int>(blockIdx.x / a.n_seg);
  }
  if (r >= a.rows) return;  // the same for every CTA of a cluster
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) sh_ccount = 0;
  const int64_t n = row_length(a, r);
  int64_t lo, hi;
  if (CLUSTER) {
    const int64_t per = ((n + nparts - 1) / nparts + 3) & ~static_cast<int64_t>(3);
    lo = min(n, static_cast<int64_t>(part) * per);
    hi = min(n, lo + per);
  } else {
    lo = static_cast<int64_t>(seg) * a.seg_len;
    hi = a.n_seg == 1 ? n : min(n, lo + a.seg_len);
  }
  const int64_t len = hi > lo ? hi - lo : 0;
  const float* vals = a.vals + static_cast<int64_t>(r) * a.ld + lo;
  const int32_t* in_idx = a.in_idx ? a.in_idx + static_cast<int64_t>(r) * a.ld + lo : nullptr;
  const int32_t* map =
      a.idx_map ? a.idx_map + static_cast<int64_t>(r / a.rows_per_batch) * a.map_stride : nullptr;
  const int64_t out_base = (static_cast<int64_t>(r) * a.n_seg + seg) * a.out_ld;
  const int K = a.K;

  // ---- load: thread t owns elements [t*ITEMS, (t+1)*ITEMS) of this CTA's range -------------
  uint32_t key[ITEMS];
  const int64_t my0 = static_cast<int64_t>(threadIdx.x) * ITEMS;
  const bool vec = ((reinterpret_cast<uintptr_t>(vals) & 15) == 0);
  uint32_t kmin = 0xffffffffu, kmax = 0u, nval = 0u;
#pragma unroll
  for (int j = 0; j < ITEMS; j += 4) {
    float v[4];
    const int64_t i0 = my0 + j;
    if (vec && i0 + 4 <= len) {
      const float4 f = *reinterpret_cast<const float4*>(vals + i0);
      v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = (i0 + u < len) ? vals[i0 + u] : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      // order key; the valid ones (-FLT_MAX .. +inf) are 0x00800000 .. 0xff800000, NaN and
      // -inf fall outside and become 0
      const uint32_t b = __float_as_uint(v[u]);
      const uint32_t kk = b ^ (static_cast<uint32_t>(static_cast<int32_t>(b) >> 31) | 0x80000000u);
      const bool ok = kk - 0x00800000u <= 0xff000000u;
      const uint32_t k = ok ? kk : 0u;
      key[j + u] = k;
      kmin = min(kmin, k - 1u);  // invalid (0) wraps to the largest value: no effect
      kmax = max(kmax, k);
      nval += ok;
    }
  }
  // common high bits of the valid keys: the first digit starts right below them
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  nval = __reduce_add_sync(0xffffffffu, nval);
  if (lane == 0) {
    red_min[warp] = kmin;
    red_max[warp] = kmax;
    red_cnt[warp] = nval;
  }
  __syncthreads();
  kmin = 0xffffffffu;
  kmax = 0u;
  nval = 0u;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    kmin = min(kmin, red_min[w]);
    kmax = max(kmax, red_max[w]);
    nval += red_cnt[w];
  }
  if constexpr (CLUSTER) {
    if (threadIdx.x == 0) {
      cl_red[0] = kmin;
      cl_red[1] = kmax;
      cl_red[2] = nval;
    }
    cg::this_cluster().sync();  // also a CTA barrier: red_* are free again
    if (warp == 0) {  // lane c reads CTA c's values
      uint32_t mn = 0xffffffffu, mx = 0u, nv = 0u;
      if (lane < nparts) {
        const uint32_t* rc = cg::this_cluster().map_shared_rank(cl_red, lane);
        mn = rc[0];
        mx = rc[1];
        nv = rc[2];
      }
      mn = __reduce_min_sync(0xffffffffu, mn);
      mx = __reduce_max_sync(0xffffffffu, mx);
      nv = __reduce_add_sync(0xffffffffu, nv);
      if (lane == 0) {
        red_min[0] = mn;
        red_max[0] = mx;
        red_cnt[0] = nv;
      }
    }
    __syncthreads();
    kmin = red_min[0];
    kmax = red_max[0];
    nval = red_cnt[0];
  }

  kmin += 1u;  // the minimum was taken over key - 1
  uint32_t prefix = 0;
  int shift = 32;            // number of low key bits not yet resolved
  uint32_t need = K;
  const bool take_all = nval <= static_cast<uint32_t>(K);
  if (!take_all) {
    const uint32_t diff = kmin ^ kmax;
    shift = diff == 0u ? 0 : 32 - __clz(diff);  // bits above `shift` are common to all keys
    prefix = shift >= 32 ? 0u : (kmax >> shift);
  }
  int hb = 0;
  bool first = true;
#pragma unroll 1
  while (!take_all && shift > 0) {
    const int wbits = min(DIGIT, shift);
    const int nb = 1 << wbits;
    const int nshift = shift - wbits;
    uint32_t* h = hist[hb];
    for (int i = threadIdx.x; i < nb; i += THREADS) h[i] = 0;
    __syncthreads();
    if (first) {
      // every valid key carries the common prefix
#pragma unroll
      for (int j = 0; j < ITEMS; ++j) {
        const uint32_t u = key[j];
        if (u != 0u) atomicAdd(&h[(u >> nshift) & (nb - 1)], 1u);
      }
    } else {
#pragma unroll
      for (int j = 0; j < ITEMS; ++j) {
        const uint32_t u = key[j];
        if (u != 0u && (u >> shift) == prefix) atomicAdd(&h[(u >> nshift) & (nb - 1)], 1u);
      }
    }
    __syncthreads();
    // thread t owns bins nb-1-t*bpt .. nb-(t+1)*bpt: thread 0 the highest ones
    const int bpt = nb >= THREADS ? nb / THREADS : 1;
    const bool owner = threadIdx.x * bpt < nb;
    const int b0 = nb - (threadIdx.x + 1) * bpt;  // lowest bin of this thread
    uint32_t mine = 0;
    if (owner) {
      if (bpt % 4 == 0) {
        for (int q = 0; q < bpt; q += 4) {
          const uint4 v4 = *reinterpret_cast<const uint4*>(h + b0 + q);
          mine += v4.x + v4.y + v4.z + v4.w;
        }
      } else {
        for (int j = 0; j < bpt; ++j) mine += h[b0 + j];
      }
    }
    if constexpr (CLUSTER) {
      // the row's count of this thread's bins: the same thread's partial in every CTA
      cl_part[hb][threadIdx.x] = mine;
      cg::this_cluster().sync();
      mine = 0;
#pragma unroll
      for (int c = 0; c < kClusterMaxCtas; ++c)
        if (c < nparts) mine += cg::this_cluster().map_shared_rank(cl_part[hb], c)[threadIdx.x];
    }
    unsigned long long tot64;
    const uint32_t excl = static_cast<uint32_t>(block_exclusive_scan64<THREADS>(mine, warp_tot64, tot64));
    const bool finder = owner && excl < need && need <= excl + mine;
    constexpr int BPT = NB >= THREADS ? NB / THREADS : 1;
    if constexpr (CLUSTER && BPT == 8 && kClusterMaxCtas == 8) {
      // The finder's warp reads the finder's bins from every CTA together: lane 8*c4 + j
      // loads bin j of CTAs c4 and c4 + 4; shuffles add the CTAs up.
      const unsigned fm = __ballot_sync(0xffffffffu, finder);
      if (fm != 0u && bpt == BPT) {
        const int fl = __ffs(fm) - 1;
        const int fb0 = __shfl_sync(0xffffffffu, b0, fl);
        const int c4 = lane >> 3, j = lane & 7;
        const int bin = fb0 + BPT - 1 - j;
        uint32_t v = 0;
        if (c4 < nparts) v += cg::this_cluster().map_shared_rank(h, c4)[bin];
        if (c4 + 4 < nparts) v += cg::this_cluster().map_shared_rank(h, c4 + 4)[bin];
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        uint32_t cnt[BPT];
#pragma unroll
        for (int q = 0; q < BPT; ++q) cnt[q] = __shfl_sync(0xffffffffu, v, q);
        if (lane == fl) {
          uint32_t above = excl;
#pragma unroll
          for (int q = 0; q < BPT; ++q) {
            if (above < need) {
              if (above + cnt[q] >= need) {
                sh_bin = static_cast<uint32_t>(fb0 + BPT - 1 - q);
                sh_above = above;
                sh_inbin = cnt[q];
              }
              above += cnt[q];
            }
          }
        }
      } else if (finder) {
        uint32_t cnt[BPT];
#pragma unroll
        for (int q = 0; q < BPT; ++q) cnt[q] = 0;
#pragma unroll
        for (int c = 0; c < kClusterMaxCtas; ++c) {
          if (c < nparts) {
            const uint32_t* hc = cg::this_cluster().map_shared_rank(h, c);
#pragma unroll
            for (int q = 0; q < BPT; ++q)
              if (q < bpt) cnt[q] += hc[b0 + bpt - 1 - q];
          }
        }
        uint32_t above = excl;
#pragma unroll
        for (int q = 0; q < BPT; ++q) {
          if (q < bpt && above < need) {
            if (above + cnt[q] >= need) {
              sh_bin = static_cast<uint32_t>(b0 + bpt - 1 - q);
              sh_above = above;
              sh_inbin = cnt[q];
            }
            above += cnt[q];
          }
        }
      }
    } else if (finder) {
      // the row's count of each of this thread's bins, highest bin first
      uint32_t cnt[BPT];
#pragma unroll
      for (int j = 0; j < BPT; ++j) cnt[j] = 0;
      if constexpr (CLUSTER) {
#pragma unroll
        for (int c = 0; c < kClusterMaxCtas; ++c) {
          if (c < nparts) {
            const uint32_t* hc = cg::this_cluster().map_shared_rank(h, c);
#pragma unroll
            for (int j = 0; j < BPT; ++j)
              if (j < bpt) cnt[j] += hc[b0 + bpt - 1 - j];
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < BPT; ++j)
          if (j < bpt) cnt[j] = h[b0 + bpt - 1 - j];
      }
      uint32_t above = excl;
#pragma unroll
      for (int j = 0; j < BPT; ++j) {
        if (j < bpt && above < need) {
          if (above + cnt[j] >= need) {
            sh_bin = static_cast<uint32_t>(b0 + bpt - 1 - j);
            sh_above = above;
            sh_inbin = cnt[j];
          }
          above += cnt[j];
        }
      }
    }
    __syncthreads();
    const uint32_t bin = sh_bin;
    need -= sh_above;
    const uint32_t in_bin = sh_inbin;
    prefix = (shift < 32 ? (prefix << wbits) : 0u) | bin;
    shift = nshift;
    if (CLUSTER) hb ^= 1;
    first = false;
    if (in_bin == need) break;  // the whole bin is taken: no further digits needed
    if (shift > 0 && in_bin <= static_cast<uint32_t>(kGatherMax)) {
      // Few keys left in the threshold bin: gather them into shared memory and finish the
      // selection there instead of more passes over the whole row.
#pragma unroll
      for (int j = 0; j < ITEMS; ++j) {
        const uint32_t u = key[j];
        if (u != 0u && (u >> shift) == prefix) c_key[atomicAdd(&sh_ccount, 1u)] = u;
      }
      const uint32_t m = in_bin;
      const uint32_t* ck = c_key;
      if constexpr (CLUSTER) {
        cg::this_cluster().sync();
        if (warp == 0) {  // lane c reads CTA c's count
          const uint32_t cnt =
              lane < nparts ? *cg::this_cluster().map_shared_rank(&sh_ccount, lane) : 0u;
          uint32_t incl = cnt;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          if (lane <= nparts) c_off[lane] = incl - cnt;
        }
        __syncthreads();
        // the cluster's keys, gathered into the output staging area (not yet in use)
        uint32_t* c_all = reinterpret_cast<uint32_t*>(stage_smem);
        for (uint32_t i = threadIdx.x; i < m; i += THREADS) {
          int c = 0;
          while (c + 1 < nparts && c_off[c + 1] <= i) ++c;
          c_all[i] = cg::this_cluster().map_shared_rank(c_key, c)[i - c_off[c]];
        }
        ck = c_all;
      }
      __syncthreads();
      if (m <= static_cast<uint32_t>(kCountMax)) {
        // the threshold key is the candidate with fewer than `need` keys above it and at
        // least `need` at or above it
        if (threadIdx.x < m) {
          const uint32_t kc = ck[threadIdx.x];
          uint32_t gt = 0, ge = 0;
#pragma unroll 8
          for (uint32_t j = 0; j < m; ++j) {
            const uint32_t v = ck[j];
            gt += v > kc;
            ge += v >= kc;
          }
          if (gt < need && need <= ge) {
            sh_theta = kc;
            sh_needt = need - gt;
          }
        }
        __syncthreads();
        prefix = sh_theta;
        need = sh_needt;
        shift = 0;
      } else {
#pragma unroll 1
        while (shift > 0) {
          const int wb = min(8, shift);
          const int nbs = 1 << wb;
          const int ns = shift - wb;
          for (int i = threadIdx.x; i < nbs; i += THREADS) h_small[i] = 0;
          __syncthreads();
          for (uint32_t i = threadIdx.x; i < m; i += THREADS) {
            const uint32_t u = ck[i];
            if ((u >> shift) == prefix) atomicAdd(&h_small[(u >> ns) & (nbs - 1)], 1u);
          }
          __syncthreads();
          if (warp == 0) {
            // lane l owns bins nbs-1-l*bpl .. nbs-(l+1)*bpl: lane 0 the highest ones
            const int bpl = nbs >= 32 ? nbs / 32 : 1;
            const bool own = lane * bpl < nbs;
            const int lb0 = nbs - (lane + 1) * bpl;
            uint32_t c = 0;
            if (own)
              for (int q = 0; q < bpl; ++q) c += h_small[lb0 + q];
            uint32_t incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
              if (lane >= o) incl += y;
            }
            if (own && incl - c < need && need <= incl) {
              uint32_t above = incl - c;
              for (int q = bpl - 1; q >= 0; --q) {
                const uint32_t hc = h_small[lb0 + q];
                if (above + hc >= need) {
                  sh_bin = static_cast<uint32_t>(lb0 + q);
                  sh_above = above;
                  sh_inbin = hc;
                  break;
                }
                above += hc;
              }
            }
          }
          __syncthreads();
          need -= sh_above;
          prefix = (prefix << wb) | sh_bin;
          shift = ns;
          const uint32_t ib = sh_inbin;
          __syncthreads();  // h_small and the shared results are rewritten by the next digit
          if (ib == need) break;
        }
      }
      break;
    }
  }

  // ---- output: one scan of (above, equal) counts, then each thread writes its run ------
  // the threshold bin as a key range [lo, hi]: above it selected, inside it the lowest-indexed
  // keys up to need; every valid key is above an empty bin (hi = 0) when all are taken
  uint32_t bin_lo = 1u, bin_hi = 0u;
  if (!take_all) {
    const uint32_t base = shift >= 32 ? 0u : (prefix << shift);
    bin_hi = shift >= 32 ? 0xffffffffu : (base | ((1u << shift) - 1u));
    bin_lo = max(base, 1u);
  }
  Mask gt_mask = 0, eq_mask = 0;
#pragma unroll
  for (int j = 0; j < ITEMS; ++j) {
    const uint32_t u = key[j];
    const bool g = u > bin_hi;
    gt_mask |= Mask(g) << j;
    eq_mask |= Mask(!g && u >= bin_lo) << j;
  }
  constexpr unsigned long long kLow = 0xffffffffull;
  unsigned long long tot;
  const unsigned long long packed =
      (static_cast<unsigned long long>(__popcll(gt_mask)) << 32) | __popcll(eq_mask);
  const unsigned long long ex = block_exclusive_scan64<THREADS>(packed, warp_tot64, tot);
  // packed counts of the CTAs before this one (cluster) and of the whole row
  unsigned long long off = 0, all = tot;
  if constexpr (CLUSTER) {
    // every CTA's counts are pushed into every CTA of the cluster; after the barrier each
    // thread adds them up from its own shared memory. No CTA touches another's shared memory
    // after this barrier, so a CTA may leave as soon as its own writes are done.
    if (static_cast<int>(threadIdx.x) < nparts)
      *cg::this_cluster().map_shared_rank(&cl_tots[part], static_cast<int>(threadIdx.x)) = tot;
    cg::this_cluster().sync();
    all = 0ull;
#pragma unroll
    for (int c = 0; c < kClusterMaxCtas; ++c) {
      if (c < nparts) {
        const unsigned long long v = cl_tots[c];
        off += c < part ? v : 0ull;
        all += v;
      }
    }
  }
  const uint32_t gt_before = static_cast<uint32_t>((off + ex) >> 32);
  const uint32_t eq_before = static_cast<uint32_t>((off + ex) & kLow);
  const uint32_t n_sel_total =
      static_cast<uint32_t>(all >> 32) + min(static_cast<uint32_t>(all & kLow), need);
  // first output slot of this CTA and its number of selected elements
  const uint32_t eq_off = static_cast<uint32_t>(off & kLow);
  const uint32_t cta_slot0 = static_cast<uint32_t>(off >> 32) + min(eq_off, need);
  const uint32_t cta_sel = static_cast<uint32_t>(tot >> 32) +
                           min(eq_off + static_cast<uint32_t>(tot & kLow), need) - min(eq_off, need);
  uint32_t slot = gt_before + min(eq_before, need);
  // the equal keys this thread takes: its lowest-indexed ones, up to need over the row
  const uint32_t eq_take =
      need > eq_before ? min(need - eq_before, static_cast<uint32_t>(__popcll(eq_mask))) : 0u;
  Mask sel = gt_mask;
  {
    Mask rest = eq_mask;
    for (uint32_t q = 0; q < eq_take; ++q) {
      const Mask low = rest & (~rest + 1);
      sel |= low;
      rest ^= low;
    }
  }
  const bool staged = K <= kStageMaxK;
  int32_t* st_idx = reinterpret_cast<int32_t*>(stage_smem);
  // selected elements in index order; scores are read back from the row (still in cache)
  while (sel != 0 && slot < static_cast<uint32_t>(K)) {
    const int64_t i = my0 + lowest_set_bit(sel);
    sel &= sel - 1;
    if (staged) {
      st_idx[slot - cta_slot0] = static_cast<int32_t>(i);
    } else {
      int32_t id = in_idx ? in_idx[i] : static_cast<int32_t>(lo + i);
      id = map_id(map, id, a.map_shift);
      a.out_idx[out_base + slot] = id;
      if (a.out_val) a.out_val[out_base + slot] = vals[i];
    }
    ++slot;
  }
  if (staged) {
    __syncthreads();
    const uint32_t n_out =
        cta_slot0 >= static_cast<uint32_t>(K) ? 0u : min(cta_sel, static_cast<uint32_t>(K) - cta_slot0);
    for (uint32_t sl = threadIdx.x; sl < n_out; sl += THREADS) {
      const int32_t i = st_idx[sl];
      int32_t id = in_idx ? in_idx[i] : static_cast<int32_t>(lo + i);
      id = map_id(map, id, a.map_shift);
      a.out_idx[out_base + cta_slot0 + sl] = id;
      if (a.out_val) a.out_val[out_base + cta_slot0 + sl] = vals[i];
    }
  }
  for (int64_t j = n_sel_total + static_cast<int64_t>(part) * THREADS + threadIdx.x; j < K;
       j += static_cast<int64_t>(THREADS) * nparts) {
    a.out_idx[out_base + j] = -1;
    if (a.out_val) a.out_val[out_base + j] = -INFINITY;
  }
}

// ---------------------------------------------------------------------------------------
// Many rows longer than a register-resident select holds (chunked prefill past 32K keys):
// a threshold from a sample, then one streaming pass.
//   1. Sample: every kSampleStride-th tile of 128 elements (m of the row's n), kept in shared
//      memory after its first read. Its key range and a 12-bit histogram below the range's
//      common high bits give the bins of the sample's r-th and 4r-th largest keys,
//      r = 5/4 * K * m / n + 8, whose lower edges are the thresholds tau: about 5/4 of K
//      elements of the row are expected at or above the first.
//   2. One pass gathers every valid element >= tau into shared memory in index order: the
//      row streams through a ring of 16 KB bulk copies (up to four in flight), each thread
//      tests 8 consecutive elements of a step, and one warp ballot (a shuffle scan when a lane
//      has two or more) plus one barrier with warp reductions give their slots. Fewer than K
//      gathered (the estimate was too high): the pass is repeated at the lower tau, then at
//      every element; more than the buffer holds (many equal keys): the row takes the
//      multi-pass radix select.
//   3. The exact K-th largest among the gathered keys (8-bit digit histograms), and the
//      selected elements written in index order: every key above it and the lowest-indexed
//      keys equal to it.
// ---------------------------------------------------------------------------------------
constexpr int kSampleStride = 16;
constexpr int kLongCap = 4096;                    // gathered elements
constexpr int kRingStep = 4096;                   // elements per gather step (8 per thread)
constexpr int kRingSlots = 5;                     // steps in the copy ring (up to four in flight)
constexpr int kRingFloats = kRingSlots * kRingStep;
constexpr int kLongSmem = (kRingFloats + 2 * kLongCap) * 4;
constexpr uint64_t kLongTimeoutNs = 2000000000ull;  // bound on one copy's wait
static_assert(kRingStep == 8 * kSelThreads, "eight elements per thread per step");
static_assert(kRingFloats >= kBins && 2 * kLongCap >= kBins, "histograms fit either region");

// Bit j set when element j of (d0, d1) is >= t (a NaN compares false).
__device__ __forceinline__ uint32_t ge_bits8(const float4& d0, const float4& d1, float t) {
  const float v[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t r;
    asm("set.ge.u32.f32 %0, %1, %2;" : "=r"(r) : "f"(v[j]), "f"(t));
    m |= r & (1u << j);
  }
  return m;
}

// Inclusive prefix sum over the warp (all lanes take part).
__device__ __forceinline__ uint32_t warp_inclusive_sum(uint32_t x) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1)
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .u32 y;\n\t"
        "shfl.sync.up.b32 y|p, %0, %1, 0, -1;\n\t"
        "@p add.u32 %0, %0, y;\n\t}"
        : "+r"(x)
        : "r"(o));
  return x;
}

// One bulk copy (no multicast) of `bytes` from global memory into this CTA's shared memory,
// completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__global__ void __launch_bounds__(kSelThreads, 2) long_select_kernel(const SelectArgs a, int row0) {
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t step_tot[2][kSelWarps];
  __shared__ uint32_t sh[2];
  extern __shared__ __align__(16) uint32_t long_smem[];
  float* ring = reinterpret_cast<float*>(long_smem);    // the sample, then the gather's copies
  float* samp = ring;
  uint32_t* hist = long_smem;                            // radix histograms once the ring is idle
  uint32_t* ck = long_smem + kRingFloats;                // gathered keys, index order
  int32_t* cix = reinterpret_cast<int32_t*>(ck + kLongCap);  // their element indices
  uint32_t* hist_s = ck;                                 // the sample's histogram (before gathering)
  __shared__ uint32_t red_min[kSelWarps], red_max[kSelWarps], red_cnt[kSelWarps];
  __shared__ uint32_t sh_bin, sh_above, sh_inbin, sh_tau_bin[2];
  __shared__ unsigned long long warp_tot64[kSelWarps];
  __shared__ __align__(8) uint64_t full[kRingSlots];  // one per ring slot: its copy landed
  __shared__ int abort_s;

  const int r = row0 + static_cast<int>(blockIdx.x);
  if (r >= a.rows) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t n = row_length(a, r);
  const float* vals = a.vals + static_cast<int64_t>(r) * a.ld;
  const int32_t* in_idx = a.in_idx ? a.in_idx + static_cast<int64_t>(r) * a.ld : nullptr;
  const uint32_t lanes_below = (1u << lane) - 1u;
  const int32_t* map =
      a.idx_map ? a.idx_map + static_cast<int64_t>(r / a.rows_per_batch) * a.map_stride : nullptr;
  const int64_t out_base = static_cast<int64_t>(r) * a.out_ld;
  const uint32_t K = static_cast<uint32_t>(a.K);
  // the copies move whole 16-byte chunks: rows must start aligned and end inside their stride
  // (and the gathering pass counts elements in 32 bits)
  if ((reinterpret_cast<uintptr_t>(vals) & 15) != 0 || (a.ld & 3) != 0 || n > a.ld ||
      n > 0x7fffffff - kRingStep) {
    radix_row(a, r, 0, hist, warp_tot, sh);
    return;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kRingSlots; ++i) mbar_init(&full[i], 1);
    abort_s = 0;
    fence_mbarrier_init();
  }

  // ---- 1. the sample's key range, then its histogram below the common high bits
  const int64_t n_tiles = (n + 127) / 128;
  const int64_t n_samp = (n_tiles + kSampleStride - 1) / kSampleStride;
  const bool cached = n_samp * 128 <= kRingFloats;  // the sample is kept for the second read
  // lane l of a warp reads elements 4l .. 4l + 3 of a sampled tile; a warp has four tiles'
  // loads in flight at once
  uint32_t kmin = 0xffffffffu, kmax = 0u, cnt = 0u;
  for (int64_t t0 = warp; t0 < n_samp; t0 += 4 * kSelWarps) {
    float4 q[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t t = t0 + u * kSelWarps;
      const int64_t i = t * kSampleStride * 128 + 4 * lane;
      if (t < n_samp && i + 4 <= n) {
        q[u] = *reinterpret_cast<const float4*>(vals + i);
      } else {
        const bool in = t < n_samp;
        q[u] = make_float4(in && i < n ? vals[i] : -INFINITY, in && i + 1 < n ? vals[i + 1] : -INFINITY,
                           in && i + 2 < n ? vals[i + 2] : -INFINITY,
                           in && i + 3 < n ? vals[i + 3] : -INFINITY);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t t = t0 + u * kSelWarps;
      if (t < n_samp) {
        if (cached) reinterpret_cast<float4*>(samp + t * 128)[lane] = q[u];
        const float v4[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (is_valid(v4[c])) {
            const uint32_t k = order_key(v4[c]);
            kmin = min(kmin, k);
            kmax = max(kmax, k);
            ++cnt;
          }
        }
      }
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  if (lane == 0) {
    red_min[warp] = kmin;
    red_max[warp] = kmax;
    red_cnt[warp] = cnt;
  }
  for (int i = threadIdx.x; i < kBins; i += kSelThreads) hist_s[i] = 0;
  __syncthreads();
  kmin = 0xffffffffu;
  kmax = 0u;
  uint32_t m = 0u;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) {
    kmin = min(kmin, red_min[w]);
    kmax = max(kmax, red_max[w]);
    m += red_cnt[w];
  }
  const uint32_t diff = kmin ^ kmax;
  const int shift = diff == 0u ? 0 : 32 - __clz(diff);   // bits above are common to the sample
  const int wbits = min(12, shift);
  const int ns = shift - wbits;
  const uint32_t top = shift >= 32 ? 0u : (kmax >> shift);
  const uint32_t bmask = (1u << wbits) - 1u;
  if (cached) {  // the sample as kept (elements past the row's end are -inf)
    for (int64_t i = threadIdx.x; i < n_samp * 128; i += kSelThreads) {
      const float v = samp[i];
      if (is_valid(v)) atomicAdd(&hist_s[(order_key(v) >> ns) & bmask], 1u);
    }
  } else {
    for (int64_t t = warp; t < n_samp; t += kSelWarps) {
      const int64_t base = t * kSampleStride * 128;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t i = base + u * 32 + lane;
        const float v = i < n ? vals[i] : -INFINITY;
        if (is_valid(v)) atomicAdd(&hist_s[(order_key(v) >> ns) & bmask], 1u);
      }
    }
  }
  __syncthreads();

  // the bins holding the sample's want-th largest key for want = r0 and 4 r0, by one block
  // scan from the top; a want beyond the sample takes every element (tau = 0: valid keys > 0)
  const uint64_t r0 = static_cast<uint64_t>(1.25 * K * (static_cast<double>(m) / (n > 0 ? n : 1))) + 8;
  uint32_t tau0 = 0u, tau1 = 0u;
  {
    const int nb = 1 << wbits;
    const int bpt = nb >= kSelThreads ? nb / kSelThreads : 1;
    const bool owner = static_cast<int>(threadIdx.x) * bpt < nb;
    const int b0 = nb - (static_cast<int>(threadIdx.x) + 1) * bpt;
    uint32_t mine = 0;
    if (owner)
      for (int q = 0; q < bpt; ++q) mine += hist_s[b0 + q];
    uint32_t tot;
    const uint32_t incl = block_inclusive_scan(mine, warp_tot, tot);
    const uint32_t excl = incl - mine;
#pragma unroll
    for (int wi = 0; wi < 2; ++wi) {
      const uint64_t want = wi == 0 ? r0 : r0 * 4;
      if (owner && want < m && excl < want && want <= incl) {
        uint32_t above = excl;
        for (int q = bpt - 1; q >= 0; --q) {
          above += hist_s[b0 + q];
          if (above >= want) {
            sh_tau_bin[wi] = static_cast<uint32_t>(b0 + q);
            break;
          }
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int wi = 0; wi < 2; ++wi) {
      const uint64_t want = wi == 0 ? r0 : r0 * 4;
      if (want < m) {
        const uint32_t b = sh_tau_bin[wi];
        const uint32_t t = shift >= 32 ? (b << ns) : ((top << shift) | (b << ns));
        (wi == 0 ? tau0 : tau1) = t == 0u ? 1u : t;
      }
    }
  }

  // ---- 2. one gathering pass (repeated at a lower threshold if it found fewer than K)
  uint32_t C = 0;        // valid elements >= tau in the row
  uint32_t tau = 0u;
  const int64_t n_steps = (n + kRingStep - 1) / kRingStep;
  // Fill f of the ring (counted over every pass) goes to slot f % kRingSlots and completes
  // phase (f / kRingSlots) & 1 of that slot's barrier; thread 0 issues the copies and waits.
  uint32_t fbase = 0;
  auto fill = [&](int64_t st) {  // thread 0: copy step st of this pass
    const uint32_t f = fbase + static_cast<uint32_t>(st);
    const int slot = static_cast<int>(f % kRingSlots);
    const int64_t e0 = st * kRingStep;
    const int64_t cnt = min(static_cast<int64_t>(kRingStep), n - e0);
    const uint32_t bytes = static_cast<uint32_t>((cnt * 4 + 15) & ~static_cast<int64_t>(15));
    mbar_arrive_expect_tx(&full[slot], bytes);
    bulk_load(ring + slot * kRingStep, vals + e0, bytes, &full[slot]);
  };
  auto landed = [&](int64_t st) {  // thread 0: bounded wait for step st's copy
    const uint32_t f = fbase + static_cast<uint32_t>(st);
    return mbar_wait(&full[f % kRingSlots], (f / kRingSlots) & 1u, &abort_s, kLongTimeoutNs);
  };
#pragma unroll 1
  for (int attempt = 0; attempt < 3; ++attempt) {
    tau = attempt == 0 ? tau0 : (attempt == 1 ? tau1 : 0u);
    if (attempt == 1 && tau == tau0) continue;  // the same threshold again: take every element
    // The test is one float compare against the value whose key is tau (clamped to the finite
    // range: every valid element passes tau = 1), a superset of key >= tau that differs only
    // at -0.0; keys are formed for the gathered elements alone.
    const float tau_f = tau <= 0x00800000u ? -FLT_MAX : key_value_long(tau);
    C = 0;
    int ok = 1;
    if (threadIdx.x == 0) {
      fence_proxy_async_smem();  // the ring's earlier contents were written by the threads
      for (int64_t j = 0; j < kRingSlots - 1 && j < n_steps; ++j) fill(j);
      ok = n_steps < 1 || landed(0);
    }
    // 32-bit loop state (the row is shorter than 2^31 - kRingStep elements); the slot and its
    // phase advance with the step
    const int ns = static_cast<int>(n_steps);
    int slot = static_cast<int>(fbase % kRingSlots);
    uint32_t ph = (fbase / kRingSlots) & 1u;
    uint32_t i0 = 8u * threadIdx.x;  // index of this thread's first element of the step
    int s = 0;
    if (__syncthreads_and(ok)) {
#pragma unroll 1
      for (; s < ns; ++s, i0 += kRingStep) {
        (void)mbar_try_wait(&full[slot], ph);  // complete: orders the reads
        const float* mine = ring + slot * kRingStep + 8 * threadIdx.x;
        const float4 d0 = reinterpret_cast<const float4*>(mine)[0];
        const float4 d1 = reinterpret_cast<const float4*>(mine)[1];
        // bit j: element j of this thread is >= tau (past the row's end on the last step: no)
        uint32_t msk = ge_bits8(d0, d1, tau_f);
        if (s + 1 == ns) {
          const int left = static_cast<int>(static_cast<uint32_t>(n) - i0);
          msk &= left >= 8 ? 0xffu : (left <= 0 ? 0u : ((1u << left) - 1u));
        }
        const uint32_t nm = __popc(msk);
        // this lane's first slot in the warp and the warp's count: one ballot while no lane
        // has two or more (the usual case: about 1 % of the elements pass), else a scan
        uint32_t ex, wt;
        if (__any_sync(0xffffffffu, nm > 1u)) {
          const uint32_t incl = warp_inclusive_sum(nm);
          ex = incl - nm;
          wt = __shfl_sync(0xffffffffu, incl, 31);
        } else {
          const uint32_t b = __ballot_sync(0xffffffffu, nm != 0u);
          ex = __popc(b & lanes_below);
          wt = __popc(b);
        }
        uint32_t* st = step_tot[s & 1];
        if (lane == 0) st[warp] = wt;
        ok = 1;
        if (threadIdx.x == 0 && s + 1 < ns) ok = landed(s + 1);
        // every thread is done with the previous step's slot, which takes step s + R - 1
        if (!__syncthreads_and(ok)) break;
        if (threadIdx.x == 0 && s + kRingSlots - 1 < ns) fill(s + kRingSlots - 1);
        const uint32_t x = lane < kSelWarps ? st[lane] : 0u;
        const uint32_t tot = __reduce_add_sync(0xffffffffu, x);
        const uint32_t before = __reduce_add_sync(0xffffffffu, lane < warp ? x : 0u);
        // this thread's elements >= tau, in index order; their values are read again from the
        // slot, which is not refilled before the next step's barrier
        uint32_t at = C + before + ex;
        for (uint32_t mm = msk; mm != 0u; mm &= mm - 1u, ++at) {
          const int j = __ffs(mm) - 1;
          if (at < static_cast<uint32_t>(kLongCap)) {
            ck[at] = order_key(mine[j]);
            cix[at] = static_cast<int32_t>(i0 + j);
          }
        }
        C += tot;
        if (++slot == kRingSlots) {
          slot = 0;
          ph ^= 1u;
        }
      }
    }
    if (s < ns) {
      // a copy did not land in time: report it, let every copy of this pass that was issued
      // land (bounded) before the CTA's shared memory is released, and leave the row
      if (threadIdx.x == 0) {
        if (a.status != nullptr && atomicCAS(&a.status->code, 0, static_cast<int>(ADX_ETIMEOUT)) == 0) {
          a.status->where = kWhereSelect;
          a.status->info0 = 3;
          a.status->info1 = r;
        }
        volatile int never = 0;
        const int64_t issued = min(n_steps, static_cast<int64_t>(s) + kRingSlots - 1);  // fills s .. issued-1 may be pending
        for (int64_t j = s; j < issued; ++j) {
          const uint32_t f = fbase + static_cast<uint32_t>(j);
          (void)mbar_wait(&full[f % kRingSlots], (f / kRingSlots) & 1u, &never, kLongTimeoutNs);
        }
      }
      return;
    }
    fbase += static_cast<uint32_t>(n_steps);
    __syncthreads();
    if (C >= K || tau == 0u) break;
  }
  if (C > static_cast<uint32_t>(kLongCap)) {  // too many equal keys to gather: radix passes
    radix_row(a, r, 0, hist, warp_tot, sh);
    return;
  }

  // ---- 3. the K-th largest gathered key (C > K), then the output in index order
  uint32_t prefix = 0, need = 0;
  int sh2 = 32;  // gathered keys compare by their bits above sh2 (32: every one is selected)
  if (C > K) {
    // common high bits of the gathered keys
    uint32_t gmin = 0xffffffffu, gmax = 0u;
    for (uint32_t i = threadIdx.x; i < C; i += kSelThreads) {
      gmin = min(gmin, ck[i]);
      gmax = max(gmax, ck[i]);
    }
    gmin = __reduce_min_sync(0xffffffffu, gmin);
    gmax = __reduce_max_sync(0xffffffffu, gmax);
    if (lane == 0) {
      red_min[warp] = gmin;
      red_max[warp] = gmax;
    }
    __syncthreads();
    gmin = 0xffffffffu;
    gmax = 0u;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) {
      gmin = min(gmin, red_min[w]);
      gmax = max(gmax, red_max[w]);
    }
    const uint32_t gd = gmin ^ gmax;
    sh2 = gd == 0u ? 0 : 32 - __clz(gd);
    prefix = sh2 >= 32 ? 0u : (gmax >> sh2);
    need = K;
    __syncthreads();  // red_* are read; hist is free
#pragma unroll 1
    while (sh2 > 0) {
      const int wb = min(8, sh2);
      const int nbs = 1 << wb;
      const int nsh = sh2 - wb;
      for (int i = threadIdx.x; i < nbs; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      for (uint32_t i = threadIdx.x; i < C; i += kSelThreads) {
        const uint32_t u = ck[i];
        if (sh2 >= 32 || (u >> sh2) == prefix) atomicAdd(&hist[(u >> nsh) & (nbs - 1)], 1u);
      }
      __syncthreads();
      if (warp == 0) {  // lane l owns bins nbs-1-l*bpl .. nbs-(l+1)*bpl
        const int bpl = nbs >= 32 ? nbs / 32 : 1;
        const bool own = lane * bpl < nbs;
        const int lb0 = nbs - (lane + 1) * bpl;
        uint32_t c = 0;
        if (own)
          for (int q = 0; q < bpl; ++q) c += hist[lb0 + q];
        uint32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        if (own && incl - c < need && need <= incl) {
          uint32_t above = incl - c;
          for (int q = bpl - 1; q >= 0; --q) {
            const uint32_t hc = hist[lb0 + q];
            if (above + hc >= need) {
              sh_bin = static_cast<uint32_t>(lb0 + q);
              sh_above = above;
              sh_inbin = hc;
              break;
            }
            above += hc;
          }
        }
      }
      __syncthreads();
      need -= sh_above;
      prefix = (sh2 >= 32 ? 0u : (prefix << wb)) | sh_bin;
      sh2 = nsh;
      const uint32_t ib = sh_inbin;
      __syncthreads();
      if (ib == need) break;
    }
  }
  // thread t writes the gathered elements [t * ipt, (t + 1) * ipt) of its share
  const uint32_t ipt = (C + kSelThreads - 1) / kSelThreads;
  const uint32_t e0 = min(C, threadIdx.x * ipt), e1 = min(C, e0 + ipt);
  uint32_t gt = 0, eq = 0;
  for (uint32_t i = e0; i < e1; ++i) {
    const uint32_t t = sh2 >= 32 ? 1u : (ck[i] >> sh2);
    if (sh2 >= 32 || t > prefix) ++gt;
    else if (t == prefix) ++eq;
  }
  unsigned long long tot64;
  const unsigned long long ex = block_exclusive_scan64<kSelThreads>(
      (static_cast<unsigned long long>(gt) << 32) | eq, warp_tot64, tot64);
  uint32_t gt_b = static_cast<uint32_t>(ex >> 32), eq_b = static_cast<uint32_t>(ex & 0xffffffffull);
  const uint32_t eq_need = sh2 >= 32 ? 0u : need;
  for (uint32_t i = e0; i < e1; ++i) {
    const uint32_t u = ck[i];
    const uint32_t t = sh2 >= 32 ? 1u : (u >> sh2);
    const bool g = sh2 >= 32 || t > prefix;
    const bool e = !g && t == prefix;
    if (g || (e && eq_b < eq_need)) {
      const uint32_t slot = gt_b + min(eq_b, eq_need);
      if (slot < K) {
        int32_t id = in_idx ? in_idx[cix[i]] : cix[i];
        id = map_id(map, id, a.map_shift);
        a.out_idx[out_base + slot] = id;
        if (a.out_val) a.out_val[out_base + slot] = key_value_long(u);
      }
    }
    gt_b += g;
    eq_b += e;
  }
  const uint32_t n_sel = min(K, static_cast<uint32_t>(tot64 >> 32) +
                                   min(static_cast<uint32_t>(tot64 & 0xffffffffull), eq_need));
  for (uint32_t j = n_sel + threadIdx.x; j < K; j += kSelThreads) {
    a.out_idx[out_base + j] = -1;
    if (a.out_val) a.out_val[out_base + j] = -INFINITY;
  }
}

// ---------------------------------------------------------------------------------------
// Short rows (up to 32 x ITEMS elements, e.g. the block rows of the hierarchical indexer):
// one warp per row. Lane l holds elements j*32 + l (coalesced loads). The K-th largest key
// is found bit by bit below the row's common high bits (a warp-wide count of keys at or
// above each candidate); the keys above it and the lowest-indexed keys equal to it are
// written in ascending index order, slots from ballot prefix counts.
// ---------------------------------------------------------------------------------------
constexpr int kWarpSelRows = 8;  // rows (warps) per CTA

__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

template <int ITEMS>
__global__ void __launch_bounds__(32 * kWarpSelRows) select_warp_kernel(const SelectArgs a) {
  const int lane = threadIdx.x & 31;
  const int r = static_cast<int>(blockIdx.x) * kWarpSelRows + static_cast<int>(threadIdx.x >> 5);
  if (r >= a.rows) return;  // the whole warp
  const int64_t n = row_length(a, r);
  const float* vals = a.vals + static_cast<int64_t>(r) * a.ld;
  const int32_t* in_idx = a.in_idx ? a.in_idx + static_cast<int64_t>(r) * a.ld : nullptr;
  const int32_t* map =
      a.idx_map ? a.idx_map + static_cast<int64_t>(r / a.rows_per_batch) * a.map_stride : nullptr;
  const int64_t out_base = static_cast<int64_t>(r) * a.out_ld;
  const uint32_t K = static_cast<uint32_t>(a.K);
  uint32_t key[ITEMS];
  uint32_t nval = 0, kmin = 0xffffffffu, kmax = 0u;
  int64_t forced = -1;  // besides element 0
  if (a.force_blk != nullptr) {
    const int32_t cur = a.force_blk[r];
    if (cur + 1 > a.force_n) forced = cur;
  }
#pragma unroll
  for (int j = 0; j < ITEMS; ++j) {
    const int64_t i = static_cast<int64_t>(j) * 32 + lane;
    float v = i < n ? vals[i] : -INFINITY;
    if (forced >= 0 && (i == 0 || i == forced)) v = INFINITY;
    const bool ok = is_valid(v);
    key[j] = ok ? order_key(v) : 0u;  // 0 = invalid (valid keys are > 0)
    nval += ok;
    kmin = ok ? min(kmin, key[j]) : kmin;
    kmax = max(kmax, key[j]);
  }
  nval = __reduce_add_sync(0xffffffffu, nval);
  const bool take_all = nval <= K;
  uint32_t theta = 1u, need_eq = 0u;
  if (!take_all) {
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    const uint32_t diff = kmin ^ kmax;
    const int hb = diff == 0u ? 0 : 32 - __clz(diff);  // bits hb.. are common to every key
    theta = hb >= 32 ? 0u : (kmax >> hb) << hb;        // count(key >= theta) = nval >= K
    for (int b = hb - 1; b >= 0; --b) {
      const uint32_t cand = theta | (1u << b);
      uint32_t c = 0;
#pragma unroll
      for (int j = 0; j < ITEMS; ++j) c += key[j] >= cand;
      if (__reduce_add_sync(0xffffffffu, c) >= K) theta = cand;
    }
    uint32_t gt = 0;
#pragma unroll
    for (int j = 0; j < ITEMS; ++j) gt += key[j] > theta;
    need_eq = K - __reduce_add_sync(0xffffffffu, gt);  // >= 1 equal keys to take
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint32_t base = 0, eq_seen = 0;
#pragma unroll
  for (int j = 0; j < ITEMS; ++j) {
    const uint32_t u = key[j];
    const bool eq = !take_all && u == theta;
    const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
    const bool sel = take_all ? u != 0u : (u > theta || (eq && eq_seen + __popc(eqb & lt_mask) < need_eq));
    eq_seen += __popc(eqb);
    const uint32_t sb = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const uint32_t slot = base + __popc(sb & lt_mask);
      const int32_t i = j * 32 + lane;
      int32_t id = in_idx ? in_idx[i] : i;
      id = map_id(map, id, a.map_shift);
      a.out_idx[out_base + slot] = id;
      if (a.out_val) a.out_val[out_base + slot] = key_value(u);
    }
    base += __popc(sb);
  }
  for (uint32_t sl = base + lane; sl < K; sl += 32) {
    a.out_idx[out_base + sl] = -1;
    if (a.out_val) a.out_val[out_base + sl] = -INFINITY;
  }
}

static_assert(kWarpSelectMax == 32 * 40, "the widest warp select instance");

template <int ITEMS>
cudaError_t launch_warp_select(const SelectArgs& a, cudaStream_t s, int* launched) {
  const int64_t grid = (static_cast<int64_t>(a.rows) + kWarpSelRows - 1) / kWarpSelRows;
  select_warp_kernel<ITEMS><<<static_cast<unsigned>(grid), 32 * kWarpSelRows, 0, s>>>(a);
  *launched = 1;
  return cudaGetLastError();
}

template <int THREADS, int DIGIT, int ITEMS = kRegItems>
cudaError_t launch_reg(const SelectArgs& a, int row0, int row1, cudaStream_t s, int* launched) {
  const int64_t grid = static_cast<int64_t>(row1 - row0) * a.n_seg;
  if (grid <= 0) return cudaSuccess;
  const size_t smem = a.K <= kStageMaxK ? static_cast<size_t>(a.K) * 4 : 0;
  auto kern = select_reg_kernel<THREADS, DIGIT, ITEMS, false>;
  if (smem > 0) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  kern<<<static_cast<unsigned>(grid), THREADS, smem, s>>>(a, row0);
  ++*launched;
  return cudaGetLastError();
}

// Rows [row0, row1) of a launch through the sample-threshold select (whole rows, K <= 2048).
cudaError_t launch_long(const SelectArgs& a, int row0, int row1, cudaStream_t s, int* launched) {
  const int64_t grid = static_cast<int64_t>(row1 - row0);
  if (grid <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(long_select_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kLongSmem);
  if (e != cudaSuccess) return e;
  // two CTAs per SM need the largest shared-memory carveout
  e = cudaFuncSetAttribute(long_select_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  long_select_kernel<<<static_cast<unsigned>(grid), kSelThreads, kLongSmem, s>>>(a, row0);
  ++*launched;
  return cudaGetLastError();
}

}  // namespace

int select_cluster_ctas(int64_t rows, int64_t n_max, int K, int sms, bool any_k) {
  constexpr int64_t cap = static_cast<int64_t>(kClusterThreads) * kClusterItems;
  if (rows <= 0 || rows >= sms || (!any_k && n_max <= 8ll * K)) return 0;
  const int64_t need = (n_max + cap - 1) / cap;
  if (need > kClusterMaxCtas) return 0;
  const int64_t fill = (2ll * sms) / rows;       // two CTAs of this class fit on an SM
  const int64_t useful = (n_max + 4095) / 4096;  // at least 4096 elements per CTA
  const int64_t cl = std::max(need, std::min(std::min(fill, useful), int64_t(kClusterMaxCtas)));
  return cl > 1 ? static_cast<int>(cl) : 0;
}

cudaError_t launch_select_cluster(const SelectArgs& a, int ctas, cudaStream_t s, int* launched) {
  *launched = 0;
  if (a.rows <= 0) return cudaSuccess;
  if (a.n_seg != 1 || ctas < 2 || ctas > kClusterMaxCtas ||
      static_cast<int64_t>(a.len_cap) > static_cast<int64_t>(ctas) * kClusterThreads * kClusterItems)
    return cudaErrorInvalidValue;
  auto kern = select_reg_kernel<kClusterThreads, 12, kClusterItems, true>;
  // output staging, which first holds the gathered keys of the threshold bin
  const size_t smem = std::max<size_t>(a.K <= kStageMaxK ? static_cast<size_t>(a.K) * 4 : 0,
                                       static_cast<size_t>(kGatherMax) * 4);
  if (smem > 0) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.rows) * static_cast<unsigned>(ctas), 1, 1);
  cfg.blockDim = dim3(kClusterThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(ctas);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a, 0);
  *launched = 1;
  return e;
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s, int* launched) {
  *launched = 0;
  const int64_t grid = static_cast<int64_t>(a.rows) * a.n_seg;
  if (grid <= 0) return cudaSuccess;
  const int64_t seg = a.n_seg == 1 ? a.len_cap : a.seg_len;
  // row-length classes (CTA size x elements per thread): 128x32, 256x32, 256x36, 512x32,
  // 1024x32; 256x36 takes rows just above 8192 (a bank of 8192 plus a window) at four CTAs
  // per SM instead of half-empty 512-thread CTAs at two
  constexpr int NC = 4;
  constexpr int64_t cap[NC] = {128 * kRegItems, 256 * kRegItems, 256 * kWideItems,
                               512 * kRegItems};
  constexpr int64_t c1024 = 1024 * kRegItems;
  if (a.n_seg == 1 && seg <= kWarpSelectMax) {  // short rows: one warp per row
    if (seg <= 32 * 8) return launch_warp_select<8>(a, s, launched);
    if (seg <= 32 * 16) return launch_warp_select<16>(a, s, launched);
    if (seg <= 32 * 32) return launch_warp_select<32>(a, s, launched);
    return launch_warp_select<40>(a, s, launched);
  }
  if (seg > c1024) {
    // whole long rows with K small enough for the gather buffer: the sample-threshold select;
    // segments of split rows and large K: the multi-pass radix select
    if (a.n_seg == 1 && a.K <= kLongCap / 2) return launch_long(a, 0, a.rows, s, launched);
    select_kernel<<<static_cast<unsigned>(grid), kSelThreads, 0, s>>>(a);
    *launched = 1;
    return cudaGetLastError();
  }
  int end[NC];  // rows [end[c-1], end[c]) go to class c, rows from end[NC-1] on to 1024x32
  if (a.len_mode == 1 && a.n_seg == 1 && a.pos_step > 0) {
    // rows of a causal prefix grow with the row index: split the launch by length class
    auto rows_upto = [&](int64_t c) {  // number of leading rows of length <= c
      const int64_t num = c - 1 - a.pos_base;
      if (num < 0) return 0;
      return static_cast<int>(std::min<int64_t>(a.rows, num / a.pos_step + 1));
    };
    for (int c = 0; c < NC; ++c) end[c] = std::max(c ? end[c - 1] : 0, rows_upto(cap[c]));
  } else {
    int first = NC;  // smallest class that holds every row
    for (int c = NC - 1; c >= 0; --c)
      if (seg <= cap[c]) first = c;
    for (int c = 0; c < NC; ++c) end[c] = c >= first ? a.rows : 0;
  }
  cudaError_t e;
  if ((e = launch_reg<128, 10>(a, 0, end[0], s, launched)) != cudaSuccess) return e;
  if ((e = launch_reg<256, 11>(a, end[0], end[1], s, launched)) != cudaSuccess) return e;
  if ((e = launch_reg<256, 11, kWideItems>(a, end[1], end[2], s, launched)) != cudaSuccess)
    return e;
  if ((e = launch_reg<512, 12>(a, end[2], end[3], s, launched)) != cudaSuccess) return e;
  return launch_reg<1024, 12>(a, end[3], a.rows, s, launched);
}

}  // namespace adx

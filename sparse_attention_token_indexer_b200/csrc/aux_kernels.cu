// Small memory-bound helpers of the indexer path:
//  * candidate packing: gather each group's candidate key rows (and scales, positions) into
//    a contiguous block so that refinement streams them with tiled TMA loads
//    (ADIndex, arXiv 2611.12956v1, §4.3 Eq. (14): C_i = bank U post-anchor positions);
//  * query preparation: gate folding for rows with non-negative gates
//    (w * ReLU(x) = ReLU(w * x)), so the scoring epilogue needs no gate loads for them, and
//    e4m3 (re)quantisation;
//  * post-anchor columns of a bank: the positions every member of a group adds to the
//    shared bank (Eq. (14)), stored beside the bank so refinement needs no extra inputs.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <cstdint>

#include "adx_internal.h"
#include "sm100_ptx.cuh"

namespace adx {

namespace {

// One thread per 16-byte piece of a packed candidate row.
__global__ void pack_kernel(const uint8_t* __restrict__ k, const float* __restrict__ k_scale,
                            int64_t key_batch_stride, int32_t per_group_keys, int32_t group_div,
                            int32_t S_valid,
                            const int32_t* __restrict__ cand, int32_t n_groups, int32_t n_cand,
                            int32_t n_cand_pad, int32_t row_bytes, uint8_t* __restrict__ packed,
                            float* __restrict__ packed_scale, int32_t* __restrict__ packed_pos) {
  const int pieces = row_bytes / 16;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(n_groups) * n_cand_pad * pieces;
  if (gid >= total) return;
  const int piece = static_cast<int>(gid % pieces);
  const int64_t slot = gid / pieces;  // g * n_cand_pad + c
  const int g = static_cast<int>(slot / n_cand_pad);
  const int c = static_cast<int>(slot % n_cand_pad);
  const int32_t p = c < n_cand ? cand[static_cast<int64_t>(g) * n_cand + c] : -1;
  const bool valid = p >= 0 && p < S_valid;
  const int64_t krow =
      (per_group_keys ? static_cast<int64_t>(g / group_div) * key_batch_stride : 0) + p;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (valid) v = reinterpret_cast<const uint4*>(k + krow * row_bytes)[piece];
  reinterpret_cast<uint4*>(packed + slot * row_bytes)[piece] = v;
  if (piece == 0) {
    if (packed_pos) packed_pos[slot] = valid ? p : INT32_MAX;
    if (packed_scale) packed_scale[slot] = (valid && k_scale) ? k_scale[krow] : 0.f;
  }
}

// Post-anchor slots of packed decode banks: slot c in [first, width) of row t holds the key at
// position bank[t, c] of cache t; the slots at or before the row's position seq_len[t] - 1 are
// copied from the cache (one thread per 16 bytes of a slot).
__global__ void refresh_post_kernel(const uint8_t* __restrict__ k, const float* __restrict__ k_scale,
                                    int64_t S, const int32_t* __restrict__ seq_len,
                                    const int32_t* __restrict__ bank, int32_t rows, int32_t width,
                                    int32_t first, int32_t row_bytes, uint8_t* __restrict__ packed,
                                    float* __restrict__ packed_scale) {
  const int pieces = row_bytes / 16;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t per_row = static_cast<int64_t>(width - first) * pieces;
  if (gid >= rows * per_row) return;
  const int t = static_cast<int>(gid / per_row);
  const int c = first + static_cast<int>((gid % per_row) / pieces);
  const int piece = static_cast<int>(gid % pieces);
  const int64_t slot = static_cast<int64_t>(t) * width + c;
  const int32_t p = bank[slot];
  if (p < 0 || p >= S || p > seq_len[t] - 1) return;
  const int64_t krow = static_cast<int64_t>(t) * S + p;
  reinterpret_cast<uint4*>(packed + slot * row_bytes)[piece] =
      reinterpret_cast<const uint4*>(k + krow * row_bytes)[piece];
  if (piece == 0 && packed_scale) packed_scale[slot] = k_scale ? k_scale[krow] : 0.f;
}

// MTP window positions: query j of sequence b at seq_len[b] - m + j; group g's anchor (its
// first query) at seq_len[b] - m + g*G.
__global__ void mtp_positions_kernel(const int32_t* __restrict__ seq_len, int32_t Bs, int32_t m,
                                     int32_t G, int32_t* __restrict__ row_pos_q,
                                     int32_t* __restrict__ row_pos_g) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(Bs) * m) return;
  const int b = static_cast<int>(i / m), j = static_cast<int>(i % m);
  const int32_t p = seq_len[b] - m + j;
  row_pos_q[i] = p;
  if (j % G == 0) row_pos_g[static_cast<int64_t>(b) * (m / G) + j / G] = p;
}

// One thread per (group, column) of the MTP candidate rows.
__global__ void mtp_candidates_kernel(int32_t* __restrict__ cand, int32_t n_groups, int32_t width,
                                      int32_t P, int32_t G, int32_t m,
                                      const int32_t* __restrict__ seq_len,
                                      const int32_t* __restrict__ anchor_pos) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(n_groups) * width) return;
  const int g = static_cast<int>(i / width), c = static_cast<int>(i % width);
  const int b = g / (m / G);
  const int32_t first_visible = seq_len[b] - m + 1;  // keys the window's first query sees
  const int32_t a = anchor_pos[g];
  int32_t v;
  if (first_visible <= P) {
    v = c < a + G ? c : -1;  // plain indexer: every position up to the last member's
  } else if (c < P) {
    return;  // the bank
  } else {
    v = c < P + G - 1 ? a + 1 + (c - P) : -1;  // post-anchor positions, then padding
  }
  cand[i] = v;
}

// Failure-detection check: one thread waits, with the indexer kernels' bounded wait, on an
// mbarrier that nothing completes, and records the timeout in the status word as they do.
__global__ void wait_timeout_kernel(DeviceStatus* status, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag, timeout_ns) &&
      atomicCAS(&status->code, 0, 6 /* ADX_ETIMEOUT */) == 0) {
    status->where = kWhereCheck;
    status->info0 = 0;
    status->info1 = 0;
  }
}

// Union size of the Top-K sets of one group of G consecutive rows: a bitmap of the S
// positions in shared memory, one bit set per index, then a population count.
__global__ void __launch_bounds__(256)
union_sizes_kernel(const int32_t* __restrict__ topk, int32_t K, int32_t G, int32_t S,
                   int32_t* __restrict__ out) {
  extern __shared__ uint32_t bits[];
  __shared__ uint32_t red[8];
  const int nw = (S + 31) / 32;
  for (int i = threadIdx.x; i < nw; i += blockDim.x) bits[i] = 0u;
  __syncthreads();
  const int32_t* rows = topk + static_cast<int64_t>(blockIdx.x) * G * K;
  for (int i = threadIdx.x; i < G * K; i += blockDim.x) {
    const int32_t v = rows[i];
    if (v >= 0 && v < S) atomicOr(&bits[v >> 5], 1u << (v & 31));
  }
  __syncthreads();
  uint32_t c = 0;
  for (int i = threadIdx.x; i < nw; i += blockDim.x) c += __popc(bits[i]);
  c = __reduce_add_sync(0xffffffffu, c);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t t = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x / 32); ++w) t += red[w];
    out[blockIdx.x] = static_cast<int32_t>(t);
  }
}

// Shared-bank coverage, one CTA per complete group: the group's bank row is marked in a
// shared-memory bitmap of the S positions, then each warp takes one member row at a time and
// counts its Top-K positions (entries >= 0) and how many of them the bitmap holds.
__global__ void __launch_bounds__(256)
bank_coverage_kernel(const int32_t* __restrict__ topk, int32_t K,
                     const int32_t* __restrict__ bank, int32_t bank_w, int32_t G, int32_t S,
                     int32_t* __restrict__ hits, int32_t* __restrict__ count) {
  extern __shared__ uint32_t bits[];
  const int nw = (S + 31) / 32;
  for (int i = threadIdx.x; i < nw; i += blockDim.x) bits[i] = 0u;
  __syncthreads();
  const int32_t* brow = bank + static_cast<int64_t>(blockIdx.x) * bank_w;
  for (int i = threadIdx.x; i < bank_w; i += blockDim.x) {
    const int32_t v = brow[i];
    if (v >= 0 && v < S) atomicOr(&bits[v >> 5], 1u << (v & 31));
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = static_cast<int>(blockDim.x >> 5);
  for (int m = warp; m < G; m += nwarps) {
    const int64_t r = static_cast<int64_t>(blockIdx.x) * G + m;
    const int32_t* row = topk + r * K;
    uint32_t h = 0, c = 0;
    for (int j = lane; j < K; j += 32) {
      const int32_t v = row[j];
      if (v >= 0) {
        ++c;
        if (v < S && ((bits[v >> 5] >> (v & 31)) & 1u)) ++h;
      }
    }
    h = __reduce_add_sync(0xffffffffu, h);
    c = __reduce_add_sync(0xffffffffu, c);
    if (lane == 0) {
      hits[r] = static_cast<int32_t>(h);
      count[r] = static_cast<int32_t>(c);
    }
  }
}

__global__ void fill_post_kernel(int32_t* bank, int32_t n_groups, int32_t bank_w, int32_t first_col,
                                 int32_t count, int64_t pos_base, int32_t pos_step,
                                 const int32_t* seq_len, int32_t start_off) {
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= static_cast<int64_t>(n_groups) * count) return;
  const int g = static_cast<int>(gid / count);
  const int j = static_cast<int>(gid % count);
  const int64_t anchor =
      seq_len ? static_cast<int64_t>(seq_len[g]) - 1 : pos_base + static_cast<int64_t>(g) * pos_step;
  bank[static_cast<int64_t>(g) * bank_w + first_col + j] = static_cast<int32_t>(anchor + start_off + j);
}

// Query preparation for the scoring kernel, one CTA per query row. A row whose gates are all
// >= 0 is stored gate-folded, w[r, j] * q[r, j, :], because w * ReLU(q . k) = ReLU((w q) . k)
// for w >= 0; the scoring epilogue then needs no gates for it. Any other row is stored as
// given. fold_flag[r] = 1 marks a folded row. Output codes are bf16 (bf16 input) or e4m3 with
// a new per-row scale (e4m3 input, or bf16 input quantised for an e4m3 key cache).
template <bool IN_E4M3>
__device__ __forceinline__ void load8(const void* q, int64_t e, float sin, float (&x)[8]) {
  if constexpr (IN_E4M3) {
    const uint2 v = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(q) + e);
    const __nv_fp8_e4m3* c = reinterpret_cast<const __nv_fp8_e4m3*>(&v);
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = static_cast<float>(c[u]) * sin;
  } else {
    const uint4 v = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(q) + e);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(h[u]);
      x[2 * u] = f.x;
      x[2 * u + 1] = f.y;
    }
  }
}

// THREADS threads per row; each thread holds up to G = 1024 / THREADS groups of 8 elements
// in registers (rows of up to 8192 elements), so the row is read once and every load of a
// thread is in flight together.
template <bool IN_E4M3, bool OUT_E4M3, int THREADS>
__global__ void __launch_bounds__(THREADS)
prepare_q_kernel(const void* __restrict__ q_in, const float* __restrict__ q_scale_in,
                 const float* __restrict__ w, int H, int d, void* __restrict__ q_out,
                 float* __restrict__ q_scale_out, int8_t* __restrict__ fold_flag,
                 RowBlocks rb) {
  constexpr int G = 1024 / THREADS;
  __shared__ float red[THREADS / 32];
  const int64_t r = blockIdx.x;
  if (rb.out != nullptr && threadIdx.x == 0) {
    const int64_t p = rb.seq_len != nullptr ? static_cast<int64_t>(rb.seq_len[r]) - 1 : rb.q_pos0 + r;
    rb.out[r] = static_cast<int32_t>(p < 0 ? -1 : p / kTileM);
  }
  const float* wr = w + r * H;
  const int ng = H * d / 8;  // groups of 8 elements; a group lies within one head
  const int64_t base = r * static_cast<int64_t>(H) * d;
  const float sin = IN_E4M3 ? q_scale_in[r] : 1.f;
  float x[G][8], g[G];
  int neg = 0;
#pragma unroll
  for (int k = 0; k < G; ++k) {
    const int i = threadIdx.x + k * THREADS;
    g[k] = 1.f;
    if (i < ng) {
      load8<IN_E4M3>(q_in, base + static_cast<int64_t>(i) * 8, sin, x[k]);
      g[k] = wr[(i * 8) / d];
      neg |= g[k] < 0.f;
    }
  }
  // every head has d/8 groups, so the threads together have seen every gate of the row
  const bool fold = __syncthreads_or(neg) == 0;
  if (threadIdx.x == 0) fold_flag[r] = fold ? 1 : 0;
  if constexpr (IN_E4M3 && OUT_E4M3) {
    if (!fold) {  // keep the given codes and scale
      const uint2* in = reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(q_in) + base);
      uint2* out = reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(q_out) + base);
      for (int i = threadIdx.x; i < ng; i += THREADS) out[i] = in[i];
      if (threadIdx.x == 0) q_scale_out[r] = sin;
      return;
    }
  }
  if (!fold) {
#pragma unroll
    for (int k = 0; k < G; ++k) g[k] = 1.f;
  }
  float sc = 1.f;
  if constexpr (OUT_E4M3) {
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < G; ++k)
      if (threadIdx.x + k * THREADS < ng)
#pragma unroll
        for (int u = 0; u < 8; ++u) amax = fmaxf(amax, fabsf(x[k][u] * g[k]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    float m = 0.f;
#pragma unroll
    for (int i2 = 0; i2 < THREADS / 32; ++i2) m = fmaxf(m, red[i2]);
    sc = m > 0.f ? m / 448.f : 1.f;
    if (threadIdx.x == 0) q_scale_out[r] = sc;
  }
#pragma unroll
  for (int k = 0; k < G; ++k) {
    const int i = threadIdx.x + k * THREADS;
    if (i >= ng) continue;
    if constexpr (OUT_E4M3) {
      uint2 v;
      uint8_t* c = reinterpret_cast<uint8_t*>(&v);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        c[u] = static_cast<uint8_t>(
            __nv_cvt_float_to_fp8((x[k][u] * g[k]) / sc, __NV_SATFINITE, __NV_E4M3));
      reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(q_out) + base)[i] = v;
    } else {
      uint4 v;
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        h[u] = __floats2bfloat162_rn(x[k][2 * u] * g[k], x[k][2 * u + 1] * g[k]);
      reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(q_out) + base)[i] = v;
    }
  }
}

// Mean-pooled group query, one CTA per group of G consecutive rows: each thread owns 8
// consecutive elements of the first Hg heads and sums them over the members in fp32.
template <bool IN_E4M3>
__global__ void __launch_bounds__(256)
group_mean_kernel(const void* __restrict__ q, const float* __restrict__ q_scale,
                  const float* __restrict__ w, int H, int d, int G, int Hg,
                  __nv_bfloat16* __restrict__ qbar, float* __restrict__ wbar) {
  const int64_t g = blockIdx.x;
  const int n8 = Hg * d / 8;
  const float inv = 1.f / static_cast<float>(G);
  for (int e = threadIdx.x; e < n8; e += blockDim.x) {
    const int j = (e * 8) / d, c = (e * 8) % d;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < G; ++i) {
      const int64_t r = g * G + i;
      float x[8];
      load8<IN_E4M3>(q, (r * H + j) * d + c, IN_E4M3 ? q_scale[r] : 1.f, x);
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[u] += x[u];
    }
    uint4 v;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int u = 0; u < 4; ++u) h[u] = __floats2bfloat162_rn(acc[2 * u] * inv, acc[2 * u + 1] * inv);
    reinterpret_cast<uint4*>(qbar + (g * Hg + j) * d + c)[0] = v;
  }
  for (int j = threadIdx.x; j < Hg; j += blockDim.x) {
    float a = 0.f;
    for (int i = 0; i < G; ++i) a += w[(g * G + i) * H + j];
    wbar[g * Hg + j] = a * inv;
  }
}

template <bool IN_E4M3, bool OUT_E4M3>
cudaError_t launch_prepare_rows(const void* q, const float* q_scale, const float* w, int64_t rows,
                                int H, int d, void* q_out, float* q_scale_out, int8_t* fold_flag,
                                RowBlocks rb, cudaStream_t s) {
  // few rows (decode): spread each row over more threads
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaErrorUnknown;
  const unsigned g = static_cast<unsigned>(rows);
  if (rows < 2ll * sms)
    prepare_q_kernel<IN_E4M3, OUT_E4M3, 1024>
        <<<g, 1024, 0, s>>>(q, q_scale, w, H, d, q_out, q_scale_out, fold_flag, rb);
  else
    prepare_q_kernel<IN_E4M3, OUT_E4M3, 256>
        <<<g, 256, 0, s>>>(q, q_scale, w, H, d, q_out, q_scale_out, fold_flag, rb);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prepare_q(const void* q, const float* q_scale, bool in_e4m3, bool out_e4m3,
                             const float* w, int64_t rows, int H, int d, void* q_out,
                             float* q_scale_out, int8_t* fold_flag, cudaStream_t s, RowBlocks rb) {
  if (rows <= 0) return cudaSuccess;
  if (static_cast<int64_t>(H) * d > 8192 || d % 8 != 0) return cudaErrorNotSupported;
  if (!in_e4m3 && !out_e4m3)
    return launch_prepare_rows<false, false>(q, q_scale, w, rows, H, d, q_out, q_scale_out,
                                             fold_flag, rb, s);
  if (in_e4m3 && out_e4m3)
    return launch_prepare_rows<true, true>(q, q_scale, w, rows, H, d, q_out, q_scale_out,
                                           fold_flag, rb, s);
  if (!in_e4m3 && out_e4m3)
    return launch_prepare_rows<false, true>(q, q_scale, w, rows, H, d, q_out, q_scale_out,
                                            fold_flag, rb, s);
  return launch_prepare_rows<true, false>(q, q_scale, w, rows, H, d, q_out, q_scale_out,
                                          fold_flag, rb, s);
}

cudaError_t launch_pack_candidates(const void* k, const float* k_scale, int64_t key_batch_stride,
                                   int32_t per_group_keys, int32_t group_div, int32_t S_valid,
                                   const int32_t* cand,
                                   int32_t n_groups, int32_t n_cand, int32_t n_cand_pad,
                                   int32_t row_bytes, void* packed, float* packed_scale,
                                   int32_t* packed_pos, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(n_groups) * n_cand_pad * (row_bytes / 16);
  if (total <= 0) return cudaSuccess;
  const int threads = 256;
  pack_kernel<<<static_cast<unsigned>((total + threads - 1) / threads), threads, 0, s>>>(
      static_cast<const uint8_t*>(k), k_scale, key_batch_stride, per_group_keys,
      group_div > 1 ? group_div : 1, S_valid, cand,
      n_groups, n_cand, n_cand_pad, row_bytes, static_cast<uint8_t*>(packed), packed_scale,
      packed_pos);
  return cudaGetLastError();
}

cudaError_t launch_mtp_positions(const int32_t* seq_len, int32_t Bs, int32_t m, int32_t G,
                                 int32_t* row_pos_q, int32_t* row_pos_g, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(Bs) * m;
  if (total <= 0) return cudaSuccess;
  mtp_positions_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(
      seq_len, Bs, m, G, row_pos_q, row_pos_g);
  return cudaGetLastError();
}

cudaError_t launch_mtp_candidates(int32_t* cand, int32_t n_groups, int32_t width, int32_t P,
                                  int32_t G, int32_t m, const int32_t* seq_len,
                                  const int32_t* anchor_pos, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(n_groups) * width;
  if (total <= 0) return cudaSuccess;
  mtp_candidates_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(
      cand, n_groups, width, P, G, m, seq_len, anchor_pos);
  return cudaGetLastError();
}

cudaError_t launch_group_mean(const void* q, const float* q_scale, bool in_e4m3, const float* w,
                              int64_t n_groups, int H, int d, int G, int Hg, void* qbar,
                              float* wbar, cudaStream_t s) {
  if (n_groups <= 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>(n_groups);
  __nv_bfloat16* qb = static_cast<__nv_bfloat16*>(qbar);
  if (in_e4m3)
    group_mean_kernel<true><<<grid, 256, 0, s>>>(q, q_scale, w, H, d, G, Hg, qb, wbar);
  else
    group_mean_kernel<false><<<grid, 256, 0, s>>>(q, q_scale, w, H, d, G, Hg, qb, wbar);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout(DeviceStatus* status, uint64_t timeout_ns, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

cudaError_t launch_union_sizes(const int32_t* topk, int32_t K, int32_t G, int32_t S,
                               int32_t n_groups, int32_t* out, cudaStream_t s) {
  if (n_groups <= 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>((S + 31) / 32) * 4;
  if (smem > kUnionMaxBitmapBytes) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(
        union_sizes_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  union_sizes_kernel<<<static_cast<unsigned>(n_groups), 256, smem, s>>>(topk, K, G, S, out);
  return cudaGetLastError();
}

cudaError_t launch_bank_coverage(const int32_t* topk, int32_t K, const int32_t* bank,
                                 int32_t bank_w, int32_t G, int32_t S, int32_t n_groups,
                                 int32_t* hits, int32_t* count, cudaStream_t s) {
  if (n_groups <= 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>((S + 31) / 32) * 4;
  if (smem > kUnionMaxBitmapBytes) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(
        bank_coverage_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  bank_coverage_kernel<<<static_cast<unsigned>(n_groups), 256, smem, s>>>(topk, K, bank, bank_w,
                                                                         G, S, hits, count);
  return cudaGetLastError();
}

cudaError_t launch_refresh_post(const void* k, const float* k_scale, int64_t S,
                                const int32_t* seq_len, const int32_t* bank, int32_t rows,
                                int32_t width, int32_t first, int32_t row_bytes, void* packed,
                                float* packed_scale, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(rows) * (width - first) * (row_bytes / 16);
  if (total <= 0) return cudaSuccess;
  refresh_post_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(
      static_cast<const uint8_t*>(k), k_scale, S, seq_len, bank, rows, width, first, row_bytes,
      static_cast<uint8_t*>(packed), packed_scale);
  return cudaGetLastError();
}

cudaError_t launch_fill_post_anchor(int32_t* bank, int32_t n_groups, int32_t bank_w,
                                    int32_t first_col, int32_t count, int64_t pos_base,
                                    int32_t pos_step, const int32_t* seq_len, int32_t start_off,
                                    cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(n_groups) * count;
  if (total <= 0) return cudaSuccess;
  fill_post_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(
      bank, n_groups, bank_w, first_col, count, pos_base, pos_step, seq_len, start_off);
  return cudaGetLastError();
}

}  // namespace adx

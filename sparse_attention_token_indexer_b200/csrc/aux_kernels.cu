// Small memory-bound helpers of the indexer path:
//  * per-token FP8-e4m3 quantisation of bf16 queries (decode with an e4m3 key cache);
//  * candidate packing: gather each group's candidate key rows (and scales, positions) into
//    a contiguous block so that refinement streams them with tiled TMA loads
//    (ADIndex, arXiv 2611.12956v1, §4.3 Eq. (14): C_i = bank U post-anchor positions);
//  * gate folding for bf16 queries with non-negative gates (w * ReLU(x) = ReLU(w * x)), so
//    the scoring epilogue needs no gate loads;
//  * post-anchor columns of a bank: the positions every member of a group adds to the
//    shared bank (Eq. (14)), stored beside the bank so refinement needs no extra inputs.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <cstdint>

#include "adx_internal.h"

namespace adx {

namespace {

constexpr int kQuantThreads = 256;

__global__ void __launch_bounds__(kQuantThreads)
quantize_rows_kernel(const __nv_bfloat16* __restrict__ x, int64_t cols, uint8_t* __restrict__ codes,
                     float* __restrict__ scale) {
  __shared__ float red[kQuantThreads / 32];
  const int64_t row = blockIdx.x;
  const __nv_bfloat16* xr = x + row * cols;
  float amax = 0.f;
  for (int64_t i = threadIdx.x; i < cols; i += kQuantThreads)
    amax = fmaxf(amax, fabsf(__bfloat162float(xr[i])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < kQuantThreads / 32 ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float m = red[0];
  const float s = m > 0.f ? m / 448.f : 1.f;
  if (threadIdx.x == 0) scale[row] = s;
  uint8_t* cr = codes + row * cols;
  for (int64_t i = threadIdx.x; i < cols; i += kQuantThreads) {
    const float y = __bfloat162float(xr[i]) / s;
    cr[i] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3));
  }
}

// One thread per 16-byte piece of a packed candidate row.
__global__ void pack_kernel(const uint8_t* __restrict__ k, const float* __restrict__ k_scale,
                            int64_t key_batch_stride, int32_t per_group_keys, int32_t S_valid,
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
  const int64_t krow = (per_group_keys ? static_cast<int64_t>(g) * key_batch_stride : 0) + p;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (valid) v = reinterpret_cast<const uint4*>(k + krow * row_bytes)[piece];
  reinterpret_cast<uint4*>(packed + slot * row_bytes)[piece] = v;
  if (piece == 0) {
    packed_pos[slot] = valid ? p : INT32_MAX;
    if (packed_scale) packed_scale[slot] = (valid && k_scale) ? k_scale[krow] : 0.f;
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

// q'[r, j, :] = bf16(w[r, j] * q[r, j, :]) for rows whose gates are all >= 0, where
// w * ReLU(q . k) = ReLU((w q) . k); neg_row[r] = 1 marks rows with a negative gate (their
// folded copy is not used).
__global__ void __launch_bounds__(256)
fold_gates_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w, int H, int d,
                  __nv_bfloat16* __restrict__ qf, int8_t* __restrict__ neg_row) {
  const int64_t r = blockIdx.x;
  const float* wr = w + r * H;
  int neg = 0;
  for (int j = threadIdx.x; j < H; j += blockDim.x) neg |= wr[j] < 0.f;
  neg = __syncthreads_or(neg);
  if (threadIdx.x == 0) neg_row[r] = static_cast<int8_t>(neg != 0);
  if (neg) return;
  const int64_t n = static_cast<int64_t>(H) * d;
  const uint4* src = reinterpret_cast<const uint4*>(q + r * n);
  uint4* dst = reinterpret_cast<uint4*>(qf + r * n);
  for (int64_t i = threadIdx.x; i < n / 8; i += blockDim.x) {
    const float g = wr[(i * 8) / d];
    uint4 v = src[i];
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(h[u]);
      h[u] = __floats2bfloat162_rn(f.x * g, f.y * g);
    }
    dst[i] = v;
  }
}

}  // namespace

cudaError_t launch_fold_gates_bf16(const uint16_t* q, const float* w, int64_t rows, int H, int d,
                                   uint16_t* qf, int8_t* neg_row, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  fold_gates_kernel<<<static_cast<unsigned>(rows), 256, 0, s>>>(
      reinterpret_cast<const __nv_bfloat16*>(q), w, H, d, reinterpret_cast<__nv_bfloat16*>(qf),
      neg_row);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows_e4m3(const uint16_t* x_bf16, int64_t rows, int64_t cols,
                                      uint8_t* codes, float* scale, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  quantize_rows_kernel<<<static_cast<unsigned>(rows), kQuantThreads, 0, s>>>(
      reinterpret_cast<const __nv_bfloat16*>(x_bf16), cols, codes, scale);
  return cudaGetLastError();
}

cudaError_t launch_pack_candidates(const void* k, const float* k_scale, int64_t key_batch_stride,
                                   int32_t per_group_keys, int32_t S_valid, const int32_t* cand,
                                   int32_t n_groups, int32_t n_cand, int32_t n_cand_pad,
                                   int32_t row_bytes, void* packed, float* packed_scale,
                                   int32_t* packed_pos, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(n_groups) * n_cand_pad * (row_bytes / 16);
  if (total <= 0) return cudaSuccess;
  const int threads = 256;
  pack_kernel<<<static_cast<unsigned>((total + threads - 1) / threads), threads, 0, s>>>(
      static_cast<const uint8_t*>(k), k_scale, key_batch_stride, per_group_keys, S_valid, cand,
      n_groups, n_cand, n_cand_pad, row_bytes, static_cast<uint8_t*>(packed), packed_scale,
      packed_pos);
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

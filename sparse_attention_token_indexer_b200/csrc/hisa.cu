// Kernels of the hierarchical (block, then token) indexer of "HISA: Efficient Hierarchical
// Indexing for Fine-Grained Sparse Attention" (arXiv 2603.28458v3), with the settings the
// ADIndex paper uses for it (Appendix C.5): 128-key blocks pooled by their mean, the first
// block and the query's own block always among the candidates.
//   * block keys: the mean of each block of 128 keys (decoded with their scales for e4m3),
//     stored in bf16 for either key format, so block scores carry no FP8 rounding of their
//     own (the block pass scores them against bf16 queries);
//   * forcing: the two forced blocks' scores raised to +inf ahead of the block Top-n (for
//     block rows longer than the one-warp select holds; that select forces them itself).
// The block of each row's position is a by-product of the query preparation.
// The block scores, both selections and the token refinement run on the scoring and select
// kernels (the refinement in their block-list mode).
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "adx_internal.h"

namespace adx {
namespace {

constexpr int kBlk = kTileM;  // keys per block: one MMA tile
constexpr int kBkThreads = 256;

// One CTA per (block, key range). Threads are (row group, column); row group g sums the rows
// g, g + RG, ... of the block in fp32, then the groups are added in shared memory.
template <bool FP8>
__global__ void __launch_bounds__(kBkThreads)
block_keys_kernel(const uint8_t* __restrict__ k, const float* __restrict__ k_scale, int64_t S,
                  int d, const int32_t* __restrict__ seq_len, int32_t len_fixed, int last_only,
                  int nbmax, uint8_t* __restrict__ kbar) {
  __shared__ float part[kBkThreads];
  const int64_t b = blockIdx.y;
  int64_t len = seq_len != nullptr ? seq_len[b] : len_fixed;
  len = len < S ? len : S;
  if (len <= 0) return;
  const int64_t blk = last_only ? (len - 1) / kBlk : blockIdx.x;
  const int64_t r0 = blk * kBlk;
  if (r0 >= len || blk >= nbmax) return;
  const int n = static_cast<int>(len - r0 < kBlk ? len - r0 : kBlk);
  const int RG = kBkThreads / d;  // d divides kBkThreads (d = 64 or 128)
  const int g = threadIdx.x / d, e = threadIdx.x % d;
  const int64_t row0 = b * S + r0;
  float acc = 0.f;
  for (int i = g; i < n; i += RG) {
    const int64_t row = row0 + i;
    if constexpr (FP8) {
      const __nv_fp8_e4m3 c = reinterpret_cast<const __nv_fp8_e4m3*>(k)[row * d + e];
      acc += static_cast<float>(c) * k_scale[row];
    } else {
      acc += __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(k)[row * d + e]);
    }
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  float mean = 0.f;
  if (threadIdx.x < d) {
    float s = 0.f;
    for (int gg = 0; gg < RG; ++gg) s += part[gg * d + threadIdx.x];
    mean = s / static_cast<float>(n);
  }
  const int64_t out = b * nbmax + blk;
  if (threadIdx.x < d)
    reinterpret_cast<__nv_bfloat16*>(kbar)[out * d + threadIdx.x] = __float2bfloat16_rn(mean);
}

// Forced blocks: where more than n_blocks blocks are visible, block 0 and the row's own block
// take +inf so that the block Top-n keeps them and fills the other slots by score.
__global__ void force_blocks_kernel(float* __restrict__ scores, int64_t ld, int32_t R,
                                    const int32_t* __restrict__ row_blk, int32_t n_blocks) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= R) return;
  const int32_t cur = row_blk[r];
  if (cur + 1 <= n_blocks) return;
  scores[r * ld] = INFINITY;
  scores[r * ld + cur] = INFINITY;
}

// Union of the block lists of `tok` consecutive rows (one CTA per group, one thread per list
// entry, P = the entry count rounded up to a power of two): the entries, keyed
// (block, row, slot), are sorted (bitonic, in shared memory); the first entry of each block
// number gives it its union position, and every entry records its slot in its row's list
// as byte `row` of the union position's slot word (0xFF where a row lacks the block).
__global__ void block_union_kernel(const int32_t* __restrict__ blocks, int32_t n_blocks,
                                   int32_t R, int32_t tok, int32_t stride,
                                   int32_t* __restrict__ uni, int32_t* __restrict__ slot,
                                   int32_t* __restrict__ count) {
  extern __shared__ uint64_t key_s[];  // [P] keys, then [stride] slot words
  const int P = blockDim.x;
  uint32_t* slot_s = reinterpret_cast<uint32_t*>(key_s + P);
  __shared__ int warp_n[32];
  const int64_t g = blockIdx.x;
  const int i = threadIdx.x;
  const int row = i / n_blocks, j = i % n_blocks;
  const int64_t r = g * tok + row;
  int32_t v = -1;
  if (i < tok * n_blocks && r < R) v = blocks[r * n_blocks + j];
  key_s[i] = v >= 0 ? (static_cast<uint64_t>(v) << 16) | (static_cast<uint64_t>(row) << 8) |
                          static_cast<uint64_t>(j)
                    : ~0ull;
  for (int u = i; u < stride; u += P) slot_s[u] = 0xFFFFFFFFu;
  __syncthreads();
  for (int k = 2; k <= P; k <<= 1) {
    for (int h = k >> 1; h > 0; h >>= 1) {
      const int o = i ^ h;
      if (o > i) {
        const uint64_t a = key_s[i], b = key_s[o];
        if (((i & k) == 0) == (a > b)) {
          key_s[i] = b;
          key_s[o] = a;
        }
      }
      __syncthreads();
    }
  }
  const uint64_t kk = key_s[i];
  const bool valid = kk != ~0ull;
  const bool first = valid && (i == 0 || (key_s[i - 1] >> 16) != (kk >> 16));
  // union position = number of first entries at or before i, minus one
  const unsigned bal = __ballot_sync(0xffffffffu, first);
  const int lane = i & 31, wid = i >> 5;
  if (lane == 31) warp_n[wid] = __popc(bal);
  __syncthreads();
  int before = 0, total = 0;
  for (int w = 0; w < P / 32; ++w) {
    if (w < wid) before += warp_n[w];
    total += warp_n[w];
  }
  const int u = before + __popc(bal & ((2u << lane) - 1u)) - 1;
  if (valid) {
    const int rr = static_cast<int>((kk >> 8) & 0xFF), jj = static_cast<int>(kk & 0xFF);
    reinterpret_cast<uint8_t*>(slot_s)[u * 4 + rr] = static_cast<uint8_t>(jj);
    if (first) uni[g * stride + u] = static_cast<int32_t>(kk >> 16);
  }
  __syncthreads();
  for (int q = i; q < total; q += P) slot[g * stride + q] = static_cast<int32_t>(slot_s[q]);
  if (i == 0) count[g] = total;
}

}  // namespace

cudaError_t launch_block_union(const int32_t* blocks, int32_t n_blocks, int32_t R, int32_t tok,
                               int32_t* uni, int32_t* slot, int32_t* count, cudaStream_t s) {
  if (R <= 0) return cudaSuccess;
  const int n = tok * n_blocks;
  if (tok < 1 || tok > 4 || n_blocks < 1 || n_blocks > 255 || n > 1024)
    return cudaErrorInvalidValue;
  int P = 32;
  while (P < n) P <<= 1;
  const int stride = n;
  const size_t smem = static_cast<size_t>(P) * 8 + static_cast<size_t>(stride) * 4;
  const int groups = (R + tok - 1) / tok;
  block_union_kernel<<<static_cast<unsigned>(groups), P, smem, s>>>(blocks, n_blocks, R, tok,
                                                                     stride, uni, slot, count);
  return cudaGetLastError();
}

cudaError_t launch_block_keys(const void* k, const float* k_scale, bool fp8, int64_t S, int d,
                              int32_t n_seq, const int32_t* seq_len, int32_t len_fixed,
                              bool last_only, int32_t nbmax, void* kbar, cudaStream_t s) {
  if (n_seq <= 0 || nbmax <= 0) return cudaSuccess;
  if (kBkThreads % d != 0) return cudaErrorInvalidValue;
  const dim3 grid(last_only ? 1 : nbmax, n_seq);
  const uint8_t* kc = static_cast<const uint8_t*>(k);
  uint8_t* out = static_cast<uint8_t*>(kbar);
  if (fp8)
    block_keys_kernel<true><<<grid, kBkThreads, 0, s>>>(kc, k_scale, S, d, seq_len, len_fixed,
                                                        last_only ? 1 : 0, nbmax, out);
  else
    block_keys_kernel<false><<<grid, kBkThreads, 0, s>>>(kc, k_scale, S, d, seq_len, len_fixed,
                                                         last_only ? 1 : 0, nbmax, out);
  return cudaGetLastError();
}

cudaError_t launch_force_blocks(float* scores, int64_t ld, int32_t R, const int32_t* row_blk,
                                int32_t n_blocks, cudaStream_t s) {
  if (R <= 0) return cudaSuccess;
  force_blocks_kernel<<<static_cast<unsigned>((R + 255) / 256), 256, 0, s>>>(scores, ld, R,
                                                                            row_blk, n_blocks);
  return cudaGetLastError();
}

}  // namespace adx

// The group indexer's queries and gates (ADIndex, arXiv 2611.12956v1, §4.2, Eqs. (6)-(7)):
// for each group of G consecutive tokens with anchor t,
//   c-bar = W_pool [max_i c_i ; min_i c_i ; mean_i c_i]      (query latents, element-wise)
//   h-bar = mean_i h_i                                       (normalized hidden states)
//   q-bar_j = RoPE_t([W_Q c-bar]_j),   w-bar_j = sigmoid([W_G h-bar]_j).
// A pooling kernel (16-byte loads, HBM-bound) builds [max; min; mean] and, from h-bar in fp32,
// the gate projection's partial sums; the two projections (W_pool, W_Q) run on this library's
// tcgen05 GEMM (gemm_sm100.cu: bf16 operands, fp32 accumulation in TMEM); a last kernel
// applies RoPE at the anchor and the sigmoid.
// RoPE rotates the pairs (2i, 2i+1), i < rope_dim/2, by the angle t * base^(-2i/rope_dim)
// (the paper names RoPE at the anchor, not its layout).
#include <cuda_bf16.h>

#include <cstdint>
#include <mutex>

#include "../../include/adx.h"
#include "adx_internal.h"

namespace adx {
namespace {

constexpr size_t kAlignGi = 256;
constexpr uint64_t kGemmTimeoutNs = 2000000000ull;  // 2 s per device-side wait

size_t up(size_t x) { return (x + kAlignGi - 1) / kAlignGi * kAlignGi; }

constexpr int kPoolThreads = 256;
constexpr int kPoolWarps = kPoolThreads / 32;
constexpr int kPoolUnroll = 8;
constexpr int kMaxHeads = 64;   // H_S bound: one shared-memory slot per head and warp
constexpr int kGateBatch = 16;
constexpr int kMaxRopePairs = 256;

union Vec8 {
  uint4 u;
  __nv_bfloat162 h[4];
};

// One thread per 8 consecutive columns of one group: columns [0, d_c) of the query latents
// (max, min and mean, written as bf16) followed by columns [0, d_h) of the hidden states,
// whose fp32 mean goes straight into the gate projection: each CTA writes, per head, its
// partial sum of W_G[j, e] * h-bar[e] over its columns to gpart[g, blockIdx.x, j]; the finish
// kernel adds the partials in a fixed order, so the result is deterministic and h-bar is never
// stored. The G member rows are read with 16-byte loads, kPoolUnroll in flight per thread.
__global__ void __launch_bounds__(kPoolThreads)
gi_pool_kernel(const __nv_bfloat16* __restrict__ cq, const __nv_bfloat16* __restrict__ h,
               const __nv_bfloat16* __restrict__ wg, int G, int dc, int dh, int HS,
               __nv_bfloat16* __restrict__ pooled, float* __restrict__ gpart) {
  __shared__ float red[kMaxHeads][kPoolWarps];
  const int64_t g = blockIdx.y;
  const int v = blockIdx.x * kPoolThreads + threadIdx.x;
  const int vc = dc / 8, vh = dh / 8;
  const bool active = v < vc + vh;
  const bool latent = v < vc;
  const bool hid = active && !latent;
  const int col = latent ? v * 8 : (v - vc) * 8;
  const int ld = latent ? dc : dh;

  float sm[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) sm[e] = 0.f;
  const float inv = 1.f / static_cast<float>(G);
  if (active && latent) {
    // max and min on bf16 pairs (exact: members' own values), the sum in fp32
    const __nv_bfloat16* src = cq + g * G * ld + col;
    Vec8 mx, mn;
    mx.u = mn.u = __ldg(reinterpret_cast<const uint4*>(src));
    for (int i0 = 0; i0 < G; i0 += kPoolUnroll) {
      Vec8 r[kPoolUnroll];
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u)
        if (i0 + u < G)
          r[u].u = __ldg(reinterpret_cast<const uint4*>(src + static_cast<int64_t>(i0 + u) * ld));
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u) {
        if (i0 + u >= G) break;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          mx.h[e] = __hmax2(mx.h[e], r[u].h[e]);
          mn.h[e] = __hmin2(mn.h[e], r[u].h[e]);
          const float2 f = __bfloat1622float2(r[u].h[e]);
          sm[2 * e] += f.x, sm[2 * e + 1] += f.y;
        }
      }
    }
    __nv_bfloat16* row = pooled + g * 3 * dc + col;
    *reinterpret_cast<uint4*>(row) = mx.u;
    *reinterpret_cast<uint4*>(row + dc) = mn.u;
    Vec8 o;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      o.h[e] = __floats2bfloat162_rn(sm[2 * e] * inv, sm[2 * e + 1] * inv);
    *reinterpret_cast<uint4*>(row + 2 * dc) = o.u;
  } else if (hid) {
    const __nv_bfloat16* src = h + g * G * ld + col;
    for (int i0 = 0; i0 < G; i0 += kPoolUnroll) {
      Vec8 r[kPoolUnroll];
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u)
        if (i0 + u < G)
          r[u].u = __ldg(reinterpret_cast<const uint4*>(src + static_cast<int64_t>(i0 + u) * ld));
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u) {
        if (i0 + u >= G) break;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(r[u].h[e]);
          sm[2 * e] += f.x, sm[2 * e + 1] += f.y;
        }
      }
    }
  }
  // gate projection of this CTA's hidden-state columns (zero for latent columns): the W_G
  // entries of kGateBatch heads are loaded together, after the stream
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int e = 0; e < 8; ++e) sm[e] *= inv;
  for (int j0 = 0; j0 < HS; j0 += kGateBatch) {
    Vec8 w[kGateBatch];
#pragma unroll
    for (int u = 0; u < kGateBatch; ++u)
      w[u].u = hid && j0 + u < HS
                   ? __ldg(reinterpret_cast<const uint4*>(wg + static_cast<int64_t>(j0 + u) * dh + col))
                   : make_uint4(0u, 0u, 0u, 0u);
    float acc[kGateBatch];
#pragma unroll
    for (int u = 0; u < kGateBatch; ++u) {
      acc[u] = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(w[u].h[e]);
        acc[u] = fmaf(f.x, sm[2 * e], acc[u]);
        acc[u] = fmaf(f.y, sm[2 * e + 1], acc[u]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < kGateBatch; ++u) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], o);
    if (lane == 0)
#pragma unroll
      for (int u = 0; u < kGateBatch; ++u)
        if (j0 + u < HS) red[j0 + u][warp] = acc[u];
  }
  __syncthreads();
  if (threadIdx.x < HS) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kPoolWarps; ++w) t += red[threadIdx.x][w];
    gpart[(g * gridDim.x + blockIdx.x) * HS + threadIdx.x] = t;
  }
}

// RoPE at the group's anchor and the sigmoid gate. The angle pos * base^(-2i/rope_dim) is
// formed in double (anchors reach 1e5 and more, beyond fp32's resolution of radians), reduced
// to [-pi, pi] in double by subtracting the nearest multiple of 2 pi, and only then handed to
// the fp32 sincos.
__global__ void __launch_bounds__(256)
gi_finish_kernel(const float* __restrict__ qpre, const float* __restrict__ gpart, int nparts,
                 int HS, int d, int rope_dim, double base, int64_t q_pos0, int G,
                 __nv_bfloat16* __restrict__ qbar, float* __restrict__ wbar) {
  __shared__ double inv_freq[kMaxRopePairs];
  const int64_t g = blockIdx.x;
  for (int i = threadIdx.x; i < rope_dim / 2; i += blockDim.x)
    inv_freq[i] = pow(base, -2.0 * i / rope_dim);
  __syncthreads();
  const double pos = static_cast<double>(q_pos0 + g * G);
  const double two_pi = 6.283185307179586, inv_two_pi = 0.15915494309189535;
  const int half = d / 2, pairs = HS * half;
  const float2* src = reinterpret_cast<const float2*>(qpre) + g * pairs;
  __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(qbar) + g * pairs;
#pragma unroll 4
  for (int p = threadIdx.x; p < pairs; p += blockDim.x) {
    const int i = p % half;
    float2 y = src[p];
    if (2 * i < rope_dim) {
      const double a = pos * inv_freq[i];
      float sn, cs;
      sincosf(static_cast<float>(fma(-rint(a * inv_two_pi), two_pi, a)), &sn, &cs);
      y = make_float2(y.x * cs - y.y * sn, y.x * sn + y.y * cs);
    }
    dst[p] = __floats2bfloat162_rn(y.x, y.y);
  }
  for (int j = threadIdx.x; j < HS; j += blockDim.x) {
    float z = 0.f;
    for (int c = 0; c < nparts; ++c) z += gpart[(g * nparts + c) * HS + j];
    wbar[g * HS + j] = 1.f / (1.f + __expf(-z));
  }
}

int pool_ctas(const adx_group_indexer* gi) {
  return (gi->d_c / 8 + gi->d_h / 8 + kPoolThreads - 1) / kPoolThreads;
}

bool gi_valid(const adx_group_indexer* gi, int G) {
  const uintptr_t addr = reinterpret_cast<uintptr_t>(gi ? gi->cq : nullptr) |
                         reinterpret_cast<uintptr_t>(gi ? gi->h : nullptr);
  return gi && gi->cq && gi->h && gi->w_pool && gi->w_q && gi->w_g && G > 0 && gi->T >= G &&
         addr % 16 == 0 && gi->d_c > 0 && gi->d_c % 8 == 0 && gi->d_h > 0 && gi->d_h % 8 == 0 &&
         gi->H_S > 0 && gi->H_S <= kMaxHeads && gi->d > 0 && gi->d % 2 == 0 &&
         gi->T / G <= 65535 && reinterpret_cast<uintptr_t>(gi->w_g) % 16 == 0 &&
         gi->rope_dim >= 0 && gi->rope_dim % 2 == 0 && gi->rope_dim <= gi->d &&
         gi->rope_dim / 2 <= kMaxRopePairs &&
         gi->rope_base > 0.f && gi->q_pos0 >= 0;
}

size_t gi_workspace(const adx_group_indexer* gi, int G) {
  const size_t ng = gi->T / G;
  return kStatusBytes + up(ng * 3 * gi->d_c * 2) + up(ng * pool_ctas(gi) * gi->H_S * 4) +
         up(ng * gi->d_c * 2) + up(ng * gi->H_S * gi->d * 4);
}

}  // namespace
}  // namespace adx

using namespace adx;

extern "C" {

size_t adx_group_indexer_workspace_size(const adx_group_indexer* gi, int32_t G) {
  return gi_valid(gi, G) ? gi_workspace(gi, G) : 0;
}

adx_status adx_group_indexer_queries(const adx_group_indexer* gi, int32_t G, void* qbar_out,
                                     float* wbar_out, void* ws, size_t ws_bytes, void* stream) {
  if (!gi_valid(gi, G) || !qbar_out || !wbar_out || !ws) return ADX_EINVAL;
  if (ws_bytes < gi_workspace(gi, G)) return ADX_EWORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int ng = gi->T / G, dc = gi->d_c, dh = gi->d_h, HS = gi->H_S, d = gi->d;
  uint8_t* p = static_cast<uint8_t*>(ws);
  auto take = [&](size_t bytes) {
    uint8_t* r = p;
    p += up(bytes);
    return r;
  };
  auto* st = reinterpret_cast<DeviceStatus*>(take(kStatusBytes));
  const int nparts = pool_ctas(gi);
  auto* pooled = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(ng) * 3 * dc * 2));
  auto* gpart = reinterpret_cast<float*>(take(static_cast<size_t>(ng) * nparts * HS * 4));
  auto* cbar = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(ng) * dc * 2));
  auto* qpre = reinterpret_cast<float*>(take(static_cast<size_t>(ng) * HS * d * 4));
  // tensor maps of both projections: W rows and X rows in boxes of 128 rows x 64 k-elements
  CUtensorMap tw_pool, tx_pool, tw_q, tx_q;
  const int box = gemm_box_rows();
  if (!encode_rows(&tw_pool, gi->w_pool, false, 3 * dc, dc, box) ||
      !encode_rows(&tx_pool, pooled, false, 3 * dc, ng, box) ||
      !encode_rows(&tw_q, gi->w_q, false, dc, static_cast<int64_t>(HS) * d, box) ||
      !encode_rows(&tx_q, cbar, false, dc, ng, box))
    return ADX_EINVAL;
  gi_pool_kernel<<<dim3(nparts, ng), kPoolThreads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(gi->cq), static_cast<const __nv_bfloat16*>(gi->h),
      static_cast<const __nv_bfloat16*>(gi->w_g), G, dc, dh, HS, pooled, gpart);
  if (cudaGetLastError() != cudaSuccess) return ADX_ECUDA;
  add_launches(1);
  // c-bar [ng, d_c] = pooled [ng, 3 d_c] W_pool^T;  q-bar before RoPE [ng, H_S d] = c-bar W_Q^T
  if (launch_gemm_bf16(tw_pool, tx_pool, cbar, false, dc, ng, 3 * dc, st, kGemmTimeoutNs, s) !=
          cudaSuccess ||
      launch_gemm_bf16(tw_q, tx_q, qpre, true, HS * d, ng, dc, st, kGemmTimeoutNs, s) !=
          cudaSuccess)
    return ADX_ECUDA;
  add_launches(2);
  gi_finish_kernel<<<ng, 256, 0, s>>>(qpre, gpart, nparts, HS, d, gi->rope_dim, gi->rope_base,
                                      gi->q_pos0, G, static_cast<__nv_bfloat16*>(qbar_out),
                                      wbar_out);
  if (cudaGetLastError() != cudaSuccess) return ADX_ECUDA;
  add_launches(1);
  return ADX_OK;
}

}  // extern "C"

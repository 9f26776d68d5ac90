// Dense projection Y = X W^T on sm_100a tensor cores, for the group indexer's two linear maps
// (ADIndex, arXiv 2611.12956v1, §4.2: W_pool applied to the pooled latents, Eq. (6), and W_Q
// applied to c-bar, Eq. (7)).
//
//   X [n, k] bf16 row-major (one row per query group), W [m, k] bf16 row-major ([out, in]),
//   Y [n, m] row-major, bf16 or fp32, accumulated in fp32.
//
// One CTA per 128 x 128 output tile. W rows are the MMA's M side (128 output features = 128
// TMEM lanes), X rows its N side (128 groups), both K-major in shared memory with the 128-byte
// swizzle, fed by TMA (no multicast) through a ring of stages of 64 k-elements. Warp 0 issues
// the TMA loads, warp 1 allocates TMEM and issues tcgen05.mma (one thread), warps 2-5 read the
// fp32 accumulator tile back with tcgen05.ld (warp w reads lane quadrant w % 4) and store it:
// thread i of a warp holds output feature m0 + 32*(w % 4) + i, so each store instruction writes
// 32 consecutive features of one row of Y. Edges past m, n or k are zero-filled by TMA and
// masked at the store. Every wait is bounded and reports through a device status word.
#include <cuda_bf16.h>

#include "adx_internal.h"
#include "sm100_ptx.cuh"

namespace adx {
namespace {

constexpr int kGemmBM = 128;          // output features per tile (MMA M)
constexpr int kGemmBN = 128;          // groups per tile (MMA N)
constexpr int kGemmBK = 64;           // k-elements per stage (128 bytes of bf16)
constexpr int kGemmStages = 6;
constexpr int kGemmThreads = 192;
constexpr int kStageBytes = (kGemmBM + kGemmBN) * 128;
constexpr int kGemmSmem = kGemmStages * kStageBytes + 1024 + 256;

__device__ __forceinline__ void gemm_timeout(DeviceStatus* st, int role) {
  if (st != nullptr && atomicCAS(&st->code, 0, 6 /* ADX_ETIMEOUT */) == 0) {
    st->where = kWhereGemm;
    st->info0 = role;
    st->info1 = static_cast<int>(blockIdx.x);
  }
}

__device__ __forceinline__ void drain(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  volatile int never = 0;
  (void)mbar_wait(bar, parity, &never, timeout_ns);
}

template <bool OUT_F32>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
            void* __restrict__ y, int m, int n, int k, DeviceStatus* st, uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGemmStages * kStageBytes);
  uint64_t* empty = full + kGemmStages;
  uint64_t* acc_full = empty + kGemmStages;
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_s + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int m_tiles = (m + kGemmBM - 1) / kGemmBM;
  const int m0 = (blockIdx.x % m_tiles) * kGemmBM;
  const int n0 = (blockIdx.x / m_tiles) * kGemmBN;
  const int kc = (k + kGemmBK - 1) / kGemmBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *abort_s = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(tmem_s, kGemmBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_s;

  if (warp == 0) {
    if (lane == 0) {  // TMA producer
      uint32_t issued = 0, parity = 0;
      for (int c = 0; c < kc; ++c) {
        const int s = c % kGemmStages;
        const uint32_t ph = static_cast<uint32_t>(c / kGemmStages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_s, timeout_ns)) break;
        uint8_t* a_s = smem + s * kStageBytes;
        uint8_t* b_s = a_s + kGemmBM * 128;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        tma_load_2d(a_s, &tm_w, &full[s], c * kGemmBK, m0);
        tma_load_2d(b_s, &tm_x, &full[s], c * kGemmBK, n0);
        issued |= 1u << s;
        parity = (parity & ~(1u << s)) | (ph << s);
      }
      if (*abort_s) gemm_timeout(st, 0);
      for (int s = 0; s < kGemmStages; ++s)  // every issued copy lands before the CTA exits
        if (issued & (1u << s)) drain(&full[s], (parity >> s) & 1u, timeout_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      constexpr uint32_t idesc = instr_desc<false>(kGemmBN);
      bool any = false;
      for (int c = 0; c < kc; ++c) {
        const int s = c % kGemmStages;
        const uint32_t ph = static_cast<uint32_t>(c / kGemmStages) & 1u;
        if (!mbar_wait(&full[s], ph, abort_s, timeout_ns)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * kStageBytes);
        const uint32_t b_addr = a_addr + kGemmBM * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 4 x 16 k-elements (32 bytes) per 128-byte row
          umma_ss<false>(tmem, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32),
                         idesc, (c > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
        any = true;
      }
      if (*abort_s) gemm_timeout(st, 1);
      // the accumulator is complete once every MMA issued so far has finished
      if (any) umma_commit(acc_full);
      else mbar_arrive(acc_full);
    }
  } else {  // epilogue: warps 2..5, lane quadrant warp % 4
    const int lq = warp & 3;
    const int row = m0 + lq * 32 + lane;  // output feature of this thread
    int got = 0;
    if (lane == 0) got = mbar_wait(acc_full, 0, abort_s, timeout_ns) ? 1 : 0;
    got = __shfl_sync(0xffffffffu, got, 0);
    if (got && !*abort_s) {
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < kGemmBN; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(lq * 32) << 16) + static_cast<uint32_t>(c0), v);
        tmem_wait_ld();
        if (row < m) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int g = n0 + c0 + j;
            if (g < n) {
              const int64_t at = static_cast<int64_t>(g) * m + row;
              if constexpr (OUT_F32) {
                static_cast<float*>(y)[at] = v[j];
              } else {
                static_cast<__nv_bfloat16*>(y)[at] = __float2bfloat16_rn(v[j]);
              }
            }
          }
        }
      }
    } else if (lane == 0) {
      gemm_timeout(st, 2);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // an MMA still in flight after an abort must finish before its TMEM is freed
    if (lane == 0 && *abort_s) drain(acc_full, 0, timeout_ns);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kGemmBN);
  }
}

}  // namespace

cudaError_t launch_gemm_bf16(const CUtensorMap& tm_w, const CUtensorMap& tm_x, void* y,
                             bool out_f32, int m, int n, int k, DeviceStatus* st,
                             uint64_t timeout_ns, cudaStream_t s) {
  if (m <= 0 || n <= 0 || k <= 0) return cudaSuccess;
  const int64_t tiles = static_cast<int64_t>((m + kGemmBM - 1) / kGemmBM) *
                        ((n + kGemmBN - 1) / kGemmBN);
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  auto kern = out_f32 ? gemm_kernel<true> : gemm_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(tiles), kGemmThreads, kGemmSmem, s>>>(tm_w, tm_x, y, m, n, k, st,
                                                                     timeout_ns);
  return cudaGetLastError();
}

int gemm_box_rows() { return kGemmBM; }

}  // namespace adx

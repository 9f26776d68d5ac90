// Indexer scoring on sm_100a tensor cores.
//
// Computes, for every (query row r, key c) pair that the work decomposition covers,
//     I[r, c] = k_scale[c] * sum_j (w[r, j] * q_scale[r]) * ReLU(q[r, j] . k[c])
// which is the DSA indexer score (ADIndex, arXiv 2611.12956v1, §3 Eq. (1)); with bf16
// operands both scales are 1, with e4m3 operands the per-token scales factor out of the
// ReLU because they are positive. Keys the query may not see (position > query position,
// or beyond the key range) are written as -inf.
//
// Mapping onto tcgen05: keys are the MMA's M side (128 keys = 128 TMEM lanes) and
// (query token, head) pairs are its N side (N = tokens * H <= 256), both K-major in shared
// memory with the 128-byte swizzle, fed by TMA. The fp32 accumulator tile lives in TMEM
// (double-buffered); each epilogue thread owns one key (one TMEM lane) and reduces the
// heads of every token in registers - ReLU, gate and head sum never leave the SM, so the
// per-head logits [T, H, S] are never written anywhere.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 allocates TMEM and issues the
// MMAs (one thread), warps 2-5 run the epilogue. The grid is persistent: CTA c takes work
// items c, c + gridDim.x, ... where an item is (row block, chunk of key tiles).
#include <cuda_bf16.h>

#include "adx_internal.h"
#include "sm100_ptx.cuh"

namespace adx {

namespace {

constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;

__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }
__host__ __device__ constexpr int pow2ceil(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

template <int H_, int TOK_, int DB_, bool FP8_>
struct Cfg {
  static constexpr int H = H_;
  static constexpr int TOK = TOK_;
  static constexpr int DB = DB_;             // bytes per q/k row (d * element size)
  static constexpr bool FP8 = FP8_;
  static constexpr int N = TOK * H;          // MMA N
  static constexpr int KC = DB / 128;        // 128-byte K chunks
  static constexpr int ELEMS_PER_CHUNK = FP8 ? 128 : 64;
  static constexpr int KSTEPS = DB / 32;     // 32 bytes of K per MMA instruction
  static constexpr int QBYTES = N * DB;
  static constexpr int KBYTES = kTileM * DB;
  static constexpr int ST = cmin(8, (200 * 1024 - QBYTES) / KBYTES);
  static constexpr int ACC = 2;
  static constexpr int TMEM_COLS = pow2ceil(cmax(32, ACC * N));
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = QBYTES;
  static constexpr int OFF_W = OFF_K + ST * KBYTES;
  static constexpr int OFF_BAR = OFF_W + kEpiWarps * N * 4;  // one gate copy per epilogue warp
  static constexpr int NBAR = 2 * ST + 2 * ACC + 3;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "invalid MMA N");
  static_assert(DB % 128 == 0, "rows must be a multiple of 128 bytes");
  static_assert(QBYTES % 1024 == 0 && KBYTES % 1024 == 0, "alignment");
  static_assert(ST >= 2, "not enough shared memory for a pipeline");
};

struct Item {
  int b, row0, row_end, t_begin, t_end, nkeys;
  int64_t key_row0;  // first key row of the batch in the key tensor map
};

__device__ __forceinline__ int64_t row_position(const ScoreArgs& a, int r) {
  if (a.seq_len != nullptr) return static_cast<int64_t>(a.seq_len[r / a.rows_per_batch]) - 1;
  return a.pos_base + static_cast<int64_t>(r) * a.pos_step;
}

template <int TOK>
__device__ __forceinline__ bool decode_item(const ScoreArgs& a, int it, Item& x) {
  const int kc = it % a.chunks_per_block;
  int rbg = it / a.chunks_per_block;
  const int total_rb = a.row_blocks_per_batch * a.n_batches;
  if (a.reverse_order) rbg = total_rb - 1 - rbg;
  x.b = rbg / a.row_blocks_per_batch;
  const int rb = rbg % a.row_blocks_per_batch;
  x.row0 = x.b * a.rows_per_batch + rb * TOK;
  x.row_end = min(min(x.row0 + TOK, (x.b + 1) * a.rows_per_batch), a.R);
  if (x.row0 >= x.row_end) return false;
  int64_t nk;
  if (a.key_pos != nullptr) {
    nk = a.keys_per_batch;
  } else if (a.seq_len != nullptr) {
    nk = min(static_cast<int64_t>(a.seq_len[x.b]), static_cast<int64_t>(a.keys_per_batch));
  } else {
    nk = min(row_position(a, x.row_end - 1) + 1, static_cast<int64_t>(a.keys_per_batch));
  }
  if (nk <= 0) return false;
  x.nkeys = static_cast<int>(nk);
  const int ntiles = (x.nkeys + kTileM - 1) / kTileM;
  x.t_begin = kc * a.chunk_tiles;
  x.t_end = min(x.t_begin + a.chunk_tiles, ntiles);
  x.key_row0 = static_cast<int64_t>(x.b) * a.key_batch_stride;
  return x.t_begin < x.t_end;
}

__device__ __forceinline__ void raise_timeout(const ScoreArgs& a, int role) {
  if (a.status != nullptr && atomicCAS(&a.status->code, 0, 6 /* ADX_ETIMEOUT */) == 0) {
    a.status->where = kWhereScore;
    a.status->info0 = role;
    a.status->info1 = static_cast<int>(blockIdx.x);
  }
}

// Waits for completion of the given phase with a bound but without giving up early on the
// abort flag: used to drain copies and MMAs in flight before the CTA exits.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  volatile int never = 0;
  (void)mbar_wait(bar, parity, &never, timeout_ns);
}

template <class C>
__global__ void __launch_bounds__(kThreads, 1)
score_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const ScoreArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* q_s = smem + C::OFF_Q;
  uint8_t* k_s = smem + C::OFF_K;
  float* w_s = reinterpret_cast<float*>(smem + C::OFF_W);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::ST;
  uint64_t* acc_full = bars + 2 * C::ST;
  uint64_t* acc_empty = acc_full + C::ACC;
  uint64_t* q_full = acc_empty + C::ACC;
  uint64_t* q_empty = q_full + 1;
  uint64_t* drain = q_full + 2;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_s = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < C::ACC; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiWarps);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(drain, 1);
    *abort_s = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_s, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_s;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t q_phase = 0;
      bool q_loaded = false;
      uint32_t issued_mask = 0, issued_parity = 0;
      for (int it = blockIdx.x; it < a.n_items && !*abort_s; it += gridDim.x) {
        Item x;
        if (!decode_item<C::TOK>(a, it, x)) continue;
        if (q_loaded) {
          if (!mbar_wait(q_empty, q_phase ^ 1u, abort_s, a.timeout_ns)) break;
        }
        mbar_arrive_expect_tx(q_full, C::QBYTES);
#pragma unroll
        for (int kc = 0; kc < C::KC; ++kc)
          tma_load_2d(q_s + kc * C::N * 128, &tm_q, q_full, kc * C::ELEMS_PER_CHUNK,
                      x.row0 * C::H);
        q_loaded = true;
        q_phase ^= 1u;
        for (int t = x.t_begin; t < x.t_end; ++t) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_s, a.timeout_ns)) break;
          mbar_arrive_expect_tx(&full[stage], C::KBYTES);
          const int32_t y = static_cast<int32_t>(x.key_row0 + static_cast<int64_t>(t) * kTileM);
#pragma unroll
          for (int kc = 0; kc < C::KC; ++kc)
            tma_load_2d(k_s + stage * C::KBYTES + kc * kTileM * 128, &tm_k, &full[stage],
                        kc * C::ELEMS_PER_CHUNK, y);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::ST) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_s) raise_timeout(a, 0);
      // drain: every issued copy must land before the CTA may exit
      for (int s = 0; s < C::ST; ++s)
        if (issued_mask & (1u << s)) drain_wait(&full[s], (issued_parity >> s) & 1u, a.timeout_ns);
      if (q_loaded) drain_wait(q_full, q_phase ^ 1u, a.timeout_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc<C::FP8>(C::N);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t q_phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      for (int it = blockIdx.x; it < a.n_items && !*abort_s; it += gridDim.x) {
        Item x;
        if (!decode_item<C::TOK>(a, it, x)) continue;
        if (!mbar_wait(q_full, q_phase, abort_s, a.timeout_ns)) break;
        q_phase ^= 1u;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(q_s);
        bool ok = true;
        for (int t = x.t_begin; t < x.t_end; ++t) {
          if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_s, a.timeout_ns) ||
              !mbar_wait(&full[stage], phase, abort_s, a.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(k_s + stage * C::KBYTES);
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::N);
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            const uint32_t koff = static_cast<uint32_t>((kk / 4) * kTileM * 128 + (kk % 4) * 32);
            const uint32_t qoff = static_cast<uint32_t>((kk / 4) * C::N * 128 + (kk % 4) * 32);
            umma_ss<C::FP8>(d_tmem, smem_desc_sw128(k_addr + koff), smem_desc_sw128(q_addr + qoff),
                            idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          umma_commit(&acc_full[acc]);
          any = true;
          if (++stage == C::ST) {
            stage = 0;
            phase ^= 1u;
          }
          if (++acc == C::ACC) {
            acc = 0;
            acc_phase ^= 1u;
          }
        }
        umma_commit(q_empty);  // Q buffer is free once this item's MMAs complete
        if (!ok) break;
      }
      if (*abort_s) raise_timeout(a, 1);
      if (any) {
        umma_commit(drain);
        drain_wait(drain, 0, a.timeout_ns);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - 2;                  // 0..3
    const int lq = warp & 3;                  // TMEM lane quadrant this warp may access
    const int m = lq * 32 + lane;             // key row within the tile = TMEM lane
    constexpr int CW = C::N < 32 ? C::N : 32; // TMEM columns per load
    float* w_w = w_s + ew * C::N;             // this warp's copy of the gates
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int it = blockIdx.x; it < a.n_items && !*abort_s; it += gridDim.x) {
      Item x;
      if (!decode_item<C::TOK>(a, it, x)) continue;
      // gates of this item's rows, with the per-token query scale folded in
      __syncwarp();
      for (int i = lane; i < C::N; i += 32) {
        const int r = x.row0 + i / C::H;
        float wv = 0.f;
        if (r < x.row_end) {
          wv = a.w[static_cast<int64_t>(r) * C::H + (i % C::H)];
          if (a.q_scale != nullptr) wv *= a.q_scale[r];
        }
        w_w[i] = wv;
      }
      __syncwarp();
      int64_t rpos[C::TOK];
#pragma unroll
      for (int tt = 0; tt < C::TOK; ++tt)
        rpos[tt] = (x.row0 + tt < x.row_end) ? row_position(a, x.row0 + tt) : -1;

      bool ok = true;
      for (int t = x.t_begin; t < x.t_end; ++t) {
        int got = 0;
        if (lane == 0) got = mbar_wait(&acc_full[acc], acc_phase, abort_s, a.timeout_ns) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int c = t * kTileM + m;  // key index within the batch
        const bool key_ok = c < x.nkeys;
        int64_t kpos = c;
        float ks = 1.f;
        if (key_ok) {
          const int64_t kr = x.key_row0 + c;
          if (a.key_pos != nullptr) kpos = a.key_pos[kr];
          if (a.k_scale != nullptr) ks = a.k_scale[kr];
        }
        float accum[C::TOK];
#pragma unroll
        for (int tt = 0; tt < C::TOK; ++tt) accum[tt] = 0.f;
        const uint32_t taddr =
            tmem_base + (static_cast<uint32_t>(lq * 32) << 16) + static_cast<uint32_t>(acc * C::N);
#pragma unroll
        for (int c0 = 0; c0 < C::N; c0 += CW) {
          float v[CW];
          if constexpr (CW == 32) {
            tmem_ld32(taddr + c0, v);
          } else {
            tmem_ld16(taddr + c0, v);
          }
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < CW; ++i) {
            const int col = c0 + i;
            accum[col / C::H] = fmaf(w_w[col], fmaxf(v[i], 0.f), accum[col / C::H]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
        if (++acc == C::ACC) {
          acc = 0;
          acc_phase ^= 1u;
        }
#pragma unroll
        for (int tt = 0; tt < C::TOK; ++tt) {
          const int r = x.row0 + tt;
          if (r < x.row_end) {
            const bool vis = key_ok && kpos <= rpos[tt];
            a.scores[static_cast<int64_t>(r) * a.score_ld + c] = vis ? ks * accum[tt] : -INFINITY;
          }
        }
      }
      if (!ok) break;
    }
    if (lane == 0 && *abort_s) raise_timeout(a, 2);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <class C>
cudaError_t launch_cfg(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const ScoreArgs& a,
                       int grid, cudaStream_t s) {
  auto kern = score_kernel<C>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, C::SMEM, s>>>(tm_q, tm_k, a);
  return cudaGetLastError();
}

}  // namespace

int score_tokens_per_tile(int H) {
  switch (H) {
    case 4: return 64;
    case 8: return 32;
    case 16: return 16;
    case 32: return 8;
    case 64: return 4;
    default: return 0;
  }
}

bool score_config_supported(bool fp8, int H, int d) {
  if (score_tokens_per_tile(H) == 0) return false;
  if (fp8) return d == 128;
  return d == 64 || d == 128;
}

#define ADX_SCORE_CONFIGS(X)  \
  /* prefill tiles: N = tokens * H = 256 */ \
  X(false, 64, 4, 128) X(true, 64, 4, 128) X(false, 16, 16, 128) X(true, 16, 16, 128) \
  X(false, 4, 64, 64) X(false, 4, 64, 128) X(true, 4, 64, 128) X(false, 8, 32, 128)  \
  X(true, 8, 32, 128) X(false, 32, 8, 128) X(true, 32, 8, 128) X(false, 64, 4, 64)   \
  X(false, 16, 16, 64)                                                                 \
  /* one query per key batch (decode and its bank refresh): N = H */                  \
  X(false, 64, 1, 128) X(true, 64, 1, 128) X(false, 16, 1, 128) X(true, 16, 1, 128)   \
  X(false, 32, 1, 128) X(true, 32, 1, 128)

// tok: tokens per N tile; either score_tokens_per_tile(H) (prefill) or 1 (one query per
// key batch: decode and its bank refresh).
cudaError_t launch_score(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const ScoreArgs& a,
                         bool fp8, int H, int d, int tok, int grid, cudaStream_t s) {
#define ADX_CASE(FP, HH, TT, DD)                                                        \
  if (fp8 == FP && H == HH && tok == TT && d == DD)                                     \
    return launch_cfg<Cfg<HH, TT, (FP ? DD : 2 * DD), FP>>(tm_q, tm_k, a, grid, s);
  ADX_SCORE_CONFIGS(ADX_CASE)
#undef ADX_CASE
  return cudaErrorNotSupported;
}

// Resident CTAs per SM for a configuration (shared memory and TMEM columns both bound it),
// 0 when the configuration is not compiled.
int score_blocks_per_sm(bool fp8, int H, int d, int tok) {
#define ADX_CASE(FP, HH, TT, DD)                                                        \
  if (fp8 == FP && H == HH && tok == TT && d == DD) {                                   \
    using C = Cfg<HH, TT, (FP ? DD : 2 * DD), FP>;                                      \
    return cmin(cmin((227 * 1024) / C::SMEM, 512 / C::TMEM_COLS), 2);                  \
  }
  ADX_SCORE_CONFIGS(ADX_CASE)
#undef ADX_CASE
  return 0;
}

}  // namespace adx

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
// Warp roles: warp 0 issues TMA loads, warp 1 allocates TMEM and issues the MMAs (one
// thread), the remaining one or two warpgroups run the epilogue (each owns half of the
// tile's query tokens). The grid is persistent and statically balanced: all (row block,
// key tile) pairs are laid end to end, longest rows first, and every CTA takes an equal
// contiguous share, loading a row block's queries once for its whole run of key tiles.
#include <cuda_bf16.h>

#include "adx_internal.h"
#include "sm100_ptx.cuh"

namespace adx {

namespace {

constexpr int kMaxThreads = 320;

__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }
__host__ __device__ constexpr int pow2ceil(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// Key tiles: contiguous rows (0), rows gathered one by one with tile::gather4 (1), or whole
// 128-row blocks from a per-batch block list (2).
constexpr int kKeysContiguous = 0, kKeysGather = 1, kKeysBlocks = 2;

template <int H_, int TOK_, int DB_, bool FP8_, int KM_ = kKeysContiguous>
struct Cfg {
  static constexpr int H = H_;
  static constexpr int TOK = TOK_;
  static constexpr int DB = DB_;             // bytes per q/k row (d * element size)
  static constexpr bool FP8 = FP8_;
  static constexpr bool GATHER = KM_ == kKeysGather;  // key rows gathered (tile::gather4)
  static constexpr bool BLOCKS = KM_ == kKeysBlocks;  // key tiles from a block list
  static constexpr int N = TOK * H;          // MMA N
  static constexpr int KC = DB / 128;        // 128-byte K chunks
  static constexpr int ELEMS_PER_CHUNK = FP8 ? 128 : 64;
  static constexpr int KSTEPS = DB / 32;     // 32 bytes of K per MMA instruction
  // Epilogue warpgroups. With narrow tiles (one token, or N <= 64: BUF_SPLIT), the tiles go
  // round the warpgroups: warpgroup g reduces the tiles whose accumulator buffer index is g
  // modulo EG, all their tokens, so each warp has EG MMA periods per tile (one warpgroup per
  // tile cannot keep up with the key stream there). With wide tiles the two warpgroups split
  // the tokens of every tile instead (keeps the per-thread partial sums in registers).
  static constexpr bool BUF_SPLIT = TOK == 1 || TOK * H <= 64;
  static constexpr int EG = 2;
  static constexpr int EPI_WARPS = 4 * EG;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int TOKG = BUF_SPLIT ? TOK : TOK / EG;  // tokens one warp reduces per tile
  static constexpr int NG = TOKG * H;        // accumulator columns one warp reads per tile
  static constexpr int CW = NG < 32 ? NG : 32;  // TMEM columns per load
  static constexpr int NCH = NG / CW;        // loads per tile per thread
  static constexpr int NP = (H >= 16 && TOKG <= 4) ? 4 : 1;  // partial sums per token
  static constexpr int QBYTES = N * DB;
  static constexpr int KBYTES = kTileM * DB;
  static constexpr int ST = cmin(8, (200 * 1024 - QBYTES) / KBYTES);
  static constexpr int ACC = BUF_SPLIT ? 2 * EG : 2;  // accumulator buffers in TMEM
  static constexpr int TMEM_COLS = pow2ceil(cmax(32, ACC * N));
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = QBYTES;
  static constexpr int OFF_W = OFF_K + ST * KBYTES;
  static constexpr int OFF_BAR = OFF_W + EPI_WARPS * NG * 4;  // one gate copy per epilogue warp
  static constexpr int NBAR = 2 * ST + 2 * ACC + 3;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_SCAN = OFF_MISC + 64;
  // gathered key rows of a tile, read as 16-byte vectors
  static constexpr int OFF_IDX = (OFF_SCAN + 8 * (THREADS / 32) + 15) / 16 * 16;
  static constexpr int SMEM = OFF_IDX + (GATHER ? kTileM * 4 : 0) + 1024;  // + alignment slack
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "invalid MMA N");
  static_assert(DB % 128 == 0, "rows must be a multiple of 128 bytes");
  static_assert(QBYTES % 1024 == 0 && KBYTES % 1024 == 0, "alignment");
  static_assert(ST >= 2, "not enough shared memory for a pipeline");
  static_assert(NG % CW == 0 && CW % 4 == 0 && (H >= 32 ? H % CW == 0 : CW % H == 0),
                "epilogue chunking");
  static_assert(THREADS <= kMaxThreads, "block size");
  static_assert(ACC % EG == 0, "every epilogue warpgroup owns the same number of buffers");
  static_assert(OFF_IDX % 16 == 0 && OFF_BAR % 8 == 0 && OFF_K % 1024 == 0, "alignment");
};

// One row block of the work: TOK consecutive query rows of one key batch and the key
// tiles they need.
struct Block {
  int b, row0, row_end, nkeys, ntiles;
  int64_t key_row0;  // first key row of the batch in the key tensor map
};

__device__ __forceinline__ int64_t row_position(const ScoreArgs& a, int r) {
  if (a.row_pos != nullptr) return a.row_pos[r];
  if (a.seq_len != nullptr) return static_cast<int64_t>(a.seq_len[r / a.rows_per_batch]) - 1;
  return a.pos_base + static_cast<int64_t>(r) * a.pos_step;
}

// Row block number i of the schedule (longest first for a causal prefix).
template <int TOK>
__device__ __forceinline__ void block_info(const ScoreArgs& a, int i, Block& x) {
  const int nb = a.row_blocks_per_batch * a.n_batches;
  const int rbg = a.reverse_order ? nb - 1 - i : i;
  x.b = rbg / a.row_blocks_per_batch;
  const int rb = rbg % a.row_blocks_per_batch;
  x.row0 = x.b * a.rows_per_batch + rb * TOK;
  x.row_end = min(min(x.row0 + TOK, (x.b + 1) * a.rows_per_batch), a.R);
  x.key_row0 = static_cast<int64_t>(x.b / (a.key_batch_div > 1 ? a.key_batch_div : 1)) *
               a.key_batch_stride;
  x.nkeys = 0;
  x.ntiles = 0;
  if (x.row0 >= x.row_end) return;
  int64_t nk;
  if (a.key_blk != nullptr) {
    nk = a.key_blk_count != nullptr
             ? static_cast<int64_t>(a.key_blk_count[x.b]) * kTileM
             : (row_position(a, x.row_end - 1) / kTileM + 1) * kTileM;
    nk = min(nk, static_cast<int64_t>(a.keys_per_batch));
  } else if (a.key_pos != nullptr || a.key_idx != nullptr) {
    nk = a.keys_per_batch;
  } else if (a.seq_len != nullptr && a.row_pos == nullptr) {
    nk = min(static_cast<int64_t>(a.seq_len[x.b]), static_cast<int64_t>(a.keys_per_batch));
  } else {
    nk = min(row_position(a, x.row_end - 1) + 1, static_cast<int64_t>(a.keys_per_batch));
  }
  if (nk <= 0) return;
  x.nkeys = static_cast<int>(nk);
  x.ntiles = (x.nkeys + kTileM - 1) / kTileM;
}

// Cost of a row block in tile units: its tiles plus a fixed kRowBlockCost for starting it
// (its query tile's load into the single query buffer after the previous block's last MMA,
// the gates): without it the CTAs that get the many short row blocks at the end of a causal
// schedule finish about a quarter later than the rest. Tile t of a block whose costs start at
// unit cum is unit cum + kRowBlockCost + t.
constexpr int64_t kRowBlockCost = 2;

__device__ __forceinline__ int64_t block_cost(const Block& x) {
  return x.ntiles > 0 ? x.ntiles + kRowBlockCost : 0;
}

// Balanced static partition: all row blocks laid end to end in schedule order, each as its
// cost units; CTA c owns the units [c*W/grid, (c+1)*W/grid) and scores the tiles whose units
// it owns. Computed once per CTA by all its threads; returns the first row block touching the
// range and the unit at which that block's costs start.
template <class C>
__device__ __forceinline__ void partition(const ScoreArgs& a, int64_t* scan_s, int64_t& start,
                                          int64_t& end, int& b0, int64_t& base0) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = C::THREADS / 32;
  const int nb = a.row_blocks_per_batch * a.n_batches;
  const int per = (nb + C::THREADS - 1) / C::THREADS;
  const int lo = min(nb, tid * per), hi = min(nb, lo + per);
  int64_t mine = 0;
  for (int i = lo; i < hi; ++i) {
    Block x;
    block_info<C::TOK>(a, i, x);
    mine += block_cost(x);
  }
  int64_t incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) scan_s[warp] = incl;
  __syncthreads();
  int64_t before = 0, total = 0;
  for (int w = 0; w < NW; ++w) {
    const int64_t v = scan_s[w];
    if (w < warp) before += v;
    total += v;
  }
  const int64_t excl = before + incl - mine;
  start = static_cast<int64_t>(blockIdx.x) * total / gridDim.x;
  end = static_cast<int64_t>(blockIdx.x + 1) * total / gridDim.x;
  __syncthreads();  // everyone has read scan_s
  if (start < end && excl <= start && start < excl + mine) {
    int64_t cum = excl;
    for (int i = lo; i < hi; ++i) {
      Block x;
      block_info<C::TOK>(a, i, x);
      if (start < cum + block_cost(x)) {
        scan_s[0] = i;
        scan_s[1] = cum;
        break;
      }
      cum += block_cost(x);
    }
  }
  __syncthreads();
  b0 = start < end ? static_cast<int>(scan_s[0]) : 0;
  base0 = start < end ? scan_s[1] : 0;
}

// The sequence of (row block, key tile range) a CTA works through; identical in every role.
struct WorkIter {
  int64_t start, end, cum;
  int bi, nblocks;
  bool rr;

  template <int TOK>
  __device__ __forceinline__ bool next(const ScoreArgs& a, Block& x, int& t_lo, int& t_hi) {
    if (rr) {
      while (bi < nblocks) {
        block_info<TOK>(a, bi, x);
        bi += gridDim.x;
        if (x.ntiles > 0) {
          t_lo = 0;
          t_hi = x.ntiles;
          return true;
        }
      }
      return false;
    }
    while (bi < nblocks && cum < end) {
      block_info<TOK>(a, bi, x);
      ++bi;
      const int64_t t0 = cum + kRowBlockCost;  // unit of the block's first tile
      const int64_t lo = max(start - t0, int64_t(0));
      const int64_t hi = min(end - t0, static_cast<int64_t>(x.ntiles));
      cum += block_cost(x);
      if (lo < hi) {
        t_lo = static_cast<int>(lo);
        t_hi = static_cast<int>(hi);
        return true;
      }
    }
    return false;
  }
};

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

template <int CW>
__device__ __forceinline__ void tmem_ld_chunk(uint32_t taddr, float (&v)[CW]) {
  if constexpr (CW == 32) {
    tmem_ld32(taddr, v);
  } else {
    tmem_ld16(taddr, v);
  }
}

// ReLU, gate and head sum of one chunk of accumulator columns (group-local columns
// c0 .. c0+CW-1), as packed fp32x2 FMAs into independent partial sums.
template <class C>
__device__ __forceinline__ void reduce_chunk(const float (&v)[C::CW], const float* w, int c0,
                                             float2 (&acc)[C::TOKG][C::NP]) {
#pragma unroll
  for (int i = 0; i < C::CW; i += 4) {
    const int col = c0 + i;
    const int tt = col / C::H;
    const int m = (col % C::H) / 2;
    const float4 w4 = *reinterpret_cast<const float4*>(w + col);
    const float2 r01 = make_float2(fmaxf(v[i], 0.f), fmaxf(v[i + 1], 0.f));
    const float2 r23 = make_float2(fmaxf(v[i + 2], 0.f), fmaxf(v[i + 3], 0.f));
    acc[tt][m % C::NP] = __ffma2_rn(r01, make_float2(w4.x, w4.y), acc[tt][m % C::NP]);
    acc[tt][(m + 1) % C::NP] =
        __ffma2_rn(r23, make_float2(w4.z, w4.w), acc[tt][(m + 1) % C::NP]);
  }
}

// Gate-folded variant of reduce_chunk: the queries were pre-multiplied by their (non-negative)
// gates, so a column's contribution is just ReLU(x).
template <class C>
__device__ __forceinline__ void reduce_chunk_folded(const float (&v)[C::CW], int c0,
                                                    float2 (&acc)[C::TOKG][C::NP]) {
#pragma unroll
  for (int i = 0; i < C::CW; i += 2) {
    const int col = c0 + i;
    const int tt = col / C::H;
    const int m = (col % C::H) / 2;
    acc[tt][m % C::NP] =
        __fadd2_rn(acc[tt][m % C::NP], make_float2(fmaxf(v[i], 0.f), fmaxf(v[i + 1], 0.f)));
  }
}

// One score of the output matrix; streaming (evict-first) stores for matrices far larger
// than the L2, so that they do not displace the key tiles every row block re-reads.
__device__ __forceinline__ void store_score(const ScoreArgs& a, int64_t at, float v) {
  if (a.stream_scores) __stcs(a.scores + at, v);
  else a.scores[at] = v;
}

// True when the queries of every row of the block carry their gates already.
__device__ __forceinline__ bool block_folded(const ScoreArgs& a, const Block& x) {
  if (a.fold_flag == nullptr) return false;
  int all = 1;
  for (int r = x.row0; r < x.row_end; ++r) all &= a.fold_flag[r];
  return all != 0;
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
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
  int64_t* scan_s = reinterpret_cast<int64_t*>(smem + C::OFF_SCAN);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < C::ACC; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::BUF_SPLIT ? 4 : C::EPI_WARPS);
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
  int64_t start = 0, end = 0, base0 = 0;
  int b0 = blockIdx.x;
  if (!a.round_robin) partition<C>(a, scan_s, start, end, b0, base0);  // contains __syncthreads
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_s;
  const int nblocks = a.row_blocks_per_batch * a.n_batches;
  const WorkIter work0{start, end, base0, b0, nblocks, a.round_robin != 0};

  if (warp == 0 && C::GATHER) {
    // ---------------------------------------------- TMA producer, gathered key rows
    // The warp reads a tile's 128 key positions (4 per lane) into shared memory; lane 0
    // waits for the stage, then issues 32 four-row gathers per 128-byte column chunk.
    int32_t* idx_s = reinterpret_cast<int32_t*>(smem + C::OFF_IDX);
    int stage = 0;
    uint32_t phase = 0;
    uint32_t q_phase = 0;
    bool q_loaded = false;
    uint32_t issued_mask = 0, issued_parity = 0;
    WorkIter work = work0;
    Block x;
    int t_lo, t_hi;
    int ok = 1;
    while (ok && !*abort_s && work.next<C::TOK>(a, x, t_lo, t_hi)) {
      if (lane == 0) {
        if (q_loaded && !mbar_wait(q_empty, q_phase ^ 1u, abort_s, a.timeout_ns)) {
          ok = 0;
        } else {
          mbar_arrive_expect_tx(q_full, C::QBYTES);
#pragma unroll
          for (int kc = 0; kc < C::KC; ++kc)
            tma_load_2d(q_s + kc * C::N * 128, &tm_q, q_full, kc * C::ELEMS_PER_CHUNK,
                        x.row0 * C::H);
          q_loaded = true;
          q_phase ^= 1u;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const int32_t* kidx = a.key_idx + static_cast<int64_t>(x.b) * a.key_idx_stride;
      // rows of tile t held by this lane (tile rows lane*4 .. lane*4+3); a slot with no key
      // loads some row of the range, and the epilogue masks it
      auto tile_rows = [&](int t, int32_t (&r)[4]) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = t * kTileM + lane * 4 + u;
          const int32_t p = c < a.n_idx ? kidx[c] : -1;
          const bool v = p >= 0 && p < a.S_valid;
          r[u] = static_cast<int32_t>(x.key_row0 + (v ? p : 0));
        }
      };
      int32_t nxt[4];
      if (t_lo < t_hi) tile_rows(t_lo, nxt);
      for (int t = t_lo; t < t_hi; ++t) {
#pragma unroll
        for (int u = 0; u < 4; ++u) idx_s[lane * 4 + u] = nxt[u];
        if (t + 1 < t_hi) tile_rows(t + 1, nxt);  // in flight while lane 0 issues this tile
        __syncwarp();
        if (lane == 0) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_s, a.timeout_ns)) {
            ok = 0;
          } else {
            mbar_arrive_expect_tx(&full[stage], C::KBYTES);
#pragma unroll
            for (int kc = 0; kc < C::KC; ++kc) {
#pragma unroll 8
              for (int g = 0; g < kTileM / 4; ++g) {
                const int4 rr = *reinterpret_cast<const int4*>(idx_s + 4 * g);
                tma_gather4_2d(k_s + stage * C::KBYTES + kc * kTileM * 128 + g * 512, &tm_k,
                               &full[stage], kc * C::ELEMS_PER_CHUNK, rr.x, rr.y, rr.z, rr.w);
              }
            }
            issued_mask |= 1u << stage;
            issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);  // also: lane 0 has read idx_s
        if (!ok) break;
        if (++stage == C::ST) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (lane == 0) {
      if (*abort_s) raise_timeout(a, 0);
      // drain: every issued copy must land before the CTA may exit
      for (int s2 = 0; s2 < C::ST; ++s2)
        if (issued_mask & (1u << s2))
          drain_wait(&full[s2], (issued_parity >> s2) & 1u, a.timeout_ns);
      if (q_loaded) drain_wait(q_full, q_phase ^ 1u, a.timeout_ns);
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t q_phase = 0;
      bool q_loaded = false;
      uint32_t issued_mask = 0, issued_parity = 0;
      WorkIter work = work0;
      Block x;
      int t_lo, t_hi;
      while (!*abort_s && work.next<C::TOK>(a, x, t_lo, t_hi)) {
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
        for (int t = t_lo; t < t_hi; ++t) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_s, a.timeout_ns)) break;
          mbar_arrive_expect_tx(&full[stage], C::KBYTES);
          int64_t tile_row = static_cast<int64_t>(t) * kTileM;
          if constexpr (C::BLOCKS) {
            const int32_t bk = __ldg(a.key_blk + static_cast<int64_t>(x.b) * a.key_blk_stride + t);
            tile_row = bk >= 0 ? static_cast<int64_t>(bk) * kTileM : 0;  // no tile: masked
          }
          const int32_t y = static_cast<int32_t>(x.key_row0 + tile_row);
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
      WorkIter work = work0;
      Block x;
      int t_lo, t_hi;
      while (!*abort_s && work.next<C::TOK>(a, x, t_lo, t_hi)) {
        if (!mbar_wait(q_full, q_phase, abort_s, a.timeout_ns)) break;
        q_phase ^= 1u;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(q_s);
        bool ok = true;
        for (int t = t_lo; t < t_hi; ++t) {
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
        umma_commit(q_empty);  // Q buffer is free once this block's MMAs complete
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
    const int ew = warp - 2;                  // 0 .. EPI_WARPS-1
    const int grp = ew / 4;                   // epilogue warpgroup
    const int lq = warp & 3;                  // TMEM lane quadrant this warp may access
    const int m = lq * 32 + lane;             // key row within the tile = TMEM lane
    float* w_w = w_s + ew * C::NG;            // this warp's copy of the gates
    const int tok0 = C::BUF_SPLIT ? 0 : grp * C::TOKG;  // first token this warp reduces
    int64_t gi = 0;                           // tile counter of this CTA (selects the buffer)
    WorkIter work = work0;
    Block x;
    int t_lo, t_hi;
    while (!*abort_s && work.next<C::TOK>(a, x, t_lo, t_hi)) {
      // Gates of this block's rows with the per-token query scale folded in; a row whose
      // queries carry their gates already gets gate 1. When every row of the block does, the
      // epilogue needs no gates at all and applies only the per-token scale.
      const bool folded = block_folded(a, x);
      __syncwarp();
      const int rowg = x.row0 + tok0;
      for (int i = lane; i < C::NG && !folded; i += 32) {
        const int r = rowg + i / C::H;
        float wv = 0.f;
        if (r < x.row_end) {
          const bool fr = a.fold_flag != nullptr && a.fold_flag[r];
          wv = fr ? 1.f : a.w[static_cast<int64_t>(r) * C::H + (i % C::H)];
          if (a.q_scale != nullptr) wv *= a.q_scale[r];
        }
        w_w[i] = wv;
      }
      __syncwarp();
      int32_t rpos[C::TOKG];
      float tokf[C::TOKG];
#pragma unroll
      for (int tt = 0; tt < C::TOKG; ++tt) {
        const bool in = rowg + tt < x.row_end;
        rpos[tt] = in ? static_cast<int32_t>(row_position(a, rowg + tt)) : -1;
        tokf[tt] = (folded && in && a.q_scale != nullptr) ? a.q_scale[rowg + tt] : 1.f;
      }

      // Per-key metadata of a tile (position for the causal test, key scale, block slots) in
      // two steps: the loads are issued a tile ahead into raw registers, and nothing depends
      // on them until the tile is reduced, when they are turned into (ks, kpos, slots). A test
      // or conversion right after the load would make the warp wait for it there.
      struct MetaRaw {
        int32_t i;       // key position, gathered key row or block (-1: none)
        float ks;        // key scale (plain layout)
        uint32_t slots;  // block slots of the tile's tokens
      };
      auto meta_load = [&](int t, MetaRaw& r) {
        const int c = t * kTileM + m;
        r.i = -1;
        r.ks = 1.f;
        r.slots = 0u;
        if constexpr (C::GATHER) {
          if (c < x.nkeys && c < a.n_idx)
            r.i = a.key_idx[static_cast<int64_t>(x.b) * a.key_idx_stride + c];
        } else if constexpr (C::BLOCKS) {
          const int64_t e = static_cast<int64_t>(x.b) * a.key_blk_stride + t;
          if (c < x.nkeys) r.i = a.key_blk[e];
          if (a.key_blk_slot != nullptr) r.slots = static_cast<uint32_t>(a.key_blk_slot[e]);
        } else if (c < x.nkeys) {
          const int64_t kr = x.key_row0 + c;
          if (a.key_pos != nullptr) r.i = a.key_pos[kr];  // negative: an empty slot
          if (a.k_scale != nullptr) r.ks = a.k_scale[kr];
        }
      };
      auto meta_finish = [&](int t, const MetaRaw& r, float& ks, int64_t& kpos, uint32_t& slots) {
        const int c = t * kTileM + m;
        ks = 1.f;
        slots = r.slots;
        if constexpr (C::GATHER) {
          kpos = INT64_MAX;  // no key: never visible
          if (r.i >= 0 && r.i < a.S_valid) {
            kpos = r.i;
            if (a.k_scale != nullptr) ks = a.k_scale[x.key_row0 + r.i];
          }
        } else if constexpr (C::BLOCKS) {
          kpos = INT64_MAX;
          const int64_t p = static_cast<int64_t>(r.i) * kTileM + m;
          if (r.i >= 0 && p < a.S_valid) {
            kpos = p;
            if (a.k_scale != nullptr) ks = a.k_scale[x.key_row0 + p];
          }
        } else {
          kpos = c;
          ks = r.ks;
          if (c < x.nkeys && a.key_pos != nullptr) kpos = r.i < 0 ? INT64_MAX : r.i;
        }
      };
      // tile t of this range is the CTA's tile number g = gi_lo + (t - t_lo); it lands in
      // accumulator buffer g % ACC, and with BUF_SPLIT only the warpgroup g % EG reduces it
      const int64_t gi_lo = gi;
      gi += t_hi - t_lo;
      constexpr int TSTEP = C::BUF_SPLIT ? C::EG : 1;
      int t0 = t_lo;
      if (C::BUF_SPLIT) t0 += static_cast<int>(((grp - gi_lo) % C::EG + C::EG) % C::EG);
      MetaRaw raw_next;
      if (t0 < t_hi) meta_load(t0, raw_next);
      bool ok = true;
      for (int t = t0; t < t_hi; t += TSTEP) {
        const MetaRaw raw = raw_next;
        if (t + TSTEP < t_hi) meta_load(t + TSTEP, raw_next);
        float ks;
        int64_t kpos;
        uint32_t slots;
        meta_finish(t, raw, ks, kpos, slots);
        const int64_t g = gi_lo + (t - t_lo);
        const int acc = static_cast<int>(g % C::ACC);
        const uint32_t acc_phase = static_cast<uint32_t>((g / C::ACC) & 1);
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
        float2 part[C::TOKG][C::NP];
#pragma unroll
        for (int tt = 0; tt < C::TOKG; ++tt)
#pragma unroll
          for (int p = 0; p < C::NP; ++p) part[tt][p] = make_float2(0.f, 0.f);
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(lq * 32) << 16) +
                               static_cast<uint32_t>(acc * C::N + tok0 * C::H);
        // software pipeline: the next chunk's TMEM load is in flight while this one reduces
        float va[C::CW], vb[C::CW];
        tmem_ld_chunk<C::CW>(taddr, va);
        tmem_wait_ld();
        if (folded) {
#pragma unroll
          for (int ch = 0; ch < C::NCH; ++ch) {
            if (ch % 2 == 0) {
              if (ch + 1 < C::NCH) tmem_ld_chunk<C::CW>(taddr + (ch + 1) * C::CW, vb);
              reduce_chunk_folded<C>(va, ch * C::CW, part);
            } else {
              if (ch + 1 < C::NCH) tmem_ld_chunk<C::CW>(taddr + (ch + 1) * C::CW, va);
              reduce_chunk_folded<C>(vb, ch * C::CW, part);
            }
            if (ch + 1 < C::NCH) tmem_wait_ld();
          }
        } else {
#pragma unroll
          for (int ch = 0; ch < C::NCH; ++ch) {
            if (ch % 2 == 0) {
              if (ch + 1 < C::NCH) tmem_ld_chunk<C::CW>(taddr + (ch + 1) * C::CW, vb);
              reduce_chunk<C>(va, w_w, ch * C::CW, part);
            } else {
              if (ch + 1 < C::NCH) tmem_ld_chunk<C::CW>(taddr + (ch + 1) * C::CW, va);
              reduce_chunk<C>(vb, w_w, ch * C::CW, part);
            }
            if (ch + 1 < C::NCH) tmem_wait_ld();
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
#pragma unroll
        for (int tt = 0; tt < C::TOKG; ++tt) {
          const int r = rowg + tt;
          if (r < x.row_end) {
            float sc = 0.f;
#pragma unroll
            for (int p = 0; p < C::NP; ++p) sc += part[tt][p].x + part[tt][p].y;
            const bool vis = key_ok && kpos <= rpos[tt];
            const float out = vis ? (ks * tokf[tt]) * sc : -INFINITY;
            if constexpr (C::BLOCKS) {
              // with a slot table, tile t is block slots.byte[token] of the token's own list
              // (0xFF: not one of its blocks); without one, every token's slot is t
              int col = c;
              if (a.key_blk_slot != nullptr) {
                const uint32_t sl = (slots >> (8 * (tok0 + tt))) & 0xFFu;
                col = sl == 0xFFu ? -1 : static_cast<int>(sl) * kTileM + m;
              }
              if (col >= 0) store_score(a, static_cast<int64_t>(r) * a.score_ld + col, out);
            } else {
              store_score(a, static_cast<int64_t>(r) * a.score_ld + c, out);
            }
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
  kern<<<grid, C::THREADS, C::SMEM, s>>>(tm_q, tm_k, a);
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
  X(false, 32, 1, 128) X(true, 32, 1, 128)                                             \
  /* a few group queries per key batch (MTP windows): N = 2 or 4 tokens x 16 heads */  \
  X(false, 16, 2, 128) X(true, 16, 2, 128) X(false, 16, 4, 128) X(true, 16, 4, 128)

// Block-list configurations (HISA refinement): one decode row per key batch, or a group of
// score_tokens_per_tile(H) prefill rows scoring the union of their blocks.
#define ADX_BLOCK_CONFIGS(X) \
  X(false, 64, 1, 128) X(true, 64, 1, 128) X(false, 64, 4, 128) X(true, 64, 4, 128)

// tok: tokens per N tile; score_tokens_per_tile(H) (prefill), 1 (one query per key batch:
// decode and its bank refresh), or 2 / 4 with 16 heads (the group queries of an MTP window).
cudaError_t launch_score(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const ScoreArgs& a,
                         bool fp8, int H, int d, int tok, int grid, cudaStream_t s) {
  const bool gather = a.key_idx != nullptr;
  if (a.key_blk != nullptr) {
#define ADX_CASE(FP, HH, TT, DD)                                                        \
  if (fp8 == FP && H == HH && tok == TT && d == DD)                                     \
    return launch_cfg<Cfg<HH, TT, (FP ? DD : 2 * DD), FP, kKeysBlocks>>(tm_q, tm_k, a, grid, s);
    ADX_BLOCK_CONFIGS(ADX_CASE)
#undef ADX_CASE
    return cudaErrorNotSupported;
  }
#define ADX_CASE(FP, HH, TT, DD)                                                        \
  if (fp8 == FP && H == HH && tok == TT && d == DD)                                     \
    return gather ? launch_cfg<Cfg<HH, TT, (FP ? DD : 2 * DD), FP, kKeysGather>>(tm_q, tm_k, a, grid, s) \
                  : launch_cfg<Cfg<HH, TT, (FP ? DD : 2 * DD), FP>>(tm_q, tm_k, a, grid, s);
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

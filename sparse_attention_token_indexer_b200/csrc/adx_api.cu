// C ABI of the indexer library: argument validation, workspace layout, TMA descriptors and
// the launch sequence of each entry point. Every step of the computation runs in this
// library's kernels; this file only plans and launches them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/adx.h"
#include "adx_internal.h"

namespace adx {
namespace {

constexpr size_t kAlign = 256;
constexpr int64_t kSelectRegCapacity = 32768;  // longest row the register-resident select holds

// Optional instrumentation (adx_set_timing_events / adx_launch_count).
thread_local void* const* g_events = nullptr;
thread_local int g_n_events = 0;
std::atomic<long long> g_launches{0};

void mark(int i, cudaStream_t s) {
  if (g_events != nullptr && i < g_n_events && g_events[i] != nullptr)
    cudaEventRecord(static_cast<cudaEvent_t>(g_events[i]), s);
}

cudaError_t counted(cudaError_t e, int n = 1) {
  if (e == cudaSuccess) g_launches += n;
  return e;
}
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s per device-side wait
// Score matrices above this size are stored evict-first (twice the L2 of a B200)
constexpr double kStreamScoreBytes = 256.0 * (1 << 20);

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t ld_for(int64_t n) { return (n + kTileM - 1) / kTileM * kTileM; }

struct Carve {
  uint8_t* base;
  size_t off = 0;
  explicit Carve(void* p) : base(static_cast<uint8_t*>(p)) {}
  template <class T>
  T* take(size_t bytes) {
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += align_up(bytes, kAlign);
    return p;
  }
};

// ------------------------------------------------------------------------------------
// device properties and the driver's tensor-map encoder
// ------------------------------------------------------------------------------------
int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  static int cache[64] = {0};
  if (dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

// 2-D map over `rows` rows of `d` elements (1 or 2 bytes), 128-byte swizzled boxes of
// (128 bytes) x box_rows.
bool encode_rows(CUtensorMap* m, const void* base, bool one_byte, int d, int64_t rows,
                 int box_rows) {
  EncodeTiledFn enc = encoder();
  if (!enc || rows <= 0 || rows > INT32_MAX) return false;
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0) return false;
  const int esz = one_byte ? 1 : 2;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * esz};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, one_byte ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// ------------------------------------------------------------------------------------
// validation
// ------------------------------------------------------------------------------------
adx_status check_operands(const adx_operands* o, bool decode) {
  if (!o || !o->q || !o->w || !o->k) return ADX_EINVAL;
  if (o->T <= 0 || o->H <= 0 || o->d <= 0 || o->S <= 0) return ADX_EINVAL;
  if ((o->q_dtype != ADX_BF16 && o->q_dtype != ADX_E4M3) ||
      (o->k_dtype != ADX_BF16 && o->k_dtype != ADX_E4M3))
    return ADX_EINVAL;
  if ((o->q_dtype == ADX_E4M3) != (o->q_scale != nullptr)) return ADX_EINVAL;
  if ((o->k_dtype == ADX_E4M3) != (o->k_scale != nullptr)) return ADX_EINVAL;
  if (decode != (o->seq_len != nullptr)) return ADX_EINVAL;
  if (!decode && (o->q_pos0 < 0 || o->q_pos0 + o->T > o->S)) return ADX_EINVAL;
  if (o->q_dtype != o->k_dtype && !(decode && o->q_dtype == ADX_BF16 && o->k_dtype == ADX_E4M3))
    return ADX_EUNSUPPORTED;
  if (!score_config_supported(o->k_dtype == ADX_E4M3, o->H, o->d)) return ADX_EUNSUPPORTED;
  if (static_cast<int64_t>(o->T) * o->H > INT32_MAX) return ADX_EINVAL;
  if (decode && static_cast<int64_t>(o->T) * o->S > INT32_MAX) return ADX_EINVAL;
  return ADX_OK;
}

bool fp8_keys(const adx_operands* o) { return o->k_dtype == ADX_E4M3; }
int row_bytes(const adx_operands* o) { return o->d * (fp8_keys(o) ? 1 : 2); }

// split of a long row into segments for a two-stage select (few long rows)
void plan_split(int64_t rows, int64_t n, int K, int& n_seg, int& seg_len) {
  n_seg = 1;
  seg_len = static_cast<int>(std::min<int64_t>(n, INT32_MAX));
  const int sms = std::max(sm_count(), 1);
  if (rows >= sms || n < 8ll * K || n <= kWarpSelectMax) return;
  const int64_t want = (2ll * sms + rows - 1) / rows;
  const int64_t most = n / (4ll * K);
  // keep the second stage (n_seg * K candidates per row) inside the register-resident select,
  // and the segments too when possible
  const int64_t fit = std::max<int64_t>(2, kSelectRegCapacity / K);
  const int64_t need = (n + kSelectRegCapacity - 1) / kSelectRegCapacity;
  n_seg = static_cast<int>(std::max<int64_t>(need, std::min(std::min(want, most), fit)));
  if (n_seg == 1) return;
  seg_len = static_cast<int>(align_up((n + n_seg - 1) / n_seg, 4));
  n_seg = static_cast<int>((n + seg_len - 1) / seg_len);
}

// ------------------------------------------------------------------------------------
// query preparation: the scoring kernel reads prepared query rows (gate-folded where all
// gates of the row are >= 0, else as given; e4m3 with per-row scales for e4m3 keys)
// ------------------------------------------------------------------------------------
struct Prepared {
  const void* q = nullptr;
  const float* q_scale = nullptr;
  const int8_t* fold = nullptr;
};

size_t ws_prepare(const adx_operands* o, int64_t R) {
  const bool out8 = fp8_keys(o);
  return align_up(static_cast<size_t>(R) * o->H * o->d * (out8 ? 1 : 2), kAlign) +
         (out8 ? align_up(static_cast<size_t>(R) * 4, kAlign) : 0) +
         align_up(static_cast<size_t>(R), kAlign);
}

// R rows of q / q_scale / w starting at the given pointers.
adx_status prepare(const adx_operands* o, const void* q, const float* q_scale, const float* w,
                   int64_t R, Carve& cv, cudaStream_t s, Prepared& out,
                   int32_t* row_blk = nullptr) {
  const bool in8 = o->q_dtype == ADX_E4M3, out8 = fp8_keys(o);
  void* qo = cv.take<uint8_t>(static_cast<size_t>(R) * o->H * o->d * (out8 ? 1 : 2));
  float* so = out8 ? cv.take<float>(static_cast<size_t>(R) * 4) : nullptr;
  int8_t* fl = cv.take<int8_t>(static_cast<size_t>(R));
  RowBlocks rb;
  rb.out = row_blk;
  rb.q_pos0 = o->q_pos0;
  rb.seq_len = o->seq_len;
  if (counted(launch_prepare_q(q, q_scale, in8, out8, w, R, o->H, o->d, qo, so, fl, s, rb)) !=
      cudaSuccess)
    return ADX_ECUDA;
  out.q = qo;
  out.q_scale = so;
  out.fold = fl;
  return ADX_OK;
}

// ------------------------------------------------------------------------------------
// building blocks
// ------------------------------------------------------------------------------------
struct ScorePlan {
  ScoreArgs a{};
  bool fp8 = false;
  int H = 0, d = 0, tok = 0;
};

ScorePlan base_plan(const adx_operands* o, const Prepared& pq, int tok) {
  ScorePlan p;
  p.fp8 = fp8_keys(o);
  p.H = o->H;
  p.d = o->d;
  p.tok = tok;
  p.a.w = o->w;
  p.a.q_scale = pq.q_scale;
  p.a.k_scale = o->k_scale;
  p.a.fold_flag = pq.fold;
  p.a.timeout_ns = kTimeoutNs;
  return p;
}

// Chooses the key-chunk size and the persistent grid for a score launch.
void finish_plan(ScorePlan& p, int64_t max_tiles_per_block) {
  const int bps = score_blocks_per_sm(p.fp8, p.H, p.d, p.tok);
  const int grid_cap = std::max(1, sm_count() * std::max(bps, 1));
  const int64_t blocks = static_cast<int64_t>(p.a.row_blocks_per_batch) * p.a.n_batches;
  int64_t chunk = max_tiles_per_block;
  const int64_t want_items = 4ll * grid_cap;
  if (blocks * ((max_tiles_per_block + chunk - 1) / chunk) < want_items)
    chunk = std::max<int64_t>(8, (blocks * max_tiles_per_block + want_items - 1) / want_items);
  chunk = std::min<int64_t>(chunk, 32);
  chunk = std::max<int64_t>(1, std::min(chunk, max_tiles_per_block));
  p.a.chunk_tiles = static_cast<int>(chunk);
  p.a.chunks_per_block = static_cast<int>((max_tiles_per_block + chunk - 1) / chunk);
  p.a.n_items = static_cast<int>(blocks * p.a.chunks_per_block);
}

adx_status run_score(const ScorePlan& p, const void* q_codes, const void* keys, int64_t key_rows,
                     cudaStream_t s) {
  CUtensorMap tq, tk;
  const int n = p.tok * p.H;
  if (!encode_rows(&tq, q_codes, p.fp8, p.d, static_cast<int64_t>(p.a.R) * p.H, n))
    return ADX_EINVAL;
  // gathered keys (tile::gather4) need one-row boxes
  if (!encode_rows(&tk, keys, p.fp8, p.d, key_rows, p.a.key_idx ? 1 : kTileM)) return ADX_EINVAL;
  if (p.a.n_items <= 0) return ADX_OK;
  const int bps = score_blocks_per_sm(p.fp8, p.H, p.d, p.tok);
  const int grid = std::min<int64_t>(p.a.n_items, static_cast<int64_t>(sm_count()) * bps);
  if (grid <= 0) return ADX_EUNSUPPORTED;
  ScoreArgs a = p.a;
  // not in the block-list mode, whose rows are written block by block in slot order (plain
  // stores measured faster there)
  a.stream_scores = a.key_blk == nullptr &&
                    static_cast<double>(a.R) * static_cast<double>(a.score_ld) * 4.0 > kStreamScoreBytes;
  mark(0, s);
  const cudaError_t e = counted(launch_score(tq, tk, a, p.fp8, p.H, p.d, p.tok, grid, s));
  mark(1, s);
  if (e == cudaErrorNotSupported) return ADX_EUNSUPPORTED;
  return e == cudaSuccess ? ADX_OK : ADX_ECUDA;
}

size_t select_scratch_bytes(int64_t rows, int64_t n, int K) {
  if (select_cluster_ctas(rows, n, K, sm_count()) > 0) return 0;
  int n_seg, seg_len;
  plan_split(rows, n, K, n_seg, seg_len);
  if (n_seg == 1) return 0;
  const size_t c = static_cast<size_t>(rows) * n_seg * K;
  return align_up(c * 4, kAlign) * 2;
}

// Top-K per row of a score matrix. Few long rows go to the cluster select (one cluster of
// CTAs per row) when a cluster holds the row, else to a two-stage split.
adx_status run_select(SelectArgs a, int64_t n_max, Carve& cv, DeviceStatus* st, cudaStream_t s) {
  a.status = st;
  n_max = std::max<int64_t>(n_max, a.len_cap);
  const int ctas = select_cluster_ctas(a.rows, n_max, a.K, sm_count());
  if (ctas > 0) {
    a.n_seg = 1;
    a.seg_len = static_cast<int32_t>(std::min<int64_t>(n_max, INT32_MAX));
    mark(2, s);
    int nl = 0;
    const cudaError_t e0 = launch_select_cluster(a, ctas, s, &nl);
    const cudaError_t e = counted(e0, nl);
    mark(3, s);
    return e == cudaSuccess ? ADX_OK : ADX_ECUDA;
  }
  int n_seg, seg_len;
  plan_split(a.rows, n_max, a.K, n_seg, seg_len);
  mark(2, s);
  if (n_seg == 1) {
    a.n_seg = 1;
    a.seg_len = static_cast<int32_t>(std::min<int64_t>(n_max, INT32_MAX));
    int nl = 0;
    const cudaError_t e0 = launch_select(a, s, &nl);
    const cudaError_t e = counted(e0, nl);
    mark(3, s);
    return e == cudaSuccess ? ADX_OK : ADX_ECUDA;
  }
  const size_t c = static_cast<size_t>(a.rows) * n_seg * a.K;
  float* cv_val = cv.take<float>(c * 4);
  int32_t* cv_idx = cv.take<int32_t>(c * 4);
  SelectArgs s1 = a;
  s1.n_seg = n_seg;
  s1.seg_len = seg_len;
  s1.idx_map = nullptr;
  s1.out_idx = cv_idx;
  s1.out_val = cv_val;
  s1.out_ld = a.K;
  int nl = 0;
  const cudaError_t e1 = launch_select(s1, s, &nl);
  if (counted(e1, nl) != cudaSuccess) return ADX_ECUDA;
  SelectArgs s2 = a;
  s2.vals = cv_val;
  s2.in_idx = cv_idx;
  s2.ld = static_cast<int64_t>(n_seg) * a.K;
  s2.len_mode = 0;
  s2.len_fixed = static_cast<int32_t>(s2.ld);
  s2.len_cap = s2.len_fixed;
  s2.n_seg = 1;
  s2.seg_len = s2.len_fixed;
  // candidates beyond what one CTA holds in registers: one cluster per row, when one holds them
  const int ctas2 = s2.len_fixed > kSelectRegCapacity
                        ? select_cluster_ctas(s2.rows, s2.len_fixed, s2.K, sm_count(), true)
                        : 0;
  const cudaError_t e2 =
      ctas2 > 0 ? launch_select_cluster(s2, ctas2, s, &nl) : launch_select(s2, s, &nl);
  const cudaError_t e = counted(e2, nl);
  mark(3, s);
  return e == cudaSuccess ? ADX_OK : ADX_ECUDA;
}

// ---- flat prefill ------------------------------------------------------------------
size_t ws_flat(const adx_operands* o, int K, bool scores_external) {
  size_t b = kStatusBytes + ws_prepare(o, o->T);
  if (!scores_external) b += align_up(static_cast<size_t>(o->T) * ld_for(o->S) * 4, kAlign);
  b += select_scratch_bytes(o->T, o->S, K);
  return b;
}

adx_status run_flat(const adx_operands* o, int K, int32_t* topk_idx, float* topk_score,
                    float* scores_ext, int64_t scores_ld, Carve& cv, DeviceStatus* st,
                    cudaStream_t s) {
  Prepared pq;
  adx_status r = prepare(o, o->q, o->q_scale, o->w, o->T, cv, s, pq);
  if (r != ADX_OK) return r;
  const int64_t ld = scores_ext ? scores_ld : ld_for(o->S);
  float* scores = scores_ext ? scores_ext : cv.take<float>(static_cast<size_t>(o->T) * ld * 4);
  ScorePlan p = base_plan(o, pq, score_tokens_per_tile(o->H));
  ScoreArgs& a = p.a;
  a.scores = scores;
  a.score_ld = ld;
  a.pos_base = o->q_pos0;
  a.pos_step = 1;
  a.R = o->T;
  a.rows_per_batch = o->T;
  a.n_batches = 1;
  a.keys_per_batch = o->S;
  a.row_blocks_per_batch = (o->T + p.tok - 1) / p.tok;
  a.reverse_order = 1;
  a.status = st;
  const int64_t max_keys = std::min<int64_t>(o->S, o->q_pos0 + o->T);
  finish_plan(p, (max_keys + kTileM - 1) / kTileM);
  if ((r = run_score(p, pq.q, o->k, o->S, s)) != ADX_OK) return r;
  SelectArgs sa{};
  sa.vals = scores;
  sa.ld = ld;
  sa.rows_per_batch = o->T;
  sa.len_mode = 1;
  sa.len_cap = static_cast<int32_t>(max_keys);  // no row is longer: picks the select class
  sa.pos_base = o->q_pos0;
  sa.pos_step = 1;
  sa.K = K;
  sa.out_idx = topk_idx;
  sa.out_val = topk_score;
  sa.out_ld = K;
  sa.rows = o->T;
  return run_select(sa, max_keys, cv, st, s);
}

// ---- decode-layout scoring (one query per key cache) --------------------------------
ScorePlan rowwise_plan(const adx_operands* o, const Prepared& pq, float* scores, int64_t ld) {
  ScorePlan p = base_plan(o, pq, 1);
  ScoreArgs& a = p.a;
  a.seq_len = o->seq_len;
  a.scores = scores;
  a.score_ld = ld;
  a.R = o->T;
  a.rows_per_batch = 1;
  a.n_batches = o->T;
  a.key_batch_stride = o->S;
  a.keys_per_batch = o->S;
  a.row_blocks_per_batch = 1;
  return p;
}

size_t ws_decode(const adx_operands* o, int K) {
  return kStatusBytes + ws_prepare(o, o->T) +
         align_up(static_cast<size_t>(o->T) * ld_for(o->S) * 4, kAlign) +
         select_scratch_bytes(o->T, o->S, K);
}

// ---- group bank ---------------------------------------------------------------------
struct BankShape {
  int bank_k, post_count, post_start_off, width;
  int64_t scan_pos_off;  // scan row position = anchor + scan_pos_off
};

BankShape bank_shape(int B, int G, int mode) {
  BankShape b{};
  if (mode == ADX_BANK_PAPER) {
    b.bank_k = B;
    b.post_count = G - 1;
    b.post_start_off = 1;
    b.scan_pos_off = 0;
  } else {
    b.bank_k = B - G;
    b.post_count = G;
    b.post_start_off = 0;
    b.scan_pos_off = -1;
  }
  b.width = b.bank_k + b.post_count;
  return b;
}

adx_status check_bank_args(const adx_operands* o, int G, int B, int mode) {
  if (G <= 0 || B <= 0) return ADX_EINVAL;
  if (mode != ADX_BANK_PAPER && mode != ADX_BANK_WINDOW) return ADX_EINVAL;
  if (mode == ADX_BANK_WINDOW && B <= G) return ADX_EINVAL;
  if (o->seq_len != nullptr && mode != ADX_BANK_PAPER) return ADX_EUNSUPPORTED;
  return ADX_OK;
}

size_t ws_bank(const adx_operands* o, int G, int B, int mode) {
  const BankShape bs = bank_shape(B, G, mode);
  return kStatusBytes + ws_prepare(o, o->T) +
         align_up(static_cast<size_t>(o->T) * ld_for(o->S) * 4, kAlign) +
         select_scratch_bytes(o->T, o->S, bs.bank_k);
}

// ---- refine -------------------------------------------------------------------------
size_t ws_refine(const adx_operands* o, int G, int B, int mode, int K) {
  const BankShape bs = bank_shape(B, G, mode);
  const int64_t bcp = ld_for(bs.width);
  const bool dec = o->seq_len != nullptr;
  const int64_t ng = dec ? o->T : o->T / G;
  const int64_t rows = dec ? o->T : ng * G;
  size_t b = kStatusBytes + ws_prepare(o, rows);
  if (!dec) {  // packed candidate keys, scales, positions (decode gathers them instead)
    b += align_up(static_cast<size_t>(ng) * bcp * row_bytes(o), kAlign);
    b += align_up(static_cast<size_t>(ng) * bcp * 4, kAlign) * 2;
  }
  b += align_up(static_cast<size_t>(rows) * bcp * 4, kAlign);             // scores
  b += select_scratch_bytes(rows, bcp, K);
  if (!dec && rows < o->T) {
    adx_operands tail = *o;
    tail.T = static_cast<int32_t>(o->T - rows);
    b += ws_flat(&tail, K, false) - kStatusBytes;
  }
  return b;
}

// ---- decode refinement over a packed bank ----------------------------------------------
size_t ws_refine_packed(const adx_operands* o, int G, int B, int K) {
  const int64_t W = static_cast<int64_t>(B) + G - 1;
  return kStatusBytes + ws_prepare(o, o->T) +
         align_up(static_cast<size_t>(o->T) * ld_for(W) * 4, kAlign) +
         select_scratch_bytes(o->T, W, K);
}

adx_status check_packed(const adx_operands* o, int G, int B) {
  adx_status r = check_operands(o, true);
  if (r != ADX_OK) return r;
  if (G <= 0 || B <= 0 || static_cast<int64_t>(B) + G - 1 > INT32_MAX / 2) return ADX_EINVAL;
  if (static_cast<int64_t>(o->T) * (static_cast<int64_t>(B) + G - 1) > INT32_MAX)
    return ADX_EINVAL;
  return ADX_OK;
}

// ---- flat prefill from host buffers ---------------------------------------------------
// Copy engines of a device: two non-blocking streams (host to device, device to host) and the
// events that chain a chunk's copy-in, indexing and copy-out. Created on first use and kept.
constexpr int kHostMaxChunks = 64;
constexpr int kMaxDevices = 64;
struct CopyEngines {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t in[kHostMaxChunks], done[kHostMaxChunks], out;
  bool ready = false;
};
std::mutex g_copy_mutex;
CopyEngines g_copy[kMaxDevices];

adx_status copy_engines(CopyEngines** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ADX_ECUDA;
  std::lock_guard<std::mutex> lock(g_copy_mutex);
  CopyEngines& c = g_copy[dev];
  if (!c.ready) {
    if (cudaStreamCreateWithFlags(&c.h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&c.d2h, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.out, cudaEventDisableTiming) != cudaSuccess)
      return ADX_ECUDA;
    for (int i = 0; i < kHostMaxChunks; ++i)
      if (cudaEventCreateWithFlags(&c.in[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&c.done[i], cudaEventDisableTiming) != cudaSuccess)
        return ADX_ECUDA;
    c.ready = true;
  }
  *out = &c;
  return ADX_OK;
}

struct HostLayout {
  size_t q_row, k_row;  // bytes of a query row (all heads) and of a key row
  int64_t C, chunks;
};

bool host_layout(const adx_operands* o, int C, HostLayout& h) {
  if (C <= 0) return false;
  h.q_row = static_cast<size_t>(o->H) * o->d * (o->q_dtype == ADX_E4M3 ? 1 : 2);
  h.k_row = static_cast<size_t>(o->d) * (o->k_dtype == ADX_E4M3 ? 1 : 2);
  h.C = C;
  h.chunks = (o->T + C - 1) / C;
  return h.chunks <= kHostMaxChunks;
}

size_t ws_prefill_host(const adx_operands* o, int K, const HostLayout& h) {
  const size_t T = o->T, S = o->S;
  size_t b = kStatusBytes;
  b += align_up(T * h.q_row, kAlign) + (o->q_scale ? align_up(T * 4, kAlign) : 0) +
       align_up(T * o->H * 4, kAlign);
  b += align_up(S * h.k_row, kAlign) + (o->k_scale ? align_up(S * 4, kAlign) : 0);
  b += align_up(T * K * 4, kAlign) * 2;  // indices, scores
  adx_operands chunk = *o;
  chunk.T = static_cast<int32_t>(std::min<int64_t>(h.C, o->T));
  return b + ws_flat(&chunk, K, false) - kStatusBytes;
}

// ---- MTP target verification ----------------------------------------------------------
struct MtpShape {
  int64_t Bs, ng, width, bcp;
  int gps;
};

// Validates an MTP call and builds the group operand set over full's keys.
adx_status mtp_check(const adx_operands* full, const adx_operands* grp, int m, int G, int P,
                     int K, MtpShape& sh, adx_operands& gops) {
  if (!full || !grp || !full->seq_len) return ADX_EINVAL;
  adx_status r = check_operands(full, true);
  if (r != ADX_OK) return r;
  if (m <= 0 || m > 64 || G < 4 || m % G != 0 || P <= 0 || K <= 0) return ADX_EINVAL;
  if (full->T % m != 0) return ADX_EINVAL;
  sh.Bs = full->T / m;
  sh.gps = m / G;
  sh.ng = sh.Bs * sh.gps;
  sh.width = static_cast<int64_t>(P) + m - 1;
  sh.bcp = ld_for(sh.width);
  if (sh.ng * sh.width > INT32_MAX || sh.Bs * full->S > INT32_MAX) return ADX_EINVAL;
  gops = *full;
  gops.q_dtype = grp->q_dtype;
  gops.q = grp->q;
  gops.q_scale = grp->q_scale;
  gops.w = grp->w;
  gops.H = grp->H;
  gops.T = static_cast<int32_t>(sh.ng);
  if (grp->d != full->d || grp->T != sh.ng) return ADX_EINVAL;
  return check_operands(&gops, true);
}

size_t ws_mtp(const adx_operands* full, const adx_operands* gops, const MtpShape& sh, int m,
              int P, int K) {
  const int64_t R = sh.Bs * m;
  size_t b = kStatusBytes;
  b += align_up(static_cast<size_t>(R) * 4, kAlign) + align_up(static_cast<size_t>(sh.ng) * 4, kAlign);
  b += align_up(static_cast<size_t>(sh.ng) * sh.width * 4, kAlign);  // candidate rows
  b += ws_prepare(gops, sh.ng) +
       align_up(static_cast<size_t>(sh.ng) * ld_for(full->S) * 4, kAlign) +  // bank scan scores
       select_scratch_bytes(sh.ng, full->S, P);
  b += ws_prepare(full, R) + align_up(static_cast<size_t>(R) * sh.bcp * 4, kAlign) +
       select_scratch_bytes(R, sh.bcp, K);
  b += align_up(static_cast<size_t>(sh.ng) * sh.bcp * row_bytes(full), kAlign) +  // packed keys
       align_up(static_cast<size_t>(sh.ng) * sh.bcp * 4, kAlign) * 2;            // scales, positions
  return b;
}

// ---- HISA (block filter, then token refinement) ------------------------------------
constexpr int kHisaShift = 7;  // log2 of the block size (one MMA tile of keys)
static_assert((1 << kHisaShift) == kTileM, "a HISA block is one key tile");

constexpr int kHisaHeads = 64;  // the block-list scoring configurations
// prefill rows per union group (the rows of one N = 256 tile)
constexpr int kHisaGroup = 4;

int64_t hisa_nbmax(const adx_operands* o) { return (o->S + kTileM - 1) / kTileM; }

adx_status hisa_check(const adx_operands* o, int32_t n_blocks, int32_t K) {
  const adx_status r = check_operands(o, o != nullptr && o->seq_len != nullptr);
  if (r != ADX_OK) return r;
  if (n_blocks < 2 || n_blocks > 255 || K <= 0 || K > n_blocks * kTileM) return ADX_EINVAL;
  if (o->H != kHisaHeads) return ADX_EUNSUPPORTED;
  if (static_cast<int64_t>(o->T) * n_blocks * kTileM > INT32_MAX) return ADX_EINVAL;
  return ADX_OK;
}

// bf16 queries for the block pass, prepared apart when the keys are e4m3 (the block keys are
// bf16 in both formats)
size_t ws_prepare_bf16(const adx_operands* o, int64_t R) {
  return align_up(static_cast<size_t>(R) * o->H * o->d * 2, kAlign) +
         align_up(static_cast<size_t>(R), kAlign);
}

size_t ws_hisa(const adx_operands* o, int32_t n_blocks, int32_t K, bool blocks_external) {
  const int64_t T = o->T, nbmax = hisa_nbmax(o), nc = static_cast<int64_t>(n_blocks) * kTileM;
  size_t b = kStatusBytes + ws_prepare(o, T);
  if (fp8_keys(o)) b += ws_prepare_bf16(o, T);
  b += align_up(static_cast<size_t>(T) * 4, kAlign);                         // row blocks
  b += align_up(static_cast<size_t>(T) * ld_for(nbmax) * 4, kAlign);         // block scores
  if (!blocks_external) b += align_up(static_cast<size_t>(T) * n_blocks * 4, kAlign);
  b += align_up(static_cast<size_t>(T) * nc * 4, kAlign);                    // token scores
  if (o->seq_len == nullptr) {  // prefill: block unions of groups of rows
    const size_t ng = static_cast<size_t>((T + kHisaGroup - 1) / kHisaGroup);
    const size_t width = static_cast<size_t>(kHisaGroup) * n_blocks;
    b += 2 * align_up(ng * width * 4, kAlign) + align_up(ng * 4, kAlign);
  }
  b += select_scratch_bytes(T, nbmax, n_blocks) + select_scratch_bytes(T, nc, K);
  return b;
}

}  // namespace

adx_status check_prefill_args(const adx_operands* o, int32_t K) {
  const adx_status r = check_operands(o, false);
  if (r != ADX_OK) return r;
  return K <= 0 ? ADX_EINVAL : ADX_OK;
}

void add_launches(int n) { g_launches += n; }

}  // namespace adx

using namespace adx;

extern "C" {

int32_t adx_abi_version(void) { return ADX_ABI_VERSION; }

void adx_set_timing_events(void* const* events, int32_t n) {
  g_events = (events != nullptr && n > 0) ? events : nullptr;
  g_n_events = g_events ? n : 0;
}

int64_t adx_launch_count(void) { return g_launches.load(); }

int32_t adx_bank_width(int32_t B, int32_t G, int32_t mode) {
  if (B <= 0 || G <= 0 || (mode != ADX_BANK_PAPER && mode != ADX_BANK_WINDOW)) return 0;
  if (mode == ADX_BANK_WINDOW && B <= G) return 0;
  return bank_shape(B, G, mode).width;
}

const char* adx_status_string(adx_status s) {
  switch (s) {
    case ADX_OK: return "ok";
    case ADX_EINVAL: return "invalid argument";
    case ADX_EUNSUPPORTED: return "unsupported shape or dtype";
    case ADX_EWORKSPACE: return "workspace too small";
    case ADX_ECUDA: return "CUDA error";
    case ADX_EOVERFLOW: return "internal buffer overflow";
    case ADX_ETIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

size_t adx_workspace_size(int32_t op, const adx_operands* ops, int32_t K, int32_t B, int32_t G,
                          int32_t mode) {
  if (!ops) return 0;
  switch (op) {
    case ADX_OP_PREFILL:
      if (K <= 0 || check_operands(ops, false) != ADX_OK) return 0;
      return ws_flat(ops, K, false);
    case ADX_OP_DECODE:
      if (K <= 0 || check_operands(ops, true) != ADX_OK) return 0;
      return ws_decode(ops, K);
    case ADX_OP_GROUP_BANK:
      if (check_operands(ops, ops->seq_len != nullptr) != ADX_OK ||
          check_bank_args(ops, G, B, mode) != ADX_OK)
        return 0;
      return ws_bank(ops, G, B, mode);
    case ADX_OP_PREFILL_HOST: {
      HostLayout h;
      if (K <= 0 || check_operands(ops, false) != ADX_OK || !host_layout(ops, B, h)) return 0;
      return ws_prefill_host(ops, K, h);
    }
    case ADX_OP_BANK_REFINE:
      if (K <= 0 || check_operands(ops, ops->seq_len != nullptr) != ADX_OK ||
          check_bank_args(ops, G, B, mode) != ADX_OK)
        return 0;
      return ws_refine(ops, G, B, mode, K);
    case ADX_OP_BANK_REFINE_PACKED:
      if (K <= 0 || mode != ADX_BANK_PAPER || check_packed(ops, G, B) != ADX_OK) return 0;
      return ws_refine_packed(ops, G, B, K);
    default:
      return 0;
  }
}

adx_status adx_index_prefill(const adx_operands* o, int32_t K, int32_t* topk_idx,
                             float* topk_score, float* scores_out, int64_t scores_ld, void* ws,
                             size_t ws_bytes, void* stream) {
  adx_status r = check_operands(o, false);
  if (r != ADX_OK) return r;
  if (K <= 0 || !topk_idx || !ws) return ADX_EINVAL;
  // score rows are read with 16-byte vector loads
  if (scores_out && (scores_ld < ld_for(o->S) || scores_ld % 4 != 0 ||
                     (reinterpret_cast<uintptr_t>(scores_out) & 15) != 0))
    return ADX_EINVAL;
  if (ws_bytes < ws_flat(o, K, scores_out != nullptr)) return ADX_EWORKSPACE;
  Carve cv(ws);
  DeviceStatus* st = cv.take<DeviceStatus>(kStatusBytes);
  return run_flat(o, K, topk_idx, topk_score, scores_out, scores_ld, cv, st,
                  static_cast<cudaStream_t>(stream));
}

adx_status adx_index_decode(const adx_operands* o, int32_t K, int32_t* topk_idx,
                            float* topk_score, void* ws, size_t ws_bytes, void* stream) {
  adx_status r = check_operands(o, true);
  if (r != ADX_OK) return r;
  if (K <= 0 || !topk_idx || !ws) return ADX_EINVAL;
  if (ws_bytes < ws_decode(o, K)) return ADX_EWORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carve cv(ws);
  DeviceStatus* st = cv.take<DeviceStatus>(kStatusBytes);
  Prepared pq;
  if ((r = prepare(o, o->q, o->q_scale, o->w, o->T, cv, s, pq)) != ADX_OK) return r;
  const int64_t ld = ld_for(o->S);
  float* scores = cv.take<float>(static_cast<size_t>(o->T) * ld * 4);
  ScorePlan p = rowwise_plan(o, pq, scores, ld);
  p.a.status = st;
  finish_plan(p, (o->S + kTileM - 1) / kTileM);
  if ((r = run_score(p, pq.q, o->k, static_cast<int64_t>(o->T) * o->S, s)) != ADX_OK) return r;
  SelectArgs sa{};
  sa.vals = scores;
  sa.ld = ld;
  sa.rows_per_batch = 1;
  sa.len_mode = 2;
  sa.len_cap = o->S;
  sa.seq_len = o->seq_len;
  sa.K = K;
  sa.out_idx = topk_idx;
  sa.out_val = topk_score;
  sa.out_ld = K;
  sa.rows = o->T;
  return run_select(sa, o->S, cv, st, s);
}

adx_status adx_group_bank(const adx_operands* o, int32_t G, int32_t B, int32_t mode,
                          int32_t* bank_idx, void* ws, size_t ws_bytes, void* stream) {
  if (!o) return ADX_EINVAL;
  const bool dec = o->seq_len != nullptr;
  adx_status r = check_operands(o, dec);
  if (r != ADX_OK) return r;
  if ((r = check_bank_args(o, G, B, mode)) != ADX_OK) return r;
  if (!bank_idx || !ws) return ADX_EINVAL;
  if (ws_bytes < ws_bank(o, G, B, mode)) return ADX_EWORKSPACE;
  if (!dec && o->q_pos0 + static_cast<int64_t>(o->T - 1) * G >= o->S) return ADX_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const BankShape bs = bank_shape(B, G, mode);
  Carve cv(ws);
  DeviceStatus* st = cv.take<DeviceStatus>(kStatusBytes);
  Prepared pq;
  if ((r = prepare(o, o->q, o->q_scale, o->w, o->T, cv, s, pq)) != ADX_OK) return r;
  const int64_t ld = ld_for(o->S);
  float* scores = cv.take<float>(static_cast<size_t>(o->T) * ld * 4);
  SelectArgs sa{};
  if (dec) {
    ScorePlan p = rowwise_plan(o, pq, scores, ld);
    p.a.status = st;
    finish_plan(p, (o->S + kTileM - 1) / kTileM);
    if ((r = run_score(p, pq.q, o->k, static_cast<int64_t>(o->T) * o->S, s)) != ADX_OK) return r;
    sa.len_mode = 2;
    sa.seq_len = o->seq_len;
  } else {
    ScorePlan p = base_plan(o, pq, score_tokens_per_tile(o->H));
    ScoreArgs& a = p.a;
    a.scores = scores;
    a.score_ld = ld;
    a.pos_base = o->q_pos0 + bs.scan_pos_off;
    a.pos_step = G;
    a.R = o->T;
    a.rows_per_batch = o->T;
    a.n_batches = 1;
    a.keys_per_batch = o->S;
    a.row_blocks_per_batch = (o->T + p.tok - 1) / p.tok;
    a.reverse_order = 1;
    a.status = st;
    const int64_t last = o->q_pos0 + bs.scan_pos_off + static_cast<int64_t>(o->T - 1) * G;
    const int64_t max_keys = std::max<int64_t>(0, std::min<int64_t>(o->S, last + 1));
    finish_plan(p, std::max<int64_t>(1, (max_keys + kTileM - 1) / kTileM));
    if ((r = run_score(p, pq.q, o->k, o->S, s)) != ADX_OK) return r;
    sa.len_mode = 1;
    sa.pos_base = o->q_pos0 + bs.scan_pos_off;
    sa.pos_step = G;
  }
  sa.vals = scores;
  sa.ld = ld;
  sa.rows_per_batch = 1;
  sa.len_cap = o->S;
  sa.K = bs.bank_k;
  sa.out_idx = bank_idx;
  sa.out_ld = bs.width;
  sa.rows = o->T;
  if ((r = run_select(sa, o->S, cv, st, s)) != ADX_OK) return r;
  if (counted(launch_fill_post_anchor(bank_idx, o->T, bs.width, bs.bank_k, bs.post_count,
                                      o->q_pos0, G, o->seq_len, bs.post_start_off, s)) !=
      cudaSuccess)
    return ADX_ECUDA;
  return ADX_OK;
}

adx_status adx_pack_bank_keys(const adx_operands* o, int32_t G, int32_t B,
                              const int32_t* bank_idx, void* bank_keys, float* bank_kscale,
                              void* stream) {
  adx_status r = check_packed(o, G, B);
  if (r != ADX_OK) return r;
  if (!bank_idx || !bank_keys || fp8_keys(o) != (bank_kscale != nullptr)) return ADX_EINVAL;
  if (reinterpret_cast<uintptr_t>(bank_keys) % 16 != 0) return ADX_EINVAL;
  const int32_t W = B + G - 1;
  return counted(launch_pack_candidates(o->k, o->k_scale, o->S, 1, 1, o->S, bank_idx, o->T, W, W,
                                        row_bytes(o), bank_keys, bank_kscale, nullptr,
                                        static_cast<cudaStream_t>(stream))) == cudaSuccess
             ? ADX_OK
             : ADX_ECUDA;
}

adx_status adx_bank_refine_packed(const adx_operands* o, int32_t G, int32_t B,
                                  const int32_t* bank_idx, void* bank_keys, float* bank_kscale,
                                  int32_t K, int32_t* topk_idx, float* topk_score, void* ws,
                                  size_t ws_bytes, void* stream) {
  adx_status r = check_packed(o, G, B);
  if (r != ADX_OK) return r;
  if (K <= 0 || !bank_idx || !bank_keys || !topk_idx || !ws ||
      fp8_keys(o) != (bank_kscale != nullptr))
    return ADX_EINVAL;
  if (reinterpret_cast<uintptr_t>(bank_keys) % 16 != 0) return ADX_EINVAL;
  if (ws_bytes < ws_refine_packed(o, G, B, K)) return ADX_EWORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int32_t W = B + G - 1;
  const int64_t ld = ld_for(W);
  Carve cv(ws);
  DeviceStatus* st = cv.take<DeviceStatus>(kStatusBytes);
  Prepared pq;
  if ((r = prepare(o, o->q, o->q_scale, o->w, o->T, cv, s, pq)) != ADX_OK) return r;
  // the post-anchor keys this step sees, from the cache into their packed slots
  if (counted(launch_refresh_post(o->k, o->k_scale, o->S, o->seq_len, bank_idx, o->T, W, B,
                                  row_bytes(o), bank_keys, bank_kscale, s)) != cudaSuccess)
    return ADX_ECUDA;
  float* scores = cv.take<float>(static_cast<size_t>(o->T) * ld * 4);
  ScorePlan p = rowwise_plan(o, pq, scores, ld);
  p.a.key_batch_stride = W;  // row t streams slots [t W, t W + W) of the packed bank
  p.a.keys_per_batch = W;
  p.a.key_pos = bank_idx;
  p.a.k_scale = bank_kscale;
  p.a.status = st;
  finish_plan(p, ld / kTileM);
  if ((r = run_score(p, pq.q, bank_keys, static_cast<int64_t>(o->T) * W, s)) != ADX_OK) return r;
  SelectArgs sa{};
  sa.vals = scores;
  sa.ld = ld;
  sa.idx_map = bank_idx;
  sa.map_stride = W;
  sa.rows_per_batch = 1;
  sa.len_mode = 0;
  sa.len_fixed = W;
  sa.len_cap = W;
  sa.K = K;
  sa.out_idx = topk_idx;
  sa.out_val = topk_score;
  sa.out_ld = K;
  sa.rows = o->T;
  return run_select(sa, W, cv, st, s);
}

adx_status adx_bank_refine(const adx_operands* o, int32_t G, int32_t B, int32_t mode,
                           const int32_t* bank_idx, int32_t K, int32_t* topk_idx,
                           float* topk_score, void* ws, size_t ws_bytes, void* stream) {
  if (!o) return ADX_EINVAL;
  const bool dec = o->seq_len != nullptr;
  adx_status r = check_operands(o, dec);
  if (r != ADX_OK) return r;
  if ((r = check_bank_args(o, G, B, mode)) != ADX_OK) return r;
  if (K <= 0 || !bank_idx || !topk_idx || !ws) return ADX_EINVAL;
  if (ws_bytes < ws_refine(o, G, B, mode, K)) return ADX_EWORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const BankShape bs = bank_shape(B, G, mode);
  const int64_t bcp = ld_for(bs.width);
  const int64_t ng = dec ? o->T : o->T / G;
  const int64_t rows = dec ? o->T : ng * G;
  if (ng * bcp > INT32_MAX) return ADX_EINVAL;
  Carve cv(ws);
  DeviceStatus* st = cv.take<DeviceStatus>(kStatusBytes);
  if (rows > 0) {
    Prepared pq;
    if ((r = prepare(o, o->q, o->q_scale, o->w, rows, cv, s, pq)) != ADX_OK) return r;
    float* scores = cv.take<float>(static_cast<size_t>(rows) * bcp * 4);
    ScorePlan p;
    const void* keys = o->k;
    int64_t key_rows = 0;
    const int32_t* slot_pos = bank_idx;  // candidate slot -> key position, for the select
    int64_t slot_stride = bs.width;
    if (dec) {
      // one query per group: its candidate keys are gathered straight from its own
      // sequence (tile::gather4), slot c of sequence g at position bank_idx[g, c]
      p = rowwise_plan(o, pq, scores, bcp);
      p.a.key_idx = bank_idx;
      p.a.key_idx_stride = bs.width;
      p.a.n_idx = bs.width;
      p.a.S_valid = o->S;
      key_rows = static_cast<int64_t>(o->T) * o->S;
    } else {
      // G queries share a group's candidates: pack them once into contiguous rows, which
      // every row block of the group then streams with whole-tile loads
      const int rb = row_bytes(o);
      uint8_t* packed = cv.take<uint8_t>(static_cast<size_t>(ng) * bcp * rb);
      float* pscale = cv.take<float>(static_cast<size_t>(ng) * bcp * 4);
      int32_t* ppos = cv.take<int32_t>(static_cast<size_t>(ng) * bcp * 4);
      if (counted(launch_pack_candidates(o->k, o->k_scale, o->S, 0, 1, o->S, bank_idx,
                                         static_cast<int32_t>(ng), bs.width,
                                         static_cast<int32_t>(bcp), rb, packed,
                                         fp8_keys(o) ? pscale : nullptr, ppos, s)) != cudaSuccess)
        return ADX_ECUDA;
      p = base_plan(o, pq, score_tokens_per_tile(o->H));
      p.a.pos_base = o->q_pos0;
      p.a.pos_step = 1;
      p.a.R = static_cast<int32_t>(rows);
      p.a.rows_per_batch = G;
      p.a.n_batches = static_cast<int32_t>(ng);
      p.a.row_blocks_per_batch = (G + p.tok - 1) / p.tok;
      p.a.round_robin = 1;  // a group's row blocks run together and share its packed keys
      p.a.scores = scores;
      p.a.score_ld = bcp;
      p.a.k_scale = fp8_keys(o) ? pscale : nullptr;
      p.a.key_pos = ppos;
      keys = packed;
      key_rows = ng * bcp;
      slot_pos = ppos;
      slot_stride = bcp;
    }
    p.a.key_batch_stride = dec ? o->S : bcp;
    p.a.keys_per_batch = static_cast<int32_t>(bcp);
    p.a.status = st;
    finish_plan(p, bcp / kTileM);
    if ((r = run_score(p, pq.q, keys, key_rows, s)) != ADX_OK) return r;
    SelectArgs sa{};
    sa.vals = scores;
    sa.ld = bcp;
    sa.idx_map = slot_pos;
    sa.map_stride = slot_stride;
    sa.rows_per_batch = dec ? 1 : G;
    sa.len_mode = 0;
    sa.len_fixed = static_cast<int32_t>(bcp);
    sa.len_cap = static_cast<int32_t>(bcp);
    sa.K = K;
    sa.out_idx = topk_idx;
    sa.out_val = topk_score;
    sa.out_ld = K;
    sa.rows = static_cast<int32_t>(rows);
    if ((r = run_select(sa, bcp, cv, st, s)) != ADX_OK) return r;
  }
  if (!dec && rows < o->T) {
    // incomplete trailing group: the plain indexer on those rows
    adx_operands tail = *o;
    tail.T = static_cast<int32_t>(o->T - rows);
    tail.q = static_cast<const uint8_t*>(o->q) +
             rows * o->H * o->d * (o->q_dtype == ADX_E4M3 ? 1 : 2);
    tail.q_scale = o->q_scale ? o->q_scale + rows : nullptr;
    tail.w = o->w + rows * o->H;
    tail.q_pos0 = o->q_pos0 + rows;
    return run_flat(&tail, K, topk_idx + rows * K, topk_score ? topk_score + rows * K : nullptr,
                    nullptr, 0, cv, st, s);
  }
  return ADX_OK;
}

size_t adx_mtp_workspace_size(const adx_operands* full, const adx_operands* grp, int32_t m,
                              int32_t G, int32_t P, int32_t K) {
  MtpShape sh;
  adx_operands gops;
  if (mtp_check(full, grp, m, G, P, K, sh, gops) != ADX_OK) return 0;
  return ws_mtp(full, &gops, sh, m, P, K);
}

adx_status adx_index_prefill_host(const adx_operands* o, int32_t K, int32_t rows_per_chunk,
                                  int32_t* topk_idx, float* topk_score, void* ws,
                                  size_t ws_bytes, void* stream) {
  adx_status r = check_operands(o, false);
  if (r != ADX_OK) return r;
  HostLayout h;
  if (K <= 0 || !topk_idx || !ws || !host_layout(o, rows_per_chunk, h)) return ADX_EINVAL;
  if (ws_bytes < ws_prefill_host(o, K, h)) return ADX_EWORKSPACE;
  CopyEngines* ce = nullptr;
  if ((r = copy_engines(&ce)) != ADX_OK) return r;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t T = o->T, S = o->S, H = o->H;
  Carve cv(ws);
  DeviceStatus* st = cv.take<DeviceStatus>(kStatusBytes);
  uint8_t* dq = cv.take<uint8_t>(static_cast<size_t>(T) * h.q_row);
  float* dqs = o->q_scale ? cv.take<float>(static_cast<size_t>(T) * 4) : nullptr;
  float* dw = cv.take<float>(static_cast<size_t>(T) * H * 4);
  uint8_t* dk = cv.take<uint8_t>(static_cast<size_t>(S) * h.k_row);
  float* dks = o->k_scale ? cv.take<float>(static_cast<size_t>(S) * 4) : nullptr;
  int32_t* didx = cv.take<int32_t>(static_cast<size_t>(T) * K * 4);
  float* dsc = cv.take<float>(static_cast<size_t>(T) * K * 4);
  uint8_t* chunk_ws = cv.base + cv.off;
  auto copy = [](void* dst, const void* src, size_t n, cudaMemcpyKind k, cudaStream_t cs) {
    return n == 0 || cudaMemcpyAsync(dst, src, n, k, cs) == cudaSuccess;
  };
  // the copies start once everything queued on `stream` before this call is done
  if (cudaEventRecord(ce->out, s) != cudaSuccess ||
      cudaStreamWaitEvent(ce->h2d, ce->out, 0) != cudaSuccess)
    return ADX_ECUDA;
  if (!copy(dk, o->k, static_cast<size_t>(S) * h.k_row, cudaMemcpyHostToDevice, ce->h2d) ||
      (dks && !copy(dks, o->k_scale, static_cast<size_t>(S) * 4, cudaMemcpyHostToDevice, ce->h2d)))
    return ADX_ECUDA;
  // longest rows first: the indexing work then shrinks chunk by chunk, so what follows the
  // last copy in is the cheapest chunk and its copy out
  for (int64_t i = 0; i < h.chunks; ++i) {
    const int64_t c = h.chunks - 1 - i;
    const int64_t r0 = c * h.C, r1 = std::min(T, r0 + h.C), n = r1 - r0;
    // chunk c in, while `stream` indexes the chunk before it
    if (!copy(dq + r0 * h.q_row, static_cast<const uint8_t*>(o->q) + r0 * h.q_row, n * h.q_row,
              cudaMemcpyHostToDevice, ce->h2d) ||
        !copy(dw + r0 * H, o->w + r0 * H, n * H * 4, cudaMemcpyHostToDevice, ce->h2d) ||
        (dqs && !copy(dqs + r0, o->q_scale + r0, n * 4, cudaMemcpyHostToDevice, ce->h2d)))
      return ADX_ECUDA;
    if (cudaEventRecord(ce->in[c], ce->h2d) != cudaSuccess ||
        cudaStreamWaitEvent(s, ce->in[c], 0) != cudaSuccess)
      return ADX_ECUDA;
    adx_operands chunk = *o;
    chunk.q = dq + r0 * h.q_row;
    chunk.q_scale = dqs ? dqs + r0 : nullptr;
    chunk.w = dw + r0 * H;
    chunk.k = dk;
    chunk.k_scale = dks;
    chunk.T = static_cast<int32_t>(n);
    chunk.q_pos0 = o->q_pos0 + r0;
    Carve ccv(chunk_ws);
    if ((r = run_flat(&chunk, K, didx + r0 * K, topk_score ? dsc + r0 * K : nullptr, nullptr, 0,
                      ccv, st, s)) != ADX_OK)
      return r;
    // chunk c out, while `stream` indexes the next one
    if (cudaEventRecord(ce->done[c], s) != cudaSuccess ||
        cudaStreamWaitEvent(ce->d2h, ce->done[c], 0) != cudaSuccess)
      return ADX_ECUDA;
    if (!copy(topk_idx + r0 * K, didx + r0 * K, n * K * 4, cudaMemcpyDeviceToHost, ce->d2h) ||
        (topk_score &&
         !copy(topk_score + r0 * K, dsc + r0 * K, n * K * 4, cudaMemcpyDeviceToHost, ce->d2h)))
      return ADX_ECUDA;
  }
  // `stream` completes only after the last copy out
  if (cudaEventRecord(ce->out, ce->d2h) != cudaSuccess ||
      cudaStreamWaitEvent(s, ce->out, 0) != cudaSuccess)
    return ADX_ECUDA;
  return ADX_OK;
}

adx_status adx_index_mtp(const adx_operands* full, const adx_operands* grp, int32_t m, int32_t G,
                         int32_t P, int32_t K, int32_t* topk_idx, float* topk_score,
                         int32_t* bank_out, void* ws, size_t ws_bytes, void* stream) {
  MtpShape sh;
  adx_operands gops;
  adx_status r = mtp_check(full, grp, m, G, P, K, sh, gops);
  if (r != ADX_OK) return r;
  if (!topk_idx || !ws) return ADX_EINVAL;
  if (ws_bytes < ws_mtp(full, &gops, sh, m, P, K)) return ADX_EWORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t R = sh.Bs * m, S = full->S, ld = ld_for(S);
  const int W = static_cast<int>(sh.width);
  Carve cv(ws);
  DeviceStatus* st = cv.take<DeviceStatus>(kStatusBytes);
  int32_t* pos_q = cv.take<int32_t>(static_cast<size_t>(R) * 4);
  int32_t* pos_g = cv.take<int32_t>(static_cast<size_t>(sh.ng) * 4);
  int32_t* cand = cv.take<int32_t>(static_cast<size_t>(sh.ng) * W * 4);
  if (bank_out != nullptr) cand = bank_out;
  if (counted(launch_mtp_positions(full->seq_len, static_cast<int32_t>(sh.Bs), m, G, pos_q,
                                   pos_g, s)) != cudaSuccess)
    return ADX_ECUDA;

  // banks: each group query scans the history its anchor sees, in its own sequence
  {
    Prepared pq;
    if ((r = prepare(&gops, gops.q, gops.q_scale, gops.w, sh.ng, cv, s, pq)) != ADX_OK) return r;
    float* scores = cv.take<float>(static_cast<size_t>(sh.ng) * ld * 4);
    // one row block per sequence holds its m/G groups: with 16 heads, tiles of 2 or 4
    // tokens keep the epilogue from reducing empty token slots
    const int tok = gops.H == 16 && sh.gps <= 4 ? (sh.gps <= 2 ? 2 : 4)
                                                : score_tokens_per_tile(gops.H);
    ScorePlan p = base_plan(&gops, pq, tok);
    p.a.scores = scores;
    p.a.score_ld = ld;
    p.a.R = static_cast<int32_t>(sh.ng);
    p.a.rows_per_batch = sh.gps;
    p.a.n_batches = static_cast<int32_t>(sh.Bs);
    p.a.row_blocks_per_batch = (sh.gps + p.tok - 1) / p.tok;
    p.a.row_pos = pos_g;
    p.a.key_batch_stride = S;
    p.a.keys_per_batch = static_cast<int32_t>(S);
    p.a.status = st;
    finish_plan(p, (S + kTileM - 1) / kTileM);
    if ((r = run_score(p, pq.q, full->k, sh.Bs * S, s)) != ADX_OK) return r;
    SelectArgs sa{};
    sa.vals = scores;
    sa.ld = ld;
    sa.rows_per_batch = 1;
    sa.len_mode = 3;
    sa.row_pos = pos_g;
    sa.len_off = 0;
    sa.len_cap = static_cast<int32_t>(S);
    sa.K = P;
    sa.out_idx = cand;
    sa.out_ld = W;
    sa.rows = static_cast<int32_t>(sh.ng);
    if ((r = run_select(sa, S, cv, st, s)) != ADX_OK) return r;
    if (counted(launch_mtp_candidates(cand, static_cast<int32_t>(sh.ng), W, P, G, m,
                                      full->seq_len, pos_g, s)) != cudaSuccess)
      return ADX_ECUDA;
  }

  // refinement: every query scores its group's candidates, packed once per group from its
  // sequence into contiguous rows (a group's G queries share them)
  const int rb = row_bytes(full);
  uint8_t* packed = cv.take<uint8_t>(static_cast<size_t>(sh.ng) * sh.bcp * rb);
  float* pscale = cv.take<float>(static_cast<size_t>(sh.ng) * sh.bcp * 4);
  int32_t* ppos = cv.take<int32_t>(static_cast<size_t>(sh.ng) * sh.bcp * 4);
  if (counted(launch_pack_candidates(full->k, full->k_scale, S, 1, sh.gps,
                                     static_cast<int32_t>(S), cand,
                                     static_cast<int32_t>(sh.ng), W,
                                     static_cast<int32_t>(sh.bcp), rb, packed,
                                     fp8_keys(full) ? pscale : nullptr, ppos, s)) != cudaSuccess)
    return ADX_ECUDA;
  Prepared pq;
  if ((r = prepare(full, full->q, full->q_scale, full->w, R, cv, s, pq)) != ADX_OK) return r;
  float* scores = cv.take<float>(static_cast<size_t>(R) * sh.bcp * 4);
  ScorePlan p = base_plan(full, pq, score_tokens_per_tile(full->H));
  p.a.scores = scores;
  p.a.score_ld = sh.bcp;
  p.a.R = static_cast<int32_t>(R);
  p.a.rows_per_batch = G;
  p.a.n_batches = static_cast<int32_t>(sh.ng);
  p.a.row_blocks_per_batch = (G + p.tok - 1) / p.tok;
  p.a.row_pos = pos_q;
  p.a.k_scale = fp8_keys(full) ? pscale : nullptr;
  p.a.key_pos = ppos;
  p.a.key_batch_stride = sh.bcp;
  p.a.keys_per_batch = static_cast<int32_t>(sh.bcp);
  p.a.status = st;
  finish_plan(p, sh.bcp / kTileM);
  if ((r = run_score(p, pq.q, packed, sh.ng * sh.bcp, s)) != ADX_OK) return r;
  SelectArgs sa{};
  sa.vals = scores;
  sa.ld = sh.bcp;
  sa.idx_map = ppos;
  sa.map_stride = sh.bcp;
  sa.rows_per_batch = G;
  sa.len_mode = 0;
  sa.len_fixed = static_cast<int32_t>(sh.bcp);
  sa.len_cap = static_cast<int32_t>(sh.bcp);
  sa.K = K;
  sa.out_idx = topk_idx;
  sa.out_val = topk_score;
  sa.out_ld = K;
  sa.rows = static_cast<int32_t>(R);
  return run_select(sa, sh.bcp, cv, st, s);
}

adx_status adx_group_query_mean(int32_t q_dtype, const void* q, const float* q_scale,
                                const float* w, int32_t T, int32_t H, int32_t d, int32_t G,
                                int32_t Hg, void* qbar_out, float* wbar_out, void* stream) {
  if (!q || !w || !qbar_out || !wbar_out || T <= 0 || H <= 0 || d <= 0 || G <= 0) return ADX_EINVAL;
  if (Hg <= 0 || Hg > H || d % 8 != 0) return ADX_EINVAL;
  if (q_dtype != ADX_BF16 && q_dtype != ADX_E4M3) return ADX_EINVAL;
  if ((q_dtype == ADX_E4M3) != (q_scale != nullptr)) return ADX_EINVAL;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(qbar_out)) % 16 != 0)
    return ADX_EINVAL;
  const cudaError_t e = counted(launch_group_mean(q, q_scale, q_dtype == ADX_E4M3, w, T / G, H,
                                                  d, G, Hg, qbar_out, wbar_out,
                                                  static_cast<cudaStream_t>(stream)));
  return e == cudaSuccess ? ADX_OK : ADX_ECUDA;
}

adx_status adx_group_union_sizes(const int32_t* topk_idx, int32_t T, int32_t K, int32_t G,
                                 int32_t S, int32_t* union_out, void* stream) {
  if (!topk_idx || !union_out || T <= 0 || K <= 0 || G <= 0 || S <= 0) return ADX_EINVAL;
  if (static_cast<int64_t>(G) * K > INT32_MAX) return ADX_EINVAL;
  if (static_cast<size_t>((S + 31) / 32) * 4 > kUnionMaxBitmapBytes) return ADX_EUNSUPPORTED;
  const cudaError_t e = counted(launch_union_sizes(topk_idx, K, G, S, T / G, union_out,
                                                   static_cast<cudaStream_t>(stream)));
  return e == cudaSuccess ? ADX_OK : ADX_ECUDA;
}

adx_status adx_bank_coverage(const int32_t* topk_idx, int32_t T, int32_t K,
                             const int32_t* bank_idx, int32_t bank_w, int32_t G, int32_t S,
                             int32_t* hits_out, int32_t* count_out, void* stream) {
  if (!topk_idx || !bank_idx || !hits_out || !count_out) return ADX_EINVAL;
  if (T <= 0 || K <= 0 || bank_w <= 0 || G <= 0 || S <= 0) return ADX_EINVAL;
  if (static_cast<size_t>((S + 31) / 32) * 4 > kUnionMaxBitmapBytes) return ADX_EUNSUPPORTED;
  const cudaError_t e = counted(launch_bank_coverage(topk_idx, K, bank_idx, bank_w, G, S, T / G,
                                                     hits_out, count_out,
                                                     static_cast<cudaStream_t>(stream)));
  return e == cudaSuccess ? ADX_OK : ADX_ECUDA;
}

adx_status adx_check_wait_timeout(void* ws, uint64_t timeout_ns, void* stream) {
  if (!ws || timeout_ns == 0 || timeout_ns > 1000000000ull) return ADX_EINVAL;
  const cudaError_t e = counted(launch_wait_timeout(static_cast<DeviceStatus*>(ws), timeout_ns,
                                                    static_cast<cudaStream_t>(stream)));
  return e == cudaSuccess ? ADX_OK : ADX_ECUDA;
}

adx_status adx_read_device_status(void* ws, void* stream) {
  if (!ws) return ADX_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return ADX_ECUDA;
  DeviceStatus h{};
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return ADX_ECUDA;
  if (cudaMemset(ws, 0, sizeof(h)) != cudaSuccess) return ADX_ECUDA;
  return static_cast<adx_status>(h.code);
}

size_t adx_hisa_workspace_size(const adx_operands* o, int32_t n_blocks, int32_t K,
                               int32_t blocks_external) {
  if (hisa_check(o, n_blocks, K) != ADX_OK) return 0;
  return ws_hisa(o, n_blocks, K, blocks_external != 0);
}

adx_status adx_hisa_block_keys(const adx_operands* o, int32_t last_only, void* kbar,
                               float* kbar_scale, void* stream) {
  const bool decode = o != nullptr && o->seq_len != nullptr;
  adx_status r = check_operands(o, decode);
  if (r != ADX_OK) return r;
  (void)kbar_scale;  // block keys are bf16 for either key format
  if (!kbar) return ADX_EINVAL;
  const int64_t len = decode ? 0 : std::min<int64_t>(o->S, o->q_pos0 + o->T);
  const cudaError_t e = counted(launch_block_keys(
      o->k, o->k_scale, fp8_keys(o), o->S, o->d, decode ? o->T : 1, o->seq_len,
      static_cast<int32_t>(len), last_only != 0, static_cast<int32_t>(hisa_nbmax(o)), kbar,
      static_cast<cudaStream_t>(stream)));
  if (e == cudaErrorInvalidValue) return ADX_EUNSUPPORTED;
  return e == cudaSuccess ? ADX_OK : ADX_ECUDA;
}

adx_status adx_index_hisa(const adx_operands* o, const void* kbar, const float* kbar_scale,
                          int32_t n_blocks, int32_t K, int32_t* topk_idx, float* topk_score,
                          int32_t* blocks_out, void* ws, size_t ws_bytes, void* stream) {
  adx_status r = hisa_check(o, n_blocks, K);
  if (r != ADX_OK) return r;
  (void)kbar_scale;  // block keys are bf16 for either key format
  if (!kbar || !topk_idx || !ws) return ADX_EINVAL;
  if (ws_bytes < ws_hisa(o, n_blocks, K, blocks_out != nullptr)) return ADX_EWORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool decode = o->seq_len != nullptr;
  const int32_t T = o->T;
  const int64_t nbmax = hisa_nbmax(o), ldb = ld_for(nbmax);
  const int32_t nc = n_blocks * kTileM;
  Carve cv(ws);
  DeviceStatus* st = cv.take<DeviceStatus>(kStatusBytes);
  int32_t* row_blk = cv.take<int32_t>(static_cast<size_t>(T) * 4);
  Prepared pq;  // the preparation also writes each row's block
  if ((r = prepare(o, o->q, o->q_scale, o->w, T, cv, s, pq, row_blk)) != ADX_OK) return r;
  // the block pass scores bf16 block keys, so it takes bf16 queries: the same preparation
  // without the e4m3 step when the keys are e4m3
  Prepared pb = pq;
  if (fp8_keys(o)) {
    void* qo = cv.take<uint8_t>(static_cast<size_t>(T) * o->H * o->d * 2);
    int8_t* fl = cv.take<int8_t>(static_cast<size_t>(T));
    if (counted(launch_prepare_q(o->q, o->q_scale, o->q_dtype == ADX_E4M3, false, o->w, T, o->H,
                                 o->d, qo, nullptr, fl, s)) != cudaSuccess)
      return ADX_ECUDA;
    pb.q = qo;
    pb.q_scale = nullptr;
    pb.fold = fl;
  }
  float* bsc = cv.take<float>(static_cast<size_t>(T) * ldb * 4);
  int32_t* blocks =
      blocks_out ? blocks_out : cv.take<int32_t>(static_cast<size_t>(T) * n_blocks * 4);
  float* tsc = cv.take<float>(static_cast<size_t>(T) * nc * 4);

  // 1. block scores: Eq. (1) on the block keys, block b visible to a row whose position lies
  //    in block >= b
  {
    ScorePlan p = decode ? rowwise_plan(o, pb, bsc, ldb)
                         : base_plan(o, pb, score_tokens_per_tile(o->H));
    p.fp8 = false;
    ScoreArgs& a = p.a;
    a.k_scale = nullptr;
    a.row_pos = row_blk;
    a.status = st;
    a.scores = bsc;
    a.score_ld = ldb;
    a.R = T;
    a.keys_per_batch = static_cast<int32_t>(nbmax);
    if (decode) {
      a.key_batch_stride = nbmax;
    } else {
      a.rows_per_batch = T;
      a.n_batches = 1;
      a.row_blocks_per_batch = (T + p.tok - 1) / p.tok;
      a.reverse_order = 1;
    }
    const int64_t vis_blocks =
        decode ? nbmax : (std::min<int64_t>(o->S, o->q_pos0 + T) + kTileM - 1) / kTileM;
    finish_plan(p, (vis_blocks + kTileM - 1) / kTileM);
    if ((r = run_score(p, pb.q, kbar, (decode ? T : 1) * nbmax, s)) != ADX_OK) return r;
  }
  // 2. forced blocks, then the block Top-n; rows that fit the one-warp select get the forced
  //    blocks there, longer ones from a kernel that raises their scores first
  const bool warp_rows = nbmax <= kWarpSelectMax;
  if (!warp_rows &&
      counted(launch_force_blocks(bsc, ldb, T, row_blk, n_blocks, s)) != cudaSuccess)
    return ADX_ECUDA;
  {
    SelectArgs sa{};
    if (warp_rows) {
      sa.force_blk = row_blk;
      sa.force_n = n_blocks;
    }
    sa.vals = bsc;
    sa.ld = ldb;
    sa.rows_per_batch = 1;
    sa.len_mode = 3;
    sa.row_pos = row_blk;
    sa.len_cap = static_cast<int32_t>(nbmax);
    sa.K = n_blocks;
    sa.out_idx = blocks;
    sa.out_ld = n_blocks;
    sa.rows = T;
    if ((r = run_select(sa, nbmax, cv, st, s)) != ADX_OK) return r;
  }
  // 3. token refinement: a decode row scores the key tiles of its own blocks; a group of
  //    kHisaGroup prefill rows scores the union of its rows' blocks in one N = 256 tile, each
  //    row's scores landing in the slots of its own list (no row sees a block it did not keep)
  {
    ScorePlan p = decode ? rowwise_plan(o, pq, tsc, nc) : base_plan(o, pq, kHisaGroup);
    ScoreArgs& a = p.a;
    a.key_blk = blocks;
    a.key_blk_stride = n_blocks;
    a.S_valid = o->S;
    a.keys_per_batch = nc;
    a.status = st;
    int64_t max_tiles = n_blocks;
    if (!decode) {
      const int32_t ng = (T + kHisaGroup - 1) / kHisaGroup, width = kHisaGroup * n_blocks;
      int32_t* uni = cv.take<int32_t>(static_cast<size_t>(ng) * width * 4);
      int32_t* slot = cv.take<int32_t>(static_cast<size_t>(ng) * width * 4);
      int32_t* cnt = cv.take<int32_t>(static_cast<size_t>(ng) * 4);
      if (counted(launch_block_union(blocks, n_blocks, T, kHisaGroup, uni, slot, cnt, s)) !=
          cudaSuccess)
        return ADX_ECUDA;
      a.key_blk = uni;
      a.key_blk_stride = width;
      a.key_blk_count = cnt;
      a.key_blk_slot = slot;
      a.keys_per_batch = width * kTileM;
      a.scores = tsc;
      a.score_ld = nc;
      a.pos_base = o->q_pos0;
      a.pos_step = 1;
      a.R = T;
      a.rows_per_batch = kHisaGroup;
      a.n_batches = ng;
      a.key_batch_div = ng;
      a.key_batch_stride = 0;
      a.row_blocks_per_batch = 1;
      a.reverse_order = 1;
      max_tiles = width;
    }
    finish_plan(p, max_tiles);
    if ((r = run_score(p, pq.q, o->k, decode ? static_cast<int64_t>(T) * o->S : o->S, s)) !=
        ADX_OK)
      return r;
  }
  // 4. final Top-K over the candidate slots, mapped to key positions through the block list
  SelectArgs sa{};
  sa.vals = tsc;
  sa.ld = nc;
  sa.rows_per_batch = 1;
  sa.idx_map = blocks;
  sa.map_stride = n_blocks;
  sa.map_shift = kHisaShift;
  sa.len_mode = 3;
  sa.row_pos = row_blk;
  sa.len_mul = kTileM;
  sa.len_cap = nc;
  sa.K = K;
  sa.out_idx = topk_idx;
  sa.out_val = topk_score;
  sa.out_ld = K;
  sa.rows = T;
  return run_select(sa, nc, cv, st, s);
}

}  // extern "C"

// Internal declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/adx.h"

namespace adx {

// Device status word at the start of every workspace (sticky until read).
struct DeviceStatus {
  int32_t code;    // 0 = ok, otherwise an adx_status value
  int32_t where;   // which kernel raised it
  int32_t info0;
  int32_t info1;
};
constexpr size_t kStatusBytes = 256;
constexpr int kWhereScore = 1;
constexpr int kWhereSelect = 2;
constexpr int kWhereCheck = 3;
constexpr int kWhereGemm = 4;

constexpr int kTileM = 128;  // keys per MMA tile (TMEM lanes)

// Work decomposition and epilogue parameters of the scoring kernel.
//
// Query rows r = 0..R-1 are split into batches of rows_per_batch rows; every batch owns a
// key range of keys_per_batch rows in the key tensor map, starting at row
// (b / key_batch_div) * key_batch_stride (key_batch_div consecutive batches share one range;
// 0 counts as 1). The position of row r is row_pos[r] when row_pos is given, seq_len[b] - 1
// when seq_len is given (decode), else pos_base + r * pos_step. Key c of batch b sits at position key_pos[...]
// when key_pos is given (packed candidate lists), at the position the index list gives for
// slot c with gathered keys (key_idx), else at position c.
struct ScoreArgs {
  const float* w;          // [R, H] gates
  const float* q_scale;    // [R] or null
  const float* k_scale;    // [n_batches * key_batch_stride] or null
  const int32_t* key_pos;  // [n_batches * key_batch_stride] or null
  // Gathered keys (a key tensor map with one-row boxes): slot c < keys_per_batch of batch b is
  // the key at position key_idx[b * key_idx_stride + c] (c < n_idx) of the batch's key range;
  // a negative position, one >= S_valid, or c >= n_idx is no key. Null: contiguous key rows.
  const int32_t* key_idx;
  int64_t key_idx_stride;
  int32_t n_idx;
  int32_t S_valid;
  // Key blocks: tile t of batch b is the 128 key rows starting at
  // 128 * key_blk[b * key_blk_stride + t] of the batch's key range; a negative entry is no
  // tile, and rows at or past S_valid are no key. The batch scores key_blk_count[b] tiles
  // (null: min(keys_per_batch / 128, last row position / 128 + 1)). key_blk_slot (same layout,
  // or null): byte j is the slot of tile t in the block list of the batch's row j, whose
  // score row receives the tile at columns [128 * slot, 128 * slot + 128) (0xFF: not one of
  // that row's blocks); null: slot t for every row. Null key_blk: contiguous tiles.
  const int32_t* key_blk;
  int64_t key_blk_stride;
  const int32_t* key_blk_count;
  const int32_t* key_blk_slot;
  const int32_t* seq_len;  // [n_batches] or null
  const int32_t* row_pos;  // [R] or null
  const int8_t* fold_flag; // [R]: 1 = the row's queries carry its gates already; null = none do
  float* scores;           // [R, score_ld]
  int64_t score_ld;
  // 1: score stores bypass the L2's normal retention (evict-first), for score matrices far
  // larger than the L2 that would otherwise push the key tiles out of it
  int32_t stream_scores;
  int64_t pos_base;
  int32_t pos_step;
  int32_t R;
  int32_t rows_per_batch;
  int32_t n_batches;
  int64_t key_batch_stride;
  int32_t key_batch_div;
  int32_t keys_per_batch;
  int32_t row_blocks_per_batch;
  int32_t chunks_per_block;
  int32_t chunk_tiles;
  int32_t n_items;
  int32_t reverse_order;
  // 1: CTA c takes whole row blocks c, c + grid, ... (for equal-length row blocks: the row
  // blocks of one key batch then run at the same time and share its keys through L2);
  // 0: balanced contiguous ranges of (row block, key tile) pairs.
  int32_t round_robin;
  DeviceStatus* status;
  uint64_t timeout_ns;
};

// Row-wise Top-K over a score matrix (radix select).
struct SelectArgs {
  const float* vals;       // [rows, ld]
  int64_t ld;
  const int32_t* in_idx;   // [rows, ld] element ids (second stage of a split select) or null
  const int32_t* idx_map;  // position of element c of row r: idx_map[(r / rows_per_batch) * map_stride + c], or null
  int64_t map_stride;
  int32_t rows_per_batch;
  // row length: len_mode 0 -> fixed len_fixed; 1 -> min(len_cap, pos_base + r*pos_step + 1);
  //             2 -> min(len_cap, seq_len[r / rows_per_batch]);
  //             3 -> min(len_cap, (row_pos[r] + 1 + len_off) * max(1, len_mul))
  int32_t len_mode;
  int32_t len_fixed;
  int32_t len_cap;
  int64_t pos_base;
  int32_t pos_step;
  const int32_t* seq_len;
  const int32_t* row_pos;
  int32_t len_off;
  int32_t len_mul;
  // Forced elements (one-warp select only): on a row r with force_blk[r] + 1 > force_n,
  // elements 0 and force_blk[r] count as +inf (HISA's first and own block). Null: none.
  const int32_t* force_blk;
  int32_t force_n;
  // with idx_map: 0 -> element c maps to map[c]; s > 0 -> to (map[c >> s] << s) + (c & (2^s - 1))
  // (the map lists blocks of 2^s consecutive positions)
  int32_t map_shift;
  int32_t K;
  int32_t n_seg;           // split each row into n_seg segments of seg_len (first stage)
  int32_t seg_len;
  int32_t* out_idx;        // [rows * n_seg, out_ld]
  float* out_val;          // same layout, or null
  int64_t out_ld;
  int32_t rows;
  DeviceStatus* status;
};

// Longest row the one-warp-per-row select holds (32 lanes x 40 keys); launches whose rows all
// fit (and are not split into segments) take it.
constexpr int64_t kWarpSelectMax = 32 * 40;

// Launchers (return a cudaError_t from the launch).
cudaError_t launch_score(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const ScoreArgs& a,
                         bool fp8, int H, int d, int tok, int grid, cudaStream_t s);
// tm_k must have one-row boxes when a.key_idx is set (gathered keys).
int score_tokens_per_tile(int H);  // tokens per N tile for a head count (0 = unsupported)
bool score_config_supported(bool fp8, int H, int d);
// Launches one to three kernels (row-length classes); *launched receives how many.
cudaError_t launch_select(const SelectArgs& a, cudaStream_t s, int* launched);
// Few long rows: CTAs per row of the cluster select (one thread-block cluster per row, the
// row held in registers across the cluster), or 0 when it does not apply. By default rows of
// at most 8 K keys are left to the one-CTA selects; any_k drops that rule (the second stage of
// a split select, whose rows are n_seg * K candidates).
int select_cluster_ctas(int64_t rows, int64_t n_max, int K, int sms, bool any_k = false);
// One launch of the cluster select with `ctas` CTAs per row (a.n_seg must be 1).
cudaError_t launch_select_cluster(const SelectArgs& a, int ctas, cudaStream_t s, int* launched);
// Packs candidate key rows: slot c of group g is key cand[g * n_cand + c] of key range
// g / group_div (per_group_keys; else of the one shared range). packed_pos may be null.
cudaError_t launch_pack_candidates(const void* k, const float* k_scale, int64_t key_batch_stride,
                                   int32_t per_group_keys, int32_t group_div, int32_t S_valid,
                                   const int32_t* cand,
                                   int32_t n_groups, int32_t n_cand, int32_t n_cand_pad,
                                   int32_t row_bytes, void* packed, float* packed_scale,
                                   int32_t* packed_pos, cudaStream_t s);
// MTP windows: positions of the window queries (row_pos_q [Bs*m]) and of the group anchors
// (row_pos_g [Bs*m/G]) from seq_len[b] = keys in sequence b's cache, the window included.
cudaError_t launch_mtp_positions(const int32_t* seq_len, int32_t Bs, int32_t m, int32_t G,
                                 int32_t* row_pos_q, int32_t* row_pos_g, cudaStream_t s);
// MTP windows: completes each group's candidate row cand [n_groups, width] (columns < P hold
// the bank): a banked window adds the post-anchor positions and pads with -1; a window whose
// first query sees at most P keys gets every position up to its last member's instead.
cudaError_t launch_mtp_candidates(int32_t* cand, int32_t n_groups, int32_t width, int32_t P,
                                  int32_t G, int32_t m, const int32_t* seq_len,
                                  const int32_t* anchor_pos, cudaStream_t s);
// One CTA whose bounded wait on a barrier nothing completes runs out after timeout_ns and is
// recorded in *status (code ADX_ETIMEOUT) like a wait of the indexer's kernels.
cudaError_t launch_wait_timeout(DeviceStatus* status, uint64_t timeout_ns, cudaStream_t s);
// Mean-pooled group queries qbar [n_groups, Hg, d] bf16 and gates wbar [n_groups, Hg].
cudaError_t launch_group_mean(const void* q, const float* q_scale, bool in_e4m3, const float* w,
                              int64_t n_groups, int H, int d, int G, int Hg, void* qbar,
                              float* wbar, cudaStream_t s);
// Union sizes of the Top-K sets of n_groups groups of G consecutive rows of topk [*, K]
// (positions outside [0, S) are not indices). S is limited by the shared-memory bitmap.
constexpr size_t kUnionMaxBitmapBytes = 200 * 1024;
cudaError_t launch_union_sizes(const int32_t* topk, int32_t K, int32_t G, int32_t S,
                               int32_t n_groups, int32_t* out, cudaStream_t s);
// Coverage of each complete group's bank row (bank [n_groups, bank_w]) over the Top-K rows of
// its G members (topk [n_groups * G, K]): hits = positions found in the bank, count = positions.
cudaError_t launch_bank_coverage(const int32_t* topk, int32_t K, const int32_t* bank,
                                 int32_t bank_w, int32_t G, int32_t S, int32_t n_groups,
                                 int32_t* hits, int32_t* count, cudaStream_t s);
// Packed decode banks [rows, width] of key rows: copies the slots c in [first, width) whose
// position bank[t, c] is at or before row t's position (seq_len[t] - 1) from cache t.
cudaError_t launch_refresh_post(const void* k, const float* k_scale, int64_t S,
                                const int32_t* seq_len, const int32_t* bank, int32_t rows,
                                int32_t width, int32_t first, int32_t row_bytes, void* packed,
                                float* packed_scale, cudaStream_t s);
cudaError_t launch_fill_post_anchor(int32_t* bank, int32_t n_groups, int32_t bank_w,
                                    int32_t first_col, int32_t count, int64_t pos_base,
                                    int32_t pos_step, const int32_t* seq_len, int32_t start_off,
                                    cudaStream_t s);
int score_blocks_per_sm(bool fp8, int H, int d, int tok);
// Writes the prepared query rows (gate-folded where all gates are >= 0, else as given), with
// fold flags and, for e4m3 output, one scale per row.
// Optional by-product of the query preparation: out[r] = block (of kTileM positions) of row
// r's position, q_pos0 + r, or seq_len[r] - 1 when seq_len is set.
struct RowBlocks {
  int32_t* out = nullptr;
  int64_t q_pos0 = 0;
  const int32_t* seq_len = nullptr;
};
cudaError_t launch_prepare_q(const void* q, const float* q_scale, bool in_e4m3, bool out_e4m3,
                             const float* w, int64_t rows, int H, int d, void* q_out,
                             float* q_scale_out, int8_t* fold_flag, cudaStream_t s,
                             RowBlocks rb = RowBlocks{});

// HISA block keys: the mean of each 128-key block of each key range (n_seq ranges of S rows;
// length seq_len[b], or len_fixed without seq_len; e4m3 keys decoded with their scales), in
// bf16 in kbar [n_seq, nbmax, d]; last_only: just the block holding each range's last key.
cudaError_t launch_block_keys(const void* k, const float* k_scale, bool fp8, int64_t S, int d,
                              int32_t n_seq, const int32_t* seq_len, int32_t len_fixed,
                              bool last_only, int32_t nbmax, void* kbar, cudaStream_t s);
// Union of the block lists (blocks [R, n_blocks], -1 padded) of each group of `tok`
// consecutive rows: uni [groups, tok * n_blocks] distinct blocks, count [groups] how many,
// slot [groups, tok * n_blocks] byte j = slot of the union entry in row j's list (0xFF: none).
// tok <= 4, n_blocks <= 255.
cudaError_t launch_block_union(const int32_t* blocks, int32_t n_blocks, int32_t R, int32_t tok,
                               int32_t* uni, int32_t* slot, int32_t* count, cudaStream_t s);
// Raises the scores of block 0 and of the row's own block to +inf on rows that see more than
// n_blocks blocks.
cudaError_t launch_force_blocks(float* scores, int64_t ld, int32_t R, const int32_t* row_blk,
                                int32_t n_blocks, cudaStream_t s);

// Argument checks of adx_index_prefill that need no device: the operands (prefill layout)
// and K. ADX_OK, ADX_EINVAL or ADX_EUNSUPPORTED, exactly as adx_index_prefill returns them.
adx_status check_prefill_args(const adx_operands* o, int32_t K);

// 2-D tensor map over `rows` rows of `d` elements (1 or 2 bytes each) with 128-byte swizzled
// boxes of 128 bytes x box_rows; false when the driver's encoder rejects it.
bool encode_rows(CUtensorMap* m, const void* base, bool one_byte, int d, int64_t rows,
                 int box_rows);
// Y [n, m] (bf16, or fp32 with out_f32) = X [n, k] W^T for bf16 W [m, k] (tm_w) and X [n, k]
// (tm_x), both mapped by encode_rows with gemm_box_rows() rows per box. Timeouts of the
// kernel's bounded waits are recorded in *st.
cudaError_t launch_gemm_bf16(const CUtensorMap& tm_w, const CUtensorMap& tm_x, void* y,
                             bool out_f32, int m, int n, int k, DeviceStatus* st,
                             uint64_t timeout_ns, cudaStream_t s);
int gemm_box_rows();

// Adds n to the library's launch counter (kernels launched outside the API file).
void add_launches(int n);

}  // namespace adx

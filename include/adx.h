/*
 * adx.h - C ABI of the B200 (sm_100a) sparse-attention token indexer.
 *
 * The library computes the DeepSeek Sparse Attention token indexer and ADIndex's
 * group-shared variant of it, as defined in "ADIndex: Layer-Adaptive Sparse Attention
 * Indexing via Group-Level Distillation" (arXiv 2611.12956v1):
 *
 *   score      I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s])          (§3, Eq. (1))
 *   selection  T_t = TopK_{s <= pos(t)} I[t,s]                        (§3, Eq. (2))
 *   bank       P = TopK over the group query's scores of a scan      (§4.3, Eq. (13))
 *   refine     T_i = TopK_{s in C_i} I[i,s], C_i = bank U post-anchor (§4.3, Eq. (14))
 *   group indexer  q-bar, w-bar from pooled query latents and hidden states (§4.2, Eqs. (6)-(7))
 *   HISA       block Top-n over mean-pooled 128-key blocks, then Top-K of the kept blocks'
 *              tokens ("HISA: Efficient Hierarchical Indexing for Fine-Grained Sparse
 *              Attention", arXiv 2603.28458v3; ADIndex Appendix C.5)
 *
 * Conventions shared by every entry point
 *  - Every pointer argument is a DEVICE pointer unless stated otherwise. The caller owns
 *    all memory; the library allocates nothing, keeps no state between calls besides
 *    cached device properties (and, created on first use per device: two copy streams and
 *    their events for adx_index_prefill_host), and launches all work asynchronously on
 *    `stream` (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *    One exception: adx_index_prefill_noalloc runs on a fixed device array of
 *    ADX_STATIC_SCRATCH_BYTES compiled into the library (held on every GPU that loads it) and
 *    caches that array's device address per device and context.
 *  - Argument errors are detected on the host and returned before any launch.
 *  - Errors the device detects (a bounded wait that ran out) are recorded in a status word
 *    at the start of the workspace and reported by adx_read_device_status(). The word is
 *    sticky: it holds the first error since the workspace was zeroed or last read. Zero the
 *    workspace's first ADX_STATUS_BYTES once before the first call.
 *  - Positions are absolute token positions starting at 0. Key s is visible to a query at
 *    position p iff s <= p.
 *  - Output rows hold key positions (int32) in ascending candidate order (flat: ascending
 *    position), padded with -1 when fewer than K keys are visible; the optional score
 *    outputs hold the matching fp32 scores, padded with -inf. Ties at the K-th score are
 *    broken towards the lower candidate index.
 *  - Operands: bf16, or FP8-e4m3 codes (uint8) with one fp32 scale per token row (a query
 *    token's scale covers all its heads). Score arithmetic is fp32 with fp32 tensor-core
 *    accumulation.
 */
#ifndef ADX_H_
#define ADX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ADX_ABI_VERSION 1
#define ADX_STATUS_BYTES 256

typedef enum {
  ADX_OK = 0,
  ADX_EINVAL = 1,        /* bad argument (null pointer, size or range) */
  ADX_EUNSUPPORTED = 2,  /* shape/dtype combination without a compiled kernel */
  ADX_EWORKSPACE = 3,    /* workspace too small (see adx_workspace_size) */
  ADX_ECUDA = 4,         /* a CUDA runtime call or launch failed */
  ADX_EOVERFLOW = 5,     /* an internal buffer would overflow */
  ADX_ETIMEOUT = 6       /* a device-side bounded wait ran out (device status only) */
} adx_status;

typedef enum { ADX_BF16 = 0, ADX_E4M3 = 1 } adx_dtype;

/* Readings of the shared bank (ADIndex §4.3). For a group whose first query sits at
 * position a and whose members are a .. a+G-1:
 *   ADX_BANK_PAPER  - the group query scans s <= a; the bank keeps the B best; member i adds
 *                     the post-anchor positions a+1 .. i (Eqs. (13)-(14)). Bank width B+G-1.
 *   ADX_BANK_WINDOW - the group query scans s < a; the bank keeps the B-G best plus the
 *                     group's window a .. a+G-1; member i uses the bank entries <= i.
 *                     Bank width B. */
typedef enum { ADX_BANK_PAPER = 0, ADX_BANK_WINDOW = 1 } adx_bank_mode;

typedef enum {
  ADX_OP_PREFILL = 0,
  ADX_OP_DECODE = 1,
  ADX_OP_GROUP_BANK = 2,
  ADX_OP_BANK_REFINE = 3,
  ADX_OP_PREFILL_HOST = 4,  /* adx_workspace_size: B = rows_per_chunk */
  ADX_OP_BANK_REFINE_PACKED = 5
} adx_op;

/* One indexer operand set.
 *
 * Prefill layout (seq_len == NULL): T query rows at positions q_pos0 .. q_pos0+T-1 share
 *   one key array k [S, d]; requires 0 <= q_pos0 and q_pos0 + T <= S.
 * Decode layout (seq_len != NULL): row t owns key cache t of k [T, S, d] (S = capacity)
 *   and sits at position seq_len[t] - 1; requires 1 <= seq_len[t] <= S (not checked on the
 *   host: seq_len lives on the device).
 *
 * q        [T, H, d] row-major, bf16 or e4m3 codes (q_dtype)
 * q_scale  [T] fp32, required iff q_dtype == ADX_E4M3
 * w        [T, H] fp32 gates, any sign
 * k        key rows of d elements, bf16 or e4m3 codes (k_dtype); 16-byte aligned
 * k_scale  one fp32 per key row, required iff k_dtype == ADX_E4M3
 * Supported: H in {4, 8, 16, 32, 64}; d = 128 (bf16 or e4m3) or d = 64 (bf16 only);
 * q_dtype == k_dtype, except bf16 queries with an e4m3 key cache in the decode layout (the
 * queries are then quantised to e4m3 per token inside the call). */
typedef struct {
  int32_t q_dtype;
  int32_t k_dtype;
  const void* q;
  const float* q_scale;
  const float* w;
  const void* k;
  const float* k_scale;
  int32_t T, H, d, S;
  int64_t q_pos0;
  const int32_t* seq_len;
} adx_operands;

/* Bytes of workspace `op` needs for these operands (K: Top-K size; B, G, mode: bank
 * parameters, ignored by the flat ops). Returns 0 for invalid or unsupported arguments. */
size_t adx_workspace_size(int32_t op, const adx_operands* ops, int32_t K, int32_t B, int32_t G,
                          int32_t mode);

/* Columns of a bank row for (B, G, mode): B + G - 1 (PAPER) or B (WINDOW). */
int32_t adx_bank_width(int32_t B, int32_t G, int32_t mode);

/* Flat causal indexer over a prefix (ADIndex §3, Eqs. (1)-(2)); prefill layout.
 * topk_idx    [T, K] int32 out
 * topk_score  [T, K] fp32 out, or NULL
 * scores_out  [T, scores_ld] fp32 out, or NULL: every score I[t, s] (s <= pos(t); -inf for
 *             invisible keys up to the tile end). scores_ld >= S rounded up to 128 and a
 *             multiple of 4; scores_out 16-byte aligned (ADX_EINVAL otherwise).
 * ws          workspace of ws_bytes >= adx_workspace_size(ADX_OP_PREFILL, ...) */
adx_status adx_index_prefill(const adx_operands* ops, int32_t K, int32_t* topk_idx,
                             float* topk_score, float* scores_out, int64_t scores_ld, void* ws,
                             size_t ws_bytes, void* stream);

/* Flat causal indexer over host buffers (same computation as adx_index_prefill, prefill
 * layout): q, q_scale, w, k, k_scale of `ops` and topk_idx [T, K] / topk_score [T, K] (or NULL)
 * are HOST pointers, page-locked for the copies to overlap the work. The rows are indexed in
 * chunks of rows_per_chunk (at most 64 chunks), the last (longest) rows first: one chunk's
 * queries and gates are copied in while the chunk before it is indexed on `stream`, and each
 * chunk's Top-K rows are copied out while the next one is indexed, on two copy streams the
 * library keeps per device. The call returns once everything
 * is queued; the results are in the host arrays when `stream` has completed. Work queued on
 * `stream` before the call finishes before the first copy starts. Calls on one device must
 * not be issued from several host threads at the same time.
 * ws  device workspace of ws_bytes >= adx_workspace_size(ADX_OP_PREFILL_HOST, ops, K,
 *     rows_per_chunk, 0, 0): device copies of the operands and results, one chunk's indexer
 *     workspace. */
adx_status adx_index_prefill_host(const adx_operands* ops, int32_t K, int32_t rows_per_chunk,
                                  int32_t* topk_idx, float* topk_score, void* ws,
                                  size_t ws_bytes, void* stream);

/* Flat indexer for one query per sequence against that sequence's key cache (§3,
 * Eqs. (1)-(2), one decode step); decode layout. topk_idx [T, K], topk_score [T, K] or NULL. */
adx_status adx_index_decode(const adx_operands* ops, int32_t K, int32_t* topk_idx,
                            float* topk_score, void* ws, size_t ws_bytes, void* stream);

/* ---- HISA: block filter, then token refinement -----------------------------------------
 * The hierarchical indexer of "HISA: Efficient Hierarchical Indexing for Fine-Grained Sparse
 * Attention" (arXiv 2603.28458v3, abstract) with the settings of ADIndex Appendix C.5:
 * keys are pooled into blocks of ADX_HISA_BLOCK consecutive positions by their mean; a query
 * at position p sees blocks 0 .. p / ADX_HISA_BLOCK; when more than n_blocks are visible it
 * keeps block 0, its own block and the n_blocks - 2 best other blocks by Eq. (1) on the
 * block keys (all visible blocks otherwise); the visible tokens of the kept blocks are then
 * scored with Eq. (1) and the Top-K of them returned (all of them when at most K).
 * Both layouts of adx_operands apply: prefill (one key range of S keys, rows at q_pos0 + r)
 * and decode (row r = sequence r at position seq_len[r] - 1, its own S-row cache). */
#define ADX_HISA_BLOCK 128

/* Block keys kbar [n_seq, ceil(S / 128), d] bf16, for either key format (e4m3 keys are decoded
 * with their scales first): the mean of each block's keys, n_seq = 1 (prefill) or T (decode).
 * A trailing partial block is the mean of the keys it holds. Prefill: the blocks of the first
 * min(S, q_pos0 + T) keys. Decode: the blocks of the first seq_len[r] keys of each cache;
 * last_only != 0 recomputes only the block holding each sequence's last key (the one a decode
 * step's appended key changes). kbar_scale is ignored (NULL). Device pointers. */
adx_status adx_hisa_block_keys(const adx_operands* ops, int32_t last_only, void* kbar,
                               float* kbar_scale, void* stream);

/* Workspace bytes for adx_index_hisa (blocks_external: a blocks_out array is given), 0 when
 * the arguments are invalid. */
size_t adx_hisa_workspace_size(const adx_operands* ops, int32_t n_blocks, int32_t K,
                               int32_t blocks_external);

/* HISA indexer step. kbar from adx_hisa_block_keys (bf16, read only; kbar_scale is ignored):
 * the block scores take bf16 queries (e4m3 queries decoded with their scales), the token
 * refinement the operands as given. Requires
 * 2 <= n_blocks <= 255, K <= n_blocks * 128, T * n_blocks * 128 < 2^31, H = 64 (else
 * ADX_EUNSUPPORTED). Prefill rows are refined in groups of 4 consecutive rows that score the
 * union of their kept blocks together; each row's Top-K still ranges over its own blocks.
 * topk_idx [T, K] int32 out: key positions (within the row's key range), -1 padded;
 * topk_score [T, K] or NULL; blocks_out [T, n_blocks] or NULL: the kept blocks, -1 padded. */
adx_status adx_index_hisa(const adx_operands* ops, const void* kbar, const float* kbar_scale,
                          int32_t n_blocks, int32_t K, int32_t* topk_idx, float* topk_score,
                          int32_t* blocks_out, void* ws, size_t ws_bytes, void* stream);

/* Shared token banks (ADIndex §4.3, Eq. (13)); `grp` holds the group queries: q = q-bar
 * [Ng, H_g, d], w = w-bar [Ng, H_g], with Ng = grp->T.
 *  prefill layout: group g has members at positions q_pos0 + g*G .. q_pos0 + g*G + G-1.
 *  decode layout:  group g is sequence g, refreshed at position seq_len[g]-1 and reused by
 *                  the next G-1 decode steps; mode must be ADX_BANK_PAPER.
 * bank_idx [Ng, adx_bank_width(B, G, mode)] int32 out: the scan's Top-B (PAPER) or Top-(B-G)
 * (WINDOW) positions in ascending order, -1 padded when fewer keys were scanned, followed by
 * the group's post-anchor positions (PAPER: a+1 .. a+G-1; WINDOW: a .. a+G-1). */
adx_status adx_group_bank(const adx_operands* grp, int32_t G, int32_t B, int32_t mode,
                          int32_t* bank_idx, void* ws, size_t ws_bytes, void* stream);

/* Query-specific refinement (ADIndex §4.3, Eq. (14)) with the full indexer `full`.
 *  prefill layout: the floor(T/G) complete groups use bank row g = row // G; the rows of an
 *                  incomplete trailing group use the flat indexer (§4.3, "Application to
 *                  Prefill and MTP").
 *  decode layout:  row t uses bank row t; candidates are its bank entries <= seq_len[t]-1.
 * bank_idx as written by adx_group_bank with the same (G, B, mode) and layout.
 * topk_idx [T, K] out; topk_score [T, K] or NULL. */
adx_status adx_bank_refine(const adx_operands* full, int32_t G, int32_t B, int32_t mode,
                           const int32_t* bank_idx, int32_t K, int32_t* topk_idx,
                           float* topk_score, void* ws, size_t ws_bytes, void* stream);

/* Decode bank reuse over a packed bank (ADIndex §4.3, Eqs. (13)-(14), decode layout, PAPER
 * banks): the key rows a refresh's banks hold, copied once into contiguous rows, so that the
 * refinement of each following decode step streams them instead of gathering them from the
 * cache.
 * adx_pack_bank_keys: bank_idx [T, W] as written by adx_group_bank (W = adx_bank_width(B, G,
 *   ADX_BANK_PAPER)); writes bank_keys [T, W, d] in the key format and, for e4m3 keys,
 *   bank_kscale [T, W] (else NULL): slot c of row t holds the key at position bank_idx[t, c]
 *   of cache t (zeros, scale 0, for -1 entries). Slots of positions not yet in the cache are
 *   filled by each refinement that sees them.
 * adx_bank_refine_packed: the result of adx_bank_refine (decode layout, same bank_idx) with
 *   the candidate keys read from bank_keys / bank_kscale; it first copies, for each row, the
 *   post-anchor keys at or before its position from the cache into their slots (bank_keys is
 *   updated in place). ws >= adx_workspace_size(ADX_OP_BANK_REFINE_PACKED, full, K, B, G,
 *   ADX_BANK_PAPER). bank_keys 16-byte aligned. */
adx_status adx_pack_bank_keys(const adx_operands* ops, int32_t G, int32_t B,
                              const int32_t* bank_idx, void* bank_keys, float* bank_kscale,
                              void* stream);
adx_status adx_bank_refine_packed(const adx_operands* full, int32_t G, int32_t B,
                                  const int32_t* bank_idx, void* bank_keys, float* bank_kscale,
                                  int32_t K, int32_t* topk_idx, float* topk_score, void* ws,
                                  size_t ws_bytes, void* stream);

/* MTP target verification (ADIndex §4.3, "Application to Prefill and MTP", and Appendix A.2,
 * "Bank Sharing During MTP Target Verification"): each of Bs sequences verifies a window of
 * m draft tokens in one call.
 * full  the full indexer in an MTP layout: q [Bs*m, H, d], w [Bs*m, H] (row b*m + j = window
 *       query j of sequence b), k [Bs, S, d] key caches (S = capacity) with k_scale [Bs, S]
 *       for e4m3, seq_len [Bs] device: keys in sequence b's cache, the window's own included,
 *       so query j sits at position seq_len[b] - m + j (requires m <= seq_len[b] <= S, not
 *       checked on the host). bf16 queries with an e4m3 cache are quantised inside the call.
 * grp   the group queries: q = q-bar [Bs*m/G, H_g, d], q_scale, w = w-bar [Bs*m/G, H_g]
 *       (group g of sequence b is row b*m/G + g), q_dtype, H = H_g; its key fields, S, T and
 *       seq_len are not used (the keys are full's).
 * The window is split into m/G groups of G consecutive queries (m % G == 0, G >= 4, m <= 64);
 * group g's anchor is its first query. When the window's first query sees more than P keys,
 * every group builds a bank of the P best keys over the history its anchor sees (group query,
 * Eq. (13)) and each member refines over bank U {anchor+1 .. own position} (Eq. (14));
 * otherwise the whole window uses the plain indexer (window-level fallback).
 * topk_idx [Bs*m, K] int32 out (ascending positions, -1 padded); topk_score [Bs*m, K] or NULL.
 * bank_out [Bs*m/G, P+m-1] int32 out, or NULL: each group's candidate positions - a banked
 *       window's bank (ascending, -1 padded) then its post-anchor positions, a falling-back
 *       window's every position up to its last member's - then -1 padding.
 * ws    workspace of ws_bytes >= adx_mtp_workspace_size(full, grp, m, G, P, K). */
size_t adx_mtp_workspace_size(const adx_operands* full, const adx_operands* grp, int32_t m,
                              int32_t G, int32_t P, int32_t K);
adx_status adx_index_mtp(const adx_operands* full, const adx_operands* grp, int32_t m, int32_t G,
                         int32_t P, int32_t K, int32_t* topk_idx, float* topk_score,
                         int32_t* bank_out, void* ws, size_t ws_bytes, void* stream);

/* Training-free group queries: the proxy of the PIVOT baseline the paper compares with
 * (ADIndex, Appendix B, "PIVOT": the group's indexing queries and gates, mean-pooled). For
 * every complete group of G consecutive rows (g < T/G) of q [T, H, d] (bf16, or e4m3 codes
 * with q_scale [T]) and w [T, H]:
 *   qbar_out [T/G, Hg, d] bf16 out: the member mean of each of the first Hg heads (summed in
 *            fp32, rounded to nearest even)
 *   wbar_out [T/G, Hg] fp32 out: the member mean of those heads' gates.
 * Device pointers; q and qbar_out 16-byte aligned; d a multiple of 8; no workspace. */
adx_status adx_group_query_mean(int32_t q_dtype, const void* q, const float* q_scale,
                                const float* w, int32_t T, int32_t H, int32_t d, int32_t G,
                                int32_t Hg, void* qbar_out, float* wbar_out, void* stream);

/* The group indexer's queries and gates (ADIndex §4.2, Eqs. (6)-(7)) from the backbone's
 * per-token query latents and hidden states. For each complete group g of G consecutive
 * tokens (anchor t = q_pos0 + g*G):
 *   c-bar = W_pool [max_i c_i ; min_i c_i ; mean_i c_i]   (element-wise over the members)
 *   h-bar = mean_i h_i
 *   q-bar_j = RoPE_t([W_Q c-bar]_j)   (pairs (2i, 2i+1), i < rope_dim/2, rotated by
 *                                      t * rope_base^(-2i/rope_dim))
 *   w-bar_j = sigmoid([W_G h-bar]_j)
 * All pointers are device pointers to bf16 row-major arrays; weights in the [out, in] layout.
 * Requires d_c and d_h multiples of 8; cq, h, w_pool, w_q and w_g 16-byte aligned; H_S <= 64;
 * rope_dim <= 512; T / G <= 65535. Tokens past the last complete group are ignored. Invalid
 * arguments return ADX_EINVAL. The gate projection is taken from h-bar in fp32 inside the
 * pooling kernel, as per-column-block partial sums added in a fixed order (deterministic).
 * The projections W_pool and W_Q run on the library's tcgen05 GEMM (bf16 operands, fp32
 * accumulation); c-bar is rounded to bf16 between them. The workspace starts with the device
 * status word (ADX_STATUS_BYTES, zeroed once before the first call; read it with
 * adx_read_device_status). */
typedef struct {
  const void* cq;      /* [T, d_c] query latents */
  const void* h;       /* [T, d_h] normalized hidden states */
  const void* w_pool;  /* [d_c, 3*d_c] */
  const void* w_q;     /* [H_S*d, d_c] */
  const void* w_g;     /* [H_S, d_h] */
  int32_t T, d_c, d_h, H_S, d, rope_dim;  /* rope_dim even, <= d */
  float rope_base;
  int64_t q_pos0;      /* position of token 0 */
} adx_group_indexer;

/* Workspace bytes for adx_group_indexer_queries, 0 for invalid arguments. */
size_t adx_group_indexer_workspace_size(const adx_group_indexer* gi, int32_t G);

/* qbar_out [T/G, H_S, d] bf16 out, wbar_out [T/G, H_S] fp32 out (device). */
adx_status adx_group_indexer_queries(const adx_group_indexer* gi, int32_t G, void* qbar_out,
                                     float* wbar_out, void* ws, size_t ws_bytes, void* stream);

/* Calibration statistic of layer-wise reuse (ADIndex §4.1, Eq. (4)): for every complete group
 * of G consecutive rows of topk_idx [T, K] (rows g*G .. g*G+G-1, g < T/G), the number of
 * distinct positions in [0, S) among the group's Top-K sets (-1 padding and other values
 * outside [0, S) are not positions). U^max of the page is the maximum over groups.
 * topk_idx  device, as written by the flat indexer (adx_index_prefill)
 * union_out [T/G] int32 device out
 * Needs no workspace; S up to 200 KiB of bitmap (6.5M positions), else ADX_EUNSUPPORTED. */
adx_status adx_group_union_sizes(const int32_t* topk_idx, int32_t T, int32_t K, int32_t G,
                                 int32_t S, int32_t* union_out, void* stream);

/* Shared-bank coverage (ADIndex §1, Figure 1(c), and Appendix B.4: the fraction of a query's
 * original Top-K selections that its group's shared bank includes). For every query row i of
 * a complete group g = i / G (g < T / G):
 *   count_out[i] = the number of positions (entries >= 0) in row i of topk_idx [T, K], the
 *                  original indexer's Top-K (as written by adx_index_prefill);
 *   hits_out[i]  = how many of them row g of bank_idx [T / G, bank_w] holds (entries < 0 are
 *                  padding). Pass the bank rows as adx_group_bank writes them: the bank plus
 *                  the post-anchor (PAPER) or window (WINDOW) positions every member scans,
 *                  so hits == count exactly when refinement recovers the full Top-K.
 * coverage_i = hits_out[i] / count_out[i]. Positions must lie in [0, S); larger ones count as
 * not held. Device pointers; no workspace; S up to 200 KiB of bitmap (6.5M positions), else
 * ADX_EUNSUPPORTED. */
adx_status adx_bank_coverage(const int32_t* topk_idx, int32_t T, int32_t K,
                             const int32_t* bank_idx, int32_t bank_w, int32_t G, int32_t S,
                             int32_t* hits_out, int32_t* count_out, void* stream);

/* Failure-detection check (no counterpart in the paper): one CTA waits, with the bounded wait
 * the indexer's kernels use, on a barrier that nothing completes; after timeout_ns (at most
 * 1 s) the wait gives up and records ADX_ETIMEOUT in the status word of `ws`, as a real wait
 * that ran out would. The device stays usable; adx_read_device_status(ws) then returns
 * ADX_ETIMEOUT (and clears it). */
adx_status adx_check_wait_timeout(void* ws, uint64_t timeout_ns, void* stream);

/* Synchronises `stream`, returns the device status recorded in `ws` (ADX_OK if none) and
 * clears it. */
adx_status adx_read_device_status(void* ws, void* stream);

/* Static description of a status code. */
const char* adx_status_string(adx_status s);

/* ADX_ABI_VERSION of the built library. */
int32_t adx_abi_version(void);

/* Instrumentation (no counterpart in the paper). When `events` (n cudaEvent_t handles,
 * host array, owned by the caller) is set, later calls on this host thread record
 * events[0] / events[1] on their stream right before / after each scoring-kernel launch and
 * events[2] / events[3] before / after each Top-K selection; later records overwrite
 * earlier ones. NULL switches it off. */
void adx_set_timing_events(void* const* events, int32_t n);

/* Number of kernels this library has launched in the process so far. */
int64_t adx_launch_count(void);

/* Bytes of the fixed device scratch array behind adx_index_prefill_noalloc. */
#define ADX_STATIC_SCRATCH_BYTES (32u << 20)

/* adx_index_prefill for callers that cannot allocate device memory (an engine that plans all
 * device buffers ahead in its own arena, a plugin host without an allocator, plain C code):
 * same operands, outputs and results as adx_index_prefill, but no workspace argument. The
 * paper has no counterpart; this exists only for such callers.
 * Scratch is a fixed array of ADX_STATIC_SCRATCH_BYTES inside the library; every GPU that
 * loads the library holds it until the process exits. Problems that need more (see
 * adx_workspace_size(ADX_OP_PREFILL, ...)) return ADX_EWORKSPACE before any launch, invalid
 * or unsupported operands with the codes adx_index_prefill returns; nothing is ever
 * allocated. The first call on a device looks up the array's device address with that
 * device current (again after a device reset): make it before any stream capture. All calls
 * on a device share the array, so calls that overlap on the GPU race; serialise them. Each call clears the status word on
 * `stream` first; device_status (a device int32, or NULL) receives the call's device status
 * (ADX_OK or ADX_ETIMEOUT) asynchronously on `stream`. */
adx_status adx_index_prefill_noalloc(const adx_operands* ops, int32_t K, int32_t* topk_idx,
                                     float* topk_score, int32_t* device_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ADX_H_ */

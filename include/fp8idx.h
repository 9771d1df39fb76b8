/*
 * fp8idx.h -- C ABI of the B200 (sm_100a) fp8 MQA indexer library.
 *
 * The operation (the sparse-attention indexer of the
 * "bench_mqa_logits_chunking.py" page: module docstring, `_build` and
 * `_run_chunked`, which call `deep_gemm.fp8_mqa_logits(q, (kv, kv_scales),
 * weights, ks, ke)` and then `fast_topk_transform_fused(score, lengths, ...,
 * topk, row_starts)`; GLM-5.1 shapes index_n_heads = 32, index_head_dim =
 * 128, index_topk = 2048):
 *
 *   logits[i,j] = s[j] * sum_{h<H} w[i,h] * max(0, sum_{d<D} q[i,h,d] * k[j,d])
 *                 for max(ks[i],0) <= j < min(ke[i],n), and -inf otherwise;
 *   out[i,:]    = the k key indices of row i with the largest logits, ties
 *                 going to the lower index, padded with -1 when fewer than
 *                 k keys are valid.  The order inside a row is unspecified.
 *
 * q and k are fp8 e4m3fn bytes (the "e4m3fn" format named on the
 * "Serve GLM-5.3-Flash on SM80" page, commit notes); s and w are fp32; ks
 * and ke are int32.  H is 32 (the pages' index_n_heads) or 64; D is 128.
 *
 * Conventions shared by every call:
 *   - All data pointers are DEVICE pointers owned by the caller.  The library
 *     never allocates, frees, synchronises the stream or reads device data on
 *     the host (except fp8idx_read_device_status, which is for tests).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     only enqueues work on it and returns.
 *   - Layouts are dense row-major: q [m, H, D], k [n, D], s [n], w [m, H],
 *     ks/ke [m], out [m, topk].
 *   - Alignment: q, k and k_pages 16 bytes (TMA), s_pages 16 bytes (bulk
 *     copies of page scales); everything else 4 bytes;
 *     workspaces 256 bytes.
 *   - Errors are reported before anything is launched and leave the outputs
 *     untouched: FP8IDX_EINVAL (null pointer, misalignment, negative size,
 *     topk outside [1, 2048], ld_logits < n), FP8IDX_EUNSUPPORTED (H not 32
 *     or 64, D != 128, page_size != 64, rows per request outside [1, 8], or
 *     above 4 with H = 64),
 *     FP8IDX_EWORKSPACE (workspace smaller than the *_workspace() size),
 *     FP8IDX_ECUDA (a CUDA call failed; see fp8idx_last_error()).
 *     m == 0 (or B == 0) is a no-op returning FP8IDX_OK.
 *   - Device-side problems that the host cannot see (a block-table entry
 *     outside [0, num_pages), a sequence length beyond max_blocks * 64, a
 *     pipeline wait that timed out) set bits in a status word at the head
 *     of the workspace; read it with fp8idx_read_device_status().
 *   - fp8 inputs holding NaN bytes (0x7F / 0xFF) give unspecified output.
 */
#ifndef FP8IDX_H_
#define FP8IDX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  FP8IDX_OK = 0,
  FP8IDX_EINVAL = 1,
  FP8IDX_EUNSUPPORTED = 2,
  FP8IDX_EWORKSPACE = 3,
  FP8IDX_ECUDA = 4
};

/* device status bits (fp8idx_read_device_status) */
enum {
  FP8IDX_STATUS_WAIT_TIMEOUT = 1,   /* a pipeline wait gave up; outputs are invalid      */
  FP8IDX_STATUS_BAD_PAGE = 2,       /* a block-table entry outside [0, num_pages)        */
  FP8IDX_STATUS_SEQ_TOO_LONG = 4,   /* seq_lens[b] > max_blocks * page_size (clamped)    */
  FP8IDX_STATUS_CAND_OVERFLOW = 8   /* internal: a candidate was dropped; outputs invalid */
};

/*
 * Materialised logits (the `fp8_mqa_logits` call of the
 * "bench_mqa_logits_chunking.py" page, `_run_chunked`), except that every
 * entry outside [ks[i], ke[i]) is written as -inf.
 *   q       [m, H, D] e4m3 bytes          k  [n, D] e4m3 bytes
 *   s       [n] fp32 key scales           w  [m, H] fp32 head weights
 *   ks, ke  [m] int32 (clamped to [0, n] on the device)
 *   logits  [m, ld_logits] fp32 output; columns [0, n) of every row are
 *           written, ld_logits >= n.  Needs m * ld_logits * 4 bytes: callers
 *           with large m * n chunk the rows (one call per row chunk, passing
 *           offset q, w, ks, ke and logits pointers).
 * No workspace.  Device status of this call: fp8idx_read_device_status(NULL, ...).
 */
int fp8idx_mqa_logits(const uint8_t* q, const uint8_t* k, const float* s, const float* w,
                      const int32_t* ks, const int32_t* ke, int64_t m, int64_t n, int H, int D,
                      float* logits, int64_t ld_logits, void* stream);

/*
 * Top-k of materialised logit rows (the `fast_topk_transform_fused(score,
 * lengths, ..., topk, row_starts)` call of the same page with the identity
 * page table): for each row i, the topk largest logits[i, j] over
 * max(ks[i],0) <= j < min(ke[i],n), ties to the lower j, padded with -1.
 *   logits [m, ld] fp32; ks, ke [m] int32; out [m, topk] int32.
 * No workspace.
 */
int fp8idx_topk_rows(const float* logits, int64_t ld, const int32_t* ks, const int32_t* ke,
                     int64_t m, int64_t n, int topk, int32_t* out, void* stream);

/*
 * Fused logits + top-k: the same result as fp8idx_mqa_logits followed by
 * fp8idx_topk_rows, computed by streaming over 128-key tiles without ever
 * holding the m x n logits.  Arguments as above; out_idx [m, topk] int32;
 * out_vals [m, topk] fp32 receives the matching logits (-inf padding) and
 * may be NULL.  ws / ws_bytes: caller-owned device workspace of at least
 * fp8idx_mqa_logits_topk_workspace(m, n, H, D, topk) bytes, 256-byte
 * aligned, reused freely between calls on the same stream (calls that may
 * overlap on the device need separate workspaces).  The size depends on the
 * current device's SM count.
 */
size_t fp8idx_mqa_logits_topk_workspace(int64_t m, int64_t n, int H, int D, int topk);
int fp8idx_mqa_logits_topk(const uint8_t* q, const uint8_t* k, const float* s, const float* w,
                           const int32_t* ks, const int32_t* ke, int64_t m, int64_t n, int H,
                           int D, int topk, int32_t* out_idx, float* out_vals, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * Paged decode / verify form (the paged MQA logits named on the
 * "Serve GLM-5.3-Flash on SM80" page, commit notes): B requests with R query
 * rows each (MTP width R).  Key j of request b is slot j % 64 of physical
 * page block_table[b * max_blocks + j / 64]; row t of request b (global row
 * b * R + t) sees keys [0, seq_lens[b] - R + t + 1), clamped to
 * [0, seq_lens[b]].  Output indices are logical token positions.
 *   q           [B * R, H, D] e4m3 bytes     w        [B * R, H] fp32
 *   k_pages     [num_pages, 64, D] e4m3       s_pages  [num_pages, 64] fp32
 *   block_table [B, max_blocks] int32 (entries past a request's pages are
 *               never read)                   seq_lens [B] int32
 *   out_idx     [B * R, topk] int32           out_vals [B * R, topk] fp32 or NULL
 * R is 1 (decode) to 8 (MTP verify widths; the megakernels page names
 * q4-q8), at most 4 with H = 64; page_size must be 64.
 */
size_t fp8idx_paged_mqa_logits_topk_workspace(int64_t B, int R, int max_blocks, int H, int D,
                                              int topk);
int fp8idx_paged_mqa_logits_topk(const uint8_t* q, const uint8_t* k_pages, const float* s_pages,
                                 const float* w, const int32_t* block_table,
                                 const int32_t* seq_lens, int64_t B, int R, int max_blocks,
                                 int64_t num_pages, int page_size, int H, int D, int topk,
                                 int32_t* out_idx, float* out_vals, void* ws, size_t ws_bytes,
                                 void* stream);

/*
 * fp8idx_paged_mqa_logits_topk with the top-k transform applied where the
 * indices are written: each selected position j of request b comes out as
 * its physical KV slot block_table[b, j / 64] * 64 + j % 64, the slot the
 * sparse attention reads (the paged form of `fast_topk_transform_fused`'s
 * page-table mapping on the "bench_mqa_logits_chunking.py" page).  -1
 * padding stays -1; a selected key on a page entry outside [0, num_pages)
 * (which also sets the BAD_PAGE status bit) comes out as -1.  Same
 * arguments, workspace size, ownership and errors as
 * fp8idx_paged_mqa_logits_topk; the values in out_vals are unchanged.
 */
int fp8idx_paged_mqa_logits_topk_slots(const uint8_t* q, const uint8_t* k_pages, const float* s_pages,
                                       const float* w, const int32_t* block_table,
                                       const int32_t* seq_lens, int64_t B, int R, int max_blocks,
                                       int64_t num_pages, int page_size, int H, int D, int topk,
                                       int32_t* out_slots, float* out_vals, void* ws, size_t ws_bytes,
                                       void* stream);

/*
 * Allocation-free variant of fp8idx_mqa_logits_topk (the pages have no
 * counterpart: it exists for callers that cannot allocate device memory at
 * call time, such as code inside a framework-owned CUDA graph or a runtime
 * with a fixed, pre-planned memory budget).  Same arguments and result as
 * fp8idx_mqa_logits_topk without ws / ws_bytes: the library keeps a fixed
 * 64 MiB device array as its workspace, created when the library's device
 * code loads on a GPU and held until the process exits.  The first call on a
 * device looks up that array's address; make it before any stream capture.
 * Large problems run on fewer SMs so that the workspace fits; a problem that
 * does not fit at all returns FP8IDX_EWORKSPACE.  All calls share the array:
 * calls that can overlap on the GPU race and must be serialised by the
 * caller.  The status block of the last call is the head of that array: read
 * it with fp8idx_read_device_status(FP8IDX_NOALLOC_WS, ...) (and the stats
 * likewise).  The array's device address is looked up once per device index
 * and kept for the life of the process, so the library must not be used
 * across a cudaDeviceReset (or any teardown of the primary context), after
 * which the array may live elsewhere.
 */
#define FP8IDX_NOALLOC_WS ((const void*)1)
int fp8idx_mqa_logits_topk_noalloc(const uint8_t* q, const uint8_t* k, const float* s,
                                   const float* w, const int32_t* ks, const int32_t* ke, int64_t m,
                                   int64_t n, int H, int D, int topk, int32_t* out_idx,
                                   float* out_vals, void* stream);

/*
 * Key quantisation into the paged key pool: the producer of k_pages /
 * s_pages above (the `act_quant` step and the fp8 k-pool stores named on the
 * "Serve GLM-5.3-Flash on SM80" page, commit notes).  The pages do not print
 * the scale rule; the one taken is a per-token fp32 scale
 *     s_t = max(max_d |x[t,d]|, 1e-4) / 448
 * and codes e4m3(x[t,d] / s_t), rounded to nearest even and saturated at
 * +-448, both computed in fp32.  Token t goes to pool slot slot[t]
 * (physical page slot[t] / 64, row slot[t] % 64); a slot outside
 * [0, num_slots) is skipped.
 *   x       [T, D] bf16 bit patterns, D must be 128, 8-byte aligned
 *   slot    [T] int64, 8-byte aligned
 *   k_pool  [num_slots, 128] e4m3 bytes (k_pages viewed as slots), 4-byte aligned
 *   s_pool  [num_slots] fp32 (s_pages viewed as slots), 4-byte aligned
 * NaN elements of x are left out of the row maximum and get a NaN code
 * (0x7F or 0xFF); the other codes of the row are unaffected.
 * Slots not named by any token are left untouched; two tokens naming one
 * slot race.  No workspace.
 */
int fp8idx_act_quant_store(const uint16_t* x, int64_t T, int D, const int64_t* slot, int64_t num_slots,
                           uint8_t* k_pool, float* s_pool, void* stream);

/*
 * Index preparation (the `gen_nsa_ks_ke` step of the "reuse inference
 * metadata and streamline FP8 prefill" page: its description table, the
 * walkthrough of the ragged-index copy, and the review's expected ragged
 * buffer).  B requests are laid out back to back in one ragged key space:
 * request b owns key positions [koff_b, koff_b + seq_len[b]), koff_b the sum
 * of the earlier seq_len; its query rows (its last q_len[b] tokens) are rows
 * [qoff_b, qoff_b + q_len[b]) of the batch, qoff_b the sum of the earlier
 * q_len.  For row t of request b:
 *     ks = koff_b,  ke = koff_b + clamp(seq_len[b] - q_len[b] + t + 1, 0, seq_len[b]),
 *     row_table = req_idx[b]                          (the row's token-table row),
 * and, when `ragged` is not NULL, the token slots of every request are copied
 * in the same order (the long-context copy, parallel over all positions):
 *     ragged[koff_b + p] = req_to_token[req_idx[b] * ld_table + p],  p < seq_len[b]
 * (-1 where req_idx[b] is outside [0, table_rows) or p >= ld_table).
 *   seq_len, q_len, req_idx [B] int32 (negative lengths count as 0); B <= 8192
 *   req_to_token  [table_rows, ld_table] int32 token slots (LightLLM's
 *                 req_to_token_indexs; several requests may share a row, as
 *                 the HOLD padding requests do)
 *   ks, ke        [q_cap] int32; rows past the batch's sum of q_len are
 *                 written empty (ks = ke = 0, row_table = -1)
 *   row_table     [q_cap] int32 or NULL
 *   ragged        [ragged_cap] int32 or NULL; positions past the batch's sum
 *                 of seq_len are not written
 * The sums are formed on the device, so the call never reads device data on
 * the host: the caller sizes q_cap and ragged_cap as upper bounds, and every
 * key position must stay below 2^31.  No workspace.
 */
int fp8idx_prepare_ragged(const int32_t* seq_len, const int32_t* q_len, const int32_t* req_idx, int B,
                          const int32_t* req_to_token, int64_t table_rows, int64_t ld_table, int32_t* ks,
                          int32_t* ke, int32_t* row_table, int64_t q_cap, int32_t* ragged, int64_t ragged_cap,
                          void* stream);

/*
 * Top-k transform: selected key positions to physical slots through a page
 * table (the `page_table_size_1` argument of `fast_topk_transform_fused`,
 * "bench_mqa_logits_chunking.py" page; with page_size 64 the block table of
 * the paged form).  For row i and each r < topk:
 *     p = idx[i, r] - row_base[i]           (row_base NULL: 0)
 *     t = row_table[i]                      (row_table NULL: i / rows_per_table_row)
 *     out[i, r] = page_table[t * ld_table + p / page_size] * page_size + p % page_size
 * and -1 where idx[i, r] is negative, p < 0, t is outside [0, table_rows),
 * p / page_size >= ld_table, or the table entry is negative.  With the rows
 * of fp8idx_prepare_ragged: row_base = ks, row_table = its row_table, the
 * token table and page_size 1.  With the paged form's output: row_base NULL,
 * rows_per_table_row = R, the block table and page_size 64.
 *   idx, out [rows, topk] int32 (may be the same buffer); slots must fit int32.
 * No workspace.
 */
int fp8idx_topk_transform(const int32_t* idx, int64_t rows, int topk, const int32_t* row_base,
                          const int32_t* row_table, int rows_per_table_row, const int32_t* page_table,
                          int64_t table_rows, int64_t ld_table, int page_size, int32_t* out, void* stream);

/*
 * Tests and diagnostics.  fp8idx_read_device_status synchronises `stream`
 * and copies the status word written by the last call that used workspace
 * `ws` into *status_out.  ws == NULL names the last fp8idx_mqa_logits call,
 * ws == FP8IDX_NOALLOC_WS the last fp8idx_mqa_logits_topk_noalloc call on
 * the current device.
 */
int fp8idx_read_device_status(const void* ws, int* status_out, void* stream);
/* Copies the first `count` (<= 64) 32-bit words of a workspace's status block:
 * word 0 the status bits above; for fp8idx_mqa_logits_topk and the paged form,
 * word 1 the in-kernel compactions of a full candidate buffer, word 2 the rows
 * whose final selection took the general radix path, word 3 the candidates
 * collected (summed over rows and key chunks), word 4 the largest
 * boundary-bin population, word 5 the rows whose estimated threshold the
 * check rejected (their row block or request was recomputed exactly).
 * Synchronises `stream`; for tuning and tests. */
int fp8idx_read_device_stats(const void* ws, uint32_t* out, int count, void* stream);
/* Message for the last non-OK return on this thread ("" if none). */
const char* fp8idx_last_error(void);
/* Number of SMs of the current device (what the workspace sizes assume). */
int fp8idx_num_sms(void);
/* Upper bound in nanoseconds on any single pipeline wait inside a kernel
 * (default 2e9), taken by calls made after it.  With 0, every wait that does
 * not succeed at once gives up: the kernel sets FP8IDX_STATUS_WAIT_TIMEOUT,
 * drains its own copies and returns (the tests use this to exercise the
 * timeout path). */
void fp8idx_set_wait_limit_ns(uint64_t ns);
/* Tests only (no counterpart on the pages).  While `on` is nonzero, each CTA
 * of the fused and paged calls made afterwards never issues the load of its
 * first key tile, so the MMA's bounded wait on that tile runs out after the
 * wait limit: the call returns with FP8IDX_STATUS_WAIT_TIMEOUT set and its
 * outputs invalid, and the context stays usable.  Off by default. */
void fp8idx_debug_withhold_first_tile(int on);

#ifdef __cplusplus
}
#endif

#endif /* FP8IDX_H_ */

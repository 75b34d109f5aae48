/*
 * qsa.h - C ABI of the QSA (Qwen Sparse Attention) MQA indexer score for
 * NVIDIA B200 (sm_100a).
 *
 * The indexer scores compressed 4-token key blocks for every query token:
 *
 *     score[t, n] = scale * sum_{h<4} max(0, q[t, h, :] . k[n, :])
 *
 * with 4 query heads of dimension 128 sharing one compressed key head of
 * dimension 128, and scale = 1/sqrt(128) by default (QSA docs, MATE, section
 * "MQA score": "Scores sum the four head-wise ReLU dot products, scaled by
 * 1/sqrt(128)"; "scale is a multiplier").  Blocks that are not yet complete
 * or lie in the future are masked to -inf.  A query token at logical
 * position pos = seq_len - query_len + i (vLLM qsa_cache.py,
 * "_logical_positions") sees the compressed keys
 *
 *     n < visible = max(0, min((pos + 1) / 4, seq_len / 4))   (floor division)
 *
 * (vLLM qsa_cache.py, metadata kernel, "visible_blocks"; the vLLM PR
 * "Separate prefill and decode paths for QSA indexer", section "Main changes",
 * names the same quantity).
 *
 * Conventions shared by every call:
 *  - Pointers named q, k, k_cache, page_table, seq_lens, ks, ke, lengths,
 *    scores, out, idx, workspace are DEVICE pointers owned by the caller.
 *    The library allocates nothing, never synchronises the stream and never
 *    reads device memory from the host; every call is asynchronous on
 *    `stream` (a cudaStream_t; NULL means the legacy default stream).
 *  - bf16 / fp16 tensors are passed as raw pointers with strides in ELEMENTS;
 *    the feature (last) stride is always 1.
 *  - Host-side validation runs before any launch.  On a non-OK status nothing
 *    was launched and qsa_last_error_detail() describes the problem.
 *  - Kernels never trap.  A device-side wait that runs out of time sets a bit
 *    in the library's device error word (qsa_device_error) and the kernel
 *    returns early; the output is then incomplete.
 */
#ifndef QSA_H_
#define QSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qsa_status {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARG = 1, /* a size, count, pointer or value is out of range */
  QSA_ERR_ALIGNMENT = 2,   /* a base address or stride breaks the layout rules */
  QSA_ERR_UNSUPPORTED = 3, /* a configuration this build does not implement */
  QSA_ERR_WORKSPACE = 4,   /* the workspace is too small */
  QSA_ERR_CUDA = 5         /* a CUDA runtime/driver call or a launch failed */
} qsa_status_t;

/* Bits of the device error word. */
#define QSA_DEVERR_WAIT_TIMEOUT 0x1u /* an mbarrier wait ran out of time */
#define QSA_DEVERR_SELECT 0x2u       /* top-k threshold search did not converge */

/* Static text for a status code. */
const char* qsa_status_string(qsa_status_t status);

/* Detail of the last non-OK status returned on the calling host thread
 * (thread-local; empty string if none). */
const char* qsa_last_error_detail(void);

/* Reads the device error word of the current device into *bits and clears
 * it.  This call synchronises the device (it is for tests and diagnostics,
 * never for the hot path). */
qsa_status_t qsa_device_error(uint32_t* bits);

/* qsa_selftest_bounded_wait - a diagnostic of the failure handling above; the
 * pages have no counterpart.  Launches one warp on `stream` whose first
 * thread waits, with the same bounded wait the kernels use and a limit of
 * timeout_ns (at most 10 s), on an mbarrier phase that nothing completes
 * (arrive == 0) or that the thread completes itself first (arrive != 0).  A
 * wait that runs out sets QSA_DEVERR_WAIT_TIMEOUT in the device error word and
 * the kernel returns; the context stays usable.  For tests. */
qsa_status_t qsa_selftest_bounded_wait(uint64_t timeout_ns, int32_t arrive, void* stream);

/*
 * qsa_mqa_decode - decode and speculative-decode scores over a paged
 * compressed key cache.
 *
 * Defined by the QSA docs (MATE), section "MQA score" ("qsa_mqa_decode takes
 * paged compressed keys [pages, page_size, 1, dim], a page table and
 * compressed context lengths"; the context length is passed here in TOKENS
 * so that each of the Q query tokens gets its own causal visible count), with
 * the page addressing of vLLM qsa_cache.py, "_logical_to_physical_qsa_slots".
 *
 *   q          bf16 [B, Q, 4, 128]; element (b, i, h, c) at
 *              q + b*q_stride_b + i*q_stride_t + h*q_stride_h + c.
 *              Strides are non-negative multiples of 8; a stride of 0
 *              broadcasts that axis.  16-byte aligned.
 *   k_cache    bf16 [num_pages, page_size, 1, 128]; row r of page p at
 *              k_cache + p*k_page_stride + r*k_row_stride.  16-byte aligned,
 *              both strides multiples of 8, k_row_stride >= 128.
 *   page_size  8 .. 1024 rows per page.  The QSA docs list 8, 16, 32 and 64
 *              as the native sizes; the vLLM PR measures at 196, its
 *              production size.  Sizes that are not powers of two take a
 *              per-key page lookup (integer multiply-shift division).
 *   page_table int32 [B, max_pages], row stride pt_stride (>= max_pages).
 *              Key n of request b lives in page page_table[b, n / page_size]
 *              at row n % page_size.  Entries may be -1; an entry that is
 *              negative or >= num_pages (or a block past max_pages) masks the
 *              keys it would hold to -inf.
 *   seq_lens   int32 [B]: tokens of request b, its Q query tokens included.
 *              Query row i sits at logical position seq_lens[b] - Q + i.
 *   Q          query tokens per request, 1..4 (4 = three speculative tokens).
 *   scale      score multiplier (1/sqrt(128) for the QSA indexer); finite.
 *   out        fp32 [B, Q, W]; element (b, i, n) at
 *              out + b*out_stride_b + i*out_stride_t + n.
 *              out[b, i, n] = score for n < visible(b, i), else -inf, for
 *              every n < W (columns past the visible keys are filled with
 *              -inf).  W >= max visible is the caller's choice; keys at
 *              n >= W are not scored.  out must not overlap any input.
 *              Requests are launched in groups of at most
 *              min(8192, floor((2^32 - 1) / ceil(W / 8))) so that the
 *              kernel's 32-bit count of 8-key tiles cannot overflow.
 */
qsa_status_t qsa_mqa_decode(const void* q, int64_t q_stride_b, int64_t q_stride_t, int64_t q_stride_h,
                            const void* k_cache, int64_t num_pages, int32_t page_size, int64_t k_page_stride,
                            int64_t k_row_stride, const int32_t* page_table, int64_t pt_stride,
                            int32_t max_pages, const int32_t* seq_lens, int32_t B, int32_t Q, float scale,
                            float* out, int64_t out_stride_b, int64_t out_stride_t, int32_t W, void* stream);

/* qsa_mqa_decode_f16 - qsa_mqa_decode with fp16 q and k_cache (QSA docs,
 * MATE, section "MQA score": queries and keys are BF16 or FP16).  The
 * products accumulate in fp32 as for bf16; arguments, layout and errors as
 * qsa_mqa_decode. */
qsa_status_t qsa_mqa_decode_f16(const void* q, int64_t q_stride_b, int64_t q_stride_t, int64_t q_stride_h,
                                const void* k_cache, int64_t num_pages, int32_t page_size, int64_t k_page_stride,
                                int64_t k_row_stride, const int32_t* page_table, int64_t pt_stride,
                                int32_t max_pages, const int32_t* seq_lens, int32_t B, int32_t Q, float scale,
                                float* out, int64_t out_stride_b, int64_t out_stride_t, int32_t W, void* stream);

/*
 * qsa_mqa_decode_fp8 - qsa_mqa_decode over an fp8 E4M3 compressed key cache.
 *
 * The cache dtype is the optional e4m3 indexer cache of vLLM qsa_cache.py
 * (the QSA state backend's cache dtypes "fp8" / "fp8_e4m3"); its writer
 * (vLLM qsa_prepare.py, "_to_dst_dtype") rounds a key to bf16, divides it by
 * the cache scale and stores the E4M3 code.  Key element c of a row is read
 * as E4M3(code) * k_scale, and the score is the bf16 one on those keys:
 * scale * sum_h max(0, q_h . k).  Arguments as qsa_mqa_decode, except:
 *
 *   k_cache    E4M3 codes (one byte each) [num_pages, page_size, 1, 128],
 *              strides in bytes: 16-byte aligned, k_row_stride and
 *              k_page_stride multiples of 16, k_row_stride >= 128.  The NaN
 *              codes 0x7f / 0xff are outside the contract (the writer does
 *              not produce them for finite keys).
 *   k_scale    dequantisation scale: finite and > 0 (scale * k_scale finite).
 */
qsa_status_t qsa_mqa_decode_fp8(const void* q, int64_t q_stride_b, int64_t q_stride_t, int64_t q_stride_h,
                                const void* k_cache, float k_scale, int64_t num_pages, int32_t page_size,
                                int64_t k_page_stride, int64_t k_row_stride, const int32_t* page_table,
                                int64_t pt_stride, int32_t max_pages, const int32_t* seq_lens, int32_t B, int32_t Q,
                                float scale, float* out, int64_t out_stride_b, int64_t out_stride_t, int32_t W,
                                void* stream);

/*
 * qsa_mqa_prefill - prefill scores of packed query rows against shared keys
 * with one key interval per row.
 *
 * Defined by the QSA docs (MATE), section "MQA score" ("qsa_mqa_prefill takes
 * packed queries, shared keys and per-row key intervals").  Column j of row t
 * holds key ks[t] + j (request-local block index, the frame in which the
 * docs' "Core Attention" section consumes selected blocks).
 *
 *   q        bf16 [T, 4, 128]; element (t, h, c) at q + t*q_stride_t +
 *            h*q_stride_h + c.  16-byte aligned, strides positive multiples
 *            of 8 (q_stride_t is free when T == 1).
 *   k        bf16 [Nk, 128], row stride k_stride (multiple of 8, >= 128).
 *            16-byte aligned.
 *   ks, ke   int32 [T]: row t sees keys n with max(ks[t], 0) <= n <
 *            min(ke[t], Nk); an empty interval gives a row of -inf.
 *   out      fp32 [T, W], row stride out_stride (>= W when T > 1):
 *            out[t, j] = score(t, ks[t] + j) if that key is in the row's
 *            interval, else -inf, for every j < W.  Must not overlap inputs.
 *   T        rows, 0 <= T <= 2^31 - 1 (larger T returns
 *            QSA_ERR_UNSUPPORTED); the rows are launched in groups of at
 *            most 131,072.
 */
qsa_status_t qsa_mqa_prefill(const void* q, int64_t q_stride_t, int64_t q_stride_h, const void* k,
                             int64_t k_stride, int64_t Nk, const int32_t* ks, const int32_t* ke, int64_t T,
                             float scale, float* out, int64_t out_stride, int32_t W, void* stream);

/* qsa_mqa_prefill_f16 - qsa_mqa_prefill with fp16 q and k (QSA docs, MATE,
 * section "MQA score": queries and keys are BF16 or FP16).  The products
 * accumulate in fp32 as for bf16; arguments, layout and errors as
 * qsa_mqa_prefill. */
qsa_status_t qsa_mqa_prefill_f16(const void* q, int64_t q_stride_t, int64_t q_stride_h, const void* k,
                                 int64_t k_stride, int64_t Nk, const int32_t* ks, const int32_t* ke, int64_t T,
                                 float scale, float* out, int64_t out_stride, int32_t W, void* stream);

/*
 * qsa_prefill_intervals - per-row key intervals of a packed prefill batch,
 * computed on the device (one thread per row).
 *
 * Sequence s owns query rows cu_seqlens_q[s] .. cu_seqlens_q[s+1]-1, has
 * seq_lens[s] tokens in all (cached prefix plus its query rows) and its
 * compressed keys start at key_offsets[s] in the packed key array.  Row
 * t = cu_seqlens_q[s] + i gets ks[t] = key_offsets[s] and
 * ke[t] = key_offsets[s] + visible(pos), pos = seq_lens[s] - qlen_s + i
 * (vLLM qsa_cache.py, "_logical_positions" and "visible_blocks").
 *
 *   cu_seqlens_q int32 [S + 1], non-decreasing, cu_seqlens_q[0] == 0,
 *                cu_seqlens_q[S] == T.  seq_lens, key_offsets int32 [S].
 *   ks, ke       int32 [T] outputs.
 */
qsa_status_t qsa_prefill_intervals(const int32_t* cu_seqlens_q, const int32_t* seq_lens,
                                   const int32_t* key_offsets, int32_t S, int64_t T, int32_t* ks, int32_t* ke,
                                   void* stream);

/*
 * qsa_topk - per-row top-k block selection over score rows.
 *
 * The selection step between the indexer and core attention (QSA docs,
 * MATE: the caller keeps the top-scoring blocks; "Core Attention": block
 * hint widths from 1 to 512; the vLLM PR's review thread uses top-k widths
 * 512, 1024 and 2048).  Among columns j < len(r) of row r whose score is not
 * -inf (masked blocks are never selected) the k largest are kept, ties going
 * to the lower column; their column indices are written in ascending order
 * to idx[r, 0..], and the remaining slots are -1.  -0.0 and +0.0 compare
 * equal.  NaN scores are never selected.
 *
 *   scores   fp32 [rows, W], row stride score_stride (>= W when rows > 1),
 *            4-byte aligned.
 *   lengths  int32 [rows] or NULL: len(r) = min(max(lengths[r], 0), W);
 *            with NULL, len(r) = W.
 *   k        1..2048.
 *   idx      int32 [rows, k], row stride idx_stride (>= k when rows > 1).
 *   W        1..65536.
 */
qsa_status_t qsa_topk(const float* scores, int64_t score_stride, const int32_t* lengths, int64_t rows,
                      int32_t W, int32_t k, int32_t* idx, int64_t idx_stride, void* stream);

/*
 * qsa_topk_ws - qsa_topk with a caller workspace: the same selection and
 * result, computed in passes that stage each row's candidates in the
 * workspace (a filter pass over the scores, a per-row selection on the
 * staged candidates, an exact pass over the rows the first two cannot
 * resolve), which is faster for many rows.
 *
 *   workspace        device memory of at least
 *                    qsa_topk_workspace_size(rows, W, k) bytes, 256-byte
 *                    aligned, not overlapping scores, lengths or idx.  Its
 *                    contents on entry do not change the result; a workspace
 *                    reused from one call to the next carries the selection's
 *                    threshold predictions along, which only speeds the next
 *                    call up.  Contents on return are undefined.
 *   workspace_bytes  its size.
 * Other arguments as for qsa_topk, checked the same way; then
 * QSA_ERR_INVALID_ARG for a null workspace or one that overlaps an argument,
 * QSA_ERR_ALIGNMENT when it is not 256-byte aligned, QSA_ERR_WORKSPACE when
 * workspace_bytes is too small; nothing is launched on an error.  Rows whose
 * start is not 16-byte aligned, or W not a multiple of 4, run as in qsa_topk
 * (the workspace is then unused).
 */
qsa_status_t qsa_topk_ws(const float* scores, int64_t score_stride, const int32_t* lengths, int64_t rows,
                         int32_t W, int32_t k, int32_t* idx, int64_t idx_stride, void* workspace,
                         size_t workspace_bytes, void* stream);

/* Bytes of workspace qsa_topk_ws needs (about 25.7 KB per row); 0 for rows <= 0. */
size_t qsa_topk_workspace_size(int64_t rows, int32_t W, int32_t k);

/*
 * qsa_mqa_prefill_topk - prefill scores followed by per-row top-k, without
 * materialising more than one workspace of scores at a time.
 *
 * Rows are processed in chunks whose scores fit in the workspace (the vLLM
 * PR, "Main changes": prefill logits are bounded by a workspace limit and
 * processed chunk by chunk); each chunk runs qsa_mqa_prefill into the
 * workspace (row stride W) and then qsa_topk over it.  Arguments as for the
 * two calls; the result is idx only.  The workspace must be 16-byte aligned
 * and hold 4096 bytes of selection state plus at least min(T, 64) rows of W
 * floats; qsa_prefill_topk_workspace_size gives the size that needs a single
 * chunk.
 * A workspace of a few tens of MB keeps each chunk's scores in the B200's
 * 126 MB L2 between the two kernels, but leaves each chunk a few hundred
 * rows for 148 SMs.  Measured on B200 for 4 x 4,096 rows of 26,624 keys,
 * top-512: a 64 MiB workspace 1.96 ms per call, 512 MiB 1.26 ms, and the two
 * separate calls over every row 1.13 ms.  The workspace bounds memory; larger
 * chunks are faster.
 */
qsa_status_t qsa_mqa_prefill_topk(const void* q, int64_t q_stride_t, int64_t q_stride_h, const void* k,
                                  int64_t k_stride, int64_t Nk, const int32_t* ks, const int32_t* ke, int64_t T,
                                  float scale, int32_t W, int32_t topk_k, int32_t* idx, int64_t idx_stride,
                                  void* workspace, size_t workspace_bytes, void* stream);

size_t qsa_prefill_topk_workspace_size(int64_t T, int32_t W);

/*
 * qsa_mqa_prefill_topk_noalloc - qsa_mqa_prefill_topk without a caller
 * workspace.
 *
 * The pages have no counterpart to this call.  It is for callers that cannot
 * allocate device memory at call time: a host program whose device memory is
 * planned up front by a framework that hands out fixed pools, or code on a
 * thread where cudaMalloc is not allowed because it may synchronise the
 * device.  The scores pass through a 16 MiB static array compiled into this
 * library (every GPU that loads the library keeps it until the process
 * exits); no cudaMalloc, cudaFree or allocating library routine is called.
 * Arguments and results as for qsa_mqa_prefill_topk.
 *
 *  - One chunk of min(T, 64) rows of W floats plus 4096 bytes of selection
 *    state must fit in the 16 MiB: larger W returns QSA_ERR_WORKSPACE
 *    (W <= 65520 always fits).  Longer batches are processed in more chunks.
 *  - The first call on a device, with that device current, looks up the
 *    array's device address (cudaGetSymbolAddress); make that first call
 *    before any stream capture.
 *  - All calls share the array, which keeps the last call's contents; the
 *    call clears the part that must start at zero.  Calls that overlap on
 *    the GPU (different streams, or different host threads on one device)
 *    race on the array and must be serialised by the caller.
 */
qsa_status_t qsa_mqa_prefill_topk_noalloc(const void* q, int64_t q_stride_t, int64_t q_stride_h, const void* k,
                                          int64_t k_stride, int64_t Nk, const int32_t* ks, const int32_t* ke,
                                          int64_t T, float scale, int32_t W, int32_t topk_k, int32_t* idx,
                                          int64_t idx_stride, void* stream);

/*
 * qsa_expand_block_indices - selected compressed blocks to token indices.
 *
 * The step between top-k selection and core attention (QSA docs, MATE,
 * section "Core Attention": with a block hint the token list is
 * 4 * blocks + 3 wide, at most 4 * 512 + 3 = 2051 tokens).  Block b stands
 * for request-local tokens 4b .. 4b + 3; the 3 extra slots hold the row's
 * open group, the tokens after its last complete 4-token group (positions
 * 4 * visible .. pos, at most 3), which no compressed key covers yet.
 *
 *   blocks       int32 [T, k], row stride blk_stride (>= k when T > 1);
 *                negative entries are skipped (padding).  1 <= k <= 512.
 *   cu_seqlens_q int32 [R + 1], seq_lens int32 [R]: query rows of request r
 *                are cu_seqlens_q[r] .. cu_seqlens_q[r+1] - 1, row i of it at
 *                logical position seq_lens[r] - qlen_r + i (vLLM qsa_cache.py,
 *                "_logical_positions").  cu_seqlens_q[R] == T.
 *   token_idx    int32 [T, 4k + 3] output, row stride tok_stride: the four
 *                tokens of each non-negative block in the given order, then
 *                the open-group tokens ascending, then -1.
 */
qsa_status_t qsa_expand_block_indices(const int32_t* blocks, int64_t blk_stride, int32_t k,
                                      const int32_t* cu_seqlens_q, const int32_t* seq_lens, int32_t R, int64_t T,
                                      int32_t* token_idx, int64_t tok_stride, void* stream);

/*
 * qsa_sparse_attention - sparse core attention over selected tokens of a
 * paged K/V cache (QSA docs, MATE, section "Core Attention": request-local
 * token indices shared by all query heads, -1 pads, invalid and future
 * tokens masked, paged K/V [pages, page_size, Hkv, 256], optional sigmoid
 * gate, natural-log LSE; empty selections give zero output and -inf LSE).
 *
 * For query row t of request r (at logical position pos, as in
 * qsa_expand_block_indices) and query head h (KV head g = h / (Hq / Hkv)),
 * over the listed tokens j with 0 <= j <= pos, j < seq_lens[r] and a valid
 * page (page_table[r, j / page_size] in [0, num_pages)), each listed
 * occurrence counting once:
 *     s_j = scale * q[t, h] . K[j, g],   out[t, h] = sum_j softmax(s)_j V[j, g]
 * times sigmoid(gate[t, h]) when gate is given; lse[t, h] = log(sum_j e^s_j).
 *
 *   q          bf16 [T, Hq, 256]: row stride q_stride_t, head stride
 *              q_stride_h (>= 256), multiples of 8; 16-byte aligned.
 *   k_cache,   bf16 [num_pages, page_size, Hkv, 256] with the given page,
 *   v_cache    row and head strides (elements, multiples of 8); 16-byte
 *              aligned.  Hq a multiple of Hkv, Hq / Hkv <= 16 (24 / 2 is the
 *              QSA geometry).
 *   page_table int32 [R, max_pages], row stride pt_stride.
 *   token_idx  int32 [T, width], row stride tok_stride (>= width).
 *   gate       fp32 [T, Hq] or NULL.   scale: softmax scale (finite).
 *   out        bf16 [T, Hq, 256], row stride out_stride_t (>= Hq * 256),
 *              heads contiguous; 16-byte aligned; must not overlap inputs.
 *   lse        fp32 [T, Hq] or NULL.
 *   workspace  16-byte aligned, qsa_sparse_attention_workspace_size(T, Hq,
 *              Hkv, width) bytes (split-KV partial results); smaller returns
 *              QSA_ERR_WORKSPACE.
 * Two launches on `stream`: the split-KV attention and the merge of splits.
 */
qsa_status_t qsa_sparse_attention(const void* q, int64_t q_stride_t, int64_t q_stride_h, int32_t Hq,
                                  const void* k_cache, const void* v_cache, int64_t num_pages, int32_t page_size,
                                  int64_t kv_page_stride, int64_t kv_row_stride, int64_t kv_head_stride, int32_t Hkv,
                                  const int32_t* page_table, int64_t pt_stride, int32_t max_pages,
                                  const int32_t* cu_seqlens_q, const int32_t* seq_lens, int32_t R,
                                  const int32_t* token_idx, int64_t tok_stride, int32_t width, int64_t T,
                                  const float* gate, float scale, void* out, int64_t out_stride_t, float* lse,
                                  void* workspace, size_t workspace_bytes, void* stream);

size_t qsa_sparse_attention_workspace_size(int64_t T, int32_t Hq, int32_t Hkv, int32_t width);

/*
 * qsa_mqa_paged_batch - indexer scores of a mixed decode + prefill batch,
 * every request read from the paged compressed key cache, in one call.
 *
 * The vLLM PR "Separate prefill and decode paths for QSA indexer" ("Main
 * changes") splits a batch into uniform decode requests and prefill
 * requests, computes the visible block counts in the metadata step (vLLM
 * qsa_cache.py, the metadata kernel: logical positions and visible_blocks,
 * chained to its consumers with programmatic dependent launches) and scores
 * each part with its own kernel.  This call does the same on the device, on
 * `stream`, in four launches chained the same way: the decode kernel on
 * requests 0 .. D-1; a metadata kernel that gives every prefill row its key
 * interval and packs the prefill requests' keys out of their pages; the
 * tcgen05 prefill kernel on those rows; a fix-up that sets the scores of keys
 * whose page is missing to -inf.
 *
 *   q          bf16 [T, 4, 128] (row stride q_stride_t, head stride
 *              q_stride_h; multiples of 8; 16-byte aligned): the D *
 *              decode_query_len decode rows first, then the prefill rows.
 *   k_cache..  as qsa_mqa_decode (page_size 8 .. 1024), for all R requests.
 *   cu_seqlens_q int32 [R + 1], seq_lens int32 [R] (tokens, query rows
 *              included): the caller guarantees cu_seqlens_q[r] =
 *              r * decode_query_len for r <= D (the device contents are not
 *              read on the host).  Row i of request r sits at logical
 *              position seq_lens[r] - qlen_r + i.
 *   num_decodes D requests (0 .. R) are decodes with decode_query_len
 *              (1 .. 4) rows each; R - D <= 8192 prefill requests with
 *              (R - D) * W <= 2^31 - 1.
 *   out        fp32 [T, W], row stride out_stride: out[t, n] = score of
 *              request-local key n for n < visible(t) (and n < W), -inf
 *              otherwise; keys in missing pages are -inf.
 *   workspace  16-byte aligned, qsa_mqa_paged_batch_workspace_size(R, D,
 *              decode_query_len, T, W) bytes (packed keys and intervals);
 *              smaller returns QSA_ERR_WORKSPACE.  Not needed (may be NULL)
 *              when every request is a decode.
 */
qsa_status_t qsa_mqa_paged_batch(const void* q, int64_t q_stride_t, int64_t q_stride_h, const void* k_cache,
                                 int64_t num_pages, int32_t page_size, int64_t k_page_stride, int64_t k_row_stride,
                                 const int32_t* page_table, int64_t pt_stride, int32_t max_pages,
                                 const int32_t* cu_seqlens_q, const int32_t* seq_lens, int32_t R, int32_t num_decodes,
                                 int32_t decode_query_len, int64_t T, float scale, float* out, int64_t out_stride,
                                 int32_t W, void* workspace, size_t workspace_bytes, void* stream);

size_t qsa_mqa_paged_batch_workspace_size(int32_t R, int32_t num_decodes, int32_t decode_query_len, int64_t T,
                                          int32_t W);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H_ */

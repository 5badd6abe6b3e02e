/*
 * tg.h -- C ABI of the TokenGate gated-prefill path on B200 (sm_100a).
 *
 * The path (MarkTechPost page on TokenGate, French translation, section "Comment
 * TokenGate a-t-il appris le fonctionnement de la réduction des tokens ?"): a small
 * gate MLP scores every token from its post-attention residual at the gate layer
 * L; a top-K selector keeps the best-scoring tokens of the droppable document
 * while the question is always kept; layers above L see only the K kept tokens
 * and write KV only for them; their attention adds each kept key's score to the
 * logits through a per-head gain and scales the logits by a per-head temperature
 * (section "Qu'est-ce que l'attention gérée par des tokens ?").
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is a DEVICE pointer unless its comment says "host".
 *     The caller owns every buffer (scratch included, sized by the matching
 *     *_workspace_size query); the library allocates no device memory.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) and never synchronises the host, except tg_device_status().
 *   - Every call returns a tg_status; no exception crosses the ABI. Argument
 *     errors are detected on the host before any launch. Errors found on the
 *     device (a bounded wait that ran out, an inconsistent size) are recorded in a
 *     per-device status word read by tg_device_status(); the kernel then skips the
 *     remaining work instead of trapping.
 *   - Rows are token-major and dense: a [rows, cols] array has row stride cols.
 *   - Ragged batches use cumulative offsets: sequence b owns rows
 *     [cu[b], cu[b+1]) of a packed array; cu has batch+1 entries, cu[0] = 0.
 *   - bf16 is IEEE binary32 truncated to its top 16 bits (round to nearest even
 *     on output).
 */
#ifndef TOKENGATE_TG_H_
#define TOKENGATE_TG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TG_OK = 0,
  TG_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad span, K mismatch */
  TG_ERR_UNSUPPORTED = 2,   /* shape outside the kernels' supported set */
  TG_ERR_MISALIGNED = 3,    /* pointer or row size not 16-byte aligned */
  TG_ERR_WORKSPACE = 4,     /* caller-provided scratch too small */
  TG_ERR_CUDA = 5,          /* a CUDA runtime call failed (launch, attribute) */
  TG_ERR_TIMEOUT = 6,       /* device: a bounded wait ran out (see tg_device_status) */
  TG_ERR_DEVICE_CHECK = 7,  /* device: a size or index check failed, work skipped */
  TG_ERR_DEBUG_BOUNDS = 8   /* device, debug library only: an index outside its buffer, access skipped */
} tg_status;

typedef enum { TG_F32 = 0, TG_BF16 = 1 } tg_dtype;

typedef struct CUstream_st* tg_stream_t; /* same type as cudaStream_t */

/* Version of this ABI (bumped on any signature change). */
int tg_abi_version(void);

/*
 * 1 in the debug library (libtokengate_debug.so, compiled with TG_DEBUG), 0 in the
 * release library. The debug library checks the index of every data-dependent
 * global load and store (gathers through kept indices, scatters to kept rows,
 * cache rows, the per-sequence rows of every output) against the extent of its
 * buffer; an index outside it skips that access and records TG_ERR_DEBUG_BOUNDS
 * in the status word (tg_device_status), so a kernel's own index arithmetic can be
 * checked without a memory fault and without a sanitizer. The arithmetic and the
 * results are otherwise those of the release library, bit for bit.
 */
int tg_debug_build(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* tg_status_string(tg_status s);

/*
 * Gate MLP scorer (MarkTechPost page, "Comment TokenGate a-t-il appris ...": an
 * MLP scores each token from its residual at layer L). For every token i:
 *     s[i] = b2 + sum_k w2[k] * GELU(b1[k] + sum_c x[i,c] * w1[k,c]),
 * GELU(u) = u * Phi(u) (exact erf form).
 *   x       [n_tokens, d]   dtype         residual stream at the gate layer
 *   w1      [h, d]          dtype         first layer, nn.Linear layout (out x in)
 *   b1, w2  [h]             f32
 *   b2                      f32 scalar, by value
 *   scores  [n_tokens]      f32 output
 * TG_BF16 (tensor-core path): d % 64 == 0, h in {64, 128, 256}, x and w1 16-byte
 * aligned. TG_F32 (exact fp32 path, for small checks): 1 <= h <= 1024, d >= 1.
 * n_tokens == 0 is a no-op.
 */
tg_status tg_gate_score(const void* x, tg_dtype dtype, int64_t n_tokens, int d, const void* w1,
                        const float* b1, const float* w2, float b2, int h, float* scores,
                        tg_stream_t stream);

/*
 * Top-K selection with question protection (MarkTechPost page, "Comment TokenGate
 * a-t-il appris ...": a top-K selector keeps the best-scoring tokens; only the
 * document part of the prompt can be dropped, never the question; "Comment
 * déployer TokenGate ?": a {state} placeholder marks the droppable document and
 * max_kept_prefill_tokens is the budget).
 * For each sequence b (rows [cu_seqlens[b], cu_seqlens[b+1]) of `scores`), with
 * droppable span [doc_begin[b], doc_end[b]) in positions local to the sequence:
 * keep the min(k_doc[b], span length) span tokens of highest score and every
 * token outside the span. Ties go to the lower position; -0 equals +0; NaN ranks
 * below -inf; k_doc < 0 counts as 0.
 *   scores      [total_tokens]  f32
 *   cu_seqlens  [batch+1]       int32   (device)
 *   doc_begin, doc_end, k_doc [batch] int32 (device)
 *   kept_idx    [total_kept]    int32 output: kept rows' global row ids
 *                                       (indices into `scores`), ascending
 *   kept_scores [total_kept]    f32 output, may be NULL: scores[kept_idx[r]]
 *   kept_pos    [total_kept]    int32 output, may be NULL: the kept rows'
 *                                       positions within their own sequence
 *                                       (kept_idx[r] - cu_seqlens[b])
 *   cu_kept     [batch+1]       int32 output: cumulative kept counts
 * total_kept must equal sum_b (len_b - span_b + min(max(k_doc_b,0), span_b)); the
 * caller knows every term, so no device-to-host read is needed to size outputs.
 * max_seqlen bounds every len_b; max_seqlen <= TG_SELECT_MAX_SEQLEN; the
 * scores of sequence b must lie inside [0, total_tokens). A sequence whose rows or
 * span fall outside these bounds, or a total that differs from total_kept, is
 * found on the device: TG_ERR_DEVICE_CHECK is recorded, the sequence's output
 * rows get row id -1 (score 0, position -1), and cu_kept still advances by its
 * clamped count, clipped to total_kept, so every offset stays inside the outputs.
 */
#define TG_SELECT_MAX_SEQLEN 196608
tg_status tg_select_topk(const float* scores, const int32_t* cu_seqlens, const int32_t* doc_begin,
                         const int32_t* doc_end, const int32_t* k_doc, int batch,
                         int64_t total_tokens, int64_t total_kept, int max_seqlen,
                         int32_t* kept_idx, float* kept_scores, int32_t* kept_pos,
                         int32_t* cu_kept, tg_stream_t stream);

/*
 * Stable compaction (MarkTechPost page, "Comment TokenGate a-t-il appris ...":
 * layers above L process only the K kept tokens and never create KV entries for
 * the dropped ones). For t < n_tensors and r < n_kept:
 *     dst[t] row r  =  src[t] row kept_idx[r]      (row_bytes[t] bytes per row)
 *   src, dst    host arrays of n_tensors device pointers (1 <= n_tensors <= 8)
 *   row_bytes   host array of n_tensors sizes; each a positive multiple of 16
 *   kept_idx    [n_kept] int32 device, row ids into every src (from tg_select_topk)
 *   n_src_rows  rows of every src: an index outside [0, n_src_rows) is skipped
 *               (that dst row is left as it was) and TG_ERR_DEVICE_CHECK recorded
 * Every src/dst pointer must be 16-byte aligned.
 */
tg_status tg_compact_kv(const void* const* src, void* const* dst, const int64_t* row_bytes,
                        int n_tensors, const int32_t* kept_idx, int64_t n_kept,
                        int64_t n_src_rows, tg_stream_t stream);

/*
 * Token-gated causal GQA attention over the kept tokens (MarkTechPost page,
 * "Qu'est-ce que l'attention gérée par des tokens ?": each kept token's score is
 * a bias on the attention logits with a learnable per-head gain; a learnable
 * per-head temperature corrects for each query seeing fewer keys). For sequence
 * b (kept rows [cu_kept[b], cu_kept[b+1])), query head hq, kept row i:
 *     z_j = (q_i . k_j) / (sqrt(head_dim) * tau[hq]) + gain[hq] * s_kept[j],  j <= i
 *     out_i = sum_j softmax_j(z) * v_j
 * with KV head hq / (n_hq / n_hkv). Key j is visible to query i iff j <= i in the
 * position-ordered kept list (the original causal order).
 *   q    [total_kept, n_hq,  head_dim]  dtype
 *   k, v [total_kept, n_hkv, head_dim]  dtype
 *   s_kept [total_kept] f32 (from tg_select_topk), gain, tau [n_hq] f32
 *   cu_kept [batch+1] int32 device; max_kept >= every cu_kept[b+1]-cu_kept[b]
 *   out  [total_kept, n_hq, head_dim]  dtype output
 *   lse  [n_hq, total_kept] f32 output, may be NULL: each row's log-sum-exp
 *        log(sum_j exp(z_j)) (natural log), which the backward reads
 * A sequence whose kept range is not inside [0, total_kept] or is longer than
 * max_kept is skipped (its out rows are left as they were) and TG_ERR_DEVICE_CHECK
 * is recorded.
 * TG_BF16 (tensor-core path): head_dim == 128, n_hq % n_hkv == 0, q/k/v/out
 * 16-byte aligned. TG_F32 (exact fp32 path): head_dim <= 256.
 */
tg_status tg_gated_attention(const void* q, const void* k, const void* v, tg_dtype dtype,
                             const float* s_kept, const float* gain, const float* tau,
                             const int32_t* cu_kept, int batch, int64_t total_kept, int max_kept,
                             int n_hq, int n_hkv, int head_dim, void* out, float* lse,
                             tg_stream_t stream);

/*
 * Backward of tg_gated_attention (MarkTechPost page on TokenGate, section "Qu'est-ce
 * que l'attention gérée par des tokens ?": the key score enters the logits as a bias
 * so that gradients reach the scorer; gain and temperature are learned per head).
 * Given dout = dL/dout for a forward call (same q, k, v, s_kept, gain, tau, cu_kept)
 * and that call's out and lse, with c_h = 1 / (sqrt(head_dim) tau[h]),
 * P = softmax_j(z), dZ_ij = P_ij (dout_i . v_j - dout_i . out_i):
 *   dq [total_kept, n_hq, head_dim]  dtype   c_h sum_j dZ_ij k_j
 *   dk, dv [total_kept, n_hkv, head_dim] dtype   sum over the group's heads of
 *                                     c_h sum_i dZ_ij q_i and sum_i P_ij dout_i
 *   ds [total_kept] f32               dL/ds_j = sum_h gain[h] sum_i dZ_ij
 *   dgain, dtau [n_hq] f32            sum_ij dZ_ij s_j and -(c_h/tau_h) sum_ij dZ_ij q_i.k_j
 * Every output is overwritten. workspace: caller-owned device scratch of at least
 * tg_gated_attention_bwd_workspace_size(...) bytes, 16-byte aligned, no initial
 * value needed (too small: TG_ERR_WORKSPACE). TG_BF16: head_dim == 128 (tensor
 * cores), pointers 16-byte aligned; TG_F32: head_dim <= 256 (exact SIMT path).
 * Sequences whose kept range is invalid are skipped and TG_ERR_DEVICE_CHECK recorded.
 */
size_t tg_gated_attention_bwd_workspace_size(tg_dtype dtype, int batch, int64_t total_kept,
                                             int max_kept, int n_hq, int n_hkv, int head_dim);
tg_status tg_gated_attention_bwd(const void* q, const void* k, const void* v, const void* out,
                                 const void* dout, tg_dtype dtype, const float* lse,
                                 const float* s_kept, const float* gain, const float* tau,
                                 const int32_t* cu_kept, int batch, int64_t total_kept,
                                 int max_kept, int n_hq, int n_hkv, int head_dim, void* dq,
                                 void* dk, void* dv, float* ds, float* dgain, float* dtau,
                                 void* workspace, size_t workspace_bytes, tg_stream_t stream);

/*
 * The kept tokens' q/k/v projections for the layers above the gate layer, so the
 * KV cache is written for the kept tokens only (MarkTechPost page, section
 * "Comment TokenGate a-t-il appris le fonctionnement de la réduction des tokens
 * ?": layers above the gate layer process only the K kept tokens). For every row r:
 *     y = W xc[r],  W = [Wq; Wk; Wv]  [(n_hq + 2 n_hkv) head_dim, d]  (nn.Linear layout)
 * split per head; q and k heads are rotated at pos[r] (rotary embedding with the
 * rotate-half pairing (i, i + head_dim/2) and theta_i = rope_base^(-2i/head_dim), the
 * convention of the Qwen models the pages evaluate; the pages do not describe it),
 * v heads are copied. The angle pos * theta_i is taken in turns as an integer
 * product with theta_i / (2 pi) in 64-bit fixed point (exact modulo one turn),
 * rounded to 2^-24 of a turn, before an fp32 sine and cosine.
 *   xc  [n_rows, d] bf16: the compacted residual rows (tg_compact_kv)
 *   pos [n_rows] int32 device, >= 0: original positions within each sequence
 *   q [n_rows, n_hq, head_dim], k and v [n_rows, n_hkv, head_dim] bf16 outputs
 * head_dim == 128, n_hq + 2 n_hkv even, d % 64 == 0, rope_base > 1, every pointer
 * 16-byte aligned; the caller owns every buffer.
 */
tg_status tg_qkv_rope(const void* xc, int64_t n_rows, int d, const void* w_qkv, int n_hq,
                      int n_hkv, int head_dim, float rope_base, const int32_t* pos, void* q,
                      void* k, void* v, tg_stream_t stream);

/*
 * The compaction fused into the projection (same section): tg_qkv_rope on the rows
 * xc[r] = x[kept_idx[r]], read straight from the full residual, so the projection
 * does not wait for a separate compaction. The compacted rows themselves are also
 * written to xc when xc != NULL (the layers above the gate layer carry them on).
 * q, k, v are bit-identical to tg_compact_kv followed by tg_qkv_rope. On a B200
 * the two calls are the faster path at every size measured (1.9k to 22k rows): the
 * 16-byte row gathers feed the tensor cores less steadily than TMA loads of rows
 * already compacted. This one needs no compacted-row buffer when xc is NULL.
 *   x        [n_src, d] bf16 device: the residual rows at the gate layer
 *   kept_idx [n_rows] int32 device: row ids into x (tg_select_topk's kept_idx); an
 *            id outside [0, n_src) projects a zero row, leaves that xc row as it
 *            was and records TG_ERR_DEVICE_CHECK
 *   xc       [n_rows, d] bf16 device output, or NULL
 *   pos, w_qkv, q, k, v, and the shape rules: as tg_qkv_rope (n_src <= INT32_MAX).
 */
tg_status tg_compact_qkv_rope(const void* x, int64_t n_src, int d, const int32_t* kept_idx,
                              int64_t n_rows, void* xc, const void* w_qkv, int n_hq, int n_hkv,
                              int head_dim, float rope_base, const int32_t* pos, void* q, void* k,
                              void* v, tg_stream_t stream);

/*
 * Decode over the compacted cache (MarkTechPost page on TokenGate, section
 * "Comment déployer TokenGate ?": generation runs on the cache the pruned prefill
 * leaves, bounded by max_kept_prefill_tokens; section "Qu'est-ce que l'attention
 * gérée par des tokens ?": the key-score bias with per-head gain, and the per-head
 * temperature). The cache of sequence b is rows [b*cap, b*cap + cache_len[b]) of
 *   k_cache, v_cache  [batch, cap, n_hkv, head_dim] bf16 (dense, token-major)
 *   s_cache           [batch, cap] f32            (each cached key's gate score)
 * as left by the prefill's compaction (tg_compact_kv of the kept rows) and grown by
 * tg_cache_append. In the layers up to the gate layer (no score bias) pass
 * gain = 0 and tau = 1: the same call is then plain causal attention.
 *
 * tg_cache_append: for every sequence b, writes k_new[b], v_new[b] ([batch, n_hkv,
 * head_dim] bf16) and s_new[b] (f32) into row cache_len[b] of its cache and adds
 * one to cache_len[b] (int32 [batch], device). A full cache (cache_len[b] >= cap)
 * is left unchanged and TG_ERR_DEVICE_CHECK recorded. head_dim == 128.
 */
tg_status tg_cache_append(const void* k_new, const void* v_new, const float* s_new, int batch,
                          int cap, int n_hkv, int head_dim, void* k_cache, void* v_cache,
                          float* s_cache, int32_t* cache_len, tg_stream_t stream);

/*
 * tg_gated_decode: one new query row per sequence (q [batch, n_hq, head_dim] bf16,
 * its own k/v already appended) attends over cache rows j < cache_len[b]:
 *     z_j = q . k_j / (sqrt(head_dim) * tau[hq]) + gain[hq] * s_j
 *     out[b, hq] = sum_j softmax_j(z) v_j          (bf16 [batch, n_hq, head_dim])
 * with KV head hq / (n_hq / n_hkv). max_len (host) bounds every cache_len[b] and
 * sizes the launch; max_len <= cap. head_dim == 128, n_hq / n_hkv <= 8; q, the
 * caches, out and workspace 16-byte aligned. An empty cache gives zeros. A length
 * outside [0, min(cap, max_len)] leaves that row of out unchanged and records
 * TG_ERR_DEVICE_CHECK.
 * workspace: caller-owned device scratch of at least
 * tg_gated_decode_workspace_size(batch, n_hq, head_dim, max_len) bytes (per-chunk
 * partial results; no initial value needed; calls that overlap on the GPU must not
 * share it). Too small a workspace returns TG_ERR_WORKSPACE.
 */
size_t tg_gated_decode_workspace_size(int batch, int n_hq, int head_dim, int max_len);
tg_status tg_gated_decode(const void* q, const void* k_cache, const void* v_cache,
                          const float* s_cache, const int32_t* cache_len, int batch, int cap,
                          int max_len, int n_hq, int n_hkv, int head_dim, const float* gain,
                          const float* tau, void* out, void* workspace, size_t workspace_bytes,
                          tg_stream_t stream);

/*
 * tg_gated_decode_noalloc: tg_gated_decode without a caller-provided workspace.
 * There is no counterpart on the pages; this is a convenience of this library.
 * It is for callers that cannot allocate device memory where they decode: a host
 * program whose device memory all belongs to another runtime's pool (a library may
 * not, or cannot, call cudaMalloc behind it), or a token-by-token generation loop
 * that must not allocate because cudaMalloc and cudaFree can synchronise the whole
 * device. The per-chunk partials go to a fixed array in the library's own device
 * memory, TG_DECODE_NOALLOC_SCRATCH_BYTES large, which every device that loads the
 * library holds until the process exits. Arguments, outputs and checks are those
 * of tg_gated_decode; a call whose partials would need more than the array
 * (tg_gated_decode_workspace_size(batch, n_hq, head_dim, max_len) >
 * TG_DECODE_NOALLOC_SCRATCH_BYTES) returns TG_ERR_WORKSPACE and launches nothing.
 * It allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture. All calls share the one array and it keeps what the last
 * call left there (nothing in it needs to start at zero): calls whose kernels
 * overlap on the GPU (different streams, or different host threads) race on it.
 */
#define TG_DECODE_NOALLOC_SCRATCH_BYTES (8u << 20)
tg_status tg_gated_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                  const float* s_cache, const int32_t* cache_len, int batch,
                                  int cap, int max_len, int n_hq, int n_hkv, int head_dim,
                                  const float* gain, const float* tau, void* out,
                                  tg_stream_t stream);

/*
 * Gated delta rule over the kept tokens: the recurrence of the hybrid model's Gated
 * DeltaNet layers, which TokenGate also prunes (MarkTechPost page on TokenGate,
 * section "Est-ce que cela fonctionne avec les modèles d'attention hybrides ?" and
 * the comparison table). For each sequence b (rows [cu_seqlens[b], cu_seqlens[b+1])
 * of the packed kept rows) and head h, a state S (head_dim_k x head_dim_v) starts at
 * zero and, for the sequence's rows t in order,
 *     S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *     out_t = S_t^T q_t
 * computed in chunks of 64 rows (a parallel per-chunk pass, then one sequential
 * pass over each sequence's chunks).
 *   q, k  [total, n_heads, head_dim_k] bf16 (the caller normalises k; with |k| = 1
 *         and alpha, beta in [0, 1] the state stays bounded)
 *   v     [total, n_heads, head_dim_v] bf16
 *   alpha, beta [total, n_heads] f32 (decay and write strength per token and head)
 *   max_seqlen  bounds every sequence's length (host value; sizes the grid)
 *   out   [total, n_heads, head_dim_v] bf16 output
 *   workspace   caller-owned device scratch of at least
 *               tg_gated_delta_rule_workspace_size(...) bytes, 16-byte aligned
 *               (per 64-row chunk and head: the chunk's products that do not depend
 *               on the state)
 * TG_BF16 only; head_dim_k == 128, head_dim_v a multiple of 16 up to 1024; q, k, v,
 * out 16-byte aligned. A sequence outside [0, total] or longer than max_seqlen is
 * skipped (its rows of out are not written) and TG_ERR_DEVICE_CHECK recorded.
 */
size_t tg_gated_delta_rule_workspace_size(int batch, int64_t total, int n_heads,
                                          int head_dim_v);
tg_status tg_gated_delta_rule(const void* q, const void* k, const void* v, tg_dtype dtype,
                              const float* alpha, const float* beta, const int32_t* cu_seqlens,
                              int batch, int64_t total, int max_seqlen, int n_heads,
                              int head_dim_k, int head_dim_v, void* out, void* workspace,
                              size_t workspace_bytes, tg_stream_t stream);

/*
 * Synchronises `stream`, then returns the first error any kernel recorded on the
 * current device since the last reset (TG_OK if none). reset != 0 clears it.
 */
tg_status tg_device_status(tg_stream_t stream, int reset);

/*
 * Failure-detection self test: launches one kernel that waits, with the same
 * bounded wait the other kernels use, on a device flag that nothing sets. After
 * timeout_ns nanoseconds the wait gives up and records TG_ERR_TIMEOUT in the
 * status word (read it with tg_device_status). 1000 <= timeout_ns <= 1e10.
 */
tg_status tg_selftest_bounded_wait(int64_t timeout_ns, tg_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TOKENGATE_TG_H_ */

/*
 * ulysses.h -- C ABI of the Ulysses per-rank attention path on one B200.
 *
 * Ulysses sequence parallelism (page "Hugging Face并行加速：10倍提升超长序列训练效率",
 * section "Ulysses的工作原理"; page "DeepSpeed Ulysses 详解", section
 * "DeepSpeed-Ulysses 的核心机制") splits a sequence of N tokens over P GPUs,
 * exchanges the projected Q/K/V with an all-to-all so that every GPU holds the
 * whole sequence for H/P heads, runs ordinary attention on those heads, and
 * exchanges the output back to sequence shards. On one GPU the P ranks are
 * emulated as P buffers and the all-to-all as an in-HBM permutation.
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library
 *    never allocates device memory and keeps no pointer after a call returns.
 *  - bf16 tensors are contiguous, row-major, 16-byte aligned.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream). Argument errors are detected on the host before any
 *    launch and return ULYSSES_ERR_INVALID / ULYSSES_ERR_UNSUPPORTED /
 *    ULYSSES_ERR_WORKSPACE without touching device memory.
 *  - A launch failure returns ULYSSES_ERR_CUDA.
 *  - Device-side waits are bounded. A wait that runs out records a flag in
 *    the workspace and the kernel drains and returns; ulysses_sync_status()
 *    reports it as ULYSSES_ERR_TIMEOUT. Each attention call clears the flag
 *    when it starts, so the status describes the latest call on that
 *    workspace.
 *  - ulysses_last_error() returns a thread-local message for the last failure.
 *  - Head dimension d must be 32, 64 or 128.
 */
#ifndef ULYSSES_H
#define ULYSSES_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ULYSSES_OK = 0,
    ULYSSES_ERR_INVALID = -1,     /* null or misaligned pointer, H % P, Hkv % P, N % P, H % Hkv, d, ... */
    ULYSSES_ERR_UNSUPPORTED = -2, /* a valid request the library does not implement */
    ULYSSES_ERR_CUDA = -3,        /* a CUDA runtime/driver call failed */
    ULYSSES_ERR_TIMEOUT = -4,     /* a bounded device-side wait ran out */
    ULYSSES_ERR_WORKSPACE = -5    /* workspace missing or smaller than ulysses_attn_workspace_bytes() */
} ulysses_status;

/* Thread-local text of the last failure (empty string if none). Never NULL. */
const char *ulysses_last_error(void);

/* Library version string. */
const char *ulysses_version(void);

/*
 * Sequence-to-head exchange (the first all-to-all).
 * Page "Hugging Face并行加速：10倍提升超长序列训练效率", section "Ulysses的工作原理",
 * steps 序列分片 and 全体间通信; page "DeepSpeed Ulysses 详解", section
 * "DeepSpeed-Ulysses 的核心机制", item 3.
 *
 *   src  [P][N/P][Hx][d] bf16: rank i's buffer holds tokens [i*N/P, (i+1)*N/P)
 *        for all Hx heads (this is also the plain [N][Hx][d] layout).
 *   rank < 0:  dst [P][N][Hx/P][d]: every rank's head slice,
 *              dst[r][n][h][:] = src[n/(N/P)][n%(N/P)][r*Hx/P + h][:].
 *   rank = r:  dst [N][Hx/P][d]: rank r's head slice only.
 * Hx is H for Q and Hkv for K and V. Requires N % P == 0, Hx % P == 0,
 * d in {32,64,128}; src and dst must not overlap. A bit copy (bit-exact).
 * N == 0 is a no-op.
 */
int ulysses_seq_to_head(const void *src, void *dst, int64_t N, int P, int Hx, int d,
                        int rank, void *stream);

/*
 * Head-to-sequence exchange (the second all-to-all), the inverse of
 * ulysses_seq_to_head. Same page, step 全体间通信复原; page "DeepSpeed Ulysses
 * 详解", item 5.
 *
 *   rank < 0:  src [P][N][Hx/P][d] (every rank's slice) -> dst [P][N/P][Hx][d],
 *              dst[p][m][r*Hx/P + h][:] = src[r][p*N/P + m][h][:].
 *   rank = r:  src [N][Hx/P][d] (rank r's slice); writes only heads
 *              [r*Hx/P, (r+1)*Hx/P) of dst [P][N/P][Hx][d], leaving the rest.
 */
int ulysses_head_to_seq(const void *src, void *dst, int64_t N, int P, int Hx, int d,
                        int rank, void *stream);

/*
 * The same two exchanges for a slice of heads: the sequence-side rows hold
 * row_heads heads ([P][N/P][row_heads][d]), of which heads [head0, head0+Hx)
 * are exchanged, read from (seq_to_head) or written into (head_to_seq) those
 * rows in place; the head side is as above for Hx heads. This is the exchange
 * of one chunk of heads of the head-chunked variant (page "Ulysses 序列並行：百萬
 * Token 上下文訓練", section "競品分析", UPipe), with no copy of the chunk.
 * Requires head0 >= 0 and head0 + Hx <= row_heads, plus the conditions above.
 */
int ulysses_seq_to_head_heads(const void *src, void *dst, int64_t N, int P, int Hx, int d, int rank,
                              int row_heads, int head0, void *stream);
int ulysses_head_to_seq_heads(const void *src, void *dst, int64_t N, int P, int Hx, int d, int rank,
                              int row_heads, int head0, void *stream);

/*
 * Bytes of device workspace that ulysses_attn_fwd (backward = 0) or
 * ulysses_attn_bwd (backward = 1) need for these sizes. The workspace holds
 * the per-token document starts, per-tile key ranges, the tile schedule, the
 * backward's row statistics and a status word. Its contents need not be
 * initialised by the caller.
 */
size_t ulysses_attn_workspace_bytes(int64_t N, int Hl, int Hkvl, int d, int backward);

/*
 * Attention forward for one rank's head slice ("本地注意力计算": ordinary
 * attention per head on the full sequence; heads are independent).
 *
 *   q     [N][Hl][d]   bf16, query head h uses KV head h / (Hl/Hkvl)
 *   k, v  [N][Hkvl][d] bf16
 *   position_ids [N] int32 (device): a document starts wherever the id is 0,
 *         and at token 0 (page "Ulysses verteilt Millionen-Token-Kontexte auf
 *         mehrere GPUs", section "Integration in den Hugging-Face-Stack").
 *   scale softmax scale; <= 0 means 1/sqrt(d).
 *   o     [N][Hl][d]   bf16 output (round to nearest even).
 *   lse   [Hl][N]      fp32 natural-log logsumexp of the scaled logits.
 * Row i attends to keys j with doc_start(i) <= j <= i. Requires Hl % Hkvl == 0.
 */
int ulysses_attn_fwd(const void *q, const void *k, const void *v, const int32_t *position_ids,
                     int64_t N, int Hl, int Hkvl, int d, float scale,
                     void *o, float *lse, void *ws, size_t ws_bytes, void *stream);

/*
 * Fused form: the same attention, reading rank `rank`'s head slice directly
 * from the sequence-sharded buffers and writing O straight back to the
 * sequence-sharded layout, so neither exchange is materialised.
 *
 *   q_seq [N][H][d], k_seq / v_seq [N][Hkv][d]  (= [P][N/P][heads][d])
 *   o_seq [N][H][d]: only heads [rank*H/P, (rank+1)*H/P) are written.
 *   lse   [H/P][N] for this rank's heads.
 */
int ulysses_attn_fwd_fused(const void *q_seq, const void *k_seq, const void *v_seq,
                           const int32_t *position_ids, int64_t N, int P, int H, int Hkv,
                           int d, int rank, float scale, void *o_seq, float *lse,
                           void *ws, size_t ws_bytes, void *stream);

/*
 * One ring step of the Ulysses x ring hybrid (for Hkv < P, where Ulysses
 * alone runs out of heads: page "Ulysses 序列並行：百萬 Token 上下文訓練",
 * section "競品分析"; page "Ulysses verteilt Millionen-Token-Kontexte auf
 * mehrere GPUs", section "Wann Ulysses sinnvoll ist"): the attention of the
 * query rows [q_lo, q_hi) over the keys [kv_lo, kv_hi) only -- the chunk of
 * keys and values a rank holds at that step of the ring.
 *
 *   q [N][Hl][d], k, v [N][Hkvl][d], position_ids [N]: as ulysses_attn_fwd
 *         (whole-sequence indices; only the rows and keys of the windows are read).
 *   o     [q_hi - q_lo][Hl][d] bf16: row i - q_lo is the partial output of row i,
 *         normalised over the keys it sees in the window.
 *   lse   [Hl][q_hi - q_lo] fp32: natural-log sum of exp over those keys.
 * Row i sees keys j with max(doc_start(i), kv_lo) <= j <= min(i, kv_hi - 1); a
 * row that sees none gets o = 0 and lse = -inf. Requires 0 <= q_lo <= q_hi <= N
 * and 0 <= kv_lo <= kv_hi <= N (ULYSSES_ERR_INVALID otherwise). The workspace
 * is the forward one for (N, Hl). Partials of disjoint windows combine with
 * ulysses_attn_merge into the attention over their union.
 */
int ulysses_attn_fwd_window(const void *q, const void *k, const void *v, const int32_t *position_ids,
                            int64_t N, int Hl, int Hkvl, int d, int64_t q_lo, int64_t q_hi, int64_t kv_lo,
                            int64_t kv_hi, float scale, void *o, float *lse, void *ws, size_t ws_bytes,
                            void *stream);

/*
 * Merge of R partial attention results over disjoint key sets (the ring
 * steps of one rank) into the result over their union:
 *   L = log sum_s exp(lse_s),  o = sum_s exp(lse_s - L) o_s,  lse = L.
 *   o_parts   [R][M][Hl][d] bf16, lse_parts [R][Hl][M] fp32 (lse_s = -inf: no key).
 *   o         [M][Hl][d] bf16 (rounded once), lse [Hl][lse_ld] fp32 (first M
 *             columns of each row written); a row with no key in any part
 *             gets o = 0, lse = -inf.
 * Requires 1 <= R <= 64 and lse_ld >= M. Accumulates in fp32.
 */
int ulysses_attn_merge(const void *o_parts, const float *lse_parts, int R, int64_t M, int Hl, int d, void *o,
                       float *lse, int64_t lse_ld, void *stream);

/*
 * Attention backward for one rank's head slice: gradients of sum(dout * o).
 *   D_i = sum_c dout_ic o_ic;  P_ij = exp(scale q_i.k_j - lse_i);
 *   dS_ij = P_ij (dout_i.v_j - D_i);
 *   dq_i = scale sum_j dS_ij k_j;  dk_j = scale sum_{h in group} sum_i dS_ij q_i;
 *   dv_j = sum_{h in group} sum_i P_ij dout_i.
 * Inputs are those of ulysses_attn_fwd plus its outputs o and lse, and the
 * upstream gradient dout [N][Hl][d]. Outputs dq [N][Hl][d], dk and dv
 * [N][Hkvl][d], bf16. dq, dk, dv are fully overwritten.
 */
int ulysses_attn_bwd(const void *q, const void *k, const void *v, const void *o,
                     const void *dout, const float *lse, const int32_t *position_ids,
                     int64_t N, int Hl, int Hkvl, int d, float scale,
                     void *dq, void *dk, void *dv, void *ws, size_t ws_bytes, void *stream);

/*
 * Fused form of the backward, as ulysses_attn_fwd_fused is of the forward:
 * rank `rank`'s head slice is read from the sequence-sharded buffers and its
 * gradients are written straight into the sequence-sharded layout, so none
 * of the backward's exchanges (dout in; dq, dk, dv out) is materialised.
 *
 *   q_seq, o_seq, dout_seq [N][H][d]; k_seq, v_seq [N][Hkv][d]
 *         (= [P][N/P][heads][d]); lse [H/P][N] for this rank's heads.
 *   dq_seq [N][H][d], dk_seq / dv_seq [N][Hkv][d]: only this rank's heads
 *         ([rank*H/P, (rank+1)*H/P) and [rank*Hkv/P, (rank+1)*Hkv/P)) are
 *         written, so the calls of all ranks together fill them.
 * Same checks as ulysses_attn_fwd_fused; the workspace is the backward one for
 * (N, H/P, Hkv/P, d).
 */
int ulysses_attn_bwd_fused(const void *q_seq, const void *k_seq, const void *v_seq,
                           const void *o_seq, const void *dout_seq, const float *lse,
                           const int32_t *position_ids, int64_t N, int P, int H, int Hkv,
                           int d, int rank, float scale, void *dq_seq, void *dk_seq, void *dv_seq,
                           void *ws, size_t ws_bytes, void *stream);

/*
 * No counterpart in the pages: ulysses_attn_fwd for callers that cannot
 * allocate device memory, such as a plugin inside a host framework that owns
 * all device memory through its own pool and hands over only input and output
 * buffers, or a latency-critical path that must not call cudaMalloc (which can
 * synchronise the device). Same arguments and results as ulysses_attn_fwd
 * without the workspace: the scratch lives in a static device array inside the
 * library (544 KiB, held by every GPU that loads the library until exit).
 *  - N > 131072 returns ULYSSES_ERR_UNSUPPORTED.
 *  - Nothing is allocated. The first call on each device looks up the array's
 *    address (cudaGetSymbolAddress) with that device current; make that first
 *    call before any stream capture.
 *  - All calls on a device share the array; calls that overlap on the GPU
 *    (different streams, unordered threads) race and give wrong results.
 *  - A bounded device wait that runs out is not reported by this entry point.
 */
int ulysses_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                             const int32_t *position_ids, int64_t N, int Hl, int Hkvl, int d,
                             float scale, void *o, float *lse, void *stream);

/*
 * The projections on either side of the exchange, with the exchange fused in
 * (page "Hugging Face并行加速：10倍提升超长序列训练效率", section
 * "Ulysses的工作原理", steps QKV投影 and 输出投影; page "DeepSpeed Ulysses 详解",
 * section "DeepSpeed-Ulysses 的核心机制", items 2 and 6). Every rank projects its
 * own tokens with the full weights; here the tokens of all P ranks are
 * projected by one tensor-core GEMM (bf16 operands, fp32 accumulation, bf16
 * results rounded once). The workspace is ulysses_proj_workspace_bytes()
 * bytes of device memory (a status word; bounded device waits report there,
 * read by ulysses_sync_status).
 */
size_t ulysses_proj_workspace_bytes(void);

/*
 * QKV projection fused with the first exchange:
 *   x      [N][hidden] bf16: the P sequence shards ([P][N/P][hidden]).
 *   w_qkv  [(H+2Hkv)*d][hidden] bf16: output column c = x . w_qkv[c]; columns
 *          [0, H*d) are Q's heads, then K's, then V's, d per head.
 *   q_heads [P][N][H/P][d], k_heads, v_heads [P][N][Hkv/P][d]: every rank's
 *          head slice (the layout ulysses_seq_to_head produces): head g of token
 *          n lands in rank g/(heads/P), slot g%(heads/P).
 * Requires H % P == Hkv % P == 0, N % P == 0, d in {32,64,128}, hidden a
 * positive multiple of 64 and (H+2Hkv)*d a multiple of 128
 * (ULYSSES_ERR_UNSUPPORTED otherwise).
 */
int ulysses_qkv_proj(const void *x, const void *w_qkv, int64_t N, int hidden, int P, int H, int Hkv, int d,
                     void *q_heads, void *k_heads, void *v_heads, void *ws, size_t ws_bytes, void *stream);

/*
 * Output projection fused with the second exchange:
 *   o_heads [P][N][H/P][d] bf16: every rank's head slice of the attention
 *           output; read in the sequence order of heads (global head
 *           r*H/P + h at columns ((r*H/P + h)*d ...) of a token's row).
 *   w_o     [hidden][H*d] bf16.
 *   y       [N][hidden] bf16: y[n] = o_seq[n] . w_o^T.
 * Requires H % P == 0, N % P == 0, d in {64,128} (ULYSSES_ERR_UNSUPPORTED for
 * d = 32) and hidden a multiple of 128.
 */
int ulysses_out_proj(const void *o_heads, const void *w_o, int64_t N, int hidden, int P, int H, int d, void *y,
                     void *ws, size_t ws_bytes, void *stream);

/*
 * Synchronise `stream` and report the status the latest attention call left
 * in `ws`: ULYSSES_ERR_TIMEOUT if a bounded device wait ran out, else
 * ULYSSES_OK (or ULYSSES_ERR_CUDA if synchronisation failed). Clears the flag.
 */
int ulysses_sync_status(void *ws, void *stream);

/*
 * Device-side wait limit in nanoseconds for later launches from this process
 * (default 1e9). Values <= 0 restore the default.
 */
void ulysses_set_wait_limit_ns(int64_t ns);

/*
 * Test hook for the failure path (no counterpart in the pages). Bit 0: later
 * forward launches make their first CTA wait on a barrier that nothing ever
 * arrives on; bit 1: the same for the first CTA of the backward's dK/dV
 * kernel. The bounded wait runs out, the launch drains and returns (the
 * backward's dQ kernel, launched after it, finds the status set and skips its
 * work), and ulysses_sync_status() reports ULYSSES_ERR_TIMEOUT. Nothing faults
 * or hangs. 0 (the default) disables it.
 */
void ulysses_set_debug_flags(uint32_t flags);

#ifdef __cplusplus
}
#endif

#endif /* ULYSSES_H */

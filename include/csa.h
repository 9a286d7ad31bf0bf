/*
 * csa.h -- C ABI of libcsa.so: the hybrid long-context attention step of
 * DeepSeek-V4 (Compressed Sparse Attention, CSA, and Heavily Compressed
 * Attention, HCA) on one NVIDIA B200 (sm_100a).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  * Buffers are caller-owned DEVICE memory unless stated otherwise,
 *    row-major and contiguous, base pointers 16-byte aligned.  Calls that
 *    need scratch take a caller workspace sized by the matching
 *    *_workspace_bytes() query.  The one allocation the library makes is the
 *    weight table of csa_compress at large m (stream ordered, from a memory
 *    pool of the library that keeps its memory: 2m*d*4 bytes, at most 2 MiB,
 *    per call in flight).
 *  * bf16 tensors are passed as `const uint16_t *` holding bf16 bit patterns.
 *  * `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 *    asynchronous on that stream and returns after enqueueing its kernels.
 *  * Return value: CSA_OK (0) or a negative csa_status.  Validation errors
 *    (CSA_ERR_INVALID / CSA_ERR_UNSUPPORTED / CSA_ERR_WORKSPACE) are detected
 *    on the host before any launch, so nothing was enqueued.  CSA_ERR_CUDA
 *    reports a launch error.  Device-side failures (a bounded wait that ran
 *    out) are recorded in a device status word and reported by
 *    csa_sync_status().  No exception crosses the ABI.
 *  * Notation: batch = independent sequences; T = tokens per sequence; m =
 *    compression ratio; N = compressed entries per sequence (floor(T/m) when
 *    built by csa_compress); a query at position t sees the first
 *    n_vis(t) = min(N, floor((t+1)/m)) entries (an entry is visible once all
 *    of its newest-m tokens are at or before t).
 *
 * Sources: "DeepSeek v4" (it.peoplentools.com) section "Compressed Sparse
 * Attention" (compressed entries, lightning indexer, top-k selector, sliding
 * window) and the hybrid-attention section (HCA, m' >> m); "DeepSeek-AI (2026)
 * - ARXIV-2606.19348" (dmarx anthology record) "Key takeaways" (two latent KV
 * streams, overlapping 2m-token windows, RMSNorm on query heads and on the
 * compressed KV head); "DeepSeek-V4-Pro - Model techniques map" table
 * "Checked in its code" (one KV head for 128 query heads, window 128, top-k
 * 1024 with -1 for invalid slots, 64x128 indexer) and list "inference
 * quantization" (FP4 indexer); "DeepSeek V4 paper full version is out, FP4
 * QAT details and stability tricks [D]" (FP4 activations on the indexer QK path).
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CSA_OK = 0,
    CSA_ERR_INVALID = -1,     /* null / misaligned pointer, bad size or argument   */
    CSA_ERR_UNSUPPORTED = -2, /* a shape outside what the compiled kernels handle   */
    CSA_ERR_CUDA = -3,        /* a CUDA launch or runtime error                     */
    CSA_ERR_WORKSPACE = -4,   /* workspace pointer NULL or smaller than required    */
    CSA_ERR_TIMEOUT = -5      /* a device-side bounded wait expired (see csa_sync_status) */
} csa_status;

/* Human-readable text for a csa_status (static storage, never NULL). */
const char *csa_strerror(int status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int csa_version(void);

/*
 * csa_compress -- build compressed KV entries from the two latent streams.
 *   ("DeepSeek v4" -> "Compressed Sparse Attention" -> compressed Key-Value
 *    entry; anthology record "Key takeaways": overlapping 2m-token windows.)
 *
 * For every sequence b, entry i in [0, N), N = floor(T/m), and channel c:
 *   w_j[c]  = softmax over j = 0..2m-1 of logits[j][c]
 *   C_i[c]  = sum_{j<m} w_j[c] * B[(i-1)m + j][c] + sum_{j<m} w_{m+j}[c] * A[im + j][c]
 * Rows 0..m-1 of the logits weight the previous m tokens (stream B), rows
 * m..2m-1 the newest m tokens (stream A).  Entry 0 has no previous block: its
 * softmax runs over the A half only.  If apply_rmsnorm != 0 each entry is then
 *   y[c] = C_i[c] / sqrt(mean_c(C_i^2) + eps) * gain[c]   (gain NULL -> 1).
 * Arithmetic in fp32; the result is rounded to bf16 once.
 *
 *   A, B    [batch][T][d] bf16          stream A (newest half), stream B (previous half)
 *   logits  [2m][d] fp32                static per-channel pooling logits
 *   gain    [d] fp32 or NULL
 *   out     [batch][floor(T/m)][d] bf16
 * Requirements: batch >= 1, T >= m >= 1, d % 8 == 0, 8 <= d <= 1024, m <= 256
 * (m > 16 or 24*m*d > 96 KiB additionally needs logits 16-byte aligned;
 * CSA_ERR_UNSUPPORTED otherwise).  Those shapes write the 2m x d softmax
 * weights into a table taken from a memory pool of the library (stream
 * ordered, 2m*d*4 bytes per call in flight; the pool keeps its memory
 * between calls) and pool every entry but the first with them; entry 0 runs the
 * csa_compress_dynamic kernel with no Z rows (its logits Z + bias are then
 * these logits); where the pool cannot be had, on a stream being captured
 * into a CUDA graph, and for d / 8 not in {32, 64, 128}, that kernel computes
 * every entry.  Results agree with the small-m
 * kernel up to fp32 rounding order.
 */
int csa_compress(const uint16_t *A, const uint16_t *B, const float *logits,
                 int batch, long long T, int d, int m,
                 int apply_rmsnorm, const float *gain, float eps,
                 uint16_t *out, void *stream);

/*
 * csa_compress_dynamic -- compressed KV entries with input-dependent
 * compression weights ("DeepSeek v4" -> "Compressed Sparse Attention" ->
 * compressed Key-Value entry: from the hidden states, per token, the KV rows
 * C_a, C_b and the compression weights Z_a, Z_b; learnable positional biases
 * B_a, B_b; a softmax over the 2m elements of each entry; Z_b = -inf and
 * C_b = 0 before the first block).
 *
 * For every sequence b, entry i in [i0, i0 + ni) and channel c:
 *   l_j  = Zb[(i-1)m + j][c] + bias[j][c]        j = 0..m-1    (previous block, i >= 1)
 *   l_j  = Za[im + j-m][c]   + bias[j][c]        j = m..2m-1   (own block)
 *   C_i[c] = sum_j softmax_j(l)[j] * x_j[c]      x_j = B[(i-1)m + j][c], resp. A[im + j-m][c]
 * Entry 0 has no previous block: its softmax runs over the A half only.  A
 * NULL Za or Zb counts as all zeros (with both NULL the result is
 * csa_compress's with logits = bias).  If apply_rmsnorm != 0 each entry is
 * then y[c] = C_i[c] / sqrt(mean_c(C_i^2) + eps) * gain[c] (gain NULL -> 1).
 * Arithmetic in fp32 (online softmax); the result is rounded to bf16 once and
 * written to out[b][i][:].  Rows of out outside [i0, i0 + ni) are untouched, so
 * at decode time the newest entry (i0 = N - 1, ni = 1) is appended to a cache.
 *
 *   A, B      [batch][T][d] bf16     stream A (own block), stream B (previous block)
 *   Za, Zb    [batch][T][d] bf16 or NULL   compression-weight rows of A and B
 *   bias      [2m][d] fp32           rows 0..m-1: B's positional bias, m..2m-1: A's
 *   gain      [d] fp32 or NULL
 *   out       [batch][n_out][d] bf16, n_out >= i0 + ni
 * Logits must be finite or -inf (an -inf logit drops its row; a channel with
 * every logit -inf gives 0).  Requirements: batch >= 1, T >= m >= 1,
 * d % 8 == 0, 8 <= d, 0 <= i0, 0 <= ni, (i0 + ni) * m <= T; A, B, Za, Zb,
 * bias and out 16-byte aligned, gain 4-byte aligned (CSA_ERR_INVALID);
 * d <= 2048 (CSA_ERR_UNSUPPORTED).
 */
int csa_compress_dynamic(const uint16_t *A, const uint16_t *B, const uint16_t *Za, const uint16_t *Zb,
                         const float *bias, int batch, long long T, int d, int m,
                         int apply_rmsnorm, const float *gain, float eps,
                         long long i0, long long ni, uint16_t *out, long long n_out, void *stream);

/*
 * csa_index -- lightning-indexer scores ("DeepSeek v4" -> "sparse selection
 * Lightning Indexer": per-head weight times ReLU(q . K), summed over heads).
 *   S[b][q][s] = sum_h w[b][q][h] * max(0, q_idx[b][q][h] . k_idx[b][s])   for s < n_vis(q_pos[b][q])
 *   S[b][q][s] = -inf                                                      otherwise
 * bf16 operands on the tensor cores, fp32 accumulation and epilogue.
 *
 *   q_idx  [batch][nq][H_I][d_I] bf16     w [batch][nq][H_I] fp32
 *   k_idx  [batch][N][d_I] bf16           q_pos [batch][nq] int32 (0 <= t)
 *   scores [batch][nq][N] fp32 (output)
 * Requirements: d_I % 16 == 0, 16 <= d_I (else CSA_ERR_INVALID); d_I in
 * {32, 64, 128, 256} and 1 <= H_I <= 256 (padded to a multiple of 16
 * internally), else CSA_ERR_UNSUPPORTED; m >= 1; 1 <= N < 2^31.
 */
int csa_index(const uint16_t *q_idx, const float *w, const uint16_t *k_idx,
              const int *q_pos, int batch, int nq, long long N, int H_I, int d_I,
              int m, float *scores, void *stream);

/*
 * csa_quantize_fp4 -- e2m1 elements with one e4m3 scale per 16-element block
 * (the FP4 activations of the indexer QK path; "FP4 QAT details" forum post,
 * techniques map "FP4 precision for the attention indexer").
 * Per block x_0..x_15:  s = e4m3_RNE_satfinite(fp32(absmax / 6));
 *   s == 0 -> codes 0;  else q_j = e2m1_RNE_satfinite(fp32(x_j / s)), and a
 *   code whose magnitude rounds to 0 is stored as +0.
 *   x       [rows][d] bf16
 *   packed  [rows][d/2] uint8   element 2i in the low nibble, 2i+1 in the high one
 *   scales  [rows][d/16] uint8  e4m3 bit patterns
 * Requirements: rows >= 1, d % 16 == 0.
 */
int csa_quantize_fp4(const uint16_t *x, long long rows, int d,
                     uint8_t *packed, uint8_t *scales, void *stream);

/*
 * csa_index_fp4 -- csa_index on FP4 operands (layouts of csa_quantize_fp4):
 * the score is the same formula on the dequantised values e2m1 * e4m3, with
 * exact products and fp32 accumulation: block-scaled FP4 tensor-core MMAs
 * multiply the e2m1 codes and apply both operands' e4m3 block scales.  d_I in
 * {64, 128, 256}, H_I <= 128 (else CSA_ERR_UNSUPPORTED); k4s aligned to d_I/16
 * bytes and q4s to 4 bytes (else CSA_ERR_INVALID).
 *   q4 [batch][nq][H_I][d_I/2]   q4s [batch][nq][H_I][d_I/16]   w [batch][nq][H_I] fp32
 *   k4 [batch][N][d_I/2]         k4s [batch][N][d_I/16]         scores [batch][nq][N] fp32
 * Requirements: as csa_index.
 */
int csa_index_fp4(const uint8_t *q4, const uint8_t *q4s, const float *w,
                  const uint8_t *k4, const uint8_t *k4s, const int *q_pos,
                  int batch, int nq, long long N, int H_I, int d_I, int m,
                  float *scores, void *stream);

/*
 * csa_topk -- causal top-k selector ("DeepSeek v4" -> top-k selector;
 * techniques map: indices at or beyond the causal threshold become -1).
 * For each query the k largest scores among the first n_vis(t) entries; ties
 * are broken towards the lower entry index.  The chosen indices are written in
 * ascending index order; the remaining slots (when n_vis < k) are -1.
 *   scores [batch][nq][N] fp32, q_pos [batch][nq], idx [batch][nq][k] int32.
 * Requirements: 1 <= k <= 8192; N <= 2^19.  Workspace: csa_topk_workspace_bytes
 * (currently 0: the selection runs in distributed shared memory).
 */
size_t csa_topk_workspace_bytes(int batch, int nq, long long N, int k);
int csa_topk(const float *scores, const int *q_pos, int batch, int nq, long long N,
             int m, int k, int *idx, void *workspace, size_t workspace_bytes,
             void *stream);

/*
 * csa_rescore_topk -- re-ranks FP4-indexer candidates with the bf16 index keys.
 * The FP4 page ("DeepSeek V4 paper full version is out, FP4 QAT details")
 * reports 99.7 % recall of the full-precision selection for FP4 activations in
 * the indexer QK path (on real activations).  On i.i.d. synthetic data a
 * single FP4 selection recalls ~86 % of the bf16-operand top-k; this call is
 * the second stage of an over-select-and-re-score reading of that passage:
 * csa_index_fp4 + csa_topk pick kc > k candidates, then for each candidate
 *   S_c[j] = sum_h w[h] * max(0, q_idx[h] . k_idx[cand[j]])   (bf16 operands,
 *            fp32 arithmetic -- exactly the csa_index score; -1 or out-of-range
 *            candidates score -inf)
 * and idx = the k best candidates (ties towards the lower candidate slot, i.e.
 * the lower entry index when cand is ascending), written in candidate order
 * (ascending entries for ascending cand), -1 padded.
 *   q_idx [batch][nq][H_I][d_I] bf16   w [batch][nq][H_I] fp32
 *   k_idx [batch][N][d_I] bf16         cand [batch][nq][kc] int32 (from csa_topk)
 *   idx   [batch][nq][k] int32
 * Requirements: k <= 8192; kc <= 2^19; H_I and d_I as csa_index (the
 * tensor-core indexer scores the candidates; other shapes return
 * CSA_ERR_UNSUPPORTED).  Workspace:
 * csa_rescore_workspace_bytes(batch, nq, kc, k, d_I) bytes, 256-byte aligned
 * (CSA_ERR_WORKSPACE otherwise): candidate scores, chosen positions and a copy
 * of the candidates' key rows (scored by the tensor-core indexer).
 * Causality is the candidates' (they come from a causal csa_topk).
 */
size_t csa_rescore_workspace_bytes(int batch, int nq, int kc, int k, int d_I);
int csa_rescore_topk(const uint16_t *q_idx, const float *w, const uint16_t *k_idx,
                     const int *cand, int kc, int batch, int nq, long long N, int H_I,
                     int d_I, int k, int *idx, void *workspace, size_t workspace_bytes,
                     void *stream);

/*
 * csa_attend -- core attention of CSA: multi-query attention with H query
 * heads sharing one KV head (K = V) over the selected compressed entries plus
 * a sliding window of raw stream-A rows (techniques map rows "Grouped-query
 * attention" and "Sliding-window attention"; "DeepSeek v4" Figure 3 text).
 *   q_hat_h = RMSNorm(q_h) (eps, q_gain [D] or NULL = unit gain)
 *   sinks   [H] fp32 or NULL: a learnable per-head sink logit that joins each
 *             head's softmax denominator with no value row (techniques map,
 *             "Learnable attention sink"); NULL = no sink
 *   rope_cos, rope_sin [rope_positions][32] fp32 or both NULL: partial RoPE
 *             (techniques map "Partial RoPE", "Gated attention output"): the
 *             trailing 64 channels of q_hat_h rotate at the query position t
 *             in the rotate-half form (channel D-64+i with D-32+i, angle of
 *             pair i: cos/sin[t][i]) before the dot products, and out_h gets
 *             the conjugate rotation at t.  Keys and window rows must already
 *             be rotated at their own positions.  A query position outside
 *             [0, rope_positions) is not rotated.
 *   J       = { kv[b][j] : j in idx[b][q], 0 <= j < N }
 *             U { stream-A row of position u : max(0, t-W+1) <= u <= t }
 *   out_h   = R_t^-1 sum_{x in J} softmax(scale * (R_t q_hat_h) . x) * x   (R = identity without RoPE)
 * bf16 operands, fp32 softmax and accumulation, bf16 output.
 *   q       [batch][nq][H][D] bf16      kv [batch][N][D] bf16
 *   idx     [batch][nq][k] int32 (-1 = invalid slot; entries outside [0, N) are skipped)
 *   win_src [batch][win_rows][D] bf16   stream-A rows of positions win_pos0 .. win_pos0+win_rows-1
 *           (a whole stream: win_pos0 = 0, win_rows = T; a decode window cache:
 *           win_pos0 = t-W+1, win_rows = W).  Window positions the buffer does not
 *           hold are skipped.
 *   q_pos   [batch][nq] int32           out [batch][nq][H][D] bf16
 * Requirements: D in {64, 128, 256, 512}; 1 <= H <= 128; W >= 1; k >= 0.
 * Workspace: csa_attend_workspace_bytes(batch, nq, H, D, k + W).
 */
size_t csa_attend_workspace_bytes(int batch, int nq, int H, int D, long long max_keys);
int csa_attend(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
               const float *rope_sin, long long rope_positions, const uint16_t *kv, long long N,
               const int *idx, int k, const uint16_t *win_src, long long win_pos0,
               long long win_rows, int W,
               const int *q_pos, int batch, int nq, int H, int D, float scale, float eps,
               uint16_t *out, void *workspace, size_t workspace_bytes, void *stream);

/*
 * hca_attend -- core attention of HCA: as csa_attend with the key set
 * { kv[b][j] : j < n_vis(t) } U window, i.e. dense attention over every
 * visible compressed entry ("DeepSeek v4" hybrid-attention section: HCA
 * compresses every m' >> m tokens and keeps attention dense).
 * Workspace: csa_attend_workspace_bytes(batch, nq, H, D, N + W).
 */
int hca_attend(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
               const float *rope_sin, long long rope_positions, const uint16_t *kv, long long N, int m,
               const uint16_t *win_src, long long win_pos0, long long win_rows, int W,
               const int *q_pos,
               int batch, int nq, int H, int D, float scale, float eps,
               uint16_t *out, void *workspace, size_t workspace_bytes, void *stream);

/*
 * csa_decode_step -- one CSA step as a single call: csa_index -> csa_topk ->
 * csa_attend on the same stream, with the results of the three calls
 * (scores, idx, out).  The top-k and attention kernels are launched as
 * programmatic dependents of their predecessor: each starts while the
 * previous kernel finishes and waits for it only before reading its output,
 * so the attention's query load and RMSNorm overlap the top-k.  This is safe
 * because the predecessors are the library's own kernels; the separate calls
 * are ordinary launches.
 *   q_idx, w, k_idx, H_I, d_I, m: as csa_index (scores [batch][nq][N] fp32 is
 *   written, caller-owned); k, idx: as csa_topk; q .. out, workspace: as
 *   csa_attend (workspace: csa_attend_workspace_bytes(batch, nq, H, D, k + W)).
 * Requirements: those of the three calls; every argument is checked before
 * anything is launched.
 */
int csa_decode_step(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, int H_I, int d_I, int m, int k,
                    float *scores, int *idx, const uint16_t *q, const float *q_gain, const float *sinks,
                    const float *rope_cos, const float *rope_sin, long long rope_positions, const uint16_t *kv,
                    long long N, const uint16_t *win_src, long long win_pos0, long long win_rows, int W,
                    const int *q_pos, int batch, int nq, int H, int D, float scale, float eps, uint16_t *out,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * csa_attend_noalloc -- csa_attend for callers that cannot allocate device
 * memory.  No passage of the pages corresponds to it: it is a deployment
 * convenience of this library.
 *
 * Who needs it: a plugin or embedded runtime handed only a stream and tensor
 * pointers; a serving loop that must not call cudaMalloc on its hot path (it
 * synchronises the whole device); code being recorded into a CUDA graph,
 * where allocation is not allowed.  csa_attend needs caller scratch for its
 * split-KV partial results; here that scratch is a file-scope device array of
 * CSA_ATTEND_NOALLOC_MAX_BYTES per device, held by every GPU that loads the
 * library until the process exits.
 *
 * Arguments, layouts and results are those of csa_attend without the
 * workspace.  Returns CSA_ERR_WORKSPACE when csa_attend_workspace_bytes(batch,
 * nq, H, D, k + W) exceeds CSA_ATTEND_NOALLOC_MAX_BYTES (use csa_attend with
 * a caller workspace then).  Nothing is allocated or freed.
 * The first call on a device looks up the array's device address on that
 * device (cudaGetSymbolAddress); make that first call before any stream
 * capture.  That address is kept for the life of the process: after a
 * cudaDeviceReset of a device, do not call this entry point on it again (the
 * device status word of csa_sync_status has the same limit).  Bad arguments
 * are reported as csa_attend reports them, before the size check.
 * All calls share the array and it keeps the last call's contents
 * (nothing in it needs clearing: every slot read is written by the same
 * call); calls that overlap on the GPU -- different streams or host threads --
 * race on it, so serialise them.
 */
#define CSA_ATTEND_NOALLOC_MAX_BYTES (32u * 1024u * 1024u)
int csa_attend_noalloc(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
                       const float *rope_sin, long long rope_positions, const uint16_t *kv, long long N,
                       const int *idx, int k, const uint16_t *win_src, long long win_pos0,
                       long long win_rows, int W, const int *q_pos, int batch, int nq, int H, int D,
                       float scale, float eps, uint16_t *out, void *stream);

/*
 * FP8 KV cache ("DeepSeek-V4-Pro - Model techniques map", list "inference
 * quantization": FP8 KV-cache quantisation; the pages give no format).
 *
 * csa_quantize_fp8_kv -- rows x [rows][d] bf16 -> e4m3 codes [rows][d] u8 and
 * one UE8M0 exponent byte per 128 channels, exps [rows][d/128] u8, value =
 * code * 2^(e - 127).  Per 128-channel block: s = 2^k the smallest power of
 * two with absmax / s <= 448, k kept in [-124, 119] (so every code times s is
 * a finite bf16 number); codes = e4m3 round-to-nearest-even of x / s with
 * saturation, a zero magnitude stored as +0; an all-zero block has e = 127.
 * Requirements: d % 128 == 0, rows >= 0; x and codes 16-byte aligned, exps
 * non-NULL (CSA_ERR_INVALID otherwise).
 *
 * csa_attend_fp8kv / hca_attend_fp8kv -- csa_attend / hca_attend with the
 * compressed entries (kv8 [batch][N][D], kv8_exp [batch][N][D/128]) and the
 * window rows (win8 [batch][win_rows][D], win8_exp [batch][win_rows][D/128])
 * stored as above.  Each row is converted to bf16 exactly while it is
 * gathered, so the result is that of the bf16 call on the dequantised rows.
 * Requirements: those of csa_attend / hca_attend, D in {128, 256, 512}
 * (CSA_ERR_UNSUPPORTED otherwise), kv8 and win8 16-byte aligned, exponent
 * arrays non-NULL.  Workspace: as the bf16 calls.
 */
int csa_quantize_fp8_kv(const uint16_t *x, long long rows, int d, uint8_t *codes, uint8_t *exps, void *stream);
int csa_attend_fp8kv(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
                     const float *rope_sin, long long rope_positions, const uint8_t *kv8, const uint8_t *kv8_exp,
                     long long N, const int *idx, int k, const uint8_t *win8, const uint8_t *win8_exp,
                     long long win_pos0, long long win_rows, int W, const int *q_pos, int batch, int nq, int H,
                     int D, float scale, float eps, uint16_t *out, void *workspace, size_t workspace_bytes,
                     void *stream);
int hca_attend_fp8kv(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
                     const float *rope_sin, long long rope_positions, const uint8_t *kv8, const uint8_t *kv8_exp,
                     long long N, int m, const uint8_t *win8, const uint8_t *win8_exp, long long win_pos0,
                     long long win_rows, int W, const int *q_pos, int batch, int nq, int H, int D, float scale,
                     float eps, uint16_t *out, void *workspace, size_t workspace_bytes, void *stream);

/*
 * csa_sync_status -- synchronise `stream`, then read and clear the device
 * status word.  Returns CSA_ERR_TIMEOUT if a kernel gave up a bounded wait
 * since the last call, CSA_ERR_CUDA on a CUDA error, else CSA_OK.
 */
int csa_sync_status(void *stream);

/*
 * csa_set_wait_budget_ns -- upper bound (nanoseconds of device global time)
 * on any single device-side wait (mbarrier or flag) in the library's kernels;
 * 0 restores the default (2 s).  Affects kernels launched after the call.
 */
void csa_set_wait_budget_ns(unsigned long long ns);

/*
 * csa_selftest_wait_timeout -- launches one CTA that waits on an mbarrier
 * nothing ever arrives on, under the current wait budget.  The wait must give
 * up, record CSA_ERR_TIMEOUT in the status word and return; the context stays
 * usable.  Used to test the failure path without faulting the GPU.
 */
int csa_selftest_wait_timeout(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */

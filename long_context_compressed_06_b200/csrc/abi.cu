// abi.cu -- the extern "C" surface of libcsa.so (include/csa.h): argument
// validation, the device status word, the wait budget and the self-test.
// Every entry point validates on the host, then enqueues kernels on the
// caller's stream; nothing here allocates device memory.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/csa.h"
#include "common.cuh"
#include "kernels.h"

namespace {

__device__ int g_status = 0;  // CSA_OK or the first device-side error recorded

constexpr unsigned long long kDefaultBudgetNs = 2000000000ull;  // 2 s
unsigned long long g_budget_ns = kDefaultBudgetNs;

int *status_ptr() {
    // one address per device; cudaGetSymbolAddress is cheap but cache it anyway
    static int *cache[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!cache[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
        cache[dev] = static_cast<int *>(p);
    }
    return cache[dev];
}

bool ctx_for_launch(csa::DevCtx *ctx) {
    ctx->status = status_ptr();
    ctx->budget_ns = g_budget_ns;
    return ctx->status != nullptr;
}

inline bool al16(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool al4(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
inline cudaStream_t S(void *s) { return static_cast<cudaStream_t>(s); }

// selftest: an mbarrier nothing arrives on, waited for under the budget
__global__ void selftest_wait_kernel(csa::DevCtx ctx) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        csa::mbar_init(&bar, 1);
        abort_flag = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) csa::mbar_wait(csa::smem_u32(&bar), 0, ctx, &abort_flag);
    __syncthreads();
}

}  // namespace

namespace csa {
int launch_selftest_wait(const DevCtx &ctx, cudaStream_t st) {
    selftest_wait_kernel<<<1, 32, 0, st>>>(ctx);
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}
}  // namespace csa

extern "C" {

const char *csa_strerror(int status) {
    switch (status) {
        case CSA_OK: return "ok";
        case CSA_ERR_INVALID: return "invalid argument (null/misaligned pointer or bad size)";
        case CSA_ERR_UNSUPPORTED: return "unsupported shape for the compiled kernels";
        case CSA_ERR_CUDA: return "CUDA launch or runtime error";
        case CSA_ERR_WORKSPACE: return "workspace missing or too small";
        case CSA_ERR_TIMEOUT: return "a device-side bounded wait expired";
        default: return "unknown csa_status";
    }
}

int csa_version(void) { return 10000; }

void csa_set_wait_budget_ns(unsigned long long ns) { g_budget_ns = ns ? ns : kDefaultBudgetNs; }

int csa_sync_status(void *stream) {
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return CSA_ERR_CUDA;
    int *p = status_ptr();
    if (!p) return CSA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return CSA_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpy(p, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return CSA_ERR_CUDA;
    }
    return v;
}

int csa_selftest_wait_timeout(void *stream) {
    csa::DevCtx ctx;
    if (!ctx_for_launch(&ctx)) return CSA_ERR_CUDA;
    return csa::launch_selftest_wait(ctx, S(stream));
}

int csa_compress(const uint16_t *A, const uint16_t *B, const float *logits, int batch, long long T, int d,
                 int m, int apply_rmsnorm, const float *gain, float eps, uint16_t *out, void *stream) {
    if (!al16(A) || !al16(B) || !al4(logits) || !al16(out)) return CSA_ERR_INVALID;
    if (gain && !al4(gain)) return CSA_ERR_INVALID;
    if (batch < 1 || m < 1 || T < m || d < 8 || d % 8 != 0 || !(eps >= 0.f)) return CSA_ERR_INVALID;
    if (d > 1024 || m > 256) return CSA_ERR_UNSUPPORTED;
    return csa::launch_compress(A, B, logits, batch, T, d, m, apply_rmsnorm, gain, eps, out, S(stream));
}

int csa_compress_dynamic(const uint16_t *A, const uint16_t *B, const uint16_t *Za, const uint16_t *Zb,
                         const float *bias, int batch, long long T, int d, int m, int apply_rmsnorm,
                         const float *gain, float eps, long long i0, long long ni, uint16_t *out, long long n_out,
                         void *stream) {
    if (!al16(A) || !al16(B) || !al16(bias) || !al16(out)) return CSA_ERR_INVALID;
    if ((Za && !al16(Za)) || (Zb && !al16(Zb)) || (gain && !al4(gain))) return CSA_ERR_INVALID;
    if (batch < 1 || m < 1 || T < m || d < 8 || d % 8 != 0 || !(eps >= 0.f)) return CSA_ERR_INVALID;
    // overflow-free form of 0 <= i0, 0 <= ni, i0 + ni <= floor(T / m) <= n_out
    if (i0 < 0 || ni < 0 || ni > T / m || i0 > T / m - ni || n_out < i0 + ni) return CSA_ERR_INVALID;
    if (d > 2048) return CSA_ERR_UNSUPPORTED;
    return csa::launch_compress_dynamic(A, B, Za, Zb, bias, batch, T, d, m, apply_rmsnorm, gain, eps, i0, ni,
                                        n_out, out, S(stream));
}

int csa_index(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, const int *q_pos, int batch,
              int nq, long long N, int H_I, int d_I, int m, float *scores, void *stream) {
    if (!al16(q_idx) || !al4(w) || !al16(k_idx) || !al4(q_pos) || !al16(scores)) return CSA_ERR_INVALID;
    if (batch < 1 || nq < 1 || N < 1 || H_I < 1 || d_I < 16 || d_I % 16 != 0 || m < 1)
        return CSA_ERR_INVALID;
    if (!csa::index_tc_supported(H_I, d_I) || N > (1LL << 31) - 1) return CSA_ERR_UNSUPPORTED;
    csa::DevCtx ctx;
    if (!ctx_for_launch(&ctx)) return CSA_ERR_CUDA;
    return csa::launch_index(q_idx, w, k_idx, q_pos, batch, nq, N, H_I, d_I, m, scores, ctx, S(stream));
}

int csa_quantize_fp4(const uint16_t *x, long long rows, int d, uint8_t *packed, uint8_t *scales,
                     void *stream) {
    if (!al16(x) || !al16(packed) || !scales) return CSA_ERR_INVALID;
    if (rows < 1 || d < 16 || d % 16 != 0) return CSA_ERR_INVALID;
    return csa::launch_quantize_fp4(x, rows, d, packed, scales, S(stream));
}

int csa_index_fp4(const uint8_t *q4, const uint8_t *q4s, const float *w, const uint8_t *k4, const uint8_t *k4s,
                  const int *q_pos, int batch, int nq, long long N, int H_I, int d_I, int m, float *scores,
                  void *stream) {
    if (!al16(q4) || !q4s || !al4(w) || !al16(k4) || !k4s || !al4(q_pos) || !al16(scores))
        return CSA_ERR_INVALID;
    if (batch < 1 || nq < 1 || N < 1 || H_I < 1 || d_I < 16 || d_I % 16 != 0 || m < 1)
        return CSA_ERR_INVALID;
    if (!csa::index_fp4_tc_supported(H_I, d_I) || N > (1LL << 31) - 1) return CSA_ERR_UNSUPPORTED;
    // each key's d_I/16 scale bytes move as one copy aligned to their size; the
    // query scales are read as 32-bit words
    if (reinterpret_cast<uintptr_t>(k4s) % (uintptr_t)(d_I / 16) != 0 || reinterpret_cast<uintptr_t>(q4s) % 4 != 0)
        return CSA_ERR_INVALID;
    csa::DevCtx ctx;
    if (!ctx_for_launch(&ctx)) return CSA_ERR_CUDA;
    return csa::launch_index_fp4(q4, q4s, w, k4, k4s, q_pos, batch, nq, N, H_I, d_I, m, scores, ctx,
                                 S(stream));
}

size_t csa_topk_workspace_bytes(int batch, int nq, long long N, int k) {
    return csa::topk_workspace_bytes(batch, nq, N, k);
}

int csa_topk(const float *scores, const int *q_pos, int batch, int nq, long long N, int m, int k, int *idx,
             void *workspace, size_t workspace_bytes, void *stream) {
    if (!al16(scores) || !al4(q_pos) || !al4(idx)) return CSA_ERR_INVALID;
    if (batch < 1 || nq < 1 || N < 1 || m < 1 || k < 1) return CSA_ERR_INVALID;
    if (k > 8192 || N > (1LL << 19)) return CSA_ERR_UNSUPPORTED;
    if (workspace_bytes < csa::topk_workspace_bytes(batch, nq, N, k)) return CSA_ERR_WORKSPACE;
    (void)workspace;
    return csa::launch_topk(scores, q_pos, batch, nq, N, m, k, idx, S(stream));
}

size_t csa_rescore_workspace_bytes(int batch, int nq, int kc, int k, int d_I) {
    if (batch < 1 || nq < 1 || kc < 1 || k < 1 || d_I < 1) return 0;
    return csa::rescore_workspace_bytes(batch, nq, kc, k, d_I);
}

int csa_rescore_topk(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, const int *cand, int kc,
                     int batch, int nq, long long N, int H_I, int d_I, int k, int *idx, void *workspace,
                     size_t workspace_bytes, void *stream) {
    if (!al16(q_idx) || !al4(w) || !al16(k_idx) || !al4(cand) || !al4(idx)) return CSA_ERR_INVALID;
    if (batch < 1 || nq < 1 || N < 1 || kc < 1 || k < 1 || H_I < 1 || d_I < 16 || d_I % 16 != 0)
        return CSA_ERR_INVALID;
    if (k > 8192 || kc > (1 << 19) || N > (1LL << 31) - 1 || !csa::rescore_supported(H_I, d_I))
        return CSA_ERR_UNSUPPORTED;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
        workspace_bytes < csa::rescore_workspace_bytes(batch, nq, kc, k, d_I))
        return CSA_ERR_WORKSPACE;
    csa::DevCtx ctx;
    if (!ctx_for_launch(&ctx)) return CSA_ERR_CUDA;
    return csa::launch_rescore_topk(q_idx, w, k_idx, cand, kc, batch, nq, N, H_I, d_I, k, idx, workspace, ctx,
                                    S(stream));
}

size_t csa_attend_workspace_bytes(int batch, int nq, int H, int D, long long max_keys) {
    if (batch < 1 || nq < 1 || H < 1 || D < 1 || max_keys < 1) return 0;
    return csa::attend_workspace_bytes(batch, nq, H, D, max_keys);
}

static int validate_attend(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
                           const float *rope_sin, long long rope_positions, const uint16_t *kv, long long N,
                           const uint16_t *win, long long win_pos0, long long win_rows, int W, const int *q_pos,
                           int batch, int nq, int H, int D, float eps, const void *out) {
    if (!al16(q) || !al16(kv) || !al16(win) || !al4(q_pos) || !al16(out)) return CSA_ERR_INVALID;
    if ((q_gain && !al4(q_gain)) || (sinks && !al4(sinks))) return CSA_ERR_INVALID;
    if ((rope_cos == nullptr) != (rope_sin == nullptr)) return CSA_ERR_INVALID;
    if (rope_cos && (!al4(rope_cos) || !al4(rope_sin) || rope_positions < 1)) return CSA_ERR_INVALID;
    if (batch < 1 || nq < 1 || N < 1 || win_pos0 < 0 || win_rows < 1 || W < 1 || H < 1 || D < 1 || !(eps >= 0.f))
        return CSA_ERR_INVALID;
    if (H > 128 || !(D == 64 || D == 128 || D == 256 || D == 512)) return CSA_ERR_UNSUPPORTED;
    return CSA_OK;
}

}  // extern "C"

namespace csa {
// The argument checks of csa_attend before its workspace check (shared with
// csa_attend_noalloc, so that call reports a bad argument as such rather than
// as a workspace shortfall).
int check_attend_args(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
                      const float *rope_sin, long long rope_positions, const uint16_t *kv, long long N,
                      const int *idx, int k, const uint16_t *win, long long win_pos0, long long win_rows, int W,
                      const int *q_pos, int batch, int nq, int H, int D, float eps, const void *out) {
    const int rc = validate_attend(q, q_gain, sinks, rope_cos, rope_sin, rope_positions, kv, N, win, win_pos0,
                                   win_rows, W, q_pos, batch, nq, H, D, eps, out);
    if (rc != CSA_OK) return rc;
    if (k < 0 || (k > 0 && !al4(idx))) return CSA_ERR_INVALID;
    return CSA_OK;
}
}  // namespace csa

extern "C" {

int csa_attend(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
               const float *rope_sin, long long rope_positions, const uint16_t *kv, long long N,
               const int *idx, int k,
               const uint16_t *win_src, long long win_pos0, long long win_rows, int W, const int *q_pos, int batch,
               int nq, int H, int D, float scale, float eps, uint16_t *out, void *workspace, size_t workspace_bytes,
               void *stream) {
    const int rc = csa::check_attend_args(q, q_gain, sinks, rope_cos, rope_sin, rope_positions, kv, N, idx, k,
                                          win_src, win_pos0, win_rows, W, q_pos, batch, nq, H, D, eps, out);
    if (rc != CSA_OK) return rc;
    if (workspace_bytes < csa::attend_workspace_bytes(batch, nq, H, D, (long long)k + W) ||
        (workspace_bytes > 0 && !al16(workspace)))
        return CSA_ERR_WORKSPACE;
    csa::DevCtx ctx;
    if (!ctx_for_launch(&ctx)) return CSA_ERR_CUDA;
    return csa::launch_attend(q, q_gain, sinks, rope_cos, rope_sin, rope_positions, nullptr, kv, N, 1, k > 0 ? idx : nullptr, k, false, win_src, win_pos0,
                              win_rows, W,
                              q_pos, batch, nq, H, D, scale, eps, out, workspace, workspace_bytes, ctx, S(stream));
}

int hca_attend(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
               const float *rope_sin, long long rope_positions, const uint16_t *kv, long long N, int m,
               const uint16_t *win_src, long long win_pos0, long long win_rows, int W, const int *q_pos, int batch,
               int nq, int H, int D, float scale, float eps, uint16_t *out, void *workspace, size_t workspace_bytes,
               void *stream) {
    int rc = validate_attend(q, q_gain, sinks, rope_cos, rope_sin, rope_positions, kv, N, win_src, win_pos0,
                             win_rows, W, q_pos, batch, nq, H, D, eps, out);
    if (rc != CSA_OK) return rc;
    if (m < 1) return CSA_ERR_INVALID;
    if (workspace_bytes < csa::attend_workspace_bytes(batch, nq, H, D, N + W) ||
        (workspace_bytes > 0 && !al16(workspace)))
        return CSA_ERR_WORKSPACE;
    csa::DevCtx ctx;
    if (!ctx_for_launch(&ctx)) return CSA_ERR_CUDA;
    return csa::launch_attend(q, q_gain, sinks, rope_cos, rope_sin, rope_positions, nullptr, kv, N, m, nullptr, 0, true, win_src, win_pos0, win_rows, W, q_pos,
                              batch,
                              nq, H, D, scale, eps, out, workspace, workspace_bytes, ctx, S(stream));
}

int csa_decode_step(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, int H_I, int d_I, int m, int k,
                    float *scores, int *idx, const uint16_t *q, const float *q_gain, const float *sinks,
                    const float *rope_cos, const float *rope_sin, long long rope_positions, const uint16_t *kv,
                    long long N, const uint16_t *win_src, long long win_pos0, long long win_rows, int W,
                    const int *q_pos, int batch, int nq, int H, int D, float scale, float eps, uint16_t *out,
                    void *workspace, size_t workspace_bytes, void *stream) {
    // every argument of the three calls first: nothing is launched for a bad one
    if (!al16(q_idx) || !al4(w) || !al16(k_idx) || !al4(q_pos) || !al16(scores) || !al4(idx)) return CSA_ERR_INVALID;
    if (batch < 1 || nq < 1 || N < 1 || H_I < 1 || d_I < 16 || d_I % 16 != 0 || m < 1 || k < 1)
        return CSA_ERR_INVALID;
    if (!csa::index_tc_supported(H_I, d_I) || k > 8192 || N > (1LL << 19)) return CSA_ERR_UNSUPPORTED;
    if (csa::topk_workspace_bytes(batch, nq, N, k) != 0) return CSA_ERR_UNSUPPORTED;
    int rc = csa::check_attend_args(q, q_gain, sinks, rope_cos, rope_sin, rope_positions, kv, N, idx, k, win_src,
                                    win_pos0, win_rows, W, q_pos, batch, nq, H, D, eps, out);
    if (rc != CSA_OK) return rc;
    if (workspace_bytes < csa::attend_workspace_bytes(batch, nq, H, D, (long long)k + W) ||
        (workspace_bytes > 0 && !al16(workspace)))
        return CSA_ERR_WORKSPACE;
    csa::DevCtx ctx;
    if (!ctx_for_launch(&ctx)) return CSA_ERR_CUDA;
    rc = csa::launch_index(q_idx, w, k_idx, q_pos, batch, nq, N, H_I, d_I, m, scores, ctx, S(stream));
    if (rc != CSA_OK) return rc;
    rc = csa::launch_topk(scores, q_pos, batch, nq, N, m, k, idx, S(stream), /*pdl=*/true);
    if (rc != CSA_OK) return rc;
    return csa::launch_attend(q, q_gain, sinks, rope_cos, rope_sin, rope_positions, nullptr, kv, N, 1, idx, k, false,
                              win_src, win_pos0, win_rows, W, q_pos, batch, nq, H, D, scale, eps, out, workspace,
                              workspace_bytes, ctx, S(stream), /*pdl=*/true);
}

int csa_quantize_fp8_kv(const uint16_t *x, long long rows, int d, uint8_t *codes, uint8_t *exps, void *stream) {
    if (!al16(x) || !al16(codes) || !exps) return CSA_ERR_INVALID;
    if (rows < 0 || d < 128 || d % 128 != 0) return CSA_ERR_INVALID;
    return csa::launch_quantize_fp8_kv(x, rows, d, codes, exps, S(stream));
}

static int validate_fp8kv(const uint8_t *kv8, const uint8_t *kv8_exp, const uint8_t *win8, const uint8_t *win8_exp,
                          int D) {
    if (!al16(kv8) || !al16(win8) || !kv8_exp || !win8_exp) return CSA_ERR_INVALID;
    if (D % 128 != 0) return CSA_ERR_UNSUPPORTED;
    return CSA_OK;
}

int csa_attend_fp8kv(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
                     const float *rope_sin, long long rope_positions, const uint8_t *kv8, const uint8_t *kv8_exp,
                     long long N, const int *idx, int k, const uint8_t *win8, const uint8_t *win8_exp,
                     long long win_pos0, long long win_rows, int W, const int *q_pos, int batch, int nq, int H, int D,
                     float scale, float eps, uint16_t *out, void *workspace, size_t workspace_bytes, void *stream) {
    int rc = validate_attend(q, q_gain, sinks, rope_cos, rope_sin, rope_positions,
                             reinterpret_cast<const uint16_t *>(kv8), N, reinterpret_cast<const uint16_t *>(win8),
                             win_pos0, win_rows, W, q_pos, batch, nq, H, D, eps, out);
    if (rc != CSA_OK) return rc;
    rc = validate_fp8kv(kv8, kv8_exp, win8, win8_exp, D);
    if (rc != CSA_OK) return rc;
    if (k < 0 || (k > 0 && !al4(idx))) return CSA_ERR_INVALID;
    if (workspace_bytes < csa::attend_workspace_bytes(batch, nq, H, D, (long long)k + W) ||
        (workspace_bytes > 0 && !al16(workspace)))
        return CSA_ERR_WORKSPACE;
    csa::DevCtx ctx;
    if (!ctx_for_launch(&ctx)) return CSA_ERR_CUDA;
    const csa::Fp8Kv f8 = {kv8, kv8_exp, win8, win8_exp};
    return csa::launch_attend(q, q_gain, sinks, rope_cos, rope_sin, rope_positions, &f8, nullptr, N, 1,
                              k > 0 ? idx : nullptr, k, false, nullptr, win_pos0, win_rows, W, q_pos, batch, nq, H, D,
                              scale, eps, out, workspace, workspace_bytes, ctx, S(stream));
}

int hca_attend_fp8kv(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
                     const float *rope_sin, long long rope_positions, const uint8_t *kv8, const uint8_t *kv8_exp,
                     long long N, int m, const uint8_t *win8, const uint8_t *win8_exp, long long win_pos0,
                     long long win_rows, int W, const int *q_pos, int batch, int nq, int H, int D, float scale,
                     float eps, uint16_t *out, void *workspace, size_t workspace_bytes, void *stream) {
    int rc = validate_attend(q, q_gain, sinks, rope_cos, rope_sin, rope_positions,
                             reinterpret_cast<const uint16_t *>(kv8), N, reinterpret_cast<const uint16_t *>(win8),
                             win_pos0, win_rows, W, q_pos, batch, nq, H, D, eps, out);
    if (rc != CSA_OK) return rc;
    rc = validate_fp8kv(kv8, kv8_exp, win8, win8_exp, D);
    if (rc != CSA_OK) return rc;
    if (m < 1) return CSA_ERR_INVALID;
    if (workspace_bytes < csa::attend_workspace_bytes(batch, nq, H, D, N + W) ||
        (workspace_bytes > 0 && !al16(workspace)))
        return CSA_ERR_WORKSPACE;
    csa::DevCtx ctx;
    if (!ctx_for_launch(&ctx)) return CSA_ERR_CUDA;
    const csa::Fp8Kv f8 = {kv8, kv8_exp, win8, win8_exp};
    return csa::launch_attend(q, q_gain, sinks, rope_cos, rope_sin, rope_positions, &f8, nullptr, N, m, nullptr, 0,
                              true, nullptr, win_pos0, win_rows, W, q_pos, batch, nq, H, D, scale, eps, out,
                              workspace, workspace_bytes, ctx, S(stream));
}

}  // extern "C"

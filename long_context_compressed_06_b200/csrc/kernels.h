// kernels.h -- internal host-side launchers (validated arguments in, status out).
// The C ABI in abi.cu validates every argument and then calls these.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace csa {

struct DevCtx;

int launch_compress(const uint16_t *A, const uint16_t *B, const float *logits, int batch, long long T,
                    int d, int m, int apply_rmsnorm, const float *gain, float eps, uint16_t *out,
                    cudaStream_t st);

int launch_compress_dynamic(const uint16_t *A, const uint16_t *B, const uint16_t *Za, const uint16_t *Zb,
                            const float *bias, int batch, long long T, int d, int m, int apply_rmsnorm,
                            const float *gain, float eps, long long i0, long long ni, long long n_out,
                            uint16_t *out, cudaStream_t st);

int launch_quantize_fp8_kv(const uint16_t *x, long long rows, int d, uint8_t *codes, uint8_t *exps, cudaStream_t st);

int launch_index(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, const int *q_pos,
                 int batch, int nq, long long N, int H_I, int d_I, int m, float *scores,
                 const DevCtx &ctx, cudaStream_t st);

int launch_quantize_fp4(const uint16_t *x, long long rows, int d, uint8_t *packed, uint8_t *scales,
                        cudaStream_t st);

int launch_index_fp4(const uint8_t *q4, const uint8_t *q4s, const float *w, const uint8_t *k4,
                     const uint8_t *k4s, const int *q_pos, int batch, int nq, long long N, int H_I,
                     int d_I, int m, float *scores, const DevCtx &ctx, cudaStream_t st);

size_t topk_workspace_bytes(int batch, int nq, long long N, int k);
// q_pos may be null inside the library: every entry is then eligible.
// pdl: launched as a programmatic dependent of the stream's previous kernel
// (the kernel waits for it before reading scores) -- only for chains whose
// predecessor is this library's own kernel (csa_decode_step).
int launch_topk(const float *scores, const int *q_pos, int batch, int nq, long long N, int m, int k,
                int *idx, cudaStream_t st, bool pdl = false);

size_t rescore_workspace_bytes(int batch, int nq, int kc, int k, int d_I);
bool rescore_supported(int H_I, int d_I);
int launch_rescore_topk(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, const int *cand, int kc,
                        int batch, int nq, long long N, int H_I, int d_I, int k, int *idx, void *ws,
                        const DevCtx &ctx, cudaStream_t st);

// Shapes the tensor-core indexers take (the only implementation).
bool index_tc_supported(int H_I, int d_I);
bool index_fp4_tc_supported(int H_I, int d_I);
int launch_index_tc(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, const int *q_pos, int batch,
                    int nq, long long N, int H_I, int d_I, int m, float *scores, const DevCtx &ctx,
                    cudaStream_t st);

// Attention: dense selects the HCA key set of the first n_vis(t) entries;
// otherwise the k selected entries idx (may be null when k == 0).
size_t attend_workspace_bytes(int batch, int nq, int H, int D, long long max_keys);
// The FP8 KV cache of one attention call: e4m3 codes and UE8M0 exponent
// bytes of the compressed entries and of the window rows.
struct Fp8Kv {
    const uint8_t *kv, *kv_exp, *win, *win_exp;
};

int launch_attend(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
                  const float *rope_sin, long long rope_npos, const Fp8Kv *fp8, const uint16_t *kv, long long N, int m,
                  const int *idx, int k, bool dense, const uint16_t *win, long long win_pos0, long long win_rows,
                  int W, const int *q_pos,
                  int batch, int nq, int H, int D, float scale, float eps, uint16_t *out,
                  void *ws, size_t ws_bytes, const DevCtx &ctx, cudaStream_t st, bool pdl = false);

int launch_selftest_wait(const DevCtx &ctx, cudaStream_t st);

// Host-side argument checks of csa_attend (everything but the workspace).
int check_attend_args(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
                      const float *rope_sin, long long rope_positions, const uint16_t *kv, long long N,
                      const int *idx, int k, const uint16_t *win, long long win_pos0, long long win_rows, int W,
                      const int *q_pos, int batch, int nq, int H, int D, float eps, const void *out);

}  // namespace csa

// index.cu -- csa_index / csa_index_fp4 dispatch.
#include "common.cuh"
#include "kernels.h"

namespace csa {

int launch_index_simt(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, const int *q_pos,
                      int batch, int nq, long long N, int H_I, int d_I, int m, float *scores,
                      cudaStream_t st);
int launch_index_fp4_simt(const uint8_t *q4, const uint8_t *q4s, const float *w, const uint8_t *k4,
                          const uint8_t *k4s, const int *q_pos, int batch, int nq, long long N, int H_I,
                          int d_I, int m, float *scores, cudaStream_t st);

bool index_tc_supported(int H_I, int d_I);
int launch_index_tc(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, const int *q_pos, int batch,
                    int nq, long long N, int H_I, int d_I, int m, float *scores, const DevCtx &ctx,
                    cudaStream_t st);

bool index_fp4_tc_supported(int H_I, int d_I);
int launch_index_fp4_tc(const uint8_t *q4, const uint8_t *q4s, const float *w, const uint8_t *k4,
                        const uint8_t *k4s, const int *q_pos, int batch, int nq, long long N, int H_I, int d_I,
                        int m, float *scores, const DevCtx &ctx, cudaStream_t st);

int launch_index(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, const int *q_pos, int batch,
                 int nq, long long N, int H_I, int d_I, int m, float *scores, const DevCtx &ctx,
                 cudaStream_t st) {
    if (index_tc_supported(H_I, d_I))
        return launch_index_tc(q_idx, w, k_idx, q_pos, batch, nq, N, H_I, d_I, m, scores, ctx, st);
    return launch_index_simt(q_idx, w, k_idx, q_pos, batch, nq, N, H_I, d_I, m, scores, st);
}

int launch_index_fp4(const uint8_t *q4, const uint8_t *q4s, const float *w, const uint8_t *k4,
                     const uint8_t *k4s, const int *q_pos, int batch, int nq, long long N, int H_I, int d_I,
                     int m, float *scores, const DevCtx &ctx, cudaStream_t st) {
    // the tensor-core path copies each key's d_I/16 scale bytes with one cp.async,
    // which needs them aligned to their size
    const bool scales_aligned = reinterpret_cast<uintptr_t>(k4s) % (uintptr_t)(d_I / 16) == 0 &&
                                reinterpret_cast<uintptr_t>(q4s) % 2 == 0;
    if (index_fp4_tc_supported(H_I, d_I) && scales_aligned)
        return launch_index_fp4_tc(q4, q4s, w, k4, k4s, q_pos, batch, nq, N, H_I, d_I, m, scores, ctx, st);
    return launch_index_fp4_simt(q4, q4s, w, k4, k4s, q_pos, batch, nq, N, H_I, d_I, m, scores, st);
}

}  // namespace csa

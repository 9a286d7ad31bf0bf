// index.cu -- csa_index / csa_index_fp4 dispatch to the tensor-core kernels.
// Shapes outside their compiled tiles return CSA_ERR_UNSUPPORTED; there is no
// second (CUDA-core) implementation.
#include "common.cuh"
#include "kernels.h"

namespace csa {

int launch_index_fp4_tc(const uint8_t *q4, const uint8_t *q4s, const float *w, const uint8_t *k4,
                        const uint8_t *k4s, const int *q_pos, int batch, int nq, long long N, int H_I, int d_I,
                        int m, float *scores, const DevCtx &ctx, cudaStream_t st);

int launch_index(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, const int *q_pos, int batch,
                 int nq, long long N, int H_I, int d_I, int m, float *scores, const DevCtx &ctx,
                 cudaStream_t st) {
    if (!index_tc_supported(H_I, d_I)) return CSA_ERR_UNSUPPORTED;
    return launch_index_tc(q_idx, w, k_idx, q_pos, batch, nq, N, H_I, d_I, m, scores, ctx, st);
}

int launch_index_fp4(const uint8_t *q4, const uint8_t *q4s, const float *w, const uint8_t *k4,
                     const uint8_t *k4s, const int *q_pos, int batch, int nq, long long N, int H_I, int d_I,
                     int m, float *scores, const DevCtx &ctx, cudaStream_t st) {
    if (!index_fp4_tc_supported(H_I, d_I)) return CSA_ERR_UNSUPPORTED;
    return launch_index_fp4_tc(q4, q4s, w, k4, k4s, q_pos, batch, nq, N, H_I, d_I, m, scores, ctx, st);
}

}  // namespace csa

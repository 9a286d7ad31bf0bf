// index_simt.cu -- lightning-indexer scores on CUDA cores (csa_index /
// csa_index_fp4 for shapes the tensor-core kernels do not take).
//
//   S[q][s] = sum_h w[q][h] * max(0, q_I[q][h] . K_I[s])  for s < n_vis(t_q), else -inf
// ("DeepSeek v4" -> "sparse selection Lightning Indexer").  One thread per
// compressed entry; the query's indexer heads sit in shared memory as fp32.
// FP4 operands are dequantised exactly (e2m1 value times e4m3 scale) into
// fp32 before the same dot products.
#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kSimtKeys = 128;

CSA_DEVINL float e2m1_val(uint32_t code) {
    // magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} for codes 0..7, bit 3 = sign
    const float mag = (code & 6u) == 0u ? 0.5f * (float)(code & 1u)
                                        : __uint_as_float(((code >> 1 & 3u) + 126u) << 23) *
                                              (1.0f + 0.5f * (float)(code & 1u));
    return (code & 8u) ? -mag : mag;
}

CSA_DEVINL float e4m3_val(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, mt = c & 7u;
    const float v = e == 0u ? (float)mt * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (mt << 20));
    return (c & 0x80u) ? -v : v;
}

struct Bf16Keys {
    const uint16_t *k;
    int d_I;
    // 16 consecutive key elements starting at j (j % 16 == 0) as fp32
    CSA_DEVINL void load16(long long row, int j, float f[16]) const {
        const uint16_t *p = k + (size_t)row * d_I + j;
        unpack8(ldg16(p), f);
        unpack8(ldg16(p + 8), f + 8);
    }
};

struct Fp4Keys {
    const uint8_t *k4, *k4s;
    int d_I;
    CSA_DEVINL void load16(long long row, int j, float f[16]) const {
        const uint2 c = __ldg(reinterpret_cast<const uint2 *>(k4 + (size_t)row * (d_I / 2) + j / 2));
        const float s = e4m3_val(__ldg(k4s + (size_t)row * (d_I / 16) + j / 16));
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            f[i] = e2m1_val((c.x >> (4 * i)) & 15u) * s;
            f[8 + i] = e2m1_val((c.y >> (4 * i)) & 15u) * s;
        }
    }
};

// q_s: [H_I][d_I] fp32 in shared memory, w_s: [H_I]
template <class Keys>
__global__ void __launch_bounds__(kSimtKeys) index_simt_kernel(Keys keys, const void *__restrict__ qsrc,
                                                               const uint8_t *__restrict__ q4s,
                                                               int q_is_fp4, const float *__restrict__ w,
                                                               const int *__restrict__ q_pos, int nq,
                                                               long long N, int H_I, int d_I, int m,
                                                               float *__restrict__ scores) {
    extern __shared__ __align__(16) float sm[];
    float *q_s = sm;
    float *w_s = sm + H_I * d_I;
    const long long bq = blockIdx.y;
    const long long b = bq / nq;
    for (int i = threadIdx.x; i < H_I * d_I; i += blockDim.x) {
        float v;
        if (q_is_fp4) {
            const uint8_t *q4 = reinterpret_cast<const uint8_t *>(qsrc) + (size_t)bq * H_I * (d_I / 2);
            const uint32_t byte = q4[i / 2];
            v = e2m1_val((i & 1) ? byte >> 4 : byte & 15u) *
                e4m3_val(q4s[(size_t)bq * H_I * (d_I / 16) + i / 16]);
        } else {
            const uint16_t *q = reinterpret_cast<const uint16_t *>(qsrc) + (size_t)bq * H_I * d_I;
            v = __uint_as_float((uint32_t)q[i] << 16);
        }
        q_s[i] = v;
    }
    for (int h = threadIdx.x; h < H_I; h += blockDim.x) w_s[h] = w[bq * H_I + h];
    __syncthreads();

    const long long s = (long long)blockIdx.x * kSimtKeys + threadIdx.x;
    if (s >= N) return;
    const long long nv = n_visible(q_pos[bq], m, N);
    float score = -INFINITY;
    if (s < nv) {
        score = 0.f;
        const long long row = b * N + s;
        for (int h0 = 0; h0 < H_I; h0 += 16) {
            float acc[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) acc[h] = 0.f;
            for (int j = 0; j < d_I; j += 16) {
                float kf[16];
                keys.load16(row, j, kf);
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    if (h0 + h < H_I) {
                        const float4 *qv = reinterpret_cast<const float4 *>(q_s + (size_t)(h0 + h) * d_I + j);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4) {
                            const float4 qq = qv[v4];
                            acc[h] = fmaf(qq.x, kf[4 * v4 + 0], acc[h]);
                            acc[h] = fmaf(qq.y, kf[4 * v4 + 1], acc[h]);
                            acc[h] = fmaf(qq.z, kf[4 * v4 + 2], acc[h]);
                            acc[h] = fmaf(qq.w, kf[4 * v4 + 3], acc[h]);
                        }
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < 16; ++h)
                if (h0 + h < H_I) score = fmaf(w_s[h0 + h], fmaxf(acc[h], 0.f), score);
        }
    }
    scores[bq * N + s] = score;
}

template <class Keys>
int run(Keys keys, const void *q, const uint8_t *q4s, int q_is_fp4, const float *w, const int *q_pos,
        int batch, int nq, long long N, int H_I, int d_I, int m, float *scores, cudaStream_t st) {
    const size_t smem = ((size_t)H_I * d_I + H_I) * sizeof(float);
    auto k = index_simt_kernel<Keys>;
    if (smem > 48 * 1024) {
        if (smem > 200 * 1024) return CSA_ERR_UNSUPPORTED;
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return CSA_ERR_CUDA;
    }
    dim3 grid((unsigned)((N + kSimtKeys - 1) / kSimtKeys), (unsigned)(batch * nq));
    k<<<grid, kSimtKeys, smem, st>>>(keys, q, q4s, q_is_fp4, w, q_pos, nq, N, H_I, d_I, m, scores);
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // namespace

int launch_index_simt(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, const int *q_pos,
                      int batch, int nq, long long N, int H_I, int d_I, int m, float *scores,
                      cudaStream_t st) {
    return run(Bf16Keys{k_idx, d_I}, q_idx, nullptr, 0, w, q_pos, batch, nq, N, H_I, d_I, m, scores, st);
}

int launch_index_fp4_simt(const uint8_t *q4, const uint8_t *q4s, const float *w, const uint8_t *k4,
                          const uint8_t *k4s, const int *q_pos, int batch, int nq, long long N, int H_I,
                          int d_I, int m, float *scores, cudaStream_t st) {
    return run(Fp4Keys{k4, k4s, d_I}, q4, q4s, 1, w, q_pos, batch, nq, N, H_I, d_I, m, scores, st);
}

}  // namespace csa

// compress.cu -- compressed KV entries from the two latent streams (csa_compress).
//
// Entry i pools 2m rows per channel with a per-channel softmax over static
// logits: rows 0..m-1 weight the previous m tokens of stream B, rows m..2m-1
// the newest m tokens of stream A; entry 0 pools its m A tokens only.  An
// optional RMSNorm over the d channels follows ("DeepSeek v4", section
// "Compressed Sparse Attention" -> compressed Key-Value entry; anthology
// record "Key takeaways": RMSNorm on the single compressed KV head).
//
// The op streams 2*T*d bf16 from HBM and writes T/m*d bf16: it is HBM bound.
//   * small m (2m*d weights fit comfortably in shared memory): the softmax
//     weights are static, so each CTA computes them once into shared memory
//     and every element costs one FMA; one warp per entry, the whole row in
//     registers, RMSNorm by a warp reduction;
//   * large m (HCA, m = 128): the input-dependent compressor with no Z rows
//     (its logits Z + bias reduce to the static logits as the bias), a thread
//     per (entry, 8 channels) with an online softmax over the 2m rows: the
//     weights of all d channels do not fit in shared memory, and a cluster
//     that split the channels and exchanged the RMSNorm sums measured 1.18
//     TB/s against this kernel's rate.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa {
namespace {

// Per-channel softmax weights of the 2m logits (w_full) and of the A half
// alone (w_first, entry 0), for channels [c0, c0 + dc), into shared memory.
__device__ void pooling_weights(const float *__restrict__ logits, int d, int m, int c0, int dc,
                                float *w_full, float *w_first) {
    for (int c = threadIdx.x; c < dc; c += blockDim.x) {
        const float *L = logits + c0 + c;
        float mx = -INFINITY, mx0 = -INFINITY;
        for (int j = 0; j < 2 * m; ++j) {
            mx = fmaxf(mx, L[(size_t)j * d]);
            if (j >= m) mx0 = fmaxf(mx0, L[(size_t)j * d]);
        }
        float den = 0.f, den0 = 0.f;
        for (int j = 0; j < 2 * m; ++j) {
            den += expf(L[(size_t)j * d] - mx);
            if (j >= m) den0 += expf(L[(size_t)j * d] - mx0);
        }
        for (int j = 0; j < 2 * m; ++j) {
            w_full[(size_t)j * dc + c] = expf(L[(size_t)j * d] - mx) / den;
            if (j >= m) w_first[(size_t)(j - m) * dc + c] = expf(L[(size_t)j * d] - mx0) / den0;
        }
    }
}

CSA_DEVINL void fma8(float acc[8], const float *w, const uint4 &x) {
    float f[8];
    unpack8(x, f);
    const float4 w0 = *reinterpret_cast<const float4 *>(w);
    const float4 w1 = *reinterpret_cast<const float4 *>(w + 4);
    acc[0] = fmaf(w0.x, f[0], acc[0]); acc[1] = fmaf(w0.y, f[1], acc[1]);
    acc[2] = fmaf(w0.z, f[2], acc[2]); acc[3] = fmaf(w0.w, f[3], acc[3]);
    acc[4] = fmaf(w1.x, f[4], acc[4]); acc[5] = fmaf(w1.y, f[5], acc[5]);
    acc[6] = fmaf(w1.z, f[6], acc[6]); acc[7] = fmaf(w1.w, f[7], acc[7]);
}

// ------------------------------------------------------------------ small m
// MT: compile-time m (0 = runtime); CPL: 8-channel chunks per lane.
template <int MT, int CPL>
__global__ void __launch_bounds__(256) compress_small_kernel(
    const uint16_t *__restrict__ A, const uint16_t *__restrict__ B, const float *__restrict__ logits,
    int batch, long long T, int d, int m_rt, int apply_rms, const float *__restrict__ gain, float eps,
    uint16_t *__restrict__ out, long long N) {
    const int m = MT ? MT : m_rt;
    extern __shared__ __align__(16) float smem[];
    float *w_full = smem;              // [2m][d]
    float *w_first = smem + 2 * m * d; // [m][d]
    pooling_weights(logits, d, m, 0, d, w_full, w_first);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nchunk = d >> 3;
    const long long total = (long long)batch * N;
    for (long long e = (long long)blockIdx.x * 8 + warp; e < total; e += (long long)gridDim.x * 8) {
        const long long b = e / N, i = e - b * N;
        const uint16_t *Ab = A + (size_t)b * T * d;
        const uint16_t *Bb = B + (size_t)b * T * d;
        float acc[CPL][8];
        float ss = 0.f;
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc) {
            const int ch = lane + 32 * cc;
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[cc][q] = 0.f;
            if (ch < nchunk) {
                const int c0 = ch * 8;
                if (i == 0) {
#pragma unroll 8
                    for (int j = 0; j < m; ++j)
                        fma8(acc[cc], w_first + (size_t)j * d + c0, ldg_stream(Ab + (size_t)j * d + c0));
                } else {
                    const uint16_t *Bp = Bb + (size_t)(i - 1) * m * d + c0;
                    const uint16_t *Ap = Ab + (size_t)i * m * d + c0;
#pragma unroll 8
                    for (int j = 0; j < m; ++j)
                        fma8(acc[cc], w_full + (size_t)j * d + c0, ldg_stream(Bp + (size_t)j * d));
#pragma unroll 8
                    for (int j = 0; j < m; ++j)
                        fma8(acc[cc], w_full + (size_t)(m + j) * d + c0, ldg_stream(Ap + (size_t)j * d));
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) ss = fmaf(acc[cc][q], acc[cc][q], ss);
            }
        }
        float r = 1.f;
        if (apply_rms) {
            ss = warp_sum(ss);
            r = 1.0f / sqrtf(ss / (float)d + eps);
        }
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc) {
            const int ch = lane + 32 * cc;
            if (ch < nchunk) {
                const int c0 = ch * 8;
                float o[8];
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    o[q] = acc[cc][q] * r * ((apply_rms && gain) ? __ldg(gain + c0 + q) : 1.f);
                *reinterpret_cast<uint4 *>(out + (size_t)e * d + c0) = pack8(o);
            }
        }
    }
}

template <int MT, int CPL>
cudaError_t run_small(const uint16_t *A, const uint16_t *B, const float *logits, int batch, long long T,
                      int d, int m, int apply_rms, const float *gain, float eps, uint16_t *out,
                      long long N, size_t smem, int grid, cudaStream_t st) {
    auto k = compress_small_kernel<MT, CPL>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k<<<grid, 256, smem, st>>>(A, B, logits, batch, T, d, m, apply_rms, gain, eps, out, N);
    return cudaGetLastError();
}

}  // namespace

int launch_compress(const uint16_t *A, const uint16_t *B, const float *logits, int batch, long long T,
                    int d, int m, int apply_rmsnorm, const float *gain, float eps, uint16_t *out,
                    cudaStream_t st) {
    const long long N = T / m;
    if (N <= 0) return CSA_OK;
    const long long total = (long long)batch * N;
    const int sms = num_sms();
    const size_t small_smem = (size_t)3 * m * d * sizeof(float);
    cudaError_t err;
    if (m <= 16 && small_smem <= 96 * 1024 && d <= 1024) {
        const int grid = (int)std::min<long long>((total + 7) / 8, (long long)sms * 8);
        const int nchunk = d / 8;
        if (m == 4 && nchunk <= 64)
            err = run_small<4, 2>(A, B, logits, batch, T, d, m, apply_rmsnorm, gain, eps, out, N, small_smem, grid, st);
        else if (nchunk <= 32)
            err = run_small<0, 1>(A, B, logits, batch, T, d, m, apply_rmsnorm, gain, eps, out, N, small_smem, grid, st);
        else if (nchunk <= 64)
            err = run_small<0, 2>(A, B, logits, batch, T, d, m, apply_rmsnorm, gain, eps, out, N, small_smem, grid, st);
        else
            err = run_small<0, 4>(A, B, logits, batch, T, d, m, apply_rmsnorm, gain, eps, out, N, small_smem, grid, st);
        return err == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
    }
    // large m: the input-dependent compressor without Z rows, the logits as its
    // bias (read as float4: 16-byte aligned)
    if ((reinterpret_cast<uintptr_t>(logits) & 15) != 0) return CSA_ERR_UNSUPPORTED;
    return launch_compress_dynamic(A, B, nullptr, nullptr, logits, batch, T, d, m, apply_rmsnorm, gain, eps, 0, N,
                                   N, out, st);
}

}  // namespace csa

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
// The softmax weights are static, so each CTA computes them once into shared
// memory and every element costs one FMA.  Two kernels:
//   * small m (2m*d weights fit comfortably in shared memory): one warp per
//     entry, the whole row in registers, RMSNorm by a warp reduction;
//   * large m (HCA, m = 128): a thread-block cluster splits the channels, each
//     CTA keeps the weights of its channel slice in shared memory, and the
//     RMSNorm sum of squares is exchanged through distributed shared memory.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace cg = cooperative_groups;

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

// ------------------------------------------------------------------ large m
// A cluster of G CTAs handles groups of E = 256/dc consecutive entries; CTA
// `rank` owns channels [rank*dc, (rank+1)*dc).  The 256 threads are RG row
// groups x (dc/8) channel chunks while pooling (thread sums rows rg, rg+RG, ..)
// and E entries x dc channels (one output each) while reducing/normalising.
// A thread issues the 16-byte loads of NR of its rows of every entry of the
// group before the first FMA, so E*NR loads per thread are in flight (the op
// is bound by HBM latency x bytes in flight); larger m takes several batches.
template <int E, int NR>
__global__ void __launch_bounds__(256, 1) compress_cluster_kernel(
    const uint16_t *__restrict__ A, const uint16_t *__restrict__ B, const float *__restrict__ logits,
    int batch, long long T, int d, int m, int apply_rms, const float *__restrict__ gain, float eps,
    uint16_t *__restrict__ out, long long N, int G) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int dc = d / G, c_base = rank * dc;  // E * dc == 256
    const int nchunk = dc >> 3, RG = 256 / nchunk;
    extern __shared__ __align__(16) float smem[];
    float *w_full = smem;                      // [2m][dc]
    float *w_first = w_full + 2 * m * dc;      // [m][dc]
    float *red = w_first + m * dc;             // [RG][E][dc]
    float *part = red + (size_t)RG * E * dc;   // [2][E] partial sums of squares (double buffered)
    float *wsum = part + 2 * E;                // [8] warp partials
    pooling_weights(logits, d, m, c_base, dc, w_full, w_first);
    __syncthreads();

    const int chunk = threadIdx.x % nchunk, rg = threadIdx.x / nchunk;
    const int my_e = threadIdx.x / dc, my_c = threadIdx.x % dc;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long groups = (N + E - 1) / E;
    const long long items = (long long)batch * groups;
    const long long cid = blockIdx.x / G, ncl = gridDim.x / G;
    int round = 0;
    for (long long it = cid; it < items; it += ncl, ++round) {
        const long long b = it / groups, i0 = (it - b * groups) * E;
        const uint16_t *Ab = A + (size_t)b * T * d + c_base + chunk * 8;
        const uint16_t *Bb = B + (size_t)b * T * d + c_base + chunk * 8;
        float acc[E][8];
#pragma unroll
        for (int e = 0; e < E; ++e)
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[e][q] = 0.f;
        for (int r0 = rg; r0 < 2 * m; r0 += RG * NR) {
            // all loads of this batch first (rows past 2m or N, and entry 0's missing B half, read nothing)
            uint4 x[E][NR];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const long long i = i0 + e;
#pragma unroll
                for (int k = 0; k < NR; ++k) {
                    const int r = r0 + RG * k;
                    const uint16_t *src = nullptr;
                    if (i < N && r < 2 * m) {
                        if (r >= m)
                            src = Ab + (size_t)(i * m + r - m) * d;
                        else if (i > 0)
                            src = Bb + (size_t)((i - 1) * m + r) * d;
                    }
                    x[e][k] = src ? ldg_stream(src) : make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const long long i = i0 + e;
#pragma unroll
                for (int k = 0; k < NR; ++k) {
                    const int r = r0 + RG * k;
                    if (r >= 2 * m) continue;
                    if (i == 0) {
                        if (r >= m) fma8(acc[e], w_first + (size_t)(r - m) * dc + chunk * 8, x[e][k]);
                    } else {
                        fma8(acc[e], w_full + (size_t)r * dc + chunk * 8, x[e][k]);
                    }
                }
            }
        }
#pragma unroll
        for (int e = 0; e < E; ++e) {
            float4 *dst = reinterpret_cast<float4 *>(red + ((size_t)rg * E + e) * dc + chunk * 8);
            dst[0] = make_float4(acc[e][0], acc[e][1], acc[e][2], acc[e][3]);
            dst[1] = make_float4(acc[e][4], acc[e][5], acc[e][6], acc[e][7]);
        }
        __syncthreads();
        float v = 0.f;
        for (int g = 0; g < RG; ++g) v += red[((size_t)g * E + my_e) * dc + my_c];
        float rn = 1.f;
        if (apply_rms) {
            const int slot = round & 1;
            const float s = warp_sum(v * v);
            if (lane == 0) wsum[warp] = s;
            __syncthreads();
            if (threadIdx.x < E) {
                const int wpe = dc / 32;  // warps per entry
                float t = 0.f;
                for (int w8 = 0; w8 < wpe; ++w8) t += wsum[threadIdx.x * wpe + w8];
                part[slot * E + threadIdx.x] = t;
            }
            cluster.sync();
            float tot = 0.f;
            for (int g = 0; g < G; ++g) tot += cluster.map_shared_rank(part, g)[slot * E + my_e];
            rn = 1.0f / sqrtf(tot / (float)d + eps);
        }
        const long long i = i0 + my_e;
        if (i < N) {
            const float g = (apply_rms && gain) ? __ldg(gain + c_base + my_c) : 1.f;
            const __nv_bfloat16 o = __float2bfloat16_rn(v * rn * g);
            out[((size_t)b * N + i) * d + c_base + my_c] = *reinterpret_cast<const uint16_t *>(&o);
        }
        __syncthreads();  // red[] and wsum[] are rewritten by the next round
    }
    cluster.sync();  // no CTA leaves while a peer may still read its part[]
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
    // cluster path: channel slices of dc = d / G, G = min(8, d / 64), E = 256 / dc
    if (d % 64 != 0) return CSA_ERR_UNSUPPORTED;
    const int G = std::min(8, d / 64);
    const int dc = d / G;
    if (dc > 256 || 256 % dc != 0) return CSA_ERR_UNSUPPORTED;
    const int E = 256 / dc;
    const int RG = 256 / (dc / 8);
    const size_t smem = ((size_t)3 * m * dc + (size_t)RG * E * dc + 2 * E + 8) * sizeof(float);
    if (smem > 220 * 1024) return CSA_ERR_UNSUPPORTED;
    // loads in flight per thread: E entries x NR rows (32 registers of uint4 at most)
    const int rows_per_thread = (2 * m + RG - 1) / RG;
    int NR = 32 / E;
    while (NR > 1 && NR / 2 >= rows_per_thread) NR /= 2;
    void (*k)(const uint16_t *, const uint16_t *, const float *, int, long long, int, int, int, const float *,
              float, uint16_t *, long long, int) = nullptr;
#define CSA_CK(e_, nr_) \
    if (E == e_ && NR == nr_) k = compress_cluster_kernel<e_, nr_>;
    CSA_CK(4, 1) CSA_CK(4, 2) CSA_CK(4, 4) CSA_CK(4, 8)
    CSA_CK(2, 1) CSA_CK(2, 2) CSA_CK(2, 4) CSA_CK(2, 8) CSA_CK(2, 16)
    CSA_CK(1, 1) CSA_CK(1, 2) CSA_CK(1, 4) CSA_CK(1, 8) CSA_CK(1, 16) CSA_CK(1, 32)
#undef CSA_CK
    if (!k) return CSA_ERR_UNSUPPORTED;
    err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return CSA_ERR_CUDA;
    const long long items = (long long)batch * ((N + E - 1) / E);
    const long long nclusters = std::min<long long>(items, std::max(1, sms / G));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(nclusters * G));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, k, A, B, logits, batch, T, d, m, apply_rmsnorm, gain, eps, out, N, G);
    return err == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // namespace csa

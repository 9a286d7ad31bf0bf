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
//   * large m (HCA, m = 128): the 2m x d weights do not fit in shared memory;
//     a small kernel writes them once per call into a stream-ordered
//     allocation (a pool of the library that keeps its memory between calls),
//     and a thread per (entry, 8 channels) reads them through L1
//     (shared by the CTA's entries), one FMA per element with kStepRows rows'
//     loads in flight; an entry's channels stay in one CTA for the RMSNorm.
//     Entry 0 of each sequence (its A half only, other weights) runs the
//     input-dependent compressor with no Z rows, whose logits reduce to the
//     static ones.  That compressor alone (an online softmax per element)
//     measured 1.43 ms on the 1M-token cache; weights recomputed per CTA in
//     row chunks, 0.85 ms; a channel-split cluster 1.18 TB/s.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <mutex>

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

// ------------------------------------------------------------------ large m
constexpr int kTableThreads = 256;
constexpr int kStepRows = 6;  // rows whose loads are in flight together (64 registers: four CTAs per SM)

// Softmax weights of the 2m logits of every channel: w[j][c] (one warp per
// channel; the lanes' partial maxima and sums are combined in a fixed order).
__global__ void pool_weight_table_kernel(const float *__restrict__ logits, int d, int m, float *__restrict__ w) {
    const int c = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (c >= d) return;  // warp-uniform
    const float *L = logits + c;
    float mx = -INFINITY;
    for (int j = lane; j < 2 * m; j += 32) mx = fmaxf(mx, L[(size_t)j * d]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float den = 0.f;
    for (int j = lane; j < 2 * m; j += 32) den += expf(L[(size_t)j * d] - mx);
    den = warp_sum(den);
    for (int j = lane; j < 2 * m; j += 32) w[(size_t)j * d + c] = expf(L[(size_t)j * d] - mx) / den;
}

// Entries 1..N-1 of every sequence, one entry per tpe = d / 8 threads (whole
// warps), 256 / tpe entries per CTA; every element costs one FMA with its
// weight from the table (read through L1, shared by the CTA's entries).
__global__ void __launch_bounds__(kTableThreads, 4) compress_table_kernel(
    const uint16_t *__restrict__ A, const uint16_t *__restrict__ B, const float *__restrict__ w, int batch,
    long long T, int d, int m, int apply_rms, const float *__restrict__ gain, float eps,
    uint16_t *__restrict__ out, long long N) {
    __shared__ float red[kTableThreads / 32];
    const int tpe = d >> 3;
    const int el_n = kTableThreads / tpe;
    const int el = threadIdx.x / tpe;
    const int c0 = (threadIdx.x - el * tpe) * 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long per_seq = N - 1;
    const long long e = (long long)blockIdx.x * el_n + el;
    const bool act = e < (long long)batch * per_seq;
    const long long b = act ? e / per_seq : 0;
    const long long i = act ? 1 + (e - b * per_seq) : 1;
    const uint16_t *brow = B + ((size_t)b * T + (size_t)(i - 1) * m) * d + c0;  // previous block, stream B
    const uint16_t *arow = A + ((size_t)b * T + (size_t)i * m) * d + c0;        // this block, stream A
    const int two_m = 2 * m;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    if (act) {
        for (int r0 = 0; r0 < two_m; r0 += kStepRows) {
            uint4 xv[kStepRows];
#pragma unroll
            for (int u = 0; u < kStepRows; ++u) {
                const int r = r0 + u;
                xv[u] = make_uint4(0u, 0u, 0u, 0u);
                if (r < two_m) xv[u] = ldg_stream(r < m ? brow + (size_t)r * d : arow + (size_t)(r - m) * d);
            }
#pragma unroll
            for (int u = 0; u < kStepRows; ++u)
                if (r0 + u < two_m) {
                    const float *wr = w + (size_t)(r0 + u) * d + c0;
                    float wv[8];
                    const float4 w0 = __ldg(reinterpret_cast<const float4 *>(wr));
                    const float4 w1 = __ldg(reinterpret_cast<const float4 *>(wr + 4));
                    wv[0] = w0.x; wv[1] = w0.y; wv[2] = w0.z; wv[3] = w0.w;
                    wv[4] = w1.x; wv[5] = w1.y; wv[6] = w1.z; wv[7] = w1.w;
                    fma8(acc, wv, xv[u]);
                }
        }
    }
    // RMSNorm over the entry's d channels: its tpe threads are whole warps
    float rn = 1.f;
    if (apply_rms) {
        float ss = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) ss = fmaf(acc[q], acc[q], ss);
        ss = warp_sum(ss);
        if (lane == 0) red[warp] = ss;
        __syncthreads();
        const int w0 = el * (tpe >> 5);
        float t = 0.f;
        for (int k = 0; k < (tpe >> 5); ++k) t += red[w0 + k];
        rn = 1.0f / sqrtf(t / (float)d + eps);
    }
    if (act) {
        float o[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) o[q] = acc[q] * rn * ((apply_rms && gain) ? __ldg(gain + c0 + q) : 1.f);
        *reinterpret_cast<uint4 *>(out + ((size_t)b * N + i) * d + c0) = pack8(o);
    }
}

// Stream-ordered pool of the current device for the weight table: it keeps its
// memory between calls (release threshold at the maximum), so that a call does
// not map memory while its kernels are queued.
cudaMemPool_t table_pool() {
    static cudaMemPool_t cache[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return nullptr;
        uint64_t keep = UINT64_MAX;
        if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess) {
            cudaMemPoolDestroy(pool);
            return nullptr;
        }
        cache[dev] = pool;
    }
    return cache[dev];
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
    // large m.  Entry 0 of every sequence: the input-dependent compressor
    // without Z rows, the logits as its bias (read as float4: 16-byte aligned)
    if ((reinterpret_cast<uintptr_t>(logits) & 15) != 0) return CSA_ERR_UNSUPPORTED;
    const int tpe = d / 8;
    const bool tabled = (tpe == 32 || tpe == 64 || tpe == 128 || tpe == 256) && N > 1;
    float *table = nullptr;
    // a stream being captured into a graph takes the allocation-free path
    cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
    bool capturing = false;
    if (cudaStreamIsCapturing(st, &capture) != cudaSuccess) {
        cudaGetLastError();  // the query failed (e.g. the legacy stream during a capture): treat as capturing
        capturing = true;
    } else {
        capturing = capture != cudaStreamCaptureStatusNone;
    }
    cudaMemPool_t pool = (tabled && !capturing) ? table_pool() : nullptr;
    if (!pool || cudaMallocFromPoolAsync(reinterpret_cast<void **>(&table), (size_t)2 * m * d * sizeof(float), pool,
                                         st) != cudaSuccess) {
        cudaGetLastError();  // no table: the online-softmax kernel does every entry
        return launch_compress_dynamic(A, B, nullptr, nullptr, logits, batch, T, d, m, apply_rmsnorm, gain, eps, 0,
                                       N, N, out, st);
    }
    int rcode = launch_compress_dynamic(A, B, nullptr, nullptr, logits, batch, T, d, m, apply_rmsnorm, gain, eps, 0,
                                        1, N, out, st);
    if (rcode == CSA_OK) {
        pool_weight_table_kernel<<<(d + 3) / 4, 128, 0, st>>>(logits, d, m, table);
        const int el_n = kTableThreads / tpe;
        const long long blocks = ((long long)batch * (N - 1) + el_n - 1) / el_n;
        if (blocks > INT_MAX) rcode = CSA_ERR_UNSUPPORTED;
        else
            compress_table_kernel<<<(unsigned)blocks, kTableThreads, 0, st>>>(A, B, table, batch, T, d, m,
                                                                               apply_rmsnorm, gain, eps, out, N);
        if (rcode == CSA_OK && cudaGetLastError() != cudaSuccess) rcode = CSA_ERR_CUDA;
    }
    if (cudaFreeAsync(table, st) != cudaSuccess && rcode == CSA_OK) rcode = CSA_ERR_CUDA;
    return rcode;
}

}  // namespace csa

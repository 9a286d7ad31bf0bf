// compress_dynamic.cu -- compressed KV entries with input-dependent
// compression weights (csa_compress_dynamic).
//
// "DeepSeek v4", section "Compressed Sparse Attention" -> compressed
// Key-Value entry: per token the hidden states give two KV rows (streams A and
// B) and two compression-weight rows Z_a, Z_b.  Entry i pools, per channel c,
// the m B rows of the previous block and the m A rows of its own block under a
// softmax over the 2m logits Z[row][c] + bias[j][c] (entry 0 has no previous
// block: the A half only), then an optional RMSNorm over its d channels.
// Entries [i0, i0 + ni) of every sequence are computed and written to rows i
// of out[b][n_out][d], so one call builds a whole cache or appends the newest
// entry at decode time.
//
// The weights differ per entry and channel, so unlike csa_compress nothing is
// precomputed: a thread owns 8 channels of one entry and runs an online softmax
// over the 2m rows in fp32 (running maximum, rescaled denominator and
// accumulator, in log2 units).  Every stream row is read once, so the op
// streams 4*T*d*2 bytes (A, B, Z_a, Z_b) plus the T/m*d*2 written: it is HBM
// bound.  The loads of kRows rows are issued before the first is used.  The
// RMSNorm sum of squares is reduced in a fixed order (warp shuffles, then the
// entry's warps in shared memory; or the entry's threads in shared memory when
// d/8 is not a multiple of 32), so results do not depend on scheduling.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kRows = 4;                         // rows whose loads are in flight together (three CTAs per SM)
constexpr int kMaxThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;

__global__ void __launch_bounds__(kMaxThreads, 3) compress_dynamic_kernel(
    const uint16_t *__restrict__ A, const uint16_t *__restrict__ B, const uint16_t *__restrict__ Za,
    const uint16_t *__restrict__ Zb, const float *__restrict__ bias, int batch, long long T, int d, int m,
    int apply_rms, const float *__restrict__ gain, float eps, long long i0, long long ni, long long n_out,
    uint16_t *__restrict__ out) {
    __shared__ float red[kMaxThreads];
    const int tpe = d >> 3;                       // threads per entry, 8 channels each
    const int epb = blockDim.x / tpe;             // entries per block (blockDim = epb * tpe)
    const int le = threadIdx.x / tpe;
    const int c0 = (threadIdx.x - le * tpe) * 8;
    const long long e = (long long)blockIdx.x * epb + le;  // (sequence, entry) pair
    const bool active = e < (long long)batch * ni;

    float mx[8], den[8], acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        mx[q] = -INFINITY;
        den[q] = 0.f;
        acc[q] = 0.f;
    }
    long long b = 0, i = 0;
    if (active) {
        b = e / ni;
        i = i0 + (e - b * ni);
        const size_t seq = (size_t)b * T * d + c0;
        for (int r0 = i == 0 ? m : 0; r0 < 2 * m; r0 += kRows) {
            uint4 zv[kRows], xv[kRows];
#pragma unroll
            for (int k = 0; k < kRows; ++k) {
                const int r = r0 + k;
                zv[k] = make_uint4(0u, 0u, 0u, 0u);
                xv[k] = zv[k];
                if (r < 2 * m) {
                    const bool prev = r < m;  // B row of the previous block, else A row of this block
                    const size_t off = seq + (size_t)(prev ? (i - 1) * m + r : i * m + (r - m)) * d;
                    const uint16_t *z = prev ? Zb : Za;
                    xv[k] = ldg_stream((prev ? B : A) + off);
                    if (z) zv[k] = ldg_stream(z + off);
                }
            }
#pragma unroll
            for (int k = 0; k < kRows; ++k) {
                const int r = r0 + k;
                if (r < 2 * m) {
                    float zf[8], xf[8];
                    unpack8(zv[k], zf);
                    unpack8(xv[k], xf);
                    const float4 b0 = __ldg(reinterpret_cast<const float4 *>(bias + (size_t)r * d + c0));
                    const float4 b1 = __ldg(reinterpret_cast<const float4 *>(bias + (size_t)r * d + c0 + 4));
                    const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float l = (zf[q] + bb[q]) * kLog2e;
                        if (l > mx[q]) {  // new maximum: rescale what has been summed so far
                            const float s = exp2f(mx[q] - l);
                            den[q] *= s;
                            acc[q] *= s;
                            mx[q] = l;
                        }
                        const float w = l == -INFINITY ? 0.f : exp2f(l - mx[q]);
                        den[q] += w;
                        acc[q] = fmaf(w, xf[q], acc[q]);
                    }
                }
            }
        }
    }

    float y[8];
    float ss = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        y[q] = den[q] > 0.f ? acc[q] / den[q] : 0.f;
        ss = fmaf(y[q], y[q], ss);
    }
    if (apply_rms) {  // uniform over the grid: every thread reaches the barrier
        float tot = 0.f;
        if ((tpe & 31) == 0) {
            ss = warp_sum(ss);
            if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
            __syncthreads();
            const int wpe = tpe >> 5;
            for (int w = 0; w < wpe; ++w) tot += red[le * wpe + w];
        } else {
            red[threadIdx.x] = ss;
            __syncthreads();
            for (int t = 0; t < tpe; ++t) tot += red[le * tpe + t];
        }
        const float rn = 1.0f / sqrtf(tot / (float)d + eps);
#pragma unroll
        for (int q = 0; q < 8; ++q) y[q] *= rn * (gain ? __ldg(gain + c0 + q) : 1.f);
    }
    if (active) *reinterpret_cast<uint4 *>(out + ((size_t)b * n_out + i) * d + c0) = pack8(y);
}

}  // namespace

int launch_compress_dynamic(const uint16_t *A, const uint16_t *B, const uint16_t *Za, const uint16_t *Zb,
                            const float *bias, int batch, long long T, int d, int m, int apply_rmsnorm,
                            const float *gain, float eps, long long i0, long long ni, long long n_out,
                            uint16_t *out, cudaStream_t st) {
    if (ni == 0) return CSA_OK;
    const int tpe = d / 8;
    if (tpe < 1 || tpe > kMaxThreads) return CSA_ERR_UNSUPPORTED;
    const int epb = std::max(1, kMaxThreads / tpe);
    const long long blocks = ((long long)batch * ni + epb - 1) / epb;
    if (blocks > INT_MAX) return CSA_ERR_UNSUPPORTED;
    compress_dynamic_kernel<<<(unsigned)blocks, epb * tpe, 0, st>>>(A, B, Za, Zb, bias, batch, T, d, m,
                                                                    apply_rmsnorm, gain, eps, i0, ni, n_out, out);
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // namespace csa

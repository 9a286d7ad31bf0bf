// quant_fp8.cu -- FP8 KV-cache quantisation (csa_quantize_fp8_kv).
//
// "DeepSeek-V4-Pro - Model techniques map", list "inference quantization":
// the KV cache is quantised to FP8.  The pages give no format; the one used
// here: e4m3 codes with one power-of-two scale per 128 channels of a row,
// stored as a UE8M0 byte e (s = 2^(e - 127)); s is the smallest power of two
// with absmax / s <= 448 (the largest finite e4m3 magnitude), its exponent k
// kept in [-124, 119] so that every code times s is a finite bf16 number; the
// codes are round-to-nearest-even with saturation, a zero magnitude stored as
// +0, and an all-zero block has e = 127.
//
// A thread owns 8 consecutive elements; the 16 threads of a 128-element block
// are 16 consecutive lanes and reduce its absmax with shuffles.  The op reads
// 2 bytes and writes 1 + 1/128 bytes per element: HBM bound.
#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kThreads = 256;

// two floats -> two e4m3 codes (lo in the low byte), RNE, saturating
CSA_DEVINL uint32_t e4m3x2_rn_sat(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// a code of -0 (0x80) becomes +0
CSA_DEVINL uint32_t plus_zero(uint32_t w) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (((w >> (8 * i)) & 0xffu) == 0x80u) w &= ~(0xffu << (8 * i));
    return w;
}

__global__ void __launch_bounds__(kThreads) quantize_fp8_kv_kernel(const uint16_t *__restrict__ x, long long n8,
                                                                   uint8_t *__restrict__ codes,
                                                                   uint8_t *__restrict__ exps) {
    const long long t = (long long)blockIdx.x * kThreads + threadIdx.x;  // unit of 8 elements
    const bool active = t < n8;  // n8 is a multiple of 16: a block's 16 lanes agree
    float f[8];
    if (active) {
        unpack8(ldg_stream(x + t * 8), f);
    } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) f[q] = 0.f;
    }
    float amax = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) amax = fmaxf(amax, fabsf(f[q]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    // smallest k with amax <= 448 * 2^k = 1.75 * 2^(8 + k), from amax's bit fields
    int k = 0;
    if (amax > 0.f) {
        const uint32_t bits = __float_as_uint(amax);
        const int ef = (int)((bits >> 23) & 0xffu);
        if (ef == 0) {
            k = -124;  // subnormal absmax: far below the floor
        } else {
            const int E = ef - 127;
            k = (bits & 0x7fffffu) <= 0x600000u ? E - 8 : E - 7;  // mantissa <= 1.75 or above
        }
        k = k < -124 ? -124 : (k > 119 ? 119 : k);
    }
    const float inv = __uint_as_float((uint32_t)(127 - k) << 23);  // 2^-k, exact
    const uint32_t w0 = plus_zero(e4m3x2_rn_sat(f[0] * inv, f[1] * inv) | (e4m3x2_rn_sat(f[2] * inv, f[3] * inv) << 16));
    const uint32_t w1 = plus_zero(e4m3x2_rn_sat(f[4] * inv, f[5] * inv) | (e4m3x2_rn_sat(f[6] * inv, f[7] * inv) << 16));
    if (active) {
        *reinterpret_cast<uint2 *>(codes + t * 8) = make_uint2(w0, w1);
        if ((t & 15) == 0) exps[t >> 4] = (uint8_t)(k + 127);
    }
}

}  // namespace

int launch_quantize_fp8_kv(const uint16_t *x, long long rows, int d, uint8_t *codes, uint8_t *exps,
                           cudaStream_t st) {
    const long long n8 = rows * (d / 8);
    if (n8 == 0) return CSA_OK;
    const long long blocks = (n8 + kThreads - 1) / kThreads;
    if (blocks > 0x7fffffffLL) return CSA_ERR_UNSUPPORTED;
    quantize_fp8_kv_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(x, n8, codes, exps);
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // namespace csa

// quant_fp4.cu -- FP4 activations for the indexer QK path (csa_quantize_fp4).
//
// e2m1 elements with one e4m3 scale per 16-element block ("DeepSeek V4 paper
// full version is out, FP4 QAT details and stability tricks [D]": FP4
// activations in the CSA indexer QK path; techniques map "FP4 precision for
// the attention indexer").  Per block:
//   s = e4m3_RNE_satfinite(absmax / 6)            (IEEE fp32 division)
//   q_j = e2m1_RNE_satfinite(x_j / s), or 0 for the whole block when s == 0;
//   a code whose magnitude is 0 is stored as +0.
// Both conversions use the sm_100a cvt.rn.satfinite instructions.  One thread
// per block: 32 B of bf16 in, 8 B of codes + 1 B of scale out (HBM bound).
#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

CSA_DEVINL uint32_t cvt_e4m3(float s) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(s));
    return r & 0xffu;
}

// value of an e4m3 code as fp32 (exact); code 0x7F/0xFF never produced (satfinite)
CSA_DEVINL float e4m3_value(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, mt = c & 7u;
    const float v = e == 0u ? (float)mt * 0.001953125f /* 2^-9 */
                            : __uint_as_float(((e + 120u) << 23) | (mt << 20));
    return (c & 0x80u) ? -v : v;
}

// 8 fp32 -> 8 e2m1 codes packed in a u32 (element 2j low nibble of byte j)
CSA_DEVINL uint32_t cvt_e2m1x8(const float v[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    // store signed zeros as +0: keep a nibble's sign bit only if its magnitude is non-zero
    const uint32_t nz = (out | (out >> 1) | (out >> 2)) & 0x11111111u;
    return out & (0x77777777u | (nz << 3));
}

__global__ void __launch_bounds__(256) quantize_fp4_kernel(const uint16_t *__restrict__ x, long long nblocks,
                                                           uint8_t *__restrict__ packed,
                                                           uint8_t *__restrict__ scales) {
    for (long long blk = (long long)blockIdx.x * blockDim.x + threadIdx.x; blk < nblocks;
         blk += (long long)gridDim.x * blockDim.x) {
        const uint4 v0 = ldg_stream(x + blk * 16);
        const uint4 v1 = ldg_stream(x + blk * 16 + 8);
        float f[16];
        unpack8(v0, f);
        unpack8(v1, f + 8);
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(f[j]));
        const uint32_t sc = cvt_e4m3(__fdiv_rn(amax, 6.0f));
        const float s = e4m3_value(sc);
        uint2 codes = make_uint2(0u, 0u);
        if (s != 0.f) {
            float q[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) q[j] = __fdiv_rn(f[j], s);
            codes.x = cvt_e2m1x8(q);
            codes.y = cvt_e2m1x8(q + 8);
        }
        *reinterpret_cast<uint2 *>(packed + blk * 8) = codes;
        scales[blk] = (uint8_t)sc;
    }
}

}  // namespace

int launch_quantize_fp4(const uint16_t *x, long long rows, int d, uint8_t *packed, uint8_t *scales,
                        cudaStream_t st) {
    const long long nblocks = rows * (d / 16);
    if (nblocks == 0) return CSA_OK;
    const long long want = (nblocks + 255) / 256;
    const int grid = (int)(want < 148LL * 16 ? want : 148LL * 16);
    quantize_fp4_kernel<<<grid, 256, 0, st>>>(x, nblocks, packed, scales);
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // namespace csa

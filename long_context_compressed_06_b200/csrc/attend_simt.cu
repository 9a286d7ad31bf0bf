// attend_simt.cu -- CSA / HCA core attention on CUDA cores (csa_attend,
// hca_attend for shapes the tensor-core kernel does not take), and the
// split-KV combine shared by every attention kernel.
//
// One KV head (K = V) shared by H RMSNorm'd query heads; key set = selected
// compressed entries (CSA) or every visible entry (HCA), plus the sliding
// window of raw stream-A rows (techniques map rows "Grouped-query attention",
// "Sliding-window attention", "QK normalization"; "DeepSeek v4" hybrid
// attention section for HCA).
//
// Grid: (head groups of 16, key splits, queries).  A warp owns two heads;
// each lane holds D/32 consecutive dims of q_hat and of the running output.
// Per key: two warp-reduced dot products, an online-softmax update in fp32.
// Splits write unnormalised partial outputs + (max, sum) to the workspace and
// attend_combine merges them in split order (a fixed, deterministic order).
#include <algorithm>

#include "attend_common.cuh"
#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kHeadsPerCta = 16;

template <int DPL>
CSA_DEVINL void load_lane_dims(const uint16_t *row, int lane, float x[DPL]) {
    const uint16_t *p = row + lane * DPL;
    if constexpr (DPL == 16) {
        unpack8(ldg16(p), x);
        unpack8(ldg16(p + 8), x + 8);
    } else if constexpr (DPL == 8) {
        unpack8(ldg16(p), x);
    } else if constexpr (DPL == 4) {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
        x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x); x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
    } else {
        const uint32_t v = __ldg(reinterpret_cast<const uint32_t *>(p));
        x[0] = bf16_lo(v); x[1] = bf16_hi(v);
    }
}

template <int DPL>
__global__ void __launch_bounds__(256) attend_simt_kernel(AttendArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long bq = blockIdx.z;
    const long long b = bq / a.nq;
    const int split = blockIdx.y;
    const int D = DPL * 32;
    const long long t = a.q_pos[bq];
    const KeySet ks = key_set(a, b, bq, t);
    const long long e0 = (long long)split * a.keys_per_split;
    const long long e1 = std::min(ks.total, e0 + a.keys_per_split);

    // q_hat for this warp's two heads, pre-scaled by scale * log2(e)
    float q[2][DPL];
    int head[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        head[hh] = blockIdx.x * kHeadsPerCta + warp * 2 + hh;
        const int h = head[hh] < a.H ? head[hh] : a.H - 1;
        load_lane_dims<DPL>(a.q + ((size_t)bq * a.H + h) * D, lane, q[hh]);
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) ss = fmaf(q[hh][i], q[hh][i], ss);
        ss = warp_sum(ss);
        const float r = (1.0f / sqrtf(ss / (float)D + a.eps)) * a.scale * 1.4426950408889634f;
#pragma unroll
        for (int i = 0; i < DPL; ++i)
            q[hh][i] *= r * (a.q_gain ? __ldg(a.q_gain + lane * DPL + i) : 1.f);
    }

    float mrun[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    float o[2][DPL];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[hh][i] = 0.f;

    for (long long e = e0; e < e1; ++e) {
        const uint16_t *row = key_row(a, ks, b, bq, e);
        if (!row) continue;
        float x[DPL];
        load_lane_dims<DPL>(row, lane, x);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < DPL; ++i) s = fmaf(q[hh][i], x[i], s);
            s = warp_sum(s);
            const float mn = fmaxf(mrun[hh], s);
            const float alpha = exp2f(mrun[hh] - mn);
            const float p = exp2f(s - mn);
            l[hh] = l[hh] * alpha + p;
#pragma unroll
            for (int i = 0; i < DPL; ++i) o[hh][i] = fmaf(p, x[i], o[hh][i] * alpha);
            mrun[hh] = mn;
        }
    }

#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int h = head[hh];
        if (h >= a.H) continue;
        if (a.splits == 1) {
            // the head's sink logit joins the denominator (natural units -> log2 units)
            const float L = l[hh] + (a.sinks ? exp2f(__ldg(a.sinks + h) * 1.4426950408889634f - mrun[hh]) : 0.f);
            const float inv = L > 0.f ? 1.0f / L : 0.f;
            float f[DPL];
#pragma unroll
            for (int i = 0; i < DPL; ++i) f[i] = o[hh][i] * inv;
            store_lane_dims<DPL>(a.out + ((size_t)bq * a.H + h) * D, lane, f);
        } else {
            float *po = a.part_o + (((size_t)split * a.n_bq + bq) * a.H + h) * D + lane * DPL;
            if constexpr (DPL == 2) {
                *reinterpret_cast<float2 *>(po) = make_float2(o[hh][0], o[hh][1]);
            } else {
#pragma unroll
                for (int i = 0; i < DPL; i += 4)
                    *reinterpret_cast<float4 *>(po + i) =
                        make_float4(o[hh][i], o[hh][i + 1], o[hh][i + 2], o[hh][i + 3]);
            }
            if (lane == 0)
                a.part_ml[((size_t)split * a.n_bq + bq) * a.H + h] = make_float2(mrun[hh], l[hh]);
        }
    }
}

}  // namespace

// Split count: enough CTAs to cover the SMs a few times, at least 32 keys per split.
int attend_simt_splits(long long n_bq, int H, long long max_keys) {
    const long long base = n_bq * ((H + kHeadsPerCta - 1) / kHeadsPerCta);
    const long long target = 148LL * 4;
    long long s = (target + base - 1) / base;
    s = std::max(1LL, std::min(s, (max_keys + 31) / 32));
    return (int)std::min(s, 64LL);
}

int launch_attend_simt(const AttendArgs &a, cudaStream_t st) {
    dim3 grid((unsigned)((a.H + kHeadsPerCta - 1) / kHeadsPerCta), (unsigned)a.splits, (unsigned)a.n_bq);
    switch (a.D) {
        case 64: attend_simt_kernel<2><<<grid, 256, 0, st>>>(a); break;
        case 128: attend_simt_kernel<4><<<grid, 256, 0, st>>>(a); break;
        case 256: attend_simt_kernel<8><<<grid, 256, 0, st>>>(a); break;
        case 512: attend_simt_kernel<16><<<grid, 256, 0, st>>>(a); break;
        default: return CSA_ERR_UNSUPPORTED;
    }
    if (cudaGetLastError() != cudaSuccess) return CSA_ERR_CUDA;
    return a.splits > 1 ? launch_attend_combine(a, st) : CSA_OK;
}

}  // namespace csa

// attend_common.cuh -- argument block, key-set enumeration and split-KV
// workspace layout shared by the attention kernels.
#pragma once

#include "common.cuh"

namespace csa {

// Partial RoPE: the trailing kRopeDim channels of every head rotate in the
// rotate-half form (channel n+i with n+kRopeDim/2+i, n = D - kRopeDim): the
// normalised query at its position before the dot products, the output by the
// conjugate rotation at the same position; keys arrive already rotated.
constexpr int kRopeDim = 64;

struct AttendArgs {
    const uint16_t *q;      // [n_bq][H][D]
    const float *q_gain;    // [D] or null
    const float *sinks;     // [H] per-head sink logits (natural units) or null
    const float *rope_cos;  // [rope_npos][kRopeDim / 2] partial-RoPE tables, or null (no RoPE)
    const float *rope_sin;  // [rope_npos][kRopeDim / 2]
    long long rope_npos;
    const uint16_t *kv;     // [batch][N][D]
    // FP8 KV cache (instead of kv / win when kv8 is set): e4m3 codes and one
    // UE8M0 exponent byte per 128 channels, value = code * 2^(e - 127)
    const uint8_t *kv8, *kv8e;    // [batch][N][D], [batch][N][D/128]
    const uint8_t *win8, *win8e;  // [batch][win_rows][D], [batch][win_rows][D/128]
    long long N;
    int m;                  // compression ratio (dense key set only)
    const int *idx;         // [n_bq][k] selected entries (CSA); unused when dense
    int k;
    bool dense;             // HCA: every visible entry is a key
    const uint16_t *win;    // [batch][win_rows][D] stream-A rows of positions win_pos0..
    long long win_pos0, win_rows;
    int W;
    const int *q_pos;       // [n_bq]
    int nq;
    long long n_bq;         // batch * nq
    int H, D;
    float scale, eps;
    uint16_t *out;          // [n_bq][H][D]
    float *part_o;          // [splits][n_bq][H][D] unnormalised partial outputs
    float2 *part_ml;        // [splits][n_bq][H] (running max in log2 units, sum)
    int splits;
    long long keys_per_split;
};

// (cos, sin) of rotated pair i (< kRopeDim / 2) at position t; (1, 0) -- no
// rotation -- when RoPE is off or t lies outside the tables.
CSA_DEVINL float2 rope_cs(const AttendArgs &a, long long t, int i) {
    if (!a.rope_cos || t < 0 || t >= a.rope_npos) return make_float2(1.f, 0.f);
    const size_t o = (size_t)t * (kRopeDim / 2) + i;
    return make_float2(__ldg(a.rope_cos + o), __ldg(a.rope_sin + o));
}

// The key set J of one query is enumerated as e = 0 .. total-1: first the
// nsel selected (CSA: idx slots, HCA: entries 0..n_vis-1), then the window
// positions u0 .. u0 + nwin - 1 of stream A held by the window buffer.
struct KeySet {
    long long nsel, u0, total;
};

CSA_DEVINL KeySet key_set(const AttendArgs &a, long long /*b*/, long long /*bq*/, long long t) {
    KeySet ks;
    ks.nsel = a.dense ? n_visible(t, a.m, a.N) : a.k;
    long long u0 = t - a.W + 1;
    u0 = u0 < 0 ? 0 : u0;
    ks.u0 = u0 < a.win_pos0 ? a.win_pos0 : u0;
    const long long last = a.win_pos0 + a.win_rows - 1;
    const long long u1 = t < last ? t : last;
    const long long nwin = u1 >= ks.u0 ? u1 - ks.u0 + 1 : 0;
    ks.total = ks.nsel + nwin;
    return ks;
}

// Row of key e, or null for an invalid selection slot (-1 or out of range).
CSA_DEVINL const uint16_t *key_row(const AttendArgs &a, const KeySet &ks, long long b, long long bq,
                                   long long e) {
    if (e < ks.nsel) {
        const long long j = a.dense ? e : (long long)__ldg(a.idx + bq * a.k + e);
        if (j < 0 || j >= a.N) return nullptr;
        return a.kv + ((size_t)b * a.N + j) * a.D;
    }
    return a.win + ((size_t)b * a.win_rows + (ks.u0 - a.win_pos0) + (e - ks.nsel)) * a.D;
}

template <int DPL>
CSA_DEVINL void store_lane_dims(uint16_t *row, int lane, const float f[DPL]) {
    uint16_t *p = row + lane * DPL;
    if constexpr (DPL >= 8) {
#pragma unroll
        for (int i = 0; i < DPL; i += 8) *reinterpret_cast<uint4 *>(p + i) = pack8(f + i);
    } else if constexpr (DPL == 4) {
        *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
    } else {
        *reinterpret_cast<uint32_t *>(p) = pack_bf16x2(f[0], f[1]);
    }
}

int launch_attend_combine(const AttendArgs &a, cudaStream_t st);

}  // namespace csa

// attend_common.cuh -- argument block and split-KV workspace layout shared by
// the attention kernel and the split combine.
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
    uint16_t *part_o;       // [splits][n_bq][H][D] bf16 partial outputs, each divided by its own sum
    int part_perm;          // part_o rows of one (split, query) in warp-store order (see attend_combine)
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

int launch_attend_combine(const AttendArgs &a, cudaStream_t st);

}  // namespace csa

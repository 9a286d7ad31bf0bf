// attend.cu -- csa_attend / hca_attend dispatch, workspace sizing and the
// split-KV combine.
//
// The combine merges the partial results of the key splits of one (query,
// head) with the usual log-sum-exp rule, always in split order, so the output
// does not depend on scheduling (the pages' inference stack relies on
// batch-invariant, deterministic split reductions; techniques map
// "Separate split-K outputs with deterministic reduction").
#include <algorithm>

#include "attend_common.cuh"
#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

// One thread per 8 output columns of one head: the splits' (max, sum) first,
// then their bf16 rows in split order, 8 splits' loads in flight at a time.
//   out = sum_s 2^(m_s - M) l_s O_s / (sum_s 2^(m_s - M) l_s + sink)
// with O_s the split's row already divided by its own sum l_s.
//
// Partial layout.  Standard: [H][D] per (split, query).  Warp-store order
// (part_perm, H % 64 == 0): the attention's softmax warp of lane quarter sp
// holds 16 heads x 64 columns of each 64-column slab, a thread 8 columns per
// store; it stores them as one contiguous 2 KiB block per warp and slab (16-byte
// piece j*32 + lane, lane = head%16 + 16 * (column half)), so that every store
// instruction writes whole sectors.  Piece P of a (split, query) region then
// holds head hh*64 + sp*16 + (lane & 15), columns slab*64 + (lane >> 4)*32 + j*8
// with (hh*slabs + slab, sp, j, lane) = P's digits (slabs = D/64); the merge
// takes one piece per thread, so its loads of the partials are coalesced.
constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads) attend_combine_kernel(AttendArgs a) {
    const int tph = a.D / 8;                              // threads per head
    const long long bq = blockIdx.x;
    int h, c0;
    long long piece;  // 16-byte piece of the (split, query) region this thread merges
    if (a.part_perm) {
        const int P = blockIdx.y * kCombineThreads + threadIdx.x;
        const int ln = P & 31, j = (P >> 5) & 3, sp = (P >> 7) & 3, rest = P >> 9, slabs = a.D / 64;
        h = (rest / slabs) * 64 + sp * 16 + (ln & 15);
        c0 = (rest % slabs) * 64 + (ln >> 4) * 32 + j * 8;
        piece = P;
    } else {
        h = blockIdx.y * (kCombineThreads / tph) + threadIdx.x / tph;
        c0 = (threadIdx.x % tph) * 8;
        piece = (long long)h * tph + c0 / 8;
    }
    const bool active = h < a.H;  // no early exit: the RoPE shuffles need whole warps
    // launched as a programmatic dependent of the attention kernel: its partials
    // are complete only once that grid is
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const size_t stride = (size_t)a.n_bq * a.H;          // between splits, in rows
    const size_t row = (size_t)bq * a.H + (active ? h : 0);
    float M = -INFINITY;
    float L = 0.f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const uint16_t *src0 = a.part_o + (size_t)bq * a.H * a.D + (size_t)(active ? piece : 0) * 8;
    if (a.splits <= 16) {
        // every split's (max, sum) and row issued before any is used: one L2 round
        // trip instead of two (same arithmetic, same order as below)
        float2 ml[16];
        uint4 v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < a.splits) {
                ml[j] = a.part_ml[j * stride + row];
                v[j] = *reinterpret_cast<const uint4 *>(src0 + (size_t)j * stride * a.D);
            }
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < a.splits) M = fmaxf(M, ml[j].x);
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < a.splits) {
                const float wl = ml[j].x == -INFINITY ? 0.f : exp2f(ml[j].x - M) * ml[j].y;
                L += wl;
                float f[8];
                unpack8(v[j], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(wl, f[e], acc[e]);
            }
    }
    if (a.splits > 16)
        for (int s = 0; s < a.splits; ++s) M = fmaxf(M, a.part_ml[s * stride + row].x);
    for (int s0 = 0; a.splits > 16 && s0 < a.splits; s0 += 8) {
        const int ns = a.splits - s0 < 8 ? a.splits - s0 : 8;
        float2 ml[8];
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < ns) {
                ml[j] = a.part_ml[(s0 + j) * stride + row];
                v[j] = *reinterpret_cast<const uint4 *>(
                    a.part_o + ((s0 + j) * stride + (size_t)bq * a.H) * a.D + (size_t)(active ? piece : 0) * 8);
            }
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < ns) {
                const float wl = ml[j].x == -INFINITY ? 0.f : exp2f(ml[j].x - M) * ml[j].y;
                L += wl;
                float f[8];
                unpack8(v[j], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(wl, f[e], acc[e]);
            }
    }
    // the head's sink logit (natural units; the partials are in log2 units)
    if (a.sinks && active) L += exp2f(__ldg(a.sinks + h) * 1.4426950408889634f - M);
    const float inv = L > 0.f ? 1.0f / L : 0.f;
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = acc[e] * inv;
    if (a.rope_cos) {
        // conjugate rotation of the trailing kRopeDim channels: channel D-64+j pairs
        // with D-32+j, held by the thread 4 lanes away (32 channels; 16 lanes in
        // the warp-store order)
        float pv[8];
        const int pl = a.part_perm ? 16 : 4;
#pragma unroll
        for (int e = 0; e < 8; ++e) pv[e] = __shfl_xor_sync(0xffffffffu, o[e], pl);
        if (c0 >= a.D - kRopeDim) {
            const long long t = __ldg(a.q_pos + bq);
            const bool first = c0 < a.D - kRopeDim / 2;
            const int i0 = (c0 - (a.D - kRopeDim)) & (kRopeDim / 2 - 1);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float2 cs = rope_cs(a, t, i0 + e);
                o[e] = first ? o[e] * cs.x + pv[e] * cs.y : o[e] * cs.x - pv[e] * cs.y;
            }
        }
    }
    if (active) *reinterpret_cast<uint4 *>(a.out + row * a.D + c0) = pack8(o);  // row = bq * H + h
}

// [splits][n_bq][H][D] bf16 rows, then [splits][n_bq][H] float2 (max, sum)
size_t ws_bytes_for(long long n_bq, int H, int D, int splits) {
    if (splits <= 1) return 0;
    return (size_t)splits * n_bq * H * ((size_t)D * sizeof(uint16_t) + sizeof(float2));
}

}  // namespace

int launch_attend_combine(const AttendArgs &a, cudaStream_t st) {
    const int hpb = kCombineThreads / (a.D / 8);  // heads per block (D in {64, ..., 512})
    // a programmatic dependent of the attention kernel just launched on st (which
    // lets it launch once every attention CTA has started): the combine CTAs are
    // resident and waiting when the last partial lands
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.n_bq, (unsigned)((a.H + hpb - 1) / hpb));
    cfg.blockDim = dim3(kCombineThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attend_combine_kernel, a) == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

bool attend_tc_supported(int H, int D);
void attend_tc_plan(long long n_bq, int H, long long max_keys, int *splits, long long *kps);
int launch_attend_tc(AttendArgs a, const DevCtx &ctx, cudaStream_t st, bool pdl);

// Split plan of the tensor-core kernel for these shapes (one split when the
// shapes are outside the compiled tiles: the launch then returns
// CSA_ERR_UNSUPPORTED before using any workspace).
static void plan_splits(long long n_bq, int H, int D, long long max_keys, int *splits, long long *kps) {
    if (attend_tc_supported(H, D)) {
        attend_tc_plan(n_bq, H, max_keys, splits, kps);
    } else {
        *splits = 1;
        *kps = max_keys;
    }
}

size_t attend_workspace_bytes(int batch, int nq, int H, int D, long long max_keys) {
    const long long n_bq = (long long)batch * nq;
    int splits;
    long long kps;
    plan_splits(n_bq, H, D, max_keys, &splits, &kps);
    return ws_bytes_for(n_bq, H, D, splits);
}

int launch_attend(const uint16_t *q, const float *q_gain, const float *sinks, const float *rope_cos,
                  const float *rope_sin, long long rope_npos, const Fp8Kv *fp8, const uint16_t *kv, long long N, int m,
                  const int *idx, int k, bool dense, const uint16_t *win, long long win_pos0, long long win_rows,
                  int W, const int *q_pos,
                  int batch, int nq, int H, int D, float scale, float eps, uint16_t *out, void *ws,
                  size_t ws_bytes, const DevCtx &ctx, cudaStream_t st, bool pdl) {
    AttendArgs a = {};
    a.q = q; a.q_gain = q_gain; a.sinks = sinks; a.rope_cos = rope_cos; a.rope_sin = rope_sin;
    a.rope_npos = rope_npos; a.kv = kv;
    if (fp8) {
        a.kv8 = fp8->kv; a.kv8e = fp8->kv_exp; a.win8 = fp8->win; a.win8e = fp8->win_exp;
    } a.N = N; a.m = m; a.idx = idx; a.k = k; a.dense = dense;
    a.win = win; a.win_pos0 = win_pos0; a.win_rows = win_rows; a.W = W; a.q_pos = q_pos; a.nq = nq; a.n_bq = (long long)batch * nq;
    a.H = H; a.D = D; a.scale = scale; a.eps = eps; a.out = out;
    if (a.n_bq == 0) return CSA_OK;
    if (!attend_tc_supported(H, D)) return CSA_ERR_UNSUPPORTED;
    const long long max_keys = (dense ? N : (long long)k) + W;
    plan_splits(a.n_bq, H, D, max_keys, &a.splits, &a.keys_per_split);
    const size_t need = ws_bytes_for(a.n_bq, H, D, a.splits);
    if (need > 0) {
        if (!ws || ws_bytes < need) return CSA_ERR_WORKSPACE;
        a.part_o = reinterpret_cast<uint16_t *>(ws);
        a.part_perm = H % 64 == 0 ? 1 : 0;
        a.part_ml = reinterpret_cast<float2 *>(reinterpret_cast<char *>(ws) +
                                               (size_t)a.splits * a.n_bq * H * D * sizeof(uint16_t));
    }
    return launch_attend_tc(a, ctx, st, pdl);
}

}  // namespace csa

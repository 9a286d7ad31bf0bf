// index_tc.cu -- lightning-indexer scores on the 5th-generation tensor cores.
//
//   S[q][s] = sum_h w[q][h] * max(0, q_I[q][h] . K_I[s])   (s < n_vis(t_q), else -inf)
// ("DeepSeek v4" -> "sparse selection Lightning Indexer").
//
// GEMM view per sequence: D[s][(q,h)] = K_I[s] . q_I[q][h], M = 128 keys per
// tile, N = NQ queries x H_pad heads (<= 256), K = d_I.  The keys are the
// streamed operand (A); the NQ queries' heads (B) stay in shared memory while
// the CTA walks key tiles.  Each TMEM lane holds one key, so the epilogue
// sum_h w_h * ReLU(.) is a loop over columns inside one thread, and a warp
// stores 32 consecutive scores.
//
// Warp roles:  warp 0 -- TMA producer (key tiles into a STAGES ring, query
// tile once per query group); warp 1 -- TMEM owner and MMA issuer (lane 0
// issues; tcgen05.mma kind::f16, fp32 accumulate, four accumulator buffers when
// N <= 128, else two); then two epilogue groups of EW warps taking alternate
// tiles (tcgen05.ld, ReLU, weighted head sum, causal mask, store).  Every
// mbarrier wait is bounded (csa_sync_status reports a timeout).  Decode (one
// query per tile) streams the key cache from HBM: EW = 4, one warp per TMEM
// lane quarter.  Prefill is bound by the epilogue (64 FMAs per key per query)
// rather than the tensor cores: with four queries per tile one warp's pass
// over 256 accumulator columns took longer than the MMAs of two tiles, so
// EW = 8 splits the queries between two warps of the same lanes (1.69 ->
// 1.35 ms on the 4096-query prefill); at decode the extra warps cost ~1 us.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int kTileKeys = 128;
constexpr int kMaxStages = 6;
constexpr int kMaxAcc = 4;   // TMEM accumulators (two when N = NQ x H_pad > 128)

struct IndexTcParams {
    const float *w;       // [batch][nq][H_I]
    const int *q_pos;     // [batch][nq]
    float *scores;        // [batch][nq][N]
    long long N;
    int nq, H_I, H_pad, d_I, m, NQ;
    int groups_per_batch, n_ktiles;
    long long total_work;
    int stages, nchunk, chunk_elems, row_bytes, layout;
    uint32_t stage_bytes, q_bytes, idesc;
    int n_cols;           // N of the MMA = NQ * H_pad
    int n_acc;            // TMEM accumulators (2 or 4)
    uint32_t tmem_cols;   // allocated columns (n_acc accumulators)
    int split;            // MMA-issuing warps (2: each issues half of the N columns)
    uint32_t idesc_half;  // instruction descriptor of N = n_cols / 2
    DevCtx ctx;
};

// Position in a CTA's work range (sequence b, query group g, key tile kt),
// advanced without divisions.
struct Cursor {
    long long w;
    int kt, g, b;
};

CSA_DEVINL Cursor cursor_at(const IndexTcParams &p, long long w) {
    Cursor c;
    c.w = w;
    const long long grp = w / p.n_ktiles;
    c.kt = (int)(w - grp * p.n_ktiles);
    c.b = (int)(grp / p.groups_per_batch);
    c.g = (int)(grp - (long long)c.b * p.groups_per_batch);
    return c;
}

CSA_DEVINL void advance(const IndexTcParams &p, Cursor &c) {
    ++c.w;
    if (++c.kt == p.n_ktiles) {
        c.kt = 0;
        if (++c.g == p.groups_per_batch) {
            c.g = 0;
            ++c.b;
        }
    }
}

// Named barrier of one epilogue group of EW warps.
template <int EW>
CSA_DEVINL void group_bar(int eg) {
    asm volatile("bar.sync %0, %1;" ::"r"(eg + 1), "n"(EW * 32) : "memory");
}

// Slot and phase of a ring of n barriers.
struct Ring {
    int idx = 0;
    uint32_t phase = 0;
    CSA_DEVINL void next(int n) {
        if (++idx == n) {
            idx = 0;
            phase ^= 1u;
        }
    }
};

// Threads: producer and MMA warps, two epilogue groups of EW warps, and with
// EW = 8 (several queries per tile) a second MMA-issuing warp.
constexpr int index_threads(int EW) { return 64 + 64 * EW + (EW == 8 ? 32 : 0); }

template <int EW, int OCC>  // warps per epilogue group (4: one per TMEM lane quarter, 8: two); CTAs per SM
__global__ void __launch_bounds__(index_threads(EW), OCC)
    index_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                    const IndexTcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned carve-up: key stages | query tile | weights | barriers
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *k_smem = base;
    uint8_t *q_smem = k_smem + (size_t)p.stages * p.stage_bytes;
    float *w_s = reinterpret_cast<float *>(q_smem + p.q_bytes);          // [2 groups][NQ][H_pad]
    int *nvis_s = reinterpret_cast<int *>(w_s + 2 * p.NQ * p.H_pad);     // [2 groups][NQ]
    uint64_t *bars = reinterpret_cast<uint64_t *>(
        (reinterpret_cast<uintptr_t>(nvis_s + 2 * p.NQ) + 7) & ~uintptr_t(7));
    uint64_t *full = bars, *empty = bars + kMaxStages;
    uint64_t *tfull = bars + 2 * kMaxStages, *tempty = tfull + kMaxAcc;
    uint64_t *qfull = tempty + kMaxAcc, *qempty = qfull + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(qempty + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    // a successor launched as a programmatic dependent (csa_decode_step's top-k)
    // may start now; it waits for this grid before reading the scores
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long w0 = (long long)blockIdx.x * p.total_work / gridDim.x;
    const long long w1 = (long long)(blockIdx.x + 1) * p.total_work / gridDim.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, p.split);  // one commit per MMA issuer
        }
        for (int a = 0; a < p.n_acc; ++a) {
            mbar_init(tfull + a, p.split);
            mbar_init(tempty + a, EW);
        }
        mbar_init(qfull, 1);
        mbar_init(qempty, p.split);
        *abort_flag = 0;
        fence_mbar_init();
        tc::prefetch_tmap(&kmap);
        tc::prefetch_tmap(&qmap);
    }
    if (warp == 1) {
        tc::tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    // The single-thread roles keep their whole warp in the loop: every lane
    // polls the barriers (votes keep the warp converged) and lane 0 issues
    // through guarded instructions, never a branch.
    const auto wait_all = [&](uint64_t *bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), parity, p.ctx, abort_flag));
    };
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        long long it = 0, gi = 0;
        Ring kr;
        for (Cursor cu = cursor_at(p, w0); cu.w < w1; advance(p, cu)) {
            if (cu.w == w0 || cu.kt == 0) {
                if (!wait_all(qempty, (uint32_t)((gi & 1) ^ 1))) break;
                mbar_arrive_expect_tx(smem_u32(qfull), p.q_bytes, lane == 0);
                for (int c = 0; c < p.nchunk; ++c)
                    tc::tma_load_4d(smem_u32(q_smem + (size_t)c * p.n_cols * p.row_bytes), &qmap, smem_u32(qfull),
                                    c * p.chunk_elems, 0, cu.g * p.NQ, cu.b, lane == 0);
                ++gi;
            }
            const int st = kr.idx;
            if (!wait_all(empty + st, kr.phase ^ 1u)) break;
            mbar_arrive_expect_tx(smem_u32(full + st), p.stage_bytes, lane == 0);
            uint8_t *dst = k_smem + (size_t)st * p.stage_bytes;
            for (int c = 0; c < p.nchunk; ++c)
                tc::tma_load_3d(smem_u32(dst + (size_t)c * kTileKeys * p.row_bytes), &kmap, smem_u32(full + st),
                                c * p.chunk_elems, cu.kt * kTileKeys, cu.b, lane == 0);
            kr.next(p.stages);
            ++it;
        }
        // drain: wait (bounded) for the copies this warp issued last into each stage
        for (long long j = std::max(0LL, it - p.stages); j < it; ++j)
            mbar_wait(smem_u32(full + (j % p.stages)), (uint32_t)((j / p.stages) & 1), p.ctx, nullptr);
        if (gi > 0) mbar_wait(smem_u32(qfull), (uint32_t)((gi - 1) & 1), p.ctx, nullptr);
        __syncwarp();
    } else if (warp == 1 || (EW == 8 && p.split == 2 && warp == 2 + 2 * EW)) {
        // ------------------------------------------------------------ MMA issuers
        // With several queries per tile two warps issue, each the N / 2 columns
        // of its half of the query heads (a thread issues a tcgen05.mma only
        // every ~100-160 cycles, which held the tensor pipe to ~37 % at N = 256);
        // both wait on the same barriers and commit to the ones the tile releases.
        const int half = (p.split == 2 && warp != 1) ? 1 : 0;
        const int ncol = p.n_cols / p.split;
        const uint32_t idesc = p.split == 2 ? p.idesc_half : p.idesc;
        long long gi = 0;
        Ring kr, ar;
        const uint32_t sbo = 8u * p.row_bytes;
        // descriptors built once, advanced by constant offsets (16-byte units)
        const uint64_t kdesc0 = tc::smem_desc(smem_u32(k_smem), sbo, p.layout);
        const uint64_t qdesc0 = tc::smem_desc(smem_u32(q_smem), sbo, p.layout);
        const bool issuer = lane == 0;
        for (Cursor cu = cursor_at(p, w0); cu.w < w1; advance(p, cu)) {
            if (cu.w == w0 || cu.kt == 0) {
                if (!wait_all(qfull, (uint32_t)(gi & 1))) break;
                ++gi;
            }
            const int acc = ar.idx;
            if (!wait_all(tempty + acc, ar.phase ^ 1u)) break;
            const int st = kr.idx;
            if (!wait_all(full + st, kr.phase)) break;
            tc::fence_after_sync();
            const uint32_t d_tmem = tmem_base + (uint32_t)(acc * p.n_cols + half * ncol);
            const uint64_t kd = kdesc0 + ((uint64_t)(st * p.stage_bytes) >> 4);
            uint32_t accumulate = 0;
            for (int c = 0; c < p.nchunk; ++c) {
                for (int kk = 0; kk < p.chunk_elems / 16; ++kk) {
                    tc::mma_f16(d_tmem, kd + ((uint32_t)(c * kTileKeys * p.row_bytes + kk * 32) >> 4),
                                qdesc0 + ((uint32_t)((c * p.n_cols + half * ncol) * p.row_bytes + kk * 32) >> 4), idesc,
                                accumulate,
                                issuer);
                    accumulate = 1;
                }
            }
            tc::mma_commit(smem_u32(empty + st), issuer);
            tc::mma_commit(smem_u32(tfull + acc), issuer);
            if (cu.w == w1 - 1 || cu.kt == p.n_ktiles - 1) tc::mma_commit(smem_u32(qempty), issuer);
            kr.next(p.stages);
            ar.next(p.n_acc);
        }
    } else if (warp >= 2 && warp < 2 + 2 * EW) {
        // ------------------------------------------------------------ epilogue
        // Two groups of EW warps take alternate tiles (tile i -> group i & 1,
        // accumulator i % n_acc), doubling the epilogue rate; with EW = 8 the two
        // warps of a lane quarter take the even and the odd queries of a tile.
        constexpr int kLoads = (EW == 4 && OCC == 1) ? 4 : 2;  // 16-column TMEM loads per wait (registers)
        const int eg = (warp - 2) / EW;
        const int half = ((warp - 2) % EW) >> 2;
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int row = quarter * 32 + lane;
        const int et = (threadIdx.x - 64) % (EW * 32);
        float *ws_g = w_s + eg * p.NQ * p.H_pad;
        int *nv_g = nvis_s + eg * p.NQ;
        int loaded_b = -1, loaded_g = -1;
        for (Cursor cu = cursor_at(p, w0); cu.w < w1; advance(p, cu)) {
            const int li = (int)(cu.w - w0);
            if ((li & 1) != eg) continue;
            const int b = cu.b, g = cu.g;
            if (b != loaded_b || g != loaded_g) {
                group_bar<EW>(eg);
                for (int i = et; i < p.NQ * p.H_pad; i += EW * 32) {
                    const int qi = i / p.H_pad, h = i - qi * p.H_pad;
                    const int q = g * p.NQ + qi;
                    ws_g[i] = (q < p.nq && h < p.H_I) ? __ldg(p.w + ((size_t)b * p.nq + q) * p.H_I + h) : 0.f;
                }
                for (int qi = et; qi < p.NQ; qi += EW * 32) {
                    const int q = g * p.NQ + qi;
                    nv_g[qi] = q < p.nq ? (int)n_visible(__ldg(p.q_pos + (size_t)b * p.nq + q), p.m, p.N) : 0;
                }
                group_bar<EW>(eg);
                loaded_b = b;
                loaded_g = g;
            }
            const int acc = li & (p.n_acc - 1);
            const uint32_t aph = (uint32_t)((li / p.n_acc) & 1);
            // every lane polls and the warp votes (tcgen05.ld below is warp-collective;
            // a single polling lane leaves the warp's following code much slower)
            const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(tfull + acc), aph, p.ctx, abort_flag));
            if (!ok) break;
            tc::fence_after_sync();
            const long long s = (long long)cu.kt * kTileKeys + row;
            const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * p.n_cols);
            for (int qi = half; qi < p.NQ; qi += EW / 4) {
                const int q = g * p.NQ + qi;
                if (q >= p.nq) break;
                // independent partial sums (one per 16-column load) keep the FMA
                // chains short
                float part[kLoads];
#pragma unroll
                for (int u = 0; u < kLoads; ++u) part[u] = 0.f;
                for (int hc = 0; hc < p.H_pad; hc += 16 * kLoads) {
                    float v[16 * kLoads];
                    const int nl = min(kLoads, (p.H_pad - hc) >> 4);
#pragma unroll
                    for (int u = 0; u < kLoads; ++u)
                        if (u < nl) tc::tmem_ld16(tbase + (uint32_t)(qi * p.H_pad + hc + 16 * u), v + 16 * u);
                    tc::tmem_wait_ld();
                    const float *ws = ws_g + qi * p.H_pad + hc;
#pragma unroll
                    for (int u = 0; u < kLoads; ++u)
                        if (u < nl) {
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                part[u] = fmaf(ws[16 * u + i], fmaxf(v[16 * u + i], 0.f), part[u]);
                        }
                }
                float score = 0.f;
#pragma unroll
                for (int u = 0; u < kLoads; ++u) score += part[u];
                if (s < p.N) p.scores[((size_t)b * p.nq + q) * p.N + s] = s < nv_g[qi] ? score : -INFINITY;
            }
            tc::fence_before_sync();
            __syncwarp();
            mbar_arrive(smem_u32(tempty + acc), lane == 0);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem_base, p.tmem_cols);
    }
}

}  // namespace

// The tensor-core path takes d_I in {32, 64, 128, 256} and up to 256 heads,
// as long as one query's heads and two key stages fit in shared memory.
bool index_tc_supported(int H_I, int d_I) {
    if (!(d_I == 32 || d_I == 64 || d_I == 128 || d_I == 256) || H_I < 1 || H_I > 256) return false;
    const size_t h_pad = (size_t)std::max(16, (H_I + 15) / 16 * 16);
    return h_pad * d_I * 2 + 2 * (size_t)kTileKeys * d_I * 2 <= 200 * 1024;
}

int launch_index_tc(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, const int *q_pos, int batch,
                    int nq, long long N, int H_I, int d_I, int m, float *scores, const DevCtx &ctx,
                    cudaStream_t st) {
    IndexTcParams p = {};
    p.w = w; p.q_pos = q_pos; p.scores = scores; p.N = N; p.nq = nq; p.H_I = H_I; p.d_I = d_I; p.m = m;
    p.ctx = ctx;
    p.H_pad = std::max(16, (H_I + 15) / 16 * 16);
    p.chunk_elems = d_I >= 64 ? 64 : d_I;           // one swizzle row of bf16
    p.row_bytes = p.chunk_elems * 2;
    p.layout = p.row_bytes == 128 ? tc::kLayoutSw128 : tc::kLayoutSw64;
    p.nchunk = d_I / p.chunk_elems;
    p.stage_bytes = (uint32_t)(kTileKeys * d_I * 2);
    // queries per tile: as many as fit in N <= 256 and in shared memory
    const size_t smem_cap = 200 * 1024;
    int NQ = std::max(1, std::min(nq, std::min(16, 256 / p.H_pad)));
    while (NQ > 1 && (size_t)NQ * p.H_pad * d_I * 2 + 2 * p.stage_bytes > smem_cap) NQ /= 2;
    p.NQ = NQ;
    p.n_cols = NQ * p.H_pad;
    p.q_bytes = (uint32_t)(p.n_cols * d_I * 2);
    // One query per tile (decode): two CTAs per SM, two stages each -- finer work
    // ranges and two independent pipelines per SM even out the CTAs' finishing
    // times (decode 128K: 21.0 -> 18.6 us).
    const bool two_per_sm = NQ == 1 && (size_t)p.q_bytes + 2 * (size_t)p.stage_bytes + 4096 <= 108 * 1024;
    const size_t cta_cap = two_per_sm ? 108 * 1024 : smem_cap;
    p.stages = (int)std::min<size_t>(kMaxStages, (cta_cap - p.q_bytes) / p.stage_bytes);
    if (p.stages < 2) return CSA_ERR_UNSUPPORTED;
    p.idesc = tc::idesc_f16(p.n_cols, true);
    p.n_acc = p.n_cols <= 128 ? 4 : 2;
    uint32_t cols = 32;
    while (cols < (uint32_t)(p.n_acc * p.n_cols)) cols *= 2;
    p.tmem_cols = cols;
    p.groups_per_batch = (nq + NQ - 1) / NQ;
    p.n_ktiles = (int)((N + kTileKeys - 1) / kTileKeys);
    p.total_work = (long long)batch * p.groups_per_batch * p.n_ktiles;

    const CUtensorMapSwizzle sw = p.row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap kmap, qmap;
    {
        const uint64_t dims[3] = {(uint64_t)d_I, (uint64_t)N, (uint64_t)batch};
        const uint64_t strides[2] = {(uint64_t)d_I * 2, (uint64_t)N * d_I * 2};
        const uint32_t box[3] = {(uint32_t)p.chunk_elems, (uint32_t)kTileKeys, 1};
        if (!encode_tensor_map(&kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k_idx, dims, strides, box, sw))
            return CSA_ERR_CUDA;
    }
    {
        const uint64_t dims[4] = {(uint64_t)d_I, (uint64_t)H_I, (uint64_t)nq, (uint64_t)batch};
        const uint64_t strides[3] = {(uint64_t)d_I * 2, (uint64_t)H_I * d_I * 2, (uint64_t)nq * H_I * d_I * 2};
        const uint32_t box[4] = {(uint32_t)p.chunk_elems, (uint32_t)p.H_pad, (uint32_t)NQ, 1};
        if (!encode_tensor_map(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, q_idx, dims, strides, box, sw))
            return CSA_ERR_CUDA;
    }
    const size_t smem = 1024 + (size_t)p.stages * p.stage_bytes + p.q_bytes + 2 * ((size_t)NQ * p.H_pad * 4 + NQ * 4) +
                        8 + (2 * kMaxStages + 2 * kMaxAcc + 2) * 8 + 16;
    // several queries per tile: two warps per TMEM lane quarter split them
    const int EW = NQ >= 2 ? 8 : 4;
    // two MMA issuers when each half of N is a valid MMA width starting on an
    // 8-row swizzle atom of the query tile
    p.split = (EW == 8 && (p.n_cols / 2) % 16 == 0) ? 2 : 1;
    p.idesc_half = tc::idesc_f16(std::max(16, p.n_cols / 2), true);
    void (*kern)(const CUtensorMap, const CUtensorMap, const IndexTcParams) =
        EW == 8 ? index_tc_kernel<8, 1> : (two_per_sm ? index_tc_kernel<4, 2> : index_tc_kernel<4, 1>);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return CSA_ERR_CUDA;
    const int grid = (int)std::min<long long>(p.total_work, (two_per_sm ? 2 : 1) * num_sms());
    kern<<<grid, index_threads(EW), smem, st>>>(kmap, qmap, p);
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // namespace csa

// index_fp4_bs.cu -- FP4 lightning-indexer scores on block-scaled FP4 tensor-core MMAs.
//
//   S[q][s] = sum_h w[q][h] * max(0, q_I[q][h] . K_I[s])   (s < n_vis(t_q), else -inf)
// with q_I and K_I stored as e2m1 codes and one e4m3 scale per 16 elements
// ("DeepSeek V4 paper full version is out, FP4 QAT details" -- FP4 activations
// in the indexer QK path; techniques map, "inference quantization").
//
// tcgen05.mma kind::mxf4nvf4 (scale_vec::4X) multiplies the packed e2m1 codes
// directly and applies one e4m3 (unsigned) scale factor of A and one of B per
// 16-element block, accumulating in fp32: every product is exact, so the
// scores differ from the exact FP4 dot products only by the summation order.
// The keys stream from HBM as they are stored, 64 code bytes per key at
// d_I = 128, plus 8 scale bytes.
//
// GEMM view per sequence: D[s][(q,h)] = sum_k A[s][k] B[(q,h)][k] with A = a
// 128-key sub-tile (M = 128, K-major packed rows of d_I/2 bytes), B = the query
// group's heads (N = NQ x H_pad <= 128 rows), K = d_I in steps of 64.  A tile
// (one TMA box, one ring stage) holds two sub-tiles when their accumulators fit
// three tiles deep in tensor memory, else one.  The
// scale factors live in tensor memory, a block of 4 columns per K step (byte j
// of a 32-bit cell scales 16-element block j of the step): the key scales of
// each tile in a ring of slots, key row m at lane m, column m / 32 of the
// block; the query-head scales once per query group, head row n at lane
// n % 32, column n / 32 of the block, copied into each of the four lane
// quarters (the rows of A in a quarter read B's scale factors there).
//
// Warp roles (736 threads): warp 0 -- TMA producer (key tiles into a ring of
// stages, the query group's codes once per group); warp 1 -- TMEM owner and
// MMA issuer of sub-tile 0, warp 22 -- MMA issuer of sub-tile 1 (lane 0 issues
// through guarded instructions; one thread issues a tcgen05.mma only every
// ~100 cycles, two threads twice as fast); warps 2..5 -- scale
// movers (each thread stages its key row's scale bytes with cp.async several
// tiles ahead and writes them into the tile's tensor-memory slot; the
// query-head scales once per group); warps 6..21 -- four epilogue groups of
// four warps (a tile's two sub-tiles to a pair of groups, the pairs taking
// the tiles in turn; one-sub-tile tiles: one group per accumulator)
// (tcgen05.ld, ReLU, weighted head sum, causal mask, store).  Every wait is
// bounded and every role warp stays converged.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int kEpiGroups = 4;  // epilogue groups of four warps, taking tiles in turn
constexpr int kMma2Warp = 6 + 4 * kEpiGroups;  // the second MMA issuer (sub-tile 1)
constexpr int kThreads = 192 + 128 * kEpiGroups + 32;
constexpr int kSubKeys = 128;   // keys of one MMA (M); a tile holds p.sub of them
constexpr int kMaxStages = 20;
constexpr int kMaxAcc = 4;
constexpr int kSfSlots = 4;     // key-scale slots in tensor memory (tiles in flight)
constexpr int kSfAhead = 8;     // tiles whose key scales a mover thread prefetches

struct Fp4BsParams {
    const uint8_t *k4s;   // [batch][N][d_I/16] key scales (e4m3, non-negative)
    const uint8_t *q4s;   // [batch][nq][H_I][d_I/16]
    const float *w;       // [batch][nq][H_I]
    const int *q_pos;     // [batch][nq]
    float *scores;        // [batch][nq][N]
    long long N;
    int nq, H_I, H_pad, d_I, m, NQ;
    int groups_per_batch, n_ktiles;
    long long total_work;
    int stages, kb, nks;  // ring depth, scale bytes per row (d_I/16), MMA K steps (d_I/64)
    int sub, tile_keys;   // M = 128 sub-tiles per tile (1 or 2) and keys per tile
    uint32_t sub_desc;    // start-address step of the second sub-tile in a smem descriptor
    uint32_t stage_bytes, q_bytes, idesc, sbo, layout;
    int n_cols, n_acc;
    uint32_t tmem_cols, sfa_col, sfb_col;
    DevCtx ctx;
};

struct Cursor {
    long long w;
    int kt, g, b;
};

CSA_DEVINL Cursor cursor_at(const Fp4BsParams &p, long long w) {
    Cursor c;
    c.w = w;
    const long long grp = w / p.n_ktiles;
    c.kt = (int)(w - grp * p.n_ktiles);
    c.b = (int)(grp / p.groups_per_batch);
    c.g = (int)(grp - (long long)c.b * p.groups_per_batch);
    return c;
}

CSA_DEVINL void advance(const Fp4BsParams &p, Cursor &c) {
    ++c.w;
    if (++c.kt == p.n_ktiles) {
        c.kt = 0;
        if (++c.g == p.groups_per_batch) {
            c.g = 0;
            ++c.b;
        }
    }
}

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

// Named barrier of one epilogue group (128 threads), ids 1..kEpiGroups.
CSA_DEVINL void group_bar(int eg) { asm volatile("bar.sync %0, 128;" ::"r"(eg + 1) : "memory"); }

// Block-scaled FP4 MMA: D (+)= A . B^T with per-16-element scale factors of A
// and B read from tensor memory at sfa / sfb.
CSA_DEVINL void mma_fp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t sfa,
                        uint32_t sfb, uint32_t accumulate, bool pred) {
    asm volatile(
        "{\n\t.reg .pred p, g;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "setp.ne.b32 g, %7, 0;\n\t"
        "@g tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate), "r"((int)pred)
        : "memory");
}

// One 32-bit tensor-memory cell per lane of this warp (column taddr).
CSA_DEVINL void tmem_st1(uint32_t taddr, uint32_t v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v) : "memory");
}

// The scale bytes of one row (KB = d_I/16 bytes, NKS = KB/4 columns).
template <int KB>
CSA_DEVINL void cp_async_row(uint32_t dst, const uint8_t *src, bool valid) {
    // src-size 0 fills the destination with zeros (rows past N)
    const uint32_t n = valid ? KB : 0;
    if constexpr (KB == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;" ::"r"(dst), "l"(src), "n"(KB), "r"(n) : "memory");
}

// Query-head scales of group g of sequence b for head rows n = 32 gq + lane:
// v[gq][j] = the j-th 32-bit word of row n's scale bytes (zero past the heads).
template <int NKS>
CSA_DEVINL void load_qscales(const Fp4BsParams &p, int b, int g, int lane, uint32_t (&v)[4][NKS]) {
    constexpr int KB = 4 * NKS;
#pragma unroll
    for (int gq = 0; gq < 4; ++gq) {
        const int n = 32 * gq + lane;
#pragma unroll
        for (int j = 0; j < NKS; ++j) v[gq][j] = 0u;
        if (n < p.n_cols) {
            const int qi = n / p.H_pad, h = n - qi * p.H_pad, q = g * p.NQ + qi;
            if (q < p.nq && h < p.H_I) {
                const uint8_t *src = p.q4s + (((size_t)b * p.nq + q) * p.H_I + h) * KB;
#pragma unroll
                for (int j = 0; j < NKS; ++j) v[gq][j] = __ldg(reinterpret_cast<const uint32_t *>(src) + j);
            }
        }
    }
}

template <int KB>
__global__ void __launch_bounds__(kThreads, 1)
    index_fp4_bs_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                        const Fp4BsParams p) {
    constexpr int NKS = KB / 4;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned carve-up: key stages | query tile | key-scale staging | weights | barriers
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *k_smem = base;
    uint8_t *q_smem = k_smem + (size_t)p.stages * p.stage_bytes;
    uint8_t *sf_smem = q_smem + ((p.q_bytes + 1023u) & ~1023u);            // [kSfAhead][tile rows][KB]
    float *w_s = reinterpret_cast<float *>(sf_smem + kSfAhead * p.tile_keys * KB);  // [groups][NQ][H_pad]
    int *nvis_s = reinterpret_cast<int *>(w_s + kEpiGroups * p.NQ * p.H_pad);     // [groups][NQ]
    uint64_t *bars = reinterpret_cast<uint64_t *>(
        (reinterpret_cast<uintptr_t>(nvis_s + kEpiGroups * p.NQ) + 7) & ~uintptr_t(7));
    uint64_t *full = bars, *empty = bars + kMaxStages;
    uint64_t *tfull = empty + kMaxStages, *tempty = tfull + kMaxAcc;
    uint64_t *sfull = tempty + kMaxAcc, *sempty = sfull + kSfSlots;       // key-scale slots
    uint64_t *qfull = sempty + kSfSlots, *qempty = qfull + 1;             // query codes (TMA)
    uint64_t *qsfull = qempty + 1, *qsempty = qsfull + 1;                 // query-head scales
    uint64_t *sfld = qsempty + 1;                                         // key-scale staging slots
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sfld + kSfAhead);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long w0 = (long long)blockIdx.x * p.total_work / gridDim.x;
    const long long w1 = (long long)(blockIdx.x + 1) * p.total_work / gridDim.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, p.sub);  // one commit per MMA issuer
        }
        for (int a = 0; a < p.n_acc; ++a) {
            mbar_init(tfull + a, p.sub);
            mbar_init(tempty + a, p.sub == 2 ? 8 : 4);  // the warps of the groups that read it
        }
        for (int s = 0; s < kSfSlots; ++s) {
            mbar_init(sfull + s, 4);
            mbar_init(sempty + s, p.sub);
        }
        mbar_init(qfull, 1);
        mbar_init(qempty, p.sub);
        mbar_init(qsfull, 4);
        mbar_init(qsempty, p.sub);
        for (int s = 0; s < kSfAhead; ++s) mbar_init(sfld + s, 128);  // one cp.async arrival per mover thread
        *abort_flag = 0;
        fence_mbar_init();
        tc::prefetch_tmap(&kmap);
        tc::prefetch_tmap(&qmap);
    }
    if (warp == 1) {
        tc::tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
        tc::tmem_relinquish();
    }
    // Scale movers (warps 2..5): thread r owns row r of every sub-tile and query-head
    // row r of every group.  The first kSfAhead tiles' key scales and the first
    // group's query-head scales are requested before the setup barrier, i.e.
    // before the producer fills its ring: issued after it, they waited behind the
    // ring's key tiles in the memory queues and the first MMA came ~6.8 us after
    // entry.  (The copies' barrier arrivals follow the barrier initialisation.)
    const int mv_r = (warp & 3) * 32 + lane;
    const uint32_t mv_row = smem_u32(sf_smem + mv_r * KB);
    const auto prefetch_copies = [&](const Cursor &c, long long i) {
        for (int h = 0; h < p.sub; ++h) {
            const long long key = (long long)c.kt * p.tile_keys + h * kSubKeys + mv_r;
            const bool valid = key < p.N;
            cp_async_row<KB>(mv_row + (uint32_t)(((i % kSfAhead) * p.tile_keys + h * kSubKeys) * KB),
                             p.k4s + ((size_t)c.b * p.N + (valid ? key : 0)) * KB, valid);
        }
    };
    uint32_t q_first[4][NKS];
    if (warp >= 2 && warp < 6 && w0 < w1) {
        Cursor pf0 = cursor_at(p, w0);
        load_qscales<NKS>(p, pf0.b, pf0.g, lane, q_first);
        for (int i = 0; i < kSfAhead && pf0.w < w1; ++i, advance(p, pf0)) prefetch_copies(pf0, i);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
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
                tc::tma_load_4d(smem_u32(q_smem), &qmap, smem_u32(qfull), 0, 0, cu.g * p.NQ, cu.b, lane == 0);
                ++gi;
            }
            const int st = kr.idx;
            if (!wait_all(empty + st, kr.phase ^ 1u)) break;
            mbar_arrive_expect_tx(smem_u32(full + st), p.stage_bytes, lane == 0);
            tc::tma_load_3d(smem_u32(k_smem + (size_t)st * p.stage_bytes), &kmap, smem_u32(full + st), 0,
                            cu.kt * p.tile_keys, cu.b, lane == 0);
            kr.next(p.stages);
            ++it;
        }
        // drain: wait (bounded) for the copies this warp issued last into each stage
        for (long long j = std::max(0LL, it - p.stages); j < it; ++j)
            mbar_wait(smem_u32(full + (j % p.stages)), (uint32_t)((j / p.stages) & 1), p.ctx, nullptr);
        if (gi > 0) mbar_wait(smem_u32(qfull), (uint32_t)((gi - 1) & 1), p.ctx, nullptr);
        __syncwarp();
    } else if (warp == 1 || (warp == kMma2Warp && p.sub == 2)) {
        // ------------------------------------------------------------ MMA issuers
        // One warp per sub-tile (warp 1: sub-tile 0, the last warp: sub-tile 1):
        // a single thread issues a tcgen05.mma every ~100 cycles at best
        // (measured), so the two sub-tiles' independent accumulators are fed
        // by two issuing threads.  Both wait on the same barriers and each
        // commits to the ones the tile releases (counts of two).
        const int h = warp == 1 ? 0 : 1;
        long long gi = 0;
        Ring kr, ar, sr;
        const uint64_t kdesc0 = tc::smem_desc(smem_u32(k_smem), p.sbo, p.layout);
        const uint64_t qdesc0 = tc::smem_desc(smem_u32(q_smem), p.sbo, p.layout);
        const bool issuer = lane == 0;
        for (Cursor cu = cursor_at(p, w0); cu.w < w1; advance(p, cu)) {
            if (cu.w == w0 || cu.kt == 0) {
                if (!wait_all(qfull, (uint32_t)(gi & 1))) break;
                if (!wait_all(qsfull, (uint32_t)(gi & 1))) break;
                ++gi;
            }
            const int acc = ar.idx;
            if (!wait_all(tempty + acc, ar.phase ^ 1u)) break;
            const int st = kr.idx;
            if (!wait_all(full + st, kr.phase)) break;
            const int sl = sr.idx;
            if (!wait_all(sfull + sl, sr.phase)) break;
            tc::fence_after_sync();
            const uint64_t kd = kdesc0 + ((uint64_t)(st * p.stage_bytes) >> 4);
            {
                // sub-tile h: keys 128h.. of the tile into its own accumulator
                const uint32_t d_tmem = tmem_base + (uint32_t)((acc * p.sub + h) * p.n_cols);
                for (int ks = 0; ks < NKS; ++ks)
                    // K step ks: 64 codes = 32 bytes into each swizzled row; its scale
                    // factors in the 4-column blocks of the sub-tile's slot and of the group
                    mma_fp4(d_tmem, kd + (uint64_t)(h * p.sub_desc + ks * 2), qdesc0 + (uint64_t)(ks * 2), p.idesc,
                            tmem_base + p.sfa_col + (uint32_t)(4 * ((sl * p.sub + h) * NKS + ks)),
                            tmem_base + p.sfb_col + (uint32_t)(4 * ks), ks > 0 ? 1u : 0u, issuer);
            }
            tc::mma_commit(smem_u32(empty + st), issuer);
            tc::mma_commit(smem_u32(sempty + sl), issuer);
            tc::mma_commit(smem_u32(tfull + acc), issuer);
            if (cu.w == w1 - 1 || cu.kt == p.n_ktiles - 1) {
                tc::mma_commit(smem_u32(qempty), issuer);
                tc::mma_commit(smem_u32(qsempty), issuer);
            }
            kr.next(p.stages);
            ar.next(p.n_acc);
            sr.next(kSfSlots);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ scale movers (warps 2..5)
        // Thread r (0..127) owns row r of every sub-tile (the keys r and 128 + r of
        // a two-sub-tile tile) and query-head row r of every group.  Its key-scale bytes are staged with
        // cp.async kSfAhead tiles ahead, each staging slot completed by an mbarrier
        // that counts the movers' cp.async arrivals: issued only a few tiles ahead,
        // these small loads wait behind the deep ring of key-tile copies in the
        // memory queues and set the pace.  A thread reads and refills only its own
        // row of a slot, so a slot needs no barrier between the movers.
        const int sub = warp & 3;  // tensor-memory lanes this warp may access
        const int r = mv_r;
        const uint32_t lane_off = (uint32_t)(sub * 32) << 16;
        const auto prefetch = [&](const Cursor &c, long long i) {
            if (c.w < w1) {
                prefetch_copies(c, i);
                asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];"
                             ::"r"(smem_u32(sfld + (int)(i % kSfAhead))) : "memory");
            }
        };
        // the arrivals of the copies issued before the setup barrier (each tracks
        // all of this thread's copies so far)
        Cursor pf = cursor_at(p, w0);
        for (int i = 0; i < kSfAhead; ++i) {
            if (pf.w < w1) {
                asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];"
                             ::"r"(smem_u32(sfld + i)) : "memory");
                advance(p, pf);
            }
        }
        long long gi = 0, i = 0;
        Ring sr;
        for (Cursor cu = cursor_at(p, w0); cu.w < w1; advance(p, cu), ++i) {
            if (cu.w == w0 || cu.kt == 0) {
                // query-head scales of this group: head row n = qi * H_pad + h sits at
                // lane n % 32, column n / 32 of each K step's block, in every
                // sub-partition (the rows of A in sub-partition s read B's scale
                // factors from the lanes of s), so each warp writes its own copy
                if (!wait_all(qsempty, (uint32_t)((gi & 1) ^ 1))) break;
                tc::fence_after_sync();
                uint32_t v[4][NKS];
                if (cu.w == w0) {
#pragma unroll
                    for (int gq = 0; gq < 4; ++gq)
#pragma unroll
                        for (int j = 0; j < NKS; ++j) v[gq][j] = q_first[gq][j];
                } else {
                    load_qscales<NKS>(p, cu.b, cu.g, lane, v);
                }
#pragma unroll
                for (int gq = 0; gq < 4; ++gq)
#pragma unroll
                    for (int j = 0; j < NKS; ++j)
                        tmem_st1(tmem_base + lane_off + p.sfb_col + (uint32_t)(4 * j + gq), v[gq][j]);
                tc::tmem_wait_st();
                tc::fence_before_sync();
                __syncwarp();
                mbar_arrive(smem_u32(qsfull), lane == 0);
                ++gi;
            }
            // this tile's key scales: staged kSfAhead tiles ago
            if (!wait_all(sfld + (int)(i % kSfAhead), (uint32_t)((i / kSfAhead) & 1))) break;
            const int sl = sr.idx;
            if (!wait_all(sempty + sl, sr.phase ^ 1u)) break;
            tc::fence_after_sync();
            for (int h = 0; h < p.sub; ++h) {
                uint32_t v[NKS];
                const uint8_t *row = sf_smem + ((size_t)(i % kSfAhead) * p.tile_keys + h * kSubKeys + r) * KB;
#pragma unroll
                for (int j = 0; j < NKS; ++j) v[j] = reinterpret_cast<const uint32_t *>(row)[j];
                // key row r of sub-tile h at lane r, column r / 32 = sub of each K step's block
#pragma unroll
                for (int j = 0; j < NKS; ++j)
                    tmem_st1(tmem_base + lane_off + p.sfa_col + (uint32_t)(4 * ((sl * p.sub + h) * NKS + j) + sub), v[j]);
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            __syncwarp();
            mbar_arrive(smem_u32(sfull + sl), lane == 0);
            sr.next(kSfSlots);
            // refill the staging slot just read with the tile kSfAhead ahead
            __syncwarp();
            prefetch(pf, i + kSfAhead);
            if (pf.w < w1) advance(p, pf);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp < kMma2Warp) {
        // ------------------------------------------------------------ epilogue (warps 6..21)
        // Groups of four warps.  Two-sub-tile tiles: tile i -> accumulator i % n_acc
        // and the group pair i % 2, sub-tile h to group 2 (i % 2) + h, so that a
        // tile's two sub-tiles are summed in parallel (one group per tile took
        // ~2 us per tile, the accumulators' turnaround set the pace).  One
        // sub-tile: tile i -> accumulator and group i % n_acc.  A group never
        // waits on a tfull phase two phases ahead of the one it means: the next
        // use of its accumulator needs this group's tempty arrival.
        const int eg = (warp - 6) >> 2;
        const bool pairs = p.sub == 2;
        const int pair = eg >> 1, hsel = eg & 1;
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int row = quarter * 32 + lane;
        const int et = (threadIdx.x - 192) & 127;  // thread within its group
        float *ws_g = w_s + eg * p.NQ * p.H_pad;
        int *nv_g = nvis_s + eg * p.NQ;
        int loaded_b = -1, loaded_g = -1;
        for (Cursor cu = cursor_at(p, w0); cu.w < w1; advance(p, cu)) {
            const int li = (int)(cu.w - w0);
            if (pairs ? ((li & 1) != pair) : (li % p.n_acc != eg)) continue;
            const int b = cu.b, g = cu.g;
            if (b != loaded_b || g != loaded_g) {
                group_bar(eg);
                for (int i = et; i < p.NQ * p.H_pad; i += 128) {
                    const int qi = i / p.H_pad, h = i - qi * p.H_pad;
                    const int q = g * p.NQ + qi;
                    ws_g[i] = (q < p.nq && h < p.H_I) ? __ldg(p.w + ((size_t)b * p.nq + q) * p.H_I + h) : 0.f;
                }
                for (int qi = et; qi < p.NQ; qi += 128) {
                    const int q = g * p.NQ + qi;
                    nv_g[qi] = q < p.nq ? (int)n_visible(__ldg(p.q_pos + (size_t)b * p.nq + q), p.m, p.N) : 0;
                }
                group_bar(eg);
                loaded_b = b;
                loaded_g = g;
            }
            const int acc = li % p.n_acc;
            const uint32_t aph = (uint32_t)((li / p.n_acc) & 1);
            const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(tfull + acc), aph, p.ctx, abort_flag));
            if (!ok) break;
            tc::fence_after_sync();
            for (int h = 0; h < p.sub; ++h) {
                if (pairs && h != hsel) continue;
                const long long s = (long long)cu.kt * p.tile_keys + h * kSubKeys + row;
                const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)((acc * p.sub + h) * p.n_cols);
                for (int qi = 0; qi < p.NQ; ++qi) {
                    const int q = g * p.NQ + qi;
                    if (q >= p.nq) break;
                    // 32 columns per TMEM load round (two 16-column loads in flight), two
                    // partial sums per round keep the FMA chains short
                    float part[2] = {0.f, 0.f};
                    for (int hc = 0; hc < p.H_pad; hc += 32) {
                        float v[32];
                        const int nl = min(2, (p.H_pad - hc) >> 4);
#pragma unroll
                        for (int u = 0; u < 2; ++u)
                            if (u < nl) tc::tmem_ld16(tbase + (uint32_t)(qi * p.H_pad + hc + 16 * u), v + 16 * u);
                        tc::tmem_wait_ld();
                        const float *ws = ws_g + qi * p.H_pad + hc;
#pragma unroll
                        for (int u = 0; u < 2; ++u)
                            if (u < nl) {
#pragma unroll
                                for (int i = 0; i < 16; ++i)
                                    part[u] = fmaf(ws[16 * u + i], fmaxf(v[16 * u + i], 0.f), part[u]);
                            }
                    }
                    const float score = part[0] + part[1];
                    if (s < p.N) p.scores[((size_t)b * p.nq + q) * p.N + s] = s < nv_g[qi] ? score : -INFINITY;
                }
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

// kind::mxf4nvf4 instruction descriptor: A and B e2m1 (format 1), K-major,
// scale factors ue4m3 (scale format 0, factor ids 0), fp32 accumulate (implied).
constexpr uint32_t idesc_mxf4nvf4(int m, int n) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

}  // namespace

// d_I in {64, 128, 256} (one to four K steps of 64), up to 128 query-head rows per tile.
bool index_fp4_tc_supported(int H_I, int d_I) {
    return (d_I == 64 || d_I == 128 || d_I == 256) && H_I >= 1 && H_I <= 128;
}

int launch_index_fp4_tc(const uint8_t *q4, const uint8_t *q4s, const float *w, const uint8_t *k4,
                        const uint8_t *k4s, const int *q_pos, int batch, int nq, long long N, int H_I, int d_I,
                        int m, float *scores, const DevCtx &ctx, cudaStream_t st) {
    Fp4BsParams p = {};
    p.k4s = k4s; p.q4s = q4s; p.w = w; p.q_pos = q_pos; p.scores = scores;
    p.N = N; p.nq = nq; p.H_I = H_I; p.d_I = d_I; p.m = m; p.ctx = ctx;
    p.H_pad = std::max(16, (H_I + 15) / 16 * 16);
    p.kb = d_I / 16;
    p.nks = d_I / 64;
    const uint32_t row_bytes = (uint32_t)(d_I / 2);  // packed codes per row: 32, 64 or 128
    p.layout = row_bytes == 128 ? tc::kLayoutSw128 : (row_bytes == 64 ? tc::kLayoutSw64 : tc::kLayoutSw32);
    const CUtensorMapSwizzle sw = row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                                   : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                                      : CU_TENSOR_MAP_SWIZZLE_32B);
    p.sbo = 8u * row_bytes;
    // queries per tile: as many as fit in N <= 128 rows
    const int NQ = std::max(1, std::min(nq, 128 / p.H_pad));
    p.NQ = NQ;
    p.n_cols = NQ * p.H_pad;
    p.q_bytes = (uint32_t)p.n_cols * row_bytes;
    // Tensor memory: accumulators, then the key-scale slots, then the query-head
    // scales (a 4-column block per K step).  A tile is two M = 128 sub-tiles
    // (256 keys) when three tiles' accumulators still fit: the MMA warp's fixed
    // cost per tile (barrier waits, commits) is then spread over twice the keys.
    int sf_cols = 0;
    for (p.sub = 2;; p.sub = 1) {
        sf_cols = (kSfSlots * p.sub + 1) * 4 * p.nks;
        p.n_acc = std::min(kMaxAcc, (512 - sf_cols) / (p.n_cols * p.sub));
        if (p.n_acc >= 3 || p.sub == 1) break;
    }
    if (p.n_acc < 2) return CSA_ERR_UNSUPPORTED;
    p.tile_keys = kSubKeys * p.sub;
    p.sub_desc = (uint32_t)(kSubKeys * row_bytes) >> 4;
    p.stage_bytes = (uint32_t)p.tile_keys * row_bytes;
    const size_t smem_cap = 200 * 1024;
    const size_t fixed = ((p.q_bytes + 1023u) & ~1023u) + (size_t)kSfAhead * p.tile_keys * p.kb +
                         kEpiGroups * ((size_t)NQ * p.H_pad * 4 + NQ * 4) + 1024;
    p.stages = (int)std::min<size_t>(kMaxStages, (smem_cap - fixed) / p.stage_bytes);
    if (p.stages < 2) return CSA_ERR_UNSUPPORTED;
    p.sfa_col = (uint32_t)(p.n_acc * p.sub * p.n_cols);
    p.sfb_col = p.sfa_col + (uint32_t)(kSfSlots * p.sub * 4 * p.nks);
    p.tmem_cols = 512;
    p.idesc = idesc_mxf4nvf4(kSubKeys, p.n_cols);
    p.groups_per_batch = (nq + NQ - 1) / NQ;
    p.n_ktiles = (int)((N + p.tile_keys - 1) / p.tile_keys);
    p.total_work = (long long)batch * p.groups_per_batch * p.n_ktiles;

    CUtensorMap kmap, qmap;
    memset(&kmap, 0, sizeof(kmap));
    memset(&qmap, 0, sizeof(qmap));
    {
        const uint64_t dims[3] = {row_bytes, (uint64_t)N, (uint64_t)batch};
        const uint64_t strides[2] = {row_bytes, (uint64_t)N * row_bytes};
        const uint32_t box[3] = {row_bytes, (uint32_t)p.tile_keys, 1};
        if (!encode_tensor_map(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, k4, dims, strides, box, sw))
            return CSA_ERR_CUDA;
    }
    {
        const uint64_t dims[4] = {row_bytes, (uint64_t)H_I, (uint64_t)nq, (uint64_t)batch};
        const uint64_t strides[3] = {row_bytes, (uint64_t)H_I * row_bytes, (uint64_t)nq * H_I * row_bytes};
        const uint32_t box[4] = {row_bytes, (uint32_t)p.H_pad, (uint32_t)NQ, 1};
        if (!encode_tensor_map(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, q4, dims, strides, box, sw))
            return CSA_ERR_CUDA;
    }
    const size_t smem = 1024 + (size_t)p.stages * p.stage_bytes + fixed +
                        (2 * kMaxStages + 2 * kMaxAcc + 2 * kSfSlots + 4 + kSfAhead) * 8 + 16;
    void (*kern)(const CUtensorMap, const CUtensorMap, const Fp4BsParams) =
        p.kb == 16 ? index_fp4_bs_kernel<16> : (p.kb == 8 ? index_fp4_bs_kernel<8> : index_fp4_bs_kernel<4>);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return CSA_ERR_CUDA;
    const int grid = (int)std::min<long long>(p.total_work, num_sms());
    kern<<<grid, kThreads, smem, st>>>(kmap, qmap, p);
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // namespace csa

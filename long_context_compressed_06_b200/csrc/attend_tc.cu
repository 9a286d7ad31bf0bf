// attend_tc.cu -- CSA / HCA core attention on the 5th-generation tensor cores.
//
// One query at a time: H (<= 128) RMSNorm'd query heads share one KV head of
// dim D (K = V); the key set is the selected compressed entries (CSA) or all
// visible entries (HCA) plus the sliding window of raw stream-A rows
// (techniques map rows "Grouped-query attention", "Sliding-window attention",
// "QK normalization").  Flash-style, per tile of 64 keys:
//   S = Q K^T       (tcgen05.mma M = 64 heads, N = 64 keys, fp32 in TMEM),
//                   scaled per head by its 1/RMS (the RMSNorm of the query)
//   online softmax in fp32, log2 domain; the running max is raised only when
//   it grows by more than 2^8, so the O rescale in TMEM is rare
//   O += P V        (tcgen05.mma M = 64 heads, N <= 256 dims per MMA, V read
//                    MN-major from the same shared-memory tile as K)
//
// TMEM budget: O for 128 heads x 512 dims in fp32 would take all of one SM's
// tensor memory, so each CTA owns 64 heads (M = 64).  An M = 64 accumulator
// occupies lanes 0-15 of every 32-lane sub-partition; O sits there (all D
// columns) and the two S buffers sit at lane offset 16 (columns 0..127), with
// the item's Q Q^T beside them (columns 128..191).  The
// 16x32bx2 TMEM access shape keeps every warp inside the lane half it means
// to touch.  The two head halves of a query are independent CTAs: no cluster,
// no exchange; each streams the gathered rows itself (the second read of a
// row is an L2 hit).
//
// Warp roles (352 threads): warp 0 TMEM owner, TMA loader of each work
// item's raw query rows and, with warp 8, MMA issuer (lane 0 issues through
// guarded instructions; each issuer takes half of every product); warps 1..3
// and 9..10 gather the key rows with 16-byte cp.async into
// the 128-byte swizzled layout (one 512-byte coalesced row segment per warp
// instruction; HCA tiles of consecutive entries arrive as TMA tiles instead)
// from kernel entry on, each tile's key-validity mask travelling with it
// (FP8 rows: the e4m3 codes are copied the same way and expanded to bf16 in
// place once the next tile's copies are issued);
// warps 4..7 take each head's 1/RMS from the diagonal of Q Q^T (rewriting the
// query tile only for a gain or RoPE), then run the softmax, two threads per
// head (keys 0-31 / 32-63, D/2 output columns each), and store the output
// rows from registers (64 contiguous bytes per thread and 64-column slab; a
// shared-memory staging for TMA tile stores measured slower).  The roles only
// meet at mbarriers, so the gathers of the next work item overlap the output
// of the current one.  Work items are (query, key split, head half); splits
// write bf16 partial rows (each divided by its own sum) + (max, sum) that
// attend_combine merges in a fixed order.  Every wait is bounded and every
// role warp stays converged.
#include <algorithm>
#include <cstring>

#include "attend_common.cuh"
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int kMma2Warp = 8;   // the second MMA issuer
constexpr int kThreads = 352;  // warp 0 and 8: MMA; 1-3 and 9-10: gathers; 4-7: softmax
constexpr int kTileKeys = 64;
constexpr int kHeads = 64;          // heads per CTA (M of every MMA)
constexpr int kSoftmaxWarp0 = 4;
// gather warps 1, 2, 3, 9, 10 (five: issuing a tile's 4096 16-byte copies took ~0.8 us
// with three, on the critical path between a stage's release and its next tile)
constexpr int kProducerWarps = 5;
CSA_DEVINL bool is_producer_warp(int w) { return (w >= 1 && w < 4) || w >= 9; }
CSA_DEVINL int producer_index(int w) { return w < 4 ? w - 1 : w - 6; }
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kMaxStages = 4;

struct AttTcParams {
    AttendArgs a;
    int kv_tma;         // dense key set over bf16 rows: whole tiles of entries arrive by TMA
    int HH;             // head halves per query (1 or 2)
    int stages;
    uint32_t idesc_qk, idesc_pv;
    long long n_work;   // n_bq * splits * HH
    DevCtx ctx;
};

template <int D>
struct Layout {
    static constexpr int kChunks = D / 64;                       // 64-dim, 128-byte swizzle rows
    static constexpr uint32_t kQBytes = kHeads * D * 2;          // [kChunks][64 heads][128 B]
    static constexpr uint32_t kStageBytes = kTileKeys * D * 2;   // [kChunks][64 keys][128 B]
    static constexpr uint32_t kPBytes = kHeads * kTileKeys * 2;  // [64 heads][128 B]
    static constexpr int kPvN = D < 256 ? D : 256;               // N of one P.V MMA
};

struct Smem {
    uint8_t *q, *k, *p;
    uint64_t *kfull, *kempty, *sfull, *sempty, *pfull, *pempty, *oready, *qready, *qempty, *qfull, *qqready;
    uint64_t *kmask;  // [stage] validity of the 64 keys in the stage
    uint32_t *tmem_slot;
    int *abort_flag;
};

template <int D>
CSA_DEVINL Smem carve(uint8_t *raw, int stages) {
    using Lt = Layout<D>;
    Smem s;
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    s.q = base;
    s.k = s.q + Lt::kQBytes;
    s.p = s.k + (size_t)stages * Lt::kStageBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(s.p + 2 * Lt::kPBytes);
    s.kfull = bars;
    s.kempty = bars + kMaxStages;
    s.sfull = bars + 2 * kMaxStages;
    s.sempty = s.sfull + 2;
    s.pfull = s.sempty + 2;
    s.pempty = s.pfull + 2;
    s.oready = s.pempty + 2;
    s.qready = s.oready + 2;
    s.qempty = s.qready + 1;
    s.qfull = s.qempty + 1;
    s.qqready = s.qfull + 1;
    s.kmask = s.qqready + 1;
    s.tmem_slot = reinterpret_cast<uint32_t *>(s.kmask + kMaxStages);
    s.abort_flag = reinterpret_cast<int *>(s.tmem_slot + 1);
    return s;
}

template <int D>
size_t smem_bytes(int stages) {
    using Lt = Layout<D>;
    return 1024 + Lt::kQBytes + (size_t)stages * Lt::kStageBytes + 2 * Lt::kPBytes + (3 * kMaxStages + 14) * 8 + 16;
}

// ---------------------------------------------------------------- TMEM, 16-lane access shape
// 16x32bx2 with a split offset of 32 columns: threads 0-15 read lanes
// base..base+15 at columns [c, c+32), threads 16-31 the same lanes at
// columns [c+32, c+64).
CSA_DEVINL void tmem_ld_half32(uint32_t taddr, float v[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

CSA_DEVINL void tmem_st_half32(uint32_t taddr, const float v[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], 32, {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
          "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
          "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
          "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
          "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
          "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
          "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
          "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
          "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
          "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
          "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

// ---------------------------------------------------------------- key enumeration
// Key e of one query: e < nsel4 -> selection slot e (slots >= nsel are padding),
// else window row e - nsel4.  nsel4 = nsel rounded up to a multiple of 4.
struct Keys {
    long long nsel, nsel4, nwin, u0, total;
};

CSA_DEVINL Keys query_keys(const AttendArgs &a, long long t) {
    Keys k;
    k.nsel = a.dense ? n_visible(t, a.m, a.N) : a.k;
    k.nsel4 = (k.nsel + 3) & ~3LL;
    long long u0 = t - a.W + 1;
    u0 = u0 < 0 ? 0 : u0;
    k.u0 = u0 < a.win_pos0 ? a.win_pos0 : u0;
    const long long last = a.win_pos0 + a.win_rows - 1;
    const long long u1 = t < last ? t : last;
    k.nwin = u1 >= k.u0 ? u1 - k.u0 + 1 : 0;
    k.total = k.nsel4 + k.nwin;
    return k;
}

// The selection index of key e as stored (loaded only: the value is consumed
// by key_row_index, so that the load can be issued a tile ahead).
CSA_DEVINL int key_index_raw(const AttendArgs &a, const Keys &ks, long long bq, long long e, long long e_end) {
    if (e >= e_end) e = e_end - 1;
    return (!a.dense && e >= 0 && e < ks.nsel) ? __ldg(a.idx + bq * a.k + e) : 0;
}

// Row of key e -- its index in kv (win == false) or in the window buffer --
// and whether it takes part (keys past e_end, selection padding and
// out-of-range indices read a valid row; their scores are masked).  jraw is
// key_index_raw(e).
CSA_DEVINL size_t key_row_index(const AttendArgs &a, const Keys &ks, long long b, long long e, long long e_end,
                                int jraw, bool &valid, bool &win) {
    win = false;
    valid = e < e_end;
    if (!valid) e = e_end - 1;  // e_end >= 1 whenever a tile exists
    if (e < ks.nsel4) {
        long long j = 0;
        if (e < ks.nsel) {
            j = a.dense ? e : (long long)jraw;
            if (j < 0 || j >= a.N) {
                j = 0;
                valid = false;
            }
        } else {
            valid = false;
        }
        return (size_t)b * a.N + j;
    }
    long long w = e - ks.nsel4;
    if (w >= ks.nwin) valid = false;
    w = w < ks.nwin ? w : ks.nwin - 1;
    w = w < 0 ? 0 : w;
    win = true;
    return (size_t)b * a.win_rows + (ks.u0 - a.win_pos0) + w;
}

CSA_DEVINL const uint16_t *key_slot(const AttendArgs &a, const Keys &ks, long long b, long long e, long long e_end,
                                    int jraw, bool &valid) {
    bool win;
    const size_t r = key_row_index(a, ks, b, e, e_end, jraw, valid, win);
    return (win ? a.win : a.kv) + r * a.D;
}

// FP8 rows: the codes of key e (the row's exponent bytes follow from the same index)
CSA_DEVINL const uint8_t *key_slot8(const AttendArgs &a, const Keys &ks, long long b, long long e, long long e_end,
                                    int jraw, bool &valid, const uint8_t *&exps) {
    bool win;
    const size_t r = key_row_index(a, ks, b, e, e_end, jraw, valid, win);
    exps = (win ? a.win8e : a.kv8e) + r * (a.D / 128);
    return (win ? a.win8 : a.kv8) + r * a.D;
}

// 8 e4m3 codes times 2^(e - 127) -> 8 bf16, exactly: e4m3 -> f16 is exact, the
// power-of-two scale is exact in fp32, and the product has at most 4
// significant bits inside bf16's range (the quantiser keeps e in [3, 246]).
CSA_DEVINL uint4 e4m3x8_bf16x8(uint2 raw, uint32_t e) {
    const float sc = __uint_as_float(e << 23);
    const uint32_t w[2] = {raw.x, raw.y};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t h;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)(w[i >> 1] >> (16 * (i & 1)))));
        const float lo = __half2float(__ushort_as_half((unsigned short)(h & 0xffffu))) * sc;
        const float hi = __half2float(__ushort_as_half((unsigned short)(h >> 16))) * sc;
        o[i] = pack_bf16x2(lo, hi);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Warp-uniform bounded wait.  Every lane polls and the outcome is voted: a
// wait polled by one lane while the others park at a shuffle leaves the warp
// running its following code far slower (measured: 4x on a pass over the query tile).
CSA_DEVINL bool warp_wait(uint32_t bar, uint32_t parity, const DevCtx &ctx, volatile int *abort) {
    const bool ok = mbar_wait(bar, parity, ctx, abort);
    return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------- query rows
// The raw query rows of a work item arrive by TMA, already in the swizzled
// K-major tile [D/64][64 heads][128 B] (heads past H are zero-filled).  The
// RMSNorm is applied to the scores (each head's 1/RMS from the diagonal of
// Q Q^T, computed by the tensor cores on the raw rows), so the tile is used as
// it landed unless a per-channel gain or partial RoPE asks for a rewrite:
//   Q' = q * gain, then the rotation of the trailing kRopeDim channels.
// A lane owns whole 16-byte units (8 dims) of a row; every shared-memory
// access is a conflict-free 16-byte access.
template <int D>
struct QLanes {
    static constexpr int UR = D / 8;               // 16-byte units per row
    static constexpr int LPR = UR < 32 ? UR : 32;  // lanes per row
    static constexpr int RPI = 32 / LPR;           // rows per warp instruction
    static constexpr int UPL = UR / LPR;           // units per lane
    static constexpr int PASSES = (kHeads / 4) / RPI;
};

// With partial RoPE the row's last kRopeDim / 8 units (all in a lane's last
// unit slot, since kRopeDim <= D) rotate after the gain: unit r0 + j pairs
// with r0 + j + 4, held by lane ^ 4 in the same slot, so one shuffle fetches
// the partner values.
template <int D>
CSA_DEVINL void rewrite_q(const AttendArgs &a, const Smem &s, int sw, const float (&g)[QLanes<D>::UPL][8],
                          long long t) {
    using QL = QLanes<D>;
    static_assert(D >= kRopeDim && kRopeDim / 8 == 8, "rope units: 8 per row, partners 4 units apart");
    const int lane = threadIdx.x & 31;
    const int sub = lane / QL::LPR, ul = lane % QL::LPR;
#pragma unroll 4
    for (int pass = 0; pass < QL::PASSES; ++pass) {
        const int hl = sw * (kHeads / 4) + pass * QL::RPI + sub;
        uint4 *ptr[QL::UPL];
        float x[QL::UPL][8];
#pragma unroll
        for (int u = 0; u < QL::UPL; ++u) {
            const int unit = ul + u * QL::LPR;
            ptr[u] = reinterpret_cast<uint4 *>(s.q + (size_t)(unit >> 3) * kHeads * 128 + hl * 128 +
                                               (((unit & 7) ^ (hl & 7)) << 4));
            unpack8(*ptr[u], x[u]);
#pragma unroll
            for (int e = 0; e < 8; ++e) x[u][e] *= g[u][e];
        }
        if (a.rope_cos) {  // uniform over the grid: every lane takes the shuffles
            constexpr int u = QL::UPL - 1;
            constexpr int r0 = QL::UR - kRopeDim / 8;  // first rotated unit
            const int unit = ul + u * QL::LPR;
            float pv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pv[e] = __shfl_xor_sync(0xffffffffu, x[u][e], 4);
            if (unit >= r0) {
                const bool first = unit < r0 + 4;  // first half of the rotated slice
                const int i0 = ((unit - r0) & 3) * 8;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float2 cs = rope_cs(a, t, i0 + e);
                    x[u][e] = first ? x[u][e] * cs.x - pv[e] * cs.y : x[u][e] * cs.x + pv[e] * cs.y;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < QL::UPL; ++u) *ptr[u] = pack8(x[u]);
    }
}

// One work item: (query, key split, head half).  The query's tiles of 64 keys
// are dealt to the splits in balanced contiguous ranges.
struct Item {
    long long bq, b, e0, e1;
    Keys ks;
    int split, head0, ntiles;
};

CSA_DEVINL Item work_item(const AttTcParams &p, long long wi) {
    const AttendArgs &a = p.a;
    Item it;
    const int hh = (int)(wi % p.HH);
    const long long rest = wi / p.HH;
    it.split = (int)(rest % a.splits);
    it.bq = rest / a.splits;
    it.b = it.bq / a.nq;
    it.head0 = hh * kHeads;
    it.ks = query_keys(a, __ldg(a.q_pos + it.bq));
    const long long T = (it.ks.total + kTileKeys - 1) / kTileKeys;
    const long long t0 = T * it.split / a.splits, t1 = T * (it.split + 1) / a.splits;
    it.e0 = t0 * kTileKeys;
    it.e1 = std::min(it.ks.total, t1 * kTileKeys);
    it.ntiles = (int)(t1 - t0);
    return it;
}

template <int D, bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kvmap,
                     const AttTcParams p) {
    using Lt = Layout<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const Smem s = carve<D>(smem_raw, p.stages);
    const AttendArgs &a = p.a;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; ++i) {
            // one cp.async completion arrive per producer thread + the key-mask arrive
            mbar_init(s.kfull + i, kProducerWarps * 32 + 1);
            mbar_init(s.kempty + i, 2);  // one commit per MMA issuer
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(s.sfull + i, 2);
            mbar_init(s.sempty + i, 128);
            mbar_init(s.pfull + i, 128);
            mbar_init(s.pempty + i, 2);
        }
        mbar_init(s.oready, 2);
        mbar_init(s.oready + 1, 2);
        mbar_init(s.qready, 128);
        mbar_init(s.qempty, 2);
        mbar_init(s.qfull, 1);
        mbar_init(s.qqready, 2);
        *s.abort_flag = 0;
        fence_mbar_init();
        tc::prefetch_tmap(&qmap);
        if (p.kv_tma) tc::prefetch_tmap(&kvmap);
    }
    // per-dimension query gains of this lane's units (softmax warps), read once
    float qg[QLanes<D>::UPL][8];
#pragma unroll
    for (int u = 0; u < QLanes<D>::UPL; ++u)
#pragma unroll
        for (int e = 0; e < 8; ++e)
            qg[u][e] = (warp >= kSoftmaxWarp0 && a.q_gain)
                           ? __ldg(a.q_gain + (lane % QLanes<D>::LPR + u * QLanes<D>::LPR) * 8 + e)
                           : 1.f;
    if (warp == 0) {
        tc::tmem_alloc(smem_u32(s.tmem_slot), 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // the split merge (a programmatic dependent) may launch once every CTA is here
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t tmem = *s.tmem_slot;
    const uint32_t tmem_o = tmem;                  // lanes 0-15 of each sub-partition, columns 0..D-1
    const uint32_t tmem_s = tmem + (16u << 16);    // lanes 16-31, columns 0..127 (two S buffers)
    const uint32_t tmem_qq = tmem_s + 128;          // lanes 16-31, columns 128..191 (Q Q^T of the item)
    // the second MMA issuer's halves of S and Q Q^T: lanes 16-31, columns 192..383
    constexpr uint32_t kIss2Cols = 192;
    // the query tile is rewritten in shared memory only for a gain or partial RoPE
    const bool q_rw = a.q_gain != nullptr || a.rope_cos != nullptr;

    // The roles run decoupled across work items; their only contacts are the
    // mbarriers (key ring kfull/kempty, S buffers sfull/sempty, P buffers
    // pfull/pempty, the query tile qfull/qqready/qready/qempty, and oready[g & 1], committed after the
    // P.V of tile g).  A parity wait is exact only if the barrier's previous
    // phase is known complete; oready alternates between two barriers because
    // the softmax may wait for P.V g while P.V g-1 is still running, whereas
    // P.V g-2 is known complete (the P buffer it read was released before P_g
    // was written).  jt counts the tiles this CTA has processed, identically in
    // every role.
    if (is_producer_warp(warp)) {
        // ------------------------------------------------------------ producers (cp.async gather)
        // Each warp copies keys pw, pw+3, ...: lane l moves 16-byte units l, l+32,
        // .. of the row (coalesced 512 B per instruction).  Row pointers of the
        // tile's 64 keys are computed once per tile, two per lane.
        const int pw = producer_index(warp);
        long long jt = 0;
        bool ok = true;
        bool dep_done = false;
        // FP8 rows: a tile's codes are copied (cp.async) into its stage as they
        // are stored -- the 64 codes of a key's 64-dimension chunk in the first
        // half of the 128-byte row that chunk's bf16 values will fill -- and
        // expanded in place once the next tile's copies are issued, so that the
        // copies of one tile overlap the conversion of the other.  f8_st is the
        // stage waiting for its conversion (-1: none), with its key mask and this
        // lane's block exponent of every key the warp copies.
        constexpr int kKeysPerWarp = (kTileKeys + kProducerWarps - 1) / kProducerWarps;
        int f8_st = -1;
        uint64_t f8_mask = 0;
        uint32_t f8_e[kKeysPerWarp];
#pragma unroll
        for (int i = 0; i < kKeysPerWarp; ++i) f8_e[i] = 0u;
        // expands the codes of stage f8_st (after the copies of this thread are
        // complete up to the newest `newer` groups) and marks the tile full
        const auto f8_convert = [&](bool newer) {
            if constexpr (FP8) {
                if (newer) asm volatile("cp.async.wait_group 1;" ::: "memory");
                else asm volatile("cp.async.wait_group 0;" ::: "memory");
                __syncwarp();
                const uint32_t stage = smem_u32(s.k + (size_t)f8_st * Lt::kStageBytes);
                // keys in batches of kBatch: their codes read, then (after every lane has
                // read its own) the rows overwritten with the bf16 values
                constexpr int kBatch = 4;
#pragma unroll
                for (int i0 = 0; i0 < kKeysPerWarp; i0 += kBatch) {
                    uint4 c[kBatch];
#pragma unroll
                    for (int j = 0; j < kBatch; ++j) {
                        const int key = pw + kProducerWarps * (i0 + j);
                        c[j] = make_uint4(0u, 0u, 0u, 0u);
                        // lane l holds codes 16l..16l+15: chunk l / 4, bytes 16 (l % 4).. of its row
                        if (i0 + j < kKeysPerWarp && key < kTileKeys && lane < D / 16)
                            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                         : "=r"(c[j].x), "=r"(c[j].y), "=r"(c[j].z), "=r"(c[j].w)
                                         : "r"(stage + (lane >> 2) * (kTileKeys * 128) + key * 128 + (lane & 3) * 16));
                    }
                    __syncwarp();  // every lane has its codes before any lane overwrites the rows
#pragma unroll
                    for (int j = 0; j < kBatch; ++j) {
                        const int key = pw + kProducerWarps * (i0 + j);
                        if (i0 + j < kKeysPerWarp && key < kTileKeys && lane < D / 16) {
                            const uint32_t row = stage + (lane >> 2) * (kTileKeys * 128) + key * 128;
                            const uint4 lo = e4m3x8_bf16x8(make_uint2(c[j].x, c[j].y), f8_e[i0 + j]);
                            const uint4 hi = e4m3x8_bf16x8(make_uint2(c[j].z, c[j].w), f8_e[i0 + j]);
                            const int u0 = (lane & 3) * 2;  // the 16-byte units of these 16 values
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + ((u0 ^ (key & 7)) << 4)),
                                         "r"(lo.x), "r"(lo.y), "r"(lo.z), "r"(lo.w)
                                         : "memory");
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                         ::"r"(row + (((u0 + 1) ^ (key & 7)) << 4)), "r"(hi.x), "r"(hi.y), "r"(hi.z),
                                         "r"(hi.w)
                                         : "memory");
                        }
                    }
                }
                tc::fence_proxy_async_smem();  // the generic stores before the MMA's reads
                mbar_arrive(smem_u32(s.kfull + f8_st));
                if (pw == 0) {  // the mask travels with the tile (release by lane 0's arrive)
                    if (lane == 0) s.kmask[f8_st] = f8_mask;
                    mbar_arrive(smem_u32(s.kfull + f8_st), lane == 0);
                }
                f8_st = -1;
            }
        };
        for (long long wi = blockIdx.x; wi < p.n_work && ok; wi += gridDim.x) {
            const Item it = work_item(p, wi);
            // As a programmatic dependent (csa_decode_step) the selection is
            // complete only once the top-k grid is: wait before the first item
            // that reads selected slots (the query prologue and the window-only
            // items run meanwhile).  A no-op for an ordinary launch.
            if (!dep_done && !a.dense && it.e0 < it.ks.nsel4) {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                dep_done = true;
            }
            // Row pointers of the tile's 64 keys, two per lane.  The selection
            // indices of tile j + 1 are loaded while tile j is issued (an L2 round
            // trip that would otherwise separate the tiles' gathers); only the next
            // iteration uses them.
            int nraw0 = 0, nraw1 = 0;
            if (it.ntiles > 0) {
                nraw0 = key_index_raw(a, it.ks, it.bq, it.e0 + lane, it.e1);
                nraw1 = key_index_raw(a, it.ks, it.bq, it.e0 + 32 + lane, it.e1);
            }
            for (int j = 0; j < it.ntiles; ++j) {
                const long long g = jt + j;
                const int st = (int)(g % p.stages);
                const long long ebase = it.e0 + (long long)j * kTileKeys;
                const int raw0 = nraw0, raw1 = nraw1;
                if (j + 1 < it.ntiles) {
                    nraw0 = key_index_raw(a, it.ks, it.bq, ebase + kTileKeys + lane, it.e1);
                    nraw1 = key_index_raw(a, it.ks, it.bq, ebase + kTileKeys + 32 + lane, it.e1);
                }
                bool v0, v1;
                const uint16_t *r0 = nullptr, *r1 = nullptr;
                const uint8_t *c0 = nullptr, *c1 = nullptr, *x0 = nullptr, *x1 = nullptr;
                if constexpr (FP8) {
                    c0 = key_slot8(a, it.ks, it.b, ebase + lane, it.e1, raw0, v0, x0);
                    c1 = key_slot8(a, it.ks, it.b, ebase + 32 + lane, it.e1, raw1, v1, x1);
                } else {
                    r0 = key_slot(a, it.ks, it.b, ebase + lane, it.e1, raw0, v0);
                    r1 = key_slot(a, it.ks, it.b, ebase + 32 + lane, it.e1, raw1, v1);
                }
                const uint32_t mlo = __ballot_sync(0xffffffffu, v0), mhi = __ballot_sync(0xffffffffu, v1);
                if (!warp_wait(smem_u32(s.kempty + st), (uint32_t)(((g / p.stages) & 1) ^ 1), p.ctx, s.abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t stage = smem_u32(s.k + (size_t)st * Lt::kStageBytes);
                // HCA: a tile of 64 consecutive visible entries is one contiguous run of
                // kv rows, loaded by TMA tiles (one per 64-dim chunk) instead of row gathers
                const bool tma_tile = !FP8 && p.kv_tma && ebase + kTileKeys <= it.ks.nsel;
                if (tma_tile) {
                    if (pw == 0) {  // the mask arrive carries the TMA byte count
                        if (lane == 0) s.kmask[st] = ((uint64_t)mhi << 32) | mlo;
                        mbar_arrive_expect_tx(smem_u32(s.kfull + st), Lt::kStageBytes, lane == 0);
                        for (int c = 0; c < Lt::kChunks; ++c)
                            tc::tma_load_3d(stage + c * (kTileKeys * 128), &kvmap, smem_u32(s.kfull + st), c * 64,
                                            (int)ebase, (int)it.b, lane == 0);
                    }
                    // the producers' cp.async arrivals (none pending for this tile)
                    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(s.kfull + st))
                                 : "memory");
                    continue;
                }
                if constexpr (FP8) {
                    // this tile's codes and block exponents in flight, then the previous
                    // tile's expansion
                    uint32_t e_new[kKeysPerWarp];
#pragma unroll
                    for (int i = 0; i < kKeysPerWarp; ++i) {
                        const int key = pw + kProducerWarps * i;
                        e_new[i] = 0u;
                        if (key < kTileKeys) {
                            const uint8_t *crow = reinterpret_cast<const uint8_t *>(
                                __shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(key < 32 ? c0 : c1), key & 31));
                            const uint8_t *xrow = reinterpret_cast<const uint8_t *>(
                                __shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(key < 32 ? x0 : x1), key & 31));
                            if (lane < D / 16) {
                                const uint32_t dst = stage + (lane >> 2) * (kTileKeys * 128) + key * 128 + (lane & 3) * 16;
                                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(crow + lane * 16)
                                             : "memory");
                                e_new[i] = __ldg(xrow + (lane >> 3));  // the block of 128 codes holding 16l..16l+15
                            }
                        }
                    }
                    asm volatile("cp.async.commit_group;" ::: "memory");
                    if (f8_st >= 0) f8_convert(true);
                    f8_st = st;
                    f8_mask = ((uint64_t)mhi << 32) | mlo;
#pragma unroll
                    for (int i = 0; i < kKeysPerWarp; ++i) f8_e[i] = e_new[i];
                } else {
                    // Each warp copies keys pw, pw+3, ...: lane l moves 16-byte units l,
                    // l+32, .. of the row (coalesced 512 B per instruction).
#pragma unroll 2
                    for (int key = pw; key < kTileKeys; key += kProducerWarps) {
                        const uint16_t *row = reinterpret_cast<const uint16_t *>(
                            __shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(key < 32 ? r0 : r1), key & 31));
                        const uint32_t krow = stage + key * 128;
#pragma unroll
                        for (int u = lane; u < D / 8; u += 32) {  // 16-byte units of the row
                            const uint32_t dst = krow + (u >> 3) * (kTileKeys * 128) + (((u & 7) ^ (key & 7)) << 4);
                            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(row + u * 8)
                                         : "memory");
                        }
                    }
                    if (pw == 0) {  // the mask travels with the tile (release by lane 0's arrive)
                        if (lane == 0) s.kmask[st] = ((uint64_t)mhi << 32) | mlo;
                        mbar_arrive(smem_u32(s.kfull + st), lane == 0);
                    }
                    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(s.kfull + st))
                                 : "memory");
                }
            }
            jt += it.ntiles;
        }
        if (ok && f8_st >= 0) f8_convert(false);  // the last tile's expansion
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == 0 || warp == kMma2Warp) {
        // ------------------------------------------------------------ MMA issuers
        // Event driven: P.V for tile i as soon as P_i is written, QK for the
        // next tile as soon as its keys have landed and an S buffer is free.
        // The whole warp runs the loop and polls (decisions are lane 0's, made
        // warp-uniform by a shuffle); lane 0 issues through guarded
        // instructions, never a branch.  Descriptors are built
        // once and advanced by constant offsets.
        // Two issuers (warp 0 and warp 8) run the same loop: one thread issues a
        // tcgen05.mma only every ~100 cycles (measured), so each issues half of
        // every product -- Q Q^T and QK split along the head dimension into two
        // accumulators that the softmax adds, P.V by the two 256-column halves
        // of O (D = 512; below that the first issuer takes all of P.V) -- and
        // commits to every barrier the products release (counts of two).
        const int iss = warp == 0 ? 0 : 1;
        constexpr int kQkSteps = Lt::kChunks * 4;  // K steps of 16 over the head dimension
        const int qk0 = iss * (kQkSteps / 2), qk1 = qk0 + kQkSteps / 2;
        constexpr bool kPvSplit = D == 512;
        const int pv0 = kPvSplit ? iss * (D / 2) : (iss == 0 ? 0 : D), pv1 = kPvSplit ? pv0 + D / 2 : D;
        const uint32_t s_off = iss ? kIss2Cols : 0u;
        const uint64_t qdesc = tc::smem_desc(smem_u32(s.q), 1024, tc::kLayoutSw128);
        const uint64_t kdesc0 = tc::smem_desc(smem_u32(s.k), 1024, tc::kLayoutSw128);
        const uint64_t vdesc0 = tc::smem_desc_lbo(smem_u32(s.k), kTileKeys * 128, 1024, tc::kLayoutSw128);
        const uint64_t pdesc0 = tc::smem_desc(smem_u32(s.p), 1024, tc::kLayoutSw128);
        const auto ready = [&](bool v) { return __shfl_sync(0xffffffffu, v ? 1 : 0, 0) != 0; };
        long long jt = 0;
        uint32_t n_items = 0;
        bool ok = true;
        for (long long wi = blockIdx.x; wi < p.n_work && ok; wi += gridDim.x, ++n_items) {
            const Item it = work_item(p, wi);
            // raw query rows of this item by TMA, once the previous item's QK MMAs are done with the tile
            if (n_items > 0 && !__all_sync(0xffffffffu, mbar_wait(smem_u32(s.qempty), (n_items - 1) & 1u, p.ctx,
                                                                 s.abort_flag)))
                break;
            mbar_arrive_expect_tx(smem_u32(s.qfull), Lt::kQBytes, lane == 0 && iss == 0);
            for (int c = 0; c < Lt::kChunks; ++c)
                tc::tma_load_3d(smem_u32(s.q + (size_t)c * kHeads * 128), &qmap, smem_u32(s.qfull), c * 64,
                                it.head0, (int)it.bq, lane == 0 && iss == 0);
            // Q Q^T of the raw rows: its diagonal gives every head's sum of squares
            // for the RMSNorm (applied to the scores in fp32)
            if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(s.qfull), n_items & 1u, p.ctx, s.abort_flag))) break;
            tc::fence_after_sync();
            for (int t = qk0; t < qk1; ++t) {
                const int c = t >> 2, kk = t & 3;
                tc::mma_f16(tmem_qq + s_off, qdesc + ((c * kHeads * 128 + kk * 32) >> 4),
                            qdesc + ((c * kHeads * 128 + kk * 32) >> 4), p.idesc_qk, t > qk0 ? 1u : 0u, lane == 0);
            }
            tc::mma_commit(smem_u32(s.qqready), lane == 0);
            // the softmax warps have read the diagonal (so the next item's Q Q^T may
            // overwrite it) and, with a gain or RoPE, rewritten the tile
            if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(s.qready), n_items & 1u, p.ctx, s.abort_flag))) break;
            tc::fence_after_sync();
            if (it.ntiles == 0) mbar_arrive(smem_u32(s.qempty), lane == 0);
            int nqk = 0, npv = 0;
            uint64_t t_idle = 0;
            while (npv < it.ntiles) {
                bool progressed = false;
                if (nqk < it.ntiles && nqk < npv + 2) {
                    const long long g = jt + nqk;
                    const int st = (int)(g % p.stages), sb = (int)(g & 1);
                    const bool k_in = mbar_test_wait(smem_u32(s.kfull + st), (uint32_t)((g / p.stages) & 1));
                    const bool s_free = mbar_test_wait(smem_u32(s.sempty + sb), (uint32_t)(((g >> 1) & 1) ^ 1));
                    if (ready(k_in && s_free)) {
                        const bool issuer = lane == 0;
                        tc::fence_proxy_async_smem();  // cp.async data -> tensor-core reads
                        tc::fence_after_sync();
                        const uint64_t kd = kdesc0 + ((uint64_t)(st * Lt::kStageBytes) >> 4);
                        for (int t = qk0; t < qk1; ++t) {
                            const int c = t >> 2, kk = t & 3;
                            tc::mma_f16(tmem_s + s_off + sb * kTileKeys, qdesc + ((c * kHeads * 128 + kk * 32) >> 4),
                                        kd + ((c * kTileKeys * 128 + kk * 32) >> 4), p.idesc_qk, t > qk0 ? 1u : 0u,
                                        issuer);
                        }
                        tc::mma_commit(smem_u32(s.sfull + sb), issuer);
                        if (nqk + 1 == it.ntiles) tc::mma_commit(smem_u32(s.qempty), issuer);  // query tile no longer read
                        ++nqk;
                        progressed = true;
                    }
                }
                if (npv < nqk) {
                    const long long g = jt + npv;
                    const int pb = (int)(g & 1), st = (int)(g % p.stages);
                    if (ready(mbar_test_wait(smem_u32(s.pfull + pb), (uint32_t)((g >> 1) & 1)))) {
                        const bool issuer = lane == 0;
                        tc::fence_after_sync();
                        const uint64_t pd = pdesc0 + ((uint64_t)(pb * Lt::kPBytes) >> 4);
                        const uint64_t vd = vdesc0 + ((uint64_t)(st * Lt::kStageBytes) >> 4);
#pragma unroll
                        for (int kk = 0; kk < kTileKeys / 16; ++kk)
                            for (int n0 = pv0; n0 < pv1; n0 += Lt::kPvN)
                                // V[keys][dims] read MN-major: 64-dim groups kTileKeys*128 bytes
                                // apart (LBO), 8-key groups 1024 bytes apart (SBO); K step = 16 keys
                                tc::mma_f16(tmem_o + n0, pd + ((kk * 32) >> 4),
                                            vd + (((n0 / 64) * kTileKeys * 128 + kk * 16 * 128) >> 4), p.idesc_pv,
                                            (npv == 0 && kk == 0) ? 0u : 1u, issuer);
                        tc::mma_commit(smem_u32(s.kempty + st), issuer);
                        tc::mma_commit(smem_u32(s.pempty + pb), issuer);
                        tc::mma_commit(smem_u32(s.oready + pb), issuer);
                        ++npv;
                        progressed = true;
                    }
                }
                if (progressed) {
                    t_idle = 0;
                } else {
                    const uint64_t now = global_timer_ns();
                    if (t_idle == 0) {
                        t_idle = now;
                    } else if (ready(now - t_idle > p.ctx.budget_ns || *s.abort_flag)) {
                        if (lane == 0) {
                            record_status(p.ctx.status, CSA_ERR_TIMEOUT);
                            *s.abort_flag = 1;
                        }
                        __syncwarp();
                        ok = false;
                        break;
                    }
                }
            }
            jt += it.ntiles;
        }
    } else {
        // ------------------------------------------------------------ softmax + output (warps 4..7)
        // Thread (quarter sp, lane l): head 16*sp + l%16 of this CTA's 64,
        // keys 32*(l/16) .. +31 of each tile; the two threads of a head
        // combine their row max / sum with one shuffle.
        const int sp = warp & 3;
        const int hl = sp * 16 + (lane & 15), kh = lane >> 4;
        const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
        long long jt = 0;
        uint32_t n_items = 0;
        bool ok = true;
        for (long long wi = blockIdx.x; wi < p.n_work && ok; wi += gridDim.x, ++n_items) {
            const Item it = work_item(p, wi);
            const int h = it.head0 + hl;
            if (!warp_wait(smem_u32(s.qfull), n_items & 1u, p.ctx, s.abort_flag)) break;
            const long long tq = __ldg(a.q_pos + it.bq);
            // this head's 1 / RMS (times the softmax scale, in log2 units) from the
            // diagonal of Q Q^T: column hl of row hl, held by the thread of the
            // head's pair whose 32 columns contain it
            if (!warp_wait(smem_u32(s.qqready), n_items & 1u, p.ctx, s.abort_flag)) break;
            tc::fence_after_sync();
            float rq;
            {
                float v[32], v2[32];
                tmem_ld_half32(tmem_qq + lane_base, v);
                tmem_ld_half32(tmem_qq + kIss2Cols + lane_base, v2);  // the second issuer's half
                tc::tmem_wait_ld();
                // select v[hl & 31] without an indexed (local-memory) access
                const int di = hl & 31;
                float d = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) d += (i == di) ? v[i] + v2[i] : 0.f;
                const float other = __shfl_xor_sync(0xffffffffu, d, 16);
                const float ss = kh == (hl >> 5) ? d : other;
                rq = (1.0f / sqrtf(ss / (float)D + a.eps)) * a.scale * 1.4426950408889634f;
            }
            tc::fence_before_sync();
            if (q_rw) {
                rewrite_q<D>(a, s, sp, qg, tq);
                tc::fence_proxy_async_smem();
            }
            mbar_arrive(smem_u32(s.qready));

            float m_run = -INFINITY, l = 0.f;
            for (int j = 0; j < it.ntiles && ok; ++j) {
                const long long g = jt + j;
                const int sb = (int)(g & 1);
                if (!warp_wait(smem_u32(s.sfull + sb), (uint32_t)((g >> 1) & 1), p.ctx, s.abort_flag)) {
                    ok = false;
                    break;
                }
                // the stage's key mask (completed phase: acquires the producer's write)
                const int st = (int)(g % p.stages);
                if (!warp_wait(smem_u32(s.kfull + st), (uint32_t)((g / p.stages) & 1), p.ctx, s.abort_flag)) {
                    ok = false;
                    break;
                }
                const uint64_t vmask = s.kmask[st] >> (32 * kh);
                tc::fence_after_sync();
                float sc[32], sc2[32];
                tmem_ld_half32(tmem_s + lane_base + sb * kTileKeys, sc);
                tmem_ld_half32(tmem_s + kIss2Cols + lane_base + sb * kTileKeys, sc2);  // second issuer's half
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) sc[i] += sc2[i];
                tc::fence_before_sync();
                mbar_arrive(smem_u32(s.sempty + sb));
                float mt = -INFINITY;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    sc[i] = (vmask >> i) & 1u ? sc[i] * rq : -INFINITY;
                    mt = fmaxf(mt, sc[i]);
                }
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
                // raise the running max only when it grows by more than 2^8: O (after the
                // previous P.V) and l are then scaled by 2^(m_old - m_new)
                const bool mine = m_run != -INFINITY && mt > m_run + kRescaleThreshold;
                if (__any_sync(0xffffffffu, mine)) {
                    if (!warp_wait(smem_u32(s.oready + ((g - 1) & 1)), (uint32_t)(((g - 1) >> 1) & 1), p.ctx,
                                   s.abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const float f = mine ? exp2f(m_run - mt) : 1.0f;
                    for (int c = 0; c < D; c += 64) {
                        float v[32];
                        tmem_ld_half32(tmem_o + lane_base + c, v);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] *= f;
                        tmem_st_half32(tmem_o + lane_base + c, v);
                    }
                    tc::tmem_wait_st();
                    if (mine) {
                        l *= f;
                        m_run = mt;
                    }
                }
                if (m_run == -INFINITY) m_run = mt;
                const float mref = m_run == -INFINITY ? 0.f : m_run;
                float ps = 0.f;
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float p0 = exp2f(sc[i] - mref), p1 = exp2f(sc[i + 1] - mref);
                    ps += p0 + p1;
                    pk[i / 2] = pack_bf16x2(p0, p1);
                }
                l += ps + __shfl_xor_sync(0xffffffffu, ps, 16);
                const int pb = (int)(g & 1);
                if (!warp_wait(smem_u32(s.pempty + pb), (uint32_t)(((g >> 1) & 1) ^ 1), p.ctx, s.abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t *prow = s.p + pb * Lt::kPBytes + hl * 128;
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    *reinterpret_cast<uint4 *>(prow + (((4 * kh + u) ^ (hl & 7)) << 4)) =
                        make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                tc::fence_proxy_async_smem();
                tc::fence_before_sync();
                mbar_arrive(smem_u32(s.pfull + pb));
            }
            if (!ok) break;
            // output: O / l (one split, the output rows) or O / l of this split (a
            // partial row; the merge weighs the splits), each thread storing its
            // head's 32 columns of every 64-column slab as four 16-byte stores.
            if (it.ntiles > 0) {
                const long long gl = jt + it.ntiles - 1;
                if (!warp_wait(smem_u32(s.oready + (gl & 1)), (uint32_t)((gl >> 1) & 1), p.ctx, s.abort_flag)) break;
                tc::fence_after_sync();
            }
            // one split: normalise here, the head's sink logit (natural units ->
            // log2 units) joining the denominator; several: each split's rows are
            // divided by its own sum and the merge weighs them (and adds the sink)
            const float L = a.splits == 1
                                ? l + ((a.sinks && h < a.H) ? exp2f(__ldg(a.sinks + h) * 1.4426950408889634f - m_run) : 0.f)
                                : l;
            const float inv = L > 0.f ? 1.0f / L : 0.f;
            const int orow = (int)(a.splits == 1 ? it.bq : (long long)it.split * a.n_bq + it.bq);
            for (int c = 0; c < D; c += 64) {
                float v[32];
                if (it.ntiles > 0) {
                    tmem_ld_half32(tmem_o + lane_base + c, v);  // every lane (warp-collective)
                    tc::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0.f;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= inv;
                if (a.splits == 1 && a.rope_cos && c == D - kRopeDim) {
                    // conjugate rotation of the rotated slice (this 64-column slab):
                    // column i pairs with i + 32, held by the head's other thread
                    // (with several splits the merge rotates the merged row)
                    const bool first = kh == 0;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float pv = __shfl_xor_sync(0xffffffffu, v[i], 16);
                        const float2 cs = rope_cs(a, tq, i);
                        v[i] = first ? v[i] * cs.x + pv * cs.y : v[i] * cs.x - pv * cs.y;
                    }
                }
                if (a.splits > 1 && a.part_perm) {
                    // split partials in warp-store order (the merge reads them so): this
                    // warp's 16 heads x 64 columns of the slab as one 2 KiB block, piece
                    // j * 32 + lane, so that every store writes whole sectors
                    uint8_t *blk = reinterpret_cast<uint8_t *>(a.part_o + ((size_t)orow * a.H + it.head0) * D) +
                                   (size_t)(c / 64) * 8192 + (size_t)sp * 2048;
#pragma unroll
                    for (int j = 0; j < 4; ++j) reinterpret_cast<uint4 *>(blk)[j * 32 + lane] = pack8(v + 8 * j);
                } else if (h < a.H) {
                    uint16_t *dst = (a.splits == 1 ? a.out : a.part_o) + ((size_t)orow * a.H + h) * D + c + 32 * kh;
#pragma unroll
                    for (int j = 0; j < 4; ++j) reinterpret_cast<uint4 *>(dst)[j] = pack8(v + 8 * j);
                }
            }
            if (h < a.H && a.splits > 1 && kh == 0)
                a.part_ml[((size_t)it.split * a.n_bq + it.bq) * a.H + h] =
                    it.ntiles > 0 ? make_float2(m_run, l) : make_float2(-INFINITY, 0.f);
            jt += it.ntiles;
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// M = 64 instruction descriptor (kind::f16, bf16 operands, fp32 accumulate)
constexpr uint32_t idesc_m64(int n, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn ? (1u << 16) : 0u) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(64 >> 4) << 24);
}

template <int D, bool FP8>
int launch_d(const AttendArgs &a, const DevCtx &ctx, cudaStream_t st, bool pdl) {
    AttTcParams p = {};
    p.a = a;
    p.ctx = ctx;
    p.HH = (a.H + kHeads - 1) / kHeads;
    p.idesc_qk = idesc_m64(kTileKeys, false);
    p.idesc_pv = idesc_m64(Layout<D>::kPvN, true);
    p.n_work = a.n_bq * a.splits * p.HH;
    int stages = kMaxStages;
    while (stages > 2 && smem_bytes<D>(stages) > 225 * 1024) --stages;
    p.stages = stages;
    // at least 120 KiB so that one CTA owns an SM (it allocates all 512 TMEM columns)
    const size_t smem = std::max<size_t>(smem_bytes<D>(stages), 120 * 1024);
    auto kern = attend_tc_kernel<D, FP8>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return CSA_ERR_CUDA;
    CUtensorMap qmap;
    {
        const uint64_t dims[3] = {(uint64_t)D, (uint64_t)a.H, (uint64_t)a.n_bq};
        const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)a.H * D * 2};
        const uint32_t box[3] = {64, (uint32_t)kHeads, 1};
        if (!encode_tensor_map(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.q, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_128B))
            return CSA_ERR_CUDA;
    }
    CUtensorMap kvmap;
    memset(&kvmap, 0, sizeof(kvmap));
    p.kv_tma = a.dense && !FP8 ? 1 : 0;
    if (p.kv_tma) {
        // kv [batch][N][D] bf16: boxes of 64 dims x 64 entries, 128-byte swizzle
        const uint64_t dims[3] = {(uint64_t)D, (uint64_t)a.N, (uint64_t)(a.n_bq / a.nq)};
        const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)a.N * D * 2};
        const uint32_t box[3] = {64, (uint32_t)kTileKeys, 1};
        if (!encode_tensor_map(&kvmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.kv, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_128B))
            return CSA_ERR_CUDA;
    }
    const int grid = (int)std::min<long long>(p.n_work, num_sms());
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kern, qmap, kvmap, p) != cudaSuccess) return CSA_ERR_CUDA;
    return a.splits > 1 ? launch_attend_combine(a, st) : CSA_OK;
}

}  // namespace

bool attend_tc_supported(int H, int D) { return H >= 1 && H <= 128 && (D == 64 || D == 128 || D == 256 || D == 512); }

// Key splits per query: enough (query, split, head half) items to fill the
// SMs, chosen to minimise the tiles of the busiest CTA (plus a small per-item
// and per-split overhead).  The kernel deals each query's 64-key tiles to its
// splits in balanced contiguous ranges, so the plan only needs the count.
void attend_tc_plan(long long n_bq, int H, long long max_keys, int *splits, long long *kps) {
    const long long HH = (H + kHeads - 1) / kHeads;
    const long long ctas = num_sms();
    const long long tiles = (max_keys + kTileKeys - 1) / kTileKeys;
    long long best_cost = -1;
    int best = 1;
    for (int sp = 1; sp <= 64; ++sp) {
        const long long per = (tiles + sp - 1) / sp;
        const long long items = n_bq * HH * sp;
        const long long waves = (items + ctas - 1) / ctas;
        const long long cost = waves * (per + 3) + (sp > 1 ? 1 : 0);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = sp;
        }
        if (per <= 1) break;
    }
    *splits = best;
    *kps = ((tiles + best - 1) / best) * kTileKeys;
}

int launch_attend_tc(AttendArgs a, const DevCtx &ctx, cudaStream_t st, bool pdl) {
    if (a.kv8) {  // FP8 rows: 128-channel scale blocks
        switch (a.D) {
            case 128: return launch_d<128, true>(a, ctx, st, pdl);
            case 256: return launch_d<256, true>(a, ctx, st, pdl);
            case 512: return launch_d<512, true>(a, ctx, st, pdl);
            default: return CSA_ERR_UNSUPPORTED;
        }
    }
    switch (a.D) {
        case 64: return launch_d<64, false>(a, ctx, st, pdl);
        case 128: return launch_d<128, false>(a, ctx, st, pdl);
        case 256: return launch_d<256, false>(a, ctx, st, pdl);
        case 512: return launch_d<512, false>(a, ctx, st, pdl);
        default: return CSA_ERR_UNSUPPORTED;
    }
}

}  // namespace csa

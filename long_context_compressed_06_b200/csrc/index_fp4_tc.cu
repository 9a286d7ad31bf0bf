// index_fp4_tc.cu -- FP4 lightning-indexer scores on the 5th-generation tensor cores.
//
//   S[q][s] = sum_h w[q][h] * max(0, q_I[q][h] . K_I[s])   (s < n_vis(t_q), else -inf)
// with q_I and K_I stored as e2m1 codes and one e4m3 scale per 16 elements
// ("DeepSeek V4 paper full version is out, FP4 QAT details" -- FP4 activations
// in the indexer QK path; techniques map, "inference quantization").
//
// An e2m1 value (at most 2 significant bits) times an e4m3 scale (4 significant
// bits) has at most 5 significant bits and lies within f16's normal range, so
// dequantising to f16 (hardware e2m1x2 / e4m3x2 conversions and one f16x2
// multiply per pair) is exact; the scores then come from an f16 tensor-core
// contraction with fp32 accumulation, and differ from the exact FP4 dot
// products only by the fp32 summation order.  HBM moves
// 72 bytes per key (64 packed + 8 scale bytes at d_I = 128) instead of 256.
//
// Warp roles (320 threads): warp 0 -- producer: TMA of the packed key rows and
// cp.async of their scales into a ring of raw stages; warp 1 -- TMEM owner and
// MMA issuer (lane 0 issues through guarded instructions); warps 2..5 --
// epilogue (tcgen05.ld, ReLU, weighted head sum, causal mask, store); warps
// 6..9 -- dequantisation of raw stages into the 128-byte-swizzled f16 tiles
// the MMA reads, and of each query group's indexer heads.  Every wait is
// bounded and every role warp stays converged (all lanes poll).
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int kThreads = 320;
constexpr int kTileKeys = 128;
constexpr int kMaxRaw = 12;
constexpr int kMaxStages = 4;

struct Fp4TcParams {
    const uint8_t *k4s;   // [batch][N][d_I/16] key scales (e4m3)
    const uint8_t *q4;    // [batch][nq][H_I][d_I/2]
    const uint8_t *q4s;   // [batch][nq][H_I][d_I/16]
    const float *w;       // [batch][nq][H_I]
    const int *q_pos;     // [batch][nq]
    float *scores;        // [batch][nq][N]
    long long N;
    int nq, H_I, H_pad, d_I, m, NQ;
    int groups_per_batch, n_ktiles;
    long long total_work;
    int raw_stages, stages, nchunk;
    uint32_t raw_bytes, pk_bytes, stage_bytes, q_bytes, idesc;
    int n_cols, n_acc;
    uint32_t tmem_cols;
    DevCtx ctx;
};

struct Cursor {
    long long w;
    int kt, g, b;
};

CSA_DEVINL Cursor cursor_at(const Fp4TcParams &p, long long w) {
    Cursor c;
    c.w = w;
    const long long grp = w / p.n_ktiles;
    c.kt = (int)(w - grp * p.n_ktiles);
    c.b = (int)(grp / p.groups_per_batch);
    c.g = (int)(grp - (long long)c.b * p.groups_per_batch);
    return c;
}

CSA_DEVINL void advance(const Fp4TcParams &p, Cursor &c) {
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

// Two e2m1 codes (element 2i in the low nibble) -> f16x2 (low half = element
// 2i), and two e4m3 codes -> f16x2; both conversions are exact.
CSA_DEVINL uint32_t e2m1x2_f16x2(uint32_t byte) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(r) : "r"(byte));
    return r;
}

CSA_DEVINL uint32_t e4m3x2_f16x2(uint32_t two) {
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"((uint16_t)two));
    return r;
}

CSA_DEVINL uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// 32 consecutive elements: 16 packed bytes and their two scales -> four
// 16-byte units of f16.  Every product (at most 5 significant bits, magnitude
// in [2^-10, 2688]) is exact in f16, so the operands the MMA sees are exactly
// the dequantised FP4 values.
CSA_DEVINL void dequant32(uint4 pk, uint32_t s01, uint4 out[4]) {
    const uint32_t sc = e4m3x2_f16x2(s01);
    const uint32_t s0 = (sc & 0xffffu) * 0x10001u, s1 = (sc >> 16) * 0x10001u;
    const uint32_t wds[4] = {pk.x, pk.y, pk.z, pk.w};
    uint32_t r[16];
#pragma unroll
    for (int wd = 0; wd < 4; ++wd)
#pragma unroll
        for (int j = 0; j < 4; ++j) r[wd * 4 + j] = hmul2(e2m1x2_f16x2(wds[wd] >> (8 * j)), wd < 2 ? s0 : s1);
    out[0] = make_uint4(r[0], r[1], r[2], r[3]);
    out[1] = make_uint4(r[4], r[5], r[6], r[7]);
    out[2] = make_uint4(r[8], r[9], r[10], r[11]);
    out[3] = make_uint4(r[12], r[13], r[14], r[15]);
}

// Byte offset of 16-byte unit u (0..7) of row r in a 128-byte-swizzled chunk.
CSA_DEVINL uint32_t sw128(int r, int u) { return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4)); }

__global__ void __launch_bounds__(kThreads, 1)
    index_fp4_tc_kernel(const __grid_constant__ CUtensorMap kmap, const Fp4TcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned carve-up: bf16 key stages | bf16 query tile | raw stages | weights | barriers
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *k_smem = base;
    uint8_t *q_smem = k_smem + (size_t)p.stages * p.stage_bytes;
    uint8_t *raw = q_smem + p.q_bytes;                                    // [raw_stages][packed | scales]
    float *w_s = reinterpret_cast<float *>(raw + (size_t)p.raw_stages * p.raw_bytes);  // [NQ][H_pad]
    int *nvis_s = reinterpret_cast<int *>(w_s + p.NQ * p.H_pad);          // [NQ]
    uint64_t *bars = reinterpret_cast<uint64_t *>(
        (reinterpret_cast<uintptr_t>(nvis_s + p.NQ) + 7) & ~uintptr_t(7));
    uint64_t *rfull = bars, *rempty = rfull + kMaxRaw;
    uint64_t *full = rempty + kMaxRaw, *empty = full + kMaxStages;
    uint64_t *tfull = empty + kMaxStages, *tempty = tfull + 4;
    uint64_t *qfull = tempty + 4, *qempty = qfull + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(qempty + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long w0 = (long long)blockIdx.x * p.total_work / gridDim.x;
    const long long w1 = (long long)(blockIdx.x + 1) * p.total_work / gridDim.x;
    const int sbytes = p.d_I / 16;  // scale bytes per key row

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.raw_stages; ++s) {
            mbar_init(rfull + s, 1 + 32);  // expect_tx arrive + one cp.async arrive per producer lane
            mbar_init(rempty + s, 4);
        }
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(full + s, 4);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < p.n_acc; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, 4);
        }
        mbar_init(qfull, 4);
        mbar_init(qempty, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tc::prefetch_tmap(&kmap);
    }
    if (warp == 1) {
        tc::tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const auto wait_all = [&](uint64_t *bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), parity, p.ctx, abort_flag));
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        Ring rr;
        long long it = 0;
        for (Cursor cu = cursor_at(p, w0); cu.w < w1; advance(p, cu)) {
            const int rs = rr.idx;
            if (!wait_all(rempty + rs, rr.phase ^ 1u)) break;
            uint8_t *dst = raw + (size_t)rs * p.raw_bytes;
            mbar_arrive_expect_tx(smem_u32(rfull + rs), p.pk_bytes, lane == 0);
            tc::tma_load_3d(smem_u32(dst), &kmap, smem_u32(rfull + rs), 0, cu.kt * kTileKeys, cu.b, lane == 0);
            // scales: rows past N read the last row (their scores are never stored)
            uint8_t *sdst = dst + p.pk_bytes;
            for (int r = lane; r < kTileKeys; r += 32) {
                const long long key = std::min((long long)cu.kt * kTileKeys + r, p.N - 1);
                const uint8_t *src = p.k4s + ((size_t)cu.b * p.N + key) * sbytes;
                const uint32_t d = smem_u32(sdst + r * sbytes);
                if (sbytes == 16)
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
                else if (sbytes == 8)
                    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(d), "l"(src) : "memory");
                else
                    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(src) : "memory");
            }
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(rfull + rs))
                         : "memory");
            rr.next(p.raw_stages);
            ++it;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        // drain: the TMA copies issued last into each raw stage
        for (long long j = std::max(0LL, it - p.raw_stages); j < it; ++j)
            mbar_wait(smem_u32(rfull + (j % p.raw_stages)), (uint32_t)((j / p.raw_stages) & 1), p.ctx, nullptr);
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        long long gi = 0;
        Ring kr, ar;
        const uint32_t sbo = 8u * 128u;
        const uint64_t kdesc0 = tc::smem_desc(smem_u32(k_smem), sbo, tc::kLayoutSw128);
        const uint64_t qdesc0 = tc::smem_desc(smem_u32(q_smem), sbo, tc::kLayoutSw128);
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
            const uint32_t d_tmem = tmem_base + (uint32_t)(acc * p.n_cols);
            const uint64_t kd = kdesc0 + ((uint64_t)(st * p.stage_bytes) >> 4);
            uint32_t accumulate = 0;
            for (int c = 0; c < p.nchunk; ++c) {
                for (int kk = 0; kk < 4; ++kk) {
                    tc::mma_f16(d_tmem, kd + ((uint32_t)(c * kTileKeys * 128 + kk * 32) >> 4),
                                qdesc0 + ((uint32_t)(c * p.n_cols * 128 + kk * 32) >> 4), p.idesc, accumulate,
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
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue (warps 2..5)
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int row = quarter * 32 + lane;
        const int et = threadIdx.x - 64;  // 0..127
        Ring ar;
        for (Cursor cu = cursor_at(p, w0); cu.w < w1; advance(p, cu)) {
            const int b = cu.b, g = cu.g;
            if (cu.w == w0 || cu.kt == 0) {
                asm volatile("bar.sync 1, 128;" ::: "memory");
                for (int i = et; i < p.NQ * p.H_pad; i += 128) {
                    const int qi = i / p.H_pad, h = i - qi * p.H_pad;
                    const int q = g * p.NQ + qi;
                    w_s[i] = (q < p.nq && h < p.H_I) ? __ldg(p.w + ((size_t)b * p.nq + q) * p.H_I + h) : 0.f;
                }
                for (int qi = et; qi < p.NQ; qi += 128) {
                    const int q = g * p.NQ + qi;
                    nvis_s[qi] = q < p.nq ? (int)n_visible(__ldg(p.q_pos + (size_t)b * p.nq + q), p.m, p.N) : 0;
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
            }
            const int acc = ar.idx;
            if (!wait_all(tfull + acc, ar.phase)) break;
            tc::fence_after_sync();
            const long long s = (long long)cu.kt * kTileKeys + row;
            const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * p.n_cols);
            for (int qi = 0; qi < p.NQ; ++qi) {
                const int q = g * p.NQ + qi;
                if (q >= p.nq) break;
                float part[4] = {0.f, 0.f, 0.f, 0.f};
                for (int hc = 0; hc < p.H_pad; hc += 64) {
                    float v[64];
                    const int nl = min(4, (p.H_pad - hc) >> 4);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (u < nl) tc::tmem_ld16(tbase + (uint32_t)(qi * p.H_pad + hc + 16 * u), v + 16 * u);
                    tc::tmem_wait_ld();
                    const float *ws = w_s + qi * p.H_pad + hc;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (u < nl) {
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                part[u] = fmaf(ws[16 * u + i], fmaxf(v[16 * u + i], 0.f), part[u]);
                        }
                }
                const float score = (part[0] + part[1]) + (part[2] + part[3]);
                if (s < p.N) p.scores[((size_t)b * p.nq + q) * p.N + s] = s < nvis_s[qi] ? score : -INFINITY;
            }
            tc::fence_before_sync();
            __syncwarp();
            mbar_arrive(smem_u32(tempty + acc), lane == 0);
            ar.next(p.n_acc);
        }
    } else {
        // ------------------------------------------------------------ dequantisation (warps 6..9)
        // Thread (row, u): 32 elements of a key row -- one 16-byte packed unit and
        // its two scales -- into four bf16 units of the swizzled tile.  A warp
        // instruction covers consecutive packed bytes and conflict-free stores.
        const int dt = threadIdx.x - 192;  // 0..127
        const int upr = p.d_I / 32;        // packed 16-byte units per row
        Ring rr, kr;
        long long gi = 0;
        for (Cursor cu = cursor_at(p, w0); cu.w < w1; advance(p, cu)) {
            if (cu.w == w0 || cu.kt == 0) {
                // this query group's indexer heads, once the previous group's MMAs are done with them
                if (gi > 0 && !wait_all(qempty, (uint32_t)((gi - 1) & 1))) break;
                const int rows = p.NQ * p.H_pad;
                for (int i = dt; i < rows * upr; i += 128) {
                    const int r = i / upr, u = i - r * upr;
                    const int qi = r / p.H_pad, h = r - qi * p.H_pad;
                    const int q = cu.g * p.NQ + qi;
                    uint4 out[4] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u),
                                    make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
                    if (q < p.nq && h < p.H_I) {
                        const size_t hr = ((size_t)cu.b * p.nq + q) * p.H_I + h;
                        const uint4 pk = __ldg(reinterpret_cast<const uint4 *>(p.q4 + hr * (p.d_I / 2) + u * 16));
                        const uint32_t s01 = *reinterpret_cast<const uint16_t *>(p.q4s + hr * sbytes + 2 * u);
                        dequant32(pk, s01, out);
                    }
                    uint8_t *qc = q_smem + (size_t)(u >> 1) * p.n_cols * 128;
#pragma unroll
                    for (int j = 0; j < 4; ++j) *reinterpret_cast<uint4 *>(qc + sw128(r, (u & 1) * 4 + j)) = out[j];
                }
                tc::fence_proxy_async_smem();
                __syncwarp();
                mbar_arrive(smem_u32(qfull), lane == 0);
                ++gi;
            }
            const int rs = rr.idx, st = kr.idx;
            if (!wait_all(rfull + rs, rr.phase)) break;
            if (!wait_all(empty + st, kr.phase ^ 1u)) break;
            const uint8_t *src = raw + (size_t)rs * p.raw_bytes;
            const uint8_t *ssrc = src + p.pk_bytes;
            uint8_t *dst = k_smem + (size_t)st * p.stage_bytes;
            for (int i = dt; i < kTileKeys * upr; i += 128) {
                const int r = i / upr, u = i - r * upr;
                const uint4 pk = *reinterpret_cast<const uint4 *>(src + r * (p.d_I / 2) + u * 16);
                const uint32_t s01 = *reinterpret_cast<const uint16_t *>(ssrc + r * sbytes + 2 * u);
                uint4 out[4];
                dequant32(pk, s01, out);
                uint8_t *kc = dst + (size_t)(u >> 1) * kTileKeys * 128;
#pragma unroll
                for (int j = 0; j < 4; ++j) *reinterpret_cast<uint4 *>(kc + sw128(r, (u & 1) * 4 + j)) = out[j];
            }
            tc::fence_proxy_async_smem();
            __syncwarp();
            mbar_arrive(smem_u32(full + st), lane == 0);
            mbar_arrive(smem_u32(rempty + rs), lane == 0);
            rr.next(p.raw_stages);
            kr.next(p.stages);
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

// The tensor-core path takes d_I in {64, 128, 256} and up to 256 heads.
bool index_fp4_tc_supported(int H_I, int d_I) {
    return (d_I == 64 || d_I == 128 || d_I == 256) && H_I >= 1 && H_I <= 256;
}

int launch_index_fp4_tc(const uint8_t *q4, const uint8_t *q4s, const float *w, const uint8_t *k4,
                        const uint8_t *k4s, const int *q_pos, int batch, int nq, long long N, int H_I, int d_I,
                        int m, float *scores, const DevCtx &ctx, cudaStream_t st) {
    Fp4TcParams p = {};
    p.k4s = k4s; p.q4 = q4; p.q4s = q4s; p.w = w; p.q_pos = q_pos; p.scores = scores;
    p.N = N; p.nq = nq; p.H_I = H_I; p.d_I = d_I; p.m = m; p.ctx = ctx;
    p.H_pad = std::max(16, (H_I + 15) / 16 * 16);
    p.nchunk = d_I / 64;
    p.stage_bytes = (uint32_t)(kTileKeys * d_I * 2);
    p.pk_bytes = (uint32_t)(kTileKeys * (d_I / 2));
    p.raw_bytes = (p.pk_bytes + kTileKeys * (d_I / 16) + 1023u) & ~1023u;
    const size_t smem_cap = 200 * 1024;
    p.stages = 2;
    int NQ = std::max(1, std::min(nq, std::min(16, 256 / p.H_pad)));
    while (NQ > 1 && (size_t)NQ * p.H_pad * d_I * 2 + (size_t)p.stages * p.stage_bytes + 4 * p.raw_bytes > smem_cap)
        NQ /= 2;
    p.NQ = NQ;
    p.n_cols = NQ * p.H_pad;
    p.q_bytes = (uint32_t)(p.n_cols * d_I * 2);
    const size_t fixed = (size_t)p.q_bytes + (size_t)p.stages * p.stage_bytes;
    if (fixed >= smem_cap) return CSA_ERR_UNSUPPORTED;
    p.raw_stages = (int)std::min<size_t>(kMaxRaw, (smem_cap - fixed) / p.raw_bytes);
    if (p.raw_stages < 2) return CSA_ERR_UNSUPPORTED;
    p.idesc = tc::idesc_f16(p.n_cols, false);  // f16 operands
    p.n_acc = p.n_cols <= 128 ? 4 : 2;
    uint32_t cols = 32;
    while (cols < (uint32_t)(p.n_acc * p.n_cols)) cols *= 2;
    p.tmem_cols = cols;
    p.groups_per_batch = (nq + NQ - 1) / NQ;
    p.n_ktiles = (int)((N + kTileKeys - 1) / kTileKeys);
    p.total_work = (long long)batch * p.groups_per_batch * p.n_ktiles;

    CUtensorMap kmap;
    {
        const uint64_t dims[3] = {(uint64_t)(d_I / 2), (uint64_t)N, (uint64_t)batch};
        const uint64_t strides[2] = {(uint64_t)(d_I / 2), (uint64_t)N * (d_I / 2)};
        const uint32_t box[3] = {(uint32_t)(d_I / 2), (uint32_t)kTileKeys, 1};
        if (!encode_tensor_map(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, k4, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_NONE))
            return CSA_ERR_CUDA;
    }
    const size_t smem = 1024 + fixed + (size_t)p.raw_stages * p.raw_bytes + (size_t)NQ * p.H_pad * 4 + NQ * 4 + 8 +
                        (2 * kMaxRaw + 2 * kMaxStages + 10) * 8 + 16;
    if (cudaFuncSetAttribute(index_fp4_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return CSA_ERR_CUDA;
    const int grid = (int)std::min<long long>(p.total_work, num_sms());
    index_fp4_tc_kernel<<<grid, kThreads, smem, st>>>(kmap, p);
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // namespace csa

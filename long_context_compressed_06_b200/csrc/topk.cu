// topk.cu -- causal top-k selector (csa_topk).
//
// For each query, the k largest scores among its n_vis(t) visible entries,
// ties broken towards the lower index; invalid slots are -1 ("DeepSeek v4"
// -> top-k selector; techniques map: indices at or beyond the causal threshold
// become -1).  Output indices are in ascending order.
//
// Design: one query is handled by one CTA of 1024 threads or, for long rows
// and for small batches, by a thread-block cluster of CS CTAs; each thread
// keeps R consecutive scores (CS*1024*R >= N) in registers as order-preserving
// uint32 keys, so the scores are read from memory once.
//
// First pass: a histogram over 1024 bins linear in the score between the
// smallest and largest visible score (pushed by every CTA into every other's
// shared memory before one cluster barrier).  The threshold bin -- the bin that
// holds the k-th largest score -- then has few keys: every key above it is
// selected, and the keys inside it (at most 256) are pushed, with the per-CTA
// counts, into every CTA's shared memory, where each CTA ranks them directly
// (score descending, index ascending; up to 32 of them by one warp with
// shuffles and a ballot, more by the whole block) and writes its own selected
// indices in index order.  After that barrier no CTA touches another's memory.
// Every block scan takes one block barrier (each warp scans the warp totals).
//
// The value-linear pass runs at up to 8 keys per thread (the decode batches);
// longer rows per thread, a non-finite score range, or a threshold bin above
// 256 keys take the exact radix select instead: digits of 11 key bits per
// pass, from the highest bit where the smallest and largest key differ, with
// per-CTA shared-memory histograms
// read by the peers through distributed shared memory after a cluster barrier;
// it stops once the threshold bin holds exactly the number still needed, and
// compacts stably (block scan plus a cluster scan over the CTA totals).
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace csa {
namespace {

constexpr int kTopkThreads = 1024;
constexpr int kBins = 2048;      // bins of a radix pass over the key bits (two per thread)
constexpr int kLinBins = 1024;   // bins of the value-linear pass (one per thread)
constexpr int kCandCap = 256;    // threshold-bin keys ranked directly (larger bins: radix passes)
constexpr int kMaxCluster = 16;  // CTAs per query at most

// order-preserving map fp32 -> uint32 (-0 folded onto +0)
CSA_DEVINL uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// its inverse (the score of a key, -0 read back as +0)
CSA_DEVINL float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Inclusive scan over the 1024 threads (32 warps) of the block; returns this
// thread's inclusive prefix and writes the block total to *total.  One block
// barrier: every warp scans the 32 warp totals itself.  The caller places a
// block barrier between this scan and the next write of warp_buf.
template <typename T>
CSA_DEVINL T block_scan_incl(T v, T *warp_buf, T *total) {
    static_assert(kTopkThreads == 1024, "one warp total per lane");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const T n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) warp_buf[warp] = v;
    __syncthreads();
    T w = warp_buf[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const T n = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += n;
    }
    const T before = __shfl_sync(0xffffffffu, w, (warp + 31) & 31);  // warps below this one
    *total = __shfl_sync(0xffffffffu, w, 31);
    return warp > 0 ? v + before : v;
}

// Value-linear digit of a key: floor((v - vmin) * scale), capped at the last bin.
// Rounded subtraction and multiplication by a positive constant preserve order,
// so the digit is non-decreasing in the key; the explicit roundings keep it the
// same function of the key in every thread.
CSA_DEVINL int lin_digit(uint32_t key, float vmin, float scale) {
    const float x = __fmul_rn(__fsub_rn(key_value(key), vmin), scale);
    return __float2int_rz(fminf(x, (float)(kLinBins - 1)));
}

// CL: the query's row is split over a cluster of CS CTAs (ranges, candidates
// and counts pushed into every rank's shared memory, histograms read through
// distributed shared memory, cluster barriers); without it one CTA holds the
// row and every barrier is a block barrier.
template <int R, bool CL>
__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(const float *__restrict__ scores,
                                                               const int *__restrict__ q_pos, long long N,
                                                               int m, int k, int *__restrict__ idx, int CS) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = CL ? (int)cluster.block_rank() : 0;
    const long long bq = blockIdx.x / CS;
    const auto sync_all = [&]() {
        if constexpr (CL) cluster.sync(); else __syncthreads();
    };
    const auto peer = [&](auto *p, int r) {
        if constexpr (CL) return cluster.map_shared_rank(p, r); else return p;
    };
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    __shared__ __align__(8) uint32_t hist[2][kBins];  // this CTA's histogram, double-buffered over passes
    __shared__ uint32_t warp_u32[32];
    __shared__ unsigned long long warp_u64[32];
    __shared__ unsigned long long cta_total;           // radix passes: (gt << 32) | eq, read by higher ranks
    __shared__ uint32_t r_min[kMaxCluster], r_max[kMaxCluster];  // every rank's key range (pushed by that rank)
    __shared__ unsigned long long r_tot[kMaxCluster];  // every rank's (above << 32) | in-bin counts (pushed)
    __shared__ uint32_t seg_key[kMaxCluster][kCandCap];  // every rank's threshold-bin keys in index order (pushed)
    __shared__ uint32_t all_key[kCandCap];              // the segments concatenated (index order)
    __shared__ uint32_t rank_part[kTopkThreads / kCandCap][kCandCap];
    __shared__ uint32_t sel_pre[kCandCap + 1];          // selected among the first x candidates
    __shared__ uint32_t s_off[kMaxCluster + 1];         // list offset of each rank, then the total
    __shared__ uint32_t s_bin, s_cnt;
    __shared__ long long s_krem, s_above_before;

    // as a programmatic dependent: the scores are complete only once the
    // predecessor grid is (a no-op otherwise); the successor may launch now
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int i = threadIdx.x; i < 2 * kBins; i += kTopkThreads) (&hist[0][0])[i] = 0u;

    // the score loads do not wait for the query position (they stay inside the
    // row); entries past n_vis are masked afterwards
    const int t_q = q_pos ? __ldg(q_pos + bq) : 0;
    const long long seg0 = ((long long)rank * kTopkThreads + threadIdx.x) * R;
    const int nrow = (int)(N - seg0 <= 0 ? 0 : (N - seg0 >= R ? R : N - seg0));
    uint32_t key[R];
    const float *row = scores + bq * N;
    if (nrow == R && (N & 3) == 0) {
#pragma unroll
        for (int r = 0; r < R; r += 4) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(row + seg0 + r));
            key[r] = order_key(v.x); key[r + 1] = order_key(v.y);
            key[r + 2] = order_key(v.z); key[r + 3] = order_key(v.w);
        }
    } else {
#pragma unroll
        for (int r = 0; r < R; ++r) key[r] = r < nrow ? order_key(__ldg(row + seg0 + r)) : 0u;
    }
    // visible entries floor((t + 1) / m) clipped to [0, N] (no q_pos: every entry), in 32-bit arithmetic
    long long nv = N;
    if (q_pos) {
        const long long v = t_q < 0 ? 0 : (long long)(((uint32_t)t_q + 1u) / (uint32_t)m);
        nv = v < N ? v : N;
    }
    const long long kk = nv < k ? nv : k;
    const int nloc = (int)(nv - seg0 <= 0 ? 0 : (nv - seg0 >= R ? R : nv - seg0));

    // key range of the visible entries, pushed into every rank
    uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
    for (int r = 0; r < R; ++r)
        if (r < nloc) {
            kmin = min(kmin, key[r]);
            kmax = max(kmax, key[r]);
        }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
        warp_u32[warp] = kmin;
        reinterpret_cast<uint32_t *>(warp_u64)[warp] = kmax;
    }
    __syncthreads();
    if (warp == 0) {
        const uint32_t a = __reduce_min_sync(0xffffffffu, warp_u32[lane]);
        const uint32_t b = __reduce_max_sync(0xffffffffu, reinterpret_cast<uint32_t *>(warp_u64)[lane]);
        if (lane < CS) {
            *peer(&r_min[rank], lane) = a;
            *peer(&r_max[rank], lane) = b;
        }
    }
    sync_all();  // every rank's range delivered, histograms cleared
    uint32_t gmin = 0xffffffffu, gmax = 0u;
    for (int r2 = 0; r2 < CS; ++r2) {
        gmin = min(gmin, r_min[r2]);
        gmax = max(gmax, r_max[r2]);
    }

    // Threshold bin of the cluster-wide 2048-bin histogram in hloc (every rank's
    // copy): the highest bin b with (count above b) < krem_in <= (count above b)
    // + count(b), into s_bin, s_cnt and s_krem (what is still needed from b).
    const auto find_bin = [&](const uint32_t *hloc, long long krem_in) {
        uint32_t c_lo = 0u, c_hi = 0u;
        for (int r0 = 0; r0 < CS; r0 += 4) {
            uint2 v[4];  // this thread's two bins of up to four ranks, loads issued together
#pragma unroll
            for (int j = 0; j < 4; ++j)
                v[j] = r0 + j < CS ? *reinterpret_cast<const uint2 *>(peer(hloc, r0 + j) + 2 * threadIdx.x)
                                   : make_uint2(0u, 0u);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                c_lo += v[j].x;
                c_hi += v[j].y;
            }
        }
        uint32_t tot;
        const uint32_t incl = block_scan_incl<uint32_t>(c_lo + c_hi, warp_u32, &tot);
        const long long above = (long long)tot - incl;  // count in bins of higher threads
        if (above < krem_in && above + c_hi >= krem_in) {
            s_bin = 2 * threadIdx.x + 1; s_cnt = c_hi; s_krem = krem_in - above;
        } else if (above + c_hi < krem_in && above + c_hi + c_lo >= krem_in) {
            s_bin = 2 * threadIdx.x; s_cnt = c_lo; s_krem = krem_in - above - c_hi;
        }
        __syncthreads();
    };

    uint32_t prefix = 0u, mask = 0u;
    long long krem = kk;
    bool done = nv <= k;  // every visible entry is selected
    int top = -1;
    bool lin = false;     // value-linear first pass possible (finite, distinct range)
    float vmin = 0.f, lscale = 0.f;
    if (!done) {
        if (gmin == gmax) {
            prefix = gmax;
            mask = 0xffffffffu;  // all keys equal: the lowest indices win
            done = true;
        } else {
            top = 31 - __clz(gmin ^ gmax);
            mask = top == 31 ? 0u : ~((2u << top) - 1u);
            prefix = gmax & mask;
            vmin = key_value(gmin);
            const float vmax = key_value(gmax);
            const float range = __fsub_rn(vmax, vmin);
            lscale = __fdividef((float)kLinBins, range);  // any value: every thread computes the same
            // Only with few keys per thread (their digits then stay in registers):
            // at 16 or 32 keys per thread the radix passes measured faster
            // (prefill rows 0.28 vs 0.37 ms, 262144-entry rows 29 vs 45 us).
            lin = R <= 8 && isfinite(vmin) && isfinite(vmax) && isfinite(range) && range > 0.f && isfinite(lscale);
        }
    }
    // Pass 1: bins linear in the score between the smallest and largest visible
    // score.  Scores bunch in a few binary exponents, so bins taken from the key
    // bits would pile most keys into a handful of bins (shared-memory atomics on
    // one address serialise); linear bins spread them, and the threshold bin
    // holds few keys.  Those candidates are ranked directly below.
    int p0 = 0;
    int t1 = 0;
    // the value-linear digits, two per register, kept when the registers allow
    // (1024 threads have 64 each); otherwise recomputed from the keys
    constexpr bool kKeepDigits = R <= 8;
    uint32_t dg[kKeepDigits ? R / 2 : 1];
    const auto digit = [&](int r) -> int {
        if constexpr (kKeepDigits) return (int)((dg[r / 2] >> (16 * (r & 1))) & 0xffffu);
        else return lin_digit(key[r], vmin, lscale);
    };
    if (lin) {
        if constexpr (kKeepDigits) {
#pragma unroll
            for (int r = 0; r < R; r += 2) {
                const uint32_t d0 = (uint32_t)lin_digit(key[r], vmin, lscale);
                const uint32_t d1 = (uint32_t)lin_digit(key[r + 1], vmin, lscale);
                dg[r / 2] = d0 | (d1 << 16);
                if (r < nloc) atomicAdd(&hist[0][d0], 1u);
                if (r + 1 < nloc) atomicAdd(&hist[0][d1], 1u);
            }
        } else {
#pragma unroll
            for (int r = 0; r < R; ++r)
                if (r < nloc) atomicAdd(&hist[0][lin_digit(key[r], vmin, lscale)], 1u);
        }
        sync_all();  // every CTA's histogram is complete
        // cluster-wide count of bin threadIdx.x (one bin per thread)
        uint32_t c = 0u;
        for (int r0 = 0; r0 < CS; r0 += 8) {
            uint32_t v[8];  // up to eight ranks' loads in flight
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = r0 + j < CS ? *peer(&hist[0][threadIdx.x], r0 + j) : 0u;
#pragma unroll
            for (int j = 0; j < 8; ++j) c += v[j];
        }
        uint32_t tot;
        const uint32_t incl = block_scan_incl<uint32_t>(c, warp_u32, &tot);
        const long long above = (long long)tot - incl;
        if (above < krem && above + c >= krem) {
            s_bin = threadIdx.x;
            s_cnt = c;
            s_krem = krem - above;
        }
        __syncthreads();
        p0 = 1;  // a radix pass after this one starts on the other buffer
        lin = s_cnt <= (uint32_t)kCandCap;  // the same cluster-wide count in every CTA
        if (lin) {
            t1 = (int)s_bin;
            krem = s_krem;
        }
    }

    int *out = idx + bq * k;
    if (lin) {
        // ------------------------------------------------ threshold bin ranked directly
        uint32_t n_above = 0u, n_in = 0u;
#pragma unroll
        for (int r = 0; r < R; ++r)
            if (r < nloc) {
                const int d = digit(r);
                n_above += d > t1;
                n_in += d == t1;
            }
        // (above << 16) | in-bin: a CTA holds at most 1024 * 8 keys on this path
        uint32_t blk_tot;
        const uint32_t mine = (n_above << 16) | n_in;
        const uint32_t excl = block_scan_incl<uint32_t>(mine, warp_u32, &blk_tot) - mine;
        // this CTA's candidates into its segment of every rank's list, in index order
        uint32_t cp = excl & 0xffffu;
#pragma unroll
        for (int r = 0; r < R; ++r)
            if (r < nloc && digit(r) == t1) {
                for (int r2 = 0; r2 < CS; ++r2) *peer(&seg_key[rank][cp], r2) = key[r];
                ++cp;
            }
        if ((int)threadIdx.x < CS)
            *peer(&r_tot[rank], (int)threadIdx.x) = ((unsigned long long)(blk_tot >> 16) << 32) | (blk_tot & 0xffffu);
        // every rank's candidates and counts delivered; from here on no CTA
        // touches another's shared memory, so none waits for the others to exit
        sync_all();
        // the candidate count, the same in every CTA
        uint32_t C = 0u;
        for (int r2 = 0; r2 < CS; ++r2) C += (uint32_t)r_tot[r2];
        if (warp == 0) {
            // prefix over ranks of the (above, in-bin) counts: list offsets, and the
            // keys above the bin in lower ranks (this rank's first output slot)
            const unsigned long long t = lane < CS ? r_tot[lane] : 0ull;
            unsigned long long inc = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long n = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += n;
            }
            if (lane < CS) s_off[lane] = (uint32_t)(inc - t);
            if (lane == CS - 1) s_off[CS] = (uint32_t)inc;
            if (lane == rank) s_above_before = (long long)((inc - t) >> 32);
            if (C <= 32u) {
                // up to 32 candidates: one warp gathers, ranks and counts them
                __syncwarp();
                // candidate `lane` lies in the segment of the last rank whose offset is <= lane
                const uint32_t my_off = (uint32_t)(inc - t);
                int r2 = 0;
#pragma unroll
                for (int j = 1; j < kMaxCluster; ++j) {
                    const uint32_t off_j = __shfl_sync(0xffffffffu, my_off, j);
                    r2 += j < CS && off_j <= (uint32_t)lane;
                }
                const int seg_start = (int)__shfl_sync(0xffffffffu, my_off, r2);  // every lane takes part
                const uint32_t ki = (uint32_t)lane < C ? seg_key[r2][lane - seg_start] : 0u;
                uint32_t rk = 0u;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const uint32_t kj = __shfl_sync(0xffffffffu, ki, j);
                    rk += j < (int)C && ((kj > ki) || (kj == ki && j < lane));
                }
                const uint32_t selb = __ballot_sync(0xffffffffu, (uint32_t)lane < C && (long long)rk < krem);
                if ((uint32_t)lane < C) sel_pre[lane + 1] = __popc(selb & (0xffffffffu >> (31 - lane)));
                if (lane == 0) sel_pre[0] = 0u;
            }
        }
        __syncthreads();
        if (C > 32u) {
            for (int i = threadIdx.x; i < (int)C; i += kTopkThreads) {
                int r2 = 0;
                while (r2 + 1 < CS && s_off[r2 + 1] <= (uint32_t)i) ++r2;
                all_key[i] = seg_key[r2][i - (int)s_off[r2]];
            }
            __syncthreads();
            {
                // candidates preceding candidate i in (score desc, index asc), counted
                // over four slices of the list by four threads
                constexpr int kParts = kTopkThreads / kCandCap;
                const int i = threadIdx.x % kCandCap, part = threadIdx.x / kCandCap;
                if (i < (int)C) {
                    const int chunk = ((int)C + kParts - 1) / kParts;
                    const int j0 = part * chunk, j1 = min((int)C, j0 + chunk);
                    const uint32_t ki = all_key[i];
                    uint32_t cnt = 0u;
                    for (int j = j0; j < j1; ++j) {
                        const uint32_t kj = all_key[j];
                        cnt += (kj > ki) || (kj == ki && j < i);
                    }
                    rank_part[part][i] = cnt;
                }
            }
            __syncthreads();
            uint32_t sel = 0u;
            if ((int)threadIdx.x < (int)C) {
                uint32_t rk = 0u;
#pragma unroll
                for (int q = 0; q < kTopkThreads / kCandCap; ++q) rk += rank_part[q][threadIdx.x];
                sel = (long long)rk < krem;
            }
            uint32_t sel_tot;
            const uint32_t sel_incl = block_scan_incl<uint32_t>(sel, warp_u32, &sel_tot);
            if ((int)threadIdx.x < (int)C) sel_pre[threadIdx.x + 1] = sel_incl;
            if (threadIdx.x == 0) sel_pre[0] = 0u;
            __syncthreads();
        }
        // outputs in index order: keys above the threshold bin and selected candidates
        uint32_t ci = s_off[rank] + (excl & 0xffffu);
        int pos = (int)s_above_before + (int)(excl >> 16) + (int)sel_pre[ci];
        const int kk32 = (int)kk;
#pragma unroll
        for (int r = 0; r < R; ++r)
            if (r < nloc) {
                const int d = digit(r);
                // pos < kk by construction (kk - krem keys above the bin, krem selected in it)
                if (d > t1 || (d == t1 && sel_pre[ci + 1] != sel_pre[ci])) {
                    if (pos < kk32) out[pos] = (int)(seg0 + r);
                    ++pos;
                }
                ci += d == t1;
            }
        if (rank == 0)
            for (long long i = kk + threadIdx.x; i < k; i += kTopkThreads) out[i] = -1;
        return;
    }

    // ---------------------------------------------------- radix select on the key bits
    // From the highest bit where the smallest and largest key differ (bits above
    // it are shared by every candidate), 11 bits per pass.
#pragma unroll 1
    for (int p = p0; !done && top >= 0; ++p) {
        const int width = top + 1 < 11 ? top + 1 : 11;
        const int sh = top - width + 1;
        const uint32_t dmask = (1u << width) - 1u;
        uint32_t *hloc = hist[p & 1];
#pragma unroll
        for (int r = 0; r < R; ++r)
            if (r < nloc && (key[r] & mask) == prefix) atomicAdd(hloc + ((key[r] >> sh) & dmask), 1u);
        sync_all();  // every CTA's histogram of this pass is complete
        find_bin(hloc, krem);
        hist[(p + 1) & 1][2 * threadIdx.x] = 0u;      // peers finished reading it in the previous pass
        hist[(p + 1) & 1][2 * threadIdx.x + 1] = 0u;
        prefix |= s_bin << sh;
        mask |= dmask << sh;
        krem = s_krem;
        done = (long long)s_cnt == krem;
        top = sh - 1;
        __syncthreads();
    }

    // stable compaction in index order
    uint32_t gt = 0u, eq = 0u;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (r < nloc) {
            const uint32_t u = key[r] & mask;
            gt += u > prefix;
            eq += u == prefix;
        }
    }
    unsigned long long blk_tot;
    const unsigned long long mine = ((unsigned long long)gt << 32) | eq;
    const unsigned long long excl = block_scan_incl<unsigned long long>(mine, warp_u64, &blk_tot) - mine;
    unsigned long long base = 0ull;
    if constexpr (CL) {
        if (threadIdx.x == 0) cta_total = blk_tot;
        cluster.sync();
        for (int r2 = 0; r2 < rank; ++r2) base += *cluster.map_shared_rank(&cta_total, r2);
    }
    long long gt_before = (long long)((base + excl) >> 32);
    long long eq_before = (long long)((base + excl) & 0xffffffffull);
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (r < nloc) {
            const uint32_t u = key[r] & mask;
            if (u > prefix) {
                const long long pos = gt_before + (eq_before < krem ? eq_before : krem);
                if (pos < kk) out[pos] = (int)(seg0 + r);
                ++gt_before;
            } else if (u == prefix) {
                if (eq_before < krem && gt_before + eq_before < kk) out[gt_before + eq_before] = (int)(seg0 + r);
                ++eq_before;
            }
        }
    }
    if (rank == 0)
        for (long long i = kk + threadIdx.x; i < k; i += kTopkThreads) out[i] = -1;
    if constexpr (CL) cluster.sync();  // peers may still read this CTA's histogram / cta_total
}

struct TopkPlan {
    int CS, R;
};

TopkPlan plan(long long n_queries, long long N) {
    const long long need = (N + kTopkThreads - 1) / kTopkThreads;  // elements per thread with one CTA
    int CS = 1;
    while ((need + CS - 1) / CS > 32) CS *= 2;
    int R = 4;
    while ((long long)R * CS < need) R *= 2;
    // Spread small batches over more SMs: measured on the 8-query decode batch
    // at 32768 entries, clusters of 8 (4 keys per thread) take 10.4 us per
    // launch against 12.4 us for clusters of 4 (8 keys per thread) and 19.9 us
    // for one CTA per query (32 keys per thread).
    while (n_queries * CS < 148 && CS < 8 && R > 4) {
        CS *= 2;
        R /= 2;
    }
    return {CS, R};
}

}  // namespace

size_t topk_workspace_bytes(int, int, long long, int) { return 0; }

int launch_topk(const float *scores, const int *q_pos, int batch, int nq, long long N, int m, int k, int *idx,
                cudaStream_t st, bool pdl) {
    const long long nqry = (long long)batch * nq;
    if (nqry == 0) return CSA_OK;
    const TopkPlan pl = plan(nqry, N);
    if (pl.CS > kMaxCluster || pl.R > 32) return CSA_ERR_UNSUPPORTED;
    void (*kern)(const float *, const int *, long long, int, int, int *, int) = nullptr;
    const bool cl = pl.CS > 1;
    switch (pl.R) {
        case 4: kern = cl ? topk_kernel<4, true> : topk_kernel<4, false>; break;
        case 8: kern = cl ? topk_kernel<8, true> : topk_kernel<8, false>; break;
        case 16: kern = cl ? topk_kernel<16, true> : topk_kernel<16, false>; break;
        case 32: kern = cl ? topk_kernel<32, true> : topk_kernel<32, false>; break;
        default: return CSA_ERR_UNSUPPORTED;
    }
    if (pl.CS > 8 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
        return CSA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(nqry * pl.CS));
    cfg.blockDim = dim3(kTopkThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (cl) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = pl.CS;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, scores, q_pos, N, m, k, idx, pl.CS);
    return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // namespace csa

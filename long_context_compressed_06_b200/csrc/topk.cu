// topk.cu -- causal top-k selector (csa_topk).
//
// For each query, the k largest scores among its n_vis(t) visible entries,
// ties broken towards the lower index; invalid slots are -1 ("DeepSeek v4"
// -> top-k selector; techniques map: indices at or beyond the causal threshold
// become -1).  Output indices are in ascending order.
//
// Design: a radix select over the scores mapped to order-preserving uint32
// keys.  One query is handled by one CTA of 1024 threads or, for long rows and
// for small batches, by a thread-block cluster of CS CTAs; each thread keeps R
// consecutive keys in registers (CS*1024*R >= N),
// so the scores are read from memory exactly once.  The digits start at the
// highest bit where the cluster-wide smallest and largest key differ (the bits
// above are shared by every candidate), 11 bits per pass; each CTA counts its
// candidates into its own shared-memory histogram and, after one cluster
// barrier, reads its peers' histograms through distributed shared memory.
// The selection stops once the threshold bin holds exactly the number of
// elements still needed.  Selection is a stable compaction: per-thread
// counts, a block scan, and a cluster scan over CTA totals via DSMEM.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace csa {
namespace {

constexpr int kTopkThreads = 1024;
constexpr int kBins = 2048;

// order-preserving map fp32 -> uint32 (-0 folded onto +0)
CSA_DEVINL uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive scan over the 1024 threads of the block; returns this thread's
// inclusive prefix and writes the block total to *total.
template <typename T>
CSA_DEVINL T block_scan_incl(T v, T *warp_buf, T *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const T n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) warp_buf[warp] = v;
    __syncthreads();
    if (warp == 0) {
        T w = warp_buf[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const T n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        warp_buf[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    if (warp > 0) v += warp_buf[warp - 1];
    const T tot = warp_buf[31];
    __syncthreads();  // warp_buf is reused by the next scan
    *total = tot;
    return v;
}

// CL: the query's row is split over a cluster of CS CTAs (histograms and CTA
// totals merged through distributed shared memory, cluster barriers); without
// it one CTA holds the row and every barrier is a block barrier.
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
    __shared__ unsigned long long cta_total;           // (gt << 32) | eq, read by higher ranks
    __shared__ uint32_t cta_min, cta_max;               // this CTA's key range, read by peers
    __shared__ uint32_t s_min, s_max, s_bin, s_cnt;
    __shared__ long long s_krem;

    // as a programmatic dependent: the scores are complete only once the
    // predecessor grid is (a no-op otherwise); the successor may launch now
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int i = threadIdx.x; i < 2 * kBins; i += kTopkThreads) (&hist[0][0])[i] = 0u;

    const long long nv = q_pos ? n_visible(q_pos[bq], m, N) : N;  // no q_pos: every entry is eligible
    const long long kk = nv < k ? nv : k;
    const long long seg0 = ((long long)rank * kTopkThreads + threadIdx.x) * R;
    const int nloc = (int)(nv - seg0 <= 0 ? 0 : (nv - seg0 >= R ? R : nv - seg0));

    uint32_t key[R];
    const float *row = scores + bq * N;
    if (nloc == R && (N & 3) == 0) {
#pragma unroll
        for (int r = 0; r < R; r += 4) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(row + seg0 + r));
            key[r] = order_key(v.x); key[r + 1] = order_key(v.y);
            key[r + 2] = order_key(v.z); key[r + 3] = order_key(v.w);
        }
    } else {
#pragma unroll
        for (int r = 0; r < R; ++r) key[r] = r < nloc ? order_key(__ldg(row + seg0 + r)) : 0u;
    }
    // key range of the visible entries (cluster-wide)
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
        if (lane == 0) {
            cta_min = a;
            cta_max = b;
        }
    }
    sync_all();  // key ranges published, histograms cleared
    if (warp == 0) {
        const uint32_t a = lane < CS ? *peer(&cta_min, lane) : 0xffffffffu;
        const uint32_t b = lane < CS ? *peer(&cta_max, lane) : 0u;
        const uint32_t ga = __reduce_min_sync(0xffffffffu, a), gb = __reduce_max_sync(0xffffffffu, b);
        if (lane == 0) {
            s_min = ga;
            s_max = gb;
            s_bin = 0u;
            s_cnt = 0u;
            s_krem = 0;
        }
    }
    __syncthreads();

    // Radix select from the highest bit where the smallest and largest key
    // differ (bits above it are shared by every candidate), 11 bits per pass.
    uint32_t prefix = 0u, mask = 0u;
    long long krem = kk;
    bool done = nv <= k;  // every visible entry is selected
    int top = -1;
    if (!done) {
        if (s_min == s_max) {
            prefix = s_max;
            mask = 0xffffffffu;  // all keys equal: the lowest indices win
            done = true;
        } else {
            top = 31 - __clz(s_min ^ s_max);
            mask = top == 31 ? 0u : ~((2u << top) - 1u);
            prefix = s_max & mask;
        }
    }
#pragma unroll 1
    for (int p = 0; !done && top >= 0; ++p) {
        const int width = top + 1 < 11 ? top + 1 : 11;
        const int sh = top - width + 1;
        const uint32_t dmask = (1u << width) - 1u;
        uint32_t *hloc = hist[p & 1];
#pragma unroll
        for (int r = 0; r < R; ++r)
            if (r < nloc && (key[r] & mask) == prefix) atomicAdd(hloc + ((key[r] >> sh) & dmask), 1u);
        sync_all();  // every CTA's histogram of this pass is complete
        // cluster-wide counts of this thread's two bins: read every rank's histogram
        uint32_t c_lo = 0u, c_hi = 0u;
        for (int r2 = 0; r2 < CS; ++r2) {
            const uint2 v = *reinterpret_cast<const uint2 *>(peer(hloc, r2) + 2 * threadIdx.x);
            c_lo += v.x;
            c_hi += v.y;
        }
        hist[(p + 1) & 1][2 * threadIdx.x] = 0u;      // peers finished reading it in the previous pass
        hist[(p + 1) & 1][2 * threadIdx.x + 1] = 0u;
        // threshold bin: the highest bin b with (count above b) < krem <= (count above b) + hist[b]
        uint32_t tot;
        const uint32_t incl = block_scan_incl<uint32_t>(c_lo + c_hi, warp_u32, &tot);
        const long long above = (long long)tot - incl;  // count in bins of higher threads
        if (above < krem && above + c_hi >= krem) {
            s_bin = 2 * threadIdx.x + 1; s_cnt = c_hi; s_krem = krem - above;
        } else if (above + c_hi < krem && above + c_hi + c_lo >= krem) {
            s_bin = 2 * threadIdx.x; s_cnt = c_lo; s_krem = krem - above - c_hi;
        }
        __syncthreads();
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
    int *out = idx + bq * k;
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
    // at 32768 entries, clusters of 4 (8 keys per thread) take 13.7 us per
    // launch against 19.9 us for one CTA per query (32 keys per thread), and
    // beat clusters of 2 and 8.
    while (n_queries * CS < 148 && CS < 4 && R > 4) {
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
    if (pl.CS > 16 || pl.R > 32) return CSA_ERR_UNSUPPORTED;
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

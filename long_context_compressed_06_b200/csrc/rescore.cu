// rescore.cu -- re-ranking of FP4-indexer candidates with the bf16 index keys
// (csa_rescore_topk).
//
// The FP4 indexer ("DeepSeek V4 paper full version is out, FP4 QAT details"
// page: FP4 activations in the indexer QK path at 99.7 % recall of the
// full-precision selection) scores every entry cheaply; selecting the top k
// from those scores directly recalls only ~86 % of the bf16-operand top-k on
// i.i.d. synthetic data.  Here the FP4 stage over-selects kc > k candidates,
// each candidate is re-scored exactly as csa_index would score it (bf16
// operands, fp32 arithmetic), and the k best candidates are kept:
//   S_c[j] = sum_h w_h * max(0, q_I[h] . K_I[cand[j]])    (cand[j] < 0 -> -inf)
//   idx    = cand[ top-k of S_c ]   (ascending entry order, -1 padded)
// The candidate key rows are gathered into a contiguous buffer and scored by
// the tensor-core indexer (each query is its own sequence of kc entries, all
// visible), invalid slots are set to -inf, the top-k selector runs over the kc
// scores and the chosen positions are mapped back to entry indices.  Shapes the tensor-core indexer does not take return
// CSA_ERR_UNSUPPORTED.
#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

// idx[bq][i] = cand[bq][local[bq][i]] (local < 0, or a candidate slot holding -1, stays -1)
__global__ void remap_kernel(const int *__restrict__ cand, const int *__restrict__ local, int kc, int k,
                             long long n, int *__restrict__ idx) {
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n) return;
    const long long bq = t / k;
    const int l = local[t];
    idx[t] = (l >= 0 && l < kc) ? cand[bq * kc + l] : -1;
}

// gathered[bq][j][:] = k_idx[b][cand[bq][j]][:] (zeros for invalid slots); pos[bq] = kc - 1
__global__ void gather_kernel(const uint16_t *__restrict__ k_idx, const int *__restrict__ cand, int kc, int nq,
                              long long N, int d_I, long long n16, uint16_t *__restrict__ gathered,
                              int *__restrict__ pos) {
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;  // 16-byte unit
    if (t >= n16) return;
    const int upr = d_I / 8;  // 16-byte units per row
    const long long row = t / upr;  // bq * kc + j
    const int u = (int)(t - row * upr);
    const long long bq = row / kc;
    const int c = cand[row];
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (c >= 0 && c < N) v = ldg16(k_idx + ((size_t)(bq / nq) * N + c) * d_I + u * 8);
    *reinterpret_cast<uint4 *>(gathered + (size_t)row * d_I + u * 8) = v;
    if (row - bq * kc == 0 && u == 0) pos[bq] = kc - 1;
}

// scores of invalid candidate slots -> -inf
__global__ void mask_kernel(const int *__restrict__ cand, long long n, long long N, float *__restrict__ sc) {
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n) return;
    const int c = cand[t];
    if (c < 0 || c >= N) sc[t] = -INFINITY;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

// [scores fp32 nbq x kc][chosen positions int nbq x k][gathered keys bf16 nbq x kc x d_I][positions int nbq]
size_t rescore_workspace_bytes(int batch, int nq, int kc, int k, int d_I) {
    const size_t nbq = (size_t)batch * nq;
    return align256(nbq * kc * sizeof(float)) + align256(nbq * k * sizeof(int)) +
           align256(nbq * kc * (size_t)d_I * 2) + align256(nbq * sizeof(int));
}

bool rescore_supported(int H_I, int d_I) { return index_tc_supported(H_I, d_I); }

int launch_rescore_topk(const uint16_t *q_idx, const float *w, const uint16_t *k_idx, const int *cand, int kc,
                        int batch, int nq, long long N, int H_I, int d_I, int k, int *idx, void *ws,
                        const DevCtx &ctx, cudaStream_t st) {
    const long long nbq = (long long)batch * nq;
    char *wsb = reinterpret_cast<char *>(ws);
    float *sc = reinterpret_cast<float *>(wsb);
    wsb += align256((size_t)nbq * kc * sizeof(float));
    int *local = reinterpret_cast<int *>(wsb);
    wsb += align256((size_t)nbq * k * sizeof(int));
    uint16_t *gathered = reinterpret_cast<uint16_t *>(wsb);
    wsb += align256((size_t)nbq * kc * (size_t)d_I * 2);
    int *pos = reinterpret_cast<int *>(wsb);
    if (!index_tc_supported(H_I, d_I)) return CSA_ERR_UNSUPPORTED;
    const long long n16 = nbq * kc * (d_I / 8);
    gather_kernel<<<(unsigned)((n16 + 255) / 256), 256, 0, st>>>(k_idx, cand, kc, nq, N, d_I, n16, gathered, pos);
    if (cudaGetLastError() != cudaSuccess) return CSA_ERR_CUDA;
    // every (sequence, query) is one sequence of kc entries with its query at position kc - 1 (m = 1)
    int rc = launch_index_tc(q_idx, w, gathered, pos, (int)nbq, 1, kc, H_I, d_I, 1, sc, ctx, st);
    if (rc != CSA_OK) return rc;
    const long long n = nbq * kc;
    mask_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(cand, n, N, sc);
    if (cudaGetLastError() != cudaSuccess) return CSA_ERR_CUDA;
    rc = launch_topk(sc, nullptr, batch, nq, kc, 1, k, local, st);
    if (rc != CSA_OK) return rc;
    const long long nk = nbq * k;
    remap_kernel<<<(unsigned)((nk + 255) / 256), 256, 0, st>>>(cand, local, kc, k, nk, idx);
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // namespace csa

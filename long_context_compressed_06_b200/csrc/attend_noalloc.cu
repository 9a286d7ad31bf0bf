// attend_noalloc.cu -- csa_attend for callers that cannot allocate device memory.
//
// Some callers of this library have no way to allocate: a plugin or embedded
// runtime that is handed only a stream and pointers to its tensors, a serving
// loop that forbids cudaMalloc on its hot path (it synchronises the device),
// or code recording work into a CUDA graph, where allocation is not permitted.
// csa_attend needs caller scratch for its split-KV partial results; this entry
// point supplies it from a file-scope device array instead, so the caller
// passes only inputs and outputs.
//
// The array is a fixed CSA_ATTEND_NOALLOC_MAX_BYTES per device; every GPU that
// loads the library holds it until the process exits.  All calls share it and
// it keeps the last call's contents; nothing needs clearing (every slot the
// combine step reads is written earlier in the same call), but calls that
// overlap on the GPU -- on different streams, or from several host threads --
// race on it.
#include <cuda_runtime.h>

#include "../../include/csa.h"
#include "kernels.h"

namespace {

__device__ __align__(256) unsigned char g_attend_scratch[CSA_ATTEND_NOALLOC_MAX_BYTES];

// Device address of the array on the current device.  In host code the
// symbol is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress; it is looked up once per device, with that device
// current, on the first call made on it.  The cached address outlives a
// cudaDeviceReset of that device, after which it is stale: callers that reset
// a device must not use this entry point on it again in the same process.
void *scratch_on_current_device() {
    static void *cache[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!cache[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_attend_scratch) != cudaSuccess) return nullptr;
        cache[dev] = p;
    }
    return cache[dev];
}

}  // namespace

extern "C" int csa_attend_noalloc(const uint16_t *q, const float *q_gain, const float *sinks,
                                  const float *rope_cos, const float *rope_sin, long long rope_positions,
                                  const uint16_t *kv, long long N,
                                  const int *idx, int k, const uint16_t *win_src, long long win_pos0,
                                  long long win_rows, int W, const int *q_pos, int batch, int nq, int H, int D,
                                  float scale, float eps, uint16_t *out, void *stream) {
    // the same argument checks as csa_attend first, then the array's size limit
    const int rc = csa::check_attend_args(q, q_gain, sinks, rope_cos, rope_sin, rope_positions, kv, N, idx, k,
                                          win_src, win_pos0, win_rows, W, q_pos, batch, nq, H, D, eps, out);
    if (rc != CSA_OK) return rc;
    const size_t need = csa_attend_workspace_bytes(batch, nq, H, D, (long long)k + W);
    if (need > (size_t)CSA_ATTEND_NOALLOC_MAX_BYTES) return CSA_ERR_WORKSPACE;
    void *scratch = scratch_on_current_device();
    if (!scratch) return CSA_ERR_CUDA;
    return csa_attend(q, q_gain, sinks, rope_cos, rope_sin, rope_positions, kv, N, idx, k, win_src, win_pos0, win_rows, W, q_pos, batch, nq, H, D, scale, eps,
                      out, scratch, (size_t)CSA_ATTEND_NOALLOC_MAX_BYTES, stream);
}

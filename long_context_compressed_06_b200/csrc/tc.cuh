// tc.cuh -- sm_100a tensor-core plumbing: TMA tensor maps and loads, TMEM
// allocation, tcgen05.mma (kind::f16) with shared-memory descriptors,
// tcgen05.commit / tcgen05.ld, written as inline PTX.
//
// Operand convention used by every kernel here: both MMA operands K-major in
// shared memory with the canonical 128-byte (or 64-byte) swizzle that TMA
// writes, so D[m][n] = sum_k A[m][k] * B[n][k]; accumulators fp32 in TMEM with
// row m in lane m (M = 128, cta_group::1).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace csa {
namespace tc {

// ---------------------------------------------------------------- TMA
CSA_DEVINL void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// The issue helpers below take a guard `pred`: a warp that keeps all its lanes
// on the same path and lets one lane issue (pred = lane == 0) stays converged.
// Branching around the issue instead (if (lane == 0) {...}) leaves the warp
// diverged while the other lanes wait, which was measured to slow the issuing
// lane several-fold.
CSA_DEVINL void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1, int c2,
                            bool pred = true) {
    asm volatile(
        "{\n\t.reg .pred g;\n\tsetp.ne.b32 g, %6, 0;\n\t"
        "@g cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];\n\t}"
        ::"r"(dst), "l"(map), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"((int)pred)
        : "memory");
}

CSA_DEVINL void tma_load_4d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1, int c2, int c3,
                            bool pred = true) {
    asm volatile(
        "{\n\t.reg .pred g;\n\tsetp.ne.b32 g, %7, 0;\n\t"
        "@g cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];\n\t}"
        ::"r"(dst), "l"(map), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"((int)pred)
        : "memory");
}

// ---------------------------------------------------------------- TMEM
// Warp-wide: allocates `ncols` (power of two >= 32) columns, address written to smem.
CSA_DEVINL void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
CSA_DEVINL void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
CSA_DEVINL void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

CSA_DEVINL void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
CSA_DEVINL void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// generic-proxy shared-memory writes -> visible to the tensor core (async proxy)
CSA_DEVINL void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------- descriptors
enum : uint32_t { kLayoutSw128 = 2, kLayoutSw64 = 4, kLayoutSw32 = 6 };

// K-major operand in shared memory, swizzled rows of `row_bytes`, 8-row groups
// `sbo` bytes apart.  The start address may be advanced inside a swizzle row
// (by 32 bytes per 16-element bf16 K step).
CSA_DEVINL uint64_t smem_desc(uint32_t saddr, uint32_t sbo, uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;                          // leading byte offset (unused: swizzled K-major)
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;      // stride byte offset
    d |= (uint64_t)1u << 46;                          // descriptor version (sm100)
    d |= (uint64_t)(layout & 7u) << 61;
    return d;
}

// Same, with an explicit leading byte offset (MN-major operands: the stride
// between consecutive 64-element groups along M/N).
CSA_DEVINL uint64_t smem_desc_lbo(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)(layout & 7u) << 61;
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulate, A/B both bf16 (or both
// f16), both K-major, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(int n, bool bf16) {
    return (1u << 4)                                   // D format: f32
           | ((bf16 ? 1u : 0u) << 7)                   // A format
           | ((bf16 ? 1u : 0u) << 10)                  // B format
           | ((uint32_t)(n >> 3) << 17)                // N >> 3
           | ((uint32_t)(128 >> 4) << 24);             // M >> 4
}

// ---------------------------------------------------------------- MMA
CSA_DEVINL void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate,
                        bool pred = true) {
    asm volatile(
        "{\n\t.reg .pred p, g;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.ne.b32 g, %5, 0;\n\t"
        "@g tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"((int)pred)
        : "memory");
}

// arrive once on the mbarrier when every tcgen05.mma issued so far by this thread completes
CSA_DEVINL void mma_commit(uint32_t bar, bool pred = true) {
    asm volatile(
        "{\n\t.reg .pred g;\n\tsetp.ne.b32 g, %1, 0;\n\t"
        "@g tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}"
        ::"r"(bar), "r"((int)pred)
        : "memory");
}

// ---------------------------------------------------------------- TMEM -> registers
// 32 lanes x 16 consecutive 32-bit columns; thread i gets lane (base + i).
CSA_DEVINL void tmem_ld16(uint32_t taddr, float v[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

CSA_DEVINL void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

CSA_DEVINL void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

}  // namespace tc

// Host: encode a tiled tensor map through the driver entry point (no libcuda link).
bool encode_tensor_map(CUtensorMap *map, CUtensorMapDataType dtype, uint32_t rank, const void *base,
                       const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
                       CUtensorMapSwizzle swizzle);

int num_sms();

}  // namespace csa

// common.cuh -- device utilities shared by the libcsa kernels (sm_100a).
//
// * bf16 <-> fp32 helpers and 16-byte vector loads,
// * the device status word protocol (a kernel that gives up a bounded wait
//   records CSA_ERR_TIMEOUT there; csa_sync_status() reads and clears it),
// * bounded mbarrier waits on %globaltimer (no wait in this library can spin
//   forever: after `budget_ns` it records the timeout and returns false).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa.h"

#define CSA_DEVINL __device__ __forceinline__

namespace csa {

// ---------------------------------------------------------------- launch context
// Passed by value to every kernel that can fail on the device.
struct DevCtx {
    int *status;                  // device status word (CSA_OK or CSA_ERR_*)
    unsigned long long budget_ns; // limit for any single device-side wait
};

// ---------------------------------------------------------------- bf16 helpers
CSA_DEVINL float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
CSA_DEVINL float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// 8 bf16 packed in a uint4 -> 8 floats
CSA_DEVINL void unpack8(const uint4 &v, float f[8]) {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// round-to-nearest-even fp32 -> bf16 pair packed low|high
CSA_DEVINL uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}

CSA_DEVINL uint4 pack8(const float f[8]) {
    uint4 v;
    v.x = pack_bf16x2(f[0], f[1]);
    v.y = pack_bf16x2(f[2], f[3]);
    v.z = pack_bf16x2(f[4], f[5]);
    v.w = pack_bf16x2(f[6], f[7]);
    return v;
}

// streaming 16-byte load that does not allocate in L1 (read-once data)
CSA_DEVINL uint4 ldg_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

CSA_DEVINL uint4 ldg16(const void *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

// ---------------------------------------------------------------- misc
CSA_DEVINL long long n_visible(long long t, int m, long long N) {
    long long v = (t + 1) / m;
    v = v < 0 ? 0 : v;
    return v > N ? N : v;
}

CSA_DEVINL uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

CSA_DEVINL uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

CSA_DEVINL void record_status(int *status, int code) {
    if (status) atomicCAS(status, CSA_OK, code);
}

// ---------------------------------------------------------------- mbarriers
CSA_DEVINL void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

CSA_DEVINL void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

CSA_DEVINL bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking probe of a phase (for loops that poll several barriers).
CSA_DEVINL bool mbar_test_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of the mbarrier at shared address `bar`.  Gives up
// after ctx.budget_ns of global time, or at once if *abort (a CTA-wide flag in
// shared memory) is set; on giving up it records CSA_ERR_TIMEOUT, sets *abort
// and returns false.
CSA_DEVINL bool mbar_wait(uint32_t bar, uint32_t parity, const DevCtx &ctx, volatile int *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (abort && *abort) return false;
        if (global_timer_ns() - t0 > ctx.budget_ns) {
            record_status(ctx.status, CSA_ERR_TIMEOUT);
            if (abort) *abort = 1;
            return false;
        }
    }
}

// `pred` guards the arrive (one lane of a converged warp arrives).
CSA_DEVINL void mbar_arrive(uint32_t bar, bool pred = true) {
    asm volatile(
        "{\n\t.reg .pred g;\n\tsetp.ne.b32 g, %1, 0;\n\t@g mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}"
        ::"r"(bar), "r"((int)pred) : "memory");
}

CSA_DEVINL void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes, bool pred = true) {
    asm volatile(
        "{\n\t.reg .pred g;\n\tsetp.ne.b32 g, %2, 0;\n\t"
        "@g mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}"
        ::"r"(bar), "r"(bytes), "r"((int)pred) : "memory");
}

// ---------------------------------------------------------------- warp helpers
CSA_DEVINL float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

CSA_DEVINL float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

}  // namespace csa

// Device helpers shared by the k3moe kernels (sm_100a).
//
// Written from the public PTX ISA: cp.async.bulk (bulk asynchronous copy,
// global -> shared, completion counted on an mbarrier), mbarrier
// init/arrive.expect_tx/try_wait.parity, mma.sync m16n8k16, griddepcontrol,
// and cvt.rn.f16x2.e2m1x2 through cuda_fp4.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "k3moe.h"

namespace k3 {

// ----------------------------------------------------------------- status --
// Workspace status word bits (first word of the workspace header).
constexpr uint32_t kStDeviceCheck = 1u;  // a device-side argument check failed
constexpr uint32_t kStTimeout = 2u;      // a bounded wait gave up

// Bounded waits give up after this many nanoseconds of wall time.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct WsHeader {
    uint32_t status;
    uint32_t router_done;  // router rows finished in this call; back to 0 by its end
    uint32_t n_unique;     // distinct routed experts in the current token chunk
    uint32_t pad[61];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void set_status(WsHeader *h, uint32_t bits) {
    atomicOr(&h->status, bits);
}

// ------------------------------------------------------------ shared mem --
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// Bulk asynchronous copy global -> shared (this CTA), completion counted in
// bytes on `bar`.  dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, for at most kWaitLimitNs.
// Returns false (and sets the timeout bit) when the limit is reached.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, WsHeader *h) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > kWaitLimitNs) {
            set_status(h, kStTimeout);
            return false;
        }
    }
}

// ------------------------------------------------- programmatic launches --
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// --------------------------------------------------------------- formats --
// Two E2M1 codes (low nibble = even element) -> f16x2 (low half = even element).
// The conversion is exact: every E2M1 value is an f16.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    __half2_raw r = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte), __NV_E2M1);
    return static_cast<uint32_t>(r.x) | (static_cast<uint32_t>(r.y) << 16);
}

// E8M0 byte -> 2^(e-127) as fp32 (e = 0 -> 2^-127, a subnormal; e = 255 -> NaN).
__device__ __forceinline__ float e8m0_to_f32(uint32_t e) {
    uint32_t bits = (e == 0u) ? 0x00400000u : (e == 255u ? 0x7FC00000u : (e << 23));
    return __uint_as_float(bits);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Power-of-two exponent s such that max_abs * 2^s lies in [2^14, 2^15):
// values scaled by 2^s then fit f16 (max 65504) with full precision for the
// larger elements.  max_abs == 0 -> 0.
__device__ __forceinline__ int f16_prescale(float max_abs) {
    if (!(max_abs > 0.0f) || !isfinite(max_abs)) return 0;
    int e;
    frexpf(max_abs, &e);  // max_abs = m 2^e, m in [0.5, 1)
    int s = 15 - e;
    return s < -120 ? -120 : (s > 120 ? 120 : s);
}

// ------------------------------------------------------------------- mma --
// D = A(16x16, row) * B(16x8, col) + C, f16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Same with bf16 inputs.
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

}  // namespace k3

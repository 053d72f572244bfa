// Device helpers shared by the k3moe kernels (sm_100a).
//
// Written from the public PTX ISA: cp.async.bulk (bulk asynchronous copy,
// global -> shared, completion counted on an mbarrier), mbarrier
// init/arrive.expect_tx/try_wait.parity, griddepcontrol, gpu-scope atomics.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "k3moe.h"

namespace k3 {

// ----------------------------------------------------------------- status --
// Workspace status word bits (first word of the workspace header).
constexpr uint32_t kStDeviceCheck = 1u;  // a device-side argument check failed
constexpr uint32_t kStTimeout = 2u;      // a bounded wait gave up

// Bounded waits give up after this many nanoseconds of wall time (the
// default; every kernel takes its limit as a launch parameter).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct WsHeader {
    uint32_t status;
    uint32_t router_done;  // router rows finished in this call; back to 0 by its end
    uint32_t n_unique;     // distinct routed experts in the current token chunk
    uint32_t topk_done;    // tokens whose top-k other CTAs finished; back to 0 by its end
    uint32_t prep_done;    // CTAs whose tensor maps and x pieces are written (decode; back to 0
                           // by the end of the call)
    uint32_t gu_done;      // gate/up items whose activations are written (layer kernel)
    uint32_t exit_cnt;     // CTAs of the layer kernel that have finished (the last resets)
    uint32_t disp_cnt;     // 1 once the chunk's dispatch is written (released for the down pass)
    uint32_t disp_seen;    // down-pass CTAs that have read the dispatch (the last resets both)
    uint32_t pad[55];
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

// try_wait without a time hint: the hardware's own short wait window, then
// the caller polls again (no long suspension between phase completion and
// wake-up on the pipeline's critical path).
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

// Wait for phase `parity` of `bar` to complete, for at most limit_ns.
// Returns false (and sets the timeout bit) when the limit is reached.
// The clock is read only every 64 polls: the waits sit on the pipelines'
// critical paths.
// try_wait that lets the hardware suspend the thread (up to about a
// microsecond) until the phase completes, instead of returning at once.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(1000u)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, WsHeader *h,
                                                  uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait_sleep(bar, parity)) return true;
        if ((i & 63u) == 0u && globaltimer() - t0 > limit_ns) {
            set_status(h, kStTimeout);
            return false;
        }
    }
}

// Wait (bounded, no status) for phase `parity` of `bar`: used on the way
// out of a kernel whose pipeline gave up, so that bulk copies this thread
// issued have landed before the CTA's shared memory is released.
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > limit_ns) return;
    }
}

// E8M0 byte 0xFF encodes NaN: nonzero when any of the 8 bytes of (a, b) is.
__device__ __forceinline__ uint32_t e8m0_nan8(uint32_t a, uint32_t b) {
    return __vcmpeq4(a, 0xFFFFFFFFu) | __vcmpeq4(b, 0xFFFFFFFFu);
}

// ------------------------------------------------- gpu-scope atomics --
// Release: this thread's earlier writes are visible to whoever acquires the
// counter after it; acquire: writes released by others are visible after.
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t *p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void red_add_release(uint32_t *p, uint32_t v) {
    asm volatile("red.add.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Wait until *ctr >= target: one acquire load first (the count is often
// there already); else relaxed polls with a short sleep, then one acquire
// fence (a relaxed read that sees the producers' release, followed by the
// fence, orders everything they published before this thread's later reads),
// so the acquire is paid once and not on every poll.  False after
// limit_ns, or at once when *abort (if given) becomes nonzero.
__device__ __forceinline__ bool spin_geq(const uint32_t *ctr, uint32_t target, uint64_t limit_ns,
                                         const volatile int *abort = nullptr) {
    if (ld_acquire(ctr) >= target) return true;  // already there: one acquire load, no fence
    if (ld_relaxed(ctr) < target) {
        const uint64_t t0 = globaltimer();
        do {
            if ((abort && *abort) || globaltimer() - t0 > limit_ns) return false;
            __nanosleep(32);
        } while (ld_relaxed(ctr) < target);
    }
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    return true;
}

// ------------------------------------------------- programmatic launches --
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 8-byte asynchronous copy global -> shared (no register staging); complete
// after cp_async_wait_all.  Both addresses 8-byte aligned.
__device__ __forceinline__ void cp_async8(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n cp.async.wait_all;" ::: "memory");
}

// --------------------------------------------------------------- formats --
__device__ __forceinline__ float exp2i(int s) {  // 2^s for -126 <= s <= 127
    return __uint_as_float((uint32_t)(127 + s) << 23);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

// ------------------------------------------------------------- RMSNorm --
// 1 / sqrt(mean(h^2) + eps) of one token of d bf16 values, by one warp: lane
// l sums the squares of elements l, l + 32, ... in fp32, then a fixed
// butterfly adds the lanes, so every warp that runs it gets the same bits.
__device__ __forceinline__ float warp_rms_inv(const uint16_t *h, int d, float eps) {
    const int lane = threadIdx.x & 31;
    float ss = 0.f;
    for (int j = lane; j < d; j += 32) {
        const float v = __uint_as_float((uint32_t)h[j] << 16);
        ss = fmaf(v, v, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    return 1.0f / sqrtf(ss / (float)d + eps);
}
// One element of the normalised token: RNE_bf16((h * r) * g), bf16 bits.
__device__ __forceinline__ uint16_t rms_norm_bf16(uint16_t h, float r, uint16_t g) {
    const float v = (__uint_as_float((uint32_t)h << 16) * r) * __uint_as_float((uint32_t)g << 16);
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

}  // namespace k3

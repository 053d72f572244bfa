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
#include <cuda_fp8.h>
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

// try_wait with a suspend-time hint: the warp sleeps in hardware until the
// phase completes (or ~1 ms passes) instead of spinning on the barrier.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
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

// E2M1 nibbles -> E4M3 bytes by bit placement (ALU only, no conversion unit).
// An E2M1 code s.e1e0.m becomes the E4M3 byte s.00e1e0.m00, whose value is
// exactly 2^-6 times the E2M1 value: for exponent field e >= 1 both are
// 2^(e-1)(1+m/2) resp. 2^(e-7)(1+m/2), and the E2M1 subnormal 0.5 (e=0, m=1)
// lands on the E4M3 subnormal 4/8 * 2^-6.  The four even (low) nibbles of a
// word give one word of four E4M3 bytes, the four odd (high) nibbles another.
__device__ __forceinline__ uint32_t e2m1_even_to_e4m3(uint32_t w) {
    return ((w << 4) & 0x80808080u) | ((w << 2) & 0x1C1C1C1Cu);
}
__device__ __forceinline__ uint32_t e2m1_odd_to_e4m3(uint32_t w) {
    return (w & 0x80808080u) | ((w >> 2) & 0x1C1C1C1Cu);
}

// E2M1 nibbles -> f16 by bit placement (ALU only).  The code s.e1e0.m is put
// at f16 bits 15 (sign) and 11..9 (low exponent bits, top mantissa bit): the
// f16 value is exactly 2^-14 times the E2M1 value (the E2M1 subnormal 0.5
// becomes the f16 subnormal 2^-15).  One register holds nibbles i and i+4 of
// a word (16 bits apart), so both halves take the same shifts:
//   pair 0: columns 0,4   pair 1: columns 1,5   pair 2: 2,6   pair 3: 3,7
__device__ __forceinline__ uint32_t e2m1_pair0_f16(uint32_t w) {
    return ((w << 9) & 0x0E000E00u) | ((w << 12) & 0x80008000u);
}
__device__ __forceinline__ uint32_t e2m1_pair1_f16(uint32_t w) {
    return ((w << 5) & 0x0E000E00u) | ((w << 8) & 0x80008000u);
}
__device__ __forceinline__ uint32_t e2m1_pair2_f16(uint32_t w) {
    return ((w << 1) & 0x0E000E00u) | ((w << 4) & 0x80008000u);
}
__device__ __forceinline__ uint32_t e2m1_pair3_f16(uint32_t w) {
    return ((w >> 3) & 0x0E000E00u) | (w & 0x80008000u);
}
// Position of column c of an 8-column group in the pair order 0,4,1,5,2,6,3,7.
__device__ __forceinline__ int pairpos(int c) { return (c & ~7) + 2 * (c & 3) + ((c >> 2) & 1); }

// fp32 <-> E4M3 (OCP E4M3FN: bias 7, subnormals, no infinities) on the ALU
// and FMA pipes.  Scaling by 2^-120 maps every E4M3 value, normal or
// subnormal, onto fp32 bit patterns whose bits 30..20 are the E4M3 bits 6..0
// (fp32 subnormals included, which fp32 arithmetic keeps when not flushing),
// so rounding is an integer add at bit 20 (ties to even).  |v| <= 448.
__device__ __forceinline__ uint32_t f32_to_e4m3_rn(float v) {
    const uint32_t u = __float_as_uint(v * 0x1p-120f);
    uint32_t m = u & 0x7FFFFFFFu;
    m += 0x7FFFFu + ((m >> 20) & 1u);
    return ((u >> 24) & 0x80u) | (m >> 20);
}
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    return __uint_as_float(((b & 0x80u) << 24) | ((b & 0x7Fu) << 20)) * 0x1p120f;
}

// Piece `piece` (0-based) of v written as a greedy sum of E4M3 values (each
// step rounds the remaining residual to nearest; every residual is exact in
// fp32).  Each piece carries 4 significant bits, so n pieces reproduce v
// exactly while its low bits stay at or above the E4M3 step 2^-9.
__device__ __forceinline__ uint32_t e4m3_piece(float v, int piece) {
    uint32_t b = 0;
    for (int i = 0; i <= piece; ++i) {
        b = f32_to_e4m3_rn(v);
        v -= e4m3_to_f32(b);
    }
    return b;
}

// Power-of-two exponent s with max_abs * 2^s in [128, 256): the largest
// prescaled activation then fits E4M3 (max 448) with room for rounding up.
__device__ __forceinline__ int e4m3_prescale(float max_abs) {
    if (!(max_abs > 0.0f) || !isfinite(max_abs)) return 0;
    int e;
    frexpf(max_abs, &e);
    int s = 8 - e;
    return s < -100 ? -100 : (s > 100 ? 100 : s);
}

__device__ __forceinline__ float exp2i(int s) {  // 2^s for -126 <= s <= 127
    return __uint_as_float((uint32_t)(127 + s) << 23);
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

// D = A(16x32, row) * B(32x8, col) + C, E4M3 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_e4m3(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
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

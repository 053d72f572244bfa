// The grouped path's router GEMM on the tensor cores: logits[t][e] =
// sum_j x[t][j] W_r[e][j] (+ b[e]) for a whole pass of tokens.
//
// The router is fp32 and x bf16; the tensor cores take bf16 x bf16.  Each
// fp32 weight is split exactly into three bf16 parts, w = w1 + w2 + w3 (w1 =
// bf16(w), w2 = bf16(w - w1), w3 = w - w1 - w2, which has at most 8
// significant bits left), so every product x * w_i is exact in the fp32
// accumulator and their sum is the exact product x * w: the three parts are
// three bf16 MMAs into one accumulator (kind::f16, fp32 accumulate).  The
// tutorial page's section 2.4 computes the same gate scores as a GEMV per
// token; here one pass of tokens is one GEMM.
//
// Tiles of 128 experts x 128 tokens, K in steps of 64 (one 128-byte swizzled
// TMA box per operand per step: the three weight parts and the tokens), a
// ring of stages; CTAs take tiles round-robin.  The tensor core accumulates
// one K-chunk of 256 at a time into a tensor-memory buffer (two buffers,
// alternating); the epilogue adds each chunk's partial sums into fp32
// registers.  A single accumulation chain over all of d = 7168 (1344 MMAs of
// K = 16) drifted by up to about 1e-5 relative from the exact logits, which is
// the size of the top-k tie gap the results are held to; chains of 48 MMAs
// with the chunk sums rounded to nearest keep the drift well below it.
// Warps: 0 TMEM allocation, 1 copies, 2 MMA issue, 4-7 epilogue (one lane
// quadrant each: lane = expert, column = token).
#pragma once

#include "common.cuh"
#include "layout.cuh"
#include "umma.cuh"

namespace k3 {

constexpr int kRmThreads = 256;
constexpr int kRmTile = 128;       // experts and tokens per tile
constexpr int kRmKStep = 64;       // bf16 per K-step (128 bytes of every row)
constexpr int kRmBox = kRmTile * 128;  // 16 KB: one operand box
constexpr int kRmStageBytes = 4 * kRmBox;  // three weight parts + the tokens
constexpr int kRmStages = 3;
constexpr int kRmChunk = 4;     // K-steps per tensor-core accumulation chunk

__host__ __device__ inline int rm_smem_bytes() { return 1024 + kRmStages * kRmStageBytes + 256; }

struct RouterMmaParams {
    uint4 tw[3][8];      // tensor maps of the three bf16 parts [E][d] (box 64 x 128, 128-byte swizzle)
    uint4 tx[8];         // tensor map of x [T][d] bf16 (same box)
    const float *bias;   // [E] or null
    int T, d, E;
    float *out;          // logits [T][E]
    uint8_t *ws;         // workspace (status word)
    uint64_t wait_ns;
};

// w -> (w1, w2, w3) bf16, element by element; n a multiple of 4.
struct RouterSplitParams {
    const float *w;
    size_t n;
    uint16_t *w1, *w2, *w3;
};
__global__ void pf_router_split_kernel(const __grid_constant__ RouterSplitParams p) {
    const size_t n4 = p.n / 4;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        const float4 v = __ldcs(reinterpret_cast<const float4 *>(p.w) + i);
        const float a[4] = {v.x, v.y, v.z, v.w};
        uint16_t h1[4], h2[4], h3[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const __nv_bfloat16 b1 = __float2bfloat16_rn(a[q]);
            const float r1 = a[q] - __bfloat162float(b1);  // exact
            const __nv_bfloat16 b2 = __float2bfloat16_rn(r1);
            const float r2 = r1 - __bfloat162float(b2);    // exact, at most 8 significant bits
            const __nv_bfloat16 b3 = __float2bfloat16_rn(r2);
            h1[q] = __bfloat16_as_ushort(b1);
            h2[q] = __bfloat16_as_ushort(b2);
            h3[q] = __bfloat16_as_ushort(b3);
        }
        reinterpret_cast<uint2 *>(p.w1)[i] = make_uint2(h1[0] | ((uint32_t)h1[1] << 16), h1[2] | ((uint32_t)h1[3] << 16));
        reinterpret_cast<uint2 *>(p.w2)[i] = make_uint2(h2[0] | ((uint32_t)h2[1] << 16), h2[2] | ((uint32_t)h2[3] << 16));
        reinterpret_cast<uint2 *>(p.w3)[i] = make_uint2(h3[0] | ((uint32_t)h3[1] << 16), h3[2] | ((uint32_t)h3[3] << 16));
    }
}

__global__ void __launch_bounds__(kRmThreads, 1) pf_router_mma_kernel(const __grid_constant__ RouterMmaParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kRmStages * kRmStageBytes);
    uint64_t *empty = full + kRmStages;
    uint64_t *afull = empty + kRmStages;
    uint64_t *aempty = afull + 2;
    uint64_t *mdone = aempty + 2;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mdone + 1);
    volatile int *s_abort = reinterpret_cast<volatile int *>(tslot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kRmStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&afull[b], 1);
            mbar_init(&aempty[b], 4);
        }
        mbar_init(mdone, 1);
        fence_mbar_init();
        *s_abort = 0;
    }
    constexpr uint32_t kCols = 256u;
    if (warp == 0) umma::tmem_alloc(tslot, kCols);
    umma::fence_before();
    __syncthreads();
    umma::fence_after();
    const uint32_t tbase = *tslot;
    const int ne = ceil_div(p.E, kRmTile), ntt = ceil_div(p.T, kRmTile);
    const int ntiles = ne * ntt, nks = ceil_div(p.d, kRmKStep);
    const int G = gridDim.x;
    auto wait = [&](uint64_t *bar, uint32_t parity) {
        if (*s_abort) return false;
        if (mbar_wait_bounded(bar, parity, hdr, p.wait_ns)) return true;
        *s_abort = 1;
        return false;
    };
    if (warp == 1) {
        if (lane == 0) {
            int i = 0;
            for (int tile = blockIdx.x; tile < ntiles && !*s_abort; tile += G) {
                const int e0 = (tile % ne) * kRmTile, t0 = (tile / ne) * kRmTile;
                for (int ks = 0; ks < nks; ++ks, ++i) {
                    const int s = i % kRmStages;
                    if (i >= kRmStages && !wait(&empty[s], (uint32_t)(((i / kRmStages) + 1) & 1))) break;
                    uint8_t *st = smem + s * kRmStageBytes;
                    mbar_arrive_expect_tx(&full[s], (uint32_t)kRmStageBytes);
#pragma unroll
                    for (int q = 0; q < 3; ++q) umma::tma_load_2d(st + q * kRmBox, p.tw[q], ks * kRmKStep, e0, &full[s]);
                    umma::tma_load_2d(st + 3 * kRmBox, p.tx, ks * kRmKStep, t0, &full[s]);
                }
            }
            if (*s_abort) {
                for (int q = 0; q < kRmStages && q < i; ++q) {
                    const int last = q + ((i - 1 - q) / kRmStages) * kRmStages;
                    mbar_drain(&full[q], (uint32_t)((last / kRmStages) & 1), p.wait_ns);
                }
            }
        }
    } else if (warp == 2) {
        if (lane == 0) {
            const uint64_t desc0 = umma::smem_desc(smem_u32(smem), 16u, 1024u, umma::kLayoutSw128);
            const uint32_t idesc = umma::idesc_bf16(kRmTile);
            int i = 0, q = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok && !*s_abort; tile += G) {
                for (int k0 = 0; k0 < nks && ok; k0 += kRmChunk, ++q) {
                    const int buf = q & 1;
                    if (q >= 2 && !wait(&aempty[buf], (uint32_t)(((q >> 1) + 1) & 1))) { ok = false; break; }
                    umma::fence_after();
                    const uint32_t dcol = tbase + (uint32_t)(buf * kRmTile);
                    uint32_t acc = 0u;
                    const int k1 = min(nks, k0 + kRmChunk);
                    for (int ks = k0; ks < k1; ++ks, ++i) {
                        const int s = i % kRmStages;
                        if (!wait(&full[s], (uint32_t)((i / kRmStages) & 1))) { ok = false; break; }
                        umma::fence_after();
                        const uint64_t a = desc0 + ((uint32_t)(s * kRmStageBytes) >> 4);
                        const uint64_t b = a + ((uint32_t)(3 * kRmBox) >> 4);
                        const int nk = min(4, (p.d - ks * kRmKStep) / 16);
#pragma unroll
                        for (int part = 0; part < 3; ++part) {
#pragma unroll
                            for (int sk = 0; sk < 4; ++sk) {
                                if (sk < nk) {
                                    umma::mma_bf16(dcol, a + (uint32_t)(part * (kRmBox >> 4)) + 2 * sk, b + 2 * sk, idesc, acc);
                                    acc = 1u;
                                }
                            }
                        }
                        umma::commit(&empty[s]);
                    }
                    umma::commit(&afull[buf]);
                }
            }
            umma::commit(mdone);
            mbar_drain(mdone, 0u, p.wait_ns);
        }
    } else if (warp >= 4) {
        // epilogue: lane quadrant (warp - 4), lane = expert row of the tile
        const uint32_t lb = umma::lane_base(warp);
        const int row = 32 * (warp - 4) + lane;
        int q = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < ntiles && ok; tile += G) {
            const int e0 = (tile % ne) * kRmTile, t0 = (tile / ne) * kRmTile;
            float sum[kRmTile];
#pragma unroll
            for (int j = 0; j < kRmTile; ++j) sum[j] = 0.f;
            for (int k0 = 0; k0 < nks; k0 += kRmChunk, ++q) {
                const int buf = q & 1;
                int got = 0;
                if (lane == 0) got = wait(&afull[buf], (uint32_t)((q >> 1) & 1)) ? 1 : 0;
                got = __shfl_sync(0xffffffffu, got, 0);
                umma::fence_after();
                if (got) {
#pragma unroll
                    for (int c = 0; c < kRmTile; c += 32) {
                        uint32_t v[32];
                        umma::ld32(tbase + lb + (uint32_t)(buf * kRmTile + c), v);
                        umma::wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) sum[c + j] += __uint_as_float(v[j]);
                    }
                }
                umma::fence_before();
                __syncwarp();
                if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&aempty[buf])) : "memory");
                if (!got) { ok = false; break; }
            }
            const int e = e0 + row;
            if (ok && e < p.E) {
                const float b = p.bias ? p.bias[e] : 0.f;
#pragma unroll
                for (int j = 0; j < kRmTile; ++j) {
                    const int t = t0 + j;
                    if (t < p.T) p.out[(size_t)t * p.E + e] = sum[j] + b;
                }
            }
        }
    }
    umma::fence_before();
    __syncthreads();
    if (warp == 0) {
        umma::fence_after();
        umma::tmem_dealloc(tbase, kCols);
    }
}

}  // namespace k3

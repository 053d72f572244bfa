// Decode path of the MoE layer (up to kChunk tokens per pass).
//
//   route_shared  router GEMV (fp32 weights, CUDA cores) + the shared
//                 expert's gate/up rows (bf16) + SwiGLU; the CTA that
//                 finishes the last router row then runs softmax, top-k and
//                 the expert dispatch for the chunk
//   expert_gu     routed experts' gate/up on the packed MXFP4 rows: bulk
//                 asynchronous copies into a shared-memory ring, E2M1 decoded
//                 exactly to f16 in registers, mma.sync with the tokens as
//                 the n dimension, E8M0 applied per 32-element block in fp32,
//                 SwiGLU fused
//   expert_down   down projection of every selected expert and of the shared
//                 expert, same ring + mma scheme, activations split hi/lo
//   combine       y = S + sum_j w_j o_j in slot order, rounded once
// Prior art: the kimi-k3-in-c project card ("P053"), core features (routed
// experts multiplied directly on the packed nibbles, never dequantised to a
// resident buffer); the tutorial page's section 2.4 moe_forward (route, then
// per selected expert FFN, then weighted combine).
#pragma once

#include "common.cuh"
#include "layout.cuh"

namespace k3 {

// =========================================================== route_shared ==

struct RouteParams {
    const uint16_t *x;  // bf16 [Tc][d] of this chunk
    int Tc;
    const float *wr;    // fp32 [E][d]
    const float *bias;  // fp32 [E] or null
    const uint16_t *swg, *swu;  // bf16 [ffs][d] or null
    int ffs;            // shared rows handled here (0 = none)
    int d, E, k;
    uint8_t *ws;
    Layout L;
    const uint8_t *const *blobs;  // device array [E], null: no dispatch (route only)
    int32_t *idx_out;   // optional [Tc][k]
    float *w_out;       // optional [Tc][k]
};

constexpr int kRouteThreads = 256;
constexpr int kRouteTok = 4;  // tokens per pass over the rows (x kept in smem as fp32)

// Softmax over all E logits and the top-k (descending, ties to the lower
// index) of one token, by one warp.  NPL logits per lane stay in registers.
template <int NPL>
__device__ void warp_topk(const float *row, int E, int k, int lane, int32_t *idx, float *wt,
                          int32_t *idx2, float *wt2) {
    float v[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        int e = lane + 32 * i;
        v[i] = e < E ? __ldcg(row + e) : -INFINITY;
    }
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < NPL; ++i) m = fmaxf(m, v[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        if (lane + 32 * i < E) s += expf(v[i] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float inv_s = 1.0f / s;
    uint32_t taken = 0;
    for (int j = 0; j < k; ++j) {
        float bv = 0.f;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            int e = lane + 32 * i;
            bool cand = e < E && !((taken >> i) & 1u);
            if (cand && (bi == 0x7fffffff || v[i] > bv)) {
                bv = v[i];
                bi = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            bool better = (oi != 0x7fffffff) &&
                          (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi));
            if (better) {
                bv = ov;
                bi = oi;
            }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == 0) {
            float w = expf(bv - m) * inv_s;
            idx[j] = bi;
            wt[j] = w;
            if (idx2) idx2[j] = bi;
            if (wt2) wt2[j] = w;
        }
    }
}

__device__ void topk_dispatch(const RouteParams &p, WsHeader *hdr) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Layout &L = p.L;
    float *logits = reinterpret_cast<float *>(p.ws + L.logits);
    int32_t *idx = reinterpret_cast<int32_t *>(p.ws + L.idx);
    float *wt = reinterpret_cast<float *>(p.ws + L.wt);
    __threadfence();
    if (warp < p.Tc) {
        const int t = warp;
        const float *row = logits + (size_t)t * p.E;
        int32_t *i2 = p.idx_out ? p.idx_out + (size_t)t * p.k : nullptr;
        float *w2 = p.w_out ? p.w_out + (size_t)t * p.k : nullptr;
        int32_t *i1 = idx + t * p.k;
        float *w1 = wt + t * p.k;
        if (p.E <= 32) warp_topk<1>(row, p.E, p.k, lane, i1, w1, i2, w2);
        else if (p.E <= 64) warp_topk<2>(row, p.E, p.k, lane, i1, w1, i2, w2);
        else if (p.E <= 128) warp_topk<4>(row, p.E, p.k, lane, i1, w1, i2, w2);
        else if (p.E <= 256) warp_topk<8>(row, p.E, p.k, lane, i1, w1, i2, w2);
        else if (p.E <= 512) warp_topk<16>(row, p.E, p.k, lane, i1, w1, i2, w2);
        else warp_topk<32>(row, p.E, p.k, lane, i1, w1, i2, w2);
    }
    if (p.blobs == nullptr) return;  // route only: no dispatch
    // per-token f16 prescale of x (used by the gate/up pass)
    if (warp < p.Tc) {
        const uint16_t *xr = p.x + (size_t)warp * p.d;
        float mx = 0.f;
        for (int j = lane; j < p.d; j += 32) mx = fmaxf(mx, fabsf(__uint_as_float((uint32_t)xr[j] << 16)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) reinterpret_cast<int32_t *>(p.ws + L.sigx)[warp] = f16_prescale(mx);
    }
    __syncthreads();
    // distinct experts of the chunk, ascending expert id
    __shared__ uint32_t bitmap[32];
    __shared__ uint32_t prefix[32];
    __shared__ uint32_t umask[kChunk * 32];
    const int TK = p.Tc * p.k;
    const int nwords = (p.E + 31) >> 5;
    if (threadIdx.x < 32) bitmap[threadIdx.x] = 0u;
    for (int i = threadIdx.x; i < kChunk * 32; i += blockDim.x) umask[i] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < TK; i += blockDim.x) {
        int e = idx[i];
        atomicOr(&bitmap[e >> 5], 1u << (e & 31));
    }
    __syncthreads();
    if (warp == 0) {
        uint32_t c = lane < nwords ? __popc(bitmap[lane]) : 0u;
        uint32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        prefix[lane] = incl - c;
        if (lane == 31) hdr->n_unique = incl;
    }
    __syncthreads();
    int8_t *uslot = reinterpret_cast<int8_t *>(p.ws + L.uniq_slot);
    for (int i = threadIdx.x; i < TK * kChunk; i += blockDim.x) uslot[i] = -1;
    uint32_t *hmax = reinterpret_cast<uint32_t *>(p.ws + L.hmax);
    for (int i = threadIdx.x; i < kChunk * p.k; i += blockDim.x) hmax[i] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < TK; i += blockDim.x) {
        int e = idx[i];
        int t = i / p.k, j = i - t * p.k;
        uint32_t u = prefix[e >> 5] + __popc(bitmap[e >> 5] & ((1u << (e & 31)) - 1u));
        uslot[u * kChunk + t] = (int8_t)j;
        atomicOr(&umask[u], 1u << t);
    }
    __syncthreads();
    const uint32_t U = hdr->n_unique;
    const uint8_t **ublob = reinterpret_cast<const uint8_t **>(p.ws + L.uniq_blob);
    uint32_t *gmask = reinterpret_cast<uint32_t *>(p.ws + L.uniq_mask);
    for (int w = threadIdx.x; w < nwords * 32; w += blockDim.x) {
        if ((bitmap[w >> 5] >> (w & 31)) & 1u) {
            uint32_t u = prefix[w >> 5] + __popc(bitmap[w >> 5] & ((1u << (w & 31)) - 1u));
            const uint8_t *b = p.blobs[w];
            if ((reinterpret_cast<uintptr_t>(b) & 15u) != 0u || b == nullptr) {
                set_status(hdr, kStDeviceCheck);
                b = nullptr;
            }
            ublob[u] = b;
            gmask[u] = umask[u];
        }
    }
    (void)U;
}

__global__ void __launch_bounds__(kRouteThreads) route_shared_kernel(RouteParams p) {
    extern __shared__ __align__(16) float xs[];  // [kRouteTok][d]
    __shared__ float red[kRouteThreads / 32][2 * kRouteTok];
    __shared__ int s_last;
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws + p.L.hdr);
    float *logits = reinterpret_cast<float *>(p.ws + p.L.logits);
    float *hs = reinterpret_cast<float *>(p.ws + p.L.hs);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = p.E + p.ffs;
    const int G = gridDim.x;
    const int u0 = (int)(((long long)blockIdx.x * N) / G);
    const int u1 = (int)(((long long)(blockIdx.x + 1) * N) / G);
    const int nrouter = max(0, min(u1, p.E) - u0);
    const int d = p.d;
    pdl_trigger();

    for (int t0 = 0; t0 < p.Tc; t0 += kRouteTok) {
        const int nt = min(kRouteTok, p.Tc - t0);
        __syncthreads();
        for (int i = threadIdx.x; i < nt * d / 2; i += blockDim.x) {
            int t = (2 * i) / d, j = (2 * i) % d;
            uint32_t w = reinterpret_cast<const uint32_t *>(p.x + (size_t)(t0 + t) * d)[j / 2];
            xs[t * d + j] = bf16_lo(w);
            xs[t * d + j + 1] = bf16_hi(w);
        }
        __syncthreads();
        const bool last_pass = (t0 + kRouteTok >= p.Tc);
        for (int u = u0; u < u1; ++u) {
            float a0[kRouteTok], a1[kRouteTok];
#pragma unroll
            for (int t = 0; t < kRouteTok; ++t) a0[t] = a1[t] = 0.f;
            if (u < p.E) {
                // router row u: 4 fp32 weights per 16-byte chunk
                const float4 *wr = reinterpret_cast<const float4 *>(p.wr + (size_t)u * d);
                const int nc = d / 4;
#pragma unroll 4
                for (int c = threadIdx.x; c < nc; c += kRouteThreads) {
                    float4 w = __ldg(wr + c);
#pragma unroll
                    for (int t = 0; t < kRouteTok; ++t) {
                        if (t < nt) {
                            float4 xv = *reinterpret_cast<const float4 *>(xs + t * d + 4 * c);
                            a0[t] = fmaf(w.x, xv.x, a0[t]);
                            a0[t] = fmaf(w.y, xv.y, a0[t]);
                            a0[t] = fmaf(w.z, xv.z, a0[t]);
                            a0[t] = fmaf(w.w, xv.w, a0[t]);
                        }
                    }
                }
            } else {
                // shared expert rows r of W_g,s and W_u,s: 8 bf16 per chunk
                const int r = u - p.E;
                const uint4 *wg = reinterpret_cast<const uint4 *>(p.swg + (size_t)r * d);
                const uint4 *wu = reinterpret_cast<const uint4 *>(p.swu + (size_t)r * d);
                const int nc = d / 8;
#pragma unroll 2
                for (int c = threadIdx.x; c < nc; c += kRouteThreads) {
                    uint4 g = __ldg(wg + c), v = __ldg(wu + c);
                    float gf[8] = {bf16_lo(g.x), bf16_hi(g.x), bf16_lo(g.y), bf16_hi(g.y),
                                   bf16_lo(g.z), bf16_hi(g.z), bf16_lo(g.w), bf16_hi(g.w)};
                    float uf[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                                   bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
                    for (int t = 0; t < kRouteTok; ++t) {
                        if (t < nt) {
                            float4 x0 = *reinterpret_cast<const float4 *>(xs + t * d + 8 * c);
                            float4 x1 = *reinterpret_cast<const float4 *>(xs + t * d + 8 * c + 4);
                            float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                a0[t] = fmaf(gf[i], xv[i], a0[t]);
                                a1[t] = fmaf(uf[i], xv[i], a1[t]);
                            }
                        }
                    }
                }
            }
            // block reduction, fixed order
#pragma unroll
            for (int t = 0; t < kRouteTok; ++t) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    a0[t] += __shfl_xor_sync(0xffffffffu, a0[t], o);
                    a1[t] += __shfl_xor_sync(0xffffffffu, a1[t], o);
                }
            }
            if (lane == 0) {
#pragma unroll
                for (int t = 0; t < kRouteTok; ++t) {
                    red[warp][t] = a0[t];
                    red[warp][kRouteTok + t] = a1[t];
                }
            }
            __syncthreads();
            if (threadIdx.x < nt) {
                const int t = threadIdx.x;
                float s0 = 0.f, s1 = 0.f;
#pragma unroll
                for (int w = 0; w < kRouteThreads / 32; ++w) {
                    s0 += red[w][t];
                    s1 += red[w][kRouteTok + t];
                }
                if (u < p.E) {
                    if (p.bias) s0 += p.bias[u];
                    logits[(size_t)(t0 + t) * p.E + u] = s0;
                } else {
                    hs[(size_t)(t0 + t) * p.ffs + (u - p.E)] = silu_mul(s0, s1);
                }
            }
            __syncthreads();
            // after this CTA's last router row of the last pass: count it, and the
            // CTA that completes the count runs top-k + dispatch
            if (last_pass && nrouter > 0 && u == u0 + nrouter - 1) {
                if (threadIdx.x == 0) {
                    __threadfence();
                    uint32_t old = atomicAdd(&hdr->router_done, (uint32_t)nrouter);
                    s_last = (old + (uint32_t)nrouter == (uint32_t)p.E);
                }
                __syncthreads();
                if (s_last) {
                    topk_dispatch(p, hdr);
                    __syncthreads();
                    if (threadIdx.x == 0) hdr->router_done = 0u;
                }
            }
        }
    }
}

// ============================================================== expert_gu ==

struct GUParams {
    const uint16_t *x;  // bf16 [Tc][d]
    int Tc, d, ff;
    uint8_t *ws;
    Layout L;
};

constexpr int kGUThreads = 512;  // 16 warps split each item's d columns
constexpr int kStages = 3;

__host__ __device__ inline int gu_pitch(int d) { return d / 2 + 16; }
__host__ __device__ inline int gu_stage_bytes(int d) {
    return (16 * gu_pitch(d) + 2 * 8 * (d / 32) + 127) & ~127;
}
__host__ __device__ inline int gu_smem_bytes(int d) {
    return kStages * gu_stage_bytes(d) + 2 * 16 * 8 * kChunk * 2 * 4 + kStages * 8;
}

template <int NBW>
__global__ void __launch_bounds__(kGUThreads, 1) expert_gu_kernel(GUParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int d = p.d, ff = p.ff, nb = d / 32;
    const int P = gu_pitch(d), SB = gu_stage_bytes(d);
    float *red = reinterpret_cast<float *>(smem + kStages * SB);  // [2][16][8][kChunk][2]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * SB + 2 * 16 * 8 * kChunk * 2 * 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws + p.L.hdr);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();  // the dispatch of route_shared is complete and visible
    pdl_trigger();

    const int U = (int)hdr->n_unique;
    const int nrg = ff / 8;
    const int N = U * nrg;
    const int G = gridDim.x;
    const int i0 = (int)(((long long)blockIdx.x * N) / G);
    const int i1 = (int)(((long long)(blockIdx.x + 1) * N) / G);
    const uint8_t *const *ublob = reinterpret_cast<const uint8_t *const *>(p.ws + p.L.uniq_blob);
    const uint32_t *umask = reinterpret_cast<const uint32_t *>(p.ws + p.L.uniq_mask);
    const int8_t *uslot = reinterpret_cast<const int8_t *>(p.ws + p.L.uniq_slot);
    const int32_t *sigx = reinterpret_cast<const int32_t *>(p.ws + p.L.sigx);
    float *hbuf = reinterpret_cast<float *>(p.ws + p.L.h);
    uint32_t *hmax = reinterpret_cast<uint32_t *>(p.ws + p.L.hmax);
    const int k = p.L.k;
    const size_t mat = (size_t)d * ff;

    // B fragments: token n = g, columns 8q..8q+7 of each of this warp's blocks,
    // as f16 prescaled by 2^sigx[n] (exact for the bf16 inputs in range)
    uint32_t bx[NBW][2][2];
    {
        const bool tok_ok = g < p.Tc;
        const float sc = tok_ok ? __uint_as_float((uint32_t)(127 + sigx[g]) << 23) : 0.f;
#pragma unroll
        for (int i = 0; i < NBW; ++i) {
            const int b = warp + 16 * i;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (tok_ok && b < nb)
                v = *reinterpret_cast<const uint4 *>(p.x + (size_t)g * d + 32 * b + 8 * q);
            bx[i][0][0] = pack_f16x2(bf16_lo(v.x) * sc, bf16_hi(v.x) * sc);
            bx[i][0][1] = pack_f16x2(bf16_lo(v.y) * sc, bf16_hi(v.y) * sc);
            bx[i][1][0] = pack_f16x2(bf16_lo(v.z) * sc, bf16_hi(v.z) * sc);
            bx[i][1][1] = pack_f16x2(bf16_lo(v.w) * sc, bf16_hi(v.w) * sc);
        }
    }

    auto issue = [&](int it, int s) {
        // warp 0: lane 0 arms the barrier, lanes 0..17 each issue one copy
        const int u = it / nrg, rg = it - (it / nrg) * nrg;
        const uint8_t *blob = ublob[u];
        uint8_t *st = smem + s * SB;
        const uint32_t bytes = (uint32_t)(16 * (d / 2) + 2 * 8 * (d / 32));
        if (lane == 0) {
            fence_proxy_async();
            if (blob) mbar_arrive_expect_tx(&full[s], bytes);
            else asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&full[s])) : "memory");
        }
        __syncwarp();
        if (!blob) return;
        const int r0 = rg * 8;
        if (lane < 8) {
            bulk_g2s(st + lane * P, blob + (size_t)(r0 + lane) * (d / 2), d / 2, &full[s]);
        } else if (lane < 16) {
            const int r = lane - 8;
            bulk_g2s(st + lane * P, blob + mat / 2 + mat / 32 + (size_t)(r0 + r) * (d / 2), d / 2,
                     &full[s]);
        } else if (lane == 16) {
            bulk_g2s(st + 16 * P, blob + mat / 2 + (size_t)r0 * (d / 32), 8 * (d / 32), &full[s]);
        } else if (lane == 17) {
            bulk_g2s(st + 16 * P + 8 * (d / 32), blob + mat + mat / 32 + (size_t)r0 * (d / 32),
                     8 * (d / 32), &full[s]);
        }
    };

    if (warp == 0)
        for (int s = 0; s < kStages && i0 + s < i1; ++s) issue(i0 + s, s);

    for (int it = i0; it < i1; ++it) {
        const int s = (it - i0) % kStages;
        const uint32_t par = (uint32_t)(((it - i0) / kStages) & 1);
        const bool ok = mbar_wait_bounded(&full[s], par, hdr);
        const uint8_t *st = smem + s * SB;
        float ag0 = 0.f, ag1 = 0.f, au0 = 0.f, au1 = 0.f;
        if (ok) {
#pragma unroll
            for (int i = 0; i < NBW; ++i) {
                const int b = warp + 16 * i;
                if (b < nb) {
                    const uint32_t wg = *reinterpret_cast<const uint32_t *>(st + g * P + 16 * b + 4 * q);
                    const uint32_t wu =
                        *reinterpret_cast<const uint32_t *>(st + (8 + g) * P + 16 * b + 4 * q);
                    const float fg = e8m0_to_f32(st[16 * P + g * (d / 32) + b]);
                    const float fu = e8m0_to_f32(st[16 * P + 8 * (d / 32) + g * (d / 32) + b]);
                    float c[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_f16(c, e2m1x2_to_f16x2(wg & 0xFFu), e2m1x2_to_f16x2(wu & 0xFFu),
                            e2m1x2_to_f16x2((wg >> 8) & 0xFFu), e2m1x2_to_f16x2((wu >> 8) & 0xFFu),
                            bx[i][0][0], bx[i][0][1]);
                    mma_f16(c, e2m1x2_to_f16x2((wg >> 16) & 0xFFu), e2m1x2_to_f16x2((wu >> 16) & 0xFFu),
                            e2m1x2_to_f16x2(wg >> 24), e2m1x2_to_f16x2(wu >> 24), bx[i][1][0],
                            bx[i][1][1]);
                    ag0 = fmaf(c[0], fg, ag0);
                    ag1 = fmaf(c[1], fg, ag1);
                    au0 = fmaf(c[2], fu, au0);
                    au1 = fmaf(c[3], fu, au1);
                }
            }
        }
        float *rb = red + ((it - i0) & 1) * (16 * 8 * kChunk * 2);
        *reinterpret_cast<float2 *>(rb + ((warp * 8 + g) * kChunk + 2 * q) * 2) = make_float2(ag0, au0);
        *reinterpret_cast<float2 *>(rb + ((warp * 8 + g) * kChunk + 2 * q + 1) * 2) = make_float2(ag1, au1);
        __syncthreads();
        if (warp == 0 && it + kStages < i1) issue(it + kStages, s);
        if (threadIdx.x < 8 * kChunk) {
            const int r = threadIdx.x / kChunk, t = threadIdx.x % kChunk;
            const int u = it / nrg, rg = it - u * nrg;
            if (t < p.Tc && ((umask[u] >> t) & 1u) && ublob[u] != nullptr) {
                float sg = 0.f, su = 0.f;
#pragma unroll
                for (int w = 0; w < 16; ++w) {
                    float2 v = *reinterpret_cast<const float2 *>(rb + ((w * 8 + r) * kChunk + t) * 2);
                    sg += v.x;
                    su += v.y;
                }
                const float inv = __uint_as_float((uint32_t)(127 - sigx[t]) << 23);
                const float h = silu_mul(sg * inv, su * inv);
                const int j = uslot[u * kChunk + t];
                hbuf[((size_t)t * k + j) * ff + rg * 8 + r] = h;
                atomicMax(&hmax[t * k + j], __float_as_uint(fabsf(h)));
            }
        }
    }
}

// ============================================================ expert_down ==

struct DownParams {
    int Tc, d, ff, ffs;
    const uint16_t *swd;  // bf16 [d][ffs] or null
    uint8_t *ws;
    Layout L;
};

constexpr int kDownThreads = 512;
constexpr int kDownRowsQ = 32;  // MXFP4 rows per item
constexpr int kDownRowsS = 16;  // bf16 shared rows per item

__host__ __device__ inline int dn_pitch_q(int ff) { return ff / 2 + 16; }
__host__ __device__ inline int dn_pitch_s(int ffs) { return 2 * ffs + 64; }
__host__ __device__ inline int dn_stage_bytes(int ff, int ffs) {
    int a = kDownRowsQ * dn_pitch_q(ff) + kDownRowsQ * (ff / 32);
    int b = ffs > 0 ? kDownRowsS * dn_pitch_s(ffs) : 0;
    return ((a > b ? a : b) + 127) & ~127;
}
__host__ __device__ inline int dn_smem_bytes(int ff, int ffs) {
    return kStages * dn_stage_bytes(ff, ffs) + 2 * 16 * kDownRowsQ * kChunk * 4 + kStages * 8;
}

template <int NBC>
__global__ void __launch_bounds__(kDownThreads, 1) expert_down_kernel(DownParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int d = p.d, ff = p.ff, ffs = p.ffs;
    const int SB = dn_stage_bytes(ff, ffs);
    const int PQ = dn_pitch_q(ff), PS = dn_pitch_s(ffs);
    float *red = reinterpret_cast<float *>(smem + kStages * SB);  // [2][16][32][kChunk]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * SB + 2 * 16 * kDownRowsQ * kChunk * 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws + p.L.hdr);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    const int k = p.L.k;
    const int U = (int)hdr->n_unique;
    const int nq = d / kDownRowsQ;                 // items per routed expert
    const int ns = ffs > 0 ? d / kDownRowsS : 0;   // shared items
    const int N = U * nq + ns;
    const int G = gridDim.x;
    const int i0 = (int)(((long long)blockIdx.x * N) / G);
    const int i1 = (int)(((long long)(blockIdx.x + 1) * N) / G);
    const uint8_t *const *ublob = reinterpret_cast<const uint8_t *const *>(p.ws + p.L.uniq_blob);
    const uint32_t *umask = reinterpret_cast<const uint32_t *>(p.ws + p.L.uniq_mask);
    const int8_t *uslot = reinterpret_cast<const int8_t *>(p.ws + p.L.uniq_slot);
    const float *hbuf = reinterpret_cast<const float *>(p.ws + p.L.h);
    const float *hs = reinterpret_cast<const float *>(p.ws + p.L.hs);
    const uint32_t *hmax = reinterpret_cast<const uint32_t *>(p.ws + p.L.hmax);
    float *ob = reinterpret_cast<float *>(p.ws + p.L.ob);
    const size_t mat = (size_t)d * ff;

    auto issue = [&](int it, int s) {
        uint8_t *st = smem + s * SB;
        if (it < U * nq) {
            const int u = it / nq, rb = it - u * nq;
            const uint8_t *blob = ublob[u];
            const int r0 = rb * kDownRowsQ;
            if (lane == 0) {
                fence_proxy_async();
                if (blob)
                    mbar_arrive_expect_tx(&full[s], (uint32_t)(kDownRowsQ * (ff / 2) + kDownRowsQ * (ff / 32)));
                else
                    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&full[s])) : "memory");
            }
            __syncwarp();
            if (!blob) return;
            const uint8_t *dn = blob + mat + mat / 16;  // W_d nibble plane
            bulk_g2s(st + lane * PQ, dn + (size_t)(r0 + lane) * (ff / 2), ff / 2, &full[s]);
            if (lane == 0)
                bulk_g2s(st + kDownRowsQ * PQ, dn + mat / 2 + (size_t)r0 * (ff / 32),
                         kDownRowsQ * (ff / 32), &full[s]);
        } else {
            const int r0 = (it - U * nq) * kDownRowsS;
            if (lane == 0) {
                fence_proxy_async();
                mbar_arrive_expect_tx(&full[s], (uint32_t)(kDownRowsS * 2 * ffs));
            }
            __syncwarp();
            if (lane < kDownRowsS)
                bulk_g2s(st + lane * PS, p.swd + (size_t)(r0 + lane) * ffs, 2 * ffs, &full[s]);
        }
    };

    if (warp == 0)
        for (int s = 0; s < kStages && i0 + s < i1; ++s) issue(i0 + s, s);

    // B fragments of the current expert: [block][n-group][step][2]
    uint32_t bh[NBC][2][2][2];
    int cur = -1;     // current expert slot (U = shared)
    int ntok = 0;     // tokens of the current expert
    int tok[kChunk];  // token of each column pair
#pragma unroll
    for (int i = 0; i < kChunk; ++i) tok[i] = 0;

    for (int it = i0; it < i1; ++it) {
        const bool shared_item = it >= U * nq;
        const int u = shared_item ? U : it / nq;
        const int K = shared_item ? ffs : ff;
        const int nbk = K / 32;
        if (u != cur) {
            cur = u;
            // token list of this expert
            uint32_t m = shared_item ? ((1u << p.Tc) - 1u) : umask[u];
            ntok = 0;
#pragma unroll
            for (int t = 0; t < kChunk; ++t)
                if ((m >> t) & 1u) tok[ntok++] = t;
#pragma unroll
            for (int gi = 0; gi < 2; ++gi) {
                const int mi = gi * 4 + (g >> 1);
                const bool lo_part = g & 1;
                const bool col_ok = mi < ntok && (shared_item || ublob[u] != nullptr);
                int t = 0, j = 0;
                float sc = 1.f;
                if (col_ok) {
                    t = tok[mi];
                    if (!shared_item) {
                        j = uslot[u * kChunk + t];
                        const int sg = f16_prescale(__uint_as_float(__ldcg(hmax + t * k + j)));
                        sc = __uint_as_float((uint32_t)(127 + sg) << 23);
                    }
                }
                const float *src = shared_item ? hs + (size_t)t * ffs : hbuf + ((size_t)t * k + j) * ff;
#pragma unroll
                for (int i = 0; i < NBC; ++i) {
                    const int b = warp + 16 * i;
                    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    if (col_ok && b < nbk) {
                        float4 a = __ldcg(reinterpret_cast<const float4 *>(src + 32 * b + 8 * q));
                        float4 c = __ldcg(reinterpret_cast<const float4 *>(src + 32 * b + 8 * q + 4));
                        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
                        v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
                    }
                    uint32_t r[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float x0 = v[2 * e] * sc, x1 = v[2 * e + 1] * sc;
                        if (shared_item) {
                            __nv_bfloat162 hi = __floats2bfloat162_rn(x0, x1);
                            if (!lo_part) {
                                r[e] = *reinterpret_cast<uint32_t *>(&hi);
                            } else {
                                float2 hf = __bfloat1622float2(hi);
                                r[e] = pack_bf16x2(x0 - hf.x, x1 - hf.y);
                            }
                        } else {
                            __half2 hi = __floats2half2_rn(x0, x1);
                            if (!lo_part) {
                                r[e] = *reinterpret_cast<uint32_t *>(&hi);
                            } else {
                                float2 hf = __half22float2(hi);
                                r[e] = pack_f16x2(x0 - hf.x, x1 - hf.y);
                            }
                        }
                    }
                    bh[i][gi][0][0] = r[0];
                    bh[i][gi][0][1] = r[1];
                    bh[i][gi][1][0] = r[2];
                    bh[i][gi][1][1] = r[3];
                }
            }
        }
        const int ngroups = ntok > 4 ? 2 : 1;
        const int s = (it - i0) % kStages;
        const uint32_t par = (uint32_t)(((it - i0) / kStages) & 1);
        const bool ok = mbar_wait_bounded(&full[s], par, hdr);
        const uint8_t *st = smem + s * SB;
        float acc[2][2][2];  // [row group][n-group][row g / g+8]
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b2 = 0; b2 < 2; ++b2) acc[a][b2][0] = acc[a][b2][1] = 0.f;
        const bool valid = ok && (shared_item || ublob[u] != nullptr);
        if (valid && !shared_item) {
#pragma unroll
            for (int i = 0; i < NBC; ++i) {
                const int b = warp + 16 * i;
                if (b < nbk) {
#pragma unroll
                    for (int rg = 0; rg < 2; ++rg) {
                        const int ra = rg * 16 + g;
                        const uint32_t w0 = *reinterpret_cast<const uint32_t *>(st + ra * PQ + 16 * b + 4 * q);
                        const uint32_t w1 = *reinterpret_cast<const uint32_t *>(st + (ra + 8) * PQ + 16 * b + 4 * q);
                        const float f0 = e8m0_to_f32(st[kDownRowsQ * PQ + ra * (ff / 32) + b]);
                        const float f1 = e8m0_to_f32(st[kDownRowsQ * PQ + (ra + 8) * (ff / 32) + b]);
                        const uint32_t a00 = e2m1x2_to_f16x2(w0 & 0xFFu), a01 = e2m1x2_to_f16x2(w1 & 0xFFu);
                        const uint32_t a02 = e2m1x2_to_f16x2((w0 >> 8) & 0xFFu), a03 = e2m1x2_to_f16x2((w1 >> 8) & 0xFFu);
                        const uint32_t a10 = e2m1x2_to_f16x2((w0 >> 16) & 0xFFu), a11 = e2m1x2_to_f16x2((w1 >> 16) & 0xFFu);
                        const uint32_t a12 = e2m1x2_to_f16x2(w0 >> 24), a13 = e2m1x2_to_f16x2(w1 >> 24);
#pragma unroll
                        for (int gi = 0; gi < 2; ++gi) {
                            if (gi < ngroups) {
                                float c[4] = {0.f, 0.f, 0.f, 0.f};
                                mma_f16(c, a00, a01, a02, a03, bh[i][gi][0][0], bh[i][gi][0][1]);
                                mma_f16(c, a10, a11, a12, a13, bh[i][gi][1][0], bh[i][gi][1][1]);
                                acc[rg][gi][0] = fmaf(c[0] + c[1], f0, acc[rg][gi][0]);
                                acc[rg][gi][1] = fmaf(c[2] + c[3], f1, acc[rg][gi][1]);
                            }
                        }
                    }
                }
            }
        } else if (valid) {
#pragma unroll
            for (int i = 0; i < NBC; ++i) {
                const int b = warp + 16 * i;
                if (b < nbk) {
                    const uint4 r0 = *reinterpret_cast<const uint4 *>(st + g * PS + 64 * b + 16 * q);
                    const uint4 r1 = *reinterpret_cast<const uint4 *>(st + (g + 8) * PS + 64 * b + 16 * q);
#pragma unroll
                    for (int gi = 0; gi < 2; ++gi) {
                        if (gi < ngroups) {
                            float c[4] = {0.f, 0.f, 0.f, 0.f};
                            mma_bf16(c, r0.x, r1.x, r0.y, r1.y, bh[i][gi][0][0], bh[i][gi][0][1]);
                            mma_bf16(c, r0.z, r1.z, r0.w, r1.w, bh[i][gi][1][0], bh[i][gi][1][1]);
                            acc[0][gi][0] += c[0] + c[1];
                            acc[0][gi][1] += c[2] + c[3];
                        }
                    }
                }
            }
        }
        float *rb = red + ((it - i0) & 1) * (16 * kDownRowsQ * kChunk);
        const int nrg = shared_item ? 1 : 2;
#pragma unroll
        for (int rg = 0; rg < 2; ++rg) {
            if (rg < nrg) {
#pragma unroll
                for (int gi = 0; gi < 2; ++gi) {
                    const int mi = gi * 4 + q;
                    rb[(warp * kDownRowsQ + rg * 16 + g) * kChunk + mi] = acc[rg][gi][0];
                    rb[(warp * kDownRowsQ + rg * 16 + g + 8) * kChunk + mi] = acc[rg][gi][1];
                }
            }
        }
        __syncthreads();
        if (warp == 0 && it + kStages < i1) issue(it + kStages, s);
        const int rows = shared_item ? kDownRowsS : kDownRowsQ;
        if (threadIdx.x < rows * kChunk && valid) {
            const int r = threadIdx.x / kChunk, mi = threadIdx.x % kChunk;
            if (mi < ntok) {
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < 16; ++w) sum += rb[(w * kDownRowsQ + r) * kChunk + mi];
                const int t = tok[mi];
                if (shared_item) {
                    const int r0 = (it - U * nq) * kDownRowsS;
                    ob[((size_t)t * (k + 1) + 0) * d + r0 + r] = sum;
                } else {
                    const int j = uslot[u * kChunk + t];
                    const int sg = f16_prescale(__uint_as_float(__ldcg(hmax + t * k + j)));
                    const float inv = __uint_as_float((uint32_t)(127 - sg) << 23);
                    const int r0 = (it - u * nq) * kDownRowsQ;
                    ob[((size_t)t * (k + 1) + 1 + j) * d + r0 + r] = sum * inv;
                }
            }
        }
    }
}

// ================================================================ combine ==

struct CombineParams {
    int Tc, d, k;
    bool has_shared, out_fp32;
    uint8_t *ws;
    Layout L;
    void *y;  // [Tc][d] bf16 or fp32
};

__global__ void __launch_bounds__(256) combine_kernel(CombineParams p) {
    pdl_wait();
    pdl_trigger();
    const int t = blockIdx.y;
    const int i = (blockIdx.x * 256 + threadIdx.x) * 4;
    if (i >= p.d) return;
    const float *ob = reinterpret_cast<const float *>(p.ws + p.L.ob) + (size_t)t * (p.L.k + 1) * p.d;
    const float *wt = reinterpret_cast<const float *>(p.ws + p.L.wt) + t * p.L.k;
    float4 acc = p.has_shared ? __ldcg(reinterpret_cast<const float4 *>(ob + i)) : make_float4(0, 0, 0, 0);
    for (int j = 0; j < p.k; ++j) {
        const float w = __ldcg(wt + j);
        const float4 o = __ldcg(reinterpret_cast<const float4 *>(ob + (size_t)(1 + j) * p.d + i));
        acc.x = fmaf(w, o.x, acc.x);
        acc.y = fmaf(w, o.y, acc.y);
        acc.z = fmaf(w, o.z, acc.z);
        acc.w = fmaf(w, o.w, acc.w);
    }
    if (p.out_fp32) {
        *reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.y) + (size_t)t * p.d + i) = acc;
    } else {
        __nv_bfloat162 a = __floats2bfloat162_rn(acc.x, acc.y), b = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 v = make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
        *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(p.y) + (size_t)t * p.d + i) = v;
    }
}

// ======================================================= single expert ==
// Dispatch for k3moe_expert_ffn: one expert, every token of the chunk, weight 1.

struct SingleParams {
    const uint16_t *x;
    int Tc, d;
    const uint8_t *blob;
    uint8_t *ws;
    Layout L;
};

__global__ void single_expert_setup_kernel(SingleParams p) {
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws + p.L.hdr);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    if (threadIdx.x == 0) {
        hdr->n_unique = 1u;
        const uint8_t *b = p.blob;
        if ((reinterpret_cast<uintptr_t>(b) & 15u) != 0u) {
            set_status(hdr, kStDeviceCheck);
            b = nullptr;
        }
        reinterpret_cast<const uint8_t **>(p.ws + p.L.uniq_blob)[0] = b;
        reinterpret_cast<uint32_t *>(p.ws + p.L.uniq_mask)[0] = (1u << p.Tc) - 1u;
    }
    if (threadIdx.x < kChunk) {
        const int t = threadIdx.x;
        reinterpret_cast<int8_t *>(p.ws + p.L.uniq_slot)[t] = t < p.Tc ? 0 : -1;
        reinterpret_cast<float *>(p.ws + p.L.wt)[t * p.L.k] = 1.0f;
        reinterpret_cast<uint32_t *>(p.ws + p.L.hmax)[t * p.L.k] = 0u;
    }
    if (warp < p.Tc) {
        const uint16_t *xr = p.x + (size_t)warp * p.d;
        float mx = 0.f;
        for (int j = lane; j < p.d; j += 32) mx = fmaxf(mx, fabsf(__uint_as_float((uint32_t)xr[j] << 16)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) reinterpret_cast<int32_t *>(p.ws + p.L.sigx)[warp] = f16_prescale(mx);
    }
    __threadfence();
    pdl_trigger();
}

}  // namespace k3

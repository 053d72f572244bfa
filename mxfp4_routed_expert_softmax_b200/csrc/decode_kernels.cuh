// Decode path of the MoE layer (up to kChunk tokens per pass).
//
//   route_shared  router GEMV (fp32 weights) and the shared expert's gate/up
//                 rows (bf16) + SwiGLU on CUDA cores, streamed by warps over
//                 equal slices of the weight bytes (a row split between warps
//                 is summed by the last one to finish, in a fixed order); one
//                 CTA waits for the router rows and runs softmax, top-k and the
//                 expert dispatch while the others stream the shared expert
//   expert_gu     gate/up of every selected expert on its packed MXFP4 rows:
//                 bulk asynchronous copies into a shared-memory ring, E2M1
//                 nibbles re-placed as E4M3 bytes by ALU bit operations (exact),
//                 mma.sync m16n8k32 (E4M3) against the tokens, each token's x
//                 carried as two E4M3 pieces, E8M0 block scales applied to the
//                 fp32 block sums, SwiGLU fused
//   expert_down   down projections of the selected experts (same scheme, the
//                 activations h as four E4M3 pieces) and of the bf16 shared
//                 expert (mma.sync bf16, h as hi + lo bf16)
//   combine       y = S + sum_j w_j o_j in slot order, rounded once
// The routed weights are never expanded into a resident buffer: each 4-bit
// code goes from shared memory to a register operand and into the MMA (the
// kimi-k3-in-c project card ("P053"), core features: multiply directly on the
// packed nibbles).  Layer structure: the tutorial page's section 2.4
// moe_forward (route, per selected expert FFN, weighted combine).
#pragma once

#include "common.cuh"
#include "layout.cuh"
#include "umma_kernels.cuh"

namespace k3 {

constexpr int kMaxStages = 3;

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
    int nwarps;         // streaming warps: 8 per CTA, CTAs 1.. of the grid
    uint4 tmpl[2][8];   // tensor-map templates: W_g/W_u plane, W_d plane
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

// Byte position of column c inside an even/odd-permuted row: within each
// group of 8 columns the even ones come first, then the odd ones, matching the
// even/odd nibble split of the MMA A operand.
__device__ __forceinline__ int perm8(int c) { return (c & ~7) + ((c & 1) ? 4 : 0) + ((c & 7) >> 1); }

// Per-token f16 prescale exponent s of x (max |x| 2^s in [2^14, 2^15)) and
// x * 2^s as f16 in pair order (columns 0,4,1,5,2,6,3,7 of each group of 8),
// written to the workspace for the gate/up pass.  Exact for every bf16
// element at or above 2^-17 of the token's largest |x|.  Run by one CTA.
__device__ void build_x_f16(const uint16_t *x, int Tc, int d, uint8_t *ws, const Layout &L) {
    __shared__ int s_sig[kChunk];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int t = warp; t < Tc; t += nw) {
        const uint16_t *xr = x + (size_t)t * d;
        float mx = 0.f;
        for (int j = lane; j < d; j += 32) mx = fmaxf(mx, fabsf(__uint_as_float((uint32_t)xr[j] << 16)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) {
            const int sg = f16_prescale(mx);
            s_sig[t] = sg;
            reinterpret_cast<int32_t *>(ws + L.sigx)[t] = sg;
        }
    }
    __syncthreads();
    __half *xp = reinterpret_cast<__half *>(ws + L.xp);
    for (int i = threadIdx.x; i < Tc * d; i += blockDim.x) {
        const int t = i / d, c = i - t * d;
        const float v = __uint_as_float((uint32_t)x[i] << 16) * exp2i(s_sig[t]);
        xp[(size_t)t * d + pairpos(c)] = __float2half_rn(v);
    }
}

// Top-k of every token of the chunk, then the dispatch: distinct experts in
// ascending id, their token masks, the slot of each (expert, token), the
// per-token E4M3 prescale of x, zeroed |h| maxima.  Run by one whole CTA.
__device__ void topk_dispatch(const RouteParams &p, WsHeader *hdr) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Layout &L = p.L;
    float *logits = reinterpret_cast<float *>(p.ws + L.logits);
    int32_t *idx = reinterpret_cast<int32_t *>(p.ws + L.idx);
    float *wt = reinterpret_cast<float *>(p.ws + L.wt);
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
    __syncthreads();
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
            if (b != nullptr) write_expert_tmaps(p.ws, L, (int)u, b, p.tmpl);
        }
    }
}

// Warp that holds chunk c when N chunks are split evenly over W warps
// (warp j holds [floor(jN/W), floor((j+1)N/W))).
__device__ __forceinline__ int chunk_owner(long long c, long long N, int W) {
    return (int)(((c + 1) * (long long)W - 1) / N);
}

// Row sums are ready: write the logit (router) or the SwiGLU activation (shared).
template <bool ROUTER>
__device__ __forceinline__ void finalize_row(const RouteParams &p, WsHeader *hdr, int row, int t0,
                                             int nt, const float *v0, const float *v1) {
    if (ROUTER) {
        float *logits = reinterpret_cast<float *>(p.ws + p.L.logits);
        const float b = p.bias ? p.bias[row] : 0.f;
        for (int t = 0; t < nt; ++t) logits[(size_t)(t0 + t) * p.E + row] = v0[t] + b;
    } else {
        float *hs = reinterpret_cast<float *>(p.ws + p.L.hs);
        for (int t = 0; t < nt; ++t) hs[(size_t)(t0 + t) * p.ffs + row] = silu_mul(v0[t], v1[t]);
    }
}

// One warp streams its slice of a phase's rows (router rows, or shared rows
// = [W_g,s row | W_u,s row]); every row is d*4 bytes = d/4 chunks of 16 B.
// Returns (in lane 0) the number of rows this warp finished.
template <bool ROUTER>
__device__ int stream_phase(const RouteParams &p, WsHeader *hdr, const float *xs, int t0, int nt,
                            int pass, int nrows, int j, int lane) {
    int finished = 0;
    const int d = p.d;
    const int cpr = d / 4;
    const int W = p.nwarps;
    const long long N = (long long)nrows * cpr;
    long long c = (long long)j * N / W;
    const long long cend = (long long)(j + 1) * N / W;
    const int NR = p.E + p.ffs;
    const int row_base = ROUTER ? 0 : p.E;
    float *part = reinterpret_cast<float *>(p.ws + p.L.part);    // [2][NR][kMaxSeg][8]
    uint32_t *cnt = reinterpret_cast<uint32_t *>(p.ws + p.L.cnt);  // [2][NR]
    while (c < cend) {
        const int r = (int)(c / cpr);
        const int a = (int)(c - (long long)r * cpr);
        const int b = (int)min((long long)cpr, (long long)a + (cend - c));
        float a0[kRouteTok], a1[kRouteTok];
#pragma unroll
        for (int t = 0; t < kRouteTok; ++t) a0[t] = a1[t] = 0.f;
        if (ROUTER) {
            const float4 *wrow = reinterpret_cast<const float4 *>(p.wr + (size_t)r * d);
            for (int cc = a + lane; cc < b; cc += 32 * 8) {
                float4 w[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int ci = cc + 32 * u;
                    w[u] = ci < b ? __ldg(wrow + ci) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int ci = cc + 32 * u;
                    if (ci < b) {
#pragma unroll
                        for (int t = 0; t < kRouteTok; ++t) {
                            if (t < nt) {
                                const float4 xv = *reinterpret_cast<const float4 *>(xs + t * d + 4 * ci);
                                a0[t] = fmaf(w[u].x, xv.x, a0[t]);
                                a0[t] = fmaf(w[u].y, xv.y, a0[t]);
                                a0[t] = fmaf(w[u].z, xv.z, a0[t]);
                                a0[t] = fmaf(w[u].w, xv.w, a0[t]);
                            }
                        }
                    }
                }
            }
        } else {
            const int half = cpr / 2;  // chunks of one bf16 row
            const uint4 *wg = reinterpret_cast<const uint4 *>(p.swg + (size_t)r * d);
            const uint4 *wu = reinterpret_cast<const uint4 *>(p.swu + (size_t)r * d);
            for (int cc = a + lane; cc < b; cc += 32 * 4) {
                uint4 w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int ci = cc + 32 * u;
                    w[u] = ci < b ? __ldg(ci < half ? wg + ci : wu + (ci - half)) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int ci = cc + 32 * u;
                    if (ci < b) {
                        const bool is_g = ci < half;
                        const int col = 8 * (is_g ? ci : ci - half);
                        const float wf[8] = {bf16_lo(w[u].x), bf16_hi(w[u].x), bf16_lo(w[u].y),
                                             bf16_hi(w[u].y), bf16_lo(w[u].z), bf16_hi(w[u].z),
                                             bf16_lo(w[u].w), bf16_hi(w[u].w)};
#pragma unroll
                        for (int t = 0; t < kRouteTok; ++t) {
                            if (t < nt) {
                                const float4 x0 = *reinterpret_cast<const float4 *>(xs + t * d + col);
                                const float4 x1 = *reinterpret_cast<const float4 *>(xs + t * d + col + 4);
                                float s = 0.f;
                                s = fmaf(wf[0], x0.x, s);
                                s = fmaf(wf[1], x0.y, s);
                                s = fmaf(wf[2], x0.z, s);
                                s = fmaf(wf[3], x0.w, s);
                                s = fmaf(wf[4], x1.x, s);
                                s = fmaf(wf[5], x1.y, s);
                                s = fmaf(wf[6], x1.z, s);
                                s = fmaf(wf[7], x1.w, s);
                                if (is_g) a0[t] += s;
                                else a1[t] += s;
                            }
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < kRouteTok; ++t) {
            if (t < nt) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    a0[t] += __shfl_xor_sync(0xffffffffu, a0[t], o);
                    if (!ROUTER) a1[t] += __shfl_xor_sync(0xffffffffu, a1[t], o);
                }
            }
        }
        if (a == 0 && b == cpr) {
            if (lane == 0) {
                finalize_row<ROUTER>(p, hdr, r, t0, nt, a0, a1);
                ++finished;
            }
        } else if (lane == 0) {
            // the row is split between warps: park the partial; the last to
            // arrive sums all parts in slot order and finishes the row
            const long long rs = (long long)r * cpr;
            const int first = chunk_owner(rs, N, W);
            const int nseg = chunk_owner(rs + cpr - 1, N, W) - first + 1;
            const int slot = j - first;
            const int grow = row_base + r;
            float *pp = part + (((size_t)(pass & 1) * NR + grow) * kMaxSeg) * 8;
            uint32_t *pc = cnt + (size_t)(pass & 1) * NR + grow;
#pragma unroll
            for (int t = 0; t < kRouteTok; ++t) {
                pp[slot * 8 + 2 * t] = a0[t];
                pp[slot * 8 + 2 * t + 1] = a1[t];
            }
            const uint32_t old = atom_add_acq_rel(pc, 1u);  // publish the part, see the others
            if (old == (uint32_t)(nseg - 1)) {
                float s0[kRouteTok], s1[kRouteTok];
#pragma unroll
                for (int t = 0; t < kRouteTok; ++t) s0[t] = s1[t] = 0.f;
                for (int sl = 0; sl < nseg; ++sl) {
#pragma unroll
                    for (int t = 0; t < kRouteTok; ++t) {
                        s0[t] += __ldcg(pp + sl * 8 + 2 * t);
                        s1[t] += __ldcg(pp + sl * 8 + 2 * t + 1);
                    }
                }
                *pc = 0u;
                finalize_row<ROUTER>(p, hdr, r, t0, nt, s0, s1);
                ++finished;
            }
        }
        c += b - a;
    }
    return finished;
}

__global__ void __launch_bounds__(kRouteThreads, 3) route_shared_kernel(const __grid_constant__ RouteParams p) {
    extern __shared__ __align__(16) float xs[];  // [kRouteTok][d]
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws + p.L.hdr);
    pdl_trigger();
    const int npass = (p.Tc + kRouteTok - 1) / kRouteTok;
    // the gate/up pass's pieces of x need no routing: every CTA builds a share
    if (p.blobs != nullptr)
        build_x_pieces(p.x, p.Tc, p.d, p.ws, p.L, blockIdx.x * (kRouteThreads / 32) + (threadIdx.x >> 5),
                       gridDim.x * (kRouteThreads / 32));
    if (blockIdx.x == 0) {
        // wait (bounded) for every router row of every pass, then route and dispatch
        __shared__ int s_ok;
        if (threadIdx.x == 0) {
            const uint32_t target = (uint32_t)(p.E * npass);
            const uint64_t t0 = globaltimer();
            int ok = 1;
            while (ld_acquire(&hdr->router_done) < target) {
                __nanosleep(128);
                if (globaltimer() - t0 > kWaitLimitNs) {
                    set_status(hdr, kStTimeout);
                    ok = 0;
                    break;
                }
            }
            s_ok = ok;
        }
        __syncthreads();
        if (!s_ok) return;
        topk_dispatch(p, hdr);
        __syncthreads();
        if (threadIdx.x == 0) hdr->router_done = 0u;
        return;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = (blockIdx.x - 1) * (kRouteThreads / 32) + warp;
    const int d = p.d;
    for (int pass = 0; pass < npass; ++pass) {
        const int t0 = pass * kRouteTok;
        const int nt = min(kRouteTok, p.Tc - t0);
        __syncthreads();
        for (int i = threadIdx.x; i < nt * d / 2; i += blockDim.x) {
            const int t = (2 * i) / d, c = (2 * i) % d;
            const uint32_t w = reinterpret_cast<const uint32_t *>(p.x + (size_t)(t0 + t) * d)[c / 2];
            xs[t * d + c] = bf16_lo(w);
            xs[t * d + c + 1] = bf16_hi(w);
        }
        __syncthreads();
        const int nr = stream_phase<true>(p, hdr, xs, t0, nt, pass, p.E, j, lane);
        // one release per warp: its logits are visible before they are counted
        if (lane == 0 && nr > 0) red_add_release(&hdr->router_done, (uint32_t)nr);
        if (p.ffs > 0) stream_phase<false>(p, hdr, xs, t0, nt, pass, p.ffs, j, lane);
    }
}

// ============================================================== expert_gu ==

struct GUParams {
    const uint16_t *x;  // bf16 [Tc][d]
    int Tc, d, ff;
    uint8_t *ws;
    Layout L;
    int nst;  // pipeline stages
};

constexpr int kGUThreads = 512;  // 16 warps split each item's d columns

__host__ __device__ inline int gu_pitch(int d) { return d / 2 + 16; }
__host__ __device__ inline int gu_scp(int d) { return d / 32 + 1; }
__host__ __device__ inline int gu_stage_bytes(int d) {
    return (16 * gu_pitch(d) + 16 * (d / 32) + 127) & ~127;
}
__host__ __device__ inline int gu_red_floats() { return 16 * 8 * kChunk * 2; }
__host__ __device__ inline int gu_smem_bytes(int d, int nst) {
    return nst * gu_stage_bytes(d) + 2 * 16 * gu_scp(d) * 4 + 2 * gu_red_floats() * 4 +
           kMaxStages * 8;
}

// E8M0 bytes [rows][nb] of a stage -> fp32 [rows][SCP], all threads of the
// CTA, walking (row, block) without divisions.
__device__ __forceinline__ void convert_scales(const uint8_t *sc8, float *dst, int rows, int nb,
                                               int scp, int nthreads) {
    const int step_r = nthreads / nb, step_b = nthreads - step_r * nb;
    int r = threadIdx.x / nb, b = threadIdx.x - r * nb;
    for (int i = threadIdx.x; i < rows * nb; i += nthreads) {
        dst[r * scp + b] = e8m0_to_f32(sc8[i]);
        r += step_r;
        b += step_b;
        if (b >= nb) {
            b -= nb;
            ++r;
        }
    }
}

// NBW: blocks of 32 columns per warp (>= d/32/16).
template <int NBW>
__global__ void __launch_bounds__(kGUThreads, 1) expert_gu_kernel(GUParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int d = p.d, ff = p.ff, nb = d / 32, nst = p.nst;
    const int P = gu_pitch(d), SB = gu_stage_bytes(d), SCP = gu_scp(d);
    float *scf = reinterpret_cast<float *>(smem + nst * SB);  // [2][16][SCP]
    float *red = scf + 2 * 16 * SCP;                           // [2][16][8][kChunk][2]
    uint64_t *full = reinterpret_cast<uint64_t *>(red + 2 * gu_red_floats());
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws + p.L.hdr);
    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) mbar_init(&full[s], 1);
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

    // B operand (column n = g = token): the lane's 8 columns 8q..8q+7 of a
    // block as f16 pairs (0,4) (1,5) (2,6) (3,7), matching the nibble pairs
    // the A operand is decoded into.
    uint32_t bx[NBW][2][2];
    {
        const uint8_t *xp = p.ws + p.L.xp;
#pragma unroll
        for (int i = 0; i < NBW; ++i) {
            const int b = warp + 16 * i;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (g < p.Tc && b < nb)
                v = __ldcg(reinterpret_cast<const uint4 *>(xp + ((size_t)g * d + 32 * b + 8 * q) * 2));
            bx[i][0][0] = v.x;
            bx[i][0][1] = v.y;
            bx[i][1][0] = v.z;
            bx[i][1][1] = v.w;
        }
    }

    auto issue = [&](int it, int s) {
        // warp 0: lane 0 arms the barrier, lanes 0..17 each issue one copy
        const int u = it / nrg, rg = it - (it / nrg) * nrg;
        const uint8_t *blob = ublob[u];
        uint8_t *st = smem + s * SB;
        const uint32_t bytes = (uint32_t)(16 * (d / 2) + 16 * (d / 32));
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
        for (int s = 0; s < nst && i0 + s < i1; ++s) issue(i0 + s, s);

    // The scales of item it+1 are converted before the barrier that ends item
    // it, so each item needs one barrier: it protects the stage being
    // refilled, the reduction buffer and the next item's scales.
    bool ok = true;
    if (i0 < i1) {
        ok = mbar_wait_bounded(&full[0], 0u, hdr);
        convert_scales(smem + 16 * P, scf, 16, nb, SCP, kGUThreads);
        __syncthreads();
    }
    for (int it = i0; it < i1; ++it) {
        const int s = (it - i0) % nst;
        const uint8_t *st = smem + s * SB;
        const float *sc = scf + ((it - i0) & 1) * 16 * SCP;
        float *rb = red + ((it - i0) & 1) * gu_red_floats();
        float ag0 = 0.f, ag1 = 0.f, au0 = 0.f, au1 = 0.f;
        if (ok) {
#pragma unroll
            for (int i = 0; i < NBW; ++i) {
                const int b = warp + 16 * i;
                if (b < nb) {
                    const uint32_t wg = *reinterpret_cast<const uint32_t *>(st + g * P + 16 * b + 4 * q);
                    const uint32_t wu =
                        *reinterpret_cast<const uint32_t *>(st + (8 + g) * P + 16 * b + 4 * q);
                    const float fg = sc[g * SCP + b], fu = sc[(8 + g) * SCP + b];
                    float c[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_f16(c, e2m1_pair0_f16(wg), e2m1_pair0_f16(wu), e2m1_pair1_f16(wg),
                            e2m1_pair1_f16(wu), bx[i][0][0], bx[i][0][1]);
                    mma_f16(c, e2m1_pair2_f16(wg), e2m1_pair2_f16(wu), e2m1_pair3_f16(wg),
                            e2m1_pair3_f16(wu), bx[i][1][0], bx[i][1][1]);
                    ag0 = fmaf(c[0], fg, ag0);
                    ag1 = fmaf(c[1], fg, ag1);
                    au0 = fmaf(c[2], fu, au0);
                    au1 = fmaf(c[3], fu, au1);
                }
            }
        }
        // columns 2q, 2q+1 are tokens 2q, 2q+1
        *reinterpret_cast<float2 *>(rb + ((warp * 8 + g) * kChunk + 2 * q) * 2) = make_float2(ag0, au0);
        *reinterpret_cast<float2 *>(rb + ((warp * 8 + g) * kChunk + 2 * q + 1) * 2) = make_float2(ag1, au1);
        bool ok_next = true;
        if (it + 1 < i1) {
            const int sn = (it + 1 - i0) % nst;
            ok_next = mbar_wait_bounded(&full[sn], (uint32_t)(((it + 1 - i0) / nst) & 1), hdr);
            convert_scales(smem + sn * SB + 16 * P, scf + ((it + 1 - i0) & 1) * 16 * SCP, 16, nb,
                           SCP, kGUThreads);
        }
        __syncthreads();
        if (warp == 0 && it + nst < i1) issue(it + nst, s);
        if (threadIdx.x < 8 * kChunk) {
            const int r = threadIdx.x / kChunk, t = threadIdx.x % kChunk;
            const int u = it / nrg, rg = it - u * nrg;
            if (t < p.Tc && ((umask[u] >> t) & 1u) && ublob[u] != nullptr) {
                float sg = 0.f, su = 0.f;
#pragma unroll
                for (int w = 0; w < 16; ++w) {
                    const float2 v = *reinterpret_cast<const float2 *>(rb + ((w * 8 + r) * kChunk + t) * 2);
                    sg += v.x;
                    su += v.y;
                }
                // undo the 2^-14 of the f16 placement and the x prescale
                const float inv = exp2i(14 - sigx[t]);
                const float h = silu_mul(sg * inv, su * inv);
                const int j = uslot[u * kChunk + t];
                hbuf[((size_t)t * k + j) * ff + rg * 8 + r] = h;
                atomicMax(&hmax[t * k + j], __float_as_uint(fabsf(h)));
            }
        }
        ok = ok_next;
    }
}

// ============================================================ expert_down ==

struct DownParams {
    int Tc, d, ff, ffs;
    const uint16_t *swd;  // bf16 [d][ffs] or null
    uint8_t *ws;
    Layout L;
    int nst;
    int skip_routed;  // only the shared expert's rows (the routed ones run on the tensor cores)
};

constexpr int kDownThreads = 512;
constexpr int kDownRowsQ = 64;  // MXFP4 rows per routed item (4 row groups)
constexpr int kDownRowsS = 16;  // bf16 rows per shared item

__host__ __device__ inline int dn_pitch_q(int ff) { return ff / 2 + 16; }
__host__ __device__ inline int dn_pitch_s(int ffs) { return 2 * ffs + 64; }
__host__ __device__ inline int dn_scp(int ff) { return ff / 32 + 1; }
__host__ __device__ inline int dn_pc_pitch(int ff) { return 2 * ff + 64; }  // one (token, part) f16 row
__host__ __device__ inline int dn_stage_bytes(int ff, int ffs) {
    int a = kDownRowsQ * dn_pitch_q(ff) + kDownRowsQ * (ff / 32);
    int b = ffs > 0 ? kDownRowsS * dn_pitch_s(ffs) : 0;
    return ((a > b ? a : b) + 127) & ~127;
}
// partial sums of one pass: routed [4 K-quarters][64 rows][4 tokens],
// shared [16 warps][16 rows][8 tokens]
__host__ __device__ inline int dn_red_floats() {
    const int a = 16 * 16 * kChunk, b = 4 * kDownRowsQ * 4;
    return a > b ? a : b;
}
__host__ __device__ inline int dn_smem_bytes(int ff, int ffs, int nst) {
    return nst * dn_stage_bytes(ff, ffs) + 2 * kDownRowsQ * dn_scp(ff) * 4 +
           8 * dn_pc_pitch(ff) + 2 * dn_red_floats() * 4 + kMaxStages * 8;
}

// NBQ: blocks per K-quarter for routed items (>= ff/32/4); NBS: blocks per warp
// for shared items (>= ffs/32/16).
template <int NBQ, int NBS>
__global__ void __launch_bounds__(kDownThreads, 1) expert_down_kernel(DownParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int d = p.d, ff = p.ff, ffs = p.ffs, nst = p.nst;
    const int SB = dn_stage_bytes(ff, ffs);
    const int PQ = dn_pitch_q(ff), PS = dn_pitch_s(ffs), SCP = dn_scp(ff), PCP = dn_pc_pitch(ff);
    const int nbk = ff / 32;
    float *scf = reinterpret_cast<float *>(smem + nst * SB);                // [2][64][SCP]
    uint8_t *pcs = reinterpret_cast<uint8_t *>(scf + 2 * kDownRowsQ * SCP);  // [4 tok][hi,lo][PCP]
    float *red = reinterpret_cast<float *>(pcs + 8 * PCP);                  // [2][dn_red_floats]
    uint64_t *full = reinterpret_cast<uint64_t *>(red + 2 * dn_red_floats());
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws + p.L.hdr);
    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    const int k = p.L.k;
    const int U = (int)hdr->n_unique;
    const int nq = d / kDownRowsQ;
    const int ns = ffs > 0 ? d / kDownRowsS : 0;
    const int NQ = p.skip_routed ? 0 : U * nq;
    const int N = NQ + ns;
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
        if (it < NQ) {
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
            bulk_g2s(st + (lane + 32) * PQ, dn + (size_t)(r0 + lane + 32) * (ff / 2), ff / 2, &full[s]);
            if (lane == 0)
                bulk_g2s(st + kDownRowsQ * PQ, dn + mat / 2 + (size_t)r0 * (ff / 32),
                         kDownRowsQ * (ff / 32), &full[s]);
        } else {
            const int r0 = (it - NQ) * kDownRowsS;
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
        for (int s = 0; s < nst && i0 + s < i1; ++s) issue(i0 + s, s);

    // routed items: warp = (row group rgw, K-quarter kq); B column n = g is
    // token g/2 of the pass, part g&1 (hi, lo) of its prescaled h in f16
    const int rgw = warp & 3, kq = warp >> 2;
    uint32_t bq[NBQ][2][2];
    uint32_t bs[NBS][2][2][2];  // shared: [block][token group][step][2], bf16 hi/lo
    int cur_key = -1;           // (expert, pass) whose pieces are loaded
    bool shared_loaded = false;

    // Reduce one pass of a routed item (tokens tb.. of the expert) into ob.
    auto reduce_routed = [&](const float *rb, int u, int it, int tb, int nt, const int *tok) {
        for (int i = threadIdx.x; i < kDownRowsQ * nt; i += kDownThreads) {
            const int r = i / nt, mi = i - r * nt;
            float sum = 0.f;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) sum += rb[(qq * kDownRowsQ + r) * 4 + mi];
            const int t = tok[tb + mi];
            const int j = uslot[u * kChunk + t];
            const int sgm = f16_prescale(__uint_as_float(__ldcg(hmax + t * k + j)));
            const int r0 = (it - u * nq) * kDownRowsQ;
            // undo the 2^-14 of the f16 placement and the h prescale
            ob[((size_t)t * (k + 1) + 1 + j) * d + r0 + r] = sum * exp2i(14 - sgm);
        }
    };

    // The E8M0 scales of item it+1 are converted before the barrier that ends
    // item it: one barrier per item protects the refilled stage, the
    // reduction buffer and the next item's scales.
    bool ok = true;
    if (i0 < i1) {
        ok = mbar_wait_bounded(&full[0], 0u, hdr);
        if (i0 < NQ) convert_scales(smem + kDownRowsQ * PQ, scf, kDownRowsQ, nbk, SCP, kDownThreads);
        __syncthreads();
    }
    for (int it = i0; it < i1; ++it) {
        const bool shared_item = it >= NQ;
        const int u = shared_item ? U : it / nq;
        const int s = (it - i0) % nst;
        const uint8_t *st = smem + s * SB;
        const float *sc = scf + ((it - i0) & 1) * kDownRowsQ * SCP;
        float *rb = red + ((it - i0) & 1) * dn_red_floats();
        const bool valid = ok && (shared_item || ublob[u] != nullptr);
        int ntok;
        int tok[kChunk];
        if (!shared_item) {
            const uint32_t m = umask[u];
            ntok = 0;
#pragma unroll
            for (int t = 0; t < kChunk; ++t)
                if ((m >> t) & 1u) tok[ntok++] = t;
        } else {
            ntok = p.Tc;
#pragma unroll
            for (int t = 0; t < kChunk; ++t) tok[t] = t;
        }
        const int npass = shared_item ? 1 : (ntok + 3) / 4;
        for (int pass = 0; pass < npass; ++pass) {
            const int tb = pass * 4;
            const int nt = min(4, ntok - tb);
            if (!shared_item) {
                const int key = u * 2 + pass;
                if (key != cur_key) {
                    // h of up to 4 of this expert's tokens, prescaled, as f16 hi + lo
                    // in pair order, one smem row per (token, part)
                    __syncthreads();  // earlier reads of the pieces are done
                    for (int i = threadIdx.x; i < nt * ff; i += kDownThreads) {
                        const int mi = i / ff, c = i - mi * ff;
                        float v = 0.f;
                        if (ublob[u] != nullptr) {
                            const int t = tok[tb + mi];
                            const int j = uslot[u * kChunk + t];
                            const int sgm = f16_prescale(__uint_as_float(__ldcg(hmax + t * k + j)));
                            v = __ldcg(hbuf + ((size_t)t * k + j) * ff + c) * exp2i(sgm);
                        }
                        const __half hi = __float2half_rn(v);
                        const __half lo = __float2half_rn(v - __half2float(hi));
                        reinterpret_cast<__half *>(pcs + (mi * 2 + 0) * PCP)[pairpos(c)] = hi;
                        reinterpret_cast<__half *>(pcs + (mi * 2 + 1) * PCP)[pairpos(c)] = lo;
                    }
                    __syncthreads();
                    {
                        const int mi = g >> 1, part = g & 1;
#pragma unroll
                        for (int i = 0; i < NBQ; ++i) {
                            const int b = kq + 4 * i;
                            uint4 v = make_uint4(0, 0, 0, 0);
                            if (b < nbk && mi < nt)
                                v = *reinterpret_cast<const uint4 *>(pcs + (mi * 2 + part) * PCP + (32 * b + 8 * q) * 2);
                            bq[i][0][0] = v.x;
                            bq[i][0][1] = v.y;
                            bq[i][1][0] = v.z;
                            bq[i][1][1] = v.w;
                        }
                    }
                    cur_key = key;
                }
            } else if (!shared_loaded) {
                // shared expert: h as bf16 hi + lo; token group ng = tokens 4ng..4ng+3
#pragma unroll
                for (int ng = 0; ng < 2; ++ng) {
                    const int t = 4 * ng + (g >> 1);
                    const bool lo_part = g & 1;
                    const bool col_ok = t < p.Tc;
#pragma unroll
                    for (int i = 0; i < NBS; ++i) {
                        const int b = warp + 16 * i;
                        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                        if (col_ok && b < ffs / 32) {
                            const float *src = hs + (size_t)t * ffs + 32 * b + 8 * q;
                            const float4 a = __ldcg(reinterpret_cast<const float4 *>(src));
                            const float4 c = __ldcg(reinterpret_cast<const float4 *>(src + 4));
                            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
                            v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
                        }
                        uint32_t r[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            __nv_bfloat162 hi = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
                            if (!lo_part) {
                                r[e] = *reinterpret_cast<uint32_t *>(&hi);
                            } else {
                                const float2 hf = __bfloat1622float2(hi);
                                r[e] = pack_bf16x2(v[2 * e] - hf.x, v[2 * e + 1] - hf.y);
                            }
                        }
                        bs[i][ng][0][0] = r[0];
                        bs[i][ng][0][1] = r[1];
                        bs[i][ng][1][0] = r[2];
                        bs[i][ng][1][1] = r[3];
                    }
                }
                shared_loaded = true;
            }
            float acc[2][2];  // [token group][row g / g+8]
#pragma unroll
            for (int a = 0; a < 2; ++a) acc[a][0] = acc[a][1] = 0.f;
            if (valid && !shared_item) {
                const int ra = rgw * 16 + g;
                float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                for (int i = 0; i < NBQ; ++i) {
                    const int b = kq + 4 * i;
                    if (b < nbk) {
                        const uint32_t w0 = *reinterpret_cast<const uint32_t *>(st + ra * PQ + 16 * b + 4 * q);
                        const uint32_t w1 = *reinterpret_cast<const uint32_t *>(st + (ra + 8) * PQ + 16 * b + 4 * q);
                        const float f0 = sc[ra * SCP + b], f1 = sc[(ra + 8) * SCP + b];
                        float c[4] = {0.f, 0.f, 0.f, 0.f};
                        mma_f16(c, e2m1_pair0_f16(w0), e2m1_pair0_f16(w1), e2m1_pair1_f16(w0),
                                e2m1_pair1_f16(w1), bq[i][0][0], bq[i][0][1]);
                        mma_f16(c, e2m1_pair2_f16(w0), e2m1_pair2_f16(w1), e2m1_pair3_f16(w0),
                                e2m1_pair3_f16(w1), bq[i][1][0], bq[i][1][1]);
                        // columns 2q, 2q+1: hi and lo part of token q of the pass
                        acc0 = fmaf(c[0] + c[1], f0, acc0);
                        acc1 = fmaf(c[2] + c[3], f1, acc1);
                    }
                }
                rb[(kq * kDownRowsQ + ra) * 4 + q] = acc0;
                rb[(kq * kDownRowsQ + ra + 8) * 4 + q] = acc1;
                if (pass + 1 < npass) {
                    // more tokens follow in another pass: reduce this one now
                    __syncthreads();
                    reduce_routed(rb, u, it, tb, nt, tok);
                    __syncthreads();
                }
            } else if (valid) {
#pragma unroll
                for (int i = 0; i < NBS; ++i) {
                    const int b = warp + 16 * i;
                    if (b < ffs / 32) {
                        const uint4 r0 = *reinterpret_cast<const uint4 *>(st + g * PS + 64 * b + 16 * q);
                        const uint4 r1 = *reinterpret_cast<const uint4 *>(st + (g + 8) * PS + 64 * b + 16 * q);
#pragma unroll
                        for (int ng = 0; ng < 2; ++ng) {
                            if (4 * ng < p.Tc) {
                                float c[4] = {0.f, 0.f, 0.f, 0.f};
                                mma_bf16(c, r0.x, r1.x, r0.y, r1.y, bs[i][ng][0][0], bs[i][ng][0][1]);
                                mma_bf16(c, r0.z, r1.z, r0.w, r1.w, bs[i][ng][1][0], bs[i][ng][1][1]);
                                acc[ng][0] += c[0] + c[1];
                                acc[ng][1] += c[2] + c[3];
                            }
                        }
                    }
                }
#pragma unroll
                for (int ng = 0; ng < 2; ++ng) {
                    const int t = 4 * ng + q;
                    rb[(warp * 16 + g) * kChunk + t] = acc[ng][0];
                    rb[(warp * 16 + g + 8) * kChunk + t] = acc[ng][1];
                }
            }
        }
        bool ok_next = true;
        if (it + 1 < i1) {
            const int sn = (it + 1 - i0) % nst;
            ok_next = mbar_wait_bounded(&full[sn], (uint32_t)(((it + 1 - i0) / nst) & 1), hdr);
            if (it + 1 < NQ)
                convert_scales(smem + sn * SB + kDownRowsQ * PQ, scf + ((it + 1 - i0) & 1) * kDownRowsQ * SCP,
                               kDownRowsQ, nbk, SCP, kDownThreads);
        }
        __syncthreads();
        if (warp == 0 && it + nst < i1) issue(it + nst, s);
        if (valid && !shared_item) {
            const int tb = (npass - 1) * 4;
            reduce_routed(rb, u, it, tb, ntok - tb, tok);
        } else if (valid) {
            for (int i = threadIdx.x; i < kDownRowsS * p.Tc; i += kDownThreads) {
                const int r = i / p.Tc, t = i - r * p.Tc;
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < 16; ++w) sum += rb[(w * 16 + r) * kChunk + t];
                const int r0 = (it - NQ) * kDownRowsS;
                ob[((size_t)t * (k + 1) + 0) * d + r0 + r] = sum;
            }
        }
        ok = ok_next;
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
    uint4 tmpl[2][8];
};

__global__ void single_expert_setup_kernel(const __grid_constant__ SingleParams p) {
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws + p.L.hdr);
    pdl_wait();
    if (blockIdx.x == 0) {
        if (threadIdx.x == 0) {
            hdr->n_unique = 1u;
            const uint8_t *b = p.blob;
            if ((reinterpret_cast<uintptr_t>(b) & 15u) != 0u) {
                set_status(hdr, kStDeviceCheck);
                b = nullptr;
            }
            reinterpret_cast<const uint8_t **>(p.ws + p.L.uniq_blob)[0] = b;
            reinterpret_cast<uint32_t *>(p.ws + p.L.uniq_mask)[0] = (1u << p.Tc) - 1u;
            if (b != nullptr) write_expert_tmaps(p.ws, p.L, 0, b, p.tmpl);
        }
        if (threadIdx.x < kChunk) {
            const int t = threadIdx.x;
            reinterpret_cast<int8_t *>(p.ws + p.L.uniq_slot)[t] = t < p.Tc ? 0 : -1;
            reinterpret_cast<float *>(p.ws + p.L.wt)[t * p.L.k] = 1.0f;
        }
    }
    build_x_pieces(p.x, p.Tc, p.d, p.ws, p.L, blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5),
                   gridDim.x * (blockDim.x >> 5));
    pdl_trigger();
}

}  // namespace k3

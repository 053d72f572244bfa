// Routing of one token chunk (up to kChunk tokens): the router GEMV on its
// fp32 weights, streamed by warps over equal slices of the weight bytes (a
// row split between warps is summed by the last one to finish, in a fixed
// order); one CTA waits for every router row, then runs the softmax over all
// experts, the top-k and the dispatch (distinct experts, their tensor maps).
// Every CTA first builds its share of the activation pieces the tensor-core
// gate/up pass reads.  Layer structure: the tutorial page's section 2.4
// moe_forward (route, per selected expert FFN, weighted combine); the expert
// FFNs themselves are in umma_kernels.cuh.
#pragma once

#include "common.cuh"
#include "layout.cuh"
#include "umma_kernels.cuh"

namespace k3 {

// ================================================================= route ==

struct RouteParams {
    const uint16_t *x;  // bf16 [Tc][d] of this chunk
    int Tc;
    const float *wr;    // fp32 [E][d]
    const float *bias;  // fp32 [E] or null
    int d, E, k;
    uint8_t *ws;
    Layout L;
    const uint8_t *const *blobs;  // device array [E], null: no dispatch (route only)
    int32_t *idx_out;   // optional [Tc][k]
    float *w_out;       // optional [Tc][k]
    int nwarps;         // streaming warps: 8 per CTA, CTAs 1.. of the grid
    uint4 tmpl[2][8];   // tensor-map templates: W_g/W_u plane, W_d plane
    uint4 smap[3][8];   // shared expert tensor maps (W_g, W_u, W_d), when has_shared
    int has_shared;     // the tensor-core kernels run a shared expert
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
    if (threadIdx.x == 0 && p.has_shared) write_shared_tmaps(p.ws, L, p.smap);
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

// A router row's sums are ready: write its logits (bias added).
__device__ __forceinline__ void finalize_row(const RouteParams &p, int row, int t0, int nt, const float *v) {
    float *logits = reinterpret_cast<float *>(p.ws + p.L.logits);
    const float b = p.bias ? p.bias[row] : 0.f;
    for (int t = 0; t < nt; ++t) logits[(size_t)(t0 + t) * p.E + row] = v[t] + b;
}

// One warp streams its slice of the router rows; every row is d*4 bytes =
// d/4 chunks of 16 B.  Returns (in lane 0) the number of rows it finished.
__device__ int stream_router(const RouteParams &p, const float *xs, int t0, int nt, int pass, int j, int lane) {
    int finished = 0;
    const int d = p.d;
    const int cpr = d / 4;
    const int W = p.nwarps;
    const long long N = (long long)p.E * cpr;
    long long c = (long long)j * N / W;
    const long long cend = (long long)(j + 1) * N / W;
    float *part = reinterpret_cast<float *>(p.ws + p.L.part);    // [2][E][kMaxSeg][kRouteTok]
    uint32_t *cnt = reinterpret_cast<uint32_t *>(p.ws + p.L.cnt);  // [2][E]
    while (c < cend) {
        const int r = (int)(c / cpr);
        const int a = (int)(c - (long long)r * cpr);
        const int b = (int)min((long long)cpr, (long long)a + (cend - c));
        float a0[kRouteTok];
#pragma unroll
        for (int t = 0; t < kRouteTok; ++t) a0[t] = 0.f;
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
#pragma unroll
        for (int t = 0; t < kRouteTok; ++t)
            if (t < nt)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) a0[t] += __shfl_xor_sync(0xffffffffu, a0[t], o);
        if (a == 0 && b == cpr) {
            if (lane == 0) {
                finalize_row(p, r, t0, nt, a0);
                ++finished;
            }
        } else if (lane == 0) {
            // the row is split between warps: park the partial; the last to
            // arrive sums all parts in slot order and finishes the row
            const long long rs = (long long)r * cpr;
            const int first = chunk_owner(rs, N, W);
            const int nseg = chunk_owner(rs + cpr - 1, N, W) - first + 1;
            const int slot = j - first;
            float *pp = part + (((size_t)(pass & 1) * p.E + r) * kMaxSeg) * kRouteTok;
            uint32_t *pc = cnt + (size_t)(pass & 1) * p.E + r;
#pragma unroll
            for (int t = 0; t < kRouteTok; ++t) pp[slot * kRouteTok + t] = a0[t];
            const uint32_t old = atom_add_acq_rel(pc, 1u);  // publish the part, see the others
            if (old == (uint32_t)(nseg - 1)) {
                float s0[kRouteTok];
#pragma unroll
                for (int t = 0; t < kRouteTok; ++t) s0[t] = 0.f;
                for (int sl = 0; sl < nseg; ++sl)
#pragma unroll
                    for (int t = 0; t < kRouteTok; ++t) s0[t] += __ldcg(pp + sl * kRouteTok + t);
                *pc = 0u;
                finalize_row(p, r, t0, nt, s0);
                ++finished;
            }
        }
        c += b - a;
    }
    return finished;
}

__global__ void __launch_bounds__(kRouteThreads, 3) route_kernel(const __grid_constant__ RouteParams p) {
    extern __shared__ __align__(16) float xs[];  // [kRouteTok][d]
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws + p.L.hdr);
    pdl_trigger();
    const int npass = (p.Tc + kRouteTok - 1) / kRouteTok;
    // the gate/up pass's pieces of x need no routing: every CTA builds a share
    if (p.blobs != nullptr)
        build_x_pieces(p.x, p.Tc, p.d, p.ws, p.L, blockIdx.x * (kRouteThreads / 32) + (threadIdx.x >> 5),
                       gridDim.x * (kRouteThreads / 32), p.has_shared != 0);
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
        const int nr = stream_router(p, xs, t0, nt, pass, j, lane);
        // one release per warp: its logits are visible before they are counted
        if (lane == 0 && nr > 0) red_add_release(&hdr->router_done, (uint32_t)nr);
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
                   gridDim.x * (blockDim.x >> 5), false);
    pdl_trigger();
}

}  // namespace k3

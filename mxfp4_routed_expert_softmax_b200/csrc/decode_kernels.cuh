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
    uint4 tmpl[4][8];   // tensor-map templates: W_g/W_u, W_d nibble planes; their scale planes
    int scale_mask;     // which scale-plane templates exist (bit 0: W_g/W_u, bit 1: W_d)
    uint4 smap[3][8];   // shared expert tensor maps (W_g, W_u, W_d), when has_shared
    int has_shared;     // the tensor-core kernels run a shared expert
};

constexpr int kRouteThreads = 256;
constexpr int kRouteTok = 4;  // tokens per pass over the rows (x kept in smem as fp32)

// Order-preserving 32-bit key of a float (larger float -> larger key; -0 is
// first made +0 so that equal values have equal keys) and its inverse.
__device__ __forceinline__ uint32_t fkey(float v) {
    const uint32_t u = __float_as_uint(v + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float fkey_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

constexpr uint32_t kNone = 0xffffffffu;

// The k largest keys among NPL (key, id) slots per lane (id kNone: empty),
// ties to the lower id, written by lane 0 to okey/oid (kNone once the slots
// run out).  Each lane keeps its best remaining slot; a round takes the
// warp's largest key (redux max) and, among the lanes holding it, the lowest
// id (redux min): two warp reductions and one lane's rescan of NPL slots.
template <int NPL>
__device__ void warp_select(const uint32_t (&key)[NPL], const uint32_t (&id)[NPL], int k, int lane,
                            uint32_t *okey, uint32_t *oid) {
    uint32_t taken = 0u, bk = 0u, bi = kNone;
    int bs = 0;
    auto best = [&]() {
        bk = 0u;
        bi = kNone;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            if (id[i] != kNone && !((taken >> i) & 1u) &&
                (bi == kNone || key[i] > bk || (key[i] == bk && id[i] < bi))) {
                bk = key[i];
                bi = id[i];
                bs = i;
            }
        }
    };
    best();
    for (int j = 0; j < k; ++j) {
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, bi != kNone ? bk : 0u);
        const uint32_t imin = __reduce_min_sync(0xffffffffu, (bi != kNone && bk == kmax) ? bi : kNone);
        if (imin != kNone && bi == imin) {
            taken |= 1u << bs;
            best();
        }
        if (lane == 0) {
            okey[j] = kmax;
            oid[j] = imin;
        }
    }
}

// Softmax over all E logits and the top-k (descending logit, ties to the
// lower index) of token t, by one whole CTA: each warp selects the top-k of
// its eighth of the experts (up to 4 logits per lane), warp 0 selects the
// top-k of those 8k candidates.  Thread 0 writes the results.
__device__ void cta_topk(const RouteParams &p, int t) {
    __shared__ uint32_t s_ck[8][32], s_ci[8][32];
    __shared__ float s_red[2][8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float *row = reinterpret_cast<const float *>(p.ws + p.L.logits) + (size_t)t * p.E;
    const int S = (p.E + 7) / 8;  // <= 128: 4 per lane
    float v[4];
    uint32_t key[4], id[4];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int o = lane + 32 * i, e = warp * S + o;
        const bool ok = o < S && e < p.E;
        v[i] = ok ? __ldcg(row + e) : -INFINITY;
        key[i] = fkey(v[i]);
        id[i] = ok ? (uint32_t)e : kNone;
        mx = fmaxf(mx, v[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_red[0][warp] = mx;
    __syncthreads();
    float m = s_red[0][0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, s_red[0][w]);
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (id[i] != kNone) sum += expf(v[i] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) s_red[1][warp] = sum;
    warp_select<4>(key, id, p.k, lane, s_ck[warp], s_ci[warp]);
    __syncthreads();
    if (warp != 0) return;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += s_red[1][w];
    const float inv_s = 1.0f / s;
    uint32_t ck[8], ci[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int c = lane + 32 * i, w = c / p.k, jj = c - w * p.k;
        const bool ok = w < 8;
        ck[i] = ok ? s_ck[w][jj] : 0u;
        ci[i] = ok ? s_ci[w][jj] : kNone;
    }
    __syncwarp();
    uint32_t *fk = s_ck[0], *fi = s_ci[0];  // reused for the result (lane 0 writes after reading)
    warp_select<8>(ck, ci, p.k, lane, fk, fi);
    __syncwarp();
    if (lane == 0) {
        int32_t *i1 = reinterpret_cast<int32_t *>(p.ws + p.L.idx) + t * p.k;
        float *w1 = reinterpret_cast<float *>(p.ws + p.L.wt) + t * p.k;
        for (int j = 0; j < p.k; ++j) {
            const float w = expf(fkey_value(fk[j]) - m) * inv_s;
            i1[j] = (int32_t)fi[j];
            w1[j] = w;
            if (p.idx_out) p.idx_out[(size_t)t * p.k + j] = (int32_t)fi[j];
            if (p.w_out) p.w_out[(size_t)t * p.k + j] = w;
        }
    }
}

// The dispatch of a chunk whose top-k is done: distinct experts in ascending
// id, their token masks, the slot of each (expert, token), their blob
// pointers (checked) and ids.  Run by one whole CTA.
__device__ void dispatch(const RouteParams &p, WsHeader *hdr) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Layout &L = p.L;
    const int32_t *idx = reinterpret_cast<const int32_t *>(p.ws + L.idx);
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
        const int e = __ldcg(idx + i);
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
        const int e = __ldcg(idx + i);
        int t = i / p.k, j = i - t * p.k;
        uint32_t u = prefix[e >> 5] + __popc(bitmap[e >> 5] & ((1u << (e & 31)) - 1u));
        uslot[u * kChunk + t] = (int8_t)j;
        atomicOr(&umask[u], 1u << t);
    }
    __syncthreads();
    const uint8_t **ublob = reinterpret_cast<const uint8_t **>(p.ws + L.uniq_blob);
    int32_t *ueid = reinterpret_cast<int32_t *>(p.ws + L.uniq_eid);
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
            ueid[u] = w;
            gmask[u] = umask[u];
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

// Wait (bounded) until *ctr reaches target; false (timeout bit set) if not.
__device__ bool wait_count(const uint32_t *ctr, uint32_t target, WsHeader *hdr) {
    const uint64_t t0 = globaltimer();
    while (ld_acquire(ctr) < target) {
        __nanosleep(64);
        if (globaltimer() - t0 > kWaitLimitNs) {
            set_status(hdr, kStTimeout);
            return false;
        }
    }
    return true;
}

// Cooperative launch (every CTA resident).  CTAs 1.. stream the router rows;
// once all rows are in, token t's top-k runs on CTA t mod G (all its warps),
// and CTA 0, after its own tokens, waits for the others' and dispatches.
// Meanwhile the streaming CTAs build the gate/up pass's activation pieces and
// every expert's tensor maps, which need no routing.
__global__ void __launch_bounds__(kRouteThreads, 3) route_kernel(const __grid_constant__ RouteParams p) {
    extern __shared__ __align__(16) float xs[];  // [kRouteTok][d]
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws + p.L.hdr);
    __shared__ int s_ok;
    pdl_trigger();
    const int npass = (p.Tc + kRouteTok - 1) / kRouteTok;
    const int G = gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (blockIdx.x > 0) {
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
    // top-k of this CTA's tokens once every router row is in
    if ((int)blockIdx.x < p.Tc) {
        __syncthreads();
        if (threadIdx.x == 0) s_ok = wait_count(&hdr->router_done, (uint32_t)(p.E * npass), hdr);
        __syncthreads();
        if (!s_ok) return;
        for (int t = blockIdx.x; t < p.Tc; t += G) {
            cta_topk(p, t);
            __syncthreads();
        }
        if (blockIdx.x > 0 && threadIdx.x == 0) {
            int mine = 0;
            for (int t = blockIdx.x; t < p.Tc; t += G) ++mine;
            red_add_release(&hdr->topk_done, (uint32_t)mine);  // after thread 0's own result stores
        }
    }
    if (blockIdx.x == 0) {
        int mine = 0;
        for (int t = 0; t < p.Tc; t += G) ++mine;
        if (threadIdx.x == 0) s_ok = wait_count(&hdr->topk_done, (uint32_t)(p.Tc - mine), hdr);
        __syncthreads();
        if (!s_ok) return;
        if (p.blobs != nullptr) dispatch(p, hdr);
        __syncthreads();
        if (threadIdx.x == 0) {
            hdr->router_done = 0u;
            hdr->topk_done = 0u;
        }
        return;
    }
    if (p.blobs == nullptr) return;
    // work of the gate/up pass that needs no routing
    const int j = (blockIdx.x - 1) * (kRouteThreads / 32) + warp;
    build_x_pieces(p.x, p.Tc, p.d, p.ws, p.L, j, p.nwarps, p.has_shared != 0);
    const int tid = (blockIdx.x - 1) * kRouteThreads + threadIdx.x;
    for (int e = tid; e < p.E; e += (G - 1) * kRouteThreads) {
        const uint8_t *b = p.blobs[e];
        if (b != nullptr && (reinterpret_cast<uintptr_t>(b) & 15u) == 0u) write_expert_tmaps(p.ws, p.L, e, b, p.tmpl, p.scale_mask);
    }
    if (tid == 0 && p.has_shared) write_shared_tmaps(p.ws, p.L, p.smap);
}

// ======================================================= single expert ==
// Dispatch for k3moe_expert_ffn: one expert, every token of the chunk, weight 1.

struct SingleParams {
    const uint16_t *x;
    int Tc, d;
    const uint8_t *blob;
    uint8_t *ws;
    Layout L;
    uint4 tmpl[4][8];
    int scale_mask;
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
            reinterpret_cast<int32_t *>(p.ws + p.L.uniq_eid)[0] = 0;
            reinterpret_cast<uint32_t *>(p.ws + p.L.uniq_mask)[0] = (1u << p.Tc) - 1u;
            if (b != nullptr) write_expert_tmaps(p.ws, p.L, 0, b, p.tmpl, p.scale_mask);
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

// Grouped prefill (more than one chunk of tokens): the routing of the whole
// pass, the sort of its (token, slot) pairs by expert, the activation pieces
// of every token, and the final sum of each token's expert outputs.  The
// expert projections run in umma_expert_kernel<GU, true> between the pieces
// and the sum.  Layer structure: the tutorial page's section 2.4 moe_forward
// (gate scores, softmax, top-k, the per-selected-expert FFN, the weighted
// combine) with the loop over tokens turned inside out: tokens are sorted by
// expert so that each selected expert's packed weights stream through the
// tensor cores once for all of its tokens.
#pragma once

#include "common.cuh"
#include "decode_kernels.cuh"
#include "layout.cuh"
#include "prefill_umma.cuh"
#include "umma_kernels.cuh"

namespace k3 {

// ---------------------------------------------------------------- router --
// logits[t][e] = sum_j x[t][j] W_r[e][j] (+ b[e]) in fp32 on the CUDA cores,
// every sum in ascending j (split s of nsplit takes a contiguous range of j;
// the splits are then added in s order), so the result does not depend on
// the launch shape.  CTA tile: 128 experts x 128 tokens, K in steps of 16
// through shared memory (double-buffered), 8 x 8 outputs per thread.
constexpr int kPrBM = 128, kPrBN = 128, kPrBK = 16, kPrThreads = 256;

struct PfRouterParams {
    const uint16_t *x;   // bf16 [T][d]
    const float *wr;     // fp32 [E][d]
    const float *bias;   // fp32 [E] or null (added only when nsplit == 1)
    int T, d, E;
    int nsplit;          // K splits (gridDim.z)
    float *out;          // nsplit == 1: logits [T][E]; else partials [nsplit][T][E]
};

__global__ void __launch_bounds__(kPrThreads) pf_router_kernel(const __grid_constant__ PfRouterParams p) {
    __shared__ __align__(16) float Ws[2][kPrBK][kPrBM];
    __shared__ __align__(16) float Xs[2][kPrBK][kPrBN];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int e0 = blockIdx.x * kPrBM, t0 = blockIdx.y * kPrBN;
    const int kper = ((p.d / p.nsplit) + kPrBK - 1) / kPrBK * kPrBK;
    const int kb = blockIdx.z * kper, ke = min(p.d, kb + kper);
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    float4 wreg[2];
    uint4 xreg;
    // global -> registers for the K-step at k0 (zeros outside E, T, [kb, ke))
    auto fetch = [&](int k0) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int id = tid + i * kPrThreads, e = id >> 2, kq = (id & 3) * 4;
            wreg[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (e0 + e < p.E && k0 + kq < ke)
                wreg[i] = __ldg(reinterpret_cast<const float4 *>(p.wr + (size_t)(e0 + e) * p.d + k0 + kq));
        }
        const int t = tid >> 1, kh = (tid & 1) * 8;
        xreg = make_uint4(0u, 0u, 0u, 0u);
        if (t0 + t < p.T && k0 + kh < ke)
            xreg = __ldg(reinterpret_cast<const uint4 *>(p.x + (size_t)(t0 + t) * p.d + k0 + kh));
    };
    auto stash = [&](int buf) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int id = tid + i * kPrThreads, e = id >> 2, kq = (id & 3) * 4;
            Ws[buf][kq + 0][e] = wreg[i].x;
            Ws[buf][kq + 1][e] = wreg[i].y;
            Ws[buf][kq + 2][e] = wreg[i].z;
            Ws[buf][kq + 3][e] = wreg[i].w;
        }
        const int t = tid >> 1, kh = (tid & 1) * 8;
        Xs[buf][kh + 0][t] = bf16_lo(xreg.x);
        Xs[buf][kh + 1][t] = bf16_hi(xreg.x);
        Xs[buf][kh + 2][t] = bf16_lo(xreg.y);
        Xs[buf][kh + 3][t] = bf16_hi(xreg.y);
        Xs[buf][kh + 4][t] = bf16_lo(xreg.z);
        Xs[buf][kh + 5][t] = bf16_hi(xreg.z);
        Xs[buf][kh + 6][t] = bf16_lo(xreg.w);
        Xs[buf][kh + 7][t] = bf16_hi(xreg.w);
    };
    int buf = 0;
    if (kb < ke) {
        fetch(kb);
        stash(0);
    }
    __syncthreads();
    for (int k0 = kb; k0 < ke; k0 += kPrBK) {
        const bool more = k0 + kPrBK < ke;
        if (more) fetch(k0 + kPrBK);
#pragma unroll
        for (int kk = 0; kk < kPrBK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4 *>(&Ws[buf][kk][tx * 4]);
            const float4 a1 = *reinterpret_cast<const float4 *>(&Ws[buf][kk][64 + tx * 4]);
            const float4 b0 = *reinterpret_cast<const float4 *>(&Xs[buf][kk][ty * 4]);
            const float4 b1 = *reinterpret_cast<const float4 *>(&Xs[buf][kk][64 + ty * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = __fmaf_rn(av[i], bv[j], acc[i][j]);
        }
        if (more) {
            stash(buf ^ 1);
            __syncthreads();
            buf ^= 1;
        }
    }
    float *out = p.out + (p.nsplit > 1 ? (size_t)blockIdx.z * p.T * p.E : 0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = e0 + (i < 4 ? tx * 4 + i : 64 + tx * 4 + i - 4);
        if (e >= p.E) continue;
        const float b = (p.nsplit == 1 && p.bias) ? p.bias[e] : 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int t = t0 + (j < 4 ? ty * 4 + j : 64 + ty * 4 + j - 4);
            if (t < p.T) out[(size_t)t * p.E + e] = acc[i][j] + b;
        }
    }
}

// Split-K partials -> logits, added in split order, then the bias.
struct PfRouterSumParams {
    const float *part;  // [nsplit][T][E]
    int nsplit;
    const float *bias;  // [E] or null
    int T, E;
    float *lg;          // [T][E]
};
__global__ void pf_router_sum_kernel(const __grid_constant__ PfRouterSumParams p) {
    const size_t n = (size_t)p.T * p.E;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        float s = p.part[i];
        for (int q = 1; q < p.nsplit; ++q) s += p.part[(size_t)q * n + i];
        p.lg[i] = s + (p.bias ? p.bias[i % p.E] : 0.f);
    }
}

// ------------------------------------------------------------------ top-k --
struct PfRouteParams {
    RouteParams r;       // shapes, blobs, tensor-map templates (r.L: the decode layout)
    PLayout P;
    int T;               // tokens of this pass
    int ngs;             // shared groups of this pass (0: no shared expert)
    int ff, ffs;         // expert and shared-expert hidden sizes
};

// One CTA per token: softmax over all E and the top-k (as in decode).
__global__ void __launch_bounds__(kRouteThreads) pf_topk_kernel(const __grid_constant__ PfRouteParams p) {
    const int t = blockIdx.x, E = p.r.E, k = p.r.k;
    uint8_t *ws = p.r.ws;
    cta_topk_row(reinterpret_cast<const float *>(ws + p.P.lg) + (size_t)t * E, E, k,
                 reinterpret_cast<int32_t *>(ws + p.P.idx) + (size_t)t * k,
                 reinterpret_cast<float *>(ws + p.P.wt) + (size_t)t * k,
                 p.r.idx_out ? p.r.idx_out + (size_t)t * k : nullptr, p.r.w_out ? p.r.w_out + (size_t)t * k : nullptr,
                 (p.r.route_flags & kRouteBiasSelect) ? p.r.bias : nullptr, (p.r.route_flags & kRouteRenorm) != 0,
                 nullptr, false);
}

// --------------------------------------------------------------- dispatch --
// A counting sort of the pass's T*k pairs by expert, stable in token order:
// (1) picks per (block of kPfHistTok tokens, expert); (2) per expert, the
// exclusive prefix over blocks, its total, its first position and its first
// group (one CTA); (3) each pair's position = expert start + block prefix +
// pairs of the same expert at earlier tokens of its block.
__global__ void __launch_bounds__(kRouteThreads) pf_hist_kernel(const __grid_constant__ PfRouteParams p) {
    __shared__ uint32_t h[1024];
    const int E = p.r.E, k = p.r.k;
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0u;
    __syncthreads();
    const int t0 = blockIdx.x * kPfHistTok, t1 = min(p.T, t0 + kPfHistTok);
    const int32_t *idx = reinterpret_cast<const int32_t *>(p.r.ws + p.P.idx);
    for (int i = t0 * k + threadIdx.x; i < t1 * k; i += blockDim.x) atomicAdd(&h[idx[i]], 1u);
    __syncthreads();
    uint32_t *hist = reinterpret_cast<uint32_t *>(p.r.ws + p.P.hist) + (size_t)blockIdx.x * E;
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = h[e];
    // the experts' tensor maps, spread over the CTAs
    refresh_tmaps(p.r, blockIdx.x * blockDim.x + threadIdx.x, gridDim.x * blockDim.x);
}

constexpr int kPfScanThreads = 1024;

__global__ void __launch_bounds__(kPfScanThreads) pf_scan_kernel(const __grid_constant__ PfRouteParams p) {
    __shared__ uint32_t s_tot[32];
    const int E = p.r.E, e = threadIdx.x, nhb = ceil_div(p.T, kPfHistTok);
    uint8_t *ws = p.r.ws;
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws + p.r.L.hdr);
    uint32_t *hist = reinterpret_cast<uint32_t *>(ws + p.P.hist);
    uint32_t n = 0u;
    if (e < E) {
#pragma unroll 16
        for (int b = 0; b < nhb; ++b) {
            const uint32_t v = hist[(size_t)b * E + e];
            hist[(size_t)b * E + e] = n;
            n += v;
        }
    }
    const uint32_t ng = (n + kGroup - 1) / kGroup;
    // block-wide exclusive scans of n (positions) and ng (groups) over experts
    auto scan = [&](uint32_t v) {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        uint32_t incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        __syncthreads();
        if (lane == 31) s_tot[warp] = incl;
        __syncthreads();
        uint32_t add = 0u;
        for (int w = 0; w < warp; ++w) add += s_tot[w];
        return add + incl - v;
    };
    const uint32_t pos = scan(n);
    const uint32_t g0 = scan(ng);
    __shared__ uint32_t s_ng;
    if (threadIdx.x == kPfScanThreads - 1) s_ng = g0 + ng;
    __syncthreads();
    const uint32_t NG = s_ng;
    int4 *grp = reinterpret_cast<int4 *>(ws + p.P.grp);
    if (e < E) {
        reinterpret_cast<uint32_t *>(ws + p.P.ecnt)[e] = n;
        reinterpret_cast<uint32_t *>(ws + p.P.eoff)[e] = pos;
        reinterpret_cast<uint32_t *>(ws + p.P.goff)[e] = g0;
        int ok = 1;
        if (n > 0u) {
            const uint8_t *b = p.r.blobs[e];
            if (b == nullptr || (reinterpret_cast<uintptr_t>(b) & 15u) != 0u) {
                set_status(hdr, kStDeviceCheck);
                ok = 0;
            }
        }
        for (uint32_t i = 0; i < ng; ++i)
            grp[g0 + i] = make_int4(e, (int)(pos + kGroup * i), (int)min((uint32_t)kGroup, n - kGroup * i), ok);
    }
    for (int s = threadIdx.x; s < p.ngs; s += blockDim.x)
        grp[NG + s] = make_int4(-1, kGroup * s, min(kGroup, p.T - kGroup * s), 1);
    if (threadIdx.x == 0) hdr->n_unique = NG;
}

__global__ void __launch_bounds__(kRouteThreads) pf_place_kernel(const __grid_constant__ PfRouteParams p) {
    __shared__ int32_t s_idx[kPfHistTok * 32];
    const int E = p.r.E, k = p.r.k;
    const int t0 = blockIdx.x * kPfHistTok, t1 = min(p.T, t0 + kPfHistTok);
    const int32_t *idx = reinterpret_cast<const int32_t *>(p.r.ws + p.P.idx);
    for (int i = threadIdx.x; i < (t1 - t0) * k; i += blockDim.x) s_idx[i] = idx[t0 * k + i];
    __syncthreads();
    const uint32_t *hist = reinterpret_cast<const uint32_t *>(p.r.ws + p.P.hist) + (size_t)blockIdx.x * E;
    const uint32_t *eoff = reinterpret_cast<const uint32_t *>(p.r.ws + p.P.eoff);
    const uint32_t *goff = reinterpret_cast<const uint32_t *>(p.r.ws + p.P.goff);
    int32_t *ploc = reinterpret_cast<int32_t *>(p.r.ws + p.P.ploc);
    int32_t *perm = reinterpret_cast<int32_t *>(p.r.ws + p.P.perm);
    float *pw = reinterpret_cast<float *>(p.r.ws + p.P.pw);
    const float *wt = reinterpret_cast<const float *>(p.r.ws + p.P.wt);
    for (int i = threadIdx.x; i < (t1 - t0) * k; i += blockDim.x) {
        const int e = s_idx[i], tl = i / k;
        uint32_t r = 0u;  // pairs of expert e at earlier tokens of the block (one per token at most)
        for (int q = 0; q < tl * k; ++q) r += s_idx[q] == e ? 1u : 0u;
        const int pid = (t0 + tl) * k + (i - tl * k);
        const uint32_t rel = hist[e] + r;  // rank among expert e's pairs
        perm[eoff[e] + rel] = pid;
        pw[eoff[e] + rel] = wt[pid];
        ploc[pid] = (int)((goff[e] + rel / kGroup) * kGroup + rel % kGroup);
    }
}

// Items of the expert kernels in run order: group by group (an expert's
// groups are consecutive), its 128-row blocks innermost; the shared expert's
// groups last.  Entry: (group | row block << 20, expert or -1, first position
// or token, tokens | blob ok << 8).  One thread per (group, row block).
__global__ void pf_items_kernel(const __grid_constant__ PfRouteParams p) {
    const uint8_t *ws = p.r.ws;
    const int NG = (int)*reinterpret_cast<const volatile uint32_t *>(
        &reinterpret_cast<const WsHeader *>(ws + p.r.L.hdr)->n_unique);
    const int4 *grp = reinterpret_cast<const int4 *>(ws + p.P.grp);
    int4 *itg = reinterpret_cast<int4 *>(p.r.ws + p.P.itg);
    int4 *itd = reinterpret_cast<int4 *>(p.r.ws + p.P.itd);
    const int nrb_ff = ceil_div(p.ff, kTileM), nrb_d = ceil_div(p.r.d, kTileM);
    const int nrbs_ff = p.ngs > 0 ? ceil_div(p.ffs, kTileM) : 0;
    const int per = nrb_ff > nrb_d ? nrb_ff : nrb_d;
    const long long n = (long long)(NG + p.ngs) * per;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const int g = (int)(i / per), rb = (int)(i - (long long)g * per);
        const int4 gr = __ldcg(grp + g);  // (expert or -1, first position / token, tokens, blob ok)
        const int4 rec = make_int4(g | (rb << 20), gr.x, gr.y, gr.z | (gr.w << 8));
        if (g < NG) {
            if (rb < nrb_ff) itg[(size_t)g * nrb_ff + rb] = rec;
            if (rb < nrb_d) itd[(size_t)g * nrb_d + rb] = rec;
        } else {
            const int s = g - NG;
            if (rb < nrbs_ff) itg[(size_t)NG * nrb_ff + (size_t)s * nrbs_ff + rb] = rec;
            if (rb < nrb_d) itd[(size_t)NG * nrb_d + (size_t)s * nrb_d + rb] = rec;
        }
    }
}

// -------------------------------------------------------------- x pieces --
// x as kPfPieces E2M1 pieces, written straight into the B tile of every group
// that has the token (the gate/up MMA's layout: chunk c of B row 4s + piece
// at c*(kPfN/8)*128 + (row/8)*128 + (row%8)*16, scale words [2][kPfN]).  One
// warp per (token, K-tile): the 8 blocks of 32 are quantised into a
// shared-memory staging block, then lane 4c + piece holds chunk c's 16 bytes
// of that piece and stores them for each of the token's k groups.  With a
// shared expert, x also goes as bf16 into the shared groups' tiles (MMA N =
// 32 rows, one per token; rows of absent tokens zero).
constexpr int kPrepWarps = kRouteThreads / 32;

__global__ void __launch_bounds__(kRouteThreads) pf_prep_kernel(const __grid_constant__ PfRouteParams p) {
    __shared__ __align__(16) uint8_t stage[kPrepWarps][8][kPfPieces][16];
    __shared__ __align__(16) uint8_t sstage[kPrepWarps][2][kPfPieces][4];
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5, d = p.r.d, k = p.r.k;
    const int nkt = ceil_div(d, kTileK), nb = d / 32;
    const int nkts = ceil_div(d, kTileKs);
    const int gw = blockIdx.x * kPrepWarps + wl, nw = gridDim.x * kPrepWarps;
    uint8_t *ws = p.r.ws;
    const int32_t *ploc = reinterpret_cast<const int32_t *>(ws + p.P.ploc);
    const int Tpad = p.ngs > 0 ? p.ngs * kGroup : p.T;
    for (int i = gw; i < Tpad * nkt; i += nw) {
        const int t = i / nkt, kt = i - t * nkt;
        const bool real = t < p.T;
        const int nbk = min(8, nb - kt * 8);  // 32-blocks in this K-tile
        if (lane < 8) *reinterpret_cast<uint32_t *>(&sstage[wl][lane >> 2][lane & 3][0]) = 0u;
        __syncwarp();
        for (int c = 0; c < nbk; ++c) {
            const int col = 32 * (kt * 8 + c) + lane;
            const uint16_t xv = real ? p.r.x[(size_t)t * d + col] : (uint16_t)0;
            if (real)
                quantize_pieces_t<kPfPieces>(__uint_as_float((uint32_t)xv << 16), lane, 0, c, kPfPieces * 16, 0,
                                             kPfPieces, &stage[wl][0][0][0], &sstage[wl][0][0][0]);
            if (p.ngs > 0) {
                const int gs = t / kGroup, j = t - gs * kGroup;
                uint8_t *tile = ws + p.P.xbf + ((size_t)gs * nkts + col / kTileKs) * kPfNsGU * 128;
                const int cc = (col % kTileKs) / 8, e = col % 8;
                *reinterpret_cast<uint16_t *>(tile + cc * (kPfNsGU / 8) * 128 + (j / 8) * 128 + (j % 8) * 16 + e * 2) = xv;
            }
        }
        if (!real) continue;
        __syncwarp();
        const int c = lane >> 2, pc = lane & 3;
        const uint4 row = c < nbk ? *reinterpret_cast<const uint4 *>(&stage[wl][c][pc][0]) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t sw = lane < 8 ? *reinterpret_cast<const uint32_t *>(&sstage[wl][lane >> 2][lane & 3][0]) : 0u;
        const int myloc = lane < k ? __ldcg(ploc + (size_t)t * k + lane) : 0;
        for (int j = 0; j < k; ++j) {
            const int loc = __shfl_sync(0xffffffffu, myloc, j);
            const int g = loc / kGroup, s = loc - g * kGroup;
            const size_t tb = (size_t)g * nkt + kt;
            uint8_t *tile = ws + p.P.xg + tb * kPfN * 128;
            *reinterpret_cast<uint4 *>(tile + c * (kPfN / 8) * 128 + (s >> 1) * 128 + (s & 1) * 64 + pc * 16) = row;
            if (lane < 8)
                reinterpret_cast<uint32_t *>(ws + p.P.xgs + tb * 2 * kPfN * 4)[(lane >> 2) * kPfN + 4 * s + (lane & 3)] = sw;
        }
        __syncwarp();
    }
}

// ------------------------------------------------------------- pre-norm --
// xn[t] = RMSNorm(h[t]) rounded to bf16, one warp per token (the same
// per-token arithmetic as the decode kernel's).
struct PfNormParams {
    const uint16_t *h;       // bf16 [T][d]
    const uint16_t *norm_w;  // bf16 [d]
    float eps;
    int T, d;
    uint16_t *xn;            // bf16 [T][d]
};
__global__ void pf_rmsnorm_kernel(const __grid_constant__ PfNormParams p) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= p.T) return;
    const uint16_t *h = p.h + (size_t)t * p.d;
    const float r = warp_rms_inv(h, p.d, p.eps);
    for (int j = lane; j < p.d; j += 32) p.xn[(size_t)t * p.d + j] = rms_norm_bf16(h[j], r, p.norm_w[j]);
}

// -------------------------------------------------------------- combine --
// y[t] = sum_j o[t][j] (j < k, routing weights already applied) + o[t][k]
// (the shared expert), in that order (+ the residual h[t] for pre-norm
// calls), rounded once.
struct PfCombineParams {
    const float *o;      // [T][k+1][d]
    int T, d, k, has_shared, out_fp32;
    void *y;             // [T][d]
    const uint16_t *resid;  // bf16 [T][d] or null
};

__global__ void pf_combine_kernel(const __grid_constant__ PfCombineParams p) {
    const int nq = p.d / 4;
    const size_t n = (size_t)p.T * nq;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const size_t t = i / nq, q = i - t * nq;
        const float4 *src = reinterpret_cast<const float4 *>(p.o + t * (size_t)(p.k + 1) * p.d) + q;
        float4 s = __ldcs(src);
        const int ns = p.k + (p.has_shared ? 1 : 0);
        for (int j = 1; j < ns; ++j) {
            const float4 v = __ldcs(src + (size_t)j * nq);
            s.x += v.x;
            s.y += v.y;
            s.z += v.z;
            s.w += v.w;
        }
        if (p.resid) {
            const uint2 hv = *reinterpret_cast<const uint2 *>(p.resid + 4 * i);
            s.x += bf16_lo(hv.x);
            s.y += bf16_hi(hv.x);
            s.z += bf16_lo(hv.y);
            s.w += bf16_hi(hv.y);
        }
        if (p.out_fp32) {
            reinterpret_cast<float4 *>(p.y)[i] = s;
        } else {
            __nv_bfloat162 a = __floats2bfloat162_rn(s.x, s.y), b = __floats2bfloat162_rn(s.z, s.w);
            uint2 w;
            w.x = *reinterpret_cast<uint32_t *>(&a);
            w.y = *reinterpret_cast<uint32_t *>(&b);
            reinterpret_cast<uint2 *>(p.y)[i] = w;
        }
    }
}

}  // namespace k3

// The whole decode layer for one pass of up to kChunk tokens in ONE
// persistent launch (one CTA per SM): router GEMV, softmax and top-k, the
// dispatch, the shared expert and the routed experts' gate/up + SwiGLU and
// down projections with the weighted combine.  Layer structure: the tutorial
// page's section 2.4 moe_forward (gate scores over all experts, softmax,
// top-k, each selected expert's FFN, weighted combine) and section 1.2's
// always-on shared expert; the routed experts' packed MXFP4 weights go
// straight into the tensor cores (the kimi-k3-in-c project card, core
// features).
//
// Every CTA runs the same four ranges of "units" (each range split evenly
// over the CTAs, stream-K) through one ring of shared-memory stages:
//   R0  the fp32 router, 32 KB per unit (bulk copies), summed on the CUDA
//       cores by the scale warps (their tensor-memory work starts later);
//   R1  the shared expert's gate/up (bf16 MMAs, x as bf16);
//   R2  the routed experts' gate/up (block-scaled kind::mxf4 MMAs, x as E2M1
//       pieces), once the routing is known;
//   R3  the down projections: one accumulator per 128 rows of d, K running
//       over every distinct routed expert's ff (two 256-weight K-tiles per
//       unit) and then the shared expert's ff_s (two 64-weight bf16 K-tiles
//       per unit), so the routing weights (folded into the activation pieces)
//       and the shared expert are combined by the tensor core itself.
// So the router bytes and the shared expert stream while the routing is
// still being decided, and the W_d tiles of the first down units are loaded
// before the gate/up results they multiply are complete (only their B tiles
// wait).
//
// Routing in every CTA: once all router rows are in (a counter in the
// workspace header), warps 0-3 and 10 each take a token and find its top-k
// with warp reductions, then warp 10 builds the dispatch (distinct experts in
// ascending id, each token's weight per expert) in shared memory -- every CTA
// derives the same routing from the same logits, so no further grid-wide
// exchange is needed before the routed units start.
//
// Roles (352 threads): warps 0-3 epilogue (one TMEM lane quadrant each; they
// also take part in the top-k), warps 4-7 router sums (R0) and scale factors
// into TMEM (R2, R3), warp 8 copies (TMA, bulk), warp 9 MMA issue, warp 10
// set-up (tensor maps, activation pieces), top-k and dispatch.
#pragma once

#include "common.cuh"
#include "decode_kernels.cuh"
#include "layout.cuh"
#include "umma.cuh"
#include "umma_kernels.cuh"

namespace k3 {

constexpr int kLThreads = 352;
constexpr int kLMaxCtas = 160;        // grid cap (one CTA per SM)
constexpr int kLRUnit = 8192;         // router floats per R0 unit at most (32 KB): whole rows
constexpr int kRMaxRows = 72;         // router rows one CTA sums at most
constexpr int kLSfc = 32;             // TMEM scale columns per stage
constexpr int kLTopkWarps = 5;        // warps 0-3 and 10
constexpr int kTkCand = 128;          // top-k candidates per warp (scratch: keys, then ids)
constexpr int kTkWords = 2 * kTkCand + 4;  // a top-k warp's scratch: candidates, count, max, sum

struct LayerParams {
    RouteParams r;     // x, Tc, router, shapes, workspace, blobs, maps, wait_ns
    int ff, ffs;       // expert and shared-expert hidden sizes (ffs 0: none)
    int nst, sb;       // pipeline stages, bytes per stage
    int sf_tma_gu;     // W_g / W_u scales by TMA (d a multiple of 512)
    int sf_tma_dn;     // W_d scales by TMA (ff a multiple of 512)
    int out_fp32;
    void *y;           // [Tc][d] of this pass
    int strict;        // flag E8M0 NaN bytes among the weight scales read
    int inject;        // failure-path tests: 1 = the routing is never signalled
    // pre-norm and residual (null: the layer alone): r.x holds the residual
    // stream h; the layer's input is x = RMSNorm(h) with these weights, and
    // the output y + resid
    const uint16_t *norm_w;  // bf16 [d]
    float eps;
    const uint16_t *resid;   // bf16 [Tc][d], added to the layer's output before its rounding
    // kLayerFull; kLayerRouteOnly: stop after the top-k (CTA 0 writes the
    // routing into the workspace); kLayerRouted: take the routing from the
    // workspace (written by a route-only launch of the same pass) instead of
    // computing it -- the two launches together give the bits of one full one
    int mode;
};
constexpr int kLayerFull = 0, kLayerRouteOnly = 1, kLayerRouted = 2;

// ---------------------------------------------------------- smem layout --
// One stage: two A boxes (2 x 16 KB, 1024-byte aligned for the 128-byte
// swizzle; a router unit fills both), two B tiles of N rows x 128 bytes, two
// A scale boxes (128 rows x 16 bytes), two B scale blocks (2 x kSfRow words).
__host__ __device__ inline int lk_b_off() { return 2 * kAtile; }
__host__ __device__ inline int lk_sfa_off(int N) { return 2 * kAtile + 2 * N * 128; }
__host__ __device__ inline int lk_sfb_off(int N) { return lk_sfa_off(N) + 2 * 2048; }
__host__ __device__ inline int lk_stage_bytes(int N) { return (lk_sfb_off(N) + 2 * 2 * kSfRow * 4 + 1023) & ~1023; }

// Router rows per R0 unit: as many whole rows of d floats as fit in kLRUnit.
__host__ __device__ inline int lk_rows_per_unit(int d) { return d >= kLRUnit ? 1 : kLRUnit / d; }

// The rest, after the stages (byte offsets from the end of the stages),
// sized for this pass: E experts, top-k, Tc tokens, hidden size d.
struct LkSmem {
    int bars, ptab, blob, eid, wu, tidx, tw, racc, misc, rn, tk, total;
};
__host__ __device__ inline LkSmem lk_smem(int E, int k, int Tc, int d) {
    LkSmem s;
    const int umax = E < Tc * k ? E : Tc * k;
    auto a16 = [](int v) { return (v + 15) & ~15; };
    int o = 0;
    s.bars = o;   o += 512;                           // mbarriers, TMEM slot, flags
    s.ptab = o;   o += a16(E * 8);                    // blob pointer of every expert
    s.blob = o;   o += a16(umax * 8);                 // per distinct expert: blob pointer,
    s.eid = o;    o += a16(umax * 4);                 //   expert id,
    s.wu = o;     o += a16(umax * Tc * 4);            //   weight of each token (0: not selected)
    s.tidx = o;   o += Tc * 32 * 4;                   // top-k of each token: experts
    s.tw = o;     o += Tc * 32 * 4;                   //   and weights
    s.racc = o;   o += a16(4 * kRMaxRows * Tc * 4);   // router row sums of this CTA's rows, per warp
    s.misc = o;   o += 64 * 4;                        // dispatch bitmap / prefix
    s.rn = o;     o += kChunk * 4;                    // 1 / rms of each token (pre-norm)
    s.tk = o;     o += kLTopkWarps * kTkWords * 4;   // top-k candidates of each top-k warp
    s.total = o;
    return s;
}
__host__ __device__ inline int lk_smem_bytes(int N, int nst, int E, int k, int Tc, int d) {
    return 1024 + nst * lk_stage_bytes(N) + lk_smem(E, k, Tc, d).total;
}

// --------------------------------------------------------------- top-k --
// Softmax over all E logits and the top-k of one token, by one warp.  Lane l
// holds experts l, l + 32, ...  Picks come out in descending key (the
// order-preserving bits of the logit) with ties to the lower expert id.
// w = exp(l - max) / sum over all E of exp(l_e - max), fp32.  sel_bias
// (non-null): the selection runs on l + sel_bias[e], the softmax on l;
// renorm: the k weights are divided by their sum.
//
// Selection: the k-th largest of the 32 lane maxima, L, is a lower bound of
// the k-th largest key (k lanes hold a key >= L), so only keys >= L can be
// picked; those candidates (about k plus a few for spread logits) go to the
// warp's scratch and the k rounds (warp max of the lanes' best candidate,
// lowest id among equal keys) run over at most four per lane.  More than
// kTkCand candidates (many equal keys) take the rounds over all keys.
__device__ void warp_topk(const float *row, int E, int k, int32_t *idx_out, float *w_out,
                          const float *sel_bias, bool renorm, uint32_t *scratch) {
    const int lane = threadIdx.x & 31;
    constexpr int kPer = 32;  // E <= 1024
    uint32_t key[kPer];
    float mx = -INFINITY;
    uint32_t lmax = 0u;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        const float v = e < E ? __ldcg(row + e) : -INFINITY;
        key[i] = e < E ? fkey(sel_bias ? v + __ldg(sel_bias + e) : v) : 0u;  // real keys are > 0
        mx = fmaxf(mx, v);
        lmax = max(lmax, key[i]);
    }
    const float m = fkey_value(__reduce_max_sync(0xffffffffu, fkey(mx)));
    // the softmax runs on the logits themselves (read again when the keys
    // hold biased scores)
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        if (e < E) sum += expf((sel_bias ? __ldcg(row + e) : fkey_value(key[i])) - m);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv_s = 1.0f / sum;

    // L: the lane maximum of rank k - 1 (larger first, lower lane first)
    int rank = 0;
#pragma unroll
    for (int o = 0; o < 32; ++o) {
        const uint32_t other = __shfl_sync(0xffffffffu, lmax, o);
        rank += (other > lmax || (other == lmax && o < lane)) ? 1 : 0;
    }
    const uint32_t at = __ballot_sync(0xffffffffu, rank == k - 1);
    const uint32_t L = __shfl_sync(0xffffffffu, lmax, __ffs(at) - 1);
    int c = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) c += key[i] >= L ? 1 : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (total <= kTkCand) {
        int pos = incl - c;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            if (key[i] >= L) {
                scratch[pos] = key[i];
                scratch[kTkCand + pos] = (uint32_t)(lane + 32 * i);
                ++pos;
            }
        }
        __syncwarp();
        uint32_t ck[kTkCand / 32], ci[kTkCand / 32];
#pragma unroll
        for (int q = 0; q < kTkCand / 32; ++q) {
            const int j = 32 * q + lane;
            ck[q] = j < total ? scratch[j] : 0u;
            ci[q] = j < total ? scratch[kTkCand + j] : 0xFFFFFFFFu;
        }
        for (int j = 0; j < k; ++j) {
            uint32_t bk = 0u, bi = 0xFFFFFFFFu;
#pragma unroll
            for (int q = 0; q < kTkCand / 32; ++q) {
                if (ck[q] > bk || (ck[q] == bk && ci[q] < bi)) {
                    bk = ck[q];
                    bi = ci[q];
                }
            }
            const uint32_t K = __reduce_max_sync(0xffffffffu, bk);
            const uint32_t win = __reduce_min_sync(0xffffffffu, bk == K ? bi : 0xFFFFFFFFu);
            if (lane == 0) {
                idx_out[j] = (int32_t)win;
                w_out[j] = fkey_value(K);  // the pick's key value (its logit when unbiased)
            }
#pragma unroll
            for (int q = 0; q < kTkCand / 32; ++q)
                if (ci[q] == win) ck[q] = 0u;
        }
    } else {
        // every key is a candidate: the rounds over all of them
        uint32_t taken = 0u;
        for (int j = 0; j < k; ++j) {
            uint32_t bk = 0u;
            int bq = -1;
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const uint32_t kv = ((taken >> i) & 1u) ? 0u : key[i];
                if (kv > bk) {
                    bk = kv;
                    bq = i;
                }
            }
            const uint32_t K = __reduce_max_sync(0xffffffffu, bk);
            const uint32_t cand = (bk == K && bq >= 0) ? (uint32_t)(lane + 32 * bq) : 0xFFFFFFFFu;
            const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
            if (lane == 0) {
                idx_out[j] = (int32_t)win;
                w_out[j] = fkey_value(K);
            }
            if ((int)(win & 31u) == lane) taken |= 1u << bq;
        }
    }
    __syncwarp();
    // weights: lane j takes pick j
    float num = 0.f;
    if (lane < k) {
        const float lv = sel_bias ? __ldcg(row + idx_out[lane]) : w_out[lane];
        num = expf(lv - m);
    }
    float w = num * inv_s;
    if (renorm) {
        float z = num;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        w = num / z;
    }
    __syncwarp();
    if (lane < k) w_out[lane] = w;
    __syncwarp();
}

// One token's top-k by four warps (one token per pass is the decode case):
// warp q takes the slice [e0, e1) of the row (lane l: e0 + l + 32 i) and
// posts its candidates (keys >= the k-th largest of its 32 lane maxima, so
// every key of the token's top-k that lies in the slice) with their ids,
// their count (kTkCand + 1 when they do not fit) and its softmax partial:
// max of the logits and sum of exp(l - max) over the slice.
__device__ void warp_topk_part(const float *row, int e0, int e1, int k, const float *sel_bias, uint32_t *scratch) {
    const int lane = threadIdx.x & 31;
    constexpr int kPer = 8;  // slices of at most 256
    uint32_t key[kPer];
    float val[kPer];
    float mx = -INFINITY;
    uint32_t lmax = 0u;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = e0 + lane + 32 * i;
        const float v = e < e1 ? __ldcg(row + e) : -INFINITY;
        val[i] = v;
        key[i] = e < e1 ? fkey(sel_bias ? v + __ldg(sel_bias + e) : v) : 0u;  // real keys are > 0
        mx = fmaxf(mx, v);
        lmax = max(lmax, key[i]);
    }
    const float m = fkey_value(__reduce_max_sync(0xffffffffu, fkey(mx)));
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
        if (e0 + lane + 32 * i < e1) sum += expf(val[i] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    int rank = 0;
#pragma unroll
    for (int o = 0; o < 32; ++o) {
        const uint32_t other = __shfl_sync(0xffffffffu, lmax, o);
        rank += (other > lmax || (other == lmax && o < lane)) ? 1 : 0;
    }
    const uint32_t at = __ballot_sync(0xffffffffu, rank == k - 1);
    const uint32_t L = at ? __shfl_sync(0xffffffffu, lmax, __ffs(at) - 1) : 0u;
    int c = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) c += (key[i] != 0u && key[i] >= L) ? 1 : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (total <= kTkCand) {
        int pos = incl - c;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            if (key[i] != 0u && key[i] >= L) {
                scratch[pos] = key[i];
                scratch[kTkCand + pos] = (uint32_t)(e0 + lane + 32 * i);
                ++pos;
            }
        }
    }
    if (lane == 0) {
        scratch[2 * kTkCand] = (uint32_t)(total <= kTkCand ? total : kTkCand + 1);
        scratch[2 * kTkCand + 1] = __float_as_uint(m);
        scratch[2 * kTkCand + 2] = __float_as_uint(sum);
    }
}

// The merge of the four parts by one warp: the k rounds over the union of
// the candidates (warp max of the lanes' best, lowest id among equal keys),
// the softmax from the parts' partials (max over the parts, sums rescaled to
// it).  False (nothing written) when the candidates do not fit: the caller
// then runs warp_topk over the whole row.
__device__ bool warp_topk_merge(const float *row, int k, int32_t *idx_out, float *w_out, const float *sel_bias,
                                bool renorm, const uint32_t *scratch) {
    const int lane = threadIdx.x & 31;
    int cnt[4], off[4], C = 0;
    bool fit = true;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        cnt[q] = (int)scratch[q * kTkWords + 2 * kTkCand];
        fit = fit && cnt[q] <= kTkCand;
        off[q] = C;
        C += cnt[q];
    }
    if (!fit || C > kTkCand) return false;
    float m = -INFINITY;
#pragma unroll
    for (int q = 0; q < 4; ++q) m = fmaxf(m, __uint_as_float(scratch[q * kTkWords + 2 * kTkCand + 1]));
    float z = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float mq = __uint_as_float(scratch[q * kTkWords + 2 * kTkCand + 1]);
        const float sq = __uint_as_float(scratch[q * kTkWords + 2 * kTkCand + 2]);
        if (sq > 0.f) z += sq * expf(mq - m);
    }
    uint32_t ck[kTkCand / 32], ci[kTkCand / 32];
#pragma unroll
    for (int r = 0; r < kTkCand / 32; ++r) {
        const int j = 32 * r + lane;
        ck[r] = 0u;
        ci[r] = 0xFFFFFFFFu;
        if (j < C) {
            int q = 0, base = 0;
#pragma unroll
            for (int qq = 1; qq < 4; ++qq) {
                if (j >= off[qq]) {
                    q = qq;
                    base = off[qq];
                }
            }
            ck[r] = scratch[q * kTkWords + (j - base)];
            ci[r] = scratch[q * kTkWords + kTkCand + (j - base)];
        }
    }
    for (int j = 0; j < k; ++j) {
        uint32_t bk = 0u, bi = 0xFFFFFFFFu;
#pragma unroll
        for (int r = 0; r < kTkCand / 32; ++r) {
            if (ck[r] > bk || (ck[r] == bk && ci[r] < bi)) {
                bk = ck[r];
                bi = ci[r];
            }
        }
        const uint32_t K = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t win = __reduce_min_sync(0xffffffffu, bk == K ? bi : 0xFFFFFFFFu);
        if (lane == 0) {
            idx_out[j] = (int32_t)win;
            w_out[j] = fkey_value(K);
        }
#pragma unroll
        for (int r = 0; r < kTkCand / 32; ++r)
            if (ci[r] == win) ck[r] = 0u;
    }
    __syncwarp();
    float num = 0.f;
    if (lane < k) {
        const float lv = sel_bias ? __ldcg(row + idx_out[lane]) : w_out[lane];
        num = expf(lv - m);
    }
    float w = num / z;
    if (renorm) {
        float zz = num;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) zz += __shfl_xor_sync(0xffffffffu, zz, o);
        w = num / zz;
    }
    __syncwarp();
    if (lane < k) w_out[lane] = w;
    __syncwarp();
    return true;
}

// --------------------------------------------------------------- kernel --
// kTc: the tokens of the pass when fixed at compile time (1: one decode
// token, every per-token loop folds to one iteration and the code the SM
// fetches shrinks accordingly), 0: from the parameters.  kSf: the A scale
// boxes come by TMA (both reduction lengths multiples of 512), fixed at
// compile time; false: from the parameters.
template <int kTc, bool kSf>
__global__ void __launch_bounds__(kLThreads, 1) layer_kernel(const __grid_constant__ LayerParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const RouteParams &rp = p.r;
    const Layout &L = rp.L;
    const int nst = p.nst, SB = p.sb, Tc = kTc > 0 ? kTc : rp.Tc, N = act_n(Tc);
    const bool sf_gu = kSf || p.sf_tma_gu, sf_dn = kSf || p.sf_tma_dn;
    // accumulator chains: each matrix slot of 64 columns holds Q chains of W
    // columns (independent MMAs overlap in the tensor pipe; the epilogue sums)
    const int Q = N <= 32 ? 2 : 1, W = 64 / Q;
    const int d = rp.d, E = rp.E, k = rp.k;
    const LkSmem so = lk_smem(E, k, Tc, d);
    uint8_t *tail = smem + nst * SB;
    uint64_t *full = reinterpret_cast<uint64_t *>(tail + so.bars);  // stage bytes landed
    uint64_t *sfr = full + 8;                                        // stage scales in TMEM (4 warps)
    uint64_t *empty = sfr + 8;                                       // stage consumed
    uint64_t *afull = empty + 8;
    uint64_t *aempty = afull + 2;
    uint64_t *mready = aempty + 2;  // the routing is in shared memory
    uint64_t *mdone = mready + 1;   // every MMA this CTA issued has completed
    uint64_t *rnready = mdone + 1;  // the tokens' 1 / rms are in shared memory (pre-norm)
    uint64_t *rdready = rnready + 1;  // every router row is in (warp 0 polled router_done)
    uint64_t *tkready = rdready + 1;  // the top-k warps are done (picks in shared memory)
    uint64_t *tkpart = tkready + 1;   // the four parts of a one-token top-k are posted
    uint32_t *tslot = reinterpret_cast<uint32_t *>(tkpart + 1);
    volatile int *s_abort = reinterpret_cast<volatile int *>(tslot + 1);
    volatile int *s_U = s_abort + 1;
    volatile int *s_last = s_abort + 2;
    volatile int *s_rdone = s_abort + 3;  // router rows this CTA finished
    volatile int *s_rok = s_abort + 4;    // every router row is in (top-k warps)
    int *s_r0c = const_cast<int *>(s_abort) + 8;  // [stage]: warps done with a router unit
    const uint8_t **s_ptab = reinterpret_cast<const uint8_t **>(tail + so.ptab);
    const uint8_t **s_blob = reinterpret_cast<const uint8_t **>(tail + so.blob);
    int32_t *s_eid = reinterpret_cast<int32_t *>(tail + so.eid);
    float *s_wu = reinterpret_cast<float *>(tail + so.wu);      // [u][Tc]
    int32_t *s_tidx = reinterpret_cast<int32_t *>(tail + so.tidx);  // [t][32]
    float *s_tw = reinterpret_cast<float *>(tail + so.tw);
    float *s_racc = reinterpret_cast<float *>(tail + so.racc);  // [warp][row][Tc]
    uint32_t *s_misc = reinterpret_cast<uint32_t *>(tail + so.misc);
    float *s_rn = reinterpret_cast<float *>(tail + so.rn);
    uint32_t *s_tk = reinterpret_cast<uint32_t *>(tail + so.tk);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WsHeader *hdr = reinterpret_cast<WsHeader *>(rp.ws + L.hdr);
    const int G = gridDim.x, cta = blockIdx.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&sfr[s], 4);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&afull[b], 1);
            mbar_init(&aempty[b], 4);
        }
        mbar_init(mready, 1);
        mbar_init(mdone, 1);
        mbar_init(rnready, 1);
        mbar_init(rdready, 1);
        mbar_init(tkready, kLTopkWarps);
        mbar_init(tkpart, 4);
        fence_mbar_init();
        *s_abort = 0;
        *s_U = 0;
        *s_rdone = 0;
        for (int q = 0; q < 8; ++q) s_r0c[q] = 0;
    }
    constexpr uint32_t kCols = 512u;
    if (warp == 0) umma::tmem_alloc(tslot, kCols);
    umma::fence_before();
    __syncthreads();
    umma::fence_after();
    const uint32_t tbase = *tslot;
    // Zero a buffer's accumulator chains (this warp's lane quadrant): at the
    // start, and by the epilogue after reading them, so every MMA accumulates.
    auto zero_acc = [&](int buf) {
        const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int q = 0; q < 2; ++q)
                if (q < Q)
#pragma unroll
                    for (int n0 = 0; n0 < kNMax; n0 += 8)
                        if (n0 < N) umma::st8(tbase + umma::lane_base(warp) + (uint32_t)(buf * 128 + m * 64 + q * W + n0), z);
        umma::wait_st();
    };
    if (warp < 4) {
        zero_acc(0);
        zero_acc(1);
    }
    umma::fence_before();
    __syncthreads();
    umma::fence_after();
    // TMEM columns: accumulators [buf][mat] at (2*buf + mat) * 64 (N <= 48),
    // then kLSfc scale columns per stage: A box 0 (+0), A box 1 (+8), B tile
    // 0 (+16), B tile 1 (+24).
    const uint32_t sf0 = 256u;

    // ------------------------------------------------------------ shapes --
    const int ffs = p.ffs, ff = p.ff;
    const int rpu = lk_rows_per_unit(d);                        // router rows per unit
    const int n0 = (E + rpu - 1) / rpu;                         // router units
    const int nkts_d = ceil_div(d, kTileKs);                    // shared gate/up K-tiles (64)
    const int nrbs = ffs > 0 ? ceil_div(ffs, kTileM) : 0;       // shared gate/up items
    const int nkt_d = ceil_div(d, kTileK);                      // routed gate/up K-tiles (256)
    const int nrb_ff = ceil_div(ff, kTileM);                    // routed gate/up items per expert
    const int nkt_ff = ceil_div(ff, kTileK);                    // routed down K-tiles per expert
    const int ndu = (nkt_ff + 1) / 2;                           // ... in units of two
    const int nkts_ffs = ffs > 0 ? ceil_div(ffs, kTileKs) : 0;  // shared down K-tiles (64)
    const int nsdu = (nkts_ffs + 1) / 2;
    const int nrb_d = ceil_div(d, kTileM);                      // down items
    int U = 0;                                                  // distinct routed experts (after mready)

    // A range of n units split evenly over the CTAs (CTA c of G' = min(G, n)
    // takes [c n / G', (c+1) n / G')); an item cut between CTAs is finished
    // by the last of them to arrive.
    struct Range {
        int n, G, a, b;
    };
    auto make_range = [&](int n) {
        Range r;
        r.n = n;
        r.G = min(G, max(n, 1));
        r.a = cta < r.G && n > 0 ? (int)(((long long)cta * n) / r.G) : 0;
        r.b = cta < r.G && n > 0 ? (int)(((long long)(cta + 1) * n) / r.G) : 0;
        return r;
    };
    auto start_of = [&](const Range &r, int c) { return (int)(((long long)c * r.n) / r.G); };
    auto owner = [&](const Range &r, int unit) { return (int)((((long long)unit + 1) * r.G - 1) / r.n); };
    // (scalars, not an array: an array indexed by a loop counter would live
    // in local memory)
    Range rg0 = make_range(p.mode == kLayerRouted ? 0 : n0);
    Range rg1 = make_range(p.mode == kLayerRouteOnly ? 0 : nrbs * nkts_d);
    Range rg2 = make_range(0);
    Range rg3 = make_range(0);
    auto rgr = [&](int r) { return r == 0 ? rg0 : (r == 1 ? rg1 : (r == 2 ? rg2 : rg3)); };
    // units per item of the ranges with items (R1, R2, R3)
    auto upi = [&](int r) { return r == 1 ? nkts_d : (r == 2 ? nkt_d : U * ndu + nsdu); };
    // Bounded wait that gives up at once after any role has given up.
    auto wait = [&](uint64_t *bar, uint32_t parity) {
        if (*s_abort) return false;
        if (mbar_wait_bounded(bar, parity, hdr, rp.wait_ns)) return true;
        *s_abort = 1;
        return false;
    };
    // Before R2: the routing (one lane waits, its warp follows when warp_wide).
    auto routed_ranges = [&](bool warp_wide) {
        if (p.mode == kLayerRouteOnly) return false;  // nothing after the routing
        int ok = 1;
        if (lane == 0) {
            ok = (!*s_abort && mbar_wait_bounded(mready, 0u, hdr, rp.wait_ns)) ? 1 : 0;
            if (!ok) *s_abort = 1;
        }
        if (warp_wide) ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) return false;
        U = *s_U;
        rg2 = make_range(U * nrb_ff * nkt_d);
        rg3 = make_range(nrb_d * (U * ndu + nsdu));
        return true;
    };
    // Unit u of range r (r >= 1): item, its unit span, expert, row block,
    // first K-tile and K-tiles in the unit; kind 1 shared gate/up, 2 routed
    // gate/up, 3 routed down, 4 shared down.
    struct Unit {
        int kind, item, istart, iend, u, rb, kt, nt;
    };
    auto decode = [&](int r, int unit) {
        Unit x;
        const int per = upi(r);
        x.item = unit / per;
        x.istart = x.item * per;
        x.iend = x.istart + per;
        const int j = unit - x.istart;
        if (r == 1) {
            x.kind = 1; x.u = -1; x.rb = x.item; x.kt = j; x.nt = 1;
        } else if (r == 2) {
            x.kind = 2; x.u = x.item / nrb_ff; x.rb = x.item - x.u * nrb_ff; x.kt = j; x.nt = 1;
        } else {
            x.rb = x.item;
            if (j < U * ndu) {
                x.kind = 3; x.u = j / ndu; x.kt = 2 * (j - x.u * ndu); x.nt = min(2, nkt_ff - x.kt);
            } else {
                x.kind = 4; x.u = -1; x.kt = 2 * (j - U * ndu); x.nt = min(2, nkts_ffs - x.kt);
            }
        }
        return x;
    };
    const size_t mat = (size_t)d * ff;
    const uint8_t *smaps = rp.ws + L.tmap + (size_t)E * kMapsPerExpert * 128;

    if (warp == 10) {
        // ================================================= set-up, routing --
        // the tokens' 1 / rms (pre-norm calls) and the blob pointer of every
        // expert -> shared memory (the dispatch reads them)
        if (p.norm_w) {
            // 1 / rms of every token (the same bits in every CTA)
            for (int t = 0; t < Tc; ++t) {
                const float r = warp_rms_inv(rp.x + (size_t)t * d, d, p.eps);
                if (lane == 0) s_rn[t] = r;
            }
            __syncwarp();
            if (lane == 0)
                asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(rnready)) : "memory");
        }
        if (p.mode != kLayerRouteOnly)
            for (int e = lane; e < E; e += 32) s_ptab[e] = rp.blobs[e];
    } else if ((warp == 1 || warp == 2) && p.mode != kLayerRouteOnly) {
        // set-up shared with two of the top-k warps (idle until the router
        // rows are in): warp 1 this CTA's share of the tensor maps, warp 2
        // its share of the activation pieces; each counts on prep_done
        // (2 per CTA), which the copies warps wait for before their first
        // B tile or tensor map
        if (warp == 1) {
            refresh_tmaps(rp, cta * 32 + lane, G * 32);
        } else {
            int ok = 1;
            if (p.norm_w) {
                if (lane == 0) ok = mbar_wait_bounded(rnready, 0u, hdr, rp.wait_ns) ? 1 : 0;
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (ok) (void)mbar_try_wait(rnready, 0u);
            }
            if (ok) build_x_pieces(rp.x, Tc, d, rp.ws, L, cta, G, rp.has_shared != 0, p.norm_w, s_rn);
        }
        __syncwarp();
        if (lane == 0) red_add_release(&hdr->prep_done, 1u);
    }

    if ((warp < 4 || warp == 10) && !(p.mode == kLayerRouteOnly && cta != 0)) {
        // top-k of the tokens, warps 0-3 and 10 (160 threads) once every
        // router row is in (or the routing a route-only launch left)
        const int tw = warp == 10 ? 4 : warp;
        int ok = 1;
        if (p.mode == kLayerRouted) {
            const int32_t *gi = reinterpret_cast<const int32_t *>(rp.ws + L.idx);
            const float *gw = reinterpret_cast<const float *>(rp.ws + L.wt);
            for (int t = tw; t < Tc; t += kLTopkWarps)
                if (lane < k) {
                    s_tidx[t * 32 + lane] = __ldcg(gi + t * k + lane);
                    s_tw[t * 32 + lane] = __ldcg(gw + t * k + lane);
                }
        } else {
            // one poller per CTA (the counter's line is shared by the whole
            // grid); the other top-k warps wait on rdready
            if (lane == 0) {
                if (warp == 0) {
                    if (!spin_geq(&hdr->router_done, (uint32_t)E, rp.wait_ns, s_abort)) {
                        set_status(hdr, kStTimeout);
                        *s_abort = 1;
                        ok = 0;
                    }
                    *s_rok = ok;
                    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(rdready)) : "memory");
                } else {
                    ok = mbar_wait_bounded(rdready, 0u, hdr, rp.wait_ns) && *s_rok ? 1 : 0;
                    if (!ok) *s_abort = 1;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            // every lane acquires the poller's release (which follows its
            // acquire of the other CTAs' logits)
            if (ok) (void)mbar_try_wait(rdready, 0u);
        }
        if (ok && p.mode != kLayerRouted) {
            const float *logits = reinterpret_cast<const float *>(rp.ws + L.logits);
            const float *sb = (rp.route_flags & kRouteBiasSelect) ? rp.bias : nullptr;
            const bool rn = (rp.route_flags & kRouteRenorm) != 0;
            if (Tc == 1) {
                // one token: a quarter of the row per warp 0-3, merged by warp 0
                if (warp < 4) {
                    const int per = (E + 3) / 4;
                    const int e0 = warp * per, e1 = min(E, e0 + per);
                    warp_topk_part(logits, e0, e1, k, sb, s_tk + warp * kTkWords);
                    __syncwarp();
                    if (lane == 0)
                        asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(tkpart)) : "memory");
                    if (warp == 0) {
                        int all = 1;
                        if (lane == 0) all = mbar_wait_bounded(tkpart, 0u, hdr, rp.wait_ns) ? 1 : 0;
                        all = __shfl_sync(0xffffffffu, all, 0);
                        if (all) {
                            (void)mbar_try_wait(tkpart, 0u);
                            if (!warp_topk_merge(logits, k, s_tidx, s_tw, sb, rn, s_tk))
                                warp_topk(logits, E, k, s_tidx, s_tw, sb, rn, s_tk + 4 * kTkWords);
                        } else {
                            *s_abort = 1;
                        }
                    }
                }
            } else {
                for (int t = tw; t < Tc; t += kLTopkWarps)
                    warp_topk(logits + (size_t)t * E, E, k, s_tidx + t * 32, s_tw + t * 32, sb, rn, s_tk + tw * kTkWords);
            }
        }
        // the picks are in shared memory: each top-k warp counts on tkready,
        // the dispatching warp waits for all of them
        __syncwarp();
        if (lane == 0)
            asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(tkready)) : "memory");
        if (warp == 10) {
            int all = 1;
            if (lane == 0) all = mbar_wait_bounded(tkready, 0u, hdr, rp.wait_ns) ? 1 : 0;
            all = __shfl_sync(0xffffffffu, all, 0);
            if (all) (void)mbar_try_wait(tkready, 0u);
            else { ok = 0; *s_abort = 1; }
        }
        if (warp == 10 && ok && !*s_abort && p.mode == kLayerRouteOnly) {
            // route only: the picks into the workspace (and the caller's copies)
            for (int i = lane; i < Tc * k; i += 32) {
                const int t = i / k, j = i - t * k;
                reinterpret_cast<int32_t *>(rp.ws + L.idx)[i] = s_tidx[t * 32 + j];
                reinterpret_cast<float *>(rp.ws + L.wt)[i] = s_tw[t * 32 + j];
                if (rp.idx_out) rp.idx_out[i] = s_tidx[t * 32 + j];
                if (rp.w_out) rp.w_out[i] = s_tw[t * 32 + j];
            }
        } else if (warp == 10 && ok && !*s_abort) {
            // dispatch: distinct experts in ascending id (bitmap + prefix),
            // each one's blob (checked) and per-token weight
            uint32_t *bitmap = s_misc, *prefix = s_misc + 32;
            const int nwords = (E + 31) >> 5;
            bitmap[lane] = 0u;
            __syncwarp();
            for (int i = lane; i < Tc * k; i += 32) {
                const int e = s_tidx[(i / k) * 32 + i % k];
                atomicOr(&bitmap[e >> 5], 1u << (e & 31));
            }
            __syncwarp();
            const uint32_t c = lane < nwords ? __popc(bitmap[lane]) : 0u;
            uint32_t incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            prefix[lane] = incl - c;
            const int Ut = (int)__shfl_sync(0xffffffffu, incl, 31);
            __syncwarp();
            for (int i = lane; i < Ut * Tc; i += 32) s_wu[i] = 0.f;
            if (lane < nwords) {
                // lane l: the set bits of word l, in ascending expert id
                uint32_t bits = bitmap[lane], u = prefix[lane];
                while (bits != 0u) {
                    const int w = 32 * lane + __ffs(bits) - 1;
                    bits &= bits - 1u;
                    const uint8_t *b = s_ptab[w];
                    if (b == nullptr || (reinterpret_cast<uintptr_t>(b) & 15u) != 0u) {
                        set_status(hdr, kStDeviceCheck);
                        b = nullptr;
                    }
                    s_blob[u] = b;
                    s_eid[u] = w;
                    ++u;
                }
            }
            __syncwarp();
            for (int i = lane; i < Tc * k; i += 32) {
                const int t = i / k, j = i - t * k;
                const int e = s_tidx[t * 32 + j];
                const uint32_t u = prefix[e >> 5] + __popc(bitmap[e >> 5] & ((1u << (e & 31)) - 1u));
                s_wu[u * Tc + t] = s_tw[t * 32 + j];
                if (cta == 0) {
                    if (rp.idx_out) rp.idx_out[(size_t)t * k + j] = e;
                    if (rp.w_out) rp.w_out[(size_t)t * k + j] = s_tw[t * 32 + j];
                }
            }
            if (lane == 0) {
                *s_U = Ut;
                if (cta == 0) hdr->n_unique = (uint32_t)Ut;
            }
            __syncwarp();
            if (lane == 0 && p.inject != 1)
                asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(mready)) : "memory");
        }
    }

    if (warp == 8) {
        // ========================================================= copies --
        if (lane == 0) {
            int i = 0;  // this CTA's unit counter over all ranges (stage i % nst)
            bool prep_ok = false, gu_ok = false;
            uint32_t gu_total = 0u;
            // B tiles of down units whose weights are issued but whose
            // activations were not ready yet (at most nst, in stage order)
            int pend_s[8], pend_unit[8];
            int npend = 0;
            const uint8_t *acq_maps = nullptr, *acq_sc = nullptr;  // last tensor maps acquired
            auto issue_b = [&](int s, const Unit &x) {
                uint8_t *st = smem + s * SB;
                // the B scale words travel with the stage when the A scales do
                const bool sfb = x.kind == 3 && sf_dn && s_blob[x.u] != nullptr;
                for (int tt = 0; tt < x.nt; ++tt) {
                    const size_t bt = x.kind == 3 ? (size_t)x.u * nkt_ff + x.kt + tt : (size_t)(x.kt + tt);
                    const uint8_t *bsrc = x.kind == 3 ? rp.ws + L.hb + bt * N * 128 : rp.ws + L.hsb + bt * N * 128;
                    bulk_g2s(st + lk_b_off() + tt * N * 128, bsrc, (uint32_t)(N * 128), &full[s]);
                    if (sfb)
                        bulk_g2s(st + lk_sfb_off(N) + tt * 2 * kSfRow * 4, rp.ws + L.hsf + bt * 2 * kSfRow * 4,
                                 (uint32_t)(2 * kSfRow * 4), &full[s]);
                }
            };
            auto gu_ready = [&](bool block) {
                if (gu_ok) return true;
                if (!block) {
                    if (ld_relaxed(&hdr->gu_done) < gu_total) return false;
                    asm volatile("fence.acq_rel.gpu;" ::: "memory");
                } else if (!spin_geq(&hdr->gu_done, gu_total, rp.wait_ns, s_abort)) {
                    set_status(hdr, kStTimeout);
                    *s_abort = 1;
                    return false;
                }
                asm volatile("fence.proxy.async.global;" ::: "memory");  // before bulk copies read h
                gu_ok = true;
                return true;
            };
            for (int r = 0; r < 4 && !*s_abort; ++r) {
                if (r == 2) {
                    if (!routed_ranges(false)) break;
                    gu_total = (uint32_t)(nrbs + U * nrb_ff);
                }
                const Range R = rgr(r);
                for (int unit = R.a; unit < R.b && !*s_abort; ++unit, ++i) {
                    const int s = i % nst;
                    const uint32_t ph = (uint32_t)((i / nst) & 1);
                    if (r == 3 && npend == nst) {
                        // every stage waits for activations: wait for them
                        if (!gu_ready(true)) break;
                        for (int q = 0; q < npend; ++q) issue_b(pend_s[q], decode(3, pend_unit[q]));
                        npend = 0;
                    }
                    if (r == 3 && npend > 0 && gu_ready(false)) {
                        for (int q = 0; q < npend; ++q) issue_b(pend_s[q], decode(3, pend_unit[q]));
                        npend = 0;
                    }
                    if (i >= nst && !wait(&empty[s], ph ^ 1u)) break;
                    uint8_t *st = smem + s * SB;
                    if (r == 0) {
                        const int ur0 = unit * rpu;
                        const uint32_t bytes = (uint32_t)(min(rpu, E - ur0) * d * 4);
                        mbar_arrive_expect_tx(&full[s], bytes);
                        bulk_g2s(st, rp.wr + (size_t)ur0 * d, bytes, &full[s]);
                        continue;
                    }
                    if (!prep_ok) {
                        // x pieces, x as bf16 and the tensor maps are published
                        // by every CTA's set-up warp
                        if (!spin_geq(&hdr->prep_done, (uint32_t)(2 * G), rp.wait_ns, s_abort)) {
                            set_status(hdr, kStTimeout);
                            *s_abort = 1;
                            break;
                        }
                        asm volatile("fence.proxy.async.global;" ::: "memory");
                        prep_ok = true;
                    }
                    const Unit x = decode(r, unit);
                    const uint8_t *maps, *scmaps = nullptr;
                    bool blob_ok = true;
                    if (x.kind == 1 || x.kind == 4) {
                        maps = smaps + (x.kind == 1 ? 0 : 256);
                    } else {
                        const uint8_t *em = rp.ws + L.tmap + (size_t)s_eid[x.u] * kMapsPerExpert * 128;
                        maps = em + (x.kind == 2 ? 0 : 256);
                        scmaps = em + (x.kind == 2 ? 384 : 640);
                        blob_ok = s_blob[x.u] != nullptr;
                    }
                    const bool sf_dma = blob_ok && ((x.kind == 2 && sf_gu) || (x.kind == 3 && sf_dn));
                    // bytes: A boxes, B tiles, A scale box(es), B scale words
                    uint32_t tx = 0u;
                    const int nbox = (x.kind == 1 || x.kind == 2) ? 2 : x.nt;
                    const int nb = (x.kind == 1 || x.kind == 2) ? 1 : x.nt;
                    if (blob_ok) tx += (uint32_t)(nbox * kAtile);
                    tx += (uint32_t)(nb * N * 128);
                    if (sf_dma) tx += (uint32_t)((x.kind == 2 ? 2 : 1) * 2048 + nb * 2 * kSfRow * 4);
                    mbar_arrive_expect_tx(&full[s], tx);
                    if (blob_ok) {
                        // the maps were written through the generic proxy (this
                        // launch or an earlier one): one acquire per map and CTA
                        if (maps != acq_maps) {
                            umma::tmap_acquire(maps);
                            if (x.kind <= 2) umma::tmap_acquire(maps + 128);
                            acq_maps = maps;
                        }
                        if (x.kind <= 2) {
                            // gate/up: W_g box and W_u box of K-tile kt (128 bytes of every row)
                            umma::tma_load_2d(st, maps, x.kt * 128, x.rb * kTileM, &full[s]);
                            umma::tma_load_2d(st + kAtile, maps + 128, x.kt * 128, x.rb * kTileM, &full[s]);
                        } else {
                            for (int tt = 0; tt < x.nt; ++tt)
                                umma::tma_load_2d(st + tt * kAtile, maps, (x.kt + tt) * 128, x.rb * kTileM, &full[s]);
                        }
                        if (sf_dma) {
                            uint8_t *sfa = st + lk_sfa_off(N);
                            if (scmaps != acq_sc) {
                                umma::tmap_acquire(scmaps);
                                if (x.kind == 2) umma::tmap_acquire(scmaps + 128);
                                acq_sc = scmaps;
                            }
                            umma::tma_load_2d(sfa, scmaps, (x.kt >> 1) * 16, x.rb * kTileM, &full[s]);
                            if (x.kind == 2) {
                                umma::tma_load_2d(sfa + 2048, scmaps + 128, (x.kt >> 1) * 16, x.rb * kTileM, &full[s]);
                            }
                        }
                    }
                    if (x.kind == 1) {
                        bulk_g2s(st + lk_b_off(), rp.ws + L.xbf + (size_t)x.kt * N * 128, (uint32_t)(N * 128), &full[s]);
                    } else if (x.kind == 2) {
                        bulk_g2s(st + lk_b_off(), rp.ws + L.xb + (size_t)x.kt * N * 128, (uint32_t)(N * 128), &full[s]);
                        if (sf_dma)
                            bulk_g2s(st + lk_sfb_off(N), rp.ws + L.xsf + (size_t)x.kt * 2 * kSfRow * 4,
                                     (uint32_t)(2 * kSfRow * 4), &full[s]);
                    } else if (gu_ready(false)) {
                        issue_b(s, x);
                    } else {
                        pend_s[npend] = s;
                        pend_unit[npend] = unit;
                        ++npend;
                    }
                }
            }
            if (npend > 0 && !*s_abort && gu_ready(true)) {
                for (int q = 0; q < npend; ++q) issue_b(pend_s[q], decode(3, pend_unit[q]));
                npend = 0;
            }
            if (*s_abort) {
                // a wait gave up somewhere: wait (bounded) for the last copy
                // issued into each stage, so none lands after the CTA's
                // shared memory is released
                for (int q = 0; q < nst && q < i; ++q) {
                    const int last = q + ((i - 1 - q) / nst) * nst;
                    mbar_drain(&full[q], (uint32_t)((last / nst) & 1), rp.wait_ns);
                }
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ============================ router sums (R0), scales -> TMEM =====
        const int tid = threadIdx.x - 128;  // 0..127
        const int wl = warp - 4;
        const uint32_t lb = umma::lane_base(warp);
        uint32_t nanb = 0u;
        // this CTA's router rows: row_base .. row_base + nrows - 1 (whole
        // rows: a unit is rpu rows)
        const Range R0 = rg0;
        const int row_base = R0.a * rpu;
        const int nrows = R0.a < R0.b ? min(E, R0.b * rpu) - row_base : 0;
        for (int q = tid; q < 4 * kRMaxRows * Tc; q += 128) s_racc[q] = 0.f;
        bool go = true;
        if (p.norm_w) {
            // the router reads x = RMSNorm(h): wait for the tokens' 1 / rms
            int ok = 1;
            if (lane == 0) ok = mbar_wait_bounded(rnready, 0u, hdr, rp.wait_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (ok) (void)mbar_try_wait(rnready, 0u);
            go = umma::bar_red_and(2, 128, ok != 0);
            if (!go) *s_abort = 1;
        } else {
            umma::bar_sync(2, 128);
        }
        // this thread's 64 floats of a unit: row rin_t of the unit, columns
        // col_t .. col_t + 63 (the same in every unit)
        const int f_t = 64 * tid;
        const int rin_t = f_t / d, col_t = f_t - rin_t * d;
        // Token t's 64 columns of x: eight 16-byte loads issued together,
        // chunk (q + lane) mod 8 into register q, so the weight reads (the
        // same rotated order) spread over the shared-memory banks and every
        // register index stays static.  x = RMSNorm(h) on pre-norm calls.
        auto load_x = [&](int t, uint4 (&xr)[8]) {
            const uint4 *xv = reinterpret_cast<const uint4 *>(rp.x + (size_t)t * d + col_t);
#pragma unroll
            for (int q = 0; q < 8; ++q) xr[q] = __ldg(xv + ((q + lane) & 7));
            if (p.norm_w) {
                const uint4 *gv = reinterpret_cast<const uint4 *>(p.norm_w + col_t);
                const float rt = s_rn[t];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint4 g = __ldg(gv + ((q + lane) & 7));
                    uint32_t *xw = reinterpret_cast<uint32_t *>(&xr[q]);
                    const uint32_t *gw = reinterpret_cast<const uint32_t *>(&g);
#pragma unroll
                    for (int h = 0; h < 4; ++h)
                        xw[h] = (uint32_t)rms_norm_bf16((uint16_t)(xw[h] & 0xFFFFu), rt, (uint16_t)(gw[h] & 0xFFFFu)) |
                                ((uint32_t)rms_norm_bf16((uint16_t)(xw[h] >> 16), rt, (uint16_t)(gw[h] >> 16)) << 16);
                }
            }
        };
        // 64 products (each exact), summed in fp32 in this order
        auto dot_w = [&](const float4 *w4, const uint4 (&xr)[8]) {
            float acc = 0.f;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int jq = (q + lane) & 7;
                const float4 a = w4[2 * jq], b = w4[2 * jq + 1];
                acc = fmaf(a.x, bf16_lo(xr[q].x), acc);
                acc = fmaf(a.y, bf16_hi(xr[q].x), acc);
                acc = fmaf(a.z, bf16_lo(xr[q].y), acc);
                acc = fmaf(a.w, bf16_hi(xr[q].y), acc);
                acc = fmaf(b.x, bf16_lo(xr[q].z), acc);
                acc = fmaf(b.y, bf16_hi(xr[q].z), acc);
                acc = fmaf(b.z, bf16_lo(xr[q].w), acc);
                acc = fmaf(b.w, bf16_hi(xr[q].w), acc);
            }
            return acc;
        };
        int i = 0;
        bool act_ok[2] = {false, false};  // x pieces' scales / h pieces' scales seen (no-TMA path)
        // ---- R0: the router rows of this CTA.  One token (ONE): its columns
        // of x stay in registers for the whole slice; more tokens: loaded per
        // unit, the next token's loads in flight during this one's products.
        auto router_units = [&](auto one) {
            constexpr bool ONE = decltype(one)::value;
            uint4 x0[8];
            if (ONE && f_t < rpu * d) load_x(0, x0);
            const Range R = rg0;
            for (int unit = R.a; unit < R.b; ++unit, ++i) {
                const int s = i % nst;
                const uint32_t ph = (uint32_t)((i / nst) & 1);
                int ok = 0;
                if (lane == 0) ok = wait(&full[s], ph) ? 1 : 0;
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) {
                    go = false;
                    break;
                }
                (void)mbar_try_wait(&full[s], ph);  // every lane sees the landed bytes
                const uint8_t *st = smem + s * SB;
                // Each warp on its own: 64 consecutive floats of the unit
                // per thread (inside one row: d is a multiple of 64), the
                // same columns of x in every unit; the warp's sums per row
                // (segmented over lanes, fixed order) go into its own row
                // accumulators, unit after unit; the last of the four warps
                // to finish a unit releases its stage.
                const int ur0 = unit * rpu;  // first row of the unit
                const int ufl = min(rpu, E - ur0) * d;
                int row = -1;
                float v[kChunk];
#pragma unroll
                for (int t = 0; t < kChunk; ++t) v[t] = 0.f;
                if (f_t < ufl) {
                    row = ur0 + rin_t - row_base;
                    const float4 *w4 = reinterpret_cast<const float4 *>(st) + tid * 16;
                    if constexpr (ONE) {
                        v[0] = dot_w(w4, x0);
                    } else {
                        uint4 xa[8], xb[8];
                        load_x(0, xa);
#pragma unroll
                        for (int t = 0; t < kChunk; ++t) {
                            if (t < Tc) {
                                if (t + 1 < Tc) load_x(t + 1, (t & 1) ? xa : xb);
                                v[t] = dot_w(w4, (t & 1) ? xb : xa);
                            }
                        }
                    }
                }
                // segmented sum over lanes of equal row (rows do not decrease along lanes)
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int rn = __shfl_down_sync(0xffffffffu, row, o);
#pragma unroll
                    for (int t = 0; t < kChunk; ++t) {
                        if (t < Tc) {
                            const float vn = __shfl_down_sync(0xffffffffu, v[t], o);
                            if (lane + o < 32 && rn == row) v[t] += vn;
                        }
                    }
                }
                const int rprev = __shfl_up_sync(0xffffffffu, row, 1);
                if (row >= 0 && (lane == 0 || rprev != row)) {
                    float *acc = s_racc + ((size_t)wl * kRMaxRows + row) * Tc;
#pragma unroll
                    for (int t = 0; t < kChunk; ++t)
                        if (t < Tc) acc[t] += v[t];
                }
                __syncwarp();
                if (lane == 0 && atomicAdd(&s_r0c[s], 1) == 3) {
                    s_r0c[s] = 0;
                    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&empty[s])) : "memory");
                }
            }
        };
        if (go) {
            if (Tc == 1)
                router_units(std::integral_constant<bool, true>{});
            else
                router_units(std::integral_constant<bool, false>{});
            // the slice's rows: the four warps' sums in warp order, one
            // release per CTA on router_done (the barrier orders every
            // thread's logit stores before thread 0's release)
            go = umma::bar_red_and(2, 128, go);
            if (go && tid < nrows) {
                const int rr = row_base + tid;
                float *logits = reinterpret_cast<float *>(rp.ws + L.logits);
                const float bias = (rp.bias && !(rp.route_flags & kRouteBiasSelect)) ? rp.bias[rr] : 0.f;
                for (int t = 0; t < Tc; ++t) {
                    float o = s_racc[(size_t)tid * Tc + t];
#pragma unroll
                    for (int w2 = 1; w2 < 4; ++w2) o += s_racc[((size_t)w2 * kRMaxRows + tid) * Tc + t];
                    logits[(size_t)t * E + rr] = o + bias;
                }
            }
            umma::bar_sync(2, 128);
            if (tid == 0 && go && nrows > 0) red_add_release(&hdr->router_done, (uint32_t)nrows);
        }
        // ---- R1 .. R3: the scale factors of the matrix units
        for (int r = 1; r < 4 && go; ++r) {
            if (r == 2 && !routed_ranges(true)) break;
            const Range R = rgr(r);
            for (int unit = R.a; unit < R.b; ++unit, ++i) {
                const int s = i % nst;
                const uint32_t ph = (uint32_t)((i / nst) & 1);
                int ok = 0;
                if (lane == 0) ok = wait(&full[s], ph) ? 1 : 0;
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) {
                    go = false;
                    break;
                }
                (void)mbar_try_wait(&full[s], ph);  // every lane sees the landed bytes
                const uint8_t *st = smem + s * SB;
                {
                    const Unit x = decode(r, unit);
                    if (x.kind == 2 || x.kind == 3) {
                        const uint8_t *blob = s_blob[x.u];
                        const bool has = blob != nullptr;
                        const bool tma_sc = x.kind == 2 ? sf_gu : sf_dn;
                        const uint32_t col = tbase + lb + sf0 + (uint32_t)(s * kLSfc);
                        const int K = x.kind == 2 ? d : ff, M = x.kind == 2 ? ff : d;
                        const int nbox = x.kind == 2 ? 2 : x.nt;
                        // A scales: box m holds matrix m (gate/up) or K-tile kt + m (down)
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            if (m < nbox) {
                                const int ktm = x.kind == 2 ? x.kt : x.kt + m;
                                uint32_t w[8];
                                if (tma_sc) {
                                    const uint8_t *sfa = st + lk_sfa_off(N) + (x.kind == 2 ? m * 2048 : 0) + (ktm & 1) * 8;
#pragma unroll
                                    for (int j = 0; j < 4; ++j) {
                                        const uint2 v = has ? *reinterpret_cast<const uint2 *>(sfa + (32 * j + lane) * 16)
                                                            : make_uint2(0u, 0u);
                                        nanb |= e8m0_nan8(v.x, v.y);
                                        w[j] = v.x;
                                        w[4 + j] = v.y;
                                    }
                                } else {
                                    const uint8_t *plane = nullptr;
                                    if (has)
                                        plane = x.kind == 2 ? (m == 0 ? blob + mat / 2 : blob + mat + mat / 32)
                                                            : blob + mat + mat / 16 + mat / 2;
                                    const int nks = min(4, (K - ktm * kTileK) / 64);
#pragma unroll
                                    for (int j = 0; j < 4; ++j) {
                                        const int row = x.rb * kTileM + 32 * j + lane;
                                        uint2 v = make_uint2(0u, 0u);
                                        if (plane != nullptr && row < M) v = load_sf8(plane + (size_t)row * (K / 32) + ktm * 8, nks);
                                        nanb |= e8m0_nan8(v.x, v.y);
                                        w[j] = v.x;
                                        w[4 + j] = v.y;
                                    }
                                }
                                umma::st8(col + 8 * m, w);
                            }
                        }
                        // B scales: tile tt at column 16 + 8 tt (rows 0-31, 32-63 per group)
                        const int nbt = x.kind == 2 ? 1 : x.nt;
#pragma unroll
                        for (int tt = 0; tt < 2; ++tt) {
                            if (tt < nbt) {
                                uint32_t b0, b1, b2, b3;
                                if (tma_sc) {
                                    const uint32_t *sb = reinterpret_cast<const uint32_t *>(st + lk_sfb_off(N) + tt * 2 * kSfRow * 4);
                                    b0 = sb[lane]; b1 = sb[32 + lane]; b2 = sb[kSfRow + lane]; b3 = sb[kSfRow + 32 + lane];
                                } else {
                                    // written by other CTAs: acquire their counter once
                                    const int ai = x.kind == 2 ? 0 : 1;
                                    if (!act_ok[ai]) {
                                        const uint32_t *ctr = ai == 0 ? &hdr->prep_done : &hdr->gu_done;
                                        const uint32_t want = ai == 0 ? (uint32_t)(2 * G) : (uint32_t)(nrbs + U * nrb_ff);
                                        (void)spin_geq(ctr, want, rp.wait_ns);
                                        act_ok[ai] = true;
                                    }
                                    const uint32_t *sb = x.kind == 2
                                        ? reinterpret_cast<const uint32_t *>(rp.ws + L.xsf) + (size_t)x.kt * 2 * kSfRow
                                        : reinterpret_cast<const uint32_t *>(rp.ws + L.hsf) +
                                              ((size_t)x.u * nkt_ff + x.kt + tt) * 2 * kSfRow;
                                    b0 = __ldcg(sb + lane); b1 = __ldcg(sb + 32 + lane);
                                    b2 = __ldcg(sb + kSfRow + lane); b3 = __ldcg(sb + kSfRow + 32 + lane);
                                }
                                if (!has) b0 = b1 = b2 = b3 = 0u;
                                const uint32_t w[8] = {b0, b1, 0u, 0u, b2, b3, 0u, 0u};
                                umma::st8(col + 16 + 8 * tt, w);
                            }
                        }
                        umma::wait_st();
                    }
                    umma::fence_before();
                    // sfr counts the stage's matrix units only: the MMA warp
                    // never waits on a router unit, so a phase it does not
                    // track could let a parity wait pass early
                    __syncwarp();
                    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&sfr[s])) : "memory");
                }
            }
        }
        if (p.strict && __any_sync(0xffffffffu, nanb != 0u) && lane == 0) set_status(hdr, kStDeviceCheck);
    } else if (warp == 9) {
        // ====================================================== MMA issue --
        if (lane == 0) {
            const uint64_t adesc0 = umma::smem_desc(smem_u32(smem), 16u, 1024u, umma::kLayoutSw128);
            const uint64_t bdesc0 = umma::smem_desc(smem_u32(smem) + lk_b_off(), (uint32_t)((N / 8) * 128), 128u,
                                                    umma::kLayoutNone);
            const uint32_t bstep = (uint32_t)(2 * (N / 8) * 128) >> 4;  // one k-step of B (2 chunks)
            const uint32_t btile = (uint32_t)(N * 128) >> 4;            // B tile 1 after tile 0
            const uint32_t idesc4 = umma::idesc_mxf4(N), idesc16 = umma::idesc_bf16(N);
            const uint32_t id4[2] = {umma::idesc_sf_id(idesc4, 0u), umma::idesc_sf_id(idesc4, 2u)};
            int i = 0, seg = 0;
            // router units (the first n0 of the ring) are consumed by the
            // scale warps and do not complete sfr: stage s's matrix use
            // number is its use number minus its router uses
            const int n0 = rg0.b - rg0.a;
            for (int r = 0; r < 4 && !*s_abort; ++r) {
                if (r == 2 && !routed_ranges(false)) break;
                const Range R = rgr(r);
                if (r == 0) {
                    i += n0;
                    continue;
                }
                for (int unit = R.a; unit < R.b && !*s_abort; ++seg) {
                    Unit x = decode(r, unit);
                    const int seg_end = min(R.b, x.iend);
                    const int buf = seg & 1;
                    if (seg >= 2 && !wait(&aempty[buf], (uint32_t)(((seg >> 1) + 1) & 1))) break;
                    umma::fence_after();
                    const uint32_t dcol = tbase + (uint32_t)(buf * 128);
                    // the epilogue zeroes every accumulator after reading it (and
                    // all of them at the start), so each MMA accumulates
                    constexpr uint32_t acc = 1u;
                    for (int un = unit; un < seg_end; ++un, ++i) {
                        if (un != unit) x = decode(r, un);
                        const int s = i % nst;
                        const uint32_t ph = (uint32_t)((i / nst) & 1);
                        const int r0s = n0 > s ? (n0 - 1 - s) / nst + 1 : 0;
                        const uint32_t phs = (uint32_t)(((i / nst) - r0s) & 1);
                        // sfr first: the scale warps arrive on it only after
                        // this use's bytes landed, so full is then at most
                        // this use's phase ahead and its parity wait is exact
                        if (!wait(&sfr[s], phs) || !wait(&full[s], ph)) break;
                        umma::fence_after();
                        const uint32_t soff = (uint32_t)(s * SB) >> 4;
                        const uint64_t a0 = adesc0 + soff, b0 = bdesc0 + soff;
                        const uint32_t sfc = tbase + sf0 + (uint32_t)(s * kLSfc);
                        if (x.kind == 1) {
                            // shared gate/up: bf16, W_g -> matrix 0, W_u -> matrix 1,
                            // k-step sk into chain sk mod Q of its matrix
                            const int nks = min(4, (d - x.kt * kTileKs) / 16);
#pragma unroll
                            for (int sk = 0; sk < 4; ++sk) {
                                if (sk < nks) {
                                    const uint64_t bd = b0 + sk * bstep;
                                    const uint32_t cq = (uint32_t)((sk % Q) * W);
                                    umma::mma_bf16(dcol + cq, a0 + 2 * sk, bd, idesc16, acc);
                                    umma::mma_bf16(dcol + 64 + cq, a0 + (kAtile >> 4) + 2 * sk, bd, idesc16, acc);
                                }
                            }
                        } else if (x.kind == 2) {
                            const int nks = min(4, (d - x.kt * kTileK) / 64);
#pragma unroll
                            for (int sk = 0; sk < 4; ++sk) {
                                if (sk < nks) {
                                    const uint64_t bd = b0 + sk * bstep;
                                    const uint32_t cq = (uint32_t)((sk % Q) * W);
                                    const uint32_t sfid = (uint32_t)(2 * (sk & 1)) << 30;
                                    const uint32_t sfb = (sfc + 16 + (sk >> 1) * 4) | sfid;
                                    umma::mma_mxf4(dcol + cq, a0 + 2 * sk, bd, id4[sk & 1], acc, (sfc + (sk >> 1) * 4) | sfid, sfb);
                                    umma::mma_mxf4(dcol + 64 + cq, a0 + (kAtile >> 4) + 2 * sk, bd, id4[sk & 1], acc,
                                                   (sfc + 8 + (sk >> 1) * 4) | sfid, sfb);
                                }
                            }
                        } else {
                            // down: K-tiles kt, kt + 1 (A box tt, B tile tt); MMA j
                            // (= 4 tt + sk) into chain j mod 2Q (matrix slots of
                            // both halves: the epilogue sums them all)
                            for (int tt = 0; tt < x.nt; ++tt) {
                                const uint64_t at = a0 + (uint32_t)(tt * (kAtile >> 4));
                                const uint64_t bt = b0 + tt * btile;
                                if (x.kind == 3) {
                                    const int nks = min(4, (ff - (x.kt + tt) * kTileK) / 64);
#pragma unroll
                                    for (int sk = 0; sk < 4; ++sk) {
                                        if (sk < nks) {
                                            const int c = (4 * tt + sk) % (2 * Q);
                                            const uint32_t cc = (uint32_t)((c / Q) * 64 + (c % Q) * W);
                                            const uint32_t sfid = (uint32_t)(2 * (sk & 1)) << 30;
                                            umma::mma_mxf4(dcol + cc, at + 2 * sk, bt + sk * bstep, id4[sk & 1], acc,
                                                           (sfc + 8 * tt + (sk >> 1) * 4) | sfid,
                                                           (sfc + 16 + 8 * tt + (sk >> 1) * 4) | sfid);
                                        }
                                    }
                                } else {
                                    const int nks = min(4, (ffs - (x.kt + tt) * kTileKs) / 16);
#pragma unroll
                                    for (int sk = 0; sk < 4; ++sk) {
                                        if (sk < nks) {
                                            const int c = (4 * tt + sk) % (2 * Q);
                                            const uint32_t cc = (uint32_t)((c / Q) * 64 + (c % Q) * W);
                                            umma::mma_bf16(dcol + cc, at + 2 * sk, bt + sk * bstep, idesc16, acc);
                                        }
                                    }
                                }
                            }
                        }
                        umma::commit(&empty[s]);
                    }
                    umma::commit(&afull[buf]);
                    unit = seg_end;
                }
            }
            // the CTA frees its tensor memory only after every MMA issued here
            // has completed (on an early exit too)
            umma::commit(mdone);
            mbar_drain(mdone, 0u, rp.wait_ns);
        }
    }

    if (warp < 4) {
        // ======================================================= epilogue --
        const uint32_t lb = umma::lane_base(warp);
        const int rowl = 32 * warp + lane;  // row of the 128-row item
        float *spart = reinterpret_cast<float *>(rp.ws + L.spart);
        int seg = 0;
        for (int r = 1; r < 4; ++r) {
            // the four warps agree on going on (they share named barrier 1)
            if (r == 2 && !umma::bar_red_and(1, 128, routed_ranges(true))) break;
            const Range R = rgr(r);
            const int NM = r == 3 ? 1 : 2;
            uint32_t *icnt = reinterpret_cast<uint32_t *>(rp.ws + L.icnt) +
                             (r == 1 ? L.umax * nrb_ff : (r == 2 ? 0 : L.umax * nrb_ff + nrbs));
            for (int unit = R.a; unit < R.b; ++seg) {
                const Unit x = decode(r, unit);
                const int item = x.item;
                const int seg_end = min(R.b, x.iend);
                const int buf = seg & 1;
                float acc[2][kChunk];
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int t = 0; t < kChunk; ++t) acc[m][t] = 0.f;
                // every epilogue warp runs the same sequence of named barriers,
                // so after a failed wait it carries on (with unused values)
                if (lane == 0) wait(&afull[buf], (uint32_t)((seg >> 1) & 1));
                __syncwarp();
                umma::fence_after();
                // matrix m's chains (R3: both matrix slots hold chains of the one
                // output); then zero them for the MMAs of this buffer's next use
#pragma unroll
                for (int m = 0; m < 2; ++m) {
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        if (q < Q) {
#pragma unroll
                            for (int n0 = 0; n0 < kNMax; n0 += 8) {
                                if (n0 < N) {
                                    uint32_t v[8];
                                    umma::ld8(tbase + lb + (uint32_t)(buf * 128 + m * 64 + q * W + n0), v);
                                    umma::wait_ld();
#pragma unroll
                                    for (int jj = 0; jj < 8; ++jj) {
                                        const int t = (n0 + jj) / kPieces;
                                        if (t < kChunk) acc[m][t] += __uint_as_float(v[jj]);
                                    }
                                }
                            }
                        }
                    }
                }
                if (r == 3) {
#pragma unroll
                    for (int t = 0; t < kChunk; ++t) {
                        acc[0][t] += acc[1][t];
                        acc[1][t] = 0.f;
                    }
                }
                zero_acc(buf);
                umma::fence_before();
                __syncwarp();
                if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&aempty[buf])) : "memory");

                const bool whole = unit == x.istart && seg_end == x.iend;
                bool fin = whole;
                if (!whole) {
                    const int slot = 2 * (r - 1) + (unit == R.a ? 0 : 1);
                    float *sp = spart + (size_t)((cta * 6 + slot) * 2) * kChunk * kTileM;
#pragma unroll
                    for (int m = 0; m < 2; ++m)
#pragma unroll
                        for (int t = 0; t < kChunk; ++t)
                            if (m < NM && t < Tc) sp[(m * kChunk + t) * kTileM + rowl] = acc[m][t];
                    umma::bar_sync(1, 128);
                    const int c0 = owner(R, x.istart), c1 = owner(R, x.iend - 1);
                    if (threadIdx.x == 0) {
                        const uint32_t old = atom_add_acq_rel(icnt + item, 1u);
                        const int last = old == (uint32_t)(c1 - c0);
                        if (last) icnt[item] = 0u;
                        *s_last = last;
                    }
                    umma::bar_sync(1, 128);
                    fin = *s_last != 0;
                    if (fin) {
                        // sum every part of the item in K order
#pragma unroll
                        for (int m = 0; m < 2; ++m)
#pragma unroll
                            for (int t = 0; t < kChunk; ++t) acc[m][t] = 0.f;
                        for (int cc = c0; cc <= c1; ++cc) {
                            const int sl = 2 * (r - 1) + (start_of(R, cc) < x.istart ? 1 : 0);
                            const float *q = spart + (size_t)((cc * 6 + sl) * 2) * kChunk * kTileM;
#pragma unroll
                            for (int m = 0; m < 2; ++m)
#pragma unroll
                                for (int t = 0; t < kChunk; ++t)
                                    if (m < NM && t < Tc) acc[m][t] += __ldcg(q + (m * kChunk + t) * kTileM + rowl);
                        }
                    }
                }
                if (fin) {
                    if (r == 2) {
                        const int f = x.rb * kTileM + rowl;  // ff row of this thread
                        const uint8_t *blob = s_blob[x.u];
                        const int blk = x.rb * 4 + warp;  // 32-row block of ff
                        const int kt = blk >> 3;
                        uint8_t *tile = rp.ws + L.hb + ((size_t)x.u * nkt_ff + kt) * N * 128;
                        uint8_t *sfw = rp.ws + L.hsf + ((size_t)x.u * nkt_ff + kt) * 2 * kSfRow * 4;
#pragma unroll
                        for (int t = 0; t < kChunk; ++t) {
                            if (t < Tc) {
                                float h = 0.f;
                                const float w = s_wu[x.u * Tc + t];
                                if (blob != nullptr && w != 0.f && f < ff) h = silu_mul(acc[0][t], acc[1][t]) * w;
                                quantize_pieces(h, lane, t, blk & 7, N, tile, sfw);
                            }
                        }
                    } else if (r == 1) {
                        const int f = x.rb * kTileM + rowl;  // ff_s row of this thread
                        if (f < ffs) {
                            // h as bf16 hi + lo (pieces 0, 1; the others zero), weight 1
                            uint8_t *tile = rp.ws + L.hsb + (size_t)(f / kTileKs) * N * 128;
                            const int c = (f % kTileKs) / 8, e = f % 8;
#pragma unroll
                            for (int t = 0; t < kChunk; ++t) {
                                if (t < Tc) {
                                    const float h = silu_mul(acc[0][t], acc[1][t]);
                                    const __nv_bfloat16 hi = __float2bfloat16_rn(h);
                                    const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
#pragma unroll
                                    for (int pc = 0; pc < kPieces; ++pc) {
                                        const int n = t * kPieces + pc;
                                        const __nv_bfloat16 v = pc == 0 ? hi : (pc == 1 ? lo : __float2bfloat16_rn(0.f));
                                        *reinterpret_cast<__nv_bfloat16 *>(tile + (c * (N / 8) + n / 8) * 128 +
                                                                           (n % 8) * 16 + e * 2) = v;
                                    }
                                }
                            }
                        }
                    } else {
                        const int row = item * kTileM + rowl;
                        if (row < d) {
#pragma unroll
                            for (int t = 0; t < kChunk; ++t) {
                                if (t < Tc) {
                                    float yv = acc[0][t];
                                    if (p.resid) yv += __uint_as_float((uint32_t)p.resid[(size_t)t * d + row] << 16);
                                    if (p.out_fp32)
                                        reinterpret_cast<float *>(p.y)[(size_t)t * d + row] = yv;
                                    else
                                        reinterpret_cast<__nv_bfloat16 *>(p.y)[(size_t)t * d + row] = __float2bfloat16_rn(yv);
                                }
                            }
                        }
                    }
                    if (r != 3) {
                        // this gate/up item's activations are written: count it
                        // for the down units' copies
                        umma::bar_sync(1, 128);
                        if (threadIdx.x == 0) red_add_release(&hdr->gu_done, 1u);
                    }
                }
                unit = seg_end;
            }
        }
    }

    umma::fence_before();
    __syncthreads();
    if (warp == 0) {
        umma::fence_after();
        umma::tmem_dealloc(tbase, kCols);
    }
    if (threadIdx.x == 0) {
        // the last CTA out returns the header's counters to zero for the next call
        const uint32_t old = atom_add_acq_rel(&hdr->exit_cnt, 1u);
        if (old == (uint32_t)(G - 1)) {
            hdr->router_done = 0u;
            hdr->prep_done = 0u;
            hdr->gu_done = 0u;
            hdr->exit_cnt = 0u;
        }
    }
}

}  // namespace k3

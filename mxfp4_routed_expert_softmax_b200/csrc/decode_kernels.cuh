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
    int nstage;         // router ring stages (kRStage bytes each)
    uint4 tmpl[4][8];   // tensor-map templates: W_g/W_u, W_d nibble planes; their scale planes
    int scale_mask;     // which scale-plane templates exist (bit 0: W_g/W_u, bit 1: W_d)
    uint4 smap[3][8];   // shared expert tensor maps (W_g, W_u, W_d), when has_shared
    int has_shared;     // the tensor-core kernels run a shared expert
    const uint8_t *sw[3];  // the shared expert's W_g, W_u, W_d (the key of its cached maps)
    uint64_t wait_ns;   // bound of every device wait
    int route_flags;    // kRouteRenorm | kRouteBiasSelect
};

constexpr int kRouteThreads = 256;
// Routing variants: the k weights renormalised over the picks; the bias
// moving only the selection (the logits and the softmax stay unbiased).
constexpr int kRouteRenorm = 1;
constexpr int kRouteBiasSelect = 2;
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

// Block-wide inclusive scan of v over the 256 threads in thread order.
__device__ __forceinline__ uint32_t block_scan_incl(uint32_t v, uint32_t *s_tot) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) s_tot[warp] = v;
    __syncthreads();
    uint32_t add = 0;
    for (int w = 0; w < warp; ++w) add += s_tot[w];
    __syncthreads();
    return v + add;
}

// Softmax over all E logits and the top-k (descending logit, ties to the
// lower index) of token t, by one whole CTA (E <= 1024: 4 consecutive experts
// per thread).  Radix select on the order-preserving keys: four 8-bit digit
// passes (shared histogram, one warp's suffix scan) find the k-th largest key
// K exactly; every key above K is taken, and of the keys equal to K the
// lowest indices (a prefix count in index order).  The k winners are then
// ranked by (key descending, index ascending) for the output order.
// sel_bias (non-null): the selection runs on logit + sel_bias[e] while the
// softmax stays on the logits; renorm: the k weights are divided by their
// sum (in pick order).
__device__ void cta_topk_row(const float *row, int E, int k, int32_t *idx_row, float *w_row, int32_t *idx_out_row,
                             float *w_out_row, const float *sel_bias = nullptr, bool renorm = false) {
    __shared__ uint32_t s_hist[256];
    __shared__ uint32_t s_tot[8];
    __shared__ float s_red[2][8];
    __shared__ uint32_t s_pref, s_need, s_cnt;
    __shared__ uint32_t s_selk[32], s_seli[32];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float v[4];
    uint32_t key[4];
    bool ok[4];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = 4 * tid + i;
        ok[i] = e < E;
        v[i] = ok[i] ? __ldcg(row + e) : -INFINITY;
        key[i] = ok[i] ? fkey(sel_bias ? v[i] + __ldg(sel_bias + e) : v[i]) : 0u;  // real keys are > 0
        mx = fmaxf(mx, v[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_red[0][warp] = mx;
    if (tid == 0) s_cnt = 0u;
    __syncthreads();
    float m = s_red[0][0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, s_red[0][w]);
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (ok[i]) sum += expf(v[i] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) s_red[1][warp] = sum;
    // radix select of the k-th largest key
    uint32_t pref = 0u, pmask = 0u;
    uint32_t need = (uint32_t)k;
    for (int pass = 0; pass < 4; ++pass) {
        const int sh = 24 - 8 * pass;
        s_hist[tid] = 0u;
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (ok[i] && (key[i] & pmask) == pref) atomicAdd(&s_hist[(key[i] >> sh) & 255u], 1u);
        __syncthreads();
        if (warp == 0) {
            // lane l holds digits 255-8l down to 248-8l (descending)
            uint32_t c[8], lsum = 0u;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                c[jj] = s_hist[255 - 8 * lane - jj];
                lsum += c[jj];
            }
            uint32_t incl = lsum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            const uint32_t excl = incl - lsum;
            if (excl < need && need <= incl) {
                uint32_t acc = excl;
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    if (acc < need && acc + c[jj] >= need) {
                        s_pref = pref | ((uint32_t)(255 - 8 * lane - jj) << sh);
                        s_need = need - acc;
                    }
                    acc += c[jj];
                }
            }
        }
        __syncthreads();
        pref = s_pref;
        need = s_need;
        pmask |= 0xFFu << sh;
    }
    // pref = the k-th largest key; take every key above it and the `need`
    // lowest-index keys equal to it
    uint32_t ties = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) ties += (ok[i] && key[i] == pref) ? 1u : 0u;
    uint32_t rank = block_scan_incl(ties, s_tot) - ties;  // ties at lower indices
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        bool take = ok[i] && key[i] > pref;
        if (ok[i] && key[i] == pref) {
            take = rank < need;
            ++rank;
        }
        if (take) {
            const uint32_t slot = atomicAdd(&s_cnt, 1u);
            s_selk[slot] = key[i];
            s_seli[slot] = (uint32_t)(4 * tid + i);
        }
    }
    __syncthreads();
    if (warp != 0) return;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += s_red[1][w];
    const float inv_s = 1.0f / s;
    uint32_t mk = 0u, mi = 0u;
    int r = 0;
    if (lane < k) {
        mk = s_selk[lane];
        mi = s_seli[lane];
        for (int q = 0; q < k; ++q) {
            const uint32_t qk = s_selk[q], qi = s_seli[q];
            r += (qk > mk || (qk == mk && qi < mi)) ? 1 : 0;
        }
    }
    // the pick's softmax numerator (its own logit: the key holds it unless
    // the selection was biased)
    const float lv = lane < k ? (sel_bias ? __ldcg(row + mi) : fkey_value(mk)) : 0.f;
    float num = lane < k ? expf(lv - m) : 0.f;
    float w = num * inv_s;
    if (renorm) {
        // sum of the k numerators in pick order (lane r holds pick r)
        __shared__ float s_num[32];
        if (lane < k) s_num[r] = num;
        __syncwarp();
        float z = 0.f;
        for (int q = 0; q < k; ++q) z += s_num[q];
        w = num / z;
    }
    if (lane < k) {
        idx_row[r] = (int32_t)mi;
        w_row[r] = w;
        if (idx_out_row) idx_out_row[r] = (int32_t)mi;
        if (w_out_row) w_out_row[r] = w;
    }
}
// Token t of a decode chunk: logits, picks and weights in the workspace.
__device__ void cta_topk(const RouteParams &p, int t) {
    const int k = p.k;
    cta_topk_row(reinterpret_cast<const float *>(p.ws + p.L.logits) + (size_t)t * p.E, p.E, k,
                 reinterpret_cast<int32_t *>(p.ws + p.L.idx) + t * k, reinterpret_cast<float *>(p.ws + p.L.wt) + t * k,
                 p.idx_out ? p.idx_out + (size_t)t * k : nullptr, p.w_out ? p.w_out + (size_t)t * k : nullptr,
                 (p.route_flags & kRouteBiasSelect) ? p.bias : nullptr, (p.route_flags & kRouteRenorm) != 0);
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

// Tensor maps hold only plane addresses: an expert's maps are rewritten only
// when its blob pointer differs from the one they were written for (kept in
// the workspace).  Thread i of n takes experts i, i + n, ...; index E is the
// shared expert.
__device__ void refresh_tmaps(const RouteParams &p, int i0, int n) {
    const uint8_t **cache = reinterpret_cast<const uint8_t **>(p.ws + p.L.tcache);
    for (int e = i0; e < p.E + 1; e += n) {
        if (e < p.E) {
            const uint8_t *b = p.blobs[e];
            if (b != cache[e] && b != nullptr && (reinterpret_cast<uintptr_t>(b) & 15u) == 0u) {
                write_expert_tmaps(p.ws, p.L, e, b, p.tmpl, p.scale_mask);
                cache[e] = b;
            }
        } else if (p.has_shared) {
            if (cache[p.E] != p.sw[0] || cache[p.E + 1] != p.sw[1] || cache[p.E + 2] != p.sw[2]) {
                write_shared_tmaps(p.ws, p.L, p.smap);
                cache[p.E] = p.sw[0];
                cache[p.E + 1] = p.sw[1];
                cache[p.E + 2] = p.sw[2];
            }
        }
    }
}

// Warp that holds chunk c when N chunks are split evenly over W warps
// (warp j holds [floor(jN/W), floor((j+1)N/W))).
__device__ __forceinline__ int chunk_owner(long long c, long long N, int W) {
    return (int)(((c + 1) * (long long)W - 1) / N);
}

// ------------------------------------------------------ router stream --
// Router GEMV l = W_r x + b.  The fp32 router is one array of E*d floats; CTA
// c of G owns the contiguous units [c*U/G, (c+1)*U/G) of 16 floats (U =
// E*d/16; rows are whole units since d is a multiple of 64).  Its slice goes
// through a ring of kRStage-byte shared-memory stages filled by bulk
// asynchronous copies, so one thread keeps the SM's memory pipe full.  Thread
// i of a stage takes its 16 floats (one row), the warp sums lanes of equal
// row with a fixed shuffle tree (segmented), and after the stage's barrier
// threads fold the warps' row sums into the CTA's row accumulators in warp
// order, so every sum has a fixed order.  Rows cut by a CTA boundary are
// finished by the last of their CTAs to arrive, summing the CTAs' parts in
// CTA order.
constexpr int kRStage = 16384;               // bytes per ring stage
constexpr int kRFloats = kRStage / 4;        // 4096 floats: 256 units of 16
constexpr int kRSegs = 16;                   // row segments per warp and stage (512 floats, d >= 64)
constexpr int kRMaxRows = 72;                // rows of one CTA's slice (E/G + 2 <= 66)
constexpr int kRFast = 8;                    // slices of at most this many rows: per-thread row sums

struct RouteSmem {
    float acc[kRMaxRows][kRouteTok];
    int seg_row[2][8][kRSegs];
    float seg_val[2][8][kRSegs][kRouteTok];
    int seg_n[2][8];
};

__host__ __device__ inline int route_smem_bytes(int d, int nt, int nstage) {
    return nstage * kRStage + nt * d * 4 + (int)sizeof(RouteSmem) + nstage * 8 + 64;
}

// This CTA's router slice: units [u0, u1) of 16 floats, in stages of 256.
__device__ __forceinline__ void router_slice(const RouteParams &p, long long &u0, long long &u1) {
    const long long U = (long long)p.E * p.d / 16;
    u0 = (long long)blockIdx.x * U / gridDim.x;
    u1 = (long long)(blockIdx.x + 1) * U / gridDim.x;
}
__device__ __forceinline__ void router_issue(const RouteParams &p, uint8_t *ring, uint64_t *full, long long u0,
                                             long long u1, int j, int slot) {
    const long long a = u0 + 256LL * j;
    const long long e = min(u1, a + 256);
    const uint32_t bytes = (uint32_t)((e - a) * 64);
    mbar_arrive_expect_tx(&full[slot], bytes);
    bulk_g2s(ring + (size_t)slot * kRStage, p.wr + a * 16, bytes, &full[slot]);
}
// One thread: the first stages of a pass (the ring is free), issued before
// anything else so the weight stream starts at once.
__device__ void router_prefetch(const RouteParams &p, uint8_t *ring, uint64_t *full, int nstage, int chunk) {
    long long u0, u1;
    router_slice(p, u0, u1);
    const int nch = (int)((u1 - u0 + 255) / 256);
    for (int j = 0; j < nch && j < nstage; ++j) router_issue(p, ring, full, u0, u1, j, (chunk + j) % nstage);
}

// Streams this CTA's router slice once for tokens t0 .. t0+nt-1 (x in xs as
// fp32 [nt][d]; the first stages already issued by router_prefetch);
// finishes the rows it can and counts them on router_done.  `chunk` numbers
// the CTA's stages across passes (ring phase).  All threads.
__device__ void stream_router(const RouteParams &p, WsHeader *hdr, uint8_t *ring, uint64_t *full, int nstage,
                              const float *xs, RouteSmem &sm, int t0, int nt, int pass, int &chunk) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int d = p.d, G = gridDim.x, c = blockIdx.x;
    const long long U = (long long)p.E * d / 16;
    long long u0, u1;
    router_slice(p, u0, u1);
    const int row_base = (int)(u0 * 16 / d);
    const int nrows = u1 > u0 ? (int)((u1 * 16 - 1) / d) - row_base + 1 : 0;
    const int nch = (int)((u1 - u0 + 255) / 256);
    for (int i = tid; i < kRMaxRows * kRouteTok; i += blockDim.x) (&sm.acc[0][0])[i] = 0.f;
    auto issue = [&](int j, int slot) { router_issue(p, ring, full, u0, u1, j, slot); };
    // Few rows per slice (the usual case): each thread keeps its own sum per
    // row of the slice across all stages, and the warps reduce once at the
    // end.  Otherwise the row sums are reduced and folded stage by stage.
    const bool fast = nrows <= kRFast;
    float racc[kRFast][kRouteTok];
#pragma unroll
    for (int k = 0; k < kRFast; ++k)
#pragma unroll
        for (int t = 0; t < kRouteTok; ++t) racc[k][t] = 0.f;
    __syncthreads();  // the accumulators are cleared
    for (int j = 0; j < nch; ++j, ++chunk) {
        const int slot = chunk % nstage;
        const uint32_t par = (uint32_t)((chunk / nstage) & 1);
        // bounded; after a timeout the CTA keeps going (its barriers stay in
        // step) with unused values, the status word says so
        {
            // lane 0 polls; the others then take the completed phase themselves
            int ok = 1;
            if (lane == 0) ok = mbar_wait_bounded(&full[slot], par, hdr, p.wait_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (ok && lane != 0) (void)mbar_try_wait(&full[slot], par);
        }
        const long long unit = u0 + 256LL * j + tid;
        int row = -1;
        float v[kRouteTok];
#pragma unroll
        for (int t = 0; t < kRouteTok; ++t) v[t] = 0.f;
        if (unit < u1) {
            const uint32_t f = (uint32_t)unit * 16u;  // E*d < 2^31 floats
            row = (int)(f / (uint32_t)d);
            const int col = (int)(f - (uint32_t)row * (uint32_t)d);
            const float4 *w4 = reinterpret_cast<const float4 *>(ring + (size_t)slot * kRStage) + tid * 4;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 w = w4[q];
#pragma unroll
                for (int t = 0; t < kRouteTok; ++t) {
                    if (t < nt) {
                        const float4 xv = *reinterpret_cast<const float4 *>(xs + t * d + col + 4 * q);
                        v[t] = fmaf(w.x, xv.x, v[t]);
                        v[t] = fmaf(w.y, xv.y, v[t]);
                        v[t] = fmaf(w.z, xv.z, v[t]);
                        v[t] = fmaf(w.w, xv.w, v[t]);
                    }
                }
            }
        }
        if (fast) {
            if (row >= 0) {
                const int k = row - row_base;
#pragma unroll
                for (int kk = 0; kk < kRFast; ++kk)
                    if (kk == k)
#pragma unroll
                        for (int t = 0; t < kRouteTok; ++t) racc[kk][t] += v[t];
            }
            if (j + nstage < nch) {
                __syncthreads();  // every thread is done with this stage: refill it
                if (tid == 0) issue(j + nstage, slot);
            }
            continue;
        }
        // segmented sum over lanes of equal row (rows do not decrease along lanes)
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int rn = __shfl_down_sync(0xffffffffu, row, o);
#pragma unroll
            for (int t = 0; t < kRouteTok; ++t) {
                const float vn = __shfl_down_sync(0xffffffffu, v[t], o);
                if (lane + o < 32 && rn == row) v[t] += vn;
            }
        }
        const int rprev = __shfl_up_sync(0xffffffffu, row, 1);
        const bool head = row >= 0 && (lane == 0 || rprev != row);
        const uint32_t heads = __ballot_sync(0xffffffffu, head);
        const int b = j & 1;
        if (head) {
            const int k = __popc(heads & ((1u << lane) - 1u));
            sm.seg_row[b][warp][k] = row;
#pragma unroll
            for (int t = 0; t < kRouteTok; ++t) sm.seg_val[b][warp][k][t] = v[t];
        }
        if (lane == 0) sm.seg_n[b][warp] = __popc(heads);
        __syncthreads();  // this stage is read and its row sums posted
        if (tid == 0 && j + nstage < nch) issue(j + nstage, slot);
        if (tid < nrows) {
            const int r = row_base + tid;
            for (int w = 0; w < 8; ++w)
                for (int k = 0; k < sm.seg_n[b][w]; ++k)
                    if (sm.seg_row[b][w][k] == r)
#pragma unroll
                        for (int t = 0; t < kRouteTok; ++t) sm.acc[tid][t] += sm.seg_val[b][w][k][t];
        }
    }
    if (fast) {
        // per row: the warp's sum (fixed butterfly), then the warps in order
#pragma unroll
        for (int k = 0; k < kRFast; ++k) {
            if (k < nrows) {
#pragma unroll
                for (int t = 0; t < kRouteTok; ++t) {
                    if (t < nt) {
                        float v = racc[k][t];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                        if (lane == 0) sm.seg_val[0][warp][k][t] = v;
                    }
                }
            }
        }
        __syncthreads();
        if (tid < nrows)
            for (int w = 0; w < 8; ++w)
#pragma unroll
                for (int t = 0; t < kRouteTok; ++t)
                    if (t < nt) sm.acc[tid][t] += sm.seg_val[0][w][tid][t];
    }
    // every stage this CTA issued has been waited for above (a stage whose
    // wait ran out is the only copy that may not have landed)
    __syncthreads();  // every fold is done
    if (tid < nrows) {
        const int r = row_base + tid;
        const long long rs = (long long)r * d / 16, re = (long long)(r + 1) * d / 16;  // its units
        float *logits = reinterpret_cast<float *>(p.ws + p.L.logits);
        const float bias = (p.bias && !(p.route_flags & kRouteBiasSelect)) ? p.bias[r] : 0.f;
        bool done = false;
        float out[kRouteTok];
        if (rs >= u0 && re <= u1) {
#pragma unroll
            for (int t = 0; t < kRouteTok; ++t) out[t] = sm.acc[tid][t];
            done = true;
        } else {
            // cut by a CTA boundary: park this CTA's part; the last to arrive
            // sums the parts in CTA order
            const int first = chunk_owner(rs, U, G);
            const int nseg = chunk_owner(re - 1, U, G) - first + 1;
            float *pp = reinterpret_cast<float *>(p.ws + p.L.part) + (((size_t)(pass & 1) * p.E + r) * kMaxSeg) * kRouteTok;
            uint32_t *pc = reinterpret_cast<uint32_t *>(p.ws + p.L.cnt) + (size_t)(pass & 1) * p.E + r;
#pragma unroll
            for (int t = 0; t < kRouteTok; ++t) pp[(c - first) * kRouteTok + t] = sm.acc[tid][t];
            const uint32_t old = atom_add_acq_rel(pc, 1u);
            if (old == (uint32_t)(nseg - 1)) {
#pragma unroll
                for (int t = 0; t < kRouteTok; ++t) out[t] = 0.f;
                for (int sl = 0; sl < nseg; ++sl)
#pragma unroll
                    for (int t = 0; t < kRouteTok; ++t) out[t] += __ldcg(pp + sl * kRouteTok + t);
                *pc = 0u;
                done = true;
            }
        }
        if (done) {
            for (int t = 0; t < nt; ++t) logits[(size_t)(t0 + t) * p.E + r] = out[t] + bias;
            red_add_release(&hdr->router_done, 1u);  // after this thread's logit stores
        }
    }
}

// Wait (bounded) until *ctr reaches target; false (timeout bit set) if not.
__device__ bool wait_count(const uint32_t *ctr, uint32_t target, WsHeader *hdr, uint64_t limit_ns) {
    if (spin_geq(ctr, target, limit_ns)) return true;
    set_status(hdr, kStTimeout);
    return false;
}

// Cooperative launch (every CTA resident), one CTA per SM.  Every CTA
// streams its slice of the router; once all rows are in, token t's top-k runs
// on CTA t mod G (all its warps), and CTA 0, after its own tokens, waits for
// the others' and dispatches.  Meanwhile CTAs 1.. (CTA 0 when it is alone)
// build the gate/up pass's activation pieces and every expert's tensor maps,
// which need no routing.
__global__ void __launch_bounds__(kRouteThreads, 1) route_kernel(const __grid_constant__ RouteParams p) {
    extern __shared__ __align__(128) uint8_t rsm[];
    const int nstage = p.nstage;
    const int ntmax = min(p.Tc, kRouteTok);
    uint8_t *ring = rsm;
    float *xs = reinterpret_cast<float *>(rsm + (size_t)nstage * kRStage);  // [ntmax][d]
    RouteSmem &sm = *reinterpret_cast<RouteSmem *>(xs + (size_t)ntmax * p.d);
    uint64_t *full = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(&sm) + sizeof(RouteSmem));
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws + p.L.hdr);
    __shared__ int s_ok;
    if (threadIdx.x == 0) {
        for (int st = 0; st < nstage; ++st) mbar_init(&full[st], 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_trigger();
    const int npass = (p.Tc + kRouteTok - 1) / kRouteTok;
    const int G = gridDim.x;
    const int warp = threadIdx.x >> 5;
    int chunk = 0;
    if (threadIdx.x == 0) router_prefetch(p, ring, full, nstage, 0);  // pass 0's first stages
    // while the first router stages are in flight
    if (p.blobs != nullptr) {
        refresh_tmaps(p, blockIdx.x * kRouteThreads + threadIdx.x, G * kRouteThreads);
        if (blockIdx.x == 0 && G > 1) {
            // CTA 0 builds no x pieces: its maps are all it publishes to the
            // gate/up pass's shared units (the other CTAs count after their pieces)
            __syncthreads();
            if (threadIdx.x == 0) red_add_release(&hdr->prep_done, 1u);
        }
    }
    for (int pass = 0; pass < npass; ++pass) {
        const int t0 = pass * kRouteTok;
        const int nt = min(kRouteTok, p.Tc - t0);
        __syncthreads();  // the previous pass no longer reads xs or the ring
        if (pass > 0 && threadIdx.x == 0) router_prefetch(p, ring, full, nstage, chunk);
        // x of these tokens as fp32: 16-byte loads, several in flight per thread
        const uint4 *xv = reinterpret_cast<const uint4 *>(p.x + (size_t)t0 * p.d);
        const int n8 = nt * p.d / 8;
#pragma unroll 4
        for (int i = threadIdx.x; i < n8; i += blockDim.x) {
            const uint4 w = __ldg(xv + i);
            float4 *o = reinterpret_cast<float4 *>(xs + 8 * i);
            o[0] = make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
            o[1] = make_float4(bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w));
        }
        __syncthreads();
        stream_router(p, hdr, ring, full, nstage, xs, sm, t0, nt, pass, chunk);
    }
    // work of the gate/up pass that needs no routing (before the top-k wait
    // on a lone CTA, after it elsewhere is not needed: other CTAs do it)
    auto prep = [&](int first_cta) {
        if (p.blobs == nullptr) return;
        const int nworkers = G - first_cta;
        const int wi = (blockIdx.x - first_cta) * (kRouteThreads / 32) + warp;
        build_x_pieces(p.x, p.Tc, p.d, p.ws, p.L, wi, nworkers * (kRouteThreads / 32), p.has_shared != 0);
    };
    if (G == 1 && p.blobs != nullptr) {
        prep(0);
        __syncthreads();
        if (threadIdx.x == 0) red_add_release(&hdr->prep_done, 1u);
    }
    // top-k of this CTA's tokens once every router row is in
    if ((int)blockIdx.x < p.Tc) {
        __syncthreads();
        if (threadIdx.x == 0) s_ok = wait_count(&hdr->router_done, (uint32_t)(p.E * npass), hdr, p.wait_ns);
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
        if (threadIdx.x == 0) s_ok = wait_count(&hdr->topk_done, (uint32_t)(p.Tc - mine), hdr, p.wait_ns);
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
    prep(1);
    if (p.blobs != nullptr) {
        __syncthreads();
        if (threadIdx.x == 0) red_add_release(&hdr->prep_done, 1u);  // after this CTA's pieces and maps
    }
}

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
            if (b != nullptr) {
                // slot 0's maps now hold this blob (the layer's map cache sees it)
                write_expert_tmaps(p.ws, p.L, 0, b, p.tmpl, p.scale_mask);
                reinterpret_cast<const uint8_t **>(p.ws + p.L.tcache)[0] = b;
            }
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

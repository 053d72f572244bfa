// Routing of one token chunk (up to kChunk tokens): the router GEMV on its
// fp32 weights, streamed by warps with plain loads over equal ranges of row
// parts (a row's parts are summed by the last one to finish, in part order);
// one CTA per token waits for every router row, then runs the softmax over
// all experts and the token's top-k; CTA 0 dispatches (distinct experts, their
// slots and blob pointers).  The streaming CTAs then build the activation
// pieces the tensor-core gate/up pass reads.  Layer structure: the tutorial page's
// section 2.4 moe_forward (route, per selected expert FFN, weighted combine);
// the expert FFNs themselves are in umma_kernels.cuh.
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
    int nded;           // CTAs 0 .. nded-1 run no router stream (pieces, top-k, dispatch)
    uint4 tmpl[kTemplates][8];  // tensor-map templates (see kTemplates)
    int scale_mask;     // which scale-plane templates exist (bit 0: W_g/W_u, bit 1: W_d)
    uint4 smap[kSharedMaps][8];  // shared expert tensor maps (W_g, W_u, W_d, W_d 256-row), when has_shared
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
constexpr int kRouteTok = 4;  // tokens per pass over the router (their x columns held in registers)
// the router partial sums are double-buffered by pass parity: at most two passes
static_assert(kChunk <= 2 * kRouteTok, "a chunk takes at most two router passes");
// Dynamic shared memory of the route kernel: CTA 0's copies of the blob
// pointer table and of the maps' blob pointers, and a placeholder row.
__host__ __device__ inline int route_dyn_bytes(int E) { return E * (8 + 8 + 4); }

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
// idx_sh (optional, shared memory): the picks again, for a dispatch by the
// same CTA.  row_shared: row is in shared memory (else global, written by
// other CTAs: read through L2).  Not inlined: one copy of the code serves
// every call, so a call on placeholder data warms the instruction caches for
// the real one.
__device__ __noinline__ void cta_topk_row(const float *row, int E, int k, int32_t *idx_row, float *w_row,
                                          int32_t *idx_out_row, float *w_out_row, const float *sel_bias,
                                          bool renorm, int32_t *idx_sh, bool row_shared) {
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
        v[i] = ok[i] ? (row_shared ? row[e] : __ldcg(row + e)) : -INFINITY;
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
    const float lv = lane < k ? (sel_bias ? (row_shared ? row[mi] : __ldcg(row + mi)) : fkey_value(mk)) : 0.f;
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
        if (idx_sh) idx_sh[r] = (int32_t)mi;
        if (idx_out_row) idx_out_row[r] = (int32_t)mi;
        if (w_out_row) w_out_row[r] = w;
    }
}
// ptab, tc: the blob pointer table and the maps' blob pointers, copied to
// shared memory by the caller.
__device__ void dispatch(const RouteParams &p, WsHeader *hdr, const uint8_t *const *ptab, const uint8_t **tc) {
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
            const uint8_t *b = ptab[w];
            if ((reinterpret_cast<uintptr_t>(b) & 15u) != 0u || b == nullptr) {
                set_status(hdr, kStDeviceCheck);
                b = nullptr;
            }
            ublob[u] = b;
            ueid[u] = w;
            gmask[u] = umask[u];
            // the expert's tensor maps, rewritten when its blob pointer changed
            if (b != nullptr && tc[w] != b) {
                write_expert_tmaps(p.ws, L, w, b, p.tmpl, p.scale_mask);
                reinterpret_cast<const uint8_t **>(p.ws + L.tcache)[w] = b;
            }
        }
    }
}

// Tensor maps hold only plane addresses: an expert's maps are rewritten only
// when its blob pointer differs from the one they were written for (kept in
// the workspace).  Thread i of n takes experts i, i + n, ...; index E is the
// shared expert.
// Indices from i0 below e_end only (default: all of them).
__device__ void refresh_tmaps(const RouteParams &p, int i0, int n, int e_end = -1) {
    const uint8_t **cache = reinterpret_cast<const uint8_t **>(p.ws + p.L.tcache);
    if (e_end < 0) e_end = p.E + 1;
    for (int e = i0; e < e_end; e += n) {
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

// ------------------------------------------------------ router stream --
// Router GEMV l = W_r x + b.  Row r of the fp32 router is summed as P = d / Ls
// parts of Ls floats (router_part_len); part q of row r is segment s = q*E + r
// (part-major, so consecutive segments of a warp share their x columns).  The
// streaming warps take equal contiguous ranges of the E*P segments.  A warp
// reads a segment with plain 16-byte loads straight from HBM (no shared-memory
// staging: several segments' loads are in flight per lane, so the SM's load
// path, not its bulk-copy engine, sets the rate), multiplies it with the x
// columns it holds in registers and sums the 32 lanes with a fixed butterfly.
// The part's sum goes to the workspace; the last of a row's P parts to arrive
// adds the P sums in part order (q = 0 .. P-1), so every logit has one fixed
// summation order whatever the grid.
// Segments whose loads a lane issues together (8 x 2 KB per warp in flight
// with one token; with four tokens the x columns take the registers of half).
template <int NT>
__host__ __device__ constexpr int router_batch() { return NT == 1 ? 8 : 4; }

template <int NT>
__device__ void stream_router(const RouteParams &p, WsHeader *hdr, int t0, int nt, int pass, int wi, int nw) {
    const int lane = threadIdx.x & 31;
    const int d = p.d, E = p.E;
    const int Ls = router_part_len(d), P = d / Ls;
    const int nv = Ls >= 128 ? Ls / 128 : 1;  // float4 per lane per segment
    const bool lact = Ls >= 128 || lane < 16;
    const int NS = E * P;  // E*d < 2^31 floats
    const int s0 = (int)((long long)wi * NS / nw), s1 = (int)((long long)(wi + 1) * NS / nw);
    float *part = reinterpret_cast<float *>(p.ws + p.L.part) + (size_t)(pass & 1) * NS * kRouteTok;
    uint32_t *cnt = reinterpret_cast<uint32_t *>(p.ws + p.L.cnt) + (size_t)(pass & 1) * E;
    float *logits = reinterpret_cast<float *>(p.ws + p.L.logits);
    const bool add_bias = p.bias && !(p.route_flags & kRouteBiasSelect);
    float xr[NT][16];
    int xq = -1;
    // x columns q*Ls + 128 i + 4 lane .. +3 of each token (bf16 -> fp32)
    auto load_x = [&](int q) {
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (t < nt && i < nv && lact) {
                    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p.x + (size_t)(t0 + t) * d + (size_t)q * Ls +
                                                                          128 * i + 4 * lane));
                    xr[t][4 * i + 0] = bf16_lo(u.x);
                    xr[t][4 * i + 1] = bf16_hi(u.x);
                    xr[t][4 * i + 2] = bf16_lo(u.y);
                    xr[t][4 * i + 3] = bf16_hi(u.y);
                }
        xq = q;
    };
    if (s0 < s1) load_x(s0 / E);  // before the weight loads, so it lands first
    for (int g0 = s0; g0 < s1; g0 += 32) {
        // lane j owns segment g0 + j of this group: it stores the segment's sum
        // and counts it on its row
        const int ng = min(32, s1 - g0);
        constexpr int kRSeg = router_batch<NT>();
        for (int b0 = 0; b0 < ng; b0 += kRSeg) {
            float4 w[kRSeg][4];
#pragma unroll
            for (int b = 0; b < kRSeg; ++b) {
                if (b0 + b < ng) {
                    const int s = g0 + b0 + b, q = s / E, r = s - q * E;
                    const float4 *src = reinterpret_cast<const float4 *>(p.wr + (size_t)r * d + (size_t)q * Ls) + lane;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (i < nv && lact) w[b][i] = __ldcs(src + 32 * i);
                }
            }
            // every segment's products first, then the lane sums of all of
            // them side by side (independent shuffle chains overlap)
            float v[kRSeg][NT];
#pragma unroll
            for (int b = 0; b < kRSeg; ++b) {
#pragma unroll
                for (int t = 0; t < NT; ++t) v[b][t] = 0.f;
                if (b0 + b < ng) {
                    const int q = (g0 + b0 + b) / E;
                    if (q != xq) load_x(q);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (i < nv && lact) {
                            const float4 wv = w[b][i];
#pragma unroll
                            for (int t = 0; t < NT; ++t) {
                                v[b][t] = fmaf(wv.x, xr[t][4 * i + 0], v[b][t]);
                                v[b][t] = fmaf(wv.y, xr[t][4 * i + 1], v[b][t]);
                                v[b][t] = fmaf(wv.z, xr[t][4 * i + 2], v[b][t]);
                                v[b][t] = fmaf(wv.w, xr[t][4 * i + 3], v[b][t]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int b = 0; b < kRSeg; ++b)
#pragma unroll
                    for (int t = 0; t < NT; ++t) v[b][t] += __shfl_xor_sync(0xffffffffu, v[b][t], o);
#pragma unroll
            for (int b = 0; b < kRSeg; ++b) {
                if (b0 + b < ng && lane == b0 + b) {
                    const int s = g0 + b0 + b, q = s / E, r = s - q * E;
                    float *dst = part + ((size_t)r * P + q) * kRouteTok;
#pragma unroll
                    for (int t = 0; t < NT; ++t)
                        if (t < nt) dst[t] = v[b][t];
                }
            }
        }
        if (lane < ng) {
            const int s = g0 + lane, q = s / E, r = s - q * E;
            (void)q;
            // release: this lane's part store; acquire: the other parts of the row
            const uint32_t old = atom_add_acq_rel(&cnt[r], 1u);
            if (old == (uint32_t)(P - 1)) {
                float out[NT];
#pragma unroll
                for (int t = 0; t < NT; ++t) out[t] = 0.f;
                const float *src = part + (size_t)r * P * kRouteTok;
#pragma unroll 7
                for (int qq = 0; qq < P; ++qq)
#pragma unroll
                    for (int t = 0; t < NT; ++t)
                        if (t < nt) out[t] += __ldcg(src + qq * kRouteTok + t);
                cnt[r] = 0u;
                const float bv = add_bias ? __ldg(p.bias + r) : 0.f;
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    if (t < nt) logits[(size_t)(t0 + t) * E + r] = out[t] + bv;
                red_add_release(&hdr->router_done, 1u);  // after this lane's logit stores
            }
        }
    }
}

// Wait (bounded) until *ctr reaches target; false (timeout bit set) if not.
__device__ bool wait_count(const uint32_t *ctr, uint32_t target, WsHeader *hdr, uint64_t limit_ns) {
    if (spin_geq(ctr, target, limit_ns)) return true;
    set_status(hdr, kStTimeout);
    return false;
}

// One token (Tc == 1): the dispatch by warp 0 right after the token's top-k
// (its k picks are k distinct experts): expert of pick j goes to distinct
// slot u = number of picks with a smaller id, so the slots are in ascending
// id as the general dispatch orders them; the picked experts' tensor maps
// are rewritten where their blob pointer changed.  picks: the k picks in shared
// memory; ptab, tc: shared copies of the blob pointer table and of the maps'
// blob pointers; o: the workspace's dispatch arrays.
// Where dispatch_one writes (the workspace's dispatch arrays).
struct DispatchOut {
    const uint8_t **ublob;
    int32_t *ueid;
    uint32_t *umask;
    int8_t *uslot;
    uint32_t *n_unique;
};
__device__ __noinline__ void dispatch_one(const RouteParams &p, WsHeader *hdr, int k, const int32_t *picks,
                                          const uint8_t *const *ptab, const uint8_t *const *tc, DispatchOut o) {
    const int lane = threadIdx.x & 31;
    int e = 0x7FFFFFFF;
    if (lane < k) e = picks[lane];
    int u = 0;
    for (int q = 0; q < k; ++q) u += __shfl_sync(0xffffffffu, e, q) < e ? 1 : 0;
    if (lane < k) {
        const uint8_t *b = ptab[e];
        if ((reinterpret_cast<uintptr_t>(b) & 15u) != 0u || b == nullptr) {
            set_status(hdr, kStDeviceCheck);
            b = nullptr;
        }
        // the expert's tensor maps, rewritten when its blob pointer changed
        if (b != nullptr && tc[e] != b) {
            write_expert_tmaps(p.ws, p.L, e, b, p.tmpl, p.scale_mask);
            reinterpret_cast<const uint8_t **>(p.ws + p.L.tcache)[e] = b;
        }
        o.ublob[u] = b;
        o.ueid[u] = e;
        o.umask[u] = 1u;
#pragma unroll
        for (int t = 0; t < kChunk; ++t) o.uslot[(size_t)u * kChunk + t] = t == 0 ? (int8_t)lane : (int8_t)-1;
    }
    if (lane == 0) *o.n_unique = (uint32_t)k;
}

// Cooperative launch (every CTA resident), one CTA per SM.  CTAs 0 .. Tc-1
// (p.nded of them) stream nothing: they run their top-k code once on
// placeholder data (so the code is cached when the router rows arrive), wait
// for every router row, and each runs the softmax and top-k of token t = its
// index; CTA 0 then dispatches (at once for one token, else after the other
// tokens' top-k), refreshing the selected experts' maps.  The other CTAs
// stream the router (all tokens of the chunk, NT per pass) and then build the
// gate/up pass's activation pieces (the last one also the shared expert's
// maps).  Every CTA counts on prep_done once, after what it writes there.
template <int NT>
__global__ void __launch_bounds__(kRouteThreads, 1) route_kernel(const __grid_constant__ RouteParams p) {
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws + p.L.hdr);
    __shared__ int s_ok;
    __shared__ int32_t s_didx[32];
    __shared__ float s_dw[32];
    extern __shared__ __align__(16) uint8_t rdyn[];  // route_dyn_bytes(E): CTA 0's tables
    pdl_trigger();
    const int G = gridDim.x, nded = p.nded;
    const int warp = threadIdx.x >> 5;
    const int npass = (p.Tc + NT - 1) / NT;
    if ((int)blockIdx.x >= nded) {
        const int nw = (G - nded) * (kRouteThreads / 32);
        const int wi = ((int)blockIdx.x - nded) * (kRouteThreads / 32) + warp;
        for (int pass = 0; pass < npass; ++pass)
            stream_router<NT>(p, hdr, pass * NT, min(NT, p.Tc - pass * NT), pass, wi, nw);
        if (p.blobs != nullptr) {
            // a share of the activation pieces (x is in L2 by now): one
            // 32-column block per warp for most warps; the last CTA (which
            // has no pieces at the usual sizes) the shared expert's maps
            build_x_pieces(p.x, p.Tc, p.d, p.ws, p.L, wi, nw, p.has_shared != 0);
            if ((int)blockIdx.x == G - 1 && threadIdx.x == 0) refresh_tmaps(p, p.E, 1);  // index E
            __syncthreads();
            if (threadIdx.x == 0) red_add_release(&hdr->prep_done, 1u);  // after this CTA's pieces (and maps)
        }
        return;
    }
    // ---- CTAs 0 .. nded-1: top-k (they write nothing the gate/up pass's
    // shared units read: they count on prep_done at once).  Everything the
    // top-k and the dispatch take from the launch parameters is read here,
    // at the start, into shared memory: after the last router row arrives
    // no constant-bank miss sits on the path.
    struct TopkArgs {
        const float *row;
        int32_t *idx_row, *idx_out;
        float *w_row, *w_out;
        const float *sel_bias;
        DispatchOut out;
        uint64_t wait_ns;
        uint32_t rows_target;
        int E, k, renorm, Tc, dispatch;
    };
    __shared__ TopkArgs s_a;
    const int t = blockIdx.x;  // this CTA's token (nded = Tc)
    if (threadIdx.x == 0) {
        s_a.row = reinterpret_cast<const float *>(p.ws + p.L.logits) + (size_t)t * p.E;
        s_a.idx_row = reinterpret_cast<int32_t *>(p.ws + p.L.idx) + t * p.k;
        s_a.w_row = reinterpret_cast<float *>(p.ws + p.L.wt) + t * p.k;
        s_a.idx_out = p.idx_out ? p.idx_out + (size_t)t * p.k : nullptr;
        s_a.w_out = p.w_out ? p.w_out + (size_t)t * p.k : nullptr;
        s_a.sel_bias = (p.route_flags & kRouteBiasSelect) ? p.bias : nullptr;
        s_a.out = DispatchOut{reinterpret_cast<const uint8_t **>(p.ws + p.L.uniq_blob),
                              reinterpret_cast<int32_t *>(p.ws + p.L.uniq_eid),
                              reinterpret_cast<uint32_t *>(p.ws + p.L.uniq_mask),
                              reinterpret_cast<int8_t *>(p.ws + p.L.uniq_slot), &hdr->n_unique};
        s_a.wait_ns = p.wait_ns;
        s_a.rows_target = (uint32_t)(p.E * npass);
        s_a.E = p.E;
        s_a.k = p.k;
        s_a.renorm = (p.route_flags & kRouteRenorm) != 0;
        s_a.Tc = p.Tc;
        s_a.dispatch = p.blobs != nullptr;
        if (p.blobs != nullptr) red_add_release(&hdr->prep_done, 1u);
    }
    const uint8_t **s_ptab = reinterpret_cast<const uint8_t **>(rdyn);  // [E] blob pointers
    const uint8_t **s_tc = s_ptab + p.E;                                // [E] the maps' blob pointers
    float *s_row = reinterpret_cast<float *>(s_tc + p.E);               // [E] placeholder row
    for (int e = threadIdx.x; e < p.E; e += kRouteThreads) s_row[e] = 0.f;  // the placeholder row
    if (p.blobs != nullptr && blockIdx.x == 0) {
        // the dispatch reads these from shared memory: asynchronous copies,
        // waited for only before the dispatch
        const uint8_t *const *gtc = reinterpret_cast<const uint8_t *const *>(p.ws + p.L.tcache);
        for (int e = threadIdx.x; e < p.E; e += kRouteThreads) {
            cp_async8(&s_ptab[e], &p.blobs[e]);
            cp_async8(&s_tc[e], &gtc[e]);
        }
    }
    __syncthreads();
    const int E = s_a.E, k = s_a.k;
    // The top-k code runs once on placeholder data (a row of zeros in shared
    // memory: all ties, k valid picks; results to shared scratch) while the
    // router streams: the first run of that code on this SM waits on
    // instruction fetches (about 10 us at the K3 shape), the real run after
    // the last router row does not.  (A dry dispatch as well would end after
    // the router rows: the dispatch runs cold.)
    cta_topk_row(s_row, E, k, s_didx, s_dw, nullptr, nullptr, s_a.sel_bias, s_a.renorm != 0, nullptr, true);
    cp_async_wait_all();  // this thread's table copies
    __syncthreads();
    const bool one = s_a.Tc == 1 && s_a.dispatch;
    if (threadIdx.x == 0) s_ok = wait_count(&hdr->router_done, s_a.rows_target, hdr, s_a.wait_ns);
    __syncthreads();
    if (!s_ok) return;
    cta_topk_row(s_a.row, E, k, s_a.idx_row, s_a.w_row, s_a.idx_out, s_a.w_out, s_a.sel_bias, s_a.renorm != 0,
                 s_didx, false);
    __syncthreads();
    if (blockIdx.x > 0) {
        if (threadIdx.x == 0) red_add_release(&hdr->topk_done, 1u);  // after thread 0's own result stores
        return;
    }
    if (s_a.Tc > 1) {
        // the other tokens' top-k (their CTAs count on topk_done)
        if (threadIdx.x == 0) s_ok = wait_count(&hdr->topk_done, (uint32_t)(s_a.Tc - 1), hdr, s_a.wait_ns);
        __syncthreads();
        if (!s_ok) return;
        if (s_a.dispatch) dispatch(p, hdr, s_ptab, s_tc);
    } else if (one && warp == 0) {
        dispatch_one(p, hdr, k, s_didx, s_ptab, s_tc, s_a.out);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // the down pass reads the dispatch (and the selected experts' maps)
        // before the gate/up pass completes: publish it
        if (s_a.dispatch) red_add_release(&hdr->disp_cnt, 1u);
        hdr->router_done = 0u;
        hdr->topk_done = 0u;
    }
}

struct SingleParams {
    const uint16_t *x;
    int Tc, d;
    const uint8_t *blob;
    uint8_t *ws;
    Layout L;
    uint4 tmpl[kTemplates][8];
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
        __syncthreads();
        if (threadIdx.x == 0) red_add_release(&hdr->disp_cnt, 1u);  // the dispatch is written
    }
    build_x_pieces(p.x, p.Tc, p.d, p.ws, p.L, blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5),
                   gridDim.x * (blockDim.x >> 5), false);
    pdl_trigger();
}

}  // namespace k3

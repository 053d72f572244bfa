// Routed-expert projections on the 5th-generation tensor cores
// (tcgen05.mma kind::mxf4, block-scaled E2M1 x E2M1 with E8M0 scales).
//
// The packed expert blob goes straight into the tensor core: TMA copies
// 128-row x 128-byte boxes of a nibble plane into shared memory (128-byte
// swizzle) and the E8M0 scale bytes are written into tensor memory, so the
// MMA itself decodes every 4-bit weight and applies its block scale -- no
// per-weight thread work (the kimi-k3-in-c project card ("P053"), core
// features: multiply directly on the packed nibbles, never dequantise).
//
// Activations (x for gate/up, w*h for down) are carried as kPieces E2M1
// pieces per element, each 32-element block of each piece with its own E8M0
// scale chosen from the block's remaining residual; the pieces sum exactly
// to the activation up to the last residual (about 2^-19 of the block's
// largest element).  Piece p of token t is B-operand row n = t*kPieces + p,
// so a whole chunk of tokens and pieces is one MMA of N = act_n(Tc) columns
// and the pieces are summed per token in the epilogue.
//
// Work: "items" of 128 weight rows, each a run of K-tiles (256 weights of
// every row); the K-tiles of all items are split evenly over the CTAs
// (stream-K).  An item split between CTAs is finished by the last one to
// arrive, summing the per-token partials in piece order (deterministic).
//
// CTA roles (352 threads): warps 0-3 epilogue (one TMEM lane quadrant each),
// warps 4-7 write the scale factors of each stage into TMEM (each writes the
// same values into its own quadrant, as the MMA reads them replicated),
// warp 8 issues the TMA / bulk copies, warp 9 issues the MMAs, warp 10 (gate/
// up) loads the routing once the router kernel has finished.
//
// Gate/up runs two ranges of units, each split over the CTAs: first the
// shared expert's (they need no routing: x as bf16 and the shared tensor maps
// are published by the router kernel's CTAs through a counter), then the
// routed experts'.  So the shared expert streams while the router kernel's
// last CTAs still run the top-k and the dispatch.
#pragma once

#include "common.cuh"
#include "layout.cuh"
#include "umma.cuh"

namespace k3 {

constexpr int kUThreads = 352;
constexpr int kAtile = kTileM * 128;  // 128 rows x 128 bytes (16 KB) of an A operand
// Host-encoded tensor-map templates: [0] W_g/W_u nibbles, [1] W_d nibbles,
// [2] W_g/W_u scales, [3] W_d scales (128-row boxes), [4] W_d nibbles, [5]
// W_d scales (256-row boxes).
constexpr int kTemplates = 6;

// ---------------------------------------------------------------- pieces --
// One 32-element activation block (element = this lane's v) of token t ->
// kPieces E2M1 pieces.  Piece p: scale exponent e from the largest |residual|
// r of the block (smallest e with max|r| <= 6 * 2^e; the order of
// non-negative floats is the order of their bits, so one warp max-reduction
// of the bits finds it), codes = r / 2^e rounded to the nearest E2M1 value
// (ties to the even code), residual r -= code * 2^e (exact in fp32: the
// subtracted value is a multiple of the residual's unit in the last place).
// Rounding to the E2M1 grid: below 2 the grid step is 0.5, below 4 it is 1,
// up to 6 it is 2; adding then subtracting 2^22, 2^23 or 2^24 rounds an fp32
// of that size to a multiple of the step, ties to even.  The code of a grid
// value q >= 1 is read off its fp32 bits (exponent and top mantissa bit),
// below 1 it is 0 or 1 (0.5).
// Writes the 16-byte nibble row of each piece into a K-tile of the B operand
// (no-swizzle K-major core matrices; this block is 16-byte chunk c of the
// tile; element 2i in the low nibble of byte i): B row n = t*P + p goes to
// tile + c*cs + (n/8)*gs + (n%8)*16 (an MMA tile of N rows: cs = N/8*128,
// gs = 128), and its scale byte to the tile's scale words (sfw[(c/4)*sfrow +
// n], byte c%4).  All 32 lanes of the warp call it.
template <int P>
__device__ __forceinline__ void quantize_pieces_t(float v, int lane, int t, int c, int cs, int gs, int sfrow,
                                                  uint8_t *tile, uint8_t *sfw) {
    float r = v;
#pragma unroll
    for (int p = 0; p < P; ++p) {
        const uint32_t bits = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(r)));
        // amax = 1.f * 2^e0: 6 * 2^(e0-2) = 1.5 * 2^e0 covers 1.f <= 1.5
        int e = (int)(bits >> 23) - 127 - 2 + ((bits & 0x7FFFFFu) > 0x400000u ? 1 : 0);
        e = max(-126, min(126, e));
        const float s = r * exp2i(-e);
        const float m = fabsf(s);
        const float C = m < 2.f ? 4194304.f : (m < 4.f ? 8388608.f : 16777216.f);
        const float q = __fsub_rn(__fadd_rn(m, C), C);
        const uint32_t qb = __float_as_uint(q);
        uint32_t code = q >= 1.f ? (qb >> 22) - 252u : (q > 0.f ? 1u : 0u);
        code |= (s < 0.f && code != 0u) ? 8u : 0u;
        r = __fmaf_rn(-copysignf(q, s), exp2i(e), r);
        const uint32_t hi = __shfl_down_sync(0xffffffffu, code, 1);
        const int n = t * P + p;
        uint8_t *row = tile + c * cs + (n / 8) * gs + (n % 8) * 16;
        if ((lane & 1) == 0) row[lane >> 1] = (uint8_t)(code | (hi << 4));
        if (lane == 0) sfw[((c >> 2) * sfrow + n) * 4 + (c & 3)] = (uint8_t)(e + 127);
    }
}
// The same for NB tokens t0..t0+NB-1 at once (values v[b]): the NB chains
// of dependent steps interleave, so one warp keeps its pipeline busy.
template <int P, int NB>
__device__ __forceinline__ void quantize_pieces_batch(const float (&v)[NB], int lane, int t0, int c, int cs, int gs,
                                                      int sfrow, uint8_t *tile, uint8_t *sfw) {
    float r[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) r[b] = v[b];
#pragma unroll
    for (int p = 0; p < P; ++p) {
        uint32_t bits[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) bits[b] = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(r[b])));
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            int e = (int)(bits[b] >> 23) - 127 - 2 + ((bits[b] & 0x7FFFFFu) > 0x400000u ? 1 : 0);
            e = max(-126, min(126, e));
            const float s = r[b] * exp2i(-e);
            const float m = fabsf(s);
            const float C = m < 2.f ? 4194304.f : (m < 4.f ? 8388608.f : 16777216.f);
            const float q = __fsub_rn(__fadd_rn(m, C), C);
            const uint32_t qb = __float_as_uint(q);
            uint32_t code = q >= 1.f ? (qb >> 22) - 252u : (q > 0.f ? 1u : 0u);
            code |= (s < 0.f && code != 0u) ? 8u : 0u;
            r[b] = __fmaf_rn(-copysignf(q, s), exp2i(e), r[b]);
            const uint32_t hi = __shfl_down_sync(0xffffffffu, code, 1);
            const int n = (t0 + b) * P + p;
            uint8_t *row = tile + c * cs + (n / 8) * gs + (n % 8) * 16;
            if ((lane & 1) == 0) row[lane >> 1] = (uint8_t)(code | (hi << 4));
            if (lane == 0) sfw[((c >> 2) * sfrow + n) * 4 + (c & 3)] = (uint8_t)(e + 127);
        }
    }
}

__device__ __forceinline__ void quantize_pieces(float v, int lane, int t, int c, int N, uint8_t *tile,
                                                uint8_t *sfw) {
    quantize_pieces_t<kPieces>(v, lane, t, c, (N / 8) * 128, 128, kSfRow, tile, sfw);
}

// x of the chunk -> pieces (routed gate/up B operand) and, with a shared
// expert, x as bf16 in rows t*kPieces of the shared gate/up B operand (the
// other piece rows zero).  Blocks spread over every warp of the grid (warp
// index gw of nw).  norm_w (non-null): x is RMSNorm(h) of the given tokens,
// x_j = RNE_bf16((h_j * rnorm[t]) * norm_w[j]).
__device__ void build_x_pieces(const uint16_t *x, int Tc, int d, uint8_t *ws, const Layout &L, int gw, int nw,
                               bool shared, const uint16_t *norm_w = nullptr, const float *rnorm = nullptr) {
    const int lane = threadIdx.x & 31, N = act_n(Tc), nb = d / 32;
    for (int i = gw; i < Tc * nb; i += nw) {
        const int t = i / nb, b = i - t * nb;
        const int col = 32 * b + lane;
        uint16_t xv = x[(size_t)t * d + col];
        if (norm_w) xv = rms_norm_bf16(xv, rnorm[t], norm_w[col]);
        const float v = __uint_as_float((uint32_t)xv << 16);
        const int kt = b >> 3;
        quantize_pieces(v, lane, t, b & 7, N, ws + L.xb + (size_t)kt * N * 128,
                        ws + L.xsf + (size_t)kt * 2 * kSfRow * 4);
        if (shared) {
            uint8_t *tile = ws + L.xbf + (size_t)(col / kTileKs) * N * 128;
            const int c = (col % kTileKs) / 8, e = col % 8;
#pragma unroll
            for (int pc = 0; pc < kPieces; ++pc) {
                const int n = t * kPieces + pc;
                *reinterpret_cast<uint16_t *>(tile + (c * (N / 8) + n / 8) * 128 + (n % 8) * 16 + e * 2) =
                    pc == 0 ? xv : (uint16_t)0;
            }
        }
    }
}

// The shared expert's three tensor maps (encoded by the host with their real
// addresses) into the workspace, where the tensor-core kernels read them.
__device__ void write_shared_tmaps(uint8_t *ws, const Layout &L, const uint4 (&smap)[kSharedMaps][8]) {
    uint4 *o = reinterpret_cast<uint4 *>(ws + L.tmap + (size_t)L.E * kMapsPerExpert * 128);
#pragma unroll
    for (int m = 0; m < kSharedMaps; ++m)
#pragma unroll
        for (int j = 0; j < 8; ++j) o[m * 8 + j] = smap[m][j];
    umma::tmap_release();
}

// Tensor maps of expert e: copies of the host-encoded templates pointed at
// the expert's planes.  Templates: [0] W_g/W_u nibbles (ff rows of d/2 bytes),
// [1] W_d nibbles (d rows of ff/2 bytes), [2] W_g/W_u scales (ff rows of d/32
// bytes), [3] W_d scales (d rows of ff/32 bytes); the scale maps are written
// only where scale_mask says their template exists (bit 0: W_g/W_u, bit 1:
// W_d; the reduction length a multiple of 512).  One thread.  Not inlined:
// callers run it only when an expert's blob pointer changed and keep their
// hot code short.
__device__ __noinline__ void write_expert_tmaps(uint8_t *ws, const Layout &L, int e, const uint8_t *blob,
                                   const uint4 (&tmpl)[kTemplates][8], int scale_mask) {
    const size_t mat = (size_t)L.d * L.ff;
    uint8_t *dst = ws + L.tmap + (size_t)e * kMapsPerExpert * 128;
    const uint8_t *addr[kMapsPerExpert] = {blob,           blob + mat / 2 + mat / 32, blob + mat + mat / 16,
                                           blob + mat / 2, blob + mat + mat / 32,     blob + mat + mat / 16 + mat / 2,
                                           blob + mat + mat / 16, blob + mat + mat / 16 + mat / 2};
    const int which[kMapsPerExpert] = {0, 0, 1, 2, 2, 3, 4, 5};
#pragma unroll
    for (int m = 0; m < kMapsPerExpert; ++m) {
        if (which[m] == 2 && !(scale_mask & 1)) continue;
        if ((which[m] == 3 || which[m] == 5) && !(scale_mask & 2)) continue;
        const uint4 *src = tmpl[which[m]];
        uint4 *o = reinterpret_cast<uint4 *>(dst + m * 128);
#pragma unroll
        for (int j = 0; j < 8; ++j) o[j] = src[j];
        umma::tmap_set_address(dst + m * 128, addr[m]);
    }
    umma::tmap_release();
}

// ---------------------------------------------------------------- kernel --
struct UmmaParams {
    int Tc, d, ff, k;
    int ffs;          // shared expert rows (0: none)
    uint8_t *ws;
    Layout L;
    int nst;          // pipeline stages
    int sb;           // bytes per stage (umma_stage_bytes for this N)
    int sf_tma;       // A scales arrive by TMA with the stage (K a multiple of 512)
    // down only
    int out_fp32;     // y in fp32 (else bf16, rounded once)
    void *y;          // [Tc][d] of this chunk
    const uint16_t *resid;  // bf16 [Tc][d] added before the rounding (pre-norm calls), or null
    // gate/up: router-kernel CTAs that announce their x pieces and tensor maps
    // in the header's prep_done (0: nothing to wait for)
    int route_ctas;
    uint64_t wait_ns;  // bound of every device wait
    int strict;        // flag E8M0 NaN bytes (0xFF) among the weight scales read
    int inject;        // failure-path tests: 1 = never signal "routing loaded"
    // down only: the shared expert's W_d tensor map (256-row boxes), encoded by
    // the host with its real address (read from the launch parameters, so the
    // pass can stream it before the gate/up pass completes)
    alignas(64) uint4 smap_d[8];
};

// One pipeline stage for MMA width N: the A boxes (16 KB per matrix, first,
// so they stay 1024-byte aligned for the 128-byte swizzle), the B tile (N rows
// x 128 bytes), the A scale boxes (128 rows x 16 bytes per matrix: the scales
// of this K-tile and its neighbour) and the B scale words (2 x kSfRow words),
// rounded up to 1024 bytes.
__host__ __device__ inline int umma_sfa_off(bool, int N) { return 2 * kAtile + N * 128; }
__host__ __device__ inline int umma_sfb_off(bool gu, int N) { return umma_sfa_off(gu, N) + 2 * 2048; }
__host__ __device__ inline int umma_stage_bytes(bool gu, int N) {
    return (umma_sfb_off(gu, N) + 2 * kSfRow * 4 + 1023) & ~1023;
}
// TMEM scale columns of one stage, every group aligned: A scales 8 per matrix
// (2 groups x 4 row blocks), then B scales (group g at +4g, up to 2 columns).
__host__ __device__ inline int umma_sf_cols(bool) { return 32; }
// Per-call metadata copied into shared memory by every CTA: blob pointer,
// expert id and per-token routing weight (0 where the token did not select
// it) of each distinct expert.  Global loads issued while the weight stream
// saturates HBM wait thousands of cycles, so the pipeline never makes them.
constexpr int kMetaU = kChunk * 32;  // distinct experts of a chunk (top_k <= 32)
constexpr int kMetaBytes = kMetaU * 8 + kMetaU * 4 + kMetaU * kChunk * 4;
constexpr int kUBarBytes = 512;  // mbarriers, the TMEM address and flags after the stages
__host__ __device__ inline int umma_smem_bytes(bool gu, int N, int nst) {
    return 1024 + nst * umma_stage_bytes(gu, N) + kUBarBytes + kMetaBytes;
}

// Load the (up to) 8 scale bytes of one weight row for one K-tile: nks valid
// 2-byte pairs (one per MMA k-step); zero beyond.
__device__ __forceinline__ uint2 load_sf8(const uint8_t *p, int nks) {
    if (nks == 4 && (reinterpret_cast<uintptr_t>(p) & 7u) == 0u) return __ldg(reinterpret_cast<const uint2 *>(p));
    const unsigned short *h = reinterpret_cast<const unsigned short *>(p);
    uint32_t w0 = 0u, w1 = 0u;
    if (nks > 0) w0 |= (uint32_t)__ldg(h);
    if (nks > 1) w0 |= (uint32_t)__ldg(h + 1) << 16;
    if (nks > 2) w1 |= (uint32_t)__ldg(h + 2);
    if (nks > 3) w1 |= (uint32_t)__ldg(h + 3) << 16;
    return make_uint2(w0, w1);
}

// GU: routed items (distinct expert u, 128 rows of ff; K = d in 256-weight
// tiles) then the shared expert's items (128 rows of ff_s; K = d in 64-weight
// bf16 tiles).  Down: one item per 128 rows of d whose K runs over every
// distinct routed expert's ff (256-weight tiles) and then the shared
// expert's ff_s (64-weight bf16 tiles), all into one accumulator, so the
// routing weights (folded into the routed pieces) and the shared expert are
// combined by the tensor core itself.
template <bool GU>
__global__ void __launch_bounds__(kUThreads, 1) umma_expert_kernel(const __grid_constant__ UmmaParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    // Two 128-row A operands per stage: W_g and W_u (gate/up), or the two
    // halves of one 256-row box of W_d (down: one copy per 32 KB of weights)
    constexpr int NMAT = 2;
    constexpr int RB = GU ? kTileM : 2 * kTileM;  // weight rows per item
    constexpr int SFC = 32;                       // TMEM scale columns per stage (8-aligned)
    const int nst = p.nst, SB = p.sb;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + nst * SB);  // stage bytes landed (TMA)
    uint64_t *sfr = full + nst;                                        // stage scales in TMEM (4 warps)
    uint64_t *empty = sfr + nst;                                       // stage consumed (MMA commit)
    uint64_t *afull = empty + nst;
    uint64_t *aempty = afull + 2;
    uint64_t *mready = aempty + 2;  // the routing is in shared memory (gate/up)
    uint64_t *mdone = mready + 1;   // every MMA this CTA issued has completed
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mdone + 1);
    volatile int *s_abort = reinterpret_cast<volatile int *>(tslot + 1);
    volatile int *s_last = s_abort + 1;
    volatile int *s_U = s_last + 1;
    const uint8_t **s_blob = reinterpret_cast<const uint8_t **>(smem + nst * SB + kUBarBytes);
    int32_t *s_eid = reinterpret_cast<int32_t *>(s_blob + kMetaU);
    float *s_wu = reinterpret_cast<float *>(s_eid + kMetaU);  // [u][t]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Layout &L = p.L;
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws + L.hdr);
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
        fence_mbar_init();
        *s_abort = 0;
    }
    constexpr uint32_t kCols = 512u;
    if (warp == 0) umma::tmem_alloc(tslot, kCols);
    umma::fence_before();
    __syncthreads();
    umma::fence_after();
    const uint32_t tbase = *tslot;
    const int Tc = p.Tc, N = act_n(Tc);
    // the routing of the chunk (written by the router kernel) -> shared memory
    auto load_meta = [&](int i0, int nthr) {
        const int U = (int)*reinterpret_cast<volatile uint32_t *>(&hdr->n_unique);
        const uint8_t *const *gb = reinterpret_cast<const uint8_t *const *>(p.ws + L.uniq_blob);
        const int32_t *ge = reinterpret_cast<const int32_t *>(p.ws + L.uniq_eid);
        const uint32_t *gm = reinterpret_cast<const uint32_t *>(p.ws + L.uniq_mask);
        const int8_t *gs = reinterpret_cast<const int8_t *>(p.ws + L.uniq_slot);
        const float *gw = reinterpret_cast<const float *>(p.ws + L.wt);
        for (int i = i0; i < U; i += nthr) {
            s_blob[i] = gb[i];
            s_eid[i] = ge[i];
        }
        // pairs (expert u, token t < Tc) only (the epilogue reads no others);
        // the mask and the slot are loaded side by side, then the weight
        for (int j = i0; j < U * Tc; j += nthr) {
            const int u = j / Tc, t = j - u * Tc;
            const uint32_t m = gm[u];
            const int sl = gs[u * kChunk + t];
            s_wu[u * kChunk + t] = ((m >> t) & 1u) ? gw[t * p.k + sl] : 0.f;
        }
        return U;
    };
    if constexpr (!GU) {
        // The routing comes from the router kernel's dispatch, published by a
        // release on disp_cnt: read it without waiting for the gate/up pass,
        // so the producer can start the weight stream at once.  Everything the
        // gate/up pass writes (h pieces and scales) is read after griddepcontrol
        // .wait: by the producer after its first weight copies, by every other
        // thread here.
        pdl_trigger();
        if (threadIdx.x == 0 && !spin_geq(&hdr->disp_cnt, 1u, p.wait_ns)) {
            set_status(hdr, kStTimeout);
            *s_abort = 1;
        }
        __syncthreads();
        const int U0 = load_meta(threadIdx.x, kUThreads);
        if (threadIdx.x == 0) *s_U = U0;
        __syncthreads();
        if (threadIdx.x == 0) {
            // the last CTA to have read the dispatch resets the two counters
            // (the next router kernel starts after this grid completes)
            const uint32_t old = atom_add_acq_rel(&hdr->disp_seen, 1u);
            if (old == gridDim.x - 1) {
                hdr->disp_seen = 0u;
                hdr->disp_cnt = 0u;
            }
        }
        if (!(warp == 8 && lane == 0)) pdl_wait();
    } else {
        pdl_trigger();
        if (warp == 10) {
            pdl_wait();
            const int U0 = load_meta(lane, 32);
            if (lane == 0) *s_U = U0;
            __syncwarp();
            if (lane == 0 && p.inject != 1)
                asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(mready)) : "memory");
        }
    }
    const int K = GU ? p.d : p.ff;   // routed reduction length
    const int M = GU ? p.ff : p.d;   // routed weight rows
    const int Ks = GU ? p.d : p.ffs; // shared reduction length
    const int nkt = ceil_div(K, kTileK);
    const int nrb = ceil_div(M, RB);
    const int nkts = p.ffs > 0 ? ceil_div(Ks, kTileKs) : 0;
    const int nrbs = (GU && p.ffs > 0) ? ceil_div(p.ffs, kTileM) : 0;
    const int S = GU ? nrbs * nkts : 0;               // shared units (gate/up: the first range)
    // down: the routing is known here; gate/up: only after mready
    int U = GU ? 0 : *s_U;
    int upi = GU ? 0 : U * nkt + nkts;                // units per item (down)
    const int cta = blockIdx.x;
    // A range of units [base, base + n) split evenly over the CTAs (CTA c of
    // G takes [start(c), start(c + 1))); an item cut between CTAs is finished
    // by the last of them to arrive.
    struct Range {
        int base, n, G, a, b;
    };
    auto make_range = [&](int base, int n, int ctas) {
        Range r;
        r.base = base;
        r.n = n;
        r.G = min(ctas, max(n, 1));
        r.a = cta < r.G && n > 0 ? base + (int)(((long long)cta * n) / r.G) : base;
        r.b = cta < r.G && n > 0 ? base + (int)(((long long)(cta + 1) * n) / r.G) : base;
        return r;
    };
    auto start = [&](const Range &r, int c) { return r.base + (int)(((long long)c * r.n) / r.G); };
    auto owner = [&](const Range &r, int unit) {
        return (int)((((long long)(unit - r.base) + 1) * r.G - 1) / r.n);
    };
    // gate/up: [shared units | routed units]; down: [all units | nothing]
    // (two scalars, not an array: an array indexed by a loop counter would
    // live in local memory)
    // The gate/up shared range leaves out the last CTA: CTAs start in index
    // order as the router kernel's CTAs leave their SMs, and the last one
    // waits for the router's top-k CTA; it starts its share with the routed
    // range, which every CTA begins at the same time.
    const int G = gridDim.x;
    Range rng0 = GU ? make_range(0, S, G > 1 ? G - 1 : 1) : make_range(0, nrb * upi, G);
    Range rng1 = make_range(0, 0, G);
    auto rng = [&](int ri) { return ri == 0 ? rng0 : rng1; };
    // gate/up, before the routed range: wait for the routing (lane 0 of the
    // calling warp waits, the warp follows), then size the routed range
    auto routed_range = [&](bool warp_wide) {
        int ok = 1;
        if (lane == 0) {
            ok = (!*s_abort && mbar_wait_bounded(mready, 0u, hdr, p.wait_ns)) ? 1 : 0;
            if (!ok) *s_abort = 1;
        }
        if (warp_wide) ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) return false;
        U = *s_U;
        rng1 = make_range(S, U * nrb * nkt, G);
        return true;
    };
    const size_t mat = (size_t)p.d * p.ff;
    const uint8_t *const *ublob = s_blob;
    const uint8_t *smaps = p.ws + L.tmap + (size_t)L.E * kMapsPerExpert * 128;
    const int32_t *ueid = s_eid;
    const uint32_t idesc4 = umma::idesc_mxf4(N), idesc16 = umma::idesc_bf16(N);
    // TMEM columns: accumulators [buf][mat] at (buf*NMAT + mat)*64 (N <= 64), then
    // the scale columns of each stage from sf0
    const uint32_t sf0 = 256u;

    // Bounded wait that gives up at once after any role has given up, so a
    // failure ends the kernel in bounded time.
    auto wait = [&](uint64_t *bar, uint32_t parity) {
        if (*s_abort) return false;
        if (mbar_wait_bounded(bar, parity, hdr, p.wait_ns)) return true;
        *s_abort = 1;
        return false;
    };

    struct Unit {
        int item, u, rb, kt, istart, iend;
        bool shared;
    };
    auto decode = [&](int unit) {
        Unit x;
        if constexpr (GU) {
            if (unit < S) {
                // shared item j (counter j), K-tiles of 64 bf16
                const int j = unit / nkts;
                x.item = j;
                x.istart = j * nkts;
                x.iend = x.istart + nkts;
                x.u = -1;
                x.rb = j;
                x.shared = true;
            } else {
                // routed item (u, rb) (counter nrbs + u*nrb + rb)
                const int ir = (unit - S) / nkt;
                x.item = nrbs + ir;
                x.istart = S + ir * nkt;
                x.iend = x.istart + nkt;
                x.u = ir / nrb;
                x.rb = ir - x.u * nrb;
                x.shared = false;
            }
            x.kt = unit - x.istart;
        } else {
            x.item = unit / upi;
            x.istart = x.item * upi;
            x.iend = x.istart + upi;
            x.rb = x.item;
            const int r = unit - x.istart;
            x.shared = r >= U * nkt;
            if (!x.shared) {
                x.u = r / nkt;
                x.kt = r - x.u * nkt;
            } else {
                x.u = -1;
                x.kt = r - U * nkt;
            }
        }
        return x;
    };
    // MMA k-steps of a unit (32 bytes of every row each)
    auto ksteps = [&](const Unit &x) {
        return x.shared ? min(4, (Ks - x.kt * kTileKs) / 16) : min(4, (K - x.kt * kTileK) / 64);
    };
    // The unit after x (no divisions): next K-tile, then the next expert
    // (down), then the shared K-tiles; at the end of an item, a full decode.
    auto advance = [&](const Unit &x, int unit_next, int end) {
        Unit y = x;
        if (unit_next >= x.iend) return unit_next < end ? decode(unit_next) : x;
        ++y.kt;
        if constexpr (!GU) {
            if (!y.shared && y.kt == nkt) {
                y.kt = 0;
                if (++y.u == U) {
                    y.u = -1;
                    y.shared = true;
                }
            }
        }
        return y;
    };

    if (warp == 8) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0) {
            int last_u = -2;
            uint32_t ph = 0u;  // phase of the current pass over the stages
            int it = 0, s = 0;
            if (GU && rng0.a < rng0.b && p.route_ctas > 0) {
                // the shared units read x as bf16 and the shared tensor maps,
                // which the router kernel's CTAs publish by counting prep_done
                if (!spin_geq(&hdr->prep_done, (uint32_t)p.route_ctas, p.wait_ns)) {
                    set_status(hdr, kStTimeout);
                    *s_abort = 1;
                }
                asm volatile("fence.proxy.async.global;" ::: "memory");  // before the bulk copies read x
            }
            // The B operand (and its scale words) of a unit: activation pieces
            // written by the previous kernel of the layer.
            auto b_src = [&](const Unit &x, const uint8_t *&bsrc, const uint8_t *&sfbsrc) {
                if (x.shared) {
                    bsrc = (GU ? p.ws + L.xbf : p.ws + L.hsb) + (size_t)x.kt * N * 128;
                    sfbsrc = nullptr;
                } else {
                    bsrc = GU ? p.ws + L.xb + (size_t)x.kt * N * 128
                              : p.ws + L.hb + ((size_t)x.u * nkt + x.kt) * N * 128;
                    sfbsrc = GU ? p.ws + L.xsf + (size_t)x.kt * 2 * kSfRow * 4
                                : p.ws + L.hsf + ((size_t)x.u * nkt + x.kt) * 2 * kSfRow * 4;
                }
            };
            auto sf_dma_of = [&](const Unit &x) {
                return p.sf_tma && !x.shared && ublob[x.u] != nullptr;
            };
            // B copies of stage s (after the A copies and the stage's expect_tx)
            auto issue_b = [&](const Unit &x, int s) {
                uint8_t *st = smem + s * SB;
                const uint8_t *bsrc, *sfbsrc;
                b_src(x, bsrc, sfbsrc);
                if (sf_dma_of(x)) bulk_g2s(st + umma_sfb_off(GU, N), sfbsrc, (uint32_t)(2 * kSfRow * 4), &full[s]);
                bulk_g2s(st + NMAT * kAtile, bsrc, (uint32_t)(N * 128), &full[s]);
            };
            // down: the first two stages' weight copies go out before the wait
            // for the gate/up pass (weights need nothing from it), their B copies
            // after (more stages in flight there slow that pass's last writes)
            const int npre = GU ? 0 : min(min(nst, 2), rng0.b - rng0.a);
            for (int ri = 0; ri < 2 && !*s_abort; ++ri) {
            if (ri == 1 && (!GU || !routed_range(false))) break;
            const Range rg = rng(ri);
            Unit x = rg.a < rg.b ? decode(rg.a) : Unit{};
            for (int unit = rg.a; unit < rg.b && !*s_abort; x = advance(x, ++unit, rg.b), ++it) {
                if (it >= nst && !wait(&empty[s], ph ^ 1u)) break;
                uint8_t *st = smem + s * SB;
                const uint8_t *blob = x.shared ? nullptr : ublob[x.u];
                const uint8_t *maps = nullptr;
                const uint8_t *scmaps = nullptr;  // the A scale planes' maps (TMA scale path)
                bool ws_map = true;               // the map lives in the workspace (acquire it)
                if (x.shared) {
                    if (GU) {
                        maps = smaps;
                    } else {
                        maps = reinterpret_cast<const uint8_t *>(p.smap_d);
                        ws_map = false;
                    }
                } else {
                    const uint8_t *em = p.ws + L.tmap + (size_t)ueid[x.u] * kMapsPerExpert * 128;
                    maps = em + (GU ? 0 : 768);
                    scmaps = em + (GU ? 384 : 896);
                }
                const bool sf_dma = sf_dma_of(x);
                if (x.shared || blob != nullptr) {
                    if (x.u != last_u) {
                        if (ws_map) umma::tmap_acquire(maps);
                        if (GU) umma::tmap_acquire(maps + 128);
                        if (sf_dma) {
                            umma::tmap_acquire(scmaps);
                            if (GU) umma::tmap_acquire(scmaps + 128);
                        }
                        last_u = x.u;
                    }
                    mbar_arrive_expect_tx(&full[s], (uint32_t)(NMAT * kAtile + N * 128 +
                                                               (sf_dma ? NMAT * 2048 + 2 * kSfRow * 4 : 0)));
                    umma::tma_load_2d(st, maps, x.kt * 128, x.rb * RB, &full[s]);
                    if (GU) umma::tma_load_2d(st + kAtile, maps + 128, x.kt * 128, x.rb * RB, &full[s]);
                    if (sf_dma) {
                        // 16 scale bytes per row: this K-tile's 8 and its neighbour's
                        uint8_t *sfa = st + umma_sfa_off(GU, N);
                        umma::tma_load_2d(sfa, scmaps, (x.kt >> 1) * 16, x.rb * RB, &full[s]);
                        if (GU) umma::tma_load_2d(sfa + 2048, scmaps + 128, (x.kt >> 1) * 16, x.rb * RB, &full[s]);
                    }
                } else {
                    mbar_arrive_expect_tx(&full[s], (uint32_t)(N * 128));
                }
                if (it >= npre) issue_b(x, s);
                if (it + 1 == npre || (npre > 0 && it + 1 < npre && unit + 1 == rg.b)) {
                    // the pre-issued stages: now wait for the gate/up pass and
                    // send their B copies
                    pdl_wait();
                    hdr->prep_done = 0u;  // every gate/up CTA has read it (that grid is complete)
                    asm volatile("fence.proxy.async.global;" ::: "memory");  // before the bulk copies read h
                    Unit y = decode(rg.a);
                    for (int q = 0; q <= it; ++q, y = advance(y, rg.a + q, rg.b)) issue_b(y, q);
                }
                if (++s == nst) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            }
            if (!GU && npre == 0) {
                pdl_wait();
                hdr->prep_done = 0u;
            }
            if (*s_abort) {
                // a wait gave up somewhere: wait (bounded) for the last copy
                // issued into each stage, so none lands after the CTA's
                // shared memory is released
                for (int q = 0; q < nst && q < it; ++q) {
                    const int last = q + ((it - 1 - q) / nst) * nst;  // its last use
                    mbar_drain(&full[q], (uint32_t)((last / nst) & 1), p.wait_ns);
                }
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // --------------------------------------- scale factors -> TMEM --
        const uint32_t lb = umma::lane_base(warp);
        uint32_t nanb = 0u;  // E8M0 NaN bytes met among the weight scales (strict mode)
        if (p.sf_tma) {
            // The scales came with the stage's TMA copy: wait for the stage,
            // then move this K-tile's 8 scale bytes of each row (and the B
            // scales) into TMEM.  An expert whose blob failed its check gets
            // zero scale bytes (finite 2^-127), so it adds exactly nothing.
            uint32_t ph = 0u;
            int s = 0;
            for (int ri = 0; ri < 2; ++ri) {
            if (ri == 1 && (!GU || !routed_range(true))) break;
            const Range rg = rng(ri);
            Unit x = rg.a < rg.b ? decode(rg.a) : Unit{};
            bool go_on = true;
            for (int unit = rg.a; unit < rg.b; x = advance(x, ++unit, rg.b)) {
                int go = 0;
                if (lane == 0) go = wait(&full[s], ph);
                if (!__shfl_sync(0xffffffffu, go, 0)) {
                    go_on = false;
                    break;
                }
                if (!x.shared) {
                    const uint8_t *st = smem + s * SB;
                    const bool has = ublob[x.u] != nullptr;
                    const uint32_t col = tbase + lb + sf0 + (uint32_t)(s * SFC);
#pragma unroll
                    for (int m = 0; m < NMAT; ++m) {
                        const uint8_t *sfa = st + umma_sfa_off(GU, N) + m * 2048 + (x.kt & 1) * 8;
                        uint32_t w[8];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint2 v = has ? *reinterpret_cast<const uint2 *>(sfa + (32 * j + lane) * 16)
                                                : make_uint2(0u, 0u);
                            nanb |= e8m0_nan8(v.x, v.y);
                            w[j] = v.x;      // group 0: k-steps 0, 1
                            w[4 + j] = v.y;  // group 1: k-steps 2, 3
                        }
                        umma::st8(col + 8 * m, w);
                    }
                    const uint32_t *sb = reinterpret_cast<const uint32_t *>(st + umma_sfb_off(GU, N));
                    const uint32_t w[8] = {has ? sb[lane] : 0u,          has ? sb[32 + lane] : 0u,          0u, 0u,
                                           has ? sb[kSfRow + lane] : 0u, has ? sb[kSfRow + 32 + lane] : 0u, 0u, 0u};
                    umma::st8(col + 8 * NMAT, w);
                    umma::wait_st();
                }
                umma::fence_before();
                __syncwarp();
                if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&sfr[s])) : "memory");
                if (++s == nst) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (!go_on) break;
            }
        } else {
        // The global loads of a unit's scales are issued kLook units ahead of
        // its TMEM stores (a ring of registers), so their latency overlaps the
        // pipeline instead of adding to every stage.  Shared (bf16) units have
        // no scales: the warps only keep the stage protocol.
        constexpr int kLook = 3;
        struct SfRegs {
            uint32_t a[NMAT][8];  // column 8m + 4g + j: group g, row block j
            uint32_t b[4];        // B scales: (g0, rows 0-31), (g0, 32-63), (g1, ...), (g1, ...)
            bool on;
        };
        auto load = [&](int unit, SfRegs &r) {
            const Unit x = decode(unit);
            r.on = !x.shared;
            if (x.shared) return;
            const uint8_t *blob = ublob[x.u];
            const int nks = ksteps(x);
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
                const uint8_t *plane = nullptr;
                if (blob != nullptr)
                    plane = GU ? (m == 0 ? blob + mat / 2 : blob + mat + mat / 32) : blob + mat + mat / 16 + mat / 2;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int row = x.rb * RB + (GU ? 0 : m * kTileM) + 32 * j + lane;
                    uint2 v = make_uint2(0u, 0u);
                    if (plane != nullptr && row < M) v = load_sf8(plane + (size_t)row * (K / 32) + x.kt * 8, nks);
                    nanb |= e8m0_nan8(v.x, v.y);
                    r.a[m][j] = v.x;      // group 0: k-steps 0, 1
                    r.a[m][4 + j] = v.y;  // group 1: k-steps 2, 3
                }
            }
            const uint32_t *sfb = GU ? reinterpret_cast<const uint32_t *>(p.ws + L.xsf) + (size_t)x.kt * 2 * kSfRow
                                     : reinterpret_cast<const uint32_t *>(p.ws + L.hsf) +
                                           ((size_t)x.u * nkt + x.kt) * 2 * kSfRow;
            r.b[0] = __ldcg(sfb + lane);
            r.b[1] = __ldcg(sfb + 32 + lane);
            r.b[2] = __ldcg(sfb + kSfRow + lane);
            r.b[3] = __ldcg(sfb + kSfRow + 32 + lane);
        };
        auto store = [&](int it, const SfRegs &r) {
            const int s = it % nst;
            // lane 0 decides, the warp follows (the TMEM stores are warp-collective)
            int go = 0;
            if (lane == 0) go = it < nst ? !*s_abort : wait(&empty[s], (uint32_t)(((it / nst) + 1) & 1));
            if (!__shfl_sync(0xffffffffu, go, 0)) return false;
            if (r.on) {
                const uint32_t col = tbase + lb + sf0 + (uint32_t)(s * SFC);
#pragma unroll
                for (int m = 0; m < NMAT; ++m) umma::st8(col + 8 * m, r.a[m]);
                const uint32_t w[8] = {r.b[0], r.b[1], 0u, 0u, r.b[2], r.b[3], 0u, 0u};
                umma::st8(col + 8 * NMAT, w);
                umma::wait_st();
            }
            umma::fence_before();
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&sfr[s])) : "memory");
            return true;
        };
        SfRegs R4[kLook + 1];
        bool go = true;
        int done = 0;  // stages passed in earlier ranges
        for (int ri = 0; ri < 2 && go; ++ri) {
            if (ri == 1 && (!GU || !routed_range(true))) break;
            const Range rg = rng(ri);
            const int a = rg.a, n = rg.b - rg.a;
#pragma unroll
            for (int i = 0; i < kLook; ++i)
                if (i < n) load(a + i, R4[i]);
            for (int it0 = 0; it0 < n && go; it0 += kLook + 1) {
#pragma unroll
                for (int q = 0; q <= kLook; ++q) {
                    const int it = it0 + q;
                    if (it < n && go) {
                        if (it + kLook < n) load(a + it + kLook, R4[(q + kLook) % (kLook + 1)]);
                        go = store(done + it, R4[q]);
                    }
                }
            }
            done += n;
        }
        }
        if (p.strict && __any_sync(0xffffffffu, nanb != 0u) && lane == 0) set_status(hdr, kStDeviceCheck);
    } else if (warp == 9) {
        // ------------------------------------------------- MMA issuer --
        // One thread; everything per MMA is an add on precomputed descriptors
        // (the start-address field of a descriptor is its low 14 bits, and
        // every operand address here stays below 256 KB).
        if (lane == 0) {
            const uint64_t adesc0 = umma::smem_desc(smem_u32(smem), 16u, 1024u, umma::kLayoutSw128);
            const uint64_t bdesc0 = umma::smem_desc(smem_u32(smem) + NMAT * kAtile, (uint32_t)((N / 8) * 128), 128u,
                                                    umma::kLayoutNone);
            const uint32_t bstep = (uint32_t)(2 * (N / 8) * 128) >> 4;  // one k-step of B (2 chunks)
            const uint32_t id4[2] = {umma::idesc_sf_id(idesc4, 0u), umma::idesc_sf_id(idesc4, 2u)};
            int seg = 0, s = 0;
            uint32_t ph = 0u;
            for (int ri = 0; ri < 2 && !*s_abort; ++ri) {
            if (ri == 1 && (!GU || !routed_range(false))) break;
            const Range rg = rng(ri);
            for (int unit = rg.a; unit < rg.b && !*s_abort; ++seg) {
                Unit x = decode(unit);
                const int seg_end = min(rg.b, x.iend);
                const int buf = seg & 1;
                if (seg >= 2 && !wait(&aempty[buf], (uint32_t)(((seg >> 1) + 1) & 1))) break;
                umma::fence_after();
                const uint32_t dcol = tbase + (uint32_t)(buf * NMAT * 64);
                uint32_t acc = 0u;
                for (int un = unit; un < seg_end; x = advance(x, ++un, rg.b)) {
                    if (!wait(&full[s], ph) || !wait(&sfr[s], ph)) break;
                    umma::fence_after();
                    const uint32_t soff = (uint32_t)(s * SB) >> 4;
                    const uint64_t a0 = adesc0 + soff, b0 = bdesc0 + soff;
                    const int nks = ksteps(x);
                    if (x.shared) {
#pragma unroll
                        for (int sk = 0; sk < 4; ++sk) {
                            if (sk < nks) {
                                const uint64_t bd = b0 + sk * bstep;
                                umma::mma_bf16(dcol, a0 + 2 * sk, bd, idesc16, acc);
                                umma::mma_bf16(dcol + 64, a0 + (kAtile >> 4) + 2 * sk, bd, idesc16, acc);
                                acc = 1u;
                            }
                        }
                    } else {
                        const uint32_t sfc = tbase + sf0 + (uint32_t)(s * SFC);
#pragma unroll
                        for (int sk = 0; sk < 4; ++sk) {
                            if (sk < nks) {
                                const uint64_t bd = b0 + sk * bstep;
                                const uint32_t sfid = (uint32_t)(2 * (sk & 1)) << 30;
                                const uint32_t sfb = (sfc + 8 * NMAT + (sk >> 1) * 4) | sfid;
                                umma::mma_mxf4(dcol, a0 + 2 * sk, bd, id4[sk & 1], acc, (sfc + (sk >> 1) * 4) | sfid,
                                               sfb);
                                umma::mma_mxf4(dcol + 64, a0 + (kAtile >> 4) + 2 * sk, bd, id4[sk & 1], acc,
                                               (sfc + 8 + (sk >> 1) * 4) | sfid, sfb);
                                acc = 1u;
                            }
                        }
                    }
                    umma::commit(&empty[s]);
                    if (++s == nst) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                umma::commit(&afull[buf]);
                unit = seg_end;
            }
            }
            // the CTA frees its tensor memory only after every MMA issued here
            // has completed (on an early exit too)
            umma::commit(mdone);
            mbar_drain(mdone, 0u, p.wait_ns);
        }
    } else if (warp < 4) {
        // --------------------------------------------------- epilogue --
        const uint32_t lb = umma::lane_base(warp);
        const int rowl = 32 * warp + lane;  // row of the 128-row item
        float *spart = reinterpret_cast<float *>(p.ws + L.spart);
        uint32_t *icnt = reinterpret_cast<uint32_t *>(p.ws + L.icnt) +
                         (GU ? 0 : L.umax * ceil_div(p.ff, kTileM) + ceil_div(L.ffs, kTileM));
        int seg = 0;
        for (int ri = 0; ri < 2; ++ri) {
        if (ri == 1 && (!GU || !routed_range(true))) break;
        const Range rg = rng(ri);
        for (int unit = rg.a; unit < rg.b; ++seg) {
            const Unit x = decode(unit);
            const int item = x.item;
            const int seg_end = min(rg.b, x.iend);
            const int buf = seg & 1;
            float acc[NMAT][kChunk];
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int t = 0; t < kChunk; ++t) acc[m][t] = 0.f;
            // every epilogue warp runs the same sequence of named barriers, so
            // after a failed wait it carries on (with unused values)
            if (lane == 0) wait(&afull[buf], (uint32_t)((seg >> 1) & 1));
            __syncwarp();
            umma::fence_after();
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
#pragma unroll
                for (int n0 = 0; n0 < kNMax; n0 += 8) {
                    if (n0 < N) {
                        uint32_t r[8];
                        umma::ld8(tbase + lb + (uint32_t)((buf * NMAT + m) * 64 + n0), r);
                        umma::wait_ld();
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj) {
                            const int t = (n0 + jj) / kPieces;
                            if (t < kChunk) acc[m][t] += __uint_as_float(r[jj]);
                        }
                    }
                }
            }
            umma::fence_before();
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&aempty[buf])) : "memory");

            const bool whole = unit == x.istart && seg_end == x.iend;
            bool fin = whole;
            if (!whole) {
                const int slot = 2 * ri + (unit == rg.a ? 0 : 1);
                float *sp = spart + (size_t)((cta * 4 + slot) * 2) * kChunk * kTileM;
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
#pragma unroll
                    for (int t = 0; t < kChunk; ++t)
                        if (t < Tc) sp[(m * kChunk + t) * kTileM + rowl] = acc[m][t];
                umma::bar_sync(1, 128);
                const int c0 = owner(rg, x.istart), c1 = owner(rg, x.iend - 1);
                if (threadIdx.x == 0) {
                    const uint32_t old = atom_add_acq_rel(icnt + item, 1u);
                    const int last = old == (uint32_t)(c1 - c0);
                    if (last) icnt[item] = 0u;
                    *s_last = last;
                }
                umma::bar_sync(1, 128);
                fin = *s_last != 0;
                if (fin) {
                    // sum every piece of the item in K order
#pragma unroll
                    for (int m = 0; m < NMAT; ++m)
#pragma unroll
                        for (int t = 0; t < kChunk; ++t) acc[m][t] = 0.f;
                    for (int cc = c0; cc <= c1; ++cc) {
                        const int sl = 2 * ri + (start(rg, cc) < x.istart ? 1 : 0);
                        const float *q = spart + (size_t)((cc * 4 + sl) * 2) * kChunk * kTileM;
#pragma unroll
                        for (int m = 0; m < NMAT; ++m)
#pragma unroll
                            for (int t = 0; t < kChunk; ++t)
                                if (t < Tc) acc[m][t] += __ldcg(q + (m * kChunk + t) * kTileM + rowl);
                    }
                }
            }
            if (fin) {
                if constexpr (GU) {
                    const int f = x.rb * kTileM + rowl;  // ff (or ff_s) row of this thread
                    if (!x.shared) {
                        const uint8_t *blob = ublob[x.u];
                        const int nkt_ff = ceil_div(p.ff, kTileK);
                        const int blk = x.rb * 4 + warp;  // 32-row block of ff
                        const int kt = blk >> 3;
                        uint8_t *tile = p.ws + L.hb + ((size_t)x.u * nkt_ff + kt) * N * 128;
                        uint8_t *sfw = p.ws + L.hsf + ((size_t)x.u * nkt_ff + kt) * 2 * kSfRow * 4;
#pragma unroll
                        for (int t = 0; t < kChunk; ++t) {
                            if (t < Tc) {
                                float h = 0.f;
                                const float w = s_wu[x.u * kChunk + t];
                                if (blob != nullptr && w != 0.f && f < p.ff) h = silu_mul(acc[0][t], acc[1][t]) * w;
                                quantize_pieces(h, lane, t, blk & 7, N, tile, sfw);
                            }
                        }
                    } else if (f < p.ffs) {
                        // shared: h as bf16 hi + lo (pieces 0, 1; the others zero), weight 1
                        uint8_t *tile = p.ws + L.hsb + (size_t)(f / kTileKs) * N * 128;
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
#pragma unroll
                    for (int m = 0; m < NMAT; ++m) {
                        const int row = item * RB + m * kTileM + rowl;
                        if (row < p.d) {
#pragma unroll
                            for (int t = 0; t < kChunk; ++t) {
                                if (t < Tc) {
                                    float y = acc[m][t];
                                    if (p.resid) y += __uint_as_float((uint32_t)p.resid[(size_t)t * p.d + row] << 16);
                                    if (p.out_fp32)
                                        reinterpret_cast<float *>(p.y)[(size_t)t * p.d + row] = y;
                                    else
                                        reinterpret_cast<__nv_bfloat16 *>(p.y)[(size_t)t * p.d + row] =
                                            __float2bfloat16_rn(y);
                                }
                            }
                        }
                    }
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
}

}  // namespace k3

// Grouped-prefill expert projections on the 5th-generation tensor cores: the
// same block-scaled MMA as the decode kernel (packed E2M1 weight tiles by TMA,
// E8M0 scales in TMEM, activations as E2M1 pieces), organised for many tokens
// per expert.
//
// Items are (group of up to kGroup tokens of one expert, 128 weight rows) and
// run whole on one CTA; CTA c takes items c, c + G, c + 2G, ... of a list in
// group order with the row blocks innermost.  So at any time the CTAs work on
// a few groups of a few experts, in step (every routed item has the same
// length): a group's B tile is read by the CTAs of its row blocks at about
// the same time, and an expert's weight tiles by the CTAs of its groups, so
// most of both come from L2.  The shared expert's items (bf16 weights,
// kind::f16) follow the routed ones.
//
// Warps: 0-3 epilogue (TMEM lane quadrants), 4-7 scale factors into TMEM,
// 8 copies (TMA weight tiles, bulk copies of the group's B tile), 9 MMA issue,
// 10 loads each item's group description into a ring of shared-memory slots
// ahead of use.
#pragma once

#include "common.cuh"
#include "layout.cuh"
#include "umma.cuh"
#include "umma_kernels.cuh"

namespace k3 {

constexpr int kPfThreads = 352;
constexpr int kPfSlots = 4;  // group descriptions in flight

struct PfUmmaParams {
    int d, ff, k, ffs;
    uint8_t *ws;
    Layout L;          // decode layout: header, tensor maps
    PLayout P;         // prefill region
    int ngs;           // shared groups of this pass (0: none)
    int nst, sb;       // pipeline stages and bytes per stage
    int sf_tma;        // weight scales by TMA (reduction length a multiple of 512)
    const uint8_t *const *blobs;  // device array [E] (weight-scale loads without TMA)
    uint64_t wait_ns;  // bound of every device wait
    int strict;        // flag E8M0 NaN bytes (0xFF) among the weight scales read
};

struct PfSlot {
    int32_t eid;         // expert (-1: shared)
    int32_t g;           // group index (shared: routed groups + s)
    int32_t rb;          // 128-row block of the item
    int32_t n;           // tokens
    int32_t ok;          // the expert's blob passed its check
    int32_t pad[3];
    int32_t pair[kGroup];  // t*k + slot (shared: token)
    int32_t orow[kGroup];  // output row t*(k+1) + slot (shared: slot k)
    float w[kGroup];       // routing weight (shared: 1)
};

// One pipeline stage: the weight boxes (16 KB per matrix, 1024-byte aligned
// for the 128-byte swizzle), the B tile (kPfN rows x 128 bytes), the weight
// scale boxes (128 rows x 16 bytes per matrix) and the B scale words
// (2 groups x kPfN rows), rounded up to 1024 bytes.
__host__ __device__ inline int pf_sfa_off(bool gu) { return (gu ? 2 : 1) * kAtile + kPfN * 128; }
__host__ __device__ inline int pf_sfb_off(bool gu) { return pf_sfa_off(gu) + (gu ? 2 : 1) * 2048; }
__host__ __device__ inline int pf_stage_bytes(bool gu) { return (pf_sfb_off(gu) + 2 * kPfN * 4 + 1023) & ~1023; }
__host__ __device__ inline int pf_smem_bytes(bool gu, int nst) {
    return 1024 + nst * pf_stage_bytes(gu) + 512 + kPfSlots * (int)sizeof(PfSlot);
}

template <bool GU>
__global__ void __launch_bounds__(kPfThreads, 1) pf_expert_kernel(const __grid_constant__ PfUmmaParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    constexpr int NMAT = GU ? 2 : 1;
    // accumulators: gate/up one buffer (two matrices of kPfN columns), down two
    // buffers; then the scale columns of each stage (8-aligned groups)
    constexpr int NBUF = GU ? 1 : 2;
    constexpr int SFC = GU ? 32 : 16;
    constexpr int NS = GU ? kPfNsGU : kPfNsDn;  // MMA N of a shared item
    const int nst = p.nst, SB = p.sb;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + nst * SB);
    uint64_t *sfr = full + nst;
    uint64_t *empty = sfr + nst;
    uint64_t *afull = empty + nst;
    uint64_t *aempty = afull + 2;
    uint64_t *mfull = aempty + 2;
    uint64_t *mempty = mfull + kPfSlots;
    uint64_t *mdone = mempty + kPfSlots;  // every MMA this CTA issued has completed
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mdone + 1);
    volatile int *s_abort = reinterpret_cast<volatile int *>(tslot + 1);
    PfSlot *slots = reinterpret_cast<PfSlot *>(smem + nst * SB + 512);
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
        for (int s = 0; s < kPfSlots; ++s) {
            mbar_init(&mfull[s], 1);
            mbar_init(&mempty[s], 9);  // copies warp, 4 scale warps, 4 epilogue warps
        }
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
    pdl_wait();
    pdl_trigger();

    const int NG = (int)*reinterpret_cast<volatile uint32_t *>(&hdr->n_unique);  // routed groups
    const int K = GU ? p.d : p.ff;   // routed reduction length
    const int M = GU ? p.ff : p.d;   // weight rows
    const int Ks = GU ? p.d : p.ffs; // shared reduction length
    const int nkt = ceil_div(K, kTileK);
    const int nrb = ceil_div(M, kTileM);
    const int nkts = p.ffs > 0 ? ceil_div(Ks, kTileKs) : 0;
    const int nrbs = p.ffs > 0 ? (GU ? ceil_div(p.ffs, kTileM) : nrb) : 0;
    const int IR = NG * nrb;                 // routed items
    const int NI = IR + p.ngs * nrbs;        // all items
    const int G = gridDim.x, cta = blockIdx.x;
    const int nmine = cta < NI ? (NI - cta + G - 1) / G : 0;  // this CTA's items
    const int4 *items = reinterpret_cast<const int4 *>(p.ws + (GU ? p.P.itg : p.P.itd));
    const size_t mat = (size_t)p.d * p.ff;
    const uint8_t *smaps = p.ws + L.tmap + (size_t)L.E * kMapsPerExpert * 128;
    const uint32_t idesc4 = umma::idesc_mxf4(kPfN), idesc16 = umma::idesc_bf16(NS);
    const uint32_t sf0 = (uint32_t)(NBUF * NMAT * kPfN);
    auto item_of = [&](int q) { return cta + q * G; };
    auto nk_of = [&](int it) { return it < IR ? nkt : nkts; };
    auto wait = [&](uint64_t *bar, uint32_t parity) {
        if (*s_abort) return false;
        if (mbar_wait_bounded(bar, parity, hdr, p.wait_ns)) return true;
        *s_abort = 1;
        return false;
    };
    // the q-th item's description is in slot q % kPfSlots once mfull says so
    auto slot_wait = [&](int q) -> PfSlot * {
        int go = 0;
        if (lane == 0) go = wait(&mfull[q % kPfSlots], (uint32_t)((q / kPfSlots) & 1));
        go = __shfl_sync(0xffffffffu, go, 0);
        return go ? &slots[q % kPfSlots] : nullptr;
    };
    auto slot_done = [&](int q) {
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&mempty[q % kPfSlots])) : "memory");
    };

    if (warp == 10) {
        // ---------------------------------------------- group descriptions --
        // Two items in flight: the record of item q+2 and the pairs of item
        // q+1 load while item q's slot is written.
        const int32_t *perm = reinterpret_cast<const int32_t *>(p.ws + p.P.perm);
        const float *pw = reinterpret_cast<const float *>(p.ws + p.P.pw);
        auto pairs_of = [&](const int4 &rec, int &pid, float &w) {
            const int n = rec.w & 255;
            pid = 0;
            w = 0.f;
            if (lane < n) {
                if (rec.y >= 0) {
                    pid = __ldcg(perm + rec.z + lane);
                    w = __ldcg(pw + rec.z + lane);
                } else {
                    pid = rec.z + lane;
                    w = 1.f;
                }
            }
        };
        int4 r1 = make_int4(0, 0, 0, 0), r2 = make_int4(0, 0, 0, 0);
        int pid1 = 0;
        float w1 = 0.f;
        if (nmine > 0) r1 = __ldcg(items + item_of(0));
        if (nmine > 1) r2 = __ldcg(items + item_of(1));
        if (nmine > 0) pairs_of(r1, pid1, w1);
        for (int q = 0; q < nmine; ++q) {
            const int4 rec = r1;
            const int pid = pid1;
            const float w = w1;
            r1 = r2;
            if (q + 2 < nmine) r2 = __ldcg(items + item_of(q + 2));
            if (q + 1 < nmine) pairs_of(r1, pid1, w1);
            int go = 1;
            if (lane == 0 && q >= kPfSlots) go = wait(&mempty[q % kPfSlots], (uint32_t)(((q / kPfSlots) + 1) & 1));
            if (!__shfl_sync(0xffffffffu, go, 0)) break;
            PfSlot &sl = slots[q % kPfSlots];
            sl.pair[lane] = pid;
            sl.orow[lane] = rec.y >= 0 ? pid + pid / p.k : pid * (p.k + 1) + p.k;
            sl.w[lane] = w;
            if (lane == 0) {
                sl.eid = rec.y;
                sl.g = rec.x & 0xFFFFF;
                sl.rb = rec.x >> 20;
                sl.n = rec.w & 255;
                sl.ok = rec.w >> 8;
            }
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&mfull[q % kPfSlots])) : "memory");
        }
    } else if (warp == 8) {
        // ------------------------------------------------------- copies --
        int s = 0, it_stage = 0;
        uint32_t ph = 0u;
        for (int q = 0; q < nmine && !*s_abort; ++q) {
            const PfSlot *sl = slot_wait(q);
            if (!sl) break;
            const int it = item_of(q);
            const bool shared = it >= IR;
            const int n = sl->n, rb = sl->rb, g = sl->g;
            const bool ok = sl->ok != 0;
            const bool sf_dma = p.sf_tma && !shared && ok;
            const uint8_t *maps, *scmaps = nullptr;
            if (shared) {
                maps = smaps + (GU ? 0 : 256);
            } else {
                const uint8_t *em = p.ws + L.tmap + (size_t)sl->eid * kMapsPerExpert * 128;
                maps = em + (GU ? 0 : 256);
                scmaps = em + (GU ? 384 : 640);
            }
            if (lane == 0 && (shared || ok)) {
                umma::tmap_acquire(maps);
                if (GU) umma::tmap_acquire(maps + 128);
                if (sf_dma) {
                    umma::tmap_acquire(scmaps);
                    if (GU) umma::tmap_acquire(scmaps + 128);
                }
            }
            const int nk = nk_of(it);
            for (int kt = 0; kt < nk; ++kt, ++it_stage) {
                int go = 1;
                if (lane == 0 && it_stage >= nst) go = wait(&empty[s], ph ^ 1u);
                if (!__shfl_sync(0xffffffffu, go, 0)) break;
                uint8_t *st = smem + s * SB;
                uint8_t *bdst = st + NMAT * kAtile;
                uint8_t *sfb = st + pf_sfb_off(GU);
                if (lane == 0) {
                    uint32_t tx;
                    if (shared) {
                        tx = (uint32_t)(NMAT * kAtile + NS * 128);
                    } else {
                        tx = (uint32_t)(kPfN * 128 + 2 * kPfN * 4);
                    }
                    if (!shared && ok) tx += (uint32_t)(NMAT * kAtile + (sf_dma ? NMAT * 2048 : 0));
                    mbar_arrive_expect_tx(&full[s], tx);
                    if (shared || ok) {
                        umma::tma_load_2d(st, maps, kt * 128, rb * kTileM, &full[s]);
                        if (GU) umma::tma_load_2d(st + kAtile, maps + 128, kt * 128, rb * kTileM, &full[s]);
                    }
                    if (sf_dma) {
                        uint8_t *sfa = st + pf_sfa_off(GU);
                        umma::tma_load_2d(sfa, scmaps, (kt >> 1) * 16, rb * kTileM, &full[s]);
                        if (GU) umma::tma_load_2d(sfa + 2048, scmaps + 128, (kt >> 1) * 16, rb * kTileM, &full[s]);
                    }
                    if (shared) {
                        const size_t off = (GU ? p.P.xbf : p.P.hsb) + ((size_t)(g - NG) * nkts + kt) * NS * 128;
                        bulk_g2s(bdst, p.ws + off, (uint32_t)(NS * 128), &full[s]);
                    } else {
                        // the group's B tile (x pieces for gate/up, w*h pieces for down)
                        const size_t blk = (size_t)g * nkt + kt;
                        bulk_g2s(bdst, p.ws + (GU ? p.P.xg : p.P.hb) + blk * kPfN * 128, (uint32_t)(kPfN * 128), &full[s]);
                        bulk_g2s(sfb, p.ws + (GU ? p.P.xgs : p.P.hsf) + blk * 2 * kPfN * 4, (uint32_t)(2 * kPfN * 4),
                                 &full[s]);
                    }
                }
                if (++s == nst) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            slot_done(q);
        }
        if (*s_abort && lane == 0) {
            // wait (bounded) for the last copy issued into each stage, so none
            // lands after the CTA's shared memory is released
            for (int q = 0; q < nst && q < it_stage; ++q) {
                const int last = q + ((it_stage - 1 - q) / nst) * nst;
                mbar_drain(&full[q], (uint32_t)((last / nst) & 1), p.wait_ns);
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // --------------------------------------- scale factors -> TMEM --
        const uint32_t lb = umma::lane_base(warp);
        int s = 0;
        uint32_t ph = 0u;
        uint32_t nanb = 0u;  // E8M0 NaN bytes met among the weight scales (strict mode)
        for (int q = 0; q < nmine; ++q) {
            const PfSlot *sl = slot_wait(q);
            if (!sl) break;
            const int it = item_of(q);
            const bool shared = it >= IR;
            const bool ok = sl->ok != 0;
            const int rb = sl->rb;
            const uint8_t *blob = (!shared && ok && !p.sf_tma) ? p.blobs[sl->eid] : nullptr;
            const int nk = nk_of(it);
            bool go = true;
            for (int kt = 0; kt < nk; ++kt) {
                int w0 = 0;
                if (lane == 0) w0 = wait(&full[s], ph);
                if (!__shfl_sync(0xffffffffu, w0, 0)) {
                    go = false;
                    break;
                }
                if (!shared) {
                    const uint8_t *st = smem + s * SB;
                    const uint32_t col = tbase + lb + sf0 + (uint32_t)(s * SFC);
#pragma unroll
                    for (int m = 0; m < NMAT; ++m) {
                        uint32_t w[8];
                        if (p.sf_tma) {
                            const uint8_t *sfa = st + pf_sfa_off(GU) + m * 2048 + (kt & 1) * 8;
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const uint2 v = ok ? *reinterpret_cast<const uint2 *>(sfa + (32 * j + lane) * 16)
                                                   : make_uint2(0u, 0u);
                                nanb |= e8m0_nan8(v.x, v.y);
                                w[j] = v.x;
                                w[4 + j] = v.y;
                            }
                        } else {
                            const uint8_t *plane = nullptr;
                            if (blob != nullptr)
                                plane = GU ? (m == 0 ? blob + mat / 2 : blob + mat + mat / 32)
                                           : blob + mat + mat / 16 + mat / 2;
                            const int nks = min(4, (K - kt * kTileK) / 64);
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const int row = rb * kTileM + 32 * j + lane;
                                uint2 v = make_uint2(0u, 0u);
                                if (plane != nullptr && row < M) v = load_sf8(plane + (size_t)row * (K / 32) + kt * 8, nks);
                                nanb |= e8m0_nan8(v.x, v.y);
                                w[j] = v.x;
                                w[4 + j] = v.y;
                            }
                        }
                        umma::st8(col + 8 * m, w);
                    }
                    // B scales: column 4g + n/32, lane n%32
                    const uint32_t *sb = reinterpret_cast<const uint32_t *>(st + pf_sfb_off(GU));
                    const uint32_t w[8] = {sb[lane],        sb[32 + lane],        sb[64 + lane],        sb[96 + lane],
                                           sb[kPfN + lane], sb[kPfN + 32 + lane], sb[kPfN + 64 + lane], sb[kPfN + 96 + lane]};
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
            slot_done(q);
            if (!go) break;
        }
        if (p.strict && __any_sync(0xffffffffu, nanb != 0u) && lane == 0) set_status(hdr, kStDeviceCheck);
    } else if (warp == 9) {
        // ------------------------------------------------- MMA issuer --
        if (lane == 0) {
            const uint32_t bbase = smem_u32(smem) + NMAT * kAtile;
            const uint64_t adesc0 = umma::smem_desc(smem_u32(smem), 16u, 1024u, umma::kLayoutSw128);
            const uint64_t bdesc0 = umma::smem_desc(bbase, (uint32_t)((kPfN / 8) * 128), 128u, umma::kLayoutNone);
            const uint32_t bstep = (uint32_t)(2 * (kPfN / 8) * 128) >> 4;
            const uint64_t bdesc0s = umma::smem_desc(bbase, (uint32_t)((NS / 8) * 128), 128u, umma::kLayoutNone);
            const uint32_t bsteps = (uint32_t)(2 * (NS / 8) * 128) >> 4;
            const uint32_t id4[2] = {umma::idesc_sf_id(idesc4, 0u), umma::idesc_sf_id(idesc4, 2u)};
            int s = 0;
            uint32_t ph = 0u;
            for (int q = 0; q < nmine && !*s_abort; ++q) {
                const int it = item_of(q);
                const bool shared = it >= IR;
                const int buf = q % NBUF;
                if (q >= NBUF && !wait(&aempty[buf], (uint32_t)(((q / NBUF) + 1) & 1))) break;
                umma::fence_after();
                const uint32_t dcol = tbase + (uint32_t)(buf * NMAT * kPfN);
                uint32_t acc = 0u;
                const int nk = nk_of(it);
                bool go = true;
                for (int kt = 0; kt < nk; ++kt) {
                    if (!wait(&full[s], ph) || !wait(&sfr[s], ph)) {
                        go = false;
                        break;
                    }
                    umma::fence_after();
                    const uint32_t soff = (uint32_t)(s * SB) >> 4;
                    const uint64_t a0 = adesc0 + soff;
                    if (shared) {
                        const uint64_t b0 = bdesc0s + soff;
                        const int nks = min(4, (Ks - kt * kTileKs) / 16);
#pragma unroll
                        for (int sk = 0; sk < 4; ++sk) {
                            if (sk < nks) {
                                const uint64_t bd = b0 + sk * bsteps;
                                umma::mma_bf16(dcol, a0 + 2 * sk, bd, idesc16, acc);
                                if (GU) umma::mma_bf16(dcol + kPfN, a0 + (kAtile >> 4) + 2 * sk, bd, idesc16, acc);
                                acc = 1u;
                            }
                        }
                    } else {
                        const uint64_t b0 = bdesc0 + soff;
                        const int nks = min(4, (K - kt * kTileK) / 64);
                        const uint32_t sfc = tbase + sf0 + (uint32_t)(s * SFC);
#pragma unroll
                        for (int sk = 0; sk < 4; ++sk) {
                            if (sk < nks) {
                                const uint64_t bd = b0 + sk * bstep;
                                const uint32_t sfid = (uint32_t)(2 * (sk & 1)) << 30;
                                const uint32_t sfb = (sfc + 8 * NMAT + (sk >> 1) * 4) | sfid;
                                umma::mma_mxf4(dcol, a0 + 2 * sk, bd, id4[sk & 1], acc, (sfc + (sk >> 1) * 4) | sfid, sfb);
                                if (GU)
                                    umma::mma_mxf4(dcol + kPfN, a0 + (kAtile >> 4) + 2 * sk, bd, id4[sk & 1], acc,
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
                if (!go) break;
            }
            // the CTA frees its tensor memory only after every MMA issued here
            // has completed (on an early exit too)
            umma::commit(mdone);
            mbar_drain(mdone, 0u, p.wait_ns);
        }
    } else {
        // --------------------------------------------------- epilogue --
        const uint32_t lb = umma::lane_base(warp);
        const int rowl = 32 * warp + lane;
        for (int q = 0; q < nmine; ++q) {
            const PfSlot *sl = slot_wait(q);
            if (!sl) break;
            const int it = item_of(q);
            const bool shared = it >= IR;
            const int buf = q % NBUF;
            const int n = sl->n, rb = sl->rb;
            const bool ok = sl->ok != 0;
            int go = 0;
            if (lane == 0) go = wait(&afull[buf], (uint32_t)((q / NBUF) & 1));
            go = __shfl_sync(0xffffffffu, go, 0);
            umma::fence_after();
            float acc[NMAT][kGroup];
            if (!shared) {
                // token j: the sum of its kPfPieces columns 4j..4j+3 (32 columns
                // per TMEM load, one wait per load)
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
#pragma unroll
                    for (int c32 = 0; c32 < kPfN / 32; ++c32) {
                        uint32_t r[32];
                        umma::ld32(tbase + lb + (uint32_t)((buf * NMAT + m) * kPfN + 32 * c32), r);
                        umma::wait_ld();
#pragma unroll
                        for (int t = 0; t < 8; ++t)
                            acc[m][8 * c32 + t] = (__uint_as_float(r[4 * t]) + __uint_as_float(r[4 * t + 1])) +
                                                  (__uint_as_float(r[4 * t + 2]) + __uint_as_float(r[4 * t + 3]));
                    }
                }
            } else {
                // gate/up: column j (x of token j); down: column j (h high) + 32 + j (h low)
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    uint32_t r[32];
                    umma::ld32(tbase + lb + (uint32_t)((buf * NMAT + m) * kPfN), r);
                    umma::wait_ld();
#pragma unroll
                    for (int jj = 0; jj < kGroup; ++jj) acc[m][jj] = __uint_as_float(r[jj]);
                    if (!GU) {
                        umma::ld32(tbase + lb + (uint32_t)((buf * NMAT + m) * kPfN + kGroup), r);
                        umma::wait_ld();
#pragma unroll
                        for (int jj = 0; jj < kGroup; ++jj) acc[m][jj] += __uint_as_float(r[jj]);
                    }
                }
            }
            umma::fence_before();
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&aempty[buf])) : "memory");
            if (go) {
                if constexpr (GU) {
                    const int f = rb * kTileM + rowl;  // ff (or ff_s) row of this thread
                    if (!shared) {
                        // w*h of the group's tokens -> the group's down B operand
                        const int nkt_ff = ceil_div(p.ff, kTileK);
                        const int blk = rb * 4 + warp;  // 32-row block of ff
                        const size_t tb = (size_t)sl->g * nkt_ff + (blk >> 3);
                        uint8_t *tile = p.ws + p.P.hb + tb * kPfN * 128;
                        uint8_t *sfw = p.ws + p.P.hsf + tb * 2 * kPfN * 4;
                        // 4 tokens at a time (absent tokens' rows get zeros; nothing reads them)
#pragma unroll
                        for (int j0 = 0; j0 < kGroup; j0 += 4) {
                            if (j0 < n) {
                                float h[4];
#pragma unroll
                                for (int b = 0; b < 4; ++b) {
                                    const int j = j0 + b;
                                    h[b] = (ok && f < p.ff && j < n) ? silu_mul(acc[0][j], acc[1][j]) * sl->w[j] : 0.f;
                                }
                                quantize_pieces_batch<kPfPieces, 4>(h, lane, j0, blk & 7, (kPfN / 8) * 128, 128, kPfN,
                                                                    tile, sfw);
                            }
                        }
                    } else if (f < p.ffs) {
                        // shared: h as bf16 high (row j) + low (row 32 + j), weight 1
                        const int gs = sl->g - NG;
                        const int nkts_ff = ceil_div(p.ffs, kTileKs);
                        uint8_t *tile = p.ws + p.P.hsb + ((size_t)gs * nkts_ff + f / kTileKs) * kPfNsDn * 128;
                        const int c = (f % kTileKs) / 8, e = f % 8;
#pragma unroll
                        for (int j = 0; j < kGroup; ++j) {
                            if (j < n) {
                                const float h = silu_mul(acc[0][j], acc[1][j]);
                                const __nv_bfloat16 hi = __float2bfloat16_rn(h);
                                const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
                                const int nh = j, nl = kGroup + j;
                                uint8_t *base = tile + c * (kPfNsDn / 8) * 128 + e * 2;
                                *reinterpret_cast<__nv_bfloat16 *>(base + (nh / 8) * 128 + (nh % 8) * 16) = hi;
                                *reinterpret_cast<__nv_bfloat16 *>(base + (nl / 8) * 128 + (nl % 8) * 16) = lo;
                            }
                        }
                    }
                } else {
                    // down: this item's rows of o[token][slot] (slot k: the shared expert)
                    const int row = rb * kTileM + rowl;
                    if (row < p.d) {
                        float *o = reinterpret_cast<float *>(p.ws + p.P.o);
#pragma unroll
                        for (int j = 0; j < kGroup; ++j) {
                            if (j < n) {
                                o[(size_t)sl->orow[j] * p.d + row] = acc[0][j];
                            }
                        }
                    }
                }
            }
            slot_done(q);
            if (!go) break;
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

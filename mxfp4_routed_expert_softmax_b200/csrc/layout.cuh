// Workspace layout of one token chunk (up to kChunk tokens) of the layer.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace k3 {

constexpr int kChunk = 8;   // tokens per decode pass
constexpr int kMaxSeg = 8;  // most warps that share one router/shared row

// Tensor-core path: each activation element enters the MMA as kPieces E2M1
// values with their own per-32 E8M0 scales; B-operand row n = t*kPieces + p.
constexpr int kPieces = 6;
constexpr int kNMax = kChunk * kPieces;  // 48: widest MMA N of a chunk
constexpr int kSfRow = 64;               // scale words per (K-tile, group): rows n < 64
constexpr int kTileK = 256;              // MXFP4 weights per K-tile (128 bytes of nibbles per row)
constexpr int kTileKs = 64;              // bf16 weights per K-tile (128 bytes per row)
constexpr int kTileM = 128;              // MMA M: weight rows per item
constexpr int kMaxCtas = 256;            // grid cap of the tensor-core kernels
// MMA N of a chunk: a multiple of 16 (kind::f16 with M = 128 needs it)
__host__ __device__ inline int act_n(int Tc) { return (Tc * kPieces + 15) & ~15; }
__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

struct Layout {
    size_t hdr;        // WsHeader
    size_t logits;     // f32 [kChunk][E]
    size_t idx;        // i32 [kChunk][k]
    size_t wt;         // f32 [kChunk][k]
    size_t uniq_blob;  // u64 [kChunk*k]    blob pointer of each distinct selected expert
    size_t uniq_eid;   // i32 [kChunk*k]    its expert id (index of its tensor maps)
    size_t uniq_mask;  // u32 [kChunk*k]    tokens (bit t) that selected it
    size_t uniq_slot;  // i8  [kChunk*k][kChunk] slot j of token t for it, -1 if none
    size_t part;       // f32 [2][E][kMaxSeg][4] partial sums of router rows split between warps
    size_t cnt;        // u32 [2][E] arrivals per split row (back to 0 after each row)
    size_t tmap;       // 128-byte tensor maps [E][6]: W_g, W_u, W_d nibble planes and their
                       // scale planes, of each expert; then the shared expert's W_g, W_u,
                       // W_d (bf16) at [E*6 ..]
    size_t tcache;     // u64 [E+3] the blob (and shared-expert) pointers the maps were written for
    size_t xb;         // u8  [nkt_d][N*128] E2M1 pieces of x (gate/up B operand)
    size_t xsf;        // u32 [nkt_d][2][kSfRow] their E8M0 scales (byte = block in group)
    size_t hb;         // u8  [umax][nkt_ff][N*128] pieces of w*h (down B operand)
    size_t hsf;        // u32 [umax][nkt_ff][2][kSfRow]
    size_t xbf;        // u8  [ceil(d/64)][N*128] x as bf16 (rows t*kPieces), shared gate/up B
    size_t hsb;        // u8  [ceil(ffs/64)][N*128] shared h as bf16 hi, lo (rows t*kPieces, +1)
    size_t spart;      // f32 [kMaxCtas][2][2][kChunk][kTileM] split-item partial sums
    size_t icnt;       // u32 [umax*nrb_ff + nrb_ffs + nrb_d] arrivals per split item (back to 0)
    size_t total;
    int d, ff, E, k, ffs, umax;
};

__host__ __device__ inline Layout make_layout(int d, int ff, int E, int k, int ffs) {
    Layout L;
    L.d = d;
    L.ff = ff;
    L.E = E;
    L.k = k;
    L.ffs = ffs;
    const size_t C = kChunk;
    size_t o = 0;
    L.hdr = o;
    o = align256(o + 256);
    L.logits = o;
    o = align256(o + C * E * 4);
    L.idx = o;
    o = align256(o + C * k * 4);
    L.wt = o;
    o = align256(o + C * k * 4);
    L.uniq_blob = o;
    o = align256(o + C * k * 8);
    L.uniq_eid = o;
    o = align256(o + C * k * 4);
    L.uniq_mask = o;
    o = align256(o + C * k * 4);
    L.uniq_slot = o;
    o = align256(o + C * k * C);
    L.part = o;
    o = align256(o + (size_t)2 * E * kMaxSeg * 4 * 4);
    L.cnt = o;
    o = align256(o + (size_t)2 * E * 4);
    const int umax = E < kChunk * k ? E : kChunk * k;
    const int nkt_d = ceil_div(d, kTileK), nkt_ff = ceil_div(ff, kTileK);
    L.umax = umax;
    L.tmap = o;
    o = align256(o + ((size_t)E * 6 + 3) * 128);
    L.tcache = o;
    o = align256(o + ((size_t)E + 3) * 8);
    L.xb = o;
    o = align256(o + (size_t)nkt_d * kNMax * 128);
    L.xsf = o;
    o = align256(o + (size_t)nkt_d * 2 * kSfRow * 4);
    L.hb = o;
    o = align256(o + (size_t)umax * nkt_ff * kNMax * 128);
    L.hsf = o;
    o = align256(o + (size_t)umax * nkt_ff * 2 * kSfRow * 4);
    L.xbf = o;
    o = align256(o + (size_t)ceil_div(d, kTileKs) * kNMax * 128);
    L.hsb = o;
    o = align256(o + (size_t)(ffs > 0 ? ceil_div(ffs, kTileKs) : 1) * kNMax * 128);
    L.spart = o;
    o = align256(o + (size_t)kMaxCtas * 2 * 2 * kChunk * kTileM * 4);
    L.icnt = o;
    o = align256(o + ((size_t)umax * ceil_div(ff, kTileM) + ceil_div(ffs, kTileM) + ceil_div(d, kTileM)) * 4);
    L.total = o;
    return L;
}

// ---------------------------------------------------------------- prefill --
// Grouped prefill (more than kChunk tokens): the pairs (token, slot) are
// sorted by expert, each expert's pairs cut into groups of up to kGroup
// tokens; a tensor-core item is (group, 128 weight rows), so each expert's
// weights stream once per call while its groups run side by side.  The
// shared expert takes groups of kGroup consecutive tokens.  Activations enter
// as kPfPieces E2M1 pieces per element: token j of a group owns B rows
// 8j..8j+7, one 1024-byte block per K-tile ([16-byte chunk c][piece][16 B]),
// so a token's block of a K-tile is one contiguous copy.
constexpr int kGroup = 8;       // tokens per group
constexpr int kPfPieces = 8;    // pieces per activation element (rows per token)
constexpr int kPfN = kGroup * kPfPieces;  // 64: MMA N of a routed group
constexpr int kPfNs = 16;       // MMA N of a shared-expert group (bf16 rows 0-7, 8-15)
constexpr int kPfMetaG = 160;   // groups one CTA's share of a pass may touch (shared memory)
constexpr int kPfMaxTokens = 8192;  // tokens per prefill pass
constexpr int kPfHistTok = 16;  // tokens per block of the dispatch histogram

struct PLayout {
    size_t lg;     // f32 [Tp][E] router logits
    size_t idx;    // i32 [Tp][k]
    size_t wt;     // f32 [Tp][k]
    size_t hist;   // u32 [nhb][E] picks per (16-token block, expert), then their exclusive
                   // prefix over blocks
    size_t ecnt;   // u32 [E] pairs per expert
    size_t eoff;   // u32 [E] first position of each expert in perm
    size_t goff;   // u32 [E] first group of each expert
    size_t perm;   // i32 [Tp*k] pair ids t*k+j sorted by (expert, token)
    size_t grp;    // int4 [ngmax] routed groups then shared groups: (expert or -1, first
                   // position / first token, tokens, blob ok)
    size_t xp;     // u8 [Tp][nkt_d][1024] pieces of x, one block per (token, K-tile)
    size_t xps;    // u8 [Tp][nkt_d][2][8][4] their scales ([group of 4 blocks][piece][block])
    size_t xbf;    // u8 [ngs][nkts_d][kPfNs*128] x as bf16 per shared group (rows 0-7)
    size_t hb;     // u8 [ngr][nkt_ff][kPfN*128] w*h pieces per routed group (down B)
    size_t hsf;    // u32 [ngr][nkt_ff][2][kSfRow]
    size_t hsb;    // u8 [ngs][nkts_ff][kPfNs*128] shared h as bf16 hi (rows 0-7), lo (8-15)
    size_t o;      // f32 [Tp][k+1][d] expert outputs per (token, slot); slot k: shared
    size_t icnt;   // u32 [gate/up items + down items] arrivals per split item (back to 0)
    size_t total;  // end offset (absolute: the prefill region follows the decode layout)
    int Tp, ngr, ngs, nhb;
};

__host__ __device__ inline int pf_routed_groups_max(int Tp, int E, int k) {
    const int pairs = Tp * k;
    return pairs / kGroup + (E < pairs ? E : pairs);
}

__host__ __device__ inline PLayout make_playout(size_t base, int d, int ff, int E, int k, int ffs, int Tp) {
    PLayout P;
    P.Tp = Tp;
    P.ngr = pf_routed_groups_max(Tp, E, k);
    P.ngs = ffs > 0 ? ceil_div(Tp, kGroup) : 0;
    P.nhb = ceil_div(Tp, kPfHistTok);
    const int nkt_d = ceil_div(d, kTileK), nkt_ff = ceil_div(ff, kTileK);
    const int nkts_d = ceil_div(d, kTileKs), nkts_ff = ffs > 0 ? ceil_div(ffs, kTileKs) : 0;
    size_t o = align256(base);
    P.lg = o;
    o = align256(o + (size_t)Tp * E * 4);
    P.idx = o;
    o = align256(o + (size_t)Tp * k * 4);
    P.wt = o;
    o = align256(o + (size_t)Tp * k * 4);
    P.hist = o;
    o = align256(o + (size_t)P.nhb * E * 4);
    P.ecnt = o;
    o = align256(o + (size_t)E * 4);
    P.eoff = o;
    o = align256(o + (size_t)E * 4);
    P.goff = o;
    o = align256(o + (size_t)E * 4);
    P.perm = o;
    o = align256(o + (size_t)Tp * k * 4);
    P.grp = o;
    o = align256(o + (size_t)(P.ngr + P.ngs) * 16);
    P.xp = o;
    o = align256(o + (size_t)Tp * nkt_d * 1024);
    P.xps = o;
    o = align256(o + (size_t)Tp * nkt_d * 64);
    P.xbf = o;
    o = align256(o + (size_t)P.ngs * nkts_d * kPfNs * 128);
    P.hb = o;
    o = align256(o + (size_t)P.ngr * nkt_ff * kPfN * 128);
    P.hsf = o;
    o = align256(o + (size_t)P.ngr * nkt_ff * 2 * kSfRow * 4);
    P.hsb = o;
    o = align256(o + (size_t)P.ngs * nkts_ff * kPfNs * 128);
    P.o = o;
    o = align256(o + (size_t)Tp * (k + 1) * d * 4);
    P.icnt = o;
    const size_t items = (size_t)P.ngr * ceil_div(ff, kTileM) + (size_t)P.ngs * (ffs > 0 ? ceil_div(ffs, kTileM) : 0) +
                         (size_t)(P.ngr + P.ngs) * ceil_div(d, kTileM);
    o = align256(o + items * 4);
    P.total = o;
    return P;
}

}  // namespace k3

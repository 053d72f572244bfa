// Workspace layout of one token chunk (up to kChunk tokens) of the layer.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace k3 {

constexpr int kChunk = 8;   // tokens per decode pass

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
    size_t part;       // f32 [2][E][P][4] partial sums of the P parts of each router row
    size_t cnt;        // u32 [2][E] parts summed per router row (back to 0 after each row)
    size_t xn;         // bf16 [kChunk][d] the normalised input of pre-norm calls
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
    size_t spart;      // f32 [kMaxCtas][4][2][kChunk][kTileM] split-item partial sums (2 unit
                       // ranges x first/last item of a CTA)
    size_t icnt;       // u32 [umax*nrb_ff + nrb_ffs + nrb_d] arrivals per split item (back to 0)
    size_t total;
    int d, ff, E, k, ffs, umax;
};

// The decode router sums a row of d floats as d / Ls parts of Ls floats
// (Ls = 512 where d allows it; d is a multiple of 64).
__host__ __device__ inline int router_part_len(int d) {
    return d % 512 == 0 ? 512 : d % 256 == 0 ? 256 : d % 128 == 0 ? 128 : 64;
}

// Tensor maps in the workspace: per expert W_g, W_u, W_d nibble planes and
// their scale planes (128-row boxes), then W_d's nibble and scale planes again
// with 256-row boxes (the decode down pass); after all experts the shared
// expert's W_g, W_u, W_d (128-row boxes) and W_d (256-row boxes).
constexpr int kMapsPerExpert = 8;
constexpr int kSharedMaps = 4;

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
    o = align256(o + (size_t)2 * E * (d / router_part_len(d)) * 4 * 4);
    L.cnt = o;
    o = align256(o + (size_t)2 * E * 4);
    L.xn = o;
    o = align256(o + C * d * 2);
    const int umax = E < kChunk * k ? E : kChunk * k;
    const int nkt_d = ceil_div(d, kTileK), nkt_ff = ceil_div(ff, kTileK);
    L.umax = umax;
    L.tmap = o;
    o = align256(o + ((size_t)E * kMapsPerExpert + kSharedMaps) * 128);
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
    o = align256(o + (size_t)kMaxCtas * 4 * 2 * kChunk * kTileM * 4);
    L.icnt = o;
    o = align256(o + ((size_t)umax * ceil_div(ff, kTileM) + ceil_div(ffs, kTileM) + ceil_div(d, kTileM)) * 4);
    L.total = o;
    return L;
}

// ---------------------------------------------------------------- prefill --
// Grouped prefill (more than kChunk tokens): the pairs (token, slot) are
// sorted by expert and each expert's pairs cut into groups of up to kGroup
// tokens; a tensor-core item is (group, 128 weight rows).  Items run in group
// order, row blocks innermost, dealt round-robin to the CTAs: the CTAs that
// run side by side share the groups' B tiles and the experts' weight tiles
// through L2.  The shared expert takes groups of kGroup consecutive tokens.
// Activations enter as kPfPieces E2M1 pieces per element (B rows 4j..4j+3 for
// token j of a group); each group's B operand is written once per call, in
// the MMA's layout, by the pass that quantises x.
constexpr int kGroup = 32;      // tokens per group
constexpr int kPfPieces = 4;    // pieces per activation element (rows per token)
constexpr int kPfN = kGroup * kPfPieces;  // 128: MMA N of a routed group
constexpr int kPfNsGU = kGroup;           // 32: shared gate/up (x as bf16, one row per token)
constexpr int kPfNsDn = 2 * kGroup;       // 64: shared down (h as bf16 high rows, then low rows)
constexpr int kPfMaxTokens = 8192;        // tokens per prefill pass
constexpr int kPfHistTok = 16;            // tokens per block of the dispatch histogram

struct PLayout {
    size_t lg;     // f32 [Tp][E] router logits (or the router's split-K partials: see o)
    size_t idx;    // i32 [Tp][k]
    size_t wt;     // f32 [Tp][k]
    size_t hist;   // u32 [nhb][E] picks per (16-token block, expert), then their exclusive
                   // prefix over blocks
    size_t ecnt;   // u32 [E] pairs per expert
    size_t eoff;   // u32 [E] first position of each expert in perm
    size_t goff;   // u32 [E] first group of each expert
    size_t perm;   // i32 [Tp*k] pair ids t*k+j sorted by (expert, token)
    size_t pw;     // f32 [Tp*k] their routing weights, in the same order
    size_t grp;    // int4 [ngr + ngs] routed groups then shared groups: (expert or -1,
                   // first position / first token, tokens, blob ok)
    size_t itg;    // int4 [ngr*nrb_ff + ngs*nrbs_ff] gate/up items in run order: (group | rb << 20,
                   // expert or -1, first position / first token, tokens | blob ok << 8)
    size_t itd;    // int4 [(ngr + ngs)*nrb_d] down items in run order
    size_t ploc;   // i32 [Tp*k] group * kGroup + slot in the group of each pair t*k+j
    size_t xg;     // u8 [ngr][nkt_d][kPfN*128] pieces of x per routed group (gate/up B)
    size_t xgs;    // u32 [ngr][nkt_d][2][kPfN] their scales (word = 4 blocks of one row)
    size_t xbf;    // u8 [ngs][nkts_d][kPfNsGU*128] x as bf16 per shared group
    size_t hb;     // u8 [ngr][nkt_ff][kPfN*128] w*h pieces per routed group (down B)
    size_t hsf;    // u32 [ngr][nkt_ff][2][kPfN] their scales (word = 4 blocks of one row)
    size_t hsb;    // u8 [ngs][nkts_ff][kPfNsDn*128] shared h as bf16 high (rows 0-31), low (32-63)
    size_t o;      // f32 [Tp][k+1][d] expert outputs per (token, slot); slot k: shared
    size_t xn;     // bf16 [Tp][d] the layer's input RMSNorm(h) (pre-norm calls)
    size_t wsplit; // bf16 [3][E][d] the router split into three exact bf16 parts
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
    const size_t nrb_ff = ceil_div(ff, kTileM), nrbs_ff = ffs > 0 ? ceil_div(ffs, kTileM) : 0;
    const size_t nrb_d = ceil_div(d, kTileM);
    size_t o = align256(base);
    auto take = [&](size_t &field, size_t bytes) {
        field = o;
        o = align256(o + bytes);
    };
    take(P.lg, (size_t)Tp * E * 4);
    take(P.idx, (size_t)Tp * k * 4);
    take(P.wt, (size_t)Tp * k * 4);
    take(P.hist, (size_t)P.nhb * E * 4);
    take(P.ecnt, (size_t)E * 4);
    take(P.eoff, (size_t)E * 4);
    take(P.goff, (size_t)E * 4);
    take(P.perm, (size_t)Tp * k * 4);
    take(P.pw, (size_t)Tp * k * 4);
    take(P.grp, (size_t)(P.ngr + P.ngs) * 16);
    take(P.itg, ((size_t)P.ngr * nrb_ff + (size_t)P.ngs * nrbs_ff) * 16);
    take(P.itd, (size_t)(P.ngr + P.ngs) * nrb_d * 16);
    take(P.ploc, (size_t)Tp * k * 4);
    take(P.xg, (size_t)P.ngr * nkt_d * kPfN * 128);
    take(P.xgs, (size_t)P.ngr * nkt_d * 2 * kPfN * 4);
    take(P.xbf, (size_t)P.ngs * nkts_d * kPfNsGU * 128);
    take(P.hb, (size_t)P.ngr * nkt_ff * kPfN * 128);
    take(P.hsf, (size_t)P.ngr * nkt_ff * 2 * kPfN * 4);
    take(P.hsb, (size_t)P.ngs * nkts_ff * kPfNsDn * 128);
    take(P.o, (size_t)Tp * (k + 1) * d * 4);
    take(P.xn, (size_t)Tp * d * 2);
    take(P.wsplit, (size_t)3 * E * d * 2);
    P.total = o;
    return P;
}

}  // namespace k3

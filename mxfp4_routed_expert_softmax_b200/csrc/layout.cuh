// Workspace layout of one token chunk (up to kChunk tokens) of the layer.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace k3 {

constexpr int kChunk = 8;   // tokens per decode pass
constexpr int kMaxSeg = 8;  // most warps that share one router/shared row

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

struct Layout {
    size_t hdr;        // WsHeader
    size_t logits;     // f32 [kChunk][E]
    size_t idx;        // i32 [kChunk][k]
    size_t wt;         // f32 [kChunk][k]
    size_t sigx;       // i32 [kChunk]      E4M3 prescale exponent of each token's x
    size_t xp;         // u8  [kChunk][2][d] x * 2^sigx as two E4M3 pieces (even/odd-permuted)
    size_t uniq_blob;  // u64 [kChunk*k]    blob pointer of each distinct selected expert
    size_t uniq_mask;  // u32 [kChunk*k]    tokens (bit t) that selected it
    size_t uniq_slot;  // i8  [kChunk*k][kChunk] slot j of token t for it, -1 if none
    size_t hmax;       // u32 [kChunk][k]   max |h| of each (token, slot), as float bits
    size_t h;          // f32 [kChunk][k][ff] SwiGLU activations of each (token, slot)
    size_t hs;         // f32 [kChunk][ff_s] shared-expert activations
    size_t ob;         // f32 [kChunk][k+1][d] expert outputs: [0] shared, [1+j] slot j
    size_t part;       // f32 [2][E+ffs][kMaxSeg][4][2] partial sums of rows split between warps
    size_t cnt;        // u32 [2][E+ffs] arrivals per split row (back to 0 after each row)
    size_t total;
    int d, ff, E, k, ffs;
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
    L.sigx = o;
    o = align256(o + C * 4);
    L.xp = o;
    o = align256(o + C * 2 * (size_t)d);
    L.uniq_blob = o;
    o = align256(o + C * k * 8);
    L.uniq_mask = o;
    o = align256(o + C * k * 4);
    L.uniq_slot = o;
    o = align256(o + C * k * C);
    L.hmax = o;
    o = align256(o + C * k * 4);
    L.h = o;
    o = align256(o + C * k * (size_t)ff * 4);
    L.hs = o;
    o = align256(o + C * (size_t)(ffs > 0 ? ffs : 1) * 4);
    L.ob = o;
    o = align256(o + C * (k + 1) * (size_t)d * 4);
    L.part = o;
    o = align256(o + (size_t)2 * (E + ffs) * kMaxSeg * 4 * 2 * 4);
    L.cnt = o;
    o = align256(o + (size_t)2 * (E + ffs) * 4);
    L.total = o;
    return L;
}

}  // namespace k3

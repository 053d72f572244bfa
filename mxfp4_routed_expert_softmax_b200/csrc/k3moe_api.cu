// C ABI of the k3moe library: argument validation, workspace layout and the
// launch sequence of each entry point.  Declarations and the contract of
// every function are in include/k3moe.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>
#include <new>
#include <cstring>
#include <mutex>
#include <string>

#include "common.cuh"
#include "decode_kernels.cuh"
#include "expert_cache.cuh"
#include "k3moe.h"
#include "layer_kernel.cuh"
#include "layout.cuh"
#include "prefill_kernels.cuh"
#include "prefill_router_mma.cuh"

namespace {

using namespace k3;

thread_local std::string g_last_error;

constexpr int kMaxDevices = 64;
constexpr int kSmemLimit = 227 * 1024;

// Scratch of k3moe_layer_noalloc: one buffer per device, in the library's own
// device data (no allocation by the library or the caller).
constexpr size_t kNoAllocBytes = (size_t)16 << 20;
static __device__ __align__(256) uint8_t g_noalloc_ws[kNoAllocBytes];

struct DeviceInfo {
    bool ready = false;
    uint8_t *noalloc = nullptr;  // device address of g_noalloc_ws on this device, once set up
    int noalloc_shape[5] = {0, 0, 0, 0, 0};  // (d, ff, E, k, ff_shared) its layout was last used for
    int sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

// Failure-path test settings (k3moe_debug_set_fault): the injected fault and
// the bound of every device wait, read at each launch.
std::atomic<int> g_fault_mode{0};
std::atomic<uint64_t> g_wait_ns{0};

uint64_t wait_limit() {
    const uint64_t v = g_wait_ns.load(std::memory_order_relaxed);
    return v ? v : kWaitLimitNs;
}

k3moe_status cuda_fail(cudaError_t e, const char *where = nullptr) {
    g_last_error = cudaGetErrorString(e);
    if (where) g_last_error = std::string(where) + ": " + g_last_error;
    return K3MOE_ERR_CUDA;
}

template <typename Kern>
cudaError_t set_smem(Kern kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}


// One-time per-device set-up: SM count and the shared-memory opt-ins.
k3moe_status device_info(DeviceInfo **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return K3MOE_ERR_INVALID_ARGUMENT;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo &di = g_dev[dev];
    if (!di.ready) {
        e = cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e);
        const int big = kSmemLimit;
        cudaError_t r = set_smem(umma_expert_kernel<true>, big);
        if (r == cudaSuccess) r = set_smem(umma_expert_kernel<false>, big);
        if (r == cudaSuccess) r = set_smem(pf_expert_kernel<true>, big);
        if (r == cudaSuccess) r = set_smem(pf_expert_kernel<false>, big);
        if (r == cudaSuccess) r = set_smem(layer_kernel<1, true>, big);
        if (r == cudaSuccess) r = set_smem(layer_kernel<0, false>, big);
        if (r == cudaSuccess) r = set_smem(pf_router_mma_kernel, rm_smem_bytes());
        if (r != cudaSuccess) return cuda_fail(r);
        di.ready = true;
    }
    *out = &di;
    return K3MOE_OK;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int shared_ff(const k3moe_dims *dm) {
    return (dm->flags & K3MOE_NO_SHARED) ? 0 : dm->ff_shared;
}

// Pipeline depth of the tensor-core kernels: as many stages as fit in shared
// memory and in the TMEM scale columns (8 stages after the accumulators).
int umma_stages(bool gu, int N) {
    int n = (kSmemLimit - umma_smem_bytes(gu, N, 0)) / umma_stage_bytes(gu, N);
    const int cap = 8;
    return n < cap ? n : cap;
}

k3moe_status check_dims(const k3moe_dims *dm) {
    if (!dm) return K3MOE_ERR_INVALID_ARGUMENT;
    if (dm->flags & ~(K3MOE_OUT_FP32 | K3MOE_NO_SHARED | K3MOE_STRICT | K3MOE_RENORM_TOPK | K3MOE_BIAS_SELECT_ONLY |
                      K3MOE_ONE_LAUNCH))
        return K3MOE_ERR_INVALID_ARGUMENT;
    if (dm->d < 64 || dm->d > 8192 || dm->d % 64) return K3MOE_ERR_UNSUPPORTED_SHAPE;
    if (dm->ff < 64 || dm->ff > 3072 || dm->ff % 64) return K3MOE_ERR_UNSUPPORTED_SHAPE;
    if (dm->n_experts < 1 || dm->n_experts > 1024) return K3MOE_ERR_UNSUPPORTED_SHAPE;
    if (dm->top_k < 1 || dm->top_k > 32 || dm->top_k > dm->n_experts)
        return K3MOE_ERR_INVALID_ARGUMENT;
    if (dm->ff_shared < 0 || dm->ff_shared > 3072 || dm->ff_shared % 64)
        return K3MOE_ERR_UNSUPPORTED_SHAPE;
    return K3MOE_OK;
}

// Routing-variant bits of the kernels' parameters from the call's flags.
int route_flags(const k3moe_dims *dm) {
    return ((dm->flags & K3MOE_RENORM_TOPK) ? kRouteRenorm : 0) |
           ((dm->flags & K3MOE_BIAS_SELECT_ONLY) ? kRouteBiasSelect : 0);
}

Layout layout_for(const k3moe_dims *dm, int k_eff) {
    return make_layout(dm->d, dm->ff, dm->n_experts, k_eff, dm->ff_shared);
}

// ---------------------------------------------------------- prefill pass --
// A pass of the grouped prefill takes up to kPfMaxTokens tokens.
int pf_pass_tokens(const k3moe_dims *dm, int T) {
    (void)dm;
    return T < kPfMaxTokens ? T : kPfMaxTokens;
}

PLayout playout_for(const k3moe_dims *dm, int Tp) {
    const Layout L = layout_for(dm, dm->top_k);
    const int ffs = (dm->flags & K3MOE_NO_SHARED) ? 0 : dm->ff_shared;
    return make_playout(L.total, dm->d, dm->ff, dm->n_experts, dm->top_k, ffs, Tp);
}

// Scratch for a call of T tokens on the grouped prefill path (0: T is one chunk).
size_t pf_need(const k3moe_dims *dm, int T) {
    if (T <= kChunk) return 0;
    const int Tp = pf_pass_tokens(dm, T);
    if (Tp <= kChunk) return 0;
    return playout_for(dm, Tp).total;
}

size_t staging_bytes(const k3moe_dims *dm, int T) {
    const size_t n = T > kChunk ? (size_t)T : (size_t)kChunk;
    return align256(n * dm->d * 2) + align256(n * dm->d * 4);
}

template <typename Kern, typename P>
cudaError_t launch(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                   const P &params) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, params);
}


// ------------------------------------------------------ tensor maps --
// Templates of the two nibble-plane tensor maps (u8 elements, 128 x 128-byte
// boxes, 128-byte swizzle): W_g / W_u (ff rows of d/2 bytes) and W_d (d rows
// of ff/2 bytes).  The device copies them per selected expert and points the
// copy at that expert's plane, so the encoded address is a placeholder.
// The encoder is reached through the runtime's driver entry point, so the
// library does not link the driver library itself.
struct TmapCache {
    int d = 0, ff = 0;
    uint4 t[kTemplates][8];
};
TmapCache g_tmaps[16];
int g_ntmaps = 0;

k3moe_status tmap_templates(int d, int ff, void *placeholder, uint4 (&out)[kTemplates][8]) {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_ntmaps; ++i)
        if (g_tmaps[i].d == d && g_tmaps[i].ff == ff) {
            memcpy(out, g_tmaps[i].t, sizeof(out));
            return K3MOE_OK;
        }
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return cuda_fail(e);
        if (q != cudaDriverEntryPointSuccess || !fn) {
            g_last_error = "cuTensorMapEncodeTiled is not available";
            return K3MOE_ERR_CUDA;
        }
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    // [0], [1]: nibble planes, 128 rows x 128 bytes, 128-byte swizzle (the
    // MMA's K-major layout); [2], [3]: scale planes, 128 rows x 16 bytes, no
    // swizzle, only when the row of scales is a multiple of 16 bytes (the
    // reduction length a multiple of 512), else left zero; [4], [5]: W_d's
    // nibble and scale planes again with 256-row boxes.
    CUtensorMap m[kTemplates];
    memset(m, 0, sizeof(m));
    for (int i = 0; i < kTemplates; ++i) {
        const bool wd = i == 1 || i == 3 || i >= 4;
        const int kdim = wd ? ff : d, rdim = wd ? d : ff;
        const bool scale = i == 2 || i == 3 || i == 5;
        if (scale && kdim % 512 != 0) continue;
        const cuuint64_t cols = (cuuint64_t)(scale ? kdim / 32 : kdim / 2), rows = (cuuint64_t)rdim;
        const cuuint64_t dims[2] = {cols, rows};
        const cuuint64_t strides[1] = {cols};
        const cuuint32_t box[2] = {scale ? 16u : 128u, (cuuint32_t)(i >= 4 ? 2 * kTileM : kTileM)};
        const cuuint32_t es[2] = {1, 1};
        CUresult r = encode(&m[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, placeholder, dims, strides, box, es,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, scale ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            g_last_error = "cuTensorMapEncodeTiled failed (" + std::to_string((int)r) + ")";
            return K3MOE_ERR_CUDA;
        }
    }
    static_assert(sizeof(CUtensorMap) == 128, "tensor map is 128 bytes");
    memcpy(out, m, sizeof(out));
    if (g_ntmaps < 16) {
        g_tmaps[g_ntmaps].d = d;
        g_tmaps[g_ntmaps].ff = ff;
        memcpy(g_tmaps[g_ntmaps].t, m, sizeof(m));
        ++g_ntmaps;
    }
    return K3MOE_OK;
}

// Tensor maps of the bf16 shared expert at its real addresses (u8 elements,
// 128 x 128-byte boxes, 128-byte swizzle): W_g, W_u (ff_s rows of 2d bytes),
// W_d (d rows of 2 ff_s bytes), and W_d again with 256-row boxes.
k3moe_status shared_tmaps(int d, int ffs, const void *wg, const void *wu, const void *wd,
                          uint4 (&out)[kSharedMaps][8]) {
    std::lock_guard<std::mutex> lock(g_mu);
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return cuda_fail(e);
        if (q != cudaDriverEntryPointSuccess || !fn) {
            g_last_error = "cuTensorMapEncodeTiled is not available";
            return K3MOE_ERR_CUDA;
        }
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const void *addr[kSharedMaps] = {wg, wu, wd, wd};
    CUtensorMap m[kSharedMaps];
    for (int i = 0; i < kSharedMaps; ++i) {
        const cuuint64_t cols = (cuuint64_t)(i < 2 ? d : ffs) * 2, rows = (cuuint64_t)(i < 2 ? ffs : d);
        const cuuint64_t dims[2] = {cols, rows};
        const cuuint64_t strides[1] = {cols};
        const cuuint32_t box[2] = {128, (cuuint32_t)(i == 3 ? 2 * kTileM : kTileM)};
        const cuuint32_t es[2] = {1, 1};
        CUresult r = encode(&m[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(addr[i]), dims, strides, box,
                            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            g_last_error = "cuTensorMapEncodeTiled failed (" + std::to_string((int)r) + ")";
            return K3MOE_ERR_CUDA;
        }
    }
    memcpy(out, m, sizeof(out));
    return K3MOE_OK;
}

// A 2-D tensor map of 16-bit elements [rows][cols] (row pitch cols * 2 bytes),
// boxes of 64 columns x 128 rows with the 128-byte swizzle (the MMA's K-major
// operand layout).
k3moe_status tmap_bf16_rows(const void *addr, int cols, int rows, uint4 (&out)[8]) {
    std::lock_guard<std::mutex> lock(g_mu);
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return cuda_fail(e);
        if (q != cudaDriverEntryPointSuccess || !fn) {
            g_last_error = "cuTensorMapEncodeTiled is not available";
            return K3MOE_ERR_CUDA;
        }
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    CUtensorMap m;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kRmKStep, (cuuint32_t)kRmTile};
    const cuuint32_t es[2] = {1, 1};
    CUresult r = encode(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(addr), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_error = "cuTensorMapEncodeTiled failed (" + std::to_string((int)r) + ")";
        return K3MOE_ERR_CUDA;
    }
    memcpy(out, &m, sizeof(out));
    return K3MOE_OK;
}

template <bool GU>
cudaError_t launch_umma(const DeviceInfo &di, UmmaParams up, cudaStream_t st) {
    const int N = act_n(up.Tc);
    up.nst = umma_stages(GU, N);
    up.sb = umma_stage_bytes(GU, N);
    up.sf_tma = (GU ? up.d : up.ff) % 512 == 0;
    up.wait_ns = wait_limit();
    up.inject = GU ? g_fault_mode.load(std::memory_order_relaxed) : 0;
    const int smem = umma_smem_bytes(GU, N, up.nst);
    const int g = di.sms < kMaxCtas ? di.sms : kMaxCtas;
    return launch(umma_expert_kernel<GU>, dim3(g), dim3(kUThreads), smem, st, true, up);
}


// Router (+ top-k + dispatch + activation pieces) for one chunk.  Cooperative
// launch (CTA t waits on the other CTAs' router rows, so all must be
// resident), one CTA per SM: Tc CTAs for the pieces and the top-k, the rest
// stream the router, about eight row parts per warp at least.  grid_out: the
// CTAs that count on prep_done (all of them; the gate/up pass waits for it).
cudaError_t launch_route(DeviceInfo &di, RouteParams rp, cudaStream_t st, int *grid_out = nullptr) {
    if (di.sms < kChunk + 1) return cudaErrorInvalidConfiguration;
    const long long nseg = (long long)rp.E * (rp.d / router_part_len(rp.d));
    long long ns = (nseg + 8 * (kRouteThreads / 32) - 1) / (8 * (kRouteThreads / 32));
    if (ns > di.sms - rp.Tc) ns = di.sms - rp.Tc;
    if (ns < 1) ns = 1;
    rp.nded = rp.Tc;
    rp.wait_ns = wait_limit();
    if (grid_out) *grid_out = (int)(rp.Tc + ns);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rp.Tc + ns));
    cfg.blockDim = dim3(kRouteThreads);
    cfg.dynamicSmemBytes = route_dyn_bytes(rp.E);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return rp.Tc == 1 ? cudaLaunchKernelEx(&cfg, route_kernel<1>, rp)
                      : cudaLaunchKernelEx(&cfg, route_kernel<kRouteTok>, rp);
}

// Decode passes of this call by the one-launch kernel (K3MOE_ONE_LAUNCH);
// the pre-norm and routing-given calls take it whatever the flag.
inline bool one_launch(const k3moe_dims *dm) { return (dm->flags & K3MOE_ONE_LAUNCH) != 0; }

// The one-launch decode pass (layer_kernel) for this shape, if it fits: the
// pipeline stages and the routing tables in one SM's shared memory, and the
// rows of one CTA's router slice in its row accumulators.  0: not supported
// (the three-kernel pass runs instead).
int layer_stages(const DeviceInfo &di, const k3moe_dims *dm, int Tc) {
    const int N = act_n(Tc);
    const int rest = kSmemLimit - 1024 - lk_smem(dm->n_experts, dm->top_k, Tc, dm->d).total;
    int nst = rest / lk_stage_bytes(N);
    if (nst > 8) nst = 8;
    if (nst < 2) return 0;
    if (dm->d > kLRUnit) return 0;  // a router unit holds whole rows
    const int rpu = lk_rows_per_unit(dm->d);
    const int n0 = (dm->n_experts + rpu - 1) / rpu;
    const int G = di.sms < kLMaxCtas ? di.sms : kLMaxCtas;
    const int g0 = n0 < G ? n0 : G;
    const int upc = (n0 + g0 - 1) / g0;  // router units of one CTA at most
    if (upc * rpu > kRMaxRows) return 0;
    return nst;
}

// Cooperative launch: the CTAs wait on each other's counters (router rows,
// activation pieces, gate/up items), so all of them must be resident.
cudaError_t launch_layer(const DeviceInfo &di, LayerParams lp, int nst, cudaStream_t st) {
    const int N = act_n(lp.r.Tc);
    lp.nst = nst;
    lp.sb = lk_stage_bytes(N);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(di.sms < kLMaxCtas ? di.sms : kLMaxCtas));
    cfg.blockDim = dim3(kLThreads);
    cfg.dynamicSmemBytes = lk_smem_bytes(N, nst, lp.r.E, lp.r.k, lp.r.Tc, lp.r.d);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // one decode token with TMA scale boxes: the specialised instance
    if (lp.r.Tc == 1 && lp.sf_tma_gu && lp.sf_tma_dn) return cudaLaunchKernelEx(&cfg, layer_kernel<1, true>, lp);
    return cudaLaunchKernelEx(&cfg, layer_kernel<0, false>, lp);
}

// The routing of one decode pass by the one-launch kernel stopped after its
// top-k (the picks land in the workspace and in idx_out / w_out): the same
// bits as the routing inside a full launch of the same pass.
cudaError_t launch_layer_route(const DeviceInfo &di, const RouteParams &rp, int nst, cudaStream_t st, bool ff_tma) {
    LayerParams lp{};
    lp.r = rp;
    lp.r.wait_ns = wait_limit();
    lp.mode = kLayerRouteOnly;
    // the instance a full launch of the same pass takes (same routing code)
    lp.sf_tma_gu = lp.sf_tma_dn = rp.d % 512 == 0 && ff_tma;
    return launch_layer(di, lp, nst, st);
}

// Launches of the grouped prefill, pass after pass; rp carries the shapes,
// blobs and tensor-map templates.  routing_only: stop after the top-k.
// norm_w (non-null): x holds the residual stream h; the layer runs on
// RMSNorm(h) (written into the pass's xn region) and h is added to its output.
k3moe_status prefill_impl(DeviceInfo &di, RouteParams rp, const k3moe_dims *dims, const uint16_t *x, int T,
                          void *y, int32_t *idx_out, float *w_out, cudaStream_t st, bool routing_only = false,
                          const uint16_t *norm_w = nullptr, float eps = 0.f) {
    const int d = dims->d, E = dims->n_experts, k = dims->top_k;
    const int ffs = rp.has_shared ? dims->ff_shared : 0;
    const bool out32 = (dims->flags & K3MOE_OUT_FP32) != 0;
    const int Tp = pf_pass_tokens(dims, T);
    const PLayout P = playout_for(dims, Tp);
    uint8_t *wsb = rp.ws;
    cudaError_t e;
    // the router as three exact bf16 parts, once per call, and their tensor maps
    RouterMmaParams rm{};
    {
        uint16_t *w1 = reinterpret_cast<uint16_t *>(wsb + P.wsplit);
        const size_t n = (size_t)E * d;
        const RouterSplitParams spp{rp.wr, n, w1, w1 + n, w1 + 2 * n};
        e = launch(pf_router_split_kernel, dim3(4 * di.sms), dim3(256), 0, st, false, spp);
        if (e != cudaSuccess) return cuda_fail(e, "router split launch");
        for (int q = 0; q < 3; ++q) {
            k3moe_status s = tmap_bf16_rows(w1 + q * n, d, E, rm.tw[q]);
            if (s != K3MOE_OK) return s;
        }
        rm.bias = (rp.route_flags & kRouteBiasSelect) ? nullptr : rp.bias;
        rm.d = d;
        rm.E = E;
        rm.ws = wsb;
        rm.wait_ns = wait_limit();
    }
    for (int t0 = 0; t0 < T; t0 += Tp) {
        const int Tq = (T - t0) < Tp ? (T - t0) : Tp;
        const uint16_t *xq = x + (size_t)t0 * d;
        if (norm_w) {
            const PfNormParams np{xq, norm_w, eps, Tq, d, reinterpret_cast<uint16_t *>(wsb + P.xn)};
            e = launch(pf_rmsnorm_kernel, dim3(ceil_div(Tq, 8)), dim3(256), 0, st, false, np);
            if (e != cudaSuccess) return cuda_fail(e, "prefill norm launch");
            xq = reinterpret_cast<const uint16_t *>(wsb + P.xn);
        }
        PfRouteParams pp{};
        pp.r = rp;
        pp.r.x = xq;
        pp.r.Tc = Tq;
        pp.r.idx_out = idx_out ? idx_out + (size_t)t0 * k : nullptr;
        pp.r.w_out = w_out ? w_out + (size_t)t0 * k : nullptr;
        pp.P = P;
        pp.T = Tq;
        pp.ngs = ffs > 0 ? ceil_div(Tq, kGroup) : 0;
        pp.ff = dims->ff;
        pp.ffs = ffs;
        // router: tiles of 128 experts x 128 tokens on the tensor cores
        {
            k3moe_status s = tmap_bf16_rows(pp.r.x, d, Tq, rm.tx);
            if (s != K3MOE_OK) return s;
            rm.T = Tq;
            rm.out = reinterpret_cast<float *>(wsb + P.lg);
            const int tiles = ceil_div(E, kRmTile) * ceil_div(Tq, kRmTile);
            e = launch(pf_router_mma_kernel, dim3(tiles < di.sms ? tiles : di.sms), dim3(kRmThreads), rm_smem_bytes(),
                       st, false, rm);
            if (e != cudaSuccess) return cuda_fail(e, "prefill router launch");
        }
        e = launch(pf_topk_kernel, dim3(Tq), dim3(kRouteThreads), 0, st, false, pp);
        if (e != cudaSuccess) return cuda_fail(e, "prefill top-k launch");
        if (routing_only) continue;
        const int nhb = ceil_div(Tq, kPfHistTok);
        e = launch(pf_hist_kernel, dim3(nhb), dim3(kRouteThreads), 0, st, false, pp);
        if (e == cudaSuccess) e = launch(pf_scan_kernel, dim3(1), dim3(kPfScanThreads), 0, st, false, pp);
        if (e == cudaSuccess) e = launch(pf_place_kernel, dim3(nhb), dim3(kRouteThreads), 0, st, false, pp);
        if (e == cudaSuccess) e = launch(pf_items_kernel, dim3(2 * di.sms), dim3(256), 0, st, false, pp);
        if (e == cudaSuccess) e = launch(pf_prep_kernel, dim3(2 * di.sms), dim3(kRouteThreads), 0, st, false, pp);
        if (e != cudaSuccess) return cuda_fail(e, "prefill dispatch launch");
        PfUmmaParams up{};
        up.d = d;
        up.ff = dims->ff;
        up.k = k;
        up.ffs = ffs;
        up.ws = wsb;
        up.L = rp.L;
        up.P = P;
        up.ngs = pp.ngs;
        up.blobs = rp.blobs;
        up.wait_ns = wait_limit();
        up.strict = (dims->flags & K3MOE_STRICT) != 0;
        for (int gu = 1; gu >= 0; --gu) {
            const int sb = pf_stage_bytes(gu != 0);
            int nst = (kSmemLimit - pf_smem_bytes(gu != 0, 0)) / sb;
            if (nst > 8) nst = 8;
            up.nst = nst;
            up.sb = sb;
            up.sf_tma = (gu ? d : dims->ff) % 512 == 0;
            const int smem = pf_smem_bytes(gu != 0, nst);
            e = gu ? launch(pf_expert_kernel<true>, dim3(di.sms), dim3(kPfThreads), smem, st, true, up)
                   : launch(pf_expert_kernel<false>, dim3(di.sms), dim3(kPfThreads), smem, st, true, up);
            if (e != cudaSuccess) return cuda_fail(e, gu ? "prefill gate/up launch" : "prefill down launch");
        }
        PfCombineParams cp{};
        cp.o = reinterpret_cast<const float *>(wsb + P.o);
        cp.T = Tq;
        cp.d = d;
        cp.k = k;
        cp.has_shared = ffs > 0;
        cp.out_fp32 = out32;
        cp.y = reinterpret_cast<uint8_t *>(y) + (size_t)t0 * d * (out32 ? 4 : 2);
        cp.resid = norm_w ? x + (size_t)t0 * d : nullptr;
        e = launch(pf_combine_kernel, dim3(4 * di.sms), dim3(256), 0, st, false, cp);
        if (e != cudaSuccess) return cuda_fail(e, "prefill combine launch");
    }
    return K3MOE_OK;
}

struct EventHook {
    cudaEvent_t *ev = nullptr;
    int n = 0;
    int next = 0;
    int kernels = 0;  // kernels of the last pass
    cudaError_t record(cudaStream_t st) {
        if (!ev || next >= n) return cudaSuccess;
        return cudaEventRecord(ev[next++], st);
    }
};

// norm_w (non-null): x is the residual stream h, the layer runs on
// RMSNorm(h) and y = h + layer (the decode passes need the one-launch kernel).
k3moe_status layer_impl(const void *x, int32_t T, const float *w_router, const float *bias,
                        const uint8_t *const *expert_blobs, const void *shared_wg,
                        const void *shared_wu, const void *shared_wd, const k3moe_dims *dims,
                        void *y, int32_t *idx_out, float *w_out, void *ws, size_t ws_bytes,
                        void *stream, const void *x_host, void *y_host, EventHook *hook = nullptr,
                        const uint16_t *norm_w = nullptr, float eps = 0.f, int layer_mode = kLayerFull) {
    k3moe_status s = check_dims(dims);
    if (s != K3MOE_OK) return s;
    const bool from_host = x_host != nullptr;
    if (T < 1) return K3MOE_ERR_INVALID_ARGUMENT;
    if (!from_host && (!x || !y || !aligned(x, 16) || !aligned(y, 16)))
        return K3MOE_ERR_INVALID_ARGUMENT;
    if (from_host && !y_host) return K3MOE_ERR_INVALID_ARGUMENT;
    if (!w_router || !aligned(w_router, 16) || !expert_blobs || !aligned(expert_blobs, 8))
        return K3MOE_ERR_INVALID_ARGUMENT;
    if (bias && !aligned(bias, 4)) return K3MOE_ERR_INVALID_ARGUMENT;
    if ((idx_out && !aligned(idx_out, 4)) || (w_out && !aligned(w_out, 4)))
        return K3MOE_ERR_INVALID_ARGUMENT;
    const int ffs = shared_ff(dims);
    if (ffs > 0) {
        if (!shared_wg || !shared_wu || !shared_wd || !aligned(shared_wg, 16) ||
            !aligned(shared_wu, 16) || !aligned(shared_wd, 16))
            return K3MOE_ERR_INVALID_ARGUMENT;
    }
    if (!ws || !aligned(ws, 256)) return K3MOE_ERR_INVALID_ARGUMENT;
    const Layout L = layout_for(dims, dims->top_k);
    // grouped prefill when the workspace holds its region (else 8-token passes)
    const size_t pfn = hook ? 0 : pf_need(dims, T);
    const bool grouped = pfn > 0 && ws_bytes >= pfn + (from_host ? staging_bytes(dims, T) : 0);
    const size_t base = grouped ? pfn : L.total;
    const size_t need = base + (from_host ? staging_bytes(dims, grouped ? T : kChunk) : 0);
    if (ws_bytes < need) return K3MOE_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo *di = nullptr;
    s = device_info(&di);
    if (s != K3MOE_OK) return s;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *wsb = reinterpret_cast<uint8_t *>(ws);
    const int d = dims->d;
    const bool out32 = (dims->flags & K3MOE_OUT_FP32) != 0;
    const size_t ybytes = out32 ? 4 : 2;
    uint8_t *xstage = wsb + base;
    uint8_t *ystage = xstage + align256((size_t)(grouped ? T : kChunk) * d * 2);

    uint4 tmpl[kTemplates][8];
    s = tmap_templates(d, dims->ff, ws, tmpl);
    if (s != K3MOE_OK) return s;
    uint4 smap[kSharedMaps][8];
    memset(smap, 0, sizeof(smap));
    if (ffs > 0) {
        s = shared_tmaps(d, ffs, shared_wg, shared_wu, shared_wd, smap);
        if (s != K3MOE_OK) return s;
    }

    if (grouped) {
        RouteParams rp{};
        rp.wr = w_router;
        rp.bias = bias;
        rp.d = d;
        rp.E = dims->n_experts;
        rp.k = dims->top_k;
        rp.ws = wsb;
        rp.L = L;
        rp.blobs = expert_blobs;
        rp.route_flags = route_flags(dims);
        memcpy(rp.tmpl, tmpl, sizeof(tmpl));
        rp.scale_mask = (d % 512 == 0 ? 1 : 0) | (dims->ff % 512 == 0 ? 2 : 0);
        memcpy(rp.smap, smap, sizeof(smap));
        rp.has_shared = ffs > 0;
        rp.sw[0] = reinterpret_cast<const uint8_t *>(shared_wg);
        rp.sw[1] = reinterpret_cast<const uint8_t *>(shared_wu);
        rp.sw[2] = reinterpret_cast<const uint8_t *>(shared_wd);
        cudaError_t e;
        if (from_host) {
            e = cudaMemcpyAsync(xstage, x_host, (size_t)T * d * 2, cudaMemcpyHostToDevice, st);
            if (e != cudaSuccess) return cuda_fail(e);
            x = xstage;
            y = ystage;
        }
        s = prefill_impl(*di, rp, dims, reinterpret_cast<const uint16_t *>(x), T, y, idx_out, w_out, st, false,
                         norm_w, eps);
        if (s != K3MOE_OK) return s;
        if (from_host) {
            e = cudaMemcpyAsync(y_host, ystage, (size_t)T * d * ybytes, cudaMemcpyDeviceToHost, st);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        return K3MOE_OK;
    }

    for (int c0 = 0; c0 < T; c0 += kChunk) {
        const int Tc = (T - c0) < kChunk ? (T - c0) : kChunk;
        const uint16_t *xc;
        void *yc;
        cudaError_t e;
        if (from_host) {
            e = cudaMemcpyAsync(xstage, reinterpret_cast<const uint8_t *>(x_host) + (size_t)c0 * d * 2,
                                (size_t)Tc * d * 2, cudaMemcpyHostToDevice, st);
            if (e != cudaSuccess) return cuda_fail(e);
            xc = reinterpret_cast<const uint16_t *>(xstage);
            yc = ystage;
        } else {
            xc = reinterpret_cast<const uint16_t *>(x) + (size_t)c0 * d;
            yc = reinterpret_cast<uint8_t *>(y) + (size_t)c0 * d * ybytes;
        }
        RouteParams rp{};
        rp.x = xc;
        rp.Tc = Tc;
        rp.wr = w_router;
        rp.bias = bias;
        rp.d = d;
        rp.E = dims->n_experts;
        rp.k = dims->top_k;
        rp.ws = wsb;
        rp.L = L;
        rp.blobs = expert_blobs;
        rp.route_flags = route_flags(dims);
        rp.idx_out = idx_out ? idx_out + (size_t)c0 * dims->top_k : nullptr;
        rp.w_out = w_out ? w_out + (size_t)c0 * dims->top_k : nullptr;
        memcpy(rp.tmpl, tmpl, sizeof(tmpl));
        rp.scale_mask = (d % 512 == 0 ? 1 : 0) | (dims->ff % 512 == 0 ? 2 : 0);
        memcpy(rp.smap, smap, sizeof(smap));
        rp.has_shared = ffs > 0;
        rp.sw[0] = reinterpret_cast<const uint8_t *>(shared_wg);
        rp.sw[1] = reinterpret_cast<const uint8_t *>(shared_wu);
        rp.sw[2] = reinterpret_cast<const uint8_t *>(shared_wd);
        EventHook none;
        EventHook &hk = hook ? *hook : none;
        if ((e = hk.record(st)) != cudaSuccess) return cuda_fail(e);
        const int lst = (one_launch(dims) || layer_mode != kLayerFull) ? layer_stages(*di, dims, Tc) : 0;
        if (layer_mode != kLayerFull && lst == 0) return K3MOE_ERR_UNSUPPORTED_SHAPE;
        if (lst > 0) {
            // the whole pass in one launch
            LayerParams lp{};
            lp.r = rp;
            lp.r.wait_ns = wait_limit();
            lp.ff = dims->ff;
            lp.ffs = ffs;
            lp.sf_tma_gu = d % 512 == 0;
            lp.sf_tma_dn = dims->ff % 512 == 0;
            lp.out_fp32 = out32;
            lp.y = yc;
            lp.strict = (dims->flags & K3MOE_STRICT) != 0;
            lp.inject = g_fault_mode.load(std::memory_order_relaxed);
            lp.norm_w = norm_w;
            lp.eps = eps;
            lp.resid = norm_w ? xc : nullptr;
            lp.mode = layer_mode;
            e = launch_layer(*di, lp, lst, st);
            if (e != cudaSuccess) return cuda_fail(e, "layer launch");
            if ((e = hk.record(st)) != cudaSuccess) return cuda_fail(e);
            hk.kernels = 1;
            if (from_host) {
                e = cudaMemcpyAsync(reinterpret_cast<uint8_t *>(y_host) + (size_t)c0 * d * ybytes, ystage,
                                    (size_t)Tc * d * ybytes, cudaMemcpyDeviceToHost, st);
                if (e != cudaSuccess) return cuda_fail(e);
            }
            continue;
        }
        hk.kernels = 3;
        if (norm_w) {
            // pre-norm: the chunk's normalised input into the workspace (the
            // residual stream xc stays for the residual add at the end)
            const PfNormParams np{xc, norm_w, eps, Tc, d, reinterpret_cast<uint16_t *>(wsb + L.xn)};
            e = launch(pf_rmsnorm_kernel, dim3(ceil_div(Tc, 8)), dim3(256), 0, st, false, np);
            if (e != cudaSuccess) return cuda_fail(e, "rmsnorm launch");
            rp.x = reinterpret_cast<const uint16_t *>(wsb + L.xn);
        }
        int route_ctas = 0;
        e = launch_route(*di, rp, st, &route_ctas);
        if (e != cudaSuccess) return cuda_fail(e, "router launch");
        if ((e = hk.record(st)) != cudaSuccess) return cuda_fail(e);

        UmmaParams up{};
        up.Tc = Tc;
        up.d = d;
        up.ff = dims->ff;
        up.k = dims->top_k;
        up.ffs = ffs;
        up.ws = wsb;
        up.L = L;
        up.out_fp32 = out32;
        up.y = yc;
        up.resid = norm_w ? xc : nullptr;
        up.route_ctas = route_ctas;
        up.strict = (dims->flags & K3MOE_STRICT) != 0;
        static_assert(sizeof(up.smap_d) == sizeof(smap[3]), "one tensor map");
        memcpy(up.smap_d, smap[3], sizeof(up.smap_d));
        e = launch_umma<true>(*di, up, st);
        if (e != cudaSuccess) return cuda_fail(e, "gate/up launch");
        if ((e = hk.record(st)) != cudaSuccess) return cuda_fail(e);

        e = launch_umma<false>(*di, up, st);
        if (e != cudaSuccess) return cuda_fail(e, "down launch");
        if ((e = hk.record(st)) != cudaSuccess) return cuda_fail(e);

        if (from_host) {
            e = cudaMemcpyAsync(reinterpret_cast<uint8_t *>(y_host) + (size_t)c0 * d * ybytes, ystage,
                                (size_t)Tc * d * ybytes, cudaMemcpyDeviceToHost, st);
            if (e != cudaSuccess) return cuda_fail(e);
        }
    }
    return K3MOE_OK;
}

// Device address of the built-in scratch of k3moe_layer_noalloc on the
// current device (looked up on the first use; the caller holds g_mu).
k3moe_status noalloc_address(DeviceInfo &di) {
    if (!di.noalloc) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_ws);
        if (e != cudaSuccess) return cuda_fail(e, "scratch address");
        di.noalloc = reinterpret_cast<uint8_t *>(p);
    }
    return K3MOE_OK;
}

// The built-in scratch of k3moe_layer_noalloc on this device.  The workspace
// layout depends on the shape, and every layout keeps counters that must
// start at zero, so the buffer is cleared (on the call's stream) whenever the
// shape differs from the one it last served, the first call included.  Every
// call also clears the header's counters (not its status word): a call that
// gave up part-way (a bounded wait ran out) may have left them raised, and
// the next call must not take them for its own progress.
k3moe_status noalloc_scratch(DeviceInfo &di, const k3moe_dims *dm, cudaStream_t st, uint8_t **out) {
    std::lock_guard<std::mutex> lock(g_mu);
    k3moe_status s = noalloc_address(di);
    if (s != K3MOE_OK) return s;
    const int shape[5] = {dm->d, dm->ff, dm->n_experts, dm->top_k, dm->ff_shared};
    cudaError_t e;
    if (memcmp(shape, di.noalloc_shape, sizeof(shape)) != 0) {
        e = cudaMemsetAsync(di.noalloc, 0, kNoAllocBytes, st);
        if (e != cudaSuccess) return cuda_fail(e, "scratch clear");
        memcpy(di.noalloc_shape, shape, sizeof(shape));
    } else {
        e = cudaMemsetAsync(di.noalloc + sizeof(uint32_t), 0, sizeof(WsHeader) - sizeof(uint32_t), st);
        if (e != cudaSuccess) return cuda_fail(e, "scratch header clear");
    }
    *out = di.noalloc;
    return K3MOE_OK;
}

}  // namespace

// The opaque cache handle of the C ABI.
struct k3moe_cache {
    k3::ExpertCache c;
    std::vector<uint64_t> table;  // the last pointer table written (host copy)
    std::vector<int> fe, fs;      // the last fetch's fills
};

extern "C" {

int k3moe_abi_version(void) { return K3MOE_ABI_VERSION; }

size_t k3moe_blob_bytes(const k3moe_dims *dims) {
    if (check_dims(dims) != K3MOE_OK) return 0;
    return (size_t)3 * dims->d * dims->ff * 17 / 32;
}

size_t k3moe_workspace_size(const k3moe_dims *dims, int32_t T_max) {
    if (check_dims(dims) != K3MOE_OK || T_max < 1) return 0;
    const size_t dec = layout_for(dims, dims->top_k).total, pf = pf_need(dims, T_max);
    return pf > dec ? pf : dec;
}

size_t k3moe_host_staging_bytes(const k3moe_dims *dims, int32_t T) {
    if (check_dims(dims) != K3MOE_OK || T < 1) return 0;
    return staging_bytes(dims, T);
}

k3moe_status k3moe_route(const void *x, int32_t T, const float *w_router, const float *bias,
                         const k3moe_dims *dims, int32_t *idx, float *weight, void *ws,
                         size_t ws_bytes, void *stream) {
    k3moe_status s = check_dims(dims);
    if (s != K3MOE_OK) return s;
    if (T < 1 || !x || !aligned(x, 16) || !w_router || !aligned(w_router, 16) || !idx ||
        !weight || !aligned(idx, 4) || !aligned(weight, 4) || (bias && !aligned(bias, 4)))
        return K3MOE_ERR_INVALID_ARGUMENT;
    if (!ws || !aligned(ws, 256)) return K3MOE_ERR_INVALID_ARGUMENT;
    const Layout L = layout_for(dims, dims->top_k);
    if (ws_bytes < L.total) return K3MOE_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo *di = nullptr;
    s = device_info(&di);
    if (s != K3MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t pfn = pf_need(dims, T);
    if (pfn > 0 && ws_bytes >= pfn) {
        // many tokens: the prefill router (a GEMM over all of them) and top-k
        RouteParams rp{};
        rp.wr = w_router;
        rp.bias = bias;
        rp.d = dims->d;
        rp.E = dims->n_experts;
        rp.k = dims->top_k;
        rp.ws = reinterpret_cast<uint8_t *>(ws);
        rp.L = L;
        rp.route_flags = route_flags(dims);
        return prefill_impl(*di, rp, dims, reinterpret_cast<const uint16_t *>(x), T, nullptr, idx, weight, st, true);
    }
    for (int c0 = 0; c0 < T; c0 += kChunk) {
        const int Tc = (T - c0) < kChunk ? (T - c0) : kChunk;
        RouteParams rp{};
        rp.x = reinterpret_cast<const uint16_t *>(x) + (size_t)c0 * dims->d;
        rp.Tc = Tc;
        rp.wr = w_router;
        rp.bias = bias;
        rp.d = dims->d;
        rp.E = dims->n_experts;
        rp.k = dims->top_k;
        rp.ws = reinterpret_cast<uint8_t *>(ws);
        rp.L = L;
        rp.blobs = nullptr;
        rp.route_flags = route_flags(dims);
        rp.idx_out = idx + (size_t)c0 * dims->top_k;
        rp.w_out = weight + (size_t)c0 * dims->top_k;
        const int lst = one_launch(dims) ? layer_stages(*di, dims, Tc) : 0;
        cudaError_t e = lst > 0 ? launch_layer_route(*di, rp, lst, st, dims->ff % 512 == 0) : launch_route(*di, rp, st);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return K3MOE_OK;
}

k3moe_status k3moe_expert_ffn(const void *x, int32_t T, const uint8_t *blob,
                              const k3moe_dims *dims, void *out, void *ws, size_t ws_bytes,
                              void *stream) {
    k3moe_status s = check_dims(dims);
    if (s != K3MOE_OK) return s;
    if (T < 1 || !x || !aligned(x, 16) || !blob || !aligned(blob, 16) || !out || !aligned(out, 16))
        return K3MOE_ERR_INVALID_ARGUMENT;
    if (!ws || !aligned(ws, 256)) return K3MOE_ERR_INVALID_ARGUMENT;
    if (ws_bytes < layout_for(dims, dims->top_k).total) return K3MOE_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo *di = nullptr;
    s = device_info(&di);
    if (s != K3MOE_OK) return s;
    const Layout L = layout_for(dims, dims->top_k);  // the layer's layout: one workspace serves every call
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *wsb = reinterpret_cast<uint8_t *>(ws);
    const int d = dims->d;
    const bool out32 = (dims->flags & K3MOE_OUT_FP32) != 0;
    uint4 tmpl[kTemplates][8];
    s = tmap_templates(d, dims->ff, ws, tmpl);
    if (s != K3MOE_OK) return s;
    for (int c0 = 0; c0 < T; c0 += kChunk) {
        const int Tc = (T - c0) < kChunk ? (T - c0) : kChunk;
        const uint16_t *xc = reinterpret_cast<const uint16_t *>(x) + (size_t)c0 * d;
        void *yc = reinterpret_cast<uint8_t *>(out) + (size_t)c0 * d * (out32 ? 4 : 2);
        SingleParams sp{};
        sp.x = xc;
        sp.Tc = Tc;
        sp.d = d;
        sp.blob = blob;
        sp.ws = wsb;
        sp.L = L;
        memcpy(sp.tmpl, tmpl, sizeof(tmpl));
        sp.scale_mask = (d % 512 == 0 ? 1 : 0) | (dims->ff % 512 == 0 ? 2 : 0);
        int nblk = (Tc * (d / 32) + 7) / 8;  // one warp per 32-element block
        if (nblk > di->sms) nblk = di->sms;
        cudaError_t e = launch(single_expert_setup_kernel, dim3(nblk), dim3(256), 0, st, false, sp);
        if (e != cudaSuccess) return cuda_fail(e, "setup launch");
        UmmaParams up{};
        up.Tc = Tc;
        up.d = d;
        up.ff = dims->ff;
        up.k = dims->top_k;
        up.ffs = 0;
        up.ws = wsb;
        up.L = L;
        up.out_fp32 = out32;
        up.y = yc;
        up.strict = (dims->flags & K3MOE_STRICT) != 0;
        e = launch_umma<true>(*di, up, st);
        if (e != cudaSuccess) return cuda_fail(e, "gate/up launch");
        e = launch_umma<false>(*di, up, st);
        if (e != cudaSuccess) return cuda_fail(e, "down launch");
    }
    return K3MOE_OK;
}

k3moe_status k3moe_layer(const void *x, int32_t T, const float *w_router, const float *bias,
                         const uint8_t *const *expert_blobs, const void *shared_wg,
                         const void *shared_wu, const void *shared_wd, const k3moe_dims *dims,
                         void *y, int32_t *idx_out, float *w_out, void *ws, size_t ws_bytes,
                         void *stream) {
    return layer_impl(x, T, w_router, bias, expert_blobs, shared_wg, shared_wu, shared_wd, dims, y,
                      idx_out, w_out, ws, ws_bytes, stream, nullptr, nullptr);
}

k3moe_status k3moe_layer_residual(const void *h, int32_t T, const void *norm_w, float eps,
                                  const float *w_router, const float *bias,
                                  const uint8_t *const *expert_blobs, const void *shared_wg,
                                  const void *shared_wu, const void *shared_wd, const k3moe_dims *dims,
                                  void *h_out, void *ws, size_t ws_bytes, void *stream) {
    if (!norm_w || !aligned(norm_w, 16) || !(eps >= 0.f) || !(eps < 1e30f)) return K3MOE_ERR_INVALID_ARGUMENT;
    return layer_impl(h, T, w_router, bias, expert_blobs, shared_wg, shared_wu, shared_wd, dims, h_out, nullptr,
                      nullptr, ws, ws_bytes, stream, nullptr, nullptr, nullptr,
                      reinterpret_cast<const uint16_t *>(norm_w), eps);
}

k3moe_status k3moe_layer_from_host(const void *x_host, int32_t T, const float *w_router,
                                   const float *bias, const uint8_t *const *expert_blobs,
                                   const void *shared_wg, const void *shared_wu,
                                   const void *shared_wd, const k3moe_dims *dims, void *y_host,
                                   void *ws, size_t ws_bytes, void *stream) {
    if (!x_host) return K3MOE_ERR_INVALID_ARGUMENT;
    return layer_impl(nullptr, T, w_router, bias, expert_blobs, shared_wg, shared_wu, shared_wd,
                      dims, nullptr, nullptr, nullptr, ws, ws_bytes, stream, x_host, y_host);
}

k3moe_status k3moe_layer_timed(const void *x, int32_t T, const float *w_router, const float *bias,
                               const uint8_t *const *expert_blobs, const void *shared_wg,
                               const void *shared_wu, const void *shared_wd,
                               const k3moe_dims *dims, void *y, void *ws, size_t ws_bytes,
                               void *stream, void *const *events, int32_t n_events,
                               int32_t *n_kernels) {
    if (T > kChunk || !events || n_events < 1 || !n_kernels) return K3MOE_ERR_INVALID_ARGUMENT;
    for (int i = 0; i < n_events; ++i)
        if (!events[i]) return K3MOE_ERR_INVALID_ARGUMENT;
    EventHook hk;
    hk.ev = reinterpret_cast<cudaEvent_t *>(const_cast<void **>(events));
    hk.n = n_events;
    k3moe_status s = layer_impl(x, T, w_router, bias, expert_blobs, shared_wg, shared_wu,
                                shared_wd, dims, y, nullptr, nullptr, ws, ws_bytes, stream, nullptr,
                                nullptr, &hk);
    *n_kernels = hk.kernels;
    return s;
}

k3moe_status k3moe_layer_noalloc(const void *x, int32_t T, const float *w_router, const float *bias,
                                 const uint8_t *const *expert_blobs, const void *shared_wg,
                                 const void *shared_wu, const void *shared_wd,
                                 const k3moe_dims *dims, void *y, void *stream) {
    k3moe_status s = check_dims(dims);
    if (s != K3MOE_OK) return s;
    const size_t need = layout_for(dims, dims->top_k).total;
    if (need > kNoAllocBytes) {
        g_last_error = "k3moe_layer_noalloc: this shape needs " + std::to_string(need) +
                       " bytes of scratch, the built-in buffer holds " + std::to_string(kNoAllocBytes);
        return K3MOE_ERR_WORKSPACE_TOO_SMALL;
    }
    if (T < 1 || !x || !y || !aligned(x, 16) || !aligned(y, 16)) return K3MOE_ERR_INVALID_ARGUMENT;
    DeviceInfo *di = nullptr;
    s = device_info(&di);
    if (s != K3MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = nullptr;
    s = noalloc_scratch(*di, dims, st, &ws);
    if (s != K3MOE_OK) return s;
    // a workspace sized for one 8-token pass: any T runs as 8-token decode
    // passes (the grouped path's region would not fit in the buffer)
    return layer_impl(x, T, w_router, bias, expert_blobs, shared_wg, shared_wu, shared_wd, dims, y,
                      nullptr, nullptr, ws, need, stream, nullptr, nullptr);
}

size_t k3moe_cache_slot_bytes(const k3moe_dims *dims) {
    if (check_dims(dims) != K3MOE_OK) return 0;
    return align256((size_t)3 * dims->d * dims->ff * 17 / 32);
}

k3moe_status k3moe_cache_create(const k3moe_dims *dims, int32_t n_slots, void *slot_mem,
                                size_t slot_mem_bytes, const void *const *host_blobs,
                                k3moe_cache **cache) {
    if (!cache) return K3MOE_ERR_INVALID_ARGUMENT;
    *cache = nullptr;
    k3moe_status s = check_dims(dims);
    if (s != K3MOE_OK) return s;
    const size_t sb = k3moe_cache_slot_bytes(dims);
    if (n_slots < 1 || !slot_mem || !aligned(slot_mem, 256) || !host_blobs ||
        slot_mem_bytes < (size_t)n_slots * sb)
        return K3MOE_ERR_INVALID_ARGUMENT;
    for (int e = 0; e < dims->n_experts; ++e)
        if (!host_blobs[e]) return K3MOE_ERR_INVALID_ARGUMENT;
    k3moe_cache *c = new (std::nothrow) k3moe_cache;
    if (!c) return K3MOE_ERR_INVALID_ARGUMENT;
    ExpertCache &x = c->c;
    x.E = dims->n_experts;
    x.S = n_slots;
    x.blob_bytes = (size_t)3 * dims->d * dims->ff * 17 / 32;
    x.slot_bytes = sb;
    x.slots = reinterpret_cast<uint8_t *>(slot_mem);
    x.host.assign(host_blobs, host_blobs + x.E);
    x.slot_of.assign(x.E, -1);
    x.expert_of.assign(n_slots, -1);
    x.last.assign(n_slots, 0);
    x.stamp.assign(x.E, 0);
    *cache = c;
    return K3MOE_OK;
}

void k3moe_cache_destroy(k3moe_cache *cache) { delete cache; }

k3moe_status k3moe_cache_plan(k3moe_cache *cache, const int32_t *experts, int32_t n, int32_t *filled,
                              int32_t *n_filled) {
    if (!cache || (n > 0 && !experts) || n < 0 || !n_filled) return K3MOE_ERR_INVALID_ARGUMENT;
    if (!cache->c.plan(experts, n, cache->fe, cache->fs)) return K3MOE_ERR_INVALID_ARGUMENT;
    *n_filled = (int32_t)cache->fe.size();
    if (filled)
        for (size_t i = 0; i < cache->fe.size(); ++i) filled[i] = cache->fe[i];
    return K3MOE_OK;
}

k3moe_status k3moe_cache_fetch(k3moe_cache *cache, const int32_t *experts, int32_t n, void *ptr_table,
                               void *stream) {
    if (!cache || (n > 0 && !experts) || n < 0 || !ptr_table || !aligned(ptr_table, 8))
        return K3MOE_ERR_INVALID_ARGUMENT;
    ExpertCache &x = cache->c;
    if (!x.plan(experts, n, cache->fe, cache->fs)) return K3MOE_ERR_INVALID_ARGUMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    for (size_t i = 0; i < cache->fe.size(); ++i) {
        cudaError_t e = cudaMemcpyAsync(x.slots + (size_t)cache->fs[i] * x.slot_bytes, x.host[cache->fe[i]],
                                        x.blob_bytes, cudaMemcpyHostToDevice, st);
        if (e != cudaSuccess) return cuda_fail(e, "expert copy");
    }
    x.table(cache->table);
    cudaError_t e = cudaMemcpyAsync(ptr_table, cache->table.data(), (size_t)x.E * 8, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "pointer table copy");
    return K3MOE_OK;
}

k3moe_status k3moe_cache_get_stats(const k3moe_cache *cache, k3moe_cache_stats *stats) {
    if (!cache || !stats) return K3MOE_ERR_INVALID_ARGUMENT;
    stats->requests = cache->c.requests;
    stats->hits = cache->c.hits;
    stats->fills = cache->c.fills;
    stats->evictions = cache->c.evictions;
    return K3MOE_OK;
}

k3moe_status k3moe_layer_cached(k3moe_cache *cache, const void *x, int32_t T, const float *w_router,
                                const float *bias, void *ptr_table, const void *shared_wg,
                                const void *shared_wu, const void *shared_wd, const k3moe_dims *dims,
                                void *y, int32_t *idx_host, void *ws, size_t ws_bytes, void *stream) {
    k3moe_status s = check_dims(dims);
    if (s != K3MOE_OK) return s;
    if (!cache || !idx_host || T < 1 || !x || !aligned(x, 16) || !y || !aligned(y, 16) || !ws ||
        !aligned(ws, 256) || cache->c.E != dims->n_experts)
        return K3MOE_ERR_INVALID_ARGUMENT;
    const Layout L = layout_for(dims, dims->top_k);
    if (ws_bytes < L.total) return K3MOE_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo *di = nullptr;
    s = device_info(&di);
    if (s != K3MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int k = dims->top_k, d = dims->d;
    const size_t ybytes = (dims->flags & K3MOE_OUT_FP32) ? 4 : 2;
    for (int c0 = 0; c0 < T; c0 += kChunk) {
        const int Tc = (T - c0) < kChunk ? (T - c0) : kChunk;
        const uint16_t *xc = reinterpret_cast<const uint16_t *>(x) + (size_t)c0 * d;
        // 1. the routing of the pass, to the host
        RouteParams rp{};
        rp.x = xc;
        rp.Tc = Tc;
        rp.wr = w_router;
        rp.bias = bias;
        rp.d = d;
        rp.E = dims->n_experts;
        rp.k = k;
        rp.ws = reinterpret_cast<uint8_t *>(ws);
        rp.L = L;
        rp.route_flags = route_flags(dims);
        // the routing by the kernel the layer call will use, so the experts
        // fetched are exactly the ones its dispatch takes
        const int lst = one_launch(dims) ? layer_stages(*di, dims, Tc) : 0;
        cudaError_t e = lst > 0 ? launch_layer_route(*di, rp, lst, st, dims->ff % 512 == 0) : launch_route(*di, rp, st);
        if (e != cudaSuccess) return cuda_fail(e, "router launch");
        e = cudaMemcpyAsync(idx_host + (size_t)c0 * k, reinterpret_cast<uint8_t *>(ws) + L.idx,
                            (size_t)Tc * k * 4, cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e, "routing to host");
        // 2. its experts into the cache, 3. the layer on the cached experts
        s = k3moe_cache_fetch(cache, idx_host + (size_t)c0 * k, Tc * k, ptr_table, stream);
        if (s != K3MOE_OK) return s;
        s = layer_impl(xc, Tc, w_router, bias, reinterpret_cast<const uint8_t *const *>(ptr_table), shared_wg,
                       shared_wu, shared_wd, dims, reinterpret_cast<uint8_t *>(y) + (size_t)c0 * d * ybytes,
                       nullptr, nullptr, ws, L.total, stream, nullptr, nullptr, nullptr, nullptr, 0.f,
                       lst > 0 ? kLayerRouted : kLayerFull);
        if (s != K3MOE_OK) return s;
    }
    return K3MOE_OK;
}

k3moe_status k3moe_device_status(void *ws, void *stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (ws == nullptr) {
        // the built-in scratch of k3moe_layer_noalloc on the current device
        DeviceInfo *di = nullptr;
        k3moe_status s = device_info(&di);
        if (s != K3MOE_OK) return s;
        uint8_t *buf = nullptr;
        {
            std::lock_guard<std::mutex> lock(g_mu);
            s = noalloc_address(*di);
            if (s != K3MOE_OK) return s;
            buf = di->noalloc;
        }
        cudaError_t e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e);
        WsHeader h;
        e = cudaMemcpy(&h, buf, sizeof(h), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e);
        if (h.status & kStTimeout) {
            // a call gave up part-way: every counter in the buffer may be
            // raised, so the whole buffer starts again from zero
            e = cudaMemset(buf, 0, kNoAllocBytes);
            if (e == cudaSuccess) e = cudaDeviceSynchronize();
            if (e != cudaSuccess) return cuda_fail(e, "scratch clear");
            return K3MOE_ERR_DEVICE_TIMEOUT;
        }
        if (h.status != 0u) {
            const uint32_t zero = 0u;
            e = cudaMemcpy(buf, &zero, sizeof(zero), cudaMemcpyHostToDevice);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        return (h.status & kStDeviceCheck) ? K3MOE_ERR_DEVICE_CHECK : K3MOE_OK;
    }
    if (!aligned(ws, 256)) return K3MOE_ERR_INVALID_ARGUMENT;
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    WsHeader h;
    e = cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e);
    if (h.status != 0u) {
        // clear the status; after a timeout also restore the counters
        WsHeader z;
        memset(&z, 0, sizeof(z));
        z.n_unique = h.n_unique;
        e = cudaMemcpy(ws, &z, sizeof(z), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    if (h.status & kStTimeout) return K3MOE_ERR_DEVICE_TIMEOUT;
    if (h.status & kStDeviceCheck) return K3MOE_ERR_DEVICE_CHECK;
    return K3MOE_OK;
}

const char *k3moe_status_string(k3moe_status status) {
    switch (status) {
        case K3MOE_OK: return "ok";
        case K3MOE_ERR_INVALID_ARGUMENT: return "invalid argument";
        case K3MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case K3MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case K3MOE_ERR_CUDA: return "CUDA error";
        case K3MOE_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case K3MOE_ERR_DEVICE_CHECK: return "device-side argument check failed";
    }
    return "unknown status";
}

const char *k3moe_last_error(void) { return g_last_error.c_str(); }

k3moe_status k3moe_debug_set_fault(int32_t mode, uint64_t wait_limit_ns) {
    if (mode < 0 || mode > 1) return K3MOE_ERR_INVALID_ARGUMENT;
    g_fault_mode.store(mode, std::memory_order_relaxed);
    g_wait_ns.store(wait_limit_ns, std::memory_order_relaxed);
    return K3MOE_OK;
}

}  // extern "C"

// ttt_api.cu -- the C ABI of libttt_b200.so (declared in include/ttt.h).
//
// Host-side argument checks, workspace sizing, the choice between the tensor-core kernels
// and the general CUDA-core kernels, TMA descriptor encoding and kernel launches.  This is
// the library's only translation unit, so every kernel shares one device error word.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <algorithm>

#include <nvtx3/nvToolsExt.h>

#include "ttt.h"
#include "common.cuh"
#include "simt.cuh"
#include "linear_tc.cuh"
#include "linear_tc5.cuh"
#include "linear_bwd_tc.cuh"
#include "block_tc.cuh"
#include "dwconv_fused.cuh"
#include "apply_tc.cuh"
#include "chunked_tc.cuh"
#include "mlp_tc.cuh"

namespace {

std::atomic<unsigned long long> g_launches{0};

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    int sms = 0;
    int smem_per_sm = 0;
    int smem_optin = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_lock;

// A host-side NVTX range around one entry point's launches (profilers show each call as a
// named range; without a tool attached it costs a branch).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

int current_device(DeviceInfo** info) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TTT_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_dev_lock);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return TTT_ERR_CUDA;
        d.ready = true;
    }
    *info = &d;
    return TTT_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int launched(int n) {
    g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed);
    return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

dim3 grid_units(long long units, long long elems) {
    return dim3((unsigned)units, (unsigned)((elems + simt::TPB - 1) / simt::TPB));
}
bool grid_ok(long long units, long long elems) {
    return units >= 1 && units <= 0x7fffffffLL && (elems + simt::TPB - 1) / simt::TPB <= 65535;
}

// ------------------------------------------------------------------ TMA descriptors ----
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// bf16 tensor [U][N][d] viewed as 3-D (d fastest), box {d, box_rows, 1}
bool tmap_bf16_3d(CUtensorMap* m, const void* base, int d, int N, int U, int box_rows,
                  CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)U};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
    cuuint32_t box[3] = {(cuuint32_t)d, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ TTT-Linear --------
// 16-bit tensor [dim2][dim1][dim0] (dim0 fastest) viewed as 3-D, box {box0, box1, 1}
bool tmap_bf16_box(CUtensorMap* m, const void* base, int dim0, int dim1, int dim2, int box0, int box1,
                   CUtensorMapSwizzle sw, CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)dim0, (cuuint64_t)dim1, (cuuint64_t)dim2};
    cuuint64_t strides[2] = {(cuuint64_t)dim0 * 2, (cuuint64_t)dim1 * dim0 * 2};
    cuuint32_t box[3] = {(cuuint32_t)box0, (cuuint32_t)box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, type, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool linear_uses_tc(int d, int dtype) { return dtype == TTT_BF16 && (d == 32 || d == 64); }

template <typename T>
int linear_simt(const void* q, const void* k, const void* v, const float* w0, void* out, float* w_star, int B,
                int H, int N, int d, float eta, void* ws, cudaStream_t st) {
    const long long U = (long long)B * H;
    if (!grid_ok(U, 2LL * d * d) || !grid_ok(U, (long long)N * d)) return TTT_ERR_UNSUPPORTED;
    float* gc = static_cast<float*>(ws);
    float* wst = reinterpret_cast<float*>(static_cast<char*>(ws) + align256((size_t)U * 2 * d * d * 4));
    const float eta_over_n = (float)((double)eta / (double)N);
    simt::linear_gram<T><<<grid_units(U, 2LL * d * d), simt::TPB, 0, st>>>(
        static_cast<const T*>(k), static_cast<const T*>(v), gc, N, d);
    simt::linear_update<<<grid_units(U, (long long)d * d), simt::TPB, 0, st>>>(gc, w0, wst, w_star, H, d,
                                                                               eta_over_n);
    simt::linear_apply<T><<<grid_units(U, (long long)N * d), simt::TPB, 0, st>>>(
        static_cast<const T*>(q), wst, static_cast<T*>(out), N, d);
    return launched(3);
}

template <int D>
int linear_tc(const void* q, const void* k, const void* v, const float* w0, void* out, float* w_star, int B,
              int H, int N, float eta, cudaStream_t st) {
    using C = lintc::Cfg<D>;
    DeviceInfo* dev = nullptr;
    if (int rc = current_device(&dev)) return rc;
    const long long U = (long long)B * H;
    if (U > 65535) return TTT_ERR_UNSUPPORTED;

    // split each unit over S CTAs of one cluster so that the grid fills two CTAs per SM
    int S = 1;
    while (S < 8 && U * S < 2LL * dev->sms && (N + 2 * S - 1) / (2 * S) >= 16) S *= 2;
    const int t_cta = (N + S - 1) / S;
    const int tiles = (t_cta + lintc::TILE_ROWS - 1) / lintc::TILE_ROWS;
    const int stages = (D == 64) ? 2 : 4;
    static_assert(C::MIN_STAGES <= 2, "scratch must fit the ring");
    const int budget = dev->smem_per_sm / 2 - 1024;  // two CTAs per SM
    auto qbytes = [&](int qres, int tt) {
        const int rows = ((qres * tt + 15) / 16) * 16;
        return ((rows * C::ROWB + 1023) / 1024) * 1024;
    };
    auto fixed = [&](int qres) { return stages * C::SLOT_BYTES + 2 * C::WT_BYTES + 8 * (2 * stages + qres) + 1024; };
    int TT = ((t_cta + tiles - 1) / tiles + 7) / 8 * 8;
    int qres = tiles;
    while (qres > 0 && fixed(qres) + qbytes(qres, TT) > budget) --qres;
    if (qres < tiles) {  // some Q tiles stream through the ring: they need 16-row tiles
        TT = ((t_cta + tiles - 1) / tiles + 15) / 16 * 16;
        qres = tiles;
        while (qres > 0 && fixed(qres) + qbytes(qres, TT) > budget) --qres;
    }
    lintc::Params p;
    p.w0 = w0;
    p.w_star = w_star;
    p.H = H;
    p.N = N;
    p.TT = TT;
    p.tiles = tiles;
    p.T = TT * tiles;
    p.q_res = qres;
    p.stages = stages;
    p.q_region_bytes = qbytes(qres, TT);
    p.eta_over_n = (float)((double)eta / (double)N);
    const lintc::Layout<D> L(p);
    const int smem = (int)L.total + 1024;
    if (smem > dev->smem_optin) return TTT_ERR_UNSUPPORTED;

    const CUtensorMapSwizzle sw = (D == 64) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap tk, tv, tq, to;
    if (!tmap_bf16_3d(&tk, k, D, N, (int)U, TT, sw) || !tmap_bf16_3d(&tv, v, D, N, (int)U, TT, sw) ||
        !tmap_bf16_3d(&tq, q, D, N, (int)U, TT, sw) || !tmap_bf16_3d(&to, out, D, N, (int)U, 8, sw))
        return TTT_ERR_CUDA;

    auto kern = lintc::linear_tc_kernel<D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dev->smem_optin) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
        return TTT_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S, (unsigned)U, 1);
    cfg.blockDim = dim3(lintc::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tk, tv, tq, to, p) != cudaSuccess) return TTT_ERR_CUDA;
    return launched(1);
}

// d = 64: tcgen05 kernel (one cluster of S CTAs per unit, one CTA per SM, no workspace).
// dh < 64: each unit's 64 features are 64 / dh heads side by side, w0 is [64 / dh][dh][dh]
// (the block's core, whose Q, K, V are token-major [B, N, 64])
int linear_tc5(const void* q, const void* k, const void* v, const float* w0, void* out, float* w_star, int B, int H,
               int N, float eta, cudaStream_t st, int dh = 64) {
    DeviceInfo* dev = nullptr;
    if (int rc = current_device(&dev)) return rc;
    const long long U = (long long)B * H;
    if (U > 65535) return TTT_ERR_UNSUPPORTED;
    lin5::Params p;
    // split each unit over S CTAs while the grid stays within one CTA per SM, then pick the
    // tile height (multiple of 16, <= 128) that gives every CTA the same number of tiles
    const int t128 = (N + lin5::MT - 1) / lin5::MT;
    int S = 1;
    while (S < 8 && U * S * 2 <= dev->sms && S * 2 <= t128) S *= 2;
    const int per_cta = (N + S - 1) / S;
    const int k_tiles = (per_cta + lin5::MT - 1) / lin5::MT;
    p.TT = ((per_cta + k_tiles - 1) / k_tiles + 15) / 16 * 16;
    p.n_tiles = (N + p.TT - 1) / p.TT;
    const int extra = lin5::FIXED_BYTES + (int)sizeof(lin5::Bars) + 1024;  // + alignment slack
    p.slots = std::min(lin5::MAX_SLOTS, (dev->smem_optin - extra) / lin5::SLOT_BYTES);
    if (p.slots < 2) return TTT_ERR_UNSUPPORTED;
    p.nq = std::min(lin5::MAX_QT, p.slots * lin5::SLOT_BYTES / lin5::TILE_BYTES);
    p.w0 = w0;
    p.w_star = w_star;
    p.H = H;
    p.N = N;
    p.dh = dh;
    p.eta_over_n = (float)((double)eta / (double)N);
    // more than half an SM's shared memory: one CTA per SM, which owns all 512 TMEM columns
    const int smem = std::max(p.slots * lin5::SLOT_BYTES + extra, dev->smem_per_sm / 2 + 1024);
    if (smem > dev->smem_optin) return TTT_ERR_UNSUPPORTED;

    CUtensorMap tk, tv, tq, to;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!tmap_bf16_3d(&tk, k, 64, N, (int)U, p.TT, sw) || !tmap_bf16_3d(&tv, v, 64, N, (int)U, p.TT, sw) ||
        !tmap_bf16_3d(&tq, q, 64, N, (int)U, p.TT, sw) || !tmap_bf16_3d(&to, out, 64, N, (int)U, p.TT, sw))
        return TTT_ERR_CUDA;
    auto kern = lin5::linear_tc5_kernel;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dev->smem_optin) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
        return TTT_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S, (unsigned)U, 1);
    cfg.blockDim = dim3(lin5::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // the kernel may start while the previous grid on the stream finishes; it waits for that
    // grid (griddepcontrol.wait) before its first global memory access
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, tk, tv, tq, to, p) != cudaSuccess) return TTT_ERR_CUDA;
    return launched(1);
}

// ------------------------------------------------------------------ TTT-Linear backward
bool linear_bwd_tc_ok(int d, int dtype) { return dtype == TTT_BF16 && d == lbw::D; }

struct BwdPlan {
    int S, TT, n_tiles;
};
// token splits per unit (one CTA per SM) and equal tiles of TT <= 128 rows, as in the forward
BwdPlan bwd_plan(long long U, int N, int sms) {
    BwdPlan b;
    const int t128 = (N + lbw::MT - 1) / lbw::MT;
    b.S = 1;
    while (b.S < 8 && U * b.S * 2 <= sms && b.S * 2 <= t128) b.S *= 2;
    const int per_cta = (N + b.S - 1) / b.S;
    const int k_tiles = (per_cta + lbw::MT - 1) / lbw::MT;
    b.TT = ((per_cta + k_tiles - 1) / k_tiles + 15) / 16 * 16;
    b.n_tiles = (N + b.TT - 1) / b.TT;
    return b;
}
size_t bwd_tc_ws(long long U, int S) {
    return align256((size_t)U * S * 3 * lbw::DD * 4) + align256((size_t)U * 8 * lbw::DD * 2) +
           align256((size_t)U * lbw::DD * 4);
}
size_t bwd_simt_ws(long long U, int d) {
    return align256((size_t)U * 3 * d * d * 4) + align256((size_t)U * 2 * d * d * 4) + align256((size_t)U * d * d * 4);
}

// Launch with programmatic dependent launch: the kernel may start while the previous grid on the
// stream finishes and waits for it (griddepcontrol.wait) before its first global memory access.
template <typename Kern, typename... Args>
int launch_pdl(Kern kern, dim3 grid, int threads, int smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t c = {};
    c.gridDim = grid;
    c.blockDim = dim3((unsigned)threads, 1, 1);
    c.dynamicSmemBytes = (size_t)smem;
    c.stream = st;
    cudaLaunchAttribute a[1];
    a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a[0].val.programmaticStreamSerializationAllowed = 1;
    c.attrs = a;
    c.numAttrs = 1;
    return cudaLaunchKernelEx(&c, kern, args...) == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

int linear_bwd_tc(const void* q, const void* k, const void* v, const float* w0, const void* g, void* dq, void* dk,
                  void* dv, float* dw0, int B, int H, int N, float eta, void* ws, cudaStream_t st) {
    DeviceInfo* dev = nullptr;
    if (int rc = current_device(&dev)) return rc;
    const long long U = (long long)B * H;
    if (U > 65535) return TTT_ERR_UNSUPPORTED;
    const BwdPlan pl = bwd_plan(U, N, dev->sms);
    if (lbw::r_smem_bytes() > dev->smem_optin || lbw::a_smem_bytes() > dev->smem_optin ||
        lbw::f_smem_bytes() > dev->smem_optin)
        return TTT_ERR_UNSUPPORTED;
    char* w = static_cast<char*>(ws);
    float* part = reinterpret_cast<float*>(w);
    w += align256((size_t)U * pl.S * 3 * lbw::DD * 4);
    __nv_bfloat16* ops = reinterpret_cast<__nv_bfloat16*>(w);
    w += align256((size_t)U * 8 * lbw::DD * 2);
    float* dw0u = reinterpret_cast<float*>(w);
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    CUtensorMap tv, tk, tq, tg, tops, tdq, tdk, tdv;
    if (!tmap_bf16_3d(&tv, v, 64, N, (int)U, pl.TT, sw) || !tmap_bf16_3d(&tk, k, 64, N, (int)U, pl.TT, sw) ||
        !tmap_bf16_3d(&tq, q, 64, N, (int)U, pl.TT, sw) || !tmap_bf16_3d(&tg, g, 64, N, (int)U, pl.TT, sw) ||
        !tmap_bf16_3d(&tdq, dq, 64, N, (int)U, pl.TT, sw) || !tmap_bf16_3d(&tdk, dk, 64, N, (int)U, pl.TT, sw) ||
        !tmap_bf16_3d(&tdv, dv, 64, N, (int)U, pl.TT, sw) ||
        !tmap_bf16_box(&tops, ops, 64, 8 * 64, (int)U, 64, 64, sw))
        return TTT_ERR_CUDA;
    if (cudaFuncSetAttribute(lbw::reduce_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, lbw::r_smem_bytes()) !=
            cudaSuccess ||
        cudaFuncSetAttribute(lbw::finish_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, lbw::f_smem_bytes()) !=
            cudaSuccess ||
        cudaFuncSetAttribute(lbw::apply_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, lbw::a_smem_bytes()) !=
            cudaSuccess)
        return TTT_ERR_CUDA;
    lbw::RParams rp;
    rp.part = part;
    rp.TT = pl.TT;
    rp.n_tiles = pl.n_tiles;
    // the four launches use programmatic dependent launch: each kernel requests its first input
    // tiles into L2 (where they are inputs of the call) and then waits for the previous grid
    auto pdl = [&](auto kern, dim3 grid, int threads, int smem, auto... args) {
        return launch_pdl(kern, grid, threads, smem, st, args...);
    };
    if (int rc = pdl(lbw::reduce_kernel, dim3(pl.S, (unsigned)U), lbw::R_THREADS, lbw::r_smem_bytes(), tv, tk, tq, tg, rp))
        return rc;
    lbw::FParams fp;
    fp.part = part;
    fp.w0 = w0;
    fp.ops = ops;
    fp.dw0u = dw0u;
    fp.H = H;
    fp.S = pl.S;
    fp.eta_over_n = (float)((double)eta / (double)N);
    if (int rc = pdl(lbw::finish_kernel, dim3((unsigned)U, 3), 256, lbw::f_smem_bytes(), fp)) return rc;
    lbw::AParams ap;
    ap.TT = pl.TT;
    ap.n_tiles = pl.n_tiles;
    if (int rc = pdl(lbw::apply_kernel, dim3(pl.S, (unsigned)U), lbw::A_THREADS, lbw::a_smem_bytes(), tops, tg, tk, tv,
                     tdq, tdk, tdv, ap))
        return rc;
    // the batch sum of dW0: 64-thread blocks, so that the 4096 elements spread over 64 SMs
    if (int rc = pdl(simt::linear_bwd_dw0, dim3((unsigned)H, (lbw::DD + 63) / 64), 64, 0, (const float*)dw0u, dw0, B, H,
                     lbw::D))
        return rc;
    return launched(4);
}

template <typename T>
int linear_bwd_simt(const void* q, const void* k, const void* v, const float* w0, const void* g, void* dq, void* dk,
                    void* dv, float* dw0, int B, int H, int N, int d, float eta, void* ws, cudaStream_t st) {
    const long long U = (long long)B * H;
    if (!grid_ok(U, 3LL * d * d) || !grid_ok(U, (long long)N * d) || !grid_ok(H, (long long)d * d))
        return TTT_ERR_UNSUPPORTED;
    char* w = static_cast<char*>(ws);
    float* gcm = reinterpret_cast<float*>(w);
    w += align256((size_t)U * 3 * d * d * 4);
    float* wsa = reinterpret_cast<float*>(w);
    w += align256((size_t)U * 2 * d * d * 4);
    float* dw0u = reinterpret_cast<float*>(w);
    const float eta_over_n = (float)((double)eta / (double)N);
    simt::linear_bwd_gram<T><<<grid_units(U, 3LL * d * d), simt::TPB, 0, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), static_cast<const T*>(g), gcm,
        N, d);
    simt::linear_bwd_finish<<<grid_units(U, (long long)d * d), simt::TPB, 0, st>>>(gcm, w0, wsa, dw0u, H, d,
                                                                                   eta_over_n);
    simt::linear_bwd_apply<T><<<grid_units(U, (long long)N * d), simt::TPB, 0, st>>>(
        static_cast<const T*>(k), static_cast<const T*>(v), static_cast<const T*>(g), gcm, wsa, static_cast<T*>(dq),
        static_cast<T*>(dk), static_cast<T*>(dv), N, d, eta_over_n);
    simt::linear_bwd_dw0<<<grid_units(H, (long long)d * d), simt::TPB, 0, st>>>(dw0u, dw0, B, H, d);
    return launched(4);
}

bool block_tc_ok(int C, int H, int Wg, int dtype) {
    return dtype == TTT_BF16 && C == blk::C && (C / H == 32 || C / H == 64) && C % H == 0 && Wg <= blk::MAX_WG;
}

int check_common(const void* q, const void* k, const void* v, const void* out, int dtype, float eta) {
    if (!q || !k || !v || !out) return TTT_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return TTT_ERR_INVALID_ARG;
    if (dtype != TTT_F32 && dtype != TTT_BF16) return TTT_ERR_INVALID_ARG;
    if (!std::isfinite(eta)) return TTT_ERR_INVALID_ARG;
    return TTT_OK;
}

// ------------------------------------------------------------------ depthwise conv ----
size_t dwconv_ws(int B, int Hg, int Wg, int C) {
    return align256((size_t)B * Hg * Wg * C * 4) + align256((size_t)B * C * 9 * 4);
}

// bf16 [B][Hg][Wg][C] viewed as 4-D (channels fastest), box {C, Wg, 1, 1}, no swizzle
bool tmap_bf16_rows(CUtensorMap* m, const void* base, int C, int Wg, int Hg, int B) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)Wg, (cuuint64_t)Hg, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)C * 2, (cuuint64_t)Wg * C * 2, (cuuint64_t)Hg * Wg * C * 2};
    cuuint32_t box[4] = {(cuuint32_t)C, (cuuint32_t)Wg, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool dwconv_fused_ok(int Hg, int Wg, int C, int dtype) {
    return dtype == TTT_BF16 && C == dwc::C && Wg <= 64 && Hg <= 8 * dwc::MAX_R;
}

int dwconv_fused(const void* q, const void* k, const void* v, const float* w0, void* out, float* w_star, int B,
                 int Hg, int Wg, float eta, cudaStream_t st) {
    DeviceInfo* dev = nullptr;
    if (int rc = current_device(&dev)) return rc;
    if (B > 65535) return TTT_ERR_UNSUPPORTED;
    // One cluster of S CTAs per image, one CTA per SM: S = 8 while the whole batch's 8-CTA
    // clusters fit on the GPU at once (15 of them on a 148-SM B200), else 4 (33 fit); more if
    // the rows per CTA would not fit, fewer for short grids (every CTA owns two rows or more).
    int S = 1;
    const int s_want = B <= 15 || (Hg + 3) / 4 > dwc::MAX_R ? 8 : 4;
    while (S < s_want && S * 2 <= Hg) S *= 2;
    dwc::Params p;
    p.R = (Hg + S - 1) / S;
    if (p.R > dwc::MAX_R) return TTT_ERR_UNSUPPORTED;
    p.cw = (Wg + dwc::PXW - 1) / dwc::PXW;
    p.nb = 2 * p.cw <= dwc::MAX_WARPS ? 2 : 1;
    p.slot_bytes = (dwc::PXW * p.cw + 2) * dwc::PXB;
    p.nslots = std::max(p.nb * (dwc::KS + dwc::VS), p.R + 2);
    p.w0 = w0;
    p.w_star = w_star;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.Hg = Hg;
    p.Wg = Wg;
    p.eta_over_n = (float)((double)eta / ((double)Hg * Wg));
    const int smem = p.nslots * p.slot_bytes + (2 + dwc::MAX_WARPS) * dwc::C * dwc::NTAP * 4 + (int)sizeof(dwc::Bars) + 128;
    if (smem > dev->smem_optin) return TTT_ERR_UNSUPPORTED;
    CUtensorMap tk, tv, tq;
    if (!tmap_bf16_rows(&tk, k, dwc::C, Wg, Hg, B) || !tmap_bf16_rows(&tv, v, dwc::C, Wg, Hg, B) ||
        !tmap_bf16_rows(&tq, q, dwc::C, Wg, Hg, B))
        return TTT_ERR_CUDA;
    auto kern = dwc::dwconv_kernel;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dev->smem_optin) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
        return TTT_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S, (unsigned)B, 1);
    cfg.blockDim = dim3((p.nb * p.cw + 1) * 32, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // programmatic dependent launch: the kernel waits for the previous grid (griddepcontrol.wait)
    // before its first global memory access
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, tk, tv, tq, p) != cudaSuccess) return TTT_ERR_CUDA;
    return launched(1);
}

template <typename T>
int dwconv_simt(const void* q, const void* k, const void* v, const float* w0, void* out, float* w_star, int B,
                int Hg, int Wg, int C, float eta, void* ws, cudaStream_t st) {
    const long long NC = (long long)Hg * Wg * C;
    if (!grid_ok(B, NC) || !grid_ok(B, 9LL * C)) return TTT_ERR_UNSUPPORTED;
    float* r = static_cast<float*>(ws);
    float* wst = reinterpret_cast<float*>(static_cast<char*>(ws) + align256((size_t)B * NC * 4));
    const float eta_over_n = (float)((double)eta / ((double)Hg * Wg));
    simt::dwconv_residual<T><<<grid_units(B, NC), simt::TPB, 0, st>>>(
        static_cast<const T*>(k), static_cast<const T*>(v), w0, r, Hg, Wg, C);
    simt::dwconv_update<T><<<grid_units(B, 9LL * C), simt::TPB, 0, st>>>(static_cast<const T*>(k), r, w0, wst,
                                                                         w_star, Hg, Wg, C, eta_over_n);
    simt::dwconv_apply<T><<<grid_units(B, NC), simt::TPB, 0, st>>>(static_cast<const T*>(q), wst,
                                                                  static_cast<T*>(out), Hg, Wg, C);
    return launched(3);
}

// ------------------------------------------------------------------ TTT-MLP -----------
size_t mlp_ws(int B, int H, int N, int d, int hd) {
    const size_t U = (size_t)B * H;
    return 2 * align256(U * N * hd * 4) + align256(U * N * d * 4) + 2 * align256(U * d * hd * 4);
}

template <typename T>
int mlp_simt(const void* q, const void* k, const void* v, const float* w1, const float* w2, void* out,
             float* w1_star, float* w2_star, int B, int H, int N, int d, int hd, float eta, void* ws,
             cudaStream_t st) {
    const long long U = (long long)B * H;
    if (!grid_ok(U, (long long)N * hd) || !grid_ok(U, (long long)N * d) || !grid_ok(U, (long long)d * hd))
        return TTT_ERR_UNSUPPORTED;
    char* w = static_cast<char*>(ws);
    float* A = reinterpret_cast<float*>(w);
    w += align256((size_t)U * N * hd * 4);
    float* GP = reinterpret_cast<float*>(w);
    w += align256((size_t)U * N * hd * 4);
    float* R = reinterpret_cast<float*>(w);
    w += align256((size_t)U * N * d * 4);
    float* W1s = reinterpret_cast<float*>(w);
    w += align256((size_t)U * d * hd * 4);
    float* W2s = reinterpret_cast<float*>(w);
    const float eta_over_n = (float)((double)eta / (double)N);
    const T* qq = static_cast<const T*>(q);
    const T* kk = static_cast<const T*>(k);
    const T* vv = static_cast<const T*>(v);
    simt::mlp_hidden<T><<<grid_units(U, (long long)N * hd), simt::TPB, 0, st>>>(kk, w1, A, GP, H, N, d, hd, 0);
    simt::mlp_out<T, false><<<grid_units(U, (long long)N * d), simt::TPB, 0, st>>>(A, w2, vv, R, nullptr, H, N,
                                                                                  d, hd, 0);
    simt::mlp_dz<<<grid_units(U, (long long)N * hd), simt::TPB, 0, st>>>(R, w2, GP, H, N, d, hd);
    simt::mlp_update_w1<T><<<grid_units(U, (long long)d * hd), simt::TPB, 0, st>>>(kk, GP, w1, W1s, w1_star, H, N,
                                                                                  d, hd, eta_over_n);
    simt::mlp_update_w2<<<grid_units(U, (long long)d * hd), simt::TPB, 0, st>>>(A, R, w2, W2s, w2_star, H, N, d,
                                                                               hd, eta_over_n);
    simt::mlp_hidden<T><<<grid_units(U, (long long)N * hd), simt::TPB, 0, st>>>(qq, W1s, A, nullptr, H, N, d, hd,
                                                                               1);
    simt::mlp_out<T, true><<<grid_units(U, (long long)N * d), simt::TPB, 0, st>>>(A, W2s, nullptr, nullptr,
                                                                                 static_cast<T*>(out), H, N, d,
                                                                                 hd, 1);
    return launched(7);
}

// tcgen05 TTT-MLP (bf16, d = 64, hidden = 256): grad -> update -> apply
bool mlp_tc_ok(int B, int H, int d, int hidden, int dtype) {
    return dtype == TTT_BF16 && d == mlp::D && hidden == mlp::HID && (long long)B * H <= 65535;
}
int mlp_splits(long long U, int N, int sms) {
    // token splits per unit: fill whole waves of one CTA per SM, at least two tiles per CTA
    int best = 1;
    double best_eff = 0.0;
    const int max_s = std::max(1, std::min(8, (N + 2 * mlp::MT - 1) / (2 * mlp::MT)));
    for (int S = 1; S <= max_s; ++S) {
        const long long ctas = U * S;
        const long long waves = (ctas + sms - 1) / sms;
        const double eff = (double)ctas / (double)(waves * sms);
        if (eff > best_eff + 1e-9) {
            best_eff = eff;
            best = S;
        }
    }
    return best;
}
size_t mlp_tc_ws(int B, int H, int N) {
    DeviceInfo* dev = nullptr;
    const int sms = current_device(&dev) == TTT_OK ? dev->sms : 148;
    const long long U = (long long)B * H;
    const int S = mlp_splits(U, N, sms);
    return align256((size_t)U * S * 2 * mlp::HID * mlp::D * 4) + align256((size_t)U * 2 * mlp::D * mlp::HID * 2) +
           align256((size_t)U * mlp::D * mlp::HID * 2) + 2 * align256((size_t)H * mlp::D * mlp::HID * 2);
}

int mlp_tc(const void* q, const void* k, const void* v, const float* w1, const float* w2, void* out,
           float* w1_star, float* w2_star, int B, int H, int N, float eta, void* ws, cudaStream_t st) {
    DeviceInfo* dev = nullptr;
    if (int rc = current_device(&dev)) return rc;
    const int U = B * H;
    const int S = mlp_splits(U, N, dev->sms);
    const int T = ((N + S - 1) / S + mlp::MT - 1) / mlp::MT * mlp::MT;
    char* w = static_cast<char*>(ws);
    float* part = reinterpret_cast<float*>(w);
    w += align256((size_t)U * S * 2 * mlp::HID * mlp::D * 4);
    __nv_bfloat16* w1b = reinterpret_cast<__nv_bfloat16*>(w);  // W1* hi and lo per unit
    w += align256((size_t)U * 2 * mlp::D * mlp::HID * 2);
    __half* w2h16 = reinterpret_cast<__half*>(w);               // W2* in fp16
    w += align256((size_t)U * mlp::D * mlp::HID * 2);
    __nv_bfloat16* w1h = reinterpret_cast<__nv_bfloat16*>(w);   // W1, W2 of every head in bf16
    w += align256((size_t)H * mlp::D * mlp::HID * 2);
    __nv_bfloat16* w2h = reinterpret_cast<__nv_bfloat16*>(w);

    CUtensorMap tk, tq, to, tw1h, tw2h, tw1s, tw2s;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!tmap_bf16_3d(&tk, k, 64, N, U, mlp::MT, sw) || !tmap_bf16_3d(&tq, q, 64, N, U, mlp::MT, sw) ||
        !tmap_bf16_3d(&to, out, 64, N, U, 32, sw) ||
        !tmap_bf16_box(&tw1h, w1h, mlp::HID, mlp::D, H, 64, 64, sw) ||
        !tmap_bf16_box(&tw2h, w2h, mlp::D, mlp::HID, H, 64, mlp::HID, sw) ||
        !tmap_bf16_box(&tw1s, w1b, mlp::HID, 2 * mlp::D, U, 64, 64, sw) ||
        !tmap_bf16_box(&tw2s, w2h16, mlp::D, mlp::HID, U, 64, mlp::HID, sw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
        return TTT_ERR_CUDA;
    const int smem_g = 2 * mlp::WBYTES + 2 * mlp::BIG + 2 * mlp::TILE + (int)sizeof(mlp::GradBars) + 1024;
    const int smem_a = 3 * mlp::WBYTES + mlp::BIG + mlp::NQB * mlp::TILE + (int)sizeof(mlp::ApplyBars) + 1024;
    if (smem_g > dev->smem_optin || smem_a > dev->smem_optin) return TTT_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(mlp::grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_g) != cudaSuccess ||
        cudaFuncSetAttribute(mlp::apply_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_a) != cudaSuccess)
        return TTT_ERR_CUDA;
    const int n8 = H * mlp::D * mlp::HID * 2 / 8;  // 8-element groups of W1 and W2
    mlp::prep_kernel<<<(n8 + 255) / 256, 256, 0, st>>>(w1, w2, w1h, w2h, n8);
    mlp::GradParams gp;
    gp.v = static_cast<const __nv_bfloat16*>(v);
    gp.part = part;
    gp.H = H;
    gp.N = N;
    gp.T = T;
    mlp::grad_kernel<<<dim3(S, U), mlp::THREADS, smem_g, st>>>(tk, tw1h, tw2h, gp);
    mlp::UpdateParams up;
    up.w1 = w1;
    up.w2 = w2;
    up.part = part;
    up.w1_star = w1_star;
    up.w2_star = w2_star;
    up.w1b = w1b;
    up.w2h = w2h16;
    up.H = H;
    up.S = S;
    up.eta_over_n = (float)((double)eta / (double)N);
    mlp::update_kernel<<<dim3(U, mlp::HID / 64), 256, 0, st>>>(up);
    mlp::ApplyParams ap;
    ap.N = N;
    ap.T = T;
    mlp::apply_kernel<<<dim3(S, U), mlp::THREADS, smem_a, st>>>(tq, to, tw1s, tw2s, ap);
    return launched(4);
}

// ------------------------------------------------------------------ chunked scan ------
// direction: 0 both scans summed, +1 raster only, -1 reverse raster only
int n_dirs(int direction) { return direction == 0 ? 2 : 1; }
size_t chunked_ws(int B, int H, int N, int d, int direction) {
    return align256((size_t)n_dirs(direction) * B * H * N * d * 4);
}

bool chunked_tc_ok(int B, int H, int d, int chunk, int dtype) {
    return dtype == TTT_BF16 && d == chk::D && chunk == chk::CB && (long long)B * H <= 65535;
}
size_t chunked_tc_ws(int B, int H, int N, int direction) {
    return direction == 0 ? align256((size_t)B * H * N * chk::D * 4) : 0;  // parked partials
}

int chunked_tc(const void* q, const void* k, const void* v, const float* w0, void* out, int B, int H, int N,
               float eta, int direction, void* ws, cudaStream_t st, int epochs = 0, float* wfin = nullptr,
               float* wout = nullptr) {
    DeviceInfo* dev = nullptr;
    if (int rc = current_device(&dev)) return rc;
    const int U = B * H;
    chk::Params p;
    p.w0 = w0;
    p.park = static_cast<float*>(ws);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.H = H;
    p.N = N;
    p.nc = N / chk::CB;
    p.both = direction == 0 ? 1 : 0;
    p.dir = direction < 0 ? 1 : 0;
    p.steps = wfin ? epochs * p.nc : p.nc;  // training mode: epochs over the chunks, no output
    p.wfin = wfin;
    p.wout = wout;
    p.eta_over_b = (float)((double)eta / (double)chk::CB);
    const int smem = 2 * chk::STAGES * chk::STAGE + 2 * chk::WBUF * chk::WFR + 2 * (chk::PF + 1) * chk::PKB +
                     (int)sizeof(chk::Bars) + 1024;
    if (smem > dev->smem_optin) return TTT_ERR_UNSUPPORTED;
    CUtensorMap tk, tq, tv, tp;
    if (!tmap_bf16_3d(&tk, k, 64, N, U, chk::CB, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tmap_bf16_3d(&tq, q, 64, N, U, chk::CB, CU_TENSOR_MAP_SWIZZLE_128B))
        return TTT_ERR_CUDA;
    {   // V: box of 16 columns x 64 tokens, no swizzle
        auto fn = encode_fn();
        if (!fn) return TTT_ERR_CUDA;
        cuuint64_t dims[3] = {64, (cuuint64_t)N, (cuuint64_t)U};
        cuuint64_t strides[2] = {128, (cuuint64_t)N * 128};
        cuuint32_t box[3] = {chk::NCOL, chk::CB, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        if (fn(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(v), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return TTT_ERR_CUDA;
        // parked partials (fp32 [U][N][64]): box of 16 columns x 32 tokens (one output warp's
        // half of a chunk), no swizzle (a one-way scan parks nothing and never uses this map; it
        // is encoded over `out` then)
        cuuint64_t pstrides[2] = {256, (cuuint64_t)N * 256};
        cuuint32_t pbox[3] = {chk::NCOL, chk::CB / 2, 1};
        void* pbase = ws ? ws : out;
        if (fn(&tp, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, pbase, dims, pstrides, pbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return TTT_ERR_CUDA;
    }
    auto kern = chk::chunked_kernel;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return TTT_ERR_CUDA;
    kern<<<dim3(chk::GROUPS, U), chk::THREADS, smem, st>>>(tk, tq, tv, tp, p);
    return launched(1);
}

template <typename T>
int chunked_simt(const void* q, const void* k, const void* v, const float* w0, void* out, int B, int H, int N,
                 int d, int chunk, float eta, int direction, void* ws, cudaStream_t st) {
    DeviceInfo* dev = nullptr;
    if (int rc = current_device(&dev)) return rc;
    const long long U = (long long)B * H;
    const long long total = U * N * d;
    if (U > 0x7fffffffLL || (total + simt::TPB - 1) / simt::TPB > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
    const int smem = (2 * d * d + simt::CH_RB * d) * 4;
    if (smem > dev->smem_optin) return TTT_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(simt::chunked_scan<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
        return TTT_ERR_CUDA;
    float* op = static_cast<float*>(ws);
    const float eta_over_b = (float)((double)eta / (double)chunk);
    simt::chunked_scan<T><<<dim3((unsigned)U, n_dirs(direction)), simt::TPB, smem, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), w0, op, H, N, d, chunk,
        eta_over_b, direction < 0 ? 1 : 0);
    simt::chunked_combine<T><<<(unsigned)((total + simt::TPB - 1) / simt::TPB), simt::TPB, 0, st>>>(
        op, static_cast<T*>(out), total, n_dirs(direction));
    return launched(2);
}

// ------------------------------------------------------------------ no-allocation scan ---
// Scratch for ttt_linear_chunked_bidir_noalloc: a fixed array in this library's device image,
// so that callers who may not allocate device memory can still run the scan.  Each device
// that loads the library holds it until the process exits.  Its device address is looked up
// once per device (host code cannot use the symbol itself: on the host it names a stand-in).
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_scratch_addr[kMaxDevices];
std::mutex g_noalloc_lock;

int noalloc_scratch(void** addr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TTT_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_noalloc_lock);
    if (!g_noalloc_scratch_addr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return TTT_ERR_CUDA;
        g_noalloc_scratch_addr[dev] = ptr;
    }
    *addr = g_noalloc_scratch_addr[dev];
    return TTT_OK;
}

}  // namespace

// ====================================================================== C ABI ==========
extern "C" {

const char* ttt_status_string(int status) {
    switch (status) {
        case TTT_OK: return "ok";
        case TTT_ERR_INVALID_ARG: return "invalid argument";
        case TTT_ERR_UNSUPPORTED: return "unsupported size";
        case TTT_ERR_WORKSPACE: return "workspace too small";
        case TTT_ERR_CUDA: return "CUDA error";
        case TTT_ERR_TIMEOUT: return "a device-side wait timed out";
        default: return "unknown status";
    }
}

int ttt_version(void) { return 100; }

unsigned long long ttt_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int ttt_device_error(unsigned int* bits) {
    unsigned int v = 0, zero = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return TTT_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g_ttt_device_error, sizeof(v)) != cudaSuccess) return TTT_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_ttt_device_error, &zero, sizeof(zero)) != cudaSuccess) return TTT_ERR_CUDA;
    if (bits) *bits = v;
    if (v & (TTT_DEVERR_TIMEOUT_TMA | TTT_DEVERR_TIMEOUT_PEER)) return TTT_ERR_TIMEOUT;
    return v ? TTT_ERR_CUDA : TTT_OK;
}

int ttt_debug_set_wait_limit(long long cycles) {
    const long long v = cycles > 0 ? cycles : (long long)TTT_SPIN_LIMIT_CYCLES;
    return cudaMemcpyToSymbol(g_ttt_wait_limit, &v, sizeof(v)) == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

int ttt_debug_arm_fault(unsigned int bits) {
    return cudaMemcpyToSymbol(g_ttt_fault, &bits, sizeof(bits)) == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

// ------------------------------------------------------------------ TTT-Linear --------
size_t ttt_linear_fullbatch_workspace_bytes(int B, int H, int N, int d, int dtype) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 0;
    if (linear_uses_tc(d, dtype)) return 0;
    const size_t U = (size_t)B * H;
    return align256(U * 2 * d * d * 4) + align256(U * d * d * 4);
}

int ttt_linear_fullbatch(const void* q, const void* k, const void* v, const float* w0, void* out, float* w_star,
                         int B, int H, int N, int d, float eta, int dtype, void* workspace,
                         size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("ttt_linear_fullbatch");
    if (int rc = check_common(q, k, v, out, dtype, eta)) return rc;
    if (!w0 || !aligned16(w0) || (w_star && !aligned16(w_star))) return TTT_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return TTT_ERR_INVALID_ARG;
    if (d > 128) return TTT_ERR_UNSUPPORTED;
    const size_t need = ttt_linear_fullbatch_workspace_bytes(B, H, N, d, dtype);
    if (workspace_bytes < need || (need && !workspace)) return TTT_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return TTT_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == TTT_BF16) {
        if (d == 64) return linear_tc5(q, k, v, w0, out, w_star, B, H, N, eta, st);
        if (d == 32) return linear_tc<32>(q, k, v, w0, out, w_star, B, H, N, eta, st);
        return linear_simt<__nv_bfloat16>(q, k, v, w0, out, w_star, B, H, N, d, eta, workspace, st);
    }
    return linear_simt<float>(q, k, v, w0, out, w_star, B, H, N, d, eta, workspace, st);
}

// ------------------------------------------------------------------ the ViT^3 block -----
size_t ttt_vit3_block_workspace_bytes(int B, int Hg, int Wg, int C, int H, int dtype) {
    if (B <= 0 || Hg <= 0 || Wg <= 0 || C <= 0 || H <= 0 || C % H != 0) return 0;
    const long long N = (long long)Hg * Wg;
    if (N > 0x7fffffffLL) return 0;
    const size_t es = dtype == TTT_BF16 ? 2 : 4;
    const size_t t = align256((size_t)B * N * C * es);
    const size_t core = ttt_linear_fullbatch_workspace_bytes(B, H, (int)N, C / H, dtype);
    const size_t z = block_tc_ok(C, H, Wg, dtype) ? 0 : align256((size_t)B * N * 2 * C * 4);
    return 5 * t + core + z;
}

int ttt_vit3_block(const void* x, const void* wqkvg, const float* w0, const float* wc, const void* wo, void* y,
                   int B, int Hg, int Wg, int C, int H, float eta, int dtype, void* workspace,
                   size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("ttt_vit3_block");
    if (!x || !wqkvg || !w0 || !wc || !wo || !y) return TTT_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(wqkvg) || !aligned16(w0) || !aligned16(wc) || !aligned16(wo) || !aligned16(y))
        return TTT_ERR_INVALID_ARG;
    if (dtype != TTT_F32 && dtype != TTT_BF16) return TTT_ERR_INVALID_ARG;
    if (!std::isfinite(eta)) return TTT_ERR_INVALID_ARG;
    if (B <= 0 || Hg <= 0 || Wg <= 0 || C <= 0 || H <= 0 || C % H != 0) return TTT_ERR_INVALID_ARG;
    const long long N = (long long)Hg * Wg;
    if (N > 0x7fffffffLL || C / H > 128 || C > 1024) return TTT_ERR_UNSUPPORTED;
    const size_t need = ttt_vit3_block_workspace_bytes(B, Hg, Wg, C, H, dtype);
    if (workspace_bytes < need || !workspace) return TTT_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return TTT_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long rows = (long long)B * N;
    const int d = C / H;
    const size_t es = dtype == TTT_BF16 ? 2 : 4;
    const size_t t = align256((size_t)rows * C * es);
    char* w = static_cast<char*>(workspace);
    void *q = w, *k = w + t, *v = w + 2 * t, *g = w + 3 * t, *o = w + 4 * t;
    void* core = w + 5 * t;
    const size_t core_bytes = ttt_linear_fullbatch_workspace_bytes(B, H, (int)N, d, dtype);
    if (block_tc_ok(C, H, Wg, dtype)) {
        DeviceInfo* dev = nullptr;
        if (int rc = current_device(&dev)) return rc;
        if (blk::p_smem_bytes() > dev->smem_optin || blk::o_smem_bytes() > dev->smem_optin) return TTT_ERR_UNSUPPORTED;
        if ((rows + blk::MT - 1) / blk::MT > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
        const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
        CUtensorMap tx, tw, two, txw, tq, tk, tv, tg;
        if (!tmap_bf16_3d(&tx, x, blk::C, (int)rows, 1, blk::MT, sw) ||
            !tmap_bf16_3d(&tq, q, blk::C, (int)rows, 1, blk::MT, sw) || !tmap_bf16_3d(&tk, k, blk::C, (int)rows, 1, blk::MT, sw) ||
            !tmap_bf16_3d(&tv, v, blk::C, (int)rows, 1, blk::MT, sw) || !tmap_bf16_3d(&tg, g, blk::C, (int)rows, 1, blk::MT, sw) ||
            !tmap_bf16_3d(&txw, x, blk::C, (int)rows, 1, blk::XW, sw) ||
            !tmap_bf16_box(&tw, wqkvg, 4 * blk::C, blk::C, 1, 64, 64, sw) ||
            !tmap_bf16_box(&two, wo, blk::C, 2 * blk::C, 1, 64, 2 * blk::C, sw))
            return TTT_ERR_CUDA;
        if (cudaFuncSetAttribute(blk::proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, blk::p_smem_bytes()) !=
                cudaSuccess ||
            cudaFuncSetAttribute(blk::out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, blk::o_smem_bytes()) !=
                cudaSuccess)
            return TTT_ERR_CUDA;
        const unsigned tiles = (unsigned)((rows + blk::MT - 1) / blk::MT);
        blk::PParams pp;
        pp.rows = rows;
        // persistent: one CTA per SM (at most), each looping over its tiles
        // programmatic dependent launch (proj and out): each kernel waits for the previous grid
        // (griddepcontrol.wait) before its first global memory access
        cudaLaunchAttribute pdl[1];
        pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        pdl[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t pc = {};
        pc.gridDim = dim3(std::min<unsigned>(tiles, (unsigned)dev->sms), 1, 1);
        pc.blockDim = dim3(blk::THREADS, 1, 1);
        pc.dynamicSmemBytes = blk::p_smem_bytes();
        pc.stream = st;
        pc.attrs = pdl;
        pc.numAttrs = 1;
        if (cudaLaunchKernelEx(&pc, blk::proj_kernel, tx, tw, tq, tk, tv, tg, pp) != cudaSuccess) return TTT_ERR_CUDA;
        if (int rc = launched(1)) return rc;
        // the core: each image is one unit of 64 features (the heads side by side, token-major),
        // W0 block-diagonal from the heads' w0
        if (int rc = linear_tc5(q, k, v, w0, o, nullptr, B, 1, (int)N, eta, st, d)) return rc;
        blk::OParams op;
        op.x = static_cast<const __nv_bfloat16*>(x);
        op.o = static_cast<const __nv_bfloat16*>(o);
        op.g = static_cast<const __nv_bfloat16*>(g);
        op.wc = wc;
        op.y = static_cast<__nv_bfloat16*>(y);
        op.rows = rows;
        op.N = (int)N;
        op.Hg = Hg;
        op.Wg = Wg;
        // persistent: one CTA per SM (at most), each looping over its tiles
        cudaLaunchConfig_t oc = pc;
        oc.blockDim = dim3(blk::O_THREADS, 1, 1);
        oc.dynamicSmemBytes = blk::o_smem_bytes();
        if (cudaLaunchKernelEx(&oc, blk::out_kernel, two, txw, op) != cudaSuccess) return TTT_ERR_CUDA;
        return launched(1);
    }
    float* z = reinterpret_cast<float*>(static_cast<char*>(core) + core_bytes);
    auto blocks = [](long long n) { return (unsigned)((n + simt::TPB - 1) / simt::TPB); };
    if ((rows * 4 * C + simt::TPB - 1) / simt::TPB > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
    if (dtype == TTT_BF16) {
        using T = __nv_bfloat16;
        simt::block_proj<T><<<blocks(rows * 4 * C), simt::TPB, 0, st>>>(
            static_cast<const T*>(x), static_cast<const T*>(wqkvg), static_cast<T*>(q), static_cast<T*>(k),
            static_cast<T*>(v), static_cast<T*>(g), rows, (int)N, C, H);
    } else {
        using T = float;
        simt::block_proj<T><<<blocks(rows * 4 * C), simt::TPB, 0, st>>>(
            static_cast<const T*>(x), static_cast<const T*>(wqkvg), static_cast<T*>(q), static_cast<T*>(k),
            static_cast<T*>(v), static_cast<T*>(g), rows, (int)N, C, H);
    }
    if (int rc = launched(1)) return rc;
    if (int rc = ttt_linear_fullbatch(q, k, v, w0, o, nullptr, B, H, (int)N, d, eta, dtype, core, core_bytes, stream))
        return rc;
    if (dtype == TTT_BF16) {
        using T = __nv_bfloat16;
        simt::block_z<T><<<blocks(rows * 2 * C), simt::TPB, 0, st>>>(static_cast<const T*>(x), static_cast<const T*>(o),
                                                                     static_cast<const T*>(g), wc, z, rows, (int)N,
                                                                     Hg, Wg, C, H);
        simt::block_outproj<T><<<blocks(rows * C), simt::TPB, 0, st>>>(z, static_cast<const T*>(wo),
                                                                       static_cast<T*>(y), rows, C);
    } else {
        using T = float;
        simt::block_z<T><<<blocks(rows * 2 * C), simt::TPB, 0, st>>>(static_cast<const T*>(x), static_cast<const T*>(o),
                                                                     static_cast<const T*>(g), wc, z, rows, (int)N,
                                                                     Hg, Wg, C, H);
        simt::block_outproj<T><<<blocks(rows * C), simt::TPB, 0, st>>>(z, static_cast<const T*>(wo),
                                                                       static_cast<T*>(y), rows, C);
    }
    return launched(2);
}

// ------------------------------------------------------------------ TTT-Linear backward
size_t ttt_linear_fullbatch_bwd_workspace_bytes(int B, int H, int N, int d, int dtype) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 0;
    const long long U = (long long)B * H;
    if (linear_bwd_tc_ok(d, dtype)) {
        DeviceInfo* dev = nullptr;
        const int sms = current_device(&dev) == TTT_OK ? dev->sms : 148;
        return bwd_tc_ws(U, bwd_plan(U, N, sms).S);
    }
    return bwd_simt_ws(U, d);
}

int ttt_linear_fullbatch_bwd(const void* q, const void* k, const void* v, const float* w0, const void* dout,
                             void* dq, void* dk, void* dv, float* dw0, int B, int H, int N, int d, float eta,
                             int dtype, void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("ttt_linear_fullbatch_bwd");
    if (int rc = check_common(q, k, v, dout, dtype, eta)) return rc;
    if (!dq || !dk || !dv || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return TTT_ERR_INVALID_ARG;
    if (!w0 || !dw0 || !aligned16(w0) || !aligned16(dw0)) return TTT_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return TTT_ERR_INVALID_ARG;
    if (d > 128) return TTT_ERR_UNSUPPORTED;
    const size_t need = ttt_linear_fullbatch_bwd_workspace_bytes(B, H, N, d, dtype);
    if (workspace_bytes < need || !workspace) return TTT_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return TTT_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (linear_bwd_tc_ok(d, dtype))
        return linear_bwd_tc(q, k, v, w0, dout, dq, dk, dv, dw0, B, H, N, eta, workspace, st);
    if (dtype == TTT_BF16)
        return linear_bwd_simt<__nv_bfloat16>(q, k, v, w0, dout, dq, dk, dv, dw0, B, H, N, d, eta, workspace, st);
    return linear_bwd_simt<float>(q, k, v, w0, dout, dq, dk, dv, dw0, B, H, N, d, eta, workspace, st);
}

// ------------------------------------------------------------------ depthwise conv ----
size_t ttt_dwconv_fullbatch_workspace_bytes(int B, int Hg, int Wg, int C, int dtype) {
    if (B <= 0 || Hg <= 0 || Wg <= 0 || C <= 0) return 0;
    if (dwconv_fused_ok(Hg, Wg, C, dtype)) return 0;
    return dwconv_ws(B, Hg, Wg, C);
}

int ttt_dwconv_fullbatch(const void* q, const void* k, const void* v, const float* w0, void* out, float* w_star,
                         int B, int Hg, int Wg, int C, float eta, int dtype, void* workspace,
                         size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("ttt_dwconv_fullbatch");
    if (int rc = check_common(q, k, v, out, dtype, eta)) return rc;
    if (!w0 || !aligned16(w0) || (w_star && !aligned16(w_star))) return TTT_ERR_INVALID_ARG;
    if (B <= 0 || Hg <= 0 || Wg <= 0 || C <= 0) return TTT_ERR_INVALID_ARG;
    const size_t need = ttt_dwconv_fullbatch_workspace_bytes(B, Hg, Wg, C, dtype);
    if (workspace_bytes < need || (need && !workspace)) return TTT_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return TTT_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dwconv_fused_ok(Hg, Wg, C, dtype)) return dwconv_fused(q, k, v, w0, out, w_star, B, Hg, Wg, eta, st);
    if (dtype == TTT_BF16)
        return dwconv_simt<__nv_bfloat16>(q, k, v, w0, out, w_star, B, Hg, Wg, C, eta, workspace, st);
    return dwconv_simt<float>(q, k, v, w0, out, w_star, B, Hg, Wg, C, eta, workspace, st);
}

// ------------------------------------------------------------------ TTT-MLP -----------
size_t ttt_mlp_fullbatch_workspace_bytes(int B, int H, int N, int d, int hidden, int dtype) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || hidden <= 0) return 0;
    if (mlp_tc_ok(B, H, d, hidden, dtype)) return mlp_tc_ws(B, H, N);
    return mlp_ws(B, H, N, d, hidden);
}

int ttt_mlp_fullbatch(const void* q, const void* k, const void* v, const float* w1, const float* w2, void* out,
                      float* w1_star, float* w2_star, int B, int H, int N, int d, int hidden, float eta, int dtype,
                      void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("ttt_mlp_fullbatch");
    if (int rc = check_common(q, k, v, out, dtype, eta)) return rc;
    if (!w1 || !w2 || !aligned16(w1) || !aligned16(w2)) return TTT_ERR_INVALID_ARG;
    if ((w1_star && !aligned16(w1_star)) || (w2_star && !aligned16(w2_star))) return TTT_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || hidden <= 0) return TTT_ERR_INVALID_ARG;
    if (d > 256 || hidden > 4096) return TTT_ERR_UNSUPPORTED;
    const size_t need = ttt_mlp_fullbatch_workspace_bytes(B, H, N, d, hidden, dtype);
    if (workspace_bytes < need || (need && !workspace)) return TTT_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return TTT_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (mlp_tc_ok(B, H, d, hidden, dtype))
        return mlp_tc(q, k, v, w1, w2, out, w1_star, w2_star, B, H, N, eta, workspace, st);
    if (dtype == TTT_BF16)
        return mlp_simt<__nv_bfloat16>(q, k, v, w1, w2, out, w1_star, w2_star, B, H, N, d, hidden, eta, workspace,
                                       st);
    return mlp_simt<float>(q, k, v, w1, w2, out, w1_star, w2_star, B, H, N, d, hidden, eta, workspace, st);
}

// ------------------------------------------------------------------ chunked scan ------
size_t ttt_linear_chunked_workspace_bytes(int B, int H, int N, int d, int chunk, int direction, int dtype) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || direction < -1 || direction > 1) return 0;
    if (chunked_tc_ok(B, H, d, chunk, dtype)) return chunked_tc_ws(B, H, N, direction);
    return chunked_ws(B, H, N, d, direction);
}

int ttt_linear_chunked(const void* q, const void* k, const void* v, const float* w0, void* out, int B, int H,
                       int N, int d, int chunk, float eta, int direction, int dtype, void* workspace,
                       size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("ttt_linear_chunked");
    if (int rc = check_common(q, k, v, out, dtype, eta)) return rc;
    if (!w0 || !aligned16(w0)) return TTT_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || chunk <= 0 || N % chunk != 0) return TTT_ERR_INVALID_ARG;
    if (direction < -1 || direction > 1) return TTT_ERR_INVALID_ARG;
    if (d > 128) return TTT_ERR_UNSUPPORTED;
    const size_t need = ttt_linear_chunked_workspace_bytes(B, H, N, d, chunk, direction, dtype);
    if (workspace_bytes < need || (need && !workspace)) return TTT_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return TTT_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (chunked_tc_ok(B, H, d, chunk, dtype))
        return chunked_tc(q, k, v, w0, out, B, H, N, eta, direction, need ? workspace : nullptr, st);
    if (dtype == TTT_BF16)
        return chunked_simt<__nv_bfloat16>(q, k, v, w0, out, B, H, N, d, chunk, eta, direction, workspace, st);
    return chunked_simt<float>(q, k, v, w0, out, B, H, N, d, chunk, eta, direction, workspace, st);
}

size_t ttt_linear_chunked_bidir_workspace_bytes(int B, int H, int N, int d, int chunk, int dtype) {
    return ttt_linear_chunked_workspace_bytes(B, H, N, d, chunk, 0, dtype);
}

int ttt_linear_chunked_bidir(const void* q, const void* k, const void* v, const float* w0, void* out, int B,
                             int H, int N, int d, int chunk, float eta, int dtype, void* workspace,
                             size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("ttt_linear_chunked_bidir");
    return ttt_linear_chunked(q, k, v, w0, out, B, H, N, d, chunk, eta, 0, dtype, workspace, workspace_bytes,
                              stream);
}

// ------------------------------------------------------------------ mini-batch training --
size_t ttt_linear_minibatch_workspace_bytes(int B, int H, int N, int d, int chunk, int epochs, int dtype) {
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || chunk <= 0 || epochs <= 0) return 0;
    const size_t own = align256((size_t)B * H * d * d * 4);
    if (chunk == N && epochs == 1) return std::max(own, ttt_linear_fullbatch_workspace_bytes(B, H, N, d, dtype));
    return own;
}

// O = Q W per unit for a given fp32 W [U][64][64], bf16 Q and O [U][N][64]: the tensor-core output pass.
int apply_w_tc(const void* q, const float* w, void* out, long long U, int N, cudaStream_t st) {
    if (U > 65535) return TTT_ERR_UNSUPPORTED;
    CUtensorMap tq, to;
    if (!tmap_bf16_3d(&tq, q, atc::D, N, (int)U, atc::MT, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tmap_bf16_3d(&to, out, atc::D, N, (int)U, atc::MT, CU_TENSOR_MAP_SWIZZLE_128B))
        return TTT_ERR_CUDA;
    if (cudaFuncSetAttribute(atc::apply_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, atc::smem_bytes()) !=
        cudaSuccess)
        return TTT_ERR_CUDA;
    atc::apply_kernel<<<dim3((unsigned)((N + atc::MT - 1) / atc::MT), (unsigned)U), atc::THREADS, atc::smem_bytes(),
                        st>>>(tq, to, w);
    return launched(1);
}

int ttt_linear_minibatch(const void* q, const void* k, const void* v, const float* w0, void* out, float* w_final,
                         int B, int H, int N, int d, int chunk, int epochs, float eta, int dtype, void* workspace,
                         size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("ttt_linear_minibatch");
    if (int rc = check_common(q, k, v, out, dtype, eta)) return rc;
    if (!w0 || !aligned16(w0) || (w_final && !aligned16(w_final))) return TTT_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || chunk <= 0 || N % chunk != 0 || epochs <= 0)
        return TTT_ERR_INVALID_ARG;
    if (d > 128) return TTT_ERR_UNSUPPORTED;
    const size_t need = ttt_linear_minibatch_workspace_bytes(B, H, N, d, chunk, epochs, dtype);
    if (workspace_bytes < need || !workspace) return TTT_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return TTT_ERR_INVALID_ARG;
    // one epoch over one chunk of all N tokens is the full-batch step
    if (chunk == N && epochs == 1)
        return ttt_linear_fullbatch(q, k, v, w0, out, w_final, B, H, N, d, eta, dtype, workspace, workspace_bytes,
                                    stream);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DeviceInfo* dev = nullptr;
    if (int rc = current_device(&dev)) return rc;
    const long long U = (long long)B * H;
    if (!grid_ok(U, (long long)N * d) || U > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
    const int smem = (2 * d * d + simt::CH_RB * d) * 4;
    if (smem > dev->smem_optin) return TTT_ERR_UNSUPPORTED;
    float* wfin = static_cast<float*>(workspace);
    const float eta_over_b = (float)((double)eta / (double)chunk);
    if (chunked_tc_ok(B, H, d, chunk, dtype)) {  // the tensor-core recurrence in training mode
        if (int rc = chunked_tc(q, k, v, w0, out, B, H, N, eta, 1, nullptr, st, epochs, wfin, w_final)) return rc;
        return apply_w_tc(q, wfin, out, U, N, st);
    }
    if (dtype == TTT_BF16) {
        using T = __nv_bfloat16;
        if (cudaFuncSetAttribute(simt::minibatch_train<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
            return TTT_ERR_CUDA;
        simt::minibatch_train<T><<<(unsigned)U, simt::TPB, smem, st>>>(
            static_cast<const T*>(k), static_cast<const T*>(v), w0, wfin, w_final, H, N, d, chunk, epochs, eta_over_b);
        if (d == atc::D) {  // the output pass on the tensor cores
            if (int rc = launched(1)) return rc;
            return apply_w_tc(q, wfin, out, U, N, st);
        }
        simt::linear_apply<T><<<grid_units(U, (long long)N * d), simt::TPB, 0, st>>>(static_cast<const T*>(q), wfin,
                                                                                    static_cast<T*>(out), N, d);
    } else {
        using T = float;
        if (cudaFuncSetAttribute(simt::minibatch_train<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
            return TTT_ERR_CUDA;
        simt::minibatch_train<T><<<(unsigned)U, simt::TPB, smem, st>>>(
            static_cast<const T*>(k), static_cast<const T*>(v), w0, wfin, w_final, H, N, d, chunk, epochs, eta_over_b);
        simt::linear_apply<T><<<grid_units(U, (long long)N * d), simt::TPB, 0, st>>>(static_cast<const T*>(q), wfin,
                                                                                    static_cast<T*>(out), N, d);
    }
    return launched(2);
}

// ------------------------------------------------------------------ conv-preprocessed scan
size_t ttt_linear_chunked_conv_workspace_bytes(int B, int H, int Hg, int Wg, int d, int chunk, int direction,
                                               int dtype) {
    if (B <= 0 || H <= 0 || Hg <= 0 || Wg <= 0 || d <= 0) return 0;
    const long long N = (long long)Hg * Wg;
    if (N > 0x7fffffffLL) return 0;
    const size_t es = dtype == TTT_BF16 ? 2 : 4;
    return 2 * align256((size_t)B * H * N * d * es) +
           ttt_linear_chunked_workspace_bytes(B, H, (int)N, d, chunk, direction, dtype);
}

int ttt_linear_chunked_conv(const void* q, const void* k, const void* v, const float* w0, const float* wk,
                            const float* wv, void* out, int B, int H, int Hg, int Wg, int d, int chunk, float eta,
                            int direction, int dtype, void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("ttt_linear_chunked_conv");
    if (int rc = check_common(q, k, v, out, dtype, eta)) return rc;
    if (!w0 || !wk || !wv || !aligned16(w0) || !aligned16(wk) || !aligned16(wv)) return TTT_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || Hg <= 0 || Wg <= 0 || d <= 0 || chunk <= 0) return TTT_ERR_INVALID_ARG;
    const long long N = (long long)Hg * Wg;
    if (N > 0x7fffffffLL || N % chunk != 0 || direction < -1 || direction > 1) return TTT_ERR_INVALID_ARG;
    if (d > 128) return TTT_ERR_UNSUPPORTED;
    const size_t need = ttt_linear_chunked_conv_workspace_bytes(B, H, Hg, Wg, d, chunk, direction, dtype);
    if (workspace_bytes < need || !workspace) return TTT_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return TTT_ERR_INVALID_ARG;
    const long long U = (long long)B * H;
    if (!grid_ok(U, N * d)) return TTT_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t es = dtype == TTT_BF16 ? 2 : 4;
    char* w = static_cast<char*>(workspace);
    void* kp = w;
    void* vp = w + align256((size_t)U * N * d * es);
    void* rest = w + 2 * align256((size_t)U * N * d * es);
    const size_t rest_bytes = workspace_bytes - 2 * align256((size_t)U * N * d * es);
    int prep_launches = 2;
    if (dtype == TTT_BF16 && d == 64 && U <= 65535) {
        using T = __nv_bfloat16;
        const long long nblk = (long long)((Wg + 31) / 32) * ((Hg + simt::PS_ROWS - 1) / simt::PS_ROWS);
        if (nblk > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
        simt::dwconv_prep_strip_bf16<<<dim3((unsigned)nblk, (unsigned)U, 2), 256, 0, st>>>(
            static_cast<const T*>(k), static_cast<const T*>(v), wk, wv, static_cast<T*>(kp), static_cast<T*>(vp), H, Hg,
            Wg);
        prep_launches = 1;
    } else if (dtype == TTT_BF16 && d % 8 == 0) {
        using T = __nv_bfloat16;
        dim3 grid = grid_units(U, N * (d / 8));
        grid.z = 2;
        simt::dwconv_prep2_bf16<<<grid, simt::TPB, d * 9 * 4, st>>>(static_cast<const T*>(k), static_cast<const T*>(v),
                                                                    wk, wv, static_cast<T*>(kp), static_cast<T*>(vp),
                                                                    H, Hg, Wg, d);
        prep_launches = 1;
    } else if (dtype == TTT_BF16) {
        using T = __nv_bfloat16;
        simt::dwconv_prep<T><<<grid_units(U, N * d), simt::TPB, 0, st>>>(static_cast<const T*>(k), wk,
                                                                         static_cast<T*>(kp), H, Hg, Wg, d);
        simt::dwconv_prep<T><<<grid_units(U, N * d), simt::TPB, 0, st>>>(static_cast<const T*>(v), wv,
                                                                         static_cast<T*>(vp), H, Hg, Wg, d);
    } else {
        using T = float;
        simt::dwconv_prep<T><<<grid_units(U, N * d), simt::TPB, 0, st>>>(static_cast<const T*>(k), wk,
                                                                         static_cast<T*>(kp), H, Hg, Wg, d);
        simt::dwconv_prep<T><<<grid_units(U, N * d), simt::TPB, 0, st>>>(static_cast<const T*>(v), wv,
                                                                         static_cast<T*>(vp), H, Hg, Wg, d);
    }
    if (int rc = launched(prep_launches)) return rc;
    return ttt_linear_chunked(q, kp, vp, w0, out, B, H, (int)N, d, chunk, eta, direction, dtype, rest, rest_bytes,
                              stream);
}

// ------------------------------------------------------------------ no-allocation scan ---
int ttt_linear_chunked_bidir_noalloc(const void* q, const void* k, const void* v, const float* w0, void* out,
                                     int B, int H, int N, int d, int chunk, float eta, int dtype, void* stream) {
    const size_t need = ttt_linear_chunked_bidir_workspace_bytes(B, H, N, d, chunk, dtype);
    if (need > kNoAllocScratchBytes) return TTT_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (int rc = noalloc_scratch(&scratch)) return rc;
    return ttt_linear_chunked_bidir(q, k, v, w0, out, B, H, N, d, chunk, eta, dtype, scratch, kNoAllocScratchBytes,
                                    stream);
}

size_t ttt_linear_chunked_bidir_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

}  // extern "C"

// dwconv_fused.cuh -- 3x3 depthwise-conv inner model, full batch, bf16, C = 64, one kernel.
//
// Operation ("ViT^3" blog, design study: a 3x3 depthwise convolution as the visual inner
// module; layer = train on (K, V), then apply to Q), per image b and channel c on the
// Hg x Wg token grid (channels-last, zero padding, no bias, tap (a, b) reads offset
// (a-1, b-1)):
//     r(p)    = sum_t w0[c][t] K(p + off_t) - V(p)
//     g[t]    = (1/N) sum_p r(p) K(p + off_t)          (N = Hg * Wg)
//     w*[c]   = w0[c] - eta g
//     O(p)    = sum_t w*[c][t] Q(p + off_t)
// Design (B200): one thread-block cluster of S CTAs per image, CTA r owning output rows
// [r*R, r*R + R).  A producer warp streams K rows (with the one-row halo above and below,
// zero-filled by TMA outside the image) and V rows through two small TMA rings; eight
// consumer warps each own a strip of pixels, each lane a pair of channels, and keep the
// 3-row x (strip + 2) window of K in registers: the residual and the nine tap gradients
// are accumulated with packed fp32 FMAs (fma.rn.f32x2).  The per-warp gradients are summed
// in shared memory, the S per-CTA partials over distributed shared memory in rank order
// (deterministic), every CTA forms w* for all channels, and the apply pass reads the Q rows
// that were prefetched into L2 during the gradient pass.  All waits are bounded.
#pragma once
#include "common.cuh"

namespace dwc {

constexpr int C = 64;
constexpr int PXB = C * 2;               // bytes per pixel
constexpr int PXW = 8;                   // pixels per consumer-warp strip
constexpr int MAX_CW = 8;                // consumer warps (ceil(Wg / 8)), plus one producer warp
constexpr int KS = 5, VS = 4;            // K ring and V ring slots (rows)
constexpr int MAX_R = 16;                // output rows per CTA
constexpr int NTAP = 9;

struct Params {
    const float* w0;     // [C][9]
    float* w_star;       // [B][C][9] or nullptr
    __nv_bfloat16* out;  // [B][Hg][Wg][C]
    int Hg, Wg, R;
    int cw;              // consumer warps: 8 * cw >= Wg
    int slot_bytes;      // one padded row: (8 * cw + 2) pixels
    int nslots;          // max(KS + VS, R + 2)
    float eta_over_n;
};

struct Bars {
    uint64_t kfull[KS], kempty[KS], vfull[VS], vempty[VS], qfull[MAX_R + 2], qgo;
};

__device__ __forceinline__ float2 bf2(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(d)
        : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)),
          "l"(*reinterpret_cast<uint64_t*>(&c)));
    return *reinterpret_cast<float2*>(&d);
}
__device__ __forceinline__ void consumers_sync(int n) { asm volatile("bar.sync 1, %0;" ::"r"(n) : "memory"); }
__device__ __forceinline__ float dsmem_ld_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* m, int c0, int c1, int c2, int c3,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_prefetch_l2_4d(const CUtensorMap* m, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}

// Consumer warp w owns image pixels [8w, 8w + 8).  Shared-memory pixel x+1 holds image
// pixel x; pixels 0 and Wg+1 .. 8*cw+1 of every row slot stay zero (horizontal zero padding).
__global__ void __launch_bounds__((MAX_CW + 1) * 32, 1)
    dwconv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_q, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint8_t* slots = smem;
    float* partial = reinterpret_cast<float*>(smem + p.nslots * p.slot_bytes);  // [C][9], read by peers
    float* wst = partial + C * NTAP;                                             // [C][9]
    float* red = wst + C * NTAP;                                                 // [cw][9][C]
    Bars* bars = reinterpret_cast<Bars*>(red + MAX_CW * NTAP * C);
    const int CW = p.cw;
    const int THREADS = (CW + 1) * 32;

    const uint32_t S = gridDim.x;
    const uint32_t rank = cluster_ctarank();
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int y0 = (int)rank * p.R;
    const int rows = max(0, min(p.Hg - y0, p.R));
    const int row_bytes = p.Wg * PXB;
    auto slot = [&](int s) { return slots + s * p.slot_bytes; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < KS; ++s) {
            mbar_init(&bars->kfull[s], 1);
            mbar_init(&bars->kempty[s], CW);
        }
        for (int s = 0; s < VS; ++s) {
            mbar_init(&bars->vfull[s], 1);
            mbar_init(&bars->vempty[s], CW);
        }
        for (int s = 0; s < MAX_R + 2; ++s) mbar_init(&bars->qfull[s], 1);
        mbar_init(&bars->qgo, 1);
        mbar_fence_init();
    }
    // zero the padding pixels of slots [0, n) (TMA writes pixels 1..Wg only)
    auto zero_pads = [&](int n, int tid, int nthreads) {
        const int px_per_slot = p.slot_bytes / PXB;
        const int pad_px = px_per_slot - p.Wg;  // pixel 0 and Wg+1 .. end
        for (int e = tid; e < n * pad_px * (PXB / 16); e += nthreads) {
            const int s = e / (pad_px * (PXB / 16)), r = e % (pad_px * (PXB / 16));
            const int px = r / (PXB / 16), w = r % (PXB / 16);
            const int pix = px == 0 ? 0 : p.Wg + px;
            *reinterpret_cast<uint4*>(slot(s) + pix * PXB + w * 16) = make_uint4(0, 0, 0, 0);
        }
    };
    zero_pads(p.nslots, threadIdx.x, THREADS);
    fence_proxy_async_smem();
    __syncthreads();

    if (warp == CW) {
        // ================================ producer ======================================
        if (lane == 0) {
            auto load_k = [&](int k) {  // K row y0 - 1 + k
                const int s = k % KS, use = k / KS;
                if (use > 0) mbar_wait(&bars->kempty[s], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                mbar_expect_tx(&bars->kfull[s], row_bytes);
                tma_load_4d(slot(s) + PXB, &tm_k, 0, 0, y0 - 1 + k, b, &bars->kfull[s]);
            };
            auto load_v = [&](int j) {  // V row y0 + j
                const int s = j % VS, use = j / VS;
                if (use > 0) mbar_wait(&bars->vempty[s], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                mbar_expect_tx(&bars->vfull[s], row_bytes);
                tma_load_4d(slot(KS + s) + PXB, &tm_v, 0, 0, y0 + j, b, &bars->vfull[s]);
            };
            if (rows > 0) {
                for (int k = 0; k < min(KS, rows + 2); ++k) load_k(k);
                for (int j = 0; j < min(VS, rows); ++j) load_v(j);
                for (int j = 0; j < rows; ++j) {  // refill as the consumers release rows
                    if (j + KS < rows + 2) load_k(j + KS);
                    if (j + VS < rows) load_v(j + VS);
                }
                for (int k = 0; k < rows + 2; ++k)
                    if (y0 - 1 + k >= 0 && y0 - 1 + k < p.Hg) tma_prefetch_l2_4d(&tm_q, 0, 0, y0 - 1 + k, b);
            }
            mbar_wait(&bars->qgo, 0, TTT_DEVERR_TIMEOUT_PEER);  // slots free again
            fence_proxy_async_smem();
            for (int k = 0; k < (rows > 0 ? rows + 2 : 0); ++k) {
                mbar_expect_tx(&bars->qfull[k], row_bytes);
                tma_load_4d(slot(k) + PXB, &tm_q, 0, 0, y0 - 1 + k, b, &bars->qfull[k]);
            }
        }
        __syncwarp();
        cluster_sync_all();
        cluster_arrive_release();
        cluster_wait_acquire();
        return;
    }

    // =================================== consumers =======================================
    const int px0 = warp * PXW;  // first image pixel of this warp's strip
    const int c = 2 * lane;      // channels c, c + 1
    float2 w0f[NTAP];
#pragma unroll
    for (int t = 0; t < NTAP; ++t) w0f[t] = make_float2(__ldg(&p.w0[c * NTAP + t]), __ldg(&p.w0[(c + 1) * NTAP + t]));
    float2 g[NTAP];
#pragma unroll
    for (int t = 0; t < NTAP; ++t) g[t] = make_float2(0.f, 0.f);

    // The 3-row K window lives in registers and slides by one row per output row: each K
    // row is awaited, read and released (kempty) once; likewise each V row.
    const uint8_t* kbase = slots + px0 * PXB + c * 2;  // smem pixel px0 = image pixel px0 - 1
    auto load_krow = [&](int k, float2* dst) {
        const int s = k % KS;
        mbar_wait(&bars->kfull[s], (k / KS) & 1, TTT_DEVERR_TIMEOUT_TMA);
#pragma unroll
        for (int xi = 0; xi < PXW + 2; ++xi)
            dst[xi] = bf2(*reinterpret_cast<const uint32_t*>(kbase + s * p.slot_bytes + xi * PXB));
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->kempty[s]);  // the row is in registers now
    };
    float2 kw[3][PXW + 2];
    if (rows > 0) {
        load_krow(0, kw[0]);
        load_krow(1, kw[1]);
    }
    for (int j = 0; j < rows; ++j) {
        load_krow(j + 2, kw[2]);
        const int vs = j % VS;
        mbar_wait(&bars->vfull[vs], (j / VS) & 1, TTT_DEVERR_TIMEOUT_TMA);
        const uint8_t* vbase = slot(KS + vs) + (px0 + 1) * PXB + c * 2;
#pragma unroll
        for (int i = 0; i < PXW; ++i) {
            if (px0 + i < p.Wg) {
                const float2 v = bf2(*reinterpret_cast<const uint32_t*>(vbase + i * PXB));
                float2 r = make_float2(-v.x, -v.y);
#pragma unroll
                for (int t = 0; t < NTAP; ++t) r = ffma2(w0f[t], kw[t / 3][i + t % 3], r);
#pragma unroll
                for (int t = 0; t < NTAP; ++t) g[t] = ffma2(r, kw[t / 3][i + t % 3], g[t]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->vempty[vs]);
#pragma unroll
        for (int xi = 0; xi < PXW + 2; ++xi) {
            kw[0][xi] = kw[1][xi];
            kw[1][xi] = kw[2][xi];
        }
    }
    // every K/V row has been read: the slots may take the Q rows while the gradients reduce
    fence_proxy_async_smem();
    consumers_sync(CW * 32);
    if (threadIdx.x == 0) mbar_arrive(&bars->qgo);
    // ---- per-CTA partial: sum the warps' gradients (dedicated buffer) ----------------------
#pragma unroll
    for (int t = 0; t < NTAP; ++t) {
        red[(warp * NTAP + t) * C + c] = g[t].x;
        red[(warp * NTAP + t) * C + c + 1] = g[t].y;
    }
    consumers_sync(CW * 32);
    for (int e = threadIdx.x; e < C * NTAP; e += CW * 32) {
        const int ch = e / NTAP, t = e % NTAP;
        float sum = 0.f;
        for (int w = 0; w < CW; ++w) sum += red[(w * NTAP + t) * C + ch];
        partial[e] = sum;
    }
    cluster_sync_all();

    // ---- w* = w0 - (eta/N) sum over the cluster, in rank order ------------------------------
    for (int e = threadIdx.x; e < C * NTAP; e += CW * 32) {
        float x[16];
        const uint32_t n = min(S, 16u);
#pragma unroll
        for (uint32_t q = 0; q < 16; ++q)
            if (q < n) x[q] = dsmem_ld_f32(dsmem_map(&partial[e], q));
        float s = 0.f;
#pragma unroll
        for (uint32_t q = 0; q < 16; ++q)
            if (q < n) s += x[q];
        const float w = __ldg(&p.w0[e]) - p.eta_over_n * s;
        wst[e] = w;
        if (p.w_star && rank == 0) p.w_star[(size_t)b * C * NTAP + e] = w;
    }
    cluster_arrive_release();  // done reading the peers' partials
    consumers_sync(CW * 32);

    // ---- O = conv(Q, w*) ------------------------------------------------------------------
    float2 wf[NTAP];
#pragma unroll
    for (int t = 0; t < NTAP; ++t) wf[t] = make_float2(wst[c * NTAP + t], wst[(c + 1) * NTAP + t]);
    const uint8_t* qbase = slots + px0 * PXB + c * 2;
    auto load_qrow = [&](int k, float2* dst) {  // Q row y0 - 1 + k lives in slot k
        mbar_wait(&bars->qfull[k], 0, TTT_DEVERR_TIMEOUT_TMA);
#pragma unroll
        for (int xi = 0; xi < PXW + 2; ++xi)
            dst[xi] = bf2(*reinterpret_cast<const uint32_t*>(qbase + k * p.slot_bytes + xi * PXB));
    };
    float2 qw[3][PXW + 2];
    if (rows > 0) {
        load_qrow(0, qw[0]);
        load_qrow(1, qw[1]);
    }
    for (int j = 0; j < rows; ++j) {
        load_qrow(j + 2, qw[2]);
        __nv_bfloat16* orow = p.out + (((size_t)b * p.Hg + y0 + j) * p.Wg) * C + c;
#pragma unroll
        for (int i = 0; i < PXW; ++i) {
            if (px0 + i < p.Wg) {
                float2 o = make_float2(0.f, 0.f);
#pragma unroll
                for (int t = 0; t < NTAP; ++t) o = ffma2(wf[t], qw[t / 3][i + t % 3], o);
                *reinterpret_cast<uint32_t*>(orow + (size_t)(px0 + i) * C) = pack_bf16(o.x, o.y);
            }
        }
#pragma unroll
        for (int xi = 0; xi < PXW + 2; ++xi) {
            qw[0][xi] = qw[1][xi];
            qw[1][xi] = qw[2][xi];
        }
    }
    cluster_wait_acquire();
}

}  // namespace dwc

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
// [r*R, r*R + R).  The CTA's rows form NB bands (two when the width allows fourteen consumer
// warps) that advance side by side; at a 56-token width that is fifteen warps and one CTA per
// SM, so every CTA of a cluster runs at the same pace (with two CTAs per SM, some SMs held
// one and the clusters waited for their SM-sharing CTAs).
// A producer warp streams each band's K rows (with the one-row halo above and below,
// zero-filled by TMA outside the image) and V rows through small TMA rings; the consumer
// warps of a band each own a strip of pixels, each lane a pair of channels, and keep the
// 3-row x (strip + 2) window of K in registers: the residual and the nine tap gradients
// are accumulated with packed fp32 FMAs (__ffma2_rn, one fma.rn.f32x2 per channel pair).
// The per-warp gradients are summed in shared memory in warp order; the S per-CTA partials
// are exchanged in two hops (deterministic, fixed order): every CTA sends slice q of its
// partial to CTA q (st.async), CTA q adds the S slices in rank order, forms that slice of w*
// and sends it to every CTA (st.async).  The apply pass reads the Q rows that were
// prefetched into L2 during the gradient pass.  All waits are bounded.
#pragma once
#include "common.cuh"

namespace dwc {

constexpr int C = 64;
constexpr int PXB = C * 2;               // bytes per pixel
constexpr int PXW = 8;                   // pixels per consumer-warp strip
constexpr int MAX_CW = 8;                // consumer warps of a band (ceil(Wg / 8))
constexpr int MAX_NB = 2;                // bands
constexpr int MAX_WARPS = 14;            // consumer warps in all (nb * cw), plus one producer warp
constexpr int KS = 5, VS = 4;            // K ring and V ring slots (rows) of a band
constexpr int MAX_R = 16;                // output rows per CTA
constexpr int NTAP = 9;

struct Params {
    const float* w0;     // [C][9]
    float* w_star;       // [B][C][9] or nullptr
    __nv_bfloat16* out;  // [B][Hg][Wg][C]
    int Hg, Wg, R;
    int cw;              // consumer warps of a band: 8 * cw >= Wg
    int nb;              // bands (nb * cw <= MAX_WARPS)
    int slot_bytes;      // one padded row: (8 * cw + 2) pixels
    int nslots;          // max(nb * (KS + VS), R + 2)
    float eta_over_n;
};

struct Bars {
    uint64_t kfull[MAX_NB][KS], kempty[MAX_NB][KS], vfull[MAX_NB][VS], vempty[MAX_NB][VS];
    uint64_t qfull[MAX_R + 2], qgo;
    uint64_t rfull;  // the peers' parts of this CTA's slice of the partial (st.async bytes)
    uint64_t wfull;  // the peers' slices of w* (st.async bytes)
};

// A bf16 pair (low half = first element) as two fp32 values; byte permute and mask keep the
// conversion off the FMA pipe.
__device__ __forceinline__ float2 bf2(uint32_t v) {
    return make_float2(__uint_as_float(__byte_perm(v, 0u, 0x1054)), __uint_as_float(v & 0xffff0000u));
}
__device__ __forceinline__ void consumers_sync(int n) { asm volatile("bar.sync 1, %0;" ::"r"(n) : "memory"); }
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

// Consumer warp w works in band w / cw on image pixels [8 (w % cw), 8 (w % cw) + 8).
// Shared-memory pixel x+1 holds image pixel x; pixels 0 and Wg+1 .. 8*cw+1 of every row slot
// stay zero (horizontal zero padding).  Band n's K ring is slots n (KS + VS) + [0, KS), its V
// ring the next VS slots; after the gradient pass Q row y0 - 1 + k goes to slot k.
// 128 registers: fifteen warps fit one CTA per SM.
__global__ void __maxnreg__(128)
    dwconv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_q, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align<128>(smem_raw);
    uint8_t* slots = smem;
    float* gather = reinterpret_cast<float*>(smem + p.nslots * p.slot_bytes);  // [S][C*9/S]: slice parts
    float* wst = gather + C * NTAP;                                            // [C][9]
    float* red = wst + C * NTAP;                                               // [warps][C][9]
    Bars* bars = reinterpret_cast<Bars*>(red + MAX_WARPS * NTAP * C);
    const int CW = p.cw, NB = p.nb, NW = NB * CW;
    const int THREADS = (NW + 1) * 32;

    const uint32_t S = gridDim.x;
    const uint32_t rank = cluster_ctarank();
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int y0 = (int)rank * p.R;
    const int rows = max(0, min(p.Hg - y0, p.R));
    const int band_rows = (rows + NB - 1) / NB;  // rows of every band but the last
    auto rows_of = [&](int n) { return max(0, min(rows - n * band_rows, band_rows)); };
    const int row_bytes = p.Wg * PXB;
    const int slice = C * NTAP / (int)S;  // taps (in [C][9] order) whose w* this CTA forms
    auto slot = [&](int s) { return slots + s * p.slot_bytes; };

    if (warp == 0) {  // barrier initialisation, spread over the lanes of warp 0
        for (int i = lane; i < NB * (KS + VS) + MAX_R + 2; i += 32) {
            if (i < NB * (KS + VS)) {
                const int n = i / (KS + VS), s = i % (KS + VS);
                if (s < KS) {
                    mbar_init(&bars->kfull[n][s], 1);
                    mbar_init(&bars->kempty[n][s], CW);
                } else {
                    mbar_init(&bars->vfull[n][s - KS], 1);
                    mbar_init(&bars->vempty[n][s - KS], CW);
                }
            } else {
                mbar_init(&bars->qfull[i - NB * (KS + VS)], 1);
            }
        }
        if (lane == 0) {
            mbar_init(&bars->qgo, 1);
            mbar_init(&bars->rfull, 1);
            mbar_init(&bars->wfull, 1);
            mbar_expect_tx(&bars->rfull, (S - 1) * slice * 4);
            mbar_expect_tx(&bars->wfull, (S - 1) * slice * 4);
        }
        mbar_fence_init();
    }
    {  // zero the padding pixels of every slot (TMA writes pixels 1..Wg only)
        const int px_per_slot = p.slot_bytes / PXB;
        const int pad_px = px_per_slot - p.Wg;  // pixel 0 and Wg+1 .. end
        for (int e = threadIdx.x; e < p.nslots * pad_px * (PXB / 16); e += THREADS) {
            const int s = e / (pad_px * (PXB / 16)), r = e % (pad_px * (PXB / 16));
            const int px = r / (PXB / 16), w = r % (PXB / 16);
            const int pix = px == 0 ? 0 : p.Wg + px;
            *reinterpret_cast<uint4*>(slot(s) + pix * PXB + w * 16) = make_uint4(0, 0, 0, 0);
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    cluster_arrive_release();  // this CTA's barriers are initialised (waited on before any st.async)
    // Launched with programmatic stream serialization: the first K and V rows go into L2 while the
    // previous grid on the stream may still run (a prefetch only warms the coherent L2); every
    // load and store of this grid comes after griddep_wait.
    if (threadIdx.x == 32 * NW && rows > 0)
        for (int n = 0; n < NB; ++n)
            for (int k = 0; k < min(KS, rows_of(n) + 2); ++k) {
                const int y = y0 + n * band_rows - 1 + k;
                if (y >= 0 && y < p.Hg) tma_prefetch_l2_4d(&tm_k, 0, 0, y, b);
                if (k < min(VS, rows_of(n)) && y + 1 < p.Hg) tma_prefetch_l2_4d(&tm_v, 0, 0, y + 1, b);
            }
    griddep_wait();
    griddep_launch();  // one wave: the next grid's CTAs start only as SMs free up

    if (warp == NW) {
        // ================================ producer ======================================
        if (lane == 0) {
            auto load_k = [&](int n, int k) {  // K row y_n - 1 + k of band n
                const int s = k % KS, use = k / KS;
                if (use > 0) mbar_wait(&bars->kempty[n][s], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                mbar_expect_tx(&bars->kfull[n][s], row_bytes);
                tma_load_4d(slot(n * (KS + VS) + s) + PXB, &tm_k, 0, 0, y0 + n * band_rows - 1 + k, b,
                            &bars->kfull[n][s]);
            };
            auto load_v = [&](int n, int j) {  // V row y_n + j of band n
                const int s = j % VS, use = j / VS;
                if (use > 0) mbar_wait(&bars->vempty[n][s], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                mbar_expect_tx(&bars->vfull[n][s], row_bytes);
                tma_load_4d(slot(n * (KS + VS) + KS + s) + PXB, &tm_v, 0, 0, y0 + n * band_rows + j, b,
                            &bars->vfull[n][s]);
            };
            if (rows > 0) {
                // in the order the consumers need them: K rows y-1, y of every band, then
                // (K row y+1, V row y) of every band, step by step
                for (int n = 0; n < NB; ++n)
                    if (rows_of(n) > 0) {
                        load_k(n, 0);
                        load_k(n, 1);
                    }
                for (int j = 0; j < band_rows; ++j)
                    for (int n = 0; n < NB; ++n)
                        if (j < rows_of(n)) {
                            load_k(n, j + 2);
                            load_v(n, j);
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
        cluster_wait_acquire();
        cluster_arrive_release();
        cluster_wait_acquire();
        return;
    }

    // =================================== consumers =======================================
    const int band = warp / CW;
    const int px0 = (warp % CW) * PXW;  // first image pixel of this warp's strip
    const int c = 2 * lane;             // channels c, c + 1
    const int nrows = rows_of(band), yb = y0 + band * band_rows;
    float2 w0f[NTAP];
#pragma unroll
    for (int t = 0; t < NTAP; ++t) w0f[t] = make_float2(__ldg(&p.w0[c * NTAP + t]), __ldg(&p.w0[(c + 1) * NTAP + t]));
    float2 g[NTAP];
#pragma unroll
    for (int t = 0; t < NTAP; ++t) g[t] = make_float2(0.f, 0.f);

    // The 3-row K window lives in registers and slides by one row per output row: each K
    // row is awaited, read and released (kempty) once; likewise each V row.
    const uint8_t* kbase = slot(band * (KS + VS)) + px0 * PXB + c * 2;  // smem pixel px0 = image pixel px0 - 1
    auto load_krow = [&](int k, float2* dst) {
        const int s = k % KS;
        mbar_wait(&bars->kfull[band][s], (k / KS) & 1, TTT_DEVERR_TIMEOUT_TMA);
#pragma unroll
        for (int xi = 0; xi < PXW + 2; ++xi)
            dst[xi] = bf2(*reinterpret_cast<const uint32_t*>(kbase + s * p.slot_bytes + xi * PXB));
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->kempty[band][s]);  // the row is in registers now
    };
    float2 kw[3][PXW + 2];
    if (nrows > 0) {
        load_krow(0, kw[0]);
        load_krow(1, kw[1]);
    }
    for (int j = 0; j < nrows; ++j) {
        load_krow(j + 2, kw[2]);
        const int vs = j % VS;
        mbar_wait(&bars->vfull[band][vs], (j / VS) & 1, TTT_DEVERR_TIMEOUT_TMA);
        const uint8_t* vbase = slot(band * (KS + VS) + KS + vs) + (px0 + 1) * PXB + c * 2;
#pragma unroll
        for (int i = 0; i < PXW; ++i) {
            const float2 v = bf2(*reinterpret_cast<const uint32_t*>(vbase + i * PXB));
            float2 r = make_float2(-v.x, -v.y);
#pragma unroll
            for (int t = 0; t < NTAP; ++t) r = __ffma2_rn(w0f[t], kw[t / 3][i + t % 3], r);
            if (px0 + i >= p.Wg) r = make_float2(0.f, 0.f);  // past the image: no term
#pragma unroll
            for (int t = 0; t < NTAP; ++t) g[t] = __ffma2_rn(r, kw[t / 3][i + t % 3], g[t]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->vempty[band][vs]);
#pragma unroll
        for (int xi = 0; xi < PXW + 2; ++xi) {
            kw[0][xi] = kw[1][xi];
            kw[1][xi] = kw[2][xi];
        }
    }
    // every K/V row has been read: the slots may take the Q rows while the gradients reduce
    fence_proxy_async_smem();
    consumers_sync(NW * 32);
    if (threadIdx.x == 0) mbar_arrive(&bars->qgo);
    // ---- per-CTA partial: sum the warps' gradients (dedicated buffer) ----------------------
#pragma unroll
    for (int t = 0; t < NTAP; ++t) {
        red[(warp * C + c) * NTAP + t] = g[t].x;
        red[(warp * C + c + 1) * NTAP + t] = g[t].y;
    }
    consumers_sync(NW * 32);
    cluster_wait_acquire();  // every CTA of the cluster has initialised its barriers
    // part of the partial: the warps in warp order; float4 group q goes to the owner of its slice
    for (int q = threadIdx.x; q < C * NTAP / 4; q += NW * 32) {
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        for (int w = 0; w < NW; ++w) {
            const float4 v = *reinterpret_cast<const float4*>(red + w * C * NTAP + 4 * q);
            x[0] += v.x;
            x[1] += v.y;
            x[2] += v.z;
            x[3] += v.w;
        }
        const uint32_t owner = (uint32_t)(4 * q / slice);
        float* dst = gather + rank * slice + (4 * q) % slice;
        if (owner == rank)
            *reinterpret_cast<float4*>(dst) = make_float4(x[0], x[1], x[2], x[3]);
        else
            st_async_v4(mapa_u32(smem_u32(dst), owner), mapa_u32(smem_u32(&bars->rfull), owner), __float_as_uint(x[0]),
                        __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
    }
    consumers_sync(NW * 32);                                      // this CTA's own parts
    mbar_wait_cluster(&bars->rfull, 0, TTT_DEVERR_TIMEOUT_PEER);  // the peers' parts

    // ---- slice of w* = w0 - (eta/N) sum over the cluster, in rank order; sent to every CTA ----
    for (int q = threadIdx.x; q < slice / 4; q += NW * 32) {
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
        for (uint32_t src = 0; src < S; ++src) {
            const float4 v = *reinterpret_cast<const float4*>(gather + src * slice + 4 * q);
            sum.x += v.x;
            sum.y += v.y;
            sum.z += v.z;
            sum.w += v.w;
        }
        const int e = (int)rank * slice + 4 * q;
        const float4 w0 = __ldg(reinterpret_cast<const float4*>(p.w0 + e));
        const float4 w = make_float4(w0.x - p.eta_over_n * sum.x, w0.y - p.eta_over_n * sum.y,
                                     w0.z - p.eta_over_n * sum.z, w0.w - p.eta_over_n * sum.w);
        if (p.w_star) *reinterpret_cast<float4*>(p.w_star + (size_t)b * C * NTAP + e) = w;
        *reinterpret_cast<float4*>(wst + e) = w;
        for (uint32_t k = 1; k < S; ++k) {
            const uint32_t peer = (rank + k) % S;
            st_async_v4(mapa_u32(smem_u32(wst + e), peer), mapa_u32(smem_u32(&bars->wfull), peer),
                        __float_as_uint(w.x), __float_as_uint(w.y), __float_as_uint(w.z), __float_as_uint(w.w));
        }
    }
    consumers_sync(NW * 32);                                      // this CTA's own slice
    mbar_wait_cluster(&bars->wfull, 0, TTT_DEVERR_TIMEOUT_PEER);  // the peers' slices
    cluster_arrive_release();

    // ---- O = conv(Q, w*) on the band's rows -------------------------------------------------
    float2 wf[NTAP];
#pragma unroll
    for (int t = 0; t < NTAP; ++t) wf[t] = make_float2(wst[c * NTAP + t], wst[(c + 1) * NTAP + t]);
    const int k0 = yb - y0;  // Q row yb - 1 + k lives in slot k0 + k
    const uint8_t* qbase = slots + px0 * PXB + c * 2;
    auto load_qrow = [&](int k, float2* dst) {
        mbar_wait(&bars->qfull[k0 + k], 0, TTT_DEVERR_TIMEOUT_TMA);
#pragma unroll
        for (int xi = 0; xi < PXW + 2; ++xi)
            dst[xi] = bf2(*reinterpret_cast<const uint32_t*>(qbase + (k0 + k) * p.slot_bytes + xi * PXB));
    };
    float2 qw[3][PXW + 2];
    if (nrows > 0) {
        load_qrow(0, qw[0]);
        load_qrow(1, qw[1]);
    }
    for (int j = 0; j < nrows; ++j) {
        load_qrow(j + 2, qw[2]);
        __nv_bfloat16* orow = p.out + (((size_t)b * p.Hg + yb + j) * p.Wg) * C + c;
#pragma unroll
        for (int i = 0; i < PXW; ++i) {
            float2 o = make_float2(0.f, 0.f);
#pragma unroll
            for (int t = 0; t < NTAP; ++t) o = __ffma2_rn(wf[t], qw[t / 3][i + t % 3], o);
            if (px0 + i < p.Wg) *reinterpret_cast<uint32_t*>(orow + (size_t)(px0 + i) * C) = pack_bf16(o.x, o.y);
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

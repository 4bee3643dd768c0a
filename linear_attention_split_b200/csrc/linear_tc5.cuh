// linear_tc5.cuh -- TTT-Linear full-batch step on the 5th-generation tensor cores (tcgen05),
// bf16 inputs, d = 64, one kernel per call.
//
// Operation ("ViT^3" blog, online-learning rewrite of attention, steps 1-3; TTT-Linear of the
// TTT abstract), per unit u = (batch b, head h) with Q, K, V in R^{N x 64}:
//     G = K^T K,  C = K^T V,   W* = W0 - (eta/N) (G W0 - C),   O = Q W*
// ((G W0 - C)/N is the full-batch gradient of (1/N) sum_i 1/2 ||k_i W - v_i||^2 at W0.)
//
// Layout of the work:
//   * one thread-block cluster of S CTAs per unit (S in {1, 2, 4, 8}); CTA r owns tokens
//     [r*T, r*T + T);
//   * warp 0 (producer) streams K/V tiles of TT <= 64 tokens through a 3-slot TMA ring
//     (128-byte swizzle, no multicast), then prefetches this CTA's Q rows into a resident
//     region, so that Q's HBM traffic overlaps the in-cluster reduction;
//   * warp 1 (MMA issuer) computes [G ; C^T] = [K | V]^T K with tcgen05.mma, M = 128
//     (features of K then of V), N = 64, K-dim = tokens, both operands MN-major straight from
//     the TMA tiles, fp32 accumulator in tensor memory (TMEM); a commit per tile frees its
//     ring slot;
//   * warps 2-5 (epilogue) move the 128 x 64 partial from TMEM to shared memory, sum the S
//     partials in rank order over distributed shared memory (each CTA reduces its 64/S rows
//     of W*; deterministic, no atomics), form W* rows in fp32, and broadcast them to every
//     CTA of the cluster as bf16 W*^T = hi + lo (hi = bf16(W*), lo = bf16(W* - hi));
//   * after a second cluster barrier the issuer computes O = Q hi + Q lo per 128-token tile
//     (K-major operands) into one of four TMEM buffers, and the epilogue converts O to bf16
//     in place over Q and stores it with TMA (rows >= N are clipped by the hardware).
// If a CTA's Q rows do not fit the resident region, the rest stream through two ring slots
// after the reduction.  All waits are bounded (common.cuh).
#pragma once
#include "common.cuh"

namespace lin5 {

constexpr int D = 64;
constexpr int ROWB = 128;                 // bytes per token row (64 bf16)
constexpr int THREADS = 192;              // producer, issuer, 4 epilogue warps
constexpr int TILE_ROWS = 64;             // rows reserved per K or V tile in a ring slot
constexpr int TILE_BYTES = TILE_ROWS * ROWB;
constexpr int SLOT_BYTES = 2 * TILE_BYTES;  // K tile, V tile
constexpr int STAGES = 3;
constexpr int RING_BYTES = STAGES * SLOT_BYTES;
constexpr int SCR_BYTES = 128 * 64 * 4;   // [G ; C^T] fp32, 32 KB = ring slots 0-1
constexpr int WT_OFF = SCR_BYTES;         // W*^T hi at ring + 32 KB, lo at + 40 KB (slot 2)
constexpr int WT_BYTES = D * D * 2;
constexpr int MT = 128;                   // tokens per phase-2 MMA tile
constexpr int TMEM_COLS = 256;            // phase-1 accumulator, then four phase-2 buffers
constexpr int MAX_QBOX = 32;              // resident Q TMA boxes per CTA
constexpr uint32_t IDESC_GRAM = tc::idesc_bf16(128, 64, 1, 1);
constexpr uint32_t IDESC_APPLY = tc::idesc_bf16(128, 64, 0, 0);

struct Params {
    const float* w0;   // [H][64][64]
    float* w_star;     // [U][64][64] or nullptr
    int H, N;
    int T;             // tokens per CTA
    int TT;            // tokens per K/V tile (multiple of 8, <= 64)
    int q_rows;        // resident Q rows (multiple of 8; multiple of 128 when Q streams)
    int q_region;      // bytes of the resident region (multiple of 1024)
    float eta_over_n;
};

struct Bars {
    uint64_t full[STAGES], empty[STAGES], qfull[MAX_QBOX], gram_done, tfull[4], tempty[4], sfull[2],
        sempty[2];
    uint32_t tmem_base;
};

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

// scratch: fp32 [128 rows][64 cols], float4 chunks XOR-swizzled by row to spread banks
__device__ __forceinline__ int scr_idx(int r, int c) { return r * 64 + ((((c >> 2) ^ (r & 15))) << 2) + (c & 3); }

__global__ void __launch_bounds__(THREADS, 2)
    linear_tc5_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_q128,
                      const __grid_constant__ CUtensorMap tm_o, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* qreg = smem;
    uint8_t* ring = smem + p.q_region;
    float* scr = reinterpret_cast<float*>(ring);
    uint8_t* wt = ring + WT_OFF;
    Bars* bars = reinterpret_cast<Bars*>(ring + RING_BYTES);

    const uint32_t S = gridDim.x;  // one cluster spans the x dimension
    const uint32_t rank = cluster_ctarank();
    const int u = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = (int)rank * p.T;
    const int n_valid = max(0, min(p.N - t0, p.T));
    const int nkv = (n_valid + p.TT - 1) / p.TT;                   // K/V tiles with data
    const int q_valid = min(n_valid, p.q_rows);                      // resident rows with data
    const int nqbox = (q_valid + p.TT - 1) / p.TT;                   // resident Q boxes
    const int n_res_mt = (q_valid + MT - 1) / MT;                    // resident 128-row tiles
    const int n_mt = (n_valid + MT - 1) / MT;                        // all 128-row tiles

    // ---- set-up ------------------------------------------------------------------------
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int j = 0; j < MAX_QBOX; ++j) mbar_init(&bars->qfull[j], 1);
        mbar_init(&bars->gram_done, 1);
        for (int b = 0; b < 4; ++b) {
            mbar_init(&bars->tfull[b], 1);
            mbar_init(&bars->tempty[b], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->sfull[b], 1);
            mbar_init(&bars->sempty[b], 4);
        }
        mbar_fence_init();
    }
    if (p.TT < TILE_ROWS) {  // token rows [TT, 64) of every K/V tile: zero K-dim padding
        const int pad16 = (TILE_ROWS - p.TT) * ROWB / 16;
        for (int e = threadIdx.x; e < STAGES * 2 * pad16; e += THREADS) {
            const int tile = e / pad16, w = e % pad16;
            *reinterpret_cast<uint4*>(ring + tile * TILE_BYTES + p.TT * ROWB + w * 16) = make_uint4(0, 0, 0, 0);
        }
    }
    if (warp == 1) tc::alloc(&bars->tmem_base, TMEM_COLS);
    fence_proxy_async_smem();
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ================================ producer ======================================
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_q);
            for (int i = 0; i < nkv; ++i) {
                const int slot = i % STAGES, use = i / STAGES;
                if (use > 0) mbar_wait(&bars->empty[slot], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                uint8_t* dst = ring + slot * SLOT_BYTES;
                mbar_expect_tx(&bars->full[slot], 2 * p.TT * ROWB);
                tma_load_3d(dst, &tm_k, 0, t0 + i * p.TT, u, &bars->full[slot]);
                tma_load_3d(dst + TILE_BYTES, &tm_v, 0, t0 + i * p.TT, u, &bars->full[slot]);
            }
            for (int j = 0; j < nqbox; ++j) {  // resident Q, behind the K/V traffic
                mbar_expect_tx(&bars->qfull[j], p.TT * ROWB);
                tma_load_3d(qreg + j * p.TT * ROWB, &tm_q, 0, t0 + j * p.TT, u, &bars->qfull[j]);
            }
        }
        __syncwarp();
        cluster_sync_all();
        cluster_sync_all();
        if (lane == 0 && n_mt > n_res_mt) {  // Q tiles beyond the resident region
            fence_proxy_async_smem();
            for (int t = n_res_mt; t < n_mt; ++t) {
                const int k = t - n_res_mt, slot = k & 1, use = k >> 1;
                if (use > 0) mbar_wait(&bars->sempty[slot], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                mbar_expect_tx(&bars->sfull[slot], MT * ROWB);
                tma_load_3d(ring + slot * SLOT_BYTES, &tm_q128, 0, t0 + t * MT, u, &bars->sfull[slot]);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ================================ MMA issuer =====================================
        if (lane == 0) {
            for (int i = 0; i < nkv; ++i) {
                const int slot = i % STAGES, use = i / STAGES;
                mbar_wait(&bars->full[slot], use & 1, TTT_DEVERR_TIMEOUT_TMA);
                tc::fence_after();
                const uint32_t kb = smem_u32(ring + slot * SLOT_BYTES);
                const int ks_n = (p.TT + 15) / 16;
                for (int ks = 0; ks < ks_n; ++ks) {
                    // A = [K | V]^T: MN-major, atoms K tile / V tile (LBO), 8-token groups (SBO)
                    const uint64_t a = tc::smem_desc(kb + ks * 2048, TILE_BYTES, 1024, 2);
                    const uint64_t b = tc::smem_desc(kb + ks * 2048, TILE_BYTES, 1024, 2);
                    tc::mma_bf16(tmem, a, b, IDESC_GRAM, (i > 0 || ks > 0) ? 1 : 0);
                }
                tc::commit(&bars->empty[slot]);
            }
            if (nkv > 0) tc::commit(&bars->gram_done);
        }
        __syncwarp();
        cluster_sync_all();
        cluster_sync_all();
        if (lane == 0 && n_mt > 0) {
            fence_proxy_async_smem();
            tc::fence_after();
            const uint32_t wb = smem_u32(wt);
            for (int t = 0; t < n_mt; ++t) {
                const int buf = t & 3;
                if (t >= 4) mbar_wait(&bars->tempty[buf], ((t >> 2) - 1) & 1, TTT_DEVERR_TIMEOUT_PEER);
                uint32_t ab;
                if (t < n_res_mt) {
                    const int r_lo = t * MT, r_hi = min(q_valid, r_lo + MT) - 1;
                    for (int j = r_lo / p.TT; j <= r_hi / p.TT; ++j)
                        mbar_wait(&bars->qfull[j], 0, TTT_DEVERR_TIMEOUT_TMA);
                    ab = smem_u32(qreg) + t * MT * ROWB;
                } else {
                    const int k = t - n_res_mt;
                    mbar_wait(&bars->sfull[k & 1], (k >> 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                    ab = smem_u32(ring) + (k & 1) * SLOT_BYTES;
                }
                tc::fence_after();
                const uint32_t d = tmem + buf * 64;
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t a = tc::smem_desc(ab + ks * 32, 16, 1024, 2);
                        const uint64_t b = tc::smem_desc(wb + part * WT_BYTES + ks * 32, 16, 1024, 2);
                        tc::mma_bf16(d, a, b, IDESC_APPLY, (part | ks) ? 1 : 0);
                    }
                tc::commit(&bars->tfull[buf]);
            }
        }
        __syncwarp();
    } else {
        // ================================ epilogue =======================================
        const int q4 = warp & 3;              // TMEM lane quarter this warp may access
        const int row = q4 * 32 + lane;       // accumulator row (lane) owned by this thread
        const int et = threadIdx.x - 64;      // 0..127
        const int jc = et & 63;               // W* column this thread forms
        const float* W0 = p.w0 + (size_t)(u % p.H) * D * D;
        float w0c[D];                         // column jc of W0, loaded while phase 1 runs
#pragma unroll
        for (int m = 0; m < D; ++m) w0c[m] = __ldg(&W0[m * D + jc]);

        // ---- partial [G ; C^T] of this CTA: TMEM -> shared scratch --------------------
        float acc[64];
        if (nkv > 0) {
            mbar_wait(&bars->gram_done, 0, TTT_DEVERR_TIMEOUT_TMA);
            tc::fence_after();
#pragma unroll
            for (int c = 0; c < 64; c += 16) tc::ld16(tmem + ((uint32_t)(q4 * 32) << 16) + c, &acc[c]);
            tc::wait_ld();
        } else {
#pragma unroll
            for (int c = 0; c < 64; ++c) acc[c] = 0.f;
        }
        fence_proxy_async_smem();  // the ring was last touched by TMA and the tensor cores
#pragma unroll
        for (int c = 0; c < 64; c += 4)
            *reinterpret_cast<float4*>(&scr[scr_idx(row, c)]) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
        tc::fence_before();
        cluster_sync_all();

        // ---- sum over the cluster, rows of W* [r0, r0 + rp) -----------------------------
        const int rp = D / (int)S;
        const int r0 = (int)rank * rp;
        if (S > 1) {
            const int n_g = rp * 16;  // float4 items of G rows r0..; then C^T columns r0..
            const int n_c = 64 * (rp / 4);
            for (int it = et; it < n_g + n_c; it += 128) {
                int r, c;
                if (it < n_g) {
                    r = r0 + it / 16;
                    c = (it % 16) * 4;
                } else {
                    const int k = it - n_g;
                    r = 64 + k / (rp / 4);
                    c = r0 + (k % (rp / 4)) * 4;
                }
                float* loc = &scr[scr_idx(r, c)];
                float4 part[8];
                float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                for (uint32_t q0 = 0; q0 < S; q0 += 8) {
                    const uint32_t nq = min(8u, S - q0);
#pragma unroll
                    for (uint32_t q = 0; q < 8; ++q)
                        if (q < nq) part[q] = dsmem_ld_f4(dsmem_map(loc, q0 + q));
#pragma unroll
                    for (uint32_t q = 0; q < 8; ++q)
                        if (q < nq) {
                            sum.x += part[q].x;
                            sum.y += part[q].y;
                            sum.z += part[q].z;
                            sum.w += part[q].w;
                        }
                }
                *reinterpret_cast<float4*>(loc) = sum;
            }
            epi_sync();
        }

        // ---- W*[i][jc] = W0[i][jc] - (eta/N)(sum_m G[i][m] W0[m][jc] - C[i][jc]) -----------
        {
            const int pairs = rp / 2;
            for (int pi = et >> 6; pi < pairs; pi += 2) {
                const int i = r0 + 2 * pi;
                float s0 = 0.f, s1 = 0.f;
#pragma unroll
                for (int m = 0; m < D; m += 4) {
                    const float4 g0 = *reinterpret_cast<const float4*>(&scr[scr_idx(i, m)]);
                    const float4 g1 = *reinterpret_cast<const float4*>(&scr[scr_idx(i + 1, m)]);
                    s0 = fmaf(g0.x, w0c[m], s0);
                    s0 = fmaf(g0.y, w0c[m + 1], s0);
                    s0 = fmaf(g0.z, w0c[m + 2], s0);
                    s0 = fmaf(g0.w, w0c[m + 3], s0);
                    s1 = fmaf(g1.x, w0c[m], s1);
                    s1 = fmaf(g1.y, w0c[m + 1], s1);
                    s1 = fmaf(g1.z, w0c[m + 2], s1);
                    s1 = fmaf(g1.w, w0c[m + 3], s1);
                }
                const float c0 = scr[scr_idx(64 + jc, i)], c1 = scr[scr_idx(64 + jc, i + 1)];
                const float wa = __ldg(&W0[i * D + jc]) - p.eta_over_n * (s0 - c0);
                const float wb = __ldg(&W0[(i + 1) * D + jc]) - p.eta_over_n * (s1 - c1);
                if (p.w_star) {
                    float* ws = p.w_star + (size_t)u * D * D;
                    ws[i * D + jc] = wa;
                    ws[(i + 1) * D + jc] = wb;
                }
                const __nv_bfloat162 hi = __floats2bfloat162_rn(wa, wb);
                const uint32_t phi = *reinterpret_cast<const uint32_t*>(&hi);
                const uint32_t plo = pack_bf16(wa - __low2float(hi), wb - __high2float(hi));
                uint8_t* dst = wt + swz<3>(jc * ROWB + i * 2);  // W*^T[jc][i..i+1]
                for (uint32_t q = 0; q < S; ++q) {
                    dsmem_st_u32(dsmem_map(dst, q), phi);
                    dsmem_st_u32(dsmem_map(dst + WT_BYTES, q), plo);
                }
            }
        }
        fence_proxy_async_all();  // W*^T is read next by the tensor cores of every CTA
        cluster_sync_all();

        // ---- O tiles: TMEM -> bf16 in place over Q -> TMA store ----------------------------
        for (int t = 0; t < n_mt; ++t) {
            const int buf = t & 3;
            mbar_wait(&bars->tfull[buf], (t >> 2) & 1, TTT_DEVERR_TIMEOUT_PEER);
            tc::fence_after();
            float o[64];
#pragma unroll
            for (int c = 0; c < 64; c += 16) tc::ld16(tmem + ((uint32_t)(q4 * 32) << 16) + buf * 64 + c, &o[c]);
            tc::wait_ld();
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->tempty[buf]);
            const bool streamed = t >= n_res_mt;
            uint8_t* tile = streamed ? ring + ((t - n_res_mt) & 1) * SLOT_BYTES : qreg + t * MT * ROWB;
            const int tok = t * MT + row;  // token index inside this CTA
            if (tok < n_valid) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint4 v;
                    v.x = pack_bf16(o[8 * c + 0], o[8 * c + 1]);
                    v.y = pack_bf16(o[8 * c + 2], o[8 * c + 3]);
                    v.z = pack_bf16(o[8 * c + 4], o[8 * c + 5]);
                    v.w = pack_bf16(o[8 * c + 6], o[8 * c + 7]);
                    *reinterpret_cast<uint4*>(tile + swz<3>(row * ROWB + c * 16)) = v;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                for (int k = 0; k < 4; ++k) {
                    const int r8 = q4 * 32 + 8 * k;  // 8-row box inside the tile
                    if (t * MT + r8 < n_valid) tma_store_3d(&tm_o, 0, t0 + t * MT + r8, u, tile + r8 * ROWB);
                }
                tma_store_commit();
                if (streamed) {
                    tma_store_wait_read_all();
                    mbar_arrive(&bars->sempty[(t - n_res_mt) & 1]);
                }
            }
            __syncwarp();
        }
        if (lane == 0) tma_store_wait_all();
    }

    tc::fence_before();
    __syncthreads();
    if (warp == 1) tc::dealloc(tmem, TMEM_COLS);
}

}  // namespace lin5

// linear_tc.cuh -- TTT-Linear full-batch step for bf16 inputs, d in {32, 64}, one kernel.
//
// Operation ("ViT^3" blog, online-learning rewrite of attention, steps 1-3; TTT-Linear of the
// TTT abstract): per unit (batch b, head h) with Q, K, V in R^{N x d},
//     G = K^T K,  C = K^T V            (the full-batch gradient of (1/N) sum 1/2||k W - v||^2
//                                       at W0 is (G W0 - C) / N)
//     W* = W0 - (eta/N) (G W0 - C)
//     O  = Q W*
// Design (B200):
//   * one thread-block cluster of S CTAs per unit; CTA r owns tokens [r*T, (r+1)*T);
//   * a producer warp streams K/V tiles through a TMA ring (128B/64B-swizzled, no multicast)
//     and prefetches this CTA's Q tiles into a resident region at the start, so Q's HBM
//     traffic overlaps the Gram pass and the in-cluster reduction;
//   * four consumer warps accumulate [G | C] = K^T [K | V] on bf16 tensor cores (fp32
//     accumulate), then the S partials are summed in fixed rank order through distributed
//     shared memory (each CTA reduces D/S rows, deterministic, no atomics, no spinning);
//   * each CTA forms its rows of W* in fp32 and broadcasts them into every CTA of the cluster
//     as two bf16 matrices W*^T = hi + lo (hi = bf16(W*), lo = bf16(W* - hi): about 16
//     mantissa bits, so the apply adds no error beyond the bf16 rounding of O itself);
//   * after a second cluster barrier it computes O = Q hi + Q lo from shared memory, writes
//     O in place over Q and stores it with TMA (the hardware clips rows >= N).
// Q tiles that do not fit the resident region are streamed through the ring after the
// reduction.  All waits are bounded (see common.cuh).
#pragma once
#include "common.cuh"

namespace lintc {

constexpr int CONSUMER_WARPS = 4;
constexpr int THREADS = (CONSUMER_WARPS + 1) * 32;
constexpr int TILE_ROWS = 64;  // shared-memory rows reserved per tile (tile tokens TT <= 64)

template <int D>
struct Cfg {
    static constexpr int ROWB = D * 2;                      // bytes per token row
    static constexpr int SW = (D == 64) ? 3 : 2;            // swizzle: 128B (D=64), 64B (D=32)
    static constexpr int TILE_BYTES = TILE_ROWS * ROWB;     // one tensor tile in a ring slot
    static constexpr int SLOT_BYTES = 2 * TILE_BYTES;       // K tile + V tile
    static constexpr int WT_BYTES = D * D * 2;              // one bf16 copy of W*^T (hi or lo)
    static constexpr int SCR_LD = 2 * D;                    // fp32 words per scratch row
    static constexpr int SCR_BYTES = D * SCR_LD * 4;        // [G | C] partial, fp32
    static constexpr int ROW_SLABS = D / 16;                // 16-row slabs of [G | C]
    static constexpr int COL_GROUPS = CONSUMER_WARPS / ROW_SLABS;
    static constexpr int NT = (2 * D / 8) / COL_GROUPS;     // 8-column MMA tiles per warp
    static constexpr int MIN_STAGES = (SCR_BYTES + SLOT_BYTES - 1) / SLOT_BYTES;
};

struct Params {
    const float* w0;   // [H][D][D] fp32
    float* w_star;     // [U][D][D] fp32 or nullptr
    int H, N;
    int T;             // tokens per CTA (multiple of 8)
    int TT;            // tokens per tile (multiple of 8, <= 64; multiple of 16 when streaming Q)
    int tiles;         // T / TT
    int q_res;         // Q tiles kept resident (<= tiles)
    int stages;        // ring slots
    int q_region_bytes;
    float eta_over_n;
};

template <int D>
struct Layout {
    uint32_t ring, qreg, wt, bars, total;
    __host__ __device__ Layout(const Params& p) {
        using C = Cfg<D>;
        ring = 0;
        qreg = ring + p.stages * C::SLOT_BYTES;
        wt = qreg + p.q_region_bytes;
        bars = wt + 2 * C::WT_BYTES;  // W*^T hi, then W*^T lo
        total = bars + 8 * (2 * p.stages + p.q_res);
    }
};

__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int D>
__global__ void __maxnreg__(200)
    linear_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
                     const Params p) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align<1024>(smem_raw);
    const Layout<D> L(p);
    uint8_t* ring = smem + L.ring;
    uint8_t* qreg = smem + L.qreg;
    uint8_t* wt = smem + L.wt;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* empty = full + p.stages;
    uint64_t* qfull = empty + p.stages;
    float* scr = reinterpret_cast<float*>(ring);  // aliases the ring between the two phases

    const uint32_t S = gridDim.x;  // the cluster spans the whole x dimension
    const uint32_t rank = cluster_ctarank();
    const int u = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = (int)rank * p.T;
    const int n_valid = max(0, min(p.N - t0, p.T));
    const int ntiles = (n_valid + p.TT - 1) / p.TT;
    const int nres = min(ntiles, p.q_res);

    // ---- set-up: barriers, zero rows that no TMA writes but MMAs read ------------------
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], CONSUMER_WARPS);
        }
        for (int j = 0; j < p.q_res; ++j) mbar_init(&qfull[j], 1);
        mbar_fence_init();
    }
    if (p.TT < TILE_ROWS) {  // K/V rows [TT, 64) of every slot are MMA padding
        const int pad_words = (TILE_ROWS - p.TT) * C::ROWB / 16;
        for (int e = threadIdx.x; e < p.stages * 2 * pad_words; e += THREADS) {
            const int tile = e / pad_words, w = e % pad_words;
            *reinterpret_cast<uint4*>(ring + tile * C::TILE_BYTES + p.TT * C::ROWB + w * 16) = make_uint4(0, 0, 0, 0);
        }
    }
    {   // resident-Q rows beyond the loaded tiles up to the region end (16-row MMA padding)
        const int first = nres * p.TT * C::ROWB;
        for (int off = first + threadIdx.x * 16; off < p.q_region_bytes; off += THREADS * 16)
            *reinterpret_cast<uint4*>(qreg + off) = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();

    if (warp == CONSUMER_WARPS) {
        // ================================ producer warp ==================================
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_o);
            auto issue_kv = [&](int i) {
                const int slot = i % p.stages, use = i / p.stages;
                if (use > 0) mbar_wait(&empty[slot], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                uint8_t* dst = ring + slot * C::SLOT_BYTES;
                mbar_expect_tx(&full[slot], 2 * p.TT * C::ROWB);
                tma_load_3d(dst, &tm_k, 0, t0 + i * p.TT, u, &full[slot]);
                tma_load_3d(dst + C::TILE_BYTES, &tm_v, 0, t0 + i * p.TT, u, &full[slot]);
            };
            auto issue_q = [&](int j) {
                mbar_expect_tx(&qfull[j], p.TT * C::ROWB);
                tma_load_3d(qreg + j * p.TT * C::ROWB, &tm_q, 0, t0 + j * p.TT, u, &qfull[j]);
            };
            // K/V tiles first; each resident Q tile follows `stages` K/V tiles behind, so the
            // last Q tiles are in flight while the cluster reduces the Gram partials
            int jq = 0;
            for (int i = 0; i < ntiles; ++i) {
                issue_kv(i);
                if (i >= p.stages && jq < nres) issue_q(jq++);
            }
            while (jq < nres) issue_q(jq++);
        }
        __syncwarp();
        cluster_sync_all();  // partials published
        cluster_sync_all();  // W* broadcast complete; scratch free
        if (lane == 0 && ntiles > nres) {
            fence_proxy_async_smem();
            for (int j = nres; j < ntiles; ++j) {
                const int i = ntiles + (j - nres);
                const int slot = i % p.stages, use = i / p.stages;
                if (use > 0) mbar_wait(&empty[slot], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                mbar_expect_tx(&full[slot], p.TT * C::ROWB);
                tma_load_3d(ring + slot * C::SLOT_BYTES, &tm_q, 0, t0 + j * p.TT, u, &full[slot]);
            }
        }
        __syncwarp();
        return;
    }

    // =================================== consumer warps ==================================
    const int rslab = warp % C::ROW_SLABS;            // rows [16*rslab, +16) of [G | C]
    const int cgroup = warp / C::ROW_SLABS;           // columns [cgroup*NT*8, +NT*8)
    const int colbase = cgroup * C::NT * 8;
    float acc[C::NT][4];
#pragma unroll
    for (int n = 0; n < C::NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

    const int ksteps = (p.TT + 15) / 16;
    for (int i = 0; i < ntiles; ++i) {
        const int slot = i % p.stages, use = i / p.stages;
        mbar_wait(&full[slot], use & 1, TTT_DEVERR_TIMEOUT_TMA);
        const uint32_t kbase = smem_u32(ring + slot * C::SLOT_BYTES);
        const uint32_t vbase = kbase + C::TILE_BYTES;
        for (int ks = 0; ks < ksteps; ++ks) {
            // A = K^T (rows = features of this slab, cols = 16 tokens): transposed loads of K
            uint32_t a[4];
            {
                const int row = ks * 16 + (lane >> 4) * 8 + (lane & 7);
                const int chunk = rslab * 2 + ((lane >> 3) & 1);
                ldsm_x4_t(kbase + swz<C::SW>(row * C::ROWB + chunk * 16), a[0], a[1], a[2], a[3]);
            }
#pragma unroll
            for (int pp = 0; pp < C::NT / 2; ++pp) {
                const int col = colbase + pp * 16;  // 16 columns of [K | V]
                const uint32_t base = col < D ? kbase : vbase;
                const int ccol = col < D ? col : col - D;
                const int row = ks * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
                const int chunk = ccol / 8 + (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(base + swz<C::SW>(row * C::ROWB + chunk * 16), b0, b1, b2, b3);
                mma_bf16(acc[2 * pp], a, b0, b1);
                mma_bf16(acc[2 * pp + 1], a, b2, b3);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
    }

    // ---- publish this CTA's partial [G | C] (fp32) in the scratch that aliases the ring ---
    consumers_sync();  // every consumer is done reading the ring
#pragma unroll
    for (int n = 0; n < C::NT; ++n) {
        const int row = rslab * 16 + (lane >> 2);
        const int col = colbase + n * 8 + 2 * (lane & 3);
        *reinterpret_cast<float2*>(&scr[row * C::SCR_LD + col]) = make_float2(acc[n][0], acc[n][1]);
        *reinterpret_cast<float2*>(&scr[(row + 8) * C::SCR_LD + col]) = make_float2(acc[n][2], acc[n][3]);
    }
    cluster_sync_all();

    // ---- reduce rows [r0, r0 + D/S) over the S CTAs in rank order (in place, own rows) ----
    const int rows_per = D / (int)S;
    const int r0 = (int)rank * rows_per;
    const int tid = threadIdx.x;  // 0..127
    if (S > 1) {
        constexpr int V4 = 2 * D / 4;
        for (int it = tid; it < rows_per * V4; it += 128) {
            const int row = r0 + it / V4, c4 = it % V4;
            float* loc = &scr[row * C::SCR_LD + 4 * c4];
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
            for (uint32_t q = 0; q < S; ++q) {
                const float4 x = dsmem_ld_f4(dsmem_map(loc, q));
                sum.x += x.x;
                sum.y += x.y;
                sum.z += x.z;
                sum.w += x.w;
            }
            *reinterpret_cast<float4*>(loc) = sum;
        }
        consumers_sync();
    }

    // ---- W* rows: W*[i][j] = W0[i][j] - (eta/N)(sum_m G[i][m] W0[m][j] - C[i][j]) ----------
    {
        const float* W0 = p.w0 + (size_t)(u % p.H) * D * D;
        const int pairs = rows_per / 2;
        for (int it = tid; it < pairs * D; it += 128) {
            const int i = r0 + 2 * (it / D), j = it % D;
            const float* g0 = &scr[i * C::SCR_LD];
            const float* g1 = g0 + C::SCR_LD;
            float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
            for (int m = 0; m < D; ++m) {
                const float w = __ldg(&W0[m * D + j]);
                s0 = fmaf(g0[m], w, s0);
                s1 = fmaf(g1[m], w, s1);
            }
            const float wa = __ldg(&W0[i * D + j]) - p.eta_over_n * (s0 - g0[D + j]);
            const float wb = __ldg(&W0[(i + 1) * D + j]) - p.eta_over_n * (s1 - g1[D + j]);
            if (p.w_star) {
                float* ws = p.w_star + (size_t)u * D * D;
                ws[i * D + j] = wa;
                ws[(i + 1) * D + j] = wb;
            }
            // W*^T[j][i], W*^T[j][i+1] as hi and lo bf16 pairs
            const __nv_bfloat162 hi = __floats2bfloat162_rn(wa, wb);
            const uint32_t phi = *reinterpret_cast<const uint32_t*>(&hi);
            const uint32_t plo = pack_bf16(wa - __low2float(hi), wb - __high2float(hi));
            uint8_t* dst = wt + swz<C::SW>(j * C::ROWB + i * 2);
            for (uint32_t q = 0; q < S; ++q) {
                dsmem_st_u32(dsmem_map(dst, q), phi);
                dsmem_st_u32(dsmem_map(dst + C::WT_BYTES, q), plo);
            }
        }
    }
    cluster_sync_all();

    // ---- O = Q W* -------------------------------------------------------------------------
    uint32_t bw[2][D / 8][D / 16][2];  // [hi|lo][n-tile][k-step][reg]
#pragma unroll
    for (int part = 0; part < 2; ++part) {
        const uint32_t wbase = smem_u32(wt) + part * C::WT_BYTES;
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
            for (int ks = 0; ks < D / 16; ks += 2) {
                const int row = nt * 8 + (lane & 7);
                const int chunk = 2 * ks + (lane >> 3);
                ldsm_x4(wbase + swz<C::SW>(row * C::ROWB + chunk * 16), bw[part][nt][ks][0],
                        bw[part][nt][ks][1], bw[part][nt][ks + 1][0], bw[part][nt][ks + 1][1]);
            }
    }
    auto mtile = [&](uint8_t* rows, int valid_rows, int tok) {
        // rows: 16 token rows (swizzle-atom aligned); valid_rows <= 16 of them are stored
        const uint32_t abase = smem_u32(rows);
        float o[D / 8][4];
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t a[4];
            const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
            const int chunk = 2 * ks + (lane >> 4);
            ldsm_x4(abase + swz<C::SW>(row * C::ROWB + chunk * 16), a[0], a[1], a[2], a[3]);
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt) {
                mma_bf16(o[nt], a, bw[0][nt][ks][0], bw[0][nt][ks][1]);
                mma_bf16(o[nt], a, bw[1][nt][ks][0], bw[1][nt][ks][1]);
            }
        }
        __syncwarp();
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
            const int row = lane >> 2, col = nt * 8 + 2 * (lane & 3);
            *reinterpret_cast<uint32_t*>(rows + swz<C::SW>(row * C::ROWB + col * 2)) = pack_bf16(o[nt][0], o[nt][1]);
            *reinterpret_cast<uint32_t*>(rows + swz<C::SW>((row + 8) * C::ROWB + col * 2)) =
                pack_bf16(o[nt][2], o[nt][3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_3d(&tm_o, 0, tok, u, rows);
            if (valid_rows > 8) tma_store_3d(&tm_o, 0, tok + 8, u, rows + 8 * C::ROWB);
            tma_store_commit();
        }
    };

    // resident Q: rows [0, R) of the region, 16-row tiles dealt round-robin to the warps
    const int R = min(n_valid, nres * p.TT);
    for (int mt = warp; mt * 16 < R; mt += CONSUMER_WARPS) {
        const int j_lo = (mt * 16) / p.TT, j_hi = min(R - 1, mt * 16 + 15) / p.TT;
        for (int j = j_lo; j <= j_hi; ++j) mbar_wait(&qfull[j], 0, TTT_DEVERR_TIMEOUT_TMA);
        mtile(qreg + mt * 16 * C::ROWB, min(16, R - mt * 16), t0 + mt * 16);
    }
    // streamed Q tiles (TT is a multiple of 16 here): tile rows [16w, 16w + 16) go to warp w
    for (int j = nres; j < ntiles; ++j) {
        const int i = ntiles + (j - nres);
        const int slot = i % p.stages, use = i / p.stages;
        mbar_wait(&full[slot], use & 1, TTT_DEVERR_TIMEOUT_TMA);
        const int rows = min(p.TT, n_valid - j * p.TT);
        if (warp * 16 < rows)
            mtile(ring + slot * C::SLOT_BYTES + warp * 16 * C::ROWB, min(16, rows - warp * 16),
                  t0 + j * p.TT + warp * 16);
        if (lane == 0) tma_store_wait_read_all();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
    }
    if (lane == 0) tma_store_wait_all();
}

}  // namespace lintc

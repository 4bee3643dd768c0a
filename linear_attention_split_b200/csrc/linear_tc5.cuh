// linear_tc5.cuh -- TTT-Linear full-batch step on the 5th-generation tensor cores (tcgen05),
// bf16 inputs, d = 64, one kernel per call.
//
// Operation ("ViT^3" blog, online-learning rewrite of attention, steps 1-3; TTT-Linear of the
// TTT abstract), per unit u = (batch b, head h) with Q, K, V in R^{N x 64}:
//     G = K^T K,  C = K^T V,   W* = W0 - (eta/N) (G W0 - C),   O = Q W*
// ((G W0 - C)/N is the full-batch gradient of (1/N) sum_i 1/2 ||k_i W - v_i||^2 at W0.)
//
// Layout of the work (one thread-block cluster of S CTAs per unit, S in {1, 2, 4, 8}; CTA r
// owns tokens [r*T, r*T + T); warp 0 = TMA producer, warp 1 = MMA issuer, warps 2-5 =
// epilogue).  Shared memory is one pool used three ways in turn:
//   1. Gram pass: the whole pool is a ring of 16 KB K/V slots (128-byte swizzle, plain TMA,
//      no multicast); the issuer computes [G ; C^T] = [K | V]^T K with tcgen05.mma, M = 128
//      (features of K then of V), N = 64, K-dim = tokens, both operands MN-major straight
//      from the tiles, fp32 accumulator in tensor memory (TMEM).  Once the last K/V tile has
//      landed the producer prefetches this CTA's Q rows into L2 (no shared memory needed).
//   2. Reduction: the epilogue writes the partial as fp32 rows [G | C] (scratch).  After one
//      cluster barrier each CTA pushes row block r' of its partial to CTA r' with bulk
//      copies (completion counted on the receiver's mbarrier); CTA r adds the S blocks of
//      rows [64r/S, 64(r+1)/S) in rank order (deterministic, no atomics), forms those rows of
//      W* in fp32, stores them as bf16 hi + lo (hi = bf16(W*), lo = bf16(W* - hi)) in an
//      MN-major block and pushes that block to every other CTA the same way.
//   3. Apply: Q is copied from L2 into the region the received partials occupied, the issuer
//      computes O = Q hi + Q lo per 128-token tile into four TMEM buffers, and the epilogue
//      converts O to bf16 in place over Q and stores it with TMA (rows >= N are clipped).
// If a CTA's Q rows do not fit the resident region, the rest stream through the scratch area
// at the end.  A split cluster barrier (arrive once everything destined to a CTA has arrived,
// wait before exit) keeps every pushed-from buffer alive until its copies are done.  Every
// wait is bounded (common.cuh).
#pragma once
#include "common.cuh"

namespace lin5 {

constexpr int D = 64;
constexpr int ROWB = 128;                 // bytes per token row (64 bf16)
constexpr int THREADS = 192;              // producer, issuer, 4 epilogue warps
constexpr int TILE_ROWS = 64;             // rows reserved per K or V tile in a ring slot
constexpr int TILE_BYTES = TILE_ROWS * ROWB;
constexpr int SLOT_BYTES = 2 * TILE_BYTES;  // K tile, V tile
constexpr int MAX_SLOTS = 12;
constexpr int SCR_LD = 2 * D;             // scratch row: G[i][0..63] | C[i][0..63], fp32
constexpr int SCR_BYTES = D * SCR_LD * 4; // 32 KB
constexpr int RECV_OFF = SCR_BYTES;       // received partial blocks, later the Q region
constexpr int WG_BYTES = 2048;            // one 8-row group of W*: hi atom, then lo atom
constexpr int W_BYTES = 8 * WG_BYTES;
constexpr int MT = 128;                   // tokens per phase-2 MMA tile
constexpr int TMEM_COLS = 256;            // phase-1 accumulator, then four phase-2 buffers
constexpr int MAX_QBOX = 32;              // resident Q TMA boxes per CTA
constexpr uint32_t IDESC_GRAM = tc::idesc_bf16(128, 64, 1, 1);
constexpr uint32_t IDESC_APPLY = tc::idesc_bf16(128, 64, 0, 1);

struct Params {
    const float* w0;   // [H][64][64]
    float* w_star;     // [U][64][64] or nullptr
    int H, N;
    int T;             // tokens per CTA
    int TT;            // tokens per K/V tile (multiple of 8, <= 64)
    int q_rows;        // resident Q rows (multiple of 8; multiple of 128 when Q streams)
    int w_off;         // byte offset of the W* block area in the pool
    int slots;         // K/V ring slots during the Gram pass (pool / 16 KB)
    float eta_over_n;
};

struct Bars {
    uint64_t full[MAX_SLOTS], empty[MAX_SLOTS], qfull[MAX_QBOX], gram_done, rfull, wfull, qgo, tfull[4],
        tempty[4], sfull[2], sempty[2];
    uint32_t tmem_base;
};

__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ void wready_sync() { asm volatile("bar.sync 2, 160;" ::: "memory"); }

// scratch [64 rows][128 cols] fp32; float4 chunks XOR-swizzled by row to spread banks
__device__ __forceinline__ int scr_idx(int r, int c) { return r * SCR_LD + ((((c >> 2) ^ (r & 31))) << 2) + (c & 3); }
// W* element (i, j) of part p (0 = hi, 1 = lo): MN-major, 128-byte swizzled 8-row groups
__device__ __forceinline__ uint32_t w_off(int i, int j, int p) {
    return (i >> 3) * WG_BYTES + p * 1024 + swz<3>((i & 7) * ROWB + j * 2);
}

__global__ void __launch_bounds__(THREADS, 2)
    linear_tc5_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_q128,
                      const __grid_constant__ CUtensorMap tm_o8, const __grid_constant__ CUtensorMap tm_o32,
                      const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* pool = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* scr = reinterpret_cast<float*>(pool);
    uint8_t* recv = pool + RECV_OFF;
    uint8_t* qreg = pool + RECV_OFF;
    uint8_t* wblk = pool + p.w_off;
    Bars* bars = reinterpret_cast<Bars*>(pool + p.w_off + W_BYTES);

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
    const int rp = D / (int)S;                                       // W* rows formed here
    const int r0 = (int)rank * rp;
    const uint32_t pblk_bytes = (uint32_t)rp * SCR_LD * 4;           // one partial row block
    const uint32_t wblk_bytes = (uint32_t)rp / 8 * WG_BYTES;         // one W* row block

    // ---- set-up ------------------------------------------------------------------------
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.slots; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int j = 0; j < MAX_QBOX; ++j) mbar_init(&bars->qfull[j], 1);
        mbar_init(&bars->gram_done, 1);
        mbar_init(&bars->rfull, 1);
        mbar_init(&bars->wfull, 1);
        mbar_init(&bars->qgo, 128);
        for (int b = 0; b < 4; ++b) {
            mbar_init(&bars->tfull[b], 1);
            mbar_init(&bars->tempty[b], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->sfull[b], 1);
            mbar_init(&bars->sempty[b], 4);
        }
        mbar_fence_init();
        // partial blocks and W* blocks of the S-1 other CTAs land here (bulk copies, in bytes)
        mbar_expect_tx(&bars->rfull, (S - 1) * pblk_bytes);
        mbar_expect_tx(&bars->wfull, (S - 1) * wblk_bytes);
    }
    if (p.TT < TILE_ROWS) {  // token rows [TT, 64) of every K/V tile: zero K-dim padding
        const int pad16 = (TILE_ROWS - p.TT) * ROWB / 16;
        for (int e = threadIdx.x; e < p.slots * 2 * pad16; e += THREADS) {
            const int tile = e / pad16, w = e % pad16;
            *reinterpret_cast<uint4*>(pool + tile * TILE_BYTES + p.TT * ROWB + w * 16) = make_uint4(0, 0, 0, 0);
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
                const int slot = i % p.slots, use = i / p.slots;
                if (use > 0) mbar_wait(&bars->empty[slot], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                uint8_t* dst = pool + slot * SLOT_BYTES;
                mbar_expect_tx(&bars->full[slot], 2 * p.TT * ROWB);
                tma_load_3d(dst, &tm_k, 0, t0 + i * p.TT, u, &bars->full[slot]);
                tma_load_3d(dst + TILE_BYTES, &tm_v, 0, t0 + i * p.TT, u, &bars->full[slot]);
            }
            // Q to L2 once the last K/V tile has landed: the Gram pass gets the bandwidth first
            if (nkv > 0)
                mbar_wait(&bars->full[(nkv - 1) % p.slots], ((nkv - 1) / p.slots) & 1, TTT_DEVERR_TIMEOUT_TMA);
            for (int j = 0; j < nqbox; ++j) tma_prefetch_l2_3d(&tm_q, 0, t0 + j * p.TT, u);
        }
        __syncwarp();
        cluster_sync_all();          // all Gram passes done: pools of every CTA may receive
        if (lane == 0) {             // Q into shared memory once the received partials are summed
            mbar_wait(&bars->qgo, 0, TTT_DEVERR_TIMEOUT_PEER);
            fence_proxy_async_smem();
            for (int j = 0; j < nqbox; ++j) {
                mbar_expect_tx(&bars->qfull[j], p.TT * ROWB);
                tma_load_3d(qreg + j * p.TT * ROWB, &tm_q, 0, t0 + j * p.TT, u, &bars->qfull[j]);
            }
        }
        __syncwarp();
        cluster_arrive_relaxed();
        cluster_wait_acquire();      // every CTA received everything: scratch reusable
        if (lane == 0 && n_mt > n_res_mt) {  // Q tiles beyond the resident region
            fence_proxy_async_smem();
            for (int t = n_res_mt; t < n_mt; ++t) {
                const int k = t - n_res_mt, slot = k & 1, use = k >> 1;
                if (use > 0) mbar_wait(&bars->sempty[slot], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                mbar_expect_tx(&bars->sfull[slot], MT * ROWB);
                tma_load_3d(pool + slot * SLOT_BYTES, &tm_q128, 0, t0 + t * MT, u, &bars->sfull[slot]);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ================================ MMA issuer =====================================
        if (lane == 0) {
            for (int i = 0; i < nkv; ++i) {
                const int slot = i % p.slots, use = i / p.slots;
                mbar_wait(&bars->full[slot], use & 1, TTT_DEVERR_TIMEOUT_TMA);
                tc::fence_after();
                const uint32_t kb = smem_u32(pool + slot * SLOT_BYTES);
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
        wready_sync();  // this CTA's own W* block is written
        if (lane == 0) mbar_wait(&bars->wfull, 0, TTT_DEVERR_TIMEOUT_PEER);  // and the peers' blocks
        __syncwarp();
        cluster_arrive_relaxed();
        if (lane == 0 && n_mt > 0) {
            tc::fence_after();
            const uint32_t wb = smem_u32(wblk);
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
                    ab = smem_u32(pool) + (k & 1) * SLOT_BYTES;
                }
                tc::fence_after();
                const uint32_t d = tmem + buf * 64;
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        // A = Q tile, K-major; B = W* (rows = K-dim), MN-major, 8-row groups 2 KB apart
                        const uint64_t a = tc::smem_desc(ab + ks * 32, 16, 1024, 2);
                        const uint64_t b = tc::smem_desc(wb + part * 1024 + ks * 2 * WG_BYTES, 16384, WG_BYTES, 2);
                        tc::mma_bf16(d, a, b, IDESC_APPLY, (part | ks) ? 1 : 0);
                    }
                tc::commit(&bars->tfull[buf]);
            }
        }
        __syncwarp();
        cluster_wait_acquire();
    } else {
        // ================================ epilogue =======================================
        const int q4 = warp & 3;              // TMEM lane quarter this warp may access
        const int row = q4 * 32 + lane;       // accumulator row (lane) owned by this thread
        const int et = threadIdx.x - 64;      // 0..127
        const int jc = et & 63;               // W* column this thread forms
        const float* W0 = p.w0 + (size_t)(u % p.H) * D * D;

        // ---- partial of this CTA: TMEM -> scratch rows [G | C] -------------------------
        {
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
            fence_proxy_async_smem();  // the pool was last touched by TMA and the tensor cores
            if (row < 64) {            // row `row` of G
#pragma unroll
                for (int c = 0; c < 64; c += 4)
                    *reinterpret_cast<float4*>(&scr[scr_idx(row, c)]) =
                        make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
            } else {                   // row j of C^T = column j of C
                const int j = row - 64;
#pragma unroll
                for (int i = 0; i < 64; ++i) scr[scr_idx(i, 64 + j)] = acc[i];
            }
        }
        fence_proxy_async_smem();      // the scratch is read next by bulk copies
        // column jc of W0, requested now so that the loads fly during the exchange below
        float w0c[D], w0r[4];  // and W0[i][jc] for this thread's first four rows of W*
#pragma unroll
        for (int m = 0; m < D; ++m)
            asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(w0c[m]) : "l"(W0 + m * D + jc));
#pragma unroll
        for (int k = 0; k < 4; ++k)
            asm volatile("ld.global.nc.f32 %0, [%1];"
                         : "=f"(w0r[k])
                         : "l"(W0 + min(r0 + (et >> 6) + 2 * k, D - 1) * D + jc));
        tc::fence_before();
        cluster_sync_all();            // every CTA of the cluster is past its Gram pass

        // ---- reduce-scatter: push block r' to CTA r', then sum the blocks of rows r0.. -----
        if (S > 1) {
            if (et == 0) {
                for (uint32_t k = 1; k < S; ++k) {
                    const uint32_t dst = (rank + k) % S;
                    // slot of this CTA in the receiver's area: (rank - dst - 1) mod S
                    const uint32_t slot = (rank + S - dst - 1) % S;
                    bulk_push(reinterpret_cast<const uint8_t*>(scr) + dst * pblk_bytes, recv + slot * pblk_bytes,
                              &bars->rfull, dst, pblk_bytes);
                }
            }
            mbar_wait(&bars->rfull, 0, TTT_DEVERR_TIMEOUT_PEER);
            // the S blocks of rows r0.. in rank order; every block has the same in-block layout
            const uint32_t scr_a = smem_u32(scr), recv_a = smem_u32(recv) - (uint32_t)r0 * SCR_LD * 4;
            const int items = rp * (SCR_LD / 4);
            for (int it = et; it < items; it += 128) {
                const uint32_t off = (uint32_t)scr_idx(r0 + it / 32, (it % 32) * 4) * 4;
                float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                for (uint32_t q = 0; q < S; ++q) {
                    const uint32_t slot = (q + S - rank - 1) % S;
                    const uint32_t a = (q == rank) ? scr_a + off : recv_a + slot * pblk_bytes + off;
                    float4 x;
                    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                 : "=f"(x.x), "=f"(x.y), "=f"(x.z), "=f"(x.w)
                                 : "r"(a));
                    sum.x += x.x;
                    sum.y += x.y;
                    sum.z += x.z;
                    sum.w += x.w;
                }
                *reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(scr) + off) = sum;
            }
        }
        fence_proxy_async_smem();      // the receive area is written next by TMA (Q)
        mbar_arrive(&bars->qgo);
        epi_sync();

        // ---- W*[i][jc] = W0[i][jc] - (eta/N)(sum_m G[i][m] W0[m][jc] - C[i][jc]) -------------
        // rows r0 + (et>>6) + 2k, four at a time with split accumulators (independent chains)
        for (int i0 = r0 + (et >> 6); i0 < r0 + rp; i0 += 8) {
            float w0i[4], cij[4], s0[4], s1[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = min(i0 + 2 * k, D - 1);
                w0i[k] = (i0 == r0 + (et >> 6)) ? w0r[k] : __ldg(&W0[i * D + jc]);  // W0[i][jc]
                cij[k] = scr[scr_idx(i, 64 + jc)];
                s0[k] = 0.f;
                s1[k] = 0.f;
            }
#pragma unroll
            for (int m = 0; m < D; m += 8) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = min(i0 + 2 * k, D - 1);
                    const float4 g0 = *reinterpret_cast<const float4*>(&scr[scr_idx(i, m)]);
                    const float4 g1 = *reinterpret_cast<const float4*>(&scr[scr_idx(i, m + 4)]);
                    s0[k] = fmaf(g0.x, w0c[m], s0[k]);
                    s1[k] = fmaf(g0.y, w0c[m + 1], s1[k]);
                    s0[k] = fmaf(g0.z, w0c[m + 2], s0[k]);
                    s1[k] = fmaf(g0.w, w0c[m + 3], s1[k]);
                    s0[k] = fmaf(g1.x, w0c[m + 4], s0[k]);
                    s1[k] = fmaf(g1.y, w0c[m + 5], s1[k]);
                    s0[k] = fmaf(g1.z, w0c[m + 6], s0[k]);
                    s1[k] = fmaf(g1.w, w0c[m + 7], s1[k]);
                }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = i0 + 2 * k;
                const float w = w0i[k] - p.eta_over_n * ((s0[k] + s1[k]) - cij[k]);
                const float hi = __bfloat162float(__float2bfloat16_rn(w));
                const float lo = w - hi;
                const float hi_n = __shfl_xor_sync(0xffffffffu, hi, 1);
                const float lo_n = __shfl_xor_sync(0xffffffffu, lo, 1);
                if (i < r0 + rp) {
                    if (p.w_star) p.w_star[(size_t)u * D * D + i * D + jc] = w;
                    if ((jc & 1) == 0) {  // columns jc, jc+1 as one bf16 pair
                        *reinterpret_cast<uint32_t*>(wblk + w_off(i, jc, 0)) = pack_bf16(hi, hi_n);
                        *reinterpret_cast<uint32_t*>(wblk + w_off(i, jc, 1)) = pack_bf16(lo, lo_n);
                    }
                }
            }
        }
        fence_proxy_async_smem();  // read next by the bulk copies and the tensor cores
        wready_sync();
        if (et == 0) {
            const uint8_t* src = wblk + (r0 >> 3) * WG_BYTES;
            for (uint32_t k = 1; k < S; ++k) bulk_push(src, src, &bars->wfull, (rank + k) % S, wblk_bytes);
        }
        cluster_arrive_relaxed();  // all partials destined here arrived and were consumed

        // ---- O tiles: TMEM -> bf16 in place over Q -> TMA store; the next tile's accumulator
        //      is read from TMEM while the current one is converted and stored
        float o[64];
        if (n_mt > 0) {
            mbar_wait(&bars->tfull[0], 0, TTT_DEVERR_TIMEOUT_PEER);
            tc::fence_after();
#pragma unroll
            for (int c = 0; c < 64; c += 16) tc::ld16(tmem + ((uint32_t)(q4 * 32) << 16) + c, &o[c]);
            tc::wait_ld();
        }
        for (int t = 0; t < n_mt; ++t) {
            const int buf = t & 3;
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) pk[c] = pack_bf16(o[2 * c], o[2 * c + 1]);
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->tempty[buf]);
            if (t + 1 < n_mt) {  // start reading the next accumulator
                const int nb = (t + 1) & 3;
                mbar_wait(&bars->tfull[nb], ((t + 1) >> 2) & 1, TTT_DEVERR_TIMEOUT_PEER);
                tc::fence_after();
#pragma unroll
                for (int c = 0; c < 64; c += 16) tc::ld16(tmem + ((uint32_t)(q4 * 32) << 16) + nb * 64 + c, &o[c]);
            }
            const bool streamed = t >= n_res_mt;
            uint8_t* tile = streamed ? pool + ((t - n_res_mt) & 1) * SLOT_BYTES : qreg + t * MT * ROWB;
            const int tok = t * MT + row;  // token index inside this CTA
            if (tok < n_valid) {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4*>(tile + swz<3>(row * ROWB + c * 16)) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int r32 = q4 * 32;  // this warp's 32 rows of the tile
                if (t * MT + r32 + 32 <= n_valid) {
                    tma_store_3d(&tm_o32, 0, t0 + t * MT + r32, u, tile + r32 * ROWB);
                } else {
                    for (int k = 0; k < 4; ++k)
                        if (t * MT + r32 + 8 * k < n_valid)
                            tma_store_3d(&tm_o8, 0, t0 + t * MT + r32 + 8 * k, u, tile + (r32 + 8 * k) * ROWB);
                }
                tma_store_commit();
                if (streamed) {
                    tma_store_wait_read_all();
                    mbar_arrive(&bars->sempty[(t - n_res_mt) & 1]);
                }
            }
            __syncwarp();
            if (t + 1 < n_mt) tc::wait_ld();
        }
        if (lane == 0) tma_store_wait_all();
        cluster_wait_acquire();
    }

    tc::fence_before();
    __syncthreads();
    if (warp == 1) tc::dealloc(tmem, TMEM_COLS);
}

}  // namespace lin5

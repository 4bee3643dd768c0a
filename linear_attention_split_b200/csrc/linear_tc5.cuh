// linear_tc5.cuh -- TTT-Linear full-batch step on the 5th-generation tensor cores (tcgen05),
// bf16 inputs, d = 64, one kernel per call.
//
// Operation ("ViT^3" blog, online-learning rewrite of attention, steps 1-3; TTT-Linear of the
// TTT abstract), per unit u = (batch b, head h) with Q, K, V in R^{N x 64}:
//     G = K^T K,  C = K^T V,   grad = G W0 - C,   W* = W0 - (eta/N) grad,   O = Q W*
// (grad/N is the full-batch gradient of (1/N) sum_i 1/2 ||k_i W - v_i||^2 at W0.)
//
// Work layout: one thread-block cluster of S CTAs per unit (S in {1, 2, 4, 8}), one CTA per
// SM.  The unit's tokens are cut into tiles of TT <= 128 rows (TT a multiple of 16, chosen so
// that every CTA gets the same number of tiles); CTA r takes tiles r, r + S, r + 2S, ...
// Warp 0 = TMA producer, warp 1 = tcgen05 MMA issuer (one thread), warps 2-9 = epilogue
// (warp w reads TMEM lane quarter w % 4, column half (w - 2) / 4).  The design keeps the
// shared-memory traffic per HBM byte low: each K/V byte is written once by TMA and read once
// or twice by the tensor cores.
//
//   1. Gram pass, per tile (V, K land in a ring slot by plain TMA, 128-byte swizzle):
//        A += [V | K]^T K    tcgen05, M = 128 (features of V, then of K), N = 64, K-dim = the
//                            TT token rows, both operands MN-major straight from the slot;
//                            TMEM rows 0-63 hold this CTA's part of C^T, rows 64-127 of G.
//      Once the ring is primed the remaining K/V tiles are requested into L2, so that HBM
//      sees the whole stream at once.  Q is requested only once the Gram pass is done: it is
//      not needed before the exchange below has finished, and it would slow K and V down.
//   2. Partial gradient, transposed (G is symmetric):  grad^T = W0^T G - C^T.
//      The epilogue writes this CTA's G as bf16 hi + lo (a K-major operand), the issuer
//      computes D = W0_hi^T [G_hi | G_lo] (N = 128) and adds W0_lo^T G_hi to its first half
//      (M = 128 MMAs whose rows >= 64 are not used), so that lane f holds D[f] and C^T[f] and
//      D[f][0:64] + D[f][64:128] - C^T[f] is row f of this CTA's grad^T, with W0 and G kept to
//      2^-17.
//   3. Exchange: CTA c owns W* columns [c 64/S, (c+1) 64/S).  Every epilogue thread of lane
//      quarters 0-1 sends its row half of D - C^T to the owner with st.async (completion
//      counted on the owner's mbarrier); the owner adds the S contributions in rank order
//      (deterministic, no atomics), forms W*^T rows = W0^T - (eta/N) grad^T in fp32 and sends
//      them as bf16 hi + lo to every CTA of the cluster, again with st.async.
//   4. Apply: Q tiles are loaded into the ring region, O = Q W*_hi + Q W*_lo (two N = 64
//      MMA chains accumulating into one 64-column buffer) in eight TMEM buffers (all of
//      TMEM: the Gram and W0^T G accumulators have been read by then); the Q tiles that fit
//      are awaited while the exchange is in flight.  The epilogue warps form two groups of
//      four (one warp per lane quarter) that take alternate tiles: write O as bf16 over the
//      consumed Q tile, one TMA store per tile (rows >= N are clipped by the hardware).  A CTA ends once its last store has read shared memory;
//      the writes drain to memory while the next grid starts.
// Every wait is bounded (common.cuh); after a wait has run out on the device, later waits give
// up at once and the kernel runs to its normal end (results are then invalid and the host is
// told through the device error word).  Launched with programmatic stream serialization: the
// kernel waits for the previous grid before its first global access.
#pragma once
#include "common.cuh"

namespace lin5 {

constexpr int D = 64;
constexpr int ROWB = 128;                      // bytes per token row (64 bf16)
constexpr int MT = 128;                        // rows reserved per tile (TT <= MT are used)
constexpr int TILE_BYTES = MT * ROWB;          // 16 KB
constexpr int SLOT_BYTES = 2 * TILE_BYTES;     // K, V
constexpr int MAX_SLOTS = 6;
constexpr int MAX_QT = 2 * MAX_SLOTS;          // Q tile buffers carved from the ring
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;   // producer, issuer, 8 epilogue warps
constexpr int EPI_THREADS = 32 * EPI_WARPS;
constexpr int OP_BYTES = D * ROWB;             // one 64 x 64 bf16 K-major operand, 8 KB
constexpr int RECV_BYTES = D * D * 4;          // S sources x (64/S) rows x 64 fp32 = 16 KB
constexpr int FIXED_BYTES = 4 * OP_BYTES + RECV_BYTES;  // W0 hi/lo, W* hi/lo, receive area
constexpr int TMEM_COLS = 512;
constexpr int COL_A = 0;                       // Gram accumulator [C^T ; G]
constexpr int COL_D = 64;                      // W0^T [G_hi | G_lo] (rows 0-63), 128 columns
constexpr int COL_O = 0;                       // eight O buffers of 64 columns (apply)
constexpr int OBUFS = 8;
static_assert((OBUFS & (OBUFS - 1)) == 0, "OBUFS is a power of two");
constexpr uint32_t IDESC_GRAM = tc::idesc_bf16(128, 64, 1, 1);   // A MN-major, B MN-major
constexpr uint32_t IDESC_WG = tc::idesc_bf16(128, 64, 0, 0);     // A K-major, B K-major
constexpr uint32_t IDESC_WG2 = tc::idesc_bf16(128, 128, 0, 0);   // A K-major, B K-major, N = 128
constexpr uint32_t IDESC_APPLY = tc::idesc_bf16(128, 64, 0, 0);  // A K-major (Q), B K-major (W*^T)

struct Params {
    const float* w0;    // [H][64][64]; with dh < 64: [64 / dh][dh][dh] (one per head of the unit)
    float* w_star;      // [U][64][64] or nullptr
    int H, N;
    int dh;             // 64, or the width of the heads that sit side by side in a unit's 64 features
    int TT;             // token rows per tile (multiple of 16, <= 128)
    int n_tiles;        // tiles per unit, ceil(N / TT)
    int slots;          // ring slots (32 KB each)
    int nq;             // Q tile buffers (16 KB each, carved from the ring)
    float eta_over_n;
};

struct Bars {
    uint64_t full[MAX_SLOTS], empty[MAX_SLOTS], qfull[MAX_QT], qempty[MAX_QT], tfull[OBUFS], tempty[OBUFS],
        w0ready, gram_done, gready, dfull, rfull, wfull, wlocal;
    uint32_t tmem_base;
};

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ void group_sync(int g) { asm volatile("bar.sync %0, 128;" ::"r"(2 + g) : "memory"); }

// Byte offset of element (row n, column k) in a 64 x 64 bf16 K-major operand, 128-byte swizzle.
__device__ __forceinline__ uint32_t op_off(int n, int k) {
    return (uint32_t)(n >> 3) * 1024u + swz<3>((uint32_t)(n & 7) * ROWB + (uint32_t)k * 2u);
}
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

__global__ void __launch_bounds__(THREADS, 1)
    linear_tc5_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
                      const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_align<1024>(smem_raw);
    uint8_t* pool = base;                                   // ring slots, then Q tiles
    uint8_t* fixed = base + p.slots * SLOT_BYTES;
    uint8_t* w0op = fixed;                                  // [W0_hi^T ; W0_lo^T] (K-major, 128 rows)
    uint8_t* wsop = fixed + 2 * OP_BYTES;                   // G hi, lo; later [W*_hi^T ; W*_lo^T]
    float* recv = reinterpret_cast<float*>(fixed + 4 * OP_BYTES);
    Bars* bars = reinterpret_cast<Bars*>(fixed + FIXED_BYTES);

    const uint32_t S = gridDim.x;  // one cluster spans the x dimension
    const uint32_t rank = cluster_ctarank();
    const int u = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_t = (int)rank < p.n_tiles ? (p.n_tiles - (int)rank + (int)S - 1) / (int)S : 0;  // tiles here
    const int rp = D / (int)S;             // W* columns owned by each CTA
    const int r0 = (int)rank * rp;
    const int NS = p.slots, NQ = p.nq, TT = p.TT;

    // ---- set-up ------------------------------------------------------------------------
    // The first ring's worth of K and V tiles into L2 while the previous grid on the stream may
    // still run: a prefetch only warms the (coherent) L2; the loads themselves wait for that
    // grid below.  (Prefetching every K, V and Q tile here was slower: 14.9 against 13.8 µs a
    // call; the burst queues ahead of the tiles needed first.)
    if (threadIdx.x == 0)
        for (int i = 0; i < min(NS, n_t); ++i) {
            tma_prefetch_l2_3d(&tm_k, 0, ((int)rank + i * (int)S) * TT, u);
            tma_prefetch_l2_3d(&tm_v, 0, ((int)rank + i * (int)S) * TT, u);
        }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int j = 0; j < NQ; ++j) {
            mbar_init(&bars->qfull[j], 1);
            mbar_init(&bars->qempty[j], 1);
        }
        for (int b = 0; b < OBUFS; ++b) {
            mbar_init(&bars->tfull[b], 1);
            mbar_init(&bars->tempty[b], EPI_WARPS / 2);
        }
        mbar_init(&bars->w0ready, EPI_WARPS);
        mbar_init(&bars->gram_done, 1);
        mbar_init(&bars->gready, EPI_WARPS / 2);
        mbar_init(&bars->dfull, 1);
        mbar_init(&bars->rfull, 1);
        mbar_init(&bars->wfull, 1);
        mbar_init(&bars->wlocal, EPI_WARPS);
        mbar_fence_init();
        // gradient rows and W* rows from the S - 1 other CTAs (st.async bytes)
        mbar_expect_tx(&bars->rfull, (S - 1) * (uint32_t)rp * D * 4u);
        mbar_expect_tx(&bars->wfull, (S - 1) * (uint32_t)rp * 2u * ROWB);
    }
    if (warp == 1) tc::alloc(&bars->tmem_base, TMEM_COLS);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    cluster_arrive_release();  // this CTA's barriers exist: peers may signal them
    griddep_wait();            // the previous grid on the stream has completed
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ================================ producer ======================================
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_o);
            const bool skip_last = (*reinterpret_cast<volatile unsigned int*>(&g_ttt_fault) & TTT_FAULT_SKIP_LOAD) != 0;
            for (int i = 0; i < n_t; ++i) {
                const int slot = i % NS, use = i / NS;
                if (use > 0) mbar_wait(&bars->empty[slot], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                uint8_t* dst = pool + slot * SLOT_BYTES;
                const int row = ((int)rank + i * (int)S) * TT;
                if (!(skip_last && i == n_t - 1)) {  // test hook: the last tile's data never arrives
                    mbar_expect_tx(&bars->full[slot], 2 * TT * ROWB);
                    tma_load_3d(dst, &tm_v, 0, row, u, &bars->full[slot]);
                    tma_load_3d(dst + TILE_BYTES, &tm_k, 0, row, u, &bars->full[slot]);
                }
                if (i == NS - 1)  // the rest of K and V into L2 now
                    for (int j = NS; j < n_t; ++j) {
                        tma_prefetch_l2_3d(&tm_k, 0, ((int)rank + j * (int)S) * TT, u);
                        tma_prefetch_l2_3d(&tm_v, 0, ((int)rank + j * (int)S) * TT, u);
                    }
            }
            // the ring is free once every Gram MMA has completed
            if (n_t > 0) mbar_wait(&bars->gram_done, 0, TTT_DEVERR_TIMEOUT_TMA);
            griddep_launch();
            for (int t = 0; t < n_t; ++t) {
                const int qs = t % NQ, use = t / NQ;
                if (use > 0) mbar_wait(&bars->qempty[qs], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                mbar_expect_tx(&bars->qfull[qs], TT * ROWB);
                tma_load_3d(pool + qs * TILE_BYTES, &tm_q, 0, ((int)rank + t * (int)S) * TT, u, &bars->qfull[qs]);
            }
        }
        __syncwarp();
        cluster_wait_acquire();
        cluster_arrive_release();
    } else if (warp == 1) {
        // ================================ MMA issuer =====================================
        if (lane == 0) {
            // ---- Gram pass: A += [V | K]^T K per tile -------------------------------------
            for (int i = 0; i < n_t; ++i) {
                const int slot = i % NS;
                mbar_wait(&bars->full[slot], (i / NS) & 1, TTT_DEVERR_TIMEOUT_TMA);
                tc::fence_after();
                const uint32_t vb = smem_u32(pool + slot * SLOT_BYTES);
                // A = [V | K]^T: MN-major, atoms V tile / K tile (LBO), 8-token groups (SBO); a
                // k-step of 16 tokens moves both start addresses by 2 KB (start field += 128)
                const uint64_t da = tc::smem_desc(vb, TILE_BYTES, 1024, 2);
                const uint64_t db = tc::smem_desc(vb + TILE_BYTES, TILE_BYTES, 1024, 2);
                for (int ks = 0; ks < TT / 16; ++ks)
                    tc::mma_bf16(tmem + COL_A, da + (uint64_t)(ks * 128), db + (uint64_t)(ks * 128), IDESC_GRAM,
                                 (i > 0 || ks > 0) ? 1 : 0);
                tc::commit(&bars->empty[slot]);
            }
            if (n_t > 0) {
                tc::commit(&bars->gram_done);
                // ---- D = W0_hi^T [G_hi | G_lo], then D[:, 0:64] += W0_lo^T G_hi ----------------
                // A rows 0-63 are W0_hi^T (or W0_lo^T); rows 64-127 read whatever operand follows
                // in shared memory and land in D rows that are never read.
                mbar_wait(&bars->w0ready, 0, TTT_DEVERR_TIMEOUT_PEER);
                mbar_wait(&bars->gready, 0, TTT_DEVERR_TIMEOUT_PEER);
                tc::fence_after();
                // K-major operands: a k-step of 16 elements moves the start address by 32 B (+2)
                const uint64_t dw = tc::smem_desc(smem_u32(w0op), 16, 1024, 2);
                const uint64_t dwl = tc::smem_desc(smem_u32(w0op) + OP_BYTES, 16, 1024, 2);
                const uint64_t dg = tc::smem_desc(smem_u32(wsop), 16, 1024, 2);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tmem + COL_D, dw + 2 * ks, dg + 2 * ks, IDESC_WG2, ks > 0 ? 1 : 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) tc::mma_bf16(tmem + COL_D, dwl + 2 * ks, dg + 2 * ks, IDESC_WG, 1);
                tc::commit(&bars->dfull);
            }

            // ---- apply: O = Q W*_hi + Q W*_lo per tile, accumulated in one 64-column buffer ---
            const int q_first = n_t < NQ ? n_t : NQ;  // tiles whose Q is loaded up front
            for (int t = 0; t < q_first; ++t) mbar_wait(&bars->qfull[t], 0, TTT_DEVERR_TIMEOUT_TMA);
            mbar_wait_cluster(&bars->wfull, 0, TTT_DEVERR_TIMEOUT_PEER);   // the peers' W* rows
            mbar_wait(&bars->wlocal, 0, TTT_DEVERR_TIMEOUT_PEER);          // and this CTA's own
            fence_proxy_async_smem();  // W* rows were written by generic stores (local and st.async)
            tc::fence_after();
            const uint64_t dwh = tc::smem_desc(smem_u32(wsop), 16, 1024, 2);
            const uint64_t dwo = tc::smem_desc(smem_u32(wsop) + OP_BYTES, 16, 1024, 2);
            auto apply_tile = [&](int t, int qs) {
                const int b = t & (OBUFS - 1);
                const uint64_t dq = tc::smem_desc(smem_u32(pool + qs * TILE_BYTES), 16, 1024, 2);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tmem + COL_O + b * 64, dq + 2 * ks, dwh + 2 * ks, IDESC_APPLY, ks > 0 ? 1 : 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tmem + COL_O + b * 64, dq + 2 * ks, dwo + 2 * ks, IDESC_APPLY, 1);
                tc::commit(&bars->tfull[b]);
            };
            // Tiles whose Q tile has landed and whose TMEM buffer has never been used are issued
            // by a loop with no waits in it (a bounded wait in the loop body, even one not taken,
            // costs a few hundred cycles per tile between the MMA batches).
            const int t_free = q_first < OBUFS ? q_first : OBUFS;
            int t = 0;
            for (; t < t_free; ++t) apply_tile(t, t);
            for (; t < n_t; ++t) {
                const int qs = t % NQ;
                if (t >= OBUFS) mbar_wait(&bars->tempty[t & (OBUFS - 1)], (t / OBUFS - 1) & 1, TTT_DEVERR_TIMEOUT_PEER);
                if (t >= q_first) mbar_wait(&bars->qfull[qs], (t / NQ) & 1, TTT_DEVERR_TIMEOUT_TMA);
                tc::fence_after();
                apply_tile(t, qs);
            }
        }
        __syncwarp();
        cluster_wait_acquire();
        cluster_arrive_release();
    } else {
        // ================================ epilogue =======================================
        const int q4 = warp & 3;               // TMEM lane quarter this warp may access
        const int h = (warp - 2) >> 2;         // column half
        const int row = q4 * 32 + lane;        // tile row / accumulator lane of this thread
        const int et = threadIdx.x - 64;       // 0..255
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
        const float* W0 = p.dh == D ? p.w0 + (size_t)(u % p.H) * D * D : p.w0;
        // element (m, f) of this unit's 64 x 64 W0.  With heads of dh < 64 side by side in the
        // unit's features, W0 is block-diagonal (head h's block is w0[h]); the kernel then
        // zeroes W*'s off-diagonal blocks, and each head's block of W* and of O is exactly its
        // own full-batch step (G W0 and C are taken block by block).
        auto w0at = [&](int m, int f) -> float {
            if (p.dh == D) return __ldg(&W0[m * D + f]);
            return (m / p.dh == f / p.dh) ? __ldg(&W0[((m / p.dh) * p.dh + m % p.dh) * p.dh + f % p.dh]) : 0.f;
        };

        // ---- W0^T as bf16 hi + lo, K-major (row = output feature f, k = input feature m) --
        {
            const int f = et & 63, mg = et >> 6;  // 16 input features per thread
            uint32_t hi[8], lo[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int m = mg * 16 + 2 * k;
                split_bf16(w0at(m, f), w0at(m + 1, f), hi[k], lo[k]);
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const uint32_t off = op_off(f, mg * 16 + 8 * c);
                *reinterpret_cast<uint4*>(w0op + off) = make_uint4(hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
                *reinterpret_cast<uint4*>(w0op + OP_BYTES + off) =
                    make_uint4(lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->w0ready);
        }
        // W0[4 cg + i][r0 + fl] for the W* entries this thread forms (up to four items)
        const int items = rp * 16;
        float w0o[4][4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int it = et + k * EPI_THREADS;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                w0o[k][i] = it < items ? w0at(4 * (it & 15) + i, r0 + (it >> 4)) : 0.f;
        }

        // ---- G rows of this CTA as bf16 hi + lo (a K-major operand; G is symmetric) -------
        if (n_t > 0) {
            mbar_wait(&bars->gram_done, 0, TTT_DEVERR_TIMEOUT_TMA);
            tc::fence_after();
            if (row >= D) {  // lane 64 + i holds G row i
                float g[32];
                tc::ld16(lane_base + COL_A + h * 32, &g[0]);
                tc::ld16(lane_base + COL_A + h * 32 + 16, &g[16]);
                tc::wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) split_bf16(g[8 * c + 2 * k], g[8 * c + 2 * k + 1], hi[k], lo[k]);
                    const uint32_t off = op_off(row - D, h * 32 + 8 * c);
                    *reinterpret_cast<uint4*>(wsop + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4*>(wsop + OP_BYTES + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                }
                fence_proxy_async_smem();  // read next by the tensor cores
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->gready);
            }
        }

        // ---- exchange: send this thread's row half of grad^T to the column owner -----------
        cluster_wait_acquire();  // every CTA of the cluster has initialised its barriers
        if (row < D) {
            float x[32];
            if (n_t > 0) {
                float c[32], y[32];
                mbar_wait(&bars->dfull, 0, TTT_DEVERR_TIMEOUT_TMA);
                tc::fence_after();
                tc::ld16(lane_base + COL_D + h * 32, &x[0]);
                tc::ld16(lane_base + COL_D + h * 32 + 16, &x[16]);
                tc::ld16(lane_base + COL_D + 64 + h * 32, &y[0]);
                tc::ld16(lane_base + COL_D + 64 + h * 32 + 16, &y[16]);
                tc::ld16(lane_base + COL_A + h * 32, &c[0]);
                tc::ld16(lane_base + COL_A + h * 32 + 16, &c[16]);
                tc::wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k) x[k] = (x[k] + y[k]) - c[k];
            } else {
#pragma unroll
                for (int k = 0; k < 32; ++k) x[k] = 0.f;
            }
            const uint32_t owner = (uint32_t)(row / rp);  // row = W* column f
            float* dst = recv + ((size_t)(rank * rp + row % rp) * D + h * 32);
            if (owner == rank) {
#pragma unroll
                for (int k = 0; k < 32; k += 4)
                    *reinterpret_cast<float4*>(dst + k) = make_float4(x[k], x[k + 1], x[k + 2], x[k + 3]);
            } else {
                const uint32_t ra = mapa_u32(smem_u32(dst), owner);
                const uint32_t rb = mapa_u32(smem_u32(&bars->rfull), owner);
#pragma unroll
                for (int k = 0; k < 32; k += 4)
                    st_async_v4(ra + k * 4, rb, __float_as_uint(x[k]), __float_as_uint(x[k + 1]),
                                __float_as_uint(x[k + 2]), __float_as_uint(x[k + 3]));
            }
        }
        tc::fence_before();
        epi_sync();  // this CTA's own contributions are in the receive area; D and G are read
        mbar_wait_cluster(&bars->rfull, 0, TTT_DEVERR_TIMEOUT_PEER);

        // ---- W*^T rows r0.. : sum the S contributions in rank order, then send ------------
        {
            const uint32_t wfull_peer_base = smem_u32(&bars->wfull);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int it = et + k * EPI_THREADS;
                if (it < items) {
                    const int fl = it >> 4, cg = it & 15;
                    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (uint32_t src = 0; src < S; ++src) {
                        const float4 v = *reinterpret_cast<const float4*>(recv + (size_t)(src * rp + fl) * D + 4 * cg);
                        s.x += v.x;
                        s.y += v.y;
                        s.z += v.z;
                        s.w += v.w;
                    }
                    const int f = r0 + fl;
                    float w[4] = {w0o[k][0] - p.eta_over_n * s.x, w0o[k][1] - p.eta_over_n * s.y,
                                  w0o[k][2] - p.eta_over_n * s.z, w0o[k][3] - p.eta_over_n * s.w};
                    if (p.dh < D)  // heads side by side: W* keeps only its diagonal blocks
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            if ((4 * cg + i) / p.dh != f / p.dh) w[i] = 0.f;
                    if (p.w_star) {
                        float* ws = p.w_star + (size_t)u * D * D;
#pragma unroll
                        for (int i = 0; i < 4; ++i) ws[(4 * cg + i) * D + f] = w[i];
                    }
                    uint32_t hi0, lo0, hi1, lo1;
                    split_bf16(w[0], w[1], hi0, lo0);
                    split_bf16(w[2], w[3], hi1, lo1);
                    const uint32_t off = op_off(f, 4 * cg);
                    *reinterpret_cast<uint2*>(wsop + off) = make_uint2(hi0, hi1);
                    *reinterpret_cast<uint2*>(wsop + OP_BYTES + off) = make_uint2(lo0, lo1);
                    for (uint32_t kk = 1; kk < S; ++kk) {
                        const uint32_t peer = (rank + kk) % S;
                        const uint32_t rb = mapa_u32(wfull_peer_base, peer);
                        st_async_v2(mapa_u32(smem_u32(wsop + off), peer), rb, hi0, hi1);
                        st_async_v2(mapa_u32(smem_u32(wsop + OP_BYTES + off), peer), rb, lo0, lo1);
                    }
                }
            }
            fence_proxy_async_smem();  // read next by the tensor cores
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->wlocal);
        }
        cluster_arrive_release();  // every remote store of this thread has been issued

        // ---- O tiles: group h (one warp per lane quarter) takes tiles t = h, h + 2, ...:
        //      TMEM -> bf16 over the Q tile -> one TMA store per tile ------------------------------
        const bool storer = (q4 == 0 && lane == 0);
        for (int t = h; t < n_t; t += 2) {
            const int b = t % OBUFS, qs = t % NQ;
            uint8_t* tile = pool + qs * TILE_BYTES;  // the MMA that read this Q tile has completed
            mbar_wait(&bars->tfull[b], (t / OBUFS) & 1, TTT_DEVERR_TIMEOUT_PEER);
            tc::fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float o[32];
                const uint32_t ob = lane_base + COL_O + b * 64 + half * 32;
                tc::ld16(ob, &o[0]);
                tc::ld16(ob + 16, &o[16]);
                tc::wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    *reinterpret_cast<uint4*>(tile + swz<3>((uint32_t)row * ROWB + half * 64 + c * 16)) =
                        make_uint4(pack_bf16(o[8 * c], o[8 * c + 1]), pack_bf16(o[8 * c + 2], o[8 * c + 3]),
                                   pack_bf16(o[8 * c + 4], o[8 * c + 5]), pack_bf16(o[8 * c + 6], o[8 * c + 7]));
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->tempty[b]);
            fence_proxy_async_smem();
            group_sync(h);  // the group's 128 rows are written
            if (storer) {
                const int grow = ((int)rank + t * (int)S) * TT;  // rows >= N are clipped
                tma_store_3d(&tm_o, 0, grow, u, tile);
                tma_store_commit();
                if (t + NQ < n_t) {  // the buffer is reloaded with a later Q tile
                    tma_store_wait_read_all();
                    mbar_arrive(&bars->qempty[qs]);
                }
            }
        }
        if (storer) tma_store_wait_read_all();  // the writes drain to memory after the CTA ends
        cluster_wait_acquire();
    }

    tc::fence_before();
    __syncthreads();
    if (warp == 1) tc::dealloc(tmem, TMEM_COLS);
}

}  // namespace lin5

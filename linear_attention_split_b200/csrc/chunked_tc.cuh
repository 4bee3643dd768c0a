// chunked_tc.cuh -- chunked bidirectional TTT-Linear scan, bf16, d = 64, chunk = 64.
//
// Operation (Vision-TTT gist, "Technische samenvatting": W_t = W_{t-1} - eta grad l(W_{t-1}; x_t)
// applied per mini-batch, tokens scanned forward and backward), per unit u = (b, h) and
// direction, over chunks c of b = 64 consecutive tokens:
//     R   = K_c W - V_c
//     W  <- W - (eta/b) K_c^T R
//     O_c = Q_c W                      (W after the chunk's update)
// raster order from W0 and reverse raster order from W0; the layer output is the sum.
// The output columns of W evolve independently (column j of the update only involves column
// j of W, V and O), so a CTA owns 16 of the 64 columns and both directions of one unit:
// warps 0-3 scan forward (chunk s at step s), warps 4-7 backward (chunk nc-1-s at step s),
// each warp owning 16 tokens of R and O and 16 rows (features) of the W update.  The MMAs
// are bf16 mma.sync m16n8k16 with fp32 accumulation; W's master copy stays fp32 in
// registers, and its bf16 copy (the B operand of K_c W and Q_c W) goes through shared memory
// once per step.  A producer warp streams K_c, Q_c (128B-swizzled) and the CTA's 16 columns
// of V_c through a TMA ring.  The two directions meet in the middle: at step s < nc/2 each
// direction parks its fp32 partial output for its chunk in the workspace; at step s >= nc/2
// it adds the partner's parked partial, rounds once to bf16 and stores O (deterministic).
#pragma once
#include "common.cuh"

namespace chk {

constexpr int D = 64;
constexpr int CB = 64;                  // chunk size (tokens)
constexpr int NCOL = 16;                // columns of W per CTA
constexpr int GROUPS = D / NCOL;        // 4 column groups
constexpr int ROWB = 128;               // bytes per token row of K / Q
constexpr int TILE = CB * ROWB;         // 8 KB
constexpr int VT = CB * NCOL * 2;       // V columns tile: 2 KB
constexpr int STAGE = 2 * TILE + VT;    // one direction's data for one step
constexpr int STAGES = 3;
constexpr int WLD = 24;                 // bf16 row pitch (48 B) of the W and R tiles
constexpr int WT = D * WLD * 2;         // one 64 x 16 bf16 tile (padded)
constexpr int THREADS = 9 * 32;         // 8 compute warps + producer

struct Params {
    const float* w0;    // [H][64][64]
    float* park;        // workspace [U][N][64] fp32 (partial outputs)
    __nv_bfloat16* out; // [U][N][64]
    int H, N, nc;       // nc = N / 64
    float eta_over_b;
};

struct Bars {
    uint64_t full[2][STAGES], empty[2][STAGES];
};

__device__ __forceinline__ void group_sync(int dir) {
    if (dir == 0)
        asm volatile("bar.sync 1, 128;" ::: "memory");
    else
        asm volatile("bar.sync 2, 128;" ::: "memory");
}

__global__ void __launch_bounds__(THREADS, 1)
    chunked_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_v16, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;                                    // [dir][stage] {K, Q, V16}
    uint8_t* wtile = ring + 2 * STAGES * STAGE;              // [dir] W bf16 [64 feats][16 cols]
    uint8_t* rtile = wtile + 2 * WT;                         // [dir] R bf16 [64 tokens][16 cols]
    Bars* bars = reinterpret_cast<Bars*>(rtile + 2 * WT);

    const int grp = blockIdx.x, u = blockIdx.y;
    const int col0 = grp * NCOL;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nc = p.nc;
    auto stage_ptr = [&](int dir, int s) { return ring + (dir * STAGES + s) * STAGE; };
    auto chunk_of = [&](int dir, int step) { return dir == 0 ? step : nc - 1 - step; };

    if (threadIdx.x == 0) {
        for (int d = 0; d < 2; ++d)
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(&bars->full[d][s], 1);
                mbar_init(&bars->empty[d][s], 4);
            }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == 8) {
        // ================================ producer ======================================
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_v16);
            for (int step = 0; step < nc; ++step)
                for (int dir = 0; dir < 2; ++dir) {
                    const int s = step % STAGES, use = step / STAGES;
                    if (use > 0) mbar_wait(&bars->empty[dir][s], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                    const int t0 = chunk_of(dir, step) * CB;
                    uint8_t* dst = stage_ptr(dir, s);
                    mbar_expect_tx(&bars->full[dir][s], STAGE);
                    tma_load_3d(dst, &tm_k, 0, t0, u, &bars->full[dir][s]);
                    tma_load_3d(dst + TILE, &tm_q, 0, t0, u, &bars->full[dir][s]);
                    tma_load_3d(dst + 2 * TILE, &tm_v16, col0, t0, u, &bars->full[dir][s]);
                }
        }
        return;
    }

    // =================================== compute warps ===================================
    const int dir = warp >> 2;          // 0 forward, 1 backward
    const int wq = warp & 3;            // 16-row block of this warp
    uint8_t* wt = wtile + dir * WT;
    uint8_t* rt = rtile + dir * WT;
    const uint32_t wt_a = smem_u32(wt), rt_a = smem_u32(rt);

    // master W rows [16 wq, 16 wq + 16) x my 16 columns, C-fragment layout of m16n8
    float wm[2][4];
    {
        const float* W0 = p.w0 + (size_t)(u % p.H) * D * D;
        const int r = 16 * wq + (lane >> 2);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int cj = col0 + nt * 8 + 2 * (lane & 3);
            wm[nt][0] = W0[r * D + cj];
            wm[nt][1] = W0[r * D + cj + 1];
            wm[nt][2] = W0[(r + 8) * D + cj];
            wm[nt][3] = W0[(r + 8) * D + cj + 1];
        }
    }
    // publish W rows as bf16 [feature][col] (pitch 48 B)
    auto publish = [&](uint8_t* tile, const float (*v)[4], int rbase) {
        const int r = rbase + (lane >> 2);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int cj = nt * 8 + 2 * (lane & 3);
            *reinterpret_cast<uint32_t*>(tile + (r * WLD + cj) * 2) = pack_bf16(v[nt][0], v[nt][1]);
            *reinterpret_cast<uint32_t*>(tile + ((r + 8) * WLD + cj) * 2) = pack_bf16(v[nt][2], v[nt][3]);
        }
    };
    // B fragments (k = rows of a [64][16] bf16 tile, n = 16 columns) for four k-steps
    auto load_b = [&](uint32_t base, uint32_t (*b)[2][2]) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const int row = ks * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
            const int colb = (lane >> 4) * 16;  // bytes: columns 0-7 or 8-15
            ldsm_x4_t(base + row * WLD * 2 + colb, b[ks][0][0], b[ks][0][1], b[ks][1][0], b[ks][1][1]);
        }
    };
    publish(wt, wm, 16 * wq);
    group_sync(dir);
    uint32_t bw[4][2][2];  // B fragments of the current W (bf16)
    load_b(wt_a, bw);
    // The partner direction's parked partials, read PF steps before they are added (all of
    // them are written before the barrier at step nc/2), so that the read's latency stays
    // off the step-to-step chain.
    constexpr int PF = 2;
    float2 pre0[4], pre1[4];  // steps of even / odd parity
    const int rr = 16 * wq + (lane >> 2);
    auto adds_at = [&](int st) { return st >= nc / 2 && !(2 * st == nc - 1 && dir == 0); };
    auto fetch = [&](int st) {  // parked partial of the chunk this direction visits at step st
        const size_t t0c = (size_t)u * p.N + (size_t)chunk_of(dir, st) * CB;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float2 x =
                    *reinterpret_cast<const float2*>(&p.park[(t0c + rr + 8 * h) * D + col0 + nt * 8 + 2 * (lane & 3)]);
                if (st & 1)
                    pre1[2 * nt + h] = x;
                else
                    pre0[2 * nt + h] = x;
            }
    };

    for (int step = 0; step < nc; ++step) {
        const int s = step % STAGES;
        mbar_wait(&bars->full[dir][s], (step / STAGES) & 1, TTT_DEVERR_TIMEOUT_TMA);
        const int c = chunk_of(dir, step);
        uint8_t* st = stage_ptr(dir, s);
        const uint32_t kb = smem_u32(st), qb = kb + TILE;
        const uint8_t* vt = st + 2 * TILE;

        // ---- R = K_c W - V_c for tokens [16 wq, +16) -------------------------------------
        float acc[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t a[4];
            const int row = 16 * wq + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int chunk = 2 * ks + (lane >> 4);
            ldsm_x4(kb + swz<3>(row * ROWB + chunk * 16), a[0], a[1], a[2], a[3]);
            mma_bf16(acc[0], a, bw[ks][0][0], bw[ks][0][1]);
            mma_bf16(acc[1], a, bw[ks][1][0], bw[ks][1][1]);
        }
        {
            const int r = 16 * wq + (lane >> 2);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int cj = nt * 8 + 2 * (lane & 3);
                const float2 v0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vt + (r * NCOL + cj) * 2));
                const float2 v1 =
                    __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vt + ((r + 8) * NCOL + cj) * 2));
                acc[nt][0] -= v0.x;
                acc[nt][1] -= v0.y;
                acc[nt][2] -= v1.x;
                acc[nt][3] -= v1.y;
            }
        }
        publish(rt, acc, 16 * wq);
        group_sync(dir);  // R complete; every warp has read W for this step
        // ---- W rows [16 wq, +16) -= (eta/b) K_c^T R ---------------------------------------
        uint32_t br[4][2][2];
        load_b(rt_a, br);
        float dw[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {  // k = tokens 16 ks..
            uint32_t a[4];
            const int row = ks * 16 + (lane >> 4) * 8 + (lane & 7);
            const int chunk = wq * 2 + ((lane >> 3) & 1);
            ldsm_x4_t(kb + swz<3>(row * ROWB + chunk * 16), a[0], a[1], a[2], a[3]);
            mma_bf16(dw[0], a, br[ks][0][0], br[ks][0][1]);
            mma_bf16(dw[1], a, br[ks][1][0], br[ks][1][1]);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) wm[nt][e] -= p.eta_over_b * dw[nt][e];
        publish(wt, wm, 16 * wq);  // every warp read the old W before the barrier above
        group_sync(dir);  // new W tile complete
        // ---- O_c = Q_c W for tokens [16 wq, +16) ------------------------------------------
        load_b(wt_a, bw);
        float o[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t a[4];
            const int row = 16 * wq + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int chunk = 2 * ks + (lane >> 4);
            ldsm_x4(qb + swz<3>(row * ROWB + chunk * 16), a[0], a[1], a[2], a[3]);
            mma_bf16(o[0], a, bw[ks][0][0], bw[ks][0][1]);
            mma_bf16(o[1], a, bw[ks][1][0], bw[ks][1][1]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->empty[dir][s]);  // K, Q, V of this step consumed
        // ---- combine the two directions ---------------------------------------------------
        // chunk c is visited by the forward warps at step c and by the backward warps at step
        // nc-1-c: the first visit parks its partial, the second adds it.  For odd nc both
        // visit the middle chunk at the same step: the forward warps park, then the backward
        // warps add.  One barrier over the compute warps at step nc/2 orders all parks
        // before all additions.
        const int r = 16 * wq + (lane >> 2);
        const size_t tok0 = (size_t)u * p.N + (size_t)c * CB;
        const bool first = 2 * step < nc - 1;
        const bool middle = 2 * step == nc - 1;
        auto visit = [&](bool park) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int cj = col0 + nt * 8 + 2 * (lane & 3);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const size_t idx = (tok0 + r + 8 * h) * D + cj;
                    const float2 val = make_float2(o[nt][2 * h], o[nt][2 * h + 1]);
                    if (park) {
                        *reinterpret_cast<float2*>(&p.park[idx]) = val;
                    } else {
                        const float2 other = (step & 1) ? pre1[2 * nt + h] : pre0[2 * nt + h];
                        *reinterpret_cast<uint32_t*>(&p.out[idx]) = pack_bf16(val.x + other.x, val.y + other.y);
                    }
                }
            }
        };
        if (first || (middle && dir == 0)) visit(true);
        if (step == nc / 2) {
            asm volatile("bar.sync 3, 256;" ::: "memory");  // every park is written
#pragma unroll
            for (int k = 0; k < PF; ++k)
                if (step + k < nc && adds_at(step + k)) fetch(step + k);
        }
        if (!first && !(middle && dir == 0)) visit(false);
        if (step >= nc / 2 && step + PF < nc && adds_at(step + PF)) fetch(step + PF);  // slot of this step
    }
}

}  // namespace chk

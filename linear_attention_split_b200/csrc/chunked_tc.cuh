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
// j of W, V and O), so a CTA owns 16 of the 64 columns and both directions of one unit.
//
// One recurrence warp per direction (warp 0 forward: chunk s at step s; warp 1 backward:
// chunk nc-1-s at step s) keeps the whole 64 x 16 slice of W in registers, as its transpose:
// the fp32 master copy of W^T in the m16n8 accumulator layout of mma.sync m16n8k16, and its
// bf16 copy as A fragments.  A step computes R_i^T = W^T K_i^T - V_i^T for the chunk's four
// 16-token tiles (32 MMAs), then dW^T = sum_i R_i^T K_i (32 MMAs).  In this orientation each
// accumulator, packed to bf16 pairs, already is the next product's operand (R_i^T's for dW^T,
// W^T's for the next step's R^T and for Q W); K_i, K_i^T and V_i^T come from the TMA tiles by
// plain and transposing ldmatrix.  Nothing of the recurrence goes through shared memory, and
// no other warp takes part in it.  The step's K, Q and the CTA's 16 V
// columns arrive through a TMA ring filled by a producer warp (warp 4).  Each step the
// recurrence warp hands its fp32 copy of W (4 KB) to the two output warps of its direction
// (warps 2, 3 forward, 6, 7 backward; each takes two of the chunk's four 16-token tiles; a
// warp runs on sub-partition warp % 4, so the recurrence warps 0 and 1 share theirs with
// nothing but the mostly idle producer, and warp 5 has no work)
// through a small ring (wready / wfree); an output warp splits W into bf16 hi + lo B
// fragments and computes O = Q W_hi + Q W_lo for its 32 tokens (W kept to 2^-17 in the
// output) and the combine of the two directions, which meet in the middle: at step s < nc/2
// each direction parks its fp32 partial output for its chunk in the workspace; at step
// s >= nc/2 it adds the partner's parked partial, rounds once to bf16 and stores O
// (deterministic).  A unidirectional scan (raster or reverse raster alone: the original,
// one-way TTT scan that the Vision-TTT gist's bidirectional scan extends) runs one recurrence
// warp and its two output warps, which round each chunk's O = Q_c W once and store it, with
// nothing parked.
// Training mode (mini-batch / multi-epoch inner training, the design-study options of the
// ViT^3 blog) runs the raster recurrence over `steps` = epochs x nc chunks with no output warp
// and no Q, and leaves W_final (fp32) in global memory for the apply pass.
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
constexpr int WBUF = 4;                 // depth of the W hand-over ring
constexpr int WFR = 32 * 32 * 4;        // one W slice (fp32 master copy): 32 registers x 32 lanes
constexpr int THREADS = 8 * 32;         // 2 recurrence warps, 2 x 2 output warps, producer, one idle
constexpr int OUT_TILES = 2;            // 16-token tiles of a chunk per output warp
constexpr int PF = 2;                   // steps ahead that the partner's partials are copied
constexpr int PKB = CB * NCOL * 4;       // one chunk's partials for the CTA's columns (4 KB)
constexpr int PKH = PKB / 2;            // the half of them that one output warp adds

struct Params {
    const float* w0;    // [H][64][64]
    float* park;        // workspace [U][N][64] fp32 (partial outputs; both directions only)
    __nv_bfloat16* out; // [U][N][64]
    int H, N, nc;       // nc = N / 64
    int both;           // 1: both directions, summed; 0: direction `dir` alone
    int dir;            // the direction of a one-way scan: 0 raster, 1 reverse raster
    int steps;          // recurrence steps: nc, or epochs x nc in training mode
    float* wfin;        // training mode: W_final [U][64][64] fp32 (else nullptr)
    float* wout;        // training mode: optional copy of W_final for the caller (or nullptr)
    float eta_over_b;
};

struct Bars {
    uint64_t full[2][STAGES], empty[2][STAGES], wready[2][WBUF], wfree[2][WBUF], pfull[2][2][PF + 1];
};

__global__ void __launch_bounds__(THREADS, 1)
    chunked_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_v16, const __grid_constant__ CUtensorMap tm_park,
                   const Params p) {
    extern __shared__ uint8_t smem_raw[];
    // Rounded through an integer on purpose (the other kernels use smem_align): measured on
    // B200, the 80x80 bidirectional scan takes 94.4 us this way against 96.1 us with
    // smem_align (the one-way scan 79.3 against 78.2); the hot loop's shared-memory traffic is
    // ldmatrix through inline PTX either way.
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;                                    // [dir][stage] {K, Q, V16}
    uint8_t* wfr = ring + 2 * STAGES * STAGE;                // [dir][WBUF] W B fragments
    uint8_t* pkr = wfr + 2 * WBUF * WFR;                     // [dir][PF + 1] parked partials
    Bars* bars = reinterpret_cast<Bars*>(pkr + 2 * (PF + 1) * PKB);

    const int grp = blockIdx.x, u = blockIdx.y;
    const int col0 = grp * NCOL;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;  // fragment row / column-pair of this lane
    const int nc = p.nc;
    auto stage_ptr = [&](int dir, int s) { return ring + (dir * STAGES + s) * STAGE; };
    const bool train = p.wfin != nullptr;
    const int steps = p.steps;
    auto chunk_of = [&](int dir, int step) { return dir == 0 ? step % nc : nc - 1 - step; };
    auto wfr_ptr = [&](int dir, int b) { return reinterpret_cast<uint4*>(wfr + (dir * WBUF + b) * WFR); };
    auto active = [&](int dir) { return p.both || dir == p.dir; };

    if (threadIdx.x == 0) {
        for (int d = 0; d < 2; ++d) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(&bars->full[d][s], 1);
                mbar_init(&bars->empty[d][s], train ? 1 : 3);  // the direction's recurrence (and output) warps
            }
            for (int b = 0; b < WBUF; ++b) {
                mbar_init(&bars->wready[d][b], 1);
                mbar_init(&bars->wfree[d][b], 2);  // both output warps of the direction
            }
            for (int h = 0; h < 2; ++h)
                for (int b = 0; b <= PF; ++b) mbar_init(&bars->pfull[d][h][b], 1);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == 5) return;  // keeps the output warps off the recurrence warps' sub-partitions
    if (warp == 4) {
        // ================================ producer ======================================
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_v16);
            // every wait of this kernel leaves out the suspend-time hint: the chain of chunk
            // steps hands off through barriers, and the hardware's own limit wakes it sooner
            for (int step = 0; step < steps; ++step)
                for (int dir = 0; dir < 2; ++dir) {
                    if (!active(dir)) continue;
                    const int s = step % STAGES, use = step / STAGES;
                    if (use > 0) mbar_wait<false>(&bars->empty[dir][s], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                    const int t0 = chunk_of(dir, step) * CB;
                    uint8_t* dst = stage_ptr(dir, s);
                    mbar_expect_tx(&bars->full[dir][s], train ? STAGE - TILE : STAGE);
                    tma_load_3d(dst, &tm_k, 0, t0, u, &bars->full[dir][s]);
                    if (!train) tma_load_3d(dst + TILE, &tm_q, 0, t0, u, &bars->full[dir][s]);
                    tma_load_3d(dst + 2 * TILE, &tm_v16, col0, t0, u, &bars->full[dir][s]);
                }
        }
        return;
    }

    // A fragments (16 tokens x 16 features, k-step ks) of a 128B-swizzled [token][64] tile
    auto load_a = [&](uint32_t tile, int i, int ks, uint32_t* a) {
        const int row = 16 * i + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int chunk = 2 * ks + (lane >> 4);
        ldsm_x4(tile + swz<3>(row * ROWB + chunk * 16), a[0], a[1], a[2], a[3]);
    };

    if (warp < 2) {
        // ============================ recurrence warps ==================================
        // The warp works on transposes, so that every accumulator is already in the layout of
        // the next product's operand: R_i^T = W^T K_i^T - V_i^T and dW^T = sum_i R_i^T K_i.
        // Master copy: W^T (16 columns x 64 features) in the m16n8 accumulator layout, n-tile n
        // = features 8 n..: wt[n] = {W[8n+2t][g], W[8n+2t+1][g], W[8n+2t][8+g], W[8n+2t+1][8+g]}
        // (column indices relative to this CTA's slice).
        const int dir = warp;
        if (!active(dir)) return;
        float wt[8][4];
        {
            const float* W0 = p.w0 + (size_t)(u % p.H) * D * D + col0;
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const int f = 8 * n + 2 * t;
                wt[n][0] = W0[f * D + g];
                wt[n][1] = W0[(f + 1) * D + g];
                wt[n][2] = W0[f * D + 8 + g];
                wt[n][3] = W0[(f + 1) * D + 8 + g];
            }
        }
        // bf16 W^T as A fragments, k-step ks = features 16 ks..: pairs of the accumulators.
        // The same registers are the B fragments of W for O = Q W: (ks, column tile j) takes
        // {wa[ks][j], wa[ks][2 + j]}.
        uint32_t wa[4][4];
        auto make_a = [&]() {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                wa[ks][0] = pack_bf16(wt[2 * ks][0], wt[2 * ks][1]);
                wa[ks][1] = pack_bf16(wt[2 * ks][2], wt[2 * ks][3]);
                wa[ks][2] = pack_bf16(wt[2 * ks + 1][0], wt[2 * ks + 1][1]);
                wa[ks][3] = pack_bf16(wt[2 * ks + 1][2], wt[2 * ks + 1][3]);
            }
        };
        make_a();
        // K_i fragments (ldmatrix of the [token][feature] tile, tokens 16 i.., features
        // 16 ks..): registers {0, 2} / {1, 3} are the B fragments of K_i^T for tokens
        // 16 i + 0..7 / 16 i + 8..15.
        uint32_t ka[4][4][4];
        mbar_wait<false>(&bars->full[dir][0], 0, TTT_DEVERR_TIMEOUT_TMA);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) load_a(smem_u32(stage_ptr(dir, 0)), i, ks, ka[i][ks]);
        for (int step = 0; step < steps; ++step) {
            const int s = step % STAGES;
            uint8_t* st = stage_ptr(dir, s);
            const uint32_t kb = smem_u32(st);
            const uint32_t vb = kb + 2 * TILE;
            // ---- R_i^T = W^T K_i^T for the four tiles (k-steps outermost) ------------------
            float rt[4][2][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int nn = 0; nn < 2; ++nn)
#pragma unroll
                    for (int e = 0; e < 4; ++e) rt[i][nn][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int nn = 0; nn < 2; ++nn) mma_bf16(rt[i][nn], wa[ks], ka[i][ks][nn], ka[i][ks][2 + nn]);
            // the next step's tile and a free hand-over slot, tested now so that the tests'
            // latency passes under the dW work
            const int b = step % WBUF, use = step / WBUF;
            const int sn = (step + 1) % STAGES;
            const bool nf = step + 1 >= steps || mbar_test_wait(&bars->full[dir][sn], ((step + 1) / STAGES) & 1);
            const bool wf = train || use == 0 || mbar_test_wait(&bars->wfree[dir][b], (use - 1) & 1);
            // K_i as B fragments of dW^T (k = tokens 16 i.., n = features): transposing loads;
            // (features 16 mt + 0..7) takes {kt[i][mt][0], [2]}, (16 mt + 8..15) {[1], [3]}
            uint32_t kt[4][4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int mt = 0; mt < 4; ++mt) {
                    const int row = 16 * i + (lane >> 4) * 8 + (lane & 7);
                    const int chunk = 2 * mt + ((lane >> 3) & 1);
                    ldsm_x4_t(kb + swz<3>(row * ROWB + chunk * 16), kt[i][mt][0], kt[i][mt][1], kt[i][mt][2],
                              kt[i][mt][3]);
                }
            // R_i^T - V_i^T as the A fragments of dW^T (rows = columns, k = tokens 16 i..).
            // V_i^T comes from a transposing load of the [token][16 column] V tile: matrices
            // (tokens +0..7 | +8..15) x (columns 0..7 | 8..15).
            uint32_t ra[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t vr[4];
                const int vrow = 16 * i + ((lane >> 4) & 1) * 8 + (lane & 7);
                ldsm_x4_t(vb + vrow * (NCOL * 2) + ((lane >> 3) & 1) * 16, vr[0], vr[1], vr[2], vr[3]);
#pragma unroll
                for (int q = 0; q < 4; ++q) {  // q = 2 nn + (rows 8..15)
                    const int nn = q >> 1, hi = q & 1;
                    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vr[2 * nn + hi]));
                    // A fragment order: {rows 0-7, k 0-7}, {rows 8-15, k 0-7}, {rows 0-7, k 8-15}, ...
                    ra[i][2 * nn + hi] = pack_bf16(rt[i][nn][2 * hi] - v.x, rt[i][nn][2 * hi + 1] - v.y);
                }
            }
            // ---- dW^T = sum_i R_i^T K_i (n-tiles of 8 features) -------------------------------
            float dwt[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) dwt[n][e] = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int mt = 0; mt < 4; ++mt) {
                    mma_bf16(dwt[2 * mt], ra[i], kt[i][mt][0], kt[i][mt][2]);
                    mma_bf16(dwt[2 * mt + 1], ra[i], kt[i][mt][1], kt[i][mt][3]);
                }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->empty[dir][s]);  // K, V of this step consumed
            // the next step's K fragments load while this step's dW drains
            if (step + 1 < steps) {
                if (!nf) mbar_wait<false>(&bars->full[dir][sn], ((step + 1) / STAGES) & 1, TTT_DEVERR_TIMEOUT_TMA);
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) load_a(smem_u32(stage_ptr(dir, sn)), i, ks, ka[i][ks]);
            }
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) wt[n][e] -= p.eta_over_b * dwt[n][e];
            make_a();
            if (train) continue;  // training mode: no output per chunk
            // ---- hand W (after this step, fp32) to the output warp ---------------------------
            if (!wf) mbar_wait<false>(&bars->wfree[dir][b], (use - 1) & 1, TTT_DEVERR_TIMEOUT_PEER);
            {
                float4* dst = reinterpret_cast<float4*>(wfr_ptr(dir, b));
#pragma unroll
                for (int n = 0; n < 8; ++n) dst[n * 32 + lane] = make_float4(wt[n][0], wt[n][1], wt[n][2], wt[n][3]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->wready[dir][b]);
        }
        if (train) {  // W_final: wt[n] = {W[8n+2t][g], W[8n+2t+1][g], W[8n+2t][8+g], W[8n+2t+1][8+g]}
            float* wf = p.wfin + (size_t)u * D * D + col0;
            float* wo = p.wout ? p.wout + (size_t)u * D * D + col0 : nullptr;
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const int f = 8 * n + 2 * t;
                const float v[4] = {wt[n][0], wt[n][1], wt[n][2], wt[n][3]};
                const int fi[4] = {f, f + 1, f, f + 1}, ci[4] = {g, g, 8 + g, 8 + g};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    wf[fi[e] * D + ci[e]] = v[e];
                    if (wo) wo[fi[e] * D + ci[e]] = v[e];
                }
            }
        }
        return;
    }

    // ================================= output warps ========================================
    // O_c = Q_c W (W after the chunk's update) for the chunk's 64 tokens x 16 columns, then
    // the combine: chunk c is visited by the forward direction at step c and by the backward
    // direction at step nc-1-c; the first visit parks its fp32 partial, the second adds it.
    // For odd nc both visit the middle chunk at the same step: the forward warp parks, then
    // the backward warp adds.  One barrier over the two output warps at step nc/2 orders all
    // parks before all additions.  The partner's parked partials (64 tokens x 16 columns,
    // fp32) are fetched PF steps ahead by one TMA box each into a ring of PF + 1 slots.
    const int dir = warp >> 2, hf = warp & 1;  // warps 2, 3 / 6, 7; tiles 2 hf, 2 hf + 1 of each chunk
    if (train || !active(dir)) return;
    uint8_t* pk = pkr + dir * (PF + 1) * PKB + hf * PKH;
    const int a0 = (nc & 1) && dir == 0 ? nc / 2 + 1 : nc / 2;  // first step that adds
    auto fetch = [&](int st) {  // this warp's half of the parked partial of its step-st chunk
        if (lane == 0 && st < nc && st >= a0) {
            const int sl = (st - a0) % (PF + 1);
            mbar_expect_tx(&bars->pfull[dir][hf][sl], PKH);
            tma_load_3d(pk + sl * PKB, &tm_park, col0, chunk_of(dir, st) * CB + hf * (CB / 2), u,
                        &bars->pfull[dir][hf][sl]);
        }
    };
    for (int step = 0; step < nc; ++step) {
        const int s = step % STAGES;
        const int b = step % WBUF, use = step / WBUF;
        mbar_wait<false>(&bars->full[dir][s], (step / STAGES) & 1, TTT_DEVERR_TIMEOUT_TMA);
        const uint32_t qb = smem_u32(stage_ptr(dir, s)) + TILE;
        uint32_t qa[4][4];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) load_a(qb, OUT_TILES * hf, ks, qa[ks]);
        mbar_wait<false>(&bars->wready[dir][b], use & 1, TTT_DEVERR_TIMEOUT_PEER);
        // B fragments of W as bf16 hi + lo: k-step ks, column tile j (the recurrence warp's
        // W^T accumulator pairs, packed as its A fragments are)
        uint32_t bw[2][4][2][2];
        {
            const float4* src = reinterpret_cast<const float4*>(wfr_ptr(dir, b));
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const float4 x = src[(2 * ks) * 32 + lane], y = src[(2 * ks + 1) * 32 + lane];
                const float v[4][2] = {{x.x, x.y}, {x.z, x.w}, {y.x, y.y}, {y.z, y.w}};
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    hi[e] = pack_bf16(v[e][0], v[e][1]);
                    const float2 hf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hi[e]));
                    lo[e] = pack_bf16(v[e][0] - hf.x, v[e][1] - hf.y);
                }
                // A-fragment order {wa0, wa1, wa2, wa3} -> B fragments (j = 0: {0, 2}, j = 1: {1, 3})
                bw[0][ks][0][0] = hi[0];
                bw[0][ks][1][0] = hi[1];
                bw[0][ks][0][1] = hi[2];
                bw[0][ks][1][1] = hi[3];
                bw[1][ks][0][0] = lo[0];
                bw[1][ks][1][0] = lo[1];
                bw[1][ks][0][1] = lo[2];
                bw[1][ks][1][1] = lo[3];
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->wfree[dir][b]);
        float o[OUT_TILES][2][4];  // tile 2 hf + i
#pragma unroll
        for (int i = 0; i < OUT_TILES; ++i) {
            uint32_t qn[4][4];
            if (i + 1 < OUT_TILES) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) load_a(qb, OUT_TILES * hf + i + 1, ks, qn[ks]);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) o[i][j][e] = 0.f;
#pragma unroll
            for (int hl = 0; hl < 2; ++hl)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int j = 0; j < 2; ++j) mma_bf16(o[i][j], qa[ks], bw[hl][ks][j][0], bw[hl][ks][j][1]);
            if (i + 1 < OUT_TILES) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int e = 0; e < 4; ++e) qa[ks][e] = qn[ks][e];
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->empty[dir][s]);  // Q of this step consumed
        const size_t tok0 = (size_t)u * p.N + (size_t)chunk_of(dir, step) * CB;
        auto out_index = [&](int i, int j, int h) {  // i: this warp's tile 2 hf + i
            return (tok0 + 16 * (OUT_TILES * hf + i) + g + 8 * h) * D + col0 + 8 * j + 2 * t;
        };
        if (!p.both) {  // one-way scan: this is the chunk's output
#pragma unroll
            for (int i = 0; i < OUT_TILES; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        *reinterpret_cast<uint32_t*>(&p.out[out_index(i, j, h)]) = pack_bf16(o[i][j][2 * h], o[i][j][2 * h + 1]);
            continue;
        }
        if (step < a0) {  // first visit: park the fp32 partial
#pragma unroll
            for (int i = 0; i < OUT_TILES; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        *reinterpret_cast<float2*>(&p.park[out_index(i, j, h)]) =
                            make_float2(o[i][j][2 * h], o[i][j][2 * h + 1]);
        }
        if (step == nc / 2) {
            // every park is written, and visible to the tensor-copy reads that follow
            asm volatile("fence.proxy.async.global;" ::: "memory");
            asm volatile("bar.sync 1, 128;" ::: "memory");  // the four output warps
#pragma unroll
            for (int k = 0; k < PF; ++k) fetch(a0 + k);
        }
        if (step >= a0) {
            // second visit: add the partner's partial, round once, store O.  Every read of the
            // slot is issued before the first store, so that no read waits behind a store.
            mbar_wait<false>(&bars->pfull[dir][hf][(step - a0) % (PF + 1)], ((step - a0) / (PF + 1)) & 1,
                      TTT_DEVERR_TIMEOUT_TMA);
            const float* other = reinterpret_cast<const float*>(pk + ((step - a0) % (PF + 1)) * PKB);
            float2 x[OUT_TILES][2][2];
#pragma unroll
            for (int i = 0; i < OUT_TILES; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        x[i][j][h] = *reinterpret_cast<const float2*>(other + (16 * i + g + 8 * h) * NCOL + 8 * j + 2 * t);
#pragma unroll
            for (int i = 0; i < OUT_TILES; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        *reinterpret_cast<uint32_t*>(&p.out[out_index(i, j, h)]) =
                            pack_bf16(o[i][j][2 * h] + x[i][j][h].x, o[i][j][2 * h + 1] + x[i][j][h].y);
            __syncwarp();  // every lane has read the slot before it is refilled
            fetch(step + PF);
        }
    }
}

}  // namespace chk

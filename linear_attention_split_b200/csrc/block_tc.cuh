// block_tc.cuh -- the ViT^3 TTT block around the TTT-Linear core on the tcgen05 tensor cores,
// bf16, block width C = 64 (the high-resolution stage-1 width of the hierarchical model).
//
// Operation (ViT^3 blog: the block projects its input to Q, K, V, trains the inner model on
// (K, V) and applies it to Q -- "TTT Block 长什么样" -- and its official code joins a GLU-style
// main branch with a 3x3 depthwise-conv branch, concatenates them and projects back to the
// input width -- "从官方代码看…"), per image with x [N, C] on the Hg x Wg grid:
//     [Q | K | V | G] = x Wqkvg,   O = TTT-Linear(Q, K, V) per head,
//     y = [O * sigmoid(G) | dwconv3x3(x)] Wo
// Two kernels around the core (the full-batch step needs every token's K and V before any
// output, so the core is a kernel of its own):
//   proj : persistent, one CTA per SM looping over the 128-token tiles: x tiles through a TMA
//          ring, Wqkvg resident (MN-major), x Wqkvg into one of two 256-column TMEM
//          accumulators, so that the epilogue -- Q, K, V and G token-major [B, N, C] in bf16,
//          staged per tile in one of two shared-memory buffers (128-byte swizzle) and written
//          by one TMA store per tensor -- of one tile overlaps the loads and the MMAs of the
//          next, and its stores drain while the next tile is staged.  The heads of Q, K, V sit
//          side by side in each token's C = 64 features, the layout in which the core (the
//          tensor-core TTT-Linear kernel) takes an image as one unit of 64 features with a
//          block-diagonal W0.
//   out  : persistent, one CTA per SM looping over the 128-token tiles.  Per tile sixteen warps
//          build Z = [O * sigmoid(G) | dwconv3x3(x)] (128 x 128, fp32, kept as bf16 hi + lo,
//          K-major) in shared memory -- the gate from O and G rows (16-byte loads, issued one
//          tile ahead into registers), the conv from a window of x rows that one TMA box brings
//          in (the tile's rows and one grid row plus one token on each side, at most 256 rows,
//          so Wg <= 63) -- then one MMA chain Z_hi Wo + Z_lo Wo (K = 128, N = 64) and the
//          epilogue stores y in bf16.  Two x windows, two Z buffers and two TMEM accumulators:
//          while the tensor cores project tile i, the warps build tile i + 1 and the producer
//          brings tile i + 2's window.
// No token-tile output is written twice and no intermediate of the out kernel (Z) goes to HBM.
#pragma once
#include "common.cuh"

namespace blk {

constexpr int C = 64;
constexpr int ROWB = C * 2;             // 128 bytes per token row
constexpr int MT = 128;                 // tokens per tile
constexpr int XT = MT * ROWB;           // 16 KB
constexpr int WQ = C * 4 * C * 2;       // Wqkvg, 32 KB (four 64-column atoms)
constexpr int ZT = MT * 2 * C * 2;      // Z hi or lo, 32 KB each (two 64-column K-major atoms)
constexpr int WO = 2 * C * C * 2;       // Wo, 16 KB
constexpr int XW = 256;                 // rows of the x window (tile + halo)
constexpr int MAX_WG = (XW - MT) / 2 - 1;  // widest grid the window covers (63)
constexpr int P_WARPS = 8;              // proj: eight epilogue warps (row quarter x column half)
constexpr int THREADS = 32 * P_WARPS + 64;  // + one MMA issuer warp and one x-tile producer warp
constexpr int PXS = 4;                  // proj: x tile ring slots
constexpr int O_WARPS = 16;             // out: sixteen Z / epilogue warps (row quarter x 16 channels)
constexpr int O_THREADS = 32 * O_WARPS + 32;

struct PParams {
    long long rows;                     // B * N (Q, K, V, G [B, N, C] each, heads side by side in C)
};
struct PBars {
    uint64_t wfull, xfull[PXS], xempty[PXS], done[2], tfree[2];
    uint32_t tmem_base;
};
constexpr int p_smem_bytes() { return PXS * XT + WQ + 8 * XT + (int)sizeof(PBars) + 1024; }

__global__ void __launch_bounds__(THREADS, 1)
    proj_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g, const PParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* xs = smem_align<1024>(smem_raw);
    uint8_t* ws = xs + PXS * XT;
    uint8_t* st = ws + WQ;  // two buffers of a tile's Q, K, V, G (16 KB each, 128-byte swizzle) for the TMA stores
    PBars* bars = reinterpret_cast<PBars*>(st + 8 * XT);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long ntiles = (p.rows + MT - 1) / MT;
    const int nj = (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);  // tiles of this CTA (>= 1)
    auto row0_of = [&](int j) { return ((long long)blockIdx.x + (long long)j * gridDim.x) * MT; };
    // Launched with programmatic stream serialization: the first x tiles go into L2 while the
    // previous grid on the stream may still run (a prefetch only warms the coherent L2); every
    // load and store of this grid comes after griddep_wait.
    if (threadIdx.x == 32 * (P_WARPS + 1))
        for (int j = 0; j < min(PXS, nj); ++j) tma_prefetch_l2_3d(&tm_x, 0, (int)row0_of(j), 0);
    griddep_wait();
    griddep_launch();
    if (threadIdx.x == 32 * P_WARPS) {
        mbar_init(&bars->wfull, 1);
        for (int s = 0; s < PXS; ++s) {
            mbar_init(&bars->xfull[s], 1);
            mbar_init(&bars->xempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->done[b], 1);
            mbar_init(&bars->tfree[b], P_WARPS);
        }
        mbar_fence_init();
    }
    if (warp == P_WARPS) tc::alloc(&bars->tmem_base, 512);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = bars->tmem_base;
    if (warp == P_WARPS + 1) {
        // ================================ producer: weights, then the x tiles ================
        if (lane == 0) {
            mbar_expect_tx(&bars->wfull, WQ);
#pragma unroll
            for (int a = 0; a < 4; ++a) tma_load_3d(ws + a * 8192, &tm_w, a * 64, 0, 0, &bars->wfull);
            for (int j = 0; j < nj; ++j) {
                const int s = j % PXS, use = j / PXS;
                if (use > 0) mbar_wait(&bars->xempty[s], (use - 1) & 1, TTT_DEVERR_TIMEOUT_PEER);
                mbar_expect_tx(&bars->xfull[s], XT);  // out-of-range rows are zero-filled and counted
                tma_load_3d(xs + s * XT, &tm_x, 0, (int)row0_of(j), 0, &bars->xfull[s]);
            }
        }
    } else if (warp == P_WARPS) {
        // ================================ MMA issuer ===========================================
        if (lane == 0) {
            mbar_wait(&bars->wfull, 0, TTT_DEVERR_TIMEOUT_TMA);
            const uint32_t wa = smem_u32(ws);
            constexpr uint32_t ID = tc::idesc_bf16(128, 256, 0, 1);  // A K-major, B MN-major, N = 256
            for (int j = 0; j < nj; ++j) {
                const int s = j % PXS, b = j & 1;
                mbar_wait(&bars->xfull[s], (j / PXS) & 1, TTT_DEVERR_TIMEOUT_TMA);
                if (j >= 2) mbar_wait(&bars->tfree[b], ((j >> 1) - 1) & 1, TTT_DEVERR_TIMEOUT_PEER);
                tc::fence_after();
                const uint32_t xa = smem_u32(xs + s * XT);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tmem + b * 256, tc::smem_desc(xa + ks * 32, 16, 1024, 2),
                                 tc::smem_desc(wa + ks * 2048, 8192, 1024, 2), ID, ks > 0 ? 1 : 0);
                tc::commit(&bars->done[b]);
                tc::commit(&bars->xempty[s]);  // the slot may take a later tile
            }
        }
    } else {
        // ================================ epilogue (eight warps) ===============================
        const int q4 = warp & 3, ch = warp >> 2;  // lane quarter, column half (Q, K | V, G)
        const int row = q4 * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
        const CUtensorMap* maps[4] = {&tm_q, &tm_k, &tm_v, &tm_g};
        const bool storer = threadIdx.x == 0;
        for (int j = 0; j < nj; ++j) {
            const int b = j & 1;
            mbar_wait(&bars->done[b], (j >> 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
            tc::fence_after();
            // the stores of tile j - 2 (this staging buffer) have read it; tile j - 1's may go on
            uint8_t* stj = st + (j & 1) * 4 * XT;
            if (storer) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
            asm volatile("bar.sync 1, %0;" ::"n"(32 * P_WARPS) : "memory");
            // this warp's 128 columns in two TMEM round trips of four 16-column chunks
#pragma unroll 1
            for (int g4 = 0; g4 < 2; ++g4) {
                float v[4][16];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) tc::ld16(lane_base + b * 256 + ch * 2 * C + (4 * g4 + c4) * 16, v[c4]);
                tc::wait_ld();
                if (g4 == 1) {  // the accumulator has been read: the next tile but one may use it
                    tc::fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->tfree[b]);
                }
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const int j0 = ch * 2 * C + (4 * g4 + c4) * 16;
                    const int which = j0 / C, c = j0 % C;
                    const float* x = v[c4];
                    uint8_t* tile = stj + which * XT + row * ROWB;
                    const int k0 = c / 8;  // 16-byte chunk of the 128-byte row
                    *reinterpret_cast<uint4*>(tile + ((k0 ^ (row & 7)) << 4)) =
                        make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                                   pack_bf16(x[6], x[7]));
                    *reinterpret_cast<uint4*>(tile + (((k0 + 1) ^ (row & 7)) << 4)) =
                        make_uint4(pack_bf16(x[8], x[9]), pack_bf16(x[10], x[11]), pack_bf16(x[12], x[13]),
                                   pack_bf16(x[14], x[15]));
                }
            }
            fence_proxy_async_smem();  // read next by the TMA stores
            asm volatile("bar.sync 1, %0;" ::"n"(32 * P_WARPS) : "memory");
            if (storer) {  // rows past the tensor are clipped by the hardware
#pragma unroll
                for (int w = 0; w < 4; ++w) tma_store_3d(maps[w], 0, (int)row0_of(j), 0, stj + w * XT);
                tma_store_commit();
            }
        }
        if (storer) tma_store_wait_all();
    }
    tc::fence_before();
    __syncthreads();
    if (warp == P_WARPS) tc::dealloc(tmem, 512);
}

struct OParams {
    const __nv_bfloat16* x;             // [B, N, C]
    const __nv_bfloat16* o;             // [B, N, C] (the core's output, heads side by side)
    const __nv_bfloat16* g;             // [B, N, C]
    const float* wc;                    // [C, 3, 3]
    __nv_bfloat16* y;                   // [B, N, C]
    long long rows;
    int N, Hg, Wg;
};
struct OBars {
    uint64_t wfull, xfull[2], xempty[2], zready[2], done[2], tfree[2];
    uint32_t tmem_base;
};
constexpr int o_smem_bytes() { return 4 * ZT + 2 * XW * ROWB + WO + C * 9 * 4 + (int)sizeof(OBars) + 1024; }

// 1 / (1 + e^-z) with the fast exponential and the fast (approximate, ~2 ulp) division
__device__ __forceinline__ float sigmoidf_(float z) { return __fdividef(1.f, 1.f + __expf(-z)); }
// eight fp32 values -> bf16 hi and lo = bf16(x - hi), packed
__device__ __forceinline__ void split8(const float* v, uint4& hi, uint4& lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        h[i] = pack_bf16(v[2 * i], v[2 * i + 1]);
        const float2 hf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h[i]));
        l[i] = pack_bf16(v[2 * i] - hf.x, v[2 * i + 1] - hf.y);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__global__ void __launch_bounds__(O_THREADS, 1)
    out_kernel(const __grid_constant__ CUtensorMap tm_wo, const __grid_constant__ CUtensorMap tm_xw, const OParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_align<1024>(smem_raw);
    auto zbuf = [&](int b) { return base + b * 2 * ZT; };              // Z hi, then Z lo
    auto xwin = [&](int b) { return base + 4 * ZT + b * XW * ROWB; };  // x rows around a tile (128-byte swizzle)
    uint8_t* wos = base + 4 * ZT + 2 * XW * ROWB;
    float* wcs = reinterpret_cast<float*>(wos + WO);
    OBars* bars = reinterpret_cast<OBars*>(wcs + C * 9);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long ntiles = (p.rows + MT - 1) / MT;
    const int nj = (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);  // tiles of this CTA
    auto tile_of = [&](int j) { return (long long)blockIdx.x + (long long)j * gridDim.x; };
    // Launched with programmatic stream serialization: the first two x windows go into L2 while
    // the previous grid (the core) may still run; every load and store comes after griddep_wait.
    if (threadIdx.x == 32 * O_WARPS)
        for (int j = 0; j < 2 && j < nj; ++j)
            tma_prefetch_l2_3d(&tm_xw, 0, (int)max(0LL, tile_of(j) * MT - (p.Wg + 1)), 0);
    griddep_wait();
    griddep_launch();
    if (threadIdx.x == 32 * O_WARPS) {
        mbar_init(&bars->wfull, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->xfull[b], 1);
            mbar_init(&bars->xempty[b], O_WARPS);
            mbar_init(&bars->zready[b], O_WARPS);
            mbar_init(&bars->done[b], 1);
            mbar_init(&bars->tfree[b], O_WARPS);
        }
        mbar_fence_init();
    }
    // taps regrouped as [8-channel chunk][tap][8 channels]: one tap of a chunk is two float4
    for (int e = threadIdx.x; e < C * 9; e += O_THREADS) {
        const int ch = e / 9, tap = e % 9;
        wcs[((ch >> 3) * 9 + tap) * 8 + (ch & 7)] = p.wc[e];
    }
    if (warp == O_WARPS) tc::alloc(&bars->tmem_base, 128);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = bars->tmem_base;
    if (warp == O_WARPS) {
        // ======================= producer of the x windows and MMA issuer =========================
        if (lane == 0) {
            auto load_x = [&](int j) {  // the window of this CTA's j-th tile into buffer j & 1
                const int b = j & 1;
                if (j >= 2) mbar_wait(&bars->xempty[b], ((j >> 1) - 1) & 1, TTT_DEVERR_TIMEOUT_PEER);
                mbar_expect_tx(&bars->xfull[b], XW * ROWB);  // rows outside the tensor are zero-filled
                tma_load_3d(xwin(b), &tm_xw, 0, (int)(tile_of(j) * MT - (p.Wg + 1)), 0, &bars->xfull[b]);
            };
            mbar_expect_tx(&bars->wfull, WO);
            tma_load_3d(wos, &tm_wo, 0, 0, 0, &bars->wfull);
            for (int j = 0; j < 2 && j < nj; ++j) load_x(j);
            mbar_wait(&bars->wfull, 0, TTT_DEVERR_TIMEOUT_TMA);
            const uint32_t wa = smem_u32(wos);
            constexpr uint32_t ID = tc::idesc_bf16(128, 64, 0, 1);  // A K-major, B MN-major
            for (int j = 0; j < nj; ++j) {
                const int b = j & 1;
                mbar_wait(&bars->zready[b], (j >> 1) & 1, TTT_DEVERR_TIMEOUT_PEER);
                if (j >= 2) mbar_wait(&bars->tfree[b], ((j >> 1) - 1) & 1, TTT_DEVERR_TIMEOUT_PEER);
                tc::fence_after();
#pragma unroll
                for (int hl = 0; hl < 2; ++hl) {
                    const uint32_t za = smem_u32(zbuf(b) + hl * ZT);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        tc::mma_bf16(tmem + b * 64, tc::smem_desc(za + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, 2),
                                     tc::smem_desc(wa + ks * 2048, 8192, 1024, 2), ID, (hl > 0 || ks > 0) ? 1 : 0);
                }
                tc::commit(&bars->done[b]);
                if (j + 2 < nj) load_x(j + 2);  // this tile's window has been read (zready)
            }
        }
    } else {
        // ======================= Z builders and epilogue (sixteen warps) ==========================
        // warp w: token rows of lane quarter w % 4, channels 16 (w / 4) .. + 15 (two 8-channel chunks)
        const int q4 = warp & 3, cg = warp >> 2;
        const int row = q4 * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
        // the gate half's O and G rows of tile j (two 8-channel chunks each)
        struct OG {
            uint4 o[2], g[2];
        };
        auto load_og = [&](int j) {
            OG r;
            const long long R = tile_of(j) * MT + row;
            const bool valid = R < p.rows;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int c = cg * 16 + q * 8;
                r.o[q] = valid ? *reinterpret_cast<const uint4*>(p.o + R * C + c) : make_uint4(0, 0, 0, 0);
                r.g[q] = valid ? *reinterpret_cast<const uint4*>(p.g + R * C + c) : make_uint4(0, 0, 0, 0);
            }
            return r;
        };
        auto epilogue = [&](int j) {  // y of tile j from its TMEM accumulator
            const int b = j & 1;
            mbar_wait(&bars->done[b], (j >> 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
            tc::fence_after();
            float v[16];
            tc::ld16(lane_base + b * 64 + cg * 16, v);
            tc::wait_ld();
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->tfree[b]);
            const long long R = tile_of(j) * MT + row;
            if (R < p.rows) {
                uint4* d4 = reinterpret_cast<uint4*>(p.y + R * C + cg * 16);
                d4[0] = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                                   pack_bf16(v[6], v[7]));
                d4[1] = make_uint4(pack_bf16(v[8], v[9]), pack_bf16(v[10], v[11]), pack_bf16(v[12], v[13]),
                                   pack_bf16(v[14], v[15]));
            }
        };
        OG cur = load_og(0);  // nj >= 1: the grid has at most one CTA per tile
        for (int j = 0; j < nj; ++j) {
            const int b = j & 1;
            const OG nxt = load_og(j + 1 < nj ? j + 1 : j);  // next tile's rows, requested before this tile's work
            const long long R = tile_of(j) * MT + row;
            const bool valid = R < p.rows;
            const long long t = valid ? R % p.N : 0;
            const int py = (int)(t / p.Wg), px = (int)(t % p.Wg);
            // Z buffer b was last read by tile j - 2's MMAs, which this warp's epilogue of tile
            // j - 2 (previous iteration) waited for
            mbar_wait(&bars->xfull[b], (j >> 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
            const uint8_t* xw = xwin(b);
            uint8_t* zs = zbuf(b);
            uint8_t* zl = zs + ZT;
            const int wrow = row + p.Wg + 1;  // this token's row in the x window
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int c = cg * 16 + q * 8, chunk = c >> 3;
                uint4 mz = make_uint4(0, 0, 0, 0), dz = mz, mzl = mz, dzl = mz;
                if (valid) {
                    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&cur.o[q]);
                    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&cur.g[q]);
                    float m[8];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 of = __bfloat1622float2(o2[i]), gf = __bfloat1622float2(g2[i]);
                        m[2 * i] = of.x * sigmoidf_(gf.x);
                        m[2 * i + 1] = of.y * sigmoidf_(gf.y);
                    }
                    split8(m, mz, mzl);
                    float2 acc2[4] = {};  // channel pairs (2i, 2i + 1)
#pragma unroll
                    for (int a = 0; a < 3; ++a)
#pragma unroll
                        for (int bb = 0; bb < 3; ++bb) {
                            const int yy = py + a - 1, xx = px + bb - 1;
                            if (yy < 0 || yy >= p.Hg || xx < 0 || xx >= p.Wg) continue;
                            const int wr = wrow + (a - 1) * p.Wg + (bb - 1);  // same image: inside the window
                            const uint4 raw = *reinterpret_cast<const uint4*>(xw + wr * ROWB + ((chunk ^ (wr & 7)) << 4));
                            const float4* wt = reinterpret_cast<const float4*>(wcs + (chunk * 9 + a * 3 + bb) * 8);
                            const float4 w0 = wt[0], w1 = wt[1];
                            const float2 wp[4] = {make_float2(w0.x, w0.y), make_float2(w0.z, w0.w),
                                                  make_float2(w1.x, w1.y), make_float2(w1.z, w1.w)};
                            const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i)  // bf16 pair -> fp32 pair, then one packed fma
                                acc2[i] = __ffma2_rn(wp[i],
                                                     make_float2(__uint_as_float(rw[i] << 16),
                                                                 __uint_as_float(rw[i] & 0xffff0000u)),
                                                     acc2[i]);
                        }
                    float acc[8];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        acc[2 * i] = acc2[i].x;
                        acc[2 * i + 1] = acc2[i].y;
                    }
                    split8(acc, dz, dzl);
                }
                const uint32_t off = swz<3>((uint32_t)row * ROWB + c * 2);
                *reinterpret_cast<uint4*>(zs + off) = mz;
                *reinterpret_cast<uint4*>(zs + 16384 + off) = dz;
                *reinterpret_cast<uint4*>(zl + off) = mzl;
                *reinterpret_cast<uint4*>(zl + 16384 + off) = dzl;
            }
            fence_proxy_async_smem();  // read next by the tensor cores
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars->xempty[b]);  // the window may take tile j + 2's rows
                mbar_arrive(&bars->zready[b]);
            }
            if (j >= 1) epilogue(j - 1);
            cur = nxt;
        }
        epilogue(nj - 1);
    }
    tc::fence_before();
    __syncthreads();
    if (warp == O_WARPS) tc::dealloc(tmem, 128);
}

}  // namespace blk

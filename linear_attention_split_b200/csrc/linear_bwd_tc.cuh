// linear_bwd_tc.cuh -- backward of the TTT-Linear full-batch step on the tcgen05 tensor cores,
// bf16, d = 64 (outer training through the inner step).
//
// Operation: the layer ("ViT^3" blog, steps 1-3; TTT-Linear of the TTT abstract) is, per unit,
//     W* = W0 - (eta/N)(G W0 - C),  G = K^T K,  C = K^T V,   O = Q W*,
// and for an upstream gradient dO the chain rule gives (M = Q^T dO, A = W0 M^T + M W0^T):
//     dQ = dO W*^T,   dV = (eta/N) K M,   dK = -(eta/N)(K A - V M^T),
//     dW0 = sum over the batch entries of a head of  M - (eta/N) G M.
// The gradient of the inner step is written by hand, as the ViT^3 blog notes the official code
// does ("从官方代码看…", third point).  Four launches:
//   reduce : CTAs split each unit's tokens (as the forward does); per tile of V, K, Q, dO two
//            tcgen05 MMAs accumulate [V | K]^T K (C^T and G) and [Q | dO]^T dO (M in its first
//            64 rows) in TMEM; each CTA writes its partial G, C^T, M (fp32) to the workspace.
//   finish : three blocks per unit, one per d x d product (G W0, W0 M^T, G M), add the partials
//            in split order (deterministic) and form, in fp32 on the CUDA cores, W*, A and
//            dW0_u; they write the four d x d right-hand operands of the token pass -- W*,
//            (eta/N) M^T, -(eta/N) A, (eta/N) M -- each as bf16 hi + lo (row-major rows = output
//            columns, i.e. K-major).
//   apply  : per tile of dO, K, V: dQ = dO W*, dV = K (eta/N) M^T-operand, dK = K (-eta/N A) +
//            V (eta/N M), each product taken as hi + lo into one 64-column TMEM accumulator;
//            the outputs are written as bf16 over the consumed input tiles and stored by TMA.
//   dw0    : dW0[h] = sum_b dW0_(b,h) in batch order (the CUDA-core kernel of simt.cuh).
// Every wait is bounded (common.cuh).
#pragma once
#include "common.cuh"

namespace lbw {

constexpr int D = 64;
constexpr int ROWB = 128;                 // bytes per token row (64 bf16)
constexpr int MT = 128;                   // rows reserved per tile (TT <= MT are used)
constexpr int TILE = MT * ROWB;           // 16 KB
constexpr int OP = D * ROWB;              // one 64 x 64 bf16 K-major operand, 8 KB
constexpr int DD = D * D;

// ----------------------------------------------------------------------------- reduce ----
constexpr int R_STAGES = 3;
constexpr int R_STAGE = 4 * TILE;         // V, K, Q, dO
constexpr int R_THREADS = 64 + 128;       // producer, issuer, 4 epilogue warps
constexpr uint32_t IDESC_GRAM = tc::idesc_bf16(128, 64, 1, 1);  // A MN-major, B MN-major
constexpr uint32_t IDESC_N64 = tc::idesc_bf16(128, 64, 0, 0);   // A K-major, B K-major
constexpr uint32_t IDESC_N128 = tc::idesc_bf16(128, 128, 0, 0); // A K-major, B K-major

struct RParams {
    float* part;      // [U][S][3][64][64]: G, C^T, M
    int TT, n_tiles;  // token rows per tile, tiles per unit
};
struct RBars {
    uint64_t full[R_STAGES], empty[R_STAGES], done;
    uint32_t tmem_base;
};
constexpr int r_smem_bytes() { return R_STAGES * R_STAGE + (int)sizeof(RBars) + 1024; }

__global__ void __launch_bounds__(R_THREADS, 1)
    reduce_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_g, const RParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = smem_align<1024>(smem_raw);
    RBars* bars = reinterpret_cast<RBars*>(ring + R_STAGES * R_STAGE);
    const int S = gridDim.x, r = blockIdx.x, u = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int TT = p.TT;
    const int n_t = r < p.n_tiles ? (p.n_tiles - r + S - 1) / S : 0;
    // Launched with programmatic stream serialization: the first tiles go into L2 while the
    // previous grid on the stream may still run (a prefetch only warms the coherent L2); every
    // load and store of this grid comes after griddep_wait.
    if (threadIdx.x == 0)
        for (int i = 0; i < min(R_STAGES, n_t); ++i) {
            const int row = (r + i * S) * TT;
            tma_prefetch_l2_3d(&tm_v, 0, row, u);
            tma_prefetch_l2_3d(&tm_k, 0, row, u);
            tma_prefetch_l2_3d(&tm_q, 0, row, u);
            tma_prefetch_l2_3d(&tm_g, 0, row, u);
        }
    griddep_wait();
    griddep_launch();
    if (threadIdx.x == 0) {
        for (int s = 0; s < R_STAGES; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        mbar_init(&bars->done, 1);
        mbar_fence_init();
    }
    if (warp == 1) tc::alloc(&bars->tmem_base, 128);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_g);
            for (int i = 0; i < n_t; ++i) {
                const int slot = i % R_STAGES, use = i / R_STAGES;
                if (use > 0) mbar_wait(&bars->empty[slot], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                uint8_t* dst = ring + slot * R_STAGE;
                const int row = (r + i * S) * TT;
                mbar_expect_tx(&bars->full[slot], 4 * TT * ROWB);
                tma_load_3d(dst, &tm_v, 0, row, u, &bars->full[slot]);
                tma_load_3d(dst + TILE, &tm_k, 0, row, u, &bars->full[slot]);
                tma_load_3d(dst + 2 * TILE, &tm_q, 0, row, u, &bars->full[slot]);
                tma_load_3d(dst + 3 * TILE, &tm_g, 0, row, u, &bars->full[slot]);
                if (i == R_STAGES - 1)  // the rest of this CTA's tiles into L2 now
                    for (int j = R_STAGES; j < n_t; ++j) {
                        const int rj = (r + j * S) * TT;
                        tma_prefetch_l2_3d(&tm_v, 0, rj, u);
                        tma_prefetch_l2_3d(&tm_k, 0, rj, u);
                        tma_prefetch_l2_3d(&tm_q, 0, rj, u);
                        tma_prefetch_l2_3d(&tm_g, 0, rj, u);
                    }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int i = 0; i < n_t; ++i) {
                const int slot = i % R_STAGES;
                mbar_wait(&bars->full[slot], (i / R_STAGES) & 1, TTT_DEVERR_TIMEOUT_TMA);
                tc::fence_after();
                const uint32_t vb = smem_u32(ring + slot * R_STAGE);
                // [V | K]^T K and [Q | dO]^T dO: A MN-major over two adjacent tiles (LBO), B MN-major
                const uint64_t a1 = tc::smem_desc(vb, TILE, 1024, 2), b1 = tc::smem_desc(vb + TILE, TILE, 1024, 2);
                const uint64_t a2 = tc::smem_desc(vb + 2 * TILE, TILE, 1024, 2);
                const uint64_t b2 = tc::smem_desc(vb + 3 * TILE, TILE, 1024, 2);
                for (int ks = 0; ks < TT / 16; ++ks) {
                    const int acc = (i > 0 || ks > 0) ? 1 : 0;
                    tc::mma_bf16(tmem, a1 + (uint64_t)(ks * 128), b1 + (uint64_t)(ks * 128), IDESC_GRAM, acc);
                    tc::mma_bf16(tmem + 64, a2 + (uint64_t)(ks * 128), b2 + (uint64_t)(ks * 128), IDESC_GRAM, acc);
                }
                tc::commit(&bars->empty[slot]);
            }
            tc::commit(&bars->done);
        }
    } else {
        // lane row: rows 0-63 hold C^T (first accumulator) and M (second), rows 64-127 hold G
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
        float* part = p.part + ((size_t)u * S + r) * 3 * DD;
        if (n_t > 0) {
            mbar_wait(&bars->done, 0, TTT_DEVERR_TIMEOUT_TMA);
            tc::fence_after();
        }
#pragma unroll
        for (int acc = 0; acc < 2; ++acc) {
            if (acc == 1 && row >= D) break;  // rows 64-127 of [Q | dO]^T dO are not needed
            float* dst = acc == 0 ? (row >= D ? part + (row - D) * D : part + DD + row * D) : part + 2 * DD + row * D;
#pragma unroll
            for (int c16 = 0; c16 < 4; ++c16) {
                float x[16];
                if (n_t > 0) {
                    tc::ld16(lane_base + acc * 64 + c16 * 16, x);
                    tc::wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    *reinterpret_cast<float4*>(dst + c16 * 16 + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
            }
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) tc::dealloc(tmem, 128);
}

// ----------------------------------------------------------------------------- finish ----
// Grid (U, 3): block (u, j) forms one d x d product of unit u on the CUDA cores in fp32 --
// j = 0: G W0,  j = 1: W0 M^T,  j = 2: G M -- with 256 threads, each holding a 4 x 4 tile of
// it (outer products over k from two shared-memory operands laid out [k][row] and [k][col]:
// two float4 reads per k), and writes what follows from that product:
//   j = 0: W* = W0 - (eta/N)(G W0 - C)                          -> W* hi/lo
//   j = 1: A = W0 M^T + (W0 M^T)^T                              -> -(eta/N) A hi/lo, and the
//          M operands (eta/N) M^T hi/lo, (eta/N) M hi/lo
//   j = 2: dW0_u = M - (eta/N) G M
// The S partials are added in split order (deterministic), and every load of a matrix is
// issued before the first of them is used (the partials were written by the previous kernel).
struct FParams {
    const float* part;     // [U][S][3][64][64]: G, C^T, M
    const float* w0;       // [H][64][64]
    __nv_bfloat16* ops;    // [U][8][64][64]: the slots OP_* below (W*, (eta/N) M^T, -(eta/N) A, (eta/N) M, hi and lo)
    float* dw0u;           // [U][64][64]
    int H, S;              // S <= 8
    float eta_over_n;
};
constexpr int FLD = D + 4;                // padded row of the shared-memory operands (float4 aligned)
// Slots of the eight right-hand operands (64 x 64 bf16 each, [U][8][64][64]).  (eta/N) M^T and
// -(eta/N) A sit side by side, hi next to hi and lo next to lo, so that K [M^T-op | A-op] is one
// N = 128 product giving dV and the first term of dK in adjacent accumulator columns.
constexpr int OP_WS_HI = 0, OP_WS_LO = 1, OP_MT_HI = 2, OP_A_HI = 3, OP_MT_LO = 4, OP_A_LO = 5, OP_M_HI = 6,
              OP_M_LO = 7;
constexpr int f_smem_bytes() { return 2 * D * FLD * 4; }

// x[i] = sum over s < S (in order) of matrix `which` of the partials, float4 i of this thread
// (elements 4 (tid + 256 i) ..): all S x 4 loads are issued before the first add
__device__ __forceinline__ void f_load_sum(const float* part, int S, int which, int tid, float4 (&x)[4]) {
    float4 v[8][4];
#pragma unroll
    for (int s = 0; s < 8; ++s)
        if (s < S)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                v[s][i] = __ldg(reinterpret_cast<const float4*>(part + ((size_t)s * 3 + which) * DD) + tid + 256 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < 8; ++s)
        if (s < S)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                x[i].x += v[s][i].x;
                x[i].y += v[s][i].y;
                x[i].z += v[s][i].z;
                x[i].w += v[s][i].w;
            }
}
// float4 f of a d x d matrix (elements 4 f .. 4 f + 3 of row 4 f / 64) into an operand, as is
// ([row][col]) or transposed
__device__ __forceinline__ void f_put4(float* op, int f, float4 x, bool transposed) {
    const int row = f >> 4, col = (f & 15) * 4;
    if (transposed) {
        op[col * FLD + row] = x.x;
        op[(col + 1) * FLD + row] = x.y;
        op[(col + 2) * FLD + row] = x.z;
        op[(col + 3) * FLD + row] = x.w;
    } else {
        *reinterpret_cast<float4*>(op + row * FLD + col) = x;
    }
}
__device__ __forceinline__ void put_hilo4(__nv_bfloat16* ops, int mh, int ml, int row, int col, const float (&x)[4]) {
    uint32_t hi[2], lo[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
        const float2 hf = __bfloat1622float2(h);
        const __nv_bfloat162 l = __floats2bfloat162_rn(x[2 * q] - hf.x, x[2 * q + 1] - hf.y);
        hi[q] = *reinterpret_cast<const uint32_t*>(&h);
        lo[q] = *reinterpret_cast<const uint32_t*>(&l);
    }
    *reinterpret_cast<uint2*>(ops + ((size_t)mh * D + row) * D + col) = make_uint2(hi[0], hi[1]);
    *reinterpret_cast<uint2*>(ops + ((size_t)ml * D + row) * D + col) = make_uint2(lo[0], lo[1]);
}

__global__ void __launch_bounds__(256) finish_kernel(const FParams p) {
    extern __shared__ float fsm[];
    float* Aop = fsm;                 // [k][row]
    float* Bop = fsm + D * FLD;       // [k][col]
    const int u = blockIdx.x, j = blockIdx.y, tid = threadIdx.x;
    griddep_wait();  // the partials of the reduce grid
    griddep_launch();
    const float* W0 = p.w0 + (size_t)(u % p.H) * DD;
    const float* part = p.part + (size_t)u * p.S * 3 * DD;
    // operands: j = 0: A[k][r] = G[k][r] (= G[r][k]: G = K^T K from exact bf16 products is
    // symmetric), B = W0;  j = 1: A[k][r] = W0[r][k], B[k][c] = M[c][k];  j = 2: A = G, B = M
    {
        float4 a[4], b[4];
        if (j == 1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = __ldg(reinterpret_cast<const float4*>(W0) + tid + 256 * i);
        } else {
            f_load_sum(part, p.S, 0, tid, a);
        }
        if (j == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) b[i] = __ldg(reinterpret_cast<const float4*>(W0) + tid + 256 * i);
        } else {
            f_load_sum(part, p.S, 2, tid, b);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f_put4(Aop, tid + 256 * i, a[i], j == 1);
            f_put4(Bop, tid + 256 * i, b[i], j == 1);
        }
    }
    __syncthreads();
    const int tr = tid >> 4, tc = tid & 15;  // rows 4 tr .. 4 tr + 3, columns 4 tc .. 4 tc + 3
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][q] = 0.f;
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
        const float4 av = *reinterpret_cast<const float4*>(Aop + k * FLD + 4 * tr);
        const float4 bv = *reinterpret_cast<const float4*>(Bop + k * FLD + 4 * tc);
        const float ax[4] = {av.x, av.y, av.z, av.w}, bx[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[i][q] = fmaf(ax[i], bx[q], acc[i][q]);
    }
    const float en = p.eta_over_n;
    __nv_bfloat16* ops = p.ops + (size_t)u * 8 * DD;
    const int c0 = 4 * tc;
    if (j == 0) {
        // C[r][c] = C^T[c][r]: for each column c, rows 4 tr .. 4 tr + 3 are one float4 of C^T
        float4 cs[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) cs[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < p.S; ++s) {
            float4 v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                v[q] = __ldg(reinterpret_cast<const float4*>(part + ((size_t)s * 3 + 1) * DD + (c0 + q) * D + 4 * tr));
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                cs[q].x += v[q].x;
                cs[q].y += v[q].y;
                cs[q].z += v[q].z;
                cs[q].w += v[q].w;
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * tr + i;
            float w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float c = i == 0 ? cs[q].x : i == 1 ? cs[q].y : i == 2 ? cs[q].z : cs[q].w;
                w[q] = Bop[r * FLD + c0 + q] - en * (acc[i][q] - c);
            }
            put_hilo4(ops, OP_WS_HI, OP_WS_LO, r, c0, w);
        }
    } else if (j == 1) {
        // A = P + P^T: the product goes through shared memory (over A's operand, now read)
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4*>(Aop + (4 * tr + i) * FLD + c0) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * tr + i;
            float a[4], mt[4], m[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int c = c0 + q;
                a[q] = -en * (acc[i][q] + Aop[c * FLD + r]);
                mt[q] = en * Bop[r * FLD + c];  // (eta/N) M[c][r]
                m[q] = en * Bop[c * FLD + r];   // (eta/N) M[r][c]
            }
            put_hilo4(ops, OP_A_HI, OP_A_LO, r, c0, a);
            put_hilo4(ops, OP_MT_HI, OP_MT_LO, r, c0, mt);
            put_hilo4(ops, OP_M_HI, OP_M_LO, r, c0, m);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * tr + i;
            float4 o;
            o.x = Bop[r * FLD + c0] - en * acc[i][0];
            o.y = Bop[r * FLD + c0 + 1] - en * acc[i][1];
            o.z = Bop[r * FLD + c0 + 2] - en * acc[i][2];
            o.w = Bop[r * FLD + c0 + 3] - en * acc[i][3];
            *reinterpret_cast<float4*>(p.dw0u + (size_t)u * DD + r * D + c0) = o;
        }
    }
}

// ----------------------------------------------------------------------------- apply -----
constexpr int A_STAGES = 3;
constexpr int A_STAGE = 3 * TILE;         // dO, K, V (dQ, dK, dV are written over them)
constexpr int OPS = 8 * OP;               // the eight right-hand operands, 64 KB
constexpr int A_EPI_WARPS = 8;
constexpr int A_THREADS = 64 + 32 * A_EPI_WARPS;

struct AParams {
    int TT, n_tiles;
};
struct ABars {
    uint64_t opfull, full[A_STAGES], empty[A_STAGES], tfull[2], tempty[2];
    uint32_t tmem_base;
};
constexpr int a_smem_bytes() { return OPS + A_STAGES * A_STAGE + (int)sizeof(ABars) + 1024; }

__device__ __forceinline__ void group_sync(int g) { asm volatile("bar.sync %0, 128;" ::"r"(2 + g) : "memory"); }

__global__ void __launch_bounds__(A_THREADS, 1)
    apply_kernel(const __grid_constant__ CUtensorMap tm_ops, const __grid_constant__ CUtensorMap tm_g,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dk,
                 const __grid_constant__ CUtensorMap tm_dv, const AParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ops = smem_align<1024>(smem_raw);
    uint8_t* ring = ops + OPS;
    ABars* bars = reinterpret_cast<ABars*>(ring + A_STAGES * A_STAGE);
    const int S = gridDim.x, r = blockIdx.x, u = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int TT = p.TT;
    const int n_t = r < p.n_tiles ? (p.n_tiles - r + S - 1) / S : 0;
    // the first dO, K, V tiles (inputs of the call) into L2 before waiting for the finish grid
    if (threadIdx.x == 0)
        for (int i = 0; i < min(A_STAGES, n_t); ++i) {
            const int row = (r + i * S) * TT;
            tma_prefetch_l2_3d(&tm_g, 0, row, u);
            tma_prefetch_l2_3d(&tm_k, 0, row, u);
            tma_prefetch_l2_3d(&tm_v, 0, row, u);
        }
    griddep_wait();
    griddep_launch();
    if (threadIdx.x == 0) {
        mbar_init(&bars->opfull, 1);
        for (int s = 0; s < A_STAGES; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->tfull[b], 1);
            mbar_init(&bars->tempty[b], A_EPI_WARPS / 2);
        }
        mbar_fence_init();
    }
    if (warp == 1) tc::alloc(&bars->tmem_base, 512);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_ops);
            tma_prefetch_desc(&tm_g);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_expect_tx(&bars->opfull, OPS);
            for (int m = 0; m < 8; ++m) tma_load_3d(ops + m * OP, &tm_ops, 0, m * D, u, &bars->opfull);
            for (int i = 0; i < n_t; ++i) {
                const int slot = i % A_STAGES, use = i / A_STAGES;
                if (use > 0) mbar_wait(&bars->empty[slot], (use - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                uint8_t* dst = ring + slot * A_STAGE;
                const int row = (r + i * S) * TT;
                mbar_expect_tx(&bars->full[slot], 3 * TT * ROWB);
                tma_load_3d(dst, &tm_g, 0, row, u, &bars->full[slot]);
                tma_load_3d(dst + TILE, &tm_k, 0, row, u, &bars->full[slot]);
                tma_load_3d(dst + 2 * TILE, &tm_v, 0, row, u, &bars->full[slot]);
                if (i == A_STAGES - 1)
                    for (int j = A_STAGES; j < n_t; ++j) {
                        const int rj = (r + j * S) * TT;
                        tma_prefetch_l2_3d(&tm_g, 0, rj, u);
                        tma_prefetch_l2_3d(&tm_k, 0, rj, u);
                        tma_prefetch_l2_3d(&tm_v, 0, rj, u);
                    }
            }
            mbar_wait(&bars->opfull, 0, TTT_DEVERR_TIMEOUT_TMA);  // no load in flight at exit
        }
    } else if (warp == 1) {
        if (lane == 0 && n_t > 0) {
            mbar_wait(&bars->opfull, 0, TTT_DEVERR_TIMEOUT_TMA);
            const uint32_t ob = smem_u32(ops);
            uint64_t od[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) od[m] = tc::smem_desc(ob + m * OP, 16, 1024, 2);
            for (int t = 0; t < n_t; ++t) {
                const int b = t & 1, slot = t % A_STAGES;
                if (t >= 2) mbar_wait(&bars->tempty[b], ((t >> 1) - 1) & 1, TTT_DEVERR_TIMEOUT_PEER);
                mbar_wait(&bars->full[slot], (t / A_STAGES) & 1, TTT_DEVERR_TIMEOUT_TMA);
                tc::fence_after();
                const uint32_t sb = smem_u32(ring + slot * A_STAGE);
                const uint64_t dg = tc::smem_desc(sb, 16, 1024, 2);
                const uint64_t dk = tc::smem_desc(sb + TILE, 16, 1024, 2);
                const uint64_t dv = tc::smem_desc(sb + 2 * TILE, 16, 1024, 2);
                const uint32_t acc0 = tmem + b * 256;
                // dQ (columns 0-63), then [dV | dK] (64-191) = K [M^T-op | A-op] as one N = 128
                // product, then dK += V M-op; each right operand as hi + lo
#pragma unroll
                for (int hl = 0; hl < 2; ++hl)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const int acc = (hl > 0 || ks > 0) ? 1 : 0;
                        tc::mma_bf16(acc0, dg + 2 * ks, od[hl ? OP_WS_LO : OP_WS_HI] + 2 * ks, IDESC_N64, acc);
                        tc::mma_bf16(acc0 + 64, dk + 2 * ks, od[hl ? OP_MT_LO : OP_MT_HI] + 2 * ks, IDESC_N128, acc);
                    }
#pragma unroll
                for (int hl = 0; hl < 2; ++hl)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        tc::mma_bf16(acc0 + 128, dv + 2 * ks, od[hl ? OP_M_LO : OP_M_HI] + 2 * ks, IDESC_N64, 1);
                tc::commit(&bars->tfull[b]);
            }
        }
    } else {
        const int q4 = warp & 3;
        const int grp = (warp - 2) >> 2;  // tile group: tiles grp, grp + 2, ...
        const int row = q4 * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
        const bool storer = (q4 == 0 && lane == 0);
        for (int t = grp; t < n_t; t += 2) {
            const int b = t & 1, slot = t % A_STAGES;
            uint8_t* st = ring + slot * A_STAGE;
            mbar_wait(&bars->tfull[b], (t >> 1) & 1, TTT_DEVERR_TIMEOUT_PEER);
            tc::fence_after();
            // accumulator j -> tile: dQ over dO (tile 0), dV over V (tile 2), dK over K (tile 1)
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                uint8_t* tile = st + (j == 0 ? 0 : j == 1 ? 2 * TILE : TILE);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float o[32];
                    tc::ld16(lane_base + b * 256 + j * 64 + half * 32, &o[0]);
                    tc::ld16(lane_base + b * 256 + j * 64 + half * 32 + 16, &o[16]);
                    tc::wait_ld();
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *reinterpret_cast<uint4*>(tile + swz<3>((uint32_t)row * ROWB + half * 64 + c * 16)) =
                            make_uint4(pack_bf16(o[8 * c], o[8 * c + 1]), pack_bf16(o[8 * c + 2], o[8 * c + 3]),
                                       pack_bf16(o[8 * c + 4], o[8 * c + 5]), pack_bf16(o[8 * c + 6], o[8 * c + 7]));
                }
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->tempty[b]);
            fence_proxy_async_smem();
            group_sync(grp);  // all 128 rows of the three output tiles are written
            if (storer) {
                const int grow = (r + t * S) * TT;  // rows >= N are clipped
                tma_store_3d(&tm_dq, 0, grow, u, st);
                tma_store_3d(&tm_dk, 0, grow, u, st + TILE);
                tma_store_3d(&tm_dv, 0, grow, u, st + 2 * TILE);
                tma_store_commit();
                tma_store_wait_read_all();  // the stage may be refilled
                mbar_arrive(&bars->empty[slot]);
            }
        }
        if (storer) tma_store_wait_all();
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) tc::dealloc(tmem, 512);
}

}  // namespace lbw

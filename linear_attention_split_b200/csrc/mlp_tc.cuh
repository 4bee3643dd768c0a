// mlp_tc.cuh -- TTT-MLP full-batch step on the tcgen05 tensor cores, bf16, d = 64, h = 256.
//
// Operation (TTT abstract of Sun et al.: hidden state a two-layer MLP; layer and recipe of
// the ViT^3 blog: one full-batch gradient step of (1/N) sum 1/2 ||F(k) - v||^2, gradient
// derived by hand), per unit u = (b, head) with F(x) = gelu_tanh(x W1) W2:
//     Z = K W1,  A = gelu(Z),  P = A W2,  R = P - V
//     gW2 = A^T R,  dA = R W2^T,  dZ = dA * gelu'(Z),  gW1 = K^T dZ
//     W1* = W1 - (eta/N) gW1,  W2* = W2 - (eta/N) gW2,   O = gelu(Q W1*) W2*
// Three kernels:
//   grad   : CTAs split each unit's tokens; per 128-token tile five tcgen05 MMAs (operands in
//            shared memory, fp32 accumulators in TMEM).  gW1^T and gW2 (256 x 64 each) stay
//            resident in TMEM for the whole token range; the other 256 TMEM columns hold Z,
//            then P, then dA.  Eight epilogue warps turn Z into A and gelu'(Z), P into R, and
//            dA into dZ.  The K tile and the R tile alternate between two buffers so the next
//            K tile loads while the current tile's backward runs.  Each CTA writes its
//            partial gradients (fp32) to the workspace.
//   update : sums the partials of a unit in split order (deterministic) and forms W1*, W2*
//            (fp32 outputs if requested; for the apply pass W1* as bf16 hi + lo, W2* as fp16).
//   apply  : per 128-token tile Z = Q W1*_hi + Q W1*_lo, A = gelu(Z) rounded to fp16,
//            O = A W2* (fp16 x fp16, fp32 accumulate), stored as bf16 by TMA.  W1* is kept to
//            2^-17 and A, W2* to 2^-11, so that O stays within a few tenths of a percent of the
//            RMS of its exact value beyond the final bf16 rounding.
// gelu uses the tanh form with the hardware tanh approximation (tanh.approx.f32).
#pragma once
#include "common.cuh"

namespace mlp {

constexpr int D = 64, HID = 256, MT = 128;
constexpr int ROWB = 128;                       // bytes per 64-element bf16 row
constexpr int TILE = MT * ROWB;                 // 16 KB: 128 tokens x 64 features
constexpr int BIG = MT * HID * 2;               // 64 KB: 128 tokens x 256 hidden
constexpr int WBYTES = D * HID * 2;             // 32 KB: one bf16 weight matrix
constexpr int EPI_WARPS = 8;
constexpr int THREADS = (2 + EPI_WARPS) * 32;   // producer, issuer, epilogue
constexpr uint32_t COL_T = 0, COL_G2 = 256, COL_G1 = 384;

// shared-memory layouts (all 128-byte swizzled, 1024-byte atoms)
//  W1 [d][h]  : MN-major B of Z = K W1:   (k, n) -> (n/64)*8192 + (k/8)*1024 + swz((k%8)*128 + (n%64)*2)
//  W2 [h][d]  : MN-major B of P = A W2 and K-major B of dA = R W2^T: (h, d) -> (h/8)*1024 + swz((h%8)*128 + d*2)
//  A / gp / dZ [token][h]: K-major A (rows = tokens) and MN-major A^T: (t, c) -> (c/64)*16384 + swz(t*128 + (c%64)*2)
//  K / R [token][d] : (t, d) -> swz(t*128 + d*2)
__device__ __forceinline__ uint32_t w1_off(int k, int n) {
    return (n >> 6) * 8192 + (k >> 3) * 1024 + swz<3>((k & 7) * 128 + (n & 63) * 2);
}
__device__ __forceinline__ uint32_t w2_off(int h, int d) { return (h >> 3) * 1024 + swz<3>((h & 7) * 128 + d * 2); }
__device__ __forceinline__ uint32_t big_off(int t, int c) { return (c >> 6) * 16384 + swz<3>(t * 128 + (c & 63) * 2); }

__device__ __forceinline__ float tanh_fast(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Packed fp32 pairs (one instruction for two lanes' worth of math: fma/mul/add.rn.f32x2).
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
    return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ float lo2(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi2(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t tanh2(uint64_t x) { return pk2(tanh_fast(lo2(x)), tanh_fast(hi2(x))); }

// gelu_tanh(u) = u/2 (1 + t), t = tanh(u s (1 + a u^2)), s = sqrt(2/pi), a = 0.044715, and its
// derivative gelu'(u) = (1 + t)/2 + u/2 (1 - t^2) s (1 + 3 a u^2), for a pair of u:
// ten packed operations and two hardware tanh per pair.
__device__ __forceinline__ uint64_t gelu_gp2(uint64_t u, uint64_t* gp) {
    const float s = 0.7978845608028654f, a = 0.044715f;
    const uint64_t half = pk2(0.5f, 0.5f);
    const uint64_t u2 = mul2(u, u);
    const uint64_t t = tanh2(mul2(u, fma2(pk2(a * s, a * s), u2, pk2(s, s))));      // tanh(u s (1 + a u^2))
    const uint64_t hu = mul2(u, half);
    const uint64_t omt = fma2(t ^ 0x8000000080000000ull, t, pk2(1.f, 1.f));         // 1 - t^2
    const uint64_t p = fma2(pk2(3.f * a * s, 3.f * a * s), u2, pk2(s, s));          // s (1 + 3 a u^2)
    *gp = fma2(mul2(hu, omt), p, fma2(half, t, half));
    return fma2(hu, t, hu);
}
__device__ __forceinline__ uint64_t gelu2(uint64_t u) {
    const float s = 0.7978845608028654f, a = 0.044715f;
    const uint64_t hu = mul2(u, pk2(0.5f, 0.5f));
    const uint64_t t = tanh2(mul2(u, fma2(pk2(a * s, a * s), mul2(u, u), pk2(s, s))));
    return fma2(hu, t, hu);
}
__device__ __forceinline__ uint32_t pack2_bf16(uint64_t v) { return pack_bf16(lo2(v), hi2(v)); }
__device__ __forceinline__ void ld32(uint32_t taddr, float* v) {
    tc::ld16(taddr, v);
    tc::ld16(taddr + 16, v + 16);
}
__device__ __forceinline__ void store8_bf16(uint8_t* base, uint32_t off, const float* v) {
    *reinterpret_cast<uint4*>(base + off) = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                                                       pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
}

// ----------------------------------------------------------------------------- grad ----
struct GradParams {
    const __nv_bfloat16* v; // [U][N][64]
    float* part;            // [U][S][2][256][64]: gW1^T then gW2 (chunk-swizzled rows, see below)
    int H, N, T;            // T = tokens per CTA (multiple of 128)
};

struct GradBars {
    uint64_t wfull, kfull[2], bfree[2], z0full, z1full, a0ready, a1ready, pfull, rready, da0full, da1full,
        dz0ready, dz1ready, gdone;
    uint32_t tmem_base;
};

// W1 [H][64][256] and W2 [H][256][64], fp32 -> bf16 (row-major), once per call, so that every
// CTA can bring its head's weights into shared memory with five TMA loads.
__global__ void __launch_bounds__(256) prep_kernel(const float* w1, const float* w2, __nv_bfloat16* w1h,
                                                   __nv_bfloat16* w2h, int n8) {
    for (int e = blockIdx.x * 256 + threadIdx.x; e < n8; e += gridDim.x * 256) {
        const float* src = e < n8 / 2 ? w1 + (size_t)e * 8 : w2 + (size_t)(e - n8 / 2) * 8;
        __nv_bfloat16* dst = e < n8 / 2 ? w1h + (size_t)e * 8 : w2h + (size_t)(e - n8 / 2) * 8;
        const float4 a = *reinterpret_cast<const float4*>(src);
        const float4 b = *reinterpret_cast<const float4*>(src + 4);
        *reinterpret_cast<uint4*>(dst) =
            make_uint4(pack_bf16(a.x, a.y), pack_bf16(a.z, a.w), pack_bf16(b.x, b.y), pack_bf16(b.z, b.w));
    }
}

// W1 (bf16 [idx][64][256]) as four 64 x 64 boxes -> the MN-major w1_off layout, W2 (bf16
// [idx][256][64]) as one 256 x 64 box -> the w2_off layout; 128-byte swizzle, 64 KB on `bar`.
__device__ __forceinline__ void tma_load_weights(uint8_t* w1s, uint8_t* w2s, const CUtensorMap* tw1,
                                                 const CUtensorMap* tw2, int idx, uint64_t* bar) {
    mbar_expect_tx(bar, 2 * WBYTES);
#pragma unroll
    for (int a = 0; a < HID / 64; ++a) tma_load_3d(w1s + a * 8192, tw1, a * 64, 0, idx, bar);
    tma_load_3d(w2s, tw2, 0, 0, idx, bar);
}

__global__ void __launch_bounds__(THREADS, 1)
    grad_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_w1,
                const __grid_constant__ CUtensorMap tm_w2, const GradParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align<1024>(smem_raw);
    uint8_t* w1s = smem;                 // 32 KB
    uint8_t* w2s = w1s + WBYTES;         // 32 KB
    uint8_t* at = w2s + WBYTES;          // 64 KB  A = gelu(Z)
    uint8_t* gt = at + BIG;              // 64 KB  gelu'(Z), then dZ
    uint8_t* buf = gt + BIG;             // 2 x 16 KB: K and R alternate
    GradBars* bars = reinterpret_cast<GradBars*>(buf + 2 * TILE);

    const int split = blockIdx.x, S = gridDim.x, u = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = split * p.T;
    const int n_valid = max(0, min(p.N - t0, p.T));
    const int ntiles = (n_valid + MT - 1) / MT;
    const int hd = u % p.H;

    if (threadIdx.x == 0) {
        mbar_init(&bars->wfull, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->kfull[b], 1);
            mbar_init(&bars->bfree[b], 1);
        }
        mbar_init(&bars->z0full, 1);
        mbar_init(&bars->z1full, 1);
        mbar_init(&bars->a0ready, EPI_WARPS);
        mbar_init(&bars->a1ready, EPI_WARPS);
        mbar_init(&bars->pfull, 1);
        mbar_init(&bars->rready, EPI_WARPS);
        mbar_init(&bars->da0full, 1);
        mbar_init(&bars->da1full, 1);
        mbar_init(&bars->dz0ready, EPI_WARPS);
        mbar_init(&bars->dz1ready, EPI_WARPS);
        mbar_init(&bars->gdone, 1);
        mbar_fence_init();
    }
    if (warp == 1) tc::alloc(&bars->tmem_base, 512);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ================================ producer: K tiles ============================
        // tile i's K lives in buf[i & 1]; that buffer last held tile i-1's R, freed once the
        // MMAs reading R (gW2, dA) of tile i-1 completed (bfree)
        if (lane == 0) {
            tma_load_weights(w1s, w2s, &tm_w1, &tm_w2, hd, &bars->wfull);
            for (int i = 0; i < ntiles; ++i) {
                const int b = i & 1;
                if (i >= 1) mbar_wait(&bars->bfree[b], ((i - 1) >> 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                mbar_expect_tx(&bars->kfull[b], TILE);
                tma_load_3d(buf + b * TILE, &tm_k, 0, t0 + i * MT, u, &bars->kfull[b]);
            }
            mbar_wait(&bars->wfull, 0, TTT_DEVERR_TIMEOUT_TMA);  // no load in flight at exit
        }
    } else if (warp == 1) {
        // ================================ MMA issuer ===================================
        // The 256 TMEM columns for Z / P / dA are two halves, T0 (hidden units 0-127, and P in
        // its first 64 columns) and T1 (hidden units 128-255), so that the epilogue works on
        // one half while the tensor cores fill the other.  Order per tile i:
        //   P = A0 W2[0:128] (after a0ready), P += A1 W2[128:256] (after a1ready) -> pfull
        //   dA0 = R W2[0:128]^T -> T0, dA1 = R W2[128:256]^T -> T1, then gW2 += A^T R (after rready)
        //   gW1[0:128] += dZ0^T K (after dz0ready), then Z0 of tile i+1 -> T0,
        //   gW1[128:256] += dZ1^T K (after dz1ready), then Z1 of tile i+1 -> T1.
        // The tensor pipe runs MMAs in issue order, so a commit also covers every earlier MMA.
        if (lane == 0 && ntiles > 0) {
            const uint32_t w1a = smem_u32(w1s), w2a = smem_u32(w2s), aa = smem_u32(at), ga = smem_u32(gt);
            const uint32_t IZ = tc::idesc_bf16(128, 128, 0, 1);   // K (K-major) x W1 half (MN-major)
            const uint32_t IP = tc::idesc_bf16(128, 64, 0, 1);    // A (K-major) x W2 (MN-major)
            const uint32_t IG = tc::idesc_bf16(128, 64, 1, 1);    // A^T/dZ^T (MN-major) x R/K (MN-major)
            const uint32_t ID = tc::idesc_bf16(128, 128, 0, 0);   // R (K-major) x W2^T half (K-major)
            auto issue_z = [&](int i, int half) {  // Z half of tile i: K W1[:, 128 half ..]
                const uint32_t kb = smem_u32(buf + (i & 1) * TILE);
                tc::fence_after();
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tmem + COL_T + half * 128, tc::smem_desc(kb + ks * 32, 16, 1024, 2),
                                 tc::smem_desc(w1a + half * 2 * 8192 + ks * 2048, 8192, 1024, 2), IZ, ks > 0);
                tc::commit(half ? &bars->z1full : &bars->z0full);
            };
            mbar_wait(&bars->wfull, 0, TTT_DEVERR_TIMEOUT_TMA);
            mbar_wait(&bars->kfull[0], 0, TTT_DEVERR_TIMEOUT_TMA);
            issue_z(0, 0);
            issue_z(0, 1);
            for (int i = 0; i < ntiles; ++i) {
                const int b = i & 1;
                const uint32_t kb = smem_u32(buf + b * TILE), rb = smem_u32(buf + (b ^ 1) * TILE);
                const uint32_t ph = i & 1;
                // P = A W2 in two K halves (T0 columns 0..63)
                for (int half = 0; half < 2; ++half) {
                    mbar_wait(half ? &bars->a1ready : &bars->a0ready, ph, TTT_DEVERR_TIMEOUT_PEER);
                    tc::fence_after();
                    for (int ks = half * 8; ks < half * 8 + 8; ++ks)
                        tc::mma_bf16(tmem + COL_T,
                                     tc::smem_desc(aa + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, 2),
                                     tc::smem_desc(w2a + ks * 2048, 8192, 1024, 2), IP, ks > 0);
                }
                tc::commit(&bars->pfull);
                // gW2 += A^T R (two 128-row halves of h); dA0 -> T0, dA1 -> T1
                mbar_wait(&bars->rready, ph, TTT_DEVERR_TIMEOUT_PEER);
                tc::fence_after();
                for (int half = 0; half < 2; ++half) {  // dA first: the epilogue waits for it
                    for (int ks = 0; ks < 4; ++ks)
                        tc::mma_bf16(tmem + COL_T + half * 128, tc::smem_desc(rb + ks * 32, 16, 1024, 2),
                                     tc::smem_desc(w2a + half * 16384 + ks * 32, 16, 1024, 2), ID, ks > 0);
                    tc::commit(half ? &bars->da1full : &bars->da0full);
                }
                for (int hh = 0; hh < 2; ++hh)
                    for (int ks = 0; ks < 8; ++ks)
                        tc::mma_bf16(tmem + COL_G2 + hh * 64,
                                     tc::smem_desc(aa + hh * 2 * 16384 + ks * 2048, 16384, 1024, 2),
                                     tc::smem_desc(rb + ks * 2048, 8192, 1024, 2), IG, (i > 0 || ks > 0));
                tc::commit(&bars->bfree[b ^ 1]);  // R buffer free once these MMAs completed
                // gW1^T += dZ^T K per half of h; the freed T half takes the next tile's Z half
                for (int hh = 0; hh < 2; ++hh) {
                    mbar_wait(hh ? &bars->dz1ready : &bars->dz0ready, ph, TTT_DEVERR_TIMEOUT_PEER);
                    tc::fence_after();
                    for (int ks = 0; ks < 8; ++ks)
                        tc::mma_bf16(tmem + COL_G1 + hh * 64,
                                     tc::smem_desc(ga + hh * 2 * 16384 + ks * 2048, 16384, 1024, 2),
                                     tc::smem_desc(kb + ks * 2048, 8192, 1024, 2), IG, (i > 0 || ks > 0));
                    if (i + 1 < ntiles) {
                        if (hh == 0) mbar_wait(&bars->kfull[b ^ 1], ((i + 1) >> 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                        issue_z(i + 1, hh);
                    }
                }
            }
            tc::commit(&bars->gdone);
        }
    } else {
        // ================================ epilogue (8 warps) ===========================
        // the epilogue's waits leave out the suspend-time hint (the tile's chain runs through
        // them; 0.425 -> 0.417 ms per call with the apply kernel's likewise), the issuer's keep it
        const int q4 = warp & 3;                 // TMEM lane quarter
        const int ch = (warp - 2) >> 2;          // column half handled by this warp
        const int r = q4 * 32 + lane;            // token row of the tile
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
        const __nv_bfloat16* vu = p.v + (size_t)u * p.N * D;
        for (int i = 0; i < ntiles; ++i) {
            const int b = i & 1;
            const uint32_t ph = i & 1;
            uint8_t* rbuf = buf + (b ^ 1) * TILE;
            const int tok = t0 + i * MT + r;
            // V row (32 columns of this half) fetched early
            uint4 vv[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                vv[c] = tok < p.N ? *reinterpret_cast<const uint4*>(vu + (size_t)tok * D + ch * 32 + c * 8)
                                  : make_uint4(0, 0, 0, 0);
            // ---- Z half -> A = gelu(Z), gelu'(Z), hidden units [128 half, 128 half + 128) -----
            // this warp: 64 of those columns (ch), lanes = its 32 token rows
            for (int half = 0; half < 2; ++half) {
                mbar_wait<false>(half ? &bars->z1full : &bars->z0full, ph, TTT_DEVERR_TIMEOUT_PEER);
                tc::fence_after();
                {
                    const int c0 = half * 128 + ch * 64;  // 64 columns, one TMEM round trip
                    float z[64];
                    ld32(lane_base + COL_T + c0, z);
                    ld32(lane_base + COL_T + c0 + 32, z + 32);
                    tc::wait_ld();
#pragma unroll
                    for (int j = 0; j < 64; j += 8) {
                        uint32_t a[4], g[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            uint64_t gp;
                            a[e] = pack2_bf16(gelu_gp2(pk2(z[j + 2 * e], z[j + 2 * e + 1]), &gp));
                            g[e] = pack2_bf16(gp);
                        }
                        *reinterpret_cast<uint4*>(at + big_off(r, c0 + j)) = make_uint4(a[0], a[1], a[2], a[3]);
                        *reinterpret_cast<uint4*>(gt + big_off(r, c0 + j)) = make_uint4(g[0], g[1], g[2], g[3]);
                    }
                }
                fence_proxy_async_smem();
                tc::fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(half ? &bars->a1ready : &bars->a0ready);
            }
            // ---- P -> R = P - V ---------------------------------------------------------------
            mbar_wait<false>(&bars->pfull, ph, TTT_DEVERR_TIMEOUT_PEER);
            tc::fence_after();
            {
                float pv[32];
                ld32(lane_base + COL_T + ch * 32, pv);
                tc::wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t w[4] = {vv[c].x, vv[c].y, vv[c].z, vv[c].w};
                    float rr[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        rr[2 * j] = pv[c * 8 + 2 * j] - __uint_as_float(w[j] << 16);
                        rr[2 * j + 1] = pv[c * 8 + 2 * j + 1] - __uint_as_float(w[j] & 0xffff0000u);
                    }
                    if (tok >= p.N)
#pragma unroll
                        for (int j = 0; j < 8; ++j) rr[j] = 0.f;
                    store8_bf16(rbuf, swz<3>(r * ROWB + (ch * 32 + c * 8) * 2), rr);
                }
            }
            fence_proxy_async_smem();
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->rready);
            // ---- dA half -> dZ = dA * gelu'(Z), in place over gelu'(Z) ---------------------------
            for (int half = 0; half < 2; ++half) {
                mbar_wait<false>(half ? &bars->da1full : &bars->da0full, ph, TTT_DEVERR_TIMEOUT_PEER);
                tc::fence_after();
                {
                    const int c0 = half * 128 + ch * 64;  // 64 columns, one TMEM round trip
                    float da[64];
                    ld32(lane_base + COL_T + c0, da);
                    ld32(lane_base + COL_T + c0 + 32, da + 32);
                    tc::wait_ld();
#pragma unroll
                    for (int j = 0; j < 64; j += 8) {
                        const uint32_t off = big_off(r, c0 + j);
                        const uint4 gq = *reinterpret_cast<const uint4*>(gt + off);
                        const uint32_t w[4] = {gq.x, gq.y, gq.z, gq.w};
                        float dz[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            dz[2 * e] = da[j + 2 * e] * __uint_as_float(w[e] << 16);
                            dz[2 * e + 1] = da[j + 2 * e + 1] * __uint_as_float(w[e] & 0xffff0000u);
                        }
                        store8_bf16(gt, off, dz);
                    }
                }
                fence_proxy_async_smem();
                tc::fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(half ? &bars->dz1ready : &bars->dz0ready);
            }
        }
        // ---- partial gradients: TMEM -> workspace --------------------------------------------
        float* part = p.part + ((size_t)u * S + split) * 2 * HID * D;
        if (ntiles > 0) {
            mbar_wait<false>(&bars->gdone, 0, TTT_DEVERR_TIMEOUT_PEER);
            tc::fence_after();
        }
        // TMEM lane = h row within a 128-row half; this warp: half ch, rows q4*32 + lane.
        // Both gradients are staged in the (now idle) A and gelu' buffers, 64 KB each, and
        // leave with one bulk copy apiece.  Row h keeps its 16 float4 chunks at positions
        // c ^ (h & 7) (the workspace layout; the update kernel reads it back the same way), so
        // that the 32 rows a warp writes spread over all banks.
        const int hrow = ch * 128 + r;
        for (int which = 0; which < 2; ++which) {  // 0: gW1^T -> at, 1: gW2 -> gt
            const uint32_t col = (which == 0 ? COL_G1 : COL_G2) + ch * 64;
            float* srow = reinterpret_cast<float*>(which == 0 ? at : gt) + (size_t)hrow * D;
            float g[64];
            if (ntiles > 0) {
                ld32(lane_base + col, g);
                ld32(lane_base + col + 32, g + 32);
                tc::wait_ld();
            } else {
#pragma unroll
                for (int j = 0; j < 64; ++j) g[j] = 0.f;
            }
#pragma unroll
            for (int c = 0; c < 16; ++c)
                *reinterpret_cast<float4*>(srow + 4 * (c ^ (hrow & 7))) =
                    make_float4(g[4 * c], g[4 * c + 1], g[4 * c + 2], g[4 * c + 3]);
        }
        fence_proxy_async_smem();  // read next by the bulk copies
        asm volatile("bar.sync 1, %0;" ::"r"(EPI_WARPS * 32) : "memory");
        if (warp == 2 && lane == 0) {
            asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(part),
                         "r"(smem_u32(at)), "r"(HID * D * 4)
                         : "memory");
            asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(part + HID * D),
                         "r"(smem_u32(gt)), "r"(HID * D * 4)
                         : "memory");
            tma_store_commit();
            tma_store_wait_all();
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) tc::dealloc(tmem, 512);
}

// ----------------------------------------------------------------------------- update --
struct UpdateParams {
    const float* w1;            // [H][64][256]
    const float* w2;            // [H][256][64]
    const float* part;          // [U][S][2][256][64]
    float* w1_star;             // [U][64][256] fp32 or nullptr
    float* w2_star;             // [U][256][64] fp32 or nullptr
    __nv_bfloat16* w1b;         // [U][2][64][256] bf16: W1* hi, then lo = W1* - hi
    __half* w2h;                // [U][256][64] fp16
    int H, S;
    float eta_over_n;
};

// Block (u, c): rows h in [64 c, 64 c + 64) of gW1^T and gW2.  The S partials are added in
// split order (deterministic).  W2*[h][d] is written row by row; W1*[d][h] is the transpose of
// the gW1^T block, so that block goes through shared memory and leaves row by row as well.
// Each thread takes four consecutive columns (one float4 chunk of the swizzled partials), so
// every load is 16 bytes and every store 8 or 16.
__global__ void __launch_bounds__(256) update_kernel(const UpdateParams p) {
    __shared__ float tile[64][65];  // W1*^T block: [h - h0][d]
    const int u = blockIdx.x, hd = u % p.H, h0 = blockIdx.y * 64;
    const float* part = p.part + (size_t)u * p.S * 2 * HID * D;
    const int c = threadIdx.x & 15, ty = threadIdx.x >> 4;  // 16 chunks of 4 columns x 16 rows per pass
    for (int rr = ty; rr < 64; rr += 16) {
        const int h = h0 + rr;
        // columns d = 4 c .. 4 c + 3 of row h: float4 chunk c ^ (h & 7) of that row in a partial
        const int pe = h * D + ((c ^ (h & 7)) << 2);
        float g1[4] = {0.f, 0.f, 0.f, 0.f}, g2[4] = {0.f, 0.f, 0.f, 0.f};
        for (int sp = 0; sp < p.S; ++sp) {  // split order
            const float4 a = *reinterpret_cast<const float4*>(part + (size_t)sp * 2 * HID * D + pe);
            const float4 b = *reinterpret_cast<const float4*>(part + (size_t)sp * 2 * HID * D + HID * D + pe);
            g1[0] += a.x;
            g1[1] += a.y;
            g1[2] += a.z;
            g1[3] += a.w;
            g2[0] += b.x;
            g2[1] += b.y;
            g2[2] += b.z;
            g2[3] += b.w;
        }
        const size_t o2 = (size_t)h * D + 4 * c;
        const float4 w2o = *reinterpret_cast<const float4*>(p.w2 + (size_t)hd * HID * D + o2);
        const float w2[4] = {w2o.x - p.eta_over_n * g2[0], w2o.y - p.eta_over_n * g2[1],
                             w2o.z - p.eta_over_n * g2[2], w2o.w - p.eta_over_n * g2[3]};  // W2*[h][d]
        if (p.w2_star)
            *reinterpret_cast<float4*>(p.w2_star + (size_t)u * HID * D + o2) = make_float4(w2[0], w2[1], w2[2], w2[3]);
        const __half2 f01 = __floats2half2_rn(w2[0], w2[1]), f23 = __floats2half2_rn(w2[2], w2[3]);
        *reinterpret_cast<uint2*>(p.w2h + (size_t)u * HID * D + o2) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&f01), *reinterpret_cast<const uint32_t*>(&f23));
#pragma unroll
        for (int i = 0; i < 4; ++i) tile[rr][4 * c + i] = g1[i];  // gW1^T[h][d]
    }
    __syncthreads();
    for (int dd = ty; dd < 64; dd += 16) {  // W1*[d][h0 + 4 c .. h0 + 4 c + 3]
        const size_t idx = (size_t)dd * HID + h0 + 4 * c;
        const float4 w1o = *reinterpret_cast<const float4*>(p.w1 + (size_t)hd * D * HID + idx);
        const float w1[4] = {w1o.x - p.eta_over_n * tile[4 * c][dd], w1o.y - p.eta_over_n * tile[4 * c + 1][dd],
                             w1o.z - p.eta_over_n * tile[4 * c + 2][dd], w1o.w - p.eta_over_n * tile[4 * c + 3][dd]};
        if (p.w1_star)
            *reinterpret_cast<float4*>(p.w1_star + (size_t)u * D * HID + idx) = make_float4(w1[0], w1[1], w1[2], w1[3]);
        uint32_t hi[2], lo[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const __nv_bfloat16 h0b = __float2bfloat16_rn(w1[2 * j]), h1b = __float2bfloat16_rn(w1[2 * j + 1]);
            const __nv_bfloat16 l0b = __float2bfloat16_rn(w1[2 * j] - __bfloat162float(h0b));
            const __nv_bfloat16 l1b = __float2bfloat16_rn(w1[2 * j + 1] - __bfloat162float(h1b));
            hi[j] = (uint32_t)__bfloat16_as_ushort(h0b) | ((uint32_t)__bfloat16_as_ushort(h1b) << 16);
            lo[j] = (uint32_t)__bfloat16_as_ushort(l0b) | ((uint32_t)__bfloat16_as_ushort(l1b) << 16);
        }
        *reinterpret_cast<uint2*>(p.w1b + (size_t)u * 2 * D * HID + idx) = make_uint2(hi[0], hi[1]);
        *reinterpret_cast<uint2*>(p.w1b + (size_t)u * 2 * D * HID + D * HID + idx) = make_uint2(lo[0], lo[1]);
    }
}

// ----------------------------------------------------------------------------- apply ---
struct ApplyParams {
    int N, T;
};

struct ApplyBars {
    uint64_t wfull, qfull[4], qfree[4], z0full, z1full, a0ready, a1ready, ofull[2], oread[2];
    uint32_t tmem_base;
};
constexpr uint32_t COL_O = 256;  // apply: two 64-column O buffers after the two Z halves
constexpr int NQB = 4;           // apply: Q tile buffers (O of a tile is staged over its Q tile)

__device__ __forceinline__ uint32_t pack2_f16(uint64_t v) {
    __half2 h = __floats2half2_rn(lo2(v), hi2(v));
    return *reinterpret_cast<uint32_t*>(&h);
}

__global__ void __launch_bounds__(THREADS, 1)
    apply_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
                 const __grid_constant__ CUtensorMap tm_w1, const __grid_constant__ CUtensorMap tm_w2,
                 const ApplyParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align<1024>(smem_raw);
    uint8_t* w1s = smem;                 // W1* hi (bf16)
    uint8_t* w1l = w1s + WBYTES;         // W1* lo (bf16)
    uint8_t* w2s = w1l + WBYTES;         // W2* (fp16)
    uint8_t* at = w2s + WBYTES;          // A = gelu(Z) (fp16)
    uint8_t* qb = at + BIG;  // NQB x 16 KB: Q tiles, O staged in place
    ApplyBars* bars = reinterpret_cast<ApplyBars*>(qb + NQB * TILE);

    const int split = blockIdx.x, u = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = split * p.T;
    const int n_valid = max(0, min(p.N - t0, p.T));
    const int ntiles = (n_valid + MT - 1) / MT;

    if (threadIdx.x == 0) {
        mbar_init(&bars->wfull, 1);
        for (int b = 0; b < NQB; ++b) {
            mbar_init(&bars->qfull[b], 1);
            mbar_init(&bars->qfree[b], EPI_WARPS);
        }
        mbar_init(&bars->z0full, 1);
        mbar_init(&bars->z1full, 1);
        mbar_init(&bars->a0ready, EPI_WARPS);
        mbar_init(&bars->a1ready, EPI_WARPS);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->ofull[b], 1);
            mbar_init(&bars->oread[b], EPI_WARPS);
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
            // this unit's W1* hi and lo (rows 0-63 and 64-127 of its block) and W2*
            mbar_expect_tx(&bars->wfull, 3 * WBYTES);
#pragma unroll
            for (int a = 0; a < HID / 64; ++a) {
                tma_load_3d(w1s + a * 8192, &tm_w1, a * 64, 0, u, &bars->wfull);
                tma_load_3d(w1l + a * 8192, &tm_w1, a * 64, D, u, &bars->wfull);
            }
            tma_load_3d(w2s, &tm_w2, 0, 0, u, &bars->wfull);
            for (int i = 0; i < ntiles; ++i) {
                const int b = i % NQB;
                if (i >= NQB) mbar_wait(&bars->qfree[b], (i / NQB - 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                mbar_expect_tx(&bars->qfull[b], TILE);
                tma_load_3d(qb + b * TILE, &tm_q, 0, t0 + i * MT, u, &bars->qfull[b]);
            }
            mbar_wait(&bars->wfull, 0, TTT_DEVERR_TIMEOUT_TMA);  // no load in flight at exit
        }
    } else if (warp == 1) {
        // Z in two hidden halves (T0, T1) and O in two buffers: Z0 of tile i+1 is issued once
        // the epilogue has read Z0 of tile i, while it still works on Z1 and on O of tile i.
        if (lane == 0 && ntiles > 0) {
            const uint32_t w1a = smem_u32(w1s), w1b = smem_u32(w1l), w2a = smem_u32(w2s), aa = smem_u32(at);
            const uint32_t IZ = tc::idesc_bf16(128, 128, 0, 1);
            const uint32_t IO = tc::idesc_f16(128, 64, 0, 1);
            auto issue_z = [&](int i, int half) {
                const uint32_t qa = smem_u32(qb + (i % NQB) * TILE);
                tc::fence_after();
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tmem + COL_T + half * 128, tc::smem_desc(qa + ks * 32, 16, 1024, 2),
                                 tc::smem_desc(w1a + half * 2 * 8192 + ks * 2048, 8192, 1024, 2), IZ, ks > 0);
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tmem + COL_T + half * 128, tc::smem_desc(qa + ks * 32, 16, 1024, 2),
                                 tc::smem_desc(w1b + half * 2 * 8192 + ks * 2048, 8192, 1024, 2), IZ, 1);
                tc::commit(half ? &bars->z1full : &bars->z0full);
            };
            mbar_wait(&bars->wfull, 0, TTT_DEVERR_TIMEOUT_TMA);
            mbar_wait(&bars->qfull[0], 0, TTT_DEVERR_TIMEOUT_TMA);
            issue_z(0, 0);
            issue_z(0, 1);
            for (int i = 0; i < ntiles; ++i) {
                const int ob = i & 1;
                if (i >= 2) mbar_wait(&bars->oread[ob], ((i - 2) >> 1) & 1, TTT_DEVERR_TIMEOUT_PEER);
                for (int half = 0; half < 2; ++half) {
                    mbar_wait(half ? &bars->a1ready : &bars->a0ready, i & 1, TTT_DEVERR_TIMEOUT_PEER);
                    tc::fence_after();
                    for (int ks = half * 8; ks < half * 8 + 8; ++ks)
                        tc::mma_bf16(tmem + COL_O + ob * 64,
                                     tc::smem_desc(aa + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, 2),
                                     tc::smem_desc(w2a + ks * 2048, 8192, 1024, 2), IO, ks > 0);
                    if (half) tc::commit(&bars->ofull[ob]);
                    if (i + 1 < ntiles) {
                        if (half == 0)
                            mbar_wait(&bars->qfull[(i + 1) % NQB], ((i + 1) / NQB) & 1, TTT_DEVERR_TIMEOUT_TMA);
                        issue_z(i + 1, half);
                    }
                }
            }
        }
    } else {
        // as in the grad kernel, the epilogue waits without the suspend-time hint
        const int q4 = warp & 3, ch = (warp - 2) >> 2;
        const int r = q4 * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
        // O of tile j: TMEM -> bf16 over its Q tile (the Z MMAs that read it have completed) -> TMA
        auto o_store = [&](int j) {
            const int b = j % NQB, ob = j & 1;
            uint8_t* tile = qb + b * TILE;
            mbar_wait<false>(&bars->ofull[ob], (j >> 1) & 1, TTT_DEVERR_TIMEOUT_PEER);
            tc::fence_after();
            {
                float o[32];
                ld32(lane_base + COL_O + ob * 64 + ch * 32, o);
                tc::wait_ld();
#pragma unroll
                for (int c = 0; c < 32; c += 8) store8_bf16(tile, swz<3>(r * ROWB + (ch * 32 + c) * 2), &o[c]);
            }
            tc::fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->oread[ob]);
            // both column halves of every row quarter are in shared memory once oread completes
            mbar_wait<false>(&bars->oread[ob], (j >> 1) & 1, TTT_DEVERR_TIMEOUT_PEER);
            if (ch == 0) {
                // the row quarter's store; this warp releases the Q buffer of tile j - 1 once that
                // tile's store has read it, so no store is waited for on the way to the next gelu
                if (lane == 0) {
                    const int row0 = j * MT + q4 * 32;
                    if (row0 < n_valid) {
                        tma_store_3d(&tm_o, 0, t0 + row0, u, tile + q4 * 32 * ROWB);
                        tma_store_commit();
                        asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                    } else {
                        tma_store_wait_read_all();
                    }
                }
                __syncwarp();
                if (lane == 0 && j >= 1) mbar_arrive(&bars->qfree[(j - 1) % NQB]);
            } else {
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->qfree[b]);
            }
        };
        // gelu of tile i, then the output of tile i - 1 (whose MMAs ran meanwhile)
        for (int i = 0; i < ntiles; ++i) {
            for (int half = 0; half < 2; ++half) {  // A = gelu(Z), 64 columns per warp and half
                mbar_wait<false>(half ? &bars->z1full : &bars->z0full, i & 1, TTT_DEVERR_TIMEOUT_PEER);
                tc::fence_after();
                const int c0 = half * 128 + ch * 64;
                float z[64];
                ld32(lane_base + COL_T + c0, z);
                ld32(lane_base + COL_T + c0 + 32, z + 32);
                tc::wait_ld();
#pragma unroll
                for (int j = 0; j < 64; j += 8) {
                    uint32_t a[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) a[e] = pack2_f16(gelu2(pk2(z[j + 2 * e], z[j + 2 * e + 1])));
                    *reinterpret_cast<uint4*>(at + big_off(r, c0 + j)) = make_uint4(a[0], a[1], a[2], a[3]);
                }
                fence_proxy_async_smem();
                tc::fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(half ? &bars->a1ready : &bars->a0ready);
            }
            if (i >= 1) o_store(i - 1);
        }
        if (ntiles > 0) o_store(ntiles - 1);
        if (lane == 0) tma_store_wait_all();
        __syncwarp();
        if (ch == 0 && lane == 0 && ntiles > 0) mbar_arrive(&bars->qfree[(ntiles - 1) % NQB]);
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) tc::dealloc(tmem, 512);
}

}  // namespace mlp

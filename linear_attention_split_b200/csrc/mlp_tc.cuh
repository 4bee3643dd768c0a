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
//            (fp32 outputs if requested, bf16 copies for the apply pass).
//   apply  : per 128-token tile Z = Q W1*, A = gelu(Z), O = A W2*, stored as bf16 by TMA.
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
// gelu_tanh(u) and its derivative from the same t = tanh(sqrt(2/pi)(u + 0.044715 u^3))
__device__ __forceinline__ float gelu_gp(float u, float* gp) {
    const float s = 0.7978845608028654f, a = 0.044715f;
    const float u2 = u * u;
    const float t = tanh_fast(s * u * fmaf(a, u2, 1.f));
    *gp = 0.5f * (1.f + t) + 0.5f * u * (1.f - t * t) * s * fmaf(3.f * a, u2, 1.f);
    return 0.5f * u * (1.f + t);
}
__device__ __forceinline__ float gelu_only(float u) {
    const float s = 0.7978845608028654f, a = 0.044715f;
    return 0.5f * u * (1.f + tanh_fast(s * u * fmaf(a, u * u, 1.f)));
}
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
    const float* w1;        // [H][64][256]
    const float* w2;        // [H][256][64]
    const __nv_bfloat16* v; // [U][N][64]
    float* part;            // [U][S][2][256][64]: gW1^T then gW2
    int H, N, T;            // T = tokens per CTA (multiple of 128)
};

struct GradBars {
    uint64_t kfull[2], bfree[2], zfull, aready, pfull, rready, dafull, dzready, gdone;
    uint32_t tmem_base;
};

__device__ __forceinline__ void load_weights(uint8_t* w1s, uint8_t* w2s, const float* w1, const float* w2, int tid,
                                             int nthreads) {
    // W1 [64][256] and W2 [256][64], fp32 -> bf16 swizzled; 8 consecutive elements per store
    for (int e = tid; e < D * HID / 8; e += nthreads) {
        const int k = e / (HID / 8), n = (e % (HID / 8)) * 8;
        float v[8];
        const float4 a = *reinterpret_cast<const float4*>(&w1[k * HID + n]);
        const float4 b = *reinterpret_cast<const float4*>(&w1[k * HID + n + 4]);
        v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
        store8_bf16(w1s, w1_off(k, n), v);
    }
    for (int e = tid; e < HID * D / 8; e += nthreads) {
        const int h = e / (D / 8), d = (e % (D / 8)) * 8;
        float v[8];
        const float4 a = *reinterpret_cast<const float4*>(&w2[h * D + d]);
        const float4 b = *reinterpret_cast<const float4*>(&w2[h * D + d + 4]);
        v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
        store8_bf16(w2s, w2_off(h, d), v);
    }
}

__global__ void __launch_bounds__(THREADS, 1)
    grad_kernel(const __grid_constant__ CUtensorMap tm_k, const GradParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->kfull[b], 1);
            mbar_init(&bars->bfree[b], 1);
        }
        mbar_init(&bars->zfull, 1);
        mbar_init(&bars->aready, EPI_WARPS);
        mbar_init(&bars->pfull, 1);
        mbar_init(&bars->rready, EPI_WARPS);
        mbar_init(&bars->dafull, 1);
        mbar_init(&bars->dzready, EPI_WARPS);
        mbar_init(&bars->gdone, 1);
        mbar_fence_init();
    }
    load_weights(w1s, w2s, p.w1 + (size_t)hd * D * HID, p.w2 + (size_t)hd * HID * D, threadIdx.x, THREADS);
    if (warp == 1) tc::alloc(&bars->tmem_base, 512);
    fence_proxy_async_smem();
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ================================ producer: K tiles ============================
        // tile i's K lives in buf[i & 1]; that buffer last held tile i-1's R, freed once the
        // MMAs reading R (gW2, dA) of tile i-1 completed (bfree)
        if (lane == 0) {
            for (int i = 0; i < ntiles; ++i) {
                const int b = i & 1;
                if (i >= 1) mbar_wait(&bars->bfree[b], ((i - 1) >> 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                mbar_expect_tx(&bars->kfull[b], TILE);
                tma_load_3d(buf + b * TILE, &tm_k, 0, t0 + i * MT, u, &bars->kfull[b]);
            }
        }
    } else if (warp == 1) {
        // ================================ MMA issuer ===================================
        if (lane == 0 && ntiles > 0) {
            const uint32_t w1a = smem_u32(w1s), w2a = smem_u32(w2s), aa = smem_u32(at), ga = smem_u32(gt);
            const uint32_t IZ = tc::idesc_bf16(128, 256, 0, 1);   // K (K-major) x W1 (MN-major)
            const uint32_t IP = tc::idesc_bf16(128, 64, 0, 1);    // A (K-major) x W2 (MN-major)
            const uint32_t IG = tc::idesc_bf16(128, 64, 1, 1);    // A^T/dZ^T (MN-major) x R/K (MN-major)
            const uint32_t ID = tc::idesc_bf16(128, 256, 0, 0);   // R (K-major) x W2^T (K-major)
            for (int i = 0; i < ntiles; ++i) {
                const int b = i & 1;
                const uint32_t kb = smem_u32(buf + b * TILE), rb = smem_u32(buf + (b ^ 1) * TILE);
                const uint32_t ph = i & 1;
                // Z = K W1  (T region, 256 columns)
                mbar_wait(&bars->kfull[b], (i >> 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                if (i > 0) mbar_wait(&bars->dzready, (i - 1) & 1, TTT_DEVERR_TIMEOUT_PEER);  // T free
                tc::fence_after();
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tmem + COL_T, tc::smem_desc(kb + ks * 32, 16, 1024, 2),
                                 tc::smem_desc(w1a + ks * 2048, 8192, 1024, 2), IZ, ks > 0);
                tc::commit(&bars->zfull);
                // P = A W2  (T columns 0..63)
                mbar_wait(&bars->aready, ph, TTT_DEVERR_TIMEOUT_PEER);
                tc::fence_after();
                for (int ks = 0; ks < 16; ++ks)
                    tc::mma_bf16(tmem + COL_T, tc::smem_desc(aa + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, 2),
                                 tc::smem_desc(w2a + ks * 2048, 8192, 1024, 2), IP, ks > 0);
                tc::commit(&bars->pfull);
                // gW2 += A^T R (two 128-row halves of h) and dA = R W2^T (T region)
                mbar_wait(&bars->rready, ph, TTT_DEVERR_TIMEOUT_PEER);
                tc::fence_after();
                for (int hh = 0; hh < 2; ++hh)
                    for (int ks = 0; ks < 8; ++ks)
                        tc::mma_bf16(tmem + COL_G2 + hh * 64,
                                     tc::smem_desc(aa + hh * 2 * 16384 + ks * 2048, 16384, 1024, 2),
                                     tc::smem_desc(rb + ks * 2048, 8192, 1024, 2), IG, (i > 0 || ks > 0));
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tmem + COL_T, tc::smem_desc(rb + ks * 32, 16, 1024, 2),
                                 tc::smem_desc(w2a + ks * 32, 16, 1024, 2), ID, ks > 0);
                tc::commit(&bars->dafull);
                tc::commit(&bars->bfree[b ^ 1]);  // R buffer free once these MMAs completed
                // gW1^T += dZ^T K
                mbar_wait(&bars->dzready, ph, TTT_DEVERR_TIMEOUT_PEER);
                tc::fence_after();
                for (int hh = 0; hh < 2; ++hh)
                    for (int ks = 0; ks < 8; ++ks)
                        tc::mma_bf16(tmem + COL_G1 + hh * 64,
                                     tc::smem_desc(ga + hh * 2 * 16384 + ks * 2048, 16384, 1024, 2),
                                     tc::smem_desc(kb + ks * 2048, 8192, 1024, 2), IG, (i > 0 || ks > 0));
            }
            tc::commit(&bars->gdone);
        }
    } else {
        // ================================ epilogue (8 warps) ===========================
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
            // ---- Z -> A = gelu(Z), gelu'(Z) -------------------------------------------------
            mbar_wait(&bars->zfull, ph, TTT_DEVERR_TIMEOUT_PEER);
            tc::fence_after();
            for (int c0 = ch * 128; c0 < ch * 128 + 128; c0 += 32) {
                float z[32];
                ld32(lane_base + COL_T + c0, z);
                tc::wait_ld();
                float a[32], g[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) a[j] = gelu_gp(z[j], &g[j]);
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                    store8_bf16(at, big_off(r, c0 + j), &a[j]);
                    store8_bf16(gt, big_off(r, c0 + j), &g[j]);
                }
            }
            fence_proxy_async_smem();
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->aready);
            // ---- P -> R = P - V ---------------------------------------------------------------
            mbar_wait(&bars->pfull, ph, TTT_DEVERR_TIMEOUT_PEER);
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
            // ---- dA -> dZ = dA * gelu'(Z), in place over gelu'(Z) --------------------------------
            mbar_wait(&bars->dafull, ph, TTT_DEVERR_TIMEOUT_PEER);
            tc::fence_after();
            for (int c0 = ch * 128; c0 < ch * 128 + 128; c0 += 32) {
                float da[32];
                ld32(lane_base + COL_T + c0, da);
                tc::wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
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
            if (lane == 0) mbar_arrive(&bars->dzready);
        }
        // ---- partial gradients: TMEM -> workspace --------------------------------------------
        float* part = p.part + ((size_t)u * S + split) * 2 * HID * D;
        if (ntiles > 0) {
            mbar_wait(&bars->gdone, 0, TTT_DEVERR_TIMEOUT_PEER);
            tc::fence_after();
        }
        // TMEM lane = h row within a 128-row half; this warp: half ch, rows q4*32 + lane
        const int hrow = ch * 128 + r;
        for (int which = 0; which < 2; ++which) {  // 0: gW1^T, 1: gW2
            const uint32_t col = (which == 0 ? COL_G1 : COL_G2) + ch * 64;
            float* dst = part + (size_t)which * HID * D + (size_t)hrow * D;
            for (int c0 = 0; c0 < 64; c0 += 32) {
                float g[32];
                if (ntiles > 0) {
                    ld32(lane_base + col + c0, g);
                    tc::wait_ld();
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) g[j] = 0.f;
                }
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4*>(dst + c0 + j) = make_float4(g[j], g[j + 1], g[j + 2], g[j + 3]);
            }
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
    __nv_bfloat16* w1b;         // [U][64][256] bf16
    __nv_bfloat16* w2b;         // [U][256][64] bf16
    int H, S;
    float eta_over_n;
};

__global__ void __launch_bounds__(256) update_kernel(const UpdateParams p) {
    const int u = blockIdx.x, hd = u % p.H;
    const float* part = p.part + (size_t)u * p.S * 2 * HID * D;
    for (int e = threadIdx.x + blockIdx.y * 256; e < HID * D; e += 256 * gridDim.y) {
        const int hr = e / D, dc = e % D;  // element (h, d) of gW1^T and gW2
        float g1 = 0.f, g2 = 0.f;
        for (int s = 0; s < p.S; ++s) {   // split order
            g1 += part[(size_t)s * 2 * HID * D + e];
            g2 += part[(size_t)s * 2 * HID * D + HID * D + e];
        }
        const float w1 = p.w1[(size_t)hd * D * HID + dc * HID + hr] - p.eta_over_n * g1;  // W1*[d][h]
        const float w2 = p.w2[(size_t)hd * HID * D + e] - p.eta_over_n * g2;              // W2*[h][d]
        if (p.w1_star) p.w1_star[(size_t)u * D * HID + dc * HID + hr] = w1;
        if (p.w2_star) p.w2_star[(size_t)u * HID * D + e] = w2;
        p.w1b[(size_t)u * D * HID + dc * HID + hr] = __float2bfloat16_rn(w1);
        p.w2b[(size_t)u * HID * D + e] = __float2bfloat16_rn(w2);
    }
}

// ----------------------------------------------------------------------------- apply ---
struct ApplyParams {
    const __nv_bfloat16* w1b;  // [U][64][256]
    const __nv_bfloat16* w2b;  // [U][256][64]
    int N, T;
};

struct ApplyBars {
    uint64_t qfull[2], qfree[2], zfull, aready, ofull, oread;
    uint32_t tmem_base;
};

__global__ void __launch_bounds__(THREADS, 1)
    apply_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
                 const ApplyParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* w1s = smem;
    uint8_t* w2s = w1s + WBYTES;
    uint8_t* at = w2s + WBYTES;
    uint8_t* qb = at + BIG;  // 2 x 16 KB: Q tiles, O staged in place
    ApplyBars* bars = reinterpret_cast<ApplyBars*>(qb + 2 * TILE);

    const int split = blockIdx.x, u = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = split * p.T;
    const int n_valid = max(0, min(p.N - t0, p.T));
    const int ntiles = (n_valid + MT - 1) / MT;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->qfull[b], 1);
            mbar_init(&bars->qfree[b], EPI_WARPS);
        }
        mbar_init(&bars->zfull, 1);
        mbar_init(&bars->aready, EPI_WARPS);
        mbar_init(&bars->ofull, 1);
        mbar_init(&bars->oread, EPI_WARPS);
        mbar_fence_init();
    }
    {   // W1*, W2* (bf16) -> swizzled shared memory
        const __nv_bfloat16* w1 = p.w1b + (size_t)u * D * HID;
        const __nv_bfloat16* w2 = p.w2b + (size_t)u * HID * D;
        for (int e = threadIdx.x; e < D * HID / 8; e += THREADS) {
            const int k = e / (HID / 8), n = (e % (HID / 8)) * 8;
            *reinterpret_cast<uint4*>(w1s + w1_off(k, n)) = *reinterpret_cast<const uint4*>(w1 + k * HID + n);
        }
        for (int e = threadIdx.x; e < HID * D / 8; e += THREADS) {
            const int h = e / (D / 8), d = (e % (D / 8)) * 8;
            *reinterpret_cast<uint4*>(w2s + w2_off(h, d)) = *reinterpret_cast<const uint4*>(w2 + h * D + d);
        }
    }
    if (warp == 1) tc::alloc(&bars->tmem_base, 512);
    fence_proxy_async_smem();
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            for (int i = 0; i < ntiles; ++i) {
                const int b = i & 1;
                if (i >= 2) mbar_wait(&bars->qfree[b], ((i - 2) >> 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                mbar_expect_tx(&bars->qfull[b], TILE);
                tma_load_3d(qb + b * TILE, &tm_q, 0, t0 + i * MT, u, &bars->qfull[b]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && ntiles > 0) {
            const uint32_t w1a = smem_u32(w1s), w2a = smem_u32(w2s), aa = smem_u32(at);
            const uint32_t IZ = tc::idesc_bf16(128, 256, 0, 1);
            const uint32_t IO = tc::idesc_bf16(128, 64, 0, 1);
            for (int i = 0; i < ntiles; ++i) {
                const int b = i & 1;
                mbar_wait(&bars->qfull[b], (i >> 1) & 1, TTT_DEVERR_TIMEOUT_TMA);
                if (i > 0) mbar_wait(&bars->oread, (i - 1) & 1, TTT_DEVERR_TIMEOUT_PEER);  // TMEM free
                tc::fence_after();
                const uint32_t qa = smem_u32(qb + b * TILE);
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_bf16(tmem + COL_T, tc::smem_desc(qa + ks * 32, 16, 1024, 2),
                                 tc::smem_desc(w1a + ks * 2048, 8192, 1024, 2), IZ, ks > 0);
                tc::commit(&bars->zfull);
                mbar_wait(&bars->aready, i & 1, TTT_DEVERR_TIMEOUT_PEER);
                tc::fence_after();
                for (int ks = 0; ks < 16; ++ks)
                    tc::mma_bf16(tmem + COL_G2, tc::smem_desc(aa + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, 2),
                                 tc::smem_desc(w2a + ks * 2048, 8192, 1024, 2), IO, ks > 0);
                tc::commit(&bars->ofull);
            }
        }
    } else {
        const int q4 = warp & 3, ch = (warp - 2) >> 2;
        const int r = q4 * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
        for (int i = 0; i < ntiles; ++i) {
            const int b = i & 1;
            uint8_t* tile = qb + b * TILE;
            mbar_wait(&bars->zfull, i & 1, TTT_DEVERR_TIMEOUT_PEER);
            tc::fence_after();
            for (int c0 = ch * 128; c0 < ch * 128 + 128; c0 += 32) {
                float z[32];
                ld32(lane_base + COL_T + c0, z);
                tc::wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) z[j] = gelu_only(z[j]);
#pragma unroll
                for (int j = 0; j < 32; j += 8) store8_bf16(at, big_off(r, c0 + j), &z[j]);
            }
            fence_proxy_async_smem();
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->aready);
            // O = A W2* -> bf16 over the Q tile (its MMA finished before zfull) -> TMA store
            mbar_wait(&bars->ofull, i & 1, TTT_DEVERR_TIMEOUT_PEER);
            tc::fence_after();
            {
                float o[32];
                ld32(lane_base + COL_G2 + ch * 32, o);
                tc::wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j += 8) store8_bf16(tile, swz<3>(r * ROWB + (ch * 32 + j) * 2), &o[j]);
            }
            tc::fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars->oread);
                // rows q4*32 .. +31 of this tile, columns of this half are written by this warp;
                // the other half's warp writes the other 32 columns: one store per row-quarter
                // is issued by the ch == 0 warp after both halves have arrived (oread phase)
            }
            // wait until both column halves of this row quarter are in shared memory
            mbar_wait(&bars->oread, i & 1, TTT_DEVERR_TIMEOUT_PEER);
            if (ch == 0 && lane == 0) {
                const int row0 = i * MT + q4 * 32;
                if (row0 < n_valid) {
                    tma_store_3d(&tm_o, 0, t0 + row0, u, tile + q4 * 32 * ROWB);
                    tma_store_commit();
                    tma_store_wait_read_all();
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->qfree[b]);
        }
        if (lane == 0) tma_store_wait_all();
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) tc::dealloc(tmem, 512);
}

}  // namespace mlp

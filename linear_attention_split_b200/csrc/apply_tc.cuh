// apply_tc.cuh -- O = Q W for a given fp32 W per unit, bf16 Q and O, d = 64: the output pass of
// the mini-batch / multi-epoch path ("ViT^3" blog, design study "inner training 怎么配": after
// the inner epochs the layer outputs F_W(q) = q W with the final weights).
//
// One CTA per 128-token tile of a unit: the Q tile arrives by TMA (128-byte swizzle, rows past N
// zero-filled); the four warps turn the unit's W (fp32, 16 KB, L2-resident across the unit's
// tiles) into bf16 hi + lo K-major operands, W = W_hi + W_lo to about 2^-16 relative; one thread
// issues O = Q W_hi + Q W_lo as eight M = 128, N = 64, K = 16 tcgen05 MMAs into 64 TMEM
// columns; each warp reads its 32 rows back, writes O in bf16 over the Q tile, and one TMA store
// writes the tile (rows past N clipped).  About 33 KB of shared memory and 64 TMEM columns per
// CTA, so several CTAs share an SM and one's loads overlap another's MMAs and stores.
#pragma once
#include "common.cuh"

namespace atc {

constexpr int D = 64;
constexpr int MT = 128;               // tokens per tile
constexpr int ROWB = D * 2;           // bytes per token row
constexpr int TILE = MT * ROWB;       // 16 KB
constexpr int OPB = D * ROWB;         // one 64 x 64 bf16 operand, 8 KB
constexpr int THREADS = 128;
constexpr uint32_t IDESC = tc::idesc_bf16(128, 64, 0, 0);  // A = Q K-major, B = W^T K-major

struct Bars {
    uint64_t qfull, mfull;
    uint32_t tmem_base;
};
constexpr int smem_bytes() { return TILE + 2 * OPB + (int)sizeof(Bars) + 1024; }

// byte offset of element (row n, column k) in a 64 x 64 bf16 K-major operand, 128-byte swizzle
__device__ __forceinline__ uint32_t op_off(int n, int k) {
    return (uint32_t)(n >> 3) * 1024u + swz<3>((uint32_t)(n & 7) * ROWB + (uint32_t)k * 2u);
}

__global__ void __launch_bounds__(THREADS)
    apply_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
                 const float* __restrict__ w) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* qt = smem_align<1024>(smem_raw);  // the Q tile, then the O tile
    uint8_t* wh = qt + TILE;                    // W^T hi
    uint8_t* wl = wh + OPB;                     // W^T lo
    Bars* bars = reinterpret_cast<Bars*>(wl + OPB);
    const int tile = blockIdx.x, u = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&bars->qfull, 1);
        mbar_init(&bars->mfull, 1);
        mbar_fence_init();
    }
    if (warp == 0) tc::alloc(&bars->tmem_base, 64);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = bars->tmem_base;
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tm_q);
        mbar_expect_tx(&bars->qfull, TILE);  // rows past N are zero-filled and counted
        tma_load_3d(qt, &tm_q, 0, tile * MT, u, &bars->qfull);
    }
    // W (row k = input feature, column n = output feature) -> operand row n, column k, as
    // bf16 hi + lo; consecutive threads take consecutive n, so the reads of W are coalesced
    // (all of a thread's loads are issued before any is used: one L2 round trip)
    const float* wu = w + (size_t)u * D * D;
    constexpr int PER = D * D / 2 / THREADS;  // input-row pairs per thread
    float wa[PER], wb[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = threadIdx.x + i * THREADS, n = e % D, kp = e / D;
        wa[i] = __ldg(wu + (2 * kp) * D + n);
        wb[i] = __ldg(wu + (2 * kp + 1) * D + n);
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = threadIdx.x + i * THREADS, n = e % D, kp = e / D;
        const uint32_t hi = pack_bf16(wa[i], wb[i]);
        const float ha = __uint_as_float(hi << 16), hb = __uint_as_float(hi & 0xffff0000u);
        *reinterpret_cast<uint32_t*>(wh + op_off(n, 2 * kp)) = hi;
        *reinterpret_cast<uint32_t*>(wl + op_off(n, 2 * kp)) = pack_bf16(wa[i] - ha, wb[i] - hb);
    }
    fence_proxy_async_smem();  // read next by the tensor cores
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (threadIdx.x == 0) {
        mbar_wait(&bars->qfull, 0, TTT_DEVERR_TIMEOUT_TMA);
        tc::fence_after();
        const uint64_t dq = tc::smem_desc(smem_u32(qt), 16, 1024, 2);
        const uint64_t dh = tc::smem_desc(smem_u32(wh), 16, 1024, 2);
        const uint64_t dl = tc::smem_desc(smem_u32(wl), 16, 1024, 2);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) tc::mma_bf16(tmem, dq + 2 * ks, dh + 2 * ks, IDESC, ks > 0 ? 1 : 0);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) tc::mma_bf16(tmem, dq + 2 * ks, dl + 2 * ks, IDESC, 1);
        tc::commit(&bars->mfull);
    }
    // O: warp w reads TMEM lanes 32w .. 32w + 31 (token rows) and writes them over the Q tile
    mbar_wait(&bars->mfull, 0, TTT_DEVERR_TIMEOUT_TMA);
    tc::fence_after();
    const int row = warp * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        float o[32];
        tc::ld16(lane_base + half * 32, &o[0]);
        tc::ld16(lane_base + half * 32 + 16, &o[16]);
        tc::wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(qt + swz<3>((uint32_t)row * ROWB + half * 64 + c * 16)) =
                make_uint4(pack_bf16(o[8 * c], o[8 * c + 1]), pack_bf16(o[8 * c + 2], o[8 * c + 3]),
                           pack_bf16(o[8 * c + 4], o[8 * c + 5]), pack_bf16(o[8 * c + 6], o[8 * c + 7]));
    }
    tc::fence_before();
    fence_proxy_async_smem();  // read next by the TMA store
    __syncthreads();
    if (threadIdx.x == 0) {
        tma_store_3d(&tm_o, 0, tile * MT, u, qt);  // rows past N are clipped
        tma_store_commit();
        tma_store_wait_read_all();  // the tile stays in shared memory until the store has read it
    }
    __syncwarp();
    if (warp == 0) tc::dealloc(tmem, 64);
}

}  // namespace atc

// common.cuh -- device helpers shared by the TTT-layer kernels (sm_100a).
//
// Hand-written inline PTX for: mbarriers with bounded waits, TMA tensor loads/stores
// (never with cluster multicast: every CTA fetches its own tiles), thread-block-cluster
// barriers and distributed shared memory, ldmatrix and bf16 mma.sync fragments, the
// shared-memory swizzle that matches TMA's 128B/64B swizzle modes, and packed fp32 math.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#ifndef TTT_SPIN_LIMIT_CYCLES
// Default upper bound on any wait for data that another agent produces (TMA, the tensor
// cores, another CTA): about one second at the boost clock.
#define TTT_SPIN_LIMIT_CYCLES (2000000000LL)
#endif

// Device-side error word (one per device, this library's module).  Bits set by kernels:
#define TTT_DEVERR_TIMEOUT_TMA 0x1u      // a TMA transaction never completed
#define TTT_DEVERR_TIMEOUT_PEER 0x2u     // a peer CTA never published its data
#define TTT_DEVERR_BAD_LAUNCH 0x4u       // a kernel found its launch shape inconsistent
#define TTT_DEVERR_TIMEOUT_ANY (TTT_DEVERR_TIMEOUT_TMA | TTT_DEVERR_TIMEOUT_PEER)

__device__ unsigned int g_ttt_device_error;
// Wait limit in SM clock cycles (host-settable for tests through ttt_debug_set_wait_limit).
__device__ long long g_ttt_wait_limit = TTT_SPIN_LIMIT_CYCLES;
// Test hook armed from the host (ttt_debug_arm_fault); 0 in normal operation.  Bit
// TTT_FAULT_SKIP_LOAD (declared in ttt.h): the TTT-Linear producer leaves out its last K/V load.
__device__ unsigned int g_ttt_fault;

__device__ __forceinline__ void ttt_raise(unsigned int bits) { atomicOr(&g_ttt_device_error, bits); }
// True once any wait on this device has run out (until the host reads the error word): every
// later wait then gives up at once, so one lost transfer costs one wait limit per kernel and
// the kernel still reaches its normal teardown.
__device__ __forceinline__ bool ttt_timed_out() {
    return (*reinterpret_cast<volatile unsigned int*>(&g_ttt_device_error) & TTT_DEVERR_TIMEOUT_ANY) != 0;
}
__device__ __forceinline__ long long ttt_wait_limit() {
    return *reinterpret_cast<volatile long long*>(&g_ttt_wait_limit);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// The dynamic shared-memory base `raw` rounded up to ALIGN bytes.  The rounding is pointer
// arithmetic on the __shared__ array (not a round trip through an integer), so the compiler
// still sees a shared-memory pointer and accesses through it become shared-memory loads and
// stores with immediate offsets instead of 64-bit generic ones.
template <uint32_t ALIGN>
__device__ __forceinline__ uint8_t* smem_align(uint8_t* raw) {
    return raw + ((ALIGN - (smem_u32(raw) & (ALIGN - 1u))) & (ALIGN - 1u));
}

// ----------------------------------------------------------------------- mbarrier ----
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// With SUSPEND the waiting thread is suspended (it issues nothing) until the phase completes
// or, at the latest, TTT_WAIT_SUSPEND_NS have passed, so waiting warps leave the issue slots to
// the warps that have work.  Without it the wait uses the hardware's own time limit.  Measured
// on B200, per kernel: the suspend hint is faster where many warps wait while a few compute
// (TTT-Linear full batch 13.84 against 14.09 us, the ViT^3 block, the backward), the hardware
// limit where a latency-bound chain hands off through barriers (the chunked scan 92.7 against
// 94.2 us).
#ifndef TTT_WAIT_SUSPEND_NS
#define TTT_WAIT_SUSPEND_NS 1000000u
#endif
template <bool SUSPEND = true>
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    if constexpr (SUSPEND)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity), "r"(TTT_WAIT_SUSPEND_NS)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
    return ok != 0;
}
// Non-blocking test of a phase (for polling several barriers in turn).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: returns false (and raises `err`) if the phase does not complete within the
// wait limit, and at once if another wait on this device has already run out.
template <bool SUSPEND = true>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned int err) {
    if (mbar_try_wait<SUSPEND>(bar, parity)) return true;
    const long long limit = ttt_wait_limit();
    const long long t0 = clock64();
    while (!mbar_try_wait<SUSPEND>(bar, parity)) {
        if (ttt_timed_out()) return false;
        if (clock64() - t0 > limit) {
            ttt_raise(err);
            return false;
        }
    }
    return true;
}

// ----------------------------------------------------------------------- TMA ---------
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
// 3-D tiled load into this CTA's shared memory, completion counted on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, int c0, int c1,
                                            int c2, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}
// 3-D tiled store from shared memory; rows outside the tensor are clipped by the hardware.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, int c0, int c1, int c2,
                                             const void* src) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::
            "l"(reinterpret_cast<uint64_t>(m)),
        "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(src))
        : "memory");
}
__device__ __forceinline__ void tma_store_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void tma_store_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void tma_store_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ----------------------------------------------------------------------- grid dependency ---
// Programmatic dependent launch: wait until the previous grid on the stream has completed (and
// its writes are visible); let the next grid's CTAs start launching.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ----------------------------------------------------------------------- clusters ----
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
    cluster_arrive_release();
    cluster_wait_acquire();
}
// Address of the same shared-memory variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t dsmem_map(const void* local, uint32_t rank) {
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(local)), "r"(rank));
    return out;
}
__device__ __forceinline__ float4 dsmem_ld_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}
__device__ __forceinline__ void dsmem_st_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// Bounded wait with cluster-scope acquire (data written by peer CTAs with st.async).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, unsigned int err) {
    const long long limit = ttt_wait_limit();
    const long long t0 = clock64();
    for (;;) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (ok) return true;
        if (ttt_timed_out()) return false;
        if (clock64() - t0 > limit) {
            ttt_raise(err);
            return false;
        }
    }
}
// 16 / 8 bytes into another CTA's shared memory, completion counted on its mbarrier.
__device__ __forceinline__ void st_async_v4(uint32_t raddr, uint32_t rbar, uint32_t a, uint32_t b, uint32_t c,
                                            uint32_t d) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                     raddr),
                 "r"(a), "r"(b), "r"(c), "r"(d), "r"(rbar)
                 : "memory");
}
__device__ __forceinline__ void st_async_v2(uint32_t raddr, uint32_t rbar, uint32_t a, uint32_t b) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];" ::"r"(raddr),
                 "r"(a), "r"(b), "r"(rbar)
                 : "memory");
}
__device__ __forceinline__ uint32_t mapa_u32(uint32_t saddr, uint32_t rank) {
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(saddr), "r"(rank));
    return out;
}

// ----------------------------------------------------------------------- swizzle -----
// Byte offset -> swizzled byte offset inside a region aligned to the swizzle atom.
// SW = 3 matches CU_TENSOR_MAP_SWIZZLE_128B (8 rows of 128 B), SW = 2 the 64B mode.
template <int SW>
__device__ __forceinline__ uint32_t swz(uint32_t off) {
    return off ^ (((off >> 7) & ((1u << SW) - 1u)) << 4);
}

// ----------------------------------------------------------------------- mma.sync ----
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r0), "=r"(r1)
                 : "r"(addr));
}
// D(16x8 f32) += A(16x16 bf16, row) * B(16x8 bf16, col)
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// ----------------------------------------------------------------------- scalar I/O --
template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) {
    return x;
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) {
    return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// gelu with the tanh form and its derivative, sharing t (full-precision tanhf)
__device__ __forceinline__ float gelu_tanh_f(float u, float* dgelu) {
    const float s = 0.7978845608028654f;  // sqrt(2/pi)
    const float a = 0.044715f;
    float t = tanhf(s * (u + a * u * u * u));
    if (dgelu) *dgelu = 0.5f * (1.f + t) + 0.5f * u * (1.f - t * t) * s * (1.f + 3.f * a * u * u);
    return 0.5f * u * (1.f + t);
}

// ----------------------------------------------------------------------- tcgen05 -----
// 5th-generation tensor cores: MMA issued by one thread, operands in shared memory
// (described by 64-bit matrix descriptors), fp32 accumulator in tensor memory (TMEM).
namespace tc {

// Shared-memory matrix descriptor: start address, leading/stride byte offsets (16-byte
// units), descriptor version 1, swizzle mode (2 = 128-byte swizzle, 4 = 64-byte).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t swz_mode) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)(swz_mode & 7u) << 61;
    return d;
}
// Instruction descriptor for kind::f16 with bf16 A/B, fp32 D.  mn_a / mn_b select the
// MN-major (transposed) operand layout.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int mn_a, int mn_b) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)mn_a << 15) | ((uint32_t)mn_b << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// The same for fp16 A/B (both operands of one MMA share the type), fp32 D.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int mn_a, int mn_b) {
    return (1u << 4) | ((uint32_t)mn_a << 15) | ((uint32_t)mn_b << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, int acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// Arrive once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
// Warp-collective TMEM allocation; the base address is written to *dst (shared memory).
__device__ __forceinline__ void alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// 32 lanes x 16 consecutive 32-bit columns: thread t gets lane (base lane + t), 16 columns.
__device__ __forceinline__ void ld16(uint32_t taddr, float* v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
        "%13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

}  // namespace tc

// ----------------------------------------------------------------------- bulk DSMEM --
// Copy `bytes` (multiple of 16) from this CTA's shared memory into CTA `rank` of the
// cluster, at the same offset as `local_dst`; completion is counted on that CTA's barrier
// at the same offset as `local_bar`.  (Plain bulk copy: no multicast.)
__device__ __forceinline__ void bulk_push(const void* local_src, const void* local_dst, const uint64_t* local_bar,
                                          uint32_t rank, uint32_t bytes) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dsmem_map(local_dst, rank)),
        "r"(smem_u32(local_src)), "r"(bytes), "r"(dsmem_map(local_bar, rank))
        : "memory");
}

// Prefetch a 3-D tile of a tensor into L2 (no shared-memory destination).
__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap* m, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}

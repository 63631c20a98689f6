// lcs_common.cuh -- device helpers shared by the liblcs kernels (sm_100a only).
//
// PTX wrappers for mbarriers, TMA, cp.async and the 5th-generation tensor cores
// (tcgen05: TMEM allocation, MMA issue, commit, TMEM loads), shared-memory
// matrix descriptors, bounded waits that report a timeout instead of hanging,
// and the number-format conversions of the storage types.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_fp4.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lcs.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "liblcs targets sm_100a (B200) only"
#endif

namespace lcs {

// ---------------------------------------------------------------- status word
// The first 256 bytes of every workspace.  status[0] holds the first error code
// recorded by any kernel since it was last cleared; status[1] a detail word
// (which wait gave up).
struct Status {
    int code;
    int detail;
};

__device__ __forceinline__ void set_status(int* status, int code, int detail) {
    if (status == nullptr) return;
    if (atomicCAS(status, 0, code) == 0) status[1] = detail;
}

// Bounded waits give up after this many nanoseconds of %globaltimer.
constexpr uint64_t kWaitBudgetNs = 2000000000ull;   // 2 s

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ addresses
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounds a polling loop: every 64 polls, gives up (false) once the grid's status word
// is non-zero or the budget is spent (recording LCS_ERR_TIMEOUT with `where`).  The
// status word is read one check ahead of its use, so the load completes while the
// caller polls and a wait that is about to succeed never sits behind a memory round trip.
struct WaitBudget {
    uint64_t t0, budget_ns;
    uint32_t polls = 0;
    int seen = 0;
    __device__ __forceinline__ explicit WaitBudget(uint64_t ns = kWaitBudgetNs) : t0(globaltimer()), budget_ns(ns) {}
    __device__ __forceinline__ bool ok(int* status, int where) {
        if ((++polls & 63u) != 0) return true;
        if (seen != 0) return false;
        if (status != nullptr) seen = *(volatile int*)status;
        if (globaltimer() - t0 > budget_ns) {
            set_status(status, LCS_ERR_TIMEOUT, where);
            return false;
        }
        return true;
    }
};

// Waits for the phase with the given parity to complete.  Returns false (and
// records LCS_ERR_TIMEOUT with `where` as detail) if it does not within the
// budget.  Once any wait in the grid has failed (status non-zero) later waits
// give up at a following check so that every thread reaches its exit path.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status, int where,
                                          uint64_t budget_ns = kWaitBudgetNs) {
    if (mbar_try_wait(bar, parity)) return true;
    WaitBudget wb(budget_ns);
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (!wb.ok(status, where)) return false;
    }
}

// ------------------------------------------------------------------ cp.async
__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gmem_src, bool valid) {
    const uint32_t n = valid ? 16u : 0u;   // 0 source bytes -> 16 zero bytes
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src),
                 "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Arrive on an mbarrier when all of this thread's prior cp.async copies land.
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Make generic-proxy shared-memory writes visible to the async proxy (the
// tensor cores read operands through it).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
            "r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
            "r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// (group, tile, request) of a linear tile index it = g * tiles_per + tile, with
// g = b * Q + q, advanced by one tile without integer division.
struct TileIt {
    int64_t g, b;
    int tile, q;
    __device__ __forceinline__ TileIt(int64_t it, int tiles_per, int Q) {
        g = it / tiles_per;
        tile = (int)(it - g * tiles_per);
        b = g / Q;
        q = (int)(g - b * Q);
    }
    __device__ __forceinline__ void next(int tiles_per, int Q) {
        if (++tile == tiles_per) {
            tile = 0;
            ++g;
            if (++q == Q) {
                q = 0;
                ++b;
            }
        }
    }
};

// ------------------------------------------------------------ clusters / DSMEM
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Every thread of every CTA of the cluster; shared-memory writes before it are visible
// to the cluster's reads after it.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of this CTA's shared variable `p` in the shared memory of cluster CTA `rank`.
__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ uint32_t ld_dsmem_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}
// Remote (or local) shared-memory reduction in a cluster CTA; no value is returned, so the
// issuing thread does not wait for it.
__device__ __forceinline__ void red_dsmem_add_u32(uint32_t addr, uint32_t v) {
    asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_dsmem_u64(uint32_t addr) {
    unsigned long long v;
    asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D(tmem) (+)= A(smem desc) * B(smem desc), kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D(tmem) (+)= A * B, kind::f8f6f4 (both operands E2M1 in 8-bit containers).
__device__ __forceinline__ void mma_f8f6f4_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when all prior tcgen05.mma of this thread complete.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 bits, 8 consecutive columns (thread i: lane base + i, register j: column
// base + j).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
// 32 lanes x 32 bits, 16 consecutive columns: thread i of the warp gets lane
// (base lane + i), registers j = column (base column + j).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
// 16 lanes x 32 bits, two column halves: threads 0-15 read lanes base..base+15 at
// columns [c, c+32), threads 16-31 the same lanes at columns [c+32, c+64).
__device__ __forceinline__ void tmem_ld16x2_32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// TMEM address: lane in bits 31..16, column in bits 15..0.
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
    return base + (lane << 16) + col;
}

// Shared-memory matrix descriptor, 128-byte swizzle (SW128), sm_100 version 1.
//   K-major operand: rows of 128 bytes (64 bf16 of K) in 8-row, 1024-byte atoms;
//     sbo = byte stride between 8-row groups (1024 for dense atoms), lbo unused.
//   MN-major operand: 128 bytes (64 bf16) along M/N per row, 8 K-rows per atom;
//     lbo = byte stride between 64-element M/N blocks, sbo = stride between 8-row K groups.
// The start address may step inside an atom (e.g. +32 bytes per K=16 bf16 step
// of a K-major operand); the atom base must be 1024-byte aligned.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr & 0x3FFFF) >> 4);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;   // layout: SWIZZLE_128B
    return d;
}

// Shared-memory matrix descriptor, 64-byte swizzle (SW64), sm_100 version 1: K-major rows
// of 64 bytes in 8-row, 512-byte atoms; sbo = byte stride between 8-row groups (512 for
// dense atoms), lbo unused.  The start address may step inside an atom (e.g. +32 bytes per
// K=64 step of packed FP4); the atom base must be 512-byte aligned.
__device__ __forceinline__ uint64_t sw64_desc(uint32_t smem_addr, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr & 0x3FFFF) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version (sm_100)
    d |= (uint64_t)4 << 61;   // layout: SWIZZLE_64B
    return d;
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> fp32, dense.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4)                          // D format fp32
           | (1u << 7)                        // A bf16
           | (1u << 10)                       // B bf16
           | ((a_mn_major ? 1u : 0u) << 15)   // A major
           | ((b_mn_major ? 1u : 0u) << 16)   // B major
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Instruction descriptor, kind::f8f6f4: E2M1 x E2M1 -> fp32, dense, K-major.
__host__ __device__ constexpr uint32_t idesc_e2m1(int M, int N) {
    return (1u << 4) | (5u << 7) | (5u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Byte offset of the 16-byte chunk `c` (0..7) of row `r` inside a SW128 atom column.
__device__ __forceinline__ uint32_t sw128_off(uint32_t r, uint32_t c) {
    return r * 128u + ((c ^ (r & 7u)) << 4);
}

// ----------------------------------------------------------------- formats
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&h);
}

// Two floats -> two bf16 packed (low half = a).
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    return (uint32_t)f32_to_bf16_bits(a) | ((uint32_t)f32_to_bf16_bits(b) << 16);
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
    return __half2float(*reinterpret_cast<__half*>(&h));
}

__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
    return (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ uint8_t f32_to_e2m1(float x) {
    return (uint8_t)__nv_cvt_float_to_fp4(x, __NV_E2M1, cudaRoundNearest) & 0xF;
}

// Order-preserving keys: larger float -> larger unsigned key; -0 maps like +0.
__device__ __forceinline__ uint32_t f32_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ uint32_t bf16_key(uint16_t b) {
    uint32_t u = b;
    if (u == 0x8000u) u = 0;
    return (u & 0x8000u) ? (~u & 0xFFFFu) : (u | 0x8000u);
}

// ------------------------------------------------------ shared cache writers
// Rotate-half RoPE of one pair (x1 at dim c0 + i, x2 at dim c0 + i + d_rope/2) at position
// pos: angle pos * theta^(-2i/d_rope), formed and reduced in double so that positions near
// 2^20 keep full fp32 accuracy after the reduction.
__device__ __forceinline__ void rope_pair(float x1, float x2, int64_t pos, int i, int d_rope, float theta, float& o1,
                                          float& o2) {
    const double freq = pow((double)theta, -2.0 * i / (double)d_rope);
    double a = (double)pos * freq;
    a -= 6.283185307179586 * rint(a * 0.15915494309189535);
    float sn, cs;
    sincosf((float)a, &sn, &cs);
    o1 = x1 * cs - x2 * sn;
    o2 = x2 * cs + x1 * sn;
}

__device__ __forceinline__ float warp_max(float v);

// One warp writes one mixed-precision KV row: each 128-dim content block as E4M3 codes of
// x / scale with the smallest power-of-two scale >= amax/448 (1 when amax is 0), then the
// d_r RoPE dims as bf16, then the fp32 scales.  xr: d_c + d_r floats, 16-byte aligned.
__device__ __forceinline__ void quant_kv_fp8_row_warp(const float* xr, int d_c, int d_r, uint8_t* o) {
    const int lane = threadIdx.x & 31;
    const int nb = d_c / 128;
    for (int b = 0; b < nb; ++b) {
        const float4 v = *reinterpret_cast<const float4*>(xr + b * 128 + 4 * lane);
        float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
        amax = warp_max(amax);
        // smallest power of two >= amax/448: round the fp32 bit pattern up to the next exponent
        const float t = amax / 448.0f;
        const uint32_t tb = __float_as_uint(t);
        const float sc = (t > 0.0f) ? __uint_as_float((tb + 0x007FFFFFu) & 0xFF800000u) : 1.0f;
        const uint32_t c = (uint32_t)f32_to_e4m3(v.x / sc) | ((uint32_t)f32_to_e4m3(v.y / sc) << 8) |
                           ((uint32_t)f32_to_e4m3(v.z / sc) << 16) | ((uint32_t)f32_to_e4m3(v.w / sc) << 24);
        *reinterpret_cast<uint32_t*>(o + b * 128 + 4 * lane) = c;
        if (lane == 0) *reinterpret_cast<float*>(o + d_c + 2 * d_r + 4 * b) = sc;
    }
    for (int j = lane; j < d_r; j += 32) {
        const uint16_t h = f32_to_bf16_bits(xr[d_c + j]);
        *reinterpret_cast<uint16_t*>(o + d_c + 2 * j) = h;
    }
}

// One warp quantises one 32-element FP4 block (lane = element v): scale = E4M3(amax/6), 1
// when that is 0; code = E2M1(v / scale).  Writes the 16 packed bytes (element 2j in the
// low nibble of byte j) and the scale byte.
__device__ __forceinline__ void quant_fp4_block_warp(float v, uint8_t* packed16, uint8_t* scale) {
    const int lane = threadIdx.x & 31;
    const float amax = warp_max(fabsf(v));
    uint8_t sc_code = f32_to_e4m3(amax / 6.0f);
    if ((sc_code & 0x7F) == 0) sc_code = 0x38;   // 1.0
    const float sc = e4m3_to_f32(sc_code);
    const uint32_t q = f32_to_e2m1(v / sc);
    const uint32_t other = __shfl_down_sync(0xffffffffu, q, 1);
    if ((lane & 1) == 0) packed16[lane / 2] = (uint8_t)(q | (other << 4));
    if (lane == 0) *scale = sc_code;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace lcs

// common.cuh -- small device helpers shared by the RAM-Net kernels (sm_100a only).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/ramnet.h"
#include "kernels.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "the RAM-Net kernels are written for sm_100a (B200) only"
#endif

namespace ramnet {

// Bounded spin limit for every cross-block wait (try_wait polls; ~seconds worst case).
constexpr uint32_t kSpinLimit = 1u << 26;

__device__ __forceinline__ float load_in(const void* p, size_t i, int is_bf16)
{
    if (is_bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
    return reinterpret_cast<const float*>(p)[i];
}

// N consecutive fp32 values from / to global memory, vectorised (p aligned to 4*N bytes,
// or 16 bytes for N = 8).
template <int N>
__device__ __forceinline__ void load_row_g(const float* p, float (&v)[N])
{
    if constexpr (N == 1) {
        v[0] = p[0];
    } else if constexpr (N == 2) {
        const float2 a = *reinterpret_cast<const float2*>(p);
        v[0] = a.x;
        v[1] = a.y;
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            const float4 a = *reinterpret_cast<const float4*>(p + i);
            v[i] = a.x;
            v[i + 1] = a.y;
            v[i + 2] = a.z;
            v[i + 3] = a.w;
        }
    }
}

template <int N>
__device__ __forceinline__ void store_row_g(float* p, const float (&v)[N])
{
    if constexpr (N == 1) {
        p[0] = v[0];
    } else if constexpr (N == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 4) *reinterpret_cast<float4*>(p + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    }
}

__device__ __forceinline__ void store_out(void* p, size_t i, float x, int is_bf16)
{
    if (is_bf16) reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
    else reinterpret_cast<float*>(p)[i] = x;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bit)
{
    if (status) atomicOr(status, bit);
}

// Range check of an index computed on the device.  In a build with RAMNET_DEBUG defined a
// failing check records kDevCheck in the status word and the caller skips the access; in
// the normal build the check compiles away.  No trap and no assert either way.
__device__ __forceinline__ bool dcheck(bool ok, uint32_t* status)
{
#ifdef RAMNET_DEBUG
    if (!ok) set_status(status, kDevCheck);
    return ok;
#else
    (void)status;
    return ok || true;
#endif
}

// ------------------------------------------------------------------ cluster / mbarrier

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared variable in cluster CTA `rank` (shared::cluster window).
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank)
{
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(saddr), "r"(rank));
    return out;
}

// Whole-cluster hardware barrier with release/acquire ordering.  Used where every thread of
// every CTA of the cluster reaches it unconditionally: after the mbarriers are initialised
// (before any CTA arrives on a peer's barrier) and before exit (so that no CTA leaves while
// a peer may still write into its shared memory).
__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init_cluster()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Arrive (release, cluster scope) on the mbarrier at shared::cluster address `caddr`, which
// may be in this CTA or in a peer of its cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t caddr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}

// 16-byte store into a peer CTA's shared memory (shared::cluster address).
__device__ __forceinline__ void st_cluster_v4(uint32_t caddr, float a, float b, float c, float d)
{
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(caddr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// ------------------------------------------------------------------ tensor memory (TMEM)

// Allocate `ncols` columns (power of two, >= 32) for this CTA; executed by one full warp.
// The base address is written to shared memory at `holder`.
__device__ __forceinline__ void tmem_alloc(uint32_t* holder, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(holder)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tmem_fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Warp-wide load of N consecutive 32-bit columns starting at `taddr` (lane field = the
// warp's quadrant); lane i receives row (quadrant base + i).
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[N]);
template <>
__device__ __forceinline__ void tmem_ld<1>(uint32_t a, float (&v)[1])
{
    uint32_t r0;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r0) : "r"(a));
    v[0] = __uint_as_float(r0);
}
template <>
__device__ __forceinline__ void tmem_ld<2>(uint32_t a, float (&v)[2])
{
    uint32_t r0, r1;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(a));
    v[0] = __uint_as_float(r0);
    v[1] = __uint_as_float(r1);
}
template <>
__device__ __forceinline__ void tmem_ld<4>(uint32_t a, float (&v)[4])
{
    uint32_t r0, r1, r2, r3;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(a));
    v[0] = __uint_as_float(r0);
    v[1] = __uint_as_float(r1);
    v[2] = __uint_as_float(r2);
    v[3] = __uint_as_float(r3);
}
template <>
__device__ __forceinline__ void tmem_ld<8>(uint32_t a, float (&v)[8])
{
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(a));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

template <int N>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const float (&v)[N]);
template <>
__device__ __forceinline__ void tmem_st<1>(uint32_t a, const float (&v)[1])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(a), "r"(__float_as_uint(v[0])) : "memory");
}
template <>
__device__ __forceinline__ void tmem_st<2>(uint32_t a, const float (&v)[2])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1,%2};" ::"r"(a), "r"(__float_as_uint(v[0])),
                 "r"(__float_as_uint(v[1]))
                 : "memory");
}
template <>
__device__ __forceinline__ void tmem_st<4>(uint32_t a, const float (&v)[4])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(__float_as_uint(v[0])),
                 "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3]))
                 : "memory");
}
template <>
__device__ __forceinline__ void tmem_st<8>(uint32_t a, const float (&v)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(a),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
                 : "memory");
}

}  // namespace ramnet

// lb_common.cuh - device helpers shared by the library's kernels (sm_100a).
//
// Thin wrappers over PTX: asynchronous global->shared copies, the register
// tensor-core MMA used by the decode kernels, programmatic dependent launch,
// thread-block-cluster barriers and distributed shared memory, and the device
// status word.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "lb.h"

namespace lb {

// ---------------------------------------------------------------- status word
// Kernels record the first device-side failure here (see lb_device_status).
__device__ __forceinline__ void set_status(int *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------- cp.async
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte async copy global -> shared; bytes past `src_bytes` (0 or 16) are zero-filled.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes = 16)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n"
                 :: "r"(smem_u32(dst)), "l"(src), "r"(src_bytes) : "memory");
}



// 16, 8 or 4 bytes global -> shared (address in the shared window), both aligned
__device__ __forceinline__ void cp_async16s(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src) : "memory");
}
// wait until at most N of this thread's most recent cp.async groups are pending
template <int N>
__device__ __forceinline__ void cp_async_wait_group()
{
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// Loads issued where they stand in the program: weights fetched ahead of use
// (at kernel entry, or K-blocks ahead) so that their latency overlaps other
// work.  The compiler does not move a volatile asm past another one (such as
// a dependency wait or a barrier), nor sink it to the first use of its result.
__device__ __forceinline__ uint4 ldg_early_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ uint2 ldg_early_v2(const void *p)
{
    uint2 v;
    asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ldg_early_u32(const void *p)
{
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint16_t ldg_early_u16(const void *p)
{
    uint16_t v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// ---------------------------------------------------------------- PDL
// Wait until the grids this one depends on (programmatic stream
// serialisation) have completed and their writes are visible.  A no-op when
// the kernel was launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
// Let the next grid on the stream start its prologue early.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// Full cluster barrier with release/acquire semantics for shared::cluster memory.
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n"
                 "barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
// Split cluster barrier: arrive early, wait later (no memory ordering; used
// to know that every CTA of the cluster has started before touching its
// shared memory).
__device__ __forceinline__ void cluster_arrive_relaxed()
{
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;\n" ::: "memory"); }
// Address of `p` (a shared-memory variable of this CTA) in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_shared_rank(const void *p, uint32_t rank)
{
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
    return out;
}
__device__ __forceinline__ void st_shared_cluster_f32(uint32_t addr, float v)
{
    asm volatile("st.shared::cluster.f32 [%0], %1;\n" ::"r"(addr), "f"(v) : "memory");
}
// Shared-memory address `addr` of this CTA mapped to CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_shared_addr(uint32_t addr, uint32_t rank)
{
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(out) : "r"(addr), "r"(rank));
    return out;
}
__device__ __forceinline__ void st_shared_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}


// ---------------------------------------------------------------- numerics
__device__ __forceinline__ float bf16_bits_to_float(uint32_t b16) { return __uint_as_float(b16 << 16); }

__device__ __forceinline__ float f16_bits_to_float(uint16_t b)
{
    float f;
    asm("cvt.f32.f16 %0, %1;\n" : "=f"(f) : "h"(b));
    return f;
}

// Two floats -> packed fp16x2 (round to nearest even); lo in bits 0..15.
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two floats -> packed bf16x2 (round to nearest even); lo in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf162(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// float -> bf16 bits, round to nearest even.
__device__ __forceinline__ uint16_t float_to_bf16_bits(float v)
{
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;\n" : "=h"(r) : "f"(v));
    return r;
}

// True if |v| would round to an fp16 infinity (or v is not finite).
__device__ __forceinline__ bool beyond_f16(float v) { return !(fabsf(v) < 65520.0f); }

}  // namespace lb

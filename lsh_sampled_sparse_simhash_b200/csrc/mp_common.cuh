// Shared device helpers of the sm_100a LSH-sampled decode-attention library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "magicpig.h"

namespace mp {

constexpr int kHeadDim = 128;
constexpr int kMaxGroup = 8;
constexpr int kSplitsK8 = 8;       // byte codes: tables l = ts, ts + 8, ... per split
constexpr int kSplitsPlanes = 8;   // bit planes: tables l = ts, ts + 8, ... per split (a warp each)
constexpr int kChunkBytes = 512;   // scan chunk (tokens) for byte codes: 32 groups x 16 tokens
constexpr int kChunkPlanes = 1024; // scan chunk (tokens) for bit planes: 32 words of 32 tokens

struct Shape {
    int B, Hq, Hkv, G, d, Ncap, K, L, LK, sink, window;
    int planes;  // 1: bit-plane codes, 0: one byte per (table, token)
};

inline int chunk_tokens(const Shape &s) { return s.planes ? kChunkPlanes : kChunkBytes; }

// Device-side status word: the first error wins, later ones are dropped.
__device__ __forceinline__ void set_status(int32_t *status, int32_t code)
{
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_lo(uint32_t packed) { return __uint_as_float(packed << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t packed) { return __uint_as_float(packed & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// Programmatic dependent launch: block until the preceding kernel in the
// stream has completed and its memory is visible, then let the next kernel
// start launching.  Both are no-ops for a kernel launched without the
// programmatic-serialization attribute.
__device__ __forceinline__ void grid_dependency_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// The two halves, for a kernel with work that does not depend on its
// immediate predecessor.  The kernels of this library let their successor
// launch only after their own wait has returned (the query hash only at its
// very end, after clearing the status words and ready flags), so when a
// kernel starts, all stream work before its predecessor is complete and
// visible: code before grid_wait() may read that (cached codes, lengths), but
// nothing its predecessor writes.  Two exceptions, each with its own
// ordering: the collision scan lets the attention launch as soon as it starts
// (the attention then waits per chunk on the scan's ready flags, not on the
// scan grid), and the attention lets the merge launch once its own flags are
// in (the merge waits for the whole attention grid before reading).
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global->shared copy; src_bytes = 0 zero-fills the destination.
__device__ __forceinline__ void cp_async_16(void *smem_dst, const void *gmem_src, int src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem_dst)),
                 "l"(gmem_src), "r"(src_bytes));
}
// The same with a 32-bit shared-memory address.
__device__ __forceinline__ void cp_async_16_s(uint32_t smem_dst, const void *gmem_src, int src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_dst), "l"(gmem_src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldmatrix_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                                            const void *smem_row)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(smem_row)));
}

// D(16x8, fp32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float &d0, float &d1, float &d2, float &d3, uint32_t a0,
                                               uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d0), "+f"(d1), "+f"(d2), "+f"(d3)
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------ mbarriers, bulk copies ----
// Every spin on an mbarrier in this library gives up after kWaitLimitNs of
// %globaltimer, records MP_ERR_CUDA in the status word and lets the kernel
// wind down instead of hanging.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t a, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t a, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t a)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(a) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t a, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait for phase `parity` of mbarrier `a`: false once kWaitLimitNs
// has passed.  The first test is inline, the polling loop out of line.
static __device__ __noinline__ bool mbar_wait_bounded_slow(uint32_t a, uint32_t parity)
{
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(a, parity))
        if (globaltimer() - t0 > kWaitLimitNs) return false;
    return true;
}
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t a, uint32_t parity)
{
    return mbar_try_wait(a, parity) || mbar_wait_bounded_slow(a, parity);
}

// Per-chunk ready flags between the collision scan and the attention (see
// attend_kernel): a release store after the chunk's list is written, an
// acquire load before it is read.
__device__ __forceinline__ int ld_acquire_gpu(const int32_t *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(int32_t *p, int v)
{
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Bounded wait for a nonzero flag: false once kWaitLimitNs has passed.
static __device__ __noinline__ bool flag_wait_bounded_slow(const int32_t *p)
{
    const uint64_t t0 = globaltimer();
    while (ld_acquire_gpu(p) == 0) {
        if (globaltimer() - t0 > kWaitLimitNs) return false;
        __nanosleep(128);
    }
    return true;
}
__device__ __forceinline__ bool flag_wait_bounded(const int32_t *p)
{
    return ld_acquire_gpu(p) != 0 || flag_wait_bounded_slow(p);
}

// Orders this thread's earlier generic-proxy shared-memory accesses before its
// later async-proxy ones (a buffer that was read is about to be refilled).
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

}  // namespace mp

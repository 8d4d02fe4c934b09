// tma_util.cuh -- sm_100a tensor-memory-accelerator (TMA) loads, mbarriers and
// named barriers, in inline PTX.
//
// Only plain (non-multicast) TMA loads are issued: every tile is fetched by
// the CTA that uses it, from this GPU's own memory.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace bimamba {

// Error word of the library on each device (bit flags, see kErr*).  A wait
// that gives up sets a bit here instead of hanging; the host reads it with
// bimamba_device_error().
__device__ unsigned int g_device_error;
constexpr unsigned kErrTmaTimeout = 1u;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async proxy (TMA unit).
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Plain arrival (no transaction bytes) of the calling thread.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for phase `parity` of the barrier to complete, for at most about
// `limit_cycles` SM clocks.  On timeout the device error word records it and
// the caller carries on (its data is then garbage, but every thread still
// reaches every later barrier, so the kernel ends).
__device__ __forceinline__ void mbar_wait_bounded(uint64_t* bar, uint32_t parity, long long limit_cycles) {
    if (mbar_try_wait(bar, parity)) return;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit_cycles) {
            atomicOr(&g_device_error, kErrTmaTimeout);
            return;
        }
    }
}

// A segment's conv halo written over the zeros that a TMA x tile holds
// outside the sequence: rows r0 .. r0+2 of the tile (row stride xw
// elements), columns col0 + [0, nch) = channels d0 + [0, nch), from halo_b
// ([3][D], rows in token order).  One warp; the proxy fence orders these
// generic-proxy writes before a later TMA refill of the same stage, and the
// warp sync before the warp's own reads of the tile.
template <typename T>
__device__ __forceinline__ void put_conv_halo(T* tile, int xw, int r0, int col0, int d0, int nch, const T* halo_b,
                                              int D, int lane) {
    for (int e = lane; e < 3 * nch; e += 32) {
        const int q = e / nch, c = e % nch;
        if (d0 + c < D) tile[(r0 + q) * xw + col0 + c] = halo_b[(int64_t)q * D + d0 + c];
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
}

// 3-D tiled TMA load into shared memory, completing on `bar` (transaction
// bytes).  Coordinates are element indices, innermost first; a box that
// reaches outside the tensor reads zeros there.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
        "[%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// 2-D tiled TMA load into shared memory, completing on `bar` (transaction
// bytes); c0 is the inner (contiguous) coordinate.  A box reaching outside the
// tensor reads zeros there.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// Asynchronous global -> shared copy of BYTES (4, 8 or 16; both addresses
// aligned to BYTES); with pred false nothing is read and zeros are written.
template <int BYTES>
__device__ __forceinline__ void cp_async(void* dst, const void* src, bool pred) {
    static_assert(BYTES == 4 || BYTES == 8 || BYTES == 16, "cp.async size");
    const int n = pred ? BYTES : 0;
    if constexpr (BYTES == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(n)
                     : "memory");
    else if constexpr (BYTES == 8)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(n)
                     : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(n)
                     : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
// Wait until at most N of this thread's committed copy groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait_pending() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace bimamba

// proj.cuh -- the mixer layer's neighbours ("DiffuMamba: High-Throughput
// Diffusion LMs with Mamba Backbone", App. A.1 Eq. (10)-(11) and Table 12):
// the timestep-conditioned AdaLN in front of the mixer, the input projection
// that produces the layer's inputs, and the output projection after it.
//
// AdaLN (Eq. (10)): out = gamma_b * (x - mu(x)) / sigma(x) + beta_b per token
// row, gamma and beta per batch row, sigma = sqrt(var + eps); one warp per
// row, fp32 statistics (the mean, then the centred squares, over the row held
// in registers).
//
// The projections are one GEMM kernel on the tcgen05 tensor cores:
// C[m][n] = sum_k A[m][k] W[n][k], bf16 operands, fp32 accumulation in TMEM,
// bf16 results, in 128 x 256 tiles: a producer thread streams 128 x 64 A and
// 256 x 64 W tiles by TMA (128-byte swizzle) through a 4-stage shared-memory
// ring, one thread issues the MMAs of each stage (4 x K = 16) and frees the
// stage by tcgen05.commit, and four epilogue warps drain the accumulator --
// persistent CTAs with two accumulators, so that a tile's stores overlap the
// next tile's products.  Every wait is bounded.  The epilogue either writes C as is
// (output projection: A is the layer's gated output) or scatters each 8-column
// group straight into the mixer's input arrays (input projection: columns
// [x | z | dt_f | dt_b | B_f | C_f | B_b | C_b]), so the layer reads them with
// no split or copy in between.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "tcgen05_util.cuh"
#include "tma_util.cuh"

namespace bimamba {

// ---------------------------------------------------------------- AdaLN

// One warp per token row, 8 rows per CTA of 256 threads: lane l holds the
// 16-byte chunks l, l + 32, ... (CPL of them, d <= 256 CPL) in registers, so
// the mean, the centred sum of squares and the output need one read of the
// row and warp shuffles only.  The chunks stay packed bf16 and are widened
// at each of the three uses (exact), so that a thread needs 4 registers per
// chunk rather than 8: up to d = 2048, 64 registers a thread and 32 rows
// (warps) resident per SM keep twice as many rows' loads in flight.
// d % 8 == 0; batch row = row / L.
// Widening as opaque single instructions: the compiler would otherwise keep
// the widened fp32 row from the first use to the last (the 8 registers a
// chunk that packing saves).
__device__ __forceinline__ float bf16_lo(uint32_t w) {
    uint32_t o;
    asm volatile("shl.b32 %0, %1, 16;" : "=r"(o) : "r"(w));
    return __uint_as_float(o);
}
__device__ __forceinline__ float bf16_hi(uint32_t w) {
    uint32_t o;
    asm volatile("and.b32 %0, %1, 0xffff0000;" : "=r"(o) : "r"(w));
    return __uint_as_float(o);
}

template <int CPL>
__global__ void __launch_bounds__(256, CPL <= 8 ? 4 : 1) adaln_kernel(const __nv_bfloat16* x, const float* gamma, const float* beta,
                                                    __nv_bfloat16* out, int64_t rows, int64_t L, int d, float eps) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const __nv_bfloat16* xr = x + row * d;
    uint4 q[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const int c = 8 * (lane + 32 * i);
        q[i] = c < d ? *reinterpret_cast<const uint4*>(xr + c) : make_uint4(0u, 0u, 0u, 0u);
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const uint32_t w4[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
        for (int u = 0; u < 4; ++u) s += bf16_lo(w4[u]) + bf16_hi(w4[u]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    const float mu = s / (float)d;
    float q2 = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        if (8 * (lane + 32 * i) < d) {
            const uint32_t w4[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float e0 = bf16_lo(w4[u]) - mu, e1 = bf16_hi(w4[u]) - mu;
                q2 = fmaf(e0, e0, q2);
                q2 = fmaf(e1, e1, q2);
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) q2 += __shfl_xor_sync(0xffffffffu, q2, off);
    const float rstd = rsqrtf(q2 / (float)d + eps);
    const int64_t b = row / L;
    const float* g = gamma + b * d;
    const float* be = beta + b * d;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const int c = 8 * (lane + 32 * i);
        if (c >= d) continue;
        const float4 g0 = *reinterpret_cast<const float4*>(g + c), g1 = *reinterpret_cast<const float4*>(g + c + 4);
        const float4 b0 = *reinterpret_cast<const float4*>(be + c), b1 = *reinterpret_cast<const float4*>(be + c + 4);
        const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
        const uint32_t w4[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
        uint32_t o4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float a0 = fmaf(gg[2 * u], (bf16_lo(w4[u]) - mu) * rstd, bb[2 * u]);
            const float a1 = fmaf(gg[2 * u + 1], (bf16_hi(w4[u]) - mu) * rstd, bb[2 * u + 1]);
            const __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
            o4[u] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(out + row * d + c) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
}

// ---------------------------------------------------------------- GEMM

constexpr int kGemmBM = 128, kGemmBN = 256, kGemmBK = 64, kGemmStages = 4;
constexpr int kGemmATile = kGemmBM * kGemmBK * 2;    // 16 KB
constexpr int kGemmBTile = kGemmBN * kGemmBK * 2;    // 32 KB
constexpr int kGemmStage = kGemmATile + kGemmBTile;  // 48 KB
constexpr int kGemmBarOff = kGemmStages * kGemmStage;
constexpr int kGemmSmem = kGemmBarOff + 128 + 1024;  // barriers + TMEM slot, and 1024-byte alignment slack

struct GemmParams {
    int M, N, K;
    int scatter;              // 0: C [M][N]; 1: the mixer's input arrays
    __nv_bfloat16* C;
    // scatter: x, z [M][D]; dt [2][M][D]; Bm, Cm [2][M][Ns]
    __nv_bfloat16 *x, *z, *dt, *Bm, *Cm;
    int D, Ns;
    long long wait_limit;
};

// 8 results (columns n .. n+7 of row m) to their place.
__device__ __forceinline__ void gemm_store8(const GemmParams& p, int m, int n, const float* v) {
    uint32_t w4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * u], v[2 * u + 1]);
        w4[u] = *reinterpret_cast<const uint32_t*>(&h);
    }
    __nv_bfloat16* dst;
    if (!p.scatter) {
        dst = p.C + (int64_t)m * p.N + n;
    } else {
        const int64_t M = p.M, D = p.D, Ns = p.Ns;
        if (n < 2 * D) {
            dst = (n < D ? p.x + m * D + n : p.z + m * D + (n - D));
        } else if (n < 4 * D) {
            const int r = n < 3 * D ? 0 : 1;
            dst = p.dt + (r * M + m) * D + (n - (2 + r) * D);
        } else {
            const int j = n - 4 * (int)D, seg = j / (int)Ns, c = j % (int)Ns;  // B_f, C_f, B_b, C_b
            __nv_bfloat16* base = (seg & 1) ? p.Cm : p.Bm;
            dst = base + ((int64_t)(seg >> 1) * M + m) * Ns + c;
        }
    }
    *reinterpret_cast<uint4*>(dst) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
}

// C = A W^T as a persistent kernel: grid = min(tiles, SMs), block 192, dynamic
// shared memory kGemmSmem.  mapA: [M][K] bf16, box {64, 128}; mapW: [N][K]
// bf16, box {64, 256}; both 128-byte swizzled.  K % 64 == 0; N % 8 == 0.
// Warp 0 (one thread) streams the A / W tiles of every K step of every tile
// this CTA owns (tiles blockIdx.x, blockIdx.x + gridDim.x, ...) through the
// ring; warp 1 (one thread) issues the MMAs into one of two TMEM accumulators
// (2 x 256 columns) and commits "accumulator full"; warps 2-5 drain the other
// accumulator -- warp w reads TMEM lanes 32 (w % 4) .. +31 -- and hand it back
// ("accumulator empty", one arrival per warp), so a tile's stores overlap the
// next tile's products.  Tiles are taken in the banded order of
// gemm_tile_origin.  Every wait is bounded.
constexpr int kGemmPThreads = 192;
constexpr int kGemmBand = 64;  // M tiles per band of the tile order

// Tile t of the persistent order -> (m0, n0).  Tiles run M-fastest inside
// bands of kGemmBand M tiles, band after band: the CTAs of one wave share a
// few W column slices (each read from DRAM once per band) and a band's A
// rows (kGemmBand x 128 rows) stay in L2 while the band sweeps N.
__device__ __forceinline__ void gemm_tile_origin(int t, int tiles_m, int tiles_n, int& m0, int& n0) {
    const int per_band = kGemmBand * tiles_n;
    const int band = t / per_band, r = t % per_band;
    const int bm = min(kGemmBand, tiles_m - band * kGemmBand);  // M tiles in this band
    m0 = (band * kGemmBand + r % bm) * kGemmBM;
    n0 = (r / bm) * kGemmBN;
}

__global__ void __launch_bounds__(kGemmPThreads, 1) gemm_bf16_persistent_kernel(
    const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapW, const GemmParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(base + kGemmBarOff);
    uint64_t* empty = full + kGemmStages;
    uint64_t* acc_full = empty + kGemmStages;  // [2]
    uint64_t* acc_empty = acc_full + 2;        // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int nk = p.K / kGemmBK;
    const int tiles_n = (p.N + kGemmBN - 1) / kGemmBN;
    const int tiles_m = (p.M + kGemmBM - 1) / kGemmBM;
    const int tiles = tiles_n * tiles_m;

    if (t == 0) {
        for (int i = 0; i < 2 * kGemmStages + 2; ++i) mbar_init(full + i, 1);
        mbar_init(acc_empty, 4);
        mbar_init(acc_empty + 1, 4);
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc<512>(tmem_slot);
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (t == 0) {  // producer
        int g = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            int m0, n0;
            gemm_tile_origin(tile, tiles_m, tiles_n, m0, n0);
            for (int kt = 0; kt < nk; ++kt, ++g) {
                const int s = g % kGemmStages;
                if (g >= kGemmStages) mbar_wait_bounded(empty + s, (uint32_t)(((g / kGemmStages) - 1) & 1), p.wait_limit);
                unsigned char* st = base + s * kGemmStage;
                mbar_arrive_expect_tx(full + s, kGemmStage);
                tma_load_2d(st, &mapA, full + s, kt * kGemmBK, m0);
                tma_load_2d(st + kGemmATile, &mapW, full + s, kt * kGemmBK, n0);
            }
        }
    } else if (t == 32) {  // MMA issuer
        constexpr uint32_t idesc = umma_idesc_bf16(kGemmBM, kGemmBN);
        int g = 0, i = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++i) {
            const int acc = i & 1;
            if (i >= 2) mbar_wait_bounded(acc_empty + acc, (uint32_t)(((i >> 1) - 1) & 1), p.wait_limit);
            tmem_fence_after_sync();
            const uint32_t d = tmem + 256 * acc;
            for (int kt = 0; kt < nk; ++kt, ++g) {
                const int s = g % kGemmStages;
                mbar_wait_bounded(full + s, (uint32_t)((g / kGemmStages) & 1), p.wait_limit);
                tmem_fence_after_sync();
                const uint32_t a = smem_addr(base + s * kGemmStage), w = a + kGemmATile;
#pragma unroll
                for (int kk = 0; kk < kGemmBK / 16; ++kk)
                    umma_f16(d, umma_desc_sw128(a + 32 * kk), umma_desc_sw128(w + 32 * kk), idesc, kt > 0 || kk > 0);
                umma_commit(empty + s);
            }
            umma_commit(acc_full + acc);
        }
    } else if (warp >= 2) {  // epilogue
        const int q = warp & 3;  // TMEM lane quadrant of this warp
        const uint32_t lb = (uint32_t)(32 * q) << 16;
        int i = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++i) {
            const int acc = i & 1;
            int m0, n0;
            gemm_tile_origin(tile, tiles_m, tiles_n, m0, n0);
            mbar_wait_bounded(acc_full + acc, (uint32_t)((i >> 1) & 1), p.wait_limit);
            tmem_fence_after_sync();
            const int m = m0 + 32 * q + lane;
#pragma unroll 1
            for (int c = 0; c < kGemmBN / 32; ++c) {
                float v[32];
                tmem_ld32(tmem + 256 * acc + lb + 32 * c, v);
                if (m < p.M) {
#pragma unroll
                    for (int gq = 0; gq < 4; ++gq) {
                        const int n = n0 + 32 * c + 8 * gq;
                        if (n < p.N) gemm_store8(p, m, n, v + 8 * gq);
                    }
                }
            }
            tmem_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty + acc);
        }
    }
    __syncwarp();
    tmem_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc<512>(tmem);
}

}  // namespace bimamba

// bimamba_api.cu -- the C ABI (include/bimamba.h): argument checks, launch
// shapes and kernel dispatch.  All arithmetic lives in scan_kernels.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <set>
#include <type_traits>
#include <utility>

#include "bimamba.h"
#include "block_fused.cuh"
#include "carry.cuh"
#include "context_cache.h"
#include "layer_fused.cuh"
#include "layer_pscan.cuh"
#include "layer_tma.cuh"
#include "mamba2.cuh"
#include "mamba2_ssd.cuh"
#include "mamba2_block.cuh"
#include "proj.cuh"
#include "scan_kernels.cuh"

namespace {

using bimamba::KParams;
using bf16 = __nv_bfloat16;

constexpr int kT = 16;       // tokens per chunk (full layer, prefix)
constexpr int kWPD = 4;      // warps per direction per CTA (full layer)
constexpr int kWPB = 8;      // warps per CTA (prefix, block step)
// lanes sharing B across channels in the fused prefix kernel (measured best
// at batch 16 x 4096 channels: 2 is 3 % ahead of 4, 8 % ahead of 1 and 8;
// with the token loop unrolled by 4, 25.8 ms against 26.8 for 1 lane)
#ifndef BIMAMBA_PREFIX_GROUP
#define BIMAMBA_PREFIX_GROUP 2
#endif
constexpr int kPrefixGroup = BIMAMBA_PREFIX_GROUP;
constexpr int kTBlock = 64;  // longest block of the block step
constexpr int kMaxBatch = 65535;
constexpr long long kWaitCycles = 4000000000LL;   // ~2 s at 1.965 GHz
constexpr long long kStarveWaitCycles = 200000LL;  // ~0.1 ms: the starved test gives up fast

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t elem_size(bimamba_dtype_t t) { return t == BIMAMBA_F32 ? 4 : 2; }

bool dtype_ok(int t) { return t == BIMAMBA_F32 || t == BIMAMBA_BF16; }

// Raise the dynamic shared-memory limit of a kernel once per device.
int ensure_smem(const void* fn, size_t bytes) {
    if (bytes <= 48 * 1024) return BIMAMBA_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BIMAMBA_ERR_CUDA;
    static std::mutex mu;
    static std::set<std::pair<const void*, int>> done;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({fn, dev})) return BIMAMBA_OK;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return BIMAMBA_ERR_CUDA;
    done.insert({fn, dev});
    return BIMAMBA_OK;
}

int launch_status() {
    return cudaGetLastError() == cudaSuccess ? BIMAMBA_OK : BIMAMBA_ERR_CUDA;
}

// Lanes per channel: the smallest power of two that gives about one resident
// thread slot per SM thread (148 SMs x 1024), at most 8.
int pick_lanes(int64_t chains, unsigned flags) {
    const unsigned forced = (flags & BIMAMBA_LANES_MASK) >> BIMAMBA_LANES_SHIFT;
    if (forced) return (int)forced;
    const int64_t target = 148LL * 1024;
    int g = 1;
    while (g < 8 && chains * g < target) g *= 2;
    return g;
}

bool lanes_ok(unsigned flags) {
    const unsigned f = (flags & BIMAMBA_LANES_MASK) >> BIMAMBA_LANES_SHIFT;
    return f == 0 || f == 1 || f == 2 || f == 4 || f == 8 || f == 16;
}

int check_params(const bimamba_params_t* p) {
    if (!p || !p->A || !p->D || !p->dt_bias || !p->conv_w) return BIMAMBA_ERR_INVALID_ARG;
    if (!aligned(p->A, 4) || !aligned(p->D, 4) || !aligned(p->dt_bias, 4) || !aligned(p->conv_w, 4) ||
        (p->conv_b && !aligned(p->conv_b, 4)))
        return BIMAMBA_ERR_MISALIGNED;
    return BIMAMBA_OK;
}

void fill_params(KParams& k, const bimamba_params_t* p) {
    k.A = p->A;
    k.Dskip = p->D;
    k.dt_bias = p->dt_bias;
    k.conv_w = p->conv_w;
    k.conv_b = p->conv_b;
}

// ---- full layer dispatch

template <int G, typename Tin, typename Tout>
int launch_layer(const KParams& k, cudaStream_t st) {
    constexpr int CW = kWPD * (32 / G);
    const void* fn = reinterpret_cast<const void*>(&bimamba::layer_kernel<G, kT, kWPD, Tin, Tout>);
    const size_t smem = sizeof(float) * bimamba::layer_smem_floats<G, kT, kWPD>();
    int rc = ensure_smem(fn, smem);
    if (rc) return rc;
    dim3 grid((unsigned)((k.D + CW - 1) / CW), (unsigned)k.batch);
    bimamba::layer_kernel<G, kT, kWPD, Tin, Tout><<<grid, 2 * kWPD * 32, smem, st>>>(k);
    return launch_status();
}

template <typename Tin, typename Tout>
int layer_by_lanes(int g, const KParams& k, cudaStream_t st) {
    switch (g) {
        case 1: return launch_layer<1, Tin, Tout>(k, st);
        case 2: return launch_layer<2, Tin, Tout>(k, st);
        case 4: return launch_layer<4, Tin, Tout>(k, st);
        case 8: return launch_layer<8, Tin, Tout>(k, st);
        case 16: return launch_layer<16, Tin, Tout>(k, st);
    }
    return BIMAMBA_ERR_UNSUPPORTED;
}

// ---- prefix dispatch

template <int G, typename Tin>
int launch_prefix(const KParams& k, cudaStream_t st) {
    constexpr int CW = kWPB * (32 / G);
    const void* fn = reinterpret_cast<const void*>(&bimamba::prefix_kernel<G, kT, kWPB, Tin>);
    const size_t smem = sizeof(float) * bimamba::prefix_smem_floats<G, kT, kWPB>();
    int rc = ensure_smem(fn, smem);
    if (rc) return rc;
    dim3 grid((unsigned)((k.D + CW - 1) / CW), (unsigned)k.batch);
    bimamba::prefix_kernel<G, kT, kWPB, Tin><<<grid, kWPB * 32, smem, st>>>(k);
    return launch_status();
}

template <typename Tin>
int prefix_by_lanes(int g, const KParams& k, cudaStream_t st) {
    switch (g) {
        case 1: return launch_prefix<1, Tin>(k, st);
        case 2: return launch_prefix<2, Tin>(k, st);
        case 4: return launch_prefix<4, Tin>(k, st);
        case 8: return launch_prefix<8, Tin>(k, st);
        case 16: return launch_prefix<16, Tin>(k, st);
    }
    return BIMAMBA_ERR_UNSUPPORTED;
}

// ---- block-step dispatch

template <int G, int TB, typename Tin, typename Tout>
int launch_block(const KParams& k, cudaStream_t st) {
    constexpr int CW = kWPB * (32 / G);
    const void* fn = reinterpret_cast<const void*>(&bimamba::block_kernel<G, TB, kWPB, Tin, Tout>);
    const size_t smem = sizeof(float) * bimamba::block_smem_floats<G, TB, kWPB>();
    int rc = ensure_smem(fn, smem);
    if (rc) return rc;
    dim3 grid((unsigned)((k.D + CW - 1) / CW), (unsigned)k.batch);
    bimamba::block_kernel<G, TB, kWPB, Tin, Tout><<<grid, kWPB * 32, smem, st>>>(k);
    return launch_status();
}

// The whole block is one chunk held in registers, so at least 4 lanes share
// a channel (at most 16 tokens per lane); blocks of up to 32 tokens use the
// smaller shared-memory footprint.
template <typename Tin, typename Tout>
int block_by_lanes(int g, const KParams& k, cudaStream_t st) {
    if (g < 4) g = 4;
    if (k.L <= 32) {
        switch (g) {
            case 4: return launch_block<4, 32, Tin, Tout>(k, st);
            case 8: return launch_block<8, 32, Tin, Tout>(k, st);
            case 16: return launch_block<16, 32, Tin, Tout>(k, st);
        }
    } else {
        switch (g) {
            case 4: return launch_block<4, kTBlock, Tin, Tout>(k, st);
            case 8: return launch_block<8, kTBlock, Tin, Tout>(k, st);
            case 16: return launch_block<16, kTBlock, Tin, Tout>(k, st);
        }
    }
    return BIMAMBA_ERR_UNSUPPORTED;
}

// ---- TMA-fed kernels

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    return fn;
}

// 3-D map over a [batch][rows][inner] row-major tensor; the box is
// {box_inner, box_rows, 1}; out-of-range elements of a box read as zero.
bool map3d(CUtensorMap* m, const void* ptr, bool is_bf16, uint64_t inner, uint64_t rows, uint64_t batch,
           uint32_t box_inner, uint32_t box_rows) {
    EncodeTiledFn f = encode_tiled();
    if (!f) return false;
    const uint64_t esz = is_bf16 ? 2 : 4;
    cuuint64_t dims[3] = {inner, rows, batch};
    cuuint64_t strides[2] = {inner * esz, inner * rows * esz};
    cuuint32_t box[3] = {box_inner, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return f(m, is_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
             const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tma_eligible(const bimamba_inputs_t* in, int d_inner, bool need_reverse, bool need_z_c) {
    const size_t esz = elem_size(in->dtype);
    if ((d_inner * esz) % 16 != 0) return false;
    const void* ptrs[8] = {in->x, in->dt[0], in->B[0], need_z_c ? in->z : in->x, need_z_c ? in->C[0] : in->x,
                           need_reverse ? in->dt[1] : in->x, need_reverse ? in->B[1] : in->x,
                           need_reverse ? in->C[1] : in->x};
    for (const void* q : ptrs)
        if (!aligned(q, 16)) return false;
    return true;
}

constexpr int kTWD = 4;  // warps per direction per CTA
constexpr int kTNS = 2;  // pipeline stages

// The layer's workspace: the directions' fp32 partial outputs [batch][L][D],
// then (256-byte aligned) the fp32 B/C quads [2][batch][L][32] of the
// chunked kernel at 8 lanes per channel.
size_t layer_ws_bcq_offset(int batch, int64_t L, int d_inner) {
    return ((size_t)batch * (size_t)L * (size_t)d_inner * sizeof(float) + 255) & ~static_cast<size_t>(255);
}
size_t layer_ws_bcq_bytes(int batch, int64_t L) {
    return 2 * (size_t)batch * (size_t)L * 2 * bimamba::kNState * sizeof(float);
}

template <int G, int T, typename Tin, int NWD = kTWD>
bool fill_maps(bimamba::LayerMaps& m, const bimamba_inputs_t* in, int batch, int64_t L, int D, bool reverse,
               bool gated) {
    using Ge = bimamba::TmaGeo<G, T, NWD, kTNS, Tin>;
    const bool bf = std::is_same<Tin, bf16>::value;
    bool ok = map3d(&m.x, in->x, bf, D, L, batch, Ge::XW, T + 3);
    ok = ok && map3d(&m.dt[0], in->dt[0], bf, D, L, batch, Ge::XW, T);
    ok = ok && map3d(&m.B[0], in->B[0], bf, bimamba::kNState, L, batch, bimamba::kNState, T);
    if (gated) {
        ok = ok && map3d(&m.z, in->z, bf, D, L, batch, Ge::XW, T);
        ok = ok && map3d(&m.C[0], in->C[0], bf, bimamba::kNState, L, batch, bimamba::kNState, T);
    } else {
        m.z = m.x;
        m.C[0] = m.B[0];
    }
    if (reverse) {
        ok = ok && map3d(&m.dt[1], in->dt[1], bf, D, L, batch, Ge::XW, T);
        ok = ok && map3d(&m.B[1], in->B[1], bf, bimamba::kNState, L, batch, bimamba::kNState, T);
        ok = ok && map3d(&m.C[1], in->C[1], bf, bimamba::kNState, L, batch, bimamba::kNState, T);
    } else {
        m.dt[1] = m.dt[0];
        m.B[1] = m.B[0];
        m.C[1] = m.C[0];
    }
    return ok;
}

// Both directions' B and C widened to fp32 quads into k.bcq (one small
// launch), and the two tensor maps over them (boxes of T tokens) in maps_b.
template <typename Tin>
int widen_bc(const KParams& k, int T, CUtensorMap* maps_b, cudaStream_t st) {
    const int64_t rows = 2 * (int64_t)k.batch * k.L;
    const int64_t blocks = (rows + 255) / 256;
    bimamba::widen_bc_kernel<Tin><<<(unsigned)(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, st>>>(k);
    if (cudaGetLastError() != cudaSuccess) return BIMAMBA_ERR_CUDA;
    const size_t per_dir = (size_t)k.batch * (size_t)k.L * 2 * bimamba::kNState;
    for (int r = 0; r < 2; ++r)
        if (!map3d(&maps_b[r], k.bcq + r * per_dir, false, 2 * bimamba::kNState, (uint64_t)k.L, (uint64_t)k.batch,
                   2 * bimamba::kNState, (uint32_t)T))
            return BIMAMBA_ERR_CUDA;
    return BIMAMBA_OK;
}

// BCQ: B and C widened to fp32 quads in the workspace first (one small
// launch), then read by TMA in the layout the states use, with no widening in
// the scan loop.
template <int G, int T, typename Tin, typename Tout, bool CARRY = false, int NWD = kTWD, bool DIRECT = false,
          bool FULL_UNROLL = false, bool BCQ = false>
int launch_layer_tma(const KParams& k, const bimamba_inputs_t* in, cudaStream_t st) {
    using Ge = bimamba::TmaGeo<G, T, NWD, kTNS, Tin, DIRECT, BCQ>;
    bimamba::LayerMaps maps;
    if (!fill_maps<G, T, Tin, NWD>(maps, in, k.batch, k.L, k.D, true, true)) return BIMAMBA_ERR_CUDA;
    if constexpr (BCQ) {
        int rc = widen_bc<Tin>(k, T, maps.B, st);
        if (rc) return rc;
    }
    auto kern = &bimamba::layer_tma_kernel<G, T, NWD, kTNS, Tin, Tout, CARRY, DIRECT, FULL_UNROLL, BCQ>;
    int rc = ensure_smem(reinterpret_cast<const void*>(kern), Ge::SMEM);
    if (rc) return rc;
    dim3 grid((unsigned)((k.D + Ge::CW - 1) / Ge::CW), (unsigned)k.batch);
    kern<<<grid, 2 * NWD * 32, Ge::SMEM, st>>>(maps, k);
    return launch_status();
}

// With carries: 16-token chunks at 4 lanes per channel, 32 at 8 and 16 (the
// automatic choice; the chunk flag is not honoured).
template <typename Tin, typename Tout>
int layer_tma_carry_by_lanes(int g, const KParams& k, const bimamba_inputs_t* in, cudaStream_t st) {
    switch (g) {
        case 4: return launch_layer_tma<4, 16, Tin, Tout, true>(k, in, st);
        case 8: return launch_layer_tma<8, 32, Tin, Tout, true>(k, in, st);
        case 16: return launch_layer_tma<16, 32, Tin, Tout, true>(k, in, st);
    }
    return BIMAMBA_ERR_UNSUPPORTED;
}

template <typename Tin, typename Tout>
int layer_tma_by_lanes(int g, int t, const KParams& k, const bimamba_inputs_t* in, cudaStream_t st) {
    if (t == 16) {
        switch (g) {
            case 4: return launch_layer_tma<4, 16, Tin, Tout>(k, in, st);
            case 8: return launch_layer_tma<8, 16, Tin, Tout>(k, in, st);
            case 16: return launch_layer_tma<16, 16, Tin, Tout>(k, in, st);
        }
    } else {
        switch (g) {
            case 4: return launch_layer_tma<4, 32, Tin, Tout>(k, in, st);
            case 8: return launch_layer_tma<8, 32, Tin, Tout>(k, in, st);
            case 16: return launch_layer_tma<16, 32, Tin, Tout>(k, in, st);
        }
    }
    return BIMAMBA_ERR_UNSUPPORTED;
}

template <int G, typename Tin>
int launch_prefix_tma(const KParams& k, const bimamba_inputs_t* in, cudaStream_t st) {
    constexpr int T = 32;
    using Ge = bimamba::TmaGeo<G, T, kTWD, kTNS, Tin>;
    bimamba::LayerMaps maps;
    if (!fill_maps<G, T, Tin>(maps, in, k.batch, k.L, k.D, false, false)) return BIMAMBA_ERR_CUDA;
    auto kern = &bimamba::prefix_tma_kernel<G, T, kTWD, kTNS, Tin>;
    int rc = ensure_smem(reinterpret_cast<const void*>(kern), Ge::SMEM);
    if (rc) return rc;
    dim3 grid((unsigned)((k.D + Ge::CW - 1) / Ge::CW), (unsigned)k.batch);
    kern<<<grid, kTWD * 32, Ge::SMEM, st>>>(maps, k);
    return launch_status();
}

template <typename Tin>
int prefix_tma_by_lanes(int g, const KParams& k, const bimamba_inputs_t* in, cudaStream_t st) {
    switch (g) {
        case 4: return launch_prefix_tma<4, Tin>(k, in, st);
        case 8: return launch_prefix_tma<8, Tin>(k, in, st);
        case 16: return launch_prefix_tma<16, Tin>(k, in, st);
    }
    return BIMAMBA_ERR_UNSUPPORTED;
}

// ---- chunked parallel scan (few channels: 8 pieces of 8 steps per channel and chunk)

constexpr int kPNS = 2;  // pipeline stages per direction

template <int NWD, typename Tin, typename Tout, bool CARRY = false>
int launch_layer_pscan(const KParams& k, const bimamba_inputs_t* in, cudaStream_t st) {
    using Ge = bimamba::PscanGeo<NWD, kPNS, Tin>;
    const bool bf = std::is_same<Tin, bf16>::value;
    constexpr int N = bimamba::kNState, T = Ge::T;
    bimamba::LayerMaps m;
    bool ok = map3d(&m.x, in->x, bf, k.D, k.L, k.batch, Ge::XW, T + 3);
    ok = ok && map3d(&m.z, in->z, bf, k.D, k.L, k.batch, Ge::XW, T);
    for (int r = 0; r < 2; ++r) {
        ok = ok && map3d(&m.dt[r], in->dt[r], bf, k.D, k.L, k.batch, Ge::XW, T);
        ok = ok && map3d(&m.B[r], in->B[r], bf, N, k.L, k.batch, N, T);
        ok = ok && map3d(&m.C[r], in->C[r], bf, N, k.L, k.batch, N, T);
    }
    if (!ok) return BIMAMBA_ERR_CUDA;
    auto kern = &bimamba::layer_pscan_kernel<NWD, kPNS, Tin, Tout, CARRY>;
    int rc = ensure_smem(reinterpret_cast<const void*>(kern), Ge::SMEM);
    if (rc) return rc;
    dim3 grid((unsigned)((k.D + Ge::CW - 1) / Ge::CW), (unsigned)k.batch);
    kern<<<grid, 2 * NWD * 32, Ge::SMEM, st>>>(m, k);
    return launch_status();
}

// ---- per-token fused kernels (many channels)

// The boxes come from the kernel's own geometry, so the bytes each TMA load
// delivers always equal what the kernel's barrier expects.
template <int G, typename Tin>
bool fill_fused_maps(bimamba::FusedMaps& m, const bimamba_inputs_t* in, int batch, int64_t L, int D, bool layer) {
    constexpr int T = bimamba::FusedGeo<G, Tin>::T, CW = bimamba::FusedGeo<G, Tin>::CW;
    const bool bf = std::is_same<Tin, bf16>::value;
    bool ok = map3d(&m.x, in->x, bf, D, L, batch, CW, T + 3);
    ok = ok && map3d(&m.dt[0], in->dt[0], bf, D, L, batch, CW, T);
    ok = ok && map3d(&m.B[0], in->B[0], bf, bimamba::kNState, L, batch, bimamba::kNState, T);
    if (layer) {
        ok = ok && map3d(&m.z, in->z, bf, D, L, batch, CW, T);
        ok = ok && map3d(&m.C[0], in->C[0], bf, bimamba::kNState, L, batch, bimamba::kNState, T);
        ok = ok && map3d(&m.dt[1], in->dt[1], bf, D, L, batch, CW, T);
        ok = ok && map3d(&m.B[1], in->B[1], bf, bimamba::kNState, L, batch, bimamba::kNState, T);
        ok = ok && map3d(&m.C[1], in->C[1], bf, bimamba::kNState, L, batch, bimamba::kNState, T);
    } else {
        m.z = m.x;
        m.C[0] = m.B[0];
        m.dt[1] = m.dt[0];
        m.B[1] = m.B[0];
        m.C[1] = m.B[0];
    }
    return ok;
}

// BCQ (one lane per channel): B and C widened to fp32 quads in the workspace
// first, then read by TMA with no per-chunk widening.
template <int G, typename Tin, typename Tout, bool CARRY = false, bool F32BC = false, bool BCQ = false>
int launch_fused_layer(const KParams& k, const bimamba_inputs_t* in, cudaStream_t st) {
    using Ge = bimamba::FusedGeo<G, Tin, F32BC, BCQ>;
    bimamba::FusedMaps maps;
    if (!fill_fused_maps<G, Tin>(maps, in, k.batch, k.L, k.D, true)) return BIMAMBA_ERR_CUDA;
    if constexpr (BCQ) {
        int rc = widen_bc<Tin>(k, (int)Ge::T, maps.B, st);
        if (rc) return rc;
    }
    auto kern = &bimamba::fused_layer_kernel<G, Tin, Tout, CARRY, F32BC, 4, BCQ>;
    int rc = ensure_smem(reinterpret_cast<const void*>(kern), Ge::SMEM);
    if (rc) return rc;
    dim3 grid((unsigned)((k.D + Ge::CW - 1) / Ge::CW), (unsigned)k.batch);
    kern<<<grid, 64, Ge::SMEM, st>>>(maps, k);
    return launch_status();
}

template <typename Tin, typename Tout>
int fused_layer_by_group(int g, bool f32bc, const KParams& k, const bimamba_inputs_t* in, cudaStream_t st) {
    if (f32bc) {
        switch (g) {
            case 2: return launch_fused_layer<2, Tin, Tout, false, true>(k, in, st);
            case 4: return launch_fused_layer<4, Tin, Tout, false, true>(k, in, st);
        }
        return BIMAMBA_ERR_UNSUPPORTED;
    }
    switch (g) {
        case 1: return launch_fused_layer<1, Tin, Tout, false, false, true>(k, in, st);
        case 2: return launch_fused_layer<2, Tin, Tout>(k, in, st);
        case 4: return launch_fused_layer<4, Tin, Tout>(k, in, st);
        case 8: return launch_fused_layer<8, Tin, Tout>(k, in, st);
    }
    return BIMAMBA_ERR_UNSUPPORTED;
}

template <int G, typename Tin>
int launch_fused_prefix(const KParams& k, const bimamba_inputs_t* in, cudaStream_t st) {
    using Ge = bimamba::FusedGeo<G, Tin>;
    bimamba::FusedMaps maps;
    if (!fill_fused_maps<G, Tin>(maps, in, k.batch, k.L, k.D, false)) return BIMAMBA_ERR_CUDA;
    auto kern = &bimamba::fused_prefix_kernel<G, Tin>;
    int rc = ensure_smem(reinterpret_cast<const void*>(kern), Ge::SMEM);
    if (rc) return rc;
    dim3 grid((unsigned)((k.D + Ge::CW - 1) / Ge::CW), (unsigned)k.batch);
    kern<<<grid, 32, Ge::SMEM, st>>>(maps, k);
    return launch_status();
}

// Kernel family of the TMA path: forced by the flags, else the per-token
// fused kernel when one lane per channel and direction still gives at least
// 8 warps per SM, otherwise the chunked kernel.
int pick_family(int64_t lanes_total, unsigned flags) {
    const unsigned f = (flags & BIMAMBA_FAMILY_MASK) >> BIMAMBA_FAMILY_SHIFT;
    if (f) return (int)f;
    return lanes_total >= 148LL * 8 * 32 ? 2 : 1;
}

// Group size of the fused kernel: one lane per channel with all 16 states
// measured fastest at batch 8, L 2048, d_inner 4096 with the token loop
// unrolled by 4 (1.096 ms against 1.122 ms for 2 lanes x 8 states, 1.175 at
// 4 and 1.276 at 8).
int pick_group_fused(unsigned flags) {
    const unsigned f = (flags & BIMAMBA_LANES_MASK) >> BIMAMBA_LANES_SHIFT;
    return f ? (int)f : 1;
}

// Chunk length of the chunked kernel: forced by the flags, else 16 tokens
// at 4 lanes per channel and 32 at 8 or 16 (the measured optimum of each:
// shared memory per CTA grows with the chunk and shrinks with the lanes).
int pick_chunk_tma(unsigned flags, int lanes) {
    const unsigned f = (flags & BIMAMBA_CHUNK_MASK) >> BIMAMBA_CHUNK_SHIFT;
    if (f) return f == 1 ? 16 : 32;
    return lanes >= 8 ? 32 : 16;
}

// Lanes per channel of the chunked kernel: 4 when that gives about one
// thread slot per SM thread (148 SMs x 1024), else 8.  16 lanes (one state
// each) measured slower than 8 even at batch 1 (10.0 ms against 7.1 ms at
// L 65536, d_inner 4096): its per-state reduction overhead outweighs the
// extra parallelism.
int pick_lanes_tma(int64_t chains, unsigned flags) {
    const unsigned forced = (flags & BIMAMBA_LANES_MASK) >> BIMAMBA_LANES_SHIFT;
    if (forced) return (int)forced;
    return chains * 4 >= 148LL * 1024 ? 4 : 8;
}

// ---- block step on the per-token fused layout (the default)

template <typename Tin, typename Tout>
int launch_fused_block(const KParams& k, cudaStream_t st) {
    auto kern = &bimamba::fused_block_kernel<Tin, Tout>;
    const size_t smem = 2 * sizeof(float) * (size_t)bimamba::block_dir_floats((int)k.L);
    int rc = ensure_smem(reinterpret_cast<const void*>(kern), 2 * sizeof(float) * bimamba::block_dir_floats(kTBlock));
    if (rc) return rc;
    dim3 grid((unsigned)((k.D + 31) / 32), (unsigned)k.batch);
    kern<<<grid, 64, smem, st>>>(k);
    return launch_status();
}

template <typename Tin, typename Tout>
int launch_async_block(const KParams& k, cudaStream_t st) {
    auto kern = &bimamba::async_block_kernel<Tin, Tout>;
    const size_t smem = (size_t)bimamba::async_block_smem<Tin>((int)k.L);
    int rc = ensure_smem(reinterpret_cast<const void*>(kern), (size_t)bimamba::async_block_smem<Tin>(kTBlock));
    if (rc) return rc;
    dim3 grid((unsigned)((k.D + 31) / 32), (unsigned)k.batch);
    kern<<<grid, 64, smem, st>>>(k);
    return launch_status();
}

// The cp.async-staged block kernel copies 16-byte pieces of 32-channel rows:
// every row must start on a 16-byte boundary.
bool async_block_eligible(const bimamba_inputs_t* in, const void* tail, int d_inner) {
    if ((d_inner * elem_size(in->dtype)) % 16 != 0) return false;
    const void* ptrs[9] = {in->x, in->z, in->dt[0], in->dt[1], in->B[0], in->B[1], in->C[0], in->C[1], tail};
    for (const void* q : ptrs)
        if (!aligned(q, 16)) return false;
    return true;
}

int check_inputs(const bimamba_inputs_t* in, bool need_reverse, bool need_z_c) {
    if (!in || !in->x || !in->dt[0] || !in->B[0]) return BIMAMBA_ERR_INVALID_ARG;
    if (need_z_c && (!in->z || !in->C[0])) return BIMAMBA_ERR_INVALID_ARG;
    if (need_reverse && (!in->dt[1] || !in->B[1] || !in->C[1])) return BIMAMBA_ERR_INVALID_ARG;
    if (!dtype_ok(in->dtype)) return BIMAMBA_ERR_UNSUPPORTED;
    const size_t a = elem_size(in->dtype);
    const void* ptrs[8] = {in->x, in->z, in->dt[0], in->dt[1], in->B[0], in->B[1], in->C[0], in->C[1]};
    for (const void* q : ptrs)
        if (q && !aligned(q, a)) return BIMAMBA_ERR_MISALIGNED;
    return BIMAMBA_OK;
}

void fill_inputs(KParams& k, const bimamba_inputs_t* in) {
    k.x = in->x;
    k.z = in->z;
    for (int r = 0; r < 2; ++r) {
        k.dt[r] = in->dt[r];
        k.B[r] = in->B[r];
        k.C[r] = in->C[r];
    }
}

}  // namespace

extern "C" {

int bimamba_abi_version(void) { return 2; }

const char* bimamba_status_string(int status) {
    switch (status) {
        case BIMAMBA_OK: return "ok";
        case BIMAMBA_ERR_INVALID_ARG: return "invalid argument (null pointer or bad size)";
        case BIMAMBA_ERR_UNSUPPORTED: return "unsupported (d_state, dtype, block length or flag)";
        case BIMAMBA_ERR_MISALIGNED: return "pointer not aligned to its element size";
        case BIMAMBA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case BIMAMBA_ERR_CUDA: return "CUDA launch or attribute call failed";
    }
    return "unknown status";
}

int bimamba_device_error(int reset) {
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, bimamba::g_device_error, sizeof(word)) != cudaSuccess) return BIMAMBA_ERR_CUDA;
    if (reset) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(bimamba::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return BIMAMBA_ERR_CUDA;
    }
    return (int)word;
}

int bimamba_features(const bimamba_inputs_t* in, const bimamba_params_t* p, int batch, int64_t L, int d_inner,
                     float* u, float* delta, void* cuda_stream) {
    if (batch <= 0 || batch > kMaxBatch || L <= 0 || d_inner <= 0 || !u || !delta) return BIMAMBA_ERR_INVALID_ARG;
    if (!in || !in->x || !in->dt[0] || !in->dt[1]) return BIMAMBA_ERR_INVALID_ARG;
    if (!dtype_ok(in->dtype)) return BIMAMBA_ERR_UNSUPPORTED;
    if (!p || !p->conv_w || !p->dt_bias) return BIMAMBA_ERR_INVALID_ARG;
    const size_t a = elem_size(in->dtype);
    if (!aligned(in->x, a) || !aligned(in->dt[0], a) || !aligned(in->dt[1], a) || !aligned(u, 4) ||
        !aligned(delta, 4) || !aligned(p->conv_w, 4) || !aligned(p->dt_bias, 4) || !aligned(p->conv_b, 4))
        return BIMAMBA_ERR_MISALIGNED;
    const int64_t total = 2LL * batch * L * d_inner;
    const int64_t blocks = std::min<int64_t>((total + 255) / 256, 148LL * 16);
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    if (in->dtype == BIMAMBA_BF16)
        bimamba::features_kernel<bf16><<<(unsigned)blocks, 256, 0, st>>>(
            static_cast<const bf16*>(in->x), static_cast<const bf16*>(in->dt[0]),
            static_cast<const bf16*>(in->dt[1]), p->conv_w, p->conv_b, p->dt_bias, batch, L, d_inner, u, delta);
    else
        bimamba::features_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(
            static_cast<const float*>(in->x), static_cast<const float*>(in->dt[0]),
            static_cast<const float*>(in->dt[1]), p->conv_w, p->conv_b, p->dt_bias, batch, L, d_inner, u, delta);
    return launch_status();
}

size_t bimamba_workspace_bytes(int batch, int64_t L, int d_inner, int d_state, unsigned flags) {
    (void)flags;
    if (batch <= 0 || batch > kMaxBatch || L <= 0 || d_inner <= 0 || d_state != bimamba::kNState) return 0;
    return layer_ws_bcq_offset(batch, L, d_inner) + layer_ws_bcq_bytes(batch, L);
}

}  // extern "C"

namespace {

// The layer, optionally with carries (carry may be null; its pointers may be null).
int layer_fwd_impl(const bimamba_inputs_t* in, const bimamba_params_t* p, const bimamba_carry_t* carry,
                   void* out, bimamba_dtype_t out_dtype, int batch, int64_t L, int d_inner, int d_state,
                   unsigned flags, void* workspace, size_t workspace_bytes, void* cuda_stream) {
    if (batch <= 0 || batch > kMaxBatch || L <= 0 || d_inner <= 0 || !out) return BIMAMBA_ERR_INVALID_ARG;
    if (d_state != bimamba::kNState) return BIMAMBA_ERR_UNSUPPORTED;
    const unsigned known = BIMAMBA_FWD_ONLY | BIMAMBA_REV_ONLY | BIMAMBA_LANES_MASK | BIMAMBA_NO_TMA |
                           BIMAMBA_CHUNK_MASK | BIMAMBA_FAMILY_MASK | BIMAMBA_TEST_STARVE | BIMAMBA_CHUNKED_WIDE;
    const unsigned chunk_field = (flags & BIMAMBA_CHUNK_MASK) >> BIMAMBA_CHUNK_SHIFT;
    if (chunk_field == 3) return BIMAMBA_ERR_UNSUPPORTED;
    if ((flags & ~known) || !lanes_ok(flags)) return BIMAMBA_ERR_UNSUPPORTED;
    if ((flags & BIMAMBA_FWD_ONLY) && (flags & BIMAMBA_REV_ONLY)) return BIMAMBA_ERR_INVALID_ARG;
    if (!dtype_ok(out_dtype)) return BIMAMBA_ERR_UNSUPPORTED;
    int rc = check_inputs(in, true, true);
    if (rc) return rc;
    if ((rc = check_params(p))) return rc;
    if (!aligned(out, elem_size(out_dtype))) return BIMAMBA_ERR_MISALIGNED;
    const size_t need = bimamba_workspace_bytes(batch, L, d_inner, d_state, flags);
    if (!workspace || !aligned(workspace, 16) || workspace_bytes < need) return BIMAMBA_ERR_WORKSPACE;

    KParams k = {};
    fill_inputs(k, in);
    fill_params(k, p);
    k.out = out;
    k.ws = static_cast<float*>(workspace);
    k.bcq = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + layer_ws_bcq_offset(batch, L, d_inner));
    k.L = L;
    k.M = L / 2;
    k.D = d_inner;
    k.batch = batch;
    k.dir_scale[0] = (flags & BIMAMBA_REV_ONLY) ? 0.f : 1.f;
    k.dir_scale[1] = (flags & BIMAMBA_FWD_ONLY) ? 0.f : 1.f;
    k.starve = (flags & BIMAMBA_TEST_STARVE) ? 1 : 0;
    k.wait_limit = k.starve ? kStarveWaitCycles : kWaitCycles;
    bool with_carry = false;
    if (carry) {
        for (int r = 0; r < 2; ++r) {
            if (!aligned(carry->h_in[r], 4) || !aligned(carry->h_out[r], 4) || !aligned(carry->delta_sum[r], 4) ||
                !aligned(carry->conv_halo[r], elem_size(in->dtype)))
                return BIMAMBA_ERR_MISALIGNED;
            k.carry_in[r] = carry->h_in[r];
            k.carry_out[r] = carry->h_out[r];
            k.delta_sum[r] = carry->delta_sum[r];
            k.conv_halo[r] = carry->conv_halo[r];
            with_carry = with_carry || carry->h_in[r] || carry->h_out[r] || carry->delta_sum[r] || carry->conv_halo[r];
        }
    }
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    const bool in_bf = in->dtype == BIMAMBA_BF16, out_bf = out_dtype == BIMAMBA_BF16;
    const unsigned forced = (flags & BIMAMBA_LANES_MASK) >> BIMAMBA_LANES_SHIFT;
    const int fam = pick_family(2LL * batch * d_inner, flags);
    if (fam == 3) {  // the chunked parallel scan: TMA-fed; the lane and chunk fields are not read
        if ((flags & BIMAMBA_NO_TMA) || !tma_eligible(in, d_inner, true, true)) return BIMAMBA_ERR_UNSUPPORTED;
        if (with_carry) {
            if (in_bf && out_bf) return launch_layer_pscan<2, bf16, bf16, true>(k, in, st);
            if (in_bf) return launch_layer_pscan<2, bf16, float, true>(k, in, st);
            if (out_bf) return launch_layer_pscan<2, float, bf16, true>(k, in, st);
            return launch_layer_pscan<2, float, float, true>(k, in, st);
        }
        if (in_bf && out_bf) return launch_layer_pscan<2, bf16, bf16>(k, in, st);
        if (in_bf) return launch_layer_pscan<2, bf16, float>(k, in, st);
        if (out_bf) return launch_layer_pscan<2, float, bf16>(k, in, st);
        return launch_layer_pscan<2, float, float>(k, in, st);
    }
    const bool group_ok = forced == 0 || forced == 1 || forced == 2 || forced == 4 || forced == 8;
    if (!(flags & BIMAMBA_NO_TMA) && fam == 2 && group_ok &&
        tma_eligible(in, d_inner, true, true)) {
        if (with_carry) {  // carries: one lane per channel (the group size changes only the speed)
            if (in_bf && out_bf) return launch_fused_layer<1, bf16, bf16, true, false, true>(k, in, st);
            if (in_bf) return launch_fused_layer<1, bf16, float, true, false, true>(k, in, st);
            if (out_bf) return launch_fused_layer<1, float, bf16, true, false, true>(k, in, st);
            return launch_fused_layer<1, float, float, true, false, true>(k, in, st);
        }
        const int gf = pick_group_fused(flags);
        // B/C widened to fp32 once per chunk at 2 lanes per group (measured
        // 1.164 against 1.176 ms at batch 8, L 2048); the chunk field's 1
        // selects the per-use widening there, its 2 the widening at 4 lanes.
        // One lane per channel (the default) reads them as fp32 quads widened
        // once per call (1.054 against 1.098 ms for widening per chunk).
        const bool f32bc = (gf == 2 && chunk_field != 1) || (gf == 4 && chunk_field == 2);
        if (in_bf && out_bf) return fused_layer_by_group<bf16, bf16>(gf, f32bc, k, in, st);
        if (in_bf) return fused_layer_by_group<bf16, float>(gf, f32bc, k, in, st);
        if (out_bf) return fused_layer_by_group<float, bf16>(gf, f32bc, k, in, st);
        return fused_layer_by_group<float, float>(gf, f32bc, k, in, st);
    }
    if (!(flags & BIMAMBA_NO_TMA) && (forced == 0 || forced >= 4) && tma_eligible(in, d_inner, true, true)) {
        const int gt = pick_lanes_tma(2LL * batch * d_inner, flags);
        // with carries the chunk length is the automatic one (the flag is not honoured)
        const int tt = with_carry ? pick_chunk_tma(0, gt) : pick_chunk_tma(flags, gt);
        // 8 lanes per channel with 32-token chunks: one warp per direction per
        // CTA (measured 6.79 against 7.20 ms for 4-warp CTAs at batch 1,
        // L 65536, d_inner 4096: 1024 CTAs spread over the SMs evenly), the
        // group loop fully unrolled (6.24 against 6.77 ms), and B/C widened
        // to fp32 quads once per call in the workspace instead of by every
        // lane at each use.  BIMAMBA_CHUNKED_WIDE keeps the 4-warp CTAs with
        // B/C widened once per chunk in shared memory.
        if (gt == 8 && tt == 32 && !(flags & BIMAMBA_CHUNKED_WIDE)) {
            if (with_carry) {
                if (in_bf && out_bf) return launch_layer_tma<8, 32, bf16, bf16, true, 1, false, true, true>(k, in, st);
                if (in_bf) return launch_layer_tma<8, 32, bf16, float, true, 1, false, true, true>(k, in, st);
                if (out_bf) return launch_layer_tma<8, 32, float, bf16, true, 1, false, true, true>(k, in, st);
                return launch_layer_tma<8, 32, float, float, true, 1, false, true, true>(k, in, st);
            }
            if (in_bf && out_bf) return launch_layer_tma<8, 32, bf16, bf16, false, 1, false, true, true>(k, in, st);
            if (in_bf) return launch_layer_tma<8, 32, bf16, float, false, 1, false, true, true>(k, in, st);
            if (out_bf) return launch_layer_tma<8, 32, float, bf16, false, 1, false, true, true>(k, in, st);
            return launch_layer_tma<8, 32, float, float, false, 1, false, true, true>(k, in, st);
        }
        if (with_carry) {
            if (in_bf && out_bf) return layer_tma_carry_by_lanes<bf16, bf16>(gt, k, in, st);
            if (in_bf) return layer_tma_carry_by_lanes<bf16, float>(gt, k, in, st);
            if (out_bf) return layer_tma_carry_by_lanes<float, bf16>(gt, k, in, st);
            return layer_tma_carry_by_lanes<float, float>(gt, k, in, st);
        }
        if (in_bf && out_bf) return layer_tma_by_lanes<bf16, bf16>(gt, tt, k, in, st);
        if (in_bf) return layer_tma_by_lanes<bf16, float>(gt, tt, k, in, st);
        if (out_bf) return layer_tma_by_lanes<float, bf16>(gt, tt, k, in, st);
        return layer_tma_by_lanes<float, float>(gt, tt, k, in, st);
    }
    if (with_carry) return BIMAMBA_ERR_UNSUPPORTED;  // carries live in the TMA-fed kernel families
    const int g = pick_lanes(2LL * batch * d_inner, flags);
    if (in_bf && out_bf) return layer_by_lanes<bf16, bf16>(g, k, st);
    if (in_bf) return layer_by_lanes<bf16, float>(g, k, st);
    if (out_bf) return layer_by_lanes<float, bf16>(g, k, st);
    return layer_by_lanes<float, float>(g, k, st);
}

}  // namespace

extern "C" {

int bimamba_layer_fwd(const bimamba_inputs_t* in, const bimamba_params_t* p, void* out,
                      bimamba_dtype_t out_dtype, int batch, int64_t L, int d_inner, int d_state,
                      unsigned flags, void* workspace, size_t workspace_bytes, void* cuda_stream) {
    return layer_fwd_impl(in, p, nullptr, out, out_dtype, batch, L, d_inner, d_state, flags, workspace,
                          workspace_bytes, cuda_stream);
}

int bimamba_layer_fwd_carry(const bimamba_inputs_t* in, const bimamba_params_t* p, const bimamba_carry_t* carry,
                            void* out, bimamba_dtype_t out_dtype, int batch, int64_t L, int d_inner, int d_state,
                            unsigned flags, void* workspace, size_t workspace_bytes, void* cuda_stream) {
    if (!carry) return BIMAMBA_ERR_INVALID_ARG;
    if (flags & BIMAMBA_NO_TMA) return BIMAMBA_ERR_UNSUPPORTED;
    return layer_fwd_impl(in, p, carry, out, out_dtype, batch, L, d_inner, d_state, flags, workspace,
                          workspace_bytes, cuda_stream);
}

int bimamba_compose_carries(const float* h_out_all, const float* delta_sum_all, const bimamba_params_t* p,
                            int nseg, int seg, int batch, int d_inner, int d_state, float* h_in, void* cuda_stream) {
    if (!h_out_all || !delta_sum_all || !h_in || nseg < 1 || seg < 0 || seg >= nseg || batch <= 0 ||
        batch > kMaxBatch || d_inner <= 0)
        return BIMAMBA_ERR_INVALID_ARG;
    if (d_state != bimamba::kNState) return BIMAMBA_ERR_UNSUPPORTED;
    if (!p || !p->A) return BIMAMBA_ERR_INVALID_ARG;
    if (!aligned(h_out_all, 4) || !aligned(delta_sum_all, 4) || !aligned(h_in, 4) || !aligned(p->A, 4))
        return BIMAMBA_ERR_MISALIGNED;
    const int64_t n = (int64_t)batch * d_inner * bimamba::kNState;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    bimamba::compose_carries_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(h_out_all, delta_sum_all, p->A,
                                                                              nseg, seg, batch, d_inner, h_in);
    return launch_status();
}

int bimamba_prefix_state(const bimamba_inputs_t* prefix, const bimamba_params_t* p, int batch, int64_t P,
                         int d_inner, int d_state, bimamba_fwd_state_t* state_out, void* cuda_stream) {
    if (batch <= 0 || batch > kMaxBatch || P <= 0 || d_inner <= 0) return BIMAMBA_ERR_INVALID_ARG;
    if (d_state != bimamba::kNState) return BIMAMBA_ERR_UNSUPPORTED;
    int rc = check_inputs(prefix, false, false);
    if (rc) return rc;
    if ((rc = check_params(p))) return rc;
    if (!state_out || !state_out->h || !state_out->conv_x) return BIMAMBA_ERR_INVALID_ARG;
    if (!aligned(state_out->h, 4) || !aligned(state_out->conv_x, elem_size(prefix->dtype)))
        return BIMAMBA_ERR_MISALIGNED;

    KParams k = {};
    fill_inputs(k, prefix);
    fill_params(k, p);
    k.h_out = state_out->h;
    k.tail_out = state_out->conv_x;
    k.L = P;
    k.D = d_inner;
    k.batch = batch;
    k.dir_scale[0] = k.dir_scale[1] = 1.f;
    k.wait_limit = kWaitCycles;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    if (tma_eligible(prefix, d_inner, false, false) && pick_family((int64_t)batch * d_inner, 0) == 2) {
        if (prefix->dtype == BIMAMBA_BF16) return launch_fused_prefix<kPrefixGroup, bf16>(k, prefix, st);
        return launch_fused_prefix<kPrefixGroup, float>(k, prefix, st);
    }
    if (tma_eligible(prefix, d_inner, false, false)) {
        const int gt = pick_lanes_tma((int64_t)batch * d_inner, 0);
        if (prefix->dtype == BIMAMBA_BF16) return prefix_tma_by_lanes<bf16>(gt, k, prefix, st);
        return prefix_tma_by_lanes<float>(gt, k, prefix, st);
    }
    const int g = pick_lanes((int64_t)batch * d_inner, 0);
    if (prefix->dtype == BIMAMBA_BF16) return prefix_by_lanes<bf16>(g, k, st);
    return prefix_by_lanes<float>(g, k, st);
}

int bimamba_block_step(const bimamba_fwd_state_t* prefix_state, const bimamba_inputs_t* block, int block_len,
                       const bimamba_params_t* p, void* out, bimamba_dtype_t out_dtype, int batch, int d_inner,
                       int d_state, bimamba_fwd_state_t* new_state, unsigned flags, void* cuda_stream) {
    if (batch <= 0 || batch > kMaxBatch || d_inner <= 0 || !out || block_len <= 0) return BIMAMBA_ERR_INVALID_ARG;
    if (d_state != bimamba::kNState || block_len > kTBlock) return BIMAMBA_ERR_UNSUPPORTED;
    const unsigned known = BIMAMBA_FWD_ONLY | BIMAMBA_REV_ONLY | BIMAMBA_LANES_MASK | BIMAMBA_NO_TMA;
    if ((flags & ~known) || !lanes_ok(flags)) return BIMAMBA_ERR_UNSUPPORTED;
    if ((flags & BIMAMBA_FWD_ONLY) && (flags & BIMAMBA_REV_ONLY)) return BIMAMBA_ERR_INVALID_ARG;
    if (!dtype_ok(out_dtype)) return BIMAMBA_ERR_UNSUPPORTED;
    int rc = check_inputs(block, true, true);
    if (rc) return rc;
    if ((rc = check_params(p))) return rc;
    if (!prefix_state || !prefix_state->h || !prefix_state->conv_x) return BIMAMBA_ERR_INVALID_ARG;
    if (new_state && (!new_state->h || !new_state->conv_x)) return BIMAMBA_ERR_INVALID_ARG;
    const size_t a = elem_size(block->dtype);
    if (!aligned(out, elem_size(out_dtype)) || !aligned(prefix_state->h, 4) || !aligned(prefix_state->conv_x, a))
        return BIMAMBA_ERR_MISALIGNED;
    if (new_state && (!aligned(new_state->h, 4) || !aligned(new_state->conv_x, a))) return BIMAMBA_ERR_MISALIGNED;

    KParams k = {};
    fill_inputs(k, block);
    fill_params(k, p);
    k.out = out;
    k.h_in = prefix_state->h;
    k.tail_in = prefix_state->conv_x;
    k.h_out = new_state ? new_state->h : nullptr;
    k.tail_out = new_state ? new_state->conv_x : nullptr;
    k.L = block_len;
    k.D = d_inner;
    k.batch = batch;
    k.dir_scale[0] = (flags & BIMAMBA_REV_ONLY) ? 0.f : 1.f;
    k.dir_scale[1] = (flags & BIMAMBA_FWD_ONLY) ? 0.f : 1.f;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    const bool in_bf = block->dtype == BIMAMBA_BF16, out_bf = out_dtype == BIMAMBA_BF16;
    if ((flags & BIMAMBA_LANES_MASK) == 0 && !(flags & BIMAMBA_NO_TMA) &&
        async_block_eligible(block, prefix_state->conv_x, d_inner)) {
        if (in_bf && out_bf) return launch_async_block<bf16, bf16>(k, st);
        if (in_bf) return launch_async_block<bf16, float>(k, st);
        if (out_bf) return launch_async_block<float, bf16>(k, st);
        return launch_async_block<float, float>(k, st);
    }
    if ((flags & BIMAMBA_LANES_MASK) == 0) {
        if (in_bf && out_bf) return launch_fused_block<bf16, bf16>(k, st);
        if (in_bf) return launch_fused_block<bf16, float>(k, st);
        if (out_bf) return launch_fused_block<float, bf16>(k, st);
        return launch_fused_block<float, float>(k, st);
    }
    const int g = pick_lanes((int64_t)batch * d_inner, flags);
    if (in_bf && out_bf) return block_by_lanes<bf16, bf16>(g, k, st);
    if (in_bf) return block_by_lanes<bf16, float>(g, k, st);
    if (out_bf) return block_by_lanes<float, bf16>(g, k, st);
    return block_by_lanes<float, float>(g, k, st);
}

}  // extern "C"

// ---- full layer without a caller-provided workspace
//
// Some callers have no device allocator to hand: a plugin loaded into a host
// application that owns every byte of GPU memory, or a program that reaches
// this library only through the C ABI from a language with no CUDA memory
// API.  They cannot supply the workspace bimamba_layer_fwd needs, so this
// entry point uses a fixed scratch array that lives in the library itself.

// Scratch for the half-sequence partial outputs, 64 MiB on every device that
// loads this library, kept until the process exits.  In host code this name
// is only a stand-in for the symbol: its device address comes from
// cudaGetSymbolAddress below, never from the name itself.
static __device__ __align__(256) unsigned char g_noalloc_scratch[64u << 20];

namespace {

constexpr size_t kNoallocScratchBytes = sizeof(g_noalloc_scratch);
std::mutex g_noalloc_mu;
bimamba::ContextAddressCache<64> g_noalloc_addr;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_entry(const char* name) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(f);
}

// Id of the current context, or false if there is none (or the driver
// cannot tell).
bool current_context_id(unsigned long long* id) {
    static const CtxGetCurrentFn get_current = driver_entry<CtxGetCurrentFn>("cuCtxGetCurrent");
    static const CtxGetIdFn get_id = driver_entry<CtxGetIdFn>("cuCtxGetId");
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current context.  It is
// looked up with cudaGetSymbolAddress (with the device current) the first
// time a context calls, then cached under (device, context id): a context
// destroyed and created again gets a new id, so its module's new address is
// looked up afresh.  Without a context id the address is looked up on every
// call.
int noalloc_scratch(void** addr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BIMAMBA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    unsigned long long id = 0;
    if (current_context_id(&id)) {
        if (void* p = g_noalloc_addr.find({dev, id})) {
            *addr = p;
            return BIMAMBA_OK;
        }
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return BIMAMBA_ERR_CUDA;
    // the lookup makes the device's primary context current if none was
    if (current_context_id(&id)) g_noalloc_addr.put({dev, id}, p);
    *addr = p;
    return BIMAMBA_OK;
}

}  // namespace

extern "C" int bimamba_layer_fwd_noalloc(const bimamba_inputs_t* in, const bimamba_params_t* p, void* out,
                                         bimamba_dtype_t out_dtype, int batch, int64_t L, int d_inner,
                                         int d_state, unsigned flags, void* cuda_stream) {
    // Invalid sizes: the full entry point names the problem without touching the GPU.
    if (bimamba_workspace_bytes(batch, L, d_inner, d_state, flags) == 0)
        return bimamba_layer_fwd(in, p, out, out_dtype, batch, L, d_inner, d_state, flags, nullptr, 0,
                                 cuda_stream);
    void* scratch = nullptr;
    const int rc = noalloc_scratch(&scratch);
    if (rc) return rc;
    // The full entry point runs every check in its usual order; a problem too
    // large for the scratch fails its last one, the workspace size.
    return bimamba_layer_fwd(in, p, out, out_dtype, batch, L, d_inner, d_state, flags, scratch,
                             kNoallocScratchBytes, cuda_stream);
}

// ---- Mamba-2 mixer

namespace {

size_t m2_round(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

struct M2Layout {
    size_t v, dl, yf, yb, tiles, sync, total;
};

// Workspace: conv features [2][batch][L][CH] fp32 (step-by-step path),
// step sizes [2][batch][H][L], forward and reverse outputs [batch][L][H*P]
// each, all fp32, then the fp16 C/B tiles of the tensor-core path
// [2][batch][ceil(L/128)][2][128 x 128], then its ticket counter and one
// flag per (batch row, head), int32; each part 256-byte aligned.
M2Layout m2_layout(int batch, int64_t L, int H, int P, int N) {
    const size_t CH = (size_t)H * P + 2 * (size_t)N;
    const size_t nc = (size_t)((L + bimamba::kSQ - 1) / bimamba::kSQ);
    M2Layout l;
    l.v = 0;
    l.dl = m2_round(2 * (size_t)batch * (size_t)L * CH * 4);
    l.yf = l.dl + m2_round(2 * (size_t)batch * (size_t)H * (size_t)L * 4);
    l.yb = l.yf + m2_round((size_t)batch * (size_t)L * (size_t)H * P * 4);
    l.tiles = l.yb + m2_round((size_t)batch * (size_t)L * (size_t)H * P * 4);
    l.sync = l.tiles + m2_round(2 * (size_t)batch * nc * 2 * (size_t)bimamba::kTileBytes);
    l.total = l.sync + (1 + (size_t)batch * H) * 4;
    return l;
}

bool m2_sizes_ok(int batch, int64_t L, int H) {
    // grid limits: 2 * batch (z) and nheads (x) at most 65535; L bounded so
    // that token indices stay far inside int64 and the prep grid's x.
    return batch >= 1 && 2 * (int64_t)batch <= 65535 && L >= 1 && L <= (int64_t)1 << 31 && H >= 1 && H <= 65535;
}

// Chunked dual form on the tensor cores: the C/B chunk tiles, then the
// directions' chunk scans, which compute the x features and step sizes
// themselves -- both in one launch, as clusters of two CTAs that meet halfway
// when one direction's grid leaves SMs idle, else as ticket-ordered CTAs
// (forwards first, each reverse after its forward; the ticket counter and
// flags are cleared first).  When L is not a whole number of chunks, the
// ragged chunk's tiles are cleared first so that its rows past the end read
// zeros.
template <typename Tin, typename Tout>
int launch_m2_ssd(const bimamba::M2Params& k, bool no_cluster, cudaStream_t st) {
    auto kc = &bimamba::m2_ssd_cluster_kernel<Tin, Tout>;
    auto kt = &bimamba::m2_ssd_ticket_kernel<Tin, Tout>;
    int rc = ensure_smem(reinterpret_cast<const void*>(kc), bimamba::kSsdSmem);
    if (!rc) rc = ensure_smem(reinterpret_cast<const void*>(kt), bimamba::kSsdSmem);
    if (rc) return rc;
    const int64_t nc = (k.L + bimamba::kSQ - 1) / bimamba::kSQ;
    if (k.L % bimamba::kSQ) {  // the ragged chunk: the forward's last, the reverse's first in step order
        const size_t pair = 2 * (size_t)bimamba::kTileBytes;
        if (cudaMemset2DAsync(k.tiles + (nc - 1) * pair, (size_t)nc * pair, 0, pair, (size_t)k.batch, st) !=
                cudaSuccess ||
            cudaMemset2DAsync(k.tiles + (size_t)k.batch * nc * pair, (size_t)nc * pair, 0, pair, (size_t)k.batch,
                              st) != cudaSuccess)
            return BIMAMBA_ERR_CUDA;
    }
    const int64_t tok_per_cta = 4 * bimamba::kM2PrepT;
    const dim3 g1((unsigned)((k.L + tok_per_cta - 1) / tok_per_cta), 1u, (unsigned)(2 * k.batch));
    bimamba::m2_prep_kernel<Tin, true><<<g1, 128, 0, st>>>(k);
    if (cudaGetLastError() != cudaSuccess) return BIMAMBA_ERR_CUDA;
    // one direction's grid within one wave (2 CTAs per SM): both directions at once, as
    // clusters that meet halfway; else ticket-ordered CTAs (the clustered form measured
    // 0.89 against 0.80 ms for a forward launch and then a reverse one at batch 8, L 2048,
    // 120 heads)
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return BIMAMBA_ERR_CUDA;
    if (!no_cluster && (int64_t)k.H * k.batch <= 2LL * sms) {
        kc<<<dim3((unsigned)(2 * k.H), (unsigned)k.batch), bimamba::kSsdThreads, bimamba::kSsdSmem, st>>>(k);
        return launch_status();
    }
    const int64_t n1 = (int64_t)k.H * k.batch;
    if (cudaMemsetAsync(k.sync, 0, (size_t)(1 + n1) * sizeof(int), st) != cudaSuccess) return BIMAMBA_ERR_CUDA;
    kt<<<(unsigned)(2 * n1), bimamba::kSsdThreads, bimamba::kSsdSmem, st>>>(k);
    return launch_status();
}

template <typename Tin, typename Tout>
int launch_m2(const bimamba::M2Params& k, cudaStream_t st) {
    const dim3 g1((unsigned)((k.L + bimamba::kM2PrepT - 1) / bimamba::kM2PrepT), (unsigned)((k.CH + 1023) / 1024),
                  (unsigned)(2 * k.batch));
    bimamba::m2_prep_kernel<Tin, false><<<g1, 128, 0, st>>>(k);
    if (cudaGetLastError() != cudaSuccess) return BIMAMBA_ERR_CUDA;
    bimamba::m2_scan_kernel<true, Tin><<<dim3((unsigned)(2 * k.H), (unsigned)k.batch), 32, 0, st>>>(k);
    if (cudaGetLastError() != cudaSuccess) return BIMAMBA_ERR_CUDA;
    const int64_t n4 = (int64_t)k.batch * k.L * k.H * bimamba::kM2P / 4;
    const int64_t blocks = (n4 + 255) / 256;
    bimamba::m2_combine_kernel<Tin, Tout><<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), 256, 0, st>>>(k);
    return launch_status();
}

// The block step with bf16 inputs, a block of at most 32 steps and a multiple of
// 4 heads: the features and step sizes as for the step-by-step scan, then the
// block's closed form on the tensor cores (m2_block_mma_kernel), then the
// combination and gate.
template <typename Tout>
int launch_m2_block_mma(const bimamba::M2Params& k, cudaStream_t st) {
    const dim3 g1((unsigned)((k.L + bimamba::kM2PrepT - 1) / bimamba::kM2PrepT), (unsigned)((k.CH + 1023) / 1024),
                  (unsigned)(2 * k.batch));
    bimamba::m2_prep_kernel<bf16, false><<<g1, 128, 0, st>>>(k);
    if (cudaGetLastError() != cudaSuccess) return BIMAMBA_ERR_CUDA;
    bimamba::m2_block_gram_kernel<<<dim3((unsigned)k.batch, 2, bimamba::kM2BlkT / bimamba::kM2GramRows), 128, 0,
                                    st>>>(k);
    if (cudaGetLastError() != cudaSuccess) return BIMAMBA_ERR_CUDA;
    const int smem = k.S_out ? bimamba::kBlkSmemCommit : bimamba::kBlkSmemStep;
    int rc = ensure_smem(reinterpret_cast<const void*>(&bimamba::m2_block_mma_kernel), bimamba::kBlkSmemCommit);
    if (rc) return rc;
    bimamba::m2_block_mma_kernel<<<dim3((unsigned)(k.H / bimamba::kM2BlkHeads), (unsigned)k.batch, 2), 128, smem,
                                   st>>>(k);
    if (cudaGetLastError() != cudaSuccess) return BIMAMBA_ERR_CUDA;
    const int64_t n4 = (int64_t)k.batch * k.L * k.H * bimamba::kM2P / 4;
    const int64_t blocks = (n4 + 255) / 256;
    bimamba::m2_combine_kernel<bf16, Tout><<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), 256, 0, st>>>(k);
    return launch_status();
}

// Shared checks of the Mamba-2 entry points: parameters and the 16-byte
// alignment the kernels' vector accesses need.
int m2_check_params(const bimamba2_params_t* p) {
    if (!p || !p->A || !p->D || !p->dt_bias || !p->conv_w) return BIMAMBA_ERR_INVALID_ARG;
    if (!aligned(p->A, 4) || !aligned(p->D, 4) || !aligned(p->dt_bias, 4) || !aligned(p->conv_w, 16) ||
        (p->conv_b && !aligned(p->conv_b, 4)))
        return BIMAMBA_ERR_MISALIGNED;
    return BIMAMBA_OK;
}

int m2_check_state(const bimamba2_fwd_state_t* s) {
    if (!s || !s->S || !s->conv_xbc) return BIMAMBA_ERR_INVALID_ARG;
    if (!aligned(s->S, 16) || !aligned(s->conv_xbc, 16)) return BIMAMBA_ERR_MISALIGNED;
    return BIMAMBA_OK;
}

void m2_fill_params(bimamba::M2Params& k, const bimamba2_params_t* p) {
    k.A = p->A;
    k.Dskip = p->D;
    k.dt_bias = p->dt_bias;
    k.conv_w = p->conv_w;
    k.conv_b = p->conv_b;
}

}  // namespace

extern "C" {

int bimamba2_prefix_state(const bimamba2_inputs_t* prefix, const bimamba2_params_t* p, int batch, int64_t P,
                          int nheads, int headdim, int d_state, bimamba2_fwd_state_t* state_out, void* workspace,
                          size_t workspace_bytes, void* cuda_stream) {
    if (!prefix || !m2_sizes_ok(batch, P, nheads)) return BIMAMBA_ERR_INVALID_ARG;
    if (headdim != bimamba::kM2P || d_state != bimamba::kM2N) return BIMAMBA_ERR_UNSUPPORTED;
    if (!dtype_ok(prefix->dtype)) return BIMAMBA_ERR_UNSUPPORTED;
    if (!prefix->xbc[0] || !prefix->dt[0]) return BIMAMBA_ERR_INVALID_ARG;
    if (!aligned(prefix->xbc[0], 16) || !aligned(prefix->dt[0], elem_size(prefix->dtype))) return BIMAMBA_ERR_MISALIGNED;
    int rc = m2_check_params(p);
    if (rc) return rc;
    if ((rc = m2_check_state(state_out))) return rc;
    const M2Layout lay = m2_layout(batch, P, nheads, headdim, d_state);
    if (!workspace || workspace_bytes < lay.total) return BIMAMBA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BIMAMBA_ERR_MISALIGNED;
    bimamba::M2Params k = {};
    k.xbc[0] = k.xbc[1] = prefix->xbc[0];
    k.dt[0] = k.dt[1] = prefix->dt[0];
    m2_fill_params(k, p);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    k.V = reinterpret_cast<float*>(ws + lay.v);
    k.DL = reinterpret_cast<float*>(ws + lay.dl);
    k.L = P;
    k.H = nheads;
    k.CH = nheads * headdim + 2 * d_state;
    k.batch = batch;
    k.dir_scale[0] = k.dir_scale[1] = 1.f;
    k.S_out = state_out->S;
    k.tail_out = state_out->conv_xbc;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    const dim3 g1((unsigned)((P + bimamba::kM2PrepT - 1) / bimamba::kM2PrepT), (unsigned)((k.CH + 1023) / 1024),
                  (unsigned)batch);  // direction 0 only
    const dim3 g2((unsigned)nheads, (unsigned)batch);
    const dim3 g3((unsigned)((k.CH + 127) / 128), (unsigned)batch);
    if (prefix->dtype == BIMAMBA_BF16) {
        // bf16 inputs (the 2e-3 bound): the chunked dual form's state updates on the tensor cores,
        // from the B tiles of direction 0
        k.tiles = ws + lay.tiles;
        k.wait_limit = kWaitCycles;
        const int64_t nc = (P + bimamba::kSQ - 1) / bimamba::kSQ;
        if (P % bimamba::kSQ) {  // the last chunk's rows past the end read zeros
            const size_t pair = 2 * (size_t)bimamba::kTileBytes;
            if (cudaMemset2DAsync(k.tiles + (nc - 1) * pair, (size_t)nc * pair, 0, pair, (size_t)batch, st) !=
                cudaSuccess)
                return BIMAMBA_ERR_CUDA;
        }
        const int64_t tok_per_cta = 4 * bimamba::kM2PrepT;
        const dim3 gt((unsigned)((P + tok_per_cta - 1) / tok_per_cta), 1u, (unsigned)batch);  // direction 0 only
        bimamba::m2_prep_kernel<bf16, true><<<gt, 128, 0, st>>>(k);
        rc = ensure_smem(reinterpret_cast<const void*>(&bimamba::m2_ssd_prefix_kernel), bimamba::kSsdSmem);
        if (rc) return rc;
        bimamba::m2_ssd_prefix_kernel<<<g2, bimamba::kSsdThreads, bimamba::kSsdSmem, st>>>(k);
        bimamba::m2_tail_kernel<bf16><<<g3, 128, 0, st>>>(k);
    } else {
        bimamba::m2_prep_kernel<float, false><<<g1, 128, 0, st>>>(k);
        bimamba::m2_scan_kernel<false, float><<<g2, 32, 0, st>>>(k);
        bimamba::m2_tail_kernel<float><<<g3, 128, 0, st>>>(k);
    }
    return launch_status();
}

int bimamba2_block_step(const bimamba2_fwd_state_t* prefix_state, const bimamba2_inputs_t* block, int64_t block_len,
                        const bimamba2_params_t* p, void* out, bimamba_dtype_t out_dtype, int batch, int nheads,
                        int headdim, int d_state, bimamba2_fwd_state_t* new_state, unsigned flags, void* workspace,
                        size_t workspace_bytes, void* cuda_stream) {
    if (!block || !out || !m2_sizes_ok(batch, block_len, nheads)) return BIMAMBA_ERR_INVALID_ARG;
    if (headdim != bimamba::kM2P || d_state != bimamba::kM2N) return BIMAMBA_ERR_UNSUPPORTED;
    if (flags & ~(BIMAMBA_FWD_ONLY | BIMAMBA_REV_ONLY)) return BIMAMBA_ERR_UNSUPPORTED;
    if ((flags & BIMAMBA_FWD_ONLY) && (flags & BIMAMBA_REV_ONLY)) return BIMAMBA_ERR_INVALID_ARG;
    if (!dtype_ok(block->dtype) || !dtype_ok(out_dtype)) return BIMAMBA_ERR_UNSUPPORTED;
    const void* ptrs[5] = {block->xbc[0], block->xbc[1], block->z, block->dt[0], block->dt[1]};
    for (const void* q : ptrs) {
        if (!q) return BIMAMBA_ERR_INVALID_ARG;
        if (!aligned(q, elem_size(block->dtype))) return BIMAMBA_ERR_MISALIGNED;
    }
    if (!aligned(block->z, 16) || !aligned(block->xbc[0], 16) || !aligned(block->xbc[1], 16) || !aligned(out, 16))
        return BIMAMBA_ERR_MISALIGNED;
    int rc = m2_check_params(p);
    if (rc) return rc;
    if ((rc = m2_check_state(prefix_state))) return rc;
    if (new_state && (rc = m2_check_state(new_state))) return rc;
    const M2Layout lay = m2_layout(batch, block_len, nheads, headdim, d_state);
    if (!workspace || workspace_bytes < lay.total) return BIMAMBA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BIMAMBA_ERR_MISALIGNED;
    bimamba::M2Params k = {};
    for (int r = 0; r < 2; ++r) {
        k.xbc[r] = block->xbc[r];
        k.dt[r] = block->dt[r];
    }
    k.z = block->z;
    m2_fill_params(k, p);
    k.out = out;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    k.V = reinterpret_cast<float*>(ws + lay.v);
    k.DL = reinterpret_cast<float*>(ws + lay.dl);
    k.YF = reinterpret_cast<float*>(ws + lay.yf);
    k.YB = reinterpret_cast<float*>(ws + lay.yb);
    k.tiles = ws + lay.tiles;  // the tensor-core block step's G [2][batch][32][32] fp32
    k.L = block_len;
    k.H = nheads;
    k.CH = nheads * headdim + 2 * d_state;
    k.batch = batch;
    k.dir_scale[0] = (flags & BIMAMBA_REV_ONLY) ? 0.f : 1.f;
    k.dir_scale[1] = (flags & BIMAMBA_FWD_ONLY) ? 0.f : 1.f;
    k.S_in = prefix_state->S;
    k.tail_in = prefix_state->conv_xbc;
    k.S_out = new_state ? new_state->S : nullptr;
    k.tail_out = new_state ? new_state->conv_xbc : nullptr;
    k.wait_limit = kWaitCycles;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    const bool in_bf = block->dtype == BIMAMBA_BF16, out_bf = out_dtype == BIMAMBA_BF16;
    // bf16 inputs (tolerance 2e-3, fp16 operands suffice), a block of at most 32 steps and a
    // multiple of 4 heads: the tensor-core closed form; otherwise the step-by-step scan
    const bool mma = in_bf && block_len <= bimamba::kM2BlkT && nheads % bimamba::kM2BlkHeads == 0;
    if (mma) rc = out_bf ? launch_m2_block_mma<bf16>(k, st) : launch_m2_block_mma<float>(k, st);
    else if (in_bf && out_bf) rc = launch_m2<bf16, bf16>(k, st);
    else if (in_bf) rc = launch_m2<bf16, float>(k, st);
    else if (out_bf) rc = launch_m2<float, bf16>(k, st);
    else rc = launch_m2<float, float>(k, st);
    if (rc || !new_state) return rc;
    const dim3 g3((unsigned)((k.CH + 127) / 128), (unsigned)batch);
    if (in_bf)
        bimamba::m2_tail_kernel<bf16><<<g3, 128, 0, st>>>(k);
    else
        bimamba::m2_tail_kernel<float><<<g3, 128, 0, st>>>(k);
    return launch_status();
}

size_t bimamba2_workspace_bytes(int batch, int64_t L, int nheads, int headdim, int d_state) {
    if (!m2_sizes_ok(batch, L, nheads) || headdim <= 0 || d_state <= 0) return 0;
    return m2_layout(batch, L, nheads, headdim, d_state).total;
}

int bimamba2_layer_fwd(const bimamba2_inputs_t* in, const bimamba2_params_t* p, void* out,
                       bimamba_dtype_t out_dtype, int batch, int64_t L, int nheads, int headdim, int d_state,
                       unsigned flags, void* workspace, size_t workspace_bytes, void* cuda_stream) {
    if (!in || !p || !out || !m2_sizes_ok(batch, L, nheads)) return BIMAMBA_ERR_INVALID_ARG;
    if (headdim != bimamba::kM2P || d_state != bimamba::kM2N) return BIMAMBA_ERR_UNSUPPORTED;
    if (flags & ~(BIMAMBA_FWD_ONLY | BIMAMBA_REV_ONLY | BIMAMBA_NO_TMA | BIMAMBA_TEST_STARVE | BIMAMBA_M2_NO_CLUSTER))
        return BIMAMBA_ERR_UNSUPPORTED;
    if ((flags & BIMAMBA_FWD_ONLY) && (flags & BIMAMBA_REV_ONLY)) return BIMAMBA_ERR_INVALID_ARG;
    if (!dtype_ok(in->dtype) || !dtype_ok(out_dtype)) return BIMAMBA_ERR_UNSUPPORTED;
    const void* ptrs[5] = {in->xbc[0], in->xbc[1], in->z, in->dt[0], in->dt[1]};
    const size_t a = elem_size(in->dtype);
    for (const void* q : ptrs) {
        if (!q) return BIMAMBA_ERR_INVALID_ARG;
        if (!aligned(q, a)) return BIMAMBA_ERR_MISALIGNED;
    }
    // xBC rows, conv taps and z rows move in 16-byte pieces
    if (!aligned(in->z, 16) || !aligned(in->xbc[0], 16) || !aligned(in->xbc[1], 16)) return BIMAMBA_ERR_MISALIGNED;
    if (!p->A || !p->D || !p->dt_bias || !p->conv_w) return BIMAMBA_ERR_INVALID_ARG;
    if (!aligned(p->A, 4) || !aligned(p->D, 4) || !aligned(p->dt_bias, 4) || !aligned(p->conv_w, 16) ||
        (p->conv_b && !aligned(p->conv_b, 4)) || !aligned(out, 16))
        return BIMAMBA_ERR_MISALIGNED;
    const M2Layout lay = m2_layout(batch, L, nheads, headdim, d_state);
    if (!workspace || workspace_bytes < lay.total) return BIMAMBA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BIMAMBA_ERR_MISALIGNED;

    bimamba::M2Params k = {};
    for (int r = 0; r < 2; ++r) {
        k.xbc[r] = in->xbc[r];
        k.dt[r] = in->dt[r];
    }
    k.z = in->z;
    k.A = p->A;
    k.Dskip = p->D;
    k.dt_bias = p->dt_bias;
    k.conv_w = p->conv_w;
    k.conv_b = p->conv_b;
    k.out = out;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    k.V = reinterpret_cast<float*>(ws + lay.v);
    k.DL = reinterpret_cast<float*>(ws + lay.dl);
    k.YF = reinterpret_cast<float*>(ws + lay.yf);
    k.YB = reinterpret_cast<float*>(ws + lay.yb);
    k.L = L;
    k.H = nheads;
    k.CH = nheads * headdim + 2 * d_state;
    k.batch = batch;
    k.dir_scale[0] = (flags & BIMAMBA_REV_ONLY) ? 0.f : 1.f;
    k.dir_scale[1] = (flags & BIMAMBA_FWD_ONLY) ? 0.f : 1.f;
    k.starve = (flags & BIMAMBA_TEST_STARVE) ? 1 : 0;
    k.wait_limit = k.starve ? kStarveWaitCycles : kWaitCycles;
    k.meet_limit = k.starve ? kStarveWaitCycles : kWaitCycles;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    const bool in_bf = in->dtype == BIMAMBA_BF16, out_bf = out_dtype == BIMAMBA_BF16;
    if (in_bf && !(flags & BIMAMBA_NO_TMA)) {
        k.tiles = ws + lay.tiles;
        k.sync = reinterpret_cast<int*>(ws + lay.sync);
        const bool no_cluster = (flags & BIMAMBA_M2_NO_CLUSTER) != 0;
        if (out_bf) return launch_m2_ssd<bf16, bf16>(k, no_cluster, st);
        return launch_m2_ssd<bf16, float>(k, no_cluster, st);
    }
    if (in_bf && out_bf) return launch_m2<bf16, bf16>(k, st);
    if (in_bf) return launch_m2<bf16, float>(k, st);
    if (out_bf) return launch_m2<float, bf16>(k, st);
    return launch_m2<float, float>(k, st);
}

}  // extern "C"

// ---- the layer's neighbours: AdaLN and the projections

namespace {

// 2-D map over a row-major bf16 [rows][inner] matrix, box {64, box_rows},
// 128-byte swizzle (the layout the GEMM's descriptors expect).
bool map2d_sw128(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn f = encode_tiled();
    if (!f) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {(cuuint32_t)bimamba::kGemmBK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int launch_gemm(const void* a, const void* w, const bimamba::GemmParams& gp, cudaStream_t st) {
    CUtensorMap ma, mw;
    if (!map2d_sw128(&ma, a, (uint64_t)gp.K, (uint64_t)gp.M, bimamba::kGemmBM) ||
        !map2d_sw128(&mw, w, (uint64_t)gp.K, (uint64_t)gp.N, bimamba::kGemmBN))
        return BIMAMBA_ERR_CUDA;
    const void* fn = reinterpret_cast<const void*>(&bimamba::gemm_bf16_persistent_kernel);
    int rc = ensure_smem(fn, bimamba::kGemmSmem);
    if (rc) return rc;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return BIMAMBA_ERR_CUDA;
    const int64_t tiles = (int64_t)((gp.N + bimamba::kGemmBN - 1) / bimamba::kGemmBN) *
                          ((gp.M + bimamba::kGemmBM - 1) / bimamba::kGemmBM);
    const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
    bimamba::gemm_bf16_persistent_kernel<<<grid, bimamba::kGemmPThreads, bimamba::kGemmSmem, st>>>(ma, mw, gp);
    return launch_status();
}

// rows = batch * L within the GEMM grid's reach (ceil(rows / 128) <= 65535).
bool proj_rows_ok(int batch, int64_t L) {
    return batch >= 1 && batch <= kMaxBatch && L >= 1 && (int64_t)batch * L <= (int64_t)65535 * bimamba::kGemmBM;
}

}  // namespace

extern "C" {

int bimamba_adaln(const void* x, const float* gamma, const float* beta, void* out, int batch, int64_t L, int d,
                  float eps, void* cuda_stream) {
    if (!x || !gamma || !beta || !out || batch < 1 || batch > kMaxBatch || L < 1 || d < 8 || !(eps > 0.f) ||
        (int64_t)batch * L > 0x7fffffffLL)
        return BIMAMBA_ERR_INVALID_ARG;
    if (d % 8 || d > 8192) return BIMAMBA_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(out, 16) || !aligned(gamma, 16) || !aligned(beta, 16))
        return BIMAMBA_ERR_MISALIGNED;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    const int64_t rows = (int64_t)batch * L;
    const unsigned grid = (unsigned)((rows + 7) / 8);
    const bf16* xi = static_cast<const bf16*>(x);
    bf16* o = static_cast<bf16*>(out);
    const int cpl = (d + 255) / 256;  // 16-byte chunks per lane
    if (cpl <= 1) bimamba::adaln_kernel<1><<<grid, 256, 0, st>>>(xi, gamma, beta, o, rows, L, d, eps);
    else if (cpl <= 2) bimamba::adaln_kernel<2><<<grid, 256, 0, st>>>(xi, gamma, beta, o, rows, L, d, eps);
    else if (cpl <= 4) bimamba::adaln_kernel<4><<<grid, 256, 0, st>>>(xi, gamma, beta, o, rows, L, d, eps);
    else if (cpl <= 8) bimamba::adaln_kernel<8><<<grid, 256, 0, st>>>(xi, gamma, beta, o, rows, L, d, eps);
    else if (cpl <= 16) bimamba::adaln_kernel<16><<<grid, 256, 0, st>>>(xi, gamma, beta, o, rows, L, d, eps);
    else bimamba::adaln_kernel<32><<<grid, 256, 0, st>>>(xi, gamma, beta, o, rows, L, d, eps);
    return launch_status();
}

int bimamba_in_proj(const void* a, const void* w_in, int batch, int64_t L, int d_model, int d_inner, int d_state,
                    void* x, void* z, void* dt, void* B, void* C, void* cuda_stream) {
    if (!a || !w_in || !x || !z || !dt || !B || !C || !proj_rows_ok(batch, L) || d_model < 1 || d_inner < 1)
        return BIMAMBA_ERR_INVALID_ARG;
    if (d_state != bimamba::kNState || d_model % bimamba::kGemmBK || d_inner % 8) return BIMAMBA_ERR_UNSUPPORTED;
    for (const void* q : {a, w_in, (const void*)x, (const void*)z, (const void*)dt, (const void*)B, (const void*)C})
        if (!aligned(q, 16)) return BIMAMBA_ERR_MISALIGNED;
    bimamba::GemmParams gp = {};
    gp.M = (int)((int64_t)batch * L);
    gp.N = 4 * d_inner + 4 * d_state;
    gp.K = d_model;
    gp.scatter = 1;
    gp.x = static_cast<bf16*>(x);
    gp.z = static_cast<bf16*>(z);
    gp.dt = static_cast<bf16*>(dt);
    gp.Bm = static_cast<bf16*>(B);
    gp.Cm = static_cast<bf16*>(C);
    gp.D = d_inner;
    gp.Ns = d_state;
    gp.wait_limit = kWaitCycles;
    return launch_gemm(a, w_in, gp, static_cast<cudaStream_t>(cuda_stream));
}

int bimamba_out_proj(const void* y, const void* w_out, int batch, int64_t L, int d_inner, int d_model, void* out,
                     void* cuda_stream) {
    if (!y || !w_out || !out || !proj_rows_ok(batch, L) || d_model < 1 || d_inner < 1)
        return BIMAMBA_ERR_INVALID_ARG;
    if (d_inner % bimamba::kGemmBK || d_model % 8) return BIMAMBA_ERR_UNSUPPORTED;
    if (!aligned(y, 16) || !aligned(w_out, 16) || !aligned(out, 16)) return BIMAMBA_ERR_MISALIGNED;
    bimamba::GemmParams gp = {};
    gp.M = (int)((int64_t)batch * L);
    gp.N = d_model;
    gp.K = d_inner;
    gp.scatter = 0;
    gp.C = static_cast<bf16*>(out);
    gp.wait_limit = kWaitCycles;
    return launch_gemm(y, w_out, gp, static_cast<cudaStream_t>(cuda_stream));
}

}  // extern "C"


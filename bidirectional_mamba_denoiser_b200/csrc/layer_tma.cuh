// layer_tma.cuh -- TMA-fed kernels of the bidirectional Mamba mixer layer
// ("DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone", §3.2
// Eq. (4)-(6)): the full layer and the forward prefix scan (§4.3 cache).
//
// One CTA = one batch row x CW channels.  Warps [0, NWD) run the forward
// direction and warps [NWD, 2*NWD) the reverse direction over the same
// channels; each warp covers CPW = 32/G channels with G lanes per channel.
//
// Per direction the sequence is cut into chunks of T tokens on one grid
// shared by both directions (chunk k = tokens [kT, kT+T)).  Each chunk's x
// (with the 3-token conv halo), dt, B, C -- and z when the chunk is gated --
// arrive by 3-D TMA loads into an NS-stage shared-memory ring; a box that
// reaches outside [0, L) is zero-filled, which is exactly the conv's zero
// padding at the sequence ends.  Per chunk the direction's warps convert B/C
// to fp32 pairs once (shared by all its channels), meet at one named
// barrier, and the group leader then refills the stage the previous chunk
// used (every warp of the group is past it).  Tokens >= L in the last chunk
// get delta = 0 and zero drive, so their scan step is the identity.
//
// Full layer: the forward group walks chunks 0..nc-1 and the reverse group
// nc-1..0.  Chunks [0, nc/2) are the forward group's first half and the
// rest the reverse group's; each stores its fp32 y over its first half to
// the workspace, both groups meet at one barrier, and each then finishes the
// other half, adding the partner's y and applying the SiLU(z) gate.
#pragma once

#include "scan_kernels.cuh"
#include "tma_util.cuh"

namespace bimamba {

struct LayerMaps {
    CUtensorMap x;      // [batch][L][D]      box {CW, T+3, 1}
    CUtensorMap z;      // [batch][L][D]      box {CW, T, 1}
    CUtensorMap dt[2];  // [batch][L][D]      box {CW, T, 1}
    CUtensorMap B[2];   // [batch][L][16]     box {16, T, 1}
    CUtensorMap C[2];   // [batch][L][16]     box {16, T, 1}
};

constexpr int align128(int v) { return (v + 127) & ~127; }

template <int G, int T, int NWD, int NS, typename Tin>
struct TmaGeo {
    static_assert(T % G == 0 && T <= 253, "chunk");
    static constexpr int CPW = 32 / G;                    // channels per warp
    static constexpr int S = kNState / G;                 // states per lane
    static constexpr int EPL = T / G;                     // elements per lane per chunk
    static constexpr int CW = NWD * CPW;                  // channels per CTA
    static constexpr int ESZ = (int)sizeof(Tin);
    static constexpr int XB = align128((T + 3) * CW * ESZ);
    static constexpr int DTB = align128(T * CW * ESZ);
    static constexpr int BB = align128(T * kNState * ESZ);
    static constexpr int STAGE = XB + 2 * DTB + 2 * BB;   // x, dt, z, B, C
    static constexpr int BC32 = T * kNState * 2 * 4;      // one fp32 (B, C) pair buffer
    static constexpr int ED = T * CPW * 8;                // per warp: (delta, delta*u)
    static constexpr int DIR_BYTES = NS * STAGE + 2 * BC32;
    static constexpr int BAR_OFF = 2 * DIR_BYTES + 2 * NWD * ED;
    static constexpr int SMEM = BAR_OFF + 2 * NS * 8 + 128;  // + alignment slack
    static constexpr uint32_t TX_BASE = (uint32_t)(((T + 3) * CW + T * CW + 2 * T * kNState) * ESZ);
    static constexpr uint32_t TX_Z = (uint32_t)(T * CW * ESZ);
    static_assert((CW * ESZ) % 16 == 0, "TMA box rows must be whole 16-byte units");
};

// Per-lane state of one warp scanning one direction over CPW channels.
template <int G, int T, int NWD, int NS, typename Tin, int DIR>
struct TmaWorker {
    using Ge = TmaGeo<G, T, NWD, NS, Tin>;
    int lane, c, j, d, cc;  // cc: channel index inside the CTA tile
    bool dvalid;
    float A2[Ge::S];
    float w[4], cb, bias, Dd;
    float h[Ge::S];

    __device__ __forceinline__ void setup(const KParams& p, int ct0, int wg, int lane_) {
        lane = lane_;
        c = lane % Ge::CPW;
        j = lane / Ge::CPW;
        cc = wg * Ge::CPW + c;
        d = ct0 + cc;
        dvalid = d < p.D;
        const int64_t rd = (int64_t)DIR * p.D + (dvalid ? d : 0);
#pragma unroll
        for (int q = 0; q < Ge::S; ++q) {
            A2[q] = dvalid ? p.A[rd * kNState + j * Ge::S + q] * kLog2e : 0.f;
            h[q] = 0.f;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) w[k] = dvalid ? p.conv_w[rd * 4 + k] : 0.f;
        cb = (dvalid && p.conv_b) ? p.conv_b[rd] : 0.f;
        bias = dvalid ? p.dt_bias[rd] : 0.f;
        Dd = dvalid ? p.Dskip[rd] : 0.f;
    }

    // token of step s of chunk k
    __device__ __forceinline__ int64_t token(int k, int s) const {
        return DIR == 0 ? (int64_t)k * T + s : (int64_t)k * T + (T - 1 - s);
    }

    // conv + SiLU and softplus of this lane's steps; (delta, delta*u) to ed,
    // D*u to du.  Steps whose token is >= L become identity steps.
    __device__ __forceinline__ void elements(const Tin* xt, const Tin* dtt, int k, int64_t L, float2* ed,
                                             float (&du)[Ge::EPL]) {
#pragma unroll
        for (int e = 0; e < Ge::EPL; ++e) {
            const int s = j + G * e;
            const bool valid = token(k, s) < L;
            float cv = cb;
            if (DIR == 0) {
                // tile row rho holds token kT - 3 + rho: taps t-3..t are rows s..s+3
#pragma unroll
                for (int q = 0; q < 4; ++q) cv = fmaf(w[q], ldf(xt, (s + q) * Ge::CW + cc), cv);
            } else {
                // tile row rho holds token kT + rho; token t = kT + T-1-s; tap q reads t+3-q
#pragma unroll
                for (int q = 0; q < 4; ++q) cv = fmaf(w[q], ldf(xt, (T + 2 - s - q) * Ge::CW + cc), cv);
            }
            const int trow = DIR == 0 ? s : T - 1 - s;
            const float u = silu(cv);
            const float dl = softplus(ldf(dtt, trow * Ge::CW + cc) + bias);
            ed[s * Ge::CPW + c] = valid ? make_float2(dl, dl * u) : make_float2(0.f, 0.f);
            du[e] = valid ? Dd * u : 0.f;
        }
    }

    // Advance the state over the T steps; yv[e] = sum_n C h of step j + G*e.
    template <bool WITH_Y>
    __device__ __forceinline__ void scan(const float2* ed, const float* bc, float (&yv)[Ge::EPL]) {
#pragma unroll
        for (int e = 0; e < Ge::EPL; ++e) {
            float pp[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const int s = G * e + g;
                const int row = DIR == 0 ? s : T - 1 - s;
                const float2 q2 = ed[s * Ge::CPW + c];
                const float* bcr = bc + row * 2 * kNState + 2 * j * Ge::S;  // (B, C) pairs of my states
                float bcv[2 * Ge::S];
                load_states<2 * Ge::S>(bcr, bcv);
                float acc = 0.f;
#pragma unroll
                for (int q = 0; q < Ge::S; ++q) {
                    const float ea = ex2_approx(q2.x * A2[q]);
                    h[q] = fmaf(ea, h[q], q2.y * bcv[2 * q]);
                    if constexpr (WITH_Y) acc = fmaf(bcv[2 * q + 1], h[q], acc);
                }
                pp[g] = acc;
            }
            if constexpr (WITH_Y) yv[e] = group_transpose_reduce<G, Ge::CPW>(pp, j);
        }
    }
};

// Convert a chunk's B and C tiles (T x 16 each, token order) into fp32
// (B_n, C_n) pairs, cooperatively over `nthreads` threads.
template <int T, typename Tin>
__device__ __forceinline__ void convert_bc(const Tin* Bt, const Tin* Ct, float* bc, int tid, int nthreads) {
    for (int e = tid; e < T * kNState; e += nthreads) {
        bc[2 * e] = ldf(Bt, e);
        bc[2 * e + 1] = ldf(Ct, e);
    }
}

template <int G, int T, int NWD, int NS, typename Tin>
__device__ __forceinline__ void issue_chunk(const LayerMaps& maps, unsigned char* dir_base, uint64_t* full, int r,
                                            int i, int k, bool gated, int ct0, int b) {
    using Ge = TmaGeo<G, T, NWD, NS, Tin>;
    const int st = i % NS;
    unsigned char* sb = dir_base + st * Ge::STAGE;
    uint64_t* bar = full + st;
    mbar_arrive_expect_tx(bar, Ge::TX_BASE + (gated ? Ge::TX_Z : 0u));
    const int row0 = k * T;
    tma_load_3d(sb, &maps.x, bar, ct0, r == 0 ? row0 - 3 : row0, b);
    tma_load_3d(sb + Ge::XB, &maps.dt[r], bar, ct0, row0, b);
    if (gated) tma_load_3d(sb + Ge::XB + Ge::DTB, &maps.z, bar, ct0, row0, b);
    tma_load_3d(sb + Ge::XB + 2 * Ge::DTB, &maps.B[r], bar, 0, row0, b);
    tma_load_3d(sb + Ge::XB + 2 * Ge::DTB + Ge::BB, &maps.C[r], bar, 0, row0, b);
}

template <int G, int T, int NWD, int NS, typename Tin, typename Tout, int DIR>
__device__ __forceinline__ void layer_direction(const LayerMaps& maps, const KParams& p, unsigned char* base,
                                                int wg, int lane) {
    using Ge = TmaGeo<G, T, NWD, NS, Tin>;
    unsigned char* dir_base = base + DIR * Ge::DIR_BYTES;
    float* bc32 = reinterpret_cast<float*>(dir_base + NS * Ge::STAGE);
    float2* ed = reinterpret_cast<float2*>(base + 2 * Ge::DIR_BYTES + (DIR * NWD + wg) * Ge::ED);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + Ge::BAR_OFF) + DIR * NS;
    const int b = blockIdx.y;
    const int ct0 = blockIdx.x * Ge::CW;
    const int64_t L = p.L;
    const int D = p.D;
    const int nc = (int)((L + T - 1) / T);
    const int hF = nc / 2;
    const int meet = DIR == 0 ? hF : nc - hF;  // chunks before the meeting point
    const bool leader = (wg == 0 && lane == 0);
    const int gtid = wg * 32 + lane;
    const float scale = p.dir_scale[DIR];
    const float* WSr = p.ws;
    float* WSw = p.ws;
    Tout* OUT = static_cast<Tout*>(p.out);

    TmaWorker<G, T, NWD, NS, Tin, DIR> wk;
    wk.setup(p, ct0, wg, lane);

    if (leader) {
        for (int i = 0; i < NS && i < nc; ++i) {
            const int k = DIR == 0 ? i : nc - 1 - i;
            issue_chunk<G, T, NWD, NS, Tin>(maps, dir_base, full, DIR, i, k, i >= meet, ct0, b);
        }
    }

#pragma unroll 1
    for (int i = 0; i < nc; ++i) {
        const int k = DIR == 0 ? i : nc - 1 - i;
        const bool gated = i >= meet;
        if (i == meet) {
            __threadfence_block();
            named_bar_sync(3, 2 * NWD * 32);
        }
        const int st = i % NS;
        mbar_wait_bounded(full + st, (uint32_t)((i / NS) & 1));
        const unsigned char* sb = dir_base + st * Ge::STAGE;
        const Tin* xt = reinterpret_cast<const Tin*>(sb);
        const Tin* dtt = reinterpret_cast<const Tin*>(sb + Ge::XB);
        const Tin* zt = reinterpret_cast<const Tin*>(sb + Ge::XB + Ge::DTB);
        const Tin* Bt = reinterpret_cast<const Tin*>(sb + Ge::XB + 2 * Ge::DTB);
        const Tin* Ct = reinterpret_cast<const Tin*>(sb + Ge::XB + 2 * Ge::DTB + Ge::BB);
        float* bc = bc32 + (i & 1) * (T * kNState * 2);
        convert_bc<T, Tin>(Bt, Ct, bc, gtid, NWD * 32);
        named_bar_sync(1 + DIR, NWD * 32);
        if (leader && i >= 1 && i - 1 + NS < nc) {
            const int i2 = i - 1 + NS;
            issue_chunk<G, T, NWD, NS, Tin>(maps, dir_base, full, DIR, i2, DIR == 0 ? i2 : nc - 1 - i2,
                                            i2 >= meet, ct0, b);
        }
        // the partner's y over this chunk, fetched now and used after the scan
        float other[Ge::EPL];
#pragma unroll
        for (int e = 0; e < Ge::EPL; ++e) {
            const int64_t t = wk.token(k, wk.j + G * e);
            other[e] = (gated && t < L && wk.dvalid) ? WSr[((int64_t)b * L + t) * D + wk.d] : 0.f;
        }
        float du[Ge::EPL], yv[Ge::EPL];
        wk.elements(xt, dtt, k, L, ed, du);
        __syncwarp();
        wk.template scan<true>(ed, bc, yv);
#pragma unroll
        for (int e = 0; e < Ge::EPL; ++e) {
            const int s = wk.j + G * e;
            const int64_t t = wk.token(k, s);
            if (t < L && wk.dvalid) {
                const int64_t idx = ((int64_t)b * L + t) * D + wk.d;
                const float y = (yv[e] + du[e]) * scale;
                if (!gated) {
                    WSw[idx] = y;
                } else {
                    const int trow = DIR == 0 ? s : T - 1 - s;
                    stf(OUT, idx, (y + other[e]) * silu(ldf(zt, trow * Ge::CW + wk.cc)));
                }
            }
        }
        __syncwarp();
    }
    if (meet >= nc) {  // a single-chunk sequence: the reverse group meets after its only chunk
        __threadfence_block();
        named_bar_sync(3, 2 * NWD * 32);
    }
}

// Resident CTAs per SM the register budget is sized for (shared memory
// allows about this many at T = 32, bf16).
template <int G>
constexpr int layer_min_blocks() {
    return G >= 16 ? 4 : 3;
}

template <int G, int T, int NWD, int NS, typename Tin, typename Tout>
__global__ void __launch_bounds__(2 * NWD * 32, layer_min_blocks<G>())
    layer_tma_kernel(const __grid_constant__ LayerMaps maps, const KParams p) {
    using Ge = TmaGeo<G, T, NWD, NS, Tin>;
    extern __shared__ __align__(128) unsigned char smem_dyn[];
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 127) & ~static_cast<uintptr_t>(127));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        uint64_t* bars = reinterpret_cast<uint64_t*>(base + Ge::BAR_OFF);
        for (int i = 0; i < 2 * NS; ++i) mbar_init(bars + i, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (warp < NWD)
        layer_direction<G, T, NWD, NS, Tin, Tout, 0>(maps, p, base, warp, lane);
    else
        layer_direction<G, T, NWD, NS, Tin, Tout, 1>(maps, p, base, warp - NWD, lane);
}

// ---------------------------------------------------------------- prefix

// Forward scan over P = p.L tokens from zero; writes the final state and the
// last three x of the prefix.  One CTA = one batch row x CW channels, NWD
// warps, the same chunk ring as the layer (the reverse-direction half of the
// shared memory is unused).  C and z are not read.
template <int G, int T, int NWD, int NS, typename Tin>
__global__ void __launch_bounds__(NWD * 32) prefix_tma_kernel(const __grid_constant__ LayerMaps maps,
                                                              const KParams p) {
    using Ge = TmaGeo<G, T, NWD, NS, Tin>;
    extern __shared__ __align__(128) unsigned char smem_dyn[];
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 127) & ~static_cast<uintptr_t>(127));
    const int wg = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t* full = reinterpret_cast<uint64_t*>(base + Ge::BAR_OFF);
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) mbar_init(full + i, 1);
        fence_barrier_init();
    }
    __syncthreads();
    float* bc32 = reinterpret_cast<float*>(base + NS * Ge::STAGE);
    float2* ed = reinterpret_cast<float2*>(base + 2 * Ge::DIR_BYTES + wg * Ge::ED);
    const int b = blockIdx.y;
    const int ct0 = blockIdx.x * Ge::CW;
    const int64_t P = p.L;
    const int nc = (int)((P + T - 1) / T);
    const bool leader = (wg == 0 && lane == 0);
    constexpr uint32_t TX = (uint32_t)(((T + 3) * Ge::CW + T * Ge::CW + T * kNState) * Ge::ESZ);

    auto issue = [&](int i) {
        const int st = i % NS;
        unsigned char* sb = base + st * Ge::STAGE;
        uint64_t* bar = full + st;
        mbar_arrive_expect_tx(bar, TX);
        tma_load_3d(sb, &maps.x, bar, ct0, i * T - 3, b);
        tma_load_3d(sb + Ge::XB, &maps.dt[0], bar, ct0, i * T, b);
        tma_load_3d(sb + Ge::XB + 2 * Ge::DTB, &maps.B[0], bar, 0, i * T, b);
    };

    TmaWorker<G, T, NWD, NS, Tin, 0> wk;
    wk.setup(p, ct0, wg, lane);
    if (leader)
        for (int i = 0; i < NS && i < nc; ++i) issue(i);

#pragma unroll 1
    for (int i = 0; i < nc; ++i) {
        const int st = i % NS;
        mbar_wait_bounded(full + st, (uint32_t)((i / NS) & 1));
        const unsigned char* sb = base + st * Ge::STAGE;
        const Tin* xt = reinterpret_cast<const Tin*>(sb);
        const Tin* dtt = reinterpret_cast<const Tin*>(sb + Ge::XB);
        const Tin* Bt = reinterpret_cast<const Tin*>(sb + Ge::XB + 2 * Ge::DTB);
        float* bc = bc32 + (i & 1) * (T * kNState * 2);
        for (int e = wg * 32 + lane; e < T * kNState; e += NWD * 32) bc[2 * e] = ldf(Bt, e);
        named_bar_sync(1, NWD * 32);
        if (leader && i >= 1 && i - 1 + NS < nc) issue(i - 1 + NS);
        float du[Ge::EPL], yv[Ge::EPL];
        wk.elements(xt, dtt, i, P, ed, du);
        __syncwarp();
        wk.template scan<false>(ed, bc, yv);
        __syncwarp();
    }
    if (wk.dvalid) {
#pragma unroll
        for (int q = 0; q < Ge::S; ++q)
            p.h_out[((int64_t)b * p.D + wk.d) * kNState + wk.j * Ge::S + q] = wk.h[q];
        if (wk.j == 0) {
            const Tin* X = static_cast<const Tin*>(p.x);
            Tin* tail = static_cast<Tin*>(p.tail_out);
            for (int q = 0; q < 3; ++q) {
                const int64_t t = P - 3 + q;
                tail[((int64_t)b * 3 + q) * p.D + wk.d] =
                    t >= 0 ? X[((int64_t)b * P + t) * p.D + wk.d] : cvt_from<Tin>(0.f);
            }
        }
    }
}

}  // namespace bimamba

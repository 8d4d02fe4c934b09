// layer_split.cuh -- the bidirectional Mamba mixer layer for few channels
// ("DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone", §3.2
// Eq. (4)-(6)): batch 1 over a long sequence, where one lane per
// (channel, direction) chain would leave most of the GPU idle.
//
// Four lanes share a channel: lane j of the channel holds states
// [4j, 4j+4).  A warp covers 8 channels of one direction (lane = 4c + j);
// a CTA has NWD forward and NWD reverse warps over the same 8*NWD channels.
// Both directions cut the sequence into chunks of T tokens (chunk k = tokens
// [kT, kT+T)) and walk them in step space: step s of chunk k is token kT + s
// (forward) or kT + T-1-s (reverse), so the reverse conv is the causal conv
// over tokens read backwards -- nothing is flipped in memory.  Each chunk's
// x (with the 3-token conv halo), dt, B, C -- and z when the chunk is gated --
// arrive by 3-D TMA loads into an NS-stage ring per direction; a box reaching
// outside [0, L) reads zeros, the conv's zero padding at both ends.
//
// What each chunk moves through shared memory is kept small, since at batch
// 1 the shared-memory pipe rather than the special-function unit (MUFU) is
// the first to fill:
//  * B and C stay in the input dtype: a lane reads its 4 B and 4 C straight
//    from the TMA tile (two 8-byte loads for bf16) and widens them in
//    registers.
//  * The per-token work (conv + SiLU, softplus, D*u) of a chunk is spread
//    round-robin over the channel's 4 lanes (lane j takes steps j, j+4, ...)
//    and kept in registers.  A lane fetches the step size and drive of the
//    step it is scanning from the lane that computed them with a width-4
//    shuffle, and after every 4 steps a shuffle transpose-reduce of the
//    C.h partial sums leaves lane j with step 4e+j's sum -- the step whose
//    D*u it already holds.
// Steps whose token is >= L get delta = 0 and no drive, an exact identity.
//
// Full layer: the forward warps walk chunks 0..nc-1, the reverse warps
// nc-1..0.  Until they meet (the forward warps after nc/2 chunks) each
// stores its fp32 y to the workspace; after one CTA barrier each finishes
// the other half, adding the partner's y (fetched by cp.async) and applying
// the SiLU(z) gate.  Every token is gated once, by the direction that
// reaches it second.
#pragma once

#include "layer_tma.cuh"
#include "scan_kernels.cuh"
#include "tma_util.cuh"

namespace bimamba {

// XSM: the step sizes and drives reach the scanning lanes through a per-warp
// shared-memory buffer (one 8-byte load per step) instead of two shuffles,
// and D*u likewise, so the scan loop need not be unrolled (a smaller loop
// body stays in the instruction cache).
template <int T, int NWD, int NS, typename Tin, bool XSM = false>
struct SplitGeo {
    static_assert(T % 4 == 0 && T + 3 <= 256, "chunk");
    static_assert(NWD == 1 || NWD == 2, "warps per direction");
    static constexpr int G = 4;                            // lanes per channel
    static constexpr int S = 4;                            // states per lane
    static constexpr int CPW = 8;                          // channels per warp
    static constexpr int EPL = T / G;                      // steps per lane per chunk
    static constexpr int CW = NWD * CPW;                   // channels per CTA
    static constexpr int ESZ = (int)sizeof(Tin);
    static constexpr int XB = align128((T + 3) * CW * ESZ);
    static constexpr int DTB = align128(T * CW * ESZ);
    static constexpr int BB = align128(T * kNState * ESZ);
    static constexpr int STAGE = XB + 2 * DTB + 2 * BB;  // x, dt, z, B, C
    static constexpr int OWS = T * CPW * 4;               // per warp: partner's y of a chunk
    static constexpr int EDX = XSM ? T * CPW * 8 : 0;     // per warp: (delta, delta*u) of the chunk's steps
    static constexpr int EDU = XSM ? T * CPW * 4 : 0;     // per warp: D*u of the chunk's steps
    static constexpr int WARP_BYTES = OWS + EDX + EDU;
    static constexpr int DIR_BYTES = NS * STAGE;
    static constexpr int WARP_OFF = 2 * DIR_BYTES;
    static constexpr int BAR_OFF = WARP_OFF + 2 * NWD * WARP_BYTES;
    static constexpr int SMEM = BAR_OFF + 2 * NS * 8 + 128;  // + alignment slack
    static constexpr uint32_t TX_BASE = (uint32_t)(((T + 3) * CW + T * CW + 2 * T * kNState) * ESZ);
    static constexpr uint32_t TX_Z = (uint32_t)(T * CW * ESZ);
    static_assert((CW * ESZ) % 16 == 0, "TMA box rows must be whole 16-byte units");
};

// The four B (or C) of states [4j, 4j+4) of one token row, as fp32.
__device__ __forceinline__ void load_quad(const __nv_bfloat16* row, int j, float (&v)[4]) {
    const uint2 w = *reinterpret_cast<const uint2*>(row + 4 * j);
    // bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32
    v[0] = __uint_as_float(w.x << 16);
    v[1] = __uint_as_float(w.x & 0xffff0000u);
    v[2] = __uint_as_float(w.y << 16);
    v[3] = __uint_as_float(w.y & 0xffff0000u);
}
__device__ __forceinline__ void load_quad(const float* row, int j, float (&v)[4]) {
    const float4 f = *reinterpret_cast<const float4*>(row + 4 * j);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}

// Transpose-reduce over the 4 lanes of a channel (lanes 4c..4c+3): on entry
// p[g] is this lane's partial sum for step g of a group of 4; on return lane
// j holds the full sum for step j.
__device__ __forceinline__ float reduce4(const float (&p)[4], int j) {
    const bool hi2 = (j & 2) != 0;
    const float k0 = hi2 ? p[2] : p[0], s0 = hi2 ? p[0] : p[2];
    const float k1 = hi2 ? p[3] : p[1], s1 = hi2 ? p[1] : p[3];
    const float q0 = k0 + __shfl_xor_sync(0xffffffffu, s0, 2);
    const float q1 = k1 + __shfl_xor_sync(0xffffffffu, s1, 2);
    const bool hi1 = (j & 1) != 0;
    const float k = hi1 ? q1 : q0, s = hi1 ? q0 : q1;
    return k + __shfl_xor_sync(0xffffffffu, s, 1);
}

template <int T, int NWD, int NS, typename Tin, int DIR, bool XSM>
struct SplitWorker {
    using Ge = SplitGeo<T, NWD, NS, Tin, XSM>;
    int c, j, cc, d;  // cc: channel inside the CTA tile; d: global channel
    bool dvalid;
    float A2[4];      // A * log2(e) of this lane's states
    float w[4], cb, bias, Dd;
    float h[4];
    float dsum;       // step sizes of this lane's steps so far (carries)
    // this lane's steps j + 4e of the current chunk
    float dl[Ge::EPL], du[Ge::EPL], Du[Ge::EPL];

    __device__ __forceinline__ void setup(const KParams& p, int ct0, int wg, int lane) {
        c = lane >> 2;
        j = lane & 3;
        cc = wg * Ge::CPW + c;
        d = ct0 + cc;
        dvalid = d < p.D;
        const int64_t rd = (int64_t)DIR * p.D + (dvalid ? d : 0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            A2[q] = dvalid ? p.A[rd * kNState + 4 * j + q] * kLog2e : 0.f;
            h[q] = 0.f;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) w[k] = dvalid ? p.conv_w[rd * 4 + k] : 0.f;
        cb = (dvalid && p.conv_b) ? p.conv_b[rd] : 0.f;
        bias = dvalid ? p.dt_bias[rd] : 0.f;
        Dd = dvalid ? p.Dskip[rd] : 0.f;
        dsum = 0.f;
    }

    // tile row (token - kT) of step s
    static __device__ __forceinline__ int row_of(int s) { return DIR == 0 ? s : T - 1 - s; }

    // conv + SiLU, softplus and D*u of this lane's steps j + 4e; steps
    // outside [s_lo, s_hi) (tokens >= L) become identity steps.  DSUM: also
    // add the valid step sizes to dsum.
    template <bool DSUM>
    __device__ __forceinline__ void elements(const Tin* xt, const Tin* dtt, int s_lo, int s_hi, float2* edx) {
#pragma unroll
        for (int e = 0; e < Ge::EPL; ++e) {
            const int s = j + 4 * e;
            // step s-3+q is x-tile row s+q (forward: the tile starts 3 tokens
            // early) or T+2-s-q (reverse)
            float cv = cb;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int xr = DIR == 0 ? s + q : T + 2 - s - q;
                cv = fmaf(w[q], ldf(xt, xr * Ge::CW + cc), cv);
            }
            const float u = silu(cv);
            const float dlt = softplus(ldf(dtt, row_of(s) * Ge::CW + cc) + bias);
            const bool valid = s >= s_lo && s < s_hi;
            dl[e] = valid ? dlt : 0.f;
            du[e] = valid ? dlt * u : 0.f;
            Du[e] = valid ? Dd * u : 0.f;
            if constexpr (XSM) {
                edx[s * Ge::CPW + c] = make_float2(dl[e], du[e]);
                reinterpret_cast<float*>(edx + T * Ge::CPW)[s * Ge::CPW + c] = Du[e];
            }
            if constexpr (DSUM) dsum += dl[e];
        }
    }

    // States over steps 4e..4e+3; returns sum_n C h of step 4e + j.  In
    // phases: every load of the four steps, then their 16 exps (which depend
    // only on the step sizes), then the dependent updates -- so the exps can
    // keep the special-function unit busy while the loads and the state
    // chain wait.
    __device__ __forceinline__ float step_group_phased(int e, const Tin* Bt, const Tin* Ct, const float2* edx) {
        float dq[4], uq[4], bv[4][4], cv[4][4], ea[4][4];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int s = 4 * e + g;
            if constexpr (XSM) {
                const float2 q = edx[s * Ge::CPW + c];
                dq[g] = q.x;
                uq[g] = q.y;
            } else {
                dq[g] = __shfl_sync(0xffffffffu, dl[e], g, 4);
                uq[g] = __shfl_sync(0xffffffffu, du[e], g, 4);
            }
            load_quad(Bt + row_of(s) * kNState, j, bv[g]);
            load_quad(Ct + row_of(s) * kNState, j, cv[g]);
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const float2 dd = make_float2(dq[g], dq[g]);
#pragma unroll
            for (int q = 0; q < 4; q += 2) {
                const float2 v = mul2(dd, make_float2(A2[q], A2[q + 1]));
                ea[g][q] = ex2_approx(v.x);
                ea[g][q + 1] = ex2_approx(v.y);
            }
        }
        float pp[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const float2 uu = make_float2(uq[g], uq[g]);
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 4; q += 2) {
                const float2 drive = mul2(uu, make_float2(bv[g][q], bv[g][q + 1]));
                const float2 hh = fma2(make_float2(ea[g][q], ea[g][q + 1]), make_float2(h[q], h[q + 1]), drive);
                h[q] = hh.x;
                h[q + 1] = hh.y;
                acc = fma2(make_float2(cv[g][q], cv[g][q + 1]), hh, acc);
            }
            pp[g] = acc.x + acc.y;
        }
        return reduce4(pp, j);
    }

    __device__ __forceinline__ float step_group(int e, const Tin* Bt, const Tin* Ct, const float2* edx) {
        float pp[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int s = 4 * e + g;
            float dq, uq;
            if constexpr (XSM) {
                const float2 q = edx[s * Ge::CPW + c];
                dq = q.x;
                uq = q.y;
            } else {
                dq = __shfl_sync(0xffffffffu, dl[e], g, 4);
                uq = __shfl_sync(0xffffffffu, du[e], g, 4);
            }
            float bv[4], cv[4];
            load_quad(Bt + row_of(s) * kNState, j, bv);
            load_quad(Ct + row_of(s) * kNState, j, cv);
            const float2 dd = make_float2(dq, dq);
            const float2 uu = make_float2(uq, uq);
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 4; q += 2) {
                const float2 v = mul2(dd, make_float2(A2[q], A2[q + 1]));
                const float2 ea = make_float2(ex2_approx(v.x), ex2_approx(v.y));
                const float2 drive = mul2(uu, make_float2(bv[q], bv[q + 1]));
                const float2 hh = fma2(ea, make_float2(h[q], h[q + 1]), drive);
                h[q] = hh.x;
                h[q + 1] = hh.y;
                acc = fma2(make_float2(cv[q], cv[q + 1]), hh, acc);
            }
            pp[g] = acc.x + acc.y;
        }
        return reduce4(pp, j);
    }
};

template <int T, int NWD, int NS, typename Tin>
__device__ __forceinline__ void split_issue(const LayerMaps& maps, unsigned char* dir_base, uint64_t* full, int r,
                                            int i, int k, bool gated, int ct0, int b, int starve) {
    using Ge = SplitGeo<T, NWD, NS, Tin>;  // the stage layout does not depend on XSM
    if (starve) return;
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

// CARRY: start from p.carry_in, report p.carry_out and p.delta_sum (each where non-null).
template <int T, int NWD, int NS, typename Tin, typename Tout, int DIR, bool CARRY, bool XSM, bool PHASED>
__device__ __forceinline__ void split_direction(const LayerMaps& maps, const KParams& p, unsigned char* base,
                                                int wg, int lane) {
    using Ge = SplitGeo<T, NWD, NS, Tin, XSM>;
    using Wk = SplitWorker<T, NWD, NS, Tin, DIR, XSM>;
    unsigned char* dir_base = base + DIR * Ge::DIR_BYTES;
    unsigned char* wbase = base + Ge::WARP_OFF + (DIR * NWD + wg) * Ge::WARP_BYTES;
    float* ows = reinterpret_cast<float*>(wbase);
    float2* edx = reinterpret_cast<float2*>(wbase + Ge::OWS);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + Ge::BAR_OFF) + DIR * NS;
    const int b = blockIdx.y;
    const int ct0 = blockIdx.x * Ge::CW;
    const int64_t L = p.L;
    const int D = p.D;
    const int nc = (int)((L + T - 1) / T);
    const int meet = DIR == 0 ? nc / 2 : nc - nc / 2;  // chunks before the meeting point
    const bool leader = (wg == 0 && lane == 0);
    const float scale = p.dir_scale[DIR];
    const int c0w = ct0 + wg * Ge::CPW;  // first channel of this warp

    Wk wk;
    wk.setup(p, ct0, wg, lane);
    if (CARRY && p.carry_in[DIR] && wk.dvalid) {
        const float* ci = p.carry_in[DIR] + ((int64_t)b * D + wk.d) * kNState + 4 * wk.j;
#pragma unroll
        for (int q = 0; q < 4; ++q) wk.h[q] = ci[q];
    }

    if (leader)
        for (int i = 0; i < NS && i < nc; ++i)
            split_issue<T, NWD, NS, Tin>(maps, dir_base, full, DIR, i, DIR == 0 ? i : nc - 1 - i, i >= meet, ct0,
                                         b, p.starve);

#pragma unroll 1
    for (int i = 0; i < nc; ++i) {
        const int k = DIR == 0 ? i : nc - 1 - i;
        const bool gated = i >= meet;
        if (i == meet) {
            __threadfence_block();
            named_bar_sync(3, 2 * NWD * 32);
        }
        const int nvalid = (int)((L - (int64_t)k * T < T) ? (L - (int64_t)k * T) : T);
        const int s_lo = DIR == 0 ? 0 : T - nvalid;
        const int s_hi = DIR == 0 ? nvalid : T;
        const int64_t chunk_row = (int64_t)b * L + (int64_t)k * T;  // global row of the chunk's token kT

        // partner's y of this chunk -> shared memory, 16-byte pieces of 4
        // channels (d_inner is a multiple of 4 here and c0w of 8)
        if (gated) {
            for (int e = lane; e < T * 2; e += 32) {
                const int r = e >> 1, q = e & 1;
                const bool ok = (int64_t)k * T + r < L && c0w + 4 * q < D;
                const float* src = p.ws + (chunk_row + (ok ? r : 0)) * D + (ok ? c0w + 4 * q : 0);
                cp_async<16>(ows + r * Ge::CPW + 4 * q, src, ok);
            }
            cp_async_commit();
        }

        const int st = i % NS;
        mbar_wait_bounded(full + st, (uint32_t)((i / NS) & 1), p.wait_limit);
        const unsigned char* sb = dir_base + st * Ge::STAGE;
        const Tin* xt = reinterpret_cast<const Tin*>(sb);
        const Tin* dtt = reinterpret_cast<const Tin*>(sb + Ge::XB);
        const Tin* zt = reinterpret_cast<const Tin*>(sb + Ge::XB + Ge::DTB);
        const Tin* Bt = reinterpret_cast<const Tin*>(sb + Ge::XB + 2 * Ge::DTB);
        const Tin* Ct = reinterpret_cast<const Tin*>(sb + Ge::XB + 2 * Ge::DTB + Ge::BB);

        wk.template elements<CARRY>(xt, dtt, s_lo, s_hi, edx);
        if (gated) cp_async_wait_all();
        if (gated || XSM) __syncwarp();

        float* wsw = p.ws + chunk_row * D + wk.d;
        Tout* outw = static_cast<Tout*>(p.out) + chunk_row * D + wk.d;
        auto finish = [&](int e, float yr, float du_own) {
            const int s = 4 * e + wk.j;
            if (s >= s_lo && s < s_hi && wk.dvalid) {
                const int tr = Wk::row_of(s);  // token - kT
                const float y = (yr + du_own) * scale;
                if (!gated) {
                    wsw[(int64_t)tr * D] = y;
                } else {
                    const float zv = ldf(zt, tr * Ge::CW + wk.cc);
                    stf(outw, (int64_t)tr * D, (y + ows[tr * Ge::CPW + wk.c]) * silu(zv));
                }
            }
        };
        if constexpr (XSM) {
            const float* edu = reinterpret_cast<const float*>(edx + T * Ge::CPW);
#pragma unroll 2
            for (int e = 0; e < Ge::EPL; ++e) {
                const float yr = PHASED ? wk.step_group_phased(e, Bt, Ct, edx) : wk.step_group(e, Bt, Ct, edx);
                finish(e, yr, edu[(4 * e + wk.j) * Ge::CPW + wk.c]);
            }
        } else {
#pragma unroll
            for (int e = 0; e < Ge::EPL; ++e) {
                const float yr = PHASED ? wk.step_group_phased(e, Bt, Ct, edx) : wk.step_group(e, Bt, Ct, edx);
                finish(e, yr, wk.Du[e]);
            }
        }
        // every warp of this direction is done with stage st: refill it
        if constexpr (NWD == 1)
            __syncwarp();
        else
            named_bar_sync(1 + DIR, NWD * 32);
        if (leader && i + NS < nc)
            split_issue<T, NWD, NS, Tin>(maps, dir_base, full, DIR, i + NS, DIR == 0 ? i + NS : nc - 1 - i - NS,
                                         i + NS >= meet, ct0, b, p.starve);
    }
    if (meet >= nc) {  // a single-chunk sequence: the reverse warps meet after their only chunk
        __threadfence_block();
        named_bar_sync(3, 2 * NWD * 32);
    }
    if (CARRY && p.carry_out[DIR] && wk.dvalid) {
        float* co = p.carry_out[DIR] + ((int64_t)b * D + wk.d) * kNState + 4 * wk.j;
#pragma unroll
        for (int q = 0; q < 4; ++q) co[q] = wk.h[q];
    }
    if (CARRY && p.delta_sum[DIR]) {  // the 4 lanes of a channel are adjacent
        float ds = wk.dsum;
        ds += __shfl_xor_sync(0xffffffffu, ds, 1);
        ds += __shfl_xor_sync(0xffffffffu, ds, 2);
        if (wk.j == 0 && wk.dvalid) p.delta_sum[DIR][(int64_t)b * D + wk.d] = ds;
    }
}

template <int T, int NWD, int NS, typename Tin, typename Tout, bool CARRY = false, bool XSM = false,
          bool PHASED = false>
__global__ void __launch_bounds__(2 * NWD * 32) layer_split_kernel(const __grid_constant__ LayerMaps maps,
                                                                   const KParams p) {
    using Ge = SplitGeo<T, NWD, NS, Tin, XSM>;
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
        split_direction<T, NWD, NS, Tin, Tout, 0, CARRY, XSM, PHASED>(maps, p, base, warp, lane);
    else
        split_direction<T, NWD, NS, Tin, Tout, 1, CARRY, XSM, PHASED>(maps, p, base, warp - NWD, lane);
}

}  // namespace bimamba

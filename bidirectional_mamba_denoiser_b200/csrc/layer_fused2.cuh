// layer_fused2.cuh -- per-token fused kernel of the bidirectional Mamba mixer
// layer for many channels, organised in phases per chunk ("DiffuMamba:
// High-Throughput Diffusion LMs with Mamba Backbone", §3.2 Eq. (4)-(6)).
//
// A warp covers 32 channels of one batch row in one direction; lane l owns
// channel ct0 + l for the per-token work (conv + SiLU, softplus, D skip,
// output).  Lanes pair up (l, l ^ 1): lane j of a pair holds states
// [8j, 8j+8) of its own channel and of its partner's, so every B and C it
// loads serves two channels, and one shuffle completes each channel's C.h
// sum.
//
// Per chunk of T tokens, after its tiles have landed:
//  1. B and C are widened to fp32 once ([T][B 16 | C 16], shared by the warp);
//  2. every lane computes the per-token work of its channel for all T steps
//     -- T independent chains of conv, SiLU and softplus, so the
//     special-function unit has work in flight -- into a per-warp buffer
//     (step size, drive, D*u);
//  3. the scan walks the T steps with every step size already at hand (its
//     own and its partner's read from the buffer), so each step's 16 exps
//     can issue as soon as the unit is free; the loop is not unrolled, which
//     keeps its body in the instruction cache.
// A CTA is one forward and one reverse warp over the same 32 channels; each
// warp streams chunks of x (+3-token conv halo), dt, B, C (and z when gated)
// through its own NS-stage TMA ring; boxes reaching outside [0, L) read
// zeros, the conv's zero padding.  Each direction stores its fp32 y over its
// first half to the workspace, the two warps meet at one barrier, and each
// finishes the other half with the partner's y (cp.async) and the SiLU(z)
// gate.
#pragma once

#include "layer_fused.cuh"
#include "scan_kernels.cuh"
#include "tma_util.cuh"

namespace bimamba {

template <int T, int NS, typename Tin>
struct Fused2Geo {
    static_assert(T == 8 || T == 16, "chunk");
    static constexpr int CW = 32;
    static constexpr int ESZ = (int)sizeof(Tin);
    static constexpr int XB = (((T + 3) * CW * ESZ) + 127) & ~127;
    static constexpr int DTB = ((T * CW * ESZ) + 127) & ~127;
    static constexpr int BB = ((T * kNState * ESZ) + 127) & ~127;
    static constexpr int STAGE = XB + 2 * DTB + 2 * BB;  // x, dt, z, B, C
    static constexpr int OWS = T * CW * 4;               // partner's y of a chunk
    static constexpr int BCF = T * 2 * kNState * 4;      // fp32 B | C rows of a chunk
    static constexpr int ED = T * CW * 8;                // (delta, delta*u) of the chunk's steps
    static constexpr int EDU = T * CW * 4;               // D*u of the chunk's steps
    static constexpr int WARP_BYTES = NS * STAGE + OWS + BCF + ED + EDU;
    static constexpr int BAR_OFF = 2 * WARP_BYTES;
    static constexpr int SMEM = BAR_OFF + 2 * NS * 8 + 128;
    static constexpr uint32_t TX_BASE = (uint32_t)(((T + 3) * CW + T * CW + 2 * T * kNState) * ESZ);
    static constexpr uint32_t TX_Z = (uint32_t)(T * CW * ESZ);
};

template <int T, int NS, typename Tin>
__device__ __forceinline__ void fused2_issue(const FusedMaps& maps, unsigned char* wbase, uint64_t* full, int r,
                                             int i, int k, bool gated, int ct0, int b, int starve) {
    using Ge = Fused2Geo<T, NS, Tin>;
    if (starve) return;
    const int st = i % NS;
    unsigned char* sb = wbase + st * Ge::STAGE;
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
template <int T, int NS, typename Tin, typename Tout, int DIR, bool CARRY>
__device__ __forceinline__ void fused2_direction(const FusedMaps& maps, const KParams& p, unsigned char* base,
                                                 int lane) {
    using Ge = Fused2Geo<T, NS, Tin>;
    unsigned char* wbase = base + DIR * Ge::WARP_BYTES;
    float* ows = reinterpret_cast<float*>(wbase + NS * Ge::STAGE);
    float* bcf = reinterpret_cast<float*>(wbase + NS * Ge::STAGE + Ge::OWS);
    float2* ed = reinterpret_cast<float2*>(wbase + NS * Ge::STAGE + Ge::OWS + Ge::BCF);
    float* edu = reinterpret_cast<float*>(wbase + NS * Ge::STAGE + Ge::OWS + Ge::BCF + Ge::ED);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + Ge::BAR_OFF) + DIR * NS;
    const int b = blockIdx.y;
    const int ct0 = blockIdx.x * Ge::CW;
    const int64_t L = p.L;
    const int D = p.D;
    const int nc = (int)((L + T - 1) / T);
    const int meet = DIR == 0 ? nc / 2 : nc - nc / 2;
    const float scale = p.dir_scale[DIR];

    // own channel d, partner channel d ^ 1; states [8j, 8j+8) of both
    const int j = lane & 1;
    const int d = ct0 + lane, dp = ct0 + (lane ^ 1);
    const bool dvalid = d < D, pvalid = dp < D;
    float A2o[8], A2p[8], ho[8], hp[8];
    float w[4], cb, bias, Dd;
    {
        const int64_t ro = (int64_t)DIR * D + (dvalid ? d : 0);
        const int64_t rp = (int64_t)DIR * D + (pvalid ? dp : 0);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            A2o[q] = dvalid ? p.A[ro * kNState + 8 * j + q] * kLog2e : 0.f;
            A2p[q] = pvalid ? p.A[rp * kNState + 8 * j + q] * kLog2e : 0.f;
            ho[q] = 0.f;
            hp[q] = 0.f;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) w[k] = dvalid ? p.conv_w[ro * 4 + k] : 0.f;
        cb = (dvalid && p.conv_b) ? p.conv_b[ro] : 0.f;
        bias = dvalid ? p.dt_bias[ro] : 0.f;
        Dd = dvalid ? p.Dskip[ro] : 0.f;
        if (CARRY && p.carry_in[DIR]) {
            const float* ci = p.carry_in[DIR] + (int64_t)b * D * kNState;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (dvalid) ho[q] = ci[(int64_t)d * kNState + 8 * j + q];
                if (pvalid) hp[q] = ci[(int64_t)dp * kNState + 8 * j + q];
            }
        }
    }
    float dsum = 0.f;  // step sizes of the own channel so far

    if (lane == 0)
        for (int i = 0; i < NS && i < nc; ++i)
            fused2_issue<T, NS, Tin>(maps, wbase, full, DIR, i, DIR == 0 ? i : nc - 1 - i, i >= meet, ct0, b,
                                     p.starve);

#pragma unroll 1
    for (int i = 0; i < nc; ++i) {
        const int k = DIR == 0 ? i : nc - 1 - i;
        const bool gated = i >= meet;
        if (i == meet) {
            __threadfence_block();
            named_bar_sync(1, 64);
        }
        const int nvalid = (int)((L - (int64_t)k * T < T) ? (L - (int64_t)k * T) : T);
        const int s_lo = DIR == 0 ? 0 : T - nvalid;
        const int s_hi = DIR == 0 ? nvalid : T;
        const int64_t chunk_row = (int64_t)b * L + (int64_t)k * T;
        if (gated) {
            // partner's y: T rows x 32 channels, 16-byte pieces (D % 4 == 0 here)
            for (int e = lane; e < T * 8; e += 32) {
                const int r = e >> 3, q = e & 7;
                const bool ok = (int64_t)k * T + r < L && ct0 + 4 * q < D;
                const float* src = p.ws + (chunk_row + (ok ? r : 0)) * D + (ok ? ct0 + 4 * q : 0);
                cp_async<16>(ows + r * Ge::CW + 4 * q, src, ok);
            }
            cp_async_commit();
        }
        const int st = i % NS;
        mbar_wait_bounded(full + st, (uint32_t)((i / NS) & 1), p.wait_limit);
        const unsigned char* sb = wbase + st * Ge::STAGE;
        const Tin* xt = reinterpret_cast<const Tin*>(sb);
        const Tin* dtt = reinterpret_cast<const Tin*>(sb + Ge::XB);
        const Tin* zt = reinterpret_cast<const Tin*>(sb + Ge::XB + Ge::DTB);
        const Tin* Bt = reinterpret_cast<const Tin*>(sb + Ge::XB + 2 * Ge::DTB);
        const Tin* Ct = reinterpret_cast<const Tin*>(sb + Ge::XB + 2 * Ge::DTB + Ge::BB);

        // 1. B | C rows as fp32
        fused_convert_bc<T, Tin>(Bt, Ct, bcf, lane, true);

        // 2. per-token work of the own channel for the chunk's T steps (step s:
        // token kT + s forward, kT + T-1-s reverse; the forward x tile starts
        // 3 tokens early)
        {
            float x0 = ldf(xt, (DIR == 0 ? 0 : T + 2) * Ge::CW + lane);
            float x1 = ldf(xt, (DIR == 0 ? 1 : T + 1) * Ge::CW + lane);
            float x2 = ldf(xt, (DIR == 0 ? 2 : T) * Ge::CW + lane);
#pragma unroll
            for (int s = 0; s < T; ++s) {
                const float x3 = ldf(xt, (DIR == 0 ? s + 3 : T - 1 - s) * Ge::CW + lane);
                float cv = fmaf(w[0], x0, cb);
                cv = fmaf(w[1], x1, cv);
                cv = fmaf(w[2], x2, cv);
                cv = fmaf(w[3], x3, cv);
                x0 = x1; x1 = x2; x2 = x3;
                const float u = silu(cv);
                const float dlt = softplus(ldf(dtt, (DIR == 0 ? s : T - 1 - s) * Ge::CW + lane) + bias);
                const bool valid = s >= s_lo && s < s_hi;
                ed[s * Ge::CW + lane] = valid ? make_float2(dlt, dlt * u) : make_float2(0.f, 0.f);
                edu[s * Ge::CW + lane] = valid ? Dd * u : 0.f;
                if constexpr (CARRY) dsum += valid ? dlt : 0.f;
            }
        }
        if (gated) cp_async_wait_all();
        __syncwarp();

        // 3. the scan
        float* wsw = p.ws + chunk_row * D + d;
        Tout* outw = static_cast<Tout*>(p.out) + chunk_row * D + d;
#pragma unroll 1
        for (int s = 0; s < T; ++s) {
            const int row = DIR == 0 ? s : T - 1 - s;
            const float2 eo = ed[s * Ge::CW + lane], ep = ed[s * Ge::CW + (lane ^ 1)];
            float bv[8], cvv[8];
            load_states<8>(bcf + row * 2 * kNState + 8 * j, bv);
            load_states<8>(bcf + row * 2 * kNState + kNState + 8 * j, cvv);
            const float2 ddo = make_float2(eo.x, eo.x), uuo = make_float2(eo.y, eo.y);
            const float2 ddp = make_float2(ep.x, ep.x), uup = make_float2(ep.y, ep.y);
            float2 ao[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            float2 ap[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
            for (int q = 0; q < 8; q += 2) {
                const float2 bq = make_float2(bv[q], bv[q + 1]);
                const float2 cq = make_float2(cvv[q], cvv[q + 1]);
                const float2 vo = mul2(ddo, make_float2(A2o[q], A2o[q + 1]));
                const float2 vp = mul2(ddp, make_float2(A2p[q], A2p[q + 1]));
                const float2 xo = make_float2(ex2_approx(vo.x), ex2_approx(vo.y));
                const float2 xp = make_float2(ex2_approx(vp.x), ex2_approx(vp.y));
                const float2 no = fma2(xo, make_float2(ho[q], ho[q + 1]), mul2(uuo, bq));
                const float2 np = fma2(xp, make_float2(hp[q], hp[q + 1]), mul2(uup, bq));
                ho[q] = no.x; ho[q + 1] = no.y;
                hp[q] = np.x; hp[q + 1] = np.y;
                ao[(q >> 1) & 1] = fma2(cq, no, ao[(q >> 1) & 1]);
                ap[(q >> 1) & 1] = fma2(cq, np, ap[(q >> 1) & 1]);
            }
            // own channel: my 8 states plus the partner's 8 states of my channel
            const float mine = (ao[0].x + ao[1].x) + (ao[0].y + ao[1].y);
            const float theirs = (ap[0].x + ap[1].x) + (ap[0].y + ap[1].y);
            const float yr = mine + __shfl_xor_sync(0xffffffffu, theirs, 1);
            const float y = (yr + edu[s * Ge::CW + lane]) * scale;
            if (s >= s_lo && s < s_hi && dvalid) {
                if (!gated) {
                    wsw[(int64_t)row * D] = y;
                } else {
                    const float zv = ldf(zt, row * Ge::CW + lane);
                    stf(outw, (int64_t)row * D, (y + ows[row * Ge::CW + lane]) * silu(zv));
                }
            }
        }
        __syncwarp();  // the stage, the fp32 rows and ows are free for the next chunk
        if (lane == 0 && i + NS < nc) {
            const int i2 = i + NS;
            fused2_issue<T, NS, Tin>(maps, wbase, full, DIR, i2, DIR == 0 ? i2 : nc - 1 - i2, i2 >= meet, ct0, b,
                                     p.starve);
        }
    }
    if (meet >= nc) {  // single chunk: the reverse warp meets after it
        __threadfence_block();
        named_bar_sync(1, 64);
    }
    if (CARRY && p.carry_out[DIR]) {
        float* co = p.carry_out[DIR] + (int64_t)b * D * kNState;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if (dvalid) co[(int64_t)d * kNState + 8 * j + q] = ho[q];
            if (pvalid) co[(int64_t)dp * kNState + 8 * j + q] = hp[q];
        }
    }
    if (CARRY && p.delta_sum[DIR] && dvalid) p.delta_sum[DIR][(int64_t)b * D + d] = dsum;
}

template <int T, int NS, typename Tin, typename Tout, bool CARRY = false>
__global__ void __launch_bounds__(64, 8) fused2_layer_kernel(const __grid_constant__ FusedMaps maps, const KParams p) {
    using Ge = Fused2Geo<T, NS, Tin>;
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
    if (warp == 0)
        fused2_direction<T, NS, Tin, Tout, 0, CARRY>(maps, p, base, lane);
    else
        fused2_direction<T, NS, Tin, Tout, 1, CARRY>(maps, p, base, lane);
}

}  // namespace bimamba

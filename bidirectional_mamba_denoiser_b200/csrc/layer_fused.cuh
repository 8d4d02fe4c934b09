// layer_fused.cuh -- per-token fused kernels of the bidirectional Mamba mixer
// layer for problems with many channels ("DiffuMamba: High-Throughput
// Diffusion LMs with Mamba Backbone", §3.2 Eq. (4)-(6); the forward prefix
// scan is the cache of §4.3).
//
// A warp covers 32 channels of one batch row in one direction; lane l owns
// channel ct0 + l for the per-token work (conv + SiLU, softplus, D skip,
// output).  For the scan the 32 lanes form groups of G adjacent lanes; a
// group covers the G channels of its lanes, and lane j of the group holds
// states [jS, jS+S) (S = 16/G) of all G channels.  Every B_n and C_n a lane
// loads is therefore used for G channels, which cuts the shared-memory
// traffic per state update by G against one channel per lane, while each
// lane still computes exactly one channel's per-token work.  Per token the
// group gathers its G step sizes with width-G shuffles, each lane updates
// G x S states (packed f32x2 arithmetic, one MUFU exp2 each), and a
// transpose-reduce over the group leaves lane j with sum_n C h of its own
// channel.
//
// A CTA is one forward and one reverse warp over the same 32 channels.  Each
// warp streams 16-token chunks of x (+3-token conv halo), dt, B, C (and z
// when gated) through its own 2-stage TMA ring; boxes reaching outside
// [0, L) read zeros, the conv's zero padding.  As in the chunked kernels,
// each direction stores its fp32 y over its first half to the workspace, the
// two warps meet at one barrier, and each finishes the other half with the
// partner's y (cp.async) and the SiLU(z) gate.
#pragma once

#include "scan_kernels.cuh"
#include "tma_util.cuh"

namespace bimamba {

struct FusedMaps {
    CUtensorMap x;      // [batch][L][D]    box {32, T+3, 1}
    CUtensorMap z;      // [batch][L][D]    box {32, T, 1}
    CUtensorMap dt[2];  // [batch][L][D]    box {32, T, 1}
    CUtensorMap B[2];   // [batch][L][16]   box {16, T, 1}; with BCQ: fp32 quads [batch][L][32], box {32, T, 1}
    CUtensorMap C[2];   // [batch][L][16]   box {16, T, 1}; unused with BCQ
};

// F32BC: B and C are widened to fp32 once per chunk (into a per-warp buffer)
// instead of at every use.  BCQ (one lane per channel): B and C arrive
// already widened to fp32 quads (B_2q, B_2q+1, C_2q, C_2q+1) per token,
// written once per call by widen_bc_kernel, and are read from the TMA tile.
template <int G, typename Tin, bool F32BC = false, bool BCQ = false>
struct FusedGeo {
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "lanes per group");
    static constexpr int T = 16;                // tokens per chunk
    static constexpr int NS = 2;                // ring stages per direction
    static constexpr int S = kNState / G;       // states per lane
    static constexpr int CW = 32;               // channels per warp (and CTA)
    static constexpr int ESZ = (int)sizeof(Tin);
    static constexpr int XB = (((T + 3) * CW * ESZ) + 127) & ~127;
    static constexpr int DTB = ((T * CW * ESZ) + 127) & ~127;
    static constexpr int BB = ((T * kNState * ESZ) + 127) & ~127;
    static constexpr int BQB = ((T * 2 * kNState * 4) + 127) & ~127;  // the fp32 quads of a chunk
    static constexpr int STAGE = XB + 2 * DTB + (BCQ ? BQB : 2 * BB);  // x, dt, z, B and C
    static constexpr int OWS = T * CW * 4;               // partner's y of a chunk (double-buffered)
    // With G == 1 every lane needs all 16 B and C of a token, and with F32BC
    // they are wanted as fp32 anyway: they are converted once per chunk
    // (T x 32 floats) instead of per use.
    static constexpr int BCF = (!BCQ && (G == 1 || F32BC)) ? T * 2 * kNState * 4 : 0;
    static constexpr int WARP_BYTES = NS * STAGE + 2 * OWS + BCF;
    static constexpr int BAR_OFF = 2 * WARP_BYTES;
    static constexpr int SMEM = BAR_OFF + 2 * NS * 8 + 128;
    static constexpr uint32_t TX_BASE =
        (uint32_t)(((T + 3) * CW + T * CW) * ESZ + (BCQ ? T * 2 * kNState * 4 : 2 * T * kNState * ESZ));
    static constexpr uint32_t TX_Z = (uint32_t)(T * CW * ESZ);
    static_assert(T + 3 <= 256 && CW <= 256, "TMA box dimensions");
    static_assert(!BCQ || G == 1, "fp32 quads: one lane per channel");
};

// S consecutive B (or C) values of a token row, as fp32.
template <int S>
__device__ __forceinline__ void load_row(const __nv_bfloat16* p, float (&v)[S]) {
    static_assert(S % 2 == 0, "pairs");
    const uint32_t* w = reinterpret_cast<const uint32_t*>(p);
    uint32_t r[S / 2];
    if constexpr (S == 2) {
        r[0] = w[0];
    } else if constexpr (S == 4) {
        const uint2 t = *reinterpret_cast<const uint2*>(w);
        r[0] = t.x; r[1] = t.y;
    } else {
#pragma unroll
        for (int q = 0; q < S / 2; q += 4) {
            const uint4 t = *reinterpret_cast<const uint4*>(w + q);
            r[q] = t.x; r[q + 1] = t.y; r[q + 2] = t.z; r[q + 3] = t.w;
        }
    }
    // bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32
#pragma unroll
    for (int q = 0; q < S / 2; ++q) {
        v[2 * q] = __uint_as_float(r[q] << 16);
        v[2 * q + 1] = __uint_as_float(r[q] & 0xffff0000u);
    }
}
template <int S>
__device__ __forceinline__ void load_row(const float* p, float (&v)[S]) {
    load_states<S>(p, v);
}

template <int G, typename Tin, typename Tout, int DIR, bool LAYER, bool F32BC = false, bool BCQ = false>
struct FusedWarp {
    using Ge = FusedGeo<G, Tin, F32BC, BCQ>;
    static constexpr int T = Ge::T, NS = Ge::NS, S = Ge::S;

    // own channel (per-token work and output)
    int lane, d;
    bool dvalid;
    float w[4], cb, bias, Dd;
    float x0, x1, x2;  // conv window: steps s-3, s-2, s-1
    // scan: states [j*S, j*S+S) of the group's G channels
    int j;
    float A2[G][S];
    float h[G][S];

    __device__ __forceinline__ void setup(const KParams& p, int ct0, int lane_) {
        lane = lane_;
        d = ct0 + lane;
        dvalid = d < p.D;
        const int64_t rd = (int64_t)DIR * p.D + (dvalid ? d : 0);
#pragma unroll
        for (int k = 0; k < 4; ++k) w[k] = dvalid ? p.conv_w[rd * 4 + k] : 0.f;
        cb = (dvalid && p.conv_b) ? p.conv_b[rd] : 0.f;
        bias = dvalid ? p.dt_bias[rd] : 0.f;
        Dd = dvalid ? p.Dskip[rd] : 0.f;
        j = lane % G;
        const int gbase = ct0 + lane - j;  // first channel of the group
#pragma unroll
        for (int q = 0; q < G; ++q) {
            const int dq = gbase + q;
            const bool ok = dq < p.D;
            const int64_t rq = (int64_t)DIR * p.D + (ok ? dq : 0);
#pragma unroll
            for (int s = 0; s < S; ++s) {
                A2[q][s] = ok ? p.A[rq * kNState + j * S + s] * kLog2e : 0.f;
                h[q][s] = 0.f;
            }
        }
    }

    static __device__ __forceinline__ int row_of(int s) { return DIR == 0 ? s : T - 1 - s; }
    // x-tile row of step s (the forward tile starts 3 tokens early)
    static __device__ __forceinline__ int xrow_of(int s) { return DIR == 0 ? s + 3 : T - 1 - s; }

    // Load the conv window (steps -3..-1) of a chunk.
    __device__ __forceinline__ void window(const Tin* xt) {
        x0 = ldf(xt, xrow_of(-3) * Ge::CW + lane);
        x1 = ldf(xt, xrow_of(-2) * Ge::CW + lane);
        x2 = ldf(xt, xrow_of(-1) * Ge::CW + lane);
    }

    // Per-token work of the own channel at step s: step size, drive and
    // D*u (zero for an identity step).  Independent of the scan, so it is
    // computed one step ahead of the state updates that use it.
    struct Elem {
        float dl, du, Du;
    };
    __device__ __forceinline__ Elem element(int s, bool valid, const Tin* xt, const Tin* dtt) {
        const float x3 = ldf(xt, xrow_of(s) * Ge::CW + lane);
        float cv = fmaf(w[0], x0, cb);
        cv = fmaf(w[1], x1, cv);
        cv = fmaf(w[2], x2, cv);
        cv = fmaf(w[3], x3, cv);
        x0 = x1; x1 = x2; x2 = x3;
        const float u = silu(cv);
        const float dl = softplus(ldf(dtt, row_of(s) * Ge::CW + lane) + bias);
        Elem e;
        e.dl = valid ? dl : 0.f;
        e.du = valid ? dl * u : 0.f;
        e.Du = valid ? Dd * u : 0.f;
        return e;
    }

    // State updates of step s for the group's G channels (their step sizes
    // gathered from the group's lanes); returns sum_n C h of the own channel
    // (WITH_Y), before the D skip.
    // G == 1: the lane's own channel, all 16 states; B and C of the token
    // come as fp32 from the per-chunk buffer bcf ([T][B 16 | C 16]), or with
    // BCQ from the chunk's tile of fp32 quads ([T][8][B B C C]).
    template <bool WITH_Y>
    __device__ __forceinline__ float scan1(int s, const Elem& e, const float* bcf) {
        const float* rowp = bcf + row_of(s) * 2 * kNState;
        float bv[kNState], cvv[kNState];
        if constexpr (BCQ) {
#pragma unroll
            for (int q = 0; q < kNState / 2; ++q) {
                const float4 v = *reinterpret_cast<const float4*>(rowp + 4 * q);
                bv[2 * q] = v.x; bv[2 * q + 1] = v.y; cvv[2 * q] = v.z; cvv[2 * q + 1] = v.w;
            }
        } else {
            load_states<kNState>(rowp, bv);
            if constexpr (WITH_Y) load_states<kNState>(rowp + kNState, cvv);
        }
        const float2 dd = make_float2(e.dl, e.dl);
        const float2 uu = make_float2(e.du, e.du);
        float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int sp = 0; sp < kNState; sp += 2) {
            const float2 v = mul2(dd, make_float2(A2[0][sp], A2[0][sp + 1]));
            const float2 ea = make_float2(ex2_approx(v.x), ex2_approx(v.y));
            const float2 drive = mul2(uu, make_float2(bv[sp], bv[sp + 1]));
            const float2 hh = fma2(ea, make_float2(h[0][sp], h[0][sp + 1]), drive);
            h[0][sp] = hh.x;
            h[0][sp + 1] = hh.y;
            if constexpr (WITH_Y) acc2 = fma2(make_float2(cvv[sp], cvv[sp + 1]), hh, acc2);
        }
        return acc2.x + acc2.y;
    }

    template <bool WITH_Y>
    __device__ __forceinline__ float scan(int s, const Elem& e, const Tin* Bt, const Tin* Ct, const float* bcf) {
        const int row = row_of(s);
        float bv[S], cvv[S];
        if constexpr (F32BC) {
            load_states<S>(bcf + row * 2 * kNState + j * S, bv);
            if constexpr (WITH_Y) load_states<S>(bcf + row * 2 * kNState + kNState + j * S, cvv);
        } else {
            load_row<S>(Bt + row * kNState + j * S, bv);
            if constexpr (WITH_Y) load_row<S>(Ct + row * kNState + j * S, cvv);
        }
        float acc[G];
#pragma unroll
        for (int q = 0; q < G; ++q) {
            const float dq = __shfl_sync(0xffffffffu, e.dl, q, G);
            const float uq = __shfl_sync(0xffffffffu, e.du, q, G);
            const float2 dd = make_float2(dq, dq);
            const float2 uu = make_float2(uq, uq);
            // two accumulator pairs: half the dependent chain of the C.h sum
            float2 acc2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
            for (int sp = 0; sp < S; sp += 2) {
                const float2 v = mul2(dd, make_float2(A2[q][sp], A2[q][sp + 1]));
                const float2 ea = make_float2(ex2_approx(v.x), ex2_approx(v.y));
                const float2 drive = mul2(uu, make_float2(bv[sp], bv[sp + 1]));
                const float2 hh = fma2(ea, make_float2(h[q][sp], h[q][sp + 1]), drive);
                h[q][sp] = hh.x;
                h[q][sp + 1] = hh.y;
                if constexpr (WITH_Y) acc2[(sp >> 1) & 1] = fma2(make_float2(cvv[sp], cvv[sp + 1]), hh, acc2[(sp >> 1) & 1]);
            }
            acc[q] = (acc2[0].x + acc2[1].x) + (acc2[0].y + acc2[1].y);
        }
        if constexpr (WITH_Y)
            return group_transpose_reduce<G, 1>(acc, j);
        else
            return 0.f;
    }
};

// B and C rows of a chunk (T x 16 each, token order) -> fp32 [T][B 16 | C 16],
// one warp; lane l handles state l % 16 of B (l < 16) or C (l >= 16).
template <int T, typename Tin>
__device__ __forceinline__ void fused_convert_bc(const Tin* Bt, const Tin* Ct, float* bcf, int lane, bool with_c) {
    const int n = lane & (kNState - 1);
    const bool isc = lane >= kNState;
    if (isc && !with_c) return;
    const Tin* src = isc ? Ct : Bt;
#pragma unroll 4
    for (int r = 0; r < T; ++r) bcf[r * 2 * kNState + lane] = ldf(src, r * kNState + n);
}

template <int G, typename Tin, bool F32BC = false, bool BCQ = false>
__device__ __forceinline__ void fused_issue(const FusedMaps& maps, unsigned char* wbase, uint64_t* full, int r,
                                            int i, int k, bool gated, int ct0, int b, int starve) {
    using Ge = FusedGeo<G, Tin, F32BC, BCQ>;
    if (starve) return;
    const int st = i % Ge::NS;
    unsigned char* sb = wbase + st * Ge::STAGE;
    uint64_t* bar = full + st;
    mbar_arrive_expect_tx(bar, Ge::TX_BASE + (gated ? Ge::TX_Z : 0u));
    const int row0 = k * Ge::T;
    tma_load_3d(sb, &maps.x, bar, ct0, r == 0 ? row0 - 3 : row0, b);
    tma_load_3d(sb + Ge::XB, &maps.dt[r], bar, ct0, row0, b);
    if (gated) tma_load_3d(sb + Ge::XB + Ge::DTB, &maps.z, bar, ct0, row0, b);
    tma_load_3d(sb + Ge::XB + 2 * Ge::DTB, &maps.B[r], bar, 0, row0, b);
    if constexpr (!BCQ) tma_load_3d(sb + Ge::XB + 2 * Ge::DTB + Ge::BB, &maps.C[r], bar, 0, row0, b);
}

// CARRY: start from p.carry_in, report p.carry_out and p.delta_sum (each where non-null).
template <int G, typename Tin, typename Tout, int DIR, bool CARRY, bool F32BC, int UNR = 4, bool BCQ = false>
__device__ __forceinline__ void fused_layer_direction(const FusedMaps& maps, const KParams& p, unsigned char* base,
                                                      int lane) {
    using Ge = FusedGeo<G, Tin, F32BC, BCQ>;
    constexpr int T = Ge::T, NS = Ge::NS, S = Ge::S;
    using Wp = FusedWarp<G, Tin, Tout, DIR, true, F32BC, BCQ>;
    unsigned char* wbase = base + DIR * Ge::WARP_BYTES;
    float* ows = reinterpret_cast<float*>(wbase + NS * Ge::STAGE);
    float* bcf = reinterpret_cast<float*>(wbase + NS * Ge::STAGE + 2 * Ge::OWS);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + Ge::BAR_OFF) + DIR * NS;
    const int b = blockIdx.y;
    const int ct0 = blockIdx.x * Ge::CW;
    const int64_t L = p.L;
    const int D = p.D;
    const int nc = (int)((L + T - 1) / T);
    const int hF = nc / 2;
    const int meet = DIR == 0 ? hF : nc - hF;
    const float scale = p.dir_scale[DIR];
    // cp.async of the partner's fp32 y of chunk ii (T rows x 32 channels,
    // 16-byte pieces; D % 4 == 0 on this path) into buffer ii & 1
    auto fetch_partner = [&](int ii) {
        const int kk = DIR == 0 ? ii : nc - 1 - ii;
        const int64_t row = (int64_t)b * L + (int64_t)kk * T;
        float* dst = ows + (ii & 1) * (T * Ge::CW);
        for (int e = lane; e < T * 8; e += 32) {
            const int r = e >> 3, q = e & 7;
            const bool ok = (int64_t)kk * T + r < L && ct0 + 4 * q < D;
            const float* src = p.ws + (row + (ok ? r : 0)) * D + (ok ? ct0 + 4 * q : 0);
            cp_async<16>(dst + r * Ge::CW + 4 * q, src, ok);
        }
        cp_async_commit();
    };

    Wp wp;
    wp.setup(p, ct0, lane);
    const int gbase = ct0 + lane - wp.j;  // first channel of this lane's group
    if (CARRY && p.carry_in[DIR]) {
#pragma unroll
        for (int q = 0; q < G; ++q) {
            if (gbase + q < D) {
                const float* ci = p.carry_in[DIR] + ((int64_t)b * D + gbase + q) * kNState + wp.j * S;
#pragma unroll
                for (int s = 0; s < S; ++s) wp.h[q][s] = ci[s];
            }
        }
    }
    float dsum = 0.f;  // step sizes of the own channel so far
    if (lane == 0)
        for (int i = 0; i < NS && i < nc; ++i)
            fused_issue<G, Tin, F32BC, BCQ>(maps, wbase, full, DIR, i, DIR == 0 ? i : nc - 1 - i, i >= meet, ct0, b,
                                       p.starve);

#pragma unroll 1
    for (int i = 0; i < nc; ++i) {
        const int k = DIR == 0 ? i : nc - 1 - i;
        const bool gated = i >= meet;
        if (i == meet) {
            __threadfence_block();
            named_bar_sync(1, 64);
        }
        // the previous chunk's stage is free (this warp is past it): refill it
        if (lane == 0 && i >= 1 && i - 1 + NS < nc) {
            const int i2 = i - 1 + NS;
            fused_issue<G, Tin, F32BC, BCQ>(maps, wbase, full, DIR, i2, DIR == 0 ? i2 : nc - 1 - i2, i2 >= meet, ct0, b,
                                       p.starve);
        }
        const int nvalid = (int)((L - (int64_t)k * T < T) ? (L - (int64_t)k * T) : T);
        const int s_lo = DIR == 0 ? 0 : T - nvalid;
        const int s_hi = DIR == 0 ? nvalid : T;
        const int64_t chunk_row = (int64_t)b * L + (int64_t)k * T;
        // The partner's y of the gated chunks, one chunk ahead (buffer i & 1):
        // the copy of chunk i+1 runs under the scan of chunk i.  All of it was
        // stored before the meeting barrier.
        if (i == meet) fetch_partner(i);
        if (gated && i + 1 < nc) fetch_partner(i + 1);
        const int st = i % NS;
        mbar_wait_bounded(full + st, (uint32_t)((i / NS) & 1), p.wait_limit);
        const unsigned char* sb = wbase + st * Ge::STAGE;
        const Tin* xt = reinterpret_cast<const Tin*>(sb);
        const Tin* dtt = reinterpret_cast<const Tin*>(sb + Ge::XB);
        const Tin* zt = reinterpret_cast<const Tin*>(sb + Ge::XB + Ge::DTB);
        const Tin* Bt = reinterpret_cast<const Tin*>(sb + Ge::XB + 2 * Ge::DTB);
        const Tin* Ct = reinterpret_cast<const Tin*>(sb + Ge::XB + 2 * Ge::DTB + Ge::BB);
        if (CARRY && i == 0 && p.conv_halo[DIR])  // forward: tile rows 0..2 = tokens -3..-1; reverse: rows of L..L+2
            put_conv_halo(reinterpret_cast<Tin*>(wbase + st * Ge::STAGE), Ge::CW,
                          DIR == 0 ? 0 : (int)(L - (int64_t)k * T), 0, ct0, Ge::CW,
                          static_cast<const Tin*>(p.conv_halo[DIR]) + (int64_t)b * 3 * D, D, lane);
        if (gated) {
            if (i + 1 < nc)
                cp_async_wait_pending<1>();  // chunk i's copies; i+1's may still run
            else
                cp_async_wait_all();
            __syncwarp();
        }
        const float* owc = ows + (i & 1) * (T * Ge::CW);
        if constexpr (!BCQ && (G == 1 || F32BC)) {
            __syncwarp();
            fused_convert_bc<T, Tin>(Bt, Ct, bcf, lane, true);
            __syncwarp();
        }
        wp.window(xt);
        float* wsw = p.ws + chunk_row * D + wp.d;
        Tout* outw = static_cast<Tout*>(p.out) + chunk_row * D + wp.d;
        typename Wp::Elem nxt = wp.element(0, 0 >= s_lo && 0 < s_hi, xt, dtt);
#pragma unroll (UNR)
        for (int s = 0; s < T; ++s) {
            const bool valid = s >= s_lo && s < s_hi;
            const typename Wp::Elem cur = nxt;
            if constexpr (CARRY) dsum += cur.dl;  // 0 past the end
            if (s + 1 < T) nxt = wp.element(s + 1, s + 1 >= s_lo && s + 1 < s_hi, xt, dtt);
            float yr;
            if constexpr (G == 1)
                yr = wp.template scan1<true>(s, cur, BCQ ? reinterpret_cast<const float*>(Bt) : bcf);
            else
                yr = wp.template scan<true>(s, cur, Bt, Ct, bcf);
            const float y = (yr + cur.Du) * scale;
            if (valid && wp.dvalid) {
                const int tr = Wp::row_of(s);
                if (!gated) {
                    wsw[(int64_t)tr * D] = y;
                } else {
                    const float zv = ldf(zt, tr * Ge::CW + lane);
                    stf(outw, (int64_t)tr * D, (y + owc[tr * Ge::CW + lane]) * silu(zv));
                }
            }
        }
        __syncwarp();
    }
    if (meet >= nc) {  // single chunk: the reverse warp meets after it
        __threadfence_block();
        named_bar_sync(1, 64);
    }
    if (CARRY && p.carry_out[DIR]) {
#pragma unroll
        for (int q = 0; q < G; ++q) {
            if (gbase + q < D) {
                float* co = p.carry_out[DIR] + ((int64_t)b * D + gbase + q) * kNState + wp.j * S;
#pragma unroll
                for (int s = 0; s < S; ++s) co[s] = wp.h[q][s];
            }
        }
    }
    if (CARRY && p.delta_sum[DIR] && wp.dvalid) p.delta_sum[DIR][(int64_t)b * D + wp.d] = dsum;
}

// The token loop unrolled by 4 (with 2-lane groups: 1.116 against 1.154 ms
// for 2, 1.25 for 8 and 1.41 for all 16 at batch 8, L 2048, d_inner 4096;
// with one lane per channel 1.096 against 1.137 for 2 and 1.20 for 8).
template <int G, typename Tin, typename Tout, bool CARRY = false, bool F32BC = false, int UNR = 4, bool BCQ = false>
__global__ void __launch_bounds__(64, 8) fused_layer_kernel(const __grid_constant__ FusedMaps maps, const KParams p) {
    using Ge = FusedGeo<G, Tin, F32BC, BCQ>;
    extern __shared__ __align__(128) unsigned char smem_dyn[];
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 127) & ~static_cast<uintptr_t>(127));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        uint64_t* bars = reinterpret_cast<uint64_t*>(base + Ge::BAR_OFF);
        for (int i = 0; i < 2 * Ge::NS; ++i) mbar_init(bars + i, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (warp == 0)
        fused_layer_direction<G, Tin, Tout, 0, CARRY, F32BC, UNR, BCQ>(maps, p, base, lane);
    else
        fused_layer_direction<G, Tin, Tout, 1, CARRY, F32BC, UNR, BCQ>(maps, p, base, lane);
}

// Forward scan over P = p.L tokens from zero: final state and conv tail.
// One warp per CTA (32 channels); z, C and the reverse inputs are not read.
template <int G, typename Tin>
__global__ void __launch_bounds__(32, 16) fused_prefix_kernel(const __grid_constant__ FusedMaps maps, const KParams p) {
    using Ge = FusedGeo<G, Tin>;
    constexpr int T = Ge::T, NS = Ge::NS, S = Ge::S;
    extern __shared__ __align__(128) unsigned char smem_dyn[];
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 127) & ~static_cast<uintptr_t>(127));
    const int lane = threadIdx.x;
    uint64_t* full = reinterpret_cast<uint64_t*>(base + Ge::BAR_OFF);
    if (lane == 0) {
        for (int i = 0; i < NS; ++i) mbar_init(full + i, 1);
        fence_barrier_init();
    }
    __syncwarp();
    const int b = blockIdx.y;
    const int ct0 = blockIdx.x * Ge::CW;
    const int64_t P = p.L;
    const int nc = (int)((P + T - 1) / T);
    constexpr uint32_t TX = (uint32_t)(((T + 3) * Ge::CW + T * Ge::CW + T * kNState) * Ge::ESZ);
    auto issue = [&](int i) {
        if (p.starve) return;
        const int st = i % NS;
        unsigned char* sb = base + st * Ge::STAGE;
        uint64_t* bar = full + st;
        mbar_arrive_expect_tx(bar, TX);
        tma_load_3d(sb, &maps.x, bar, ct0, i * T - 3, b);
        tma_load_3d(sb + Ge::XB, &maps.dt[0], bar, ct0, i * T, b);
        tma_load_3d(sb + Ge::XB + 2 * Ge::DTB, &maps.B[0], bar, 0, i * T, b);
    };
    FusedWarp<G, Tin, float, 0, false> wp;
    wp.setup(p, ct0, lane);
    if (lane == 0)
        for (int i = 0; i < NS && i < nc; ++i) issue(i);
#pragma unroll 1
    for (int i = 0; i < nc; ++i) {
        if (lane == 0 && i >= 1 && i - 1 + NS < nc) issue(i - 1 + NS);
        const int nvalid = (int)((P - (int64_t)i * T < T) ? (P - (int64_t)i * T) : T);
        const int st = i % NS;
        mbar_wait_bounded(full + st, (uint32_t)((i / NS) & 1), p.wait_limit);
        const unsigned char* sb = base + st * Ge::STAGE;
        const Tin* xt = reinterpret_cast<const Tin*>(sb);
        const Tin* dtt = reinterpret_cast<const Tin*>(sb + Ge::XB);
        const Tin* Bt = reinterpret_cast<const Tin*>(sb + Ge::XB + 2 * Ge::DTB);
        wp.window(xt);
        auto nxt = wp.element(0, 0 < nvalid, xt, dtt);
#pragma unroll 4
        for (int s = 0; s < T; ++s) {
            const auto cur = nxt;
            if (s + 1 < T) nxt = wp.element(s + 1, s + 1 < nvalid, xt, dtt);
            wp.template scan<false>(s, cur, Bt, Bt, nullptr);
        }
        __syncwarp();
    }
    // the group's G channels x my S states
    const int gbase = ct0 + lane - wp.j;
#pragma unroll
    for (int q = 0; q < G; ++q) {
        const int dq = gbase + q;
        if (dq < p.D) {
#pragma unroll
            for (int s = 0; s < S; ++s) p.h_out[((int64_t)b * p.D + dq) * kNState + wp.j * S + s] = wp.h[q][s];
        }
    }
    if (wp.dvalid) {
        const Tin* X = static_cast<const Tin*>(p.x);
        Tin* tail = static_cast<Tin*>(p.tail_out);
        for (int q = 0; q < 3; ++q) {
            const int64_t t = P - 3 + q;
            tail[((int64_t)b * 3 + q) * p.D + wp.d] = t >= 0 ? X[((int64_t)b * P + t) * p.D + wp.d] : cvt_from<Tin>(0.f);
        }
    }
}

}  // namespace bimamba

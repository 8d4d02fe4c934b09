// scan_kernels.cuh -- sm_100a kernels of the bidirectional Mamba mixer layer.
//
// The layer ("DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone",
// §3.2 Eq. (4)-(6), App. A.1 Eq. (7)-(9)) runs, per channel, a width-4
// conv + SiLU, a softplus step size and a 16-state diagonal selective scan
// once left to right and once right to left, adds the two outputs and gates
// them with SiLU(z).  The block step (§4.3 block-cached decoding) keeps the
// reverse scan inside the active block and carries the forward state.
//
// Execution model (one CTA = one batch row x a tile of channels):
//  * Warps come in forward/reverse pairs over the same channels.  Both walk
//    the sequence in "step space": step s of direction r is token
//    t0 + s (forward) or t0 - s (reverse), so the reverse conv is the causal
//    conv applied to tokens read backwards -- no flipped copy exists.
//  * A channel's 16 states are split over G lanes (S = 16/G states each).
//    The per-token work (conv, SiLU, softplus) of a G-token group is spread
//    round-robin over those lanes and handed over through shared memory; the
//    C.h partial sums are combined by a shuffle transpose-reduce that leaves
//    lane j of the group holding token j's sum.
//  * Full layer: the forward warp covers [0, M) while its partner covers
//    [M, L) backwards; each stores its fp32 y to the workspace, the pair meets
//    at a named barrier, then each finishes the other half, reading the
//    partner's y, applying the gate and storing the output.  Every input is
//    read by each direction once; no CTA waits on another CTA.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace bimamba {

constexpr int kNState = 16;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------- math

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// silu(v) = v / (1 + e^{-v}); for v -> -inf the reciprocal of +inf is 0.
__device__ __forceinline__ float silu(float v) {
    return v * rcp_approx(1.f + ex2_approx(-v * kLog2e));
}

// softplus(v) = log(1 + e^v), with e = e^v from one MUFU exp2, in three
// ranges so that the step size keeps its relative accuracy however small:
//  * e <= 1/16: log1p(e) by its alternating Taylor series
//      e - e^2/2 + e^3/3 - e^4/4 + e^5/5 - e^6/6
//    (Horner, FP32 pipe).  The first omitted term bounds the truncation by
//    e^6/7 <= 8.5e-9 relative.  Forming 1 + e in fp32 would instead round
//    away everything below 2^-24, which is all of e once v < -17.
//  * 1/16 < e, v <= 20: log2(1 + e) * ln 2 (MUFU lg2).  The result is at
//    least log(17/16) = 0.061 here, so the absolute error of the approximate
//    log2 and the rounding of 1 + e stay a few 1e-6 of it.
//  * v > 20: v (the remainder log1p(e^-v) < 2.1e-9 is below v's half ulp).
// e^-inf = 0 makes softplus(-inf) exactly 0.
__device__ __forceinline__ float softplus(float v) {
    const float e = ex2_approx(v * kLog2e);
    float t = fmaf(e, -1.f / 6.f, 1.f / 5.f);
    t = fmaf(e, t, -0.25f);
    t = fmaf(e, t, 1.f / 3.f);
    t = fmaf(e, t, -0.5f);
    t = fmaf(e, t, 1.f);
    const float series = e * t;
    const float via_log = lg2_approx(1.f + e) * kLn2;
    return (v > 20.f) ? v : (e <= 0.0625f ? series : via_log);
}

// Packed two-lane fp32 arithmetic (sm_100a f32x2 instructions, round to
// nearest like their scalar forms): one issue slot for two multiplies or
// fused multiply-adds.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// ---------------------------------------------------------------- element I/O

__device__ __forceinline__ float ldf(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p, int64_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void stf(float* p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void stf(__nv_bfloat16* p, int64_t i, float v) { p[i] = __float2bfloat16_rn(v); }
template <typename T> __device__ __forceinline__ T cvt_from(float v);
template <> __device__ __forceinline__ float cvt_from<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 cvt_from<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// ---------------------------------------------------------------- parameters

struct KParams {
    const void* x;
    const void* z;
    const void* dt[2];
    const void* B[2];
    const void* C[2];
    const float* A;        // [2][D][16]
    const float* Dskip;    // [2][D]
    const float* dt_bias;  // [2][D]
    const float* conv_w;   // [2][D][4]
    const float* conv_b;   // [2][D] or nullptr
    void* out;             // [batch][L][D]
    float* ws;             // [batch][L][D] fp32 (layer only)
    float* bcq;            // [2][batch][L][8][4] fp32: B/C quads (chunked layer at 8 lanes)
    const float* h_in;     // [batch][D][16]   (block step)
    const void* tail_in;   // [batch][3][D]    (block step)
    float* h_out;          // [batch][D][16]   (prefix, block commit) or nullptr
    void* tail_out;        // [batch][3][D]    (prefix, block commit) or nullptr
    // layer with carries (TMA kernel families), each [2] = per direction, nullptr = unused:
    const float* carry_in[2];  // [batch][D][16]: state entering the direction's first step (else 0)
    float* carry_out[2];       // [batch][D][16]: state after the direction's last step
    float* delta_sum[2];       // [batch][D]: sum of the step sizes over the sequence
    // [batch][3][D] of the input type, rows in token order: the x the conv reads
    // outside [0, L) (forward: tokens -3..-1; reverse: tokens L..L+2), else zeros
    const void* conv_halo[2];
    int64_t L;             // sequence (or block) length
    int64_t M;             // meeting point of the two directions (layer)
    int D;
    int batch;
    float dir_scale[2];    // 1, or 0 for a disabled direction (test flags)
    long long wait_limit;  // SM clocks a wait for a tile may take before it gives up
    int starve;            // test aid: issue no tile loads, so every such wait gives up
};

// ---------------------------------------------------------------- geometry

template <int G, int T>
struct Geo {
    static_assert(G == 1 || G == 2 || G == 4 || G == 8 || G == 16, "G");
    static_assert(T % G == 0, "T must be a multiple of G");
    static constexpr int CPW = 32 / G;                 // channels per warp
    static constexpr int S = kNState / G;              // states per lane
    static constexpr int EPL = T / G;                  // elements per lane per chunk
    static constexpr int XS = ((T + 3) * CPW + 3) & ~3;  // x rows, 3 halo rows first (16-B padded)
    static constexpr int BCS = T * 2 * kNState;        // B row then C row per step
    static constexpr int DDS = T * CPW * 2;            // (delta, delta*u) per element
    static constexpr int YS = T * CPW;                 // staged forward y (block step)
    static constexpr int HN = (3 * CPW + 31) / 32;     // halo values per lane
};

template <int S>
__device__ __forceinline__ void load_states(const float* p, float (&v)[S]) {
    if constexpr (S % 4 == 0) {
#pragma unroll
        for (int q = 0; q < S; q += 4) {
            const float4 f = *reinterpret_cast<const float4*>(p + q);
            v[q] = f.x; v[q + 1] = f.y; v[q + 2] = f.z; v[q + 3] = f.w;
        }
    } else if constexpr (S == 2) {
        const float2 f = *reinterpret_cast<const float2*>(p);
        v[0] = f.x; v[1] = f.y;
    } else {
#pragma unroll
        for (int q = 0; q < S; ++q) v[q] = p[q];
    }
}

// After the call, lane j of a G-lane group (lanes j*CPW + c) holds the sum
// over the group of p[j].  Each round halves the array: a lane keeps the
// half of the tokens its sub-index bit selects and receives the partner's
// partial sums for that half.
template <int G, int CPW>
__device__ __forceinline__ float group_transpose_reduce(float (&p)[G], int j) {
#pragma unroll
    for (int half = G / 2; half >= 1; half >>= 1) {
        const bool upper = (j & half) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? p[i] : p[i + half];
            const float keep = upper ? p[i + half] : p[i];
            p[i] = keep + __shfl_xor_sync(0xffffffffu, send, half * CPW);
        }
    }
    return p[0];
}

// One warp's scan of one direction over CPW channels.
template <int G, int T, typename Tin>
struct DirScan {
    using Ge = Geo<G, T>;
    int lane, c, j, d, c0, D;
    bool dvalid;
    int64_t rowbase;  // batch row * sequence length
    float A2[Ge::S];  // A * log2(e) of this lane's states
    float w[4], cb, bias, Dd;
    float h[Ge::S];
    float* xs;
    float* bc;
    float2* dd;
    const Tin* X;
    const Tin* DT;
    const Tin* Bp;
    const Tin* Cp;

    __device__ __forceinline__ void setup(const KParams& p, int b, int c0_, int lane_, float* smem_warp) {
        lane = lane_;
        c = lane % Ge::CPW;
        j = lane / Ge::CPW;
        c0 = c0_;
        D = p.D;
        d = c0 + c;
        dvalid = d < D;
        rowbase = (int64_t)b * p.L;
        xs = smem_warp;
        bc = smem_warp + Ge::XS;
        dd = reinterpret_cast<float2*>(smem_warp + Ge::XS + Ge::BCS);
        X = static_cast<const Tin*>(p.x);
    }

    // Load direction r's parameters and inputs; zero the state and the halo.
    __device__ __forceinline__ void set_direction(const KParams& p, int r) {
        DT = static_cast<const Tin*>(p.dt[r]);
        Bp = static_cast<const Tin*>(p.B[r]);
        Cp = static_cast<const Tin*>(p.C[r]);
        const int64_t rd = (int64_t)r * D + (dvalid ? d : 0);
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
        __syncwarp();
        for (int e = lane; e < 3 * Ge::CPW; e += 32) xs[e] = 0.f;
        __syncwarp();
    }

    // Stage x and B (and, with LOAD_C, C) rows of steps [0, n) (token
    // tc + dir * s).  Without LOAD_C the C pointer is never dereferenced.
    template <bool LOAD_C>
    __device__ __forceinline__ void stage(int64_t tc, int dir, int n) {
        for (int e = lane; e < n * Ge::CPW; e += 32) {
            const int s = e / Ge::CPW, cc = e % Ge::CPW;
            const int64_t t = tc + (int64_t)dir * s;
            xs[(3 + s) * Ge::CPW + cc] = (c0 + cc < D) ? ldf(X, (rowbase + t) * D + c0 + cc) : 0.f;
        }
        if (LOAD_C || lane < kNState) {
            const Tin* src = (lane < kNState) ? Bp : Cp;
            const int col = lane & (kNState - 1);
            for (int s = 0; s < n; ++s) {
                const int64_t t = tc + (int64_t)dir * s;
                bc[s * 2 * kNState + lane] = ldf(src, (rowbase + t) * kNState + col);
            }
        }
        __syncwarp();
    }

    // conv + SiLU, softplus: (delta, delta*u) to shared memory, D*u to du.
    __device__ __forceinline__ void elements(int64_t tc, int dir, int n, float (&du)[Ge::EPL]) {
#pragma unroll
        for (int k = 0; k < Ge::EPL; ++k) {
            const int s = j + G * k;
            du[k] = 0.f;
            if (s < n) {
                const int64_t t = tc + (int64_t)dir * s;
                const float* xc = xs + s * Ge::CPW + c;  // rows s..s+3 hold steps s-3..s
                float cv = cb;
                cv = fmaf(w[0], xc[0], cv);
                cv = fmaf(w[1], xc[Ge::CPW], cv);
                cv = fmaf(w[2], xc[2 * Ge::CPW], cv);
                cv = fmaf(w[3], xc[3 * Ge::CPW], cv);
                const float u = silu(cv);
                const float dtv = dvalid ? ldf(DT, (rowbase + t) * D + d) : 0.f;
                const float dl = softplus(dtv + bias);
                dd[s * Ge::CPW + c] = make_float2(dl, dl * u);
                du[k] = Dd * u;
            }
        }
        __syncwarp();
    }

    // Advance the state over steps [0, n).  With WITH_Y, yv[k] receives
    // sum_n C h for this lane's own step j + G*k.
    template <bool WITH_Y>
    __device__ __forceinline__ void scan(int n, float (&yv)[Ge::EPL]) {
#pragma unroll
        for (int k = 0; k < Ge::EPL; ++k) {
            float pp[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const int s = G * k + g;
                float acc = 0.f;
                if (s < n) {  // warp-uniform
                    const float2 q2 = dd[s * Ge::CPW + c];
                    float Bv[Ge::S], Cv[Ge::S];
                    load_states<Ge::S>(bc + s * 2 * kNState + j * Ge::S, Bv);
                    if constexpr (WITH_Y) load_states<Ge::S>(bc + s * 2 * kNState + kNState + j * Ge::S, Cv);
#pragma unroll
                    for (int q = 0; q < Ge::S; ++q) {
                        const float e = ex2_approx(q2.x * A2[q]);
                        h[q] = fmaf(e, h[q], q2.y * Bv[q]);
                        if constexpr (WITH_Y) acc = fmaf(Cv[q], h[q], acc);
                    }
                }
                pp[g] = acc;
            }
            if constexpr (WITH_Y) yv[k] = group_transpose_reduce<G, Ge::CPW>(pp, j);
        }
    }

    // Keep the last three staged x rows (steps n-3..n-1) as the next halo.
    __device__ __forceinline__ void carry_halo(int n) {
        float tmp[Ge::HN];
#pragma unroll
        for (int i = 0; i < Ge::HN; ++i) {
            const int e = lane + 32 * i;
            tmp[i] = (e < 3 * Ge::CPW) ? xs[n * Ge::CPW + e] : 0.f;
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < Ge::HN; ++i) {
            const int e = lane + 32 * i;
            if (e < 3 * Ge::CPW) xs[e] = tmp[i];
        }
        __syncwarp();
    }
};

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------- full layer

template <int G, int T, int WPD>
constexpr int layer_smem_floats() {
    return 2 * WPD * (Geo<G, T>::XS + Geo<G, T>::BCS + Geo<G, T>::DDS);
}

// grid (ceil(D / (WPD*CPW)), batch); block 2*WPD warps: warps [0, WPD)
// forward, [WPD, 2*WPD) reverse, warp w and w+WPD on the same channels.
template <int G, int T, int WPD, typename Tin, typename Tout>
__global__ void __launch_bounds__(2 * WPD * 32) layer_kernel(const KParams p) {
    using Ge = Geo<G, T>;
    extern __shared__ __align__(16) float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = warp / WPD, wg = warp - r * WPD;
    const int b = blockIdx.y;
    const int c0 = (blockIdx.x * WPD + wg) * Ge::CPW;
    DirScan<G, T, Tin> sc;
    sc.setup(p, b, c0, lane, smem + warp * (Ge::XS + Ge::BCS + Ge::DDS));
    sc.set_direction(p, r);
    const bool active = c0 < p.D;
    const int64_t L = p.L, M = p.M;
    const int dir = (r == 0) ? 1 : -1;
    const float scale = p.dir_scale[r];
    const Tin* Z = static_cast<const Tin*>(p.z);
    Tout* OUT = static_cast<Tout*>(p.out);
    float* WS = p.ws;

#pragma unroll 1
    for (int phase = 0; phase < 2; ++phase) {
        int64_t tstart, count;
        if (r == 0) { tstart = phase ? M : 0;         count = phase ? L - M : M; }
        else        { tstart = phase ? M - 1 : L - 1; count = phase ? M : L - M; }
        if (!active) count = 0;
#pragma unroll 1
        for (int64_t done = 0; done < count; done += T) {
            const int n = (int)((count - done < T) ? (count - done) : T);
            const int64_t tc = tstart + dir * done;
            sc.template stage<true>(tc, dir, n);
            float du[Ge::EPL], yv[Ge::EPL];
            sc.elements(tc, dir, n, du);
            sc.template scan<true>(n, yv);
#pragma unroll
            for (int k = 0; k < Ge::EPL; ++k) {
                const int s = sc.j + G * k;
                if (s < n && sc.dvalid) {
                    const int64_t t = tc + (int64_t)dir * s;
                    const int64_t idx = (sc.rowbase + t) * p.D + sc.d;
                    const float y = (yv[k] + du[k]) * scale;
                    if (phase == 0) {
                        WS[idx] = y;
                    } else {
                        const float v = (y + WS[idx]) * silu(ldf(Z, idx));
                        stf(OUT, idx, v);
                    }
                }
            }
            sc.carry_halo(n);
        }
        if (phase == 0) {
            __threadfence_block();
            named_barrier(1 + wg, 64);
        }
    }
}

// ---------------------------------------------------------------- prefix state

template <int G, int T, int WPB>
constexpr int prefix_smem_floats() {
    return WPB * (Geo<G, T>::XS + Geo<G, T>::BCS + Geo<G, T>::DDS);
}

// Forward-only scan over P = p.L tokens from zero; writes h_out and the tail.
// grid (ceil(D / (WPB*CPW)), batch); block WPB warps.
template <int G, int T, int WPB, typename Tin>
__global__ void __launch_bounds__(WPB * 32) prefix_kernel(const KParams p) {
    using Ge = Geo<G, T>;
    extern __shared__ __align__(16) float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y;
    const int c0 = (blockIdx.x * WPB + warp) * Ge::CPW;
    if (c0 >= p.D) return;  // whole warp idle; no barrier follows
    DirScan<G, T, Tin> sc;
    sc.setup(p, b, c0, lane, smem + warp * (Ge::XS + Ge::BCS + Ge::DDS));
    sc.set_direction(p, 0);
    const int64_t P = p.L;
#pragma unroll 1
    for (int64_t done = 0; done < P; done += T) {
        const int n = (int)((P - done < T) ? (P - done) : T);
        sc.template stage<false>(done, 1, n);
        float du[Ge::EPL], yv[Ge::EPL];
        sc.elements(done, 1, n, du);
        sc.template scan<false>(n, yv);
        sc.carry_halo(n);
    }
    if (sc.dvalid) {
#pragma unroll
        for (int q = 0; q < Ge::S; ++q)
            p.h_out[((int64_t)b * p.D + sc.d) * kNState + sc.j * Ge::S + q] = sc.h[q];
    }
    Tin* tail = static_cast<Tin*>(p.tail_out);
    for (int e = lane; e < 3 * Ge::CPW; e += 32) {
        const int k = e / Ge::CPW, cc = e % Ge::CPW;
        if (c0 + cc < p.D) tail[((int64_t)b * 3 + k) * p.D + c0 + cc] = cvt_from<Tin>(sc.xs[e]);
    }
}

// ---------------------------------------------------------------- block step

template <int G, int T, int WPB>
constexpr int block_smem_floats() {
    return WPB * (Geo<G, T>::XS + Geo<G, T>::BCS + Geo<G, T>::DDS + Geo<G, T>::YS);
}

// One block of n = p.L <= T tokens.  Each warp runs the forward direction from
// the cached state (and commits it if asked), then the reverse direction over
// the block alone, and combines.  grid (ceil(D / (WPB*CPW)), batch).
template <int G, int T, int WPB, typename Tin, typename Tout>
__global__ void __launch_bounds__(WPB * 32) block_kernel(const KParams p) {
    using Ge = Geo<G, T>;
    extern __shared__ __align__(16) float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y;
    const int c0 = (blockIdx.x * WPB + warp) * Ge::CPW;
    if (c0 >= p.D) return;
    float* wsm = smem + warp * (Ge::XS + Ge::BCS + Ge::DDS + Ge::YS);
    float* ys = wsm + Ge::XS + Ge::BCS + Ge::DDS;
    DirScan<G, T, Tin> sc;
    sc.setup(p, b, c0, lane, wsm);
    const int n = (int)p.L;
    const int D = p.D;

    // forward, from the cached state and conv tail
    sc.set_direction(p, 0);
    if (sc.dvalid) {
#pragma unroll
        for (int q = 0; q < Ge::S; ++q)
            sc.h[q] = p.h_in[((int64_t)b * D + sc.d) * kNState + sc.j * Ge::S + q];
    }
    const Tin* tail_in = static_cast<const Tin*>(p.tail_in);
    for (int e = lane; e < 3 * Ge::CPW; e += 32) {
        const int k = e / Ge::CPW, cc = e % Ge::CPW;
        sc.xs[e] = (c0 + cc < D) ? ldf(tail_in, ((int64_t)b * 3 + k) * D + c0 + cc) : 0.f;
    }
    __syncwarp();
    {
        sc.template stage<true>(0, 1, n);
        float du[Ge::EPL], yv[Ge::EPL];
        sc.elements(0, 1, n, du);
        sc.template scan<true>(n, yv);
#pragma unroll
        for (int k = 0; k < Ge::EPL; ++k) {
            const int s = sc.j + G * k;
            if (s < n) ys[s * Ge::CPW + sc.c] = (yv[k] + du[k]) * p.dir_scale[0];
        }
        sc.carry_halo(n);
    }
    if (p.h_out) {
        if (sc.dvalid) {
#pragma unroll
            for (int q = 0; q < Ge::S; ++q)
                p.h_out[((int64_t)b * D + sc.d) * kNState + sc.j * Ge::S + q] = sc.h[q];
        }
        Tin* tail_out = static_cast<Tin*>(p.tail_out);
        for (int e = lane; e < 3 * Ge::CPW; e += 32) {
            const int k = e / Ge::CPW, cc = e % Ge::CPW;
            if (c0 + cc < D) tail_out[((int64_t)b * 3 + k) * D + c0 + cc] = cvt_from<Tin>(sc.xs[e]);
        }
    }

    // reverse, over the block alone (zero state and zero conv padding past its end)
    sc.set_direction(p, 1);
    {
        const int64_t tc = n - 1;
        sc.template stage<true>(tc, -1, n);
        float du[Ge::EPL], yv[Ge::EPL];
        sc.elements(tc, -1, n, du);
        sc.template scan<true>(n, yv);
        const Tin* Z = static_cast<const Tin*>(p.z);
        Tout* OUT = static_cast<Tout*>(p.out);
#pragma unroll
        for (int k = 0; k < Ge::EPL; ++k) {
            const int s = sc.j + G * k;
            if (s < n && sc.dvalid) {
                const int t = n - 1 - s;
                const int64_t idx = (sc.rowbase + t) * D + sc.d;
                const float y = (yv[k] + du[k]) * p.dir_scale[1] + ys[t * Ge::CPW + sc.c];
                stf(OUT, idx, y * silu(ldf(Z, idx)));
            }
        }
    }
}

// ---------------------------------------------------------------- features

// The per-token features of the layer written out (a diagnostic: the layer
// kernels keep them in registers): u_r = silu(conv_r(x)) and
// delta_r = softplus(dt_r + bias_r), with the conv accumulated in the same
// order (bias, then taps 0..3) and the same silu / softplus as the scans.
// One thread per (direction, row, token, channel); u, delta [2][batch][L][D].
template <typename Tin>
__global__ void __launch_bounds__(256) features_kernel(const Tin* __restrict__ x, const Tin* __restrict__ dt0,
                                                       const Tin* __restrict__ dt1, const float* __restrict__ conv_w,
                                                       const float* __restrict__ conv_b,
                                                       const float* __restrict__ dt_bias, int batch, int64_t L,
                                                       int D, float* __restrict__ u, float* __restrict__ delta) {
    const int64_t per_dir = (int64_t)batch * L * D;
    const int64_t total = 2 * per_dir;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int r = i >= per_dir ? 1 : 0;
        const int64_t e = i - r * per_dir;  // (b, t, d) flat
        const int d = (int)(e % D);
        const int64_t bt = e / D;
        const int64_t t = bt % L;
        const int64_t rowbase = (bt - t) * D;  // element index of (b, 0, 0)
        const int64_t rd = (int64_t)r * D + d;
        float cv = conv_b ? conv_b[rd] : 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int64_t src = r == 0 ? t - 3 + k : t + 3 - k;
            const float xv = (src >= 0 && src < L) ? ldf(x, rowbase + src * D + d) : 0.f;
            cv = fmaf(conv_w[rd * 4 + k], xv, cv);
        }
        u[i] = silu(cv);
        delta[i] = softplus(ldf(r == 0 ? dt0 : dt1, e) + dt_bias[rd]);
    }
}

}  // namespace bimamba

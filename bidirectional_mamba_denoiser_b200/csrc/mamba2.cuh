// mamba2.cuh -- the bidirectional Mamba-2 mixer at the shape of DiffuMamba's
// own denoiser ("DiffuMamba: High-Throughput Diffusion LMs with Mamba
// Backbone", §3.2 Eq. (4)-(6); App. C Table 8: Mamba-2 mixers, state
// dimension 128, conv dimension 4, no weight tie between directions; App. C
// Table 12: d_inner 3840, a conv over the 4096 channels of x, B and C, one
// group of B and C for 120 heads of 32 channels).
//
// Per direction r, batch row b and head h (P = 32 channels, N = 128 states):
//   v = silu(conv_r(xbc_r))   over x | B | C (causal forward, anti-causal reverse)
//   delta[t] = softplus(dt_r[t][h] + dt_bias_r[h])
//   S[p][n] <- exp(delta A_h) S[p][n] + delta x[t][p] B[t][n]
//   y_r[t][p] = sum_n C[t][n] S[p][n] + D_h x[t][p]
//   out = (y_0 + y_1) * silu(z)
//
// Three launches: m2_prep_kernel writes the conv + SiLU features of both
// directions and the per-head step sizes (fp32, to the workspace) -- B and C
// are shared by every head, so they are computed once, not once per head;
// m2_scan_kernel<true, ...> runs the forward and reverse scans at once,
// storing y_0 and y_1; m2_combine_kernel adds them and applies the gate.
//
// Scan: one warp per (batch row, head).  Lane (pb, nb) = (lane / 8, lane % 8)
// holds rows 8pb..8pb+7 x the 16 states {32i + 4nb + j : i, j < 4} of the
// head's 32 x 128 state, 128 registers; interleaving the states in groups of
// 4 makes every 16-byte B/C load of the 8 lanes of a row block one
// conflict-free shared-memory wavefront.  The state is kept divided by the running product of the
// decays, S~ = S / a_cum, so that a token costs one FMA per state for the
// update (S~ += (delta x / a_cum) B) and one for the readout (C . S~, times
// a_cum afterwards), instead of a multiply and two FMAs.  Before a_cum drops
// below 2^-60 the product is folded into S~ (a branch uniform over the warp:
// delta and A are the head's), so 1 / a_cum stays finite.  Rows of 8 partial
// C . S~ sums are combined over the 8 lanes of a row block by a transpose-
// reduce, after which every lane owns one (token, channel) output.  Token
// rows of x, B, C and delta (and, in reverse, the forward y and z of the
// head's channels) stream through a 2-stage shared-memory ring by cp.async;
// tokens past the end read zeros, so delta = 0 there and the step leaves the
// state exactly unchanged.
#pragma once

#include <cuda_fp16.h>

#include "scan_kernels.cuh"
#include "tcgen05_util.cuh"
#include "tma_util.cuh"

namespace bimamba {

constexpr int kM2P = 32;    // channels per head (headdim)
constexpr int kM2N = 128;   // states per channel (d_state)
constexpr int kM2T = 8;     // tokens per staged chunk of the scan
constexpr int kM2PrepT = 8;   // tokens per thread of the prep kernel
constexpr float kM2Floor = 8.673617379884035e-19f;  // 2^-60

struct M2Params {
    const void* xbc[2];    // [batch][L][CH] per direction, CH = H*P + 2N
    const void* z;         // [batch][L][H*P]
    const void* dt[2];     // [batch][L][H]
    const float* A;        // [2][H]
    const float* Dskip;    // [2][H]
    const float* dt_bias;  // [2][H]
    const float* conv_w;   // [2][CH][4]
    const float* conv_b;   // [2][CH] or nullptr
    void* out;             // [batch][L][H*P]
    float* V;              // [2][batch][L][CH]   conv + SiLU features
    float* DL;             // [2][batch][H][L]    step sizes
    float* YF;             // [batch][L][H*P]     forward y
    float* YB;             // [batch][L][H*P]     reverse y (tensor-core path: the reverse CTA's first half)
    int64_t L;
    int H, CH, batch;
    float dir_scale[2];    // 1, or 0 for a disabled direction (test flags)
    long long wait_limit;  // SM clocks a wait for a tile or a product may take (tensor-core path)
    long long meet_limit;  // SM clocks a reverse CTA may wait for its forward (tensor-core path)
    int starve;            // test aid (tensor-core path): issue no tile copies, so every wait gives up
    // tensor-core path: the prep kernel writes only the fp16 C/B tiles
    // ([2][batch][ceil(L/128)][C | B] x 128 x 128, rows in step order)
    unsigned char* tiles;
    // tensor-core path, directions as separate CTAs of one launch: [0] the
    // next ticket, [1 + b H + h] set once the forward (head h, batch row b)
    // has stored its y; zeroed before the launch
    int* sync;
    // block-cached decoding (step-by-step scan): the forward direction's cached
    // state [batch][H][P][N] fp32 and conv tail [batch][3][CH] (xBC rows before
    // token 0, oldest first); nullptr = zero state / zero halo / no commit
    const float* S_in;
    float* S_out;
    const void* tail_in;
    void* tail_out;
};

// 8 consecutive channels of one row, kept as loaded (bf16: one 16-byte
// word, unpacked on use) to hold the prep kernel's 11 rows in few registers.
template <typename Tin>
struct Row8;
template <>
struct Row8<__nv_bfloat16> {
    uint4 q;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { q = *reinterpret_cast<const uint4*>(p); }
    __device__ __forceinline__ void zero() { q = make_uint4(0u, 0u, 0u, 0u); }
    // bf16 -> fp32 is exact: the bf16 bits are the high half
    __device__ __forceinline__ float get(int i) const {
        const uint32_t w = i < 2 ? q.x : i < 4 ? q.y : i < 6 ? q.z : q.w;
        return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
    }
};
template <>
struct Row8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p) {
        a = *reinterpret_cast<const float4*>(p);
        b = *reinterpret_cast<const float4*>(p + 4);
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ float get(int i) const {
        const float4& v = i < 4 ? a : b;
        const int j = i & 3;
        return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
    }
};

constexpr int kM2Chunk = 128;  // steps per chunk of the tensor-core path

// Thread = 8 consecutive channels of one direction over 8 tokens; its 11
// input rows (8 + the 3-row conv halo) are loaded first, 16 bytes at a time,
// then the 64 outputs computed and stored as 16-byte rows.  Needs CH % 8 == 0
// and 16-byte aligned rows (CH * sizeof(Tin) % 16 == 0, aligned xbc).
// TILES = false: grid (ceil(L / 8), ceil(CH / 1024), 2 * batch), block 128;
// every channel to V (fp32) and the step sizes to DL.  TILES = true
// (tensor-core path, whose scan kernel computes the x channels and step
// sizes itself): grid (ceil(L / 32), 1, 2 * batch), block 128 = 4 token
// groups x the 32 threads of the B and C channels, written in fp16 into the
// chunk tiles at the token's step (forward: token t is step t; reverse: step
// nc*128-1-t, the chunks of both directions covering the same tokens).  C is
// K-major [step][n] (a 16-byte row of 8 channels per token); B is MN-major
// with the 8-n groups adjacent (f16_mn_kfast(step, n): a 16-byte run of 8
// steps per channel, stored once per 8-token group), the layout in which the
// scan kernel appends the state's fp16 copy to make one operand of G and
// C S^T.
template <typename Tin, bool TILES>
__global__ void __launch_bounds__(128) m2_prep_kernel(const M2Params p) {
    constexpr int TT = kM2PrepT;
    const int64_t L = p.L;
    const int CH = p.CH, H = p.H;
    const int c0 = TILES ? H * kM2P + (int)(threadIdx.x & 31) * 8 : (blockIdx.y * 128 + threadIdx.x) * 8;
    const int64_t t0 = TILES ? ((int64_t)blockIdx.x * 4 + (threadIdx.x >> 5)) * TT : (int64_t)blockIdx.x * TT;
    const int r = blockIdx.z / p.batch, b = blockIdx.z % p.batch;
    // per thread 8 rows of 16 bytes, rows of neighbouring threads 144 bytes apart (2-way bank
    // conflicts at most for the 16 B-channel threads of a warp)
    constexpr int kBStageStride = 144;
    __shared__ __align__(16) unsigned char bstage[TILES ? 128 * kBStageStride : 16];
    if (c0 < CH) {
        const Tin* X = static_cast<const Tin*>(p.xbc[r]) + (int64_t)b * L * CH + c0;
        float w[8][4], cb[8];
        {
            const float4* wp = reinterpret_cast<const float4*>(p.conv_w + ((int64_t)r * CH + c0) * 4);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 v = wp[q];
                w[q][0] = v.x; w[q][1] = v.y; w[q][2] = v.z; w[q][3] = v.w;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) cb[q] = p.conv_b ? p.conv_b[r * CH + c0 + q] : 0.f;
        }
        float* V = p.V + ((int64_t)r * p.batch + b) * L * CH + c0;
        // xw[k] = row t0 - 3 + k (forward) or t0 + k (reverse), zero outside [0, L)
        Row8<Tin> xw[TT + 3];
        const int64_t base = r == 0 ? t0 - 3 : t0;
        const Tin* tail = r == 0 && p.tail_in ? static_cast<const Tin*>(p.tail_in) + (int64_t)b * 3 * CH + c0 : nullptr;
#pragma unroll
        for (int k = 0; k < TT + 3; ++k) {
            const int64_t i = base + k;
            if (i >= 0 && i < L)
                xw[k].load(X + i * CH);
            else if (i < 0 && tail)  // forward halo from the cached tail (rows -3..-1)
                xw[k].load(tail + (3 + i) * CH);
            else
                xw[k].zero();
        }
        // TILES, B channels: the group's 8 steps of each of the thread's 8 channels gather in
        // fp16 in the thread's own shared-memory rows (one 16-byte row per channel; a token's step
        // within the group is k forward, 7 - k in reverse; steps past the end stay zero)
        const int HPc = H * kM2P;
        const bool isB = TILES && c0 < HPc + kM2N;
        unsigned char* brow = bstage + threadIdx.x * kBStageStride;
        if (isB) {
#pragma unroll
            for (int q = 0; q < 8; ++q) reinterpret_cast<uint4*>(brow + 16 * q)[0] = make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int k = 0; k < TT; ++k) {
            const int64_t t = t0 + k;
            if (t >= L) break;
            float v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                // forward: tap j on x[t-3+j] = xw[k+j]; reverse: tap j on x[t+3-j] = xw[k+3-j]
                const float a = r == 0 ? fmaf(w[q][3], xw[k + 3].get(q), fmaf(w[q][2], xw[k + 2].get(q),
                                             fmaf(w[q][1], xw[k + 1].get(q), fmaf(w[q][0], xw[k].get(q), cb[q]))))
                                       : fmaf(w[q][3], xw[k].get(q), fmaf(w[q][2], xw[k + 1].get(q),
                                             fmaf(w[q][1], xw[k + 2].get(q), fmaf(w[q][0], xw[k + 3].get(q), cb[q]))));
                v[q] = silu(a);
            }
            if constexpr (!TILES) {
                float4* dst = reinterpret_cast<float4*>(V + t * CH);
                dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                dst[1] = make_float4(v[4], v[5], v[6], v[7]);
            } else if (isB) {
                const int sl = r == 0 ? k : TT - 1 - k;
#pragma unroll
                for (int q = 0; q < 8; ++q) reinterpret_cast<__half*>(brow + 16 * q)[sl] = __float2half_rn(v[q]);
            } else {
                const __half2 h0 = __floats2half2_rn(v[0], v[1]), h1 = __floats2half2_rn(v[2], v[3]);
                const __half2 h2 = __floats2half2_rn(v[4], v[5]), h3 = __floats2half2_rn(v[6], v[7]);
                const uint4 q = make_uint4(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1),
                                           *reinterpret_cast<const uint32_t*>(&h2), *reinterpret_cast<const uint32_t*>(&h3));
                const int n0 = c0 - HPc - kM2N;
                const int64_t nc = (L + kM2Chunk - 1) / kM2Chunk;
                const int64_t step = r == 0 ? t : nc * kM2Chunk - 1 - t;  // chunks aligned in token space
                unsigned char* T = p.tiles + (((int64_t)r * p.batch + b) * nc + step / kM2Chunk) *
                                                 (2 * kM2Chunk * kM2N * 2);
                *reinterpret_cast<uint4*>(T + f16_kmajor((int)(step % kM2Chunk), n0, kM2N)) = q;
            }
        }
        if (isB && t0 < L) {  // the group's 8 steps of each channel: one 16-byte run per channel
            static_assert(TT == 8, "one 8-step group per thread");
            const int n0 = c0 - HPc;
            const int64_t nc = (L + kM2Chunk - 1) / kM2Chunk;
            const int64_t s0 = r == 0 ? t0 : nc * kM2Chunk - TT - t0;  // the group's first step
            unsigned char* T = p.tiles + (((int64_t)r * p.batch + b) * nc + s0 / kM2Chunk) * (2 * kM2Chunk * kM2N * 2) +
                               kM2Chunk * kM2N * 2;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<uint4*>(T + f16_mn_kfast((int)(s0 % kM2Chunk), n0 + q, kM2N)) =
                    reinterpret_cast<const uint4*>(brow + 16 * q)[0];
        }
    }
    if (!TILES && blockIdx.y == 0) {
        for (int h = threadIdx.x; h < H; h += 128) {
            const Tin* DT = static_cast<const Tin*>(p.dt[r]) + (int64_t)b * L * H + h;
            const float bias = p.dt_bias[r * H + h];
            float* DLh = p.DL + (((int64_t)r * p.batch + b) * H + h) * L;
#pragma unroll
            for (int k = 0; k < TT; ++k) {
                const int64_t t = t0 + k;
                if (t < L) DLh[t] = softplus(ldf(DT, t * H) + bias);
            }
        }
    }
}

// block 32: one warp scans one head of one batch row in one direction and
// stores its y (p.YF forward, p.YB reverse; not stored where null).  BOTH:
// grid (2 H, batch), CTA 2h + r runs head h in direction r, so both
// directions are in flight at once (m2_combine_kernel then adds and gates);
// else grid (H, batch), forward only (a prefix scan).
template <bool BOTH, typename Tin>
__global__ void __launch_bounds__(32, 8) m2_scan_kernel(const M2Params p) {
    constexpr int P = kM2P, N = kM2N, T = kM2T;
    __shared__ __align__(16) float xs[2][T][P];
    __shared__ __align__(16) float bs[2][T][N];
    __shared__ __align__(16) float cs[2][T][N];
    __shared__ __align__(16) float ds[2][T];
    const int lane = threadIdx.x;
    const int DIR = BOTH ? (int)(blockIdx.x & 1) : 0;
    const int h = BOTH ? (int)(blockIdx.x >> 1) : (int)blockIdx.x, b = blockIdx.y;
    const int pb = lane >> 3, nb = lane & 7;
    const int64_t L = p.L;
    const int H = p.H, CH = p.CH, HP = H * P;
    const float* Vb = p.V + ((int64_t)DIR * p.batch + b) * L * CH;
    const float* Dh = p.DL + (((int64_t)DIR * p.batch + b) * H + h) * L;
    const int nc = (int)((L + T - 1) / T);

    // chunk i of the walk (chunk k = tokens [kT, kT+T)) into ring slot buf
    auto stage = [&](int i, int buf) {
        const int64_t row0 = (int64_t)(DIR == 0 ? i : nc - 1 - i) * T;
        for (int e = lane; e < T * (P / 4); e += 32) {
            const int rr = e / (P / 4), q = e % (P / 4);
            const bool ok = row0 + rr < L;
            cp_async<16>(&xs[buf][rr][4 * q], Vb + (ok ? row0 + rr : 0) * CH + h * P + 4 * q, ok);
        }
        for (int e = lane; e < T * (N / 4); e += 32) {
            const int rr = e / (N / 4), q = e % (N / 4);
            const bool ok = row0 + rr < L;
            const float* row = Vb + (ok ? row0 + rr : 0) * CH + HP;
            cp_async<16>(&bs[buf][rr][4 * q], row + 4 * q, ok);
            cp_async<16>(&cs[buf][rr][4 * q], row + N + 4 * q, ok);
        }
        if (lane < T) {
            const bool ok = row0 + lane < L;
            cp_async<4>(&ds[buf][lane], Dh + (ok ? row0 + lane : 0), ok);
        }
        cp_async_commit();
    };

    const float A2 = p.A[DIR * H + h] * kLog2e;
    const float Dskip = p.Dskip[DIR * H + h];
    const float scale = p.dir_scale[DIR];
    float* const Y = DIR == 0 ? p.YF : p.YB;
    // S[i][4q+j] = state (row 8pb + i, state 32q + 4nb + j)
    float S[8][16];
    const int64_t sbase = ((int64_t)b * H + h) * P * N;
    if (DIR == 0 && p.S_in) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 v = *reinterpret_cast<const float4*>(p.S_in + sbase + (8 * pb + i) * N + 32 * q + 4 * nb);
                S[i][4 * q] = v.x; S[i][4 * q + 1] = v.y; S[i][4 * q + 2] = v.z; S[i][4 * q + 3] = v.w;
            }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int n = 0; n < 16; ++n) S[i][n] = 0.f;
    }
    float acum = 1.f;

    stage(0, 0);
    if (nc > 1) stage(1, 1);
#pragma unroll 1
    for (int i = 0; i < nc; ++i) {
        const int buf = i & 1;
        if (i + 1 < nc)
            cp_async_wait_pending<1>();
        else
            cp_async_wait_pending<0>();
        __syncwarp();
        const int64_t row0 = (int64_t)(DIR == 0 ? i : nc - 1 - i) * T;
#pragma unroll 1
        for (int s = 0; s < T; ++s) {
            const int rr = DIR == 0 ? s : T - 1 - s;
            const float dl = ds[buf][rr];
            const float na = acum * ex2_approx(dl * A2);
            if (na < kM2Floor) {  // fold the decay product into the state
#pragma unroll
                for (int i2 = 0; i2 < 8; ++i2)
#pragma unroll
                    for (int n = 0; n < 16; ++n) S[i2][n] *= na;
                acum = 1.f;
            } else {
                acum = na;
            }
            const float sc = dl * rcp_approx(acum);
            float xd[8], bv[16], cv[16];
            {
                const float4 x0 = *reinterpret_cast<const float4*>(&xs[buf][rr][8 * pb]);
                const float4 x1 = *reinterpret_cast<const float4*>(&xs[buf][rr][8 * pb + 4]);
                xd[0] = x0.x * sc; xd[1] = x0.y * sc; xd[2] = x0.z * sc; xd[3] = x0.w * sc;
                xd[4] = x1.x * sc; xd[5] = x1.y * sc; xd[6] = x1.z * sc; xd[7] = x1.w * sc;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 b4 = *reinterpret_cast<const float4*>(&bs[buf][rr][32 * q + 4 * nb]);
                const float4 c4 = *reinterpret_cast<const float4*>(&cs[buf][rr][32 * q + 4 * nb]);
                bv[4 * q] = b4.x; bv[4 * q + 1] = b4.y; bv[4 * q + 2] = b4.z; bv[4 * q + 3] = b4.w;
                cv[4 * q] = c4.x; cv[4 * q + 1] = c4.y; cv[4 * q + 2] = c4.z; cv[4 * q + 3] = c4.w;
            }
            float acc[8];
#pragma unroll
            for (int i2 = 0; i2 < 8; ++i2) {
                const float2 xx = make_float2(xd[i2], xd[i2]);
                float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
                for (int n = 0; n < 16; n += 2) {
                    const float2 hh = fma2(xx, make_float2(bv[n], bv[n + 1]), make_float2(S[i2][n], S[i2][n + 1]));
                    S[i2][n] = hh.x;
                    S[i2][n + 1] = hh.y;
                    a2 = fma2(make_float2(cv[n], cv[n + 1]), hh, a2);
                }
                acc[i2] = a2.x + a2.y;
            }
            const float yr = group_transpose_reduce<8, 1>(acc, nb);  // row 8pb + nb
            const int64_t t = row0 + rr;
            if (t < L) {
                const int prow = 8 * pb + nb;
                const float y = (acum * yr + Dskip * xs[buf][rr][prow]) * scale;
                const int64_t o = ((int64_t)b * L + t) * HP + (int64_t)h * P + prow;
                if (Y) Y[o] = y;  // no y for a prefix scan
            }
        }
        __syncwarp();
        if (i + 2 < nc) stage(i + 2, buf);
    }
    // commit: the forward state after the last token (each element written by the lane that read it)
    if (DIR == 0 && p.S_out) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<float4*>(p.S_out + sbase + (8 * pb + i) * N + 32 * q + 4 * nb) =
                    make_float4(acum * S[i][4 * q], acum * S[i][4 * q + 1], acum * S[i][4 * q + 2], acum * S[i][4 * q + 3]);
    }
}

// grid-stride over the call's batch * L * H*P outputs, 4 per thread (H*P % 4
// == 0): out = (y_0 + y_1) * silu(z) from p.YF and p.YB.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) m2_combine_kernel(const M2Params p) {
    const int64_t n4 = (int64_t)p.batch * p.L * p.H * kM2P / 4;
    const float4* yf = reinterpret_cast<const float4*>(p.YF);
    const float4* yb = reinterpret_cast<const float4*>(p.YB);
    const Tin* z = static_cast<const Tin*>(p.z);
    Tout* out = static_cast<Tout*>(p.out);
    for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n4; i += (int64_t)gridDim.x * 256) {
        const float4 a = yf[i], c = yb[i];
        const float s[4] = {a.x + c.x, a.y + c.y, a.z + c.z, a.w + c.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) stf(out, 4 * i + u, s[u] * silu(ldf(z, 4 * i + u)));
    }
}

// grid (ceil(CH / 128), batch), block 128: the forward conv tail after L more
// tokens of xBC (direction 0): rows L-3..L-1, reaching back into the old tail
// when L < 3.  Each thread reads its channel's three rows before writing, so
// tail_out may be tail_in.
template <typename Tin>
__global__ void __launch_bounds__(128) m2_tail_kernel(const M2Params p) {
    const int c = blockIdx.x * 128 + threadIdx.x;
    const int b = blockIdx.y;
    if (c >= p.CH) return;
    const int64_t L = p.L;
    const int CH = p.CH;
    const Tin* X = static_cast<const Tin*>(p.xbc[0]) + (int64_t)b * L * CH + c;
    const Tin* old = p.tail_in ? static_cast<const Tin*>(p.tail_in) + (int64_t)b * 3 * CH + c : nullptr;
    Tin v[3];
#pragma unroll
    for (int q = 0; q < 3; ++q) {
        const int64_t t = L - 3 + q;
        v[q] = t >= 0 ? X[t * CH] : (old ? old[(t + 3) * CH] : cvt_from<Tin>(0.f));
    }
    Tin* out = static_cast<Tin*>(p.tail_out) + (int64_t)b * 3 * CH + c;
#pragma unroll
    for (int q = 0; q < 3; ++q) out[q * CH] = v[q];
}

}  // namespace bimamba

// block_fused.cuh -- the block step of block-cached decoding ("DiffuMamba:
// High-Throughput Diffusion LMs with Mamba Backbone", §4.3; "Training Hybrid
// Block Diffusion Language Models with Partial Bidirectionality", abstract):
// the forward direction continues from the cached state over the active
// block, the reverse direction sees the block alone, and the two are added
// and gated.
//
// A CTA is a forward warp and a reverse warp over 32 channels of one batch
// row; lane l owns channel ct0 + l and all 16 of its states.  Each warp first
// stages its direction's block into shared memory in step order (step s is
// token s forward, token n-1-s in reverse): x with the 3-step conv halo in
// front (the cached tail forward, zeros past the block end in reverse), dt,
// and B|C as fp32.  It then scans the block -- per step conv + SiLU,
// softplus, 16 state updates with packed f32x2 arithmetic and one MUFU exp2
// each -- writing y per token to shared memory.  After one barrier the two
// warps gate half of the tokens each.  With a commit, the forward warp
// writes the new state and conv tail in place (each value is read and
// written by the same lane, so new_state may be the prefix state).
#pragma once

#include "scan_kernels.cuh"
#include "tma_util.cuh"

namespace bimamba {

// Shared memory of one direction for a block of up to n tokens (floats).
__host__ __device__ constexpr int block_dir_floats(int n) { return (n + 3) * 32 + n * 32 + n * 32 + n * 32; }

template <typename Tin, int DIR>
__device__ __forceinline__ void block_direction(const KParams& p, float* sm, int lane) {
    const int n = (int)p.L;
    const int b = blockIdx.y;
    const int ct0 = blockIdx.x * 32;
    const int D = p.D;
    const int d = ct0 + lane;
    const bool dvalid = d < D;
    float* xs = sm;                 // [n + 3][32]: steps -3 .. n-1
    float* dts = xs + (n + 3) * 32;  // [n][32]
    float* bcs = dts + n * 32;       // [n][B 16 | C 16]
    float* ys = bcs + n * 32;        // [n][32] y by token
    const Tin* X = static_cast<const Tin*>(p.x);
    const Tin* DT = static_cast<const Tin*>(p.dt[DIR]);
    const Tin* Bp = static_cast<const Tin*>(p.B[DIR]);
    const Tin* Cp = static_cast<const Tin*>(p.C[DIR]);
    const int64_t row0 = (int64_t)b * n;  // block tensors are [batch][n][...]

    // ---- stage the block in step order
    const Tin* tail = static_cast<const Tin*>(p.tail_in);
    for (int q = 0; q < 3; ++q)
        xs[q * 32 + lane] = (DIR == 0 && dvalid) ? ldf(tail, ((int64_t)b * 3 + q) * D + d) : 0.f;
    const int col = lane & (kNState - 1);
    const Tin* bcsrc = lane < kNState ? Bp : Cp;
    for (int s = 0; s < n; ++s) {
        const int t = DIR == 0 ? s : n - 1 - s;
        xs[(3 + s) * 32 + lane] = dvalid ? ldf(X, (row0 + t) * D + d) : 0.f;
        dts[s * 32 + lane] = dvalid ? ldf(DT, (row0 + t) * D + d) : 0.f;
        bcs[s * 32 + lane] = ldf(bcsrc, (row0 + t) * kNState + col);
    }
    __syncwarp();

    // ---- per-lane parameters and state
    const int64_t rd = (int64_t)DIR * D + (dvalid ? d : 0);
    float w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = dvalid ? p.conv_w[rd * 4 + k] : 0.f;
    const float cb = (dvalid && p.conv_b) ? p.conv_b[rd] : 0.f;
    const float bias = dvalid ? p.dt_bias[rd] : 0.f;
    const float Dd = dvalid ? p.Dskip[rd] : 0.f;
    float A2[kNState], h[kNState];
#pragma unroll
    for (int q = 0; q < kNState; ++q) {
        A2[q] = dvalid ? p.A[rd * kNState + q] * kLog2e : 0.f;
        h[q] = (DIR == 0 && dvalid) ? p.h_in[((int64_t)b * D + d) * kNState + q] : 0.f;
    }
    const float scale = p.dir_scale[DIR];
    float x0 = xs[lane], x1 = xs[32 + lane], x2 = xs[64 + lane];

    // ---- scan the block
#pragma unroll 2
    for (int s = 0; s < n; ++s) {
        const float x3 = xs[(3 + s) * 32 + lane];
        float cv = fmaf(w[0], x0, cb);
        cv = fmaf(w[1], x1, cv);
        cv = fmaf(w[2], x2, cv);
        cv = fmaf(w[3], x3, cv);
        x0 = x1; x1 = x2; x2 = x3;
        const float u = silu(cv);
        const float dl = softplus(dts[s * 32 + lane] + bias);
        const float2 dd = make_float2(dl, dl);
        const float2 uu = make_float2(dl * u, dl * u);
        const float* rowp = bcs + s * 32;
        float bv[kNState], cv16[kNState];
        load_states<kNState>(rowp, bv);
        load_states<kNState>(rowp + kNState, cv16);
        float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int sp = 0; sp < kNState; sp += 2) {
            const float2 v = mul2(dd, make_float2(A2[sp], A2[sp + 1]));
            const float2 ea = make_float2(ex2_approx(v.x), ex2_approx(v.y));
            const float2 drive = mul2(uu, make_float2(bv[sp], bv[sp + 1]));
            const float2 hh = fma2(ea, make_float2(h[sp], h[sp + 1]), drive);
            h[sp] = hh.x;
            h[sp + 1] = hh.y;
            acc2 = fma2(make_float2(cv16[sp], cv16[sp + 1]), hh, acc2);
        }
        const int t = DIR == 0 ? s : n - 1 - s;
        ys[t * 32 + lane] = (acc2.x + acc2.y + Dd * u) * scale;
    }

    // ---- commit: the forward state after the block and its last three x
    if (DIR == 0 && p.h_out && dvalid) {
#pragma unroll
        for (int q = 0; q < kNState; ++q) p.h_out[((int64_t)b * D + d) * kNState + q] = h[q];
        Tin* tail_out = static_cast<Tin*>(p.tail_out);
        // steps n-3 .. n-1 are rows n .. n+2 (the old tail when n < 3)
        for (int q = 0; q < 3; ++q) tail_out[((int64_t)b * 3 + q) * D + d] = cvt_from<Tin>(xs[(n + q) * 32 + lane]);
    }
}

// grid (ceil(D / 32), batch), block 64 (forward warp, reverse warp);
// dynamic shared memory 2 * block_dir_floats(n) * 4 bytes.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(64, 8) fused_block_kernel(const KParams p) {
    extern __shared__ __align__(16) float smb[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = (int)p.L;
    float* sm0 = smb;
    float* sm1 = smb + block_dir_floats(n);
    if (warp == 0)
        block_direction<Tin, 0>(p, sm0, lane);
    else
        block_direction<Tin, 1>(p, sm1, lane);
    named_bar_sync(1, 64);
    // gate half of the tokens per warp
    const float* y0 = sm0 + (n + 3) * 32 + 2 * n * 32;  // the ys part of each direction's area
    const float* y1 = sm1 + (n + 3) * 32 + 2 * n * 32;
    const int b = blockIdx.y;
    const int d = blockIdx.x * 32 + lane;
    if (d >= p.D) return;
    const int half = (n + 1) / 2;
    const int t0 = warp == 0 ? 0 : half, t1 = warp == 0 ? half : n;
    const Tin* Z = static_cast<const Tin*>(p.z);
    Tout* OUT = static_cast<Tout*>(p.out);
    for (int t = t0; t < t1; ++t) {
        const int64_t idx = ((int64_t)b * n + t) * p.D + d;
        stf(OUT, idx, (y0[t * 32 + lane] + y1[t * 32 + lane]) * silu(ldf(Z, idx)));
    }
}

}  // namespace bimamba

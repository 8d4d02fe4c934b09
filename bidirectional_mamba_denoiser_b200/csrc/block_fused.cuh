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
// and B|C as fp32, eight rows per batch of loads so that their DRAM latencies
// overlap.  It then scans the block -- per step conv + SiLU, softplus, 16
// state updates with packed f32x2 arithmetic and one MUFU exp2 each --
// writing y in step order over the dt slot that step has just consumed.
// After one barrier the two warps gate half of the tokens each.  With a commit, the forward warp
// writes the new state and conv tail in place (each value is read and
// written by the same lane, so new_state may be the prefix state).
#pragma once

#include "scan_kernels.cuh"
#include "tma_util.cuh"

namespace bimamba {

// Shared memory of one direction for a block of up to n tokens (floats).
// x with its halo, dt (overwritten by y), B|C.
__host__ __device__ constexpr int block_dir_floats(int n) { return (n + 3) * 32 + n * 32 + n * 32; }

constexpr int kBlockLoadBatch = 8;

template <typename Tin, int DIR>
__device__ __forceinline__ void block_direction(const KParams& p, float* sm, int lane) {
    const int n = (int)p.L;
    const int b = blockIdx.y;
    const int ct0 = blockIdx.x * 32;
    const int D = p.D;
    const int d = ct0 + lane;
    const bool dvalid = d < D;
    float* xs = sm;                  // [n + 3][32]: steps -3 .. n-1
    float* dts = xs + (n + 3) * 32;  // [n][32] dt by step, then y by step
    float* bcs = dts + n * 32;       // [n][B 16 | C 16]
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
    for (int s0 = 0; s0 < n; s0 += kBlockLoadBatch) {
        float xv[kBlockLoadBatch], dv[kBlockLoadBatch], bv[kBlockLoadBatch];
#pragma unroll
        for (int j = 0; j < kBlockLoadBatch; ++j) {
            const int s = s0 + j;
            const int t = DIR == 0 ? s : n - 1 - s;
            const bool in = s < n;
            xv[j] = (in && dvalid) ? ldf(X, (row0 + t) * D + d) : 0.f;
            dv[j] = (in && dvalid) ? ldf(DT, (row0 + t) * D + d) : 0.f;
            bv[j] = in ? ldf(bcsrc, (row0 + t) * kNState + col) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < kBlockLoadBatch; ++j) {
            const int s = s0 + j;
            if (s < n) {
                xs[(3 + s) * 32 + lane] = xv[j];
                dts[s * 32 + lane] = dv[j];
                bcs[s * 32 + lane] = bv[j];
            }
        }
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
        dts[s * 32 + lane] = (acc2.x + acc2.y + Dd * u) * scale;  // dt of step s already read
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
    // gate half of the tokens per warp; y sits in step order where dt was,
    // so token t is step t forward and step n-1-t in reverse
    const float* y0 = sm0 + (n + 3) * 32;
    const float* y1 = sm1 + (n + 3) * 32;
    const int b = blockIdx.y;
    const int d = blockIdx.x * 32 + lane;
    if (d >= p.D) return;
    const int half = (n + 1) / 2;
    const int t0 = warp == 0 ? 0 : half, t1 = warp == 0 ? half : n;
    const Tin* Z = static_cast<const Tin*>(p.z);
    Tout* OUT = static_cast<Tout*>(p.out);
    for (int tb = t0; tb < t1; tb += kBlockLoadBatch) {
        float zv[kBlockLoadBatch];
#pragma unroll
        for (int j = 0; j < kBlockLoadBatch; ++j)
            zv[j] = tb + j < t1 ? ldf(Z, ((int64_t)b * n + tb + j) * p.D + d) : 0.f;
#pragma unroll
        for (int j = 0; j < kBlockLoadBatch; ++j) {
            const int t = tb + j;
            if (t < t1)
                stf(OUT, ((int64_t)b * n + t) * p.D + d,
                    (y0[t * 32 + lane] + y1[(n - 1 - t) * 32 + lane]) * silu(zv[j]));
        }
    }
}


// ---------------------------------------------------------------- staged by cp.async
//
// The same computation with every global read of a warp in flight at once:
// before the scan each warp issues 16-byte cp.async copies of its direction's
// block rows (x with the conv halo, dt, B, C) and of z for the tokens it
// gates, in their input dtype, and only then loads its parameters and state;
// one wait_group covers all of it.  Rows are kept in token order; the step
// index maps onto them (forward step s is token s, reverse step s token
// n-1-s).  x rows: forward [tail0, tail1, tail2, x0 .. x_{n-1}], reverse
// [x0 .. x_{n-1}, 0, 0, 0], so step i in -3 .. n-1 is row i+3 forward and
// row n-1-i in reverse.  Needs d_inner * sizeof(Tin) a multiple of 16 and
// 16-byte aligned x, z, dt, B, C and conv tail.

template <typename Tin>
struct AsyncBlockGeo {
    static constexpr int ESZ = (int)sizeof(Tin);
    static constexpr int ROW = 32 * ESZ;        // bytes of one 32-channel row
    static constexpr int PIECES = ROW / 16;     // 16-byte copies per row
    // bytes of one direction's area for a block of n tokens (z: half the rows)
    static __host__ __device__ constexpr int dir_bytes(int n) {
        return (n + 3) * ROW + n * ROW + 2 * n * 16 * ESZ + n * 128 + n * 128 + ((n + 1) / 2) * ROW;
    }
};

template <typename Tin>
__host__ __device__ constexpr int async_block_smem(int n) {
    return 2 * ((AsyncBlockGeo<Tin>::dir_bytes(n) + 15) & ~15);
}

// Copy `rows` rows of 32 channels starting at channel ct0 (row r from
// src_row(r)) into dst rows; pieces past d_inner are zero-filled.
template <typename Tin, typename F>
__device__ __forceinline__ void copy_rows(unsigned char* dst, int rows, F src_row, int ct0, int D, int lane) {
    using Ge = AsyncBlockGeo<Tin>;
    constexpr int CPP = 16 / Ge::ESZ;  // channels per piece
    for (int e = lane; e < rows * Ge::PIECES; e += 32) {
        const int r = e / Ge::PIECES, q = e % Ge::PIECES;
        const bool ok = ct0 + CPP * q < D;
        const Tin* src = src_row(r) + (ok ? ct0 + CPP * q : 0);
        cp_async<16>(dst + r * Ge::ROW + 16 * q, src, ok);
    }
}

template <typename Tin, int DIR>
__device__ __forceinline__ void async_block_direction(const KParams& p, unsigned char* sm, int lane, int t0,
                                                      int t1) {
    using Ge = AsyncBlockGeo<Tin>;
    const int n = (int)p.L;
    const int b = blockIdx.y;
    const int ct0 = blockIdx.x * 32;
    const int D = p.D;
    const int d = ct0 + lane;
    const bool dvalid = d < D;
    Tin* xr = reinterpret_cast<Tin*>(sm);                          // [n + 3][32]
    Tin* dtr = reinterpret_cast<Tin*>(sm + (n + 3) * Ge::ROW);     // [n][32] by token
    Tin* br = reinterpret_cast<Tin*>(sm + (2 * n + 3) * Ge::ROW);  // [n][16]
    Tin* cr = br + n * kNState;                                     // [n][16]
    float* bcs = reinterpret_cast<float*>(cr + n * kNState);        // [n][B 16 | C 16] fp32 by token
    float* ys = bcs + n * 32;                                       // [n][32] y by token
    Tin* zr = reinterpret_cast<Tin*>(ys + n * 32);                  // [t1 - t0][32]
    const Tin* X = static_cast<const Tin*>(p.x);
    const Tin* DT = static_cast<const Tin*>(p.dt[DIR]);
    const Tin* Z = static_cast<const Tin*>(p.z);
    const int64_t row0 = (int64_t)b * n;

    // ---- all of this warp's block reads, in flight together
    if (DIR == 0) {
        const Tin* tail = static_cast<const Tin*>(p.tail_in);
        copy_rows<Tin>(sm, 3, [&](int r) { return tail + ((int64_t)b * 3 + r) * D; }, ct0, D, lane);
        copy_rows<Tin>(sm + 3 * Ge::ROW, n, [&](int r) { return X + (row0 + r) * D; }, ct0, D, lane);
    } else {
        copy_rows<Tin>(sm, n, [&](int r) { return X + (row0 + r) * D; }, ct0, D, lane);
        for (int e = lane; e < 3 * Ge::PIECES; e += 32)
            cp_async<16>(sm + n * Ge::ROW + 16 * e, X, false);  // zero rows past the block end
    }
    copy_rows<Tin>(reinterpret_cast<unsigned char*>(dtr), n, [&](int r) { return DT + (row0 + r) * D; }, ct0, D,
                   lane);
    copy_rows<Tin>(reinterpret_cast<unsigned char*>(zr), t1 - t0, [&](int r) { return Z + (row0 + t0 + r) * D; },
                   ct0, D, lane);
    {
        // B and C of the block are contiguous: n * 16 values each
        const unsigned char* Bsrc = reinterpret_cast<const unsigned char*>(static_cast<const Tin*>(p.B[DIR]) +
                                                                            row0 * kNState);
        const unsigned char* Csrc = reinterpret_cast<const unsigned char*>(static_cast<const Tin*>(p.C[DIR]) +
                                                                            row0 * kNState);
        const int pieces = n * kNState * Ge::ESZ / 16;
        for (int e = lane; e < pieces; e += 32) {
            cp_async<16>(reinterpret_cast<unsigned char*>(br) + 16 * e, Bsrc + 16 * e, true);
            cp_async<16>(reinterpret_cast<unsigned char*>(cr) + 16 * e, Csrc + 16 * e, true);
        }
    }
    cp_async_commit();

    // ---- per-lane parameters and state (their latency overlaps the copies)
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

    cp_async_wait_all();
    __syncwarp();
    // B|C to fp32, one value per lane and token
    {
        const int col = lane & (kNState - 1);
        const Tin* src = lane < kNState ? br : cr;
        for (int t = 0; t < n; ++t) bcs[t * 32 + lane] = ldf(src, t * kNState + col);
    }
    __syncwarp();

    // step i (-3 .. n-1) of x is row i+3 forward, n-1-i in reverse
    auto xrow = [&](int i) { return DIR == 0 ? i + 3 : n - 1 - i; };
    float x0 = dvalid ? ldf(xr, xrow(-3) * 32 + lane) : 0.f;
    float x1 = dvalid ? ldf(xr, xrow(-2) * 32 + lane) : 0.f;
    float x2 = dvalid ? ldf(xr, xrow(-1) * 32 + lane) : 0.f;

#pragma unroll 2
    for (int s = 0; s < n; ++s) {
        const int t = DIR == 0 ? s : n - 1 - s;
        const float x3 = dvalid ? ldf(xr, xrow(s) * 32 + lane) : 0.f;
        float cv = fmaf(w[0], x0, cb);
        cv = fmaf(w[1], x1, cv);
        cv = fmaf(w[2], x2, cv);
        cv = fmaf(w[3], x3, cv);
        x0 = x1; x1 = x2; x2 = x3;
        const float u = silu(cv);
        const float dl = softplus((dvalid ? ldf(dtr, t * 32 + lane) : 0.f) + bias);
        const float2 dd = make_float2(dl, dl);
        const float2 uu = make_float2(dl * u, dl * u);
        const float* rowp = bcs + t * 32;
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
        ys[t * 32 + lane] = (acc2.x + acc2.y + Dd * u) * scale;
    }

    // ---- commit: the forward state after the block and its last three x
    if (DIR == 0 && p.h_out && dvalid) {
#pragma unroll
        for (int q = 0; q < kNState; ++q) p.h_out[((int64_t)b * D + d) * kNState + q] = h[q];
        Tin* tail_out = static_cast<Tin*>(p.tail_out);
        // rows n .. n+2 hold steps n-3 .. n-1 (the old tail rows when n < 3)
        for (int q = 0; q < 3; ++q) tail_out[((int64_t)b * 3 + q) * D + d] = xr[(n + q) * 32 + lane];
    }
}

// grid (ceil(D / 32), batch), block 64 (forward warp, reverse warp); the
// forward warp gates tokens [0, ceil(n/2)), the reverse warp the rest.
// Dynamic shared memory async_block_smem<Tin>(n) bytes.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(64, 7) async_block_kernel(const KParams p) {
    using Ge = AsyncBlockGeo<Tin>;
    extern __shared__ __align__(16) unsigned char sma[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = (int)p.L;
    const int half = (n + 1) / 2;
    const int t0 = warp == 0 ? 0 : half, t1 = warp == 0 ? half : n;
    const int area = (Ge::dir_bytes(n) + 15) & ~15;
    unsigned char* sm0 = sma;
    unsigned char* sm1 = sma + area;
    if (warp == 0)
        async_block_direction<Tin, 0>(p, sm0, lane, t0, t1);
    else
        async_block_direction<Tin, 1>(p, sm1, lane, t0, t1);
    named_bar_sync(1, 64);
    // y areas of both directions and this warp's z rows (see the layout above)
    const int ys_off = (2 * n + 3) * Ge::ROW + 2 * n * kNState * Ge::ESZ + n * 128;
    const float* y0 = reinterpret_cast<const float*>(sm0 + ys_off);
    const float* y1 = reinterpret_cast<const float*>(sm1 + ys_off);
    const Tin* zr = reinterpret_cast<const Tin*>((warp == 0 ? sm0 : sm1) + ys_off + n * 128);
    const int b = blockIdx.y;
    const int d = blockIdx.x * 32 + lane;
    if (d >= p.D) return;
    Tout* OUT = static_cast<Tout*>(p.out);
    for (int t = t0; t < t1; ++t)
        stf(OUT, ((int64_t)b * n + t) * p.D + d,
            (y0[t * 32 + lane] + y1[t * 32 + lane]) * silu(ldf(zr, (t - t0) * 32 + lane)));
}

}  // namespace bimamba

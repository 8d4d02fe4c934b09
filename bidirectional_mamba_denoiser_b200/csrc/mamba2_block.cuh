// mamba2_block.cuh -- the Mamba-2 block step's scan on the sm_100a tensor
// cores: one block of at most 32 steps per direction, the forward from the
// cached state ("DiffuMamba: High-Throughput Diffusion LMs with Mamba
// Backbone", §4.3 block-cached decoding), the reverse over the block alone.
//
// With c_t = sum_{u <= t} delta_u A_h (log2 units, inclusive), the block's
// initial state S_ (P x N per head) and G = C B^T (one 32 x 32 matrix per
// batch row and direction, shared by all heads):
//   y_t   = 2^{c_t} (C_t . S_) + sum_{s <= t} 2^{c_t - c_s} G[t][s] delta_s x_s + D x_t
//   S_end = 2^{c_end} S_ + sum_s 2^{c_end - c_s} delta_s x_s B_s^T
// the closed form of the step-by-step recurrence over the block.  Four heads
// of one (batch row, direction) share a CTA of 128 threads; thread (h, p) =
// warp h, lane p owns state row (h, p), which is TMEM lane 32 h + p:
//   Y2^T = S_ C^T         M = 128 (h, p), N = 32 (t), K = 128 (n)  tcgen05, TMEM cols [128, 160)
//   S_end = 2^{c_end} S_ + W B    M = 128 (h, p), N = 128 (n), K = 32 (t)  tcgen05, TMEM cols [0, 128)
//   G (once per batch row and direction, m2_block_gram_kernel) and the masked
//   intra-block sum (Y1): CUDA cores, fp32.
// fp16 operands with fp32 accumulation, as in the chunked dual form; used for
// bf16 I/O only.  Steps past the block's end are identity steps (delta 0,
// x 0); their outputs are not stored.
#pragma once

#include <cuda_fp16.h>

#include "mamba2.cuh"
#include "tcgen05_util.cuh"

namespace bimamba {

constexpr int kM2BlkT = 32;    // steps per block on this path
constexpr int kM2BlkHeads = 4;  // heads per CTA
constexpr int kM2GramRows = 4;  // G rows per CTA of the Gram kernel
// shared memory (bytes); the operands of the state update (B and W) only in a
// commit's forward CTAs, which launch with the larger size
constexpr int kBlkS16 = 0;        // state fp16, K-major [(h, p) 128][n 128]        32 KB
constexpr int kBlkC16 = 32768;    // C fp16, K-major [t 32][n 128]                  8 KB
constexpr int kBlkG = 40960;      // G fp32 [t][s]                                  4 KB
constexpr int kBlkCc = 45056;     // c fp32 [h][t]                                  512 B
constexpr int kBlkDl = 45568;     // delta fp32 [h][t]                              512 B
constexpr int kBlkSpan = 46080;   // int [h]: the head's decay span is too large to factor
constexpr int kBlkBar = 46096;    // mbarrier
constexpr int kBlkTmem = 46104;   // TMEM address
constexpr int kBlkB16 = 47104;    // B fp16, MN-major (n along MN, t along K)       8 KB  (commit)
constexpr int kBlkW16 = 55296;    // W fp16, K-major [(h, p) 128][t 32]              8 KB  (commit)
constexpr int kBlkSmemStep = 46108 + 128;    // + alignment slack
constexpr int kBlkSmemCommit = 63488 + 128;
constexpr float kBlkSpanMax = 100.f;  // largest log2 decay span taken in factored form

// G[r][b][t][s] = C_t . B_s of the block (fp32, 32 x 32 per batch row and
// direction; zero rows past the block's end), into p.tiles.  grid (batch, 2,
// 32 / kM2GramRows), block 128: CTA z computes rows t = 4z .. 4z + 3, thread
// (t, s) one entry.  The rows sit in shared memory with a 129-float stride,
// so that the 32 lanes of a warp read 32 distinct B rows in distinct banks.
__global__ void __launch_bounds__(128) m2_block_gram_kernel(const M2Params p) {
    constexpr int T = kM2BlkT, N = kM2N, RS = N + 1, R = kM2GramRows;
    __shared__ float sCr[R * RS], sBr[T * RS];
    const int b = blockIdx.x, DIR = blockIdx.y, t0 = blockIdx.z * R, tid = threadIdx.x;
    const int64_t L = p.L;
    const int CH = p.CH, HP = p.H * kM2P;
    const float* Vb = p.V + ((int64_t)DIR * p.batch + b) * L * CH;
    auto row_of = [&](int t) -> const float* {
        return Vb + (DIR == 0 ? (int64_t)t : L - 1 - t) * CH + HP;
    };
    // 16-byte loads, all of a thread's issued together
    float4 bq[T * N / 4 / 128];
#pragma unroll
    for (int j = 0; j < T * N / 4 / 128; ++j) {
        const int e = tid + 128 * j, t = e / (N / 4), q = e % (N / 4);
        bq[j] = t < L ? reinterpret_cast<const float4*>(row_of(t))[q] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int ec = tid, tc = ec / (N / 4), qc = ec % (N / 4);  // R * N / 4 == 128: one C load each
    const float4 cq = t0 + tc < L ? reinterpret_cast<const float4*>(row_of(t0 + tc) + N)[qc]
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < T * N / 4 / 128; ++j) {
        const int e = tid + 128 * j, t = e / (N / 4), q = e % (N / 4);
        float* d = sBr + t * RS + 4 * q;
        d[0] = bq[j].x; d[1] = bq[j].y; d[2] = bq[j].z; d[3] = bq[j].w;
    }
    {
        float* d = sCr + tc * RS + 4 * qc;
        d[0] = cq.x; d[1] = cq.y; d[2] = cq.z; d[3] = cq.w;
    }
    static_assert(R * N / 4 == 128, "one 16-byte C load per thread");
    __syncthreads();
    const int tl = tid >> 5, s = tid & 31;
    float g = 0.f;
#pragma unroll 16
    for (int n = 0; n < N; ++n) g = fmaf(sCr[tl * RS + n], sBr[s * RS + n], g);
    reinterpret_cast<float*>(p.tiles)[((int64_t)DIR * p.batch + b) * T * T + (t0 + tl) * T + s] = g;
}

// grid (H / 4, batch, 2), block 128, dynamic shared memory kBlkSmemCommit when
// p.S_out (a commit) else kBlkSmemStep.  L <= 32; G from m2_block_gram_kernel
// in p.tiles.  Writes y (times the direction's scale) to p.YF / p.YB like
// m2_scan_kernel, and, forward with p.S_out, the state after the block.  Which
// products run depends on the CTA: the reverse starts from zero (no C S_^T)
// and keeps no state, and the forward updates the state only on a commit.
__global__ void __launch_bounds__(128, 4) m2_block_mma_kernel(const M2Params p) {
    constexpr int T = kM2BlkT, P = kM2P, N = kM2N;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                                         ~static_cast<uintptr_t>(127));
    unsigned char* sS16 = sm + kBlkS16;
    unsigned char* sC16 = sm + kBlkC16;
    unsigned char* sB16 = sm + kBlkB16;
    unsigned char* sW16 = sm + kBlkW16;
    float* sG = reinterpret_cast<float*>(sm + kBlkG);
    float* sc = reinterpret_cast<float*>(sm + kBlkCc);
    float* sdl = reinterpret_cast<float*>(sm + kBlkDl);
    int* sbig = reinterpret_cast<int*>(sm + kBlkSpan);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kBlkBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kBlkTmem);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x * kM2BlkHeads + warp;  // this warp's head
    const int b = blockIdx.y, DIR = blockIdx.z;
    const bool with_state = DIR == 0 && p.S_in != nullptr;  // C S_^T runs
    const bool commit = DIR == 0 && p.S_out != nullptr;     // the state update runs and is stored
    const bool mma = with_state || commit;
    // TMEM: the state [0, 128) and C S_^T [128, 160) on a commit, else C S_^T alone in [0, 32)
    const uint32_t y2col = commit ? 128u : 0u;
    const int64_t L = p.L;
    const int H = p.H, CH = p.CH, HP = H * P;
    const float* Vb = p.V + ((int64_t)DIR * p.batch + b) * L * CH;
    // step t of the block is token t (forward) or L - 1 - t (reverse); steps >= L are identity steps
    auto token_of = [&](int t) -> int64_t { return DIR == 0 ? (int64_t)t : L - 1 - t; };

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        if (commit)
            tmem_alloc<256>(tmem_slot);
        else if (with_state)
            tmem_alloc<32>(tmem_slot);
    }

    // ---- step sizes and c_t of this warp's head (lane = step)
    const float A2 = p.A[DIR * H + h] * kLog2e;
    float dl = 0.f;
    if (lane < L) dl = p.DL[(((int64_t)DIR * p.batch + b) * H + h) * L + token_of(lane)];
    float c = dl * A2;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float v = __shfl_up_sync(0xffffffffu, c, off);
        if (lane >= off) c += v;
    }
    sc[warp * T + lane] = c;
    sdl[warp * T + lane] = dl;
    const float c_first = __shfl_sync(0xffffffffu, c, 0);
    const float c_end = __shfl_sync(0xffffffffu, c, 31);
    if (lane == 0) sbig[warp] = (c_first - c_end > kBlkSpanMax) ? 1 : 0;

    // ---- G, and the block's C (and, on a commit, B) rows as fp16 operand tiles (zeros past the end)
    {
        const float4* Gg = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.tiles) +
                                                           ((int64_t)DIR * p.batch + b) * T * T);
#pragma unroll
        for (int i = 0; i < 2; ++i) reinterpret_cast<float4*>(sG)[tid + 128 * i] = Gg[tid + 128 * i];
    }
    if (mma) {
        const int t = tid >> 2, n0 = 32 * (tid & 3);
        const bool ok = t < L;
        const float* row = Vb + (ok ? token_of(t) : 0) * CH + HP;
#pragma unroll
        for (int j = 0; j < 4; ++j) {  // 8 states at a time
            const int n = n0 + 8 * j;
            float bv[8], cv[8];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const float4 c4 = ok ? reinterpret_cast<const float4*>(row + N + n)[q] : make_float4(0.f, 0.f, 0.f, 0.f);
                cv[4 * q] = c4.x; cv[4 * q + 1] = c4.y; cv[4 * q + 2] = c4.z; cv[4 * q + 3] = c4.w;
                if (commit) {
                    const float4 b4 = ok ? reinterpret_cast<const float4*>(row + n)[q] : make_float4(0.f, 0.f, 0.f, 0.f);
                    bv[4 * q] = b4.x; bv[4 * q + 1] = b4.y; bv[4 * q + 2] = b4.z; bv[4 * q + 3] = b4.w;
                }
            }
            st_half8(sC16 + f16_kmajor(t, n, N), cv);
            if (commit) st_half8(sB16 + f16_mnmajor(n, t, N), bv);
        }
    }
    // ---- a decoding step's state row (h, p) (no commit): every load issued at once, stored as
    // the fp16 operand of C S_^T
    if (with_state && !commit) {
        const float4* srow = reinterpret_cast<const float4*>(p.S_in + (((int64_t)b * H + h) * P + lane) * N);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {  // two halves of 64 states, each half's loads issued together
            float4 v4[N / 8];
#pragma unroll
            for (int i = 0; i < N / 8; ++i) v4[i] = srow[hh * (N / 8) + i];
#pragma unroll
            for (int g = 0; g < N / 16; ++g) {
                const float v[8] = {v4[2 * g].x, v4[2 * g].y, v4[2 * g].z, v4[2 * g].w,
                                    v4[2 * g + 1].x, v4[2 * g + 1].y, v4[2 * g + 1].z, v4[2 * g + 1].w};
                st_half8(sS16 + f16_kmajor(tid, hh * (N / 2) + 8 * g, N), v);
            }
        }
    }
    // ---- x of this thread's channel (h, p = lane) at every step
    float x[T];
#pragma unroll
    for (int t = 0; t < T; ++t) x[t] = t < L ? Vb[token_of(t) * CH + (int64_t)h * P + lane] : 0.f;

    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tmem = mma ? *tmem_slot : 0u;
    const uint32_t lb = (uint32_t)(warp * 32) << 16;

    if (mma) {
        // ---- on a commit, the state row (h, p) (the cached state or zero): fp16 copy for C S_^T
        // and decayed fp32 in TMEM
        const float* srow = with_state ? p.S_in + (((int64_t)b * H + h) * P + lane) * N : nullptr;
        const float fdec = ex2_approx(c_end);
#pragma unroll 1
        for (int q = 0; q < (commit ? 4 : 0); ++q) {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 s4 = srow ? *reinterpret_cast<const float4*>(srow + 32 * q + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                v[i] = s4.x; v[i + 1] = s4.y; v[i + 2] = s4.z; v[i + 3] = s4.w;
            }
#pragma unroll
            for (int g = 0; g < 4; ++g) st_half8(sS16 + f16_kmajor(tid, 32 * q + 8 * g, N), v + 8 * g);
            if (commit) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= fdec;
                tmem_st32(tmem + 32 * q + lb, v);
            }
        }
        if (commit) {  // W row (h, p): 2^{c_end - c_t} delta_t x_t
            float w[T];
#pragma unroll
            for (int t = 0; t < T; ++t) w[t] = ex2_approx(c_end - sc[warp * T + t]) * sdl[warp * T + t] * x[t];
#pragma unroll
            for (int g = 0; g < 4; ++g) st_half8(sW16 + f16_kmajor(tid, 8 * g, T), w + 8 * g);
        }
        fence_async_smem();
        tmem_fence_before_sync();
        __syncthreads();
        tmem_fence_after_sync();
        if (tid == 0) {
            const uint32_t aS = smem_addr(sS16), aC = smem_addr(sC16);
            // Y2^T = S_ C^T: A K-major (rows (h, p), K = n), B K-major (rows t, K = n)
            umma_f16_k8<256 / 16, 256 / 16>(tmem + y2col, umma_desc(aS, 128, 2048), umma_desc(aC, 128, 2048),
                                            umma_idesc_f16(128, 32, false, false), false);
            if (commit) {
                // S += W B: A K-major (rows (h, p), K = t), B MN-major (MN = n, K = t)
                const uint32_t aB = smem_addr(sB16), aW = smem_addr(sW16);
                constexpr uint32_t ID_S = umma_idesc_f16(128, 128, false, true);
                umma_f16(tmem + 0, umma_desc(aW, 128, 512), umma_desc(aB, 2048, 128), ID_S, true);
                umma_f16(tmem + 0, umma_desc(aW + 256, 128, 512), umma_desc(aB + 4096, 2048, 128), ID_S, true);
            }
            umma_commit(bar);
        }
    }

    // ---- Y1 on the CUDA cores (while the products run): y_t starts at D x_t, then
    // + sum_{s <= t} 2^{c_t - c_s} G[t][s] delta_s x_s, factored through c_first while the span is small
    const float Dsk = p.Dskip[DIR * H + h];
    const float* cw = sc + warp * T;
    const float* dw = sdl + warp * T;
    float y[T];
#pragma unroll
    for (int t = 0; t < T; ++t) y[t] = Dsk * x[t];
    if (!sbig[warp]) {
#pragma unroll
        for (int s = 0; s < T; ++s) x[s] *= ex2_approx(c_first - cw[s]) * dw[s];  // x becomes z_s
#pragma unroll
        for (int t = 0; t < T; ++t) {
            float acc = 0.f;
#pragma unroll
            for (int s = 0; s <= t; ++s) acc = fmaf(sG[t * T + s], x[s], acc);
            y[t] = fmaf(ex2_approx(cw[t] - c_first), acc, y[t]);
        }
    } else {
#pragma unroll
        for (int s = 0; s < T; ++s) x[s] *= dw[s];
#pragma unroll
        for (int t = 0; t < T; ++t) {
            float acc = 0.f;
#pragma unroll
            for (int s = 0; s <= t; ++s) acc = fmaf(sG[t * T + s] * ex2_approx(cw[t] - cw[s]), x[s], acc);
            y[t] += acc;
        }
    }

    // ---- y_t (+ 2^{c_t} Y2 with a state), times the direction's scale
    if (mma) {
        mbar_wait_bounded(bar, 0, p.wait_limit);
        tmem_fence_after_sync();
        float y2[32];
        tmem_ld32(tmem + y2col + lb, y2);
#pragma unroll
        for (int t = 0; t < T; ++t) y[t] = fmaf(ex2_approx(cw[t]), y2[t], y[t]);
    }
    {
        const float scale = p.dir_scale[DIR];
        float* Y = DIR == 0 ? p.YF : p.YB;
        if (Y) {
#pragma unroll
            for (int t = 0; t < T; ++t)
                if (t < L) Y[((int64_t)b * L + token_of(t)) * HP + (int64_t)h * P + lane] = y[t] * scale;
        }
    }
    // ---- the forward state after the block
    if (commit) {
        float* orow = p.S_out + (((int64_t)b * H + h) * P + lane) * N;
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
            float v[32];
            tmem_ld32(tmem + 32 * q + lb, v);
#pragma unroll
            for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(orow + 32 * q + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    }
    if (mma) {
        tmem_fence_before_sync();
        __syncthreads();
        if (warp == 0) {
            if (commit)
                tmem_dealloc<256>(tmem);
            else
                tmem_dealloc<32>(tmem);
        }
    }
}

}  // namespace bimamba

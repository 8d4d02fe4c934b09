// mamba2_ssd.cuh -- the Mamba-2 mixer's scan in its chunked dual form on the
// sm_100a tensor cores (tcgen05, fp16 operands, fp32 accumulation in TMEM).
//
// Per direction, batch row b and head h, the scan over a chunk of Q = 128
// steps with a_t = delta_t A_h, c_t = sum_{u <= t} a_u (inside the chunk) and
// the state S_ (P x N) carried in from the previous chunk is
//   S_t = e^{c_t} S_ + sum_{s <= t} e^{c_t - c_s} delta_s x_s B_s^T
//   y_t = e^{c_t} (C_t . S_) + sum_{s <= t} (C_t . B_s) e^{c_t - c_s} delta_s x_s + D x_t
// (the same recurrence as the step-by-step scan, summed in closed form; the
// state-space-dual view of Mamba-2 the pages cite).  Four matrix products:
//   G   = C B^T                     (Q x Q, K = N)      -> TMEM cols [0, 128)
//   Y2  = C S_^T                    (Q x P, K = N)      -> TMEM cols [128, 160)
//         (one product: C times the B tile with the state's fp16 copy appended)
//   S^T = e^{c_end} S_^T + B^T W    (N x P, K = Q), W_s = e^{c_end - c_s} delta_s x_s
//                                                        -> TMEM cols [192, 224)
//   Y1  = M (delta x), M = G o e^{c_t - c_s} [s <= t]   (Q x P, K = Q)
//                                                        -> TMEM cols [160, 192)
//   y_t = Y1 + e^{c_t} Y2 + D x_t
// One CTA = one (head, batch row) in one direction, 256 threads: threads t
// and t + 128 own step t of the chunk (TMEM lane t) for the per-step work and
// state row n = t for the state epilogue, each for one half of the 32
// channels (and of the M row's four 32-column blocks), so that an SM's two
// CTAs give it 16 warps.  The per-step work starts from the inputs: the
// head's 32 xBC channels of step t arrive raw by cp.async into a
// shared-memory ring of 3 + 128 rows (the first three hold the last three
// steps of the previous chunk, the conv's halo, in step order -- so that the
// causal forward and the anti-causal reverse conv are the same code), the
// conv + SiLU of step t comes from rows t..t+3, and its step size
// softplus(dt + bias) from dt (computed by both threads of the step).  The
// chunk's C and B arrive as fp16 tiles by bulk copies (written by
// m2_prep_kernel<Tin, true>, in step order so that the reverse direction needs
// no other code): C K-major [step][n]; B MN-major with its 8-n groups
// adjacent, followed in shared memory by the carried state's fp16 copy in the
// same layout, so that G and C S_^T are one product of N = 160.  The B tile
// of the next chunk is fetched as soon as the
// products that read B are done, the C tile once M (which reuses C's
// buffer) has been consumed, and the next chunk's xBC rows and step sizes
// once this chunk's conv has read them.  Every mbarrier wait is bounded.
//
// Precision: fp16 operands (11-bit significands, like tf32) with fp32
// accumulation; the carried state stays fp32 in TMEM.  Used for bf16 I/O
// (within the 2e-3 bound); fp32 I/O runs the step-by-step CUDA-core scan.
#pragma once

#include <cuda_fp16.h>

#include "mamba2.cuh"
#include "tcgen05_util.cuh"

namespace bimamba {

constexpr int kSQ = kM2Chunk;               // steps per chunk (= MMA M)
constexpr int kTileBytes = kSQ * kM2N * 2;  // one fp16 C or B tile
// shared memory of one dual-form CTA (either kernel)
constexpr int kSsdC = 0, kSsdB = 32768, kSsdS = 65536, kSsdDX = 73728, kSsdW = 81920, kSsdC2 = 90112,
              kSsdTot = 90624, kSsdBar = 90688, kSsdTmem = 90728, kSsdX = 90752, kSsdE = 101232,
              kSsdCW = 101744, kSsdCB = 102256, kSsdSmem = 102384;
constexpr float kSsdSpanMax = 100.f;  // largest log2 decay span of a 32-step block taken in factored form
constexpr int kSsdXStride = 40;  // bf16 per xBC row in shared memory (80 B: conflict-free 16-byte accesses)
constexpr int kSsdThreads = 256;  // threads of a dual-form CTA: two per step of the chunk

// 8 fp32 values -> 8 fp16 in one 16-byte store.
__device__ __forceinline__ void st_half8(unsigned char* dst, const float* v) {
    __half2 h0 = __floats2half2_rn(v[0], v[1]), h1 = __floats2half2_rn(v[2], v[3]);
    __half2 h2 = __floats2half2_rn(v[4], v[5]), h3 = __floats2half2_rn(v[6], v[7]);
    *reinterpret_cast<uint4*>(dst) =
        make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                   *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
}

// 4 consecutive outputs: one 16-byte (fp32) or 8-byte (bf16) store.
__device__ __forceinline__ void store4(float* dst, const float (&v)[4]) {
    *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16* dst, const float (&v)[4]) {
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]), h1 = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(dst) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1));
}

// Both directions cut the sequence into the same chunks of Q tokens (chunk j
// = tokens [jQ, jQ + Q)); the forward walks chunks 0 .. nc-1 with step t of
// chunk j at token jQ + t, the reverse walks nc-1 .. 0 with step t at token
// jQ + Q-1-t.  When L % Q != 0 the reverse's first chunk starts with steps
// past the end, identity steps (step size 0, x zero).
// Both directions of a (head, batch row) run as the two CTAs of a cluster.
// Each walks its chunks in its own order; over the first half (forward:
// chunks 0 .. nc/2 - 1; reverse: chunks nc-1 .. nc/2) it stores its y to the
// workspace (p.YF forward, p.YB reverse).  The two then meet at a cluster
// barrier (release / acquire: each sees the other's stores), and over the
// second half each adds the partner's stored y to its own and applies the
// SiLU(z) gate.  Every token is gated exactly once, by the direction that
// reaches it second.
__device__ __forceinline__ void cluster_meet() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// CL: the two directions run as a cluster and meet halfway (above).  Without
// it the forward stores y for every chunk (p.YF) and the reverse, launched
// after it, gates every chunk with that y.  PREFIX (forward, no cluster): the
// prefix state of block-cached decoding -- only the state update runs (no G,
// C S_^T, M or output), from zero, and the final state goes to p.S_out.
template <int DIR, typename Tin, typename Tout, bool CL, bool PREFIX = false>
__device__ __forceinline__ void m2_ssd_dir(const M2Params& p, unsigned char* sm, const int h, const int b) {
    constexpr int Q = kSQ, P = kM2P;
    static_assert(sizeof(Tin) == 2, "the dual form reads bf16 inputs");
    static_assert(kSsdThreads == 2 * Q, "two threads per step");
    unsigned char* sC = sm + kSsdC;
    unsigned char* sB = sm + kSsdB;
    unsigned char* sDX = sm + kSsdDX;
    unsigned char* sW = sm + kSsdW;
    unsigned char* sS = sm + kSsdS;
    float* c2s = reinterpret_cast<float*>(sm + kSsdC2);
    float* wtot = reinterpret_cast<float*>(sm + kSsdTot);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kSsdBar);  // B tile, C tile, G + Y2, Y1, S
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kSsdTmem);
    Tin* sX = reinterpret_cast<Tin*>(sm + kSsdX);      // [3 + 128][kSsdXStride]: row 3 + s = xBC of step s
    float* sE = reinterpret_cast<float*>(sm + kSsdE);  // [128]: 2^(c of step 32j - c of step s), s in block j
    float* sCW = reinterpret_cast<float*>(sm + kSsdCW);  // [4][32]: conv tap j of the head's channel p
    float* sCB = reinterpret_cast<float*>(sm + kSsdCB);    // [32]: conv bias
    int* bigspan = reinterpret_cast<int*>(sm + kSsdTot + 16);  // [4]: block j's decay span exceeds kSsdSpanMax
    const int tid = threadIdx.x;
    const int t = tid & (Q - 1);      // the step (TMEM lane, state row) this thread works on
    const int hf = tid >> 7;          // which half of the step's 32 channels: 16 hf .. 16 hf + 15
    const int warp = (tid >> 5) & 3;  // the step block, = the TMEM lane quarter this warp may access
    const int lane = tid & 31;
    const int64_t L = p.L;
    const int H = p.H, HP = H * P;
    const int nc = (int)((L + Q - 1) / Q);
    const int meetk = CL ? (DIR == 0 ? nc / 2 : nc - nc / 2) : (DIR == 0 ? nc : 0);  // chunks before the meeting
    float* own_y = DIR == 0 ? p.YF : p.YB;
    const float* partner_y = DIR == 0 ? p.YB : p.YF;
    const unsigned char* tileb = p.tiles + ((int64_t)DIR * p.batch + b) * nc * (2 * kTileBytes);
    const int CH = p.CH;
    const Tin* Xr = static_cast<const Tin*>(p.xbc[DIR]) + (int64_t)b * L * CH + (int64_t)h * P;
    const Tin* DTr = static_cast<const Tin*>(p.dt[DIR]) + (int64_t)b * L * H + h;
    const float bias = p.dt_bias[DIR * H + h];
    const float A2 = p.A[DIR * H + h] * kLog2e;
    const float Dsk = p.Dskip[DIR * H + h];
    const float scale = p.dir_scale[DIR];

    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(bars + i, 1);
        fence_barrier_init();
    }
    if (tid < 32) tmem_alloc<256>(tmem_slot);
    for (int e = tid; e < 8192 / 16; e += kSsdThreads) reinterpret_cast<uint4*>(sS)[e] = make_uint4(0u, 0u, 0u, 0u);
    if (tid < P) {
        const int64_t ch = (int64_t)DIR * CH + (int64_t)h * P + tid;
        const float4 w = reinterpret_cast<const float4*>(p.conv_w)[ch];
        sCW[tid] = w.x;
        sCW[32 + tid] = w.y;
        sCW[64 + tid] = w.z;
        sCW[96 + tid] = w.w;
        sCB[tid] = p.conv_b ? p.conv_b[ch] : 0.f;
    }
    if (tid < 3 * 4)  // the first chunk's halo: zeros (before token 0 forward, past token L-1 in reverse)
        reinterpret_cast<uint4*>(sX + (tid >> 2) * kSsdXStride)[tid & 3] = make_uint4(0u, 0u, 0u, 0u);
    fence_async_smem();
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lb = (uint32_t)(warp * 32) << 16;
    const uint32_t ch16 = (uint32_t)(16 * hf);  // this thread's 16 columns of a 32-column block
    {
        float zero[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) zero[i] = 0.f;
        tmem_st16(tmem + 192 + ch16 + lb, zero);  // state row n = t starts at 0
    }
    static_assert(!PREFIX || (DIR == 0 && !CL), "the prefix state is the forward's");
    if (tid == 0 && !p.starve) {
        mbar_arrive_expect_tx(bars + 0, kTileBytes);
        bulk_g2s(sB, tileb + kTileBytes, kTileBytes, bars + 0);
        if constexpr (!PREFIX) {
            mbar_arrive_expect_tx(bars + 1, kTileBytes);
            bulk_g2s(sC, tileb, kTileBytes, bars + 1);
        }
    }
    // step t of chunk kk: this half's 16 xBC channels of the head into row 3 + t of sX (zeros past
    // either end) and dt into a register, used one chunk later
    float dt_next = 0.f;
    bool ok_next = false;
    auto fetch_step = [&](int kk) {
        const int64_t tk = DIR == 0 ? (int64_t)kk * Q + t : (int64_t)(nc - kk) * Q - 1 - t;
        const bool ok = tk >= 0 && tk < L;
        const Tin* src = Xr + (ok ? tk : 0) * CH;
#pragma unroll
        for (int ii = 0; ii < 2; ++ii) {
            const int i = 2 * hf + ii;
            cp_async<16>(sX + (3 + t) * kSsdXStride + 8 * i, src + 8 * i, ok);
        }
        cp_async_commit();
        dt_next = ok ? ldf(DTr, tk * H) : 0.f;
        ok_next = ok;
    };
    fetch_step(0);
    const uint32_t aC = smem_addr(sC), aB = smem_addr(sB), aDX = smem_addr(sDX), aW = smem_addr(sW);
    // [G | Y2] = C [B ; S_]^T: the B tile and the state's fp16 copy right after it form one
    // MN-major operand of 160 rows (f16_mn_kfast layout, 8-MN groups 2048 bytes apart)
    constexpr uint32_t ID_GY = umma_idesc_f16(128, 160, false, true);
    constexpr uint32_t ID_Y = umma_idesc_f16(128, 32, false, true);
    // S^T += B^T W: the same B tile read K-major (rows = states n, K = steps s)
    constexpr uint32_t ID_S = umma_idesc_f16(128, 32, false, true);
    // The operands' descriptors at K step 0 (C and M K-major; B K-major for G and MN-major for
    // the state update; the state, delta x and W MN-major), formed where the MMAs are issued:
    // each chain of eight MMAs advances them.

#pragma unroll 1
    for (int k = 0; k < nc; ++k) {
        const uint32_t ph = (uint32_t)(k & 1);
        const bool gated = CL ? k >= meetk : DIR == 1;
        if (CL && k == meetk) cluster_meet();
        // ---- step t of chunk k: x (this half's 16 channels) and delta
        float x[16];
        uint32_t sraw[16];
        tmem_ld16_async(tmem + 192 + ch16 + lb, sraw);  // carried state row n = t; waited for after the scan
        const float dtk = dt_next;
        const bool okk = ok_next;
        // the next chunk's tiles into L2 a chunk ahead of their copies into shared memory
        if (tid == 0 && k + 1 < nc && !p.starve) {
            if constexpr (PREFIX)
                prefetch_l2(tileb + (int64_t)(k + 1) * 2 * kTileBytes + kTileBytes, kTileBytes);
            else
                prefetch_l2(tileb + (int64_t)(k + 1) * 2 * kTileBytes, 2 * kTileBytes);
        }
        cp_async_wait_all();
        // every xBC row of the chunk is in shared memory, and the previous chunk's epilogue is
        // done with the staging block and with its TMEM reads
        tmem_fence_before_sync();
        __syncthreads();
        tmem_fence_after_sync();
        // conv + SiLU of step t: rows t..t+3 hold steps t-3..t, and tap j multiplies step t-3+j in
        // both directions (the reverse scan's steps run backwards in time)
#pragma unroll
        for (int ii = 0; ii < 2; ++ii) {  // channels 8i .. 8i+7, in pairs
            const int i = 2 * hf + ii;
            float2 acc[4];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const float4 cb = reinterpret_cast<const float4*>(sCB)[2 * i + q];
                acc[2 * q] = make_float2(cb.x, cb.y);
                acc[2 * q + 1] = make_float2(cb.z, cb.w);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 rw = *reinterpret_cast<const uint4*>(sX + (t + j) * kSsdXStride + 8 * i);
                const uint32_t wd[4] = {rw.x, rw.y, rw.z, rw.w};
                const float4 w0 = reinterpret_cast<const float4*>(sCW + 32 * j)[2 * i];
                const float4 w1 = reinterpret_cast<const float4*>(sCW + 32 * j)[2 * i + 1];
                const float2 wp[4] = {make_float2(w0.x, w0.y), make_float2(w0.z, w0.w), make_float2(w1.x, w1.y),
                                      make_float2(w1.z, w1.w)};
#pragma unroll
                for (int u = 0; u < 4; ++u)  // bf16 -> fp32 is exact: the bf16 bits are the high half
                    acc[u] = fma2(wp[u], make_float2(__uint_as_float(wd[u] << 16), __uint_as_float(wd[u] & 0xffff0000u)),
                                  acc[u]);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                x[8 * ii + 2 * u] = silu(acc[u].x);
                x[8 * ii + 2 * u + 1] = silu(acc[u].y);
            }
        }
        const float dl = okk ? softplus(dtk + bias) : 0.f;
        // ---- c_t: inclusive scan of delta A (log2 units) over the chunk (both halves alike)
        float a = dl * A2;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, a, off);
            if (lane >= off) a += v;
        }
        if (lane == 31 && hf == 0) wtot[warp] = a;
        __syncthreads();
        if (t >= Q - 3) {  // the conv has read every row: the last three steps become the next halo
#pragma unroll
            for (int ii = 0; ii < 2; ++ii) {
                const int i = 2 * hf + ii;
                reinterpret_cast<uint4*>(sX + (t + 3 - Q) * kSsdXStride)[i] =
                    reinterpret_cast<const uint4*>(sX + (t + 3) * kSsdXStride)[i];
            }
        }
        // ---- G = C B^T and Y2 = C S_^T need only the tiles and the state of the previous
        // chunk: they run on the tensor cores while the steps below are computed
        if (!PREFIX && tid == 0) {
            mbar_wait_bounded(bars + 0, ph, p.wait_limit);
            mbar_wait_bounded(bars + 1, ph, p.wait_limit);
            tmem_fence_after_sync();
            umma_f16_k8<256 / 16, 256 / 16>(tmem + 0, umma_desc(aC, 128, 2048), umma_desc(aB, 128, 2048), ID_GY,
                                            false);
            umma_commit(bars + 2);
        }
        float base = 0.f;
        for (int w = 0; w < warp; ++w) base += wtot[w];
        const float c = a + base;
        const float cend = wtot[0] + wtot[1] + wtot[2] + wtot[3];
        {
            // block j = warp: step s's factor 2^(c_{32j} - c_s) >= 1, usable while the span is small
            const float cref = __shfl_sync(0xffffffffu, c, 0);
            const float span = cref - __shfl_sync(0xffffffffu, c, 31);
            if (!PREFIX && hf == 0) {
                c2s[t] = c;
                sE[t] = ex2_approx(fminf(cref - c, kSsdSpanMax));
                if (lane == 0) bigspan[warp] = span > kSsdSpanMax ? 1 : 0;
            }
        }
        // ---- delta x and W rows of step t (MN-major [s][p]), this half's channels
        {
            const float wdec = ex2_approx(cend - c);
            float dx[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) dx[i] = dl * x[i];
            if constexpr (!PREFIX) {
#pragma unroll
                for (int pg = 0; pg < 2; ++pg) st_half8(sDX + f16_mnmajor(16 * hf + 8 * pg, t, P), dx + 8 * pg);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) dx[i] *= wdec;
#pragma unroll
            for (int pg = 0; pg < 2; ++pg) st_half8(sW + f16_mnmajor(16 * hf + 8 * pg, t, P), dx + 8 * pg);
        }
        if (k + 1 < nc) fetch_step(k + 1);  // the conv and the halo copy are done with this chunk's rows
        // a gated chunk's partner y and z, in flight while the products run, in the row-contiguous mapping
        // of the output stores: row 32 warp + 4 i + lane / 8 (i = 4 hf .. 4 hf + 3), channels
        // 4 (lane % 8) .. + 3
        float4 yfc[4];
        uint2 zc[4];
        if (gated) {
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
                const int r = 32 * warp + 4 * (4 * hf + ii) + (lane >> 3);
                const int64_t tk = DIR == 0 ? (int64_t)k * Q + r : (int64_t)(nc - k) * Q - 1 - r;
                yfc[ii] = make_float4(0.f, 0.f, 0.f, 0.f);
                zc[ii] = make_uint2(0u, 0u);
                if (tk >= 0 && tk < L) {
                    const int64_t o = ((int64_t)b * L + tk) * HP + (int64_t)h * P + 4 * (lane & 7);
                    yfc[ii] = *reinterpret_cast<const float4*>(partner_y + o);
                    zc[ii] = *reinterpret_cast<const uint2*>(static_cast<const Tin*>(p.z) + o);
                }
            }
        }
        // ---- carried state row n = t (this half's columns) decays over the whole chunk
        {
            tmem_wait_ld(sraw);
            float s[16];
            const float f = ex2_approx(cend);
#pragma unroll
            for (int i = 0; i < 16; ++i) s[i] = __uint_as_float(sraw[i]) * f;
            tmem_st16(tmem + 192 + ch16 + lb, s);
        }
        fence_async_smem();
        tmem_fence_before_sync();
        __syncthreads();
        tmem_fence_after_sync();
        // ---- S^T += B^T W (onto the decayed state)
        if (tid == 0) {
            if constexpr (PREFIX) {
                mbar_wait_bounded(bars + 0, ph, p.wait_limit);
                tmem_fence_after_sync();
            }
            umma_f16_k8<4096 / 16, 1024 / 16>(tmem + 192, umma_desc(aB, 2048, 128), umma_desc(aW, 512, 128), ID_S,
                                              true);
            umma_commit(bars + 4);
        }
        if constexpr (PREFIX) {  // the state is all a prefix needs
            mbar_wait_bounded(bars + 4, ph, p.wait_limit);
            tmem_fence_after_sync();
            if (tid == 0 && k + 1 < nc && !p.starve) {  // B's buffer is free: next chunk's B tile
                mbar_arrive_expect_tx(bars + 0, kTileBytes);
                bulk_g2s(sB, tileb + (int64_t)(k + 1) * 2 * kTileBytes + kTileBytes, kTileBytes, bars + 0);
            }
            continue;
        }
        mbar_wait_bounded(bars + 2, ph, p.wait_limit);
        tmem_fence_after_sync();
        // ---- M row t (into C's buffer, K-major [t][s]): this half's column blocks jb = hf, hf + 2.
        // Columns s >= 32 jb reach step t = 32 warp + lane only for jb <= warp;
        // e^(c_t - c_s) = 2^(c_t - c_{32jb}) 2^(c_{32jb} - c_s) while block jb's span is small
#pragma unroll 1
        for (int jj = 0; jj < 2; ++jj) {
            const int jb = hf + 2 * jj;
            uint32_t gr[32];
            if (jb <= warp) tmem_ld32_async(tmem + 32 * jb + lb, gr);
            tmem_wait_ld(gr);
            float m[32];
            if (jb <= warp) {
                const float cref = c2s[32 * jb];
                if (!bigspan[jb]) {
                    const float F = ex2_approx(c - cref);
                    const float2 FF = make_float2(F, F);
                    const float4* e4 = reinterpret_cast<const float4*>(sE + 32 * jb);
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float4 ev = e4[i / 4];
                        const float2 m01 = mul2(make_float2(__uint_as_float(gr[i]), __uint_as_float(gr[i + 1])),
                                                mul2(FF, make_float2(ev.x, ev.y)));
                        const float2 m23 = mul2(make_float2(__uint_as_float(gr[i + 2]), __uint_as_float(gr[i + 3])),
                                                mul2(FF, make_float2(ev.z, ev.w)));
                        m[i] = m01.x; m[i + 1] = m01.y; m[i + 2] = m23.x; m[i + 3] = m23.y;
                    }
                    if (jb == warp) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i > lane) m[i] = 0.f;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int s = 32 * jb + i;
                        m[i] = s <= t ? __uint_as_float(gr[i]) * ex2_approx(c - c2s[s]) : 0.f;
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) m[i] = 0.f;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) st_half8(sC + f16_kmajor(t, 32 * jb + 8 * q, Q), m + 8 * q);
        }
        // ---- the new state row n = t (this half's columns) as the fp16 operand of the next C S_^T
        mbar_wait_bounded(bars + 4, ph, p.wait_limit);
        tmem_fence_after_sync();
        if (tid == 0 && k + 1 < nc && !p.starve) {  // B's buffer is free: next chunk's B tile
            mbar_arrive_expect_tx(bars + 0, kTileBytes);
            bulk_g2s(sB, tileb + (int64_t)(k + 1) * 2 * kTileBytes + kTileBytes, kTileBytes, bars + 0);
        }
        {
            uint32_t sn[16];
            tmem_ld16_async(tmem + 192 + ch16 + lb, sn);
            tmem_wait_ld(sn);
            float sv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) sv[i] = __uint_as_float(sn[i]);
#pragma unroll
            for (int pg = 0; pg < 2; ++pg) st_half8(sS + f16_mn_kfast(16 * hf + 8 * pg, t, kM2N), sv + 8 * pg);
        }
        fence_async_smem();
        tmem_fence_before_sync();
        __syncthreads();
        tmem_fence_after_sync();
        // ---- Y1 = M (delta x)
        if (tid == 0) {
            umma_f16_k8<256 / 16, 1024 / 16>(tmem + 160, umma_desc(aC, 128, 2048), umma_desc(aDX, 512, 128), ID_Y,
                                             false);
            umma_commit(bars + 3);
        }
        mbar_wait_bounded(bars + 3, ph, p.wait_limit);
        tmem_fence_after_sync();
        if (tid == 0 && k + 1 < nc && !p.starve) {  // C's buffer is free: next chunk's C tile
            mbar_arrive_expect_tx(bars + 1, kTileBytes);
            bulk_g2s(sC, tileb + (int64_t)(k + 1) * 2 * kTileBytes, kTileBytes, bars + 1);
        }
        // ---- output of step t: the two halves of each row go through the row block's 32-row
        // staging block (the delta x / W buffers, free once Y1 is done; 16-byte chunks
        // XOR-swizzled by row) and are stored row-contiguously, four whole 128-byte rows per warp
        // instruction
        {
            uint32_t r1[16], r2[16];
            tmem_ld16_async(tmem + 160 + ch16 + lb, r1);
            tmem_ld16_async(tmem + 128 + ch16 + lb, r2);
            tmem_wait_ld(r1);
            tmem_wait_ld(r2);
            const float e = ex2_approx(c);
            float4* stg = reinterpret_cast<float4*>(sDX) + warp * 256;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float4 v;
                v.x = (__uint_as_float(r1[4 * q]) + e * __uint_as_float(r2[4 * q]) + Dsk * x[4 * q]) * scale;
                v.y = (__uint_as_float(r1[4 * q + 1]) + e * __uint_as_float(r2[4 * q + 1]) + Dsk * x[4 * q + 1]) * scale;
                v.z = (__uint_as_float(r1[4 * q + 2]) + e * __uint_as_float(r2[4 * q + 2]) + Dsk * x[4 * q + 2]) * scale;
                v.w = (__uint_as_float(r1[4 * q + 3]) + e * __uint_as_float(r2[4 * q + 3]) + Dsk * x[4 * q + 3]) * scale;
                stg[lane * 8 + ((4 * hf + q) ^ (lane & 7))] = v;
            }
            named_bar_sync(1 + warp, 64);  // the row block's two warps (warp, warp + 4) wrote its staging block
            const int cq = lane & 7;
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
                const int r = 4 * (4 * hf + ii) + (lane >> 3);
                const float4 v = stg[r * 8 + (cq ^ (r & 7))];
                const int step = 32 * warp + r;
                const int64_t tk = DIR == 0 ? (int64_t)k * Q + step : (int64_t)(nc - k) * Q - 1 - step;
                if (tk >= 0 && tk < L) {
                    const int64_t o = ((int64_t)b * L + tk) * HP + (int64_t)h * P + 4 * cq;
                    if (!gated) {
                        *reinterpret_cast<float4*>(own_y + o) = v;
                    } else {
                        // bf16 -> fp32 is exact: the bf16 bits are the high half
                        const float z0 = __uint_as_float(zc[ii].x << 16), z1 = __uint_as_float(zc[ii].x & 0xffff0000u);
                        const float z2 = __uint_as_float(zc[ii].y << 16), z3 = __uint_as_float(zc[ii].y & 0xffff0000u);
                        float ov[4];
                        ov[0] = (yfc[ii].x + v.x) * silu(z0);
                        ov[1] = (yfc[ii].y + v.y) * silu(z1);
                        ov[2] = (yfc[ii].z + v.z) * silu(z2);
                        ov[3] = (yfc[ii].w + v.w) * silu(z3);
                        store4(static_cast<Tout*>(p.out) + o, ov);
                    }
                }
            }
        }
    }
    if (CL && meetk >= nc) cluster_meet();  // a one-chunk sequence: the reverse CTA meets after its chunk
    if constexpr (PREFIX) {  // the final state: row n = t, this half's channels p
        uint32_t sn[16];
        tmem_ld16_async(tmem + 192 + ch16 + lb, sn);
        tmem_wait_ld(sn);
        float* so = p.S_out + ((int64_t)b * H + h) * P * kM2N + t;
#pragma unroll
        for (int i = 0; i < 16; ++i) so[(int64_t)(16 * hf + i) * kM2N] = __uint_as_float(sn[i]);
    }
    tmem_fence_before_sync();
    __syncthreads();
    if (tid < 32) tmem_dealloc<256>(tmem);
}

// The forward prefix state of block-cached decoding on the tensor cores
// (bf16 inputs): grid (H, batch), block kSsdThreads, dynamic shared memory
// kSsdSmem; the B tiles from m2_prep_kernel<bf16, true>.
__global__ void __launch_bounds__(kSsdThreads, 2) m2_ssd_prefix_kernel(const M2Params p) {
    extern __shared__ __align__(128) unsigned char sm[];
    m2_ssd_dir<0, __nv_bfloat16, float, false, true>(p, sm, (int)blockIdx.x, (int)blockIdx.y);
}

// grid (2 H, batch) in clusters of 2: CTA 2h runs head h forward, CTA 2h+1 in
// reverse; block 128, dynamic shared memory kSsdSmem.  For calls whose
// per-direction grid leaves SMs idle: both directions run at once.
template <typename Tin, typename Tout>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kSsdThreads, 2) m2_ssd_cluster_kernel(const M2Params p) {
    extern __shared__ __align__(128) unsigned char sm[];
    if (blockIdx.x & 1)
        m2_ssd_dir<1, Tin, Tout, true>(p, sm, (int)(blockIdx.x >> 1), (int)blockIdx.y);
    else
        m2_ssd_dir<0, Tin, Tout, true>(p, sm, (int)(blockIdx.x >> 1), (int)blockIdx.y);
}

// Both directions as separate CTAs of one launch, for calls whose
// per-direction grid fills the GPU: grid (2 H batch), block 128, dynamic
// shared memory kSsdSmem.  Each CTA takes a ticket from p.sync[0] when it
// starts; tickets [0, H batch) run the forward of (h, b) = (ticket mod H,
// ticket / H) and store its y for every chunk, the rest the reverse of the
// same pairs in the same order, which gates with that y.  A reverse CTA
// waits for its forward's flag before its first chunk.  The forward CTA holds
// a smaller ticket, so it has started by then and only waits on its own
// copies and products: the wait always ends.  It is still bounded (p.meet_limit,
// ~2 s; on timeout bit 1 of the device error word is set and the CTA carries
// on).
// Compared with a forward launch followed by a reverse launch, the reverse
// CTAs fill the SMs the forward's last partial wave leaves idle.
constexpr unsigned kErrPartnerTimeout = 2u;

__device__ __forceinline__ void m2_flag_release(int* f) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(f), "r"(1) : "memory");
}
__device__ __forceinline__ int m2_flag_acquire(const int* f) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    return v;
}

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kSsdThreads, 2) m2_ssd_ticket_kernel(const M2Params p) {
    extern __shared__ __align__(128) unsigned char sm[];
    __shared__ int ticket;
    if (threadIdx.x == 0) ticket = atomicAdd(p.sync, 1);
    __syncthreads();
    const int n1 = p.H * p.batch;
    const int tk = ticket;
    if (tk < n1) {
        m2_ssd_dir<0, Tin, Tout, false>(p, sm, tk % p.H, tk / p.H);
        // every thread's y stores are visible device-wide before the flag
        __threadfence();
        __syncthreads();
        // (under the starving test aid the flag is never set, so that the
        // reverse's bounded wait is exercised too)
        if (threadIdx.x == 0 && !p.starve) m2_flag_release(p.sync + 1 + tk);
    } else {
        const int x = tk - n1;
        if (threadIdx.x == 0) {
            const int* f = p.sync + 1 + x;
            if (!m2_flag_acquire(f)) {
                const long long t0 = clock64();
                while (!m2_flag_acquire(f)) {
                    if (clock64() - t0 > p.meet_limit) {
                        atomicOr(&g_device_error, kErrPartnerTimeout);
                        break;
                    }
                    __nanosleep(256);
                }
            }
        }
        __syncthreads();
        m2_ssd_dir<1, Tin, Tout, false>(p, sm, x % p.H, x / p.H);
    }
}

}  // namespace bimamba

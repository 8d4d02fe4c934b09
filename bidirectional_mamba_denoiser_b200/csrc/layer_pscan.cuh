// layer_pscan.cuh -- the bidirectional Mamba mixer layer as a chunked scan
// whose carries are combined with warp shuffles ("DiffuMamba:
// High-Throughput Diffusion LMs with Mamba Backbone", §3.2 Eq. (4)-(6)),
// for few channels (batch 1 over a long sequence).
//
// Each step of a channel's recurrence is an affine map of its 16-state
// vector: h -> a_t * h + b_t with a_t = exp(delta_t A) and
// b_t = delta_t u_t B_t (per state, elementwise).  Maps compose
// associatively: (P1, h1) then (P2, h2) is (P2 P1, P2 h1 + h2).  So a
// chunk of steps can be cut into pieces scanned side by side, the pieces'
// maps combined by a prefix scan, and every step's true state rebuilt from
// its piece-local state: h_t = P_t * s_in + hloc_t, where P_t and hloc_t are
// the product and the state of the piece's steps up to t taken from zero,
// and s_in the state entering the piece.  Every exp is computed once.
//
// Layout: a CTA is NWD forward and NWD reverse warps over the same
// CW = 4 NWD channels.  A warp covers 4 channels; the 8 lanes of a channel
// (lane = 8c + pc) take the 8 pieces of 8 steps of a chunk of T = 64 steps.
// Both directions cut the sequence into the same 64-token chunks and walk
// them in step space (step s of chunk k is token 64k + s forward, 64k + 63-s
// in reverse), so the reverse conv is the causal conv over tokens read
// backwards; nothing is flipped in memory.  Per chunk:
//  1. its x (+3-token conv halo), dt, B, C (and z when gated) arrive by TMA
//     into an NS-stage ring per direction (boxes outside [0, L) read zeros:
//     the conv padding); the direction's warps widen B and C to fp32 once,
//     state pairs interleaved and rows in step order, so a lane reads its
//     piece's 8 B (or C) pairs with four 16-byte loads (pieces padded apart
//     so that a channel's 8 lanes read distinct banks);
//  2. each lane computes conv + SiLU, the step size and D*u of its 8 steps
//     (a sliding conv window over 11 x rows) into registers;
//  3. for each of the 8 state pairs (packed f32x2 arithmetic, one MUFU exp2
//     per state and step): the piece-local scan from zero; an inclusive scan
//     of the 8 pieces' (P, hloc) in 3 shuffle rounds within the channel's 8
//     lanes, shifted to exclusive; the state entering the piece from the
//     chunk's carry (kept per channel in shared memory); the states of the
//     8 steps and their C.h into the outputs; lane 7 stores the new carry;
//  4. y = sum of the pairs + D*u, stored (first half of the walk, fp32, for
//     the other direction) or added to the other direction's y and gated by
//     SiLU(z) (second half).
// Steps whose token is >= L get delta = 0 and no drive: a = 1, b = 0, the
// identity map, so ragged chunks need no branches in the scan.  The two
// directions meet halfway at one CTA barrier, as in the other layer kernels.
#pragma once

#include "layer_tma.cuh"
#include "scan_kernels.cuh"
#include "tma_util.cuh"

namespace bimamba {

template <int NWD, int NS, typename Tin>
struct PscanGeo {
    static constexpr int T = 64;     // steps per chunk
    static constexpr int PL = 8;     // steps per piece (lane)
    static constexpr int CPW = 4;    // channels per warp
    static constexpr int CW = NWD * CPW;  // channels per CTA
    static constexpr int ESZ = (int)sizeof(Tin);
    // x/dt/z tile rows: CW channels, widened to the aligned 16 bytes around them if fewer
    static constexpr int XW = CW * ESZ >= 16 ? CW : 16 / ESZ;
    static constexpr int XB = align128((T + 3) * XW * ESZ);
    static constexpr int DTB = align128(T * XW * ESZ);
    static constexpr int BB = align128(T * kNState * ESZ);
    static constexpr int STAGE = XB + 2 * DTB + 2 * BB;   // x, dt, z, B, C
    // fp32 B then C: [pair 8][piece 8][step 8][2], pieces padded to PS floats and
    // pairs to QS, so that the 8 pieces of a channel read distinct banks
    static constexpr int PS = 2 * PL + 4;
    static constexpr int QS = 8 * PS + 4;
    static constexpr int BCS = 8 * QS;                    // floats of B (or C)
    static constexpr int BCF = 2 * BCS * 4;
    static constexpr int AS = kNState + 2;                // floats per channel row of A and of the carry
    static constexpr int A2B = CW * AS * 4;               // A * log2(e) of the CTA's channels
    static constexpr int CRB = CW * AS * 4;               // carried state of the CTA's channels
    static constexpr int OWS = T * CPW * 4;               // per warp: partner's y of a chunk
    static constexpr int DIR_BYTES = NS * STAGE + BCF + A2B + CRB + NWD * OWS;
    static constexpr int BAR_OFF = 2 * DIR_BYTES;
    static constexpr int SMEM = BAR_OFF + 2 * NS * 8 + 128;  // + alignment slack
    static constexpr uint32_t TX_BASE = (uint32_t)(((T + 3) * XW + T * XW + 2 * T * kNState) * ESZ);
    static constexpr uint32_t TX_Z = (uint32_t)(T * XW * ESZ);
    static_assert(NWD == 1 || NWD == 2, "warps per direction");
    static_assert((XW * ESZ) % 16 == 0 && XW % CW == 0, "TMA box rows must be whole 16-byte units");
};

template <int NWD, int NS, typename Tin>
__device__ __forceinline__ void pscan_issue(const LayerMaps& maps, unsigned char* dir_base, uint64_t* full, int r,
                                            int i, int k, bool gated, int ct0, int b, int starve) {
    using Ge = PscanGeo<NWD, NS, Tin>;
    if (starve) return;
    const int st = i % NS;
    unsigned char* sb = dir_base + st * Ge::STAGE;
    uint64_t* bar = full + st;
    mbar_arrive_expect_tx(bar, Ge::TX_BASE + (gated ? Ge::TX_Z : 0u));
    const int row0 = k * Ge::T;
    const int x0 = ct0 - ct0 % Ge::XW;  // the aligned tile row around the CTA's channels
    tma_load_3d(sb, &maps.x, bar, x0, r == 0 ? row0 - 3 : row0, b);
    tma_load_3d(sb + Ge::XB, &maps.dt[r], bar, x0, row0, b);
    if (gated) tma_load_3d(sb + Ge::XB + Ge::DTB, &maps.z, bar, x0, row0, b);
    tma_load_3d(sb + Ge::XB + 2 * Ge::DTB, &maps.B[r], bar, 0, row0, b);
    tma_load_3d(sb + Ge::XB + 2 * Ge::DTB + Ge::BB, &maps.C[r], bar, 0, row0, b);
}

// B and C of the chunk's T rows -> fp32 pairs in step order (the layout
// above), by the direction's NWD warps; consecutive threads take consecutive
// pairs of a row.
template <int NWD, int NS, typename Tin, int DIR>
__device__ __forceinline__ void pscan_widen_bc(const Tin* Bt, const Tin* Ct, float* bcf, int tid) {
    using Ge = PscanGeo<NWD, NS, Tin>;
    constexpr int T = Ge::T;
    for (int e = tid; e < 2 * T * 8; e += NWD * 32) {
        const int which = e / (T * 8);  // 0 = B, 1 = C
        const int row = (e / 8) % T, q = e % 8;
        const Tin* src = (which ? Ct : Bt) + row * kNState + 2 * q;
        const int step = DIR == 0 ? row : T - 1 - row;
        const int pc = step / Ge::PL, j = step % Ge::PL;
        *reinterpret_cast<float2*>(bcf + which * Ge::BCS + q * Ge::QS + pc * Ge::PS + 2 * j) =
            make_float2(ldf(src, 0), ldf(src, 1));
    }
}

// CARRY: start from p.carry_in, report p.carry_out and p.delta_sum (each where non-null).
template <int NWD, int NS, typename Tin, typename Tout, int DIR, bool CARRY>
__device__ __forceinline__ void pscan_direction(const LayerMaps& maps, const KParams& p, unsigned char* base,
                                                int wg, int lane) {
    using Ge = PscanGeo<NWD, NS, Tin>;
    constexpr int T = Ge::T, PL = Ge::PL;
    unsigned char* dir_base = base + DIR * Ge::DIR_BYTES;
    float* bcf = reinterpret_cast<float*>(dir_base + NS * Ge::STAGE);
    float* a2s = reinterpret_cast<float*>(dir_base + NS * Ge::STAGE + Ge::BCF);
    float* crs = reinterpret_cast<float*>(dir_base + NS * Ge::STAGE + Ge::BCF + Ge::A2B);
    float* ows = reinterpret_cast<float*>(dir_base + NS * Ge::STAGE + Ge::BCF + Ge::A2B + Ge::CRB + wg * Ge::OWS);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + Ge::BAR_OFF) + DIR * NS;
    const int b = blockIdx.y;
    const int ct0 = blockIdx.x * Ge::CW;
    const int64_t L = p.L;
    const int D = p.D;
    const int nc = (int)((L + T - 1) / T);
    const int meet = DIR == 0 ? nc / 2 : nc - nc / 2;  // chunks before the meeting point
    const bool leader = (wg == 0 && lane == 0);
    const float scale = p.dir_scale[DIR];
    const int tid = wg * 32 + lane;
    const int c = lane >> 3, pc = lane & 7;      // channel in the warp, piece
    const int cc = wg * Ge::CPW + c;             // channel in the CTA
    const int d = ct0 + cc;
    const int tc = ct0 % Ge::XW + cc;            // column in the x/dt/z tiles
    const bool dvalid = d < D;
    const int c0w = ct0 + wg * Ge::CPW;          // first channel of this warp

    // per-channel parameters; A * log2(e) and the carried state in shared memory
    const int64_t rd = (int64_t)DIR * D + (dvalid ? d : 0);
    float w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = dvalid ? p.conv_w[rd * 4 + k] : 0.f;
    const float cb = (dvalid && p.conv_b) ? p.conv_b[rd] : 0.f;
    const float bias = dvalid ? p.dt_bias[rd] : 0.f;
    const float Dd = dvalid ? p.Dskip[rd] : 0.f;
    for (int e = tid; e < Ge::CW * kNState; e += NWD * 32) {
        const int ch = ct0 + e / kNState, n = e % kNState;
        const bool ok = ch < D;
        const int o = (e / kNState) * Ge::AS + n;
        a2s[o] = ok ? p.A[((int64_t)DIR * D + ch) * kNState + n] * kLog2e : 0.f;
        crs[o] = (CARRY && ok && p.carry_in[DIR]) ? p.carry_in[DIR][((int64_t)b * D + ch) * kNState + n] : 0.f;
    }
    float dsum = 0.f;  // step sizes of this lane's valid steps (carries)

    if (leader)
        for (int i = 0; i < NS && i < nc; ++i)
            pscan_issue<NWD, NS, Tin>(maps, dir_base, full, DIR, i, DIR == 0 ? i : nc - 1 - i, i >= meet, ct0, b,
                                      p.starve);

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

        // partner's y of this chunk -> shared memory (16-byte pieces of the
        // warp's 4 channels; d_inner is a multiple of 4 here)
        if (gated) {
            for (int e = lane; e < T; e += 32) {
                const bool ok = (int64_t)k * T + e < L && c0w < D;
                const float* src = p.ws + (chunk_row + (ok ? e : 0)) * D + (ok ? c0w : 0);
                cp_async<16>(ows + e * Ge::CPW, src, ok);
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
        if (CARRY && i == 0 && p.conv_halo[DIR])  // forward: tile rows 0..2 = tokens -3..-1; reverse: rows of L..L+2
            put_conv_halo(reinterpret_cast<Tin*>(dir_base + st * Ge::STAGE), Ge::XW,
                          DIR == 0 ? 0 : (int)(L - (int64_t)k * T), ct0 % Ge::XW + wg * Ge::CPW, c0w, Ge::CPW,
                          static_cast<const Tin*>(p.conv_halo[DIR]) + (int64_t)b * 3 * D, D, lane);

        // 1. B and C as fp32 pairs in step order (the previous chunk's are
        // no longer read: every warp of the direction is past its scan)
        pscan_widen_bc<NWD, NS, Tin, DIR>(Bt, Ct, bcf, tid);

        // 2. per-step work of my 8 steps: step s-3+j is x-tile row s+j (forward:
        // the tile starts 3 tokens early) or T+2-s-j (reverse)
        float dl[PL], du[PL], Du[PL];
        {
            const int s0 = PL * pc;
            auto xrow = [&](int s) { return DIR == 0 ? s + 3 : T - 1 - s; };
            float x0 = ldf(xt, xrow(s0 - 3) * Ge::XW + tc);
            float x1 = ldf(xt, xrow(s0 - 2) * Ge::XW + tc);
            float x2 = ldf(xt, xrow(s0 - 1) * Ge::XW + tc);
#pragma unroll
            for (int j = 0; j < PL; ++j) {
                const int s = s0 + j;
                const float x3 = ldf(xt, xrow(s) * Ge::XW + tc);
                float cv = fmaf(w[0], x0, cb);
                cv = fmaf(w[1], x1, cv);
                cv = fmaf(w[2], x2, cv);
                cv = fmaf(w[3], x3, cv);
                x0 = x1; x1 = x2; x2 = x3;
                const float u = silu(cv);
                const float dlt = softplus(ldf(dtt, (DIR == 0 ? s : T - 1 - s) * Ge::XW + tc) + bias);
                const bool valid = s >= s_lo && s < s_hi;
                dl[j] = valid ? dlt : 0.f;
                du[j] = valid ? dlt * u : 0.f;
                Du[j] = valid ? Dd * u : 0.f;
                if constexpr (CARRY) dsum += dl[j];
            }
        }
        if (gated) cp_async_wait_all();
        if constexpr (NWD == 1)
            __syncwarp();
        else
            named_bar_sync(1 + DIR, NWD * 32);  // the fp32 B/C rows are written

        // the previous chunk's stage is free (every warp of the direction is past it): refill it
        if (leader && i >= 1 && i - 1 + NS < nc) {
            const int i2 = i - 1 + NS;
            pscan_issue<NWD, NS, Tin>(maps, dir_base, full, DIR, i2, DIR == 0 ? i2 : nc - 1 - i2, i2 >= meet, ct0,
                                      b, p.starve);
        }

        // 3. the 8 state pairs
        float2 y[PL];
#pragma unroll
        for (int j = 0; j < PL; ++j) y[j] = make_float2(0.f, 0.f);
        const float* bfp = bcf + pc * Ge::PS;                   // pair 0, my first step
        const float* cfp = bcf + Ge::BCS + pc * Ge::PS;
#pragma unroll 1
        for (int q = 0; q < 8; ++q) {
            const float2 a2 = *reinterpret_cast<const float2*>(a2s + cc * Ge::AS + 2 * q);
            const float2 carry = *reinterpret_cast<const float2*>(crs + cc * Ge::AS + 2 * q);
            float2 bp[PL];
#pragma unroll
            for (int j = 0; j < PL; j += 2) {
                const float4 v = *reinterpret_cast<const float4*>(bfp + q * Ge::QS + 2 * j);
                bp[j] = make_float2(v.x, v.y);
                bp[j + 1] = make_float2(v.z, v.w);
            }
            // piece-local scan from zero
            float2 hl[PL], Pl[PL];
            float2 h = make_float2(0.f, 0.f), P = make_float2(1.f, 1.f);
#pragma unroll
            for (int j = 0; j < PL; ++j) {
                const float2 v = mul2(make_float2(dl[j], dl[j]), a2);
                const float2 ea = make_float2(ex2_approx(v.x), ex2_approx(v.y));
                h = fma2(ea, h, mul2(make_float2(du[j], du[j]), bp[j]));
                P = mul2(P, ea);
                hl[j] = h;
                Pl[j] = P;
            }
            // inclusive scan of the pieces' maps over the channel's 8 lanes
            float2 Pi = P, hi = h;
#pragma unroll
            for (int off = 1; off < PL; off <<= 1) {
                const float2 Pp = make_float2(__shfl_up_sync(0xffffffffu, Pi.x, off, PL),
                                              __shfl_up_sync(0xffffffffu, Pi.y, off, PL));
                const float2 hp = make_float2(__shfl_up_sync(0xffffffffu, hi.x, off, PL),
                                              __shfl_up_sync(0xffffffffu, hi.y, off, PL));
                if (pc >= off) {  // earlier pieces' map first, then mine
                    hi = fma2(Pi, hp, hi);
                    Pi = mul2(Pi, Pp);
                }
            }
            // exclusive: the map of the pieces before mine (identity for piece 0)
            float2 Pe = make_float2(__shfl_up_sync(0xffffffffu, Pi.x, 1, PL),
                                    __shfl_up_sync(0xffffffffu, Pi.y, 1, PL));
            float2 he = make_float2(__shfl_up_sync(0xffffffffu, hi.x, 1, PL),
                                    __shfl_up_sync(0xffffffffu, hi.y, 1, PL));
            if (pc == 0) {
                Pe = make_float2(1.f, 1.f);
                he = make_float2(0.f, 0.f);
            }
            const float2 sin = fma2(Pe, carry, he);  // state entering my piece
            __syncwarp();                            // every lane has read the carry
            if (pc == PL - 1)                        // state after the chunk's last step
                *reinterpret_cast<float2*>(crs + cc * Ge::AS + 2 * q) = fma2(Pi, carry, hi);
            // the steps' states and C.h
#pragma unroll
            for (int j = 0; j < PL; j += 2) {
                const float4 cv = *reinterpret_cast<const float4*>(cfp + q * Ge::QS + 2 * j);
                y[j] = fma2(make_float2(cv.x, cv.y), fma2(Pl[j], sin, hl[j]), y[j]);
                y[j + 1] = fma2(make_float2(cv.z, cv.w), fma2(Pl[j + 1], sin, hl[j + 1]), y[j + 1]);
            }
        }

        // 4. outputs of my 8 steps
        {
            float* wsw = p.ws + chunk_row * D + d;
            Tout* outw = static_cast<Tout*>(p.out) + chunk_row * D + d;
#pragma unroll
            for (int j = 0; j < PL; ++j) {
                const int s = PL * pc + j;
                if (s >= s_lo && s < s_hi && dvalid) {
                    const int tr = DIR == 0 ? s : T - 1 - s;  // token - kT
                    const float yv = (y[j].x + y[j].y + Du[j]) * scale;
                    if (!gated) {
                        wsw[(int64_t)tr * D] = yv;
                    } else {
                        const float zv = ldf(zt, tr * Ge::XW + tc);
                        stf(outw, (int64_t)tr * D, (yv + ows[tr * Ge::CPW + c]) * silu(zv));
                    }
                }
            }
        }
        // every warp of the direction is done with this chunk's fp32 B/C rows
        // and the stage before the next chunk's widening refills them
        if constexpr (NWD == 1)
            __syncwarp();
        else
            named_bar_sync(1 + DIR, NWD * 32);
    }
    if (meet >= nc) {  // a single-chunk sequence: the reverse warps meet after their only chunk
        __threadfence_block();
        named_bar_sync(3, 2 * NWD * 32);
    }
    if (CARRY && p.carry_out[DIR]) {
        __syncwarp();
        for (int e = lane; e < Ge::CPW * kNState; e += 32) {
            const int ch = c0w + e / kNState;
            if (ch < D)
                p.carry_out[DIR][((int64_t)b * D + ch) * kNState + e % kNState] =
                    crs[(wg * Ge::CPW + e / kNState) * Ge::AS + e % kNState];
        }
    }
    if (CARRY && p.delta_sum[DIR]) {  // the 8 lanes of a channel are adjacent
        float ds = dsum;
#pragma unroll
        for (int off = 1; off < PL; off <<= 1) ds += __shfl_xor_sync(0xffffffffu, ds, off);
        if (pc == 0 && dvalid) p.delta_sum[DIR][(int64_t)b * D + d] = ds;
    }
}

// At most 128 registers: batch 1 x 4096 channels makes 512 CTAs, which
// need 4 resident per SM.
template <int NWD, int NS, typename Tin, typename Tout, bool CARRY = false>
__global__ void __launch_bounds__(2 * NWD * 32, 4) layer_pscan_kernel(const __grid_constant__ LayerMaps maps,
                                                                   const KParams p) {
    using Ge = PscanGeo<NWD, NS, Tin>;
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
        pscan_direction<NWD, NS, Tin, Tout, 0, CARRY>(maps, p, base, warp, lane);
    else
        pscan_direction<NWD, NS, Tin, Tout, 1, CARRY>(maps, p, base, warp - NWD, lane);
}

}  // namespace bimamba

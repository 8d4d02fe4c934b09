// layer_tma.cuh -- TMA-fed kernels of the bidirectional Mamba mixer layer
// ("DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone", §3.2
// Eq. (4)-(6)): the full layer and the forward prefix scan (§4.3 cache).
//
// One CTA = one batch row x CW channels.  Warps [0, NWD) run the forward
// direction and warps [NWD, 2*NWD) the reverse direction over the same
// channels; each warp covers CPW = 32/G channels with G lanes per channel,
// each lane holding S = 16/G of a channel's states.
//
// Both directions cut the sequence into the same chunks of T tokens
// (chunk k = tokens [kT, kT+T)) and walk them in "step space": step s of
// chunk k is token kT + s (forward) or kT + T-1-s (reverse), so the reverse
// conv is the causal conv over tokens read backwards; nothing is flipped in
// memory.  Each chunk's x (with the 3-token conv halo), dt, B, C -- and z
// when the chunk is gated -- arrive by 3-D TMA loads into an NS-stage
// shared-memory ring; a box reaching outside [0, L) reads zeros, which is
// the conv's zero padding at both sequence ends.  Per chunk a direction's
// warps convert B/C to fp32 once (shared by all its channels) and meet at
// one named barrier, after which the group leader refills the stage the
// previous chunk used.  Steps whose token is >= L get delta = 0 and no
// drive, so they leave the state exactly unchanged.
//
// Per chunk a warp (1) computes conv + SiLU, softplus and D*u for its
// elements into shared memory, (2) advances its states step by step with
// packed f32x2 arithmetic and one MUFU exp2 per state, and after every G
// steps combines the C.h partial sums across the G lanes (shuffle
// transpose-reduce) so that each lane owns one finished step, which it
// writes out at once.
//
// Full layer: the forward group walks chunks 0..nc-1, the reverse group
// nc-1..0.  Until they meet (the forward group after nc/2 chunks) each
// stores its fp32 y to the workspace; after one CTA barrier each finishes
// the other half, adding the partner's y (fetched by cp.async) and applying
// the SiLU(z) gate.
#pragma once

#include "scan_kernels.cuh"
#include "tma_util.cuh"

namespace bimamba {

struct LayerMaps {
    CUtensorMap x;      // [batch][L][D]      box {CW, T+3, 1}
    CUtensorMap z;      // [batch][L][D]      box {CW, T, 1}
    CUtensorMap dt[2];  // [batch][L][D]      box {CW, T, 1}
    CUtensorMap B[2];   // [batch][L][16]     box {16, T, 1}; with BCQ: fp32 quads [batch][L][32], box {32, T, 1}
    CUtensorMap C[2];   // [batch][L][16]     box {16, T, 1}; unused with BCQ
};

constexpr int align128(int v) { return (v + 127) & ~127; }

// DIRECT: B and C are read straight from the TMA tiles, so the fp32 B/C
// buffers are not allocated.  BCQ: B and C arrive already widened to fp32
// quads (widen_bc_kernel), one TMA tile per chunk in the layout of the fp32
// B/C buffer, which the states read in place.
template <int G, int T, int NWD, int NS, typename Tin, bool DIRECT = false, bool BCQ = false>
struct TmaGeo {
    static_assert(G == 4 || G == 8 || G == 16, "lanes per channel");
    static_assert(T % G == 0 && T <= 253, "chunk");
    static constexpr int CPW = 32 / G;                    // channels per warp
    static constexpr int S = kNState / G;                 // states per lane
    static constexpr int EPL = T / G;                     // elements per lane per chunk
    static constexpr int CW = NWD * CPW;                  // channels per CTA
    static constexpr int ESZ = (int)sizeof(Tin);
    // channels per x/dt/z tile row: CW, widened to the aligned 16 bytes around
    // the CTA's channels when CW of them are fewer (TMA rows are 16-byte units)
    static constexpr int XW = CW * ESZ >= 16 ? CW : 16 / ESZ;
    static constexpr int XB = align128((T + 3) * XW * ESZ);
    static constexpr int DTB = align128(T * XW * ESZ);
    static constexpr int BB = align128(T * kNState * ESZ);
    static constexpr int BC32 = T * kNState * 2 * 4;      // one fp32 B/C buffer
    static constexpr int STAGE = XB + 2 * DTB + (BCQ ? align128(BC32) : 2 * BB);  // x, dt, z, B and C
    static constexpr int ED2 = T * CPW * 8;               // per warp: (delta, delta*u)
    static constexpr int EDU = T * CPW * 4;               // per warp: D*u
    static constexpr int OWS = T * CPW * 4;               // per warp: partner's y of a chunk
    static constexpr int WARP_BYTES = ED2 + EDU + 2 * OWS;  // partner's y double-buffered
    static constexpr int DIR_BYTES = NS * STAGE + ((DIRECT || BCQ) ? 0 : 2 * BC32);
    static constexpr int WARP_OFF = 2 * DIR_BYTES;
    static constexpr int BAR_OFF = WARP_OFF + 2 * NWD * WARP_BYTES;
    static constexpr int SMEM = BAR_OFF + 2 * NS * 8 + 128;  // + alignment slack
    static constexpr uint32_t TX_BASE =
        (uint32_t)(((T + 3) * XW + T * XW) * ESZ + (BCQ ? BC32 : 2 * T * kNState * ESZ));
    static constexpr uint32_t TX_Z = (uint32_t)(T * XW * ESZ);
    static_assert((XW * ESZ) % 16 == 0 && XW % CW == 0, "TMA box rows must be whole 16-byte units");
    static_assert(!(BCQ && DIRECT), "one source of B/C");
};

// B and C of both directions widened to fp32 once per call, for the chunked
// kernel's BCQ form: bcq[r][b][t] = 8 quads (B_2q, B_2q+1, C_2q, C_2q+1), the
// layout of its fp32 B/C buffer (bf16 widening is exact).  One thread per
// (direction, batch row, token); grid-stride.
template <typename Tin>
__global__ void __launch_bounds__(256) widen_bc_kernel(const KParams p) {
    const int64_t rows = (int64_t)p.batch * p.L;
    for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < 2 * rows; i += (int64_t)gridDim.x * 256) {
        const int r = (int)(i / rows);
        const int64_t bt = i - r * rows;
        const Tin* Bp = static_cast<const Tin*>(p.B[r]) + bt * kNState;
        const Tin* Cp = static_cast<const Tin*>(p.C[r]) + bt * kNState;
        float bv[kNState], cv[kNState];
        if constexpr (sizeof(Tin) == 2) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 wb = reinterpret_cast<const uint4*>(Bp)[h];
                const uint4 wc = reinterpret_cast<const uint4*>(Cp)[h];
                const uint32_t b4[4] = {wb.x, wb.y, wb.z, wb.w}, c4[4] = {wc.x, wc.y, wc.z, wc.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {  // the bf16 bits are the high half of the fp32
                    bv[8 * h + 2 * u] = __uint_as_float(b4[u] << 16);
                    bv[8 * h + 2 * u + 1] = __uint_as_float(b4[u] & 0xffff0000u);
                    cv[8 * h + 2 * u] = __uint_as_float(c4[u] << 16);
                    cv[8 * h + 2 * u + 1] = __uint_as_float(c4[u] & 0xffff0000u);
                }
            }
        } else {
#pragma unroll
            for (int n = 0; n < kNState; ++n) {
                bv[n] = ldf(Bp, n);
                cv[n] = ldf(Cp, n);
            }
        }
        float4* o = reinterpret_cast<float4*>(p.bcq + i * 2 * kNState);
#pragma unroll
        for (int q = 0; q < kNState / 2; ++q) o[q] = make_float4(bv[2 * q], bv[2 * q + 1], cv[2 * q], cv[2 * q + 1]);
    }
}

// fp32 B/C layout per token: 8 quads (B_2p, B_2p+1, C_2p, C_2p+1), so that a
// lane's state pairs and their B and C are register pairs.
__device__ __forceinline__ int bc_quad_index(int n) { return (n >> 1) * 4 + (n & 1); }

template <int T, typename Tin>
__device__ __forceinline__ void convert_bc(const Tin* Bt, const Tin* Ct, float* bc, int tid, int nthreads,
                                           bool with_c) {
    for (int e = tid; e < T * kNState; e += nthreads) {
        const int row = e >> 4, n = e & 15;
        float* q = bc + row * 2 * kNState + bc_quad_index(n);
        q[0] = ldf(Bt, e);
        if (with_c) q[2] = ldf(Ct, e);
    }
}


// One warp's scan of one direction over CPW channels.
template <int G, int T, int NWD, int NS, typename Tin, int DIR>
struct TmaWorker {
    using Ge = TmaGeo<G, T, NWD, NS, Tin>;
    int c, j, cc, d;  // cc: channel inside the CTA tile; d: global channel
    int tc;           // column of the channel in the x/dt/z tiles
    bool dvalid;
    float A2[Ge::S];  // A * log2(e) of this lane's states
    float w[4], cb, bias, Dd;
    float h[Ge::S];
    float dsum;  // step sizes of this lane's steps (j, j+G, ...) so far

    __device__ __forceinline__ void setup(const KParams& p, int ct0, int wg, int lane) {
        dsum = 0.f;
        c = lane % Ge::CPW;
        j = lane / Ge::CPW;
        cc = wg * Ge::CPW + c;
        d = ct0 + cc;
        tc = ct0 % Ge::XW + cc;
        dvalid = d < p.D;
        const int64_t rd = (int64_t)DIR * p.D + (dvalid ? d : 0);
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
    }

    // tile row (token - kT) of step s
    static __device__ __forceinline__ int row_of(int s) { return DIR == 0 ? s : T - 1 - s; }

    // conv + SiLU and softplus of this lane's steps j, j+G, ...; steps
    // outside [s_lo, s_hi) (tokens >= L) become identity steps.  DSUM: also
    // add the valid step sizes to dsum.
    template <bool DSUM = false>
    __device__ __forceinline__ void elements(const Tin* xt, const Tin* dtt, int s_lo, int s_hi, float2* ed2,
                                             float* edu) {
#pragma unroll 2
        for (int e = 0; e < Ge::EPL; ++e) {
            const int s = j + G * e;
            // step s-3+q is x-tile row s+q (forward) or T+2-s-q (reverse)
            float cv = cb;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int xr = DIR == 0 ? s + q : T + 2 - s - q;
                cv = fmaf(w[q], ldf(xt, xr * Ge::XW + tc), cv);
            }
            const float u = silu(cv);
            const float dl = softplus(ldf(dtt, row_of(s) * Ge::XW + tc) + bias);
            const bool valid = s >= s_lo && s < s_hi;
            if constexpr (DSUM) dsum += valid ? dl : 0.f;
            ed2[s * Ge::CPW + c] = valid ? make_float2(dl, dl * u) : make_float2(0.f, 0.f);
            edu[s * Ge::CPW + c] = valid ? Dd * u : 0.f;
        }
    }

    // The S B (or C) values of states [jS, jS+S) of tile row r straight from
    // a TMA tile of the input dtype (bf16 widened in registers: exact).
    static __device__ __forceinline__ void tile_states(const Tin* t, int r, int jj, float (&v)[Ge::S]) {
        const Tin* q = t + r * kNState + jj * Ge::S;
        if constexpr (sizeof(Tin) == 4) {
#pragma unroll
            for (int i = 0; i < Ge::S; ++i) v[i] = ldf(q, i);
        } else if constexpr (Ge::S == 2) {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(q);
            v[0] = __uint_as_float(w << 16);
            v[1] = __uint_as_float(w & 0xffff0000u);
        } else if constexpr (Ge::S == 4) {
            const uint2 w = *reinterpret_cast<const uint2*>(q);
            v[0] = __uint_as_float(w.x << 16);
            v[1] = __uint_as_float(w.x & 0xffff0000u);
            v[2] = __uint_as_float(w.y << 16);
            v[3] = __uint_as_float(w.y & 0xffff0000u);
        } else {
            v[0] = ldf(q, 0);
        }
    }

    // Advance the states over steps G*e .. G*e+G-1; returns, for this lane,
    // sum_n C h of step G*e + j (WITH_Y) after the cross-lane combination.
    // DIRECT: B and C come from the TMA tiles Bt, Ct instead of the fp32
    // buffer bc.
    template <bool WITH_Y, bool DIRECT = false>
    __device__ __forceinline__ float step_group(int e, const float2* ed2, const float* bc, const Tin* Bt = nullptr,
                                                const Tin* Ct = nullptr) {
        if constexpr (DIRECT) {
            float pp[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const int s = G * e + g;
                const float2 q2 = ed2[s * Ge::CPW + c];
                float bv[Ge::S], cv[Ge::S];
                tile_states(Bt, row_of(s), j, bv);
                if constexpr (WITH_Y) tile_states(Ct, row_of(s), j, cv);
                float acc = 0.f;
                if constexpr (Ge::S == 1) {
                    const float ea = ex2_approx(q2.x * A2[0]);
                    h[0] = fmaf(ea, h[0], q2.y * bv[0]);
                    if constexpr (WITH_Y) acc = cv[0] * h[0];
                } else {
                    const float2 dd = make_float2(q2.x, q2.x);
                    const float2 du = make_float2(q2.y, q2.y);
                    float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int pq = 0; pq < Ge::S / 2; ++pq) {
                        const float2 v = mul2(dd, make_float2(A2[2 * pq], A2[2 * pq + 1]));
                        const float2 ea = make_float2(ex2_approx(v.x), ex2_approx(v.y));
                        const float2 drive = mul2(du, make_float2(bv[2 * pq], bv[2 * pq + 1]));
                        const float2 hh = fma2(ea, make_float2(h[2 * pq], h[2 * pq + 1]), drive);
                        h[2 * pq] = hh.x;
                        h[2 * pq + 1] = hh.y;
                        if constexpr (WITH_Y) acc2 = fma2(make_float2(cv[2 * pq], cv[2 * pq + 1]), hh, acc2);
                    }
                    acc = acc2.x + acc2.y;
                }
                pp[g] = acc;
            }
            if constexpr (WITH_Y)
                return group_transpose_reduce<G, Ge::CPW>(pp, j);
            else
                return 0.f;
        } else {
            float pp[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const int s = G * e + g;
                const float2 q2 = ed2[s * Ge::CPW + c];
                const float* row = bc + row_of(s) * 2 * kNState;
                float acc = 0.f;
                if constexpr (Ge::S == 1) {
                    const float ea = ex2_approx(q2.x * A2[0]);
                    h[0] = fmaf(ea, h[0], q2.y * row[bc_quad_index(j)]);
                    if constexpr (WITH_Y) acc = row[bc_quad_index(j) + 2] * h[0];
                } else {
                    const float2 dd = make_float2(q2.x, q2.x);
                    const float2 du = make_float2(q2.y, q2.y);
                    float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int pq = 0; pq < Ge::S / 2; ++pq) {
                        const float4 bcq = *reinterpret_cast<const float4*>(row + (j * Ge::S / 2 + pq) * 4);
                        const float2 v = mul2(dd, make_float2(A2[2 * pq], A2[2 * pq + 1]));
                        const float2 ea = make_float2(ex2_approx(v.x), ex2_approx(v.y));
                        const float2 drive = mul2(du, make_float2(bcq.x, bcq.y));
                        const float2 hh = fma2(ea, make_float2(h[2 * pq], h[2 * pq + 1]), drive);
                        h[2 * pq] = hh.x;
                        h[2 * pq + 1] = hh.y;
                        if constexpr (WITH_Y) acc2 = fma2(make_float2(bcq.z, bcq.w), hh, acc2);
                    }
                    acc = acc2.x + acc2.y;
                }
                pp[g] = acc;
            }
            if constexpr (WITH_Y)
                return group_transpose_reduce<G, Ge::CPW>(pp, j);
            else
                return 0.f;
        }
    }
};

template <int G, int T, int NWD, int NS, typename Tin, bool BCQ = false>
__device__ __forceinline__ void issue_chunk(const LayerMaps& maps, unsigned char* dir_base, uint64_t* full, int r,
                                            int i, int k, bool gated, int ct0, int b, int starve) {
    using Ge = TmaGeo<G, T, NWD, NS, Tin, false, BCQ>;
    if (starve) return;
    const int st = i % NS;
    unsigned char* sb = dir_base + st * Ge::STAGE;
    uint64_t* bar = full + st;
    mbar_arrive_expect_tx(bar, Ge::TX_BASE + (gated ? Ge::TX_Z : 0u));
    const int row0 = k * T;
    const int x0 = ct0 - ct0 % Ge::XW;  // the aligned tile row around the CTA's channels
    tma_load_3d(sb, &maps.x, bar, x0, r == 0 ? row0 - 3 : row0, b);
    tma_load_3d(sb + Ge::XB, &maps.dt[r], bar, x0, row0, b);
    if (gated) tma_load_3d(sb + Ge::XB + Ge::DTB, &maps.z, bar, x0, row0, b);
    tma_load_3d(sb + Ge::XB + 2 * Ge::DTB, &maps.B[r], bar, 0, row0, b);
    if constexpr (!BCQ) tma_load_3d(sb + Ge::XB + 2 * Ge::DTB + Ge::BB, &maps.C[r], bar, 0, row0, b);
}

// CARRY: start from p.carry_in, report p.carry_out and p.delta_sum (each where non-null).
template <int G, int T, int NWD, int NS, typename Tin, typename Tout, int DIR, bool CARRY, bool DIRECT,
          bool FULL_UNROLL = false, bool BCQ = false>
__device__ __forceinline__ void layer_direction(const LayerMaps& maps, const KParams& p, unsigned char* base,
                                                int wg, int lane) {
    using Ge = TmaGeo<G, T, NWD, NS, Tin, DIRECT, BCQ>;
    using Wk = TmaWorker<G, T, NWD, NS, Tin, DIR>;
    unsigned char* dir_base = base + DIR * Ge::DIR_BYTES;
    float* bc32 = reinterpret_cast<float*>(dir_base + NS * Ge::STAGE);
    unsigned char* wbase = base + Ge::WARP_OFF + (DIR * NWD + wg) * Ge::WARP_BYTES;
    float2* ed2 = reinterpret_cast<float2*>(wbase);
    float* edu = reinterpret_cast<float*>(wbase + Ge::ED2);
    float* ows = reinterpret_cast<float*>(wbase + Ge::ED2 + Ge::EDU);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + Ge::BAR_OFF) + DIR * NS;
    const int b = blockIdx.y;
    const int ct0 = blockIdx.x * Ge::CW;
    const int64_t L = p.L;
    const int D = p.D;
    const int nc = (int)((L + T - 1) / T);
    const int hF = nc / 2;
    const int meet = DIR == 0 ? hF : nc - hF;  // chunks before the meeting point
    const bool leader = (wg == 0 && lane == 0);
    const int gtid = wg * 32 + lane;
    const float scale = p.dir_scale[DIR];
    const int c0w = ct0 + wg * Ge::CPW;  // first channel of this warp
    // cp.async of the partner's fp32 y of chunk ii into buffer ii & 1, in pieces
    // of PC = min(4, CPW) channels.  D is a multiple of 4 on this path and c0w
    // a multiple of PC, so a piece that starts inside a row ends inside it and
    // is aligned to its size.
    auto fetch_partner = [&](int ii) {
        constexpr int PC = Ge::CPW < 4 ? Ge::CPW : 4;
        constexpr int PIECES = Ge::CPW / PC;
        const int kk = DIR == 0 ? ii : nc - 1 - ii;
        const int64_t row = (int64_t)b * L + (int64_t)kk * T;
        float* dst = ows + (ii & 1) * (T * Ge::CPW);
        for (int e = lane; e < T * PIECES; e += 32) {
            const int r = e / PIECES, q = e % PIECES;
            const bool ok = (int64_t)kk * T + r < L && c0w + PC * q < D;
            const float* src = p.ws + (row + (ok ? r : 0)) * D + (ok ? c0w + PC * q : 0);
            cp_async<PC * 4>(dst + r * Ge::CPW + PC * q, src, ok);
        }
        cp_async_commit();
    };

    Wk wk;
    wk.setup(p, ct0, wg, lane);
    if (CARRY && p.carry_in[DIR] && wk.dvalid) {
        const float* ci = p.carry_in[DIR] + ((int64_t)b * D + wk.d) * kNState + wk.j * Ge::S;
#pragma unroll
        for (int q = 0; q < Ge::S; ++q) wk.h[q] = ci[q];
    }

    if (leader) {
        for (int i = 0; i < NS && i < nc; ++i) {
            const int k = DIR == 0 ? i : nc - 1 - i;
            issue_chunk<G, T, NWD, NS, Tin, BCQ>(maps, dir_base, full, DIR, i, k, i >= meet, ct0, b, p.starve);
        }
    }

#pragma unroll 1
    for (int i = 0; i < nc; ++i) {
        const int k = DIR == 0 ? i : nc - 1 - i;
        const bool gated = i >= meet;
        if (i == meet) {
            __threadfence_block();
            named_bar_sync(3, 2 * NWD * 32);
        }
        // valid steps of this chunk: tokens < L
        const int nvalid = (int)((L - (int64_t)k * T < T) ? (L - (int64_t)k * T) : T);
        const int s_lo = DIR == 0 ? 0 : T - nvalid;
        const int s_hi = DIR == 0 ? nvalid : T;
        const int64_t chunk_row = (int64_t)b * L + (int64_t)k * T;  // global row of the chunk's token kT

        // The partner's y of the gated chunks -> shared memory, one chunk ahead
        // (buffer i & 1), so that the copy of chunk i+1 runs under the scan of
        // chunk i.  All of it was stored before the meeting barrier.
        if (i == meet) fetch_partner(i);
        if (gated && i + 1 < nc) fetch_partner(i + 1);

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
        float* bc = BCQ ? reinterpret_cast<float*>(dir_base + st * Ge::STAGE + Ge::XB + 2 * Ge::DTB)
                        : bc32 + (i & 1) * (T * kNState * 2);
        if constexpr (!DIRECT && !BCQ) convert_bc<T, Tin>(Bt, Ct, bc, gtid, NWD * 32, true);
        // every warp of the direction is past the previous chunk (and, unless
        // DIRECT, the fp32 B/C rows of this one are written)
        if constexpr (NWD == 1)
            __syncwarp();
        else
            named_bar_sync(1 + DIR, NWD * 32);
        if (leader && i >= 1 && i - 1 + NS < nc) {
            const int i2 = i - 1 + NS;
            issue_chunk<G, T, NWD, NS, Tin, BCQ>(maps, dir_base, full, DIR, i2, DIR == 0 ? i2 : nc - 1 - i2,
                                                 i2 >= meet, ct0, b, p.starve);
        }

        wk.template elements<CARRY>(xt, dtt, s_lo, s_hi, ed2, edu);
        if (gated) {
            if (i + 1 < nc)
                cp_async_wait_pending<1>();  // chunk i's copies; i+1's may still run
            else
                cp_async_wait_all();
        }
        __syncwarp();
        const float* owc = ows + (i & 1) * (T * Ge::CPW);

        float* wsw = p.ws + chunk_row * D + wk.d;
        Tout* outw = static_cast<Tout*>(p.out) + chunk_row * D + wk.d;
#pragma unroll (FULL_UNROLL ? Ge::EPL : 2)
        for (int e = 0; e < Ge::EPL; ++e) {
            const float yr = wk.template step_group<true, DIRECT>(e, ed2, bc, Bt, Ct);
            const int s = G * e + wk.j;
            if (s >= s_lo && s < s_hi && wk.dvalid) {
                const int tr = Wk::row_of(s);  // token - kT
                const float y = (yr + edu[s * Ge::CPW + wk.c]) * scale;
                if (!gated) {
                    wsw[(int64_t)tr * D] = y;
                } else {
                    const float zv = ldf(zt, tr * Ge::XW + wk.tc);
                    stf(outw, (int64_t)tr * D, (y + owc[tr * Ge::CPW + wk.c]) * silu(zv));
                }
            }
        }
        __syncwarp();
    }
    if (meet >= nc) {  // a single-chunk sequence: the reverse group meets after its only chunk
        __threadfence_block();
        named_bar_sync(3, 2 * NWD * 32);
    }
    if (CARRY && p.carry_out[DIR] && wk.dvalid) {
        float* co = p.carry_out[DIR] + ((int64_t)b * D + wk.d) * kNState + wk.j * Ge::S;
#pragma unroll
        for (int q = 0; q < Ge::S; ++q) co[q] = wk.h[q];
    }
    if (CARRY && p.delta_sum[DIR]) {  // the G lanes of a channel are CPW apart
        float ds = wk.dsum;
#pragma unroll
        for (int off = Ge::CPW; off < 32; off <<= 1) ds += __shfl_xor_sync(0xffffffffu, ds, off);
        if (wk.j == 0 && wk.dvalid) p.delta_sum[DIR][(int64_t)b * D + wk.d] = ds;
    }
}

// Resident CTAs per SM the register budget is sized for.  One warp per
// direction: 7 two-warp CTAs, so that the 1024 CTAs of a 4096-channel batch
// row (4 channels each) are resident at once on 148 SMs.
template <int G, int T, int NWD>
constexpr int layer_min_blocks() {
    return NWD == 1 ? 7 : (T <= 16 || G >= 16) ? 4 : 3;
}

template <int G, int T, int NWD, int NS, typename Tin, typename Tout, bool CARRY = false, bool DIRECT = false,
          bool FULL_UNROLL = false, bool BCQ = false>
__global__ void __launch_bounds__(2 * NWD * 32, (layer_min_blocks<G, T, NWD>()))
    layer_tma_kernel(const __grid_constant__ LayerMaps maps, const KParams p) {
    using Ge = TmaGeo<G, T, NWD, NS, Tin, DIRECT, BCQ>;
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
        layer_direction<G, T, NWD, NS, Tin, Tout, 0, CARRY, DIRECT, FULL_UNROLL, BCQ>(maps, p, base, warp, lane);
    else
        layer_direction<G, T, NWD, NS, Tin, Tout, 1, CARRY, DIRECT, FULL_UNROLL, BCQ>(maps, p, base, warp - NWD,
                                                                                     lane);
}

// ---------------------------------------------------------------- prefix

// Forward scan over P = p.L tokens from zero; writes the final state and the
// last three x of the prefix.  One CTA = one batch row x CW channels, NWD
// forward warps and the same chunk ring as the layer (only the forward
// half of its shared memory is used).  C and z are not read.
template <int G, int T, int NWD, int NS, typename Tin>
__global__ void __launch_bounds__(NWD * 32) prefix_tma_kernel(const __grid_constant__ LayerMaps maps,
                                                              const KParams p) {
    using Ge = TmaGeo<G, T, NWD, NS, Tin>;
    extern __shared__ __align__(128) unsigned char smem_dyn[];
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 127) & ~static_cast<uintptr_t>(127));
    const int wg = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t* full = reinterpret_cast<uint64_t*>(base + Ge::BAR_OFF);
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) mbar_init(full + i, 1);
        fence_barrier_init();
    }
    __syncthreads();
    float* bc32 = reinterpret_cast<float*>(base + NS * Ge::STAGE);
    unsigned char* wbase = base + Ge::WARP_OFF + wg * Ge::WARP_BYTES;
    float2* ed2 = reinterpret_cast<float2*>(wbase);
    float* edu = reinterpret_cast<float*>(wbase + Ge::ED2);
    const int b = blockIdx.y;
    const int ct0 = blockIdx.x * Ge::CW;
    const int64_t P = p.L;
    const int nc = (int)((P + T - 1) / T);
    const bool leader = (wg == 0 && lane == 0);
    constexpr uint32_t TX = (uint32_t)(((T + 3) * Ge::XW + T * Ge::XW + T * kNState) * Ge::ESZ);
    const int x0 = ct0 - ct0 % Ge::XW;  // the aligned tile row around the CTA's channels

    auto issue = [&](int i) {
        if (p.starve) return;
        const int st = i % NS;
        unsigned char* sb = base + st * Ge::STAGE;
        uint64_t* bar = full + st;
        mbar_arrive_expect_tx(bar, TX);
        tma_load_3d(sb, &maps.x, bar, x0, i * T - 3, b);
        tma_load_3d(sb + Ge::XB, &maps.dt[0], bar, x0, i * T, b);
        tma_load_3d(sb + Ge::XB + 2 * Ge::DTB, &maps.B[0], bar, 0, i * T, b);
    };

    TmaWorker<G, T, NWD, NS, Tin, 0> wk;
    wk.setup(p, ct0, wg, lane);
    if (leader)
        for (int i = 0; i < NS && i < nc; ++i) issue(i);

#pragma unroll 1
    for (int i = 0; i < nc; ++i) {
        const int st = i % NS;
        mbar_wait_bounded(full + st, (uint32_t)((i / NS) & 1), p.wait_limit);
        const unsigned char* sb = base + st * Ge::STAGE;
        const Tin* xt = reinterpret_cast<const Tin*>(sb);
        const Tin* dtt = reinterpret_cast<const Tin*>(sb + Ge::XB);
        const Tin* Bt = reinterpret_cast<const Tin*>(sb + Ge::XB + 2 * Ge::DTB);
        float* bc = bc32 + (i & 1) * (T * kNState * 2);
        convert_bc<T, Tin>(Bt, Bt, bc, wg * 32 + lane, NWD * 32, false);
        named_bar_sync(1, NWD * 32);
        if (leader && i >= 1 && i - 1 + NS < nc) issue(i - 1 + NS);
        const int nvalid = (int)((P - (int64_t)i * T < T) ? (P - (int64_t)i * T) : T);
        wk.elements(xt, dtt, 0, nvalid, ed2, edu);
        __syncwarp();
#pragma unroll 2
        for (int e = 0; e < Ge::EPL; ++e) wk.template step_group<false>(e, ed2, bc);
        __syncwarp();
    }
    if (wk.dvalid) {
#pragma unroll
        for (int q = 0; q < Ge::S; ++q)
            p.h_out[((int64_t)b * p.D + wk.d) * kNState + wk.j * Ge::S + q] = wk.h[q];
        if (wk.j == 0) {
            const Tin* X = static_cast<const Tin*>(p.x);
            Tin* tail = static_cast<Tin*>(p.tail_out);
            for (int q = 0; q < 3; ++q) {
                const int64_t t = P - 3 + q;
                tail[((int64_t)b * 3 + q) * p.D + wk.d] =
                    t >= 0 ? X[((int64_t)b * P + t) * p.D + wk.d] : cvt_from<Tin>(0.f);
            }
        }
    }
}

}  // namespace bimamba

// carry.cuh -- composing the scan carries of a sequence cut into segments
// ("DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone", §3.2
// Eq. (4)-(5): the recurrence h_t = exp(Delta_t A) h_{t-1} + Delta_t B_t u_t).
//
// The recurrence is affine in h, so a segment j run from a zero state leaves
// h_end_j, and run from a state h leaves exp(A * sum_{t in j} Delta_t) h +
// h_end_j (the decays of its steps multiply).  The forward state entering
// segment s is therefore the fold of segments 0..s-1 in order, and the reverse
// state entering segment s (at its last token) the fold of segments
// nseg-1..s+1, each with its own direction's A.
#pragma once

#include <stdint.h>

#include "scan_kernels.cuh"

namespace bimamba {

// h_out_all [nseg][2][batch][D][16]: each segment's final states from zero
// (direction 0 after its last token, direction 1 after its first);
// dsum_all [nseg][2][batch][D]: each segment's sum of step sizes; A [2][D][16].
// Writes h_in [2][batch][D][16], the states entering segment `seg`.
// One thread per (batch row, channel, state).
__global__ void compose_carries_kernel(const float* h_out_all, const float* dsum_all, const float* A, int nseg,
                                       int seg, int batch, int D, float* h_in) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t per_dir = (int64_t)batch * D * kNState;
    if (i >= per_dir) return;
    const int64_t bd = i / kNState;  // batch row * D + channel
    const int n = (int)(i % kNState);
    const int d = (int)(bd % D);
    const int64_t seg_h = 2 * per_dir, seg_ds = 2 * (int64_t)batch * D;
    float hf = 0.f;
    const float af = A[(int64_t)d * kNState + n];
    for (int j = 0; j < seg; ++j)
        hf = fmaf(expf(af * dsum_all[j * seg_ds + bd]), hf, h_out_all[j * seg_h + i]);
    float hb = 0.f;
    const float ab = A[((int64_t)D + d) * kNState + n];
    for (int j = nseg - 1; j > seg; --j)
        hb = fmaf(expf(ab * dsum_all[j * seg_ds + (int64_t)batch * D + bd]), hb, h_out_all[j * seg_h + per_dir + i]);
    h_in[i] = hf;
    h_in[per_dir + i] = hb;
}

}  // namespace bimamba

/*
 * bimamba.h -- C ABI of the B200 (sm_100a) bidirectional Mamba mixer layer.
 *
 * The layer is the sequence mixer of DiffuMamba's masked-diffusion denoiser
 * ("DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone",
 * arXiv 2511.15927v4, §3.2 Eq. (4)-(6), App. A.1 Eq. (7)-(9)): two
 * independent Mamba layers, one over the sequence left to right and one right
 * to left, whose outputs are added.  Its inputs are the already-projected
 * x, z, dt, B, C.  Per batch row b, channel d and direction r (0 = forward,
 * 1 = reverse):
 *
 *   u_r[t]     = silu(conv_b[r][d] + sum_{k<4} conv_w[r][d][k] * x[t - 3 + k])   (r = 0)
 *              = silu(conv_b[r][d] + sum_{k<4} conv_w[r][d][k] * x[t + 3 - k])   (r = 1)
 *                (zero outside [0, L): causal / anti-causal width-4 conv, §3.2)
 *   delta_r[t] = softplus(dt_r[t] + dt_bias[r][d])
 *   h_n        = exp(delta_r[t] * A[r][d][n]) * h_n + delta_r[t] * B_r[t][n] * u_r[t]
 *                over t = 0..L-1 (r = 0, Eq. (4)) or t = L-1..0 (r = 1, Eq. (5)), h = 0 first
 *   y_r[t]     = sum_n C_r[t][n] * h_n + D[r][d] * u_r[t]
 *   out[t]     = (y_0[t] + y_1[t]) * silu(z[t])                   (Eq. (6), SiLU(z) gate)
 *
 * The block step is the block-cached decoding form (§4.3: right-to-left
 * state updates stay inside the current block while the cached forward states
 * carry across blocks; "Training Hybrid Block Diffusion Language Models with
 * Partial Bidirectionality", arXiv 2607.02805, abstract: restricting the
 * reverse scan to the active block makes caching across blocks exact).
 *
 * Conventions for every entry point:
 *  - All tensors are caller-owned device memory, row-major and contiguous in
 *    the layouts given below.  The library allocates nothing, never
 *    synchronises the stream and never reads device data on the host.
 *  - Work is enqueued on `cuda_stream` (a cudaStream_t; NULL = legacy default
 *    stream) and runs asynchronously; errors of the kernels themselves appear
 *    at the caller's next synchronisation.
 *  - Return value 0 (BIMAMBA_OK) or a negative BIMAMBA_ERR_* code; nothing is
 *    launched when a check fails.  No C++ exception crosses this boundary.
 *  - Outputs must not alias inputs, except where stated (state commit).
 *  - d_state must be 16 (the state dimension of the layer's S4D-real
 *    parameterisation); other values return BIMAMBA_ERR_UNSUPPORTED.
 *  - Pointers must be aligned to their element size.
 */
#ifndef BIMAMBA_H
#define BIMAMBA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BIMAMBA_OK                0
#define BIMAMBA_ERR_INVALID_ARG  (-1)  /* NULL pointer, size <= 0, size too large */
#define BIMAMBA_ERR_UNSUPPORTED  (-2)  /* d_state != 16, unknown dtype or flag    */
#define BIMAMBA_ERR_MISALIGNED   (-3)  /* a pointer not aligned to its element    */
#define BIMAMBA_ERR_WORKSPACE    (-4)  /* workspace NULL or smaller than needed   */
#define BIMAMBA_ERR_CUDA         (-5)  /* a CUDA launch or attribute call failed  */

/* Element type of x, z, dt, B, C, the conv tail and the output. */
typedef enum { BIMAMBA_F32 = 0, BIMAMBA_BF16 = 1 } bimamba_dtype_t;

/* flags (bitwise OR) */
#define BIMAMBA_FWD_ONLY   0x1u   /* y_1 taken as 0: out = y_0 * silu(z) (test aid) */
#define BIMAMBA_REV_ONLY   0x2u   /* y_0 taken as 0: out = y_1 * silu(z) (test aid) */
/* Bits 8..12 select the number of lanes that share one channel's 16 states
 * (1, 2, 4, 8 or 16; 0 = chosen from the problem size).  A tuning knob: the
 * result does not depend on it beyond fp32 rounding order. */
#define BIMAMBA_LANES_SHIFT 8
#define BIMAMBA_LANES_MASK  (0x1fu << BIMAMBA_LANES_SHIFT)
/* Use the kernel that stages tiles with ordinary loads instead of the
 * TMA-fed one (test aid; the TMA kernel is otherwise chosen whenever every
 * x/z/dt/B/C pointer is 16-byte aligned and a row of d_inner elements is a
 * whole number of 16-byte units). */
#define BIMAMBA_NO_TMA      0x4000u
/* Bits 16..17 select the chunk length of the TMA-fed kernel (0 = chosen from
 * the problem size, 1 = 16 tokens, 2 = 32 tokens).  A tuning knob like the
 * lane count. */
#define BIMAMBA_CHUNK_SHIFT 16
#define BIMAMBA_CHUNK_MASK  (0x3u << BIMAMBA_CHUNK_SHIFT)
/* Bits 18..19 select the TMA-fed kernel family (0 = chosen from the problem
 * size).  1: chunked -- G lanes share one channel's states, for few channels
 * (batch 1, long sequences).  2: per-token fused -- one lane per channel,
 * groups of G lanes share B/C across G channels, for many channels.  With
 * family 2 the lane field (bits 8..12) is the group size (1, 2, 4 or 8; 0 =
 * 1: a lane per channel with all 16 states and B/C widened to fp32 once per
 * chunk); at 2 lanes B/C are widened once per chunk unless the chunk field
 * is 1, at 4 only if it is 2.  3: chunked parallel scan -- per 64-token chunk a
 * channel's 8 lanes scan 8-step pieces and combine their carries with warp
 * shuffles (the lane and chunk fields are not read).  Tuning knobs: the
 * result does not depend on the family beyond fp32 rounding order. */
#define BIMAMBA_FAMILY_SHIFT 18
#define BIMAMBA_FAMILY_MASK  (0x3u << BIMAMBA_FAMILY_SHIFT)
/* Family 1 at 8 lanes per channel: 4 warps per direction per CTA with B/C
 * widened to fp32 once per chunk, instead of one warp per direction reading
 * B/C from the tile (tuning knob). */
#define BIMAMBA_CHUNKED_WIDE 0x2000u
/* bimamba2_layer_fwd, tensor-core path: run the two directions as separate
 * ticket-ordered CTAs of one launch even when one direction's grid fits in
 * one wave, where the clustered form is otherwise taken (test aid; the result
 * does not depend on it beyond fp32 rounding order). */
#define BIMAMBA_M2_NO_CLUSTER 0x8000u
/* Test aid for the failure path: the TMA-fed kernels issue no tile loads,
 * so every wait for a tile gives up (after ~0.1 ms instead of ~2 s); the
 * kernel still finishes, its output is undefined, and bit 0 of
 * bimamba_device_error() is set.  bimamba_layer_fwd only. */
#define BIMAMBA_TEST_STARVE 0x100000u

/* Parameters of both directions, fp32 device pointers, index 0 = forward. */
typedef struct {
    const float *A;        /* [2][d_inner][d_state]   state matrix diagonal (negative) */
    const float *D;        /* [2][d_inner]            skip weight                       */
    const float *dt_bias;  /* [2][d_inner]            added to dt before softplus       */
    const float *conv_w;   /* [2][d_inner][4]         conv taps, see the formula above  */
    const float *conv_b;   /* [2][d_inner] or NULL    conv bias (NULL reads as 0)       */
} bimamba_params_t;

/* Layer inputs, device pointers of type `dtype`.  x and z are shared by the
 * two directions; dt, B and C are per direction (dt[1] may equal dt[0], and
 * likewise for B and C, to share them). */
typedef struct {
    const void *x;         /* [batch][L][d_inner]  */
    const void *z;         /* [batch][L][d_inner]  */
    const void *dt[2];     /* [batch][L][d_inner]  raw step size, before bias and softplus */
    const void *B[2];      /* [batch][L][d_state]  */
    const void *C[2];      /* [batch][L][d_state]  */
    bimamba_dtype_t dtype;
} bimamba_inputs_t;

/* The cached forward state a block step starts from. */
typedef struct {
    float *h;              /* [batch][d_inner][d_state] fp32: forward scan state          */
    void *conv_x;          /* [batch][3][d_inner] of the inputs' dtype: x of the last
                              three prefix tokens, oldest first (zeros before token 0)   */
} bimamba_fwd_state_t;

/* Bytes of device workspace bimamba_layer_fwd needs: one fp32 per
 * (batch, token, channel) for the half-sequence partial outputs the two
 * directions hand each other, rounded up to 256 bytes, plus 32 fp32 per
 * (direction, batch, token) for B and C widened once per call (the chunked
 * kernel at 8 lanes per channel).  Returns 0 for invalid sizes. */
size_t bimamba_workspace_bytes(int batch, int64_t L, int d_inner, int d_state, unsigned flags);

/* Full-sequence bidirectional layer (§3.2 Eq. (4)-(6)).
 *   in          inputs; in->dtype is the input element type
 *   p           parameters
 *   out         [batch][L][d_inner] of out_dtype
 *   workspace   >= bimamba_workspace_bytes(...) bytes of device memory, 16-byte
 *               aligned, contents ignored on entry and undefined on exit
 * One kernel launch (two for the chunked kernel at 8 lanes per channel: the
 * B/C widening, then the layer). */
int bimamba_layer_fwd(const bimamba_inputs_t *in, const bimamba_params_t *p,
                      void *out, bimamba_dtype_t out_dtype,
                      int batch, int64_t L, int d_inner, int d_state, unsigned flags,
                      void *workspace, size_t workspace_bytes, void *cuda_stream);

/* Scan carries of one layer call (a segment of a longer sequence).  Each
 * [2] is per direction (0 forward, 1 reverse); every pointer may be NULL
 * (unused).  Device memory, fp32, caller-owned, 4-byte aligned.
 *   h_in       [batch][d_inner][d_state]: the state entering the direction's
 *              first step (forward: before token 0; reverse: after token L-1),
 *              instead of zero
 *   h_out      [batch][d_inner][d_state]: the state after the direction's last
 *              step (forward: after token L-1; reverse: after token 0)
 *   delta_sum  [batch][d_inner]: sum over the L tokens of the direction's step
 *              size softplus(dt + dt_bias)
 *   conv_halo  [batch][3][d_inner] of the input dtype, rows in token order,
 *              aligned to its element: the x the direction's conv reads outside
 *              [0, L) (forward: the three tokens before token 0; reverse: the
 *              three after token L-1), instead of zeros */
typedef struct {
    const float *h_in[2];
    float *h_out[2];
    float *delta_sum[2];
    const void *conv_halo[2];
} bimamba_carry_t;

/* bimamba_layer_fwd with carries: the recurrences of §3.2 Eq. (4)-(5) start
 * from carry->h_in and report their final states and step-size sums.  With
 * these a sequence cut into segments (one per GPU) is scanned exactly: run
 * each segment from zero for h_out and delta_sum, compose the carries with
 * bimamba_compose_carries, run again from them.  The conv reads the
 * neighbouring segments' x rows from conv_halo (zeros where it is NULL), so
 * a segment is passed as it is, with no copy.  h_in may alias
 * h_out only if both are the same direction's (each state word is read
 * before it is written, by the same thread).  Runs the TMA-fed kernel
 * families only: inputs that bimamba_layer_fwd would run on its fallback
 * kernels (pointers not 16-byte aligned, d_inner % 8 != 0, or flags with
 * BIMAMBA_NO_TMA or a fallback lane count) return BIMAMBA_ERR_UNSUPPORTED; with
 * carries the per-token family runs one lane per channel and the chunked
 * family its automatic chunk length, whatever the lane-group and chunk flags
 * ask.
 * carry == NULL returns BIMAMBA_ERR_INVALID_ARG.  Other arguments, checks
 * and errors: as bimamba_layer_fwd.  One kernel launch. */
int bimamba_layer_fwd_carry(const bimamba_inputs_t *in, const bimamba_params_t *p, const bimamba_carry_t *carry,
                            void *out, bimamba_dtype_t out_dtype,
                            int batch, int64_t L, int d_inner, int d_state, unsigned flags,
                            void *workspace, size_t workspace_bytes, void *cuda_stream);

/* The carries entering segment `seg` of a sequence cut into nseg segments
 * (in token order), from every segment's bimamba_layer_fwd_carry run from
 * zero: since each step is affine in the state, a segment run from state h
 * ends in exp(A * delta_sum) * h + h_out.
 *   h_out_all      [nseg][2][batch][d_inner][d_state]: segment j's h_out[0], h_out[1]
 *   delta_sum_all  [nseg][2][batch][d_inner]: segment j's delta_sum[0], delta_sum[1]
 *   p              only p->A is read
 *   h_in           [2][batch][d_inner][d_state] out: forward = fold of segments
 *                  0..seg-1, reverse = fold of segments nseg-1..seg+1 (zero at the ends)
 * Device pointers, fp32, 4-byte aligned; h_in must not alias the inputs.
 * One kernel launch. */
int bimamba_compose_carries(const float *h_out_all, const float *delta_sum_all, const bimamba_params_t *p,
                            int nseg, int seg, int batch, int d_inner, int d_state, float *h_in, void *cuda_stream);

/* The full layer for callers that cannot allocate device memory -- a plugin
 * inside a host application that owns all GPU memory, or a caller that
 * reaches this library only through the C ABI with no CUDA allocator -- and
 * so cannot hand bimamba_layer_fwd a workspace.  The paper has no
 * counterpart: this is an interface convenience, computing exactly what
 * bimamba_layer_fwd computes.
 *   Instead of a caller's workspace it uses a scratch array built into the
 * library: 64 MiB that every GPU loading the library holds until the process
 * exits.  It therefore accepts the sizes whose bimamba_workspace_bytes fits
 * in 64 MiB (batch * L * (4 d_inner + 256) bytes, about batch * L * d_inner
 * <= 16.5 M at d_inner 4096) and returns BIMAMBA_ERR_WORKSPACE above that.
 * It allocates and frees nothing.
 *   The first call in a CUDA context looks up the scratch array's device
 * address (cudaGetSymbolAddress, with the device current) and caches it for
 * that context; a context created anew (after cudaDeviceReset, say) looks it
 * up again.  That first lookup may load the library's module into the
 * context, which reserves the 64 MiB and may synchronise the device: make
 * one call on each device before any stream capture or latency-sensitive
 * work.  All calls on a device share the one array: the kernel writes every
 * scratch value before reading it, so nothing needs clearing between calls,
 * but two calls whose kernels overlap on the GPU (other streams, or other
 * host threads) race on it and give undefined output.  Other arguments,
 * checks and errors: as bimamba_layer_fwd, in the same order, the workspace
 * check last (a problem too large for the scratch returns
 * BIMAMBA_ERR_WORKSPACE only once every other argument has passed). */
int bimamba_layer_fwd_noalloc(const bimamba_inputs_t *in, const bimamba_params_t *p,
                              void *out, bimamba_dtype_t out_dtype,
                              int batch, int64_t L, int d_inner, int d_state, unsigned flags,
                              void *cuda_stream);

/* Forward-only scan over a prefix of P tokens from a zero state (§4.3: the
 * cache a decoded block leaves behind).  Reads prefix->x, prefix->dt[0],
 * prefix->B[0] (z, C and the reverse inputs are not read and may be NULL).
 * Writes state_out->h and state_out->conv_x.  One kernel launch. */
int bimamba_prefix_state(const bimamba_inputs_t *prefix, const bimamba_params_t *p,
                         int batch, int64_t P, int d_inner, int d_state,
                         bimamba_fwd_state_t *state_out, void *cuda_stream);

/* One denoising step on the active block of block_len tokens (§4.3; the
 * follow-up's abstract).  The forward direction starts from *prefix_state;
 * the reverse direction sees the block alone (zero state after its last token,
 * conv zero-padded past its end).  out: [batch][block_len][d_inner] of
 * out_dtype.  If new_state is not NULL the forward state after the block is
 * written there (commit); new_state may be prefix_state itself (in place).
 * block_len must be in [1, 64].  One kernel launch.  The block's rows are
 * staged with asynchronous 16-byte copies when every x/z/dt/B/C pointer and
 * prefix_state->conv_x is 16-byte aligned and a row of d_inner elements is a
 * whole number of 16-byte units; otherwise, or with BIMAMBA_NO_TMA, with
 * ordinary loads.  A non-zero lane field in flags (bits 8..12) selects the
 * earlier kernel that splits a channel's states over that many lanes (test
 * aid).  The results do not depend on the kernel beyond fp32 rounding order. */
int bimamba_block_step(const bimamba_fwd_state_t *prefix_state, const bimamba_inputs_t *block,
                       int block_len, const bimamba_params_t *p,
                       void *out, bimamba_dtype_t out_dtype,
                       int batch, int d_inner, int d_state,
                       bimamba_fwd_state_t *new_state, unsigned flags, void *cuda_stream);

/* ---------------------------------------------------------------- Mamba-2
 * The bidirectional Mamba-2 mixer at the shape of the pages' own denoiser
 * ("DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone", §3.2
 * Eq. (4)-(6); App. C Table 8: Mamba-2, state dimension 128, conv dimension
 * 4, no weight tie between directions; App. C Table 12: d_inner 3840 = 120
 * heads x 32, conv over the x | B | C channels, one group of B and C).  Per
 * direction r, batch row b, head h (headdim P, d_state N, conv channels
 * CH = nheads*P + 2N):
 *   v = silu(conv_r(xbc_r))            causal (r = 0) / anti-causal (r = 1),
 *                                      zero outside [0, L); x | B | C = v
 *   delta[t] = softplus(dt_r[t][h] + dt_bias_r[h])
 *   S[p][n] <- exp(delta A_r[h]) S[p][n] + delta x[t][h*P+p] B[t][n]
 *   y_r[t][h*P+p] = sum_n C[t][n] S[p][n] + D_r[h] x[t][h*P+p]
 *   out[t] = (y_0[t] + y_1[t]) * silu(z[t])
 * The gated RMSNorm and out_proj of a Mamba-2 block are not part of this
 * call.  This version supports headdim 32 and d_state 128 (the pages'
 * shape; anything else returns BIMAMBA_ERR_UNSUPPORTED). */

/* Parameters of both directions, fp32 device pointers, index 0 = forward. */
typedef struct {
    const float *A;        /* [2][nheads] (negative: the decay is exp(delta*A)) */
    const float *D;        /* [2][nheads] */
    const float *dt_bias;  /* [2][nheads] */
    const float *conv_w;   /* [2][CH][4], 16-byte aligned: forward tap k multiplies x[t-3+k], reverse tap k x[t+3-k] */
    const float *conv_b;   /* [2][CH] or NULL (= 0) */
} bimamba2_params_t;

/* Inputs, device pointers of `dtype`, row-major. */
typedef struct {
    const void *xbc[2];    /* [batch][L][CH] per direction (the same pointer twice = shared), 16-byte aligned */
    const void *z;         /* [batch][L][nheads*headdim], 16-byte aligned */
    const void *dt[2];     /* [batch][L][nheads] per direction */
    bimamba_dtype_t dtype;
} bimamba2_inputs_t;

/* Bytes of device workspace bimamba2_layer_fwd needs (fp32 conv features of
 * both directions, step sizes, the forward and reverse outputs, the tensor
 * path's C/B tiles, its ticket counter and per-(batch row, head) flags); 0
 * for invalid sizes. */
size_t bimamba2_workspace_bytes(int batch, int64_t L, int nheads, int headdim, int d_state);

/* The full-sequence Mamba-2 mixer.  out: [batch][L][nheads*headdim] of
 * out_dtype, 16-byte aligned, must not alias an input.  workspace: device memory of at least
 * bimamba2_workspace_bytes(), 256-byte aligned, caller-owned.
 * bf16 inputs run the scan in its chunked dual form on the tensor cores
 * (chunks of 128 steps; fp16 operands, fp32 accumulation and state; within
 * 2e-3 of the exact result normwise): the C/B chunk tiles, then the two
 * directions' chunk scans, which compute their x features and step sizes
 * from xbc and dt themselves: when batch * nheads <= 2 x the SM count both
 * run in one launch as the two CTAs of a thread-block cluster (each stores
 * its y over the first half of its walk and, after meeting at a cluster
 * barrier, combines and gates over the second half), else in one launch as
 * separate CTAs ordered by tickets taken at their start (the forwards first,
 * storing y; each reverse waits for its own forward's flag, then gates; the
 * counter and flags are cleared by a memset before the launch); plus a
 * clearing of the ragged chunk's tiles when L % 128 != 0.  A reverse CTA's
 * wait is bounded (~2 s): on timeout bit 1 of bimamba_device_error() is set
 * and the output is undefined.  fp32 inputs, or flags with
 * BIMAMBA_NO_TMA, run the step-by-step scan on the CUDA cores in fp32: three
 * launches.  Other flags: BIMAMBA_FWD_ONLY, BIMAMBA_REV_ONLY, BIMAMBA_M2_NO_CLUSTER (test aids);
 * BIMAMBA_TEST_STARVE (tensor-core path: no tile copies are issued, every
 * wait gives up after ~0.1 ms and sets bit 0 of bimamba_device_error(); in
 * the ticket-ordered form no forward sets its flag either, so every reverse
 * CTA's wait gives up after ~0.1 ms and sets bit 1; the output is
 * undefined).  Nothing is launched when a check fails.  Returns
 * BIMAMBA_OK or a negative status. */
int bimamba2_layer_fwd(const bimamba2_inputs_t *in, const bimamba2_params_t *p,
                       void *out, bimamba_dtype_t out_dtype,
                       int batch, int64_t L, int nheads, int headdim, int d_state,
                       unsigned flags, void *workspace, size_t workspace_bytes, void *cuda_stream);

/* Cached forward state of the Mamba-2 mixer for block-cached decoding
 * ([DM] §4.3; [BD] abstract: the reverse scan restricted to the active block
 * makes the forward state an exact cache). */
typedef struct {
    float *S;          /* [batch][nheads][headdim][d_state] fp32, 16-byte aligned */
    void *conv_xbc;    /* [batch][3][CH] of the input dtype, 16-byte aligned: the forward
                          direction's last three xBC rows, oldest first */
} bimamba2_fwd_state_t;

/* Forward scan of the Mamba-2 mixer over a prefix of P tokens from a zero
 * state: writes state_out->S and state_out->conv_xbc.  Reads prefix->xbc[0]
 * and prefix->dt[0] (the rest may be NULL).  workspace: at least
 * bimamba2_workspace_bytes(batch, P, ...) bytes, 256-byte aligned.  bf16
 * inputs: the chunked dual form's state updates on the tensor cores (fp16
 * operands, fp32 state; within the 2e-3 bound of bf16 I/O): the C/B tiles,
 * the state pass, the conv tail (3 launches and a memset when P % 128 != 0).
 * fp32 inputs: conv features, the step-by-step forward scan on the CUDA cores
 * in fp32, the conv tail (3 launches). */
int bimamba2_prefix_state(const bimamba2_inputs_t *prefix, const bimamba2_params_t *p,
                          int batch, int64_t P, int nheads, int headdim, int d_state,
                          bimamba2_fwd_state_t *state_out, void *workspace, size_t workspace_bytes,
                          void *cuda_stream);

/* One denoising step of the Mamba-2 mixer on the active block of block_len
 * tokens: the forward direction continues from *prefix_state (its conv reads
 * the cached tail before the block), the reverse direction sees the block
 * alone (zero state after its last token, conv zero-padded past its end);
 * out = (y_0 + y_1) * silu(z), [batch][block_len][nheads*headdim].  If
 * new_state is not NULL the forward state and conv tail after the block are
 * written there (commit); new_state may be prefix_state itself.  workspace:
 * at least bimamba2_workspace_bytes(batch, block_len, ...) bytes.  Flags:
 * BIMAMBA_FWD_ONLY, BIMAMBA_REV_ONLY or 0.  bf16 inputs with block_len <= 32
 * and nheads % 4 == 0: the block's closed form, C S^T and the state update on
 * the tensor cores with fp16 operands (within the 2e-3 bound for bf16 I/O);
 * 4 launches, 5 with a commit.  Otherwise the step-by-step scan on the CUDA
 * cores in fp32; 3 launches, 4 with a commit. */
int bimamba2_block_step(const bimamba2_fwd_state_t *prefix_state, const bimamba2_inputs_t *block,
                        int64_t block_len, const bimamba2_params_t *p,
                        void *out, bimamba_dtype_t out_dtype,
                        int batch, int nheads, int headdim, int d_state,
                        bimamba2_fwd_state_t *new_state, unsigned flags,
                        void *workspace, size_t workspace_bytes, void *cuda_stream);

/* ---- The layer's neighbours (App. A.1 Eq. (10)-(11), Table 12): AdaLN in
 * front of the mixer and the projections around it.  bf16 in and out,
 * device pointers, caller-owned, 16-byte aligned (gamma, beta: fp32).
 * Rows are the batch * L tokens in [batch][L] order.  Nothing is launched when
 * a check fails; returns BIMAMBA_OK or a negative status. */

/* AdaLN (Eq. (10)): out[r] = gamma[b] * (x[r] - mu(x[r])) / sigma(x[r]) + beta[b]
 * for every token row r of batch row b, mu and sigma^2 the mean and (biased)
 * variance of the row's d values, sigma = sqrt(variance + eps).
 *   x, out     [batch][L][d] bf16 (out must not alias x)
 *   gamma, beta [batch][d] fp32, 16-byte aligned: the timestep embedding's modulation
 * d % 8 == 0 and d <= 8192 (else UNSUPPORTED); eps > 0.  One kernel launch. */
int bimamba_adaln(const void *x, const float *gamma, const float *beta, void *out,
                  int batch, int64_t L, int d, float eps, void *cuda_stream);

/* The input projection, written straight into the layer's input arrays:
 * for each token row r, y[r][n] = sum_k a[r][k] * w_in[n][k] (fp32
 * accumulation on the tensor cores, rounded to bf16), with the columns n of
 * w_in laid out as [x | z | dt_f | dt_b | B_f | C_f | B_b | C_b] (d_inner,
 * d_inner, d_inner, d_inner, then d_state each: 4 d_inner + 4 d_state rows).
 *   a      [batch][L][d_model]      (e.g. bimamba_adaln's output)
 *   w_in   [4 d_inner + 4 d_state][d_model]
 *   x, z   [batch][L][d_inner];  dt [2][batch][L][d_inner];  B, C [2][batch][L][d_state]
 * (the layouts bimamba_layer_fwd reads, with dir_stride 0 for x and z).
 * d_model % 64 == 0, d_inner % 8 == 0, d_state == 16 (else UNSUPPORTED);
 * batch * L <= 8,388,480.  One kernel launch. */
int bimamba_in_proj(const void *a, const void *w_in, int batch, int64_t L, int d_model, int d_inner, int d_state,
                    void *x, void *z, void *dt, void *B, void *C, void *cuda_stream);

/* The output projection of the layer's gated output (the sum of the two
 * directions and the SiLU(z) gate are already applied by bimamba_layer_fwd):
 * out[r][n] = sum_k y[r][k] * w_out[n][k], fp32 accumulation, bf16 result.
 *   y      [batch][L][d_inner];  w_out [d_model][d_inner];  out [batch][L][d_model]
 * d_inner % 64 == 0, d_model % 8 == 0 (else UNSUPPORTED); batch * L <= 8,388,480.
 * One kernel launch. */
int bimamba_out_proj(const void *y, const void *w_out, int batch, int64_t L, int d_inner, int d_model, void *out,
                     void *cuda_stream);

/* The per-token features the layer computes before its scans, written out
 * for inspection (a diagnostic: the layer kernels keep them in registers and
 * never store them).  With the definitions at the top of this header:
 *   u      [2][batch][L][d_inner] fp32 out: u_r[t] = silu(conv_r(x)[t])
 *   delta  [2][batch][L][d_inner] fp32 out: delta_r[t] = softplus(dt_r[t] + dt_bias[r][d])
 * computed by the same device code the layer, prefix and block-step kernels
 * inline (conv accumulated bias first, then taps 0..3; the same silu and
 * softplus).  Reads in->x, in->dt[0], in->dt[1] (z, B, C may be NULL) and
 * p->conv_w, p->conv_b, p->dt_bias.  Pointers aligned to their element size.
 * One kernel launch. */
int bimamba_features(const bimamba_inputs_t *in, const bimamba_params_t *p, int batch, int64_t L, int d_inner,
                     float *u, float *delta, void *cuda_stream);

/* Read (and, if reset != 0, clear) the error word of the current device.
 * Kernels never wait without bound: a wait for a tile that gives up after
 * about two seconds sets bit 0 (a tile load that never arrived), a Mamba-2
 * reverse CTA's wait for its forward that gives up sets bit 1, and the kernel
 * finishes with undefined output instead of hanging.  Synchronises the
 * device.  Returns the word, or BIMAMBA_ERR_CUDA if it cannot be read. */
int bimamba_device_error(int reset);

/* Human-readable text for a status code (static storage). */
const char *bimamba_status_string(int status);

/* ABI version: bumps when a signature or layout above changes. */
int bimamba_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* BIMAMBA_H */

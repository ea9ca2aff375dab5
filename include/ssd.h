/*
 * ssd.h -- C ABI of the B200 (sm_100a) Mamba-2 selective-state (SSD) layer.
 *
 * The layer (Video-Ma2mba / VAMBA backbone; pith.science verdict record for
 * arXiv 2411.19460):
 *   v = silu(causal_conv1d_k4(u))        on the packed x|B|C stream
 *       (skeptic_critique.load_bearing_attack: "causal Conv1d", kernel 4)
 *   per head h:  h_t = exp(dt_t*A_h) h_{t-1} + dt_t * x_t B_t^T
 *                y_t = C_t^T h_t + D_h x_t
 *       (pith_extraction.core_discovery, Eq. (1) h_t = A_t h_{t-1} + B_t x_t,
 *        discretised per Mamba-2 head)
 *   h_ckpt[k] = state after (k+1)*s tokens
 *       (pith_extraction.key_machinery, "Algorithm 1" sequence checkpoint Sckpt)
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or retains them.  Strides are in ELEMENTS.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  The return value reports argument errors and launch
 *    failures detected on the host.  Errors detected on the device (a bounded
 *    wait that timed out) are latched in a per-device status word and read by
 *    ssd_sync_status().
 *  - Every call returns an ssd_status.  On error nothing is launched, and
 *    ssd_last_error_string() (thread-local) describes the failure.
 *  - The library computes everything in its own CUDA kernels; there is no CPU
 *    fallback.  Shapes the GPU kernels do not support return
 *    SSD_ERR_UNSUPPORTED.
 *  - dtype SSD_BF16: x/B/C, u, v, y and the conv tails are bfloat16; SSD_F32:
 *    they are float.  dt, A, D, conv weights/bias, h0, h_final and h_ckpt are
 *    always float (fp32 state).
 *  - Environment variables, read once per process at the first scan call
 *    (test and diagnostic hooks; leave them unset in production):
 *      SSD_WAIT_LIMIT_MS   bound of every device-side wait in milliseconds
 *                          (default 2000); a wait that runs out latches
 *                          SSD_ERR_TIMEOUT in the device status word.
 *      SSD_TEST_DROP_UNIT  index of one work unit (CTA) of the tensor-core
 *                          scan whose loads are never issued, so that its
 *                          waits run out (failure-detection test); it applies
 *                          to the first scan call of the process only.
 *      SSD_SCAN_PATH       "generic" forces the CUDA-core scan kernels.
 */
#ifndef SSD_H_
#define SSD_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *ssd_stream_t; /* same type as cudaStream_t */

typedef enum ssd_dtype { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype;

typedef enum ssd_status {
    SSD_OK = 0,
    SSD_ERR_NULL = 1,        /* a required pointer is NULL */
    SSD_ERR_SHAPE = 2,       /* inconsistent or out-of-range sizes */
    SSD_ERR_ALIGN = 3,       /* a pointer or row stride breaks 16-byte alignment */
    SSD_ERR_STRIDE = 4,      /* strides smaller than the rows they step over */
    SSD_ERR_DTYPE = 5,       /* unknown dtype code */
    SSD_ERR_UNSUPPORTED = 6, /* valid, but no GPU kernel for this shape */
    SSD_ERR_LAUNCH = 7,      /* CUDA launch or runtime error */
    SSD_ERR_TIMEOUT = 8,     /* a bounded device-side wait gave up (device status) */
    SSD_ERR_WORKSPACE = 9    /* workspace missing or smaller than required */
} ssd_status;

/*
 * ssd_conv_forward -- depthwise causal conv1d (kernel 4) + SiLU.
 * Defines: v[bi,t,c] = silu(bias[c] + sum_{k=0..3} w[c,k] * u[bi,t-3+k,c]),
 * silu(z) = z / (1 + exp(-z)); u at t < 0 is tail_in[bi, 3+t, c] (zeros when
 * tail_in is NULL).  tail_out[bi, r, c] = u at position L-3+r (from tail_in
 * when that position is negative): the conv buffer that, with the SSD state,
 * makes a resumed call exact (skeptic_critique.headline, desk_editor.letter).
 *   u        [b][L][C_ch], element (bi,t,c) at u[bi*u_batch_stride + t*u_row_stride + c]
 *   w        [C_ch][4] float; bias [C_ch] float or NULL (zero bias)
 *   tail_in  [b][3][C_ch] contiguous or NULL; tail_out same layout or NULL.
 *            tail_out may alias tail_in (it is written after all reads).
 *   v        [b][L][C_ch] output, strides like u; must not overlap u.
 * Requirements: C_ch a multiple of 8 (bf16) or 4 (f32); u, v, tails 16-byte
 * aligned and row/batch strides multiples of 16 bytes (SSD_ERR_ALIGN).
 */
SSD_API int ssd_conv_forward(const void *u, int64_t u_batch_stride, int64_t u_row_stride,
                     const float *w, const float *bias,
                     const void *tail_in, void *tail_out,
                     void *v, int64_t v_batch_stride, int64_t v_row_stride,
                     int b, int64_t L, int C_ch, int dtype, ssd_stream_t stream);

/*
 * Arguments of the selective scan (see ssd_scan_forward).
 *   x   element (bi,t,h,p) at x[bi*x_batch_stride + t*x_row_stride + h*P + p]
 *   B,C element (bi,t,g,n) at B[bi*B_batch_stride + t*B_row_stride + g*N + n]
 *       (x, B and C may be column slices of the conv output v)
 *   dt  [b][L][H] float, contiguous, > 0
 *   A   [H] float (A <= 0 expected; not checked), D [H] float or NULL (no skip)
 *   h0  [b][H][P][N] float or NULL (zero state); may alias h_final
 *   y   element (bi,t,h,p) at y[bi*y_batch_stride + t*y_row_stride + h*P + p]
 *   h_final [b][H][P][N] float or NULL
 *   h_ckpt  [b][floor(L/s)][H][P][N] float or NULL (no checkpoints written)
 *   s   checkpoint stride in tokens, a multiple of Q, or 0 (none)
 *   Q   chunk length: 32, 64 or 128
 *   workspace: device scratch of at least ssd_scan_workspace_size() bytes,
 *       256-byte aligned; NULL allowed when that size is 0.  Contents on
 *       entry are ignored; the call overwrites them.
 */
typedef struct ssd_scan_args {
    int dtype;
    int b;
    int64_t L;
    int H, P, N, G, Q;
    int64_t s;
    const void *x;
    int64_t x_batch_stride, x_row_stride;
    const void *B;
    int64_t B_batch_stride, B_row_stride;
    const void *C;
    int64_t C_batch_stride, C_row_stride;
    const float *dt;
    const float *A;
    const float *D;
    const float *h0;
    void *y;
    int64_t y_batch_stride, y_row_stride;
    float *h_final;
    float *h_ckpt;
    void *workspace;
    size_t workspace_bytes;
    /* dt as given, or dt_eff = clamp(f(dt + dt_bias[h]), dt_min, dt_max): dt_bias [H]
     * fp32 or NULL (none), f = softplus(v) = log(1 + e^v) when dt_softplus != 0 and
     * the identity otherwise, the clamp applied only when dt_max > 0.  A
     * zero-initialised struct leaves dt unchanged.  (The Mamba-2 block's
     * dt_bias + softplus, fused here; the pages give dt itself.) */
    const float *dt_bias;
    int dt_softplus;
    float dt_min, dt_max;
} ssd_scan_args;

/*
 * ssd_scan_forward -- chunked selective scan with state checkpoints.
 * Computes, for every batch row and head, the recurrence stated at the top
 * of this header from h0, writing y for every token, h_ckpt every s tokens
 * and h_final after the last token.  H must be a multiple of G; P and N in
 * {16, 32, 64, 128}; L >= 0 (L need not be a multiple of Q or s).
 */
SSD_API int ssd_scan_forward(const ssd_scan_args *args, ssd_stream_t stream);

/* Bytes of workspace ssd_scan_forward / ssd_stream_forward need for this shape
 * on the current device (the stripe plan depends on its SM count): the stripe
 * states, then room for the effective dt [b][L][H] fp32.  Calls that ask for
 * none of dt_bias / softplus / clamp need only the first part, which is 0 when
 * the sequence is a single stripe. */
SSD_API size_t ssd_scan_workspace_size(int b, int64_t L, int H, int P, int N, int Q);

/*
 * Arguments of one streamed segment (see ssd_stream_forward).  u is the
 * segment's pre-conv x|B|C stream [b][L][C_ch], C_ch = H*P + 2*G*N, channel
 * order x, then B, then C.  v receives the conv output (the scan reads its
 * column slices).  tail_in/h0 carry the previous segment's conv buffer and
 * state; tail_out/h_final receive this segment's (they may alias them).
 */
typedef struct ssd_stream_args {
    int dtype;
    int b;
    int64_t L;
    int H, P, N, G, Q;
    int64_t s;
    const void *u;
    int64_t u_batch_stride, u_row_stride;
    const float *conv_w;
    const float *conv_bias;
    const void *tail_in;
    void *tail_out;
    void *v;
    int64_t v_batch_stride, v_row_stride;
    const float *dt;
    const float *A;
    const float *D;
    const float *h0;
    void *y;
    int64_t y_batch_stride, y_row_stride;
    float *h_final;
    float *h_ckpt;
    void *workspace;
    size_t workspace_bytes;
    /* dt as given, or dt_eff = clamp(f(dt + dt_bias[h]), dt_min, dt_max): dt_bias [H]
     * fp32 or NULL (none), f = softplus(v) = log(1 + e^v) when dt_softplus != 0 and
     * the identity otherwise, the clamp applied only when dt_max > 0.  A
     * zero-initialised struct leaves dt unchanged.  (The Mamba-2 block's
     * dt_bias + softplus, fused here; the pages give dt itself.) */
    const float *dt_bias;
    int dt_softplus;
    float dt_min, dt_max;
    /* conv_ckpt [b][floor(L/s)][3][C_ch] (I/O dtype) or NULL: the conv buffer at every
     * checkpoint, conv_ckpt[bi,k,r,:] = u[bi,(k+1)*s-3+r,:] -- with h_ckpt[k] it is
     * what a cell's exact recompute needs (ssd_layer_backward). */
    void *conv_ckpt;
} ssd_stream_args;

/*
 * ssd_stream_forward -- one segment of a long stream: conv (tail_in ->
 * tail_out) then scan (h0 -> h_final, checkpoints every s tokens of this
 * segment).  Calling it on consecutive segments, each resumed from the
 * previous (h_final, tail_out), equals one call on the whole sequence
 * (sequence-axis checkpointing of pith_extraction.key_machinery, with the
 * conv buffer the skeptic_critique asks for).
 * On the tensor-core scan's shapes (bf16, P = 64, N = 128, Q = 128, heads in
 * pairs per group) with more than one stripe (ssd_scan_workspace_size > 0),
 * the conv of x runs inside the scan's first pass, which reads x's columns of
 * u and writes the conv output of x to v; a conv kernel covers only the B and
 * C channels.  Elsewhere one conv kernel writes all of v.  Either way v ends
 * up holding the whole conv output, bit for bit the same.
 * v may be NULL: the conv output then lives in the workspace, which must hold
 * ssd_stream_workspace_size() bytes instead of ssd_scan_workspace_size().
 * tail_out is written last, so it may alias tail_in.
 */
SSD_API int ssd_stream_forward(const ssd_stream_args *args, ssd_stream_t stream);

/* Bytes of workspace ssd_stream_forward needs when v is NULL (the scan's
 * workspace, then room for the conv output [b][L][C_ch]), for dtype SSD_F32
 * or SSD_BF16 on the current device. */
SSD_API size_t ssd_stream_workspace_size(int b, int64_t L, int H, int P, int N, int G, int Q, int dtype);

/*
 * Arguments of one decode step: a single new token of b independent streams
 * (online inference on a video consumed as one continuous stream at 1 FPS --
 * video-ma2mba-0.3b catalog page, "What is Video-Ma2mba?").  Per stream:
 *   u       [b][C_ch] this token's pre-conv x|B|C (I/O dtype), C_ch = H*P + 2*G*N,
 *           batch stride u_batch_stride elements, 16-byte aligned rows
 *   conv_w  [C_ch][4] fp32, conv_bias [C_ch] fp32 or NULL
 *   tail_in [b][3][C_ch] the three previous pre-conv tokens (oldest first), or
 *           NULL for zeros (the first token of a stream)
 *   tail_out[b][3][C_ch] receives [tail_in[1], tail_in[2], u]; may alias tail_in; NULL: not kept
 *   dt      [b][H] fp32 (positive), A [H] fp32, D [H] fp32 or NULL
 *   h_in    [b][H][P][N] fp32 state before the token, or NULL for zeros
 *   h_out   [b][H][P][N] fp32 state after the token; may alias h_in
 *   y       [b][H*P] (I/O dtype), batch stride y_batch_stride elements
 * P, N in {16, 32, 64, 128}; H % G == 0.
 */
typedef struct ssd_decode_args {
    int dtype;
    int b;
    int H, P, N, G;
    const void *u;
    int64_t u_batch_stride;
    const float *conv_w;
    const float *conv_bias;
    const void *tail_in;
    void *tail_out;
    const float *dt;
    const float *A;
    const float *D;
    const float *h_in;
    float *h_out;
    void *y;
    int64_t y_batch_stride;
    /* dt as given, or dt_eff = clamp(f(dt + dt_bias[h]), dt_min, dt_max): dt_bias [H]
     * fp32 or NULL (none), f = softplus(v) = log(1 + e^v) when dt_softplus != 0 and
     * the identity otherwise, the clamp applied only when dt_max > 0.  A
     * zero-initialised struct leaves dt unchanged.  (The Mamba-2 block's
     * dt_bias + softplus, fused here; the pages give dt itself.) */
    const float *dt_bias;
    int dt_softplus;
    float dt_min, dt_max;
} ssd_decode_args;

/*
 * ssd_decode_step -- the layer on one token: v = silu(causal conv4 of
 * (tail, u)), then h = exp(dt*A) h + dt x B^T and y = C h + D x per head
 * (Eq. (1) of the pages with the discretisation of the selective scan).
 * Equal, up to rounding, to ssd_stream_forward on a one-token segment; a
 * sequence of decode steps equals one call on the whole sequence.
 * Asynchronous on `stream`; status as for the other entry points.
 */
SSD_API int ssd_decode_step(const ssd_decode_args *args, ssd_stream_t stream);

/*
 * Arguments of the backward pass of the scan (see ssd_scan_backward).
 *   dtype, b, L, H, P, N, G, x, B, C, dt, A, D, h0: as given to the forward
 *           call whose gradients are wanted (x, B, C laid out and aligned as
 *           for ssd_scan_forward).  dt is the step size the scan USED: when
 *           the forward applied dt_bias / softplus / a clamp, pass the
 *           effective dt_eff = clamp(f(dt + dt_bias)) (the forward keeps it only
 *           in its workspace), and ddt is then dLoss/d(dt_eff): the chain
 *           rule through the bias, softplus and clamp is the caller's
 *           elementwise step.
 *   h_ckpt  [b][floor(L/s)][H][P][N] float: that call's checkpoints, s their
 *           stride (a multiple of 64).  Or NULL (s ignored): the states are
 *           then rebuilt from h0 over the whole sequence.
 *   dy      element (bi,t,h,p) at dy[bi*dy_batch_stride + t*dy_row_stride + h*P + p],
 *           I/O dtype, 16-byte aligned rows: dLoss/dy.
 *   dh_final [b][H][P][N] float or NULL (zero): dLoss/dh_final.
 * Outputs, float, contiguous, every element written:
 *   dx [b][L][H][P]; dB, dC [b][L][G][N] (summed over the heads of each
 *   group); ddt [b][L][H]; dA [H]; dD [H] or NULL (both summed over the batch
 *   rows); dh0 [b][H][P][N] or NULL.  They must not overlap the inputs.
 *   workspace: at least ssd_scan_backward_workspace_size() bytes, 256-byte
 *   aligned; contents on entry are ignored.
 */
typedef struct ssd_scan_bwd_args {
    int dtype;
    int b;
    int64_t L;
    int H, P, N, G;
    int64_t s;
    const void *x;
    int64_t x_batch_stride, x_row_stride;
    const void *B;
    int64_t B_batch_stride, B_row_stride;
    const void *C;
    int64_t C_batch_stride, C_row_stride;
    const float *dt;
    const float *A;
    const float *D;
    const float *h0;
    const float *h_ckpt;
    const void *dy;
    int64_t dy_batch_stride, dy_row_stride;
    const float *dh_final;
    float *dx, *dB, *dC, *ddt, *dA, *dD, *dh0;
    void *workspace;
    size_t workspace_bytes;
} ssd_scan_bwd_args;

/*
 * ssd_scan_backward -- gradients of a scalar loss through the scan, given
 * dLoss/dy and dLoss/dh_final: the reverse mode of the recurrence at the top
 * of this header.  With checkpoints, the states of each cell of s tokens are
 * rebuilt from the checkpoint that starts it (h0 for the first cell), and no
 * state is carried across cells: the grid-cell recompute of MA-GC
 * (pith_extraction.key_machinery, "Algorithm 1") on the sequence axis, whose
 * gradients must match plain backpropagation (skeptic_critique.concrete_test).
 * All arithmetic is fp32 on CUDA cores.  Asynchronous on `stream`.
 */
SSD_API int ssd_scan_backward(const ssd_scan_bwd_args *args, ssd_stream_t stream);

/* Bytes of workspace ssd_scan_backward needs: per 64-token chunk and head two
 * P x N fp32 states, and per token and head two N-vectors of fp32. */
SSD_API size_t ssd_scan_backward_workspace_size(int b, int64_t L, int H, int P, int N);

/*
 * Arguments of the backward pass of the whole layer (see ssd_layer_backward).
 *   dtype, b, L, H, P, N, G, u (+ strides), conv_w, conv_bias, tail_in, dt, A,
 *   D, h0: as given to the forward (ssd_stream_forward; dt is the step size the
 *   scan used, see ssd_scan_bwd_args).
 *   h_ckpt [b][floor(L/s)][H][P][N] float and conv_ckpt [b][floor(L/s)][3][C_ch]
 *           (I/O dtype): the forward's state checkpoints and conv buffers, s a
 *           multiple of 64.  Both or neither: without them the states and the
 *           conv are rebuilt from h0 and tail_in over the whole sequence.
 *   dy      dLoss/dy laid out as for ssd_scan_bwd_args; dh_final [b][H][P][N]
 *           float or NULL; dtail_out [b][3][C_ch] float or NULL: dLoss/d(tail_out).
 * Outputs, float, contiguous, every element written:
 *   du [b][L][C_ch] (row-major, C_ch = H*P + 2*G*N); dtail_in [b][3][C_ch] or
 *   NULL; dconv_w [C_ch][4]; dconv_bias [C_ch] or NULL; ddt [b][L][H]; dA [H];
 *   dD [H] or NULL; dh0 [b][H][P][N] or NULL.  They must not overlap the inputs.
 *   workspace: at least ssd_layer_backward_workspace_size() bytes, 256-byte
 *   aligned; contents on entry are ignored.
 */
typedef struct ssd_layer_bwd_args {
    int dtype;
    int b;
    int64_t L;
    int H, P, N, G;
    int64_t s;
    const void *u;
    int64_t u_batch_stride, u_row_stride;
    const float *conv_w;
    const float *conv_bias;
    const void *tail_in;
    const void *conv_ckpt;
    const float *dt;
    const float *A;
    const float *D;
    const float *h0;
    const float *h_ckpt;
    const void *dy;
    int64_t dy_batch_stride, dy_row_stride;
    const float *dh_final;
    const float *dtail_out;
    float *du, *dtail_in, *dconv_w, *dconv_bias, *ddt, *dA, *dD, *dh0;
    void *workspace;
    size_t workspace_bytes;
} ssd_layer_bwd_args;

/*
 * ssd_layer_backward -- gradients of a scalar loss through the whole layer
 * (conv1d + SiLU, then the scan), given dLoss/dy, dLoss/dh_final and
 * dLoss/d(tail_out).  With checkpoints, each cell of s tokens is rebuilt on its
 * own: its conv output from ITS OWN rows of u and the 3-row conv buffer stored
 * with the checkpoint that starts it (tail_in for the first cell), its states
 * from that checkpoint's state (h0 for the first cell) -- MA-GC's grid-cell
 * recompute (pith_extraction.key_machinery, "Algorithm 1"), exact because the
 * conv buffer is stored along with the SSD state (skeptic_critique.headline).
 * Then the scan's reverse mode (as ssd_scan_backward) and the conv's:
 *   dz = dv silu'(z), du[t'] = sum_j w[:,3-j] dz[t'+j], dw[:,k] = sum_t dz[t] u[t-3+k],
 *   dbias = sum_t dz[t]; the gradient of a cell's conv buffer is that of the
 *   rows of u it copies (of tail_in for the first cell).
 * The rounding of the conv output to the I/O dtype is taken as the identity.
 * All arithmetic is fp32 on CUDA cores.  Asynchronous on `stream`.
 */
SSD_API int ssd_layer_backward(const ssd_layer_bwd_args *args, ssd_stream_t stream);

/* Bytes of workspace ssd_layer_backward needs: the rebuilt conv output, the
 * conv output's gradients (fp32), per 64-token block partial sums of the conv
 * weight gradients, and the scan backward's own workspace. */
SSD_API size_t ssd_layer_backward_workspace_size(int b, int64_t L, int H, int P, int N, int G, int dtype);

/*
 * ssd_gated_rmsnorm_forward -- the output norm of the Mamba-2 block on the
 * layer's y (the pages end at y; this is the plainest reading of the block
 * around it: normalise after gating, over groups of consecutive channels):
 *   v = y * silu(z),  silu(z) = z / (1 + exp(-z))
 *   out[r,c] = v[r,c] / sqrt(mean_{c' in group(c)} v[r,c']^2 + eps) * weight[c]
 *   y, z, out  rows r = 0..rows-1 of d channels, element (r,c) at ptr[r*row_stride + c],
 *              I/O dtype; a [b][L][d] tensor is rows = b*L when its batches
 *              are consecutive rows.  out may alias y (same stride).
 *   weight     [d] float;  eps >= 0;  group_size: channels per group, a
 *              multiple of 8 dividing d, or 0 for one group of all d.
 * d a multiple of 8, at most 8192; pointers and row strides 16-byte aligned.
 * Asynchronous on `stream`.
 */
SSD_API int ssd_gated_rmsnorm_forward(const void *y, int64_t y_row_stride, const void *z, int64_t z_row_stride,
                                      const float *weight, float eps, int group_size,
                                      void *out, int64_t out_row_stride, int64_t rows, int d, int dtype,
                                      ssd_stream_t stream);

/*
 * ssd_scan_forward_static_scratch -- ssd_scan_forward for callers that cannot
 * allocate device memory.  (The pages have no counterpart: this is a
 * deployment aid of this library, not part of the layer they describe.)
 *
 * ssd_scan_forward needs a caller-allocated `workspace`.  Callers that may not
 * call cudaMalloc (a memory pool that forbids new allocations, plugin code
 * that is handed only its input and output buffers, code that must not risk
 * the device synchronisation or out-of-memory failure an allocation can
 * bring) use this variant instead: the scratch comes from a fixed 80 MiB array
 * compiled into the library.  The `workspace` fields of `args` are ignored;
 * all other arguments, results and errors are those of ssd_scan_forward.
 *  - Every GPU that loads the library holds those 80 MiB until process exit.
 *  - A shape whose ssd_scan_workspace_size() exceeds 80 MiB is rejected with
 *    SSD_ERR_WORKSPACE before anything is launched.
 *  - The first call on each device looks up the array's device address, with
 *    that device current; make that first call before any stream capture.
 *  - All calls on a device share the array, which keeps the last call's
 *    contents (each call writes every element it reads, so nothing needs to
 *    start at zero).  Calls whose kernels overlap on the GPU race on it:
 *    serialise them (one stream, or synchronise between streams).
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
SSD_API int ssd_scan_forward_static_scratch(const ssd_scan_args *args, ssd_stream_t stream);

/*
 * ssd_sync_status -- synchronise `stream`, then return SSD_ERR_LAUNCH if the
 * CUDA runtime reports an error, else the device status word latched by
 * this library's kernels on the current device (SSD_OK or SSD_ERR_TIMEOUT),
 * which it then clears.
 */
SSD_API int ssd_sync_status(ssd_stream_t stream);

/*
 * Per-kernel timing (tracing).  Between ssd_profile_begin() and
 * ssd_profile_end(), every kernel this library launches from the calling
 * host thread is bracketed by two CUDA events recorded on the launch stream.
 * ssd_profile_end() waits for those events and fills `out` (up to
 * `capacity` entries; *count receives the number of distinct kernels) with
 * the launch count and the summed event time of each kernel, by name.  The
 * names are static strings owned by the library.  Profiling adds two event
 * records per launch; time the workload without it when the total matters.
 */
typedef struct ssd_kernel_stat {
    const char *name;
    int64_t launches;
    double total_ms;
} ssd_kernel_stat;

SSD_API int ssd_profile_begin(void);
SSD_API int ssd_profile_end(ssd_kernel_stat *out, int capacity, int *count);

/* Description of the last error on this host thread ("" if none). */
SSD_API const char *ssd_last_error_string(void);

/* ABI version: major*10000 + minor*100 + patch. */
SSD_API int ssd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H_ */

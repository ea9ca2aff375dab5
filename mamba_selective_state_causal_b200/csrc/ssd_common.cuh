// ssd_common.cuh -- types and small device helpers shared by the SSD kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// Device status codes latched by kernels (mirrors ssd_status in include/ssd.h).
enum : unsigned int { kDevOk = 0u, kDevUnsupported = 6u, kDevTimeout = 8u };

// Everything a scan kernel needs, passed by value.
struct ScanParams {
    int b;
    int64_t L;
    int H, P, N, G, Q;
    int64_t s;
    const void *x;
    int64_t xbs, xrs;
    const void *B;
    int64_t Bbs, Brs;
    const void *C;
    int64_t Cbs, Crs;
    const float *dt;
    const float *A;
    const float *D;
    const float *h0;
    void *y;
    int64_t ybs, yrs;
    float *h_final;
    float *h_ckpt;
    // stripe decomposition of the sequence (see make_plan)
    int64_t T;          // stripe length in tokens, a multiple of Q
    int64_t ns;         // number of stripes = ceil(L / T)
    float *ws_S;        // [b][ns][H][P][N] stripe state from a zero start
    float *ws_hin;      // [b][ns][H][P][N] exact state entering each stripe
    float *ws_dA;       // [b][ns][H] sum of dt*A over the stripe
    unsigned int *status;
    // bounded waits give up after this many nanoseconds (SSD_WAIT_LIMIT_MS)
    uint64_t wait_limit_ns;
    // failure-detection test hook (SSD_TEST_DROP_UNIT): the work unit whose
    // loads are never issued, so that its waits run out; -1 = none
    int64_t test_drop_unit;
    // the dt surroundings (dt_effective): applied by a pre-pass into the workspace, so the
    // scan kernels themselves always read plain dt
    const float *dt_bias;
    int dt_softplus;
    float dt_min, dt_max;
    // the conv of x fused into pass A (ssd_stream_forward on the tensor-core shapes):
    // pass A reads x's columns of the conv input u, turns them into
    // silu(conv(u)) in shared memory and writes that x to conv_v (which the
    // output pass then reads as x); NULL conv_w means x is given
    const void *conv_u;
    int64_t conv_ubs, conv_urs;
    void *conv_v;
    int64_t conv_vbs, conv_vrs;
    const float *conv_w;        // [C_ch][4]
    const float *conv_bias;     // [C_ch] or NULL
    const void *conv_tail;      // [b][3][C_ch] (the rows before token 0) or NULL (zeros)
    int conv_cch;
};

struct ConvParams {
    const void *u;
    int64_t ubs, urs;
    const float *w;
    const float *bias;
    const void *tail_in;
    void *tail_out;
    void *v;
    int64_t vbs, vrs;
    int b;
    int64_t L;
    int C_ch;
    int64_t tail_rs;    // row stride of tail_in / tail_out (C_ch, or wider for a column slice)
};

// One decode step (decode.cu).
struct DecodeParams {
    int b, H, P, N, G;
    const void *u;
    int64_t ubs;
    const float *w;
    const float *bias;
    const void *tail_in;
    void *tail_out;
    const float *dt;
    const float *A;
    const float *D;
    const float *h_in;
    float *h_out;
    void *y;
    int64_t ybs;
    const float *dt_bias;
    int dt_softplus;
    float dt_min, dt_max;
};

// The backward pass of the scan (scan_bwd.cu).
struct BwdParams {
    int b;
    int64_t L;
    int H, P, N, G;
    int64_t s, n_ckpt;
    int64_t nch;            // chunks of kQb = 64 tokens
    int64_t cell_chunks;    // chunks per recompute cell (s / 64, or nch without checkpoints)
    const void *x;
    int64_t xbs, xrs;
    const void *B;
    int64_t Bbs, Brs;
    const void *C;
    int64_t Cbs, Crs;
    const void *dy;
    int64_t dybs, dyrs;
    const float *dt;
    const float *A;
    const float *D;
    const float *h0;
    const float *h_ckpt;
    const float *dh_final;
    float *dx, *dB, *dC, *ddt, *dA, *dD, *dh0;
    float *ws_h;            // [b][H][nch][P][N] S_c, then the state entering chunk c
    float *ws_g;            // [b][H][nch][P][N] Gl_c, then the adjoint leaving chunk c
    float *ws_lam;          // [b][H][nch] sum of dt*A over the chunk
    float *ws_dBh, *ws_dCh; // [b][L][H][N] per-head dB and dC
    float *ws_pA, *ws_pD;   // [b][H][nch] per-chunk dA and dD
    int stage_adjoint;      // set by the launcher: copy Gam and h_prev into shared memory
    unsigned int *status;   // device status word (a bounded wait that gave up)
    uint64_t wait_limit_ns; // bound of every device-side wait
};

// The conv part of the layer's backward pass (conv1d_silu.cu, layer_bwd.cu): the
// conv input u and its per-cell conv buffers, and the gradients of the conv output.
struct ConvBwdParams {
    int b;
    int64_t L;
    int C_ch, HP, GN;           // channels: x (HP), then B (GN), then C (GN)
    const void *u;
    int64_t ubs, urs;
    const float *w;
    const float *bias;
    const void *tail_in;        // [b][3][C_ch] buffer of the first cell, or NULL (zeros)
    const void *conv_ckpt;      // [b][n_ckpt][3][C_ch] buffer of cell k at k-1, or NULL (one cell)
    int64_t s, n_ckpt;          // cell length and number of checkpoints (cells when conv_ckpt is set)
    void *v;                    // recomputed conv output [b][L][C_ch] (I/O dtype, contiguous)
    const float *dx, *dB, *dC;  // [b][L][HP], [b][L][GN], [b][L][GN] gradients of the conv output
    const float *dtail_out;     // [b][3][C_ch] or NULL
    float *du;                  // [b][L][C_ch]
    float *dtail_in;            // [b][3][C_ch] or NULL
    float *ws_dw, *ws_dbias;    // per (batch row, token block) partial sums [..][C_ch][4], [..][C_ch]
    float *dw, *dbias;          // [C_ch][4], [C_ch] (dbias may be NULL)
};

// The gated RMS norm of the layer output (gated_norm.cu).
struct NormParams {
    const void *y;
    int64_t yrs;
    const void *z;
    int64_t zrs;
    const float *w;
    float eps;
    int group;
    void *out;
    int64_t ors;
    int64_t rows;
    int d;
};

// The step size a kernel uses for a raw dt value of head h: dt + dt_bias[h]
// (bias optional), through softplus(v) = log(1 + e^v) when asked (v itself
// above 20, where the two agree in fp32), clamped to [dt_min, dt_max] when
// dt_max > 0.  With no bias, no softplus and dt_max <= 0 it is dt unchanged.
__device__ __forceinline__ float dt_effective(float raw, const float *bias, int h, int softplus, float lo,
                                              float hi)
{
    float v = bias ? raw + bias[h] : raw;
    if (softplus) v = v > 20.0f ? v : log1pf(__expf(v));
    if (hi > 0.0f) v = fminf(fmaxf(v, lo), hi);
    return v;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&r);
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v)
{
    return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v)
{
    return __float2bfloat16_rn(v);
}

// Kernel timing hooks (ssd_api.cu): no-ops unless ssd_profile_begin() is active
// on the calling thread.
enum KernelId : int {
    kKConv = 0, kKConvTail, kKStateTc, kKChain, kKOutputTc, kKStateGeneric, kKOutputGeneric, kKDecode,
    kKBwdSummary, kKBwdChain, kKBwdGrad, kKBwdReduce, kKGatedNorm, kKConvCells, kKConvCkpt, kKConvBwd,
    kKBwdAdjoint, kKCount
};
void prof_begin(cudaStream_t st, int id);
void prof_end(cudaStream_t st, int id);

// Launchers (defined in the .cu files).
int launch_conv(const ConvParams &p, int dtype, cudaStream_t st);
int launch_conv_cells(const ConvBwdParams &p, int dtype, cudaStream_t st);
int launch_conv_ckpt(const void *u, int64_t ubs, int64_t urs, void *conv_ckpt, int b, int64_t L, int C_ch,
                     int64_t s, int dtype, cudaStream_t st);
int launch_conv_backward(const ConvBwdParams &p, int dtype, cudaStream_t st);
int64_t conv_bwd_blocks(int64_t L);
int launch_decode(const DecodeParams &p, int dtype, cudaStream_t st);
int launch_scan_generic(const ScanParams &p, int dtype, cudaStream_t st);
int launch_dt_prepare(const ScanParams &p, float *out, cudaStream_t st);
bool tc_scan_supported(const ScanParams &p, int dtype);
bool tc_scan_shape(int dtype, int H, int P, int N, int G, int Q);
int launch_conv_tail(const ConvParams &p, int dtype, cudaStream_t st);
int launch_scan_backward(const BwdParams &p, int dtype, cudaStream_t st);
size_t bwd_grad_smem_bytes(int P, int N);
int launch_gated_norm(const NormParams &p, int dtype, cudaStream_t st);
int launch_scan_tc(const ScanParams &p, cudaStream_t st);
}  // namespace ssd

// scan_generic.cu -- chunked selective scan on CUDA cores (fp32 math).
//
// The recurrence of the Mamba-2 head (pith.science verdict for arXiv
// 2411.19460, pith_extraction.core_discovery, Eq. (1), discretised as
// A_t = exp(dt_t*A_h), input dt_t * x_t B_t^T, output C_t^T h_t + D_h x_t) is
// evaluated chunk by chunk.  Inside a chunk of Q tokens with chunk-local
// cumulative log-decay cs_i = sum_{k<=i} dt_k*A:
//   y_i   = sum_{j<=i} exp(cs_i - cs_j) dt_j (C_i . B_j) x_j     (intra-chunk)
//         + exp(cs_i) C_i h_prev^T                              (carried state)
//         + D x_i
//   h_new = exp(cs_last) h_prev + sum_j dt_j exp(cs_last - cs_j) x_j B_j^T
// Only non-positive differences cs_i - cs_j (i >= j) are exponentiated, so
// nothing overflows and underflow to 0 is the exact limit.
//
// The sequence is cut into stripes of T tokens (a multiple of Q):
//   pass A  (stripe, head): the stripe's end state from a zero start, and
//           its total log-decay;
//   chain   (head, state element): h_in[k+1] = exp(dA_k) h_in[k] + S_k, from h0;
//   pass C  (stripe, head): walk the chunks from h_in[k], emit y, the
//           checkpoints that fall in the stripe (state after every s tokens,
//           "Algorithm 1" Sckpt of pith_extraction.key_machinery) and h_final.
// This file is the general path: any supported P, N, Q and both dtypes.
#include <algorithm>

#include "ssd_common.cuh"

namespace ssd {
int launch_chain(const ScanParams &p, cudaStream_t st);
namespace {

constexpr int kThreads = 256;
constexpr int kMaxEPT = 64;     // state elements per thread (P*N <= 16384)
constexpr int kRowBlock = 32;   // rows of the masked intra-chunk matrix kept in smem

template <typename T>
__device__ __forceinline__ void load_tile(float *dst, const T *src, int64_t row_stride,
                                          int rows_valid, int rows, int cols)
{
    for (int i = threadIdx.x; i < rows * cols; i += blockDim.x) {
        const int r = i / cols, c = i % cols;
        dst[i] = r < rows_valid ? to_f32<T>(src[(int64_t)r * row_stride + c]) : 0.0f;
    }
}

// chunk-local inclusive cumsum of dt*A (serial: Q <= 128, deterministic)
__device__ __forceinline__ void chunk_cumsum(const float *dts, float *cs, int Q, float A)
{
    if (threadIdx.x == 0) {
        float acc = 0.0f;
        for (int i = 0; i < Q; ++i) { acc += dts[i] * A; cs[i] = acc; }
    }
}

// ---------------------------------------------------------------- pass A
template <typename T>
__global__ void __launch_bounds__(kThreads) stripe_state_kernel(ScanParams p)
{
    extern __shared__ float sm[];
    const int k = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    const int P = p.P, N = p.N, Q = p.Q;
    const int g = (int)((int64_t)h * p.G / p.H);
    float *xs = sm;                 // [Q][P]
    float *Bs = xs + Q * P;         // [Q][N]
    float *dts = Bs + Q * N;        // [Q]
    float *cs = dts + Q;            // [Q]
    float *wts = cs + Q;            // [Q]

    const int PN = P * N;
    const int ept = (PN + kThreads - 1) / kThreads;
    float acc[kMaxEPT];
#pragma unroll
    for (int e = 0; e < kMaxEPT; ++e) acc[e] = 0.0f;
    const float A = p.A[h];
    float dA = 0.0f;

    const int64_t s0 = (int64_t)k * p.T;
    const int64_t s1 = min(p.L, s0 + p.T);
    const T *xb = reinterpret_cast<const T *>(p.x) + bi * p.xbs + (int64_t)h * P;
    const T *Bb = reinterpret_cast<const T *>(p.B) + bi * p.Bbs + (int64_t)g * N;
    for (int64_t c0 = s0; c0 < s1; c0 += Q) {
        const int qv = (int)min((int64_t)Q, s1 - c0);
        __syncthreads();
        load_tile<T>(xs, xb + c0 * p.xrs, p.xrs, qv, Q, P);
        load_tile<T>(Bs, Bb + c0 * p.Brs, p.Brs, qv, Q, N);
        for (int i = threadIdx.x; i < Q; i += blockDim.x)
            dts[i] = i < qv ? p.dt[((int64_t)bi * p.L + c0 + i) * p.H + h] : 0.0f;
        __syncthreads();
        chunk_cumsum(dts, cs, Q, A);
        __syncthreads();
        const float tot = cs[Q - 1];
        for (int i = threadIdx.x; i < Q; i += blockDim.x) wts[i] = dts[i] * expf(tot - cs[i]);
        __syncthreads();
        const float dec = expf(tot);
        dA += tot;
#pragma unroll
        for (int e = 0; e < kMaxEPT; ++e) {
            if (e < ept) {
                const int idx = threadIdx.x + e * kThreads;
                if (idx < PN) {
                    const int pp = idx / N, nn = idx % N;
                    float s = 0.0f;
                    for (int j = 0; j < Q; ++j) s = fmaf(wts[j] * xs[j * P + pp], Bs[j * N + nn], s);
                    acc[e] = fmaf(dec, acc[e], s);
                }
            }
        }
    }
    float *dst = p.ws_S + (((int64_t)bi * p.ns + k) * p.H + h) * PN;
#pragma unroll
    for (int e = 0; e < kMaxEPT; ++e) {
        if (e < ept) {
            const int idx = threadIdx.x + e * kThreads;
            if (idx < PN) dst[idx] = acc[e];
        }
    }
    if (threadIdx.x == 0) p.ws_dA[((int64_t)bi * p.ns + k) * p.H + h] = dA;
}

// ---------------------------------------------------------------- chain
__global__ void __launch_bounds__(kThreads) stripe_chain_kernel(ScanParams p)
{
    const int PN = p.P * p.N;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const int h = blockIdx.y, bi = blockIdx.z;
    if (e >= PN) return;
    float st = p.h0 ? p.h0[((int64_t)bi * p.H + h) * PN + e] : 0.0f;
    for (int64_t k = 0; k < p.ns; ++k) {
        const int64_t base = ((int64_t)bi * p.ns + k) * p.H + h;
        p.ws_hin[base * PN + e] = st;
        st = fmaf(expf(p.ws_dA[base]), st, p.ws_S[base * PN + e]);
    }
}

// ---------------------------------------------------------------- pass C
template <typename T>
__global__ void __launch_bounds__(kThreads) chunk_output_kernel(ScanParams p)
{
    extern __shared__ float sm[];
    const int k = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    const int P = p.P, N = p.N, Q = p.Q;
    const int PN = P * N;
    const int g = (int)((int64_t)h * p.G / p.H);
    float *xs = sm;                   // [Q][P]
    float *Bs = xs + Q * P;           // [Q][N]
    float *Cs = Bs + Q * N;           // [Q][N]
    float *hs = Cs + Q * N;           // [P][N] running state
    float *Mr = hs + PN;              // [kRowBlock][Q]
    float *dts = Mr + kRowBlock * Q;  // [Q]
    float *cs = dts + Q;              // [Q]
    float *wts = cs + Q;              // [Q]

    // state entering this stripe
    const float *hin = (k == 0) ? (p.h0 ? p.h0 + ((int64_t)bi * p.H + h) * PN : nullptr)
                                : p.ws_hin + (((int64_t)bi * p.ns + k) * p.H + h) * PN;
    for (int i = threadIdx.x; i < PN; i += blockDim.x) hs[i] = hin ? hin[i] : 0.0f;

    const float A = p.A[h];
    const float Dh = p.D ? p.D[h] : 0.0f;
    const int64_t n_ckpt = p.s > 0 ? p.L / p.s : 0;
    const int64_t s0 = (int64_t)k * p.T;
    const int64_t s1 = min(p.L, s0 + p.T);
    const T *xb = reinterpret_cast<const T *>(p.x) + bi * p.xbs + (int64_t)h * P;
    const T *Bb = reinterpret_cast<const T *>(p.B) + bi * p.Bbs + (int64_t)g * N;
    const T *Cb = reinterpret_cast<const T *>(p.C) + bi * p.Cbs + (int64_t)g * N;
    T *yb = reinterpret_cast<T *>(p.y) + bi * p.ybs + (int64_t)h * P;

    for (int64_t c0 = s0; c0 < s1; c0 += Q) {
        const int qv = (int)min((int64_t)Q, s1 - c0);
        __syncthreads();
        load_tile<T>(xs, xb + c0 * p.xrs, p.xrs, qv, Q, P);
        load_tile<T>(Bs, Bb + c0 * p.Brs, p.Brs, qv, Q, N);
        load_tile<T>(Cs, Cb + c0 * p.Crs, p.Crs, qv, Q, N);
        for (int i = threadIdx.x; i < Q; i += blockDim.x)
            dts[i] = i < qv ? p.dt[((int64_t)bi * p.L + c0 + i) * p.H + h] : 0.0f;
        __syncthreads();
        chunk_cumsum(dts, cs, Q, A);
        __syncthreads();
        const float tot = cs[Q - 1];
        for (int i = threadIdx.x; i < Q; i += blockDim.x) wts[i] = dts[i] * expf(tot - cs[i]);

        // outputs, kRowBlock rows at a time
        for (int r0 = 0; r0 < qv; r0 += kRowBlock) {
            const int rb = min(kRowBlock, qv - r0);
            __syncthreads();
            for (int idx = threadIdx.x; idx < rb * Q; idx += blockDim.x) {
                const int ii = idx / Q, j = idx % Q, i = r0 + ii;
                float m = 0.0f;
                if (j <= i) {
                    float dot = 0.0f;
                    for (int n = 0; n < N; ++n) dot = fmaf(Cs[i * N + n], Bs[j * N + n], dot);
                    m = dot * expf(cs[i] - cs[j]) * dts[j];
                }
                Mr[idx] = m;
            }
            __syncthreads();
            for (int idx = threadIdx.x; idx < rb * P; idx += blockDim.x) {
                const int ii = idx / P, pp = idx % P, i = r0 + ii;
                float diag = 0.0f;
                for (int j = 0; j <= i; ++j) diag = fmaf(Mr[ii * Q + j], xs[j * P + pp], diag);
                float off = 0.0f;
                for (int n = 0; n < N; ++n) off = fmaf(Cs[i * N + n], hs[pp * N + n], off);
                const float yv = diag + expf(cs[i]) * off + Dh * xs[i * P + pp];
                yb[(c0 + i) * p.yrs + pp] = from_f32<T>(yv);
            }
        }
        __syncthreads();
        // state update
        const float dec = expf(tot);
        for (int idx = threadIdx.x; idx < PN; idx += blockDim.x) {
            const int pp = idx / N, nn = idx % N;
            float s = 0.0f;
            for (int j = 0; j < qv; ++j) s = fmaf(wts[j] * xs[j * P + pp], Bs[j * N + nn], s);
            hs[idx] = fmaf(dec, hs[idx], s);
        }
        __syncthreads();
        const int64_t t_end = c0 + qv;
        if (p.h_ckpt && p.s > 0 && qv == Q && t_end % p.s == 0) {
            const int64_t kk = t_end / p.s - 1;
            if (kk < n_ckpt) {
                float *dst = p.h_ckpt + (((int64_t)bi * n_ckpt + kk) * p.H + h) * PN;
                for (int i = threadIdx.x; i < PN; i += blockDim.x) dst[i] = hs[i];
            }
        }
    }
    if (p.h_final && s1 == p.L) {
        __syncthreads();
        float *dst = p.h_final + ((int64_t)bi * p.H + h) * PN;
        for (int i = threadIdx.x; i < PN; i += blockDim.x) dst[i] = hs[i];
    }
}

template <typename T>
int launch_t(const ScanParams &p, cudaStream_t st)
{
    const int P = p.P, N = p.N, Q = p.Q;
    const size_t smA = sizeof(float) * ((size_t)Q * (P + N) + 3 * Q);
    const size_t smC = sizeof(float) * ((size_t)Q * (P + 2 * N) + (size_t)P * N + kRowBlock * Q + 3 * Q);
    if (smC > 227 * 1024 || smA > 227 * 1024) return 6;
    if (cudaFuncSetAttribute(stripe_state_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smA) != cudaSuccess) return 7;
    if (cudaFuncSetAttribute(chunk_output_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smC) != cudaSuccess) return 7;
    if (p.ns > 65535 || p.H > 65535 || p.b > 65535) return 6;
    const dim3 grid((unsigned)p.ns, (unsigned)p.H, (unsigned)p.b);
    if (p.ns > 1) {
        prof_begin(st, kKStateGeneric);
        stripe_state_kernel<T><<<grid, kThreads, smA, st>>>(p);
        prof_end(st, kKStateGeneric);
        const int rc = launch_chain(p, st);
        if (rc) return rc;
    }
    prof_begin(st, kKOutputGeneric);
    chunk_output_kernel<T><<<grid, kThreads, smC, st>>>(p);
    prof_end(st, kKOutputGeneric);
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

// dt_eff[b][L][H] = dt_effective(dt) for the scan kernels, which then read it as plain dt
__global__ void dt_prepare_kernel(ScanParams p, float *out)
{
    const int64_t n = (int64_t)p.b * p.L * p.H;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = dt_effective(p.dt[i], p.dt_bias, (int)(i % p.H), p.dt_softplus, p.dt_min, p.dt_max);
}

}  // namespace

int launch_chain(const ScanParams &p, cudaStream_t st)
{
    const dim3 g((unsigned)((p.P * p.N + kThreads - 1) / kThreads), (unsigned)p.H, (unsigned)p.b);
    prof_begin(st, kKChain);
    stripe_chain_kernel<<<g, kThreads, 0, st>>>(p);
    prof_end(st, kKChain);
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

int launch_scan_generic(const ScanParams &p, int dtype, cudaStream_t st)
{
    if (p.P * p.N > kThreads * kMaxEPT) return 6;
    return dtype == 1 ? launch_t<__nv_bfloat16>(p, st) : launch_t<float>(p, st);
}

int launch_dt_prepare(const ScanParams &p, float *out, cudaStream_t st)
{
    const int64_t n = (int64_t)p.b * p.L * p.H;
    if (n > 0) {
        const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 16);
        dt_prepare_kernel<<<(unsigned)blocks, 256, 0, st>>>(p, out);
    }
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

}  // namespace ssd

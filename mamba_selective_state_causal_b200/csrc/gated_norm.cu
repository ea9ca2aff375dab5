// gated_norm.cu -- the Mamba-2 block's output norm on the layer's y:
//   v = y * silu(z),   out = v / sqrt(mean over the channel group of v^2 + eps) * w
// The pages end at y; this is the plainest reading of the block around it
// (normalise after gating, groups of `group` consecutive channels).
//
// One CTA per row (grid-stride over rows), one thread per 8 channels: a row of
// y and z is read once with 16-byte loads (the next row's loads are issued
// before this row's reduction), each thread keeps its 8 values of v in registers, the group sums of squares are reduced in a fixed order (per-
// thread partials in shared memory, then one warp per group), and the row is
// written once.  HBM traffic per row: d elements of y and z in, d out.
#include <algorithm>

#include "ssd_common.cuh"

namespace ssd {
namespace {

constexpr int kVec = 8;   // channels per thread

__device__ __forceinline__ void load8(const float *p, float (&v)[8])
{
    const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&v)[8])
{
    uint4 u;
    u.x = pack_bf16x2(v[0], v[1]); u.y = pack_bf16x2(v[2], v[3]);
    u.z = pack_bf16x2(v[4], v[5]); u.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(p) = u;
}

__device__ __forceinline__ void store8(float *p, const float (&v)[8])
{
    reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// 8 elements as loaded: one 16-byte vector for bf16, two for fp32 (kept packed while in flight)
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 a;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) { a = *reinterpret_cast<const uint4 *>(p); }
    __device__ __forceinline__ void unpack(float (&v)[8]) const
    {
        v[0] = bf16_lo(a.x); v[1] = bf16_hi(a.x); v[2] = bf16_lo(a.y); v[3] = bf16_hi(a.y);
        v[4] = bf16_lo(a.z); v[5] = bf16_hi(a.z); v[6] = bf16_lo(a.w); v[7] = bf16_hi(a.w);
    }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float *p)
    {
        a = reinterpret_cast<const float4 *>(p)[0];
        b = reinterpret_cast<const float4 *>(p)[1];
    }
    __device__ __forceinline__ void unpack(float (&v)[8]) const
    {
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

template <typename T>
__global__ void __launch_bounds__(1024) gated_rmsnorm_kernel(NormParams p)
{
    extern __shared__ float part[];          // [blockDim.x] partial sums, then [d / group] scales
    float *scale = part + blockDim.x;
    const int i = threadIdx.x;
    const int nthr = p.d / kVec;
    const int ngroups = p.d / p.group, per_group = p.group / kVec;
    const int warp = i >> 5, lane = i & 31, nw = blockDim.x >> 5;
    const T *yb = reinterpret_cast<const T *>(p.y) + kVec * i;
    const T *zb = reinterpret_cast<const T *>(p.z) + kVec * i;
    Raw8<T> yn, zn;
    if (i < nthr && blockIdx.x < p.rows) {
        yn.load(yb + (int64_t)blockIdx.x * p.yrs);
        zn.load(zb + (int64_t)blockIdx.x * p.zrs);
    }
    for (int64_t r = blockIdx.x; r < p.rows; r += gridDim.x) {
        float v[8];
        float ss = 0.0f;
        if (i < nthr) {
            float yv[8], zv[8];
            yn.unpack(yv);
            zn.unpack(zv);
            // the next row's loads stay in flight through this row's reduction and store
            const int64_t rn = r + gridDim.x;
            if (rn < p.rows) {
                yn.load(yb + rn * p.yrs);
                zn.load(zb + rn * p.zrs);
            }
#pragma unroll
            for (int k = 0; k < kVec; ++k) {
                // silu(z) = z / (1 + e^-z) with the hardware exponential and a fast division; z is
                // clamped at -80 inside the exponential so the divisor stays below 2^126 (below -80
                // silu is below 1e-33 either way)
                const float e = __expf(-fmaxf(zv[k], -80.0f));
                v[k] = yv[k] * __fdividef(zv[k], 1.0f + e);
                ss = fmaf(v[k], v[k], ss);
            }
        }
        part[i] = ss;
        __syncthreads();
        for (int g = warp; g < ngroups; g += nw) {
            float s = 0.0f;
            for (int k = lane; k < per_group; k += 32) s += part[g * per_group + k];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) scale[g] = 1.0f / sqrtf(s / (float)p.group + p.eps);
        }
        __syncthreads();
        if (i < nthr) {
            const float sc = scale[(kVec * i) / p.group];
            float o[8], wv[8];
            load8(p.w + kVec * i, wv);
#pragma unroll
            for (int k = 0; k < kVec; ++k) o[k] = v[k] * sc * wv[k];
            store8(reinterpret_cast<T *>(p.out) + r * p.ors + kVec * i, o);
        }
        __syncthreads();   // part and scale are reused by the next row
    }
}

template <typename T>
int launch_norm_t(const NormParams &p, cudaStream_t st)
{
    const int nthr = p.d / kVec;
    const int block = std::max(32, (nthr + 31) / 32 * 32);
    const size_t smem = sizeof(float) * (size_t)(block + p.d / p.group);
    const int64_t grid = std::min<int64_t>(p.rows, 148 * 64);
    prof_begin(st, kKGatedNorm);
    gated_rmsnorm_kernel<T><<<(unsigned)grid, block, smem, st>>>(p);
    prof_end(st, kKGatedNorm);
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

}  // namespace

int launch_gated_norm(const NormParams &p, int dtype, cudaStream_t st)
{
    if (p.rows == 0) return 0;
    return dtype == 1 ? launch_norm_t<__nv_bfloat16>(p, st) : launch_norm_t<float>(p, st);
}

}  // namespace ssd

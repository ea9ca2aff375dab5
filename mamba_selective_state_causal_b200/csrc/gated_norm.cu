// gated_norm.cu -- the Mamba-2 block's output norm on the layer's y:
//   v = y * silu(z),   out = v / sqrt(mean over the channel group of v^2 + eps) * w
// The pages end at y; this is the plainest reading of the block around it
// (normalise after gating, groups of `group` consecutive channels).
//
// bf16 rows with d a multiple of 256 up to 2048 and groups of a multiple of 256
// channels: one warp per row (grid-stride over rows); lane l holds the 8-channel
// chunks l, l + 32, ... of the row in registers, all of the row's 16-byte loads
// are in flight at once, and a group's sum of squares is a warp reduction per
// chunk plus a fixed-order sum over the group's chunks, so no CTA barrier is
// needed.  Otherwise one CTA per row (grid-stride over rows), one thread per 8
// channels: a row of y and z is read once with 16-byte loads (the next row's
// loads are issued before this row's reduction), each thread keeps its 8 values
// of v in registers, the group sums of squares are reduced in a fixed order (per-
// thread partials in shared memory, then one warp per group), and the row is
// written once.  HBM traffic per row: d elements of y and z in, d out.
#include <algorithm>
#include <type_traits>

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

// silu(z) y, with the hardware exponential and a fast division; z is clamped at -80 inside the
// exponential so the divisor stays below 2^126 (below -80 silu is below 1e-33 either way)
__device__ __forceinline__ float gated(float y, float z)
{
    const float e = __expf(-fmaxf(z, -80.0f));
    return y * __fdividef(z, 1.0f + e);
}

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
                v[k] = gated(yv[k], zv[k]);
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

constexpr int kNormWarpThreads = 256;

template <int kChunks>   // d = 256 kChunks
__global__ void __launch_bounds__(kNormWarpThreads, 2) gated_rmsnorm_warp_kernel(NormParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (kNormWarpThreads / 32);
    const int m = p.group / 256;   // chunks per group
    const float inv_group = 1.0f / (float)p.group;
    for (int64_t r = (int64_t)blockIdx.x * (kNormWarpThreads / 32) + (threadIdx.x >> 5); r < p.rows; r += nwarps) {
        const __nv_bfloat16 *yr = reinterpret_cast<const __nv_bfloat16 *>(p.y) + r * p.yrs + 8 * lane;
        const __nv_bfloat16 *zr = reinterpret_cast<const __nv_bfloat16 *>(p.z) + r * p.zrs + 8 * lane;
        Raw8<__nv_bfloat16> yv[kChunks], zv[kChunks];
#pragma unroll
        for (int k = 0; k < kChunks; ++k) {
            yv[k].load(yr + 256 * k);
            zv[k].load(zr + 256 * k);
        }
        float v[kChunks][8], sq[kChunks];
#pragma unroll
        for (int k = 0; k < kChunks; ++k) {
            float a[8], b[8];
            yv[k].unpack(a);
            zv[k].unpack(b);
            float s = 0.0f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                v[k][e] = gated(a[e], b[e]);
                s = fmaf(v[k][e], v[k][e], s);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            sq[k] = s;
        }
        __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.out) + r * p.ors + 8 * lane;
#pragma unroll
        for (int k = 0; k < kChunks; ++k) {
            // the group of chunk k: chunks m (k / m) .. m (k / m) + m - 1, summed in order
            float s = 0.0f;
#pragma unroll
            for (int k2 = 0; k2 < kChunks; ++k2) s += (k2 / m == k / m) ? sq[k2] : 0.0f;
            const float sc = 1.0f / sqrtf(s * inv_group + p.eps);
            float wv[8], o[8];
            load8(p.w + 256 * k + 8 * lane, wv);
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = v[k][e] * sc * wv[e];
            store8(orow + 256 * k, o);
        }
    }
}

template <int kChunks>
int launch_norm_warp(const NormParams &p, cudaStream_t st)
{
    const int64_t grid = std::min<int64_t>((p.rows + kNormWarpThreads / 32 - 1) / (kNormWarpThreads / 32), 148 * 2);
    prof_begin(st, kKGatedNorm);
    gated_rmsnorm_warp_kernel<kChunks><<<(unsigned)grid, kNormWarpThreads, 0, st>>>(p);
    prof_end(st, kKGatedNorm);
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

template <typename T>
int launch_norm_t(const NormParams &p, cudaStream_t st)
{
    if (std::is_same<T, __nv_bfloat16>::value && p.d % 256 == 0 && p.d <= 2048 && p.group % 256 == 0) {
        switch (p.d / 256) {
        case 1: return launch_norm_warp<1>(p, st);
        case 2: return launch_norm_warp<2>(p, st);
        case 3: return launch_norm_warp<3>(p, st);
        case 4: return launch_norm_warp<4>(p, st);
        case 5: return launch_norm_warp<5>(p, st);
        case 6: return launch_norm_warp<6>(p, st);
        case 7: return launch_norm_warp<7>(p, st);
        default: return launch_norm_warp<8>(p, st);
        }
    }
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

// conv1d_silu.cu -- depthwise causal conv1d (kernel 4) + SiLU over the packed
// x|B|C stream (pith.science verdict for arXiv 2411.19460,
// skeptic_critique.load_bearing_attack: the causal Conv1d in front of the SSD,
// output at t uses inputs t-3..t; concrete_test: kernel = 4).
//
// Pure HBM stream: each thread owns one 16-byte channel vector (8 bf16 or
// 4 fp32 channels) over a block of TT consecutive tokens.  The 3-token halo
// lives in registers and slides along the token block, so every input row is
// read once (plus a 3-row halo per token block) and written once.
#include <cuda.h>

#include <algorithm>

#include "ssd_common.cuh"

namespace ssd {
namespace {

constexpr int kTokensPerThread = 64;
constexpr int kUnroll = 4;

struct alignas(16) Vec16 { uint32_t w[4]; };

__device__ __forceinline__ Vec16 ld_stream(const void *p)
{
    Vec16 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3])
                 : "l"(p));
    return r;
}

// Unpack a 16-byte vector into floats (8 bf16 or 4 fp32).
template <typename T> struct VecIO;
template <> struct VecIO<__nv_bfloat16> {
    static constexpr int kN = 8;
    __device__ __forceinline__ static void unpack(const Vec16 &v, float *f)
    {
#pragma unroll
        for (int i = 0; i < 4; ++i) { f[2 * i] = bf16_lo(v.w[i]); f[2 * i + 1] = bf16_hi(v.w[i]); }
    }
    __device__ __forceinline__ static Vec16 pack(const float *f)
    {
        Vec16 v;
#pragma unroll
        for (int i = 0; i < 4; ++i) v.w[i] = pack_bf16x2(f[2 * i], f[2 * i + 1]);
        return v;
    }
    // fast SiLU; the result is rounded to bf16 right after
    __device__ __forceinline__ static float silu(float z) { return __fdividef(z, 1.0f + __expf(-z)); }
};
template <> struct VecIO<float> {
    static constexpr int kN = 4;
    __device__ __forceinline__ static void unpack(const Vec16 &v, float *f)
    {
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = __uint_as_float(v.w[i]);
    }
    __device__ __forceinline__ static Vec16 pack(const float *f)
    {
        Vec16 v;
#pragma unroll
        for (int i = 0; i < 4; ++i) v.w[i] = __float_as_uint(f[i]);
        return v;
    }
    // accurate SiLU for the fp32 I/O path
    __device__ __forceinline__ static float silu(float z) { return z / (1.0f + expf(-z)); }
};

template <typename T>
__global__ void __launch_bounds__(256, 2) conv1d_silu_kernel(ConvParams p, int64_t n_tblk)
{
    using IO = VecIO<T>;
    constexpr int V = IO::kN;
    const int ncv = p.C_ch / V;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int cv = (int)(gid % ncv);
    const int64_t rest = gid / ncv;
    const int64_t tb = rest % n_tblk;
    const int64_t bi = rest / n_tblk;
    if (bi >= p.b) return;
    const int c0 = cv * V;

    float w0[V], w1[V], w2[V], w3[V], bs[V];
    {
        const float4 *wp = reinterpret_cast<const float4 *>(p.w + (int64_t)c0 * 4);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            float4 q = __ldg(wp + i);
            w0[i] = q.x; w1[i] = q.y; w2[i] = q.z; w3[i] = q.w;
            bs[i] = p.bias ? __ldg(p.bias + c0 + i) : 0.0f;
        }
    }
    const T *u = reinterpret_cast<const T *>(p.u) + bi * p.ubs + c0;
    T *v = reinterpret_cast<T *>(p.v) + bi * p.vbs + c0;
    const T *tin = p.tail_in ? reinterpret_cast<const T *>(p.tail_in) + bi * 3 * p.C_ch + c0 : nullptr;

    const int64_t t0 = tb * kTokensPerThread;
    const int64_t t1 = min(p.L, t0 + kTokensPerThread);

    // halo: m3 = u[t-3], m2 = u[t-2], m1 = u[t-1]
    float m3[V], m2[V], m1[V];
    {
        float *dst[3] = {m3, m2, m1};
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const int64_t pos = t0 - 3 + k;
            if (pos >= 0) {
                IO::unpack(ld_stream(u + pos * p.urs), dst[k]);
            } else if (tin) {
                IO::unpack(*reinterpret_cast<const Vec16 *>(tin + (3 + pos) * p.C_ch), dst[k]);
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i) dst[k][i] = 0.0f;
            }
        }
    }

    for (int64_t t = t0; t < t1; t += kUnroll) {
        Vec16 raw[kUnroll];
#pragma unroll
        for (int j = 0; j < kUnroll; ++j)
            if (t + j < t1) raw[j] = ld_stream(u + (t + j) * p.urs);
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
            if (t + j < t1) {
                float cur[V], out[V];
                IO::unpack(raw[j], cur);
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    float z = bs[i];
                    z = fmaf(w0[i], m3[i], z);
                    z = fmaf(w1[i], m2[i], z);
                    z = fmaf(w2[i], m1[i], z);
                    z = fmaf(w3[i], cur[i], z);
                    out[i] = IO::silu(z);
                    m3[i] = m2[i]; m2[i] = m1[i]; m1[i] = cur[i];
                }
                *reinterpret_cast<Vec16 *>(v + (t + j) * p.vrs) = IO::pack(out);
            }
        }
    }
}

// ---------------------------------------------------------------- TMA-staged variant
// Persistent CTAs stream tiles of [128 + 3 halo tokens] x [128 bytes of
// channels] through an 8-stage shared-memory ring filled by TMA, so that each
// SM keeps ~130 KB of loads in flight without spending registers on them.
// Tiles are ordered token-block-major: CTAs working at the same time read
// adjacent 128-byte pieces of the same rows.  Compute: 256 threads, thread =
// (16-byte channel vector cv, strip of 4 consecutive tokens).
constexpr int kTileTok = 128;
constexpr int kTileRows = kTileTok + 3;
constexpr int kStagesConv = 8;
constexpr int kConvThreads = 288;   // 8 compute warps + 1 producer warp

struct ConvSmem {
    uint8_t tile[kStagesConv][kTileRows * 128 + 128];  // row r = token t0 - 3 + r; padded to 128 B
    uint64_t full[kStagesConv], empty[kStagesConv];
    int abort;
};

__device__ __forceinline__ void conv_mbar_init(uint64_t *bar, uint32_t n)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"((uint32_t)__cvta_generic_to_shared(bar)), "r"(n));
}
__device__ __forceinline__ bool conv_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"((uint32_t)__cvta_generic_to_shared(bar)), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t conv_now()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// bounded wait: gives up after limit_ns or when another thread has aborted
__device__ __forceinline__ bool conv_wait(uint64_t *bar, uint32_t parity, volatile int *abort, uint64_t limit_ns)
{
    if (conv_try_wait(bar, parity)) return true;
    const uint64_t t0 = conv_now();
    while (!conv_try_wait(bar, parity)) {
        if (abort && *abort) return false;
        if (conv_now() - t0 > limit_ns) return false;
    }
    return true;
}

template <typename T>
__global__ void __launch_bounds__(kConvThreads, 1)
conv1d_silu_tma_kernel(const __grid_constant__ CUtensorMap umap, ConvParams p, int n_cb, int64_t n_tb,
                       int64_t n_tiles, unsigned int *status, uint64_t limit_ns)
{
    using IO = VecIO<T>;
    constexpr int V = IO::kN;               // channels per 16-byte vector
    constexpr int CB = 128 / sizeof(T);     // channels per tile
    extern __shared__ uint8_t craw[];
    ConvSmem &s = *reinterpret_cast<ConvSmem *>((reinterpret_cast<uintptr_t>(craw) + 127) & ~uintptr_t(127));
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        for (int i = 0; i < kStagesConv; ++i) { conv_mbar_init(&s.full[i], 1); conv_mbar_init(&s.empty[i], 256); }
        s.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    volatile int *abort = &s.abort;
    const int64_t first = blockIdx.x, step = gridDim.x;
    if (warp == 8) {
        if ((tid & 31) == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&umap)) : "memory");
            int64_t n = 0;
            for (int64_t tile = first; tile < n_tiles; tile += step, ++n) {
                const int st = (int)(n % kStagesConv);
                const uint32_t u = (uint32_t)(n / kStagesConv);
                if (n >= kStagesConv && !conv_wait(&s.empty[st], (u - 1) & 1, abort, limit_ns)) {
                    *abort = 1; atomicOr(status, kDevTimeout); break;
                }
                const int64_t tb = tile / ((int64_t)n_cb * p.b);
                const int64_t rem = tile % ((int64_t)n_cb * p.b);
                const int bi = (int)(rem / n_cb), cb = (int)(rem % n_cb);
                const uint32_t bar = (uint32_t)__cvta_generic_to_shared(&s.full[st]);
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"((uint32_t)(kTileRows * 128)) : "memory");
                asm volatile(
                    "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
                    ::"r"((uint32_t)__cvta_generic_to_shared(s.tile[st])), "l"(reinterpret_cast<uint64_t>(&umap)),
                      "r"(cb * CB), "r"((int)(tb * kTileTok - 3)), "r"(bi), "r"(bar)
                    : "memory");
            }
        }
        return;
    }
    const int cv = tid & 7;         // 16-byte vector within the tile's 128 bytes
    const int strip = tid >> 3;     // tokens 4 strip .. 4 strip + 3 of the tile
    int cur_cb = -1;
    float w0[V], w1[V], w2[V], w3[V], bs[V];
    int64_t n = 0;
    for (int64_t tile = first; tile < n_tiles; tile += step, ++n) {
        const int st = (int)(n % kStagesConv);
        const uint32_t u = (uint32_t)(n / kStagesConv);
        const int64_t tb = tile / ((int64_t)n_cb * p.b);
        const int64_t rem = tile % ((int64_t)n_cb * p.b);
        const int bi = (int)(rem / n_cb), cb = (int)(rem % n_cb);
        const int c0 = cb * CB + cv * V;
        const bool cvalid = c0 < p.C_ch;
        if (cb != cur_cb) {
            cur_cb = cb;
            if (cvalid) {
                const float4 *wp = reinterpret_cast<const float4 *>(p.w + (int64_t)c0 * 4);
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const float4 q = __ldg(wp + i);
                    w0[i] = q.x; w1[i] = q.y; w2[i] = q.z; w3[i] = q.w;
                    bs[i] = p.bias ? __ldg(p.bias + c0 + i) : 0.0f;
                }
            }
        }
        if (!conv_wait(&s.full[st], u & 1, abort, limit_ns)) {
            *abort = 1; atomicOr(status, kDevTimeout); break;
        }
        const int64_t t0 = tb * kTileTok;
        const uint8_t *tl = s.tile[st] + cv * 16;
        // rows 4 strip .. 4 strip + 6 of the tile hold tokens t - 3 .. t + 3 for t = t0 + 4 strip
        float rv[7][V];
#pragma unroll
        for (int k = 0; k < 7; ++k) {
            const int64_t tok = t0 + 4 * strip - 3 + k;
            if (tok < 0) {
                // before the stream start: the conv tail (zeros without one)
                if (p.tail_in && cvalid) {
                    IO::unpack(*reinterpret_cast<const Vec16 *>(reinterpret_cast<const T *>(p.tail_in) +
                                                              ((int64_t)bi * 3 + (3 + tok)) * p.C_ch + c0), rv[k]);
                } else {
#pragma unroll
                    for (int i = 0; i < V; ++i) rv[k][i] = 0.0f;
                }
            } else {
                IO::unpack(*reinterpret_cast<const Vec16 *>(tl + (4 * strip + k) * 128), rv[k]);
            }
        }
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"((uint32_t)__cvta_generic_to_shared(&s.empty[st])) : "memory");
        if (cvalid) {
            T *vb = reinterpret_cast<T *>(p.v) + (int64_t)bi * p.vbs + c0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t t = t0 + 4 * strip + j;
                if (t < p.L) {
                    float out[V];
#pragma unroll
                    for (int i = 0; i < V; ++i) {
                        float z = bs[i];
                        z = fmaf(w0[i], rv[j][i], z);
                        z = fmaf(w1[i], rv[j + 1][i], z);
                        z = fmaf(w2[i], rv[j + 2][i], z);
                        z = fmaf(w3[i], rv[j + 3][i], z);
                        out[i] = IO::silu(z);
                    }
                    *reinterpret_cast<Vec16 *>(vb + t * p.vrs) = IO::pack(out);
                }
            }
        }
    }
}

// tail_out[bi, r, c] = u at position L-3+r, or tail_in[bi, 3+pos, c] when pos < 0,
// or 0.  Runs after the conv kernel on the same stream, so tail_out may alias
// tail_in; each thread reads its three values before writing any.
template <typename T>
__global__ void conv_tail_kernel(ConvParams p)
{
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)p.b * p.C_ch) return;
    const int64_t bi = gid / p.C_ch;
    const int c = (int)(gid % p.C_ch);
    const T *u = reinterpret_cast<const T *>(p.u) + bi * p.ubs + c;
    const T *tin = p.tail_in ? reinterpret_cast<const T *>(p.tail_in) + bi * 3 * p.C_ch + c : nullptr;
    T vals[3];
#pragma unroll
    for (int r = 0; r < 3; ++r) {
        const int64_t pos = p.L - 3 + r;
        if (pos >= 0) vals[r] = u[pos * p.urs];
        else vals[r] = tin ? tin[(3 + pos) * p.C_ch] : from_f32<T>(0.0f);
    }
    T *tout = reinterpret_cast<T *>(p.tail_out) + bi * 3 * p.C_ch + c;
#pragma unroll
    for (int r = 0; r < 3; ++r) tout[r * p.C_ch] = vals[r];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn conv_encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// TMA-staged launch; returns false (nothing launched) when a tensor map for u cannot be built.
template <typename T>
bool launch_conv_tma(const ConvParams &p, cudaStream_t st, unsigned int *status, uint64_t limit_ns)
{
    EncodeTiledFn enc = conv_encode_fn();
    if (!enc || p.L >= (1LL << 31) - 256) return false;
    constexpr int CB = 128 / sizeof(T);
    const int64_t bs = p.b == 1 ? p.urs * p.L : p.ubs;
    const cuuint64_t dims[3] = {(cuuint64_t)p.C_ch, (cuuint64_t)p.L, (cuuint64_t)p.b};
    const cuuint64_t strides[2] = {(cuuint64_t)p.urs * sizeof(T), (cuuint64_t)bs * sizeof(T)};
    const cuuint32_t box[3] = {(cuuint32_t)CB, (cuuint32_t)kTileRows, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    CUtensorMap umap;
    if (enc(&umap, sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
            const_cast<void *>(p.u), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    int dev = 0, nsm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = sizeof(ConvSmem) + 128;
    static bool attr_set[2][64] = {{false}};
    const int ti = sizeof(T) == 2 ? 1 : 0;
    if (dev >= 0 && dev < 64 && !attr_set[ti][dev]) {
        if (cudaFuncSetAttribute(conv1d_silu_tma_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return false;
        attr_set[ti][dev] = true;
    }
    const int n_cb = (p.C_ch + CB - 1) / CB;
    const int64_t n_tb = (p.L + kTileTok - 1) / kTileTok;
    const int64_t n_tiles = n_tb * n_cb * p.b;
    const int64_t grid = std::min<int64_t>(n_tiles, nsm > 0 ? nsm : 148);
    conv1d_silu_tma_kernel<T><<<(unsigned)grid, kConvThreads, smem, st>>>(umap, p, n_cb, n_tb, n_tiles, status, limit_ns);
    return true;
}

template <typename T>
int launch_conv_t(const ConvParams &p, cudaStream_t st)
{
    constexpr int V = VecIO<T>::kN;
    if (p.b > 0 && p.L > 0) {
        prof_begin(st, kKConv);
        // the TMA-staged variant measured slower than the register-streaming kernel (its
        // 128-byte row pieces spread the DRAM accesses), so it is not selected
        const bool tma = false && p.status && launch_conv_tma<T>(p, st, p.status, p.wait_limit_ns);
        if (!tma) {
            const int64_t n_tblk = (p.L + kTokensPerThread - 1) / kTokensPerThread;
            const int64_t threads = (int64_t)p.b * n_tblk * (p.C_ch / V);
            const int64_t blocks = (threads + 255) / 256;
            if (blocks > 0x7fffffffLL) return 2;
            conv1d_silu_kernel<T><<<(unsigned)blocks, 256, 0, st>>>(p, n_tblk);
        }
        prof_end(st, kKConv);
    }
    if (p.tail_out && p.b > 0) {
        const int64_t n = (int64_t)p.b * p.C_ch;
        prof_begin(st, kKConvTail);
        conv_tail_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(p);
        prof_end(st, kKConvTail);
    }
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

}  // namespace

int launch_conv(const ConvParams &p, int dtype, cudaStream_t st)
{
    return dtype == 1 ? launch_conv_t<__nv_bfloat16>(p, st) : launch_conv_t<float>(p, st);
}

}  // namespace ssd

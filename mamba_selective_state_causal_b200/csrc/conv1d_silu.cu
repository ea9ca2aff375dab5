// conv1d_silu.cu -- depthwise causal conv1d (kernel 4) + SiLU over the packed
// x|B|C stream (pith.science verdict for arXiv 2411.19460,
// skeptic_critique.load_bearing_attack: the causal Conv1d in front of the SSD,
// output at t uses inputs t-3..t; concrete_test: kernel = 4).
//
// Pure HBM stream: each thread owns one 16-byte channel vector (8 bf16 or
// 4 fp32 channels) over a block of 64 consecutive tokens.  Its rows stream in
// through a private 16-row ring in shared memory filled by cp.async, which
// keeps 128 KB of loads in flight per SM without holding registers.  The
// 3-token halo lives in registers and slides along the token block, so every
// input row is read once (plus a 3-row halo per token block) and written once.
#include <algorithm>
#include <atomic>

#include "ssd_common.cuh"

namespace ssd {
namespace {

constexpr int kTokensPerThread = 64;

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
    // The conv sums with halved weights and bias (kPre; a power-of-two scale, exact), so
    // that silu() receives h = z / 2, and SiLU(z) = z sigmoid(z) = h + h tanh(h): one
    // hardware tanh (relative error about 2^-11) and one fma instead of an exponential and
    // a reciprocal; the result is rounded to bf16 right after
    static constexpr float kPre = 0.5f;
    __device__ __forceinline__ static float silu(float h)
    {
        float t;
        asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
        return fmaf(h, t, h);
    }
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
    // accurate SiLU for the fp32 I/O path, on the unscaled sum
    static constexpr float kPre = 1.0f;
    __device__ __forceinline__ static float silu(float z) { return z / (1.0f + expf(-z)); }
};

// cp.async of one 16-byte vector into shared memory (its own commit group per row)
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

constexpr int kRing = 16;          // rows in flight per thread, staged in shared memory
constexpr int kConvThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kConvThreads, 2) conv1d_silu_kernel(ConvParams p, int64_t n_tblk)
{
    using IO = VecIO<T>;
    constexpr int V = IO::kN;
    // each thread streams its own rows through its own ring slots: [row slot][thread]
    extern __shared__ Vec16 ring_raw[];
    Vec16 (*ring)[kConvThreads] = reinterpret_cast<Vec16 (*)[kConvThreads]>(ring_raw);
    const int ncv = p.C_ch / V;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int cv = (int)(gid % ncv);
    const int64_t rest = gid / ncv;
    const int64_t tb = rest % n_tblk;
    const int64_t bi = rest / n_tblk;
    const bool active = bi < p.b;
    const int c0 = cv * V;

    float w0[V], w1[V], w2[V], w3[V], bs[V];
    const T *u = reinterpret_cast<const T *>(p.u) + bi * p.ubs + c0;
    T *v = reinterpret_cast<T *>(p.v) + bi * p.vbs + c0;
    const T *tin = p.tail_in ? reinterpret_cast<const T *>(p.tail_in) + bi * 3 * p.tail_rs + c0 : nullptr;
    const int64_t t0 = tb * kTokensPerThread;
    const int n = active ? (int)(min(p.L, t0 + kTokensPerThread) - t0) : 0;
    Vec16 *slot = &ring[0][threadIdx.x];
    const T *up = u + t0 * p.urs;
    // fill the ring: one commit group per row (empty groups past the end keep the count uniform)
#pragma unroll
    for (int j = 0; j < kRing; ++j) {
        if (j < n) cp_async16(slot + j * kConvThreads, up + j * p.urs);
        cp_async_commit();
    }
    if (!active) return;
    {
        const float4 *wp = reinterpret_cast<const float4 *>(p.w + (int64_t)c0 * 4);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            float4 q = __ldg(wp + i);
            w0[i] = IO::kPre * q.x; w1[i] = IO::kPre * q.y; w2[i] = IO::kPre * q.z; w3[i] = IO::kPre * q.w;
            bs[i] = p.bias ? IO::kPre * __ldg(p.bias + c0 + i) : 0.0f;
        }
    }
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
                IO::unpack(*reinterpret_cast<const Vec16 *>(tin + (3 + pos) * p.tail_rs), dst[k]);
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i) dst[k][i] = 0.0f;
            }
        }
    }
    T *vp = v + t0 * p.vrs;
    up += kRing * p.urs;
    for (int i0 = 0; i0 < n; i0 += kRing) {
#pragma unroll
        for (int j = 0; j < kRing; ++j) {
            if (i0 + j < n) {
                cp_async_wait<kRing - 1>();      // row i0 + j has landed (its group is the oldest)
                float cur[V], out[V];
                IO::unpack(slot[j * kConvThreads], cur);
                // refill the slot with row i0 + j + kRing
                if (i0 + j + kRing < n) cp_async16(slot + j * kConvThreads, up);
                cp_async_commit();
                up += p.urs;
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
                *reinterpret_cast<Vec16 *>(vp) = IO::pack(out);
                vp += p.vrs;
            }
        }
    }
    cp_async_wait<0>();
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
    const T *tin = p.tail_in ? reinterpret_cast<const T *>(p.tail_in) + bi * 3 * p.tail_rs + c : nullptr;
    T vals[3];
#pragma unroll
    for (int r = 0; r < 3; ++r) {
        const int64_t pos = p.L - 3 + r;
        if (pos >= 0) vals[r] = u[pos * p.urs];
        else vals[r] = tin ? tin[(3 + pos) * p.tail_rs] : from_f32<T>(0.0f);
    }
    T *tout = reinterpret_cast<T *>(p.tail_out) + bi * 3 * p.tail_rs + c;
#pragma unroll
    for (int r = 0; r < 3; ++r) tout[r * p.tail_rs] = vals[r];
}

template <typename T>
int launch_conv_t(const ConvParams &p, cudaStream_t st)
{
    constexpr int V = VecIO<T>::kN;
    if (p.b > 0 && p.L > 0) {
        prof_begin(st, kKConv);
        const int64_t n_tblk = (p.L + kTokensPerThread - 1) / kTokensPerThread;
        const int64_t threads = (int64_t)p.b * n_tblk * (p.C_ch / V);
        const int64_t blocks = (threads + kConvThreads - 1) / kConvThreads;
        if (blocks > 0x7fffffffLL) return 2;
        constexpr int smem = kRing * kConvThreads * (int)sizeof(Vec16);
        static std::atomic<bool> attr_set[64];   // set once per device (a repeat is harmless)
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev >= 0 && dev < 64 && !attr_set[dev]) {
            if (cudaFuncSetAttribute(conv1d_silu_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
                return 7;
            attr_set[dev] = true;
        }
        conv1d_silu_kernel<T><<<(unsigned)blocks, kConvThreads, smem, st>>>(p, n_tblk);
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

// The conv output rebuilt cell by cell for the backward pass: v[bi, t, c] from
// the cell's own rows of u and its 3-row conv buffer, with the forward
// kernel's arithmetic (same order of fused multiply-adds, same SiLU), so that a
// cell rebuilt from exact buffers reproduces the forward's v bit for bit.
constexpr int kCellTB = 64;      // tokens per thread of the cell rebuild

// One thread per (batch row, block of kCellTB tokens, channel pair), consecutive threads on
// consecutive pairs (4-byte bf16 pairs in and out); the block's cell is found once (a block never
// crosses a cell: blocks and cells are multiples of 64 tokens), the thread slides the conv window
// of u along its block in registers, and the next eight rows of u are loaded before their
// arithmetic.  The arithmetic of each channel is the forward conv's, in its order.
__device__ __forceinline__ float2 cells_ld2(const float *q) { return *reinterpret_cast<const float2 *>(q); }
__device__ __forceinline__ float2 cells_ld2(const __nv_bfloat16 *q)
{
    const uint32_t v = *reinterpret_cast<const uint32_t *>(q);
    return make_float2(bf16_lo(v), bf16_hi(v));
}
__device__ __forceinline__ void cells_st2(float *q, float a, float b) { *reinterpret_cast<float2 *>(q) = make_float2(a, b); }
__device__ __forceinline__ void cells_st2(__nv_bfloat16 *q, float a, float b)
{
    const __nv_bfloat16 ha = __float2bfloat16_rn(a), hb = __float2bfloat16_rn(b);
    *reinterpret_cast<uint32_t *>(q) = (uint32_t)__bfloat16_as_ushort(ha) | ((uint32_t)__bfloat16_as_ushort(hb) << 16);
}

constexpr int kCellAhead = 8;
template <typename T>
__global__ void __launch_bounds__(256, 3) conv_cells2_kernel(ConvBwdParams p, int64_t nblk)
{
    const int np = p.C_ch >> 1;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)p.b * nblk * np) return;
    const int c = 2 * (int)(gid % np);
    const int64_t blk = (gid / np) % nblk;
    const int64_t bi = gid / ((int64_t)np * nblk);
    const int64_t t0 = blk * kCellTB;
    const int64_t t1 = min(p.L, t0 + kCellTB);
    // weights and bias scaled as the forward conv scales them (VecIO::kPre)
    constexpr float pre = VecIO<T>::kPre;
    const float4 qa = __ldg(reinterpret_cast<const float4 *>(p.w) + c);
    const float4 qb = __ldg(reinterpret_cast<const float4 *>(p.w) + c + 1);
    const float4 wa = make_float4(pre * qa.x, pre * qa.y, pre * qa.z, pre * qa.w);
    const float4 wb = make_float4(pre * qb.x, pre * qb.y, pre * qb.z, pre * qb.w);
    const float ba = p.bias ? pre * __ldg(p.bias + c) : 0.0f, bb = p.bias ? pre * __ldg(p.bias + c + 1) : 0.0f;
    const T *u = reinterpret_cast<const T *>(p.u) + bi * p.ubs + c;
    // the window u[t0-3 .. t0-1]: rows before the cell come from its conv buffer
    const int64_t kc = p.conv_ckpt ? t0 / p.s : 0;
    const int64_t cstart = p.conv_ckpt ? kc * p.s : 0;
    float2 uw[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const int64_t tt = t0 - 3 + k;
        if (tt >= cstart) {
            uw[k] = cells_ld2(u + tt * p.urs);
        } else {
            const int64_t r = tt - cstart + 3;
            if (kc == 0)
                uw[k] = p.tail_in ? cells_ld2(reinterpret_cast<const T *>(p.tail_in) + (bi * 3 + r) * p.C_ch + c)
                                  : make_float2(0.0f, 0.0f);
            else
                uw[k] = cells_ld2(reinterpret_cast<const T *>(p.conv_ckpt) + ((bi * p.n_ckpt + (kc - 1)) * 3 + r) * p.C_ch + c);
        }
    }
    T *v = reinterpret_cast<T *>(p.v) + (bi * p.L) * p.C_ch + c;
    for (int64_t tg = t0; tg < t1; tg += kCellAhead) {
        float2 un[kCellAhead];
#pragma unroll
        for (int i = 0; i < kCellAhead; ++i) un[i] = tg + i < t1 ? cells_ld2(u + (tg + i) * p.urs) : make_float2(0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < kCellAhead; ++i) {
            const int64_t t = tg + i;
            if (t >= t1) break;
            float za = ba, zb = bb;
            za = fmaf(wa.x, uw[0].x, za); zb = fmaf(wb.x, uw[0].y, zb);
            za = fmaf(wa.y, uw[1].x, za); zb = fmaf(wb.y, uw[1].y, zb);
            za = fmaf(wa.z, uw[2].x, za); zb = fmaf(wb.z, uw[2].y, zb);
            za = fmaf(wa.w, un[i].x, za); zb = fmaf(wb.w, un[i].y, zb);
            cells_st2(v + t * p.C_ch, VecIO<T>::silu(za), VecIO<T>::silu(zb));
            uw[0] = uw[1]; uw[1] = uw[2]; uw[2] = un[i];
        }
    }
}

// conv_ckpt[bi, k, r, c] = u[bi, (k+1) s - 3 + r, c]: the conv buffer at every checkpoint
template <typename T>
__global__ void conv_ckpt_kernel(const T *u, int64_t ubs, int64_t urs, T *out, int b, int64_t n_ckpt, int C_ch,
                                 int64_t s)
{
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)b * n_ckpt * 3 * C_ch) return;
    const int c = (int)(gid % C_ch);
    const int64_t r = (gid / C_ch) % 3;
    const int64_t k = (gid / ((int64_t)3 * C_ch)) % n_ckpt;
    const int64_t bi = gid / ((int64_t)3 * C_ch * n_ckpt);
    out[gid] = u[bi * ubs + ((k + 1) * s - 3 + r) * urs + c];
}

}  // namespace

int launch_conv_cells(const ConvBwdParams &p, int dtype, cudaStream_t st)
{
    const int64_t nblk = (p.L + kCellTB - 1) / kCellTB;
    // two channels per thread: P and N are multiples of 16, so C_ch is even
    const int64_t n = (int64_t)p.b * nblk * (p.C_ch / 2);
    if (n == 0) return 0;
    const int64_t blocks = (n + 255) / 256;
    if (blocks > 0x7fffffffLL) return 2;
    prof_begin(st, kKConvCells);
    if (dtype == 1) conv_cells2_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(p, nblk);
    else conv_cells2_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(p, nblk);
    prof_end(st, kKConvCells);
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

int launch_conv_ckpt(const void *u, int64_t ubs, int64_t urs, void *conv_ckpt, int b, int64_t L, int C_ch,
                     int64_t s, int dtype, cudaStream_t st)
{
    const int64_t n_ckpt = s > 0 ? L / s : 0;
    const int64_t n = (int64_t)b * n_ckpt * 3 * C_ch;
    if (n == 0) return 0;
    const int64_t blocks = (n + 255) / 256;
    if (blocks > 0x7fffffffLL) return 2;
    prof_begin(st, kKConvCkpt);
    if (dtype == 1)
        conv_ckpt_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
            reinterpret_cast<const __nv_bfloat16 *>(u), ubs, urs, reinterpret_cast<__nv_bfloat16 *>(conv_ckpt), b,
            n_ckpt, C_ch, s);
    else
        conv_ckpt_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const float *>(u), ubs, urs,
                                                                 reinterpret_cast<float *>(conv_ckpt), b, n_ckpt,
                                                                 C_ch, s);
    prof_end(st, kKConvCkpt);
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

int launch_conv_tail(const ConvParams &p, int dtype, cudaStream_t st)
{
    if (!p.tail_out || p.b <= 0) return 0;
    const int64_t n = (int64_t)p.b * p.C_ch;
    prof_begin(st, kKConvTail);
    if (dtype == 1) conv_tail_kernel<__nv_bfloat16><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(p);
    else conv_tail_kernel<float><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(p);
    prof_end(st, kKConvTail);
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

int launch_conv(const ConvParams &p, int dtype, cudaStream_t st)
{
    return dtype == 1 ? launch_conv_t<__nv_bfloat16>(p, st) : launch_conv_t<float>(p, st);
}

}  // namespace ssd

// layer_bwd.cu -- the conv half of the layer's backward pass: from the
// gradients of the conv output v = [x | B | C] (which the scan's backward
// pass returns) to the gradients of the conv input u, of the conv weights and
// bias, and of the conv buffer that started the sequence.
//
// The layer's conv (pith.science verdict for arXiv 2411.19460,
// skeptic_critique.load_bearing_attack: a causal Conv1d of kernel 4 before
// the SSD) is v[t,c] = silu(z[t,c]), z[t,c] = bias_c + sum_k w[c,k] u[t-3+k,c].
// Its reverse mode:
//   dz[t,c]     = dv[t,c] silu'(z[t,c]),  silu'(z) = sig(z) (1 + z (1 - sig(z)))
//   du[t',c]    = sum_{j=0..3} w[c,3-j] dz[t'+j,c]     (+ dLoss/dtail_out for the last 3 rows)
//   dw[c,k]     = sum_t dz[t,c] u[t-3+k,c],   dbias_c = sum_t dz[t,c]
// Each cell of s tokens is rebuilt on its own (MA-GC's grid-cell recompute,
// pith_extraction.key_machinery): z of a token reads the rows before its cell
// from that cell's stored 3-row conv buffer, which is what makes the
// recompute exact (skeptic_critique.headline).  The rounding of v to the I/O
// dtype is taken as the identity, and dz is fp32 (sigma through the hardware exponential).
#include "ssd_common.cuh"

namespace ssd {
namespace {

constexpr int kTB = 64;          // tokens per thread, walked from the last
constexpr int kConvBwdThreads = 256;

// dz = dv silu'(z) from the conv window u[t-3 .. t] (as token t's cell sees it)
__device__ __forceinline__ float dz_of(float dv, const float4 &wq, float bs, const float (&uw)[4])
{
    float z = bs;
    z = fmaf(wq.x, uw[0], z);
    z = fmaf(wq.y, uw[1], z);
    z = fmaf(wq.z, uw[2], z);
    z = fmaf(wq.w, uw[3], z);
    // sigma(z) with the hardware exponential and a fast division; -z is clamped at 80 inside the
    // exponential so the divisor stays below 2^126 (sigma(z) is below 2e-35 there either way)
    const float sg = __fdividef(1.0f, 1.0f + __expf(fminf(-z, 80.0f)));
    return dv * (sg * (1.0f + z * (1.0f - sg)));
}

// ---- two consecutive channels per thread (8-byte loads of dv and stores of du, 4 bytes of bf16 u)
__device__ __forceinline__ float2 ld2(const float *q) { return *reinterpret_cast<const float2 *>(q); }
__device__ __forceinline__ float2 ld2(const __nv_bfloat16 *q)
{
    const uint32_t v = *reinterpret_cast<const uint32_t *>(q);
    return make_float2(bf16_lo(v), bf16_hi(v));
}

// dLoss/dv of channels c, c+1 (both in one of x, B, C) at row (bi, t)
__device__ __forceinline__ float2 dv2_at(const ConvBwdParams &p, int64_t bi, int64_t t, int c)
{
    const int64_t row = bi * p.L + t;
    if (c < p.HP) return ld2(p.dx + row * p.HP + c);
    if (c < p.HP + p.GN) return ld2(p.dB + row * p.GN + (c - p.HP));
    return ld2(p.dC + row * p.GN + (c - p.HP - p.GN));
}

// Row tt of the conv input, channels c and c+1, as a token of cell k (which starts at `start`)
// sees it when each cell is rebuilt on its own: rows before the cell come from its 3-row conv
// buffer (conv_ckpt[k-1] for cell k > 0, tail_in or zeros for the first cell), the others from u
template <typename T>
__device__ __forceinline__ float2 cell2k(const ConvBwdParams &p, int64_t bi, int64_t k, int64_t start, int64_t tt, int c)
{
    if (tt >= start) return ld2(reinterpret_cast<const T *>(p.u) + bi * p.ubs + tt * p.urs + c);
    const int64_t r = tt - start + 3;
    if (k == 0)
        return p.tail_in ? ld2(reinterpret_cast<const T *>(p.tail_in) + (bi * 3 + r) * p.C_ch + c)
                         : make_float2(0.0f, 0.0f);
    return ld2(reinterpret_cast<const T *>(p.conv_ckpt) + ((bi * p.n_ckpt + (k - 1)) * 3 + r) * p.C_ch + c);
}

// the same for token t (its cell found from t)
template <typename T>
__device__ __forceinline__ float2 cell2(const ConvBwdParams &p, int64_t bi, int64_t t, int64_t tt, int c)
{
    const int64_t k = p.conv_ckpt ? t / p.s : 0;
    return cell2k<T>(p, bi, k, p.conv_ckpt ? k * p.s : 0, tt, c);
}

template <typename T>
__device__ __forceinline__ float2 dz2_at(const ConvBwdParams &p, int64_t bi, int64_t t, int c, const float4 (&wq)[2],
                                         const float2 &bs)
{
    if (t >= p.L) return make_float2(0.0f, 0.0f);
    float2 uw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) uw[k] = cell2<T>(p, bi, t, t - 3 + k, c);
    const float2 dv = dv2_at(p, bi, t, c);
    const float wa[4] = {uw[0].x, uw[1].x, uw[2].x, uw[3].x}, wb[4] = {uw[0].y, uw[1].y, uw[2].y, uw[3].y};
    return make_float2(dz_of(dv.x, wq[0], bs.x, wa), dz_of(dv.y, wq[1], bs.y, wb));
}

// asynchronous copies of 4 or 8 bytes into shared memory (the stream of one thread)
template <int kBytes>
__device__ __forceinline__ void cp_async_small(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src),
                 "n"(kBytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit_b() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_b() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// One thread per (batch row, block of kTB tokens, channel pair), consecutive threads on
// consecutive pairs; the thread walks its block from the last token with the conv window of u
// and a 4-deep window of dz in registers (a block never crosses a cell: blocks and cells are
// multiples of 64 tokens).  Each
// thread streams its tokens' dv and the u rows its window needs through its own slots of a ring
// in shared memory (kRingB tokens in flight, 4- and 8-byte asynchronous copies), so the loads in
// flight cost no registers; the block's cell (where its conv buffer starts) is found once.
constexpr int kRingB = 16;
template <typename T>
__global__ void __launch_bounds__(kConvBwdThreads, 2) conv_bwd2_kernel(ConvBwdParams p, int64_t nblk)
{
    extern __shared__ __align__(16) uint8_t cbw_raw[];
    float2 *rdv = reinterpret_cast<float2 *>(cbw_raw);                                   // [kRingB][threads]
    T *ru = reinterpret_cast<T *>(cbw_raw + sizeof(float2) * kRingB * kConvBwdThreads);   // [kRingB][threads][2]
    const int tid = threadIdx.x;
    const int np = p.C_ch >> 1;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + tid;
    if (gid >= (int64_t)p.b * nblk * np) return;
    const int c = 2 * (int)(gid % np);
    const int64_t blk = (gid / np) % nblk;
    const int64_t bi = gid / ((int64_t)np * nblk);
    const int64_t t0 = blk * kTB;
    const int64_t t1 = min(p.L, t0 + kTB);
    const int n = (int)(t1 - t0);
    // the block's tokens are all in one cell (blocks and cells are multiples of 64 tokens)
    const int64_t kc = p.conv_ckpt ? t0 / p.s : 0;
    const int64_t cstart = p.conv_ckpt ? kc * p.s : 0;
    auto dv_ptr = [&](int64_t t) -> const float * {
        const int64_t row = bi * p.L + t;
        if (c < p.HP) return p.dx + row * p.HP + c;
        if (c < p.HP + p.GN) return p.dB + row * p.GN + (c - p.HP);
        return p.dC + row * p.GN + (c - p.HP - p.GN);
    };
    auto u_ptr = [&](int64_t tt) -> const T * {
        if (tt >= cstart) return reinterpret_cast<const T *>(p.u) + bi * p.ubs + tt * p.urs + c;
        const int64_t r = tt - cstart + 3;
        if (kc == 0) return p.tail_in ? reinterpret_cast<const T *>(p.tail_in) + (bi * 3 + r) * p.C_ch + c : nullptr;
        return reinterpret_cast<const T *>(p.conv_ckpt) + ((bi * p.n_ckpt + (kc - 1)) * 3 + r) * p.C_ch + c;
    };
    // token j of the walk is t = t1 - 1 - j: its dv, and u[t - 4], the row its window takes next
    auto issue = [&](int j) {
        if (j < n) {
            const int64_t t = t1 - 1 - j;
            const int sl = (j % kRingB) * kConvBwdThreads + tid;
            cp_async_small<8>(&rdv[sl], dv_ptr(t));
            if (t > t0) {
                const T *q = u_ptr(t - 4);
                if (q) cp_async_small<2 * sizeof(T)>(&ru[2 * sl], q);
            }
        }
        cp_async_commit_b();
    };
#pragma unroll 1
    for (int j = 0; j < kRingB; ++j) issue(j);

    float4 wq[2];
    wq[0] = __ldg(reinterpret_cast<const float4 *>(p.w) + c);
    wq[1] = __ldg(reinterpret_cast<const float4 *>(p.w) + c + 1);
    const float2 bs = p.bias ? make_float2(__ldg(p.bias + c), __ldg(p.bias + c + 1)) : make_float2(0.0f, 0.0f);
    // window of dz at t'+0 .. t'+3, walked from t' = t1-1 down to t0
    float2 d1 = dz2_at<T>(p, bi, t1, c, wq, bs), d2 = dz2_at<T>(p, bi, t1 + 1, c, wq, bs),
           d3 = dz2_at<T>(p, bi, t1 + 2, c, wq, bs);
    float2 gw[4] = {}, gb = make_float2(0.0f, 0.0f);
    float2 uw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) uw[k] = cell2k<T>(p, bi, kc, cstart, t1 - 4 + k, c);
#pragma unroll 1
    for (int j = 0; j < n; ++j) {
        const int64_t t = t1 - 1 - j;
        cp_async_wait_b<kRingB - 1>();          // token j's group is the oldest
        const int sl = (j % kRingB) * kConvBwdThreads + tid;
        const float2 dvv = rdv[sl];
        float2 un = make_float2(0.0f, 0.0f);
        if (t > t0 && u_ptr(t - 4)) {
            if (sizeof(T) == 2) {
                const uint32_t v = *reinterpret_cast<const uint32_t *>(&ru[2 * sl]);
                un = make_float2(bf16_lo(v), bf16_hi(v));
            } else {
                un = *reinterpret_cast<const float2 *>(&ru[2 * sl]);
            }
        }
        issue(j + kRingB);                       // refill the slot just read
        const float wa[4] = {uw[0].x, uw[1].x, uw[2].x, uw[3].x}, wb[4] = {uw[0].y, uw[1].y, uw[2].y, uw[3].y};
        const float2 d0 = make_float2(dz_of(dvv.x, wq[0], bs.x, wa), dz_of(dvv.y, wq[1], bs.y, wb));
        float2 g;
        g.x = fmaf(wq[0].x, d3.x, fmaf(wq[0].y, d2.x, fmaf(wq[0].z, d1.x, wq[0].w * d0.x)));
        g.y = fmaf(wq[1].x, d3.y, fmaf(wq[1].y, d2.y, fmaf(wq[1].z, d1.y, wq[1].w * d0.y)));
        if (p.dtail_out && t >= p.L - 3) {
            const float2 dto = ld2(p.dtail_out + (bi * 3 + (t - (p.L - 3))) * p.C_ch + c);
            g.x += dto.x;
            g.y += dto.y;
        }
        *reinterpret_cast<float2 *>(p.du + (bi * p.L + t) * p.C_ch + c) = g;
        gb.x += d0.x;
        gb.y += d0.y;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            gw[k].x = fmaf(d0.x, wa[k], gw[k].x);
            gw[k].y = fmaf(d0.y, wb[k], gw[k].y);
        }
        d3 = d2; d2 = d1; d1 = d0;
        uw[3] = uw[2]; uw[2] = uw[1]; uw[1] = uw[0]; uw[0] = un;
    }
    cp_async_wait_b<0>();
    const int64_t slot = (bi * nblk + blk) * p.C_ch + c;
    reinterpret_cast<float4 *>(p.ws_dw)[slot] = make_float4(gw[0].x, gw[1].x, gw[2].x, gw[3].x);
    reinterpret_cast<float4 *>(p.ws_dw)[slot + 1] = make_float4(gw[0].y, gw[1].y, gw[2].y, gw[3].y);
    p.ws_dbias[slot] = gb.x;
    p.ws_dbias[slot + 1] = gb.y;
    if (blk == 0 && p.dtail_in) {
        // the rows before the sequence (positions -3, -2, -1): d1, d2, d3 now hold dz at 0, 1, 2
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
            float *dt = p.dtail_in + bi * 3 * p.C_ch + c + ch;
            const float e1 = ch ? d1.y : d1.x, e2 = ch ? d2.y : d2.x, e3 = ch ? d3.y : d3.x;
            float g2 = fmaf(wq[ch].z, e1, fmaf(wq[ch].y, e2, wq[ch].x * e3));   // position -1
            float g1 = fmaf(wq[ch].y, e1, wq[ch].x * e2);                        // position -2
            float g0 = wq[ch].x * e1;                                            // position -3
            if (p.dtail_out) {
                for (int r = 0; r < 3; ++r) {
                    const int64_t pos = p.L - 3 + r;
                    if (pos >= 0) continue;
                    const float gt = p.dtail_out[(bi * 3 + r) * p.C_ch + c + ch];
                    if (pos == -3) g0 += gt;
                    else if (pos == -2) g1 += gt;
                    else g2 += gt;
                }
            }
            dt[0] = g0;
            dt[p.C_ch] = g1;
            dt[2 * p.C_ch] = g2;
        }
    }
}

// dw and dbias: the partial sums of every (batch row, token block), added in a fixed order.  A CTA
// takes 32 channels; its 8 warps each add every 8th partial of them (8 loads in flight per
// thread), then warp 0 adds the 8 warp sums in order.
constexpr int kRedSlices = 8;
__global__ void __launch_bounds__(32 * kRedSlices) conv_bwd_reduce_kernel(ConvBwdParams p, int64_t nparts)
{
    __shared__ float4 sw[kRedSlices][32];
    __shared__ float sb[kRedSlices][32];
    const int cl = threadIdx.x & 31, sl = threadIdx.x >> 5;
    const int c = blockIdx.x * 32 + cl;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    float ab = 0.0f;
    if (c < p.C_ch) {
        for (int64_t i0 = sl; i0 < nparts; i0 += 8 * kRedSlices) {
            float4 v[8];
            float b[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t i = i0 + (int64_t)u * kRedSlices;
                v[u] = i < nparts ? reinterpret_cast<const float4 *>(p.ws_dw)[i * p.C_ch + c]
                                  : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                b[u] = i < nparts ? p.ws_dbias[i * p.C_ch + c] : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                acc.x += v[u].x; acc.y += v[u].y; acc.z += v[u].z; acc.w += v[u].w;
                ab += b[u];
            }
        }
    }
    sw[sl][cl] = acc;
    sb[sl][cl] = ab;
    __syncthreads();
    if (sl == 0 && c < p.C_ch) {
        for (int k = 1; k < kRedSlices; ++k) {
            const float4 v = sw[k][cl];
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            ab += sb[k][cl];
        }
        reinterpret_cast<float4 *>(p.dw)[c] = acc;
        if (p.dbias) p.dbias[c] = ab;
    }
}

}  // namespace

int64_t conv_bwd_blocks(int64_t L) { return (L + kTB - 1) / kTB; }

int launch_conv_backward(const ConvBwdParams &p, int dtype, cudaStream_t st)
{
    const int64_t nblk = conv_bwd_blocks(p.L);
    // two channels per thread: P and N are multiples of 16, so a channel pair never straddles x, B, C
    const int64_t n = (int64_t)p.b * nblk * (p.C_ch / 2);
    const int64_t blocks = (n + kConvBwdThreads - 1) / kConvBwdThreads;
    if (blocks > 0x7fffffffLL) return 2;
    prof_begin(st, kKConvBwd);
    if (n > 0) {
        const int smem = (int)((sizeof(float2) + 2 * (dtype == 1 ? 2 : 4)) * kRingB * kConvBwdThreads);
        if (dtype == 1) {
            if (cudaFuncSetAttribute(conv_bwd2_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     smem) != cudaSuccess)
                return 7;
            conv_bwd2_kernel<__nv_bfloat16><<<(unsigned)blocks, kConvBwdThreads, smem, st>>>(p, nblk);
        } else {
            if (cudaFuncSetAttribute(conv_bwd2_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess)
                return 7;
            conv_bwd2_kernel<float><<<(unsigned)blocks, kConvBwdThreads, smem, st>>>(p, nblk);
        }
    }
    conv_bwd_reduce_kernel<<<(unsigned)((p.C_ch + 31) / 32), 32 * kRedSlices, 0, st>>>(p, (int64_t)p.b * nblk);
    prof_end(st, kKConvBwd);
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

}  // namespace ssd

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
// dtype is taken as the identity, and dz is fp32 with an accurate exponential.
#include "ssd_common.cuh"

namespace ssd {
namespace {

constexpr int kTB = 64;          // tokens per thread, walked from the last
constexpr int kConvBwdThreads = 256;

// dLoss/dv of channel c at row (bi, t)
__device__ __forceinline__ float dv_at(const ConvBwdParams &p, int64_t bi, int64_t t, int c)
{
    const int64_t row = bi * p.L + t;
    if (c < p.HP) return p.dx[row * p.HP + c];
    if (c < p.HP + p.GN) return p.dB[row * p.GN + (c - p.HP)];
    return p.dC[row * p.GN + (c - p.HP - p.GN)];
}

// dz = dv silu'(z) from the conv window u[t-3 .. t] (as token t's cell sees it)
__device__ __forceinline__ float dz_of(float dv, const float4 &wq, float bs, const float (&uw)[4])
{
    float z = bs;
    z = fmaf(wq.x, uw[0], z);
    z = fmaf(wq.y, uw[1], z);
    z = fmaf(wq.z, uw[2], z);
    z = fmaf(wq.w, uw[3], z);
    const float sg = 1.0f / (1.0f + expf(-z));
    return dv * (sg * (1.0f + z * (1.0f - sg)));
}

template <typename T>
__device__ __forceinline__ void load_window(const ConvBwdParams &p, int64_t bi, int64_t t, int c, float (&uw)[4])
{
#pragma unroll
    for (int k = 0; k < 4; ++k) uw[k] = cell_val<T>(p, bi, t, t - 3 + k, c);
}

template <typename T>
__device__ __forceinline__ float dz_at(const ConvBwdParams &p, int64_t bi, int64_t t, int c, const float4 &wq,
                                       float bs)
{
    if (t >= p.L) return 0.0f;
    float uw[4];
    load_window<T>(p, bi, t, c, uw);
    return dz_of(dv_at(p, bi, t, c), wq, bs, uw);
}

// One thread per (batch row, block of kTB tokens, channel); consecutive threads
// take consecutive channels, so every row access is coalesced.  The thread walks
// its block from the last token with the conv window of u in registers, one new
// row per token (rows before a cell come from its conv buffer).
// four CTAs per SM (at most 64 registers): enough warps to cover the loads of the serial walk
template <typename T>
__global__ void __launch_bounds__(kConvBwdThreads, 4) conv_bwd_kernel(ConvBwdParams p, int64_t nblk)
{
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)p.b * nblk * p.C_ch) return;
    const int c = (int)(gid % p.C_ch);
    const int64_t blk = (gid / p.C_ch) % nblk;
    const int64_t bi = gid / ((int64_t)p.C_ch * nblk);
    const int64_t t0 = blk * kTB;
    const int64_t t1 = min(p.L, t0 + kTB);
    const float4 wq = __ldg(reinterpret_cast<const float4 *>(p.w) + c);
    const float bs = p.bias ? __ldg(p.bias + c) : 0.0f;
    // window of dz at t'+0 .. t'+3, walked from t' = t1-1 down to t0
    float d1 = dz_at<T>(p, bi, t1, c, wq, bs), d2 = dz_at<T>(p, bi, t1 + 1, c, wq, bs),
          d3 = dz_at<T>(p, bi, t1 + 2, c, wq, bs);
    float gw0 = 0.0f, gw1 = 0.0f, gw2 = 0.0f, gw3 = 0.0f, gb = 0.0f;
    float uw[4];
    load_window<T>(p, bi, t1 - 1, c, uw);
    // a block never crosses a cell (blocks and cells are multiples of 64 tokens), so the window
    // only slides; each group of four tokens issues its loads before it computes
    for (int64_t tg = t1 - 1; tg >= t0; tg -= 4) {
        float dvv[4], un[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t t = tg - i;
            dvv[i] = t >= t0 ? dv_at(p, bi, t, c) : 0.0f;
            un[i] = t > t0 ? cell_val<T>(p, bi, t - 1, t - 4, c) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t t = tg - i;
            if (t < t0) break;
            const float d0 = dz_of(dvv[i], wq, bs, uw);
            float g = wq.w * d0;
            g = fmaf(wq.z, d1, g);
            g = fmaf(wq.y, d2, g);
            g = fmaf(wq.x, d3, g);
            if (p.dtail_out && t >= p.L - 3) g += p.dtail_out[(bi * 3 + (t - (p.L - 3))) * p.C_ch + c];
            p.du[(bi * p.L + t) * p.C_ch + c] = g;
            gb += d0;
            gw0 = fmaf(d0, uw[0], gw0);
            gw1 = fmaf(d0, uw[1], gw1);
            gw2 = fmaf(d0, uw[2], gw2);
            gw3 = fmaf(d0, uw[3], gw3);
            d3 = d2; d2 = d1; d1 = d0;
            uw[3] = uw[2]; uw[2] = uw[1]; uw[1] = uw[0]; uw[0] = un[i];
        }
    }
    const int64_t slot = (bi * nblk + blk) * p.C_ch + c;
    reinterpret_cast<float4 *>(p.ws_dw)[slot] = make_float4(gw0, gw1, gw2, gw3);
    p.ws_dbias[slot] = gb;
    if (blk == 0 && p.dtail_in) {
        // the rows before the sequence (positions -3, -2, -1): d1, d2, d3 now hold dz at 0, 1, 2
        float *dt = p.dtail_in + bi * 3 * p.C_ch + c;
        float g2 = fmaf(wq.z, d1, fmaf(wq.y, d2, wq.x * d3));   // position -1
        float g1 = fmaf(wq.y, d1, wq.x * d2);                   // position -2
        float g0 = wq.x * d1;                                   // position -3
        if (p.dtail_out) {
            // tail_out rows that are rows of tail_in when L < 3
            for (int r = 0; r < 3; ++r) {
                const int64_t pos = p.L - 3 + r;
                if (pos >= 0) continue;
                const float gt = p.dtail_out[(bi * 3 + r) * p.C_ch + c];
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

// dw and dbias: the partial sums of every (batch row, token block), added in a fixed order
__global__ void conv_bwd_reduce_kernel(ConvBwdParams p, int64_t nparts)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= p.C_ch) return;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    float ab = 0.0f;
    for (int64_t i = 0; i < nparts; ++i) {
        const float4 v = reinterpret_cast<const float4 *>(p.ws_dw)[i * p.C_ch + c];
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        ab += p.ws_dbias[i * p.C_ch + c];
    }
    reinterpret_cast<float4 *>(p.dw)[c] = acc;
    if (p.dbias) p.dbias[c] = ab;
}

}  // namespace

int64_t conv_bwd_blocks(int64_t L) { return (L + kTB - 1) / kTB; }

int launch_conv_backward(const ConvBwdParams &p, int dtype, cudaStream_t st)
{
    const int64_t nblk = conv_bwd_blocks(p.L);
    const int64_t n = (int64_t)p.b * nblk * p.C_ch;
    const int64_t blocks = (n + kConvBwdThreads - 1) / kConvBwdThreads;
    if (blocks > 0x7fffffffLL) return 2;
    prof_begin(st, kKConvBwd);
    if (n > 0) {
        if (dtype == 1) conv_bwd_kernel<__nv_bfloat16><<<(unsigned)blocks, kConvBwdThreads, 0, st>>>(p, nblk);
        else conv_bwd_kernel<float><<<(unsigned)blocks, kConvBwdThreads, 0, st>>>(p, nblk);
    }
    conv_bwd_reduce_kernel<<<(unsigned)((p.C_ch + 127) / 128), 128, 0, st>>>(p, (int64_t)p.b * nblk);
    prof_end(st, kKConvBwd);
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

}  // namespace ssd

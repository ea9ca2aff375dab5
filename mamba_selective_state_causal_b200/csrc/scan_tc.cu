// scan_tc.cu -- tensor-core path of the chunked selective scan for sm_100a:
// bf16 I/O, head dim P = 64, state dim N = 128, chunk Q = 128.
//
// Same decomposition as the CUDA-core path (scan_generic.cu): the sequence is
// cut into stripes; pass A computes each stripe's end state from a zero start,
// a chain pass links the stripes from h0, and pass C walks the chunks of each
// stripe from its exact entering state, emitting y, the state checkpoints
// every s tokens (pith.science verdict for arXiv 2411.19460,
// pith_extraction.key_machinery, "Algorithm 1" Sckpt) and h_final.
//
// Per chunk of 128 tokens of one head (cs = chunk-local cumulative dt*A, kept
// in log2 units so that exp(x) = ex2(x * log2 e)):
//   G  = C B^T                                     tcgen05, 128x128x128, TMEM
//   Pm = G o [exp(cs_i - cs_j) dt_j, j <= i]       CUDA cores, TMEM -> TMEM (bf16)
//   Yd = Pm X                                      tcgen05, A from TMEM, 128x64x128
//   Yo = C h_prev^T                                tcgen05, 128x128x128 (both heads)
//   y  = Yd + exp(cs_i) Yo + D x                   CUDA cores (fp32) -> smem -> TMA store
//   S  = B^T (w o X),  w_j = dt_j exp(cs_last - cs_j)   tcgen05, 128x128x128 (both heads)
//   h  = exp(cs_last) h + S                        fp32 state in TMEM, S accumulated into it
// Only non-positive differences of cs are exponentiated.  The state is kept in
// fp32; its bf16 copy only feeds the C h_prev^T product.  Both kernels take
// two heads per CTA: they share B (and C), so G is computed once per pair and
// the products with a shared operand run at N = 128.
//
// All waits are bounded (tc::mbar_wait): on a timeout the CTA raises an abort
// flag, every thread unwinds, outstanding MMAs and loads are drained, TMEM is
// freed and the device status word reports SSD_ERR_TIMEOUT.
#include <atomic>

#include <cuda.h>

#include "ssd_common.cuh"
#include "tc_ptx.cuh"

namespace ssd {

int launch_chain(const ScanParams &p, cudaStream_t st);

namespace {

using namespace tc;

constexpr int kQ = 128, kP = 64, kN = 128;
constexpr uint32_t kBox = 128 * 64 * 2;   // one 128-row x 64-col bf16 TMA box (16 KB)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct Maps {
    CUtensorMap x, B, C, y;
    CUtensorMap ux;     // fused conv: x columns of the conv input u, boxes of 136 rows (8-row halo)
};

constexpr int kHaloRows = 8;                                   // rows before a chunk in a fused X box
constexpr uint32_t kBoxX = kBox + kHaloRows * 128;             // a fused X box: 136 rows x 128 bytes

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Bounded wait whose outcome is the same for every lane of the warp, so that
// the warp stays converged for the .sync.aligned TMEM instructions after it.
__device__ __forceinline__ bool ewait(uint64_t *bar, uint32_t parity, volatile int *abort, uint64_t limit_ns)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, limit_ns));
}

// byte offset of 16-byte chunk c of row r in a 128B-swizzled tile of 128-byte rows
__device__ __forceinline__ uint32_t swz(int r, int c)
{
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint4 lds128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ void sts128(uint8_t *p, uint4 v) { *reinterpret_cast<uint4 *>(p) = v; }


// fp32 pair -> bf16x2 by integer rounding (half an ulp added, ties away from zero), on the
// integer pipe so that it runs beside the conversion unit; inputs are finite
__device__ __forceinline__ uint32_t pack_bf16x2_int(float lo, float hi)
{
    return __byte_perm(__float_as_uint(lo) + 0x8000u, __float_as_uint(hi) + 0x8000u, 0x7632);
}

__device__ __forceinline__ uint32_t scale_bf16x2_int(uint32_t v, float w)
{
    return pack_bf16x2_int(bf16_lo(v) * w, bf16_hi(v) * w);
}

// two fp32 products / fused multiply-adds in one instruction (sm_100 packed fp32, through the
// CUDA float2 intrinsics, which leave the register pairing to the compiler); each lane rounds
// exactly as the scalar instruction does
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

__device__ __forceinline__ float2 unpack2(uint32_t v) { return make_float2(bf16_lo(v), bf16_hi(v)); }

// Conv + SiLU of 8 channels (4 pairs) of one token: window m3 = u[t-3], m2, m1, cur = u[t],
// weights w[pair][tap] and bias as channel pairs, both already halved, so that the sum is
// h = z / 2 and SiLU(z) = z sigmoid(z) = h + h tanh(h) takes one hardware tanh and one fma.
// The same operations, in the same order and rounding, as the conv kernel's scalar code,
// two channels per instruction.
__device__ __forceinline__ uint4 conv8(const float2 (&w)[4][4], const float2 (&bs)[4], const float2 (&m3)[4],
                                       const float2 (&m2)[4], const float2 (&m1)[4], const float2 (&cur)[4])
{
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 h = fma2(w[i][0], m3[i], bs[i]);
        h = fma2(w[i][1], m2[i], h);
        h = fma2(w[i][2], m1[i], h);
        h = fma2(w[i][3], cur[i], h);
        float2 t;
        asm("tanh.approx.f32 %0, %1;" : "=f"(t.x) : "f"(h.x));
        asm("tanh.approx.f32 %0, %1;" : "=f"(t.y) : "f"(h.y));
        const float2 sg = fma2(h, t, h);
        o[i] = pack_bf16x2(sg.x, sg.y);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void unpack8(uint4 v, float2 (&f)[4])
{
    f[0] = unpack2(v.x); f[1] = unpack2(v.y); f[2] = unpack2(v.z); f[3] = unpack2(v.w);
}

// bf16 pair times w, rounded to nearest even (cvt)
__device__ __forceinline__ uint32_t scale_bf16x2_rn(uint32_t v, float2 w2)
{
    const float2 p = mul2(unpack2(v), w2);
    return pack_bf16x2(p.x, p.y);
}

__device__ __forceinline__ void raise_timeout(const ScanParams &p, volatile int *abort)
{
    *abort = 1;
    atomicOr(p.status, kDevTimeout);
}

// =============================================================== pass A
// One CTA per (stripe, head pair): S[n][(h,p)] = sum_j B[j][n] (w_h o X_h)[j][p]
// over the whole stripe, both heads side by side on N = 128, accumulated in
// TMEM.  Chunks are walked backwards so that the decay from each chunk to the
// stripe end (a suffix sum) is known when the chunk is scaled:
//   w_j = dt_j exp(sum of dt*A after token j, up to the stripe end).
// Warps 0..15 scale X in place (half a token row of one head per thread);
// warp 16 issues the TMA loads (B and X of both heads, 3-stage ring) and the
// MMAs; warp 17 runs the dt scan that yields w, up to three chunks ahead.
// Fused conv (kFused): each X box holds the chunk's 128 rows of the conv
// input u plus the 8 rows before it, and the scaling warps first turn u into
// x = silu(conv(u)) (rounded to bf16, as the conv kernel stores it), write
// that x to global memory for the output pass (a warp writes 4 whole 128-byte
// row segments per store), then scale: thread (head, 16-byte column, 4-row
// group) reads the 3 rows before its group, waits until every thread has (a
// bounded barrier), then rewrites its 4 rows in place.
constexpr int kStagesA = 3;
constexpr int kScaleWarpsA = 16;
constexpr int kThreadsA = 32 * (kScaleWarpsA + 2);
constexpr uint32_t kStageA = 2 * kBox + 2 * kBoxX;   // B box 0, B box 1, X box of head a, of head b

struct SmemA {
    uint8_t stage[kStagesA][kStageA];    // an X box's MMA operand starts kHaloRows rows in
    float w[kStagesA][2][kQ];            // w_j of head a / b for the chunk in the stage
    uint64_t full[kStagesA], w_ready[kStagesA], xw_ready[kStagesA], empty[kStagesA], halo_read[kStagesA];
    uint64_t acc_full, fin;
    uint32_t tmem;
    int abort;
};

template <bool kFused>
__global__ void __launch_bounds__(kThreadsA, 1)
stripe_state_tc_kernel(const __grid_constant__ Maps maps, const ScanParams p)
{
    extern __shared__ __align__(1024) uint8_t sma_raw[];
    SmemA &s = *reinterpret_cast<SmemA *>((reinterpret_cast<uintptr_t>(sma_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t unit = blockIdx.x;
    const int hpairs = p.H / 2;
    const int ha = 2 * (int)(unit % hpairs);
    const int64_t k = (unit / hpairs) % p.ns;
    const int bi = (int)(unit / ((int64_t)hpairs * p.ns));
    const int g = (int)((int64_t)ha * p.G / p.H);  // both heads of the pair share a group (H/G even)
    const int64_t s0 = k * p.T;
    const int64_t s1 = min(p.L, s0 + p.T);
    const int nc = (int)((s1 - s0 + kQ - 1) / kQ);
    const uint64_t lim = p.wait_limit_ns;
    constexpr int PN = kP * kN;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStagesA; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.w_ready[i], 1);
            mbar_init(&s.xw_ready[i], kScaleWarpsA);
            mbar_init(&s.empty[i], 1);
            mbar_init(&s.halo_read[i], kScaleWarpsA);
        }
        mbar_init(&s.acc_full, 1);
        mbar_init(&s.fin, 1);
        s.abort = 0;
        fence_mbar_init();
        prefetch_tmap(kFused ? &maps.ux : &maps.x);
        prefetch_tmap(&maps.B);
    }
    if (warp == 0) { tmem_alloc(&s.tmem, 128); tmem_relinquish(); }
    __syncthreads();
    tc_fence_after();
    const uint32_t tS = s.tmem;
    volatile int *abort = &s.abort;
    const bool live = unit != p.test_drop_unit;

    if (warp < kScaleWarpsA) {
        // ================================================= scaling warps
        const int hd = warp >> 3, j = 32 * (warp & 3) + lane, c0 = 4 * ((warp >> 2) & 1);
        // fused conv: 16-byte column ch (8 channels) of rows 4 rg .. 4 rg + 3 of head hd
        const int ch = lane & 7, rg = (lane >> 3) + 4 * (warp & 7);
        float2 cw[4][4], cb[4];   // weights [channel pair][tap] and bias of this thread's 8 channels
        if (kFused) {
            const int c0ch = (ha + hd) * kP + 8 * ch;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 qa = __ldg(reinterpret_cast<const float4 *>(p.conv_w) + c0ch + 2 * i);
                const float4 qb = __ldg(reinterpret_cast<const float4 *>(p.conv_w) + c0ch + 2 * i + 1);
                // halved (exact) for conv8's h = z / 2
                cw[i][0] = make_float2(0.5f * qa.x, 0.5f * qb.x); cw[i][1] = make_float2(0.5f * qa.y, 0.5f * qb.y);
                cw[i][2] = make_float2(0.5f * qa.z, 0.5f * qb.z); cw[i][3] = make_float2(0.5f * qa.w, 0.5f * qb.w);
                cb[i] = p.conv_bias ? make_float2(0.5f * __ldg(p.conv_bias + c0ch + 2 * i), 0.5f * __ldg(p.conv_bias + c0ch + 2 * i + 1))
                                    : make_float2(0.0f, 0.0f);
            }
        }
        bool ok = true;
        for (int it = 0; it < nc; ++it) {
            const int st = it % kStagesA;
            const uint32_t ph = (uint32_t)(it / kStagesA) & 1;
            ok = ewait(&s.full[st], ph, abort, lim) && ewait(&s.w_ready[st], ph, abort, lim);
            if (!ok) break;
            if (kFused) {
                uint8_t *box = s.stage[st] + 2 * kBox + hd * kBoxX;   // row r of the chunk is box row r + 8
                const int64_t t0 = s0 + (int64_t)(nc - 1 - it) * kQ;
                float2 m3[4], m2[4], m1[4];
                if (t0 == 0 && rg == 0) {
                    // the rows before the sequence: the conv buffer handed in, or zeros
                    const __nv_bfloat16 *tin = p.conv_tail
                        ? reinterpret_cast<const __nv_bfloat16 *>(p.conv_tail) + (int64_t)bi * 3 * p.conv_cch +
                              (ha + hd) * kP + 8 * ch
                        : nullptr;
                    const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
                    unpack8(tin ? *reinterpret_cast<const uint4 *>(tin) : z4, m3);
                    unpack8(tin ? *reinterpret_cast<const uint4 *>(tin + p.conv_cch) : z4, m2);
                    unpack8(tin ? *reinterpret_cast<const uint4 *>(tin + 2 * p.conv_cch) : z4, m1);
                } else {
                    const int r0 = 4 * rg + kHaloRows;
                    unpack8(lds128(box + swz(r0 - 3, ch)), m3);
                    unpack8(lds128(box + swz(r0 - 2, ch)), m2);
                    unpack8(lds128(box + swz(r0 - 1, ch)), m1);
                }
                // every thread has read the rows before its group: rows may now be rewritten
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.halo_read[st]);
                ok = ewait(&s.halo_read[st], ph, abort, lim);
                if (!ok) break;
                // x rows 4 rg .. 4 rg + 3 of the chunk in global memory (rows past the sequence end skipped)
                __nv_bfloat16 *xo = reinterpret_cast<__nv_bfloat16 *>(p.conv_v) + (int64_t)bi * p.conv_vbs +
                                    (t0 + 4 * rg) * p.conv_vrs + (ha + hd) * kP + 8 * ch;
                const int64_t nrows = s1 - t0 - 4 * rg;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = 4 * rg + i;
                    uint8_t *a = box + swz(r + kHaloRows, ch);
                    float2 cur[4];
                    unpack8(lds128(a), cur);
                    uint4 v = conv8(cw, cb, m3, m2, m1, cur);
                    if (i < nrows) *reinterpret_cast<uint4 *>(xo) = v;
                    xo += p.conv_vrs;
                    const float w = s.w[st][hd][r];
                    const float2 w2 = make_float2(w, w);
                    v.x = scale_bf16x2_rn(v.x, w2); v.y = scale_bf16x2_rn(v.y, w2);
                    v.z = scale_bf16x2_rn(v.z, w2); v.w = scale_bf16x2_rn(v.w, w2);
                    sts128(a, v);
#pragma unroll
                    for (int e = 0; e < 4; ++e) { m3[e] = m2[e]; m2[e] = m1[e]; m1[e] = cur[e]; }
                }
            } else {
                const float w = s.w[st][hd][j];
                const float2 w2 = make_float2(w, w);
                uint8_t *xrow = s.stage[st] + 2 * kBox + hd * kBoxX + kHaloRows * 128;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const uint32_t o = swz(j, c0 + cc);
                    uint4 vv = lds128(xrow + o);
                    vv.x = scale_bf16x2_rn(vv.x, w2); vv.y = scale_bf16x2_rn(vv.y, w2);
                    vv.z = scale_bf16x2_rn(vv.z, w2); vv.w = scale_bf16x2_rn(vv.w, w2);
                    sts128(xrow + o, vv);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.xw_ready[st]);
        }
        if (!ok) {
            if (lane == 0) raise_timeout(p, abort);
        } else if (warp < 8) {
            if (ewait(&s.acc_full, 0, abort, lim)) {
                // S[n][(h,p)]: lane quarter q holds state rows n = 32 q .. 32 q + 31; warp 4 hd' + q takes head hd'
                tc_fence_after();
                const int q = warp & 3, hq = warp >> 2, n = 32 * q + lane;
                const uint32_t lane_base = (uint32_t)(32 * q) << 16;
                float *dst = p.ws_S + (((int64_t)bi * p.ns + k) * p.H + ha + hq) * PN + n;
#pragma unroll
                for (int c32 = 0; c32 < 2; ++c32) {
                    uint32_t a[32];
                    tmem_ld32(tS + lane_base + 64 * hq + 32 * c32, a);
                    tmem_wait_ld(a);
#pragma unroll
                    for (int pp = 0; pp < 32; ++pp) dst[(int64_t)(32 * c32 + pp) * kN] = __uint_as_float(a[pp]);
                }
            } else if (lane == 0) {
                raise_timeout(p, abort);
            }
        }
    } else if (warp == kScaleWarpsA) {
        // ================================================= issuing warp (the whole warp waits, lane 0 issues)
        int issued = 0;   // lane 0: loads issued (consumed loads are those of the MMAs issued)
        auto issue_load = [&](int it) {
            const int st = it % kStagesA;
            const int t0 = (int)(s0 + (int64_t)(nc - 1 - it) * kQ);
            uint8_t *sb = s.stage[st];
            uint8_t *xb = sb + 2 * kBox;
            if (kFused) {
                // the chunk's rows of u and the 8 before them (a negative start row reads zeros)
                mbar_arrive_expect_tx(&s.full[st], 2 * kBox + 2 * kBoxX);
                tma_load_3d(sb, &maps.B, &s.full[st], g * kN, t0, bi);
                tma_load_3d(sb + kBox, &maps.B, &s.full[st], g * kN + 64, t0, bi);
                tma_load_3d(xb, &maps.ux, &s.full[st], ha * kP, t0 - kHaloRows, bi);
                tma_load_3d(xb + kBoxX, &maps.ux, &s.full[st], (ha + 1) * kP, t0 - kHaloRows, bi);
            } else {
                mbar_arrive_expect_tx(&s.full[st], 4 * kBox);
                tma_load_3d(sb, &maps.B, &s.full[st], g * kN, t0, bi);
                tma_load_3d(sb + kBox, &maps.B, &s.full[st], g * kN + 64, t0, bi);
                tma_load_3d(xb + kHaloRows * 128, &maps.x, &s.full[st], ha * kP, t0, bi);
                tma_load_3d(xb + kBoxX + kHaloRows * 128, &maps.x, &s.full[st], (ha + 1) * kP, t0, bi);
            }
            ++issued;
        };
        const uint32_t id_s = idesc_bf16(128, 128, 1, 1);   // A = B^T (MN-major), B = w o X (MN-major)
        // descriptors of each stage's B^T and w o X, built once; a K-step adds 2048 B (128 units)
        uint64_t dB[kStagesA], dXw[kStagesA];
#pragma unroll
        for (int i = 0; i < kStagesA; ++i) {
            const uint32_t sb = smem_u32(s.stage[i]);
            dB[i] = smem_desc(sb, kBox, 1024);
            dXw[i] = smem_desc(sb + 2 * kBox + kHaloRows * 128, kBoxX, 1024);
        }
        bool ok = live;
        int mmas = 0;
        if (ok && lane == 0)
            for (int it = 0; it < min(nc, kStagesA); ++it) issue_load(it);
        for (int it = 0; ok && it < nc; ++it) {
            const int st = it % kStagesA;
            ok = ewait(&s.xw_ready[st], (uint32_t)(it / kStagesA) & 1, abort, lim);
            if (!ok) break;
            tc_fence_after();
            if (lane == 0) {
                const uint64_t db = st == 0 ? dB[0] : (st == 1 ? dB[1] : dB[2]);
                const uint64_t dx = st == 0 ? dXw[0] : (st == 1 ? dXw[1] : dXw[2]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tS, db + (uint64_t)(kk * 128), dx + (uint64_t)(kk * 128), id_s, it > 0 || kk > 0);
                mma_commit(&s.empty[st]);
            }
            ++mmas;
            __syncwarp();
            // refill this stage with step it + 3 once the product has read it, so that three
            // stages stay in flight (the next product cannot start before this one ends anyway)
            if (it + kStagesA < nc) {
                ok = ewait(&s.empty[st], (uint32_t)(it / kStagesA) & 1, abort, lim);
                if (!ok) break;
                if (lane == 0) issue_load(it + kStagesA);
                __syncwarp();
            }
        }
        if (lane == 0) {
            if (live && !ok) raise_timeout(p, abort);
            mma_commit(&s.acc_full);
            mma_commit(&s.fin);
            mbar_wait(&s.fin, 0, nullptr, 100000000ull);
            if (*abort) {
                // drain: every load issued but not consumed by an MMA
                for (int it = mmas; it < issued; ++it)
                    mbar_wait(&s.full[it % kStagesA], (uint32_t)(it / kStagesA) & 1, nullptr, 100000000ull);
            }
        }
        __syncwarp();
    } else {
        // ================================================= scan warp: w of every step, in order
        const float A2a = p.A[ha] * kLog2e, A2b = p.A[ha + 1] * kLog2e;
        float sufa = 0.0f, sufb = 0.0f;     // sum of dt*A (log2 units) after the chunks scanned so far
        float2 dtn[4];                      // dt of tokens 4 lane .. 4 lane + 3 of the next chunk
        auto load_dt = [&](int it) {
            const int64_t t0 = s0 + (int64_t)(nc - 1 - it) * kQ;
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
                const int64_t t = t0 + 4 * lane + kq;
                dtn[kq] = t < s1 ? *reinterpret_cast<const float2 *>(p.dt + ((int64_t)bi * p.L + t) * p.H + ha)
                                 : make_float2(0.0f, 0.0f);
            }
        };
        bool ok = live;
        if (ok) load_dt(0);
        for (int it = 0; ok && it < nc; ++it) {
            const int st = it % kStagesA;
            // the scaling warps are done with w[st] once step it - 3 is scaled
            if (it >= kStagesA) {
                ok = ewait(&s.xw_ready[st], (uint32_t)(it / kStagesA - 1) & 1, abort, lim);
                if (!ok) break;
            }
            float ca[4], cb[4];
            float sa = 0.0f, sb = 0.0f;
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
                sa += dtn[kq].x * A2a; ca[kq] = sa;
                sb += dtn[kq].y * A2b; cb[kq] = sb;
            }
            const float2 dcur[4] = {dtn[0], dtn[1], dtn[2], dtn[3]};
            if (it + 1 < nc) load_dt(it + 1);
            float ia = sa, ib = sb;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float ta = __shfl_up_sync(0xffffffffu, ia, o);
                const float tb = __shfl_up_sync(0xffffffffu, ib, o);
                if (lane >= o) { ia += ta; ib += tb; }
            }
            float xa = __shfl_up_sync(0xffffffffu, ia, 1), xb = __shfl_up_sync(0xffffffffu, ib, 1);
            if (lane == 0) { xa = 0.0f; xb = 0.0f; }
            const float tota = __shfl_sync(0xffffffffu, ia, 31), totb = __shfl_sync(0xffffffffu, ib, 31);
            // decay from token j (exclusive) to the stripe end: tot - cs_j + suffix of the later chunks
            reinterpret_cast<float4 *>(s.w[st][0])[lane] =
                make_float4(dcur[0].x * ex2(tota - (ca[0] + xa) + sufa), dcur[1].x * ex2(tota - (ca[1] + xa) + sufa),
                            dcur[2].x * ex2(tota - (ca[2] + xa) + sufa), dcur[3].x * ex2(tota - (ca[3] + xa) + sufa));
            reinterpret_cast<float4 *>(s.w[st][1])[lane] =
                make_float4(dcur[0].y * ex2(totb - (cb[0] + xb) + sufb), dcur[1].y * ex2(totb - (cb[1] + xb) + sufb),
                            dcur[2].y * ex2(totb - (cb[2] + xb) + sufb), dcur[3].y * ex2(totb - (cb[3] + xb) + sufb));
            sufa += tota;
            sufb += totb;
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.w_ready[st]);
        }
        if (lane == 0) {
            if (live && !ok) raise_timeout(p, abort);
            if (ok && !*abort) {
                p.ws_dA[((int64_t)bi * p.ns + k) * p.H + ha] = sufa * kLn2;
                p.ws_dA[((int64_t)bi * p.ns + k) * p.H + ha + 1] = sufb * kLn2;
            }
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tS, 128);
}

// =============================================================== pass C
// One CTA per (stripe, head pair), one CTA per SM: 16 compute warps, an issuing
// warp, a store warp and a B/C warp.  The two heads share their B and C tiles
// and G = C B^T; the chunks of the stripe are walked in order.
//
// The output accumulator T of a chunk first receives Ys = C [hp_a | hp_b]^T
// (the contribution of the state entering the chunk), which the compute warps
// scale row by row by exp(cs_i); Y = Pm X then accumulates onto it, so the
// epilogue only adds D x.  The masked decay Pm of a chunk is formed during the
// previous chunk, under its S, so per chunk the compute warps scale T (Y may
// start at once), write w o X into the C half of the chunk's B/C slot (spent
// once G and Ys have read C) while Y runs, form the next chunk's decay once Y
// has read Pm while S = B^T (w o X) runs, and then take the state step and y.
// Ys of chunk c+1 runs while the warps form y of chunk c.  (Issuing a group of
// MMAs holds the issuing lane for most of its run time, and a load can take a
// microsecond to land: loads, stores and G, whose operands arrive by TMA, are
// kept off the warp that issues Y, S and Ys.)
// Issuing warp, per chunk c (the whole warp waits, one lane issues):
//   Pm written and T scaled -> Y_a = Pm_a X_a, Y_b = Pm_b X_b accumulated into
//   T; w o X ready -> S = B^T [Xw_a | Xw_b], accumulated straight into the fp32
//   state H in TMEM; T read and hp of chunk c+1 written -> Ys of chunk c+1
//   into T.  (G and Ys of chunk 0 in the prologue.)
// B/C warp, per chunk c: products done -> the B/C slot is refilled with chunk
// c+2; the decay of chunk c+1 has read G, the slot has landed and Ys of chunk
// c+1 is done -> G of chunk c+2 into R0.
// Store warp, per chunk c: y staged -> TMA store of y, and, once the store has
// read its slot, X of chunk c+2 is loaded there.  Chunk c's X sits in X slot
// c & 1 and its y is staged back in place.
// Warp 4 (no masked-decay work of its own) also publishes the chunk cumsum of
// dt*A of both heads for chunk c+1 once every warp has written chunk c's w o X
// (the last use of chunk c's values before the next decay).
// Compute warp (TMEM lane quarter q = warp & 3, column slice cs = warp >> 2 of
// the 128 (head, p) columns; head hd = cs >> 1), per chunk c:
//   T *= exp(cs_i) on its rows and columns (T holds Ys)
//   w o X of head hd into the C half of the B/C slot (rows split over the
//         head's 8 warps)
//   mask of chunk c+1: Pm columns 32 cs .. 32 cs + 31, i.e. head hd's 32-token
//         column blocks 2 (cs & 1) and 2 (cs & 1) + 1 of its 32 rows:
//         Pm[i][j] = G[i][j] exp(cs_i - cs_j) dt_j (j <= i), 0 above
//   the state step of chunk c+1: H (h after chunk c) -> bf16 copy hp,
//         checkpoint, then H = exp(cs_last(c+1)) H, to which S of chunk c+1 is added;
//   then y = T + D x in fp32 -> bf16 -> the X slot (same swizzle as the y map)
// A warp reads and writes only TMEM columns it owns (and G's, which nobody
// writes while the decay runs), so no barrier among the compute warps is
// needed; hand-offs go through mbarriers (one arrival per warp).
// TMEM (512 columns): R0 = 0..127 G (fp32); R1 = 128..255 Pm_a | Pm_b (bf16);
// T = 256..383 (a | b); H = 384..511 (a | b), the fp32 state, rows n.
// Shared memory: B/C ring of 2 (a slot holds a chunk's C and B, then its w o X
// in the C half), two X slots (a chunk's X, then its y), hp, and the per-head
// scan values (about 227 KB).
constexpr int kComputeWarps = 16;
constexpr int kThreadsC = 32 * (kComputeWarps + 3);

struct SmemC {
    uint8_t bc[2][4 * kBox];   // ring slot: C box 0, C box 1, B box 0, B box 1; later w o X in the C half
    uint8_t x[2][2 * kBox];    // X slot: head a box, head b box (X, then y)
    uint8_t hp[2 * kBox];      // bf16 h_prev of head a, head b (rows n, cols p), 128B-swizzled
    float cvs[2][kQ];          // chunk-inclusive cumsum of dt*A (log2 units), per head
    float dvs[2][kQ];          // dt, per head
    float fs[2][3 * 32];       // dt_j exp(cs_end(J) - cs_j) for the 32-token blocks J = 0..2
    uint64_t full_bc[2], full_x[2], g_done, ys_done, ymma_done, mma_done[2];   // TMA / MMA / issuer -> warps
    uint64_t fin, fin2;                                                        // end of each issuing warp's MMAs
    uint64_t pmw, pm_ready, xw_ready, ys_go, st0_ready, scan_ready;            // warps -> issuing warp
    uint64_t y_ready[2];       // warps -> store warp, by X slot (the store warp may still be storing the
                               // previous chunk's y when this one's is staged)
    uint32_t tmem;
    int abort;
};

__global__ void __launch_bounds__(kThreadsC, 1)
chunk_output_tc_kernel(const __grid_constant__ Maps maps, const ScanParams p)
{
    extern __shared__ __align__(1024) uint8_t smc_raw[];
    SmemC &s = *reinterpret_cast<SmemC *>(smc_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int HP = p.H >> 1;
    const int64_t unit = blockIdx.x;
    const int ha = 2 * (int)(unit % HP);         // head a; head b = ha + 1
    const int64_t k = (unit / HP) % p.ns;
    const int bi = (int)(unit / ((int64_t)HP * p.ns));
    const int g = (int)((int64_t)ha * p.G / p.H);
    const int64_t s0 = k * p.T;
    const int64_t s1 = min(p.L, s0 + p.T);
    const int nc = (int)((s1 - s0 + kQ - 1) / kQ);
    const uint64_t lim = p.wait_limit_ns;
    constexpr int PN = kP * kN;

    // the 128B-swizzled tiles need a 1024-byte aligned base (no room to pad)
    if (smem_u32(smc_raw) & 1023u) {
        if (tid == 0) atomicOr(p.status, kDevUnsupported);
        return;
    }
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) { mbar_init(&s.full_bc[i], 1); mbar_init(&s.full_x[i], 1); }
        mbar_init(&s.g_done, 1);
        mbar_init(&s.ys_done, 1);
        mbar_init(&s.ymma_done, 1);
        mbar_init(&s.mma_done[0], 1);
        mbar_init(&s.mma_done[1], 1);
        mbar_init(&s.fin, 1);
        mbar_init(&s.fin2, 1);
        mbar_init(&s.pmw, kComputeWarps);
        mbar_init(&s.pm_ready, kComputeWarps);
        mbar_init(&s.xw_ready, kComputeWarps);
        mbar_init(&s.ys_go, kComputeWarps);
        mbar_init(&s.y_ready[0], kComputeWarps);
        mbar_init(&s.y_ready[1], kComputeWarps);
        mbar_init(&s.st0_ready, kComputeWarps);
        mbar_init(&s.scan_ready, 1);
        s.abort = 0;
        fence_mbar_init();
        prefetch_tmap(&maps.x);
        prefetch_tmap(&maps.B);
        prefetch_tmap(&maps.C);
        prefetch_tmap(&maps.y);
    }
    if (warp == 0) { tmem_alloc(&s.tmem, 512); tmem_relinquish(); }
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = s.tmem;
    const uint32_t tG = tm, tPm = tm + 128, tT = tm + 256, tH = tm + 384;
    volatile int *abort = &s.abort;
    const bool live = unit != p.test_drop_unit;

    if (warp < kComputeWarps) {
        // ================================================= compute warps
        const int q = warp & 3, cs = warp >> 2, hd = cs >> 1, p0 = 32 * (cs & 1);
        const int r = 32 * q + lane;             // token row / TMEM lane / state row n
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int hh = ha + hd;
        auto fail = [&]() { if (lane == 0) raise_timeout(p, abort); };

        // state entering the stripe -> H: thread (n = r, cs) owns h[p0 .. p0 + 31][n] of head hh
        {
            const float *hin = (k == 0) ? (p.h0 ? p.h0 + ((int64_t)bi * p.H + hh) * PN : nullptr)
                                        : p.ws_hin + (((int64_t)bi * p.ns + k) * p.H + hh) * PN;
            uint32_t hv[32];
#pragma unroll
            for (int pp = 0; pp < 32; ++pp) hv[pp] = __float_as_uint(hin ? hin[(p0 + pp) * kN + r] : 0.0f);
            tmem_st32(tH + lane_base + 32 * cs, hv);
            tmem_wait_st();
        }
        // the checkpoint slot of the state after the chunk ending at t_end, or -1
        const int64_t n_ckpt = p.s > 0 ? p.L / p.s : 0;
        auto ckpt_slot = [&](int64_t t_end) -> int64_t {
            if (!p.h_ckpt || p.s <= 0 || t_end > s1 || t_end % p.s != 0) return -1;
            const int64_t kc = t_end / p.s - 1;
            return kc < n_ckpt ? kc : -1;
        };
        auto store_state = [&](float *dst, const uint32_t (&hv)[32]) {
#pragma unroll
            for (int pp = 0; pp < 32; ++pp) dst[pp * kN] = __uint_as_float(hv[pp]);
        };
        auto ckpt_ptr = [&](int64_t kc) {
            return p.h_ckpt + (((int64_t)bi * n_ckpt + kc) * p.H + hh) * PN + (int64_t)p0 * kN + r;
        };

        // chunk cumsum of both heads (warp 4, which has no masked-decay work): lane l holds
        // tokens 4 l .. 4 l + 3; dt is prefetched a chunk ahead
        const float A2a = p.A[ha] * kLog2e, A2b = p.A[ha + 1] * kLog2e;
        float2 dtn[4];
        auto load_dt = [&](int c) {
            const int64_t t0 = s0 + (int64_t)c * kQ;
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
                const int64_t t = t0 + 4 * lane + kq;
                dtn[kq] = t < s1 ? *reinterpret_cast<const float2 *>(p.dt + ((int64_t)bi * p.L + t) * p.H + ha)
                                 : make_float2(0.0f, 0.0f);
            }
        };
        auto scan = [&]() {
            float ca[4], cb[4];
            float sa = 0.0f, sb = 0.0f;
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
                sa += dtn[kq].x * A2a; ca[kq] = sa;
                sb += dtn[kq].y * A2b; cb[kq] = sb;
            }
            float ia = sa, ib = sb;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float ta = __shfl_up_sync(0xffffffffu, ia, o);
                const float tb = __shfl_up_sync(0xffffffffu, ib, o);
                if (lane >= o) { ia += ta; ib += tb; }
            }
            float xa = __shfl_up_sync(0xffffffffu, ia, 1), xb = __shfl_up_sync(0xffffffffu, ib, 1);
            if (lane == 0) { xa = 0.0f; xb = 0.0f; }
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) { ca[kq] += xa; cb[kq] += xb; }
            // cumsum at the end of this lane's 32-token block (token 32 J + 31 = lane 8 J + 7)
            const float ea = __shfl_sync(0xffffffffu, ca[3], lane | 7);
            const float eb = __shfl_sync(0xffffffffu, cb[3], lane | 7);
            reinterpret_cast<float4 *>(s.cvs[0])[lane] = make_float4(ca[0], ca[1], ca[2], ca[3]);
            reinterpret_cast<float4 *>(s.cvs[1])[lane] = make_float4(cb[0], cb[1], cb[2], cb[3]);
            reinterpret_cast<float4 *>(s.dvs[0])[lane] = make_float4(dtn[0].x, dtn[1].x, dtn[2].x, dtn[3].x);
            reinterpret_cast<float4 *>(s.dvs[1])[lane] = make_float4(dtn[0].y, dtn[1].y, dtn[2].y, dtn[3].y);
            if (lane < 24) {
                reinterpret_cast<float4 *>(s.fs[0])[lane] =
                    make_float4(dtn[0].x * ex2(ea - ca[0]), dtn[1].x * ex2(ea - ca[1]),
                                dtn[2].x * ex2(ea - ca[2]), dtn[3].x * ex2(ea - ca[3]));
                reinterpret_cast<float4 *>(s.fs[1])[lane] =
                    make_float4(dtn[0].y * ex2(eb - cb[0]), dtn[1].y * ex2(eb - cb[1]),
                                dtn[2].y * ex2(eb - cb[2]), dtn[3].y * ex2(eb - cb[3]));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.scan_ready);
        };

        const bool scan_warp = warp == 4;
        if (scan_warp && live) {
            load_dt(0);
            scan();
            if (nc > 1) load_dt(1);
        }
        const float Dh = p.D ? p.D[hh] : 0.0f;

        // H = h after chunk c-1: its bf16 copy feeds C hp^T of chunk c (checkpointed when a
        // checkpoint ends there), then H *= exp(cs_last(c)), to which chunk c's S is added.
        auto state_step = [&](int c, uint32_t (&hv)[32]) {
            const int64_t kc = c > 0 ? ckpt_slot(s0 + (int64_t)c * kQ) : -1;
            if (kc >= 0) store_state(ckpt_ptr(kc), hv);
            uint8_t *dst = s.hp + hd * kBox;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                uint4 v;
                v.x = pack_bf16x2_int(__uint_as_float(hv[8 * c4 + 0]), __uint_as_float(hv[8 * c4 + 1]));
                v.y = pack_bf16x2_int(__uint_as_float(hv[8 * c4 + 2]), __uint_as_float(hv[8 * c4 + 3]));
                v.z = pack_bf16x2_int(__uint_as_float(hv[8 * c4 + 4]), __uint_as_float(hv[8 * c4 + 5]));
                v.w = pack_bf16x2_int(__uint_as_float(hv[8 * c4 + 6]), __uint_as_float(hv[8 * c4 + 7]));
                sts128(dst + swz(r, (p0 >> 3) + c4), v);
            }
            const float dec = ex2(s.cvs[hd][kQ - 1]);
#pragma unroll
            for (int pp = 0; pp < 32; ++pp) hv[pp] = __float_as_uint(dec * __uint_as_float(hv[pp]));
            tmem_st32(tH + lane_base + 32 * cs, hv);
        };
        // y = T + D x for 16 columns (fp32) -> bf16, in place over x in the X slot (same
        // swizzle as the y map)
        auto y_half = [&](uint8_t *xs, const uint32_t (&tv)[16], int hf) {
            uint8_t *dst = xs + hd * kBox;
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                uint8_t *a = dst + swz(r, (p0 >> 3) + 2 * hf + c2);
                uint4 v = lds128(a);
                uint32_t *vw = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    const int i = 8 * c2 + 2 * e2;
                    vw[e2] = pack_bf16x2(fmaf(Dh, bf16_lo(vw[e2]), __uint_as_float(tv[i])),
                                         fmaf(Dh, bf16_hi(vw[e2]), __uint_as_float(tv[i + 1])));
                }
                sts128(a, v);
            }
        };

        // masked decay of the chunk whose scan values are published: column blocks
        // J = 2 (cs & 1) + jb of head hd, rows of quarter q (G of that chunk is in TMEM, and
        // Y of the chunk before it has read Pm)
        auto decay = [&]() {
            const float csr = s.cvs[hd][r];
#pragma unroll
            for (int jb = 0; jb < 2; ++jb) {
                const int J = 2 * (cs & 1) + jb;
                uint32_t pk[16];
                if (J < q) {
                    // whole block below the diagonal: exp(cs_r - cs_j) = exp(cs_r - m_J) exp(m_J - cs_j)
                    const float E = ex2(csr - s.cvs[hd][32 * J + 31]);
                    const float2 E2 = make_float2(E, E);
                    uint32_t gv[32];
                    tmem_ld32(tG + lane_base + 32 * J, gv);
                    tmem_wait_ld(gv);
                    const float4 *f4 = reinterpret_cast<const float4 *>(&s.fs[hd][32 * J]);
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 f = f4[i4];
                        const float2 a = mul2(make_float2(__uint_as_float(gv[4 * i4]), __uint_as_float(gv[4 * i4 + 1])),
                                              mul2(make_float2(f.x, f.y), E2));
                        const float2 b = mul2(make_float2(__uint_as_float(gv[4 * i4 + 2]), __uint_as_float(gv[4 * i4 + 3])),
                                              mul2(make_float2(f.z, f.w), E2));
                        pk[2 * i4] = pack_bf16x2(a.x, a.y);
                        pk[2 * i4 + 1] = pack_bf16x2(b.x, b.y);
                    }
                } else if (J == q) {
                    // diagonal block as 16x16 quarters: the two on the diagonal exponentiate each
                    // entry; the one below factors through m = cs at the block's column 15
                    uint32_t gv[32];
                    tmem_ld32(tG + lane_base + 32 * J, gv);
                    tmem_wait_ld(gv);
                    const float *cvb = &s.cvs[hd][32 * J], *dvb = &s.dvs[hd][32 * J];
                    const float m16 = cvb[15];
                    const bool lo = lane < 16;
                    const float a_r = ex2(csr - m16);                                   // <= 1 for lane >= 16
                    const float b_own = dvb[lane & 15] * ex2(m16 - cvb[lane & 15]);     // <= dt for lane < 16
                    const int xo = lo ? 0 : 16;
#pragma unroll
                    for (int k2 = 0; k2 < 8; ++k2) {
                        float vl[2], vh[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int k = 2 * k2 + e;
                            const int x = xo + k;
                            const float g_x = __uint_as_float(lo ? gv[k] : gv[16 + k]);
                            float t = g_x * ex2(csr - cvb[x]) * dvb[x];
                            t = x > lane ? 0.0f : t;
                            const float bk = __shfl_sync(0xffffffffu, b_own, k);
                            vl[e] = lo ? t : __uint_as_float(gv[k]) * (a_r * bk);
                            vh[e] = lo ? 0.0f : t;
                        }
                        pk[k2] = pack_bf16x2(vl[0], vl[1]);
                        pk[8 + k2] = pack_bf16x2(vh[0], vh[1]);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = 0u;
                }
                tmem_st16(tPm + lane_base + 16 * (2 * cs + jb), pk);
            }
        };

        bool ok = ewait(&s.scan_ready, 0, abort, lim);
        if (ok) {
            uint32_t hv[32];
            tmem_ld32(tH + lane_base + 32 * cs, hv);
            tmem_wait_ld(hv);
            state_step(0, hv);
            tmem_wait_st();
            fence_proxy_async_smem();   // hp, read by Ys of chunk 0
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.st0_ready);
            // the masked decay of chunk 0
            ok = ewait(&s.g_done, 0, abort, lim);
            if (ok) {
                tc_fence_after();
                decay();
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.pmw);
            }
        }
        if (!ok) fail();
        for (int c = 0; ok && c < nc; ++c) {
            uint8_t *xs = s.x[c & 1];

            // ---- T (= Ys of this chunk) *= exp(cs_r) on this warp's rows and columns
            if (!ewait(&s.ys_done, c & 1, abort, lim)) { fail(); break; }
            tc_fence_after();
            {
                const float e_r = ex2(s.cvs[hd][r]);
                uint32_t tv[32];
                tmem_ld32(tT + lane_base + 32 * cs, tv);
                tmem_wait_ld(tv);
#pragma unroll
                for (int i = 0; i < 32; ++i) tv[i] = __float_as_uint(e_r * __uint_as_float(tv[i]));
                tmem_st32(tT + lane_base + 32 * cs, tv);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.pm_ready);   // Pm written and T scaled

            // ---- w o X of head hd into the C half of this chunk's B/C slot (free: G and Ys have read
            //      C), for S = B^T (w o X), which runs after Y = Pm X: 4 chunks of 16 B per thread
            if (!ewait(&s.full_x[c & 1], (c >> 1) & 1, abort, lim)) { fail(); break; }
            {
                const int ti = 32 * (warp & 7) + lane;
                const int j = ti >> 1, ch = 4 * (ti & 1);
                const float w = s.dvs[hd][j] * ex2(s.cvs[hd][kQ - 1] - s.cvs[hd][j]);
                const uint8_t *src = xs + hd * kBox;
                uint8_t *dst = s.bc[c & 1] + hd * kBox;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint4 v = lds128(src + swz(j, ch + u));
                    v.x = scale_bf16x2_int(v.x, w); v.y = scale_bf16x2_int(v.y, w);
                    v.z = scale_bf16x2_int(v.z, w); v.w = scale_bf16x2_int(v.w, w);
                    sts128(dst + swz(j, ch + u), v);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.xw_ready);

            // every warp has read this chunk's scan values once all have written w o X:
            // publish the next chunk's
            if (scan_warp && c + 1 < nc) {
                if (!ewait(&s.xw_ready, c & 1, abort, lim)) { fail(); break; }
                scan();
                if (c + 2 < nc) load_dt(c + 2);
            }

            // ---- the masked decay of chunk c+1 while S of this chunk runs: Y has read Pm, G of
            //      chunk c+1 is in TMEM, its scan values are published
            if (c + 1 < nc) {
                if (!(ewait(&s.ymma_done, c & 1, abort, lim) && ewait(&s.g_done, (c + 1) & 1, abort, lim) &&
                      ewait(&s.scan_ready, (c + 1) & 1, abort, lim))) { fail(); break; }
                tc_fence_after();
                decay();
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.pmw);
            }

            // ---- once every product of the chunk is done: y of chunk c and the state step of chunk c+1
            if (!ewait(&s.mma_done[c & 1], (c >> 1) & 1, abort, lim)) { fail(); break; }
            tc_fence_after();
            if (c + 1 < nc) {
                uint32_t hv[32], t0v[16], t1v[16];
                tmem_ld32(tH + lane_base + 32 * cs, hv);
                tmem_ld16(tT + lane_base + 32 * cs, t0v);
                tmem_ld16(tT + lane_base + 32 * cs + 16, t1v);
                tmem_wait_ld(t0v, t1v);
                tmem_wait_ld(hv);
                // the state step first: with T read and hp written, Ys of chunk c+1 may start
                // while y is formed from the registers
                state_step(c + 1, hv);
                tmem_wait_st();
                fence_proxy_async_smem();   // hp, read by Ys of chunk c+1
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.ys_go);
                y_half(xs, t0v, 0);
                y_half(xs, t1v, 1);
            } else {
                uint32_t t0v[16], t1v[16];
                tmem_ld16(tT + lane_base + 32 * cs, t0v);
                tmem_ld16(tT + lane_base + 32 * cs + 16, t1v);
                tmem_wait_ld(t0v, t1v);
                y_half(xs, t0v, 0);
                y_half(xs, t1v, 1);
            }
            tmem_wait_st();
            fence_proxy_async_smem();   // y, read by the TMA store
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.y_ready[c & 1]);
        }
        if (!__any_sync(0xffffffffu, *abort != 0)) {
            // the state after the stripe's last chunk
            uint32_t hv[32];
            tmem_ld32(tH + lane_base + 32 * cs, hv);
            tmem_wait_ld(hv);
            const int64_t kc = ckpt_slot(s0 + (int64_t)nc * kQ);
            if (kc >= 0) store_state(ckpt_ptr(kc), hv);
            if (p.h_final && s1 == p.L) store_state(p.h_final + ((int64_t)bi * p.H + hh) * PN + (int64_t)p0 * kN + r, hv);
        }
    } else {
        // shared-memory descriptors of every operand tile, built once per slot: a K-step only adds
        // a constant to the start-address field (in 16-byte units; addresses stay below 256 KB)
        const uint32_t bc0 = smem_u32(s.bc[0]), bc1 = smem_u32(s.bc[1]);
        const uint32_t x0 = smem_u32(s.x[0]), x1 = smem_u32(s.x[1]);
        const uint64_t dC0 = smem_desc(bc0, 16, 1024), dC1 = smem_desc(bc1, 16, 1024);   // C, K-major
        const uint64_t dBk0 = smem_desc(bc0 + 2 * kBox, 16, 1024), dBk1 = smem_desc(bc1 + 2 * kBox, 16, 1024);  // B, K-major
        const uint64_t dBt0 = smem_desc(bc0 + 2 * kBox, kBox, 1024), dBt1 = smem_desc(bc1 + 2 * kBox, kBox, 1024);  // B^T, MN-major
        const uint64_t dX0 = smem_desc(x0, 0, 1024), dX1 = smem_desc(x1, 0, 1024);           // X of one head, MN-major, N = 64
        const uint64_t dXw0 = smem_desc(bc0, kBox, 1024), dXw1 = smem_desc(bc1, kBox, 1024);  // w o X (C half of the B/C slot), N = 128
        const uint64_t dHp = smem_desc(smem_u32(s.hp), kBox, 1024);                          // hp of both heads, N = 128
        constexpr uint64_t kBoxD = kBox >> 4;
        auto koff = [](int kk) -> uint64_t { return (uint64_t)((kk >> 2) * kBoxD + (kk & 3) * 2); };  // K-major K-step
        auto moff = [](int kk) -> uint64_t { return (uint64_t)(kk * 128); };                          // MN-major K-step
        // G = C B^T of chunk c into the TMEM columns at tG (its B/C slot has landed)
        auto issue_g = [&](int c) {
            const uint64_t dc = (c & 1) ? dC1 : dC0, db = (c & 1) ? dBk1 : dBk0;
            const uint32_t id_g = idesc_bf16(128, 128, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) mma_ss(tG, dc + koff(kk), db + koff(kk), id_g, kk > 0);
            mma_commit(&s.g_done);
        };
        // The whole warp waits (warp-uniform outcome); lane 0 issues.
        if (warp == kComputeWarps) {
            // ============================================= issuing warp: Y, S, Ys (and G of chunk 0)
            // Ys = C hp^T of chunk c into T (its B/C slot has landed, hp is written, T is free)
            auto issue_ys = [&](int c) {
                const uint64_t dc = (c & 1) ? dC1 : dC0;
                const uint32_t id_ys = idesc_bf16(128, 128, 0, 1);    // A = C (K-major), B = hp (MN-major)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) mma_ss(tT, dc + koff(kk), dHp + moff(kk), id_ys, kk > 0);
                mma_commit(&s.ys_done);
            };
            const uint32_t id_pm = idesc_bf16(128, 64, 0, 1);     // A = Pm (TMEM), B = X (MN-major)
            const uint32_t id_s = idesc_bf16(128, 128, 1, 1);     // A = B^T (MN-major), B = w o X (MN-major)
            bool ok = live;
            if (ok) {
                // G of chunk 0 once its B/C slot has landed, Ys of chunk 0 once the warps have
                // written hp of the state entering the stripe
                ok = ewait(&s.full_bc[0], 0, abort, lim);
                if (ok) {
                    tc_fence_after();
                    if (lane == 0) issue_g(0);
                    __syncwarp();
                    ok = ewait(&s.st0_ready, 0, abort, lim);
                    if (ok) {
                        tc_fence_after();
                        if (lane == 0) issue_ys(0);
                        __syncwarp();
                    }
                }
            }
            for (int c = 0; ok && c < nc; ++c) {
                // Pm written and T (= Ys) scaled, X landed: Y_a, Y_b accumulate into T while the
                // warps write w o X
                ok = ewait(&s.pm_ready, c & 1, abort, lim) && ewait(&s.full_x[c & 1], (c >> 1) & 1, abort, lim);
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint64_t dx = (c & 1) ? dX1 : dX0;
#pragma unroll
                    for (int hd2 = 0; hd2 < 2; ++hd2)
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ts(tT + 64 * hd2, tPm + 64 * hd2 + kk * 8, dx + hd2 * kBoxD + moff(kk), id_pm, true);
                    mma_commit(&s.ymma_done);
                }
                __syncwarp();
                // w o X of both heads written (into the C half of this chunk's B/C slot):
                // S = B^T [Xw_a | Xw_b] accumulates into H
                ok = ewait(&s.xw_ready, c & 1, abort, lim);
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint64_t dbt = (c & 1) ? dBt1 : dBt0, dxw = (c & 1) ? dXw1 : dXw0;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) mma_ss(tH, dbt + moff(kk), dxw + moff(kk), id_s, true);
                    mma_commit(&s.mma_done[c & 1]);
                }
                __syncwarp();
                // T read and hp of chunk c+1 written: Ys of chunk c+1 into T
                if (c + 1 < nc) {
                    ok = ewait(&s.ys_go, c & 1, abort, lim);
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) issue_ys(c + 1);
                    __syncwarp();
                }
            }
            if (lane == 0) {
                if (live && !ok) raise_timeout(p, abort);
                // every MMA of this warp complete before TMEM is freed
                mma_commit(&s.fin);
                mbar_wait(&s.fin, 0, nullptr, 100000000ull);
            }
            __syncwarp();
        } else if (warp == kComputeWarps + 1) {
            // ============================================= store warp: y out, X in
            // (kept off the issuing warp, whose lane would otherwise sit in the wait for the
            // store to read its slot while the next products could be issued)
            int x_issued = 0;   // lane 0's bookkeeping
            auto issue_x = [&](int c) {
                const int t0 = (int)(s0 + (int64_t)c * kQ);
                uint8_t *d = s.x[c & 1];
                uint64_t *bar = &s.full_x[c & 1];
                mbar_arrive_expect_tx(bar, 2 * kBox);
                tma_load_3d(d, &maps.x, bar, ha * kP, t0, bi);
                tma_load_3d(d + kBox, &maps.x, bar, (ha + 1) * kP, t0, bi);
                ++x_issued;
            };
            bool ok = live;
            if (ok && lane == 0) {
                issue_x(0);
                if (nc > 1) issue_x(1);
            }
            for (int c = 0; ok && c < nc; ++c) {
                const int64_t t0 = s0 + (int64_t)c * kQ;
                uint8_t *xs = s.x[c & 1];
                // y staged: store it; once the store has read the slot, X of chunk c+2 is loaded there
                ok = ewait(&s.y_ready[c & 1], (c >> 1) & 1, abort, lim);
                if (!ok) break;
                if (lane == 0) {
                    tma_store_3d(&maps.y, xs, ha * kP, (int)t0, bi);
                    tma_store_3d(&maps.y, xs + kBox, (ha + 1) * kP, (int)t0, bi);
                    tma_store_commit();
                    if (c + 2 < nc) {
                        tma_store_wait_read<0>();
                        issue_x(c + 2);
                    }
                }
                __syncwarp();
            }
            if (lane == 0) {
                if (live && !ok) raise_timeout(p, abort);
                if (*abort) {
                    // the last load issued into each X slot lands before the CTA's shared memory is
                    // released (an earlier load into the same slot has been waited on by the compute warps)
                    for (int i = x_issued > 2 ? x_issued - 2 : 0; i < x_issued; ++i)
                        mbar_wait(&s.full_x[i & 1], (i >> 1) & 1, nullptr, 100000000ull);
                }
                tma_store_wait<0>();
            }
            __syncwarp();
        } else {
            // ============================================= B/C warp: B and C in, G of chunks 1..
            // (G of chunk c+2 waits for its slot to land, which must not hold up Y and S)
            int bc_issued = 0;   // lane 0's bookkeeping
            auto issue_bc = [&](int c) {
                const int t0 = (int)(s0 + (int64_t)c * kQ);
                uint8_t *d = s.bc[c & 1];
                uint64_t *bar = &s.full_bc[c & 1];
                mbar_arrive_expect_tx(bar, 4 * kBox);
                tma_load_3d(d, &maps.C, bar, g * kN, t0, bi);
                tma_load_3d(d + kBox, &maps.C, bar, g * kN + 64, t0, bi);
                tma_load_3d(d + 2 * kBox, &maps.B, bar, g * kN, t0, bi);
                tma_load_3d(d + 3 * kBox, &maps.B, bar, g * kN + 64, t0, bi);
                ++bc_issued;
            };
            bool ok = live;
            if (ok) {
                if (lane == 0) {
                    issue_bc(0);
                    if (nc > 1) issue_bc(1);
                }
                // G of chunk 1 once the warps have read G of chunk 0
                if (nc > 1) {
                    ok = ewait(&s.pmw, 0, abort, lim) && ewait(&s.full_bc[1], 0, abort, lim);
                    if (ok) {
                        tc_fence_after();
                        if (lane == 0) issue_g(1);
                        __syncwarp();
                    }
                }
            }
            for (int c = 0; ok && c + 2 < nc; ++c) {
                // S of chunk c done: its B/C slot (C, B, w o X) is spent -- refill it with chunk c+2
                ok = ewait(&s.mma_done[c & 1], (c >> 1) & 1, abort, lim);
                if (!ok) break;
                if (lane == 0) issue_bc(c + 2);
                __syncwarp();
                // G of chunk c+2 into R0 once the warps have read G of chunk c+1, the slot has landed
                // and Ys of chunk c+1 is done (G must not sit in front of Ys in the tensor pipe: Ys
                // is on the chunk's critical path, G of chunk c+2 is not needed for a while)
                ok = ewait(&s.pmw, (c + 1) & 1, abort, lim) &&
                     ewait(&s.full_bc[c & 1], ((c + 2) >> 1) & 1, abort, lim) &&
                     ewait(&s.ys_done, (c + 1) & 1, abort, lim);
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) issue_g(c + 2);
                __syncwarp();
            }
            if (lane == 0) {
                if (live && !ok) raise_timeout(p, abort);
                // every MMA of this warp complete before TMEM is freed
                mma_commit(&s.fin2);
                mbar_wait(&s.fin2, 0, nullptr, 100000000ull);
                if (*abort) {
                    // the last load issued into each B/C slot lands before the CTA's shared memory
                    // is released (an earlier load into the same slot has been waited on for its G)
                    for (int i = bc_issued > 2 ? bc_issued - 2 : 0; i < bc_issued; ++i)
                        mbar_wait(&s.full_bc[i & 1], (i >> 1) & 1, nullptr, 100000000ull);
                }
            }
            __syncwarp();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 512);
}

// =============================================================== host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    // looked up once per process (a function-local static is initialised thread-safely)
    static const EncodeTiledFn fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(f);
        return (EncodeTiledFn) nullptr;
    }();
    return fn;
}

// [b][L][cols] view with element strides (rs, bs); box = 64 columns x 128 rows
bool encode_bf16(EncodeTiledFn enc, CUtensorMap *m, const void *base, int64_t cols, int64_t L, int b,
                 int64_t rs, int64_t bs, uint32_t box_rows = 128)
{
    if (b == 1) bs = rs * L;
    const cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)L, (cuuint64_t)b};
    const cuuint64_t strides[2] = {(cuuint64_t)rs * 2, (cuuint64_t)bs * 2};
    const cuuint32_t box[3] = {64, box_rows, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


constexpr size_t kSmemA = sizeof(SmemA) + 1024;
constexpr size_t kSmemC = sizeof(SmemC);   // no alignment pad: the base is checked in the kernel
static_assert(kSmemC <= 232448, "pass C shared memory");
static_assert(kSmemA <= 232448, "pass A shared memory");

}  // namespace

bool tc_scan_shape(int dtype, int H, int P, int N, int G, int Q)
{
    return dtype == 1 && P == kP && N == kN && Q == kQ && H % 2 == 0 && G > 0 && (H / G) % 2 == 0;
}

bool tc_scan_supported(const ScanParams &p, int dtype)
{
    if (!tc_scan_shape(dtype, p.H, p.P, p.N, p.G, p.Q)) return false;   // head pairs share a B/C group
    if ((reinterpret_cast<uintptr_t>(p.dt) & 7u) != 0) return false;  // dt of a head pair read as float2
    if (p.L >= (1LL << 31) || (int64_t)p.b * p.ns * p.H >= (1LL << 31)) return false;
    return encode_fn() != nullptr;
}

int launch_scan_tc(const ScanParams &p, cudaStream_t st)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return 6;
    Maps maps;
    const int64_t gn = (int64_t)p.G * p.N;
    const bool fused = p.conv_w != nullptr;
    if (fused && (p.ns <= 1 || !encode_bf16(enc, &maps.ux, p.conv_u, (int64_t)p.H * p.P, p.L, p.b, p.conv_urs,
                                            p.conv_ubs, kQ + kHaloRows)))
        return 6;   // the fused conv lives in pass A, which a single stripe does not run
    if (!encode_bf16(enc, &maps.x, p.x, (int64_t)p.H * p.P, p.L, p.b, p.xrs, p.xbs) ||
        !encode_bf16(enc, &maps.B, p.B, gn, p.L, p.b, p.Brs, p.Bbs) ||
        !encode_bf16(enc, &maps.C, p.C, gn, p.L, p.b, p.Crs, p.Cbs) ||
        !encode_bf16(enc, &maps.y, p.y, (int64_t)p.H * p.P, p.L, p.b, p.yrs, p.ybs))
        return 6;
    static std::atomic<bool> attr_set[64];   // set once per device (a repeat is harmless)
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(stripe_state_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemA) != cudaSuccess ||
            cudaFuncSetAttribute(stripe_state_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemA) != cudaSuccess ||
            cudaFuncSetAttribute(chunk_output_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemC) != cudaSuccess)
            return 7;
        attr_set[dev] = true;
    }
    const int64_t units = (int64_t)p.b * p.ns * p.H;
    if (p.ns > 1) {
        prof_begin(st, kKStateTc);
        if (fused) stripe_state_tc_kernel<true><<<(unsigned)(units / 2), kThreadsA, kSmemA, st>>>(maps, p);
        else stripe_state_tc_kernel<false><<<(unsigned)(units / 2), kThreadsA, kSmemA, st>>>(maps, p);
        prof_end(st, kKStateTc);
        const int rc = launch_chain(p, st);
        if (rc) return rc;
    }
    prof_begin(st, kKOutputTc);
    chunk_output_tc_kernel<<<(unsigned)(units / 2), kThreadsC, kSmemC, st>>>(maps, p);
    prof_end(st, kKOutputTc);
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

}  // namespace ssd

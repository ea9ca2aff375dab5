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
//   Yo = C h_prev^T                                tcgen05, 128x64x128
//   y  = Yd + exp(cs_i) Yo + D x                   CUDA cores -> global (bf16)
//   S  = B^T (w o X),  w_j = dt_j exp(cs_last - cs_j)   tcgen05, 128x64x128
//   h  = exp(cs_last) h + S                        CUDA cores, fp32 state in registers
// Only non-positive differences of cs are exponentiated.  The state is kept in
// fp32; its bf16 copy only feeds the C h_prev^T product.
//
// Warp roles (192 threads): warp 0 issues TMA loads into a 2-stage ring,
// warp 1 issues the MMAs (one thread), warps 2..5 (128 threads, one per
// token row / TMEM lane) do the masked decay, the outputs and the state.
// All waits are bounded (tc::mbar_wait): on a timeout the CTA raises an abort
// flag, every role unwinds, outstanding MMAs are drained, TMEM is freed and
// the device status word reports SSD_ERR_TIMEOUT.
#include <cuda.h>

#include "ssd_common.cuh"
#include "tc_ptx.cuh"

namespace ssd {

int launch_chain(const ScanParams &p, cudaStream_t st);

namespace {

using namespace tc;

constexpr int kQ = 128, kP = 64, kN = 128;
constexpr uint32_t kBox = 128 * 64 * 2;   // one 128-row x 64-col bf16 TMA box (16 KB)
constexpr uint32_t kDtBox = 128 * 4 * 4;  // dt box: [128 tokens][4 heads] fp32 (2 KB)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kThreads = 192;

struct Maps {
    CUtensorMap x, B, C, dt;
};

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

// Barrier among the 128 epilogue threads, built on an mbarrier so that the
// wait is bounded like every other wait (a bar.sync could not be abandoned).
// `ph` counts the completed phases of `bar` seen by this thread.
__device__ __forceinline__ bool epi_sync(uint64_t *bar, uint32_t &ph, volatile int *abort, uint64_t limit_ns)
{
    mbar_arrive(bar);
    const bool ok = ewait(bar, ph & 1, abort, limit_ns);
    ++ph;
    return ok;
}

// byte offset of 16-byte chunk c of row r in a 128B-swizzled tile of 128-byte rows
__device__ __forceinline__ uint32_t swz(int r, int c)
{
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint4 lds128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ void sts128(uint8_t *p, uint4 v) { *reinterpret_cast<uint4 *>(p) = v; }

__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t v, float w)
{
    return pack_bf16x2(bf16_lo(v) * w, bf16_hi(v) * w);
}

// Inclusive scan of one value per epilogue thread (row r) over the 128 rows.
// scratch holds two buffers of 4 floats, used alternately by consecutive
// calls (a thread can be at most one call ahead of the slowest one).
__device__ __forceinline__ bool epi_scan(float &v, int r, float *scratch, float &total, uint64_t *bar,
                                         uint32_t &ph, volatile int *abort, uint64_t limit_ns)
{
    const int lane = r & 31, q = r >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) scratch[q] = v;
    if (!epi_sync(bar, ph, abort, limit_ns)) return false;
    const float s0 = scratch[0], s1 = scratch[1], s2 = scratch[2], s3 = scratch[3];
    float pre = 0.0f;
    if (q > 0) pre += s0;
    if (q > 1) pre += s1;
    if (q > 2) pre += s2;
    total = ((s0 + s1) + s2) + s3;
    v = q == 3 ? v + ((s0 + s1) + s2) : v + pre;
    return true;
}

__device__ __forceinline__ void raise_timeout(const ScanParams &p, volatile int *abort)
{
    *abort = 1;
    atomicOr(p.status, kDevTimeout);
}

// =============================================================== pass A
// Two heads per CTA: S^T[(h,p)][n] = sum_j (w_h o X_h)[j][p] B[j][n] for the
// head pair, accumulated in TMEM over the whole stripe (M = 128 rows = 2 heads
// x 64, N = 128 as two N=64 halves).  Chunks are walked backwards so that the
// decay from each chunk to the stripe end (a suffix sum) is known when the
// chunk is scaled.
struct SmemA {
    uint8_t stage[2][4 * kBox + kDtBox];  // B (two boxes), X of head h0, X of head h1, dt
    uint8_t xw[2][2 * kBox];              // w o X for both heads (h0 box, h1 box)
    float scratch[2][8];
    uint64_t full[2], empty[2], xw_full[2], xw_empty[2], acc_full, fin, epi;
    uint32_t tmem;
    int abort;
};

__global__ void __launch_bounds__(kThreads, 1)
stripe_state_tc_kernel(const __grid_constant__ Maps maps, const ScanParams p)
{
    extern __shared__ uint8_t smraw[];
    SmemA &s = *reinterpret_cast<SmemA *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t unit = blockIdx.x;
    const int hpairs = p.H / 2;
    const int h0 = 2 * (int)(unit % hpairs);
    const int64_t k = (unit / hpairs) % p.ns;
    const int bi = (int)(unit / ((int64_t)hpairs * p.ns));
    const int g = (int)((int64_t)h0 * p.G / p.H);  // both heads of the pair share a group (H/G even)
    const int64_t s0 = k * p.T;
    const int64_t s1 = min(p.L, s0 + p.T);
    const int nc = (int)((s1 - s0 + kQ - 1) / kQ);
    const uint64_t lim = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1 + 128);
            mbar_init(&s.xw_full[i], 128);
            mbar_init(&s.xw_empty[i], 1);
        }
        mbar_init(&s.acc_full, 1);
        mbar_init(&s.fin, 1);
        mbar_init(&s.epi, 128);
        s.abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&maps.x);
        prefetch_tmap(&maps.B);
        prefetch_tmap(&maps.dt);
    }
    if (warp == 1) { tmem_alloc(&s.tmem, 128); tmem_relinquish(); }
    __syncthreads();
    tc_fence_after();
    const uint32_t tS = s.tmem;
    volatile int *abort = &s.abort;

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            for (int it = 0; it < nc; ++it) {
                const int st = it & 1, u = it >> 1;
                if (it >= 2 && !mbar_wait(&s.empty[st], (u - 1) & 1, abort, lim)) { raise_timeout(p, abort); break; }
                if (unit == p.test_drop_unit) break;  // test hook: this unit's loads never arrive
                const int c = nc - 1 - it;  // chunks in reverse order
                const int t0 = (int)(s0 + (int64_t)c * kQ);
                uint8_t *sb = s.stage[st];
                mbar_arrive_expect_tx(&s.full[st], 4 * kBox + kDtBox);
                tma_load_3d(sb, &maps.B, &s.full[st], g * kN, t0, bi);
                tma_load_3d(sb + kBox, &maps.B, &s.full[st], g * kN + 64, t0, bi);
                tma_load_3d(sb + 2 * kBox, &maps.x, &s.full[st], h0 * kP, t0, bi);
                tma_load_3d(sb + 3 * kBox, &maps.x, &s.full[st], (h0 + 1) * kP, t0, bi);
                tma_load_3d(sb + 4 * kBox, &maps.dt, &s.full[st], h0 & ~3, t0, bi);
                issued = it + 1;
            }
            if (*abort) {  // let copies in flight land before the CTA exits
                for (int it = max(0, issued - 2); it < issued; ++it)
                    mbar_wait(&s.full[it & 1], (it >> 1) & 1, nullptr, 100000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id = idesc_bf16(128, 64, 1, 1);
            for (int it = 0; it < nc; ++it) {
                const int st = it & 1, u = it >> 1, xb = it & 1;
                if (!mbar_wait(&s.full[st], u & 1, abort, lim) || !mbar_wait(&s.xw_full[xb], (it >> 1) & 1, abort, lim)) {
                    raise_timeout(p, abort);
                    break;
                }
                tc_fence_after();
                const uint32_t sB = smem_u32(s.stage[st]);
                const uint32_t sXw = smem_u32(s.xw[xb]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t da = smem_desc(sXw + kk * 2048, kBox, 1024);  // rows (h,p): two atoms
                    mma_ss(tS, da, smem_desc(sB + kk * 2048, 0, 1024), id, it > 0 || kk > 0);
                    mma_ss(tS + 64, da, smem_desc(sB + kBox + kk * 2048, 0, 1024), id, it > 0 || kk > 0);
                }
                mma_commit(&s.empty[st]);
                mma_commit(&s.xw_empty[xb]);
            }
            mma_commit(&s.acc_full);
            mma_commit(&s.fin);
            mbar_wait(&s.fin, 0, nullptr, 200000000ull);
        }
    } else {
        const int q = warp & 3;
        const int r = 32 * q + lane;  // token row j; TMEM lane (h,p) for the result
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const float A2a = p.A[h0] * kLog2e, A2b = p.A[h0 + 1] * kLog2e;
        float sufa = 0.0f, sufb = 0.0f;
        bool okk = true;
        uint32_t eph = 0;
        for (int it = 0; it < nc; ++it) {
            const int st = it & 1, u = it >> 1, xb = it & 1;
            if (!ewait(&s.full[st], u & 1, abort, lim)) { raise_timeout(p, abort); okk = false; break; }
            const uint8_t *sb = s.stage[st];
            const float *dtrow = reinterpret_cast<const float *>(sb + 4 * kBox) + r * 4 + (h0 & 3);
            const float dta = dtrow[0], dtb = dtrow[1];
            float va = dta * A2a, vb = dtb * A2b;
            const int lq = r & 31;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float ta = __shfl_up_sync(0xffffffffu, va, o);
                const float tb = __shfl_up_sync(0xffffffffu, vb, o);
                if (lq >= o) { va += ta; vb += tb; }
            }
            float *scr = s.scratch[it & 1];
            if (lq == 31) { scr[q] = va; scr[4 + q] = vb; }
            if (!epi_sync(&s.epi, eph, abort, lim)) { raise_timeout(p, abort); okk = false; break; }
            float prea = 0.0f, preb = 0.0f;
            if (q > 0) { prea += scr[0]; preb += scr[4]; }
            if (q > 1) { prea += scr[1]; preb += scr[5]; }
            if (q > 2) { prea += scr[2]; preb += scr[6]; }
            const float tota = ((scr[0] + scr[1]) + scr[2]) + scr[3];
            const float totb = ((scr[4] + scr[5]) + scr[6]) + scr[7];
            const float wa = dta * ex2((tota - (va + prea)) + sufa);
            const float wb = dtb * ex2((totb - (vb + preb)) + sufb);
            if (it >= 2 && !ewait(&s.xw_empty[xb], ((it >> 1) - 1) & 1, abort, lim)) {
                raise_timeout(p, abort);
                okk = false;
                break;
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint8_t *xrow = sb + (2 + hh) * kBox;
                uint8_t *xwt = s.xw[xb] + hh * kBox;
                const float w = hh ? wb : wa;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const uint32_t o = swz(r, cc);
                    uint4 vv = lds128(xrow + o);
                    vv.x = scale_bf16x2(vv.x, w); vv.y = scale_bf16x2(vv.y, w);
                    vv.z = scale_bf16x2(vv.z, w); vv.w = scale_bf16x2(vv.w, w);
                    sts128(xwt + o, vv);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&s.xw_full[xb]);
            mbar_arrive(&s.empty[st]);
            sufa += tota;
            sufb += totb;
        }
        if (okk && ewait(&s.acc_full, 0, abort, lim)) {
            tc_fence_after();
            const int hh = r >> 6, pp = r & 63;  // lane r holds state row p of head h0 + hh
            float *dst = p.ws_S + (((int64_t)bi * p.ns + k) * p.H + h0 + hh) * (kP * kN) + (int64_t)pp * kN;
#pragma unroll
            for (int c32 = 0; c32 < 4; ++c32) {
                uint32_t a[32];
                tmem_ld32(tS + lane_base + 32 * c32, a);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    reinterpret_cast<uint4 *>(dst + 32 * c32)[i] = make_uint4(a[4 * i], a[4 * i + 1], a[4 * i + 2], a[4 * i + 3]);
            }
            if (r == 0) {
                p.ws_dA[((int64_t)bi * p.ns + k) * p.H + h0] = sufa * kLn2;
                p.ws_dA[((int64_t)bi * p.ns + k) * p.H + h0 + 1] = sufb * kLn2;
            }
        } else if (okk) {
            raise_timeout(p, abort);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tS, 128);
}

// =============================================================== pass C
// One CTA per (stripe, head), two CTAs per SM: each CTA walks its chunks in a
// plain sequence and the two co-resident CTAs hide each other's latencies.
// Per chunk (all 256 threads; thread = TMEM lane quarter q, column half hs):
//   G  = C B^T                         one elected thread issues the MMAs
//   cumsum of dt*A (each warp on its own), Pm from G, D x into Y
//   EC = exp(cs_i) C_i (bf16, TMEM) ; w o X written over the spent C tile
//   Y += Pm X ; Y += EC h_prev^T ; S = B^T (w o X)      (one commit)
//   -> every input slot is free: the next chunk's TMA is issued here
//   y = Y -> global ; h = exp(cs_last) h + S ; h_prev (bf16) -> smem ; checkpoints
// TMEM (256 columns): G 0..127, then EC 0..63 and S 64..127 | Pm 128..191 | Y 192..255.
constexpr int kThreadsC = 256;

struct SmemC {
    uint8_t cb[4 * kBox];      // C (two boxes: K 0..63, 64..127), B (two boxes); C is reused for w o X
    uint8_t x[kBox];           // X, rows j (tokens), 128B-swizzled
    uint8_t hp[kBox];          // bf16 h_prev, rows n, 128B-swizzled
    float dt[kQ * 4];          // dt box: [128 tokens][4 heads]
    uint64_t full, g_done, mma_done, fin;
    uint32_t tmem;
    int abort;
};

__device__ __forceinline__ float sel4(const float (&v)[4], int i)
{
    return i == 0 ? v[0] : (i == 1 ? v[1] : (i == 2 ? v[2] : v[3]));
}

__global__ void __launch_bounds__(kThreadsC, 2)
chunk_output_tc_kernel(const __grid_constant__ Maps maps, const ScanParams p)
{
    extern __shared__ uint8_t smraw[];
    SmemC &s = *reinterpret_cast<SmemC *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, hs = warp >> 2;
    const int r = 32 * q + lane;                 // token row / TMEM lane / state column n
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const int64_t unit = blockIdx.x;
    const int h = (int)(unit % p.H);
    const int64_t k = (unit / p.H) % p.ns;
    const int bi = (int)(unit / ((int64_t)p.H * p.ns));
    const int g = (int)((int64_t)h * p.G / p.H);
    const int64_t s0 = k * p.T;
    const int64_t s1 = min(p.L, s0 + p.T);
    const int nc = (int)((s1 - s0 + kQ - 1) / kQ);
    const uint64_t lim = p.wait_limit_ns;
    const int PN = kP * kN;

    if (tid == 0) {
        mbar_init(&s.full, 1);
        mbar_init(&s.g_done, 1);
        mbar_init(&s.mma_done, 1);
        mbar_init(&s.fin, 1);
        s.abort = 0;
        fence_mbar_init();
        prefetch_tmap(&maps.x);
        prefetch_tmap(&maps.B);
        prefetch_tmap(&maps.C);
        prefetch_tmap(&maps.dt);
    }
    if (warp == 0) { tmem_alloc(&s.tmem, 256); tmem_relinquish(); }
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = s.tmem;
    const uint32_t tG = tm, tEC = tm, tS = tm + 64, tPm = tm + 128, tY = tm + 192;
    volatile int *abort = &s.abort;

    auto issue_loads = [&](int c) {
        const int t0 = (int)(s0 + (int64_t)c * kQ);
        mbar_arrive_expect_tx(&s.full, 5 * kBox + kDtBox);
        tma_load_3d(s.cb, &maps.C, &s.full, g * kN, t0, bi);
        tma_load_3d(s.cb + kBox, &maps.C, &s.full, g * kN + 64, t0, bi);
        tma_load_3d(s.cb + 2 * kBox, &maps.B, &s.full, g * kN, t0, bi);
        tma_load_3d(s.cb + 3 * kBox, &maps.B, &s.full, g * kN + 64, t0, bi);
        tma_load_3d(s.x, &maps.x, &s.full, h * kP, t0, bi);
        tma_load_3d(s.dt, &maps.dt, &s.full, h & ~3, t0, bi);
    };
    int pending = -1;   // (thread 0) chunk whose loads are issued but not yet waited for
    if (tid == 0 && nc > 0 && unit != p.test_drop_unit) { issue_loads(0); pending = 0; }

    // state entering the stripe: thread (r = n, hs) owns h[32 hs .. 32 hs + 31][n]
    float hr[32];
    {
        const float *hin = (k == 0) ? (p.h0 ? p.h0 + ((int64_t)bi * p.H + h) * PN : nullptr)
                                    : p.ws_hin + (((int64_t)bi * p.ns + k) * p.H + h) * PN;
#pragma unroll
        for (int pp = 0; pp < 32; ++pp) hr[pp] = hin ? hin[(32 * hs + pp) * kN + r] : 0.0f;
    }
    auto write_hp = [&]() {
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            uint4 v;
            v.x = pack_bf16x2(hr[8 * c4 + 0], hr[8 * c4 + 1]);
            v.y = pack_bf16x2(hr[8 * c4 + 2], hr[8 * c4 + 3]);
            v.z = pack_bf16x2(hr[8 * c4 + 4], hr[8 * c4 + 5]);
            v.w = pack_bf16x2(hr[8 * c4 + 6], hr[8 * c4 + 7]);
            sts128(s.hp + swz(r, 4 * hs + c4), v);
        }
    };
    write_hp();
    fence_proxy_async_smem();

    const float A2 = p.A[h] * kLog2e;
    const float Dh = p.D ? p.D[h] : 0.0f;
    const int64_t n_ckpt = p.s > 0 ? p.L / p.s : 0;
    __nv_bfloat16 *ybase = reinterpret_cast<__nv_bfloat16 *>(p.y) + (int64_t)bi * p.ybs + (int64_t)h * kP + 32 * hs;
    const uint32_t id_g = idesc_bf16(128, 128, 0, 0);
    const uint32_t id_kmn = idesc_bf16(128, 64, 0, 1);
    const uint32_t id_mnmn = idesc_bf16(128, 64, 1, 1);

    for (int c = 0; c < nc; ++c) {
        const int64_t t0 = s0 + (int64_t)c * kQ;
        // ---- operands of this chunk
        bool ok = mbar_wait(&s.full, c & 1, abort, lim);
        if (!__syncthreads_and(ok)) { raise_timeout(p, abort); break; }
        pending = -1;
        tc_fence_after();
        if (tid == 0) {
            const uint32_t sC = smem_u32(s.cb), sB = sC + 2 * kBox;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                mma_ss(tG, smem_desc(sC + off, 16, 1024), smem_desc(sB + off, 16, 1024), id_g, kk > 0);
            }
            mma_commit(&s.g_done);
        }
        // ---- chunk cumsum (each warp on its own: lane l holds rows l + 32 J)
        float dv[4], cv[4], fv[4], r2[4];
#pragma unroll
        for (int J = 0; J < 4; ++J) dv[J] = s.dt[(lane + 32 * J) * 4 + (h & 3)];
#pragma unroll
        for (int J = 0; J < 4; ++J) {
            float v = dv[J] * A2;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float t = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += t;
            }
            cv[J] = v;
        }
        {
            float run = 0.0f;
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                const float bt = __shfl_sync(0xffffffffu, cv[J], 31);
                cv[J] += run;
                run += bt;
                r2[J] = run;
            }
        }
        const float tot2 = r2[3];
#pragma unroll
        for (int J = 0; J < 4; ++J) fv[J] = dv[J] * ex2(r2[J] - cv[J]);
        const float cs2 = sel4(cv, q);
        const float dt_r = sel4(dv, q);
        // ---- D x into Y (this half's 32 columns of p)
        {
            uint32_t dx[32];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const uint4 xv = lds128(s.x + swz(r, 4 * hs + c4));
                const uint32_t w4[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    dx[8 * c4 + 2 * i] = __float_as_uint(Dh * bf16_lo(w4[i]));
                    dx[8 * c4 + 2 * i + 1] = __float_as_uint(Dh * bf16_hi(w4[i]));
                }
            }
            uint32_t d0[16], d1[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) { d0[i] = dx[i]; d1[i] = dx[16 + i]; }
            tmem_st16(tY + lane_base + 32 * hs, d0);
            tmem_st16(tY + lane_base + 32 * hs + 16, d1);
        }
        // ---- masked decay Pm[r][j] = G[r][j] exp(cs_r - cs_j) dt_j (j <= r): blocks {hs, hs + 2}
        ok = mbar_wait(&s.g_done, c & 1, abort, lim);
        if (!__all_sync(0xffffffffu, ok)) { *abort = 1; }
        tc_fence_after();
        if (!*abort) {
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int J = 2 * jj + hs;
                uint32_t pk[16];
                if (J < q) {
                    const float E = ex2(cs2 - sel4(r2, J));
                    uint32_t gv[32];
                    tmem_ld32(tG + lane_base + 32 * J, gv);
                    tmem_wait_ld();
                    const float fJ = sel4(fv, J);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float f0 = __shfl_sync(0xffffffffu, fJ, 2 * i);
                        const float f1 = __shfl_sync(0xffffffffu, fJ, 2 * i + 1);
                        pk[i] = pack_bf16x2(__uint_as_float(gv[2 * i]) * f0 * E,
                                            __uint_as_float(gv[2 * i + 1]) * f1 * E);
                    }
                } else if (J == q) {
                    uint32_t gv[32];
                    tmem_ld32(tG + lane_base + 32 * J, gv);
                    tmem_wait_ld();
                    const float cJ = sel4(cv, J), dJ = sel4(dv, J);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float c0 = __shfl_sync(0xffffffffu, cJ, 2 * i);
                        const float c1 = __shfl_sync(0xffffffffu, cJ, 2 * i + 1);
                        const float d0 = __shfl_sync(0xffffffffu, dJ, 2 * i);
                        const float d1 = __shfl_sync(0xffffffffu, dJ, 2 * i + 1);
                        float v0 = __uint_as_float(gv[2 * i]) * ex2(cs2 - c0) * d0;
                        float v1 = __uint_as_float(gv[2 * i + 1]) * ex2(cs2 - c1) * d1;
                        if (2 * i > lane) v0 = 0.0f;
                        if (2 * i + 1 > lane) v1 = 0.0f;
                        pk[i] = pack_bf16x2(v0, v1);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = 0u;
                }
                tmem_st16(tPm + lane_base + 16 * J, pk);
            }
        }
        tmem_wait_st();
        tc_fence_before();
        if (__syncthreads_or(*abort)) { raise_timeout(p, abort); break; }   // all reads of G done
        tc_fence_after();
        // ---- EC = exp(cs_r) C_r over G's columns 0..63 (this half: K = 64 hs .. 64 hs + 63)
        {
            const float e = ex2(cs2);
            const uint8_t *cbox = s.cb + hs * kBox;
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                uint32_t ev[16];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const uint4 cvv = lds128(cbox + swz(r, 4 * q2 + c4));
                    ev[4 * c4 + 0] = scale_bf16x2(cvv.x, e);
                    ev[4 * c4 + 1] = scale_bf16x2(cvv.y, e);
                    ev[4 * c4 + 2] = scale_bf16x2(cvv.z, e);
                    ev[4 * c4 + 3] = scale_bf16x2(cvv.w, e);
                }
                tmem_st16(tEC + lane_base + 32 * hs + 16 * q2, ev);
            }
        }
        tmem_wait_st();
        __syncthreads();   // every read of C is done: w o X may overwrite it
        // ---- w o X for the state update, written over C's first box (rows j, same swizzle)
        {
            const float w = dt_r * ex2(tot2 - cs2);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const int cc = 4 * hs + c4;
                uint4 vv = lds128(s.x + swz(r, cc));
                vv.x = scale_bf16x2(vv.x, w); vv.y = scale_bf16x2(vv.y, w);
                vv.z = scale_bf16x2(vv.z, w); vv.w = scale_bf16x2(vv.w, w);
                sts128(s.cb + swz(r, cc), vv);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            const uint32_t sX = smem_u32(s.x), sHp = smem_u32(s.hp), sXw = smem_u32(s.cb);
            const uint32_t sB = sXw + 2 * kBox;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_ts(tY, tPm + kk * 8, smem_desc(sX + kk * 2048, 0, 1024), id_kmn, true);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_ts(tY, tEC + kk * 8, smem_desc(sHp + kk * 2048, 0, 1024), id_kmn, true);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_ss(tS, smem_desc(sB + kk * 2048, kBox, 1024), smem_desc(sXw + kk * 2048, 0, 1024),
                       id_mnmn, kk > 0);
            mma_commit(&s.mma_done);
        }
        ok = mbar_wait(&s.mma_done, c & 1, abort, lim);
        if (!__syncthreads_and(ok)) { raise_timeout(p, abort); break; }
        tc_fence_after();
        // every operand slot is free: fetch the next chunk while this one finishes
        if (tid == 0 && c + 1 < nc) {
            issue_loads(c + 1);
            pending = c + 1;
        }
        // ---- y = Y, this half's 32 columns
        {
            uint32_t yv[32];
            tmem_ld32(tY + lane_base + 32 * hs, yv);
            tmem_wait_ld();
            if (t0 + r < s1) {
                __nv_bfloat16 *yrow = ybase + (t0 + r) * p.yrs;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t o4[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2)
                        o4[e2] = pack_bf16x2(__uint_as_float(yv[8 * c4 + 2 * e2]), __uint_as_float(yv[8 * c4 + 2 * e2 + 1]));
                    *reinterpret_cast<uint4 *>(yrow + 8 * c4) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
                }
            }
        }
        // ---- state: h = exp(cs_last) h + S  (columns p of this half, state column n = r)
        {
            uint32_t sa[32];
            tmem_ld32(tS + lane_base + 32 * hs, sa);
            tmem_wait_ld();
            const float dec = ex2(tot2);
#pragma unroll
            for (int pp = 0; pp < 32; ++pp) hr[pp] = fmaf(dec, hr[pp], __uint_as_float(sa[pp]));
        }
        if (c + 1 < nc) {
            write_hp();
            fence_proxy_async_smem();   // before the barrier that orders it with the next MMAs
        }
        const int64_t t_end = t0 + kQ;
        if (p.h_ckpt && p.s > 0 && t_end <= s1 && t_end % p.s == 0) {
            const int64_t kk = t_end / p.s - 1;
            if (kk < n_ckpt) {
                float *dst = p.h_ckpt + (((int64_t)bi * n_ckpt + kk) * p.H + h) * PN + (int64_t)(32 * hs) * kN + r;
#pragma unroll
                for (int pp = 0; pp < 32; ++pp) dst[pp * kN] = hr[pp];
            }
        }
        tc_fence_before();
    }
    if (!*abort && p.h_final && s1 == p.L) {
        float *dst = p.h_final + ((int64_t)bi * p.H + h) * PN + (int64_t)(32 * hs) * kN + r;
#pragma unroll
        for (int pp = 0; pp < 32; ++pp) dst[pp * kN] = hr[pp];
    }
    // drain: MMAs and loads that may still be in flight after an abort
    if (tid == 0 && *abort) {
        mma_commit(&s.fin);
        mbar_wait(&s.fin, 0, nullptr, 100000000ull);
        if (pending >= 0) mbar_wait(&s.full, pending & 1, nullptr, 100000000ull);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 256);
}

// =============================================================== host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
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

// [b][L][cols] view with element strides (rs, bs); box = 64 columns x 128 rows
bool encode_bf16(EncodeTiledFn enc, CUtensorMap *m, const void *base, int64_t cols, int64_t L, int b,
                 int64_t rs, int64_t bs)
{
    if (b == 1) bs = rs * L;
    const cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)L, (cuuint64_t)b};
    const cuuint64_t strides[2] = {(cuuint64_t)rs * 2, (cuuint64_t)bs * 2};
    const cuuint32_t box[3] = {64, 128, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_dt(EncodeTiledFn enc, CUtensorMap *m, const float *dt, int H, int64_t L, int b)
{
    const cuuint64_t dims[3] = {(cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)b};
    const cuuint64_t strides[2] = {(cuuint64_t)H * 4, (cuuint64_t)H * 4 * L};
    const cuuint32_t box[3] = {4, 128, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(dt), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t kSmemA = sizeof(SmemA) + 1024;
constexpr size_t kSmemC = sizeof(SmemC) + 1024;
static_assert(kSmemC <= 232448, "pass C shared memory");
static_assert(kSmemA <= 232448, "pass A shared memory");

}  // namespace

bool tc_scan_supported(const ScanParams &p, int dtype)
{
    if (dtype != 1 || p.P != kP || p.N != kN || p.Q != kQ) return false;
    if (p.H % 4 != 0 || (p.H / p.G) % 2 != 0) return false;  // head pairs share a B/C group
    if ((reinterpret_cast<uintptr_t>(p.dt) & 15u) != 0) return false;
    if (p.L >= (1LL << 31) || (int64_t)p.b * p.ns * p.H >= (1LL << 31)) return false;
    return encode_fn() != nullptr;
}

int launch_scan_tc(const ScanParams &p, cudaStream_t st)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return 6;
    Maps maps;
    const int64_t gn = (int64_t)p.G * p.N;
    if (!encode_bf16(enc, &maps.x, p.x, (int64_t)p.H * p.P, p.L, p.b, p.xrs, p.xbs) ||
        !encode_bf16(enc, &maps.B, p.B, gn, p.L, p.b, p.Brs, p.Bbs) ||
        !encode_bf16(enc, &maps.C, p.C, gn, p.L, p.b, p.Crs, p.Cbs) ||
        !encode_dt(enc, &maps.dt, p.dt, p.H, p.L, p.b))
        return 6;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(stripe_state_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemA) != cudaSuccess ||
            cudaFuncSetAttribute(chunk_output_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemC) != cudaSuccess)
            return 7;
        attr_set[dev] = true;
    }
    const int64_t units = (int64_t)p.b * p.ns * p.H;
    if (p.ns > 1) {
        prof_begin(st, kKStateTc);
        stripe_state_tc_kernel<<<(unsigned)(units / 2), kThreads, kSmemA, st>>>(maps, p);
        prof_end(st, kKStateTc);
        const int rc = launch_chain(p, st);
        if (rc) return rc;
    }
    prof_begin(st, kKOutputTc);
    chunk_output_tc_kernel<<<(unsigned)units, kThreadsC, kSmemC, st>>>(maps, p);
    prof_end(st, kKOutputTc);
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

}  // namespace ssd

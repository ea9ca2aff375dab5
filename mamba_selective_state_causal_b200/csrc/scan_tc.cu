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
struct SmemA {
    uint8_t stage[3][3 * kBox + kDtBox];  // B (two boxes), X, dt
    uint8_t xw[2][kBox];
    float scratch[2][4];
    uint64_t full[3], empty[3], xw_full[2], xw_empty[2], acc_full, fin, epi;
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
    const int h = (int)(unit % p.H);
    const int64_t k = (unit / p.H) % p.ns;
    const int bi = (int)(unit / ((int64_t)p.H * p.ns));
    const int g = (int)((int64_t)h * p.G / p.H);
    const int64_t s0 = k * p.T;
    const int64_t s1 = min(p.L, s0 + p.T);
    const int nc = (int)((s1 - s0 + kQ - 1) / kQ);

    if (threadIdx.x == 0) {
        for (int i = 0; i < 3; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1 + 128); }
        for (int i = 0; i < 2; ++i) { mbar_init(&s.xw_full[i], 128); mbar_init(&s.xw_empty[i], 1); }
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
    if (warp == 1) { tmem_alloc(&s.tmem, 64); tmem_relinquish(); }
    __syncthreads();
    tc_fence_after();
    const uint32_t tS = s.tmem;
    volatile int *abort = &s.abort;

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            for (int it = 0; it < nc; ++it) {
                const int st = it % 3, u = it / 3;
                if (it >= 3 && !mbar_wait(&s.empty[st], (u - 1) & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
                if (unit == p.test_drop_unit) break;  // test hook: this unit's loads never arrive
                const int c = nc - 1 - it;  // chunks in reverse order
                const int t0 = (int)(s0 + (int64_t)c * kQ);
                uint8_t *sb = s.stage[st];
                mbar_arrive_expect_tx(&s.full[st], 3 * kBox + kDtBox);
                tma_load_3d(sb, &maps.B, &s.full[st], g * kN, t0, bi);
                tma_load_3d(sb + kBox, &maps.B, &s.full[st], g * kN + 64, t0, bi);
                tma_load_3d(sb + 2 * kBox, &maps.x, &s.full[st], h * kP, t0, bi);
                tma_load_3d(sb + 3 * kBox, &maps.dt, &s.full[st], h & ~3, t0, bi);
                issued = it + 1;
            }
            if (*abort) {  // let copies in flight land before the CTA exits
                for (int it = max(0, issued - 3); it < issued; ++it)
                    mbar_wait(&s.full[it % 3], (it / 3) & 1, nullptr, 100000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id = idesc_bf16(128, 64, 1, 1);
            bool okk = true;
            for (int it = 0; it < nc && okk; ++it) {
                const int st = it % 3, u = it / 3, xb = it & 1;
                if (!mbar_wait(&s.full[st], u & 1, abort, p.wait_limit_ns) || !mbar_wait(&s.xw_full[xb], (it >> 1) & 1, abort, p.wait_limit_ns)) {
                    raise_timeout(p, abort);
                    okk = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sB = smem_u32(s.stage[st]);
                const uint32_t sXw = smem_u32(s.xw[xb]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tS, smem_desc(sB + kk * 2048, kBox, 1024), smem_desc(sXw + kk * 2048, 0, 1024), id,
                           it > 0 || kk > 0);
                mma_commit(&s.empty[st]);
                mma_commit(&s.xw_empty[xb]);
            }
            mma_commit(&s.acc_full);
            mma_commit(&s.fin);
            mbar_wait(&s.fin, 0, nullptr, 200000000ull);
        }
    } else {
        const int r = 32 * (warp & 3) + lane;  // token row / TMEM lane
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        const float A2 = p.A[h] * kLog2e;
        float suf2 = 0.0f;
        bool okk = true;
        uint32_t eph = 0;
        for (int it = 0; it < nc; ++it) {
            const int st = it % 3, u = it / 3, xb = it & 1;
            if (!ewait(&s.full[st], u & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); okk = false; break; }
            const uint8_t *sb = s.stage[st];
            const float dt_r = reinterpret_cast<const float *>(sb + 3 * kBox)[r * 4 + (h & 3)];
            float tot2, cs2 = dt_r * A2;
            if (!epi_scan(cs2, r, s.scratch[it & 1], tot2, &s.epi, eph, abort, p.wait_limit_ns)) {
                raise_timeout(p, abort);
                okk = false;
                break;
            }
            const float w = dt_r * ex2((tot2 - cs2) + suf2);
            if (it >= 2 && !ewait(&s.xw_empty[xb], ((it >> 1) - 1) & 1, abort, p.wait_limit_ns)) {
                raise_timeout(p, abort);
                okk = false;
                break;
            }
            const uint8_t *xrow = sb + 2 * kBox;
            uint8_t *xwt = s.xw[xb];
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                const uint32_t o = swz(r, cc);
                uint4 v = lds128(xrow + o);
                v.x = scale_bf16x2(v.x, w); v.y = scale_bf16x2(v.y, w);
                v.z = scale_bf16x2(v.z, w); v.w = scale_bf16x2(v.w, w);
                sts128(xwt + o, v);
            }
            fence_proxy_async_smem();
            mbar_arrive(&s.xw_full[xb]);
            mbar_arrive(&s.empty[st]);
            suf2 += tot2;
        }
        if (okk && ewait(&s.acc_full, 0, abort, p.wait_limit_ns)) {
            tc_fence_after();
            uint32_t a[32], b[32];
            tmem_ld32(tS + lane_base, a);
            tmem_ld32(tS + lane_base + 32, b);
            tmem_wait_ld();
            float *dst = p.ws_S + (((int64_t)bi * p.ns + k) * p.H + h) * (kP * kN) + r;
#pragma unroll
            for (int pp = 0; pp < 32; ++pp) dst[pp * kN] = __uint_as_float(a[pp]);
#pragma unroll
            for (int pp = 0; pp < 32; ++pp) dst[(pp + 32) * kN] = __uint_as_float(b[pp]);
            if (r == 0) p.ws_dA[((int64_t)bi * p.ns + k) * p.H + h] = suf2 * kLn2;
        } else if (okk) {
            raise_timeout(p, abort);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tS, 64);
}

// =============================================================== pass C
struct SmemC {
    uint8_t stage[2][5 * kBox + kDtBox];  // C (two boxes), B (two boxes), X, dt
    uint8_t xw[kBox];
    uint8_t hp[kBox];                     // bf16 h_prev, rows n, 128B-swizzled
    float cs2[kQ];
    float dts[kQ];
    float scratch[2][4];
    uint64_t full[2], empty[2], g_full[2], pm_full[2], pm_free[2];
    uint64_t y_full, acc_empty, xw_full, xw_empty, s_full, s_empty, hp_full, fin, epi;
    uint32_t tmem;
    int abort;
};

__device__ __forceinline__ void write_hp(uint8_t *hp, int n, const float (&hr)[64])
{
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        uint4 v;
        v.x = pack_bf16x2(hr[8 * cc + 0], hr[8 * cc + 1]);
        v.y = pack_bf16x2(hr[8 * cc + 2], hr[8 * cc + 3]);
        v.z = pack_bf16x2(hr[8 * cc + 4], hr[8 * cc + 5]);
        v.w = pack_bf16x2(hr[8 * cc + 6], hr[8 * cc + 7]);
        sts128(hp + swz(n, cc), v);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_output_tc_kernel(const __grid_constant__ Maps maps, const ScanParams p)
{
    extern __shared__ uint8_t smraw[];
    SmemC &s = *reinterpret_cast<SmemC *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t unit = blockIdx.x;
    const int h = (int)(unit % p.H);
    const int64_t k = (unit / p.H) % p.ns;
    const int bi = (int)(unit / ((int64_t)p.H * p.ns));
    const int g = (int)((int64_t)h * p.G / p.H);
    const int64_t s0 = k * p.T;
    const int64_t s1 = min(p.L, s0 + p.T);
    const int nc = (int)((s1 - s0 + kQ - 1) / kQ);

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1 + 128);
            mbar_init(&s.g_full[i], 1);
            mbar_init(&s.pm_full[i], 128);
            mbar_init(&s.pm_free[i], 1);
        }
        mbar_init(&s.y_full, 1);
        mbar_init(&s.acc_empty, 128);
        mbar_init(&s.xw_full, 128);
        mbar_init(&s.xw_empty, 1);
        mbar_init(&s.s_full, 1);
        mbar_init(&s.s_empty, 128);
        mbar_init(&s.hp_full, 128);
        mbar_init(&s.fin, 1);
        mbar_init(&s.epi, 128);
        s.abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&maps.x);
        prefetch_tmap(&maps.B);
        prefetch_tmap(&maps.C);
        prefetch_tmap(&maps.dt);
    }
    if (warp == 1) { tmem_alloc(&s.tmem, 512); tmem_relinquish(); }
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = s.tmem;
    const uint32_t tYd = tm + 256, tYo = tm + 320, tS = tm + 384;
    volatile int *abort = &s.abort;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int c = 0; c < nc; ++c) {
                const int st = c & 1, u = c >> 1;
                if (c >= 2 && !mbar_wait(&s.empty[st], (u - 1) & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
                if (unit == p.test_drop_unit) break;  // test hook: this unit's loads never arrive
                const int t0 = (int)(s0 + (int64_t)c * kQ);
                uint8_t *sb = s.stage[st];
                mbar_arrive_expect_tx(&s.full[st], 5 * kBox + kDtBox);
                tma_load_3d(sb, &maps.C, &s.full[st], g * kN, t0, bi);
                tma_load_3d(sb + kBox, &maps.C, &s.full[st], g * kN + 64, t0, bi);
                tma_load_3d(sb + 2 * kBox, &maps.B, &s.full[st], g * kN, t0, bi);
                tma_load_3d(sb + 3 * kBox, &maps.B, &s.full[st], g * kN + 64, t0, bi);
                tma_load_3d(sb + 4 * kBox, &maps.x, &s.full[st], h * kP, t0, bi);
                tma_load_3d(sb + 5 * kBox, &maps.dt, &s.full[st], h & ~3, t0, bi);
                issued = c + 1;
            }
            if (*abort) {
                for (int c = max(0, issued - 2); c < issued; ++c)
                    mbar_wait(&s.full[c & 1], (c >> 1) & 1, nullptr, 100000000ull);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_g = idesc_bf16(128, 128, 0, 0);
            const uint32_t id_kmn = idesc_bf16(128, 64, 0, 1);
            const uint32_t id_mnmn = idesc_bf16(128, 64, 1, 1);
            const uint32_t sHp = smem_u32(s.hp), sXw = smem_u32(s.xw);
            for (int c = 0; c < nc; ++c) {
                const int st = c & 1, u = c >> 1, buf = c & 1;
                const uint32_t tG = tm + 128 * buf;
                if (!mbar_wait(&s.full[st], u & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
                if (c >= 2 && !mbar_wait(&s.pm_free[buf], ((c >> 1) - 1) & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
                tc_fence_after();
                const uint32_t sC = smem_u32(s.stage[st]);
                const uint32_t sB = sC + 2 * kBox, sX = sC + 4 * kBox;
                // G = C B^T
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                    mma_ss(tG, smem_desc(sC + off, 16, 1024), smem_desc(sB + off, 16, 1024), id_g, kk > 0);
                }
                mma_commit(&s.g_full[buf]);
                // Yo = C h_prev^T
                if (!mbar_wait(&s.hp_full, c & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
                if (c >= 1 && !mbar_wait(&s.acc_empty, (c - 1) & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                    mma_ss(tYo, smem_desc(sC + off, 16, 1024), smem_desc(sHp + kk * 2048, 0, 1024), id_kmn, kk > 0);
                }
                // Yd = Pm X   (Pm: bf16 in TMEM, written over G)
                if (!mbar_wait(&s.pm_full[buf], (c >> 1) & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tYd, tG + kk * 8, smem_desc(sX + kk * 2048, 0, 1024), id_kmn, kk > 0);
                mma_commit(&s.y_full);
                mma_commit(&s.pm_free[buf]);
                // S = B^T (w o X)
                if (!mbar_wait(&s.xw_full, c & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
                if (c >= 1 && !mbar_wait(&s.s_empty, (c - 1) & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tS, smem_desc(sB + kk * 2048, kBox, 1024), smem_desc(sXw + kk * 2048, 0, 1024),
                           id_mnmn, kk > 0);
                mma_commit(&s.s_full);
                mma_commit(&s.xw_empty);
                mma_commit(&s.empty[st]);
            }
            mma_commit(&s.fin);
            mbar_wait(&s.fin, 0, nullptr, 200000000ull);
        }
    } else {
        // ------------------------------------------------ epilogue: rows r = TMEM lanes
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const float A2 = p.A[h] * kLog2e;
        const float Dh = p.D ? p.D[h] : 0.0f;
        const int64_t n_ckpt = p.s > 0 ? p.L / p.s : 0;
        const int PN = kP * kN;
        float hr[64];
        {
            const float *hin = (k == 0) ? (p.h0 ? p.h0 + ((int64_t)bi * p.H + h) * PN : nullptr)
                                        : p.ws_hin + (((int64_t)bi * p.ns + k) * p.H + h) * PN;
#pragma unroll
            for (int pp = 0; pp < 64; ++pp) hr[pp] = hin ? hin[pp * kN + r] : 0.0f;
        }
        write_hp(s.hp, r, hr);
        fence_proxy_async_smem();
        mbar_arrive(&s.hp_full);

        __nv_bfloat16 *ybase = reinterpret_cast<__nv_bfloat16 *>(p.y) + (int64_t)bi * p.ybs + (int64_t)h * kP;
        uint32_t eph = 0;
        for (int c = 0; c < nc; ++c) {
            const int st = c & 1, u = c >> 1, buf = c & 1;
            const uint32_t tG = tm + 128 * buf;
            const int64_t t0 = s0 + (int64_t)c * kQ;
            if (!ewait(&s.full[st], u & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
            const uint8_t *sb = s.stage[st];
            const uint8_t *xt = sb + 4 * kBox;
            const float dt_r = reinterpret_cast<const float *>(sb + 5 * kBox)[r * 4 + (h & 3)];
            float tot2, cs2 = dt_r * A2;
            if (!epi_scan(cs2, r, s.scratch[c & 1], tot2, &s.epi, eph, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
            s.cs2[r] = cs2;
            s.dts[r] = dt_r;
            if (!epi_sync(&s.epi, eph, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }

            // ---- w o X for the state update
            if (c >= 1 && !ewait(&s.xw_empty, (c - 1) & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
            {
                const float w = dt_r * ex2(tot2 - cs2);
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const uint32_t o = swz(r, cc);
                    uint4 v = lds128(xt + o);
                    v.x = scale_bf16x2(v.x, w); v.y = scale_bf16x2(v.y, w);
                    v.z = scale_bf16x2(v.z, w); v.w = scale_bf16x2(v.w, w);
                    sts128(s.xw + o, v);
                }
                fence_proxy_async_smem();
                mbar_arrive(&s.xw_full);
            }

            // ---- masked decay: Pm[r][j] = G[r][j] * exp(cs_r - cs_j) * dt_j for j <= r
            if (!ewait(&s.g_full[buf], (c >> 1) & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
            tc_fence_after();
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) {
                uint32_t pk[16];
                if (jb <= q) {
                    uint32_t gv[32];
                    tmem_ld32(tG + lane_base + 32 * jb, gv);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int j0 = 32 * jb + 2 * i;
                        float v0 = __uint_as_float(gv[2 * i]) * ex2(cs2 - s.cs2[j0]) * s.dts[j0];
                        float v1 = __uint_as_float(gv[2 * i + 1]) * ex2(cs2 - s.cs2[j0 + 1]) * s.dts[j0 + 1];
                        if (j0 > r) v0 = 0.0f;
                        if (j0 + 1 > r) v1 = 0.0f;
                        pk[i] = pack_bf16x2(v0, v1);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = 0u;
                }
                tmem_st16(tG + lane_base + 16 * jb, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&s.pm_full[buf]);

            // ---- outputs y = Yd + exp(cs_r) Yo + D x
            if (!ewait(&s.y_full, c & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
            tc_fence_after();
            {
                const float e = ex2(cs2);
                const bool valid = t0 + r < s1;
                __nv_bfloat16 *yrow = ybase + (t0 + r) * p.yrs;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t yd[32], yo[32];
                    tmem_ld32(tYd + lane_base + 32 * half, yd);
                    tmem_ld32(tYo + lane_base + 32 * half, yo);
                    tmem_wait_ld();
                    if (half == 1) {
                        tc_fence_before();
                        mbar_arrive(&s.acc_empty);
                    }
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const int cc = 4 * half + c4;
                        const uint4 xv = lds128(xt + swz(r, cc));
                        const uint32_t xw4[4] = {xv.x, xv.y, xv.z, xv.w};
                        uint32_t o4[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int i0 = 8 * c4 + 2 * e2;
                            const float a0 = __uint_as_float(yd[i0]) + e * __uint_as_float(yo[i0]) + Dh * bf16_lo(xw4[e2]);
                            const float a1 = __uint_as_float(yd[i0 + 1]) + e * __uint_as_float(yo[i0 + 1]) + Dh * bf16_hi(xw4[e2]);
                            o4[e2] = pack_bf16x2(a0, a1);
                        }
                        if (valid) *reinterpret_cast<uint4 *>(yrow + 8 * cc) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
                    }
                }
            }
            mbar_arrive(&s.empty[st]);

            // ---- state update h = exp(cs_last) h + S  (thread r owns state column n = r)
            if (!ewait(&s.s_full, c & 1, abort, p.wait_limit_ns)) { raise_timeout(p, abort); break; }
            tc_fence_after();
            {
                uint32_t sa[32], sbv[32];
                tmem_ld32(tS + lane_base, sa);
                tmem_ld32(tS + lane_base + 32, sbv);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&s.s_empty);
                const float dec = ex2(tot2);
#pragma unroll
                for (int pp = 0; pp < 32; ++pp) hr[pp] = fmaf(dec, hr[pp], __uint_as_float(sa[pp]));
#pragma unroll
                for (int pp = 0; pp < 32; ++pp) hr[pp + 32] = fmaf(dec, hr[pp + 32], __uint_as_float(sbv[pp]));
            }
            if (c + 1 < nc) {
                write_hp(s.hp, r, hr);
                fence_proxy_async_smem();
                mbar_arrive(&s.hp_full);
            }
            const int64_t t_end = t0 + kQ;
            if (p.h_ckpt && p.s > 0 && t_end <= s1 && t_end % p.s == 0) {
                const int64_t kk = t_end / p.s - 1;
                if (kk < n_ckpt) {
                    float *dst = p.h_ckpt + (((int64_t)bi * n_ckpt + kk) * p.H + h) * PN + r;
#pragma unroll
                    for (int pp = 0; pp < 64; ++pp) dst[pp * kN] = hr[pp];
                }
            }
        }
        if (!*abort && p.h_final && s1 == p.L) {
            float *dst = p.h_final + ((int64_t)bi * p.H + h) * PN + r;
#pragma unroll
            for (int pp = 0; pp < 64; ++pp) dst[pp * kN] = hr[pp];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tm, 512);
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
    if (p.H % 4 != 0) return false;
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
        stripe_state_tc_kernel<<<(unsigned)units, kThreads, kSmemA, st>>>(maps, p);
        prof_end(st, kKStateTc);
        const int rc = launch_chain(p, st);
        if (rc) return rc;
    }
    prof_begin(st, kKOutputTc);
    chunk_output_tc_kernel<<<(unsigned)units, kThreads, kSmemC, st>>>(maps, p);
    prof_end(st, kKOutputTc);
    return cudaGetLastError() == cudaSuccess ? 0 : 7;
}

}  // namespace ssd

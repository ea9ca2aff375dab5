// ssd_api.cu -- the C ABI declared in include/ssd.h: argument checks, the
// stripe plan, workspace carving and dispatch to the CUDA kernels.
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <atomic>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/ssd.h"
#include "ssd_common.cuh"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int ok()
{
    g_last_error.clear();
    return SSD_OK;
}

// Per-device status word written by kernels when a bounded wait gives up.
__device__ unsigned int g_device_status;

constexpr int kMaxDevices = 64;
// Looked up once per device.  Host threads may race on the first lookup; they all
// store the same value, and the atomics make that race well defined.
std::atomic<unsigned int *> g_status_ptr[kMaxDevices];

unsigned int *status_ptr()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    unsigned int *sp = g_status_ptr[dev].load(std::memory_order_acquire);
    if (!sp) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        sp = static_cast<unsigned int *>(p);
        g_status_ptr[dev].store(sp, std::memory_order_release);
    }
    return sp;
}

// Test and diagnostic hooks, read from the environment once per process (the
// first scan call) and documented in include/ssd.h:
//   SSD_WAIT_LIMIT_MS   bound of every device-side wait, in ms (default 2000)
//   SSD_TEST_DROP_UNIT  index of one work unit of the first scan call of the process
//                       whose loads are never issued, so that its waits run out
//                       (failure-detection test); later calls run normally
//   SSD_SCAN_PATH       "generic" forces the CUDA-core scan kernels
struct EnvHooks {
    uint64_t wait_limit_ns;
    int64_t test_drop_unit;
    bool force_generic;
};

const EnvHooks &env_hooks()
{
    static const EnvHooks h = [] {
        EnvHooks e{};
        const char *lim = getenv("SSD_WAIT_LIMIT_MS");
        const long long ms = lim ? atoll(lim) : 2000;
        e.wait_limit_ns = (uint64_t)(ms > 0 ? ms : 2000) * 1000000ull;
        const char *drop = getenv("SSD_TEST_DROP_UNIT");
        e.test_drop_unit = drop ? atoll(drop) : -1;
        const char *path = getenv("SSD_SCAN_PATH");
        e.force_generic = path && strcmp(path, "generic") == 0;
        return e;
    }();
    return h;
}

size_t elem_size(int dtype) { return dtype == SSD_BF16 ? 2 : 4; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool pow2_dim(int v) { return v == 16 || v == 32 || v == 64 || v == 128; }

struct Plan {
    int64_t T = 0, ns = 0;
    size_t off_S = 0, off_hin = 0, off_dA = 0, bytes = 0;
    // the dt surroundings' buffer (effective dt [b][L][H] fp32) follows the stripe states;
    // it is needed only when a call asks for dt_bias / softplus / a clamp
    size_t off_dt = 0, bytes_dt = 0;
};

size_t round256(size_t v) { return (v + 255) & ~size_t(255); }

// Stripe plan: the sequence is split into stripes of T tokens (a multiple of Q).
// The tensor-core passes run one CTA per SM and one (stripe, head pair) unit
// per CTA, so a pass takes about
//     waves x (chunks per stripe + 2),   waves = ceil(units / SMs),
// the 2 standing for a unit's fixed cost (pipeline fill and drain) in chunks.
// The plan takes the stripe length that minimises it on the current device and,
// among equal costs, the fewest stripes (less chain work, smaller workspace).
int sm_count()
{
    static std::atomic<int> cached[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    int n = cached[dev].load(std::memory_order_acquire);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev].store(n, std::memory_order_release);
    }
    return n;
}

Plan make_plan(int b, int64_t L, int H, int P, int N, int Q)
{
    Plan pl;
    if (b <= 0 || L <= 0 || H <= 0 || Q <= 0) return pl;
    const int64_t nchunks = (L + Q - 1) / Q;
    const int64_t hp = (H % 2 == 0) ? H / 2 : H;
    const int64_t nsm = sm_count();
    int64_t best_cost = -1, best_tc = nchunks;
    const int64_t max_ns = std::min<int64_t>(nchunks, 16384);
    for (int64_t ns = 1; ns <= max_ns; ++ns) {
        const int64_t tc = (nchunks + ns - 1) / ns;      // chunks per stripe
        const int64_t real_ns = (nchunks + tc - 1) / tc;
        if (real_ns != ns) continue;                     // the same plan as a smaller ns
        const int64_t waves = ((int64_t)b * real_ns * hp + nsm - 1) / nsm;
        const int64_t cost = waves * (tc + 2);
        if (best_cost < 0 || cost < best_cost) { best_cost = cost; best_tc = tc; }
    }
    pl.T = best_tc * Q;
    pl.ns = (L + pl.T - 1) / pl.T;
    if (pl.ns > 1) {
        const size_t state = sizeof(float) * (size_t)b * pl.ns * H * P * N;
        pl.off_S = 0;
        pl.off_hin = round256(state);
        pl.off_dA = pl.off_hin + round256(state);
        pl.bytes = pl.off_dA + round256(sizeof(float) * (size_t)b * pl.ns * H);
    }
    pl.off_dt = round256(pl.bytes);
    pl.bytes_dt = pl.off_dt + round256(sizeof(float) * (size_t)b * L * H);
    return pl;
}

int check_scan_shape(int dtype, int b, int64_t L, int H, int P, int N, int G, int Q, int64_t s)
{
    if (dtype != SSD_F32 && dtype != SSD_BF16) return fail(SSD_ERR_DTYPE, "unknown dtype %d", dtype);
    if (b < 0 || L < 0) return fail(SSD_ERR_SHAPE, "negative b (%d) or L (%lld)", b, (long long)L);
    if (H <= 0 || G <= 0 || H % G != 0)
        return fail(SSD_ERR_SHAPE, "need H > 0, G > 0 and H %% G == 0 (H=%d, G=%d)", H, G);
    if (!pow2_dim(P) || !pow2_dim(N))
        return fail(SSD_ERR_SHAPE, "P and N must be 16, 32, 64 or 128 (P=%d, N=%d)", P, N);
    if (Q != 32 && Q != 64 && Q != 128) return fail(SSD_ERR_SHAPE, "Q must be 32, 64 or 128 (Q=%d)", Q);
    if (s < 0 || (s > 0 && s % Q != 0))
        return fail(SSD_ERR_SHAPE, "checkpoint stride s=%lld must be 0 or a multiple of Q=%d",
                    (long long)s, Q);
    return SSD_OK;
}

int check_rows(const char *name, const void *ptr, int64_t bs, int64_t rs, int64_t width,
               int b, int64_t L, int dtype, bool need_align)
{
    if (!ptr) return fail(SSD_ERR_NULL, "%s is NULL", name);
    if (rs < width) return fail(SSD_ERR_STRIDE, "%s row stride %lld < row width %lld", name,
                                (long long)rs, (long long)width);
    if (b > 1 && bs < rs * L)
        return fail(SSD_ERR_STRIDE, "%s batch stride %lld < L * row stride", name, (long long)bs);
    if (bs < 0) return fail(SSD_ERR_STRIDE, "%s batch stride is negative", name);
    if (need_align) {
        const size_t es = elem_size(dtype);
        if (!aligned16(ptr) || (rs * es) % 16 != 0 || (bs * es) % 16 != 0)
            return fail(SSD_ERR_ALIGN, "%s must be 16-byte aligned with 16-byte row/batch strides", name);
    }
    return SSD_OK;
}

int scan_impl(const ssd_scan_args *a, cudaStream_t st)
{
    if (!a) return fail(SSD_ERR_NULL, "args is NULL");
    int rc = check_scan_shape(a->dtype, a->b, a->L, a->H, a->P, a->N, a->G, a->Q, a->s);
    if (rc) return rc;
    if (a->b == 0) return ok();
    if (a->L > 0) {
        if ((rc = check_rows("x", a->x, a->x_batch_stride, a->x_row_stride, (int64_t)a->H * a->P, a->b, a->L, a->dtype, true))) return rc;
        if ((rc = check_rows("B", a->B, a->B_batch_stride, a->B_row_stride, (int64_t)a->G * a->N, a->b, a->L, a->dtype, true))) return rc;
        if ((rc = check_rows("C", a->C, a->C_batch_stride, a->C_row_stride, (int64_t)a->G * a->N, a->b, a->L, a->dtype, true))) return rc;
        if ((rc = check_rows("y", a->y, a->y_batch_stride, a->y_row_stride, (int64_t)a->H * a->P, a->b, a->L, a->dtype, true))) return rc;
        if (!a->dt) return fail(SSD_ERR_NULL, "dt is NULL");
        if (!a->A) return fail(SSD_ERR_NULL, "A is NULL");
    }
    const Plan pl = make_plan(a->b, a->L, a->H, a->P, a->N, a->Q);
    const bool dtx = a->dt_bias || a->dt_softplus || a->dt_max > 0.0f;
    const size_t need = dtx ? pl.bytes_dt : pl.bytes;
    if (need > 0) {
        if (!a->workspace || a->workspace_bytes < need)
            return fail(SSD_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                        a->workspace ? a->workspace_bytes : (size_t)0);
        if ((reinterpret_cast<uintptr_t>(a->workspace) & 255u) != 0)
            return fail(SSD_ERR_ALIGN, "workspace must be 256-byte aligned");
    }
    const size_t state_bytes = sizeof(float) * (size_t)a->b * a->H * a->P * a->N;
    if (a->L == 0) {
        // no token: the final state is the initial state
        if (a->h_final && a->h_final != a->h0) {
            cudaError_t e = a->h0 ? cudaMemcpyAsync(a->h_final, a->h0, state_bytes, cudaMemcpyDeviceToDevice, st)
                                  : cudaMemsetAsync(a->h_final, 0, state_bytes, st);
            if (e != cudaSuccess) return fail(SSD_ERR_LAUNCH, "%s", cudaGetErrorString(e));
        }
        return ok();
    }
    ssd::ScanParams p{};
    p.b = a->b; p.L = a->L; p.H = a->H; p.P = a->P; p.N = a->N; p.G = a->G; p.Q = a->Q; p.s = a->s;
    p.x = a->x; p.xbs = a->x_batch_stride; p.xrs = a->x_row_stride;
    p.B = a->B; p.Bbs = a->B_batch_stride; p.Brs = a->B_row_stride;
    p.C = a->C; p.Cbs = a->C_batch_stride; p.Crs = a->C_row_stride;
    p.dt = a->dt; p.A = a->A; p.D = a->D; p.h0 = a->h0;
    p.dt_bias = a->dt_bias; p.dt_softplus = a->dt_softplus; p.dt_min = a->dt_min; p.dt_max = a->dt_max;
    p.y = a->y; p.ybs = a->y_batch_stride; p.yrs = a->y_row_stride;
    p.h_final = a->h_final; p.h_ckpt = a->h_ckpt;
    p.T = pl.T; p.ns = pl.ns;
    char *ws = static_cast<char *>(a->workspace);
    p.ws_S = pl.bytes ? reinterpret_cast<float *>(ws + pl.off_S) : nullptr;
    p.ws_hin = pl.bytes ? reinterpret_cast<float *>(ws + pl.off_hin) : nullptr;
    p.ws_dA = pl.bytes ? reinterpret_cast<float *>(ws + pl.off_dA) : nullptr;
    if (dtx) {
        // the effective dt goes to the workspace first; the scan kernels read it as plain dt
        float *dte = reinterpret_cast<float *>(ws + pl.off_dt);
        if (ssd::launch_dt_prepare(p, dte, st))
            return fail(SSD_ERR_LAUNCH, "dt launch failed: %s", cudaGetErrorString(cudaGetLastError()));
        p.dt = dte;
        p.dt_bias = nullptr; p.dt_softplus = 0; p.dt_min = 0.0f; p.dt_max = 0.0f;
    }
    p.status = status_ptr();
    if (!p.status) return fail(SSD_ERR_LAUNCH, "no CUDA device available");
    const EnvHooks &hooks = env_hooks();
    p.wait_limit_ns = hooks.wait_limit_ns;
    static std::atomic<bool> drop_used{false};
    p.test_drop_unit = (hooks.test_drop_unit >= 0 && !drop_used.exchange(true)) ? hooks.test_drop_unit : -1;
    // SSD_SCAN_PATH=generic forces the CUDA-core kernels (used to cross-check the paths)
    const bool force_generic = hooks.force_generic;
    rc = 6;
    if (!force_generic && ssd::tc_scan_supported(p, a->dtype)) rc = ssd::launch_scan_tc(p, st);
    if (rc == 6) rc = ssd::launch_scan_generic(p, a->dtype, st);
    if (rc == 6) return fail(SSD_ERR_UNSUPPORTED, "no GPU kernel for this shape (P=%d N=%d Q=%d)", a->P, a->N, a->Q);
    if (rc) return fail(SSD_ERR_LAUNCH, "scan launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    return ok();
}

// Backward workspace: ws_h, ws_g [b][H][nch][P][N]; ws_lam, ws_pA, ws_pD [b][H][nch];
// ws_dBh, ws_dCh [b][L][H][N] (all fp32, each part 256-byte aligned).
struct BwdPlan {
    int64_t nch = 0;
    size_t off_h = 0, off_g = 0, off_lam = 0, off_pA = 0, off_pD = 0, off_dB = 0, off_dC = 0, bytes = 0;
};

BwdPlan make_bwd_plan(int b, int64_t L, int H, int P, int N)
{
    BwdPlan pl;
    if (b <= 0 || L <= 0 || H <= 0 || P <= 0 || N <= 0) return pl;
    pl.nch = (L + 63) / 64;
    const size_t states = sizeof(float) * (size_t)b * H * pl.nch * P * N;
    const size_t per_chunk = sizeof(float) * (size_t)b * H * pl.nch;
    const size_t per_token = sizeof(float) * (size_t)b * L * H * N;
    pl.off_h = 0;
    pl.off_g = round256(states);
    pl.off_lam = pl.off_g + round256(states);
    pl.off_pA = pl.off_lam + round256(per_chunk);
    pl.off_pD = pl.off_pA + round256(per_chunk);
    pl.off_dB = pl.off_pD + round256(per_chunk);
    pl.off_dC = pl.off_dB + round256(per_token);
    pl.bytes = pl.off_dC + round256(per_token);
    return pl;
}

int scan_bwd_impl(const ssd_scan_bwd_args *a, cudaStream_t st)
{
    if (!a) return fail(SSD_ERR_NULL, "args is NULL");
    const bool ck = a->h_ckpt != nullptr;
    int rc = check_scan_shape(a->dtype, a->b, a->L, a->H, a->P, a->N, a->G, 64, ck ? a->s : 0);
    if (rc) return rc;
    if (ck && a->s <= 0) return fail(SSD_ERR_SHAPE, "h_ckpt given with checkpoint stride s=%lld", (long long)a->s);
    if (a->b == 0) return ok();
    const size_t state_bytes = sizeof(float) * (size_t)a->b * a->H * a->P * a->N;
    if (!a->dA) return fail(SSD_ERR_NULL, "dA is NULL");
    if (a->L == 0) {
        // no token: dh0 = dh_final, every parameter gradient is zero
        cudaError_t e = cudaMemsetAsync(a->dA, 0, sizeof(float) * a->H, st);
        if (e == cudaSuccess && a->dD) e = cudaMemsetAsync(a->dD, 0, sizeof(float) * a->H, st);
        if (e == cudaSuccess && a->dh0)
            e = a->dh_final ? cudaMemcpyAsync(a->dh0, a->dh_final, state_bytes, cudaMemcpyDeviceToDevice, st)
                            : cudaMemsetAsync(a->dh0, 0, state_bytes, st);
        if (e != cudaSuccess) return fail(SSD_ERR_LAUNCH, "%s", cudaGetErrorString(e));
        return ok();
    }
    if ((rc = check_rows("x", a->x, a->x_batch_stride, a->x_row_stride, (int64_t)a->H * a->P, a->b, a->L, a->dtype, true))) return rc;
    if ((rc = check_rows("B", a->B, a->B_batch_stride, a->B_row_stride, (int64_t)a->G * a->N, a->b, a->L, a->dtype, true))) return rc;
    if ((rc = check_rows("C", a->C, a->C_batch_stride, a->C_row_stride, (int64_t)a->G * a->N, a->b, a->L, a->dtype, true))) return rc;
    if ((rc = check_rows("dy", a->dy, a->dy_batch_stride, a->dy_row_stride, (int64_t)a->H * a->P, a->b, a->L, a->dtype, true))) return rc;
    if (!a->dt || !a->A) return fail(SSD_ERR_NULL, "dt and A must not be NULL");
    if (!a->dx || !a->dB || !a->dC || !a->ddt) return fail(SSD_ERR_NULL, "dx, dB, dC and ddt must not be NULL");
    const void *vec[] = {a->h0, a->h_ckpt, a->dh_final, a->dx, a->dB, a->dC, a->dh0};
    for (const void *v : vec)
        if (v && !aligned16(v)) return fail(SSD_ERR_ALIGN, "states and gradient outputs must be 16-byte aligned");
    const BwdPlan pl = make_bwd_plan(a->b, a->L, a->H, a->P, a->N);
    if (!a->workspace || a->workspace_bytes < pl.bytes)
        return fail(SSD_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", pl.bytes,
                    a->workspace ? a->workspace_bytes : (size_t)0);
    if ((reinterpret_cast<uintptr_t>(a->workspace) & 255u) != 0)
        return fail(SSD_ERR_ALIGN, "workspace must be 256-byte aligned");
    int dev = 0, smem_optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return fail(SSD_ERR_LAUNCH, "no CUDA device available");
    if (ssd::bwd_grad_smem_bytes(a->P, a->N) > (size_t)smem_optin)
        return fail(SSD_ERR_UNSUPPORTED, "backward needs %zu bytes of shared memory, the device has %d",
                    ssd::bwd_grad_smem_bytes(a->P, a->N), smem_optin);
    ssd::BwdParams p{};
    p.b = a->b; p.L = a->L; p.H = a->H; p.P = a->P; p.N = a->N; p.G = a->G;
    p.s = ck ? a->s : 0;
    p.n_ckpt = ck ? a->L / a->s : 0;
    p.nch = pl.nch;
    p.cell_chunks = ck ? a->s / 64 : pl.nch;
    p.x = a->x; p.xbs = a->x_batch_stride; p.xrs = a->x_row_stride;
    p.B = a->B; p.Bbs = a->B_batch_stride; p.Brs = a->B_row_stride;
    p.C = a->C; p.Cbs = a->C_batch_stride; p.Crs = a->C_row_stride;
    p.dy = a->dy; p.dybs = a->dy_batch_stride; p.dyrs = a->dy_row_stride;
    p.dt = a->dt; p.A = a->A; p.D = a->D; p.h0 = a->h0; p.h_ckpt = a->h_ckpt; p.dh_final = a->dh_final;
    p.dx = a->dx; p.dB = a->dB; p.dC = a->dC; p.ddt = a->ddt; p.dA = a->dA; p.dD = a->dD; p.dh0 = a->dh0;
    char *ws = static_cast<char *>(a->workspace);
    p.ws_h = reinterpret_cast<float *>(ws + pl.off_h);
    p.ws_g = reinterpret_cast<float *>(ws + pl.off_g);
    p.ws_lam = reinterpret_cast<float *>(ws + pl.off_lam);
    p.ws_pA = reinterpret_cast<float *>(ws + pl.off_pA);
    p.ws_pD = reinterpret_cast<float *>(ws + pl.off_pD);
    p.ws_dBh = reinterpret_cast<float *>(ws + pl.off_dB);
    p.ws_dCh = reinterpret_cast<float *>(ws + pl.off_dC);
    if (p.nch > 2147483647LL || (int64_t)p.b * p.H > 65535LL * 65535LL)
        return fail(SSD_ERR_SHAPE, "sequence too long for the backward grid");
    if (a->H > 65535 || a->b > 65535) return fail(SSD_ERR_SHAPE, "H and b must be at most 65535");
    rc = ssd::launch_scan_backward(p, a->dtype, st);
    if (rc) return fail(SSD_ERR_LAUNCH, "backward launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    return ok();
}

int conv_impl(const void *u, int64_t ubs, int64_t urs, const float *w, const float *bias,
              const void *tail_in, void *tail_out, void *v, int64_t vbs, int64_t vrs,
              int b, int64_t L, int C_ch, int dtype, cudaStream_t st)
{
    if (dtype != SSD_F32 && dtype != SSD_BF16) return fail(SSD_ERR_DTYPE, "unknown dtype %d", dtype);
    if (b < 0 || L < 0 || C_ch <= 0) return fail(SSD_ERR_SHAPE, "need b >= 0, L >= 0, C_ch > 0");
    const int vec = (int)(16 / elem_size(dtype));
    if (C_ch % vec != 0) return fail(SSD_ERR_SHAPE, "C_ch=%d must be a multiple of %d", C_ch, vec);
    if (b == 0) return ok();
    int rc;
    if (L > 0) {
        if ((rc = check_rows("u", u, ubs, urs, C_ch, b, L, dtype, true))) return rc;
        if ((rc = check_rows("v", v, vbs, vrs, C_ch, b, L, dtype, true))) return rc;
        if (!w) return fail(SSD_ERR_NULL, "conv weight w is NULL");
        if (!aligned16(w)) return fail(SSD_ERR_ALIGN, "conv weight w must be 16-byte aligned");
    } else if (!u && tail_out) {
        // tail_out from tail_in only; u is never read
    }
    if ((tail_in && !aligned16(tail_in)) || (tail_out && !aligned16(tail_out)))
        return fail(SSD_ERR_ALIGN, "conv tails must be 16-byte aligned");
    ssd::ConvParams p{};
    p.u = u; p.ubs = ubs; p.urs = urs; p.w = w; p.bias = bias; p.tail_in = tail_in;
    p.tail_out = tail_out; p.v = v; p.vbs = vbs; p.vrs = vrs; p.b = b; p.L = L; p.C_ch = C_ch;
    rc = ssd::launch_conv(p, dtype, st);
    if (rc == 2) return fail(SSD_ERR_SHAPE, "conv grid too large");
    if (rc) return fail(SSD_ERR_LAUNCH, "conv launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    return ok();
}

// ---------------------------------------------------------------- kernel timing
const char *const kKernelNames[ssd::kKCount] = {
    "conv1d_silu", "conv_tail", "stripe_state_tc", "stripe_chain", "chunk_output_tc",
    "stripe_state_generic", "chunk_output_generic", "decode_step", "bwd_chunk_summary", "bwd_chains",
    "bwd_chunk_grad", "bwd_reduce", "gated_rmsnorm"};

struct ProfRecord {
    int id;
    cudaEvent_t a, b;
};

struct ProfState {
    bool on = false;
    std::vector<ProfRecord> recs;
    std::vector<cudaEvent_t> pool;
    cudaEvent_t pending = nullptr;
    cudaEvent_t take()
    {
        if (!pool.empty()) {
            cudaEvent_t e = pool.back();
            pool.pop_back();
            return e;
        }
        cudaEvent_t e = nullptr;
        cudaEventCreate(&e);
        return e;
    }
};

thread_local ProfState g_prof;

}  // namespace

namespace ssd {
int set_error(int code, const char *msg) { return fail(code, "%s", msg); }

void prof_begin(cudaStream_t st, int)
{
    if (!g_prof.on) return;
    g_prof.pending = g_prof.take();
    cudaEventRecord(g_prof.pending, st);
}
void prof_end(cudaStream_t st, int id)
{
    if (!g_prof.on || !g_prof.pending) return;
    cudaEvent_t e = g_prof.take();
    cudaEventRecord(e, st);
    g_prof.recs.push_back({id, g_prof.pending, e});
    g_prof.pending = nullptr;
}
}  // namespace ssd

extern "C" {

int ssd_profile_begin(void)
{
    for (auto &r : g_prof.recs) { g_prof.pool.push_back(r.a); g_prof.pool.push_back(r.b); }
    g_prof.recs.clear();
    g_prof.on = true;
    return ok();
}

int ssd_profile_end(ssd_kernel_stat *out, int capacity, int *count)
{
    g_prof.on = false;
    int64_t launches[ssd::kKCount] = {0};
    double ms[ssd::kKCount] = {0};
    for (auto &r : g_prof.recs) {
        float t = 0.0f;
        cudaError_t e = cudaEventSynchronize(r.b);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
        if (e != cudaSuccess) return fail(SSD_ERR_LAUNCH, "profiling events: %s", cudaGetErrorString(e));
        launches[r.id] += 1;
        ms[r.id] += t;
    }
    int n = 0;
    for (int i = 0; i < ssd::kKCount; ++i) {
        if (!launches[i]) continue;
        if (out && n < capacity) out[n] = ssd_kernel_stat{kKernelNames[i], launches[i], ms[i]};
        ++n;
    }
    if (count) *count = n;
    for (auto &r : g_prof.recs) { g_prof.pool.push_back(r.a); g_prof.pool.push_back(r.b); }
    g_prof.recs.clear();
    return ok();
}


int ssd_conv_forward(const void *u, int64_t u_batch_stride, int64_t u_row_stride,
                     const float *w, const float *bias, const void *tail_in, void *tail_out,
                     void *v, int64_t v_batch_stride, int64_t v_row_stride,
                     int b, int64_t L, int C_ch, int dtype, ssd_stream_t stream)
{
    return conv_impl(u, u_batch_stride, u_row_stride, w, bias, tail_in, tail_out, v,
                     v_batch_stride, v_row_stride, b, L, C_ch, dtype, (cudaStream_t)stream);
}

int ssd_scan_forward(const ssd_scan_args *args, ssd_stream_t stream)
{
    return scan_impl(args, (cudaStream_t)stream);
}

size_t ssd_scan_workspace_size(int b, int64_t L, int H, int P, int N, int Q)
{
    return make_plan(b, L, H, P, N, Q).bytes_dt;
}

int ssd_stream_forward(const ssd_stream_args *a, ssd_stream_t stream)
{
    if (!a) return fail(SSD_ERR_NULL, "args is NULL");
    int rc = check_scan_shape(a->dtype, a->b, a->L, a->H, a->P, a->N, a->G, a->Q, a->s);
    if (rc) return rc;
    const int d_inner = a->H * a->P;
    const int C_ch = d_inner + 2 * a->G * a->N;
    if (a->L > 0 && !a->v) return fail(SSD_ERR_NULL, "v is NULL");
    rc = conv_impl(a->u, a->u_batch_stride, a->u_row_stride, a->conv_w, a->conv_bias, a->tail_in,
                   a->tail_out, a->v, a->v_batch_stride, a->v_row_stride, a->b, a->L, C_ch,
                   a->dtype, (cudaStream_t)stream);
    if (rc) return rc;
    const size_t es = elem_size(a->dtype);
    const char *v = static_cast<const char *>(a->v);
    ssd_scan_args s{};
    s.dtype = a->dtype; s.b = a->b; s.L = a->L; s.H = a->H; s.P = a->P; s.N = a->N; s.G = a->G;
    s.Q = a->Q; s.s = a->s;
    s.x = v; s.x_batch_stride = a->v_batch_stride; s.x_row_stride = a->v_row_stride;
    s.B = v ? v + es * d_inner : nullptr;
    s.B_batch_stride = a->v_batch_stride; s.B_row_stride = a->v_row_stride;
    s.C = v ? v + es * (d_inner + (size_t)a->G * a->N) : nullptr;
    s.C_batch_stride = a->v_batch_stride; s.C_row_stride = a->v_row_stride;
    s.dt = a->dt; s.A = a->A; s.D = a->D; s.h0 = a->h0;
    s.dt_bias = a->dt_bias; s.dt_softplus = a->dt_softplus; s.dt_min = a->dt_min; s.dt_max = a->dt_max;
    s.y = a->y; s.y_batch_stride = a->y_batch_stride; s.y_row_stride = a->y_row_stride;
    s.h_final = a->h_final; s.h_ckpt = a->h_ckpt;
    s.workspace = a->workspace; s.workspace_bytes = a->workspace_bytes;
    return scan_impl(&s, (cudaStream_t)stream);
}

int ssd_scan_backward(const ssd_scan_bwd_args *args, ssd_stream_t stream)
{
    return scan_bwd_impl(args, (cudaStream_t)stream);
}

size_t ssd_scan_backward_workspace_size(int b, int64_t L, int H, int P, int N)
{
    return make_bwd_plan(b, L, H, P, N).bytes;
}

int ssd_gated_rmsnorm_forward(const void *y, int64_t y_row_stride, const void *z, int64_t z_row_stride,
                              const float *weight, float eps, int group_size, void *out, int64_t out_row_stride,
                              int64_t rows, int d, int dtype, ssd_stream_t stream)
{
    if (dtype != SSD_F32 && dtype != SSD_BF16) return fail(SSD_ERR_DTYPE, "unknown dtype %d", dtype);
    if (rows < 0) return fail(SSD_ERR_SHAPE, "negative rows (%lld)", (long long)rows);
    if (d <= 0 || d % 8 != 0 || d > 8192)
        return fail(SSD_ERR_SHAPE, "d=%d must be a positive multiple of 8, at most 8192", d);
    const int group = group_size == 0 ? d : group_size;
    if (group <= 0 || group % 8 != 0 || d % group != 0)
        return fail(SSD_ERR_SHAPE, "group_size=%d must be a multiple of 8 that divides d=%d", group_size, d);
    if (!(eps >= 0.0f)) return fail(SSD_ERR_SHAPE, "eps must be >= 0");
    if (rows == 0) return ok();
    if (!y || !z || !weight || !out) return fail(SSD_ERR_NULL, "y, z, weight and out must not be NULL");
    if (y_row_stride < d || z_row_stride < d || out_row_stride < d)
        return fail(SSD_ERR_STRIDE, "row strides must be at least d");
    const size_t es = elem_size(dtype);
    if (!aligned16(y) || !aligned16(z) || !aligned16(out) || !aligned16(weight) || (y_row_stride * es) % 16 != 0 ||
        (z_row_stride * es) % 16 != 0 || (out_row_stride * es) % 16 != 0)
        return fail(SSD_ERR_ALIGN, "y, z, out, weight and the row strides must be 16-byte aligned");
    ssd::NormParams p{};
    p.y = y; p.yrs = y_row_stride; p.z = z; p.zrs = z_row_stride; p.w = weight; p.eps = eps; p.group = group;
    p.out = out; p.ors = out_row_stride; p.rows = rows; p.d = d;
    if (ssd::launch_gated_norm(p, dtype, (cudaStream_t)stream))
        return fail(SSD_ERR_LAUNCH, "norm launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    return ok();
}

int ssd_decode_step(const ssd_decode_args *a, ssd_stream_t stream)
{
    if (!a) return fail(SSD_ERR_NULL, "args is NULL");
    if (a->dtype != SSD_F32 && a->dtype != SSD_BF16) return fail(SSD_ERR_DTYPE, "unknown dtype %d", a->dtype);
    if (a->b < 0) return fail(SSD_ERR_SHAPE, "negative b (%d)", a->b);
    if (a->H <= 0 || a->G <= 0 || a->H % a->G != 0)
        return fail(SSD_ERR_SHAPE, "need H > 0, G > 0 and H %% G == 0 (H=%d, G=%d)", a->H, a->G);
    if (!pow2_dim(a->P) || !pow2_dim(a->N))
        return fail(SSD_ERR_SHAPE, "P and N must be 16, 32, 64 or 128 (P=%d, N=%d)", a->P, a->N);
    if (a->b == 0) return ok();
    const int64_t C_ch = (int64_t)a->H * a->P + 2LL * a->G * a->N;
    const size_t es = elem_size(a->dtype);
    if (!a->u || !a->conv_w || !a->dt || !a->A || !a->h_out || !a->y)
        return fail(SSD_ERR_NULL, "u, conv_w, dt, A, h_out and y must not be NULL");
    if (a->u_batch_stride < C_ch || (a->b > 1 && a->y_batch_stride < (int64_t)a->H * a->P) || a->y_batch_stride < 0)
        return fail(SSD_ERR_STRIDE, "batch strides smaller than a row");
    if (!aligned16(a->u) || (a->u_batch_stride * es) % 16 != 0 || !aligned16(a->conv_w) ||
        (a->tail_in && !aligned16(a->tail_in)) || (a->tail_out && !aligned16(a->tail_out)) ||
        (a->h_in && !aligned16(a->h_in)) || !aligned16(a->h_out))
        return fail(SSD_ERR_ALIGN, "u rows, conv_w, tails and states must be 16-byte aligned");
    ssd::DecodeParams p{};
    p.b = a->b; p.H = a->H; p.P = a->P; p.N = a->N; p.G = a->G;
    p.u = a->u; p.ubs = a->u_batch_stride; p.w = a->conv_w; p.bias = a->conv_bias;
    p.tail_in = a->tail_in; p.tail_out = a->tail_out; p.dt = a->dt; p.A = a->A; p.D = a->D;
    p.h_in = a->h_in; p.h_out = a->h_out; p.y = a->y; p.ybs = a->y_batch_stride;
    p.dt_bias = a->dt_bias; p.dt_softplus = a->dt_softplus; p.dt_min = a->dt_min; p.dt_max = a->dt_max;
    const int rc = ssd::launch_decode(p, a->dtype, (cudaStream_t)stream);
    if (rc) return fail(SSD_ERR_LAUNCH, "decode launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    return ok();
}

int ssd_sync_status(ssd_stream_t stream)
{
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return fail(SSD_ERR_LAUNCH, "CUDA error: %s", cudaGetErrorString(e));
    unsigned int *sp = status_ptr();
    if (!sp) return fail(SSD_ERR_LAUNCH, "no CUDA device available");
    unsigned int v = 0;
    e = cudaMemcpy(&v, sp, sizeof v, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(SSD_ERR_LAUNCH, "CUDA error: %s", cudaGetErrorString(e));
    if (v != 0) {
        const unsigned int zero = 0;
        cudaMemcpy(sp, &zero, sizeof zero, cudaMemcpyHostToDevice);
        return fail((int)v, "device status %u (a bounded wait gave up)", v);
    }
    return ok();
}

const char *ssd_last_error_string(void) { return g_last_error.c_str(); }

int ssd_version(void) { return 200; }   // 0.2.0: backward, its workspace size, gated norm

}  // extern "C"

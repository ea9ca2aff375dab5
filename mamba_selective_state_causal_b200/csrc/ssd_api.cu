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

// The conv of x fused into the tensor-core scan (ssd_stream_forward without v): x is read
// from u's x columns and turned into silu(conv(u)) inside the scan kernels.
struct FusedConv {
    const void *u;
    int64_t ubs, urs;
    const float *w, *bias;
    const void *tail;
    int C_ch;
    void *v;                 // where pass A writes the conv output of x
    int64_t vbs, vrs;
};

int scan_impl(const ssd_scan_args *a, cudaStream_t st, const FusedConv *fc = nullptr)
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
    if (fc) {
        p.conv_u = fc->u; p.conv_ubs = fc->ubs; p.conv_urs = fc->urs;
        p.conv_w = fc->w; p.conv_bias = fc->bias; p.conv_tail = fc->tail; p.conv_cch = fc->C_ch;
        p.conv_v = fc->v; p.conv_vbs = fc->vbs; p.conv_vrs = fc->vrs;
    }
    const EnvHooks &hooks = env_hooks();
    p.wait_limit_ns = hooks.wait_limit_ns;
    static std::atomic<bool> drop_used{false};
    p.test_drop_unit = (hooks.test_drop_unit >= 0 && !drop_used.exchange(true)) ? hooks.test_drop_unit : -1;
    // SSD_SCAN_PATH=generic forces the CUDA-core kernels (used to cross-check the paths)
    const bool force_generic = hooks.force_generic;
    rc = 6;
    if (!force_generic && ssd::tc_scan_supported(p, a->dtype)) rc = ssd::launch_scan_tc(p, st);
    if (fc && rc == 6) return fail(SSD_ERR_UNSUPPORTED, "the fused conv needs the tensor-core scan");
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
    p.status = status_ptr();
    if (!p.status) return fail(SSD_ERR_LAUNCH, "no CUDA device available");
    p.wait_limit_ns = env_hooks().wait_limit_ns;
    if (p.nch > 2147483647LL || (int64_t)p.b * p.H > 65535LL * 65535LL)
        return fail(SSD_ERR_SHAPE, "sequence too long for the backward grid");
    if (a->H > 65535 || a->b > 65535) return fail(SSD_ERR_SHAPE, "H and b must be at most 65535");
    rc = ssd::launch_scan_backward(p, a->dtype, st);
    if (rc) return fail(SSD_ERR_LAUNCH, "backward launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    return ok();
}

// Layer backward workspace: the rebuilt conv output v [b][L][C_ch] (I/O dtype); dx [b][L][H*P],
// dB, dC [b][L][G*N] fp32; the conv weight partial sums [b*blocks][C_ch][4] and [b*blocks][C_ch]
// fp32; then the scan backward's workspace.
struct LayerBwdPlan {
    size_t off_v = 0, off_dx = 0, off_dB = 0, off_dC = 0, off_pw = 0, off_pb = 0, off_scan = 0, bytes = 0;
};

LayerBwdPlan make_layer_bwd_plan(int b, int64_t L, int H, int P, int N, int G, int dtype)
{
    LayerBwdPlan pl;
    if (b <= 0 || L <= 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0) return pl;
    const size_t cch = (size_t)H * P + 2 * (size_t)G * N;
    const size_t rows = (size_t)b * L;
    const size_t parts = (size_t)b * ssd::conv_bwd_blocks(L);
    pl.off_v = 0;
    pl.off_dx = round256(rows * cch * elem_size(dtype));
    pl.off_dB = pl.off_dx + round256(sizeof(float) * rows * H * P);
    pl.off_dC = pl.off_dB + round256(sizeof(float) * rows * G * N);
    pl.off_pw = pl.off_dC + round256(sizeof(float) * rows * G * N);
    pl.off_pb = pl.off_pw + round256(sizeof(float) * parts * cch * 4);
    pl.off_scan = pl.off_pb + round256(sizeof(float) * parts * cch);
    pl.bytes = pl.off_scan + make_bwd_plan(b, L, H, P, N).bytes;
    return pl;
}

int layer_bwd_impl(const ssd_layer_bwd_args *a, cudaStream_t st)
{
    if (!a) return fail(SSD_ERR_NULL, "args is NULL");
    const bool ck = a->h_ckpt != nullptr || a->conv_ckpt != nullptr;
    if ((a->h_ckpt == nullptr) != (a->conv_ckpt == nullptr))
        return fail(SSD_ERR_NULL, "h_ckpt and conv_ckpt must be given together");
    int rc = check_scan_shape(a->dtype, a->b, a->L, a->H, a->P, a->N, a->G, 64, ck ? a->s : 0);
    if (rc) return rc;
    if (ck && a->s <= 0) return fail(SSD_ERR_SHAPE, "checkpoints given with stride s=%lld", (long long)a->s);
    if (a->b == 0) return ok();
    const int HP = a->H * a->P, GN = a->G * a->N;
    const int C_ch = HP + 2 * GN;
    if (!a->dconv_w || !a->dA || (a->L > 0 && (!a->du || !a->ddt)))
        return fail(SSD_ERR_NULL, "du, dconv_w, ddt and dA must not be NULL");
    if (!a->conv_w || !aligned16(a->conv_w) || !aligned16(a->dconv_w))
        return fail(SSD_ERR_ALIGN, "conv_w and dconv_w must be given, 16-byte aligned");
    const void *vec[] = {a->tail_in, a->conv_ckpt, a->du, a->dtail_in, a->h0, a->h_ckpt, a->dh_final, a->dh0};
    for (const void *v : vec)
        if (v && !aligned16(v)) return fail(SSD_ERR_ALIGN, "buffers must be 16-byte aligned");
    if (a->L == 0) {
        // no token: tail_out is tail_in, every other gradient is zero or passes through
        const size_t tail_bytes = sizeof(float) * (size_t)a->b * 3 * C_ch;
        const size_t state_bytes = sizeof(float) * (size_t)a->b * a->H * a->P * a->N;
        cudaError_t e = cudaMemsetAsync(a->dconv_w, 0, sizeof(float) * 4 * C_ch, st);
        if (e == cudaSuccess && a->dconv_bias) e = cudaMemsetAsync(a->dconv_bias, 0, sizeof(float) * C_ch, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(a->dA, 0, sizeof(float) * a->H, st);
        if (e == cudaSuccess && a->dD) e = cudaMemsetAsync(a->dD, 0, sizeof(float) * a->H, st);
        if (e == cudaSuccess && a->dtail_in)
            e = a->dtail_out ? cudaMemcpyAsync(a->dtail_in, a->dtail_out, tail_bytes, cudaMemcpyDeviceToDevice, st)
                             : cudaMemsetAsync(a->dtail_in, 0, tail_bytes, st);
        if (e == cudaSuccess && a->dh0)
            e = a->dh_final ? cudaMemcpyAsync(a->dh0, a->dh_final, state_bytes, cudaMemcpyDeviceToDevice, st)
                            : cudaMemsetAsync(a->dh0, 0, state_bytes, st);
        if (e != cudaSuccess) return fail(SSD_ERR_LAUNCH, "%s", cudaGetErrorString(e));
        return ok();
    }
    if ((rc = check_rows("u", a->u, a->u_batch_stride, a->u_row_stride, C_ch, a->b, a->L, a->dtype, true))) return rc;
    const LayerBwdPlan pl = make_layer_bwd_plan(a->b, a->L, a->H, a->P, a->N, a->G, a->dtype);
    if (!a->workspace || a->workspace_bytes < pl.bytes)
        return fail(SSD_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", pl.bytes,
                    a->workspace ? a->workspace_bytes : (size_t)0);
    if ((reinterpret_cast<uintptr_t>(a->workspace) & 255u) != 0)
        return fail(SSD_ERR_ALIGN, "workspace must be 256-byte aligned");
    char *ws = static_cast<char *>(a->workspace);
    ssd::ConvBwdParams cp{};
    cp.b = a->b; cp.L = a->L; cp.C_ch = C_ch; cp.HP = HP; cp.GN = GN;
    cp.u = a->u; cp.ubs = a->u_batch_stride; cp.urs = a->u_row_stride;
    cp.w = a->conv_w; cp.bias = a->conv_bias; cp.tail_in = a->tail_in;
    cp.conv_ckpt = ck ? a->conv_ckpt : nullptr;
    cp.s = ck ? a->s : 0;
    cp.n_ckpt = ck ? a->L / a->s : 0;
    cp.v = ws + pl.off_v;
    cp.dx = reinterpret_cast<float *>(ws + pl.off_dx);
    cp.dB = reinterpret_cast<float *>(ws + pl.off_dB);
    cp.dC = reinterpret_cast<float *>(ws + pl.off_dC);
    cp.dtail_out = a->dtail_out;
    cp.du = a->du; cp.dtail_in = a->dtail_in;
    cp.ws_dw = reinterpret_cast<float *>(ws + pl.off_pw);
    cp.ws_dbias = reinterpret_cast<float *>(ws + pl.off_pb);
    cp.dw = a->dconv_w; cp.dbias = a->dconv_bias;
    // 1. every cell's conv output from its own rows of u and its conv buffer
    rc = ssd::launch_conv_cells(cp, a->dtype, st);
    if (rc == 2) return fail(SSD_ERR_SHAPE, "layer backward grid too large");
    if (rc) return fail(SSD_ERR_LAUNCH, "conv recompute launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    // 2. the scan's reverse mode on that output's x, B and C, each cell from its state checkpoint
    ssd_scan_bwd_args sb{};
    sb.dtype = a->dtype; sb.b = a->b; sb.L = a->L; sb.H = a->H; sb.P = a->P; sb.N = a->N; sb.G = a->G;
    sb.s = ck ? a->s : 0;
    const size_t es = elem_size(a->dtype);
    const char *v = static_cast<const char *>(cp.v);
    sb.x = v; sb.x_batch_stride = a->L * C_ch; sb.x_row_stride = C_ch;
    sb.B = v + es * HP; sb.B_batch_stride = a->L * C_ch; sb.B_row_stride = C_ch;
    sb.C = v + es * (HP + GN); sb.C_batch_stride = a->L * C_ch; sb.C_row_stride = C_ch;
    sb.dt = a->dt; sb.A = a->A; sb.D = a->D; sb.h0 = a->h0; sb.h_ckpt = ck ? a->h_ckpt : nullptr;
    sb.dy = a->dy; sb.dy_batch_stride = a->dy_batch_stride; sb.dy_row_stride = a->dy_row_stride;
    sb.dh_final = a->dh_final;
    sb.dx = const_cast<float *>(cp.dx); sb.dB = const_cast<float *>(cp.dB); sb.dC = const_cast<float *>(cp.dC);
    sb.ddt = a->ddt; sb.dA = a->dA; sb.dD = a->dD; sb.dh0 = a->dh0;
    sb.workspace = ws + pl.off_scan; sb.workspace_bytes = pl.bytes - pl.off_scan;
    rc = scan_bwd_impl(&sb, st);
    if (rc) return rc;
    // 3. the conv's reverse mode
    rc = ssd::launch_conv_backward(cp, a->dtype, st);
    if (rc == 2) return fail(SSD_ERR_SHAPE, "layer backward grid too large");
    if (rc) return fail(SSD_ERR_LAUNCH, "conv backward launch failed: %s", cudaGetErrorString(cudaGetLastError()));
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
    p.tail_rs = C_ch;
    rc = ssd::launch_conv(p, dtype, st);
    if (rc == 2) return fail(SSD_ERR_SHAPE, "conv grid too large");
    if (rc) return fail(SSD_ERR_LAUNCH, "conv launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    return ok();
}

// ---------------------------------------------------------------- kernel timing
const char *const kKernelNames[ssd::kKCount] = {
    "conv1d_silu", "conv_tail", "stripe_state_tc", "stripe_chain", "chunk_output_tc",
    "stripe_state_generic", "chunk_output_generic", "decode_step", "bwd_chunk_summary", "bwd_state_chain",
    "bwd_chunk_grad", "bwd_reduce", "gated_rmsnorm", "conv_cells", "conv_ckpt", "conv_bwd", "bwd_adjoint_chain"};

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

namespace {

// Workspace of ssd_stream_forward without v: the scan's workspace, then the conv output
// v [b][L][C_ch] that the output pass reads.
struct StreamPlan {
    size_t off_v = 0, bytes = 0;
};

StreamPlan make_stream_plan(int b, int64_t L, int H, int P, int N, int G, int Q, int dtype)
{
    StreamPlan sp;
    const Plan pl = make_plan(b, L, H, P, N, Q);
    sp.off_v = round256(pl.bytes_dt);
    sp.bytes = sp.off_v + round256((size_t)b * L * ((size_t)H * P + 2 * (size_t)G * N) * elem_size(dtype));
    return sp;
}

// One streamed segment, L > 0 and b > 0.  On the tensor-core shapes with more than one
// stripe the conv of x runs inside pass A (which writes x = v[:, :H*P]) and a conv kernel
// covers only the B and C channels; otherwise one conv kernel covers every channel.
int stream_impl(const ssd_stream_args *a, cudaStream_t st)
{
    const int HP = a->H * a->P, GN = a->G * a->N;
    const int C_ch = HP + 2 * GN;
    const size_t es = elem_size(a->dtype);
    int rc = check_rows("u", a->u, a->u_batch_stride, a->u_row_stride, C_ch, a->b, a->L, a->dtype, true);
    if (rc) return rc;
    if (!a->conv_w) return fail(SSD_ERR_NULL, "conv weight w is NULL");
    if (!aligned16(a->conv_w)) return fail(SSD_ERR_ALIGN, "conv weight w must be 16-byte aligned");
    if ((a->tail_in && !aligned16(a->tail_in)) || (a->tail_out && !aligned16(a->tail_out)) ||
        (a->conv_ckpt && !aligned16(a->conv_ckpt)))
        return fail(SSD_ERR_ALIGN, "conv tails and conv_ckpt must be 16-byte aligned");
    char *v;
    int64_t vbs, vrs;
    size_t scan_ws_bytes = a->workspace_bytes;
    if (a->v) {
        if ((rc = check_rows("v", a->v, a->v_batch_stride, a->v_row_stride, C_ch, a->b, a->L, a->dtype, true)))
            return rc;
        v = static_cast<char *>(a->v); vbs = a->v_batch_stride; vrs = a->v_row_stride;
    } else {
        const StreamPlan sp = make_stream_plan(a->b, a->L, a->H, a->P, a->N, a->G, a->Q, a->dtype);
        if (!a->workspace || a->workspace_bytes < sp.bytes)
            return fail(SSD_ERR_WORKSPACE, "workspace of %zu bytes needed (ssd_stream_workspace_size), %zu given",
                        sp.bytes, a->workspace ? a->workspace_bytes : (size_t)0);
        if ((reinterpret_cast<uintptr_t>(a->workspace) & 255u) != 0)
            return fail(SSD_ERR_ALIGN, "workspace must be 256-byte aligned");
        v = static_cast<char *>(a->workspace) + sp.off_v; vbs = a->L * C_ch; vrs = C_ch;
        scan_ws_bytes = sp.off_v;
    }
    const Plan pl = make_plan(a->b, a->L, a->H, a->P, a->N, a->Q);
    const bool fuse = ssd::tc_scan_shape(a->dtype, a->H, a->P, a->N, a->G, a->Q) && pl.ns > 1 &&
                      !env_hooks().force_generic && (reinterpret_cast<uintptr_t>(a->dt) & 7u) == 0 &&
                      a->L < (1LL << 31) && (int64_t)a->b * pl.ns * a->H < (1LL << 31);
    ssd::ConvParams cp{};
    cp.ubs = a->u_batch_stride; cp.urs = a->u_row_stride; cp.tail_rs = C_ch;
    cp.vbs = vbs; cp.vrs = vrs; cp.b = a->b; cp.L = a->L;
    if (fuse) {
        // the B and C channels' conv into v[:, H*P:] (their rows before token 0 from tail_in's B/C columns)
        cp.u = static_cast<const char *>(a->u) + es * HP;
        cp.w = a->conv_w + 4 * HP; cp.bias = a->conv_bias ? a->conv_bias + HP : nullptr;
        cp.tail_in = a->tail_in ? static_cast<const char *>(a->tail_in) + es * HP : nullptr;
        cp.v = v + es * HP; cp.C_ch = 2 * GN;
    } else {
        cp.u = a->u; cp.w = a->conv_w; cp.bias = a->conv_bias; cp.tail_in = a->tail_in;
        cp.v = v; cp.C_ch = C_ch;
    }
    rc = ssd::launch_conv(cp, a->dtype, st);
    if (rc == 2) return fail(SSD_ERR_SHAPE, "conv grid too large");
    if (rc) return fail(SSD_ERR_LAUNCH, "conv launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    ssd_scan_args s{};
    s.dtype = a->dtype; s.b = a->b; s.L = a->L; s.H = a->H; s.P = a->P; s.N = a->N; s.G = a->G;
    s.Q = a->Q; s.s = a->s;
    s.x = v; s.x_batch_stride = vbs; s.x_row_stride = vrs;
    s.B = v + es * HP; s.B_batch_stride = vbs; s.B_row_stride = vrs;
    s.C = v + es * (HP + GN); s.C_batch_stride = vbs; s.C_row_stride = vrs;
    s.dt = a->dt; s.A = a->A; s.D = a->D; s.h0 = a->h0;
    s.dt_bias = a->dt_bias; s.dt_softplus = a->dt_softplus; s.dt_min = a->dt_min; s.dt_max = a->dt_max;
    s.y = a->y; s.y_batch_stride = a->y_batch_stride; s.y_row_stride = a->y_row_stride;
    s.h_final = a->h_final; s.h_ckpt = a->h_ckpt;
    s.workspace = a->workspace; s.workspace_bytes = scan_ws_bytes;
    FusedConv fc{a->u, a->u_batch_stride, a->u_row_stride, a->conv_w, a->conv_bias, a->tail_in, C_ch, v, vbs, vrs};
    rc = scan_impl(&s, st, fuse ? &fc : nullptr);
    if (rc) return rc;
    // the conv buffers: at every checkpoint, and tail_out (last: it may alias tail_in)
    if (a->conv_ckpt && a->s > 0 && a->L >= a->s) {
        if (ssd::launch_conv_ckpt(a->u, a->u_batch_stride, a->u_row_stride, a->conv_ckpt, a->b, a->L, C_ch, a->s,
                                  a->dtype, st))
            return fail(SSD_ERR_LAUNCH, "conv checkpoint launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    }
    if (a->tail_out) {
        ssd::ConvParams tp{};
        tp.u = a->u; tp.ubs = a->u_batch_stride; tp.urs = a->u_row_stride; tp.tail_in = a->tail_in;
        tp.tail_out = a->tail_out; tp.b = a->b; tp.L = a->L; tp.C_ch = C_ch; tp.tail_rs = C_ch;
        if (ssd::launch_conv_tail(tp, a->dtype, st))
            return fail(SSD_ERR_LAUNCH, "conv tail launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    }
    return ok();
}

}  // namespace

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

size_t ssd_stream_workspace_size(int b, int64_t L, int H, int P, int N, int G, int Q, int dtype)
{
    if (b <= 0 || L <= 0 || H <= 0 || G <= 0) return 0;
    return make_stream_plan(b, L, H, P, N, G, Q, dtype).bytes;
}

int ssd_stream_forward(const ssd_stream_args *a, ssd_stream_t stream)
{
    if (!a) return fail(SSD_ERR_NULL, "args is NULL");
    int rc = check_scan_shape(a->dtype, a->b, a->L, a->H, a->P, a->N, a->G, a->Q, a->s);
    if (rc) return rc;
    if (a->L > 0 && a->b > 0) return stream_impl(a, (cudaStream_t)stream);
    // no token (or no batch row): tail_out from tail_in, h_final from h0
    const int d_inner = a->H * a->P;
    const int C_ch = d_inner + 2 * a->G * a->N;
    if (a->conv_ckpt && a->s > 0 && a->L >= a->s) {
        if (!aligned16(a->conv_ckpt)) return fail(SSD_ERR_ALIGN, "conv_ckpt must be 16-byte aligned");
        if (!a->u) return fail(SSD_ERR_NULL, "u is NULL");
    }
    rc = conv_impl(a->u, a->u_batch_stride, a->u_row_stride, a->conv_w, a->conv_bias, a->tail_in,
                   a->tail_out, a->v, a->v_batch_stride, a->v_row_stride, a->b, a->L, C_ch,
                   a->dtype, (cudaStream_t)stream);
    if (rc) return rc;
    if (a->conv_ckpt && a->s > 0 && a->L >= a->s && a->b > 0) {
        // the conv buffer at every checkpoint: the 3 rows of u before it
        if (ssd::launch_conv_ckpt(a->u, a->u_batch_stride, a->u_row_stride, a->conv_ckpt, a->b, a->L, C_ch, a->s,
                                  a->dtype, (cudaStream_t)stream))
            return fail(SSD_ERR_LAUNCH, "conv checkpoint launch failed: %s", cudaGetErrorString(cudaGetLastError()));
    }
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

size_t ssd_layer_backward_workspace_size(int b, int64_t L, int H, int P, int N, int G, int dtype)
{
    return make_layer_bwd_plan(b, L, H, P, N, G, dtype).bytes;
}

int ssd_layer_backward(const ssd_layer_bwd_args *a, ssd_stream_t stream)
{
    return layer_bwd_impl(a, (cudaStream_t)stream);
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

int ssd_version(void) { return 300; }   // 0.3.0: layer backward, conv buffers at the checkpoints

}  // extern "C"

// hm_api.cu -- the extern "C" entry points of libhm.so (declared in include/hm.h).
//
// Host side only: argument validation (before anything is enqueued),
// workspace carving, and the sequence of kernel launches for each call.
// Every arithmetic step runs in this library's CUDA kernels.
#include <cstdio>
#include <cstdarg>
#include <cstring>
#include <atomic>
#include <mutex>

#include <algorithm>

#include "tc_common.cuh"

namespace hm {

__device__ unsigned int g_hm_err[4];

unsigned int *device_error_word() {
    static std::mutex mu;
    static unsigned int *addr[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> g(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_hm_err) != cudaSuccess) return nullptr;
        addr[dev] = (unsigned int *)p;
    }
    return addr[dev];
}

static std::atomic<unsigned long long> g_launches{0};
void count_launches(unsigned int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

namespace {

thread_local char g_detail[512] = {0};

hm_status fail(hm_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
    va_end(ap);
    return s;
}

}  // namespace

void set_error_detail(const char *msg) { snprintf(g_detail, sizeof(g_detail), "%s", msg ? msg : ""); }

namespace {

hm_status cuda_fail(cudaError_t e, const char *what) {
    return fail(HM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

size_t dsize(hm_dtype t) { return t == HM_BF16 ? 2 : 4; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool valid_dtype(hm_dtype t) { return t == HM_F32 || t == HM_BF16; }

// ------------------------------------------------------------------ featmap

hm_status check_featmap(const void *x, hm_dtype xt, int64_t rows, int H, int d, int p,
                        const void *W, const void *phi, hm_dtype pt) {
    if (!valid_dtype(xt) || !valid_dtype(pt)) return fail(HM_ERR_INVALID_ARG, "featmap: bad dtype");
    if (rows < 0 || H < 1) return fail(HM_ERR_INVALID_ARG, "featmap: rows < 0 or H < 1");
    if (d < 1 || d > 512 || p < 1 || p > 256)
        return fail(HM_ERR_UNSUPPORTED, "featmap: need 1 <= d <= 512 and 1 <= p <= 256 (d=%d p=%d)", d, p);
    if (rows > 0 && (!x || !W || !phi)) return fail(HM_ERR_INVALID_ARG, "featmap: null pointer");
    if (!aligned16(x) || !aligned16(W) || !aligned16(phi))
        return fail(HM_ERR_INVALID_ARG, "featmap: pointers must be 16-byte aligned");
    return HM_OK;
}

cudaError_t run_featmap(const void *x, hm_dtype xt, int64_t rows, int H, int d, int p,
                        const void *W, int64_t wstride, const float *bias, void *phi, hm_dtype pt,
                        cudaStream_t s, void *phi_lo = nullptr) {
    if (xt == HM_BF16 && featmap_tc_supported(rows, H, d, p, wstride))
        return launch_featmap_tc(x, rows, H, d, p, W, wstride, bias, phi, pt,
                                 DevErr{device_error_word()}, s, phi_lo);
    return launch_featmap_simt(x, xt, rows, H, d, p, W, wstride, bias, phi, pt, s, phi_lo);
}

// phi(q) and phi(k): one tensor-core launch when the shape has a kernel.
cudaError_t run_featmap_qk(const void *q, const void *k, hm_dtype xt, int64_t rows, int H, int d, int p,
                           const void *W_q, const void *W_k, int64_t wstride, const float *b_q,
                           const float *b_k, void *phq, void *phk, hm_dtype pt, cudaStream_t s,
                           void *phk_lo = nullptr) {
    if (xt == HM_BF16 && featmap_tc_supported(rows, H, d, p, wstride))
        return launch_featmap_tc2(q, W_q, b_q, phq, nullptr, k, W_k, b_k, phk, phk_lo, rows, H, d, p, wstride, pt,
                                  DevErr{device_error_word()}, s);
    cudaError_t e = launch_featmap_simt(q, xt, rows, H, d, p, W_q, wstride, b_q, phq, pt, s, nullptr);
    if (e != cudaSuccess) return e;
    return launch_featmap_simt(k, xt, rows, H, d, p, W_k, wstride, b_k, phk, pt, s, phk_lo);
}

}  // namespace

cudaError_t run_featmap_f32(const void *x, hm_dtype xt, int64_t rows, int H, int d, int p, const void *W,
                            float *phi, cudaStream_t s) {
    return run_featmap(x, xt, rows, H, d, p, W, 0, nullptr, phi, HM_F32, s);
}

namespace {

// ------------------------------------------------------------------ backward

hm_status check_scan_bwd(const hm_scan_bwd_args *a, ScanBwdCore *core) {
    if (!a) return fail(HM_ERR_INVALID_ARG, "scan_bwd: null args");
    if (!valid_dtype(a->io_dtype)) return fail(HM_ERR_INVALID_ARG, "scan_bwd: bad io dtype");
    if (a->B < 0 || a->L < 0 || a->H < 1 || a->d < 1 || a->dv < 1)
        return fail(HM_ERR_INVALID_ARG, "scan_bwd: bad sizes");
    if ((a->W_q == nullptr) != (a->W_k == nullptr))
        return fail(HM_ERR_INVALID_ARG, "scan_bwd: W_q and W_k must both be given or both NULL");
    if ((a->S0 == nullptr) != (a->z0 == nullptr))
        return fail(HM_ERR_INVALID_ARG, "scan_bwd: S0 and z0 must both be given or both NULL");
    if ((a->grad_S0 == nullptr) != (a->grad_z0 == nullptr))
        return fail(HM_ERR_INVALID_ARG, "scan_bwd: grad_S0 and grad_z0 must both be given or both NULL");
    if (a->dt && (!a->A_log || !a->grad_dt || !a->grad_A_log))
        return fail(HM_ERR_INVALID_ARG, "scan_bwd: dt needs A_log, grad_dt and grad_A_log");
    const int F = a->W_q ? 2 * a->p : a->d;
    if (a->W_q && (a->p < 1 || a->p > 256)) return fail(HM_ERR_UNSUPPORTED, "scan_bwd: need 1 <= p <= 256");
    if (F > 256) return fail(HM_ERR_UNSUPPORTED, "scan_bwd: feature dim F=%d > 256", F);
    if (a->d > 512) return fail(HM_ERR_UNSUPPORTED, "scan_bwd: d=%d > 512", a->d);
    if (a->B * a->H > 65535) return fail(HM_ERR_UNSUPPORTED, "scan_bwd: B*H > 65535");
    const int64_t rows = a->B * a->L * a->H;
    if (rows > 0 && (!a->q || !a->k || !a->v || !a->dout || !a->grad_q || !a->grad_k || !a->grad_v ||
                     (a->W_q && (!a->grad_W_q || !a->grad_W_k))))
        return fail(HM_ERR_INVALID_ARG, "scan_bwd: null input or gradient pointer");
    const void *ptrs[] = {a->q, a->k, a->v, a->W_q, a->W_k, a->dt, a->A_log, a->S0, a->z0, a->dout, a->grad_q,
                          a->grad_k, a->grad_v, a->grad_W_q, a->grad_W_k, a->grad_dt, a->grad_A_log, a->grad_S0, a->grad_z0};
    for (const void *p : ptrs)
        if (!aligned16(p)) return fail(HM_ERR_INVALID_ARG, "scan_bwd: pointers must be 16-byte aligned");
    ScanBwdCore c{};
    c.B = a->B; c.L = a->L; c.H = a->H; c.d = a->d; c.p = a->p; c.F = F; c.dv = a->dv;
    c.io_dtype = a->io_dtype;
    c.q = a->q; c.k = a->k; c.v = a->v; c.dout = a->dout; c.W_q = a->W_q; c.W_k = a->W_k;
    c.dt = a->dt; c.A_log = a->A_log; c.S0 = a->S0; c.z0 = a->z0;
    c.dq = a->grad_q; c.dk = a->grad_k; c.dv_out = a->grad_v; c.dW_q = a->grad_W_q; c.dW_k = a->grad_W_k;
    c.ddt = a->grad_dt; c.dA_log = a->grad_A_log; c.dS0 = a->grad_S0; c.dz0 = a->grad_z0;
    *core = c;
    return HM_OK;
}

// ------------------------------------------------------------------ scan

struct ScanPlan {
    int F;
    hm_dtype feat;
    size_t phi_bytes;  // one of phq / phk (0 when q, k are features already)
    size_t lo_bytes;   // rounding remainder of phk (tensor-core path with a returned state)
    size_t tc_bytes;   // tensor-core scan scratch
    bool tc;
    size_t total;
};

hm_status check_scan(const hm_scan_args *a, ScanPlan *plan) {
    if (!a) return fail(HM_ERR_INVALID_ARG, "scan: null args");
    if (!valid_dtype(a->io_dtype)) return fail(HM_ERR_INVALID_ARG, "scan: bad io dtype");
    if (a->B < 0 || a->L < 0 || a->H < 1 || a->d < 1 || a->dv < 1)
        return fail(HM_ERR_INVALID_ARG, "scan: bad sizes B=%lld L=%lld H=%d d=%d dv=%d",
                    (long long)a->B, (long long)a->L, a->H, a->d, a->dv);
    if ((a->W_q == nullptr) != (a->W_k == nullptr))
        return fail(HM_ERR_INVALID_ARG, "scan: W_q and W_k must both be given or both NULL");
    if ((a->S0 == nullptr) != (a->z0 == nullptr))
        return fail(HM_ERR_INVALID_ARG, "scan: S0 and z0 must both be given or both NULL");
    if ((a->S_out == nullptr) != (a->z_out == nullptr))
        return fail(HM_ERR_INVALID_ARG, "scan: S_out and z_out must both be given or both NULL");
    if (a->dt && !a->A_log) return fail(HM_ERR_INVALID_ARG, "scan: dt given without A_log");
    if (a->flags & ~(unsigned)(HM_FLAG_DT_SCALED_INPUT | HM_FLAG_PER_FEATURE_DECAY | HM_FLAG_ROPE))
        return fail(HM_ERR_INVALID_ARG, "scan: unknown flag bits 0x%x", a->flags);
    if ((a->flags & (HM_FLAG_DT_SCALED_INPUT | HM_FLAG_PER_FEATURE_DECAY)) && !a->dt)
        return fail(HM_ERR_INVALID_ARG, "scan: the step-scaled input and the per-feature decay need dt");
    const bool rope = (a->flags & HM_FLAG_ROPE) != 0;
    if (rope && (!(a->rope_base > 0.0) || a->pos0 < 0))
        return fail(HM_ERR_INVALID_ARG, "scan: the rotary embedding needs rope_base > 0 and pos0 >= 0");
    const int F = a->W_q ? 2 * a->p : a->d;
    if (rope && F % 2 != 0) return fail(HM_ERR_INVALID_ARG, "scan: the rotary embedding needs an even F");
    if (a->W_q && (a->p < 1 || a->p > 256)) return fail(HM_ERR_UNSUPPORTED, "scan: need 1 <= p <= 256");
    if (F > 256) return fail(HM_ERR_UNSUPPORTED, "scan: feature dim F=%d > 256", F);
    if (a->d > 512) return fail(HM_ERR_UNSUPPORTED, "scan: d=%d > 512", a->d);
    if (a->dv % 4 != 0) return fail(HM_ERR_UNSUPPORTED, "scan: dv must be a multiple of 4");
    if (a->B * a->H > 65535) return fail(HM_ERR_UNSUPPORTED, "scan: B*H > 65535");
    const int64_t rows = a->B * a->L * a->H;
    // o == NULL: a state-only call (the final state, and the log decay, are its results)
    if (!a->o && !a->S_out) return fail(HM_ERR_INVALID_ARG, "scan: o may be NULL only when S_out is given");
    if (rows > 0 && (!a->k || !a->v || (a->o && !a->q)))
        return fail(HM_ERR_INVALID_ARG, "scan: null q/k/v");
    const void *ptrs[] = {a->q, a->k, a->v, a->W_q, a->W_k, a->b_q, a->b_k, a->dt, a->A_log,
                          a->S0, a->z0, a->o, a->S_out, a->z_out, a->log_decay_out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return fail(HM_ERR_INVALID_ARG, "scan: pointers must be 16-byte aligned");
    ScanPlan pl{};
    pl.F = F;
    ScanCore c{};
    c.B = a->B; c.L = a->L; c.H = a->H; c.F = F; c.dv = a->dv;
    c.feat_dtype = a->io_dtype; c.io_dtype = a->io_dtype;
    c.dt_scaled = (a->flags & HM_FLAG_DT_SCALED_INPUT) != 0;
    c.per_feature = (a->flags & HM_FLAG_PER_FEATURE_DECAY) != 0;
    pl.tc = scan_tc_supported(c);
    // Features computed here are kept in fp32 for the CUDA-core path: its state
    // update then adds exact products instead of bf16-rounded ones.  When
    // W_q == NULL the caller's q / k are the features and keep their dtype.
    pl.feat = a->W_q ? (pl.tc ? HM_BF16 : HM_F32) : a->io_dtype;
    c.feat_dtype = pl.feat;
    // rotated caller features (W_q == NULL with the rotary embedding) are
    // written to the workspace too: the caller's q, k are never modified
    pl.phi_bytes = (a->W_q || rope) ? round_up((size_t)rows * F * dsize(pl.feat), 256) : 0;
    pl.lo_bytes = (pl.tc && a->W_q && a->S_out) ? pl.phi_bytes : 0;
    pl.tc_bytes = pl.tc ? round_up(scan_tc_workspace(c), 256) : 0;
    pl.total = 2 * pl.phi_bytes + pl.lo_bytes + pl.tc_bytes;
    *plan = pl;
    return HM_OK;
}

// ------------------------------------------------------------------ decode

hm_status check_decode(const hm_decode_args *a, DecodePlan *plan) {
    if (!a) return fail(HM_ERR_INVALID_ARG, "decode: null args");
    if (!valid_dtype(a->io_dtype)) return fail(HM_ERR_INVALID_ARG, "decode: bad io dtype");
    if (a->B < 0 || a->H < 1 || a->d < 1 || a->dv < 1)
        return fail(HM_ERR_INVALID_ARG, "decode: bad sizes");
    if ((a->W_q == nullptr) != (a->W_k == nullptr))
        return fail(HM_ERR_INVALID_ARG, "decode: W_q and W_k must both be given or both NULL");
    if (a->dt && !a->A_log) return fail(HM_ERR_INVALID_ARG, "decode: dt given without A_log");
    if (a->flags & ~(unsigned)(HM_FLAG_DT_SCALED_INPUT | HM_FLAG_PER_FEATURE_DECAY | HM_FLAG_ROPE))
        return fail(HM_ERR_INVALID_ARG, "decode: unknown flag bits 0x%x", a->flags);
    if ((a->flags & (HM_FLAG_DT_SCALED_INPUT | HM_FLAG_PER_FEATURE_DECAY)) && !a->dt)
        return fail(HM_ERR_INVALID_ARG, "decode: the step-scaled input and the per-feature decay need dt");
    const bool rope = (a->flags & HM_FLAG_ROPE) != 0;
    if (rope && (!(a->rope_base > 0.0) || !a->positions || !aligned16(a->positions)))
        return fail(HM_ERR_INVALID_ARG, "decode: the rotary embedding needs rope_base > 0 and positions");
    const int F = a->W_q ? 2 * a->p : a->d;
    if (rope && F % 2 != 0) return fail(HM_ERR_INVALID_ARG, "decode: the rotary embedding needs an even F");
    if (a->W_q && (a->p < 1 || a->p > 256)) return fail(HM_ERR_UNSUPPORTED, "decode: need 1 <= p <= 256");
    if (F > 256) return fail(HM_ERR_UNSUPPORTED, "decode: feature dim F=%d > 256", F);
    if (a->d > 512) return fail(HM_ERR_UNSUPPORTED, "decode: d=%d > 512", a->d);
    if (a->dv % 4 != 0) return fail(HM_ERR_UNSUPPORTED, "decode: dv must be a multiple of 4");
    if (a->B > 0x7fffffffLL || a->B * a->H > 0x7fffffffLL)
        return fail(HM_ERR_UNSUPPORTED, "decode: B*H too large");
    if (a->B > 0 && (!a->q || !a->k || !a->v || !a->o || !a->S || !a->z))
        return fail(HM_ERR_INVALID_ARG, "decode: null q/k/v/o/S/z");
    const void *ptrs[] = {a->q, a->k, a->v, a->W_q, a->W_k, a->b_q, a->b_k, a->dt, a->A_log,
                          a->S, a->z, a->o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return fail(HM_ERR_INVALID_ARG, "decode: pointers must be 16-byte aligned");
    DecodePlan pl{};
    pl.F = F;
    pl.feat_values = (a->W_q || rope) ? a->B * a->H * F : 0;
    pl.phi_bytes = pl.feat_values ? round_up((size_t)pl.feat_values * sizeof(float), 256) : 0;
    pl.total = 2 * pl.phi_bytes;
    *plan = pl;
    return HM_OK;
}

}  // namespace

hm_status check_decode_args(const hm_decode_args *a, DecodePlan *plan) { return check_decode(a, plan); }

// The decode step after its arguments were checked: per-token feature maps
// into phq_buf / phk_buf (fp32, pl.feat_values each; unused when W_q == NULL),
// then the state update.  Both decode entry points enqueue through here, so
// they produce identical results.  The features are fp32 whatever the io
// dtype: the state adds phi(k) v^T at every step, and a bf16 phi(k) would put
// a 2^-9 relative error on each increment of S.
hm_status decode_enqueue(const hm_decode_args *a, const DecodePlan &pl, void *phq_buf, void *phk_buf,
                         cudaStream_t s) {
    const int64_t rows = a->B * a->H;
    if (rows == 0) return HM_OK;
    const void *phq = a->q, *phk = a->k;
    hm_dtype ft = a->io_dtype;
    cudaError_t e;
    if (a->W_q) {
        e = run_featmap_qk(a->q, a->k, a->io_dtype, rows, a->H, a->d, a->p, a->W_q, a->W_k, a->w_head_stride,
                           a->b_q, a->b_k, phq_buf, phk_buf, HM_F32, s);
        if (e != cudaSuccess) return cuda_fail(e, "decode: feature maps");
        phq = phq_buf;
        phk = phk_buf;
        ft = HM_F32;
    }
    if (a->flags & HM_FLAG_ROPE) {
        // rotary embedding at each sequence's position: in place on the fp32
        // maps above, or from the caller's features into the fp32 planes
        e = launch_rope(phq, nullptr, phq_buf, nullptr, ft, a->B, 1, a->H, pl.F, a->rope_base, 0, a->positions, s);
        if (e == cudaSuccess)
            e = launch_rope(phk, nullptr, phk_buf, nullptr, ft, a->B, 1, a->H, pl.F, a->rope_base, 0, a->positions,
                            s);
        if (e != cudaSuccess) return cuda_fail(e, "decode: rotary embedding");
        phq = phq_buf;
        phk = phk_buf;
    }
    DecodeCore c{};
    c.B = a->B; c.H = a->H; c.F = pl.F; c.dv = a->dv;
    c.feat_dtype = ft; c.io_dtype = a->io_dtype;
    c.phq = phq; c.phk = phk; c.v = a->v; c.dt = a->dt; c.A_log = a->A_log;
    c.S = a->S; c.z = a->z; c.o = a->o;
    c.dt_scaled = (a->flags & HM_FLAG_DT_SCALED_INPUT) != 0;
    c.per_feature = (a->flags & HM_FLAG_PER_FEATURE_DECAY) != 0;
    e = launch_decode(c, s);
    return e == cudaSuccess ? HM_OK : cuda_fail(e, "decode launch");
}

namespace {

// ------------------------------------------------------------------ mixer

struct MixerPlan {
    size_t off_g, off_dt, off_q, off_k, off_v, off_o, off_scan;   // byte offsets
    size_t scan_bytes;
    size_t total;
    hm_scan_args scan;
};

hm_status check_mixer(const hm_mixer_args *a, MixerPlan *plan) {
    if (!a) return fail(HM_ERR_INVALID_ARG, "mixer: null args");
    if (a->B < 0 || a->L < 0 || a->d_model < 1 || a->H < 1 || a->E < 1 || a->p < 1 ||
        a->conv_k < 1 || a->conv_k > 8)
        return fail(HM_ERR_INVALID_ARG, "mixer: bad sizes");
    if (a->E % a->H != 0) return fail(HM_ERR_INVALID_ARG, "mixer: E must be a multiple of H");
    if (a->E % 16 != 0 || a->d_model % 16 != 0)
        return fail(HM_ERR_UNSUPPORTED, "mixer: E and d_model must be multiples of 16");
    const int64_t M = a->B * a->L;
    if (M > 0 && (!a->x || !a->W_q || !a->W_k || !a->W_v || !a->W_g || !a->W_dt || !a->conv_w ||
                  !a->W_hq || !a->W_hk || !a->A_log || !a->W_o || !a->out))
        return fail(HM_ERR_INVALID_ARG, "mixer: null pointer");
    const void *ptrs[] = {a->x, a->W_q, a->W_k, a->W_v, a->W_g, a->W_dt, a->b_dt, a->b_g,
                          a->conv_w, a->conv_b, a->W_hq, a->W_hk, a->A_log, a->W_o, a->out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return fail(HM_ERR_INVALID_ARG, "mixer: pointers must be 16-byte aligned");
    if (M > 0 && (!gemm_tc_supported(M, a->E, a->d_model) || !gemm_tc_supported(M, a->d_model, a->E)))
        return fail(HM_ERR_UNSUPPORTED, "mixer: no tensor-core GEMM for these sizes");
    MixerPlan pl{};
    const size_t E = (size_t)a->E;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = round_up(off + bytes, 256); return o; };
    // fp32: the activated gate SiLU(x W_g^T + b_g) (a bf16 gate would add a
    // rounding on top of y's) and dt; bf16: the gated scan output y and the
    // conv outputs (the scan's q, k, v)
    pl.off_g = take((size_t)M * E * 4);
    pl.off_o = take((size_t)M * E * 2);
    pl.off_dt = take((size_t)M * a->H * 4);
    pl.off_q = take((size_t)M * E * 2);
    pl.off_k = take((size_t)M * E * 2);
    pl.off_v = take((size_t)M * E * 2);
    hm_scan_args s{};
    s.B = a->B; s.L = a->L; s.H = a->H; s.d = a->E / a->H; s.p = a->p; s.dv = a->E / a->H;
    s.io_dtype = HM_BF16;
    // placeholders (aligned, non-null) so that the shape check below sizes the scan
    s.q = s.k = s.v = (const void *)256;
    s.o = (void *)256;
    s.W_q = a->W_hq ? a->W_hq : (const void *)16;  // non-null marker for sizing
    s.W_k = a->W_hk ? a->W_hk : (const void *)16;
    s.dt = (const float *)16;
    s.A_log = (const float *)16;
    ScanPlan sp{};
    hm_status st = check_scan(&s, &sp);
    if (st != HM_OK) return st;
    pl.scan_bytes = sp.total;
    pl.off_scan = take(sp.total);
    pl.total = off;
    pl.scan = s;
    *plan = pl;
    return HM_OK;
}

// dt[r, h] = x[r, :] . W_dt[h, :] + b_dt[h]: N = H is too small for a GEMM
// tile, so a warp takes a row and all H dot products at once (x read once, its
// 16-byte pieces reused for every head), with W_dt staged in shared memory when
// it fits (NH heads at compile time; the generic kernel below reads it through
// L1).
template <int NH>
__global__ void dt_proj_heads_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ W,
                                     const float *__restrict__ b, int64_t rows, int D, float *__restrict__ dt) {
    extern __shared__ uint4 wsm[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nv = D / 8;   // 16-byte pieces per row
    for (int i = threadIdx.x; i < NH * nv; i += blockDim.x) wsm[i] = reinterpret_cast<const uint4 *>(W)[i];
    __syncthreads();
    const int64_t wpb = blockDim.x >> 5;
    for (int64_t r = blockIdx.x * wpb + warp; r < rows; r += (int64_t)gridDim.x * wpb) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(x + r * D);
        float acc[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) acc[h] = 0.f;
        for (int c = lane; c < nv; c += 32) {
            const uint4 xv = xr[c];
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
            float xf[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xw[e]));
                xf[2 * e] = t.x;
                xf[2 * e + 1] = t.y;
            }
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                const uint4 wv = wsm[h * nv + c];
                const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ww[e]));
                    acc[h] = fmaf(xf[2 * e], t.x, acc[h]);
                    acc[h] = fmaf(xf[2 * e + 1], t.y, acc[h]);
                }
            }
        }
#pragma unroll
        for (int h = 0; h < NH; ++h) acc[h] = warp_sum(acc[h]);
        if (lane < NH) {
            float v = acc[0];
#pragma unroll
            for (int h = 1; h < NH; ++h)
                if (lane == h) v = acc[h];
            dt[r * NH + lane] = v + (b ? b[lane] : 0.f);
        }
    }
}

// generic H: one warp per row, a dot product per head
__global__ void dt_proj_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ W,
                               const float *__restrict__ b, int64_t rows, int D, int H,
                               float *__restrict__ dt) {
    const int lane = threadIdx.x & 31;
    int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (r >= rows) return;
    const __nv_bfloat16 *xr = x + r * D;
    for (int h = 0; h < H; ++h) {
        const __nv_bfloat16 *wh = W + (int64_t)h * D;
        float acc = 0.f;
        for (int i = lane * 8; i < D; i += 256) {
            const __nv_bfloat162 *xv = reinterpret_cast<const __nv_bfloat162 *>(xr + i);
            const __nv_bfloat162 *wv = reinterpret_cast<const __nv_bfloat162 *>(wh + i);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float2 a = __bfloat1622float2(xv[j]);
                float2 c = __bfloat1622float2(wv[j]);
                acc = fmaf(a.x, c.x, acc);
                acc = fmaf(a.y, c.y, acc);
            }
        }
        acc = warp_sum(acc);
        if (lane == 0) dt[r * H + h] = acc + (b ? b[h] : 0.f);
    }
}

template <int NH>
cudaError_t launch_dt_heads(const void *x, const void *W, const float *b, int64_t rows, int D, float *dt,
                            cudaStream_t s) {
    const size_t smem = (size_t)NH * D * 2;
    cudaError_t e = tc::ensure_smem_limit(dt_proj_heads_kernel<NH>, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (rows + 7) / 8;
    const unsigned grid = (unsigned)std::min<int64_t>(want, (int64_t)sms * 4);
    dt_proj_heads_kernel<NH><<<grid, 256, smem, s>>>((const __nv_bfloat16 *)x, (const __nv_bfloat16 *)W, b, rows, D,
                                                     dt);
    return cudaGetLastError();
}

// dt = x W_dt^T (+ b_dt), [rows, H] fp32
cudaError_t launch_dt_proj(const void *x, const void *W, const float *b, int64_t rows, int D, int H, float *dt,
                           cudaStream_t s) {
    cudaError_t e;
    const bool staged = (size_t)H * D * 2 <= 96 * 1024;
    if (staged && H == 8) e = launch_dt_heads<8>(x, W, b, rows, D, dt, s);
    else if (staged && H == 4) e = launch_dt_heads<4>(x, W, b, rows, D, dt, s);
    else if (staged && H == 16) e = launch_dt_heads<16>(x, W, b, rows, D, dt, s);
    else {
        const unsigned blocks = (unsigned)((rows * 32 + 255) / 256);
        dt_proj_kernel<<<blocks, 256, 0, s>>>((const __nv_bfloat16 *)x, (const __nv_bfloat16 *)W, b, rows, D, H, dt);
        e = cudaGetLastError();
    }
    count_launches(1);
    return e;
}

}  // namespace
}  // namespace hm

using namespace hm;

extern "C" {

const char *hm_status_string(hm_status s) {
    switch (s) {
        case HM_OK: return "HM_OK";
        case HM_ERR_INVALID_ARG: return "HM_ERR_INVALID_ARG: invalid argument";
        case HM_ERR_UNSUPPORTED: return "HM_ERR_UNSUPPORTED: no kernel for this shape or dtype";
        case HM_ERR_CUDA: return "HM_ERR_CUDA: CUDA runtime or launch failure";
        case HM_ERR_TIMEOUT: return "HM_ERR_TIMEOUT: a kernel's bounded wait expired";
        case HM_ERR_DEVICE: return "HM_ERR_DEVICE: a kernel reported an internal fault";
    }
    return "unknown hm_status";
}

const char *hm_last_error_detail(void) { return g_detail; }

const char *hm_version(void) { return "hm 0.1 (sm_100a)"; }

uint64_t hm_launch_count(void) { return (uint64_t)g_launches.load(std::memory_order_relaxed); }

hm_status hm_featmap(const void *x, hm_dtype xt, int64_t rows, int H, int d, int p, const void *W,
                     int64_t w_head_stride, const float *bias, void *phi, hm_dtype pt,
                     hm_stream_t stream) {
    g_detail[0] = 0;
    hm_status st = check_featmap(x, xt, rows, H, d, p, W, phi, pt);
    if (st != HM_OK) return st;
    if (w_head_stride < 0) return fail(HM_ERR_INVALID_ARG, "featmap: negative head stride");
    if (!aligned16(bias)) return fail(HM_ERR_INVALID_ARG, "featmap: bias must be 16-byte aligned");
    cudaError_t e = run_featmap(x, xt, rows, H, d, p, W, w_head_stride, bias, phi, pt,
                                (cudaStream_t)stream);
    return e == cudaSuccess ? HM_OK : cuda_fail(e, "featmap launch");
}

size_t hm_scan_workspace_size(const hm_scan_args *a) {
    ScanPlan pl;
    if (check_scan(a, &pl) != HM_OK) return 0;
    return pl.total;
}

}  // extern "C"

namespace hm {
namespace {

// The prefill; with o_f32 (tensor-core path only) o is written as fp32.
hm_status scan_impl(const hm_scan_args *a, bool o_f32, hm_stream_t stream, const void *gate = nullptr) {
    ScanPlan pl;
    hm_status st = check_scan(a, &pl);
    if (st != HM_OK) return st;
    if (pl.total > 0 && (!a->workspace || a->workspace_bytes < pl.total))
        return fail(HM_ERR_INVALID_ARG, "scan: workspace too small (%zu < %zu bytes)",
                    a->workspace_bytes, pl.total);
    if (((uintptr_t)a->workspace & 255u) != 0)
        return fail(HM_ERR_INVALID_ARG, "scan: workspace must be 256-byte aligned");
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t rows = a->B * a->L * a->H;
    char *ws = (char *)a->workspace;
    const void *phq = a->q, *phk = a->k, *phk_lo = nullptr;
    cudaError_t e;
    if (a->W_q && rows > 0) {
        void *wq = ws, *wk = ws + pl.phi_bytes;
        void *wkl = pl.lo_bytes ? ws + 2 * pl.phi_bytes : nullptr;
        if (a->o) {
            e = run_featmap_qk(a->q, a->k, a->io_dtype, rows, a->H, a->d, a->p, a->W_q, a->W_k,
                               a->w_head_stride, a->b_q, a->b_k, wq, wk, pl.feat, s, wkl);
            phq = wq;
        } else {
            // state only: phi(q) is not needed
            e = run_featmap(a->k, a->io_dtype, rows, a->H, a->d, a->p, a->W_k, a->w_head_stride, a->b_k, wk,
                            pl.feat, s, wkl);
            phq = nullptr;
        }
        if (e != cudaSuccess) return cuda_fail(e, "scan: feature maps");
        phk = wk;
        phk_lo = wkl;
    }
    if (!a->o) phq = nullptr;
    if ((a->flags & HM_FLAG_ROPE) && rows > 0) {
        // rotary embedding of phi(q), phi(k): in place on the maps computed
        // above, or from the caller's features into the workspace
        void *wq = ws, *wk = ws + pl.phi_bytes;
        void *wkl = pl.lo_bytes ? ws + 2 * pl.phi_bytes : nullptr;
        if (phq) {
            e = launch_rope(phq, nullptr, wq, nullptr, pl.feat, a->B, a->L, a->H, pl.F, a->rope_base, a->pos0,
                            nullptr, s);
            if (e != cudaSuccess) return cuda_fail(e, "scan: rotary embedding");
            phq = wq;
        }
        e = launch_rope(phk, phk_lo, wk, wkl, pl.feat, a->B, a->L, a->H, pl.F, a->rope_base, a->pos0, nullptr, s);
        if (e != cudaSuccess) return cuda_fail(e, "scan: rotary embedding");
        phk = wk;
        phk_lo = wkl;
    }
    if (a->log_decay_out) {
        e = launch_logdecay_sum(a->B, a->L, a->H, pl.F, (a->flags & HM_FLAG_PER_FEATURE_DECAY) != 0, a->dt,
                                a->A_log, a->log_decay_out, s);
        if (e != cudaSuccess) return cuda_fail(e, "scan: log decay sum");
    }
    ScanCore c{};
    c.B = a->B; c.L = a->L; c.H = a->H; c.F = pl.F; c.dv = a->dv;
    c.feat_dtype = pl.feat; c.io_dtype = a->io_dtype;
    c.phq = phq; c.phk = phk; c.phk_lo = phk_lo; c.v = a->v;
    c.dt = a->dt; c.A_log = a->A_log; c.S0 = a->S0; c.z0 = a->z0;
    c.o = a->o; c.S_out = a->S_out; c.z_out = a->z_out;
    c.o_f32 = o_f32 && pl.tc;
    c.dt_scaled = (a->flags & HM_FLAG_DT_SCALED_INPUT) != 0;
    c.per_feature = (a->flags & HM_FLAG_PER_FEATURE_DECAY) != 0;
    c.gate = pl.tc ? gate : nullptr;
    if (pl.tc)
        e = launch_scan_tc(c, ws + 2 * pl.phi_bytes + pl.lo_bytes, pl.tc_bytes,
                           DevErr{device_error_word()}, s);
    else
        e = launch_scan_simt(c, s);
    return e == cudaSuccess ? HM_OK : cuda_fail(e, "scan launch");
}

bool scan_uses_tc(const hm_scan_args *a) {
    ScanPlan pl;
    return check_scan(a, &pl) == HM_OK && pl.tc;
}

// The mixer on input x (the block passes its normalised input) into `out`,
// with `out_ep` the epilogue of the output projection (a plain bf16 store, or
// the block's residual addition).  Each step follows its producer without a
// trip through HBM of its own where an epilogue can take it:
//   q, k, v = causal conv of x W^T         (projection GEMMs, conv in the epilogue)
//   gate    = SiLU(x W_g^T + b_g)          (GEMM, SiLU in the epilogue; kept in fp32)
//   dt      = x W_dt^T + b_dt              (CUDA cores: 8 columns)
//   y       = scan(q, k, v) * gate         (the gate applied as the scan stores o)
//   out     = y W_o^T                      (GEMM, out_ep)
hm_status mixer_run(const hm_mixer_args *a, const void *x, const MixerPlan &pl, char *ws, GemmEpiArgs out_ep,
                    void *out, cudaStream_t s) {
    const int64_t M = a->B * a->L;
    if (M == 0) return HM_OK;
    const int E = a->E, D = a->d_model, H = a->H;
    DevErr err{device_error_word()};
    void *gate = ws + pl.off_g, *y = ws + pl.off_o;
    void *qc = ws + pl.off_q, *kc = ws + pl.off_k, *vc = ws + pl.off_v;
    float *dt = (float *)(ws + pl.off_dt);
    cudaError_t e;
    const void *Wp[3] = {a->W_q, a->W_k, a->W_v};
    void *dst[3] = {qc, kc, vc};
    for (int i = 0; i < 3; ++i) {
        GemmEpiArgs ep;
        ep.mode = EPI_CONV_BF16;
        ep.conv_w = a->conv_w + (size_t)i * E * a->conv_k;
        ep.conv_k = a->conv_k;
        ep.bias = a->conv_b ? a->conv_b + (size_t)i * E : nullptr;
        ep.seq_len = a->L;
        e = launch_gemm_tc_ex(x, Wp[i], M, E, D, dst[i], E, ep, err, s);
        if (e != cudaSuccess) return cuda_fail(e, "mixer: projection GEMM with conv");
    }
    {
        GemmEpiArgs ep;
        ep.mode = EPI_SILU_F32;
        ep.bias = a->b_g;
        e = launch_gemm_tc_ex(x, a->W_g, M, E, D, gate, E, ep, err, s);
        if (e != cudaSuccess) return cuda_fail(e, "mixer: gate GEMM");
    }
    e = launch_dt_proj(x, a->W_dt, a->b_dt, M, D, H, dt, s);
    if (e != cudaSuccess) return cuda_fail(e, "mixer: dt projection");
    hm_scan_args sa = pl.scan;
    sa.q = qc; sa.k = kc; sa.v = vc;
    sa.W_q = a->W_hq; sa.W_k = a->W_hk; sa.w_head_stride = 0;
    sa.b_q = nullptr; sa.b_k = nullptr;
    sa.dt = dt; sa.A_log = a->A_log;
    sa.S0 = nullptr; sa.z0 = nullptr; sa.S_out = nullptr; sa.z_out = nullptr;
    sa.o = y;
    sa.workspace = ws + pl.off_scan;
    sa.workspace_bytes = pl.scan_bytes;
    const bool fused_gate = scan_uses_tc(&sa);
    hm_status st = scan_impl(&sa, false, s, fused_gate ? gate : nullptr);
    if (st != HM_OK) return st;
    if (!fused_gate) {
        // the CUDA-core scan stores o as it is: y = o * gate in place
        e = launch_gate_mul(y, false, gate, M, E, y, s);
        if (e != cudaSuccess) return cuda_fail(e, "mixer: gate");
    }
    e = launch_gemm_tc_ex(y, a->W_o, M, D, E, out, D, out_ep, err, s);
    if (e != cudaSuccess) return cuda_fail(e, "mixer: out projection");
    return HM_OK;
}

}  // namespace
}  // namespace hm

using namespace hm;

extern "C" hm_status hm_scan_chunked_fwd(const hm_scan_args *a, hm_stream_t stream) {
    g_detail[0] = 0;
    return scan_impl(a, false, stream);
}

extern "C" {

size_t hm_scan_bwd_workspace_size(const hm_scan_bwd_args *a) {
    ScanBwdCore c;
    if (check_scan_bwd(a, &c) != HM_OK) return 0;
    return scan_bwd_workspace(c);
}

hm_status hm_scan_bwd(const hm_scan_bwd_args *a, hm_stream_t stream) {
    g_detail[0] = 0;
    ScanBwdCore c;
    hm_status st = check_scan_bwd(a, &c);
    if (st != HM_OK) return st;
    const size_t need = scan_bwd_workspace(c);
    if (!a->workspace || a->workspace_bytes < need)
        return fail(HM_ERR_INVALID_ARG, "scan_bwd: workspace too small (%zu < %zu bytes)", a->workspace_bytes, need);
    if (((uintptr_t)a->workspace & 255u) != 0)
        return fail(HM_ERR_INVALID_ARG, "scan_bwd: workspace must be 256-byte aligned");
    cudaError_t e = launch_scan_bwd(c, a->workspace, (cudaStream_t)stream);
    return e == cudaSuccess ? HM_OK : cuda_fail(e, "scan_bwd launch");
}

size_t hm_decode_workspace_size(const hm_decode_args *a) {
    DecodePlan pl;
    if (check_decode(a, &pl) != HM_OK) return 0;
    return pl.total;
}

hm_status hm_step_decode(const hm_decode_args *a, hm_stream_t stream) {
    g_detail[0] = 0;
    DecodePlan pl;
    hm_status st = check_decode(a, &pl);
    if (st != HM_OK) return st;
    if (pl.total > 0 && (!a->workspace || a->workspace_bytes < pl.total))
        return fail(HM_ERR_INVALID_ARG, "decode: workspace too small (%zu < %zu bytes)",
                    a->workspace_bytes, pl.total);
    if (((uintptr_t)a->workspace & 255u) != 0)
        return fail(HM_ERR_INVALID_ARG, "decode: workspace must be 256-byte aligned");
    char *ws = (char *)a->workspace;
    return decode_enqueue(a, pl, ws, ws + pl.phi_bytes, (cudaStream_t)stream);
}

size_t hm_mixer_workspace_size(const hm_mixer_args *a) {
    MixerPlan pl;
    if (check_mixer(a, &pl) != HM_OK) return 0;
    return pl.total;
}

hm_status hm_mixer_fwd(const hm_mixer_args *a, void *workspace, size_t ws_bytes, hm_stream_t stream) {
    g_detail[0] = 0;
    MixerPlan pl;
    hm_status st = check_mixer(a, &pl);
    if (st != HM_OK) return st;
    if (!workspace || ws_bytes < pl.total)
        return fail(HM_ERR_INVALID_ARG, "mixer: workspace too small (%zu < %zu bytes)", ws_bytes, pl.total);
    if (((uintptr_t)workspace & 255u) != 0)
        return fail(HM_ERR_INVALID_ARG, "mixer: workspace must be 256-byte aligned");
    const int64_t M = a->B * a->L;
    if (M == 0) return HM_OK;
    return mixer_run(a, a->x, pl, (char *)workspace, GemmEpiArgs{}, a->out, (cudaStream_t)stream);
}

namespace {

struct BlockPlan {
    MixerPlan mixer;
    size_t off_h1, off_h2, off_sum, off_u, off_mixer, total;
};

hm_status check_block(const hm_block_args *a, BlockPlan *plan) {
    if (!a) return fail(HM_ERR_INVALID_ARG, "block: null args");
    hm_mixer_args m = a->mixer;
    hm_status st = check_mixer(&m, &plan->mixer);
    if (st != HM_OK) return st;
    const int64_t M = m.B * m.L;
    const int D = m.d_model;
    if (a->d_ff < 64 || a->d_ff % 64 != 0)
        return fail(HM_ERR_UNSUPPORTED, "block: d_ff must be a multiple of 64");
    if (D % 256 != 0 || D > 4096)
        return fail(HM_ERR_UNSUPPORTED, "block: d_model must be a multiple of 256, at most 4096");
    if (!(a->eps > 0.f)) return fail(HM_ERR_INVALID_ARG, "block: eps must be > 0");
    if (M > 0 && (!a->W_fc1 || !a->W_fc2)) return fail(HM_ERR_INVALID_ARG, "block: null MLP weight");
    const void *ptrs[] = {a->ln1_w, a->ln1_b, a->ln2_w, a->ln2_b, a->W_fc1, a->b_fc1, a->W_fc2, a->b_fc2};
    for (const void *p : ptrs)
        if (!aligned16(p)) return fail(HM_ERR_INVALID_ARG, "block: pointers must be 16-byte aligned");
    if (M > 0 && (!gemm_tc_supported(M, a->d_ff, D) || !gemm_tc_supported(M, D, a->d_ff)))
        return fail(HM_ERR_UNSUPPORTED, "block: no tensor-core GEMM for these sizes");
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = round_up(off + bytes, 256); return o; };
    plan->off_h1 = take((size_t)M * D * 2);
    plan->off_h2 = take((size_t)M * D * 2);
    plan->off_sum = take((size_t)M * D * 4);
    plan->off_u = take((size_t)M * a->d_ff * 2);
    plan->off_mixer = take(plan->mixer.total);
    plan->total = off;
    return HM_OK;
}

}  // namespace

size_t hm_block_workspace_size(const hm_block_args *a) {
    BlockPlan pl;
    if (check_block(a, &pl) != HM_OK) return 0;
    return pl.total;
}

hm_status hm_block_fwd(const hm_block_args *a, void *workspace, size_t ws_bytes, hm_stream_t stream) {
    g_detail[0] = 0;
    BlockPlan pl;
    hm_status st = check_block(a, &pl);
    if (st != HM_OK) return st;
    if (!workspace || ws_bytes < pl.total)
        return fail(HM_ERR_INVALID_ARG, "block: workspace too small (%zu < %zu bytes)", ws_bytes, pl.total);
    if (((uintptr_t)workspace & 255u) != 0)
        return fail(HM_ERR_INVALID_ARG, "block: workspace must be 256-byte aligned");
    const hm_mixer_args &m = a->mixer;
    const int64_t M = m.B * m.L;
    if (M == 0) return HM_OK;
    const int D = m.d_model;
    cudaStream_t s = (cudaStream_t)stream;
    char *ws = (char *)workspace;
    void *h1 = ws + pl.off_h1, *h2 = ws + pl.off_h2, *u = ws + pl.off_u;
    float *sum = (float *)(ws + pl.off_sum);
    DevErr err{device_error_word()};
    cudaError_t e = launch_layernorm2(m.x, M, D, a->eps, a->ln1_w, a->ln1_b, a->ln2_w, a->ln2_b, h1, h2, s);
    if (e != cudaSuccess) return cuda_fail(e, "block: layer norms");
    // mixer branch: sum = x + mixer(h1), the residual added in the output projection's epilogue
    GemmEpiArgs ep;
    ep.mode = EPI_ADD_F32;
    ep.res = m.x;
    ep.ldr = D;
    st = mixer_run(&m, h1, pl.mixer, ws + pl.off_mixer, ep, sum, s);
    if (st != HM_OK) return st;
    // MLP branch: u = GELU(h2 W_fc1^T + b_fc1); out = u W_fc2^T + b_fc2 + sum
    GemmEpiArgs e1;
    e1.mode = EPI_GELU_BF16;
    e1.bias = a->b_fc1;
    e = launch_gemm_tc_ex(h2, a->W_fc1, M, a->d_ff, D, u, a->d_ff, e1, err, s);
    if (e != cudaSuccess) return cuda_fail(e, "block: MLP up projection");
    GemmEpiArgs e2;
    e2.mode = EPI_ADD_BF16;
    e2.bias = a->b_fc2;
    e2.res = sum;
    e2.ldr = D;
    e = launch_gemm_tc_ex(u, a->W_fc2, M, D, a->d_ff, m.out, D, e2, err, s);
    if (e != cudaSuccess) return cuda_fail(e, "block: MLP down projection");
    return HM_OK;
}

hm_status hm_get_device_error(hm_stream_t stream) {
    g_detail[0] = 0;
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    unsigned int *w = device_error_word();
    if (!w) return fail(HM_ERR_CUDA, "no device error word");
    unsigned int host[4] = {0, 0, 0, 0};
    e = cudaMemcpy(host, w, sizeof(host), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "read device error word");
    if (host[0] == 0) return HM_OK;
    unsigned int zero[4] = {0, 0, 0, 0};
    e = cudaMemcpy(w, zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
    return fail((hm_status)host[0], "kernel id %u, block %u, site %u", host[1], host[2], host[3]);
}

}  // extern "C"

// decode_noalloc.cu -- hm_step_decode_noalloc: the recurrent decode step for
// callers that cannot allocate device memory.
//
// hm_step_decode needs a small device workspace for the two feature vectors
// phi(q), phi(k) of every (batch, head).  Some callers have no way to provide
// one: for example a plugin whose host application owns all device memory and
// hands it no allocator, or a serving loop that must not allocate after start-
// up.  This entry point keeps that scratch in a fixed file-scope device array
// instead, so the caller passes only inputs and outputs.
//
// The array holds at most kMaxFeatures fp32 values per feature plane (two
// planes, 4 MiB in total); every GPU that loads the library keeps it for the
// life of the process.  All calls share it: two calls whose kernels overlap on
// the GPU (different streams, or different host threads on one device) race on
// it and must be serialised by the caller.  The planes are fully rewritten by
// each call before they are read, so nothing has to start at zero.
//
// Host code cannot use the array's name as a device address: the address is
// looked up once per device with cudaGetSymbolAddress (that device current)
// on the first call made on that device, which should therefore happen before
// any stream capture.
#include <cstdio>
#include <mutex>

#include "hm_internal.h"

namespace hm {

namespace {

constexpr int64_t kMaxFeatures = int64_t(1) << 19;  // per plane: B * H * F <= 524288

static __device__ __align__(256) float g_decode_scratch[2 * kMaxFeatures];

// Device address of g_decode_scratch on the current device (nullptr on error).
float *scratch_address(cudaError_t *err) {
    static std::mutex mu;
    static float *addr[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        *err = e != cudaSuccess ? e : cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> g(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) {
            *err = e;
            return nullptr;
        }
        addr[dev] = (float *)p;
    }
    *err = cudaSuccess;
    return addr[dev];
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

hm_status reject(hm_status s, const char *msg) {
    set_error_detail(msg);
    return s;
}

}  // namespace

}  // namespace hm

using namespace hm;

extern "C" hm_status hm_step_decode_noalloc(const hm_decode_args *a, hm_stream_t stream) {
    set_error_detail("");
    if (!a) return reject(HM_ERR_INVALID_ARG, "decode_noalloc: null args");
    if (a->io_dtype != HM_F32 && a->io_dtype != HM_BF16)
        return reject(HM_ERR_INVALID_ARG, "decode_noalloc: bad io dtype");
    if (a->B < 0 || a->H < 1 || a->d < 1 || a->dv < 1)
        return reject(HM_ERR_INVALID_ARG, "decode_noalloc: bad sizes");
    if ((a->W_q == nullptr) != (a->W_k == nullptr))
        return reject(HM_ERR_INVALID_ARG, "decode_noalloc: W_q and W_k must both be given or both NULL");
    if (a->dt && !a->A_log) return reject(HM_ERR_INVALID_ARG, "decode_noalloc: dt given without A_log");
    const int F = a->W_q ? 2 * a->p : a->d;
    if (a->W_q && (a->p < 1 || a->p > 256))
        return reject(HM_ERR_UNSUPPORTED, "decode_noalloc: need 1 <= p <= 256");
    if (F > 256) return reject(HM_ERR_UNSUPPORTED, "decode_noalloc: feature dim F > 256");
    if (a->d > 512) return reject(HM_ERR_UNSUPPORTED, "decode_noalloc: d > 512");
    if (a->dv % 4 != 0) return reject(HM_ERR_UNSUPPORTED, "decode_noalloc: dv must be a multiple of 4");
    if (a->B > 0 && (!a->q || !a->k || !a->v || !a->o || !a->S || !a->z))
        return reject(HM_ERR_INVALID_ARG, "decode_noalloc: null q/k/v/o/S/z");
    const void *ptrs[] = {a->q, a->k, a->v, a->W_q, a->W_k, a->b_q, a->b_k, a->dt, a->A_log,
                          a->S, a->z, a->o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return reject(HM_ERR_INVALID_ARG, "decode_noalloc: pointers must be 16-byte aligned");
    const int64_t rows = a->B * a->H;
    if (a->W_q && rows * F > kMaxFeatures) {
        static thread_local char msg[160];
        snprintf(msg, sizeof(msg),
                 "decode_noalloc: B*H*F = %lld exceeds the fixed scratch of %lld features per plane; "
                 "use hm_step_decode with a workspace",
                 (long long)(rows * F), (long long)kMaxFeatures);
        return reject(HM_ERR_INVALID_ARG, msg);
    }
    if (rows == 0) return HM_OK;
    cudaStream_t s = (cudaStream_t)stream;
    const void *phq = a->q, *phk = a->k;
    hm_dtype ft = a->io_dtype;
    cudaError_t e;
    if (a->W_q) {
        float *scratch = scratch_address(&e);
        if (!scratch) {
            set_error_detail(cudaGetErrorString(e));
            return HM_ERR_CUDA;
        }
        float *fq = scratch, *fk = scratch + kMaxFeatures;
        if (a->io_dtype == HM_BF16 && featmap_tc_supported(rows, a->H, a->d, a->p, a->w_head_stride)) {
            e = launch_featmap_tc(a->q, rows, a->H, a->d, a->p, a->W_q, a->w_head_stride, a->b_q, fq,
                                  HM_F32, DevErr{device_error_word()}, s);
            if (e == cudaSuccess)
                e = launch_featmap_tc(a->k, rows, a->H, a->d, a->p, a->W_k, a->w_head_stride, a->b_k, fk,
                                      HM_F32, DevErr{device_error_word()}, s);
        } else {
            e = launch_featmap_simt(a->q, a->io_dtype, rows, a->H, a->d, a->p, a->W_q, a->w_head_stride,
                                    a->b_q, fq, HM_F32, s);
            if (e == cudaSuccess)
                e = launch_featmap_simt(a->k, a->io_dtype, rows, a->H, a->d, a->p, a->W_k, a->w_head_stride,
                                        a->b_k, fk, HM_F32, s);
        }
        if (e != cudaSuccess) {
            set_error_detail(cudaGetErrorString(e));
            return HM_ERR_CUDA;
        }
        phq = fq;
        phk = fk;
        ft = HM_F32;
    }
    DecodeCore c{};
    c.B = a->B;
    c.H = a->H;
    c.F = F;
    c.dv = a->dv;
    c.feat_dtype = ft;
    c.io_dtype = a->io_dtype;
    c.phq = phq;
    c.phk = phk;
    c.v = a->v;
    c.dt = a->dt;
    c.A_log = a->A_log;
    c.S = a->S;
    c.z = a->z;
    c.o = a->o;
    e = launch_decode(c, s);
    if (e != cudaSuccess) {
        set_error_detail(cudaGetErrorString(e));
        return HM_ERR_CUDA;
    }
    return HM_OK;
}

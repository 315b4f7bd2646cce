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
// life of the process.  Apart from where the feature planes live, the call is
// hm_step_decode: the same argument checks, the same launches in the same
// order (fp32 features), so its results are bit-identical.  All calls share
// the array: two calls whose kernels overlap on the GPU (different streams, or
// different host threads on one device) race on it and must be serialised by
// the caller.  The planes are fully rewritten by each call before they are
// read, so nothing has to start at zero.
//
// Host code cannot use the array's name as a device address: the address is
// looked up with cudaGetSymbolAddress (that device current) on the first call
// made on each device and cached for the process, so that first call should
// come before any stream capture.  The cached address belongs to the device's
// primary context; after cudaDeviceReset it is stale, and this entry point must
// not be called again in that process.
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

hm_status reject(hm_status s, const char *msg) {
    set_error_detail(msg);
    return s;
}

}  // namespace

}  // namespace hm

using namespace hm;

extern "C" hm_status hm_step_decode_noalloc(const hm_decode_args *a, hm_stream_t stream) {
    set_error_detail("");
    DecodePlan pl;
    const hm_status st = check_decode_args(a, &pl);   // same checks and messages as hm_step_decode
    if (st != HM_OK) return st;
    if (pl.feat_values > kMaxFeatures) {
        static thread_local char msg[160];
        snprintf(msg, sizeof(msg),
                 "decode_noalloc: B*H*F = %lld exceeds the fixed scratch of %lld features per plane; "
                 "use hm_step_decode with a workspace",
                 (long long)pl.feat_values, (long long)kMaxFeatures);
        return reject(HM_ERR_INVALID_ARG, msg);
    }
    if (a->B == 0) return HM_OK;
    float *fq = nullptr, *fk = nullptr;
    if (pl.feat_values > 0) {   // feature planes: the Hedgehog maps, or rotated caller features
        cudaError_t e = cudaSuccess;
        float *scratch = scratch_address(&e);
        if (!scratch) return reject(HM_ERR_CUDA, cudaGetErrorString(e));
        fq = scratch;
        fk = scratch + kMaxFeatures;
    }
    // every value of both planes that the step reads is written by its own
    // feature-map launch first, so nothing left by an earlier call is read
    return decode_enqueue(a, pl, fq, fk, (cudaStream_t)stream);
}

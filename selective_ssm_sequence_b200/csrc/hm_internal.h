// hm_internal.h -- shared declarations of the libhm.so translation units.
// Not part of the public ABI (that is include/hm.h).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "hm.h"

namespace hm {

// Per-device error word written by kernels whose bounded waits expire.
// [0] = status (HM_ERR_TIMEOUT / HM_ERR_DEVICE), [1] = kernel id,
// [2] = block index, [3] = site / detail.  Kernels receive its address.
struct DevErr {
    unsigned int *word;
};

enum KernelId : unsigned int {
    KID_FEATMAP_SIMT = 1,
    KID_FEATMAP_TC = 2,
    KID_SCAN_SIMT = 3,
    KID_SCAN_TC_STATE = 4,
    KID_SCAN_TC_CARRY = 5,
    KID_SCAN_TC_OUT = 6,
    KID_DECODE = 7,
    KID_GEMM_TC = 8,
    KID_CONV = 9,
    KID_SELFTEST = 10,
    KID_BWD_DW_TC = 11,
};

unsigned int *device_error_word();  // address of this device's error word (host)

// Host-side count of kernels enqueued by the library (hm_launch_count).
void count_launches(unsigned int n);

// Sets the text hm_last_error_detail() returns on this host thread.
void set_error_detail(const char *msg);

// ---------------------------------------------------------------- device helpers

__device__ __forceinline__ float hm_ld(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float hm_ld(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void hm_st(float *p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void hm_st(__nv_bfloat16 *p, int64_t i, float v) { p[i] = __float2bfloat16_rn(v); }

// softplus(x) = log(1 + e^x) without overflow; fp32.
__device__ __forceinline__ float hm_softplus(float x) {
    return x > 0.f ? x + log1pf(expf(-x)) : log1pf(expf(x));
}

// log of the decay a = exp(-softplus(dt) * exp(A_log)).
__device__ __forceinline__ float hm_log_decay(float dt, float a_log) {
    float rate = expf(a_log);
    return rate == 0.f ? 0.f : -hm_softplus(dt) * rate;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ void report_error(DevErr e, unsigned int status, unsigned int kid,
                                             unsigned int site) {
    if (atomicCAS(e.word, 0u, status) == 0u) {
        e.word[1] = kid;
        e.word[2] = blockIdx.x + 65536u * blockIdx.y;
        e.word[3] = site;
    }
}

// ---------------------------------------------------------------- launchers

// Hedgehog map, SIMT (any dtype, any d/p that the host validated).
cudaError_t launch_featmap_simt(const void *x, hm_dtype xt, int64_t rows, int H, int d, int p,
                                const void *W, int64_t w_head_stride, const float *bias,
                                void *phi, hm_dtype pt, cudaStream_t s, void *phi_lo = nullptr);

// Hedgehog map on tcgen05 (bf16 in, bf16 or fp32 out).  With phi_lo (bf16
// out only), also writes the rounding remainder phi - bf16(phi).  Returns
// cudaErrorNotSupported if the shape has no tensor-core kernel.
cudaError_t launch_featmap_tc(const void *x, int64_t rows, int H, int d, int p, const void *W,
                              int64_t w_head_stride, const float *bias, void *phi, hm_dtype pt,
                              DevErr err, cudaStream_t s, void *phi_lo = nullptr);
bool featmap_tc_supported(int64_t rows, int H, int d, int p, int64_t w_head_stride);
// Two feature maps of the same shape (e.g. q and k) in one launch.
cudaError_t launch_featmap_tc2(const void *x0, const void *W0, const float *bias0, void *phi0, void *lo0,
                               const void *x1, const void *W1, const float *bias1, void *phi1, void *lo1,
                               int64_t rows, int H, int d, int p, int64_t w_head_stride, hm_dtype pt, DevErr err,
                               cudaStream_t s);

// Generic SIMT chunk-free scan over precomputed features (fp32 state).
struct ScanCore {
    int64_t B, L;
    int H, F, dv;
    hm_dtype feat_dtype;  // dtype of phq/phk
    hm_dtype io_dtype;    // dtype of v and o
    const void *phq, *phk, *v;
    const void *phk_lo;   // optional rounding remainder of phk (bf16), tensor-core path
    const float *dt, *A_log;
    const float *S0, *z0;
    void *o;
    bool o_f32;           // tensor-core path: write o as fp32 instead of io_dtype
    float *S_out, *z_out;
    bool dt_scaled;       // HM_FLAG_DT_SCALED_INPUT: input term times softplus(dt)
    bool per_feature;     // HM_FLAG_PER_FEATURE_DECAY: A_log is [H, F]
    // tensor-core path only: o is multiplied by this activated gate ([B, L, H,
    // dv] fp32, the layout of o) before it is stored (the mixer's o * SiLU(g))
    const void *gate = nullptr;
};
cudaError_t launch_scan_simt(const ScanCore &c, cudaStream_t s);

// Tensor-core chunked scan (bf16 features / v / o, F = 256, dv = 256).
bool scan_tc_supported(const ScanCore &c);
size_t scan_tc_workspace(const ScanCore &c);
cudaError_t launch_scan_tc(const ScanCore &c, void *ws, size_t ws_bytes, DevErr err,
                           cudaStream_t s);

// lambda = sum over the L tokens of log a_t per (b, h) ([B, H]) or per
// (b, h, f) with the per-feature decay ([B, H, F]); zeros when dt is NULL.
cudaError_t launch_logdecay_sum(int64_t B, int64_t L, int H, int F, bool per_feature, const float *dt,
                                const float *A_log, float *out, cudaStream_t s);

// Rotary embedding of feature rows [B, L, H, F] (ft = fp32 or bf16, with an
// optional bf16 remainder plane), src -> dst (may alias): pair (i, i + F/2) at
// angle (positions ? positions[b] : pos0 + t) * base^(-2i/F).
cudaError_t launch_rope(const void *src, const void *src_lo, void *dst, void *dst_lo, hm_dtype ft, int64_t B,
                        int64_t L, int H, int F, double base, int64_t pos0, const int64_t *positions,
                        cudaStream_t s);

// Backward of the scan and of the Hedgehog maps (CUDA cores, fp32).
struct ScanBwdCore {
    int64_t B, L;
    int H, d, p, F, dv;
    hm_dtype io_dtype;
    const void *q, *k, *v, *dout;
    const void *W_q, *W_k;    // shared Hedgehog weights, or null: q, k are the features
    const float *dt, *A_log, *S0, *z0;
    float *dq, *dk, *dv_out, *dW_q, *dW_k, *ddt, *dA_log, *dS0, *dz0;
};
size_t scan_bwd_workspace(const ScanBwdCore &c);
cudaError_t launch_scan_bwd(const ScanBwdCore &c, void *ws, cudaStream_t s);
// The Hedgehog map into fp32 features (tensor cores when the shape has a kernel).
cudaError_t run_featmap_f32(const void *x, hm_dtype xt, int64_t rows, int H, int d, int p, const void *W,
                            float *phi, cudaStream_t s);

// Decode step over precomputed features.
struct DecodeCore {
    int64_t B;
    int H, F, dv;
    hm_dtype feat_dtype, io_dtype;
    const void *phq, *phk, *v;
    const float *dt, *A_log;
    float *S, *z;
    void *o;
    bool dt_scaled;       // as in ScanCore
    bool per_feature;
};
cudaError_t launch_decode(const DecodeCore &c, cudaStream_t s);

// softplus(dt): the step size of the step-scaled input variant.
__device__ __forceinline__ float hm_step_size(float dt) { return hm_softplus(dt); }

// Checked shape of a decode call: F, and the size of each per-token feature
// plane (B * H * F values when W_q != NULL, else 0) and of the workspace.
struct DecodePlan {
    int F;
    int64_t feat_values;
    size_t phi_bytes;   // one feature plane, fp32, rounded up to 256 bytes
    size_t total;       // workspace bytes of hm_step_decode
};

// Argument check shared by every decode entry point (sets the error detail).
hm_status check_decode_args(const hm_decode_args *a, DecodePlan *plan);

// Enqueues a checked decode step with its feature planes at phq_buf / phk_buf
// (fp32, plan.feat_values each; ignored when W_q == NULL).
hm_status decode_enqueue(const hm_decode_args *a, const DecodePlan &plan, void *phq_buf, void *phk_buf,
                         cudaStream_t s);

// bf16 GEMM C[M,N] = A[M,K] B[N,K]^T on tcgen05 with a fused epilogue.
enum GemmEpi : int {
    EPI_STORE_BF16 = 0,  // C bf16 = acc (+ bias)
    EPI_STORE_F32 = 1,   // C fp32 = acc (+ bias)
    EPI_CONV_BF16 = 2,   // C bf16 = depthwise causal conv of acc along each sequence (+ bias)
    EPI_SILU_F32 = 3,    // C fp32 = SiLU(acc + bias)
    EPI_GELU_BF16 = 4,   // C bf16 = GELU(acc + bias), exact (erf) form
    EPI_ADD_F32 = 5,     // C fp32 = acc + bias + R, R bf16 [M, ldr]
    EPI_ADD_BF16 = 6,    // C bf16 = acc + bias + R, R fp32 [M, ldr]
};
// What the GEMM's epilogue does with the fp32 accumulator tile.
struct GemmEpiArgs {
    GemmEpi mode = EPI_STORE_BF16;
    const float *bias = nullptr;      // [N] per column, or null
    const float *conv_w = nullptr;    // EPI_CONV_BF16: [N, conv_k]; bias is the conv bias
    int conv_k = 1;                   // 1..8
    int64_t seq_len = 0;              // EPI_CONV_BF16: row r is token r % seq_len of its sequence
    const void *res = nullptr;        // EPI_ADD_*: residual
    int64_t ldr = 0;
};
bool gemm_tc_supported(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemm_tc(const void *A, const void *Bm, int64_t M, int64_t N, int64_t K,
                           void *C, int64_t ldc, GemmEpi epi, const float *bias, DevErr err,
                           cudaStream_t s);
cudaError_t launch_gemm_tc_ex(const void *A, const void *Bm, int64_t M, int64_t N, int64_t K, void *C,
                              int64_t ldc, const GemmEpiArgs &ep, DevErr err, cudaStream_t s);

// h1, h2 = layer norms of the rows of x [rows, D] bf16 with (w1, b1) and
// (w2, b2) (fp32 [D] each, NULL = 1 / 0), bf16 out
cudaError_t launch_layernorm2(const void *x, int64_t rows, int D, float eps, const float *w1, const float *b1,
                              const float *w2, const float *b2, void *h1, void *h2, cudaStream_t s);
// y = o * gate (o fp32 or bf16; the gate fp32, already activated: SiLU(g + b_g)
// from the gate GEMM's epilogue; y bf16, may alias o)
cudaError_t launch_gate_mul(const void *o, bool o_f32, const void *gate, int64_t rows, int E, void *y,
                            cudaStream_t s);

}  // namespace hm

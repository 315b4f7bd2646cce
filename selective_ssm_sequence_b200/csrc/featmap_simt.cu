// featmap_simt.cu -- Hedgehog feature map on CUDA cores (fp32 math).
//
// phi = softmax([W x + b, -(W x + b)]) over the 2p features (HedgeMamba
// explainer sec. 2.1 and 5.3: one Linear layer, concatenation with its
// negation, softmax along the feature axis).  One warp per row: the d-long
// dot products are split across lanes and reduced with shuffles; the max and
// the normaliser of the 2p-wide softmax are warp reductions.  Used for fp32
// inputs (where tensor-core TF32 would not meet a 1e-4 tolerance) and for
// shapes without a tensor-core kernel.
#include "hm_internal.h"

namespace hm {

namespace {

constexpr int kWarps = 8;
constexpr int kMaxPerLane = 8;  // p <= 256

template <typename TX, typename TP>
__global__ void __launch_bounds__(32 * kWarps)
featmap_simt_kernel(const TX *__restrict__ x, int64_t rows, int H, int d, int p,
                    const TX *__restrict__ W, int64_t w_head_stride,
                    const float *__restrict__ bias, TP *__restrict__ phi,
                    __nv_bfloat16 *__restrict__ phi_lo) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    for (int64_t r = (int64_t)blockIdx.x * kWarps + warp; r < rows;
         r += (int64_t)gridDim.x * kWarps) {
        const int h = (int)(r % H);
        const TX *Wh = W + (int64_t)h * w_head_stride;
        const float *bh = bias ? bias + (w_head_stride ? (int64_t)h * p : 0) : nullptr;
        const TX *xr = x + r * d;
        float u[kMaxPerLane];
#pragma unroll
        for (int m = 0; m < kMaxPerLane; ++m) u[m] = 0.f;
        // u_j = sum_i W[j, i] x[i]: lanes split i, reduce; lane (j % 32) keeps u_j
        for (int j = 0; j < p; ++j) {
            float acc = 0.f;
            for (int i = lane; i < d; i += 32) acc = fmaf(hm_ld(Wh, (int64_t)j * d + i), hm_ld(xr, i), acc);
            acc = warp_sum(acc);
            if ((j & 31) == lane) u[j >> 5] = acc + (bh ? bh[j] : 0.f);
        }
        float m = 0.f;  // max over [u, -u] = max |u| >= 0
#pragma unroll
        for (int t = 0; t < kMaxPerLane; ++t)
            if (t * 32 + lane < p) m = fmaxf(m, fabsf(u[t]));
        m = warp_max(m);
        float Z = 0.f;
#pragma unroll
        for (int t = 0; t < kMaxPerLane; ++t)
            if (t * 32 + lane < p) Z += expf(u[t] - m) + expf(-u[t] - m);
        Z = warp_sum(Z);
        const float inv = 1.f / Z;
        TP *out = phi + r * 2 * p;
#pragma unroll
        for (int t = 0; t < kMaxPerLane; ++t) {
            int j = t * 32 + lane;
            if (j < p) {
                const float e1 = expf(u[t] - m) * inv, e2 = expf(-u[t] - m) * inv;
                hm_st(out, j, e1);
                hm_st(out, p + j, e2);
                if (phi_lo) {
                    // rounding remainder of the bf16 value just stored
                    __nv_bfloat16 *lo = phi_lo + r * 2 * p;
                    lo[j] = __float2bfloat16_rn(e1 - __bfloat162float(__float2bfloat16_rn(e1)));
                    lo[p + j] = __float2bfloat16_rn(e2 - __bfloat162float(__float2bfloat16_rn(e2)));
                }
            }
        }
    }
}

template <typename TX, typename TP>
cudaError_t go(const void *x, int64_t rows, int H, int d, int p, const void *W, int64_t ws,
               const float *bias, void *phi, void *phi_lo, cudaStream_t s) {
    int64_t blocks = (rows + kWarps - 1) / kWarps;
    if (blocks > 148 * 64) blocks = 148 * 64;
    if (blocks < 1) return cudaSuccess;
    featmap_simt_kernel<TX, TP><<<(unsigned)blocks, 32 * kWarps, 0, s>>>(
        (const TX *)x, rows, H, d, p, (const TX *)W, ws, bias, (TP *)phi, (__nv_bfloat16 *)phi_lo);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_featmap_simt(const void *x, hm_dtype xt, int64_t rows, int H, int d, int p,
                                const void *W, int64_t w_head_stride, const float *bias,
                                void *phi, hm_dtype pt, cudaStream_t s, void *phi_lo) {
    if (rows == 0) return cudaSuccess;
    if (phi_lo && pt != HM_BF16) return cudaErrorInvalidValue;
    if (xt == HM_F32 && pt == HM_F32)
        return go<float, float>(x, rows, H, d, p, W, w_head_stride, bias, phi, nullptr, s);
    if (xt == HM_F32 && pt == HM_BF16)
        return go<float, __nv_bfloat16>(x, rows, H, d, p, W, w_head_stride, bias, phi, phi_lo, s);
    if (xt == HM_BF16 && pt == HM_F32)
        return go<__nv_bfloat16, float>(x, rows, H, d, p, W, w_head_stride, bias, phi, nullptr, s);
    return go<__nv_bfloat16, __nv_bfloat16>(x, rows, H, d, p, W, w_head_stride, bias, phi, phi_lo, s);
}

}  // namespace hm

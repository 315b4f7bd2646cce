// rope.cu -- rotary position embedding of feature vectors (HM_FLAG_ROPE).
//
// HedgeMamba explainer sec. 5.2: the mixer applies RoPE to phi(Q) and phi(K)
// before the scan.  Pairing feature i with feature i + F/2 ("rotate half", the
// convention of the GPT-NeoX / Pythia models the pages distil from), at angle
// pos * base^(-2i/F):
//     x_i'       = x_i cos - x_{i+F/2} sin
//     x_{i+F/2}' = x_i sin + x_{i+F/2} cos
// One thread per (row, pair).  The angle is formed and reduced modulo 2 pi in
// double precision (positions reach 10^5 and more, where an fp32 product
// would already be off by ~10^-2 rad), then sin / cos of the reduced angle in
// fp32.  bf16 features may carry a remainder plane (hi + lo, ~16 bits): the
// rotation then reads hi + lo and writes both again.  Runs as its own pass
// over the feature buffers, out of place or in place.
#include "hm_internal.h"

namespace hm {

namespace {

struct RopeArgs {
    double theta[128];       // base^(-2i/F), i < F/2
    int64_t rows, L;
    int H, F;
    int64_t pos0;
    const int64_t *positions;  // per batch (decode), or null: pos0 + t
};

__device__ __forceinline__ float ldf(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }

template <typename T>
__global__ void __launch_bounds__(256)
rope_kernel(RopeArgs a, const T *__restrict__ src, const __nv_bfloat16 *__restrict__ src_lo, T *dst,
            __nv_bfloat16 *dst_lo) {
    const int half = a.F / 2;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= a.rows * half) return;
    const int64_t r = gid / half;
    const int i = (int)(gid % half);
    // row r of a token-major [B, L, H] tensor: batch r / (L H), token (r / H) mod L
    const int64_t t = (r / a.H) % a.L;
    const int64_t pos = (a.positions ? a.positions[r / ((int64_t)a.L * a.H)] : a.pos0) + t;
    const double ang = (double)pos * a.theta[i];
    const double two_pi = 6.283185307179586476925;
    const float red = (float)(ang - rint(ang / two_pi) * two_pi);
    float sn, cs;
    sincosf(red, &sn, &cs);
    const int64_t ia = r * a.F + i, ib = ia + half;
    float x0 = ldf(src, ia), x1 = ldf(src, ib);
    if (src_lo) {
        x0 += __bfloat162float(src_lo[ia]);
        x1 += __bfloat162float(src_lo[ib]);
    }
    const float y0 = x0 * cs - x1 * sn, y1 = x0 * sn + x1 * cs;
    hm_st(dst, ia, y0);
    hm_st(dst, ib, y1);
    if (dst_lo) {
        // remainder of the bf16 value just stored (round to nearest, as hm_st)
        dst_lo[ia] = __float2bfloat16_rn(y0 - __bfloat162float(__float2bfloat16_rn(y0)));
        dst_lo[ib] = __float2bfloat16_rn(y1 - __bfloat162float(__float2bfloat16_rn(y1)));
    }
}

}  // namespace

cudaError_t launch_rope(const void *src, const void *src_lo, void *dst, void *dst_lo, hm_dtype ft, int64_t B,
                        int64_t L, int H, int F, double base, int64_t pos0, const int64_t *positions,
                        cudaStream_t s) {
    const int64_t rows = B * L * H;
    if (rows == 0) return cudaSuccess;
    if (F % 2 != 0 || F / 2 > 128 || !(base > 0.0)) return cudaErrorInvalidValue;
    if ((src_lo || dst_lo) && ft != HM_BF16) return cudaErrorInvalidValue;
    RopeArgs a{};
    for (int i = 0; i < F / 2; ++i) a.theta[i] = pow(base, -2.0 * (double)i / (double)F);
    a.rows = rows;
    a.L = L;
    a.H = H;
    a.F = F;
    a.pos0 = pos0;
    a.positions = positions;
    const int64_t threads = rows * (F / 2);
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    if (ft == HM_BF16)
        rope_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(a, (const __nv_bfloat16 *)src,
                                                          (const __nv_bfloat16 *)src_lo, (__nv_bfloat16 *)dst,
                                                          (__nv_bfloat16 *)dst_lo);
    else
        rope_kernel<float><<<blocks, 256, 0, s>>>(a, (const float *)src, nullptr, (float *)dst, nullptr);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace hm

// layernorm.cu -- the two layer norms at the head of the parallel block.
//
// The GPT-NeoX / Pythia block normalises its input twice, once for the mixer
// branch and once for the MLP branch (HedgeMamba explainer sec. 5.1):
//   h_i = (x - mean) / sqrt(var + eps) * w_i + b_i,   i = 1, 2,
// with the population variance over the row.  Both outputs come from one read
// of x: a warp per row, the row's mean and then its centred variance by warp
// sums (two passes over the row, the second from L1), then both affine maps
// written as bf16.  Bandwidth-bound: 2 B read and 4 B written per element.
#include "hm_internal.h"

namespace hm {

namespace {

__device__ __forceinline__ void ld8(const __nv_bfloat16 *p, float *f) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

__device__ __forceinline__ uint4 pk8(const float *f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void layernorm2_kernel(const __nv_bfloat16 *__restrict__ x, int64_t rows, int D, float eps,
                                  const float *__restrict__ w1, const float *__restrict__ b1,
                                  const float *__restrict__ w2, const float *__restrict__ b2,
                                  __nv_bfloat16 *__restrict__ h1, __nv_bfloat16 *__restrict__ h2) {
    const int lane = threadIdx.x & 31;
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (r >= rows) return;
    const __nv_bfloat16 *xr = x + r * D;
    float sum = 0.f;
    for (int c = lane * 8; c < D; c += 256) {
        float f[8];
        ld8(xr + c, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) sum += f[i];
    }
    const float mean = warp_sum(sum) / (float)D;
    float sq = 0.f;
    for (int c = lane * 8; c < D; c += 256) {
        float f[8];
        ld8(xr + c, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float dlt = f[i] - mean;
            sq = fmaf(dlt, dlt, sq);
        }
    }
    const float rstd = rsqrtf(warp_sum(sq) / (float)D + eps);
    for (int c = lane * 8; c < D; c += 256) {
        float f[8], o1[8], o2[8];
        ld8(xr + c, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float n = (f[i] - mean) * rstd;
            o1[i] = fmaf(n, w1 ? w1[c + i] : 1.f, b1 ? b1[c + i] : 0.f);
            o2[i] = fmaf(n, w2 ? w2[c + i] : 1.f, b2 ? b2[c + i] : 0.f);
        }
        *reinterpret_cast<uint4 *>(h1 + r * D + c) = pk8(o1);
        *reinterpret_cast<uint4 *>(h2 + r * D + c) = pk8(o2);
    }
}

}  // namespace

cudaError_t launch_layernorm2(const void *x, int64_t rows, int D, float eps, const float *w1, const float *b1,
                              const float *w2, const float *b2, void *h1, void *h2, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    if (D % 8 != 0) return cudaErrorInvalidValue;
    const unsigned blocks = (unsigned)((rows * 32 + 255) / 256);
    layernorm2_kernel<<<blocks, 256, 0, s>>>((const __nv_bfloat16 *)x, rows, D, eps, w1, b1, w2, b2,
                                             (__nv_bfloat16 *)h1, (__nv_bfloat16 *)h2);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace hm

// layernorm.cu -- the two layer norms at the head of the parallel block.
//
// The GPT-NeoX / Pythia block normalises its input twice, once for the mixer
// branch and once for the MLP branch (HedgeMamba explainer sec. 5.1):
//   h_i = (x - mean) / sqrt(var + eps) * w_i + b_i,   i = 1, 2,
// with the population variance over the row.  Both outputs come from one read
// of x: a warp per row with the row in registers (D a multiple of 256, at
// most 4096), its mean and then its centred variance by warp sums, then both
// affine maps written as bf16.  Bandwidth-bound: 2 B read and 4 B written per
// element.
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

// 8 consecutive fp32 parameters (16-byte aligned), or the default when null
__device__ __forceinline__ void ldp8(const float *p, int c, float dflt, float *f) {
    if (!p) {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = dflt;
        return;
    }
    const float4 a = *reinterpret_cast<const float4 *>(p + c);
    const float4 b = *reinterpret_cast<const float4 *>(p + c + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// NCH = D / 256 pieces of 8 elements per lane, held in registers: x is read
// once, the mean and the centred variance come from the registers.
template <int NCH>
__global__ void layernorm2_kernel(const __nv_bfloat16 *__restrict__ x, int64_t rows, int D, float eps,
                                  const float *__restrict__ w1, const float *__restrict__ b1,
                                  const float *__restrict__ w2, const float *__restrict__ b2,
                                  __nv_bfloat16 *__restrict__ h1, __nv_bfloat16 *__restrict__ h2) {
    const int lane = threadIdx.x & 31;
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (r >= rows) return;
    const __nv_bfloat16 *xr = x + r * D;
    float f[NCH][8];
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
        ld8(xr + k * 256 + lane * 8, f[k]);
#pragma unroll
        for (int i = 0; i < 8; ++i) sum += f[k][i];
    }
    const float mean = warp_sum(sum) / (float)D;
    float sq = 0.f;
#pragma unroll
    for (int k = 0; k < NCH; ++k)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float dlt = f[k][i] - mean;
            sq = fmaf(dlt, dlt, sq);
        }
    const float rstd = rsqrtf(warp_sum(sq) / (float)D + eps);
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
        const int c = k * 256 + lane * 8;
        float pw1[8], pb1[8], pw2[8], pb2[8], o1[8], o2[8];
        ldp8(w1, c, 1.f, pw1);
        ldp8(b1, c, 0.f, pb1);
        ldp8(w2, c, 1.f, pw2);
        ldp8(b2, c, 0.f, pb2);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float n = (f[k][i] - mean) * rstd;
            o1[i] = fmaf(n, pw1[i], pb1[i]);
            o2[i] = fmaf(n, pw2[i], pb2[i]);
        }
        *reinterpret_cast<uint4 *>(h1 + r * D + c) = pk8(o1);
        *reinterpret_cast<uint4 *>(h2 + r * D + c) = pk8(o2);
    }
}

}  // namespace

cudaError_t launch_layernorm2(const void *x, int64_t rows, int D, float eps, const float *w1, const float *b1,
                              const float *w2, const float *b2, void *h1, void *h2, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    if (D % 256 != 0 || D > 256 * 16) return cudaErrorInvalidValue;
    const unsigned blocks = (unsigned)((rows * 32 + 255) / 256);
    auto xb = (const __nv_bfloat16 *)x;
    auto o1 = (__nv_bfloat16 *)h1;
    auto o2 = (__nv_bfloat16 *)h2;
    switch (D / 256) {
#define HM_LN_CASE(N) \
    case N: layernorm2_kernel<N><<<blocks, 256, 0, s>>>(xb, rows, D, eps, w1, b1, w2, b2, o1, o2); break;
        HM_LN_CASE(1) HM_LN_CASE(2) HM_LN_CASE(3) HM_LN_CASE(4) HM_LN_CASE(5) HM_LN_CASE(6) HM_LN_CASE(7)
        HM_LN_CASE(8) HM_LN_CASE(9) HM_LN_CASE(10) HM_LN_CASE(11) HM_LN_CASE(12) HM_LN_CASE(13) HM_LN_CASE(14)
        HM_LN_CASE(15) HM_LN_CASE(16)
#undef HM_LN_CASE
        default: return cudaErrorInvalidValue;
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace hm

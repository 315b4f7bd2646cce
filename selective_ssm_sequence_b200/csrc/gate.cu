// gate.cu -- y = o * gate, the mixer's output gate when the scan runs on the
// CUDA cores (HedgeMamba explainer sec. 2.3 / 5.2: the gate multiplies the
// normalised scan output).  The gate arrives activated and in fp32 (SiLU(x W_g^T
// + b_g), applied in the gate GEMM's epilogue); the tensor-core scan multiplies it in
// as it stores o, so this kernel only serves the other shapes.  8 channels per
// thread, 16-byte loads and stores; bandwidth-bound.
#include "hm_internal.h"

namespace hm {

namespace {

__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float *f) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
__device__ __forceinline__ void load8(const float *p, float *f) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    const float4 b = *reinterpret_cast<const float4 *>(p + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

template <typename TO>
__global__ void gate_mul_kernel(const TO *o, const float *__restrict__ gate, int64_t rows, int E,
                                __nv_bfloat16 *y) {
    const int evec = E / 8;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= rows * evec) return;
    const int64_t i0 = (gid / evec) * E + (gid % evec) * 8;
    float fo[8], fg[8];
    load8(o + i0, fo);
    load8(gate + i0, fg);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(fo[2 * i] * fg[2 * i], fo[2 * i + 1] * fg[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(y + i0) = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace

cudaError_t launch_gate_mul(const void *o, bool o_f32, const void *gate, int64_t rows, int E, void *y,
                            cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    if (E % 8 != 0) return cudaErrorInvalidValue;
    const int64_t threads = rows * (E / 8);
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    auto yb = (__nv_bfloat16 *)y;
    auto gb = (const float *)gate;
    if (o_f32)
        gate_mul_kernel<float><<<blocks, 256, 0, s>>>((const float *)o, gb, rows, E, yb);
    else
        gate_mul_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>((const __nv_bfloat16 *)o, gb, rows, E, yb);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace hm

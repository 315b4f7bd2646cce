// conv_gate.cu -- the mixer's short causal conv and SiLU gate (bandwidth-bound).
//
// Depthwise causal conv along the sequence (the Mamba short conv that the
// HedgeMamba mixer keeps, HedgeMamba explainer sec. 2.2 / 2.3):
//   y[b, t, c] = bias[c] + sum_{j<K} w[c, j] * x[b, t-(K-1)+j, c],  x = 0 before t = 0,
// no activation.  Gate (sec. 2.3 / 5.2: applied after num/den):
//   y = o * SiLU(g + b_g).
// Each thread handles 8 adjacent channels of a run of consecutive tokens,
// keeping the last K-1 inputs in registers so every input element is read
// once.  Inputs may be fp32 (projection outputs kept unrounded) or bf16.
#include "hm_internal.h"

namespace hm {

namespace {

constexpr int kTokRun = 32;  // tokens per thread

struct alignas(16) bf8 {
    __nv_bfloat162 h[4];
};

__device__ __forceinline__ void unpack(const bf8 &v, float *f) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(v.h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
__device__ __forceinline__ bf8 pack(const float *f) {
    bf8 v;
#pragma unroll
    for (int i = 0; i < 4; ++i) v.h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return v;
}

__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float *f) {
    unpack(*reinterpret_cast<const bf8 *>(p), f);
}
__device__ __forceinline__ void load8(const float *p, float *f) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    const float4 b = *reinterpret_cast<const float4 *>(p + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

template <int K, typename TX>
__global__ void causal_conv_kernel(const TX *__restrict__ x, int64_t x_ld, int64_t L,
                                   int C, const float *__restrict__ w, const float *__restrict__ bias,
                                   __nv_bfloat16 *__restrict__ y, int64_t y_ld, int64_t runs) {
    const int cvec = C / 8;
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= runs * cvec) return;
    const int c0 = (int)(gid % cvec) * 8;
    const int64_t run = gid / cvec;
    const int64_t runs_per_seq = (L + kTokRun - 1) / kTokRun;
    const int64_t b = run / runs_per_seq;
    const int64_t t0 = (run % runs_per_seq) * kTokRun;

    float wk[8][K], bb[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        bb[i] = bias ? bias[c0 + i] : 0.f;
#pragma unroll
        for (int j = 0; j < K; ++j) wk[i][j] = w[(int64_t)(c0 + i) * K + j];
    }
    // history: hist[j] holds x at t - (K-1) + j for j < K-1
    float hist[K > 1 ? K - 1 : 1][8];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
        int64_t s = t0 - (K - 1) + j;
        if (s >= 0) {
            load8(x + (b * L + s) * x_ld + c0, hist[j]);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) hist[j][i] = 0.f;
        }
    }
    const int64_t t1 = (t0 + kTokRun < L) ? t0 + kTokRun : L;
    for (int64_t t = t0; t < t1; ++t) {
        float cur[8];
        load8(x + (b * L + t) * x_ld + c0, cur);
        float out[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float acc = bb[i];
#pragma unroll
            for (int j = 0; j < K - 1; ++j) acc = fmaf(wk[i][j], hist[j][i], acc);
            out[i] = fmaf(wk[i][K - 1], cur[i], acc);
        }
        *reinterpret_cast<bf8 *>(y + (b * L + t) * y_ld + c0) = pack(out);
#pragma unroll
        for (int j = 0; j + 1 < K - 1; ++j)
#pragma unroll
            for (int i = 0; i < 8; ++i) hist[j][i] = hist[j + 1][i];
        if (K > 1) {
#pragma unroll
            for (int i = 0; i < 8; ++i) hist[K > 1 ? K - 2 : 0][i] = cur[i];
        }
    }
}

template <typename TO, typename TG>
__global__ void gate_kernel(const TO *__restrict__ o, const TG *__restrict__ g,
                            int64_t g_ld, const float *__restrict__ b_g, int64_t rows, int E,
                            __nv_bfloat16 *__restrict__ y) {
    const int evec = E / 8;
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= rows * evec) return;
    const int64_t r = gid / evec;
    const int c0 = (int)(gid % evec) * 8;
    float fo[8], fg[8], out[8];
    load8(o + r * E + c0, fo);
    load8(g + r * g_ld + c0, fg);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float gg = fg[i] + (b_g ? b_g[c0 + i] : 0.f);
        out[i] = fo[i] * (gg / (1.f + expf(-gg)));
    }
    *reinterpret_cast<bf8 *>(y + r * E + c0) = pack(out);
}

}  // namespace

cudaError_t launch_causal_conv(const void *x, bool x_f32, int64_t x_ld, int64_t B, int64_t L, int C,
                               int K, const float *w, const float *bias, void *y, int64_t y_ld,
                               cudaStream_t s) {
    if (B * L == 0) return cudaSuccess;
    const int64_t runs = B * ((L + kTokRun - 1) / kTokRun);
    const int64_t threads = runs * (C / 8);
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    auto yb = (__nv_bfloat16 *)y;
    switch (K) {
#define HM_CONV_CASE(KK)                                                                           \
    case KK:                                                                                       \
        if (x_f32)                                                                                 \
            causal_conv_kernel<KK, float><<<blocks, 256, 0, s>>>((const float *)x, x_ld, L, C, w,  \
                                                                 bias, yb, y_ld, runs);            \
        else                                                                                       \
            causal_conv_kernel<KK, __nv_bfloat16><<<blocks, 256, 0, s>>>(                          \
                (const __nv_bfloat16 *)x, x_ld, L, C, w, bias, yb, y_ld, runs);                    \
        break;
        HM_CONV_CASE(1)
        HM_CONV_CASE(2)
        HM_CONV_CASE(3)
        HM_CONV_CASE(4)
        HM_CONV_CASE(5)
        HM_CONV_CASE(6)
        HM_CONV_CASE(7)
        HM_CONV_CASE(8)
#undef HM_CONV_CASE
        default:
            return cudaErrorInvalidValue;
    }
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_gate(const void *o, bool o_f32, const void *g, bool g_f32, int64_t g_ld,
                        const float *b_g, int64_t rows, int E, void *y, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const int64_t threads = rows * (E / 8);
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    auto yb = (__nv_bfloat16 *)y;
    if (o_f32 && g_f32)
        gate_kernel<float, float><<<blocks, 256, 0, s>>>((const float *)o, (const float *)g, g_ld, b_g, rows, E, yb);
    else if (o_f32)
        gate_kernel<float, __nv_bfloat16><<<blocks, 256, 0, s>>>((const float *)o, (const __nv_bfloat16 *)g, g_ld,
                                                                  b_g, rows, E, yb);
    else if (g_f32)
        gate_kernel<__nv_bfloat16, float><<<blocks, 256, 0, s>>>((const __nv_bfloat16 *)o, (const float *)g, g_ld,
                                                                  b_g, rows, E, yb);
    else
        gate_kernel<__nv_bfloat16, __nv_bfloat16><<<blocks, 256, 0, s>>>(
            (const __nv_bfloat16 *)o, (const __nv_bfloat16 *)g, g_ld, b_g, rows, E, yb);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace hm

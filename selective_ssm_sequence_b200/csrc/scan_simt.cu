// scan_simt.cu -- the decayed normalised recurrence on CUDA cores, fp32.
//
//   S_t = a_t S_{t-1} + phik_t v_t^T,  z_t = a_t z_{t-1} + phik_t,
//   o_t = phiq_t^T S_t / phiq_t^T z_t,  a_t = exp(-softplus(dt_t) exp(A_log_h))
//
// (HedgeMamba explainer sec. 2.3 / 5.2 doubled state and division;
// linear-attention tutorial sec. 3 recurrent form.)  One CTA owns one
// (batch, head) and a 32-column slice of v; its 8 warps split the F feature
// rows of the state (warp w holds rows w, w+8, ...; lane = value column), so
// S lives in registers.  Tokens are staged 16 at a time in shared memory;
// per-token partial numerators / denominators are reduced across warps once
// per 16 tokens.  This is the fp32 path (a 1e-4 tolerance rules out bf16 or
// TF32 tensor-core operands) and the path for shapes without a tensor-core
// kernel; it performs the recurrence in exactly the order of its definition.
//
// Variants (the scan's flags): with the step-scaled input the staged phik of
// token t is multiplied by Delta_t = softplus(dt_t) (Mamba's B-bar = Delta B);
// with the per-feature decay a_t is staged per (token, feature) from A_log
// [H, F] and scales row f of S and entry f of z (gated linear attention's
// diag(alpha_t)).
#include "hm_internal.h"

namespace hm {

namespace {

constexpr int kW = 8;        // warps
constexpr int kTB = 16;      // tokens staged per round
constexpr int kMaxRows = 32; // F <= 256 -> at most 32 rows per warp

template <typename TF, typename TIO>
__global__ void __launch_bounds__(32 * kW)
scan_simt_kernel(int64_t L, int H, int F, int dv, const TF *__restrict__ phq,
                 const TF *__restrict__ phk, const TIO *__restrict__ v,
                 const float *__restrict__ dt, const float *__restrict__ A_log,
                 const float *__restrict__ S0, const float *__restrict__ z0, TIO *__restrict__ o,
                 float *__restrict__ S_out, float *__restrict__ z_out, int dt_scaled, int per_feature) {
    extern __shared__ float smem[];
    float *sq = smem;                      // [kTB][F]
    float *sk = sq + kTB * F;              // [kTB][F]
    float *sv = sk + kTB * F;              // [kTB][32]
    float *sa = sv + kTB * 32;             // [kTB]
    float *red = sa + kTB;                 // [kTB][kW][32]
    float *rden = red + kTB * kW * 32;     // [kTB][kW]
    float *saf = rden + kTB * kW;          // [kTB][F] per-feature decay (per_feature only)
    float *sdl = saf + (per_feature ? kTB * F : 0);   // [kTB] step sizes

    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t bh = blockIdx.y;
    const int64_t b = bh / H;
    const int h = (int)(bh % H);
    const int col = blockIdx.x * 32 + lane;
    const bool col_ok = col < dv;
    const float a_rate = (dt != nullptr && !per_feature) ? A_log[h] : 0.f;

    float S[kMaxRows], z[kMaxRows];
#pragma unroll
    for (int m = 0; m < kMaxRows; ++m) {
        int f = w + kW * m;
        S[m] = 0.f;
        z[m] = 0.f;
        if (f < F) {
            if (S0 && col_ok) S[m] = S0[(bh * F + f) * dv + col];
            if (z0) z[m] = z0[bh * F + f];
        }
    }

    for (int64_t t0 = 0; t0 < L; t0 += kTB) {
        const int nt = (int)((L - t0) < kTB ? (L - t0) : kTB);
        for (int i = threadIdx.x; i < nt * F; i += blockDim.x) {
            int t = i / F, f = i % F;
            int64_t row = (b * L + t0 + t) * H + h;
            sq[t * F + f] = phq ? hm_ld(phq, row * F + f) : 0.f;   // no phq: state-only call
            sk[t * F + f] = hm_ld(phk, row * F + f);
        }
        for (int i = threadIdx.x; i < nt * 32; i += blockDim.x) {
            int t = i / 32, c = blockIdx.x * 32 + (i % 32);
            int64_t row = (b * L + t0 + t) * H + h;
            sv[i] = c < dv ? hm_ld(v, row * dv + c) : 0.f;
        }
        if (threadIdx.x < nt) {
            int64_t row = (b * L + t0 + threadIdx.x) * H + h;
            sa[threadIdx.x] = (dt && !per_feature) ? expf(hm_log_decay(dt[row], a_rate)) : 1.f;
            sdl[threadIdx.x] = dt_scaled ? hm_step_size(dt[row]) : 1.f;
        }
        if (per_feature)
            for (int i = threadIdx.x; i < nt * F; i += blockDim.x) {
                int t = i / F, f = i % F;
                int64_t row = (b * L + t0 + t) * H + h;
                saf[i] = expf(hm_log_decay(dt[row], A_log[(int64_t)h * F + f]));
            }
        __syncthreads();
        if (dt_scaled) {
            for (int i = threadIdx.x; i < nt * F; i += blockDim.x) sk[i] *= sdl[i / F];
            __syncthreads();
        }
        for (int t = 0; t < nt; ++t) {
            const float at = sa[t];
            const float vv = sv[t * 32 + lane];
            float num = 0.f, den = 0.f;
#pragma unroll
            for (int m = 0; m < kMaxRows; ++m) {
                int f = w + kW * m;
                if (f < F) {
                    const float a = per_feature ? saf[t * F + f] : at;
                    float kf = sk[t * F + f], qf = sq[t * F + f];
                    S[m] = fmaf(a, S[m], kf * vv);
                    num = fmaf(qf, S[m], num);
                    z[m] = fmaf(a, z[m], kf);
                    den = fmaf(qf, z[m], den);
                }
            }
            red[(t * kW + w) * 32 + lane] = num;
            if (lane == 0) rden[t * kW + w] = den;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < nt * 32; i += blockDim.x) {
            int t = i / 32, c = i % 32;
            float num = 0.f, den = 0.f;
#pragma unroll
            for (int ww = 0; ww < kW; ++ww) {
                num += red[(t * kW + ww) * 32 + c];
                den += rden[t * kW + ww];
            }
            int cc = blockIdx.x * 32 + c;
            if (cc < dv && o) {
                int64_t row = (b * L + t0 + t) * H + h;
                hm_st(o, row * dv + cc, num / den);
            }
        }
        __syncthreads();
    }

#pragma unroll
    for (int m = 0; m < kMaxRows; ++m) {
        int f = w + kW * m;
        if (f < F) {
            if (S_out && col_ok) S_out[(bh * F + f) * dv + col] = S[m];
            if (z_out && blockIdx.x == 0 && lane == 0) z_out[bh * F + f] = z[m];
        }
    }
}

template <typename TF, typename TIO>
cudaError_t go(const ScanCore &c, cudaStream_t s) {
    dim3 grid((unsigned)((c.dv + 31) / 32), (unsigned)(c.B * c.H));
    size_t smem = sizeof(float) * (size_t)(2 * kTB * c.F + kTB * 32 + kTB + kTB * kW * 32 + kTB * kW +
                                           (c.per_feature ? kTB * c.F : 0) + kTB);
    auto kern = scan_simt_kernel<TF, TIO>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<grid, 32 * kW, smem, s>>>(c.L, c.H, c.F, c.dv, (const TF *)c.phq, (const TF *)c.phk,
                                     (const TIO *)c.v, c.dt, c.A_log, c.S0, c.z0, (TIO *)c.o,
                                     c.S_out, c.z_out, c.dt_scaled ? 1 : 0, c.per_feature ? 1 : 0);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scan_simt(const ScanCore &c, cudaStream_t s) {
    if (c.B * c.H == 0) return cudaSuccess;
    if (c.feat_dtype == HM_F32 && c.io_dtype == HM_F32) return go<float, float>(c, s);
    if (c.feat_dtype == HM_F32 && c.io_dtype == HM_BF16) return go<float, __nv_bfloat16>(c, s);
    if (c.feat_dtype == HM_BF16 && c.io_dtype == HM_F32) return go<__nv_bfloat16, float>(c, s);
    return go<__nv_bfloat16, __nv_bfloat16>(c, s);
}

}  // namespace hm

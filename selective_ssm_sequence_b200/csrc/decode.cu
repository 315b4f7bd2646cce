// decode.cu -- one recurrent decode step per (batch, head), fp32 state.
//
//   S <- a S + phik v^T,  z <- a z + phik,  o = phiq^T S / phiq^T z
//
// (linear-attention tutorial sec. 3 recurrent form and sec. 5 recurrent
// mode for token-by-token inference.)  The step is bound by HBM: the whole
// fp32 state is read and written once.  Each CTA owns one (batch, head) and a
// 64-column tile of the state at a time; its 256 threads each own 4 adjacent columns
// (one 16-byte vector) of every 16th feature row, so a warp touches two full
// 256-byte row segments per access.  All row loads of a thread are issued
// before any arithmetic (16 x 16 B in flight per thread) with streaming
// cache hints, the update is done in registers and written back in place;
// the 16 row-group partial numerators are reduced through shared memory
// while the next tile's loads are already in flight.
// One CTA walks all column tiles of its head, so z (shared by every column)
// is read and rewritten by the same thread with no cross-CTA race.
// The scan's variants are supported: phik times softplus(dt) for the
// step-scaled input, and one decay per feature row with A_log [H, F].
#include "hm_internal.h"

namespace hm {

namespace {

constexpr int kThreads = 256;
constexpr int kCols = 64;          // columns per CTA
constexpr int kColThreads = kCols / 4;
constexpr int kRowGroups = kThreads / kColThreads;  // 16
constexpr int kMaxRowsPerThread = 16;               // F <= 256

__device__ __forceinline__ float4 ld_stream(const float4 *p) {
    float4 r;
    asm volatile("ld.global.cs.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ void st_stream(float4 *p, float4 v) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}

template <typename TF, typename TIO>
__global__ void __launch_bounds__(kThreads)
decode_kernel(int H, int F, int dv, const TF *__restrict__ phq, const TF *__restrict__ phk,
              const TIO *__restrict__ v, const float *__restrict__ dt,
              const float *__restrict__ A_log, float *__restrict__ S, float *__restrict__ z,
              TIO *__restrict__ o, int dt_scaled, int per_feature) {
    __shared__ float sq[256], sk[256], sa[256];
    __shared__ float snum[kRowGroups][kCols];
    __shared__ float sden[kThreads / 32];

    const int64_t bh = blockIdx.x;
    const int h = (int)(bh % H);
    const int tid = threadIdx.x;
    const int cg = tid % kColThreads;   // 4-column group inside a tile
    const int rg = tid / kColThreads;   // row group
    float4 *Sbh = reinterpret_cast<float4 *>(S + bh * (int64_t)F * dv);

    // variants: the step-scaled input multiplies phik by softplus(dt); the
    // per-feature decay takes one rate per (head, feature) from A_log [H, F]
    const float a = (dt && !per_feature) ? expf(hm_log_decay(dt[bh], A_log[h])) : 1.f;
    const float delta = dt_scaled ? hm_step_size(dt[bh]) : 1.f;

    // first tile's state loads go out before anything else
    float4 s[kMaxRowsPerThread];
    {
        const int c0 = cg * 4;
#pragma unroll
        for (int m = 0; m < kMaxRowsPerThread; ++m) {
            int f = rg + kRowGroups * m;
            if (f < F && c0 < dv) s[m] = ld_stream(Sbh + ((int64_t)f * dv + c0) / 4);
        }
    }
    for (int f = tid; f < F; f += kThreads) {
        sq[f] = hm_ld(phq, bh * F + f);
        sk[f] = hm_ld(phk, bh * F + f) * delta;
        sa[f] = per_feature ? expf(hm_log_decay(dt[bh], A_log[(int64_t)h * F + f])) : a;
    }
    __syncthreads();

    // denominator: z' = a z + phik (written back by the thread that read it);
    // den = phiq . z'
    float dpart = 0.f;
    for (int f = tid; f < F; f += kThreads) {
        float zf = fmaf(sa[f], z[bh * F + f], sk[f]);
        dpart = fmaf(sq[f], zf, dpart);
        z[bh * F + f] = zf;
    }
    dpart = warp_sum(dpart);
    if ((tid & 31) == 0) sden[tid >> 5] = dpart;
    __syncthreads();
    float den = 0.f;
#pragma unroll
    for (int i = 0; i < kThreads / 32; ++i) den += sden[i];
    const float inv_den = 1.f / den;

    for (int tile = 0; tile * kCols < dv; ++tile) {
        const int c0 = tile * kCols + cg * 4;
        const bool cols_ok = c0 < dv;  // dv % 4 == 0 (host-checked)
        float4 vv = make_float4(0.f, 0.f, 0.f, 0.f);
        if (cols_ok) {
            vv.x = hm_ld(v, bh * dv + c0 + 0);
            vv.y = hm_ld(v, bh * dv + c0 + 1);
            vv.z = hm_ld(v, bh * dv + c0 + 2);
            vv.w = hm_ld(v, bh * dv + c0 + 3);
        }
        float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < kMaxRowsPerThread; ++m) {
            int f = rg + kRowGroups * m;
            if (f < F && cols_ok) {
                const float kf = sk[f], qf = sq[f], af = sa[f];
                float4 t = s[m];
                t.x = fmaf(af, t.x, kf * vv.x);
                t.y = fmaf(af, t.y, kf * vv.y);
                t.z = fmaf(af, t.z, kf * vv.z);
                t.w = fmaf(af, t.w, kf * vv.w);
                st_stream(Sbh + ((int64_t)f * dv + c0) / 4, t);
                num.x = fmaf(qf, t.x, num.x);
                num.y = fmaf(qf, t.y, num.y);
                num.z = fmaf(qf, t.z, num.z);
                num.w = fmaf(qf, t.w, num.w);
            }
        }
        // the next tile's state rows go out before the reduction of this one
        {
            const int cn = c0 + kCols;
            if (cn < dv) {
#pragma unroll
                for (int m = 0; m < kMaxRowsPerThread; ++m) {
                    int f = rg + kRowGroups * m;
                    if (f < F) s[m] = ld_stream(Sbh + ((int64_t)f * dv + cn) / 4);
                }
            }
        }
        snum[rg][cg * 4 + 0] = num.x;
        snum[rg][cg * 4 + 1] = num.y;
        snum[rg][cg * 4 + 2] = num.z;
        snum[rg][cg * 4 + 3] = num.w;
        __syncthreads();
        if (tid < kCols) {
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < kRowGroups; ++r) acc += snum[r][tid];
            int c = tile * kCols + tid;
            if (c < dv) hm_st(o, bh * dv + c, acc * inv_den);
        }
        __syncthreads();
    }
}

template <typename TF, typename TIO>
cudaError_t go(const DecodeCore &c, cudaStream_t s) {
    dim3 grid((unsigned)(c.B * c.H));
    decode_kernel<TF, TIO><<<grid, kThreads, 0, s>>>(c.H, c.F, c.dv, (const TF *)c.phq,
                                                     (const TF *)c.phk, (const TIO *)c.v, c.dt,
                                                     c.A_log, c.S, c.z, (TIO *)c.o, c.dt_scaled ? 1 : 0,
                                                     c.per_feature ? 1 : 0);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeCore &c, cudaStream_t s) {
    if (c.B * c.H == 0) return cudaSuccess;
    if (c.feat_dtype == HM_F32 && c.io_dtype == HM_F32) return go<float, float>(c, s);
    if (c.feat_dtype == HM_F32 && c.io_dtype == HM_BF16) return go<float, __nv_bfloat16>(c, s);
    if (c.feat_dtype == HM_BF16 && c.io_dtype == HM_F32) return go<__nv_bfloat16, float>(c, s);
    return go<__nv_bfloat16, __nv_bfloat16>(c, s);
}

}  // namespace hm

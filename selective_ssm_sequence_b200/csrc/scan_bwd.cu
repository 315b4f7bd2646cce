// scan_bwd.cu -- gradients of the decayed normalised scan and of the Hedgehog
// feature map on CUDA cores, fp32.
//
// The mixer is trained (HedgeMamba explainer sec. 3: two-stage distillation),
// and Mamba-style scans recompute their states in the backward pass instead
// of storing them (SSM article sec. 4.3).  For L = sum_t do_t . o_t with
//   S_t = a_t S_{t-1} + phik_t v_t^T,  z_t = a_t z_{t-1} + phik_t,
//   n_t = S_t^T phiq_t,  d_t = phiq_t . z_t,  o_t = n_t / d_t
// and dn_t = do_t / d_t, dd_t = -(do_t . o_t) / d_t:
//   dphiq_t = S_t dn_t + z_t dd_t                          (forward in time)
//   G_t = phiq_t dn_t^T + a_{t+1} G_{t+1},  g_t likewise   (backward in time)
//   dphik_t = G_t v_t + g_t,   dv_t = G_t^T phik_t,   dS0 = a_1 G_1, dz0 = a_1 g_1
//   dlog a_t = -sum_{i >= t} phik_i . dphik_i
// The last line holds because o_t is normalised: the factors exp(cum_i) that
// a decay puts on the query side of S_i cancel between n_i and d_i, so only
// the key side of each pair (j < t <= i) carries the gradient, and that is the
// key's phik_j . dphik_j.  It needs neither forward nor backward state, so no
// pass has to hold S and G at once.
//
// Passes, each one CTA per (batch, head, 32 value columns) with the state's
// 256 x 32 slice in registers:
//   PA forward (a thread per feature row): the slice's shares of
//      sum_c do_t[c] n_t[c] and of S_t dn_t
//   PB backward (warp w holds feature rows w, w + 8, ..., lane = column, as
//      in the CUDA-core forward scan): the slice's share of G_t v_t, dv_t, dS0
// and three passes over the denominator's state alone, one CTA per (batch,
// head) with a thread per feature: d_t (before PA), then z_t dd_t (once PA has
// given do_t . n_t), then g_t and dz0, written as one more share.  Keeping z
// out of the value-slice passes halves their registers, so two of their CTAs
// fit on an SM, and PA needs only d_t, not dd_t.
// then a reduction of the slices' shares (and the suffix sums of dlog a),
// the feature-map backward (softmax Jacobian, dx = du W, dW = sum du x^T) and
// the decay's (d dt = dlog a (-sigmoid(dt) e^A_log), dA_log = sum dlog a * log a).
#include "hm_internal.h"

namespace hm {

namespace {

constexpr int kW = 8;        // warps
constexpr int kTB = 16;      // tokens staged per round
constexpr int kMaxRows = 32; // F <= 256

struct BwdArgs {
    int64_t B, L;
    int H, F, dv, ns;        // ns = column slices (dv / 32, rounded up)
    const float *phq, *phk;  // [B, L, H, F] fp32
    const void *v;           // [B, L, H, dv] of io dtype
    const void *dout;        // [B, L, H, dv] of io dtype
    const float *dt, *A_log;
    const float *S0, *z0;
    float *den;              // [B, L, H]
    float *e_part;           // [ns][B, L, H]: slices' shares of do . n
    float *dq_part, *dk_part;   // [ns + 1][B, L, H, F]: the slices' shares, then the denominator's
    float *dv_out;           // [B, L, H, dv] fp32
    float *dS0, *dz0;        // nullable
};

// v[m] is this lane's contribution to row m (m = 0..31); afterwards v[0] of
// lane l is the sum over the warp of row l.  Recursive halving: at step `off`
// each lane keeps the half of its rows selected by its lane bit `off` and
// adds the partner's copy of that half (31 shuffles instead of 32 reductions
// of 5).
__device__ __forceinline__ float warp_reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int j = 0; j < off; ++j) {
            const float send = upper ? v[j] : v[j + off];
            const float keep = upper ? v[j + off] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return v[0];
}

// PB, tokens from the last to the first (the state layout of the forward
// CUDA-core scan: warp w holds feature rows w, w + 8, ..., lane = column).
template <typename TIO>
__global__ void __launch_bounds__(32 * kW, 2)
bwd_pb_kernel(BwdArgs a) {
    extern __shared__ float smem[];
    const int F = a.F, dv = a.dv;
    float *sq = smem;                      // [kTB][F]
    float *sk = sq + kTB * F;              // [kTB][F]
    float *sv = sk + kTB * F;              // [kTB][32]   v
    float *sg = sv + kTB * 32;             // [kTB][32]   do
    float *sa = sg + kTB * 32;             // [kTB]       a_t
    float *sa1 = sa + kTB;                 // [kTB]       a_{t+1} (PB)
    float *sden = sa1 + kTB;               // [kTB]
    float *red = sden + kTB;               // [kTB][kW][32]
    float *sout = red + kTB * kW * 32;     // [kTB][F]: the slice's shares of dphiq / dphik

    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t bh = blockIdx.y;
    const int64_t b = bh / a.H;
    const int h = (int)(bh % a.H);
    const int slice = blockIdx.x;
    const int col = slice * 32 + lane;
    const bool col_ok = col < dv;
    const float alog = a.dt ? a.A_log[h] : 0.f;
    const TIO *v = (const TIO *)a.v;
    const TIO *dout = (const TIO *)a.dout;
    const int64_t L = a.L;
    auto rowi = [&](int64_t t) { return (b * L + t) * a.H + h; };

    float S[kMaxRows];   // G, the adjoint of S, from zero after the last token
#pragma unroll
    for (int m = 0; m < kMaxRows; ++m) S[m] = 0.f;
    const int64_t nblk = (L + kTB - 1) / kTB;
    for (int64_t bi = 0; bi < nblk; ++bi) {
        // PB walks the token blocks from the last to the first
        const int64_t t0 = (nblk - 1 - bi) * kTB;
        const int nt = (int)((L - t0) < kTB ? (L - t0) : kTB);
        for (int i = threadIdx.x; i < nt * F; i += blockDim.x) {
            const int t = i / F, f = i % F;
            sq[i] = a.phq[rowi(t0 + t) * F + f];
            sk[i] = a.phk[rowi(t0 + t) * F + f];
        }
        for (int i = threadIdx.x; i < nt * 32; i += blockDim.x) {
            const int t = i / 32, c = slice * 32 + (i % 32);
            const bool ok = c < dv;
            sv[i] = ok ? hm_ld(v, rowi(t0 + t) * dv + c) : 0.f;
            sg[i] = ok ? hm_ld(dout, rowi(t0 + t) * dv + c) : 0.f;
        }
        if (threadIdx.x < nt) {
            const int t = threadIdx.x;
            const int64_t r = rowi(t0 + t);
            sa[t] = a.dt ? expf(hm_log_decay(a.dt[r], alog)) : 1.f;
            // a_{t+1}: the decay that carries G_{t+1} back to token t (none after the last token)
            sa1[t] = (t0 + t + 1 < L && a.dt) ? expf(hm_log_decay(a.dt[rowi(t0 + t + 1)], alog)) : 1.f;
            sden[t] = a.den[r];
        }
        __syncthreads();
        {
            // PB: G_t = phiq_t dn_t^T + a_{t+1} G_{t+1} (S holds G)
            for (int t = nt - 1; t >= 0; --t) {
                const float a1 = sa1[t];
                const float dn = sg[t * 32 + lane] / sden[t];
                const float vv = sv[t * 32 + lane];
                float dvp = 0.f;
                float x[kMaxRows];
#pragma unroll
                for (int m = 0; m < kMaxRows; ++m) {
                    const int f = w + kW * m;
                    x[m] = 0.f;
                    if (f < F) {
                        const float qf = sq[t * F + f], kf = sk[t * F + f];
                        S[m] = fmaf(a1, S[m], qf * dn);
                        dvp = fmaf(S[m], kf, dvp);
                        x[m] = S[m] * vv;
                    }
                }
                // the slice's share of sum_c G_t[f, c] v_t[c]
                const float tot = warp_reduce_scatter32(x, lane);
                const int fl = w + kW * lane;
                if (fl < F) sout[t * F + fl] = tot;
                red[(t * kW + w) * 32 + lane] = dvp;
            }
            __syncthreads();
            for (int i = threadIdx.x; i < nt * 32; i += blockDim.x) {
                const int t = i / 32, c = i % 32;
                float acc = 0.f;
                for (int ww = 0; ww < kW; ++ww) acc += red[(t * kW + ww) * 32 + c];
                const int cc = slice * 32 + c;
                if (cc < dv) a.dv_out[rowi(t0 + t) * dv + cc] = acc;
            }
            {
                float *dk = a.dk_part + (int64_t)slice * a.B * L * a.H * F;
                for (int i = threadIdx.x; i < nt * F; i += blockDim.x)
                    dk[rowi(t0 + i / F) * F + (i % F)] = sout[i];
            }
            if (t0 == 0 && a.dS0 && col_ok) {
                // dS0 = a_1 G_1 (a_1 = the first token's decay)
                const float a0 = sa[0];
#pragma unroll
                for (int m = 0; m < kMaxRows; ++m) {
                    const int f = w + kW * m;
                    if (f < F) a.dS0[(bh * F + f) * dv + col] = a0 * S[m];
                }
            }
        }
        __syncthreads();
    }
}

// PA with a thread per feature row (the 32 columns of the slice in its
// registers): S_t[f, :] = a_t S_(t-1)[f, :] + phik_t[f] v_t and
// u_f = sum_c S_t[f, c] do_t[c] stay within the thread; the slice's share of
// dphiq_t[f] is u_f / d_t and its share of do_t . n_t = sum_f phiq_t[f] u_f
// is one block reduction per token.
template <typename TIO>
__global__ void __launch_bounds__(256, 2)
bwd_pa_kernel(BwdArgs a) {
    extern __shared__ float smem[];
    const int F = a.F, dv = a.dv;
    float *sq = smem;                      // [kTB][F]
    float *sk = sq + kTB * F;              // [kTB][F]
    float *sv = sk + kTB * F;              // [kTB][32]   v
    float *sg = sv + kTB * 32;             // [kTB][32]   do
    float *sa = sg + kTB * 32;             // [kTB]       a_t
    float *sden = sa + kTB;                // [kTB]
    float *red = sden + kTB;               // [kTB][kW]
    float *sout = red + kTB * kW;          // [kTB][F]

    const int f = threadIdx.x, lane = f & 31, w = f >> 5;
    const bool fok = f < F;
    const int64_t bh = blockIdx.y;
    const int64_t b = bh / a.H;
    const int h = (int)(bh % a.H);
    const int slice = blockIdx.x;
    const int c0 = slice * 32;
    const int ncol = dv - c0 < 32 ? dv - c0 : 32;
    const float alog = a.dt ? a.A_log[h] : 0.f;
    const TIO *v = (const TIO *)a.v;
    const TIO *dout = (const TIO *)a.dout;
    const int64_t L = a.L;
    const int64_t rows = a.B * L * a.H;
    auto rowi = [&](int64_t t) { return (b * L + t) * a.H + h; };

    float S[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) S[c] = (a.S0 && fok && c < ncol) ? a.S0[(bh * F + f) * dv + c0 + c] : 0.f;
    const int64_t nblk = (L + kTB - 1) / kTB;
    for (int64_t bi = 0; bi < nblk; ++bi) {
        const int64_t t0 = bi * kTB;
        const int nt = (int)((L - t0) < kTB ? (L - t0) : kTB);
        for (int i = threadIdx.x; i < nt * F; i += blockDim.x) {
            const int t = i / F, ff = i % F;
            sq[i] = a.phq[rowi(t0 + t) * F + ff];
            sk[i] = a.phk[rowi(t0 + t) * F + ff];
        }
        for (int i = threadIdx.x; i < nt * 32; i += blockDim.x) {
            const int t = i / 32, c = i % 32;
            const bool ok = c < ncol;
            sv[i] = ok ? hm_ld(v, rowi(t0 + t) * dv + c0 + c) : 0.f;
            sg[i] = ok ? hm_ld(dout, rowi(t0 + t) * dv + c0 + c) : 0.f;
        }
        if (threadIdx.x < nt) {
            const int64_t r = rowi(t0 + threadIdx.x);
            sa[threadIdx.x] = a.dt ? expf(hm_log_decay(a.dt[r], alog)) : 1.f;
            sden[threadIdx.x] = a.den[r];
        }
        __syncthreads();
        for (int t = 0; t < nt; ++t) {
            const float at = sa[t];
            const float kf = fok ? sk[t * F + f] : 0.f;
            float u = 0.f;
            const float4 *v4 = reinterpret_cast<const float4 *>(sv + t * 32);
            const float4 *g4 = reinterpret_cast<const float4 *>(sg + t * 32);
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
                const float4 vv = v4[c4], gg = g4[c4];
                S[4 * c4 + 0] = fmaf(at, S[4 * c4 + 0], kf * vv.x);
                S[4 * c4 + 1] = fmaf(at, S[4 * c4 + 1], kf * vv.y);
                S[4 * c4 + 2] = fmaf(at, S[4 * c4 + 2], kf * vv.z);
                S[4 * c4 + 3] = fmaf(at, S[4 * c4 + 3], kf * vv.w);
                u = fmaf(S[4 * c4 + 0], gg.x, u);
                u = fmaf(S[4 * c4 + 1], gg.y, u);
                u = fmaf(S[4 * c4 + 2], gg.z, u);
                u = fmaf(S[4 * c4 + 3], gg.w, u);
            }
            if (fok) sout[t * F + f] = u / sden[t];
            const float ep = warp_sum(fok ? sq[t * F + f] * u : 0.f);
            if (lane == 0) red[t * kW + w] = ep;
        }
        __syncthreads();
        float *dq = a.dq_part + (int64_t)slice * rows * F;
        for (int i = threadIdx.x; i < nt * F; i += blockDim.x) dq[rowi(t0 + i / F) * F + (i % F)] = sout[i];
        if (threadIdx.x < nt) {
            float e = 0.f;
#pragma unroll
            for (int ww = 0; ww < kW; ++ww) e += red[threadIdx.x * kW + ww];
            a.e_part[(int64_t)slice * rows + rowi(t0 + threadIdx.x)] = e;
        }
        __syncthreads();
    }
}

// The denominator's state z alone, one CTA per (batch, head), thread f =
// feature f (the same three passes as above):
//   MODE 0 forward:  z_t = a_t z_(t-1) + phik_t, d_t = phiq_t . z_t
//   MODE 1 forward:  z_t again; its share of dphiq_t is z_t dd_t
//   MODE 2 backward: g_t = a_(t+1) g_(t+1) + phiq_t dd_t, its share of dphik_t;
//                    dz0 = a_1 g_1
// The shares go to plane ns of dq_part / dk_part, after the value slices'.
template <int MODE>
__global__ void __launch_bounds__(256)
bwd_z_kernel(BwdArgs a) {
    __shared__ float sa[kTB], sa1[kTB], sdd[kTB];
    __shared__ float red[kTB][kW];
    const int f = threadIdx.x, lane = f & 31, w = f >> 5;
    const int64_t bh = blockIdx.x;
    const int64_t b = bh / a.H;
    const int h = (int)(bh % a.H);
    const int F = a.F;
    const bool fok = f < F;
    const float alog = a.dt ? a.A_log[h] : 0.f;
    const int64_t L = a.L;
    const int64_t rows = a.B * L * a.H;
    auto rowi = [&](int64_t t) { return (b * L + t) * a.H + h; };
    float zs = (MODE < 2 && a.z0 && fok) ? a.z0[bh * F + f] : 0.f;
    const int64_t nblk = (L + kTB - 1) / kTB;
    for (int64_t bi = 0; bi < nblk; ++bi) {
        const int64_t t0 = (MODE == 2 ? nblk - 1 - bi : bi) * kTB;
        const int nt = (int)((L - t0) < kTB ? (L - t0) : kTB);
        __syncthreads();
        if (threadIdx.x < nt) {
            const int t = threadIdx.x;
            const int64_t r = rowi(t0 + t);
            sa[t] = a.dt ? expf(hm_log_decay(a.dt[r], alog)) : 1.f;
            sa1[t] = (t0 + t + 1 < L && a.dt) ? expf(hm_log_decay(a.dt[rowi(t0 + t + 1)], alog)) : 1.f;
            if (MODE >= 1) {
                const float d = a.den[r];
                float e = 0.f;
                for (int s = 0; s < a.ns; ++s) e += a.e_part[(int64_t)s * rows + r];
                sdd[t] = -e / (d * d);   // dd = -(do . o) / d = -(do . n) / d^2
            }
        }
        __syncthreads();
        // the block's features of this thread, all loads in flight at once
        float xk[kTB], xq[kTB];
#pragma unroll
        for (int t = 0; t < kTB; ++t) {
            const bool ok = fok && t < nt;
            xk[t] = (MODE < 2 && ok) ? a.phk[rowi(t0 + t) * F + f] : 0.f;
            xq[t] = (MODE != 1 && ok) ? a.phq[rowi(t0 + t) * F + f] : 0.f;
        }
        if (MODE < 2) {
#pragma unroll
            for (int t = 0; t < kTB; ++t) {
                if (t >= nt) break;
                zs = fmaf(sa[t], zs, xk[t]);
                if (MODE == 0) {
                    const float p = warp_sum(xq[t] * zs);
                    if (lane == 0) red[t][w] = p;
                } else if (fok) {
                    a.dq_part[(int64_t)a.ns * rows * F + rowi(t0 + t) * F + f] = zs * sdd[t];
                }
            }
            if (MODE == 0) {
                __syncthreads();
                if (threadIdx.x < nt) {
                    float d = 0.f;
#pragma unroll
                    for (int ww = 0; ww < kW; ++ww) d += red[threadIdx.x][ww];
                    a.den[rowi(t0 + threadIdx.x)] = d;
                }
            }
        } else {
#pragma unroll
            for (int t = kTB - 1; t >= 0; --t) {
                if (t >= nt) continue;
                zs = fmaf(sa1[t], zs, xq[t] * sdd[t]);
                if (fok) a.dk_part[(int64_t)a.ns * rows * F + rowi(t0 + t) * F + f] = zs;
            }
            if (t0 == 0 && a.dz0 && fok) a.dz0[bh * F + f] = sa[0] * zs;
        }
    }
}

// dphiq, dphik = sums of the slices' shares, and kd_r = phik_r . dphik_r;
// one warp per row (lanes over the features).
__global__ void __launch_bounds__(256)
bwd_reduce_kernel(BwdArgs a, float *__restrict__ dphq, float *__restrict__ dphk, float *__restrict__ kd) {
    const int lane = threadIdx.x & 31;
    const int64_t rows = a.B * a.L * a.H;
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (r >= rows) return;
    const int64_t plane = rows * (int64_t)a.F;
    float acc = 0.f;
    for (int f = lane; f < a.F; f += 32) {
        float sq = 0.f, sk = 0.f;
        for (int s = 0; s <= a.ns; ++s) {
            sq += a.dq_part[s * plane + r * a.F + f];
            sk += a.dk_part[s * plane + r * a.F + f];
        }
        dphq[r * a.F + f] = sq;
        dphk[r * a.F + f] = sk;
        acc = fmaf(a.phk[r * a.F + f], sk, acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) kd[r] = acc;
}

// dlog a_t = -sum_{i >= t} kd_i per (b, h): one warp per (b, h) walks the
// tokens from the end in blocks of 32 with a warp suffix scan.
__global__ void __launch_bounds__(256)
bwd_suffix_kernel(int64_t B, int64_t L, int H, const float *__restrict__ kd, float *__restrict__ dla) {
    const int lane = threadIdx.x & 31;
    const int64_t bh = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (bh >= B * H) return;
    const int64_t b = bh / H;
    const int h = (int)(bh % H);
    float carry = 0.f;
    for (int64_t tb = L - 1; tb >= 0; tb -= 32) {
        const int64_t t = tb - lane;   // lane 0 = the latest token of the block
        float x = t >= 0 ? kd[(b * L + t) * H + h] : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (t >= 0) dla[(b * L + t) * H + h] = -(carry + x);
        carry += __shfl_sync(0xffffffffu, x, 31);
    }
}

// fp32 copy of caller-supplied features (for the passes above).
template <typename T>
__global__ void to_f32_kernel(const T *__restrict__ x, int64_t n, float *__restrict__ y) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) y[i] = hm_ld(x, i);
}

// Feature-map backward, per row: phi = softmax([u, -u]), so
// de = phi (.) (dphi - sum(phi (.) dphi)), du = de[:p] - de[p:].  One warp per row.
__global__ void __launch_bounds__(256)
featmap_bwd_du_kernel(const float *__restrict__ phi, const float *__restrict__ dphi, int64_t rows, int p,
                      float *__restrict__ du) {
    const int lane = threadIdx.x & 31;
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (r >= rows) return;
    const float *ph = phi + r * 2 * p, *dp = dphi + r * 2 * p;
    float s = 0.f;
    for (int f = lane; f < 2 * p; f += 32) s = fmaf(ph[f], dp[f], s);
    s = warp_sum(s);
    for (int j = lane; j < p; j += 32)
        du[r * p + j] = ph[j] * (dp[j] - s) - ph[p + j] * (dp[p + j] - s);
}

// Four consecutive elements of a row as fp32; `valid` of them in bounds (the
// rest read as 0).  vec: rows start 16-byte (fp32) / 8-byte (bf16) aligned.
__device__ __forceinline__ float4 ld4(const float *p, int64_t i, int valid, bool vec) {
    if (vec && valid >= 4) return *reinterpret_cast<const float4 *>(p + i);
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
    if (valid > 0) r.x = p[i];
    if (valid > 1) r.y = p[i + 1];
    if (valid > 2) r.z = p[i + 2];
    if (valid > 3) r.w = p[i + 3];
    return r;
}

__device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p, int64_t i, int valid, bool vec) {
    if (vec && valid >= 4) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p + i);
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
        return make_float4(lo.x, lo.y, hi.x, hi.y);
    }
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
    if (valid > 0) r.x = __bfloat162float(p[i]);
    if (valid > 1) r.y = __bfloat162float(p[i + 1]);
    if (valid > 2) r.z = __bfloat162float(p[i + 2]);
    if (valid > 3) r.w = __bfloat162float(p[i + 3]);
    return r;
}

// The feature map's two gradient products, dx = du W and dW = du^T x, as one
// register-tiled fp32 contraction C (+)= A B on the CUDA cores: a CTA owns a
// 128 x 128 tile of C and each thread an 8 x 8 block of it (rows ty*4.. and
// 64 + ty*4.., columns tx*4.. and 64 + tx*4..), fed from 16-deep slices of A
// and B in double-buffered shared memory; the next slice's global loads are in
// flight while the current one's 16 x 64 FMAs run, and each FMA step reads two
// float4 of A and two of B (four shared loads for 64 FMAs).
// A is [k][m] (m contiguous; dW, where A = du^T) or, with A_MK, [m][k]
// (dx, A = du), transposed on its way into shared memory; B is [k][n] with n
// contiguous; C is [m][n].  Grid: (m tiles, n tiles, k splits); with SPLIT each
// CTA covers kchunk of k and adds its tile to C (zeroed first) atomically.
// vec: every leading dimension is a multiple of 4, so groups of 4 that are
// fully in bounds use vector loads, stores and atomics.
constexpr int kGM = 128, kGN = 128, kGK = 16, kGS = 132;   // kGS: padded smem row

template <bool A_MK, typename TB, bool SPLIT>
__global__ void __launch_bounds__(256, 2)
featmap_bwd_gemm_kernel(const float *__restrict__ A, int64_t lda, const TB *__restrict__ Bm, int64_t ldb,
                        float *__restrict__ C, int64_t ldc, int64_t M, int64_t N, int64_t K, int64_t kchunk,
                        bool vec) {
    __shared__ __align__(16) float As[2][kGK][kGS];
    __shared__ __align__(16) float Bs[2][kGK][kGS];
    const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
    const int64_t m0 = (int64_t)blockIdx.x * kGM, n0 = (int64_t)blockIdx.y * kGN;
    const int64_t kb = SPLIT ? (int64_t)blockIdx.z * kchunk : 0;
    const int64_t ke = SPLIT ? (kb + kchunk < K ? kb + kchunk : K) : K;
    auto nvalid = [](int64_t lim, int64_t col) { return (int)(lim - col >= 4 ? 4 : (lim > col ? lim - col : 0)); };
    // this thread's two groups of 4 in each slice: A (and, with A_MK, its row
    // bound) and B at slice start k = 0; a slice at k0 adds k0 (A_MK) or
    // k0 * ld to the pointer
    const float *pa[2];
    const TB *pb[2];
    int64_t acol[2];
    bool arow_ok[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int g = t + 256 * u;
        if (A_MK) {   // four lanes per row of A: 64 contiguous bytes
            const int64_t row = m0 + (g >> 2);
            acol[u] = 4 * (g & 3);
            arow_ok[u] = row < M;
            pa[u] = A + row * lda + acol[u];
        } else {
            acol[u] = m0 + 4 * (g & 31);
            arow_ok[u] = true;
            pa[u] = A + (int64_t)(g >> 5) * lda + acol[u];
        }
        pb[u] = Bm + (int64_t)(g >> 5) * ldb + n0 + 4 * (g & 31);
    }
    const int bval = nvalid(N, n0 + 4 * (t & 31));
    float4 ra[2], rb[2];
    auto load = [&](int64_t k0) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t krow = k0 + (t >> 5) + 8 * u;   // the B row (and A row without A_MK)
            if (A_MK)
                ra[u] = ld4(pa[u] + k0, 0, arow_ok[u] ? nvalid(ke, k0 + acol[u]) : 0, vec);
            else
                ra[u] = ld4(pa[u] + k0 * lda, 0, krow < ke ? nvalid(M, acol[u]) : 0, vec);
            rb[u] = ld4(pb[u] + k0 * ldb, 0, krow < ke ? bval : 0, vec);
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int g = t + 256 * u;
            if (A_MK) {
                const int m = g >> 2, k = 4 * (g & 3);
                As[buf][k][m] = ra[u].x;
                As[buf][k + 1][m] = ra[u].y;
                As[buf][k + 2][m] = ra[u].z;
                As[buf][k + 3][m] = ra[u].w;
            } else {
                *reinterpret_cast<float4 *>(&As[buf][g >> 5][4 * (g & 31)]) = ra[u];
            }
            *reinterpret_cast<float4 *>(&Bs[buf][g >> 5][4 * (g & 31)]) = rb[u];
        }
    };
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    const int nst = ke > kb ? (int)((ke - kb + kGK - 1) / kGK) : 0;
    if (nst == 0) return;   // (a split past the end; the launcher makes none)
    load(kb);
    store(0);
    __syncthreads();
    for (int s = 0; s < nst; ++s) {
        const int cur = s & 1;
        if (s + 1 < nst) load(kb + (int64_t)(s + 1) * kGK);
#pragma unroll
        for (int k = 0; k < kGK; ++k) {
            const float4 a0 = *reinterpret_cast<const float4 *>(&As[cur][k][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4 *>(&As[cur][k][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[cur][k][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[cur][k][64 + tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        if (s + 1 < nst) store(cur ^ 1);
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t row = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
        if (row >= M) continue;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t col = n0 + h * 64 + tx * 4;
            const int valid = nvalid(N, col);
            float *dst = C + row * ldc + col;
            const float4 v = make_float4(acc[i][4 * h], acc[i][4 * h + 1], acc[i][4 * h + 2], acc[i][4 * h + 3]);
            if (vec && valid == 4) {
                if (SPLIT)
                    atomicAdd(reinterpret_cast<float4 *>(dst), v);
                else
                    *reinterpret_cast<float4 *>(dst) = v;
            } else {
                const float ve[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (e < valid) {
                        if (SPLIT)
                            atomicAdd(dst + e, ve[e]);
                        else
                            dst[e] = ve[e];
                    }
            }
        }
    }
}

// dx = du W ([rows, p] x [p, d]) and dW = du^T x ([p, rows] x [rows, d], k
// split so that about two CTAs per SM run; dW is zeroed first).
template <typename T>
cudaError_t run_featmap_bwd_products(const float *du, const T *W, const T *x, int64_t rows, int p, int d,
                                     float *dx, float *dW, cudaStream_t s) {
    const bool vec = p % 4 == 0 && d % 4 == 0;
    const unsigned nt = (unsigned)((d + kGN - 1) / kGN);
    dim3 gx((unsigned)((rows + kGM - 1) / kGM), nt, 1);
    featmap_bwd_gemm_kernel<true, T, false><<<gx, 256, 0, s>>>(du, p, W, d, dx, d, rows, d, p, p, vec);
    cudaError_t e = cudaMemsetAsync(dW, 0, sizeof(float) * (size_t)p * d, s);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t mt = (p + kGM - 1) / kGM;
    const int64_t want = (2 * (int64_t)sms + mt * nt - 1) / (mt * nt);
    int64_t kchunk = (rows + want - 1) / want;
    kchunk = (kchunk + kGK - 1) / kGK * kGK;
    dim3 gw((unsigned)mt, nt, (unsigned)((rows + kchunk - 1) / kchunk));
    featmap_bwd_gemm_kernel<false, T, true><<<gw, 256, 0, s>>>(du, p, x, d, dW, d, p, d, rows, kchunk, vec);
    count_launches(2);
    return cudaGetLastError();
}

// d dt = dlog a * (-sigmoid(dt) e^A_log);  dA_log[h] += sum dlog a * log a.
__global__ void __launch_bounds__(256)
decay_bwd_kernel(const float *__restrict__ dt, const float *__restrict__ A_log, const float *__restrict__ dla,
                 int64_t BL, int H, float *__restrict__ ddt, float *__restrict__ dA) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    float contrib = 0.f;
    int h = 0;
    if (i < BL * H) {
        h = (int)(i % H);
        const float x = dt[i], rate = expf(A_log[h]);
        const float sig = 1.f / (1.f + expf(-x));
        ddt[i] = dla[i] * (-sig * rate);
        contrib = dla[i] * hm_log_decay(x, A_log[h]);
    }
    // lanes of a warp may hold different heads: one addition per element
    if (i < BL * H) atomicAdd(&dA[h], contrib);
}

template <typename TIO>
cudaError_t run_passes(const BwdArgs &a, cudaStream_t s) {
    dim3 grid((unsigned)a.ns, (unsigned)(a.B * a.H));
    const size_t smem = sizeof(float) * (size_t)(3 * kTB * a.F + 2 * kTB * 32 + 3 * kTB + kTB * kW * 32);
    cudaError_t e;
    auto k1 = bwd_pa_kernel<TIO>;
    auto k2 = bwd_pb_kernel<TIO>;
    const size_t smem1 = sizeof(float) * (size_t)(3 * kTB * a.F + 2 * kTB * 32 + 2 * kTB + kTB * kW);
    e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned zgrid = (unsigned)(a.B * a.H);
    bwd_z_kernel<0><<<zgrid, 256, 0, s>>>(a);
    k1<<<grid, 256, smem1, s>>>(a);
    bwd_z_kernel<1><<<zgrid, 256, 0, s>>>(a);
    k2<<<grid, 32 * kW, smem, s>>>(a);
    bwd_z_kernel<2><<<zgrid, 256, 0, s>>>(a);
    count_launches(5);
    return cudaGetLastError();
}

}  // namespace

size_t scan_bwd_workspace(const ScanBwdCore &c) {
    const int ns = (c.dv + 31) / 32;
    const size_t rows = (size_t)c.B * c.L * c.H;
    auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
    size_t n = 0;
    n += 2 * r256(rows * c.F * 4);             // phq, phk (fp32)
    n += r256(rows * 4);                       // den
    n += r256((size_t)ns * rows * 4);          // e_part
    n += 2 * r256((size_t)(ns + 1) * rows * c.F * 4);  // dq_part, dk_part
    n += 2 * r256(rows * c.F * 4);             // dphq, dphk
    n += 2 * r256(rows * 4);                   // kd, dlog a
    if (c.W_q) n += r256(rows * c.p * 4);      // du
    return n;
}

cudaError_t launch_scan_bwd(const ScanBwdCore &c, void *ws, cudaStream_t s) {
    const int ns = (c.dv + 31) / 32;
    const int64_t rows = c.B * c.L * c.H;
    if (rows == 0) {
        // no token reaches an output: the gradients of the weights, of A_log
        // and of the initial state are zero
        const size_t BH = (size_t)c.B * c.H;
        cudaError_t e = cudaSuccess;
        if (c.W_q && c.dW_q) e = cudaMemsetAsync(c.dW_q, 0, sizeof(float) * (size_t)c.p * c.d, s);
        if (e == cudaSuccess && c.W_q && c.dW_k) e = cudaMemsetAsync(c.dW_k, 0, sizeof(float) * (size_t)c.p * c.d, s);
        if (e == cudaSuccess && c.A_log && c.dA_log) e = cudaMemsetAsync(c.dA_log, 0, sizeof(float) * (size_t)c.H, s);
        if (e == cudaSuccess && c.dS0 && BH > 0) {
            e = cudaMemsetAsync(c.dS0, 0, sizeof(float) * BH * c.F * c.dv, s);
            if (e == cudaSuccess) e = cudaMemsetAsync(c.dz0, 0, sizeof(float) * BH * c.F, s);
        }
        return e;
    }
    auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
    char *w = (char *)ws;
    auto take = [&](size_t bytes) { char *p = w; w += r256(bytes); return p; };
    float *phq = (float *)take(rows * c.F * 4), *phk = (float *)take(rows * c.F * 4);
    BwdArgs a{};
    a.B = c.B; a.L = c.L; a.H = c.H; a.F = c.F; a.dv = c.dv; a.ns = ns;
    a.phq = phq; a.phk = phk; a.v = c.v; a.dout = c.dout; a.dt = c.dt; a.A_log = c.A_log;
    a.S0 = c.S0; a.z0 = c.z0;
    a.den = (float *)take(rows * 4);
    a.e_part = (float *)take((size_t)ns * rows * 4);
    a.dq_part = (float *)take((size_t)(ns + 1) * rows * c.F * 4);
    a.dk_part = (float *)take((size_t)(ns + 1) * rows * c.F * 4);
    float *dphq = (float *)take(rows * c.F * 4), *dphk = (float *)take(rows * c.F * 4);
    float *kd = (float *)take(rows * 4);
    float *dla = (float *)take(rows * 4);
    float *du = c.W_q ? (float *)take(rows * c.p * 4) : nullptr;
    a.dv_out = c.dv_out;
    a.dS0 = c.dS0;
    a.dz0 = c.dz0;
    cudaError_t e;
    // the features in fp32: the Hedgehog maps, or the caller's features
    if (c.W_q) {
        e = run_featmap_f32(c.q, c.io_dtype, rows, c.H, c.d, c.p, c.W_q, phq, s);
        if (e == cudaSuccess) e = run_featmap_f32(c.k, c.io_dtype, rows, c.H, c.d, c.p, c.W_k, phk, s);
    } else {
        const int64_t n = rows * c.F;
        const unsigned nb = (unsigned)((n + 255) / 256);
        if (c.io_dtype == HM_BF16) {
            to_f32_kernel<__nv_bfloat16><<<nb, 256, 0, s>>>((const __nv_bfloat16 *)c.q, n, phq);
            to_f32_kernel<__nv_bfloat16><<<nb, 256, 0, s>>>((const __nv_bfloat16 *)c.k, n, phk);
        } else {
            to_f32_kernel<float><<<nb, 256, 0, s>>>((const float *)c.q, n, phq);
            to_f32_kernel<float><<<nb, 256, 0, s>>>((const float *)c.k, n, phk);
        }
        count_launches(2);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    e = c.io_dtype == HM_BF16 ? run_passes<__nv_bfloat16>(a, s) : run_passes<float>(a, s);
    if (e != cudaSuccess) return e;
    const unsigned wb = (unsigned)((rows * 32 + 255) / 256);
    bwd_reduce_kernel<<<wb, 256, 0, s>>>(a, dphq, dphk, kd);
    bwd_suffix_kernel<<<(unsigned)((c.B * c.H * 32 + 255) / 256), 256, 0, s>>>(c.B, c.L, c.H, kd, dla);
    count_launches(2);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (c.W_q) {
        const float *dphis[2] = {dphq, dphk};
        const float *phis[2] = {phq, phk};
        const void *xs[2] = {c.q, c.k};
        const void *Ws[2] = {c.W_q, c.W_k};
        float *dxs[2] = {c.dq, c.dk};
        float *dWs[2] = {c.dW_q, c.dW_k};
        for (int m = 0; m < 2; ++m) {
            featmap_bwd_du_kernel<<<wb, 256, 0, s>>>(phis[m], dphis[m], rows, c.p, du);
            count_launches(1);
            e = c.io_dtype == HM_BF16
                    ? run_featmap_bwd_products(du, (const __nv_bfloat16 *)Ws[m], (const __nv_bfloat16 *)xs[m], rows,
                                               c.p, c.d, dxs[m], dWs[m], s)
                    : run_featmap_bwd_products(du, (const float *)Ws[m], (const float *)xs[m], rows, c.p, c.d,
                                               dxs[m], dWs[m], s);
            if (e != cudaSuccess) return e;
        }
    } else {
        // caller features: their gradients are dphiq and dphik
        e = cudaMemcpyAsync(c.dq, dphq, (size_t)rows * c.F * 4, cudaMemcpyDeviceToDevice, s);
        if (e == cudaSuccess) e = cudaMemcpyAsync(c.dk, dphk, (size_t)rows * c.F * 4, cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return e;
    }
    if (c.dt) {
        e = cudaMemsetAsync(c.dA_log, 0, sizeof(float) * (size_t)c.H, s);
        if (e != cudaSuccess) return e;
        const int64_t BL = c.B * c.L;
        decay_bwd_kernel<<<(unsigned)((BL * c.H + 255) / 256), 256, 0, s>>>(c.dt, c.A_log, dla, BL, c.H, c.ddt,
                                                                         c.dA_log);
        count_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace hm

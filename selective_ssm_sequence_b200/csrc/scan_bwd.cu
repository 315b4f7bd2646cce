// scan_bwd.cu -- gradients of the decayed normalised scan and of the Hedgehog
// feature map: the recurrences on CUDA cores in fp32, the feature map's two
// gradient products (dx = du W, dW = du^T x) on the tensor cores over du split
// into bf16 hi and lo parts where the shapes allow.
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
// Passes, each one CTA per (batch, head, 32 value columns), token blocks of
// 16 copied by cp.async one block ahead:
//   PA forward (a thread per feature row, the slice's 32 columns of S in its
//      registers): the slice's shares of sum_c do_t[c] n_t[c] and of S_t dn_t;
//      the denominator's state z rides along (a thread per feature), so PA
//      also gives d_t
//   PB backward (each thread an 8 x 4 block of the slice's G): the slice's
//      share of G_t v_t, dv_t and dS0
// and two passes over the denominator's state alone, one CTA per (batch,
// head), run as extra CTAs of PB's launch: z_t dd_t (once PA has given
// do_t . n_t and d_t), and g_t and dz0, each written as one more share.
// Keeping z out of PB halves its registers, so two of its CTAs fit on an SM.
// Then a reduction of the slices' shares (and the suffix sums of dlog a),
// the feature-map backward (softmax Jacobian, dx = du W, dW = sum du x^T) and
// the decay's (d dt = dlog a (-sigmoid(dt) e^A_log), dA_log = sum dlog a * log a).
#include "hm_internal.h"
#include "tc_common.cuh"

namespace hm {

namespace {

constexpr int kW = 8;        // warps
constexpr int kTB = 16;      // tokens staged per round

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

// ------------------------------------------------------------ token blocks

constexpr int kFP = 256;   // feature stride of a staged row (F <= 256; zero past F)

// cp.async: 16 or 4 bytes global -> shared; the bytes past src_bytes are
// zero-filled (src_bytes = 0 reads nothing).
__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src, int src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

template <typename T>
__device__ __forceinline__ T zero_of() { return T(0.f); }
template <>
__device__ __forceinline__ __nv_bfloat16 zero_of<__nv_bfloat16>() { return __float2bfloat16(0.f); }

// One token block as copied from global memory: the phiq and phik rows
// (zero past F), the slice's 32 columns of v and do in the io dtype, dt of
// the block's tokens and of the token after it, and d_t.
template <typename TIO>
struct alignas(16) BwdBlk {
    float q[kTB][kFP];
    float k[kTB][kFP];
    TIO v[kTB][32];
    TIO g[kTB][32];
    float dt[kTB + 1];
    float den[kTB];
};

// Copies tokens t0 .. t0 + nt - 1 of (b, h) (and dt of token t0 + nt) into
// bk.  fast: every row starts 16-byte aligned (F % 4 == 0, the slice's rows of
// v and do a multiple of 16 bytes) and the copies are cp.async, completed by
// the caller's wait; otherwise plain loads into the same layout.
template <typename TIO>
__device__ __forceinline__ void issue_block(BwdBlk<TIO> *bk, const BwdArgs &a, int64_t b, int h, int64_t t0, int nt,
                                            int c0, bool fast, bool with_den) {
    const int F = a.F, dv = a.dv, H = a.H;
    const int64_t L = a.L;
    const TIO *v = (const TIO *)a.v;
    const TIO *dout = (const TIO *)a.dout;
    auto rowi = [&](int64_t t) { return (b * L + t) * H + h; };
    const int tid = threadIdx.x;
    if (fast) {
        for (int c = tid; c < kTB * (kFP / 4); c += blockDim.x) {
            const int t = c / (kFP / 4), f = (c % (kFP / 4)) * 4;
            const bool ok = t < nt && f < F;
            const int64_t off = ok ? rowi(t0 + t) * F + f : 0;
            cp_async16(&bk->q[t][f], a.phq + off, ok ? 16 : 0);
            cp_async16(&bk->k[t][f], a.phk + off, ok ? 16 : 0);
        }
        constexpr int kPer = 16 / (int)sizeof(TIO);   // elements per 16 bytes
        constexpr int kRow = 32 / kPer;               // 16-byte groups per token
        for (int c = tid; c < kTB * kRow; c += blockDim.x) {
            const int t = c / kRow, e = (c % kRow) * kPer;
            const bool ok = t < nt && c0 + e < dv;
            const int64_t off = ok ? rowi(t0 + t) * dv + c0 + e : 0;
            cp_async16(&bk->v[t][e], v + off, ok ? 16 : 0);
            cp_async16(&bk->g[t][e], dout + off, ok ? 16 : 0);
        }
        if (tid <= kTB && a.dt) {
            const bool ok = tid <= nt && t0 + tid < L;
            cp_async4(&bk->dt[tid], a.dt + (ok ? rowi(t0 + tid) : 0), ok ? 4 : 0);
        }
        if (with_den && tid < kTB) {
            const bool ok = tid < nt;
            cp_async4(&bk->den[tid], a.den + (ok ? rowi(t0 + tid) : 0), ok ? 4 : 0);
        }
    } else {
        for (int c = tid; c < kTB * kFP; c += blockDim.x) {
            const int t = c / kFP, f = c % kFP;
            const bool ok = t < nt && f < F;
            bk->q[t][f] = ok ? a.phq[rowi(t0 + t) * F + f] : 0.f;
            bk->k[t][f] = ok ? a.phk[rowi(t0 + t) * F + f] : 0.f;
        }
        for (int c = tid; c < kTB * 32; c += blockDim.x) {
            const int t = c / 32, e = c % 32;
            const bool ok = t < nt && c0 + e < dv;
            bk->v[t][e] = ok ? v[rowi(t0 + t) * dv + c0 + e] : zero_of<TIO>();
            bk->g[t][e] = ok ? dout[rowi(t0 + t) * dv + c0 + e] : zero_of<TIO>();
        }
        if (tid <= kTB && a.dt) bk->dt[tid] = (tid <= nt && t0 + tid < L) ? a.dt[rowi(t0 + tid)] : 0.f;
        if (with_den && tid < kTB) bk->den[tid] = tid < nt ? a.den[rowi(t0 + tid)] : 0.f;
    }
}

template <typename TIO>
__device__ __forceinline__ bool blocks_fast(const BwdArgs &a) {
    return a.F % 4 == 0 && (a.dv * (int)sizeof(TIO)) % 16 == 0;
}

// ------------------------------------------------------------ PA

// PA (forward in time), a thread per feature row f with the slice's 32
// columns of S in registers: S_t[f, :] = a_t S_(t-1)[f, :] + phik_t[f] v_t and
// u_f = sum_c S_t[f, c] do_t[c] (four partial sums).  The denominator's state
// z_t[f] = a_t z_(t-1)[f] + phik_t[f] rides along, so d_t = sum_f phiq_t[f]
// z_t[f] needs no pass of its own.  Per token the thread leaves u_f and
// phiq_f u_f in place of the block's phiq and phik entries (read by this
// thread alone) and phiq_f z_f beside them; at the block's end the sums over f
// give d_t (slice 0 stores it) and the slice's share of do_t . n_t, and the
// slice's share of dphiq_t[f] is u_f / d_t.  Blocks are copied one ahead.
template <typename TIO>
__global__ void __launch_bounds__(256, 2)
bwd_pa_kernel(BwdArgs a) {
    extern __shared__ __align__(16) uint8_t smem_pa[];
    BwdBlk<TIO> *blk = reinterpret_cast<BwdBlk<TIO> *>(smem_pa);   // two buffers
    float *sqz = reinterpret_cast<float *>(blk + 2);               // [kTB][kFP] phiq z
    float *sv = sqz + kTB * kFP;                                   // [kTB][32]
    float *sg = sv + kTB * 32;                                     // [kTB][32]
    float *sa = sg + kTB * 32;                                     // [kTB] a_t
    float *sden = sa + kTB;                                        // [kTB] 1 / d_t

    const int f = threadIdx.x, lane = f & 31, w = f >> 5;
    const int F = a.F, dv = a.dv;
    const bool fok = f < F;
    const int64_t bh = blockIdx.y;
    const int64_t b = bh / a.H;
    const int h = (int)(bh % a.H);
    const int slice = blockIdx.x;
    const int c0 = slice * 32;
    const int ncol = dv - c0 < 32 ? dv - c0 : 32;
    const float alog = a.dt ? a.A_log[h] : 0.f;
    const int64_t L = a.L;
    const int64_t rows = a.B * L * a.H;
    auto rowi = [&](int64_t t) { return (b * L + t) * a.H + h; };
    const bool fast = blocks_fast<TIO>(a);

    float S[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) S[c] = (a.S0 && fok && c < ncol) ? a.S0[(bh * F + f) * dv + c0 + c] : 0.f;
    float z = (a.z0 && fok) ? a.z0[bh * F + f] : 0.f;
    float *dq = a.dq_part + (int64_t)slice * rows * F;
    const int64_t nblk = (L + kTB - 1) / kTB;
    auto ntok = [&](int64_t t0) { return (int)(L - t0 < kTB ? L - t0 : kTB); };
    issue_block(&blk[0], a, b, h, 0, ntok(0), c0, fast, false);
    cp_async_commit();
    for (int64_t bi = 0; bi < nblk; ++bi) {
        const int64_t t0 = bi * kTB;
        const int nt = ntok(t0);
        BwdBlk<TIO> *bk = &blk[bi & 1];
        if (bi + 1 < nblk) issue_block(&blk[(bi + 1) & 1], a, b, h, t0 + kTB, ntok(t0 + kTB), c0, fast, false);
        cp_async_commit();
        cp_async_wait1();
        __syncthreads();
        if (f < nt) sa[f] = a.dt ? expf(hm_log_decay(bk->dt[f], alog)) : 1.f;
        for (int i = f; i < kTB * 32; i += blockDim.x) {
            sv[i] = hm_ld(&bk->v[0][0], i);
            sg[i] = hm_ld(&bk->g[0][0], i);
        }
        __syncthreads();
        for (int t = 0; t < nt; ++t) {
            const float at = sa[t];
            const float qf = bk->q[t][f], kf = bk->k[t][f];
            z = fmaf(at, z, kf);
            float u0 = 0.f, u1 = 0.f, u2 = 0.f, u3 = 0.f;
            const float4 *v4 = reinterpret_cast<const float4 *>(sv + t * 32);
            const float4 *g4 = reinterpret_cast<const float4 *>(sg + t * 32);
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
                const float4 vv = v4[c4], gg = g4[c4];
                S[4 * c4 + 0] = fmaf(at, S[4 * c4 + 0], kf * vv.x);
                S[4 * c4 + 1] = fmaf(at, S[4 * c4 + 1], kf * vv.y);
                S[4 * c4 + 2] = fmaf(at, S[4 * c4 + 2], kf * vv.z);
                S[4 * c4 + 3] = fmaf(at, S[4 * c4 + 3], kf * vv.w);
                u0 = fmaf(S[4 * c4 + 0], gg.x, u0);
                u1 = fmaf(S[4 * c4 + 1], gg.y, u1);
                u2 = fmaf(S[4 * c4 + 2], gg.z, u2);
                u3 = fmaf(S[4 * c4 + 3], gg.w, u3);
            }
            const float u = (u0 + u1) + (u2 + u3);
            bk->q[t][f] = u;
            bk->k[t][f] = qf * u;
            sqz[t * kFP + f] = qf * z;
        }
        __syncthreads();
        // per token (warp w: tokens w, w + 8): d_t = sum_f phiq z and the
        // slice's share of do . n = sum_f phiq u
        for (int tt = w; tt < nt; tt += kW) {
            float d = 0.f, e = 0.f;
#pragma unroll
            for (int j = 0; j < kFP / 32; ++j) {
                d += sqz[tt * kFP + lane + 32 * j];
                e += bk->k[tt][lane + 32 * j];
            }
            d = warp_sum(d);
            e = warp_sum(e);
            if (lane == 0) {
                sden[tt] = 1.f / d;
                const int64_t r = rowi(t0 + tt);
                a.e_part[(int64_t)slice * rows + r] = e;
                if (slice == 0) a.den[r] = d;
            }
        }
        __syncthreads();
        if (fok)
            for (int t = 0; t < nt; ++t) dq[rowi(t0 + t) * F + f] = bk->q[t][f] * sden[t];
        // the buffer is copied into again two blocks on
        __syncthreads();
    }
}

// ------------------------------------------------------------ z passes

// The denominator's state alone for one (batch, head), thread f = feature f:
//   MODE 1 forward:  z_t again; its share of dphiq_t is z_t dd_t
//   MODE 2 backward: g_t = a_(t+1) g_(t+1) + phiq_t dd_t, its share of dphik_t;
//                    dz0 = a_1 g_1
// (dd_t = -(do_t . o_t) / d_t = -(do_t . n_t) / d_t^2).  The shares go to
// plane ns of dq_part / dk_part, after the value slices'.
template <int MODE>
__device__ __forceinline__ void bwd_z_pass(const BwdArgs &a, int64_t bh) {
    __shared__ float sa[kTB], sa1[kTB], sdd[kTB];
    const int f = threadIdx.x;
    const int64_t b = bh / a.H;
    const int h = (int)(bh % a.H);
    const int F = a.F;
    const bool fok = f < F;
    const float alog = a.dt ? a.A_log[h] : 0.f;
    const int64_t L = a.L;
    const int64_t rows = a.B * L * a.H;
    auto rowi = [&](int64_t t) { return (b * L + t) * a.H + h; };
    float zs = (MODE == 1 && a.z0 && fok) ? a.z0[bh * F + f] : 0.f;
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
            const float d = a.den[r];
            float e = 0.f;
            for (int s = 0; s < a.ns; ++s) e += a.e_part[(int64_t)s * rows + r];
            sdd[t] = -e / (d * d);
        }
        __syncthreads();
        // the block's features of this thread, all loads in flight at once
        float x[kTB];
#pragma unroll
        for (int t = 0; t < kTB; ++t) {
            const bool ok = fok && t < nt;
            x[t] = ok ? (MODE == 1 ? a.phk : a.phq)[rowi(t0 + t) * F + f] : 0.f;
        }
        if (MODE == 1) {
#pragma unroll
            for (int t = 0; t < kTB; ++t) {
                if (t >= nt) break;
                zs = fmaf(sa[t], zs, x[t]);
                if (fok) a.dq_part[(int64_t)a.ns * rows * F + rowi(t0 + t) * F + f] = zs * sdd[t];
            }
        } else {
#pragma unroll
            for (int t = kTB - 1; t >= 0; --t) {
                if (t >= nt) continue;
                zs = fmaf(sa1[t], zs, x[t] * sdd[t]);
                if (fok) a.dk_part[(int64_t)a.ns * rows * F + rowi(t0 + t) * F + f] = zs;
            }
            if (t0 == 0 && a.dz0 && fok) a.dz0[bh * F + f] = sa[0] * zs;
        }
    }
}

// ------------------------------------------------------------ PB

// PB (backward in time) over a 32-column slice: G_t = phiq_t dn_t^T +
// a_(t+1) G_(t+1), the slice's share of G_t v_t (a row sum), dv_t = G_t^T
// phik_t (a column sum) and dS0 = a_1 G_1.  Each thread holds an 8 x 4 block
// of G (rows 32 w + 8 (lane >> 3) .., columns 4 (lane & 7) ..), so a row sum
// is a reduce-scatter over 8 lanes and a column sum one over 4 lanes (then
// over the warps at the block's end); the warp's sums go in place of its own
// rows of the block's phiq and phik (read by this warp alone).  Blocks are
// copied one ahead, from the last to the first.
// The grid's first 2 B H CTAs run the z passes (modes 1 and 2), which need
// what PA wrote and nothing of PB, on the SMs the slices leave free.
template <typename TIO>
__global__ void __launch_bounds__(256, 2)
bwd_pb_kernel(BwdArgs a) {
    const int64_t BH = a.B * a.H;
    if ((int64_t)blockIdx.x < 2 * BH) {
        if ((int64_t)blockIdx.x < BH)
            bwd_z_pass<1>(a, blockIdx.x);
        else
            bwd_z_pass<2>(a, blockIdx.x - BH);
        return;
    }
    extern __shared__ __align__(16) uint8_t smem_pb[];
    BwdBlk<TIO> *blk = reinterpret_cast<BwdBlk<TIO> *>(smem_pb);   // two buffers
    float *sdn = reinterpret_cast<float *>(blk + 2);               // [kTB][32] do / d
    float *sv = sdn + kTB * 32;                                    // [kTB][32]
    float *sa1 = sv + kTB * 32;                                    // [kTB] a_(t+1)
    float *sa0 = sa1 + kTB;                                        // a of the first token

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int rgl = lane >> 3, cg = lane & 7;
    const int r0 = 32 * w + 8 * rgl, cc = 4 * cg;
    const int64_t idx = (int64_t)blockIdx.x - 2 * BH;
    const int slice = (int)(idx % a.ns);
    const int64_t bh = idx / a.ns;
    const int64_t b = bh / a.H;
    const int h = (int)(bh % a.H);
    const int F = a.F, dv = a.dv;
    const int c0 = slice * 32;
    const float alog = a.dt ? a.A_log[h] : 0.f;
    const int64_t L = a.L;
    const int64_t rows = a.B * L * a.H;
    auto rowi = [&](int64_t t) { return (b * L + t) * a.H + h; };
    const bool fast = blocks_fast<TIO>(a);
    float *dk = a.dk_part + (int64_t)slice * rows * F;

    float G[8][4];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) G[r][c] = 0.f;
    const int64_t nblk = (L + kTB - 1) / kTB;
    auto first = [&](int64_t bi) { return (nblk - 1 - bi) * kTB; };
    auto ntok = [&](int64_t t0) { return (int)(L - t0 < kTB ? L - t0 : kTB); };
    issue_block(&blk[0], a, b, h, first(0), ntok(first(0)), c0, fast, true);
    cp_async_commit();
    for (int64_t bi = 0; bi < nblk; ++bi) {
        const int64_t t0 = first(bi);
        const int nt = ntok(t0);
        BwdBlk<TIO> *bk = &blk[bi & 1];
        if (bi + 1 < nblk) issue_block(&blk[(bi + 1) & 1], a, b, h, first(bi + 1), kTB, c0, fast, true);
        cp_async_commit();
        cp_async_wait1();
        __syncthreads();
        if (tid < nt)
            sa1[tid] = (a.dt && t0 + tid + 1 < L) ? expf(hm_log_decay(bk->dt[tid + 1], alog)) : 1.f;
        if (tid == 0 && t0 == 0) sa0[0] = a.dt ? expf(hm_log_decay(bk->dt[0], alog)) : 1.f;
        for (int i = tid; i < kTB * 32; i += blockDim.x) {
            const int t = i / 32;
            sv[i] = hm_ld(&bk->v[0][0], i);
            sdn[i] = t < nt ? hm_ld(&bk->g[0][0], i) / bk->den[t] : 0.f;
        }
        __syncthreads();
        for (int t = nt - 1; t >= 0; --t) {
            const float a1 = sa1[t];
            const float4 qa = *reinterpret_cast<const float4 *>(&bk->q[t][r0]);
            const float4 qb = *reinterpret_cast<const float4 *>(&bk->q[t][r0 + 4]);
            const float4 ka = *reinterpret_cast<const float4 *>(&bk->k[t][r0]);
            const float4 kb = *reinterpret_cast<const float4 *>(&bk->k[t][r0 + 4]);
            const float4 d4v = *reinterpret_cast<const float4 *>(sdn + t * 32 + cc);
            const float4 v4v = *reinterpret_cast<const float4 *>(sv + t * 32 + cc);
            const float q8[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
            const float k8[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
            const float dn[4] = {d4v.x, d4v.y, d4v.z, d4v.w};
            const float vv[4] = {v4v.x, v4v.y, v4v.z, v4v.w};
            float x[8], y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                x[r] = 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    G[r][c] = fmaf(q8[r], dn[c], a1 * G[r][c]);
                    x[r] = fmaf(G[r][c], vv[c], x[r]);
                    y[c] = fmaf(G[r][c], k8[r], y[c]);
                }
            }
            // row sums over the 8 lanes of a row group (lane bits 0..2): lane
            // ends with row r0 + cg = 32 w + lane
#pragma unroll
            for (int off = 4; off >= 1; off >>= 1) {
                const bool upper = (lane & off) != 0;
#pragma unroll
                for (int j = 0; j < off; ++j) {
                    const float send = upper ? x[j] : x[j + off];
                    const float keep = upper ? x[j + off] : x[j];
                    x[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
            // column sums over the warp's 4 row groups (lane bits 4, 3): lane
            // ends with column cc + rgl
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const int off = 16 >> s, half = 2 >> s;
                const bool upper = (lane & off) != 0;
#pragma unroll
                for (int j = 0; j < half; ++j) {
                    const float send = upper ? y[j] : y[j + half];
                    const float keep = upper ? y[j + half] : y[j];
                    y[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
            bk->q[t][32 * w + lane] = x[0];
            bk->k[t][32 * w + cc + rgl] = y[0];
        }
        __syncthreads();
        // dv_t = the warps' column sums; the slice's share of dphik_t
        for (int i = tid; i < nt * 32; i += blockDim.x) {
            const int t = i / 32, c = i % 32;
            float acc = 0.f;
#pragma unroll
            for (int ww = 0; ww < kW; ++ww) acc += bk->k[t][32 * ww + c];
            if (c0 + c < dv) a.dv_out[rowi(t0 + t) * dv + c0 + c] = acc;
        }
        if (tid < F)
            for (int t = 0; t < nt; ++t) dk[rowi(t0 + t) * F + tid] = bk->q[t][tid];
        if (t0 == 0 && a.dS0) {
            // dS0 = a_1 G_1 (a_1 = the first token's decay)
            const float a0 = sa0[0];
#pragma unroll
            for (int r = 0; r < 8; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (r0 + r < F && c0 + cc + c < dv) a.dS0[(bh * F + r0 + r) * dv + c0 + cc + c] = a0 * G[r][c];
        }
        // the buffer is copied into again two blocks on
        __syncthreads();
    }
}

// dphiq, dphik = sums of the slices' shares (and the denominator's, plane
// ns), and kd_r = phik_r . dphik_r; one warp per row, lanes over groups of 4
// features, the planes' loads of a group issued together (up to 9 at a
// time) and added in plane order.
__global__ void __launch_bounds__(256)
bwd_reduce_kernel(BwdArgs a, float *__restrict__ dphq, float *__restrict__ dphk, float *__restrict__ kd) {
    constexpr int kPl = 9;
    const int lane = threadIdx.x & 31;
    const int64_t rows = a.B * a.L * a.H;
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (r >= rows) return;
    const int F = a.F, ns = a.ns;
    const int64_t plane = rows * (int64_t)F;
    const float *__restrict__ pq = a.dq_part + r * F;
    const float *__restrict__ pk = a.dk_part + r * F;
    float acc = 0.f;
    if (F % 4 == 0) {
        for (int f = 4 * lane; f < F; f += 128) {
            float4 sq = make_float4(0.f, 0.f, 0.f, 0.f), sk = sq;
            for (int s0 = 0; s0 <= ns; s0 += kPl) {
                float4 vq[kPl], vk[kPl];
#pragma unroll
                for (int j = 0; j < kPl; ++j) {
                    const bool ok = s0 + j <= ns;
                    vq[j] = ok ? __ldcs(reinterpret_cast<const float4 *>(pq + (s0 + j) * plane + f)) : sq;
                    vk[j] = ok ? __ldcs(reinterpret_cast<const float4 *>(pk + (s0 + j) * plane + f)) : sk;
                }
#pragma unroll
                for (int j = 0; j < kPl; ++j) {
                    if (s0 + j > ns) break;
                    sq.x += vq[j].x; sq.y += vq[j].y; sq.z += vq[j].z; sq.w += vq[j].w;
                    sk.x += vk[j].x; sk.y += vk[j].y; sk.z += vk[j].z; sk.w += vk[j].w;
                }
            }
            *reinterpret_cast<float4 *>(dphq + r * F + f) = sq;
            *reinterpret_cast<float4 *>(dphk + r * F + f) = sk;
            const float4 k4 = *reinterpret_cast<const float4 *>(a.phk + r * F + f);
            acc = fmaf(k4.x, sk.x, acc);
            acc = fmaf(k4.y, sk.y, acc);
            acc = fmaf(k4.z, sk.z, acc);
            acc = fmaf(k4.w, sk.w, acc);
        }
    } else {
        for (int f = lane; f < F; f += 32) {
            float sq = 0.f, sk = 0.f;
            for (int s = 0; s <= ns; ++s) {
                sq += pq[s * plane + f];
                sk += pk[s * plane + f];
            }
            dphq[r * F + f] = sq;
            dphk[r * F + f] = sk;
            acc = fmaf(a.phk[r * F + f], sk, acc);
        }
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
// de = phi (.) (dphi - sum(phi (.) dphi)), du = de[:p] - de[p:].  One warp per
// row.  With dus, du is also written as bf16 segments [hi | lo (| hi)] of
// a row of nseg * p (hi = du rounded to bf16, lo = the rounded remainder):
// the operand of dx = du W (and of dW = du^T x) on the tensor cores; du
// itself (fp32) may then be null.
__global__ void __launch_bounds__(256)
featmap_bwd_du_kernel(const float *__restrict__ phi, const float *__restrict__ dphi, int64_t rows, int p,
                      float *__restrict__ du, __nv_bfloat16 *__restrict__ dus, int nseg) {
    const int lane = threadIdx.x & 31;
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (r >= rows) return;
    const float *ph = phi + r * 2 * p, *dp = dphi + r * 2 * p;
    float s = 0.f;
    for (int f = lane; f < 2 * p; f += 32) s = fmaf(ph[f], dp[f], s);
    s = warp_sum(s);
    for (int j = lane; j < p; j += 32) {
        const float x = ph[j] * (dp[j] - s) - ph[p + j] * (dp[p + j] - s);
        if (du) du[r * p + j] = x;
        if (dus) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(x);
            const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
            __nv_bfloat16 *row = dus + r * nseg * p;
            row[j] = hi;
            row[p + j] = lo;
            if (nseg == 3) row[2 * p + j] = hi;
        }
    }
}

// B operand of dx = du W on the tensor cores: Wt[i][s p + j] for the segments
// s of the A operand's [hi | lo (| hi)]: W[j][i] rounded to bf16 twice, then
// (fp32 W) its rounded remainder, so that the GEMM sums hi W_hi + lo W_hi
// (+ hi W_lo).  A bf16 W is exact in one bf16 (two segments).
template <typename TW>
__global__ void __launch_bounds__(256)
featmap_bwd_wsplit_kernel(const TW *__restrict__ W, int p, int d, int nseg, __nv_bfloat16 *__restrict__ Wt) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)p * d) return;
    const int j = (int)(i / d), col = (int)(i % d);
    const float w = hm_ld(W, i);
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    __nv_bfloat16 *row = Wt + (int64_t)col * nseg * p;
    row[j] = hi;
    row[p + j] = hi;
    if (nseg == 3) row[2 * p + j] = __float2bfloat16_rn(w - __bfloat162float(hi));
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

// ------------------------------------------------------------ dW on the tensor cores

// dW = du^T x for p = 128 and bf16 x with d a multiple of 64 up to 256: each
// CTA takes a run of 64-token blocks and accumulates du_hi^T x + du_lo^T x
// over them in one 128 x d fp32 TMEM tile, then adds the tile to dW (zeroed
// first) with float4 atomics.  Both operands are MN-major (tokens are the
// contraction): 64-token x 64-feature boxes of the du kernel's bf16 [hi | lo]
// rows and of x, loaded by TMA through a 3-stage ring.  Warp 0 loads, warp 1
// issues the MMAs, warps 2..5 (one per TMEM lane quarter) add the tile.
constexpr int kDwStages = 3;
constexpr int kDwBox = 64 * 64 * 2;              // one 64-token x 64-feature bf16 box
constexpr int kDwA = 2 * kDwBox;                 // du hi (or lo): 128 features
constexpr int kDwStage = 2 * kDwA + 4 * kDwBox;  // hi, lo and up to 256 features of x
constexpr int kDwSmem = kDwStages * kDwStage + 1024 + 256;

struct DwAux {
    uint64_t full[kDwStages], empty[kDwStages], dfull;
    uint32_t tmem;
    int abort;
};

__global__ void __launch_bounds__(192, 1)
featmap_dw_tc_kernel(const __grid_constant__ CUtensorMap tmu, const __grid_constant__ CUtensorMap tmx,
                     int64_t nblk, int64_t per, int p, int d, float *__restrict__ dW, DevErr err) {
    using namespace tc;
    extern __shared__ uint8_t smem_dw[];
    uint8_t *smem = align_smem_1024(smem_dw);
    DwAux *X = reinterpret_cast<DwAux *>(smem + kDwStages * kDwStage);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t blk0 = (int64_t)blockIdx.x * per;
    const int64_t blk1 = blk0 + per < nblk ? blk0 + per : nblk;
    const int nb = blk1 > blk0 ? (int)(blk1 - blk0) : 0;
    const int nfb = d / 64;
    volatile int *abort_flag = &X->abort;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kDwStages; ++s) {
            mbar_init(&X->full[s], 1);
            mbar_init(&X->empty[s], 1);
        }
        mbar_init(&X->dfull, 1);
        X->abort = 0;
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(&X->tmem, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = X->tmem;
    if (warp == 0) {
        if (elect_one()) {
            tma_prefetch_desc(&tmu);
            tma_prefetch_desc(&tmx);
            int it = 0;
            for (; it < nb; ++it) {
                const int s = it % kDwStages;
                if (!mbar_wait(&X->empty[s], ((it / kDwStages) & 1) ^ 1, abort_flag, err, KID_BWD_DW_TC, 1)) break;
                uint8_t *st = smem + s * kDwStage;
                const int r0 = (int)((blk0 + it) * 64);
                mbar_arrive_expect_tx(&X->full[s], (uint32_t)((4 + nfb) * kDwBox));
                for (int h = 0; h < 2; ++h)          // hi, then lo
                    for (int fb = 0; fb < 2; ++fb)
                        tma_load_2d(st + h * kDwA + fb * kDwBox, &tmu, &X->full[s], h * p + fb * 64, r0);
                for (int fb = 0; fb < nfb; ++fb)
                    tma_load_2d(st + 2 * kDwA + fb * kDwBox, &tmx, &X->full[s], fb * 64, r0);
            }
            // no copy may still be landing when the CTA exits
            for (int j = it > kDwStages ? it - kDwStages : 0; j < it; ++j)
                for (uint32_t i = 0; i < kWaitPolls; ++i)
                    if (mbar_try_wait(&X->full[j % kDwStages], (j / kDwStages) & 1)) break;
        }
    } else if (warp == 1) {
        if (elect_one()) {
            const uint32_t idesc = idesc_bf16(128, d, true, true);
            bool ok = true;
            for (int it = 0; it < nb; ++it) {
                const int s = it % kDwStages;
                if (!mbar_wait(&X->full[s], (it / kDwStages) & 1, abort_flag, err, KID_BWD_DW_TC, 2)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a = smem_u32(smem + s * kDwStage);
                const uint32_t bx = a + 2 * kDwA;
#pragma unroll
                for (int k = 0; k < 4; ++k) {   // 16 tokens per MMA
                    const uint64_t db = desc_mn_sw128(bx + k * 2048, kDwBox, 1024);
                    mma_ss(tmem, desc_mn_sw128(a + k * 2048, kDwBox, 1024), db, idesc, (it > 0 || k > 0) ? 1u : 0u);
                    mma_ss(tmem, desc_mn_sw128(a + kDwA + k * 2048, kDwBox, 1024), db, idesc, 1u);
                }
                mma_commit(&X->empty[s]);
            }
            if (nb > 0) {
                mma_commit(&X->dfull);
                // the MMAs are complete before TMEM is released, whatever the epilogue did
                if (ok) mbar_wait(&X->dfull, 0, abort_flag, err, KID_BWD_DW_TC, 4);
            }
        }
    } else {
        // warps 2..5: TMEM lane quarter warp % 4 holds rows 32 (warp % 4) .. + 31 of dW
        const int q = warp & 3;
        const int row = 32 * q + lane;
        if (nb > 0 && mbar_wait(&X->dfull, 0, abort_flag, err, KID_BWD_DW_TC, 3)) {
            tc_fence_after();
            const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16);
            float *dst = dW + (int64_t)row * d;
#pragma unroll 1
            for (int c0 = 0; c0 < d; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(ta + c0, r);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    atomicAdd(reinterpret_cast<float4 *>(dst + c0 + 4 * u),
                              make_float4(__uint_as_float(r[4 * u]), __uint_as_float(r[4 * u + 1]),
                                          __uint_as_float(r[4 * u + 2]), __uint_as_float(r[4 * u + 3])));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// The shapes featmap_dw_tc_kernel takes (bf16 inputs: two segments).
__host__ __device__ constexpr bool dw_tc_shape(bool have_dus, int nseg, int p, int d) {
    return have_dus && nseg == 2 && p == 128 && d % 64 == 0 && d <= 256;
}

// dW on the tensor cores (the shapes featmap_dw_tc_kernel takes): dus is the
// du kernel's [rows][2p] bf16 [hi | lo], x [rows][d] bf16; dW zeroed here.
cudaError_t run_featmap_dw_tc(const __nv_bfloat16 *dus, const __nv_bfloat16 *x, int64_t rows, int p, int d,
                              float *dW, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(dW, 0, sizeof(float) * (size_t)p * d, s);
    if (e != cudaSuccess) return e;
    CUtensorMap tmu, tmx;
    {
        const uint64_t dims[2] = {(uint64_t)2 * p, (uint64_t)rows};
        const uint64_t strides[1] = {(uint64_t)2 * p * 2};
        const uint32_t box[2] = {64, 64};
        if (!tc::make_tmap_bf16(&tmu, dus, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[2] = {(uint64_t)d, (uint64_t)rows};
        const uint64_t strides[1] = {(uint64_t)d * 2};
        const uint32_t box[2] = {64, 64};
        if (!tc::make_tmap_bf16(&tmx, x, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t nblk = (rows + 63) / 64;
    const int64_t per = (nblk + sms - 1) / sms;
    const unsigned grid = (unsigned)((nblk + per - 1) / per);
    e = tc::ensure_smem_limit(featmap_dw_tc_kernel, kDwSmem);
    if (e != cudaSuccess) return e;
    featmap_dw_tc_kernel<<<grid, 192, kDwSmem, s>>>(tmu, tmx, nblk, per, p, d, dW, DevErr{device_error_word()});
    count_launches(1);
    return cudaGetLastError();
}

// dx = du W ([rows, p] x [p, d]) and dW = du^T x ([p, rows] x [rows, d], k
// split so that about two CTAs per SM run; dW is zeroed first).  With dus
// (the du kernel's bf16 segments) and Wt, dx is one tensor-core GEMM over K =
// nseg p: the products of the segments carry du to about 2^-17 of itself
// (the hi and lo parts) and W exactly (bf16) or to 2^-17 (fp32); otherwise
// the CUDA-core contraction.
template <typename T>
cudaError_t run_featmap_bwd_products(const float *du, const __nv_bfloat16 *dus, __nv_bfloat16 *Wt, int nseg,
                                     const T *W, const T *x, int64_t rows, int p, int d, float *dx, float *dW,
                                     cudaStream_t s) {
    const bool vec = p % 4 == 0 && d % 4 == 0;
    const unsigned nt = (unsigned)((d + kGN - 1) / kGN);
    if (dus) {
        const int64_t n = (int64_t)p * d;
        featmap_bwd_wsplit_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(W, p, d, nseg, Wt);
        count_launches(1);
        GemmEpiArgs ep;
        ep.mode = EPI_STORE_F32;
        cudaError_t e = launch_gemm_tc_ex(dus, Wt, rows, d, (int64_t)nseg * p, dx, d, ep,
                                          DevErr{device_error_word()}, s);
        if (e != cudaSuccess) return e;
        count_launches(1);
    } else {
        dim3 gx((unsigned)((rows + kGM - 1) / kGM), nt, 1);
        featmap_bwd_gemm_kernel<true, T, false><<<gx, 256, 0, s>>>(du, p, W, d, dx, d, rows, d, p, p, vec);
        count_launches(1);
    }
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        if (dw_tc_shape(dus != nullptr, nseg, p, d)) return run_featmap_dw_tc(dus, x, rows, p, d, dW, s);
    }
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
    count_launches(1);
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
    const int64_t BH = a.B * a.H;
    auto k1 = bwd_pa_kernel<TIO>;
    auto k2 = bwd_pb_kernel<TIO>;
    const size_t smem1 = 2 * sizeof(BwdBlk<TIO>) + sizeof(float) * (size_t)(kTB * kFP + 2 * kTB * 32 + 2 * kTB);
    const size_t smem2 = 2 * sizeof(BwdBlk<TIO>) + sizeof(float) * (size_t)(2 * kTB * 32 + kTB + 4);
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
    if (e != cudaSuccess) return e;
    k1<<<dim3((unsigned)a.ns, (unsigned)BH), 256, smem1, s>>>(a);
    k2<<<(unsigned)(2 * BH + (int64_t)a.ns * BH), 256, smem2, s>>>(a);
    count_launches(2);
    return cudaGetLastError();
}

// Segments of the bf16 split that carries dx = du W to the tensor cores (2
// for a bf16 W, 3 for fp32), or 0 where the GEMM does not take the shape.
int dx_segments(const ScanBwdCore &c) {
    if (!c.W_q) return 0;
    const int nseg = c.io_dtype == HM_BF16 ? 2 : 3;
    return gemm_tc_supported(c.B * c.L * c.H, c.d, (int64_t)nseg * c.p) ? nseg : 0;
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
    if (const int nseg = dx_segments(c))      // du and W^T as bf16 segments
        n += r256(rows * nseg * c.p * 2) + r256((size_t)c.d * nseg * c.p * 2);
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
    const int nseg = dx_segments(c);
    __nv_bfloat16 *dus = nseg ? (__nv_bfloat16 *)take((size_t)rows * nseg * c.p * 2) : nullptr;
    __nv_bfloat16 *Wt = nseg ? (__nv_bfloat16 *)take((size_t)c.d * nseg * c.p * 2) : nullptr;
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
            // fp32 du only where a CUDA-core product reads it
            float *du_f32 = dw_tc_shape(dus != nullptr, nseg, c.p, c.d) ? nullptr : du;
            featmap_bwd_du_kernel<<<wb, 256, 0, s>>>(phis[m], dphis[m], rows, c.p, du_f32, dus, nseg);
            count_launches(1);
            e = c.io_dtype == HM_BF16
                    ? run_featmap_bwd_products(du, dus, Wt, nseg, (const __nv_bfloat16 *)Ws[m],
                                               (const __nv_bfloat16 *)xs[m], rows, c.p, c.d, dxs[m], dWs[m], s)
                    : run_featmap_bwd_products(du, dus, Wt, nseg, (const float *)Ws[m], (const float *)xs[m], rows,
                                               c.p, c.d, dxs[m], dWs[m], s);
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

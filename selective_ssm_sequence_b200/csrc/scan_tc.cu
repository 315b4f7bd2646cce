// scan_tc.cu -- chunkwise decayed normalised scan on the 5th-generation tensor cores.
//
// Computes, for features phiq, phik (bf16, F = 256), values v (bf16) and the
// decay a_t = exp(-softplus(dt_t) exp(A_log_h)):
//   S_t = a_t S_{t-1} + phik_t v_t^T,  z_t = a_t z_{t-1} + phik_t,
//   o_t = phiq_t^T S_t / phiq_t^T z_t
// (HedgeMamba explainer sec. 2.3 / 5.2; linear-attention tutorial sec. 3-5).
//
// Chunkwise form (chunks of C = 64 tokens; cum_i = sum of log a over the
// chunk up to token i; gamma = exp(cum_last)):
//   P        = phiQ phiK^T                                     (tensor cores)
//   Pt_ij    = P_ij exp(cum_i - cum_j) [j <= i]                (registers; the
//              decay is applied elementwise, or as a product of two factors
//              that are both <= 1, so no term overflows)
//   O        = Pt V + diag(exp(cum)) phiQ S_prev               (tensor cores)
//   den      = rowsum(Pt) + exp(cum) (phiQ z_prev)
//   S        = gamma S_prev + (w phiK)^T V,  w_j = exp(cum_last - cum_j) <= 1
//            = gamma S_prev + phiK^T (w V)   (the kernels weight the 128 value
//              channels of their CTA rather than the 256 features)
//   z        = gamma z_prev + sum_j w_j phik_j
// These are exact rewrites of the recurrence.  The state is kept transposed
// (S^T, value channel x feature) in TMEM: the state update V^T (w phiK) and the
// readout S^T (e^cum phiQ)^T then both have the 128 value channels of a CTA as
// their M dimension, and the readout takes its A operand (a bf16 copy of S^T)
// straight from TMEM.
//
// Step-scaled input (HM_FLAG_DT_SCALED_INPUT, Mamba's B-bar = Delta B): every
// factor that weights key j -- w_j, the decay of column j of Pt -- also
// carries Delta_j = softplus(dt_j); the decay warp folds log2(Delta_j) into the
// key-side prefix sums, so the chunk loop is unchanged.  (The per-feature
// decay variant has no tensor-core kernel: it runs on the CUDA-core scan.)
//
// Long sequences are cut into segments that run in parallel.  Three kernels:
//   A  scan_state_kernel  local end state of each part (a run of chunks) from a
//                         zero start, weights relative to the part end; with
//                         hi / lo bf16 splits of w (.) v and of phik the state
//                         update is accurate to ~16 bits (used for the
//                         returned state).
//   B  scan_carry_kernel  composes the parts' affine maps (S -> g S + S_part,
//                         SSM article sec. 4.2) in fp32 to get each segment's
//                         start state and the final state.
//   C  scan_out_kernel    the chunk loop above over one segment, from its start
//                         state, writing o.
// One CTA owns (batch, head, half of the value channels, segment).
#include <algorithm>

#include "tc_common.cuh"

namespace hm {

namespace {

using namespace tc;

constexpr int kC = 64;        // tokens per chunk
constexpr int kF = 256;       // feature dimension
constexpr int kN = 128;       // value channels per CTA
constexpr int kBlk = kC * 128;  // one [64 rows x 128 B] block = 8 KB
constexpr int kTileF = 4 * kBlk;   // [64 x 256] bf16 tile = 32 KB
constexpr int kTileV = 2 * kBlk;   // [64 x 128] bf16 tile = 16 KB

// e^x for the decay factors (arguments <= 0 except the log-space prefix sums
// of a chunk; results are used at bf16 / fp32-accumulate precision)
__device__ __forceinline__ float fexp(float x) { return ex2_approx(x * 1.4426950408889634f); }
constexpr float kLog2e = 1.4426950408889634f;

struct Geo {
    int64_t B, L;
    int H, dv;
    int nchunks;     // ceil(L / C)
    int seg_chunks;  // chunks per output segment (multiple of part_chunks)
    int G;           // output segments
    int part_chunks; // chunks per state part
    int NP;          // parts in the whole sequence
    int NPc;         // parts whose state phase A computes (a prefix)
};

// ------------------------------------------------------------------ phase A

constexpr int kABuild = 8;              // builder warps of the state kernel
constexpr int kAWB = 16 * 128;          // weight rows for z: [16 rows x 64 tokens] bf16, K-major
constexpr int kAStageBudget = 200 * 1024;

struct AAux {
    float w[4][kC];    // weights of the chunk in each stage
    uint64_t full[4], empty[4], built[4], wfull[4], done;
    uint32_t tmem;
    int abort;
};

// Stage layout of the state kernel: phiK (hi) [64 x 256], phiK lo when the
// caller passes it, V [64 x 128] (overwritten by w (.) V, bf16 hi), the lo
// part of w (.) V when the state is returned, and the weight rows of the z
// product.  As many stages as fit the budget, at most 4.
struct ALay {
    int kl, v, vl, wb, stage, nst;
};
__host__ __device__ constexpr ALay a_layout(int split, int add_lo) {
    ALay l{};
    int o = kTileF;
    l.kl = add_lo ? o : 0;
    o += add_lo ? kTileF : 0;
    l.v = o;
    o += kTileV;
    l.vl = split ? o : 0;
    o += split ? kTileV : 0;
    l.wb = o;
    o += kAWB;
    l.stage = o;
    l.nst = kAStageBudget / o < 4 ? kAStageBudget / o : 4;
    return l;
}
static_assert(a_layout(1, 1).nst >= 2 && a_layout(0, 0).nst == 4, "state kernel stages");

constexpr int kAOffAux = kAStageBudget;
constexpr int kASmem = kAOffAux + (int)sizeof(AAux) + 1024;
static_assert(kASmem <= 227 * 1024, "phase A shared memory");

// One CTA: (batch, head, value half, part).  Chunks of the part run from the
// last to the first so that the suffix sums of log a (the weights relative to
// the part end) are accumulated from small to large magnitudes.  Per chunk:
//   S_part^T += (w (.) V)^T phiK     (M = 128 value channels, N = 256 features)
//   z_part   += phiK^T w             (M = the 128 features of the CTA's value
//                                     half's index, N = 16: the weight rows
//                                     w_hi, w_lo and 14 zero rows)
// The builder warps only weight the CTA's 128 value channels; the z sums run
// on the tensor cores, each value half taking half of the features; the
// weights of the chunks come from one more warp that runs ahead of the
// builders.
constexpr int kAThreads = 64 + 32 * kABuild + 32;

__global__ void __launch_bounds__(kAThreads, 1)
scan_state_kernel(const __grid_constant__ CUtensorMap tmkh, const __grid_constant__ CUtensorMap tmkl,
                  const __grid_constant__ CUtensorMap tmv, Geo g, const float *__restrict__ dt,
                  const float *__restrict__ A_log, int split, int add_lo, int dt_scaled, float *__restrict__ S_part,
                  float *__restrict__ z_part, float *__restrict__ lsum_part, DevErr err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    AAux *X = (AAux *)(smem + kAOffAux);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = blockIdx.x & 1;
    const int part = (blockIdx.x >> 1) % g.NPc;
    const int64_t bh = (blockIdx.x >> 1) / g.NPc;
    const int64_t b = bh / g.H;
    const int h = (int)(bh % g.H);
    const int dv0 = half * kN;
    const int c_first = part * g.part_chunks;
    const int c_last = min(g.nchunks, c_first + g.part_chunks) - 1;
    const int n = c_last - c_first + 1;
    const ALay lay = a_layout(split, add_lo);
    const int nst = lay.nst;
    volatile int *abort_flag = &X->abort;
    auto stage = [&](int s) { return smem + s * lay.stage; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(&X->full[s], 1);
            mbar_init(&X->empty[s], 1);
            mbar_init(&X->built[s], kABuild);   // one arrival per builder warp
            mbar_init(&X->wfull[s], 1);
        }
        mbar_init(&X->done, 1);
        X->abort = 0;
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(&X->tmem, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = X->tmem;

    if (warp == 0) {
        if (elect_one()) {
            tma_prefetch_desc(&tmkh);
            tma_prefetch_desc(&tmkl);
            tma_prefetch_desc(&tmv);
            const uint32_t tx = kTileF + kTileV + (add_lo ? kTileF : 0);
            int it = 0, s = 0;
            uint32_t ph = 0;
            for (; it < n; ++it) {
                if (!mbar_wait(&X->empty[s], ph ^ 1, abort_flag, err, KID_SCAN_TC_STATE, 1)) break;
                const int t0 = (c_last - it) * kC;
                uint8_t *st = stage(s);
                mbar_arrive_expect_tx(&X->full[s], tx);
                for (int bb = 0; bb < 4; ++bb)
                    tma_load_4d(st + bb * kBlk, &tmkh, &X->full[s], bb * 64, h, t0, (int)b);
                if (add_lo)
                    for (int bb = 0; bb < 4; ++bb)
                        tma_load_4d(st + lay.kl + bb * kBlk, &tmkl, &X->full[s], bb * 64, h, t0, (int)b);
                for (int bb = 0; bb < 2; ++bb)
                    tma_load_4d(st + lay.v + bb * kBlk, &tmv, &X->full[s], dv0 + bb * 64, h, t0, (int)b);
                if (++s == nst) {
                    s = 0;
                    ph ^= 1;
                }
            }
            // on an early exit, the loads still in flight land before the CTA ends
            for (int j = max(0, it - nst); j < it; ++j) {
                for (uint32_t i = 0; i < kWaitPolls; ++i)
                    if (mbar_try_wait(&X->full[j % nst], (j / nst) & 1)) break;
            }
        }
    } else if (warp == 1) {
        if (elect_one()) {
            constexpr uint32_t idS = idesc_bf16(128, 256, true, true);
            constexpr uint32_t idZ = idesc_bf16(128, 16, true, false);
            int s = 0;
            uint32_t ph = 0;
            for (int it = 0; it < n; ++it) {
                if (!mbar_wait(&X->full[s], ph, abort_flag, err, KID_SCAN_TC_STATE, 2)) break;
                if (!mbar_wait(&X->built[s], ph, abort_flag, err, KID_SCAN_TC_STATE, 3)) break;
                tc_fence_after();
                const uint32_t kh = smem_u32(stage(s));
                const uint32_t kl = kh + lay.kl, vv = kh + lay.v, vl = kh + lay.vl, wb = kh + lay.wb;
                for (int k = 0; k < kC / 16; ++k) {
                    const uint32_t acc = (it > 0 || k > 0) ? 1u : 0u;
                    const uint64_t bk = desc_mn_sw128(kh + k * 2048, kBlk, 1024);
                    const uint64_t av = desc_mn_sw128(vv + k * 2048, kBlk, 1024);
                    mma_ss(tmem, av, bk, idS, acc);
                    if (split) mma_ss(tmem, desc_mn_sw128(vl + k * 2048, kBlk, 1024), bk, idS, 1u);
                    if (add_lo) mma_ss(tmem, av, desc_mn_sw128(kl + k * 2048, kBlk, 1024), idS, 1u);
                    const uint64_t bw = desc_k_sw128(wb + k * 32);
                    mma_ss(tmem + 256, desc_mn_sw128(kh + half * 2 * kBlk + k * 2048, kBlk, 1024), bw, idZ, acc);
                    if (add_lo)
                        mma_ss(tmem + 256, desc_mn_sw128(kl + half * 2 * kBlk + k * 2048, kBlk, 1024), bw, idZ, 1u);
                }
                mma_commit(&X->empty[s]);
                if (++s == nst) {
                    s = 0;
                    ph ^= 1;
                }
            }
            mma_commit(&X->done);
            // TMEM is released only after the issued MMAs have completed
            for (uint32_t i = 0; i < kWaitPolls; ++i)
                if (mbar_try_wait(&X->done, 0)) break;
        }
    } else if (warp == 2 + kABuild) {
        // weights: w_j = exp(sum of log a over the tokens after j up to the
        // part end); lane: tokens 2 lane and 2 lane + 1 of each chunk
        const float alog = dt ? A_log[h] : 0.f;
        // dt of the chunk it + i in da[i], db[i] (fetched four chunks ahead)
        auto token_dt = [&](int it, int j) {
            const int64_t t = (int64_t)(c_last - it) * kC + j;
            return (dt && it < n && t < g.L) ? dt[(b * g.L + t) * g.H + h] : -INFINITY;
        };
        float da[4], db[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            da[i] = token_dt(i, 2 * lane);
            db[i] = token_dt(i, 2 * lane + 1);
        }
        float suf = 0.f;
        int s = 0;
        uint32_t ph = 0;
        bool okw = true;
        for (int it = 0; it < n; ++it) {
            const float l0 = hm_log_decay(da[0], alog), l1 = hm_log_decay(db[0], alog);
            // step-scaled input: the token's weight also carries softplus(dt)
            const float d0 = dt_scaled ? hm_step_size(da[0]) : 1.f;
            const float d1 = dt_scaled ? hm_step_size(db[0]) : 1.f;
#pragma unroll
            for (int i = 0; i < 3; ++i) {
                da[i] = da[i + 1];
                db[i] = db[i + 1];
            }
            da[3] = token_dt(it + 4, 2 * lane);
            db[3] = token_dt(it + 4, 2 * lane + 1);
            // inclusive suffix sums of the token pairs over the lanes
            const float pair = l0 + l1;
            float x = pair;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, x, o);
                if (lane + o < 32) x += y;
            }
            const float tot = __shfl_sync(0xffffffffu, x, 0);
            const float ex1 = x - pair;   // tokens after 2 lane + 1
            const float ex0 = ex1 + l1;   // tokens after 2 lane
            // the stage's weights were last read by the build of chunk it - nst
            if (it >= nst) okw = mbar_wait(&X->built[s], ph ^ 1, abort_flag, err, KID_SCAN_TC_STATE, 6);
            okw = __all_sync(0xffffffffu, okw);
            if (!okw) break;
            *reinterpret_cast<float2 *>(&X->w[s][2 * lane]) =
                make_float2(fexp(suf + ex0) * d0, fexp(suf + ex1) * d1);
            __syncwarp();
            if (lane == 0) mbar_arrive(&X->wfull[s]);
            suf += tot;
            if (++s == nst) {
                s = 0;
                ph ^= 1;
            }
        }
        if (okw && half == 0 && lane == 0) lsum_part[bh * g.NPc + part] = suf;
    } else {
        // builders: warps 2..9 (256 threads).  Thread: one 16-byte chunk (8
        // channels) of four consecutive token rows of V.
        constexpr int kNB = 32 * kABuild;
        const int tb = threadIdx.x - 64;
        const int vb = (tb >> 3) & 1, vc = tb & 7, r0 = (tb >> 4) * 4;
        // zero rows 2..15 of every stage's weight tile (rows 0 and 1 are
        // rewritten for each chunk)
        for (int i = tb; i < nst * (kAWB - 256) / 16; i += kNB) {
            const int st = i / ((kAWB - 256) / 16), r = i % ((kAWB - 256) / 16);
            *reinterpret_cast<uint4 *>(stage(st) + lay.wb + 256 + r * 16) = make_uint4(0, 0, 0, 0);
        }
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int it = 0; it < n; ++it) {
            // each builder warp runs on its own (no named barrier in the loop)
            bool okw = mbar_wait(&X->wfull[s], ph, abort_flag, err, KID_SCAN_TC_STATE, 7) &&
                       mbar_wait(&X->full[s], ph, abort_flag, err, KID_SCAN_TC_STATE, 4);
            if (!__all_sync(0xffffffffu, okw)) {
                ok = false;
                break;
            }
            uint8_t *const st = stage(s);
            const float *__restrict__ wv = X->w[s];
            // weight rows of the z product: row 0 = bf16(w), row 1 = the remainder
            if (tb < kC) {
                const float wmine = wv[tb];
                const __nv_bfloat16 wh = __float2bfloat16_rn(wmine);
                const __nv_bfloat16 wl = __float2bfloat16_rn(wmine - __bfloat162float(wh));
                const int c8 = tb >> 3, e = tb & 7;
                *reinterpret_cast<__nv_bfloat16 *>(st + lay.wb + (c8 << 4) + 2 * e) = wh;
                *reinterpret_cast<__nv_bfloat16 *>(st + lay.wb + 128 + ((c8 ^ 1) << 4) + 2 * e) = wl;
            }
            // w (.) V in place as bf16, the rounding remainder into its own tile
            uint8_t *__restrict__ vt = st + lay.v + vb * kBlk;
            uint8_t *__restrict__ vlt = st + lay.vl + vb * kBlk;
            uint4 xv[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) xv[jj] = *reinterpret_cast<const uint4 *>(vt + sw128_off(r0 + jj, vc));
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                uint32_t *ph32 = reinterpret_cast<uint32_t *>(&xv[jj]);
                uint4 lo;
                uint32_t *pl = reinterpret_cast<uint32_t *>(&lo);
                const float wj = wv[r0 + jj];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 vv = unpack_bf16x2(ph32[e]);
                    const float t0 = wj * vv.x, t1 = wj * vv.y;
                    ph32[e] = pack_bf16x2(t0, t1);
                    if (split) {
                        const float2 hf = unpack_bf16x2(ph32[e]);
                        pl[e] = pack_bf16x2(t0 - hf.x, t1 - hf.y);
                    }
                }
                const uint32_t off = sw128_off(r0 + jj, vc);
                *reinterpret_cast<uint4 *>(vt + off) = xv[jj];
                if (split) *reinterpret_cast<uint4 *>(vlt + off) = lo;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&X->built[s]);
            if (++s == nst) {
                s = 0;
                ph ^= 1;
            }
        }
        if (ok && mbar_wait(&X->done, 0, abort_flag, err, KID_SCAN_TC_STATE, 5)) {
            tc_fence_after();
            // two warps per TMEM lane quarter: features 0..127 and 128..255
            const int q = warp & 3;
            const int ch = 32 * q + lane;
            const int fh = (warp - 2) >> 2;
            const int64_t pidx = bh * g.NPc + part;
            float *Sp = S_part + pidx * (int64_t)kF * g.dv + dv0 + ch;
            for (int c0 = fh * 128; c0 < fh * 128 + 128; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(tmem + c0 + ((uint32_t)(32 * q) << 16), r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) Sp[(int64_t)(c0 + j) * g.dv] = __uint_as_float(r[j]);
            }
            if (fh == 0) {
                // z: TMEM lane = feature within the CTA's half, columns 0 (w hi) and 1 (w lo)
                uint32_t r[16];
                tmem_ld16(tmem + 256 + ((uint32_t)(32 * q) << 16), r);
                tmem_wait_ld();
                z_part[pidx * kF + half * 128 + ch] = __uint_as_float(r[0]) + __uint_as_float(r[1]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ phase B

// Per (batch, head) and 4-element groups of the state: walks the parts in
// order,
//   acc <- exp(lsum_p) acc + part_p,
// storing the state at each segment start and, when every part was
// computed, the final state.  Elements [0, F*dv) are S, [F*dv, F*dv + F) are z.
// A thread owns COLS groups, 256 apart (coalesced), and loads PF parts of all
// of them before combining them, so that enough bytes are in flight to stream
// the parts at HBM speed: many heads take COLS = 2, PF = 2; few heads (and
// then many parts) COLS = 1, PF = 8 (more CTAs, deeper prefetch).
template <int COLS, int PF>
__global__ void __launch_bounds__(256, 4)
scan_carry_kernel(Geo g, const float *__restrict__ S_part, const float *__restrict__ z_part,
                  const float *__restrict__ lsum_part, const float *__restrict__ S0, const float *__restrict__ z0,
                  float *__restrict__ S_start, float *__restrict__ z_start, float *__restrict__ S_out,
                  float *__restrict__ z_out) {
    const int64_t bh = blockIdx.y;
    const int nS = kF * g.dv;
    const int pps = g.seg_chunks / g.part_chunks;
    // group j: element e = 4 * col; S element e, or z element e - nS
    auto elem = [&](const float *S, const float *z, int64_t blk, int c) -> const float * {
        const int e = 4 * c;
        return e < nS ? S + blk * nS + e : z + blk * kF + (e - nS);
    };
    auto elem_w = [&](float *S, float *z, int64_t blk, int c) -> float * {
        const int e = 4 * c;
        return e < nS ? S + blk * nS + e : z + blk * kF + (e - nS);
    };
    const int ncol = (nS + kF) / 4;
    int col[COLS];
    float4 acc[COLS];
#pragma unroll
    for (int j = 0; j < COLS; ++j) {
        col[j] = (blockIdx.x * COLS + j) * blockDim.x + threadIdx.x;
        acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (col[j] < ncol) {
            const bool isz = 4 * col[j] >= nS;
            if (isz ? z0 != nullptr : S0 != nullptr)
                acc[j] = *reinterpret_cast<const float4 *>(elem(S0, z0, bh, col[j]));
        }
    }
    for (int p0 = 0; p0 <= g.NPc; p0 += PF) {
        float4 v[PF][COLS];
        float lg[PF];
#pragma unroll
        for (int u = 0; u < PF; ++u) {
            const int p = p0 + u;
            lg[u] = p < g.NPc ? lsum_part[bh * g.NPc + p] : 0.f;
#pragma unroll
            for (int j = 0; j < COLS; ++j)
                v[u][j] = (p < g.NPc && col[j] < ncol)
                              ? *reinterpret_cast<const float4 *>(elem(S_part, z_part, bh * g.NPc + p, col[j]))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < PF; ++u) {
            const int p = p0 + u;
            if (p > g.NPc) break;
            if (p > 0 && p % pps == 0 && p / pps < g.G) {
#pragma unroll
                for (int j = 0; j < COLS; ++j)
                    if (col[j] < ncol)
                        *reinterpret_cast<float4 *>(elem_w(S_start, z_start, bh * g.G + p / pps, col[j])) = acc[j];
            }
            if (p < g.NPc) {
                const float gam = expf(lg[u]);
#pragma unroll
                for (int j = 0; j < COLS; ++j)
                    acc[j] = make_float4(fmaf(gam, acc[j].x, v[u][j].x), fmaf(gam, acc[j].y, v[u][j].y),
                                         fmaf(gam, acc[j].z, v[u][j].z), fmaf(gam, acc[j].w, v[u][j].w));
            }
        }
    }
    if (g.NPc == g.NP) {
#pragma unroll
        for (int j = 0; j < COLS; ++j) {
            if (col[j] >= ncol) continue;
            const bool isz = 4 * col[j] >= nS;
            if (isz ? z_out != nullptr : S_out != nullptr)
                *reinterpret_cast<float4 *>(elem_w(S_out, z_out, bh, col[j])) = acc[j];
        }
    }
}

// ------------------------------------------------------------------ phase C

// TMEM columns
constexpr uint32_t kColS = 0;    // S^T fp32        [128 value lanes x 256 features]
constexpr uint32_t kColSB = 256; // S^T bf16 pairs  [128 x 128]
constexpr uint32_t kColO = 384;  // O^T fp32        [128 x 64 tokens]
constexpr uint32_t kColP = 448;  // [phiK; phiQ] phiK^T fp32 [128 x 64]; lanes 64..127 = P

constexpr int kHelpers = 160;    // threads of the five helper warps

struct CAux {
    float cum[2][kC];
    float ck[2][kC];     // key-side cums: cum_j - log2(Delta_j) (= cum_j without the step-scaled input)
    float bq[2][32];     // e^(cum_(j|7) - cum_j), j < 32: column factors of the below-diagonal quadrant
    float qs[2][kC];
    float w[2][kC];
    float rden[2][kC];   // 1 / den
    float dint[2][2][kC];   // per chunk parity: row sums of Pt, [0] columns 0..31, [1] columns 32..63
    float dotq[2][4][kC];   // per chunk parity: phiq_i . z_prev over each quarter of the features
    alignas(16) float zb[2][kF];   // z after chunk c in zb[c & 1]; the start z in zb[1]
    float gam[2];
    float redd[4];
    // per stage: the phiQ blocks and the phiK + V blocks are loaded and
    // released separately
    uint64_t fullq[2], fullkv[2], emptyq[2], emptykv[2];
    uint64_t stg_free[2];   // the stage's Pt buffer, used to stage outputs, has been read out
    uint64_t p_full[2], p_consumed, epib_done, o_full, o_empty, s_full, sbf_ready;
    uint64_t den_ready[2], den_free[2];   // 1 / den of a stage written / read
    uint64_t pro_full[3];                 // start-state rounds landed (prologue staging)
    uint64_t dec_full[2], dec_free[2];    // decay vectors of a parity written / read
    uint64_t zfull[2], zfree[2];          // z buffer of a parity written / read
    int szero;           // gamma of the next state MMA's chunk is 0: that MMA overwrites S
    uint32_t tmem;
    int abort;
};

// Phase C stage: for each 64-feature block bb, the 64 phiK rows and the 64
// phiQ rows are stored back to back ([K | Q], 16 KB), so that one M = 128
// operand [phiK; phiQ] gives the score tile P = phiQ phiK^T in TMEM lanes
// 64..127 with the plain 128-lane accumulator layout (lanes 0..63 hold
// phiK phiK^T, which is not used).  Lanes 64..127 are read by warps 2, 3, 6,
// 7, which share no SM sub-partition with the TMA and MMA warps.
constexpr int kQKBlk = 2 * kBlk;                       // [K | Q] of one feature block
constexpr int kCStage = 4 * kQKBlk + kTileV;           // Q, K, V of one chunk
constexpr int kCPBytes = 2 * kC * 128;                 // Pt as bf16 hi (8 KB) then lo (8 KB)
constexpr int kCOffP = 2 * kCStage;                    // one Pt buffer per stage
constexpr int kCOffVt = kCOffP + 2 * kCPBytes;         // w (.) V of the current chunk
constexpr int kCOffAux = kCOffVt + kTileV;
constexpr int kCSmem = kCOffAux + (int)sizeof(CAux) + 1024;
static_assert(kCSmem <= 227 * 1024, "phase C shared memory");

struct OutArgs {
    Geo g;
    const float *dt, *A_log;
    void *o;
    int o_f32;                       // o stored as fp32 (else bf16)
    int dt_scaled;                   // step-scaled input: key j weighted by softplus(dt_j)
    const float *S0, *z0;            // segment 0 start state (caller layout) or null
    const float *S_start, *z_start;  // segments >= 1: [BH][G][F*dv], [BH][G][F]
    const float *gate;               // o is multiplied by this (fp32, layout of o) before it is stored, or null
};

// dt of token t0 + tg for the first 64 threads of a group; -inf (log a = 0)
// past the end of the sequence, for the other threads, or without dt.  The
// raw value is fetched a chunk ahead and turned into log a when it is used,
// so the load's latency is never waited for.
__device__ __forceinline__ float token_dt(const OutArgs &a, int64_t b, int h, int64_t t0, int tg) {
    if (tg >= 0 && tg < kC && a.dt && t0 + tg < a.g.L) return a.dt[(b * a.g.L + t0 + tg) * a.g.H + h];
    return -INFINITY;
}

// sum of the 64 per-token values l over the first two warps of a 128-thread
// group (named barrier `bar_id`)
__device__ __forceinline__ float chunk_total(float l, int tg, float *red, int bar_id) {
    l = warp_sum(l);
    if ((tg & 31) == 0 && tg < kC) red[tg >> 5] = l;
    named_sync(bar_id, 128);
    const float tot = red[0] + red[1];
    named_sync(bar_id, 128);
    return tot;
}

// Warp roles (19 warps):
//   0      TMA producer (phiQ, phiK, V of each chunk; two stages)
//   1      MMA issuer
//   2, 3, 14, 5..9  compute group (256 threads): per chunk the decayed score
//          tile Pt (three 32 x 32 quadrants: rows 0..31 need only columns
//          0..31), w (.) V, the scaled queries e^cum (.) phiQ with
//          phiq . z_prev, and the denominators
//   10..13 outputs: o = O^T / den for the chunk, staged in the chunk's Pt
//          buffer (dead once the PV product is complete) and written by TMA
//          bulk stores
//   15..18 z and state pass: the chunk's weighted key-feature sums and z (two
//          features per thread, as soon as the chunk's phiK has landed), then
//          S^T (fp32, TMEM) -> bf16 copy for the next readout and S^T <- gamma
//          S^T before the next state MMA.  The outputs of a chunk and its
//          state pass run at the same time on separate warps, so the next
//          readout waits only for the state pass.
//   4      decay vectors, one chunk ahead of the compute group (prefix sums
//          of log a, e^cum, e^(cum_last - cum), the below-diagonal column
//          factors, gamma), two tokens per lane
// The output and state-pass roles each take four consecutive warps, so that
// every TMEM lane quarter is read by one warp of each.
// Per chunk the MMA issuer runs: scores of the next chunk, then the readout
// O^T = S^T (e^cum phiQ)^T, O^T += V^T Pt^T (hi and lo), and the state
// update S^T += (w V)^T phiK.
constexpr int kCThreads = 608;

// GATE: o is multiplied by the mixer's activated gate before it is stored (a
// separate instantiation, so that the plain scan carries none of its code: the
// kernel's roles together already run more code per chunk than the
// instruction cache holds).
template <bool GATE>
__global__ void __launch_bounds__(kCThreads, 1)
scan_out_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                const __grid_constant__ CUtensorMap tms, OutArgs a, DevErr err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    CAux *X = (CAux *)(smem + kCOffAux);
    const Geo &g = a.g;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = blockIdx.x & 1;
    const int seg = (blockIdx.x >> 1) % g.G;
    const int64_t bh = (blockIdx.x >> 1) / g.G;
    const int64_t b = bh / g.H;
    const int h = (int)(bh % g.H);
    const int dv0 = half * kN;
    const int c_begin = seg * g.seg_chunks;
    const int c_end = min(g.nchunks, c_begin + g.seg_chunks);
    const int nch = c_end - c_begin;
    const float alog = a.dt ? a.A_log[h] : 0.f;
    volatile int *abort_flag = &X->abort;
    const uint32_t sbase = smem_u32(smem);
    // block bb of phiK at sK(s) + bb * kQKBlk, of phiQ at sQ(s) + bb * kQKBlk
    auto sQ = [&](int s) { return sbase + s * kCStage + kBlk; };
    auto sK = [&](int s) { return sbase + s * kCStage; };
    auto sV = [&](int s) { return sbase + s * kCStage + 4 * kQKBlk; };
    auto sP = [&](int s) { return sbase + kCOffP + s * kCPBytes; };
    const uint32_t sVt = sbase + kCOffVt;
    // pointers to the same buffers, for CUDA-core accesses
    auto gQ = [&](int s) { return smem + s * kCStage + kBlk; };
    auto gK = [&](int s) { return smem + s * kCStage; };
    auto gV = [&](int s) { return smem + s * kCStage + 4 * kQKBlk; };
    auto gP = [&](int s) { return smem + kCOffP + s * kCPBytes; };
    uint8_t *const gVt = smem + kCOffVt;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&X->fullq[s], 1);
            mbar_init(&X->fullkv[s], 1);
            mbar_init(&X->emptyq[s], 1);
            mbar_init(&X->stg_free[s], 1);
            // phiK + V: the chunk's MMAs and the four state-pass warps' key-feature sums
            mbar_init(&X->emptykv[s], 5);
        }
        mbar_init(&X->p_full[0], 1);   // the scores of a chunk of each parity
        mbar_init(&X->p_full[1], 1);
        mbar_init(&X->p_consumed, 3);   // the three score-quadrant warps have loaded P
        mbar_init(&X->epib_done, 1);
        mbar_init(&X->o_full, 1);
        mbar_init(&X->o_empty, 4);      // one arrival per output warp
        mbar_init(&X->s_full, 1);
        mbar_init(&X->sbf_ready, 4);     // one arrival per state-pass warp
        for (int s = 0; s < 2; ++s) {
            mbar_init(&X->den_ready[s], 1);
            mbar_init(&X->den_free[s], 4);
        }
        for (int r = 0; r < 3; ++r) mbar_init(&X->pro_full[r], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&X->dec_full[s], 1);
            mbar_init(&X->dec_free[s], 5);   // the compute group and the four state-pass warps
            mbar_init(&X->zfull[s], 4);      // one arrival per state-pass warp
            mbar_init(&X->zfree[s], 1);
        }
        X->abort = 0;
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(&X->tmem, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = X->tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmq);
            tma_prefetch_desc(&tmk);
            tma_prefetch_desc(&tmv);
            int nkv = 0, nq = 0;   // chunks whose phiK + V / phiQ loads were issued
            for (int it = 0; it < nch; ++it) {
                const int s = it & 1;
                const uint32_t par = ((it >> 1) & 1) ^ 1;
                const int t0 = (c_begin + it) * kC;
                uint8_t *q = smem + s * kCStage;
                if (!mbar_wait(&X->emptykv[s], par, abort_flag, err, KID_SCAN_TC_OUT, 1)) break;
                mbar_arrive_expect_tx(&X->fullkv[s], 4 * kBlk + kTileV);
                for (int bb = 0; bb < 4; ++bb)
                    tma_load_4d(q + bb * kQKBlk, &tmk, &X->fullkv[s], bb * 64, h, t0, (int)b);
                for (int bb = 0; bb < 2; ++bb)
                    tma_load_4d(q + 4 * kQKBlk + bb * kBlk, &tmv, &X->fullkv[s], dv0 + bb * 64, h, t0, (int)b);
                ++nkv;
                if (!mbar_wait(&X->emptyq[s], par, abort_flag, err, KID_SCAN_TC_OUT, 15)) break;
                mbar_arrive_expect_tx(&X->fullq[s], 4 * kBlk);
                for (int bb = 0; bb < 4; ++bb)
                    tma_load_4d(q + bb * kQKBlk + kBlk, &tmq, &X->fullq[s], bb * 64, h, t0, (int)b);
                ++nq;
            }
            // no copy may still be landing when the CTA exits
            for (int j = nkv - 2; j < nkv; ++j) {
                if (j < 0) continue;
                for (uint32_t i = 0; i < kWaitPolls; ++i)
                    if (mbar_try_wait(&X->fullkv[j & 1], (j >> 1) & 1)) break;
            }
            for (int j = nq - 2; j < nq; ++j) {
                if (j < 0) continue;
                for (uint32_t i = 0; i < kWaitPolls; ++i)
                    if (mbar_try_wait(&X->fullq[j & 1], (j >> 1) & 1)) break;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (elect_one()) {
            constexpr uint32_t idP = idesc_bf16(128, 64, false, false);    // [phiK; phiQ] phiK^T
            constexpr uint32_t idOi = idesc_bf16(128, 64, false, false);   // O^T = S^T phiQ~^T
            constexpr uint32_t idOa = idesc_bf16(128, 64, true, false);    // O^T += V^T Pt^T
            constexpr uint32_t idS = idesc_bf16(128, 256, true, true);     // S^T += (wV)^T phiK
            // score MMA of chunk c: [phiK; phiQ] phiK^T into the P columns,
            // once the compute group has loaded P of chunk c - 1
            auto issue_scores = [&](int c) -> bool {
                const int sc = c & 1;
                if (!mbar_wait(&X->fullkv[sc], (c >> 1) & 1, abort_flag, err, KID_SCAN_TC_OUT, 2)) return false;
                if (!mbar_wait(&X->fullq[sc], (c >> 1) & 1, abort_flag, err, KID_SCAN_TC_OUT, 16)) return false;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < kF / 16; ++k) {
                    const uint32_t off = (k >> 2) * kQKBlk + (k & 3) * 32;
                    mma_ss(tmem + kColP, desc_k_sw128(sK(sc) + off), desc_k_sw128(sK(sc) + off), idP,
                           k > 0 ? 1u : 0u);
                }
                mma_commit(&X->p_full[c & 1]);
                return true;
            };
            bool ok = nch > 0 && issue_scores(0);
            for (int it = 0; ok && it < nch; ++it) {
                const int s = it & 1;
                const uint32_t par = it & 1;
                // the next chunk's scores go as soon as this chunk's P has been
                // loaded into registers, so that they run under the compute
                // group's work on this chunk
                if (it + 1 < nch) {
                    if (!mbar_wait(&X->p_consumed, par, abort_flag, err, KID_SCAN_TC_OUT, 3)) break;
                    if (!issue_scores(it + 1)) break;
                }
                if (!mbar_wait(&X->epib_done, par, abort_flag, err, KID_SCAN_TC_OUT, 4)) break;
                if (!mbar_wait(&X->sbf_ready, par, abort_flag, err, KID_SCAN_TC_OUT, 5)) break;
                if (!mbar_wait(&X->o_empty, par ^ 1, abort_flag, err, KID_SCAN_TC_OUT, 6)) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < kF / 16; ++k) {
                    const uint32_t off = (k >> 2) * kQKBlk + (k & 3) * 32;
                    mma_ts(tmem + kColO, tmem + kColSB + k * 8, desc_k_sw128(sQ(s) + off), idOi,
                           k > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int k = 0; k < kC / 16; ++k) {
                    const uint64_t va = desc_mn_sw128(sV(s) + k * 2048, kBlk, 1024);
                    mma_ss(tmem + kColO, va, desc_k_sw128(sP(s) + k * 32), idOa, 1u);
                    mma_ss(tmem + kColO, va, desc_k_sw128(sP(s) + kC * 128 + k * 32), idOa, 1u);
                }
                mma_commit(&X->o_full);
                // a chunk whose decay gamma underflowed to 0 forgets the state:
                // its update overwrites S (the state pass then skipped S <- 0 S)
                const uint32_t acc0 = X->szero ? 0u : 1u;
#pragma unroll
                for (int k = 0; k < kC / 16; ++k)
                    mma_ss(tmem + kColS, desc_mn_sw128(sVt + k * 2048, kBlk, 1024),
                           desc_mn_sw128(sK(s) + k * 2048, kQKBlk, 1024), idS, k == 0 ? acc0 : 1u);
                mma_commit(&X->s_full);
                mma_commit(&X->emptykv[s]);
                mma_commit(&X->emptyq[s]);
            }
        }
    } else if ((warp >= 2 && warp < 10 && warp != 4) || warp == 14) {
        // ------------------------------------------------------------ compute group
        // warps 2, 3, 14, 5, 6, 7, 8, 9 (warp 14 stands in for warp 4, which
        // runs the decay vectors on the less busy SM sub-partition 0)
        const int gt = (warp == 14 ? 2 : warp - 2) * 32 + lane;   // 0..255
        const int q = warp & 3;            // TMEM lane quarter of this warp
        // every exit from this loop is taken by the whole group (after a
        // barrier-AND), so no thread is left waiting at a named barrier
        bool ok = named_sync_and(1, 256, true);
        bool dok = true;   // the denominator warps' step (4) of the previous chunk went through
        for (int it = 0; it < nch; ++it) {
            const int s = it & 1;
            // (1) the chunk's decay vectors (from the decay warp; chunk 0: the
            // state prologue, which stages in the Pt and w V buffers, must also
            // be complete before they are written).  There is no group barrier
            // before the chunk's work: the denominator warps may still be on
            // step (4) of chunk it - 1, and the group meets at the end of step
            // (3), where a failed wait of any thread ends the loop for all.
            // (2) the chunk's stage is loaded and its score MMA has completed:
            // every thread waits for both -- the score MMA reads phiQ of the
            // stage, which step (3) scales in place.  The scores of the two
            // chunk parities complete on barriers of their own, so a waiter
            // never meets the next chunk's phase.  Score-quadrant warps
            // (P rows 0..31 in TMEM lanes 64..95, rows 32..63 in lanes 96..127):
            // warp 2: rows 0..31 x columns 0..31 (and the zeros of columns
            // 32..63); warp 3: rows 32..63 x columns 0..31 (all below the
            // diagonal); warp 7: rows 32..63 x columns 32..63.  Each reads its
            // quadrant from TMEM 8 columns at a time as it goes and then
            // arrives on p_consumed (count 3), after which the next chunk's
            // scores may overwrite it.
            const bool pwarp = warp == 2 || warp == 3 || warp == 7;
            bool okw = dok && mbar_wait(&X->dec_full[s], (it >> 1) & 1, abort_flag, err, KID_SCAN_TC_OUT, 22) &&
                       (it > 0 || mbar_wait(&X->sbf_ready, 0, abort_flag, err, KID_SCAN_TC_OUT, 21)) &&
                       mbar_wait(&X->fullkv[s], (it >> 1) & 1, abort_flag, err, KID_SCAN_TC_OUT, 8) &&
                       mbar_wait(&X->fullq[s], (it >> 1) & 1, abort_flag, err, KID_SCAN_TC_OUT, 17) &&
                       mbar_wait(&X->p_full[s], (it >> 1) & 1, abort_flag, err, KID_SCAN_TC_OUT, 7);
            okw = __all_sync(0xffffffffu, okw);
            tc_fence_after();
            const int i = 32 * (q - 2) + lane;
            const int jc = warp == 7 ? 32 : 0;
            const uint32_t ptm = tmem + kColP + jc + ((uint32_t)(32 * q) << 16);
            if (pwarp) {
                // (The 8-column block loops below stay rolled: the kernel's roles
                // together run more code per chunk than the instruction cache
                // holds, and rolling them measured faster.)
                // Pt = P * exp(cum_i - cum_j) on j <= i, as bf16 hi + lo (the PV
                // product runs on both: a few-token weighted average would
                // otherwise carry the 2^-9 rounding of each weight), and row sums
                const bool masked = warp != 3;
                // the buffer staged chunk it - 2's outputs
                okw = __all_sync(0xffffffffu, okw && mbar_wait(&X->stg_free[s], ((it >> 1) & 1) ^ 1, abort_flag,
                                                                   err, KID_SCAN_TC_OUT, 18));
                if (okw && !masked) {
                    // every 8-column block lies below the diagonal:
                    // e^(cum_i - cum_j) = e^(cum_i - cum_b) e^(cum_b - cum_j), b the
                    // block's last column, both factors <= 1
                    const float ci = X->cum[s][i];
                    uint8_t *__restrict__ prow = gP(s);
                    float2 rs2 = make_float2(0.f, 0.f);
#pragma unroll 1
                    for (int c4 = 0; c4 < 4; ++c4) {
                        uint32_t pr[8];
                        tmem_ld8(ptm + 8 * c4, pr);
                        const float ai = ex2_approx(ci - X->cum[s][8 * c4 + 7]);
                        const float2 a2 = make_float2(ai, ai);
                        const float4 ba = *reinterpret_cast<const float4 *>(&X->bq[s][8 * c4]);
                        const float4 bb = *reinterpret_cast<const float4 *>(&X->bq[s][8 * c4 + 4]);
                        const float2 bv[4] = {make_float2(ba.x, ba.y), make_float2(ba.z, ba.w),
                                              make_float2(bb.x, bb.y), make_float2(bb.z, bb.w)};
                        uint4 hi, lo;
                        uint32_t *pk = reinterpret_cast<uint32_t *>(&hi);
                        uint32_t *pl = reinterpret_cast<uint32_t *>(&lo);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 ev = mul2(make_float2(__uint_as_float(pr[2 * e]), __uint_as_float(pr[2 * e + 1])),
                                                   mul2(a2, bv[e]));
                            pk[e] = pack_bf16x2(ev.x, ev.y);
                            const float2 r = sub2(ev, unpack_bf16x2(pk[e]));
                            pl[e] = pack_bf16x2(r.x, r.y);
                            rs2 = add2(rs2, ev);
                        }
                        *reinterpret_cast<uint4 *>(prow + sw128_off(i, c4)) = hi;
                        *reinterpret_cast<uint4 *>(prow + kC * 128 + sw128_off(i, c4)) = lo;
                    }
                    X->dint[s][0][i] = rs2.x + rs2.y;
                } else if (okw) {
                    const float ci = X->cum[s][i];
                    const float2 ci2 = make_float2(ci, ci);
                    const float *__restrict__ cj = X->ck[s] + jc;
                    uint8_t *__restrict__ prow = gP(s);
                    float2 rs2 = make_float2(0.f, 0.f);
#pragma unroll 1
                    for (int c4 = 0; c4 < 4; ++c4) {
                        uint32_t pr[8];
                        tmem_ld8(ptm + 8 * c4, pr);
                        uint4 hi, lo;
                        uint32_t *pk = reinterpret_cast<uint32_t *>(&hi);
                        uint32_t *pl = reinterpret_cast<uint32_t *>(&lo);
                        const float4 ca = *reinterpret_cast<const float4 *>(cj + c4 * 8);
                        const float4 cb = *reinterpret_cast<const float4 *>(cj + c4 * 8 + 4);
                        const float2 cv[4] = {make_float2(ca.x, ca.y), make_float2(ca.z, ca.w),
                                              make_float2(cb.x, cb.y), make_float2(cb.z, cb.w)};
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = jc + c4 * 8 + 2 * e;
                            const float2 d = sub2(ci2, cv[e]);
                            float2 ev = mul2(make_float2(__uint_as_float(pr[2 * e]), __uint_as_float(pr[2 * e + 1])),
                                             make_float2(ex2_approx(d.x), ex2_approx(d.y)));
                            if (masked && j > i) ev.x = 0.f;
                            if (masked && j + 1 > i) ev.y = 0.f;
                            pk[e] = pack_bf16x2(ev.x, ev.y);
                            const float2 r = sub2(ev, unpack_bf16x2(pk[e]));
                            pl[e] = pack_bf16x2(r.x, r.y);
                            rs2 = add2(rs2, ev);
                        }
                        const int cc = (jc >> 3) + c4;
                        *reinterpret_cast<uint4 *>(prow + sw128_off(i, cc)) = hi;
                        *reinterpret_cast<uint4 *>(prow + kC * 128 + sw128_off(i, cc)) = lo;
                        if (warp == 2) {
                            // rows 0..31 x columns 32..63 are zero
                            *reinterpret_cast<uint4 *>(prow + sw128_off(i, 4 + c4)) = make_uint4(0u, 0u, 0u, 0u);
                            *reinterpret_cast<uint4 *>(prow + kC * 128 + sw128_off(i, 4 + c4)) =
                                make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                    X->dint[s][jc ? 1 : 0][i] = rs2.x + rs2.y;
                }
                // P has been read: the next chunk's scores may overwrite it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&X->p_consumed);
            } else {
                // helpers (warps 14, 5, 6, 8, 9)
                const int hx = (warp == 14 ? 0 : (warp < 7 ? warp - 4 : warp - 5)) * 32 + lane;   // 0..159
                const float *__restrict__ wv = X->w[s];
                // w (.) V into its own tile, once the previous chunk's state MMA
                // has read that tile
                if (it > 0) okw = mbar_wait(&X->s_full, (it - 1) & 1, abort_flag, err, KID_SCAN_TC_OUT, 13) && okw;
                okw = __all_sync(0xffffffffu, okw);
                if (okw) {
                    const uint8_t *__restrict__ vsrc = gV(s);
#pragma unroll 1
                    for (int u = hx; u < kC * 16; u += kHelpers) {
                        const int j = u >> 4, ci = u & 15;
                        const uint32_t off = (uint32_t)((ci >> 3) * kBlk) + sw128_off(j, ci & 7);
                        uint4 vv = *reinterpret_cast<const uint4 *>(vsrc + off);
                        const float wj = wv[j];
                        const uint32_t w2 = pack_bf16x2(wj, wj);
                        uint32_t *pv = reinterpret_cast<uint32_t *>(&vv);
#pragma unroll
                        for (int e = 0; e < 4; ++e) pv[e] = mul_bf16x2(pv[e], w2);
                        *reinterpret_cast<uint4 *>(gVt + off) = vv;
                    }
                }
            }
            // (3) every thread: the query row scaled by e^cum_i, in place, and
            // phiq_i . z_prev over one quarter of the features (on the unscaled
            // bf16 values; the scale is applied to the sum).  z_prev = z after
            // chunk it - 1 (the start z for it = 0), from the state-pass warps: buffer
            // (it - 1) & 1, whose (it >> 1)-th write it is.
            okw = __all_sync(0xffffffffu, okw && mbar_wait(&X->zfull[(it - 1) & 1], (it >> 1) & 1, abort_flag,
                                                               err, KID_SCAN_TC_OUT, 24));
            if (okw) {
                const int i = gt & 63, qf = gt >> 6;
                const float qsi = X->qs[s][i];
                const uint32_t q2 = pack_bf16x2(qsi, qsi);
                uint8_t *__restrict__ qb = gQ(s) + qf * kQKBlk;
                const float *__restrict__ zq = X->zb[(it - 1) & 1] + qf * 64;
                float2 d2 = make_float2(0.f, 0.f);
#pragma unroll 1
                for (int k0 = 0; k0 < 8; k0 += 2) {
                    uint4 v[2];
#pragma unroll
                    for (int k = 0; k < 2; ++k) v[k] = *reinterpret_cast<const uint4 *>(qb + sw128_off(i, k0 + k));
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        uint32_t *pv = reinterpret_cast<uint32_t *>(&v[k]);
                        const float4 za = *reinterpret_cast<const float4 *>(zq + (k0 + k) * 8);
                        const float4 zb = *reinterpret_cast<const float4 *>(zq + (k0 + k) * 8 + 4);
                        const float2 zz[4] = {make_float2(za.x, za.y), make_float2(za.z, za.w),
                                              make_float2(zb.x, zb.y), make_float2(zb.z, zb.w)};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            d2 = fma2(unpack_bf16x2(pv[e]), zz[e], d2);
                            pv[e] = mul_bf16x2(pv[e], q2);
                        }
                    }
#pragma unroll
                    for (int k = 0; k < 2; ++k) *reinterpret_cast<uint4 *>(qb + sw128_off(i, k0 + k)) = v[k];
                }
                X->dotq[s][qf][i] = d2.x + d2.y;
            }
            fence_proxy_async_smem();
            ok = named_sync_and(1, 256, okw);
            if (!ok) break;
            if (gt == 0) {
                mbar_arrive(&X->epib_done);
                mbar_arrive(&X->zfree[(it - 1) & 1]);   // z_prev has been read
            }
            // (4) denominators, on warps 8 and 9 (helpers, on the SM
            // sub-partitions the quadrant warps do not use), once the outputs of
            // chunk it - 2 have read this stage's 1 / den; the chunk's MMAs and
            // the other warps' chunk it + 1 run meanwhile (the row sums and dot
            // products are kept per chunk parity).  Then the chunk's decay
            // vectors have had their last reader.
            if (gt >= 256 - kC) {
                const int i = gt - (256 - kC);
                dok = mbar_wait(&X->den_free[s], ((it >> 1) & 1) ^ 1, abort_flag, err, KID_SCAN_TC_OUT, 14);
                const float dq = (X->dotq[s][0][i] + X->dotq[s][1][i]) + (X->dotq[s][2][i] + X->dotq[s][3][i]);
                // the inter-chunk term with the query scale as the readout used it
                // (rounded to bf16), so that numerator and denominator agree
                const float qsr = __bfloat162float(__float2bfloat16_rn(X->qs[s][i]));
                const float den = X->dint[s][0][i] + (i >= 32 ? X->dint[s][1][i] : 0.f) + qsr * dq;
                X->rden[s][i] = 1.f / den;
                named_sync(3, 64);
                if (i == 0) {
                    mbar_arrive(&X->den_ready[s]);
                    mbar_arrive(&X->dec_free[s]);
                }
            }
        }
    } else if (warp == 4) {
        // ------------------------------------------------------------ decay vectors
        // Iteration c: the decay vectors of chunk c, one chunk ahead of the
        // compute group.  Lane: tokens 2 lane and 2 lane + 1 (dt two chunks
        // ahead).
        float da[2], db[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            da[i] = i < nch ? token_dt(a, b, h, (int64_t)(c_begin + i) * kC, 2 * lane) : -INFINITY;
            db[i] = i < nch ? token_dt(a, b, h, (int64_t)(c_begin + i) * kC, 2 * lane + 1) : -INFINITY;
        }
        for (int c = 0; c < nch; ++c) {
          {
            const int sc = c & 1;
            const float l0 = hm_log_decay(da[0], alog) * kLog2e, l1 = hm_log_decay(db[0], alog) * kLog2e;
            // step-scaled input: log2 of softplus(dt) of the two tokens, added
            // to every factor that weights a key (-inf past the sequence end)
            const float g0 = a.dt_scaled ? lg2_approx(hm_step_size(da[0])) : 0.f;
            const float g1 = a.dt_scaled ? lg2_approx(hm_step_size(db[0])) : 0.f;
            da[0] = da[1];
            db[0] = db[1];
            da[1] = c + 2 < nch ? token_dt(a, b, h, (int64_t)(c_begin + c + 2) * kC, 2 * lane) : -INFINITY;
            db[1] = c + 2 < nch ? token_dt(a, b, h, (int64_t)(c_begin + c + 2) * kC, 2 * lane + 1) : -INFINITY;
            // inclusive prefix sums of the token pairs over the lanes: x = cum
            // at token 2 lane + 1
            float x = l0 + l1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            const float x0 = x - l1;                                   // cum at token 2 lane
            const float total = __shfl_sync(0xffffffffu, x, 31);
            const float xe = __shfl_sync(0xffffffffu, x, lane | 3);   // cum at the end of the 8-block
            // the parity's buffers were last read during chunk c - 2
            bool okw = c < 2 || mbar_wait(&X->dec_free[sc], ((c >> 1) & 1) ^ 1, abort_flag, err, KID_SCAN_TC_OUT, 23);
            if (!__all_sync(0xffffffffu, okw)) break;
            if (lane < 16)
                *reinterpret_cast<float2 *>(&X->bq[sc][2 * lane]) =
                    make_float2(ex2_approx(xe - x0 + g0), ex2_approx(xe - x + g1));
            *reinterpret_cast<float2 *>(&X->cum[sc][2 * lane]) = make_float2(x0, x);
            *reinterpret_cast<float2 *>(&X->ck[sc][2 * lane]) = make_float2(x0 - g0, x - g1);
            *reinterpret_cast<float2 *>(&X->qs[sc][2 * lane]) = make_float2(ex2_approx(x0), ex2_approx(x));
            *reinterpret_cast<float2 *>(&X->w[sc][2 * lane]) =
                make_float2(ex2_approx(total - x0 + g0), ex2_approx(total - x + g1));
            if (lane == 0) X->gam[sc] = ex2_approx(total);
            __syncwarp();
            if (lane == 0) mbar_arrive(&X->dec_full[sc]);
          }
        }
    } else if (warp < 14) {
        // ------------------------------------------------------------ outputs
        const int td = threadIdx.x - 320;
        const int q = warp & 3;
        const int ch = 32 * q + lane;
        const uint32_t lanebase = (uint32_t)(32 * q) << 16;
        bool ok = true;
        for (int it = 0; it < nch; ++it) {
            const int s = it & 1;
            // outputs of the chunk: o = O^T / den (lane = value channel, column = token),
            // times the gate when there is one (in quarters of 16 tokens)
            const int t0c = (c_begin + it) * kC;
            float gq[16];   // the gate's values for the next quarter's tokens of this channel
            auto load_gate = [&](int qt) {
                const int64_t tb = t0c + 16 * qt;
                const float *gp = a.gate + ((b * g.L + tb) * g.H + h) * (int64_t)g.dv + dv0 + ch;
                const int tstride = g.H * g.dv;
                const int nt = g.L - tb < 16 ? (int)(g.L - tb) : 16;
#pragma unroll
                for (int i = 0; i < 16; ++i) gq[i] = i < nt ? gp[i * tstride] : 0.f;
            };
            if constexpr (GATE) {
                load_gate(0);   // the loads run while this warp waits for O
                // the next chunk's gate lines into L2: lane l fetches the line of
                // this warp's 32 channels for tokens l and l + 32
                const int64_t tn = t0c + kC + lane;
                const float *gn = a.gate + ((b * g.L + tn) * g.H + h) * (int64_t)g.dv + dv0 + 32 * q;
                if (tn < g.L) asm volatile("prefetch.global.L2 [%0];" ::"l"(gn));
                if (tn + 32 < g.L)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(gn + 32 * (int64_t)g.H * g.dv));
            }
            bool okc = ok && mbar_wait(&X->o_full, it & 1, abort_flag, err, KID_SCAN_TC_OUT, 9) &&
                       mbar_wait(&X->den_ready[s], (it >> 1) & 1, abort_flag, err, KID_SCAN_TC_OUT, 10);
            okc = __all_sync(0xffffffffu, okc);
            // staging in the chunk's Pt buffer (16 KB), in two rounds of 32
            // tokens: box cb = channels 64 cb.. of the CTA's value half, rows of
            // 64 channels, no swizzle.  bf16 boxes are 4 KB (round th at 8 KB
            // th); fp32 boxes 8 KB, both rounds at offset 0 (round 1 waits
            // until round 0 has been read out).
            uint8_t *const stg = gP(s);
            const int cb = ch >> 6, cl = ch & 63;
            const float *rd = X->rden[s];
#pragma unroll 1
            for (int th = 0; th < 2; ++th) {
                if (okc && !GATE) {
                    tc_fence_after();
                    uint32_t r[32];
                    tmem_ld32(tmem + kColO + 32 * th + lanebase, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 d4 = *reinterpret_cast<const float4 *>(rd + 32 * th + 4 * i4);
                        r[4 * i4 + 0] = __float_as_uint(__uint_as_float(r[4 * i4 + 0]) * d4.x);
                        r[4 * i4 + 1] = __float_as_uint(__uint_as_float(r[4 * i4 + 1]) * d4.y);
                        r[4 * i4 + 2] = __float_as_uint(__uint_as_float(r[4 * i4 + 2]) * d4.z);
                        r[4 * i4 + 3] = __float_as_uint(__uint_as_float(r[4 * i4 + 3]) * d4.w);
                    }
                    if (a.o_f32) {
                        float *box = reinterpret_cast<float *>(stg + cb * 8192) + cl;
#pragma unroll
                        for (int i = 0; i < 32; ++i) box[i * 64] = __uint_as_float(r[i]);
                    } else {
                        __nv_bfloat16 *box = reinterpret_cast<__nv_bfloat16 *>(stg + th * 8192 + cb * 4096) + cl;
#pragma unroll
                        for (int i = 0; i < 32; ++i) box[i * 64] = __float2bfloat16_rn(__uint_as_float(r[i]));
                    }
                } else if (GATE && okc) {
                    // with the gate: quarters of 16 tokens, the next quarter's gate
                    // values loading while this one is staged (bf16 out)
                    tc_fence_after();
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int qt = 2 * th + hh;   // token quarter of the chunk
                        uint32_t r[16];
                        tmem_ld16(tmem + kColO + 16 * qt + lanebase, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int i4 = 0; i4 < 4; ++i4) {
                            const float4 d4 = *reinterpret_cast<const float4 *>(rd + 16 * qt + 4 * i4);
                            r[4 * i4 + 0] = __float_as_uint(__uint_as_float(r[4 * i4 + 0]) * d4.x * gq[4 * i4 + 0]);
                            r[4 * i4 + 1] = __float_as_uint(__uint_as_float(r[4 * i4 + 1]) * d4.y * gq[4 * i4 + 1]);
                            r[4 * i4 + 2] = __float_as_uint(__uint_as_float(r[4 * i4 + 2]) * d4.z * gq[4 * i4 + 2]);
                            r[4 * i4 + 3] = __float_as_uint(__uint_as_float(r[4 * i4 + 3]) * d4.w * gq[4 * i4 + 3]);
                        }
                        if (qt < 3) load_gate(qt + 1);   // under this quarter's staging
                        __nv_bfloat16 *box =
                            reinterpret_cast<__nv_bfloat16 *>(stg + th * 8192 + cb * 4096) + cl + 16 * hh * 64;
#pragma unroll
                        for (int i = 0; i < 16; ++i) box[i * 64] = __float2bfloat16_rn(__uint_as_float(r[i]));
                    }
                }
                if (th == 1) {
                    // O^T may be overwritten, and this stage's 1 / den rewritten
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&X->den_free[s]);
                        mbar_arrive(&X->o_empty);
                    }
                }
                fence_proxy_async_smem();
                okc = named_sync_and(2, 128, okc);
                if (td == 0 && okc && t0c + 32 * th < g.L) {
                    for (int c2 = 0; c2 < 2; ++c2) {
                        const uint8_t *src = a.o_f32 ? stg + c2 * 8192 : stg + th * 8192 + c2 * 4096;
                        tma_store_4d(&tmo, src, dv0 + 64 * c2, h, t0c + 32 * th, (int)b);
                    }
                    bulk_commit();
                    if (a.o_f32 || th == 1) bulk_wait_read_all();
                }
                if (a.o_f32 && th == 0) named_sync(2, 128);   // round 0 has been read out
            }
            if (td == 0) mbar_arrive(&X->stg_free[s]);   // the Pt buffer may be rewritten
            ok = ok && okc;
            if (!ok) break;
        }
        // the output stores must have completed before the CTA's shared memory goes away
        if (td == 0) bulk_wait_all();
    } else {
        // ------------------------------------------------------------ state pass
        const int td = threadIdx.x - 480;
        const int q = warp & 3;
        const int ch = 32 * q + lane;
        const uint32_t lanebase = (uint32_t)(32 * q) << 16;
        // the start z (z before the segment) as the first write of buffer 1;
        // this thread's features: f0, f0 + 1 (the warp's 64-feature block)
        const int f0 = 64 * q + 2 * lane;
        {
            const float *zi = seg == 0 ? (a.z0 ? a.z0 + bh * kF : nullptr) : a.z_start + (bh * g.G + seg) * kF;
            *reinterpret_cast<float2 *>(&X->zb[1][f0]) = zi ? make_float2(zi[f0], zi[f0 + 1]) : make_float2(0.f, 0.f);
            __syncwarp();
            if (lane == 0) mbar_arrive(&X->zfull[1]);
        }
        // prologue: start state -> bf16 copy (for the first readout) and fp32 x gamma_0
        float dt_next = token_dt(a, b, h, (int64_t)c_begin * kC, td);
        {
            const float gam0 = fexp(chunk_total(hm_log_decay(dt_next, alog), td, X->redd, 5));
            if (nch > 1) dt_next = token_dt(a, b, h, (int64_t)(c_begin + 1) * kC, td);
            if (seg > 0) {
                // segment start state [F][dv] (fp32, in L2): rounds of 32 feature rows
                // x the CTA's 128 channels (16 KB) land by TMA in three rotating
                // buffers (the Pt and w V tiles, unused until the first chunk)
                const int row0 = (int)((bh * g.G + seg) * kF);
                uint8_t *const pbuf = gP(0);
                if (td == 0)
                    for (int r = 0; r < 3; ++r) {
                        mbar_arrive_expect_tx(&X->pro_full[r], 32 * kN * 4);
                        tma_load_2d(pbuf + r * 32 * kN * 4, &tms, &X->pro_full[r], dv0, row0 + 32 * r);
                    }
#pragma unroll 1
                for (int r = 0; r < kF / 32; ++r) {
                    mbar_wait(&X->pro_full[r % 3], (r / 3) & 1, abort_flag, err, KID_SCAN_TC_OUT, 22);
                    const float *buf = reinterpret_cast<const float *>(pbuf + (r % 3) * 32 * kN * 4) + ch;
                    uint32_t v[32], pk[16];
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(buf[j * kN]);
#pragma unroll
                    for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
                    tmem_st16(tmem + kColSB + 16 * r + lanebase, pk);
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * gam0);
                    tmem_st32(tmem + kColS + 32 * r + lanebase, v);
                    named_sync(5, 128);   // every thread has read this buffer
                    if (td == 0 && r + 3 < kF / 32) {
                        mbar_arrive_expect_tx(&X->pro_full[r % 3], 32 * kN * 4);
                        tma_load_2d(pbuf + (r % 3) * 32 * kN * 4, &tms, &X->pro_full[r % 3], dv0, row0 + 32 * (r + 3));
                    }
                }
            } else {
                const float *src = a.S0 ? a.S0 + bh * (int64_t)kF * g.dv : nullptr;
                for (int c0 = 0; c0 < kF; c0 += 32) {
                    uint32_t v[32], pk[16];
                    if (src) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(src[(int64_t)(c0 + j) * g.dv + dv0 + ch]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = 0u;
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
                    tmem_st16(tmem + kColSB + c0 / 2 + lanebase, pk);
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * gam0);
                    tmem_st32(tmem + kColS + c0 + lanebase, v);
                }
            }
            tmem_wait_st();
            if (td == 0) X->szero = gam0 == 0.f ? 1 : 0;
            tc_fence_before();
            named_sync(5, 128);   // szero is written before any warp's arrival
            if (lane == 0) mbar_arrive(&X->sbf_ready);
        }
        bool ok = true;
        for (int it = 0; it < nch; ++it) {
            // z after chunk it, z_it = gamma_it z_(it-1) + sum_j w_j phik_j, into
            // zb[it & 1] for the compute group's denominators of chunk it + 1,
            // once the compute group has read the buffer's previous z (z_(it-2),
            // or the start z for it = 1) in chunk it - 1: zfree, whose
            // ((it - 1) >> 1)-th completion that is; then these warps release
            // the chunk's stage and decay vectors
            const int s1 = it & 1;
            bool okz = mbar_wait(&X->dec_full[s1], (it >> 1) & 1, abort_flag, err, KID_SCAN_TC_OUT, 23) &&
                       mbar_wait(&X->fullkv[s1], (it >> 1) & 1, abort_flag, err, KID_SCAN_TC_OUT, 25) &&
                       (it < 1 || mbar_wait(&X->zfree[s1], ((it - 1) >> 1) & 1, abort_flag, err, KID_SCAN_TC_OUT, 26));
            ok = named_sync_and(5, 128, okz);
            if (!ok) break;
            {
                const uint8_t *__restrict__ kb = gK(s1) + q * kQKBlk + (lane & 3) * 4;
                const float *__restrict__ wv = X->w[s1];
                float2 za = make_float2(0.f, 0.f);
#pragma unroll 8
                for (int j = 0; j < kC; ++j) {
                    const uint32_t kv = *reinterpret_cast<const uint32_t *>(kb + sw128_off(j, lane >> 2));
                    const float wj = wv[j];
                    za = fma2(unpack_bf16x2(kv), make_float2(wj, wj), za);
                }
                const float gm = X->gam[s1];
                const float2 zp = *reinterpret_cast<const float2 *>(&X->zb[(it - 1) & 1][f0]);
                *reinterpret_cast<float2 *>(&X->zb[s1][f0]) = make_float2(fmaf(gm, zp.x, za.x), fmaf(gm, zp.y, za.y));
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&X->emptykv[s1]);
                    mbar_arrive(&X->dec_free[s1]);
                    mbar_arrive(&X->zfull[s1]);
                }
            }
            if (it + 1 >= nch) break;   // no state pass after the last chunk
            const float gn = fexp(chunk_total(hm_log_decay(dt_next, alog), td, X->redd, 5));
            if (it + 2 < nch) dt_next = token_dt(a, b, h, (int64_t)(c_begin + it + 2) * kC, td);
            ok = named_sync_and(5, 128, mbar_wait(&X->s_full, it & 1, abort_flag, err, KID_SCAN_TC_OUT, 11));
            if (!ok) break;
            tc_fence_after();
            // 32-column blocks: S^T -> its bf16 copy for the next readout, and
            // S^T <- gamma S^T before the next state MMA.  gn is the same in
            // every thread; when it is 0 the next state MMA overwrites S instead
            // (szero), so S is only converted.
            const bool gz = gn == 0.f;
            const float2 g2 = make_float2(gn, gn);
#pragma unroll 1
            for (int blk = 0; blk < kF / 32; ++blk) {
                uint32_t cur[32], pk[16];
                tmem_ld32(tmem + kColS + 32 * blk + lanebase, cur);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    pk[j] = pack_bf16x2(__uint_as_float(cur[2 * j]), __uint_as_float(cur[2 * j + 1]));
                tmem_st16(tmem + kColSB + 16 * blk + lanebase, pk);
                if (!gz) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float2 y = mul2(make_float2(__uint_as_float(cur[2 * j]), __uint_as_float(cur[2 * j + 1])), g2);
                        cur[2 * j] = __float_as_uint(y.x);
                        cur[2 * j + 1] = __float_as_uint(y.y);
                    }
                    tmem_st32(tmem + kColS + 32 * blk + lanebase, cur);
                }
            }
            tmem_wait_st();
            if (td == 0) X->szero = gz ? 1 : 0;
            tc_fence_before();
            named_sync(5, 128);   // szero is written before any warp's arrival
            if (lane == 0) mbar_arrive(&X->sbf_ready);
        }
        // the MMAs of the last chunk must be complete before TMEM is released
        if (ok && nch > 0) mbar_wait(&X->s_full, (nch - 1) & 1, abort_flag, err, KID_SCAN_TC_OUT, 12);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ host side

struct Plan {
    Geo g;
    size_t off_Spart, off_zpart, off_lsum, off_Sstart, off_zstart, total;
};

int num_sms() {
    static int sms = 0;
    if (!sms) {
        int dev = 0, v = 148;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
            sms = v;
        else
            sms = 148;
    }
    return sms;
}

size_t rup(size_t x) { return (x + 255) / 256 * 256; }

Plan make_plan(const ScanCore &c, bool want_state) {
    Plan p{};
    Geo &g = p.g;
    g.B = c.B;
    g.L = c.L;
    g.H = c.H;
    g.dv = c.dv;
    g.nchunks = (int)((c.L + kC - 1) / kC);
    const int64_t heads2 = c.B * c.H * (c.dv / kN);  // CTAs per segment (value halves)
    const int sms = num_sms();
    int G = (int)std::max<int64_t>(1, sms / std::max<int64_t>(1, heads2));
    if (G > g.nchunks) G = std::max(1, g.nchunks);
    int seg_chunks = g.nchunks > 0 ? (g.nchunks + G - 1) / G : 1;
    // parts: divide each segment so that the state phase fills the GPU
    const int seg_state = want_state ? G : G - 1;
    int pps = 1;
    if (seg_state > 0) {
        for (int d = seg_chunks; d >= 1; --d) {
            if (seg_chunks % d) continue;
            if (heads2 * seg_state * d <= sms) {
                pps = d;
                break;
            }
        }
    }
    g.part_chunks = seg_chunks / pps;
    g.seg_chunks = seg_chunks;
    g.G = g.nchunks > 0 ? (g.nchunks + seg_chunks - 1) / seg_chunks : 1;
    g.NP = g.nchunks > 0 ? (g.nchunks + g.part_chunks - 1) / g.part_chunks : 0;
    g.NPc = want_state ? g.NP : std::min(g.NP, (g.G - 1) * pps);
    const int64_t BH = c.B * c.H;
    const size_t nS = (size_t)kF * c.dv;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = rup(off + bytes); return o; };
    p.off_Spart = take(sizeof(float) * BH * g.NPc * nS);
    p.off_zpart = take(sizeof(float) * BH * g.NPc * kF);
    p.off_lsum = take(sizeof(float) * BH * g.NPc);
    p.off_Sstart = take(sizeof(float) * BH * g.G * nS);
    p.off_zstart = take(sizeof(float) * BH * g.G * kF);
    p.total = off;
    return p;
}

bool tmap_tokens(CUtensorMap *m, const void *base, int64_t B, int64_t L, int H, int X, int box_x) {
    // [B, L, H, X] bf16 viewed as (X, H, L, B); box (box_x, 1, C, 1)
    uint64_t dims[4] = {(uint64_t)X, (uint64_t)H, (uint64_t)L, (uint64_t)B};
    uint64_t strides[3] = {(uint64_t)X * 2, (uint64_t)H * X * 2, (uint64_t)L * H * X * 2};
    uint32_t box[4] = {(uint32_t)box_x, 1, kC, 1};
    return make_tmap_bf16(m, base, 4, dims, strides, box);
}

}  // namespace

bool scan_tc_supported(const ScanCore &c) {
    return !c.per_feature && c.io_dtype == HM_BF16 && c.feat_dtype == HM_BF16 && c.F == kF && c.dv % kN == 0 &&
           c.dv == 2 * kN && c.L < (int64_t)1 << 30 && c.B < 65536 && c.H < 65536;
}

size_t scan_tc_workspace(const ScanCore &c) { return make_plan(c, true).total; }

cudaError_t launch_scan_tc_impl(const ScanCore &c, const void *phk_lo, void *ws, size_t ws_bytes,
                                DevErr err, cudaStream_t s) {
    const bool want_state = c.S_out != nullptr;
    Plan p = make_plan(c, want_state);
    if (p.total > ws_bytes) return cudaErrorInvalidValue;
    Geo &g = p.g;
    const int64_t BH = c.B * c.H;
    const size_t nS = (size_t)kF * c.dv;
    char *w = (char *)ws;
    float *S_part = (float *)(w + p.off_Spart), *z_part = (float *)(w + p.off_zpart);
    float *lsum = (float *)(w + p.off_lsum);
    float *S_start = (float *)(w + p.off_Sstart), *z_start = (float *)(w + p.off_zstart);
    cudaError_t e;
    if (g.nchunks == 0) {
        // empty sequence: the final state is the initial state
        if (want_state) {
            e = c.S0 ? cudaMemcpyAsync(c.S_out, c.S0, sizeof(float) * BH * nS, cudaMemcpyDeviceToDevice, s)
                     : cudaMemsetAsync(c.S_out, 0, sizeof(float) * BH * nS, s);
            if (e != cudaSuccess) return e;
            e = c.z0 ? cudaMemcpyAsync(c.z_out, c.z0, sizeof(float) * BH * kF, cudaMemcpyDeviceToDevice, s)
                     : cudaMemsetAsync(c.z_out, 0, sizeof(float) * BH * kF, s);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    // a state-only call (o == NULL) runs phases A and B and no output kernel
    const bool outputs = c.o != nullptr;
    CUtensorMap tq, tk, tkl, tv;
    if (!tmap_tokens(&tk, c.phk, c.B, c.L, c.H, kF, 64) || !tmap_tokens(&tv, c.v, c.B, c.L, c.H, c.dv, 64))
        return cudaErrorInvalidValue;
    if (outputs && !tmap_tokens(&tq, c.phq, c.B, c.L, c.H, kF, 64)) return cudaErrorInvalidValue;
    // with a returned state, the weighted features of the state phase are split
    // into bf16 hi + lo (and phik's own rounding remainder is added when given)
    const bool split = want_state;
    const bool add_lo = want_state && phk_lo != nullptr;
    if (!tmap_tokens(&tkl, add_lo ? phk_lo : c.phk, c.B, c.L, c.H, kF, 64)) return cudaErrorInvalidValue;

    if (g.NPc > 0) {
        e = ensure_smem_limit(scan_state_kernel, kASmem);
        if (e != cudaSuccess) return e;
        const unsigned grid = (unsigned)(2 * g.NPc * BH);
        scan_state_kernel<<<grid, kAThreads, kASmem, s>>>(tk, tkl, tv, g, c.dt, c.A_log, split ? 1 : 0,
                                                    add_lo ? 1 : 0, c.dt_scaled ? 1 : 0, S_part, z_part,
                                                    lsum, err);
        count_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t ncol = (int64_t)(nS + kF) / 4;
        const int64_t wide_ctas = BH * ((ncol + 511) / 512);
        if (wide_ctas >= 2 * (int64_t)num_sms()) {
            dim3 gb((unsigned)((ncol + 511) / 512), (unsigned)BH);
            scan_carry_kernel<2, 2><<<gb, 256, 0, s>>>(g, S_part, z_part, lsum, c.S0, c.z0, S_start, z_start,
                                                       c.S_out, c.z_out);
        } else {
            dim3 gb((unsigned)((ncol + 255) / 256), (unsigned)BH);
            scan_carry_kernel<1, 8><<<gb, 256, 0, s>>>(g, S_part, z_part, lsum, c.S0, c.z0, S_start, z_start,
                                                       c.S_out, c.z_out);
        }
        count_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (!outputs) return cudaSuccess;
    OutArgs oa{};
    oa.g = g;
    oa.dt = c.dt;
    oa.A_log = c.A_log;
    oa.o = c.o;
    oa.o_f32 = c.o_f32 ? 1 : 0;
    oa.dt_scaled = c.dt_scaled ? 1 : 0;
    oa.S0 = c.S0;
    oa.z0 = c.z0;
    oa.S_start = S_start;
    oa.z_start = z_start;
    oa.gate = (const float *)c.gate;
    // output tiles: boxes of 64 channels x 32 tokens, stored from unswizzled staging rows
    CUtensorMap to;
    {
        const uint64_t es = c.o_f32 ? 4 : 2;
        uint64_t dims[4] = {(uint64_t)c.dv, (uint64_t)c.H, (uint64_t)c.L, (uint64_t)c.B};
        uint64_t strides[3] = {(uint64_t)c.dv * es, (uint64_t)c.H * c.dv * es, (uint64_t)c.L * c.H * c.dv * es};
        uint32_t box[4] = {64, 1, 32, 1};
        if (!make_tmap(&to, c.o_f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c.o, 4,
                       dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    // segment start states [BH * G * F][dv] fp32: boxes of 32 feature rows x 128 channels
    CUtensorMap tss;
    {
        uint64_t dims[2] = {(uint64_t)c.dv, (uint64_t)BH * g.G * kF};
        uint64_t strides[1] = {(uint64_t)c.dv * 4};
        uint32_t box[2] = {(uint32_t)kN, 32};
        if (!make_tmap(&tss, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, S_start, 2, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    if (c.gate && c.o_f32) return cudaErrorInvalidValue;   // the gated output is bf16
    auto out_kernel = c.gate ? scan_out_kernel<true> : scan_out_kernel<false>;
    e = ensure_smem_limit(out_kernel, kCSmem);
    if (e != cudaSuccess) return e;
    out_kernel<<<(unsigned)(2 * g.G * BH), kCThreads, kCSmem, s>>>(tq, tk, tv, to, tss, oa, err);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_scan_tc(const ScanCore &c, void *ws, size_t ws_bytes, DevErr err, cudaStream_t s) {
    return launch_scan_tc_impl(c, c.phk_lo, ws, ws_bytes, err, s);
}

}  // namespace hm

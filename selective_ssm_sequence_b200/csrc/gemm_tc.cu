// gemm_tc.cu -- C[M, N] = A[M, K] . B[N, K]^T on the 5th-generation tensor cores.
//
// The dense projections of the HedgeMamba mixer (q, k, v, gate and output
// projections; HedgeMamba explainer sec. 2.3 and 5.2) are plain GEMMs with
// nn.Linear weights (y = x W^T), so both operands are K-major.  Persistent
// kernel, one CTA per SM: 128 x 256 output tiles, 64-wide K blocks streamed by
// TMA through a 4-stage ring, tcgen05.mma (bf16 -> fp32 in TMEM) issued by one
// thread, and two TMEM accumulators so that the epilogue of one tile overlaps
// the MMAs of the next.  Warp roles: 0 = TMA, 1 = MMA, 2..9 = epilogue (two
// warps per TMEM lane quarter, one per half of the tile's 256 columns).
//
// The epilogue applies what follows the GEMM in the mixer and the block around
// it (HedgeMamba explainer sec. 2.3, 5.1, 5.2), so that those steps cost no
// trip through HBM of their own: the short causal conv of the q, k, v
// projections, the gate's SiLU, the MLP's GELU and the residual additions.
// The conv runs along the tokens, so that GEMM is computed transposed,
// C^T = W x^T: TMEM lanes are channels and columns are tokens, and each
// epilogue thread holds consecutive tokens of one channel, with the conv's
// window in its own registers.  Token tiles overlap by K - 1 columns (a tile
// covers tokens n0 - (K-1) .. n0 + 255 - (K-1) and writes the last 257 - K;
// TMA fills tokens before 0 with zeros), and a window never reaches back past
// its sequence's first token.
#include <utility>

#include "tc_common.cuh"

namespace hm {

namespace {

using namespace tc;

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;   // 16 KB
constexpr int kBBytes = kBN * kBK * 2;   // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;

constexpr int kMaxConv = 8;   // conv width
constexpr int kEpiWarps = 8;
constexpr int kGThreads = 64 + 32 * kEpiWarps;
constexpr int kHalfN = kBN / 2;   // columns per epilogue warp

struct GAux {
    uint64_t full[kStages], empty[kStages];
    uint64_t accf[2], acce[2];
    uint32_t tmem;
    int abort;
};

constexpr int kGSmem = kStages * kStageBytes + (int)sizeof(GAux) + 1024;

// SiLU with the fast exponential and division (about 2 ulp): the gate feeds a
// bf16 product.  For v < -88 the exponential is +inf and the quotient 0.
__device__ __forceinline__ float silu_f(float v) { return __fdividef(v, 1.f + __expf(-v)); }
__device__ __forceinline__ float gelu_f(float v) { return 0.5f * v * (1.f + erff(v * 0.70710678118654752f)); }

// Conv epilogue of one tile (transposed GEMM): this thread holds channel m
// for tokens n0 .. n0 + 255 in TMEM columns; it writes
// y[t] = bias + sum_j w[m][KC-1-j] x[t-j] for the tokens past the halo, with
// the window cut at the start of each sequence.  KC is the conv width, or
// kMaxConv for any width up to it (the missing taps weigh 0).
template <int KC>
__device__ __forceinline__ void conv_epilogue(GAux *X, uint32_t ta, int b, int64_t m, int64_t n0, int64_t M,
                                              int64_t N, int halo, const GemmEpiArgs &ep, __nv_bfloat16 *C,
                                              int64_t ldc, int cbeg) {
    float wr[KC];   // wr[j]: the weight of token t - j
#pragma unroll
    for (int j = 0; j < KC; ++j)
        wr[j] = (m < M && j < ep.conv_k) ? ep.conv_w[m * ep.conv_k + ep.conv_k - 1 - j] : 0.f;
    const float bs = (ep.bias && m < M) ? ep.bias[m] : 0.f;
    float hist[KC - 1 > 0 ? KC - 1 : 1];   // the KC - 1 tokens before the block, oldest first
#pragma unroll
    for (int j = 0; j < KC - 1; ++j) hist[j] = 0.f;
    if (cbeg > 0 && KC > 1) {
        // the second half's window starts with the last columns of the first
        uint32_t h8[8];
        tmem_ld8(ta + cbeg - 8, h8);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < KC - 1; ++j) hist[j] = __uint_as_float(h8[8 - (KC - 1) + j]);
    }
    const int L = (int)ep.seq_len;
    // position in its sequence of the block's first token (negative: the
    // zero-filled tokens before the first)
    const int64_t nb = n0 + cbeg;
    int tpos = nb >= 0 ? (int)(nb % ep.seq_len) : (int)nb;
    const bool live = m < M;
#pragma unroll 1
    for (int c0 = cbeg; c0 < cbeg + kHalfN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(ta + c0, r);
        tmem_wait_ld();
        if (c0 + 32 >= cbeg + kHalfN) {
            tc_fence_before();
            mbar_arrive(&X->acce[b]);
        }
        float win[KC - 1 + 32];
#pragma unroll
        for (int j = 0; j < KC - 1; ++j) win[j] = hist[j];
#pragma unroll
        for (int i = 0; i < 32; ++i) win[KC - 1 + i] = __uint_as_float(r[i]);
        const int64_t tok0 = n0 + c0;
        __nv_bfloat16 *dst = C + tok0 * ldc + m;
        const int i0 = c0 < halo ? halo - c0 : 0;            // first column past the halo
        const int iend = N - tok0 < 32 ? (int)(N - tok0) : 32; // columns before the end
        if (tpos >= KC - 1 && tpos + 31 < L) {
            // no sequence starts inside the window of any token of the block
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float y = bs;
#pragma unroll
                for (int j = 0; j < KC; ++j) y = fmaf(wr[j], win[KC - 1 + i - j], y);
                if (live && i >= i0 && i < iend) dst[(int64_t)i * ldc] = __float2bfloat16_rn(y);
            }
            tpos += 32;
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float y = bs;
#pragma unroll
                for (int j = 0; j < KC; ++j)
                    if (j <= tpos) y = fmaf(wr[j], win[KC - 1 + i - j], y);
                if (live && i >= i0 && i < iend) dst[(int64_t)i * ldc] = __float2bfloat16_rn(y);
                if (++tpos == L) tpos = 0;
            }
        }
        if (tpos >= L) tpos -= L;
#pragma unroll
        for (int j = 0; j < KC - 1; ++j) hist[j] = win[32 + j];
    }
}

template <int EPI>
__global__ void __launch_bounds__(kGThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb,
               int64_t M, int64_t N, int64_t K, void *__restrict__ C, int64_t ldc, GemmEpiArgs ep,
               DevErr err) {
    const float *__restrict__ bias = ep.bias;
    // conv (transposed: M = channels, N = tokens): token tiles overlap by
    // `halo` columns; column 0 of tile tn is token tn * step - halo
    const int halo = EPI == EPI_CONV_BF16 ? ep.conv_k - 1 : 0;
    const int step = kBN - halo;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    GAux *X = (GAux *)(smem + kStages * kStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tiles_m = (M + kBM - 1) / kBM, tiles_n = (N + step - 1) / step;
    const int64_t ntiles = tiles_m * tiles_n;
    const int kblocks = (int)(K / kBK);
    volatile int *abort_flag = &X->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&X->full[s], 1);
            mbar_init(&X->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&X->accf[b], 1);
            mbar_init(&X->acce[b], 32 * kEpiWarps);
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
        if (elect_one()) {
            tma_prefetch_desc(&tma);
            tma_prefetch_desc(&tmb);
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
                const int m0 = (int)((t / tiles_n) * kBM), n0 = (int)((t % tiles_n) * step) - halo;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % kStages;
                    if (!mbar_wait(&X->empty[s], ((it / kStages) & 1) ^ 1, abort_flag, err, KID_GEMM_TC, 1)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + s * kStageBytes;
                    mbar_arrive_expect_tx(&X->full[s], kStageBytes);
                    tma_load_2d(st, &tma, &X->full[s], kb * kBK, m0);
                    tma_load_2d(st + kABytes, &tmb, &X->full[s], kb * kBK, n0);
                }
            }
            // no copy may still be landing when the CTA exits
            for (uint32_t j = (it > kStages ? it - kStages : 0); j < it; ++j)
                for (uint32_t i = 0; i < kWaitPolls; ++i)
                    if (mbar_try_wait(&X->full[j % kStages], (j / kStages) & 1)) break;
        }
    } else if (warp == 1) {
        if (elect_one()) {
            constexpr uint32_t idesc = idesc_bf16(kBM, kBN, false, false);
            uint32_t it = 0;
            int tl = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++tl) {
                const int b = tl & 1;
                if (!mbar_wait(&X->acce[b], ((tl >> 1) & 1) ^ 1, abort_flag, err, KID_GEMM_TC, 2)) break;
                tc_fence_after();
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % kStages;
                    if (!mbar_wait(&X->full[s], (it / kStages) & 1, abort_flag, err, KID_GEMM_TC, 3)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * kStageBytes);
                    const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        mma_ss(tmem + b * kBN, desc_k_sw128(a_addr + k * 32), desc_k_sw128(b_addr + k * 32),
                               idesc, (kb > 0 || k > 0) ? 1u : 0u);
                    mma_commit(&X->empty[s]);
                }
                mma_commit(&X->accf[b]);
            }
        }
    } else {
        const int q = warp & 3;
        const int row = 32 * q + lane;
        const int cbeg = ((warp - 2) >> 2) * kHalfN;   // this warp's half of the columns
        int tl = 0;
        for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++tl) {
            const int b = tl & 1;
            if (!mbar_wait(&X->accf[b], (tl >> 1) & 1, abort_flag, err, KID_GEMM_TC, 4)) break;
            tc_fence_after();
            const int64_t m = (t / tiles_n) * kBM + row;
            const int64_t n0 = (t % tiles_n) * step - halo;
            const uint32_t ta = tmem + b * kBN + ((uint32_t)(32 * q) << 16);
            if constexpr (EPI == EPI_CONV_BF16) {
                if (ep.conv_k == 4)
                    conv_epilogue<4>(X, ta, b, m, n0, M, N, halo, ep, (__nv_bfloat16 *)C, ldc, cbeg);
                else
                    conv_epilogue<kMaxConv>(X, ta, b, m, n0, M, N, halo, ep, (__nv_bfloat16 *)C, ldc, cbeg);
                continue;
            }
            const bool out_row = m < M;
#pragma unroll 1
            for (int c0 = cbeg; c0 < cbeg + kHalfN; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(ta + c0, r);
                tmem_wait_ld();
                if (c0 + 32 >= cbeg + kHalfN) {
                    tc_fence_before();
                    mbar_arrive(&X->acce[b]);
                }
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
                if (out_row) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int64_t c = n0 + c0 + i;
                        if (bias && c < N) v[i] += bias[c];
                    }
                    if constexpr (EPI == EPI_SILU_F32) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = silu_f(v[i]);
                    }
                    if constexpr (EPI == EPI_GELU_BF16) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = gelu_f(v[i]);
                    }
                    if constexpr (EPI == EPI_ADD_F32) {
                        const __nv_bfloat16 *rr = (const __nv_bfloat16 *)ep.res + m * ep.ldr + n0 + c0;
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            if (n0 + c0 + 8 * u < N) {
                                const uint4 w = *reinterpret_cast<const uint4 *>(rr + 8 * u);
                                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float2 f = unpack_bf16x2(ww[e]);
                                    v[8 * u + 2 * e] += f.x;
                                    v[8 * u + 2 * e + 1] += f.y;
                                }
                            }
                        }
                    }
                    if constexpr (EPI == EPI_ADD_BF16) {
                        const float *rr = (const float *)ep.res + m * ep.ldr + n0 + c0;
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            if (n0 + c0 + 4 * u < N) {
                                const float4 w = *reinterpret_cast<const float4 *>(rr + 4 * u);
                                v[4 * u] += w.x;
                                v[4 * u + 1] += w.y;
                                v[4 * u + 2] += w.z;
                                v[4 * u + 3] += w.w;
                            }
                        }
                    }
                    if constexpr (EPI == EPI_STORE_F32 || EPI == EPI_ADD_F32 || EPI == EPI_SILU_F32) {
                        float *dst = (float *)C + m * ldc + n0 + c0;
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            if (n0 + c0 + 4 * u < N)
                                *reinterpret_cast<float4 *>(dst + 4 * u) =
                                    make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                    } else {
                        __nv_bfloat16 *dst = (__nv_bfloat16 *)C + m * ldc + n0 + c0;
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            if (n0 + c0 + 8 * u < N) {
                                uint4 w;
                                w.x = pack_bf16x2(v[8 * u + 0], v[8 * u + 1]);
                                w.y = pack_bf16x2(v[8 * u + 2], v[8 * u + 3]);
                                w.z = pack_bf16x2(v[8 * u + 4], v[8 * u + 5]);
                                w.w = pack_bf16x2(v[8 * u + 6], v[8 * u + 7]);
                                *reinterpret_cast<uint4 *>(dst + 8 * u) = w;
                            }
                        }
                    }
                }
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

}  // namespace

bool gemm_tc_supported(int64_t M, int64_t N, int64_t K) {
    return M >= 1 && N >= 16 && N % 16 == 0 && K >= kBK && K % kBK == 0 && M < ((int64_t)1 << 31) &&
           N < ((int64_t)1 << 31);
}

namespace {

template <int EPI>
cudaError_t launch_epi(const CUtensorMap &tma, const CUtensorMap &tmb, unsigned grid, int64_t M, int64_t N,
                       int64_t K, void *C, int64_t ldc, const GemmEpiArgs &ep, DevErr err, cudaStream_t s) {
    cudaError_t e = ensure_smem_limit(gemm_tc_kernel<EPI>, kGSmem);
    if (e != cudaSuccess) return e;
    gemm_tc_kernel<EPI><<<grid, kGThreads, kGSmem, s>>>(tma, tmb, M, N, K, C, ldc, ep, err);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_tc_ex(const void *A, const void *Bm, int64_t M, int64_t N, int64_t K, void *C,
                              int64_t ldc, const GemmEpiArgs &ep, DevErr err, cudaStream_t s) {
    if (!gemm_tc_supported(M, N, K)) return cudaErrorNotSupported;
    if (ep.mode == EPI_CONV_BF16 && (ep.conv_k < 1 || ep.conv_k > kMaxConv || !ep.conv_w || ep.seq_len < 1))
        return cudaErrorInvalidValue;
    if (ep.mode == EPI_CONV_BF16) {
        // computed transposed: the kernel's A is the weight (rows = the N output
        // channels) and its B the input (rows = the M tokens)
        std::swap(A, Bm);
        std::swap(M, N);
    }
    if ((ep.mode == EPI_ADD_F32 || ep.mode == EPI_ADD_BF16) && (!ep.res || ep.ldr < N))
        return cudaErrorInvalidValue;
    CUtensorMap tma, tmb;
    {
        uint64_t dims[2] = {(uint64_t)K, (uint64_t)M};
        uint64_t strides[1] = {(uint64_t)K * 2};
        uint32_t box[2] = {kBK, kBM};
        if (!make_tmap_bf16(&tma, A, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        uint64_t dims[2] = {(uint64_t)K, (uint64_t)N};
        uint64_t strides[1] = {(uint64_t)K * 2};
        uint32_t box[2] = {kBK, kBN};
        if (!make_tmap_bf16(&tmb, Bm, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t step = ep.mode == EPI_CONV_BF16 ? kBN - (ep.conv_k - 1) : kBN;
    const int64_t ntiles = ((M + kBM - 1) / kBM) * ((N + step - 1) / step);
    const unsigned grid = (unsigned)(ntiles < sms ? ntiles : sms);
    switch (ep.mode) {
        case EPI_STORE_BF16: return launch_epi<EPI_STORE_BF16>(tma, tmb, grid, M, N, K, C, ldc, ep, err, s);
        case EPI_STORE_F32: return launch_epi<EPI_STORE_F32>(tma, tmb, grid, M, N, K, C, ldc, ep, err, s);
        case EPI_CONV_BF16: return launch_epi<EPI_CONV_BF16>(tma, tmb, grid, M, N, K, C, ldc, ep, err, s);
        case EPI_SILU_F32: return launch_epi<EPI_SILU_F32>(tma, tmb, grid, M, N, K, C, ldc, ep, err, s);
        case EPI_GELU_BF16: return launch_epi<EPI_GELU_BF16>(tma, tmb, grid, M, N, K, C, ldc, ep, err, s);
        case EPI_ADD_F32: return launch_epi<EPI_ADD_F32>(tma, tmb, grid, M, N, K, C, ldc, ep, err, s);
        case EPI_ADD_BF16: return launch_epi<EPI_ADD_BF16>(tma, tmb, grid, M, N, K, C, ldc, ep, err, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_gemm_tc(const void *A, const void *Bm, int64_t M, int64_t N, int64_t K, void *C,
                           int64_t ldc, GemmEpi epi, const float *bias, DevErr err, cudaStream_t s) {
    GemmEpiArgs ep;
    ep.mode = epi;
    ep.bias = bias;
    return launch_gemm_tc_ex(A, Bm, M, N, K, C, ldc, ep, err, s);
}

}  // namespace hm

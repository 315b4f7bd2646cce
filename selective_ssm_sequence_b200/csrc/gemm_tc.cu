// gemm_tc.cu -- C[M, N] = A[M, K] . B[N, K]^T on the 5th-generation tensor cores.
//
// The dense projections of the HedgeMamba mixer (q, k, v, gate and output
// projections; HedgeMamba explainer sec. 2.3 and 5.2) are plain GEMMs with
// nn.Linear weights (y = x W^T), so both operands are K-major.  Persistent
// kernel, one CTA per SM: 128 x 256 output tiles, 64-wide K blocks streamed by
// TMA through a 4-stage ring, tcgen05.mma (bf16 -> fp32 in TMEM) issued by one
// thread, and two TMEM accumulators so that the epilogue of one tile overlaps
// the MMAs of the next.  Warp roles: 0 = TMA, 1 = MMA, 2..5 = epilogue.
#include "tc_common.cuh"

namespace hm {

namespace {

using namespace tc;

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;   // 16 KB
constexpr int kBBytes = kBN * kBK * 2;   // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;

struct GAux {
    uint64_t full[kStages], empty[kStages];
    uint64_t accf[2], acce[2];
    uint32_t tmem;
    int abort;
};

constexpr int kGSmem = kStages * kStageBytes + (int)sizeof(GAux) + 1024;

template <int EPI>
__global__ void __launch_bounds__(192, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb,
               int64_t M, int64_t N, int64_t K, void *__restrict__ C, int64_t ldc,
               const float *__restrict__ bias, DevErr err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    GAux *X = (GAux *)(smem + kStages * kStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tiles_m = (M + kBM - 1) / kBM, tiles_n = (N + kBN - 1) / kBN;
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
            mbar_init(&X->acce[b], 128);
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
                const int m0 = (int)((t / tiles_n) * kBM), n0 = (int)((t % tiles_n) * kBN);
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
        int tl = 0;
        for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++tl) {
            const int b = tl & 1;
            if (!mbar_wait(&X->accf[b], (tl >> 1) & 1, abort_flag, err, KID_GEMM_TC, 4)) break;
            tc_fence_after();
            const int64_t m = (t / tiles_n) * kBM + row;
            const int64_t n0 = (t % tiles_n) * kBN;
            const uint32_t ta = tmem + b * kBN + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(ta + c0, r);
                tmem_wait_ld();
                if (c0 + 32 >= kBN) {
                    tc_fence_before();
                    mbar_arrive(&X->acce[b]);
                }
                if (m < M) {
                    if constexpr (EPI == EPI_STORE_BF16) {
                        __nv_bfloat16 *dst = (__nv_bfloat16 *)C + m * ldc + n0 + c0;
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            if (n0 + c0 + 8 * v < N) {
                                uint4 w;
                                w.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
                                w.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
                                w.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
                                w.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
                                *reinterpret_cast<uint4 *>(dst + 8 * v) = w;
                            }
                        }
                    } else {
                        float *dst = (float *)C + m * ldc + n0 + c0;
#pragma unroll
                        for (int v = 0; v < 8; ++v) {
                            if (n0 + c0 + 4 * v < N) {
                                float4 w;
                                const int64_t nn = n0 + c0 + 4 * v;
                                w.x = __uint_as_float(r[4 * v + 0]) + (bias ? bias[nn + 0] : 0.f);
                                w.y = __uint_as_float(r[4 * v + 1]) + (bias ? bias[nn + 1] : 0.f);
                                w.z = __uint_as_float(r[4 * v + 2]) + (bias ? bias[nn + 2] : 0.f);
                                w.w = __uint_as_float(r[4 * v + 3]) + (bias ? bias[nn + 3] : 0.f);
                                *reinterpret_cast<float4 *>(dst + 4 * v) = w;
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

cudaError_t launch_gemm_tc(const void *A, const void *Bm, int64_t M, int64_t N, int64_t K, void *C,
                           int64_t ldc, GemmEpi epi, const float *bias, DevErr err, cudaStream_t s) {
    if (!gemm_tc_supported(M, N, K)) return cudaErrorNotSupported;
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
    const int64_t ntiles = ((M + kBM - 1) / kBM) * ((N + kBN - 1) / kBN);
    const unsigned grid = (unsigned)(ntiles < sms ? ntiles : sms);
    cudaError_t e;
    if (epi == EPI_STORE_BF16) {
        e = ensure_smem_limit(gemm_tc_kernel<EPI_STORE_BF16>, kGSmem);
        if (e != cudaSuccess) return e;
        gemm_tc_kernel<EPI_STORE_BF16><<<grid, 192, kGSmem, s>>>(tma, tmb, M, N, K, C, ldc, bias, err);
    } else {
        e = ensure_smem_limit(gemm_tc_kernel<EPI_STORE_F32>, kGSmem);
        if (e != cudaSuccess) return e;
        gemm_tc_kernel<EPI_STORE_F32><<<grid, 192, kGSmem, s>>>(tma, tmb, M, N, K, C, ldc, bias, err);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace hm

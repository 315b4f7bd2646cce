// featmap_tc.cu -- Hedgehog feature map on the 5th-generation tensor cores.
//
//   u = W x (+ b)  ;  phi = softmax([u, -u])  over the 2p features
//
// (HedgeMamba explainer sec. 2.1 and 5.3.)  The projection is a dense GEMM
// (rows x d) . (d x p), so it runs as tcgen05.mma (bf16 operands from shared
// memory, fp32 accumulator in TMEM).  Per CTA: one head (blockIdx.y) whose
// W [p, d] is loaded once by TMA and stays in shared memory; 128-row tiles of
// x stream through a 2-stage TMA ring.  Warp roles:
//   warp 0      TMA producer (one elected lane)
//   warp 1      TMEM allocator and MMA issuer (one elected lane)
//   warps 2..13 three epilogue warpgroups taking tiles in turn: one
//               accumulator row per thread, read from TMEM in two passes (a
//               running max / normaliser, then the normalised features), the
//               negate / concatenate / softmax in registers in the log2
//               domain (one FMA-free exp2 per feature).  The features (bf16
//               or fp32) leave through a per-warpgroup staging buffer and TMA
//               stores of 128 rows x 64 bytes: a thread owns a row, so direct
//               stores would touch 32 rows (1-2 KB apart) per instruction.
// Four TMEM accumulators let the MMAs run ahead of the epilogue warpgroups.
#include "tc_common.cuh"

namespace hm {

namespace {

using namespace tc;

constexpr int kBM = 128;     // rows per tile (MMA M)
constexpr int kStages = 2;   // x tiles in flight
constexpr int kEpiWG = 3;    // epilogue warpgroups (tiles in turn)
constexpr int kThreads = 64 + 128 * kEpiWG;

template <int D, int P>
struct FmLayout {
    static constexpr int kChunks = D / 64;                  // 128-byte K chunks
    static constexpr int kWBytes = kChunks * P * 128;       // W tile
    static constexpr int kXChunkBytes = kBM * 128;          // one K chunk of an x tile
    static constexpr int kXBytes = kChunks * kXChunkBytes;  // one x tile
    static constexpr int kOffW = 0;
    static constexpr int kOffX = kWBytes;
    static constexpr int kStgBytes = kBM * 64;               // output staging: 128 rows x 64 bytes
    static constexpr int kOffStg = kOffX + kStages * kXBytes;
    static constexpr int kOffBar = kOffStg + kEpiWG * kStgBytes;
    static constexpr int kSmem = kOffBar + 256 + 1024;      // + barriers, + alignment slack
    static_assert(kSmem <= 227 * 1024, "feature-map shared memory");
    static constexpr int kAcc = 512 / P >= 4 ? 4 : 2;       // TMEM accumulators
    static constexpr int kTmemCols = kAcc * P <= 256 ? 256 : 512;
};

struct FmBars {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t wbar;
    uint64_t accf[4];
    uint64_t acce[4];
    uint32_t tmem;
    int abort;
};

constexpr float kLog2e = 1.4426950408889634f;

template <int D, int P, typename TP, bool kHasBias>
__global__ void __launch_bounds__(kThreads, 1)
featmap_tc_kernel(const __grid_constant__ CUtensorMap tmx0, const __grid_constant__ CUtensorMap tmw0,
                  const __grid_constant__ CUtensorMap tmx1, const __grid_constant__ CUtensorMap tmw1,
                  const __grid_constant__ CUtensorMap tmo0, const __grid_constant__ CUtensorMap tmo1,
                  int64_t Tv, int Hv, const float *__restrict__ bias0, const float *__restrict__ bias1,
                  int bias_per_head, TP *__restrict__ phi0, TP *__restrict__ phi1,
                  __nv_bfloat16 *__restrict__ phi_lo0, __nv_bfloat16 *__restrict__ phi_lo1, DevErr err) {
    // blockIdx.z selects one of two independent inputs of the same shape (the
    // q and k maps of a scan run in one launch)
    const bool second = blockIdx.z != 0;
    const CUtensorMap &tmx = second ? tmx1 : tmx0;
    const CUtensorMap &tmw = second ? tmw1 : tmw0;
    const CUtensorMap &tmo = second ? tmo1 : tmo0;   // phi as (F, H, rows), 64-byte swizzle
    const float *__restrict__ bias = second ? bias1 : bias0;
    __nv_bfloat16 *__restrict__ phi_lo = second ? phi_lo1 : phi_lo0;
    using Lay = FmLayout<D, P>;
    constexpr int NA = Lay::kAcc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    uint8_t *sW = smem + Lay::kOffW;
    uint8_t *sX = smem + Lay::kOffX;
    FmBars *bars = (FmBars *)(smem + Lay::kOffBar);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int64_t ntiles = (Tv + kBM - 1) / kBM;
    volatile int *abort_flag = &bars->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        mbar_init(&bars->wbar, 1);
        for (int b = 0; b < NA; ++b) {
            mbar_init(&bars->accf[b], 1);
            mbar_init(&bars->acce[b], 4);   // one arrival per epilogue warp
        }
        bars->abort = 0;
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(&bars->tmem, Lay::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (elect_one()) {
            tma_prefetch_desc(&tmx);
            tma_prefetch_desc(&tmw);
            mbar_arrive_expect_tx(&bars->wbar, Lay::kWBytes);
            for (int c = 0; c < Lay::kChunks; ++c)
                tma_load_2d(sW + c * P * 128, &tmw, &bars->wbar, c * 64, h * P);
            int it = 0;
            for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
                const int s = it % kStages;
                const uint32_t ph = (it / kStages) & 1;
                if (!mbar_wait(&bars->empty[s], ph ^ 1, abort_flag, err, KID_FEATMAP_TC, 1)) break;
                mbar_arrive_expect_tx(&bars->full[s], Lay::kXBytes);
                uint8_t *dst = sX + s * Lay::kXBytes;
                for (int c = 0; c < Lay::kChunks; ++c)
                    tma_load_3d(dst + c * Lay::kXChunkBytes, &tmx, &bars->full[s], c * 64, h,
                                (int)(tile * kBM));
            }
            // make sure no copy is still landing in shared memory before exit
            const int issued = it;
            for (int j = issued - kStages; j < issued; ++j) {
                if (j < 0) continue;
                const int s = j % kStages;
                for (uint32_t i = 0; i < kWaitPolls; ++i)
                    if (mbar_try_wait(&bars->full[s], (j / kStages) & 1)) break;
            }
            for (uint32_t i = 0; i < kWaitPolls; ++i)
                if (mbar_try_wait(&bars->wbar, 0)) break;
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (elect_one()) {
            constexpr uint32_t idesc = idesc_bf16(kBM, P, false, false);
            bool ok = mbar_wait(&bars->wbar, 0, abort_flag, err, KID_FEATMAP_TC, 2);
            int it = 0;
            for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++it) {
                const int s = it % kStages;
                const uint32_t ph = (it / kStages) & 1;
                const int b = it % NA;
                const uint32_t bph = (it / NA) & 1;
                if (!mbar_wait(&bars->acce[b], bph ^ 1, abort_flag, err, KID_FEATMAP_TC, 3)) break;
                if (!mbar_wait(&bars->full[s], ph, abort_flag, err, KID_FEATMAP_TC, 4)) break;
                tc_fence_after();
                const uint32_t xa = smem_u32(sX + s * Lay::kXBytes);
                const uint32_t wa = smem_u32(sW);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const int c = k >> 2, kk = k & 3;
                    const uint64_t ad = desc_k_sw128(xa + c * Lay::kXChunkBytes + kk * 32);
                    const uint64_t bd = desc_k_sw128(wa + c * P * 128 + kk * 32);
                    mma_ss(tmem + b * P, ad, bd, idesc, k > 0 ? 1u : 0u);
                }
                mma_commit(&bars->empty[s]);
                mma_commit(&bars->accf[b]);
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        // warpgroup e takes tiles e, e + kEpiWG, ...; each thread one row.
        const int e = (warp - 2) >> 2;
        const int q = warp & 3;              // TMEM lane quarter of this warp
        const int row_in_tile = q * 32 + lane;
        const int wt = threadIdx.x - 64 - 128 * e;   // thread within the warpgroup
        uint8_t *const stg = smem + Lay::kOffStg + e * Lay::kStgBytes;
        constexpr int F = 2 * P;
        const float *bh = bias ? bias + (bias_per_head ? (int64_t)h * P : 0) : nullptr;
        int it = e;
        for (int64_t tile = blockIdx.x + (int64_t)e * gridDim.x; tile < ntiles;
             tile += (int64_t)kEpiWG * gridDim.x, it += kEpiWG) {
            const int b = it % NA;
            const uint32_t bph = (it / NA) & 1;
            const bool okw = mbar_wait(&bars->accf[b], bph, abort_flag, err, KID_FEATMAP_TC, 5);
            // the warpgroup leaves together (its threads meet at named barriers)
            if (!named_sync_and(1 + e, 128, okw)) break;
            tc_fence_after();
            const uint32_t tbase = tmem + b * P + ((uint32_t)(q * 32) << 16);
            const int64_t t = tile * kBM + row_in_tile;
            const bool valid = t < Tv;
            __nv_bfloat16 *lo = (phi_lo && valid) ? phi_lo + (t * Hv + h) * (int64_t)F : nullptr;
            // Everything in the log2 domain: y = u log2(e).  Pass 1: running max
            // m of |y| and normaliser Z = sum 2^(y - m) + 2^(-y - m), rescaled
            // when m grows.  Pass 2: phi = 2^(+-y - sh) with sh = m + log2 Z, so
            // the normalisation costs nothing per feature.  The TMEM load of
            // the next 32 columns is in flight while a block is processed.
            auto yv = [&](const uint32_t *r, int c, int j) {
                return (__uint_as_float(r[j]) + ((kHasBias && bh) ? bh[c + j] : 0.f)) * kLog2e;
            };
            float m = 0.f, Z = 0.f;
            auto pass1 = [&](const uint32_t *r, int c) {
                float mc = m;
#pragma unroll
                for (int j = 0; j < 32; ++j) mc = fmaxf(mc, fabsf(yv(r, c, j)));
                float z0 = 0.f, z1 = 0.f;
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float y0 = yv(r, c, j), y1 = yv(r, c, j + 1);
                    z0 += ex2_approx(y0 - mc) + ex2_approx(-y0 - mc);
                    z1 += ex2_approx(y1 - mc) + ex2_approx(-y1 - mc);
                }
                Z = Z * ex2_approx(m - mc) + (z0 + z1);
                m = mc;
            };
            {
                uint32_t ra[32], rb[32];
                tmem_ld32(tbase, ra);
                tmem_wait_ld();
#pragma unroll 1
                for (int c = 0; c < P; c += 64) {
                    tmem_ld32(tbase + c + 32, rb);
                    pass1(ra, c);
                    tmem_wait_ld();
                    if (c + 64 < P) tmem_ld32(tbase + c + 64, ra);
                    pass1(rb, c + 32);
                    tmem_wait_ld();
                }
            }
            const float sh = m + lg2_approx(Z);
            if constexpr (sizeof(TP) == 2) {
                // bf16 phi: each half of a 32-column block (32 features of one
                // row per thread) goes through the warpgroup's staging buffer
                // (64-byte rows, 64-byte swizzle: conflict-free 16-byte writes)
                // and leaves by one TMA store of 128 rows x 64 bytes
                auto stage_half = [&](const uint32_t *r, int c, int hf) {
                    uint32_t pk[16];
                    const float sg = hf ? -1.f : 1.f;
                    uint32_t lw[4];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float y0 = sg * yv(r, c, 2 * j), y1 = sg * yv(r, c, 2 * j + 1);
                        const float p0 = ex2_approx(y0 - sh), p1 = ex2_approx(y1 - sh);
                        pk[j] = pack_bf16x2(p0, p1);
                        if (lo) {
                            // remainder phi - bf16(phi), so that hi + lo carries ~16 bits
                            const float2 hv = unpack_bf16x2(pk[j]);
                            lw[j & 3] = pack_bf16x2(p0 - hv.x, p1 - hv.y);
                            if ((j & 3) == 3)
                                *reinterpret_cast<uint4 *>(lo + hf * P + c + 2 * (j - 3)) =
                                    make_uint4(lw[0], lw[1], lw[2], lw[3]);
                        }
                    }
                    if (wt == 0) bulk_wait_read_all();   // the previous store has read the buffer
                    named_sync(1 + e, 128);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int pc = j ^ ((row_in_tile >> 1) & 3);
                        *reinterpret_cast<uint4 *>(stg + row_in_tile * 64 + pc * 16) =
                            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                    }
                    fence_proxy_async_smem();
                    named_sync(1 + e, 128);
                    if (wt == 0) {
                        tma_store_3d(&tmo, stg, hf * P + c, h, (int)(tile * kBM));
                        bulk_commit();
                    }
                };
#pragma unroll 1
                for (int c = 0; c < P; c += 32) {
                    uint32_t r[32];
                    tmem_ld32(tbase + c, r);
                    tmem_wait_ld();
                    if (c + 32 >= P) {
                        // the last read of this accumulator has landed
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bars->acce[b]);
                    }
                    stage_half(r, c, 0);
                    stage_half(r, c, 1);
                }
            } else {
                // fp32 phi: as the bf16 path, through the warpgroup's staging
                // buffer, 16 features (64 bytes) of each row per TMA store of
                // 128 rows (a thread owns a row, so direct stores would touch 32
                // rows 1 KB apart per instruction)
                auto stage16 = [&](const uint32_t *r, int c, int neg, int q16) {
                    float ev[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float y = yv(r, c, 16 * q16 + j);
                        ev[j] = ex2_approx((neg ? -y : y) - sh);
                    }
                    if (wt == 0) bulk_wait_read_all();   // the previous store has read the buffer
                    named_sync(1 + e, 128);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int pc = j ^ ((row_in_tile >> 1) & 3);
                        *reinterpret_cast<float4 *>(stg + row_in_tile * 64 + pc * 16) =
                            make_float4(ev[4 * j], ev[4 * j + 1], ev[4 * j + 2], ev[4 * j + 3]);
                    }
                    fence_proxy_async_smem();
                    named_sync(1 + e, 128);
                    if (wt == 0) {
                        tma_store_3d(&tmo, stg, neg * P + c + 16 * q16, h, (int)(tile * kBM));
                        bulk_commit();
                    }
                };
#pragma unroll 1
                for (int c = 0; c < P; c += 32) {
                    uint32_t r[32];
                    tmem_ld32(tbase + c, r);
                    tmem_wait_ld();
                    if (c + 32 >= P) {
                        // the last read of this accumulator has landed
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bars->acce[b]);
                    }
                    stage16(r, c, 0, 0);
                    stage16(r, c, 0, 1);
                    stage16(r, c, 1, 0);
                    stage16(r, c, 1, 1);
                }
            }
        }
        // the staging buffer is read (and the stores issued) before the CTA ends
        if (wt == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, Lay::kTmemCols);
    }
}

// One launch for up to two inputs (x1 == nullptr: one).
template <int D, int P, typename TP>
cudaError_t go(const void *x0, const void *W0, const float *bias0, void *phi0, void *lo0, const void *x1,
               const void *W1, const float *bias1, void *phi1, void *lo1, int64_t rows, int H,
               int64_t w_head_stride, DevErr err, cudaStream_t s) {
    using Lay = FmLayout<D, P>;
    const bool per_head = w_head_stride != 0;
    const int Hv = per_head ? H : 1;
    const int64_t Tv = rows / Hv;
    const int nz = x1 ? 2 : 1;
    CUtensorMap tmx[2], tmw[2], tmo[2];
    for (int z = 0; z < nz; ++z) {
        if constexpr (sizeof(TP) == 2) {
            // phi [rows, F] bf16 viewed as (F, Hv, Tv); boxes of 32 features x 128 rows
            uint64_t dims[3] = {(uint64_t)(2 * P), (uint64_t)Hv, (uint64_t)Tv};
            uint64_t strides[2] = {(uint64_t)(2 * P) * 2, (uint64_t)Hv * (2 * P) * 2};
            uint32_t box[3] = {32, 1, kBM};
            if (!tc::make_tmap(&tmo[z], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, z ? phi1 : phi0, 3, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_64B))
                return cudaErrorInvalidValue;
        }
        {
            uint64_t dims[3] = {(uint64_t)D, (uint64_t)Hv, (uint64_t)Tv};
            uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)Hv * D * 2};
            uint32_t box[3] = {64, 1, kBM};
            if (!tc::make_tmap_bf16(&tmx[z], z ? x1 : x0, 3, dims, strides, box)) return cudaErrorInvalidValue;
        }
        {
            // W rows: head h's [P, D] starts at row h * P when the stride is P * D
            uint64_t dims[2] = {(uint64_t)D, (uint64_t)Hv * P};
            uint64_t strides[1] = {(uint64_t)D * 2};
            uint32_t box[2] = {64, (uint32_t)P};
            if (!tc::make_tmap_bf16(&tmw[z], z ? W1 : W0, 2, dims, strides, box)) return cudaErrorInvalidValue;
        }
    }
    if constexpr (sizeof(TP) != 2) {
        // phi [rows, F] fp32 viewed as (F, Hv, Tv); boxes of 16 features x 128 rows
        for (int z = 0; z < nz; ++z) {
            uint64_t dims[3] = {(uint64_t)(2 * P), (uint64_t)Hv, (uint64_t)Tv};
            uint64_t strides[2] = {(uint64_t)(2 * P) * 4, (uint64_t)Hv * (2 * P) * 4};
            uint32_t box[3] = {16, 1, kBM};
            if (!tc::make_tmap(&tmo[z], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, z ? phi1 : phi0, 3, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_64B))
                return cudaErrorInvalidValue;
        }
    }
    if (nz == 1) {
        tmx[1] = tmx[0];
        tmw[1] = tmw[0];
        tmo[1] = tmo[0];
    }
    auto kern = (bias0 || bias1) ? featmap_tc_kernel<D, P, TP, true> : featmap_tc_kernel<D, P, TP, false>;
    cudaError_t e = ensure_smem_limit(kern, Lay::kSmem);
    if (e != cudaSuccess) return e;
    const int64_t ntiles = (Tv + kBM - 1) / kBM;
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t per_head_ctas = (sms + Hv * nz - 1) / (Hv * nz);
    if (per_head_ctas > ntiles) per_head_ctas = ntiles;
    if (per_head_ctas < 1) per_head_ctas = 1;
    dim3 grid((unsigned)per_head_ctas, (unsigned)Hv, (unsigned)nz);
    kern<<<grid, kThreads, Lay::kSmem, s>>>(tmx[0], tmw[0], tmx[1], tmw[1], tmo[0], tmo[1], Tv, Hv, bias0, bias1, per_head ? 1 : 0,
                                            (TP *)phi0, (TP *)phi1, (__nv_bfloat16 *)lo0, (__nv_bfloat16 *)lo1,
                                            err);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

bool featmap_tc_supported(int64_t rows, int H, int d, int p, int64_t w_head_stride) {
    if (rows <= 0) return false;
    if (!(d == 64 || d == 128 || d == 256)) return false;
    if (!(p == 64 || p == 128)) return false;
    if (w_head_stride != 0 && (w_head_stride != (int64_t)p * d || rows % H != 0 || H > 65535)) return false;
    const int Hv = w_head_stride ? H : 1;
    if (rows / Hv > 0x7fffffffLL - 256) return false;  // TMA coordinates are 32-bit
    return true;
}

cudaError_t launch_featmap_tc2(const void *x0, const void *W0, const float *bias0, void *phi0, void *lo0,
                               const void *x1, const void *W1, const float *bias1, void *phi1, void *lo1,
                               int64_t rows, int H, int d, int p, int64_t w_head_stride, hm_dtype pt, DevErr err,
                               cudaStream_t s) {
    if (!featmap_tc_supported(rows, H, d, p, w_head_stride)) return cudaErrorNotSupported;
    if ((lo0 || lo1) && pt != HM_BF16) return cudaErrorInvalidValue;
#define HM_FM_CASE(DD, PP)                                                                              \
    if (d == DD && p == PP)                                                                             \
        return pt == HM_BF16 ? go<DD, PP, __nv_bfloat16>(x0, W0, bias0, phi0, lo0, x1, W1, bias1, phi1, lo1, \
                                                         rows, H, w_head_stride, err, s)                  \
                             : go<DD, PP, float>(x0, W0, bias0, phi0, nullptr, x1, W1, bias1, phi1, nullptr, \
                                                 rows, H, w_head_stride, err, s);
    HM_FM_CASE(64, 64)
    HM_FM_CASE(64, 128)
    HM_FM_CASE(128, 64)
    HM_FM_CASE(128, 128)
    HM_FM_CASE(256, 64)
    HM_FM_CASE(256, 128)
#undef HM_FM_CASE
    return cudaErrorNotSupported;
}

cudaError_t launch_featmap_tc(const void *x, int64_t rows, int H, int d, int p, const void *W,
                              int64_t w_head_stride, const float *bias, void *phi, hm_dtype pt,
                              DevErr err, cudaStream_t s, void *phi_lo) {
    return launch_featmap_tc2(x, W, bias, phi, phi_lo, nullptr, nullptr, nullptr, nullptr, nullptr, rows, H, d, p,
                              w_head_stride, pt, err, s);
}

}  // namespace hm

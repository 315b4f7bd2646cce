// segment.cu -- what a sequence cut into consecutive segments (one per GPU,
// say) needs besides the per-segment scans: each segment's total log decay,
// and the start state of every segment from the segments' zero-start end
// states.
//
// A segment's effect on the state it starts from is the affine map
//     S -> exp(lambda) (.) S + S_seg,   z -> exp(lambda) (.) z + z_seg
// with lambda = sum over its tokens of log a_t (one value per head, or per
// (head, feature) with the per-feature decay) and (S_seg, z_seg) its end state
// from a zero start.  These maps compose associatively (SSM article sec. 4.2,
// the affine-map composition behind the parallel scan), so the start of
// segment r is the composition of segments 0..r-1 applied to the initial
// state.  Both kernels are bandwidth-bound and small next to the scan.
#include "hm_internal.h"

namespace hm {

namespace {

// lambda[b, h] (or [b, h, f]) = sum_t log a_t over the L tokens of the call.
// log a_t = -softplus(dt_t) * rate with a rate per head (or per (head,
// feature)) that does not depend on t, so lambda = -rate * sum_t softplus(dt_t)
// (0 when the rate is 0).  One warp per (b, h): lanes over tokens, a warp
// reduction, then one value (or F values) written.
__global__ void __launch_bounds__(256)
logdecay_sum_kernel(int64_t B, int64_t L, int H, int F, int per_feature, const float *__restrict__ dt,
                    const float *__restrict__ A_log, float *__restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t bh = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (bh >= B * H) return;
    const int64_t b = bh / H;
    const int h = (int)(bh % H);
    float sp = 0.f;
    for (int64_t t = lane; t < L; t += 32) sp += hm_softplus(dt[(b * L + t) * H + h]);
    sp = warp_sum(sp);
    if (!per_feature) {
        if (lane == 0) {
            const float rate = expf(A_log[h]);
            out[bh] = rate == 0.f ? 0.f : -sp * rate;
        }
    } else {
        for (int f = lane; f < F; f += 32) {
            const float rate = expf(A_log[(int64_t)h * F + f]);
            out[bh * F + f] = rate == 0.f ? 0.f : -sp * rate;
        }
    }
}

// Start states of consecutive segments.  Thread: 4 consecutive elements of
// one head's [S | z] (S: F * dv values, then z: F values; F * dv and F are
// multiples of 4).  It walks the parts in order, writing the running state
// before adding each part.
__global__ void __launch_bounds__(256)
combine_kernel(hm_combine_args a) {
    const int64_t nS = (int64_t)a.F * a.dv;
    const int64_t per_head = (nS + a.F) / 4;                 // 16-byte groups per head
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= a.BH * per_head) return;
    const int64_t bh = gid / per_head;
    const int64_t e = (gid % per_head) * 4;                  // element within [S | z]
    const bool isz = e >= nS;
    const int f = isz ? (int)(e - nS) : (int)(e / a.dv);     // feature of the first element
    // log-decay values per record, padded to 16 bytes so that S and z stay aligned
    const int64_t nl = ((a.per_feature ? a.BH * a.F : a.BH) + 3) / 4 * 4;
    const int64_t offS = nl, offz = nl + a.BH * nS;
    const int64_t dst = isz ? bh * a.F + (e - nS) : bh * nS + e;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float *src0 = isz ? a.z0 : a.S0;
    if (src0) acc = *reinterpret_cast<const float4 *>(src0 + dst);
    float *ds = isz ? a.z_start : a.S_start;
    const int64_t blk = isz ? a.BH * a.F : a.BH * nS;        // one part's block of starts
    for (int64_t r = 0; r < a.n_parts; ++r) {
        if (a.only_part < 0) *reinterpret_cast<float4 *>(ds + r * blk + dst) = acc;
        else if (a.only_part == r) *reinterpret_cast<float4 *>(ds + dst) = acc;
        const float *rec = a.parts + r * a.part_len;
        const float4 p = *reinterpret_cast<const float4 *>(rec + (isz ? offz : offS) + dst);
        float g[4];
        if (a.per_feature) {
            // z: four features; S: four value columns of one feature row
#pragma unroll
            for (int j = 0; j < 4; ++j) g[j] = expf(rec[bh * a.F + (isz ? f + j : f)]);
        } else {
            const float gg = expf(rec[bh]);
#pragma unroll
            for (int j = 0; j < 4; ++j) g[j] = gg;
        }
        acc = make_float4(fmaf(g[0], acc.x, p.x), fmaf(g[1], acc.y, p.y), fmaf(g[2], acc.z, p.z),
                          fmaf(g[3], acc.w, p.w));
    }
    float *de = isz ? a.z_end : a.S_end;
    if (de) *reinterpret_cast<float4 *>(de + dst) = acc;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

cudaError_t launch_logdecay_sum(int64_t B, int64_t L, int H, int F, bool per_feature, const float *dt,
                                const float *A_log, float *out, cudaStream_t s) {
    if (B * H == 0) return cudaSuccess;
    if (!dt || L == 0) {
        // no decay (or no tokens): the call applies no decay, lambda = 0
        return cudaMemsetAsync(out, 0, sizeof(float) * (size_t)(per_feature ? B * H * F : B * H), s);
    }
    const unsigned blocks = (unsigned)((B * H * 32 + 255) / 256);
    logdecay_sum_kernel<<<blocks, 256, 0, s>>>(B, L, H, F, per_feature ? 1 : 0, dt, A_log, out);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace hm

using namespace hm;

extern "C" hm_status hm_scan_combine(const hm_combine_args *a, hm_stream_t stream) {
    set_error_detail("");
    auto reject = [](const char *msg) {
        set_error_detail(msg);
        return HM_ERR_INVALID_ARG;
    };
    if (!a) return reject("combine: null args");
    if (a->n_parts < 0 || a->BH < 0 || a->F < 1 || a->dv < 1) return reject("combine: bad sizes");
    if (a->F % 4 != 0 || a->dv % 4 != 0 || a->part_len % 4 != 0)
        return reject("combine: F, dv and part_len must be multiples of 4");
    if (a->only_part < -1 || a->only_part >= a->n_parts) return reject("combine: only_part out of range");
    const int64_t nS = (int64_t)a->F * a->dv;
    const int64_t need = ((a->per_feature ? a->BH * a->F : a->BH) + 3) / 4 * 4 + a->BH * nS + a->BH * a->F;
    if (a->part_len < need) return reject("combine: part_len smaller than one [log_decay | S | z] record");
    if ((a->S0 == nullptr) != (a->z0 == nullptr)) return reject("combine: S0 and z0 must both be given or both NULL");
    if ((a->S_end == nullptr) != (a->z_end == nullptr))
        return reject("combine: S_end and z_end must both be given or both NULL");
    if (a->n_parts > 0 && a->BH > 0 && (!a->parts || !a->S_start || !a->z_start))
        return reject("combine: null parts or start buffers");
    const void *ptrs[] = {a->parts, a->S0, a->z0, a->S_start, a->z_start, a->S_end, a->z_end};
    for (const void *p : ptrs)
        if (!aligned16(p)) return reject("combine: pointers must be 16-byte aligned");
    const int64_t threads = a->BH * (nS + a->F) / 4;
    if (threads == 0) return HM_OK;
    combine_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, (cudaStream_t)stream>>>(*a);
    count_launches(1);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error_detail(cudaGetErrorString(e));
        return HM_ERR_CUDA;
    }
    return HM_OK;
}

// decode_step.cu -- one decode step inside a window, reading only the sketch.
//
// SketchSSM (arXiv 2609.33051v1), Abstract: each decode step combines the
// sketch vectors with query-dependent coefficients instead of reading the full
// state; agihunt digest, bullet "Mechanism details": within a window the state
// is fixed and only the query changes, so a query written as a combination of
// basis vectors has as output the same combination of the stored outputs.
//
// Step j of a window: tokens 0..j-1 of the buffer are not in the window-start
// state S0 whose sketch is P.  Since S_j = M_j S_{j-1} + b_j k_j v_j^T,
//     S_j^T q = S0^T q~ + o_buf,
// where the backward pass over the buffered tokens carries the query back
// (q~ = M_1^T ... M_j^T q) and collects their exact contribution o_buf.  The
// sketch replaces S0^T q~ by P (R q~).  Nothing is written to S.
//
// One warp per head (heads in (h, b) order, so a CTA's warps share R rows).
// A decode step is one memory round trip per head: the head's buffered k and v
// (and KDA decay) rows are contiguous blocks of the head-major window buffer
// and arrive by TMA bulk copies into the warp's shared-memory slots, while the
// query, the per-token scalars (one token per lane), the first eight R rows and
// the matching sketch rows are loaded into registers at the same time.  The
// backward pass then runs from shared memory: per token one warp reduction for
// k . w and one axpy.  Scalar decay is kept as a running scale next to the
// carried query (w = g w^), so Mamba-2's dot products do not depend on each
// other.  The wait on the copies is bounded: a give-up is counted in a device
// flag (sketchssm_device_error_count) and the warp returns.
#include "internal.h"
#include "state_tile.cuh"

namespace skssm {

constexpr int DEC_WARPS = 8;  // one head per warp
constexpr int DEC_RPRE = 8;   // coefficient rows held in registers from the start
constexpr unsigned DEC_WAIT_TRIES = 1u << 22;

__device__ unsigned g_device_error;

__device__ __forceinline__ unsigned dec_smem(const void *p) { return (unsigned)__cvta_generic_to_shared(p); }

__device__ __forceinline__ bool dec_wait(const uint64_t *bar, int phase) {
    for (unsigned it = 0; it < DEC_WAIT_TRIES; ++it) {
        unsigned done;
        asm volatile(
            "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }\n"
            : "=r"(done)
            : "r"(dec_smem(bar)), "r"(phase)
            : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ void dec_bulk(void *dst, const void *src, int bytes, const uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                     dec_smem(dst)),
                 "l"(src), "r"(bytes), "r"(dec_smem(bar))
                 : "memory");
}

// Per-warp shared memory: barrier (16 B), then jc slots of k rows, v rows, (KDA) decay rows.
template <int KIND, int DK, int DV, typename QT>
struct DecSlots {
    static constexpr int KB = DK * (int)sizeof(QT), VB = DV * (int)sizeof(QT);
    static constexpr int AB = KIND == KDA ? DK * 4 : 0;
    __host__ __device__ static int bytes(int jc) { return 16 + jc * (KB + VB + AB); }
};

template <int N, typename T>
__device__ __forceinline__ void load_n(const T *p, float *out) {
    if constexpr (N == 4) load4(p, out);
    else load2(p, out);
}

template <int KIND, int DK, int DV, typename QT>
__global__ void __launch_bounds__(DEC_WARPS * 32)
decode_step_kernel(const float *__restrict__ P, const float *__restrict__ R, const QT *__restrict__ qv,
                   const QT *__restrict__ kbuf, const QT *__restrict__ vbuf,
                   const float *__restrict__ abuf, const float *__restrict__ bbuf,
                   float *__restrict__ o, int B, int H, int r, int j, int W, int jc) {
    using SL = DecSlots<KIND, DK, DV, QT>;
    constexpr int KPL = DK / 32, VPL = DV / 32;  // channels of the carried query / output per lane
    extern __shared__ __align__(16) char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NH = B * H;
    const int oi = blockIdx.x * DEC_WARPS + warp;
    if (oi >= NH) return;  // the whole warp
    const int h = oi / B;
    const int head = (oi % B) * H + h;
    char *wb = smem + (size_t)warp * SL::bytes(jc);
    uint64_t *bar = reinterpret_cast<uint64_t *>(wb);
    char *ks = wb + 16, *vs = ks + jc * SL::KB, *as = vs + jc * SL::VB;
    if (lane == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(dec_smem(bar)) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncwarp();

    // registers, all requested before the first wait: query, R rows, sketch rows
    float w[KPL], rr[DEC_RPRE][KPL], pp[VPL][DEC_RPRE], ob[VPL];
    load_n<KPL>(qv + (size_t)head * DK + lane * KPL, w);
    const float *Rh = R + (size_t)h * r * DK;
#pragma unroll
    for (int m = 0; m < DEC_RPRE; ++m) {
        if (m < r) load_n<KPL>(Rh + (size_t)m * DK + lane * KPL, rr[m]);
        else {
#pragma unroll
            for (int e = 0; e < KPL; ++e) rr[m][e] = 0.f;
        }
    }
    const float *Ph = P + (size_t)head * DV * r;
#pragma unroll
    for (int e = 0; e < VPL; ++e) {
        const float *row = Ph + (size_t)(lane * VPL + e) * r;
        if ((r & 3) == 0 && r >= DEC_RPRE) {
            load4(row, pp[e]);
            load4(row + 4, pp[e] + 4);
        } else {
#pragma unroll
            for (int m = 0; m < DEC_RPRE; ++m) pp[e][m] = m < r ? row[m] : 0.f;
        }
        ob[e] = 0.f;
    }
    float gsc = 1.f;  // w = gsc * w^ (Mamba-2, GDN)

    int phase = 0;
    for (int thi = j - 1; thi >= 0; thi -= jc) {
        const int tlo = thi - jc + 1 > 0 ? thi - jc + 1 : 0;
        const int nt = thi - tlo + 1;
        const size_t row0 = (size_t)head * W + tlo;  // the chunk's rows are contiguous
        const float a_l = (KIND != KDA && lane < nt) ? abuf[row0 + lane] : 1.f;
        const float b_l = (KIND != MAMBA2 && lane < nt) ? bbuf[row0 + lane] : 1.f;
        if (lane == 0) {
            asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(dec_smem(bar)),
                         "r"(nt * (SL::KB + SL::VB + SL::AB))
                         : "memory");
            dec_bulk(ks, kbuf + row0 * DK, nt * SL::KB, bar);
            dec_bulk(vs, vbuf + row0 * DV, nt * SL::VB, bar);
            if (KIND == KDA) dec_bulk(as, abuf + row0 * DK, nt * SL::AB, bar);
        }
        if (!dec_wait(bar, phase)) {
            if (lane == 0) atomicAdd(&g_device_error, 1u);
            dec_wait(bar, phase);  // give the copies in flight a last bounded chance to land
            return;
        }
        phase ^= 1;
        for (int t = thi; t >= tlo; --t) {
            const int sl = t - tlo;
            float kf[KPL], vf[VPL];
            load_n<KPL>(reinterpret_cast<const QT *>(ks + sl * SL::KB) + lane * KPL, kf);
            load_n<VPL>(reinterpret_cast<const QT *>(vs + sl * SL::VB) + lane * VPL, vf);
            const float at = __shfl_sync(FULL, a_l, sl), bt = __shfl_sync(FULL, b_l, sl);
            float x = 0.f;
#pragma unroll
            for (int e = 0; e < KPL; ++e) x = fmaf(kf[e], w[e], x);
            x = warp_sum(x);  // k . w (k . w^ for scalar decay)
            if (KIND == KDA) {
                const float s = bt * x;
#pragma unroll
                for (int e = 0; e < VPL; ++e) ob[e] = fmaf(s, vf[e], ob[e]);
                float a[KPL];
                load_n<KPL>(reinterpret_cast<const float *>(as + sl * SL::AB) + lane * KPL, a);
#pragma unroll
                for (int e = 0; e < KPL; ++e) w[e] = a[e] * fmaf(-s, kf[e], w[e]);
            } else {
                const float s = bt * gsc * x;  // b (k . w), w = gsc w^
#pragma unroll
                for (int e = 0; e < VPL; ++e) ob[e] = fmaf(s, vf[e], ob[e]);
                if (KIND == GDN) {
#pragma unroll
                    for (int e = 0; e < KPL; ++e) w[e] = fmaf(-bt * x, kf[e], w[e]);  // w^ -= b (k . w^) k
                }
                gsc *= at;
            }
        }
        __syncwarp();  // every lane is done with the slots before the next chunk refills them
    }
    if (KIND != KDA) {
#pragma unroll
        for (int e = 0; e < KPL; ++e) w[e] *= gsc;
    }

    // c = R q~, o = P c + o_buf: the first DEC_RPRE rows from registers, the rest streamed
    float acc[VPL];
#pragma unroll
    for (int e = 0; e < VPL; ++e) acc[e] = ob[e];
#pragma unroll
    for (int m = 0; m < DEC_RPRE; ++m) {
        if (m < r) {
            float p = 0.f;
#pragma unroll
            for (int e = 0; e < KPL; ++e) p = fmaf(rr[m][e], w[e], p);
            const float c = warp_sum(p);
#pragma unroll
            for (int e = 0; e < VPL; ++e) acc[e] = fmaf(pp[e][m], c, acc[e]);
        }
    }
    for (int m = DEC_RPRE; m < r; ++m) {
        float rv[KPL];
        load_n<KPL>(Rh + (size_t)m * DK + lane * KPL, rv);
        float p = 0.f;
#pragma unroll
        for (int e = 0; e < KPL; ++e) p = fmaf(rv[e], w[e], p);
        const float c = warp_sum(p);
#pragma unroll
        for (int e = 0; e < VPL; ++e) acc[e] = fmaf(Ph[(size_t)(lane * VPL + e) * r + m], c, acc[e]);
    }
    float *oh = o + (size_t)head * DV + lane * VPL;
    if constexpr (VPL == 4) *reinterpret_cast<float4 *>(oh) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    else *reinterpret_cast<float2 *>(oh) = make_float2(acc[0], acc[1]);
}

int launch_decode_step(const sketchssm_dims &d, const float *P, const float *R, const void *q,
                       const void *k, const void *v, const float *alpha, const float *beta, int j,
                       float *o, cudaStream_t stream) {
    // the kernel does not touch the state: both state dtypes dispatch to the same instantiation
    return dispatch(d, [&](auto K, auto D, auto *, auto *qp) -> int {
        using QT = std::remove_pointer_t<decltype(qp)>;
        constexpr int KIND = decltype(K)::value, DK = decltype(D)::value;
        const int NH = d.B * d.H;
        const int grid = (NH + DEC_WARPS - 1) / DEC_WARPS;
        auto go = [&](auto DVc) -> int {
            constexpr int DV = decltype(DVc)::value;
            const int jmax = KIND == KDA ? 16 : 32;  // tokens per bulk round trip (<= 32: one per lane)
            const int jc = j < jmax ? j : jmax;
            const size_t smem = (size_t)DEC_WARPS * DecSlots<KIND, DK, DV, QT>::bytes(jc);
            auto kern = decode_step_kernel<KIND, DK, DV, QT>;
            static bool opted_in = false;
            if (!opted_in) {
                if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
                    cudaSuccess)
                    return SKSSM_ERR_CUDA;
                opted_in = true;
            }
            kern<<<grid, DEC_WARPS * 32, smem, stream>>>(P, R, static_cast<const QT *>(q),
                                                         static_cast<const QT *>(k), static_cast<const QT *>(v),
                                                         alpha, beta, o, d.B, d.H, d.r, j, d.W, jc);
            return launch_status();
        };
        if (d.dv == 64) return go(std::integral_constant<int, 64>());
        if (d.dv == 128) return go(std::integral_constant<int, 128>());
        return SKSSM_ERR_DIMS;
    });
}

}  // namespace skssm

extern "C" int sketchssm_device_error_count(int reset) {
    unsigned n = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return SKSSM_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&n, skssm::g_device_error, sizeof(n)) != cudaSuccess) return SKSSM_ERR_CUDA;
    if (reset && n) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(skssm::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return SKSSM_ERR_CUDA;
    }
    return (int)n;
}

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
// query, the per-token scalars (one token per lane) and the first eight sketch
// columns are loaded into registers at the same time.  The backward pass then
// runs from shared memory: per token one warp reduction for k . w and one axpy.
// Scalar decay is kept as a running scale next to the carried query (w = g w^),
// so Mamba-2's dot products do not depend on each other and eight of them share
// one warp all-reduce.  The coefficient rows R (the same for every b) are read
// after the pass, from L1/L2, so that they hold no registers while the copies
// are in flight: 64 registers per thread keep eight 4-warp CTAs on an SM.  The
// wait on the copies is bounded: a give-up is counted in a device flag
// (sketchssm_device_error_count) and the warp returns.
#include "internal.h"
#include "state_tile.cuh"

namespace skssm {

constexpr int DEC_WARPS = 4;  // one head per warp; small CTAs pack the SMs more tightly (measured)
constexpr int DEC_RPRE = 8;   // sketch columns held in registers from the start; R rows per all-reduce
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

    // registers, all requested before the first wait: query and the first sketch rows (the
    // coefficient rows R are shared by the warps of a head index h and come from L1/L2 later)
    float w[KPL], pp[VPL][DEC_RPRE], ob[VPL];
    load_n<KPL>(qv + (size_t)head * DK + lane * KPL, w);
    const float *Rh = R + (size_t)h * r * DK;
    const float *Ph = P + (size_t)head * DV * r;
#pragma unroll
    for (int e = 0; e < VPL; ++e) {
        const float *row = Ph + (size_t)(lane * VPL + e) * r;
        if ((r & 3) == 0 && r >= DEC_RPRE) {
            const float4 a = *reinterpret_cast<const float4 *>(row), b = *reinterpret_cast<const float4 *>(row + 4);
            pp[e][0] = a.x; pp[e][1] = a.y; pp[e][2] = a.z; pp[e][3] = a.w;
            pp[e][4] = b.x; pp[e][5] = b.y; pp[e][6] = b.z; pp[e][7] = b.w;
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
        if constexpr (KIND == MAMBA2) {
            // w stays q: the dots of eight tokens are independent and share one warp all-reduce
            for (int t0 = thi; t0 >= tlo; t0 -= 8) {
                float x[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    x[u] = 0.f;
                    if (t0 - u >= tlo) {
                        float kf[KPL];
                        load_n<KPL>(reinterpret_cast<const QT *>(ks + (t0 - u - tlo) * SL::KB) + lane * KPL, kf);
#pragma unroll
                        for (int e = 0; e < KPL; ++e) x[u] = fmaf(kf[e], w[e], x[u]);
                    }
                }
                warp_allreduce8(x, lane);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (t0 - u >= tlo) {  // warp-uniform
                        const int sl = t0 - u - tlo;
                        float vf[VPL];
                        load_n<VPL>(reinterpret_cast<const QT *>(vs + sl * SL::VB) + lane * VPL, vf);
                        const float s = gsc * x[u];  // (k . q) times the decay of the later tokens
#pragma unroll
                        for (int e = 0; e < VPL; ++e) ob[e] = fmaf(s, vf[e], ob[e]);
                        gsc *= __shfl_sync(FULL, a_l, sl);
                    }
                }
            }
        } else
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

    // c = R q~ in blocks of eight rows (one warp all-reduce per block), o = P c + o_buf; the
    // sketch rows of the first block are already in registers
    float acc[VPL];
#pragma unroll
    for (int e = 0; e < VPL; ++e) acc[e] = ob[e];
#pragma unroll 1
    for (int m0 = 0; m0 < r; m0 += DEC_RPRE) {
        float c[DEC_RPRE];  // rows m >= r are zero
#pragma unroll
        for (int mm = 0; mm < DEC_RPRE; ++mm) {
            c[mm] = 0.f;
            if (m0 + mm < r) {
                float rv[KPL];
                load_n<KPL>(Rh + (size_t)(m0 + mm) * DK + lane * KPL, rv);
#pragma unroll
                for (int e = 0; e < KPL; ++e) c[mm] = fmaf(rv[e], w[e], c[mm]);
            }
        }
        warp_allreduce8(c, lane);
        if (m0 == 0) {
#pragma unroll
            for (int mm = 0; mm < DEC_RPRE; ++mm)
#pragma unroll
                for (int e = 0; e < VPL; ++e) acc[e] = fmaf(pp[e][mm], c[mm], acc[e]);
        } else {
#pragma unroll
            for (int mm = 0; mm < DEC_RPRE; ++mm)
                if (m0 + mm < r) {
#pragma unroll
                    for (int e = 0; e < VPL; ++e)
                        acc[e] = fmaf(Ph[(size_t)(lane * VPL + e) * r + m0 + mm], c[mm], acc[e]);
                }
        }
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
            // tokens per bulk round trip (<= 32: one per lane); KDA rows are twice as wide, and fewer
            // of them per trip keep more warps resident
            const int jmax = KIND == KDA ? 8 : 32;
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

int skssm::decode_wait_giveups(bool reset, unsigned *count) {
    return read_counter(&g_device_error, reset, count);
}

extern "C" int sketchssm_device_error_count(int reset) {
    if (cudaDeviceSynchronize() != cudaSuccess) return SKSSM_ERR_CUDA;
    unsigned dec = 0, upd = 0;
    if (skssm::decode_wait_giveups(reset != 0, &dec) != SKSSM_OK ||
        skssm::update_wait_giveups(reset != 0, &upd) != SKSSM_OK)
        return SKSSM_ERR_CUDA;
    return (int)(dec + upd);
}

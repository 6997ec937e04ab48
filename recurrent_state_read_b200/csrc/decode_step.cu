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
// One warp per head: the lane holds dk/32 channels of the carried query and
// dv/32 channels of the output.  Per buffered token: one warp all-reduce for
// k . w; tokens are fetched four at a time so their loads overlap.  Traffic per
// head: P (dv*r*4 B), q, j buffered tokens (L2-resident within a window), o.
#include "internal.h"
#include "state_tile.cuh"

namespace skssm {

constexpr int DEC_WARPS = 4;

template <int N> struct Lanes;
template <> struct Lanes<2> {
    template <typename T> __device__ static void ld(const T *p, float *o) { load2(p, o); }
};
template <> struct Lanes<4> {
    template <typename T> __device__ static void ld(const T *p, float *o) { load4(p, o); }
};

template <int KIND, int DK, int DV, typename QT>
__global__ void __launch_bounds__(DEC_WARPS * 32)
decode_step_kernel(const float *__restrict__ P, const float *__restrict__ R, const QT *__restrict__ qv,
                   const QT *__restrict__ kbuf, const QT *__restrict__ vbuf,
                   const float *__restrict__ abuf, const float *__restrict__ bbuf,
                   float *__restrict__ o, int NH, int H, int r, int j) {
    constexpr int KPL = DK / 32, VPL = DV / 32;
    constexpr int APL = KIND == KDA ? KPL : 1;
    __shared__ float scoef[DEC_WARPS][128];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int head = blockIdx.x * DEC_WARPS + warp;
    if (head >= NH) return;  // whole warp leaves together
    const int h = head % H;

    float w[KPL], ob[VPL];
    Lanes<KPL>::ld(qv + (size_t)head * DK + lane * KPL, w);
#pragma unroll
    for (int e = 0; e < VPL; ++e) ob[e] = 0.f;

    for (int t = j - 1; t >= 0; t -= 4) {
        float kr[4][KPL], vr[4][VPL], ar[4][APL], br[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int tt = t - u;
            if (tt >= 0) {
                const size_t base = (size_t)tt * NH + head;
                Lanes<KPL>::ld(kbuf + base * DK + lane * KPL, kr[u]);
                Lanes<VPL>::ld(vbuf + base * DV + lane * VPL, vr[u]);
                if (KIND == KDA) Lanes<KPL>::ld(abuf + base * DK + lane * KPL, ar[u]);
                else ar[u][0] = abuf[base];
                br[u] = KIND == MAMBA2 ? 1.f : bbuf[base];
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (t - u >= 0) {
                float x = 0.f;
#pragma unroll
                for (int e = 0; e < KPL; ++e) x = fmaf(kr[u][e], w[e], x);
                x = warp_sum(x);
                const float s = br[u] * x;
#pragma unroll
                for (int e = 0; e < VPL; ++e) ob[e] = fmaf(s, vr[u][e], ob[e]);
#pragma unroll
                for (int e = 0; e < KPL; ++e) {
                    const float a = KIND == KDA ? ar[u][e] : ar[u][0];
                    w[e] = KIND == MAMBA2 ? a * w[e] : a * fmaf(-s, kr[u][e], w[e]);
                }
            }
        }
    }

    // coefficients c = R q~
    const float *Rh = R + (size_t)h * r * DK + lane * KPL;
    for (int m = 0; m < r; ++m) {
        float rv[KPL];
        Lanes<KPL>::ld(Rh + (size_t)m * DK, rv);
        float p = 0.f;
#pragma unroll
        for (int e = 0; e < KPL; ++e) p = fmaf(rv[e], w[e], p);
        p = warp_sum(p);
        if (lane == 0) scoef[warp][m] = p;
    }
    __syncwarp();

    // o = P c + o_buf
#pragma unroll
    for (int e = 0; e < VPL; ++e) {
        const int c = lane * VPL + e;
        const float *row = P + ((size_t)head * DV + c) * r;
        float acc = ob[e];
        int m = 0;
        if ((r & 3) == 0) {
            for (; m < r; m += 4) {
                const float4 pv = *reinterpret_cast<const float4 *>(row + m);
                acc = fmaf(pv.x, scoef[warp][m], acc);
                acc = fmaf(pv.y, scoef[warp][m + 1], acc);
                acc = fmaf(pv.z, scoef[warp][m + 2], acc);
                acc = fmaf(pv.w, scoef[warp][m + 3], acc);
            }
        }
        for (; m < r; ++m) acc = fmaf(row[m], scoef[warp][m], acc);
        o[(size_t)head * DV + c] = acc;
    }
}

int launch_decode_step(const sketchssm_dims &d, const float *P, const float *R, const void *q,
                       const void *k, const void *v, const float *alpha, const float *beta, int j,
                       float *o, cudaStream_t stream) {
    if (d.r > 128) return SKSSM_ERR_DIMS;
    return dispatch(d, [&](auto K, auto D, auto *, auto *qp) -> int {
        using QT = std::remove_pointer_t<decltype(qp)>;
        constexpr int KIND = decltype(K)::value, DK = decltype(D)::value;
        const int NH = d.B * d.H;
        const int grid = (NH + DEC_WARPS - 1) / DEC_WARPS;
        auto go = [&](auto DVc) -> int {
            constexpr int DV = decltype(DVc)::value;
            decode_step_kernel<KIND, DK, DV, QT><<<grid, DEC_WARPS * 32, 0, stream>>>(
                P, R, static_cast<const QT *>(q), static_cast<const QT *>(k), static_cast<const QT *>(v),
                alpha, beta, o, NH, d.H, d.r, j);
            return launch_status();
        };
        if (d.dv == 64) return go(std::integral_constant<int, 64>());
        if (d.dv == 128) return go(std::integral_constant<int, 128>());
        return SKSSM_ERR_DIMS;
    });
}

}  // namespace skssm

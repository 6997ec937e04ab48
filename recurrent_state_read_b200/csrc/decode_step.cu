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
// Mapping: a lane octet (8 lanes) per head, four heads per warp.  A lane holds
// dk/8 channels of the carried query and dv/8 channels of the output, in runs
// of one 16-byte q/k/v vector (the state tile's interleave), so every load of a
// token row is a 128-byte run per octet and each dot product needs a 3-level
// octet reduction.  Scalar decay is kept as a running scale g next to the
// carried query (w = g w^): for Mamba-2 w^ = q never changes, so all buffered
// tokens' dot products are independent; for GDN each token costs one dot and
// one axpy.  Tokens are fetched TB at a time ahead of use, and the head's
// sketch rows are prefetched into L2 when the warp starts.
#include "internal.h"
#include "state_tile.cuh"

namespace skssm {

constexpr int DEC_WARPS = 4;
constexpr int DEC_HEADS_PER_WARP = 4;

template <int KIND, int DK, int DV, typename QT>
__global__ void __launch_bounds__(DEC_WARPS * 32)
decode_step_kernel(const float *__restrict__ P, const float *__restrict__ R, const QT *__restrict__ qv,
                   const QT *__restrict__ kbuf, const QT *__restrict__ vbuf,
                   const float *__restrict__ abuf, const float *__restrict__ bbuf,
                   float *__restrict__ o, int NH, int H, int r, int j) {
    using QV = typename Vec<QT>::type;
    constexpr int QN = Vec<QT>::N;         // elements per 16-byte q/k/v vector
    constexpr int KPL = DK / 8, VPL = DV / 8;
    constexpr int KQ = KPL / QN, VQ = VPL / QN;
    constexpr int APL = KIND == KDA ? KPL : 1;
    constexpr int TB = KIND == KDA ? 2 : 4;  // tokens fetched ahead
    static_assert(KQ >= 1 && VQ >= 1, "unsupported widths");

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int l = lane & 7, g = lane >> 3;
    const int head_raw = (blockIdx.x * DEC_WARPS + warp) * DEC_HEADS_PER_WARP + g;
    const bool live = head_raw < NH;
    const int head = live ? head_raw : NH - 1;  // dead octets mirror a valid head and store nothing
    const int h = head % H;
    auto kch = [&](int q, int e) { return QN * (l + 8 * q) + e; };  // lane's channel runs

    // the sketch rows of this head go to L2 first
    {
        const char *prow = reinterpret_cast<const char *>(P + (size_t)head * DV * r);
        const int bytes = DV * r * 4;
        for (int off = l * 128; off < bytes; off += 8 * 128)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(prow + off));
    }

    float w[KPL], ob[VPL];
#pragma unroll
    for (int q = 0; q < KQ; ++q) {
        const QV a = *reinterpret_cast<const QV *>(qv + (size_t)head * DK + kch(q, 0));
        unpack16<QT>(a, w + q * QN);
    }
#pragma unroll
    for (int e = 0; e < VPL; ++e) ob[e] = 0.f;
    float gsc = 1.f;  // w = gsc * w^ (Mamba-2, GDN)

    for (int t0 = j - 1; t0 >= 0; t0 -= TB) {
        QV kr[TB][KQ], vr[TB][VQ];
        float ar[TB][APL], br[TB];
#pragma unroll
        for (int u = 0; u < TB; ++u) {
            const int t = t0 - u;
            if (t >= 0) {
                const size_t base = (size_t)t * NH + head;
#pragma unroll
                for (int q = 0; q < KQ; ++q) kr[u][q] = *reinterpret_cast<const QV *>(kbuf + base * DK + kch(q, 0));
#pragma unroll
                for (int q = 0; q < VQ; ++q) vr[u][q] = *reinterpret_cast<const QV *>(vbuf + base * DV + kch(q, 0));
                if (KIND == KDA) {
#pragma unroll
                    for (int q = 0; q < KQ; ++q)
#pragma unroll
                        for (int e4 = 0; e4 < QN; e4 += 4) {
                            const float4 a = *reinterpret_cast<const float4 *>(abuf + base * DK + kch(q, e4));
                            ar[u][q * QN + e4] = a.x; ar[u][q * QN + e4 + 1] = a.y;
                            ar[u][q * QN + e4 + 2] = a.z; ar[u][q * QN + e4 + 3] = a.w;
                        }
                } else {
                    ar[u][0] = abuf[base];
                }
                br[u] = KIND == MAMBA2 ? 1.f : bbuf[base];
            }
        }
#pragma unroll
        for (int u = 0; u < TB; ++u) {
            if (t0 - u >= 0) {
                float kf[KPL], vf[VPL];
#pragma unroll
                for (int q = 0; q < KQ; ++q) unpack16<QT>(kr[u][q], kf + q * QN);
#pragma unroll
                for (int q = 0; q < VQ; ++q) unpack16<QT>(vr[u][q], vf + q * QN);
                const float xh = octet_sum(dot<KPL>(kf, w));  // k . w (w^ for scalar decay)
                if (KIND == KDA) {
                    const float s = br[u] * xh;
#pragma unroll
                    for (int e = 0; e < VPL; ++e) ob[e] = fmaf(s, vf[e], ob[e]);
#pragma unroll
                    for (int e = 0; e < KPL; ++e) w[e] = ar[u][e] * fmaf(-s, kf[e], w[e]);
                } else {
                    const float s = br[u] * gsc * xh;  // b (k . w), w = gsc w^
#pragma unroll
                    for (int e = 0; e < VPL; ++e) ob[e] = fmaf(s, vf[e], ob[e]);
                    if (KIND == GDN) axpy<KPL>(w, kf, -br[u] * xh);  // w^ -= b (k . w^) k
                    gsc *= ar[u][0];
                }
            }
        }
    }
    if (KIND != KDA) {
#pragma unroll
        for (int e = 0; e < KPL; ++e) w[e] *= gsc;
    }

    // c = R q~ (chunks of 8 coefficients: per-lane partials, octet reduce-scatter,
    // octet all-gather), then o = P c + o_buf
    const float *Rh = R + (size_t)h * r * DK;
    const float *Ph = P + (size_t)head * DV * r;
    float acc[VPL];
#pragma unroll
    for (int e = 0; e < VPL; ++e) acc[e] = ob[e];
    for (int m0 = 0; m0 < r; m0 += 8) {
        float part[8];
#pragma unroll
        for (int mm = 0; mm < 8; ++mm) {
            part[mm] = 0.f;
            if (m0 + mm < r) {
                float rv[KPL];
#pragma unroll
                for (int q = 0; q < KQ; ++q)
#pragma unroll
                    for (int e4 = 0; e4 < QN; e4 += 4) load4(Rh + (size_t)(m0 + mm) * DK + kch(q, e4), rv + q * QN + e4);
                part[mm] = dot<KPL>(rv, w);
            }
        }
        float coef[8];
        octet_all_gather(octet_reduce_scatter(part, lane), coef);
#pragma unroll
        for (int q = 0; q < VQ; ++q)
#pragma unroll
            for (int e = 0; e < QN; ++e) {
                const float *row = Ph + (size_t)kch(q, e) * r + m0;
                float a = acc[q * QN + e];
                if ((r & 3) == 0) {
                    const float4 p0 = *reinterpret_cast<const float4 *>(row);
                    a = fmaf(p0.x, coef[0], a); a = fmaf(p0.y, coef[1], a);
                    a = fmaf(p0.z, coef[2], a); a = fmaf(p0.w, coef[3], a);
                    if (m0 + 4 < r) {
                        const float4 p1 = *reinterpret_cast<const float4 *>(row + 4);
                        a = fmaf(p1.x, coef[4], a); a = fmaf(p1.y, coef[5], a);
                        a = fmaf(p1.z, coef[6], a); a = fmaf(p1.w, coef[7], a);
                    }
                } else {
#pragma unroll
                    for (int mm = 0; mm < 8; ++mm)
                        if (m0 + mm < r) a = fmaf(row[mm], coef[mm], a);
                }
                acc[q * QN + e] = a;
            }
    }
    if (live) {
        float *oh = o + (size_t)head * DV;
#pragma unroll
        for (int q = 0; q < VQ; ++q)
#pragma unroll
            for (int e4 = 0; e4 < QN; e4 += 4)
                *reinterpret_cast<float4 *>(oh + kch(q, e4)) =
                    make_float4(acc[q * QN + e4], acc[q * QN + e4 + 1], acc[q * QN + e4 + 2], acc[q * QN + e4 + 3]);
    }
}

int launch_decode_step(const sketchssm_dims &d, const float *P, const float *R, const void *q,
                       const void *k, const void *v, const float *alpha, const float *beta, int j,
                       float *o, cudaStream_t stream) {
    // the kernel does not touch the state: both state dtypes dispatch to the same instantiation
    return dispatch(d, [&](auto K, auto D, auto *, auto *qp) -> int {
        using QT = std::remove_pointer_t<decltype(qp)>;
        constexpr int KIND = decltype(K)::value, DK = decltype(D)::value;
        const int NH = d.B * d.H;
        const int per_cta = DEC_WARPS * DEC_HEADS_PER_WARP;
        const int grid = (NH + per_cta - 1) / per_cta;
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

// fullread.cu -- the full-read baseline: one decode step that reads, updates and
// writes the whole state and returns o = S_t^T q_t.
//
// This is the access pattern the SketchSSM abstract compares against (the
// standard vLLM decode path), and the one the agihunt digest's "Background"
// bullet describes: every decode step reads the full recurrent state.  The
// kernel streams each head's state once (one read, one write) with the same
// register tile as the window update, and folds the read into the same pass:
//   Mamba-2  S' = a S + k v^T                 o_c = a (q.S_c) + (q.k) v_c
//   GDN      x = k.S_c, u = b (v_c - a x)     S' = a S + k u,      o_c = a (q.S_c) + (q.k) u
//   KDA      x = (k(.)a).S_c, u = b (v_c - x) S' = a(.)S + k u,   o_c = (q(.)a).S_c + (q.k) u
// so each column needs at most two dot products, reduced across its lane octet.
#include "internal.h"
#include "state_tile.cuh"

namespace skssm {

template <int KIND, int DK, typename ST, typename QT>
__global__ void __launch_bounds__(128)
fullread_kernel(ST *__restrict__ S, const QT *__restrict__ qv, const QT *__restrict__ kv,
                const QT *__restrict__ vv, const float *__restrict__ av, const float *__restrict__ bv,
                float *__restrict__ o, int NH, int dv) {
    using TL = TileLayout<DK, ST>;
    constexpr int EPL = TL::EPL;
    const int head = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane & 7, g = lane >> 3;
    const int c0 = warp * 32 + g * 8;

    float s[8][EPL];
    ST *Sh = S + (size_t)head * dv * DK;
    load_tile<DK, ST>(Sh, c0, l, s);

    float kk[EPL], qq[EPL];
    lane_channels_global<DK, ST, QT>(kv + (size_t)head * DK, l, kk);
    lane_channels_global<DK, ST, QT>(qv + (size_t)head * DK, l, qq);
    const float qk = octet_sum(dot<EPL>(qq, kk));

    float out;
    if (KIND == MAMBA2) {
        const float a = av[head];
        float d[8];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) d[cc] = dot<EPL>(qq, s[cc]);
        const float y = octet_reduce_scatter(d, lane);
        float vc8[8];
        load4(vv + (size_t)head * dv + c0, vc8);
        load4(vv + (size_t)head * dv + c0 + 4, vc8 + 4);
        float vmine = vc8[0];
#pragma unroll
        for (int cc = 1; cc < 8; ++cc) vmine = (l == cc) ? vc8[cc] : vmine;
        out = a * y + qk * vmine;
        const float2 a2 = make_float2(a, a);
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
            const float2 v2 = make_float2(vc8[cc], vc8[cc]);
#pragma unroll
            for (int e = 0; e < EPL; e += 2) {
                float2 r = fma2(make_float2(s[cc][e], s[cc][e + 1]), a2,
                                fma2(make_float2(kk[e], kk[e + 1]), v2, make_float2(0.f, 0.f)));
                s[cc][e] = r.x; s[cc][e + 1] = r.y;
            }
        }
    } else {
        const float b = bv[head];
        float aa[EPL];
        float a = 1.f;
        if (KIND == KDA) {
            float ka[EPL], qa[EPL];
#pragma unroll
            for (int q = 0; q < TL::NQ; ++q)
#pragma unroll
                for (int e4 = 0; e4 < TL::VEC; e4 += 4)
                    load4(av + (size_t)head * DK + TL::chan(l, q, e4), aa + q * TL::VEC + e4);
#pragma unroll
            for (int e = 0; e < EPL; ++e) { ka[e] = kk[e] * aa[e]; qa[e] = qq[e] * aa[e]; }
            float dx[8], dy[8];
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) { dx[cc] = dot<EPL>(ka, s[cc]); dy[cc] = dot<EPL>(qa, s[cc]); }
            const float x = octet_reduce_scatter(dx, lane);
            const float y = octet_reduce_scatter(dy, lane);
            const float vc = ld1(vv + (size_t)head * dv + c0 + l);
            const float u = b * (vc - x);
            out = y + qk * u;
            float uu[8];
            octet_all_gather(u, uu);
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                const float2 u2 = make_float2(uu[cc], uu[cc]);
#pragma unroll
                for (int e = 0; e < EPL; e += 2) {
                    float2 r = fma2(make_float2(aa[e], aa[e + 1]), make_float2(s[cc][e], s[cc][e + 1]),
                                    fma2(make_float2(kk[e], kk[e + 1]), u2, make_float2(0.f, 0.f)));
                    s[cc][e] = r.x; s[cc][e + 1] = r.y;
                }
            }
        } else {
            a = av[head];
            float dx[8], dy[8];
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) { dx[cc] = dot<EPL>(kk, s[cc]); dy[cc] = dot<EPL>(qq, s[cc]); }
            const float x = octet_reduce_scatter(dx, lane);
            const float y = octet_reduce_scatter(dy, lane);
            const float vc = ld1(vv + (size_t)head * dv + c0 + l);
            const float u = b * (vc - a * x);
            out = a * y + qk * u;
            float uu[8];
            octet_all_gather(u, uu);
            const float2 a2 = make_float2(a, a);
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                const float2 u2 = make_float2(uu[cc], uu[cc]);
#pragma unroll
                for (int e = 0; e < EPL; e += 2) {
                    float2 r = fma2(make_float2(s[cc][e], s[cc][e + 1]), a2,
                                    fma2(make_float2(kk[e], kk[e + 1]), u2, make_float2(0.f, 0.f)));
                    s[cc][e] = r.x; s[cc][e + 1] = r.y;
                }
            }
        }
    }
    o[(size_t)head * dv + c0 + l] = out;
    store_tile<DK, ST>(Sh, c0, l, s);
}

int launch_fullread(const sketchssm_dims &d, void *S, const void *q, const void *k, const void *v,
                    const float *alpha, const float *beta, float *o, cudaStream_t stream) {
    return dispatch(d, [&](auto K, auto D, auto *sp, auto *qp) -> int {
        using ST = std::remove_pointer_t<decltype(sp)>;
        using QT = std::remove_pointer_t<decltype(qp)>;
        constexpr int KIND = decltype(K)::value, DK = decltype(D)::value;
        const int NH = d.B * d.H;
        fullread_kernel<KIND, DK, ST, QT><<<NH, d.dv, 0, stream>>>(
            static_cast<ST *>(S), static_cast<const QT *>(q), static_cast<const QT *>(k),
            static_cast<const QT *>(v), alpha, beta, o, NH, d.dv);
        return launch_status();
    });
}

}  // namespace skssm

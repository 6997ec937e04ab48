// decode_common.cuh -- the backward pass over buffered tokens shared by the sketch
// decode step and the full-state (ReplaySSM-style) decode step.
//
// Step j of a window: tokens 0..j-1 of the buffer are not in the window-start
// state S0.  Since S_j = M_j S_{j-1} + b_j k_j v_j^T,  S_j^T q = S0^T q~ + o_buf,
// where the pass carries the query back through the buffered tokens (q~) and
// collects their exact contribution o_buf (SketchSSM abstract; the buffering of
// keys and values between state updates is ReplaySSM's).
#pragma once

#include "internal.h"
#include "state_tile.cuh"

namespace skssm {

constexpr int DEC_RPRE = 8;   // sketch columns held in registers from the start; R rows per all-reduce

__device__ __forceinline__ unsigned dec_smem(const void *p) { return smem_u32(p); }

// Shared-memory slots of buffered tokens: 16 bytes (a barrier where one is used), then
// jc k rows, jc v rows and (KDA) jc decay rows, each in its storage type.
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

// The backward pass over one chunk of buffered tokens held in shared memory
// (slots 0 .. nt-1, oldest first; ks/vs/as their k, v and KDA decay rows), newest
// first: per token x = k . w, o_buf += b x v, w <- M^T w.  Lane t holds the chunk's
// token-t scalars a_l, b_l.  For scalar decay w is kept as gsc * w^.
template <int KIND, int DK, int DV, typename QT>
__device__ __forceinline__ void backward_chunk(const char *ks, const char *vs, const char *as, int nt, float a_l,
                                               float b_l, float (&w)[DK / 32], float (&ob)[DV / 32], float &gsc,
                                               int lane) {
    using SL = DecSlots<KIND, DK, DV, QT>;
    constexpr int KPL = DK / 32, VPL = DV / 32;
    if constexpr (KIND == MAMBA2) {
        // w stays q: the dots of eight tokens are independent and share one warp all-reduce
        for (int t0 = nt - 1; t0 >= 0; t0 -= 8) {
            float x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                x[u] = 0.f;
                if (t0 - u >= 0) {
                    float kf[KPL];
                    load_n<KPL>(reinterpret_cast<const QT *>(ks + (t0 - u) * SL::KB) + lane * KPL, kf);
#pragma unroll
                    for (int e = 0; e < KPL; ++e) x[u] = fmaf(kf[e], w[e], x[u]);
                }
            }
            warp_allreduce8(x, lane);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (t0 - u >= 0) {  // warp-uniform
                    const int sl = t0 - u;
                    float vf[VPL];
                    load_n<VPL>(reinterpret_cast<const QT *>(vs + sl * SL::VB) + lane * VPL, vf);
                    const float s = gsc * x[u];  // (k . q) times the decay of the later tokens
#pragma unroll
                    for (int e = 0; e < VPL; ++e) ob[e] = fmaf(s, vf[e], ob[e]);
                    gsc *= __shfl_sync(FULL, a_l, sl);
                }
            }
        }
    } else {
        for (int sl = nt - 1; sl >= 0; --sl) {
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
    }
}

// acc[e] += sum_{mm < 8, m0 + mm < lim} P[c_e][m0 + mm] c[mm] for the lane's value channels
// c_e = VPL lane + e (sketch rows of r floats at Ph), four columns at a time: one 16-byte
// piece per row when r is a multiple of 4, else one column at a time.
template <int VPL>
__device__ __forceinline__ void sketch_block(const float *Ph, int r, int m0, int lim, const float (&c)[8],
                                             float (&acc)[VPL], int lane) {
#pragma unroll
    for (int q = 0; q < 8; q += 4) {
        if (m0 + q >= lim) break;  // warp-uniform
        float pv[VPL][4];
#pragma unroll
        for (int e = 0; e < VPL; ++e) {
            const float *row = Ph + (size_t)(lane * VPL + e) * r + m0 + q;
            if ((r & 3) == 0) {
                const float4 a = *reinterpret_cast<const float4 *>(row);
                pv[e][0] = a.x; pv[e][1] = a.y; pv[e][2] = a.z; pv[e][3] = a.w;
            } else {
#pragma unroll
                for (int mm = 0; mm < 4; ++mm) pv[e][mm] = m0 + q + mm < r ? row[mm] : 0.f;
            }
        }
#pragma unroll
        for (int mm = 0; mm < 4; ++mm)
            if (m0 + q + mm < lim) {
#pragma unroll
                for (int e = 0; e < VPL; ++e) acc[e] = fmaf(pv[e][mm], c[q + mm], acc[e]);
            }
    }
}

}  // namespace skssm

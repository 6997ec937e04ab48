// wy_decode.cu -- the delta-rule decode step with the buffered tokens' key Gram
// matrix kept across the window's steps (WY / T-matrix form of the backward pass).
//
// The sketch decode step (decode_step.cu) carries the query back through the
// buffered tokens one token at a time, and every token waits on the previous
// token's warp reduction.  Written out, the pass solves a triangular system
// (GDN, KDA; with scalar decay a_v is the same in every key channel):
//     D_t = a_{t+1} (.) ... (.) a_{j-1}              (decay after token t, D_{j-1} = 1)
//     p_t = sum_i k_t[i] q[i] D_t[i]
//     G_ut = sum_i k_t[i] k_u[i] a_{t+1}[i] ... a_u[i]        (t < u; independent of j)
//     s_u = b_u (p_u - sum_{t' > u} G_t'u s_t')   for u = j-1 down to 0
//     o_buf = sum_u s_u v_u
//     q~ = D_{-1} (.) q - sum_u s_u k_u (.) E_u,   E_u = a_0 (.) ... (.) a_u
// (the same quantities the token-by-token pass produces: x_u = k_u . w_u and
// s_u = b_u x_u).  Column u of G only involves tokens up to u, so step j computes
// one new column (u = j-1) and reads the others from a per-head buffer that the
// window's earlier steps wrote: all dot products of a step are independent, and
// the only sequential part is a scalar triangular solve (one shuffle and one
// FMA per token).  The buffer costs (j-1) W4 4 bytes of reads and (j-1) 4 bytes of
// writes per head and step, against j (dk + dv) q/k/v bytes of buffered tokens.
//
// The Gram buffer is [B][H][W][W4] fp32 (W4 = W rounded up to a multiple of 4, so that
// every row starts on a 16-byte boundary): row u holds G_ut for t < u.
// One warp per head (4 per CTA, heads in (h, b) order); lane t holds token t
// (W <= 32).  The head's buffered rows and Gram rows land in shared memory by
// 16-byte cp.async; the sketch read c = R q~, o = P c + o_buf follows decode_step.cu.
#include "decode_common.cuh"

namespace skssm {

constexpr int WY_WARPS = 4;

// Reduce-scatter of 32 per-lane partials: afterwards lane t holds the warp total of x[t].
__device__ __forceinline__ float warp_reduce_scatter32(float (&x)[32], int lane) {
#pragma unroll
    for (int half = 16; half >= 1; half >>= 1) {
        const bool up = lane & half;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = up ? x[i] : x[i + half];
            const float keep = up ? x[i + half] : x[i];
            x[i] = keep + __shfl_xor_sync(FULL, send, half);
        }
    }
    return x[0];
}

template <int KIND, int DK, int DV, typename QT>
__global__ void __launch_bounds__(WY_WARPS * 32)
decode_wy_kernel(const float *__restrict__ P, const float *__restrict__ R, const QT *__restrict__ qv,
                 const QT *__restrict__ kbuf, const QT *__restrict__ vbuf, const float *__restrict__ abuf,
                 const float *__restrict__ bbuf, float *__restrict__ Gbuf, float *__restrict__ o, int B, int H,
                 int r, int j, int W) {
    using SL = DecSlots<KIND, DK, DV, QT>;
    constexpr int KPL = DK / 32, VPL = DV / 32;
    extern __shared__ __align__(16) char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NH = B * H;
    const int oi = blockIdx.x * WY_WARPS + warp;
    if (oi >= NH) return;  // the whole warp
    const int h = oi / B;
    const int head = (oi % B) * H + h;
    const int W4 = (W + 3) & ~3;  // Gram row stride: rows start on 16-byte boundaries
    const int gbytes = (j - 1) * W4 * 4;
    char *wb = smem + (size_t)warp * (j * (SL::KB + SL::VB + SL::AB) + W * W4 * 4);
    char *ks = wb, *vs = ks + j * SL::KB, *as = vs + j * SL::VB, *gs = as + j * SL::AB;
    const float *Gs = reinterpret_cast<const float *>(gs);  // rows u < j-1: G[u][t]
    float *Gh = Gbuf + (size_t)head * W * W4;

    // 1. the head's buffered rows and Gram rows into shared memory; query, scalars, sketch rows
    const size_t row0 = (size_t)head * W;
    auto copy = [&](char *dst, const void *src, int bytes) {
        const char *sp = static_cast<const char *>(src);
        for (int i = lane * 16; i < bytes; i += 32 * 16)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dec_smem(dst + i)), "l"(sp + i)
                         : "memory");
    };
    copy(ks, kbuf + row0 * DK, j * SL::KB);
    copy(vs, vbuf + row0 * DV, j * SL::VB);
    if (KIND == KDA) copy(as, abuf + row0 * DK, j * SL::AB);
    if (gbytes > 0) copy(gs, Gh, gbytes);
    asm volatile("cp.async.commit_group;\n" ::: "memory");

    float q[KPL];
    load_n<KPL>(qv + (size_t)head * DK + lane * KPL, q);
    const float a_l = (KIND != KDA && lane < j) ? abuf[row0 + lane] : 1.f;
    const float b_l = lane < j ? bbuf[row0 + lane] : 0.f;
    float pp[VPL][DEC_RPRE];
    const float *Ph = P + (size_t)head * DV * r;
#pragma unroll
    for (int e = 0; e < VPL; ++e) {
        const float *row = Ph + (size_t)(lane * VPL + e) * r;
        if ((r & 3) == 0 && r >= DEC_RPRE) {
            const float4 x = *reinterpret_cast<const float4 *>(row), y = *reinterpret_cast<const float4 *>(row + 4);
            pp[e][0] = x.x; pp[e][1] = x.y; pp[e][2] = x.z; pp[e][3] = x.w;
            pp[e][4] = y.x; pp[e][5] = y.y; pp[e][6] = y.z; pp[e][7] = y.w;
        } else {
#pragma unroll
            for (int m = 0; m < DEC_RPRE; ++m) pp[e][m] = m < r ? row[m] : 0.f;
        }
    }
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncwarp();

    // scalar decay: D_t and E_t as products over lanes (lane t: token t)
    float Dl = 1.f, El = 1.f, Dall = 1.f;
    if (KIND != KDA) {
        float incl = a_l;  // a_t ... a_{j-1}
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_down_sync(FULL, incl, off);
            if (lane + off < 32) incl *= y;
        }
        Dall = __shfl_sync(FULL, incl, 0);
        Dl = __shfl_down_sync(FULL, incl, 1);  // a_{t+1} ... a_{j-1}
        if (lane == 31) Dl = 1.f;
        El = a_l;  // a_0 ... a_t
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(FULL, El, off);
            if (lane >= off) El *= y;
        }
    }

    // 2. partial dots of every buffered token with q (. D_t) and with the newest key (. D_t)
    float xp[32], xg[32];
    float kn[KPL], D[KPL];
    load_n<KPL>(reinterpret_cast<const QT *>(ks + (j - 1) * SL::KB) + lane * KPL, kn);
#pragma unroll
    for (int e = 0; e < KPL; ++e) D[e] = 1.f;
#pragma unroll
    for (int tt = 31; tt >= 0; --tt) {
        xp[tt] = 0.f;
        xg[tt] = 0.f;
        if (tt < j) {  // warp-uniform
            float kf[KPL];
            load_n<KPL>(reinterpret_cast<const QT *>(ks + tt * SL::KB) + lane * KPL, kf);
#pragma unroll
            for (int e = 0; e < KPL; ++e) {
                const float kd = KIND == KDA ? kf[e] * D[e] : kf[e];
                xp[tt] = fmaf(kd, q[e], xp[tt]);
                xg[tt] = fmaf(kd, kn[e], xg[tt]);
            }
            if (KIND == KDA) {  // D_{t-1} = D_t (.) a_t
                float a[KPL];
                load_n<KPL>(reinterpret_cast<const float *>(as + tt * SL::AB) + lane * KPL, a);
#pragma unroll
                for (int e = 0; e < KPL; ++e) D[e] *= a[e];
            }
        }
    }
    float p_l = warp_reduce_scatter32(xp, lane);   // lane t: p_t (scalar decay: before D_t)
    float gn_l = warp_reduce_scatter32(xg, lane);  // lane t: G[j-1][t]
    if (KIND != KDA) {
        p_l *= Dl;
        gn_l *= Dl;
    }
    if (lane < j - 1) Gh[(size_t)(j - 1) * W4 + lane] = gn_l;  // the new column, for the window's later steps

    // 3. the triangular solve, newest token first: lane t keeps its running p_t - sum G s
    float acc = p_l, s_l = 0.f;
    for (int u = j - 1; u >= 0; --u) {
        const float su = __shfl_sync(FULL, b_l * acc, u);
        if (lane == u) s_l = su;
        const float g = u == j - 1 ? gn_l : (lane < u ? Gs[u * W4 + lane] : 0.f);
        if (lane < u) acc = fmaf(-g, su, acc);
    }

    // 4. o_buf = sum_u s_u v_u;  q~ = D_{-1} (.) q - sum_u s_u k_u (.) E_u
    float ob[VPL], w[KPL];
#pragma unroll
    for (int e = 0; e < VPL; ++e) ob[e] = 0.f;
    if (KIND == KDA) {
#pragma unroll
        for (int e = 0; e < KPL; ++e) w[e] = D[e] * q[e];  // D is now D_{-1}
    } else {
#pragma unroll
        for (int e = 0; e < KPL; ++e) w[e] = Dall * q[e];
    }
    float E[KPL];
#pragma unroll
    for (int e = 0; e < KPL; ++e) E[e] = 1.f;
    const float sE_l = KIND == KDA ? s_l : s_l * El;
    for (int u = 0; u < j; ++u) {
        const float su = __shfl_sync(FULL, s_l, u);
        const float cu = __shfl_sync(FULL, sE_l, u);
        float vf[VPL], kf[KPL];
        load_n<VPL>(reinterpret_cast<const QT *>(vs + u * SL::VB) + lane * VPL, vf);
        load_n<KPL>(reinterpret_cast<const QT *>(ks + u * SL::KB) + lane * KPL, kf);
#pragma unroll
        for (int e = 0; e < VPL; ++e) ob[e] = fmaf(su, vf[e], ob[e]);
        if (KIND == KDA) {
            float a[KPL];
            load_n<KPL>(reinterpret_cast<const float *>(as + u * SL::AB) + lane * KPL, a);
#pragma unroll
            for (int e = 0; e < KPL; ++e) {
                E[e] *= a[e];
                w[e] = fmaf(-su * E[e], kf[e], w[e]);
            }
        } else {
#pragma unroll
            for (int e = 0; e < KPL; ++e) w[e] = fmaf(-cu, kf[e], w[e]);
        }
    }

    // 5. c = R q~ and o = P c + o_buf, as the sketch decode step
    const float *Rh = R + (size_t)h * r * DK;
    float out[VPL];
#pragma unroll
    for (int e = 0; e < VPL; ++e) out[e] = ob[e];
#pragma unroll 1
    for (int m0 = 0; m0 < r; m0 += DEC_RPRE) {
        float c[DEC_RPRE];
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
                for (int e = 0; e < VPL; ++e) out[e] = fmaf(pp[e][mm], c[mm], out[e]);
        } else {
            sketch_block<VPL>(Ph, r, m0, r, c, out, lane);
        }
    }
    float *oh = o + (size_t)head * DV + lane * VPL;
    if constexpr (VPL == 4) *reinterpret_cast<float4 *>(oh) = make_float4(out[0], out[1], out[2], out[3]);
    else *reinterpret_cast<float2 *>(oh) = make_float2(out[0], out[1]);
}

int launch_decode_wy(const sketchssm_dims &d, const float *P, const float *R, const void *q, const void *k,
                     const void *v, const float *alpha, const float *beta, int j, float *G, float *o,
                     cudaStream_t stream) {
    if (d.kind == SKSSM_MAMBA2)  // no delta chain: the sketch decode step as it is
        return launch_decode_step(d, P, R, q, k, v, alpha, beta, j, nullptr, 0, nullptr, o, stream);
    return dispatch(d, [&](auto K, auto D, auto *, auto *qp) -> int {
        using QT = std::remove_pointer_t<decltype(qp)>;
        constexpr int KIND = decltype(K)::value, DK = decltype(D)::value;
        if constexpr (KIND == MAMBA2) {
            return SKSSM_ERR_DIMS;
        } else {
            const int NH = d.B * d.H;
            const int grid = (NH + WY_WARPS - 1) / WY_WARPS;
            auto go = [&](auto DVc) -> int {
                constexpr int DV = decltype(DVc)::value;
                using SL = DecSlots<KIND, DK, DV, QT>;
                const size_t smem =
                    (size_t)WY_WARPS * (j * (SL::KB + SL::VB + SL::AB) + (size_t)d.W * ((d.W + 3) & ~3) * 4);
                if (smem > 227 * 1024) return SKSSM_ERR_DIMS;
                auto kern = decode_wy_kernel<KIND, DK, DV, QT>;
                if (allow_max_smem(reinterpret_cast<const void *>(kern)) != SKSSM_OK) return SKSSM_ERR_CUDA;
                kern<<<grid, WY_WARPS * 32, smem, stream>>>(P, R, static_cast<const QT *>(q),
                                                             static_cast<const QT *>(k), static_cast<const QT *>(v),
                                                             alpha, beta, G, o, d.B, d.H, d.r, j, d.W);
                return launch_status();
            };
            if (d.dv == 64) return go(std::integral_constant<int, 64>());
            if (d.dv == 128) return go(std::integral_constant<int, 128>());
            return SKSSM_ERR_DIMS;
        }
    });
}

}  // namespace skssm

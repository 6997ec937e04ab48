// update_window.cu -- the once-per-window full-state update with fused sketch refresh.
//
// SketchSSM (arXiv 2609.33051v1), Abstract: at each state update the full state
// is read once and the outputs of the offline basis vectors are precomputed
// into a compact sketch; agihunt digest, bullet "Error control": the window's
// state update and the sketch refresh happen in the same kernel.
//
// One CTA per head (b, h), dv/32 warps, each warp owning 32 value columns of S
// (state_tile.cuh layout, 8 columns per lane).  The CTA loads the head's state
// straight into registers with 16-byte streaming loads, stages the window's
// tokens once in shared memory (converted to fp32, per-token scalars folded
// in), applies the n tokens in order from registers, stores the state once and
// writes P = S^T U from the same registers (basis rows staged in shared memory).
// Several CTAs share an SM: while one applies its tokens, the others' state
// loads are in flight.
//
// Scalar decay (Mamba-2, GDN) is folded into a running scale: S_t = g_t S^_t
// with g_t = a_1 ... a_t, so a token costs one dot product and one rank-1
// update per element:
//   Mamba-2  S^ += k (v / g_t)
//   GDN      d = k . S^;  S^ += k (b_t v / g_t - b_t d)
// KDA folds its per-channel decay the same way with g_{t,i} = prod a_{s,i}:
//   d = (k (.) g_t) . S^;  S^ += (b_t k / g_t) (v - d)
// and the stored state is S = g (.) S^ (scalar g for Mamba-2 and GDN).
#include "internal.h"
#include "state_tile.cuh"

namespace skssm {

constexpr int UPD_NC = 8;  // value columns per lane (state_tile.cuh)

// Inclusive prefix product across the warp.
__device__ __forceinline__ float warp_prefix_product(float x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x *= y;
    }
    return x;
}

// Rows t < n of a token array (row t of this head at src + t * row_stride + off, `len` elements of T) into fp32 shared memory
// dst[t * len + i], each multiplied by scale[t] when scale is given.  Every
// thread issues up to four 16-byte loads before it converts any of them.
template <typename T>
__device__ __forceinline__ void stage_rows(const T *__restrict__ src, size_t row_stride, size_t off, int len,
                                           int n, float *__restrict__ dst, const float *scale, int tid,
                                           int nthr) {
    constexpr int V = Vec<T>::N;
    const int per_row = len / V, total = n * per_row;
    for (int base = tid; base < total; base += 4 * nthr) {
        typename Vec<T>::type raw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int idx = base + u * nthr;
            if (idx < total) {
                const int t = idx / per_row, c = (idx - t * per_row) * V;
                raw[u] = *reinterpret_cast<const typename Vec<T>::type *>(src + (size_t)t * row_stride + off + c);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int idx = base + u * nthr;
            if (idx < total) {
                const int t = idx / per_row, c = (idx - t * per_row) * V;
                float f[V];
                unpack16<T>(raw[u], f);
                const float sc = scale ? scale[t] : 1.f;
#pragma unroll
                for (int e = 0; e < V; e += 4)
                    *reinterpret_cast<float4 *>(dst + t * len + c + e) =
                        make_float4(f[e] * sc, f[e + 1] * sc, f[e + 2] * sc, f[e + 3] * sc);
            }
        }
    }
}

template <int KIND, int DK, typename ST, typename QT, int NC>
__global__ void __launch_bounds__(256)
update_window_kernel(ST *__restrict__ S, float *__restrict__ P, const float *__restrict__ U,
                     const QT *__restrict__ kbuf, const QT *__restrict__ vbuf,
                     const float *__restrict__ abuf, const float *__restrict__ bbuf, int B, int H,
                     int dv, int r, int n, int W) {
    using TL = TileLayout<DK, ST>;
    constexpr int EPL = TL::EPL;
    extern __shared__ __align__(16) float smem[];

    // heads in (h, b) order: neighbouring CTAs share their basis rows in L2
    const int h = blockIdx.x / B;
    const int head = (blockIdx.x % B) * H + h;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane & 7, g = lane >> 3;
    const int c0 = warp * 4 * NC + g * NC;
    const int cl = NC == 8 ? l : l >> 1;  // the column whose reduced values this lane holds
    const int nthr = blockDim.x;

    // shared memory, each array a multiple of 4 floats: dot vectors, update
    // vectors (KDA), values, final scale(s), per-token scalars
    float *sk = smem;                                      // [n][DK]
    float *su = sk + (size_t)n * DK;                       // [n][DK] (KDA)
    float *sv = su + (KIND == KDA ? (size_t)n * DK : 0);   // [n][dv]
    float *sg = sv + (size_t)n * dv;                       // [DK]
    float *sut = sg + DK;                                  // [r][DK]: the head's basis rows
    float *ss1 = sut + (size_t)r * DK;                     // [n4]: b_t / g_t (Mamba-2: 1 / g_t)
    float *ss2 = ss1 + ((n + 3) & ~3);                     // [n4]: b_t

    // 1. the state goes in flight first, straight into registers
    float s[NC][EPL];
    load_tile<DK, ST, NC>(S + (size_t)head * dv * DK, c0, l, s);

    // 2. the basis rows, per-token scalars, then the tokens in fp32 with the scalars folded in
    {
        const float4 *src = reinterpret_cast<const float4 *>(U + (size_t)h * r * DK);
        for (int i = tid; i < r * DK / 4; i += nthr) reinterpret_cast<float4 *>(sut)[i] = src[i];
    }
    if (KIND != KDA) {
        if (warp == 0) {
            // g_t = a_1 ... a_t by a warp prefix product (n <= 64: two tokens per lane)
            float a0 = 1.f, a1 = 1.f, b0 = 1.f, b1 = 1.f;
            if (lane < n) { a0 = abuf[(size_t)head * W + lane]; if (KIND == GDN) b0 = bbuf[(size_t)head * W + lane]; }
            if (lane + 32 < n) {
                a1 = abuf[(size_t)head * W + lane + 32];
                if (KIND == GDN) b1 = bbuf[(size_t)head * W + lane + 32];
            }
            const float p0 = warp_prefix_product(a0, lane);
            const float p1 = warp_prefix_product(a1, lane) * __shfl_sync(FULL, p0, 31);
            if (lane < n) { ss1[lane] = b0 / p0; ss2[lane] = b0; }
            if (lane + 32 < n) { ss1[lane + 32] = b1 / p1; ss2[lane + 32] = b1; }
            const float g_lo = __shfl_sync(FULL, p0, (n >= 1 && n <= 32) ? n - 1 : 31);
            const float g_hi = __shfl_sync(FULL, p1, n > 32 ? n - 33 : 0);
            if (lane == 0) sg[0] = n == 0 ? 1.f : (n <= 32 ? g_lo : g_hi);
        }
        stage_rows<QT>(kbuf, DK, (size_t)head * W * DK, DK, n, sk, nullptr, tid, nthr);
        __syncthreads();
        stage_rows<QT>(vbuf, dv, (size_t)head * W * dv, dv, n, sv, ss1, tid, nthr);
    } else {
        stage_rows<QT>(kbuf, DK, (size_t)head * W * DK, DK, n, sk, nullptr, tid, nthr);
        stage_rows<QT>(vbuf, dv, (size_t)head * W * dv, dv, n, sv, nullptr, tid, nthr);
        stage_rows<float>(abuf, DK, (size_t)head * W * DK, DK, n, su, nullptr, tid, nthr);
        for (int t = tid; t < n; t += nthr) ss2[t] = bbuf[(size_t)head * W + t];
        __syncthreads();
        // per key channel: g_{t,i} = a_{1,i} ... a_{t,i}; dot vector k g_t (over k),
        // update vector b k / g_t (over the decay it replaces)
        for (int i = tid; i < DK; i += nthr) {
            float gam = 1.f;
            for (int t = 0; t < n; ++t) {
                gam *= su[t * DK + i];
                const float k = sk[t * DK + i];
                sk[t * DK + i] = k * gam;
                su[t * DK + i] = ss2[t] * k * (1.f / gam);
            }
            sg[i] = gam;
        }
    }
    __syncthreads();

    // 3. the buffered tokens, in order
    for (int t = 0; t < n; ++t) {
        float kv[EPL];
        lane_channels_smem<DK, ST>(sk + t * DK, l, kv);
        if (KIND == MAMBA2) {
            float vv[NC];
#pragma unroll
            for (int c4 = 0; c4 < NC; c4 += 4) {
                const float4 a = *reinterpret_cast<const float4 *>(sv + t * dv + c0 + c4);
                vv[c4] = a.x; vv[c4 + 1] = a.y; vv[c4 + 2] = a.z; vv[c4 + 3] = a.w;
            }
#pragma unroll
            for (int cc = 0; cc < NC; ++cc) axpy<EPL>(s[cc], kv, vv[cc]);
        } else {
            float d[NC];
#pragma unroll
            for (int cc = 0; cc < NC; ++cc) d[cc] = dot<EPL>(kv, s[cc]);
            float dsum;
            if constexpr (NC == 8) dsum = octet_reduce_scatter(d, lane);
            else dsum = octet_reduce4(d, lane);
            const float vc = sv[t * dv + c0 + cl];
            const float u = KIND == GDN ? vc - ss2[t] * dsum : vc - dsum;
            float uu[NC];
            if constexpr (NC == 8) octet_all_gather(u, uu);
            else octet_all_gather4(u, uu);
            if (KIND == KDA) lane_channels_smem<DK, ST>(su + t * DK, l, kv);
#pragma unroll
            for (int cc = 0; cc < NC; ++cc) axpy<EPL>(s[cc], kv, uu[cc]);
        }
    }

    // 4. final scale, storage rounding, one store of the state
    if (KIND != KDA) {
        const float gam = sg[0];
#pragma unroll
        for (int cc = 0; cc < NC; ++cc)
#pragma unroll
            for (int e = 0; e < EPL; ++e) s[cc][e] = as_stored<ST>(s[cc][e] * gam);
    } else {
        float gv[EPL];
        lane_channels_smem<DK, ST>(sg, l, gv);
#pragma unroll
        for (int cc = 0; cc < NC; ++cc)
#pragma unroll
            for (int e = 0; e < EPL; ++e) s[cc][e] = as_stored<ST>(s[cc][e] * gv[e]);
    }
    if (n > 0) store_tile<DK, ST, NC>(S + (size_t)head * dv * DK, c0, l, s);

    // 5. sketch refresh P[c][m] = sum_i S[i][c] U[i][m] from the stored values: per
    //    basis row m one dot per column and one octet reduction, after which lane
    //    l holds P[c0 + cl][m]; four basis rows per pass bound the rows in flight
    float *Prow = P + ((size_t)head * dv + c0 + cl) * r;
    const bool writer = NC == 8 || (l & 1) == 0;
#pragma unroll 1
    for (int m0 = 0; m0 < r; m0 += 4) {
        float pm[4];
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {
            pm[mm] = 0.f;
            if (m0 + mm < r) {
                float uv[EPL];
                lane_channels_smem<DK, ST>(sut + (m0 + mm) * DK, l, uv);
                float d[NC];
#pragma unroll
                for (int cc = 0; cc < NC; ++cc) d[cc] = dot<EPL>(uv, s[cc]);
                if constexpr (NC == 8) pm[mm] = octet_reduce_scatter(d, lane);
                else pm[mm] = octet_reduce4(d, lane);
            }
        }
        if (writer) {
            if ((r & 3) == 0) {
                *reinterpret_cast<float4 *>(Prow + m0) = make_float4(pm[0], pm[1], pm[2], pm[3]);
            } else {
#pragma unroll
                for (int mm = 0; mm < 4; ++mm)
                    if (m0 + mm < r) Prow[m0 + mm] = pm[mm];
            }
        }
    }
}

static size_t update_smem_bytes(const sketchssm_dims &d, int n) {
    const size_t n4 = (n + 3) & ~3;
    const size_t fl = (size_t)n * d.dk * (d.kind == SKSSM_KDA ? 2 : 1) + (size_t)n * d.dv + d.dk +
                      (size_t)d.r * d.dk + 2 * n4;
    return fl * sizeof(float);
}

int launch_update_window(const sketchssm_dims &d, void *S, float *P, const float *U, const void *k,
                         const void *v, const float *alpha, const float *beta, int n,
                         cudaStream_t stream) {
    const size_t smem = update_smem_bytes(d, n);
    if (smem > 227 * 1024) return SKSSM_ERR_DIMS;
    return dispatch(d, [&](auto K, auto D, auto *sp, auto *qp) -> int {
        using ST = std::remove_pointer_t<decltype(sp)>;
        using QT = std::remove_pointer_t<decltype(qp)>;
        constexpr int KIND = decltype(K)::value, DK = decltype(D)::value;
        auto kern = update_window_kernel<KIND, DK, ST, QT, UPD_NC>;
        // Opt in to the largest dynamic shared memory once per instantiation, so
        // that later calls (for example inside a graph capture) make no attribute call.
        static bool opted_in = false;
        if (!opted_in) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
                cudaSuccess)
                return SKSSM_ERR_CUDA;
            opted_in = true;
        }
        const int NH = d.B * d.H;
        kern<<<NH, d.dv * 8 / UPD_NC, smem, stream>>>(static_cast<ST *>(S), P, U, static_cast<const QT *>(k),
                                                      static_cast<const QT *>(v), alpha, beta, d.B, d.H, d.dv,
                                                      d.r, n, d.W);
        return launch_status();
    });
}

}  // namespace skssm

// update_window.cu -- the once-per-window full-state update with fused sketch refresh.
//
// SketchSSM (arXiv 2609.33051v1), Abstract: at each state update the full state
// is read once and the outputs of the offline basis vectors are precomputed
// into a compact sketch; agihunt digest, bullet "Error control": the window's
// state update and the sketch refresh happen in the same kernel.
//
// One CTA per head (b, h), dv/32 warps, each warp owning 32 value columns of S
// (layout in state_tile.cuh).  The kernel reads the head's state once into
// registers, applies the n buffered tokens in order, stores S once and writes
// P = S^T U from the same registers.  HBM traffic per head: S read + S write +
// P write + the n buffered tokens + U (L2-resident, shared by all b).
//
// Scalar decay (Mamba-2, GDN) is folded into a running scale: S_t = g_t S^_t
// with g_t = a_1 ... a_t, so each token costs one dot product and one rank-1
// update per element:
//   Mamba-2  S^ += k (v / g_t)
//   GDN      d = k . S^;  S^ += k (b_t v / g_t - b_t d)
// KDA folds its per-channel decay the same way with g_{t,i} = prod a_{s,i}:
//   d = (k (.) g_t) . S^;  S^ += (b_t k / g_t) (v - d)
// and the stored state is S = g (.) S^ (scalar g for Mamba-2 and GDN).
#include "internal.h"
#include "state_tile.cuh"

namespace skssm {

// Rows [0, n) of a strided token array (row t at src + t*row_stride + off, `len`
// elements of T each) into fp32 shared memory dst[t*len + i].  Each thread
// issues up to four 16-byte loads before converting any of them.
template <typename T>
__device__ __forceinline__ void stage_rows(const T *__restrict__ src, size_t row_stride, size_t off, int len,
                                           int n, float *__restrict__ dst, int tid, int nthr) {
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
#pragma unroll
                for (int e = 0; e < V; e += 4)
                    *reinterpret_cast<float4 *>(dst + t * len + c + e) = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
            }
        }
    }
}

// U [DK][r] (global, fp32) -> U^T [r][DK] in shared memory.
__device__ __forceinline__ void stage_transposed(const float *__restrict__ Uh, int DK, int r,
                                                 float *__restrict__ sut, int tid, int nthr) {
    if ((r & 3) == 0) {
        const int r4 = r / 4, total = DK * r4;
        for (int idx = tid; idx < total; idx += nthr) {
            const int i = idx / r4, m = (idx - i * r4) * 4;
            const float4 a = *reinterpret_cast<const float4 *>(Uh + (size_t)i * r + m);
            sut[(m + 0) * DK + i] = a.x;
            sut[(m + 1) * DK + i] = a.y;
            sut[(m + 2) * DK + i] = a.z;
            sut[(m + 3) * DK + i] = a.w;
        }
    } else {
        for (int idx = tid; idx < DK * r; idx += nthr) {
            const int i = idx / r, m = idx - i * r;
            sut[m * DK + i] = Uh[idx];
        }
    }
}

// Inclusive prefix product across the warp.
__device__ __forceinline__ float warp_prefix_product(float x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x *= y;
    }
    return x;
}

template <int KIND, int DK, typename ST, typename QT>
__global__ void __launch_bounds__(128)
update_window_kernel(ST *__restrict__ S, float *__restrict__ P, const float *__restrict__ U,
                     const QT *__restrict__ kbuf, const QT *__restrict__ vbuf,
                     const float *__restrict__ abuf, const float *__restrict__ bbuf, int NH, int H,
                     int dv, int r, int n) {
    using TL = TileLayout<DK, ST>;
    constexpr int EPL = TL::EPL;
    extern __shared__ __align__(16) float smem[];

    const int head = blockIdx.x;
    const int h = head % H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane & 7, g = lane >> 3;
    const int c0 = warp * 32 + g * 8;
    const int nthr = blockDim.x;

    // shared memory (every array but the two scalar ones is a multiple of 4 floats,
    // so each starts 16-byte aligned): dot vectors, update vectors (KDA), values,
    // final per-channel scale, U^T, token scalars
    float *sk = smem;                                      // [n][DK]
    float *sku = sk + (size_t)n * DK;                      // [n][DK] (KDA)
    float *sv = sku + (KIND == KDA ? (size_t)n * DK : 0);  // [n][dv]
    float *sg = sv + (size_t)n * dv;                       // [DK]
    float *sut = sg + DK;                                  // [r][DK]
    float *ss1 = sut + (size_t)r * DK;                     // [n]
    float *ss2 = ss1 + n;                                  // [n]

    // 1. the state slice goes in flight first
    float s[8][EPL];
    const ST *Sh = S + (size_t)head * dv * DK;
    load_tile<DK, ST>(Sh, c0, l, s);

    // 2. stage the buffered tokens and U^T in shared memory: every thread issues
    //    all of its 16-byte loads before it converts and stores any of them
    stage_rows<QT>(kbuf, (size_t)NH * DK, (size_t)head * DK, DK, n, sk, tid, nthr);
    stage_rows<QT>(vbuf, (size_t)NH * dv, (size_t)head * dv, dv, n, sv, tid, nthr);
    if (KIND == KDA) stage_rows<float>(abuf, (size_t)NH * DK, (size_t)head * DK, DK, n, sku, tid, nthr);
    stage_transposed(U + (size_t)h * DK * r, DK, r, sut, tid, nthr);
    if (KIND != KDA && warp == 0) {
        // g_t = a_1 ... a_t by a warp prefix product (n <= 64: two tokens per lane)
        float a0 = 1.f, a1 = 1.f, b0 = 1.f, b1 = 1.f;
        if (lane < n) { a0 = abuf[(size_t)lane * NH + head]; if (KIND == GDN) b0 = bbuf[(size_t)lane * NH + head]; }
        if (lane + 32 < n) {
            a1 = abuf[(size_t)(lane + 32) * NH + head];
            if (KIND == GDN) b1 = bbuf[(size_t)(lane + 32) * NH + head];
        }
        const float p0 = warp_prefix_product(a0, lane);
        const float p1 = warp_prefix_product(a1, lane) * __shfl_sync(FULL, p0, 31);
        if (lane < n) { ss1[lane] = b0 / p0; ss2[lane] = b0; }
        if (lane + 32 < n) { ss1[lane + 32] = b1 / p1; ss2[lane + 32] = b1; }
        const float g_lo = __shfl_sync(FULL, p0, (n >= 1 && n <= 32) ? n - 1 : 31);
        const float g_hi = __shfl_sync(FULL, p1, n > 32 ? n - 33 : 0);
        if (lane == 0) sg[0] = n == 0 ? 1.f : (n <= 32 ? g_lo : g_hi);
    }
    if (KIND == KDA)
        for (int t = tid; t < n; t += nthr) ss2[t] = bbuf[(size_t)t * NH + head];
    __syncthreads();
    if (KIND == KDA) {
        // per key channel: g_{t,i} = a_{1,i} ... a_{t,i}; dot vector k g_t, update vector b k / g_t
        for (int i = tid; i < DK; i += nthr) {
            float gam = 1.f;
            for (int t = 0; t < n; ++t) {
                gam *= sku[t * DK + i];
                const float b = ss2[t];
                const float kr = sk[t * DK + i];
                sk[t * DK + i] = kr * gam;
                sku[t * DK + i] = b * kr * (1.f / gam);
            }
            sg[i] = gam;
        }
        __syncthreads();
    }

    // 3. the buffered tokens, in order
    for (int t = 0; t < n; ++t) {
        float kd[EPL];
        lane_channels_smem<DK, ST>(sk + t * DK, l, kd);
        if (KIND == MAMBA2) {
            const float s1 = ss1[t];
            const float4 va = *reinterpret_cast<const float4 *>(sv + t * dv + c0);
            const float4 vb = *reinterpret_cast<const float4 *>(sv + t * dv + c0 + 4);
            const float vv[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) axpy<EPL>(s[cc], kd, vv[cc] * s1);
        } else {
            float d[8];
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) d[cc] = dot<EPL>(kd, s[cc]);
            const float dsum = octet_reduce_scatter(d, lane);
            const float vc = sv[t * dv + c0 + l];
            const float u = KIND == GDN ? ss1[t] * vc - ss2[t] * dsum : vc - dsum;
            float uu[8];
            octet_all_gather(u, uu);
            if (KIND == KDA) lane_channels_smem<DK, ST>(sku + t * DK, l, kd);
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) axpy<EPL>(s[cc], kd, uu[cc]);
        }
    }

    // 4. final scale, storage rounding, one store of the state
    if (KIND != KDA) {
        const float gam = sg[0];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
#pragma unroll
            for (int e = 0; e < EPL; ++e) s[cc][e] = as_stored<ST>(s[cc][e] * gam);
    } else {
        float gv[EPL];
        lane_channels_smem<DK, ST>(sg, l, gv);
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
#pragma unroll
            for (int e = 0; e < EPL; ++e) s[cc][e] = as_stored<ST>(s[cc][e] * gv[e]);
    }
    if (n > 0) store_tile<DK, ST>(S + (size_t)head * dv * DK, c0, l, s);

    // 5. sketch refresh P[c][m] = sum_i S[i][c] U[i][m], from the stored values: for
    //    each m one dot per column and one reduce-scatter over the octet, after which
    //    lane l holds P[c0 + l][m]
    float *Prow = P + ((size_t)head * dv + c0 + l) * r;
    for (int m0 = 0; m0 < r; m0 += 8) {
        float pm[8];
#pragma unroll
        for (int mm = 0; mm < 8; ++mm) {
            pm[mm] = 0.f;
            if (m0 + mm < r) {
                float uv[EPL];
                lane_channels_smem<DK, ST>(sut + (m0 + mm) * DK, l, uv);
                float d[8];
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) d[cc] = dot<EPL>(uv, s[cc]);
                pm[mm] = octet_reduce_scatter(d, lane);
            }
        }
        if ((r & 3) == 0) {
            *reinterpret_cast<float4 *>(Prow + m0) = make_float4(pm[0], pm[1], pm[2], pm[3]);
            if (m0 + 4 < r) *reinterpret_cast<float4 *>(Prow + m0 + 4) = make_float4(pm[4], pm[5], pm[6], pm[7]);
        } else {
#pragma unroll
            for (int mm = 0; mm < 8; ++mm)
                if (m0 + mm < r) Prow[m0 + mm] = pm[mm];
        }
    }
}

static size_t update_smem_bytes(const sketchssm_dims &d, int n) {
    size_t fl = (size_t)n * d.dk * (d.kind == SKSSM_KDA ? 2 : 1) + (size_t)n * d.dv + 2 * (size_t)n +
                d.dk + (size_t)d.r * d.dk;
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
        auto kern = update_window_kernel<KIND, DK, ST, QT>;
        // Opt in to the largest dynamic shared memory once per instantiation, on the
        // first call that needs more than the default, so later calls (for example
        // inside a CUDA graph capture) make no attribute call.
        static bool opted_in = false;
        if (smem > 48 * 1024 && !opted_in) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
                cudaSuccess)
                return SKSSM_ERR_CUDA;
            opted_in = true;
        }
        const int NH = d.B * d.H;
        kern<<<NH, d.dv, smem, stream>>>(static_cast<ST *>(S), P, U, static_cast<const QT *>(k),
                                         static_cast<const QT *>(v), alpha, beta, NH, d.H, d.dv, d.r, n);
        return launch_status();
    });
}

}  // namespace skssm

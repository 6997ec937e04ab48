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
//
// The fold divides by g_t, so it holds only while every running product stays
// a normal fp32 number: a zero decay (a state reset), or a window whose decay
// product underflows (16 tokens at a = 1e-3, a KDA channel decaying at 1e-6),
// would turn 1/g_t into inf and the state into 0 * inf = NaN.  Each head checks
// its products first; if any g_t (any channel's, for KDA) leaves
// [FOLD_LO, FOLD_HI] or is not finite, that head takes the plain recurrence
// instead -- per token the state is multiplied by the token's decay, then the
// delta step runs with g = 1 -- which divides by nothing.  The decision is
// per head and uniform over the CTA; workload decays (a ~ 0.9) never leave
// the range, so the fast path is what runs there.
#include "internal.h"
#include "state_tile.cuh"

namespace skssm {

constexpr int UPD_NC = 8;  // value columns per lane (state_tile.cuh)

// Range of the running decay product g_t inside which the fold is used.  With
// |g_t| >= 2^-64 the folded values stay below 2^64 |b v| per token, far from
// fp32 overflow; a product outside the range (or NaN) selects the plain path.
constexpr float FOLD_LO = 0x1p-64f, FOLD_HI = 0x1p64f;
__device__ __forceinline__ bool fold_ok(float g) { return g >= FOLD_LO && g <= FOLD_HI; }

// bounded waits that gave up, and sequence indices out of range, in either update kernel
__device__ unsigned g_update_wait_giveups;
constexpr int PER_NC = 4;      // the same for the persistent kernel
constexpr int PER_STAGES = 1;  // shared-memory stages per persistent CTA: with one stage more CTAs fit on an
                               // SM, which hides the copies better than a deeper pipeline per CTA (measured)

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

// Rows of head index h's basis in use: rank[h], with a value outside 0..r counted as a
// device error and clamped (so that no row past r is ever read).
__device__ __forceinline__ int ranked_rows(const int *rank, int h, int r) {
    const int v = rank[h];
    if (v < 0 || v > r) {
        if (threadIdx.x == 0) atomicAdd(&g_update_wait_giveups, 1u);
        return v < 0 ? 0 : r;
    }
    return v;
}

// Steps shared by both window-update kernels, for one head whose state is in
// registers: apply the n staged tokens in order, scale, round to the storage
// type, store the state once, and refresh the sketch from the same registers.
//
// Staged per token t (fast path, the fold):  sk = k (KDA: k (.) g_t);
// sv = v b_t / g_t (GDN), v / g_t (Mamba-2), v (KDA); su = b_t k / g_t (KDA);
// ss2 = b_t; sg = g_n (KDA: per channel).  Plain path (slow): sk = k;
// sv = v b_t (GDN), v (Mamba-2, KDA); su = the decay row a_t (KDA); sa = a_t
// (Mamba-2, GDN); ss2 = b_t; sg = 1.
template <int KIND, int DK, typename ST, int NC, bool READ, bool SEQS>
__device__ __forceinline__ void apply_store_refresh(float (&s)[NC][DK / 8], const float *sk, const float *su,
                                                    const float *sv, const float *sg, const float *sut,
                                                    const float *ss2, const float *sa, const float *sq,
                                                    ST *__restrict__ S, float *__restrict__ P,
                                                    float *__restrict__ o, int head, int dv, int r, int r_used, int n,
                                                    bool slow, int c0, int l, int lane) {
    using TL = TileLayout<DK, ST>;
    constexpr int EPL = TL::EPL;
    const int cl = NC == 8 ? l : l >> 1;  // the column whose reduced values this lane holds
    // the buffered tokens, in order
    auto token = [&](int t, auto SLOWc) {
        constexpr bool SLOW = decltype(SLOWc)::value;
        if constexpr (SLOW) {  // the plain recurrence: the token's decay applied to the state itself
            if constexpr (KIND == KDA) {
                float av[EPL];
                lane_channels_smem<DK, ST>(su + t * DK, l, av);
#pragma unroll
                for (int cc = 0; cc < NC; ++cc)
#pragma unroll
                    for (int e = 0; e < EPL; ++e) s[cc][e] *= av[e];
            } else {
                const float at = sa[t];
#pragma unroll
                for (int cc = 0; cc < NC; ++cc)
#pragma unroll
                    for (int e = 0; e < EPL; ++e) s[cc][e] *= at;
            }
        }
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
        } else if constexpr (NC == 4) {
            // two independent column pairs, each reduced over the octet on its own (lanes
            // l < 4 end with the pair's first column, l >= 4 with its second), so that one
            // pair's shuffles overlap the other pair's FMAs, and, with two tokens unrolled,
            // the next token's dots
            const bool hi = lane & 4;
            float x[2];
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const float d0 = dot<EPL>(kv, s[2 * p]), d1 = dot<EPL>(kv, s[2 * p + 1]);
                float y = (hi ? d1 : d0) + __shfl_xor_sync(FULL, hi ? d0 : d1, 4);
                y += __shfl_xor_sync(FULL, y, 2);
                x[p] = y + __shfl_xor_sync(FULL, y, 1);
            }
            const float b2 = KIND == GDN ? ss2[t] : 1.f;
            float uA = sv[t * dv + c0 + hi] - b2 * x[0];
            float uB = sv[t * dv + c0 + 2 + hi] - b2 * x[1];
            if constexpr (KIND == KDA && SLOW) {  // b_t (v - x): b is not folded into the keys
                uA *= ss2[t];
                uB *= ss2[t];
            }
            float uu[4] = {__shfl_sync(FULL, uA, 0, 8), __shfl_sync(FULL, uA, 4, 8),
                           __shfl_sync(FULL, uB, 0, 8), __shfl_sync(FULL, uB, 4, 8)};
            if (KIND == KDA && !SLOW) lane_channels_smem<DK, ST>(su + t * DK, l, kv);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) axpy<EPL>(s[cc], kv, uu[cc]);
        } else {
            float d[NC];
#pragma unroll
            for (int cc = 0; cc < NC; ++cc) d[cc] = dot<EPL>(kv, s[cc]);
            const float dsum = octet_reduce_scatter(d, lane);
            const float vc = sv[t * dv + c0 + cl];
            float u = KIND == GDN ? vc - ss2[t] * dsum : vc - dsum;
            if constexpr (KIND == KDA && SLOW) u *= ss2[t];
            float uu[NC];
            octet_all_gather(u, uu);
            if (KIND == KDA && !SLOW) lane_channels_smem<DK, ST>(su + t * DK, l, kv);
#pragma unroll
            for (int cc = 0; cc < NC; ++cc) axpy<EPL>(s[cc], kv, uu[cc]);
        }
    };
    if (slow) {  // CTA-uniform
#pragma unroll 1
        for (int t = 0; t < n; ++t) token(t, std::true_type());
    } else if constexpr (KIND != MAMBA2 && NC == 4 && DK == 128 && !READ && !SEQS) {
        // (two tokens per iteration only where the registers allow it without spilling: the
        // plain update of dk = 128 heads)
#pragma unroll 2
        for (int t = 0; t < n; ++t) token(t, std::false_type());
    } else {
        for (int t = 0; t < n; ++t) token(t, std::false_type());
    }

    // final scale
    if (KIND != KDA) {
        const float gam = sg[0];
#pragma unroll
        for (int cc = 0; cc < NC; ++cc)
#pragma unroll
            for (int e = 0; e < EPL; ++e) s[cc][e] *= gam;
    } else {
        float gv[EPL];
        lane_channels_smem<DK, ST>(sg, l, gv);
#pragma unroll
        for (int cc = 0; cc < NC; ++cc)
#pragma unroll
            for (int e = 0; e < EPL; ++e) s[cc][e] *= gv[e];
    }
    // the exact read of the window's last step, o = S^T q, from the updated fp32 state (the
    // full-read step reads before storage rounding too)
    if constexpr (READ) {
        float qv[EPL];
        lane_channels_smem<DK, ST>(sq, l, qv);
        float d[NC];
#pragma unroll
        for (int cc = 0; cc < NC; ++cc) d[cc] = dot<EPL>(qv, s[cc]);
        float x;
        if constexpr (NC == 8) x = octet_reduce_scatter(d, lane);
        else x = octet_reduce4(d, lane);
        if (NC == 8 || (l & 1) == 0) o[(size_t)head * dv + c0 + cl] = x;
    }
    // storage rounding, one store of the state
#pragma unroll
    for (int cc = 0; cc < NC; ++cc)
#pragma unroll
        for (int e = 0; e < EPL; ++e) s[cc][e] = as_stored<ST>(s[cc][e]);
    if (n > 0) store_tile<DK, ST, NC>(S + (size_t)head * dv * DK, c0, l, s);

    // sketch refresh (skipped when P is NULL: a plain buffered state update)
    if (P == nullptr) return;
    // sketch refresh P[c][m] = sum_i S[i][c] U[i][m] from the stored values: per
    //    basis row m one dot per column and one octet reduction, after which lane
    //    l holds P[c0 + cl][m]; four basis rows per pass bound the rows in flight
    float *Prow = P + ((size_t)head * dv + c0 + cl) * r;
    const uint64_t keep = l2_evict_last_policy();  // the decode steps re-read P from L2
    const bool writer = NC == 8 || (l & 1) == 0;
#pragma unroll 1
    for (int m0 = 0; m0 < r; m0 += 4) {
        float pm[4];
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {
            pm[mm] = 0.f;
            if (m0 + mm < r_used) {  // rows past a head's rank (zero basis rows) are written as zero
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
                st_keep(Prow + m0, make_float4(pm[0], pm[1], pm[2], pm[3]), keep);
            } else {
#pragma unroll
                for (int mm = 0; mm < 4; ++mm)
                    if (m0 + mm < r) st_keep1(Prow + m0 + mm, pm[mm], keep);
            }
        }
    }
}

template <int KIND, int DK, typename ST, typename QT, int NC, bool READ, bool SEQS>
__global__ void __launch_bounds__(256)
update_window_kernel(ST *__restrict__ S, float *__restrict__ P, const float *__restrict__ U,
                     const QT *__restrict__ kbuf, const QT *__restrict__ vbuf,
                     const float *__restrict__ abuf, const float *__restrict__ bbuf,
                     const QT *__restrict__ qv, float *__restrict__ o, int B, int H,
                     int dv, int r, int n, int W, const int *__restrict__ seqs, int n_seqs) {
    using TL = TileLayout<DK, ST>;
    constexpr int EPL = TL::EPL;
    extern __shared__ __align__(16) float smem[];

    // heads in (h, b) order: neighbouring CTAs share their basis rows in L2; the call's sequences
    // are all B or the n_seqs listed in seqs (an index outside 0..B-1 is counted and skipped)
    const int NB = SEQS ? n_seqs : B;
    const int h = blockIdx.x / NB;
    const int b = SEQS ? seqs[blockIdx.x % NB] : blockIdx.x % NB;
    if (SEQS && (b < 0 || b >= B)) {
        if (threadIdx.x == 0) atomicAdd(&g_update_wait_giveups, 1u);
        return;  // the whole CTA
    }
    const int head = b * H + h;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane & 7, g = lane >> 3;
    const int c0 = warp * 4 * NC + g * NC;
    const int nthr = blockDim.x;

    // shared memory, each array a multiple of 4 floats: dot vectors, update
    // vectors (KDA), values, final scale(s), per-token scalars
    const int n4 = (n + 3) & ~3;
    float *sk = smem;                                      // [n][DK]
    float *su = sk + (size_t)n * DK;                       // [n][DK] (KDA)
    float *sv = su + (KIND == KDA ? (size_t)n * DK : 0);   // [n][dv]
    float *sg = sv + (size_t)n * dv;                       // [DK]
    float *sut = sg + DK;                                  // [r][DK]: the head's basis rows
    float *ss1 = sut + (size_t)r * DK;                     // [n4]: b_t / g_t (Mamba-2: 1 / g_t)
    float *ss2 = ss1 + n4;                                 // [n4]: b_t
    float *sa = ss2 + n4;                                  // [n4]: a_t (the plain path)
    int *sflag = reinterpret_cast<int *>(sa + n4);         // [4]: this head takes the plain path
    float *sq = sa + n4 + 4;                               // [DK]: the last step's query (when read)

    // 1. the state goes in flight first, straight into registers
    float s[NC][EPL];
    load_tile<DK, ST, NC>(S + (size_t)head * dv * DK, c0, l, s);

    // 2. the basis rows, per-token scalars, then the tokens in fp32 with the scalars folded in
    if (U != nullptr) {
        const float4 *src = reinterpret_cast<const float4 *>(U + (size_t)h * r * DK);
        for (int i = tid; i < r * DK / 4; i += nthr) reinterpret_cast<float4 *>(sut)[i] = src[i];
    }
    if constexpr (READ)
        for (int i = tid; i < DK; i += nthr) sq[i] = ld1(qv + (size_t)head * DK + i);
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
            // every g_t in range: the fold; otherwise the plain recurrence for this head
            const bool slow = !__all_sync(FULL, (lane >= n || fold_ok(p0)) && (lane + 32 >= n || fold_ok(p1)));
            if (lane < n) { ss1[lane] = slow ? b0 : b0 / p0; ss2[lane] = b0; sa[lane] = a0; }
            if (lane + 32 < n) { ss1[lane + 32] = slow ? b1 : b1 / p1; ss2[lane + 32] = b1; sa[lane + 32] = a1; }
            const float g_lo = __shfl_sync(FULL, p0, (n >= 1 && n <= 32) ? n - 1 : 31);
            const float g_hi = __shfl_sync(FULL, p1, n > 32 ? n - 33 : 0);
            if (lane == 0) {
                sg[0] = (n == 0 || slow) ? 1.f : (n <= 32 ? g_lo : g_hi);
                sflag[0] = slow;
            }
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
        // per key channel: g_{t,i} = a_{1,i} ... a_{t,i}, all in range for the fold
        bool bad = false;
        for (int i = tid; i < DK; i += nthr) {
            float gam = 1.f;
            for (int t = 0; t < n; ++t) {
                gam *= su[t * DK + i];
                bad |= !fold_ok(gam);
            }
        }
        if (__syncthreads_or(bad)) {  // the plain recurrence: raw keys and decay rows stay as staged
            for (int i = tid; i < DK; i += nthr) sg[i] = 1.f;
            if (tid == 0) sflag[0] = 1;
        } else {
            // dot vector k g_t (over k), update vector b k / g_t (over the decay it replaces)
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
            if (tid == 0) sflag[0] = 0;
        }
    }
    __syncthreads();

    apply_store_refresh<KIND, DK, ST, NC, READ, SEQS>(s, sk, su, sv, sg, sut, ss2, sa, sq, S, P, o, head, dv, r, r,
                                                      n, sflag[0] != 0, c0, l, lane);
}

// ---------------------------------------------------------------------------
// Persistent, pipelined variant.  A CTA owns a contiguous run of heads in
// (h, b) order.  Each head's state (one contiguous dv x dk block) and its window
// tokens (contiguous blocks of the head-major buffer) arrive by TMA bulk copies
// into one of NS shared-memory stages, signalled by that stage's mbarrier; while
// the CTA applies head i's tokens from registers, heads i+1 .. i+NS-1 are in
// flight.  A stage is refilled as soon as the CTA has moved its head into
// registers and fp32 staging.  Waits are bounded: a give-up is counted
// (sketchssm_device_error_count) and the CTA returns.
// ---------------------------------------------------------------------------

__host__ __device__ inline int up16(int x) { return (x + 15) & ~15; }

// Byte offsets of the persistent kernel's shared memory (host and device agree).
struct PerLayout {
    int stage_bytes, st, kr, vr, ar, qr;  // inside a stage: state, raw k, raw v, raw decay (KDA), raw query
    int stages;                           // first stage (NS stages follow, stage_bytes apart)
    int sk, su, sv, sg, sut, ss2, sa, sq, total;
};

__host__ __device__ inline PerLayout per_layout(int kind, int DK, int dv, int r, int n, int sbytes, int qbytes,
                                                int ns, bool read) {
    PerLayout L;
    int t = 0;
    L.st = t; t += up16(dv * DK * sbytes);
    L.kr = t; t += up16(n * DK * qbytes);
    L.vr = t; t += up16(n * dv * qbytes);
    L.ar = t; t += kind == KDA ? up16(n * DK * 4) : 0;
    L.qr = t; t += read ? up16(DK * qbytes) : 0;
    L.stage_bytes = t;
    int off = 16 * 2;  // two mbarriers, 16 bytes apart
    L.stages = off; off += ns * t;
    L.sk = off; off += up16(n * DK * 4);
    L.su = off; off += kind == KDA ? up16(n * DK * 4) : 0;
    L.sv = off; off += up16(n * dv * 4);
    L.sg = off; off += up16(DK * 4);
    L.sut = off; off += up16(r * DK * 4);
    L.ss2 = off; off += up16(n * 4);
    L.sa = off; off += kind == KDA ? 0 : up16(n * 4);
    L.sq = off; off += read ? up16(DK * 4) : 0;
    L.total = off;
    return L;
}

template <int KIND, int DK, typename ST, typename QT, int NC, bool READ, bool SEQS, bool RANKED>
__global__ void __launch_bounds__(256)
update_window_persistent(ST *__restrict__ S, float *__restrict__ P, const float *__restrict__ U,
                         const QT *__restrict__ kbuf, const QT *__restrict__ vbuf,
                         const float *__restrict__ abuf, const float *__restrict__ bbuf,
                         const QT *__restrict__ qv, float *__restrict__ o, int B, int H, int dv, int r, int n, int W,
                         int ns, const int *__restrict__ seqs, int n_seqs, const int *__restrict__ rank) {
    using TL = TileLayout<DK, ST>;
    constexpr int EPL = TL::EPL;
    extern __shared__ __align__(128) float psm_f[];
    char *smem = reinterpret_cast<char *>(psm_f);
    const PerLayout L = per_layout(KIND, DK, dv, r, n, sizeof(ST), sizeof(QT), ns, READ);
    // the call's sequences: all B, or the n_seqs listed in seqs (an index outside 0..B-1 is counted
    // as a device error and its heads are skipped); work item w = (h, i) in (h, i) order
    const int NB = SEQS ? n_seqs : B;
    const int NH = NB * H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane & 7, g = lane >> 3;
    const int c0 = warp * 4 * NC + g * NC;
    const int nthr = blockDim.x;

    const int per = (NH + gridDim.x - 1) / gridDim.x;
    const int w_begin = blockIdx.x * per;
    const int w_end = min(NH, w_begin + per);
    auto head_of = [&](int w) -> int {
        if constexpr (!SEQS) return (w % B) * H + w / B;
        const int b = seqs[w % NB];
        return (b >= 0 && b < B) ? b * H + w / NB : -1;
    };

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    float *sk = reinterpret_cast<float *>(smem + L.sk);
    float *su = reinterpret_cast<float *>(smem + L.su);
    float *sv = reinterpret_cast<float *>(smem + L.sv);
    float *sg = reinterpret_cast<float *>(smem + L.sg);
    float *sut = reinterpret_cast<float *>(smem + L.sut);
    float *ss2 = reinterpret_cast<float *>(smem + L.ss2);
    float *sa = reinterpret_cast<float *>(smem + L.sa);
    float *sq = reinterpret_cast<float *>(smem + L.sq);
    const int state_bytes = dv * DK * (int)sizeof(ST);
    const int kbytes = n * DK * (int)sizeof(QT), vbytes = n * dv * (int)sizeof(QT);
    const int abytes = KIND == KDA ? n * DK * 4 : 0;
    const int qbytes = READ ? DK * (int)sizeof(QT) : 0;

    auto issue = [&](int w, int stage) {  // one thread
        char *sb = smem + L.stages + stage * L.stage_bytes;
        const int head = head_of(w);
        uint64_t *bar = bars + 2 * stage;
        if (SEQS && head < 0) {  // nothing to copy: complete the stage's phase at once
            atomicAdd(&g_update_wait_giveups, 1u);
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
            return;
        }
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
                     "r"(state_bytes + kbytes + vbytes + abytes + qbytes)
                     : "memory");
        bulk_g2s(sb + L.st, S + (size_t)head * dv * DK, state_bytes, bar);
        if constexpr (READ) bulk_g2s(sb + L.qr, qv + (size_t)head * DK, qbytes, bar);
        if (n > 0) {
            bulk_g2s(sb + L.kr, kbuf + (size_t)head * W * DK, kbytes, bar);
            bulk_g2s(sb + L.vr, vbuf + (size_t)head * W * dv, vbytes, bar);
            if (KIND == KDA) bulk_g2s(sb + L.ar, abuf + (size_t)head * W * DK, abytes, bar);
        }
    };

    if (tid == 0) {
        for (int st = 0; st < ns; ++st)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(bars + 2 * st)) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    if (tid == 0)
        for (int st = 0; st < ns && w_begin + st < w_end; ++st) issue(w_begin + st, st);

    // per-token scalars of the current head: lanes t and t + 32 of every warp
    auto load_scalars = [&](int w, float &a0, float &a1, float &b0, float &b1) {
        a0 = a1 = b0 = b1 = 1.f;
        const int hd = head_of(w);
        if (SEQS && hd < 0) return;
        const size_t base = (size_t)hd * W;
        if (KIND != KDA) {
            if (lane < n) a0 = abuf[base + lane];
            if (lane + 32 < n) a1 = abuf[base + lane + 32];
        }
        if (KIND != MAMBA2) {
            if (lane < n) b0 = bbuf[base + lane];
            if (lane + 32 < n) b1 = bbuf[base + lane + 32];
        }
    };
    float a0, a1, b0, b1;
    if (w_begin < w_end) load_scalars(w_begin, a0, a1, b0, b1);

    int h_prev = -1;
    for (int w = w_begin, it = 0; w < w_end; ++w, ++it) {
        const int stage = it % ns;
        const int parity = (it / ns) & 1;
        const int head = head_of(w), h = w / NB;
        const char *sb = smem + L.stages + stage * L.stage_bytes;
        const bool landed = mbar_wait(bars + 2 * stage, parity);
        // one decision for the whole CTA; the barrier also orders the previous
        // head's reads of the fp32 staging before this head's writes
        if (__syncthreads_or(!landed)) {
            if (tid == 0) {  // count the give-up, then drain the copies still in flight (bounded)
                atomicAdd(&g_update_wait_giveups, 1u);
                for (int k2 = 0; k2 < ns && w + k2 < w_end; ++k2)
                    mbar_wait(bars + 2 * ((it + k2) % ns), ((it + k2) / ns) & 1);
            }
            __syncthreads();
            return;
        }

        // state to registers
        float s[NC][EPL];
        const ST *st = reinterpret_cast<const ST *>(sb + L.st);
#pragma unroll
        for (int cc = 0; cc < NC; ++cc)
#pragma unroll
            for (int q = 0; q < TL::NQ; ++q)
                load16<ST>(st + (size_t)(c0 + cc) * DK + TL::chan(l, q, 0), &s[cc][q * TL::VEC]);
        if (h != h_prev && U != nullptr) {
            const float4 *src = reinterpret_cast<const float4 *>(U + (size_t)h * r * DK);
            for (int i = tid; i < r * DK / 4; i += nthr) reinterpret_cast<float4 *>(sut)[i] = src[i];
            h_prev = h;
        }
        if constexpr (READ) {
            const QT *qr = reinterpret_cast<const QT *>(sb + L.qr);
            for (int i = tid; i < DK; i += nthr) sq[i] = ld1(qr + i);
        }
        const QT *kr = reinterpret_cast<const QT *>(sb + L.kr);
        const QT *vr = reinterpret_cast<const QT *>(sb + L.vr);
        bool slow = false;  // this head takes the plain recurrence (made CTA-uniform below)
        if (KIND != KDA) {
            // every warp forms g_t = a_1 ... a_t itself (prefix product over lanes t, t + 32)
            const float p0 = warp_prefix_product(a0, lane);
            const float p1 = warp_prefix_product(a1, lane) * __shfl_sync(FULL, p0, 31);
            slow = !__all_sync(FULL, (lane >= n || fold_ok(p0)) && (lane + 32 >= n || fold_ok(p1)));
            const float s_lo = slow ? b0 : b0 / p0, s_hi = slow ? b1 : b1 / p1;  // b_t / g_t (plain: b_t)
            if (warp == 0) {
                const float g_lo = __shfl_sync(FULL, p0, (n >= 1 && n <= 32) ? n - 1 : 31);
                const float g_hi = __shfl_sync(FULL, p1, n > 32 ? n - 33 : 0);
                if (lane == 0) sg[0] = (n == 0 || slow) ? 1.f : (n <= 32 ? g_lo : g_hi);
                if (KIND == GDN) {
                    if (lane < n) ss2[lane] = b0;
                    if (lane + 32 < n) ss2[lane + 32] = b1;
                }
                if (lane < n) sa[lane] = a0;
                if (lane + 32 < n) sa[lane + 32] = a1;
            }
            for (int idx = tid * 4; idx < n * DK; idx += nthr * 4) {
                float f[4];
                load4(kr + idx, f);
                *reinterpret_cast<float4 *>(sk + idx) = make_float4(f[0], f[1], f[2], f[3]);
            }
            const int vtot = n * dv;  // warp-uniform trips: every lane takes part in the shuffles
            for (int base = warp * 128; base < vtot; base += (nthr / 32) * 128) {
                const int idx = base + lane * 4;
                const int t = (idx < vtot ? idx : vtot - 4) / dv;
                const float slo = __shfl_sync(FULL, s_lo, t & 31), shi = __shfl_sync(FULL, s_hi, t & 31);
                if (idx < vtot) {
                    const float sc = t < 32 ? slo : shi;
                    float f[4];
                    load4(vr + idx, f);
                    *reinterpret_cast<float4 *>(sv + idx) = make_float4(f[0] * sc, f[1] * sc, f[2] * sc, f[3] * sc);
                }
            }
        } else {
            const float *ar = reinterpret_cast<const float *>(sb + L.ar);
            if (warp == 0) {
                if (lane < n) ss2[lane] = b0;
                if (lane + 32 < n) ss2[lane + 32] = b1;
            }
            for (int i = tid; i < DK; i += nthr) {
                float gam = 1.f;
                for (int t = 0; t < n; ++t) {
                    gam *= ar[t * DK + i];
                    slow |= !fold_ok(gam);
                    const float bt = __shfl_sync(__activemask(), t < 32 ? b0 : b1, t & 31);
                    const float k = ld1(kr + t * DK + i);
                    sk[t * DK + i] = k * gam;
                    su[t * DK + i] = bt * k * (1.f / gam);
                }
                sg[i] = gam;
            }
            for (int idx = tid * 4; idx < n * dv; idx += nthr * 4) {
                float f[4];
                load4(vr + idx, f);
                *reinterpret_cast<float4 *>(sv + idx) = make_float4(f[0], f[1], f[2], f[3]);
            }
        }
        if (w + 1 < w_end) load_scalars(w + 1, a0, a1, b0, b1);  // in flight behind this head
        // the fp32 staging is ready; one decision for the CTA
        slow = __syncthreads_or(slow);
        if (KIND == KDA && slow) {  // the plain recurrence: raw keys and decay rows, from the still-intact stage
            const float *ar = reinterpret_cast<const float *>(sb + L.ar);
            for (int idx = tid; idx < n * DK; idx += nthr) {
                sk[idx] = ld1(kr + idx);
                su[idx] = ar[idx];
            }
            for (int i = tid; i < DK; i += nthr) sg[i] = 1.f;
            __syncthreads();
        }
        if (tid == 0 && w + ns < w_end) issue(w + ns, stage);  // the stage is consumed

        if (!SEQS || head >= 0)  // CTA-uniform
            apply_store_refresh<KIND, DK, ST, NC, READ, SEQS>(s, sk, su, sv, sg, sut, ss2, sa, sq, S, P, o, head, dv,
                                                              r, RANKED ? ranked_rows(rank, h, r) : r, n, slow, c0,
                                                              l, lane);
    }
}

static size_t update_smem_bytes(const sketchssm_dims &d, int n) {
    const size_t n4 = (n + 3) & ~3;
    const size_t fl = (size_t)n * d.dk * (d.kind == SKSSM_KDA ? 2 : 1) + (size_t)n * d.dv + d.dk +
                      (size_t)d.r * d.dk + 3 * n4 + 4 + d.dk;
    return fl * sizeof(float);
}

int launch_update_window(const sketchssm_dims &d, void *S, float *P, const float *U, const void *k,
                         const void *v, const float *alpha, const float *beta, int n, const void *q, float *o,
                         const int *seqs, int n_seqs, int sm_share, const int *rank, cudaStream_t stream) {
    constexpr int LIMIT = 227 * 1024;
    return dispatch(d, [&](auto K, auto D, auto *sp, auto *qp) -> int {
        using ST = std::remove_pointer_t<decltype(sp)>;
        using QT = std::remove_pointer_t<decltype(qp)>;
        constexpr int KIND = decltype(K)::value, DK = decltype(D)::value;
        const int NH = (seqs != nullptr ? n_seqs : d.B) * d.H;
        if (NH == 0) return SKSSM_OK;
        // the fused exact read is a separate instantiation: its code, even untaken, costs the plain
        // update a few percent (measured)
        auto run = [&](auto READc, auto SEQSc, auto RANKEDc) -> int {
            constexpr bool READ = decltype(READc)::value, SEQS = decltype(SEQSc)::value;
            constexpr bool RANKED = decltype(RANKEDc)::value;
            // persistent kernel, state and tokens by bulk copies; one CTA per head if its layout does not fit
            const int ns = PER_STAGES;
            const PerLayout L = per_layout(KIND, DK, d.dv, d.r, n, sizeof(ST), sizeof(QT), ns, READ);
            if (L.total <= LIMIT) {
                auto kern = update_window_persistent<KIND, DK, ST, QT, PER_NC, READ, SEQS, RANKED>;
                const int threads = d.dv * 8 / PER_NC;
                if (allow_max_smem(reinterpret_cast<const void *>(kern)) != SKSSM_OK) return SKSSM_ERR_CUDA;
                int sms = 0, per_sm = 0;
                if (sm_count(&sms) != SKSSM_OK ||
                    blocks_per_sm(reinterpret_cast<const void *>(kern), threads, L.total, &per_sm) != SKSSM_OK)
                    return SKSSM_ERR_CUDA;
                if (per_sm >= 1) {
                    if (sm_share > 0 && sm_share < per_sm) per_sm = sm_share;  // leave room for another kernel
                    const int grid = NH < sms * per_sm ? NH : sms * per_sm;
                    kern<<<grid, threads, L.total, stream>>>(static_cast<ST *>(S), P, U, static_cast<const QT *>(k),
                                                             static_cast<const QT *>(v), alpha, beta,
                                                             static_cast<const QT *>(q), o, d.B, d.H, d.dv, d.r, n,
                                                             d.W, ns, seqs, n_seqs, rank);
                    return launch_status();
                }
            }
            // one CTA per head
            const int threads = d.dv * 8 / UPD_NC;
            const size_t smem = update_smem_bytes(d, n);
            if (smem > (size_t)LIMIT) return SKSSM_ERR_DIMS;
            auto kern = update_window_kernel<KIND, DK, ST, QT, UPD_NC, READ, SEQS>;
            if (allow_max_smem(reinterpret_cast<const void *>(kern)) != SKSSM_OK) return SKSSM_ERR_CUDA;
            kern<<<NH, threads, smem, stream>>>(static_cast<ST *>(S), P, U, static_cast<const QT *>(k),
                                                static_cast<const QT *>(v), alpha, beta, static_cast<const QT *>(q),
                                                o, d.B, d.H, d.dv, d.r, n, d.W, seqs, n_seqs);
            return launch_status();
        };
        using T = std::true_type;
        using F = std::false_type;
        if (rank != nullptr) return run(F(), F(), T());  // the ranked update: no read, all sequences
        if (seqs != nullptr) {
            if (q != nullptr) return run(T(), T(), F());
            return run(F(), T(), F());
        }
        if (q != nullptr) return run(T(), F(), F());
        return run(F(), F(), F());
    });
}

int update_wait_giveups(bool reset, unsigned *count) {
    unsigned tc = 0;
    if (read_counter(&g_update_wait_giveups, reset, count) != SKSSM_OK || update_tc_giveups(reset, &tc) != SKSSM_OK)
        return SKSSM_ERR_CUDA;
    *count += tc;
    return SKSSM_OK;
}

}  // namespace skssm

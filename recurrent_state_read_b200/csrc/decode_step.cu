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
// Three kernels, one warp per head each, heads in (h, b) order (a CTA's warps share R
// rows); the launcher takes the first that applies:
//  - decode_step_deep (r = 8, one step index for all heads, at least 8 resident warps):
//    persistent warps, the whole per-head working set staged by cp.async, two stages;
//  - decode_step_persistent (per-sequence steps, per-head ranks, other r; at least 12
//    resident warps): persistent warps, token rows staged by cp.async, sketch columns
//    and per-token scalars prefetched into registers one head ahead;
//  - decode_step_kernel (the rest: long windows, KDA's wide token rows): one head per
//    warp, the head's buffered rows by TMA bulk copies on a bounded mbarrier wait, in
//    chunks of up to 32 tokens, while the query, the per-token scalars and the first
//    eight sketch columns load into registers; R rows are read after the backward pass
//    from L1/L2 (64 registers: eight 4-warp CTAs per SM).
// All three run the same backward pass (decode_common.cuh): per token one warp
// reduction for k . w and one axpy; scalar decay is kept as a running scale next to the
// carried query (w = g w^), so Mamba-2's dots do not depend on each other and eight of
// them share one warp all-reduce.  A bounded wait that gives up is counted
// (sketchssm_device_error_count) and the warp returns.
#include "decode_common.cuh"

namespace skssm {

constexpr int DEC_WARPS = 4;  // one head per warp; small CTAs pack the SMs more tightly (measured)
constexpr int DEC_DEEP_STAGES = 2;       // shared-memory stages per warp of the deep-pipelined kernel (2 beat 3 and 4: more warps fit)
constexpr int DEC_DEEP_MIN_WARPS = 8;     // fewest resident warps per SM for it
constexpr int DEC_PERSIST_MIN_WARPS = 12;  // fewest resident warps per SM for the pipelined kernel (measured crossover)

__device__ unsigned g_device_error;



template <int KIND, int DK, int DV, typename QT>
__global__ void __launch_bounds__(DEC_WARPS * 32)
decode_step_kernel(const float *__restrict__ P, const float *__restrict__ R, const QT *__restrict__ qv,
                   const QT *__restrict__ kbuf, const QT *__restrict__ vbuf,
                   const float *__restrict__ abuf, const float *__restrict__ bbuf,
                   float *__restrict__ o, int B, int H, int r, int j, int W, int jc,
                   const int *__restrict__ jv) {
    using SL = DecSlots<KIND, DK, DV, QT>;
    constexpr int KPL = DK / 32, VPL = DV / 32;  // channels of the carried query / output per lane
    extern __shared__ __align__(16) char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NH = B * H;
    const int oi = blockIdx.x * DEC_WARPS + warp;
    if (oi >= NH) return;  // the whole warp
    const int h = oi / B;
    const int head = (oi % B) * H + h;
    if (jv != nullptr) {  // the step of this head's sequence within its own window
        j = jv[oi % B];
        if (j < 0 || j > W) {
            if (lane == 0) atomicAdd(&g_device_error, 1u);
            return;
        }
        if (j == 0) return;  // the sequence takes no sketch step now
    }
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
            bulk_g2s(ks, kbuf + row0 * DK, nt * SL::KB, bar);
            bulk_g2s(vs, vbuf + row0 * DV, nt * SL::VB, bar);
            if (KIND == KDA) bulk_g2s(as, abuf + row0 * DK, nt * SL::AB, bar);
        }
        if (!mbar_wait(bar, phase)) {
            if (lane == 0) atomicAdd(&g_device_error, 1u);
            mbar_wait(bar, phase);  // give the copies in flight a last bounded chance to land
            return;
        }
        phase ^= 1;
        backward_chunk<KIND, DK, DV, QT>(ks, vs, as, nt, a_l, b_l, w, ob, gsc, lane);
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
            sketch_block<VPL>(Ph, r, m0, r, c, acc, lane);
        }
    }
    float *oh = o + (size_t)head * DV + lane * VPL;
    if constexpr (VPL == 4) *reinterpret_cast<float4 *>(oh) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    else *reinterpret_cast<float2 *>(oh) = make_float2(acc[0], acc[1]);
}

// ---------------------------------------------------------------------------
// Persistent, pipelined decode step.  A warp owns a contiguous run of heads in
// (h, b) order and keeps two shared-memory stages: while it computes head i from
// one stage, head i+1's query row and its j buffered k, v (and KDA decay) rows
// (contiguous blocks) land in the other by 16-byte cp.async copies, one commit
// group per head, and head i+1's per-token scalars and first eight sketch columns
// are in flight into registers.  The sketch columns stay in registers because
// each lane reads whole sketch rows, which in shared memory would put every lane
// of a warp on the same bank.  The coefficient rows R of the warp's head index h
// stay in registers and are reloaded only when h changes.  The per-head
// arithmetic is that of the kernel above.  Fewer warps fit per SM than for that
// kernel (two stages, more registers), so the launcher takes this one only where
// at least DEC_PERSIST_MIN_WARPS stay resident.
// ---------------------------------------------------------------------------
// A warp copies `bytes` (a multiple of 16) from global to shared memory in 16-byte
// cp.async pieces (L2 only), lane-strided.
__device__ __forceinline__ void copy16(char *dst, const void *src, int bytes, int lane) {
    const char *s = static_cast<const char *>(src);
    for (int i = lane * 16; i < bytes; i += 32 * 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dec_smem(dst + i)), "l"(s + i) : "memory");
}

template <int KIND, int DK, int DV, typename QT>
struct DecStage {
    static constexpr int QB = DK * (int)sizeof(QT);
    using SL = DecSlots<KIND, DK, DV, QT>;
    __host__ __device__ static int tokens(int j) { return j * (SL::KB + SL::VB + SL::AB); }
    // query row, k rows, v rows, decay rows: each a multiple of 16 bytes
    __host__ __device__ static int bytes(int j) { return QB + tokens(j); }
};

template <int KIND, int DK, int DV, typename QT, bool JV, bool RANKED>
__global__ void __launch_bounds__(DEC_WARPS * 32)
decode_step_persistent(const float *__restrict__ P, const float *__restrict__ R, const QT *__restrict__ qv,
                       const QT *__restrict__ kbuf, const QT *__restrict__ vbuf,
                       const float *__restrict__ abuf, const float *__restrict__ bbuf,
                       float *__restrict__ o, int B, int H, int r, int j, int W, const int *__restrict__ jv,
                       const int *__restrict__ rank) {
    using SL = DecSlots<KIND, DK, DV, QT>;
    using STG = DecStage<KIND, DK, DV, QT>;
    constexpr int KPL = DK / 32, VPL = DV / 32;
    extern __shared__ __align__(16) char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NH = B * H;
    const int sbytes = STG::bytes(j);
    char *const stage0 = smem + (size_t)warp * 2 * sbytes;

    // this warp's run of heads (flat (h, b) order index i; head = b * H + h)
    const int GW = gridDim.x * DEC_WARPS;
    const int per = (NH + GW - 1) / GW;
    const int i0 = (blockIdx.x * DEC_WARPS + warp) * per;
    const int i1 = min(NH, i0 + per);
    if (i0 >= i1) return;  // the whole warp; the kernel has no CTA-wide barrier

    // every lane starts its share of the 16-byte copies of one head's jh tokens into stage s (one
    // commit group, empty when the head takes no step); stages are sized for j tokens, j >= jh
    auto issue = [&](int head, int jh, int s) {
        char *sb = stage0 + s * sbytes;
        char *qs = sb, *ks = qs + STG::QB, *vs = ks + j * SL::KB, *as = vs + j * SL::VB;
        if (jh > 0) {
            copy16(qs, qv + (size_t)head * DK, STG::QB, lane);
            copy16(ks, kbuf + (size_t)head * W * DK, jh * SL::KB, lane);
            copy16(vs, vbuf + (size_t)head * W * DV, jh * SL::VB, lane);
            if (KIND == KDA) copy16(as, abuf + (size_t)head * W * DK, jh * SL::AB, lane);
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    };
    // the step of sequence b within its own window (every head of the call when jv is NULL); an index
    // outside 0..j is counted as a device error and the head is skipped
    auto step_of = [&](int b) -> int {
        if constexpr (!JV) return j;
        const int jh = jv[b];
        if (jh < 0 || jh > j) {
            if (lane == 0) atomicAdd(&g_device_error, 1u);
            return 0;
        }
        return jh;
    };
    // every lane: the per-token scalars of one head (token t in lane t, j <= 32) and the first
    // DEC_RPRE sketch columns of the lane's value channels, into registers
    auto scalars = [&](int head, int jh, float &al, float &bl, float (&pp)[VPL][DEC_RPRE]) {
        al = (KIND != KDA && lane < jh) ? abuf[(size_t)head * W + lane] : 1.f;
        bl = (KIND != MAMBA2 && lane < jh) ? bbuf[(size_t)head * W + lane] : 1.f;
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
        }
    };

    int nh = i0 / B, nb = i0 - nh * B;  // the next head to issue
    int ch = nh, cb = nb;               // the head being computed
    float a_c, b_c, a_n = 1.f, b_n = 1.f, pp_c[VPL][DEC_RPRE], pp_n[VPL][DEC_RPRE];
    int j_c = step_of(nb);
    issue(nb * H + nh, JV ? j_c : j, 0);
    scalars(nb * H + nh, JV ? j_c : j, a_c, b_c, pp_c);
    if (++nb == B) { nb = 0; ++nh; }
    int j_n = JV && i0 + 1 < i1 ? step_of(nb) : 0;  // the step of the next head, one head ahead of its copies

    int h_rows = -1, rh = r;  // rh: the rank of head index h_rows (rows past it are zero)
    float rr[DEC_RPRE][KPL];
    for (int i = i0, it = 0; i < i1; ++i, ++it) {
        const int s = it & 1;
        const int head = cb * H + ch;
        const bool more = i + 1 < i1;
        int j_nn = 0;
        if (more) {
            issue(nb * H + nh, JV ? j_n : j, s ^ 1);
            scalars(nb * H + nh, JV ? j_n : j, a_n, b_n, pp_n);
            if (++nb == B) { nb = 0; ++nh; }
            if (JV && i + 2 < i1) j_nn = step_of(nb);
        }
        const float *Rh = R + (size_t)ch * r * DK;
        if (ch != h_rows) {  // warp-uniform
#pragma unroll
            for (int m = 0; m < DEC_RPRE; ++m) {
                if (m < r) load_n<KPL>(Rh + (size_t)m * DK + lane * KPL, rr[m]);
                else {
#pragma unroll
                    for (int e = 0; e < KPL; ++e) rr[m][e] = 0.f;
                }
            }
            h_rows = ch;
            if constexpr (RANKED) {  // a rank outside 0..r is counted and clamped: no row past r is read
                rh = rank[ch];
                if (rh < 0 || rh > r) {
                    if (lane == 0) atomicAdd(&g_device_error, 1u);
                    rh = rh < 0 ? 0 : r;
                }
            }
        }
        // this head's group has landed (the next head's may still be in flight); the warp
        // barrier makes every lane's copies visible to the whole warp
        if (more) asm volatile("cp.async.wait_group 1;\n" ::: "memory");
        else asm volatile("cp.async.wait_group 0;\n" ::: "memory");
        __syncwarp();
        const char *sb = stage0 + s * sbytes;
        const char *qs = sb, *ks = qs + STG::QB, *vs = ks + j * SL::KB, *as = vs + j * SL::VB;

        if (!JV || j_c > 0) {  // warp-uniform
            float acc[VPL];
            float w[KPL], ob[VPL];
            load_n<KPL>(reinterpret_cast<const QT *>(qs) + lane * KPL, w);
#pragma unroll
            for (int e = 0; e < VPL; ++e) ob[e] = 0.f;
            float gsc = 1.f;
            backward_chunk<KIND, DK, DV, QT>(ks, vs, as, JV ? j_c : j, a_c, b_c, w, ob, gsc, lane);
            if (KIND != KDA) {
#pragma unroll
                for (int e = 0; e < KPL; ++e) w[e] *= gsc;
            }

            // c = R q~ (eight rows per warp all-reduce; rows past the first eight from L1/L2),
            // o = P c + o_buf (the first eight sketch columns from registers, the rest from L1/L2)
            const float *Ph = P + (size_t)head * DV * r;
#pragma unroll
            for (int e = 0; e < VPL; ++e) acc[e] = ob[e];
#pragma unroll 1
            for (int m0 = 0; m0 < rh; m0 += DEC_RPRE) {
                float c[DEC_RPRE];
#pragma unroll
                for (int mm = 0; mm < DEC_RPRE; ++mm) {
                    c[mm] = 0.f;
                    if (m0 == 0) {
#pragma unroll
                        for (int e = 0; e < KPL; ++e) c[mm] = fmaf(rr[mm][e], w[e], c[mm]);
                    } else if (m0 + mm < rh) {
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
                        for (int e = 0; e < VPL; ++e) acc[e] = fmaf(pp_c[e][mm], c[mm], acc[e]);
                } else {
                    sketch_block<VPL>(Ph, r, m0, rh, c, acc, lane);
                }
            }
            float *oh = o + (size_t)head * DV + lane * VPL;
            if constexpr (VPL == 4) *reinterpret_cast<float4 *>(oh) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            else *reinterpret_cast<float2 *>(oh) = make_float2(acc[0], acc[1]);
        }

        __syncwarp();  // every lane is done with this stage before it is refilled
        a_c = a_n;
        b_c = b_n;
        j_c = j_n;
        j_n = j_nn;
#pragma unroll
        for (int e = 0; e < VPL; ++e)
#pragma unroll
            for (int m = 0; m < DEC_RPRE; ++m) pp_c[e][m] = pp_n[e][m];
        if (++cb == B) { cb = 0; ++ch; }
    }
}

// ---------------------------------------------------------------------------
// Deep-pipelined decode step (uniform step index, r = 8).  Everything a head needs arrives in one shared-memory
// stage by cp.async -- query row, sketch rows, buffered k, v (and KDA decay) rows,
// and the per-token scalars -- so a warp can keep NS - 1 heads in flight while it
// computes one, with no register double-buffering.  One commit group per head; the
// loop always commits exactly one group per iteration (empty past the warp's run),
// so `cp.async.wait_group NS-1` always means "the current head has landed".
//
// The sketch rows are read per lane (lane l: rows VPL l .. VPL l + VPL-1, NP = VPL r / 4
// sixteen-byte pieces).  Copied as they are, the lanes of a quarter-warp would hit the
// same banks (a row pitch of 32 or 64 bytes), so the copy rotates each lane's pieces:
// piece k of lane l goes to slot NP l + ((k + rot(l)) mod NP), rot(l) = l NP / 8 for
// NP < 8 and l otherwise, which puts the eight lanes of a quarter-warp on distinct
// 16-byte bank groups.
// ---------------------------------------------------------------------------
template <int KIND, int DK, int DV, typename QT>
struct DeepStage {
    using SL = DecSlots<KIND, DK, DV, QT>;
    static constexpr int QB = DK * (int)sizeof(QT);
    // dv = 64: a lane's two sketch rows (32 bytes) go straight to registers at the start of the
    // head, under the backward pass; dv = 128: its 64 bytes are staged (registers measured slower)
    static constexpr bool P_IN_REGS = DV == 64;
    __host__ __device__ static int pbytes(int r) { return P_IN_REGS ? 0 : DV * r * 4; }
    __host__ __device__ static int sbytes(int j) {  // per-token scalars: decay (not KDA), b (not Mamba-2)
        return ((KIND != KDA ? 1 : 0) + (KIND != MAMBA2 ? 1 : 0)) * ((j * 4 + 15) & ~15);
    }
    __host__ __device__ static int bytes(int r, int j) {
        return QB + pbytes(r) + j * (SL::KB + SL::VB + SL::AB) + sbytes(j);
    }
};

__device__ __forceinline__ void cp_async4(char *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dec_smem(dst)), "l"(src) : "memory");
}

template <int NS>
__device__ __forceinline__ void cp_async_wait_ns() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(NS - 1) : "memory");
}

template <int KIND, int DK, int DV, typename QT, int NS>
__global__ void __launch_bounds__(DEC_WARPS * 32)
decode_step_deep(const float *__restrict__ P, const float *__restrict__ R, const QT *__restrict__ qv,
                 const QT *__restrict__ kbuf, const QT *__restrict__ vbuf, const float *__restrict__ abuf,
                 const float *__restrict__ bbuf, float *__restrict__ o, int B, int H, int r, int j, int W) {
    using SL = DecSlots<KIND, DK, DV, QT>;
    using STG = DeepStage<KIND, DK, DV, QT>;
    constexpr int KPL = DK / 32, VPL = DV / 32;
    extern __shared__ __align__(16) char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NH = B * H;
    const int sbytes = STG::bytes(r, j);
    const int pbytes = STG::pbytes(r);
    constexpr int NP = VPL * 2;                         // sixteen-byte sketch pieces per lane (r = 8)
    const int rot = NP < 8 ? (lane * NP) >> 3 : lane;  // this lane's piece rotation
    char *const stage0 = smem + (size_t)warp * NS * sbytes;

    const int GW = gridDim.x * DEC_WARPS;
    const int per = (NH + GW - 1) / GW;
    const int i0 = (blockIdx.x * DEC_WARPS + warp) * per;
    const int i1 = min(NH, i0 + per);
    if (i0 >= i1) return;  // the whole warp; the kernel has no CTA-wide barrier

    // the head run in (h, b) order: the issue cursor (ih, ib) runs NS - 1 heads ahead
    int ih = i0 / B, ib = i0 - ih * B;
    auto issue = [&](int i, int s) {  // one commit group, empty when i is past the run
        if (i < i1) {
            const int head = ib * H + ih;
            char *sb = stage0 + s * sbytes;
            char *qs = sb, *ps = qs + STG::QB, *ks = ps + pbytes, *vs = ks + j * SL::KB, *as = vs + j * SL::VB;
            char *sc = as + j * SL::AB;
            copy16(qs, qv + (size_t)head * DK, STG::QB, lane);
            if (!STG::P_IN_REGS) {  // sketch rows, each lane's pieces rotated (see above)
                const char *src = reinterpret_cast<const char *>(P + (size_t)head * DV * r);
                for (int pc = lane; pc < 32 * NP; pc += 32) {
                    const int l = pc / NP, k = pc - l * NP;  // source piece k of lane l's rows
                    const int rl = NP < 8 ? (l * NP) >> 3 : l;
                    const int slot = l * NP + (k + rl) % NP;
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dec_smem(ps + slot * 16)),
                                 "l"(src + pc * 16)
                                 : "memory");
                }
            }
            copy16(ks, kbuf + (size_t)head * W * DK, j * SL::KB, lane);
            copy16(vs, vbuf + (size_t)head * W * DV, j * SL::VB, lane);
            if (KIND == KDA) copy16(as, abuf + (size_t)head * W * DK, j * SL::AB, lane);
            if (lane < j) {
                const int sstride = (j * 4 + 15) & ~15;
                if (KIND != KDA) cp_async4(sc + lane * 4, abuf + (size_t)head * W + lane);
                if (KIND != MAMBA2) cp_async4(sc + (KIND != KDA ? sstride : 0) + lane * 4, bbuf + (size_t)head * W + lane);
            }
            if (++ib == B) { ib = 0; ++ih; }
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    };
#pragma unroll
    for (int s = 0; s < NS - 1; ++s) issue(i0 + s, s);

    int ch = i0 / B, cb = i0 - ch * B;  // the head being computed
    int h_rows = -1;
    float rr[DEC_RPRE][KPL];
    for (int i = i0, it = 0; i < i1; ++i, ++it) {
        issue(i + NS - 1, (it + NS - 1) % NS);
        const float *Rh = R + (size_t)ch * r * DK;
        if (ch != h_rows) {  // warp-uniform
#pragma unroll
            for (int m = 0; m < DEC_RPRE; ++m) {
                if (m < r) load_n<KPL>(Rh + (size_t)m * DK + lane * KPL, rr[m]);
                else {
#pragma unroll
                    for (int e = 0; e < KPL; ++e) rr[m][e] = 0.f;
                }
            }
            h_rows = ch;
        }
        cp_async_wait_ns<NS>();  // this head's group has landed (later heads may be in flight)
        __syncwarp();
        const char *sb = stage0 + (it % NS) * sbytes;
        const char *qs = sb, *ps = qs + STG::QB, *ks = ps + pbytes, *vs = ks + j * SL::KB, *as = vs + j * SL::VB;
        const float *sc = reinterpret_cast<const float *>(as + j * SL::AB);
        const int sstride = ((j * 4 + 15) & ~15) / 4;
        const float a_l = (KIND != KDA && lane < j) ? sc[lane] : 1.f;
        const float b_l = (KIND != MAMBA2 && lane < j) ? sc[(KIND != KDA ? sstride : 0) + lane] : 1.f;
        const int head = cb * H + ch;
        float4 pr[STG::P_IN_REGS ? NP : 1];
        if constexpr (STG::P_IN_REGS) {
            const float4 *pg = reinterpret_cast<const float4 *>(P + (size_t)head * DV * 8) + lane * NP;
#pragma unroll
            for (int k = 0; k < NP; ++k) pr[k] = pg[k];
        }

        float w[KPL], ob[VPL];
        load_n<KPL>(reinterpret_cast<const QT *>(qs) + lane * KPL, w);
#pragma unroll
        for (int e = 0; e < VPL; ++e) ob[e] = 0.f;
        float gsc = 1.f;
        backward_chunk<KIND, DK, DV, QT>(ks, vs, as, j, a_l, b_l, w, ob, gsc, lane);
        if (KIND != KDA) {
#pragma unroll
            for (int e = 0; e < KPL; ++e) w[e] *= gsc;
        }
        // c = R q~ (rows in registers), o = P c + o_buf with the lane's sketch rows from the stage
        float c[DEC_RPRE];
#pragma unroll
        for (int mm = 0; mm < DEC_RPRE; ++mm) {
            c[mm] = 0.f;
#pragma unroll
            for (int e = 0; e < KPL; ++e) c[mm] = fmaf(rr[mm][e], w[e], c[mm]);
        }
        warp_allreduce8(c, lane);
        float acc[VPL];
#pragma unroll
        for (int e = 0; e < VPL; ++e) acc[e] = ob[e];
        const float4 *pl = reinterpret_cast<const float4 *>(ps) + lane * NP;
#pragma unroll
        for (int k = 0; k < NP; ++k) {  // piece k: row VPL lane + k / 2, columns 4 (k mod 2) .. + 3
            const float4 pv = STG::P_IN_REGS ? pr[k] : pl[(k + rot) % NP];
            const int e = k / 2, m = 4 * (k % 2);
            acc[e] = fmaf(pv.x, c[m], acc[e]);
            acc[e] = fmaf(pv.y, c[m + 1], acc[e]);
            acc[e] = fmaf(pv.z, c[m + 2], acc[e]);
            acc[e] = fmaf(pv.w, c[m + 3], acc[e]);
        }
        float *oh = o + (size_t)head * DV + lane * VPL;
        if constexpr (VPL == 4) *reinterpret_cast<float4 *>(oh) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        else *reinterpret_cast<float2 *>(oh) = make_float2(acc[0], acc[1]);

        __syncwarp();  // every lane is done with this stage before it is refilled
        if (++cb == B) { cb = 0; ++ch; }
    }
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");  // the empty groups past the run
}

int launch_decode_step(const sketchssm_dims &d, const float *P, const float *R, const void *q,
                       const void *k, const void *v, const float *alpha, const float *beta, int j,
                       const int *jv, int sm_share, const int *rank, float *o, cudaStream_t stream) {
    if (jv != nullptr) j = d.W;  // per-sequence steps: size everything for the longest
    // the kernel does not touch the state: both state dtypes dispatch to the same instantiation
    return dispatch(d, [&](auto K, auto D, auto *, auto *qp) -> int {
        using QT = std::remove_pointer_t<decltype(qp)>;
        constexpr int KIND = decltype(K)::value, DK = decltype(D)::value;
        const int NH = d.B * d.H;
        const int grid = (NH + DEC_WARPS - 1) / DEC_WARPS;
        auto go = [&](auto DVc) -> int {
            constexpr int DV = decltype(DVc)::value;
            // the persistent pipelined kernel, when a warp's two stages leave enough warps per SM
            if (j <= 32 && d.r == 8 && jv == nullptr && rank == nullptr && sm_share == 0) {
                const size_t dsmem = (size_t)DEC_WARPS * DEC_DEEP_STAGES * DeepStage<KIND, DK, DV, QT>::bytes(8, j);
                if (dsmem <= 227 * 1024) {
                    auto dk = decode_step_deep<KIND, DK, DV, QT, DEC_DEEP_STAGES>;
                    if (allow_max_smem(reinterpret_cast<const void *>(dk)) != SKSSM_OK) return SKSSM_ERR_CUDA;
                    int sms = 0, per_sm = 0;
                    if (sm_count(&sms) != SKSSM_OK ||
                        blocks_per_sm(reinterpret_cast<const void *>(dk), DEC_WARPS * 32, dsmem, &per_sm) != SKSSM_OK)
                        return SKSSM_ERR_CUDA;
                    if (per_sm * DEC_WARPS >= DEC_DEEP_MIN_WARPS) {
                        const int dgrid = grid < sms * per_sm ? grid : sms * per_sm;
                        dk<<<dgrid, DEC_WARPS * 32, dsmem, stream>>>(P, R, static_cast<const QT *>(q),
                                                                     static_cast<const QT *>(k),
                                                                     static_cast<const QT *>(v), alpha, beta, o, d.B,
                                                                     d.H, d.r, j, d.W);
                        return launch_status();
                    }
                }
            }
            if (j <= 32) {
                const size_t psmem = (size_t)DEC_WARPS * 2 * DecStage<KIND, DK, DV, QT>::bytes(j);
                if (psmem <= 227 * 1024) {
                    // per-sequence steps are a separate instantiation: their checks cost the uniform
                    // step a few percent (measured)
                    auto persist = [&](auto JVc, auto RANKEDc) -> int {
                        auto pk = decode_step_persistent<KIND, DK, DV, QT, decltype(JVc)::value,
                                                         decltype(RANKEDc)::value>;
                        if (allow_max_smem(reinterpret_cast<const void *>(pk)) != SKSSM_OK) return SKSSM_ERR_CUDA;
                        int sms = 0, per_sm = 0;
                        if (sm_count(&sms) != SKSSM_OK ||
                            blocks_per_sm(reinterpret_cast<const void *>(pk), DEC_WARPS * 32, psmem, &per_sm) !=
                                SKSSM_OK)
                            return SKSSM_ERR_CUDA;
                        if (sm_share > 0 && sm_share < per_sm) per_sm = sm_share;  // leave room for another kernel
                        if (per_sm < 1 || (per_sm * DEC_WARPS < DEC_PERSIST_MIN_WARPS && sm_share == 0))
                            return 1;  // not taken: the one-head-per-warp kernel below
                        const int pgrid = grid < sms * per_sm ? grid : sms * per_sm;
                        pk<<<pgrid, DEC_WARPS * 32, psmem, stream>>>(
                            P, R, static_cast<const QT *>(q), static_cast<const QT *>(k), static_cast<const QT *>(v),
                            alpha, beta, o, d.B, d.H, d.r, j, d.W, jv, rank);
                        return launch_status();
                    };
                    using T = std::true_type;
                    using F = std::false_type;
                    const int rc = jv != nullptr ? persist(T(), F()) : rank != nullptr ? persist(F(), T()) : persist(F(), F());
                    if (rc != 1) return rc;
                }
            }
            // tokens per bulk round trip (<= 32: one per lane); KDA rows are twice as wide, and fewer
            // of them per trip keep more warps resident
            const int jmax = KIND == KDA ? 8 : 32;
            const int jc = j < jmax ? j : jmax;
            const size_t smem = (size_t)DEC_WARPS * DecSlots<KIND, DK, DV, QT>::bytes(jc);
            auto kern = decode_step_kernel<KIND, DK, DV, QT>;
            if (allow_max_smem(reinterpret_cast<const void *>(kern)) != SKSSM_OK) return SKSSM_ERR_CUDA;
            kern<<<grid, DEC_WARPS * 32, smem, stream>>>(P, R, static_cast<const QT *>(q),
                                                         static_cast<const QT *>(k), static_cast<const QT *>(v),
                                                         alpha, beta, o, d.B, d.H, d.r, j, d.W, jc, jv);
            return launch_status();
        };
        if (d.dv == 64) return go(std::integral_constant<int, 64>());
        if (d.dv == 128) return go(std::integral_constant<int, 128>());
        return SKSSM_ERR_DIMS;
    });
}

}  // namespace skssm

namespace skssm {
// The failure path every copy wait of the library shares, made to run: a bounded wait
// on an mbarrier that nothing arrives on gives up after `tries` polls, is counted,
// and the kernel returns, leaving the context usable.
__global__ void wait_giveup_probe(unsigned tries) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(&bar)) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncwarp();
    const bool landed = mbar_wait(&bar, 0, tries);
    if (!landed && threadIdx.x == 0) atomicAdd(&g_device_error, 1u);
}
}  // namespace skssm

extern "C" int sketchssm_selftest_wait_giveup(unsigned tries, void *stream) {
    if (tries == 0 || tries > (1u << 20)) return SKSSM_ERR_RANGE;
    skssm::wait_giveup_probe<<<1, 32, 0, (cudaStream_t)stream>>>(tries);
    return skssm::launch_status();
}

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

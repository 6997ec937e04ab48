// replay.cu -- the full-state read of a buffered window: ReplaySSM-style decode.
//
// SketchSSM (arXiv 2609.33051v1), Abstract, and the agihunt digest's "Background"
// bullet: ReplaySSM buffers the keys and values of a window and writes the state
// once per window, but every decode step still reads the full (unchanged)
// window-start state.  This kernel is that step:
//     o = S0^T q~ + o_buf,
// the same backward pass over the buffered tokens as the sketch decode step
// (decode_common.cuh), with the exact read of S0 in place of the sketch.  S is
// read, never written; the window update (without a sketch refresh) writes it
// once per window.  It is the second comparison point of the sketch path: it
// removes the full-read step's state write but keeps its state read.
//
// One CTA per head, dv threads, the register tile of state_tile.cuh (8 value
// columns per lane).  The state is requested first; while it streams in, the
// CTA copies the head's buffered token rows into shared memory (16-byte cp.async)
// and warp 0 then runs the backward pass; the other warps wait at the barrier
// with their state loads in flight.
#include "decode_common.cuh"

namespace skssm {

template <int KIND, int DK, int DV, typename ST, typename QT>
__global__ void __launch_bounds__(128)
replay_decode_kernel(const ST *__restrict__ S, const QT *__restrict__ qv, const QT *__restrict__ kbuf,
                     const QT *__restrict__ vbuf, const float *__restrict__ abuf, const float *__restrict__ bbuf,
                     float *__restrict__ o, int j, int W) {
    using TL = TileLayout<DK, ST>;
    using SL = DecSlots<KIND, DK, DV, QT>;
    constexpr int EPL = TL::EPL;
    constexpr int KPL = DK / 32, VPL = DV / 32;
    extern __shared__ __align__(16) char smem[];
    const int head = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = lane & 7, g = lane >> 3;
    const int c0 = warp * 32 + g * 8;
    const int nthr = blockDim.x;

    // 1. the state, straight into registers
    float s[8][EPL];
    load_tile<DK, ST>(S + (size_t)head * DV * DK, c0, l, s);

    // 2. the buffered rows into shared memory: k rows, v rows, (KDA) decay rows
    char *ks = smem + 16, *vs = ks + j * SL::KB, *as = vs + j * SL::VB;
    float *sq = reinterpret_cast<float *>(as + j * SL::AB);  // [DK]: q~
    float *sob = sq + DK;                                     // [DV]: o_buf
    auto copy = [&](char *dst, const void *src, int bytes) {
        const char *sp = static_cast<const char *>(src);
        for (int i = tid * 16; i < bytes; i += nthr * 16)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(
                             (unsigned)__cvta_generic_to_shared(dst + i)),
                         "l"(sp + i)
                         : "memory");
    };
    const size_t row0 = (size_t)head * W;
    copy(ks, kbuf + row0 * DK, j * SL::KB);
    copy(vs, vbuf + row0 * DV, j * SL::VB);
    if (KIND == KDA) copy(as, abuf + row0 * DK, j * SL::AB);
    asm volatile("cp.async.commit_group;\n" ::: "memory");

    float w[KPL], ob[VPL];
    if (warp == 0) load_n<KPL>(qv + (size_t)head * DK + lane * KPL, w);
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncthreads();

    // 3. warp 0: the backward pass, newest chunk of up to 32 tokens first
    if (warp == 0) {
#pragma unroll
        for (int e = 0; e < VPL; ++e) ob[e] = 0.f;
        float gsc = 1.f;
        for (int thi = j - 1; thi >= 0; thi -= 32) {
            const int tlo = thi - 31 > 0 ? thi - 31 : 0;
            const int nt = thi - tlo + 1;
            const float a_l = (KIND != KDA && lane < nt) ? abuf[row0 + tlo + lane] : 1.f;
            const float b_l = (KIND != MAMBA2 && lane < nt) ? bbuf[row0 + tlo + lane] : 1.f;
            backward_chunk<KIND, DK, DV, QT>(ks + tlo * SL::KB, vs + tlo * SL::VB, as + tlo * SL::AB, nt, a_l, b_l,
                                             w, ob, gsc, lane);
        }
#pragma unroll
        for (int e = 0; e < KPL; ++e) sq[lane * KPL + e] = KIND != KDA ? w[e] * gsc : w[e];
#pragma unroll
        for (int e = 0; e < VPL; ++e) sob[lane * VPL + e] = ob[e];
    }
    __syncthreads();

    // 4. o = S0^T q~ + o_buf: per column one dot and one octet reduction
    float qq[EPL];
    lane_channels_smem<DK, ST>(sq, l, qq);
    float d[8];
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) d[cc] = dot<EPL>(qq, s[cc]);
    const float y = octet_reduce_scatter(d, lane);  // column c0 + l
    o[(size_t)head * DV + c0 + l] = y + sob[c0 + l];
}

int launch_replay_decode(const sketchssm_dims &d, const void *S, const void *q, const void *k, const void *v,
                         const float *alpha, const float *beta, int j, float *o, cudaStream_t stream) {
    return dispatch(d, [&](auto K, auto D, auto *sp, auto *qp) -> int {
        using ST = std::remove_pointer_t<decltype(sp)>;
        using QT = std::remove_pointer_t<decltype(qp)>;
        constexpr int KIND = decltype(K)::value, DK = decltype(D)::value;
        const int NH = d.B * d.H;
        auto go = [&](auto DVc) -> int {
            constexpr int DV = decltype(DVc)::value;
            using SL = DecSlots<KIND, DK, DV, QT>;
            const size_t smem = 16 + (size_t)j * (SL::KB + SL::VB + SL::AB) + (DK + DV) * sizeof(float);
            auto kern = replay_decode_kernel<KIND, DK, DV, ST, QT>;
            if (allow_max_smem(reinterpret_cast<const void *>(kern)) != SKSSM_OK) return SKSSM_ERR_CUDA;
            kern<<<NH, DV, smem, stream>>>(static_cast<const ST *>(S), static_cast<const QT *>(q),
                                           static_cast<const QT *>(k), static_cast<const QT *>(v), alpha, beta, o,
                                           j, d.W);
            return launch_status();
        };
        if (d.dv == 64) return go(std::integral_constant<int, 64>());
        if (d.dv == 128) return go(std::integral_constant<int, 128>());
        return SKSSM_ERR_DIMS;
    });
}

}  // namespace skssm

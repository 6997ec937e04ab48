// state_tile.cuh -- register layout of a warp's slice of one head's state.
//
// The state is stored transposed, S_T[c][i] = S[i][c]: each value column c of
// S is one contiguous dk-vector.  All three recurrences, the exact read and the
// sketch refresh act on each column independently, and every reduction they
// need (k . S[:,c], q . S[:,c], U^T S[:,c]) runs along that contiguous vector.
//
// A warp owns 4 NC columns.  Lane = 8 g + l holds the NC columns c0 + cc
// (c0 = 4 NC warp + NC g, cc < NC; NC = 8 or 4) and, in each of them, the key channels
//     i = VEC (l + 8 q) + e,   q < NQ, e < VEC,
// where VEC elements fill one 16-byte vector of the storage type.  One warp-wide
// 16-byte load instruction therefore reads four 128-byte runs (one per lane
// octet), every byte of which is used.  A column's reductions are a per-lane
// partial over EPL = dk/8 channels followed by a reduction across the 8 lanes
// of an octet; with 8 columns per lane one octet reduce-scatter (7 shuffles)
// and all-gather (8 shuffles) serve 8 columns at a time, with 4 columns per
// lane 4 + 4 shuffles serve 4 (and half the registers hold the tile).
#pragma once

#include "common.cuh"

namespace skssm {

template <int DK, typename ST>
struct TileLayout {
    static constexpr int VEC = Vec<ST>::N;  // elements per 16-byte vector
    static constexpr int EPL = DK / 8;      // key channels held per lane and column
    static constexpr int NQ = EPL / VEC;    // 16-byte vectors per lane and column
    static_assert(NQ >= 1 && NQ * VEC == EPL, "unsupported dk for this storage type");
    __device__ static __forceinline__ int chan(int l, int q, int e) { return VEC * (l + 8 * q) + e; }
};

// Load the lane's EPL channels of a dk-vector held in shared memory (fp32).
template <int DK, typename ST>
__device__ __forceinline__ void lane_channels_smem(const float *x, int l, float (&out)[DK / 8]) {
    using TL = TileLayout<DK, ST>;
#pragma unroll
    for (int q = 0; q < TL::NQ; ++q)
#pragma unroll
        for (int e4 = 0; e4 < TL::VEC; e4 += 4) {
            float4 a = *reinterpret_cast<const float4 *>(x + TL::chan(l, q, e4));
            out[q * TL::VEC + e4 + 0] = a.x;
            out[q * TL::VEC + e4 + 1] = a.y;
            out[q * TL::VEC + e4 + 2] = a.z;
            out[q * TL::VEC + e4 + 3] = a.w;
        }
}

// Same from global memory in the q/k storage type QT.
template <int DK, typename ST, typename QT>
__device__ __forceinline__ void lane_channels_global(const QT *x, int l, float (&out)[DK / 8]) {
    using TL = TileLayout<DK, ST>;
#pragma unroll
    for (int q = 0; q < TL::NQ; ++q)
#pragma unroll
        for (int e4 = 0; e4 < TL::VEC; e4 += 4) load4(x + TL::chan(l, q, e4), out + q * TL::VEC + e4);
}

template <int DK, typename ST, int NC = 8>
__device__ __forceinline__ void load_tile(const ST *Sh, int c0, int l, float (&s)[NC][DK / 8]) {
    using TL = TileLayout<DK, ST>;
#pragma unroll
    for (int cc = 0; cc < NC; ++cc)
#pragma unroll
        for (int q = 0; q < TL::NQ; ++q)
            load16_stream<ST>(Sh + (size_t)(c0 + cc) * DK + TL::chan(l, q, 0), &s[cc][q * TL::VEC]);
}

template <int DK, typename ST, int NC = 8>
__device__ __forceinline__ void store_tile(ST *Sh, int c0, int l, const float (&s)[NC][DK / 8]) {
    using TL = TileLayout<DK, ST>;
#pragma unroll
    for (int cc = 0; cc < NC; ++cc)
#pragma unroll
        for (int q = 0; q < TL::NQ; ++q)
            store16_stream<ST>(Sh + (size_t)(c0 + cc) * DK + TL::chan(l, q, 0), &s[cc][q * TL::VEC]);
}

}  // namespace skssm

// common.cuh -- device helpers shared by the SketchSSM kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace skssm {

constexpr unsigned FULL = 0xffffffffu;
enum Kind { MAMBA2 = 0, GDN = 1, KDA = 2 };

// ---- storage <-> fp32 -------------------------------------------------------
template <typename T> struct Vec;  // 16-byte vector of T
template <> struct Vec<float> {
    static constexpr int N = 4;
    using type = float4;
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    using type = uint4;
};

__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// 16-byte load of N values of T, widened to fp32.
template <typename T>
__device__ __forceinline__ void load16(const T *p, float *out);
template <>
__device__ __forceinline__ void load16<float>(const float *p, float *out) {
    float4 a = *reinterpret_cast<const float4 *>(p);
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
}
template <>
__device__ __forceinline__ void load16<__nv_bfloat16>(const __nv_bfloat16 *p, float *out) {
    uint4 a = *reinterpret_cast<const uint4 *>(p);
    out[0] = bf16lo(a.x); out[1] = bf16hi(a.x); out[2] = bf16lo(a.y); out[3] = bf16hi(a.y);
    out[4] = bf16lo(a.z); out[5] = bf16hi(a.z); out[6] = bf16lo(a.w); out[7] = bf16hi(a.w);
}

// Streaming (evict-first) variants for the state, which is touched once per pass.
template <typename T>
__device__ __forceinline__ void load16_stream(const T *p, float *out);
template <>
__device__ __forceinline__ void load16_stream<float>(const float *p, float *out) {
    float4 a = __ldcs(reinterpret_cast<const float4 *>(p));
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
}
template <>
__device__ __forceinline__ void load16_stream<__nv_bfloat16>(const __nv_bfloat16 *p, float *out) {
    uint4 a = __ldcs(reinterpret_cast<const uint4 *>(p));
    out[0] = bf16lo(a.x); out[1] = bf16hi(a.x); out[2] = bf16lo(a.y); out[3] = bf16hi(a.y);
    out[4] = bf16lo(a.z); out[5] = bf16hi(a.z); out[6] = bf16lo(a.w); out[7] = bf16hi(a.w);
}

// Unpack one 16-byte vector of T to fp32.
template <typename T>
__device__ __forceinline__ void unpack16(const typename Vec<T>::type &a, float *out);
template <>
__device__ __forceinline__ void unpack16<float>(const float4 &a, float *out) {
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
}
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4 &a, float *out) {
    out[0] = bf16lo(a.x); out[1] = bf16hi(a.x); out[2] = bf16lo(a.y); out[3] = bf16hi(a.y);
    out[4] = bf16lo(a.z); out[5] = bf16hi(a.z); out[6] = bf16lo(a.w); out[7] = bf16hi(a.w);
}

// fp32 -> bf16 bits, round to nearest even (finite inputs; NaN kept quiet).
__device__ __forceinline__ uint32_t bf16_bits(float x) {
    uint32_t u = __float_as_uint(x);
    if ((u & 0x7f800000u) == 0x7f800000u) return (u >> 16) | ((u & 0x007fffffu) ? 0x40u : 0u);
    return (u + 0x7fffu + ((u >> 16) & 1u)) >> 16;
}
__device__ __forceinline__ float round_bf16(float x) { return __uint_as_float(bf16_bits(x) << 16); }

template <typename T>
__device__ __forceinline__ void store16_stream(T *p, const float *in);
template <>
__device__ __forceinline__ void store16_stream<float>(float *p, const float *in) {
    __stcs(reinterpret_cast<float4 *>(p), make_float4(in[0], in[1], in[2], in[3]));
}
template <>
__device__ __forceinline__ void store16_stream<__nv_bfloat16>(__nv_bfloat16 *p, const float *in) {
    uint4 a;
    a.x = bf16_bits(in[0]) | (bf16_bits(in[1]) << 16);
    a.y = bf16_bits(in[2]) | (bf16_bits(in[3]) << 16);
    a.z = bf16_bits(in[4]) | (bf16_bits(in[5]) << 16);
    a.w = bf16_bits(in[6]) | (bf16_bits(in[7]) << 16);
    __stcs(reinterpret_cast<uint4 *>(p), a);
}

// Value as stored: identity for fp32, bf16 round trip for bf16.
template <typename T> __device__ __forceinline__ float as_stored(float x);
template <> __device__ __forceinline__ float as_stored<float>(float x) { return x; }
template <> __device__ __forceinline__ float as_stored<__nv_bfloat16>(float x) { return round_bf16(x); }

// Scalar load of one element widened to fp32.
__device__ __forceinline__ float ld1(const float *p) { return *p; }
__device__ __forceinline__ float ld1(const __nv_bfloat16 *p) {
    return __uint_as_float(uint32_t(*reinterpret_cast<const uint16_t *>(p)) << 16);
}

// 8-byte load of 4 values (fp32: 16 B, bf16: 8 B) widened to fp32.
__device__ __forceinline__ void load4(const float *p, float *out) {
    float4 a = *reinterpret_cast<const float4 *>(p);
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float *out) {
    uint2 a = *reinterpret_cast<const uint2 *>(p);
    out[0] = bf16lo(a.x); out[1] = bf16hi(a.x); out[2] = bf16lo(a.y); out[3] = bf16hi(a.y);
}
// 2 values (fp32: 8 B, bf16: 4 B).
__device__ __forceinline__ void load2(const float *p, float *out) {
    float2 a = *reinterpret_cast<const float2 *>(p);
    out[0] = a.x; out[1] = a.y;
}
__device__ __forceinline__ void load2(const __nv_bfloat16 *p, float *out) {
    uint32_t a = *reinterpret_cast<const uint32_t *>(p);
    out[0] = bf16lo(a); out[1] = bf16hi(a);
}

// ---- packed fp32 arithmetic (sm_100 FFMA2) ----------------------------------
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// dot of n (even) values as two interleaved partial sums
template <int NE>
__device__ __forceinline__ float dot(const float *a, const float *b) {
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < NE; e += 2)
        acc = fma2(make_float2(a[e], a[e + 1]), make_float2(b[e], b[e + 1]), acc);
    return acc.x + acc.y;
}

// y[e] += a[e] * s   (s broadcast)
template <int NE>
__device__ __forceinline__ void axpy(float *y, const float *a, float s) {
    const float2 s2 = make_float2(s, s);
#pragma unroll
    for (int e = 0; e < NE; e += 2) {
        float2 r = fma2(make_float2(a[e], a[e + 1]), s2, make_float2(y[e], y[e + 1]));
        y[e] = r.x; y[e + 1] = r.y;
    }
}

// ---- warp reductions --------------------------------------------------------
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
    return x;
}

// Reduce-scatter of 8 values over the 8 lanes of an aligned lane octet: on
// entry lane l holds partials d[0..7]; on exit it returns the octet-wide sum of
// d[l & 7].  7 shuffles.
__device__ __forceinline__ float octet_reduce_scatter(const float (&d)[8], int lane) {
    const bool b2 = lane & 4, b1 = lane & 2, b0 = lane & 1;
    float a[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        float send = b2 ? d[m] : d[m + 4];
        float keep = b2 ? d[m + 4] : d[m];
        a[m] = keep + __shfl_xor_sync(FULL, send, 4);
    }
    float b[2];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        float send = b1 ? a[m] : a[m + 2];
        float keep = b1 ? a[m + 2] : a[m];
        b[m] = keep + __shfl_xor_sync(FULL, send, 2);
    }
    float send = b0 ? b[0] : b[1];
    float keep = b0 ? b[1] : b[0];
    return keep + __shfl_xor_sync(FULL, send, 1);
}

// All-gather within a lane octet: out[m] = value held by octet lane m.
__device__ __forceinline__ void octet_all_gather(float x, float (&out)[8]) {
#pragma unroll
    for (int m = 0; m < 8; ++m) out[m] = __shfl_sync(FULL, x, m, 8);
}

// Octet reduction of 4 values: on entry lane l holds partials d[0..3]; on exit
// lanes l and l^1 both hold the octet-wide sum of d[(l & 7) >> 1].  4 shuffles.
__device__ __forceinline__ float octet_reduce4(const float (&d)[4], int lane) {
    const bool b2 = lane & 4, b1 = lane & 2;
    float a[2];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        float send = b2 ? d[m] : d[m + 2];
        float keep = b2 ? d[m + 2] : d[m];
        a[m] = keep + __shfl_xor_sync(FULL, send, 4);
    }
    float send = b1 ? a[0] : a[1];
    float keep = b1 ? a[1] : a[0];
    float x = keep + __shfl_xor_sync(FULL, send, 2);
    return x + __shfl_xor_sync(FULL, x, 1);
}

// out[m] = value held by octet lanes 2m (and 2m+1) after octet_reduce4.
__device__ __forceinline__ void octet_all_gather4(float x, float (&out)[4]) {
#pragma unroll
    for (int m = 0; m < 4; ++m) out[m] = __shfl_sync(FULL, x, 2 * m, 8);
}

__device__ __forceinline__ float octet_sum(float x) {
    x += __shfl_xor_sync(FULL, x, 1);
    x += __shfl_xor_sync(FULL, x, 2);
    x += __shfl_xor_sync(FULL, x, 4);
    return x;
}

// ---- bounded mbarrier waits and bulk copies ---------------------------------
// Every wait of the library on a shared-memory mbarrier polls a bounded number
// of times; a wait that gives up returns false and the caller counts it
// (sketchssm_device_error_count) instead of hanging the GPU.
constexpr unsigned WAIT_TRIES = 1u << 22;

__device__ __forceinline__ unsigned smem_u32(const void *p) { return (unsigned)__cvta_generic_to_shared(p); }

__device__ __forceinline__ bool mbar_wait(const uint64_t *bar, int parity, unsigned tries = WAIT_TRIES) {
    for (unsigned it = 0; it < tries; ++it) {
        unsigned done;
        asm volatile(
            "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }\n"
            : "=r"(done)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// One bulk copy global -> shared memory (TMA, no multicast), completing on bar.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, int bytes, const uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// ---- L2 eviction priority hints ---------------------------------------------
// The sketch P is re-read by every decode step of a window: the window update
// writes it with an evict-last policy so that it stays in L2 while the state
// streams past (the decode steps read it with plain loads: an evict-last read
// measured slower on the Mamba-2 workload).
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void st_keep(float *p, float4 a, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(a.x), "f"(a.y),
                 "f"(a.z), "f"(a.w), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void st_keep1(float *p, float a, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(a), "l"(pol) : "memory");
}

// Reduce 8 per-lane partials over the whole warp; on return every lane holds all
// 8 totals.  A reduce-scatter over lane bits 4, 3, 2 (7 shuffles), an all-reduce
// over bits 1, 0 (2 shuffles), then an all-gather (8 shuffles).
__device__ __forceinline__ void warp_allreduce8(float (&v)[8], int lane) {
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    float a[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float send = b4 ? v[m] : v[m + 4];
        const float keep = b4 ? v[m + 4] : v[m];
        a[m] = keep + __shfl_xor_sync(FULL, send, 16);
    }
    float b[2];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const float send = b3 ? a[m] : a[m + 2];
        const float keep = b3 ? a[m + 2] : a[m];
        b[m] = keep + __shfl_xor_sync(FULL, send, 8);
    }
    float x = (b2 ? b[1] : b[0]) + __shfl_xor_sync(FULL, b2 ? b[0] : b[1], 4);
    x += __shfl_xor_sync(FULL, x, 2);
    x += __shfl_xor_sync(FULL, x, 1);
    // lane l now holds the total of index (l >> 2) & 7
#pragma unroll
    for (int m = 0; m < 8; ++m) v[m] = __shfl_sync(FULL, x, 4 * m);
}

}  // namespace skssm

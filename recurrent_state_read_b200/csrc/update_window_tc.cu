// update_window_tc.cu -- the delta-rule window update (Gated DeltaNet, KDA) on the tensor cores.
//
// SketchSSM (arXiv 2609.33051v1), Abstract: once per window the full state is
// read, the buffered tokens are applied exactly and the basis outputs are
// refreshed into the sketch; agihunt digest, bullet "Error control": the state
// update and the sketch refresh happen in the same kernel.
//
// The window's n tokens are applied in chunked (WY) form.  With tokens t = 0..n-1,
// decays a_t, strengths b_t, g_t = a_0 ... a_t and gamma_{t,s} = a_{s+1} ... a_t
// (products only; nothing is divided), the recurrence
//     S_t = a_t (I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T
// unrolls to S_t = g_t S_0 + sum_{s<=t} gamma_{t,s} k_s w_s^T, where the rows
// w_t (one value per value channel c) solve a unit lower-triangular system:
//     w_t = b_t v_t - b_t g_t x_t - sum_{s<t} b_t gamma_{t,s} (k_t . k_s) w_s,
//     x_t = S_0^T k_t.
// Per head (dk = dv = 128, S stored transposed, row c = column c of S):
//   1. [X | S_0^T U^T] = S_0^T [K; U]   tcgen05.mma kind::tf32, M = 128 (c), N = 16 + 2 RP,
//                                      K = 128 (i): one pass with the state as it
//                                      arrived, one with its TF32 remainder
//   2. the key Gram K K^T and K U^T    fp32 on the CUDA cores, under step 1
//   3. the triangular solve            CUDA cores, one value channel per thread
//   4. D^T = W~^T K, W~_s = gamma_{n-1,s} w_s
//                                      tcgen05.mma, M = 128, N = 128, K = n, W~ in
//                                      tensor memory (A), the keys MN-major (B)
//   5. S_n^T = g_{n-1} S_0^T + D^T, and the sketch
//          P = S_n^T U = g_{n-1} S_0^T U + sum_t W~_t (K U^T)_t
// fp32 accuracy from the TF32 tensor cores.  A TF32 operand keeps the top 11
// significant bits of an fp32 value: the tensor core drops the 13 low mantissa
// bits (measured: 1 + 0.75 ulp of TF32 enters as 1).  The state goes in as it
// arrived (the tensor core takes its TF32 part t(S_0)) and as its remainder
// S_0 - t(S_0), exact in fp32, of which the tensor core keeps the top 11 bits;
// Gated DeltaNet's keys are bf16, exact in TF32; the basis rows go in split as
// U = hi + lo with hi exactly TF32.  So
// every product of step 1 is off by less than 2^-21 of its terms.  W~ is split
// the same way for step 4.
//
// Data movement: a persistent CTA (one per SM) walks a contiguous run of heads in
// (h, b) order.  Each head's state arrives by four TMA tiled copies
// (cp.async.bulk.tensor, 128 rows x 32 fp32 each, 128-byte swizzle) into one of
// two shared-memory stages, which is the A operand of step 1's first pass, one
// head ahead.  Each thread keeps its 64 values of S_0 in registers from the split
// (step 1) to step 5 and writes the remainder into tensor memory, from where the
// second pass reads it (A operand in tensor memory).  Step 5 writes S_n back
// into the stage, from where it leaves by TMA tiled stores (a thread per row
// storing to global memory directly costs one transaction per row per store).
// The keys and values arrive by 1-D bulk copies one head ahead.  Roles: warp 0
// issues the MMAs, warp 1 the copies; warps 2, 3, 6 and 7 compute the key Gram and
// the system matrix A[t][s] = b_t gamma_{t,s} (k_t . k_s) under step 1 (off the
// issuers' sub-partitions), warps 1 and 5 K U^T (r <= 8; for r = 16 the Gram
// warps take it too); warps 0-3 (one value channel per thread) solve, while
// warp 4 builds the next head's decay products.  Tensor memory (512
// columns): the remainder (128), [X | S_0^T U] (<= 128), D (128), W~ hi | lo (32).
// KDA (decay per key channel i, S_t = (I - b_t k_t k_t^T) diag(a_t) S_{t-1} + b_t k_t v_t^T): the
// same steps with g_t, gamma_{t,s} per channel, x_t = S_0^T (g_t o k_t), A[t][s] = b_t
// sum_i gamma_{t,s,i} k_t,i k_s,i, W~ = w, the keys of step 4 gamma_{n-1,s} o k_s, the basis rows
// of step 1 g_{n-1} o U, and the store S_n = g_{n-1} o S_0 + D per key channel.  Those keys and
// rows are fp32, so they are split hi + lo too (step 4 takes a third pass: W~ hi against the keys'
// lo).  Per-channel prefix and suffix products are formed by one thread per channel.
// Every wait is bounded; a wait that gives up is counted
// (sketchssm_device_error_count), the CTA drains what it has in flight (bounded),
// frees its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "internal.h"
#include "common.cuh"

namespace skssm {

__device__ unsigned g_update_tc_giveups;

namespace {

constexpr int TC_THREADS = 256;  // 8 warps; warps w and w + 4 share tensor-memory lanes 32 (w % 4) ..
constexpr int TC_NS = 2;         // state stages
constexpr int TC_NPAD = 16;      // token rows of the operands (tokens n .. 15 are zero)
constexpr int TC_PANEL = 128 * 128;    // bytes of one 32-column panel of a head's state (128 rows x 128 B)
constexpr int TC_STATE = 4 * TC_PANEL;
constexpr uint32_t TM_COLS = 512;
constexpr uint32_t TM_LO = 0;    // the state's TF32 remainder, 128 columns (A of step 1's second pass)
constexpr uint32_t TM_D1 = 128;  // [X | S_0^T U hi-part | S_0^T U lo-part], N1 <= 48 columns
constexpr uint32_t TM_D2 = 256;  // the state increment D^T, 128 columns
constexpr uint32_t TM_W = 384;   // W~^T hi (16 columns) then lo (16): A of step 4
constexpr int TC_SMEM_LIMIT = 227 * 1024;

__host__ __device__ inline int round_up(int x, int a) { return (x + a - 1) / a * a; }
// rows of B1: key rows (16; KDA: 16 hi + 16 lo of the decayed keys), then U hi and U lo (rp each)
__host__ __device__ constexpr int tc_nk(bool kda) { return kda ? 2 * TC_NPAD : TC_NPAD; }
__host__ __device__ constexpr int tc_n1(int rp, bool kda) { return (tc_nk(kda) + 2 * rp + 15) / 16 * 16; }

// Shared-memory layout: byte offsets from the 1024-aligned base.
struct TcLayout {
    int stages;     // TC_NS x 64 KB: state stages (TMA destination; A of step 1's first pass)
    int b1;         // B of step 1: N1 rows [keys | U hi (RP) | U lo (RP) | 0] x 128 fp32, K-major,
                    // 128-byte swizzle, 4 panels of N1 rows x 128 B
    int kbm;        // the keys of step 4, MN-major TF32 layout: 4 panels x 16 rows x 128 B (KDA: the
                    // decayed keys, hi then lo)
    int tok;        // two token buffers: 16 key rows, 16 value rows (bf16), KDA: 16 decay rows (fp32)
    int tok_bytes;  // bytes of one token buffer
    int uf;         // KDA: the basis rows of the current head index, fp32 [RP][128]
    int gnv;        // KDA: the window's decay product per key channel, fp32 [128]
    int xo;         // the exact read's partial sums of the second column half, fp32 [128]
    int am;         // by head parity: A, decay table [2][16][20] each, K U^T [2][16][RP], b_t g_t,
                    // gamma_{n-1,t}, b_t [2][16] each, g [2]
    int bars;       // mbarriers: 2 stages, 2 token buffers, step 1, step 4, drain
    int slot;       // tensor-memory base address written by tcgen05.alloc
    int total;      // bytes to request (with slack for aligning the base)
};

__host__ __device__ inline TcLayout tc_layout(int rp, bool kda) {
    TcLayout L;
    const int n1 = tc_n1(rp, kda);
    int o = 0;
    L.stages = o; o += TC_NS * TC_STATE;
    L.b1 = o; o += round_up(n1 * 512, 1024);
    L.kbm = o; o += (kda ? 2 : 1) * TC_NPAD * 512;
    L.tok_bytes = 2 * TC_NPAD * 128 * 2 + (kda ? TC_NPAD * 128 * 4 : 0);
    L.tok = o; o += 2 * L.tok_bytes;
    L.uf = o; o += kda ? rp * 512 : 0;
    L.gnv = o; o += kda ? 512 : 0;
    L.xo = o; o += 512;
    L.am = o; o += round_up((4 * TC_NPAD * (TC_NPAD + 4) + 2 * TC_NPAD * rp + 6 * TC_NPAD + 4) * 4, 16);
    L.bars = o; o += 8 * (TC_NS + 5);
    L.slot = o; o += 16;
    L.total = o + 1024;
    return L;
}

// ---- PTX wrappers -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// TMA tiled load of one box (no multicast), completing on bar
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// TMA tiled store of one box from shared memory
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, int x, int y, const void *src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(smem_u32(src))
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem descriptor], kind::tf32, issued by one thread
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, int accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// arrive on bar once every tcgen05 operation this thread issued before has completed
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

#define TC_R8(a, i) "=r"(a[i]), "=r"(a[i + 1]), "=r"(a[i + 2]), "=r"(a[i + 3]), "=r"(a[i + 4]), "=r"(a[i + 5]), \
                    "=r"(a[i + 6]), "=r"(a[i + 7])
#define TC_W8(a, i) "r"(a[i]), "r"(a[i + 1]), "r"(a[i + 2]), "r"(a[i + 3]), "r"(a[i + 4]), "r"(a[i + 5]), \
                    "r"(a[i + 6]), "r"(a[i + 7])

// 32 consecutive columns of this warp's 32 lanes: thread l gets lane (base lane + l)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : TC_R8(v, 0), TC_R8(v, 8), TC_R8(v, 16), TC_R8(v, 24)
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : TC_R8(v, 0), TC_R8(v, 8)
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        TC_W8(v, 0), TC_W8(v, 8), TC_W8(v, 16), TC_W8(v, 24)
        : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16};" ::"r"(taddr),
        TC_W8(v, 0), TC_W8(v, 8)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// fp32 value with the 13 low mantissa bits cleared: exactly a TF32 value
__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xffffe000u); }
// The TF32 value the tensor core takes of an fp32 operand that is not already TF32 (the state
// stage): its 13 low mantissa bits dropped.
__device__ __forceinline__ float tc_tf32(float x) { return tf32_hi(x); }

// Shared-memory matrix descriptors.  K-major, 128-byte swizzle: atoms of 8 rows x 128 B, 1024 B
// apart (the leading offset is unused); a K step of 8 TF32 values advances the start by 32 B inside
// the atom.  MN-major TF32 takes the 128-byte swizzle with 32-byte atomicity (the only MN-major
// layout for 32-bit types): atoms of 4 K-rows x 128 B (32 MN-values), 512 B apart, 32-byte chunks
// permuted by the row; the leading offset is the distance between 32-value MN blocks.
__device__ __forceinline__ uint64_t smem_desc_kmajor_sw128(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3fff) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}
__device__ __forceinline__ uint64_t smem_desc_mnmajor_sw128_32b(uint32_t addr, uint32_t lbo_bytes) {
    return (uint64_t)((addr >> 4) & 0x3fff) | ((uint64_t)((lbo_bytes >> 4) & 0x3fff) << 16) |
           ((uint64_t)(512 >> 4) << 32) | (1ull << 46) | (1ull << 61);
}
// Instruction descriptor: kind::tf32, fp32 accumulator, A K-major, B K-major (b_mn = 0) or MN-major (1).
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, int b_mn) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// byte offset of element (row, col) in a panel of 128-byte rows (col < 32, fp32): 128-byte swizzle
// (16-byte chunks permuted by row mod 8), and 128-byte swizzle with 32-byte atomicity (32-byte
// chunks permuted by row mod 4)
__device__ __forceinline__ int sw128(int row, int col) {
    return row * 128 + ((((col >> 2) ^ row) & 7) << 4) + (col & 3) * 4;
}
__device__ __forceinline__ int sw128_32b(int row, int col) {
    return row * 128 + ((((col >> 3) ^ row) & 3) << 5) + (col & 7) * 4;
}

template <typename QT>
__device__ __forceinline__ float ldq(const unsigned char *p, int idx) {
    return ld1(reinterpret_cast<const QT *>(p) + idx);
}

// 8 consecutive columns of this warp's 32 lanes
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t *v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t *v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}
// D[tmem] (+)= A[smem descriptor] * B[smem descriptor], kind::tf32
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, int accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// one lane of a converged warp (the lowest): the issuer of the warp's single-thread operations
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .b32 r;\n\t.reg .pred p;\n\telect.sync r|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(pred));
    return pred != 0;
}

// Recursive-halving reduce-scatter of 32 per-lane partials: on return lane l holds in v[0] the sum
// over the warp of every lane's v[l] (31 shuffles).
__device__ __forceinline__ void warp_reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
            const float send = up ? v[i] : v[i + o];
            const float keep = up ? v[i + o] : v[i];
            v[i] = keep + __shfl_xor_sync(FULL, send, o);
        }
    }
}

// 4-wide fp32 dot product
__device__ __forceinline__ float dot4(float4 a, float4 b) {
    return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

template <int KIND, int RP, bool READ>
__global__ void __launch_bounds__(TC_THREADS, 1)
update_window_delta_tc(const __grid_constant__ CUtensorMap tmS, float *__restrict__ P,
                     const float *__restrict__ U, const __nv_bfloat16 *__restrict__ kbuf,
                     const __nv_bfloat16 *__restrict__ vbuf, const float *__restrict__ abuf,
                     const float *__restrict__ bbuf, const __nv_bfloat16 *__restrict__ qv,
                     float *__restrict__ o, int B, int H, int r, int n, int W) {
    using QT = __nv_bfloat16;
    constexpr bool KD = KIND == KDA;
    constexpr int NPAD = TC_NPAD, NK = tc_nk(KD), N1 = tc_n1(RP, KD), as = NPAD + 4;  // A, G rows: 16-B aligned
    constexpr int B1P = N1 * 128;  // bytes of one 32-column panel of B1
    extern __shared__ __align__(1024) unsigned char tc_raw[];
    unsigned char *sm = tc_raw + ((1024 - (smem_u32(tc_raw) & 1023)) & 1023);
    const TcLayout L = tc_layout(RP, KD);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quad = warp & 3, half = warp >> 2;
    const int row = 32 * quad + lane;  // this thread's state row (value channel) and tensor-memory lane
    const int NH = B * H;
    const int per = (NH + gridDim.x - 1) / gridDim.x;
    const int w_begin = blockIdx.x * per, w_end = min(NH, w_begin + per);
    if (w_begin >= w_end) return;  // the whole CTA, before anything is allocated

    uint64_t *bar_s = reinterpret_cast<uint64_t *>(sm + L.bars);  // [2] state stages
    uint64_t *bar_t = bar_s + TC_NS;                              // [2] key buffers
    uint64_t *bar_1 = bar_t + 2;                                  // step 1 complete
    uint64_t *bar_4 = bar_1 + 1;                                  // step 4 complete
    uint64_t *bar_d = bar_4 + 1;                                  // the drain after a give-up
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L.slot);
    // per head parity:
    // A[t][s] = b_t gamma_{t,s} G[t][s] (GDN) or b_t sum_i gamma_{t,s,i} k_t,i k_s,i (KDA), s < t; else 0
    float *Am = reinterpret_cast<float *>(sm + L.am);  // [2][16][as]
    float *Gam = Am + 2 * NPAD * as;                    // [2][16][as]: b_t gamma_{t,s} (KDA: b_t), s < t; else 0
    float *kus = Gam + 2 * NPAD * as;                   // [2][16][RP]: (K U^T)[t][m]
    float *ev = kus + 2 * NPAD * RP;                    // [2][16]: b_t g_t
    float *cv = ev + 2 * NPAD;                          // [2][16]: gamma_{n-1,s}
    float *bv = cv + 2 * NPAD;                          // [2][16]: b_t
    float *gn = bv + 2 * NPAD;                          // [2]:  g_{n-1}
    unsigned char *b1 = sm + L.b1, *kbm = sm + L.kbm;
    const uint32_t b1_a = smem_u32(b1), kbm_a = smem_u32(kbm);
    float *uf = reinterpret_cast<float *>(sm + L.uf);    // KDA: [RP][128] basis rows of the current h
    float *gnv = reinterpret_cast<float *>(sm + L.gnv);  // KDA: [128] the window's decay product g_{n-1}
    float *xo = reinterpret_cast<float *>(sm + L.xo);    // [128] the exact read, second column half
    const int kbytes = n * 128 * (int)sizeof(QT);
    constexpr int AOFF = 2 * NPAD * 128 * (int)sizeof(QT);  // KDA: decay rows after the keys and values

    auto head_of = [&](int w) { return (w % B) * H + w / B; };
    auto stage_of = [&](int st) { return sm + L.stages + st * TC_STATE; };
    auto tok_of = [&](int i) { return sm + L.tok + i * L.tok_bytes; };
    // single-thread issues (the elected lane of warp 1)
    auto issue_state = [&](int w, int st) {
        uint64_t *bar = bar_s + st;
        mbar_expect_tx(bar, TC_STATE);
        for (int p = 0; p < 4; ++p) tma_load_2d(stage_of(st) + p * TC_PANEL, &tmS, 32 * p, head_of(w) * 128, bar);
    };
    auto issue_tok = [&](int w, int i) {
        uint64_t *bar = bar_t + i;
        const size_t off = (size_t)head_of(w) * W * 128;
        mbar_expect_tx(bar, 2 * kbytes + (KD ? n * 512 : 0));
        bulk_g2s(tok_of(i), kbuf + off, kbytes, bar);
        bulk_g2s(tok_of(i) + NPAD * 128 * sizeof(QT), vbuf + off, kbytes, bar);
        if (KD) bulk_g2s(tok_of(i) + AOFF, abuf + off, n * 512, bar);
    };

    float a_nx = 1.f, b_nx = 0.f;  // warp 4, lane t: a_t and b_t of the next head to build a system for
    // warp 4: a head's decay table from its token scalars (lane t holds a_t, b_t; lanes >= n: a = 1, b = 0)
    auto decay_table = [&](float a_l, float b_l, int buf) {
        const float at = lane < n ? a_l : 1.f, bt = lane < n ? b_l : 0.f;
        float g = at;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(FULL, g, o);
            if (lane >= o) g *= y;
        }
        float sp = at;  // suffix products: sp_s = a_s ... a_31
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_down_sync(FULL, sp, o);
            if (lane + o < 32) sp *= y;
        }
        const float c = __shfl_down_sync(FULL, sp, 1);
        if (lane < NPAD) {
            ev[buf * NPAD + lane] = bt * g;
            bv[buf * NPAD + lane] = bt;
            cv[buf * NPAD + lane] = c;  // gamma_{n-1,s} = a_{s+1} ... a_{n-1} (a = 1 past n)
        }
        const float gl = __shfl_sync(FULL, g, n - 1);
        if (lane == 0) gn[buf] = gl;
        float *gm = Gam + buf * NPAD * as;
        float gam = 1.f;  // gamma_{t,s} for t = lane, s descending
#pragma unroll
        for (int s = NPAD - 1; s >= 0; --s) {
            const float a1 = __shfl_sync(FULL, at, s + 1);
            if (lane > s) gam *= a1;
            if (lane < NPAD) gm[lane * as + s] = lane > s && lane < n ? bt * gam : 0.f;
        }
    };

    // warps 2, 3, 6, 7 (not the sub-partitions of the MMA and copy issuers): this head's key Gram and
    // K U^T, and A = (b_t gamma_{t,s}) o G into buffer buf.  GDN: from the fp32 rows of B1 (keys, U hi
    // and lo).  KDA: from the token buffer tk (keys, per-channel decays) and the basis rows uf, with
    // the channel decays between the two tokens inside the dot.
    auto gram_system = [&](int buf, const unsigned char *tk) {
        const int t0 = 4 * ((warp & 1) + (warp >> 1 & 2));  // rows t0 .. t0 + 3
        if constexpr (KD) {
            const QT *kr = reinterpret_cast<const QT *>(tk);
            const float *ar = reinterpret_cast<const float *>(tk + AOFF);
            auto krow = [&](int t) {  // key channels 4 lane .. + 3 of token t (zero past n)
                float f[4] = {0.f, 0.f, 0.f, 0.f};
                if (t < n) load4(kr + t * 128 + 4 * lane, f);
                return make_float4(f[0], f[1], f[2], f[3]);
            };
            auto arow = [&](int t) { return *reinterpret_cast<const float4 *>(ar + t * 128 + 4 * lane); };
            auto mul4 = [](float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); };
            float4 ks[NPAD];
#pragma unroll
            for (int j = 0; j < NPAD; ++j) ks[j] = krow(j);
#pragma unroll
            for (int g = 0; g < 2; ++g) {  // rows t0 + 2g, t0 + 2g + 1: sum_i gamma_{t,s,i} k_t,i k_s,i, s < t
                float v[32];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int t = t0 + 2 * g + rr;
                    const float4 kt_ = krow(t);
                    float4 gm = make_float4(1.f, 1.f, 1.f, 1.f);
#pragma unroll
                    for (int s2 = NPAD - 1; s2 >= 0; --s2) {
                        if (s2 < t && t < n) {
                            gm = mul4(gm, arow(s2 + 1));  // gamma_{t,s} = a_{s+1} ... a_t
                            v[16 * rr + s2] = dot4(mul4(kt_, gm), ks[s2]);
                        } else {
                            v[16 * rr + s2] = 0.f;
                        }
                    }
                }
                warp_reduce_scatter32(v, lane);
                const int tt = t0 + 2 * g + (lane >> 4), ss = lane & 15;
                Am[(buf * NPAD + tt) * as + ss] = Gam[(buf * NPAD + tt) * as + ss] * v[0];
            }
            float4 kk[4];  // gamma_{n-1,t} o k_t for the warp's rows
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = t0 + j;
                float4 gm = make_float4(1.f, 1.f, 1.f, 1.f);
                for (int u = t + 1; u < n; ++u) gm = mul4(gm, arow(u));
                kk[j] = mul4(krow(t), gm);
            }
#pragma unroll
            for (int m0 = 0; m0 < RP; m0 += 8) {  // (gamma_{n-1,t} o k_t) . U_m
                float4 uu[8];
#pragma unroll
                for (int m = 0; m < 8; ++m)
                    uu[m] = m0 + m < RP ? *reinterpret_cast<const float4 *>(uf + (m0 + m) * 128 + 4 * lane)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = dot4(kk[i >> 3], uu[i & 7]);
                warp_reduce_scatter32(v, lane);
                const int m = m0 + (lane & 7);
                if (m < RP) kus[(buf * NPAD + t0 + (lane >> 3)) * RP + m] = v[0];
            }
            return;
        }
        // lane l: key channels 4l .. 4l+3 (panel l / 8, chunk l % 8 of its 128-byte rows)
        const unsigned char *pn = b1 + (lane >> 3) * B1P;
        auto rowv = [&](int rr) {
            return *reinterpret_cast<const float4 *>(pn + rr * 128 + ((((lane & 7) ^ rr) & 7) << 4));
        };
        float4 ks[NPAD];  // every key row once (rows n .. 15 are zero)
#pragma unroll
        for (int j = 0; j < NPAD; ++j) ks[j] = rowv(j);
        float4 kt[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) kt[j] = rowv(t0 + j);
#pragma unroll
        for (int g = 0; g < 2; ++g) {  // rows t0 + 2g, t0 + 2g + 1 against every key row
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = dot4(kt[2 * g + (i >> 4)], ks[i & 15]);
            warp_reduce_scatter32(v, lane);
            const int tt = t0 + 2 * g + (lane >> 4), ss = lane & 15;
            Am[(buf * NPAD + tt) * as + ss] = Gam[(buf * NPAD + tt) * as + ss] * v[0];
        }
        if constexpr (RP > 8) {  // K U^T (U = hi + lo) here too: 16 basis rows would make warps 1 and 5 the
                                 // slower side (measured)
#pragma unroll
            for (int m0 = 0; m0 < RP; m0 += 8) {
                float4 uu[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float4 uh = rowv(NK + m0 + m), ul = rowv(NK + RP + m0 + m);
                    uu[m] = make_float4(uh.x + ul.x, uh.y + ul.y, uh.z + ul.z, uh.w + ul.w);
                }
                float v[32];  // index i = 8 (row) + m
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = dot4(kt[i >> 3], uu[i & 7]);
                warp_reduce_scatter32(v, lane);
                kus[(buf * NPAD + t0 + (lane >> 3)) * RP + m0 + (lane & 7)] = v[0];
            }
        }
    };
    // GDN with RP <= 8, warps 1 and 5 (idle under step 1 once warp 1 has issued its copy): K U^T with U = hi + lo for
    // key rows 8 (warp / 4) .. + 7, into buffer buf
    auto ku_system = [&](int buf) {
        const int t0 = 8 * (warp >> 2);
        const unsigned char *pn = b1 + (lane >> 3) * B1P;
        auto rowv = [&](int rr) {
            return *reinterpret_cast<const float4 *>(pn + rr * 128 + ((((lane & 7) ^ rr) & 7) << 4));
        };
        float4 kt[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) kt[j] = rowv(t0 + j);
#pragma unroll
        for (int m0 = 0; m0 < RP; m0 += 4) {  // four basis rows at a time: 8 rows x 4 = 32 dots
            float4 uu[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 uh = rowv(NK + m0 + m), ul = rowv(NK + RP + m0 + m);
                uu[m] = make_float4(uh.x + ul.x, uh.y + ul.y, uh.z + ul.z, uh.w + ul.w);
            }
            float v[32];  // index i = 4 (row) + m
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = dot4(kt[i >> 2], uu[i & 3]);
            warp_reduce_scatter32(v, lane);
            kus[(buf * NPAD + t0 + (lane >> 2)) * RP + m0 + (lane & 3)] = v[0];
        }
    };

    if (warp == 0) {
        if (elect_one()) {
            for (int i = 0; i < TC_NS + 5; ++i) mbar_init(bar_s + i, 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                     "r"(TM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // the key rows n .. 15 of B1 and of the MN-major keys stay zero for the whole run (GDN; KDA rewrites
    // them every head), and so do B1's padding rows
    constexpr int KBM_BYTES = (KD ? 2 : 1) * NPAD * 512;
    for (int i = tid; i < (4 * B1P + KBM_BYTES) / 16; i += TC_THREADS) {
        unsigned char *dst = i < 4 * B1P / 16 ? b1 + 16 * i : kbm + 16 * (i - 4 * B1P / 16);
        *reinterpret_cast<float4 *>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *slot;
    const uint32_t tlane = tbase + ((uint32_t)(32 * quad) << 16);  // this warp's lanes

    // loads issued and not yet waited on, tracked by warp 1 for a drain after a give-up (bit st:
    // stage st, bit i: key buffer i), with the parity their completion will have
    unsigned pend_s = 0, pend_t = 0, par_s = 0, par_t = 0;
    auto note_state = [&](int w, int st) {
        pend_s |= 1u << st;
        par_s = (par_s & ~(1u << st)) | ((unsigned)(((w - w_begin) / TC_NS) & 1) << st);
    };
    auto note_tok = [&](int w, int i) {
        pend_t |= 1u << i;
        par_t = (par_t & ~(1u << i)) | ((unsigned)(((w - w_begin) >> 1) & 1) << i);
    };
    if (warp == 1) {
        for (int st = 0; st < TC_NS && w_begin + st < w_end; ++st) {
            if (elect_one()) issue_state(w_begin + st, st);
            note_state(w_begin + st, st);
        }
        if (elect_one()) issue_tok(w_begin, 0);
        note_tok(w_begin, 0);
        __syncwarp();
    }
    // per-token scalars, prefetched one head ahead by warp 4 (lane t holds token t)
    if (warp == 4) {  // (KDA: the decays are per channel and enter elsewhere; its table keeps a = 1)
        if (lane < n) {
            if (!KD) a_nx = abuf[(size_t)head_of(w_begin) * W + lane];
            b_nx = bbuf[(size_t)head_of(w_begin) * W + lane];
        }
        decay_table(a_nx, b_nx, 0);  // the first head's
    }
    bool failed = false;
    int h_prev = -1;
    constexpr uint32_t idx_1 = idesc_tf32(128, N1, 0);
    constexpr uint32_t idx_4 = idesc_tf32(128, 128, 1);
    const int kc = (n + 7) >> 3;  // K steps of step 4

    for (int w = w_begin, it = 0; w < w_end; ++w, ++it) {
        const int st = it % TC_NS, tb = it & 1, ph = it & 1;
        const int head = head_of(w), h = w / B;
        unsigned char *stage = stage_of(st);
        const unsigned char *tk = tok_of(tb);
        // the next head's keys into the other buffer (its last reader, the previous head, is done)
        if (warp == 1 && w + 1 < w_end) {
            fence_proxy_async();
            if (elect_one()) issue_tok(w + 1, tb ^ 1);
            note_tok(w + 1, tb ^ 1);
            __syncwarp();
        }
        const int db = it & 1;  // this head's decay table
        if (warp == 4 && w + 1 < w_end && lane < n) {  // the next head's scalars, for its table
            if (!KD) a_nx = abuf[(size_t)head_of(w + 1) * W + lane];
            b_nx = bbuf[(size_t)head_of(w + 1) * W + lane];
        }
        if (h != h_prev) {  // basis rows of head index h (rows past r zero): GDN into B1 rows 16 .. (hi, then
                            // lo); KDA into uf (B1's rows are scaled by each head's decay product)
            for (int i = tid; i < RP * 32; i += TC_THREADS) {
                const int m = i >> 5, c4 = (i & 31) * 4;
                float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
                if (P != nullptr && m < r) u = reinterpret_cast<const float4 *>(U + ((size_t)h * r + m) * 128)[i & 31];
                if (KD) {
                    reinterpret_cast<float4 *>(uf)[i] = u;
                    continue;
                }
                const float4 uh = make_float4(tf32_hi(u.x), tf32_hi(u.y), tf32_hi(u.z), tf32_hi(u.w));
                const float4 ul = make_float4(u.x - uh.x, u.y - uh.y, u.z - uh.z, u.w - uh.w);
                unsigned char *pn = b1 + (c4 >> 5) * B1P;
                *reinterpret_cast<float4 *>(pn + sw128(NPAD + m, c4 & 31)) = uh;
                *reinterpret_cast<float4 *>(pn + sw128(NPAD + RP + m, c4 & 31)) = ul;
            }
            h_prev = h;
        }
        // ---- keys and state landed
        bool ok = true;
        if (warp == 1) {
            ok = mbar_wait(bar_t + tb, (it >> 1) & 1);
            pend_t &= ~(1u << tb);
            if (ok) {
                ok = mbar_wait(bar_s + st, (it / TC_NS) & 1);
                pend_s &= ~(1u << st);
            }
        }
        if (__syncthreads_or(!ok)) { failed = true; break; }
        // ---- the keys as fp32 rows of B1 (K-major) and of the MN-major operand of step 4
        if constexpr (KD) {
            // per key channel i: threads 0-127 the prefix products g_t (keys of step 1: g_t o k_t,
            // hi and lo; the basis rows g_{n-1} o U_m, hi and lo; g_{n-1} for the store), threads
            // 128-255 the suffix products gamma_{n-1,s} (keys of step 4, hi and lo)
            const int i = tid & 127, ci = i & 31;
            const QT *kr = reinterpret_cast<const QT *>(tk);
            const float *ar = reinterpret_cast<const float *>(tk + AOFF);
            if (tid < 128) {
                unsigned char *pn = b1 + (i >> 5) * B1P;
                float g = 1.f;
#pragma unroll
                for (int t = 0; t < NPAD; ++t) {
                    float kg = 0.f;
                    if (t < n) {
                        g *= ar[t * 128 + i];
                        kg = g * ld1(kr + t * 128 + i);
                    }
                    const float hi = tf32_hi(kg);
                    *reinterpret_cast<float *>(pn + sw128(t, ci)) = hi;
                    *reinterpret_cast<float *>(pn + sw128(NPAD + t, ci)) = kg - hi;
                }
                gnv[i] = g;
#pragma unroll
                for (int m = 0; m < RP; ++m) {
                    const float ug = g * uf[m * 128 + i];
                    const float hi = tf32_hi(ug);
                    *reinterpret_cast<float *>(pn + sw128(NK + m, ci)) = hi;
                    *reinterpret_cast<float *>(pn + sw128(NK + RP + m, ci)) = ug - hi;
                }
            } else {
                unsigned char *dh = kbm + (i >> 5) * (NPAD * 128), *dl = dh + NPAD * 512;
                float gam = 1.f;  // gamma_{n-1,s} = a_{s+1} ... a_{n-1}, s descending
#pragma unroll
                for (int s2 = NPAD - 1; s2 >= 0; --s2) {
                    float kk = 0.f;
                    if (s2 < n) {
                        kk = gam * ld1(kr + s2 * 128 + i);
                        gam *= ar[s2 * 128 + i];
                    }
                    const float hi = tf32_hi(kk);
                    *reinterpret_cast<float *>(dh + sw128_32b(s2, ci)) = hi;
                    *reinterpret_cast<float *>(dl + sw128_32b(s2, ci)) = kk - hi;
                }
            }
        } else
        for (int i = tid; i < n * 16; i += TC_THREADS) {
            const int t = i >> 4, c8 = (i & 15) * 8;
            float x[8];
            load4(reinterpret_cast<const QT *>(tk) + t * 128 + c8, x);
            load4(reinterpret_cast<const QT *>(tk) + t * 128 + c8 + 4, x + 4);
            const float4 lo4 = make_float4(x[0], x[1], x[2], x[3]), hi4 = make_float4(x[4], x[5], x[6], x[7]);
            unsigned char *pn = b1 + (c8 >> 5) * B1P;
            *reinterpret_cast<float4 *>(pn + sw128(t, c8 & 31)) = lo4;
            *reinterpret_cast<float4 *>(pn + sw128(t, (c8 & 31) + 4)) = hi4;
            unsigned char *dst = kbm + (c8 >> 5) * (NPAD * 128) + sw128_32b(t, c8 & 31);
            *reinterpret_cast<float4 *>(dst) = lo4;
            *reinterpret_cast<float4 *>(dst + 16) = hi4;
        }
        // ---- the split: this thread's 64 state values into registers, their TF32 remainder into
        // tensor memory (lane = row, column = key channel)
        float s0[64];
#pragma unroll
        for (int j2 = 0; j2 < 2; ++j2) {
            const int pnl = 2 * half + j2;
            uint32_t lo[32];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 f = *reinterpret_cast<const float4 *>(stage + pnl * TC_PANEL + sw128(row, 4 * q));
                s0[32 * j2 + 4 * q] = f.x; s0[32 * j2 + 4 * q + 1] = f.y;
                s0[32 * j2 + 4 * q + 2] = f.z; s0[32 * j2 + 4 * q + 3] = f.w;
                lo[4 * q] = __float_as_uint(f.x - tc_tf32(f.x));
                lo[4 * q + 1] = __float_as_uint(f.y - tc_tf32(f.y));
                lo[4 * q + 2] = __float_as_uint(f.z - tc_tf32(f.z));
                lo[4 * q + 3] = __float_as_uint(f.w - tc_tf32(f.w));
            }
            tmem_st32(tlane + TM_LO + 32 * pnl, lo);
        }
        tmem_wait_st();
        fence_proxy_async();  // B1 and the MN-major keys, written here, are read by the tensor core
        tc_fence_before();
        __syncthreads();
        if (warp == 1) {  // the previous head's stage, once its store has read it, for the head two ahead
            if (it >= 1 && w - 1 + TC_NS < w_end) {
                if (elect_one()) {
                    bulk_wait_read_all();
                    fence_proxy_async();
                    issue_state(w - 1 + TC_NS, (it - 1) % TC_NS);
                }
                note_state(w - 1 + TC_NS, (it - 1) % TC_NS);
                __syncwarp();
            }
        }
        if (warp == 0) {  // ---- step 1: [X | S_0^T U] = S_0^T [K; U], the stage pass and the remainder pass
            tc_fence_after();
            // a descriptor's address field is the byte address / 16 (shared addresses < 256 KB: no carry),
            // so the K steps are offsets added to one base descriptor
            const uint64_t ad0 = smem_desc_kmajor_sw128(smem_u32(stage)), bd0 = smem_desc_kmajor_sw128(b1_a);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 16; ++kk)  // the stage as it arrived (the tensor core takes its TF32 part)
                    mma_ss(tbase + TM_D1, ad0 + (((kk >> 2) * TC_PANEL + (kk & 3) * 32) >> 4),
                           bd0 + (((kk >> 2) * B1P + (kk & 3) * 32) >> 4), idx_1, kk);
#pragma unroll
                for (int kk = 0; kk < 16; ++kk)  // the remainder, from tensor memory
                    mma_ts(tbase + TM_D1, tbase + TM_LO + 8 * kk, bd0 + (((kk >> 2) * B1P + (kk & 3) * 32) >> 4),
                           idx_1, 1);
                mma_commit(bar_1);
            }
            __syncwarp();
        } else if ((warp & 2) != 0) {  // ---- step 2 under step 1: the Gram (and, for KDA, K U^T)
            gram_system(db, tk);
        } else if (!KD && RP <= 8 && (warp == 1 || warp == 5)) {  // GDN's K U^T
            ku_system(db);
        }
        // ---- step 1 complete
        if (warp == 0) ok = mbar_wait(bar_1, ph);
        if (__syncthreads_or(!ok)) { failed = true; break; }
        const float g = gn[db];
        // ---- step 3: the triangular solve, one value channel per thread (warps 0-3), and the sketch
        if (half == 0) {
            tc_fence_after();
            float xd[N1];
            {
                uint32_t d[32];
                tmem_ld32(tlane + TM_D1, d);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) xd[j] = __uint_as_float(d[j]);
                if constexpr (N1 > 32) {
#pragma unroll
                    for (int c0 = 32; c0 < N1; c0 += 16) {
                        uint32_t e[16];
                        tmem_ld16(tlane + TM_D1 + c0, e);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) xd[c0 + j] = __uint_as_float(e[j]);
                    }
                }
            }
            const QT *vt = reinterpret_cast<const QT *>(tk + NPAD * 128 * sizeof(QT));
            float wv[NPAD];
            const float *A = Am + db * NPAD * as;
#pragma unroll
            for (int t = 0; t < NPAD; ++t) {  // (I + A) w = y, forward (A[t][s] = 0 for s >= t)
                // (value rows past n are not copied: their shared memory is not read)
                // x_t = S_0^T k_t (KDA: S_0^T (g_t o k_t), from its hi and lo key rows)
                const float xt = KD ? xd[t] + xd[NPAD + t] : xd[t];
                float y0 = t < n ? bv[db * NPAD + t] * ld1(vt + t * 128 + row) - ev[db * NPAD + t] * xt : 0.f,
                      y1 = 0.f;
#pragma unroll
                for (int s4 = 0; s4 < t; s4 += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(A + t * as + s4);
                    y0 = fmaf(-a4.x, wv[s4], y0);
                    if (s4 + 1 < t) y1 = fmaf(-a4.y, wv[s4 + 1], y1);
                    if (s4 + 2 < t) y0 = fmaf(-a4.z, wv[s4 + 2], y0);
                    if (s4 + 3 < t) y1 = fmaf(-a4.w, wv[s4 + 3], y1);
                }
                wv[t] = y0 + y1;
            }
#pragma unroll
            for (int t = 0; t < NPAD; ++t) wv[t] *= cv[db * NPAD + t];  // W~_t = gamma_{n-1,t} w_t
            // W~ split hi | lo into tensor memory, lane = value channel, column = token: the A of step 4
            {
                uint32_t hv[NPAD], lv[NPAD];
#pragma unroll
                for (int t = 0; t < NPAD; ++t) {
                    const float hi = tf32_hi(wv[t]);
                    hv[t] = __float_as_uint(hi);
                    lv[t] = __float_as_uint(wv[t] - hi);
                }
                tmem_st16(tlane + TM_W, hv);
                tmem_st16(tlane + TM_W + NPAD, lv);
                tmem_wait_st();
            }
            // P = S_n^T U = g (S_0^T U) + sum_t w~_t (K U^T)_t
            if (P != nullptr) {
                float pp[RP];
#pragma unroll
                for (int m = 0; m < RP; ++m) pp[m] = g * (xd[NK + m] + xd[NK + RP + m]);
#pragma unroll
                for (int t = 0; t < NPAD; ++t)
                    if (t < n)
#pragma unroll
                        for (int m = 0; m < RP; ++m) pp[m] = fmaf(wv[t], kus[(db * NPAD + t) * RP + m], pp[m]);
                float *prow = P + ((size_t)head * 128 + row) * r;
                if ((r & 3) == 0) {
#pragma unroll
                    for (int m = 0; m < RP; m += 4)
                        if (m < r) *reinterpret_cast<float4 *>(prow + m) = make_float4(pp[m], pp[m + 1], pp[m + 2], pp[m + 3]);
                } else {
#pragma unroll
                    for (int m = 0; m < RP; ++m)
                        if (m < r) prow[m] = pp[m];
                }
            }
        } else if (warp == 4 && w + 1 < w_end) {  // meanwhile: the next head's decay table
            decay_table(a_nx, b_nx, db ^ 1);
        }
        tc_fence_before();
        __syncthreads();
        // ---- step 4: D^T = W~^T K (W~ hi and lo passes; KDA: also W~ hi against the decayed keys' lo)
        if (warp == 0) {
            tc_fence_after();
            if (elect_one()) {
#pragma unroll 1
                for (int pass = 0; pass < (KD ? 3 : 2); ++pass)
#pragma unroll 1
                    for (int kk = 0; kk < kc; ++kk) {
                        const uint64_t bd = smem_desc_mnmajor_sw128_32b(
                            kbm_a + (pass == 2 ? NPAD * 512 : 0) + kk * 1024, NPAD * 128);
                        mma_ts(tbase + TM_D2, tbase + TM_W + (pass == 1 ? NPAD : 0) + 8 * kk, bd, idx_4, pass | kk);
                    }
                mma_commit(bar_4);
            }
            __syncwarp();
            ok = mbar_wait(bar_4, ph);
        }
        if (__syncthreads_or(!ok)) { failed = true; break; }
        tc_fence_after();
        // ---- step 5: S_n = g S_0 + D (KDA: g per key channel), back into the stage (its step-1 reads are
        // complete), then out by TMA tiled stores
        float orow = 0.f;  // the exact read o = S_n^T q over this thread's 64 key channels
        const QT *qh = READ ? qv + (size_t)head * 128 : nullptr;
#pragma unroll
        for (int j2 = 0; j2 < 2; ++j2) {
            const int pnl = 2 * half + j2;
            uint32_t d[32];
            tmem_ld32(tlane + TM_D2 + 32 * pnl, d);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 g4 = KD ? *reinterpret_cast<const float4 *>(gnv + 32 * pnl + 4 * q) : make_float4(g, g, g, g);
                const float4 sn = make_float4(fmaf(g4.x, s0[32 * j2 + 4 * q], __uint_as_float(d[4 * q])),
                                              fmaf(g4.y, s0[32 * j2 + 4 * q + 1], __uint_as_float(d[4 * q + 1])),
                                              fmaf(g4.z, s0[32 * j2 + 4 * q + 2], __uint_as_float(d[4 * q + 2])),
                                              fmaf(g4.w, s0[32 * j2 + 4 * q + 3], __uint_as_float(d[4 * q + 3])));
                *reinterpret_cast<float4 *>(stage + pnl * TC_PANEL + sw128(row, 4 * q)) = sn;
                if constexpr (READ) {  // (the same query channels for every lane: broadcast loads)
                    float qf[4];
                    load4(qh + 32 * pnl + 4 * q, qf);
                    orow = fmaf(sn.x, qf[0], fmaf(sn.y, qf[1], fmaf(sn.z, qf[2], fmaf(sn.w, qf[3], orow))));
                }
            }
        }
        if (READ && half == 1) xo[row] = orow;
        tc_fence_before();
        fence_proxy_async();  // the new state, written by these threads, is read by the TMA store
        __syncthreads();  // tensor memory and the operands are free for the next head
        if (READ && half == 0) o[(size_t)head * 128 + row] = orow + xo[row];
        if (warp == 1) {
            if (elect_one()) {
                for (int p = 0; p < 4; ++p) tma_store_2d(&tmS, 32 * p, head * 128, stage + p * TC_PANEL);
                bulk_commit();
            }
            __syncwarp();
        }
    }

    if (failed) {  // count the give-up, then let what is in flight land (bounded)
        if (warp == 1) {
            if (elect_one()) atomicAdd(&g_update_tc_giveups, 1u);
            for (int st = 0; st < TC_NS; ++st)
                if (pend_s & (1u << st)) mbar_wait(bar_s + st, (par_s >> st) & 1);
            for (int i = 0; i < 2; ++i)
                if (pend_t & (1u << i)) mbar_wait(bar_t + i, (par_t >> i) & 1);
        } else if (warp == 0) {
            if (elect_one()) mma_commit(bar_d);  // arrives once every MMA issued before it has completed
            __syncwarp();
            mbar_wait(bar_d, 0);
        }
    }
    if (warp == 1) {
        if (elect_one()) bulk_wait_all();  // the last stores have landed before the kernel ends
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(TM_COLS) : "memory");
    }
}

// ---- host ---------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
    static std::mutex mu;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

}  // namespace

int update_tc_giveups(bool reset, unsigned *count) { return read_counter(&g_update_tc_giveups, reset, count); }

// The delta-rule window update on the tensor cores, where it applies (with q and o: also the exact read
// o = S_n^T q of the window's last step, from the updated fp32 state): Gated DeltaNet or KDA,
// dk = dv = 128, fp32 state, bf16 keys and values (keys exact in TF32), 1 <= n <= 16 tokens,
// r <= 16 (KDA: r <= 8, whose split decayed keys and basis rows take more shared memory).
// Returns TC_NOT_APPLICABLE for other shapes (the caller then runs the CUDA-core kernel), else a
// sketchssm_status.
int launch_update_window_tc(const sketchssm_dims &d, void *S, float *P, const float *U, const void *k,
                            const void *v, const float *alpha, const float *beta, int n, cudaStream_t stream,
                            const void *q, float *o) {
    const bool kda = d.kind == SKSSM_KDA;
    if ((d.kind != SKSSM_GDN && !kda) || d.dk != 128 || d.dv != 128 || d.state_dtype != SKSSM_F32)
        return TC_NOT_APPLICABLE;
    if (d.qkv_dtype != SKSSM_BF16 || n < 1 || n > TC_NPAD || d.r > (kda ? 8 : 16)) return TC_NOT_APPLICABLE;
    const int rp = d.r <= 4 ? 4 : d.r <= 8 ? 8 : 16;
    const TcLayout L = tc_layout(rp, kda);
    if (L.total > TC_SMEM_LIMIT) return TC_NOT_APPLICABLE;
    const int NH = d.B * d.H;

    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_tiled();
    if (!enc) return SKSSM_ERR_CUDA;
    CUtensorMap map;
    const cuuint64_t dims[2] = {128, (cuuint64_t)NH * 128};
    const cuuint64_t strides[1] = {128 * sizeof(float)};
    const cuuint32_t box[2] = {32, 128};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, S, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return SKSSM_ERR_CUDA;

    auto run = [&](auto KINDc, auto RPc, auto READc) -> int {
        constexpr int KIND = decltype(KINDc)::value, RP = decltype(RPc)::value;
        auto kern = update_window_delta_tc<KIND, RP, decltype(READc)::value>;
        if (allow_max_smem(reinterpret_cast<const void *>(kern)) != SKSSM_OK) return SKSSM_ERR_CUDA;
        int sms = 0;
        if (sm_count(&sms) != SKSSM_OK) return SKSSM_ERR_CUDA;
        const int grid = NH < sms ? NH : sms;
        kern<<<grid, TC_THREADS, L.total, stream>>>(map, P, U, static_cast<const __nv_bfloat16 *>(k),
                                                    static_cast<const __nv_bfloat16 *>(v), alpha, beta,
                                                    static_cast<const __nv_bfloat16 *>(q), o, d.B, d.H, d.r, n, d.W);
        return launch_status();
    };
    using G = std::integral_constant<int, GDN>;
    using K = std::integral_constant<int, KDA>;
    using R4 = std::integral_constant<int, 4>;
    using R8 = std::integral_constant<int, 8>;
    using R16 = std::integral_constant<int, 16>;
    using NoRead = std::false_type;
    if (kda) {  // (the fused read is taken for Gated DeltaNet only)
        if (q != nullptr) return TC_NOT_APPLICABLE;
        return rp == 4 ? run(K(), R4(), NoRead()) : run(K(), R8(), NoRead());
    }
    if (q != nullptr) {
        using Read = std::true_type;
        if (rp == 4) return run(G(), R4(), Read());
        if (rp == 8) return run(G(), R8(), Read());
        return run(G(), R16(), Read());
    }
    if (rp == 4) return run(G(), R4(), NoRead());
    if (rp == 8) return run(G(), R8(), NoRead());
    return run(G(), R16(), NoRead());
}

}  // namespace skssm

// update_window_tc.cu -- the Gated DeltaNet window update on the tensor cores.
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
//   1. X = S_0^T K^T and S_0^T U^T  fp32 dot products on the CUDA cores (a value
//                                   channel's row against every key and basis row)
//   2. the key Gram K K^T and K U^T, fp32, CUDA cores
//   3. the triangular solve         CUDA cores, one value channel per thread
//   4. D^T = W~^T K, W~_s = gamma_{n-1,s} w_s
//                                   tcgen05.mma kind::tf32, M = 128, N = 128, K = n,
//                                   both operands in shared memory
//   5. S_n^T = g_{n-1} S_0^T + D^T, and the sketch without a pass over S_n:
//          P = S_n^T U = g_{n-1} S_0^T U + sum_t W~_t (K U^T)_t
// The tensor cores take the rank-n update (half of the arithmetic); the dot
// products stay on the CUDA cores because their N (the n tokens) is too narrow:
// a tcgen05.mma costs ~56 cycles to issue whatever N <= 128 (measured), so the
// 32 instructions X would need cost more than the dots themselves.
// fp32 accuracy from the TF32 tensor cores: a TF32 operand keeps the top 11
// significant bits of an fp32 value, so W~ is split as W~ = hi + lo with hi = W~
// with its low 13 mantissa bits cleared (exactly TF32) and lo = W~ - hi (exact
// in fp32; the tensor core keeps its top 11 bits); the keys are bf16, exact in
// TF32, so D = hi^T K + lo^T K in two passes, off by less than 2^-21 of W~.
//
// Data movement: a persistent CTA (one per SM: the shared memory below takes
// most of the SM) walks a contiguous run of heads in (h, b) order.  Each head's
// state arrives by four TMA tiled copies (cp.async.bulk.tensor, 128 rows x 32
// fp32 each, 128-byte swizzle) into one of NS shared-memory stages, one head or
// more ahead; the tokens arrive by 1-D bulk copies one head ahead.  Each thread
// keeps its 64 values of S_0 in registers from step 1 to step 5, which writes
// S_n back into the stage, from where it leaves by TMA tiled stores.  Roles:
// warp 0 issues the MMAs, warp 1 the copies (and polls their barriers), warp 4
// (lane t = token t) does the per-token scalars; the other warps sleep in CTA
// barriers rather than poll.  Tensor memory: D, 128 columns.
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
constexpr int TC_PANEL = 128 * 128;    // bytes of one 32-column panel of a head's state (128 rows x 128 B)
constexpr int TC_STATE = 4 * TC_PANEL;
constexpr uint32_t TM_COLS = 128;
constexpr uint32_t TM_D = 0;  // tensor-memory columns of the state increment D
constexpr int TC_SMEM_LIMIT = 227 * 1024;

__host__ __device__ inline int round_up(int x, int a) { return (x + a - 1) / a * a; }

// Shared-memory layout: byte offsets from the 1024-aligned base.
struct TcLayout {
    int stages;     // NS x 64 KB: state stages (TMA destination and source), 1024-aligned
    int wh, wl;     // W~^T hi and lo: 128 rows x 128 B, K-major, 128-byte swizzle (A of step 4)
    int kbm;        // the keys, MN-major TF32 layout: 4 panels x npad rows x 128 B (B of step 4)
    int kf;         // the keys, fp32 rows [npad][128] (step 1, 2)
    int uf;         // the basis rows, fp32 [rp][128] (rows r .. rp-1 zero)
    int tok;        // two token buffers: k rows then v rows of one head, bf16
    int tok_bytes;  // bytes of one token buffer
    int xex;        // partial dot products of the second column half: [128][npad + rp]
    int am;         // A [npad][npad + 1], G [npad][npad + 1], K U^T [npad][rp], b_t g_t, gamma_{n-1,t},
                    // b_t [npad] each, g
    int bars;       // mbarriers: NS stages, 2 token buffers, D, drain
    int slot;       // tensor-memory base address written by tcgen05.alloc
    int total;      // bytes to request (with slack for aligning the base)
};

__host__ __device__ inline TcLayout tc_layout(int ns, int npad, int rp, int W) {
    TcLayout L;
    int o = 0;
    L.stages = o; o += ns * TC_STATE;
    L.wh = o; o += 128 * 128;
    L.wl = o; o += 128 * 128;
    L.kbm = o; o += npad * 512;
    L.kf = o; o += npad * 512;
    L.uf = o; o += rp * 512;
    L.tok_bytes = round_up(2 * W * 128 * 2, 128);
    L.tok = o; o += 2 * L.tok_bytes;
    L.xex = o; o += 128 * (npad + rp) * 4;
    L.am = o; o += round_up((2 * npad * (npad + 1) + npad * rp + 3 * npad + 4) * 4, 16);
    L.bars = o; o += 8 * (ns + 4);
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

// fp32 value with the 13 low mantissa bits cleared: what a TF32 operand keeps of it
__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xffffe000u); }

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

template <int NPAD, int RP>
__global__ void __launch_bounds__(TC_THREADS, 1)
update_window_gdn_tc(const __grid_constant__ CUtensorMap tmS, float *__restrict__ P, const float *__restrict__ U,
                     const __nv_bfloat16 *__restrict__ kbuf, const __nv_bfloat16 *__restrict__ vbuf,
                     const float *__restrict__ abuf, const float *__restrict__ bbuf, int B, int H, int r, int n, int W,
                     int ns) {
    using QT = __nv_bfloat16;
    constexpr int npad = NPAD, NX = NPAD + RP, as = NPAD + 1;
    extern __shared__ __align__(1024) unsigned char tc_raw[];
    unsigned char *sm = tc_raw + ((1024 - (smem_u32(tc_raw) & 1023)) & 1023);
    const TcLayout L = tc_layout(ns, npad, RP, W);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quad = warp & 3, half = warp >> 2;
    const int row = 32 * quad + lane;  // this thread's state row (value channel) and tensor-memory lane
    const int NH = B * H;
    const int per = (NH + gridDim.x - 1) / gridDim.x;
    const int w_begin = blockIdx.x * per, w_end = min(NH, w_begin + per);
    if (w_begin >= w_end) return;  // the whole CTA, before anything is allocated

    uint64_t *bar_s = reinterpret_cast<uint64_t *>(sm + L.bars);  // [ns] state stages
    uint64_t *bar_t = bar_s + ns;                                 // [2] token buffers
    uint64_t *bar_c = bar_t + 2;                                  // the state increment D
    uint64_t *bar_d = bar_c + 1;                                  // the drain after a give-up
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L.slot);
    float *Am = reinterpret_cast<float *>(sm + L.am);  // [npad][as]: A[t][s] = b_t gamma_{t,s} G[t][s], s < t
    float *Gm = Am + npad * as;                         // [npad][as]: G[t][s] = k_t . k_s, s < t
    float *kus = Gm + npad * as;                        // [npad][RP]: (K U^T)[t][m]
    float *ev = kus + npad * RP;                        // [npad]: b_t g_t
    float *cv = ev + npad;                              // [npad]: gamma_{n-1,s}
    float *bv = cv + npad;                              // [npad]: b_t
    float *gn = bv + npad;                              // [1]:  g_{n-1}
    float *kf = reinterpret_cast<float *>(sm + L.kf);   // [npad][128]
    float *uf = reinterpret_cast<float *>(sm + L.uf);   // [RP][128]
    float *xex = reinterpret_cast<float *>(sm + L.xex);  // [128][NX]
    unsigned char *kbm = sm + L.kbm;
    unsigned char *wh = sm + L.wh, *wl = sm + L.wl;
    const uint32_t kbm_a = smem_u32(kbm), wh_a = smem_u32(wh), wl_a = smem_u32(wl);
    const int kbytes = n * 128 * (int)sizeof(QT);

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
        mbar_expect_tx(bar, 2 * kbytes);
        bulk_g2s(tok_of(i), kbuf + off, kbytes, bar);
        bulk_g2s(tok_of(i) + W * 128 * sizeof(QT), vbuf + off, kbytes, bar);
    };

    if (warp == 0) {
        if (elect_one()) {
            for (int i = 0; i < ns + 4; ++i) mbar_init(bar_s + i, 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                     "r"(TM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *slot;
    const uint32_t tlane = tbase + ((uint32_t)(32 * quad) << 16);  // this warp's lanes

    // loads issued and not yet waited on, tracked by warp 1 for a drain after a give-up (bit st:
    // stage st, bit i: token buffer i), with the parity their completion will have
    unsigned pend_s = 0, pend_t = 0, par_s = 0, par_t = 0;
    auto note_state = [&](int w, int st) {
        pend_s |= 1u << st;
        par_s = (par_s & ~(1u << st)) | ((unsigned)(((w - w_begin) / ns) & 1) << st);
    };
    auto note_tok = [&](int w, int i) {
        pend_t |= 1u << i;
        par_t = (par_t & ~(1u << i)) | ((unsigned)(((w - w_begin) >> 1) & 1) << i);
    };
    if (warp == 1) {
        for (int st = 0; st < ns && w_begin + st < w_end; ++st) {
            if (elect_one()) issue_state(w_begin + st, st);
            note_state(w_begin + st, st);
        }
        if (elect_one()) issue_tok(w_begin, 0);
        note_tok(w_begin, 0);
        __syncwarp();
    }
    // per-token scalars, prefetched one head ahead by warp 4 (lane t holds token t)
    float a_nx = 1.f, b_nx = 0.f;
    if (warp == 4 && lane < n) {
        a_nx = abuf[(size_t)head_of(w_begin) * W + lane];
        b_nx = bbuf[(size_t)head_of(w_begin) * W + lane];
    }
    int h_prev = -1;
    bool failed = false;
    constexpr uint32_t idx_c = idesc_tf32(128, 128, 1);
    const int kc = (n + 7) >> 3;  // K steps of the state increment

    for (int w = w_begin, it = 0; w < w_end; ++w, ++it) {
        const int st = it % ns, tb = it & 1, ph = it & 1;
        const int head = head_of(w), h = w / B;
        unsigned char *stage = stage_of(st);
        const unsigned char *tk = tok_of(tb);
        // the next head's tokens into the other buffer (its last reader, the previous head, is done)
        if (warp == 1 && w + 1 < w_end) {
            fence_proxy_async();
            if (elect_one()) issue_tok(w + 1, tb ^ 1);
            note_tok(w + 1, tb ^ 1);
            __syncwarp();
        }
        const float a_t = a_nx, b_t = b_nx;
        if (warp == 4 && w + 1 < w_end && lane < n) {
            a_nx = abuf[(size_t)head_of(w + 1) * W + lane];
            b_nx = bbuf[(size_t)head_of(w + 1) * W + lane];
        }
        if (h != h_prev) {  // basis rows of head index h (rows r .. RP-1 zero)
            for (int i = tid; i < RP * 32; i += TC_THREADS) {
                const int m = i >> 5;
                reinterpret_cast<float4 *>(uf)[i] =
                    (P != nullptr && m < r) ? reinterpret_cast<const float4 *>(U + (size_t)h * r * 128)[i]
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            h_prev = h;
        }
        // ---- tokens landed: the keys as fp32 rows, and MN-major for step 4 (rows n .. npad-1 zero)
        bool ok = true;
        if (warp == 1) {
            ok = mbar_wait(bar_t + tb, (it >> 1) & 1);
            pend_t &= ~(1u << tb);
        }
        if (__syncthreads_or(!ok)) { failed = true; break; }
        for (int i = tid; i < npad * 16; i += TC_THREADS) {
            const int t = i >> 4, c8 = (i & 15) * 8;
            float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (t < n) {
                load4(reinterpret_cast<const QT *>(tk) + t * 128 + c8, x);
                load4(reinterpret_cast<const QT *>(tk) + t * 128 + c8 + 4, x + 4);
            }
            const float4 lo4 = make_float4(x[0], x[1], x[2], x[3]), hi4 = make_float4(x[4], x[5], x[6], x[7]);
            *reinterpret_cast<float4 *>(kf + t * 128 + c8) = lo4;
            *reinterpret_cast<float4 *>(kf + t * 128 + c8 + 4) = hi4;
            unsigned char *dst = kbm + (c8 >> 5) * (npad * 128) + sw128_32b(t, c8 & 31);
            *reinterpret_cast<float4 *>(dst) = lo4;
            *reinterpret_cast<float4 *>(dst + 16) = hi4;
        }
        fence_proxy_async();  // the MN-major keys are read by the tensor core
        __syncthreads();
        // ---- the key Gram (t > s) and K U^T: one dot of two 128-vectors per task, the rows read from a
        // per-thread starting chunk so that the threads of a warp fall on distinct banks
        {
            const int ng = n * (n - 1) / 2;
            const int rot = tid & 31;
            for (int task = tid; task < ng + n * RP; task += TC_THREADS) {
                const float *x, *y;
                int t, s2;
                if (task < ng) {
                    t = 1;
                    int rem = task;
                    while (rem >= t) { rem -= t; ++t; }
                    s2 = rem;
                    x = kf + t * 128;
                    y = kf + s2 * 128;
                } else {
                    t = (task - ng) / RP;
                    s2 = (task - ng) % RP;
                    x = kf + t * 128;
                    y = uf + s2 * 128;
                }
                float2 acc2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                  make_float2(0.f, 0.f)};
#pragma unroll 4
                for (int q = 0; q < 32; ++q) {
                    const int c = ((q + rot) & 31) * 4;
                    const float4 a4 = *reinterpret_cast<const float4 *>(x + c);
                    const float4 b4 = *reinterpret_cast<const float4 *>(y + c);
                    acc2[q & 3] = fma2(make_float2(a4.x, a4.y), make_float2(b4.x, b4.y), acc2[q & 3]);
                    acc2[q & 3] = fma2(make_float2(a4.z, a4.w), make_float2(b4.z, b4.w), acc2[q & 3]);
                }
                const float dsum = (acc2[0].x + acc2[0].y) + (acc2[1].x + acc2[1].y) + (acc2[2].x + acc2[2].y) +
                                   (acc2[3].x + acc2[3].y);
                if (task < ng) Gm[t * as + s2] = dsum;
                else kus[t * RP + s2] = dsum;
            }
        }
        float at = 1.f, bt = 0.f;  // warp 4: this lane's token scalars (lanes >= n: a = 1, b = 0)
        if (warp == 4) {  // decay products
            at = lane < n ? a_t : 1.f;
            bt = lane < n ? b_t : 0.f;
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
            if (lane < npad) {
                ev[lane] = bt * g;
                bv[lane] = bt;
                cv[lane] = lane == 31 ? 1.f : c;  // gamma_{n-1,s} = a_{s+1} ... a_{n-1}
            }
            const float gl = __shfl_sync(FULL, g, n - 1);
            if (lane == 0) *gn = gl;
        }
        // ---- state landed
        if (warp == 1) {
            ok = mbar_wait(bar_s + st, (it / ns) & 1);
            pend_s &= ~(1u << st);
        }
        if (__syncthreads_or(!ok)) { failed = true; break; }  // (also: the Gram and the scalars are ready)
        if (warp == 4) {
            // the system (I + A) w = y, A[t][s] = b_t gamma_{t,s} (k_t . k_s) for s < t (lane t = row t),
            // then T~ = diag(gamma_{n-1,.}) (I + A)^-1 (lane s = column s), so that W~ = T~ y
            float gam = 1.f;  // gamma_{t,s} for t = lane, s descending
#pragma unroll
            for (int s = NPAD - 2; s >= 0; --s) {
                const float a1 = __shfl_sync(FULL, at, s + 1);
                if (lane > s) {
                    gam *= a1;
                    if (lane < n) Am[lane * as + s] = bt * gam * Gm[lane * as + s];
                }
            }
            __syncwarp();
            // column `lane` of (I + A)^-1 by forward substitution; its entries above the diagonal are
            // zero, so every row sums over all u < t without a test (two partial sums)
            float tc[NPAD];
#pragma unroll
            for (int t = 0; t < NPAD; ++t) {
                float x0 = t == lane ? 1.f : 0.f, x1 = 0.f;
                if (t < n) {
#pragma unroll
                    for (int u = 0; u < t; u += 2) {
                        x0 = fmaf(-Am[t * as + u], tc[u], x0);
                        if (u + 1 < t) x1 = fmaf(-Am[t * as + u + 1], tc[u + 1], x1);
                    }
                }
                tc[t] = t < n ? x0 + x1 : 0.f;
            }
            if (lane < NPAD)
#pragma unroll
                for (int t = 0; t < NPAD; ++t) Gm[t * as + lane] = t < n ? cv[t] * tc[t] : 0.f;  // T~ over the Gram
        } else if (warp == 1) {  // the stage of the previous head is refilled once its store has read it
            if (ns > 1 && it >= 1 && w - 1 + ns < w_end) {
                if (elect_one()) {
                    bulk_wait_read_all();
                    fence_proxy_async();
                    issue_state(w - 1 + ns, (it - 1) % ns);
                }
                note_state(w - 1 + ns, (it - 1) % ns);
                __syncwarp();
            }
        }
        // ---- step 1: this thread's 64 state values, dotted with every key and basis row
        float s0[64];
#pragma unroll
        for (int j2 = 0; j2 < 2; ++j2)
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 f =
                    *reinterpret_cast<const float4 *>(stage + (2 * half + j2) * TC_PANEL + sw128(row, 4 * q));
                s0[32 * j2 + 4 * q] = f.x; s0[32 * j2 + 4 * q + 1] = f.y;
                s0[32 * j2 + 4 * q + 2] = f.z; s0[32 * j2 + 4 * q + 3] = f.w;
            }
        float xp[NX];
        {
            // all NX dot products at once, four channels at a time: every accumulator is independent
            // (rows past n and basis rows past r are zero in shared memory)
            float2 a2[NX];
#pragma unroll
            for (int j = 0; j < NX; ++j) a2[j] = make_float2(0.f, 0.f);
            const float *kfh = kf + 64 * half, *ufh = uf + 64 * half;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float2 sa = make_float2(s0[4 * q], s0[4 * q + 1]), sb = make_float2(s0[4 * q + 2], s0[4 * q + 3]);
#pragma unroll
                for (int j = 0; j < NX; ++j) {
                    const float4 v4 = *reinterpret_cast<const float4 *>(
                        (j < NPAD ? kfh + j * 128 : ufh + (j - NPAD) * 128) + 4 * q);
                    a2[j] = fma2(sa, make_float2(v4.x, v4.y), a2[j]);
                    a2[j] = fma2(sb, make_float2(v4.z, v4.w), a2[j]);
                }
            }
#pragma unroll
            for (int j = 0; j < NX; ++j) xp[j] = a2[j].x + a2[j].y;
        }
        if (half == 1)
#pragma unroll
            for (int j = 0; j < NX; j += 4)
                *reinterpret_cast<float4 *>(xex + row * NX + j) = make_float4(xp[j], xp[j + 1], xp[j + 2], xp[j + 3]);
        __syncthreads();
        const float g = *gn;
        // ---- steps 3 and 5 (the sketch): the triangular solve, one value channel per thread (warps 0-3)
        if (half == 0) {
#pragma unroll
            for (int j = 0; j < NX; j += 4) {
                const float4 o4 = *reinterpret_cast<const float4 *>(xex + row * NX + j);
                xp[j] += o4.x; xp[j + 1] += o4.y; xp[j + 2] += o4.z; xp[j + 3] += o4.w;
            }
            const QT *vt = reinterpret_cast<const QT *>(tk + W * 128 * sizeof(QT));
            float y[NPAD], acc[NPAD];
#pragma unroll
            for (int t = 0; t < NPAD; ++t) y[t] = t < n ? bv[t] * ld1(vt + t * 128 + row) - ev[t] * xp[t] : 0.f;
            // W~ = T~ y (T~ lower triangular, zero past n)
#pragma unroll
            for (int t = 0; t < NPAD; ++t) {
                float x = 0.f;
#pragma unroll
                for (int s = 0; s <= t; ++s) x = fmaf(Gm[t * as + s], y[s], x);
                acc[t] = x;
            }
            // W~ split hi | lo, as row `row` of the A operands of step 4
#pragma unroll
            for (int q = 0; q < NPAD / 4; ++q) {
                float hv[4], lv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    hv[e] = tf32_hi(acc[4 * q + e]);
                    lv[e] = acc[4 * q + e] - hv[e];
                }
                *reinterpret_cast<float4 *>(wh + sw128(row, 4 * q)) = make_float4(hv[0], hv[1], hv[2], hv[3]);
                *reinterpret_cast<float4 *>(wl + sw128(row, 4 * q)) = make_float4(lv[0], lv[1], lv[2], lv[3]);
            }
            // P = S_n^T U = g S_0^T U + sum_t w~_t (K U^T)_t
            if (P != nullptr) {
                float pp[RP];
#pragma unroll
                for (int m = 0; m < RP; ++m) pp[m] = g * xp[NPAD + m];
#pragma unroll
                for (int t = 0; t < NPAD; ++t)
                    if (t < n)
#pragma unroll
                        for (int m = 0; m < RP; ++m) pp[m] = fmaf(acc[t], kus[t * RP + m], pp[m]);
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
            fence_proxy_async();  // W~ is read by the tensor core
        }
        __syncthreads();
        // ---- step 4: D^T = W~^T K (hi and lo passes), both operands in shared memory
        if (warp == 0) {
            tc_fence_after();
#pragma unroll 1
            for (int pass = 0; pass < 2; ++pass)
#pragma unroll 1
                for (int kk = 0; kk < kc; ++kk) {
                    const uint64_t ad = smem_desc_kmajor_sw128((pass ? wl_a : wh_a) + kk * 32);
                    const uint64_t bd = smem_desc_mnmajor_sw128_32b(kbm_a + kk * 1024, npad * 128);
                    if (elect_one()) mma_ss(tbase + TM_D, ad, bd, idx_c, pass | kk);
                }
            if (elect_one()) mma_commit(bar_c);
            __syncwarp();
            ok = mbar_wait(bar_c, ph);
        }
        if (__syncthreads_or(!ok)) { failed = true; break; }
        tc_fence_after();
        // ---- step 5: S_n = g S_0 + D, back into the stage for the TMA store
#pragma unroll
        for (int j2 = 0; j2 < 2; ++j2) {
            const int pnl = 2 * half + j2;
            uint32_t d[32];
            tmem_ld32(tlane + TM_D + 32 * pnl, d);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4 *>(stage + pnl * TC_PANEL + sw128(row, 4 * q)) =
                    make_float4(fmaf(g, s0[32 * j2 + 4 * q], __uint_as_float(d[4 * q])),
                                fmaf(g, s0[32 * j2 + 4 * q + 1], __uint_as_float(d[4 * q + 1])),
                                fmaf(g, s0[32 * j2 + 4 * q + 2], __uint_as_float(d[4 * q + 2])),
                                fmaf(g, s0[32 * j2 + 4 * q + 3], __uint_as_float(d[4 * q + 3])));
        }
        tc_fence_before();
        fence_proxy_async();  // the updated state, written by these threads, is read by the TMA store
        __syncthreads();
        if (warp == 1) {
            if (elect_one()) {
                for (int p = 0; p < 4; ++p) tma_store_2d(&tmS, 32 * p, head * 128, stage + p * TC_PANEL);
                bulk_commit();
                if (ns == 1 && w + 1 < w_end) {  // one stage: refill it as soon as the store has read it
                    bulk_wait_read_all();
                    fence_proxy_async();
                    issue_state(w + 1, 0);
                }
            }
            if (ns == 1 && w + 1 < w_end) note_state(w + 1, 0);
            __syncwarp();
        }
    }

    if (failed) {  // count the give-up, then let what is in flight land (bounded)
        if (warp == 1) {
            if (elect_one()) atomicAdd(&g_update_tc_giveups, 1u);
            for (int st = 0; st < ns; ++st)
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
        if (elect_one()) bulk_wait_all();
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

// The Gated DeltaNet window update on the tensor cores, where it applies: dk = dv = 128, fp32
// state, bf16 keys (exact in TF32, so each product takes two passes), 1 <= n <= 16 tokens, and a
// shared-memory layout with at least two state stages (r <= 16 at W <= 16).
// Returns TC_NOT_APPLICABLE for other shapes (the caller then runs the CUDA-core kernel), else a
// sketchssm_status.
int launch_update_window_tc(const sketchssm_dims &d, void *S, float *P, const float *U, const void *k,
                            const void *v, const float *alpha, const float *beta, int n, cudaStream_t stream) {
    if (d.kind != SKSSM_GDN || d.dk != 128 || d.dv != 128 || d.state_dtype != SKSSM_F32) return TC_NOT_APPLICABLE;
    if (d.qkv_dtype != SKSSM_BF16 || n < 1 || n > 16 || d.W > 32 || d.r > 32) return TC_NOT_APPLICABLE;
    const int npad = 16;
    const int rp = d.r <= 4 ? 4 : d.r <= 8 ? 8 : d.r <= 16 ? 16 : 32;
    int ns = 0;  // state stages: at least two, so that the next head's state loads behind this one
    for (int cand = 3; cand >= 2 && !ns; --cand)
        if (tc_layout(cand, npad, rp, d.W).total <= TC_SMEM_LIMIT) ns = cand;
    if (!ns) return TC_NOT_APPLICABLE;
    const TcLayout L = tc_layout(ns, npad, rp, d.W);
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

    auto run = [&](auto NPc, auto RPc) -> int {
        constexpr int NP = decltype(NPc)::value, RP = decltype(RPc)::value;
        auto kern = update_window_gdn_tc<NP, RP>;
        if (allow_max_smem(reinterpret_cast<const void *>(kern)) != SKSSM_OK) return SKSSM_ERR_CUDA;
        int sms = 0;
        if (sm_count(&sms) != SKSSM_OK) return SKSSM_ERR_CUDA;
        const int grid = NH < sms ? NH : sms;
        kern<<<grid, TC_THREADS, L.total, stream>>>(map, P, U, static_cast<const __nv_bfloat16 *>(k),
                                                    static_cast<const __nv_bfloat16 *>(v), alpha, beta, d.B, d.H, d.r,
                                                    n, d.W, ns);
        return launch_status();
    };
    auto by_r = [&](auto NPc) -> int {
        if (rp == 4) return run(NPc, std::integral_constant<int, 4>());
        if (rp == 8) return run(NPc, std::integral_constant<int, 8>());
        if (rp == 16) return run(NPc, std::integral_constant<int, 16>());
        return run(NPc, std::integral_constant<int, 32>());
    };
    return by_r(std::integral_constant<int, 16>());
}

}  // namespace skssm

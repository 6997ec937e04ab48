// internal.h -- launchers behind the C ABI (not exported).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>
#include <type_traits>
#include <vector>

#include "sketchssm.h"

namespace skssm {

// Validation of a dims struct shared by every entry point: SKSSM_OK or the status to return.
int check_dims(const sketchssm_dims *d);

// Call fn(kind, dk, state type, qkv type) with compile-time constants for the
// supported combinations; returns SKSSM_ERR_DIMS / SKSSM_ERR_DTYPE otherwise.
template <typename Fn>
int dispatch(const sketchssm_dims &d, Fn &&fn) {
    auto by_q = [&](auto K, auto D, auto S) -> int {
        if (d.qkv_dtype == SKSSM_F32) return fn(K, D, S, (float *)nullptr);
        if (d.qkv_dtype == SKSSM_BF16) return fn(K, D, S, (__nv_bfloat16 *)nullptr);
        return SKSSM_ERR_DTYPE;
    };
    auto by_s = [&](auto K, auto D) -> int {
        if (d.state_dtype == SKSSM_F32) return by_q(K, D, (float *)nullptr);
        if (d.state_dtype == SKSSM_BF16) return by_q(K, D, (__nv_bfloat16 *)nullptr);
        return SKSSM_ERR_DTYPE;
    };
    auto by_d = [&](auto K) -> int {
        if (d.dk == 64) return by_s(K, std::integral_constant<int, 64>());
        if (d.dk == 128) return by_s(K, std::integral_constant<int, 128>());
        return SKSSM_ERR_DIMS;
    };
    switch (d.kind) {
        case SKSSM_MAMBA2: return by_d(std::integral_constant<int, 0>());
        case SKSSM_GDN: return by_d(std::integral_constant<int, 1>());
        case SKSSM_KDA: return by_d(std::integral_constant<int, 2>());
        default: return SKSSM_ERR_DIMS;
    }
}

inline int launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SKSSM_OK : SKSSM_ERR_CUDA;
}

int launch_update_window(const sketchssm_dims &d, void *S, float *P, const float *U, const void *k,
                         const void *v, const float *alpha, const float *beta, int n_tokens, const void *q, float *o,
                         const int *seqs, int n_seqs, int sm_share, const int *rank, cudaStream_t stream);
// The Gated DeltaNet window update on the tensor cores (update_window_tc.cu) where it applies;
// TC_NOT_APPLICABLE otherwise (the caller runs the CUDA-core kernel).
constexpr int TC_NOT_APPLICABLE = 1;
// Fewest tokens for which sketchssm_update_window takes the tensor-core form (Gated DeltaNet): its
// cost hardly depends on n, while the CUDA-core kernel's grows with n (B = 256, H = 32, r = 8: 229
// against 266 us per launch at n = 8, 358 against 303 us at n = 16).  KDA stays on the CUDA cores:
// its tensor-core form measured slower (B = 512, r = 8, n = 16: 1004 against 793 us), the per-
// channel decay products and the decayed Gram costing more on the CUDA cores than the products save.
constexpr int TC_MIN_TOKENS = 12;
int launch_update_window_tc(const sketchssm_dims &d, void *S, float *P, const float *U, const void *k,
                            const void *v, const float *alpha, const float *beta, int n_tokens, cudaStream_t stream, const void *q = nullptr,
                            float *o = nullptr);
// Counts of bounded in-kernel waits that gave up (window update, decode step); reset clears them.
int update_wait_giveups(bool reset, unsigned *count);
int update_tc_giveups(bool reset, unsigned *count);
int decode_wait_giveups(bool reset, unsigned *count);

// Opt a kernel into the largest dynamic shared memory (227 KB) on the current device.  The
// attribute belongs to the kernel's module in each device context, so it is set once per
// (kernel, device); the record is guarded for calls from several host threads, and a failed
// attempt is not recorded (the next launch tries again).
inline int allow_max_smem(const void *kern) {
    constexpr int MAX_SMEM = 227 * 1024;
    static std::mutex mu;
    static std::vector<std::pair<const void *, int>> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SKSSM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    for (const auto &e : done)
        if (e.first == kern && e.second == dev) return SKSSM_OK;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, MAX_SMEM) != cudaSuccess)
        return SKSSM_ERR_CUDA;
    done.emplace_back(kern, dev);
    return SKSSM_OK;
}

// Resident CTAs per SM of a kernel at this block size and dynamic shared memory.
// The occupancy query costs host time comparable to a short kernel, so results are
// cached per calling thread (a few entries, replaced round-robin).
inline int blocks_per_sm(const void *kern, int threads, size_t smem, int *per_sm) {
    struct Entry {
        const void *fn;
        int dev, threads;
        size_t smem;
        int per;
    };
    thread_local Entry cache[8] = {};
    thread_local int next = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SKSSM_ERR_CUDA;
    for (const Entry &e : cache)
        if (e.fn == kern && e.dev == dev && e.threads == threads && e.smem == smem) {
            *per_sm = e.per;
            return SKSSM_OK;
        }
    int per = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kern, threads, smem) != cudaSuccess) return SKSSM_ERR_CUDA;
    cache[next] = Entry{kern, dev, threads, smem, per};
    next = (next + 1) & 7;
    *per_sm = per;
    return SKSSM_OK;
}

// SM count of the current device, cached per calling thread and device.
inline int sm_count(int *sms) {
    thread_local int dev_cached = -1, count = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SKSSM_ERR_CUDA;
    if (dev != dev_cached) {
        if (cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return SKSSM_ERR_CUDA;
        dev_cached = dev;
    }
    *sms = count;
    return SKSSM_OK;
}

// Read (and optionally clear) a __device__ counter from the host.
template <typename T>
inline int read_counter(const T *symbol, bool reset, unsigned *count) {
    *count = 0;
    if (cudaMemcpyFromSymbol(count, *symbol, sizeof(unsigned)) != cudaSuccess) return SKSSM_ERR_CUDA;
    if (reset && *count) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(*symbol, &zero, sizeof(zero)) != cudaSuccess) return SKSSM_ERR_CUDA;
    }
    return SKSSM_OK;
}
int launch_replay_decode(const sketchssm_dims &d, const void *S, const void *q, const void *k, const void *v,
                         const float *alpha, const float *beta, int j, float *o, cudaStream_t stream);
int launch_decode_wy(const sketchssm_dims &d, const float *P, const float *R, const void *q, const void *k,
                     const void *v, const float *alpha, const float *beta, int j, float *G, float *o,
                     cudaStream_t stream);
int launch_fullread(const sketchssm_dims &d, void *S, const void *q, const void *k, const void *v,
                    const float *alpha, const float *beta, float *o, cudaStream_t stream);
int launch_decode_step(const sketchssm_dims &d, const float *P, const float *R, const void *q, const void *k,
                       const void *v, const float *alpha, const float *beta, int j, const int *jv, int sm_share,
                       const int *rank, float *o, cudaStream_t stream);

size_t calibrate_workspace_bytes(const sketchssm_dims &d, int Nq, int Ns);
int launch_rank_basis(const sketchssm_dims &d, int r_avg, const double *lam, float *U, float *R, int *rank,
                      cudaStream_t stream);
int launch_calibrate(const sketchssm_dims &d, const float *q_cal, int Nq, const void *S_cal, int Ns,
                     double ridge, float *U, float *R, void *workspace, cudaStream_t stream, double *lam = nullptr);
int launch_calibrate_heads(const sketchssm_dims &d, const float *q_cal, int Nq, const void *S_cal,
                           int Ns, double ridge, float *U, float *R, void *workspace, int h0, int hc,
                           cudaStream_t stream, double *lam = nullptr);

}  // namespace skssm

// calibrate.cu -- offline calibration of the basis U and coefficient map R (fp64).
//
// SketchSSM (arXiv 2609.33051v1), Abstract: queries are approximated in a
// low-rank, state-weighted way on basis vectors that can be fixed offline;
// agihunt digest, bullet "Core idea".  Per head h:
//   G = (1/Ns) sum_s S_s S_s^T  (+ ridge tr(G)/dk I)    state weighting
//   C = (1/Nq) sum_n q_n q_n^T                          query second moment
// The averaged squared read error E ||S^T (q - U R q)||^2 = tr(C (I-UR)^T G (I-UR))
// is minimised by R = (U^T G U)^-1 U^T G for a fixed U, and over U by the span
// L^-T V_r, where G = L L^T (Cholesky) and V_r holds the eigenvectors of
// L^T C L with the r largest eigenvalues.  With U = L^-T V_r one has
// U^T G U = I, hence R = U^T G = V_r^T L^T and R U = I.
//
// Kernels (all fp64, offline, not on the decode path):
//   gram_kernel   G and C as sums of outer products, 32x32 output tiles
//   basis_kernel  one CTA per head: Cholesky in shared memory, A = L^T C L,
//                 cyclic Jacobi with a round-robin pair ordering (dk/2 disjoint
//                 rotations per round, at most 40 sweeps), top-r selection,
//                 back substitution for U, and R = V_r^T L^T.
// U is written as basis rows, U_rows[h][m][i] = U[i][m], like R.
// Workspace (caller-owned): G/L, C, T/V, each [H][dk][dk] fp64.
//
// Query PCA (the unweighted basis the state weighting is measured against): no
// calibration states, G = I, so L = I, U = V_r holds the top-r eigenvectors of
// C and R = V_r^T is the orthogonal projection onto their span.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace skssm {

// out[h][i][jj] = scale * sum_m X_h[m][i] X_h[m][jj], where row m of head h
// starts at X + h*sh + (m / mper)*sb + (m % mper)*DK.
template <typename T, int DK>
__global__ void __launch_bounds__(256)
gram_kernel(const T *__restrict__ X, size_t sh, size_t sb, int mper, int M, double scale,
            double *__restrict__ out) {
    constexpr int TB = 32, NT = DK / TB;
    __shared__ double xa[TB][TB + 1], xb[TB][TB + 1];
    const int h = blockIdx.y;
    const int ti = blockIdx.x / NT, tj = blockIdx.x % NT;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // 16 x 16 threads, 2 x 2 outputs each
    double acc[2][2] = {{0, 0}, {0, 0}};
    const T *Xh = X + (size_t)h * sh;
    for (int m0 = 0; m0 < M; m0 += TB) {
        for (int idx = threadIdx.x; idx < TB * TB; idx += 256) {
            const int mm = idx / TB, ii = idx % TB;
            const int m = m0 + mm;
            double va = 0.0, vb = 0.0;
            if (m < M) {
                const T *row = Xh + (size_t)(m / mper) * sb + (size_t)(m % mper) * DK;
                va = (double)ld1(row + ti * TB + ii);
                vb = (double)ld1(row + tj * TB + ii);
            }
            xa[mm][ii] = va;
            xb[mm][ii] = vb;
        }
        __syncthreads();
#pragma unroll 4
        for (int mm = 0; mm < TB; ++mm) {
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) acc[a][b] += xa[mm][ty * 2 + a] * xb[mm][tx * 2 + b];
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b)
            out[((size_t)h * DK + ti * TB + ty * 2 + a) * DK + tj * TB + tx * 2 + b] = acc[a][b] * scale;
}

constexpr int BASIS_THREADS = 512;
constexpr int JACOBI_MAX_SWEEPS = 40;

__device__ double block_sum(double x, double *red) {
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = x;
    __syncthreads();
    double t = 0.0;
    for (int i = 0; i < BASIS_THREADS / 32; ++i) t += red[i];
    return t;
}

template <int DK>
__global__ void __launch_bounds__(BASIS_THREADS)
basis_kernel(double *__restrict__ Gw, const double *__restrict__ Cw, double *__restrict__ Tw, int r,
             double ridge, float *__restrict__ U, float *__restrict__ R, double *__restrict__ lam) {
    constexpr int LD = DK + 1;  // padded row stride of the shared matrix
    extern __shared__ double sm[];
    double *A = sm;                   // [DK][LD]
    double *cs = A + DK * LD;         // [DK/2][2] rotation cosines / sines
    double *red = cs + DK;            // [32] reduction scratch
    int *sel = reinterpret_cast<int *>(red + 32);  // [DK] selected eigenvector indices
    int *flag = sel + DK;             // [1] any rotation applied this sweep
    const int h = blockIdx.x, tid = threadIdx.x;
    double *Gh = Gw + (size_t)h * DK * DK;  // G in, L out
    const double *Ch = Cw + (size_t)h * DK * DK;
    double *Th = Tw + (size_t)h * DK * DK;  // T = C L, then V

    // 1. G + ridge (tr G / dk) I into shared memory
    double tr = 0.0;
    for (int i = tid; i < DK; i += BASIS_THREADS) tr += Gh[(size_t)i * DK + i];
    tr = block_sum(tr, red);
    const double shift = ridge * tr / DK;
    for (int idx = tid; idx < DK * DK; idx += BASIS_THREADS) {
        const int i = idx / DK, jj = idx % DK;
        A[i * LD + jj] = Gh[idx] + (i == jj ? shift : 0.0);
    }
    __syncthreads();

    // 2. Cholesky, right-looking, lower triangle in place
    for (int kk = 0; kk < DK; ++kk) {
        if (tid == 0) {
            const double p = A[kk * LD + kk];
            A[kk * LD + kk] = sqrt(p > 0.0 ? p : 1e-300);
        }
        __syncthreads();
        const double piv = A[kk * LD + kk];
        for (int i = kk + 1 + tid; i < DK; i += BASIS_THREADS) A[i * LD + kk] /= piv;
        __syncthreads();
        const int rem = DK - kk - 1;
        for (int idx = tid; idx < rem * rem; idx += BASIS_THREADS) {
            const int i = kk + 1 + idx / rem, jj = kk + 1 + idx % rem;
            if (jj <= i) A[i * LD + jj] -= A[i * LD + kk] * A[jj * LD + kk];
        }
        __syncthreads();
    }
    for (int idx = tid; idx < DK * DK; idx += BASIS_THREADS) {
        const int i = idx / DK, jj = idx % DK;
        Gh[idx] = jj <= i ? A[i * LD + jj] : 0.0;  // L, row-major
    }
    __syncthreads();

    // 3. T = C L (global), then A = L^T T (shared), symmetrised
    for (int idx = tid; idx < DK * DK; idx += BASIS_THREADS) {
        const int i = idx / DK, jj = idx % DK;
        double acc = 0.0;
        for (int k = jj; k < DK; ++k) acc += Ch[(size_t)i * DK + k] * A[k * LD + jj];
        Th[idx] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < DK * DK; idx += BASIS_THREADS) {
        const int i = idx / DK, jj = idx % DK;
        double acc = 0.0;
        for (int k = i; k < DK; ++k) acc += Gh[(size_t)k * DK + i] * Th[(size_t)k * DK + jj];
        A[i * LD + jj] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < DK * DK; idx += BASIS_THREADS) {
        const int i = idx / DK, jj = idx % DK;
        if (jj > i) {
            const double m = 0.5 * (A[i * LD + jj] + A[jj * LD + i]);
            A[i * LD + jj] = m;
            A[jj * LD + i] = m;
        }
    }
    for (int idx = tid; idx < DK * DK; idx += BASIS_THREADS) Th[idx] = (idx / DK == idx % DK) ? 1.0 : 0.0;
    __syncthreads();

    // 4. cyclic Jacobi, round-robin ordering
    for (int sweep = 0; sweep < JACOBI_MAX_SWEEPS; ++sweep) {
        if (tid == 0) *flag = 0;
        __syncthreads();
        for (int rnd = 0; rnd < DK - 1; ++rnd) {
            auto pos = [&](int i) { return i == 0 ? 0 : 1 + (i - 1 + rnd) % (DK - 1); };
            for (int k = tid; k < DK / 2; k += BASIS_THREADS) {
                int p = pos(k), q = pos(DK - 1 - k);
                if (p > q) { const int t = p; p = q; q = t; }
                const double app = A[p * LD + p], aqq = A[q * LD + q], apq = A[p * LD + q];
                double c = 1.0, s = 0.0;
                if (fabs(apq) > 1e-300 && fabs(apq) > 1e-18 * sqrt(fabs(app * aqq))) {
                    const double tau = (aqq - app) / (2.0 * apq);
                    double t;
                    if (fabs(tau) > 1e150) t = 0.5 / tau;
                    else t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
                    c = 1.0 / sqrt(1.0 + t * t);
                    s = t * c;
                    *flag = 1;
                }
                cs[2 * k] = c;
                cs[2 * k + 1] = s;
            }
            __syncthreads();
            for (int idx = tid; idx < (DK / 2) * DK; idx += BASIS_THREADS) {  // A <- A J
                const int k = idx / DK, i = idx % DK;
                int p = pos(k), q = pos(DK - 1 - k);
                if (p > q) { const int t = p; p = q; q = t; }
                const double c = cs[2 * k], s = cs[2 * k + 1];
                const double aip = A[i * LD + p], aiq = A[i * LD + q];
                A[i * LD + p] = c * aip - s * aiq;
                A[i * LD + q] = s * aip + c * aiq;
            }
            __syncthreads();
            for (int idx = tid; idx < (DK / 2) * DK; idx += BASIS_THREADS) {  // A <- J^T A, V <- V J
                const int k = idx / DK, i = idx % DK;
                int p = pos(k), q = pos(DK - 1 - k);
                if (p > q) { const int t = p; p = q; q = t; }
                const double c = cs[2 * k], s = cs[2 * k + 1];
                const double api = A[p * LD + i], aqi = A[q * LD + i];
                A[p * LD + i] = c * api - s * aqi;
                A[q * LD + i] = s * api + c * aqi;
                const double vip = Th[(size_t)i * DK + p], viq = Th[(size_t)i * DK + q];
                Th[(size_t)i * DK + p] = c * vip - s * viq;
                Th[(size_t)i * DK + q] = s * vip + c * viq;
            }
            __syncthreads();
        }
        double off = 0.0, dia = 0.0;
        for (int idx = tid; idx < DK * DK; idx += BASIS_THREADS) {
            const int i = idx / DK, jj = idx % DK;
            const double a = A[i * LD + jj];
            if (i == jj) dia += a * a; else off += a * a;
        }
        off = block_sum(off, red);
        dia = block_sum(dia, red);
        const int any = *flag;
        __syncthreads();
        if (!any || off <= 1e-30 * dia) break;
    }

    // 5. the r largest eigenvalues, ties by index (sel starts as the identity so
    //    that a non-finite spectrum still selects valid columns)
    for (int i = tid; i < DK; i += BASIS_THREADS) sel[i] = i;
    __syncthreads();
    for (int i = tid; i < DK; i += BASIS_THREADS) {
        const double li = A[i * LD + i];
        int rank = 0;
        for (int jj = 0; jj < DK; ++jj) {
            const double lj = A[jj * LD + jj];
            rank += (lj > li) || (lj == li && jj < i);
        }
        if (rank < r) sel[rank] = i;
    }
    __syncthreads();

    // the selected eigenvalues, descending (the ranked calibration compares them across heads)
    if (lam != nullptr)
        for (int m = tid; m < r; m += BASIS_THREADS) lam[(size_t)h * r + m] = A[sel[m] * LD + sel[m]];
    __syncthreads();

    // 6. U = L^-T V_r (back substitution, one column per thread), R = V_r^T L^T
    double *X = A;  // reuse: [r][DK]
    for (int m = tid; m < r; m += BASIS_THREADS) {
        const int col = sel[m];
        for (int i = DK - 1; i >= 0; --i) {
            double acc = Th[(size_t)i * DK + col];
            for (int k = i + 1; k < DK; ++k) acc -= Gh[(size_t)k * DK + i] * X[m * DK + k];
            X[m * DK + i] = acc / Gh[(size_t)i * DK + i];
        }
    }
    __syncthreads();
    for (int idx = tid; idx < DK * r; idx += BASIS_THREADS) {
        const int m = idx / DK, i = idx % DK;
        U[((size_t)h * r + m) * DK + i] = (float)X[m * DK + i];
    }
    for (int idx = tid; idx < r * DK; idx += BASIS_THREADS) {
        const int m = idx / DK, i = idx % DK;
        const int col = sel[m];
        double acc = 0.0;
        for (int k = 0; k <= i; ++k) acc += Th[(size_t)k * DK + col] * Gh[(size_t)i * DK + k];
        R[((size_t)h * r + m) * DK + i] = (float)acc;
    }
}

// Per-head ranks under an average-rank budget: the budget takes the largest of all
// heads' selected eigenvalues together (ties: lower head, then lower index), at most
// r_max per head; head h's rank is the number of its values taken.  One CTA.
__global__ void __launch_bounds__(1024)
allocate_ranks_kernel(const double *__restrict__ lam, int H, int rmax, int budget, int *__restrict__ rank) {
    for (int h = threadIdx.x; h < H; h += blockDim.x) rank[h] = 0;
    __syncthreads();
    const int n = H * rmax;
    for (int c = threadIdx.x; c < n; c += blockDim.x) {
        const double lc = lam[c];
        int pos = 0;
        for (int c2 = 0; c2 < n; ++c2) {
            const double l2 = lam[c2];
            pos += (l2 > lc) || (l2 == lc && c2 < c);
        }
        if (pos < budget) atomicAdd(&rank[c / rmax], 1);
    }
}

// Rows m >= rank[h] of head h's basis rows U [H][r][dk] and map R [H][r][dk] set to zero.
__global__ void mask_ranks_kernel(float *__restrict__ U, float *__restrict__ R, const int *__restrict__ rank, int H,
                                  int r, int dk) {
    const size_t n = (size_t)H * r * dk;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < n; idx += (size_t)gridDim.x * blockDim.x) {
        const int m = (int)((idx / dk) % r), h = (int)(idx / ((size_t)r * dk));
        if (m >= rank[h]) {
            U[idx] = 0.f;
            R[idx] = 0.f;
        }
    }
}

int launch_rank_basis(const sketchssm_dims &d, int r_avg, const double *lam, float *U, float *R, int *rank,
                      cudaStream_t stream) {
    allocate_ranks_kernel<<<1, 1024, 0, stream>>>(lam, d.H, d.r, d.H * r_avg, rank);
    if (launch_status() != SKSSM_OK) return SKSSM_ERR_CUDA;
    const size_t n = (size_t)d.H * d.r * d.dk;
    const int grid = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    mask_ranks_kernel<<<grid, 256, 0, stream>>>(U, R, rank, d.H, d.r, d.dk);
    return launch_status();
}

// G[h] = I for every head (the query-PCA calibration's state weight).
__global__ void identity_kernel(double *__restrict__ G, int dk, size_t n) {
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        const int ij = (int)(e % ((size_t)dk * dk));
        G[e] = (ij / dk == ij % dk) ? 1.0 : 0.0;
    }
}

size_t calibrate_workspace_bytes(const sketchssm_dims &d, int, int) {
    return 3 * (size_t)d.H * d.dk * d.dk * sizeof(double);
}

template <int DK>
static size_t basis_smem() {
    return (size_t)DK * (DK + 1) * sizeof(double) + DK * sizeof(double) + 32 * sizeof(double) +
           (DK + 4) * sizeof(int);
}

int launch_calibrate(const sketchssm_dims &d, const float *q_cal, int Nq, const void *S_cal, int Ns,
                     double ridge, float *U, float *R, void *workspace, cudaStream_t stream, double *lam) {
    return launch_calibrate_heads(d, q_cal, Nq, S_cal, Ns, ridge, U, R, workspace, 0, d.H, stream, lam);
}

// Heads [h0, h0 + hc) only, with a workspace sized for hc heads: G and C (fp64 Gram
// kernels), then the per-head basis, with every head-indexed pointer offset to h0.
// S_cal == nullptr selects G = I (query PCA; ridge is then irrelevant).
int launch_calibrate_heads(const sketchssm_dims &d, const float *q_cal, int Nq, const void *S_cal,
                           int Ns, double ridge, float *U, float *R, void *workspace, int h0, int hc,
                           cudaStream_t stream, double *lam) {
    double *G = static_cast<double *>(workspace);
    double *C = G + (size_t)hc * d.dk * d.dk;
    double *T = C + (size_t)hc * d.dk * d.dk;
    auto run = [&](auto DKc) -> int {
        constexpr int DK = decltype(DKc)::value;
        const dim3 ggrid((DK / 32) * (DK / 32), hc);
        const size_t sh = (size_t)d.dv * DK, sb = (size_t)d.H * d.dv * DK;
        const size_t s_off = (size_t)h0 * d.dv * DK;
        if (!S_cal) {
            const size_t n = (size_t)hc * DK * DK;
            identity_kernel<<<(int)((n + 255) / 256 < 2048 ? (n + 255) / 256 : 2048), 256, 0, stream>>>(G, DK, n);
        } else if (d.state_dtype == SKSSM_F32)
            gram_kernel<float, DK><<<ggrid, 256, 0, stream>>>(static_cast<const float *>(S_cal) + s_off, sh,
                                                              sb, d.dv, Ns * d.dv, 1.0 / Ns, G);
        else
            gram_kernel<__nv_bfloat16, DK><<<ggrid, 256, 0, stream>>>(
                static_cast<const __nv_bfloat16 *>(S_cal) + s_off, sh, sb, d.dv, Ns * d.dv, 1.0 / Ns, G);
        if (launch_status() != SKSSM_OK) return SKSSM_ERR_CUDA;
        gram_kernel<float, DK><<<ggrid, 256, 0, stream>>>(q_cal + (size_t)h0 * Nq * DK, (size_t)Nq * DK, 0,
                                                          Nq, Nq, 1.0 / Nq, C);
        if (launch_status() != SKSSM_OK) return SKSSM_ERR_CUDA;
        const size_t smem = basis_smem<DK>();
        if (cudaFuncSetAttribute(basis_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return SKSSM_ERR_CUDA;
        basis_kernel<DK><<<hc, BASIS_THREADS, smem, stream>>>(G, C, T, d.r, ridge,
                                                               U + (size_t)h0 * DK * d.r,
                                                               R + (size_t)h0 * d.r * DK,
                                                               lam ? lam + (size_t)h0 * d.r : nullptr);
        return launch_status();
    };
    if (d.dk == 64) return run(std::integral_constant<int, 64>());
    if (d.dk == 128) return run(std::integral_constant<int, 128>());
    return SKSSM_ERR_DIMS;
}

}  // namespace skssm

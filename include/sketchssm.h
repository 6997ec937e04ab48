/*
 * sketchssm.h -- C ABI of the SketchSSM windowed linear-attention decode for
 * NVIDIA B200 (sm_100a).
 *
 * Method: "SketchSSM: Write to the Full State, Read from a Compact Sketch"
 * (arXiv 2609.33051v1), Abstract; agihunt digest of the same paper, bullets
 * "Core idea", "Mechanism details" and "Error control".  Keys and values are
 * buffered for a window of W decode steps (the ReplaySSM buffering the abstract
 * builds on).  Once per window one kernel reads each head's full recurrent
 * state S, applies the buffered tokens exactly and, in the same pass, refreshes
 * a compact sketch P = S^T U against an offline basis U.  Each decode step in
 * the window reads only the sketch: it carries its query back to the
 * window-start state through the buffered tokens (q~), adds the exact
 * contribution of those tokens, and reconstructs the state part as P (R q~).
 * Approximation error never enters S.
 *
 * Recurrences (per head; S is dk x dv, i a key channel, c a value channel):
 *   SKSSM_MAMBA2  S <- a S + k v^T                     a scalar per token/head
 *   SKSSM_GDN     S <- a (I - b k k^T) S + b k v^T     a, b scalars
 *   SKSSM_KDA     S <- (I - b k k^T) diag(a) S + b k v^T   a per key channel
 * Read: o = S^T q after the step's own token has been applied.
 *
 * ---------------------------------------------------------------------------
 * Conventions shared by every entry point
 *   - Every array pointer is DEVICE memory owned by the caller, on the device
 *     that is current for the calling thread, densely packed (C order), and
 *     16-byte aligned unless stated otherwise.  The library keeps no pointer
 *     after a call returns and allocates no memory.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous on it; kernel-side faults surface at the caller's next
 *     synchronisation.
 *   - Every call validates its arguments on the host before launching anything
 *     and returns SKSSM_OK (0) or a negative sketchssm_status; on error nothing
 *     was launched and no memory was touched.
 *   - Storage layouts (N = B*H heads, flat head index n = b*H + h):
 *       S      [B][H][dv][dk]  state, stored transposed: row c holds column c of
 *                              S, i.e. S_T[n][c][i] = S[i][c]; dtype state_dtype
 *       P      [B][H][dv][r]   fp32 sketch, P[n][c][m] = sum_i S[i][c] U[i][m]
 *       U      [H][r][dk]      fp32 basis stored as rows: U_rows[h][m][i] = U[i][m]
 *                              (the dk x r basis of head h, shared by all b)
 *       R      [H][r][dk]      fp32 coefficient map, c = R q~
 *       window buffer, head-major (a head's W slots are contiguous), slot t =
 *       token t of the window:
 *       k      [B][H][W][dk]   qkv_dtype
 *       v      [B][H][W][dv]   qkv_dtype
 *       alpha  [B][H][W]       fp32 decay (SKSSM_KDA: [B][H][W][dk]); 4-byte aligned
 *       beta   [B][H][W]       fp32 (ignored, may be NULL, for SKSSM_MAMBA2); 4-byte aligned
 *       q      [B][H][dk]      qkv_dtype, the current step's query
 *       o      [B][H][dv]      fp32 output
 *   - Supported sizes: dk in {64, 128}; dv in {64, 128}; 1 <= r <= 32 or r == dk;
 *     1 <= W <= 64; B >= 1, H >= 1, B*H < 2^31.  Other sizes: SKSSM_ERR_DIMS.
 * ---------------------------------------------------------------------------
 */
#ifndef SKETCHSSM_H
#define SKETCHSSM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { SKSSM_MAMBA2 = 0, SKSSM_GDN = 1, SKSSM_KDA = 2 } sketchssm_kind;
typedef enum { SKSSM_F32 = 0, SKSSM_BF16 = 1 } sketchssm_dtype;

typedef enum {
    SKSSM_OK = 0,
    SKSSM_ERR_NULL = -1,      /* a required pointer is NULL */
    SKSSM_ERR_DIMS = -2,      /* unsupported kind / sizes */
    SKSSM_ERR_RANGE = -3,     /* j, n_tokens, Nq or Ns out of range */
    SKSSM_ERR_ALIGN = -4,     /* a pointer breaks its alignment rule */
    SKSSM_ERR_DTYPE = -5,     /* unsupported storage dtype */
    SKSSM_ERR_CUDA = -6,      /* a CUDA runtime call or launch failed */
    SKSSM_ERR_WORKSPACE = -7  /* workspace missing or too small */
} sketchssm_status;

typedef struct sketchssm_dims {
    int32_t kind;        /* sketchssm_kind */
    int32_t B, H;        /* sequences in the batch, heads per sequence */
    int32_t dk, dv;      /* key (state rows) and value (state columns) widths */
    int32_t r;           /* sketch rank */
    int32_t W;           /* window length: slots in the token buffer */
    int32_t state_dtype; /* storage of S: SKSSM_F32 or SKSSM_BF16 */
    int32_t qkv_dtype;   /* storage of q, k, v: SKSSM_F32 or SKSSM_BF16 */
} sketchssm_dims;

/* Human-readable text of a status code (static string, never NULL). */
const char *sketchssm_status_string(int status);

/* ABI version of this library: major * 10000 + minor * 100 + patch. */
int sketchssm_version(void);

/*
 * sketchssm_update_window -- the once-per-window state update and sketch refresh.
 * Defines: SketchSSM abstract (one full-state read per state update precomputes
 * the basis outputs into the sketch); digest bullet "Error control" (the same
 * kernel updates the full state and refreshes the sketch).
 * For every head: apply buffered tokens t = 0 .. n_tokens-1 of the window
 * buffer to S, in order, exactly (fp32 arithmetic); store S (rounded to
 * state_dtype, nearest-even, for SKSSM_BF16); then write P = S_stored^T U.
 * Any decay values are accepted, including 0 (a state reset) and windows whose
 * decay product underflows or exceeds the fp32 range: such a head is updated
 * token by token instead of through the running decay scale.
 * n_tokens = 0 is a sketch refresh only (S is read, not written).
 * Implementation: SKSSM_GDN with dk = dv = 128, fp32 state, bf16 q/k/v, r <= 16
 * and 12 <= n_tokens <= 16 runs the chunked form on the tensor cores (as
 * sketchssm_update_window_tc, below); every other case runs the token-by-token
 * kernel on the CUDA cores.  Both give the recurrence's result to fp32 rounding.
 *   S        in/out [B][H][dv][dk] state_dtype
 *   P        out    [B][H][dv][r] fp32; NULL: no sketch refresh (a plain buffered
 *            state update, the window-end write of the ReplaySSM-style path)
 *   U        in     [H][r][dk] fp32 (basis rows); may be NULL when P is
 *   k, v, alpha, beta  in: window buffer slots 0..n_tokens-1 (NULL allowed when
 *            n_tokens == 0; beta NULL allowed for SKSSM_MAMBA2)
 * Errors: ERR_NULL, ERR_DIMS, ERR_DTYPE, ERR_RANGE (n_tokens < 0 or > W),
 * ERR_ALIGN, ERR_CUDA.
 */
int sketchssm_update_window(const sketchssm_dims *dims, void *S, float *P, const float *U,
                            const void *k, const void *v, const float *alpha, const float *beta,
                            int n_tokens, void *stream);

/*
 * sketchssm_update_window_read -- the window update with the exact read of the
 * window's last step fused in.  The update already holds every head's updated
 * state on chip (SketchSSM abstract: one full-state read per state update), so
 * the read of the step whose token is the last one applied, o = S^T q, costs no
 * state traffic; that step then needs no sketch read and has no approximation
 * error.  Everything sketchssm_update_window does, plus, per head:
 *     o = S_n^T q   from the updated state in fp32, before the storage rounding
 *                   (as the full-read step reads it)
 *   q   in  [B][H][dk] qkv_dtype, the query of the step whose token is slot n_tokens-1
 *   o   out [B][H][dv] fp32
 * n_tokens = 0 reads the unchanged state.
 * Errors: as sketchssm_update_window, and ERR_NULL / ERR_ALIGN for q and o.
 */
int sketchssm_update_window_read(const sketchssm_dims *dims, void *S, float *P, const float *U,
                                 const void *k, const void *v, const float *alpha, const float *beta,
                                 int n_tokens, const void *q, float *o, void *stream);

/*
 * sketchssm_update_window_tc -- sketchssm_update_window for the delta rules with the
 * window's tokens applied in chunked (WY) form, both products on the tensor cores
 * (tcgen05.mma kind::tf32): [X | S_0^T U] = S_0^T [K; U] with the state split into
 * its TF32 part and remainder, and the rank-n state increment W~^T K with W~ split
 * the same way, so the result matches the recurrence to fp32 rounding (Gated
 * DeltaNet keys are exact in TF32; KDA's keys carry the per-channel decay products
 * and are split too).  The state moves by TMA tiled copies.  Applies to SKSSM_GDN
 * (r <= 16) and SKSSM_KDA (r <= 8) with dk = dv = 128, fp32 state, bf16 q/k/v and
 * 1 <= n_tokens <= 16; other sizes return SKSSM_ERR_DIMS.  For KDA it is an
 * alternative, not the default: it measured slower than the CUDA-core kernel.  sketchssm_update_window takes this path by itself
 * for 12 <= n_tokens <= 16; this entry forces it for any n_tokens >= 1 (below 12
 * tokens the CUDA-core kernel is faster).
 * Arguments and other errors as sketchssm_update_window (n_tokens >= 1).
 */
int sketchssm_update_window_tc(const sketchssm_dims *dims, void *S, float *P, const float *U,
                               const void *k, const void *v, const float *alpha, const float *beta,
                               int n_tokens, void *stream);

/*
 * sketchssm_decode_step -- one decode step inside a window, reading only the sketch.
 * Defines: SketchSSM abstract (each decode step combines the sketch vectors with
 * query-dependent coefficients instead of reading the full state); digest
 * bullet "Mechanism details" (a query that is a combination of basis vectors
 * has as output the same combination of the stored outputs).
 * Step j of the window: tokens 0..j-1 of the buffer are not yet in the state
 * whose sketch is P (token j-1 is this step's own token).  Per head:
 *     w <- q;  o_buf <- 0
 *     for t = j-1 down to 0:  x = k_t . w;  s = b_t x (b = 1 for Mamba-2);
 *                             o_buf += s v_t;  w <- M_t^T w
 *         (M_t^T w: Mamba-2 a_t w; GDN a_t (w - s k_t); KDA a_t (.) (w - s k_t))
 *     o = P (R w) + o_buf
 *   P in [B][H][dv][r];  R in [H][r][dk];  q in [B][H][dk];
 *   k, v, alpha, beta in: window buffer slots 0..j-1;  o out [B][H][dv] fp32.
 * Errors: ERR_NULL, ERR_DIMS, ERR_DTYPE, ERR_RANGE (j < 1 or j > W), ERR_ALIGN,
 * ERR_CUDA.
 */
int sketchssm_decode_step(const sketchssm_dims *dims, const float *P, const float *R,
                          const void *q, const void *k, const void *v, const float *alpha,
                          const float *beta, int j, float *o, void *stream);

/*
 * sketchssm_decode_step_seq -- sketchssm_decode_step with a step index per
 * sequence.  In serving, sequences reach the ends of their windows at different
 * decode steps (they start at different times); j_seq[b] is sequence b's step
 * within its own window, 1..W, or 0 for a sequence that takes no sketch step now
 * (for instance, its window ends at this step and sketchssm_update_window_seqs
 * reads it exactly).  Heads of a sequence with j_seq[b] == 0 keep their o.
 *   j_seq  in device [B] int32 (4-byte aligned).  A value outside 0..W is counted
 *          by sketchssm_device_error_count and that sequence is skipped.
 *   sm_share  0: use the whole GPU; n > 0: at most n CTAs per SM, leaving room for a
 *          kernel that runs at the same time on another stream (the window updates
 *          of other sequences).
 * Other arguments as sketchssm_decode_step.
 * Errors: ERR_NULL, ERR_DIMS, ERR_DTYPE, ERR_RANGE (sm_share < 0), ERR_ALIGN, ERR_CUDA.
 */
int sketchssm_decode_step_seq(const sketchssm_dims *dims, const float *P, const float *R, const void *q,
                              const void *k, const void *v, const float *alpha, const float *beta,
                              const int32_t *j_seq, int sm_share, float *o, void *stream);

/*
 * sketchssm_update_window_seqs -- the window update (sketchssm_update_window, or
 * with q and o sketchssm_update_window_read) for the n_seqs sequences listed in
 * seqs only: every head of each listed sequence; the other sequences' state,
 * sketch and output are not touched.  Sequences whose windows end at this step
 * are updated while the others take sketch steps (sketchssm_decode_step_seq on
 * another stream, both with sm_share > 0, so that the two kernels share the GPU).
 *   seqs   in device [n_seqs] int32 sequence indices (4-byte aligned), 0 <= n_seqs <= B;
 *          an index outside 0..B-1 is counted by sketchssm_device_error_count and
 *          skipped.
 *   q, o   both NULL (no read) or both given (the exact read, as
 *          sketchssm_update_window_read).
 *   P, U   as sketchssm_update_window (P NULL: no sketch refresh).
 *   sm_share  as sketchssm_decode_step_seq.
 * Errors: ERR_NULL, ERR_DIMS, ERR_DTYPE, ERR_RANGE (n_tokens, n_seqs, sm_share), ERR_ALIGN,
 * ERR_CUDA.
 */
int sketchssm_update_window_seqs(const sketchssm_dims *dims, void *S, float *P, const float *U,
                                 const void *k, const void *v, const float *alpha, const float *beta,
                                 int n_tokens, const int32_t *seqs, int n_seqs, const void *q, float *o,
                                 int sm_share, void *stream);

/*
 * sketchssm_fullread_decode -- the baseline: one decode step with a full-state
 * read, as a standard serving engine does it (SketchSSM abstract: the vLLM
 * decode path it is compared with; digest bullet "Background": the full
 * recurrent state is read at every decode step).  Per head: S <- M S + b k v^T with this step's token,
 * S stored back (state_dtype), o = S^T q from the updated fp32 values.
 *   S in/out [B][H][dv][dk];  q, k in [B][H][dk];  v in [B][H][dv];
 *   alpha in [B][H] (KDA [B][H][dk]);  beta in [B][H] (NULL for Mamba-2);
 *   o out [B][H][dv] fp32.  (One window slot is a valid token argument.)
 * Errors: ERR_NULL, ERR_DIMS, ERR_DTYPE, ERR_ALIGN, ERR_CUDA.
 */
int sketchssm_fullread_decode(const sketchssm_dims *dims, void *S, const void *q, const void *k,
                              const void *v, const float *alpha, const float *beta, float *o,
                              void *stream);

/*
 * sketchssm_update_window_ranked, sketchssm_decode_step_ranked -- sketchssm_update_window
 * and sketchssm_decode_step for a basis with a rank per head (as
 * sketchssm_calibrate_basis_ranked makes it: U and R [H][r][dk] with rows
 * m >= rank[h] zero).  The results equal the plain calls' on the same U and R;
 * the window update skips the refresh arithmetic of the zero rows (and writes
 * zero there), and the decode step reads the sketch columns m >= rank[h] only
 * when rank[h] > 8, so that a head of rank <= 8 with r = 16 reads one 32-byte
 * sector of each sketch row instead of two.
 *   rank  in device [H] int32 (4-byte aligned); a value outside 0..r is counted by
 *         sketchssm_device_error_count and clamped.
 * Other arguments and errors as sketchssm_update_window / sketchssm_decode_step.
 */
int sketchssm_update_window_ranked(const sketchssm_dims *dims, void *S, float *P, const float *U,
                                   const int32_t *rank, const void *k, const void *v, const float *alpha,
                                   const float *beta, int n_tokens, void *stream);
int sketchssm_decode_step_ranked(const sketchssm_dims *dims, const float *P, const float *R,
                                 const int32_t *rank, const void *q, const void *k, const void *v,
                                 const float *alpha, const float *beta, int j, float *o, void *stream);

/*
 * sketchssm_decode_step_wy -- sketchssm_decode_step for the delta rules (GDN, KDA)
 * with the backward pass in WY / T-matrix form: the window's buffered keys have a
 * Gram matrix (with the decays between them) that does not change while the
 * window fills, so each step adds one column to a per-head buffer and solves a
 * small triangular system against it instead of carrying the query back one
 * token at a time.  Same results as sketchssm_decode_step (up to fp32 rounding).
 *   G   in/out device [B][H][W][W4] fp32, W4 = W rounded up to a multiple of 4,
 *       16-byte aligned, owned by the caller.  Step j writes row j-1 (entries
 *       t < j-1) and reads rows 1..j-2, so within a window the steps must run in
 *       order j = 1, 2, ..., each after the previous one (the same stream); the
 *       buffer needs no initialisation and no reset between windows.
 * SKSSM_MAMBA2 has no delta chain: the call is sketchssm_decode_step (G unused,
 * may be NULL).  Requires W <= 32 (ERR_DIMS otherwise).
 * Other arguments and errors as sketchssm_decode_step.
 */
int sketchssm_decode_step_wy(const sketchssm_dims *dims, const float *P, const float *R, const void *q,
                             const void *k, const void *v, const float *alpha, const float *beta, int j,
                             float *G, float *o, void *stream);

/*
 * sketchssm_replay_decode_step -- the second baseline: one decode step of a
 * buffered window that reads the full window-start state (ReplaySSM, as the
 * SketchSSM abstract and the digest bullet "Background" describe it: updates are
 * buffered and the state is written once per window, but every query still
 * reads the full state).  Per head, with the backward pass of
 * sketchssm_decode_step:  o = S^T q~ + o_buf  -- the exact read of step j.
 * S is read, not written; the window ends with sketchssm_update_window (P may be
 * NULL there).
 *   S   in [B][H][dv][dk] state_dtype, the window-start state
 *   q   in [B][H][dk];  k, v, alpha, beta in: window buffer slots 0..j-1
 *   o   out [B][H][dv] fp32
 * Errors: ERR_NULL, ERR_DIMS, ERR_DTYPE, ERR_RANGE (j < 1 or j > W), ERR_ALIGN,
 * ERR_CUDA.
 */
int sketchssm_replay_decode_step(const sketchssm_dims *dims, const void *S, const void *q, const void *k,
                                 const void *v, const float *alpha, const float *beta, int j, float *o,
                                 void *stream);

/*
 * sketchssm_device_error_count -- kernels never wait without bound: the decode
 * step's and the window update's waits for their bulk copies give up after a
 * fixed number of attempts, count the give-up in a device-side counter and
 * return without writing that head's results (the window update also stops
 * the rest of its CTA's heads, leaving their state and sketch as they were).
 * Per-sequence step indices and sequence indices out of range (read on the
 * device by sketchssm_decode_step_seq and sketchssm_update_window_seqs) are
 * counted the same way.
 * This call synchronises the current device and returns the sum of both counts
 * (0 in normal operation; a negative sketchssm_status if a CUDA call fails);
 * reset != 0 clears them.
 */
int sketchssm_device_error_count(int reset);

/*
 * sketchssm_selftest_wait_giveup -- makes the library's bounded-wait failure path
 * run, for tests of failure detection: one warp waits on a shared-memory
 * mbarrier that nothing arrives on, with the same wait every kernel of the
 * library uses, bounded to `tries` polls (1..2^20); the wait gives up, counts
 * itself in the sketchssm_device_error_count counter and the kernel returns,
 * leaving the context usable.
 * Errors: ERR_RANGE (tries), ERR_CUDA.
 */
int sketchssm_selftest_wait_giveup(unsigned tries, void *stream);

/*
 * sketchssm_calibrate_workspace_bytes -- device workspace that
 * sketchssm_calibrate_basis needs for these sizes (0 if dims are invalid).
 */
size_t sketchssm_calibrate_workspace_bytes(const sketchssm_dims *dims, int Nq, int Ns);

/*
 * sketchssm_calibrate_basis -- offline basis U and coefficient map R, per head.
 * Defines: SketchSSM abstract (low-rank, state-weighted query approximation on
 * basis vectors fixed offline); digest bullet "Core idea".  With
 *     G = (1/Ns) sum_s S_s S_s^T + ridge (tr G / dk) I     (state weighting)
 *     C = (1/Nq) sum_n q_n q_n^T                           (query second moment)
 * the basis spans the r-dimensional subspace that minimises the calibration-
 * averaged squared read error E ||S^T (q - U R q)||^2, and R = (U^T G U)^-1 U^T G
 * is the state-weighted least-squares coefficient map.  Computed in fp64
 * (Cholesky G = L L^T, Jacobi eigenvectors V_r of L^T C L with the r largest
 * eigenvalues, U = L^-T V_r, R = V_r^T L^T, so that R U = I); stored fp32.
 *   q_cal  in  [H][Nq][dk] fp32 calibration queries, Nq >= 1
 *   S_cal  in  [Ns][H][dv][dk] calibration states in the S layout, state_dtype,
 *              Ns >= 1 (the B field of dims is ignored here)
 *   ridge  >= 0, relative diagonal guard (1e-8 is a good default)
 *   U out [H][r][dk] fp32 (basis rows);  R out [H][r][dk] fp32
 *   workspace: device scratch of at least
 *              sketchssm_calibrate_workspace_bytes(dims, Nq, Ns) bytes, 256-byte
 *              aligned, owned by the caller; contents on entry are ignored.
 * Offline: not on the decode path.  Errors: ERR_NULL, ERR_DIMS, ERR_DTYPE,
 * ERR_RANGE, ERR_ALIGN, ERR_WORKSPACE, ERR_CUDA.
 */
int sketchssm_calibrate_basis(const sketchssm_dims *dims, const float *q_cal, int Nq,
                              const void *S_cal, int Ns, double ridge, float *U, float *R,
                              void *workspace, size_t workspace_bytes, void *stream);

/*
 * sketchssm_calibrate_query_pca -- the unweighted basis that the state weighting
 * is compared against: the top-r principal directions of the calibration
 * queries, ignoring the states.  SketchSSM abstract: the method's query
 * approximation is state-weighted; this is that approximation with the state
 * weight G replaced by the identity, so U = V_r, the eigenvectors of
 *     C = (1/Nq) sum_n q_n q_n^T
 * with the r largest eigenvalues, and R = V_r^T (orthogonal projection, R U = I).
 * Same fp64 kernels as sketchssm_calibrate_basis (Cholesky of I, Jacobi on C).
 *   q_cal  in  [H][Nq][dk] fp32, Nq >= 1
 *   U, R   out [H][r][dk] fp32
 *   workspace: at least sketchssm_calibrate_workspace_bytes(dims, Nq, 1) bytes,
 *              256-byte aligned, caller-owned.
 * Offline.  Errors: ERR_NULL, ERR_DIMS, ERR_DTYPE, ERR_RANGE, ERR_ALIGN,
 * ERR_WORKSPACE, ERR_CUDA.
 */
int sketchssm_calibrate_query_pca(const sketchssm_dims *dims, const float *q_cal, int Nq, float *U,
                                  float *R, void *workspace, size_t workspace_bytes, void *stream);

/*
 * sketchssm_calibrate_basis_ranked -- the offline calibration with a rank per head
 * under an average-rank budget.  SketchSSM abstract and digest: the traffic
 * reduction is quoted at an average sketch rank of 8, so ranks may differ across
 * heads.  With the basis of sketchssm_calibrate_basis, head h's averaged read
 * error at rank r is the sum of the eigenvalues of G^1/2 C G^1/2 past its r
 * largest; the total error over heads is smallest when the budget of H * r_avg
 * takes the largest of all heads' eigenvalues together, at most dims->r per head
 * (ties: larger value, then lower head, then lower index).  Head h's basis is the
 * first rank[h] rows of its rank-dims->r basis (U^T G U = I, so the same holds
 * for R).
 *   dims->r  r_max, the padded rank of U, R and P
 *   r_avg    1..r_max, the average rank
 *   U, R     out [H][r_max][dk] fp32, rows m >= rank[h] zero
 *   rank     out device [H] int32
 *   lam      out device [H][r_max] fp64: each head's r_max largest eigenvalues,
 *            descending (8-byte aligned)
 *   other arguments as sketchssm_calibrate_basis (same workspace size).
 * With rows past a head's rank zero, every kernel of this library gives that
 * head's rank-rank[h] results; the *_ranked calls also skip the work and the
 * sketch traffic of those rows.
 * Errors: as sketchssm_calibrate_basis; ERR_RANGE also for r_avg.
 */
int sketchssm_calibrate_basis_ranked(const sketchssm_dims *dims, const float *q_cal, int Nq,
                                     const void *S_cal, int Ns, double ridge, int r_avg, float *U,
                                     float *R, int32_t *rank, double *lam, void *workspace,
                                     size_t workspace_bytes, void *stream);

/*
 * sketchssm_calibrate_basis_noalloc -- sketchssm_calibrate_basis without a
 * workspace argument, for callers that cannot allocate device memory when they
 * calibrate (an engine that gave all free memory to its own pool at start-up,
 * a plug-in under a memory budget set by its host application, code that
 * cannot accept the device synchronisation of cudaFree).  The SketchSSM pages
 * have no counterpart: this is a deployment convenience, not part of the method.
 * Same inputs, outputs and results as sketchssm_calibrate_basis.
 *   Scratch: a fixed 3 MiB array inside the library's device image, held on
 *   every GPU that loads the library until the process exits.  One pass covers
 *   up to 8 heads at dk = 128 (32 at dk = 64); more heads run as several passes,
 *   in order on `stream`.  A size whose single head does not fit the scratch is
 *   rejected with SKSSM_ERR_WORKSPACE (no supported dk reaches that limit).
 *   Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 *   The first call on a device looks up the scratch's device address (once per
 *   device, with that device current); make that first call before any stream
 *   capture.  All calls share the one scratch array, which keeps the last call's
 *   contents (every pass overwrites what it reads, so nothing needs clearing);
 *   calls that overlap on the GPU race on it and must be ordered by the caller.
 * Errors: as sketchssm_calibrate_basis (ERR_WORKSPACE as above).
 */
int sketchssm_calibrate_basis_noalloc(const sketchssm_dims *dims, const float *q_cal, int Nq,
                                      const void *S_cal, int Ns, double ridge, float *U, float *R,
                                      void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SKETCHSSM_H */

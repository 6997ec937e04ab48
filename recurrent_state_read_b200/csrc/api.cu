// api.cu -- the exported C ABI (include/sketchssm.h): host-side validation, then launch.
//
// Every entry point checks its arguments before touching the GPU and returns a
// sketchssm_status; nothing is launched on error.  No entry point allocates.
#include <stdint.h>

#include "internal.h"

using namespace skssm;

int skssm::check_dims(const sketchssm_dims *d) {
    if (!d) return SKSSM_ERR_NULL;
    if (d->kind < SKSSM_MAMBA2 || d->kind > SKSSM_KDA) return SKSSM_ERR_DIMS;
    if (d->state_dtype != SKSSM_F32 && d->state_dtype != SKSSM_BF16) return SKSSM_ERR_DTYPE;
    if (d->qkv_dtype != SKSSM_F32 && d->qkv_dtype != SKSSM_BF16) return SKSSM_ERR_DTYPE;
    if (d->dk != 64 && d->dk != 128) return SKSSM_ERR_DIMS;
    if (d->dv != 64 && d->dv != 128) return SKSSM_ERR_DIMS;
    if (!((d->r >= 1 && d->r <= 32) || d->r == d->dk)) return SKSSM_ERR_DIMS;
    if (d->W < 1 || d->W > 64) return SKSSM_ERR_DIMS;
    if (d->B < 1 || d->H < 1) return SKSSM_ERR_DIMS;
    if ((int64_t)d->B * d->H >= (int64_t)1 << 31) return SKSSM_ERR_DIMS;
    return SKSSM_OK;
}

namespace {

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// window buffer / token pointers: k, v 16 B; alpha, beta 4 B
int check_tokens(const sketchssm_dims *d, const void *k, const void *v, const float *alpha,
                 const float *beta) {
    if (!k || !v || !alpha) return SKSSM_ERR_NULL;
    if (d->kind != SKSSM_MAMBA2 && !beta) return SKSSM_ERR_NULL;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(alpha, 4)) return SKSSM_ERR_ALIGN;
    if (beta && !aligned(beta, 4)) return SKSSM_ERR_ALIGN;
    if (d->kind == SKSSM_KDA && !aligned(alpha, 16)) return SKSSM_ERR_ALIGN;
    return SKSSM_OK;
}

}  // namespace

extern "C" {

const char *sketchssm_status_string(int status) {
    switch (status) {
        case SKSSM_OK: return "ok";
        case SKSSM_ERR_NULL: return "a required pointer is NULL";
        case SKSSM_ERR_DIMS: return "unsupported kind or sizes";
        case SKSSM_ERR_RANGE: return "step, token count or calibration count out of range";
        case SKSSM_ERR_ALIGN: return "a pointer breaks its alignment rule";
        case SKSSM_ERR_DTYPE: return "unsupported storage dtype";
        case SKSSM_ERR_CUDA: return "CUDA launch or runtime call failed";
        case SKSSM_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

int sketchssm_version(void) { return 10000; }

int sketchssm_update_window(const sketchssm_dims *d, void *S, float *P, const float *U, const void *k,
                            const void *v, const float *alpha, const float *beta, int n_tokens,
                            void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (!S || (P && !U)) return SKSSM_ERR_NULL;  // P == NULL: a state update without a sketch refresh
    if (n_tokens < 0 || n_tokens > d->W) return SKSSM_ERR_RANGE;
    if (n_tokens > 0 && (rc = check_tokens(d, k, v, alpha, beta))) return rc;
    if (!aligned(S, 16) || !aligned(P, 16) || !aligned(U, 16)) return SKSSM_ERR_ALIGN;
    if (n_tokens >= TC_MIN_TOKENS && d->kind == SKSSM_GDN) {  // the tensor-core form where it pays
        rc = launch_update_window_tc(*d, S, P, P ? U : nullptr, k, v, alpha, beta, n_tokens, (cudaStream_t)stream);
        if (rc != TC_NOT_APPLICABLE) return rc;
    }
    return launch_update_window(*d, S, P, P ? U : nullptr, k, v, alpha, beta, n_tokens, nullptr, nullptr, nullptr,
                                0, 0, nullptr, (cudaStream_t)stream);
}

int sketchssm_update_window_read(const sketchssm_dims *d, void *S, float *P, const float *U, const void *k,
                                            const void *v, const float *alpha, const float *beta, int n_tokens,
                                            const void *q, float *o, void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (!S || !P || !U || !q || !o) return SKSSM_ERR_NULL;
    if (n_tokens < 0 || n_tokens > d->W) return SKSSM_ERR_RANGE;
    if (n_tokens > 0 && (rc = check_tokens(d, k, v, alpha, beta))) return rc;
    if (!aligned(S, 16) || !aligned(P, 16) || !aligned(U, 16) || !aligned(q, 16) || !aligned(o, 16))
        return SKSSM_ERR_ALIGN;
    if (n_tokens >= TC_MIN_TOKENS && d->kind == SKSSM_GDN) {  // the tensor-core form where it pays
        rc = launch_update_window_tc(*d, S, P, U, k, v, alpha, beta, n_tokens, (cudaStream_t)stream, q, o);
        if (rc != TC_NOT_APPLICABLE) return rc;
    }
    return launch_update_window(*d, S, P, U, k, v, alpha, beta, n_tokens, q, o, nullptr, 0, 0, nullptr,
                                (cudaStream_t)stream);
}

int sketchssm_update_window_tc(const sketchssm_dims *d, void *S, float *P, const float *U, const void *k,
                               const void *v, const float *alpha, const float *beta, int n_tokens, void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (!S || (P && !U)) return SKSSM_ERR_NULL;
    if (n_tokens < 1 || n_tokens > d->W) return SKSSM_ERR_RANGE;
    if ((rc = check_tokens(d, k, v, alpha, beta))) return rc;
    if (!aligned(S, 16) || !aligned(P, 16) || !aligned(U, 16)) return SKSSM_ERR_ALIGN;
    rc = launch_update_window_tc(*d, S, P, P ? U : nullptr, k, v, alpha, beta, n_tokens, (cudaStream_t)stream);
    return rc == TC_NOT_APPLICABLE ? SKSSM_ERR_DIMS : rc;
}

int sketchssm_decode_step(const sketchssm_dims *d, const float *P, const float *R, const void *q,
                          const void *k, const void *v, const float *alpha, const float *beta, int j,
                          float *o, void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (!P || !R || !q || !o) return SKSSM_ERR_NULL;
    if (j < 1 || j > d->W) return SKSSM_ERR_RANGE;
    if ((rc = check_tokens(d, k, v, alpha, beta))) return rc;
    if (!aligned(P, 16) || !aligned(R, 16) || !aligned(q, 16) || !aligned(o, 16)) return SKSSM_ERR_ALIGN;
    return launch_decode_step(*d, P, R, q, k, v, alpha, beta, j, nullptr, 0, nullptr, o, (cudaStream_t)stream);
}

int sketchssm_fullread_decode(const sketchssm_dims *d, void *S, const void *q, const void *k,
                              const void *v, const float *alpha, const float *beta, float *o,
                              void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (!S || !q || !o) return SKSSM_ERR_NULL;
    if ((rc = check_tokens(d, k, v, alpha, beta))) return rc;
    if (!aligned(S, 16) || !aligned(q, 16) || !aligned(o, 16)) return SKSSM_ERR_ALIGN;
    return launch_fullread(*d, S, q, k, v, alpha, beta, o, (cudaStream_t)stream);
}

int sketchssm_decode_step_seq(const sketchssm_dims *d, const float *P, const float *R, const void *q, const void *k,
                              const void *v, const float *alpha, const float *beta, const int32_t *j_seq,
                              int sm_share, float *o, void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (!P || !R || !q || !o || !j_seq) return SKSSM_ERR_NULL;
    if (sm_share < 0) return SKSSM_ERR_RANGE;
    if ((rc = check_tokens(d, k, v, alpha, beta))) return rc;
    if (!aligned(P, 16) || !aligned(R, 16) || !aligned(q, 16) || !aligned(o, 16) || !aligned(j_seq, 4))
        return SKSSM_ERR_ALIGN;
    return launch_decode_step(*d, P, R, q, k, v, alpha, beta, d->W, j_seq, sm_share, nullptr, o, (cudaStream_t)stream);
}

int sketchssm_update_window_seqs(const sketchssm_dims *d, void *S, float *P, const float *U, const void *k,
                                 const void *v, const float *alpha, const float *beta, int n_tokens,
                                 const int32_t *seqs, int n_seqs, const void *q, float *o, int sm_share,
                                 void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (!S || (P && !U) || !seqs || (!q != !o)) return SKSSM_ERR_NULL;
    if (n_tokens < 0 || n_tokens > d->W || n_seqs < 0 || n_seqs > d->B || sm_share < 0) return SKSSM_ERR_RANGE;
    if (n_tokens > 0 && (rc = check_tokens(d, k, v, alpha, beta))) return rc;
    if (!aligned(S, 16) || !aligned(P, 16) || !aligned(U, 16) || !aligned(q, 16) || !aligned(o, 16) ||
        !aligned(seqs, 4))
        return SKSSM_ERR_ALIGN;
    return launch_update_window(*d, S, P, P ? U : nullptr, k, v, alpha, beta, n_tokens, q, o, seqs, n_seqs, sm_share,
                                nullptr, (cudaStream_t)stream);
}

int sketchssm_update_window_ranked(const sketchssm_dims *d, void *S, float *P, const float *U, const int32_t *rank,
                                   const void *k, const void *v, const float *alpha, const float *beta, int n_tokens,
                                   void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (!S || !P || !U || !rank) return SKSSM_ERR_NULL;
    if (n_tokens < 0 || n_tokens > d->W) return SKSSM_ERR_RANGE;
    if (n_tokens > 0 && (rc = check_tokens(d, k, v, alpha, beta))) return rc;
    if (!aligned(S, 16) || !aligned(P, 16) || !aligned(U, 16) || !aligned(rank, 4)) return SKSSM_ERR_ALIGN;
    return launch_update_window(*d, S, P, U, k, v, alpha, beta, n_tokens, nullptr, nullptr, nullptr, 0, 0, rank,
                                (cudaStream_t)stream);
}

int sketchssm_decode_step_ranked(const sketchssm_dims *d, const float *P, const float *R, const int32_t *rank,
                                 const void *q, const void *k, const void *v, const float *alpha, const float *beta,
                                 int j, float *o, void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (!P || !R || !rank || !q || !o) return SKSSM_ERR_NULL;
    if (j < 1 || j > d->W) return SKSSM_ERR_RANGE;
    if ((rc = check_tokens(d, k, v, alpha, beta))) return rc;
    if (!aligned(P, 16) || !aligned(R, 16) || !aligned(q, 16) || !aligned(o, 16) || !aligned(rank, 4))
        return SKSSM_ERR_ALIGN;
    return launch_decode_step(*d, P, R, q, k, v, alpha, beta, j, nullptr, 0, rank, o, (cudaStream_t)stream);
}

int sketchssm_decode_step_wy(const sketchssm_dims *d, const float *P, const float *R, const void *q, const void *k,
                             const void *v, const float *alpha, const float *beta, int j, float *G, float *o,
                             void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (d->W > 32) return SKSSM_ERR_DIMS;
    if (!P || !R || !q || !o || (!G && d->kind != SKSSM_MAMBA2)) return SKSSM_ERR_NULL;
    if (j < 1 || j > d->W) return SKSSM_ERR_RANGE;
    if ((rc = check_tokens(d, k, v, alpha, beta))) return rc;
    if (!aligned(P, 16) || !aligned(R, 16) || !aligned(q, 16) || !aligned(o, 16) || !aligned(G, 16))
        return SKSSM_ERR_ALIGN;
    return launch_decode_wy(*d, P, R, q, k, v, alpha, beta, j, G, o, (cudaStream_t)stream);
}

int sketchssm_replay_decode_step(const sketchssm_dims *d, const void *S, const void *q, const void *k, const void *v,
                                 const float *alpha, const float *beta, int j, float *o, void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (!S || !q || !o) return SKSSM_ERR_NULL;
    if (j < 1 || j > d->W) return SKSSM_ERR_RANGE;
    if ((rc = check_tokens(d, k, v, alpha, beta))) return rc;
    if (!aligned(S, 16) || !aligned(q, 16) || !aligned(o, 16)) return SKSSM_ERR_ALIGN;
    return launch_replay_decode(*d, S, q, k, v, alpha, beta, j, o, (cudaStream_t)stream);
}

size_t sketchssm_calibrate_workspace_bytes(const sketchssm_dims *d, int Nq, int Ns) {
    if (check_dims(d) != SKSSM_OK || Nq < 1 || Ns < 1) return 0;
    return calibrate_workspace_bytes(*d, Nq, Ns);
}

int sketchssm_calibrate_basis(const sketchssm_dims *d, const float *q_cal, int Nq, const void *S_cal,
                              int Ns, double ridge, float *U, float *R, void *workspace,
                              size_t workspace_bytes, void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (!q_cal || !S_cal || !U || !R) return SKSSM_ERR_NULL;
    if (Nq < 1 || Ns < 1 || !(ridge >= 0.0)) return SKSSM_ERR_RANGE;
    if ((int64_t)Ns * d->dv >= (int64_t)1 << 31 || (int64_t)Nq * d->H >= (int64_t)1 << 31)
        return SKSSM_ERR_RANGE;
    if (!workspace || workspace_bytes < calibrate_workspace_bytes(*d, Nq, Ns)) return SKSSM_ERR_WORKSPACE;
    if (!aligned(q_cal, 16) || !aligned(S_cal, 16) || !aligned(U, 16) || !aligned(R, 16) ||
        !aligned(workspace, 256))
        return SKSSM_ERR_ALIGN;
    return launch_calibrate(*d, q_cal, Nq, S_cal, Ns, ridge, U, R, workspace, (cudaStream_t)stream);
}

int sketchssm_calibrate_query_pca(const sketchssm_dims *d, const float *q_cal, int Nq, float *U, float *R,
                                  void *workspace, size_t workspace_bytes, void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (!q_cal || !U || !R) return SKSSM_ERR_NULL;
    if (Nq < 1 || (int64_t)Nq * d->H >= (int64_t)1 << 31) return SKSSM_ERR_RANGE;
    if (!workspace || workspace_bytes < calibrate_workspace_bytes(*d, Nq, 1)) return SKSSM_ERR_WORKSPACE;
    if (!aligned(q_cal, 16) || !aligned(U, 16) || !aligned(R, 16) || !aligned(workspace, 256))
        return SKSSM_ERR_ALIGN;
    return launch_calibrate(*d, q_cal, Nq, nullptr, 1, 0.0, U, R, workspace, (cudaStream_t)stream);
}

int sketchssm_calibrate_basis_ranked(const sketchssm_dims *d, const float *q_cal, int Nq, const void *S_cal, int Ns,
                                     double ridge, int r_avg, float *U, float *R, int32_t *rank, double *lam,
                                     void *workspace, size_t workspace_bytes, void *stream) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (!q_cal || !S_cal || !U || !R || !rank || !lam) return SKSSM_ERR_NULL;
    if (Nq < 1 || Ns < 1 || !(ridge >= 0.0) || r_avg < 1 || r_avg > d->r) return SKSSM_ERR_RANGE;
    if ((int64_t)Ns * d->dv >= (int64_t)1 << 31 || (int64_t)Nq * d->H >= (int64_t)1 << 31)
        return SKSSM_ERR_RANGE;
    if (!workspace || workspace_bytes < calibrate_workspace_bytes(*d, Nq, Ns)) return SKSSM_ERR_WORKSPACE;
    if (!aligned(q_cal, 16) || !aligned(S_cal, 16) || !aligned(U, 16) || !aligned(R, 16) ||
        !aligned(workspace, 256) || !aligned(rank, 4) || !aligned(lam, 8))
        return SKSSM_ERR_ALIGN;
    rc = launch_calibrate(*d, q_cal, Nq, S_cal, Ns, ridge, U, R, workspace, (cudaStream_t)stream, lam);
    if (rc != SKSSM_OK) return rc;
    return launch_rank_basis(*d, r_avg, lam, U, R, rank, (cudaStream_t)stream);
}

}  // extern "C"

// calibrate_noalloc.cu -- offline calibration for callers that cannot allocate device memory.
//
// sketchssm_calibrate_basis needs a caller-provided workspace.  Some callers
// cannot obtain one at the moment they calibrate: an engine that handed all
// free device memory to its own pool at start-up, a plug-in that runs under a
// memory budget fixed by its host application, or code for which the device
// synchronisation implied by cudaFree is not acceptable.  This entry point uses
// a fixed scratch array that lives in the library's own device image instead,
// and allocates nothing.
//
// Scratch: CALIB_SCRATCH_BYTES (3 MiB) of device memory, held on every GPU that
// loads this library until the process exits.  One pass needs 3 * dk * dk fp64
// per head (G, C and T/V), so a pass covers up to 8 heads at dk = 128 (32 at
// dk = 64); more heads run as several passes over the same scratch, in stream
// order.  Every pass overwrites all the scratch it reads, so nothing has to be
// cleared between calls.  All calls share the one array: calls whose work
// overlaps on the GPU (different streams or threads without ordering between
// them) race on it and must be serialised by the caller.
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t CALIB_SCRATCH_BYTES = size_t(3) << 20;
constexpr int MAX_DEVICES = 64;

// The scratch itself.  Host code must not use this name as a device address: it
// refers to a host-side shadow.  The device address is looked up per device.
static __device__ __align__(256) double g_calib_scratch[CALIB_SCRATCH_BYTES / sizeof(double)];

// Device address of the scratch per device, looked up on first use.  A failed
// lookup is not recorded, so the next call on that device tries again.
std::mutex g_setup_mu;
void *g_scratch_addr[MAX_DEVICES];

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int sketchssm_calibrate_basis_noalloc(const sketchssm_dims *d, const float *q_cal, int Nq,
                                                 const void *S_cal, int Ns, double ridge, float *U,
                                                 float *R, void *stream) {
    int rc = skssm::check_dims(d);
    if (rc) return rc;
    if (!q_cal || !S_cal || !U || !R) return SKSSM_ERR_NULL;
    if (Nq < 1 || Ns < 1 || !(ridge >= 0.0)) return SKSSM_ERR_RANGE;
    if ((int64_t)Ns * d->dv >= (int64_t)1 << 31 || (int64_t)Nq * d->H >= (int64_t)1 << 31)
        return SKSSM_ERR_RANGE;
    if (!aligned16(q_cal) || !aligned16(S_cal) || !aligned16(U) || !aligned16(R)) return SKSSM_ERR_ALIGN;
    const size_t per_head = 3 * (size_t)d->dk * d->dk * sizeof(double);
    const int heads_per_pass = (int)(CALIB_SCRATCH_BYTES / per_head);
    if (heads_per_pass < 1) return SKSSM_ERR_WORKSPACE;  // one head does not fit the fixed scratch

    // Set-up, once per device, with that device current: the scratch's device address.
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return SKSSM_ERR_CUDA;
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_setup_mu);
        if (!g_scratch_addr[dev]) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_calib_scratch) != cudaSuccess || !p) return SKSSM_ERR_CUDA;
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }

    for (int h0 = 0; h0 < d->H; h0 += heads_per_pass) {
        const int hc = d->H - h0 < heads_per_pass ? d->H - h0 : heads_per_pass;
        rc = skssm::launch_calibrate_heads(*d, q_cal, Nq, S_cal, Ns, ridge, U, R, scratch, h0,
                                           hc, (cudaStream_t)stream);
        if (rc) return rc;
    }
    return SKSSM_OK;
}

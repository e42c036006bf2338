// carve_bwd_noalloc: the backward pass with its scratch memory in a fixed, library-owned
// device array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run the backward: a
// plugin inside a host framework that owns every byte of device memory and hands the plugin
// only its input and output buffers, or a latency-critical loop that must not pay for
// cudaMalloc's implicit device synchronisation.  This entry point serves them.  It calls
// nothing that allocates: no cudaMalloc, no cudaFree, no allocating library routine.
//
// The scratch is the file-scope array below (4 MiB per GPU that loads the library, held
// until the process exits).  In host code `g_noalloc_scratch` is only a host-side stand-in
// for the symbol, not a device address, so the device address is looked up once per device
// with cudaGetSymbolAddress (with that device current) and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/carve.h"

namespace {

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on first use).
cudaError_t scratch_for_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" carve_status carve_bwd_noalloc(const carve_dims *d, const void *q, const void *k, const void *v,
                                          const float *g_logit, const float *bx, const float *w_logit,
                                          const float *A, const float *Bm, const float *Aw, const float *A_dec,
                                          const float *tau, const float *S0, const float *m_prev_in,
                                          const void *saved, const void *dO, const float *dS_final,
                                          const float *dm_prev_out, void *dq, void *dk, void *dv, float *dg_logit,
                                          float *dbx, float *dw_logit, float *dA, float *dB, float *dAw,
                                          float *dA_dec, float *dtau, float *dS0, float *dm_prev_in,
                                          void *stream) {
    const size_t need = carve_bwd_workspace_bytes(d);
    if (need == 0)  // malformed dims: carve_bwd rejects them on the host, before any launch
        return carve_bwd(d, q, k, v, g_logit, bx, w_logit, A, Bm, Aw, A_dec, tau, S0, m_prev_in, saved, dO, dS_final,
                         dm_prev_out, dq, dk, dv, dg_logit, dbx, dw_logit, dA, dB, dAw, dA_dec, dtau, dS0, dm_prev_in,
                         nullptr, stream);
    if (need > kScratchBytes) return CARVE_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return CARVE_ERR_CUDA;
    // The backward kernel zeroes the part of the scratch it accumulates into before using it,
    // so the contents left by an earlier call do not leak into this one.
    return carve_bwd(d, q, k, v, g_logit, bx, w_logit, A, Bm, Aw, A_dec, tau, S0, m_prev_in, saved, dO, dS_final,
                     dm_prev_out, dq, dk, dv, dg_logit, dbx, dw_logit, dA, dB, dAw, dA_dec, dtau, dS0, dm_prev_in,
                     scratch, stream);
}

// Device helpers shared by the CARVE kernels (product code; independent of the oracle).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace carve {

constexpr int kSub = 16;       // compute sub-chunk of the SIMT kernels (tokens)
constexpr int kThreads = 256;  // threads per CTA of the SIMT kernels

__device__ __forceinline__ float ld_io(const float *p) { return *p; }
__device__ __forceinline__ float ld_io(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_io(float *p, float x) { *p = x; }
__device__ __forceinline__ void st_io(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

// softplus(x) = log(1 + e^x), evaluated without overflow
__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))); }
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }

// log-retention of one key channel: log a = log g + log b
//   g = exp(-softplus(g_logit))        (key-axis decay gate)
//   b = sigmoid(bx + Delta) = exp(-softplus(-(bx + Delta)))  (content-aware erase gate)
__device__ __forceinline__ float log_retention(float g_logit, float beta) {
    return -softplus_f(g_logit) - softplus_f(-beta);
}

struct FwdArgs {
    const void *q, *k, *v;
    const float *g_logit, *bx, *w_logit, *A, *Bm, *S0, *m_prev_in;
    void *o;
    float *S_final, *m_prev_out;
    float *saved_states;  // [B,H,T/16,V,K] or null
    float *saved_aux;     // [B,H,NC,V+R+K] or null
    int B, H, T, R, L, mc_mode;
};

struct BwdArgs {
    const void *q, *k, *v;
    const float *g_logit, *bx, *w_logit, *A, *Bm;
    const float *saved_states, *saved_aux;
    const void *dO;
    const float *dS_final, *dm_prev_out;
    void *dq, *dk, *dv;
    float *dg_logit, *dbx, *dw_logit, *dS0, *dm_prev_in;
    float *ws;  // [B,H,K*R + R*V] per-unit dA/dB partials
    int B, H, T, R, L, mc_mode;
};

}  // namespace carve

// Constants and small helpers shared by the tensor-core forward and backward kernels.
#pragma once
#include "carve_device.cuh"
#include "carve_mma.cuh"

namespace carve {

constexpr int kLdOp = 136;                            // bf16 row stride of 128-wide tiles
constexpr float kAMin = 4.5399929762484854e-05f;      // e^-10: floor of the per-step retention
constexpr float kInvAMin = 22026.465794806718f;       // e^10

__device__ __forceinline__ int pair_index(int i, int j) { return i * (i - 1) / 2 + j; }
__device__ __forceinline__ float bf(const __nv_bfloat16 x) { return __bfloat162float(x); }

// Per-step retention of one (token, channel) in product form: a = sigma(-g_logit) sigma(beta)
// = 1 / ((1 + e^{g_logit})(1 + e^{-beta})), floored at e^-10; also returns 1/a.
__device__ __forceinline__ void retention(float g_logit, float beta, float &a, float &inv_a) {
    const float D = (1.f + __expf(g_logit)) * (1.f + __expf(-beta));
    const float r = __fdividef(1.f, D);
    const bool floor = !(r >= kAMin);
    a = floor ? kAMin : r;
    inv_a = floor ? kInvAMin : D;
}

// Factor on the gradient of log a in the backward.  The kernels differentiate the floored
// retention; where the floor binds (unfloored retention r < e^-10) the exact recurrence's
// gradient of log a is r e^10 times that one: the gradient with respect to log a_t is a_t times
// the product of the state before t with the gradient after the decay, and the floor moves
// those two only by O(e^-10) relative.  Inert rows (past a packed sequence's end) have none.
__device__ __forceinline__ float floor_scale(float r, bool inert) {
    return inert ? 0.f : (r >= kAMin ? 1.f : r * kInvAMin);
}

// softplus(x) from one fast exponential e1 = e^x; beyond x = 15, log(1 + e^x) is x to fp32
// rounding (and e^x may overflow), so it takes that value there (sigmoid(x) likewise takes 1)
__device__ __forceinline__ float softplus_fast(float x, float e1) { return x > 15.f ? x : __logf(1.f + e1); }

// The same with the decay's amplitude and bias: 1 / g = e^{amp softplus(x)}, x = g_logit + tau
// (the product form above is its amp = 1, tau = 0 case, evaluated with fewer operations).
__device__ __forceinline__ void retention_dec(float x, float amp, float beta, float &a, float &inv_a) {
    const float D = __expf(amp * softplus_fast(x, __expf(x))) * (1.f + __expf(-beta));
    const float r = __fdividef(1.f, D);
    const bool floor = !(r >= kAMin);
    a = floor ? kAMin : r;
    inv_a = floor ? kInvAMin : D;
}

// Mid-block references of one 16-token block from its retentions av (and reciprocals ia):
// rf[t] = e^{Lam_t - Lam_7}, cf[t] = 1 / rf[t], both as running products from token 7.
__device__ __forceinline__ void mid_reference(const float (&av)[16], const float (&ia)[16], float (&rf)[16],
                                              float (&cf)[16]) {
    rf[7] = cf[7] = 1.f;
#pragma unroll
    for (int t = 8; t < 16; ++t) {
        rf[t] = rf[t - 1] * av[t];
        cf[t] = cf[t - 1] * ia[t];
    }
#pragma unroll
    for (int t = 6; t >= 0; --t) {
        cf[t] = cf[t + 1] * av[t + 1];
        rf[t] = rf[t + 1] * ia[t + 1];
    }
}

// Column c of T = (I + Diag(w) A)^-1 for a strictly lower-triangular 16x16 block A (row t at
// A + t * lda) and weights w[0..16): x_t = [t == c] - w_t sum_{s<t} A_ts x_s, evaluated
// right-looking (each x_s, once final, is added into every later row's sum at once), so the
// dependent chain is 16 steps deep instead of one step per term.
__device__ __forceinline__ void unit_lower_inverse_column(const float *A, int lda, const float *w, int c,
                                                          float (&x)[16]) {
    float acc[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) acc[t] = 0.f;
#pragma unroll
    for (int s = 0; s < 16; ++s) {
        x[s] = (s == c ? 1.f : 0.f) - w[s] * acc[s];
#pragma unroll
        for (int t = s + 1; t < 16; ++t) acc[t] += A[t * lda + s] * x[s];
    }
}

// A fragment of the negated operand (sign flip of both bf16 halves)
__device__ __forceinline__ void negate_frag(uint32_t (&a)[4]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) a[e] ^= 0x80008000u;
}

}  // namespace carve

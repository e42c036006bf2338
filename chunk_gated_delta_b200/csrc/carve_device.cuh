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
//   g = exp(-amp softplus(g_logit + tau))   (key-axis decay gate; amp = e^{A_dec} is the head's
//                                             decay amplitude, tau the channel's bias; 1 and 0
//                                             without them, which leaves every bit unchanged)
//   b = sigmoid(bx + Delta) = exp(-softplus(-(bx + Delta)))  (content-aware erase gate)
__device__ __forceinline__ float log_retention(float g_logit, float beta, float amp = 1.f, float tau = 0.f) {
    return -amp * softplus_f(g_logit + tau) - softplus_f(-beta);
}

// The decay's parameters of head h: amplitude e^{A_dec[h]} (1 without A_dec) and the bias of
// channel i of K (0 without tau).
__device__ __forceinline__ float decay_amp(const float *A_dec, int h) { return A_dec ? expf(A_dec[h]) : 1.f; }
__device__ __forceinline__ float decay_bias(const float *tau, int h, int i, int K) {
    return tau ? tau[(size_t)h * K + i] : 0.f;
}

// Content signal of a chunk: z = Bh m (R outputs, dot products over V) then
// Delta = Ah z (K outputs over R).  Bh is [R][V], Ah is [K][R] (row-major, global or shared);
// every thread of the CTA must call this.  Eight threads share each z output and
// kThreads / K share each Delta output, so the loads of one output are issued together.
template <int K, int V>
__device__ __forceinline__ void content_signal(const float *Bh, const float *Ah, const float *m, float *z,
                                               float *delta, int R) {
    const int tid = threadIdx.x;
    for (int j0 = 0; j0 < R; j0 += kThreads / 8) {
        const int j = j0 + tid / 8, part = tid % 8;
        float acc = 0.f;
        if (j < R) {
            const float *row = Bh + (size_t)j * V;
#pragma unroll
            for (int r = part; r < V; r += 8) acc += row[r] * m[r];
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        if (j < R && part == 0) z[j] = acc;
    }
    __syncthreads();
    constexpr int TPO = kThreads / K;
    {
        const int kk = tid / TPO, part = tid % TPO;
        const float *row = Ah + (size_t)kk * R;
        float acc = 0.f;
#pragma unroll 8
        for (int j = part; j < R; j += TPO) acc += row[j] * z[j];
#pragma unroll
        for (int off = TPO / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (part == 0) delta[kk] = acc;
    }
    __syncthreads();
}

// Host: raise `kern`'s dynamic shared-memory limit to `bytes` on the current device, once.
cudaError_t set_smem_once(const void *kern, int bytes);

// Records of the tensor-core path, per (unit, gate chunk), in floats:
//   saved by the forward: m (128), z (R), Delta (128), mean q (128), dw (1), 3 pad
//   written by the backward for the dA / dB / dAw reduction: dDelta (128), dz (32), d(dw) (1), 3 pad
constexpr int kTcAuxFixed = 388;   // + R
constexpr int kTcAuxDw = 384;      // + R: offset of dw in the saved record
constexpr int kTcGradRec = 164;
constexpr int kTcGradDw = 160;     // offset of d(dw) in the gradient record
//   per unit, after the sweep, when the decay has parameters: d tau (128), d A_dec (1), 3 pad
constexpr int kTcDecayRec = 132;

struct FwdArgs {
    const void *q, *k, *v;
    const float *g_logit, *bx, *w_logit, *A, *Bm, *Aw, *S0, *m_prev_in;
    const float *A_dec, *tau;   // [H], [H,K] or null: the decay's log-amplitude and bias
    void *o;
    float *S_final, *m_prev_out;
    float *saved_states;  // [B,H,T/16,V,K] or null
    float *saved_aux;     // [B,H,NC,V+R+K] or null
    const int *cu_seqlens;  // [B+1] or null: B sequences packed along the token axis
    long long total;        // rows of the packed token tensors (with cu_seqlens)
    int B, H, T, R, L, mc_mode;
    uint32_t wait_limit;    // polls of each bounded barrier wait (tensor-core kernels)
    int stall;              // test hook: skip the first tile copy so that its wait gives up
};

struct BwdArgs {
    const void *q, *k, *v;
    const float *g_logit, *bx, *w_logit, *A, *Bm, *Aw;   // Aw [H,R] or null: write gate content term
    const float *A_dec, *tau;                            // [H], [H,K] or null: decay amplitude, bias
    const float *saved_states, *saved_aux;
    const void *dO;
    const float *dS_final, *dm_prev_out;
    void *dq, *dk, *dv;
    float *dg_logit, *dbx, *dw_logit, *dS0, *dm_prev_in, *dAw, *dA_dec, *dtau;
    float *ws;  // scratch: per-unit dA/dB(/dAw) partials or per-gate-chunk gradient records
    const int *cu_seqlens;  // [B+1] or null: B sequences packed along the token axis
    long long total;        // rows of the packed token tensors (with cu_seqlens)
    int B, H, T, R, L, mc_mode;
    uint32_t wait_limit;    // polls of each bounded barrier wait (tensor-core kernels)
    int stall;              // test hook: skip the first tile copy so that its wait gives up
};

// Polls of a bounded barrier wait in normal operation (each poll may suspend the thread for
// a while, so this is of the order of a second: far beyond any copy that completes).
constexpr uint32_t kWaitLimit = 1u << 26;

// Tokens of sequence b: rows [toff, toff + Tn) of tensor batch bb.  Without cu_seqlens the
// unit is batch element b with all T tokens; with it, the sequences are packed along the token
// axis of [1, total, H, *] tensors and sequence b owns rows [cu[b], cu[b+1]), which must lie
// in [0, total] and number at most T (else the sequence is treated as empty and *bad, the
// calling file's device status word, records it).
__device__ __forceinline__ void seq_tokens(const int *cu, long long total, int T, int b, int &bb, int &toff,
                                           int &Tn, int *bad) {
    if (!cu) {
        bb = b;
        toff = 0;
        Tn = T;
        return;
    }
    const int c0 = cu[b], c1 = cu[b + 1];
    bb = 0;
    toff = 0;
    Tn = 0;
    if (c0 < 0 || c1 < c0 || (long long)c1 > total || c1 - c0 > T) {
        if (threadIdx.x == 0) atomicOr(bad, 1);
        return;
    }
    toff = c0;
    Tn = c1 - c0;
}

}  // namespace carve

// CARVE single-token decode step: one CTA per (batch, head), state read once and written
// once (CARVE blog, Table 1: inference costs O(dv dk) per token).
//
// With P = S Diag(a) the token's update and output expand to three matrix-vector products
// over the same state rows, so the state is loaded into registers once:
//   m  = S q                     (mc_mode 0: content signal from the state before the token)
//   a  = exp(-softplus(g_logit)) * sigmoid(bx + A (Bm m)),  w = sigmoid(w_logit)
//   p  = S (a*k),  e = v - p
//   o  = S (a*q) + w e (k.q)     (= S' q)
//   S' = S Diag(a) + w e k^T
// Each row of S is held by TPR threads as float4 groups interleaved so that a warp's loads
// and stores cover contiguous 16-byte segments.
#include "carve_device.cuh"

namespace carve {

struct StepArgs {
    const void *q, *k, *v;
    const float *g_logit, *bx, *w_logit, *A, *Bm;
    float *S, *mstate;
    int *pos;
    void *o;
    int B, H, R, L, mc_mode;
};

template <int K, int V, typename IO>
__global__ void __launch_bounds__(kThreads) step_kernel(StepArgs a) {
    constexpr int TPR = kThreads / V;        // threads per state row
    constexpr int G4 = K / 4 / TPR;          // float4 groups per thread
    __shared__ float qv[K], kv[K], av[K], mv[V], zv[64], red[kThreads / 32];
    __shared__ float s_w, s_kq;
    const int tid = threadIdx.x, u = blockIdx.x, h = u % a.H;
    const int row = tid / TPR, seg = tid % TPR;
    const IO *q = static_cast<const IO *>(a.q) + (size_t)u * K;
    const IO *k = static_cast<const IO *>(a.k) + (size_t)u * K;
    const IO *vv = static_cast<const IO *>(a.v) + (size_t)u * V;
    float4 *Srow = reinterpret_cast<float4 *>(a.S + ((size_t)u * V + row) * K);

    float4 s[G4];
#pragma unroll
    for (int j = 0; j < G4; ++j) s[j] = Srow[seg + TPR * j];
    if (tid < K) {
        qv[tid] = ld_io(q + tid);
        kv[tid] = ld_io(k + tid);
    }
    __syncthreads();
    // content signal
    if (a.mc_mode == 0) {
        float part = 0.f;
#pragma unroll
        for (int j = 0; j < G4; ++j) {
            const int c = 4 * (seg + TPR * j);
            part += s[j].x * qv[c] + s[j].y * qv[c + 1] + s[j].z * qv[c + 2] + s[j].w * qv[c + 3];
        }
#pragma unroll
        for (int off = TPR / 2; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        if (seg == 0) mv[row] = part;
    } else if (tid < V) {
        float *msum = a.mstate + (size_t)u * 2 * V, *mprev = msum + V;
        const int p = a.pos[u];
        float m = mprev[tid];
        if (p > 0 && p % a.L == 0) {
            m = msum[tid] / (float)a.L;
            mprev[tid] = m;
            msum[tid] = 0.f;
        }
        mv[tid] = m;
    }
    // k.q (warp 0)
    if (tid < 32) {
        float x = 0.f;
        for (int i = tid; i < K; i += 32) x += kv[i] * qv[i];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        if (tid == 0) {
            s_kq = x;
            s_w = sigmoid_f(a.w_logit[u]);
        }
    }
    __syncthreads();
    if (tid < a.R) {
        float z = 0.f;
        const float *Bh = a.Bm + ((size_t)h * a.R + tid) * V;
        for (int r = 0; r < V; ++r) z += Bh[r] * mv[r];
        zv[tid] = z;
    }
    __syncthreads();
    if (tid < K) {
        float d = 0.f;
        const float *Ah = a.A + ((size_t)h * K + tid) * a.R;
        for (int j = 0; j < a.R; ++j) d += Ah[j] * zv[j];
        const size_t g = (size_t)u * K + tid;
        av[tid] = expf(log_retention(a.g_logit[g], a.bx[g] + d));
    }
    __syncthreads();
    float p = 0.f, s2 = 0.f;
#pragma unroll
    for (int j = 0; j < G4; ++j) {
        const int c = 4 * (seg + TPR * j);
        const float a0 = av[c], a1 = av[c + 1], a2 = av[c + 2], a3 = av[c + 3];
        p += s[j].x * a0 * kv[c] + s[j].y * a1 * kv[c + 1] + s[j].z * a2 * kv[c + 2] + s[j].w * a3 * kv[c + 3];
        s2 += s[j].x * a0 * qv[c] + s[j].y * a1 * qv[c + 1] + s[j].z * a2 * qv[c + 2] + s[j].w * a3 * qv[c + 3];
    }
#pragma unroll
    for (int off = TPR / 2; off >= 1; off >>= 1) {
        p += __shfl_xor_sync(0xffffffffu, p, off);
        s2 += __shfl_xor_sync(0xffffffffu, s2, off);
    }
    const float w = s_w;
    const float e = ld_io(vv + row) - p;
    const float we = w * e;
#pragma unroll
    for (int j = 0; j < G4; ++j) {
        const int c = 4 * (seg + TPR * j);
        float4 x = s[j];
        x.x = x.x * av[c] + we * kv[c];
        x.y = x.y * av[c + 1] + we * kv[c + 1];
        x.z = x.z * av[c + 2] + we * kv[c + 2];
        x.w = x.w * av[c + 3] + we * kv[c + 3];
        Srow[seg + TPR * j] = x;
    }
    if (seg == 0) {
        const float ov = s2 + we * s_kq;
        st_io(static_cast<IO *>(a.o) + (size_t)u * V + row, ov);
        if (a.mc_mode == 1) a.mstate[(size_t)u * 2 * V + row] += ov;
    }
    if (a.mc_mode == 1 && tid == 0) a.pos[u] += 1;
    (void)red;
}

template <int K, int V, typename IO>
cudaError_t launch_step_t(const StepArgs &a, cudaStream_t st) {
    step_kernel<K, V, IO><<<a.B * a.H, kThreads, 0, st>>>(a);
    return cudaGetLastError();
}

template <typename IO>
cudaError_t dispatch_step(int K, int V, const StepArgs &a, cudaStream_t st) {
    if (K == 64 && V == 64) return launch_step_t<64, 64, IO>(a, st);
    if (K == 64 && V == 128) return launch_step_t<64, 128, IO>(a, st);
    if (K == 128 && V == 64) return launch_step_t<128, 64, IO>(a, st);
    return launch_step_t<128, 128, IO>(a, st);
}

cudaError_t launch_step(int K, int V, bool bf16, const void *q, const void *k, const void *v,
                        const float *g_logit, const float *bx, const float *w_logit, const float *A,
                        const float *Bm, float *S, float *mstate, int *pos, void *o, int B, int H,
                        int R, int L, int mc_mode, cudaStream_t st) {
    StepArgs a{q, k, v, g_logit, bx, w_logit, A, Bm, S, mstate, pos, o, B, H, R, L, mc_mode};
    return bf16 ? dispatch_step<__nv_bfloat16>(K, V, a, st) : dispatch_step<float>(K, V, a, st);
}

}  // namespace carve

// CARVE exact content-aware recurrence: gate chunk L = 1 with the boundary-state readout, so
// the content signal of every token is read from the state right before it,
//   m_t = S_{t-1} q_t,  z = Bm m_t,  Delta = A z,  a_t = g_t sigmoid(bx_t + Delta),
//   w_t = sigmoid(w_logit_t + Aw . z),  S_t = S_{t-1} Diag(a_t) + w_t (v_t - S_{t-1} Diag(a_t) k_t) k_t^T,
//   o_t = S_t q_t
// (the content-aware exact recurrent model of the CARVE blog's Tables 1 and 3: O(T) parallel
// depth, the reference point the chunk-parallel form is measured against).  Nothing here is
// chunk-parallel: one CTA per (batch, head) unit runs the tokens in order with the fp32 state
// in shared memory.  The forward checkpoints the state every kSeg tokens; the backward
// recomputes the per-token states of one segment into a scratch buffer and runs
// back-propagation through time over it, in reverse.
#include "carve_device.cuh"

namespace carve {

constexpr int kSeg = 64;   // tokens between state checkpoints

cudaError_t launch_reduce_units(const float *ws, float *dA, float *dB, float *dAw, float *dtau, float *dA_dec, int B,
                                int H, int K, int V, int R, cudaStream_t st);

// Per-token helpers over an fp32 state M [V][K+1] in shared memory (256 threads).
template <int K, int V>
struct ExactOps {
    static constexpr int KP = K + 1, TPR = kThreads / V, TPC = kThreads / K;
    // out[j] = sum_i M[j][i] x[i]  (TPR threads per row)
    __device__ static void row_dot(const float *M, const float *x, float *out) {
        const int tid = threadIdx.x, j = tid / TPR, part = tid % TPR;
        const float *row = M + j * KP;
        float acc = 0.f;
#pragma unroll 8
        for (int i = part; i < K; i += TPR) acc += row[i] * x[i];
#pragma unroll
        for (int off = TPR / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (part == 0) out[j] = acc;
    }
};

template <int K, int V, typename IO>
__global__ void __launch_bounds__(kThreads, 1) exact_fwd_kernel(FwdArgs a) {
    using OP = ExactOps<K, V>;
    constexpr int KP = OP::KP;
    extern __shared__ __align__(16) float sm[];
    float *S = sm;                                   // [V][KP]
    float *qv = S + V * KP, *kv = qv + K, *av = kv + K, *akv = av + K, *glv = akv + K, *bxv = glv + K;
    float *delta = bxv + K;                          // [K]
    float *vv = delta + K, *mv = vv + V, *ev = mv + V;   // [V] each
    float *zv = ev + V;                              // [64]
    float *wsc = zv + 64;                            // [4]: w_logit, w
    const int tid = threadIdx.x, u = blockIdx.x, H = a.H, T = a.T, R = a.R;
    const int b = u / H, h = u % H;
    const float amp = decay_amp(a.A_dec, h);
    const int NSEG = (T + kSeg - 1) / kSeg;
    const IO *q = static_cast<const IO *>(a.q), *kk = static_cast<const IO *>(a.k);
    const IO *vp = static_cast<const IO *>(a.v);
    IO *o = static_cast<IO *>(a.o);

    for (int idx = tid; idx < V * K; idx += kThreads)
        S[(idx / K) * KP + idx % K] = a.S0 ? a.S0[(size_t)u * V * K + idx] : 0.f;
    __syncthreads();
    for (int t = 0; t < T; ++t) {
        if (t % kSeg == 0 && a.saved_states) {   // checkpoint: the state before token t
            float *ck = a.saved_states + ((size_t)u * NSEG + t / kSeg) * V * K;
            for (int idx = tid; idx < V * K; idx += kThreads) ck[idx] = S[(idx / K) * KP + idx % K];
        }
        const size_t row = (size_t)b * T + t;
        if (tid < K) {
            const size_t g = (row * H + h) * K + tid;
            qv[tid] = ld_io(q + g);
            kv[tid] = ld_io(kk + g);
            glv[tid] = a.g_logit[g];
            bxv[tid] = a.bx[g];
        }
        if (tid < V) vv[tid] = ld_io(vp + (row * H + h) * V + tid);
        if (tid == 0) wsc[0] = a.w_logit[row * H + h];
        __syncthreads();
        OP::row_dot(S, qv, mv);   // m_t = S_{t-1} q_t
        __syncthreads();
        content_signal<K, V>(a.Bm + (size_t)h * R * V, a.A + (size_t)h * K * R, mv, zv, delta, R);
        if (tid < K) {
            const float x = expf(log_retention(glv[tid], bxv[tid] + delta[tid], amp, decay_bias(a.tau, h, tid, K)));
            av[tid] = x;
            akv[tid] = x * kv[tid];
        }
        if (tid == 0) {
            float s = 0.f;
            if (a.Aw)
                for (int j = 0; j < R; ++j) s += a.Aw[(size_t)h * R + j] * zv[j];
            wsc[1] = sigmoid_f(wsc[0] + s);
        }
        __syncthreads();
        OP::row_dot(S, akv, ev);   // S_{t-1} Diag(a) k
        __syncthreads();
        const float w = wsc[1];
        for (int idx = tid; idx < V * K; idx += kThreads) {
            const int j = idx / K, i = idx % K;
            S[j * KP + i] = S[j * KP + i] * av[i] + w * (vv[j] - ev[j]) * kv[i];
        }
        __syncthreads();
        OP::row_dot(S, qv, mv);   // o_t = S_t q_t
        __syncthreads();
        if (tid < V) {
            st_io(o + (row * H + h) * V + tid, mv[tid]);
            if (t == T - 1 && a.m_prev_out) a.m_prev_out[(size_t)u * V + tid] = mv[tid];   // mean of the last chunk
        }
    }
    if (a.S_final)
        for (int idx = tid; idx < V * K; idx += kThreads) a.S_final[(size_t)u * V * K + idx] = S[(idx / K) * KP + idx % K];
}

template <int K, int V>
struct ExactBwdLayout {
    static constexpr int KP = K + 1, TPC = kThreads / K;
    // S, dS [V][KP]; partials dA [K*64], dB [64*V], dAw [64], dtau [K]; vectors; column partials
    static constexpr int floats = 2 * V * KP + K * 64 + 64 * V + 64 + K + 10 * K + 8 * V + 2 * 64 + 5 * TPC * K + 8;
    static constexpr size_t bytes = sizeof(float) * floats;
};

template <int K, int V, typename IO>
__global__ void __launch_bounds__(kThreads, 1) exact_bwd_kernel(BwdArgs a) {
    using OP = ExactOps<K, V>;
    constexpr int KP = OP::KP, TPC = OP::TPC;
    extern __shared__ __align__(16) float sm[];
    const int tid = threadIdx.x, u = blockIdx.x, H = a.H, T = a.T, R = a.R;
    const int b = u / H, h = u % H;
    float *S = sm, *dS = S + V * KP;                          // [V][KP] each
    float *dAp = dS + V * KP, *dBp = dAp + K * 64, *dAwp = dBp + 64 * V, *dtaup = dAwp + 64;
    float *qv = dtaup + K, *kv = qv + K, *av = kv + K, *akv = av + K, *glv = akv + K, *bxv = glv + K;
    float *delta = bxv + K, *ddelta = delta + K, *dqv = ddelta + K, *spare = dqv + K;
    float *vv = spare + K, *mv = vv + V, *ev = mv + V, *dov = ev + V, *uv = dov + V, *dev = uv + V, *dmv = dev + V;
    float *red = dmv + V;                                     // [V] block-reduction scratch
    float *zv = red + V, *dzv = zv + 64;                      // [64] each
    float *cpart = dzv + 64;                                  // [5][TPC][K] column-dot partials
    float *wsc = cpart + 5 * TPC * K;                         // [8]
    const float amp = decay_amp(a.A_dec, h);
    const int NSEG = (T + kSeg - 1) / kSeg;
    const IO *q = static_cast<const IO *>(a.q), *kk = static_cast<const IO *>(a.k);
    const IO *vp = static_cast<const IO *>(a.v), *dO = static_cast<const IO *>(a.dO);
    IO *dq = static_cast<IO *>(a.dq), *dk = static_cast<IO *>(a.dk), *dvp = static_cast<IO *>(a.dv);
    const int rec = K * R + R * V + R + K + 1;
    float *wsu = a.ws + (size_t)u * rec;
    float *scratch = a.ws + (size_t)a.B * a.H * rec + (size_t)u * kSeg * V * K;   // states of one segment
    const float *Ah = a.A + (size_t)h * K * R, *Bh = a.Bm + (size_t)h * R * V;

    for (int idx = tid; idx < V * K; idx += kThreads)
        dS[(idx / K) * KP + idx % K] = a.dS_final ? a.dS_final[(size_t)u * V * K + idx] : 0.f;
    for (int idx = tid; idx < K * R; idx += kThreads) dAp[idx] = 0.f;
    for (int idx = tid; idx < R * V; idx += kThreads) dBp[idx] = 0.f;
    if (tid < R) dAwp[tid] = 0.f;
    if (tid < K) dtaup[tid] = 0.f;
    float dadec_acc = 0.f;   // this thread's channel (tid < K)

    // stage token t's vectors and gates into shared memory; S must hold S_{t-1}
    auto stage_and_gate = [&](int t) {
        const size_t row = (size_t)b * T + t;
        if (tid < K) {
            const size_t g = (row * H + h) * K + tid;
            qv[tid] = ld_io(q + g);
            kv[tid] = ld_io(kk + g);
            glv[tid] = a.g_logit[g];
            bxv[tid] = a.bx[g];
        }
        if (tid < V) vv[tid] = ld_io(vp + (row * H + h) * V + tid);
        if (tid == 0) wsc[0] = a.w_logit[row * H + h];
        __syncthreads();
        OP::row_dot(S, qv, mv);   // m_t = S_{t-1} q_t
        __syncthreads();
        content_signal<K, V>(Bh, Ah, mv, zv, delta, R);
        if (tid < K) {
            const float x = expf(log_retention(glv[tid], bxv[tid] + delta[tid], amp, decay_bias(a.tau, h, tid, K)));
            av[tid] = x;
            akv[tid] = x * kv[tid];
        }
        if (tid == 0) {
            float s = 0.f;
            if (a.Aw)
                for (int j = 0; j < R; ++j) s += a.Aw[(size_t)h * R + j] * zv[j];
            wsc[2] = s;                       // dw_c
            wsc[1] = sigmoid_f(wsc[0] + s);   // w
        }
        __syncthreads();
        OP::row_dot(S, akv, ev);   // S_{t-1} Diag(a) k; then e = v - that
        __syncthreads();
        if (tid < V) ev[tid] = vv[tid] - ev[tid];
        __syncthreads();
    };
    // block sum of x over threads tid < V (fixed order)
    auto sum_v = [&](float x) {
        if (tid < V) red[tid] = x;
        __syncthreads();
        float s = 0.f;
        if (tid == 0) {
            for (int j = 0; j < V; ++j) s += red[j];
        }
        return s;
    };

    for (int seg = NSEG - 1; seg >= 0; --seg) {
        const int t0 = seg * kSeg, t1 = min(T, t0 + kSeg);
        // recompute the segment: scratch[t - t0] = S_{t-1}
        const float *ck = a.saved_states + ((size_t)u * NSEG + seg) * V * K;
        for (int idx = tid; idx < V * K; idx += kThreads) S[(idx / K) * KP + idx % K] = ck[idx];
        __syncthreads();
        for (int t = t0; t < t1; ++t) {
            float *dst = scratch + (size_t)(t - t0) * V * K;
            for (int idx = tid; idx < V * K; idx += kThreads) dst[idx] = S[(idx / K) * KP + idx % K];
            stage_and_gate(t);
            const float w = wsc[1];
            for (int idx = tid; idx < V * K; idx += kThreads) {
                const int j = idx / K, i = idx % K;
                S[j * KP + i] = S[j * KP + i] * av[i] + w * ev[j] * kv[i];
            }
            __syncthreads();
        }
        // reverse sweep of the segment
        for (int t = t1 - 1; t >= t0; --t) {
            const float *src = scratch + (size_t)(t - t0) * V * K;
            for (int idx = tid; idx < V * K; idx += kThreads) S[(idx / K) * KP + idx % K] = src[idx];
            const size_t row = (size_t)b * T + t;
            if (tid < V) {
                float g = ld_io(dO + (row * H + h) * V + tid);
                if (t == T - 1 && a.dm_prev_out) g += a.dm_prev_out[(size_t)u * V + tid];   // m_prev_out = o_{T-1}
                dov[tid] = g;
            }
            __syncthreads();
            stage_and_gate(t);
            const float w = wsc[1];
            // o_t = S_t q_t:  dS_t += dO q^T
            for (int idx = tid; idx < V * K; idx += kThreads) {
                const int j = idx / K, i = idx % K;
                dS[j * KP + i] += dov[j] * qv[i];
            }
            __syncthreads();
            OP::row_dot(dS, kv, uv);   // u = dS_t k
            __syncthreads();
            const float dwp = sum_v(tid < V ? ev[tid] * uv[tid] : 0.f);          // dw = e . u
            __syncthreads();
            const float edo = sum_v(tid < V ? ev[tid] * dov[tid] : 0.f);         // e . dO
            if (tid == 0) {
                wsc[3] = dwp;
                wsc[4] = edo;
            }
            if (tid < V) {
                dev[tid] = w * uv[tid];   // de = w u
                st_io(dvp + (row * H + h) * V + tid, dev[tid]);
            }
            __syncthreads();
            // column sums over the value axis: c1 = S^T dO, c2 = dS^T e, c3 = S^T de, c4 = colsum(S .* dS)
            {
                const int i = tid % K, part = tid / K;
                float c1 = 0.f, c2 = 0.f, c3 = 0.f, c4 = 0.f;
                for (int j = part; j < V; j += TPC) {
                    const float sv = S[j * KP + i], dv = dS[j * KP + i];
                    c1 += sv * dov[j];
                    c2 += dv * ev[j];
                    c3 += sv * dev[j];
                    c4 += sv * dv;
                }
                cpart[(0 * TPC + part) * K + i] = c1;
                cpart[(1 * TPC + part) * K + i] = c2;
                cpart[(2 * TPC + part) * K + i] = c3;
                cpart[(3 * TPC + part) * K + i] = c4;
            }
            __syncthreads();
            if (tid < K) {
                float c[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    float s = 0.f;
                    for (int p2 = 0; p2 < TPC; ++p2) s += cpart[(x * TPC + p2) * K + tid];
                    c[x] = s;
                }
                const float ai = av[tid], ki = kv[tid];
                dqv[tid] = ai * c[0] + w * ki * wsc[4];                       // S_t^T dO
                st_io(dk + (row * H + h) * K + tid, w * c[1] - ai * c[2]);   // from w e k^T and e = v - P k
                const float da = c[3] - ki * c[2];                           // sum_j S_ji (dS - de k^T)_ji
                const float dla = da * ai;                                   // d log a
                const float x = glv[tid] + decay_bias(a.tau, h, tid, K);
                const float dgl = -amp * sigmoid_f(x) * dla;
                const size_t g = (row * H + h) * K + tid;
                a.dg_logit[g] = dgl;
                dtaup[tid] += dgl;
                dadec_acc += dla * (-amp * softplus_f(x));
                const float dbeta = dla * sigmoid_f(-(bxv[tid] + delta[tid]));
                a.dbx[g] = dbeta;
                ddelta[tid] = dbeta;
            }
            if (tid == 0) {
                const float dwl = wsc[3] * w * (1.f - w);
                a.dw_logit[row * H + h] = dwl;
                wsc[5] = dwl;   // gradient of dw_c
            }
            __syncthreads();
            // dS_{t-1} = (dS_t - de k^T) Diag(a)
            for (int idx = tid; idx < V * K; idx += kThreads) {
                const int j = idx / K, i = idx % K;
                dS[j * KP + i] = (dS[j * KP + i] - dev[j] * kv[i]) * av[i];
            }
            // content path: dz = A^T dDelta + Aw d(dw_c); dA += dDelta z^T; dB += dz m^T; dm = B^T dz
            for (int j0 = 0; j0 < R; j0 += kThreads / 8) {
                const int j = j0 + tid / 8, part = tid % 8;
                float s = 0.f;
                if (j < R)
                    for (int i = part; i < K; i += 8) s += Ah[(size_t)i * R + j] * ddelta[i];
                s += __shfl_xor_sync(0xffffffffu, s, 4);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                if (j < R && part == 0) dzv[j] = s + (a.Aw ? a.Aw[(size_t)h * R + j] * wsc[5] : 0.f);
            }
            __syncthreads();
            for (int idx = tid; idx < K * R; idx += kThreads) dAp[idx] += ddelta[idx / R] * zv[idx % R];
            for (int idx = tid; idx < R * V; idx += kThreads) dBp[idx] += dzv[idx / V] * mv[idx % V];
            if (a.Aw && tid < R) dAwp[tid] += wsc[5] * zv[tid];
            if (tid < V) {
                float s = 0.f;
                for (int j = 0; j < R; ++j) s += Bh[(size_t)j * V + tid] * dzv[j];
                dmv[tid] = s;
            }
            __syncthreads();
            // readout m = S_{t-1} q: dS_{t-1} += dm q^T; dq += S_{t-1}^T dm
            for (int idx = tid; idx < V * K; idx += kThreads) {
                const int j = idx / K, i = idx % K;
                dS[j * KP + i] += dmv[j] * qv[i];
            }
            {
                const int i = tid % K, part = tid / K;
                float c5 = 0.f;
                for (int j = part; j < V; j += TPC) c5 += S[j * KP + i] * dmv[j];
                cpart[(4 * TPC + part) * K + i] = c5;
            }
            __syncthreads();
            if (tid < K) {
                float s = 0.f;
                for (int p2 = 0; p2 < TPC; ++p2) s += cpart[(4 * TPC + p2) * K + tid];
                st_io(dq + (row * H + h) * K + tid, dqv[tid] + s);
            }
            __syncthreads();
        }
    }
    if (a.dS0)
        for (int idx = tid; idx < V * K; idx += kThreads) a.dS0[(size_t)u * V * K + idx] = dS[(idx / K) * KP + idx % K];
    if (a.dm_prev_in && tid < V) a.dm_prev_in[(size_t)u * V + tid] = 0.f;   // unused by this readout
    // the unit's record for the fixed-order reduction over the batch
    for (int idx = tid; idx < K * R; idx += kThreads) wsu[idx] = dAp[idx];
    for (int idx = tid; idx < R * V; idx += kThreads) wsu[K * R + idx] = dBp[idx];
    if (tid < R) wsu[K * R + R * V + tid] = dAwp[tid];
    if (tid < K) wsu[K * R + R * V + R + tid] = dtaup[tid];
    __syncthreads();
    if (tid < K) cpart[tid] = dadec_acc;
    __syncthreads();
    if (tid == 0) {
        float s = 0.f;
        for (int i = 0; i < K; ++i) s += cpart[i];
        wsu[K * R + R * V + R + K] = s;
    }
}

template <int K, int V, typename IO>
cudaError_t launch_exact_fwd_t(const FwdArgs &a, cudaStream_t st) {
    constexpr size_t bytes = sizeof(float) * (V * (K + 1) + 7 * K + 3 * V + 64 + 4);
    auto kern = exact_fwd_kernel<K, V, IO>;
    cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), (int)bytes);
    if (e != cudaSuccess) return e;
    kern<<<a.B * a.H, kThreads, bytes, st>>>(a);
    return cudaGetLastError();
}

template <int K, int V, typename IO>
cudaError_t launch_exact_bwd_t(const BwdArgs &a, float *dA, float *dB, cudaStream_t st) {
    constexpr size_t bytes = ExactBwdLayout<K, V>::bytes;
    auto kern = exact_bwd_kernel<K, V, IO>;
    cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), (int)bytes);
    if (e != cudaSuccess) return e;
    kern<<<a.B * a.H, kThreads, bytes, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_reduce_units(a.ws, dA, dB, a.dAw, a.dtau, a.dA_dec, a.B, a.H, K, V, a.R, st);
}

template <typename IO>
cudaError_t dispatch_exact_fwd(int K, int V, const FwdArgs &a, cudaStream_t st) {
    if (K == 64 && V == 64) return launch_exact_fwd_t<64, 64, IO>(a, st);
    if (K == 64 && V == 128) return launch_exact_fwd_t<64, 128, IO>(a, st);
    if (K == 128 && V == 64) return launch_exact_fwd_t<128, 64, IO>(a, st);
    return launch_exact_fwd_t<128, 128, IO>(a, st);
}

template <typename IO>
cudaError_t dispatch_exact_bwd(int K, int V, const BwdArgs &a, float *dA, float *dB, cudaStream_t st) {
    if (K == 64 && V == 64) return launch_exact_bwd_t<64, 64, IO>(a, dA, dB, st);
    if (K == 64 && V == 128) return launch_exact_bwd_t<64, 128, IO>(a, dA, dB, st);
    if (K == 128 && V == 64) return launch_exact_bwd_t<128, 64, IO>(a, dA, dB, st);
    return launch_exact_bwd_t<128, 128, IO>(a, dA, dB, st);
}

cudaError_t launch_fwd_exact(int K, int V, bool bf16, const FwdArgs &a, cudaStream_t st) {
    return bf16 ? dispatch_exact_fwd<__nv_bfloat16>(K, V, a, st) : dispatch_exact_fwd<float>(K, V, a, st);
}

cudaError_t launch_bwd_exact(int K, int V, bool bf16, const BwdArgs &a, float *dA, float *dB, cudaStream_t st) {
    return bf16 ? dispatch_exact_bwd<__nv_bfloat16>(K, V, a, dA, dB, st)
                : dispatch_exact_bwd<float>(K, V, a, dA, dB, st);
}

int exact_segment() { return kSeg; }

}  // namespace carve

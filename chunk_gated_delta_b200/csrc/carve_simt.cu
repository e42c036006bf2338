// CARVE chunk-parallel WY forward and reverse-sweep backward, SIMT fp32-accumulate kernels.
//
// One CTA per (batch, head) unit sweeps the sequence chunk by chunk: the erase gate of chunk
// c depends on the state at the end of chunk c-1 (CARVE paperdance abstract: content signal
// read once per chunk from the chunk-boundary state), so chunks are serial per unit.  Inside
// a gate chunk the tokens are processed in compute sub-chunks of 16 in WY form (CARVE blog,
// section 2.3: the key-axis retention gamma does not depend on the value index, so one
// triangular system per sub-chunk serves every value channel):
//
//   Lam_t   = sum_{s<=t} log a_s                      (relative to the sub-chunk start)
//   Akk[t,s]= sum_i k_t,i k_s,i exp(Lam_t,i - Lam_s,i)    s <  t
//   Aqk[t,s]= sum_i q_t,i k_s,i exp(Lam_t,i - Lam_s,i)    s <= t
//   (I + Diag(w) Akk) U = Diag(w) (V - Kt S0^T),   Kt = k*exp(Lam), Qt = q*exp(Lam)
//   O  = Qt S0^T + Aqk U ;   S1 = S0 Diag(exp(Lam_15)) + U^T Kb,   Kb = k*exp(Lam_15 - Lam)
//
// Every exponent above is <= 0, so no decay is ever inverted and nothing overflows whatever
// the gate values.  All arithmetic is fp32; q/k/v/o and their gradients are loaded/stored in
// the I/O dtype (fp32 or bf16).  These kernels serve the fp32 mode and every shape; the
// tensor-core kernels specialise the bf16, d = 128 path.
#include "carve_device.cuh"

namespace carve {

__device__ int g_simt_bad_seqlens;   // set when a sequence's offsets are out of range

// Device status word of the sequence offsets (SIMT kernels): returns and clears it.
int simt_take_bad_seqlens() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_simt_bad_seqlens, sizeof(int)) != cudaSuccess) return 0;
    if (v) {
        const int z = 0;
        cudaMemcpyToSymbol(g_simt_bad_seqlens, &z, sizeof(int));
    }
    return v;
}

__device__ __forceinline__ size_t tk(int b, int t, int h, int i, int T, int H, int W) {
    return (((size_t)b * T + t) * H + h) * W + i;
}

template <int K, int V>
struct FwdSmem {
    static constexpr int KP = K + 1, VP = V + 1;
    static constexpr int floats = V * KP + 3 * kSub * KP + 3 * kSub * K + 3 * kSub * VP +
                                  2 * kSub * 17 + kSub + 3 * K + 3 * V + 64 + 4;
    static constexpr size_t bytes = sizeof(float) * floats;
};

template <int K, int V, typename IO>
__global__ void __launch_bounds__(kThreads, 1) fwd_simt_kernel(FwdArgs a) {
    using SM = FwdSmem<K, V>;
    constexpr int KP = SM::KP, VP = SM::VP;
    extern __shared__ __align__(16) float sm[];
    float *S = sm;                   // [V][KP] state (fp32 master)
    float *qs = S + V * KP;          // [16][KP]
    float *ks = qs + kSub * KP;      // [16][KP]
    float *lam = ks + kSub * KP;     // [16][KP] log retention, then its cumulative sum
    float *Qt = lam + kSub * KP;     // [16][K]
    float *Kt = Qt + kSub * K;       // [16][K]
    float *Kb = Kt + kSub * K;       // [16][K]
    float *vs = Kb + kSub * K;       // [16][VP] v, then R = v - Kt S0^T
    float *Us = vs + kSub * VP;      // [16][VP]
    float *Oi = Us + kSub * VP;      // [16][VP]
    float *Akk = Oi + kSub * VP;     // [16][17]
    float *Aqk = Akk + kSub * 17;    // [16][17]
    float *wv = Aqk + kSub * 17;     // [16]
    float *gam = wv + kSub;          // [K]
    float *delta = gam + K;          // [K]
    float *qbar = delta + K;         // [K]
    float *mvec = qbar + K;          // [V]
    float *osum = mvec + V;          // [V]
    float *mprev = osum + V;         // [V]
    float *zvec = mprev + V;         // [64]
    float *wsc = zvec + 64;          // [4]: the write gate's content term dw_c

    const int tid = threadIdx.x;
    const int u = blockIdx.x, H = a.H, T = a.T, R = a.R, L = a.L;
    const int b = u / H, h = u % H;
    const float amp = decay_amp(a.A_dec, h);   // e^{A_dec[h]}, 1 without the decay amplitude
    const int NC = (T + L - 1) / L, NS = T / kSub;   // record strides (T bounds every sequence)
    int bb, toff, Tn;   // this unit's tokens: rows [toff, toff + Tn) of tensor batch bb
    seq_tokens(a.cu_seqlens, a.total, T, b, bb, toff, Tn, &g_simt_bad_seqlens);
    const int NCn = (Tn + L - 1) / L;
    const IO *q = static_cast<const IO *>(a.q), *kk = static_cast<const IO *>(a.k);
    const IO *vv = static_cast<const IO *>(a.v);
    IO *o = static_cast<IO *>(a.o);

    for (int idx = tid; idx < V * K; idx += kThreads) {
        const int r = idx / K, i = idx % K;
        S[r * KP + i] = a.S0 ? a.S0[(size_t)u * V * K + idx] : 0.f;
    }
    if (tid < V) mprev[tid] = a.m_prev_in ? a.m_prev_in[(size_t)u * V + tid] : 0.f;
    __syncthreads();

    int sidx = 0;
    for (int c = 0; c < NCn; ++c) {
        const int t0 = c * L, n = min(L, Tn - t0);
        // ---- content signal of the chunk: m_c, z = Bm m_c, Delta = A z
        if (a.mc_mode == 0) {
            if (tid < K) {
                float s = 0.f;
                for (int t = t0; t < t0 + n; ++t) s += ld_io(q + tk(bb, toff + t, h, tid, T, H, K));
                qbar[tid] = s / (float)n;
            }
            __syncthreads();
            if (tid < V) {
                float m = 0.f;
                for (int i = 0; i < K; ++i) m += S[tid * KP + i] * qbar[i];
                mvec[tid] = m;
            }
        } else if (tid < V) {
            mvec[tid] = mprev[tid];
        }
        __syncthreads();
        content_signal<K, V>(a.Bm + (size_t)h * R * V, a.A + (size_t)h * K * R, mvec, zvec, delta, R);
        if (tid < V) osum[tid] = 0.f;
        if (tid == 0) {   // dw_c = Aw . z (the same projection of m_c biases the write gate)
            float s = 0.f;
            if (a.Aw)
                for (int j = 0; j < R; ++j) s += a.Aw[(size_t)h * R + j] * zvec[j];
            wsc[0] = s;
        }
        __syncthreads();
        if (a.saved_aux) {
            float *aux = a.saved_aux + ((size_t)u * NC + c) * (V + R + K);
            if (tid < V) aux[tid] = mvec[tid];
            if (tid < R) aux[V + tid] = zvec[tid];
            if (tid < K) aux[V + R + tid] = delta[tid];
        }

        for (int s0 = t0; s0 < t0 + n; s0 += kSub, ++sidx) {
            if (a.saved_states) {
                float *st = a.saved_states + ((size_t)u * NS + sidx) * V * K;
                for (int idx = tid; idx < V * K; idx += kThreads) st[idx] = S[(idx / K) * KP + idx % K];
            }
            // ---- load the sub-chunk, gate activations; rows past the sequence's end (nv <= t) are
            //      inert: q = k = v = 0, a = 1, w = 0, so they leave the state unchanged
            const int nv = min(kSub, t0 + n - s0);
            for (int idx = tid; idx < kSub * K; idx += kThreads) {
                const int t = idx / K, i = idx % K;
                const size_t g = tk(bb, toff + s0 + t, h, i, T, H, K);
                const bool in = t < nv;
                qs[t * KP + i] = in ? ld_io(q + g) : 0.f;
                ks[t * KP + i] = in ? ld_io(kk + g) : 0.f;
                lam[t * KP + i] =
                    in ? log_retention(a.g_logit[g], a.bx[g] + delta[i], amp, decay_bias(a.tau, h, i, K)) : 0.f;
            }
            for (int idx = tid; idx < kSub * V; idx += kThreads) {
                const int t = idx / V, r = idx % V;
                vs[t * VP + r] = t < nv ? ld_io(vv + tk(bb, toff + s0 + t, h, r, T, H, V)) : 0.f;
            }
            if (tid < kSub)
                wv[tid] = tid < nv ? sigmoid_f(a.w_logit[((size_t)bb * T + toff + s0 + tid) * H + h] + wsc[0]) : 0.f;
            __syncthreads();
            if (tid < K) {
                float run = 0.f;
                for (int t = 0; t < kSub; ++t) {
                    run += lam[t * KP + tid];
                    lam[t * KP + tid] = run;
                }
                gam[tid] = expf(run);
            }
            __syncthreads();
            // ---- decayed operands and the intra-sub-chunk Gram matrices
            for (int idx = tid; idx < kSub * K; idx += kThreads) {
                const int t = idx / K, i = idx % K;
                const float l = lam[t * KP + i], e = expf(l);
                Qt[t * K + i] = qs[t * KP + i] * e;
                Kt[t * K + i] = ks[t * KP + i] * e;
                Kb[t * K + i] = ks[t * KP + i] * expf(lam[(kSub - 1) * KP + i] - l);
            }
            {
                const int t = tid / kSub, s = tid % kSub;
                float aqk = 0.f, akk = 0.f;
                if (s <= t) {
                    for (int i = 0; i < K; ++i) {
                        const float ksE = ks[s * KP + i] * expf(lam[t * KP + i] - lam[s * KP + i]);
                        aqk += qs[t * KP + i] * ksE;
                        akk += ks[t * KP + i] * ksE;
                    }
                }
                Aqk[t * 17 + s] = aqk;
                Akk[t * 17 + s] = (s < t) ? akk : 0.f;
            }
            __syncthreads();
            // ---- R = v - Kt S0^T and Oi = Qt S0^T
            {
                constexpr int G = kThreads / V, RPG = 2 * kSub / G;
                const int r = tid % V, g = tid / V;
                float acc[RPG];
#pragma unroll
                for (int x = 0; x < RPG; ++x) acc[x] = 0.f;
                const float *X = (g * RPG < kSub) ? Kt + g * RPG * K : Qt + (g * RPG - kSub) * K;
                for (int i = 0; i < K; ++i) {
                    const float sv = S[r * KP + i];
#pragma unroll
                    for (int x = 0; x < RPG; ++x) acc[x] += X[x * K + i] * sv;
                }
#pragma unroll
                for (int x = 0; x < RPG; ++x) {
                    const int row = g * RPG + x;
                    if (row < kSub) vs[row * VP + r] -= acc[x];
                    else Oi[(row - kSub) * VP + r] = acc[x];
                }
            }
            __syncthreads();
            // ---- WY solve, one column (value channel) per thread
            if (tid < V) {
                float uu[kSub];
#pragma unroll
                for (int t = 0; t < kSub; ++t) {
                    float x = vs[t * VP + tid];
#pragma unroll
                    for (int s = 0; s < t; ++s) x -= Akk[t * 17 + s] * uu[s];
                    uu[t] = wv[t] * x;
                    Us[t * VP + tid] = uu[t];
                }
            }
            __syncthreads();
            // ---- outputs O = Oi + Aqk U
            for (int idx = tid; idx < kSub * V; idx += kThreads) {
                const int t = idx / V, r = idx % V;
                float x = Oi[t * VP + r];
                for (int s = 0; s <= t; ++s) x += Aqk[t * 17 + s] * Us[s * VP + r];
                Oi[t * VP + r] = x;
                if (t < nv) st_io(o + tk(bb, toff + s0 + t, h, r, T, H, V), x);
            }
            __syncthreads();
            if (tid < V)
                for (int t = 0; t < kSub; ++t) osum[tid] += Oi[t * VP + tid];
            // ---- state update S = S Diag(gamma) + U^T Kb
            for (int idx = tid; idx < V * K; idx += kThreads) {
                const int r = idx / K, i = idx % K;
                float x = S[r * KP + i] * gam[i];
#pragma unroll
                for (int s = 0; s < kSub; ++s) x += Us[s * VP + r] * Kb[s * K + i];
                S[r * KP + i] = x;
            }
            __syncthreads();
        }
        if (tid < V) mprev[tid] = osum[tid] / (float)n;
        __syncthreads();
    }
    if (a.S_final)
        for (int idx = tid; idx < V * K; idx += kThreads)
            a.S_final[(size_t)u * V * K + idx] = S[(idx / K) * KP + idx % K];
    if (a.m_prev_out && tid < V) a.m_prev_out[(size_t)u * V + tid] = mprev[tid];
}

template <int K, int V>
struct BwdSmem {
    static constexpr int KP = K + 1, VP = V + 1;
    static constexpr int floats = V * KP + 6 * kSub * KP + 3 * kSub * K + 4 * kSub * VP +
                                  4 * kSub * 17 + 2 * kSub + 5 * K + 3 * V + 2 * 64 + 4;
    static constexpr size_t bytes = sizeof(float) * floats;
};

template <int K, int V, typename IO>
__global__ void __launch_bounds__(kThreads, 1) bwd_simt_kernel(BwdArgs a) {
    using SM = BwdSmem<K, V>;
    constexpr int KP = SM::KP, VP = SM::VP;
    extern __shared__ __align__(16) float sm[];
    float *dS = sm;                  // [V][KP] state gradient (carried backwards)
    float *qs = dS + V * KP;         // [16][KP]
    float *ks = qs + kSub * KP;
    float *lam = ks + kSub * KP;
    float *dqs = lam + kSub * KP;    // [16][KP]
    float *dks = dqs + kSub * KP;
    float *dls = dks + kSub * KP;
    float *Qt = dls + kSub * KP;     // [16][K]
    float *Kt = Qt + kSub * K;
    float *Kb = Kt + kSub * K;
    float *Rs = Kb + kSub * K;       // [16][VP]
    float *Us = Rs + kSub * VP;
    float *dOs = Us + kSub * VP;
    float *dYs = dOs + kSub * VP;
    float *Akk = dYs + kSub * VP;    // [16][17]
    float *Aqk = Akk + kSub * 17;
    float *dAqk = Aqk + kSub * 17;
    float *dAkk = dAqk + kSub * 17;
    float *wv = dAkk + kSub * 17;    // [16]
    float *dwv = wv + kSub;          // [16]
    float *gam = dwv + kSub;         // [K]
    float *dgam = gam + K;
    float *delta = dgam + K;
    float *ddelta = delta + K;
    float *vecK = ddelta + K;        // [K] chunk mean of q, then the readout term of dq
    float *mvec = vecK + K;          // [V]
    float *dmv = mvec + V;           // [V]
    float *dox = dmv + V;            // [V] extra output gradient of the chunk (mc_mode 1)
    float *zvec = dox + V;           // [64]
    float *dzv = zvec + 64;          // [64]
    float *wsc = dzv + 64;           // [4]: dw_c and the gradient accumulated for it

    const int tid = threadIdx.x;
    const int u = blockIdx.x, H = a.H, T = a.T, R = a.R, L = a.L;
    const int b = u / H, h = u % H;
    const int NC = (T + L - 1) / L, NS = T / kSub;
    const IO *q = static_cast<const IO *>(a.q), *kk = static_cast<const IO *>(a.k);
    const IO *vv = static_cast<const IO *>(a.v), *dO = static_cast<const IO *>(a.dO);
    IO *dq = static_cast<IO *>(a.dq), *dk = static_cast<IO *>(a.dk), *dv = static_cast<IO *>(a.dv);
    // per-unit partials: dA [K*R], dB [R*V], dAw [R], dtau [K], dA_dec [1]
    const int rec = K * R + R * V + R + K + 1;
    float *wsu = a.ws + (size_t)u * rec;
    int bb, toff, Tn;   // this unit's tokens: rows [toff, toff + Tn) of tensor batch bb
    seq_tokens(a.cu_seqlens, a.total, T, b, bb, toff, Tn, &g_simt_bad_seqlens);
    const int NCn = (Tn + L - 1) / L;
    const float amp = decay_amp(a.A_dec, h);
    float dtau_acc = 0.f, dadec_acc = 0.f;   // this thread's channel (tid < K), over the sweep

    for (int idx = tid; idx < V * K; idx += kThreads)
        dS[(idx / K) * KP + idx % K] = a.dS_final ? a.dS_final[(size_t)u * V * K + idx] : 0.f;
    if (tid < V) {
        const int nl = Tn - (NCn - 1) * L;
        dox[tid] = a.dm_prev_out ? a.dm_prev_out[(size_t)u * V + tid] / (float)nl : 0.f;
    }
    for (int idx = tid; idx < rec; idx += kThreads) wsu[idx] = 0.f;
    __syncthreads();

    for (int c = NCn - 1; c >= 0; --c) {
        const int t0 = c * L, n = min(L, Tn - t0), nsub = (n + kSub - 1) / kSub, sub0 = t0 / kSub;
        {
            const float *aux = a.saved_aux + ((size_t)u * NC + c) * (V + R + K);
            if (tid < V) mvec[tid] = aux[tid];
            if (tid < R) zvec[tid] = aux[V + tid];
            if (tid < K) {
                delta[tid] = aux[V + R + tid];
                ddelta[tid] = 0.f;
            }
        }
        __syncthreads();
        if (tid == 0) {   // dw_c = Aw . z, and its gradient starts at 0
            float s = 0.f;
            if (a.Aw)
                for (int j = 0; j < R; ++j) s += a.Aw[(size_t)h * R + j] * zvec[j];
            wsc[0] = s;
            wsc[1] = 0.f;
        }
        __syncthreads();
        for (int jj = nsub - 1; jj >= 0; --jj) {
            const int s0 = t0 + jj * kSub;
            const float *S0g = a.saved_states + ((size_t)u * NS + sub0 + jj) * V * K;
            // ---- recompute the sub-chunk's forward quantities (rows nv.. past the sequence's end
            //      are inert, as in the forward, and carry no output gradient)
            const int nv = min(kSub, t0 + n - s0);
            for (int idx = tid; idx < kSub * K; idx += kThreads) {
                const int t = idx / K, i = idx % K;
                const size_t g = tk(bb, toff + s0 + t, h, i, T, H, K);
                const bool in = t < nv;
                qs[t * KP + i] = in ? ld_io(q + g) : 0.f;
                ks[t * KP + i] = in ? ld_io(kk + g) : 0.f;
                lam[t * KP + i] =
                    in ? log_retention(a.g_logit[g], a.bx[g] + delta[i], amp, decay_bias(a.tau, h, i, K)) : 0.f;
            }
            for (int idx = tid; idx < kSub * V; idx += kThreads) {
                const int t = idx / V, r = idx % V;
                const bool in = t < nv;
                Rs[t * VP + r] = in ? ld_io(vv + tk(bb, toff + s0 + t, h, r, T, H, V)) : 0.f;
                dOs[t * VP + r] = in ? ld_io(dO + tk(bb, toff + s0 + t, h, r, T, H, V)) + dox[r] : 0.f;
            }
            if (tid < kSub)
                wv[tid] = tid < nv ? sigmoid_f(a.w_logit[((size_t)bb * T + toff + s0 + tid) * H + h] + wsc[0]) : 0.f;
            __syncthreads();
            if (tid < K) {
                float run = 0.f;
                for (int t = 0; t < kSub; ++t) {
                    run += lam[t * KP + tid];
                    lam[t * KP + tid] = run;
                }
                gam[tid] = expf(run);
            }
            __syncthreads();
            for (int idx = tid; idx < kSub * K; idx += kThreads) {
                const int t = idx / K, i = idx % K;
                const float l = lam[t * KP + i], e = expf(l);
                Qt[t * K + i] = qs[t * KP + i] * e;
                Kt[t * K + i] = ks[t * KP + i] * e;
                Kb[t * K + i] = ks[t * KP + i] * expf(lam[(kSub - 1) * KP + i] - l);
            }
            {
                const int t = tid / kSub, s = tid % kSub;
                float aqk = 0.f, akk = 0.f;
                if (s <= t) {
                    for (int i = 0; i < K; ++i) {
                        const float ksE = ks[s * KP + i] * expf(lam[t * KP + i] - lam[s * KP + i]);
                        aqk += qs[t * KP + i] * ksE;
                        akk += ks[t * KP + i] * ksE;
                    }
                }
                Aqk[t * 17 + s] = aqk;
                Akk[t * 17 + s] = (s < t) ? akk : 0.f;
            }
            __syncthreads();
            // R = v - Kt S0^T (S0 read from the saved states)
            if (tid < V) {
                float acc[kSub];
#pragma unroll
                for (int t = 0; t < kSub; ++t) acc[t] = 0.f;
                for (int i = 0; i < K; ++i) {
                    const float sv = S0g[(size_t)tid * K + i];
#pragma unroll
                    for (int t = 0; t < kSub; ++t) acc[t] += Kt[t * K + i] * sv;
                }
#pragma unroll
                for (int t = 0; t < kSub; ++t) Rs[t * VP + tid] -= acc[t];
            }
            __syncthreads();
            // U = (I + Diag(w) Akk)^-1 Diag(w) R;   dU = Aqk^T dO + Kb dS1^T;  dY = M^-T dU
            if (tid < V) {
                float uu[kSub];
#pragma unroll
                for (int t = 0; t < kSub; ++t) {
                    float x = Rs[t * VP + tid];
#pragma unroll
                    for (int s = 0; s < t; ++s) x -= Akk[t * 17 + s] * uu[s];
                    uu[t] = wv[t] * x;
                    Us[t * VP + tid] = uu[t];
                }
                float acc[kSub];
#pragma unroll
                for (int s = 0; s < kSub; ++s) acc[s] = 0.f;
                for (int i = 0; i < K; ++i) {
                    const float d = dS[tid * KP + i];
#pragma unroll
                    for (int s = 0; s < kSub; ++s) acc[s] += Kb[s * K + i] * d;
                }
#pragma unroll
                for (int s = 0; s < kSub; ++s)
#pragma unroll
                    for (int t = s; t < kSub; ++t) acc[s] += Aqk[t * 17 + s] * dOs[t * VP + tid];
#pragma unroll
                for (int s = kSub - 1; s >= 0; --s) {
#pragma unroll
                    for (int t = s + 1; t < kSub; ++t) acc[s] -= wv[t] * Akk[t * 17 + s] * acc[t];
                }
#pragma unroll
                for (int t = 0; t < kSub; ++t) {
                    dYs[t * VP + tid] = acc[t];
                    if (t < nv) st_io(dv + tk(bb, toff + s0 + t, h, tid, T, H, V), wv[t] * acc[t]);   // dv = w dY
                }
            }
            __syncthreads();
            // dAqk = tril(dO U^T),  dM = -tril(dY U^T, -1),  dAkk = Diag(w) dM,
            // dw = rowsum(dM * Akk) + rowsum(dY * R)
            {
                const int t = tid / kSub, s = tid % kSub;
                float a1 = 0.f, a2 = 0.f, a3 = 0.f;
                if (s <= t) {
                    for (int r = 0; r < V; ++r) {
                        const float us = Us[s * VP + r];
                        a1 += dOs[t * VP + r] * us;
                        a2 += dYs[t * VP + r] * us;
                        if (s == t) a3 += dYs[t * VP + r] * Rs[t * VP + r];
                    }
                }
                const float dM = (s < t) ? -a2 : 0.f;
                dAqk[t * 17 + s] = (s <= t) ? a1 : 0.f;
                dAkk[t * 17 + s] = wv[t] * dM;
                float cw = dM * Akk[t * 17 + s] + a3;
#pragma unroll
                for (int off = 8; off >= 1; off >>= 1) cw += __shfl_xor_sync(0xffffffffu, cw, off);
                if (s == 0) dwv[t] = cw;
            }
            __syncthreads();
            if (tid < 32) {   // d w_logit, and its sum over the sub-chunk for dw_c
                float x = 0.f;
                if (tid < kSub) {
                    const float w = wv[tid];
                    x = dwv[tid] * w * (1.f - w);
                    if (tid < nv) a.dw_logit[((size_t)bb * T + toff + s0 + tid) * H + h] = x;
                }
#pragma unroll
                for (int off = 8; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
                if (tid == 0) wsc[1] += x;
            }
            // [dQt; dKt] = [dO; -dR] S0,  dKb = U dS1,  dgamma = colsum(S0 * dS1)
            {
                constexpr int G = kThreads / K, RX = 2 * kSub / G, RU = kSub / G;
                const int i = tid % K, g = tid / K;
                float ax[RX], au[RU], ag = 0.f;
#pragma unroll
                for (int x = 0; x < RX; ++x) ax[x] = 0.f;
#pragma unroll
                for (int x = 0; x < RU; ++x) au[x] = 0.f;
                for (int r = 0; r < V; ++r) {
                    const float s0v = S0g[(size_t)r * K + i], dsv = dS[r * KP + i];
#pragma unroll
                    for (int x = 0; x < RX; ++x) {
                        const int row = g * RX + x;
                        const float xv = row < kSub ? dOs[row * VP + r] : -wv[row - kSub] * dYs[(row - kSub) * VP + r];
                        ax[x] += xv * s0v;
                    }
#pragma unroll
                    for (int x = 0; x < RU; ++x) au[x] += Us[(g * RU + x) * VP + r] * dsv;
                    ag += s0v * dsv;
                }
#pragma unroll
                for (int x = 0; x < RX; ++x) {
                    const int row = g * RX + x;
                    if (row < kSub) dqs[row * KP + i] = ax[x];           // raw dQt
                    else dks[(row - kSub) * KP + i] = ax[x];              // raw dKt
                }
#pragma unroll
                for (int x = 0; x < RU; ++x) dls[(g * RU + x) * KP + i] = au[x];   // raw dKb
                if (g == 0) dgam[i] = ag;
            }
            __syncthreads();
            // d Lam_15 gathers the gamma and Kb terms: dgamma*gamma + sum_s dKb_s * Kb_s
            if (tid < K) {
                float cs = 0.f;
                for (int s = 0; s < kSub; ++s) cs += dls[s * KP + tid] * Kb[s * K + tid];
                dgam[tid] = dgam[tid] * gam[tid] + cs;
            }
            // dS0 = dS1 Diag(gamma) + dO^T Qt - dR^T Kt   (in place)
            for (int idx = tid; idx < V * K; idx += kThreads) {
                const int r = idx / K, i = idx % K;
                float x = dS[r * KP + i] * gam[i];
#pragma unroll
                for (int t = 0; t < kSub; ++t)
                    x += dOs[t * VP + r] * Qt[t * K + i] - wv[t] * dYs[t * VP + r] * Kt[t * K + i];
                dS[r * KP + i] = x;
            }
            __syncthreads();
            // per-element gradients of q, k and Lam (decay factors recomputed exactly)
            for (int idx = tid; idx < kSub * K; idx += kThreads) {
                const int t = idx / K, i = idx % K;
                const float lt = lam[t * KP + i], e = expf(lt), eb = expf(lam[(kSub - 1) * KP + i] - lt);
                const float dQt = dqs[t * KP + i], dKt = dks[t * KP + i], dKb = dls[t * KP + i];
                const float qv = qs[t * KP + i], kv = ks[t * KP + i];
                float gq = dQt * e, gk = dKt * e + dKb * eb;
                float gl = dQt * Qt[t * K + i] + dKt * Kt[t * K + i] - dKb * Kb[t * K + i];
                if (t == kSub - 1) gl += dgam[i];
                // t as the row token of Aqk / Akk
                float dqa = 0.f, dkr = 0.f;
                for (int s = 0; s <= t; ++s) {
                    const float ksE = ks[s * KP + i] * expf(lt - lam[s * KP + i]);
                    dqa += dAqk[t * 17 + s] * ksE;
                    dkr += dAkk[t * 17 + s] * ksE;
                }
                // t as the column token
                float dkc = 0.f;
                for (int tt = t; tt < kSub; ++tt) {
                    const float E = expf(lam[tt * KP + i] - lt);
                    dkc += (dAqk[tt * 17 + t] * qs[tt * KP + i] + dAkk[tt * 17 + t] * ks[tt * KP + i]) * E;
                }
                gq += dqa;
                gk += dkr + dkc;
                gl += qv * dqa + kv * dkr - kv * dkc;
                dqs[t * KP + i] = gq;   // (t,i) is read and written by this thread only
                dks[t * KP + i] = gk;
                dls[t * KP + i] = gl;
            }
            __syncthreads();
            // reverse cumulative sum of dLam -> dlog a -> gate gradients
            if (tid < K) {
                float run = 0.f;
                for (int t = kSub - 1; t >= 0; --t) {
                    run += dls[t * KP + tid];   // inert rows carry the chunk-decay term to the others
                    if (t >= nv) continue;
                    const size_t g = tk(bb, toff + s0 + t, h, tid, T, H, K);
                    const float beta = a.bx[g] + delta[tid];
                    // log g = -amp softplus(g_logit + tau): d/dg_logit = d/dtau = -amp sigmoid(.),
                    // d/dA_dec = log g
                    const float x = a.g_logit[g] + decay_bias(a.tau, h, tid, K);
                    const float dgl = -amp * sigmoid_f(x) * run;
                    a.dg_logit[g] = dgl;
                    dtau_acc += dgl;
                    dadec_acc += run * (-amp * softplus_f(x));
                    const float dbeta = sigmoid_f(-beta) * run;
                    a.dbx[g] = dbeta;
                    ddelta[tid] += dbeta;
                }
            }
            for (int idx = tid; idx < nv * K; idx += kThreads) {
                const int t = idx / K, i = idx % K;
                const size_t g = tk(bb, toff + s0 + t, h, i, T, H, K);
                st_io(dq + g, dqs[t * KP + i]);
                st_io(dk + g, dks[t * KP + i]);
            }
            __syncthreads();
        }
        // ---- chunk start: Delta = A z, z = Bm m
        for (int j0 = 0; j0 < R; j0 += kThreads / 8) {   // dz = A^T dDelta, 8 threads per output
            const int j = j0 + tid / 8, part = tid % 8;
            float s = 0.f;
            if (j < R)
#pragma unroll
                for (int i = part; i < K; i += 8) s += a.A[((size_t)h * K + i) * R + j] * ddelta[i];
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            if (j < R && part == 0) dzv[j] = s + (a.Aw ? a.Aw[(size_t)h * R + j] * wsc[1] : 0.f);
        }
        __syncthreads();
        if (a.Aw && tid < R) wsu[K * R + R * V + tid] += wsc[1] * zvec[tid];
        for (int idx = tid; idx < K * R; idx += kThreads) wsu[idx] += ddelta[idx / R] * zvec[idx % R];
        for (int idx = tid; idx < R * V; idx += kThreads) wsu[K * R + idx] += dzv[idx / V] * mvec[idx % V];
        if (tid < V) {
            float s = 0.f;
#pragma unroll 8
            for (int j = 0; j < R; ++j) s += a.Bm[((size_t)h * R + j) * V + tid] * dzv[j];
            dmv[tid] = s;
        }
        __syncthreads();
        if (a.mc_mode == 0) {
            // m = S_[c-1] qbar:  dS_[c-1] += dm qbar^T,  dq_t += S_[c-1]^T dm / n  (t in chunk)
            if (tid < K) {
                float s = 0.f;
                for (int t = t0; t < t0 + n; ++t) s += ld_io(q + tk(bb, toff + t, h, tid, T, H, K));
                vecK[tid] = s / (float)n;
            }
            __syncthreads();
            for (int idx = tid; idx < V * K; idx += kThreads) {
                const int r = idx / K, i = idx % K;
                dS[r * KP + i] += dmv[r] * vecK[i];
            }
            __syncthreads();
            if (tid < K) {
                const float *Sc = a.saved_states + ((size_t)u * NS + sub0) * V * K;
                float s = 0.f;
                for (int r = 0; r < V; ++r) s += Sc[(size_t)r * K + tid] * dmv[r];
                vecK[tid] = s / (float)n;
            }
            __syncthreads();
            for (int idx = tid; idx < n * K; idx += kThreads) {
                const size_t g = tk(bb, toff + t0 + idx / K, h, idx % K, T, H, K);
                st_io(dq + g, ld_io(dq + g) + vecK[idx % K]);
            }
            if (tid < V) dox[tid] = 0.f;
        } else if (tid < V) {
            dox[tid] = c > 0 ? dmv[tid] / (float)L : 0.f;
            if (c == 0 && a.dm_prev_in) a.dm_prev_in[(size_t)u * V + tid] = dmv[tid];
        }
        __syncthreads();
    }
    if (a.dS0)
        for (int idx = tid; idx < V * K; idx += kThreads) a.dS0[(size_t)u * V * K + idx] = dS[(idx / K) * KP + idx % K];
    if (a.dm_prev_in && tid < V) {
        if (NCn == 0)   // no token: m_prev_out is m_prev_in passed through
            a.dm_prev_in[(size_t)u * V + tid] = a.dm_prev_out ? a.dm_prev_out[(size_t)u * V + tid] : 0.f;
        else if (a.mc_mode == 0)
            a.dm_prev_in[(size_t)u * V + tid] = 0.f;
    }
    if (a.A_dec || a.tau) {   // the decay parameters' partials of this unit (fixed-order sum)
        if (tid < K) {
            wsu[K * R + R * V + R + tid] = dtau_acc;
            vecK[tid] = dadec_acc;
        }
        __syncthreads();
        if (tid == 0) {
            float s = 0.f;
            for (int i = 0; i < K; ++i) s += vecK[i];
            wsu[K * R + R * V + R + K] = s;
        }
    }
}

// Per-head sums over b (fixed order) of the unit records [dA K*R | dB R*V | dAw R | dtau K | dA_dec 1]
__global__ void reduce_dAdB_kernel(const float *ws, float *dA, float *dB, float *dAw, float *dtau, float *dA_dec,
                                   int B, int H, int KR, int RV, int R, int K) {
    const int h = blockIdx.y;
    const int x = blockIdx.x * blockDim.x + threadIdx.x;
    const int rec = KR + RV + R + K + 1;
    if (x >= rec) return;
    float s = 0.f;
    for (int b = 0; b < B; ++b) s += ws[((size_t)b * H + h) * rec + x];
    if (x < KR) dA[(size_t)h * KR + x] = s;
    else if (x < KR + RV) dB[(size_t)h * RV + (x - KR)] = s;
    else if (x < KR + RV + R) {
        if (dAw) dAw[(size_t)h * R + (x - KR - RV)] = s;
    } else if (x < rec - 1) {
        if (dtau) dtau[(size_t)h * K + (x - KR - RV - R)] = s;
    } else if (dA_dec) {
        dA_dec[h] = s;
    }
}

// Host: the reduction above over per-unit records of K*R + R*V + R + K + 1 floats (also used
// by the exact-recurrence backward).
cudaError_t launch_reduce_units(const float *ws, float *dA, float *dB, float *dAw, float *dtau, float *dA_dec, int B,
                                int H, int K, int V, int R, cudaStream_t st) {
    const int KR = K * R, RV = R * V;
    dim3 grid((KR + RV + R + K + 1 + 255) / 256, H);
    reduce_dAdB_kernel<<<grid, 256, 0, st>>>(ws, dA, dB, dAw, dtau, dA_dec, B, H, KR, RV, R, K);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
template <int K, int V, typename IO>
cudaError_t launch_fwd_simt_t(const FwdArgs &a, cudaStream_t st) {
    auto kern = fwd_simt_kernel<K, V, IO>;
    cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), (int)FwdSmem<K, V>::bytes);
    if (e != cudaSuccess) return e;
    kern<<<a.B * a.H, kThreads, FwdSmem<K, V>::bytes, st>>>(a);
    return cudaGetLastError();
}

template <int K, int V, typename IO>
cudaError_t launch_bwd_simt_t(const BwdArgs &a, float *dA, float *dB, cudaStream_t st) {
    auto kern = bwd_simt_kernel<K, V, IO>;
    cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), (int)BwdSmem<K, V>::bytes);
    if (e != cudaSuccess) return e;
    kern<<<a.B * a.H, kThreads, BwdSmem<K, V>::bytes, st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int KR = K * a.R, RV = a.R * V;
    dim3 grid((KR + RV + a.R + K + 1 + 255) / 256, a.H);
    reduce_dAdB_kernel<<<grid, 256, 0, st>>>(a.ws, dA, dB, a.dAw, a.dtau, a.dA_dec, a.B, a.H, KR, RV, a.R, K);
    return cudaGetLastError();
}

template <typename IO>
cudaError_t dispatch_fwd(int K, int V, const FwdArgs &a, cudaStream_t st) {
    if (K == 64 && V == 64) return launch_fwd_simt_t<64, 64, IO>(a, st);
    if (K == 64 && V == 128) return launch_fwd_simt_t<64, 128, IO>(a, st);
    if (K == 128 && V == 64) return launch_fwd_simt_t<128, 64, IO>(a, st);
    return launch_fwd_simt_t<128, 128, IO>(a, st);
}

template <typename IO>
cudaError_t dispatch_bwd(int K, int V, const BwdArgs &a, float *dA, float *dB, cudaStream_t st) {
    if (K == 64 && V == 64) return launch_bwd_simt_t<64, 64, IO>(a, dA, dB, st);
    if (K == 64 && V == 128) return launch_bwd_simt_t<64, 128, IO>(a, dA, dB, st);
    if (K == 128 && V == 64) return launch_bwd_simt_t<128, 64, IO>(a, dA, dB, st);
    return launch_bwd_simt_t<128, 128, IO>(a, dA, dB, st);
}

cudaError_t launch_fwd_simt(int K, int V, bool bf16, const FwdArgs &a, cudaStream_t st) {
    return bf16 ? dispatch_fwd<__nv_bfloat16>(K, V, a, st) : dispatch_fwd<float>(K, V, a, st);
}

cudaError_t launch_bwd_simt(int K, int V, bool bf16, const BwdArgs &a, float *dA, float *dB, cudaStream_t st) {
    return bf16 ? dispatch_bwd<__nv_bfloat16>(K, V, a, dA, dB, st) : dispatch_bwd<float>(K, V, a, dA, dB, st);
}

size_t fwd_simt_smem(int K, int V) {
    if (K == 64 && V == 64) return FwdSmem<64, 64>::bytes;
    if (K == 64 && V == 128) return FwdSmem<64, 128>::bytes;
    if (K == 128 && V == 64) return FwdSmem<128, 64>::bytes;
    return FwdSmem<128, 128>::bytes;
}

size_t bwd_simt_smem(int K, int V) {
    if (K == 64 && V == 64) return BwdSmem<64, 64>::bytes;
    if (K == 64 && V == 128) return BwdSmem<64, 128>::bytes;
    if (K == 128 && V == 64) return BwdSmem<128, 64>::bytes;
    return BwdSmem<128, 128>::bytes;
}

}  // namespace carve

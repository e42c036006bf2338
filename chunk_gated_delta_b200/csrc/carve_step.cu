// CARVE single-token decode step (CARVE blog, Table 1: inference costs O(dv dk) per token).
//
// With P = S Diag(a) the token's update and output expand to matrix-vector products over the
// same state rows, so each (batch, head) state is read once and written once:
//   m  = S q                     (mc_mode 0: content signal from the state before the token)
//   z  = Bm m,  a = exp(-softplus(g_logit)) * sigmoid(bx + A z),  w = sigmoid(w_logit + Aw . z)
//   p  = S (a*k),  e = v - p
//   o  = S (a*q) + w e (k.q)     (= S' q)
//   S' = S Diag(a) + w e k^T
//
// The step moves 8 dv dk bytes of state per (b,h) and little else.  One persistent CTA per
// SM walks its share of the (b,h) units with NGRP independent groups of 256 threads (each
// with its own named barrier and its own shared-memory stage), so the dependent chain of one
// unit (content signal -> z -> Delta -> gates -> update) overlaps the other group's.  A
// unit's state arrives in the group's stage by one bulk copy; the first pass moves it into
// registers, after which the stage is refilled with the group's next unit while this one
// finishes.  The updated state is stored from registers.  Thread layout: the 8 lanes of a
// lane octet share a row group and split the columns (lane seg holds float4 columns
// seg, seg + 8, ...), and a thread holds the rows rg, rg + 32, ... of its row group rg.  A
// warp's reads of a state row are then 128 contiguous bytes per octet, its reads of the
// q / k / a vectors are broadcasts (every octet reads the same 128 bytes), and each global
// store instruction writes whole 128-byte lines.  Row sums over an octet use a transposing
// reduction that halves the values exchanged at each of its three steps.
#include "carve_device.cuh"
#include "carve_mma.cuh"

namespace carve {

struct StepArgs {
    const void *q, *k, *v;
    const float *g_logit, *bx, *w_logit, *A, *Bm, *Aw;
    const float *A_dec, *tau;   // [H], [H,K] or null: the decay's log-amplitude and bias
    float *S, *mstate;
    int *pos;
    void *o;
    int B, H, R, L, mc_mode;
};

constexpr int kGroupThreads = 256;   // threads per unit group
constexpr int kStepMaxRank = 64;

__device__ int g_step_timeout;  // set when a bounded wait gives up (never expected)

// A unit's token vectors as stored in global memory (q, k, v in the I/O type).
template <int K, int V, typename IO>
struct __align__(16) StepTokens {
    IO q[K], k[K], v[V];
    float gl[K], bx[K], wl[4];
};

template <int K, int V, typename IO>
struct __align__(16) StepGroupSmem {
    float S[V * K];
    StepTokens<K, V, IO> tok[2];   // this unit's and the next unit's, filled by cp.async
    float qv[K], kv[K], glv[K], bxv[K], av[K];
    float vv[V], mv[V], msum[V], zv[kStepMaxRank];
    float w, kq;
    uint64_t bar;
};

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// Barrier over the 256 threads of group `id` (named barrier 1 + id).
__device__ __forceinline__ void group_sync(int id) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(1 + id), "r"(kGroupThreads) : "memory");
}
// The same barrier, returning whether any thread of the group passed `v` true.
__device__ __forceinline__ bool group_sync_or(int id, bool v) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(1 + id), "r"(kGroupThreads)
        : "memory");
    return r != 0;
}

// Sums x[0..N) over the 8 lanes of an aligned lane octet (lanes differing in bits 0-2 of the
// lane index; `seg` = those bits) and returns the total of x[seg >> (3 - log2 N)].
template <int N>
__device__ __forceinline__ float octet_reduce(const float (&x)[N], int seg) {
    static_assert(N == 2 || N == 4 || N == 8, "octet_reduce: N in {2, 4, 8}");
    float y[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) y[j] = j < N ? x[j] : 0.f;
    int n = N;
#pragma unroll
    for (int bit = 4; bit >= 1; bit >>= 1) {
        if (n > 1) {
            const int h = n / 2;
            const bool up = (seg & bit) != 0;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (j < h) y[j] = (up ? y[j + h] : y[j]) + __shfl_xor_sync(0xffffffffu, up ? y[j] : y[j + h], bit);
            n = h;
        } else {
            y[0] += __shfl_xor_sync(0xffffffffu, y[0], bit);
        }
    }
    return y[0];
}

// RMAX: rank bound of the factor slices held in registers (32, or 64 with one group).
template <int K, int V, typename IO, int RMAX, int NGRP>
__global__ void __launch_bounds__(kGroupThreads *NGRP, 1) step_kernel(StepArgs a, int n_units) {
    constexpr int RPT = V / 32;                // state rows per thread: rg + 32 i
    constexpr int CPT = K / 32;                // float4 columns per row per thread: seg + 8 jj
    constexpr int LRPT = RPT == 4 ? 2 : 1;     // log2 RPT
    constexpr int TPK = kGroupThreads / K;     // threads per Delta output
    constexpr int VP = V / 8;                  // entries of a z dot product per thread (8 per output)
    constexpr int ZP = RMAX / 32;              // passes of 32 z outputs
    constexpr int AP = RMAX / TPK;             // entries of a Delta dot product per thread
    constexpr uint32_t kBytes = V * K * 4;
    extern __shared__ __align__(128) unsigned char smraw[];
    const int grp = threadIdx.x / kGroupThreads, tid = threadIdx.x % kGroupThreads;
    StepGroupSmem<K, V, IO> &sm = reinterpret_cast<StepGroupSmem<K, V, IO> *>(smraw)[grp];
    const int seg = tid % 8, rg = tid / 8, lane = tid % 32, H = a.H, R = a.R;
    // this group's units: first + (NGRP i + grp) stride, i = 0, 1, ...
    const int first = blockIdx.x, stride = gridDim.x;
    const int mine = first < n_units ? (n_units - 1 - first) / stride + 1 : 0;
    const int nmine = mine > grp ? (mine - 1 - grp) / NGRP + 1 : 0;
    auto unit_of = [&](int i) { return first + (NGRP * i + grp) * stride; };

    // token vectors of the group's i-th unit into tok[i & 1], 16 bytes per copy
    auto fetch_tokens = [&](int i) {
        if (i >= nmine) return;
        const int u = unit_of(i);
        StepTokens<K, V, IO> &t = sm.tok[i & 1];
        constexpr int CQ = K * (int)sizeof(IO) / 16, CV = V * (int)sizeof(IO) / 16, CG = K * 4 / 16;
        for (int c = tid; c < 2 * CQ + CV + 2 * CG; c += kGroupThreads) {
            if (c < CQ) cp_async16(reinterpret_cast<char *>(t.q) + 16 * c,
                                   static_cast<const char *>(a.q) + (size_t)u * K * sizeof(IO) + 16 * c);
            else if (c < 2 * CQ) cp_async16(reinterpret_cast<char *>(t.k) + 16 * (c - CQ),
                                            static_cast<const char *>(a.k) + (size_t)u * K * sizeof(IO) + 16 * (c - CQ));
            else if (c < 2 * CQ + CV)
                cp_async16(reinterpret_cast<char *>(t.v) + 16 * (c - 2 * CQ),
                           static_cast<const char *>(a.v) + (size_t)u * V * sizeof(IO) + 16 * (c - 2 * CQ));
            else if (c < 2 * CQ + CV + CG)
                cp_async16(t.gl + 4 * (c - 2 * CQ - CV), a.g_logit + (size_t)u * K + 4 * (c - 2 * CQ - CV));
            else
                cp_async16(t.bx + 4 * (c - 2 * CQ - CV - CG), a.bx + (size_t)u * K + 4 * (c - 2 * CQ - CV - CG));
        }
        if (tid == kGroupThreads - 1) cp_async4(t.wl, a.w_logit + u);
        cp_async_commit();
    };

    if (tid == 0) {
        mbar_init(&sm.bar, 1);
        fence_mbar_init();
        if (nmine > 0) {
            mbar_expect_tx(&sm.bar, kBytes);
            bulk_g2s(sm.S, a.S + (size_t)unit_of(0) * V * K, kBytes, &sm.bar);
        }
    }
    fetch_tokens(0);
    group_sync(grp);

    for (int i = 0; i < nmine; ++i) {
        const int u = unit_of(i), h = u % H;
        // ---- token vectors (prefetched) into fp32 working copies, the next unit's requested;
        //      the head's factor slices into registers
        cp_async_wait_all();
        group_sync(grp);
        {
            const StepTokens<K, V, IO> &t = sm.tok[i & 1];
            if (tid < K) {
                sm.qv[tid] = ld_io(t.q + tid);
                sm.kv[tid] = ld_io(t.k + tid);
                sm.glv[tid] = t.gl[tid];
                sm.bxv[tid] = t.bx[tid];
            }
            if (tid < V) sm.vv[tid] = ld_io(t.v + tid);
        }
        fetch_tokens(i + 1);   // tok[(i + 1) & 1] was last read before the barrier above
        if (tid < V) {
            if (a.mc_mode == 1) {   // running block mean of o: close the block every L tokens
                const int p = a.pos[u];
                float m = a.mstate[(size_t)u * 2 * V + V + tid], msum = a.mstate[(size_t)u * 2 * V + tid];
                if (p > 0 && p % a.L == 0) {
                    m = msum / (float)a.L;
                    a.mstate[(size_t)u * 2 * V + V + tid] = m;
                    msum = 0.f;
                }
                sm.mv[tid] = m;
                sm.msum[tid] = msum;
            }
        }
        // the decay's log-amplitude and this thread's channel bias, used in the gate phase
        const float pAdec = a.A_dec ? a.A_dec[h] : 0.f, ptau = a.tau ? a.tau[(size_t)h * K + tid / TPK] : 0.f;
        float pB[ZP][VP], pA[AP];
#pragma unroll
        for (int zp = 0; zp < ZP; ++zp) {
            const int j = 32 * zp + tid / 8, part = tid % 8;
#pragma unroll
            for (int x = 0; x < VP; ++x) pB[zp][x] = j < R ? a.Bm[((size_t)h * R + j) * V + part + 8 * x] : 0.f;
        }
        {
            const int kk = tid / TPK, part = tid % TPK;
#pragma unroll
            for (int x = 0; x < AP; ++x) {
                const int r = part + TPK * x;
                pA[x] = r < R ? a.A[((size_t)h * K + kk) * R + r] : 0.f;
            }
        }
        // ---- state rows into registers; content signal m = S q (mc_mode 0); k.q
        const bool ok = mbar_wait(&sm.bar, (uint32_t)i & 1u);
        if (group_sync_or(grp, !ok)) {   // record; drain the copy still in flight (bounded); leave
            if (tid == 0) {
                atomicOr(&g_step_timeout, 1);
                mbar_wait(&sm.bar, (uint32_t)i & 1u);
            }
            break;
        }
        float4 s[RPT][CPT];
        {
            const float4 *S4 = reinterpret_cast<const float4 *>(sm.S);
            float part[RPT];
#pragma unroll
            for (int i2 = 0; i2 < RPT; ++i2) part[i2] = 0.f;
#pragma unroll
            for (int jj = 0; jj < CPT; ++jj) {
                const float4 qq = reinterpret_cast<const float4 *>(sm.qv)[seg + 8 * jj];
#pragma unroll
                for (int i2 = 0; i2 < RPT; ++i2) {
                    s[i2][jj] = S4[(rg + 32 * i2) * (K / 4) + seg + 8 * jj];
                    part[i2] += s[i2][jj].x * qq.x + s[i2][jj].y * qq.y + s[i2][jj].z * qq.z + s[i2][jj].w * qq.w;
                }
            }
            if (a.mc_mode == 0) {
                const float m = octet_reduce<RPT>(part, seg);   // row rg + 32 (seg >> (3 - LRPT))
                if ((seg & ((8 >> LRPT) - 1)) == 0) sm.mv[rg + 32 * (seg >> (3 - LRPT))] = m;
            }
        }
        if (tid >= kGroupThreads - 32) {   // last warp: k.q
            float x = 0.f;
            for (int c = tid - (kGroupThreads - 32); c < K; c += 32) x += sm.kv[c] * sm.qv[c];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
            if (tid == kGroupThreads - 32) sm.kq = x;
        }
        group_sync(grp);
        if (tid == 0 && i + 1 < nmine) {   // the stage is free: the group's next unit
            mbar_expect_tx(&sm.bar, kBytes);
            bulk_g2s(sm.S, a.S + (size_t)unit_of(i + 1) * V * K, kBytes, &sm.bar);
        }
        // ---- z = Bm m
#pragma unroll
        for (int zp = 0; zp < ZP; ++zp) {
            if (32 * zp < R) {
                const int j = 32 * zp + tid / 8, part = tid % 8;
                float acc = 0.f;
#pragma unroll
                for (int x = 0; x < VP; ++x) acc += pB[zp][x] * sm.mv[part + 8 * x];
                acc += __shfl_xor_sync(0xffffffffu, acc, 4);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                if (part == 0 && j < R) sm.zv[j] = acc;
            }
        }
        group_sync(grp);
        // ---- Delta = A z, gates
        {
            const int kk = tid / TPK, part = tid % TPK;
            float acc = 0.f;
#pragma unroll
            for (int x = 0; x < AP; ++x)
                if (part + TPK * x < R) acc += pA[x] * sm.zv[part + TPK * x];
#pragma unroll
            for (int off = TPK / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (tid == 0) {   // w = sigmoid(w_logit + Aw . z): the same projection biases the write gate
                float dw = 0.f;
                if (a.Aw)
                    for (int j = 0; j < R; ++j) dw += a.Aw[(size_t)h * R + j] * sm.zv[j];
                sm.w = sigmoid_f(sm.tok[i & 1].wl[0] + dw);
            }
            if (part == 0) {
                // a = sigma(-g_logit) sigma(bx + Delta) = 1 / ((1 + e^{g_logit})(1 + e^{-(bx + Delta)}));
                // with the decay's amplitude and bias, 1 / g = e^{amp softplus(g_logit + tau)}
                const float e2 = __expf(-(sm.bxv[kk] + acc));
                float ig;
                if (a.A_dec || a.tau)
                    ig = __expf(expf(pAdec) * softplus_f(sm.glv[kk] + ptau));
                else
                    ig = 1.f + __expf(sm.glv[kk]);
                sm.av[kk] = __fdividef(1.f, ig * (1.f + e2));
            }
        }
        group_sync(grp);
        // ---- p = (S a).k, s2 = (S a).q per row; update (stored from registers); output
        {
            float ps[2 * RPT];   // p of rows 0..RPT-1, then s2
#pragma unroll
            for (int x = 0; x < 2 * RPT; ++x) ps[x] = 0.f;
#pragma unroll
            for (int jj = 0; jj < CPT; ++jj) {
                const float4 av = reinterpret_cast<const float4 *>(sm.av)[seg + 8 * jj];
                const float4 kv = reinterpret_cast<const float4 *>(sm.kv)[seg + 8 * jj];
                const float4 qv = reinterpret_cast<const float4 *>(sm.qv)[seg + 8 * jj];
#pragma unroll
                for (int i2 = 0; i2 < RPT; ++i2) {
                    float4 &x = s[i2][jj];
                    x.x *= av.x;
                    x.y *= av.y;
                    x.z *= av.z;
                    x.w *= av.w;
                    ps[i2] += x.x * kv.x + x.y * kv.y + x.z * kv.z + x.w * kv.w;
                    ps[RPT + i2] += x.x * qv.x + x.y * qv.y + x.z * qv.z + x.w * qv.w;
                }
            }
            // lane seg now holds ps[idx] summed over the octet, idx = seg >> (2 - LRPT)
            const float tot = octet_reduce<2 * RPT>(ps, seg);
            const int idx = seg >> (2 - LRPT), ri = idx % RPT;
            const int row_i = rg + 32 * ri;
            const float we_mine = idx < RPT ? sm.w * (sm.vv[row_i] - tot) : 0.f;
            float we[RPT];
#pragma unroll
            for (int i2 = 0; i2 < RPT; ++i2) we[i2] = __shfl_sync(0xffffffffu, we_mine, (lane & ~7) | (i2 << (2 - LRPT)));
            float4 *Sg = reinterpret_cast<float4 *>(a.S + (size_t)u * V * K);
#pragma unroll
            for (int jj = 0; jj < CPT; ++jj) {   // S' = S Diag(a) + w e k^T
                const float4 kv = reinterpret_cast<const float4 *>(sm.kv)[seg + 8 * jj];
#pragma unroll
                for (int i2 = 0; i2 < RPT; ++i2) {
                    float4 x = s[i2][jj];
                    x.x += we[i2] * kv.x;
                    x.y += we[i2] * kv.y;
                    x.z += we[i2] * kv.z;
                    x.w += we[i2] * kv.w;
                    Sg[(rg + 32 * i2) * (K / 4) + seg + 8 * jj] = x;
                }
            }
            if (idx >= RPT && (seg & ((4 >> LRPT) - 1)) == 0) {   // one lane per row: the output
                float wr = we[0];
#pragma unroll
                for (int i2 = 1; i2 < RPT; ++i2)
                    if (ri == i2) wr = we[i2];
                const float ov = tot + wr * sm.kq;
                st_io(static_cast<IO *>(a.o) + (size_t)u * V + row_i, ov);
                if (a.mc_mode == 1) a.mstate[(size_t)u * 2 * V + row_i] = sm.msum[row_i] + ov;
            }
        }
        if (tid == 0 && a.mc_mode == 1) a.pos[u] += 1;
        group_sync(grp);   // the vectors of this unit are read; the next unit may overwrite them
    }
}

// A single thread waits, bounded, on a barrier that nothing arrives on (the expiry path of
// every bounded wait in this library, exercised on purpose).
__global__ void selftest_timeout_kernel(uint32_t iterations) {
    __shared__ uint64_t bar;
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait(&bar, 0u, iterations)) atomicOr(&g_step_timeout, 2);
}

cudaError_t launch_selftest_timeout(uint32_t iterations, cudaStream_t st) {
    selftest_timeout_kernel<<<1, 1, 0, st>>>(iterations);
    return cudaGetLastError();
}

// Device status word of this file: returns and clears it.
int step_take_timeout() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_step_timeout, sizeof(int)) != cudaSuccess) return 0;
    if (v) {
        const int z = 0;
        cudaMemcpyToSymbol(g_step_timeout, &z, sizeof(int));
    }
    return v;
}

static int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

template <int K, int V, typename IO, int RMAX, int NGRP>
cudaError_t launch_step_t(const StepArgs &a, cudaStream_t st) {
    auto kern = step_kernel<K, V, IO, RMAX, NGRP>;
    const int bytes = (int)sizeof(StepGroupSmem<K, V, IO>) * NGRP;
    cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), bytes);
    if (e != cudaSuccess) return e;
    const int units = a.B * a.H;
    const int grid = units < sm_count() ? units : sm_count();
    kern<<<grid, kGroupThreads * NGRP, bytes, st>>>(a, units);
    return cudaGetLastError();
}

template <int K, int V, typename IO>
cudaError_t launch_step_r(const StepArgs &a, cudaStream_t st) {
    return a.R <= 32 ? launch_step_t<K, V, IO, 32, 2>(a, st) : launch_step_t<K, V, IO, 64, 1>(a, st);
}

template <typename IO>
cudaError_t dispatch_step(int K, int V, const StepArgs &a, cudaStream_t st) {
    if (K == 64 && V == 64) return launch_step_r<64, 64, IO>(a, st);
    if (K == 64 && V == 128) return launch_step_r<64, 128, IO>(a, st);
    if (K == 128 && V == 64) return launch_step_r<128, 64, IO>(a, st);
    return launch_step_r<128, 128, IO>(a, st);
}

cudaError_t launch_step(int K, int V, bool bf16, const void *q, const void *k, const void *v,
                        const float *g_logit, const float *bx, const float *w_logit, const float *A,
                        const float *Bm, const float *Aw, const float *A_dec, const float *tau, float *S,
                        float *mstate, int *pos, void *o, int B, int H, int R, int L, int mc_mode, cudaStream_t st) {
    StepArgs a{q, k, v, g_logit, bx, w_logit, A, Bm, Aw, A_dec, tau, S, mstate, pos, o, B, H, R, L, mc_mode};
    return bf16 ? dispatch_step<__nv_bfloat16>(K, V, a, st) : dispatch_step<float>(K, V, a, st);
}

}  // namespace carve

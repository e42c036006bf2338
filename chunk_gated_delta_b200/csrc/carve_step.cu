// CARVE single-token decode step (CARVE blog, Table 1: inference costs O(dv dk) per token).
//
// With P = S Diag(a) the token's update and output expand to matrix-vector products over the
// same state rows, so each (batch, head) state is read once and written once:
//   m  = S q                     (mc_mode 0: content signal from the state before the token)
//   a  = exp(-softplus(g_logit)) * sigmoid(bx + A (Bm m)),  w = sigmoid(w_logit)
//   p  = S (a*k),  e = v - p
//   o  = S (a*q) + w e (k.q)     (= S' q)
//   S' = S Diag(a) + w e k^T
//
// The step moves 8 dv dk bytes of state per (b,h) and little else, so the kernel is built
// around the copy engine: one persistent CTA per SM walks its share of the (b,h) units with
// three shared-memory stages.  A unit's whole state arrives by one bulk copy issued two units
// ahead and leaves by one bulk store from the same stage, so loads, stores and the arithmetic
// of three units overlap.  The unit's token vectors and its head's slices of the low-rank
// factors are prefetched into registers one unit ahead.  Each state row is read by TPR
// threads as float4 groups in a row-rotated order (conflict-free shared-memory banks) and
// kept in registers between the content-signal pass and the update pass.
#include "carve_device.cuh"
#include "carve_mma.cuh"

namespace carve {

struct StepArgs {
    const void *q, *k, *v;
    const float *g_logit, *bx, *w_logit, *A, *Bm;
    float *S, *mstate;
    int *pos;
    void *o;
    int B, H, R, L, mc_mode;
};

constexpr int kStepThreads = 256;
constexpr int kStepStages = 3;
constexpr int kStepMaxRank = 64;

__device__ int g_step_timeout;  // set when a bounded wait gives up (never expected)

template <int K, int V>
struct __align__(16) StepSmem {
    float S[kStepStages][V * K];
    float qv[K], kv[K], glv[K], bxv[K], av[K], akv[K], aqv[K];
    float vv[V], mv[V], msum[V], zv[kStepMaxRank];
    float w, kq;
    uint64_t bar[kStepStages];
};

template <int K, int V, typename IO>
__global__ void __launch_bounds__(kStepThreads, 1) step_kernel(StepArgs a, int n_units) {
    constexpr int TPR = kStepThreads / V;     // threads per state row
    constexpr int G4 = K / 4 / TPR;           // float4 groups per thread
    constexpr int TPK = kStepThreads / K;     // threads per Delta output
    constexpr int VP = V / 8;                 // entries of a z dot product per thread (8 per output)
    constexpr int AP = kStepMaxRank / TPK;    // entries of a Delta dot product per thread
    constexpr uint32_t kBytes = V * K * 4;
    extern __shared__ __align__(128) unsigned char smraw[];
    StepSmem<K, V> &sm = *reinterpret_cast<StepSmem<K, V> *>(smraw);
    const int tid = threadIdx.x, row = tid / TPR, seg = tid % TPR, H = a.H, R = a.R;
    const int first = blockIdx.x, stride = gridDim.x;
    const int nmine = first < n_units ? (n_units - 1 - first) / stride + 1 : 0;

    if (tid == 0) {
        for (int st = 0; st < kStepStages; ++st) mbar_init(&sm.bar[st], 1);
        fence_mbar_init();
    }
    __syncthreads();
    auto issue = [&](int i) {   // the state of this CTA's i-th unit into stage i % 3
        if (tid == 0 && i < nmine) {
            const int u = first + i * stride, st = i % kStepStages;
            mbar_expect_tx(&sm.bar[st], kBytes);
            bulk_g2s(sm.S[st], a.S + (size_t)u * V * K, kBytes, &sm.bar[st]);
        }
    };
    issue(0);
    issue(1);

    // token vectors of a unit (channel tid / row tid) and the mean-output carry (mc_mode 1)
    float pq = 0.f, pk = 0.f, pgl = 0.f, pbx = 0.f, pv = 0.f, pwl = 0.f, pms = 0.f, pmp = 0.f;
    int ppos = 0;
    auto prefetch_tokens = [&](int i) {
        if (i >= nmine) return;
        const int u = first + i * stride;
        if (tid < K) {
            pq = ld_io(static_cast<const IO *>(a.q) + (size_t)u * K + tid);
            pk = ld_io(static_cast<const IO *>(a.k) + (size_t)u * K + tid);
            pgl = a.g_logit[(size_t)u * K + tid];
            pbx = a.bx[(size_t)u * K + tid];
        }
        if (tid < V) {
            pv = ld_io(static_cast<const IO *>(a.v) + (size_t)u * V + tid);
            if (a.mc_mode == 1) {
                pms = a.mstate[(size_t)u * 2 * V + tid];
                pmp = a.mstate[(size_t)u * 2 * V + V + tid];
                ppos = a.pos[u];
            }
        }
        if (tid == 0) pwl = a.w_logit[u];
    };
    // the head's slices of Bm (for z, 8 threads per output) and A (for Delta, TPK per output)
    float pB[2][VP], pA[AP];
    auto prefetch_factors = [&](int i) {
        if (i >= nmine) return;
        const int h = (first + i * stride) % H;
#pragma unroll
        for (int zp = 0; zp < 2; ++zp) {
            const int j = 32 * zp + tid / 8, part = tid % 8;
#pragma unroll
            for (int x = 0; x < VP; ++x) pB[zp][x] = j < R ? a.Bm[((size_t)h * R + j) * V + part + 8 * x] : 0.f;
        }
        const int kk = tid / TPK, part = tid % TPK;
#pragma unroll
        for (int x = 0; x < AP; ++x) {
            const int r = part + TPK * x;
            pA[x] = r < R ? a.A[((size_t)h * K + kk) * R + r] : 0.f;
        }
    };
    prefetch_tokens(0);
    prefetch_factors(0);

    bool failed = false;
    int i = 0;
    for (; i < nmine; ++i) {
        const int u = first + i * stride, st = i % kStepStages;
        float *Sst = sm.S[st];
        // ---- token vectors into shared memory, next unit's into registers
        if (tid < K) {
            sm.qv[tid] = pq;
            sm.kv[tid] = pk;
            sm.glv[tid] = pgl;
            sm.bxv[tid] = pbx;
        }
        if (tid < V) {
            sm.vv[tid] = pv;
            if (a.mc_mode == 1) {   // running block mean of o: close the block every L tokens
                float m = pmp, msum = pms;
                if (ppos > 0 && ppos % a.L == 0) {
                    m = msum / (float)a.L;
                    a.mstate[(size_t)u * 2 * V + V + tid] = m;
                    msum = 0.f;
                }
                sm.mv[tid] = m;
                sm.msum[tid] = msum;
            }
        }
        if (tid == 0) {
            sm.w = sigmoid_f(pwl);
            if (a.mc_mode == 1) a.pos[u] = ppos + 1;
        }
        prefetch_tokens(i + 1);
        __syncthreads();
        // ---- state rows into registers; content signal m = S q (mc_mode 0); k.q
        const bool ok = mbar_wait(&sm.bar[st], (uint32_t)(i / kStepStages) & 1u);
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        float4 s[G4];
        {
            float part = 0.f;
#pragma unroll
            for (int j = 0; j < G4; ++j) {
                const int f = seg + TPR * ((j + row) % G4);
                s[j] = reinterpret_cast<const float4 *>(Sst)[row * (K / 4) + f];
                const float4 qq = reinterpret_cast<const float4 *>(sm.qv)[f];
                part += s[j].x * qq.x + s[j].y * qq.y + s[j].z * qq.z + s[j].w * qq.w;
            }
            if (a.mc_mode == 0) {
#pragma unroll
                for (int off = TPR / 2; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
                if (seg == 0) sm.mv[row] = part;
            }
        }
        if (tid >= kStepThreads - 32) {   // last warp: k.q
            float x = 0.f;
            for (int c = tid - (kStepThreads - 32); c < K; c += 32) x += sm.kv[c] * sm.qv[c];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
            if (tid == kStepThreads - 32) sm.kq = x;
        }
        __syncthreads();
        // ---- z = Bm m
#pragma unroll
        for (int zp = 0; zp < 2; ++zp) {
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
        __syncthreads();
        // ---- Delta = A z, gates
        {
            const int kk = tid / TPK, part = tid % TPK;
            float acc = 0.f;
#pragma unroll
            for (int x = 0; x < AP; ++x)
                if (part + TPK * x < R) acc += pA[x] * sm.zv[part + TPK * x];
#pragma unroll
            for (int off = TPK / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (part == 0) {
                const float av = expf(log_retention(sm.glv[kk], sm.bxv[kk] + acc));
                sm.av[kk] = av;
                sm.akv[kk] = av * sm.kv[kk];
                sm.aqv[kk] = av * sm.qv[kk];
            }
        }
        prefetch_factors(i + 1);
        if (tid == 0) {   // the stage of unit i - 1 takes unit i + 2 once its store has read it
            bulk_wait_read<0>();
            issue(i + 2);
        }
        __syncthreads();
        // ---- p = S (a*k), S (a*q); update; output
        {
            float p = 0.f, s2 = 0.f;
#pragma unroll
            for (int j = 0; j < G4; ++j) {
                const int f = seg + TPR * ((j + row) % G4);
                const float4 ak = reinterpret_cast<const float4 *>(sm.akv)[f];
                const float4 aq = reinterpret_cast<const float4 *>(sm.aqv)[f];
                p += s[j].x * ak.x + s[j].y * ak.y + s[j].z * ak.z + s[j].w * ak.w;
                s2 += s[j].x * aq.x + s[j].y * aq.y + s[j].z * aq.z + s[j].w * aq.w;
            }
#pragma unroll
            for (int off = TPR / 2; off >= 1; off >>= 1) {
                p += __shfl_xor_sync(0xffffffffu, p, off);
                s2 += __shfl_xor_sync(0xffffffffu, s2, off);
            }
            const float we = sm.w * (sm.vv[row] - p);
#pragma unroll
            for (int j = 0; j < G4; ++j) {
                const int f = seg + TPR * ((j + row) % G4);
                const float4 av = reinterpret_cast<const float4 *>(sm.av)[f];
                const float4 kv = reinterpret_cast<const float4 *>(sm.kv)[f];
                float4 x = s[j];
                x.x = x.x * av.x + we * kv.x;
                x.y = x.y * av.y + we * kv.y;
                x.z = x.z * av.z + we * kv.z;
                x.w = x.w * av.w + we * kv.w;
                reinterpret_cast<float4 *>(Sst)[row * (K / 4) + f] = x;
            }
            if (seg == 0) {
                const float ov = s2 + we * sm.kq;
                st_io(static_cast<IO *>(a.o) + (size_t)u * V + row, ov);
                if (a.mc_mode == 1) a.mstate[(size_t)u * 2 * V + row] = sm.msum[row] + ov;
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            bulk_s2g(a.S + (size_t)u * V * K, Sst, kBytes);
            bulk_commit();
        }
    }
    if (failed) {   // drain the loads still in flight into this CTA's stages, bounded
        if (tid == 0) {
            atomicOr(&g_step_timeout, 1);
            for (int j = i; j < min(i + 2, nmine); ++j) mbar_wait(&sm.bar[j % kStepStages], (uint32_t)(j / kStepStages) & 1u);
        }
    }
    if (tid == 0) bulk_wait<0>();
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

template <int K, int V, typename IO>
cudaError_t launch_step_t(const StepArgs &a, cudaStream_t st) {
    auto kern = step_kernel<K, V, IO>;
    const int bytes = (int)sizeof(StepSmem<K, V>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    const int units = a.B * a.H;
    const int grid = units < sm_count() ? units : sm_count();
    kern<<<grid, kStepThreads, bytes, st>>>(a, units);
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

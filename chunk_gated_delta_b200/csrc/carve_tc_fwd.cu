// CARVE forward, tensor-core kernel for bf16 q/k/v/o with dk = dv = 128.
//
// One CTA (8 warps) per (batch, head) unit sweeps the sequence in compute chunks of
// C = 16*NB tokens (C = min(chunk, 64); a 128-token gate chunk is two compute chunks sharing
// one content signal).  Each warp owns 16 state rows (rows [16w, 16w+16) with 64-token chunks;
// with 32-token chunks rows 32 (w % 4) + 16 (w / 4) + [0, 16), the TMEM lanes the warp may
// read): its 16x128 slice of the fp32 state lives in registers as mma accumulator fragments for
// the whole sweep, so the state never round-trips through memory except when it is saved for
// the backward (and, as a bf16 tile, read by the tensor core).
//
// Per compute chunk (CARVE blog section 2.3: one WY solve shared by all value channels):
//   gates      a_t = 1 / ((1 + e^{g_logit})(1 + e^{-(bx + Delta)})) (with the decay amplitude and
//              bias: 1 / g = e^{amp softplus(g_logit + tau)}), floored at e^-10, and its
//              reciprocal (free), per key channel
//   operands   mid-block referenced q*e^{Lam_t - Lam_m}, k*e^{Lam_t - Lam_m}, k*e^{Lam_m - Lam_s}
//              (m = middle of the token's 16-block) built from running products of a and 1/a,
//              so every factor lies in [e^-80, e^80]; chunk-level factors (block products) carry
//              the rest and are all <= 1
//   Gram       Akk, Aqk: block (i,j) = rows_i . diag(e^{Lam_m(i) - Lam_m(j)}) . cols_j^T, the factor
//              split between the row operand (decay to block i's middle from block i's start)
//              and the column operand (the rest), so that neither part underflows alone
//   G          S0 [Kt; Qt]^T   (Kt = k e^{Lam}, Qt = q e^{Lam}); 32-token chunks: one tcgen05
//              MMA (M = 128, N = 64, K = 128) from the bf16 state tile and [Kt; Qt] in shared
//              memory, accumulator in TMEM, read back by each warp as mma fragments;
//              64-token chunks: per warp, mma
//   solve      X = Diag(w)(V - Kt S0^T);  U_i = (X_i - sum_j U_j M_ij^T) T_ii^T,  T_ii = (I + D A_ii)^-1
//   output     O^T = S0 Qt^T + U^T Aqk^T                                  per warp, mma
//   state      S = S Diag(gamma) + U^T Kbar,  Kbar = k e^{Lam_C - Lam}         per warp, mma
//   content   at a gate-chunk start, m for each warp's rows (S_[c-1] mean q, or the previous
//              chunk's mean output), z = B m reduced over the warps, Delta = A z per key channel,
//              from A^T and B^T staged in shared memory
// Raw q/k/v rows (and, with 32-token chunks, the gate logits) are prefetched into shared memory
// by the bulk-copy (TMA) engine while the previous chunk computes; the bf16 chunk-start state
// saved for the backward is written into the stage's consumed gate tiles (stmatrix) and leaves
// through one bulk copy.  The floor a >= e^-10 bounds the deviation from the exact recurrence
// by e^-10 per step in channels that are being erased anyway.
#include "carve_tc_common.cuh"
#include "carve_umma.cuh"

namespace carve {

constexpr int kTcMaxRank = 32;                        // low-rank factors staged in shared memory

__device__ int g_tc_timeout;  // set when a bounded wait gives up (never expected)
__device__ int g_tc_bad_seqlens;  // set when a packed sequence's offsets are out of range

template <int NB>
struct __align__(16) TcFwdSmem {
    static constexpr int C = 16 * NB, LDA = C + 8, NPAIR = NB * (NB - 1) / 2 > 0 ? NB * (NB - 1) / 2 : 1;
    // 32-token chunks: every input tile of the next chunk (q, k, v and the fp32 gate logits)
    // is brought in by TMA into a second stage while this chunk computes.  64-token chunks do
    // not fit twice: one stage, gate logits through registers.
    static constexpr int ST = NB == 2 ? 2 : 1;
    static constexpr bool GT = NB == 2;
    static constexpr int GSZ = GT ? C * 128 : 4;
    // 32-token chunks: G = S0 [Kt; Qt]^T on the 5th-generation tensor core (one M = 128, N = 64,
    // K = 128 product per chunk, accumulator in TMEM), both operands in the tensor core's
    // 128-byte-swizzle layout
    static constexpr bool UM = NB == 2;
    // raw tiles by TMA; a stage's two gate-logit tiles (32 KB with 32-token chunks) carry the
    // bf16 chunk-start state (the A operand of G, and the state saved for the backward) once
    // the gate phase has read them
    __nv_bfloat16 rq[ST][C * 128], rk[ST][C * 128], rv[ST][C * 128];
    float rgx[ST][2][GSZ];
    __nv_bfloat16 ktq[UM ? 2 * C * 128 : 8];   // [Kt; Qt]: the B operand of G
    // mid-block referenced operands; qm doubles as the output tile once the Gram has used it
    __nv_bfloat16 qm[C * kLdOp], krm[C * kLdOp], kcm[C * kLdOp], qt[UM ? 8 : C * kLdOp], kt[UM ? 8 : C * kLdOp];
    __nv_bfloat16 aqk[C * LDA], mkk[C * LDA];
    __nv_bfloat16 tii[NB * 16 * 24];
    float akk_d[NB * 16 * 17];
    float p7[NB * 128], r15[NB * 128], fm[NB * 128], cij[NPAIR * 128];
    float gam[128], wv[C], qbar[128], osum[128], mprev[128];
    float zp[8 * 32], dpart[2 * 128];   // content signal: per-warp parts of z, two parts of Delta
    float AhT[kTcMaxRank * 128], BhT[128 * kTcMaxRank];   // the head's factors: A^T [j][k], B^T [v][j]
    uint64_t bar[ST];
    uint64_t mma_bar;   // completion of G on the tensor core
    uint32_t tmem;      // TMEM base address of G's accumulator (64 columns)
    __device__ __nv_bfloat16 *ost() { return qm; }
};
// the dynamic shared-memory limit of one CTA on sm_100 (227 KB)
static_assert(sizeof(TcFwdSmem<2>) <= 232448 && sizeof(TcFwdSmem<4>) <= 232448, "shared memory");
static_assert(sizeof(TcFwdSmem<2>::rgx[0]) == 128 * 128 * 2, "a stage's gate tiles hold one bf16 state");
// tensor-core operands start on 1024-byte boundaries (the dynamic shared memory base is checked
// at run time)
static_assert(offsetof(TcFwdSmem<2>, rgx) % 1024 == 0 && sizeof(TcFwdSmem<2>::rgx[0]) % 1024 == 0 &&
                  offsetof(TcFwdSmem<2>, ktq) % 1024 == 0,
              "tensor-core operand alignment");
static_assert(offsetof(TcFwdSmem<2>, p7) % 16 == 0 && offsetof(TcFwdSmem<2>, r15) % 16 == 0 &&
                  offsetof(TcFwdSmem<2>, qm) % 16 == 0 && offsetof(TcFwdSmem<2>, krm) % 16 == 0,
              "decay factors and operands read as 16-byte vectors");

struct TileMaps {
    CUtensorMap q, k, v, gl, bx;
};

// DEC: the decay has its amplitude and bias (a.A_dec or a.tau given).  VL: the units are
// packed sequences (a.cu_seqlens); the last chunk of a sequence may be partial, its rows past
// the sequence's end are made inert (q = k = v = 0, a = 1, w = 0) and never stored.
template <int NB, bool DEC, bool VL>
__global__ void __launch_bounds__(256, 1) tc_fwd_kernel(FwdArgs a, const __grid_constant__ TileMaps maps) {
    using SM = TcFwdSmem<NB>;
    constexpr int C = SM::C, LDA = SM::LDA;
    constexpr int NP = (128 * NB + 255) / 256;  // (channel, block) pairs per thread in the gate phase
    extern __shared__ __align__(128) unsigned char smraw[];
    SM &sm = *reinterpret_cast<SM *>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, c4 = lane & 3;
    const int u = blockIdx.x, H = a.H, T = a.T, R = a.R, L = a.L;
    const int b = u / H, h = u % H;
    const int NCC = T / C, CPG = L / C, NG = (T + L - 1) / L;   // record strides
    int bb = b, toff = 0, Tn = T;   // this unit's tokens: rows [toff, toff + Tn) of tensor batch bb
    if constexpr (VL) seq_tokens(a.cu_seqlens, a.total, T, b, bb, toff, Tn, &g_tc_bad_seqlens);
    const int NCCn = VL ? (Tn + C - 1) / C : NCC;   // compute chunks of this unit
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(a.q);
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(a.o);
    const size_t tstride = (size_t)H * 128;
    const size_t base_bh = ((size_t)bb * T + toff) * tstride + (size_t)h * 128;   // token 0 of this unit
    // this warp's 16 state rows: with the tensor-core G, the rows whose TMEM lanes the warp may
    // read (lane quarter warp % 4, half warp / 4)
    const int vb = SM::UM ? 32 * (warp & 3) + 16 * (warp >> 2) : 16 * warp;
    const int v0 = vb + g, v1 = v0 + 8;
    const bool save = SM::GT && a.saved_states != nullptr;   // the bf16 chunk-start states for the backward
    __nv_bfloat16 *states = save ? reinterpret_cast<__nv_bfloat16 *>(a.saved_states) : nullptr;
    // the decay's amplitude and the biases of this thread's gate channels 2 (tid & 63) + {0, 1}
    const float amp = DEC ? decay_amp(a.A_dec, h) : 1.f;
    const float tb0 = DEC ? decay_bias(a.tau, h, 2 * (tid & 63), 128) : 0.f;
    const float tb1 = DEC ? decay_bias(a.tau, h, 2 * (tid & 63) + 1, 128) : 0.f;

    float s[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int col = 8 * j + 2 * c4;
        if (a.S0) {
            const float *S0 = a.S0 + (size_t)u * 128 * 128;
            s[j][0] = S0[v0 * 128 + col];
            s[j][1] = S0[v0 * 128 + col + 1];
            s[j][2] = S0[v1 * 128 + col];
            s[j][3] = S0[v1 * 128 + col + 1];
        } else {
            s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
        }
    }
    if (SM::UM && (smem_u32(smraw) & 1023u)) {   // operand layout needs a 1024-byte aligned base
        if (tid == 0) atomicOr(&g_tc_timeout, 4);
        return;
    }
    if (SM::UM && warp == 0) {
        tmem_alloc(&sm.tmem, 64);
        tc_fence_before_sync();
    }
    if (tid == 0) {
        if (SM::UM) mbar_init(&sm.mma_bar, 1);
        for (int i = 0; i < SM::ST; ++i) mbar_init(&sm.bar[i], 1);
        fence_mbar_init();
    }
    if (tid < 128) {
        sm.mprev[tid] = a.m_prev_in ? a.m_prev_in[(size_t)u * 128 + tid] : 0.f;
        sm.osum[tid] = 0.f;
    }
    for (int idx = tid; idx < 128 * kTcMaxRank; idx += 256) {   // zero beyond the rank
        const int j = idx >> 7, k = idx & 127;                   // AhT[j][k] = A[h][k][j]
        sm.AhT[idx] = j < R ? a.A[((size_t)h * 128 + k) * R + j] : 0.f;
        const int v = idx / kTcMaxRank, j2 = idx % kTcMaxRank;   // BhT[v][j] = B[h][j][v]
        sm.BhT[idx] = j2 < R ? a.Bm[((size_t)h * R + j2) * 128 + v] : 0.f;
    }
    __syncthreads();
    uint32_t tmem = 0, mma_phase = 0;   // G's accumulator; parity of the G product to wait for
    if (SM::UM) {
        tc_fence_after_sync();
        tmem = sm.tmem;
    }

    // Input tiles of chunk cc by TMA (one tensor copy per tile) into stage cc % ST.  With two
    // stages everything is issued at once, one chunk ahead; with one stage q/k (which = 0,
    // arming the barrier) go out mid-chunk and v (which = 1) at the end of the previous chunk.
    auto issue = [&](int cc, int which, int by = 0) {   // by: the issuing thread
        if (tid != by) return;
        const int row = bb * T + toff + cc * C, st = cc % SM::ST;
        uint64_t *bar = &sm.bar[st];
        if (which == 0) {
            mbar_expect_tx(bar, 3u * C * 256u + (SM::GT ? 2u * C * 512u : 0u));
            tma_load_3d(sm.rq[st], &maps.q, 0, h, row, bar);
            tma_load_3d(sm.rk[st], &maps.k, 0, h, row, bar);
            if (SM::GT) {
                tma_load_3d(sm.rgx[st][0], &maps.gl, 0, h, row, bar);
                tma_load_3d(sm.rgx[st][1], &maps.bx, 0, h, row, bar);
            }
        }
        if (which == 1 || SM::ST == 2) tma_load_3d(sm.rv[st], &maps.v, 0, h, row, bar);
    };
    if (tid == 0) {
        tma_prefetch_desc(&maps.q);
        tma_prefetch_desc(&maps.k);
        tma_prefetch_desc(&maps.v);
        if (SM::GT) {
            tma_prefetch_desc(&maps.gl);
            tma_prefetch_desc(&maps.bx);
        }
    }
    if ((!VL || NCCn > 0) && !a.stall) {
        issue(0, 0);
        if (SM::ST == 1) issue(0, 1);
    }
    uint32_t phase_bits = 0u;   // bit st: parity to wait for on stage st
    float dwc = 0.f;            // write-gate content term of the current gate chunk
    float wnext = (tid < C && (!VL || tid < Tn)) ? a.w_logit[((size_t)bb * T + toff + tid) * H + h] : 0.f;
    // mean q of the next gate chunk from the saved record (mode 0 with saving), one chunk ahead
    auto load_qbar = [&](int gc) {
        return (a.saved_aux && a.mc_mode == 0 && tid < 128 && gc < NG)
                   ? a.saved_aux[((size_t)u * NG + gc) * (kTcAuxFixed + R) + 256 + R + tid]
                   : 0.f;
    };
    float pqb = load_qbar(0);

    for (int cc = 0; cc < NCCn; ++cc) {
        const int t0 = cc * C, gc = cc / CPG;
        const bool first = (cc % CPG) == 0, last = (cc % CPG) == CPG - 1 || cc == NCCn - 1;
        const int n = min(L, Tn - gc * L);
        const int nv = VL ? min(C, Tn - t0) : C;   // tokens of this chunk inside the sequence
        const int st = cc % SM::ST;
        // gate inputs of this chunk, into registers (one-stage layout only; their latency
        // overlaps the readout)
        // (gate work item p: channel pair cp = p & 63, half hf = (p >> 6) & 1 of 16-token block
        //  i = p >> 7: tokens 16 i + 8 hf + [0, 8) of channels 2 cp, 2 cp + 1)
        float2 glr[NP][8], bxr[NP][8];
        if (!SM::GT) {
#pragma unroll
            for (int x = 0; x < NP; ++x) {
                const int p = tid + 256 * x, cp = p & 63, hf = (p >> 6) & 1, i = p >> 7;
                if (p < 128 * NB) {
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        const int tt = t0 + 16 * i + 8 * hf + t;
                        const size_t gi = ((size_t)bb * T + toff + tt) * tstride + (size_t)h * 128 + 2 * cp;
                        const bool in = !VL || tt < Tn;
                        glr[x][t] = in ? *reinterpret_cast<const float2 *>(a.g_logit + gi) : make_float2(0.f, 0.f);
                        bxr[x][t] = in ? *reinterpret_cast<const float2 *>(a.bx + gi) : make_float2(0.f, 0.f);
                    }
                }
            }
        }
        if (first && a.mc_mode == 0 && a.saved_aux && tid < 128) {   // the mean q, prefetched
            sm.qbar[tid] = pqb;
            pqb = load_qbar(gc + 1);
        }
        if (save && tid == 0) bulk_wait_read<0>();   // the last state copy has left its stage before that
                                                     // stage's next tile copy is issued below
        {   // a wait that gives up ends the sweep of the whole CTA: recorded, the copies of this
            // stage (the only ones in flight here) waited for once more, bounded, and left
            const bool lost = !mbar_wait(&sm.bar[st], (phase_bits >> st) & 1u, a.wait_limit);
            if (__syncthreads_or(lost)) {
                if (tid == 0) {
                    atomicOr(&g_tc_timeout, 1);
                    mbar_wait(&sm.bar[st], (phase_bits >> st) & 1u, a.wait_limit);
                }
                if (SM::UM && warp == 0) {   // no product is in flight at a chunk's start
                    tc_fence_after_sync();
                    tmem_dealloc(tmem, 64);
                }
                return;
            }
        }
        phase_bits ^= 1u << st;
        if constexpr (VL) {
            if (nv < C) {   // rows past the sequence's end (another sequence's, or zero fill): cleared
                for (int idx = tid; idx < (C - nv) * 16; idx += 256) {
                    const int off = (nv + (idx >> 4)) * 128 + (idx & 15) * 8;
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                    *reinterpret_cast<uint4 *>(&sm.rq[st][off]) = z;
                    *reinterpret_cast<uint4 *>(&sm.rk[st][off]) = z;
                    *reinterpret_cast<uint4 *>(&sm.rv[st][off]) = z;
                }
                __syncthreads();
            }
        }
        const float wcur = wnext;
        if (tid < C && cc + 1 < NCCn && (!VL || t0 + C + tid < Tn))
            wnext = a.w_logit[((size_t)bb * T + toff + t0 + C + tid) * H + h];
        // ---- content signal at a gate-chunk start: m for this warp's rows, its part of z = B m,
        //      then Delta = A z in two parts per key channel (summed by the gate phase)
        if (first) {
            float *aux = a.saved_aux ? a.saved_aux + ((size_t)u * NG + gc) * (kTcAuxFixed + R) : nullptr;
            if (a.mc_mode == 0 && !a.saved_aux) {   // mean q of the gate chunk, computed here
                if (tid < 128) {
                    float acc = 0.f;
                    if (CPG == 1) {
                        for (int t = 0; t < C; ++t) acc += bf(sm.rq[st][t * 128 + tid]);
                    } else {
#pragma unroll 8
                        for (int t = 0; t < n; ++t) acc += bf(q[base_bh + (size_t)(gc * L + t) * tstride + tid]);
                    }
                    sm.qbar[tid] = acc / (float)n;
                }
                __syncthreads();
            }
            float p0, p1;   // m[v0], m[v1] (every lane of the row's quad after the reductions)
            if (a.mc_mode == 0) {   // m = S_[c-1] qbar
                p0 = p1 = 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int col = 8 * j + 2 * c4;
                    const float q0 = sm.qbar[col], q1 = sm.qbar[col + 1];
                    p0 += s[j][0] * q0 + s[j][1] * q1;
                    p1 += s[j][2] * q0 + s[j][3] * q1;
                }
                p0 += __shfl_xor_sync(0xffffffffu, p0, 1);
                p0 += __shfl_xor_sync(0xffffffffu, p0, 2);
                p1 += __shfl_xor_sync(0xffffffffu, p1, 1);
                p1 += __shfl_xor_sync(0xffffffffu, p1, 2);
            } else {                // m = mean output of the previous gate chunk
                p0 = sm.mprev[v0];
                p1 = sm.mprev[v1];
            }
            if (aux && c4 == 0) {
                aux[v0] = p0;
                aux[v1] = p1;
            }
            {   // this warp's part of z: lane j over the warp's 16 rows
                float zz = 0.f;
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const float ma = __shfl_sync(0xffffffffu, p0, 4 * r), mb = __shfl_sync(0xffffffffu, p1, 4 * r);
                    zz += sm.BhT[(vb + r) * kTcMaxRank + lane] * ma + sm.BhT[(vb + 8 + r) * kTcMaxRank + lane] * mb;
                }
                sm.zp[warp * 32 + lane] = zz;
            }
            if (tid < 128) sm.osum[tid] = 0.f;
            __syncthreads();
            float zj = 0.f;   // z_j, j = lane, in every warp (fixed order over the parts)
#pragma unroll
            for (int w2 = 0; w2 < 8; ++w2) zj += sm.zp[w2 * 32 + lane];
            {   // dw_c = Aw . z: the same projection of m_c biases the write gate (every warp forms
                // it, so each write-gate thread holds it in a register for the whole gate chunk)
                float x = (a.Aw && lane < R) ? a.Aw[(size_t)h * R + lane] * zj : 0.f;
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
                dwc = x;
            }
            if (aux) {
                if (warp == 0 && lane < R) aux[128 + lane] = zj;
                if (tid == 0) aux[kTcAuxDw + R] = dwc;
            }
            {   // Delta = A z: two parts of sixteen rank indices each, per key channel
                const int part = tid >> 7, kk = tid & 127;
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    acc += sm.AhT[(16 * part + i) * 128 + kk] * __shfl_sync(0xffffffffu, zj, 16 * part + i);
                sm.dpart[part * 128 + kk] = acc;
            }
            __syncthreads();
            if (aux && tid < 128) aux[128 + R + tid] = sm.dpart[tid] + sm.dpart[128 + tid];
        }
        // ---- gates and mid-block referenced operands: per work item, two channels over half a
        //      16-token block, factors referenced to the block's token 7 (running products
        //      outward from it: backward over tokens 0-7, forward over tokens 8-15)
#pragma unroll
        for (int x = 0; x < NP; ++x) {
            const int p = tid + 256 * x, cp = p & 63, hf = (p >> 6) & 1, i = p >> 7, c0 = 2 * cp;
            if (p < 128 * NB) {
                const float dl0 = sm.dpart[c0] + sm.dpart[128 + c0], dl1 = sm.dpart[c0 + 1] + sm.dpart[128 + c0 + 1];
                float av[2][8], ia[2][8];
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    float2 gv, bv;
                    if (SM::GT) {
                        const int row = 16 * i + 8 * hf + t;
                        gv = *reinterpret_cast<const float2 *>(&sm.rgx[st][0][row * 128 + c0]);
                        bv = *reinterpret_cast<const float2 *>(&sm.rgx[st][1][row * 128 + c0]);
                    } else {
                        gv = glr[x][t];
                        bv = bxr[x][t];
                    }
                    if constexpr (DEC) {
                        retention_dec(gv.x + tb0, amp, bv.x + dl0, av[0][t], ia[0][t]);
                        retention_dec(gv.y + tb1, amp, bv.y + dl1, av[1][t], ia[1][t]);
                    } else {
                        retention(gv.x, bv.x + dl0, av[0][t], ia[0][t]);
                        retention(gv.y, bv.y + dl1, av[1][t], ia[1][t]);
                    }
                    if constexpr (VL) {
                        if (16 * i + 8 * hf + t >= nv) av[0][t] = av[1][t] = ia[0][t] = ia[1][t] = 1.f;   // inert row
                    }
                }
                float rf[2][8], cf[2][8];
                if (hf == 0) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        rf[e][7] = cf[e][7] = 1.f;
#pragma unroll
                        for (int t = 6; t >= 0; --t) {
                            cf[e][t] = cf[e][t + 1] * av[e][t + 1];
                            rf[e][t] = rf[e][t + 1] * ia[e][t + 1];
                        }
                    }
                    float p0 = 1.f, p1 = 1.f;
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        p0 *= av[0][t];
                        p1 *= av[1][t];
                    }
                    *reinterpret_cast<float2 *>(&sm.p7[i * 128 + c0]) = make_float2(p0, p1);
                } else {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        rf[e][0] = av[e][0];
                        cf[e][0] = ia[e][0];
#pragma unroll
                        for (int t = 1; t < 8; ++t) {
                            rf[e][t] = rf[e][t - 1] * av[e][t];
                            cf[e][t] = cf[e][t - 1] * ia[e][t];
                        }
                    }
                    *reinterpret_cast<float2 *>(&sm.r15[i * 128 + c0]) = make_float2(rf[0][7], rf[1][7]);
                }
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    const int row = 16 * i + 8 * hf + t;
                    const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162 *>(&sm.rq[st][row * 128 + c0]);
                    const __nv_bfloat162 k2 = *reinterpret_cast<const __nv_bfloat162 *>(&sm.rk[st][row * 128 + c0]);
                    const float k0 = bf(k2.x), k1 = bf(k2.y);
                    *reinterpret_cast<uint32_t *>(&sm.qm[row * kLdOp + c0]) = pack_bf16(bf(q2.x) * rf[0][t], bf(q2.y) * rf[1][t]);
                    *reinterpret_cast<uint32_t *>(&sm.krm[row * kLdOp + c0]) = pack_bf16(k0 * rf[0][t], k1 * rf[1][t]);
                    *reinterpret_cast<uint32_t *>(&sm.kcm[row * kLdOp + c0]) = pack_bf16(k0 * cf[0][t], k1 * cf[1][t]);
                }
            }
        }
        if (tid < C) sm.wv[tid] = (!VL || tid < nv) ? sigmoid_f(wcur + dwc) : 0.f;
        __syncthreads();
        __nv_bfloat16 *stile = reinterpret_cast<__nv_bfloat16 *>(sm.rgx[st]);
        if (SM::UM) {   // bf16 chunk-start state into the stage's gate tiles (read above): this warp's
                        // 16 rows, in the tensor core's operand layout (the A operand of G, and the
                        // state saved for the backward)
            const int mi = lane >> 3, r = lane & 7;   // lane l addresses row r of matrix mi of each x4
            const int row = vb + 8 * (mi & 1) + r;
#pragma unroll
            for (int q2 = 0; q2 < 8; ++q2)   // key columns 16 q2 .. 16 q2 + 15
                stsm_x4(smem_u32(stile + umma_off(row, 16 * q2 + 8 * (mi >> 1), 128)), pack_bf16(s[2 * q2][0], s[2 * q2][1]),
                        pack_bf16(s[2 * q2][2], s[2 * q2][3]), pack_bf16(s[2 * q2 + 1][0], s[2 * q2 + 1][1]),
                        pack_bf16(s[2 * q2 + 1][2], s[2 * q2 + 1][3]));
        }
        // ---- decayed operands Qt = Qm Em, Kt = Krm Em (chunk-level factors per channel alongside)
        if constexpr (SM::UM) {   // into [Kt; Qt] (rows 0 .. C-1: Kt, C .. 2C-1: Qt): one (channel,
                                  // 16-token block) item per thread; a row's chunk position in the
                                  // operand layout depends on the token index mod 8 alone
            const int ch = tid & 127, i = tid >> 7, cc = (ch >> 3) & 7;
            float E = 1.f;
            for (int j = 0; j < i; ++j) E *= sm.p7[j * 128 + ch] * sm.r15[j * 128 + ch];
            const float em = E * sm.p7[i * 128 + ch];
            __nv_bfloat16 kv[16], qv[16];   // all loads first (the stores below go through a pointer)
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const int row = 16 * i + t;
                kv[t] = __float2bfloat16_rn(bf(sm.krm[row * kLdOp + ch]) * em);
                qv[t] = __float2bfloat16_rn(bf(sm.qm[row * kLdOp + ch]) * em);
            }
            __nv_bfloat16 *kb = sm.ktq + (ch >> 6) * (2 * C * 64) + 16 * i * 64 + (ch & 7);
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const int o = t * 64 + ((cc ^ (t & 7)) << 3);
                kb[o] = kv[t];
                kb[o + C * 64] = qv[t];
            }
        } else {   // one (channel, 16-token block) item per thread
#pragma unroll
            for (int x = 0; x < NP; ++x) {
                const int p = tid + 256 * x, ch = p & 127, i = p >> 7;
                if (p < 128 * NB) {
                    float E = 1.f;
                    for (int j = 0; j < i; ++j) E *= sm.p7[j * 128 + ch] * sm.r15[j * 128 + ch];
                    const float em = E * sm.p7[i * 128 + ch];
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        const int row = 16 * i + t;
                        sm.qt[row * kLdOp + ch] = __float2bfloat16_rn(bf(sm.qm[row * kLdOp + ch]) * em);
                        sm.kt[row * kLdOp + ch] = __float2bfloat16_rn(bf(sm.krm[row * kLdOp + ch]) * em);
                    }
                }
            }
        }
        if (tid < 128) {
            float dblk[NB];   // decay over each 16-token block
#pragma unroll
            for (int i = 0; i < NB; ++i) dblk[i] = sm.p7[i * 128 + tid] * sm.r15[i * 128 + tid];
            float E = 1.f;
#pragma unroll
            for (int i = 0; i < NB; ++i) E *= dblk[i];
            sm.gam[tid] = E;
            float F = 1.f;
#pragma unroll
            for (int i = NB - 1; i >= 0; --i) {
                sm.fm[i * 128 + tid] = sm.r15[i * 128 + tid] * F;
                F *= dblk[i];
            }
            // column factor of the Gram block pair (i, j < i): e^{Lam_m(i) - Lam_m(j)} = p7_i cij,
            // cij = r15_j times the decay of the blocks between j and i; the two parts stay
            // representable where their product would underflow
#pragma unroll
            for (int i = 1; i < NB; ++i) {
                float mid = 1.f;
#pragma unroll
                for (int j = i - 1; j >= 0; --j) {
                    sm.cij[pair_index(i, j) * 128 + tid] = sm.r15[j * 128 + tid] * mid;
                    mid *= dblk[j];
                }
            }
        }
        if (SM::UM) fence_proxy_async_smem();   // the state and [Kt; Qt] tiles are read by the tensor
                                                // core and the state copy below
        __syncthreads();
        if (SM::UM && tid == 224) {   // G = S0 [Kt; Qt]^T, issued by warp 7 (no Gram block): eight
                                      // K = 16 slices, each half of the 128-byte-swizzled rows
                                      // holding four of them
            tc_fence_after_sync();
            const uint32_t a0 = smem_u32(stile), b0 = smem_u32(sm.ktq);
            constexpr uint32_t idesc = umma_idesc_bf16(128, 2 * C);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = (uint32_t)(ks & 3) * 32u;
                umma_bf16(tmem, umma_desc(a0 + (uint32_t)(ks >> 2) * (128u * 128u) + off),
                          umma_desc(b0 + (uint32_t)(ks >> 2) * (2u * C * 128u) + off), idesc, ks > 0 ? 1u : 0u);
            }
            umma_commit(&sm.mma_bar);
        }
        // the other stage's tiles were last read in the previous chunk (its state copy has been
        // waited for before this chunk's first barrier): the next chunk's tiles go there, issued
        // by warp 6, which has no Gram block to form next
        if (SM::ST == 2 && cc + 1 < NCCn) issue(cc + 1, 0, 192);
        if (save && tid == 0) {   // the chunk-start state, written to the stage's gate tiles above
            bulk_s2g(states + ((size_t)u * NCC + cc) * 128 * 128, stile, 128u * 128u * 2u);
            bulk_commit();
        }
        // ---- Gram blocks: the NB (NB + 1) / 2 blocks (i, j <= i) of each type dealt round-robin
        //      over the warps; T_ii after a diagonal Akk block, by the warp that formed it
        constexpr int NBLK = NB * (NB + 1) / 2;
        for (int q = warp; q < 2 * NBLK; q += 8) {
            const int type = q / NBLK, bq = q % NBLK;
            int i = 0;
            while ((i + 1) * (i + 2) / 2 <= bq) ++i;
            const int jd = bq - i * (i + 1) / 2;
            {
                const __nv_bfloat16 *rowop = type ? sm.qm : sm.krm;
                {
                    const int j = jd;
                    float acc[2][4] = {};
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        uint32_t af[4], bfr[4];
                        load_a(af, rowop, kLdOp, 16 * i, 16 * ks, lane);
                        load_b_nk(bfr, sm.kcm, kLdOp, 16 * j, 16 * ks, lane);
                        if (j < i) {   // e^{Lam_m(i) - Lam_m(j)} = p7 of block i (rows) x cij (columns)
                            const float *fp = sm.p7 + i * 128 + 16 * ks + 2 * c4;
                            const float *f = sm.cij + pair_index(i, j) * 128 + 16 * ks + 2 * c4;
                            af[0] = scale_bf16x2(af[0], fp[0], fp[1]);
                            af[1] = scale_bf16x2(af[1], fp[0], fp[1]);
                            af[2] = scale_bf16x2(af[2], fp[8], fp[9]);
                            af[3] = scale_bf16x2(af[3], fp[8], fp[9]);
                            bfr[0] = scale_bf16x2(bfr[0], f[0], f[1]);
                            bfr[1] = scale_bf16x2(bfr[1], f[8], f[9]);
                            bfr[2] = scale_bf16x2(bfr[2], f[0], f[1]);
                            bfr[3] = scale_bf16x2(bfr[3], f[8], f[9]);
                        }
                        mma_bf16(acc[0], af, bfr[0], bfr[1]);
                        mma_bf16(acc[1], af, bfr[2], bfr[3]);
                    }
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int tr = 16 * i + g + ((e >> 1) << 3);
                            const int sc = 16 * j + 8 * nt + 2 * c4 + (e & 1);
                            const float val = acc[nt][e];
                            if (type == 0) {
                                const bool ok = sc < tr;
                                sm.mkk[tr * LDA + sc] = __float2bfloat16_rn(ok ? sm.wv[tr] * val : 0.f);
                                if (j == i) sm.akk_d[(16 * i + tr - 16 * i) * 17 + (sc - 16 * j)] = ok ? val : 0.f;
                            } else {
                                sm.aqk[tr * LDA + sc] = __float2bfloat16_rn(sc <= tr ? val : 0.f);
                            }
                        }
                }
                if (type == 0 && jd == i) {
                    __syncwarp();
                    if (lane < 16) {   // column `lane` of T_ii = (I + Diag(w) A_ii)^-1
                        float col[16];
                        unit_lower_inverse_column(sm.akk_d + 16 * i * 17, 17, sm.wv + 16 * i, lane, col);
#pragma unroll
                        for (int t = 0; t < 16; ++t) sm.tii[(i * 16 + t) * 24 + lane] = __float2bfloat16_rn(col[t]);
                    }
                }
            }
        }
        // ---- G = S0 [Kt; Qt]^T  (rows v of this warp)
        float ga[4 * NB][4];
        if constexpr (SM::UM) {   // from the tensor core: wait for the product, load this warp's rows
            const bool lost = __any_sync(0xffffffffu, !mbar_wait(&sm.mma_bar, mma_phase, a.wait_limit));
            mma_phase ^= 1u;
            tc_fence_after_sync();
            if (!lost) tmem_ld_frags8(tmem + ((uint32_t)vb << 16), ga);
            tc_fence_before_sync();
            if (__syncthreads_or(lost)) {   // the product did not complete: recorded, waited for once
                                            // more (bounded), TMEM freed, the sweep left
                if (tid == 0) {
                    atomicOr(&g_tc_timeout, 2);
                    mbar_wait(&sm.mma_bar, mma_phase ^ 1u, a.wait_limit);
                    if (save) bulk_wait<0>();
                    if (SM::ST == 2 && cc + 1 < NCCn)   // the next chunk's tiles, issued above
                        mbar_wait(&sm.bar[(cc + 1) % SM::ST], (phase_bits >> ((cc + 1) % SM::ST)) & 1u, a.wait_limit);
                }
                if (warp == 0) {
                    tc_fence_after_sync();
                    tmem_dealloc(tmem, 64);
                }
                return;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 4 * NB; ++j) ga[j][0] = ga[j][1] = ga[j][2] = ga[j][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint32_t af[4];
                af[0] = pack_bf16(s[2 * ks][0], s[2 * ks][1]);
                af[1] = pack_bf16(s[2 * ks][2], s[2 * ks][3]);
                af[2] = pack_bf16(s[2 * ks + 1][0], s[2 * ks + 1][1]);
                af[3] = pack_bf16(s[2 * ks + 1][2], s[2 * ks + 1][3]);
#pragma unroll
                for (int np = 0; np < 2 * NB; ++np) {
                    uint32_t bfr[4];
                    load_b_nk(bfr, np < NB ? sm.kt : sm.qt, kLdOp, 16 * (np % NB), 16 * ks, lane);
                    mma_bf16(ga[2 * np], af, bfr[0], bfr[1]);
                    mma_bf16(ga[2 * np + 1], af, bfr[2], bfr[3]);
                }
            }
            __syncthreads();
        }
        if (SM::ST == 1 && cc + 1 < NCCn) issue(cc + 1, 0);
        // ---- X = Diag(w)(V - Kt S0^T), as X^T (rows v, cols t)
#pragma unroll
        for (int j = 0; j < 2 * NB; ++j) {
            const int t = 8 * j + 2 * c4;
            const float w0 = sm.wv[t], w1 = sm.wv[t + 1];
            ga[j][0] = w0 * (bf(sm.rv[st][t * 128 + v0]) - ga[j][0]);
            ga[j][1] = w1 * (bf(sm.rv[st][(t + 1) * 128 + v0]) - ga[j][1]);
            ga[j][2] = w0 * (bf(sm.rv[st][t * 128 + v1]) - ga[j][2]);
            ga[j][3] = w1 * (bf(sm.rv[st][(t + 1) * 128 + v1]) - ga[j][3]);
        }
        // ---- blocked solve:  U_i^T = (X_i^T - sum_{j<i} U_j^T M_ij^T) T_ii^T
#pragma unroll
        for (int i = 0; i < NB; ++i) {
#pragma unroll
            for (int j = 0; j < i; ++j) {
                uint32_t ua[4], bfr[4];
                ua[0] = pack_bf16(-ga[2 * j][0], -ga[2 * j][1]);
                ua[1] = pack_bf16(-ga[2 * j][2], -ga[2 * j][3]);
                ua[2] = pack_bf16(-ga[2 * j + 1][0], -ga[2 * j + 1][1]);
                ua[3] = pack_bf16(-ga[2 * j + 1][2], -ga[2 * j + 1][3]);
                load_b_nk(bfr, sm.mkk, LDA, 16 * i, 16 * j, lane);
                mma_bf16(ga[2 * i], ua, bfr[0], bfr[1]);
                mma_bf16(ga[2 * i + 1], ua, bfr[2], bfr[3]);
            }
            uint32_t ya[4], bfr[4];
            ya[0] = pack_bf16(ga[2 * i][0], ga[2 * i][1]);
            ya[1] = pack_bf16(ga[2 * i][2], ga[2 * i][3]);
            ya[2] = pack_bf16(ga[2 * i + 1][0], ga[2 * i + 1][1]);
            ya[3] = pack_bf16(ga[2 * i + 1][2], ga[2 * i + 1][3]);
            load_b_nk(bfr, sm.tii + i * 16 * 24, 24, 0, 0, lane);
            float un[2][4] = {};
            mma_bf16(un[0], ya, bfr[0], bfr[1]);
            mma_bf16(un[1], ya, bfr[2], bfr[3]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                ga[2 * i][e] = un[0][e];
                ga[2 * i + 1][e] = un[1][e];
            }
        }
        // ---- O^T = S0 Qt^T + U^T Aqk^T
#pragma unroll
        for (int i = 0; i < NB; ++i)
#pragma unroll
            for (int j = 0; j <= i; ++j) {
                uint32_t ua[4], bfr[4];
                ua[0] = pack_bf16(ga[2 * j][0], ga[2 * j][1]);
                ua[1] = pack_bf16(ga[2 * j][2], ga[2 * j][3]);
                ua[2] = pack_bf16(ga[2 * j + 1][0], ga[2 * j + 1][1]);
                ua[3] = pack_bf16(ga[2 * j + 1][2], ga[2 * j + 1][3]);
                load_b_nk(bfr, sm.aqk, LDA, 16 * i, 16 * j, lane);
                mma_bf16(ga[2 * NB + 2 * i], ua, bfr[0], bfr[1]);
                mma_bf16(ga[2 * NB + 2 * i + 1], ua, bfr[2], bfr[3]);
            }
        {
            float os0 = 0.f, os1 = 0.f;
#pragma unroll
            for (int j = 0; j < 2 * NB; ++j) {
                const float *y = ga[2 * NB + j];
                os0 += y[0] + y[1];
                os1 += y[2] + y[3];
            }
            store_frags_t<2 * NB>(sm.ost(), kLdOp, vb, ga + 2 * NB, lane);   // O^T -> [t][v]
            os0 += __shfl_xor_sync(0xffffffffu, os0, 1);
            os0 += __shfl_xor_sync(0xffffffffu, os0, 2);
            os1 += __shfl_xor_sync(0xffffffffu, os1, 1);
            os1 += __shfl_xor_sync(0xffffffffu, os1, 2);
            if (c4 == 0) {
                sm.osum[v0] += os0;
                sm.osum[v1] += os1;
            }
        }
        // ---- S = S Diag(gamma) + U^T Kbar
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int col = 8 * j + 2 * c4;
            const float g0 = sm.gam[col], g1 = sm.gam[col + 1];
            s[j][0] *= g0;
            s[j][1] *= g1;
            s[j][2] *= g0;
            s[j][3] *= g1;
        }
#pragma unroll
        for (int js = 0; js < NB; ++js) {
            uint32_t ua[4];
            ua[0] = pack_bf16(ga[2 * js][0], ga[2 * js][1]);
            ua[1] = pack_bf16(ga[2 * js][2], ga[2 * js][3]);
            ua[2] = pack_bf16(ga[2 * js + 1][0], ga[2 * js + 1][1]);
            ua[3] = pack_bf16(ga[2 * js + 1][2], ga[2 * js + 1][3]);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t bfr[4];
                load_b_kn(bfr, sm.kcm, kLdOp, 16 * np, 16 * js, lane);
                const float f0 = sm.fm[js * 128 + 16 * np + g], f1 = sm.fm[js * 128 + 16 * np + 8 + g];
                bfr[0] = scale_bf16x2(bfr[0], f0, f0);
                bfr[1] = scale_bf16x2(bfr[1], f0, f0);
                bfr[2] = scale_bf16x2(bfr[2], f1, f1);
                bfr[3] = scale_bf16x2(bfr[3], f1, f1);
                mma_bf16(s[2 * np], ua, bfr[0], bfr[1]);
                mma_bf16(s[2 * np + 1], ua, bfr[2], bfr[3]);
            }
        }
        __syncthreads();
        if (SM::ST == 1 && cc + 1 < NCCn) issue(cc + 1, 1);
        for (int idx = tid; idx < nv * 16; idx += 256) {
            const int t = idx >> 4, part = idx & 15;
            *reinterpret_cast<uint4 *>(o + base_bh + (size_t)(t0 + t) * tstride + part * 8) =
                *reinterpret_cast<const uint4 *>(sm.ost() + t * kLdOp + part * 8);
        }
        if (last) {
            if (tid < 128) sm.mprev[tid] = sm.osum[tid] / (float)n;
        }
        __syncthreads();
    }
    if (a.S_final) {
        float *Sf = a.S_final + (size_t)u * 128 * 128;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int col = 8 * j + 2 * c4;
            *reinterpret_cast<float2 *>(Sf + v0 * 128 + col) = make_float2(s[j][0], s[j][1]);
            *reinterpret_cast<float2 *>(Sf + v1 * 128 + col) = make_float2(s[j][2], s[j][3]);
        }
    }
    if (a.m_prev_out && tid < 128) a.m_prev_out[(size_t)u * 128 + tid] = sm.mprev[tid];
    if (save && tid == 0) bulk_wait<0>();   // the state copies are complete before the CTA ends
    if (SM::UM && warp == 0) {   // every warp's last load of G came before the last chunk's barriers
        tc_fence_after_sync();
        tmem_dealloc(tmem, 64);
    }
}

// Per (batch, gate chunk): mean of q over the gate chunk's tokens for every head, into the saved
// aux records (offset 256 + R of each kTcAuxFixed + R floats).  A token's H*128 channels are one
// contiguous row; each thread owns 8 consecutive channels (one 16-byte load per token).
__global__ void __launch_bounds__(256) qbar_kernel(const __nv_bfloat16 *q, float *aux, int H, int T, int L, int R,
                                                   const int *cu, long long total) {
    const int NG = (T + L - 1) / L, b = blockIdx.x / NG, gc = blockIdx.x % NG;
    int bb = b, toff = 0, Tn = T;   // cu: packed sequences
    if (cu) seq_tokens(cu, total, T, b, bb, toff, Tn, &g_tc_bad_seqlens);
    if (gc * L >= Tn) return;
    const int n = min(L, Tn - gc * L);
    const size_t row = (size_t)H * 128;
    const __nv_bfloat16 *src = q + ((size_t)bb * T + toff + (size_t)gc * L) * row;
    for (int c8 = threadIdx.x; c8 < H * 16; c8 += blockDim.x) {
        float acc[2][8] = {};
        int t = 0;
        for (; t + 2 <= n; t += 2)
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const uint4 v = *reinterpret_cast<const uint4 *>(src + (size_t)(t + x) * row + c8 * 8);
                const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc[x][2 * e] += bf(p[e].x);
                    acc[x][2 * e + 1] += bf(p[e].y);
                }
            }
        for (; t < n; ++t) {
            const uint4 v = *reinterpret_cast<const uint4 *>(src + (size_t)t * row + c8 * 8);
            const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[0][2 * e] += bf(p[e].x);
                acc[0][2 * e + 1] += bf(p[e].y);
            }
        }
        const int h = c8 / 16, ch = (c8 % 16) * 8;
        float *dst = aux + (((size_t)b * H + h) * NG + gc) * (kTcAuxFixed + R) + 256 + R + ch;
#pragma unroll
        for (int e = 0; e < 8; ++e) dst[e] = (acc[0][e] + acc[1][e]) / (float)n;
    }
}

template <int NB>
cudaError_t launch_tc_fwd_t(const FwdArgs &a, cudaStream_t st) {
    const bool dec = a.A_dec || a.tau, vl = a.cu_seqlens != nullptr;
    auto kern = vl ? (dec ? tc_fwd_kernel<NB, true, true> : tc_fwd_kernel<NB, false, true>)
                   : (dec ? tc_fwd_kernel<NB, true, false> : tc_fwd_kernel<NB, false, false>);
    const int bytes = (int)sizeof(TcFwdSmem<NB>);
    cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), bytes);
    if (e != cudaSuccess) return e;
    const int C = 16 * NB;
    // token rows of the tensors: B T, or the packed row count (at least 1 for a valid map; no
    // copy is issued for a sequence without tokens)
    const long long rows = a.cu_seqlens ? (a.total > 0 ? a.total : 1) : (long long)a.B * a.T;
    TileMaps maps;
    if ((e = make_token_tile_map(&maps.q, a.q, 2, 128, a.H, rows, C)) != cudaSuccess) return e;
    if ((e = make_token_tile_map(&maps.k, a.k, 2, 128, a.H, rows, C)) != cudaSuccess) return e;
    if ((e = make_token_tile_map(&maps.v, a.v, 2, 128, a.H, rows, C)) != cudaSuccess) return e;
    if (TcFwdSmem<NB>::GT) {
        if ((e = make_token_tile_map(&maps.gl, a.g_logit, 4, 128, a.H, rows, C)) != cudaSuccess) return e;
        if ((e = make_token_tile_map(&maps.bx, a.bx, 4, 128, a.H, rows, C)) != cudaSuccess) return e;
    }
    if (a.saved_aux && a.mc_mode == 0) {
        const int NG = (a.T + a.L - 1) / a.L;
        qbar_kernel<<<a.B * NG, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(a.q), a.saved_aux, a.H, a.T, a.L,
                                              a.R, a.cu_seqlens, a.total);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    kern<<<a.B * a.H, 256, bytes, st>>>(a, maps);
    return cudaGetLastError();
}

// Compute chunk of the tensor-core forward for a gate chunk L (0 = not supported).
int tc_compute_chunk(int L) { return L == 32 ? 32 : (L == 64 || L == 128) ? 64 : 0; }

// C = 32 or 64 tokens per compute chunk.  With a.saved_states set (32-token chunks), a bf16
// copy of the state at every compute-chunk start ([T/32][128][128] per unit, each row's 16-byte
// chunks at positions c ^ (row & 7)) and
// per gate chunk the record (m, z, Delta, mean q, dw) of kTcAuxFixed + R floats are written for the
// backward.
cudaError_t launch_fwd_tc(const FwdArgs &a, int C, cudaStream_t st) {
    return C == 32 ? launch_tc_fwd_t<2>(a, st) : launch_tc_fwd_t<4>(a, st);
}

size_t tc_fwd_smem(int L) { return tc_compute_chunk(L) == 32 ? sizeof(TcFwdSmem<2>) : sizeof(TcFwdSmem<4>); }

// Device status word of the packed-sequence offsets (this file): returns and clears it.
int tc_fwd_take_bad_seqlens() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_bad_seqlens, sizeof(int)) != cudaSuccess) return 0;
    if (v) {
        const int z = 0;
        cudaMemcpyToSymbol(g_tc_bad_seqlens, &z, sizeof(int));
    }
    return v;
}

// Device status word of this file: returns and clears it.
int tc_fwd_take_timeout() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_timeout, sizeof(int)) != cudaSuccess) return 0;
    if (v) {
        const int z = 0;
        cudaMemcpyToSymbol(g_tc_timeout, &z, sizeof(int));
    }
    return v;
}

}  // namespace carve

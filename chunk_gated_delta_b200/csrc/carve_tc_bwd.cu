// CARVE backward, tensor-core kernel for bf16 q/k/v/o with dk = dv = 128.
//
// One CTA (8 warps) per (batch, head) unit sweeps the compute chunks of 32 tokens in reverse.
// Warp w owns rows v in [16w, 16w+16) of the carried state gradient dS, kept in registers as
// mma accumulator fragments.  Per chunk, from the saved chunk-start state S0 and the saved
// content signal Delta:
//   recompute  gates (as the forward), Gram blocks Akk/Aqk, T_ii, R = V - Kt S0^T,
//              U (blocked WY solve) and E = R - Akk U (the prediction errors v - S Diag(a) k)
//   per warp   dU^T = dO^T Aqk + dS1 Kbar^T;  dY^T = dU^T M^-1 (blocked back substitution);
//              dR = Diag(w) dY;  dw_t = sum_v dY E;  dS0 = dS1 Diag(gamma) + dO^T Qt - dR^T Kt
//   cross-warp dAqk = dO U^T, dAkk = -dR U^T (reductions over v), then, per (token block,
//              channel quarter), with every decay factor folded into a B operand:
//                Gq  = dO (S0 Em) + dAqk (Kcm C)          -> dq   = r Gq
//                Gkr = -dR (S0 Em) + dAkk (Kcm C)         -> dk   = r Gkr + Gkc / r
//                Gkc = dAqk^T (Qm C) + dAkk^T (Krm C)
//                Gkb = U (dS1 Fm)                          (the Kbar part of Gkc)
//                dLam = Qm Gq + Krm Gkr - Kcm (Gkc + Gkb)
//                       (+ sum_s Kbar_s dKbar_s + gamma colsum(S0 * dS1) at the chunk's last token)
//   gates      dl = reverse cumsum of dLam; d g_logit = -amp sigma(g_logit + tau) dl (amp = 1,
//              tau = 0 without the decay parameters; d tau sums it, d A_dec sums dl log g);
//              dbx = sigma(-beta) dl
// (Qm, Krm, Kcm: mid-block referenced operands; Em, Fm, C: the block-level decay factors of the
// forward.)  The content path (dz = A^T dDelta, dm = B^T dz) closes each gate chunk; with the
// boundary-state readout its term in dq (S0^T dm / n for every token of the gate chunk) is
// stored per gate chunk and added by a parallel pass after the sweep.
// Terms that cancel pairwise in the reverse cumulative sum of dLam (a Gram entry's row and
// column token; Kbar_s against the chunk's last token) are formed from the same rounded values
// on both sides, so the cancellation stays exact to fp32 rounding.  Two such pairs have no
// dependence on Lam at all and are left out of dLam on both sides: the diagonal of Aqk
// (q_t . k_t, decay factor 1; its fp32 value goes to dq and dk directly) and the Kbar term of
// the chunk's last token (factor e^{Lam_C - Lam_C} = 1).  Under strong erasure the gradient of
// log a is tiny (proportional to a) while those pairs are O(1), so their rounding would swamp
// it.  For the same reason the off-diagonal Gram blocks' factor e^{Lam_m(1) - Lam_m(0)} is
// never formed alone (it underflows fp32 under strong decay where the whole product does
// not): the row block's part and the column block's part are applied separately.  Where the
// retention floor binds, the gradient of log a is scaled to the exact recurrence's
// (floor_scale) instead of being dropped.
#include "carve_tc_common.cuh"
#include "carve_umma.cuh"

namespace carve {

constexpr int kBC = 32;     // compute chunk of the backward
constexpr int kBNB = 2;     // 16-token blocks per compute chunk
constexpr int kLdT = 40;    // bf16 row stride of 32-wide tiles
constexpr int kTcMaxRankBwd = 32;   // rank limit of the tensor-core path
constexpr int kLdF = 136;   // fp32 row stride of the per-(token, channel) tables: the fragment
                            // lane pattern (row g, column pair c4) reads float2 without conflicts

struct BwdMaps {
    CUtensorMap q, k, v, dO;
};

struct __align__(16) TcBwdSmem {
    // TMA tiles; after the gate recompute rq / rk hold the swizzled Qt / Kt of the chunk
    __nv_bfloat16 rq[kBC * 128], rk[kBC * 128], rv[kBC * 128], rdo[kBC * 128];
    __nv_bfloat16 dop[kBC * kLdOp];
    __nv_bfloat16 qm[kBC * kLdOp], krm[kBC * kLdOp], kcm[kBC * kLdOp];
    __nv_bfloat16 s0b[128 * 128], ds1b[128 * kLdOp];   // s0b: the saved state as written (tensor-core layout)
    __nv_bfloat16 ub[kBC * kLdOp], drb[kBC * kLdOp];
    __nv_bfloat16 aqk[kBC * kLdT], akk[kBC * kLdT], mkk[kBC * kLdT], daqk[kBC * kLdT], dakk[kBC * kLdT];
    __nv_bfloat16 tii[kBNB * 16 * 24];
    float akk_d[kBC * 17];
    float rfac[kBC * kLdF], dlam[kBC * kLdF];
    float p7[kBNB * 128], r15[kBNB * 128], em[kBNB * 128], fm[kBNB * 128];
    float gam[128], wv[kBC], dwp[8 * kBC], s0ds[128], xp[8 * 128], htot[2 * kBNB * 128], pdd[2 * kBNB * 128];
    float bpart[kBNB * 128];
    float delta[128], ddelta[128], dzv[64], dmv[128], dox[128], qbar[128];
    float daqd[kBC];   // diagonal of dAqk (kept out of the bf16 tile)
    float fs0[128];    // floor_scale of the sequence's first token, per key channel (first chunk)
    float dwc, ddw;   // the write gate's content term of the gate chunk and its gradient
    uint64_t bar, bar_s0, bar_ab;
};

// the dynamic shared-memory limit of one CTA on sm_100 (227 KB); the content path's factors
// (2 x 128 x rank floats) fit in the dO and operand tiles, which are contiguous
static_assert(sizeof(TcBwdSmem) <= 232448, "shared memory");
// rows of d g_logit / dbx (staged in dlam / rfac) and dv (drb) leave by 1-D bulk copies
static_assert(offsetof(TcBwdSmem, dlam) % 16 == 0 && offsetof(TcBwdSmem, rfac) % 16 == 0 &&
                  offsetof(TcBwdSmem, drb) % 16 == 0 && (kLdF * 4) % 16 == 0 && (kLdOp * 2) % 16 == 0,
              "bulk-store sources on 16-byte boundaries");
static_assert(offsetof(TcBwdSmem, dmv) % 16 == 0, "dm read as float4");
static_assert(offsetof(TcBwdSmem, kcm) + sizeof(TcBwdSmem::kcm) - offsetof(TcBwdSmem, dop) >= 256 * kTcMaxRankBwd * 4 &&
                  offsetof(TcBwdSmem, qm) == offsetof(TcBwdSmem, dop) + sizeof(TcBwdSmem::dop) &&
                  offsetof(TcBwdSmem, kcm) == offsetof(TcBwdSmem, krm) + sizeof(TcBwdSmem::krm),
              "A and B of the content path fit in dop .. kcm");

__device__ int g_tc_bwd_timeout;
__device__ int g_tc_bwd_bad_seqlens;   // set when a packed sequence's offsets are out of range

// DEC: the decay has its amplitude and bias (a.A_dec or a.tau given).  VL: the units are
// packed sequences (a.cu_seqlens); rows of a partial last chunk past the sequence's end are
// inert, carry no output gradient and are never stored.
template <bool DEC, bool VL>
__global__ void __launch_bounds__(256, 1) tc_bwd_kernel(BwdArgs a, const __grid_constant__ BwdMaps maps) {
    constexpr int C = kBC, NB = kBNB;
    extern __shared__ __align__(128) unsigned char smraw[];
    TcBwdSmem &sm = *reinterpret_cast<TcBwdSmem *>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, c4 = lane & 3;
    const int u = blockIdx.x, H = a.H, T = a.T, R = a.R, L = a.L;
    const int b = u / H, h = u % H;
    const int NCC = T / C, CPG = L / C, NG = (T + L - 1) / L;   // record strides
    int bb = b, toff = 0, Tn = T;   // this unit's tokens: rows [toff, toff + Tn) of tensor batch bb
    if constexpr (VL) seq_tokens(a.cu_seqlens, a.total, T, b, bb, toff, Tn, &g_tc_bwd_bad_seqlens);
    const int NCCn = VL ? (Tn + C - 1) / C : NCC, NGn = VL ? (Tn + L - 1) / L : NG;
    __nv_bfloat16 *dq = static_cast<__nv_bfloat16 *>(a.dq), *dk = static_cast<__nv_bfloat16 *>(a.dk);
    __nv_bfloat16 *dv = static_cast<__nv_bfloat16 *>(a.dv);
    const size_t tstride = (size_t)H * 128;
    const size_t base_bh = ((size_t)bb * T + toff) * tstride + (size_t)h * 128;
    const int v0 = 16 * warp + g, v1 = v0 + 8;
    // bf16 chunk-start states written by the forward: 128 rows in the tensor core's 128-byte-swizzle
    // operand layout (two 64-column halves of 128-byte rows)
    const __nv_bfloat16 *states = reinterpret_cast<const __nv_bfloat16 *>(a.saved_states) + (size_t)u * NCC * 128 * 128;
    // workspace: per gate chunk dDelta (128) and dz (32) for the dA / dB reduction, then the
    // readout vectors of dq (128 per gate chunk)
    float *wsg = a.ws + (size_t)u * NG * kTcGradRec;
    float *wsv = a.ws + (size_t)a.B * a.H * NG * kTcGradRec + (size_t)u * NG * 128;
    // gate phases: channel pair c0 = 2 cp, 2 cp + 1 over tokens 8 hf + [0, 8) of 16-token block ib
    const int cp = tid & 63, hf = (tid >> 6) & 1, ib = tid >> 7, c0 = 2 * cp;
    // the decay's amplitude and this thread's channel biases; its partial sums of d tau (two
    // channels) and d A_dec over the sweep
    const float amp = DEC ? decay_amp(a.A_dec, h) : 1.f;
    const float tb[2] = {DEC ? decay_bias(a.tau, h, c0, 128) : 0.f, DEC ? decay_bias(a.tau, h, c0 + 1, 128) : 0.f};
    float dtp[2] = {0.f, 0.f}, dap = 0.f;
    // the content path's factors A [128][R] and B [R][128] of this head, brought in by a bulk copy
    // at each gate chunk's first token into the dO and operand tiles (contiguous, 34,816 bytes,
    // all consumed by then); lane j's write-gate factor
    float *abuf = reinterpret_cast<float *>(sm.dop);
    const float awj = (a.Aw && lane < R) ? a.Aw[(size_t)h * R + lane] : 0.f;
    uint32_t ab_phase = 0;

    float ds[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int col = 8 * j + 2 * c4;
        if (a.dS_final) {
            const float *D = a.dS_final + (size_t)u * 128 * 128;
            ds[j][0] = D[v0 * 128 + col];
            ds[j][1] = D[v0 * 128 + col + 1];
            ds[j][2] = D[v1 * 128 + col];
            ds[j][3] = D[v1 * 128 + col + 1];
        } else {
            ds[j][0] = ds[j][1] = ds[j][2] = ds[j][3] = 0.f;
        }
    }

    // column sums over this warp's rows of (dS .* S0), S0 from the bf16 tile, into sm.xp[warp];
    // the reduction over the 8 row lanes halves the live values at each exchange
    auto colsum_partial = [&]() {
        float v[16][2];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int col = 8 * j + 2 * c4;
            const __nv_bfloat162 s0 = *reinterpret_cast<const __nv_bfloat162 *>(sm.s0b + umma_off(v0, col, 128));
            const __nv_bfloat162 s1 = *reinterpret_cast<const __nv_bfloat162 *>(sm.s0b + umma_off(v1, col, 128));
            v[j][0] = ds[j][0] * bf(s0.x) + ds[j][2] * bf(s1.x);
            v[j][1] = ds[j][1] * bf(s0.y) + ds[j][3] * bf(s1.y);
        }
        const bool up1 = g & 4, up2 = g & 2, up3 = g & 1;
        float w1[8][2], w2[4][2], w3[2][2];
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e)
                w1[j][e] = (up1 ? v[j + 8][e] : v[j][e]) + __shfl_xor_sync(0xffffffffu, up1 ? v[j][e] : v[j + 8][e], 16);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e)
                w2[j][e] = (up2 ? w1[j + 4][e] : w1[j][e]) + __shfl_xor_sync(0xffffffffu, up2 ? w1[j][e] : w1[j + 4][e], 8);
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e)
                w3[j][e] = (up3 ? w2[j + 2][e] : w2[j][e]) + __shfl_xor_sync(0xffffffffu, up3 ? w2[j][e] : w2[j + 2][e], 4);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int jj = j + (up3 ? 2 : 0) + (up2 ? 4 : 0) + (up1 ? 8 : 0);
            sm.xp[warp * 128 + 8 * jj + 2 * c4] = w3[j][0];
            sm.xp[warp * 128 + 8 * jj + 2 * c4 + 1] = w3[j][1];
        }
    };

    if (tid == 0) {
        mbar_init(&sm.bar, 1);
        mbar_init(&sm.bar_s0, 1);
        mbar_init(&sm.bar_ab, 1);
        fence_mbar_init();
    }
    if (tid < 128) {
        const int nl = Tn - (NGn - 1) * L;
        sm.dox[tid] = a.dm_prev_out ? a.dm_prev_out[(size_t)u * 128 + tid] / (float)nl : 0.f;
    }
    auto issue = [&](int cc) {
        if (tid != 0) return;
        const int row = bb * T + toff + cc * C;
        mbar_expect_tx(&sm.bar, 4u * C * 256u);
        tma_load_3d(sm.rq, &maps.q, 0, h, row, &sm.bar);
        tma_load_3d(sm.rk, &maps.k, 0, h, row, &sm.bar);
        tma_load_3d(sm.rv, &maps.v, 0, h, row, &sm.bar);
        tma_load_3d(sm.rdo, &maps.dO, 0, h, row, &sm.bar);
    };
    auto issue_s0 = [&](int cc) {
        if (tid != 0) return;
        mbar_expect_tx(&sm.bar_s0, 128u * 128u * 2u);
        bulk_g2s(sm.s0b, states + (size_t)cc * 128 * 128, 128u * 128u * 2u, &sm.bar_s0);
    };
    if (!VL || NCCn > 0) {
        if (!a.stall) issue(NCCn - 1);
        issue_s0(NCCn - 1);
    }
    uint32_t phase = 0;
    __syncthreads();
    // gate logits of the chunk about to be processed, loaded one chunk ahead
    float2 glr[8], bxr[8];
    auto load_gates = [&](int cc) {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int tt = cc * C + 16 * ib + 8 * hf + t;
            const size_t gi = base_bh + (size_t)tt * tstride + c0;
            const bool in = !VL || tt < Tn;
            glr[t] = in ? *reinterpret_cast<const float2 *>(a.g_logit + gi) : make_float2(0.f, 0.f);
            bxr[t] = in ? *reinterpret_cast<const float2 *>(a.bx + gi) : make_float2(0.f, 0.f);
        }
    };
    if (!VL || NCCn > 0) load_gates(NCCn - 1);
    // the saved record of the next gate chunk (loaded when the current one is taken) and the
    // write logits of the next compute chunk (loaded one iteration ahead)
    float pd = 0.f, pq = 0.f, pw = 0.f, pdw = 0.f;
    auto load_aux = [&](int gc) {   // Delta, the mean q and the write-gate term of a gate chunk
        const float *aux = a.saved_aux + ((size_t)u * NG + gc) * (kTcAuxFixed + R);
        if (tid < 128) {
            pd = aux[128 + R + tid];
            pq = aux[256 + R + tid];
        }
        if (tid == 0) pdw = aux[kTcAuxDw + R];
    };
    auto load_w = [&](int cc) {
        if (tid < C && (!VL || cc * C + tid < Tn)) pw = a.w_logit[((size_t)bb * T + toff + (size_t)cc * C + tid) * H + h];
    };
    if (!VL || NCCn > 0) {
        load_aux((NCCn - 1) / CPG);
        load_w(NCCn - 1);
    }

    for (int cc = NCCn - 1; cc >= 0; --cc) {
        const int t0 = cc * C, gc = cc / CPG;
        const int nv = VL ? min(C, Tn - t0) : C;   // tokens of this chunk inside the sequence
        const bool gate_end = (cc % CPG) == CPG - 1 || cc == NCCn - 1;
        const bool gate_start = (cc % CPG) == 0;
        const int n = min(L, Tn - gc * L);
        if (gate_end) {
            if (tid < 128) {
                sm.delta[tid] = pd;
                sm.qbar[tid] = pq;
                sm.ddelta[tid] = 0.f;
            }
            if (tid == 0) {
                sm.dwc = pdw;
                sm.ddw = 0.f;
            }
            if (gc > 0) load_aux(gc - 1);   // the previous gate chunk's record, a gate chunk ahead
        }
        {   // the carried gradient as a bf16 tile [v][k]: this warp's 16 rows (stmatrix; lane l
            // addresses row l % 8 of matrix l / 8 of each x4: rows +0 / +8, columns +0 / +8)
            const int mi = lane >> 3, r = lane & 7;
            const uint32_t base = smem_u32(sm.ds1b + (16 * warp + 8 * (mi & 1) + r) * kLdOp + 8 * (mi >> 1));
#pragma unroll
            for (int q2 = 0; q2 < 8; ++q2)   // key columns 16 q2 .. 16 q2 + 15
                stsm_x4(base + 32 * q2, pack_bf16(ds[2 * q2][0], ds[2 * q2][1]), pack_bf16(ds[2 * q2][2], ds[2 * q2][3]),
                        pack_bf16(ds[2 * q2 + 1][0], ds[2 * q2 + 1][1]),
                        pack_bf16(ds[2 * q2 + 1][2], ds[2 * q2 + 1][3]));
        }
        // the previous chunk's gradient rows have left dlam / rfac / drb before the barrier below
        // (those tiles are written again in this chunk)
        if (lane < 4) bulk_wait_read<0>();
        {   // a wait that gives up ends the sweep of the whole CTA: recorded, the copies in flight
            // (this chunk's tiles and its start state) waited for once more, bounded, and left
            const bool lost = !mbar_wait(&sm.bar, phase, a.wait_limit);
            if (__syncthreads_or(lost)) {
                if (tid == 0) {
                    atomicOr(&g_tc_bwd_timeout, 1);
                    mbar_wait(&sm.bar, phase, a.wait_limit);
                    mbar_wait(&sm.bar_s0, phase, a.wait_limit);
                }
                if (lane < 4) bulk_wait<0>();
                return;
            }
        }
        if constexpr (VL) {
            if (nv < C) {   // rows past the sequence's end (another sequence's, or zero fill): cleared;
                            // the proxy fence after the Qt / Kt stores below orders these writes
                            // before the next chunk's tile copies
                for (int idx = tid; idx < (C - nv) * 16; idx += 256) {
                    const int off = (nv + (idx >> 4)) * 128 + (idx & 15) * 8;
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                    *reinterpret_cast<uint4 *>(sm.rq + off) = z;
                    *reinterpret_cast<uint4 *>(sm.rk + off) = z;
                    *reinterpret_cast<uint4 *>(sm.rv + off) = z;
                }
                __syncthreads();
            }
        }
        // dO plus the content-signal gradient carried from the next gate chunk, padded (inert
        // rows: none)
        for (int idx = tid; idx < C * 16; idx += 256) {
            const int t = idx >> 4, part = idx & 15;
            if (VL && t >= nv) {
                *reinterpret_cast<uint4 *>(sm.dop + t * kLdOp + part * 8) = make_uint4(0u, 0u, 0u, 0u);
                continue;
            }
            const uint4 x = *reinterpret_cast<const uint4 *>(sm.rdo + t * 128 + part * 8);
            const __nv_bfloat16 *xv = reinterpret_cast<const __nv_bfloat16 *>(&x);
            const float *dx = sm.dox + part * 8;
            uint4 y;
            y.x = pack_bf16(bf(xv[0]) + dx[0], bf(xv[1]) + dx[1]);
            y.y = pack_bf16(bf(xv[2]) + dx[2], bf(xv[3]) + dx[3]);
            y.z = pack_bf16(bf(xv[4]) + dx[4], bf(xv[5]) + dx[5]);
            y.w = pack_bf16(bf(xv[6]) + dx[6], bf(xv[7]) + dx[7]);
            *reinterpret_cast<uint4 *>(sm.dop + t * kLdOp + part * 8) = y;
        }
        // ---- recompute: gates and mid-block referenced operands (as the forward: running
        //      products outward from the block's token 7, two channels per thread)
        {
            const float dl0 = sm.delta[c0], dl1 = sm.delta[c0 + 1];
            float av[2][8], ia[2][8], rf[2][8], cf[2][8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                if constexpr (DEC) {
                    retention_dec(glr[t].x + tb[0], amp, bxr[t].x + dl0, av[0][t], ia[0][t]);
                    retention_dec(glr[t].y + tb[1], amp, bxr[t].y + dl1, av[1][t], ia[1][t]);
                } else {
                    retention(glr[t].x, bxr[t].x + dl0, av[0][t], ia[0][t]);
                    retention(glr[t].y, bxr[t].y + dl1, av[1][t], ia[1][t]);
                }
                if constexpr (VL) {
                    if (16 * ib + 8 * hf + t >= nv) av[0][t] = av[1][t] = ia[0][t] = ia[1][t] = 1.f;   // inert row
                }
            }
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
                *reinterpret_cast<float2 *>(&sm.p7[ib * 128 + c0]) = make_float2(p0, p1);
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
                *reinterpret_cast<float2 *>(&sm.r15[ib * 128 + c0]) = make_float2(rf[0][7], rf[1][7]);
            }
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const int row = 16 * ib + 8 * hf + t;
                const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162 *>(&sm.rq[row * 128 + c0]);
                const __nv_bfloat162 k2 = *reinterpret_cast<const __nv_bfloat162 *>(&sm.rk[row * 128 + c0]);
                const float k0 = bf(k2.x), k1 = bf(k2.y);
                *reinterpret_cast<uint32_t *>(&sm.qm[row * kLdOp + c0]) = pack_bf16(bf(q2.x) * rf[0][t], bf(q2.y) * rf[1][t]);
                *reinterpret_cast<uint32_t *>(&sm.krm[row * kLdOp + c0]) = pack_bf16(k0 * rf[0][t], k1 * rf[1][t]);
                *reinterpret_cast<uint32_t *>(&sm.kcm[row * kLdOp + c0]) = pack_bf16(k0 * cf[0][t], k1 * cf[1][t]);
                *reinterpret_cast<float2 *>(&sm.rfac[row * kLdF + c0]) = make_float2(rf[0][t], rf[1][t]);
            }
        }
        if (tid < C) sm.wv[tid] = (!VL || tid < nv) ? sigmoid_f(pw + sm.dwc) : 0.f;
        if (cc == 0 && tid < 64) {   // token 0 of the sequence (these threads hold its gate logits)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float gx = e ? glr[0].y : glr[0].x, beta = (e ? bxr[0].y : bxr[0].x) + sm.delta[c0 + e];
                const float D = DEC ? __expf(amp * softplus_fast(gx + tb[e], __expf(gx + tb[e]))) * (1.f + __expf(-beta))
                                    : (1.f + __expf(gx)) * (1.f + __expf(-beta));
                sm.fs0[c0 + e] = floor_scale(__fdividef(1.f, D), false);
            }
        }
        __syncthreads();
        if (tid < 128) {
            float dblk[NB];   // decay over each 16-token block
#pragma unroll
            for (int i = 0; i < NB; ++i) dblk[i] = sm.p7[i * 128 + tid] * sm.r15[i * 128 + tid];
            float E = 1.f;
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                sm.em[i * 128 + tid] = E * sm.p7[i * 128 + tid];
                E *= dblk[i];
            }
            sm.gam[tid] = E;
            float F = 1.f;
#pragma unroll
            for (int i = NB - 1; i >= 0; --i) {
                sm.fm[i * 128 + tid] = sm.r15[i * 128 + tid] * F;
                F *= dblk[i];
            }
        }
        // decayed operands Qt = Qm Em, Kt = Krm Em into the (now free) raw q / k tiles, swizzled:
        // items of 8 channels of one token row, each forming its block's decay prefix
        for (int it = tid; it < 2 * C * 16; it += 256) {
            const int tile = it / (C * 16), t = (it >> 4) % C, c8 = it & 15, i = t >> 4;
            const float4 *p7v = reinterpret_cast<const float4 *>(sm.p7 + i * 128 + 8 * c8);
            float em[8];
            {
                const float4 a0 = p7v[0], a1 = p7v[1];
                em[0] = a0.x; em[1] = a0.y; em[2] = a0.z; em[3] = a0.w;
                em[4] = a1.x; em[5] = a1.y; em[6] = a1.z; em[7] = a1.w;
            }
            for (int j = 0; j < i; ++j) {   // times the decay of each earlier block
                const float4 *pj = reinterpret_cast<const float4 *>(sm.p7 + j * 128 + 8 * c8);
                const float4 *rj = reinterpret_cast<const float4 *>(sm.r15 + j * 128 + 8 * c8);
                const float4 p0 = pj[0], p1 = pj[1], r0 = rj[0], r1 = rj[1];
                em[0] *= p0.x * r0.x; em[1] *= p0.y * r0.y; em[2] *= p0.z * r0.z; em[3] *= p0.w * r0.w;
                em[4] *= p1.x * r1.x; em[5] *= p1.y * r1.y; em[6] *= p1.z * r1.z; em[7] *= p1.w * r1.w;
            }
            const __nv_bfloat16 *src = (tile ? sm.krm : sm.qm) + t * kLdOp + 8 * c8;
            const uint4 x = *reinterpret_cast<const uint4 *>(src);
            const __nv_bfloat162 *xv = reinterpret_cast<const __nv_bfloat162 *>(&x);
            uint4 y;
            uint32_t *yv = reinterpret_cast<uint32_t *>(&y);
#pragma unroll
            for (int e = 0; e < 4; ++e) yv[e] = pack_bf16(bf(xv[e].x) * em[2 * e], bf(xv[e].y) * em[2 * e + 1]);
            __nv_bfloat16 *dst = tile ? sm.rk : sm.rq;
            *reinterpret_cast<uint4 *>(dst + t * 128 + ((c8 ^ (t & 7)) << 3)) = y;
        }
        fence_proxy_async_smem();   // the next chunk's tile copy overwrites these
        const bool lost_s0 = !mbar_wait(&sm.bar_s0, phase, a.wait_limit);
        colsum_partial();   // for gamma * dgamma (discarded if the state copy did not arrive)
        if (__syncthreads_or(lost_s0)) {   // the state copy is the only one in flight here
            if (tid == 0) {
                atomicOr(&g_tc_bwd_timeout, 2);
                mbar_wait(&sm.bar_s0, phase, a.wait_limit);
            }
            if (lane < 4) bulk_wait<0>();
            return;
        }
        phase ^= 1u;
        if (tid < 128) {
            float x = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) x += sm.xp[w * 128 + tid];
            sm.s0ds[tid] = x;
        }
        // ---- Gram blocks (warps 0-5: one (type, i, j) block each), T_ii on the diagonal Akk warps
        if (warp < 6) {
            const int type = warp / 3, blk = warp % 3;
            const int i = blk == 0 ? 0 : 1, jd = blk == 1 ? 0 : i;   // blocks (0,0), (1,0), (1,1)
            const __nv_bfloat16 *rowop = type ? sm.qm : sm.krm;
            {
                const int j = jd;
                float acc[2][4] = {};
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    uint32_t af[4], bfr[4];
                    load_a(af, rowop, kLdOp, 16 * i, 16 * ks, lane);
                    load_b_nk(bfr, sm.kcm, kLdOp, 16 * j, 16 * ks, lane);
                    if (j < i) {   // e^{Lam_m(1) - Lam_m(0)} split: p7 of the row block, r15 of the column block
                        const float *fp = sm.p7 + i * 128 + 16 * ks + 2 * c4, *fr = sm.r15 + j * 128 + 16 * ks + 2 * c4;
                        af[0] = scale_bf16x2(af[0], fp[0], fp[1]);
                        af[1] = scale_bf16x2(af[1], fp[0], fp[1]);
                        af[2] = scale_bf16x2(af[2], fp[8], fp[9]);
                        af[3] = scale_bf16x2(af[3], fp[8], fp[9]);
                        bfr[0] = scale_bf16x2(bfr[0], fr[0], fr[1]);
                        bfr[1] = scale_bf16x2(bfr[1], fr[8], fr[9]);
                        bfr[2] = scale_bf16x2(bfr[2], fr[0], fr[1]);
                        bfr[3] = scale_bf16x2(bfr[3], fr[8], fr[9]);
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
                            sm.akk[tr * kLdT + sc] = __float2bfloat16_rn(ok ? val : 0.f);
                            sm.mkk[tr * kLdT + sc] = __float2bfloat16_rn(ok ? sm.wv[tr] * val : 0.f);
                            if (j == i) sm.akk_d[tr * 17 + (sc - 16 * j)] = ok ? val : 0.f;
                        } else {
                            sm.aqk[tr * kLdT + sc] = __float2bfloat16_rn(sc <= tr ? val : 0.f);
                        }
                    }
            }
            if (type == 0 && jd == i) {
                __syncwarp();
                if (lane < 16) {
                    float col[16];
                    unit_lower_inverse_column(sm.akk_d + 16 * i * 17, 17, sm.wv + 16 * i, lane, col);
#pragma unroll
                    for (int t = 0; t < 16; ++t) sm.tii[(i * 16 + t) * 24 + lane] = __float2bfloat16_rn(col[t]);
                }
            }
        }
        // ---- R = V - S0 Kt^T  (rows v of this warp, cols t)
        float rr[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) rr[j][0] = rr[j][1] = rr[j][2] = rr[j][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t af[4];
            load_a_um(af, sm.s0b, 128, 16 * warp, 16 * ks, lane);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bfr[4];
                load_b_nk_swz(bfr, sm.rk, 16 * np, 16 * ks, lane);   // Kt
                mma_bf16(rr[2 * np], af, bfr[0], bfr[1]);
                mma_bf16(rr[2 * np + 1], af, bfr[2], bfr[3]);
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = 8 * j + 2 * c4;
            rr[j][0] = bf(sm.rv[t * 128 + v0]) - rr[j][0];
            rr[j][1] = bf(sm.rv[(t + 1) * 128 + v0]) - rr[j][1];
            rr[j][2] = bf(sm.rv[t * 128 + v1]) - rr[j][2];
            rr[j][3] = bf(sm.rv[(t + 1) * 128 + v1]) - rr[j][3];
        }
        __syncthreads();
        // ---- U (blocked WY solve), E = R - Akk U, U -> shared tile
        float ga[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = 8 * j + 2 * c4;
            const float w0 = sm.wv[t], w1 = sm.wv[t + 1];
            ga[j][0] = w0 * rr[j][0];
            ga[j][1] = w1 * rr[j][1];
            ga[j][2] = w0 * rr[j][2];
            ga[j][3] = w1 * rr[j][3];
        }
#pragma unroll
        for (int i = 0; i < NB; ++i) {
#pragma unroll
            for (int j = 0; j < i; ++j) {
                uint32_t ua[4], bfr[4];
                ua[0] = pack_bf16(ga[2 * j][0], ga[2 * j][1]);
                ua[1] = pack_bf16(ga[2 * j][2], ga[2 * j][3]);
                ua[2] = pack_bf16(ga[2 * j + 1][0], ga[2 * j + 1][1]);
                ua[3] = pack_bf16(ga[2 * j + 1][2], ga[2 * j + 1][3]);
                negate_frag(ua);
                load_b_nk(bfr, sm.mkk, kLdT, 16 * i, 16 * j, lane);
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
#pragma unroll
        for (int i = 0; i < NB; ++i)
#pragma unroll
            for (int j = 0; j <= i; ++j) {
                uint32_t ua[4], bfr[4];
                ua[0] = pack_bf16(ga[2 * j][0], ga[2 * j][1]);
                ua[1] = pack_bf16(ga[2 * j][2], ga[2 * j][3]);
                ua[2] = pack_bf16(ga[2 * j + 1][0], ga[2 * j + 1][1]);
                ua[3] = pack_bf16(ga[2 * j + 1][2], ga[2 * j + 1][3]);
                negate_frag(ua);
                load_b_nk(bfr, sm.akk, kLdT, 16 * i, 16 * j, lane);
                mma_bf16(rr[2 * i], ua, bfr[0], bfr[1]);
                mma_bf16(rr[2 * i + 1], ua, bfr[2], bfr[3]);
            }
        store_frags_t<4>(sm.ub, kLdOp, 16 * warp, ga, lane);   // U^T -> [t][v]
        // ---- dU^T = dO^T Aqk + dS1 Kbar^T
        float du[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) du[j][0] = du[j][1] = du[j][2] = du[j][3] = 0.f;
#pragma unroll
        for (int js = 0; js < NB; ++js)
#pragma unroll
            for (int kt = js; kt < NB; ++kt) {
                uint32_t af[4], bfr[4];
                load_a_t(af, sm.dop, kLdOp, 16 * warp, 16 * kt, lane);
                load_b_kn(bfr, sm.aqk, kLdT, 16 * js, 16 * kt, lane);
                mma_bf16(du[2 * js], af, bfr[0], bfr[1]);
                mma_bf16(du[2 * js + 1], af, bfr[2], bfr[3]);
            }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t af[4];
            af[0] = pack_bf16(ds[2 * ks][0], ds[2 * ks][1]);
            af[1] = pack_bf16(ds[2 * ks][2], ds[2 * ks][3]);
            af[2] = pack_bf16(ds[2 * ks + 1][0], ds[2 * ks + 1][1]);
            af[3] = pack_bf16(ds[2 * ks + 1][2], ds[2 * ks + 1][3]);
#pragma unroll
            for (int js = 0; js < NB; ++js) {
                uint32_t bfr[4];
                load_b_nk(bfr, sm.kcm, kLdOp, 16 * js, 16 * ks, lane);
                const float *f = sm.fm + js * 128 + 16 * ks + 2 * c4;
                bfr[0] = scale_bf16x2(bfr[0], f[0], f[1]);
                bfr[1] = scale_bf16x2(bfr[1], f[8], f[9]);
                bfr[2] = scale_bf16x2(bfr[2], f[0], f[1]);
                bfr[3] = scale_bf16x2(bfr[3], f[8], f[9]);
                mma_bf16(du[2 * js], af, bfr[0], bfr[1]);
                mma_bf16(du[2 * js + 1], af, bfr[2], bfr[3]);
            }
        }
        // ---- dY^T = dU^T M^-1:  dY_j = (dU_j - sum_{i>j} dY_i M_ij) T_jj
#pragma unroll
        for (int j = NB - 1; j >= 0; --j) {
#pragma unroll
            for (int i = j + 1; i < NB; ++i) {
                uint32_t ya[4], bfr[4];
                ya[0] = pack_bf16(du[2 * i][0], du[2 * i][1]);
                ya[1] = pack_bf16(du[2 * i][2], du[2 * i][3]);
                ya[2] = pack_bf16(du[2 * i + 1][0], du[2 * i + 1][1]);
                ya[3] = pack_bf16(du[2 * i + 1][2], du[2 * i + 1][3]);
                negate_frag(ya);
                load_b_kn(bfr, sm.mkk, kLdT, 16 * j, 16 * i, lane);
                mma_bf16(du[2 * j], ya, bfr[0], bfr[1]);
                mma_bf16(du[2 * j + 1], ya, bfr[2], bfr[3]);
            }
            uint32_t za[4], bfr[4];
            za[0] = pack_bf16(du[2 * j][0], du[2 * j][1]);
            za[1] = pack_bf16(du[2 * j][2], du[2 * j][3]);
            za[2] = pack_bf16(du[2 * j + 1][0], du[2 * j + 1][1]);
            za[3] = pack_bf16(du[2 * j + 1][2], du[2 * j + 1][3]);
            load_b_kn(bfr, sm.tii + j * 16 * 24, 24, 0, 0, lane);
            float un[2][4] = {};
            mma_bf16(un[0], za, bfr[0], bfr[1]);
            mma_bf16(un[1], za, bfr[2], bfr[3]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                du[2 * j][e] = un[0][e];
                du[2 * j + 1][e] = un[1][e];
            }
        }
        // ---- dR = Diag(w) dY (-> shared tile, dv), dw partials
        float dr[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = 8 * j + 2 * c4;
            const float w0 = sm.wv[t], w1 = sm.wv[t + 1];
            dr[j][0] = w0 * du[j][0];
            dr[j][1] = w1 * du[j][1];
            dr[j][2] = w0 * du[j][2];
            dr[j][3] = w1 * du[j][3];
            float p0 = du[j][0] * rr[j][0] + du[j][2] * rr[j][2];
            float p1 = du[j][1] * rr[j][1] + du[j][3] * rr[j][3];
#pragma unroll
            for (int off = 4; off <= 16; off <<= 1) {
                p0 += __shfl_xor_sync(0xffffffffu, p0, off);
                p1 += __shfl_xor_sync(0xffffffffu, p1, off);
            }
            if (g == 0) {
                sm.dwp[warp * C + t] = p0;
                sm.dwp[warp * C + t + 1] = p1;
            }
        }
        store_frags_t<4>(sm.drb, kLdOp, 16 * warp, dr, lane);   // dR^T -> [t][v]
        // ---- dS0 = dS1 Diag(gamma) + dO^T Qt - dR^T Kt
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int col = 8 * j + 2 * c4;
            const float g0 = sm.gam[col], g1 = sm.gam[col + 1];
            ds[j][0] *= g0;
            ds[j][1] *= g1;
            ds[j][2] *= g0;
            ds[j][3] *= g1;
        }
#pragma unroll
        for (int kt = 0; kt < NB; ++kt) {
            uint32_t ao[4], ar[4];
            load_a_t(ao, sm.dop, kLdOp, 16 * warp, 16 * kt, lane);
            ar[0] = pack_bf16(dr[2 * kt][0], dr[2 * kt][1]);
            ar[1] = pack_bf16(dr[2 * kt][2], dr[2 * kt][3]);
            ar[2] = pack_bf16(dr[2 * kt + 1][0], dr[2 * kt + 1][1]);
            ar[3] = pack_bf16(dr[2 * kt + 1][2], dr[2 * kt + 1][3]);
            negate_frag(ar);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t bq[4], bk[4];
                load_b_kn_swz(bq, sm.rq, 16 * np, 16 * kt, lane);   // Qt
                load_b_kn_swz(bk, sm.rk, 16 * np, 16 * kt, lane);   // Kt
                mma_bf16(ds[2 * np], ao, bq[0], bq[1]);
                mma_bf16(ds[2 * np + 1], ao, bq[2], bq[3]);
                mma_bf16(ds[2 * np], ar, bk[0], bk[1]);
                mma_bf16(ds[2 * np + 1], ar, bk[2], bk[3]);
            }
        }
        if (cc == 0) {   // dS0 = dP_0 Diag(a_0): where the floor binds at the first token, the exact
                         // recurrence's a_0 (floor_scale); the content term is added after this
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int col = 8 * j + 2 * c4;
                const float f0 = sm.fs0[col], f1 = sm.fs0[col + 1];
                ds[j][0] *= f0;
                ds[j][1] *= f1;
                ds[j][2] *= f0;
                ds[j][3] *= f1;
            }
        }
        __syncthreads();
        if (cc > 0) issue(cc - 1);   // q, k, v, dO and the Qt / Kt tiles of this chunk are read
        // ---- dAqk = dO U^T (s <= t), dAkk = -dR U^T (s < t): reductions over v, six 16x16 tiles
        if (warp < 6) {
            const int type = warp / 3, blk = warp % 3;
            const int i = blk == 0 ? 0 : 1, j = blk == 2 ? 1 : 0;
            float acc[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint32_t af[4], bfr[4];
                load_a(af, type ? sm.drb : sm.dop, kLdOp, 16 * i, 16 * ks, lane);
                load_b_nk(bfr, sm.ub, kLdOp, 16 * j, 16 * ks, lane);
                mma_bf16(acc[0], af, bfr[0], bfr[1]);
                mma_bf16(acc[1], af, bfr[2], bfr[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tr = 16 * i + g + ((e >> 1) << 3);
                    const int sc = 16 * j + 8 * nt + 2 * c4 + (e & 1);
                    if (type == 0) {
                        sm.daqk[tr * kLdT + sc] = __float2bfloat16_rn(sc < tr ? acc[nt][e] : 0.f);
                        if (sc == tr) sm.daqd[tr] = acc[nt][e];
                    }
                    else sm.dakk[tr * kLdT + sc] = __float2bfloat16_rn(sc < tr ? -acc[nt][e] : 0.f);
                }
        }
        __syncthreads();
        // ---- per (token block, channel quarter): Gq, Gkr, Gkc, Gkb -> dq, dk, dLam
        // Paired terms that cancel in the reverse cumulative sum of dLam are built from the same
        // rounded operands on both sides: the off-diagonal decay factor is applied to fp32
        // products, never to one side's bf16 operand.
        {
            const int ib2 = warp >> 2, ch0 = 32 * (warp & 3);
            float gq[4][4], gkr[4][4], gkc[4][4], gkb[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) gq[j][e] = gkr[j][e] = gkc[j][e] = gkb[j][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint32_t ao[4], ar[4], au[4];
                load_a(ao, sm.dop, kLdOp, 16 * ib2, 16 * ks, lane);
                load_a(ar, sm.drb, kLdOp, 16 * ib2, 16 * ks, lane);
                negate_frag(ar);
                load_a(au, sm.ub, kLdOp, 16 * ib2, 16 * ks, lane);
#pragma unroll
                for (int np2 = 0; np2 < 2; ++np2) {
                    const int n0 = ch0 + 16 * np2;
                    uint32_t bs[4], bd[4];
                    load_b_kn_um(bs, sm.s0b, 128, n0, 16 * ks, lane);
                    load_b_kn(bd, sm.ds1b, kLdOp, n0, 16 * ks, lane);
                    mma_bf16(gq[2 * np2], ao, bs[0], bs[1]);
                    mma_bf16(gq[2 * np2 + 1], ao, bs[2], bs[3]);
                    mma_bf16(gkr[2 * np2], ar, bs[0], bs[1]);
                    mma_bf16(gkr[2 * np2 + 1], ar, bs[2], bs[3]);
                    mma_bf16(gkb[2 * np2], au, bd[0], bd[1]);
                    mma_bf16(gkb[2 * np2 + 1], au, bd[2], bd[3]);
                }
            }
            // the decays of S0 (Em) and dS1 (Fm) scale output columns, fixed for this token
            // block: applied to the fp32 sums
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int ch = ch0 + 8 * nt + 2 * c4;
                const float2 e2 = *reinterpret_cast<const float2 *>(sm.em + ib2 * 128 + ch);
                const float2 f2 = *reinterpret_cast<const float2 *>(sm.fm + ib2 * 128 + ch);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float ev = (e & 1) ? e2.y : e2.x, fv = (e & 1) ? f2.y : f2.x;
                    gq[nt][e] *= ev;
                    gkr[nt][e] *= ev;
                    gkb[nt][e] *= fv;
                }
            }
            // Gram blocks: rows t of this block against columns s of block j (row side) and
            // columns s of this block against rows t of block i2 (column side)
#pragma unroll
            for (int j2 = 0; j2 < NB; ++j2) {
                const bool row_side = j2 <= ib2;   // pair (ib2, j2)
                const bool col_side = j2 >= ib2;   // pair (j2, ib2)
                const bool offdiag = j2 != ib2;
                float tq[4][4], tk[4][4], tc[4][4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e) tq[j][e] = tk[j][e] = tc[j][e] = 0.f;
                if (row_side) {
                    uint32_t aq[4], ak[4];
                    load_a(aq, sm.daqk, kLdT, 16 * ib2, 16 * j2, lane);
                    load_a(ak, sm.dakk, kLdT, 16 * ib2, 16 * j2, lane);
#pragma unroll
                    for (int np2 = 0; np2 < 2; ++np2) {
                        uint32_t bc[4];
                        load_b_kn(bc, sm.kcm, kLdOp, ch0 + 16 * np2, 16 * j2, lane);
                        mma_bf16(tq[2 * np2], aq, bc[0], bc[1]);
                        mma_bf16(tq[2 * np2 + 1], aq, bc[2], bc[3]);
                        mma_bf16(tk[2 * np2], ak, bc[0], bc[1]);
                        mma_bf16(tk[2 * np2 + 1], ak, bc[2], bc[3]);
                    }
                }
                if (col_side) {
                    uint32_t aq[4], ak[4];
                    load_a_t(aq, sm.daqk, kLdT, 16 * ib2, 16 * j2, lane);
                    load_a_t(ak, sm.dakk, kLdT, 16 * ib2, 16 * j2, lane);
#pragma unroll
                    for (int np2 = 0; np2 < 2; ++np2) {
                        uint32_t bq[4], bk[4];
                        load_b_kn(bq, sm.qm, kLdOp, ch0 + 16 * np2, 16 * j2, lane);
                        load_b_kn(bk, sm.krm, kLdOp, ch0 + 16 * np2, 16 * j2, lane);
                        mma_bf16(tc[2 * np2], aq, bq[0], bq[1]);
                        mma_bf16(tc[2 * np2 + 1], aq, bq[2], bq[3]);
                        mma_bf16(tc[2 * np2], ak, bk[0], bk[1]);
                        mma_bf16(tc[2 * np2 + 1], ak, bk[2], bk[3]);
                    }
                }
                // the off-diagonal pair's factor e^{Lam_m(i) - Lam_m(j)} (i the later block) is
                // applied in two parts, the one that bounds the operand inside the sum first: r15
                // of block j with kcm, p7 of block i with qm / krm
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = ch0 + 8 * nt + 2 * c4 + (e & 1);
                        if (!offdiag) {
                            gq[nt][e] += tq[nt][e];
                            gkr[nt][e] += tk[nt][e];
                            gkc[nt][e] += tc[nt][e];
                        } else if (row_side) {   // i = ib2, j = j2
                            const float fr = sm.r15[j2 * 128 + c], fp = sm.p7[ib2 * 128 + c];
                            gq[nt][e] += (tq[nt][e] * fr) * fp;
                            gkr[nt][e] += (tk[nt][e] * fr) * fp;
                        } else {                 // i = j2, j = ib2
                            const float fp = sm.p7[j2 * 128 + c], fr = sm.r15[ib2 * 128 + c];
                            gkc[nt][e] += (tc[nt][e] * fp) * fr;
                        }
                    }
            }
            float bsum[4][2];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) bsum[nt][0] = bsum[nt][1] = 0.f;
            const int tlast = nv - 1;   // the chunk's last live token: its Kbar factor is 1
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int t = 16 * ib2 + g + 8 * hh;
                    const int ch = ch0 + 8 * nt + 2 * c4;
                    float dqv[2], dkv[2], dlv[2];
                    const float2 r2 = *reinterpret_cast<const float2 *>(sm.rfac + t * kLdF + ch);
                    const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162 *>(sm.qm + t * kLdOp + ch);
                    const __nv_bfloat162 kr2 = *reinterpret_cast<const __nv_bfloat162 *>(sm.krm + t * kLdOp + ch);
                    const __nv_bfloat162 kc2 = *reinterpret_cast<const __nv_bfloat162 *>(sm.kcm + t * kLdOp + ch);
                    const float dgd = sm.daqd[t];
                    const bool tl = t == tlast;
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const int e = 2 * hh + e2;
                        const float r = e2 ? r2.y : r2.x;
                        const float ri = __fdividef(1.f, r);
                        const float Gq = gq[nt][e], Gkr = gkr[nt][e], Gkc = gkc[nt][e];
                        const float qmv = bf(e2 ? q2.y : q2.x), krv = bf(e2 ? kr2.y : kr2.x);
                        const float kcv = bf(e2 ? kc2.y : kc2.x);
                        dqv[e2] = r * (Gq + dgd * kcv);
                        dkv[e2] = r * Gkr + ri * (Gkc + gkb[nt][e] + dgd * qmv);
                        dlv[e2] = qmv * Gq + krv * Gkr - kcv * (tl ? Gkc : Gkc + gkb[nt][e]);
                        if (!tl) bsum[nt][e2] += kcv * gkb[nt][e];     // Kbar_t dKbar_t
                    }
                    *reinterpret_cast<float2 *>(sm.dlam + t * kLdF + ch) = make_float2(dlv[0], dlv[1]);
                    const size_t gi = base_bh + (size_t)(t0 + t) * tstride + ch;
                    if (!VL || t < nv) {
                        *reinterpret_cast<uint32_t *>(dq + gi) = pack_bf16(dqv[0], dqv[1]);
                        *reinterpret_cast<uint32_t *>(dk + gi) = pack_bf16(dkv[0], dkv[1]);
                    }
                }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    float x = bsum[nt][e2];
#pragma unroll
                    for (int off = 4; off <= 16; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
                    if (g == 0) sm.bpart[ib2 * 128 + ch0 + 8 * nt + 2 * c4 + e2] = x;
                }
        }
        __syncthreads();
        // the S0 tile is read for the last time above unless this chunk closes a gate chunk
        // with the boundary-state readout: the next chunk's state can come in now
        const bool s0_early = !(gate_start && a.mc_mode == 0);
        if (cc > 0 && s0_early) issue_s0(cc - 1);
        if (gate_start && tid == 0) {
            mbar_expect_tx(&sm.bar_ab, 256u * R * 4u);
            bulk_g2s(abuf, a.A + (size_t)h * 128 * R, 128u * R * 4u, &sm.bar_ab);
            bulk_g2s(abuf + 128 * R, a.Bm + (size_t)h * R * 128, 128u * R * 4u, &sm.bar_ab);
        }
        // ---- reverse cumulative sum of dLam within the chunk, gate gradients.  Half-block
        //      totals first (the chunk's last-token term xl joins the last half), then each
        //      thread scans its 8 tokens from the total of everything after them.
        auto last_token_term = [&](int c) {
            float xl = sm.gam[c] * sm.s0ds[c];
#pragma unroll
            for (int i2 = 0; i2 < NB; ++i2) xl += sm.bpart[i2 * 128 + c];
            return xl;
        };
        const int hb = 2 * ib + hf;   // half-block index, 0 .. 2 NB - 1
        {
            float t0s = 0.f, t1s = 0.f;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const float2 d2 = *reinterpret_cast<const float2 *>(&sm.dlam[(16 * ib + 8 * hf + t) * kLdF + c0]);
                t0s += d2.x;
                t1s += d2.y;
            }
            if (hb == 2 * NB - 1) {
                t0s += last_token_term(c0);
                t1s += last_token_term(c0 + 1);
            }
            *reinterpret_cast<float2 *>(&sm.htot[hb * 128 + c0]) = make_float2(t0s, t1s);
        }
        if (tid < C) {   // d w_logit (warp 0: C = 32), and its sum for the write-gate term
            float dw = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) dw += sm.dwp[w * C + tid];
            const float w = sm.wv[tid];
            float x = dw * w * (1.f - w);
            if (!VL || tid < nv) a.dw_logit[((size_t)bb * T + toff + t0 + tid) * H + h] = x;
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
            if (tid == 0) sm.ddw += x;
        }
        __syncthreads();
        {
            float run[2] = {0.f, 0.f};
#pragma unroll
            for (int h2 = 0; h2 < 2 * NB; ++h2)
                if (h2 > hb) {
                    const float2 x = *reinterpret_cast<const float2 *>(&sm.htot[h2 * 128 + c0]);
                    run[0] += x.x;
                    run[1] += x.y;
                }
            const float dl[2] = {sm.delta[c0], sm.delta[c0 + 1]};
            const float xl[2] = {hb == 2 * NB - 1 ? last_token_term(c0) : 0.f,
                                 hb == 2 * NB - 1 ? last_token_term(c0 + 1) : 0.f};
            float pdd[2] = {0.f, 0.f};
#pragma unroll
            for (int t = 7; t >= 0; --t) {
                const int row = 16 * ib + 8 * hf + t;
                const float2 d2 = *reinterpret_cast<const float2 *>(&sm.dlam[row * kLdF + c0]);
                const bool inert = VL && row >= nv;   // passes the running sum on, has no gate gradient
                float dg[2], db[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    run[e] += e ? d2.y : d2.x;
                    if (t == 7) run[e] += xl[e];
                    const float gx = e ? glr[t].y : glr[t].x, nb = -((e ? bxr[t].y : bxr[t].x) + dl[e]);   // nb = -beta
                    const float e2 = __expf(nb);
                    // the unfloored retention and both sigmoids from the reciprocals 1 / (1 + e^x)
                    const float rb = __fdividef(1.f, 1.f + e2), sb = nb > 15.f ? 1.f : e2 * rb;   // sigmoid(-beta)
                    if constexpr (DEC) {   // log g = -amp softplus(x), x = g_logit + tau: d/dx = -amp sigmoid(x)
                        const float x = gx + tb[e], e1 = __expf(x), sp = softplus_fast(x, e1);
                        const float ra = __fdividef(1.f, 1.f + e1);
                        const float dla = run[e] * floor_scale(__expf(-amp * sp) * rb, inert);
                        dg[e] = -amp * (x > 15.f ? 1.f : e1 * ra) * dla;
                        db[e] = sb * dla;
                        dtp[e] += dg[e];
                        dap += dla * (-amp * sp);   // d A_dec = dlog a . log g
                    } else {
                        const float e1 = __expf(gx), ra = __fdividef(1.f, 1.f + e1);
                        const float dla = run[e] * floor_scale(ra * rb, inert);
                        dg[e] = -(gx > 15.f ? 1.f : e1 * ra) * dla;
                        db[e] = sb * dla;
                    }
                    pdd[e] += db[e];
                }
                // staged in this thread's own positions for the vectorised stores below
                *reinterpret_cast<float2 *>(&sm.dlam[row * kLdF + c0]) = make_float2(dg[0], dg[1]);
                *reinterpret_cast<float2 *>(&sm.rfac[row * kLdF + c0]) = make_float2(db[0], db[1]);
            }
            *reinterpret_cast<float2 *>(&sm.pdd[hb * 128 + c0]) = make_float2(pdd[0], pdd[1]);
        }
        if (cc > 0) {   // the gate logits were read for the last time in the scan above
            load_gates(cc - 1);
            load_w(cc - 1);
        }
        fence_proxy_async_smem();   // dg / db (and dR, written earlier) are read by bulk copies next
        __syncthreads();
        if (lane < 4) {   // d g_logit, dbx and dv of token 4 warp + lane: one bulk copy per row
            const int t = 4 * warp + lane;
            if (!VL || t < nv) {
                const size_t gi = base_bh + (size_t)(t0 + t) * tstride;
                bulk_s2g(a.dg_logit + gi, sm.dlam + t * kLdF, 128u * 4u);
                bulk_s2g(a.dbx + gi, sm.rfac + t * kLdF, 128u * 4u);
                bulk_s2g(dv + gi, sm.drb + t * kLdOp, 128u * 2u);
            }
            bulk_commit();
        }
        if (tid < 128) {
            float x = 0.f;
#pragma unroll
            for (int h2 = 0; h2 < 2 * NB; ++h2) x += sm.pdd[h2 * 128 + tid];
            sm.ddelta[tid] += x;
        }
        // ---- content path at the gate chunk's first token (the other chunks need no barrier
        //      here: nothing read below this point is written before the next chunk's first one)
        if (gate_start) {
            __syncthreads();
            const float *As = abuf, *Bs = abuf + 128 * R;
            const bool lost_ab = !mbar_wait(&sm.bar_ab, ab_phase, a.wait_limit);
            if (lane < R) {   // dz = A^T dDelta: lane j, key channels warp + 8 i, partial per warp
                float s2[2] = {0.f, 0.f};
#pragma unroll
                for (int i = 0; i < 16; ++i) s2[i & 1] += As[(warp + 8 * i) * R + lane] * sm.ddelta[warp + 8 * i];
                sm.xp[warp * 32 + lane] = s2[0] + s2[1];
            }
            if (__syncthreads_or(lost_ab)) {   // the factor copy did not arrive: end the sweep; the
                                               // copies that may still be in flight are waited for
                if (tid == 0) {
                    atomicOr(&g_tc_bwd_timeout, 4);
                    mbar_wait(&sm.bar_ab, ab_phase, a.wait_limit);
                    if (cc > 0) {
                        mbar_wait(&sm.bar, phase, a.wait_limit);
                        if (s0_early) mbar_wait(&sm.bar_s0, phase, a.wait_limit);
                    }
                }
                if (lane < 4) bulk_wait<0>();
                return;
            }
            ab_phase ^= 1u;
            if (tid < R) {   // the eight partials (+ Aw d(dw))
                float z = awj * sm.ddw;
#pragma unroll
                for (int w = 0; w < 8; ++w) z += sm.xp[w * 32 + tid];
                sm.dzv[tid] = z;
                wsg[(size_t)gc * kTcGradRec + 128 + tid] = z;
            }
            if (tid < 128) wsg[(size_t)gc * kTcGradRec + tid] = sm.ddelta[tid];
            if (tid == 0) wsg[(size_t)gc * kTcGradRec + kTcGradDw] = sm.ddw;
            __syncthreads();
            {   // dm = B^T dz, two threads per output
                const int vv = tid >> 1, half = tid & 1;
                float sacc = 0.f;
#pragma unroll 8
                for (int j = half; j < R; j += 2) sacc += Bs[j * 128 + vv] * sm.dzv[j];
                sacc += __shfl_xor_sync(0xffffffffu, sacc, 1);
                if (half == 0) sm.dmv[vv] = sacc;
            }
            __syncthreads();
            if (a.mc_mode == 0) {
                // m = S0 qbar:  dS0 += dm qbar^T here;  dq_t += S0^T dm / n for every t of the gate
                // chunk is added by the readout pass after this kernel (vector stored per gate chunk)
                {   // S0^T dm: channel pair 2 cp, 2 cp + 1 over rows 32 rq .. 32 rq + 31
                    const int cpr = tid & 63, rq = tid >> 6;
                    float sa[4][2] = {};
#pragma unroll
                    for (int r = 0; r < 32; r += 8)
#pragma unroll
                        for (int x4 = 0; x4 < 2; ++x4) {
                            const float4 m4 = *reinterpret_cast<const float4 *>(sm.dmv + 32 * rq + r + 4 * x4);
                            const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                            for (int y = 0; y < 4; ++y) {
                                const int x = 4 * x4 + y;
                                const __nv_bfloat162 s2 =
                                    *reinterpret_cast<const __nv_bfloat162 *>(sm.s0b + umma_off(32 * rq + r + x, 2 * cpr, 128));
                                sa[y][0] += bf(s2.x) * mv[y];
                                sa[y][1] += bf(s2.y) * mv[y];
                            }
                        }
                    *reinterpret_cast<float2 *>(sm.pdd + rq * 128 + 2 * cpr) =
                        make_float2((sa[0][0] + sa[1][0]) + (sa[2][0] + sa[3][0]), (sa[0][1] + sa[1][1]) + (sa[2][1] + sa[3][1]));
                }
                __syncthreads();
                if (tid < 128) {
                    wsv[(size_t)gc * 128 + tid] =
                        ((sm.pdd[tid] + sm.pdd[128 + tid]) + (sm.pdd[256 + tid] + sm.pdd[384 + tid])) / (float)n;
                    sm.dox[tid] = 0.f;
                }
                const float m0 = sm.dmv[v0], m1 = sm.dmv[v1];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int col = 8 * j + 2 * c4;
                    const float q0 = sm.qbar[col], q1 = sm.qbar[col + 1];
                    ds[j][0] += m0 * q0;
                    ds[j][1] += m0 * q1;
                    ds[j][2] += m1 * q0;
                    ds[j][3] += m1 * q1;
                }
            } else if (tid < 128) {
                sm.dox[tid] = gc > 0 ? sm.dmv[tid] / (float)L : 0.f;
                if (gc == 0 && a.dm_prev_in) a.dm_prev_in[(size_t)u * 128 + tid] = sm.dmv[tid];
            }
            __syncthreads();
            if (cc > 0 && !s0_early) issue_s0(cc - 1);
        }
    }
    if (lane < 4) bulk_wait<0>();   // the last gradient rows are written before the CTA ends
    if (a.dS0) {
        float *D = a.dS0 + (size_t)u * 128 * 128;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int col = 8 * j + 2 * c4;
            *reinterpret_cast<float2 *>(D + v0 * 128 + col) = make_float2(ds[j][0], ds[j][1]);
            *reinterpret_cast<float2 *>(D + v1 * 128 + col) = make_float2(ds[j][2], ds[j][3]);
        }
    }
    if (a.dm_prev_in && tid < 128) {
        if (VL && NCCn == 0)   // no token: m_prev_out is m_prev_in passed through
            a.dm_prev_in[(size_t)u * 128 + tid] = a.dm_prev_out ? a.dm_prev_out[(size_t)u * 128 + tid] : 0.f;
        else if (a.mc_mode == 0)
            a.dm_prev_in[(size_t)u * 128 + tid] = 0.f;
    }
    if constexpr (DEC) {   // this unit's d tau (the four threads of each channel pair) and d A_dec, fixed order
        float *red = sm.xp;   // free after the sweep: [256][2] channel partials, then [256] amplitude
        *reinterpret_cast<float2 *>(&red[2 * tid]) = make_float2(dtp[0], dtp[1]);
        red[512 + tid] = dap;
        __syncthreads();
        float *dst = a.ws + (size_t)a.B * a.H * NG * (kTcGradRec + 128) + (size_t)u * kTcDecayRec;
        if (tid < 128) {
            const int pr = tid >> 1, e = tid & 1;
            dst[tid] = ((red[2 * pr + e] + red[2 * (pr + 64) + e]) + red[2 * (pr + 128) + e]) + red[2 * (pr + 192) + e];
        }
        if (warp == 0) {
            float x = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) x += red[512 + 8 * lane + j];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
            if (lane == 0) dst[128] = x;
        }
    }
}

// d tau [H,128] and d A_dec [H]: sums over b (fixed order) of the units' decay records
__global__ void reduce_decay_kernel(const float *part, float *dtau, float *dA_dec, int B, int H) {
    const int h = blockIdx.x, i = threadIdx.x;   // 128 threads
    float s = 0.f, s2 = 0.f;
    for (int b = 0; b < B; ++b) {
        const float *r = part + ((size_t)b * H + h) * kTcDecayRec;
        s += r[i];
        if (i == 0) s2 += r[128];
    }
    if (dtau) dtau[(size_t)h * 128 + i] = s;
    if (i == 0 && dA_dec) dA_dec[h] = s2;
}


// dA[h] = sum_{b, gate chunk} dDelta z^T,  dB[h] = sum dz m^T  (z, m from the saved records),
// summed in a fixed order in two passes.  Pass 1, grid (H, slices of kRedSlice records): the
// slice's records are staged kRedRec at a time in shared memory and each thread accumulates R
// of the head's 256 R outputs; the partial sums go to the workspace.  Pass 2 adds the slices
// in order.
constexpr int kRedRec = 32, kRedSlice = 64;
// With packed sequences (cu) the records of gate chunks past a sequence's end hold nothing
// and count as zero.
__global__ void __launch_bounds__(256) reduce_dAdB_partial_kernel(const float *wsg, const float *aux, float *part,
                                                                  int B, int H, int NG, int R, const int *cu,
                                                                  long long total, int T, int L) {
    __shared__ __align__(16) float gd[kRedRec][128], rm[kRedRec][128], gz[kRedRec][kTcMaxRankBwd],
        rz[kRedRec][kTcMaxRankBwd], gw[kRedRec];
    const int h = blockIdx.x, sl = blockIdx.y, tid = threadIdx.x, NR = B * NG;
    const int r0 = sl * kRedSlice, r1 = min(NR, r0 + kRedSlice);
    float accW = 0.f;   // dAw[h][tid] for tid < R
    // each thread: a 4x4 tile of dA (rows k = 4 ka + a, columns j = 4 ja + b) and of dB
    // (rows j = 4 jb + a, columns v = 4 vb + b); the operands of a record are float4 reads
    const int ka = tid >> 3, ja = tid & 7, jb = tid >> 5, vb = tid & 31;
    float accA[4][4] = {}, accB[4][4] = {};
    auto live = [&](int rec) {
        if (!cu) return true;
        int bb, toff, Tn;
        seq_tokens(cu, total, T, rec / NG, bb, toff, Tn, &g_tc_bwd_bad_seqlens);
        return (rec % NG) * L < Tn;
    };
    for (int i0 = r0; i0 < r1; i0 += kRedRec) {
        const int nr = min(kRedRec, r1 - i0);
        for (int idx = tid; idx < nr * 64; idx += 256) {   // dDelta and m, four floats per load
            const int i = idx >> 6, part4 = idx & 63, rec = i0 + i;
            const size_t u = (size_t)(rec / NG) * H + h, gc = rec % NG;
            const bool lv = live(rec);
            if (part4 < 32) {
                *reinterpret_cast<float4 *>(&gd[i][4 * part4]) =
                    lv ? *reinterpret_cast<const float4 *>(wsg + (u * NG + gc) * kTcGradRec + 4 * part4)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
                const float *r = aux + (u * NG + gc) * (kTcAuxFixed + R) + 4 * (part4 - 32);
#pragma unroll
                for (int e = 0; e < 4; ++e) rm[i][4 * (part4 - 32) + e] = lv ? r[e] : 0.f;
            }
        }
        for (int idx = tid; idx < nr * kTcMaxRankBwd; idx += 256) {   // dz and z (zero beyond R)
            const int i = idx / kTcMaxRankBwd, j = idx % kTcMaxRankBwd, rec = i0 + i;
            const size_t u = (size_t)(rec / NG) * H + h, gc = rec % NG;
            const bool lv = live(rec);
            gz[i][j] = (lv && j < R) ? wsg[(u * NG + gc) * kTcGradRec + 128 + j] : 0.f;
            rz[i][j] = (lv && j < R) ? aux[(u * NG + gc) * (kTcAuxFixed + R) + 128 + j] : 0.f;
            if (j == 0) gw[i] = lv ? wsg[(u * NG + gc) * kTcGradRec + kTcGradDw] : 0.f;
        }
        __syncthreads();
        if (tid < R)
            for (int i = 0; i < nr; ++i) accW += gw[i] * rz[i][tid];
        for (int i = 0; i < nr; ++i) {
            const float4 g4 = *reinterpret_cast<const float4 *>(&gd[i][4 * ka]);
            const float4 z4 = *reinterpret_cast<const float4 *>(&rz[i][4 * ja]);
            const float4 y4 = *reinterpret_cast<const float4 *>(&gz[i][4 * jb]);
            const float4 m4 = *reinterpret_cast<const float4 *>(&rm[i][4 * vb]);
            const float ga[4] = {g4.x, g4.y, g4.z, g4.w}, za[4] = {z4.x, z4.y, z4.z, z4.w};
            const float ya[4] = {y4.x, y4.y, y4.z, y4.w}, ma[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    accA[x][y] += ga[x] * za[y];
                    accB[x][y] += ya[x] * ma[y];
                }
        }
        __syncthreads();
    }
    // partial sums in output order: dA (k, j) at k R + j, dB (j, v) at 128 R + 128 j + v, then
    // dAw (j) at 256 R + j
    float *dst = part + ((size_t)sl * H + h) * 257 * R;
    if (tid < R) dst[256 * R + tid] = accW;
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int k = 4 * ka + x, j = 4 * ja + y;
            if (j < R) dst[k * R + j] = accA[x][y];
            const int j2 = 4 * jb + x, v = 4 * vb + y;
            if (j2 < R) dst[128 * R + 128 * j2 + v] = accB[x][y];
        }
}

__global__ void __launch_bounds__(256) reduce_dAdB_final_kernel(const float *part, float *dA, float *dB,
                                                                float *dAw, int H, int R, int S) {
    const int idx = blockIdx.x * 256 + threadIdx.x;
    if (idx >= H * 257 * R) return;
    const int h = idx / (257 * R), o = idx % (257 * R);
    float acc = 0.f;
    for (int sl = 0; sl < S; ++sl) acc += part[((size_t)sl * H + h) * 257 * R + o];
    if (o < 128 * R) dA[(size_t)h * 128 * R + o] = acc;
    else if (o < 256 * R) dB[(size_t)h * R * 128 + (o - 128 * R)] = acc;
    else if (dAw) dAw[(size_t)h * R + (o - 256 * R)] = acc;
}

// Record slices of the dA / dB reduction (B * NG records per head, kRedSlice per slice).
int tc_reduce_slices(int B, int NG) { return (B * NG + kRedSlice - 1) / kRedSlice; }

// dq_t += vec[unit][gate chunk of t] (the content-readout term of the default readout), 8
// channels per thread
__global__ void dq_readout_kernel(__nv_bfloat16 *dq, const float *vec, int H, int T, int L, size_t rows) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows * 16) return;
    const size_t row = i >> 4;                  // (b, t, h)
    const int part = (int)(i & 15), h = (int)(row % H);
    const size_t bt = row / H;
    const int t = (int)(bt % T), b = (int)(bt / T);
    const int NG = (T + L - 1) / L;
    const float *vk = vec + (((size_t)b * H + h) * NG + t / L) * 128 + part * 8;
    uint4 *p = reinterpret_cast<uint4 *>(dq + row * 128 + part * 8);
    uint4 x = *p;
    __nv_bfloat162 *xv = reinterpret_cast<__nv_bfloat162 *>(&x);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(xv[e]);
        xv[e] = __floats2bfloat162_rn(f.x + vk[2 * e], f.y + vk[2 * e + 1]);
    }
    *p = x;
}

// The same for packed sequences: one block per (unit, gate chunk), over the chunk's rows
__global__ void dq_readout_varlen_kernel(__nv_bfloat16 *dq, const float *vec, int H, int T, int L, const int *cu,
                                         long long total) {
    const int NG = (T + L - 1) / L, u = blockIdx.x / NG, gc = blockIdx.x % NG, h = u % H;
    int bb, toff, Tn;
    seq_tokens(cu, total, T, u / H, bb, toff, Tn, &g_tc_bwd_bad_seqlens);
    const int t0 = gc * L, t1 = min(Tn, t0 + L);
    const float *vk = vec + ((size_t)u * NG + gc) * 128;
    for (int i = threadIdx.x; i < (t1 - t0) * 16; i += blockDim.x) {
        const int t = t0 + (i >> 4), part = i & 15;
        uint4 *p = reinterpret_cast<uint4 *>(dq + ((size_t)(toff + t) * H + h) * 128 + part * 8);
        uint4 x = *p;
        __nv_bfloat162 *xv = reinterpret_cast<__nv_bfloat162 *>(&x);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(xv[e]);
            xv[e] = __floats2bfloat162_rn(f.x + vk[part * 8 + 2 * e], f.y + vk[part * 8 + 2 * e + 1]);
        }
        *p = x;
    }
}

cudaError_t launch_bwd_tc(const BwdArgs &a, float *dA, float *dB, cudaStream_t st) {
    const int bytes = (int)sizeof(TcBwdSmem);
    const bool dec = a.A_dec || a.tau, vl = a.cu_seqlens != nullptr;
    auto kern = vl ? (dec ? tc_bwd_kernel<true, true> : tc_bwd_kernel<false, true>)
                   : (dec ? tc_bwd_kernel<true, false> : tc_bwd_kernel<false, false>);
    cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), bytes);
    if (e != cudaSuccess) return e;
    // token rows: B T, or the packed row count (at least 1 for a valid map)
    const long long rows = vl ? (a.total > 0 ? a.total : 1) : (long long)a.B * a.T;
    BwdMaps maps;
    if ((e = make_token_tile_map(&maps.q, a.q, 2, 128, a.H, rows, kBC)) != cudaSuccess) return e;
    if ((e = make_token_tile_map(&maps.k, a.k, 2, 128, a.H, rows, kBC)) != cudaSuccess) return e;
    if ((e = make_token_tile_map(&maps.v, a.v, 2, 128, a.H, rows, kBC)) != cudaSuccess) return e;
    if ((e = make_token_tile_map(&maps.dO, a.dO, 2, 128, a.H, rows, kBC)) != cudaSuccess) return e;
    kern<<<a.B * a.H, 256, bytes, st>>>(a, maps);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (a.mc_mode == 0) {
        const size_t rows = (size_t)a.B * a.T * a.H;
        const float *vec = a.ws + (size_t)a.B * a.H * ((a.T + a.L - 1) / a.L) * kTcGradRec;
        if (vl)
            dq_readout_varlen_kernel<<<a.B * a.H * ((a.T + a.L - 1) / a.L), 256, 0, st>>>(
                static_cast<__nv_bfloat16 *>(a.dq), vec, a.H, a.T, a.L, a.cu_seqlens, a.total);
        else
            dq_readout_kernel<<<(unsigned)((rows * 16 + 255) / 256), 256, 0, st>>>(
                static_cast<__nv_bfloat16 *>(a.dq), vec, a.H, a.T, a.L, rows);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const int NG = (a.T + a.L - 1) / a.L, S = tc_reduce_slices(a.B, NG);
    const float *dec_part = a.ws + (size_t)a.B * a.H * NG * (kTcGradRec + 128);
    float *part = const_cast<float *>(dec_part) + (size_t)a.B * a.H * kTcDecayRec;
    if (dec) {
        reduce_decay_kernel<<<a.H, 128, 0, st>>>(dec_part, a.dtau, a.dA_dec, a.B, a.H);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    reduce_dAdB_partial_kernel<<<dim3(a.H, S), 256, 0, st>>>(a.ws, a.saved_aux, part, a.B, a.H, NG, a.R,
                                                              a.cu_seqlens, a.total, a.T, a.L);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    reduce_dAdB_final_kernel<<<(a.H * 257 * a.R + 255) / 256, 256, 0, st>>>(part, dA, dB, a.dAw, a.H, a.R, S);
    return cudaGetLastError();
}

size_t tc_bwd_smem() { return sizeof(TcBwdSmem); }

// Device status word of the packed-sequence offsets (this file): returns and clears it.
int tc_bwd_take_bad_seqlens() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_bwd_bad_seqlens, sizeof(int)) != cudaSuccess) return 0;
    if (v) {
        const int z = 0;
        cudaMemcpyToSymbol(g_tc_bwd_bad_seqlens, &z, sizeof(int));
    }
    return v;
}

// Device status word of this file: returns and clears it.
int tc_bwd_take_timeout() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_bwd_timeout, sizeof(int)) != cudaSuccess) return 0;
    if (v) {
        const int z = 0;
        cudaMemcpyToSymbol(g_tc_bwd_timeout, &z, sizeof(int));
    }
    return v;
}

}  // namespace carve

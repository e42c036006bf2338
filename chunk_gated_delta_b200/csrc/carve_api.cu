// Host side of the C ABI declared in include/carve.h: argument validation, buffer sizing and
// kernel dispatch.  Nothing here allocates, frees or synchronises.
#include <cuda_runtime.h>

#include <atomic>

#include "../../include/carve.h"
#include "carve_device.cuh"

namespace carve {
cudaError_t launch_fwd_simt(int K, int V, bool bf16, const FwdArgs &a, cudaStream_t st);
cudaError_t launch_fwd_tc(const FwdArgs &a, int C, cudaStream_t st);
cudaError_t launch_bwd_tc(const BwdArgs &a, float *dA, float *dB, cudaStream_t st);
int tc_compute_chunk(int L);
int tc_reduce_slices(int B, int NG);
int tc_fwd_take_timeout();
int tc_bwd_take_timeout();
int step_take_timeout();
int simt_take_bad_seqlens();
int tc_fwd_take_bad_seqlens();
int tc_bwd_take_bad_seqlens();
cudaError_t launch_selftest_timeout(uint32_t iterations, cudaStream_t st);
cudaError_t launch_bwd_simt(int K, int V, bool bf16, const BwdArgs &a, float *dA, float *dB, cudaStream_t st);
cudaError_t launch_fwd_exact(int K, int V, bool bf16, const FwdArgs &a, cudaStream_t st);
cudaError_t launch_bwd_exact(int K, int V, bool bf16, const BwdArgs &a, float *dA, float *dB, cudaStream_t st);
int exact_segment();
cudaError_t launch_step(int K, int V, bool bf16, const void *q, const void *k, const void *v,
                        const float *g_logit, const float *bx, const float *w_logit, const float *A,
                        const float *Bm, const float *Aw, const float *A_dec, const float *tau, float *S,
                        float *mstate, int *pos, void *o, int B, int H, int R, int L, int mc_mode, cudaStream_t st);
}  // namespace carve

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void *p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void *p) { return p == nullptr || aligned16(p); }

// shape checks shared by every entry point; `seq` adds the sequence-length rules
carve_status check_dims(const carve_dims *d, bool seq) {
    if (!d) return CARVE_ERR_INVALID_ARG;
    if (d->B < 1 || d->H < 1 || d->dk < 1 || d->dv < 1 || d->rank < 1 || d->chunk < 1)
        return CARVE_ERR_INVALID_ARG;
    if (d->io != CARVE_IO_FP32 && d->io != CARVE_IO_BF16) return CARVE_ERR_INVALID_ARG;
    if (d->mc_mode != CARVE_MC_BOUNDARY_STATE && d->mc_mode != CARVE_MC_PREV_MEAN_O) return CARVE_ERR_INVALID_ARG;
    if ((d->dk != 64 && d->dk != 128) || (d->dv != 64 && d->dv != 128)) return CARVE_ERR_UNSUPPORTED;
    if (d->rank > 64) return CARVE_ERR_UNSUPPORTED;
    if ((long long)d->B * d->H > (1LL << 30)) return CARVE_ERR_UNSUPPORTED;
    if (seq) {
        if (d->T < 1) return CARVE_ERR_INVALID_ARG;
        if (d->chunk != 1 && d->chunk != 16 && d->chunk != 32 && d->chunk != 64 && d->chunk != 128)
            return CARVE_ERR_UNSUPPORTED;
        if (d->chunk == 1 && d->mc_mode != CARVE_MC_BOUNDARY_STATE) return CARVE_ERR_UNSUPPORTED;
        if (d->T % carve::kSub != 0) return CARVE_ERR_UNSUPPORTED;
        if ((long long)d->B * d->T * d->H * (d->dk > d->dv ? d->dk : d->dv) > (1LL << 40)) return CARVE_ERR_UNSUPPORTED;
        if ((long long)d->B * d->T > 0x7fffffffLL) return CARVE_ERR_UNSUPPORTED;   // token rows index as int
    }
    return CARVE_OK;
}

// packed sequences: `total` rows of [1, total, H, *] token tensors
carve_status check_packed(const carve_dims *d, long long total) {
    if (total < 0 || total > 0x7fffffffLL) return CARVE_ERR_INVALID_ARG;
    if (total * d->H * (d->dk > d->dv ? d->dk : d->dv) > (1LL << 40)) return CARVE_ERR_UNSUPPORTED;
    return CARVE_OK;
}

// Test hook of carve_selftest_stall: polls of the next tensor-core call's barrier waits, 0 when
// unarmed.  Taken (and cleared) by the first carve_fwd / carve_bwd that launches a tensor-core
// sweep.
std::atomic<uint32_t> g_stall_polls{0};

template <class Args>
void set_wait(Args &a, bool tensor_core) {
    const uint32_t p = tensor_core ? g_stall_polls.exchange(0) : 0u;
    a.stall = p != 0;
    a.wait_limit = p ? p : carve::kWaitLimit;
}

size_t n_chunks(const carve_dims *d) { return (size_t)((d->T + d->chunk - 1) / d->chunk); }

// The tensor-core kernels cover bf16 I/O with dk = dv = 128, rank <= 32 and gate chunks of 32,
// 64 or 128 tokens; everything else runs the SIMT kernels.  The forward alone uses compute
// chunks of min(chunk, 64) tokens (32 when T is not a multiple of that); a forward that saves
// for the backward, and the backward, use 32-token compute chunks (T a multiple of 32).
// chunk = 1: the exact content-aware recurrence (token-sequential kernels)
bool exact(const carve_dims *d) { return d->chunk == 1; }
size_t exact_segments(const carve_dims *d) {
    return (size_t)((d->T + carve::exact_segment() - 1) / carve::exact_segment());
}

bool tc_shape(const carve_dims *d) {
    return d->chunk > 1 && d->io == CARVE_IO_BF16 && d->dk == 128 && d->dv == 128 && d->rank <= 32 &&
           carve::tc_compute_chunk(d->chunk) > 0;
}

int tc_fwd_chunk(const carve_dims *d) {
    if (!tc_shape(d)) return 0;
    const int C = carve::tc_compute_chunk(d->chunk);
    if (d->T % C == 0) return C;
    return d->T % 32 == 0 ? 32 : 0;
}

bool use_tc_bwd(const carve_dims *d) { return tc_shape(d) && d->T % 32 == 0; }

// Bytes of the boundary states at the head of the `saved` buffer: fp32 states every 16 tokens
// for the SIMT kernels; bf16 states every 32 tokens (128 rows of 256 bytes) for the tensor-core
// kernels.  The per-chunk content signals (fp32) follow.
size_t saved_states_bytes(const carve_dims *d) {
    const size_t units = (size_t)d->B * d->H;
    if (use_tc_bwd(d)) return units * (size_t)(d->T / 32) * 128 * 128 * 2;
    return units * (size_t)(d->T / carve::kSub) * d->dv * d->dk * sizeof(float);
}

}  // namespace

extern "C" {

const char *carve_status_string(carve_status s) {
    switch (s) {
        case CARVE_OK: return "CARVE_OK";
        case CARVE_ERR_INVALID_ARG: return "CARVE_ERR_INVALID_ARG";
        case CARVE_ERR_UNSUPPORTED: return "CARVE_ERR_UNSUPPORTED";
        case CARVE_ERR_CUDA: return "CARVE_ERR_CUDA";
        case CARVE_ERR_TIMEOUT: return "CARVE_ERR_TIMEOUT";
    }
    return "CARVE_ERR_UNKNOWN";
}

size_t carve_saved_bytes(const carve_dims *d) {
    if (check_dims(d, true) != CARVE_OK) return 0;
    const size_t units = (size_t)d->B * d->H;
    if (exact(d))   // the fp32 state every exact_segment() tokens
        return sizeof(float) * units * exact_segments(d) * d->dv * d->dk;
    const size_t rec = use_tc_bwd(d) ? (size_t)(carve::kTcAuxFixed + d->rank) : (size_t)(d->dv + d->rank + d->dk);
    return saved_states_bytes(d) + sizeof(float) * units * n_chunks(d) * rec;
}

size_t carve_bwd_workspace_bytes(const carve_dims *d) {
    if (check_dims(d, true) != CARVE_OK) return 0;
    const size_t units = (size_t)d->B * d->H;
    const size_t unit_rec = (size_t)d->dk * d->rank + (size_t)d->rank * d->dv + d->rank + (size_t)d->dk + 1;
    if (exact(d))   // per unit: the partial-sum record, then the states of one segment
        return sizeof(float) * units * (unit_rec + (size_t)carve::exact_segment() * d->dv * d->dk);
    if (use_tc_bwd(d))   // per gate chunk: the gradient record and the readout vector of dq;
                         // then the per-slice partial sums of dA, dB and dAw; then per unit the
                         // decay parameters' partial sums
        return sizeof(float) * (units * n_chunks(d) * (carve::kTcGradRec + (size_t)d->dk) +
                                (size_t)carve::tc_reduce_slices(d->B, (int)n_chunks(d)) * d->H * 257 * d->rank +
                                units * carve::kTcDecayRec);
    // per unit: dA, dB, dAw, dtau and dA_dec partial sums
    return sizeof(float) * units * unit_rec;
}

// cu == nullptr: [B,T,H,*] batches; else B sequences packed in `total` rows (see carve_fwd_varlen)
static carve_status fwd_impl(const carve_dims *d, const int32_t *cu, long long total, const void *q, const void *k,
                             const void *v, const float *g_logit, const float *bx, const float *w_logit,
                             const float *A, const float *Bm, const float *Aw, const float *A_dec, const float *tau,
                             const float *S0, const float *m_prev_in, void *o, float *S_final, float *m_prev_out,
                             void *saved, void *stream) {
    carve_status st = check_dims(d, true);
    if (st != CARVE_OK) return st;
    if (cu && (st = check_packed(d, total)) != CARVE_OK) return st;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(g_logit) || !ok_ptr(bx) || !ok_ptr(w_logit) ||
        !ok_ptr(A) || !ok_ptr(Bm) || !ok_opt(Aw) || !ok_opt(A_dec) || !ok_opt(tau) || !ok_ptr(o) ||
        !ok_opt(S0) || !ok_opt(m_prev_in) || !ok_opt(S_final) || !ok_opt(m_prev_out) || !ok_opt(saved))
        return CARVE_ERR_INVALID_ARG;
    carve::FwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.g_logit = g_logit; a.bx = bx; a.w_logit = w_logit; a.A = A; a.Bm = Bm;
    a.Aw = Aw; a.A_dec = A_dec; a.tau = tau; a.S0 = S0; a.m_prev_in = m_prev_in; a.o = o; a.S_final = S_final; a.m_prev_out = m_prev_out;
    const bool tc_saved = use_tc_bwd(d);
    if (saved) {
        a.saved_states = static_cast<float *>(saved);
        a.saved_aux = reinterpret_cast<float *>(static_cast<char *>(saved) + saved_states_bytes(d));
    }
    a.B = d->B; a.H = d->H; a.T = d->T; a.R = d->rank; a.L = d->chunk; a.mc_mode = d->mc_mode;
    a.cu_seqlens = cu; a.total = total;
    cudaError_t e;
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (exact(d)) {
        if (cu) return CARVE_ERR_UNSUPPORTED;   // packed sequences: chunked kernels only
        e = carve::launch_fwd_exact(d->dk, d->dv, d->io == CARVE_IO_BF16, a, cs);
    } else if (saved != nullptr && tc_saved) {
        set_wait(a, true);
        e = carve::launch_fwd_tc(a, 32, cs);
    } else if (saved == nullptr && tc_fwd_chunk(d) > 0) {
        set_wait(a, true);
        e = carve::launch_fwd_tc(a, tc_fwd_chunk(d), cs);
    } else
        e = carve::launch_fwd_simt(d->dk, d->dv, d->io == CARVE_IO_BF16, a, cs);
    return e == cudaSuccess ? CARVE_OK : CARVE_ERR_CUDA;
}

static carve_status bwd_impl(const carve_dims *d, const int32_t *cu, long long total, const void *q, const void *k,
                             const void *v, const float *g_logit, const float *bx, const float *w_logit,
                             const float *A, const float *Bm, const float *Aw, const float *A_dec, const float *tau,
                             const float *S0, const float *m_prev_in, const void *saved, const void *dO,
                             const float *dS_final, const float *dm_prev_out, void *dq, void *dk, void *dv,
                             float *dg_logit, float *dbx, float *dw_logit, float *dA, float *dB, float *dAw,
                             float *dA_dec, float *dtau, float *dS0, float *dm_prev_in, void *workspace,
                             void *stream) {
    carve_status st = check_dims(d, true);
    if (st != CARVE_OK) return st;
    if (cu && (st = check_packed(d, total)) != CARVE_OK) return st;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(g_logit) || !ok_ptr(bx) || !ok_ptr(w_logit) ||
        !ok_ptr(A) || !ok_ptr(Bm) || !ok_opt(S0) || !ok_opt(m_prev_in) || !ok_ptr(saved) || !ok_ptr(dO) ||
        !ok_opt(dS_final) || !ok_opt(dm_prev_out) || !ok_ptr(dq) || !ok_ptr(dk) || !ok_ptr(dv) ||
        !ok_ptr(dg_logit) || !ok_ptr(dbx) || !ok_ptr(dw_logit) || !ok_ptr(dA) || !ok_ptr(dB) || !ok_opt(dS0) ||
        !ok_opt(dm_prev_in) || !ok_ptr(workspace) || !ok_opt(Aw) || (Aw ? !ok_ptr(dAw) : dAw != nullptr) ||
        !ok_opt(A_dec) || (A_dec ? !ok_ptr(dA_dec) : dA_dec != nullptr) || !ok_opt(tau) ||
        (tau ? !ok_ptr(dtau) : dtau != nullptr))
        return CARVE_ERR_INVALID_ARG;
    (void)S0;
    (void)m_prev_in;  // their effect is captured by the saved states and content signals
    carve::BwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.g_logit = g_logit; a.bx = bx; a.w_logit = w_logit; a.A = A; a.Bm = Bm;
    a.Aw = Aw; a.dAw = dAw; a.A_dec = A_dec; a.tau = tau; a.dA_dec = dA_dec; a.dtau = dtau;
    const bool tc = use_tc_bwd(d);
    a.saved_states = static_cast<const float *>(saved);
    a.saved_aux = reinterpret_cast<const float *>(static_cast<const char *>(saved) + saved_states_bytes(d));
    a.dO = dO; a.dS_final = dS_final; a.dm_prev_out = dm_prev_out;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dg_logit = dg_logit; a.dbx = dbx; a.dw_logit = dw_logit;
    a.dS0 = dS0; a.dm_prev_in = dm_prev_in; a.ws = static_cast<float *>(workspace);
    a.B = d->B; a.H = d->H; a.T = d->T; a.R = d->rank; a.L = d->chunk; a.mc_mode = d->mc_mode;
    a.cu_seqlens = cu; a.total = total;
    if (exact(d)) {
        if (cu) return CARVE_ERR_UNSUPPORTED;
        const cudaError_t ex = carve::launch_bwd_exact(d->dk, d->dv, d->io == CARVE_IO_BF16, a, dA, dB,
                                                       static_cast<cudaStream_t>(stream));
        return ex == cudaSuccess ? CARVE_OK : CARVE_ERR_CUDA;
    }
    set_wait(a, tc);
    cudaError_t e = tc ? carve::launch_bwd_tc(a, dA, dB, static_cast<cudaStream_t>(stream))
                       : carve::launch_bwd_simt(d->dk, d->dv, d->io == CARVE_IO_BF16, a, dA, dB,
                                                static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CARVE_OK : CARVE_ERR_CUDA;
}

carve_status carve_fwd(const carve_dims *d, const void *q, const void *k, const void *v,
                       const float *g_logit, const float *bx, const float *w_logit,
                       const float *A, const float *Bm, const float *Aw, const float *A_dec,
                       const float *tau, const float *S0, const float *m_prev_in, void *o,
                       float *S_final, float *m_prev_out, void *saved, void *stream) {
    return fwd_impl(d, nullptr, 0, q, k, v, g_logit, bx, w_logit, A, Bm, Aw, A_dec, tau, S0, m_prev_in, o, S_final,
                    m_prev_out, saved, stream);
}

carve_status carve_fwd_varlen(const carve_dims *d, const int32_t *cu_seqlens, int64_t total_tokens,
                              const void *q, const void *k, const void *v, const float *g_logit,
                              const float *bx, const float *w_logit, const float *A, const float *Bm,
                              const float *Aw, const float *A_dec, const float *tau, const float *S0,
                              const float *m_prev_in, void *o, float *S_final, float *m_prev_out,
                              void *saved, void *stream) {
    if (!ok_ptr(cu_seqlens)) return CARVE_ERR_INVALID_ARG;
    return fwd_impl(d, cu_seqlens, total_tokens, q, k, v, g_logit, bx, w_logit, A, Bm, Aw, A_dec, tau, S0,
                    m_prev_in, o, S_final, m_prev_out, saved, stream);
}

carve_status carve_bwd(const carve_dims *d, const void *q, const void *k, const void *v,
                       const float *g_logit, const float *bx, const float *w_logit,
                       const float *A, const float *Bm, const float *Aw, const float *A_dec,
                       const float *tau, const float *S0, const float *m_prev_in, const void *saved,
                       const void *dO, const float *dS_final, const float *dm_prev_out, void *dq,
                       void *dk, void *dv, float *dg_logit, float *dbx, float *dw_logit, float *dA,
                       float *dB, float *dAw, float *dA_dec, float *dtau, float *dS0,
                       float *dm_prev_in, void *workspace, void *stream) {
    return bwd_impl(d, nullptr, 0, q, k, v, g_logit, bx, w_logit, A, Bm, Aw, A_dec, tau, S0, m_prev_in, saved, dO,
                    dS_final, dm_prev_out, dq, dk, dv, dg_logit, dbx, dw_logit, dA, dB, dAw, dA_dec, dtau, dS0,
                    dm_prev_in, workspace, stream);
}

carve_status carve_bwd_varlen(const carve_dims *d, const int32_t *cu_seqlens, int64_t total_tokens,
                              const void *q, const void *k, const void *v, const float *g_logit,
                              const float *bx, const float *w_logit, const float *A, const float *Bm,
                              const float *Aw, const float *A_dec, const float *tau, const float *S0,
                              const float *m_prev_in, const void *saved, const void *dO,
                              const float *dS_final, const float *dm_prev_out, void *dq, void *dk,
                              void *dv, float *dg_logit, float *dbx, float *dw_logit, float *dA,
                              float *dB, float *dAw, float *dA_dec, float *dtau, float *dS0,
                              float *dm_prev_in, void *workspace, void *stream) {
    if (!ok_ptr(cu_seqlens)) return CARVE_ERR_INVALID_ARG;
    return bwd_impl(d, cu_seqlens, total_tokens, q, k, v, g_logit, bx, w_logit, A, Bm, Aw, A_dec, tau, S0,
                    m_prev_in, saved, dO, dS_final, dm_prev_out, dq, dk, dv, dg_logit, dbx, dw_logit, dA, dB, dAw,
                    dA_dec, dtau, dS0, dm_prev_in, workspace, stream);
}

carve_status carve_step(const carve_dims *d, const void *q, const void *k, const void *v,
                        const float *g_logit, const float *bx, const float *w_logit,
                        const float *A, const float *Bm, const float *Aw, const float *A_dec,
                        const float *tau, float *S, float *mstate, int32_t *pos, void *o, void *stream) {
    carve_status st = check_dims(d, false);
    if (st != CARVE_OK) return st;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(g_logit) || !ok_ptr(bx) || !ok_ptr(w_logit) ||
        !ok_ptr(A) || !ok_ptr(Bm) || !ok_opt(Aw) || !ok_opt(A_dec) || !ok_opt(tau) || !ok_ptr(S) || !ok_ptr(o))
        return CARVE_ERR_INVALID_ARG;
    if (d->mc_mode == CARVE_MC_PREV_MEAN_O && (!ok_ptr(mstate) || !ok_ptr(pos))) return CARVE_ERR_INVALID_ARG;
    cudaError_t e = carve::launch_step(d->dk, d->dv, d->io == CARVE_IO_BF16, q, k, v, g_logit, bx, w_logit, A, Bm, Aw,
                                       A_dec, tau, S, mstate, pos, o, d->B, d->H, d->rank, d->chunk,
                                       d->mc_mode, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CARVE_OK : CARVE_ERR_CUDA;
}

carve_status carve_check(void *stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return CARVE_ERR_CUDA;
    const int t = carve::tc_fwd_take_timeout() | carve::tc_bwd_take_timeout() | carve::step_take_timeout();
    const int bad = carve::simt_take_bad_seqlens() | carve::tc_fwd_take_bad_seqlens() | carve::tc_bwd_take_bad_seqlens();
    return t ? CARVE_ERR_TIMEOUT : bad ? CARVE_ERR_INVALID_ARG : CARVE_OK;
}

carve_status carve_selftest_stall(uint32_t iterations) {
    if (iterations < 1 || iterations > 1000000) return CARVE_ERR_INVALID_ARG;
    g_stall_polls.store(iterations);
    return CARVE_OK;
}

carve_status carve_selftest_timeout(uint32_t iterations, void *stream) {
    if (iterations < 1 || iterations > 1000000) return CARVE_ERR_INVALID_ARG;
    return carve::launch_selftest_timeout(iterations, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? CARVE_OK
               : CARVE_ERR_CUDA;
}

}  // extern "C"

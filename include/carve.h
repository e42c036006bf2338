/*
 * carve.h -- C ABI of the B200 (sm_100a) CARVE recurrence library (libcarve.so).
 *
 * CARVE ("Content-Aware Recurrent with Value Efficiency for Chunk-Parallel Linear
 * Attention") keeps, per batch element b and head h, a state S in R^{dv x dk} and updates it
 * token by token with a key-axis gated delta rule (CARVE blog, liuzhao09.github.io,
 * section 2.1; gist.science technical summary, section 2):
 *
 *   for each chunk c of `chunk` tokens:
 *     m_c   = S_[c-1] . mean_{t in c} q_t            (mc_mode 0, chunk-boundary state readout,
 *                                                     paperdance abstract)
 *           | mean_{t in c-1} o_t                     (mc_mode 1, previous-chunk mean output,
 *                                                     CARVE blog section 2.2)
 *     z_c   = Bm m_c ;  Delta = A z_c                 (U_b = A.Bm, zero-initialisable low rank)
 *     dw_c  = Aw . z_c                                (optional, Aw may be NULL: the same projection
 *                                                     of m_c also biases the write gate, CARVE
 *                                                     blog section 2.2, Figure 1)
 *     for t in c:
 *       a_t = exp(-e^{A_dec} softplus(g_logit_t + tau)) * sigmoid(bx_t + Delta)   (key axis, length dk;
 *             A_dec, the head's log-decay amplitude, and tau, the per-channel bias, are optional
 *             (0 when NULL): the fused decay of CARVE blog section 2.3)
 *       w_t = sigmoid(w_logit_t + dw_c)                               (one scalar per head)
 *       S_t = S_{t-1} Diag(a_t) + w_t (v_t - S_{t-1} Diag(a_t) k_t) k_t^T
 *       o_t = S_t q_t
 *
 * The library evaluates this chunk-parallel in WY form on the GPU (one triangular solve per
 * chunk shared by all value channels; CARVE blog section 2.3).  Every entry point is
 * stream-ordered on the caller's stream, allocates nothing and frees nothing.  None
 * synchronises the device, with two exceptions: carve_check waits for its stream (that is
 * its purpose) and then reads and clears the device status words with synchronous copies,
 * and the first carve_bwd_noalloc call on each device looks up its scratch array's device
 * address (which may load the module).  The first tensor-core launch of each kernel on a
 * device also raises its shared-memory limit (a kernel attribute, no synchronisation).  All
 * pointers are DEVICE pointers unless stated otherwise; the caller owns every buffer.
 * Arguments are validated on the host before any launch; a rejected call launches nothing
 * and returns a non-zero status.  Apart from carve_bwd_noalloc (which shares one scratch
 * array) and the test hook carve_selftest_stall (a one-shot flag), no entry point keeps
 * mutable global state, so concurrent calls on different streams with disjoint buffers are
 * safe.
 *
 * Tensor layouts (contiguous, row-major; "io" = CARVE_IO_FP32 -> float, CARVE_IO_BF16 ->
 * bfloat16 stored as 16-bit words):
 *   q, k           [B, T, H, dk]  io        v, o           [B, T, H, dv]  io
 *   g_logit, bx    [B, T, H, dk]  float     w_logit        [B, T, H]      float
 *   A              [H, dk, rank]  float     Bm             [H, rank, dv]  float
 *   Aw             [H, rank]      float (nullable: no content term on the write gate)
 *   A_dec          [H]            float (nullable: decay amplitude e^0 = 1)
 *   tau            [H, dk]        float (nullable: decay bias 0)
 *   S0, S_final    [B, H, dv, dk] float     m vectors      [B, H, dv]     float
 * Gradients have the layout and dtype of the tensor they belong to.  Every device pointer
 * must be 16-byte aligned.
 *
 * Supported shapes: dk, dv in {64, 128}; 1 <= rank <= 64; chunk in {16, 32, 64, 128};
 * T a multiple of 16 (a shorter last chunk is allowed: its mean runs over its own tokens);
 * B*T < 2^31 token rows.
 * chunk = 1 selects the exact content-aware recurrence, whose content signal is read from the
 * state right before every token (m_t = S_{t-1} q_t; the L = 1 case of the definition, CARVE
 * blog Tables 1 and 3): token-sequential kernels, mc_mode 0 only, no packed sequences.  Its
 * `saved` buffer holds the state every 64 tokens and its workspace one 64-token segment of
 * states per unit.
 */
#ifndef CARVE_H
#define CARVE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CARVE_OK = 0,
    CARVE_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad dimension or enum value    */
    CARVE_ERR_UNSUPPORTED = 2,  /* well-formed but outside the supported shape set above    */
    CARVE_ERR_CUDA = 3,         /* a CUDA launch or attribute call failed                   */
    CARVE_ERR_TIMEOUT = 4       /* a bounded device-side wait expired (reported, not hung)  */
} carve_status;

typedef enum { CARVE_IO_FP32 = 0, CARVE_IO_BF16 = 1 } carve_io;

typedef enum {
    CARVE_MC_BOUNDARY_STATE = 0, /* m_c = S_[c-1] mean(q_c)           */
    CARVE_MC_PREV_MEAN_O = 1     /* m_c = mean of chunk c-1's outputs */
} carve_mc_mode;

/* Problem description shared by every entry point.  io and mc_mode take the enum values
 * above.  For carve_step, T is ignored and chunk is the block length of mc_mode 1. */
typedef struct {
    int B, H, T, dk, dv, rank, chunk;
    int io;
    int mc_mode;
} carve_dims;

/* Human-readable name of a status code (static storage). */
const char *carve_status_string(carve_status s);

/* Size in bytes of the `saved` buffer that carve_fwd fills for carve_bwd (chunk-boundary
 * states and per-chunk content signals).  0 if the dims are invalid. */
size_t carve_saved_bytes(const carve_dims *d);

/* Size in bytes of the scratch buffer carve_bwd needs.  0 if the dims are invalid. */
size_t carve_bwd_workspace_bytes(const carve_dims *d);

/*
 * carve_fwd -- the forward recurrence over T tokens (the chunked WY evaluation of the
 * definition above; CARVE blog sections 2.1-2.3, paperdance abstract).
 *   Aw          nullable: the write gate's content factor (dw_c = 0 when NULL)
 *   A_dec, tau  nullable, independently: the decay's log-amplitude and bias (0 when NULL)
 *   S0          nullable: initial state (treated as 0 when NULL)
 *   m_prev_in   nullable: mc_mode 1 content signal for the first chunk (0 when NULL)
 *   o           out: outputs
 *   S_final     nullable out: state after the last token
 *   m_prev_out  nullable out: mean output of the last chunk (the m_prev_in of a chained call)
 *   saved       nullable out: carve_saved_bytes(d) bytes, required if carve_bwd follows
 *   stream      a cudaStream_t (NULL = legacy default stream)
 */
carve_status carve_fwd(const carve_dims *d, const void *q, const void *k, const void *v,
                       const float *g_logit, const float *bx, const float *w_logit,
                       const float *A, const float *Bm, const float *Aw, const float *A_dec,
                       const float *tau, const float *S0, const float *m_prev_in, void *o,
                       float *S_final, float *m_prev_out, void *saved, void *stream);

/*
 * carve_bwd -- reverse sweep over the chunks: gradients of
 *   sum(dO*o) + sum(dS_final*S_final) + sum(dm_prev_out*m_prev_out)
 * with respect to every input of carve_fwd.  The forward inputs and the `saved` buffer of
 * the matching carve_fwd call must be passed unchanged.  dA and dB are overwritten (summed
 * over the batch), not accumulated.
 *   dS_final, dm_prev_out   nullable (0 when NULL)
 *   Aw, dAw                 both NULL (no write-gate content term) or both given; dAw is
 *                           overwritten with the gradient summed over the batch
 *   A_dec, dA_dec; tau, dtau  each pair both NULL or both given; dA_dec [H] and dtau [H, dk]
 *                           are overwritten with the gradients summed over the batch
 *   dS0, dm_prev_in         nullable outputs
 *   workspace               carve_bwd_workspace_bytes(d) bytes of scratch
 */
carve_status carve_bwd(const carve_dims *d, const void *q, const void *k, const void *v,
                       const float *g_logit, const float *bx, const float *w_logit,
                       const float *A, const float *Bm, const float *Aw, const float *A_dec,
                       const float *tau, const float *S0, const float *m_prev_in, const void *saved,
                       const void *dO, const float *dS_final, const float *dm_prev_out, void *dq,
                       void *dk, void *dv, float *dg_logit, float *dbx, float *dw_logit, float *dA,
                       float *dB, float *dAw, float *dA_dec, float *dtau, float *dS0,
                       float *dm_prev_in, void *workspace, void *stream);

/*
 * carve_fwd_varlen, carve_bwd_varlen -- carve_fwd / carve_bwd over variable-length sequences
 * packed along the token axis (no padding).  d->B is the number of sequences N and d->T an
 * upper bound on every sequence's length (a multiple of 16, it sizes `saved` and `workspace`
 * through carve_saved_bytes(d) and carve_bwd_workspace_bytes(d)); cu_seqlens is a DEVICE
 * int32 array [N+1] of row offsets (cu_seqlens[0] = 0, non-decreasing), sequence n owning
 * rows [cu_seqlens[n], cu_seqlens[n+1]) of the token tensors, and total_tokens is their row
 * count: q, k, g_logit, bx [total_tokens, H, dk]; v, o [total_tokens, H, dv]; w_logit
 * [total_tokens, H] (and the gradients alike).  S0, S_final, m vectors and their gradients
 * are per sequence, [N, H, ...].  Every sequence runs the recurrence above on its own: its own
 * state, content signal and chunk grid, which restarts at its first token; any length from 0
 * to d->T is allowed (a ragged last chunk computes only its own tokens, and an empty sequence
 * passes S0 and m_prev_in through).  Rows that belong to no sequence are not written.  The
 * offsets live on the device, so the host cannot check them: a sequence whose rows fall
 * outside [0, total_tokens] or number more than d->T is computed as empty and the next
 * carve_check returns CARVE_ERR_INVALID_ARG.  The kernels are chosen as for carve_fwd /
 * carve_bwd from d (the tensor-core ones for bf16, dk = dv = 128, rank <= 32, chunk >= 32
 * and a bound T that is a multiple of 32).
 */
carve_status carve_fwd_varlen(const carve_dims *d, const int32_t *cu_seqlens, int64_t total_tokens,
                              const void *q, const void *k, const void *v, const float *g_logit,
                              const float *bx, const float *w_logit, const float *A, const float *Bm,
                              const float *Aw, const float *A_dec, const float *tau, const float *S0,
                              const float *m_prev_in, void *o, float *S_final, float *m_prev_out,
                              void *saved, void *stream);

carve_status carve_bwd_varlen(const carve_dims *d, const int32_t *cu_seqlens, int64_t total_tokens,
                              const void *q, const void *k, const void *v, const float *g_logit,
                              const float *bx, const float *w_logit, const float *A, const float *Bm,
                              const float *Aw, const float *A_dec, const float *tau, const float *S0,
                              const float *m_prev_in, const void *saved, const void *dO,
                              const float *dS_final, const float *dm_prev_out, void *dq, void *dk,
                              void *dv, float *dg_logit, float *dbx, float *dw_logit, float *dA,
                              float *dB, float *dAw, float *dA_dec, float *dtau, float *dS0,
                              float *dm_prev_in, void *workspace, void *stream);

/*
 * carve_bwd_noalloc -- carve_bwd without a workspace argument, for callers that cannot
 * allocate device memory when they run the backward (for example a plugin inside a host
 * framework that owns all device memory and passes in only input and output buffers, or a
 * latency-critical loop that must avoid cudaMalloc's implicit synchronisation).  The pages
 * have no counterpart to this entry point; it only changes where the scratch lives.
 *
 * Arguments, layouts, results and errors are those of carve_bwd.  The scratch is a 4 MiB
 * array inside the library, present on every GPU that loads it until the process exits, so
 * the call allocates nothing.  Limit: carve_bwd_workspace_bytes(d) <= 4 MiB, that is
 * B*H*(dk*rank + rank*dv + rank + dk + 1) floats, or, when the tensor-core kernels run (bf16,
 * dk = dv = 128, rank <= 32), B*H*(NG*292 + 132) + ceil(B*NG/64)*H*257*rank floats with
 * NG = ceil(T/chunk) (chunk = 1 adds 64*dv*dk floats per unit); larger problems return
 * CARVE_ERR_UNSUPPORTED without launching anything.
 * The first call on each device looks up the array's device address (with that device
 * current) and caches it; make that first call before any stream capture begins.
 * Every call shares the one array: calls that overlap on the GPU (different streams, or
 * threads racing on one device) corrupt each other's dA/dB.  Serialise them.
 */
carve_status carve_bwd_noalloc(const carve_dims *d, const void *q, const void *k, const void *v,
                               const float *g_logit, const float *bx, const float *w_logit,
                               const float *A, const float *Bm, const float *Aw, const float *A_dec,
                               const float *tau, const float *S0, const float *m_prev_in,
                               const void *saved, const void *dO, const float *dS_final,
                               const float *dm_prev_out, void *dq, void *dk, void *dv,
                               float *dg_logit, float *dbx, float *dw_logit, float *dA, float *dB,
                               float *dAw, float *dA_dec, float *dtau, float *dS0,
                               float *dm_prev_in, void *stream);

/*
 * carve_step -- one decode token for every (b,h) (the recurrence above with T = 1;
 * inference costs O(dv dk) per token, CARVE blog Table 1).
 *   mc_mode 0: content signal read from the state before this token, m = S q (the chunk
 *              mean over future tokens does not exist while decoding; this is the L = 1
 *              readout).
 *   mc_mode 1: content signal = mean output of the previous complete block of d->chunk
 *              tokens.  mstate [B,H,2,dv] float holds (sum of o in the current block, mean
 *              of the previous block) and pos [B,H] int32 the tokens consumed so far; both
 *              are updated in place.  Unused (may be NULL) in mc_mode 0.
 * Inputs: q, k [B,H,dk] io; v [B,H,dv] io; g_logit, bx [B,H,dk] float; w_logit [B,H]
 * float; Aw, A_dec, tau nullable as in carve_fwd.  S [B,H,dv,dk] float is read and written
 * in place; o [B,H,dv] io.
 */
carve_status carve_step(const carve_dims *d, const void *q, const void *k, const void *v,
                        const float *g_logit, const float *bx, const float *w_logit,
                        const float *A, const float *Bm, const float *Aw, const float *A_dec,
                        const float *tau, float *S, float *mstate, int32_t *pos, void *o,
                        void *stream);

/*
 * carve_check -- blocks the host until the work queued on `stream` has finished, then
 * reports what the device saw: CARVE_ERR_CUDA if the stream reports an error,
 * CARVE_ERR_TIMEOUT if a bounded device-side wait of a carve kernel (a shared-memory
 * barrier waiting for a bulk copy or a tensor-core product) gave up since the previous
 * carve_check (the tensor-core forward also reports it, without computing anything, if its
 * dynamic shared memory were not 1024-byte aligned; never observed), CARVE_ERR_INVALID_ARG
 * if a varlen call met out-of-range sequence offsets, else CARVE_OK.  The device status words
 * are cleared by the call.  A kernel whose wait gives up records it, stops its sweep, waits
 * (again bounded) for its own copies and products in flight, frees the tensor memory it
 * holds and returns, so the CUDA context stays usable; the outputs of that call are
 * undefined.  The pages have no counterpart to this entry point.
 */
carve_status carve_check(void *stream);

/*
 * carve_selftest_timeout -- test hook for the path above: launches one thread that waits
 * on a shared-memory barrier nothing arrives on, bounded by `iterations` polls (1 to
 * 1,000,000), so the wait always gives up and records it; the next carve_check returns
 * CARVE_ERR_TIMEOUT.  Nothing else is touched.  No counterpart in the pages.
 */
carve_status carve_selftest_timeout(uint32_t iterations, void *stream);

/*
 * carve_selftest_stall -- test hook for the same path inside the tensor-core sweep kernels:
 * arms a one-shot that the next carve_fwd or carve_bwd call running a tensor-core sweep (bf16,
 * dk = dv = 128, rank <= 32) takes and clears.  That call skips the tile copy of its first
 * compute chunk and bounds each of its barrier waits by `iterations` polls (1 to 1,000,000),
 * so its first wait gives up in every CTA: the sweep records it, waits (bounded) for the
 * copies it still has in flight and ends; the call's outputs are undefined and the next
 * carve_check returns CARVE_ERR_TIMEOUT.  The one-shot is process-wide state (the one
 * exception, with carve_bwd_noalloc, to "no mutable global state" above).  No counterpart in
 * the pages.
 */
carve_status carve_selftest_stall(uint32_t iterations);

#ifdef __cplusplus
}
#endif

#endif /* CARVE_H */

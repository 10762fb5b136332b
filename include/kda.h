/*
 * kda.h -- C ABI of libkda_b200.so, the B200 (sm_100a) Kimi Delta Attention mixer.
 *
 * What the library computes, per head h with a dk x dv fp32 state S
 * ("Kimi K3: Architecture, Training, and Million-Token Agentic RL", brenchcc
 * research note):
 *   - recurrence, section 3.1 equation:
 *       S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *       o_t = S_t^T q_t            (the read follows the write; no 1/sqrt(dk))
 *     Diag(alpha_t) scales the ROWS of S, one row per key channel.
 *   - lower-bounded gate, section 3.3 equation (restated in "Kimi K3 Under the
 *     Hood", section "Sequence mixing: three KDA layers per global MLA layer"):
 *       g[t,h,c] = -5 * sigmoid(exp(A[h,c]) * z[t,h,c]),  alpha = exp(g)
 *   - chunked prefill, section 3.3 chunk I/O equation: tokens inside a chunk
 *     become matrix products, the state crosses only chunk boundaries,
 *     S_in[c+1] = S_out[c]; decode follows the recurrence one token at a time
 *     (section 3.2, (x_t, S_{t-1}) -> (y_t, S_t)).
 *   - prefix-cache resume ("Kimi K3 Under the Hood", section "Serving two
 *     incompatible cache types"; brenchcc note section 9): a request copies a
 *     cached state into its running state and resumes prefill from it -- here
 *     the optional initial_state / final_state of kda_prefill.
 *
 * Conventions shared by every entry point
 *   - All tensors are dense, row-major, contiguous, on the current CUDA device
 *     unless stated "host".  T = total packed tokens, N = sequences, H = heads.
 *       q, k, z : [T, H, dk]   storage dtype `dt`
 *       v, o    : [T, H, dv]   storage dtype `dt`
 *       beta    : [T, H]       fp32, expected in [0, 1]
 *       A       : [H, dk]      fp32 (gate log-scale, one per head and key channel)
 *       states  : [N or P, H, dk, dv] fp32, dv contiguous (row = key channel)
 *   - dk, dv in {32, 64, 128}.  Device pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call is asynchronous on that stream: it validates arguments on the
 *     host, enqueues kernels and returns; it never synchronises.
 *   - Ownership: the caller owns every buffer (inputs, outputs, states and the
 *     prefill workspace).  The library allocates no device memory, keeps no
 *     per-call state and may be called from several host threads.
 *   - Errors: argument checks run before anything is enqueued, and a failing
 *     check returns its code with nothing launched.  A launch failure returns
 *     KDA_ERR_CUDA.  NaN / Inf in the data are not detected; they propagate as
 *     the mathematics says.
 */
#ifndef KDA_B200_H
#define KDA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KDA_ABI_VERSION 3

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, bad cu_seqlens */
    KDA_ERR_UNSUPPORTED = 2,   /* valid request the library does not implement (e.g. dk=96) */
    KDA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than kda_prefill_workspace_size */
    KDA_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
    KDA_ERR_TIMEOUT = 5        /* a bounded on-device wait gave up (see kda_device_status) */
} kda_status;

typedef enum {
    KDA_DTYPE_BF16 = 0,        /* q, k, v, z, o stored as bfloat16 */
    KDA_DTYPE_F32 = 1          /* q, k, v, z, o stored as fp32 */
} kda_dtype;

typedef enum {
    KDA_ALGO_AUTO = 0,         /* tensor-core path for bf16 (split when it pays, see
                                  kda_prefill_segments), CUDA-core fp32 path for fp32 */
    KDA_ALGO_CUDA_CORE = 1,    /* chunked prefill in fp32 FMA on CUDA cores (check mode) */
    KDA_ALGO_TENSOR_CORE = 2,  /* chunked prefill on tcgen05 tensor cores (bf16 only),
                                  every sequence one chain of chunks */
    KDA_ALGO_TENSOR_CORE_SPLIT = 3  /* tensor cores with every sequence split into
                                  segments composed by an affine scan (bf16 only) */
} kda_algo;

typedef enum {
    KDA_GATE_LOWER_BOUNDED = 0,  /* K3: g = -5 sigmoid(exp(A) z), in [-5, 0] */
    KDA_GATE_SOFTPLUS = 1        /* earlier Kimi Linear: g = -softplus(exp(A) z), unbounded */
} kda_gate;

/* Version of this ABI (KDA_ABI_VERSION of the build). */
int32_t kda_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *kda_status_string(kda_status s);

/*
 * Bytes of device workspace kda_prefill needs for these sizes and algorithm.
 * The value depends only on the arguments (an upper bound over every
 * cu_seqlens with this total_tokens and num_seqs), so one buffer can be
 * reused across calls of the same shape.  Returns 0 for invalid arguments.
 */
size_t kda_prefill_workspace_size(int32_t total_tokens, int32_t num_seqs, int32_t H,
                                  int32_t dk, int32_t dv, kda_dtype dt, kda_algo algo);

/*
 * Chunked prefill over packed variable-length sequences ("Kimi K3:
 * Architecture, Training, and Million-Token Agentic RL", section 3.3).
 *
 * For each sequence n (tokens cu_seqlens[n] .. cu_seqlens[n+1]-1) and head h,
 * starts from initial_state[n,h] (zeros if initial_state is NULL), writes
 * o[t,h,:] = S_t^T q_t for every token, and, if final_state is non-NULL, the
 * state after the sequence's last token into final_state[n,h].  A sequence of
 * length 0 passes its initial state through.  final_state may equal
 * initial_state (in-place resume); no other buffers may overlap.
 *
 *   cu_seqlens_dev  [N+1] int32, device: 0 = cu[0] <= cu[1] <= ... <= cu[N] = T.
 *   cu_seqlens_host [N+1] int32, HOST copy of the same offsets, or NULL.  When
 *                   given it is validated (KDA_ERR_INVALID_ARG if malformed) and
 *                   used to schedule long sequences first; the device copy is
 *                   not read on the host.
 *   workspace       device buffer of at least
 *                   kda_prefill_workspace_size(T, N, H, dk, dv, dt, algo) bytes
 *                   (may be NULL when that size is 0); contents are scratch.
 *   algo            KDA_ALGO_AUTO, or a forced path; KDA_ALGO_TENSOR_CORE(_SPLIT)
 *                   with dt = KDA_DTYPE_F32 or dk, dv != 128 returns
 *                   KDA_ERR_UNSUPPORTED.
 *   stage_events    optional instrumentation (NULL = none): an array of
 *                   num_stage_events cudaEvent_t handles (as void*), owned by
 *                   the caller.  events[0] is recorded on `stream` before the
 *                   first kernel of the call and events[i] after its i-th
 *                   kernel, so elapsed(events[i-1], events[i]) is the duration
 *                   of kernel i.  Entries beyond kda_prefill_kernel_count() + 1
 *                   are left untouched; fewer entries record fewer boundaries.
 * kda_prefill is kda_prefill_ex with algo = KDA_ALGO_AUTO and no events.
 */
kda_status kda_prefill(const void *q, const void *k, const void *v, const void *z,
                       const float *A, const float *beta,
                       const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                       int32_t num_seqs, int32_t total_tokens, int32_t H, int32_t dk,
                       int32_t dv, kda_dtype dt, const float *initial_state,
                       float *final_state, void *o, void *workspace,
                       size_t workspace_bytes, void *stream);

kda_status kda_prefill_ex(const void *q, const void *k, const void *v, const void *z,
                          const float *A, const float *beta,
                          const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                          int32_t num_seqs, int32_t total_tokens, int32_t H, int32_t dk,
                          int32_t dv, kda_dtype dt, const float *initial_state,
                          float *final_state, void *o, void *workspace,
                          size_t workspace_bytes, kda_algo algo, void *stream,
                          void *const *stage_events, int32_t num_stage_events);

/*
 * kda_prefill_ex that also writes state checkpoints for prefix caching ("Kimi
 * K3 Under the Hood", section "Serving two incompatible cache types": prefix
 * hashes every 512 tokens, KDA states kept only at selected boundaries, a hit
 * copies the cached state into the running state and resumes prefill).
 *
 *   checkpoint_every  0 = none (checkpoints may be NULL), else a positive
 *                     multiple of 64: checkpoint j (j = 1 .. L_n / every) of
 *                     sequence n is the state after its first j * every tokens.
 *   checkpoints       device fp32 [kda_checkpoint_count(...), H, dk, dv]; row
 *                     (sum_{m<n} L_m / every) + j - 1 holds checkpoint j of
 *                     sequence n (a checkpoint at a sequence's last token equals
 *                     its final state).  16-byte aligned, caller-owned.
 * Other arguments, results and errors as kda_prefill_ex; a bad checkpoint_every
 * or a NULL checkpoints with checkpoint_every > 0 is KDA_ERR_INVALID_ARG.
 */
kda_status kda_prefill_checkpointed(const void *q, const void *k, const void *v, const void *z,
                                    const float *A, const float *beta,
                                    const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                                    int32_t num_seqs, int32_t total_tokens, int32_t H, int32_t dk,
                                    int32_t dv, kda_dtype dt, const float *initial_state,
                                    float *final_state, void *o, void *workspace,
                                    size_t workspace_bytes, kda_algo algo, void *stream,
                                    void *const *stage_events, int32_t num_stage_events,
                                    int32_t checkpoint_every, float *checkpoints);

/*
 * kda_prefill_ex with a choice of gate, without events.  KDA_GATE_LOWER_BOUNDED is
 * kda_prefill_ex itself.  KDA_GATE_SOFTPLUS is the earlier Kimi Linear gate, which
 * the pages contrast with K3's bound ("Kimi K3: Architecture, Training, and
 * Million-Token Agentic RL", section 3.3; "Kimi K3 Under the Hood", section
 * "Sequence mixing": an unbounded negative Softplus, read with K3's pre-activation
 * as g = -softplus(exp(A[h,c]) z[t,h,c])).  Its cumulative decay inside a 16-token
 * tile is unbounded, so the reciprocal factors of the dense tile form overflow and
 * every diagonal tile needs the position-pair path: the fp32 CUDA-core path
 * computes each intra-chunk decay e^{G_r - G_s} as one exponent per pair and key
 * channel.  With KDA_GATE_SOFTPLUS:
 *   - CUDA_CORE runs the fp32 CUDA-core path with that pair form for every
 *     16-token chunk (no workspace: it may be NULL with workspace_bytes = 0);
 *   - TENSOR_CORE(_SPLIT), and AUTO for bf16 with dk = dv = 128, run the
 *     tensor-core path as it stood before the bound: off-diagonal 16-token
 *     sub-tile pairs on tcgen05 with a reference between them (every factor
 *     <= 1, formed as one exponent), and the four diagonal 16 x 16 tiles of each
 *     64-token chunk computed pair by pair on CUDA cores by a separate kernel.
 *     Its workspace is kda_prefill_gated_workspace_size(..., gate), 8 KiB per
 *     (chunk, head) more than the bounded gate's.
 * The per-token log-decay is clamped at -110 (e^{-110} is 0 in fp32), which
 * changes no result and keeps a chunk's cumulative decay small enough for fp32
 * differences.  A gate value outside the enum is KDA_ERR_INVALID_ARG.
 */
kda_status kda_prefill_gated(const void *q, const void *k, const void *v, const void *z,
                             const float *A, const float *beta,
                             const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                             int32_t num_seqs, int32_t total_tokens, int32_t H, int32_t dk,
                             int32_t dv, kda_dtype dt, const float *initial_state,
                             float *final_state, void *o, void *workspace,
                             size_t workspace_bytes, kda_algo algo, kda_gate gate, void *stream);

/*
 * Workspace bytes of kda_prefill_gated with the given gate (for
 * KDA_GATE_LOWER_BOUNDED equal to kda_prefill_workspace_size); 0 for the
 * CUDA-core path or invalid arguments (an invalid gate included).
 */
size_t kda_prefill_gated_workspace_size(int32_t total_tokens, int32_t num_seqs, int32_t H,
                                        int32_t dk, int32_t dv, kda_dtype dt, kda_algo algo,
                                        kda_gate gate);

/*
 * Debug run of the tensor-core prefill (bf16, dk = dv = 128; otherwise
 * KDA_ERR_UNSUPPORTED): the same call as kda_prefill_ex with
 * KDA_ALGO_TENSOR_CORE, which also writes the intermediates that its fused
 * kernels keep on chip, per token, as fp32 [T, H, 128] (any pointer may be NULL;
 * 16-byte aligned):
 *   G_out      the cumulative log-decay of the token's 64-token chunk (chunks
 *              start at each sequence start; "Kimi K3: Architecture, Training,
 *              and Million-Token Agentic RL", section 3.3 gate equation and the
 *              inclusive in-chunk sum), from a separate kernel with the fused
 *              kernel's arithmetic;
 *   W_out      W = (I + A)^-1 Diag(beta) K e^{G}, as stored for the state pass (bf16 values);
 *   U_out      U = (I + A)^-1 Diag(beta) V, likewise;
 *   delta_out  delta = U - W S_in, the chunk's state-independent correction, as
 *              the state pass consumes it (bf16 values), S_in the state entering
 *              the chunk.
 * A debugging and test aid with no counterpart in the pages: it exposes the
 * stages of the chunked form that section 3.3 describes, so that each can be
 * compared with a plain chunkwise computation.  Sequences are never split.
 */
kda_status kda_prefill_debug(const void *q, const void *k, const void *v, const void *z,
                             const float *A, const float *beta,
                             const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                             int32_t num_seqs, int32_t total_tokens, int32_t H, int32_t dk,
                             int32_t dv, kda_dtype dt, const float *initial_state,
                             float *final_state, void *o, void *workspace,
                             size_t workspace_bytes, float *G_out, float *W_out, float *U_out,
                             float *delta_out, void *stream);

/*
 * Rows of the checkpoint tensor for these HOST offsets: sum over sequences of
 * L_n / checkpoint_every.  Returns -1 for invalid arguments (NULL offsets with
 * num_seqs > 0, checkpoint_every not a positive multiple of 64, decreasing
 * offsets).
 */
int64_t kda_checkpoint_count(const int32_t *cu_seqlens_host, int32_t num_seqs,
                             int32_t checkpoint_every);

/*
 * Number of kernels one kda_prefill_ex call (no checkpoints) launches for these
 * sizes and algorithm, for a non-empty batch: 1 on CUDA cores, 3 on tensor cores
 * (plan, intra-chunk, state), 5 when the call splits its sequences (plus the
 * segment composition and the output correction).  0 for invalid arguments.
 */
int32_t kda_prefill_kernel_count(int32_t total_tokens, int32_t num_seqs, int32_t H, int32_t dk,
                                 int32_t dv, kda_dtype dt, kda_algo algo);

/*
 * Segments per sequence that a kda_prefill_ex call without checkpoints uses
 * for these sizes: 1 = no split; 0 for invalid arguments.
 *
 * Sequence split by affine composition ("Kimi K3 Under the Hood", section
 * "Infrastructure for a 3T-class MoE", on KDA context parallelism: a sequence
 * segment is summarised by the map it applies to the
 * state, a cumulative dk x dk transition plus the state it produces from zero,
 * and these maps compose associatively).  Here the segments of one sequence run
 * on different SMs of one GPU: segment s >= 1 computes, from its chunk blocks,
 * its state from zero S_loc(s), its transition M_s and, per chunk, the matrix E
 * that maps the segment's true entry state to the missing part of the chunk's
 * outputs; then S_in(s + 1) = M_s S_in(s) + S_loc(s) in fp32 and o += E S_in(s)
 * on the tensor cores.  Results equal the unsplit path's up to rounding.
 * The count: each (sequence, head) takes 2 G - 1 concurrent state chains, so G
 * is the largest value with N H (2 G - 1) <= 148 (the B200's SMs), at most 16;
 * KDA_ALGO_AUTO additionally requires T / (64 N) >= 16 G (long sequences) and
 * KDA_ALGO_TENSOR_CORE_SPLIT at least 2.  A sequence with fewer chunks than G
 * uses one segment per chunk.  kda_prefill_checkpointed with checkpoints never
 * splits under AUTO and returns KDA_ERR_UNSUPPORTED under
 * KDA_ALGO_TENSOR_CORE_SPLIT.
 */
int32_t kda_prefill_segments(int32_t total_tokens, int32_t num_seqs, int32_t H, int32_t dk,
                             int32_t dv, kda_dtype dt, kda_algo algo);

/*
 * kda_prefill without a workspace argument, for callers that cannot allocate
 * device memory at call time (for example a serving engine that gives all free
 * HBM to its cache pool at start-up and forbids later allocations, code running
 * under another framework's allocator, or a latency-critical loop that cannot
 * pay for the device synchronisation of cudaMalloc / cudaFree).  It has no
 * counterpart in the source pages; it is a deployment convenience.
 *
 * Same arguments and results as kda_prefill on the tensor-core path (bf16,
 * dk = dv = 128; other types or sizes return KDA_ERR_UNSUPPORTED).  The scratch
 * memory is one file-scope device array of 64 MiB that the library holds on
 * every GPU where this entry point's module is loaded, until the process exits.
 * A call whose kda_prefill_workspace_size(..., KDA_ALGO_TENSOR_CORE) exceeds
 * 64 MiB (about 900 chunk-head tiles of 64 tokens, e.g. one 576-token sequence
 * at 96 heads) returns KDA_ERR_WORKSPACE and launches nothing.  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *
 * The first call on each device looks up the array's device address, and it
 * is also the call that places the array in that device's memory: the CUDA
 * runtime loads a library's device code lazily by default, so the 64 MiB are
 * taken at this first call, not when the library is loaded.  A caller that
 * later gives away all free device memory (for example to a cache pool) makes
 * one call first -- any small valid input -- before reserving that memory,
 * and before any stream capture.  The address is cached per device and
 * context; after a device reset (which destroys the context and the array's
 * contents) the next call looks it up again and places a fresh array.
 * Every call on a device shares the one array and leaves its contents behind;
 * the kernels overwrite every scratch byte they later read, so nothing needs
 * clearing.  Calls whose work overlaps on the GPU (different streams, or
 * several host threads) race on the array: the caller must serialise them,
 * e.g. by issuing them all on one stream.
 */
kda_status kda_prefill_noalloc(const void *q, const void *k, const void *v, const void *z,
                               const float *A, const float *beta,
                               const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                               int32_t num_seqs, int32_t total_tokens, int32_t H, int32_t dk,
                               int32_t dv, kda_dtype dt, const float *initial_state,
                               float *final_state, void *o, void *stream);

/*
 * One recurrent decode step for B sequences, one new token each ("Kimi K3:
 * Architecture, Training, and Million-Token Agentic RL", section 3.2 edit
 * order: Sbar = Diag(alpha) S; vhat = Sbar^T k; S = Sbar + beta k (v - vhat)^T;
 * o = S^T q).
 *
 *   q, k, z [B, H, dk], v [B, H, dv], o [B, H, dv] in dtype dt; beta [B, H] fp32.
 *   state   [P, H, dk, dv] fp32 pool, updated IN PLACE: row slots[b] (or b when
 *           slots is NULL) holds sequence b's state.  Duplicate slot values are
 *           a data race (not detected); slot values must lie in [0, P).
 *   pool_size P >= B when slots is NULL; slots is a device array of B int32.
 */
kda_status kda_decode_step(const void *q, const void *k, const void *v, const void *z,
                           const float *A, const float *beta, int32_t B, int32_t H,
                           int32_t dk, int32_t dv, kda_dtype dt, float *state,
                           int32_t pool_size, const int32_t *slots, void *o,
                           void *stream);

/*
 * Optional host-side check of a decode batch's slots (a HOST copy): KDA_OK when
 * every slot lies in [0, pool_size) and no two batch rows share one, else
 * KDA_ERR_INVALID_ARG.  kda_decode_step does not make this check itself (it
 * would need the slots on the host); two rows sharing a slot race on it.
 */
kda_status kda_decode_check_slots(const int32_t *slots_host, int32_t B, int32_t pool_size);

/*
 * kda_decode_step with a choice of gate (kda_gate, as for kda_prefill_gated; the
 * decode step needs no special path for the unbounded gate: alpha = e^{g} is
 * applied directly).  A gate value outside the enum is KDA_ERR_INVALID_ARG.
 */
kda_status kda_decode_step_gated(const void *q, const void *k, const void *v, const void *z,
                                 const float *A, const float *beta, int32_t B, int32_t H,
                                 int32_t dk, int32_t dv, kda_dtype dt, float *state,
                                 int32_t pool_size, const int32_t *slots, void *o,
                                 kda_gate gate, void *stream);

/*
 * Speculative-decoding verify and replay ("Kimi K3 Under the Hood", section
 * "Serving two incompatible cache types": rejected drafts must not advance the
 * recurrent state; the projected inputs of the drafts are kept and the accepted
 * tokens are replayed on-chip in one fused recurrence instead of saving a state
 * per draft position).  Each (sequence, head) state is read once, the tokens run
 * on-chip in the section 3.2 edit order, and the state is written at most once.
 *
 *   q, k, z [B, Tq, H, dk], v [B, Tq, H, dv] in dtype dt; beta [B, Tq, H] fp32;
 *   the Tq tokens of sequence b are consecutive positions after its state.
 *   state, pool_size, slots  as kda_decode_step (pool [P, H, dk, dv] fp32).
 *   num_tokens   device int32 [B]: tokens of sequence b to apply (clamped to
 *                [0, Tq]), or NULL for all Tq.
 *   update_state 0 = verify: o receives every applied token's output and the
 *                state in HBM is left untouched; 1 = replay/commit: the state of
 *                each sequence is advanced by its num_tokens[b] tokens in place
 *                (o is written too when non-NULL).
 *   o            [B, Tq, H, dv] dtype dt, or NULL (then update_state must be 1).
 * Tq in [1, 64].  Errors as kda_decode_step.  The kernel copies each state into
 * on-chip memory with the copy engine and waits for it with a 2 s limit; a wait
 * that gives up records KDA_ERR_TIMEOUT in the device status word
 * (kda_device_status) and the launch ends without writing that state.  Two
 * sequences must not share a slot when update_state is 1.
 */
kda_status kda_decode_multi(const void *q, const void *k, const void *v, const void *z,
                            const float *A, const float *beta, int32_t B, int32_t Tq, int32_t H,
                            int32_t dk, int32_t dv, kda_dtype dt, float *state,
                            int32_t pool_size, const int32_t *slots,
                            const int32_t *num_tokens, int32_t update_state, void *o,
                            void *stream);

/*
 * Reads and clears the library's device status word for the current device
 * (synchronises `stream` first).  Kernels that wait on an on-chip barrier
 * with an iteration limit record KDA_ERR_TIMEOUT there instead of hanging;
 * *status_out receives KDA_OK or the first recorded code.
 */
kda_status kda_device_status(void *stream, int32_t *status_out);

/*
 * Failure-detection self-test (a diagnostic with no counterpart in the source
 * pages).  Enqueues one CTA whose mbarrier wait has nothing to complete it; the
 * wait gives up after limit_ns (1 ms .. 10 s, else KDA_ERR_INVALID_ARG), writes
 * KDA_ERR_TIMEOUT into the device status word and the kernel exits normally, so
 * the context stays usable.  kda_device_status then reports KDA_ERR_TIMEOUT.
 * It exercises the same bounded-wait path every tensor-core kernel uses.
 */
kda_status kda_selftest_wait_timeout(int64_t limit_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_B200_H */

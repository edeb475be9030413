/*
 * mlstm.h -- C ABI of libmlstm, the mLSTM matrix-memory cell on NVIDIA B200 (sm_100a).
 *
 * The cell (per batch element b and head h, token t = 1..S):
 *
 *   log f_t = logsigmoid(f~_t)
 *   m_t     = max(log f_t + m_{t-1}, i~_t)                  stabilizer
 *   f'_t    = exp(log f_t + m_{t-1} - m_t),  i'_t = exp(i~_t - m_t)
 *   C_t     = f'_t C_{t-1} + i'_t k_t v_t^T                 C stored [DHQK][DHV]
 *   n_t     = f'_t n_{t-1} + i'_t k_t
 *   h_t     = o_t * (C_t^T qh_t) / max(|n_t . qh_t|, exp(-m_t)),  qh_t = q_t / sqrt(DHQK)
 *
 * Sources: "xLSTM Guide: Extended LSTM Architecture & Matrix Memory" -- sections
 * "The Stabilizer State: Preventing Numerical Overflow" (m_t and the stabilized
 * exponential gates), "mLSTM: Matrix Key-Value Memory and Covariance Updates" /
 * "Recurrent Formulation (Inference Mode)" (C_t, n_t, h_t), "The Dual
 * Formulation" (the parallel form over a causal decay matrix) and "Exploit
 * Chunkwise Hardware Kernels for Production Training" (chunks of 64 or 128
 * tokens: dense products inside a chunk, a scan across chunks).  The forget
 * gate is the sigmoid gate in log space; q carries the 1/sqrt(DHQK) factor, so
 * C and n hold raw k; the floor exp(-m_t) is the guide's floor of 1 on the
 * unstabilized states.
 *
 * Conventions for every entry point:
 *  - All data pointers are DEVICE pointers owned by the caller, contiguous,
 *    row-major, 16-byte aligned.  The library allocates no device memory.
 *    Between calls it keeps only host-side caches, each filled once and guarded
 *    by a lock, so that several host threads may call it at the same time: the
 *    dynamic shared-memory limit set on each kernel per device, the driver's
 *    tensor-map encoder function, the sLSTM kernel's cluster capacity per
 *    device, and the device address of mlstm_fwd_noalloc's built-in array.
 *    Results never depend on them.
 *  - Layouts: q, k [B][NH][S][DHQK]; v, ogate, h [B][NH][S][DHV];
 *    igate, fgate [B][NH][S] (float32 pre-activations i~, f~);
 *    C [B][NH][DHQK][DHV], n [B][NH][DHQK], m [B][NH] (float32).
 *  - q, k, v, ogate and h have the element type `dt`; gates and states are
 *    always float32.  ogate holds the already-activated output gate (for
 *    example sigmoid(o~)); NULL means o = 1.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Work is enqueued asynchronously; nothing synchronizes.
 *  - Arguments are checked on the host before anything is enqueued; a bad
 *    argument returns an error status and launches nothing.  A failed launch
 *    returns MLSTM_ERR_CUDA.  No call throws or aborts.
 */
#ifndef MLSTM_H
#define MLSTM_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mlstm_status {
    MLSTM_OK = 0,
    MLSTM_ERR_INVALID_ARG = 1,  /* NULL pointer, negative size, misaligned pointer */
    MLSTM_ERR_UNSUPPORTED = 2,  /* valid but unsupported shape / chunk / dtype */
    MLSTM_ERR_WORKSPACE = 3,    /* workspace NULL or smaller than mlstm_fwd_workspace_size() */
    MLSTM_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed */
    MLSTM_ERR_TIMEOUT = 5       /* a bounded device-side wait gave up (see mlstm_fwd_status) */
} mlstm_status;

typedef enum mlstm_dtype {
    MLSTM_F32 = 0,
    MLSTM_BF16 = 1
} mlstm_dtype;

/*
 * Bytes of device workspace mlstm_fwd needs for these arguments (0 when the
 * arguments are unsupported).  The workspace holds the gate preprocessing
 * (cumulative log forget gates, stabilizers) and the chunk-boundary states.
 */
size_t mlstm_fwd_workspace_size(int B, int NH, int S, int DHQK, int DHV, int chunk,
                                mlstm_dtype dt);

/*
 * Chunkwise parallel forward pass from the zero state (C = 0, n = 0, m = 0)
 * over S tokens.  Writes h_out and, where the pointers are non-NULL, the final
 * state C_final, n_final, m_final.  Mathematically the result equals the
 * recurrence above token by token; `chunk` (16, 32, 64 or 128) is the length
 * of the blocks inside which the causal decay matrix is used.  S may be any
 * value >= 0 (a last, shorter chunk is allowed; S == 0 writes the zero state).
 * Supported: DHQK and DHV multiples of 8 in [8, 512].
 *
 * Accuracy: bf16 inputs run on the tensor cores with fp32 accumulation and
 * state (relative L2 error of h about 3e-3 against an fp64 evaluation).  fp32
 * inputs run in fp32 on the CUDA cores; their error grows with S because the
 * cumulative log forget gates are fp32 sums: about 1e-6 at S = 64, and at
 * S = 4096 with forget pre-activations spread like N(3, 1.5) the rounding of
 * those sums alone reaches about 1.5e-5 relative error.
 *
 * The source defining the operation: the guide's "Recurrent Formulation
 * (Inference Mode)" (what is computed) and "The Dual Formulation" with
 * "Exploit Chunkwise Hardware Kernels for Production Training" (how).
 *
 * workspace: device memory of at least mlstm_fwd_workspace_size() bytes,
 * 256-byte aligned, owned by the caller, used until the enqueued work ends.
 * Two calls in flight must not share a workspace.
 */
mlstm_status mlstm_fwd(const void *q, const void *k, const void *v,
                       const float *igate, const float *fgate, const void *ogate,
                       mlstm_dtype dt, int B, int NH, int S, int DHQK, int DHV, int chunk,
                       void *h_out, float *C_final, float *n_final, float *m_final,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * Forward pass that starts from a given state instead of the zero state: the
 * chunked prefill / resume form of the recurrence (the constant-size state is
 * the whole memory of the sequence so far, "Inference VRAM and Throughput
 * Scaling" and "Deploy xLSTM for Continuous Streaming" of the xLSTM guide).
 * Same arguments as mlstm_fwd plus the initial state C0 [B][NH][DHQK][DHV],
 * n0 [B][NH][DHQK], m0 [B][NH] (float32, device, 16-byte aligned): all three,
 * or all NULL for the zero state.  Running S1 tokens and then S2 more from the
 * returned state equals one pass over S1 + S2 tokens.  The final state may
 * alias the initial one (C_final == C0 and so on) to update it in place.
 * S == 0 copies the initial state to the final-state outputs.
 */
mlstm_status mlstm_fwd_state(const void *q, const void *k, const void *v,
                             const float *igate, const float *fgate, const void *ogate,
                             mlstm_dtype dt, int B, int NH, int S, int DHQK, int DHV, int chunk,
                             const float *C0, const float *n0, const float *m0,
                             void *h_out, float *C_final, float *n_final, float *m_final,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * Sequence-parallel forward pass, the pieces.  A sequence split into R
 * consecutive slices (rank r holds slice r) is run in three steps:
 *   1. every rank: the final state of its slice from the zero state
 *      (mlstm_fwd_final_state) and the slice's total log forget decay
 *      (mlstm_log_decay_sum);
 *   2. the caller all-gathers these summaries over the ranks (NCCL);
 *   3. every rank: its start state from the summaries of the slices before it
 *      (mlstm_state_prefix), then mlstm_fwd_state over its slice from it.
 * The state after a slice is the state before it decayed by the product of the
 * slice's forget gates plus the slice's own contribution, the recurrence of
 * "Recurrent Formulation (Inference Mode)" (xLSTM guide) over the slice; this
 * is the exchange of chunk summaries the guide's "Exploit Chunkwise Hardware
 * Kernels" scan across chunks implies at the granularity of a GPU.  The
 * composed state's stabilizer m can be above the one of a single pass (the
 * slices start from m_0 = 0); C and n are scaled to match, so h and the
 * unstabilized state exp(m) C, exp(m) n are the same.
 */

/*
 * mlstm_fwd without the output stage: the final state (C, n, m) of the slice
 * from the zero state, for step 1.  Same arguments and workspace as mlstm_fwd
 * without q, ogate and h (k, v, igate, fgate as there; the final-state
 * pointers as there, each may be NULL).  No extra entry point in the pages:
 * it is mlstm_fwd with its last phase left out.
 */
mlstm_status mlstm_fwd_final_state(const void *k, const void *v,
                                   const float *igate, const float *fgate,
                                   mlstm_dtype dt, int B, int NH, int S, int DHQK, int DHV, int chunk,
                                   float *C_final, float *n_final, float *m_final,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * g_out[b][h] = sum over the S tokens of logsigmoid(fgate[b][h][t]) (float32,
 * device; fgate [B][NH][S]).  0 for S == 0.  Errors: MLSTM_ERR_INVALID_ARG for
 * negative sizes or NULL pointers, MLSTM_ERR_CUDA for a launch failure.
 */
mlstm_status mlstm_log_decay_sum(const float *fgate, int B, int NH, int S, float *g_out, void *stream);

/*
 * Start state of slice `rank` (0 <= rank < R) from the gathered summaries of
 * the R slices: C_parts [R][B][NH][DHQK][DHV], n_parts [R][B][NH][DHQK],
 * m_parts [R][B][NH] (the zero-start final states of step 1) and g_parts
 * [R][B][NH] (the log decay sums), float32 device arrays, C_parts and C0
 * 16-byte aligned.  Only slices 0 .. rank-1 are read.  Writes C0, n0, m0 in
 * the layouts of mlstm_fwd_state's initial state (rank 0 gets the zero state,
 * m = 0).  DHQK, DHV as for mlstm_fwd.  Errors: MLSTM_ERR_INVALID_ARG for a
 * bad rank, NULL or misaligned pointers; MLSTM_ERR_UNSUPPORTED for head sizes
 * mlstm_fwd rejects or more than 65535 heads; MLSTM_ERR_CUDA for a launch
 * failure.
 */
mlstm_status mlstm_state_prefix(const float *C_parts, const float *n_parts, const float *m_parts,
                                const float *g_parts, int R, int rank, int B, int NH, int DHQK, int DHV,
                                float *C0, float *n0, float *m0, void *stream);

/*
 * mlstm_fwd with per-phase timing: identical work and results, and in addition
 * records CUDA events (cudaEvent_t passed as void*, created by the caller) on
 * `stream`: events[p] just before phase p and events[MLSTM_FWD_PHASES] after
 * the last one.  Phases, in order: 0 gate preprocessing, 1 chunk or segment
 * state contributions, 2 scan of the states across chunks or segments,
 * 3 outputs (and, on the tensor-core path, the in-segment state walk).  A
 * phase that launches nothing on a given path has two events back to back.
 * Entries of `events` may be NULL (that boundary is not recorded); the array
 * itself may not.  events[MLSTM_FWD_PHASES - 1], recorded before the outputs
 * phase, completes once C_final, n_final and m_final are written: a consumer of
 * the final state (a decode step on another stream) can wait for it while the
 * outputs are still being computed.
 */
#define MLSTM_FWD_PHASES 4
mlstm_status mlstm_fwd_profiled(const void *q, const void *k, const void *v,
                                const float *igate, const float *fgate, const void *ogate,
                                mlstm_dtype dt, int B, int NH, int S, int DHQK, int DHV, int chunk,
                                void *h_out, float *C_final, float *n_final, float *m_final,
                                void *workspace, size_t workspace_bytes, void *stream,
                                void *const *events);

/*
 * Number of kernels one mlstm_fwd call with these arguments launches (0 when
 * the arguments are unsupported or there is nothing to compute).
 */
int mlstm_fwd_kernel_launches(int B, int NH, int S, int DHQK, int DHV, int chunk, mlstm_dtype dt);

/*
 * 1 when mlstm_fwd takes its tensor-core path for these head sizes, chunk and
 * element type (bf16 inputs, DHQK in {64, 128, 256}, DHV a multiple of 128,
 * chunk in {64, 128}), 0 when it takes the fp32 CUDA-core path, -1 when the
 * combination is not supported at all.  No GPU work; a host-side query.
 */
int mlstm_fwd_tensor_path(int DHQK, int DHV, int chunk, mlstm_dtype dt);

/*
 * 1 when mlstm_fwd's tensor-core path runs its in-segment walk as CTA pairs
 * (tcgen05 .cta_group::2: two CTAs share each chunk's S = Q K^T, P and the passes
 * over q and k, 256 value columns per pair; DHQK 256, DHV a multiple of 256,
 * chunk 128), 0 when the walk runs one CTA per 128 value columns, -1 when the
 * combination does not take the tensor-core path.  No GPU work; a host-side query.
 */
int mlstm_fwd_paired_walk(int DHQK, int DHV, int chunk, mlstm_dtype dt);

/*
 * Segments per head that mlstm_fwd's tensor-core path cuts the sequence into for
 * this shape (each segment's contribution is one long GEMM; the walk runs one
 * CTA per segment and 128 value columns), or 0 when the shape does not take the
 * tensor-core path or has no tokens.  No GPU work; a host-side query.
 */
int mlstm_fwd_segments(int B, int NH, int S, int DHQK, int DHV, int chunk, mlstm_dtype dt);

/*
 * Reports whether the last mlstm_fwd (or mlstm_bwd) that used `workspace` ran
 * to completion: synchronizes `stream`, reads the status word kept in the
 * workspace and returns MLSTM_OK or MLSTM_ERR_TIMEOUT (a bounded device-side
 * wait gave up; the outputs of that call are then undefined).
 */
mlstm_status mlstm_fwd_status(const void *workspace, void *stream);

/*
 * Self-test of the failure detection above (no counterpart in the pages): one
 * CTA waits, through the kernels' own bounded wait, on a barrier that nothing
 * completes; after the wait limit (2 s) it records a timeout in the status word
 * of `workspace` (a workspace of mlstm_fwd, 256-byte aligned, device) and exits.
 * A following mlstm_fwd_status on that workspace returns MLSTM_ERR_TIMEOUT, and
 * the GPU context stays usable (the next mlstm_fwd with the workspace resets
 * the word).  Asynchronous on `stream`.  Errors: MLSTM_ERR_INVALID_ARG for a
 * NULL or misaligned workspace, MLSTM_ERR_CUDA for a launch failure.
 */
mlstm_status mlstm_selftest_wait_timeout(void *workspace, void *stream);

/*
 * One recurrent decode step for every (b, h): reads the state (C, n, m),
 * applies one token and writes the new state back IN PLACE, plus h_out
 * [B][NH][DHV].  Token inputs: q, k [B][NH][DHQK] and v, ogate [B][NH][DHV]
 * in `dt`; igate, fgate [B][NH] float32.  Supported: DHQK multiple of 8 in
 * [8, 512], DHV multiple of 4 in [4, 1024].
 *
 * The source defining the operation: the guide's "Recurrent Formulation
 * (Inference Mode)", applied once.
 */
mlstm_status mlstm_step(float *C, float *n, float *m,
                        const void *q, const void *k, const void *v,
                        const float *igate, const float *fgate, const void *ogate,
                        mlstm_dtype dt, int B, int NH, int DHQK, int DHV,
                        void *h_out, void *stream);

/*
 * Backward pass of mlstm_fwd (from the zero state): the gradients of a loss
 * L = sum over b, h, t, j of dh[b][h][t][j] * h[b][h][t][j] with respect to
 * every input, the training form of the guide's "The Dual Formulation: How
 * mLSTM Enables Parallel GPU Training" and "Exploit Chunkwise Hardware Kernels
 * for Production Training".  The stabilizer m carries no gradient (h does not
 * depend on it); at the denominator's max the derivative follows the branch
 * the forward pass took.
 *
 * Inputs as for mlstm_fwd plus dh [B][NH][S][DHV] (type `dt`).  Outputs (device,
 * 16-byte aligned, caller-owned): dq, dk [B][NH][S][DHQK] and dv [B][NH][S][DHV]
 * in `dt`; digate, dfgate [B][NH][S] float32 (gradients of the pre-activations
 * i~, f~); dogate [B][NH][S][DHV] in `dt` when ogate is non-NULL (required
 * then; ignored when ogate is NULL).  No gradient flows into or out of the
 * states: the sequence starts from the zero state and the final state is not
 * part of L.  The forward pass is recomputed inside (gate preprocessing and
 * the chunk-start states).  When mlstm_bwd_tensor_path says so, the products
 * (the chunk-start states' contributions, the read-out numerator and its state
 * gradient, dq, dk and dv) run on the tensor cores (tcgen05, fp32
 * accumulation; bf16 operands, where an operand is an fp32 intermediate that
 * the result is sensitive to, as two bf16 parts, value and rounding residue)
 * and the scores, dS and the scans in fp32 on the CUDA cores; otherwise every
 * step runs in fp32 on the CUDA cores.  Shapes and chunk sizes as for
 * mlstm_fwd.  The forget-gate gradient of token j sums the terms of the token
 * pairs s < j <= t (those whose decay includes f_j) themselves, in four
 * disjoint groups (pairs inside j's chunk, pairs with one token in it, pairs
 * that skip it), rather than as a difference of cumulative sums in which all
 * other pairs cancel: strongly forgetting gates keep its accuracy.
 *
 * workspace: at least mlstm_bwd_workspace_size() bytes, 256-byte aligned
 * (it holds the chunk-start states and their gradients and the chunk's scores:
 * 8 DHQK (DHV + 1) + 8 chunk^2 + 16 bytes per chunk and head, plus 4 DHV +
 * 12 ceil(DHQK / 32) + 4 ceil(DHV / 64) + 24 bytes per token and head; on the
 * tensor-core path, where the chunk-start states, the scores and g are kept
 * as bf16 parts instead of fp32, 6 DHQK DHV + DHQK DHV / 512 + 8 DHQK +
 * 6 chunk^2 + 12 bytes per chunk and head, plus 4 DHQK + 8 DHV + 12 ceil(DHQK / 32) +
 * 4 ceil(DHV / 64) + 24 bytes per token and head; each array 256-byte
 * aligned).  A bounded
 * device-side wait of the tensor-core products that gives up records a
 * timeout that mlstm_fwd_status reads from this workspace.  Errors as for
 * mlstm_fwd.
 */
size_t mlstm_bwd_workspace_size(int B, int NH, int S, int DHQK, int DHV, int chunk, mlstm_dtype dt);

/*
 * 1 when mlstm_bwd runs its dq, dk and dv products on the tensor cores for
 * these head sizes, chunk and element type (bf16 inputs, chunk 64 or 128,
 * DHQK and DHV multiples of 128), 0 when it runs them on the CUDA cores, -1
 * when the combination is not supported at all.  No GPU work; a host-side
 * query.
 */
int mlstm_bwd_tensor_path(int DHQK, int DHV, int chunk, mlstm_dtype dt);
mlstm_status mlstm_bwd(const void *q, const void *k, const void *v,
                       const float *igate, const float *fgate, const void *ogate, const void *dh,
                       mlstm_dtype dt, int B, int NH, int S, int DHQK, int DHV, int chunk,
                       void *dq, void *dk, void *dv, float *digate, float *dfgate, void *dogate,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * mlstm_fwd for callers that cannot allocate device memory.  The pages have no
 * counterpart to this entry point; it exists for callers that may not call
 * cudaMalloc or any allocating routine: code running inside a host framework
 * that owns all device memory and hands out no scratch space (plugin and
 * extension interfaces), and latency-critical paths where an allocation's
 * implicit device synchronization is not acceptable.
 *
 * Same arguments, results and conventions as mlstm_fwd, without the workspace:
 * the scratch memory comes from one device array of MLSTM_FWD_NOALLOC_MAX_BYTES
 * built into the library.  That array exists on every GPU that loads the
 * library and stays allocated until the process exits.  This entry point
 * allocates nothing (no cudaMalloc, no cudaFree, no allocating library call).
 *
 * - Its first call on a device looks up the array's device address on that
 *   device (cudaGetSymbolAddress); make that first call before any stream
 *   capture.  The address is cached per device together with the identity of
 *   the device's context; after that context is destroyed (cudaDeviceReset) the
 *   next call looks the address up again, so make that call before a capture
 *   too.
 * - Shapes whose mlstm_fwd_workspace_size() exceeds MLSTM_FWD_NOALLOC_MAX_BYTES
 *   are rejected with MLSTM_ERR_WORKSPACE before anything is enqueued;
 *   unsupported shapes return MLSTM_ERR_UNSUPPORTED as with mlstm_fwd.
 * - Every call on a device shares the one array, and it keeps the contents of
 *   the last call (each call clears the part that must start at zero).  Calls
 *   whose work overlaps on the GPU (other streams, other host threads) race on
 *   the array: serialize them.
 * - The status word that mlstm_fwd_status reads lives at the start of the
 *   shared array: mlstm_fwd_noalloc_status() reads it.
 */
#define MLSTM_FWD_NOALLOC_MAX_BYTES (32u * 1024u * 1024u)
mlstm_status mlstm_fwd_noalloc(const void *q, const void *k, const void *v,
                               const float *igate, const float *fgate, const void *ogate,
                               mlstm_dtype dt, int B, int NH, int S, int DHQK, int DHV, int chunk,
                               void *h_out, float *C_final, float *n_final, float *m_final,
                               void *stream);

/*
 * Reports whether the last mlstm_fwd_noalloc on the current device ran to
 * completion, like mlstm_fwd_status for a caller's workspace: synchronizes
 * `stream`, reads the status word at the start of the built-in scratch array
 * and returns MLSTM_OK or MLSTM_ERR_TIMEOUT (a bounded device-side wait gave
 * up; the outputs of that call are then undefined).  Allocates nothing.  A
 * later mlstm_fwd_noalloc on the same device resets the word, and calls that
 * overlap on the GPU share it.  MLSTM_ERR_CUDA when the array's address cannot
 * be looked up or the stream fails.  The pages have no counterpart.
 */
mlstm_status mlstm_fwd_noalloc_status(void *stream);

/* Static English text for a status code. */
const char *mlstm_status_string(mlstm_status s);

#ifdef __cplusplus
}
#endif

#endif /* MLSTM_H */

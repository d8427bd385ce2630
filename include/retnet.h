/*
 * retnet.h -- C ABI of the B200 (sm_100a) multi-scale retention library.
 *
 * The operation is RetNet's retention: a linear recurrence with exponential
 * decay that can be evaluated in a parallel, a recurrent (O(1) per token,
 * no KV cache) and a chunkwise form (parallel inside a chunk, a recurrent
 * state passed between chunks), with a per-head decay gamma, xPos-like
 * relative positions, and a swish gate plus GroupNorm on the output
 * ("Retentive Network: A Successor to Transformer for Large Language
 * Models", research summary page, sections "Summary" and "Key points").
 *
 * For one head with decay g, row vectors q_t, k_t (length dk), v_t (dv):
 *   recurrent : S_t = g S_{t-1} + k_t^T v_t ,  o_t = q_t S_t
 *   chunkwise : per chunk of L tokens, local indices i, j,
 *               O = (Q K^T (.) D) V + (Q (.) xi) S_prev,  D_ij = g^(i-j) (i >= j),
 *               xi_i = g^(i+1);  S = g^L S_prev + K^T (V (.) zeta), zeta_j = g^(L-1-j)
 *   rotation  : pairs (2j, 2j+1) of q and k turned by pos * theta_j,
 *               theta_j = 10000^(-2j/dk), pos = pos0 + token index
 *   epilogue  : Y = swish(G) (.) GroupNorm(O), one group per head (dv channels)
 *
 * Conventions for every entry point
 *   - Tensors are caller-owned device memory, densely packed, row-major:
 *       q, k         [batch, seqlen, heads, dk]
 *       v, out, g, y [batch, seqlen, heads, dv]
 *       state        [batch, heads, dk, dv]   always float32
 *     Decode-step tensors drop the seqlen axis: q, k [batch, heads, dk], ...
 *   - Device pointers must be 16-byte aligned.
 *   - Element type: RETNET_F32 (float) or RETNET_BF16 (bfloat16).  Math and
 *     accumulation are float32; outputs take the input element type.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without synchronising.  Argument errors
 *     are detected on the host before anything is enqueued and leave every
 *     buffer untouched.  Faults inside kernels surface at the caller's next
 *     synchronisation, as with any CUDA work.
 *   - The library allocates no device memory in these calls; scratch space
 *     comes from a caller-provided workspace.
 *   - Calls are thread-safe; concurrent calls must not share output or
 *     workspace buffers.
 */
#ifndef RETNET_H
#define RETNET_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define RETNET_API __attribute__((visibility("default")))
#else
#define RETNET_API
#endif

struct CUstream_st;
/* Same type as cudaStream_t. */
typedef struct CUstream_st *retnet_stream_t;

typedef enum retnet_status {
    RETNET_OK = 0,
    RETNET_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or dtype */
    RETNET_ERR_UNSUPPORTED = 2,  /* well-formed request the library does not implement */
    RETNET_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
    RETNET_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up */
    RETNET_ERR_WORKSPACE = 5,    /* workspace missing or smaller than required */
    RETNET_ERR_BOUNDS = 6        /* an index check of the debug build failed */
} retnet_status;

typedef enum retnet_dtype {
    RETNET_F32 = 0,
    RETNET_BF16 = 1
} retnet_dtype;

/* Kernel family for the chunkwise prefill. */
typedef enum retnet_algo {
    RETNET_ALGO_AUTO = 0,    /* tensor-core path where it applies, else SIMT */
    RETNET_ALGO_SIMT = 1,    /* float32 CUDA-core path, any supported shape   */
    RETNET_ALGO_TENSOR = 2   /* tcgen05/TMEM path: bf16, dk = dv = 256         */
} retnet_algo;

typedef struct retnet_shape {
    int batch;       /* >= 0 */
    int heads;       /* 1 .. 256 */
    int seqlen;      /* >= 0 tokens */
    int dk;          /* key/query head dimension: 64, 128 or 256 */
    int dv;          /* value head dimension: 64, 128 or 256 */
    retnet_dtype dtype;
} retnet_shape;

/* Optional output epilogue Y = swish(G) (.) GroupNorm(O).
 * g: [batch, seqlen, heads, dv] device tensor of the prefill's dtype.
 * weight, bias: device float32 [heads * dv] affine (NULL = 1 and 0).
 * eps: added to the biased variance (for example 1e-5). */
typedef struct retnet_gate {
    const void *g;
    const float *weight;
    const float *bias;
    float eps;
} retnet_gate;

/* Human-readable name of a status code (static string, never NULL). */
RETNET_API const char *retnet_status_string(retnet_status status);

/* Number of kernels this library has launched in this process (all
 * devices, all threads).  Used to count launches inside a timed region. */
RETNET_API unsigned long long retnet_kernel_launch_count(void);

/* Launch overlap (process-wide, on by default).  When enabled, the
 * tensor-core prefill kernels and the decode step are launched with
 * programmatic stream serialisation: each is launched as the CTAs of the
 * kernel before it on the stream exit, so its launch and set-up (barriers,
 * tensor memory, descriptor prefetch) overlap that kernel's tail, and it
 * waits for that kernel to complete before touching global memory.
 * Results are identical either way; only the gaps between kernels change.
 * enable: 0 or 1, else INVALID_ARG. */
RETNET_API retnet_status retnet_set_launch_overlap(int enable);

/* How the tensor-core prefill's output pass runs (process-wide).
 *   0 (default): every CTA works alone;
 *   1: chunks of 256 tokens or more run on pairs of CTAs whose tensor
 *     cores act as one (each CTA loads half of every key, value and state
 *     tile), and the pair rotates and decay-scales q itself, so the prep
 *     pass writes only the folded keys;
 *   2: CTA pairs as in 1, with q folded by the prep pass.
 * Chunk 128 (and the shorter chunks computed as 128) always runs on single
 * CTAs.  Results agree to rounding; only the speed changes.
 * mode: 0, 1 or 2, else INVALID_ARG. */
RETNET_API retnet_status retnet_set_output_pairing(int mode);

/* Per-head decay constants gamma_h = 1 - 2^(-5-h), h = 0..heads-1, written
 * to the HOST array gammas[heads] ("Key points": gamma = 1 - 2^(-5-i)).
 * Errors: INVALID_ARG if gammas is NULL or heads is outside 1..256. */
RETNET_API retnet_status retnet_default_gammas(int heads, float *gammas);

/* xPos-like rotation prologue ("Summary": positions encoded similarly to
 * xPos).  y[b, t, h, :] = rotation of x[b, t, h, :] by (pos0 + t) * theta_j
 * on each adjacent pair (2j, 2j+1).  x and y are [batch, seqlen, heads, d]
 * device tensors of `dtype`; y == x (in place) is allowed, any other
 * overlap is not.  d must be a multiple of 8 and at most 1024; pos0 >= 0.
 * Angles are reduced in float64 before a float32 sine/cosine. */
RETNET_API retnet_status retnet_xpos_rotate(const void *x, void *y, int batch, int seqlen, int heads,
                                 int d, retnet_dtype dtype, long long pos0,
                                 retnet_stream_t stream);

/* Bytes of device workspace retnet_retention_chunkwise needs for this shape,
 * chunk length and algorithm (RETNET_ALGO_AUTO resolves as the call would).
 * Errors: as retnet_retention_chunkwise's shape checks. */
RETNET_API retnet_status retnet_chunkwise_workspace_size(const retnet_shape *shape, int chunk,
                                              retnet_algo algo, size_t *bytes);

/* Chunkwise-recurrent prefill ("Summary": computes in parallel within a
 * chunk and passes the recurrent state between chunks; "Key points": cost
 * O(d n (b + h)) with chunk b).
 *   q, k, v    device inputs (layouts above); not modified.
 *   gammas     HOST float array [heads]: the per-head decay, each in [0, 1].
 *   chunk      chunk length b, 1..1024; seqlen need not be a multiple
 *              (the last chunk is then shorter).  The tensor path takes
 *              chunk in {128, 256, 512, 1024} as given, and any chunk below
 *              128 by computing with 128-token chunks: the outputs and the
 *              final state of the chunkwise form do not depend on the chunk
 *              length, so this changes the rounding order only.
 *   out        device output [batch, seqlen, heads, dv]: O, or Y when `gate`
 *              is given.  Must not overlap q, k, v, the gate input, the
 *              states or the workspace.
 *   pos0       position of token 0 for the rotation (split prefills pass
 *              the number of tokens already consumed).
 *   rotate     1: rotate q and k by position first; 0: use them as given.
 *   state_in   device float32 [batch, heads, dk, dv] state before token 0,
 *              or NULL for a zero state.
 *   state_out  device float32 [batch, heads, dk, dv] state after the last
 *              token, or NULL.  May equal state_in.
 *   gate       optional epilogue (NULL: out = O).
 *   algo       kernel family, see retnet_algo.
 *   workspace  device scratch of at least retnet_chunkwise_workspace_size()
 *              bytes, 256-byte aligned; contents on entry are ignored.
 * Errors: INVALID_ARG (null or misaligned pointers, sizes out of range,
 * gamma outside [0,1]), UNSUPPORTED (dk/dv not in {64,128,256}, or a tensor
 * path request it cannot serve), WORKSPACE, CUDA. */
RETNET_API retnet_status retnet_retention_chunkwise(const void *q, const void *k, const void *v,
                                         const float *gammas, int chunk, void *out,
                                         const retnet_shape *shape, long long pos0, int rotate,
                                         const float *state_in, float *state_out,
                                         const retnet_gate *gate, retnet_algo algo,
                                         void *workspace, size_t workspace_bytes,
                                         retnet_stream_t stream);

/* ---- Parallel form ------------------------------------------------------
 * The parallel (training) form over the whole sequence ("Summary": the
 * parallel representation computes all tokens at once):
 *   out[b, t, h, :] = sum_{m <= t} gamma_h^(t-m) (R q_t . R k_m) v_m,
 * then swish(G) (.) GroupNorm when `gate` is given, with R the rotation of
 * retnet_retention_chunkwise.  O(n^2) work per sequence-head; the initial
 * state is zero and no state is returned.  Tensor-core kernels only: bf16,
 * dk = dv = 256, and every decay must satisfy 128 * log2(1/gamma) <= 100
 * (gamma >= 0.58); other requests return UNSUPPORTED.  Arguments as for
 * retnet_retention_chunkwise; workspace: retnet_parallel_workspace_size()
 * bytes, 1024-byte aligned.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
RETNET_API retnet_status retnet_parallel_workspace_size(const retnet_shape *shape, size_t *bytes);
RETNET_API retnet_status retnet_retention_parallel(const void *q, const void *k, const void *v,
                                        const float *gammas, void *out,
                                        const retnet_shape *shape, long long pos0, int rotate,
                                        const retnet_gate *gate, void *workspace,
                                        size_t workspace_bytes, retnet_stream_t stream);

/* ---- Prefill without any allocation ---------------------------------
 * No counterpart on the pages: an addition for callers that cannot
 * allocate device memory at run time -- for example a plugin inside a
 * serving process that reserves all device memory at start-up and hands
 * its plugins no allocator, or a latency-critical path where cudaMalloc's
 * implicit device-wide synchronisation is not allowed.  It runs exactly the
 * kernels of retnet_retention_chunkwise (same arguments and semantics, minus
 * the workspace) on a scratch array compiled into the library:
 *   - at most RETNET_NOALLOC_SCRATCH_BYTES of scratch per call; a call that
 *     would need more (see retnet_chunkwise_workspace_size for the chosen
 *     kernel family) returns RETNET_ERR_WORKSPACE and enqueues nothing;
 *   - every GPU that loads the library holds that array until exit;
 *   - it calls no cudaMalloc, cudaFree or other allocating routine;
 *   - it works on the current device (`stream` must belong to it).  Its
 *     first call in a CUDA context (the first on each device, and the first
 *     after a cudaDeviceReset) looks up the array's device address there
 *     (cudaGetSymbolAddress); make that first call before any stream
 *     capture on that device;
 *   - all calls on a device share the one array and it keeps the last
 *     call's contents (nothing in it needs to start at zero): calls whose
 *     work overlaps on the GPU (different streams, no ordering) race on it
 *     and must be serialised by the caller. */
#define RETNET_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
RETNET_API retnet_status retnet_retention_chunkwise_noalloc(
    const void *q, const void *k, const void *v, const float *gammas, int chunk, void *out,
    const retnet_shape *shape, long long pos0, int rotate, const float *state_in,
    float *state_out, const retnet_gate *gate, retnet_algo algo, retnet_stream_t stream);

/* One recurrent decode step for every (sequence, head) ("Summary": the
 * recurrent form costs O(1) per step and needs no KV cache).
 *   q, k [batch, heads, dk], v [batch, heads, dv]: this token, device, dtype.
 *   gammas   HOST float array [heads].
 *   state    device float32 [batch, heads, dk, dv], updated in place:
 *            S <- gamma S + k^T v.
 *   out      device [batch, heads, dv]: o = q S (after the update).  Must
 *            not overlap q, k, v or state (every CTA reads the whole q, k
 *            rows while others write their columns of out).
 *   pos      rotation position of this token (prefill length + steps done).
 *   rotate   1: rotate q and k by pos first; 0: use them as given.
 * Errors: INVALID_ARG, UNSUPPORTED (dk/dv not in {64,128,256}), CUDA. */
RETNET_API retnet_status retnet_retention_step(const void *q, const void *k, const void *v,
                                    const float *gammas, float *state, void *out,
                                    int batch, int heads, int dk, int dv, retnet_dtype dtype,
                                    long long pos, int rotate, retnet_stream_t stream);

/* ---- Backward pass (training) ------------------------------------------
 * Gradients of the prefill without epilogue and without initial state
 * ("Summary": the parallel form is the training form; the chunkwise form
 * computes it in chunks): for O = retention(R q, R k, v) as
 * retnet_retention_chunkwise returns it with gate = NULL and
 * state_in = NULL, and d_out = dL/dO, writes dq = dL/dq, dk, dv.
 * With A = QK^T (.) D and dA = (dO V^T) (.) D on the rotated Q, K:
 *     dV = A^T dO,   dQ = R^T (dA K),   dK = R^T (dA^T Q).
 * dQ is itself a causal retention of (dO, V, K); dK and dV are causal
 * retentions of time-reversed sequences, so the pass runs three forward
 * chunkwise retentions (tensor-core path when the shape admits it, else
 * SIMT, as for the forward call) between reorder/rotate passes.
 *   q, k [B, n, H, dk], v, d_out, dv [B, n, H, dv], dq, dk [B, n, H, dk]:
 *            device, shape->dtype, distinct from each other.
 *   chunk, algo: as for retnet_retention_chunkwise (each of the two
 *            forward shapes, (dv, dk) and (dk, dv), must admit the algo).
 *   workspace: retnet_backward_workspace_size() bytes, 1024-byte aligned.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
RETNET_API retnet_status retnet_backward_workspace_size(const retnet_shape *shape, int chunk,
                                             retnet_algo algo, size_t *bytes);
RETNET_API retnet_status retnet_retention_backward(const void *q, const void *k, const void *v,
                                        const void *d_out, const float *gammas, int chunk,
                                        void *dq, void *dk, void *dv,
                                        const retnet_shape *shape, long long pos0, int rotate,
                                        retnet_algo algo, void *workspace,
                                        size_t workspace_bytes, retnet_stream_t stream);

/* Recurrent form over a run of tokens: multi-token decode, or continuing
 * every sequence by a short chunk ("Summary": the recurrent form; the
 * chunkwise form "passes the recurrent state between chunks").  For
 * t = 0 .. seqlen-1 and every (sequence, head):
 *     S <- gamma S + k_t^T v_t ;  o_t = q_t S,
 * with q_t, k_t rotated by pos0 + t when rotate = 1.  Bit-identical to
 * seqlen calls of retnet_retention_step at positions pos0, pos0 + 1, ...,
 * but the state is read and written once per call instead of per token.
 *   q, k  device [batch, seqlen, heads, dk]; v, out [batch, seqlen, heads, dv]
 *         (shape->dtype; out receives every o_t and must not overlap q, k,
 *         v or state).
 *   state device float32 [batch, heads, dk, dv], updated in place to the
 *         state after the last token.
 * Work grows with seqlen on CUDA cores (4 dk dv flops per head-token); for
 * long runs use retnet_retention_chunkwise with state_in.
 * Errors: INVALID_ARG, UNSUPPORTED (dk/dv not in {64,128,256}), CUDA. */
RETNET_API retnet_status retnet_retention_recurrent(const void *q, const void *k, const void *v,
                                         const float *gammas, float *state, void *out,
                                         const retnet_shape *shape, long long pos0, int rotate,
                                         retnet_stream_t stream);

/* Output epilogue Y = swish(G) (.) GroupNorm(O) ("Summary": a swish gate
 * and GroupNorm are added).  o, g, y: device [rows, heads, dv] of `dtype`
 * (rows = batch * seqlen); one group per (row, head) over its dv channels,
 * biased variance, then the per-channel affine weight/bias (device float32
 * [heads * dv], NULL = 1 / 0), times swish(g) = g * sigmoid(g).
 * y may equal o.  dv must be a multiple of 8 and at most 1024. */
RETNET_API retnet_status retnet_groupnorm_swish(const void *o, const void *g, const float *weight,
                                     const float *bias, float eps, long long rows, int heads,
                                     int dv, retnet_dtype dtype, void *y,
                                     retnet_stream_t stream);

/* ---- The multi-scale retention layer ----------------------------------
 * Retention replaces multi-head attention, with a swish gate and GroupNorm
 * added on its output ("Summary"); around the operator the layer projects
 * its input and output with dense weights.  Both projections run on a
 * tcgen05 GEMM of this library (TMA-fed, bf16 operands, float32
 * accumulation, bf16 result).
 *
 * retnet_linear: y[r, :] = x[r, :] W^T for r < rows.
 *   x  device bf16 [rows, in_features]; w device bf16 [out_features,
 *      in_features] (a linear layer's weight layout); y device bf16
 *      [rows, out_features], not overlapping x or w.
 *   in_features must be a multiple of 64 and out_features of 256, else
 *   UNSUPPORTED.  Errors: INVALID_ARG (null or misaligned pointers,
 *   negative sizes), UNSUPPORTED, CUDA. */
RETNET_API retnet_status retnet_linear(const void *x, const void *w, void *y, long long rows,
                                       int in_features, int out_features,
                                       retnet_stream_t stream);

/* retnet_msr_layer: for x [batch, seqlen, hidden] (bf16, shape->dtype must
 * be RETNET_BF16 and dk = dv = d):
 *     q, k, v, g = x W_Q^T, x W_K^T, x W_V^T, x W_G^T      ([B, n, H, d] each)
 *     o = swish(g) (.) GroupNorm(retention(R q, R k, v))     (as
 *         retnet_retention_chunkwise with this gate, chunk, pos0, rotate = 1,
 *         state_in, state_out and algo AUTO)
 *     y = o W_O^T                                          ([B, n, hidden])
 *   w_qkvg  device bf16 [4 H d, hidden]: the rows of W_Q, then W_K, W_V, W_G.
 *   w_o     device bf16 [hidden, H d].
 *   gn_weight, gn_bias  device float32 [H d] GroupNorm affine, or NULL.
 *   workspace  retnet_msr_workspace_size() bytes, 1024-byte aligned.
 *   hidden must be a multiple of 256 and H d a multiple of 256, else
 *   UNSUPPORTED.  y must not overlap x, the weights, the states or the
 *   workspace.
 *   When the retention takes the tensor-core path (d = 256, chunks up to
 *   1024, decays that admit the fold), the projection's epilogue applies R
 *   and the decay fold to q and k and writes them as the prefill's operands,
 *   so q and k are never stored unrotated; the result matches the
 *   definition above to rounding (q and k are not rounded to bf16 before
 *   the rotation).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
RETNET_API retnet_status retnet_msr_workspace_size(const retnet_shape *shape, int hidden,
                                                   int chunk, size_t *bytes);
RETNET_API retnet_status retnet_msr_layer(const void *x, const void *w_qkvg, const void *w_o,
                                          const float *gammas, int chunk, void *y,
                                          const retnet_shape *shape, int hidden,
                                          long long pos0, const float *gn_weight,
                                          const float *gn_bias, float eps,
                                          const float *state_in, float *state_out,
                                          void *workspace, size_t workspace_bytes,
                                          retnet_stream_t stream);

/* Reads and clears the library's device-side error word on the current
 * device after synchronising `stream`.  Returns RETNET_OK when no kernel
 * reported a problem, RETNET_ERR_TIMEOUT when a bounded wait inside a
 * kernel gave up (its results are then invalid; the kernel let its own
 * copies and MMAs finish, freed its tensor memory and returned, so the
 * context stays usable), RETNET_ERR_BOUNDS when an index check of the debug
 * build (RETNET_CHECK_BOUNDS) failed and the access was skipped, and
 * RETNET_ERR_CUDA when the read itself failed. */
RETNET_API retnet_status retnet_check_device_errors(retnet_stream_t stream);

#ifdef RETNET_TEST_HOOKS
/* Debug build only (compiled with RETNET_TEST_HOOKS; absent from the
 * default library).  No counterpart on the pages: a way to exercise the
 * timeout path without a GPU fault.  Sets, for the tensor-core prefill
 * kernels on the current device, the wall-time limit of every pipeline
 * wait (wait_limit_ns > 0; the default build uses about 2 s), and whether
 * the state pass's first CTA skips its first TMA load (skip = 1), so that
 * its MMA warp's wait runs out and the CTA takes the timeout path.
 * Errors: INVALID_ARG, CUDA. */
RETNET_API retnet_status retnet_test_set_hooks(unsigned long long wait_limit_ns,
                                               int skip_first_state_load);
/* Debug build only: synchronises `stream` and returns in *word the raw
 * device error word (bit 0 timeout, bit 1 index check, and one bit per
 * kernel whose index check failed: 1<<8 prep, 1<<9 state, 1<<10 output,
 * 1<<11 paired output, 1<<12 decode, 1<<13 projection GEMM), clearing it.
 * Errors: INVALID_ARG, CUDA. */
RETNET_API retnet_status retnet_test_error_word(retnet_stream_t stream, unsigned *word);
#endif

/* ---- Kernel timer (diagnostics; off by default) ----------------------
 * While enabled, every kernel this library launches is bracketed by CUDA
 * events on its own stream, and per-kernel totals accumulate until reset.
 * Adds a few microseconds of host work per launch.  Launches made while the
 * stream is being captured into a CUDA graph get event-record nodes in the
 * graph: the next read or reset after the graph has run reports the times
 * of its most recent replay.  Those events stay allocated (one pair per
 * captured launch) for as long as the graph may run. */
RETNET_API retnet_status retnet_profiler_enable(int on);
/* Restricts the timer to the kernel named `name` (a NUL-terminated string
 * the library copies; one of the names retnet_profiler_read reports), or
 * lifts the restriction when `name` is NULL.  Timing one kernel keeps the
 * events' own cost out of the other kernels' boundaries. */
RETNET_API retnet_status retnet_profiler_select(const char *name);
/* Drops accumulated totals (waits for pending events first). */
RETNET_API retnet_status retnet_profiler_reset(void);
/* Totals of the index-th kernel name (0-based, sorted by name): copies the
 * name (NUL-terminated, truncated to name_len) and writes the summed device
 * milliseconds and the launch count.  Waits for pending events.
 * Returns INVALID_ARG past the last index or for NULL outputs. */
RETNET_API retnet_status retnet_profiler_read(int index, char *name, size_t name_len,
                                              double *total_ms, unsigned long long *launches);

#ifdef __cplusplus
}
#endif

#endif /* RETNET_H */

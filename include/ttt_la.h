/*
 * ttt_la.h -- C ABI of the causal TTT / linear-attention layer for B200 (sm_100a).
 *
 * The layer (from "Test-Time Training with KV Binding Is Secretly Linear
 * Attention", Liu et al.; Table 2 of the thelatestinai.com listing, Variants
 * 3-5, and the kualia.ai explainer, section "The Linear Attention
 * Equivalence"): per sequence and head, a fast weight W (d_v x d_k, fp32)
 * takes one gradient step per token on the key-value binding loss
 * L_t(W) = -sigma v_t^T W k_t, then reads out o_t = W_t q_t:
 *
 *   no momentum (beta == 0):  W_t = W_{t-1} + sigma * eta_t * v_t k_t^T
 *   SGD momentum (beta != 0): M_t = beta M_{t-1} - sigma * v_t k_t^T
 *                             W_t = W_{t-1} - eta_t * M_t
 *   o_t = W_t q_t                      (update first, then read)
 *
 * sigma = +1 (descent) or -1 (gradient ascent, Table 1 of the same listing).
 * M is the momentum buffer of gradients.  The fast weights reset for every
 * sequence (explainer "Test Time Training", wpnews.pro): state_in == NULL
 * means W_0 = 0 (and M_0 = 0).
 *
 * Three computations of the same layer:
 *   ttt_la_forward_chunked   chunk-parallel form ("fully parallel
 *                            formulations", abstract): intra-chunk causal
 *                            (Q K^T * coefficients) V plus the carried state,
 *                            on the tensor cores (bf16 inputs) or in fp32 FMA
 *                            (fp32 inputs).
 *   ttt_la_forward_recurrent token-by-token recurrence ("Recurrent Impl.",
 *                            Table 2).
 *   ttt_la_decode_step       one token for N sequences, state updated in place.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers, row-major and contiguous, 16-byte
 *    aligned.  q, k: [B,H,T,d_k]; v, o: [B,H,T,d_v]; eta: [B,H,T] fp32;
 *    state / momentum: [B,H,d_v,d_k] fp32 (row n of W holds the weights that
 *    produce output feature n).  dtype applies to q, k, v and o together.
 *  - The caller owns every buffer; the library allocates no device memory.
 *    Scratch for the chunked path is the caller's `workspace`
 *    (ttt_la_workspace_size bytes).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  Argument errors are detected on the host before any
 *    launch and return TTT_LA_ERR_INVALID_ARG / TTT_LA_ERR_UNSUPPORTED with
 *    nothing launched.  A failed launch returns TTT_LA_ERR_CUDA.
 *  - Every in-kernel wait is bounded in time.  A wait that runs out records
 *    TTT_LA_ERR_TIMEOUT in the library's device status word, the kernel
 *    drains its own copies, frees its tensor memory and returns;
 *    ttt_la_get_last_device_status reads (and clears) that word.
 *  - The chunked forward splits long sequences into segments whose blocks
 *    exchange segment states through the workspace.  Where the blocks of a
 *    head wait for one another (ttt_la_chunked_plan reports it as
 *    `cooperative`), the kernel is launched cooperatively: every block of the
 *    grid is then resident at once, or the launch fails with
 *    TTT_LA_ERR_CUDA.  Elsewhere a block only waits for blocks that started
 *    before it.  Every wait is still bounded (ttt_la_set_wait_limit_ns,
 *    default 1 s); a wait that runs out is reported through the device status
 *    word, not by the call's return value, so callers that must know check
 *    ttt_la_get_last_device_status after the work.
 *  - o must not alias q, k, v, eta or the states.  state_out may equal
 *    state_in (in place), and mom_out may equal mom_in.
 */
#ifndef TTT_LA_H
#define TTT_LA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TTT_LA_API __attribute__((visibility("default")))
#else
#define TTT_LA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TTT_LA_OK = 0,
  TTT_LA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, short workspace */
  TTT_LA_ERR_UNSUPPORTED = 2,  /* valid but not built: (d_k, d_v, chunk, dtype) combination */
  TTT_LA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  TTT_LA_ERR_TIMEOUT = 4,      /* a bounded in-kernel wait ran out (device status word) */
  TTT_LA_ERR_SCRATCH_LIMIT = 5, /* ttt_la_forward_chunked_noalloc: scratch need exceeds its fixed array */
  TTT_LA_ERR_DEVICE_CHECK = 6   /* debug builds: a device-side bounds check failed (device status word) */
} ttt_la_status;

typedef enum { TTT_LA_F32 = 0, TTT_LA_BF16 = 1 } ttt_la_dtype;

/* Arguments of a whole-sequence forward (chunked or recurrent). */
typedef struct ttt_la_args {
  int32_t B, H, T;          /* batch, heads, tokens (T >= 1, any value) */
  int32_t d_k, d_v;         /* head dims */
  int32_t dtype;            /* ttt_la_dtype of q, k, v, o */
  const void *q, *k, *v;    /* [B,H,T,d_k], [B,H,T,d_k], [B,H,T,d_v] */
  const float *eta;         /* [B,H,T] per-token learning rate, or NULL -> eta_const */
  float eta_const;          /* learning rate when eta == NULL */
  float beta;               /* SGD momentum; 0 -> plain SGD (momentum buffers unused) */
  int32_t ascent;           /* 0: gradient descent (sigma=+1); 1: ascent (sigma=-1) */
  int32_t chunk;            /* chunked path: tokens per chunk (64 or 128); ignored otherwise */
  int32_t segments;         /* chunked path: sequence segments per (b,h) run in parallel;
                               0 = automatic (fill the SMs in one wave); ignored otherwise */
  const float *state_in;    /* [B,H,d_v,d_k] W_0, or NULL -> zeros */
  float *state_out;         /* [B,H,d_v,d_k] W_T, or NULL -> not returned */
  const float *mom_in;      /* [B,H,d_v,d_k] M_0 (momentum only), or NULL -> zeros */
  float *mom_out;           /* [B,H,d_v,d_k] M_T (momentum only), or NULL -> not returned */
  void *o;                  /* [B,H,T,d_v] output, dtype */
  void *workspace;          /* device scratch, >= ttt_la_workspace_size(args) bytes */
  size_t workspace_bytes;
} ttt_la_args;

/* Bytes of caller-provided scratch that ttt_la_forward_chunked needs for
 * these arguments (0 when the call needs none; pointers are not read). */
TTT_LA_API size_t ttt_la_workspace_size(const ttt_la_args *args);

/* Chunk-parallel forward.  Within each chunk of `chunk` tokens the outputs are
 * the causal, coefficient-weighted attention of the chunk's queries on its
 * keys and values plus the read-out of the state carried in from earlier
 * chunks; the state after each chunk is the carried state plus the chunk's
 * weighted V^T K (with momentum, the pair (W, M) follows the affine chunk map
 * W' = W - g M + dW, M' = beta^C M + dM).  bf16 inputs run on the tcgen05
 * tensor cores with fp32 accumulation: d_k == d_v in {64, 128},
 * chunk in {64, 128}.  fp32 inputs run in fp32 FMA: d_k, d_v multiples of 4
 * up to 128, chunk in {16, 32, 64}.  Other combinations: UNSUPPORTED. */
TTT_LA_API ttt_la_status ttt_la_forward_chunked(const ttt_la_args *args, void *stream);

/* How ttt_la_forward_chunked would run these arguments on the current
 * device (no launch; pointers are not read; without a device the figures are
 * those of a 148-SM B200).  Fills *plan and returns TTT_LA_OK, or the status
 * the forward would return for unusable arguments. */
typedef struct ttt_la_plan {
  int32_t path;             /* 0: tensor cores, no momentum; 1: tensor cores with momentum; 2: fp32 FMA */
  int32_t tile;             /* tokens per tensor-core tile (the chunk; 64 with momentum) */
  int32_t segments;         /* blocks per (b,h) sequence (one for the fp32 path) */
  int32_t chunks_per_segment;
  int32_t cooperative;      /* 1: blocks of a head wait for one another: launched cooperatively */
  int32_t blocks;           /* grid size of the forward kernel */
  int32_t resident;         /* blocks of that kernel resident at once on the device */
  int32_t waves;            /* cooperative schedule without momentum: the sequence is cut into
                               `waves` waves of `segments` runs, and phase B of each wave re-reads
                               K and V from L2 (about 512 tokens per run; the environment variable
                               TTT_LA_WAVE_TOKENS overrides that, for tuning); 1 otherwise */
  size_t workspace_bytes;   /* = ttt_la_workspace_size(args) */
} ttt_la_plan;
TTT_LA_API ttt_la_status ttt_la_chunked_plan(const ttt_la_args *args, ttt_la_plan *plan);

/* Token-by-token forward (the recurrence itself): fp32 or bf16 inputs,
 * d_k in {32, 64, 128}, d_v <= 1024; chunk and workspace are ignored. */
TTT_LA_API ttt_la_status ttt_la_forward_recurrent(const ttt_la_args *args, void *stream);

/* One decode step for N independent sequences: for every (n, h)
 * applies the single-token update to state (and mom when beta != 0) IN PLACE
 * and writes o = W q.  q, k: [N,H,d_k]; v, o: [N,H,d_v]; eta: [N,H] or NULL;
 * state, mom: [N,H,d_v,d_k] fp32.  d_k in {32, 64, 128}; memory-bound. */
typedef struct ttt_la_decode_args {
  int32_t N, H, d_k, d_v;
  int32_t dtype;            /* of q, k, v, o */
  const void *q, *k, *v;
  const float *eta;         /* [N,H] or NULL -> eta_const */
  float eta_const, beta;
  int32_t ascent;
  float *state;             /* [N,H,d_v,d_k] fp32, read and written in place */
  float *mom;               /* [N,H,d_v,d_k] fp32 in place; required iff beta != 0 */
  void *o;                  /* [N,H,d_v] */
} ttt_la_decode_args;

TTT_LA_API ttt_la_status ttt_la_decode_step(const ttt_la_decode_args *args, void *stream);

/* Chunked forward for callers that cannot allocate device memory.  Some
 * callers only ever receive their input and output buffers: a plugin running
 * inside another engine's memory plan, or code whose device memory is owned
 * entirely by someone else's pool, has no way to call cudaMalloc (and
 * latency-critical callers avoid it because it can synchronise the device).
 * This variant computes exactly what ttt_la_forward_chunked computes, but its
 * scratch is a fixed array inside the library instead of args->workspace
 * (which is ignored):
 *  - the array holds TTT_LA_STATIC_SCRATCH_BYTES (8 MiB) and lives on every
 *    GPU that loads the library until the process exits;
 *  - a call whose ttt_la_workspace_size(args) exceeds it returns
 *    TTT_LA_ERR_SCRATCH_LIMIT with nothing launched (use the allocating entry
 *    point, or fewer segments, for such shapes);
 *  - the first call on each device looks up the array's device address (with
 *    that device current); make that first call before any stream capture;
 *  - every call on a device shares the one array, and the array keeps the last
 *    call's contents: calls whose executions overlap on the GPU (different
 *    streams, no ordering between them) race on it.  Whatever must start at
 *    zero is cleared by the call itself.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 * The paper has no counterpart of this entry point; it exists for callers. */
#define TTT_LA_STATIC_SCRATCH_BYTES (8u << 20)
TTT_LA_API ttt_la_status ttt_la_forward_chunked_noalloc(const ttt_la_args *args, void *stream);

/* Chunked forward with every tensor in host memory: q, k, v, eta, state_in,
 * mom_in are read from, and o, state_out, mom_out written to, HOST pointers
 * (page-locked memory lets the copies run asynchronously and overlap;
 * pageable memory works but serialises them).  args->workspace is ignored.
 * The B*H sequences are cut into 2 to 8 pieces of whole sequences (about
 * 24 MB of inputs each, at most one piece per sequence); piece j
 * is copied in on an internal stream while piece j-1 runs on `stream` and
 * piece j-2 is copied out on a second internal stream, through two sets of
 * staging buffers in `device_buf` (caller-owned device memory, 16-byte
 * aligned, at least ttt_la_host_staging_size(args) bytes).  Each piece runs
 * ttt_la_forward_chunked, so results agree with it up to the rounding of a
 * different segment split.  Ordering: copies in start as soon as the staging
 * set they fill is free (the last forward that read it has finished, in this
 * call or an earlier one on the device), possibly before earlier work on
 * `stream` has finished, so the host inputs must be final when the call is
 * made; the forwards and copies out follow the work already queued on
 * `stream`, and work queued on it after this call starts only once every
 * output has reached host memory.  Returns once everything is queued (the
 * host inputs must stay valid and unchanged until `stream` passes this call).
 * Calls on one device are ordered with one another through the library's
 * shared copy streams; `device_buf` must not be used by anything else while
 * such a call may still run.
 * Errors: as ttt_la_forward_chunked, plus TTT_LA_ERR_INVALID_ARG for a
 * missing, misaligned or short `device_buf`.  The paper has no counterpart of
 * this entry point; it is the end-to-end path for callers with host data. */
TTT_LA_API size_t ttt_la_host_staging_size(const ttt_la_args *args);
TTT_LA_API ttt_la_status ttt_la_forward_chunked_host(const ttt_la_args *args, void *device_buf,
                                                     size_t device_bytes, void *stream);

/* Splitting one sequence over several devices along T (one exchange step).
 * A run of tokens acts on the carried state as the affine map
 *   (W, M) -> (W - G M + dW, B M + dM),
 * with dW, dM the state the run leaves from W = M = 0, G = sum_t eta_t beta^t
 * (t = 1..L over the run) and B = beta^L ("Test-Time Training with KV Binding
 * Is Secretly Linear Attention", thelatestinai.com listing, Table 2: Variant 3
 * carries (W, M); Variants 4-5 carry W alone, G = 0, B = 1).  A device holding
 * tokens [t0, t1) of every sequence computes its run's map, the maps are
 * exchanged (all-gather), and each device composes the maps of the runs
 * before its own onto W_0, M_0 to get its start state, then calls
 * ttt_la_forward_chunked from it.
 *
 * ttt_la_segment_map: args as for ttt_la_forward_chunked over the device's
 * run (T = its length); state_in/mom_in/state_out/mom_out are ignored and
 * args->o is scratch (written, contents unspecified).  Writes dW
 * [B,H,d_v,d_k] fp32 and, with momentum, dM [B,H,d_v,d_k] fp32 and GB
 * [B,H,2] fp32 = (G, B); dM and GB may be NULL without momentum.  Device
 * pointers, 16-byte aligned.  Errors as ttt_la_forward_chunked.
 *
 * ttt_la_compose_maps: applies maps 0..nmaps-1 in order to (W0, M0) for BH
 * heads: dW, dM [nmaps,BH,d_v,d_k] and GB [nmaps,BH,2] as written by
 * ttt_la_segment_map (dM and GB both NULL: maps without momentum).  W0, M0
 * [BH,d_v,d_k] may be NULL (zeros).  Writes W_out and, if not NULL, M_out
 * [BH,d_v,d_k].  nmaps = 0 copies (W0, M0).  TTT_LA_ERR_INVALID_ARG for bad
 * sizes or exactly one of dM, GB given. */
TTT_LA_API ttt_la_status ttt_la_segment_map(const ttt_la_args *args, float *dW, float *dM, float *GB, void *stream);
TTT_LA_API ttt_la_status ttt_la_compose_maps(int32_t nmaps, int32_t BH, int32_t d_v, int32_t d_k, const float *dW,
                                             const float *dM, const float *GB, const float *W0, const float *M0,
                                             float *W_out, float *M_out, void *stream);

/* Frozen-MLP feature map of the keys and queries (Variants 1-2 of Table 2 in
 * the thelatestinai.com listing: the inner loop updates only the fast-weight
 * network's last layer, so the layers before it are fixed for the sequence
 * and act as the feature map phi of the (phi(Q) phi(K)^T) V form, kualia.ai
 * explainer, section "The Linear Attention Equivalence").  The frozen part is
 * one gated hidden layer of the "GLU Variants Improve Transformer" (SwiGLU)
 * form, applied per token:
 *
 *   phi(x) = silu(W1[h] x) * (W3[h] x),   silu(a) = a / (1 + exp(-a)),
 *
 * with fp32 accumulation and the result rounded to bf16.  The linear fast
 * weight is then trained on phi(k) and read with phi(q): call
 * ttt_la_forward_chunked (or the recurrent / decode forms) with q := phi(q),
 * k := phi(k), d_k := d_out.
 *
 * Fields: x[i], y[i] for i < n_inputs (1 or 2; typically q and k in one
 * launch).  x[i]: [B,H,T,d_in] bf16; y[i]: [B,H,T,d_out] bf16, written;
 * w1, w3: [H,d_out,d_in] bf16 (row o of w1[h] gives hidden unit o), shared by
 * every input.  (d_in, d_out) in {64,128} x {64,128}; other widths return
 * TTT_LA_ERR_UNSUPPORTED.  Device pointers, 16-byte aligned; y[i] must not
 * overlap any x[j] or the weights.  One launch, asynchronous on `stream`;
 * errors as ttt_la_forward_chunked. */
typedef struct ttt_la_feature_args {
  int32_t B, H, T, d_in, d_out;
  int32_t n_inputs;
  const void *x[2];
  void *y[2];
  const void *w1, *w3;
} ttt_la_feature_args;

TTT_LA_API ttt_la_status ttt_la_feature_map(const ttt_la_feature_args *args, void *stream);

/* Backward of the layer (the gradient needed to train it, Figure 4 of the
 * thelatestinai.com listing).  Given the forward's inputs and the upstream
 * gradients dL/do (and optionally dL/dW_T, dL/dM_T on the final states), it
 * writes dL/dq, dL/dk, dL/dv, the per-token dL/deta_t and dL/dW_0, dL/dM_0.
 * Over the tokens in reverse, with G_t = dL/dW_t and H_t = dL/dM_t:
 *   G_t = G_{t+1} + do_t q_t^T (G_{T+1} = dL/dW_T);  dq_t = W_t^T do_t
 *   momentum: H_t = beta H_{t+1} - eta_t G_t (H_T = dL/dM_T - eta_T G_T),
 *             dv_t = -sigma H_t k_t, dk_t = -sigma H_t^T v_t, deta_t = -<G_t, M_t>
 *   plain:    dv_t = sigma eta_t G_t k_t, dk_t = sigma eta_t G_t^T v_t,
 *             deta_t = sigma v_t^T G_t k_t
 *   dW_0 = G_1, dM_0 = beta H_1 (zero without momentum).
 *
 * Fields: the forward's B, H, T, d_k, d_v, dtype, q, k, v, eta, eta_const,
 * beta, ascent, state_in (W_0), mom_in (M_0) exactly as in ttt_la_args.
 * grad_o: [B,H,T,d_v] dtype.  grad_state, grad_mom: [B,H,d_v,d_k] fp32 or
 * NULL (zero).  Outputs: grad_q, grad_k [B,H,T,d_k] and grad_v [B,H,T,d_v]
 * in dtype (required); grad_eta [B,H,T] fp32 (per token, also when eta is
 * NULL: its sum is dL/deta_const), grad_state_in, grad_mom_in [B,H,d_v,d_k]
 * fp32, each optional (NULL: not written).  Device pointers, 16-byte aligned;
 * outputs must not overlap the inputs.  The workspace holds state
 * checkpoints every 32 tokens and one chunk's state history per (b,h):
 * ttt_la_backward_workspace_size bytes.
 *
 * ttt_la_backward_recurrent computes it token by token in fp32 with one
 * block per (b,h).  d_k must be 32, 64 or 128 and d_v at most 512, 256 or 128
 * respectively; other sizes return TTT_LA_ERR_UNSUPPORTED.  Errors as
 * ttt_la_forward_chunked; a workspace smaller than the size query returns
 * TTT_LA_ERR_INVALID_ARG. */
typedef struct ttt_la_grad_args {
  int32_t B, H, T, d_k, d_v;
  int32_t dtype;            /* ttt_la_dtype of q, k, v, grad_o and grad_q/k/v */
  const void *q, *k, *v;
  const float *eta;
  float eta_const, beta;
  int32_t ascent;
  const float *state_in, *mom_in;
  const void *grad_o;
  const float *grad_state, *grad_mom;
  void *grad_q, *grad_k, *grad_v;
  float *grad_eta, *grad_state_in, *grad_mom_in;
  void *workspace;
  size_t workspace_bytes;
} ttt_la_grad_args;

TTT_LA_API size_t ttt_la_backward_workspace_size(const ttt_la_grad_args *args);
TTT_LA_API ttt_la_status ttt_la_backward_recurrent(const ttt_la_grad_args *args, void *stream);

/* Chunk-parallel backward of the layer: the same gradients as
 * ttt_la_backward_recurrent ("Test-Time Training with KV Binding Is Secretly
 * Linear Attention", thelatestinai.com listing, Figure 4: training with the
 * parallel form), from chunked runs on the tensor cores.
 * Without momentum (beta == 0), with G_t = dL/dW_T + sum_{t' >= t} do_t' q_t'^T:
 *   dq_t = W_t^T do_t   the chunked forward on (q, k, v) := (do, v, k) from W_0^T;
 *   G_t k_t, G_t^T v_t  the chunked forward over the chunks last to first
 *                       (anti-causal mask) on (k, q, do) and (v, do, q), from
 *                       dL/dW_T and its transpose (the first run's final
 *                       state is dL/dW_0), whose epilogues write
 *   dv_t = sigma eta_t G_t k_t, dk_t = sigma eta_t G_t^T v_t and
 *   deta_t = sigma v_t . G_t k_t.
 * With momentum (beta != 0; bf16 only): dq is the momentum forward on
 * (do, v, k) from W_0^T and M_0^T; dv, dk, dL/dW_0 and dL/dM_0 come from a
 * reverse chunkwise kernel carrying (dL/dW, beta dL/dM), deta from a
 * forward-order one carrying (M, dL/dW); grad_mom (dL/dM_T) and mom_in (M_0)
 * are optional (zero).
 * bf16: d_k == d_v in {64, 128}; fp32 (no momentum): d_k, d_v multiples of 4
 * up to 128; momentum in fp32, or mom_in / grad_mom without momentum:
 * TTT_LA_ERR_UNSUPPORTED.  Without momentum, grad_mom_in, if given, is zeroed.
 * The workspace (ttt_la_backward_chunked_workspace_size bytes) holds the
 * transposed states and one forward workspace (fp32 also: reversed copies of
 * q, k, v, grad_o and the reverse runs' outputs; momentum also: dL/dW_0 when
 * grad_state_in is NULL).  Errors as ttt_la_backward_recurrent.
 * Streams: with momentum the call runs independent chains of launches, one
 * on `stream` and two on streams the library keeps per device (one at the
 * device's greatest stream priority), joined back into `stream` by events
 * before the call returns: work queued on `stream` afterwards sees every
 * output, as with a single stream.  Under stream capture the library's
 * streams join the capture (created beforehand by an earlier call outside
 * capture; otherwise every chain runs on `stream`). */
TTT_LA_API size_t ttt_la_backward_chunked_workspace_size(const ttt_la_grad_args *args);
TTT_LA_API ttt_la_status ttt_la_backward_chunked(const ttt_la_grad_args *args, void *stream);

/* Synchronises `stream`, returns the device status word (TTT_LA_OK,
 * TTT_LA_ERR_TIMEOUT, or in debug builds TTT_LA_ERR_DEVICE_CHECK, which wins
 * over a timeout) of the current device and clears it. */
TTT_LA_API ttt_la_status ttt_la_get_last_device_status(void *stream);

/* Debug builds (the library compiled with -DTTT_LA_DEBUG, libttt_la_debug.so):
 * the chunked kernels check every hand-indexed access to the workspace, the
 * flags and the states against the sizes of this call; a failed check
 * records TTT_LA_ERR_DEVICE_CHECK and the source line, and the access goes to
 * a private sink instead (nothing faults or traps).  Synchronises `stream`,
 * returns the line of the first failed check since the last query (0: none)
 * and clears it; -1 in release builds (no checks compiled), -2 if CUDA
 * failed. */
TTT_LA_API int32_t ttt_la_debug_check_line(void *stream);

/* Sets the time limit of every in-kernel wait (nanoseconds, >= 1000);
 * default 1e9 (one second).  Affects launches made after the call. */
TTT_LA_API ttt_la_status ttt_la_set_wait_limit_ns(int64_t limit_ns);

/* Self-test of the bounded-wait machinery: launches one block that waits on
 * an mbarrier that nothing completes, with the given limit.  The wait runs out,
 * the block records TTT_LA_ERR_TIMEOUT and returns; read it with
 * ttt_la_get_last_device_status.  Never hangs. */
TTT_LA_API ttt_la_status ttt_la_selftest_wait_timeout(int64_t limit_ns, void *stream);

/* Human-readable name of a status code (static string). */
TTT_LA_API const char *ttt_la_status_string(ttt_la_status s);

/* Library version string (static). */
TTT_LA_API const char *ttt_la_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TTT_LA_H */

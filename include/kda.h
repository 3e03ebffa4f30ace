/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention library, libkda.so.
 *
 * The operator (KimiLinear: A Next-Generation Linear Attention Architecture
 * for Long-Context LLMs, section 2.3) is the per-head recurrence
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t
 *
 * with the state S a d_k x d_v fp32 matrix (row = key channel, column = value
 * channel), g_t = log of the per-channel forget gate (acting on the rows of S;
 * g_t <= 0 for a gate in (0, 1]), beta_t a scalar write strength per token
 * and head, and o_t read from the state after token t has been written.
 *
 * Conventions shared by every call:
 *  - All tensors are dense, contiguous, row-major device buffers owned by the
 *    caller; the library allocates nothing and keeps no state between calls.
 *  - Every pointer must be 16-byte aligned, except beta, which needs only the
 *    alignment of its element type (so a sequence may be cut at any token).
 *  - `dtype` is the element type of q, k, v, g, beta and o (fp32 or bf16);
 *    the state is always fp32.  bf16 results are rounded to nearest-even.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls only enqueue work on it; none synchronises the host.  The device
 *    that owns the buffers and the stream must be the current device of the
 *    calling thread (per-device set-up is keyed by cudaGetDevice).
 *  - Arguments are validated on the host before anything is launched; a
 *    rejected call enqueues nothing.  No call raises an exception across the
 *    ABI and no kernel uses device assertions.
 *  - Results are deterministic: no atomics take part in any accumulation.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, aliasing not allowed */
  KDA_ERR_UNSUPPORTED = 2, /* valid arguments outside what the kernels implement */
  KDA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  KDA_ERR_TIMEOUT = 4      /* a bounded on-device wait gave up (reported by kda_chunk_fwd_check) */
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

/*
 * How the forget gate enters the state update (argument `gate` of the *_gate
 * entry points; the plain entry points use KDA_GATE_CHANNEL):
 *   KDA_GATE_CHANNEL  KDA ("KimiLinear: A Next-Generation Linear Attention
 *                     Architecture for Long-Context LLMs", section 2.3): one
 *                     log-gate per key channel, g [.., dk], alpha = exp(g)
 *                     scales the rows of the state before the delta step.
 *   KDA_GATE_HEAD     Gated DeltaNet (same page, section 2.2): one scalar
 *                     log-gate per token and head, g [.., 1] (layout
 *                     [B, T, H] / [N, H] like beta), alpha_t = exp(g) scales
 *                     the whole state.
 *   KDA_GATE_NONE     DeltaNet (same page, section 2.1): no forget gate,
 *                     alpha = 1; g is ignored and may be NULL.
 */
typedef enum { KDA_GATE_CHANNEL = 0, KDA_GATE_HEAD = 1, KDA_GATE_NONE = 2 } kda_gate;

/*
 * Input preparation fused into the kernels (argument `prep` of the *_ex entry
 * points, a bit set; 0 = inputs already prepared).  The pages give no formula
 * for these steps; they are the transforms that turn raw projections into the
 * operator's inputs (unit-norm keys and queries, a log-gate <= 0, a write
 * strength in (0, 1)), evaluated in fp32 inside the kernels:
 *   KDA_PREP_L2NORM_QK       q <- q (sum_c q_c^2 + 1e-6)^-1/2, same for k, per token and head
 *   KDA_PREP_GATE_LOGSIGMOID g <- log sigmoid(g) = min(g, 0) - log(1 + exp(-|g|))
 *   KDA_PREP_BETA_SIGMOID    beta <- 1 / (1 + exp(-beta))
 */
typedef enum {
  KDA_PREP_NONE = 0,
  KDA_PREP_L2NORM_QK = 1,
  KDA_PREP_GATE_LOGSIGMOID = 2,
  KDA_PREP_BETA_SIGMOID = 4
} kda_prep;

/* Human-readable name of a status code (static storage, never NULL). */
KDA_API const char* kda_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
KDA_API int kda_version(void);

/*
 * Bytes of device workspace kda_chunk_fwd needs for this problem (0 if none).
 * Returns 0 as well for arguments kda_chunk_fwd would reject.
 */
KDA_API size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk, int dtype);

/*
 * Number of kernels one kda_chunk_fwd call with these arguments launches
 * (the workspace-header clear, a memset, is not counted): 1 for the fp32
 * path; for bf16 the chunk preparation plus either one state pass or, when
 * few (sequence, head) chains cover many chunks, the three launches of the
 * chunk-parallel scan, or four for long chains (group 0's output pass runs
 * as its own launch beside the scan; three again when final_state is the
 * initial state's buffer, which this query does not see).  0 when there is
 * nothing to run (B or T zero), -1 for arguments kda_chunk_fwd would reject.
 * Pure host arithmetic.
 */
KDA_API int kda_chunk_fwd_launch_count(int B, int T, int H, int dk, int dv, int chunk, int dtype);

/*
 * Chunked prefill: runs the recurrence over T tokens for B sequences x H heads.
 *
 * Defined by the KDA update (section 2.3) evaluated with the chunkwise
 * parallel algorithm of the same article (section 3.1): the sequence is cut
 * into chunks of `chunk` tokens; inside a chunk the token interactions are
 * dense matrix products, across chunks the state is carried recursively.
 * The chunk size does not change the result (up to rounding); a last partial
 * chunk of T mod chunk tokens is handled.
 *
 *   q, k, g       : [B, T, H, dk]   (dtype)
 *   v             : [B, T, H, dv]   (dtype)
 *   beta          : [B, T, H]       (dtype)
 *   scale         : output scale (commonly 1/sqrt(dk)); it does not touch the state
 *   initial_state : [B, H, dk, dv] fp32, or NULL for a zero state
 *   o             : [B, T, H, dv]   (dtype), written
 *   final_state   : [B, H, dk, dv] fp32, or NULL to skip; may be the same
 *                   buffer as initial_state (updated in place); must not
 *                   overlap any other argument
 *   workspace     : device buffer of at least kda_chunk_fwd_workspace_size()
 *                   bytes (NULL allowed when that size is 0); its contents
 *                   on entry do not matter; it must not be shared by two
 *                   calls in flight at the same time
 *
 * Supported: dk, dv in {64, 128}; dtype KDA_F32 with any chunk in {16, 32,
 * 64}, dtype KDA_BF16 with chunk = 64 (the bf16 kernels run 128 channels, a
 * 64-channel input being zero-padded on the fly).  Anything else with valid
 * shapes returns KDA_ERR_UNSUPPORTED.  T = 0 or B = 0 is valid (the final state
 * is the initial state).
 */
KDA_API kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const void* g, const void* beta,
                         float scale, const float* initial_state, void* o, float* final_state, int B,
                         int T, int H, int dk, int dv, int chunk, int dtype, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * kda_chunk_fwd with a choice of forget gate and fused input preparation.
 * `gate` (kda_gate): KDA_GATE_CHANNEL is kda_chunk_fwd's g [B, T, H, dk];
 * KDA_GATE_HEAD takes g as [B, T, H] (dtype, element alignment like beta);
 * KDA_GATE_NONE ignores g (NULL allowed).  `prep` (kda_prep bits): the
 * inputs q, k, g, beta are raw and prepared in-kernel as listed there.  The
 * workspace size is the same for every gate and prep.  Other arguments,
 * supported shapes, checks and errors as kda_chunk_fwd; an unknown gate or
 * prep bit is KDA_ERR_INVALID_ARG.  kda_chunk_fwd(...) equals
 * kda_chunk_fwd_ex(..., KDA_GATE_CHANNEL, KDA_PREP_NONE, ...).
 */
KDA_API kda_status kda_chunk_fwd_ex(const void* q, const void* k, const void* v, const void* g, const void* beta,
                                    float scale, const float* initial_state, void* o, float* final_state, int B,
                                    int T, int H, int dk, int dv, int chunk, int dtype, int gate, int prep,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Bytes of device workspace kda_backward needs for this problem: a 256-byte
 * header holding the error word of the bounded on-device waits (the same
 * header kda_chunk_fwd_check reads), then per-chunk records (per 64-token
 * chunk and head: the chunk's operands, the state entering it and the state
 * gradient leaving it, and intermediate gradients; about 0.33 MB for bf16
 * and 0.6 MB for fp32 at dk = dv = 128); 0 for arguments kda_backward would
 * reject.
 */
KDA_API size_t kda_backward_workspace_size(int B, int T, int H, int dk, int dv, int dtype);

/*
 * Backward pass: gradients of a scalar loss L through the forward pass
 * (kda_chunk_fwd, or kda_chunk_fwd_ex with `gate` and KDA_PREP_NONE), given
 * dL/do and dL/dS_T.  Reverse-mode differentiation of the chunkwise form
 * (KimiLinear article, section 2.3 for the recurrence, sections 3.1-3.2 for
 * the chunks; sections 2.1-2.2 for the scalar gates): a per-chunk
 * recomputation of the chunk operands, a forward replay of the chunk states
 * and a reverse sweep of the state gradient (each column of the state on its
 * own), then per-chunk local gradients.  Four kernel launches (per group of
 * (sequence, head) pairs, see workspace); tensor-core products with fp32
 * accumulation: bf16 operands when dtype is KDA_BF16, tf32 operands in a
 * three-term split (fp32-level accuracy) when dtype is KDA_F32.
 *
 *   q, k, v, g, beta, scale, initial_state : the forward's inputs (layouts
 *                      and gate kinds as for kda_chunk_fwd_ex)
 *   grad_o           : [B, T, H, dv] (dtype), dL/do
 *   grad_final_state : [B, H, dk, dv] fp32 dL/dS_T, or NULL for zero
 *   grad_q, grad_k   : [B, T, H, dk] (dtype), written
 *   grad_v           : [B, T, H, dv] (dtype), written
 *   grad_g           : like g ([B, T, H, dk] per channel, [B, T, H] per
 *                      head), written; ignored (NULL allowed) for KDA_GATE_NONE
 *   grad_beta        : [B, T, H] (dtype), written
 *   grad_initial_state : [B, H, dk, dv] fp32 dL/dS_0, or NULL to skip
 *   workspace        : 16-byte aligned, contents on entry do not matter;
 *                      kda_backward_workspace_size() bytes hold every
 *                      (sequence, head) at once.  A smaller workspace works
 *                      too, down to kda_backward_workspace_size(1, T, 1, ...)
 *                      (one pair): the pairs are then processed in groups of
 *                      as many as fit, four launches per group, in order on
 *                      the stream (results identical)
 *
 * Supported: dtype KDA_F32 or KDA_BF16, dk and dv in {64, 128}.  Pointers
 * 16-byte aligned (beta, grad_beta and per-head g / grad_g: element
 * alignment); outputs must not overlap any input, each other or the
 * workspace.  Every sum runs in a fixed order (no atomics), so results are
 * bit-reproducible.  T = 0 or B = 0 is valid
 * (grad_initial_state = grad_final_state).  For bf16 at dk = dv = 128 with
 * at least 16 (sequence, head) pairs in a group, the per-chunk operands come
 * from the prefill's preparation kernel and the state passes run on the
 * tcgen05 tensor cores, both with bounded mbarrier waits;
 * kda_chunk_fwd_check(workspace, ...) afterwards returns KDA_ERR_TIMEOUT if
 * one gave up (the gradients are then not valid), KDA_OK otherwise.
 */
KDA_API kda_status kda_backward(const void* q, const void* k, const void* v, const void* g, const void* beta,
                                float scale, const float* initial_state, const void* grad_o,
                                const float* grad_final_state, void* grad_q, void* grad_k, void* grad_v,
                                void* grad_g, void* grad_beta, float* grad_initial_state, int B, int T, int H,
                                int dk, int dv, int dtype, int gate, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * Workspace bytes of kda_backward_ex: kda_backward_workspace_size plus, when
 * `prep` has bits set, room for the prepared inputs; 0 for arguments
 * kda_backward_ex would reject.
 */
KDA_API size_t kda_backward_ex_workspace_size(int B, int T, int H, int dk, int dv, int dtype, int prep);

/*
 * kda_backward for a forward that prepared raw inputs in its kernels
 * (kda_chunk_fwd_ex with the same `prep` bits): q, k, g, beta are the RAW
 * inputs and grad_q, grad_k, grad_g, grad_beta the gradients with respect to
 * them.  The library prepares the inputs into the workspace (input dtype,
 * so bf16 inputs are prepared and then rounded to bf16), runs the backward on
 * them, and applies the chain rule of each step in place (fp32):
 * dq = r (dq^ - q^ (q^ . dq^)) with r = (sum q^2 + 1e-6)^-1/2 (same for k),
 * dg = dg^ sigmoid(-g), dbeta = dbeta^ sigmoid(beta) (1 - sigmoid(beta)).
 * workspace: kda_backward_ex_workspace_size() bytes hold everything; smaller
 * works down to the prepared inputs plus one (sequence, head)'s records.  It
 * starts with the same 256-byte error-word header as kda_backward's.
 * prep = KDA_PREP_NONE is kda_backward.  Other arguments as kda_backward.
 */
KDA_API kda_status kda_backward_ex(const void* q, const void* k, const void* v, const void* g, const void* beta,
                                   float scale, const float* initial_state, const void* grad_o,
                                   const float* grad_final_state, void* grad_q, void* grad_k, void* grad_v,
                                   void* grad_g, void* grad_beta, float* grad_initial_state, int B, int T, int H,
                                   int dk, int dv, int dtype, int gate, int prep, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * kda_chunk_fwd with timing marks for measurement: `events` points to three
 * cudaEvent_t handles (created by the caller) which are recorded on `stream`
 * before the first kernel, between the chunk-preparation kernel and the
 * state-pass kernel, and after the last kernel (for the single-kernel fp32
 * path the last two marks coincide).  Same arguments, checks and results as
 * kda_chunk_fwd otherwise.
 */
KDA_API kda_status kda_chunk_fwd_profiled(const void* q, const void* k, const void* v, const void* g,
                                          const void* beta, float scale, const float* initial_state, void* o,
                                          float* final_state, int B, int T, int H, int dk, int dv, int chunk,
                                          int dtype, void* workspace, size_t workspace_bytes, void* stream,
                                          void* const* events);

/*
 * kda_chunk_fwd without a caller workspace, for callers that cannot allocate
 * device memory (a host program with no allocator of its own, or a plugin in
 * a framework that forbids further cudaMalloc calls).  The pages describe no
 * such interface; it has no counterpart there.
 *
 * Same arguments and results as kda_chunk_fwd minus the workspace.  The
 * scratch is a 64 MiB statically sized device array inside the library
 * (present on every GPU that loads it, until the process exits); problems
 * whose kda_chunk_fwd_workspace_size exceeds it (for the bf16 path about 900
 * chunk-heads, B * H * ceil(T / 64)) return KDA_ERR_UNSUPPORTED before
 * anything is launched.  The first call on a
 * device looks up the array's device address (with that device current), so
 * make it before any stream capture.  All calls share the array: calls whose
 * work overlaps on the GPU race on it and must be serialised by the caller.
 * It allocates nothing (no cudaMalloc, no cudaFree).
 */
KDA_API kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const void* g,
                                         const void* beta, float scale, const float* initial_state, void* o,
                                         float* final_state, int B, int T, int H, int dk, int dv, int chunk,
                                         int dtype, void* stream);

/*
 * The on-device error word of the static scratch used by
 * kda_chunk_fwd_noalloc (synchronises `stream`): KDA_OK, or KDA_ERR_TIMEOUT
 * if a bounded wait inside a kernel of the last kda_chunk_fwd_noalloc call on
 * the current device gave up (that call's outputs are then not valid).  It is
 * the kda_chunk_fwd_check of that path, whose scratch the caller cannot name.
 * No counterpart on the pages.  Allocates nothing.
 */
KDA_API kda_status kda_chunk_fwd_noalloc_check(void* stream);

/*
 * Reads the on-device error word that the last kda_chunk_fwd (or
 * kda_backward / kda_backward_ex) using this workspace left behind
 * (synchronises `stream`).  Returns KDA_OK, or KDA_ERR_TIMEOUT if a bounded
 * wait inside a kernel gave up (the outputs of that call are then not
 * valid).  A workspace of size 0 always reports KDA_OK.
 */
KDA_API kda_status kda_chunk_fwd_check(const void* workspace, size_t workspace_bytes, void* stream);

/*
 * Failure-path self-test: enqueues a tiny kernel whose single mbarrier wait
 * can never be satisfied; the wait gives up after a short bounded number of
 * polls and records the give-up in the workspace header, exactly like a
 * prefill kernel would.  A following kda_chunk_fwd_check on the same
 * workspace then returns KDA_ERR_TIMEOUT.  `workspace` needs 256 bytes,
 * 256-byte aligned.  Nothing faults and the GPU stays usable.
 */
KDA_API kda_status kda_wait_selftest(void* workspace, size_t workspace_bytes, void* stream);

/*
 * Single-token decode (O(1) per token, constant-size state: same article,
 * section 4.2): one step of the recurrence for N sequences x H heads, with
 * the state updated in place.
 *
 *   q, k, g : [N, H, dk] (dtype)     v, o : [N, H, dv] (dtype)     beta : [N, H] (dtype)
 *   state   : [N, H, dk, dv] fp32, read and overwritten with the new state
 *
 * Supported: dk, dv in {64, 128}, dtype KDA_F32 or KDA_BF16.
 */
KDA_API kda_status kda_recurrent_step(const void* q, const void* k, const void* v, const void* g,
                              const void* beta, float scale, float* state, void* o, int N, int H,
                              int dk, int dv, int dtype, void* stream);

/*
 * kda_recurrent_step with a choice of forget gate (kda_gate: g is [N, H, dk]
 * for KDA_GATE_CHANNEL, [N, H] for KDA_GATE_HEAD with element alignment, and
 * ignored, NULL allowed, for KDA_GATE_NONE) and fused input preparation
 * (kda_prep bits, as for kda_chunk_fwd_ex).  Otherwise as kda_recurrent_step.
 */
KDA_API kda_status kda_recurrent_step_ex(const void* q, const void* k, const void* v, const void* g,
                                         const void* beta, float scale, float* state, void* o, int N, int H,
                                         int dk, int dv, int dtype, int gate, int prep, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */

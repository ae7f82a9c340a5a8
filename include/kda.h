/*
 * libkda: Kimi Delta Attention (KDA) forward on NVIDIA B200 (sm_100a).
 *
 * KDA is the gated delta rule with one forget rate per key channel
 * (blog.gzher.com "Kimi K3论文：Kimi Linear", section 3, eq. (1)):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t                               (read after the update)
 *
 * with S_t a dk x dv state per (sequence, head), dk = dv = 128,
 * alpha_t = exp(log_alpha_t) in [0,1]^dk and beta_t in [0,1]. There is no
 * query scaling; callers that want 1/sqrt(dk) scale q themselves.
 *
 * Two entry points compute it: a chunk-parallel prefill over whole
 * sequences (section 4 of the same page: chunks of C = 64, WY representation,
 * UT transform, state passed between chunks) and a single-token recurrent
 * decode step (section 4: decode switches to the recurrent kernel).
 *
 * Conventions shared by every call
 *   - Every pointer is DEVICE memory owned by the caller. The library never
 *     allocates, frees or synchronises; calls are asynchronous on `stream`
 *     (a cudaStream_t, NULL = the legacy default stream) and may be captured
 *     in a CUDA graph (except the first kda_chunk_fwd_noalloc call on a GPU).
 *     Within a prefill call, later kernels may start while earlier ones finish
 *     (programmatic dependent launch); they wait for the earlier results on
 *     the device, so callers see ordinary stream order.
 *   - All tensors are contiguous, row-major, in the layouts given below.
 *     Token-major tensors index [token][head][channel].
 *   - q, k, v and o share one element type, `dtype` (kda_dtype). beta and
 *     the state are always fp32; log_alpha is fp32 except in the bf16 gate
 *     layout of the *_gated calls (kda_gate).
 *   - Preconditions that are not checked element by element: q and k rows
 *     L2-normalised per head (the layer's L2Norm, section 3), log_alpha
 *     finite and <= 0 (use a large finite negative number, not -inf, for
 *     alpha = 0), beta in [0, 1].
 *   - Return value: KDA_OK (0) or a negative kda_status. Argument errors are
 *     detected on the host before anything is launched; nothing is written
 *     in that case. KDA_ERR_CUDA means a launch failed (the CUDA error is
 *     left for the caller to read with cudaGetLastError).
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#define KDA_HEAD_DIM 128 /* dk = dv, fixed */
#define KDA_CHUNK 64       /* chunk length of the tensor-core prefill (bf16 inputs) */
#define KDA_CHUNK_SMALL 32 /* the other chunk length kda_chunk_fwd accepts (CUDA cores) */

typedef enum kda_dtype {
    KDA_BF16 = 0, /* q, k, v, o are bfloat16 */
    KDA_F32 = 1   /* q, k, v, o are float32 */
} kda_dtype;

/*
 * How the forget gate alpha_t is given. KDA gives every key channel its own
 * rate (blog.gzher.com "Kimi K3论文：Kimi Linear", section 3). The two models
 * that section 2 of the same page builds it from are special cases of it:
 * Gated DeltaNet has one scalar rate per head, and alpha_t times
 * (I - beta_t k_t k_t^T) S equals (I - beta_t k_t k_t^T) Diag(alpha_t 1) S
 * because a scalar commutes with the matrix. DeltaNet has no forget gate
 * (alpha_t = 1).
 * The gate is always passed as log_alpha (natural log), in one of these
 * layouts:
 */
typedef enum kda_gate {
    KDA_GATE_CHANNEL = 0,      /* fp32 [token][head][128]: one rate per key channel (KDA) */
    KDA_GATE_CHANNEL_BF16 = 1, /* the same, bfloat16 */
    KDA_GATE_HEAD = 2,         /* fp32 [token][head]: one rate per head (Gated DeltaNet) */
    KDA_GATE_NONE = 3,         /* no gate, alpha = 1 (DeltaNet); log_alpha is not read */
    /* The gate's pre-activation z (the output of the gate's low-rank projection,
     * section 3: alpha_t = f(W_up W_down x_t)), with f = sigmoid: alpha = sigmoid(z),
     * so the kernels use log alpha = log sigmoid(z) = -log(1 + exp(-z)). The page
     * leaves f open; sigmoid is the plainest map onto [0, 1]. z is any finite value. */
    KDA_GATE_CHANNEL_LOGIT = 4,     /* fp32 [token][head][128] */
    KDA_GATE_CHANNEL_LOGIT_BF16 = 5 /* the same, bfloat16 */
} kda_gate;

typedef enum kda_status {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = -1, /* null pointer, bad size, bad offsets */
    KDA_ERR_UNSUPPORTED = -2, /* C not 32 or 64, unknown dtype or unknown gate layout */
    KDA_ERR_WORKSPACE = -3,   /* workspace missing or smaller than required */
    KDA_ERR_CUDA = -4,        /* a kernel launch failed */
    KDA_ERR_TIMEOUT = -5,     /* a bounded device-side wait expired */
    KDA_ERR_SCRATCH_LIMIT = -6 /* kda_chunk_fwd_noalloc: problem needs more than its fixed scratch */
} kda_status;

/* Human-readable name of a status code (static string, never NULL). */
KDA_API const char *kda_strerror(int status);

/* Library version as 10000*major + 100*minor + patch. */
KDA_API int kda_version(void);

/*
 * Bytes of device workspace kda_chunk_fwd needs for these sizes.
 *
 * Arguments are those of kda_chunk_fwd: B batch rows of T tokens, or, when
 * n_seqs > 0, one packed row (B = 1) of T tokens split into n_seqs
 * sequences. Writes the size to *bytes (0 is possible). The workspace holds
 * per-chunk intermediates (the WY factors) between the kernels of one call;
 * it carries nothing from one call to the next.
 */
KDA_API int kda_chunk_fwd_workspace_size(int B, int64_t T, int H, int C, int n_seqs, int dtype,
                                 size_t *bytes);

/*
 * Number of libkda kernels that one kda_chunk_fwd call with these arguments
 * launches on the current device (*n_kernels), for launch accounting. The
 * bf16 path launches its prep and chain kernels (plus a chunk-offset scan for
 * packed sequences: 2 or 3), one fused cooperative kernel for batched inputs
 * with few sequence-heads and many chunks (1), or, for long batched sequences
 * with very few sequence-heads, the segment scan: prep, two chain passes and
 * a combine (4). The fp32 path launches one kernel. Returns KDA_OK, or
 * KDA_ERR_INVALID_ARG / KDA_ERR_UNSUPPORTED as kda_chunk_fwd would.
 */
KDA_API int kda_chunk_fwd_launches(int B, int64_t T, int H, int C, int n_seqs, int dtype,
                                   int *n_kernels);

/*
 * Chunk-parallel KDA prefill (blog.gzher.com section 4; chunked form of the
 * mokono.cn explainer section 2.1: S_r = P_r S_0 + H_r within a chunk).
 *
 *   q, k       [B, T, H, 128]  dtype    (with cu_seqlens: [T, H, 128], B = 1)
 *   v          [B, T, H, 128]  dtype
 *   log_alpha  [B, T, H, 128]  fp32     log of the per-channel forget gate
 *   beta       [B, T, H]       fp32     write strength
 *   S0         [Nseq, H, 128, 128] fp32 initial state (dk rows, dv columns),
 *                               or NULL for zeros
 *   o          [B, T, H, 128]  dtype    output (written)
 *   S_T        [Nseq, H, 128, 128] fp32 final state (written), or NULL
 *   C          chunk length: 64 (KDA_CHUNK) or 32 (KDA_CHUNK_SMALL); the pages
 *              name 32 to 128 as the useful range (mokono.cn section 4.1). bf16
 *              inputs with C = 64 run on the tensor cores; fp32 inputs, and C = 32
 *              in either dtype, run on the CUDA-core kernel (one launch, no
 *              workspace). C = 128 returns KDA_ERR_UNSUPPORTED:
 *              the CUDA-core kernel's fp32 working set for one chunk (about 400 KB)
 *              does not fit an SM, and the tensor-core kernels are built for 64.
 *   cu_seqlens device int32 [n_seqs + 1] token offsets of packed sequences
 *              (cu_seqlens[0] = 0, non-decreasing, cu_seqlens[n_seqs] = T),
 *              or NULL: then Nseq = B sequences of T tokens each.
 *   cu_seqlens_host  optional host copy of cu_seqlens. When given it is
 *              validated (monotone, ends at T); when NULL the device offsets
 *              are trusted.
 *   workspace  device buffer of at least kda_chunk_fwd_workspace_size bytes,
 *              16-byte aligned (NULL allowed when that size is 0).
 *
 * Chunks start at each sequence's first token; the last chunk of a sequence
 * may be shorter than C. A sequence of length 0 writes no output rows and
 * S_T = S0. S0 and S_T may point to the same buffer (in-place carry, which
 * is how a long sequence is processed as several calls). q, k, v, o must not
 * overlap.
 */
KDA_API int kda_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                  const float *beta, const float *S0, void *o, float *S_T, int B, int64_t T,
                  int H, int C, const int32_t *cu_seqlens, int n_seqs,
                  const int32_t *cu_seqlens_host, int dtype, void *workspace,
                  size_t workspace_bytes, void *stream);

/*
 * kda_chunk_fwd with the forget gate in any kda_gate layout. All other
 * arguments are those of kda_chunk_fwd. log_alpha points to a tensor of
 * `gate`'s layout ([B, T, H, 128] fp32 or bf16, or [B, T, H] fp32; packed
 * inputs drop B), finite and <= 0. For KDA_GATE_NONE it is not read and may
 * be NULL. kda_chunk_fwd(...) is kda_chunk_fwd_gated(..., KDA_GATE_CHANNEL, ...).
 * The gate layout changes neither the workspace size nor the kernels
 * launched. An unknown `gate` returns KDA_ERR_UNSUPPORTED.
 */
KDA_API int kda_chunk_fwd_gated(const void *q, const void *k, const void *v,
                                const void *log_alpha, int gate, const float *beta,
                                const float *S0, void *o, float *S_T, int B, int64_t T, int H,
                                int C, const int32_t *cu_seqlens, int n_seqs,
                                const int32_t *cu_seqlens_host, int dtype, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * Fused input and output transformations (blog.gzher.com "Kimi K3论文：Kimi
 * Linear", section 3, the neural parameterisation around the operator):
 *   q_t, k_t = L2Norm(...),  beta_t = Sigmoid(W_beta x_t),
 * and before the output projection a head-wise RMSNorm and a data-dependent
 * sigmoid output gate. The section does not write the epilogue as a formula;
 * the reading taken is, per (token, head) row o of 128 values,
 *   o <- o / sqrt(mean(o^2) + out_norm_eps) * w * sigmoid(out_gate),
 * with w the norm's weight. A zero field leaves that step out:
 *   qk_l2norm        nonzero: q and k rows (128 channels) are divided by
 *                    sqrt(sum of squares + qk_l2norm_eps) inside the kernels
 *                    (a row whose sum plus eps is 0 becomes 0); the inputs then
 *                    need not be normalised
 *   beta_logits      nonzero: beta holds logits, the kernels use sigmoid(beta)
 *   out_gate         NULL, or the gate's input, shaped like o ([B, T, H, 128] or
 *                    [N, H, 128], q's dtype; 16-byte aligned, and o too, for
 *                    prefill; 16-byte aligned for bf16 decode): applies the
 *                    output epilogue above to o
 *   out_norm_weight  [128] fp32, 16-byte aligned, or NULL for ones
 * eps values must be finite and >= 0. The gate's own pre-activation is a gate
 * layout (KDA_GATE_CHANNEL_LOGIT*), not a field here.
 */
typedef struct kda_io {
    int qk_l2norm;
    float qk_l2norm_eps;
    int beta_logits;
    const void *out_gate;
    const float *out_norm_weight;
    float out_norm_eps;
} kda_io;

/*
 * kda_chunk_fwd_gated with the fused transformations of `io` (NULL: none, which
 * is kda_chunk_fwd_gated itself). Every field works on every path (both dtypes,
 * C = 32 and 64). The input steps run inside the prefill kernels; with qk_l2norm
 * a bf16 call that would take the fused grid runs the prep and chain kernels
 * instead. The output epilogue is one more kernel after the call's others (one
 * read of o and out_gate, one write of o, in place), with the workspace unchanged.
 */
KDA_API int kda_chunk_fwd_io(const void *q, const void *k, const void *v, const void *log_alpha,
                             int gate, const float *beta, const float *S0, void *o, float *S_T,
                             int B, int64_t T, int H, int C, const int32_t *cu_seqlens, int n_seqs,
                             const int32_t *cu_seqlens_host, int dtype, void *workspace,
                             size_t workspace_bytes, const kda_io *io, void *stream);

/* kda_chunk_fwd_launches for a kda_chunk_fwd_io call with these options. */
KDA_API int kda_chunk_fwd_io_launches(int B, int64_t T, int H, int C, int n_seqs, int dtype,
                                      const kda_io *io, int *n_kernels);

/*
 * Backward pass of kda_chunk_fwd (training): the gradients of
 *   L = sum(o * dout) + sum(S_T * dS_T)
 * with respect to every input, for given dout (and dS_T). The recurrence of eq. (1)
 * (section 3) is differentiated token by token in reverse (section 4 of the same
 * page counts the training cost of the chunked form; these are the same
 * gradients). All arithmetic is fp32 on CUDA cores, for both dtypes.
 *
 *   q, k, v, log_alpha, gate, beta, S0, B, T, H, cu_seqlens, n_seqs,
 *   cu_seqlens_host, dtype, io: as for kda_chunk_fwd_io (io->out_gate must be
 *              NULL: the output epilogue has no backward here)
 *   dout       like o (dtype): dL/do
 *   dS_T       [Nseq, H, 128, 128] fp32: dL/dS_T, or NULL for zeros
 *   dq, dk, dv [.., H, 128] fp32 (written): dL/dq, dL/dk, dL/dv (with io->qk_l2norm,
 *              the gradients of the un-normalised q and k)
 *   dgate      the gate's gradient (written), fp32, in its layout's shape:
 *              [.., H, 128] for per-channel layouts (dL/dlog_alpha, or dL/dz for
 *              the logit layouts), [.., H] for KDA_GATE_HEAD; not written (may be
 *              NULL) for KDA_GATE_NONE
 *   dbeta      [.., H] fp32 (written): dL/dbeta (dL/d logit with io->beta_logits)
 *   dS0        [Nseq, H, 128, 128] fp32 (written), or NULL: dL/dS0
 *   workspace  device buffer of kda_chunk_bwd_workspace_size bytes, 16-byte
 *              aligned. It holds each token's per-slice gradient shares (6.2 KB
 *              per token-head), the state every 32 tokens (64 KB per head) and
 *              a replay scratch of 512 x 512 KiB.
 * The call launches two kernels; the result is bitwise reproducible.
 * Concurrent calls must not share a workspace.
 */
KDA_API int kda_chunk_bwd_workspace_size(int B, int64_t T, int H, int n_seqs, size_t *bytes);
KDA_API int kda_chunk_bwd(const void *q, const void *k, const void *v, const void *log_alpha, int gate,
                          const float *beta, const float *S0, const void *dout, const float *dS_T,
                          float *dq, float *dk, float *dv, float *dgate, float *dbeta, float *dS0,
                          int B, int64_t T, int H, const int32_t *cu_seqlens, int n_seqs,
                          const int32_t *cu_seqlens_host, int dtype, const kda_io *io,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * One recurrent decode step for N sequences (eq. (1) applied to one token;
 * blog.gzher.com section 4: decode uses the recurrent kernel).
 *
 *   q, k, v    [N, H, 128]  dtype
 *   log_alpha  [N, H, 128]  fp32
 *   beta       [N, H]       fp32
 *   S          [N, H, 128, 128] fp32, read and overwritten in place with S_t
 *   o          [N, H, 128]  dtype   output o_t = S_t^T q_t (written)
 */
KDA_API int kda_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                    const float *beta, float *S, void *o, int N, int H, int dtype, void *stream);

/*
 * kda_decode_step with the forget gate in any kda_gate layout: log_alpha is
 * [N, H, 128] fp32 or bf16, [N, H] fp32, or not read (KDA_GATE_NONE, may be
 * NULL). Everything else is as for kda_decode_step.
 */
KDA_API int kda_decode_step_gated(const void *q, const void *k, const void *v,
                                  const void *log_alpha, int gate, const float *beta, float *S,
                                  void *o, int N, int H, int dtype, void *stream);

/* kda_decode_step_gated with the fused transformations of `io` (NULL: none). */
KDA_API int kda_decode_step_io(const void *q, const void *k, const void *v, const void *log_alpha,
                               int gate, const float *beta, float *S, void *o, int N, int H,
                               int dtype, const kda_io *io, void *stream);

/*
 * kda_chunk_fwd for callers that cannot allocate device memory. The pages
 * describe no counterpart: this is a library-integration entry point, not
 * part of the method.
 *
 * Who needs it: code that may not call cudaMalloc, for example a plugin inside
 * a host framework that owns all device memory through its own pool and gives
 * plugins no allocation hook, or a latency-critical loop where cudaMalloc's
 * possible device-wide synchronisation is not acceptable. Such a caller still
 * passes its inputs and outputs, exactly as for kda_chunk_fwd (same argument
 * meaning, layouts and ownership), but no workspace.
 *
 * Instead of a workspace the call uses one fixed scratch buffer of
 * kda_noalloc_scratch_bytes() bytes (64 MiB) that lives in the library's
 * device image: it is reserved on each GPU where that image is loaded (at
 * context creation with CUDA_MODULE_LOADING=EAGER, otherwise on the first use
 * of the library's device code on that GPU) and held until the process
 * exits. A problem whose kda_chunk_fwd_workspace_size exceeds it is rejected
 * with KDA_ERR_SCRATCH_LIMIT before anything is launched (about a thousand
 * chunk-head pairs for bf16: B * ceil(T/64) * H <= 1015 for unpacked input
 * without segment-scan room; fp32 input needs no scratch). All calls on a GPU share the buffer and
 * it keeps the previous call's contents; nothing in it has to start at zero.
 * Calls that may overlap on the GPU (different streams, no ordering between
 * them) race on the buffer: issue them on one stream. The first call on each
 * GPU looks up the buffer's device address with that GPU current; make it
 * before any stream capture begins. The address is kept for the life of the
 * process: do not use this entry point after a device reset
 * (cudaDeviceReset). The function itself allocates nothing.
 */
KDA_API int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                  const float *log_alpha, const float *beta, const float *S0,
                                  void *o, float *S_T, int B, int64_t T, int H, int C,
                                  const int32_t *cu_seqlens, int n_seqs,
                                  const int32_t *cu_seqlens_host, int dtype, void *stream);

/* Size in bytes of the fixed scratch used by kda_chunk_fwd_noalloc. */
KDA_API size_t kda_noalloc_scratch_bytes(void);

/*
 * Reads and clears the library's device status. *status is 0 when nothing
 * has been recorded since the last read, otherwise a mask of:
 *   KDA_STATUS_TIMEOUT    a kernel gave up on a bounded wait (the outputs of
 *                         the call that timed out are invalid; KDA_ERR_TIMEOUT
 *                         describes it);
 *   KDA_STATUS_BAD_INPUT  a KDA_DEBUG build found device cu_seqlens that
 *                         break the documented contract (cu_seqlens[0] = 0,
 *                         non-decreasing, cu_seqlens[n_seqs] = T) and left
 *                         that call's outputs unwritten.
 * A timeout that has not been read yet does not affect later calls: a wait
 * gives up early only when another wait gives up while it is waiting, so
 * calls made after the failed one compute normally.
 * Synchronises with the device (a blocking symbol copy on the legacy
 * stream); do not call it inside stream capture.
 *
 * KDA_DEBUG builds. libkda_debug.so is the same library compiled with
 * KDA_DEBUG defined. Device offsets passed without a host copy are then
 * checked on the device before any kernel of the call reads a sequence span:
 * on failure the call is counted as KDA_STATUS_BAD_INPUT and its kernels
 * return at entry, so nothing outside the caller's tensors is read or
 * written. Nothing traps or faults on purpose. The ordinary build trusts
 * device offsets that come without a host copy.
 */
#define KDA_STATUS_TIMEOUT 1
#define KDA_STATUS_BAD_INPUT 2
KDA_API int kda_get_device_status(int *status);

/*
 * Failure-detection support (no counterpart on the pages; library plumbing).
 *
 * Every wait of the tensor-core kernels on an mbarrier, a ready flag or a
 * shared counter gives up after a time limit (default one second), counts a
 * timeout in the device status and lets its kernel unwind and return.
 * kda_set_wait_limit_ns sets that limit for later launches on the current
 * GPU (ns = 0 restores the default). It is meant for tests of the failure
 * path; a limit shorter than a kernel's ordinary waits makes correct calls
 * time out. Synchronises with the device like kda_get_device_status.
 *
 * kda_selftest_wait_timeout runs, on `stream`, one small kernel that makes
 * each of the three kinds of bounded wait run out: an mbarrier that nothing
 * arrives on, the device int32 *flag (which the caller keeps at 0) and a
 * shared counter that nothing raises. It writes to the device int32 *result
 * a bitmask of the waits that gave up (bit 0 mbarrier, bit 1 flag, bit 2
 * counter; 7 when all three did) and counts three timeouts in the device
 * status. It takes about three wait limits. Both pointers must be 4-byte
 * aligned device memory.
 */
KDA_API int kda_set_wait_limit_ns(uint64_t ns);
KDA_API int kda_selftest_wait_timeout(const int32_t *flag, int32_t *result, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */

/*
 * kda.h -- C ABI of libkda.so: Kimi Delta Attention (KDA) on NVIDIA B200 (sm_100a).
 *
 * KDA is the gated delta-rule sequence mixer.  For one sequence and one head,
 * with a d_k x d_v fp32 state S, per token t:
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t = S_t^T (s q_t),   s = d_k^{-1/2},   alpha_t = exp(log_alpha_t) per channel
 *
 * Definition: page "会加减乘除就够:十个问题,手算读懂 Kimi K3 心脏里的全部数学"
 * (jokeuncle.github.io), intro and 终局 (the four actions forget / correct / write /
 * read of Q3, Q4, Q6, Q8); the query scale d_k^{-1/2} is the one of the translated
 * KDA bra-ket blog (mynewscn.com), preamble.  The chunked algorithm used by
 * kda_chunk_fwd is the WY/UT form of page "22,580：从 GPT-2 到 Kimi K3" §6.3
 * (yichencityu.github.io), with the per-channel cumulative decay of its §08/§9.1.
 * Chunking changes only the rounding, never the result.
 *
 * Conventions for every entry point:
 *  - All tensor arguments are DEVICE pointers on the current CUDA device, row-major,
 *    contiguous, 16-byte aligned.  The caller allocates and owns every buffer; the
 *    library keeps no pointer after a call returns.  The only device memory the
 *    library takes itself is kda_chunk_fwd's workspace (below); kda_chunk_fwd_noalloc
 *    uses a fixed buffer instead.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and never synchronise the device.
 *  - The return value is KDA_OK (0) or a negative kda_status.  Argument errors are
 *    detected on the host before anything is launched; nothing is written then.
 *  - Input domain: log_alpha finite and <= 0 (alpha in (0, 1]); beta in [0, 1];
 *    keys are expected to be L2-normalised (not checked).  NaN/Inf inputs give
 *    unspecified values but never an out-of-bounds access.
 *  - Thread safety: entry points may be called concurrently from several host
 *    threads; kda_status_string's CUDA message is kept per host thread.
 */
#ifndef KDA_H
#define KDA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *kda_stream_t;

/* Element type of q, k, v and out.  log_alpha, beta and the state are always fp32. */
enum kda_dtype {
    KDA_F32 = 0,  /* fp32 inputs and outputs; fp32 SIMT arithmetic */
    KDA_BF16 = 1  /* bf16 inputs and outputs; bf16 tensor-core products, fp32 accumulation and state */
};

enum kda_status {
    KDA_OK = 0,
    KDA_ERR_NULL = -1,    /* a required pointer is NULL */
    KDA_ERR_DIM = -2,     /* a size is out of range: B, H < 1, T < 0, dk or dv not in {32, 64, 128},
                             or a combination the dtype does not support */
    KDA_ERR_CHUNK = -3,   /* C != 64 */
    KDA_ERR_ALIGN = -4,   /* a pointer is not 16-byte aligned */
    KDA_ERR_DTYPE = -5,   /* dtype is not a kda_dtype */
    KDA_ERR_ALIAS = -6,   /* an output overlaps an input it must not overlap */
    KDA_ERR_CUDA = -7,    /* a CUDA launch failed; kda_status_string names the CUDA error */
    KDA_ERR_TIMEOUT = -8, /* reserved for bounded device-side waits */
    KDA_ERR_SCRATCH = -9, /* kda_chunk_fwd_noalloc: the workspace would exceed its fixed buffer */
    KDA_ERR_GATE = -10,   /* _ex entry points: a bad gate form, flag or gate pointer */
    KDA_ERR_INDEX = -11   /* kda_device_status: a kda_decode_ex state index was >= the pool size */
};

/*
 * kda_chunk_fwd -- chunked prefill over whole sequences.
 *
 * Layout (T_total = B*T without cu_seqlens, T with it):
 *   q, k       [T_total, H, dk]   dtype            (B x T x H x dk when fixed-length)
 *   v          [T_total, H, dv]   dtype
 *   log_alpha  [T_total, H, dk]   fp32             per-channel log-decay, <= 0
 *   beta       [T_total, H]       fp32             write strength
 *   S0         [N, H, dk, dv]     fp32 or NULL     initial state (NULL = zero state)
 *   cu_seqlens [N + 1]            int32 or NULL    NULL: N = B sequences of T tokens each.
 *                                                 Else N = B sequences packed on the token
 *                                                 axis: sequence n is tokens
 *                                                 [cu_seqlens[n], cu_seqlens[n+1]); entries
 *                                                 must be non-decreasing from 0 to T.  They are
 *                                                 read on the device and clamped to [0, T], so
 *                                                 malformed offsets give unspecified values but
 *                                                 never an out-of-bounds access.
 *   out        [T_total, H, dv]   dtype            o_t for every token (written)
 *   S_final    [N, H, dk, dv]     fp32 or NULL     state after each sequence's last token
 *                                                 (NULL = not written).  May be the same
 *                                                 pointer as S0 (updated in place).
 *   C          chunk length; must be 64.
 * Empty sequences (and T = 0) are allowed: their S_final is S0 (or zero).
 * Workspace: with KDA_BF16 and dk = dv = 128 the call runs two kernels (one per
 * (chunk, head), then one scan per (sequence, head)) that hand each chunk's operands
 * over through a device workspace of 66,560 bytes per (chunk, head) plus 4 (2N + 1)
 * bytes (slot offsets and the scan order), rounded up to 1 KiB.  It is taken with
 * cudaMallocAsync on `stream` from the device's default memory pool and returned with
 * cudaFreeAsync on the same stream;
 * the pool's release threshold is raised on first use so the memory stays in the
 * pool between calls.  Every other dtype and size allocates nothing.
 * Supported sizes: KDA_F32 any dk, dv in {32, 64, 128}; KDA_BF16 dk = dv = 128, or
 * dk, dv in {32, 64, 128} through the same path.
 * q, k, v, log_alpha, beta and out may be NULL only when T_total = 0.
 * Errors: KDA_ERR_NULL (q, k, v, log_alpha, beta or out NULL while T_total > 0), KDA_ERR_DIM, KDA_ERR_CHUNK,
 * KDA_ERR_DTYPE, KDA_ERR_ALIGN, KDA_ERR_ALIAS (out overlapping an input; S_final
 * overlapping an input other than exactly S0), KDA_ERR_CUDA.
 */
int kda_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                  const float *beta, const float *S0, const int32_t *cu_seqlens, void *out,
                  float *S_final, int B, int T, int H, int dk, int dv, int C, int dtype,
                  kda_stream_t stream);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd that takes no device memory.
 *
 * The pages have no counterpart of this call: it adds nothing to the method.  It is
 * for callers that must not allocate during a call -- a server that reserved nearly
 * all of HBM for its caches at start-up, a runtime whose device footprint must be
 * fixed in advance, a host thread that must keep clear of allocator state.
 * Arguments, layouts, results and errors are those of kda_chunk_fwd, plus
 * KDA_ERR_SCRATCH.  Where kda_chunk_fwd takes its workspace from the memory pool,
 * this call uses a buffer of KDA_NOALLOC_SCRATCH_BYTES (64 MiB) that is part of the
 * library's device image, one per device; no allocator (CUDA's or any other) is called.
 *  - Limit: the workspace must fit: 66,560 bytes per (chunk, head) plus 4 (2N + 1)
 *    bytes rounded up to 1 KiB, counting ceil(T / 64) chunks per sequence without
 *    cu_seqlens and ceil(T / 64) + N chunks in all with it.  That is at most 1,008
 *    (chunk, head) pairs, e.g. one 4,032-token sequence with 16 heads.  A larger
 *    problem returns KDA_ERR_SCRATCH, found on the host before any CUDA call.  Only
 *    KDA_BF16 with dk = dv = 128 uses the buffer; every other case needs none.
 *  - The first call on a device looks up the buffer's device address (one CUDA runtime
 *    query, made with that device current) and keeps it for the life of the process.  A
 *    caller that records its calls into a stream capture should make one call on each
 *    device before it starts.  Resetting a device (cudaDeviceReset) after the first call
 *    on it is not supported: the kept address may no longer be the buffer's.
 *  - Nothing in the buffer needs to start at zero: each call writes every byte of it
 *    that the call later reads.
 *  - Overlapping calls race: two calls on one device that can run at the same time
 *    (different streams, or host threads with no ordering between their streams)
 *    share the buffer and corrupt each other's results.  Calls on one stream are
 *    ordered and safe.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, const float *S0, const int32_t *cu_seqlens,
                          void *out, float *S_final, int B, int T, int H, int dk, int dv, int C,
                          int dtype, kda_stream_t stream);

/*
 * Gate forms of the entry points with the _ex suffix.  Every form is the recurrence above
 * with a different way of giving alpha_t (and, with flags, beta_t and unit-length q, k):
 *
 *  KDA_GATE_CHANNEL  gate = log_alpha [.., H, dk] fp32, one decay per channel: KDA itself
 *                    ("Ten questions" Q8).  Same as kda_chunk_fwd / kda_decode_step.
 *  KDA_GATE_SCALAR   gate = log_alpha [.., H] fp32, one decay per (token, head) shared by
 *                    all channels: Gated DeltaNet ("22,580" §08).  The kernels apply the
 *                    scalar to every channel with the arithmetic of KDA_GATE_CHANNEL, so
 *                    the result is bit-identical to that form fed the broadcast gate.
 *  KDA_GATE_NONE     gate = NULL, alpha = 1: DeltaNet ("22,580" §5-§6).
 *  KDA_GATE_FUSED    gate = f [.., H, dk] in the input dtype, with A_log, dt_bias [H, dk]
 *                    fp32: log_alpha = -exp(A_log) * softplus(f + dt_bias),
 *                    softplus(x) = ln(1 + e^x) -- the gate line read out in "Ten questions"
 *                    Q9, computed in the kernel in fp32, so the log_alpha stream (4 bytes
 *                    per channel) becomes f in the input dtype.  log_alpha is kept >= -1e4
 *                    (alpha = e^-1e4 is 0 in fp32 either way).
 * Flags (any combination; 0 = none):
 *  KDA_NORM_Q, KDA_NORM_K  q (resp. k) is scaled to unit L2 length per (token, head) in the
 *                    kernel, x / max(||x||_2, 1e-12), fp32 ("22,580" §5.2 layer code).
 *  KDA_BETA_LOGIT    beta holds logits: beta_t = 1 / (1 + e^-b_t) ("Ten questions" Q9).
 * A_log and dt_bias are used (and must be non-NULL) only with KDA_GATE_FUSED.
 */
enum kda_gate_kind {
    KDA_GATE_CHANNEL = 0,
    KDA_GATE_SCALAR = 1,
    KDA_GATE_NONE = 2,
    KDA_GATE_FUSED = 3
};
enum kda_gate_flags { KDA_NORM_Q = 1, KDA_NORM_K = 2, KDA_BETA_LOGIT = 4 };

/*
 * kda_chunk_fwd_ex -- kda_chunk_fwd with a gate form and flags (above).
 * Layouts, sizes, workspace, results and errors are those of kda_chunk_fwd, with
 * log_alpha replaced by (gate_kind, gate, A_log, dt_bias, flags):
 *   gate     CHANNEL: [T_total, H, dk] fp32;  SCALAR: [T_total, H] fp32;  NONE: NULL;
 *            FUSED: f [T_total, H, dk] dtype
 *   A_log, dt_bias  FUSED only: [H, dk] fp32 each
 *   beta     [T_total, H] fp32: beta itself, or logits with KDA_BETA_LOGIT
 * Errors as kda_chunk_fwd, plus KDA_ERR_GATE (unknown gate_kind or flags, gate NULL for a
 * form that needs it or non-NULL for KDA_GATE_NONE, A_log or dt_bias NULL for KDA_GATE_FUSED).
 */
int kda_chunk_fwd_ex(const void *q, const void *k, const void *v, int gate_kind, const void *gate,
                     const float *A_log, const float *dt_bias, int flags, const float *beta,
                     const float *S0, const int32_t *cu_seqlens, void *out, float *S_final, int B,
                     int T, int H, int dk, int dv, int C, int dtype, kda_stream_t stream);

/*
 * kda_chunk_bwd -- gradients of a prefill: the backward pass for training.
 * The pages discuss training ("22,580" §6.1: the chunked prefill is the training-time path)
 * but print no backward pass; this is the reverse-mode derivative of the chunked algorithm
 * of kda_chunk_fwd ("22,580" §6.3 with the decay of §08/§9.1), recomputing the forward's
 * chunk states itself.  For L = sum(dO * o) + sum(dS_final * S_final) it returns dL/d of
 * every input.  fp32 arithmetic (the products are not on the tensor cores).
 *   q, k, v, gate_kind, gate, beta, S0, cu_seqlens, B, T, H, dk, dv, C, dtype: as
 *            kda_chunk_fwd_ex, with gate_kind KDA_GATE_CHANNEL, KDA_GATE_SCALAR or
 *            KDA_GATE_NONE and no flags (the fused gate is not differentiated here)
 *   dO       [T_total, H, dv]  dtype      gradient of o
 *   dS_final [N, H, dk, dv]    fp32 or NULL (zero)
 *   dq, dk   [T_total, H, dk]  dtype      written
 *   dv       [T_total, H, dv]  dtype      written
 *   dgate    CHANNEL: dlog_alpha [T_total, H, dk] fp32; SCALAR: [T_total, H] fp32 (the sum
 *            over channels); NONE: ignored (may be NULL)
 *   dbeta    [T_total, H]      fp32       written
 *   dS0      [N, H, dk, dv]    fp32 or NULL (not written)
 * Workspace: taken with cudaMallocAsync on `stream` from the default pool and freed on it
 * (the pool's release threshold is raised on first use, as for kda_chunk_fwd): per 16-token
 * chunk and (head, 64-column d_v half) one block of the chunk-start fp32 state and the chunk's
 * terms the backward pass reuses -- ((dk + 32) * dvh + 544) * 4 bytes, dvh = min(dv, 64) --
 * plus (3 dk + 1) * 4 bytes per token-head per d_v half.
 * Errors: as kda_chunk_fwd_ex (KDA_ERR_GATE for the fused form or any flag), KDA_ERR_NULL for
 * dO, dq, dk, dv, dbeta (or dgate with a decay form) NULL while T_total > 0, KDA_ERR_ALIAS
 * for an output overlapping an input or another output.
 */
int kda_chunk_bwd(const void *q, const void *k, const void *v, int gate_kind, const void *gate,
                  const float *beta, const float *S0, const int32_t *cu_seqlens, const void *dO,
                  const float *dS_final, void *dq, void *dk, void *dv, float *dgate, float *dbeta,
                  float *dS0, int B, int T, int H, int dk_, int dv_, int C, int dtype,
                  kda_stream_t stream);

/*
 * kda_decode_step -- one recurrent step (one new token) for N independent sequences.
 * The recurrence of the definition above, applied once: forget, look up, correct,
 * write, read ("Ten questions" Q3-Q8; the token loop of "22,580" §6.1).
 *   q, k       [N, H, dk]        dtype
 *   v          [N, H, dv]        dtype
 *   log_alpha  [N, H, dk]        fp32
 *   beta       [N, H]            fp32
 *   S_inout    [N, H, dk, dv]    fp32   state, read and overwritten in place
 *   out        [N, H, dv]        dtype  o for the new token
 * Errors: KDA_ERR_NULL, KDA_ERR_DIM (N, H < 1; dk, dv not in {32, 64, 128}),
 * KDA_ERR_DTYPE, KDA_ERR_ALIGN, KDA_ERR_ALIAS (out or S_inout overlapping an input
 * or each other), KDA_ERR_CUDA.
 */
int kda_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                    const float *beta, float *S_inout, void *out, int N, int H, int dk,
                    int dv, int dtype, kda_stream_t stream);

/*
 * kda_decode_ex -- decode from an indexed state pool, L new tokens per sequence.
 * For each sequence n < N with idx = state_idx[n] (or n when state_idx is NULL), the
 * recurrence (in the gate form given, with flags, as in kda_chunk_fwd_ex) runs over the
 * sequence's L new tokens in order from state_pool[idx], writes o for each token and
 * stores the state back to state_pool[idx] once, after the last token.  This is the step of
 * a serving cache ("Ten questions" Q10: the state is a fixed 16,384-cell board per head
 * whatever the context length) and of multi-token (speculative) steps: one call over L
 * tokens gives exactly the results of L calls with one token each.
 *   q, k          [N, L, H, dk]     dtype
 *   v             [N, L, H, dv]     dtype
 *   gate          per gate_kind: [N, L, H, dk] fp32 / [N, L, H] fp32 / NULL / f [N, L, H, dk] dtype
 *   A_log, dt_bias  [H, dk] fp32 (KDA_GATE_FUSED only)
 *   beta          [N, L, H]         fp32 (logits with KDA_BETA_LOGIT)
 *   state_pool    [P, H, dk, dv]    fp32, read and updated in place
 *   state_idx     [N] int32 or NULL: the pool slot of each sequence.  A negative entry
 *                 skips its sequence (nothing read or written, out untouched: padding).
 *                 Entries must be distinct (two sequences on one slot race).  An entry >= P
 *                 is skipped too and recorded: the next kda_device_status() returns
 *                 KDA_ERR_INDEX.  NULL means slot n for sequence n and requires P >= N.
 *   out           [N, L, H, dv]     dtype
 * Memory-bound: each selected state is read once and written once per call.
 * Errors: KDA_ERR_NULL, KDA_ERR_DIM (N, H, L, P < 1, dk or dv not in {32, 64, 128}, P < N
 * without state_idx), KDA_ERR_DTYPE, KDA_ERR_ALIGN, KDA_ERR_ALIAS (out or state_pool
 * overlapping an input or each other), KDA_ERR_GATE, KDA_ERR_CUDA.
 */
int kda_decode_ex(const void *q, const void *k, const void *v, int gate_kind, const void *gate,
                  const float *A_log, const float *dt_bias, int flags, const float *beta,
                  float *state_pool, const int32_t *state_idx, void *out, int N, int L, int H,
                  int dk, int dv, int P, int dtype, kda_stream_t stream);

/*
 * kda_device_status -- synchronises the current device, then reports whether any
 * libkda kernel since the previous call gave up one of its bounded device-side
 * waits (tensor-core completion barriers; each waits at most about two seconds
 * and then abandons its work item instead of hanging), or skipped a kda_decode_ex
 * sequence whose state index was >= the pool size.  Clears that record.
 * Returns KDA_OK, KDA_ERR_TIMEOUT (a wait gave up; reported first), KDA_ERR_INDEX, or
 * KDA_ERR_CUDA (the synchronisation failed).
 */
int kda_device_status(void);

/*
 * kda_selftest_wait_timeout -- exercises the bounded-wait machinery without a fault.  The
 * pages have no counterpart of this call.  It launches one thread on `stream` that waits on
 * an mbarrier nothing arrives at; after about `limit_us` microseconds of SM clock it gives up
 * and records a timeout exactly as the prefill kernels do when one of their waits runs out.
 * The next kda_device_status() then returns KDA_ERR_TIMEOUT and clears the record; the CUDA
 * context stays usable.  limit_us must be in [1, 1000000] (else KDA_ERR_DIM).
 * Returns KDA_OK or KDA_ERR_CUDA (launch failure).
 */
int kda_selftest_wait_timeout(int limit_us, kda_stream_t stream);

/* A static, human-readable description of a status code.  For KDA_ERR_CUDA it names
 * the CUDA error of the calling host thread's last failed launch. */
const char *kda_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */

// C ABI of libkda.so: argument validation and dispatch.  See include/kda.h.
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "../../include/kda.h"
#include "kda_common.cuh"

namespace {

thread_local char g_cuda_msg[256] = "CUDA error";

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return KDA_OK;
    snprintf(g_cuda_msg, sizeof g_cuda_msg, "CUDA error %d (%s): %s", (int)e, cudaGetErrorName(e),
             cudaGetErrorString(e));
    return KDA_ERR_CUDA;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
bool dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

struct Span {
    uintptr_t lo, hi;  // [lo, hi)
};
Span span(const void *p, size_t bytes) { return {(uintptr_t)p, (uintptr_t)p + bytes}; }
bool overlap(Span a, Span b) { return a.lo < b.hi && b.lo < a.hi && a.lo != a.hi && b.lo != b.hi; }

constexpr int kMaxDevices = 64;
// Per-device "already done" flags: only a shortcut, the set-up call is idempotent, so two host
// threads that both find a flag clear both make it, which is harmless.
std::atomic<bool> g_pool_configured[kMaxDevices] = {};

}  // namespace

cudaError_t kda_keep_pool_memory(int dev) {
    if (dev >= 0 && dev < kMaxDevices && g_pool_configured[dev].load(std::memory_order_acquire))
        return cudaSuccess;
    cudaMemPool_t pool;
    cudaError_t e = cudaDeviceGetDefaultMemPool(&pool, dev);
    if (e != cudaSuccess) return e;
    uint64_t keep = ~0ull;
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) g_pool_configured[dev].store(true, std::memory_order_release);
    return cudaSuccess;
}

extern "C" const char *kda_status_string(int status) {
    switch (status) {
    case KDA_OK: return "KDA_OK: success";
    case KDA_ERR_NULL: return "KDA_ERR_NULL: a required pointer is NULL";
    case KDA_ERR_DIM: return "KDA_ERR_DIM: a size is out of range or unsupported";
    case KDA_ERR_CHUNK: return "KDA_ERR_CHUNK: the chunk length must be 64";
    case KDA_ERR_ALIGN: return "KDA_ERR_ALIGN: a pointer is not 16-byte aligned";
    case KDA_ERR_DTYPE: return "KDA_ERR_DTYPE: dtype must be KDA_F32 or KDA_BF16";
    case KDA_ERR_ALIAS: return "KDA_ERR_ALIAS: an output overlaps an input";
    case KDA_ERR_CUDA: return g_cuda_msg;
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a bounded device-side wait gave up";
    case KDA_ERR_SCRATCH:
        return "KDA_ERR_SCRATCH: the problem needs more workspace than the fixed scratch buffer of "
               "kda_chunk_fwd_noalloc holds (KDA_NOALLOC_SCRATCH_BYTES)";
    case KDA_ERR_GATE: return "KDA_ERR_GATE: bad gate form, flags or gate pointers";
    case KDA_ERR_INDEX: return "KDA_ERR_INDEX: a kda_decode_ex state index was >= the pool size";
    default: return "unknown kda status";
    }
}

namespace {

// Gate pointers against the gate form: the form's tensor present (absent for NONE), A_log and
// dt_bias for FUSED, known flags.  Returns KDA_OK or KDA_ERR_GATE.
int check_gate(int kind, const void *gate, const float *A_log, const float *dt_bias, int flags,
               bool have_tokens) {
    if (kind < KDA_GATE_CHANNEL || kind > KDA_GATE_FUSED) return KDA_ERR_GATE;
    if (flags & ~(KDA_NORM_Q | KDA_NORM_K | KDA_BETA_LOGIT)) return KDA_ERR_GATE;
    if (kind == KDA_GATE_NONE && gate) return KDA_ERR_GATE;
    if (kind != KDA_GATE_NONE && !gate && have_tokens) return KDA_ERR_GATE;
    if (kind == KDA_GATE_FUSED && (!A_log || !dt_bias)) return KDA_ERR_GATE;
    return KDA_OK;
}

// Bytes of the gate tensor for `rows` token-heads of dk channels.
size_t gate_bytes(int kind, size_t rows, int dk, size_t es) {
    switch (kind) {
    case KDA_GATE_CHANNEL: return rows * dk * 4;
    case KDA_GATE_SCALAR: return rows * 4;
    case KDA_GATE_FUSED: return rows * dk * es;
    default: return 0;
    }
}

// Host-side checks of a chunked-prefill call; on success fills `a`.  `plain`: the call is
// kda_chunk_fwd(_noalloc), whose log_alpha counts among the required token tensors.
// `inputs_only`: the forward's inputs of a backward call (out and S_final are not used).
int prepare_chunk(const void *q, const void *k, const void *v, int gate_kind, const void *gate,
                  const float *A_log, const float *dt_bias, int flags, const float *beta,
                  const float *S0, const int32_t *cu_seqlens, void *out, float *S_final, int B, int T,
                  int H, int dk, int dv, int C, int dtype, bool plain, KdaChunkArgs &a,
                  bool inputs_only = false) {
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_DTYPE;
    if (B < 1 || H < 1 || H > 65535 || T < 0 || !dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_DIM;
    if (C != 64) return KDA_ERR_CHUNK;
    const int64_t T_total = cu_seqlens ? (int64_t)T : (int64_t)B * T;
    // Token tensors may be NULL only when there are no tokens at all.
    if (T_total > 0 && (!q || !k || !v || !beta || (!out && !inputs_only) || (plain && !gate)))
        return KDA_ERR_NULL;
    const int g = check_gate(gate_kind, gate, A_log, dt_bias, flags, T_total > 0);
    if (g != KDA_OK) return g;
    const void *ptrs[] = {q, k, v, gate, A_log, dt_bias, beta, S0, cu_seqlens, out, S_final};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_ALIGN;

    if ((int64_t)B * H > (int64_t)INT32_MAX) return KDA_ERR_DIM;
    const size_t es = dtype == KDA_F32 ? 4 : 2;
    const size_t rows = (size_t)T_total * H;
    const size_t nk = rows * dk, nv = rows * dv;
    const size_t ns = (size_t)B * H * dk * dv;
    const Span in_q = span(q, nk * es), in_k = span(k, nk * es), in_v = span(v, nv * es);
    const Span in_g = span(gate, gate ? gate_bytes(gate_kind, rows, dk, es) : 0);
    const bool fused = gate_kind == KDA_GATE_FUSED;
    const Span in_al = span(A_log, fused ? (size_t)H * dk * 4 : 0);
    const Span in_db = span(dt_bias, fused ? (size_t)H * dk * 4 : 0);
    const Span in_b = span(beta, rows * 4);
    const Span in_s0 = span(S0, S0 ? ns * 4 : 0);
    const Span in_cu = span(cu_seqlens, cu_seqlens ? (size_t)(B + 1) * 4 : 0);
    const Span o = span(out, nv * es), sf = span(S_final, S_final ? ns * 4 : 0);
    for (Span in : {in_q, in_k, in_v, in_g, in_al, in_db, in_b, in_s0, in_cu})
        if (overlap(o, in)) return KDA_ERR_ALIAS;
    for (Span in : {in_q, in_k, in_v, in_g, in_al, in_db, in_b, in_cu, o})
        if (overlap(sf, in)) return KDA_ERR_ALIAS;
    if (S0 && S_final && overlap(in_s0, sf) && (const void *)S0 != (const void *)S_final)
        return KDA_ERR_ALIAS;

    a = KdaChunkArgs{q, k, v, gate, fused ? A_log : nullptr, fused ? dt_bias : nullptr, beta, S0,
                     cu_seqlens, out, S_final, B, T, H, dk, dv, T_total, 1.0f / sqrtf((float)dk),
                     gate_kind, flags};
    return KDA_OK;
}

int run_chunk(const KdaChunkArgs &a, int dtype, cudaStream_t st) {
    if (dtype == KDA_BF16 && kda_chunk_tc_supports(a.dk, a.dv)) return cuda_status(kda_launch_chunk_tc(a, st));
    return cuda_status(dtype == KDA_F32 ? kda_launch_chunk_simt_f32(a, st) : kda_launch_chunk_simt_bf16(a, st));
}

}  // namespace

extern "C" int kda_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                             const float *beta, const float *S0, const int32_t *cu_seqlens,
                             void *out, float *S_final, int B, int T, int H, int dk, int dv, int C,
                             int dtype, kda_stream_t stream) {
    KdaChunkArgs a;
    const int rc = prepare_chunk(q, k, v, KDA_GATE_CHANNEL, log_alpha, nullptr, nullptr, 0, beta, S0,
                                 cu_seqlens, out, S_final, B, T, H, dk, dv, C, dtype, true, a);
    if (rc != KDA_OK) return rc;
    return run_chunk(a, dtype, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int kda_chunk_fwd_ex(const void *q, const void *k, const void *v, int gate_kind,
                                const void *gate, const float *A_log, const float *dt_bias, int flags,
                                const float *beta, const float *S0, const int32_t *cu_seqlens,
                                void *out, float *S_final, int B, int T, int H, int dk, int dv, int C,
                                int dtype, kda_stream_t stream) {
    KdaChunkArgs a;
    const int rc = prepare_chunk(q, k, v, gate_kind, gate, A_log, dt_bias, flags, beta, S0, cu_seqlens,
                                 out, S_final, B, T, H, dk, dv, C, dtype, false, a);
    if (rc != KDA_OK) return rc;
    return run_chunk(a, dtype, reinterpret_cast<cudaStream_t>(stream));
}

// The same computation as kda_chunk_fwd with no device allocation: the tensor-core
// path's workspace is the library's fixed per-device scratch buffer; the other paths
// need none.  The size check runs on the host before any CUDA call.
extern "C" int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                     const float *log_alpha, const float *beta, const float *S0,
                                     const int32_t *cu_seqlens, void *out, float *S_final, int B,
                                     int T, int H, int dk, int dv, int C, int dtype,
                                     kda_stream_t stream) {
    KdaChunkArgs a;
    const int rc = prepare_chunk(q, k, v, KDA_GATE_CHANNEL, log_alpha, nullptr, nullptr, 0, beta, S0,
                                 cu_seqlens, out, S_final, B, T, H, dk, dv, C, dtype, true, a);
    if (rc != KDA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == KDA_BF16 && kda_chunk_tc_supports(dk, dv)) {
        if (kda_chunk_tc_workspace_bytes(a) > (size_t)KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_SCRATCH;
        void *scratch = nullptr;
        const cudaError_t e = kda_noalloc_scratch(&scratch);
        if (e != cudaSuccess) return cuda_status(e);
        return cuda_status(kda_launch_chunk_tc_ws(a, scratch, st));
    }
    return cuda_status(dtype == KDA_F32 ? kda_launch_chunk_simt_f32(a, st)
                                        : kda_launch_chunk_simt_bf16(a, st));
}

extern "C" int kda_chunk_bwd(const void *q, const void *k, const void *v, int gate_kind, const void *gate,
                             const float *beta, const float *S0, const int32_t *cu_seqlens, const void *dO,
                             const float *dS_final, void *dq, void *dk, void *dv, float *dgate, float *dbeta,
                             float *dS0, int B, int T, int H, int dk_, int dv_, int C, int dtype,
                             kda_stream_t stream) {
    if (gate_kind == KDA_GATE_FUSED) return KDA_ERR_GATE;
    KdaChunkArgs a;
    // the forward's inputs are validated as for kda_chunk_fwd_ex; the outputs below
    const int rc = prepare_chunk(q, k, v, gate_kind, gate, nullptr, nullptr, 0, beta, S0, cu_seqlens, nullptr,
                                 nullptr, B, T, H, dk_, dv_, C, dtype, false, a, true);
    if (rc != KDA_OK) return rc;
    const int64_t rows = a.T_total * H;
    if (rows > 0 && (!dO || !dq || !dk || !dv || !dbeta || (gate_kind != KDA_GATE_NONE && !dgate)))
        return KDA_ERR_NULL;
    const void *ptrs[] = {dO, dS_final, dq, dk, dv, dgate, dbeta, dS0};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_ALIGN;
    const size_t es = dtype == KDA_F32 ? 4 : 2;
    const size_t ns = (size_t)a.N * H * dk_ * dv_ * 4;
    const Span in[] = {span(q, rows * dk_ * es), span(k, rows * dk_ * es), span(v, rows * dv_ * es),
                       span(gate, gate ? gate_bytes(gate_kind, rows, dk_, es) : 0), span(beta, rows * 4),
                       span(S0, S0 ? ns : 0), span(cu_seqlens, cu_seqlens ? (size_t)(B + 1) * 4 : 0),
                       span(dO, rows * dv_ * es), span(dS_final, dS_final ? ns : 0)};
    const Span out[] = {span(dq, rows * dk_ * es), span(dk, rows * dk_ * es), span(dv, rows * dv_ * es),
                        span(dgate, dgate && gate_kind != KDA_GATE_NONE ? gate_bytes(gate_kind, rows, dk_, 4) : 0),
                        span(dbeta, rows * 4), span(dS0, dS0 ? ns : 0)};
    for (const Span &o : out) {
        for (const Span &i : in)
            if (overlap(o, i)) return KDA_ERR_ALIAS;
        for (const Span &o2 : out)
            if (&o != &o2 && overlap(o, o2)) return KDA_ERR_ALIAS;
    }
    if (gate_kind == KDA_GATE_NONE) dgate = nullptr;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e);
    if ((e = kda_keep_pool_memory(dev)) != cudaSuccess) return cuda_status(e);
    void *ws = nullptr;
    if ((e = cudaMallocAsync(&ws, kda_chunk_bwd_workspace_bytes(a), st)) != cudaSuccess) return cuda_status(e);
    e = kda_launch_chunk_bwd(a, dtype, dO, dS_final, dq, dk, dv, dgate, dbeta, dS0, ws, st);
    const cudaError_t f = cudaFreeAsync(ws, st);
    return cuda_status(e != cudaSuccess ? e : f);
}

namespace {

int decode_common(const void *q, const void *k, const void *v, int gate_kind, const void *gate,
                  const float *A_log, const float *dt_bias, int flags, const float *beta, float *pool,
                  const int32_t *state_idx, void *out, int N, int L, int H, int dk, int dv, int P,
                  int dtype, kda_stream_t stream) {
    if (!q || !k || !v || !beta || !pool || !out) return KDA_ERR_NULL;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_DTYPE;
    if (N < 1 || L < 1 || H < 1 || P < 1 || !dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_DIM;
    if (!state_idx && P < N) return KDA_ERR_DIM;
    if ((int64_t)N * H > (int64_t)INT32_MAX || (int64_t)P * H > (int64_t)INT32_MAX) return KDA_ERR_DIM;
    const int g = check_gate(gate_kind, gate, A_log, dt_bias, flags, true);
    if (g != KDA_OK) return g;
    const void *ptrs[] = {q, k, v, gate, A_log, dt_bias, beta, pool, state_idx, out};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_ALIGN;
    const size_t es = dtype == KDA_F32 ? 4 : 2;
    const size_t rows = (size_t)N * L * H;
    const bool fused = gate_kind == KDA_GATE_FUSED;
    const Span in_q = span(q, rows * dk * es), in_k = span(k, rows * dk * es), in_v = span(v, rows * dv * es);
    const Span in_g = span(gate, gate ? gate_bytes(gate_kind, rows, dk, es) : 0);
    const Span in_al = span(A_log, fused ? (size_t)H * dk * 4 : 0);
    const Span in_db = span(dt_bias, fused ? (size_t)H * dk * 4 : 0);
    const Span in_b = span(beta, rows * 4), in_i = span(state_idx, state_idx ? (size_t)N * 4 : 0);
    const Span s = span(pool, (size_t)P * H * dk * dv * 4), o = span(out, rows * dv * es);
    for (Span in : {in_q, in_k, in_v, in_g, in_al, in_db, in_b, in_i})
        if (overlap(s, in) || overlap(o, in)) return KDA_ERR_ALIAS;
    if (overlap(s, o)) return KDA_ERR_ALIAS;
    KdaDecodeArgs a{q, k, v, gate, fused ? A_log : nullptr, fused ? dt_bias : nullptr, beta, pool, state_idx,
                    out, N, L, H, dk, dv, P, 1.0f / sqrtf((float)dk), gate_kind, flags};
    return cuda_status(kda_launch_decode(a, dtype, reinterpret_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" int kda_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                               const float *beta, float *S_inout, void *out, int N, int H, int dk,
                               int dv, int dtype, kda_stream_t stream) {
    if (!q || !k || !v || !log_alpha || !beta || !S_inout || !out) return KDA_ERR_NULL;
    return decode_common(q, k, v, KDA_GATE_CHANNEL, log_alpha, nullptr, nullptr, 0, beta, S_inout, nullptr,
                         out, N, 1, H, dk, dv, N, dtype, stream);
}

extern "C" int kda_decode_ex(const void *q, const void *k, const void *v, int gate_kind, const void *gate,
                             const float *A_log, const float *dt_bias, int flags, const float *beta,
                             float *state_pool, const int32_t *state_idx, void *out, int N, int L, int H,
                             int dk, int dv, int P, int dtype, kda_stream_t stream) {
    return decode_common(q, k, v, gate_kind, gate, A_log, dt_bias, flags, beta, state_pool, state_idx, out,
                         N, L, H, dk, dv, P, dtype, stream);
}

extern "C" int kda_selftest_wait_timeout(int limit_us, kda_stream_t stream) {
    if (limit_us < 1 || limit_us > 1000000) return KDA_ERR_DIM;
    return cuda_status(kda_launch_wait_selftest(limit_us, reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" int kda_device_status(void) {
    unsigned int st = 0, dst = 0;
    cudaError_t e = kda_read_device_status(&st, true);           // synchronises first
    if (e != cudaSuccess) return cuda_status(e);
    if ((e = kda_decode_read_status(&dst, true)) != cudaSuccess) return cuda_status(e);
    return st ? KDA_ERR_TIMEOUT : (dst ? KDA_ERR_INDEX : KDA_OK);
}

// C ABI of libkda.so: argument validation and dispatch.  See include/kda.h.
#include <stdio.h>
#include <string.h>

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

}  // namespace

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
    default: return "unknown kda status";
    }
}

namespace {

// Host-side checks of a chunked-prefill call; on success fills `a`.
int prepare_chunk(const void *q, const void *k, const void *v, const float *log_alpha,
                  const float *beta, const float *S0, const int32_t *cu_seqlens, void *out,
                  float *S_final, int B, int T, int H, int dk, int dv, int C, int dtype,
                  KdaChunkArgs &a) {
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_DTYPE;
    if (B < 1 || H < 1 || H > 65535 || T < 0 || !dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_DIM;
    if (C != 64) return KDA_ERR_CHUNK;
    const int64_t T_total = cu_seqlens ? (int64_t)T : (int64_t)B * T;
    // Token tensors may be NULL only when there are no tokens at all.
    if (T_total > 0 && (!q || !k || !v || !log_alpha || !beta || !out)) return KDA_ERR_NULL;
    const void *ptrs[] = {q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_ALIGN;

    if ((int64_t)B * H > (int64_t)INT32_MAX) return KDA_ERR_DIM;
    const size_t es = dtype == KDA_F32 ? 4 : 2;
    const size_t nk = (size_t)T_total * H * dk, nv = (size_t)T_total * H * dv;
    const size_t ns = (size_t)B * H * dk * dv;
    const Span in_q = span(q, nk * es), in_k = span(k, nk * es), in_v = span(v, nv * es);
    const Span in_la = span(log_alpha, nk * 4), in_b = span(beta, (size_t)T_total * H * 4);
    const Span in_s0 = span(S0, S0 ? ns * 4 : 0);
    const Span in_cu = span(cu_seqlens, cu_seqlens ? (size_t)(B + 1) * 4 : 0);
    const Span o = span(out, nv * es), sf = span(S_final, S_final ? ns * 4 : 0);
    for (Span in : {in_q, in_k, in_v, in_la, in_b, in_s0, in_cu})
        if (overlap(o, in)) return KDA_ERR_ALIAS;
    for (Span in : {in_q, in_k, in_v, in_la, in_b, in_cu, o})
        if (overlap(sf, in)) return KDA_ERR_ALIAS;
    if (S0 && S_final && overlap(in_s0, sf) && (const void *)S0 != (const void *)S_final)
        return KDA_ERR_ALIAS;

    a = KdaChunkArgs{q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, B, T, H, dk, dv,
                     T_total, 1.0f / sqrtf((float)dk)};
    return KDA_OK;
}

}  // namespace

extern "C" int kda_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                             const float *beta, const float *S0, const int32_t *cu_seqlens,
                             void *out, float *S_final, int B, int T, int H, int dk, int dv, int C,
                             int dtype, kda_stream_t stream) {
    KdaChunkArgs a;
    const int rc = prepare_chunk(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, B, T, H,
                                 dk, dv, C, dtype, a);
    if (rc != KDA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == KDA_BF16 && kda_chunk_tc_supports(dk, dv)) return cuda_status(kda_launch_chunk_tc(a, st));
    return cuda_status(dtype == KDA_F32 ? kda_launch_chunk_simt_f32(a, st)
                                        : kda_launch_chunk_simt_bf16(a, st));
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
    const int rc = prepare_chunk(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, B, T, H,
                                 dk, dv, C, dtype, a);
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

extern "C" int kda_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                               const float *beta, float *S_inout, void *out, int N, int H, int dk,
                               int dv, int dtype, kda_stream_t stream) {
    if (!q || !k || !v || !log_alpha || !beta || !S_inout || !out) return KDA_ERR_NULL;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_DTYPE;
    if (N < 1 || H < 1 || !dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_DIM;
    if ((int64_t)N * H > (int64_t)INT32_MAX) return KDA_ERR_DIM;
    const void *ptrs[] = {q, k, v, log_alpha, beta, S_inout, out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_ALIGN;
    const size_t es = dtype == KDA_F32 ? 4 : 2;
    const size_t P = (size_t)N * H;
    const Span in_q = span(q, P * dk * es), in_k = span(k, P * dk * es), in_v = span(v, P * dv * es);
    const Span in_la = span(log_alpha, P * dk * 4), in_b = span(beta, P * 4);
    const Span s = span(S_inout, P * dk * dv * 4), o = span(out, P * dv * es);
    for (Span in : {in_q, in_k, in_v, in_la, in_b}) {
        if (overlap(s, in) || overlap(o, in)) return KDA_ERR_ALIAS;
    }
    if (overlap(s, o)) return KDA_ERR_ALIAS;
    KdaDecodeArgs a{q, k, v, log_alpha, beta, S_inout, out, N, H, dk, dv, 1.0f / sqrtf((float)dk)};
    return cuda_status(kda_launch_decode(a, dtype, reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" int kda_selftest_wait_timeout(int limit_us, kda_stream_t stream) {
    if (limit_us < 1 || limit_us > 1000000) return KDA_ERR_DIM;
    return cuda_status(kda_launch_wait_selftest(limit_us, reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" int kda_device_status(void) {
    unsigned int st = 0;
    const cudaError_t e = kda_read_device_status(&st, true);
    if (e != cudaSuccess) return cuda_status(e);
    return st ? KDA_ERR_TIMEOUT : KDA_OK;
}

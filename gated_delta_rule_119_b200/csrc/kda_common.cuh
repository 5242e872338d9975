// Shared device helpers of libkda.so (element conversion, launch bookkeeping).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);  // round to nearest even
}

// Sequence bounds on the packed token axis, clamped to [0, T_total] so that a
// malformed cu_seqlens can never make a kernel read or write out of bounds.
__device__ __forceinline__ void seq_bounds(const int32_t *cu_seqlens, int n, int T,
                                           int64_t T_total, int64_t &t0, int64_t &t1) {
    if (cu_seqlens == nullptr) {
        t0 = (int64_t)n * T;
        t1 = t0 + T;
        return;
    }
    int64_t a = cu_seqlens[n], b = cu_seqlens[n + 1];
    a = a < 0 ? 0 : (a > T_total ? T_total : a);
    b = b < a ? a : (b > T_total ? T_total : b);
    t0 = a;
    t1 = b;
}

// Gate forms and flags (the kda_gate_kind / kda_gate_flags values of include/kda.h).
enum : int { GATE_CHANNEL = 0, GATE_SCALAR = 1, GATE_NONE = 2, GATE_FUSED = 3 };
enum : int { FLAG_NORM_Q = 1, FLAG_NORM_K = 2, FLAG_BETA_LOGIT = 4 };
constexpr float kFusedLogAlphaMin = -1e4f;   // alpha = e^-1e4 is 0 in fp32

// ln(1 + e^x) in fp32 as max(x, 0) + ln(1 + t) with t = e^-|x| in (0, 1], and
// ln(1 + t) = 2 atanh(z), z = t / (2 + t) in (0, 1/3], summed as the odd series
// 2 (z + z^3/3 + ... + z^13/13): the first term left out, 2 z^15 / 15, is below 5e-9 for z <= 1/3.
// One exponential, one division and seven multiply-adds per value.
__device__ __forceinline__ float softplus(float x) {
    const float t = __expf(-fabsf(x));
    const float z = __fdividef(t, 2.f + t);
    const float z2 = z * z;
    float p = 1.f / 13.f;
    p = fmaf(p, z2, 1.f / 11.f);
    p = fmaf(p, z2, 1.f / 9.f);
    p = fmaf(p, z2, 1.f / 7.f);
    p = fmaf(p, z2, 1.f / 5.f);
    p = fmaf(p, z2, 1.f / 3.f);
    p = fmaf(p, z2, 1.f);
    return fmaxf(x, 0.f) + 2.f * z * p;
}

// The fused gate of "Ten questions" Q9: log alpha = -exp(A_log) softplus(f + dt_bias), given
// e^A_log (computed once per channel by the caller that reuses it).
__device__ __forceinline__ float fused_log_alpha_e(float f, float exp_A_log, float dt_bias) {
    return fmaxf(-exp_A_log * softplus(f + dt_bias), kFusedLogAlphaMin);
}
__device__ __forceinline__ float fused_log_alpha(float f, float A_log, float dt_bias) {
    return fused_log_alpha_e(f, expf(A_log), dt_bias);
}

__device__ __forceinline__ float beta_of(float b, int flags) {
    return (flags & FLAG_BETA_LOGIT) ? 1.f / (1.f + expf(-b)) : b;
}

// log alpha of channel c at token-head row th (= t * H + h) for any gate form; Tin is the
// input dtype (the type of f for the fused form).
template <typename Tin>
__device__ __forceinline__ float gate_log_alpha(int kind, const void *gate, const float *A_log,
                                                const float *dt_bias, size_t th, int h, int c, int dk) {
    switch (kind) {
    case GATE_CHANNEL: return static_cast<const float *>(gate)[th * dk + c];
    case GATE_SCALAR: return static_cast<const float *>(gate)[th];
    case GATE_FUSED:
        return fused_log_alpha(to_f32(static_cast<const Tin *>(gate)[th * dk + c]), A_log[(size_t)h * dk + c],
                               dt_bias[(size_t)h * dk + c]);
    default: return 0.f;
    }
}

}  // namespace kda

// Host-side launchers (defined in the kernel files, called by kda_api.cu).
struct KdaChunkArgs {
    const void *q, *k, *v;
    const void *gate;                 // log_alpha (CHANNEL, SCALAR) or f (FUSED); NULL for NONE
    const float *A_log, *dt_bias;     // [H, dk], FUSED only
    const float *beta, *S0;
    const int32_t *cu_seqlens;
    void *out;
    float *S_final;
    int N, T, H, dk, dv;
    int64_t T_total;
    float scale;
    int gate_kind, flags;
};

struct KdaDecodeArgs {
    const void *q, *k, *v;
    const void *gate;
    const float *A_log, *dt_bias;
    const float *beta;
    float *S;                         // the state pool [P, H, dk, dv]
    const int32_t *state_idx;         // [N] or NULL (slot n)
    void *out;
    int N, L, H, dk, dv, P;
    float scale;
    int gate_kind, flags;
};

cudaError_t kda_launch_decode(const KdaDecodeArgs &a, int dtype, cudaStream_t stream);
cudaError_t kda_launch_chunk_simt_f32(const KdaChunkArgs &a, cudaStream_t stream);
cudaError_t kda_launch_chunk_simt_bf16(const KdaChunkArgs &a, cudaStream_t stream);
cudaError_t kda_launch_chunk_tc(const KdaChunkArgs &a, cudaStream_t stream);
bool kda_chunk_tc_supports(int dk, int dv);
size_t kda_chunk_tc_workspace_bytes(const KdaChunkArgs &a);
cudaError_t kda_launch_chunk_tc_ws(const KdaChunkArgs &a, void *ws, cudaStream_t stream);
// Device address of the fixed scratch buffer of the current device (kda_noalloc.cu).
cudaError_t kda_noalloc_scratch(void **ptr);
size_t kda_chunk_bwd_workspace_bytes(const KdaChunkArgs &a);
cudaError_t kda_launch_chunk_bwd(const KdaChunkArgs &a, int dtype, const void *dO, const float *dS_final,
                                 void *dq, void *dk, void *dv, float *dgate, float *dbeta, float *dS0,
                                 void *ws, cudaStream_t stream);
cudaError_t kda_read_device_status(unsigned int *status, bool clear);
cudaError_t kda_decode_read_status(unsigned int *status, bool clear);
// Raises the release threshold of device `dev`'s default memory pool once, so that workspace
// freed with cudaFreeAsync stays in the pool between calls (kda_api.cu).
cudaError_t kda_keep_pool_memory(int dev);
cudaError_t kda_launch_wait_selftest(int limit_us, cudaStream_t stream);

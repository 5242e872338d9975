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

}  // namespace kda

// Host-side launchers (defined in the kernel files, called by kda_api.cu).
struct KdaChunkArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    const int32_t *cu_seqlens;
    void *out;
    float *S_final;
    int N, T, H, dk, dv;
    int64_t T_total;
    float scale;
};

struct KdaDecodeArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta;
    float *S;
    void *out;
    int N, H, dk, dv;
    float scale;
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
cudaError_t kda_read_device_status(unsigned int *status, bool clear);
cudaError_t kda_launch_wait_selftest(int limit_us, cudaStream_t stream);

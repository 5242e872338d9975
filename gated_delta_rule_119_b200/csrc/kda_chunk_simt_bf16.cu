// bf16-input instantiations of the SIMT chunk path (kda_chunk_simt.cuh): fp32
// arithmetic on bf16 q, k, v for the head sizes the tensor-core path does not take.
#include "kda_chunk_simt.cuh"

cudaError_t kda_launch_chunk_simt_bf16(const KdaChunkArgs &a, cudaStream_t stream) {
    return kda_simt::pick_dk<__nv_bfloat16>(a, stream);
}

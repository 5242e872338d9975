// fp32 instantiations of the SIMT chunk path (kda_chunk_simt.cuh).
#include "kda_chunk_simt.cuh"

cudaError_t kda_launch_chunk_simt_f32(const KdaChunkArgs &a, cudaStream_t stream) {
    return kda_simt::pick_dk<float>(a, stream);
}

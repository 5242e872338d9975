// Tensor-core (tcgen05) chunk path: placeholder until the kernel lands.
#include "kda_common.cuh"

bool kda_chunk_tc_supports(int, int) { return false; }
cudaError_t kda_launch_chunk_tc(const KdaChunkArgs &, cudaStream_t) { return cudaErrorNotSupported; }

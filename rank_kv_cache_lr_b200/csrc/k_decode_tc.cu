// Tensor-core (tcgen05) decode path: placeholder until the kernel lands.
#include "lr_internal.cuh"

bool tc_supported(const lr_cache_desc*) { return false; }
cudaError_t tc_prepare(lr_cache*) { return cudaSuccess; }
void tc_release(lr_cache*) {}
cudaError_t launch_qproj_tc(const lr_cache*, const void*, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_decode_tc(const lr_cache*, int, int, cudaStream_t) { return cudaErrorNotSupported; }

// chunk_sm100.cu -- placeholder until the tensor-core chunk kernel lands.
#include "gdn_internal.cuh"

namespace gdn {

__device__ unsigned int g_status_word = 0;

cudaError_t launch_chunk_sm100(const Problem&, cudaStream_t) { return cudaErrorNotSupported; }

cudaError_t read_and_clear_status(unsigned int* status, cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(status, g_status_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_status_word, &zero, sizeof(unsigned int));
}

}  // namespace gdn

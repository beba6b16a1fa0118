// chunk.cu -- chunkwise forward / backward (placeholder until the kernels land).
#include "kernels.h"

namespace muir {

size_t chunk_fwd_ws_bytes(int, int, int, int, int, bool) { return 0; }
size_t chunk_bwd_ws_bytes(int, int, int, int, int, bool) { return 0; }

cudaError_t run_chunk_fwd(const ChunkProblem&, const float*, void*, float*, float*, void*,
                          size_t, cudaStream_t) {
    return cudaErrorNotSupported;
}
cudaError_t run_chunk_bwd(const ChunkProblem&, const float*, const float*, const void*,
                          const float*, void*, void*, void*, void*, void*, void*, void*, float*,
                          void*, size_t, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace muir

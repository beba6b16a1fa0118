// chunk_bf16_d64.cu -- chunkwise forward/backward instantiated for __nv_bfloat16 inputs, d = 64.
#include "chunk_impl.cuh"
#include "chunk_units.h"

namespace muir {

cudaError_t fwd_bf16_d64(const ChunkProblem& P, const float* S0, void* o, float* S_final,
                          float* S_chunks, float* M_chunks, void* ws, cudaStream_t st) {
    return fwd_impl<__nv_bfloat16, 64, 1, 0>(P, S0, o, S_final, S_chunks, M_chunks, ws, st);
}

cudaError_t bwd_bf16_d64(const ChunkProblem& P, const float* S0, const float* S_chunks,
                          const float* M_chunks, const void* dO, const float* dS_final, void* dq, void* dk, void* dv,
                          void* dg, void* de, void* dw, void* dgamma, float* dS0, void* ws,
                          cudaStream_t st) {
    return bwd_impl<__nv_bfloat16, 64, 1, 0>(P, S0, S_chunks, M_chunks, dO, dS_final, dq, dk, dv, dg, de, dw, dgamma,
                                   dS0, ws, st);
}

unsigned int timeouts_bf16_d64() { return take_wait_timeouts(); }

}  // namespace muir

// chunk_units.h -- per-(dtype, head dim) instantiations of the chunk path.
#pragma once

#include "kernels.h"

namespace muir {

cudaError_t fwd_bf16_d128(const ChunkProblem& P, const float* S0, void* o, float* S_final,
                          float* S_chunks, float* M_chunks, void* ws, cudaStream_t st);
cudaError_t bwd_bf16_d128(const ChunkProblem& P, const float* S0, const float* S_chunks,
                          const float* M_chunks, const void* dO, const float* dS_final, void* dq, void* dk, void* dv,
                          void* dg, void* de, void* dw, void* dgamma, float* dS0, void* ws,
                          cudaStream_t st);
cudaError_t fwd_bf16_d64(const ChunkProblem& P, const float* S0, void* o, float* S_final,
                          float* S_chunks, float* M_chunks, void* ws, cudaStream_t st);
cudaError_t bwd_bf16_d64(const ChunkProblem& P, const float* S0, const float* S_chunks,
                          const float* M_chunks, const void* dO, const float* dS_final, void* dq, void* dk, void* dv,
                          void* dg, void* de, void* dw, void* dgamma, float* dS0, void* ws,
                          cudaStream_t st);
cudaError_t fwd_f32_d128(const ChunkProblem& P, const float* S0, void* o, float* S_final,
                          float* S_chunks, float* M_chunks, void* ws, cudaStream_t st);
cudaError_t bwd_f32_d128(const ChunkProblem& P, const float* S0, const float* S_chunks,
                          const float* M_chunks, const void* dO, const float* dS_final, void* dq, void* dk, void* dv,
                          void* dg, void* de, void* dw, void* dgamma, float* dS0, void* ws,
                          cudaStream_t st);
cudaError_t fwd_f32_d64(const ChunkProblem& P, const float* S0, void* o, float* S_final,
                          float* S_chunks, float* M_chunks, void* ws, cudaStream_t st);
cudaError_t bwd_f32_d64(const ChunkProblem& P, const float* S0, const float* S_chunks,
                          const float* M_chunks, const void* dO, const float* dS_final, void* dq, void* dk, void* dv,
                          void* dg, void* de, void* dw, void* dgamma, float* dS0, void* ws,
                          cudaStream_t st);

// Expired bounded waits recorded by each unit's kernels since the last call.
unsigned int timeouts_bf16_d128();
unsigned int timeouts_bf16_d64();
unsigned int timeouts_f32_d128();
unsigned int timeouts_f32_d64();

}  // namespace muir

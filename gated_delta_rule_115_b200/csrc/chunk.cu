// chunk.cu -- workspace sizing and dtype / head-dim dispatch of the chunkwise
// forward and backward.  The kernels live in chunk_impl.cuh and are
// instantiated in chunk_{bf16,f32}_d{64,128}.cu.
#include "chunk_impl.cuh"
#include "chunk_units.h"

namespace muir {

size_t chunk_aux_floats(int C, int D) { return make_aux_lay(C, D).total; }

size_t chunk_fwd_ws_bytes(int B, int T, int H, int D, int C, bool have_states) {
    const size_t nch = (size_t)B * H * ((T + C - 1) / C), DD = (size_t)D * D;
    size_t f = 2 * nch * DD;               // M, Bn
    if (!have_states) f += nch * DD;       // chunk-start states
    f += (size_t)num_slots((int)nch) * slot_floats(C, D);
    f += tail_side_floats(B, T, H, D, C);
    return f * sizeof(float);
}

size_t chunk_bwd_ws_bytes(int B, int T, int H, int D, int C, bool have_states) {
    const size_t nch = (size_t)B * H * ((T + C - 1) / C), DD = (size_t)D * D;
    size_t f = 3 * nch * DD;               // M, Bn / B', dS at chunk ends
    if (!have_states) f += nch * DD;
    f += (size_t)num_slots((int)nch) * slot_floats(C, D);
    f += tail_side_floats(B, T, H, D, C);
    return f * sizeof(float);
}

cudaError_t run_chunk_fwd(const ChunkProblem& P, const float* S0, void* o, float* S_final,
                          float* S_chunks, float* M_chunks, void* ws, size_t, cudaStream_t st) {
    if (P.in_bf16) {
        if (P.D == 128) return fwd_bf16_d128(P, S0, o, S_final, S_chunks, M_chunks, ws, st);
        return fwd_bf16_d64(P, S0, o, S_final, S_chunks, M_chunks, ws, st);
    }
    if (P.D == 128) return fwd_f32_d128(P, S0, o, S_final, S_chunks, M_chunks, ws, st);
    return fwd_f32_d64(P, S0, o, S_final, S_chunks, M_chunks, ws, st);
}

cudaError_t run_chunk_bwd(const ChunkProblem& P, const float* S0, const float* S_chunks,
                          const float* M_chunks, const void* dO, const float* dS_final, void* dq, void* dk, void* dv,
                          void* dg, void* de, void* dw, void* dgamma, float* dS0, void* ws,
                          size_t, cudaStream_t st) {
#define MUIR_BWD_ARGS P, S0, S_chunks, M_chunks, dO, dS_final, dq, dk, dv, dg, de, dw, dgamma, dS0, ws, st
    if (P.in_bf16) {
        if (P.D == 128) return bwd_bf16_d128(MUIR_BWD_ARGS);
        return bwd_bf16_d64(MUIR_BWD_ARGS);
    }
    if (P.D == 128) return bwd_f32_d128(MUIR_BWD_ARGS);
    return bwd_f32_d64(MUIR_BWD_ARGS);
#undef MUIR_BWD_ARGS
}

}  // namespace muir

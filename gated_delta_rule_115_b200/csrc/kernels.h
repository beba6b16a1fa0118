// kernels.h -- internal launchers of libmuir (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace muir {

cudaError_t launch_decode(int B, int H, int D, bool in_bf16, bool out_bf16, const void* q,
                          const void* k, const void* v, const void* g, const void* e,
                          const void* w, const void* gamma, int gamma_static, float* S,
                          void* o, cudaStream_t st);

// q/k feature prologue y = SiLU(x) / ||SiLU(x)|| per row of d (bwd: dx from x, dy).
cudaError_t launch_qk_prologue(long long rows, int d, bool bf16, const void* x, const void* dy,
                               void* out, bool bwd, cudaStream_t st);

// Problem description shared by the chunk kernels.
struct ChunkProblem {
    int B, T, H, D, C;     // D = dk = dv
    int N;                 // chunks per sequence, ceil(T / C); the last one may be ragged
    bool in_bf16, out_bf16;
    const void *q, *k, *v, *g, *e, *w, *gamma;
    float* aux;            // per-chunk saved intermediates (forward: written; backward: read) or null
    const int* gate;       // non-null: every kernel returns at once unless *gate != 0
    // Stages fused around the recurrence (on-chip path only; all off by default):
    const void* zo = nullptr;   // output gate pre-activation [B][T][H][D] bf16, or null
    void* o_pre = nullptr;      // forward: pre-gate output (out dtype) or null; backward: read
    bool o_pre_f32 = false;     // dtype of o_pre in the backward
    void* dzo = nullptr;        // backward: gradient of zo (bf16)
    int qk_raw = 0;             // q, k hold raw x; SiLU and the unit L2 norm are fused
    char* fused_ws = nullptr;   // fused_ws_bytes() of workspace for the stages above
    const void* gate_proj = nullptr;  // v2::GatesArgs: gates projected from a latent (gates.cu)
};

// Workspace the fused stages add (inverse row norms, materialised q^ / k^ and
// the mixer's dO for the large-span fallback; with raw q/k, fp32 copies of the
// fallback's eight inputs and seven gradients).
inline size_t fused_ws_bytes(int B, int T, int H, int D, int C, bool qk_raw) {
    const size_t nch = (size_t)B * H * ((T + C - 1) / C);
    const size_t rows = (size_t)B * T * H;
    return 256 + nch * 2 * C * 4 + 3 * rows * D * 2 + (qk_raw ? 15 * rows * D * 4 : 0);
}
// Offset of the fp32 region inside the fused workspace.
inline size_t fused_f32_offset(int B, int T, int H, int D, int C) {
    return fused_ws_bytes(B, T, H, D, C, false);
}

// Self-test of the bounded device waits (selftest.cu): one block waits
// limit_us microseconds on a barrier nothing arrives on and records the expiry.
cudaError_t launch_expired_wait(int limit_us, cudaStream_t st);
unsigned int timeouts_selftest();

// Flag-gated helpers of the fused stages (fused.cu): each returns at once
// unless *flag != 0 (the large-span fallback ran and needs them).
cudaError_t qk_materialise_gated(const int* flag, const void* x, void* y, long long rows,
                                 bool f32_out, cudaStream_t st);
cudaError_t qk_jacobian_gated(const int* flag, const void* x, const void* dy, bool dy_f32,
                              void* dx, long long rows, cudaStream_t st);
cudaError_t upcast_gated(const int* flag, const void* src, float* dst, long long n, bool src_f16,
                         cudaStream_t st);
cudaError_t downcast_gated(const int* flag, const float* src, void* dst, long long n, cudaStream_t st);
cudaError_t out_gate_fix_gated(const int* flag, void* o, void* o_pre, const void* z, long long n,
                               bool out_bf16, cudaStream_t st);

// Up to eight tensors moved between token-major [B][T][H][D] rows of the
// ragged last chunk and a side buffer [B*H][C][D] (tail.cu).
struct TailCopy {
    const void* src[8];
    void* dst[8];
    int n;
};
// token-major -> side buffer (rows past the tail zeroed) / side -> token-major
// (tail rows only); esize = bytes per element.
cudaError_t tail_gather(const TailCopy& io, int B, int H, int T, int C, int D, int esize,
                        cudaStream_t st);
cudaError_t tail_scatter(const TailCopy& io, int B, int H, int T, int C, int D, int esize,
                         cudaStream_t st);

// Floats per chunk of the saved intermediates (muir_chunk_aux_floats).
size_t chunk_aux_floats(int C, int D);

// Workspace carving (bytes) for the chunk forward / backward.
size_t chunk_fwd_ws_bytes(int B, int T, int H, int D, int C, bool have_states, bool in_bf16);
size_t chunk_bwd_ws_bytes(int B, int T, int H, int D, int C, bool have_states, bool in_bf16);
size_t chunk_aux_total_floats(int B, int T, int H, int D, int C, bool in_bf16);

cudaError_t run_chunk_fwd(const ChunkProblem& P, const float* S0, void* o, float* S_final,
                          float* S_chunks, float* M_chunks, void* ws, size_t ws_bytes,
                          cudaStream_t st);
cudaError_t run_chunk_bwd(const ChunkProblem& P, const float* S0, const float* S_chunks,
                          const float* M_chunks, const void* dO, const float* dS_final, void* dq, void* dk, void* dv,
                          void* dg, void* de, void* dw, void* dgamma, float* dS0, void* ws,
                          size_t ws_bytes, cudaStream_t st);

}  // namespace muir

// fwd2.h -- internal interface of the tensor-core chunk path with on-chip
// intermediates (bf16 inputs, dk = dv = 128, chunk 128); not part of the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>

namespace muir {
namespace v2 {

// Per-chunk fp32 arrays are indexed by chunk c = (b * H + h) * N + n, each
// chunk a row-major 128 x 128 block.
struct IntraParams {
    CUtensorMap tq, tk, tv, tg, te, tw, tgam;  // token-major [B*T][H][128] bf16
    int B, T, H;
    float* M;      // chunk transitions M_n [j][i]: S_{n+1} = M_n S_n + B_n
    float* Mt;     // M_n transposed (optional)
    float* Bn;     // B_n [j][c]
    float* Qp;     // Q'_n [t][i]: O_n = Q'_n S_n + O_intra_n
    float* Oi;     // O_intra_n [t][c]
    int* flags;
};

struct ChainParams {
    CUtensorMap tM;      // transitions, rows of 128 fp32
    const float* Bn;
    const float* S0;     // [B*H][128][128] or null
    float* S_chunks;     // [B*H][N][128][128] or null
    float* S_final;      // [B*H][128][128] or null
    int N;
};

struct OutParams {
    CUtensorMap tQ;      // Q' rows of 128 fp32
    int B, T, H;
    const float* S_chunks;
    const float* Oi;
    void* o;             // token-major [B][T][H][128], fp32 or bf16
};

struct Fwd2Args {
    int B, T, H;
    bool out_bf16;
    const void *q, *k, *v, *g, *e, *w, *gamma;
    const float* S0;
    void* o;             // may be null (state pass only)
    float* S_final;      // may be null
    float* S_chunks;     // required
    float *M, *Mt, *Bn, *Qp, *Oi;
    int* flags;
};

bool fwd2_supported(int B, int T, int H, int D, int C, bool in_bf16);
size_t fwd2_ws_bytes(int B, int T, int H);
cudaError_t span_check(const void* g, int B, int T, int H, int* flags, cudaStream_t st);
cudaError_t run_fwd2(const Fwd2Args& a, cudaStream_t st);
unsigned int timeouts_v2();

}  // namespace v2
}  // namespace muir

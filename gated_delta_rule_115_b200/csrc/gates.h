// gates.h -- the fused low-rank gate projection on the tensor cores (gates.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace muir {
namespace v2 {

// One gate family of the projection: latent columns off .. off + r (r = 64
// or 128), up-projection U [r][H*128] bf16, bias [H*128] fp32, activation.
enum GateAct : int { kActNegSoftplus = 0, kActSigmoid = 1, kActIdentity = 2 };

struct GateFamily {
    int off, r, act;
    const void* U;
    const float* bias;
    void* out;        // forward: the gate [rows][H][128] bf16
    const void* dout; // backward: its gradient [rows][H][128] bf16
    void* dpre;       // backward: dpre [rows][H][128] as bf16 hi ...
    void* dpre_lo;    // ... plus bf16 lo (dpre - hi), both workspace
    float* dU;        // backward: [r][H*128] fp32
    float* dbias;     // backward: [H*128] fp32
};

struct GatesArgs {
    int nfam;
    GateFamily fam[5];
    const void* latent;  // [rows][R] bf16
    int R, H;
    long long rows;      // B * T, a multiple of 128
    void* dlatent;       // backward: [rows][R] bf16 (columns of no family are zeroed)
};

cudaError_t run_gates_fwd(const GatesArgs& a, cudaStream_t st);
cudaError_t run_gates_bwd(const GatesArgs& a, cudaStream_t st);
unsigned int timeouts_gates();

}  // namespace v2
}  // namespace muir

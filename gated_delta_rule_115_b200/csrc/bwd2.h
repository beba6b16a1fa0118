// bwd2.h -- internal interface of the tensor-core chunk backward with on-chip
// intermediates (companion of fwd2.h); not part of the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>

namespace muir {
namespace v2 {

struct BprepParams {
    CUtensorMap tdO;
    int T, H;
    const float* Qp;  // [nch][128][128]
    float* Bp;        // Q'^T dO per chunk (grp4 layout)
    // fused output gate (zo non-null): tdO holds the gradient of the gated
    // output; dO = dO' sigmoid(zo) is written to dO_eff as fp16 (read by the
    // later kernels) and as bf16 to dO_effb (for the boundary-pivot path), and
    // dzo = dO' o_pre sigmoid'(zo) to dzo (bf16)
    const void* zo;
    const void* o_pre;
    bool o_pre_f32;
    void* dO_eff;
    void* dO_effb;
    void* dzo;
};

struct RevParams {
    CUtensorMap tMt;        // M_n^T rows of 128 fp32
    const float* Bp;
    const float* S_chunks;  // chunk-start states
    const float* S_last;    // [B*H][128][128] final states (S_N)
    const float* dS_final;  // or null
    float* dSc;             // G_{n+1} per chunk (grp4 layout)
    float* dS0;             // or null
    float* dgb;             // dLbar partials [128 / SLAB][nch][128]
    int N, nch;
};

struct Bwd1Params {
    CUtensorMap tdO, tg;                  // dO, and g (the log decay) as token-major bf16 tiles
    CUtensorMap tv, tw, tdv, tdw;         // v, w in and dv, dw out, as token-major bf16 tiles
    int B, T, H;
    const void *q, *k, *v, *g, *e, *w, *gamma;
    const unsigned char* aux;
    const float* S_chunks;
    const float* dSc;
    // state-side partials as fp16, per chunk [16 channel groups of 8][128 rows][8],
    // with one power-of-two scale per row and 32-channel group ([nch][4][128] fp32)
    __half *Pq, *Pk, *Pa, *Pd;
    float *sq, *sk, *sa, *sd;
    unsigned char *Y16, *dYR16;
    void *dv, *dw;
    bool dO_f16;                          // tdO holds fp16 (the fused gate's dO), else bf16
};

struct Bwd2Params {
    CUtensorMap tdO, tg;
    CUtensorMap tk, te, tq, tgam;         // the readout's inputs (token-major bf16 tiles)
    CUtensorMap tdq, tdk, tdgam, tde;     // its outputs, stored as tiles (tdq, tdk unused with raw q/k)
    int B, T, H;
    const void *q, *k, *g, *e, *gamma;
    const unsigned char* aux;
    const unsigned char *Y16, *dYR16;
    const __half *Pq, *Pk, *Pa, *Pd;      // k2_bwd1's partials (scaled fp16, see Bwd1Params)
    const float *sq, *sk, *sa, *sd;
    float *dqh, *dkh;                     // fused prologue: dq^, dk^ before its Jacobian (fp32, grp4 layout)
    const float* dgb;                     // [nslab][nch][128] partials of dLbar
    int nslab;
    void *dq, *dk, *dg, *de, *dgamma;
    const float* rnorm;                   // fused prologue: [nch][2][128] inverse row norms
    int* flags;                           // flags[0] |= 1 when a chunk's decay span exceeds the single pivot
    bool dO_f16;                          // tdO holds fp16 (the fused gate's dO), else bf16
};

struct Bwd2Args {
    int B, T, H;
    const void *q, *k, *v, *g, *e, *w, *gamma, *dO;
    const void* zo;                         // fused output gate: pre-activation, or null
    const void* o_pre;                      // with zo: the forward's pre-gate output
    bool o_pre_f32;                         // its dtype (fp32, else bf16)
    void* dO_eff;                           // with zo: B*T*H*128 fp16 of workspace
    void* dO_effb;                          // with zo: the same as bf16 (boundary-pivot path)
    void* dzo;                              // with zo: gradient of zo (bf16)
    const float* rnorm;                     // fused q/k prologue: the forward's inverse row norms, or null
    const float* dS_final;                  // or null
    const unsigned char* aux;               // forward's saved records
    const float *Qp, *Mt, *S_chunks, *S_last;
    void *dq, *dk, *dv, *dg, *de, *dw, *dgamma;
    float* dS0;                             // or null
    void* ws;                               // bwd2_ws_bytes
    int* flags;                             // raised when a chunk exceeds the single pivot
};

size_t bwd2_ws_bytes(int B, int T, int H);
cudaError_t run_bwd2(const Bwd2Args& a, cudaStream_t st);
// Bitmask of the wait sites whose bounded wait expired since the last call (then cleared).
unsigned int timeouts_bwd2();

// Tensor maps shared with fwd2.cu.
bool map_tokens16(CUtensorMap* m, const void* base, int B, int T, int H);
bool map_rows32f(CUtensorMap* m, const float* base, long long rows);
bool map_2d16(CUtensorMap* m, const void* base, long long cols, long long rows, int box_rows);

}  // namespace v2
}  // namespace muir

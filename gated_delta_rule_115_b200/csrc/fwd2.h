// fwd2.h -- internal interface of the tensor-core chunk path with on-chip
// intermediates (bf16 inputs, dk = dv = 128, chunk 128); not part of the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>

namespace muir {
namespace v2 {

// Per-chunk fp32 arrays are indexed by chunk c = (b * H + h) * N + n, each
// chunk a 128 x 128 block: row-major, or 4-column-group-major where a field
// says grp4 (tc2.cuh).

// Per-chunk intermediates the forward saves for the backward ("aux"), byte
// offsets inside one chunk's record.  16-bit tiles are stored byte for byte in
// the 128B-swizzled shared-memory tile layout (tc2.cuh, T16) so the backward
// reloads them with plain bulk copies; the fp32 block is 4-column-group-major
// (tc2.cuh, grp4).
struct AuxLayout {
    static constexpr size_t kT16 = 0;                 // T = (I + L_A)^-1, fp16 tile
    static constexpr size_t kLK16 = 1 * 32768;        // strict(L_K), fp16 tile
    static constexpr size_t kMQK16 = 2 * 32768;       // incl(M_QK), fp16 tile
    static constexpr size_t kMQA16 = 3 * 32768;       // incl(M_QA), fp16 tile
    static constexpr size_t kU16 = 4 * 32768;         // U = w * v, fp16 tile
    static constexpr size_t kW16 = 5 * 32768;         // W = T K~, fp16 tile
    static constexpr size_t kAbar16 = 6 * 32768;      // Abar, fp16 tile
    static constexpr size_t kKbar16 = 7 * 32768;      // Kbar, fp16 tile
    static constexpr size_t kUp = 8 * 32768;          // U' = T L_K U, fp32 (grp4 layout)
    static constexpr size_t kBytes = 8 * 32768 + 65536;
};
// The aux buffer: nch records, then Q' [nch][128][128] fp32 (grp4 layout), then M^T
// [nch][128][128] fp32 (the reverse state pass reads M_n^T), then the final
// states S_N [B*H][128][128] fp32.
inline size_t aux_bytes(size_t nch, size_t bh) {
    return nch * (AuxLayout::kBytes + 2 * 65536 + 1024) + bh * 65536;
}
// Inverse row norms of the fused q/k prologue: [nch][2][128] floats after S_N.
inline float* aux_rn(unsigned char* aux, size_t nch, size_t bh) {
    return reinterpret_cast<float*>(aux + nch * (AuxLayout::kBytes + 2 * 65536) + bh * 65536);
}
inline float* aux_SN(unsigned char* aux, size_t nch) {
    return reinterpret_cast<float*>(aux + nch * (AuxLayout::kBytes + 2 * 65536));
}
inline float* aux_Qp(unsigned char* aux, size_t nch) {
    return reinterpret_cast<float*>(aux + nch * AuxLayout::kBytes);
}
inline float* aux_Mt(unsigned char* aux, size_t nch) {
    return reinterpret_cast<float*>(aux + nch * (AuxLayout::kBytes + 65536));
}

struct IntraParams {
    CUtensorMap tq, tk, tv, tg, te, tw, tgam;  // token-major [B*T][H][128] bf16
    CUtensorMap tM;                            // M_n as rows of 128 fp32 (stored as tiles)
    const void *q, *gamma;                     // the same tensors (plain loads)
    int B, T, H;
    float* M;      // chunk transitions M_n [j][i]: S_{n+1} = M_n S_n + B_n
    float* Mt;     // M_n transposed (optional)
    float* Bn;     // B_n [j][c] (grp4 layout)
    float* Qp;     // Q'_n [t][i] (grp4 layout): O_n = Q'_n S_n + O_intra_n
    float* Oi;     // O_intra_n [t][c] (grp4 layout)
    unsigned char* aux;  // per-chunk AuxLayout records, or null (nothing saved)
    int* flags;          // flags[0] |= 1 when a chunk's decay span exceeds the single pivot
    // fused q/k prologue: q and k hold raw x; every read applies
    // SiLU(x) / ||SiLU(x)|| per token-head row, and the row's inverse norms
    // go to rnorm[c][0][t] (q) and rnorm[c][1][t] (k) for the backward
    int qk_raw;
    float* rnorm;
};

struct ChainParams {
    CUtensorMap tM;      // transitions, rows of 128 fp32
    const float* Bn;
    const float* S0;     // [B*H][128][128] or null
    float* S_chunks;     // [B*H][N][128][128] or null
    float* S_final;      // [B*H][128][128] or null
    float* S_last;       // second copy of S_N (saved for the backward) or null
    int N;
};

struct OutParams {
    CUtensorMap to;      // o as token-major bf16 tiles (bf16 output only)
    CUtensorMap tS;      // S_n rows of 128 fp32
    int B, T, H;
    const float* Qp;     // Q' (grp4 layout)
    const float* S_chunks;
    const float* Oi;
    void* o;             // token-major [B][T][H][128], fp32 or bf16
    const void* zo;      // output-gate pre-activation [B][T][H][128] bf16, or null
    void* o_pre;         // pre-gate output (as o), or null
};

struct Fwd2Args {
    int B, T, H;
    bool out_bf16;
    const void *q, *k, *v, *g, *e, *w, *gamma;
    const float* S0;
    void* o;             // may be null (state pass only)
    const void* zo;      // output-gate pre-activation, or null (no gate)
    void* o_pre;         // receives the pre-gate output when zo is set, or null
    float* S_final;      // may be null
    float* S_chunks;     // required
    float *M, *Mt, *Bn, *Qp, *Oi;
    float* S_last;       // copy of S_N for the backward, or null
    unsigned char* aux;  // null, or nch AuxLayout records
    int* flags;
    int qk_raw;          // q and k are raw: the prologue is fused (needs rnorm)
    float* rnorm;        // with qk_raw: [nch][2][128] inverse row norms (q, k)
};

bool fwd2_supported(int B, int T, int H, int D, int C, bool in_bf16);
// Column-slab width of the two state passes for B*H heads (16 or 32).
int chain_slab(int BH);
size_t fwd2_ws_bytes(int B, int T, int H);
cudaError_t run_fwd2(const Fwd2Args& a, cudaStream_t st);
unsigned int timeouts_v2();

}  // namespace v2
}  // namespace muir

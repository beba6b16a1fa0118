// chunk.cu -- chunkwise-parallel forward and backward of the Muir gated delta
// rule ("Muir: Linear Attention with Sensitivity-Allocated Gating and
// Matched-Filter Readout", arXiv 2611.08376; wolonglab.org page, section
// "Methodology" and fig:kernel).
//
// Per chunk of C tokens with chunk-start state S (d = dk = dv, rows of S are
// key channels), with Gam_t = sum_{i<=t} g_i inside the chunk, gbar = Gam_{C-1}:
//
//   [X (*) Z]_{ts} = sum_j X_tj Z_sj exp(Gam_tj - Gam_sj)          (s <= t)
//   L_A = strict(K (*) A), L_K = strict(K (*) K),  A = e*K, U = w*V, Qh = gamma*Q
//   M_QK = incl(Qh (*) K), M_QA = incl(Qh (*) A),  T = (I + L_A)^{-1}
//   Y  = T (Kt S + L_K U),            Kt = K e^Gam      (y_t = k_t^T D_t S_{t-1})
//   O  = Qt S + M_QK U - M_QA Y,      Qt = Qh e^Gam
//   S' = diag(e^gbar) S + Kb^T U - Ab^T Y,   Kb = K e^{gbar-Gam}, Ab = A e^{gbar-Gam}
//
// Eliminating Y gives the chunk transition S' = M S + Bn with
//   Psi = T^T Ab,  M = diag(e^gbar) - Psi^T Kt,  Bn = (Kb - L_K^T Psi)^T U,
// so the sequential pass over chunks is one d x d x d product per chunk.
//
// Boundary pivots (fig:kernel "boundary-pivoted"): every exponential applied to
// an operand is <= 1, except inside a diagonal 8-token block, where the pivot is
// the block's 4th token and factors stay below exp(4 * 20) thanks to the clamp
// g >= -20.  With 8-token blocks rb and J (rb > J), e(J) = last token of J and
// b(rb) = token before rb:
//   exp(Gam_t - Gam_s) = [exp(Gam_t - Gam_b(rb))] [exp(Gam_b(rb) - Gam_e(J))] [exp(Gam_e(J) - Gam_s)]
//                      =        x8f_t          *        F[rb][J]            *      z8f_s
// and inside one block with mid pivot m: exp(Gam_t - Gam_m) * exp(Gam_m - Gam_s) = xof_t * zof_s.
//
// Kernels (one CTA of 256 threads per chunk, persistent over chunks, with a
// private float32 scratch slot in the workspace that stays resident in L2):
//   k_intra : M, Bn per chunk                         (parallel over chunks)
//   k_chain : S_{n+1} = M_n S_n + Bn_n, or its transpose for the gradient
//             (sequential over chunks, parallel over (b, h, column slabs))
//   k_out   : O per chunk from the chunk-start state  (parallel)
//   k_bprep : B'_n = Qt^T dO - Kt^T T^T M_QA^T dO      (parallel)
//   k_bwd   : all input gradients per chunk            (parallel)
// Products run on tensor cores (TF32 mma.sync, float32 accumulate; three
// split-TF32 passes for float32 inputs).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"
#include "tc.cuh"
#include "profile.h"

namespace muir {

constexpr int kThreads = 256;

// Expired bounded waits (tc::wait_mma) of the chunk kernels in this
// translation unit, read and cleared by take_wait_timeouts().
static __device__ unsigned int g_wait_timeouts;

inline unsigned int take_wait_timeouts() {
    unsigned int n = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&n, g_wait_timeouts, sizeof(n)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_wait_timeouts, &zero, sizeof(zero));
    return n;
}
constexpr int kMaxSlots = 296;  // scratch slots: at most 2 resident CTAs per SM on a 148-SM B200

// ------------------------------------------------------------------ scratch

struct Lay {
    int C, D, nb8, nb16;
    size_t LC, RC, BT, PRE, SUF, GBAR, LA, LK, MQK, MQA, TII, W[8], PXK, PXQ, PZA, PZK;
    size_t OXK, OXQ, OZA, OZK, MXK, MXQ, MZA, MZK, GK[4], GM[4];
    size_t RKT, RQT, RUU, RDO, RAB, RKB, total;  // input-derived operand rows (TF32)
};

__host__ __device__ inline Lay make_lay(int C, int D) {
    Lay L;
    L.C = C; L.D = D; L.nb8 = C / 8; L.nb16 = C / 16;
    const size_t cd = (size_t)C * D, cc = (size_t)C * C, bd = (size_t)(C / 8) * D;
    size_t o = 0;
#define MUIR_TAKE(field, n) L.field = o; o += ((size_t)(n) + 63) & ~(size_t)63;
    MUIR_TAKE(LC, cd) MUIR_TAKE(RC, cd) MUIR_TAKE(BT, bd) MUIR_TAKE(PRE, bd) MUIR_TAKE(SUF, bd)
    MUIR_TAKE(GBAR, D)
    MUIR_TAKE(LA, cc) MUIR_TAKE(LK, cc) MUIR_TAKE(MQK, cc) MUIR_TAKE(MQA, cc)
    MUIR_TAKE(TII, (size_t)C * 16)
    for (int i = 0; i < 8; ++i) { MUIR_TAKE(W[i], cd) }
    MUIR_TAKE(PXK, cd) MUIR_TAKE(PXQ, cd) MUIR_TAKE(PZA, cd) MUIR_TAKE(PZK, cd)
    const size_t pd = (size_t)128 * D, pc = (size_t)C * 128;  // tiles padded to 128 rows
    MUIR_TAKE(OXK, pd) MUIR_TAKE(OXQ, pd) MUIR_TAKE(OZA, cd) MUIR_TAKE(OZK, cd)
    MUIR_TAKE(MXK, pc) MUIR_TAKE(MXQ, pc) MUIR_TAKE(MZA, pc) MUIR_TAKE(MZK, pc)
    for (int i = 0; i < 4; ++i) { MUIR_TAKE(GK[i], cc) MUIR_TAKE(GM[i], cc) }
    MUIR_TAKE(RKT, cd) MUIR_TAKE(RQT, cd) MUIR_TAKE(RUU, cd) MUIR_TAKE(RDO, cd) MUIR_TAKE(RAB, cd)
    MUIR_TAKE(RKB, cd)
#undef MUIR_TAKE
    L.total = o;
    return L;
}

// ------------------------------------------------------------------ params

struct KParams {
    int B, T, H, C, N;
    const void *q, *k, *v, *g, *e, *w, *gamma, *dO;
    const float* S_chunks;   // chunk-start states   [B,H,N,D,D]
    const float* dS_chunks;  // gradient at chunk end [B,H,N,D,D]
    float* M;                // transition           [B,H,N,D,D]
    float* Bn;               // affine term          [B,H,N,D,D]
    void* o;
    void *dq, *dk, *dv, *dg, *de, *dw, *dgamma;
    float* scratch;
    size_t slot;             // floats per scratch slot
    float* aux;              // per-chunk saved intermediates or null
    // chunk n of sequence bh sits at index bh * nstride + noff + n of the
    // per-chunk arrays (S_chunks, dS_chunks, M, Bn, aux); a launch may cover
    // only some chunks of each sequence (the padded last chunk of a ragged
    // sequence runs as its own launch over side buffers)
    int nstride, noff;
    // device word that must be non-zero for the launch to do any work (the
    // single-pivot span flag when the on-chip path ran first), or null
    const int* gate;
};

// Accessors of one chunk's inputs; row t of a [B,T,H,D] tensor.
template <typename Tin, int D>
struct Chunk {
    const Tin *q, *k, *v, *g, *e, *w, *gm, *dO;
    size_t rs, base, sbase;  // row stride (H*D), element offset of row 0, state offset
    float* s;                // scratch slot
    Lay L;
    bool tame;               // decay span small enough for the single-pivot products
    size_t sidx;             // index of the chunk in the per-chunk arrays
    __device__ float K(int t, int j) const { return ldf(k + base + t * rs + j); }
    __device__ float Qh(int t, int j) const {
        return ldf(gm + base + t * rs + j) * ldf(q + base + t * rs + j);
    }
    __device__ float A(int t, int j) const {
        return ldf(e + base + t * rs + j) * ldf(k + base + t * rs + j);
    }
    __device__ float U(int t, int c) const {
        return ldf(w + base + t * rs + c) * ldf(v + base + t * rs + c);
    }
    __device__ float dOv(int t, int c) const { return ldf(dO + base + t * rs + c); }
    __device__ float& at(size_t off, int r, int c) const { return s[off + (size_t)r * D + c]; }
};

// CF: the chunk size when it is fixed at compile time (0 = take it from p.C).
template <typename Tin, int D, int CF>
__device__ Chunk<Tin, D> make_chunk(const KParams& p, int chunk, float* slot) {
    Chunk<Tin, D> c;
    const int n = chunk % p.N, bh = chunk / p.N, h = bh % p.H, b = bh / p.H;
    c.q = (const Tin*)p.q; c.k = (const Tin*)p.k; c.v = (const Tin*)p.v; c.g = (const Tin*)p.g;
    c.e = (const Tin*)p.e; c.w = (const Tin*)p.w; c.gm = (const Tin*)p.gamma;
    c.dO = (const Tin*)p.dO;
    c.rs = (size_t)p.H * D;
    c.base = (((size_t)b * p.T + (size_t)n * p.C) * p.H + h) * D;
    c.sidx = (size_t)bh * p.nstride + p.noff + n;
    c.sbase = c.sidx * D * D;
    c.s = slot;
    c.L = make_lay(CF ? CF : p.C, D);
    c.tame = false;
    return c;
}

// ------------------------------------------------------------------ saved intermediates

// Per-chunk layout of the intermediates the forward saves for the backward:
// L_A, L_K, M_QK, M_QA (C x C), the inverted 16 x 16 diagonal blocks (C x 16), Y (C x D).
struct AuxLay {
    size_t LA, LK, MQK, MQA, TII, Y, total;
};

__host__ __device__ inline AuxLay make_aux_lay(int C, int D) {
    AuxLay A;
    size_t o = 0;
    auto take = [&](size_t n) { const size_t r = o; o += (n + 63) & ~(size_t)63; return r; };
    const size_t cc = (size_t)C * C;
    A.LA = take(cc); A.LK = take(cc); A.MQK = take(cc); A.MQA = take(cc);
    A.TII = take((size_t)C * 16); A.Y = take((size_t)C * D);
    A.total = o;
    return A;
}

// Copy n floats (multiple of 4, 16-byte aligned) between global arrays, every
// thread's loads of a batch issued before its stores.
__device__ __forceinline__ void copy_floats(float* dst, const float* src, size_t n) {
    constexpr int BATCH = 8;
    const size_t n4 = n / 4;
    for (size_t base = threadIdx.x; base < n4; base += (size_t)BATCH * kThreads) {
        float4 v[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            const size_t idx = base + (size_t)i * kThreads;
            if (idx < n4) v[i] = reinterpret_cast<const float4*>(src)[idx];
        }
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            const size_t idx = base + (size_t)i * kThreads;
            if (idx < n4) reinterpret_cast<float4*>(dst)[idx] = v[i];
        }
    }
}

// Save (to_aux) or restore this chunk's intermediates between the scratch slot
// and the chunk's aux record; y_off is Y's place in the scratch slot; mask
// selects parts: 1 L_A, 2 L_K, 4 M_QK, 8 M_QA, 16 block inverses, 32 Y.
template <typename Tin, int D>
__device__ void aux_copy(const Chunk<Tin, D>& c, float* rec, bool to_aux, int mask, size_t y_off) {
    const Lay& L = c.L;
    const AuxLay A = make_aux_lay(L.C, D);
    const size_t cc = (size_t)L.C * L.C;
    const size_t so[6] = {L.LA, L.LK, L.MQK, L.MQA, L.TII, y_off};
    const size_t ao[6] = {A.LA, A.LK, A.MQK, A.MQA, A.TII, A.Y};
    const size_t n[6] = {cc, cc, cc, cc, (size_t)L.C * 16, (size_t)L.C * D};
    for (int i = 0; i < 6; ++i) {
        if (!(mask & (1 << i))) continue;
        if (to_aux) copy_floats(rec + ao[i], c.s + so[i], n[i]);
        else copy_floats(c.s + so[i], rec + ao[i], n[i]);
    }
    __syncthreads();
}

// ------------------------------------------------------------------ masked products

// Operand kinds for the masked products.
enum Opnd { OP_K = 0, OP_Q = 1, OP_A = 2 };

template <typename Tin, int D>
__device__ __forceinline__ float opval(const Chunk<Tin, D>& c, int kind, int t, int j) {
    return kind == OP_K ? c.K(t, j) : (kind == OP_Q ? c.Qh(t, j) : c.A(t, j));
}

#include "staged.cuh"

// ------------------------------------------------------------------ triangular solves

// T_II = (I + L_II)^{-1} for every 16 x 16 diagonal block of the unit lower
// triangular I + L (forward substitution, float32).
__device__ inline void compute_tii(float* s, const Lay& L, size_t Loff) {
    const int C = L.C, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int blk = warp; blk < L.nb16; blk += kThreads / 32) {
        const int b0 = 16 * blk;
        if (lane < 16) {
            const int col = lane;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = (r == col) ? 1.f : 0.f;
#pragma unroll
                for (int q = 0; q < r; ++q) acc -= s[Loff + (size_t)(b0 + r) * C + b0 + q] * x[q];
                x[r] = (r < col) ? 0.f : acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) s[L.TII + ((size_t)blk * 16 + r) * 16 + col] = x[r];
        }
    }
}

// ------------------------------------------------------------------ tensor-core helpers

// Four consecutive float32 scratch elements (16-byte aligned).
__device__ __forceinline__ void ld4(const float* p, float* v) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}
// Four consecutive input elements (8- or 16-byte aligned).
__device__ __forceinline__ void ld4in(const float* p, float* v) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}
__device__ __forceinline__ void ld4in(const __nv_bfloat16* p, float* v) {
    const uint2 x = __ldg(reinterpret_cast<const uint2*>(p));
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&x.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&x.y);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    v[0] = fa.x; v[1] = fa.y; v[2] = fb.x; v[3] = fb.y;
}

// Eight consecutive outputs (16-byte aligned for bf16, 32-byte for float32).
__device__ __forceinline__ void st8(float* p, const float* x) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    *reinterpret_cast<float4*>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
}
__device__ __forceinline__ void st8(__nv_bfloat16* p, const float* x) {
    uint4 u;
    __nv_bfloat162 h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    u.x = *reinterpret_cast<uint32_t*>(&h[0]); u.y = *reinterpret_cast<uint32_t*>(&h[1]);
    u.z = *reinterpret_cast<uint32_t*>(&h[2]); u.w = *reinterpret_cast<uint32_t*>(&h[3]);
    *reinterpret_cast<uint4*>(p) = u;
}

// Tensor-core state shared by one CTA's products (TMEM columns, mbarrier).
struct TcCta {
    tc::State st;
    unsigned char* sbuf;  // 1 KB aligned start of the dynamic shared memory
    int sbytes;           // bytes from sbuf to the end of the dynamic shared memory
};

// TMEM columns a chunk CTA allocates: single-pass k_bwd 512 (one CTA per SM);
// the other single-pass kernels 256 (two CTAs per SM); three-pass 128.
__host__ __device__ constexpr int tmem_cols(int passes, bool bwd = false) {
    return passes == 1 ? (bwd ? 512 : 256) : 128;
}
// CTAs per SM the single-pass forward-side kernels are compiled for.
__host__ __device__ constexpr int fwd_ctas(int passes) { return passes == 1 ? 2 : 1; }

// Product over M rows (looped in 128-row tiles) and N = NT columns.
template <int PASSES, int N, bool AR, bool BR, class FA4, class FB4, class EPI>
__device__ __forceinline__ void tc_rows(TcCta& t, int M, int K, const FA4& fa4, const FB4& fb4,
                                        const EPI& epi) {
    for (int m0 = 0; m0 < M; m0 += 128) {
        const int Mt = M - m0 < 128 ? M - m0 : 128;
        auto fa = [&](int m, int k, float* v) { fa4(m0 + m, k, v); };
        if constexpr (tc::is_row8<EPI>::value) {
            auto e8 = [&](int m, int n0, const float* v) { epi.f(m0 + m, n0, v); };
            tc::gemm<PASSES, N, AR, BR>(t.st, t.sbuf, Mt, K, fa, fb4, tc::Row8<decltype(e8)>{e8});
        } else {
            tc::gemm<PASSES, N, AR, BR>(t.st, t.sbuf, Mt, K, fa, fb4,
                                        [&](int m, int n, float x) { epi(m0 + m, n, x); });
        }
    }
}

// Same, storing raw rows (vectorised) into a row-major destination.
template <int PASSES, int N, bool AR, bool BR, class FA4, class FB4>
__device__ __forceinline__ void tc_rows(TcCta& t, int M, int K, const FA4& fa4, const FB4& fb4,
                                        tc::RowStore dst) {
    for (int m0 = 0; m0 < M; m0 += 128) {
        const int Mt = M - m0 < 128 ? M - m0 : 128;
        tc::RowStore d = {dst.dst + (size_t)m0 * dst.ld, dst.ld};
        tc::gemm<PASSES, N, AR, BR>(
            t.st, t.sbuf, Mt, K, [&](int m, int k, float* v) { fa4(m0 + m, k, v); }, fb4, d);
    }
}

// Product with asynchronous staging of the K segments asrc / bsrc describe
// (single-pass TF32); three-pass inputs take the element-producer engine.
template <int PASSES, int N, bool AR, bool BR, class ASRC, class FA4, class BSRC, class FB4,
          class EPI>
__device__ __forceinline__ void tc_rows2(TcCta& t, int M, int K, const ASRC& asrc, const FA4& fa4,
                                         const BSRC& bsrc, const FB4& fb4, const EPI& epi,
                                         int NB = N) {
    if constexpr (PASSES != 1) {
        tc_rows<PASSES, N, AR, BR>(t, M, K, fa4, fb4, epi);
    } else {
        for (int m0 = 0; m0 < M; m0 += 128) {
            const int Mt = M - m0 < 128 ? M - m0 : 128;
            auto fa = [&](int m, int k, float* v) { fa4(m0 + m, k, v); };
            auto as = [&](int k) {
                tc::Src a = asrc(k);
                if (a.p) a.p += a.mn ? (size_t)m0 : (size_t)m0 * a.ld;
                return a;
            };
            if constexpr (std::is_same<EPI, tc::RowStore>::value) {
                tc::RowStore d = {epi.dst + (size_t)m0 * epi.ld, epi.ld};
                tc::gemm_async<N>(t.st, t.sbuf, t.sbytes, Mt, NB, K, as, fa, bsrc, fb4, d);
            } else if constexpr (tc::is_row8<EPI>::value) {
                auto e8 = [&](int m, int n0, const float* v) { epi.f(m0 + m, n0, v); };
                tc::gemm_async<N>(t.st, t.sbuf, t.sbytes, Mt, NB, K, as, fa, bsrc, fb4, tc::Row8<decltype(e8)>{e8});
            } else {
                tc::gemm_async<N>(t.st, t.sbuf, t.sbytes, Mt, NB, K, as, fa, bsrc, fb4,
                                  [&](int m, int n, float x) { epi(m0 + m, n, x); });
            }
        }
    }
}

#include "panel.cuh"
#include "fast.cuh"

// Decay-masked pair: tensor-core panels for single-pass chunks of at most 128
// tokens, 8-block mma.sync tiles otherwise.
template <typename Tin, int D, int PASSES>
__device__ __forceinline__ bool use_panels(const Chunk<Tin, D>& c) {
    return PASSES == 1 && c.L.C <= 128;
}

// Per-chunk operands of the decay-masked products; decides between the
// single-pivot products (small decay span) and the 8-token panels.
template <typename Tin, int D, int PASSES>
__device__ __forceinline__ void masked_prep(Chunk<Tin, D>& c, bool with_q, bool bwd,
                                            bool pairs = true) {
    c.tame = false;
    if (!use_panels<Tin, D, PASSES>(c)) return;
    if (c.L.C >= 32) c.tame = chunk_tame(c);
    if (c.tame) fast_prep<Tin, D>(c, with_q, bwd, pairs);
    else panel_prep<Tin, D>(c, with_q);
}

// Input-derived operands of the dense products, once per chunk, as TF32-rounded
// float32 rows [C][d] in scratch, so that the products copy them (cp.async)
// instead of producing them element by element inside their K loops:
//   R_KT  Kt = K e^Gam        R_QT  Qt = gamma q e^Gam     R_UU  U = w v
//   R_DO  dO                  R_AB  Ab = e k e^{gbar-Gam}  R_KB  Kb = K e^{gbar-Gam}
enum RowOps { R_KT = 1, R_QT = 2, R_UU = 4, R_DO = 8, R_AB = 16, R_KB = 32 };

// U2: items per thread whose loads are issued together (2 where registers allow).
template <typename Tin, int D, int PASSES, int U2 = 1>
__device__ void rows_prep(const Chunk<Tin, D>& c, int ops) {
    if constexpr (PASSES != 1) return;
    const Lay& L = c.L;
    const int n4 = L.C * D / 4;
    for (int base = threadIdx.x; base < n4; base += U2 * kThreads) {
        float k4[U2][4], e4[U2][4], q4[U2][4], m4[U2][4], v4[U2][4], w4[U2][4], o4[U2][4];
        float lc[U2][4], pre[U2][4], rc[U2][4], suf[U2][4];
#pragma unroll
        for (int i = 0; i < U2; ++i) {
            const int idx = base + i * kThreads;
            if (idx >= n4) break;
            const int t = idx / (D / 4), j = 4 * (idx % (D / 4));
            const size_t g = c.base + (size_t)t * c.rs + j, x = (size_t)t * D + j;
            const size_t b = (size_t)(t >> 3) * D + j;
            if (ops & (R_KT | R_KB | R_AB)) ld4in(c.k + g, k4[i]);
            if (ops & R_AB) ld4in(c.e + g, e4[i]);
            if (ops & R_QT) { ld4in(c.q + g, q4[i]); ld4in(c.gm + g, m4[i]); }
            if (ops & R_UU) { ld4in(c.v + g, v4[i]); ld4in(c.w + g, w4[i]); }
            if (ops & R_DO) ld4in(c.dO + g, o4[i]);
            if (ops & (R_KT | R_QT)) { ld4(c.s + L.LC + x, lc[i]); ld4(c.s + L.PRE + b, pre[i]); }
            if (ops & (R_KB | R_AB)) { ld4(c.s + L.RC + x, rc[i]); ld4(c.s + L.SUF + b, suf[i]); }
        }
#pragma unroll
        for (int i = 0; i < U2; ++i) {
            const int idx = base + i * kThreads;
            if (idx >= n4) break;
            const int t = idx / (D / 4), j = 4 * (idx % (D / 4));
            const size_t x = (size_t)t * D + j;
            float4 kt, qt, uu, dd, ab, kb;
            float* pkt = &kt.x; float* pqt = &qt.x; float* puu = &uu.x; float* pdd = &dd.x;
            float* pab = &ab.x; float* pkb = &kb.x;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float eg = (ops & (R_KT | R_QT)) ? fexp<Tin>(pre[i][u] + lc[i][u]) : 0.f;
                const float egb = (ops & (R_KB | R_AB)) ? fexp<Tin>(rc[i][u] + suf[i][u]) : 0.f;
                const float kk = (ops & (R_KT | R_KB | R_AB)) ? k4[i][u] : 0.f;
                pkt[u] = tc::tf32_rn(kk * eg);
                pqt[u] = (ops & R_QT) ? tc::tf32_rn(q4[i][u] * m4[i][u] * eg) : 0.f;
                puu[u] = (ops & R_UU) ? tc::tf32_rn(v4[i][u] * w4[i][u]) : 0.f;
                pdd[u] = (ops & R_DO) ? tc::tf32_rn(o4[i][u]) : 0.f;
                pab[u] = (ops & R_AB) ? tc::tf32_rn(e4[i][u] * kk * egb) : 0.f;
                pkb[u] = tc::tf32_rn(kk * egb);
            }
            if (ops & R_KT) *reinterpret_cast<float4*>(c.s + L.RKT + x) = kt;
            if (ops & R_QT) *reinterpret_cast<float4*>(c.s + L.RQT + x) = qt;
            if (ops & R_UU) *reinterpret_cast<float4*>(c.s + L.RUU + x) = uu;
            if (ops & R_DO) *reinterpret_cast<float4*>(c.s + L.RDO + x) = dd;
            if (ops & R_AB) *reinterpret_cast<float4*>(c.s + L.RAB + x) = ab;
            if (ops & R_KB) *reinterpret_cast<float4*>(c.s + L.RKB + x) = kb;
        }
    }
    __syncthreads();
}

template <typename Tin, int D, int PASSES, int X, int Z0, int Z1>
__device__ __forceinline__ void masked_pair(const Chunk<Tin, D>& c, TcCta& tcx, float* sm,
                                            size_t out0, size_t out1, bool incl0, bool incl1) {
    if (c.tame)
        fast_masked_pair<Tin, D, X, Z0, Z1>(c, tcx, out0, out1, incl0, incl1);
    else if (use_panels<Tin, D, PASSES>(c))
        panel_masked_pair<Tin, D, X, Z0, Z1>(c, tcx, out0, out1, incl0, incl1);
    else
        masked_pair_s<Tin, D, PASSES, X, Z0, Z1>(c, sm, out0, out1, incl0, incl1);
}

// epi(integral_constant<int, N>, t0, j, v) consumes the results of N
// consecutive tokens t0.. at channel j.
template <typename Tin, int D, int PASSES, bool XSIDE, int op0, int op1, class EPI>
__device__ __forceinline__ void decayed_grad(const Chunk<Tin, D>& c, TcCta& tcx, float* sm,
                                             size_t G0, size_t G1, const EPI& epi) {
    if (use_panels<Tin, D, PASSES>(c)) {
        if constexpr (XSIDE) panel_grad_x<Tin, D, op0, op1>(c, tcx, G0, G1, epi);
        else panel_grad_z<Tin, D, op0, op1>(c, tcx, G0, G1, epi);
    } else {
        decayed_grad_any<Tin, D, PASSES, XSIDE, op0, op1>(c, sm, G0, G1, [&](int t, int j, float v) {
            epi(std::integral_constant<int, 1>{}, t, j, &v);
        });
    }
}

// ------------------------------------------------------------------ k_intra

template <typename Tin, int D, int PASSES, int CF>
__global__ void __launch_bounds__(kThreads, fwd_ctas(PASSES)) k_intra(KParams p) {
    if (p.gate && *p.gate == 0) return;
    __shared__ uint32_t tmem_slot;
    __shared__ __align__(8) uint64_t mbar;
    __shared__ int tc_status;
    extern __shared__ __align__(128) unsigned char dsm[];
    TcCta tcx;
    tcx.sbuf = dsm + ((1024u - (tc::smem_addr(dsm) & 1023u)) & 1023u);  // 1 KB aligned
    tcx.sbytes = (int)tc::dynamic_smem_bytes() - (int)(tcx.sbuf - dsm);
    tc::init(tcx.st, &tmem_slot, &mbar, &tc_status, tmem_cols(PASSES));
    float* sm = reinterpret_cast<float*>(dsm);
    float* slot = p.scratch + (size_t)blockIdx.x * p.slot;
    const int nch = p.B * p.H * p.N;
    for (int chunk = blockIdx.x; chunk < nch; chunk += gridDim.x) {
        Chunk<Tin, D> c = make_chunk<Tin, D, CF>(p, chunk, slot);
        const Lay& L = c.L;
        const int C = L.C;
        float* s = c.s;
        prologue2(c);
        masked_prep<Tin, D, PASSES>(c, false, false);
        rows_prep<Tin, D, PASSES>(c, R_KT | R_UU | R_AB | R_KB);
        masked_pair<Tin, D, PASSES, OP_K, OP_A, OP_K>(c, tcx, sm, L.LA, L.LK, false, false);
        __syncthreads();
        compute_tii(s, L, L.LA);
        // Ab (single-pass: the prepared rows; three-pass: formed here in full float32)
        const size_t ab = PASSES == 1 ? L.RAB : L.W[0];
        if (PASSES != 1)
            for (int idx = threadIdx.x; idx < C * D; idx += kThreads)
                s[ab + idx] = c.A(idx / D, idx % D) * facs(c).egb(idx / D, idx % D);
        __syncthreads();
        solve_s<D, PASSES, true>(s, sm, L, L.LA, ab);  // Psi = T^T Ab (in place)
        __syncthreads();
        float* M = p.M + c.sbase;
        const float* Psi = s + ab;
        const Fac<Tin, D> f = facs(c);
        // M = diag(e^gbar) - Psi^T Kt      (rows i, contraction over tokens)
        tc_rows2<PASSES, D, true, true>(tcx, D, C,
            [&](int) { return tc::Src{Psi, D, 0, true, false}; },
            [&](int i, int t, float* v) { for (int u = 0; u < 4; ++u) v[u] = Psi[(size_t)(t + u) * D + i]; },
            [&](int) { return tc::Src{s + L.RKT, D, 0, true, false}; },
            [&](int j, int t, float* v) {
                for (int u = 0; u < 4; ++u) v[u] = c.K(t + u, j) * f.eg(t + u, j);
            },
            [&](int i, int j, float x) {
                const float d = (i == j) ? expf(f.gbar(i)) : 0.f;
                M[(size_t)i * D + j] = d - x;
            });
        // Phi = Kb - L_K^T Psi              (rows t, contraction over tokens s)
        float* Phi = s + L.W[1];
        tc_rows2<PASSES, D, true, true>(tcx, C, C,
            [&](int) { return tc::Src{s + L.LK, C, 0, true, false}; },
            [&](int t, int k, float* v) { for (int u = 0; u < 4; ++u) v[u] = s[L.LK + (size_t)(k + u) * C + t]; },
            [&](int) { return tc::Src{Psi, D, 0, true, false}; },
            [&](int j, int k, float* v) { for (int u = 0; u < 4; ++u) v[u] = Psi[(size_t)(k + u) * D + j]; },
            [&](int t, int j, float x) {
                const float kb = PASSES == 1 ? s[L.RKB + (size_t)t * D + j] : c.K(t, j) * f.egb(t, j);
                Phi[(size_t)t * D + j] = kb - x;
            });
        // Bn = Phi^T U
        float* Bn = p.Bn + c.sbase;
        tc_rows2<PASSES, D, true, true>(tcx, D, C,
            [&](int) { return tc::Src{Phi, D, 0, true, false}; },
            [&](int i, int t, float* v) { for (int u = 0; u < 4; ++u) v[u] = Phi[(size_t)(t + u) * D + i]; },
            [&](int) { return tc::Src{s + L.RUU, D, 0, true, false}; },
            [&](int cc, int t, float* v) { for (int u = 0; u < 4; ++u) v[u] = c.U(t + u, cc); },
            tc::RowStore{Bn, D});
    }
    if (threadIdx.x == 0 && tc_status != 0) atomicAdd(&g_wait_timeouts, 1u);
    tc::release(tcx.st, tmem_cols(PASSES));
}

// ------------------------------------------------------------------ k_chain

// Sequential pass over chunks for one (b, h) and a slab of SLAB columns.
// Forward (REV = false): S_{n+1} = M_n S_n + Bn_n, records S_n.
// Reverse (REV = true):  G_n = M_n^T G_{n+1} + Bn_n, records G_{n+1}.
// M_{n+1} and the slab of Bn_{n+1} are copied into shared memory (cp.async,
// rows padded to D + 4 floats) while step n computes from M_n.
template <int D, int SLAB>
__host__ __device__ constexpr int chain_smem_bytes() {
    return (2 * D * (D + 4) + 2 * D * SLAB) * 4;
}

template <int D, int SLAB, int PASSES, bool REV>
__global__ void __launch_bounds__(kThreads) k_chain(const float* __restrict__ M,
                                                    const float* __restrict__ Bn,
                                                    const float* __restrict__ S_in,
                                                    float* __restrict__ S_rec,
                                                    float* __restrict__ S_out, int N,
                                                    const int* __restrict__ gate) {
    if (gate && *gate == 0) return;
    constexpr int NT = SLAB / 8 < 4 ? SLAB / 8 : 4;
    constexpr int MP = D + 4;  // padded row of M in shared memory
    __shared__ float buf[2][D * SLAB];
    extern __shared__ __align__(16) float csm[];
    float* mbuf = csm;                    // [2][D][MP]
    float* bbuf = csm + 2 * D * MP;       // [2][D][SLAB]
    constexpr int NSLAB = D / SLAB;
    const int bh = blockIdx.x / NSLAB, c0 = (blockIdx.x % NSLAB) * SLAB;
    const size_t DD = (size_t)D * D;
    auto prefetch = [&](int step, int slot) {
        const int n = REV ? N - 1 - step : step;
        const size_t off = ((size_t)bh * N + n) * DD;
        float* md = mbuf + slot * D * MP;
        for (int idx = threadIdx.x; idx < D * D / 4; idx += kThreads) {
            const int r = idx / (D / 4), j = 4 * (idx % (D / 4));
            tc::cp_async16(tc::smem_addr(md + r * MP + j), M + off + (size_t)r * D + j, true);
        }
        float* bd = bbuf + slot * D * SLAB;
        for (int idx = threadIdx.x; idx < D * SLAB / 4; idx += kThreads) {
            const int r = idx / (SLAB / 4), j = 4 * (idx % (SLAB / 4));
            tc::cp_async16(tc::smem_addr(bd + r * SLAB + j), Bn + off + (size_t)r * D + c0 + j, true);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    prefetch(0, 0);
    for (int idx = threadIdx.x; idx < D * SLAB; idx += kThreads) {
        const int i = idx / SLAB, cc = idx % SLAB;
        buf[0][idx] = S_in ? S_in[bh * DD + (size_t)i * D + c0 + cc] : 0.f;
    }
    int cur = 0;
    for (int step = 0; step < N; ++step) {
        const int n = REV ? N - 1 - step : step;
        const size_t off = ((size_t)bh * N + n) * DD;
        if (step + 1 < N) {
            prefetch(step + 1, (step + 1) & 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        if (S_rec)
            for (int idx = threadIdx.x; idx < D * SLAB; idx += kThreads)
                S_rec[off + (size_t)(idx / SLAB) * D + c0 + idx % SLAB] = buf[cur][idx];
        const float* Mn = mbuf + (step & 1) * D * MP;
        const float* Bb = bbuf + (step & 1) * D * SLAB;
        const float* Sc = buf[cur];
        float* Sn = buf[cur ^ 1];
        cta_tiles<NT>(D, SLAB,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, D,
                    [&](int r, int k) { return REV ? Mn[k * MP + m0 + r] : Mn[(m0 + r) * MP + k]; },
                    [&](int k, int nn) { return Sc[k * SLAB + n0 + nn]; });
            },
            [&](int i, int cc, float v) { Sn[i * SLAB + cc] = v + Bb[i * SLAB + cc]; });
        __syncthreads();
        cur ^= 1;
    }
    if (S_out)
        for (int idx = threadIdx.x; idx < D * SLAB; idx += kThreads)
            S_out[bh * DD + (size_t)(idx / SLAB) * D + c0 + idx % SLAB] = buf[cur][idx];
}

// ------------------------------------------------------------------ k_out

// Y = T (Kt S + L_K U) into scratch at Yoff (needs LA, LK, TII).
template <typename Tin, int D, int PASSES>
__device__ void compute_Y(TcCta& tcx, const Chunk<Tin, D>& c, const float* S, size_t Yoff) {
    const Lay& L = c.L;
    const int C = L.C;
    float* s = c.s;
    const Fac<Tin, D> f = facs(c);
    tc_rows2<PASSES, D, false, true>(tcx, C, D + C,
        [&](int k) {
            return k < D ? tc::Src{s + L.RKT, D, 0, false, false} : tc::Src{s + L.LK, C, D, false, false};
        },
        [&](int t, int k, float* v) {
            if (k < D) {
                ld4in(c.k + c.base + t * c.rs + k, v);
                for (int u = 0; u < 4; ++u) v[u] *= f.eg(t, k + u);
            } else {
                ld4(s + L.LK + (size_t)t * C + (k - D), v);
            }
        },
        [&](int k) { return k < D ? tc::Src{S, D, 0, true, false} : tc::Src{s + L.RUU, D, D, true, false}; },
        [&](int cc, int k, float* v) {
            if (k < D) for (int u = 0; u < 4; ++u) v[u] = __ldg(S + (size_t)(k + u) * D + cc);
            else for (int u = 0; u < 4; ++u) v[u] = c.U(k - D + u, cc);
        },
        tc::RowStore{s + Yoff, D});
    solve_s<D, PASSES, false>(s, reinterpret_cast<float*>(tcx.sbuf), L, L.LA, Yoff);
    __syncthreads();
}

template <typename Tin, typename Tout, int D, int PASSES, int CF>
__global__ void __launch_bounds__(kThreads, fwd_ctas(PASSES)) k_out(KParams p) {
    if (p.gate && *p.gate == 0) return;
    __shared__ uint32_t tmem_slot;
    __shared__ __align__(8) uint64_t mbar;
    __shared__ int tc_status;
    extern __shared__ __align__(128) unsigned char dsm[];
    TcCta tcx;
    tcx.sbuf = dsm + ((1024u - (tc::smem_addr(dsm) & 1023u)) & 1023u);  // 1 KB aligned
    tcx.sbytes = (int)tc::dynamic_smem_bytes() - (int)(tcx.sbuf - dsm);
    tc::init(tcx.st, &tmem_slot, &mbar, &tc_status, tmem_cols(PASSES));
    float* sm = reinterpret_cast<float*>(dsm);
    float* slot = p.scratch + (size_t)blockIdx.x * p.slot;
    const int nch = p.B * p.H * p.N;
    for (int chunk = blockIdx.x; chunk < nch; chunk += gridDim.x) {
        Chunk<Tin, D> c = make_chunk<Tin, D, CF>(p, chunk, slot);
        const Lay& L = c.L;
        const int C = L.C;
        float* s = c.s;
        prologue2(c);
        masked_prep<Tin, D, PASSES>(c, true, false);
        rows_prep<Tin, D, PASSES>(c, R_KT | R_QT | R_UU);
        masked_pair<Tin, D, PASSES, OP_K, OP_A, OP_K>(c, tcx, sm, L.LA, L.LK, false, false);
        masked_pair<Tin, D, PASSES, OP_Q, OP_K, OP_A>(c, tcx, sm, L.MQK, L.MQA, true, true);
        __syncthreads();
        compute_tii(s, L, L.LA);
        __syncthreads();
        const float* S = p.S_chunks + c.sbase;
        compute_Y<Tin, D, PASSES>(tcx, c, S, L.W[0]);
        if (p.aux) aux_copy(c, p.aux + c.sidx * make_aux_lay(C, D).total, true, 63, L.W[0]);
        Tout* o = (Tout*)p.o;
        const Fac<Tin, D> f = facs(c);
        const float* Y = s + L.W[0];
        // eight consecutive outputs of one row per store (16 or 32 bytes)
        auto ostore = [&](int t, int j, const float* x) { st8(o + c.base + (size_t)t * c.rs + j, x); };
        // O = Qt S + M_QK U - M_QA Y
        tc_rows2<PASSES, D, false, true>(tcx, C, D + 2 * C,
            [&](int k) {
                return k < D ? tc::Src{s + L.RQT, D, 0, false, false}
                             : (k < D + C ? tc::Src{s + L.MQK, C, D, false, false}
                                          : tc::Src{s + L.MQA, C, D + C, false, true});
            },
            [&](int t, int k, float* v) {
                if (k < D) {
                    float g4[4];
                    ld4in(c.q + c.base + t * c.rs + k, v);
                    ld4in(c.gm + c.base + t * c.rs + k, g4);
                    for (int u = 0; u < 4; ++u) v[u] *= g4[u] * f.eg(t, k + u);
                } else if (k < D + C) {
                    ld4(s + L.MQK + (size_t)t * C + (k - D), v);
                } else {
                    ld4(s + L.MQA + (size_t)t * C + (k - D - C), v);
                    for (int u = 0; u < 4; ++u) v[u] = -v[u];
                }
            },
            [&](int k) {
                return k < D ? tc::Src{S, D, 0, true, false}
                             : (k < D + C ? tc::Src{s + L.RUU, D, D, true, false}
                                          : tc::Src{Y, D, D + C, true, false});
            },
            [&](int cc, int k, float* v) {
                if (k < D) for (int u = 0; u < 4; ++u) v[u] = __ldg(S + (size_t)(k + u) * D + cc);
                else if (k < D + C) for (int u = 0; u < 4; ++u) v[u] = c.U(k - D + u, cc);
                else for (int u = 0; u < 4; ++u) v[u] = Y[(size_t)(k - D - C + u) * D + cc];
            },
            tc::Row8<decltype(ostore)>{ostore});
    }
    if (threadIdx.x == 0 && tc_status != 0) atomicAdd(&g_wait_timeouts, 1u);
    tc::release(tcx.st, tmem_cols(PASSES));
}

// ------------------------------------------------------------------ k_bprep

template <typename Tin, int D, int PASSES, int CF>
__global__ void __launch_bounds__(kThreads, fwd_ctas(PASSES)) k_bprep(KParams p) {
    if (p.gate && *p.gate == 0) return;
    __shared__ uint32_t tmem_slot;
    __shared__ __align__(8) uint64_t mbar;
    __shared__ int tc_status;
    extern __shared__ __align__(128) unsigned char dsm[];
    TcCta tcx;
    tcx.sbuf = dsm + ((1024u - (tc::smem_addr(dsm) & 1023u)) & 1023u);  // 1 KB aligned
    tcx.sbytes = (int)tc::dynamic_smem_bytes() - (int)(tcx.sbuf - dsm);
    tc::init(tcx.st, &tmem_slot, &mbar, &tc_status, tmem_cols(PASSES));
    float* sm = reinterpret_cast<float*>(dsm);
    float* slot = p.scratch + (size_t)blockIdx.x * p.slot;
    const int nch = p.B * p.H * p.N;
    for (int chunk = blockIdx.x; chunk < nch; chunk += gridDim.x) {
        Chunk<Tin, D> c = make_chunk<Tin, D, CF>(p, chunk, slot);
        const Lay& L = c.L;
        const int C = L.C;
        float* s = c.s;
        prologue2(c);
        rows_prep<Tin, D, PASSES>(c, R_KT | R_QT | R_DO);
        if (p.aux) {  // L_A, M_QA and the block inverses the forward saved
            aux_copy(c, p.aux + c.sidx * make_aux_lay(C, D).total, false, 1 | 8 | 16, 0);
        } else {
            masked_prep<Tin, D, PASSES>(c, true, false);
            masked_pair<Tin, D, PASSES, OP_K, OP_A, OP_K>(c, tcx, sm, L.LA, L.LK, false, false);
            masked_pair<Tin, D, PASSES, OP_Q, OP_K, OP_A>(c, tcx, sm, L.MQK, L.MQA, true, true);
            __syncthreads();
            compute_tii(s, L, L.LA);
            __syncthreads();
        }
        float* Xi = s + L.W[0];
        // Z0 = M_QA^T dO
        tc_rows2<PASSES, D, true, true>(tcx, C, C,
            [&](int) { return tc::Src{s + L.MQA, C, 0, true, false}; },
            [&](int t, int k, float* v) { for (int u = 0; u < 4; ++u) v[u] = s[L.MQA + (size_t)(k + u) * C + t]; },
            [&](int) { return tc::Src{s + L.RDO, D, 0, true, false}; },
            [&](int cc, int k, float* v) { for (int u = 0; u < 4; ++u) v[u] = c.dOv(k + u, cc); },
            tc::RowStore{Xi, D});
        solve_s<D, PASSES, true>(s, sm, L, L.LA, L.W[0]);  // Xi = T^T Z0
        __syncthreads();
        float* Bp = p.Bn + c.sbase;
        const Fac<Tin, D> f = facs(c);
        // B' = Qt^T dO - Kt^T Xi
        tc_rows2<PASSES, D, true, true>(tcx, D, 2 * C,
            [&](int k) {
                return k < C ? tc::Src{s + L.RQT, D, 0, true, false} : tc::Src{s + L.RKT, D, C, true, true};
            },
            [&](int i, int k, float* v) {
                if (k < C) for (int u = 0; u < 4; ++u) v[u] = c.Qh(k + u, i) * f.eg(k + u, i);
                else for (int u = 0; u < 4; ++u) v[u] = -c.K(k - C + u, i) * f.eg(k - C + u, i);
            },
            [&](int k) { return k < C ? tc::Src{s + L.RDO, D, 0, true, false} : tc::Src{Xi, D, C, true, false}; },
            [&](int cc, int k, float* v) {
                if (k < C) for (int u = 0; u < 4; ++u) v[u] = c.dOv(k + u, cc);
                else for (int u = 0; u < 4; ++u) v[u] = Xi[(size_t)(k - C + u) * D + cc];
            },
            tc::RowStore{Bp, D});
    }
    if (threadIdx.x == 0 && tc_status != 0) atomicAdd(&g_wait_timeouts, 1u);
    tc::release(tcx.st, tmem_cols(PASSES));
}

// ------------------------------------------------------------------ k_bwd

template <typename Tin, int D, int PASSES, int CF>
__global__ void __launch_bounds__(kThreads) k_bwd(KParams p) {
    if (p.gate && *p.gate == 0) return;
    __shared__ float s_colsum[D];
    __shared__ float s_segtot[kThreads];
    __shared__ float s_red[kThreads * 4];
    __shared__ uint32_t tmem_slot;
    __shared__ __align__(8) uint64_t mbar;
    __shared__ int tc_status;
    extern __shared__ __align__(128) unsigned char dsm[];
    TcCta tcx;
    tcx.sbuf = dsm + ((1024u - (tc::smem_addr(dsm) & 1023u)) & 1023u);  // 1 KB aligned
    tcx.sbytes = (int)tc::dynamic_smem_bytes() - (int)(tcx.sbuf - dsm);
    tc::init(tcx.st, &tmem_slot, &mbar, &tc_status, tmem_cols(PASSES, true));
    float* sm = reinterpret_cast<float*>(dsm);
    float* slot = p.scratch + (size_t)blockIdx.x * p.slot;
    const int nch = p.B * p.H * p.N;
    for (int chunk = blockIdx.x; chunk < nch; chunk += gridDim.x) {
        Chunk<Tin, D> c = make_chunk<Tin, D, CF>(p, chunk, slot);
        const Lay& L = c.L;
        const int C = L.C;
        float* s = c.s;
        const float* S = p.S_chunks + c.sbase;
        const float* dS = p.dS_chunks + c.sbase;
        const size_t Y = L.W[0], dR = L.W[1], dK = L.W[2], dQh = L.W[3], dA = L.W[4],
                     dU = L.W[5], dGam = L.W[6];
        prologue2(c);
        masked_prep<Tin, D, PASSES>(c, true, true, !p.aux);  // path choice and gradient operands
        rows_prep<Tin, D, PASSES, 2>(c, (p.aux ? 0 : R_KT) | R_UU | R_DO | R_AB | R_KB);  // Kt: for Y
        if (p.aux) {  // masked matrices, block inverses and Y the forward saved
            aux_copy(c, p.aux + c.sidx * make_aux_lay(C, D).total, false, 63, Y);
        } else {
            masked_pair<Tin, D, PASSES, OP_K, OP_A, OP_K>(c, tcx, sm, L.LA, L.LK, false, false);
            masked_pair<Tin, D, PASSES, OP_Q, OP_K, OP_A>(c, tcx, sm, L.MQK, L.MQA, true, true);
            __syncthreads();
            compute_tii(s, L, L.LA);
            __syncthreads();
            compute_Y<Tin, D, PASSES>(tcx, c, S, Y);
        }
        const Fac<Tin, D> f = facs(c);
        // dY = -M_QA^T dO - Ab dS'   (stored in dR, then dR = T^T dY)
        tc_rows2<PASSES, D, true, true>(tcx, C, C + D,
            [&](int k) {
                return k < C ? tc::Src{s + L.MQA, C, 0, true, false} : tc::Src{s + L.RAB, D, C, false, false};
            },
            [&](int t, int k, float* v) {
                if (k < C) for (int u = 0; u < 4; ++u) v[u] = s[L.MQA + (size_t)(k + u) * C + t];
                else {
                    float k4[4];
                    ld4in(c.e + c.base + t * c.rs + (k - C), v);
                    ld4in(c.k + c.base + t * c.rs + (k - C), k4);
                    for (int u = 0; u < 4; ++u) v[u] *= k4[u] * f.egb(t, k - C + u);
                }
            },
            [&](int k) { return k < C ? tc::Src{s + L.RDO, D, 0, true, false} : tc::Src{dS, D, C, true, false}; },
            [&](int cc, int k, float* v) {
                if (k < C) for (int u = 0; u < 4; ++u) v[u] = c.dOv(k + u, cc);
                else for (int u = 0; u < 4; ++u) v[u] = __ldg(dS + (size_t)(k - C + u) * D + cc);
            },
            [&](int t, int j, float x) { s[dR + (size_t)t * D + j] = -x; });
        solve_s<D, PASSES, true>(s, sm, L, L.LA, dR);  // dR = T^T dY
        __syncthreads();
        // B(k = c, n = j) = S[j][c] or dS'[j][c]: rows of the staged B are rows of S
        auto rowsS = [&](int j, int k, float* v) { ld4in(S + (size_t)j * D + k, v); };
        auto rowsdS = [&](int j, int k, float* v) { ld4in(dS + (size_t)j * D + k, v); };
        // raw products, then one elementwise pass applies the decay factors:
        //   dQt = dO S^T, dKt = dR S^T, dKb = U dS'^T, dAb = -Y dS'^T
        auto srcS = [&](int) { return tc::Src{S, D, 0, false, false}; };
        auto srcdS = [&](int) { return tc::Src{dS, D, 0, false, false}; };
        tc_rows2<PASSES, D, false, false>(tcx, C, D, [&](int) { return tc::Src{s + L.RDO, D, 0, false, false}; },
            [&](int t, int k, float* v) { ld4in(c.dO + c.base + t * c.rs + k, v); }, srcS, rowsS,
            tc::RowStore{s + dQh, D});
        tc_rows2<PASSES, D, false, false>(tcx, C, D,
            [&](int) { return tc::Src{s + dR, D, 0, false, false}; },
            [&](int t, int k, float* v) { ld4(s + dR + (size_t)t * D + k, v); }, srcS, rowsS,
            tc::RowStore{s + dK, D});
        tc_rows2<PASSES, D, false, false>(tcx, C, D, [&](int) { return tc::Src{s + L.RUU, D, 0, false, false}; },
            [&](int t, int k, float* v) {
                float w4[4];
                ld4in(c.v + c.base + t * c.rs + k, v);
                ld4in(c.w + c.base + t * c.rs + k, w4);
                for (int u = 0; u < 4; ++u) v[u] *= w4[u];
            },
            srcdS, rowsdS, tc::RowStore{s + dGam, D});
        tc_rows2<PASSES, D, false, false>(tcx, C, D,
            [&](int) { return tc::Src{s + Y, D, 0, false, true}; },
            [&](int t, int k, float* v) {
                ld4(s + Y + (size_t)t * D + k, v);
                for (int u = 0; u < 4; ++u) v[u] = -v[u];
            },
            srcdS, rowsdS, tc::RowStore{s + dA, D});
        float cpart[4] = {0.f, 0.f, 0.f, 0.f};  // this thread's share of the column sums
        // dQh = dQt e^Gam;  dK = dKt e^Gam + dKb e^{gbar-Gam};  dA = dAb e^{gbar-Gam};
        // dGam = dQt Qt + dKt Kt - dKb Kb - dAb Ab;  dgbar += sum_t (dKb Kb + dAb Ab)
        for (int idx = threadIdx.x; idx < C * D / 4; idx += kThreads) {
            const int t = idx / (D / 4), j = 4 * (idx % (D / 4));
            const size_t i = (size_t)t * D + j;
            float r1[4], r2[4], r3[4], r4[4], lc[4], rc[4], pre[4], suf[4], q4[4], gm4[4], k4[4], e4[4];
            ld4(s + dQh + i, r1); ld4(s + dK + i, r2); ld4(s + dGam + i, r3); ld4(s + dA + i, r4);
            ld4(s + L.LC + i, lc); ld4(s + L.RC + i, rc);
            ld4(s + L.PRE + (size_t)(t >> 3) * D + j, pre); ld4(s + L.SUF + (size_t)(t >> 3) * D + j, suf);
            const size_t gi = c.base + t * c.rs + j;
            ld4in(c.q + gi, q4); ld4in(c.gm + gi, gm4); ld4in(c.k + gi, k4); ld4in(c.e + gi, e4);
            float o1[4], o2[4], o3[4], o4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float eg = fexp<Tin>(pre[u] + lc[u]), egb = fexp<Tin>(rc[u] + suf[u]);
                const float kt = k4[u] * eg, qt = q4[u] * gm4[u] * eg;
                const float kb = k4[u] * egb, ab = e4[u] * k4[u] * egb;
                o1[u] = r1[u] * eg;
                o2[u] = r2[u] * eg + r3[u] * egb;
                o4[u] = r4[u] * egb;
                o3[u] = r1[u] * qt + r2[u] * kt - r3[u] * kb - r4[u] * ab;
                cpart[u] += r3[u] * kb + r4[u] * ab;
            }
            *reinterpret_cast<float4*>(s + dQh + i) = make_float4(o1[0], o1[1], o1[2], o1[3]);
            *reinterpret_cast<float4*>(s + dK + i) = make_float4(o2[0], o2[1], o2[2], o2[3]);
            *reinterpret_cast<float4*>(s + dGam + i) = make_float4(o3[0], o3[1], o3[2], o3[3]);
            *reinterpret_cast<float4*>(s + dA + i) = make_float4(o4[0], o4[1], o4[2], o4[3]);
        }
        // column sums in a fixed order (deterministic): every thread always saw the
        // same 4 channels, 4 * (threadIdx % (D/4)) .. + 3
#pragma unroll
        for (int u = 0; u < 4; ++u) s_red[threadIdx.x * 4 + u] = cpart[u];
        __syncthreads();
        if (threadIdx.x < D) {
            const int jg = threadIdx.x / 4, u = threadIdx.x % 4;
            float acc = 0.f;
            for (int th = jg; th < kThreads; th += D / 4) acc += s_red[th * 4 + u];
            s_colsum[threadIdx.x] = acc;
        }
        __syncthreads();
        // dU = M_QK^T dO + L_K^T dR + Kb dS'
        tc_rows2<PASSES, D, true, true>(tcx, C, 2 * C + D,
            [&](int k) {
                return k < C ? tc::Src{s + L.MQK, C, 0, true, false}
                             : (k < 2 * C ? tc::Src{s + L.LK, C, C, true, false}
                                          : tc::Src{s + L.RKB, D, 2 * C, false, false});
            },
            [&](int t, int k, float* v) {
                if (k < C) for (int u = 0; u < 4; ++u) v[u] = s[L.MQK + (size_t)(k + u) * C + t];
                else if (k < 2 * C) for (int u = 0; u < 4; ++u) v[u] = s[L.LK + (size_t)(k - C + u) * C + t];
                else {
                    ld4in(c.k + c.base + t * c.rs + (k - 2 * C), v);
                    for (int u = 0; u < 4; ++u) v[u] *= f.egb(t, k - 2 * C + u);
                }
            },
            [&](int k) {
                return k < C ? tc::Src{s + L.RDO, D, 0, true, false}
                             : (k < 2 * C ? tc::Src{s + dR, D, C, true, false}
                                          : tc::Src{dS, D, 2 * C, true, false});
            },
            [&](int cc, int k, float* v) {
                if (k < C) for (int u = 0; u < 4; ++u) v[u] = c.dOv(k + u, cc);
                else if (k < 2 * C) for (int u = 0; u < 4; ++u) v[u] = s[dR + (size_t)(k - C + u) * D + cc];
                else for (int u = 0; u < 4; ++u) v[u] = __ldg(dS + (size_t)(k - 2 * C + u) * D + cc);
            },
            tc::RowStore{s + dU, D});
        // gradients of the masked products (overwrite them): dL_A = -strict(dR Y^T),
        // dL_K = strict(dR U^T), dM_QK = incl(dO U^T), dM_QA = -incl(dO Y^T)
        for (int which = 0; which < 4; ++which) {
            const size_t out = which == 0 ? L.LA : which == 1 ? L.LK : which == 2 ? L.MQK : L.MQA;
            const bool incl = which >= 2;
            const float sg = (which == 0 || which == 3) ? -1.f : 1.f;
            for (int n0 = 0; n0 < C; n0 += 128) {
                // masked, signed rows (and, for the single-pivot products, the
                // tensor-core layouts of the same rows)
                auto gepi = [&](int t, int n, const float* x) {
                    const int s0 = n0 + n;
                    if (s0 >= C) return;
                    float w[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int ss = s0 + u;
                        w[u] = (incl ? ss <= t : ss < t) ? sg * x[u] : 0.f;
                    }
                    if (c.tame) {
                        store_g_layouts(s, L, which, t, s0, w);
                    } else {
                        float* d = s + out + (size_t)t * C + s0;
                        *reinterpret_cast<float4*>(d) = make_float4(w[0], w[1], w[2], w[3]);
                        *reinterpret_cast<float4*>(d + 4) = make_float4(w[4], w[5], w[6], w[7]);
                    }
                };
                tc_rows2<PASSES, 128, false, false>(tcx, C, D,
                    [&](int) {
                        return which < 2 ? tc::Src{s + dR, D, 0, false, false}
                                         : tc::Src{s + L.RDO, D, 0, false, false};
                    },
                    [&](int t, int k, float* v) {
                        if (which < 2) ld4(s + dR + (size_t)t * D + k, v);
                        else ld4in(c.dO + c.base + t * c.rs + k, v);
                    },
                    [&](int) {
                        return (which == 0 || which == 3)
                                   ? tc::Src{s + Y + (size_t)n0 * D, D, 0, false, false}
                                   : tc::Src{s + L.RUU + (size_t)n0 * D, D, 0, false, false};
                    },
                    [&](int n, int k, float* v) {
                        const int ss = n0 + n;
                        if (ss >= C) { v[0] = v[1] = v[2] = v[3] = 0.f; return; }
                        if (which == 0 || which == 3) ld4(s + Y + (size_t)ss * D + k, v);
                        else {
                            float w4[4];
                            ld4in(c.v + c.base + ss * c.rs + k, v);
                            ld4in(c.w + c.base + ss * c.rs + k, w4);
                            for (int u = 0; u < 4; ++u) v[u] *= w4[u];
                        }
                    },
                    tc::Row8<decltype(gepi)>{gepi},
                    C - n0 < 128 ? C - n0 : 128);
            }
        }
        __syncthreads();
        // X side: dK += dL_A (*) A + dL_K (*) K ; dQh += dM_QK (*) K + dM_QA (*) A ; dGam += X * dX
        // dst[t][j] += v and dGam[t][j] += sg * op_tj * v for N consecutive tokens
        // (all loads first, then the stores)
        auto accum = [&](size_t dst, auto opk, float sg) {
            return [&, dst, sg](auto NN, int t0, int j, const float* v) {
                constexpr int N = decltype(NN)::value;
                float a[N], gm[N], o[N];
#pragma unroll
                for (int u = 0; u < N; ++u) {
                    const size_t x = (size_t)(t0 + u) * D + j;
                    a[u] = s[dst + x];
                    gm[u] = s[dGam + x];
                    o[u] = opval(c, decltype(opk)::value, t0 + u, j);
                }
#pragma unroll
                for (int u = 0; u < N; ++u) {
                    const size_t x = (size_t)(t0 + u) * D + j;
                    s[dst + x] = a[u] + v[u];
                    s[dGam + x] = gm[u] + sg * o[u] * v[u];
                }
            };
        };
        using OK_ = std::integral_constant<int, OP_K>;
        using OQ_ = std::integral_constant<int, OP_Q>;
        using OA_ = std::integral_constant<int, OP_A>;
        Tin* gq = (Tin*)p.dq; Tin* gk = (Tin*)p.dk; Tin* gv = (Tin*)p.dv; Tin* gg = (Tin*)p.dg;
        Tin* ge = (Tin*)p.de; Tin* gw = (Tin*)p.dw; Tin* ggm = (Tin*)p.dgamma;
        if (c.tame) {
            // single-pivot products: the four gradient pairs accumulate in TMEM
            // (X side: dK, dQh; Z side: dA, dK), then one pass finishes every
            // token's gradients: dK, dQh, dA, dGam and the input gradients but dg
            fast_grad_mma<Tin, D, true, OP_A, OP_K>(c, tcx, L.LA, L.LK, 0);
            fast_grad_mma<Tin, D, true, OP_K, OP_A>(c, tcx, L.MQK, L.MQA, 128);
            fast_grad_mma<Tin, D, false, OP_K, OP_Q>(c, tcx, L.LA, L.MQA, 256);
            fast_grad_mma<Tin, D, false, OP_K, OP_Q>(c, tcx, L.LK, L.MQK, 384);
            const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
            const int q = warp & 3, half = warp >> 2, cc = 32 * q + lane;
            const uint32_t lane_base = tcx.st.tmem + ((uint32_t)(32 * q) << 16);
            if (32 * q < D) {
                const float hp = 0.5f * s[L.GBAR + cc];
                for (int I = half; I < L.nb8; I += 2) {
                    const int t0 = 8 * I;
                    float x1[8], x2[8], z1[8], z2[8];
                    tmem_ld8(lane_base + 8 * I, x1);
                    tmem_ld8(lane_base + 128 + 8 * I, x2);
                    tmem_ld8(lane_base + 256 + 8 * I, z1);
                    tmem_ld8(lane_base + 384 + 8 * I, z2);
                    const float pre = s[L.PRE + (size_t)I * D + cc];
                    // all loads of the block first, then the arithmetic and the stores
                    float lc[8], kv[8], qv[8], gmv[8], ev[8], vv[8], wv[8];
                    float dk0[8], dq0[8], da0[8], dg0[8], du0[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const size_t x = (size_t)(t0 + u) * D + cc, gi = c.base + (size_t)(t0 + u) * c.rs + cc;
                        lc[u] = s[L.LC + x];
                        kv[u] = ldf(c.k + gi); qv[u] = ldf(c.q + gi); gmv[u] = ldf(c.gm + gi);
                        ev[u] = ldf(c.e + gi); vv[u] = ldf(c.v + gi); wv[u] = ldf(c.w + gi);
                        dk0[u] = s[dK + x]; dq0[u] = s[dQh + x]; da0[u] = s[dA + x];
                        dg0[u] = s[dGam + x]; du0[u] = s[dU + x];
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const size_t x = (size_t)(t0 + u) * D + cc, gi = c.base + (size_t)(t0 + u) * c.rs + cc;
                        const float d = pre + lc[u] - hp;
                        const float fx = fexp<Tin>(d), fz = fexp<Tin>(-d);
                        const float vx1 = fx * x1[u], vx2 = fx * x2[u], vz1 = fz * z1[u], vz2 = fz * z2[u];
                        const float DK = dk0[u] + vx1 + vz2, DQ = dq0[u] + vx2, DA = da0[u] + vz1;
                        s[dGam + x] = dg0[u] + kv[u] * (vx1 - vz2) + qv[u] * gmv[u] * vx2 - ev[u] * kv[u] * vz1;
                        stf(gq + gi, DQ * gmv[u]);
                        stf(ggm + gi, DQ * qv[u]);
                        stf(ge + gi, DA * kv[u]);
                        stf(gk + gi, DK + DA * ev[u]);
                        stf(gw + gi, du0[u] * vv[u]);
                        stf(gv + gi, du0[u] * wv[u]);
                    }
                }
            }
            panel_end();
        } else {
            decayed_grad<Tin, D, PASSES, true, OP_A, OP_K>(c, tcx, sm, L.LA, L.LK, accum(dK, OK_{}, 1.f));
            decayed_grad<Tin, D, PASSES, true, OP_K, OP_A>(c, tcx, sm, L.MQK, L.MQA, accum(dQh, OQ_{}, 1.f));
            __syncthreads();
            // Z side: dA += dL_A^T (*) K + dM_QA^T (*) Qh ; dK += dL_K^T (*) K + dM_QK^T (*) Qh ; dGam -= Z * dZ
            decayed_grad<Tin, D, PASSES, false, OP_K, OP_Q>(c, tcx, sm, L.LA, L.MQA, accum(dA, OA_{}, -1.f));
            __syncthreads();
            decayed_grad<Tin, D, PASSES, false, OP_K, OP_Q>(c, tcx, sm, L.LK, L.MQK, accum(dK, OK_{}, -1.f));
            __syncthreads();
        }
        // dgbar_j = e^gbar_j sum_c S[j][c] dS'[j][c] + sum_t (dKb Kb + dAb Ab)[t][j]
        {
            const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
            for (int j = warp; j < D; j += kThreads / 32) {
                float acc = 0.f;
                for (int cc = lane; cc < D; cc += 32)
                    acc += __ldg(S + (size_t)j * D + cc) * __ldg(dS + (size_t)j * D + cc);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                if (lane == 0) s_colsum[j] += acc * expf(facs(c).gbar(j));
            }
        }
        __syncthreads();
        // dg_t = dgbar + sum_{t' >= t} dGam[t'] : token segments per thread, segment
        // totals combined through shared memory
        {
            constexpr int SEG = kThreads / D;
            const int j = threadIdx.x % D, seg = threadIdx.x / D, len = C / SEG;
            const int t0 = seg * len;
            float tot = 0.f;
            for (int t = t0; t < t0 + len; t += 8) {
                float v8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) v8[u] = s[dGam + (size_t)(t + u) * D + j];
#pragma unroll
                for (int u = 0; u < 8; ++u) tot += v8[u];
            }
            s_segtot[seg * D + j] = tot;
            __syncthreads();
            float run = s_colsum[j];
            for (int sg = seg + 1; sg < SEG; ++sg) run += s_segtot[sg * D + j];
            for (int t1 = t0 + len - 8; t1 >= t0; t1 -= 8) {
                float v8[8], g8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    v8[u] = s[dGam + (size_t)(t1 + u) * D + j];
                    g8[u] = ldf(c.g + c.base + (size_t)(t1 + u) * c.rs + j);
                }
#pragma unroll
                for (int u = 7; u >= 0; --u) {
                    run += v8[u];
                    stf(gg + c.base + (size_t)(t1 + u) * c.rs + j, g8[u] >= kLogDecayMin ? run : 0.f);
                }
            }
        }
        for (int idx = threadIdx.x; !c.tame && idx < C * D / 4; idx += kThreads) {
            const int t = idx / (D / 4), j = 4 * (idx % (D / 4));
            const size_t gi = c.base + t * c.rs + j;
            const size_t li = (size_t)t * D + j;
            float qv[4], gmv[4], kv[4], ev[4], vv[4], wv[4], dqh[4], da[4], du[4], dk4[4];
            ld4in(c.q + gi, qv); ld4in(c.gm + gi, gmv); ld4in(c.k + gi, kv);
            ld4in(c.e + gi, ev); ld4in(c.v + gi, vv); ld4in(c.w + gi, wv);
            ld4(s + dQh + li, dqh); ld4(s + dA + li, da); ld4(s + dU + li, du); ld4(s + dK + li, dk4);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                stf(gq + gi + u, dqh[u] * gmv[u]);
                stf(ggm + gi + u, dqh[u] * qv[u]);
                stf(ge + gi + u, da[u] * kv[u]);
                stf(gk + gi + u, dk4[u] + da[u] * ev[u]);
                stf(gw + gi + u, du[u] * vv[u]);
                stf(gv + gi + u, du[u] * wv[u]);
            }
        }
        __syncthreads();
    }
    if (threadIdx.x == 0 && tc_status != 0) atomicAdd(&g_wait_timeouts, 1u);
    tc::release(tcx.st, tmem_cols(PASSES, true));
}

// ------------------------------------------------------------------ host side

// Dynamic shared memory of the per-chunk kernels: the largest staging area of
// their phases (tensor-core slabs, masked products, gradient products, solves).
template <int D, int PASSES>
int dyn_bytes(int C, bool bwd) {
    int f = tc::stage_bytes<PASSES, 128>() / 4;
    if (PASSES == 1 && tc::async_stage_bytes<128>() / 4 > f) f = tc::async_stage_bytes<128>() / 4;
    const int m = masked_smem_floats(C, D), s = solve_smem_floats(C, D);
    f = f > m ? f : m;
    f = f > s ? f : s;
    if (PASSES == 1 && C <= 128) {
        const int pr = pair_smem_bytes() / 4, fp = kFastPairSmem / 4;
        f = f > pr ? f : pr;
        f = f > fp ? f : fp;
    }
    if (bwd) {
        const int g = decayed_smem_floats(C);
        f = f > g ? f : g;
        if (PASSES == 1 && C <= 128) {
            const int pg = panel_smem_bytes() / 4, fg = kFastGradSmem / 4;
            f = f > pg ? f : pg;
            f = f > fg ? f : fg;
        }
    }
    return f * 4 + 1024;  // + alignment of the staging buffers
}


template <typename Tin, int D, int PASSES, int CF>
cudaError_t set_smem_attrs(int bytes, int bwd_bytes) {
    // dynamic shared memory limit and the largest shared-memory carveout, so
    // that as many CTAs as the budgets allow fit on one SM
    auto set = [](const void* f, int n) {
        cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, n);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
        return e;
    };
    cudaError_t e = set((const void*)k_intra<Tin, D, PASSES, CF>, bytes);
    if (e == cudaSuccess) e = set((const void*)k_out<Tin, float, D, PASSES, CF>, bytes);
    if (e == cudaSuccess) e = set((const void*)k_out<Tin, __nv_bfloat16, D, PASSES, CF>, bytes);
    if (e == cudaSuccess) e = set((const void*)k_bprep<Tin, D, PASSES, CF>, bytes);
    if (e == cudaSuccess) e = set((const void*)k_bwd<Tin, D, PASSES, CF>, bwd_bytes);
    return e;
}

inline int num_slots(int nch) { return nch < kMaxSlots ? nch : kMaxSlots; }

inline size_t slot_floats(int C, int D) { return make_lay(C, D).total; }

// Side buffers of a ragged last chunk, counted in floats (4-byte elements
// bound both dtypes): 8 input tensors and 7 output tensors of [B*H][C][D].
inline size_t tail_side_floats(int B, int T, int H, int D, int C) {
    return T % C ? (size_t)15 * B * H * C * D : 0;
}

// A ragged problem (T % C != 0) runs its per-chunk kernels as two launches:
// `main` over the N - 1 whole chunks of every sequence, and `tail` over the
// last chunk of every sequence, read from a zero-padded side copy laid out
// as a problem of B*H sequences, one head, C tokens (row stride D).  Both
// address the same per-chunk arrays (nstride = N).  Staging copies the k
// input tensors (dO included in the backward) into the side buffer and points
// `tail` at it; `tail.o` / the gradient pointers go to the output side buffer.
struct Launches {
    KParams main, tail;
    bool ragged;
    size_t E;         // elements per side tensor, B*H*C*D
    char* side_out;   // output side buffer (7 tensors of E elements)
};

template <typename Tin, int D>
cudaError_t stage_tail(Launches& L, const KParams& kp, const void* const* in, int k, float* side,
                       cudaStream_t st) {
    L.main = kp;
    L.main.nstride = kp.N;
    L.main.noff = 0;
    L.ragged = kp.T % kp.C != 0;
    if (!L.ragged) return cudaSuccess;
    L.main.N = kp.N - 1;
    L.E = (size_t)kp.B * kp.H * kp.C * D;
    Tin* tin = reinterpret_cast<Tin*>(side);
    L.side_out = reinterpret_cast<char*>(side + 8 * L.E);
    KParams& t = L.tail;
    t = L.main;
    t.B = kp.B * kp.H; t.H = 1; t.T = kp.C; t.N = 1; t.noff = kp.N - 1;
    const void** dst[8] = {&t.q, &t.k, &t.v, &t.g, &t.e, &t.w, &t.gamma, &t.dO};
    TailCopy io = {};
    io.n = k;
    for (int i = 0; i < k; ++i) {
        io.src[i] = in[i];
        io.dst[i] = tin + i * L.E;
        *dst[i] = tin + i * L.E;
    }
    return tail_gather(io, kp.B, kp.H, kp.T, kp.C, D, (int)sizeof(Tin), st);
}

// Copy the tail rows of k output tensors (esize bytes per element) from the
// output side buffer to their token-major destinations.
inline cudaError_t unstage_tail(const Launches& L, const KParams& kp, void* const* out, int k,
                                int D, int esize, cudaStream_t st) {
    if (!L.ragged) return cudaSuccess;
    TailCopy io = {};
    io.n = k;
    for (int i = 0; i < k; ++i) {
        io.src[i] = L.side_out + i * L.E * esize;
        io.dst[i] = out[i];
    }
    return tail_scatter(io, kp.B, kp.H, kp.T, kp.C, D, esize, st);
}

// Persistent grid of a chunk kernel: one CTA per resident slot (SM count x
// CTAs that fit per SM by registers, shared memory and threads, from the
// kernel's attributes), at most one per scratch slot.  Call after the
// kernel's shared-memory attribute is set.  (The runtime occupancy query
// reports one CTA per SM for these kernels where two fit.)  CTAs never wait
// on one another, so an over-estimate only delays the surplus CTAs.
template <class KERNEL>
int persistent_grid(KERNEL kernel, int nch, int dyn) {
    int dev = 0, nsm = 148, regs_sm = 65536, smem_sm = 233472, reserve = 1024;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
        cudaDeviceGetAttribute(&reserve, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    }
    int occ = 1;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) == cudaSuccess && fa.numRegs > 0) {
        const int warp_regs = ((fa.numRegs * 32 + 255) / 256) * 256;  // per-warp allocation unit
        const int by_regs = regs_sm / (warp_regs * (kThreads / 32));
        const int by_smem = smem_sm / ((int)fa.sharedSizeBytes + dyn + reserve);
        const int by_thr = 2048 / kThreads;
        occ = by_regs < by_smem ? by_regs : by_smem;
        occ = occ < by_thr ? occ : by_thr;
        if (occ < 1) occ = 1;
    }
    const int g = num_slots(nch);
    return g < nsm * occ ? g : nsm * occ;
}

template <int D, int SL, int PASSES, bool REV>
cudaError_t launch_chain_slab(int BH, int N, const float* M, const float* Bn, const float* S_in,
                              float* S_rec, float* S_out, const int* gate, cudaStream_t st) {
    constexpr int bytes = chain_smem_bytes<D, SL>();
    cudaError_t e = cudaFuncSetAttribute(k_chain<D, SL, PASSES, REV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    MUIR_TIMED(REV ? "k_chain_rev" : "k_chain", st,
               k_chain<D, SL, PASSES, REV><<<BH * (D / SL), kThreads, bytes, st>>>(M, Bn, S_in, S_rec, S_out, N, gate));
    return cudaGetLastError();
}

template <int D, int PASSES, bool REV>
cudaError_t launch_chain(int BH, int N, const float* M, const float* Bn, const float* S_in,
                                float* S_rec, float* S_out, const int* gate, cudaStream_t st) {
    // column slabs: enough CTAs to cover the GPU when B*H is small
    if (BH >= 64) return launch_chain_slab<D, 32, PASSES, REV>(BH, N, M, Bn, S_in, S_rec, S_out, gate, st);
    return launch_chain_slab<D, 16, PASSES, REV>(BH, N, M, Bn, S_in, S_rec, S_out, gate, st);
}

template <typename Tin, int D, int PASSES, int CF>
cudaError_t fwd_impl(const ChunkProblem& P, const float* S0, void* o, float* S_final,
                            float* S_chunks, float* M_chunks, void* ws, cudaStream_t st) {
    const int nch = P.B * P.H * P.N, BH = P.B * P.H;
    const size_t DD = (size_t)D * D;
    float* f = static_cast<float*>(ws);
    KParams kp = {};
    kp.B = P.B; kp.T = P.T; kp.H = P.H; kp.C = P.C; kp.N = P.N;
    kp.q = P.q; kp.k = P.k; kp.v = P.v; kp.g = P.g; kp.e = P.e; kp.w = P.w; kp.gamma = P.gamma;
    kp.gate = P.gate;
    kp.M = f; f += nch * DD;
    if (M_chunks) kp.M = M_chunks;
    kp.Bn = f; f += nch * DD;
    float* Sc = S_chunks;
    if (!Sc) { Sc = f; f += nch * DD; }
    kp.scratch = f;
    kp.slot = slot_floats(P.C, D);
    kp.S_chunks = Sc;
    kp.o = o;
    kp.aux = P.aux;
    const int dyn = dyn_bytes<D, PASSES>(P.C, false);
    cudaError_t err = set_smem_attrs<Tin, D, PASSES, CF>(dyn, dyn_bytes<D, PASSES>(P.C, true));
    if (err != cudaSuccess) return err;
    const void* in[7] = {P.q, P.k, P.v, P.g, P.e, P.w, P.gamma};
    Launches Ls;
    err = stage_tail<Tin, D>(Ls, kp, in, 7, f + (size_t)num_slots(nch) * kp.slot, st);
    if (err != cudaSuccess) return err;
    if (Ls.ragged) Ls.tail.o = Ls.side_out;
    // per-chunk kernel over the whole chunks, then over the padded last chunks
    auto each = [&](auto kernel, const char* name) -> cudaError_t {
        for (int part = 0; part < 2; ++part) {
            const KParams& q = part ? Ls.tail : Ls.main;
            if ((part && !Ls.ragged) || q.N == 0) continue;
            const int grid = persistent_grid(kernel, q.B * q.H * q.N, dyn);
            MUIR_TIMED(name, st, kernel<<<grid, kThreads, dyn, st>>>(q));
            const cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    };
    if ((err = each(k_intra<Tin, D, PASSES, CF>, "k_intra")) != cudaSuccess) return err;
    err = launch_chain<D, PASSES, false>(BH, P.N, kp.M, kp.Bn, S0, Sc, S_final, P.gate, st);
    if (err != cudaSuccess) return err;
    if (P.out_bf16) err = each(k_out<Tin, __nv_bfloat16, D, PASSES, CF>, "k_out");
    else err = each(k_out<Tin, float, D, PASSES, CF>, "k_out");
    if (err != cudaSuccess) return err;
    void* out[1] = {o};
    return unstage_tail(Ls, kp, out, 1, D, P.out_bf16 ? 2 : 4, st);
}

template <typename Tin, int D, int PASSES, int CF>
cudaError_t bwd_impl(const ChunkProblem& P, const float* S0, const float* S_chunks,
                            const float* M_chunks, const void* dO, const float* dS_final, void* dq, void* dk, void* dv,
                            void* dg, void* de, void* dw, void* dgamma, float* dS0, void* ws,
                            cudaStream_t st) {
    const int nch = P.B * P.H * P.N, BH = P.B * P.H;
    const size_t DD = (size_t)D * D;
    float* f = static_cast<float*>(ws);
    KParams kp = {};
    kp.B = P.B; kp.T = P.T; kp.H = P.H; kp.C = P.C; kp.N = P.N;
    kp.q = P.q; kp.k = P.k; kp.v = P.v; kp.g = P.g; kp.e = P.e; kp.w = P.w; kp.gamma = P.gamma;
    kp.gate = P.gate;
    kp.dO = dO;
    kp.M = f; f += nch * DD;
    kp.Bn = f; f += nch * DD;
    float* dSc = f; f += nch * DD;
    float* Sc = const_cast<float*>(S_chunks);
    const bool recompute = S_chunks == nullptr;
    if (recompute) { Sc = f; f += nch * DD; }
    kp.scratch = f;
    kp.slot = slot_floats(P.C, D);
    kp.S_chunks = Sc;
    kp.dS_chunks = dSc;
    kp.dq = dq; kp.dk = dk; kp.dv = dv; kp.dg = dg; kp.de = de; kp.dw = dw; kp.dgamma = dgamma;
    kp.aux = recompute ? nullptr : P.aux;  // the saved Y belongs to the saved chunk states
    const int dyn = dyn_bytes<D, PASSES>(P.C, false), dyn_b = dyn_bytes<D, PASSES>(P.C, true);
    cudaError_t err = set_smem_attrs<Tin, D, PASSES, CF>(dyn, dyn_b);
    if (err != cudaSuccess) return err;
    const bool have_M = M_chunks != nullptr && !recompute;
    if (have_M) kp.M = const_cast<float*>(M_chunks);  // the forward's transitions: nothing to recompute
    const void* in[8] = {P.q, P.k, P.v, P.g, P.e, P.w, P.gamma, dO};
    Launches Ls;
    err = stage_tail<Tin, D>(Ls, kp, in, 8, f + (size_t)num_slots(nch) * kp.slot, st);
    if (err != cudaSuccess) return err;
    if (Ls.ragged) {
        void** g[7] = {&Ls.tail.dq, &Ls.tail.dk, &Ls.tail.dv, &Ls.tail.dg, &Ls.tail.de,
                       &Ls.tail.dw, &Ls.tail.dgamma};
        for (int i = 0; i < 7; ++i) *g[i] = Ls.side_out + i * Ls.E * sizeof(Tin);
    }
    // per-chunk kernel over the whole chunks, then over the padded last chunks
    auto each = [&](auto kernel, const char* name, int smem) -> cudaError_t {
        for (int part = 0; part < 2; ++part) {
            const KParams& q = part ? Ls.tail : Ls.main;
            if ((part && !Ls.ragged) || q.N == 0) continue;
            const int grid = persistent_grid(kernel, q.B * q.H * q.N, smem);
            MUIR_TIMED(name, st, kernel<<<grid, kThreads, smem, st>>>(q));
            const cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    };
    if (!have_M && (err = each(k_intra<Tin, D, PASSES, CF>, "k_intra", dyn)) != cudaSuccess)
        return err;
    if (recompute) {
        err = launch_chain<D, PASSES, false>(BH, P.N, kp.M, kp.Bn, S0, Sc, nullptr, P.gate, st);
        if (err != cudaSuccess) return err;
    }
    if ((err = each(k_bprep<Tin, D, PASSES, CF>, "k_bprep", dyn)) != cudaSuccess) return err;
    err = launch_chain<D, PASSES, true>(BH, P.N, kp.M, kp.Bn, dS_final, dSc, dS0, P.gate, st);
    if (err != cudaSuccess) return err;
    if ((err = each(k_bwd<Tin, D, PASSES, CF>, "k_bwd", dyn_b)) != cudaSuccess) return err;
    void* out[7] = {dq, dk, dv, dg, de, dw, dgamma};
    return unstage_tail(Ls, kp, out, 7, D, (int)sizeof(Tin), st);
}

}  // namespace muir

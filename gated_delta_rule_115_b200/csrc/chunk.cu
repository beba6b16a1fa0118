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
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"
#include "profile.h"

namespace muir {

constexpr int kThreads = 256;
constexpr int kMaxSlots = 296;  // 2 CTAs per SM on a 148-SM B200

// ------------------------------------------------------------------ scratch

struct Lay {
    int C, D, nb8, nb16;
    size_t G, EG, EGB, X8F, XOF, Z8F, ZOF, F, LA, LK, MQK, MQA, TII, W[8], total;
};

__host__ __device__ inline Lay make_lay(int C, int D) {
    Lay L;
    L.C = C; L.D = D; L.nb8 = C / 8; L.nb16 = C / 16;
    const size_t cd = (size_t)C * D, cc = (size_t)C * C;
    size_t o = 0;
#define MUIR_TAKE(field, n) L.field = o; o += ((size_t)(n) + 63) & ~(size_t)63;
    MUIR_TAKE(G, cd) MUIR_TAKE(EG, cd) MUIR_TAKE(EGB, cd)
    MUIR_TAKE(X8F, cd) MUIR_TAKE(XOF, cd) MUIR_TAKE(Z8F, cd) MUIR_TAKE(ZOF, cd)
    MUIR_TAKE(F, (size_t)(C / 8) * (C / 8) * D)
    MUIR_TAKE(LA, cc) MUIR_TAKE(LK, cc) MUIR_TAKE(MQK, cc) MUIR_TAKE(MQA, cc)
    MUIR_TAKE(TII, (size_t)C * 16)
    for (int i = 0; i < 8; ++i) { MUIR_TAKE(W[i], cd) }
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
};

// Accessors of one chunk's inputs; row t of a [B,T,H,D] tensor.
template <typename Tin, int D>
struct Chunk {
    const Tin *q, *k, *v, *g, *e, *w, *gm, *dO;
    size_t rs, base, sbase;  // row stride (H*D), element offset of row 0, state offset
    float* s;                // scratch slot
    Lay L;
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

template <typename Tin, int D>
__device__ Chunk<Tin, D> make_chunk(const KParams& p, int chunk, float* slot) {
    Chunk<Tin, D> c;
    const int n = chunk % p.N, bh = chunk / p.N, h = bh % p.H, b = bh / p.H;
    c.q = (const Tin*)p.q; c.k = (const Tin*)p.k; c.v = (const Tin*)p.v; c.g = (const Tin*)p.g;
    c.e = (const Tin*)p.e; c.w = (const Tin*)p.w; c.gm = (const Tin*)p.gamma;
    c.dO = (const Tin*)p.dO;
    c.rs = (size_t)p.H * D;
    c.base = (((size_t)b * p.T + (size_t)n * p.C) * p.H + h) * D;
    c.sbase = ((size_t)bh * p.N + n) * D * D;
    c.s = slot;
    c.L = make_lay(p.C, D);
    return c;
}

// ------------------------------------------------------------------ prologue

// Gam (clamped cumulative log decay), e^Gam, e^{gbar-Gam}, pivot factor tables.
// The cumulative sum runs as a warp-level scan: each channel's C tokens are
// split into 256/D segments held by lanes of one warp; segment totals are
// combined with shuffles.
template <typename Tin, int D>
__device__ void prologue(const Chunk<Tin, D>& c) {
    const Lay& L = c.L;
    const int C = L.C, tid = threadIdx.x;
    constexpr int S = kThreads / D;  // segments per channel
    constexpr int CPW = 32 / S;      // channels per warp
    const int warp = tid >> 5, lane = tid & 31;
    const int j = warp * CPW + (lane % CPW), seg = lane / CPW, len = C / S;
    float* G = c.s + L.G;
    float run = 0.f;
    for (int i = 0; i < len; ++i) {
        const int t = seg * len + i;
        run += fmaxf(ldf(c.g + c.base + t * c.rs + j), kLogDecayMin);
        G[(size_t)t * D + j] = run;
    }
    float incl = run;
#pragma unroll
    for (int off = CPW; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    const float excl = incl - run;
    for (int i = 0; i < len; ++i) G[(size_t)(seg * len + i) * D + j] += excl;
    __syncthreads();
    for (int idx = tid; idx < C * D; idx += kThreads) {
        const int t = idx / D, jj = idx % D;
        const float Gt = G[idx], gb = G[(size_t)(C - 1) * D + jj];
        const int st = t & ~7;
        const float Gbef = st > 0 ? G[(size_t)(st - 1) * D + jj] : 0.f;
        const float Gm = G[(size_t)(st + 3) * D + jj], Ge = G[(size_t)(st + 7) * D + jj];
        c.s[L.EG + idx] = expf(Gt);
        c.s[L.EGB + idx] = expf(gb - Gt);
        c.s[L.X8F + idx] = expf(Gt - Gbef);
        c.s[L.XOF + idx] = expf(Gt - Gm);
        c.s[L.Z8F + idx] = expf(Ge - Gt);
        c.s[L.ZOF + idx] = expf(Gm - Gt);
    }
    const int nb8 = L.nb8;
    for (int idx = tid; idx < nb8 * nb8 * D; idx += kThreads) {
        const int I8 = idx / (nb8 * D), J8 = (idx / D) % nb8, jj = idx % D;
        float f = 0.f;
        if (J8 < I8) f = expf(G[(size_t)(8 * I8 - 1) * D + jj] - G[(size_t)(8 * J8 + 7) * D + jj]);
        c.s[L.F + idx] = f;
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

// Two decay-masked products sharing X: out_p[t][s] = [X (*) Z_p]_{ts}, masked
// to s < t (strict) or s <= t, for all (t, s) of the chunk.  Work is split in
// (16-row, 8-column) tiles over the warps.
template <typename Tin, int D, int PASSES>
__device__ void masked_pair(const Chunk<Tin, D>& c, int X, int Z0, int Z1, size_t out0,
                            size_t out1, bool incl0, bool incl1) {
    const Lay& L = c.L;
    const int C = L.C, nb8 = L.nb8, nb16 = L.nb16;
    const int warp = threadIdx.x >> 5, nwarps = kThreads / 32;
    const int ntiles = nb16 * (nb16 + 1);  // sum over I16 of (2*I16 + 2)
    const float* s = c.s;
    for (int tile = warp; tile < ntiles; tile += nwarps) {
        // tile -> (I16, J8) with J8 in [0, 2*I16+1]
        int I16 = 0, rem = tile;
        while (rem >= 2 * I16 + 2) { rem -= 2 * I16 + 2; ++I16; }
        const int J8 = rem, t0 = 16 * I16, s0 = 8 * J8;
        const int rb0 = 2 * I16, rb1 = 2 * I16 + 1;
        float acc0[1][1][4], acc1[1][1][4];
        zero_acc(acc0);
        zero_acc(acc1);
        if (rb1 > J8) {  // rows strictly after column block J8: pivot at J8's end
            auto fa = [&](int r, int k) -> float {
                const int rb = r < 8 ? rb0 : rb1;
                if (rb <= J8) return 0.f;
                const int t = t0 + r;
                return opval(c, X, t, k) * s[L.X8F + (size_t)t * D + k] *
                       s[L.F + ((size_t)rb * nb8 + J8) * D + k];
            };
            warp_gemm<PASSES, 1, 1>(acc0, D, fa, [&](int k, int n) {
                return opval(c, Z0, s0 + n, k) * s[L.Z8F + (size_t)(s0 + n) * D + k];
            });
            warp_gemm<PASSES, 1, 1>(acc1, D, fa, [&](int k, int n) {
                return opval(c, Z1, s0 + n, k) * s[L.Z8F + (size_t)(s0 + n) * D + k];
            });
        }
        if (rb0 == J8 || rb1 == J8) {  // rows inside block J8: mid-block pivot
            auto fa = [&](int r, int k) -> float {
                const int rb = r < 8 ? rb0 : rb1;
                if (rb != J8) return 0.f;
                const int t = t0 + r;
                return opval(c, X, t, k) * s[L.XOF + (size_t)t * D + k];
            };
            warp_gemm<PASSES, 1, 1>(acc0, D, fa, [&](int k, int n) {
                return opval(c, Z0, s0 + n, k) * s[L.ZOF + (size_t)(s0 + n) * D + k];
            });
            warp_gemm<PASSES, 1, 1>(acc1, D, fa, [&](int k, int n) {
                return opval(c, Z1, s0 + n, k) * s[L.ZOF + (size_t)(s0 + n) * D + k];
            });
        }
        float* o0 = c.s + out0;
        float* o1 = c.s + out1;
        for_acc(acc0, [&](int r, int cc, float& v) {
            const int t = t0 + r, ss = s0 + cc;
            o0[(size_t)t * C + ss] = (incl0 ? ss <= t : ss < t) ? v : 0.f;
        });
        for_acc(acc1, [&](int r, int cc, float& v) {
            const int t = t0 + r, ss = s0 + cc;
            o1[(size_t)t * C + ss] = (incl1 ? ss <= t : ss < t) ? v : 0.f;
        });
    }
    // the strict upper part (tiles never visited) must read as zero
    for (int idx = threadIdx.x; idx < C * C; idx += kThreads) {
        const int t = idx / C, ss = idx % C;
        if ((ss >> 3) > 2 * (t >> 4) + 1) {
            c.s[out0 + idx] = 0.f;
            c.s[out1 + idx] = 0.f;
        }
    }
}

// ------------------------------------------------------------------ triangular solves

// T_II = (I + L_II)^{-1} for every 16 x 16 diagonal block of the unit lower
// triangular I + L (forward substitution, float32).
__device__ void compute_tii(float* s, const Lay& L, size_t Loff) {
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

// Solve (I + L) X = R in place (X holds R on entry), L strictly lower C x C.
// Each warp owns D/8 columns; the 16-row blocks are handled in order.
template <int D, int PASSES>
__device__ void fwd_solve(float* s, const Lay& L, size_t Loff, size_t Xoff) {
    constexpr int NT = D / 64;  // n8 tiles per warp: D/8 columns / 8
    const int C = L.C, c0 = (threadIdx.x >> 5) * (D / 8);
    float* X = s + Xoff;
    for (int I = 0; I < L.nb16; ++I) {
        float acc[1][NT][4];
        zero_acc(acc);
        if (I > 0)
            warp_gemm<PASSES, 1, NT>(
                acc, 16 * I, [&](int r, int k) { return s[Loff + (size_t)(16 * I + r) * C + k]; },
                [&](int k, int n) { return X[(size_t)k * D + c0 + n]; });
        for_acc(acc, [&](int r, int cc, float& v) {
            float& x = X[(size_t)(16 * I + r) * D + c0 + cc];
            x = x - v;
        });
        __syncwarp();
        float acc2[1][NT][4];
        zero_acc(acc2);
        warp_gemm<PASSES, 1, NT>(
            acc2, 16, [&](int r, int k) { return s[L.TII + ((size_t)I * 16 + r) * 16 + k]; },
            [&](int k, int n) { return X[(size_t)(16 * I + k) * D + c0 + n]; });
        __syncwarp();
        for_acc(acc2, [&](int r, int cc, float& v) { X[(size_t)(16 * I + r) * D + c0 + cc] = v; });
        __syncwarp();
    }
}

// Solve (I + L)^T X = R in place.
template <int D, int PASSES>
__device__ void bwd_solve(float* s, const Lay& L, size_t Loff, size_t Xoff) {
    constexpr int NT = D / 64;
    const int C = L.C, c0 = (threadIdx.x >> 5) * (D / 8);
    float* X = s + Xoff;
    for (int I = L.nb16 - 1; I >= 0; --I) {
        const int r1 = 16 * (I + 1);
        float acc[1][NT][4];
        zero_acc(acc);
        if (r1 < C)
            warp_gemm<PASSES, 1, NT>(
                acc, C - r1,
                [&](int r, int k) { return s[Loff + (size_t)(r1 + k) * C + 16 * I + r]; },
                [&](int k, int n) { return X[(size_t)(r1 + k) * D + c0 + n]; });
        for_acc(acc, [&](int r, int cc, float& v) {
            float& x = X[(size_t)(16 * I + r) * D + c0 + cc];
            x = x - v;
        });
        __syncwarp();
        float acc2[1][NT][4];
        zero_acc(acc2);
        warp_gemm<PASSES, 1, NT>(
            acc2, 16, [&](int r, int k) { return s[L.TII + ((size_t)I * 16 + k) * 16 + r]; },
            [&](int k, int n) { return X[(size_t)(16 * I + k) * D + c0 + n]; });
        __syncwarp();
        for_acc(acc2, [&](int r, int cc, float& v) { X[(size_t)(16 * I + r) * D + c0 + cc] = v; });
        __syncwarp();
    }
}

// ------------------------------------------------------------------ k_intra

template <typename Tin, int D, int PASSES>
__global__ void __launch_bounds__(kThreads) k_intra(KParams p) {
    constexpr int NT = 2;
    float* slot = p.scratch + (size_t)blockIdx.x * p.slot;
    const int nch = p.B * p.H * p.N;
    for (int chunk = blockIdx.x; chunk < nch; chunk += gridDim.x) {
        const Chunk<Tin, D> c = make_chunk<Tin, D>(p, chunk, slot);
        const Lay& L = c.L;
        const int C = L.C;
        float* s = c.s;
        prologue(c);
        masked_pair<Tin, D, PASSES>(c, OP_K, OP_A, OP_K, L.LA, L.LK, false, false);
        __syncthreads();
        compute_tii(s, L, L.LA);
        for (int idx = threadIdx.x; idx < C * D; idx += kThreads)
            s[L.W[0] + idx] = c.A(idx / D, idx % D) * s[L.EGB + idx];  // Ab
        __syncthreads();
        bwd_solve<D, PASSES>(s, L, L.LA, L.W[0]);  // Psi = T^T Ab
        __syncthreads();
        float* M = p.M + c.sbase;
        // M = diag(e^gbar) - Psi^T Kt
        cta_tiles<NT>(D, D,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, C,
                    [&](int r, int k) { return s[L.W[0] + (size_t)k * D + m0 + r]; },
                    [&](int k, int n) { return c.K(k, n0 + n) * s[L.EG + (size_t)k * D + n0 + n]; });
            },
            [&](int i, int j, float v) {
                const float d = (i == j) ? expf(s[L.G + (size_t)(C - 1) * D + i]) : 0.f;
                M[(size_t)i * D + j] = d - v;
            });
        // Phi = Kb - L_K^T Psi
        cta_tiles<NT>(C, D,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, C,
                    [&](int r, int k) { return s[L.LK + (size_t)k * C + m0 + r]; },
                    [&](int k, int n) { return s[L.W[0] + (size_t)k * D + n0 + n]; });
            },
            [&](int t, int j, float v) {
                s[L.W[1] + (size_t)t * D + j] = c.K(t, j) * s[L.EGB + (size_t)t * D + j] - v;
            });
        __syncthreads();
        float* Bn = p.Bn + c.sbase;
        // Bn = Phi^T U
        cta_tiles<NT>(D, D,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, C,
                    [&](int r, int k) { return s[L.W[1] + (size_t)k * D + m0 + r]; },
                    [&](int k, int n) { return c.U(k, n0 + n); });
            },
            [&](int i, int j, float v) { Bn[(size_t)i * D + j] = v; });
        __syncthreads();
    }
}

// ------------------------------------------------------------------ k_chain

// Sequential pass over chunks for one (b, h) and a slab of SLAB columns.
// Forward (REV = false): S_{n+1} = M_n S_n + Bn_n, records S_n.
// Reverse (REV = true):  G_n = M_n^T G_{n+1} + Bn_n, records G_{n+1}.
template <int D, int SLAB, int PASSES, bool REV>
__global__ void __launch_bounds__(kThreads) k_chain(const float* __restrict__ M,
                                                    const float* __restrict__ Bn,
                                                    const float* __restrict__ S_in,
                                                    float* __restrict__ S_rec,
                                                    float* __restrict__ S_out, int N) {
    constexpr int NT = SLAB / 8 < 4 ? SLAB / 8 : 4;
    __shared__ float buf[2][D * SLAB];
    constexpr int NSLAB = D / SLAB;
    const int bh = blockIdx.x / NSLAB, c0 = (blockIdx.x % NSLAB) * SLAB;
    const size_t DD = (size_t)D * D;
    for (int idx = threadIdx.x; idx < D * SLAB; idx += kThreads) {
        const int i = idx / SLAB, cc = idx % SLAB;
        buf[0][idx] = S_in ? S_in[bh * DD + (size_t)i * D + c0 + cc] : 0.f;
    }
    __syncthreads();
    int cur = 0;
    for (int step = 0; step < N; ++step) {
        const int n = REV ? N - 1 - step : step;
        const size_t off = ((size_t)bh * N + n) * DD;
        if (S_rec)
            for (int idx = threadIdx.x; idx < D * SLAB; idx += kThreads)
                S_rec[off + (size_t)(idx / SLAB) * D + c0 + idx % SLAB] = buf[cur][idx];
        const float* Mn = M + off;
        const float* Bb = Bn + off;
        const float* Sc = buf[cur];
        float* Sn = buf[cur ^ 1];
        cta_tiles<NT>(D, SLAB,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, D,
                    [&](int r, int k) {
                        return REV ? __ldg(Mn + (size_t)k * D + m0 + r)
                                   : __ldg(Mn + (size_t)(m0 + r) * D + k);
                    },
                    [&](int k, int n) { return Sc[k * SLAB + n0 + n]; });
            },
            [&](int i, int cc, float v) { Sn[i * SLAB + cc] = v + __ldg(Bb + (size_t)i * D + c0 + cc); });
        __syncthreads();
        cur ^= 1;
    }
    if (S_out)
        for (int idx = threadIdx.x; idx < D * SLAB; idx += kThreads)
            S_out[bh * DD + (size_t)(idx / SLAB) * D + c0 + idx % SLAB] = buf[cur][idx];
}

// ------------------------------------------------------------------ k_out

// Y = T (Kt S + L_K U) into scratch W[0] (needs LA, LK, TII).
template <typename Tin, int D, int PASSES>
__device__ void compute_Y(const Chunk<Tin, D>& c, const float* S, size_t Yoff) {
    constexpr int NT = 2;
    const Lay& L = c.L;
    const int C = L.C;
    float* s = c.s;
    cta_tiles<NT>(C, D,
        [&](float (&acc)[1][NT][4], int m0, int n0) {
            warp_gemm<PASSES, 1, NT>(acc, D,
                [&](int r, int k) { return c.K(m0 + r, k) * s[L.EG + (size_t)(m0 + r) * D + k]; },
                [&](int k, int n) { return __ldg(S + (size_t)k * D + n0 + n); });
            warp_gemm<PASSES, 1, NT>(acc, m0 + 16,
                [&](int r, int k) { return s[L.LK + (size_t)(m0 + r) * C + k]; },
                [&](int k, int n) { return c.U(k, n0 + n); });
        },
        [&](int t, int j, float v) { s[Yoff + (size_t)t * D + j] = v; });
    __syncthreads();
    fwd_solve<D, PASSES>(s, L, L.LA, Yoff);
    __syncthreads();
}

template <typename Tin, typename Tout, int D, int PASSES>
__global__ void __launch_bounds__(kThreads) k_out(KParams p) {
    constexpr int NT = 2;
    float* slot = p.scratch + (size_t)blockIdx.x * p.slot;
    const int nch = p.B * p.H * p.N;
    for (int chunk = blockIdx.x; chunk < nch; chunk += gridDim.x) {
        const Chunk<Tin, D> c = make_chunk<Tin, D>(p, chunk, slot);
        const Lay& L = c.L;
        const int C = L.C;
        float* s = c.s;
        prologue(c);
        masked_pair<Tin, D, PASSES>(c, OP_K, OP_A, OP_K, L.LA, L.LK, false, false);
        masked_pair<Tin, D, PASSES>(c, OP_Q, OP_K, OP_A, L.MQK, L.MQA, true, true);
        __syncthreads();
        compute_tii(s, L, L.LA);
        __syncthreads();
        const float* S = p.S_chunks + c.sbase;
        compute_Y<Tin, D, PASSES>(c, S, L.W[0]);
        Tout* o = (Tout*)p.o;
        cta_tiles<NT>(C, D,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, D,
                    [&](int r, int k) { return c.Qh(m0 + r, k) * s[L.EG + (size_t)(m0 + r) * D + k]; },
                    [&](int k, int n) { return __ldg(S + (size_t)k * D + n0 + n); });
                warp_gemm<PASSES, 1, NT>(acc, m0 + 16,
                    [&](int r, int k) { return s[L.MQK + (size_t)(m0 + r) * C + k]; },
                    [&](int k, int n) { return c.U(k, n0 + n); });
                warp_gemm<PASSES, 1, NT>(acc, m0 + 16,
                    [&](int r, int k) { return -s[L.MQA + (size_t)(m0 + r) * C + k]; },
                    [&](int k, int n) { return s[L.W[0] + (size_t)k * D + n0 + n]; });
            },
            [&](int t, int j, float v) { stf(o + c.base + t * c.rs + j, v); });
        __syncthreads();
    }
}

// ------------------------------------------------------------------ k_bprep

template <typename Tin, int D, int PASSES>
__global__ void __launch_bounds__(kThreads) k_bprep(KParams p) {
    constexpr int NT = 2;
    float* slot = p.scratch + (size_t)blockIdx.x * p.slot;
    const int nch = p.B * p.H * p.N;
    for (int chunk = blockIdx.x; chunk < nch; chunk += gridDim.x) {
        const Chunk<Tin, D> c = make_chunk<Tin, D>(p, chunk, slot);
        const Lay& L = c.L;
        const int C = L.C;
        float* s = c.s;
        prologue(c);
        masked_pair<Tin, D, PASSES>(c, OP_K, OP_A, OP_K, L.LA, L.LK, false, false);
        masked_pair<Tin, D, PASSES>(c, OP_Q, OP_K, OP_A, L.MQK, L.MQA, true, true);
        __syncthreads();
        compute_tii(s, L, L.LA);
        // Z0 = M_QA^T dO
        cta_tiles<NT>(C, D,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, C - m0,
                    [&](int r, int k) { return s[L.MQA + (size_t)(m0 + k) * C + m0 + r]; },
                    [&](int k, int n) { return c.dOv(m0 + k, n0 + n); });
            },
            [&](int t, int j, float v) { s[L.W[0] + (size_t)t * D + j] = v; });
        __syncthreads();
        bwd_solve<D, PASSES>(s, L, L.LA, L.W[0]);  // Xi = T^T Z0
        __syncthreads();
        float* Bp = p.Bn + c.sbase;
        // B' = Qt^T dO - Kt^T Xi
        cta_tiles<NT>(D, D,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, C,
                    [&](int r, int k) { return c.Qh(k, m0 + r) * s[L.EG + (size_t)k * D + m0 + r]; },
                    [&](int k, int n) { return c.dOv(k, n0 + n); });
                warp_gemm<PASSES, 1, NT>(acc, C,
                    [&](int r, int k) { return -c.K(k, m0 + r) * s[L.EG + (size_t)k * D + m0 + r]; },
                    [&](int k, int n) { return s[L.W[0] + (size_t)k * D + n0 + n]; });
            },
            [&](int i, int j, float v) { Bp[(size_t)i * D + j] = v; });
        __syncthreads();
    }
}

// ------------------------------------------------------------------ k_bwd

// Gradient through a decay-masked product, X side:
//   out[t][j] = sum_{s} Gm[t][s] Z_sj exp(Gam_tj - Gam_sj)   (Gm already masked)
// Z side:
//   out[s][j] = sum_{t} Gm[t][s] X_tj exp(Gam_tj - Gam_sj)
// Each 16-row output tile walks the 8-token blocks of the contraction index;
// every block is one k8 MMA step whose result is scaled by the block-pair factor.
template <typename Tin, int D, int PASSES, bool XSIDE, class EPI>
__device__ void decayed_grad(const Chunk<Tin, D>& c, size_t G0, int op0, size_t G1, int op1,
                             const EPI& epi) {
    constexpr int NT = 2;
    const Lay& L = c.L;
    const int C = L.C, nb8 = L.nb8;
    const float* s = c.s;
    const int lane = threadIdx.x & 31, gq = lane >> 2, cq = lane & 3;
    const int warp = threadIdx.x >> 5, nwarps = kThreads / 32;
    const int tn = D / (8 * NT), tiles = L.nb16 * tn;
    for (int tile = warp; tile < tiles; tile += nwarps) {
        const int m0 = (tile / tn) * 16, n0 = (tile % tn) * 8 * NT;
        const int rb0 = m0 / 8, rb1 = rb0 + 1;  // 8-blocks of the two row halves
        float off[1][NT][4], dia[1][NT][4];
        zero_acc(off);
        zero_acc(dia);
        for (int B8 = 0; B8 < nb8; ++B8) {
            // relation of each row half to block B8: 1 = off-diagonal, 2 = diagonal, 0 = none
            int rel0, rel1;
            if (XSIDE) {
                rel0 = B8 < rb0 ? 1 : (B8 == rb0 ? 2 : 0);
                rel1 = B8 < rb1 ? 1 : (B8 == rb1 ? 2 : 0);
            } else {
                rel0 = B8 > rb0 ? 1 : (B8 == rb0 ? 2 : 0);
                rel1 = B8 > rb1 ? 1 : (B8 == rb1 ? 2 : 0);
            }
            if (rel0 == 0 && rel1 == 0) continue;
            const int k0 = 8 * B8;
            for (int kind = 1; kind <= 2; ++kind) {
                if (rel0 != kind && rel1 != kind) continue;
                // A(r, k): gradient matrix entry; rows of the other kind are zero
                auto gm = [&](size_t Goff, int r, int k) -> float {
                    const int rel = r < 8 ? rel0 : rel1;
                    if (rel != kind) return 0.f;
                    return XSIDE ? s[Goff + (size_t)(m0 + r) * C + k0 + k]
                                 : s[Goff + (size_t)(k0 + k) * C + m0 + r];
                };
                // B(k, n): operand row (k0 + k), scaled by its pivot factor
                const size_t fac = XSIDE ? (kind == 1 ? L.Z8F : L.ZOF) : (kind == 1 ? L.X8F : L.XOF);
                float tmp[1][NT][4];
                zero_acc(tmp);
                warp_gemm<PASSES, 1, NT>(tmp, 8, [&](int r, int k) { return gm(G0, r, k); },
                    [&](int k, int n) {
                        return opval(c, op0, k0 + k, n0 + n) * s[fac + (size_t)(k0 + k) * D + n0 + n];
                    });
                warp_gemm<PASSES, 1, NT>(tmp, 8, [&](int r, int k) { return gm(G1, r, k); },
                    [&](int k, int n) {
                        return opval(c, op1, k0 + k, n0 + n) * s[fac + (size_t)(k0 + k) * D + n0 + n];
                    });
                if (kind == 2) {
#pragma unroll
                    for (int n = 0; n < NT; ++n)
#pragma unroll
                        for (int i = 0; i < 4; ++i) dia[0][n][i] += tmp[0][n][i];
                } else {
                    // off-diagonal block pair factor F[row block][B8] (X side) or F[B8][row block]
#pragma unroll
                    for (int n = 0; n < NT; ++n)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int rb = i < 2 ? rb0 : rb1;
                            const int col = n0 + 8 * n + 2 * cq + (i & 1);
                            const size_t fi = XSIDE ? ((size_t)rb * nb8 + B8) : ((size_t)B8 * nb8 + rb);
                            const float f = (i < 2 ? rel0 : rel1) == 1 ? s[L.F + fi * D + col] : 0.f;
                            off[0][n][i] += f * tmp[0][n][i];
                        }
                }
            }
        }
        // output-side pivot factors
        const size_t fo = XSIDE ? L.X8F : L.Z8F, fd = XSIDE ? L.XOF : L.ZOF;
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = m0 + gq + (i < 2 ? 0 : 8);
                const int col = n0 + 8 * n + 2 * cq + (i & 1);
                const size_t x = (size_t)row * D + col;
                epi(row, col, s[fo + x] * off[0][n][i] + s[fd + x] * dia[0][n][i]);
            }
    }
}

template <typename Tin, int D, int PASSES>
__global__ void __launch_bounds__(kThreads) k_bwd(KParams p) {
    constexpr int NT = 2;
    float* slot = p.scratch + (size_t)blockIdx.x * p.slot;
    const int nch = p.B * p.H * p.N;
    for (int chunk = blockIdx.x; chunk < nch; chunk += gridDim.x) {
        const Chunk<Tin, D> c = make_chunk<Tin, D>(p, chunk, slot);
        const Lay& L = c.L;
        const int C = L.C;
        float* s = c.s;
        const float* S = p.S_chunks + c.sbase;
        const float* dS = p.dS_chunks + c.sbase;
        const size_t Y = L.W[0], dR = L.W[1], dK = L.W[2], dQh = L.W[3], dA = L.W[4],
                     dU = L.W[5], dGam = L.W[6], XB = L.W[7];
        prologue(c);
        masked_pair<Tin, D, PASSES>(c, OP_K, OP_A, OP_K, L.LA, L.LK, false, false);
        masked_pair<Tin, D, PASSES>(c, OP_Q, OP_K, OP_A, L.MQK, L.MQA, true, true);
        __syncthreads();
        compute_tii(s, L, L.LA);
        __syncthreads();
        compute_Y<Tin, D, PASSES>(c, S, Y);
        // dY = -M_QA^T dO - Ab dS'
        cta_tiles<NT>(C, D,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, C - m0,
                    [&](int r, int k) { return s[L.MQA + (size_t)(m0 + k) * C + m0 + r]; },
                    [&](int k, int n) { return c.dOv(m0 + k, n0 + n); });
                warp_gemm<PASSES, 1, NT>(acc, D,
                    [&](int r, int k) { return c.A(m0 + r, k) * s[L.EGB + (size_t)(m0 + r) * D + k]; },
                    [&](int k, int n) { return __ldg(dS + (size_t)k * D + n0 + n); });
            },
            [&](int t, int j, float v) { s[dR + (size_t)t * D + j] = -v; });
        __syncthreads();
        bwd_solve<D, PASSES>(s, L, L.LA, dR);  // dR = T^T dY
        __syncthreads();
        // dQt = dO S^T  -> dQh = dQt e^Gam ; dGam = dQt * Qt
        cta_tiles<NT>(C, D,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, D, [&](int r, int k) { return c.dOv(m0 + r, k); },
                    [&](int k, int n) { return __ldg(S + (size_t)(n0 + n) * D + k); });
            },
            [&](int t, int j, float v) {
                const size_t x = (size_t)t * D + j;
                s[dQh + x] = v * s[L.EG + x];
                s[dGam + x] = v * c.Qh(t, j) * s[L.EG + x];
            });
        __syncthreads();
        // dKt = dR S^T -> dK = dKt e^Gam ; dGam += dKt * Kt
        cta_tiles<NT>(C, D,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, D, [&](int r, int k) { return s[dR + (size_t)(m0 + r) * D + k]; },
                    [&](int k, int n) { return __ldg(S + (size_t)(n0 + n) * D + k); });
            },
            [&](int t, int j, float v) {
                const size_t x = (size_t)t * D + j;
                s[dK + x] = v * s[L.EG + x];
                s[dGam + x] += v * c.K(t, j) * s[L.EG + x];
            });
        __syncthreads();
        // dKb = U dS'^T -> dK += dKb e^{gbar-Gam} ; dGam -= dKb*Kb ; XB = dKb*Kb
        cta_tiles<NT>(C, D,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, D, [&](int r, int k) { return c.U(m0 + r, k); },
                    [&](int k, int n) { return __ldg(dS + (size_t)(n0 + n) * D + k); });
            },
            [&](int t, int j, float v) {
                const size_t x = (size_t)t * D + j;
                const float kb = c.K(t, j) * s[L.EGB + x];
                s[dK + x] += v * s[L.EGB + x];
                s[dGam + x] -= v * kb;
                s[XB + x] = v * kb;
            });
        __syncthreads();
        // dAb = -Y dS'^T -> dA = dAb e^{gbar-Gam} ; dGam -= dAb*Ab ; XB += dAb*Ab
        cta_tiles<NT>(C, D,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, D, [&](int r, int k) { return -s[Y + (size_t)(m0 + r) * D + k]; },
                    [&](int k, int n) { return __ldg(dS + (size_t)(n0 + n) * D + k); });
            },
            [&](int t, int j, float v) {
                const size_t x = (size_t)t * D + j;
                const float ab = c.A(t, j) * s[L.EGB + x];
                s[dA + x] = v * s[L.EGB + x];
                s[dGam + x] -= v * ab;
                s[XB + x] += v * ab;
            });
        __syncthreads();
        // dU = M_QK^T dO + L_K^T dR + Kb dS'
        cta_tiles<NT>(C, D,
            [&](float (&acc)[1][NT][4], int m0, int n0) {
                warp_gemm<PASSES, 1, NT>(acc, C - m0,
                    [&](int r, int k) { return s[L.MQK + (size_t)(m0 + k) * C + m0 + r]; },
                    [&](int k, int n) { return c.dOv(m0 + k, n0 + n); });
                warp_gemm<PASSES, 1, NT>(acc, C - m0,
                    [&](int r, int k) { return s[L.LK + (size_t)(m0 + k) * C + m0 + r]; },
                    [&](int k, int n) { return s[dR + (size_t)(m0 + k) * D + n0 + n]; });
                warp_gemm<PASSES, 1, NT>(acc, D,
                    [&](int r, int k) { return c.K(m0 + r, k) * s[L.EGB + (size_t)(m0 + r) * D + k]; },
                    [&](int k, int n) { return __ldg(dS + (size_t)k * D + n0 + n); });
            },
            [&](int t, int j, float v) { s[dU + (size_t)t * D + j] = v; });
        __syncthreads();
        // gradients of the masked products (overwrite them): dL_A = -strict(dR Y^T),
        // dL_K = strict(dR U^T), dM_QK = incl(dO U^T), dM_QA = -incl(dO Y^T)
        for (int which = 0; which < 4; ++which) {
            const size_t out = which == 0 ? L.LA : which == 1 ? L.LK : which == 2 ? L.MQK : L.MQA;
            const bool incl = which >= 2;
            const float sg = (which == 0 || which == 3) ? -1.f : 1.f;
            cta_tiles<NT>(C, C,
                [&](float (&acc)[1][NT][4], int m0, int n0) {
                    if (n0 > m0 + 15) return;
                    warp_gemm<PASSES, 1, NT>(acc, D,
                        [&](int r, int k) {
                            return which < 2 ? s[dR + (size_t)(m0 + r) * D + k] : c.dOv(m0 + r, k);
                        },
                        [&](int k, int n) {
                            return (which == 0 || which == 3) ? s[Y + (size_t)(n0 + n) * D + k]
                                                              : c.U(n0 + n, k);
                        });
                },
                [&](int t, int ss, float v) {
                    const bool keep = incl ? ss <= t : ss < t;
                    s[out + (size_t)t * C + ss] = keep ? sg * v : 0.f;
                });
        }
        __syncthreads();
        // X side: dK += dL_A (*) A + dL_K (*) K ; dQh += dM_QK (*) K + dM_QA (*) A ; dGam += X * dX
        decayed_grad<Tin, D, PASSES, true>(c, L.LA, OP_A, L.LK, OP_K, [&](int t, int j, float v) {
            const size_t x = (size_t)t * D + j;
            s[dK + x] += v;
            s[dGam + x] += c.K(t, j) * v;
        });
        decayed_grad<Tin, D, PASSES, true>(c, L.MQK, OP_K, L.MQA, OP_A, [&](int t, int j, float v) {
            const size_t x = (size_t)t * D + j;
            s[dQh + x] += v;
            s[dGam + x] += c.Qh(t, j) * v;
        });
        __syncthreads();
        // Z side: dA += dL_A^T (*) K + dM_QA^T (*) Qh ; dK += dL_K^T (*) K + dM_QK^T (*) Qh ; dGam -= Z * dZ
        decayed_grad<Tin, D, PASSES, false>(c, L.LA, OP_K, L.MQA, OP_Q, [&](int t, int j, float v) {
            const size_t x = (size_t)t * D + j;
            s[dA + x] += v;
            s[dGam + x] -= c.A(t, j) * v;
        });
        __syncthreads();
        decayed_grad<Tin, D, PASSES, false>(c, L.LK, OP_K, L.MQK, OP_Q, [&](int t, int j, float v) {
            const size_t x = (size_t)t * D + j;
            s[dK + x] += v;
            s[dGam + x] -= c.K(t, j) * v;
        });
        __syncthreads();
        // dgbar = e^gbar rowsum(S * dS') + sum_t XB ; dg_t = sum_{t'>=t} dGam_t' + dgbar
        Tin* gq = (Tin*)p.dq; Tin* gk = (Tin*)p.dk; Tin* gv = (Tin*)p.dv; Tin* gg = (Tin*)p.dg;
        Tin* ge = (Tin*)p.de; Tin* gw = (Tin*)p.dw; Tin* ggm = (Tin*)p.dgamma;
        if (threadIdx.x < D) {
            const int j = threadIdx.x;
            float acc = 0.f;
            for (int cc = 0; cc < D; ++cc) acc += __ldg(S + (size_t)j * D + cc) * __ldg(dS + (size_t)j * D + cc);
            float dgb = acc * expf(s[L.G + (size_t)(C - 1) * D + j]);
            for (int t = 0; t < C; ++t) dgb += s[XB + (size_t)t * D + j];
            float run = dgb;
            for (int t = C - 1; t >= 0; --t) {
                run += s[dGam + (size_t)t * D + j];
                const float graw = ldf(c.g + c.base + t * c.rs + j);
                stf(gg + c.base + t * c.rs + j, graw >= kLogDecayMin ? run : 0.f);
            }
        }
        for (int idx = threadIdx.x; idx < C * D; idx += kThreads) {
            const int t = idx / D, j = idx % D;
            const size_t gi = c.base + t * c.rs + j;
            const float qv = ldf(c.q + gi), gmv = ldf(c.gm + gi), kv = ldf(c.k + gi),
                        ev = ldf(c.e + gi), vv = ldf(c.v + gi), wv = ldf(c.w + gi);
            const float dqh = s[dQh + idx], da = s[dA + idx], du = s[dU + idx];
            stf(gq + gi, dqh * gmv);
            stf(ggm + gi, dqh * qv);
            stf(ge + gi, da * kv);
            stf(gk + gi, s[dK + idx] + da * ev);
            stf(gw + gi, du * vv);
            stf(gv + gi, du * wv);
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ host side

static int num_slots(int nch) { return nch < kMaxSlots ? nch : kMaxSlots; }

static size_t slot_floats(int C, int D) { return make_lay(C, D).total; }

size_t chunk_fwd_ws_bytes(int B, int T, int H, int D, int C, bool have_states) {
    const size_t nch = (size_t)B * H * (T / C), DD = (size_t)D * D;
    size_t f = 2 * nch * DD;               // M, Bn
    if (!have_states) f += nch * DD;       // chunk-start states
    f += (size_t)num_slots((int)nch) * slot_floats(C, D);
    return f * sizeof(float);
}

size_t chunk_bwd_ws_bytes(int B, int T, int H, int D, int C, bool have_states) {
    const size_t nch = (size_t)B * H * (T / C), DD = (size_t)D * D;
    size_t f = 3 * nch * DD;               // M, Bn / B', dS at chunk ends
    if (!have_states) f += nch * DD;
    f += (size_t)num_slots((int)nch) * slot_floats(C, D);
    return f * sizeof(float);
}

template <int D, int PASSES, bool REV>
static cudaError_t launch_chain(int BH, int N, const float* M, const float* Bn, const float* S_in,
                                float* S_rec, float* S_out, cudaStream_t st) {
    // column slabs: enough CTAs to cover the GPU when B*H is small
    if (BH >= 64) {
        constexpr int SL = 32;
        MUIR_TIMED(REV ? "k_chain_rev" : "k_chain", st, k_chain<D, SL, PASSES, REV><<<BH * (D / SL), kThreads, 0, st>>>(M, Bn, S_in, S_rec, S_out, N));
    } else {
        constexpr int SL = 16;
        MUIR_TIMED(REV ? "k_chain_rev" : "k_chain", st, k_chain<D, SL, PASSES, REV><<<BH * (D / SL), kThreads, 0, st>>>(M, Bn, S_in, S_rec, S_out, N));
    }
    return cudaGetLastError();
}

template <typename Tin, int D, int PASSES>
static cudaError_t fwd_impl(const ChunkProblem& P, const float* S0, void* o, float* S_final,
                            float* S_chunks, void* ws, cudaStream_t st) {
    const int nch = P.B * P.H * P.N, BH = P.B * P.H;
    const size_t DD = (size_t)D * D;
    float* f = static_cast<float*>(ws);
    KParams kp = {};
    kp.B = P.B; kp.T = P.T; kp.H = P.H; kp.C = P.C; kp.N = P.N;
    kp.q = P.q; kp.k = P.k; kp.v = P.v; kp.g = P.g; kp.e = P.e; kp.w = P.w; kp.gamma = P.gamma;
    kp.M = f; f += nch * DD;
    kp.Bn = f; f += nch * DD;
    float* Sc = S_chunks;
    if (!Sc) { Sc = f; f += nch * DD; }
    kp.scratch = f;
    kp.slot = slot_floats(P.C, D);
    kp.S_chunks = Sc;
    kp.o = o;
    const int grid = num_slots(nch);
    MUIR_TIMED("k_intra", st, k_intra<Tin, D, PASSES><<<grid, kThreads, 0, st>>>(kp));
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    err = launch_chain<D, PASSES, false>(BH, P.N, kp.M, kp.Bn, S0, Sc, S_final, st);
    if (err != cudaSuccess) return err;
    if (P.out_bf16)
        MUIR_TIMED("k_out", st, k_out<Tin, __nv_bfloat16, D, PASSES><<<grid, kThreads, 0, st>>>(kp));
    else
        MUIR_TIMED("k_out", st, k_out<Tin, float, D, PASSES><<<grid, kThreads, 0, st>>>(kp));
    return cudaGetLastError();
}

template <typename Tin, int D, int PASSES>
static cudaError_t bwd_impl(const ChunkProblem& P, const float* S0, const float* S_chunks,
                            const void* dO, const float* dS_final, void* dq, void* dk, void* dv,
                            void* dg, void* de, void* dw, void* dgamma, float* dS0, void* ws,
                            cudaStream_t st) {
    const int nch = P.B * P.H * P.N, BH = P.B * P.H;
    const size_t DD = (size_t)D * D;
    float* f = static_cast<float*>(ws);
    KParams kp = {};
    kp.B = P.B; kp.T = P.T; kp.H = P.H; kp.C = P.C; kp.N = P.N;
    kp.q = P.q; kp.k = P.k; kp.v = P.v; kp.g = P.g; kp.e = P.e; kp.w = P.w; kp.gamma = P.gamma;
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
    const int grid = num_slots(nch);
    MUIR_TIMED("k_intra", st, k_intra<Tin, D, PASSES><<<grid, kThreads, 0, st>>>(kp));
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (recompute) {
        err = launch_chain<D, PASSES, false>(BH, P.N, kp.M, kp.Bn, S0, Sc, nullptr, st);
        if (err != cudaSuccess) return err;
    }
    MUIR_TIMED("k_bprep", st, k_bprep<Tin, D, PASSES><<<grid, kThreads, 0, st>>>(kp));
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    err = launch_chain<D, PASSES, true>(BH, P.N, kp.M, kp.Bn, dS_final, dSc, dS0, st);
    if (err != cudaSuccess) return err;
    MUIR_TIMED("k_bwd", st, k_bwd<Tin, D, PASSES><<<grid, kThreads, 0, st>>>(kp));
    return cudaGetLastError();
}

cudaError_t run_chunk_fwd(const ChunkProblem& P, const float* S0, void* o, float* S_final,
                          float* S_chunks, void* ws, size_t, cudaStream_t st) {
    if (P.in_bf16) {
        if (P.D == 128) return fwd_impl<__nv_bfloat16, 128, 1>(P, S0, o, S_final, S_chunks, ws, st);
        return fwd_impl<__nv_bfloat16, 64, 1>(P, S0, o, S_final, S_chunks, ws, st);
    }
    if (P.D == 128) return fwd_impl<float, 128, 3>(P, S0, o, S_final, S_chunks, ws, st);
    return fwd_impl<float, 64, 3>(P, S0, o, S_final, S_chunks, ws, st);
}

cudaError_t run_chunk_bwd(const ChunkProblem& P, const float* S0, const float* S_chunks,
                          const void* dO, const float* dS_final, void* dq, void* dk, void* dv,
                          void* dg, void* de, void* dw, void* dgamma, float* dS0, void* ws,
                          size_t, cudaStream_t st) {
#define MUIR_BWD_ARGS P, S0, S_chunks, dO, dS_final, dq, dk, dv, dg, de, dw, dgamma, dS0, ws, st
    if (P.in_bf16) {
        if (P.D == 128) return bwd_impl<__nv_bfloat16, 128, 1>(MUIR_BWD_ARGS);
        return bwd_impl<__nv_bfloat16, 64, 1>(MUIR_BWD_ARGS);
    }
    if (P.D == 128) return bwd_impl<float, 128, 3>(MUIR_BWD_ARGS);
    return bwd_impl<float, 64, 3>(MUIR_BWD_ARGS);
#undef MUIR_BWD_ARGS
}

}  // namespace muir

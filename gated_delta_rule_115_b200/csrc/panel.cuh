// panel.cuh -- decay-masked products and the gradients through them on the
// 5th-generation tensor cores, for chunks of at most 128 tokens with
// single-pass TF32 operands (bf16 inputs).  Included inside namespace muir
// after staged.cuh, whose header defines Lc, Rc, Bt and the pivot factors.
//
// With 8-token blocks, token s in block J and token t in a later block I:
//   exp(Gam_t - Gam_s) = [x8f_t F[I][J]] z8f_s,   F[I][J] = exp(sum_{J<K<I} Bt[K]),
// every factor <= 1.  The factor F joins the operand that runs over the long
// side, so each 8-token block gives ONE product with a fixed pivot:
//   masked product   out[t][s], s in J :  sum_c (Xx_tc F[I(t)][J]_c) Zz_sc        t in later blocks
//   X-side gradient  out[t][c], t in I :  x8f_tc sum_{s < 8I} G[t][s] (Zz_sc F[I][J(s)]_c)
//   Z-side gradient  out[s][c], s in J :  z8f_sc sum_{t >= 8J+8} G[t][s] (Xx_tc F[I(t)][J]_c)
// with Xx = X x8f and Zz = Z z8f (float32, per chunk).  Pairs inside one block
// use the mid-block pivot and run on the CUDA cores.
//
// One block's product is a chain of tcgen05.mma (M = 128, N = 16 or 32, K = 8)
// into the TMEM columns that start at the block's first token.  Columns past
// the block's 8 receive throw-away values that the next block's chain, issued
// later, overwrites (its first MMA does not accumulate), so the per-block
// accumulators tile the columns; the last block of a sweep writes no
// throw-away columns that anything reads.
#pragma once

// (included inside namespace muir)

constexpr int kPanelA = 32 * 4096;      // A operand: up to 32 K blocks of 128 rows x 8 (fp32)
constexpr int kPanelB = 30 * 1024;      // B operand
constexpr int kPanelBt = 16 * 128 * 4;  // block totals Bt of the chunk
constexpr int kPanelF = 16 * 128 * 4;   // F factors of one panel step
constexpr uint32_t kDiagCol = 256;      // TMEM column of the in-block gradient products
constexpr int kPairA = 16 * 4096;       // A region of the masked-pair panels (64 KB)

// Shared memory of the gradient panels (k_bwd) and of the masked-pair panels.
__host__ __device__ constexpr int panel_smem_bytes() { return kPanelA + kPanelB + kPanelBt + kPanelF; }
__host__ __device__ constexpr int pair_smem_bytes() { return kPairA + 16 * 512 + kPanelBt + kPanelF; }

// Shared-memory stores and loads by address; the stores carry no compiler
// memory barrier, so global loads around them can be scheduled freely.
__device__ __forceinline__ void sts128(uint32_t a, float4 v) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w));
}
__device__ __forceinline__ float4 lds128(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}

// Four consecutive channels j.. of operand OP (K, Qh or A) at token t.
template <int OP, typename Tin, int D>
__device__ __forceinline__ void opload4(const Chunk<Tin, D>& c, int t, int j, float* v) {
    const size_t g = c.base + (size_t)t * c.rs + j;
    ld4in(c.k + g, v);
    if (OP == OP_A) {
        float e[4];
        ld4in(c.e + g, e);
        for (int u = 0; u < 4; ++u) v[u] *= e[u];
    } else if (OP == OP_Q) {
        float q[4], m[4];
        ld4in(c.q + g, q);
        ld4in(c.gm + g, m);
        for (int u = 0; u < 4; ++u) v[u] = q[u] * m[u];
    }
}

// Xx = X x8f (float32) for X in {K, Qh}; Zz = tf32(Z z8f) for Z in {A, K}.
template <typename Tin, int D>
__device__ void panel_prep(const Chunk<Tin, D>& c, bool with_q) {
    const Lay& L = c.L;
    const int n4 = L.C * D / 4;
    for (int idx = threadIdx.x; idx < n4; idx += kThreads) {
        const int t = idx / (D / 4), j = 4 * (idx % (D / 4));
        const size_t g = c.base + (size_t)t * c.rs + j, x = (size_t)t * D + j;
        float k4[4], e4[4], q4[4], m4[4], lc[4], rc[4];
        ld4in(c.k + g, k4);
        ld4in(c.e + g, e4);
        if (with_q) {
            ld4in(c.q + g, q4);
            ld4in(c.gm + g, m4);
        }
        ld4(c.s + L.LC + x, lc);
        ld4(c.s + L.RC + x, rc);
        float4 xk, xq, za, zk;
        float* pxk = &xk.x; float* pxq = &xq.x; float* pza = &za.x; float* pzk = &zk.x;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float ex = fexp<Tin>(lc[u]), ez = fexp<Tin>(rc[u]);
            pxk[u] = k4[u] * ex;
            pxq[u] = with_q ? m4[u] * q4[u] * ex : 0.f;
            pza[u] = tc::tf32_rn(e4[u] * k4[u] * ez);
            pzk[u] = tc::tf32_rn(k4[u] * ez);
        }
        *reinterpret_cast<float4*>(c.s + L.PXK + x) = xk;
        if (with_q) *reinterpret_cast<float4*>(c.s + L.PXQ + x) = xq;
        *reinterpret_cast<float4*>(c.s + L.PZA + x) = za;
        *reinterpret_cast<float4*>(c.s + L.PZK + x) = zk;
    }
    __syncthreads();
}

__device__ __forceinline__ size_t panel_xx(const Lay& L, int op) { return op == OP_Q ? L.PXQ : L.PXK; }
__device__ __forceinline__ size_t panel_zz(const Lay& L, int op) { return op == OP_A ? L.PZA : L.PZK; }

struct PanelSmem {
    unsigned char* A;
    unsigned char* B;
    float* bt;  // [nb8][D]
    float* f;   // [nb8][D]
};

// Carve the panel buffers (A region of abytes, B region of bbytes) and copy
// the chunk's block totals Bt (all threads).
template <int D>
__device__ __forceinline__ PanelSmem panel_smem(const float* s, const Lay& L, unsigned char* sbuf,
                                                int abytes = kPanelA, int bbytes = kPanelB) {
    PanelSmem m;
    m.A = sbuf;
    m.B = sbuf + abytes;
    m.bt = reinterpret_cast<float*>(sbuf + abytes + bbytes);
    m.f = reinterpret_cast<float*>(sbuf + abytes + bbytes + kPanelBt);
    for (int i = threadIdx.x; i < L.nb8 * D / 4; i += kThreads)
        reinterpret_cast<float4*>(m.bt)[i] = *reinterpret_cast<const float4*>(s + L.BT + 4 * (size_t)i);
    __syncthreads();
    return m;
}

// F[I][J] = exp(sum_{J<K<I} Bt[K]) into f[I][.] for I in (J, nb8) (DOWN = false),
// or into f[J][.] for J in [0, I) with I fixed (DOWN = true).  Threads j < D.
template <typename Tin, int D, bool DOWN>
__device__ __forceinline__ void panel_ftab(const PanelSmem& m, int nb8, int fix) {
    const int j = threadIdx.x;
    if (j >= D) return;
    float sum = 0.f;
    if (!DOWN) {
        for (int I = fix + 1; I < nb8; ++I) {
            if (I > fix + 1) sum += m.bt[(I - 1) * D + j];
            m.f[I * D + j] = fexp<Tin>(sum);
        }
    } else {
        for (int J = fix - 1; J >= 0; --J) {
            m.f[J * D + j] = fexp<Tin>(sum);
            sum += m.bt[J * D + j];
        }
    }
}

// v (4 floats at shared address a) <- tf32(v * f) for f the four floats at fa.
__device__ __forceinline__ void scale_at(uint32_t a, uint32_t fa) {
    float4 v = lds128(a);
    const float4 f = lds128(fa);
    v.x = tc::tf32_rn(v.x * f.x);
    v.y = tc::tf32_rn(v.y * f.y);
    v.z = tc::tf32_rn(v.z * f.z);
    v.w = tc::tf32_rn(v.w * f.w);
    sts128(a, v);
}

// Publish the step's shared-memory operands to the tensor core, let one thread
// issue the chain, wait for it (bounded).  All threads call.
template <class ISSUE>
__device__ __forceinline__ void panel_run(tc::State& st, const ISSUE& issue) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        issue();
        tc::commit(st);
    }
    tc::wait_mma(st);
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[j]);
}

__device__ __forceinline__ void panel_end() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
}

// Thread roles for K-major operands (rows = tokens): r8 = row inside an
// 8-row core group, q4 = channel quad; one core matrix (8 rows of one quad) is
// one 128-byte store phase.  par splits the row blocks when D = 64.
template <int D>
struct KRole {
    int r8, q4, par;
    __device__ KRole() {
        constexpr int NQ = D / 4;
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        r8 = lane & 7;
        q4 = (warp * 4 + (lane >> 3)) % NQ;
        par = (warp * 4 + (lane >> 3)) / NQ;
    }
};

// Thread roles for MN-major operands (rows = channels): q4 = channel quad,
// kk = token inside the 8-token K block; eight consecutive quads of one kk fill
// one 128-byte shared-memory row (one store phase).
template <int D>
struct MnRole {
    int q4, kk, par;
    __device__ MnRole() {
        constexpr int QW = D / 32;  // warps per half of the 8 kk values
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        q4 = (lane & 7) + 8 * (warp % QW);
        kk = (lane >> 3) + 4 * ((warp / QW) & 1);
        par = warp / (2 * QW);
    }
};

// Operand with the mid-block pivot m = 8b + 3 of its token's block:
//   XSIDE: OP_tc exp(Lc_t - Lc_m)     otherwise: OP_tc exp(Lc_m - Lc_t)
// rounded to TF32, stored K-major (rows = tokens, K blocks kstride bytes apart).
template <int OP, bool XSIDE, typename Tin, int D>
__device__ void form_mid_k(const Chunk<Tin, D>& c, unsigned char* dst, int kstride) {
    constexpr int NPAR = kThreads / (2 * D);
    const KRole<D> ro;
    const Lay& L = c.L;
    const uint32_t base = tc::smem_addr(dst) + (ro.q4 >> 1) * kstride;
#pragma unroll 4
    for (int b = ro.par; b < L.nb8; b += NPAR) {
        const int t = 8 * b + ro.r8, j = 4 * ro.q4;
        float x[4], lc[4], lm[4];
        opload4<OP>(c, t, j, x);
        ld4(c.s + L.LC + (size_t)t * D + j, lc);
        ld4(c.s + L.LC + (size_t)(8 * b + 3) * D + j, lm);
        float4 o;
        o.x = tc::tf32_rn(x[0] * fexp<Tin>(XSIDE ? lc[0] - lm[0] : lm[0] - lc[0]));
        o.y = tc::tf32_rn(x[1] * fexp<Tin>(XSIDE ? lc[1] - lm[1] : lm[1] - lc[1]));
        o.z = tc::tf32_rn(x[2] * fexp<Tin>(XSIDE ? lc[2] - lm[2] : lm[2] - lc[2]));
        o.w = tc::tf32_rn(x[3] * fexp<Tin>(XSIDE ? lc[3] - lm[3] : lm[3] - lc[3]));
        sts128(base + tc::kblk_off(t, 4 * (ro.q4 & 1)), o);
    }
}

// The same operand stored MN-major (rows = channels), K block b of the tokens
// at kb0 + b (4 KB each, 128 channel rows).
template <int OP, bool XSIDE, typename Tin, int D>
__device__ void form_mid_mn(const Chunk<Tin, D>& c, unsigned char* dst, int kb0) {
    constexpr int NPAR = kThreads / (2 * D);
    const MnRole<D> ro;
    const Lay& L = c.L;
    const uint32_t base = tc::smem_addr(dst) + tc::mn_off(4 * ro.q4, ro.kk, 2048);
#pragma unroll 4
    for (int b = ro.par; b < L.nb8; b += NPAR) {
        const int t = 8 * b + ro.kk, j = 4 * ro.q4;
        float x[4], lc[4], lm[4];
        opload4<OP>(c, t, j, x);
        ld4(c.s + L.LC + (size_t)t * D + j, lc);
        ld4(c.s + L.LC + (size_t)(8 * b + 3) * D + j, lm);
        float4 o;
        o.x = tc::tf32_rn(x[0] * fexp<Tin>(XSIDE ? lc[0] - lm[0] : lm[0] - lc[0]));
        o.y = tc::tf32_rn(x[1] * fexp<Tin>(XSIDE ? lc[1] - lm[1] : lm[1] - lc[1]));
        o.z = tc::tf32_rn(x[2] * fexp<Tin>(XSIDE ? lc[2] - lm[2] : lm[2] - lc[2]));
        o.w = tc::tf32_rn(x[3] * fexp<Tin>(XSIDE ? lc[3] - lm[3] : lm[3] - lc[3]));
        sts128(base + (kb0 + b) * 4096, o);
    }
}

// Channel half hf (K blocks [hf D/16, (hf+1) D/16)) of form_mid_k, stored from
// K block 0 of dst.
template <int OP, bool XSIDE, typename Tin, int D>
__device__ void form_mid_k_half(const Chunk<Tin, D>& c, unsigned char* dst, int kstride, int hf) {
    constexpr int QH = D / 8;   // channel quads per half
    const Lay& L = c.L;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r8 = lane & 7;
    const int slot = warp * 4 + (lane >> 3);  // 0 .. 31
    const int q4 = slot % QH, par = slot / QH, NPAR = 32 / QH;
    const int j = 4 * (hf * QH + q4);
    const uint32_t base = tc::smem_addr(dst) + (q4 >> 1) * kstride;
#pragma unroll 4
    for (int b = par; b < L.nb8; b += NPAR) {
        const int t = 8 * b + r8;
        float x[4], lc[4], lm[4];
        opload4<OP>(c, t, j, x);
        ld4(c.s + L.LC + (size_t)t * D + j, lc);
        ld4(c.s + L.LC + (size_t)(8 * b + 3) * D + j, lm);
        float4 o;
        o.x = tc::tf32_rn(x[0] * fexp<Tin>(XSIDE ? lc[0] - lm[0] : lm[0] - lc[0]));
        o.y = tc::tf32_rn(x[1] * fexp<Tin>(XSIDE ? lc[1] - lm[1] : lm[1] - lc[1]));
        o.z = tc::tf32_rn(x[2] * fexp<Tin>(XSIDE ? lc[2] - lm[2] : lm[2] - lc[2]));
        o.w = tc::tf32_rn(x[3] * fexp<Tin>(XSIDE ? lc[3] - lm[3] : lm[3] - lc[3]));
        sts128(base + tc::kblk_off(t, 4 * (q4 & 1)), o);
    }
}

// ------------------------------------------------------------------ masked products

// out_p[t][s] = [X (*) Z_p]_{ts} masked to s < t (strict) or s <= t, p = 0, 1.
//  - earlier blocks: one chain per block J of s, B = [Zz_0 ; Zz_1] rows of J
//    (N = 16), A = Xx F[.][J] over the later tokens (K-major, K = channels),
//    TMEM column 16 J + 8 p + (s - 8 J); lane = t;
//  - then the in-block pairs: Xo Zo_p^T with the mid-block pivots (full C x C
//    product in two channel halves, only same-block entries are read), TMEM
//    columns 128 p + s.  At most 256 TMEM columns and 96 KB of shared memory.
template <typename Tin, int D, int X, int Z0, int Z1>
__device__ void panel_masked_pair(const Chunk<Tin, D>& c, TcCta& tcx, size_t out0, size_t out1,
                                  bool incl0, bool incl1) {
    const Lay& L = c.L;
    const int C = L.C, nb8 = L.nb8;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const PanelSmem m = panel_smem<D>(c.s, L, tcx.sbuf, kPairA, 16 * 512);
    const int q = warp & 3, pr = warp >> 2;
    const int t = 32 * q + lane;
    const size_t out = pr ? out1 : out0;
    const bool incl = pr ? incl1 : incl0;
    const uint32_t lane_base = tcx.st.tmem + ((uint32_t)(32 * q) << 16);
    // earlier blocks
    {
        const size_t xx = panel_xx(L, X), zz0 = panel_zz(L, Z0), zz1 = panel_zz(L, Z1);
        constexpr int NQ = D / 4, NPAR = kThreads / (8 * NQ);
        const KRole<D> ro;
        const uint32_t idesc = tc::idesc_tf32(128, 16);
        const uint32_t aq = tc::smem_addr(m.A) + (ro.q4 >> 1) * 4096;
        const uint32_t fq = tc::smem_addr(m.f) + 16 * ro.q4;
        for (int J = 0; J + 1 < nb8; ++J) {
            // B: rows n < 8 from Zz_0, n >= 8 from Zz_1 (tokens 8J + n % 8), already TF32
            for (int idx = tid; idx < 16 * NQ; idx += kThreads) {
                const int n = idx & 15, qq = idx >> 4;
                const float* src = c.s + (n < 8 ? zz0 : zz1) + (size_t)(8 * J + (n & 7)) * D + 4 * qq;
                tc::cp_async16(tc::smem_addr(m.B + (qq >> 1) * 512 + tc::kblk_off(n, 4 * (qq & 1))), src, true);
            }
            // A: raw Xx rows t >= 8(J + 1), each thread its own chunks
            for (int I = J + 1 + ro.par; I < nb8; I += NPAR) {
                const int tt = 8 * I + ro.r8;
                tc::cp_async16(aq + tc::kblk_off(tt, 4 * (ro.q4 & 1)), c.s + xx + (size_t)tt * D + 4 * ro.q4, true);
            }
            panel_ftab<Tin, D, false>(m, nb8, J);
            asm volatile("cp.async.wait_all;" ::: "memory");
            __syncthreads();
            for (int I = J + 1 + ro.par; I < nb8; I += NPAR)
                scale_at(aq + tc::kblk_off(8 * I + ro.r8, 4 * (ro.q4 & 1)), fq + I * D * 4);
            panel_run(tcx.st, [&]() {
                for (int kb = 0; kb < D / 8; ++kb) {
                    const uint64_t da = tc::make_desc(tc::smem_addr(m.A + kb * 4096), 128, 256);
                    const uint64_t db = tc::make_desc(tc::smem_addr(m.B + kb * 512), 128, 256);
                    tc::issue_mma(tcx.st.tmem + 16 * J, da, db, idesc, kb > 0 ? 1u : 0u);
                }
            });
        }
        // blocks before t's block from TMEM, zeros after it (t's own block later)
        for (int J = 0; J < nb8; ++J) {
            float v[8];
            if (J + 1 < nb8) tmem_ld8(lane_base + (uint32_t)(16 * J + 8 * pr), v);
            if (t < C) {
                const int I = t >> 3;
                float* d = c.s + out + (size_t)t * C + 8 * J;
                if (J < I) {
                    *reinterpret_cast<float4*>(d) = make_float4(v[0], v[1], v[2], v[3]);
                    *reinterpret_cast<float4*>(d + 4) = make_float4(v[4], v[5], v[6], v[7]);
                } else if (J > I) {
                    *reinterpret_cast<float4*>(d) = make_float4(0.f, 0.f, 0.f, 0.f);
                    *reinterpret_cast<float4*>(d + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        }
        panel_end();
    }
    // in-block pairs, in two channel halves (A = Xo, B = Zo_p, 32 KB each)
    {
        unsigned char* Bd = m.A + 32 * 1024;
        constexpr int KH = D / 16;  // K blocks per half
#pragma unroll 1
        for (int pr2 = 0; pr2 < 2; ++pr2) {
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                form_mid_k_half<X, true>(c, m.A, 4096, hf);
                if (pr2 == 0) form_mid_k_half<Z0, false>(c, Bd, C * 32, hf);
                else form_mid_k_half<Z1, false>(c, Bd, C * 32, hf);
                panel_run(tcx.st, [&]() {
                    const uint32_t idesc = tc::idesc_tf32(128, C);
                    for (int kb = 0; kb < KH; ++kb) {
                        const uint64_t da = tc::make_desc(tc::smem_addr(m.A + kb * 4096), 128, 256);
                        const uint64_t db = tc::make_desc(tc::smem_addr(Bd + kb * C * 32), 128, 256);
                        tc::issue_mma(tcx.st.tmem + 128 * pr2, da, db, idesc, (hf > 0 || kb > 0) ? 1u : 0u);
                    }
                });
            }
        }
        // t's own block (masked); the warp's 32 lanes span blocks 4q .. 4q + 3
        float v[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float x[8];
            tmem_ld8(lane_base + (uint32_t)(128 * pr + 8 * (4 * q + i)), x);
            if ((lane >> 3) == i)
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = x[u];
        }
        if (t < C) {
            const int I = t >> 3;
            float w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int s = 8 * I + u;
                w[u] = (incl ? s <= t : s < t) ? v[u] : 0.f;
            }
            float* d = c.s + out + (size_t)t * C + 8 * I;
            *reinterpret_cast<float4*>(d) = make_float4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<float4*>(d + 4) = make_float4(w[4], w[5], w[6], w[7]);
        }
    }
    panel_end();
}

// ------------------------------------------------------------------ gradients

// X side:  out[t][c] = sum_{s <= t} (G0[t][s] Z0_sc + G1[t][s] Z1_sc) exp(Gam_tc - Gam_sc)
// (G0, G1 already masked), then epi(8, t0, c, v[8]) for 8 consecutive tokens.
//  - in-block: chain per block b over K = [tokens of b for Z0 ; for Z1],
//    A = Zo_p (mid pivot, MN-major), B = G_p rows of b restricted to b (N = 16,
//    rows past 8 zero), TMEM columns kDiagCol + 8b; output factor xo_t;
//  - earlier blocks: chain per block I of t over K = [s < 8I for Z0 ; for Z1]:
//    A = Zz_p F[I][J(s)] (MN-major), B = G_p rows [8I, 8I + 16) (K-major,
//    N = 16); TMEM columns 8I; output factor x8f_t.  TMEM lane = channel.
template <typename Tin, int D, int Z0, int Z1, class EPI>
__device__ void panel_grad_x(const Chunk<Tin, D>& c, TcCta& tcx, size_t G0, size_t G1, const EPI& epi) {
    const Lay& L = c.L;
    const int C = L.C, nb8 = L.nb8;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const PanelSmem m = panel_smem<D>(c.s, L, tcx.sbuf);
    const uint32_t idesc = tc::idesc_tf32(128, 16) | (1u << 15);  // A MN-major
    // in-block products
    form_mid_mn<Z0, false>(c, m.A, 0);
    form_mid_mn<Z1, false>(c, m.A, nb8);
    for (int idx = tid; idx < 2 * nb8 * 32; idx += kThreads) {  // B: 16 rows x 2 halves per block
        const int kb = idx >> 5, r = (idx >> 1) & 15, h = idx & 1;
        const int pp = kb >= nb8, b = kb - pp * nb8;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < 8) v = *reinterpret_cast<const float4*>(c.s + (pp ? G1 : G0) + (size_t)(8 * b + r) * C + 8 * b + 4 * h);
        sts128(tc::smem_addr(m.B + kb * 512) + tc::kblk_off(r, 4 * h), v);
    }
    panel_run(tcx.st, [&]() {
        for (int b = 0; b < nb8; ++b)
            for (int pp = 0; pp < 2; ++pp) {
                const int kb = pp * nb8 + b;
                const uint64_t da = tc::make_desc_mn32(tc::smem_addr(m.A + kb * 4096), 2048);
                const uint64_t db = tc::make_desc(tc::smem_addr(m.B + kb * 512), 128, 256);
                tc::issue_mma(tcx.st.tmem + kDiagCol + 8 * b, da, db, idesc, pp ? 1u : 0u);
            }
    });
    // earlier blocks
    constexpr int NPAR = kThreads / (2 * D);
    const MnRole<D> ro;
    const size_t zz[2] = {panel_zz(L, Z0), panel_zz(L, Z1)};
    const uint32_t aq = tc::smem_addr(m.A) + tc::mn_off(4 * ro.q4, ro.kk, 2048);
    const uint32_t fq = tc::smem_addr(m.f) + 16 * ro.q4;
    for (int I = 1; I < nb8; ++I) {
        const int nb = C - 8 * I < 16 ? C - 8 * I : 16;
        // B: K block p*I + jb = G_p rows [8I, 8I + nb) x tokens of block jb (raw float32)
        for (int idx = tid; idx < 2 * I * 32; idx += kThreads) {
            const int kb = idx >> 5, r = (idx >> 1) & 15, h = idx & 1;
            const int pp = kb >= I, jb = kb - pp * I;
            const bool ok = r < nb;
            const float* src = c.s + (pp ? G1 : G0) + (size_t)(8 * I + (ok ? r : 0)) * C + 8 * jb + 4 * h;
            tc::cp_async16(tc::smem_addr(m.B + kb * 512 + tc::kblk_off(r, 4 * h)), src, ok);
        }
        // A: raw Zz_p rows, each thread its own chunks
#pragma unroll
        for (int pp = 0; pp < 2; ++pp)
            for (int jb = I - 1 - ro.par; jb >= 0; jb -= NPAR)
                tc::cp_async16(aq + (pp * I + jb) * 4096, c.s + zz[pp] + (size_t)(8 * jb + ro.kk) * D + 4 * ro.q4, true);
        panel_ftab<Tin, D, true>(m, nb8, I);
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
        for (int jb = I - 1 - ro.par; jb >= 0; jb -= NPAR) {
            scale_at(aq + jb * 4096, fq + jb * D * 4);
            scale_at(aq + (I + jb) * 4096, fq + jb * D * 4);
        }
        panel_run(tcx.st, [&]() {
            for (int kb = 0; kb < 2 * I; ++kb) {
                const uint64_t da = tc::make_desc_mn32(tc::smem_addr(m.A + kb * 4096), 2048);
                const uint64_t db = tc::make_desc(tc::smem_addr(m.B + kb * 512), 128, 256);
                tc::issue_mma(tcx.st.tmem + 8 * I, da, db, idesc, kb > 0 ? 1u : 0u);
            }
        });
    }
    // epilogue: lane = channel, 8 tokens of one block per step
    const int q = warp & 3, half = warp >> 2;
    const int cc = 32 * q + lane;
    const uint32_t lane_base = tcx.st.tmem + ((uint32_t)(32 * q) << 16);
    if (32 * q < D) {
        for (int I = half; I < nb8; I += 2) {
            const int t0 = 8 * I;
            float lc[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) lc[u] = c.s[L.LC + (size_t)(t0 + u) * D + cc];
            const float lm = lc[3];
            float pv[8], dv[8], v[8];
            if (I > 0) tmem_ld8(lane_base + (uint32_t)(8 * I), pv);
            tmem_ld8(lane_base + kDiagCol + (uint32_t)(8 * I), dv);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                v[u] = fexp<Tin>(lc[u] - lm) * dv[u];
                if (I > 0) v[u] += fexp<Tin>(lc[u]) * pv[u];
            }
            epi(std::integral_constant<int, 8>{}, t0, cc, v);
        }
    }
    panel_end();
}

// Z side:  out[s][c] = sum_{t >= s} (G0[t][s] X0_tc + G1[t][s] X1_tc) exp(Gam_tc - Gam_sc)
// (G0, G1 already masked), then epi(8, s0, c, v[8]).
//  - in-block: as on the X side with A = Xo_p, B[n][k] = G_p[8b + k][8b + n]
//    (n < 8), output factor zo_s;
//  - earlier blocks: chain per block J of s over K = [t >= 8J + 8 for X0 ; for
//    X1]: A = Xx_p F[I(t)][J] (MN-major), B = G_p[t][8J + n], n < 32
//    (MN-major, N = 32, columns past the block's 8 thrown away); TMEM
//    columns 8J; output factor z8f_s.  TMEM lane = channel.
template <typename Tin, int D, int X0, int X1, class EPI>
__device__ void panel_grad_z(const Chunk<Tin, D>& c, TcCta& tcx, size_t G0, size_t G1, const EPI& epi) {
    const Lay& L = c.L;
    const int C = L.C, nb8 = L.nb8;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const PanelSmem m = panel_smem<D>(c.s, L, tcx.sbuf);
    // in-block products
    {
        const uint32_t idesc = tc::idesc_tf32(128, 16) | (1u << 15);  // A MN-major
        form_mid_mn<X0, true>(c, m.A, 0);
        form_mid_mn<X1, true>(c, m.A, nb8);
        for (int idx = tid; idx < 2 * nb8 * 128; idx += kThreads) {  // B: 16 x 8 per block, transposed
            const int kb = idx >> 7, n = (idx >> 3) & 15, k = idx & 7;
            const int pp = kb >= nb8, b = kb - pp * nb8;
            const float v = n < 8 ? c.s[(pp ? G1 : G0) + (size_t)(8 * b + k) * C + 8 * b + n] : 0.f;
            reinterpret_cast<float*>(m.B + kb * 512 + tc::kblk_off(n, k & 4))[k & 3] = v;
        }
        panel_run(tcx.st, [&]() {
            for (int b = 0; b < nb8; ++b)
                for (int pp = 0; pp < 2; ++pp) {
                    const int kb = pp * nb8 + b;
                    const uint64_t da = tc::make_desc_mn32(tc::smem_addr(m.A + kb * 4096), 2048);
                    const uint64_t db = tc::make_desc(tc::smem_addr(m.B + kb * 512), 128, 256);
                    tc::issue_mma(tcx.st.tmem + kDiagCol + 8 * b, da, db, idesc, pp ? 1u : 0u);
                }
        });
    }
    // earlier blocks
    constexpr int NPAR = kThreads / (2 * D);
    const MnRole<D> ro;
    const size_t xx[2] = {panel_xx(L, X0), panel_xx(L, X1)};
    const uint32_t idesc = tc::idesc_tf32(128, 32) | (1u << 15) | (1u << 16);  // A, B MN-major
    const uint32_t aq = tc::smem_addr(m.A) + tc::mn_off(4 * ro.q4, ro.kk, 2048);
    const uint32_t fq = tc::smem_addr(m.f) + 16 * ro.q4;
    for (int J = 0; J + 1 < nb8; ++J) {
        const int nblk = nb8 - J - 1;  // token blocks J+1 .. nb8-1 per operand
        const int nb = C - 8 * J < 32 ? C - 8 * J : 32;
        // B: K block p*nblk + i = G_p[t][8J + n], t in block J+1+i (raw float32)
        for (int idx = tid; idx < 2 * nblk * 64; idx += kThreads) {
            const int kb = idx >> 6, kk = (idx >> 3) & 7, n = 4 * (idx & 7);
            const int pp = kb >= nblk, i = kb - pp * nblk;
            const bool ok = n < nb;
            const float* src = c.s + (pp ? G1 : G0) + (size_t)(8 * (J + 1 + i) + kk) * C + (ok ? 8 * J + n : 0);
            tc::cp_async16(tc::smem_addr(m.B + kb * 1024 + tc::mn_off(n, kk, 512)), src, ok);
        }
        // A: raw Xx_p rows, each thread its own chunks
#pragma unroll
        for (int pp = 0; pp < 2; ++pp)
            for (int i = ro.par; i < nblk; i += NPAR)
                tc::cp_async16(aq + (pp * nblk + i) * 4096,
                               c.s + xx[pp] + (size_t)(8 * (J + 1 + i) + ro.kk) * D + 4 * ro.q4, true);
        panel_ftab<Tin, D, false>(m, nb8, J);
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
        for (int i = ro.par; i < nblk; i += NPAR) {
            scale_at(aq + i * 4096, fq + (J + 1 + i) * D * 4);
            scale_at(aq + (nblk + i) * 4096, fq + (J + 1 + i) * D * 4);
        }
        panel_run(tcx.st, [&]() {
            for (int kb = 0; kb < 2 * nblk; ++kb) {
                const uint64_t da = tc::make_desc_mn32(tc::smem_addr(m.A + kb * 4096), 2048);
                const uint64_t db = tc::make_desc_mn32(tc::smem_addr(m.B + kb * 1024), 512);
                tc::issue_mma(tcx.st.tmem + 8 * J, da, db, idesc, kb > 0 ? 1u : 0u);
            }
        });
    }
    // epilogue: lane = channel, 8 tokens of one block per step
    const int q = warp & 3, half = warp >> 2;
    const int cc = 32 * q + lane;
    const uint32_t lane_base = tcx.st.tmem + ((uint32_t)(32 * q) << 16);
    if (32 * q < D) {
        for (int J = half; J < nb8; J += 2) {
            const int s0 = 8 * J;
            float lc[8], rc[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                lc[u] = c.s[L.LC + (size_t)(s0 + u) * D + cc];
                rc[u] = c.s[L.RC + (size_t)(s0 + u) * D + cc];
            }
            const float lm = lc[3];
            float pv[8], dv[8], v[8];
            if (J + 1 < nb8) tmem_ld8(lane_base + (uint32_t)(8 * J), pv);
            tmem_ld8(lane_base + kDiagCol + (uint32_t)(8 * J), dv);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                v[u] = fexp<Tin>(lm - lc[u]) * dv[u];
                if (J + 1 < nb8) v[u] += fexp<Tin>(rc[u]) * pv[u];
            }
            epi(std::integral_constant<int, 8>{}, s0, cc, v);
        }
    }
    panel_end();
}

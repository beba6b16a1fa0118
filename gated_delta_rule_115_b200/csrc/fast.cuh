// fast.cuh -- single-pivot decay-masked products and their gradients for
// chunks whose log decay spans at most kTameSpan per channel (bf16 inputs,
// chunks of 32 to 128 tokens).  Included inside namespace muir after
// panel.cuh; chunks that fail the span test take the 8-token panels there.
//
// With Gam_t = Pre[I(t)] + Lc_t (the cumulative log decay inside the chunk, a
// short sum of same-sign terms) and the per-channel pivot P = gbar / 2, every
// factor exp(Gam_t - P) and exp(P - Gam_t) lies in [e^-70, e^70] when
// |gbar| <= 140, so
//   exp(Gam_t - Gam_s) = exp(Gam_t - P) exp(P - Gam_s)
// splits into per-row operand scalings without overflow, and each product is
// one dense tensor-core GEMM over the whole chunk:
//   masked product   out[t][s] = mask_{s<t | s<=t} (Xo Zo^T)[t][s]
//   X-side gradient  out[t][c] = exp(Gam_tc - P_c) sum_s G[t][s] Zo[s][c]
//   Z-side gradient  out[s][c] = exp(P_c - Gam_sc) sum_t G[t][s] Xo[t][c]
// with Xo = X exp(Gam - P), Zo = Z exp(P - Gam).  Entries above the diagonal
// of the masked product may overflow; they are never read.  In the gradient
// sums G is zero above the diagonal and every Zo, Xo is finite, so the sums
// carry the true result times at most e^70.
//
// Operands are written once per chunk in the tensor-core shared-memory
// layouts (K-major core matrices or the MN-major 128-byte swizzle with 32-byte
// atoms) into the chunk's scratch slot, then brought into shared memory with
// one bulk copy each.
#pragma once

// (included inside namespace muir)

constexpr float kTameSpan = 140.f;
constexpr int kFastPairSmem = 3 * 32768;  // masked pair: three 32 KB half tiles
constexpr int kFastGradSmem = 2 * 65536;  // gradient products: two 64 KB tiles

// True (for all threads) when every channel's chunk log decay |gbar| <= kTameSpan.
template <typename Tin, int D>
__device__ __forceinline__ bool chunk_tame(const Chunk<Tin, D>& c) {
    const int j = threadIdx.x;
    const bool ok = j >= D || -c.s[c.L.GBAR + j] <= kTameSpan;
    return __syncthreads_and(ok) != 0;
}

// Xo (K-major, 128-row tiles) for X in {K, Qh}, Zo (K-major, C rows) for Z in
// {A, K} (with_k: the masked products run); with_mn the MN-major copies
// (rows = channels) the gradients read.
template <typename Tin, int D>
__device__ void fast_prep(const Chunk<Tin, D>& c, bool with_q, bool with_mn, bool with_k = true) {
    const Lay& L = c.L;
    const int C = L.C;
    unsigned char* base = reinterpret_cast<unsigned char*>(c.s);
    for (int idx = threadIdx.x; idx < C * D / 4; idx += kThreads) {
        const int t = idx / (D / 4), j = 4 * (idx % (D / 4));
        const size_t g = c.base + (size_t)t * c.rs + j;
        float k4[4], e4[4], q4[4], m4[4], lc[4], pre[4], gb[4];
        ld4in(c.k + g, k4);
        ld4in(c.e + g, e4);
        if (with_q) {
            ld4in(c.q + g, q4);
            ld4in(c.gm + g, m4);
        }
        ld4(c.s + L.LC + (size_t)t * D + j, lc);
        ld4(c.s + L.PRE + (size_t)(t >> 3) * D + j, pre);
        ld4(c.s + L.GBAR + j, gb);
        float4 xk, xq, za, zk;
        float* pxk = &xk.x; float* pxq = &xq.x; float* pza = &za.x; float* pzk = &zk.x;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float d = pre[u] + lc[u] - 0.5f * gb[u];
            const float ex = fexp<Tin>(d), ez = fexp<Tin>(-d);
            pxk[u] = tc::tf32_rn(k4[u] * ex);
            pxq[u] = with_q ? tc::tf32_rn(m4[u] * q4[u] * ex) : 0.f;
            pza[u] = tc::tf32_rn(e4[u] * k4[u] * ez);
            pzk[u] = tc::tf32_rn(k4[u] * ez);
        }
        const size_t ox = (size_t)(j >> 3) * 4096 + tc::kblk_off(t, j & 7);
        const size_t oz = (size_t)(j >> 3) * C * 32 + tc::kblk_off(t, j & 7);
        if (with_k) {
            *reinterpret_cast<float4*>(base + 4 * L.OXK + ox) = xk;
            if (with_q) *reinterpret_cast<float4*>(base + 4 * L.OXQ + ox) = xq;
            *reinterpret_cast<float4*>(base + 4 * L.OZA + oz) = za;
            *reinterpret_cast<float4*>(base + 4 * L.OZK + oz) = zk;
        }
        if (with_mn) {
            const size_t om = (size_t)(t >> 3) * 4096 + tc::mn_off(j, t & 7, 2048);
            *reinterpret_cast<float4*>(base + 4 * L.MXK + om) = xk;
            if (with_q) *reinterpret_cast<float4*>(base + 4 * L.MXQ + om) = xq;
            *reinterpret_cast<float4*>(base + 4 * L.MZA + om) = za;
            *reinterpret_cast<float4*>(base + 4 * L.MZK + om) = zk;
        }
    }
    __syncthreads();
}

// ------------------------------------------------------------------ bulk copies

struct Bulk {
    unsigned char* dst;  // shared memory, 16-byte aligned
    const void* src;     // global memory, 16-byte aligned
    uint32_t bytes;      // multiple of 16
};

// Copy the segments with the bulk-copy engine, completion counted on the
// CTA's barrier; all threads call and wait (bounded).
template <int N>
__device__ void bulk_load(tc::State& st, const Bulk (&b)[N]) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t total = 0;
#pragma unroll
        for (int i = 0; i < N; ++i) total += b[i].bytes;
        const uint32_t bar = tc::smem_addr(st.mbar);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(total)
                     : "memory");
#pragma unroll
        for (int i = 0; i < N; ++i)
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                ::"r"(tc::smem_addr(b[i].dst)), "l"(b[i].src), "r"(b[i].bytes), "r"(bar)
                : "memory");
    }
    tc::wait_mma(st);
}

// One thread issues the chain, all threads wait for it (bounded).  The block
// barrier first: every thread has finished waiting for the barrier's previous
// phase before this chain can complete the next one (a waiter that fell two
// phases behind would read the parity as pending).
template <class ISSUE>
__device__ __forceinline__ void fast_mma(tc::State& st, const ISSUE& issue) {
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        issue();
        tc::commit(st);
    }
    tc::wait_mma(st);
}

// ------------------------------------------------------------------ masked products

// out_p[t][s] = [X (*) Z_p]_{ts} masked to s < t (strict) or s <= t, p = 0, 1:
// Xo Zo_p^T into TMEM columns 128 p + s (lane t), the channels in two halves
// (96 KB of shared memory, 256 TMEM columns).
template <typename Tin, int D, int X, int Z0, int Z1>
__device__ void fast_masked_pair(const Chunk<Tin, D>& c, TcCta& tcx, size_t out0, size_t out1,
                                 bool incl0, bool incl1) {
    const Lay& L = c.L;
    const int C = L.C, nb8 = L.nb8;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int KH = D / 16;                 // K blocks per channel half
    const uint32_t ah = KH * 4096, bh = (uint32_t)KH * C * 32;
    unsigned char* A = tcx.sbuf;
    unsigned char* B0 = A + ah;
    unsigned char* B1 = B0 + bh;
    const unsigned char* gx = reinterpret_cast<const unsigned char*>(c.s + (X == OP_Q ? L.OXQ : L.OXK));
    const unsigned char* g0 = reinterpret_cast<const unsigned char*>(c.s + (Z0 == OP_A ? L.OZA : L.OZK));
    const unsigned char* g1 = reinterpret_cast<const unsigned char*>(c.s + (Z1 == OP_A ? L.OZA : L.OZK));
#pragma unroll 1
    for (int hf = 0; hf < 2; ++hf) {
        const Bulk b[3] = {{A, gx + hf * ah, ah}, {B0, g0 + hf * bh, bh}, {B1, g1 + hf * bh, bh}};
        bulk_load(tcx.st, b);
        fast_mma(tcx.st, [&]() {
            const uint32_t idesc = tc::idesc_tf32(128, C);
            for (int kb = 0; kb < KH; ++kb) {
                const uint64_t da = tc::make_desc(tc::smem_addr(A + kb * 4096), 128, 256);
                const uint64_t d0 = tc::make_desc(tc::smem_addr(B0 + kb * C * 32), 128, 256);
                const uint64_t d1 = tc::make_desc(tc::smem_addr(B1 + kb * C * 32), 128, 256);
                const uint32_t acc = (hf > 0 || kb > 0) ? 1u : 0u;
                tc::issue_mma(tcx.st.tmem, da, d0, idesc, acc);
                tc::issue_mma(tcx.st.tmem + 128, da, d1, idesc, acc);
            }
        });
    }
    const int q = warp & 3, pr = warp >> 2;
    const int t = 32 * q + lane;
    const size_t out = pr ? out1 : out0;
    const bool incl = pr ? incl1 : incl0;
    const uint32_t lane_base = tcx.st.tmem + ((uint32_t)(32 * q) << 16) + 128 * pr;
    for (int J = 0; J < nb8; ++J) {
        float v[8];
        tmem_ld8(lane_base + 8 * J, v);
        if (t < C) {
            float w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int s = 8 * J + u;
                w[u] = (incl ? s <= t : s < t) ? v[u] : 0.f;
            }
            float* d = c.s + out + (size_t)t * C + 8 * J;
            *reinterpret_cast<float4*>(d) = make_float4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<float4*>(d + 4) = make_float4(w[4], w[5], w[6], w[7]);
        }
    }
    panel_end();
}

// ------------------------------------------------------------------ gradients

__device__ __forceinline__ int gidx(const Lay& L, size_t G) {
    return G == L.LA ? 0 : G == L.LK ? 1 : G == L.MQK ? 2 : 3;
}

// Raw accumulators of the gradients through the masked products, into TMEM
// columns col .. col + C (lane = channel):
// X side:  acc[c][t] = sum_s (G0[t][s] Zo0[s][c] + G1[t][s] Zo1[s][c]), so that
//   sum_s (G0[t][s] Z0_sc + G1[t][s] Z1_sc) exp(Gam_tc - Gam_sc) = exp(Gam_tc - P_c) acc[c][t];
//   A = Zo_p (MN-major), B = G_p (K-major rows t);
// Z side:  acc[c][s] = sum_t (G0[t][s] Xo0[t][c] + G1[t][s] Xo1[t][c]), so that
//   sum_t (G0[t][s] X0_tc + G1[t][s] X1_tc) exp(Gam_tc - Gam_sc) = exp(P_c - Gam_sc) acc[c][s];
//   A = Xo_p (MN-major), B[s][t] = G_p[t][s] (MN-major).
template <typename Tin, int D, bool XSIDE, int O0, int O1>
__device__ void fast_grad_mma(const Chunk<Tin, D>& c, TcCta& tcx, size_t G0, size_t G1, uint32_t col) {
    const Lay& L = c.L;
    const int C = L.C;
    unsigned char* A = tcx.sbuf;
    unsigned char* B = A + 65536;
    const uint32_t idesc = tc::idesc_tf32(128, C) | (1u << 15) | (XSIDE ? 0u : (1u << 16));
#pragma unroll 1
    for (int p = 0; p < 2; ++p) {
        const int op = p ? O1 : O0;
        const size_t a = XSIDE ? (op == OP_A ? L.MZA : L.MZK) : (op == OP_Q ? L.MXQ : L.MXK);
        const int gi = gidx(L, p ? G1 : G0);
        const Bulk b[2] = {{A, c.s + a, (uint32_t)C * 512},
                           {B, c.s + (XSIDE ? L.GK[gi] : L.GM[gi]), (uint32_t)C * C * 4}};
        bulk_load(tcx.st, b);
        fast_mma(tcx.st, [&]() {
            for (int kb = 0; kb < C / 8; ++kb) {
                const uint64_t da = tc::make_desc_mn32(tc::smem_addr(A + kb * 4096), 2048);
                const uint64_t db = XSIDE ? tc::make_desc(tc::smem_addr(B + kb * C * 32), 128, 256)
                                          : tc::make_desc_mn32(tc::smem_addr(B + kb * C * 32), C / 32 * 512);
                tc::issue_mma(tcx.st.tmem + col, da, db, idesc, (p > 0 || kb > 0) ? 1u : 0u);
            }
        });
    }
}

// Rows t of the masked-product gradient G_i in the two tensor-core layouts the
// gradient products read: K-major (rows t, K = s) and MN-major (K = t, rows s).
// w[8] holds G_i[t][s0 .. s0 + 8).
__device__ __forceinline__ void store_g_layouts(float* s, const Lay& L, int i, int t, int s0,
                                                const float* w) {
    const int C = L.C;
    unsigned char* gk = reinterpret_cast<unsigned char*>(s + L.GK[i]) + (size_t)(s0 >> 3) * C * 32;
    *reinterpret_cast<float4*>(gk + tc::kblk_off(t, 0)) = make_float4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<float4*>(gk + tc::kblk_off(t, 4)) = make_float4(w[4], w[5], w[6], w[7]);
    unsigned char* gm = reinterpret_cast<unsigned char*>(s + L.GM[i]) + (size_t)(t >> 3) * C * 32;
    const uint32_t sbo = C / 32 * 512;
    *reinterpret_cast<float4*>(gm + tc::mn_off(s0, t & 7, sbo)) = make_float4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<float4*>(gm + tc::mn_off(s0 + 4, t & 7, sbo)) = make_float4(w[4], w[5], w[6], w[7]);
}

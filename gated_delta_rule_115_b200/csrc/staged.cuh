// staged.cuh -- per-chunk building blocks that stage their operands through
// shared memory: the log-decay prologue, decay-masked products, gradients
// through decay-masked products and block triangular solves.  Included by
// chunk.cu after the Chunk / Lay definitions.
//
// Log-decay bookkeeping without cancellation.  With 8-token blocks I and the
// clamped log decays g, per channel j:
//   Lc[t] = sum_{i = start(I)}^{t} g_i        (forward, inside t's block)
//   Rc[t] = sum_{i = t+1}^{end(I)} g_i        (backward, inside t's block)
//   Bt[I] = block total,  Pre[I] = sum of Bt over earlier blocks,
//   Suf[I] = sum of Bt over later blocks.
// Every factor is the exponential of a short sum of same-sign terms:
//   x8f_t  = exp(Gam_t - Gam_{start(I)-1})        = exp(Lc[t])            <= 1
//   z8f_s  = exp(Gam_{end(J)} - Gam_s)            = exp(Rc[s])            <= 1
//   F[I][J]= exp(Gam_{start(I)-1} - Gam_{end(J)}) = exp(sum_{J<K<I} Bt[K]) <= 1
//   xof_t  = exp(Gam_t - Gam_m),  zof_s = exp(Gam_m - Gam_s), m = start + 3
//   e^Gam_t = exp(Pre[I] + Lc[t]),  e^{gbar - Gam_t} = exp(Rc[t] + Suf[I]).
#pragma once

// (included inside namespace muir)

// ------------------------------------------------------------------ prologue

template <typename Tin, int D>
__device__ void prologue2(const Chunk<Tin, D>& c) {
    const Lay& L = c.L;
    const int nb8 = L.nb8, tid = threadIdx.x;
    float* LC = c.s + L.LC;
    float* RC = c.s + L.RC;
    float* BT = c.s + L.BT;
    // local forward / backward sums inside every 8-token block
    for (int idx = tid; idx < nb8 * D; idx += kThreads) {
        const int I = idx / D, j = idx % D;
        float gv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            gv[u] = fmaxf(ldf(c.g + c.base + (size_t)(8 * I + u) * c.rs + j), kLogDecayMin);
        float f = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            f += gv[u];
            LC[(size_t)(8 * I + u) * D + j] = f;
        }
        float b = 0.f;
#pragma unroll
        for (int u = 7; u >= 0; --u) {
            RC[(size_t)(8 * I + u) * D + j] = b;
            b += gv[u];
        }
        BT[(size_t)I * D + j] = f;
    }
    __syncthreads();
    // exclusive prefix and suffix of the block totals: warp-level scans over the
    // blocks of one channel (lane = block; C <= 256 gives at most 32 blocks)
    const int warp = tid >> 5, lane = tid & 31;
    for (int j = warp; j < D; j += kThreads / 32) {
        const float v = lane < nb8 ? BT[(size_t)lane * D + j] : 0.f;
        float pre = v, suf = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, pre, off);
            if (lane >= off) pre += y;
            const float z = __shfl_down_sync(0xffffffffu, suf, off);
            if (lane + off < 32) suf += z;
        }
        if (lane < nb8) {
            c.s[L.PRE + (size_t)lane * D + j] = pre - v;
            c.s[L.SUF + (size_t)lane * D + j] = suf - v;
        }
        const float total = __shfl_sync(0xffffffffu, pre, 31);
        if (lane == 0) c.s[L.GBAR + j] = total;
    }
    __syncthreads();
}

// exp for the factors: the fast hardware exp2-based form for bf16 inputs (its
// ~1e-6 relative error is far below the bf16 tolerance), the accurate one for
// float32 inputs.
template <typename Tin>
__device__ __forceinline__ float fexp(float x) {
    if constexpr (std::is_same<Tin, float>::value) return expf(x);
    else return __expf(x);
}

// Log factors (see the header comment).
template <typename Tin, int D>
struct Fac {
    const float* s;
    Lay L;
    __device__ float lx8(int t, int j) const { return s[L.LC + (size_t)t * D + j]; }
    __device__ float lz8(int t, int j) const { return s[L.RC + (size_t)t * D + j]; }
    __device__ float lxo(int t, int j) const {
        return s[L.LC + (size_t)t * D + j] - s[L.LC + (size_t)((t & ~7) + 3) * D + j];
    }
    __device__ float lzo(int t, int j) const {
        return s[L.LC + (size_t)((t & ~7) + 3) * D + j] - s[L.LC + (size_t)t * D + j];
    }
    __device__ float eg(int t, int j) const {
        return fexp<Tin>(s[L.PRE + (size_t)(t >> 3) * D + j] + s[L.LC + (size_t)t * D + j]);
    }
    __device__ float egb(int t, int j) const {
        return fexp<Tin>(s[L.RC + (size_t)t * D + j] + s[L.SUF + (size_t)(t >> 3) * D + j]);
    }
    __device__ float gbar(int j) const { return s[L.GBAR + j]; }
};

template <typename Tin, int D>
__device__ __forceinline__ Fac<Tin, D> facs(const Chunk<Tin, D>& c) {
    Fac<Tin, D> f;
    f.s = c.s;
    f.L = c.L;
    return f;
}

// ------------------------------------------------------------------ fragments

template <int PASSES>
__device__ __forceinline__ void mma_f(float (&d)[4], const float (&a)[4], const float (&b)[2]) {
    uint32_t ah[4], al[4], bh[2], bl[2];
    split_tf32<PASSES>(a, ah, al);
    split_tf32<PASSES>(b, bh, bl);
    mma_tf32(d, ah, bh);
    if (PASSES == 3) {
        mma_tf32(d, ah, bl);
        mma_tf32(d, al, bh);
    }
}

// Channels per slab so that one C x slab fp32 tile is 8 KB (small staging
// areas leave most of the SM's unified L1 / shared memory to the L1 cache).
__host__ __device__ constexpr int slab_channels(int C, int D) {
    return (2048 / C) < D ? (2048 / C) : D;
}

// Shared-memory floats masked_pair_s needs.
__host__ __device__ constexpr int masked_smem_floats(int C, int D) {
    return 6 * C * (slab_channels(C, D) + 4) + (C / 8) * (C / 8) * slab_channels(C, D);
}

// Stage F[I][J][jj] = exp(sum_{J<K<I} Bt[K][j0 + jj]) for J < I (1 for J = I - 1).
template <typename Tin>
__device__ __forceinline__ void stage_F(float* FS, const float* s, const Lay& L, int D, int j0,
                                        int SL) {
    const int nb8 = L.nb8;  // <= 32
    for (int idx = threadIdx.x; idx < nb8 * SL; idx += kThreads) {
        const int I = idx / SL, jj = idx % SL;
        float bt[32];
#pragma unroll
        for (int J = 0; J < 32; ++J)  // all block totals first (independent loads)
            bt[J] = J < I ? s[L.BT + (size_t)J * D + j0 + jj] : 0.f;
        float acc = 0.f;
#pragma unroll
        for (int J = 31; J >= 0; --J) {
            if (J < I) {
                FS[((size_t)I * nb8 + J) * SL + jj] = fexp<Tin>(acc);
                acc += bt[J];
            }
        }
    }
}

// ------------------------------------------------------------------ masked products

// Two decay-masked products sharing X: out_p[t][s] = [X (*) Z_p]_{ts}, masked to
// s < t (strict) or s <= t.  Tiles are 16 rows x 8 columns; rows of a tile lie in
// 8-blocks rb0 = 2*I16 and rb1 = rb0 + 1, columns in 8-block J8.  Off-diagonal
// rows (rb > J8): A = X x8f F[rb][J8], B = Z z8f.  Diagonal rows (rb == J8):
// A = X xof, B = Z zof.  Channels are streamed through shared memory in slabs.
template <typename Tin, int D, int PASSES, int X, int Z0, int Z1>
__device__ void masked_pair_s(const Chunk<Tin, D>& c, float* sm, size_t out0, size_t out1,
                              bool incl0, bool incl1) {
    const Lay& L = c.L;
    const Fac<Tin, D> f = facs(c);
    const int C = L.C, nb8 = L.nb8, nb16 = L.nb16;
    const int SL = slab_channels(C, D), SP = SL + 4;
    float* XH = sm;
    float* XO = XH + C * SP;
    float* ZH0 = XO + C * SP;
    float* ZH1 = ZH0 + C * SP;
    float* ZO0 = ZH1 + C * SP;
    float* ZO1 = ZO0 + C * SP;
    float* FS = ZO1 + C * SP;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, cq = lane & 3;
    const int ntiles = nb16 * (nb16 + 1);
    constexpr int TPW = 9;
    for (int tbase = 0; tbase < ntiles; tbase += 8 * TPW) {
        float acc0[TPW][4], acc1[TPW][4];
#pragma unroll
        for (int i = 0; i < TPW; ++i)
#pragma unroll
            for (int u = 0; u < 4; ++u) acc0[i][u] = acc1[i][u] = 0.f;
        for (int j0 = 0; j0 < D; j0 += SL) {
            __syncthreads();
            for (int base = 0; base < C * SL; base += 4 * kThreads) {
                float x[4], z0[4], z1[4], l8[4], lm[4], r8[4];
#pragma unroll
                for (int it = 0; it < 4; ++it) {  // loads first, so they overlap
                    const int idx = base + threadIdx.x + it * kThreads;
                    const int t = idx / SL, j = j0 + idx % SL;
                    const bool in = idx < C * SL;
                    x[it] = in ? opval(c, X, t, j) : 0.f;
                    z0[it] = in ? opval(c, Z0, t, j) : 0.f;
                    z1[it] = in ? opval(c, Z1, t, j) : 0.f;
                    l8[it] = in ? f.lx8(t, j) : 0.f;
                    lm[it] = in ? c.s[L.LC + (size_t)((t & ~7) + 3) * D + j] : 0.f;
                    r8[it] = in ? f.lz8(t, j) : 0.f;
                }
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const int idx = base + threadIdx.x + it * kThreads;
                    if (idx >= C * SL) break;
                    const int t = idx / SL, jj = idx % SL;
                    const float ex8 = fexp<Tin>(l8[it]), exo = fexp<Tin>(l8[it] - lm[it]);
                    const float ez8 = fexp<Tin>(r8[it]), ezo = fexp<Tin>(lm[it] - l8[it]);
                    const int o = t * SP + jj;
                    XH[o] = x[it] * ex8;
                    XO[o] = x[it] * exo;
                    ZH0[o] = z0[it] * ez8;
                    ZH1[o] = z1[it] * ez8;
                    ZO0[o] = z0[it] * ezo;
                    ZO1[o] = z1[it] * ezo;
                }
            }
            stage_F<Tin>(FS, c.s, L, D, j0, SL);
            __syncthreads();
#pragma unroll
            for (int i = 0; i < TPW; ++i) {
                const int tile = tbase + warp + 8 * i;
                if (tile >= ntiles) break;
                int I16 = 0, rem = tile;
                while (rem >= 2 * I16 + 2) { rem -= 2 * I16 + 2; ++I16; }
                const int J8 = rem, t0 = 16 * I16, s0 = 8 * J8;
                const int rb0 = 2 * I16, rb1 = rb0 + 1;
                const bool off0 = rb0 > J8, off1 = rb1 > J8, dg0 = rb0 == J8, dg1 = rb1 == J8;
                const float* F0 = FS + ((size_t)rb0 * nb8 + J8) * SL;
                const float* F1 = FS + ((size_t)rb1 * nb8 + J8) * SL;
                const int r0 = (t0 + g) * SP, r1 = (t0 + g + 8) * SP, rs = (s0 + g) * SP;
                for (int k = cq; k < SL; k += 8) {
                    if (off0 || off1) {
                        float a[4], b0[2], b1[2];
                        a[0] = off0 ? XH[r0 + k] * F0[k] : 0.f;
                        a[1] = off1 ? XH[r1 + k] * F1[k] : 0.f;
                        a[2] = off0 ? XH[r0 + k + 4] * F0[k + 4] : 0.f;
                        a[3] = off1 ? XH[r1 + k + 4] * F1[k + 4] : 0.f;
                        b0[0] = ZH0[rs + k]; b0[1] = ZH0[rs + k + 4];
                        b1[0] = ZH1[rs + k]; b1[1] = ZH1[rs + k + 4];
                        mma_f<PASSES>(acc0[i], a, b0);
                        mma_f<PASSES>(acc1[i], a, b1);
                    }
                    if (dg0 || dg1) {
                        float a[4], b0[2], b1[2];
                        a[0] = dg0 ? XO[r0 + k] : 0.f;
                        a[1] = dg1 ? XO[r1 + k] : 0.f;
                        a[2] = dg0 ? XO[r0 + k + 4] : 0.f;
                        a[3] = dg1 ? XO[r1 + k + 4] : 0.f;
                        b0[0] = ZO0[rs + k]; b0[1] = ZO0[rs + k + 4];
                        b1[0] = ZO1[rs + k]; b1[1] = ZO1[rs + k + 4];
                        mma_f<PASSES>(acc0[i], a, b0);
                        mma_f<PASSES>(acc1[i], a, b1);
                    }
                }
            }
        }
        // store this pass's tiles with the masks
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
            const int tile = tbase + warp + 8 * i;
            if (tile >= ntiles) break;
            int I16 = 0, rem = tile;
            while (rem >= 2 * I16 + 2) { rem -= 2 * I16 + 2; ++I16; }
            const int t0 = 16 * I16, s0 = 8 * rem;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int t = t0 + g + (u >= 2 ? 8 : 0), ss = s0 + 2 * cq + (u & 1);
                c.s[out0 + (size_t)t * C + ss] = (incl0 ? ss <= t : ss < t) ? acc0[i][u] : 0.f;
                c.s[out1 + (size_t)t * C + ss] = (incl1 ? ss <= t : ss < t) ? acc1[i][u] : 0.f;
            }
        }
    }
    // the part above the visited tiles must read as zero
    for (int idx = threadIdx.x; idx < C * C; idx += kThreads) {
        const int t = idx / C, ss = idx % C;
        if ((ss >> 3) > 2 * (t >> 4) + 1) {
            c.s[out0 + idx] = 0.f;
            c.s[out1 + idx] = 0.f;
        }
    }
    __syncthreads();
}

// ------------------------------------------------------------------ gradients through masked products

// Slab shape of decayed_grad_s: channels per output slab (CH), tokens per
// contraction slab (TS), 16-row blocks per warp (RB); C = 256 takes narrower
// channel slabs so the F table fits.
__host__ __device__ constexpr int decayed_ch(int C) { return C > 128 ? 16 : 32; }
__host__ __device__ constexpr int decayed_ts(int C) { return 32; }

// Shared-memory floats decayed_grad_s needs: two gradient slabs (C x TS or
// TS x C, padded), four operand slabs (TS tokens x CH), the F table.
__host__ __device__ constexpr int decayed_smem_floats(int C) {
    return 2 * ((C * (decayed_ts(C) + 4)) > (decayed_ts(C) * (C + 8)) ? (C * (decayed_ts(C) + 4))
                                                                       : (decayed_ts(C) * (C + 8))) +
           4 * decayed_ts(C) * (decayed_ch(C) + 8) + (C / 8) * (C / 8) * decayed_ch(C);
}

// X side (XSIDE):  out[t][j] = sum_s Gm[t][s] Z_sj exp(Gam_tj - Gam_sj)
// Z side:          out[s][j] = sum_t Gm[t][s] X_tj exp(Gam_tj - Gam_sj)
// for two gradient matrices G0/G1 (already masked) paired with operands op0/op1.
// Output tiles: 16 rows x 32 channels; contraction in slabs of 32 tokens, one
// 8-token block per MMA step; off-diagonal block pairs scale the step's result
// by F, diagonal blocks use the mid-block pivot; output-side factors at the end.
template <typename Tin, int D, int PASSES, bool XSIDE, int CH, int TS, int RB, int op0, int op1,
          class EPI>
__device__ void decayed_grad_s(const Chunk<Tin, D>& c, float* sm, size_t G0, size_t G1,
                               const EPI& epi) {
    const Lay& L = c.L;
    const Fac<Tin, D> f = facs(c);
    const int C = L.C, nb8 = L.nb8, nb16 = L.nb16;
    constexpr int OP = CH + 8;             // operand slab row pitch
    const int GP = XSIDE ? TS + 4 : C + 8; // gradient slab row pitch
    float* GS0 = sm;
    float* GS1 = GS0 + (XSIDE ? C * GP : TS * GP);
    float* ZH0 = GS1 + (XSIDE ? C * GP : TS * GP);
    float* ZO0 = ZH0 + TS * OP;
    float* ZH1 = ZO0 + TS * OP;
    float* ZO1 = ZH1 + TS * OP;
    float* FS = ZO1 + TS * OP;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, cq = lane & 3;
    for (int j0 = 0; j0 < D; j0 += CH) {
        __syncthreads();
        stage_F<Tin>(FS, c.s, L, D, j0, CH);
        // each warp owns row blocks I16 = warp, warp + 8, ... (at most 2 for C <= 256)
        constexpr int NT = CH / 8;
        float off[RB][NT][4], dia[RB][NT][4];
#pragma unroll
        for (int a = 0; a < RB; ++a)
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int u = 0; u < 4; ++u) off[a][n][u] = dia[a][n][u] = 0.f;
        const int ts = C < TS ? C : TS;  // tokens in this K slab (C = 16 has one 16-token slab)
        for (int k0 = 0; k0 < C; k0 += ts) {
            __syncthreads();
            // gradient slabs
            {
                // rows x cols of the slab (X side: all C rows x ts tokens; Z side: ts rows x C)
                const int rows = XSIDE ? C : ts, cols = XSIDE ? ts : C, q4 = cols / 4;
                const int n4 = rows * q4;
                for (int base = 0; base < n4; base += 4 * kThreads) {
                    float4 a0[4], a1[4];
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int idx = base + threadIdx.x + it * kThreads;
                        if (idx < n4) {
                            const int r = idx / q4, cc = 4 * (idx % q4);
                            const size_t go = XSIDE ? (size_t)r * C + k0 + cc : (size_t)(k0 + r) * C + cc;
                            a0[it] = *reinterpret_cast<const float4*>(c.s + G0 + go);
                            a1[it] = *reinterpret_cast<const float4*>(c.s + G1 + go);
                        }
                    }
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int idx = base + threadIdx.x + it * kThreads;
                        if (idx >= n4) break;
                        const int r = idx / q4, cc = 4 * (idx % q4);
                        float* d0 = GS0 + r * GP + cc;
                        float* d1 = GS1 + r * GP + cc;
                        d0[0] = a0[it].x; d0[1] = a0[it].y; d0[2] = a0[it].z; d0[3] = a0[it].w;
                        d1[0] = a1[it].x; d1[1] = a1[it].y; d1[2] = a1[it].z; d1[3] = a1[it].w;
                    }
                }
            }
            // operand slabs: tokens k0.. of op0/op1 over channels j0.., scaled by the
            // pivot factors of the contraction side
            for (int base = 0; base < ts * CH; base += 2 * kThreads) {
                float v0[2], v1[2], lh[2], lo[2];
#pragma unroll
                for (int it = 0; it < 2; ++it) {
                    const int idx = base + threadIdx.x + it * kThreads;
                    const int t = k0 + idx / CH, j = j0 + idx % CH;
                    const bool in = idx < ts * CH;
                    v0[it] = in ? opval(c, op0, t, j) : 0.f;
                    v1[it] = in ? opval(c, op1, t, j) : 0.f;
                    lh[it] = in ? (XSIDE ? f.lz8(t, j) : f.lx8(t, j)) : 0.f;
                    lo[it] = in ? (XSIDE ? f.lzo(t, j) : f.lxo(t, j)) : 0.f;
                }
#pragma unroll
                for (int it = 0; it < 2; ++it) {
                    const int idx = base + threadIdx.x + it * kThreads;
                    if (idx >= ts * CH) break;
                    const int tt = idx / CH, jj = idx % CH;
                    const float eh = fexp<Tin>(lh[it]), eo = fexp<Tin>(lo[it]);
                    ZH0[tt * OP + jj] = v0[it] * eh;
                    ZO0[tt * OP + jj] = v0[it] * eo;
                    ZH1[tt * OP + jj] = v1[it] * eh;
                    ZO1[tt * OP + jj] = v1[it] * eo;
                }
            }
            __syncthreads();
#pragma unroll
            for (int a = 0; a < RB; ++a) {
                const int I16 = warp + 8 * a;
                if (I16 >= nb16) break;
                const int m0 = 16 * I16, rb0 = 2 * I16, rb1 = rb0 + 1;
                for (int bb = 0; bb < ts / 8; ++bb) {
                    const int B8 = k0 / 8 + bb;
                    int rel0, rel1;  // 1 = off-diagonal, 2 = diagonal, 0 = no contribution
                    if (XSIDE) {
                        rel0 = B8 < rb0 ? 1 : (B8 == rb0 ? 2 : 0);
                        rel1 = B8 < rb1 ? 1 : (B8 == rb1 ? 2 : 0);
                    } else {
                        rel0 = B8 > rb0 ? 1 : (B8 == rb0 ? 2 : 0);
                        rel1 = B8 > rb1 ? 1 : (B8 == rb1 ? 2 : 0);
                    }
                    if (rel0 == 0 && rel1 == 0) continue;
                    for (int kind = 1; kind <= 2; ++kind) {
                        if (rel0 != kind && rel1 != kind) continue;
                        // A fragment: gradient entries; rows of the other kind are zero
                        float av0[4], av1[4];
                        const int kl = 8 * bb + cq;  // token within the slab
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int r = g + ((u & 1) ? 8 : 0), kk = kl + ((u & 2) ? 4 : 0);
                            const bool use = ((u & 1) ? rel1 : rel0) == kind;
                            float x0, x1;
                            if (XSIDE) {
                                x0 = GS0[(m0 + r) * GP + kk];
                                x1 = GS1[(m0 + r) * GP + kk];
                            } else {
                                x0 = GS0[kk * GP + m0 + r];
                                x1 = GS1[kk * GP + m0 + r];
                            }
                            av0[u] = use ? x0 : 0.f;
                            av1[u] = use ? x1 : 0.f;
                        }
                        const float* B0 = kind == 1 ? ZH0 : ZO0;
                        const float* B1 = kind == 1 ? ZH1 : ZO1;
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            float tmp[4] = {0.f, 0.f, 0.f, 0.f};
                            const float b0[2] = {B0[kl * OP + 8 * n + g], B0[(kl + 4) * OP + 8 * n + g]};
                            const float b1[2] = {B1[kl * OP + 8 * n + g], B1[(kl + 4) * OP + 8 * n + g]};
                            mma_f<PASSES>(tmp, av0, b0);
                            mma_f<PASSES>(tmp, av1, b1);
                            if (kind == 2) {
#pragma unroll
                                for (int u = 0; u < 4; ++u) dia[a][n][u] += tmp[u];
                            } else {
#pragma unroll
                                for (int u = 0; u < 4; ++u) {
                                    const int rb = u < 2 ? rb0 : rb1;
                                    const int col = 8 * n + 2 * cq + (u & 1);
                                    const size_t fi = XSIDE ? ((size_t)rb * nb8 + B8) : ((size_t)B8 * nb8 + rb);
                                    const float fv = ((u < 2) ? rel0 : rel1) == 1 ? FS[fi * CH + col] : 0.f;
                                    off[a][n][u] += fv * tmp[u];
                                }
                            }
                        }
                    }
                }
            }
        }
        // output-side pivot factors and the epilogue
#pragma unroll
        for (int a = 0; a < RB; ++a) {
            const int I16 = warp + 8 * a;
            if (I16 >= nb16) break;
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int row = 16 * I16 + g + (u < 2 ? 0 : 8);
                    const int col = j0 + 8 * n + 2 * cq + (u & 1);
                    const float fo = fexp<Tin>(XSIDE ? f.lx8(row, col) : f.lz8(row, col));
                    const float fd = fexp<Tin>(XSIDE ? f.lxo(row, col) : f.lzo(row, col));
                    epi(row, col, fo * off[a][n][u] + fd * dia[a][n][u]);
                }
        }
    }
    __syncthreads();
}

template <typename Tin, int D, int PASSES, bool XSIDE, int op0, int op1, class EPI>
__device__ __forceinline__ void decayed_grad_any(const Chunk<Tin, D>& c, float* sm, size_t G0,
                                                 size_t G1, const EPI& epi) {
    if (c.L.C > 128)
        decayed_grad_s<Tin, D, PASSES, XSIDE, 16, 32, 2, op0, op1>(c, sm, G0, G1, epi);
    else
        decayed_grad_s<Tin, D, PASSES, XSIDE, 32, 32, 1, op0, op1>(c, sm, G0, G1, epi);
}

// ------------------------------------------------------------------ triangular solves

__host__ __device__ constexpr int solve_smem_floats(int C, int D) {
    return C * (D + 4) + 16 * (C + 4) + C * 16;
}

// Solve (I + L) X = R in place (REV: (I + L)^T X = R).  X (global scratch,
// C x D) is held in shared memory for the whole solve; each step stages one
// 16-row block (or 16-column block, REV) of L; each warp owns D/8 columns.
template <int D, int PASSES, bool REV>
__device__ void solve_s(float* s, float* sm, const Lay& L, size_t Loff, size_t Xoff) {
    constexpr int XP = D + 4;
    const int C = L.C, nb16 = L.nb16;
    const int LP = C + 4;
    float* XS = sm;
    float* LS = XS + C * XP;
    float* TS = LS + 16 * LP;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, cq = lane & 3;
    constexpr int NT = D / 64;  // n8 tiles per warp
    const int c0 = warp * (D / 8);
    __syncthreads();
    for (int base = 0; base < C * D / 4; base += 4 * kThreads) {
        float4 v[4];
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int idx = base + threadIdx.x + it * kThreads;
            if (idx < C * D / 4) v[it] = *reinterpret_cast<const float4*>(s + Xoff + (size_t)4 * idx);
        }
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int idx = base + threadIdx.x + it * kThreads;
            if (idx >= C * D / 4) break;
            const int t = idx / (D / 4), j = 4 * (idx % (D / 4));
            XS[t * XP + j] = v[it].x; XS[t * XP + j + 1] = v[it].y;
            XS[t * XP + j + 2] = v[it].z; XS[t * XP + j + 3] = v[it].w;
        }
    }
    for (int idx = threadIdx.x; idx < C * 16; idx += kThreads) TS[idx] = s[L.TII + idx];
    for (int step = 0; step < nb16; ++step) {
        const int I = REV ? nb16 - 1 - step : step;
        __syncthreads();
        // stage L block: forward -> rows 16I.. (cols [0,16I)); reverse -> cols 16I.. (rows (16I+16, C))
        {
            // forward: rows 16I.. and columns [0, 16I); reverse: LS[r][k] = L[r1 + k][16I + r]
            const int r1 = 16 * (I + 1);
            const int n = REV ? 16 * (C - r1) : 16 * 16 * I;
            for (int base = 0; base < n; base += 4 * kThreads) {
                float v[4];
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const int idx = base + threadIdx.x + it * kThreads;
                    v[it] = 0.f;
                    if (idx < n) {
                        if (!REV) v[it] = s[Loff + (size_t)(16 * I + idx / (16 * I)) * C + idx % (16 * I)];
                        else v[it] = s[Loff + (size_t)(r1 + idx / 16) * C + 16 * I + idx % 16];
                    }
                }
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const int idx = base + threadIdx.x + it * kThreads;
                    if (idx >= n) break;
                    if (!REV) LS[(idx / (16 * I)) * LP + idx % (16 * I)] = v[it];
                    else LS[(idx % 16) * LP + idx / 16] = v[it];
                }
            }
        }
        __syncthreads();
        const int kb = REV ? 16 * (I + 1) : 0, ke = REV ? C : 16 * I;
        float acc[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[n][u] = 0.f;
        for (int k = kb; k < ke; k += 8) {
            const int kk = k - kb + cq;
            const float a[4] = {LS[g * LP + kk], LS[(g + 8) * LP + kk], LS[g * LP + kk + 4],
                                LS[(g + 8) * LP + kk + 4]};
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const float b[2] = {XS[(k + cq) * XP + c0 + 8 * n + g], XS[(k + cq + 4) * XP + c0 + 8 * n + g]};
                mma_f<PASSES>(acc[n], a, b);
            }
        }
        // R_I -= acc (in place), then X_I = T_II R_I (or T_II^T R_I)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int r = 16 * I + g + (u < 2 ? 0 : 8), col = c0 + 8 * n + 2 * cq + (u & 1);
                XS[r * XP + col] -= acc[n][u];
            }
        __syncwarp();
        float out[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int u = 0; u < 4; ++u) out[n][u] = 0.f;
        for (int k = 0; k < 16; k += 8) {
            const int kk = k + cq;
            float a[4];
            if (!REV) {
                a[0] = TS[(I * 16 + g) * 16 + kk];     a[1] = TS[(I * 16 + g + 8) * 16 + kk];
                a[2] = TS[(I * 16 + g) * 16 + kk + 4]; a[3] = TS[(I * 16 + g + 8) * 16 + kk + 4];
            } else {
                a[0] = TS[(I * 16 + kk) * 16 + g];     a[1] = TS[(I * 16 + kk) * 16 + g + 8];
                a[2] = TS[(I * 16 + kk + 4) * 16 + g]; a[3] = TS[(I * 16 + kk + 4) * 16 + g + 8];
            }
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const float b[2] = {XS[(16 * I + kk) * XP + c0 + 8 * n + g], XS[(16 * I + kk + 4) * XP + c0 + 8 * n + g]};
                mma_f<PASSES>(out[n], a, b);
            }
        }
        __syncwarp();
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int r = 16 * I + g + (u < 2 ? 0 : 8), col = c0 + 8 * n + 2 * cq + (u & 1);
                XS[r * XP + col] = out[n][u];
            }
        __syncwarp();
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < C * D / 4; idx += kThreads) {
        const int t = idx / (D / 4), j = 4 * (idx % (D / 4));
        float4 v;
        v.x = XS[t * XP + j]; v.y = XS[t * XP + j + 1]; v.z = XS[t * XP + j + 2]; v.w = XS[t * XP + j + 3];
        *reinterpret_cast<float4*>(s + Xoff + (size_t)t * D + j) = v;
    }
    __syncthreads();
}



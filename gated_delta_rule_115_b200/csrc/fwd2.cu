// fwd2.cu -- chunkwise forward on the 5th-generation tensor cores with every
// per-chunk intermediate held in shared memory and tensor memory.
//
// Scope: bf16 inputs, dk = dv = 128, chunk C = 128, T a multiple of 128, and
// chunks whose per-channel log decay over the chunk stays within the
// single-pivot range (|sum g| <= 140; k2_intra raises a device flag for a
// chunk beyond it, and the call then also runs the 8-token boundary-pivot path
// of chunk_impl.cuh, whose results replace these).
//
// Per chunk (wolonglab.org page, "Methodology": each chunk is a unit-lower-
// triangular system; fig:kernel: fused right-hand side, block inversion on the
// matrix unit), with L = chunk-local cumulative log decay (log2 units inside),
// P = L_C / 2 the per-channel pivot, q^ = gamma*q, a = e*k, u = w*v:
//
//   Kp = k 2^(L-P), Km = k 2^(P-L), Am = a 2^(P-L), Qp = q^ 2^(L-P)
//   L_A = strict(Kp Am^T), L_K = strict(Kp Km^T)           (bf16 operands)
//   M_QK = incl(Qp Km^T)  (bf16 hi/lo split: hi hi + hi lo + lo hi)
//   M_QA = incl(Qp Am^T)                      (Qp as bf16 hi + lo, Am bf16)
//   T = (I + L_A)^-1: 32x32 diagonal blocks by forward substitution (fp32),
//       then block merges T21 = -T22 (L21 T11) for 32 -> 64 -> 128 on tcgen05
//   X = [W | U'] = T [K~ | L_K U]   (K~ = k 2^L; one N = 256 MMA chain)
//   Z = [Q' | O_intra] = [Q~ | M_QK U] - M_QA X              (Q~ = q^ 2^L)
//   [M_n | B_n] = [diag(2^Lbar) | Kbar^T U] - Abar^T X       (Kbar = k 2^(Lbar-L), Abar = a 2^(Lbar-L))
//
// so that the chunk's output is O_n = Q'_n S_n + O_intra_n and the state
// passes as S_{n+1} = M_n S_n + B_n (k2_chain, then k2_out).  Bounded-range
// operands (T, U, L_K, L_K U, K~, X, M_QK, M_QA, Kbar, Abar) are fp16; the
// pivoted ones span up to 2^+-101 and are bf16.  Accumulation is fp32 in TMEM.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bwd2.h"
#include "fwd2.h"
#include "profile.h"
#include "tc2.cuh"

namespace muir {
namespace v2 {

using namespace t2;

constexpr int kC = 128, kD = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLogDecayMin = -20.f;      // per-token clamp of g (natural log units)
constexpr float kSpanMax = 140.f;          // single-pivot limit of |sum g| over a chunk

__device__ unsigned int g_v2_timeouts;

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Rotate a 32-entry register array left by 8: after four calls it is back in
// order.  Lets a rolled loop over four 8-column chunks use L[0..7] with
// compile-time indices (the array stays in registers).
__device__ __forceinline__ void rot8(float (&L)[32]) {
    float t[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) t[u] = L[u];
#pragma unroll
    for (int j = 0; j < 24; ++j) L[j] = L[j + 8];
#pragma unroll
    for (int u = 0; u < 8; ++u) L[24 + u] = t[u];
}

__device__ __forceinline__ void bf16_split(float x, float& hi, float& lo) {
    hi = __bfloat162float(__float2bfloat16_rn(x));
    lo = x - hi;
}

// ------------------------------------------------------------------ k2_intra

struct IntraSmem {
    alignas(16) float P2[kD];   // pivot (log2 units)
    alignas(16) float eP2[kD];  // 2^P2
    alignas(16) float Lb[kD];   // chunk total (log2 units)
    alignas(16) float lblk[4][32][36];  // strictly lower 32x32 diagonal blocks of L_A (leaf inverses)
    float nrm[4][kC];   // fused prologue: per-quarter sums of SiLU(x)^2 of each row
    uint64_t bar[16];
    uint32_t tslot;
    int bad;
};

enum { BA = 0, BB, BC, BD, BE, BF, BM1, BM2, BM3, BM4, BM5, BM6, BG, BL };

// 8 consecutive floats of a shared-memory table (32-byte aligned) in two 16-byte loads.
__device__ __forceinline__ void lds8(const float* p, float* v) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// All threads call: warp 0 polls, the block barrier releases the rest.
__device__ __forceinline__ bool waitb(IntraSmem& s, int i, uint32_t parity) {
    const bool ok = cta_wait(&s.bar[i], parity);
    if (!ok && threadIdx.x == 0) s.bad = 1;
    return ok;
}

__device__ __forceinline__ void sync_all() {
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
}

// Fused q/k prologue: x -> SiLU(x) r with r the row's inverse norm.
__device__ __forceinline__ void prologue8(float* v, float r) {
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = v[u] * sigmoid_f(v[u]) * r;
}

// Sum of SiLU(x)^2 over this thread's 32 columns of row t of a raw tile.
__device__ __forceinline__ float silu_sq32(const unsigned char* tile, int t, int h) {
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float v[8];
        ld_chunk16<true>(tile, t, 4 * h + i, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float sv = v[u] * sigmoid_f(v[u]);
            acc = fmaf(sv, sv, acc);
        }
    }
    return acc;
}

// Inverse row norm from the four quarter sums (the guard maps a zero row to zero).
__device__ __forceinline__ float row_rnorm(const float (*nrm)[kC], int t) {
    return rsqrtf(fmaxf(((nrm[0][t] + nrm[1][t]) + nrm[2][t]) + nrm[3][t], 1e-24f));
}

// Load 64 values (this thread's row t, columns 64h..64h+63) of a bf16 T16 tile.
__device__ __forceinline__ void row_ld64(const unsigned char* tile, int t, int h, float* v) {
#pragma unroll
    for (int i = 0; i < 8; ++i) ld_chunk16<true>(tile, t, 8 * h + i, v + 8 * i);
}

template <bool BF16>
__device__ __forceinline__ void row_st64(unsigned char* tile, int t, int h, const float* v) {
#pragma unroll
    for (int i = 0; i < 8; ++i) st_chunk16<BF16>(tile, t, 8 * h + i, v + 8 * i);
}

// Store 32 values at columns 32 * c32 .. +32 of row t.
template <bool BF16>
__device__ __forceinline__ void row_st32(unsigned char* tile, int t, int c32, const float* v) {
#pragma unroll
    for (int i = 0; i < 4; ++i) st_chunk16<BF16>(tile, t, 4 * c32 + i, v + 8 * i);
}

// TMEM columns [col, col + 32) of this thread's lane, waited.
__device__ __forceinline__ void tm_ld32w(uint32_t tm, int q, int col, float (&v)[32]) {
    tmem_ld32(taddr(tm, 32 * q, col), v);
    tmem_wait_ld();
}

// Copy 64 TMEM columns (this thread's half h of the 128 columns at tm + base)
// into row t of a fp16 tile, 32 at a time; mask(col) decides which survive.
template <class MASK>
__device__ __forceinline__ void tm_to_tile(uint32_t tm, int base, int q, int h, int t,
                                           unsigned char* tile, const MASK& mask) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float v[32];
        tm_ld32w(tm, q, base + 64 * h + 32 * hh, v);
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (!mask(64 * h + 32 * hh + j)) v[j] = 0.f;
        row_st32<false>(tile, t, 2 * h + hh, v);
    }
}

// Read 64 TMEM columns [col, col + 64) of this thread's lane.
__device__ __forceinline__ void tm_ld64(uint32_t tm, int q, int col, float* v) {
    float a[32], b[32];
    tmem_ld32(taddr(tm, 32 * q, col), a);
    tmem_ld32(taddr(tm, 32 * q, col + 32), b);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) { v[i] = a[i]; v[32 + i] = b[i]; }
}

// 512 threads: warp w owns rows 32 (w % 4) .. +32 (its TMEM lane quarter q) and
// columns 32 (w / 4) .. +32 (h); thread t = 32 q + lane owns row t of every
// per-chunk tile in those columns.  Thread 0 issues the TMA loads and the MMAs.
template <bool QKRAW>
__global__ void __launch_bounds__(512, 1) k2_intra(const __grid_constant__ IntraParams p) {
    extern __shared__ __align__(1024) unsigned char smraw[];
    unsigned char* sm = (unsigned char*)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    unsigned char* S[6];
#pragma unroll
    for (int i = 0; i < 6; ++i) S[i] = sm + i * kT16Bytes;
    IntraSmem& s = *reinterpret_cast<IntraSmem*>(sm + 6 * kT16Bytes);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, h = warp >> 2;
    const int t = 32 * q + lane;  // row owned by this thread
    const int c0 = 32 * h;        // first of its 32 columns
    const int N = p.T / kC;
    const int nch = p.B * p.H * N;

    if (tid == 0) {
        for (int i = 0; i < 16; ++i) mbar_init(&s.bar[i], 1);
        s.bad = 0;
        fence_barrier_init();
        prefetch_tmap(&p.tq); prefetch_tmap(&p.tk); prefetch_tmap(&p.tv); prefetch_tmap(&p.tg);
        prefetch_tmap(&p.te); prefetch_tmap(&p.tw); prefetch_tmap(&p.tgam);
    }
    if (warp == 0) tmem_alloc(&s.tslot, 512);
    sync_all();
    const uint32_t tm = s.tslot;
    const uint32_t a0 = saddr(S[0]), a1 = saddr(S[1]), a2 = saddr(S[2]), a3 = saddr(S[3]),
                   a4 = saddr(S[4]), a5 = saddr(S[5]);

    auto coords = [&](int c, int& y, int& z) {
        const int n = c % N, bh = c / N;
        y = bh % p.H;
        z = (bh / p.H) * p.T + n * kC;
    };
    auto load_tile = [&](unsigned char* dst, const CUtensorMap* map, int y, int z, int bar) {
        tma_load_3d(dst, map, 0, y, z, &s.bar[bar]);
        tma_load_3d(dst + kT16Block, map, 64, y, z, &s.bar[bar]);
    };
    // g, k, e on BA; q, gamma on BB.  Past the first chunk gamma is issued by
    // the chunk itself, once the previous chunk's M tile has left S4.
    auto issue_first = [&](int c, bool with_gamma) {
        int y, z;
        coords(c, y, z);
        mbar_arrive_expect_tx(&s.bar[BA], 3 * kT16Bytes);
        load_tile(S[0], &p.tg, y, z, BA);
        load_tile(S[1], &p.tk, y, z, BA);
        load_tile(S[2], &p.te, y, z, BA);
        mbar_arrive_expect_tx(&s.bar[BB], 2 * kT16Bytes);
        load_tile(S[3], &p.tq, y, z, BB);
        if (with_gamma) load_tile(S[4], &p.tgam, y, z, BB);
    };
    // this thread's 4 chunks of 8 columns: chunk index 4h + i
    auto ld32 = [&](const unsigned char* tile, float* v) {
#pragma unroll
        for (int i = 0; i < 4; ++i) ld_chunk16<true>(tile, t, 4 * h + i, v + 8 * i);
    };
    // TMEM columns base + c0 .. +32 of row t -> fp16 tile, masked by keep(col)
    auto tm_to_row = [&](int base, unsigned char* tile, auto keep) {
        float v[32];
        tm_ld32w(tm, q, base + c0, v);
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (!keep(c0 + j)) v[j] = 0.f;
        row_st32<false>(tile, t, h, v);
    };
    if (tid == 0 && (int)blockIdx.x < nch) issue_first(blockIdx.x, true);

    int it = 0;
    for (int c = blockIdx.x; c < nch; c += gridDim.x, ++it) {
        const uint32_t ph = (uint32_t)(it & 1);
        uint32_t pg = 0;  // parity of the merge barrier within this chunk
        int y, z;
        coords(c, y, z);

        if (tid == 0 && it > 0) {  // the previous chunk's M tile has left S4 and S5 (the wait below tells the rest)
            bulk_wait_read();
            load_tile(S[4], &p.tgam, y, z, BB);
        }
        // ---- 1. log-decay prefix, pivots
        // L = Tril(1) g: the inclusive prefix over the chunk's tokens as one
        // tensor-core product (clamped g and the ones are exact in bf16; fp32
        // accumulation), the ones tile in S5 (free until phase 2)
        waitb(s, BA, ph);
        {
            float v[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                ld_chunk16<true>(S[0], t, 4 * h + i, v);
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = fmaxf(v[u], kLogDecayMin);
                st_chunk16<true>(S[0], t, 4 * h + i, v);
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = (c0 + 8 * i + u <= t) ? 1.f : 0.f;
                st_chunk16<true>(S[5], t, 4 * h + i, v);
            }
        }
        if (QKRAW) s.nrm[h][t] = silu_sq32(S[1], t, h);
        fence_async_smem();
        sync_all();
        if (tid == 0) {
            gemm_km16(tm + 0, a5, 0, a0, 0, 0, 128, 128, kBF16, false);
            mma_commit(&s.bar[BL]);
        }
        const float rk = QKRAW ? row_rnorm(s.nrm, t) : 1.f;
        if (QKRAW && h == 0) p.rnorm[(size_t)c * 2 * kC + kC + t] = rk;
        waitb(s, BL, ph);
        float L[32];
        tm_ld32w(tm, q, c0, L);
#pragma unroll
        for (int j = 0; j < 32; ++j) L[j] *= kLog2e;
        if (t == kC - 1) {  // the chunk totals: the last row
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                s.Lb[c0 + j] = L[j];
                s.P2[c0 + j] = 0.5f * L[j];
                s.eP2[c0 + j] = ex2(0.5f * L[j]);
            }
            bool far = false;
#pragma unroll
            for (int j = 0; j < 32; ++j) far |= L[j] < -kSpanMax * kLog2e;
            // a span beyond the single pivot sends the call to the boundary-pivot path
            if (far) atomicOr(p.flags, 1);
        }
        sync_all();

        // ---- 2. pivoted key operands: Kp -> S0, Km (hi) -> S1, Km (lo) -> S2, Am -> S5
#pragma unroll 1
        for (int i = 0; i < 4; ++i, rot8(L)) {
            float kv[8], ev[8], kp[8], kmh[8], kml[8], am[8];
            ld_chunk16<true>(S[1], t, 4 * h + i, kv);
            if (QKRAW) prologue8(kv, rk);
            ld_chunk16<true>(S[2], t, 4 * h + i, ev);
            float pv8[8];
            lds8(&s.P2[c0 + 8 * i], pv8);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float pv = pv8[u];
                const float ep = ex2(L[u] - pv), em = ex2(pv - L[u]);
                kp[u] = kv[u] * ep;
                bf16_split(kv[u] * em, kmh[u], kml[u]);
                am[u] = ev[u] * kv[u] * em;
            }
            st_chunk16<true>(S[0], t, 4 * h + i, kp);
            st_chunk16<true>(S[1], t, 4 * h + i, kmh);
            st_chunk16<true>(S[2], t, 4 * h + i, kml);
            st_chunk16<true>(S[5], t, 4 * h + i, am);
        }
        fence_async_smem();
        sync_all();
        if (tid == 0) {
            gemm_kk16(tm + 0, a0, 0, a5, 0, 0, 128, 128, kBF16, false);    // L_A
            gemm_kk16(tm + 128, a0, 0, a1, 0, 0, 128, 128, kBF16, false);  // L_K
            mma_commit(&s.bar[BM1]);
        }

        // ---- 3. query operands: Qp hi -> S3, Qp lo -> S4
        waitb(s, BB, ph);
        float rq = 1.f;
        if (QKRAW) {  // (the barrier of the wait above ordered the reads of nrm for k)
            s.nrm[h][t] = silu_sq32(S[3], t, h);
            __syncthreads();
            rq = row_rnorm(s.nrm, t);
            if (h == 0) p.rnorm[(size_t)c * 2 * kC + t] = rq;
        }
#pragma unroll 1
        for (int i = 0; i < 4; ++i, rot8(L)) {
            float qv[8], gv[8], qh[8], ql[8];
            ld_chunk16<true>(S[3], t, 4 * h + i, qv);
            if (QKRAW) prologue8(qv, rq);
            ld_chunk16<true>(S[4], t, 4 * h + i, gv);
            float pv8[8];
            lds8(&s.P2[c0 + 8 * i], pv8);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float pv = pv8[u];
                bf16_split(qv[u] * gv[u] * ex2(L[u] - pv), qh[u], ql[u]);
            }
            st_chunk16<true>(S[3], t, 4 * h + i, qh);
            st_chunk16<true>(S[4], t, 4 * h + i, ql);
        }
        fence_async_smem();
        sync_all();
        if (tid == 0) {
            gemm_kk16(tm + 256, a3, 0, a1, 0, 0, 128, 128, kBF16, false);  // M_QK: hi hi
            gemm_kk16(tm + 256, a3, 0, a2, 0, 0, 128, 128, kBF16, true);   //       hi lo
            gemm_kk16(tm + 256, a4, 0, a1, 0, 0, 128, 128, kBF16, true);   //       lo hi
            gemm_kk16(tm + 384, a3, 0, a5, 0, 0, 128, 128, kBF16, false);  // M_QA: hi Am
            gemm_kk16(tm + 384, a4, 0, a5, 0, 0, 128, 128, kBF16, true);   //       lo Am
            mma_commit(&s.bar[BM2]);
        }

        // ---- 4. L_A -> LA16 (S0), leaves of T (32 x 32 diagonal blocks), L_K -> LK16 (S1)
        waitb(s, BM1, ph);
        tc_fence_after();
        const bool leaf = (h == q);  // warp (q, q) holds L_A[32q + lane][32q .. 32q + 31]
        {
            float la[32];
            tm_ld32w(tm, q, c0, la);
            if (leaf) {  // row lane of the block (rows 144 bytes apart: 16-byte stores without conflicts)
#pragma unroll
                for (int k = 0; k < 32; k += 4)
                    *reinterpret_cast<float4*>(&s.lblk[q][lane][k]) =
                        make_float4(k < lane ? la[k] : 0.f, k + 1 < lane ? la[k + 1] : 0.f,
                                    k + 2 < lane ? la[k + 2] : 0.f, k + 3 < lane ? la[k + 3] : 0.f);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (c0 + j >= t) la[j] = 0.f;
            row_st32<false>(S[0], t, h, la);
        }
        waitb(s, BM2, ph);  // S1..S5 free
        tc_fence_after();
        tm_to_row(128, S[1], [&](int col) { return col < t; });
        // T (S2): zeros outside the diagonal blocks, leaves written column-wise
        if (!leaf) {
            float z8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 4; ++i) st_chunk16<false>(S[2], t, 4 * h + i, z8);
        } else {
            // lane = column c of the block; tcol[r] = T[r][c] by forward substitution
            float tcol[32];
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                float acc = (r == lane) ? 1.f : 0.f;
#pragma unroll
                for (int k4 = 0; k4 < r; k4 += 4) {  // row r of L, four entries per (broadcast) load
                    const float4 l4 = *reinterpret_cast<const float4*>(&s.lblk[q][r][k4]);
                    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (k4 + u < r) acc -= lv[u] * tcol[k4 + u];
                }
                tcol[r] = acc;
            }
            const int col = c0 + lane;
#pragma unroll
            for (int r = 0; r < 32; ++r)
                *reinterpret_cast<__half*>(S[2] + t16_off(32 * q + r, col >> 3) + (col & 7) * 2) =
                    __float2half_rn(tcol[r]);
        }
        if (tid == 0) {  // v -> S4, w -> S5
            mbar_arrive_expect_tx(&s.bar[BC], 2 * kT16Bytes);
            load_tile(S[4], &p.tv, y, z, BC);
            load_tile(S[5], &p.tw, y, z, BC);
        }
        fence_async_smem();
        sync_all();

        // ---- 5. block merges of T on tcgen05: P = L21 T11 (into B0), T21 = -T22 P (into B1)
        unsigned char* ax = p.aux ? p.aux + (size_t)c * AuxLayout::kBytes : nullptr;
        if (ax && tid == 0) {  // L_K (S1) is final
            bulk_store(ax + AuxLayout::kLK16, S[1], kT16Bytes);
            bulk_commit();
        }
#pragma unroll 1
        for (int lvl = 0; lvl < 2; ++lvl) {
            const int b = lvl == 0 ? 32 : 64;
            if (tid == 0) {
                for (int pr = 0; pr < 128 / (2 * b); ++pr) {
                    const int F = 2 * b * pr;
                    gemm_km16(tm + F, a0, F, a2, F, F, b, b, kF16, false);
                }
                mma_commit(&s.bar[BG]);
            }
            waitb(s, BG, pg); pg ^= 1;
            tc_fence_after();
            // second-half rows of each pair and the pair's first-half columns:
            // level 32: quarters 1 and 3, columns 0..31 / 64..95; level 64: quarters 2, 3, columns 0..63
            const bool mine = (lvl == 0) ? ((q & 1) && h == 2 * (q >> 1)) : (q >= 2 && h < 2);
            if (mine) {
                float a[32];
                tm_ld32w(tm, q, c0, a);
                row_st32<false>(S[3], t, h, a);
            }
            fence_async_smem();
            sync_all();
            if (tid == 0) {
                for (int pr = 0; pr < 128 / (2 * b); ++pr) {
                    const int F2 = 2 * b * pr;
                    gemm_km16(tm + 128 + F2, a2, F2 + b, a3, F2 + b, F2, b, b, kF16, false, true);
                }
                mma_commit(&s.bar[BG]);
            }
            waitb(s, BG, pg); pg ^= 1;
            tc_fence_after();
            if (mine) {
                float a[32];
                tm_ld32w(tm + 128, q, c0, a);
                row_st32<false>(S[2], t, h, a);
            }
            fence_async_smem();
            sync_all();
        }
        if (tid == 0) {  // k -> S0 (L_A consumed by the merges) for K~ in phase 6
            mbar_arrive_expect_tx(&s.bar[BD], kT16Bytes);
            load_tile(S[0], &p.tk, y, z, BD);
        }

        if (ax && tid == 0) {  // T (S2) is final
            bulk_store(ax + AuxLayout::kT16, S[2], kT16Bytes);
            bulk_commit();
        }
        // ---- 6. U = w v (S4, in place); L_K U (B0); K~ (S0); X = T [K~ | L_K U] (B0..B1)
        waitb(s, BC, ph);
#pragma unroll 1
        for (int i = 0; i < 4; ++i) {
            float vv[8], wv[8];
            ld_chunk16<true>(S[4], t, 4 * h + i, vv);
            ld_chunk16<true>(S[5], t, 4 * h + i, wv);
#pragma unroll
            for (int u = 0; u < 8; ++u) vv[u] *= wv[u];
            st_chunk16<false>(S[4], t, 4 * h + i, vv);
        }
        fence_async_smem();
        sync_all();
        if (ax && tid == 0) {  // U (S4) is final; L_K's record has left S1 (overwritten below)
            bulk_wait_read();
            bulk_store(ax + AuxLayout::kU16, S[4], kT16Bytes);
            bulk_commit();
        }
        if (tid == 0) {
            gemm_km16(tm + 0, a1, 0, a4, 0, 0, 128, 128, kF16, false);  // L_K U
            mma_commit(&s.bar[BM3]);
        }
        waitb(s, BD, ph);
#pragma unroll 1
        for (int i = 0; i < 4; ++i, rot8(L)) {
            float kv[8];
            ld_chunk16<true>(S[0], t, 4 * h + i, kv);
            if (QKRAW) prologue8(kv, rk);
#pragma unroll
            for (int u = 0; u < 8; ++u) kv[u] *= ex2(L[u]);
            st_chunk16<false>(S[0], t, 4 * h + i, kv);
        }
        waitb(s, BM3, ph);
        tc_fence_after();
        tm_to_row(0, S[1], [](int) { return true; });
        fence_async_smem();
        sync_all();
        if (tid == 0) {
            gemm_km16(tm + 0, a2, 0, a0, 0, 0, 256, 128, kF16, false);  // X = T [K~ | L_K U]
            mma_commit(&s.bar[BM4]);
        }
        // M_QK (B2) -> S3, M_QA (B3) -> S5 (inclusive masks)
        tm_to_row(256, S[3], [&](int col) { return col <= t; });
        tm_to_row(384, S[5], [&](int col) { return col <= t; });
        waitb(s, BM4, ph);
        tc_fence_after();
        if (tid == 0) {  // k -> S2 (T consumed by X; its record stored) for Kbar in phase 7
            if (ax) bulk_wait_read();
            mbar_arrive_expect_tx(&s.bar[BE], kT16Bytes);
            load_tile(S[2], &p.tk, y, z, BE);
        }
        {
            float v[32];
            tm_ld32w(tm, q, c0, v);  // W
            row_st32<false>(S[0], t, h, v);
            tm_ld32w(tm, q, 128 + c0, v);  // U'
            row_st32<false>(S[1], t, h, v);
            if (ax) {
                float* ub = reinterpret_cast<float*>(ax + AuxLayout::kUp);
#pragma unroll
                for (int j = 0; j < 32; j += 4) *grp4(ub, t, c0 + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
            }
        }
        fence_async_smem();
        sync_all();
        if (ax && tid == 0) {  // M_QK (S3), M_QA (S5), W (S0) are final
            bulk_store(ax + AuxLayout::kMQK16, S[3], kT16Bytes);
            bulk_store(ax + AuxLayout::kMQA16, S[5], kT16Bytes);
            bulk_store(ax + AuxLayout::kW16, S[0], kT16Bytes);
            bulk_commit();
        }

        // ---- 7. Z = [Q~ | M_QK U] - M_QA [W | U'] (B2..B3)
        if (tid == 0) {
            gemm_km16(tm + 256, a5, 0, a0, 0, 0, 256, 128, kF16, false, true);
            gemm_km16(tm + 384, a3, 0, a4, 0, 0, 128, 128, kF16, true);
            mma_commit(&s.bar[BM5]);
        }
        // q and gamma of row t for Q~, requested while the products run
        uint4 qraw[4], graw[4];
        {
            const size_t ri = (((size_t)(c / N / p.H) * p.T + (size_t)(c % N) * kC + t) * p.H + y) * kD + c0;
            const __nv_bfloat16* qsrc = reinterpret_cast<const __nv_bfloat16*>(p.q) + ri;
            const __nv_bfloat16* gsrc = reinterpret_cast<const __nv_bfloat16*>(p.gamma) + ri;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                qraw[i] = __ldg(reinterpret_cast<const uint4*>(qsrc + 8 * i));
                graw[i] = __ldg(reinterpret_cast<const uint4*>(gsrc + 8 * i));
            }
        }
        waitb(s, BM5, ph);
        tc_fence_after();
        if (tid == 0) {
            if (ax) bulk_wait_read();                      // M_QK's record has left S3
            mbar_arrive_expect_tx(&s.bar[BF], kT16Bytes);  // e -> S3
            load_tile(S[3], &p.te, y, z, BF);
        }
        {
            // Q' = Q~ - M_QA W with Q~ = gamma q 2^L from the bf16 inputs
            float v[32];
            tm_ld32w(tm + 256, q, c0, v);
            float* qb = p.Qp + (size_t)c * kC * kD;
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
                const uint4 qw = qraw[j >> 3];
                const uint4 gw = graw[j >> 3];
                const uint32_t qa[4] = {qw.x, qw.y, qw.z, qw.w}, ga[4] = {gw.x, gw.y, gw.z, gw.w};
                float r[8];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float q0, q1, g0, g1;
                    unpack16<true>(qa[u], q0, q1);
                    unpack16<true>(ga[u], g0, g1);
                    if (QKRAW) {
                        q0 = q0 * sigmoid_f(q0) * rq;
                        q1 = q1 * sigmoid_f(q1) * rq;
                    }
                    r[2 * u] = v[j + 2 * u] + q0 * g0 * ex2(L[j + 2 * u]);
                    r[2 * u + 1] = v[j + 2 * u + 1] + q1 * g1 * ex2(L[j + 2 * u + 1]);
                }
                *grp4(qb, t, c0 + j) = make_float4(r[0], r[1], r[2], r[3]);
                *grp4(qb, t, c0 + j + 4) = make_float4(r[4], r[5], r[6], r[7]);
            }
            tm_ld32w(tm + 384, q, c0, v);
            float* ob = p.Oi + (size_t)c * kC * kD;
#pragma unroll
            for (int j = 0; j < 32; j += 4) *grp4(ob, t, c0 + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        }
        waitb(s, BE, ph);
        waitb(s, BF, ph);
#pragma unroll 1
        for (int i = 0; i < 4; ++i, rot8(L)) {
            float kv[8], ev[8];
            ld_chunk16<true>(S[2], t, 4 * h + i, kv);
            if (QKRAW) prologue8(kv, rk);
            ld_chunk16<true>(S[3], t, 4 * h + i, ev);
            float p8[8], e8[8];
            lds8(&s.P2[c0 + 8 * i], p8);
            lds8(&s.eP2[c0 + 8 * i], e8);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float f = ex2(p8[u] - L[u]) * e8[u];  // 2^(Lbar - L)
                kv[u] *= f;
                ev[u] *= kv[u];
            }
            st_chunk16<false>(S[2], t, 4 * h + i, kv);
            st_chunk16<false>(S[3], t, 4 * h + i, ev);

        }
        fence_async_smem();
        sync_all();

        // ---- 8. [M_n | B_n] = [diag 2^Lbar | Kbar^T U] - Abar^T [W | U'] (B0..B1)
        if (ax && tid == 0) {  // Kbar (S2), Abar (S3) are final
            bulk_store(ax + AuxLayout::kKbar16, S[2], kT16Bytes);
            bulk_store(ax + AuxLayout::kAbar16, S[3], kT16Bytes);
            bulk_commit();
        }
        if (tid == 0) {
            gemm_mm16(tm + 0, a3, 0, 0, a0, 0, 0, 256, 128, kF16, false, true);
            gemm_mm16(tm + 128, a2, 0, 0, a4, 0, 0, 128, 128, kF16, true);
            mma_commit(&s.bar[BM6]);
        }
        waitb(s, BM6, ph);
        tc_fence_after();
        const int cn = c + gridDim.x;
        if (tid == 0 && ax) bulk_wait_read();  // M_QA (S5) stored before S5 is reused
        if (tid == 0 && cn < nch) issue_first(cn, false);
        {
            float v[32];
            tm_ld32w(tm, q, c0, v);
            if (t >= c0 && t < c0 + 32) {
                const float dg = ex2(s.Lb[t]);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (c0 + j == t) v[j] += dg;
            }
            {  // M row t, columns c0 ..: 128B-swizzled fp32 box h of the tile in S4 | S5
                unsigned char* mb = (h < 2 ? S[4] : S[5]) + (h & 1) * 16384 + t * 128;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<float4*>(mb + ((i ^ (t & 7)) << 4)) =
                        make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
            if (p.Mt) {
                float* mt = p.Mt + (size_t)c * kC * kD + t;
#pragma unroll 8
                for (int j = 0; j < 32; ++j) mt[(size_t)(c0 + j) * kD] = v[j];
            }
            tm_ld32w(tm + 128, q, c0, v);
            float* bb = p.Bn + (size_t)c * kC * kD;
#pragma unroll
            for (int j = 0; j < 32; j += 4) *grp4(bb, t, c0 + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        }
        fence_async_smem();
        sync_all();  // TMEM read out before the next chunk's products; M tile complete
        if (tid == 0) {
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
                tma_store_3d(&p.tM, (kb < 2 ? S[4] : S[5]) + (kb & 1) * 16384, 32 * kb, c * kC, 0);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait_all();
    if (tid == 0 && s.bad) atomicAdd(&g_v2_timeouts, 1u);
    sync_all();
    if (warp == 0) tmem_dealloc(tm, 512);
}

// ------------------------------------------------------------------ k2_chain

// S_{n+1} = M_n S_n + B_n for one head and SLAB value columns; 128 threads,
// thread j owns row j.  M_n streams through a 3-stage TMA ring (K-major TF32
// tiles); S_n^T sits in a K-major TF32 tile of SLAB rows (the B operand).
// Records S_n (chunk-start states) and writes S_N to S_final.
template <int SLAB>
__global__ void __launch_bounds__(128, 1) k2_chain(const __grid_constant__ ChainParams p) {
    constexpr int STAGES = 3;
    constexpr uint32_t MT = 128 * 128 * 4;  // one transition tile
    extern __shared__ __align__(1024) unsigned char smraw[];
    unsigned char* sm = (unsigned char*)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    unsigned char* Mst = sm;                       // STAGES x 64 KB
    unsigned char* St = sm + STAGES * MT;          // SLAB x 128 fp32, K-major
    __shared__ uint64_t bar[STAGES + 1];
    __shared__ uint32_t tslot;
    __shared__ int bad;

    const int tid = threadIdx.x, warp = tid >> 5;
    const int nslab = kD / SLAB;
    const int bh = blockIdx.x / nslab, c0 = (blockIdx.x % nslab) * SLAB;
    const int N = p.N;
    const int j = tid;
    if (tid == 0) {
        for (int i = 0; i <= STAGES; ++i) mbar_init(&bar[i], 1);
        bad = 0;
        fence_barrier_init();
        prefetch_tmap(&p.tM);
    }
    if (warp == 0) tmem_alloc(&tslot, 32 < SLAB ? SLAB : 32);
    sync_all();
    const uint32_t tm = tslot;
    const long long row0 = (long long)bh * N * kD;  // first row of this head's transitions
    auto issue = [&](int n) {
        const int st = n % STAGES;
        mbar_arrive_expect_tx(&bar[st], MT);
        for (int kb = 0; kb < 4; ++kb)
            tma_load_3d(Mst + st * MT + kb * 128 * 128, &p.tM, 32 * kb, (int)(row0 + (long long)n * kD), 0,
                        &bar[st]);
    };
    if (tid == 0)
        for (int n = 0; n < STAGES && n < N; ++n) issue(n);

    // initial state row j, columns c0 .. c0 + SLAB
    float Sr[SLAB];
    const size_t sbase = ((size_t)bh * kD + j) * kD + c0;
#pragma unroll
    for (int c = 0; c < SLAB; ++c) Sr[c] = p.S0 ? p.S0[sbase + c] : 0.f;
    auto put_state = [&]() {
#pragma unroll
        for (int c = 0; c < SLAB; ++c)
            *reinterpret_cast<float*>(St + t32_off<SLAB>(c, j >> 2) + (j & 3) * 4) = Sr[c];
    };
    put_state();
    float Bnext[SLAB];
    auto load_B = [&](int n, float* dst) {
        const float* blk = p.Bn + ((size_t)bh * N + n) * kD * kD;
#pragma unroll
        for (int c = 0; c < SLAB; c += 4) {
            const float4 v = __ldg(grp4(blk, j, c0 + c));
            dst[c] = v.x; dst[c + 1] = v.y; dst[c + 2] = v.z; dst[c + 3] = v.w;
        }
    };
    if (N > 0) load_B(0, Bnext);
    fence_async_smem();
    sync_all();
    for (int n = 0; n < N; ++n) {
        const int st = n % STAGES;
        // only the issuing thread waits for the transition tile: it alone reads it
        // (through the MMA), and it reloads the stage later in this step, so a
        // second waiter could see the barrier two phases on and miss its phase
        if (tid == 0) {
            if (!mbar_wait(&bar[st], (uint32_t)((n / STAGES) & 1))) bad = 1;
            tc_fence_after();
            gemm_kk32<128, SLAB>(tm, saddr(Mst + st * MT), saddr(St), 0, SLAB, 128, false);
            mma_commit(&bar[STAGES]);
        }
        if (p.S_chunks) {  // record S_n while the product runs
            float* d = p.S_chunks + ((size_t)bh * N + n) * kD * kD + (size_t)j * kD + c0;
#pragma unroll
            for (int c = 0; c < SLAB; c += 4) *reinterpret_cast<float4*>(d + c) = make_float4(Sr[c], Sr[c + 1], Sr[c + 2], Sr[c + 3]);
        }
        float Bc[SLAB];
#pragma unroll
        for (int c = 0; c < SLAB; ++c) Bc[c] = Bnext[c];
        if (n + 1 < N) load_B(n + 1, Bnext);
        if (!cta_wait(&bar[STAGES], (uint32_t)(n & 1)) && tid == 0) bad = 1;
        if (tid == 0 && n + STAGES < N) issue(n + STAGES);
        float d[32];
        tmem_ld32(taddr(tm, 32 * warp, 0), d);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < SLAB; ++c) Sr[c] = d[c] + Bc[c];
        put_state();
        fence_async_smem();
        sync_all();
    }
    float* fin[2] = {p.S_final, p.S_last};
    for (int i = 0; i < 2; ++i) {
        if (!fin[i]) continue;
        float* d = fin[i] + sbase;
#pragma unroll
        for (int c = 0; c < SLAB; c += 4) *reinterpret_cast<float4*>(d + c) = make_float4(Sr[c], Sr[c + 1], Sr[c + 2], Sr[c + 3]);
    }
    if (tid == 0 && bad) atomicAdd(&g_v2_timeouts, 1u);
    sync_all();
    if (warp == 0) tmem_dealloc(tm, 32 < SLAB ? SLAB : 32);
}

// ------------------------------------------------------------------ k2_out

// O_n = Q'_n S_n + O_intra_n per chunk (TF32 products, fp32 accumulation).
// Persistent, 256 threads; the threads write Q'_n (from its group-major
// block) and S_n^T into K-major TF32 tiles.
template <typename Tout>
__global__ void __launch_bounds__(256, 1) k2_out(const __grid_constant__ OutParams p) {
    constexpr uint32_t MT = 128 * 128 * 4;
    extern __shared__ __align__(1024) unsigned char smraw[];
    unsigned char* sm = (unsigned char*)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    unsigned char* Qt = sm;
    unsigned char* St = sm + MT;
    unsigned char* Ot = sm + 2 * MT;  // bf16 output tile (T16 layout)
    unsigned char* Ss = Ot + kT16Bytes;  // S_n by TMA: four 128-byte-swizzled boxes of 32 columns
    __shared__ uint64_t bar[2];
    __shared__ uint32_t tslot;
    __shared__ int bad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, h = warp >> 2, t = 32 * q + lane;
    const int N = p.T / kC, nch = p.B * p.H * N;
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        bad = 0;
        fence_barrier_init();
        prefetch_tmap(&p.tS);
    }
    if (warp == 0) tmem_alloc(&tslot, 128);
    sync_all();
    const uint32_t tm = tslot;
    auto issue_S = [&](int cc) {
        mbar_arrive_expect_tx(&bar[0], MT);
        for (int kb = 0; kb < 4; ++kb)
            tma_load_3d(Ss + kb * 128 * 128, &p.tS, 32 * kb, cc * kD, 0, &bar[0]);
    };
    if (tid == 0 && (int)blockIdx.x < nch) issue_S(blockIdx.x);
    int it = 0;
    for (int c = blockIdx.x; c < nch; c += gridDim.x, ++it) {
        if (tid == 32) {  // the next chunk's blocks -> L2
            const int cn = c + gridDim.x;
            if (cn < nch) {
                bulk_prefetch_l2(p.Qp + (size_t)cn * kC * kD, kC * kD * 4);
                bulk_prefetch_l2(p.Oi + (size_t)cn * kC * kD, kC * kD * 4);
            }
        }
        // Q'_n into Qt: thread (row tid % 128, every other 4-column group) from
        // the group-major block, its loads issued before the wait for S_n;
        // S_n^T into St: thread (row r = tid / 2, half) reads 64 values of S_n
        // row r from the TMA boxes.
        {
            const float* qb = p.Qp + (size_t)c * kC * kD;
            const int rq = tid & 127, g0 = tid >> 7;
            const int r = tid >> 1, hf = tid & 1;
            float4 qv[16], sv[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) qv[k] = __ldg(grp4(qb, rq, 4 * (g0 + 2 * k)));
            if (!cta_wait(&bar[0], (uint32_t)(it & 1)) && tid == 0) bad = 1;
#pragma unroll
            for (int k = 0; k < 16; ++k)  // columns 64 hf + 4k .. +4: box 2 hf + k / 8, chunk k % 8
                sv[k] = *reinterpret_cast<const float4*>(Ss + (2 * hf + (k >> 3)) * 128 * 128 + r * 128 +
                                                         (((k & 7) ^ (r & 7)) << 4));
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int g = g0 + 2 * k;
                *reinterpret_cast<float4*>(Qt + (g >> 3) * 128 * 128 + rq * 128 + (((g & 7) ^ (rq & 7)) << 4)) = qv[k];
            }
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float vv[4] = {sv[k].x, sv[k].y, sv[k].z, sv[k].w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int col = 64 * hf + 4 * k + u;  // B row (value column), K index r
                    *reinterpret_cast<float*>(St + t32_off<128>(col, r >> 2) + (r & 3) * 4) = vv[u];
                }
            }
        }
        fence_async_smem();
        sync_all();
        if (tid == 0) {
            gemm_kk32<128, 128>(tm, saddr(Qt), saddr(St), 0, 128, 128, false);
            mma_commit(&bar[1]);
            if (c + (int)gridDim.x < nch) issue_S(c + gridDim.x);  // Ss read out above
            bulk_wait_read();  // the previous chunk's o tile has left Ot (the barrier below tells the rest)
        }
        float4 oa[16];  // O_intra row t, columns 64 h .. +64, loaded while the product runs
        {
            const float* oib = p.Oi + (size_t)c * kC * kD;
#pragma unroll
            for (int k = 0; k < 16; ++k) oa[k] = __ldg(grp4(oib, t, 64 * h + 4 * k));
        }
        if (!cta_wait(&bar[1], (uint32_t)(it & 1)) && tid == 0) bad = 1;
        // epilogue: o[b][n*C + t][h][64 hh ..] = D + O_intra, times sigmoid(zo)
        // when the output gate is fused (the pre-gate value then also to o_pre)
        const int n = c % N, bh = c / N, hd = bh % p.H, b = bh / p.H;
        float v[64];
        tm_ld64(tm + 64 * h, q, 0, v);
        const size_t ro = (((size_t)b * p.T + (size_t)n * kC + t) * p.H + hd) * kD + 64 * h;
        Tout* od = reinterpret_cast<Tout*>(p.o) + ro;
        Tout* pd = p.o_pre ? reinterpret_cast<Tout*>(p.o_pre) + ro : nullptr;
        const __nv_bfloat16* zr = p.zo ? reinterpret_cast<const __nv_bfloat16*>(p.zo) + ro : nullptr;
        auto put4 = [&](Tout* dst, int jj, float r0, float r1, float r2, float r3) {
            if constexpr (sizeof(Tout) == 4) {
                *reinterpret_cast<float4*>(reinterpret_cast<float*>(dst) + jj) = make_float4(r0, r1, r2, r3);
            } else {
                uint2 u;
                u.x = pack_bf16(r0, r1);
                u.y = pack_bf16(r2, r3);
                *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(dst) + jj) = u;
            }
        };
#pragma unroll
        for (int jj = 0; jj < 64; jj += 4) {
            const float4 a = oa[jj >> 2];
            float r0 = v[jj] + a.x, r1 = v[jj + 1] + a.y, r2 = v[jj + 2] + a.z, r3 = v[jj + 3] + a.w;
            if (zr) {
                if (pd) put4(pd, jj, r0, r1, r2, r3);
                const uint2 zw = __ldg(reinterpret_cast<const uint2*>(zr + jj));
                float z0, z1, z2, z3;
                unpack16<true>(zw.x, z0, z1);
                unpack16<true>(zw.y, z2, z3);
                r0 *= sigmoid_f(z0); r1 *= sigmoid_f(z1); r2 *= sigmoid_f(z2); r3 *= sigmoid_f(z3);
            }
            if constexpr (sizeof(Tout) == 4) {
                put4(od, jj, r0, r1, r2, r3);
            } else {
                v[jj] = r0; v[jj + 1] = r1; v[jj + 2] = r2; v[jj + 3] = r3;
            }
        }
        if constexpr (sizeof(Tout) == 2) {  // bf16 o leaves as a row tile by TMA store
#pragma unroll
            for (int i = 0; i < 8; ++i) st_chunk16<true>(Ot, t, 8 * h + i, v + 8 * i);
            fence_async_smem();
        }
        sync_all();
        if (sizeof(Tout) == 2 && tid == 0) {
            const int z = b * p.T + n * kC;
            tma_store_3d(&p.to, Ot, 0, hd, z);
            tma_store_3d(&p.to, Ot + kT16Block, 64, hd, z);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait_all();
    if (tid == 0 && bad) atomicAdd(&g_v2_timeouts, 1u);
    sync_all();
    if (warp == 0) tmem_dealloc(tm, 128);
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &qr) ==
                cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// Map over a token-major [B*T][H][128] bf16 tensor: box of 64 channels x 1 head x 128 tokens.
bool map_tokens16(CUtensorMap* m, const void* base, int B, int T, int H) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)B * T};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kC};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map over a row-major [rows][cols] bf16 matrix: box of 64 columns x box_rows rows
// (cols a multiple of 8, so that every row starts 16-byte aligned).
bool map_2d16(CUtensorMap* m, const void* base, long long cols, long long rows, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || cols % 8 || box_rows < 1 || box_rows > 256) return false;
    cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, 1};
    cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)cols * rows * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map over rows of 128 fp32 (a [rows][128] array): box of 32 columns x 128 rows.
bool map_rows32f(CUtensorMap* m, const float* base, long long rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)rows, 1};
    cuuint64_t strides[2] = {128 * 4, (cuuint64_t)rows * 128 * 4};
    cuuint32_t box[3] = {32, 128, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

constexpr int kIntraSmem = 6 * kT16Bytes + sizeof(IntraSmem) + 1024;
constexpr int kOutSmem = 3 * 128 * 128 * 4 + kT16Bytes + 1024;
template <int SLAB>
constexpr int chain_smem() { return 3 * 128 * 128 * 4 + SLAB * 512 + 1024; }

int chain_slab(int BH) { return BH * (kD / 32) < sm_count() ? 16 : 32; }

size_t fwd2_ws_bytes(int B, int T, int H) {
    const size_t nch = (size_t)B * H * (T / kC), CD = (size_t)kC * kD;
    // M, Bn, Q', O_intra, S_chunks, flags
    return (5 * nch * CD) * sizeof(float) + 256;
}

bool fwd2_supported(int B, int T, int H, int D, int C, bool in_bf16) {
    return in_bf16 && D == kD && C == kC && T > 0 && T % kC == 0 && B > 0 && H > 0;
}

cudaError_t run_fwd2(const Fwd2Args& a, cudaStream_t st) {
    if (!encode_fn()) return cudaErrorNotSupported;
    const int N = a.T / kC, nch = a.B * a.H * N, BH = a.B * a.H;
    IntraParams ip;
    if (!map_tokens16(&ip.tq, a.q, a.B, a.T, a.H) || !map_tokens16(&ip.tk, a.k, a.B, a.T, a.H) ||
        !map_tokens16(&ip.tv, a.v, a.B, a.T, a.H) || !map_tokens16(&ip.tg, a.g, a.B, a.T, a.H) ||
        !map_tokens16(&ip.te, a.e, a.B, a.T, a.H) || !map_tokens16(&ip.tw, a.w, a.B, a.T, a.H) ||
        !map_tokens16(&ip.tgam, a.gamma, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    ip.B = a.B; ip.T = a.T; ip.H = a.H;
    ip.q = a.q; ip.gamma = a.gamma;
    if (!map_rows32f(&ip.tM, a.M, (long long)nch * kD)) return cudaErrorInvalidValue;
    ip.M = a.M; ip.Mt = a.Mt; ip.Bn = a.Bn; ip.Qp = a.Qp; ip.Oi = a.Oi; ip.flags = a.flags;
    ip.aux = a.aux;
    ip.qk_raw = a.qk_raw; ip.rnorm = a.rnorm;
    if (a.qk_raw && !a.rnorm) return cudaErrorInvalidValue;
    auto kern = a.qk_raw ? k2_intra<true> : k2_intra<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kIntraSmem);
    if (e != cudaSuccess) return e;
    const int nsm = sm_count();
    const int grid = nch < nsm ? nch : nsm;
    MUIR_TIMED("k2_intra", st, kern<<<grid, 512, kIntraSmem, st>>>(ip));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    // one CTA per (head, column slab): 16-column slabs when 32-column ones
    // would leave SMs idle (each CTA is a sequential pass over the chunks)
    ChainParams cp;
    if (!map_rows32f(&cp.tM, a.M, (long long)nch * kD)) return cudaErrorInvalidValue;
    cp.Bn = a.Bn; cp.S0 = a.S0; cp.S_chunks = a.S_chunks; cp.S_final = a.S_final; cp.N = N;
    cp.S_last = a.S_last;
    if (chain_slab(BH) == 16) {
        e = cudaFuncSetAttribute(k2_chain<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, chain_smem<16>());
        if (e != cudaSuccess) return e;
        MUIR_TIMED("k2_chain", st, k2_chain<16><<<BH * (kD / 16), 128, chain_smem<16>(), st>>>(cp));
    } else {
        e = cudaFuncSetAttribute(k2_chain<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, chain_smem<32>());
        if (e != cudaSuccess) return e;
        MUIR_TIMED("k2_chain", st, k2_chain<32><<<BH * (kD / 32), 128, chain_smem<32>(), st>>>(cp));
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    if (a.o) {
        OutParams op;
        op.B = a.B; op.T = a.T; op.H = a.H;
        op.Qp = a.Qp; op.S_chunks = a.S_chunks; op.Oi = a.Oi; op.o = a.o;
        if (!map_rows32f(&op.tS, a.S_chunks, (long long)nch * kD)) return cudaErrorInvalidValue;
        op.zo = a.zo; op.o_pre = a.zo ? a.o_pre : nullptr;
        if (a.out_bf16) {
            if (!map_tokens16(&op.to, a.o, a.B, a.T, a.H)) return cudaErrorInvalidValue;
            e = cudaFuncSetAttribute(k2_out<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kOutSmem);
            if (e != cudaSuccess) return e;
            MUIR_TIMED("k2_out", st, k2_out<__nv_bfloat16><<<grid, 256, kOutSmem, st>>>(op));
        } else {
            e = cudaFuncSetAttribute(k2_out<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, kOutSmem);
            if (e != cudaSuccess) return e;
            MUIR_TIMED("k2_out", st, k2_out<float><<<grid, 256, kOutSmem, st>>>(op));
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

unsigned int timeouts_v2() {
    unsigned int n = 0;
    cudaMemcpyFromSymbol(&n, g_v2_timeouts, sizeof(n));
    const unsigned int z = 0;
    cudaMemcpyToSymbol(g_v2_timeouts, &z, sizeof(z));
    return n;
}

}  // namespace v2
}  // namespace muir

// bwd2.cu -- chunkwise backward on the 5th-generation tensor cores, every
// per-chunk intermediate on chip (companion of fwd2.cu: bf16 inputs,
// dk = dv = 128, chunk 128).
//
// Gradients of L = sum(o * dO) + sum(S_N * dS_N) ("custom backward pass",
// wolonglab.org page, "Methodology"), from the chunk form the forward uses,
//   O_n = Q'_n S_n + O_intra_n,   S_{n+1} = M_n S_n + B_n,
// with Y = W S + U' (Y_t = k_t^T D_t S_{t-1}):
//
//   reverse state pass  G_n = M_n^T G_{n+1} + Q'_n^T dO_n      (G_n = dL/dS_n)
//   per chunk, with G = G_{n+1}:
//     dY  = -M_QA^T dO - Abar G            dYR = T^T dY
//     dU  = M_QK^T dO + Kbar G + L_K^T dYR          -> dv = dU w, dw = dU v
//     dQ~ = dO S^T,  dK~ = dYR S^T,  dKbar = U G^T,  dAbar = -Y G^T
//     dL_A = -strict(dYR Y^T), dL_K = strict(dYR U^T),
//     dM_QA = -incl(dO Y^T),   dM_QK = incl(dO U^T)
//     decay-masked gradients (pivoted operands as in the forward):
//       dKp = dL_A Am + dL_K Km,      dQp = dM_QK Km + dM_QA Am,
//       dAm = dL_A^T Kp + dM_QA^T Qp, dKm = dL_K^T Kp + dM_QK^T Qp
//     dq^ = dQp 2^(L-P) + dQ~ 2^L,  da = dAm 2^(P-L) + dAbar 2^(Lbar-L)
//     dk  = dKp 2^(L-P) + dKm 2^(P-L) + dK~ 2^L + dKbar 2^(Lbar-L) + e da
//     dLog = dKp Kp + dQp Qp - dKm Km - dAm Am + dK~ K~ + dQ~ Q~ - dKbar Kbar - dAbar Abar
//          (the last four = Pd k + Pq q^ - Pa a with Pq = dQ~ 2^L, Pa = dAbar 2^(Lbar-L),
//           Pd = dK~ 2^L - dKbar 2^(Lbar-L))
//     dg_t = sum_{t' >= t} dLog_t' + dLbar,   dLbar_j = sum_c G[j][c] S_{n+1}[j][c]
//
// Kernels: k2_bprep (Q'^T dO), k2_chain_rev (reverse pass, dLbar), k2_bwd1
// (dY, dYR, dU -> dv, dw; the state-side terms; Y and dYR for k2_bwd2),
// k2_bwd2 (the decay-masked gradients in TF32 with the dL matrices as
// tensor-memory operands, one 64-channel half at a time; final dq, dk, dg, de,
// dgamma).  Precision: products with a state (S, G) use fp16 operands with a
// power-of-two scale per chunk, the bounded-range products fp16, the
// decay-masked gradients TF32; fp32 accumulation throughout.
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

// Expired bounded waits of this file's kernels (bit i: wait site i), read and
// cleared by timeouts_bwd2().
__device__ unsigned int g_bwd2_timeouts;

namespace {

constexpr int kC = 128, kD = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLogDecayMin = -20.f;
constexpr float kSpanMax = 140.f;  // single-pivot limit of |sum g| over a chunk (natural log)
constexpr uint32_t kT32Half = 64 * 128 * 4;  // T32 tile of 64 rows

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void sync_all() {
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
}

// 8 consecutive floats of a shared-memory table (32-byte aligned) in two 16-byte loads.
__device__ __forceinline__ void lds8(const float* p, float* v) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// 8 bf16 packed in 16 bytes -> floats.
__device__ __forceinline__ void unpack8_bf16(const uint4 u, float* v) {
    unpack16<true>(u.x, v[0], v[1]);
    unpack16<true>(u.y, v[2], v[3]);
    unpack16<true>(u.z, v[4], v[5]);
    unpack16<true>(u.w, v[6], v[7]);
}

// 8 consecutive bf16 of a token-major row -> floats.
__device__ __forceinline__ void ld8_bf16(const __nv_bfloat16* p, float* v) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    unpack16<true>(u.x, v[0], v[1]);
    unpack16<true>(u.y, v[2], v[3]);
    unpack16<true>(u.z, v[4], v[5]);
    unpack16<true>(u.w, v[6], v[7]);
}

__device__ __forceinline__ void st8_bf16(__nv_bfloat16* p, const float* v) {
    uint4 u;
    u.x = pack_bf16(v[0], v[1]);
    u.y = pack_bf16(v[2], v[3]);
    u.z = pack_bf16(v[4], v[5]);
    u.w = pack_bf16(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = u;
}

// Fused q/k prologue: x -> SiLU(x) r with r the row's inverse norm (the
// forward applies the same arithmetic).
__device__ __forceinline__ void prologue8(float* v, float r) {
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = v[u] * sigmoid_f(v[u]) * r;
}

// The scaled fp16 partials are kept channel-group-major within a chunk:
// element (t, ch) of chunk c is half 8 (c kD/8 kC + (ch/8) kC + t) + ch % 8,
// so that one 8-channel group of 32 consecutive rows is one contiguous
// 512-byte run (each warp's access, on both sides, is coalesced); the scale
// of (t, 32-channel group ch/32) sits at c 4 kC + (ch/32) kC + t.
__device__ __forceinline__ size_t pgrp(int c, int t, int ch) {  // in 16-byte words
    return (size_t)c * (kC * kD / 8) + (size_t)(ch >> 3) * kC + t;
}
__device__ __forceinline__ size_t psc(int c, int t, int ch) { return (size_t)c * 4 * kC + (size_t)(ch >> 5) * kC + t; }

// 32 values as fp16 times a power of two: the scale puts the largest
// magnitude just below 2^15 (fp16 keeps 11 significant bits of every value
// within 2^-14 of it; the sums these partials join are dominated by larger
// terms).  dst: the first of 4 groups of 8 halves, kC words apart; *scale:
// the factor.
__device__ __forceinline__ void st_scaled32(uint4* dst, float* scale, const float* v) {
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(v[j]));
    int ex = 0;
    frexpf(m, &ex);                       // m < 2^ex (m = 0: ex = 0)
    const int e = max(ex - 15, -126);
    const float inv = __int_as_float((127 - e) << 23), sc = __int_as_float((127 + e) << 23);
    *scale = sc;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint4 u;
        u.x = pack_f16(v[8 * i] * inv, v[8 * i + 1] * inv);
        u.y = pack_f16(v[8 * i + 2] * inv, v[8 * i + 3] * inv);
        u.z = pack_f16(v[8 * i + 4] * inv, v[8 * i + 5] * inv);
        u.w = pack_f16(v[8 * i + 6] * inv, v[8 * i + 7] * inv);
        dst[i * kC] = u;
    }
}

// The same for the two groups a + b and a - b (each with its own scale),
// without forming them in registers first.
__device__ __forceinline__ void st_scaled32_pm(uint4* dp, float* sp, uint4* dm, float* sm_,
                                               const float* a, const float* b) {
    float mp = 0.f, mm = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        mp = fmaxf(mp, fabsf(a[j] + b[j]));
        mm = fmaxf(mm, fabsf(a[j] - b[j]));
    }
    int ep = 0, em = 0;
    frexpf(mp, &ep);
    frexpf(mm, &em);
    ep = max(ep - 15, -126);
    em = max(em - 15, -126);
    const float ip = __int_as_float((127 - ep) << 23), im = __int_as_float((127 - em) << 23);
    *sp = __int_as_float((127 + ep) << 23);
    *sm_ = __int_as_float((127 + em) << 23);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint4 u, w;
        const int j = 8 * i;
        u.x = pack_f16((a[j] + b[j]) * ip, (a[j + 1] + b[j + 1]) * ip);
        u.y = pack_f16((a[j + 2] + b[j + 2]) * ip, (a[j + 3] + b[j + 3]) * ip);
        u.z = pack_f16((a[j + 4] + b[j + 4]) * ip, (a[j + 5] + b[j + 5]) * ip);
        u.w = pack_f16((a[j + 6] + b[j + 6]) * ip, (a[j + 7] + b[j + 7]) * ip);
        w.x = pack_f16((a[j] - b[j]) * im, (a[j + 1] - b[j + 1]) * im);
        w.y = pack_f16((a[j + 2] - b[j + 2]) * im, (a[j + 3] - b[j + 3]) * im);
        w.z = pack_f16((a[j + 4] - b[j + 4]) * im, (a[j + 5] - b[j + 5]) * im);
        w.w = pack_f16((a[j + 6] - b[j + 6]) * im, (a[j + 7] - b[j + 7]) * im);
        dp[i * kC] = u;
        dm[i * kC] = w;
    }
}

// 8 scaled fp16 values -> floats.
__device__ __forceinline__ void unpack8_scaled(const uint4 u, float sc, float* v) {
    unpack16<false>(u.x, v[0], v[1]);
    unpack16<false>(u.y, v[2], v[3]);
    unpack16<false>(u.z, v[4], v[5]);
    unpack16<false>(u.w, v[6], v[7]);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] *= sc;
}

// Store 32 values at columns 32 * c32 .. +32 of row t of a T16 tile.
template <bool BF16>
__device__ __forceinline__ void row_st32(unsigned char* tile, int t, int c32, const float* v) {
#pragma unroll
    for (int i = 0; i < 4; ++i) st_chunk16<BF16>(tile, t, 4 * c32 + i, v + 8 * i);
}

template <bool BF16>
__device__ __forceinline__ void row_ld32(const unsigned char* tile, int t, int c32, float* v) {
#pragma unroll
    for (int i = 0; i < 4; ++i) ld_chunk16<BF16>(tile, t, 4 * c32 + i, v + 8 * i);
}

__device__ __forceinline__ void tm_ld32w(uint32_t tm, int q, int col, float (&v)[32]) {
    tmem_ld32(taddr(tm, 32 * q, col), v);
    tmem_wait_ld();
}

}  // namespace

// ------------------------------------------------------------------ k2_bprep

// B'_n = Q'_n^T dO_n (fp16 operands, fp32 accumulation); one chunk per CTA.
__global__ void __launch_bounds__(256) k2_bprep(const __grid_constant__ BprepParams p) {
    extern __shared__ __align__(1024) unsigned char smraw[];
    unsigned char* sm = (unsigned char*)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    unsigned char* Qt = sm;
    unsigned char* Dt = sm + kT16Bytes;
    __shared__ uint64_t bar[2];
    __shared__ uint32_t tslot;
    __shared__ int bad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, h = warp >> 2, t = 32 * q + lane;
    const int c = blockIdx.x, N = p.T / kC;
    const int n = c % N, bh = c / N;
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        bad = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(&tslot, 128);
    sync_all();
    const uint32_t tm = tslot;
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar[0], kT16Bytes);
        const int z = (bh / p.H) * p.T + n * kC, y = bh % p.H;
        tma_load_3d(Dt, &p.tdO, 0, y, z, &bar[0]);
        tma_load_3d(Dt + kT16Block, &p.tdO, 64, y, z, &bar[0]);
    }
    {  // Q' row t, columns 64h .. +64 -> fp16
        const float* qb = p.Qp + (size_t)c * kC * kD;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float v[8];
            const float4 a = __ldg(grp4(qb, t, 64 * h + 8 * i));
            const float4 b = __ldg(grp4(qb, t, 64 * h + 8 * i + 4));
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
            st_chunk16<false>(Qt, t, 8 * h + i, v);
        }
    }
    if (!cta_wait(&bar[0], 0) && tid == 0) atomicOr(&bad, 1);
    if (p.zo) {  // fused output gate: dO = dO' sig(z) (fp16, and bf16), dz = dO' o sig (1 - sig)
        const size_t ro = (((size_t)(bh / p.H) * p.T + (size_t)n * kC + t) * p.H + bh % p.H) * kD + 64 * h;
        const __nv_bfloat16* zr = reinterpret_cast<const __nv_bfloat16*>(p.zo) + ro;
        __half* er = reinterpret_cast<__half*>(p.dO_eff) + ro;
        __nv_bfloat16* erb = reinterpret_cast<__nv_bfloat16*>(p.dO_effb) + ro;
        __nv_bfloat16* dzr = reinterpret_cast<__nv_bfloat16*>(p.dzo) + ro;
#pragma unroll 2
        for (int i = 0; i < 8; ++i) {
            float dy[8], zv[8], ov[8], dov[8], dzv[8];
            ld_chunk16<true>(Dt, t, 8 * h + i, dy);
            ld8_bf16(zr + 8 * i, zv);
            if (p.o_pre_f32) {
                const float* op = reinterpret_cast<const float*>(p.o_pre) + ro + 8 * i;
                const float4 a = __ldg(reinterpret_cast<const float4*>(op));
                const float4 b = __ldg(reinterpret_cast<const float4*>(op + 4));
                ov[0] = a.x; ov[1] = a.y; ov[2] = a.z; ov[3] = a.w;
                ov[4] = b.x; ov[5] = b.y; ov[6] = b.z; ov[7] = b.w;
            } else {
                ld8_bf16(reinterpret_cast<const __nv_bfloat16*>(p.o_pre) + ro + 8 * i, ov);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float sg = sigmoid_f(zv[u]);
                // the fp16 value the later kernels read
                dov[u] = __half2float(__float2half_rn(dy[u] * sg));
                dzv[u] = dy[u] * ov[u] * sg * (1.f - sg);
            }
            uint4 hv;
            hv.x = pack_f16(dov[0], dov[1]); hv.y = pack_f16(dov[2], dov[3]);
            hv.z = pack_f16(dov[4], dov[5]); hv.w = pack_f16(dov[6], dov[7]);
            *reinterpret_cast<uint4*>(er + 8 * i) = hv;
            st8_bf16(erb + 8 * i, dov);
            st8_bf16(dzr + 8 * i, dzv);
            st_chunk16<false>(Dt, t, 8 * h + i, dov);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {  // dO bf16 -> fp16 in place (own chunks)
            float v[8];
            ld_chunk16<true>(Dt, t, 8 * h + i, v);
            st_chunk16<false>(Dt, t, 8 * h + i, v);
        }
    }
    fence_async_smem();
    sync_all();
    if (tid == 0) {
        gemm_mm16(tm, saddr(Qt), 0, 0, saddr(Dt), 0, 0, 128, 128, kF16, false);
        mma_commit(&bar[1]);
    }
    if (!cta_wait(&bar[1], 0) && tid == 0) atomicOr(&bad, 2);
    {
        float* bb = p.Bp + (size_t)c * kD * kD;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float v[32];
            tm_ld32w(tm, q, 64 * h + 32 * hh, v);
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                *grp4(bb, t, 64 * h + 32 * hh + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        }
    }
    if (tid == 0 && bad) atomicOr(&g_bwd2_timeouts, (unsigned)bad);
    sync_all();
    if (warp == 0) tmem_dealloc(tm, 128);
}

// ------------------------------------------------------------------ k2_chain_rev

// G_n = M_n^T G_{n+1} + B'_n for one head and SLAB value columns, n = N-1 .. 0;
// records G_{n+1} in dSc[n], writes this slab's share of
// dLbar[n][j] = sum_c G_{n+1}[j][c] S_{n+1}[j][c] to its own slot (dgb[slab][n][j])
// and writes G_0 to dS0.  M_n^T streams through a 3-stage TMA ring (K-major TF32).
template <int SLAB>
__global__ void __launch_bounds__(128, 1) k2_chain_rev(const __grid_constant__ RevParams p) {
    constexpr int STAGES = 3;
    constexpr uint32_t MT = 128 * 128 * 4;
    extern __shared__ __align__(1024) unsigned char smraw[];
    unsigned char* sm = (unsigned char*)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    unsigned char* Mst = sm;
    unsigned char* Gt = sm + STAGES * MT;
    __shared__ uint64_t bar[STAGES + 1];
    __shared__ uint32_t tslot;
    __shared__ int bad;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int nslab = kD / SLAB;
    const int bh = blockIdx.x / nslab, c0 = (blockIdx.x % nslab) * SLAB;
    const int N = p.N, j = tid;
    if (tid == 0) {
        for (int i = 0; i <= STAGES; ++i) mbar_init(&bar[i], 1);
        bad = 0;
        fence_barrier_init();
        prefetch_tmap(&p.tMt);
    }
    if (warp == 0) tmem_alloc(&tslot, 32 < SLAB ? SLAB : 32);
    sync_all();
    const uint32_t tm = tslot;
    const long long row0 = (long long)bh * N * kD;
    // step s handles chunk n = N - 1 - s
    auto issue = [&](int s) {
        const int st = s % STAGES, n = N - 1 - s;
        mbar_arrive_expect_tx(&bar[st], MT);
        for (int kb = 0; kb < 4; ++kb)
            tma_load_3d(Mst + st * MT + kb * 128 * 128, &p.tMt, 32 * kb, (int)(row0 + (long long)n * kD), 0,
                        &bar[st]);
    };
    if (tid == 0)
        for (int s = 0; s < STAGES && s < N; ++s) issue(s);
    float Gr[SLAB];
    const size_t gbase = ((size_t)bh * kD + j) * kD + c0;
#pragma unroll
    for (int c = 0; c < SLAB; ++c) Gr[c] = p.dS_final ? p.dS_final[gbase + c] : 0.f;
    auto put = [&]() {
#pragma unroll
        for (int c = 0; c < SLAB; ++c)
            *reinterpret_cast<float*>(Gt + t32_off<SLAB>(c, j >> 2) + (j & 3) * 4) = Gr[c];
    };
    put();
    // B'_n and S_{n+1} of a step, loaded one step ahead (both come from DRAM)
    float Bn1[SLAB], Sn1[SLAB];
    auto load_step = [&](int n, float* Bd, float* Sd) {
        const float* bb = p.Bp + ((size_t)bh * N + n) * kD * kD;
        const float* sn1 = (n + 1 < N) ? p.S_chunks + ((size_t)bh * N + n + 1) * kD * kD + (size_t)j * kD + c0
                                       : p.S_last + gbase;
#pragma unroll
        for (int c = 0; c < SLAB; c += 4) {
            const float4 v = __ldg(grp4(bb, j, c0 + c));
            const float4 w = __ldg(reinterpret_cast<const float4*>(sn1 + c));
            Bd[c] = v.x; Bd[c + 1] = v.y; Bd[c + 2] = v.z; Bd[c + 3] = v.w;
            Sd[c] = w.x; Sd[c + 1] = w.y; Sd[c + 2] = w.z; Sd[c + 3] = w.w;
        }
    };
    if (N > 0) load_step(N - 1, Bn1, Sn1);
    fence_async_smem();
    sync_all();
    for (int s = 0; s < N; ++s) {
        const int st = s % STAGES, n = N - 1 - s;
        // the product first: only the issuing thread waits for M_n^T (see k2_chain)
        if (tid == 0) {
            if (!mbar_wait(&bar[st], (uint32_t)((s / STAGES) & 1))) atomicOr(&bad, 4);
            tc_fence_after();
            gemm_kk32<128, SLAB>(tm, saddr(Mst + st * MT), saddr(Gt), 0, SLAB, 128, false);
            mma_commit(&bar[STAGES]);
        }
        float Bc[SLAB], Sc[SLAB];
#pragma unroll
        for (int c = 0; c < SLAB; ++c) {
            Bc[c] = Bn1[c];
            Sc[c] = Sn1[c];
        }
        if (s + 1 < N) load_step(n - 1, Bn1, Sn1);
        // while it runs: record G_{n+1} and this slab's share of dLbar_n
        {
            float* gb = p.dSc + ((size_t)bh * N + n) * kD * kD;
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < SLAB; c += 4) {
                *grp4(gb, j, c0 + c) = make_float4(Gr[c], Gr[c + 1], Gr[c + 2], Gr[c + 3]);
                acc += Gr[c] * Sc[c] + Gr[c + 1] * Sc[c + 1] + Gr[c + 2] * Sc[c + 2] + Gr[c + 3] * Sc[c + 3];
            }
            // one partial per value slab, summed in a fixed order by k2_bwd2
            p.dgb[((size_t)(c0 / SLAB) * p.nch + (size_t)bh * N + n) * kD + j] = acc;
        }
        if (!cta_wait(&bar[STAGES], (uint32_t)(s & 1)) && tid == 0) atomicOr(&bad, 8);
        if (tid == 0 && s + STAGES < N) issue(s + STAGES);
        float d[32];
        tmem_ld32(taddr(tm, 32 * warp, 0), d);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < SLAB; ++c) Gr[c] = d[c] + Bc[c];
        put();
        fence_async_smem();
        sync_all();
    }
    if (p.dS0) {
        float* d = p.dS0 + gbase;
#pragma unroll
        for (int c = 0; c < SLAB; c += 4) *reinterpret_cast<float4*>(d + c) = make_float4(Gr[c], Gr[c + 1], Gr[c + 2], Gr[c + 3]);
    }
    if (tid == 0 && bad) atomicOr(&g_bwd2_timeouts, (unsigned)bad);
    sync_all();
    if (warp == 0) tmem_dealloc(tm, 32 < SLAB ? SLAB : 32);
}

// ------------------------------------------------------------------ k2_bwd1

namespace {
struct Bwd1Smem {
    alignas(16) float Lb[kD];
    float red[16];
    uint64_t bar[20];
    uint32_t tslot;
    int bad;
};
enum { B1D = 0, B1W, B1U, B1Q, B1A, B1T, B1K, B1L, B1KB, B1M1, B1M2, B1M3, B1M4, B1M5, B1M6, B1G, B1LM, B1V };

// Largest |x| over the block (512 threads, 32 values each); ends with a barrier.
__device__ __forceinline__ float block_absmax(const float (&v)[32], float* red, int warp, int lane) {
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(v[j]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    float r = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) r = fmaxf(r, red[i]);
    __syncthreads();
    return r;
}

// Power of two s with max|x| / s below 2^14 (fp16 operands keep their range); 1 for zero.
__device__ __forceinline__ float pow2_scale(float amax) {
    if (!(amax > 0.f)) return 1.f;
    return exp2f((float)(ilogbf(amax) - 13));
}
}  // namespace

// 512 threads; thread t = 32 (warp % 4) + lane owns row t, columns 32 (warp / 4) .. +32.
// Products with a state use fp16 operands with S / sS and G / sG (sS, sG per-chunk
// powers of two), every other product fp16; accumulation fp32 in tensor memory.
__global__ void __launch_bounds__(512, 1) k2_bwd1(const __grid_constant__ Bwd1Params p) {
    extern __shared__ __align__(1024) unsigned char smraw[];
    unsigned char* sm = (unsigned char*)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    unsigned char* S[6];
#pragma unroll
    for (int i = 0; i < 6; ++i) S[i] = sm + i * kT16Bytes;
    Bwd1Smem& s = *reinterpret_cast<Bwd1Smem*>(sm + 6 * kT16Bytes);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, h = warp >> 2, t = 32 * q + lane, c0 = 32 * h;
    const int N = p.T / kC, nch = p.B * p.H * N;
    if (tid == 0) {
        for (int i = 0; i < 20; ++i) mbar_init(&s.bar[i], 1);
        s.bad = 0;
        fence_barrier_init();
        prefetch_tmap(&p.tdO);
    }
    if (warp == 0) tmem_alloc(&s.tslot, 512);
    sync_all();
    const uint32_t tm = s.tslot;
    uint32_t a[6];
#pragma unroll
    for (int i = 0; i < 6; ++i) a[i] = saddr(S[i]);
    auto waitb = [&](int i, uint32_t ph) {  // all threads: warp 0 polls, the rest sleep
        if (!cta_wait(&s.bar[i], ph) && tid == 0) atomicOr(&s.bad, 1 << (8 + i));
    };
    auto bulk = [&](unsigned char* dst, const unsigned char* src, int bar) {
        mbar_arrive_expect_tx(&s.bar[bar], kT16Bytes);
        bulk_load(dst, src, kT16Bytes, &s.bar[bar]);
    };
    int it = 0;
    for (int c = blockIdx.x; c < nch; c += gridDim.x, ++it) {
        const uint32_t ph = (uint32_t)(it & 1);
        const int n = c % N, bh = c / N, hd = bh % p.H, b = bh / p.H;
        const size_t cb = (size_t)c * kC * kD + (size_t)t * kD + c0;          // per-chunk arrays
        const size_t pb = pgrp(c, t, c0), scb = psc(c, t, c0);               // partials, their scales
        const unsigned char* ax = p.aux + (size_t)c * AuxLayout::kBytes;
        unsigned char* y16 = p.Y16 + (size_t)c * kT16Bytes;
        unsigned char* r16 = p.dYR16 + (size_t)c * kT16Bytes;

        if (tid == 0) {  // dO -> S1; W -> S2, U -> S4, M_QA -> S5
            bulk_wait_read();  // the previous chunk's tile stores have left S2 and S5
            mbar_arrive_expect_tx(&s.bar[B1D], kT16Bytes);
            const int z = b * p.T + n * kC;
            tma_load_3d(S[1], &p.tdO, 0, hd, z, &s.bar[B1D]);
            tma_load_3d(S[1] + kT16Block, &p.tdO, 64, hd, z, &s.bar[B1D]);
            bulk(S[2], ax + AuxLayout::kW16, B1W);
            bulk(S[4], ax + AuxLayout::kU16, B1U);
            bulk(S[5], ax + AuxLayout::kMQA16, B1Q);
            mbar_arrive_expect_tx(&s.bar[B1G], kT16Bytes);  // g -> S0 (free until the state tile)
            tma_load_3d(S[0], &p.tg, 0, hd, z, &s.bar[B1G]);
            tma_load_3d(S[0] + kT16Block, &p.tg, 64, hd, z, &s.bar[B1G]);
        }
        // S_n and G_{n+1} rows t (from DRAM), requested before the log-decay product
        float4 srow[8], grow[8];
        {
            const float* src = p.S_chunks + cb;
            const float* gb = p.dSc + (size_t)c * kC * kD;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                srow[j] = __ldg(reinterpret_cast<const float4*>(src + 4 * j));
                grow[j] = __ldg(grp4(gb, t, c0 + 4 * j));
            }
        }
        // log decay of row t, columns c0..: L = Tril(1) clamp(g) as one product
        // (ones tile in S3, free until the gradient-state tile); E = 2^L,
        // Eb = 2^(Lbar - L), Lbar = the product's last row
        float L[32];
        {
            float v[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = (c0 + 8 * i + u <= t) ? 1.f : 0.f;
                st_chunk16<true>(S[3], t, 4 * h + i, v);
            }
            waitb(B1G, ph);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                ld_chunk16<true>(S[0], t, 4 * h + i, v);
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = fmaxf(v[u], kLogDecayMin);
                st_chunk16<true>(S[0], t, 4 * h + i, v);
            }
            fence_async_smem();
            sync_all();
            if (tid == 0) {
                gemm_km16(tm + 0, a[3], 0, a[0], 0, 0, 128, 128, kBF16, false);
                mma_commit(&s.bar[B1LM]);
            }
            waitb(B1LM, ph);
            tm_ld32w(tm, q, c0, L);
#pragma unroll
            for (int j = 0; j < 32; ++j) L[j] *= kLog2e;
            if (t == kC - 1) {
#pragma unroll
                for (int j = 0; j < 32; ++j) s.Lb[c0 + j] = L[j];
            }
        }
        // S_n / sS -> fp16 tile S0, G / sG -> fp16 tile S3 (row j = t)
        float sS, sG;
        {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 x = srow[j >> 2];
                v[j] = x.x; v[j + 1] = x.y; v[j + 2] = x.z; v[j + 3] = x.w;
            }
            sS = pow2_scale(block_absmax(v, s.red, warp, lane));
            const float is = 1.f / sS;
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= is;
            row_st32<false>(S[0], t, h, v);
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 x = grow[j >> 2];
                v[j] = x.x; v[j + 1] = x.y; v[j + 2] = x.z; v[j + 3] = x.w;
            }
            sG = pow2_scale(block_absmax(v, s.red, warp, lane));
            const float ig = 1.f / sG;
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= ig;
            row_st32<false>(S[3], t, h, v);
        }
        waitb(B1D, ph);
        if (!p.dO_f16) {  // dO bf16 -> fp16 in place (own chunks)
            float v[32];
            row_ld32<true>(S[1], t, h, v);
            row_st32<false>(S[1], t, h, v);
        }
        fence_async_smem();
        __syncthreads();
        waitb(B1W, ph);
        tc_fence_after();
        // ---- phase 1: dQ~ / sS = dO S^T (B0), W S / sS (B1)
        if (tid == 0) {
            gemm_kk16(tm + 0, a[1], 0, a[0], 0, 0, 128, 128, kF16, false);
            gemm_km16(tm + 128, a[2], 0, a[0], 0, 0, 128, 128, kF16, false);
            mma_commit(&s.bar[B1M1]);
        }
        float4 urow[8];  // U' row t, requested while the products run
        {
            const float* ub = reinterpret_cast<const float*>(ax + AuxLayout::kUp);
#pragma unroll
            for (int j = 0; j < 8; ++j) urow[j] = __ldg(grp4(ub, t, c0 + 4 * j));
        }
        waitb(B1M1, ph);
        tc_fence_after();
        // ---- phase 2: Pq; Y = W S + U' -> fp16 tile S2 (also saved for k2_bwd2)
        {
            float d[32];
            tm_ld32w(tm, q, c0, d);
#pragma unroll
            for (int j = 0; j < 32; ++j) d[j] *= sS * ex2(L[j]);
            st_scaled32(reinterpret_cast<uint4*>(p.Pq) + pb, p.sq + scb, d);
            tm_ld32w(tm, q, 128 + c0, d);
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 x = urow[j >> 2];
                d[j] = d[j] * sS + x.x; d[j + 1] = d[j + 1] * sS + x.y;
                d[j + 2] = d[j + 2] * sS + x.z; d[j + 3] = d[j + 3] * sS + x.w;
            }
            row_st32<false>(S[2], t, h, d);  // Y over W
        }
        fence_async_smem();
        sync_all();
        waitb(B1U, ph);
        waitb(B1Q, ph);
        if (tid == 0) {
            bulk_store(y16, S[2], kT16Bytes);
            bulk_commit();
            gemm_kk16(tm + 384, a[4], 0, a[3], 0, 0, 128, 128, kF16, false);         // dKbar / sG = U G^T (kept)
            gemm_kk16(tm + 128, a[2], 0, a[3], 0, 0, 128, 128, kF16, false, true);  // dAbar / sG = -Y G^T
            gemm_mm16(tm + 256, a[5], 0, 0, a[1], 0, 0, 128, 128, kF16, false, true); // -M_QA^T dO
            mma_commit(&s.bar[B1M2]);
        }
        waitb(B1M2, ph);
        if (tid == 0) {  // Abar -> S4, T -> S5 (U, M_QA consumed)
            bulk(S[4], ax + AuxLayout::kAbar16, B1A);
            bulk(S[5], ax + AuxLayout::kT16, B1T);
        }
        // ---- phase 3: Pa = dAbar 2^(Lbar - L)
        {
            float d[32];
            tm_ld32w(tm, q, 128 + c0, d);  // dAbar / sG
#pragma unroll
            for (int jj = 0; jj < 32; jj += 8) {
                float lb[8];
                lds8(&s.Lb[c0 + jj], lb);
#pragma unroll
                for (int u = 0; u < 8; ++u) d[jj + u] *= sG * ex2(lb[u] - L[jj + u]);
            }
            st_scaled32(reinterpret_cast<uint4*>(p.Pa) + pb, p.sa + scb, d);
        }
        waitb(B1A, ph);  // (its block barrier also orders the reads of B1 above)
        // ---- phase 4: Abar G / sG (B0); dY = -M_QA^T dO - Abar G
        if (tid == 0) {
            gemm_km16(tm + 0, a[4], 0, a[3], 0, 0, 128, 128, kF16, false);
            mma_commit(&s.bar[B1M3]);
        }
        waitb(B1M3, ph);
        if (tid == 0) {
            bulk_wait_read();  // Y left S2
            bulk(S[4], ax + AuxLayout::kMQK16, B1K);  // Abar consumed
        }
        {
            float d[32], e2[32];
            tm_ld32w(tm, q, 256 + c0, d);
            tm_ld32w(tm, q, c0, e2);
#pragma unroll
            for (int j = 0; j < 32; ++j) d[j] -= sG * e2[j];
            __syncthreads();                 // Y (S2) no longer read by the bulk store
            row_st32<false>(S[2], t, h, d);  // dY over Y
        }
        fence_async_smem();
        sync_all();
        waitb(B1T, ph);
        // ---- phase 5: dYR = T^T dY (B1)
        if (tid == 0) {
            gemm_mm16(tm + 128, a[5], 0, 0, a[2], 0, 0, 128, 128, kF16, false);
            mma_commit(&s.bar[B1M4]);
        }
        waitb(B1M4, ph);
        if (tid == 0) bulk(S[2], ax + AuxLayout::kLK16, B1L);  // dY consumed
        {
            float d[32];
            tm_ld32w(tm, q, 128 + c0, d);
            row_st32<false>(S[5], t, h, d);  // dYR over T
        }
        fence_async_smem();
        sync_all();
        waitb(B1K, ph);
        // ---- phase 6: dK~ / sS = dYR S^T (B0); M_QK^T dO (B2); Pk, Pd from dK~ and dKbar (B3)
        if (tid == 0) {
            bulk_store(r16, S[5], kT16Bytes);
            bulk_commit();
            gemm_kk16(tm + 0, a[5], 0, a[0], 0, 0, 128, 128, kF16, false);
            gemm_mm16(tm + 256, a[4], 0, 0, a[1], 0, 0, 128, 128, kF16, false);
            mma_commit(&s.bar[B1M5]);
        }
        waitb(B1M5, ph);
        if (tid == 0) {
            bulk(S[0], ax + AuxLayout::kKbar16, B1KB);  // S consumed
            // v -> S1, w -> S4 (dO, M_QK consumed) for the last phase
            const int z = b * p.T + n * kC;
            mbar_arrive_expect_tx(&s.bar[B1V], 2 * kT16Bytes);
            tma_load_3d(S[1], &p.tv, 0, hd, z, &s.bar[B1V]);
            tma_load_3d(S[1] + kT16Block, &p.tv, 64, hd, z, &s.bar[B1V]);
            tma_load_3d(S[4], &p.tw, 0, hd, z, &s.bar[B1V]);
            tma_load_3d(S[4] + kT16Block, &p.tw, 64, hd, z, &s.bar[B1V]);
        }
        {
            float d[32], e2[32];
            tm_ld32w(tm, q, c0, d);         // dK~ / sS
            tm_ld32w(tm, q, 384 + c0, e2);  // dKbar / sG
#pragma unroll
            for (int jj = 0; jj < 32; jj += 8) {
                float lb[8];
                lds8(&s.Lb[c0 + jj], lb);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    d[jj + u] *= sS * ex2(L[jj + u]);                 // dK~ 2^L
                    e2[jj + u] *= sG * ex2(lb[u] - L[jj + u]);       // dKbar 2^(Lbar-L)
                }
            }
            st_scaled32_pm(reinterpret_cast<uint4*>(p.Pk) + pb, p.sk + scb, reinterpret_cast<uint4*>(p.Pd) + pb, p.sd + scb, d, e2);  // Pk, Pd
        }
        waitb(B1L, ph);
        waitb(B1KB, ph);
        // ---- phase 7: dU = M_QK^T dO + L_K^T dYR (B2) + Kbar G (B1, times sG)
        if (tid == 0) {
            gemm_mm16(tm + 256, a[2], 0, 0, a[5], 0, 0, 128, 128, kF16, true);
            gemm_km16(tm + 128, a[0], 0, a[3], 0, 0, 128, 128, kF16, false);
            mma_commit(&s.bar[B1M6]);
        }
        waitb(B1M6, ph);
        {
            float d[32], e2[32], vv[8], wv[8];
            tm_ld32w(tm, q, 256 + c0, d);
            tm_ld32w(tm, q, 128 + c0, e2);
            waitb(B1V, ph);
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // dv over v (S1), dw over w (S4), stored as tiles
                ld_chunk16<true>(S[1], t, 4 * h + i, vv);
                ld_chunk16<true>(S[4], t, 4 * h + i, wv);
                float o1[8], o2[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float du = d[8 * i + u] + sG * e2[8 * i + u];
                    o1[u] = du * wv[u];
                    o2[u] = du * vv[u];
                }
                st_chunk16<true>(S[1], t, 4 * h + i, o1);
                st_chunk16<true>(S[4], t, 4 * h + i, o2);
            }
        }
        fence_async_smem();
        sync_all();
        if (tid == 0) {  // (the next chunk's loads into S1, S4 wait for these reads)
            const int z = b * p.T + n * kC;
            tma_store_3d(&p.tdv, S[1], 0, hd, z);
            tma_store_3d(&p.tdv, S[1] + kT16Block, 64, hd, z);
            tma_store_3d(&p.tdw, S[4], 0, hd, z);
            tma_store_3d(&p.tdw, S[4] + kT16Block, 64, hd, z);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait_all();
    if (tid == 0 && s.bad) atomicOr(&g_bwd2_timeouts, (unsigned)s.bad);
    sync_all();
    if (warp == 0) tmem_dealloc(tm, 512);
}

// ------------------------------------------------------------------ k2_bwd2

namespace {
struct Bwd2Smem {
    alignas(16) float P2[kD];
    alignas(16) float sfx[4][kD];  // per-quarter totals of the reverse scan
    alignas(16) float dgb[kD];     // dLbar of the chunk (value slabs summed in a fixed order)
    float dot[2][8][kC];  // fused prologue: row dots dq^.q^ and dk^.k^ per (half, warp group)
    uint64_t bar[8];
    uint32_t tslot;
    int bad;
};
enum { B2IN = 0, B2M, B2G, B2X, B2Q };
// which part of a dL product survives, for row r and column col:
// col < r, col <= r, col > r, col >= r
enum { kStrictLow = 0, kInclLow, kStrictUp, kInclUp };
}  // namespace

// 512 threads; thread t = 32 (warp % 4) + lane owns row t; for channel half hj
// it handles the 16 channels 64 hj + 16 (warp / 4) .. +16.  Per half, four
// rounds each form two dL matrices (fp16 products into TMEM columns 0..255),
// mask them in place and use them as the A operands of TF32
// products with a pivoted operand (K-major TF32 tile, 64 rows = the half's
// channels) into one of four 64-column accumulators (TMEM 256..511).
template <bool QKRAW>
__global__ void __launch_bounds__(512, 1) k2_bwd2(const __grid_constant__ Bwd2Params p) {
    extern __shared__ __align__(1024) unsigned char smraw[];
    unsigned char* sm = (unsigned char*)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    unsigned char* tdO = sm;
    unsigned char* tU = sm + 1 * kT16Bytes;
    unsigned char* tY = sm + 2 * kT16Bytes;
    unsigned char* tR = sm + 3 * kT16Bytes;
    unsigned char* Bt0 = sm + 4 * kT16Bytes;
    unsigned char* Bt1 = Bt0 + kT32Half;
    unsigned char* Kt = Bt1 + kT32Half;  // k of the current half (T16 block), by TMA
    Bwd2Smem& s = *reinterpret_cast<Bwd2Smem*>(Kt + kT16Block);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, g4 = warp >> 2, t = 32 * q + lane;
    const int N = p.T / kC, nch = p.B * p.H * N;
    if (tid == 0) {
        for (int i = 0; i < 8; ++i) mbar_init(&s.bar[i], 1);
        s.bad = 0;
        fence_barrier_init();
        prefetch_tmap(&p.tdO);
    }
    if (warp == 0) tmem_alloc(&s.tslot, 512);
    sync_all();
    const uint32_t tm = s.tslot;
    const uint32_t aO = saddr(tdO), aU = saddr(tU), aY = saddr(tY), aR = saddr(tR);
    const uint32_t aB0 = saddr(Bt0), aB1 = saddr(Bt1);
    uint32_t pm = 0;  // parity of the MMA barrier
    // Every thread waits; the barrier that follows keeps the next commit on
    // B2M from completing before the slowest thread has seen this phase.
    auto mma_wait = [&]() {
        if (!cta_wait(&s.bar[B2M], pm) && tid == 0) atomicOr(&s.bad, 1 << 24);
        pm ^= 1u;
    };
    // Mask the two dL products in place: this warp's two 32-column blocks of bank
    // g4 >> 1.  A block wholly on the kept side of the diagonal is left as it is
    // (the TF32 product truncates it), a block wholly on the other side is
    // zeroed, and only the diagonal block (block index q) is read and masked.
    auto mask_rows = [&](int mode0, int mode1) {
        const int mode = (g4 >> 1) ? mode1 : mode0;
        const bool low = mode == kStrictLow || mode == kInclLow;
        const bool incl = mode == kInclLow || mode == kInclUp;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            const int col0 = 64 * (g4 & 1) + 32 * part, cb = col0 >> 5;
            const uint32_t at = taddr(tm, 32 * q, 128 * (g4 >> 1) + col0);
            if (cb == q) {
                float v[32];
                tmem_ld32(at, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const bool keep = low ? (j < lane || (incl && j == lane)) : (j > lane || (incl && j == lane));
                    if (!keep) v[j] = 0.f;
                }
                tmem_st16(at, *reinterpret_cast<const float(*)[16]>(v));
                tmem_st16(at + 16, *reinterpret_cast<const float(*)[16]>(v + 16));
            } else if (low ? cb > q : cb < q) {
                float z[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) z[j] = 0.f;
                tmem_st16(at, z);
                tmem_st16(at + 16, z);
            }
        }
        tmem_wait_st();
    };
    // ACC[128 x 64] = A0 (TMEM cols 0..127) Bt0 + A1 (TMEM cols 128..255) Bt1, TF32
    auto acc_pair = [&](int acc_col) {
        const uint32_t id = idesc(kTF32, 128, 64, false, false);
        for (int k = 0; k < 128; k += 8)
            mma_tf32_ta(tm + acc_col, tm + k, kdesc32<64>(aB0, 0, k), id, k ? 1u : 0u);
        for (int k = 0; k < 128; k += 8)
            mma_tf32_ta(tm + acc_col, tm + 128 + k, kdesc32<64>(aB1, 0, k), id, 1u);
    };
    // 16 values of row t -> column t of a transposed K-major TF32 tile, rows r0 ..
    auto put_t = [&](unsigned char* tile, int r0, const float* v) {
#pragma unroll
        for (int u = 0; u < 16; ++u)
            *reinterpret_cast<float*>(tile + t32_off<64>(r0 + u, t >> 2) + (t & 3) * 4) = tf32_round(v[u]);
    };
    // Round r in two parts.  The first (thread 0) issues its two dL products
    // into TMEM columns 0..255; they read only the four chunk tiles, so they
    // run while the threads form the round's pivoted operand tiles.  The
    // second masks them and accumulates the TF32 pair.
    auto round_issue = [&](int r) {
        const uint32_t ax = r == 0 ? aR : r == 1 ? aO : r == 2 ? aY : aU;
        const uint32_t bx0 = r < 2 ? aY : aR, bx1 = r < 2 ? aU : aO;
        gemm_kk16(tm + 0, ax, 0, bx0, 0, 0, 128, 128, kF16, false, r != 3);
        gemm_kk16(tm + 128, ax, 0, bx1, 0, 0, 128, 128, kF16, false, r == 2);
        mma_commit(&s.bar[B2M]);
    };
    auto round_finish = [&](int r) {
        mma_wait();
        mask_rows(r == 0 ? kStrictLow : r == 1 ? kInclLow : kStrictUp,
                  r == 0 ? kStrictLow : r == 1 ? kInclLow : kInclUp);
        sync_all();  // the masks, and the operand tiles' generic writes (fenced by their writers)
        if (tid == 0) {
            acc_pair(256 + 64 * r);
            mma_commit(&s.bar[B2M]);
        }
        mma_wait();
    };

    // dO, U, Y, dYR of chunk cc into the four tiles; a chunk's loads are issued
    // as soon as the previous chunk's last products have read the tiles
    auto load_tiles = [&](int cc) {
        const int nn = cc % N, bb = cc / N;
        mbar_arrive_expect_tx(&s.bar[B2IN], 4 * kT16Bytes);
        const int z = (bb / p.H) * p.T + nn * kC;
        tma_load_3d(tdO, &p.tdO, 0, bb % p.H, z, &s.bar[B2IN]);
        tma_load_3d(tdO + kT16Block, &p.tdO, 64, bb % p.H, z, &s.bar[B2IN]);
        bulk_load(tU, p.aux + (size_t)cc * AuxLayout::kBytes + AuxLayout::kU16, kT16Bytes, &s.bar[B2IN]);
        bulk_load(tY, p.Y16 + (size_t)cc * kT16Bytes, kT16Bytes, &s.bar[B2IN]);
        bulk_load(tR, p.dYR16 + (size_t)cc * kT16Bytes, kT16Bytes, &s.bar[B2IN]);
    };
    if (tid == 0 && (int)blockIdx.x < nch) load_tiles(blockIdx.x);

    int it = 0;
    for (int c = blockIdx.x; c < nch; c += gridDim.x, ++it) {
        const uint32_t ph = (uint32_t)(it & 1);
        const int n = c % N, bh = c / N, hd = bh % p.H, b = bh / p.H;
        const size_t tok = ((size_t)b * p.T + (size_t)n * kC + t) * p.H + hd;
        const float rq = QKRAW ? __ldg(p.rnorm + (size_t)c * 2 * kC + t) : 1.f;
        const float rk = QKRAW ? __ldg(p.rnorm + (size_t)c * 2 * kC + kC + t) : 1.f;
        {  // this chunk's rows of the inputs the readout reads late -> L2
            const char* rows[5] = {static_cast<const char*>(p.k), static_cast<const char*>(p.e),
                                   static_cast<const char*>(p.q), static_cast<const char*>(p.gamma),
                                   static_cast<const char*>(p.g)};
            const size_t off = tok * kD * 2;
#pragma unroll
            for (int i = 0; i < 5; ++i) {
                if (((i * 2) & 3) == g4) prefetch_l2(rows[i] + off);
                if (((i * 2 + 1) & 3) == g4) prefetch_l2(rows[i] + off + 128);
            }
            if (tid == 32) {
                const size_t cb = (size_t)c * kC * kD * 2, sb = (size_t)c * kC * 16;
                const __half* P[4] = {p.Pq, p.Pk, p.Pa, p.Pd};
                const float* S4[4] = {p.sq, p.sk, p.sa, p.sd};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    bulk_prefetch_l2(reinterpret_cast<const char*>(P[i]) + cb, kC * kD * 2);
                    bulk_prefetch_l2(reinterpret_cast<const char*>(S4[i]) + sb, kC * 16);
                }
            }
        }
        if (tid < kD) {  // dLbar: the value slabs' partial sums in a fixed order
            float acc = 0.f;
            for (int sl = 0; sl < p.nslab; ++sl) acc += p.dgb[((size_t)sl * nch + c) * kD + tid];
            s.dgb[tid] = acc;
        }
        if (!cta_wait(&s.bar[B2IN], ph) && tid == 0) atomicOr(&s.bad, 1 << 25);
        if (!p.dO_f16) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // dO bf16 -> fp16 in place (row t, columns 32 g4 ..)
                float v[8];
                ld_chunk16<true>(tdO, t, 4 * g4 + i, v);
                st_chunk16<false>(tdO, t, 4 * g4 + i, v);
            }
        }
        if (tid == 0) bulk_wait_read();  // the previous chunk's gradient tiles have left Bt0, Bt1
        fence_async_smem();
        sync_all();

#pragma unroll 1
        for (int hj = 0; hj < 2; ++hj) {
            const int j0 = 64 * hj + 16 * g4;  // this thread's channels
            const int r0 = 16 * g4;            // their rows in the half tiles
            // e of the row for Am, requested before the log-decay product
            const __nv_bfloat16* ein = reinterpret_cast<const __nv_bfloat16*>(p.e) + tok * kD + j0;
            const uint4 eraw0 = __ldg(reinterpret_cast<const uint4*>(ein));
            const uint4 eraw1 = __ldg(reinterpret_cast<const uint4*>(ein + 8));
            // log decay of the half's 64 channels: L = Tril(1) clamp(g) as one
            // product (g block in Bt1, ones tile in Bt0: both free until the
            // pivoted operands; TMEM columns 0..63 free until the first round)
            if (tid == 0) {
                mbar_arrive_expect_tx(&s.bar[B2G], 2 * kT16Block);
                tma_load_3d(Bt1, &p.tg, 64 * hj, hd, b * p.T + n * kC, &s.bar[B2G]);
                tma_load_3d(Kt, &p.tk, 64 * hj, hd, b * p.T + n * kC, &s.bar[B2G]);  // k of the half
            }
            {
                float v[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
#pragma unroll
                    for (int u = 0; u < 8; ++u) v[u] = (32 * g4 + 8 * i + u <= t) ? 1.f : 0.f;
                    st_chunk16<true>(Bt0, t, 4 * g4 + i, v);
                }
            }
            if (!cta_wait(&s.bar[B2G], (uint32_t)((2 * it + hj) & 1)) && tid == 0) atomicOr(&s.bad, 1 << 26);
            uint32_t gkeep = 0;  // bit u: g of channel j0 + u is at or above the clamp
            {
                float v[8];
#pragma unroll
                for (int i = 0; i < 2; ++i) {  // row t, channels 16 g4 .. +16 of the block
                    ld_chunk16<true>(Bt1, t, 2 * g4 + i, v);
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        gkeep |= (v[u] >= kLogDecayMin ? 1u : 0u) << (8 * i + u);
                        v[u] = fmaxf(v[u], kLogDecayMin);
                    }
                    st_chunk16<true>(Bt1, t, 2 * g4 + i, v);
                }
            }
            fence_async_smem();
            sync_all();
            if (tid == 0) {
                gemm_km16(tm + 0, aB0, 0, aB1, 0, 0, 64, 128, kBF16, false);
                mma_commit(&s.bar[B2M]);
            }
            mma_wait();
            float L[16];
            tmem_ld16(taddr(tm, 32 * q, 16 * g4), L);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; ++u) L[u] *= kLog2e;
            if (t == kC - 1) {  // the chunk totals: the last row
                bool far = false;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    s.P2[j0 + u] = 0.5f * L[u];
                    far |= L[u] < -kSpanMax * kLog2e;
                }
                // (the forward's test: the call then also runs the boundary-pivot
                // path, which overwrites this kernel's results)
                if (far) atomicOr(p.flags, 1);
            }
            sync_all();  // every row's L has left TMEM columns 0..63
            if (tid == 0) round_issue(0);
            {  // Am -> Bt0, Km -> Bt1
                float kv[16], ev[16], am[16], km[16];
                ld_chunk16<true>(Kt, t, 2 * g4, kv); ld_chunk16<true>(Kt, t, 2 * g4 + 1, kv + 8);
                if (QKRAW) { prologue8(kv, rk); prologue8(kv + 8, rk); }
                unpack8_bf16(eraw0, ev); unpack8_bf16(eraw1, ev + 8);
float p16[16];
                lds8(&s.P2[j0], p16); lds8(&s.P2[j0 + 8], p16 + 8);
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    km[u] = kv[u] * ex2(p16[u] - L[u]);
                    am[u] = ev[u] * km[u];
                }
                put_t(Bt0, r0, am);
                put_t(Bt1, r0, km);
            }
            fence_async_smem();
            // Four rounds (one loop, so that their code is issued once):
            //  R1: dL_A = -dYR Y^T, dL_K = dYR U^T (strict) -> dKp = dL_A Am + dL_K Km
            //  R2: dM_QA = -dO Y^T, dM_QK = dO U^T (inclusive) -> dQp = dM_QA Am + dM_QK Km
            //  R3: dL_A^T = -Y dYR^T (strict upper), dM_QA^T = -Y dO^T (inclusive upper) -> dAm
            //  R4: dL_K^T = U dYR^T (strict upper), dM_QK^T = U dO^T (inclusive upper) -> dKm
            // with Am, Km in Bt0, Bt1 for R1, R2 and Kp, Qp for R3, R4.
#pragma unroll 1
            for (int r = 0; r < 4; ++r) {
                if (r == 2) {  // Kp -> Bt0, Qp -> Bt1; q and gamma of the half come by TMA into Bt1 first
                    if (tid == 0) {
                        const int z = b * p.T + n * kC;
                        mbar_arrive_expect_tx(&s.bar[B2Q], 2 * kT16Block);
                        tma_load_3d(Bt1, &p.tq, 64 * hj, hd, z, &s.bar[B2Q]);
                        tma_load_3d(Bt1 + kT16Block, &p.tgam, 64 * hj, hd, z, &s.bar[B2Q]);
                        round_issue(2);
                    }
                    float kv[16], qv[16], gv[16], kp[16], qp[16];
                    ld_chunk16<true>(Kt, t, 2 * g4, kv); ld_chunk16<true>(Kt, t, 2 * g4 + 1, kv + 8);
                    if (!cta_wait(&s.bar[B2Q], (uint32_t)hj) && tid == 0) atomicOr(&s.bad, 1 << 29);
                    ld_chunk16<true>(Bt1, t, 2 * g4, qv); ld_chunk16<true>(Bt1, t, 2 * g4 + 1, qv + 8);
                    ld_chunk16<true>(Bt1, t, 8 + 2 * g4, gv); ld_chunk16<true>(Bt1, t, 9 + 2 * g4, gv + 8);
                    __syncthreads();  // every thread has its q, gamma before Qp overwrites Bt1
                    if (QKRAW) {
                        prologue8(kv, rk); prologue8(kv + 8, rk);
                        prologue8(qv, rq); prologue8(qv + 8, rq);
                    }
                    float p16[16];
                    lds8(&s.P2[j0], p16); lds8(&s.P2[j0 + 8], p16 + 8);
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const float ep = ex2(L[u] - p16[u]);
                        kp[u] = kv[u] * ep;
                        qp[u] = qv[u] * gv[u] * ep;
                    }
                    put_t(Bt0, r0, kp);
                    put_t(Bt1, r0, qp);
                    fence_async_smem();
                } else if (r != 0 && tid == 0) {
                    round_issue(r);
                }
                round_finish(r);
            }
            // ---- readout: final gradients of channels j0 .. j0 + 15 of row t.
            // e (Bt0) and q, gamma (Bt1) of the half come by TMA into the
            // operand tiles, free now (k has its own tile); each thread forms
            // its gradients in its own inputs' places (dk in the free block of
            // Bt0) and the tiles leave by TMA store.
            if (tid == 0) {
                const int z = b * p.T + n * kC;
                mbar_arrive_expect_tx(&s.bar[B2X], 3 * kT16Block);
                tma_load_3d(Bt0 + kT16Block, &p.te, 64 * hj, hd, z, &s.bar[B2X]);
                tma_load_3d(Bt1, &p.tq, 64 * hj, hd, z, &s.bar[B2X]);
                tma_load_3d(Bt1 + kT16Block, &p.tgam, 64 * hj, hd, z, &s.bar[B2X]);
                // the second half's rounds were the tiles' last readers; the next
                // chunk's tiles queue behind the readout's inputs
                if (hj == 1 && c + (int)gridDim.x < nch) load_tiles(c + gridDim.x);
            }
            if (hj == 1 && tid < 4 * p.nslab && c + (int)gridDim.x < nch)  // the next chunk's dLbar partials -> L2
                prefetch_l2(p.dgb + ((size_t)(tid >> 2) * nch + c + gridDim.x) * kD + 32 * (tid & 3));
            {
                const size_t scb = psc(c, t, j0);  // channels j0 .. +16 share a group
                const float s_q = __ldg(p.sq + scb), s_k = __ldg(p.sk + scb);
                const float s_a = __ldg(p.sa + scb), s_d = __ldg(p.sd + scb);
                float dL[16];
                float dotq = 0.f, dotk = 0.f;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {  // 8 channels at a time
                    const int u0 = 8 * hh, ci = 2 * g4 + hh;  // ci: the 8-channel chunk in the half's tiles
                    float a_kp[8], a_q[8], a_a[8], a_km[8];
                    tmem_ld8(taddr(tm, 32 * q, 256 + 16 * g4 + u0), a_kp);
                    tmem_ld8(taddr(tm, 32 * q, 320 + 16 * g4 + u0), a_q);
                    tmem_ld8(taddr(tm, 32 * q, 384 + 16 * g4 + u0), a_a);
                    tmem_ld8(taddr(tm, 32 * q, 448 + 16 * g4 + u0), a_km);
                    float pq[8], pk[8], pa[8], pl[8];
                    const size_t pg = pgrp(c, t, j0 + u0);
                    unpack8_scaled(__ldg(reinterpret_cast<const uint4*>(p.Pq) + pg), s_q, pq);
                    unpack8_scaled(__ldg(reinterpret_cast<const uint4*>(p.Pk) + pg), s_k, pk);
                    unpack8_scaled(__ldg(reinterpret_cast<const uint4*>(p.Pa) + pg), s_a, pa);
                    unpack8_scaled(__ldg(reinterpret_cast<const uint4*>(p.Pd) + pg), s_d, pl);
                    tmem_wait_ld();
                    if (hh == 0 && !cta_wait(&s.bar[B2X], (uint32_t)hj) && tid == 0) atomicOr(&s.bad, 1 << 27);
                    float kv[8], ev[8], qv[8], gv[8];
                    ld_chunk16<true>(Kt, t, ci, kv);
                    ld_chunk16<true>(Bt0, t, 8 + ci, ev);
                    ld_chunk16<true>(Bt1, t, ci, qv);
                    ld_chunk16<true>(Bt1, t, 8 + ci, gv);
                    if (QKRAW) { prologue8(kv, rk); prologue8(qv, rq); }
                    float oq[8], og[8], ok[8], oe[8];
                    float p8[8];
                    lds8(&s.P2[j0 + u0], p8);
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int j = u0 + u;
                        const float ep = ex2(L[j] - p8[u]);
                        const float em = ex2(p8[u] - L[j]);
                        const float qh = qv[u] * gv[u];
                        const float dqh = a_q[u] * ep + pq[u];
                        oq[u] = dqh * gv[u];
                        og[u] = dqh * qv[u];
                        const float da = a_a[u] * em + pa[u];
                        oe[u] = da * kv[u];
                        ok[u] = a_kp[u] * ep + a_km[u] * em + pk[u] + ev[u] * da;
                        // dKp Kp + dQp Qp - dKm Km - dAm Am, plus the state-side part
                        // dK~ K~ + dQ~ Q~ - dKbar Kbar - dAbar Abar = Pd k + Pq q^ - Pa a
                        dL[j] = (a_kp[u] * kv[u] + a_q[u] * qh) * ep -
                                (a_km[u] * kv[u] + a_a[u] * ev[u] * kv[u]) * em +
                                pl[u] * kv[u] + pq[u] * qh - pa[u] * ev[u] * kv[u];
                    }
                    if (QKRAW) {  // dq^, dk^ (fp32, for the last pass) and row dots
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            dotq = fmaf(oq[u], qv[u], dotq);
                            dotk = fmaf(ok[u], kv[u], dotk);
                        }
                        float* qhb = p.dqh + (size_t)c * kC * kD;
                        float* khb = p.dkh + (size_t)c * kC * kD;
                        *grp4(qhb, t, j0 + u0) = make_float4(oq[0], oq[1], oq[2], oq[3]);
                        *grp4(qhb, t, j0 + u0 + 4) = make_float4(oq[4], oq[5], oq[6], oq[7]);
                        *grp4(khb, t, j0 + u0) = make_float4(ok[0], ok[1], ok[2], ok[3]);
                        *grp4(khb, t, j0 + u0 + 4) = make_float4(ok[4], ok[5], ok[6], ok[7]);
                    } else {
                        st_chunk16<true>(Bt1, t, ci, oq);  // dq over q
                        st_chunk16<true>(Bt0, t, ci, ok);  // dk over k
                    }
                    st_chunk16<true>(Bt1, t, 8 + ci, og);  // dgamma over gamma
                    st_chunk16<true>(Bt0, t, 8 + ci, oe);  // de over e
                }
                fence_async_smem();  // (the barrier below publishes the tiles to the stores)
                if (QKRAW) {
                    s.dot[0][4 * hj + g4][t] = dotq;
                    s.dot[1][4 * hj + g4][t] = dotk;
                }
                // dg_t = sum_{t' >= t} dL_t' + dLbar: warp suffix scan, then later quarters
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float o = __shfl_down_sync(0xffffffffu, dL[j], off);
                        if (lane + off < 32) dL[j] += o;
                    }
                }
                if (lane == 0) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) s.sfx[q][j0 + j] = dL[j];
                }
                __syncthreads();
                if (tid == 0) {
                    const int z = b * p.T + n * kC;
                    if (!QKRAW) {
                        tma_store_3d(&p.tdq, Bt1, 64 * hj, hd, z);
                        tma_store_3d(&p.tdk, Bt0, 64 * hj, hd, z);
                    }
                    tma_store_3d(&p.tdgam, Bt1 + kT16Block, 64 * hj, hd, z);
                    tma_store_3d(&p.tde, Bt0 + kT16Block, 64 * hj, hd, z);
                    bulk_commit();
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float o[8], post[8];
                    lds8(&s.dgb[j0 + 8 * hh], post);
                    for (int qq = q + 1; qq < 4; ++qq) {
                        float f8[8];
                        lds8(&s.sfx[qq][j0 + 8 * hh], f8);
#pragma unroll
                        for (int u = 0; u < 8; ++u) post[u] += f8[u];
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int j = 8 * hh + u;
                        // the clamp g >= -20 passes no gradient below it
                        o[u] = ((gkeep >> j) & 1u) ? dL[j] + post[u] : 0.f;
                    }
                    st8_bf16(reinterpret_cast<__nv_bfloat16*>(p.dg) + tok * kD + j0 + 8 * hh, o);
                }
            }
            // the stores have left Bt0, Bt1 before the next half writes them (after
            // the second half, before the next chunk's first half)
            if (hj == 0 && tid == 0) bulk_wait_read();
            sync_all();
        }
        if (QKRAW) {
            // the prologue's Jacobian: dx = SiLU'(x) r (dy^ - y^ (y^ . dy^)), row t,
            // channels 32 g4 .. +32 (dy^ written above by this block; its barrier
            // makes the writes visible)
            float dq_dot = 0.f, dk_dot = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                dq_dot += s.dot[0][i][t];
                dk_dot += s.dot[1][i][t];
            }
            const size_t ro = tok * kD + 32 * g4;
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                const float* dyb = (which ? p.dkh : p.dqh) + (size_t)c * kC * kD;
                const __nv_bfloat16* xr = reinterpret_cast<const __nv_bfloat16*>(which ? p.k : p.q) + ro;
                __nv_bfloat16* dx = reinterpret_cast<__nv_bfloat16*>(which ? p.dk : p.dq) + ro;
                const float r = which ? rk : rq, dot = which ? dk_dot : dq_dot;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float xv[8], o[8];
                    ld8_bf16(xr + 8 * i, xv);
                    const float4 a0 = *grp4(dyb, t, 32 * g4 + 8 * i);
                    const float4 a1 = *grp4(dyb, t, 32 * g4 + 8 * i + 4);
                    const float dv8[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float sg = sigmoid_f(xv[u]);
                        const float yh = xv[u] * sg * r;
                        o[u] = (dv8[u] - yh * dot) * r * sg * (1.f + xv[u] * (1.f - sg));
                    }
                    st8_bf16(dx + 8 * i, o);
                }
            }
            sync_all();
        }
    }
    if (tid == 0) bulk_wait_all();
    if (tid == 0 && s.bad) atomicOr(&g_bwd2_timeouts, (unsigned)s.bad);
    sync_all();
    if (warp == 0) tmem_dealloc(tm, 512);
}

// ------------------------------------------------------------------ host side

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

constexpr int kBprepSmem = 2 * kT16Bytes + 1024;
constexpr int kBwd1Smem = 6 * kT16Bytes + sizeof(Bwd1Smem) + 1024;
constexpr int kBwd2Smem = 4 * kT16Bytes + 2 * kT32Half + kT16Block + sizeof(Bwd2Smem) + 1024;
static_assert(kBwd2Smem <= 232448, "k2_bwd2 shared memory");
template <int SLAB>
constexpr int rev_smem() { return 3 * 128 * 128 * 4 + SLAB * 512 + 1024; }

}  // namespace

size_t bwd2_ws_bytes(int B, int T, int H) {
    const size_t nch = (size_t)B * H * (T / kC), blk = (size_t)kC * kD * 4;
    // Bp, dSc, dq^, dk^ (fp32 blocks), Pq, Pk, Pa, Pd (fp16 blocks) and their
    // group scales, Y16, dYR16 (fp16 tiles), dLbar per value slab (up to 8)
    return nch * (4 * blk + 4 * blk / 2 + 4 * (size_t)kC * 16 + 2 * (size_t)kT16Bytes + 8 * kD * 4) + 256;
}

cudaError_t run_bwd2(const Bwd2Args& a, cudaStream_t st) {
    const int N = a.T / kC, nch = a.B * a.H * N, BH = a.B * a.H;
    const size_t blk = (size_t)kC * kD;
    float* f = reinterpret_cast<float*>(a.ws);
    float* Bp = f; f += nch * blk;
    float* dSc = f; f += nch * blk;
    float* dqh = f; f += nch * blk;
    float* dkh = f; f += nch * blk;
    __half* P16[4];
    for (int i = 0; i < 4; ++i) { P16[i] = reinterpret_cast<__half*>(f); f += nch * blk / 2; }
    float* Psc[4];
    for (int i = 0; i < 4; ++i) { Psc[i] = f; f += (size_t)nch * kC * 4; }
    const int SLAB = chain_slab(BH);  // column slabs of the reverse state pass
    float* dgb = f; f += (size_t)(kD / SLAB) * nch * kD;
    unsigned char* Y16 = reinterpret_cast<unsigned char*>(f);
    unsigned char* dYR16 = Y16 + (size_t)nch * kT16Bytes;
    const int nsm = sm_count();
    cudaError_t e;

    // with a fused output gate, k2_bprep reads the gated output's gradient and
    // writes the mixer's dO (dO_eff), which the later kernels read
    CUtensorMap tdO, tdO_in;
    if (!map_tokens16(&tdO_in, a.dO, a.B, a.T, a.H)) return cudaErrorInvalidValue;
    if (a.zo) {
        if (!a.o_pre || !a.dO_eff || !a.dzo) return cudaErrorInvalidValue;
        if (!map_tokens16(&tdO, a.dO_eff, a.B, a.T, a.H)) return cudaErrorInvalidValue;
    } else {
        tdO = tdO_in;
    }

    BprepParams bp;
    bp.tdO = tdO_in; bp.T = a.T; bp.H = a.H; bp.Qp = a.Qp; bp.Bp = Bp;
    bp.zo = a.zo; bp.o_pre = a.o_pre; bp.o_pre_f32 = a.o_pre_f32; bp.dO_eff = a.dO_eff;
    bp.dO_effb = a.dO_effb; bp.dzo = a.dzo;
    if (a.zo && !a.dO_effb) return cudaErrorInvalidValue;
    if ((e = cudaFuncSetAttribute(k2_bprep, cudaFuncAttributeMaxDynamicSharedMemorySize, kBprepSmem)) != cudaSuccess) return e;
    MUIR_TIMED("k2_bprep", st, k2_bprep<<<nch, 256, kBprepSmem, st>>>(bp));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    RevParams rp;
    if (!map_rows32f(&rp.tMt, a.Mt, (long long)nch * kD)) return cudaErrorInvalidValue;
    rp.Bp = Bp; rp.S_chunks = a.S_chunks; rp.S_last = a.S_last; rp.dS_final = a.dS_final;
    rp.dSc = dSc; rp.dS0 = a.dS0; rp.dgb = dgb; rp.N = N; rp.nch = nch;
    if (SLAB == 16) {
        if ((e = cudaFuncSetAttribute(k2_chain_rev<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, rev_smem<16>())) != cudaSuccess) return e;
        MUIR_TIMED("k2_chain_rev", st, k2_chain_rev<16><<<BH * (kD / 16), 128, rev_smem<16>(), st>>>(rp));
    } else {
        if ((e = cudaFuncSetAttribute(k2_chain_rev<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, rev_smem<32>())) != cudaSuccess) return e;
        MUIR_TIMED("k2_chain_rev", st, k2_chain_rev<32><<<BH * (kD / 32), 128, rev_smem<32>(), st>>>(rp));
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    const int grid = nch < nsm ? nch : nsm;
    Bwd1Params p1;
    p1.tdO = tdO; p1.B = a.B; p1.T = a.T; p1.H = a.H;
    if (!map_tokens16(&p1.tg, a.g, a.B, a.T, a.H) || !map_tokens16(&p1.tv, a.v, a.B, a.T, a.H) ||
        !map_tokens16(&p1.tw, a.w, a.B, a.T, a.H) || !map_tokens16(&p1.tdv, a.dv, a.B, a.T, a.H) ||
        !map_tokens16(&p1.tdw, a.dw, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    p1.q = a.q; p1.k = a.k; p1.v = a.v; p1.g = a.g; p1.e = a.e; p1.w = a.w; p1.gamma = a.gamma;
    p1.aux = a.aux; p1.S_chunks = a.S_chunks; p1.dSc = dSc;
    p1.Pq = P16[0]; p1.Pk = P16[1]; p1.Pa = P16[2]; p1.Pd = P16[3];
    p1.sq = Psc[0]; p1.sk = Psc[1]; p1.sa = Psc[2]; p1.sd = Psc[3];
    p1.Y16 = Y16; p1.dYR16 = dYR16;
    p1.dv = a.dv; p1.dw = a.dw;
    p1.dO_f16 = a.zo != nullptr;
    if ((e = cudaFuncSetAttribute(k2_bwd1, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwd1Smem)) != cudaSuccess) return e;
    MUIR_TIMED("k2_bwd1", st, k2_bwd1<<<grid, 512, kBwd1Smem, st>>>(p1));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    Bwd2Params p2;
    p2.tdO = tdO; p2.B = a.B; p2.T = a.T; p2.H = a.H;
    if (!map_tokens16(&p2.tg, a.g, a.B, a.T, a.H)) return cudaErrorInvalidValue;
    p2.q = a.q; p2.k = a.k; p2.g = a.g; p2.e = a.e; p2.gamma = a.gamma;
    p2.aux = a.aux; p2.Y16 = Y16; p2.dYR16 = dYR16;
    p2.Pq = P16[0]; p2.Pk = P16[1]; p2.Pa = P16[2]; p2.Pd = P16[3];
    p2.sq = Psc[0]; p2.sk = Psc[1]; p2.sa = Psc[2]; p2.sd = Psc[3];
    p2.dqh = dqh; p2.dkh = dkh;
    p2.dgb = dgb; p2.nslab = kD / SLAB;
    p2.dq = a.dq; p2.dk = a.dk; p2.dg = a.dg; p2.de = a.de; p2.dgamma = a.dgamma;
    p2.rnorm = a.rnorm;
    if (!map_tokens16(&p2.tk, a.k, a.B, a.T, a.H) || !map_tokens16(&p2.te, a.e, a.B, a.T, a.H) ||
        !map_tokens16(&p2.tq, a.q, a.B, a.T, a.H) || !map_tokens16(&p2.tgam, a.gamma, a.B, a.T, a.H) ||
        !map_tokens16(&p2.tdgam, a.dgamma, a.B, a.T, a.H) || !map_tokens16(&p2.tde, a.de, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    if (!a.rnorm && (!map_tokens16(&p2.tdq, a.dq, a.B, a.T, a.H) || !map_tokens16(&p2.tdk, a.dk, a.B, a.T, a.H)))
        return cudaErrorInvalidValue;
    p2.flags = a.flags;
    p2.dO_f16 = a.zo != nullptr;
    if (!a.flags) return cudaErrorInvalidValue;
    auto k2 = a.rnorm ? k2_bwd2<true> : k2_bwd2<false>;
    if ((e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwd2Smem)) != cudaSuccess) return e;
    MUIR_TIMED("k2_bwd2", st, k2<<<grid, 512, kBwd2Smem, st>>>(p2));
    return cudaGetLastError();
}

unsigned int timeouts_bwd2() {
    unsigned int n = 0;
    cudaMemcpyFromSymbol(&n, g_bwd2_timeouts, sizeof(n));
    const unsigned int z = 0;
    cudaMemcpyToSymbol(g_bwd2_timeouts, &z, sizeof(z));
    return n;
}

}  // namespace v2
}  // namespace muir

// gates.cu -- the fused low-rank gate projection ("Muir", wolonglab.org page,
// "Methodology", eq:ours_proj; fig. 3(c)): one latent row per token, shared by
// every head, and per gate family X an up-projection U_X [r_X][H*128] with a
// channel bias, so that pre_X[t][h][c] = sum_i a[t][off_X + i] U_X[i][128h + c]
// + bias_X[128h + c]; the gates are -softplus(pre) (log decay), sigmoid(pre)
// (erase, write, readout gain) or pre itself (the output gate's
// pre-activation), stored in bf16 like gate inputs.
//
//   k2_gates       one CTA per 128-token tile: the latent slices are staged
//                  once by TMA, each head's U tile streams through a two-stage
//                  ring, the up-projection runs on tcgen05 (bf16 operands,
//                  fp32 in tensor memory, two accumulators so one head's
//                  epilogue overlaps the next head's product) and the epilogue
//                  adds the bias, applies the activation and stores the gate.
//   k2_gates_dpre  backward, one CTA per token tile: recomputes pre, forms
//                  dpre = dgate act'(pre) as a bf16 pair hi + lo (written out
//                  for k2_gates_dw) and accumulates dlatent = sum_h dpre_h U_h^T
//                  over the heads in tensor memory (one product per half).
//   k2_gates_dw    backward, one CTA per (family, head): dU^T = sum over every
//                  token tile of dpre^T a (both halves; tcgen05, accumulated in
//                  tensor memory) and dbias = column sums of hi + lo.  The pair
//                  keeps about 16 bits of dpre through the token sums.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bwd2.h"
#include "gates.h"
#include "profile.h"
#include "tc2.cuh"

namespace muir {
namespace v2 {

using namespace t2;

__device__ unsigned int g_gates_timeouts;

namespace {

constexpr int kMaxFam = 5;
constexpr uint32_t kBlk = 16384;  // one 64-column block of a 128-row T16 tile

struct GatesFwdParams {
    CUtensorMap tlat;
    CUtensorMap tU[kMaxFam];
    CUtensorMap tout[kMaxFam];  // with stage: the gates as token-major bf16 tiles
    int stage;                  // 1: the epilogue stages each head's tile and stores it by TMA
    int nfam, H;
    int off[kMaxFam], r[kMaxFam], act[kMaxFam];
    const float* bias[kMaxFam];
    __nv_bfloat16* out[kMaxFam];
};

struct GatesDpreParams {
    CUtensorMap tlat;
    CUtensorMap tU[kMaxFam];
    CUtensorMap tdo[kMaxFam];            // dgate as token-major bf16 tiles (loaded)
    CUtensorMap tdh[kMaxFam], tdlo[kMaxFam];  // dpre hi, lo (stored)
    int nfam, H, R;
    int off[kMaxFam], r[kMaxFam], act[kMaxFam];
    const float* bias[kMaxFam];
    const __nv_bfloat16* dout[kMaxFam];
    __nv_bfloat16* dpre[kMaxFam];
    __nv_bfloat16* dpre_lo[kMaxFam];
    __nv_bfloat16* dlat;
};

struct GatesDwParams {
    CUtensorMap tlat;
    CUtensorMap tdp[kMaxFam], tdl[kMaxFam];  // dpre hi, lo
    int H, ntile;
    int off[kMaxFam], r[kMaxFam];
    float* dU[kMaxFam];
    float* dbias[kMaxFam];
};

__device__ __forceinline__ void sync_all() {
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
}

// (fast intrinsics: the gates are stored in bf16)
__device__ __forceinline__ float act_f(int act, float x) {
    if (act == kActNegSoftplus) return -(fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x))));
    if (act == kActSigmoid) return sigmoid_f(x);
    return x;
}

__device__ __forceinline__ float act_grad(int act, float x) {
    if (act == kActNegSoftplus) return -sigmoid_f(x);
    if (act == kActSigmoid) {
        const float s = sigmoid_f(x);
        return s * (1.f - s);
    }
    return 1.f;
}

__device__ __forceinline__ void st8_bf16g(__nv_bfloat16* p, const float* v) {
    uint4 u;
    u.x = pack_bf16(v[0], v[1]);
    u.y = pack_bf16(v[2], v[3]);
    u.z = pack_bf16(v[4], v[5]);
    u.w = pack_bf16(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = u;
}

__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
    return (unsigned char*)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

}  // namespace

// ------------------------------------------------------------------ forward

// 512 threads: warp w reads TMEM lanes 32 (w % 4) .. (rows t) and columns
// 32 (w / 4) .. +32 (channels); thread 0 issues the copies and the products.
__global__ void __launch_bounds__(512, 1) k2_gates(const __grid_constant__ GatesFwdParams p) {
    extern __shared__ unsigned char smraw[];
    unsigned char* sm = align1024(smraw);
    __shared__ uint64_t barA, barU[2], barM[2];
    __shared__ uint32_t tslot;
    __shared__ int bad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, half = warp >> 2, t = 32 * q + lane;
    const long long row0 = (long long)blockIdx.x * 128;
    int ablk[kMaxFam], nA = 0;
    for (int X = 0; X < p.nfam; ++X) {
        ablk[X] = nA;
        nA += p.r[X] / 64;
    }
    unsigned char* A = sm;
    unsigned char* U = sm + nA * kBlk;  // two stages of two blocks
    unsigned char* O = U + 4 * kBlk;    // with stage: one head's output tile (T16)
    if (tid == 0) {
        mbar_init(&barA, 1);
        for (int s = 0; s < 2; ++s) { mbar_init(&barU[s], 1); mbar_init(&barM[s], 1); }
        bad = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(&tslot, 256);
    sync_all();
    const uint32_t tm = tslot;
    const int n = p.nfam * p.H;
    auto load_U = [&](int idx, int s) {
        const int X = idx / p.H, h = idx % p.H;
        mbar_arrive_expect_tx(&barU[s], 2u * p.r[X] * 128u);
        tma_load_3d(U + s * 2 * kBlk, &p.tU[X], 128 * h, 0, 0, &barU[s]);
        tma_load_3d(U + s * 2 * kBlk + kBlk, &p.tU[X], 128 * h + 64, 0, 0, &barU[s]);
    };
    auto issue = [&](int idx) {
        const int s = idx & 1, X = idx / p.H;
        if (!mbar_wait(&barU[s], (uint32_t)((idx >> 1) & 1))) bad = 1;
        tc_fence_after();
        gemm_km16(tm + 128 * s, saddr(A + ablk[X] * kBlk), 0, saddr(U + s * 2 * kBlk), 0, 0, 128,
                  p.r[X], kBF16, false);
        mma_commit(&barM[s]);
    };
    if (tid == 0) {
        uint32_t bytes = 0;
        for (int X = 0; X < p.nfam; ++X) bytes += (uint32_t)p.r[X] * 128u * 2u;
        mbar_arrive_expect_tx(&barA, bytes);
        for (int X = 0; X < p.nfam; ++X)
            for (int j = 0; j < p.r[X] / 64; ++j)
                tma_load_3d(A + (ablk[X] + j) * kBlk, &p.tlat, p.off[X] + 64 * j, (int)row0, 0, &barA);
        load_U(0, 0);
        if (n > 1) load_U(1, 1);
        if (!mbar_wait(&barA, 0)) bad = 1;
        issue(0);
    }
    for (int idx = 0; idx < n; ++idx) {
        const int s = idx & 1, X = idx / p.H, h = idx % p.H;
        if (tid == 0 && idx + 1 < n) issue(idx + 1);  // into the other accumulator
        if (p.stage && tid == 0) bulk_wait_read();   // the previous tile has left O (the wait below tells the rest)
        if (!cta_wait(&barM[s], (uint32_t)((idx >> 1) & 1)) && tid == 0) bad = 1;
        if (tid == 0 && idx + 2 < n) load_U(idx + 2, s);  // product idx has read stage s
        float v[32];
        tmem_ld32(taddr(tm, 32 * q, 128 * s + 32 * half), v);
        tmem_wait_ld();
        const float* bias = p.bias[X] + 128 * h + 32 * half;
        __nv_bfloat16* dst = p.out[X] + ((row0 + t) * p.H + h) * 128 + 32 * half;
        const int act = p.act[X];
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
            float o[8];
            const float4 b0 = __ldg(reinterpret_cast<const float4*>(bias + j));  // (bias 16-byte aligned)
            const float4 b1 = __ldg(reinterpret_cast<const float4*>(bias + j + 4));
            const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int u = 0; u < 8; ++u) o[u] = act_f(act, v[j + u] + bb[u]);
            if (p.stage)
                st_chunk16<true>(O, t, 4 * half + j / 8, o);
            else
                st8_bf16g(dst + j, o);
        }
        if (p.stage) fence_async_smem();
        sync_all();  // accumulator s read out before product idx + 2 overwrites it; tile complete
        if (p.stage && tid == 0) {
            tma_store_3d(&p.tout[X], O, 0, h, (int)row0);
            tma_store_3d(&p.tout[X], O + kBlk, 64, h, (int)row0);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait_all();
    if (tid == 0 && bad) atomicOr(&g_gates_timeouts, 1u);
    sync_all();
    if (warp == 0) tmem_dealloc(tm, 256);
}

// ------------------------------------------------------------------ backward

// dpre = dgate act'(pre) and dlatent, one 128-token tile per CTA; 512
// threads (warp w: TMEM lanes 32 (w % 4) .., channels 32 (w / 4) ..).
__global__ void __launch_bounds__(512, 1) k2_gates_dpre(const __grid_constant__ GatesDpreParams p) {
    extern __shared__ unsigned char smraw[];
    unsigned char* sm = align1024(smraw);
    unsigned char* A = sm;                 // the family's latent slice (2 blocks)
    unsigned char* U = sm + 2 * kBlk;      // two stages of two blocks
    unsigned char* Dp = sm + 6 * kBlk;     // dpre of one head, bf16 T16: hi, then lo (stored by TMA)
    unsigned char* Do = sm + 10 * kBlk;    // dgate of a head, two stages of a T16 tile
    __shared__ uint64_t barA, barU[2], barM, barD[2];
    __shared__ uint32_t tslot;
    __shared__ int bad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, half = warp >> 2, t = 32 * q + lane;
    const long long row0 = (long long)blockIdx.x * 128;
    if (tid == 0) {
        mbar_init(&barA, 1);
        mbar_init(&barU[0], 1);
        mbar_init(&barU[1], 1);
        mbar_init(&barM, 1);
        mbar_init(&barD[0], 1);
        mbar_init(&barD[1], 1);
        bad = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(&tslot, 256);
    sync_all();
    const uint32_t tm = tslot;  // columns 0..127: pre; 128..255: dlatent of the family
    uint32_t pm = 0;
    const int n = p.nfam * p.H;
    auto load_D = [&](int idx) {  // dgate of (family, head) idx -> stage idx & 1
        const int s = idx & 1, X = idx / p.H, h = idx % p.H;
        mbar_arrive_expect_tx(&barD[s], 2 * kBlk);
        tma_load_3d(Do + s * 2 * kBlk, &p.tdo[X], 0, h, (int)row0, &barD[s]);
        tma_load_3d(Do + s * 2 * kBlk + kBlk, &p.tdo[X], 64, h, (int)row0, &barD[s]);
    };
    if (tid == 0) {
        load_D(0);
        if (n > 1) load_D(1);
    }
    auto load_U = [&](int idx) {
        const int s = idx & 1, X = idx / p.H, h = idx % p.H;
        mbar_arrive_expect_tx(&barU[s], 2u * p.r[X] * 128u);
        tma_load_3d(U + s * 2 * kBlk, &p.tU[X], 128 * h, 0, 0, &barU[s]);
        tma_load_3d(U + s * 2 * kBlk + kBlk, &p.tU[X], 128 * h + 64, 0, 0, &barU[s]);
    };
    for (int X = 0; X < p.nfam; ++X) {
        const int r = p.r[X], act = p.act[X];
        if (tid == 0) {
            mbar_arrive_expect_tx(&barA, (uint32_t)r * 256u);
            for (int j = 0; j < r / 64; ++j)
                tma_load_3d(A + j * kBlk, &p.tlat, p.off[X] + 64 * j, (int)row0, 0, &barA);
            load_U(X * p.H);
            if (p.H > 1) load_U(X * p.H + 1);
            if (!mbar_wait(&barA, (uint32_t)(X & 1))) bad = 1;
        }
        for (int h = 0; h < p.H; ++h) {
            const int idx = X * p.H + h, s = idx & 1;
            if (tid == 0) {
                if (!mbar_wait(&barU[s], (uint32_t)((idx >> 1) & 1))) bad = 1;
                tc_fence_after();
                gemm_km16(tm, saddr(A), 0, saddr(U + s * 2 * kBlk), 0, 0, 128, r, kBF16, false);
                mma_commit(&barM);
            }
            if (tid == 0) bulk_wait_read();  // the previous head's dpre tiles have left Dp
            {  // the product and this head's dgate tile; one block barrier releases all
                int ok = 1;
                if (tid < 32) ok = (mbar_wait(&barM, pm) && mbar_wait(&barD[s], (uint32_t)((idx >> 1) & 1))) ? 1 : 0;
                ok = __syncthreads_and(ok);
                tc_fence_after();
                if (!ok && tid == 0) bad = 1;
            }
            pm ^= 1u;
            {  // dpre of row t, channels 32 half .. +32 -> the Dp tiles
                float v[32];
                tmem_ld32(taddr(tm, 32 * q, 32 * half), v);
                tmem_wait_ld();
                const float* bias = p.bias[X] + 128 * h + 32 * half;
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                    float dg[8], hi[8], lo[8];
                    ld_chunk16<true>(Do + s * 2 * kBlk, t, 4 * half + j / 8, dg);
                    const float4 b0 = __ldg(reinterpret_cast<const float4*>(bias + j));
                    const float4 b1 = __ldg(reinterpret_cast<const float4*>(bias + j + 4));
                    const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float o = dg[u] * act_grad(act, v[j + u] + bb[u]);
                        hi[u] = __bfloat162float(__float2bfloat16_rn(o));
                        lo[u] = o - hi[u];
                    }
                    st_chunk16<true>(Dp, t, 4 * half + j / 8, hi);
                    st_chunk16<true>(Dp + 2 * kBlk, t, 4 * half + j / 8, lo);
                }
            }
            fence_async_smem();
            sync_all();
            if (tid == 0) {  // dpre hi, lo leave by TMA store; the next-but-one dgate tile into stage s
                tma_store_3d(&p.tdh[X], Dp, 0, h, (int)row0);
                tma_store_3d(&p.tdh[X], Dp + kBlk, 64, h, (int)row0);
                tma_store_3d(&p.tdlo[X], Dp + 2 * kBlk, 0, h, (int)row0);
                tma_store_3d(&p.tdlo[X], Dp + 3 * kBlk, 64, h, (int)row0);
                bulk_commit();
                if (idx + 2 < n) load_D(idx + 2);
            }
            if (tid == 0) {  // dlatent (+)= dpre U_h^T: A = Dp (K = channels), B = U (rows i, K = channels)
                gemm_kk16(tm + 128, saddr(Dp), 0, saddr(U + s * 2 * kBlk), 0, 0, r, 128, kBF16, h > 0);
                gemm_kk16(tm + 128, saddr(Dp + 2 * kBlk), 0, saddr(U + s * 2 * kBlk), 0, 0, r, 128, kBF16, true);
                mma_commit(&barM);
            }
            if (!cta_wait(&barM, pm) && tid == 0) bad = 1;
            pm ^= 1u;
            if (tid == 0 && h + 2 < p.H) load_U(idx + 2);  // both products of head h read stage s
        }
        {  // dlatent of row t: columns off .. off + r (a quarter of them per thread)
            const int w = r / 4;  // 16 or 32
            float v[32];
            tmem_ld32(taddr(tm, 32 * q, 128 + w * half), v);  // w <= 32 columns used
            tmem_wait_ld();
            __nv_bfloat16* dst = p.dlat + (size_t)(row0 + t) * p.R + p.off[X] + w * half;
            st8_bf16g(dst, v);
            st8_bf16g(dst + 8, v + 8);
            if (w == 32) {
                st8_bf16g(dst + 16, v + 16);
                st8_bf16g(dst + 24, v + 24);
            }
        }
        sync_all();
    }
    if (tid == 0) bulk_wait_all();
    if (tid == 0 && bad) atomicOr(&g_gates_timeouts, 2u);
    sync_all();
    if (warp == 0) tmem_dealloc(tm, 256);
}

// dU^T [128 channels][r] of one (family, head), summed over every token tile,
// and dbias; 128 threads (thread c: channel c).
__global__ void __launch_bounds__(128, 1) k2_gates_dw(const __grid_constant__ GatesDwParams p) {
    extern __shared__ unsigned char smraw[];
    unsigned char* sm = align1024(smraw);
    // stage s (6 blocks from 6s): dpre hi (2 blocks), dpre lo (2), latent slice (2)
    __shared__ uint64_t barL[2], barM;
    __shared__ uint32_t tslot;
    __shared__ int bad;
    __shared__ __align__(16) float red[8][128];  // dbias partials of the eight row groups
    const int tid = threadIdx.x, warp = tid >> 5;
    const int X = blockIdx.x / p.H, h = blockIdx.x % p.H, r = p.r[X];
    if (tid == 0) {
        mbar_init(&barL[0], 1);
        mbar_init(&barL[1], 1);
        mbar_init(&barM, 1);
        bad = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(&tslot, 128);
    sync_all();
    const uint32_t tm = tslot;
    auto load = [&](int j) {
        const int s = j & 1;
        unsigned char* base = sm + 6 * s * kBlk;
        mbar_arrive_expect_tx(&barL[s], 4u * kBlk + (uint32_t)r * 256u);
        tma_load_3d(base, &p.tdp[X], 0, h, 128 * j, &barL[s]);
        tma_load_3d(base + kBlk, &p.tdp[X], 64, h, 128 * j, &barL[s]);
        tma_load_3d(base + 2 * kBlk, &p.tdl[X], 0, h, 128 * j, &barL[s]);
        tma_load_3d(base + 3 * kBlk, &p.tdl[X], 64, h, 128 * j, &barL[s]);
        for (int b = 0; b < r / 64; ++b)
            tma_load_3d(base + (4 + b) * kBlk, &p.tlat, p.off[X] + 64 * b, 128 * j, 0, &barL[s]);
    };
    if (tid == 0) {
        load(0);
        if (p.ntile > 1) load(1);
    }
    // dbias: thread (8-channel chunk ch, row group rg) sums its 16 rows of every tile
    const int ch = tid & 15, rg = tid >> 4;
    float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < p.ntile; ++j) {
        const int s = j & 1;
        unsigned char* base = sm + 6 * s * kBlk;
        if (!cta_wait(&barL[s], (uint32_t)((j >> 1) & 1)) && tid == 0) bad = 1;
        if (tid == 0) {  // D[c][i] (+)= sum_t dpre[t][c] a[t][i]: both operands MN-major
            gemm_mm16(tm, saddr(base), 0, 0, saddr(base + 4 * kBlk), 0, 0, r, 128, kBF16, j > 0);
            gemm_mm16(tm, saddr(base + 2 * kBlk), 0, 0, saddr(base + 4 * kBlk), 0, 0, r, 128, kBF16, true);
            mma_commit(&barM);
        }
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {  // rows 16 rg .. +16, channels 8 ch .. +8 (hi + lo)
            float a[8], b[8];
            ld_chunk16<true>(base, 16 * rg + i, ch, a);
            ld_chunk16<true>(base + 2 * kBlk, 16 * rg + i, ch, b);
#pragma unroll
            for (int u = 0; u < 8; ++u) acc8[u] += a[u] + b[u];
        }
        if (!cta_wait(&barM, (uint32_t)(j & 1)) && tid == 0) bad = 1;
        if (tid == 0 && j + 2 < p.ntile) load(j + 2);  // stage s consumed by the product and the sums
    }
    *reinterpret_cast<float4*>(&red[rg][8 * ch]) = make_float4(acc8[0], acc8[1], acc8[2], acc8[3]);
    *reinterpret_cast<float4*>(&red[rg][8 * ch + 4]) = make_float4(acc8[4], acc8[5], acc8[6], acc8[7]);
    __syncthreads();
    float colsum = 0.f;
#pragma unroll
    for (int g = 0; g < 8; ++g) colsum += red[g][tid];  // fixed order
    {
        const int c = tid;
        float* dU = p.dU[X] + 128 * h + c;  // dU[i][128 h + c]
        const size_t ld = (size_t)p.H * 128;
        for (int i0 = 0; i0 < r; i0 += 32) {
            float v[32];
            tmem_ld32(taddr(tm, 32 * warp, i0), v);
            tmem_wait_ld();
            for (int i = 0; i < 32; ++i) dU[(size_t)(i0 + i) * ld] = v[i];
        }
        p.dbias[X][128 * h + c] = colsum;
    }
    if (tid == 0 && bad) atomicOr(&g_gates_timeouts, 4u);
    sync_all();
    if (warp == 0) tmem_dealloc(tm, 128);
}

// ------------------------------------------------------------------ host side

namespace {

bool map_latent(CUtensorMap* m, const void* base, int R, long long rows) {
    return map_2d16(m, base, R, rows, 128);
}

}  // namespace

cudaError_t run_gates_fwd(const GatesArgs& a, cudaStream_t st) {
    if (a.nfam < 1 || a.nfam > kMaxFam || a.rows % 128 || a.R % 8) return cudaErrorInvalidValue;
    GatesFwdParams p;
    p.nfam = a.nfam; p.H = a.H;
    if (!map_latent(&p.tlat, a.latent, a.R, a.rows)) return cudaErrorInvalidValue;
    int nblk = 0;
    for (int X = 0; X < a.nfam; ++X) {
        const GateFamily& f = a.fam[X];
        if ((f.r != 64 && f.r != 128) || f.off % 8 || f.off + f.r > a.R) return cudaErrorInvalidValue;
        if (!map_2d16(&p.tU[X], f.U, a.H * 128, f.r, f.r)) return cudaErrorInvalidValue;
        p.off[X] = f.off; p.r[X] = f.r; p.act[X] = f.act;
        p.bias[X] = f.bias; p.out[X] = static_cast<__nv_bfloat16*>(f.out);
        nblk += f.r / 64;
    }
    // with room for a staged output tile, each head's gates leave by TMA store
    p.stage = (nblk + 6) * (int)kBlk + 1024 <= 232448;
    if (p.stage)
        for (int X = 0; X < a.nfam; ++X)
            if (!map_tokens16(&p.tout[X], a.fam[X].out, 1, (int)a.rows, a.H)) return cudaErrorInvalidValue;
    const int smem = (nblk + (p.stage ? 6 : 4)) * (int)kBlk + 1024;
    cudaError_t e = cudaFuncSetAttribute(k2_gates, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    MUIR_TIMED("k2_gates", st, k2_gates<<<(int)(a.rows / 128), 512, smem, st>>>(p));
    return cudaGetLastError();
}

cudaError_t run_gates_bwd(const GatesArgs& a, cudaStream_t st) {
    if (a.nfam < 1 || a.nfam > kMaxFam || a.rows % 128 || a.R % 8) return cudaErrorInvalidValue;
    GatesDpreParams p;
    GatesDwParams q;
    p.nfam = a.nfam; p.H = a.H; p.R = a.R;
    q.H = a.H; q.ntile = (int)(a.rows / 128);
    if (!map_latent(&p.tlat, a.latent, a.R, a.rows)) return cudaErrorInvalidValue;
    q.tlat = p.tlat;
    p.dlat = static_cast<__nv_bfloat16*>(a.dlatent);
    for (int X = 0; X < a.nfam; ++X) {
        const GateFamily& f = a.fam[X];
        if ((f.r != 64 && f.r != 128) || f.off % 8 || f.off + f.r > a.R) return cudaErrorInvalidValue;
        if (!map_2d16(&p.tU[X], f.U, a.H * 128, f.r, f.r)) return cudaErrorInvalidValue;
        if (!map_tokens16(&q.tdp[X], f.dpre, 1, (int)a.rows, a.H) ||
            !map_tokens16(&q.tdl[X], f.dpre_lo, 1, (int)a.rows, a.H) ||
            !map_tokens16(&p.tdo[X], f.dout, 1, (int)a.rows, a.H))
            return cudaErrorInvalidValue;
        p.tdh[X] = q.tdp[X];
        p.tdlo[X] = q.tdl[X];
        p.off[X] = q.off[X] = f.off; p.r[X] = q.r[X] = f.r; p.act[X] = f.act;
        p.bias[X] = f.bias;
        p.dout[X] = static_cast<const __nv_bfloat16*>(f.dout);
        p.dpre[X] = static_cast<__nv_bfloat16*>(f.dpre);
        p.dpre_lo[X] = static_cast<__nv_bfloat16*>(f.dpre_lo);
        q.dU[X] = f.dU; q.dbias[X] = f.dbias;
    }
    cudaError_t e = cudaMemsetAsync(a.dlatent, 0, (size_t)a.rows * a.R * 2, st);
    if (e != cudaSuccess) return e;
    const int smem1 = 14 * (int)kBlk + 1024;
    if ((e = cudaFuncSetAttribute(k2_gates_dpre, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1)) != cudaSuccess) return e;
    MUIR_TIMED("k2_gates_dpre", st, k2_gates_dpre<<<(int)(a.rows / 128), 512, smem1, st>>>(p));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int smem2 = 12 * (int)kBlk + 1024;
    if ((e = cudaFuncSetAttribute(k2_gates_dw, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2)) != cudaSuccess) return e;
    MUIR_TIMED("k2_gates_dw", st, k2_gates_dw<<<a.nfam * a.H, 128, smem2, st>>>(q));
    return cudaGetLastError();
}

unsigned int timeouts_gates() {
    unsigned int n = 0;
    cudaMemcpyFromSymbol(&n, g_gates_timeouts, sizeof(n));
    const unsigned int z = 0;
    cudaMemcpyToSymbol(g_gates_timeouts, &z, sizeof(z));
    return n;
}

}  // namespace v2
}  // namespace muir

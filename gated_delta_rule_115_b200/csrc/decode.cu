// decode.cu -- single-token decode step of the Muir gated delta rule.
//
// Streaming inference with a resident float32 state ("Muir: Linear Attention
// with Sensitivity-Allocated Gating and Matched-Filter Readout", wolonglab.org
// page, "Experiments": 10M-token streams in a constant float32 state;
// fig:longctx_niah for static readout).  Per (b, h), with D = dk = dv:
//
//     P = diag(exp g) S ;  y = P^T k ;  S <- P - (e*k) y^T + k (w*v)^T ;
//     o = S^T (gamma*q)
//
// The work is bound by HBM: S (D*D*4 bytes) is read once and written once;
// the token vectors are a few hundred bytes.  Two 128-thread CTAs per (b, h):
// thread (rg, cq) keeps a block of rows x 4 columns of S
// in registers (float4 loads and stores), so S never goes through shared
// memory; each (b, h) is split by columns over two CTAs.  The two column reductions (y and o)
// go through a small shared-memory table.
#include "common.cuh"
#include "kernels.h"
#include "profile.h"

namespace muir {

// NCOL columns of one (b, h) per CTA of NT threads: thread (rg, cq) keeps rows
// [rg*RPG, (rg+1)*RPG) x columns [c0 + 4cq, +4) of S in registers.
template <typename Tin, typename Tout, int D, int NCOL, int NT>
__global__ void __launch_bounds__(NT) decode_step_kernel(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
    const Tin* __restrict__ g, const Tin* __restrict__ e, const Tin* __restrict__ w,
    const Tin* __restrict__ gamma, int gamma_static, float* __restrict__ S,
    Tout* __restrict__ o, int H) {
    constexpr int CQ = NCOL / 4;   // column quads per row slice
    constexpr int RG = NT / CQ;    // row groups
    constexpr int RPG = D / RG;    // rows per thread
    constexpr int SPLIT = D / NCOL;
    __shared__ float s_k[D], s_a[D], s_dec[D], s_qh[D];
    __shared__ __align__(16) float s_u[NCOL];
    __shared__ __align__(16) float s_y[NCOL];
    __shared__ float4 s_part[RG][CQ];

    const int bh = blockIdx.x / SPLIT;
    const int cbase = (blockIdx.x % SPLIT) * NCOL;
    const int h = bh % H;
    const size_t tok = (size_t)bh * D;
    const int tid = threadIdx.x;
    const int cq = tid % CQ, rg = tid / CQ;
    const int c0 = cbase + 4 * cq, r0 = rg * RPG;
    float* Sbh = S + (size_t)bh * D * D;
    float4 st[RPG];
#pragma unroll
    for (int i = 0; i < RPG; ++i)
        st[i] = *reinterpret_cast<const float4*>(Sbh + (size_t)(r0 + i) * D + c0);
    for (int j = tid; j < D; j += NT) {
        const float kj = ldf(k + tok + j);
        s_k[j] = kj;
        s_a[j] = ldf(e + tok + j) * kj;
        s_dec[j] = expf(ldf(g + tok + j));
        float gm = 1.0f;
        if (gamma) gm = ldf(gamma + (gamma_static ? (size_t)h * D : tok) + j);
        s_qh[j] = gm * ldf(q + tok + j);
    }
    for (int cc = tid; cc < NCOL; cc += NT)
        s_u[cc] = ldf(w + tok + cbase + cc) * ldf(v + tok + cbase + cc);
    __syncthreads();

    // P = diag(exp g) S and the partial y = P^T k over this thread's rows
    float4 yp = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < RPG; ++i) {
        const float d = s_dec[r0 + i], kj = s_k[r0 + i];
        st[i].x *= d; st[i].y *= d; st[i].z *= d; st[i].w *= d;
        yp.x += st[i].x * kj; yp.y += st[i].y * kj; yp.z += st[i].z * kj; yp.w += st[i].w * kj;
    }
    s_part[rg][cq] = yp;
    __syncthreads();
    for (int cc = tid; cc < NCOL; cc += NT) {
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < RG; ++r) acc += reinterpret_cast<const float*>(&s_part[r][0])[cc];
        s_y[cc] = acc;
    }
    __syncthreads();

    // S = P - a y^T + k u^T ; partial o = S^T qhat
    const float4 y4 = *reinterpret_cast<const float4*>(&s_y[4 * cq]);
    const float4 u4 = *reinterpret_cast<const float4*>(&s_u[4 * cq]);
    float4 op = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < RPG; ++i) {
        const float aj = s_a[r0 + i], kj = s_k[r0 + i], qj = s_qh[r0 + i];
        float4 s = st[i];
        s.x = s.x - aj * y4.x + kj * u4.x;
        s.y = s.y - aj * y4.y + kj * u4.y;
        s.z = s.z - aj * y4.z + kj * u4.z;
        s.w = s.w - aj * y4.w + kj * u4.w;
        *reinterpret_cast<float4*>(Sbh + (size_t)(r0 + i) * D + c0) = s;
        op.x += s.x * qj; op.y += s.y * qj; op.z += s.z * qj; op.w += s.w * qj;
    }
    s_part[rg][cq] = op;  // every read of s_part (the y reduction) finished before the last barrier
    __syncthreads();
    for (int cc = tid; cc < NCOL; cc += NT) {
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < RG; ++r) acc += reinterpret_cast<const float*>(&s_part[r][0])[cc];
        stf(o + tok + cbase + cc, acc);
    }
}

template <typename Tin, typename Tout>
static cudaError_t launch_decode_t(int B, int H, int D, const void* q, const void* k,
                                   const void* v, const void* g, const void* e, const void* w,
                                   const void* gamma, int gamma_static, float* S, void* o,
                                   cudaStream_t st) {
    // two CTAs of 128 threads per (b, h), each on half of the columns: twice the
    // CTAs of one-per-head, which balances the single wave over the 148 SMs
    dim3 grid(B * H * 2), block(128);
#define MUIR_DEC_ARGS                                                                   \
    (const Tin*)q, (const Tin*)k, (const Tin*)v, (const Tin*)g, (const Tin*)e,          \
        (const Tin*)w, (const Tin*)gamma, gamma_static, S, (Tout*)o, H
    if (D == 128)
        MUIR_TIMED("k_decode", st, decode_step_kernel<Tin, Tout, 128, 64, 128><<<grid, block, 0, st>>>(MUIR_DEC_ARGS));
    else
        MUIR_TIMED("k_decode", st, decode_step_kernel<Tin, Tout, 64, 32, 128><<<grid, block, 0, st>>>(MUIR_DEC_ARGS));
#undef MUIR_DEC_ARGS
    return cudaGetLastError();
}

cudaError_t launch_decode(int B, int H, int D, bool in_bf16, bool out_bf16, const void* q,
                          const void* k, const void* v, const void* g, const void* e,
                          const void* w, const void* gamma, int gamma_static, float* S,
                          void* o, cudaStream_t st) {
    if (in_bf16) {
        if (out_bf16)
            return launch_decode_t<__nv_bfloat16, __nv_bfloat16>(B, H, D, q, k, v, g, e, w,
                                                                 gamma, gamma_static, S, o, st);
        return launch_decode_t<__nv_bfloat16, float>(B, H, D, q, k, v, g, e, w, gamma,
                                                     gamma_static, S, o, st);
    }
    if (out_bf16)
        return launch_decode_t<float, __nv_bfloat16>(B, H, D, q, k, v, g, e, w, gamma,
                                                     gamma_static, S, o, st);
    return launch_decode_t<float, float>(B, H, D, q, k, v, g, e, w, gamma, gamma_static, S, o,
                                         st);
}

}  // namespace muir

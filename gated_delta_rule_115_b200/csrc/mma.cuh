// mma.cuh -- warp-level TF32 tensor-core tiles (mma.sync m16n8k8) on operands
// given as element accessors, plus CTA-level tile loops.
//
// PASSES = 1: one TF32 product (inputs rounded to TF32, float32 accumulate).
// PASSES = 3: split-TF32, x = hi + lo with hi = tf32(x), lo = tf32(x - hi);
//             a*b ~ hi_a*hi_b + hi_a*lo_b + lo_a*hi_b, float32-level accuracy.
#pragma once

#include <stdint.h>

namespace muir {

__device__ __forceinline__ uint32_t f2tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4],
                                         const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

template <int PASSES, int N>
__device__ __forceinline__ void split_tf32(const float (&v)[N], uint32_t (&hi)[N],
                                           uint32_t (&lo)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
        hi[i] = f2tf32(v[i]);
        if (PASSES == 3) lo[i] = f2tf32(v[i] - __uint_as_float(hi[i]));
    }
}

// acc[MT][NT] (16*MT x 8*NT tile) += A(16*MT x K) * B(K x 8*NT).
// fa(r, k) returns A[r][k]; fb(k, n) returns B[k][n].  K % 8 == 0.
// Fragment layout (PTX ISA, mma.m16n8k8 .tf32): with g = lane/4, c = lane%4,
//   a = {A[g][c], A[g+8][c], A[g][c+4], A[g+8][c+4]}, b = {B[c][g], B[c+4][g]},
//   d = {D[g][2c], D[g][2c+1], D[g+8][2c], D[g+8][2c+1]}.
template <int PASSES, int MT, int NT, class FA, class FB>
__device__ __forceinline__ void warp_gemm(float (&acc)[MT][NT][4], int K, const FA& fa,
                                          const FB& fb) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 8) {
        uint32_t ah[MT][4], al[MT][4], bh[NT][2], bl[NT][2];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float v[4] = {fa(16 * m + g, k0 + c), fa(16 * m + g + 8, k0 + c),
                          fa(16 * m + g, k0 + c + 4), fa(16 * m + g + 8, k0 + c + 4)};
            split_tf32<PASSES>(v, ah[m], al[m]);
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            float v[2] = {fb(k0 + c, 8 * n + g), fb(k0 + c + 4, 8 * n + g)};
            split_tf32<PASSES>(v, bh[n], bl[n]);
        }
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                mma_tf32(acc[m][n], ah[m], bh[n]);
                if (PASSES == 3) {
                    mma_tf32(acc[m][n], ah[m], bl[n]);
                    mma_tf32(acc[m][n], al[m], bh[n]);
                }
            }
    }
}

template <int MT, int NT>
__device__ __forceinline__ void zero_acc(float (&acc)[MT][NT][4]) {
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[m][n][i] = 0.f;
}

// Visit the accumulator elements: f(row, col, value&) with tile-local coordinates.
template <int MT, int NT, class F>
__device__ __forceinline__ void for_acc(float (&acc)[MT][NT][4], const F& f) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            f(16 * m + g, 8 * n + 2 * c, acc[m][n][0]);
            f(16 * m + g, 8 * n + 2 * c + 1, acc[m][n][1]);
            f(16 * m + g + 8, 8 * n + 2 * c, acc[m][n][2]);
            f(16 * m + g + 8, 8 * n + 2 * c + 1, acc[m][n][3]);
        }
}

// Split an M x N output (M % 16 == 0, N % (8*NT) == 0) into 16 x 8NT warp
// tiles, round-robin over the CTA's warps.  body(acc, m0, n0) accumulates the
// tile; epi(row, col, value) consumes each element.
template <int NT, class Body, class Epi>
__device__ __forceinline__ void cta_tiles(int M, int N, const Body& body, const Epi& epi) {
    const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int tn = N / (8 * NT), tiles = (M / 16) * tn;
    for (int tile = warp; tile < tiles; tile += nwarps) {
        const int m0 = (tile / tn) * 16, n0 = (tile % tn) * 8 * NT;
        float acc[1][NT][4];
        zero_acc(acc);
        body(acc, m0, n0);
        for_acc(acc, [&](int r, int c, float& v) { epi(m0 + r, n0 + c, v); });
    }
}

}  // namespace muir

// qk.cu -- the q/k feature prologue of the Muir mixer and its backward.
//
// "Muir: Linear Attention with Sensitivity-Allocated Gating and Matched-Filter
// Readout" (arXiv 2611.08376), wolonglab.org page, "Methodology" and Figure 3(b):
// the query and key pathways end in SiLU, and the key (and the query, before
// the readout gate scales it) is unit-normalised per head:
//
//     s = SiLU(x) = x * sigmoid(x),     y = s / max(||s||_2, eps)
//
// over the d channels of one token-head row (eps = 1e-12 guards the all-zero
// row, whose output is 0).  Backward, for an upstream gradient dy:
//
//     n = max(||s||, eps);  ds = dy / n - s (s . dy) / n^3   (||s|| >= eps)
//                           ds = dy / eps                    (||s|| <  eps)
//     dx = ds * SiLU'(x),   SiLU'(x) = sig(x) (1 + x (1 - sig(x)))
//
// Both are HBM-bound (a few flops per byte): each lane of a warp moves one
// 16-byte vector of a row (8 bf16 or 4 float32), a row is d*esize/16 lanes
// (8 to 32), the row's sums reduce with butterfly shuffles inside that lane
// group, and every lane keeps kRowsInFlight rows' loads in flight so enough
// bytes are outstanding per SM to cover the HBM latency.  Arithmetic is
// float32 (the sigmoid from the fast exponential and division); the output is
// stored in the input dtype (round to nearest even).
#include "common.cuh"
#include "kernels.h"
#include "profile.h"

namespace muir {
namespace {

constexpr int kQkThreads = 256;
constexpr int kRowsInFlight = 2;
constexpr float kNormEps = 1e-12f;

// 16 bytes of a row as raw bits (kept packed while in flight), unpacked to float32.
__device__ __forceinline__ uint4 ld16raw(const void* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ void unpack16(const uint4& a, float* v, float) {
    v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
    v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
}
__device__ __forceinline__ void unpack16(const uint4& a, float* v, __nv_bfloat16) {
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void st16(float* p, const float* v) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void st16(__nv_bfloat16* p, const float* v) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// sigmoid from the fast exponential (2 + 1.173|x| ulp) and division (2 ulp): two
// special-function ops per element, so the kernels stay bound by HBM rather than
// by the longer exact expf / division sequences.  x < -88 gives exp = inf and 0.
__device__ __forceinline__ float sigm(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

// Sum over the G lanes of one row (groups of G consecutive lanes).
template <int G>
__device__ __forceinline__ float group_sum(float a) {
#pragma unroll
    for (int off = G / 2; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
    return a;
}

// BWD = false: y = SiLU(x) / max(||SiLU(x)||, eps).  BWD = true: dx from (x, dy).
// The next pass's rows are loaded (packed) before this pass's are computed, so
// every lane keeps loads in flight while it does arithmetic.
template <typename T, int D, bool BWD>
__global__ void __launch_bounds__(kQkThreads, BWD ? 3 : 6)
k_qk(const T* x, const T* dy, T* out, long long rows) {
    constexpr int V = 16 / (int)sizeof(T);  // elements per lane
    constexpr int G = D / V;                // lanes per row
    constexpr int RPW = 32 / G;             // rows per warp and pass
    constexpr int U = kRowsInFlight;
    const int lane = threadIdx.x & 31, sub = lane / G, col = (lane % G) * V;
    const long long warp = ((long long)blockIdx.x * kQkThreads + threadIdx.x) >> 5;
    const long long step = (long long)gridDim.x * (kQkThreads / 32) * RPW * U;
    auto fetch = [&](long long base, uint4* bx, uint4* bd) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long r = base + (long long)u * RPW + sub;
            bx[u] = make_uint4(0u, 0u, 0u, 0u);
            bd[u] = make_uint4(0u, 0u, 0u, 0u);
            if (r < rows) {
                bx[u] = ld16raw(x + r * D + col);
                if (BWD) bd[u] = ld16raw(dy + r * D + col);
            }
        }
    };
    long long r0 = warp * RPW * U;
    uint4 cx[U], cd[U];
    fetch(r0, cx, cd);
    for (; r0 < rows; r0 += step) {
        uint4 nx[U], nd[U];
        fetch(r0 + step, nx, nd);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float xv[V], dv[V], sv[V], sg[V], ss = 0.f, sd = 0.f;
            unpack16(cx[u], xv, T());
            if (BWD) unpack16(cd[u], dv, T());
#pragma unroll
            for (int i = 0; i < V; ++i) {
                sg[i] = sigm(xv[i]);
                sv[i] = xv[i] * sg[i];
                ss += sv[i] * sv[i];
                if (BWD) sd += sv[i] * dv[i];
            }
            // every lane takes part in the shuffles, rows past the end with zeros
            ss = group_sum<G>(ss);
            if (BWD) sd = group_sum<G>(sd);
            const float nrm = sqrtf(ss);
            const bool tiny = nrm < kNormEps;
            const float inv = 1.0f / (tiny ? kNormEps : nrm);
            float r[V];
            if (!BWD) {
#pragma unroll
                for (int i = 0; i < V; ++i) r[i] = sv[i] * inv;
            } else {
                const float c = tiny ? 0.f : sd * inv * inv * inv;
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const float ds = dv[i] * inv - sv[i] * c;
                    r[i] = ds * sg[i] * (1.0f + xv[i] * (1.0f - sg[i]));
                }
            }
            const long long row = r0 + (long long)u * RPW + sub;
            if (row < rows) st16(out + row * D + col, r);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) { cx[u] = nx[u]; cd[u] = nd[u]; }
    }
}

template <typename T, int D, bool BWD>
cudaError_t launch_qk(const void* x, const void* dy, void* out, long long rows, cudaStream_t st) {
    constexpr int RPB = (kQkThreads / 32) * (32 / (D * (int)sizeof(T) / 16)) * kRowsInFlight;
    long long blocks = (rows + RPB - 1) / RPB;
    int dev = 0, nsm = 148, occ = 1;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    // one wave of resident CTAs: a grid-stride CTA beyond it would only start
    // after a resident one has finished its whole share
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_qk<T, D, BWD>, kQkThreads, 0) !=
            cudaSuccess || occ < 1) {
        (void)cudaGetLastError();  // a failed query is not a launch error
        occ = 1;
    }
    const long long cap = (long long)nsm * occ;
    if (blocks > cap) blocks = cap;
    MUIR_TIMED(BWD ? "k_qk_bwd" : "k_qk", st,
               (k_qk<T, D, BWD><<<(unsigned)blocks, kQkThreads, 0, st>>>(
                   static_cast<const T*>(x), static_cast<const T*>(dy), static_cast<T*>(out),
                   rows)));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qk_prologue(long long rows, int d, bool bf16, const void* x, const void* dy,
                               void* out, bool bwd, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (bf16) {
        if (d == 128) return bwd ? launch_qk<__nv_bfloat16, 128, true>(x, dy, out, rows, st)
                                 : launch_qk<__nv_bfloat16, 128, false>(x, dy, out, rows, st);
        return bwd ? launch_qk<__nv_bfloat16, 64, true>(x, dy, out, rows, st)
                   : launch_qk<__nv_bfloat16, 64, false>(x, dy, out, rows, st);
    }
    if (d == 128) return bwd ? launch_qk<float, 128, true>(x, dy, out, rows, st)
                             : launch_qk<float, 128, false>(x, dy, out, rows, st);
    return bwd ? launch_qk<float, 64, true>(x, dy, out, rows, st)
               : launch_qk<float, 64, false>(x, dy, out, rows, st);
}

}  // namespace muir

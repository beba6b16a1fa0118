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

__device__ __forceinline__ void ld16(const float* p, float* v) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
__device__ __forceinline__ void ld16(const __nv_bfloat16* p, float* v) {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
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
template <typename T, int D, bool BWD>
__global__ void __launch_bounds__(kQkThreads, BWD ? 4 : 8)
k_qk(const T* x, const T* dy, T* out, long long rows) {
    constexpr int V = 16 / (int)sizeof(T);  // elements per lane
    constexpr int G = D / V;                // lanes per row
    constexpr int RPW = 32 / G;             // rows per warp and pass
    constexpr int U = kRowsInFlight;
    const int lane = threadIdx.x & 31, sub = lane / G, col = (lane % G) * V;
    const long long warp = ((long long)blockIdx.x * kQkThreads + threadIdx.x) >> 5;
    const long long nwarp = (long long)gridDim.x * (kQkThreads / 32);
    for (long long r0 = warp * RPW * U; r0 < rows; r0 += nwarp * RPW * U) {
        float xv[U][V], dv[U][V];
        bool ok[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long r = r0 + (long long)u * RPW + sub;
            ok[u] = r < rows;
#pragma unroll
            for (int i = 0; i < V; ++i) { xv[u][i] = 0.f; dv[u][i] = 0.f; }
            if (ok[u]) {
                ld16(x + r * D + col, xv[u]);
                if (BWD) ld16(dy + r * D + col, dv[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float sv[V], sg[V], ss = 0.f, sd = 0.f;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                sg[i] = sigm(xv[u][i]);
                sv[i] = xv[u][i] * sg[i];
                ss += sv[i] * sv[i];
                if (BWD) sd += sv[i] * dv[u][i];
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
                    const float ds = dv[u][i] * inv - sv[i] * c;
                    r[i] = ds * sg[i] * (1.0f + xv[u][i] * (1.0f - sg[i]));
                }
            }
            const long long row = r0 + (long long)u * RPW + sub;
            if (ok[u]) st16(out + row * D + col, r);
        }
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

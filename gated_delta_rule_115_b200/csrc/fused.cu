// fused.cu -- helpers of the stages fused around the recurrence (the q/k
// prologue, SiLU then unit L2 norm per token-head row, and the output gate
// o * sigmoid(z); "Muir", wolonglab.org page, "Methodology" and fig. 3(b))
// for the large-span fallback.  The on-chip kernels apply both stages
// themselves; when a chunk's decay span sends the work to the boundary-pivot
// path, that path needs q^ and k^ as tensors (with raw q/k it runs in fp32 on
// fp32 copies of every input, so that q^ and k^ keep full precision), its
// dq^ and dk^ mapped back through the prologue, and its o gated.  Each kernel here reads the span flag
// first and returns at once when it is clear, so in the common case they cost
// one launch each and no memory traffic.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "profile.h"

namespace muir {
namespace {

constexpr int kD = 128;

__device__ __forceinline__ float sig(float z) {
    float e;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-1.4426950408889634f * z));
    return __fdividef(1.f, 1.f + e);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// One warp per row of 128 channels, 4 per lane.
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float* v) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    v[0] = __low2float(a); v[1] = __high2float(a); v[2] = __low2float(b); v[3] = __high2float(b);
}

__device__ __forceinline__ void store4(__nv_bfloat16* p, const float* v) {
    uint2 u;
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}

__device__ __forceinline__ void store4(float* p, const float* v) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

__device__ __forceinline__ void load4(const float* p, float* v) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
}

// y = SiLU(x) r, r = 1 / ||SiLU(x)|| (the guard maps a zero row to zero).
template <typename Ty>
__global__ void __launch_bounds__(256) k_qk_mat(const int* flag, const __nv_bfloat16* x,
                                                Ty* y, long long rows) {
    if (*flag == 0) return;
    const int lane = threadIdx.x & 31;
    for (long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); r < rows; r += (long long)gridDim.x * 8) {
        float v[4];
        load4(x + r * kD + 4 * lane, v);
        float ss = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            v[u] *= sig(v[u]);
            ss = fmaf(v[u], v[u], ss);
        }
        const float rn = rsqrtf(fmaxf(warp_sum(ss), 1e-24f));
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] *= rn;
        store4(y + r * kD + 4 * lane, v);
    }
}

// dy (gradient of y^) -> dx = SiLU'(x) r (dy - y^ (y^ . dy)) (bf16, may be dy).
template <typename Td>
__global__ void __launch_bounds__(256) k_qk_jac(const int* flag, const __nv_bfloat16* x,
                                                const Td* dy, __nv_bfloat16* dx, long long rows) {
    if (*flag == 0) return;
    const int lane = threadIdx.x & 31;
    for (long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); r < rows; r += (long long)gridDim.x * 8) {
        float xv[4], d[4], sg[4], sv[4];
        load4(x + r * kD + 4 * lane, xv);
        load4(dy + r * kD + 4 * lane, d);
        float ss = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            sg[u] = sig(xv[u]);
            sv[u] = xv[u] * sg[u];
            ss = fmaf(sv[u], sv[u], ss);
        }
        const float rn = rsqrtf(fmaxf(warp_sum(ss), 1e-24f));
        float dot = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) dot = fmaf(sv[u] * rn, d[u], dot);
        dot = warp_sum(dot);
        float o[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            o[u] = (d[u] - sv[u] * rn * dot) * rn * sg[u] * (1.f + xv[u] * (1.f - sg[u]));
        store4(dx + r * kD + 4 * lane, o);
    }
}

__device__ __forceinline__ void load4(const __half* p, float* v) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __half2 a = *reinterpret_cast<const __half2*>(&u.x);
    const __half2 b = *reinterpret_cast<const __half2*>(&u.y);
    v[0] = __low2float(a); v[1] = __high2float(a); v[2] = __low2float(b); v[3] = __high2float(b);
}

// Exact bf16 (or fp16) -> fp32 copy (n a multiple of 4).
template <typename Ts>
__global__ void __launch_bounds__(256) k_upcast(const int* flag, const Ts* src, float* dst,
                                                long long n4) {
    if (*flag == 0) return;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        float v[4];
        load4(src + 4 * i, v);
        store4(dst + 4 * i, v);
    }
}

// fp32 -> bf16 (round to nearest even; n a multiple of 4).
__global__ void __launch_bounds__(256) k_downcast(const int* flag, const float* src,
                                                  __nv_bfloat16* dst, long long n4) {
    if (*flag == 0) return;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        float v[4];
        load4(src + 4 * i, v);
        store4(dst + 4 * i, v);
    }
}

// o_pre = o; o = o sigmoid(z), elementwise (groups of 4).
template <typename T>
__global__ void __launch_bounds__(256) k_ogate_fix(const int* flag, T* o, T* o_pre,
                                                   const __nv_bfloat16* z, long long n4) {
    if (*flag == 0) return;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        float zv[4], ov[4];
        load4(z + 4 * i, zv);
        if constexpr (sizeof(T) == 4) {
            const float4 a = reinterpret_cast<const float4*>(o)[i];
            ov[0] = a.x; ov[1] = a.y; ov[2] = a.z; ov[3] = a.w;
            if (o_pre) reinterpret_cast<float4*>(o_pre)[i] = a;
#pragma unroll
            for (int u = 0; u < 4; ++u) ov[u] *= sig(zv[u]);
            reinterpret_cast<float4*>(o)[i] = make_float4(ov[0], ov[1], ov[2], ov[3]);
        } else {
            load4(reinterpret_cast<const __nv_bfloat16*>(o) + 4 * i, ov);
            if (o_pre) reinterpret_cast<uint2*>(o_pre)[i] = reinterpret_cast<const uint2*>(o)[i];
#pragma unroll
            for (int u = 0; u < 4; ++u) ov[u] *= sig(zv[u]);
            store4(reinterpret_cast<__nv_bfloat16*>(o) + 4 * i, ov);
        }
    }
}

int grid_for(long long work, int per_block) {
    long long g = (work + per_block - 1) / per_block;
    return (int)(g < 1 ? 1 : (g > 1184 ? 1184 : g));  // 8 x 148 SMs at most (grid-stride)
}

}  // namespace

cudaError_t qk_materialise_gated(const int* flag, const void* x, void* y, long long rows,
                                 bool f32_out, cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    if (f32_out) {
        MUIR_TIMED("k_qk_mat", st, k_qk_mat<float><<<grid_for(rows, 8), 256, 0, st>>>(
            flag, xb, static_cast<float*>(y), rows));
    } else {
        MUIR_TIMED("k_qk_mat", st, k_qk_mat<__nv_bfloat16><<<grid_for(rows, 8), 256, 0, st>>>(
            flag, xb, static_cast<__nv_bfloat16*>(y), rows));
    }
    return cudaGetLastError();
}

cudaError_t qk_jacobian_gated(const int* flag, const void* x, const void* dy, bool dy_f32,
                              void* dx, long long rows, cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(dx);
    if (dy_f32) {
        MUIR_TIMED("k_qk_jac", st, k_qk_jac<float><<<grid_for(rows, 8), 256, 0, st>>>(
            flag, xb, static_cast<const float*>(dy), out, rows));
    } else {
        MUIR_TIMED("k_qk_jac", st, k_qk_jac<__nv_bfloat16><<<grid_for(rows, 8), 256, 0, st>>>(
            flag, xb, static_cast<const __nv_bfloat16*>(dy), out, rows));
    }
    return cudaGetLastError();
}

cudaError_t upcast_gated(const int* flag, const void* src, float* dst, long long n, bool src_f16,
                         cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    if (n % 4) return cudaErrorInvalidValue;
    if (src_f16) {
        MUIR_TIMED("k_upcast", st, k_upcast<__half><<<grid_for(n / 4, 256), 256, 0, st>>>(
            flag, static_cast<const __half*>(src), dst, n / 4));
    } else {
        MUIR_TIMED("k_upcast", st, k_upcast<__nv_bfloat16><<<grid_for(n / 4, 256), 256, 0, st>>>(
            flag, static_cast<const __nv_bfloat16*>(src), dst, n / 4));
    }
    return cudaGetLastError();
}

cudaError_t downcast_gated(const int* flag, const float* src, void* dst, long long n, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    if (n % 4) return cudaErrorInvalidValue;
    MUIR_TIMED("k_downcast", st, k_downcast<<<grid_for(n / 4, 256), 256, 0, st>>>(
        flag, src, static_cast<__nv_bfloat16*>(dst), n / 4));
    return cudaGetLastError();
}

cudaError_t out_gate_fix_gated(const int* flag, void* o, void* o_pre, const void* z, long long n,
                               bool out_bf16, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    if (n % 4) return cudaErrorInvalidValue;
    const long long n4 = n / 4;
    const __nv_bfloat16* zb = static_cast<const __nv_bfloat16*>(z);
    if (out_bf16) {
        MUIR_TIMED("k_ogate_fix", st, k_ogate_fix<__nv_bfloat16><<<grid_for(n4, 256), 256, 0, st>>>(
            flag, static_cast<__nv_bfloat16*>(o), static_cast<__nv_bfloat16*>(o_pre), zb, n4));
    } else {
        MUIR_TIMED("k_ogate_fix", st, k_ogate_fix<float><<<grid_for(n4, 256), 256, 0, st>>>(
            flag, static_cast<float*>(o), static_cast<float*>(o_pre), zb, n4));
    }
    return cudaGetLastError();
}

}  // namespace muir

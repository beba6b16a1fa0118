// tail.cu -- ragged tails of the chunkwise path (T % C != 0).
//
// The chunk kernels work on whole chunks of C tokens.  When T is not a
// multiple of C, the last chunk of every (b, h) sequence holds tail < C real
// tokens.  Its rows are copied into a side buffer of C rows per sequence whose
// rows past the tail are zero.  A zero token (q = k = v = e = w = gamma = 0,
// g = 0) is neutral for the recurrence of "Muir" (wolonglab.org page,
// "Methodology", eq:ours): D_t = I, the erase term (e*k)(k^T S) and the write
// term k (w*v)^T vanish, so S_t = S_{t-1}, and o_t = S_t^T (gamma*q) = 0; in
// the backward its Jacobian is the identity and dO = 0 adds nothing.  The full
// chunk therefore yields exactly the tail's results on its first tail rows,
// which are copied back afterwards.  The copies are plain 16-byte moves with
// one thread per 16 bytes: a few MB per call, next to the chunk kernels.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace muir {
namespace {

constexpr int kTailThreads = 256;

// to_side: token-major [B][T][H][D] rows t0 .. t0+C-1 -> side [B*H][C][D]
// (zero past the tail); otherwise side rows < tail -> token-major.
__global__ void __launch_bounds__(kTailThreads)
k_tail_copy(TailCopy io, int H, int T, int C, int t0, int tail, int row_vecs, size_t per_tensor,
            bool to_side) {
    const size_t total = per_tensor * io.n;
    for (size_t i = (size_t)blockIdx.x * kTailThreads + threadIdx.x; i < total;
         i += (size_t)gridDim.x * kTailThreads) {
        const int k = (int)(i / per_tensor);
        const size_t r = i - (size_t)k * per_tensor;
        const int x = (int)(r % row_vecs);
        const size_t row = r / row_vecs;           // bh * C + t
        const int t = (int)(row % C);
        const size_t bh = row / C;
        const size_t b = bh / H, h = bh % H;
        const size_t tok = ((b * T + t0 + t) * H + h) * row_vecs + x;  // in 16-byte units
        const size_t side = row * row_vecs + x;
        if (to_side) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (t < tail) v = reinterpret_cast<const uint4*>(io.src[k])[tok];
            reinterpret_cast<uint4*>(io.dst[k])[side] = v;
        } else if (t < tail) {
            reinterpret_cast<uint4*>(io.dst[k])[tok] = reinterpret_cast<const uint4*>(io.src[k])[side];
        }
    }
}

cudaError_t launch(const TailCopy& io, int B, int H, int T, int C, int D, int esize, bool to_side,
                   cudaStream_t st) {
    const int N = (T + C - 1) / C, t0 = (N - 1) * C, tail = T - t0;
    const int row_vecs = D * esize / 16;
    const size_t per_tensor = (size_t)B * H * C * row_vecs;
    const size_t total = per_tensor * io.n;
    size_t blocks = (total + kTailThreads - 1) / kTailThreads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    k_tail_copy<<<(unsigned)blocks, kTailThreads, 0, st>>>(io, H, T, C, t0, tail, row_vecs,
                                                            per_tensor, to_side);
    return cudaGetLastError();
}

}  // namespace

cudaError_t tail_gather(const TailCopy& io, int B, int H, int T, int C, int D, int esize,
                        cudaStream_t st) {
    return launch(io, B, H, T, C, D, esize, true, st);
}

cudaError_t tail_scatter(const TailCopy& io, int B, int H, int T, int C, int D, int esize,
                         cudaStream_t st) {
    return launch(io, B, H, T, C, D, esize, false, st);
}

}  // namespace muir

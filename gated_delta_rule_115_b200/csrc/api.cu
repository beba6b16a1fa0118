// api.cu -- the extern "C" entry points of libmuir: host-side argument checks,
// workspace sizing and dispatch to the CUDA kernels.  Nothing here computes.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/muir.h"
#include "chunk_units.h"
#include "bwd2.h"
#include "fwd2.h"
#include "gates.h"
#include "kernels.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
#ifdef MUIR_DEBUG
// Debug builds (build.py --debug) also ask the CUDA runtime where each
// pointer lives and refuse host memory the device cannot address.
bool device_addressable(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged ||
           (a.type == cudaMemoryTypeHost && a.devicePointer != nullptr);
}
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p) && device_addressable(p); }
bool ok_opt(const void* p) { return p == nullptr || (aligned16(p) && device_addressable(p)); }
#else
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }
#endif
bool ok_dtype(muir_dtype d) { return d == MUIR_BF16 || d == MUIR_FP32; }

// The kernels use sm_100a instructions: require compute capability 10.x.
muir_status check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MUIR_ERR_CUDA;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return MUIR_ERR_CUDA;
    return major == 10 ? MUIR_OK : MUIR_ERR_UNSUPPORTED;
}

// Shape checks shared by the chunk entry points (no CUDA calls).
muir_status check_shape(const muir_shape* s) {
    if (!s) return MUIR_ERR_INVALID_ARG;
    if (s->B <= 0 || s->T <= 0 || s->H <= 0 || s->dk <= 0 || s->dv <= 0 || s->chunk <= 0)
        return MUIR_ERR_INVALID_ARG;
    if (!ok_dtype(s->in_dtype) || !ok_dtype(s->out_dtype)) return MUIR_ERR_INVALID_ARG;
    if (s->dk != s->dv || (s->dk != 64 && s->dk != 128)) return MUIR_ERR_UNSUPPORTED;
    const int C = s->chunk;
    if (C != 16 && C != 32 && C != 64 && C != 128 && C != 256) return MUIR_ERR_UNSUPPORTED;
    // index arithmetic inside the kernels is 64-bit for tensors; keep counts in int range
    if ((long long)s->B * s->H * ((s->T + C - 1) / C) > (1LL << 30)) return MUIR_ERR_UNSUPPORTED;
    return MUIR_OK;
}

muir::ChunkProblem make_problem(const muir_shape* s, const void* q, const void* k,
                                const void* v, const void* g, const void* e, const void* w,
                                const void* gamma) {
    muir::ChunkProblem P;
    P.B = s->B; P.T = s->T; P.H = s->H; P.D = s->dk; P.C = s->chunk; P.N = (s->T + s->chunk - 1) / s->chunk;
    P.in_bf16 = s->in_dtype == MUIR_BF16;
    P.out_bf16 = s->out_dtype == MUIR_BF16;
    P.q = q; P.k = k; P.v = v; P.g = g; P.e = e; P.w = w; P.gamma = gamma;
    P.aux = nullptr;
    P.gate = nullptr;
    return P;
}

// Packed variable-length batch: B == 1, T = total tokens, cu_seqlens (host)
// holds num_seqs + 1 non-decreasing offsets from 0 to T.  A batch whose
// sequences are all empty (T == 0) is valid.
muir_status check_varlen(const muir_shape* s, int num_seqs, const long long* cu) {
    if (!s || num_seqs <= 0 || !cu || s->B != 1 || s->T < 0) return MUIR_ERR_INVALID_ARG;
    if (cu[0] != 0 || cu[num_seqs] != s->T) return MUIR_ERR_INVALID_ARG;
    for (int i = 0; i < num_seqs; ++i)
        if (cu[i + 1] < cu[i]) return MUIR_ERR_INVALID_ARG;
    muir_shape t = *s;
    if (t.T == 0) t.T = t.chunk > 0 ? t.chunk : 1;  // the remaining checks only
    return check_shape(&t);
}

size_t varlen_ws_bytes(const muir_shape* s, int num_seqs, const long long* cu, bool bwd) {
    size_t need = 0;
    for (int i = 0; i < num_seqs; ++i) {
        const int L = (int)(cu[i + 1] - cu[i]);
        if (L == 0) continue;
        const size_t b = bwd ? muir::chunk_bwd_ws_bytes(1, L, s->H, s->dk, s->chunk, false, s->in_dtype == MUIR_BF16)
                             : muir::chunk_fwd_ws_bytes(1, L, s->H, s->dk, s->chunk, false, s->in_dtype == MUIR_BF16);
        if (b > need) need = b;
    }
    return need;
}

const void* at_row(const void* p, long long row, size_t row_bytes) {
    return static_cast<const char*>(p) + (size_t)row * row_bytes;
}

muir_status from_cuda(cudaError_t err) {
    if (err == cudaSuccess) return MUIR_OK;
    if (err == cudaErrorNotSupported) return MUIR_ERR_UNSUPPORTED;
    return MUIR_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* muir_status_string(muir_status s) {
    switch (s) {
        case MUIR_OK: return "MUIR_OK";
        case MUIR_ERR_INVALID_ARG: return "MUIR_ERR_INVALID_ARG: null, misaligned or out-of-range argument";
        case MUIR_ERR_UNSUPPORTED: return "MUIR_ERR_UNSUPPORTED: shape, chunk or device not supported";
        case MUIR_ERR_WORKSPACE: return "MUIR_ERR_WORKSPACE: workspace missing or too small";
        case MUIR_ERR_CUDA: return "MUIR_ERR_CUDA: a CUDA runtime call or kernel launch failed";
        case MUIR_ERR_DEVICE_TIMEOUT: return "MUIR_ERR_DEVICE_TIMEOUT: a bounded device wait expired";
    }
    return "MUIR_ERR_UNKNOWN";
}

muir_status muir_device_wait_status(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return MUIR_ERR_CUDA;
    const unsigned int n = muir::timeouts_bf16_d128() + muir::timeouts_bf16_d64() +
                           muir::timeouts_f32_d128() + muir::timeouts_f32_d64() +
                           muir::v2::timeouts_v2() + muir::v2::timeouts_bwd2() +
                           muir::timeouts_selftest() + muir::v2::timeouts_gates();
    return n ? MUIR_ERR_DEVICE_TIMEOUT : MUIR_OK;
}

size_t muir_chunk_aux_floats(const muir_shape* s) {
    if (check_shape(s) != MUIR_OK) return 0;
    return muir::chunk_aux_total_floats(s->B, s->T, s->H, s->dk, s->chunk, s->in_dtype == MUIR_BF16);
}

size_t muir_chunk_fwd_workspace(const muir_shape* s) {
    if (check_shape(s) != MUIR_OK) return 0;
    return muir::chunk_fwd_ws_bytes(s->B, s->T, s->H, s->dk, s->chunk, false,
                                    s->in_dtype == MUIR_BF16);
}

size_t muir_chunk_bwd_workspace(const muir_shape* s) {
    if (check_shape(s) != MUIR_OK) return 0;
    return muir::chunk_bwd_ws_bytes(s->B, s->T, s->H, s->dk, s->chunk, false,
                                    s->in_dtype == MUIR_BF16);
}

muir_status muir_chunk_fwd(const muir_shape* s, const void* q, const void* k, const void* v,
                           const void* g, const void* e, const void* w, const void* gamma,
                           const float* S0, void* o, float* S_final, float* S_chunks,
                           float* M_chunks, float* aux, void* ws, size_t ws_bytes, void* stream) {
    muir_status st = check_shape(s);
    if (st != MUIR_OK) return st;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(g) || !ok_ptr(e) || !ok_ptr(w) ||
        !ok_ptr(gamma) || !ok_ptr(o) || !ok_opt(S0) || !ok_opt(S_final) || !ok_opt(S_chunks) ||
        !ok_opt(M_chunks) || !ok_opt(aux))
        return MUIR_ERR_INVALID_ARG;
    const size_t need = muir::chunk_fwd_ws_bytes(s->B, s->T, s->H, s->dk, s->chunk,
                                                 S_chunks != nullptr, s->in_dtype == MUIR_BF16);
    if (ws_bytes < need || (need > 0 && !ok_ptr(ws))) return MUIR_ERR_WORKSPACE;
    if ((st = check_device()) != MUIR_OK) return st;
    muir::ChunkProblem P = make_problem(s, q, k, v, g, e, w, gamma);
    P.aux = aux;
    return from_cuda(muir::run_chunk_fwd(P, S0, o, S_final, S_chunks, M_chunks, ws, ws_bytes,
                                         static_cast<cudaStream_t>(stream)));
}

muir_status muir_chunk_bwd(const muir_shape* s, const void* q, const void* k, const void* v,
                           const void* g, const void* e, const void* w, const void* gamma,
                           const float* S0, const float* S_chunks, const float* M_chunks,
                           const float* aux, const void* dO, const float* dS_final, void* dq,
                           void* dk, void* dv,
                           void* dg, void* de, void* dw, void* dgamma, float* dS0, void* ws,
                           size_t ws_bytes, void* stream) {
    muir_status st = check_shape(s);
    if (st != MUIR_OK) return st;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(g) || !ok_ptr(e) || !ok_ptr(w) ||
        !ok_ptr(gamma) || !ok_ptr(dO) || !ok_ptr(dq) || !ok_ptr(dk) || !ok_ptr(dv) ||
        !ok_ptr(dg) || !ok_ptr(de) || !ok_ptr(dw) || !ok_ptr(dgamma) || !ok_opt(S0) ||
        !ok_opt(S_chunks) || !ok_opt(M_chunks) || !ok_opt(dS_final) || !ok_opt(dS0) ||
        !ok_opt(aux) || (aux && !S_chunks))
        return MUIR_ERR_INVALID_ARG;
    const size_t need = muir::chunk_bwd_ws_bytes(s->B, s->T, s->H, s->dk, s->chunk,
                                                 S_chunks != nullptr, s->in_dtype == MUIR_BF16);
    if (ws_bytes < need || (need > 0 && !ok_ptr(ws))) return MUIR_ERR_WORKSPACE;
    if ((st = check_device()) != MUIR_OK) return st;
    muir::ChunkProblem P = make_problem(s, q, k, v, g, e, w, gamma);
    P.aux = const_cast<float*>(aux);
    return from_cuda(muir::run_chunk_bwd(P, S0, S_chunks, M_chunks, dO, dS_final, dq, dk, dv, dg,
                                         de, dw, dgamma, dS0, ws, ws_bytes,
                                         static_cast<cudaStream_t>(stream)));
}

muir_status muir_recurrent_step(int B, int H, int dk, int dv, muir_dtype dtype,
                                muir_dtype out_dtype, const void* q, const void* k,
                                const void* v, const void* g, const void* e, const void* w,
                                const void* gamma, int gamma_static, float* S, void* o,
                                void* stream) {
    if (B <= 0 || H <= 0 || dk <= 0 || dv <= 0) return MUIR_ERR_INVALID_ARG;
    if (!ok_dtype(dtype) || !ok_dtype(out_dtype)) return MUIR_ERR_INVALID_ARG;
    if (gamma_static != 0 && gamma_static != 1) return MUIR_ERR_INVALID_ARG;
    if (dk != dv || (dk != 64 && dk != 128)) return MUIR_ERR_UNSUPPORTED;
    if ((long long)B * H > (1LL << 30)) return MUIR_ERR_UNSUPPORTED;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(g) || !ok_ptr(e) || !ok_ptr(w) ||
        !ok_opt(gamma) || !ok_ptr(S) || !ok_ptr(o))
        return MUIR_ERR_INVALID_ARG;
    muir_status st = check_device();
    if (st != MUIR_OK) return st;
    return from_cuda(muir::launch_decode(B, H, dk, dtype == MUIR_BF16, out_dtype == MUIR_BF16,
                                         q, k, v, g, e, w, gamma, gamma_static, S, o,
                                         static_cast<cudaStream_t>(stream)));
}

size_t muir_chunk_varlen_workspace(const muir_shape* s, int num_seqs, const long long* cu_seqlens,
                                   int backward) {
    if (check_varlen(s, num_seqs, cu_seqlens) != MUIR_OK) return 0;
    return varlen_ws_bytes(s, num_seqs, cu_seqlens, backward != 0);
}

muir_status muir_chunk_fwd_varlen(const muir_shape* s, int num_seqs, const long long* cu_seqlens,
                                  const void* q, const void* k, const void* v, const void* g,
                                  const void* e, const void* w, const void* gamma,
                                  const float* S0, void* o, float* S_final, void* ws,
                                  size_t ws_bytes, void* stream) {
    muir_status st = check_varlen(s, num_seqs, cu_seqlens);
    if (st != MUIR_OK) return st;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(g) || !ok_ptr(e) || !ok_ptr(w) ||
        !ok_ptr(gamma) || !ok_ptr(o) || !ok_opt(S0) || !ok_opt(S_final))
        return MUIR_ERR_INVALID_ARG;
    const size_t need = varlen_ws_bytes(s, num_seqs, cu_seqlens, false);
    if (ws_bytes < need || (need > 0 && !ok_ptr(ws))) return MUIR_ERR_WORKSPACE;
    if ((st = check_device()) != MUIR_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const size_t DD = (size_t)s->dk * s->dv, row = (size_t)s->H * s->dk;
    const size_t ein = s->in_dtype == MUIR_BF16 ? 2 : 4, eout = s->out_dtype == MUIR_BF16 ? 2 : 4;
    for (int i = 0; i < num_seqs; ++i) {
        const long long r0 = cu_seqlens[i];
        const int L = (int)(cu_seqlens[i + 1] - r0);
        const float* s0 = S0 ? S0 + (size_t)i * s->H * DD : nullptr;
        float* sf = S_final ? S_final + (size_t)i * s->H * DD : nullptr;
        cudaError_t err = cudaSuccess;
        if (L == 0) {  // empty sequence: the final state is the initial one
            if (sf && s0) err = cudaMemcpyAsync(sf, s0, s->H * DD * 4, cudaMemcpyDeviceToDevice, cs);
            else if (sf) err = cudaMemsetAsync(sf, 0, s->H * DD * 4, cs);
            if (err != cudaSuccess) return from_cuda(err);
            continue;
        }
        muir_shape si = *s;
        si.T = L;
        const size_t rb = row * ein;
        muir::ChunkProblem P = make_problem(&si, at_row(q, r0, rb), at_row(k, r0, rb),
                                            at_row(v, r0, rb), at_row(g, r0, rb),
                                            at_row(e, r0, rb), at_row(w, r0, rb),
                                            at_row(gamma, r0, rb));
        err = muir::run_chunk_fwd(P, s0, const_cast<void*>(at_row(o, r0, row * eout)), sf,
                                  nullptr, nullptr, ws, ws_bytes, cs);
        if (err != cudaSuccess) return from_cuda(err);
    }
    return MUIR_OK;
}

muir_status muir_chunk_bwd_varlen(const muir_shape* s, int num_seqs, const long long* cu_seqlens,
                                  const void* q, const void* k, const void* v, const void* g,
                                  const void* e, const void* w, const void* gamma,
                                  const float* S0, const void* dO, const float* dS_final,
                                  void* dq, void* dk, void* dv, void* dg, void* de, void* dw,
                                  void* dgamma, float* dS0, void* ws, size_t ws_bytes,
                                  void* stream) {
    muir_status st = check_varlen(s, num_seqs, cu_seqlens);
    if (st != MUIR_OK) return st;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(g) || !ok_ptr(e) || !ok_ptr(w) ||
        !ok_ptr(gamma) || !ok_ptr(dO) || !ok_ptr(dq) || !ok_ptr(dk) || !ok_ptr(dv) ||
        !ok_ptr(dg) || !ok_ptr(de) || !ok_ptr(dw) || !ok_ptr(dgamma) || !ok_opt(S0) ||
        !ok_opt(dS_final) || !ok_opt(dS0))
        return MUIR_ERR_INVALID_ARG;
    const size_t need = varlen_ws_bytes(s, num_seqs, cu_seqlens, true);
    if (ws_bytes < need || (need > 0 && !ok_ptr(ws))) return MUIR_ERR_WORKSPACE;
    if ((st = check_device()) != MUIR_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const size_t DD = (size_t)s->dk * s->dv, row = (size_t)s->H * s->dk;
    const size_t rb = row * (s->in_dtype == MUIR_BF16 ? 2 : 4);
    for (int i = 0; i < num_seqs; ++i) {
        const long long r0 = cu_seqlens[i];
        const int L = (int)(cu_seqlens[i + 1] - r0);
        const float* s0 = S0 ? S0 + (size_t)i * s->H * DD : nullptr;
        const float* dsf = dS_final ? dS_final + (size_t)i * s->H * DD : nullptr;
        float* ds0 = dS0 ? dS0 + (size_t)i * s->H * DD : nullptr;
        cudaError_t err = cudaSuccess;
        if (L == 0) {  // empty sequence: the state passes through unchanged
            if (ds0 && dsf) err = cudaMemcpyAsync(ds0, dsf, s->H * DD * 4, cudaMemcpyDeviceToDevice, cs);
            else if (ds0) err = cudaMemsetAsync(ds0, 0, s->H * DD * 4, cs);
            if (err != cudaSuccess) return from_cuda(err);
            continue;
        }
        muir_shape si = *s;
        si.T = L;
        auto out = [&](void* p) { return const_cast<void*>(at_row(p, r0, rb)); };
        muir::ChunkProblem P = make_problem(&si, at_row(q, r0, rb), at_row(k, r0, rb),
                                            at_row(v, r0, rb), at_row(g, r0, rb),
                                            at_row(e, r0, rb), at_row(w, r0, rb),
                                            at_row(gamma, r0, rb));
        err = muir::run_chunk_bwd(P, s0, nullptr, nullptr, at_row(dO, r0, rb), dsf, out(dq),
                                  out(dk), out(dv), out(dg), out(de), out(dw), out(dgamma), ds0,
                                  ws, ws_bytes, cs);
        if (err != cudaSuccess) return from_cuda(err);
    }
    return MUIR_OK;
}

muir_status muir_qk_prologue(long long rows, int d, muir_dtype dtype, const void* x, void* y,
                             void* stream) {
    if (rows < 0 || !ok_dtype(dtype)) return MUIR_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return MUIR_ERR_UNSUPPORTED;
    if (rows == 0) return MUIR_OK;
    if (!ok_ptr(x) || !ok_ptr(y)) return MUIR_ERR_INVALID_ARG;
    muir_status st = check_device();
    if (st != MUIR_OK) return st;
    return from_cuda(muir::launch_qk_prologue(rows, d, dtype == MUIR_BF16, x, nullptr, y, false,
                                              static_cast<cudaStream_t>(stream)));
}

muir_status muir_qk_prologue_bwd(long long rows, int d, muir_dtype dtype, const void* x,
                                 const void* dy, void* dx, void* stream) {
    if (rows < 0 || !ok_dtype(dtype)) return MUIR_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return MUIR_ERR_UNSUPPORTED;
    if (rows == 0) return MUIR_OK;
    if (!ok_ptr(x) || !ok_ptr(dy) || !ok_ptr(dx)) return MUIR_ERR_INVALID_ARG;
    muir_status st = check_device();
    if (st != MUIR_OK) return st;
    return from_cuda(muir::launch_qk_prologue(rows, d, dtype == MUIR_BF16, x, dy, dx, true,
                                              static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// ------------------------------------------------------------ fused stages

namespace {

bool fused_any(const muir_fusion* f) { return f && (f->z_out || f->qk_raw || f->latent); }

int projected(const muir_fusion* f, int X) { return f && f->latent && f->fam[X].rank > 0; }

// The fused stages run inside the on-chip kernels: bf16 inputs, dk = dv = 128,
// chunk 128, T a multiple of 128.
muir_status check_fusion(const muir_shape* s, const muir_fusion* f) {
    if (!f) return MUIR_ERR_INVALID_ARG;
    if (f->qk_raw != 0 && f->qk_raw != 1) return MUIR_ERR_INVALID_ARG;
    if (!ok_opt(f->z_out)) return MUIR_ERR_INVALID_ARG;
    if (f->latent) {
        if (!ok_ptr(f->latent) || f->R <= 0 || f->R % 8) return MUIR_ERR_INVALID_ARG;
        int n = 0;
        for (int X = 0; X < 5; ++X) {
            const muir_gate_family& a = f->fam[X];
            if (a.rank == 0) continue;
            if (a.rank != 64 && a.rank != 128) return MUIR_ERR_UNSUPPORTED;
            if (a.off < 0 || a.off % 8 || a.off + a.rank > f->R) return MUIR_ERR_INVALID_ARG;
            if (!ok_ptr(a.U) || !ok_ptr(a.bias)) return MUIR_ERR_INVALID_ARG;
            for (int Y = 0; Y < X; ++Y) {  // latent columns of two families must not overlap
                const muir_gate_family& b = f->fam[Y];
                if (b.rank > 0 && a.off < b.off + b.rank && b.off < a.off + a.rank)
                    return MUIR_ERR_INVALID_ARG;
            }
            ++n;
        }
        if (n == 0) return MUIR_ERR_INVALID_ARG;
        if (projected(f, MUIR_FAM_OUTGATE) && f->z_out) return MUIR_ERR_INVALID_ARG;
    }
    if (fused_any(f) && !muir::v2::fwd2_supported(s->B, s->T, s->H, s->dk, s->chunk,
                                                  s->in_dtype == MUIR_BF16))
        return MUIR_ERR_UNSUPPORTED;
    return MUIR_OK;
}

size_t base_ws(const muir_shape* s, bool backward) {
    return backward
        ? muir::chunk_bwd_ws_bytes(s->B, s->T, s->H, s->dk, s->chunk, false, s->in_dtype == MUIR_BF16)
        : muir::chunk_fwd_ws_bytes(s->B, s->T, s->H, s->dk, s->chunk, false, s->in_dtype == MUIR_BF16);
}

// Per projected family: its gate, and in the backward the gate's gradient and
// dpre (a bf16 hi / lo pair).
size_t gate_buf_bytes(const muir_shape* s) { return (size_t)s->B * s->T * s->H * s->dk * 2; }

size_t fused_ws(const muir_shape* s, const muir_fusion* f, bool backward) {
    const size_t base = base_ws(s, backward);
    if (!fused_any(f)) return base;
    size_t extra = muir::fused_ws_bytes(s->B, s->T, s->H, s->dk, s->chunk, f->qk_raw != 0);
    if (f->latent) extra += 5 * (backward ? 4 : 1) * gate_buf_bytes(s);
    return ((base + 255) & ~(size_t)255) + extra;
}

char* fused_region(const muir_shape* s, void* ws, bool backward) {
    return static_cast<char*>(ws) + ((base_ws(s, backward) + 255) & ~(size_t)255);
}

// The gate projection's launch description; the projected gates (and in the
// backward their gradients and dpre) live in the workspace after the stages'
// own region.  Replaces the tensor arguments of projected families in P.
void setup_projection(const muir_shape* s, const muir_fusion* f, char* fw, bool backward,
                      muir::v2::GatesArgs& ga, muir::ChunkProblem& P, void** dgate_ptrs,
                      const muir_fusion_grads* fg) {
    static const int act[5] = {muir::v2::kActNegSoftplus, muir::v2::kActSigmoid,
                               muir::v2::kActIdentity, muir::v2::kActSigmoid,
                               muir::v2::kActSigmoid};
    const size_t gb = gate_buf_bytes(s);
    char* buf = fw + muir::fused_ws_bytes(s->B, s->T, s->H, s->dk, s->chunk, f->qk_raw != 0);
    ga = muir::v2::GatesArgs{};
    ga.latent = f->latent;
    ga.R = f->R;
    ga.H = s->H;
    ga.rows = (long long)s->B * s->T;
    ga.dlatent = fg ? fg->dlatent : nullptr;
    for (int X = 0; X < 5; ++X) {
        if (!projected(f, X)) continue;
        muir::v2::GateFamily& g = ga.fam[ga.nfam++];
        g.off = f->fam[X].off;
        g.r = f->fam[X].rank;
        g.act = act[X];
        g.U = f->fam[X].U;
        g.bias = f->fam[X].bias;
        g.out = buf + (size_t)X * gb;
        if (backward) {
            g.dout = buf + (size_t)(5 + X) * gb;
            g.dpre = buf + (size_t)(10 + X) * gb;
            g.dpre_lo = buf + (size_t)(15 + X) * gb;
            g.dU = fg->dU[X];
            g.dbias = fg->dbias[X];
            dgate_ptrs[X] = const_cast<void*>(g.dout);
        }
        switch (X) {
            case MUIR_FAM_DECAY: P.g = g.out; break;
            case MUIR_FAM_ERASE: P.e = g.out; break;
            case MUIR_FAM_OUTGATE: P.zo = g.out; break;
            case MUIR_FAM_WRITE: P.w = g.out; break;
            default: P.gamma = g.out; break;
        }
    }
    P.gate_proj = &ga;
}

}  // namespace

size_t muir_chunk_fused_workspace(const muir_shape* s, const muir_fusion* f, int backward) {
    if (check_shape(s) != MUIR_OK || check_fusion(s, f) != MUIR_OK) return 0;
    return fused_ws(s, f, backward != 0);
}

muir_status muir_chunk_fwd_fused(const muir_shape* s, const muir_fusion* f, const void* q,
                                 const void* k, const void* v, const void* g, const void* e,
                                 const void* w, const void* gamma, const float* S0, void* o,
                                 void* o_pre, float* S_final, float* S_chunks, float* M_chunks,
                                 float* aux, void* ws, size_t ws_bytes, void* stream) {
    muir_status st = check_shape(s);
    if (st != MUIR_OK) return st;
    if ((st = check_fusion(s, f)) != MUIR_OK) return st;
    const bool gate = f->z_out || projected(f, MUIR_FAM_OUTGATE);
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(o) || !ok_opt(o_pre) || !ok_opt(S0) ||
        !ok_opt(S_final) || !ok_opt(S_chunks) || !ok_opt(M_chunks) || !ok_opt(aux) ||
        (o_pre && !gate))
        return MUIR_ERR_INVALID_ARG;
    if ((!projected(f, MUIR_FAM_DECAY) && !ok_ptr(g)) || (!projected(f, MUIR_FAM_ERASE) && !ok_ptr(e)) ||
        (!projected(f, MUIR_FAM_WRITE) && !ok_ptr(w)) ||
        (!projected(f, MUIR_FAM_READOUT) && !ok_ptr(gamma)))
        return MUIR_ERR_INVALID_ARG;
    const size_t need = fused_ws(s, f, false);
    if (ws_bytes < need || (need > 0 && !ok_ptr(ws))) return MUIR_ERR_WORKSPACE;
    if ((st = check_device()) != MUIR_OK) return st;
    muir::ChunkProblem P = make_problem(s, q, k, v, g, e, w, gamma);
    P.aux = aux;
    muir::v2::GatesArgs ga;
    if (fused_any(f)) {
        P.zo = f->z_out;
        P.o_pre = o_pre;
        P.qk_raw = f->qk_raw;
        P.fused_ws = fused_region(s, ws, false);
        if (f->latent) setup_projection(s, f, P.fused_ws, false, ga, P, nullptr, nullptr);
    }
    return from_cuda(muir::run_chunk_fwd(P, S0, o, S_final, S_chunks, M_chunks, ws, ws_bytes,
                                         static_cast<cudaStream_t>(stream)));
}

muir_status muir_chunk_bwd_fused(const muir_shape* s, const muir_fusion* f, const void* q,
                                 const void* k, const void* v, const void* g, const void* e,
                                 const void* w, const void* gamma, const float* S0,
                                 const float* S_chunks, const float* M_chunks, const float* aux,
                                 const void* o_pre, const void* dO, const float* dS_final,
                                 void* dq, void* dk, void* dv, void* dg, void* de, void* dw,
                                 void* dgamma, void* dz_out, float* dS0,
                                 const muir_fusion_grads* fg, void* ws, size_t ws_bytes,
                                 void* stream) {
    muir_status st = check_shape(s);
    if (st != MUIR_OK) return st;
    if ((st = check_fusion(s, f)) != MUIR_OK) return st;
    const bool gate = f->z_out || projected(f, MUIR_FAM_OUTGATE);
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(dO) || !ok_ptr(dq) || !ok_ptr(dk) ||
        !ok_ptr(dv) || !ok_opt(S0) || !ok_opt(S_chunks) || !ok_opt(M_chunks) ||
        !ok_opt(dS_final) || !ok_opt(dS0) || !ok_opt(aux) || (aux && !S_chunks) ||
        !ok_opt(o_pre) || !ok_opt(dz_out))
        return MUIR_ERR_INVALID_ARG;
    const void* gin[5] = {g, e, nullptr, w, gamma};
    void* gout[5] = {dg, de, dz_out, dw, dgamma};
    for (int X = 0; X < 5; ++X) {
        if (X == MUIR_FAM_OUTGATE || projected(f, X)) continue;
        if (!ok_ptr(gin[X]) || !ok_ptr(gout[X])) return MUIR_ERR_INVALID_ARG;
    }
    if (gate && !o_pre) return MUIR_ERR_INVALID_ARG;
    if (f->z_out && !dz_out) return MUIR_ERR_INVALID_ARG;
    if (f->latent) {
        if (!fg || !ok_ptr(fg->dlatent)) return MUIR_ERR_INVALID_ARG;
        for (int X = 0; X < 5; ++X)
            if (projected(f, X) && (!ok_ptr(fg->dU[X]) || !ok_ptr(fg->dbias[X])))
                return MUIR_ERR_INVALID_ARG;
    }
    const size_t need = fused_ws(s, f, true);
    if (ws_bytes < need || (need > 0 && !ok_ptr(ws))) return MUIR_ERR_WORKSPACE;
    if ((st = check_device()) != MUIR_OK) return st;
    muir::ChunkProblem P = make_problem(s, q, k, v, g, e, w, gamma);
    P.aux = const_cast<float*>(aux);
    muir::v2::GatesArgs ga;
    if (fused_any(f)) {
        P.zo = f->z_out;
        P.o_pre = const_cast<void*>(o_pre);
        P.o_pre_f32 = s->out_dtype == MUIR_FP32;
        P.dzo = dz_out;
        P.qk_raw = f->qk_raw;
        P.fused_ws = fused_region(s, ws, true);
        if (f->latent) {
            setup_projection(s, f, P.fused_ws, true, ga, P, gout, fg);
            P.dzo = gout[MUIR_FAM_OUTGATE];
        }
    }
    return from_cuda(muir::run_chunk_bwd(P, S0, S_chunks, M_chunks, dO, dS_final, dq, dk, dv,
                                         gout[MUIR_FAM_DECAY], gout[MUIR_FAM_ERASE],
                                         gout[MUIR_FAM_WRITE], gout[MUIR_FAM_READOUT], dS0, ws,
                                         ws_bytes, static_cast<cudaStream_t>(stream)));
}

muir_status muir_selftest_expired_wait(int limit_us, void* stream) {
    if (limit_us < 1 || limit_us > 1000000) return MUIR_ERR_INVALID_ARG;
    muir_status st = check_device();
    if (st != MUIR_OK) return st;
    return from_cuda(muir::launch_expired_wait(limit_us, static_cast<cudaStream_t>(stream)));
}

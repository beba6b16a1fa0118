// chunk.cu -- workspace sizing and dtype / head-dim dispatch of the chunkwise
// forward and backward.  The kernels live in chunk_impl.cuh and are
// instantiated in chunk_{bf16,f32}_d{64,128}.cu.
#include "chunk_impl.cuh"
#include "chunk_units.h"
#include "bwd2.h"
#include "fwd2.h"
#include "gates.h"

namespace muir {

size_t chunk_aux_floats(int C, int D) { return make_aux_lay(C, D).total; }

static size_t old_fwd_ws_bytes(int B, int T, int H, int D, int C, bool have_states) {
    const size_t nch = (size_t)B * H * ((T + C - 1) / C), DD = (size_t)D * D;
    size_t f = 2 * nch * DD;               // M, Bn
    if (!have_states) f += nch * DD;       // chunk-start states
    f += (size_t)num_slots((int)nch) * slot_floats(C, D);
    f += tail_side_floats(B, T, H, D, C);
    return f * sizeof(float);
}

// The on-chip tensor-core forward (fwd2.cu) runs when the shape allows it;
// its first 256 bytes of workspace hold the device flags (span flag first),
// the rest is shared with the boundary-pivot path, which runs after it and
// only when the span flag is set.
static bool use_v2(const ChunkProblem& P) {
    return v2::fwd2_supported(P.B, P.T, P.H, P.D, P.C, P.in_bf16);
}

// Floats of the saved per-chunk intermediates (muir_chunk_aux_floats): the
// larger of the two paths' formats (the boundary-pivot path writes its own
// when a chunk's span exceeds the single pivot).
size_t chunk_aux_total_floats(int B, int T, int H, int D, int C, bool in_bf16) {
    const size_t nch = (size_t)B * H * ((T + C - 1) / C);
    const size_t old = nch * chunk_aux_floats(C, D);
    if (!v2::fwd2_supported(B, T, H, D, C, in_bf16)) return old;
    const size_t nv2 = v2::aux_bytes(nch, (size_t)B * H) / sizeof(float);
    return old > nv2 ? old : nv2;
}

// Workspace of the on-chip forward: flags, then M (unless given), Bn, Q'
// (unless saved), O_intra, chunk states (unless given).
static size_t v2_fwd_arrays(size_t nch) { return 5 * nch * 128 * 128 * sizeof(float); }

size_t chunk_fwd_ws_bytes(int B, int T, int H, int D, int C, bool have_states, bool in_bf16) {
    const size_t old = old_fwd_ws_bytes(B, T, H, D, C, have_states);
    if (!v2::fwd2_supported(B, T, H, D, C, in_bf16)) return old;
    const size_t nv2 = v2_fwd_arrays((size_t)B * H * (T / C));
    return 256 + (old > nv2 ? old : nv2);
}

static size_t old_bwd_ws_bytes(int B, int T, int H, int D, int C, bool have_states);

// Backward workspace: flags; then (shared with the boundary-pivot path) the
// on-chip backward's arrays and, when the forward's intermediates are not
// passed in, a recomputed forward (its arrays and saved records).
size_t chunk_bwd_ws_bytes(int B, int T, int H, int D, int C, bool have_states, bool in_bf16) {
    const size_t old = old_bwd_ws_bytes(B, T, H, D, C, have_states);
    if (!v2::fwd2_supported(B, T, H, D, C, in_bf16)) return old;
    const size_t nch = (size_t)B * H * (T / C);
    const size_t nv2 = v2::bwd2_ws_bytes(B, T, H) + v2_fwd_arrays(nch) + v2::aux_bytes(nch, (size_t)B * H);
    return 256 + (old > nv2 ? old : nv2);
}

static size_t old_bwd_ws_bytes(int B, int T, int H, int D, int C, bool have_states) {
    const size_t nch = (size_t)B * H * ((T + C - 1) / C), DD = (size_t)D * D;
    size_t f = 3 * nch * DD;               // M, Bn / B', dS at chunk ends
    if (!have_states) f += nch * DD;
    f += (size_t)num_slots((int)nch) * slot_floats(C, D);
    f += tail_side_floats(B, T, H, D, C);
    return f * sizeof(float);
}

cudaError_t run_chunk_fwd(const ChunkProblem& P, const float* S0, void* o, float* S_final,
                          float* S_chunks, float* M_chunks, void* ws, size_t, cudaStream_t st) {
    if (use_v2(P)) {
        int* flags = static_cast<int*>(ws);
        char* shared = static_cast<char*>(ws) + 256;
        const size_t blk = (size_t)128 * 128;
        const size_t nch = (size_t)P.B * P.H * P.N;
        float* f = reinterpret_cast<float*>(shared);
        v2::Fwd2Args a = {};
        a.B = P.B; a.T = P.T; a.H = P.H; a.out_bf16 = P.out_bf16;
        a.q = P.q; a.k = P.k; a.v = P.v; a.g = P.g; a.e = P.e; a.w = P.w; a.gamma = P.gamma;
        a.S0 = S0; a.o = o; a.S_final = S_final;
        a.M = M_chunks ? M_chunks : f; if (!M_chunks) f += nch * blk;
        a.Bn = f; f += nch * blk;
        a.Oi = f; f += nch * blk;
        a.S_chunks = S_chunks ? S_chunks : f; f += nch * blk;
        if (P.aux) {  // save the intermediates the backward reuses
            unsigned char* ax = reinterpret_cast<unsigned char*>(P.aux);
            a.aux = ax;
            a.Qp = v2::aux_Qp(ax, nch);
            a.Mt = v2::aux_Mt(ax, nch);
            a.S_last = v2::aux_SN(ax, nch);
        } else {
            a.Qp = f; f += nch * blk;
        }
        a.flags = flags;
        // fused stages: output gate in k2_out, q/k prologue in k2_intra (its
        // inverse row norms saved with the intermediates, else in fused_ws)
        const long long rows = (long long)P.B * P.T * P.H;
        char* fw = P.fused_ws;
        if ((P.zo || P.qk_raw) && !fw) return cudaErrorInvalidValue;
        a.zo = P.zo; a.o_pre = P.o_pre;
        a.qk_raw = P.qk_raw;
        if (P.qk_raw)
            a.rnorm = P.aux ? v2::aux_rn(reinterpret_cast<unsigned char*>(P.aux), nch, (size_t)P.B * P.H)
                            : reinterpret_cast<float*>(fw + 256);
        cudaError_t e = cudaSuccess;
        if (P.gate_proj)  // projected gates first: everything below reads them
            e = v2::run_gates_fwd(*static_cast<const v2::GatesArgs*>(P.gate_proj), st);
        if (e == cudaSuccess) e = cudaMemsetAsync(flags, 0, 16, st);  // k2_intra raises the span flag
        if (e == cudaSuccess) e = v2::run_fwd2(a, st);
        if (e != cudaSuccess) return e;
        ChunkProblem G = P;
        G.gate = flags;  // boundary-pivot path only when a chunk's span exceeds the single pivot
        if (P.qk_raw) {
            // that path reads q^ and k^ as tensors: it runs in fp32 on fp32 copies
            // of every input (q^, k^ from the prologue, the others exact), so that
            // the normalised rows keep their full precision
            float* x32 = reinterpret_cast<float*>(fw + fused_f32_offset(P.B, P.T, P.H, P.D, P.C));
            const long long n = rows * 128;
            const void* src[7] = {P.q, P.k, P.v, P.g, P.e, P.w, P.gamma};
            for (int i = 0; i < 7; ++i) {
                e = i < 2 ? qk_materialise_gated(flags, src[i], x32 + i * n, rows, true, st)
                          : upcast_gated(flags, src[i], x32 + i * n, n, false, st);
                if (e != cudaSuccess) return e;
            }
            G.q = x32; G.k = x32 + n; G.v = x32 + 2 * n; G.g = x32 + 3 * n; G.e = x32 + 4 * n;
            G.w = x32 + 5 * n; G.gamma = x32 + 6 * n;
            G.in_bf16 = false;
            e = fwd_f32_d128(G, S0, o, S_final, S_chunks, M_chunks, shared, st);
        } else {
            e = fwd_bf16_d128(G, S0, o, S_final, S_chunks, M_chunks, shared, st);
        }
        if (e != cudaSuccess) return e;
        if (P.zo && o) return out_gate_fix_gated(flags, o, P.o_pre, P.zo, rows * 128, P.out_bf16, st);
        return cudaSuccess;
    }
    if (P.in_bf16) {
        if (P.D == 128) return fwd_bf16_d128(P, S0, o, S_final, S_chunks, M_chunks, ws, st);
        return fwd_bf16_d64(P, S0, o, S_final, S_chunks, M_chunks, ws, st);
    }
    if (P.D == 128) return fwd_f32_d128(P, S0, o, S_final, S_chunks, M_chunks, ws, st);
    return fwd_f32_d64(P, S0, o, S_final, S_chunks, M_chunks, ws, st);
}

cudaError_t run_chunk_bwd(const ChunkProblem& P, const float* S0, const float* S_chunks,
                          const float* M_chunks, const void* dO, const float* dS_final, void* dq, void* dk, void* dv,
                          void* dg, void* de, void* dw, void* dgamma, float* dS0, void* ws,
                          size_t, cudaStream_t st) {
    if (use_v2(P)) {
        int* flags = static_cast<int*>(ws);
        char* shared = static_cast<char*>(ws) + 256;
        const size_t blk = (size_t)128 * 128;
        const size_t nch = (size_t)P.B * P.H * P.N;
        cudaError_t e = cudaSuccess;
        if (P.gate_proj)  // the forward's projected gates, recomputed
            e = v2::run_gates_fwd(*static_cast<const v2::GatesArgs*>(P.gate_proj), st);
        if (e == cudaSuccess) e = cudaMemsetAsync(flags, 0, 16, st);  // k2_bwd2 (and a recomputed k2_intra) raise it
        if (e != cudaSuccess) return e;
        v2::Bwd2Args b = {};
        b.B = P.B; b.T = P.T; b.H = P.H;
        b.q = P.q; b.k = P.k; b.v = P.v; b.g = P.g; b.e = P.e; b.w = P.w; b.gamma = P.gamma;
        b.dO = dO; b.dS_final = dS_final;
        b.dq = dq; b.dk = dk; b.dv = dv; b.dg = dg; b.de = de; b.dw = dw; b.dgamma = dgamma;
        b.dS0 = dS0;
        const long long rows = (long long)P.B * P.T * P.H;
        char* fw = P.fused_ws;
        if ((P.zo || P.qk_raw) && !fw) return cudaErrorInvalidValue;
        char* qh = fw ? fw + 256 + nch * 2 * 128 * 4 : nullptr;
        char* kh = qh ? qh + rows * 128 * 2 : nullptr;
        if (P.zo) {  // fused output gate: k2_bprep forms the mixer's dO and dzo
            if (!P.o_pre || !P.dzo) return cudaErrorInvalidValue;
            b.zo = P.zo; b.o_pre = P.o_pre; b.o_pre_f32 = P.o_pre_f32; b.dzo = P.dzo;
            b.dO_eff = kh + rows * 128 * 2;  // fp16
            b.dO_effb = qh;                  // bf16 (the q^ region is not used here)
        }
        char* rest = shared;
        if (P.aux && S_chunks) {  // intermediates saved by the forward
            unsigned char* ax = reinterpret_cast<unsigned char*>(P.aux);
            b.aux = ax;
            b.Qp = v2::aux_Qp(ax, nch);
            b.Mt = v2::aux_Mt(ax, nch);
            b.S_last = v2::aux_SN(ax, nch);
            b.S_chunks = S_chunks;
            if (P.qk_raw) b.rnorm = v2::aux_rn(ax, nch, (size_t)P.B * P.H);
        } else {  // recompute the forward's state pass and intermediates
            float* f = reinterpret_cast<float*>(shared);
            unsigned char* ax = reinterpret_cast<unsigned char*>(f + 4 * nch * blk);
            v2::Fwd2Args a = {};
            a.B = P.B; a.T = P.T; a.H = P.H; a.out_bf16 = false;
            a.q = P.q; a.k = P.k; a.v = P.v; a.g = P.g; a.e = P.e; a.w = P.w; a.gamma = P.gamma;
            a.S0 = S0; a.o = nullptr; a.S_final = nullptr;
            a.M = f; a.Bn = f + nch * blk; a.Oi = f + 2 * nch * blk; a.S_chunks = f + 3 * nch * blk;
            a.aux = ax;
            a.Qp = v2::aux_Qp(ax, nch);
            a.Mt = v2::aux_Mt(ax, nch);
            a.S_last = v2::aux_SN(ax, nch);
            a.flags = flags;
            a.qk_raw = P.qk_raw;
            if (P.qk_raw) a.rnorm = reinterpret_cast<float*>(fw + 256);
            if ((e = v2::run_fwd2(a, st)) != cudaSuccess) return e;
            b.aux = ax; b.Qp = a.Qp; b.Mt = a.Mt; b.S_last = a.S_last; b.S_chunks = a.S_chunks;
            b.rnorm = a.rnorm;
            rest = reinterpret_cast<char*>(ax) + v2::aux_bytes(nch, (size_t)P.B * P.H);
        }
        b.ws = rest;
        b.flags = flags;
        if ((e = v2::run_bwd2(b, st)) != cudaSuccess) return e;
        ChunkProblem G = P;
        G.gate = flags;
        const void* dO_mix = P.zo ? static_cast<const void*>(b.dO_effb) : dO;
        if (P.qk_raw) {
            // the boundary-pivot path in fp32 on fp32 copies (as in the forward);
            // its dq^, dk^ go through the prologue's Jacobian, the rest to bf16
            float* x32 = reinterpret_cast<float*>(fw + fused_f32_offset(P.B, P.T, P.H, P.D, P.C));
            const long long n = rows * 128;
            // (the fused gate's dO from its fp16 copy)
            const void* src[8] = {P.q, P.k, P.v, P.g, P.e, P.w, P.gamma, P.zo ? b.dO_eff : dO};
            for (int i = 0; i < 8; ++i) {
                e = i < 2 ? qk_materialise_gated(flags, src[i], x32 + i * n, rows, true, st)
                          : upcast_gated(flags, src[i], x32 + i * n, n, i == 7 && P.zo, st);
                if (e != cudaSuccess) return e;
            }
            G.q = x32; G.k = x32 + n; G.v = x32 + 2 * n; G.g = x32 + 3 * n; G.e = x32 + 4 * n;
            G.w = x32 + 5 * n; G.gamma = x32 + 6 * n;
            G.in_bf16 = false;
            float* g32 = x32 + 8 * n;  // dq^, dk^, dv, dg, de, dw, dgamma
            if ((e = bwd_f32_d128(G, S0, S_chunks, M_chunks, x32 + 7 * n, dS_final, g32, g32 + n,
                                  g32 + 2 * n, g32 + 3 * n, g32 + 4 * n, g32 + 5 * n, g32 + 6 * n,
                                  dS0, shared, st)) != cudaSuccess)
                return e;
            if ((e = qk_jacobian_gated(flags, P.q, g32, true, dq, rows, st)) != cudaSuccess) return e;
            if ((e = qk_jacobian_gated(flags, P.k, g32 + n, true, dk, rows, st)) != cudaSuccess) return e;
            void* outs[5] = {dv, dg, de, dw, dgamma};
            for (int i = 0; i < 5; ++i)
                if ((e = downcast_gated(flags, g32 + (2 + i) * n, outs[i], n, st)) != cudaSuccess) return e;
        } else if ((e = bwd_bf16_d128(G, S0, S_chunks, M_chunks, dO_mix, dS_final, dq, dk, dv, dg, de,
                                      dw, dgamma, dS0, shared, st)) != cudaSuccess) {
            return e;
        }
        if (P.gate_proj)  // the projected gates' gradients -> latent, U, bias
            return v2::run_gates_bwd(*static_cast<const v2::GatesArgs*>(P.gate_proj), st);
        return cudaSuccess;
    }
#define MUIR_BWD_ARGS P, S0, S_chunks, M_chunks, dO, dS_final, dq, dk, dv, dg, de, dw, dgamma, dS0, ws, st
    if (P.in_bf16) {
        if (P.D == 128) return bwd_bf16_d128(MUIR_BWD_ARGS);
        return bwd_bf16_d64(MUIR_BWD_ARGS);
    }
    if (P.D == 128) return bwd_f32_d128(MUIR_BWD_ARGS);
    return bwd_f32_d64(MUIR_BWD_ARGS);
#undef MUIR_BWD_ARGS
}

}  // namespace muir

/*
 * muir.h -- C ABI of libmuir: the Muir gated delta rule on one NVIDIA B200.
 *
 * The operation (per batch b and head h, state S in R^{dk x dv}, rows = key
 * channels) is the recurrence of "Muir: Linear Attention with
 * Sensitivity-Allocated Gating and Matched-Filter Readout" (arXiv 2611.08376),
 * wolonglab.org page, section "Methodology", eq:gdn2 and eq:ours:
 *
 *     S_t = D_t S_{t-1} - (e_t * k_t) (k_t^T D_t S_{t-1}) + k_t (w_t * v_t)^T
 *     o_t = S_t^T (gamma_t * q_t),                  D_t = diag(exp(g_t))
 *
 * g is the log decay (caller applies any -softplus; precondition g <= 0), e the
 * erase gate, w the write gate, gamma the readout (matched-filter) gate; q and k
 * are expected to be unit-normalised by the caller.  No 1/sqrt(dk) scale and no
 * output gate are applied here.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named q, k, v, g, e, w, gamma, o, dO and the gradient outputs are
 *   DEVICE pointers.  Per-token tensors are token-major [B][T][H][d]
 *   (contiguous, d fastest); decode tensors are [B][H][d].  States are float32
 *   [B][H][dk][dv], row-major.  The caller owns all memory; the library never
 *   allocates or frees device memory: scratch comes from the caller's
 *   workspace (ws, ws_bytes), whose size the *_workspace() queries return.
 * - Every pointer must be 16-byte aligned.
 * - stream is a cudaStream_t (NULL = legacy default stream).  All work is
 *   enqueued asynchronously on it; no call synchronises the host.
 * - Argument checks run on the host before anything is enqueued; a failed
 *   check returns MUIR_ERR_INVALID_ARG or MUIR_ERR_UNSUPPORTED and enqueues
 *   nothing.  A launch failure returns MUIR_ERR_CUDA.
 * - Supported: dk == dv in {64, 128}; chunk in {16, 32, 64, 128, 256}; any
 *   T >= 1; a device of compute capability 10.x.  Inside the kernels g is
 *   clamped at -20 per token (exp(-20) ~ 2e-9; a row decayed that hard is
 *   already erased).
 * - Ragged tails: N = ceil(T / chunk) chunks per sequence.  When T % chunk
 *   != 0 the last chunk's rows are staged in the workspace, padded with zero
 *   tokens (q = k = v = e = w = gamma = 0, g = 0: the state passes through
 *   unchanged and o = 0), processed as a full chunk, and copied back; the
 *   workspace queries include those side buffers.
 * - dtype MUIR_BF16 means bfloat16 inputs; MUIR_FP32 means float32 inputs.
 *   Internal arithmetic is float32 with tensor-core TF32 products (three TF32
 *   passes for float32 inputs).  out_dtype selects o's storage.
 */
#ifndef MUIR_H_
#define MUIR_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MUIR_OK = 0,
    MUIR_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size */
    MUIR_ERR_UNSUPPORTED = 2,   /* valid but not implemented (head dim, chunk, device) */
    MUIR_ERR_WORKSPACE = 3,     /* ws too small or NULL with ws_bytes > 0 */
    MUIR_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    MUIR_ERR_DEVICE_TIMEOUT = 5 /* a bounded device-side wait expired */
} muir_status;

typedef enum { MUIR_BF16 = 0, MUIR_FP32 = 1 } muir_dtype;

typedef struct {
    int B, T, H;           /* batch, tokens, heads */
    int dk, dv;            /* key / value head dims (must be equal) */
    int chunk;             /* chunk size C of the chunkwise algorithm */
    muir_dtype in_dtype;   /* dtype of q, k, v, g, e, w, gamma, dO and of the input grads */
    muir_dtype out_dtype;  /* dtype of o */
} muir_shape;

/* Human-readable name of a status code (static string, never NULL). */
const char* muir_status_string(muir_status s);

/* Bounded device waits.  The chunk kernels wait on tensor-core completion
 * barriers with an iteration limit; a wait that runs out records the fact and
 * lets the kernel finish (its results are then not to be trusted) instead of
 * hanging the GPU.  This call synchronises the current device, returns
 * MUIR_ERR_DEVICE_TIMEOUT if any such wait expired since the previous call
 * (MUIR_ERR_CUDA if the synchronisation itself failed, else MUIR_OK) and
 * clears the record. */
muir_status muir_device_wait_status(void);

/* Self-test of the bounded device waits: enqueues one block that waits
 * limit_us microseconds (1 .. 1000000) on a shared-memory barrier that nothing
 * ever arrives on, with no copy or tensor-core operation in flight.  The wait
 * runs out, the expiry is recorded as for the chunk kernels' waits, and the
 * block exits, so the next muir_device_wait_status returns
 * MUIR_ERR_DEVICE_TIMEOUT.  Any other limit is MUIR_ERR_INVALID_ARG. */
muir_status muir_selftest_expired_wait(int limit_us, void* stream);

/* Bytes of device workspace muir_chunk_fwd / muir_chunk_bwd need for this
 * shape (0 for an invalid shape).  Host-only; enqueues nothing. */
size_t muir_chunk_fwd_workspace(const muir_shape* shape);
size_t muir_chunk_bwd_workspace(const muir_shape* shape);

/* Floats of the optional per-chunk intermediates muir_chunk_fwd can save for
 * muir_chunk_bwd (`aux`; 0 for an invalid shape): the decay-masked C x C
 * matrices, the inverse of the chunk's triangular system, the chunk's
 * transformed keys and values and its chunk-end quantities, in a layout
 * private to the library (it differs between the on-chip path and the
 * boundary-pivot path, and the size covers both).  Host-only. */
size_t muir_chunk_aux_floats(const muir_shape* shape);

/*
 * Chunkwise-parallel forward.  Same page, "Methodology": each chunk of C
 * tokens is written as a unit-lower-triangular system (WY/UT form); the
 * cumulative log decay is split at block boundaries so every exponential
 * applied to an operand is <= 1 ("boundary-pivoted", fig:kernel); chunk
 * states are propagated by a sequential pass with the float32 state on chip.
 *
 *   q, k, g, e, gamma : [B][T][H][dk]   in_dtype
 *   v, w              : [B][T][H][dv]   in_dtype
 *   S0                : [B][H][dk][dv]  float32, NULL = zero initial state
 *   o                 : [B][T][H][dv]   out_dtype (written)
 *   S_final           : [B][H][dk][dv]  float32, may be NULL (written)
 *   S_chunks          : [B][H][N][dk][dv] float32 (N = ceil(T/C)), may be NULL; receives the
 *                       state at the start of every chunk, which
 *                       muir_chunk_bwd can reuse instead of recomputing it.
 *   M_chunks          : [B][H][N][dk][dk] float32, may be NULL; receives the
 *                       chunk transitions M_n (S_{n+1} = M_n S_n + B_n), which
 *                       muir_chunk_bwd reuses together with S_chunks.
 *   aux               : muir_chunk_aux_floats(shape) float32, may be NULL;
 *                       receives the per-chunk intermediates muir_chunk_bwd
 *                       reuses together with S_chunks (masked matrices, block
 *                       inverses, Y) instead of recomputing them.
 */
muir_status muir_chunk_fwd(const muir_shape* shape, const void* q, const void* k,
                           const void* v, const void* g, const void* e, const void* w,
                           const void* gamma, const float* S0, void* o, float* S_final,
                           float* S_chunks, float* M_chunks, float* aux, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * Backward of muir_chunk_fwd ("custom backward pass", same page,
 * "Methodology"): gradients of L = sum(o * dO) + sum(S_final * dS_final).
 *
 *   inputs as for muir_chunk_fwd; dO [B][T][H][dv] in_dtype;
 *   dS_final [B][H][dk][dv] float32 or NULL (= 0);
 *   S_chunks: NULL (recompute the chunk states) or the array a previous
 *             muir_chunk_fwd with the same inputs wrote;
 *   M_chunks: NULL, or (with S_chunks) the transitions that forward wrote:
 *             then the per-chunk transitions are not recomputed;
 *   aux:      NULL, or (with S_chunks) the intermediates that forward wrote;
 *             aux without S_chunks is MUIR_ERR_INVALID_ARG;
 *   dq, dk, dg, de, dgamma [B][T][H][dk] and dv, dw [B][T][H][dv] are written
 *   in in_dtype; dS0 [B][H][dk][dv] float32 may be NULL.
 */
muir_status muir_chunk_bwd(const muir_shape* shape, const void* q, const void* k,
                           const void* v, const void* g, const void* e, const void* w,
                           const void* gamma, const float* S0, const float* S_chunks,
                           const float* M_chunks, const float* aux, const void* dO,
                           const float* dS_final, void* dq, void* dk,
                           void* dv, void* dg, void* de, void* dw, void* dgamma,
                           float* dS0, void* ws, size_t ws_bytes, void* stream);

/*
 * Packed variable-length sequences (streaming prefill of documents of mixed
 * length; same page, "Experiments": long streams): num_seqs independent
 * sequences stored back to back in one token-major buffer.
 *
 *   shape      : B must be 1; T = total tokens (0 allowed); other fields as above
 *   cu_seqlens : HOST array of num_seqs + 1 offsets, cu_seqlens[0] = 0,
 *                non-decreasing, cu_seqlens[num_seqs] = T; sequence i is
 *                rows [cu_seqlens[i], cu_seqlens[i+1]) of every per-token tensor
 *   S0, S_final, dS_final, dS0 : [num_seqs][H][dk][dv] float32, each may be NULL
 *   other tensors as muir_chunk_fwd / muir_chunk_bwd with B = 1
 * Each sequence runs the chunkwise path on its own rows (its own chunk grid and
 * ragged tail), one after another on `stream`, sharing the workspace; an empty
 * sequence copies S0 to S_final (dS_final to dS0), or writes zeros.  No chunk
 * states are saved: the backward recomputes them.  Bad offsets return
 * MUIR_ERR_INVALID_ARG before anything is enqueued.
 *
 * muir_chunk_varlen_workspace: bytes of workspace for the forward (backward != 0:
 * the backward); 0 for invalid arguments.  Host-only.
 */
size_t muir_chunk_varlen_workspace(const muir_shape* shape, int num_seqs,
                                   const long long* cu_seqlens, int backward);
muir_status muir_chunk_fwd_varlen(const muir_shape* shape, int num_seqs,
                                  const long long* cu_seqlens, const void* q, const void* k,
                                  const void* v, const void* g, const void* e, const void* w,
                                  const void* gamma, const float* S0, void* o, float* S_final,
                                  void* ws, size_t ws_bytes, void* stream);
muir_status muir_chunk_bwd_varlen(const muir_shape* shape, int num_seqs,
                                  const long long* cu_seqlens, const void* q, const void* k,
                                  const void* v, const void* g, const void* e, const void* w,
                                  const void* gamma, const float* S0, const void* dO,
                                  const float* dS_final, void* dq, void* dk, void* dv, void* dg,
                                  void* de, void* dw, void* dgamma, float* dS0, void* ws,
                                  size_t ws_bytes, void* stream);

/*
 * muir_chunk_fwd for callers that cannot allocate device memory.  The paper
 * has no counterpart; this is a deployment convenience.  Some hosts hand a
 * library only input and output pointers (plugin interfaces of runtimes that
 * own all device memory; hot paths where cudaMalloc is forbidden because it
 * can synchronise the device or break a fixed memory budget).  This call runs
 * the same forward as muir_chunk_fwd with its workspace in a 16 MiB array that
 * is part of the library's device image (held on every GPU that loads the
 * library until exit) and allocates nothing.
 *   - Arguments as muir_chunk_fwd, without S_chunks and workspace.
 *   - Returns MUIR_ERR_WORKSPACE when muir_chunk_fwd_workspace(shape) exceeds
 *     16 MiB (e.g. B=1, H=2, T=1024, d=64, chunk 64 fits).
 *   - All calls share the array: calls that overlap on the GPU race; order
 *     them (one stream).  No state carries over between calls.
 *   - The first call on each device looks up the array's device address with
 *     that device current and keeps it; make it before any stream capture.
 *     A device reset (cudaDeviceReset) after that first call is not
 *     supported: the kept address would be stale.
 *   - MUIR_ERR_UNSUPPORTED on a device that is not compute capability 10.x.
 */
muir_status muir_chunk_fwd_noalloc(const muir_shape* shape, const void* q, const void* k,
                                   const void* v, const void* g, const void* e, const void* w,
                                   const void* gamma, const float* S0, void* o, float* S_final,
                                   void* stream);

/*
 * Stages fused around the recurrence ("Muir", wolonglab.org page,
 * "Methodology" and fig. 3(b)): the block's q/k pathways end in SiLU with a
 * unit-normalised key, and a rank-128 gate g_t (the output gate; the tab:abl
 * caption compares against a widened one) multiplies the mixer's output.
 *
 *   z_out  : output-gate pre-activation [B][T][H][dv] in_dtype, or NULL (no
 *            gate).  The forward writes o * sigmoid(z_out); the backward takes
 *            the gradient of that gated output.
 *   qk_raw : 0, or 1 = the q and k arguments hold the raw pre-activations
 *            x_q, x_k: the kernels use SiLU(x) / ||SiLU(x)|| per token-head
 *            row (the same prologue as muir_qk_prologue), and the backward
 *            returns dq, dk with respect to x_q, x_k.
 * Runs where the on-chip path runs (in_dtype MUIR_BF16, dk = dv = 128,
 * chunk 128, T a multiple of 128); with any stage enabled, other shapes are
 * MUIR_ERR_UNSUPPORTED.  With both stages off the calls equal muir_chunk_fwd /
 * muir_chunk_bwd.
 */
typedef struct {
    int off;            /* first latent column of the family (multiple of 8) */
    int rank;           /* 0 = the family is not projected; else 64 or 128 */
    const void* U;      /* [rank][H*dk] in_dtype: the family's up-projection */
    const float* bias;  /* [H*dk] float32: its channel biases */
} muir_gate_family;

/* Families of the fused gate projection, in the pages' order (fig. 3(c)). */
enum { MUIR_FAM_DECAY = 0, MUIR_FAM_ERASE = 1, MUIR_FAM_OUTGATE = 2, MUIR_FAM_WRITE = 3,
       MUIR_FAM_READOUT = 4 };

typedef struct {
    const void* z_out;
    int qk_raw;
    /* Fused low-rank gate projection (same page, "Methodology", eq:ours_proj):
     * latent [B][T][R] in_dtype, one row per token shared by every head, or
     * NULL.  A family with rank > 0 takes its gate from
     *   pre[t][h][c] = sum_i latent[t][off + i] U[i][h*dk + c] + bias[h*dk + c]
     * instead of the tensor argument (which may then be NULL): log decay
     * g = -softplus(pre), erase e, write w and readout gain gamma = sigmoid(pre),
     * and the output gate's pre-activation z_out = pre (then fusion.z_out must
     * be NULL).  The gates are formed on the tensor cores in float32 and kept
     * in bf16, like gate inputs.  Families' latent columns must not overlap;
     * R is a multiple of 8. */
    const void* latent;
    int R;
    muir_gate_family fam[5];
} muir_fusion;

/* Gradients of the projection's parameters, written by muir_chunk_bwd_fused
 * when fusion.latent is set (NULL otherwise). */
typedef struct {
    void* dlatent;      /* [B][T][R] in_dtype (columns of no family: 0) */
    float* dU[5];       /* per projected family: [rank][H*dk] float32 */
    float* dbias[5];    /* per projected family: [H*dk] float32 */
} muir_fusion_grads;

/* Workspace bytes of muir_chunk_fwd_fused (backward == 0) or
 * muir_chunk_bwd_fused (backward != 0); 0 for an invalid shape or fusion.
 * Host-only. */
size_t muir_chunk_fused_workspace(const muir_shape* shape, const muir_fusion* fusion,
                                  int backward);

/*
 * muir_chunk_fwd with the fused stages.  Arguments as muir_chunk_fwd, plus:
 *   o      : [B][T][H][dv] out_dtype, the gated output when z_out is set
 *   o_pre  : [B][T][H][dv] out_dtype or NULL (NULL required without z_out):
 *            receives the pre-gate output, which muir_chunk_bwd_fused needs
 *   aux    : as muir_chunk_fwd; with qk_raw it also keeps the inverse row norms
 *            of q^ and k^ for the backward
 * A large decay span (a chunk whose channel log-decay total exceeds the single
 * pivot) runs the boundary-pivot path on q^, k^ materialised in the workspace
 * (bf16) and gates its output afterwards.  With a latent, the projected gates
 * are formed in the workspace by a tensor-core pre-pass before the chunk
 * kernels read them.
 */
muir_status muir_chunk_fwd_fused(const muir_shape* shape, const muir_fusion* fusion,
                                 const void* q, const void* k, const void* v, const void* g,
                                 const void* e, const void* w, const void* gamma,
                                 const float* S0, void* o, void* o_pre, float* S_final,
                                 float* S_chunks, float* M_chunks, float* aux, void* ws,
                                 size_t ws_bytes, void* stream);

/*
 * muir_chunk_bwd with the fused stages.  Arguments as muir_chunk_bwd, plus:
 *   o_pre  : the pre-gate output muir_chunk_fwd_fused wrote (required with
 *            z_out, else ignored), out_dtype of the shape
 *   dO     : gradient of the (gated) output, in_dtype
 *   dz_out : [B][T][H][dv] in_dtype, receives the gradient of z_out (required
 *            with z_out, else ignored)
 *   aux    : as muir_chunk_bwd; with qk_raw it must come from a forward called
 *            with qk_raw
 * dq, dk are gradients with respect to the raw x_q, x_k when qk_raw is set.
 * Missing o_pre / dz_out with z_out is MUIR_ERR_INVALID_ARG.  With a latent,
 * the gradients of projected families go to fgrads (required) and their
 * dg / de / dw / dgamma / dz_out arguments may be NULL; the forward's gates
 * are recomputed from the latent.
 */
muir_status muir_chunk_bwd_fused(const muir_shape* shape, const muir_fusion* fusion,
                                 const void* q, const void* k, const void* v, const void* g,
                                 const void* e, const void* w, const void* gamma,
                                 const float* S0, const float* S_chunks, const float* M_chunks,
                                 const float* aux, const void* o_pre, const void* dO,
                                 const float* dS_final, void* dq, void* dk, void* dv, void* dg,
                                 void* de, void* dw, void* dgamma, void* dz_out, float* dS0,
                                 const muir_fusion_grads* fgrads, void* ws, size_t ws_bytes,
                                 void* stream);

/*
 * One decode token for every (b, h) against a resident float32 state (same
 * page, "Experiments": streaming inference with a constant-size float32 state;
 * fig:longctx_niah: static or dynamic readout gain).
 *
 *   q, k, g, e : [B][H][dk]   dtype;    v, w : [B][H][dv]   dtype
 *   gamma      : [B][H][dk] (gamma_static == 0), [H][dk] shared by every b
 *                (gamma_static == 1), or NULL (gamma = 1)
 *   S          : [B][H][dk][dv] float32, updated in place
 *   o          : [B][H][dv] out_dtype
 * Bandwidth bound: S is read and written once.  No workspace.
 */
muir_status muir_recurrent_step(int B, int H, int dk, int dv, muir_dtype dtype,
                                muir_dtype out_dtype, const void* q, const void* k,
                                const void* v, const void* g, const void* e, const void* w,
                                const void* gamma, int gamma_static, float* S, void* o,
                                void* stream);

/*
 * q/k feature prologue (same page, "Methodology" and fig. 3(b): the query and
 * key pathways end in SiLU, and q and k are unit-normalised per head before
 * the recurrence).  Per row of d channels (one token of one head):
 *
 *     y = SiLU(x) / max(||SiLU(x)||_2, 1e-12),   SiLU(x) = x * sigmoid(x)
 *
 * so an all-zero row maps to zero.  The output is what muir_chunk_fwd and
 * muir_recurrent_step expect as q and k.
 *
 *   rows : number of rows (B*T*H for token-major [B][T][H][d]); 0 enqueues
 *          nothing and returns MUIR_OK
 *   d    : 64 or 128 (else MUIR_ERR_UNSUPPORTED)
 *   x, y : device [rows][d] in dtype; y may equal x (in place)
 * Float32 arithmetic (sigmoid from the fast exponential and division: within
 * about 1e-6 relative for |x| <= 10), y stored in dtype (round to nearest
 * even).  Bound by HBM: each row is read once and written once.
 */
muir_status muir_qk_prologue(long long rows, int d, muir_dtype dtype, const void* x, void* y,
                             void* stream);

/*
 * Backward of muir_qk_prologue: with s = SiLU(x), n = max(||s||, 1e-12),
 *     ds = dy / n - s (s . dy) / n^3   (ds = dy / 1e-12 when ||s|| < 1e-12)
 *     dx = ds * sigmoid(x) * (1 + x * (1 - sigmoid(x)))
 *   x, dy, dx : device [rows][d] in dtype; dx may equal dy or x.
 * Arguments and errors as muir_qk_prologue.
 */
muir_status muir_qk_prologue_bwd(long long rows, int d, muir_dtype dtype, const void* x,
                                 const void* dy, void* dx, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MUIR_H_ */

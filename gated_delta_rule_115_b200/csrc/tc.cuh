// tc.cuh -- dense products on the 5th-generation tensor cores (tcgen05).
//
// D[m][n] = sum_k A(m, k) B(k, n) for m < 128, n < N (N % 16 == 0, N <= 256),
// with A and B produced by element functors, staged through shared memory in
// K slabs of KS = 32 in the K-major, no-swizzle canonical layout (core matrix =
// 8 rows x 16 bytes; LBO = 128 B between the 4-element K groups, SBO = KS/4 *
// 128 B between 8-row groups), accumulated in TMEM (row m = TMEM lane m,
// column n = TMEM column n) by kind::tf32 MMAs (M = 128, K = 8) that one thread
// issues, completion tracked by tcgen05.commit on an mbarrier, read back with
// tcgen05.ld (32 lanes x 32 bit) for an element epilogue.
//
// PASSES = 1: operands rounded to TF32 (round to nearest) when staged.
// PASSES = 3: split TF32, hi = tf32(x), lo = tf32(x - hi); hi*hi + hi*lo + lo*hi.
//
// Every wait is bounded: after kSpinLimit polls a wait gives up, records an
// error code in the CTA's status word and returns (results are then garbage,
// nothing hangs).
#pragma once

#include <stdint.h>

#include <type_traits>

namespace muir {
namespace tc {

constexpr int KS = 32;                       // K slab staged per round
constexpr uint32_t kSpinLimit = 1u << 26;    // mbarrier polls before giving up

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100
    return d;                // base offset 0, legacy LBO mode, no swizzle
}

// Descriptor of an MN-major block in the 128-byte swizzle with 32-byte atoms
// (layout type 1); the block starts on a 1024-byte boundary.
__device__ __forceinline__ uint64_t make_desc_mn32(uint32_t saddr, uint32_t sbo) {
    return make_desc(saddr, 512, sbo) | ((uint64_t)1 << 61);
}

// Instruction descriptor: kind::tf32, D = f32, A = B = tf32, both K-major.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ float tf32_rn(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

// Byte offset of element (row, k) in a K-major canonical slab with KS columns.
__device__ __forceinline__ uint32_t kmaj_off(int row, int k) {
    return (uint32_t)((row >> 3) * (KS / 4 * 128) + (k >> 2) * 128 + (row & 7) * 16 + (k & 3) * 4);
}

struct State {
    uint32_t tmem;     // TMEM base address (lane 0, first allocated column)
    uint64_t* mbar;    // completion barrier in shared memory
    uint32_t phase;    // parity of the next phase to wait for
    int* status;       // CTA status word in shared memory (0 = ok)
};

// Allocate ncols TMEM columns (power of two >= 32); all threads call it.
__device__ __forceinline__ void init(State& s, uint32_t* tmem_slot, uint64_t* mbar, int* status,
                                     int ncols) {
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(mbar)));
        *status = 0;
    }
    if (threadIdx.x < 32) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr(tmem_slot)), "r"(ncols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;");
    s.tmem = *tmem_slot;
    s.mbar = mbar;
    s.phase = 0;
    s.status = status;
}

__device__ __forceinline__ void release(const State& s, int ncols) {
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    if (threadIdx.x < 32)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(s.tmem),
                     "r"(ncols));
}

// Wait (bounded) for the mbarrier phase s.phase, then flip it.  All threads call.
__device__ __forceinline__ void wait_mma(State& s) {
    uint32_t done = 0;
    for (uint32_t it = 0; it < kSpinLimit && !done; ++it) {
        asm volatile(
            "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
            "selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(smem_addr(s.mbar)), "r"(s.phase));
    }
    if (!done) *s.status = 1;
    s.phase ^= 1u;
    asm volatile("tcgen05.fence::after_thread_sync;");
}

__device__ __forceinline__ void issue_mma(uint32_t tmem, uint64_t da, uint64_t db, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}" ::"r"(tmem),
        "l"(da), "l"(db), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void commit(const State& s) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_addr(s.mbar)));
}

// Shared-memory bytes a gemm<PASSES, N> needs for its staging buffers.
template <int PASSES, int N>
__host__ __device__ constexpr int stage_bytes() {
    return (PASSES == 3 ? 2 : 1) * (128 + N) * KS * 4;
}

// Stage one operand slab: rows [0, R) x K columns [k0, k0 + KS) into `dst`
// (and `dst_lo` for PASSES == 3).  f4(row, k, out[4]) produces elements
// (row, k..k+3) with k a multiple of 4 (zeros past kmax).  ROW_LANES: lanes
// walk rows (source contiguous along rows) instead of K groups.  All loads of a
// thread are issued before its shared-memory stores so they overlap.
template <int PASSES, bool ROW_LANES, int R, class F4>
__device__ __forceinline__ void stage(unsigned char* dst, unsigned char* dst_lo, int k0, int kmax,
                                      const F4& f4) {
    constexpr int KG = KS / 4;
    constexpr int ITEMS = (R * KG + 255) / 256;
    float v[ITEMS][4];
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) {
        const int idx = threadIdx.x + it * 256;
        int row, kg;
        if (ROW_LANES) { row = idx % R; kg = idx / R; }
        else { kg = idx % KG; row = idx / KG; }
        const int k = k0 + 4 * kg;
        v[it][0] = v[it][1] = v[it][2] = v[it][3] = 0.f;
        if (idx < R * KG && k < kmax) f4(row, k, v[it]);
    }
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) {
        const int idx = threadIdx.x + it * 256;
        if (idx >= R * KG) break;
        int row, kg;
        if (ROW_LANES) { row = idx % R; kg = idx / R; }
        else { kg = idx % KG; row = idx / KG; }
        float4 hi, lo;
        hi.x = tf32_rn(v[it][0]); hi.y = tf32_rn(v[it][1]); hi.z = tf32_rn(v[it][2]); hi.w = tf32_rn(v[it][3]);
        *reinterpret_cast<float4*>(dst + kmaj_off(row, 4 * kg)) = hi;
        if (PASSES == 3) {
            lo.x = tf32_rn(v[it][0] - hi.x); lo.y = tf32_rn(v[it][1] - hi.y);
            lo.z = tf32_rn(v[it][2] - hi.z); lo.w = tf32_rn(v[it][3] - hi.w);
            *reinterpret_cast<float4*>(dst_lo + kmaj_off(row, 4 * kg)) = lo;
        }
    }
}

struct RowStore {
    float* dst;  // row-major destination, 16-byte aligned rows
    int ld;      // floats between rows (multiple of 4)
};

// Epilogue that takes eight consecutive columns of one row at once:
// f(row, c0, v[8]) with v[j] = D[row][c0 + j].
template <class F>
struct Row8 {
    F f;
};
template <class T>
struct is_row8 : std::false_type {};
template <class F>
struct is_row8<Row8<F>> : std::true_type {};

// D (128 x N, TMEM) = sum over K of A(m, k) B(k, n).  fa4(m, k, v[4]) gives
// A(m, k..k+3); fb4(n, k, v[4]) gives B(k..k+3, n).  Rows m >= M are zero.
// Then epi(m, n, value) for m < M, n < N.  All threads of the CTA call it.
template <int PASSES, int N, bool A_ROW_LANES, bool B_ROW_LANES, class FA4, class FB4, class EPI>
__device__ void gemm(State& s, unsigned char* sbuf, int M, int K, const FA4& fa4, const FB4& fb4,
                     const EPI& epi) {
    static_assert(N % 16 == 0 && N <= 256, "N");
    constexpr int ABYTES = 128 * KS * 4, BBYTES = N * KS * 4;
    unsigned char* sA = sbuf;
    unsigned char* sB = sbuf + ABYTES;
    unsigned char* sAl = sbuf + ABYTES + BBYTES;
    unsigned char* sBl = sAl + ABYTES;
    constexpr uint32_t idesc = idesc_tf32(128, N);
    constexpr uint32_t SBO = KS / 4 * 128;
    const int nslab = (K + KS - 1) / KS;
    for (int sl = 0; sl < nslab; ++sl) {
        const int k0 = sl * KS;
        stage<PASSES, A_ROW_LANES, 128>(sA, sAl, k0, K, [&](int m, int k, float* v) {
            if (m < M) fa4(m, k, v);
        });
        stage<PASSES, B_ROW_LANES, N>(sB, sBl, k0, K, fb4);
        asm volatile("fence.proxy.async.shared::cta;");
        __syncthreads();
        if (threadIdx.x == 0) {
            asm volatile("tcgen05.fence::after_thread_sync;");
#pragma unroll
            for (int ks = 0; ks < KS / 8; ++ks) {
                const uint32_t acc = (sl > 0 || ks > 0) ? 1u : 0u;
                const uint64_t da = make_desc(smem_addr(sA) + ks * 256, 128, SBO);
                const uint64_t db = make_desc(smem_addr(sB) + ks * 256, 128, SBO);
                issue_mma(s.tmem, da, db, idesc, acc);
                if (PASSES == 3) {
                    const uint64_t dal = make_desc(smem_addr(sAl) + ks * 256, 128, SBO);
                    const uint64_t dbl = make_desc(smem_addr(sBl) + ks * 256, 128, SBO);
                    issue_mma(s.tmem, da, dbl, idesc, 1u);
                    issue_mma(s.tmem, dal, db, idesc, 1u);
                }
            }
            commit(s);
        }
        wait_mma(s);  // the slab buffers are free again and, after the last slab, D is final
    }
    // epilogue: warp w reads TMEM lanes [32 (w % 4), +32) and half of the columns
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int row = 32 * quarter + lane;
    constexpr int NH = N / 2;
    for (int c0 = half * NH; c0 < (half + 1) * NH; c0 += 8) {
        uint32_t r[8];
        const uint32_t taddr = s.tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)c0;
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                       "=r"(r[6]), "=r"(r[7])
                     : "r"(taddr));
        asm volatile("tcgen05.wait::ld.sync.aligned;");
        if (row < M) {
            if constexpr (std::is_same<EPI, RowStore>::value) {
                float* d = epi.dst + (size_t)row * epi.ld + c0;
                *reinterpret_cast<float4*>(d) = make_float4(__uint_as_float(r[0]), __uint_as_float(r[1]),
                                                            __uint_as_float(r[2]), __uint_as_float(r[3]));
                *reinterpret_cast<float4*>(d + 4) = make_float4(__uint_as_float(r[4]), __uint_as_float(r[5]),
                                                                __uint_as_float(r[6]), __uint_as_float(r[7]));
            } else if constexpr (is_row8<EPI>::value) {
                float v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[j]);
                epi.f(row, c0, v);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) epi(row, c0 + j, __uint_as_float(r[j]));
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
}


// ------------------------------------------------------------------ asynchronous staging

// One K segment of an operand that is copied verbatim from float32 memory by
// cp.async (the tensor core reads it as TF32 by truncation; used for
// intermediates only, input-derived operands keep round-to-nearest producers).
struct Src {
    const float* p;  // nullptr: this K range comes from the element producer
    int ld;          // floats between consecutive source rows
    int k0;          // first operand K index of the segment
    bool mn;         // false: source rows are the operand's rows (K contiguous);
                     // true:  source rows are K (the operand's rows contiguous)
    bool neg;        // negate the segment's products (A operand only)
};

__device__ __forceinline__ Src no_src() { return Src{nullptr, 0, 0, false, false}; }

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(g),
                 "r"(valid ? 16 : 0));
}

// One 8-deep K block of R rows.  K-major: core matrices 8 rows x 16 B,
// LBO = 128 B (second 4-element K group), SBO = 256 B (next 8 rows).  MN-major
// (32-bit operands accept only this form): 128-byte rows of 32 consecutive
// M/N elements, one row per k, 4 rows per 512-byte atom, the 32-byte chunk
// index of a row XORed with k % 4; LBO = 512 B (next 32 M/N elements), SBO =
// R / 32 * 512 B (next 4 k).
__device__ __forceinline__ uint32_t kblk_off(int r, int kk) {
    return (uint32_t)((r >> 3) * 256 + (kk >> 2) * 128 + (r & 7) * 16 + (kk & 3) * 4);
}

// Byte offset of the four consecutive M/N elements starting at m (m % 4 == 0)
// in row kk of an 8-deep MN-major K block whose 4-row groups lie sbo bytes apart.
__device__ __forceinline__ uint32_t mn_off(int m, int kk, uint32_t sbo) {
    return (uint32_t)((kk >> 2) * sbo + (m >> 5) * 512 + (kk & 3) * 128 +
                      ((((m & 31) >> 3) ^ (kk & 3)) << 5) + (m & 4) * 4);
}

template <int R>
__device__ __forceinline__ void copy_block(unsigned char* blk, const Src& a, int k, int rvalid,
                                           int kmax) {
    const uint32_t base = smem_addr(blk);
    if (!a.mn) {
        for (int idx = threadIdx.x; idx < R * 2; idx += blockDim.x) {
            const int r = idx >> 1, h = idx & 1;
            const bool ok = r < rvalid && k + 4 * h < kmax;
            const float* g = a.p + (size_t)(ok ? r : 0) * a.ld + (ok ? (k - a.k0 + 4 * h) : 0);
            cp_async16(base + (uint32_t)((r >> 3) * 256 + h * 128 + (r & 7) * 16), g, ok);
        }
    } else {
        static_assert(R % 32 == 0, "MN-major blocks hold whole 32-element rows");
        constexpr uint32_t SBO = (R / 32) * 512;
        for (int idx = threadIdx.x; idx < R * 2; idx += blockDim.x) {
            const int m = 4 * (idx % (R / 4)), kk = idx / (R / 4);
            const bool ok = m < rvalid && k + kk < kmax;
            const float* g = a.p + (size_t)(ok ? (k - a.k0 + kk) : 0) * a.ld + (ok ? m : 0);
            cp_async16(base + mn_off(m, kk, SBO), g, ok);
        }
    }
}

// K-major segments of a whole 32-deep slab (four 8-deep K blocks, block kb of
// the slab at blk + kb * R * 32) in one pass: a warp copies 64 contiguous bytes
// of each of 8 rows (sixteen 16-byte pieces of a row cover the slab), the 8
// lanes of a store phase take 8 different rows (distinct bank groups).
// MN-major segments are left to copy_block.
template <int R, class SRC>
__device__ __forceinline__ void copy_slab_k(unsigned char* blk, const SRC& src, int k0, int rvalid,
                                            int kmax) {
    constexpr int PIECES = R * 8;  // 8 pieces of 16 bytes per row per slab
    for (int idx = threadIdx.x; idx < PIECES; idx += blockDim.x) {
        const int lane = idx & 31, w = idx >> 5;
        const int r = (lane & 7) + 8 * (w % (R / 8));
        const int pc = (lane >> 3) + 4 * (w / (R / 8));  // piece of the row: 0 .. 7
        const int kb = pc >> 1, h = pc & 1;
        const int k = k0 + 8 * kb;
        if (k >= kmax) continue;
        const Src a = src(k);
        if (!a.p || a.mn) continue;
        const bool ok = r < rvalid && k + 4 * h < kmax;
        const float* g = a.p + (size_t)(ok ? r : 0) * a.ld + (ok ? (k - a.k0 + 4 * h) : 0);
        cp_async16(smem_addr(blk + kb * R * 32 + (r >> 3) * 256 + h * 128 + (r & 7) * 16), g, ok);
    }
}

template <int R, class F4>
__device__ __forceinline__ void produce_block(unsigned char* blk, int k, int rvalid, int kmax,
                                              const F4& f4) {
    constexpr int ITEMS = (R * 2 + 255) / 256;
    float v[ITEMS][4];
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) {
        const int idx = threadIdx.x + it * 256;
        const int r = idx >> 1, h = idx & 1;
        v[it][0] = v[it][1] = v[it][2] = v[it][3] = 0.f;
        if (idx < R * 2 && r < rvalid && k + 4 * h < kmax) f4(r, k + 4 * h, v[it]);
    }
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) {
        const int idx = threadIdx.x + it * 256;
        if (idx >= R * 2) break;
        const int r = idx >> 1, h = idx & 1;
        float4 x;
        x.x = tf32_rn(v[it][0]); x.y = tf32_rn(v[it][1]); x.z = tf32_rn(v[it][2]); x.w = tf32_rn(v[it][3]);
        *reinterpret_cast<float4*>(blk + kblk_off(r, 4 * h)) = x;
    }
}

template <int N>
__host__ __device__ constexpr int async_stage_bytes() {
    return 2 * 4 * (128 + N) * 32;
}

// Same product as gemm<1, N, ...> (single TF32 pass) with the K segments that
// asrc(k) / bsrc(k) describe copied asynchronously, two slabs in flight.
// sbuf starts on a 1024-byte boundary; an MN-major B segment needs N % 32 == 0.
// cp.async.wait_group with a run-time count (the instruction takes an immediate).
__device__ __forceinline__ void cp_async_wait_upto(int n) {
    switch (n) {
        case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
        case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
        case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
        case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
        case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
        case 5: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
        case 6: asm volatile("cp.async.wait_group 6;" ::: "memory"); break;
        default: asm volatile("cp.async.wait_group 7;" ::: "memory"); break;
    }
}

// Bytes of dynamic shared memory of this launch.
__device__ __forceinline__ uint32_t dynamic_smem_bytes() {
    uint32_t n;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(n));
    return n;
}

// Same product as gemm<1, N, ...> (single TF32 pass).  K is processed in
// rounds of as many 32-deep slabs as the sbytes of staging memory hold (at
// most 8): every slab's segments that asrc(k) / bsrc(k) describe are copied
// with cp.async at the start of the round (one group per slab), the others
// produced from their element functors; the MMAs of a slab are issued as soon
// as its group has landed, and the round ends with one completion wait.
// sbuf starts on a 1024-byte boundary; an MN-major B segment needs N % 32 == 0.
template <int N, class ASRC, class FA4, class BSRC, class FB4, class EPI>
__device__ void gemm_async(State& s, unsigned char* sbuf, int sbytes, int M, int NB, int K,
                           const ASRC& asrc, const FA4& fa4, const BSRC& bsrc, const FB4& fb4,
                           const EPI& epi) {
    static_assert(N % 16 == 0 && N <= 256, "N");
    constexpr int ABLK = 128 * 32, BBLK = N * 32;
    constexpr int SLAB = 4 * (ABLK + BBLK);
    const int nslab = (K + 31) / 32;
    int nbuf = sbytes / SLAB;
    nbuf = nbuf < 1 ? 1 : (nbuf > 8 ? 8 : nbuf);
    auto blkA = [&](int buf, int ks) { return sbuf + buf * SLAB + ks * ABLK; };
    auto blkB = [&](int buf, int ks) { return sbuf + buf * SLAB + 4 * ABLK + ks * BBLK; };
    for (int r0 = 0; r0 < nslab; r0 += nbuf) {
        const int nr = nslab - r0 < nbuf ? nslab - r0 : nbuf;
        for (int i = 0; i < nr; ++i) {
            copy_slab_k<128>(blkA(i, 0), asrc, (r0 + i) * 32, M, K);
            copy_slab_k<N>(blkB(i, 0), bsrc, (r0 + i) * 32, NB, K);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const int k = (r0 + i) * 32 + ks * 8;
                if (k >= K) break;
                const Src a = asrc(k), b = bsrc(k);
                if (a.p && a.mn) copy_block<128>(blkA(i, ks), a, k, M, K);
                if (b.p && b.mn) copy_block<N>(blkB(i, ks), b, k, NB, K);
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
        for (int i = 0; i < nr; ++i) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const int k = (r0 + i) * 32 + ks * 8;
                if (k >= K) break;
                if (!asrc(k).p) produce_block<128>(blkA(i, ks), k, M, K, fa4);
                if (!bsrc(k).p) produce_block<N>(blkB(i, ks), k, NB, K, fb4);
            }
        }
        for (int i = 0; i < nr; ++i) {
            cp_async_wait_upto(nr - 1 - i);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncthreads();
            if (threadIdx.x == 0) {
                asm volatile("tcgen05.fence::after_thread_sync;");
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const int k = (r0 + i) * 32 + ks * 8;
                    if (k >= K) break;
                    const Src a = asrc(k), b = bsrc(k);
                    const bool amn = a.p && a.mn, bmn = b.p && b.mn;
                    const uint64_t da = amn ? make_desc_mn32(smem_addr(blkA(i, ks)), 128 / 32 * 512)
                                            : make_desc(smem_addr(blkA(i, ks)), 128, 256);
                    const uint64_t db = bmn ? make_desc_mn32(smem_addr(blkB(i, ks)), N / 32 * 512)
                                            : make_desc(smem_addr(blkB(i, ks)), 128, 256);
                    const uint32_t idesc = idesc_tf32(128, N) | ((a.p && a.neg) ? (1u << 13) : 0u) |
                                           (amn ? (1u << 15) : 0u) | (bmn ? (1u << 16) : 0u);
                    issue_mma(s.tmem, da, db, idesc, k > 0 ? 1u : 0u);
                }
                if (i == nr - 1) commit(s);
            }
        }
        wait_mma(s);  // the round's buffers are free again; after the last round D is final
    }
    // epilogue (as in gemm)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int row = 32 * quarter + lane;
    constexpr int NH = N / 2;
    for (int c0 = half * NH; c0 < (half + 1) * NH; c0 += 8) {
        uint32_t r[8];
        const uint32_t taddr = s.tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)c0;
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                       "=r"(r[6]), "=r"(r[7])
                     : "r"(taddr));
        asm volatile("tcgen05.wait::ld.sync.aligned;");
        if (row < M) {
            if constexpr (std::is_same<EPI, RowStore>::value) {
                float* d = epi.dst + (size_t)row * epi.ld + c0;
                *reinterpret_cast<float4*>(d) = make_float4(__uint_as_float(r[0]), __uint_as_float(r[1]),
                                                            __uint_as_float(r[2]), __uint_as_float(r[3]));
                *reinterpret_cast<float4*>(d + 4) = make_float4(__uint_as_float(r[4]), __uint_as_float(r[5]),
                                                                __uint_as_float(r[6]), __uint_as_float(r[7]));
            } else if constexpr (is_row8<EPI>::value) {
                float v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[j]);
                epi.f(row, c0, v);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) epi(row, c0 + j, __uint_as_float(r[j]));
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
}

}  // namespace tc
}  // namespace muir

// tc2.cuh -- tcgen05 building blocks on 128-byte-swizzled shared-memory tiles.
//
// Tile format "T16": 128 rows x 128 columns of a 16-bit type (bf16 or fp16),
// stored as two column blocks of 64 (16 KB each); inside a block row r is 128
// bytes at r * 128, its 16-byte chunk c (columns 8c..8c+7) at position
// c ^ (r % 8) -- the layout a TMA load with CU_TENSOR_MAP_SWIZZLE_128B writes
// for a box of 64 columns x 128 rows, and the canonical 128B-swizzled layout of
// the tensor cores.  The same bytes serve as
//   * a K-major operand whose rows are the tile's rows and whose K runs along
//     the columns (a product that contracts over columns), and
//   * an MN-major operand whose K runs along the tile's rows and whose M/N runs
//     along the columns (a product that contracts over rows),
// so one row-major tile written by the thread that owns each row feeds both
// kinds of product without a transposed copy.
//
// Tile format "T32": R rows x 128 columns of float32 (TF32 operands), four
// column blocks of 32 (R * 128 bytes each), same swizzle; used K-major only.
//
// Accumulators live in tensor memory (TMEM): row m of an M = 128 product is
// lane m, column n is TMEM column n.  One thread issues the MMAs; completion
// is signalled by tcgen05.commit on an mbarrier.  Every wait is bounded in
// time: a wait that gives up returns false and the caller records a status
// instead of hanging the GPU.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace muir {
namespace t2 {

constexpr uint64_t kWaitNs = 2000000000ull;  // give up a wait after 2 s

__device__ __forceinline__ uint32_t saddr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ mbarriers

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(bar)), "r"(count));
}

// Make mbarrier initialisation visible to the async proxy (TMA, tensor cores).
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(saddr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for the phase of parity `parity` to complete; false after limit_ns.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          uint64_t limit_ns = kWaitNs) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        if (mbar_try(bar, parity)) return true;
        if (globaltimer() - t0 > limit_ns) return false;
    }
}

// Block-wide wait for a phase: warp 0 polls the barrier, every other warp
// sleeps at the block barrier instead of spending issue slots on polling.
// Returns false if the bounded wait expired.  All threads of the block call it.
__device__ __forceinline__ bool cta_wait(uint64_t* bar, uint32_t parity) {
    int ok = 1;
    if (threadIdx.x < 32) ok = mbar_wait(bar, parity) ? 1 : 0;
    ok = __syncthreads_and(ok);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    return ok != 0;
}

// Per-chunk fp32 128 x 128 blocks read only by this library's kernels (Q',
// the intra-chunk output, B_n, U') are kept 4-column-group-major: element
// (t, col) is component col % 4 of float4 number (col / 4) 128 + t.  A warp
// whose lanes own consecutive rows then moves one contiguous 512-byte run
// per 4-column group, where the row-major form costs a transaction per lane.
__device__ __forceinline__ float4* grp4(float* blk, int t, int col) {
    return reinterpret_cast<float4*>(blk) + (size_t)(col >> 2) * 128 + t;
}
__device__ __forceinline__ const float4* grp4(const float* blk, int t, int col) {
    return reinterpret_cast<const float4*>(blk) + (size_t)(col >> 2) * 128 + t;
}

// ------------------------------------------------------------------ TMA

// 3-D tiled load of one box into shared memory, completion counted in bytes
// on `bar`.  Plain per-CTA load (no multicast).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(saddr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(saddr(bar))
        : "memory");
}

// Untiled bulk copy global -> shared (bytes % 16 == 0, both 16-byte aligned),
// completion counted on `bar`.  No multicast.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            saddr(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(saddr(bar))
        : "memory");
}

// Untiled bulk copy shared -> global in this thread's bulk group; call
// bulk_commit() after a batch and bulk_wait_read() before the shared source
// is overwritten (fence_async_smem() + barrier before issuing, so generic
// writes to the source are visible).
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                     reinterpret_cast<uint64_t>(dst)),
                 "r"(saddr(src)), "r"(bytes)
                 : "memory");
}
// 3-D tiled store of one box from shared memory (the tile's layout as the
// map's swizzle gives it) in this thread's bulk group; the same rules as
// bulk_store.  Coordinates must be in range (no negative start).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y, int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z), "r"(saddr(src))
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Logistic sigmoid 1 / (1 + e^-z) through the base-2 exponential
// (e^-z = 2^(-z log2 e)) and a fast division (a few ulp; its results feed
// 16-bit operands or bf16 gates); saturates to 0 and 1 without NaN.
__device__ __forceinline__ float sigmoid_f(float z) {
    float e;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-1.4426950408889634f * z));
    return __fdividef(1.f, 1.f + e);
}

// Fetch the 128-byte line holding `ptr` into L2 (no register result).
__device__ __forceinline__ void prefetch_l2(const void* ptr) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr) : "memory");
}

// Bulk L2 prefetch of `bytes` (multiple of 16, 16-byte aligned) from global memory.
__device__ __forceinline__ void bulk_prefetch_l2(const void* ptr, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(ptr), "r"(bytes) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Generic-proxy shared-memory writes -> visible to the async proxy.
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ TMEM

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {  // one warp
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(slot)),
                 "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // one warp
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// TMEM address of (lane, column).
__device__ __forceinline__ uint32_t taddr(uint32_t base, int lane, int col) {
    return base + ((uint32_t)lane << 16) + (uint32_t)col;
}

// 32 consecutive columns of this thread's lane (32x32b shape: warp w % 4 reads
// lanes 32 (w % 4) .. +32).
__device__ __forceinline__ void tmem_ld32(uint32_t ta, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(ta));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld16(uint32_t ta, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(ta));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld8(uint32_t ta, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(ta));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t ta, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16};" ::"r"(ta),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------ descriptors

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), sm_100 version.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

constexpr uint32_t kT16Block = 128 * 128;  // bytes of one 64-column block of a T16 tile
constexpr uint32_t kT16Bytes = 2 * kT16Block;

// K-major operand from a T16 tile: rows r0.. (r0 % 8 == 0), K from column k0 (k0 % 16 == 0).
__device__ __forceinline__ uint64_t kdesc16(uint32_t tile, int r0, int k0) {
    return sdesc(tile + (uint32_t)(k0 >> 6) * kT16Block + (uint32_t)r0 * 128u +
                     (uint32_t)(k0 & 63) * 2u,
                 16, 1024);
}

// MN-major operand from a T16 tile (or a run of adjacent T16 tiles): K from
// row k0 (k0 % 8 == 0), M/N from column m0 (m0 % 64 == 0; columns past 127
// continue in the next tile).
__device__ __forceinline__ uint64_t mdesc16(uint32_t tile, int k0, int m0) {
    return sdesc(tile + (uint32_t)(m0 >> 6) * kT16Block + (uint32_t)k0 * 128u, kT16Block, 1024);
}

// K-major operand from a T32 tile of R rows: rows r0.., K from column k0 (k0 % 8 == 0).
template <int R>
__device__ __forceinline__ uint64_t kdesc32(uint32_t tile, int r0, int k0) {
    return sdesc(tile + (uint32_t)(k0 >> 5) * (R * 128u) + (uint32_t)r0 * 128u +
                     (uint32_t)(k0 & 31) * 4u,
                 16, 1024);
}

// Instruction descriptors (D = f32).
enum : uint32_t { kF16 = 0, kBF16 = 1, kTF32 = 2 };
__host__ __device__ constexpr uint32_t idesc(uint32_t fmt, int M, int N, bool a_mn, bool b_mn,
                                             bool neg_a = false) {
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((neg_a ? 1u : 0u) << 13) |
           ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d, uint64_t a, uint64_t b, uint32_t id,
                                        uint32_t acc) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d),
        "l"(a), "l"(b), "r"(id), "r"(acc));
}

__device__ __forceinline__ void mma_tf32(uint32_t d, uint64_t a, uint64_t b, uint32_t id,
                                         uint32_t acc) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}" ::"r"(d),
        "l"(a), "l"(b), "r"(id), "r"(acc));
}

// kind::tf32 with A read from tensor memory (lane m = row m, one fp32 per
// column along K) and B from a shared-memory descriptor.
__device__ __forceinline__ void mma_tf32_ta(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t id,
                                            uint32_t acc) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n}" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(id), "r"(acc));
}

__device__ __forceinline__ float tf32_round(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

// Arrive on `bar` once every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            saddr(bar))
        : "memory");
}

// ------------------------------------------------------------------ product issue
// (one thread; K multiple of 16 for 16-bit, of 8 for TF32)

// D[128][N] (+)= A[128][K] B[N][K]^T, A K-major rows 0..127 of tile `a` from column ka,
// B K-major rows nb.. of tile `b` from column kb.
__device__ __forceinline__ void gemm_kk16(uint32_t d, uint32_t a, int ka, uint32_t b, int nb,
                                          int kb, int N, int K, uint32_t fmt, bool acc,
                                          bool neg = false) {
    const uint32_t id = idesc(fmt, 128, N, false, false, neg);
    for (int k = 0; k < K; k += 16)
        mma_f16(d, kdesc16(a, 0, ka + k), kdesc16(b, nb, kb + k), id, (acc || k) ? 1u : 0u);
}

// D[128][N] (+)= A[128][K] B[K][N]: A K-major (tile a, columns ka..), B MN-major
// (tile b, rows kb.. as K, columns nb.. as N).
__device__ __forceinline__ void gemm_km16(uint32_t d, uint32_t a, int ka, uint32_t b, int kb,
                                          int nb, int N, int K, uint32_t fmt, bool acc,
                                          bool neg = false) {
    const uint32_t id = idesc(fmt, 128, N, false, true, neg);
    for (int k = 0; k < K; k += 16)
        mma_f16(d, kdesc16(a, 0, ka + k), mdesc16(b, kb + k, nb), id, (acc || k) ? 1u : 0u);
}

// D[128][N] (+)= A^T B with A MN-major (tile a: rows ka.. as K, columns ma.. as M)
// and B MN-major (tile b: rows kb.. as K, columns nb.. as N).
__device__ __forceinline__ void gemm_mm16(uint32_t d, uint32_t a, int ka, int ma, uint32_t b,
                                          int kb, int nb, int N, int K, uint32_t fmt, bool acc,
                                          bool neg = false) {
    const uint32_t id = idesc(fmt, 128, N, true, true, neg);
    for (int k = 0; k < K; k += 16)
        mma_f16(d, mdesc16(a, ka + k, ma), mdesc16(b, kb + k, nb), id, (acc || k) ? 1u : 0u);
}

// TF32: D[128][N] (+)= A[128][K] B[N][K]^T, both K-major T32 tiles (A of RA rows, B of RB rows).
template <int RA, int RB>
__device__ __forceinline__ void gemm_kk32(uint32_t d, uint32_t a, uint32_t b, int nb, int N,
                                          int K, bool acc) {
    const uint32_t id = idesc(kTF32, 128, N, false, false);
    for (int k = 0; k < K; k += 8)
        mma_tf32(d, kdesc32<RA>(a, 0, k), kdesc32<RB>(b, nb, k), id, (acc || k) ? 1u : 0u);
}

// ------------------------------------------------------------------ tile access

// Byte offset of 16-byte chunk c (columns 8c .. 8c+7, c < 16) of row r in a T16 tile.
__device__ __forceinline__ uint32_t t16_off(int r, int c) {
    return (uint32_t)(c >> 3) * kT16Block + (uint32_t)r * 128u + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

// Byte offset of 16-byte chunk c (columns 4c .. 4c+3, c < 32) of row r in a T32 tile of R rows.
template <int R>
__device__ __forceinline__ uint32_t t32_off(int r, int c) {
    return (uint32_t)(c >> 3) * (R * 128u) + (uint32_t)r * 128u + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(a)) |
           ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(b)) << 16);
}
__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
    return (uint32_t)__half_as_ushort(__float2half_rn(a)) |
           ((uint32_t)__half_as_ushort(__float2half_rn(b)) << 16);
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack16(float a, float b) {
    return BF16 ? pack_bf16(a, b) : pack_f16(a, b);
}

// Store 8 values as one 16-byte chunk (16-bit type) at chunk c of row r.
template <bool BF16>
__device__ __forceinline__ void st_chunk16(unsigned char* tile, int r, int c, const float* v) {
    uint4 u;
    u.x = pack16<BF16>(v[0], v[1]);
    u.y = pack16<BF16>(v[2], v[3]);
    u.z = pack16<BF16>(v[4], v[5]);
    u.w = pack16<BF16>(v[6], v[7]);
    *reinterpret_cast<uint4*>(tile + t16_off(r, c)) = u;
}

// Two 16-bit values packed in a word -> floats.
template <bool BF16>
__device__ __forceinline__ void unpack16(uint32_t w, float& lo, float& hi) {
    if (BF16) {
        lo = __uint_as_float(w << 16);
        hi = __uint_as_float(w & 0xFFFF0000u);
    } else {
        lo = __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu)));
        hi = __half2float(__ushort_as_half((unsigned short)(w >> 16)));
    }
}

// Load 8 values of chunk c of row r of a T16 tile.
template <bool BF16>
__device__ __forceinline__ void ld_chunk16(const unsigned char* tile, int r, int c, float* v) {
    const uint4 u = *reinterpret_cast<const uint4*>(tile + t16_off(r, c));
    unpack16<BF16>(u.x, v[0], v[1]);
    unpack16<BF16>(u.y, v[2], v[3]);
    unpack16<BF16>(u.z, v[4], v[5]);
    unpack16<BF16>(u.w, v[6], v[7]);
}

}  // namespace t2
}  // namespace muir

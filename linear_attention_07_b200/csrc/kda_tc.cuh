// sm_100a building blocks: tcgen05 MMA (kind::tf32 and kind::f16), tensor
// memory, shared memory matrix descriptors and mbarriers, as inline PTX.
//
// Shared-memory operand layouts (no swizzle).  A "core matrix" is 8 rows x
// 16 bytes stored contiguously (128 B): 4 elements of 32 bits or 8 of 16 bits
// along K.  For 32-bit elements:
//   K-major  (K contiguous):  element (mn, k) at
//       (mn / 8) * SBO + (k / 4) * LBO + (mn % 8) * 16 + (k % 4) * 4
//   MN-major (MN contiguous): element (mn, k) at
//       (mn / 4) * SBO + (k / 8) * LBO + (k % 8) * 16 + (mn % 4) * 4
// and for 16-bit elements:
//   K-major:  (mn / 8) * SBO + (k / 8) * LBO + (mn % 8) * 16 + (k % 8) * 2
//   MN-major: (mn / 8) * SBO + (k / 8) * LBO + (k % 8) * 16 + (mn % 8) * 2
// (so a K-major tile of a matrix is an MN-major tile of its transpose, with
// LBO and SBO exchanged)
// LBO is the byte distance between core matrices adjacent along K, SBO the
// distance between core matrices adjacent along M/N.  One tf32 MMA consumes
// K = 8 and one f16 MMA K = 16: two K-adjacent core matrices (K-major, and
// MN-major f16) or one (MN-major tf32), so the descriptor start advances by
// 2*LBO or LBO per step.
//
// Tensor memory: 128 lanes x 512 columns of 32 bits.  An M = 128
// accumulator puts row m in lane m; an M = 64 accumulator puts row m in
// lane (m % 16) + 32 * (m / 16).  A 16-bit A operand held in tensor memory
// packs two K-adjacent elements per column (the even k in the low half), so
// an f16 MMA reads 8 columns.  Warp w may only access lanes
// [32 (w % 4), 32 (w % 4) + 32).
#pragma once
#include <stdint.h>
#include <cuda_fp16.h>

namespace kda {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------ descriptors --

// Shared memory descriptor, no swizzle, descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;            // version
    // base offset 0, lbo mode 0, layout type 0 (no swizzle)
    return d;
}

// Instruction descriptor for kind::tf32 with fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4)                              // D format: f32
         | (2u << 7)                              // A format: tf32
         | (2u << 10)                             // B format: tf32
         | ((a_mn_major ? 1u : 0u) << 15)
         | ((b_mn_major ? 1u : 0u) << 16)
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor for kind::f16 with fp16 A and B (format code 0 for
// both) and fp32 accumulation; A K-major, B K-major or MN-major.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool b_mn_major = false) {
    return (1u << 4)                              // D format: f32
         | ((b_mn_major ? 1u : 0u) << 16)
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

// Byte offset of 16-bit element (mn, k) in the no-swizzle K-major layout.
__host__ __device__ constexpr uint32_t off16_kmajor(int mn, int k, uint32_t lbo, uint32_t sbo) {
    return (uint32_t)(mn / 8) * sbo + (uint32_t)(k / 8) * lbo + (uint32_t)(mn % 8) * 16u + (uint32_t)(k % 8) * 2u;
}

// Byte offsets inside the no-swizzle canonical layouts (32-bit elements).
__host__ __device__ constexpr uint32_t off_kmajor(int mn, int k, uint32_t lbo, uint32_t sbo) {
    return (uint32_t)(mn / 8) * sbo + (uint32_t)(k / 4) * lbo + (uint32_t)(mn % 8) * 16u + (uint32_t)(k % 4) * 4u;
}
__host__ __device__ constexpr uint32_t off_mnmajor(int mn, int k, uint32_t lbo, uint32_t sbo) {
    return (uint32_t)(mn / 4) * sbo + (uint32_t)(k / 8) * lbo + (uint32_t)(k % 8) * 16u + (uint32_t)(mn % 4) * 4u;
}

// ------------------------------------------------------------------- MMA --



// D[tmem] (+)= A[smem desc or tmem] * B[smem desc], and the commit that
// arrives on an mbarrier once every MMA issued before it has completed.
// Whole-warp forms: every lane of a converged warp calls them with the same
// (warp-uniform) arguments and one elected lane issues.  Issuing from a
// converged warp keeps the descriptors warp-uniform; a single-lane branch
// costs several times more per instruction, which bounds small-N MMAs.
__device__ __forceinline__ void mma_tf32_ss_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "setp.ne.b32 q, %4, 0;\n\t"
        "@p tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, q;\n\t}\n"
        :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_tf32_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "setp.ne.b32 q, %4, 0;\n\t"
        "@p tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, q;\n\t}\n"
        :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_f16_ss_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "setp.ne.b32 q, %4, 0;\n\t"
        "@p tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, q;\n\t}\n"
        :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_f16_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "setp.ne.b32 q, %4, 0;\n\t"
        "@p tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, q;\n\t}\n"
        :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_commit_w(uint32_t mbar_saddr) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "@p tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n"
        :: "r"(mbar_saddr) : "memory");
}


// ---------------------------------------------------------------- fences --

__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// make generic-proxy shared memory writes visible to the async proxy (MMA reads)
__device__ __forceinline__ void fence_smem_to_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ allocation --

// Whole warp: allocate `ncols` (power of two >= 32) TMEM columns; the base
// address is written to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_saddr, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(dst_saddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 :: "r"(taddr), "r"(ncols) : "memory");
}

// ------------------------------------------------------------- mbarriers --

__device__ __forceinline__ void mbar_init(uint32_t saddr, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(saddr), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ uint32_t mbar_try_wait(uint32_t saddr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok) : "r"(saddr), "r"(parity) : "memory");
    return ok;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
// Wait for phase `parity` to complete, giving up after `limit_ns`.  Each
// try_wait may block for a short, implementation-defined time before it
// returns false.  No suspend-time hint is given: with a long hint the waiting
// thread wakes measurably later (a few hundred cycles) after the phase
// completes.  Returns true on success, false on timeout.
// Non-blocking check of phase `parity` (mbarrier.test_wait).
__device__ __forceinline__ uint32_t mbar_test_wait(uint32_t saddr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok) : "r"(saddr), "r"(parity) : "memory");
    return ok;
}
// A limit of 0 checks once without blocking (tests that make waits run out).
__device__ __forceinline__ bool mbar_wait(uint32_t saddr, uint32_t parity, uint64_t limit_ns) {
    if (limit_ns == 0) return mbar_test_wait(saddr, parity);
    if (mbar_try_wait(saddr, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(saddr, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// A monotonic counter in shared memory, published with release and read with
// acquire semantics (CTA scope).  Unlike an mbarrier phase parity, a reader
// that falls behind by several steps still reads the right value.
__device__ __forceinline__ void counter_publish(uint32_t saddr, uint32_t v) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" :: "r"(saddr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t counter_read(uint32_t saddr) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(saddr) : "memory");
    return v;
}
// Wait until the counter reaches `target`; false once limit_ns has passed.
__device__ __forceinline__ bool counter_wait(uint32_t saddr, uint32_t target, uint64_t limit_ns) {
    if (counter_read(saddr) >= target) return true;
    if (limit_ns == 0) return false;
    const uint64_t t0 = globaltimer_ns();
    while (counter_read(saddr) < target) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
        __nanosleep(64);
    }
    return true;
}

// ------------------------------------------------------------------ TMA --

// Arrive on an mbarrier and add `bytes` to the transaction count it expects.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t saddr, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(saddr), "r"(bytes) : "memory");
}
// Tiled 3-D tensor load (no multicast) into shared memory; completion is
// signalled as transaction bytes on the mbarrier.
__device__ __forceinline__ void tma_load_3d(uint32_t dst_saddr, const void* tmap, int x, int y, int z,
                                            uint32_t mbar_saddr) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];"
        :: "r"(dst_saddr), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z),
           "r"(mbar_saddr) : "memory");
}

// --------------------------------------------------------------- cluster --

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Whole cluster barrier (all threads of all CTAs); release/acquire ordering.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
// Arrive on an mbarrier of another CTA of the cluster, relaxed: signals an
// event that orders no data (for example "this buffer may be overwritten"
// once every read of it has completed); much cheaper than a release arrive.
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t cluster_saddr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];"
                 :: "r"(cluster_saddr) : "memory");
}
// Cluster-scope acquiring wait (data written by other CTAs of the cluster).
__device__ __forceinline__ uint32_t mbar_try_wait_cluster(uint32_t saddr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok) : "r"(saddr), "r"(parity) : "memory");
    return ok;
}
__device__ __forceinline__ uint32_t mbar_test_wait_cluster(uint32_t saddr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok) : "r"(saddr), "r"(parity) : "memory");
    return ok;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t saddr, uint32_t parity, uint64_t limit_ns) {
    if (limit_ns == 0) return mbar_test_wait_cluster(saddr, parity);
    if (mbar_try_wait_cluster(saddr, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_cluster(saddr, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
    return true;
}
// Bulk copy of `bytes` (multiple of 16) from this CTA's shared memory to
// another CTA's shared memory in the cluster (no multicast); completion is
// counted as transaction bytes on the destination CTA's mbarrier.
__device__ __forceinline__ void bulk_copy_to_rank(uint32_t dst_cluster_saddr, uint32_t src_saddr,
                                                  uint32_t bytes, uint32_t mbar_cluster_saddr) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(dst_cluster_saddr), "r"(src_saddr), "r"(bytes), "r"(mbar_cluster_saddr) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Tiled 3-D tensor store from shared memory (a bulk group; commit it).
__device__ __forceinline__ void tma_store_3d(const void* tmap, int x, int y, int z, uint32_t src_saddr) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];"
        :: "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(src_saddr) : "memory");
}
// Wait until every committed bulk group has completed, writes included.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Plain arrive (release, CTA scope) on a local mbarrier.
__device__ __forceinline__ void mbar_arrive(uint32_t saddr) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(saddr) : "memory");
}
// Wait until the source buffers of all committed bulk copies may be reused.
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// ------------------------------------------------------ TMEM <-> registers --
// 32x32b shapes: thread l of warp w reads/writes lane 32 (w % 4) + l,
// columns [col, col + N).

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
          "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
          "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
          "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
          "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]),
          "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&v)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
        :: "r"(taddr),
           "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
           "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
           "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        :: "r"(taddr),
           "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
           "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
           "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
           "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
           "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
           "r"(__float_as_uint(v[15]))
        : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        :: "r"(taddr),
           "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
           "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
           "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
           "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
           "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
           "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
           "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
           "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
           "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
           "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
           "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

// Two fp32 values rounded to fp16 (nearest, ties to even) and packed into one
// 32-bit word, lo in the low half; returned as the word's bit pattern in a
// float register (the tensor-memory stores take 32-bit words).
__device__ __forceinline__ float pack_f16x2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return __uint_as_float(*reinterpret_cast<const uint32_t*>(&h));
}
__device__ __forceinline__ uint16_t to_f16_bits(float x) {
    return __half_as_ushort(__float2half_rn(x));
}

// Round an fp32 value to tf32 (nearest, ties away from zero): add half of the
// last kept unit to the magnitude bits and clear the 13 dropped bits.
__device__ __forceinline__ float to_tf32(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

}  // namespace tc
}  // namespace kda

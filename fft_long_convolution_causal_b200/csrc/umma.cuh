// umma.cuh -- thin wrappers over the sm_100a fifth-generation tensor-core
// instructions (tcgen05: tensor-memory allocation, MMA, commit, TMEM loads and
// stores) and the shared-memory mbarrier that MMA completion arrives on.
//
// Conventions used by the kernels (checked on B200 against exact integer
// products before use):
// * kind::f16 MMA, bf16 operands, fp32 accumulator, M = 128 (cta_group::1):
//   D row m lives in TMEM lane m, column n in TMEM column (D address + n).
// * A from TMEM: row m in lane m; 32-bit column c holds the K elements 2c (low
//   half) and 2c + 1 (high half); one K = 16 step spans 8 columns.
// * B from shared memory, K-major, no swizzle: core matrices of 8 rows (N) x
//   16 bytes (8 K elements), the two K halves 128 bytes apart (LBO) and
//   consecutive 8-row groups 256 bytes apart (SBO).
// * tcgen05.ld / st with shape 16x256b: register i of thread (g = lane / 4,
//   t = lane % 4) is TMEM lane g + 8 (i / 2), column 2 t + (i % 2) of an
//   8-column block (the mma.sync m16n8 accumulator layout); .xR repeats the
//   block over R consecutive 8-column blocks, registers 4r .. 4r + 3 for block r.
#pragma once

#include <stdint.h>

namespace fftc {
namespace um {

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// order tcgen05 operations against thread barriers
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// make generic-proxy shared-memory writes visible to the tensor core
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// instruction descriptor: bf16 x bf16 -> fp32, both operands K-major, M x N
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// shared-memory matrix descriptor, K-major, no swizzle, LBO 128 B, SBO 256 B
__device__ __forceinline__ uint64_t sdesc_kmajor(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) | ((uint64_t)(256u >> 4) << 32) |
           (1ull << 46);
}
// byte offset of element (row n, k) of a K = 16 B tile in that layout
__host__ __device__ constexpr uint32_t kmajor_off(int n, int k) {
    return (uint32_t)((n / 8) * 256 + (k / 8) * 128 + (n % 8) * 16 + (k % 8) * 2);
}

// D[tmem] (+)= A[tmem] x B[smem]; issued by one thread
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// D[tmem] (+)= A[smem] x B[smem]; issued by one thread
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// shared-memory matrix descriptor, no swizzle, with the core-matrix strides:
// lbo between core matrices adjacent along K, sbo along M or N (both majors)
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// instruction-descriptor bits: negate the A x B product; A / B MN-major
constexpr uint32_t kNegA = 1u << 13, kAmn = 1u << 15, kBmn = 1u << 16;

// arrive on the mbarrier once every MMA issued so far by this thread is complete
__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t addr, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(addr), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// One bounded probe: the thread may sleep up to ~20 us waiting for the phase.
__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\nselp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(addr), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}
// Probes of a bounded wait by default (on the order of a second) and for the
// drain that precedes freeing tensor memory after a wait gave up.
constexpr uint32_t kDefaultWaitProbes = 1u << 16;
// Bounded wait for the phase with the given parity to complete: false when
// `limit` probes pass first (limit 0: give up at once); the caller then
// reports a timeout instead of hanging.
__device__ __forceinline__ bool mbar_wait(uint32_t addr, uint32_t parity, uint32_t limit = kDefaultWaitProbes) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(addr, parity)) return true;
    return false;
}

// One non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint32_t addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(addr), "r"(parity)
        : "memory");
    return ok != 0;
}

// Arrival that also expects `bytes` of asynchronous copies on the barrier's phase.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t addr, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(addr), "r"(bytes) : "memory");
}
// One bulk tensor copy of a 5-D box at the given coordinates into this CTA's
// own shared memory at dst, completing its bytes on the barrier at mbar.
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const void* map, int c0, int c1, int c2, int c3, int c4,
                                            uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, "
        "%6}], [%7];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(mbar)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t addr) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(addr) : "memory");
}
// Named barrier among n threads (a multiple of 32) with an OR-reduction of pred.
__device__ __forceinline__ bool bar_or(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n.reg .pred p, q;\nsetp.ne.u32 q, %1, 0;\nbar.red.or.pred p, %2, %3, q;\nselp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// TMEM loads: the wait is tied to the destination registers so no use of them
// is scheduled before it.
// R consecutive 8-column blocks (R = 1, 2, 4, 8) of 16 lanes: registers 4r .. 4r + 3 hold block r
template <int R>
__device__ __forceinline__ void ld16x256(uint32_t taddr, uint32_t* r) {
    static_assert(R == 1 || R == 2 || R == 4 || R == 8, "repetitions");
    if constexpr (R == 1) {
        asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                     : "r"(taddr));
    } else if constexpr (R == 2) {
        asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                     : "r"(taddr));
    } else if constexpr (R == 4) {
        asm volatile(
            "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(taddr));
    } else {
        ld16x256<4>(taddr, r);
        ld16x256<4>(taddr + 32, r + 16);
    }
}
// Wait for every TMEM load of this thread; the N registers are tied to the
// wait so that no use of them is scheduled before it.
template <int N>
__device__ __forceinline__ void wait_ld(uint32_t* r) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i])::"memory");
}
// Shape 32x32b: thread t of the warp reads / writes TMEM lane (lane base of
// taddr) + t, consecutive 32-bit columns from the column of taddr; register i
// is column i.  Each warp may touch only its own quarter of the 128 lanes.
__device__ __forceinline__ void ld32x32_x32(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void ld32x32_x16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void st32x32_x16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// one 16x16 bf16 A tile (re) and its partner (im) into 16 TMEM columns: the
// A fragment registers (0: rows 0-7 k 0-7, 1: rows 8-15 k 0-7, 2: rows 0-7
// k 8-15, 3: rows 8-15 k 8-15) go to columns so that column c holds
// k = 2 (c / 2) + 8 (c % 2) + {0, 1}; the B images list K in that order.
__device__ __forceinline__ void st_afrag2(uint32_t taddr, const uint32_t (&re)[4], const uint32_t (&im)[4]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x2.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(re[0]),
        "r"(re[2]), "r"(re[1]), "r"(re[3]), "r"(im[0]), "r"(im[2]), "r"(im[1]), "r"(im[3])
        : "memory");
}
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// the input index k held at position kappa of a K = 16 step in TMEM column order
__host__ __device__ constexpr int kperm(int kappa) { return 2 * (kappa / 4) + 8 * ((kappa / 2) % 2) + (kappa % 2); }

}  // namespace um
}  // namespace fftc

// gad_tc.cuh - inline-PTX wrappers for the tcgen05 (5th-generation tensor core)
// verify kernel: mbarriers, named barriers with reductions, tensor-memory
// allocation / loads / stores, MMA issue and commit, shared-memory and
// instruction descriptors.
#pragma once

#include <cstdint>

#include "gad_ptx.cuh"

namespace gad {

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
    return t;
}

// Named barrier over `nthreads` threads that also ORs a predicate across them.
__device__ __forceinline__ bool bar_red_or(int id, int nthreads, bool pred) {
    uint32_t out;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n"
        " selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(out)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
        : "memory");
    return out != 0;
}

// ---- mbarrier (shared::cta) ----
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(bar)
                 : "memory");
}
// True once the phase with parity `parity` has completed.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Non-blocking probe of the same phase.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Limits of the bounded waits.  A pipeline wait gives up after WAIT_LIMIT_NS;
// the last waits of a kernel (for its own tensor-core operations and copies in
// flight, before it frees tensor memory and exits) use TEARDOWN_LIMIT_NS.
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;
constexpr unsigned long long TEARDOWN_LIMIT_NS = 2000000000ull;

// The library built for the tests of the give-up path (and only that build)
// defines GAD_TEST_GIVE_UP_AT_FIRST_MISS: there a pipeline wait whose phase has
// not completed at its first, non-blocking probe gives up at once, so every
// kernel with such a wait takes its give-up path on every run.
#ifdef GAD_TEST_GIVE_UP_AT_FIRST_MISS
constexpr bool kGiveUpAtFirstMiss = true;
#else
constexpr bool kGiveUpAtFirstMiss = false;
#endif

// Wait for phase `parity` of `bar`, giving up after `limit` ns (raising the
// abort flag), or as soon as another thread has raised it if stop_on_abort.
// Returns false on giving up.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             bool stop_on_abort = true,
                                             unsigned long long limit = WAIT_LIMIT_NS) {
    if (kGiveUpAtFirstMiss && limit == WAIT_LIMIT_NS) {
        if (mbar_test_wait(bar, parity)) return true;
        *abort_flag = 1;
        return false;
    }
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (stop_on_abort && *abort_flag) return false;
        if (global_timer_ns() - t0 > limit) {
            *abort_flag = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// ---- tcgen05: tensor memory and the 5th-generation MMA (cta_group::1) ----
// Tensor-memory addresses: lane in bits 31..16, column in bits 15..0.
__device__ __forceinline__ void tc_alloc(uint32_t dst_smem, uint32_t ncols) {  // whole warp
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_relinquish() {  // whole warp
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// Arrive once on `bar` when every tcgen05 operation issued so far by the warp's
// elected lane (the lane tc_mma_ts issues from) is done.  Whole warp.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile(
        "{\n .reg .pred e;\n .reg .b32 rx;\n elect.sync rx|e, 0xffffffff;\n"
        " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(bar)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem descriptor]^T, kind::f16 (fp16 in, fp32 accumulate).
// Called by a whole warp with warp-uniform operands; one elected lane issues.
__device__ __forceinline__ void tc_mma_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p, e;\n .reg .b32 rx;\n elect.sync rx|e, 0xffffffff;\n"
        " setp.ne.b32 p, %4, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5,%5,%5,%5}, p;\n}\n" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u)
        : "memory");
}
// Four MMAs of one K = 64 contraction (K16 steps) from one elected lane:
// D (+)= A(a[k]) * B(b[k])^T for k = 0..3, the first accumulating into D only
// if `accumulate` is nonzero, the other three always.  Whole warp, warp-uniform
// operands.  One election for the four keeps the issuing warp off the
// critical path (an election and predicate per MMA cost as much as the MMA).
__device__ __forceinline__ void tc_mma_ts4(uint32_t d, const uint32_t (&a)[4], const uint64_t (&b)[4],
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p, e, t;\n .reg .b32 rx;\n elect.sync rx|e, 0xffffffff;\n"
        " setp.ne.b32 p, %9, 0;\n setp.eq.b32 t, %10, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %5, %4, {%10,%10,%10,%10}, p;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %6, %4, {%10,%10,%10,%10}, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %7, %4, {%10,%10,%10,%10}, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%11], %8, %4, {%10,%10,%10,%10}, t;\n}\n" ::"r"(d),
        "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(idesc), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]),
        "r"(accumulate), "r"(0u), "r"(a[3])
        : "memory");
}
// Two K = 32 contractions into two accumulators from one elected lane:
// D0 (+)= A(a[0]) B(b[0])^T + A(a[1]) B(b[1])^T and D1 (+)= A(a[2]) B(b[2])^T +
// A(a[3]) B(b[3])^T, each first step accumulating only if `accumulate` is
// nonzero.  Whole warp, warp-uniform operands.
__device__ __forceinline__ void tc_mma_ts2x2(uint32_t d0, uint32_t d1, const uint32_t (&a)[4],
                                             const uint64_t (&b)[4], uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p, e, t;\n .reg .b32 rx;\n elect.sync rx|e, 0xffffffff;\n"
        " setp.ne.b32 p, %10, 0;\n setp.eq.b32 t, %11, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %7, %6, {%11,%11,%11,%11}, p;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %8, %6, {%11,%11,%11,%11}, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%1], [%4], %9, %6, {%11,%11,%11,%11}, p;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%1], [%5], %12, %6, {%11,%11,%11,%11}, t;\n}\n" ::"r"(d0),
        "r"(d1), "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(idesc), "l"(b[0]), "l"(b[1]), "l"(b[2]),
        "r"(accumulate), "r"(0u), "l"(b[3])
        : "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit columns: lane i of the warp gets row (base lane + i).
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tc_st32(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16};\n" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand (8-row x
// 128-byte atoms, 16-byte chunk c of row r stored at c ^ (r & 7)), atoms 1024
// bytes apart along the strided dimension.  Start address must lie in a
// 1024-byte aligned atom; a K offset inside the atom is added to the address.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;            // leading byte offset (unused here)
    d |= static_cast<uint64_t>(1024u >> 4) << 32;    // stride byte offset: next 8-row atom
    d |= static_cast<uint64_t>(1u) << 46;            // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2u) << 61;            // 128-byte swizzle
    return d;
}
// The same for an MN-major operand two 64-element atoms wide along N: the
// second atom (N 64..127) starts `lbo` bytes after the first (the leading
// byte offset of the MN-major swizzled layout; 8-row groups along K stay
// 1024 bytes apart).
__device__ __forceinline__ uint64_t smem_desc_sw128_mn2(uint32_t addr, uint32_t lbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;  // leading byte offset: next N atom
    d |= static_cast<uint64_t>(1024u >> 4) << 32;            // stride byte offset: next 8-row group
    d |= static_cast<uint64_t>(1u) << 46;                    // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2u) << 61;                    // 128-byte swizzle
    return d;
}

// mbarrier arrive that also expects `bytes` of asynchronous (TMA) transactions.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// 2D TMA tile load global -> shared (this CTA only, no multicast), completion
// counted in bytes on `bar`.  x is the inner coordinate in elements.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Four MMAs of a K = 64 contraction with both operands in shared memory:
// D (+)= A(a[k]) * B(b[k])^T for k = 0..3, the first accumulating only if
// `accumulate` is nonzero.  Whole warp, one elected lane issues.
__device__ __forceinline__ void tc_mma_ss4(uint32_t d, const uint64_t (&a)[4], const uint64_t (&b)[4],
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p, e, t;\n .reg .b32 rx;\n elect.sync rx|e, 0xffffffff;\n"
        " setp.ne.b32 p, %10, 0;\n setp.eq.b32 t, %11, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %5, %9, {%11,%11,%11,%11}, p;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %9, {%11,%11,%11,%11}, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %9, {%11,%11,%11,%11}, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %9, {%11,%11,%11,%11}, t;\n}\n" ::"r"(d),
        "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]),
        "r"(idesc), "r"(accumulate), "r"(0u)
        : "memory");
}

// Instruction descriptor, kind::f16: fp16 A and B, fp32 D, A K-major,
// B K-major (b_mn = 0) or MN-major (b_mn = 1), shape M x N.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, int b_mn) {
    return (1u << 4) | (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}
// The same with bf16 A and B (A and B format fields = 1).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int b_mn) {
    return idesc_f16_f32(M, N, b_mn) | (1u << 7) | (1u << 10);
}

}  // namespace gad

// Blackwell (sm_100a) primitives used by the tensor-core attention kernels:
// mbarriers with bounded waits, TMA tile loads, tcgen05 MMA / TMEM access,
// and shared-memory matrix descriptors for the 128-byte swizzled layout.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace nabla {
namespace sm100 {

// ---- mbarrier -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
    return t;
}

// Bounded wait for the phase of parity `parity` to complete.  Gives up when
// another thread of the CTA has aborted (abort flag set) or after `limit_ns`
// nanoseconds of waiting, in which case it sets the abort flag and the status
// word.  Returns false when it gave up.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort,
                                         int *status, uint32_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t n = 0;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if ((n & 63) == 63) {
            if (global_ns() - t0 > limit_ns) {
                *abort = 1;
                atomicExch(status, kDevTimeout);
                return false;
            }
            if (n > 4096) __nanosleep(64);  // long waits only
        }
    }
}


// ---- TMA --------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint64_t *bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4}], [%2];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- tcgen05 ------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_addr(dst_smem)),
                 "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols));
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// *_warp: MMA issue is warp-collective: the whole warp executes the call,
// converged, and one elected lane issues the instruction (calling one from a
// single lane deadlocks the warp).  Keeping the issuing code
// convergent lets the descriptors live in uniform registers; issuing from a
// single divergent lane costs more than an N = 64 MMA takes to execute.
//
// D[tmem] (+)= A[smem] * B[smem], kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_ss_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred e, p;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// D[tmem] (+)= A[tmem] * B[smem], kind::f16; A is M x K, K-major, 16-bit
// elements packed two per 32-bit column (a K = 16 step spans 8 columns).
__device__ __forceinline__ void mma_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred e, p;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// Four MMAs behind one elect.sync (warp-collective like the above): MMA i is
// D_i (+)= A_i * B_i.  MMAs 0 and 1 accumulate when acc0 / acc1 is nonzero,
// MMAs 2 and 3 always accumulate.  The tensor core accepts an MMA roughly when
// it starts executing it, so the issuing warp spends about an N = 64 MMA's
// execution time per issue; fewer instructions per MMA keep the issue loop
// from falling behind the pipe.
__device__ __forceinline__ void mma_ss4_warp(uint32_t d0, uint32_t d1, uint32_t d2, uint32_t d3,
                                             uint64_t a0, uint64_t a1, uint64_t a2, uint64_t a3,
                                             uint64_t b0, uint64_t b1, uint64_t b2, uint64_t b3,
                                             uint32_t idesc, uint32_t acc0, uint32_t acc1) {
    asm volatile(
        "{\n .reg .pred e, p0, p1, pt;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p0, %13, 0;\n"
        " setp.ne.b32 p1, %14, 0;\n setp.ne.b32 pt, %12, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %12, p0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%1], %5, %9, %12, p1;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%2], %6, %10, %12, pt;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%3], %7, %11, %12, pt;\n}\n" ::"r"(d0),
        "r"(d1), "r"(d2), "r"(d3), "l"(a0), "l"(a1), "l"(a2), "l"(a3), "l"(b0), "l"(b1), "l"(b2),
        "l"(b3), "r"(idesc), "r"(acc0), "r"(acc1));
}
// As mma_ss4_warp with the A operands in TMEM (column addresses a0..a3).
__device__ __forceinline__ void mma_ts4_warp(uint32_t d0, uint32_t d1, uint32_t d2, uint32_t d3,
                                             uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint64_t b0, uint64_t b1, uint64_t b2, uint64_t b3,
                                             uint32_t idesc, uint32_t acc0, uint32_t acc1) {
    asm volatile(
        "{\n .reg .pred e, p0, p1, pt;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p0, %13, 0;\n"
        " setp.ne.b32 p1, %14, 0;\n setp.ne.b32 pt, %12, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %8, %12, p0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%1], [%5], %9, %12, p1;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%2], [%6], %10, %12, pt;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%3], [%7], %11, %12, pt;\n}\n" ::"r"(d0),
        "r"(d1), "r"(d2), "r"(d3), "r"(a0), "r"(a1), "r"(a2), "r"(a3), "l"(b0), "l"(b1), "l"(b2),
        "l"(b3), "r"(idesc), "r"(acc0), "r"(acc1));
}
// As mma_ss4_warp with MMAs 0 and 2 taking their A operand from TMEM (a0, a2
// column addresses) and MMAs 1 and 3 from shared memory (a1, a3 descriptors).
__device__ __forceinline__ void mma_tsss4_warp(uint32_t d0, uint32_t d1, uint32_t d2, uint32_t d3,
                                               uint32_t a0, uint64_t a1, uint32_t a2, uint64_t a3,
                                               uint64_t b0, uint64_t b1, uint64_t b2, uint64_t b3,
                                               uint32_t idesc, uint32_t acc0, uint32_t acc1) {
    asm volatile(
        "{\n .reg .pred e, p0, p1, pt;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p0, %13, 0;\n"
        " setp.ne.b32 p1, %14, 0;\n setp.ne.b32 pt, %12, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %8, %12, p0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%1], %5, %9, %12, p1;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%2], [%6], %10, %12, pt;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%3], %7, %11, %12, pt;\n}\n" ::"r"(d0),
        "r"(d1), "r"(d2), "r"(d3), "r"(a0), "l"(a1), "r"(a2), "l"(a3), "l"(b0), "l"(b1), "l"(b2),
        "l"(b3), "r"(idesc), "r"(acc0), "r"(acc1));
}
// Single-thread forms, for an issuer whose MMAs are N = 128 or wider (then
// the issue cost is hidden behind execution and the warp's other lanes stay
// out of the issuing path).
__device__ __forceinline__ void mma_ts_1(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_ss_1(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit_1(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
            smem_addr(bar))
        : "memory");
}
// Arrive on `bar` once all previously issued tcgen05 ops of the issuing
// thread are done (warp-collective, one elected lane commits).
__device__ __forceinline__ void mma_commit_warp(uint64_t *bar) {
    asm volatile(
        "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
        " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(
            smem_addr(bar))
        : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane
// (warp_in_group * 32 + i), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    uint32_t *r = reinterpret_cast<uint32_t *>(v);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float *v) {
    const uint32_t *r = reinterpret_cast<const uint32_t *>(v);
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31]));
}
// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16};\n" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]));
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}
// Generic-proxy shared-memory writes -> visible to the tensor core.
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (1024-byte atoms of
// 8 rows x 128 bytes).  K-major operand: rows 128 B apart, 8-row groups
// `sbo` apart, `lbo` unused (16).  MN-major operand: 64 contiguous MN
// elements per 128-byte row, rows along K, 8-row groups `sbo` apart, next
// 64 MN elements `lbo` apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm_100
    d |= static_cast<uint64_t>(2) << 61;  // 128-byte swizzle
    return d;
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> fp32, M x N, operand
// majors (0 = K-major, 1 = MN-major).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4)                                    // D format: f32
           | (1u << 7)                                  // A format: bf16
           | (1u << 10)                                 // B format: bf16
           | (static_cast<uint32_t>(a_mn_major) << 15)  // A major
           | (static_cast<uint32_t>(b_mn_major) << 16)  // B major
           | (static_cast<uint32_t>(N >> 3) << 17)      // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);     // M / 16
}

// bar.sync on a named barrier among `count` threads, OR-reducing a predicate.
__device__ __forceinline__ bool bar_or(int id, int count, bool pred) {
    uint32_t out;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n"
        " selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(out)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(count)
        : "memory");
    return out != 0;
}
__device__ __forceinline__ void bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(count) : "memory");
}

// Ascending enumeration of the set bits of (ra | rb) over `words` 32-bit
// words, by one full warp: list[k] = bit index, flags[k] = bit 0 from ra,
// bit 1 from rb.  rb may be null.  Returns the number of entries (all lanes).
__device__ __forceinline__ int union_bits(const uint32_t *ra, const uint32_t *rb, int words,
                                          uint16_t *list, uint8_t *flags, int lane) {
    int U = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
        const int w = w0 + lane;
        uint32_t a = 0, b = 0;
        if (w < words) {
            a = ra[w];
            if (rb) b = rb[w];
        }
        uint32_t u = a | b;
        const int cnt = __popc(u);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        int pos = U + incl - cnt;
        while (u) {
            const int bit = __ffs(u) - 1;
            u &= u - 1;
            list[pos] = static_cast<uint16_t>(w * 32 + bit);
            flags[pos] = static_cast<uint8_t>(((a >> bit) & 1u) | (((b >> bit) & 1u) << 1));
            ++pos;
        }
        U += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
    return U;
}

// 1-D bulk copy global -> shared (size multiple of 16, both 16-byte aligned).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// wait_bar for a converged warp.  Every lane tests the barrier and the warp
// votes, so no lane leaves the others: a completed phase costs ~30 cycles this
// way, against ~180 for a test by lane 0 alone followed by a shuffle of its
// answer.  Otherwise every lane runs the bounded wait and the warp returns
// true only if all lanes saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          int *status, uint32_t limit_ns) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    const bool ok = wait_bar(bar, parity, abort, status, limit_ns);
    return __all_sync(0xffffffffu, ok);
}

// Bounded wait that ignores the abort flag (used to drain in-flight work).
__device__ __forceinline__ bool wait_plain(uint64_t *bar, uint32_t parity, uint32_t limit_ns) {
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > limit_ns) return false;
        __nanosleep(128);
    }
    return true;
}

}  // namespace sm100
}  // namespace nabla

// Host: TMA map over a [rows, D] bf16 row-major tensor (D = 64 or 128), boxes
// of 64 rows x 64 features, 128-byte swizzle (defined in attn_fwd_sm100.cu).
bool nabla_make_tmap_rows(CUtensorMap *m, const void *base, uint64_t rows, int D);

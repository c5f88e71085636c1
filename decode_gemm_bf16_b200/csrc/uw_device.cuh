// uw_device.cuh -- small device helpers shared by the kernels of libunweight:
// byte permutes for the palette lookup and the BF16 merge, and the inline PTX
// wrappers for mbarriers, TMA and the 5th-generation tensor cores (tcgen05).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace uw {

// Device status word, one per translation unit (the library is built without
// relocatable device code); the first error wins.  uw_last_device_status
// collects the words of all units.
static __device__ int g_status;

__device__ __forceinline__ void raise_status(int code) { atomicCAS(&g_status, 0, code); }

// Host side: read this unit's status word and reset it to 0.
static inline int unit_status_take() {
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return -1;
    if (v != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return -1;
    return v;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Four 4-bit palette indices (low 16 bits of x, index i in bits 4i..4i+3) ->
// four exponent bytes.  The palette is held in four registers (P0 = entries
// 0..3, ..., P3 = entries 12..15).  prmt selects a byte out of eight by the
// low 3 bits of each selector nibble; the nibble's bit 3 chooses between the
// lower and the upper eight entries through a byte mask.
__device__ __forceinline__ uint32_t palette4(uint32_t x, uint32_t P0, uint32_t P1, uint32_t P2,
                                             uint32_t P3) {
    uint32_t lo = prmt(P0, P1, x);               // right where the index is < 8
    uint32_t hi = prmt(P2, P3, x ^ 0x8888u);     // right where the index is >= 8
    uint32_t t = x & 0x8888u;
    uint32_t m = prmt(0u, 0x80u, t | (t >> 1));  // 0xFF per byte where the index is >= 8
    return (lo & ~m) | (hi & m);
}

// Same lookup when all 16 palette exponents are below 128 (|w| < 2): the
// out-of-range half of each prmt then yields 0x00 by sign replication, so
// the two halves combine with an OR.  xs = x ^ 0x8888 (shared per word).
__device__ __forceinline__ uint32_t palette4_small(uint32_t x, uint32_t xs, uint32_t P0, uint32_t P1,
                                                   uint32_t P2, uint32_t P3) {
    return prmt(P0, P1, x) | prmt(P2, P3, xs);
}

// Four exponent bytes E and four sign+mantissa bytes S -> four BF16 values
// (two words): bf16 = (s<<15) | (e<<7) | m with S = s<<7 | m.
__device__ __forceinline__ uint2 merge4(uint32_t E, uint32_t S) {
    uint32_t hi = (S & 0x80808080u) | ((E >> 1) & 0x7F7F7F7Fu);   // sign | e[7:1]
    uint32_t lo = ((E << 7) & 0x80808080u) | (S & 0x7F7F7F7Fu);   // e[0] | mantissa
    return make_uint2(prmt(lo, hi, 0x5140u), prmt(lo, hi, 0x7362u));
}

// One lane of a converged warp (the others get false).
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "elect.sync _|P, 0xffffffff;\n\t"
        "selp.b32 %0, 1, 0, P;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Shared-memory loads by 32-bit shared-window address: explicit ld.shared,
// where a pointer derived through integer arithmetic would compile to a
// generic load.
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// ---------------------------------------------------------------- tagged counters
// A 64-bit counter word holds (tag << 16) | count, tag = 48-bit id of one
// call.  A word carrying another tag (or stale bytes) counts as 0, so
// counters living in caller workspace never need clearing.
__device__ __forceinline__ unsigned arrive_counter(unsigned long long* cnt, unsigned long long tag) {
    unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(cnt);
    for (;;) {
        const unsigned long long base = (cur >> 16) == tag ? cur : (tag << 16);
        const unsigned long long nxt = base + 1;
        const unsigned long long prev = atomicCAS(cnt, cur, nxt);
        if (prev == cur) return (unsigned)(nxt & 0xFFFFu);
        cur = prev;
    }
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
// Bounded wait until *p == tag (a row published by another CTA of this call).
__device__ __forceinline__ bool wait_tag(const unsigned long long* p, unsigned long long tag, uint64_t timeout_ns,
                                         volatile int* abort);
// Bounded wait until the counter shows `want` arrivals of call `tag`.
__device__ __forceinline__ bool wait_counter(const unsigned long long* cnt, unsigned long long tag, unsigned want,
                                             uint64_t timeout_ns, volatile int* abort);

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Test for completion of the phase with the given parity; a thread whose
// phase is not complete may be suspended for up to `hint_ns` (it wakes as soon
// as the phase completes), so waiting roles do not steal issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait: returns false once `timeout_ns` has passed since the wait
// started (the deadline is only read after the first polls, so short waits
// stay cheap) or when another role of the CTA raised *abort (if given).  On
// expiry *abort is raised.  Never spins forever.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                          volatile int* abort, uint32_t hint_ns = 1000) {
    uint64_t deadline = 0;
    for (uint32_t i = 0;; i++) {
        if (mbar_try_wait(bar, parity, hint_ns)) return true;
        if ((i & 7u) == 7u) {
            if (abort && *abort) return false;
            uint64_t now = globaltimer();
            if (deadline == 0) {
                deadline = now + timeout_ns;
            } else if (now > deadline) {
                if (abort) *abort = 1;
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool wait_counter(const unsigned long long* cnt, unsigned long long tag, unsigned want,
                                             uint64_t timeout_ns, volatile int* abort) {
    uint64_t deadline = 0;
    for (uint32_t i = 0;; i++) {
        const unsigned long long v = ld_acquire_u64(cnt);
        if ((v >> 16) == tag && (unsigned)(v & 0xFFFFu) >= want) return true;
        if (abort && *abort) return false;
        const uint64_t now = globaltimer();
        if (deadline == 0) {
            deadline = now + timeout_ns;
        } else if (now > deadline) {
            if (abort) *abort = 1;
            return false;
        }
        __nanosleep(200);
    }
}

__device__ __forceinline__ bool wait_tag(const unsigned long long* p, unsigned long long tag, uint64_t timeout_ns,
                                         volatile int* abort) {
    uint64_t deadline = 0;
    for (;;) {
        if (ld_acquire_u64(p) == tag) return true;
        if (abort && *abort) return false;
        const uint64_t now = globaltimer();
        if (deadline == 0) {
            deadline = now + timeout_ns;
        } else if (now > deadline) {
            if (abort) *abort = 1;
            return false;
        }
        __nanosleep(100);
    }
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Generic-proxy writes observed (acquire) -> visible to TMA (async proxy) reads.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
// Untiled bulk copy (TMA engine) of `bytes` from global memory into this
// CTA's shared memory, completing on mbarrier `bar`.  Both addresses 16-byte
// aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
// Barrier among the `nthreads` threads (whole warps) that use barrier `id`.
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void sts16(uint32_t addr, uint16_t v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (BF16 in, FP32 accumulate).
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16: A read from tensor memory
// (row i of A in TMEM lane i, K elements 2j, 2j+1 in column j, low half first).
__device__ __forceinline__ void tc_mma_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// 32 TMEM lanes x 16 consecutive 32-bit columns <- 16 registers per thread.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05 op issued so far by this thread is done.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
// 32 TMEM lanes x 16 consecutive 32-bit columns -> 16 registers per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 16-byte asynchronous global -> shared copies (L2 only), in commit groups.
__device__ __forceinline__ void cp_async16(uint32_t dst_smem, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst_smem), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Shared-memory matrix descriptor for a K-major operand in the 128-byte
// swizzled canonical layout: rows of 128 bytes (64 BF16), 8-row atoms of
// 1024 bytes, atoms stacked every 1024 bytes (stride byte offset).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);       // start address
    d |= (uint64_t)1u << 16;                             // leading byte offset (unused here)
    d |= (uint64_t)(1024u >> 4) << 32;                   // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1u << 46;                             // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                             // 128-byte swizzle
    return d;
}

// Instruction descriptor, kind::f16: D fp32, A and B BF16, both K-major,
// shape M x N (M = 128 here).
__host__ __device__ constexpr uint32_t mma_idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

}  // namespace uw

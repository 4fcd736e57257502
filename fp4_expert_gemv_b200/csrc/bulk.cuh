// mbarrier and bulk-copy (cp.async.bulk) wrappers, bounded waits, phase
// stamps: shared by the single-launch decode kernel and its helpers.
#pragma once

#include "common.cuh"

namespace fe {

FE_DEV uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

FE_DEV void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// One arrival (release, CTA scope) on a barrier.
FE_DEV void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

FE_DEV void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Whether phase `parity` of the barrier has completed.  test_wait returns at
// once: a thread suspended in try_wait was seen to sleep for microseconds past
// the completion of the copies it waited for.
FE_DEV bool mbar_test(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase 0 of a one-shot barrier, at most timeout_ns; false on timeout.
FE_DEV bool mbar_wait0(uint32_t bar, unsigned long long timeout_ns)
{
    if (mbar_test(bar, 0)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (int it = 1;; ++it) {
        if (mbar_test(bar, 0)) return true;
        if ((it & 15) == 0 && globaltimer_ns() - t0 > timeout_ns) return false;
    }
}

// Wait for the completion of phase `parity` of a barrier that is reused, at
// most timeout_ns; false on timeout.
FE_DEV bool mbar_wait(uint32_t bar, uint32_t parity, unsigned long long timeout_ns)
{
    if (mbar_test(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (int it = 1;; ++it) {
        if (mbar_test(bar, parity)) return true;
        if ((it & 15) == 0 && globaltimer_ns() - t0 > timeout_ns) return false;
    }
}

// 16 bytes global -> shared by this thread, cached in L2 only (never a stale L1
// line of data another SM wrote); complete after cp_async_wait_all.
FE_DEV void cp_async16_cg(uint32_t dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

FE_DEV void cp_async_wait_all()
{
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

FE_DEV void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// Phase stamp i of the optional trace: %globaltimer and the SM's cycle counter.
FE_DEV void stamp(unsigned long long* trace, int i)
{
    asm volatile("" ::: "memory");
    trace[i] = globaltimer_ns();
    trace[32 + i] = (unsigned long long)clock64();
    asm volatile("" ::: "memory");
}

FE_DEV void st_relaxed_u64(unsigned long long* p, unsigned long long v)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Two 64-bit words to a 16-byte aligned address.
FE_DEV void st_relaxed_u64x2(unsigned long long* p, unsigned long long a, unsigned long long b)
{
    asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(a), "l"(b) : "memory");
}

FE_DEV unsigned long long ld_relaxed_u64(const unsigned long long* p)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

FE_DEV ulonglong2 ld_relaxed_u64x2(const unsigned long long* p)
{
    ulonglong2 v;
    asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(v.x), "=l"(v.y) : "l"(p) : "memory");
    return v;
}

FE_DEV void arrive_relaxed(unsigned long long* counter)
{
    asm volatile("red.relaxed.gpu.global.add.u64 [%0], 1;" ::"l"(counter) : "memory");
}

// Arrival counter of a launch's CTAs: every CTA's writes before its arrival
// (ordered by a gpu-scope fence and a CTA barrier) are visible to a CTA that
// observes the count with an acquire load.
FE_DEV void arrive_release(unsigned long long* counter)
{
    asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(counter) : "memory");
}

FE_DEV unsigned long long ld_acquire_u64(const unsigned long long* p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// The 128-byte line holding p into L2 (a hint; no L1 fill).
FE_DEV void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// Bring [src, src + bytes) from memory into L2 (a hint: no completion, no
// destination); src 16-byte aligned, bytes a multiple of 16.
FE_DEV void bulk_prefetch_l2(const void* src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

}  // namespace fe

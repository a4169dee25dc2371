// Thin inline-PTX wrappers for the sm_100a features the tensor-core kernels
// use: mbarriers, TMA tensor loads, tcgen05 (TMEM allocation, UMMA issue,
// commit, TMEM loads/stores and their fences).  Each wrapper is one PTX
// instruction (or a bounded wait built from one).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace arl2 {
namespace ptx {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- mbarrier -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase of `bar` with the given parity to complete.  Gives up
// after `limit_ns` of wall time, or as soon as *abort is nonzero, and then
// returns false.  Every wait in the tensor-core kernels goes through here.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  const volatile int* abort, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// Warp-uniform bounded wait: every lane of a converged warp calls it with
// the same arguments and gets the same answer.  The fast path is one
// try_wait per lane and one vote, with no divergent branch (a per-lane wait
// loop followed by a vote costs a reconvergence on every call).
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, const volatile int* abort,
                                               uint64_t limit_ns) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
        if (__any_sync(0xffffffffu, *abort != 0 || globaltimer_ns() - t0 > limit_ns)) return false;
    }
}

// ---- proxies and fences ---------------------------------------------------
// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---- TMA ------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
// 4-D tiled load into this CTA's shared memory, completing tx bytes on bar.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* m, int c0, int c1,
                                            int c2, int c3, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
        : "memory");
}

// 4-D tiled store from this CTA's shared memory (bulk async-group).  Rows
// outside the tensor are not written.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* m, uint32_t src, int c0, int c1,
                                             int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(m)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until every committed bulk store has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// ---- tcgen05: TMEM allocation ---------------------------------------------
// Whole warp.  Writes the allocated TMEM base address to shared memory.
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

// ---- tcgen05: MMA ---------------------------------------------------------
// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 inputs here),
// fp32 accumulate.  accumulate == 0 overwrites D.
__device__ __forceinline__ void umma_f16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]: A (M = 128 rows = TMEM lanes, K
// packed two bf16 per 32-bit column, 8 columns per 16-wide k-step).
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on bar when every tcgen05 op this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

// ---- warp-wide issue: one elected lane, all lanes converged ----------------
// The whole warp executes these with identical (warp-uniform) operands and
// exactly one lane issues.  Keeping the issuing code warp-uniform lets the
// compiler hold descriptors in uniform registers, which sustains the
// tensor-core issue rate (a single-lane branch does not).
__device__ __forceinline__ void umma_f16_ss_w(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_f16_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_commit_w(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx_w(uint32_t bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(bar),
        "r"(bytes)
        : "memory");
}
__device__ __forceinline__ void tma_load_4d_w(uint32_t dst, const CUtensorMap* m, int c0, int c1,
                                              int c2, int c3, uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];\n\t}" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
        : "memory");
}

// L2 prefetch of a TMA tile (a hint: no shared memory is written and no
// completion is tracked).
__device__ __forceinline__ void tma_prefetch_l2_4d(const CUtensorMap* m, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}

// ---- tcgen05: TMEM <-> registers (32 lanes x 32 columns of 32 bit) --------
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Ties 32 registers to this point of the program: uses of a tcgen05.ld
// destination cannot be scheduled above the tcgen05.wait::ld before it.
__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                   "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])::"memory");
}
__device__ __forceinline__ void reg_fence16(uint32_t (&r)[16]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])::"memory");
}
__device__ __forceinline__ void tmem_st32_u(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---- programmatic dependent launch -----------------------------------------
// pdl_trigger: this CTA allows the next kernel in the stream to be launched
// (it starts once every CTA of this grid has triggered or exited).
// pdl_wait: block until the previous kernel in the stream has completed and
// its memory operations are visible; returns at once without such a kernel.
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Wait for the previous kernel, then let the next one launch.  A kernel that
// triggers only after its wait never has a dependent running beside anything
// older than itself: a dependent that reads its own inputs before its wait
// (inputs no kernel of this chain writes) then sees them complete.
__device__ __forceinline__ void pdl_wait_then_trigger() {
    pdl_wait();
    pdl_trigger();
}

// ---- register reallocation between warpgroups ------------------------------
// Every warp of a warpgroup executes the same one.  The increases of a CTA
// draw on the registers it was launched with (threads x registers per
// thread at launch): the host checks that the split adds up before launch.
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---- named barriers and global flags --------------------------------------
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---- thread-block clusters -------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Every thread of every CTA of the cluster; shared-memory writes before it
// are visible to the cluster's reads after it.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
__device__ __forceinline__ uint32_t mapa_shared(uint32_t a, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
__device__ __forceinline__ float4 ld_shared_cluster_v4(uint32_t a) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(a)
                 : "memory");
    return v;
}

// ---- math -----------------------------------------------------------------
// ---- packed fp32 pairs (sm_100 f32x2 arithmetic: one instruction, two lanes of data)
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
// 2^x with the SFU's approximate exponential (PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- UMMA operand descriptors ---------------------------------------------
// Shared-memory matrix descriptor (sm_100): start address >> 4 in bits 0-13,
// leading byte offset >> 4 in 16-29, stride byte offset >> 4 in 32-45,
// descriptor version 1 in bits 46-47, swizzle mode in bits 61-63
// (2 = 128-byte swizzle).  The swizzle pattern is anchored to 1024-byte
// aligned shared addresses, so every operand tile starts on such a boundary.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor for kind::f16 with bf16 A and B, fp32 D.
// a_mn / b_mn select an MN-major (instead of K-major) operand.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4)                      // D format fp32
           | (1u << 7)                    // A format bf16
           | (1u << 10)                   // B format bf16
           | ((a_mn ? 1u : 0u) << 15)     // A major
           | ((b_mn ? 1u : 0u) << 16)     // B major
           | ((uint32_t)(N >> 3) << 17)   // N / 8
           | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// Operand tiles of 128 rows x 128 bf16, stored as two 128-row x 64-column
// halves of 16 KB with the 128-byte swizzle (the layout TMA writes for a
// {64, ..., 128} box).
constexpr uint32_t kTileBytes = 128 * 128 * 2;
constexpr uint32_t kHalfBytes = kTileBytes / 2;

// K-major operand (row = M or N index, 128 K values along the row): the
// descriptor of k-step kk (16 K values) starts kk*32 bytes into its half.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int kk) {
    return sdesc_sw128(tile + (uint32_t)(kk >> 2) * kHalfBytes + (uint32_t)(kk & 3) * 32u, 16u,
                       1024u);
}
// MN-major operand (row = K index, 128 M/N values along the row in two
// 64-wide halves 16 KB apart): k-step kk starts 16 rows = 2048 bytes on.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile, int kk) {
    return sdesc_sw128(tile + (uint32_t)kk * 2048u, kHalfBytes, 1024u);
}

// ---- eight k-steps of a 128x128x128 product in one issue sequence ---------
// One elected lane issues all eight MMAs of a 128-deep product.  The
// descriptors of k-step kk differ from those of step 0 only in the
// start-address field (bits 0-13 of the low word, address >> 4), and
// shared-memory addresses stay below 2^18 so that the field never carries:
// the steps are plain 32-bit adds on the low word.
//   K-major SW128 operand: + ((kk >> 2) * 16 KB + (kk & 3) * 32 B) >> 4
//   MN-major SW128 operand: + (kk * 2048 B) >> 4
// acc0 is the accumulate flag of the first step (the others accumulate).
__device__ __forceinline__ void umma_ss8_kk(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc,
                                            uint32_t acc0) {
    const uint32_t alo = (uint32_t)a0, ahi = (uint32_t)(a0 >> 32);
    const uint32_t blo = (uint32_t)b0, bhi = (uint32_t)(b0 >> 32);
    asm volatile(
        "{\n\t.reg .pred e, p, one;\n\t.reg .b64 a, b;\n\t.reg .b32 x, y;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "setp.eq.b32 one, %6, %6;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "mov.b64 a, {%1, %2};\n\tmov.b64 b, {%3, %4};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, p;\n\t"
        "add.u32 x, %1, 2;\n\tadd.u32 y, %3, 2;\n\tmov.b64 a, {x, %2};\n\tmov.b64 b, {y, %4};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, one;\n\t"
        "add.u32 x, %1, 4;\n\tadd.u32 y, %3, 4;\n\tmov.b64 a, {x, %2};\n\tmov.b64 b, {y, %4};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, one;\n\t"
        "add.u32 x, %1, 6;\n\tadd.u32 y, %3, 6;\n\tmov.b64 a, {x, %2};\n\tmov.b64 b, {y, %4};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, one;\n\t"
        "add.u32 x, %1, 1024;\n\tadd.u32 y, %3, 1024;\n\tmov.b64 a, {x, %2};\n\tmov.b64 b, {y, %4};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, one;\n\t"
        "add.u32 x, %1, 1026;\n\tadd.u32 y, %3, 1026;\n\tmov.b64 a, {x, %2};\n\tmov.b64 b, {y, %4};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, one;\n\t"
        "add.u32 x, %1, 1028;\n\tadd.u32 y, %3, 1028;\n\tmov.b64 a, {x, %2};\n\tmov.b64 b, {y, %4};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, one;\n\t"
        "add.u32 x, %1, 1030;\n\tadd.u32 y, %3, 1030;\n\tmov.b64 a, {x, %2};\n\tmov.b64 b, {y, %4};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, one;\n\t}" ::"r"(d_tmem),
        "r"(alo), "r"(ahi), "r"(blo), "r"(bhi), "r"(idesc), "r"(acc0)
        : "memory");
}
// A from TMEM (a_tmem, 8 columns of bf16 pairs per k-step), B MN-major:
// four k-steps (64 deep), for a product issued in two halves.
__device__ __forceinline__ void umma_ts4_mn(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0, uint32_t idesc,
                                            uint32_t acc0) {
    const uint32_t blo = (uint32_t)b0, bhi = (uint32_t)(b0 >> 32);
    asm volatile(
        "{\n\t.reg .pred e, p, one;\n\t.reg .b64 b;\n\t.reg .b32 t, y;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "setp.eq.b32 one, %5, %5;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "mov.b64 b, {%2, %3};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b, %4, p;\n\t"
        "add.u32 t, %1, 8;\n\tadd.u32 y, %2, 128;\n\tmov.b64 b, {y, %3};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, one;\n\t"
        "add.u32 t, %1, 16;\n\tadd.u32 y, %2, 256;\n\tmov.b64 b, {y, %3};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, one;\n\t"
        "add.u32 t, %1, 24;\n\tadd.u32 y, %2, 384;\n\tmov.b64 b, {y, %3};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, one;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "r"(blo), "r"(bhi), "r"(idesc), "r"(acc0)
        : "memory");
}
// A from TMEM (a_tmem, 8 columns of bf16 pairs per k-step), B MN-major.
__device__ __forceinline__ void umma_ts8_mn(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0, uint32_t idesc,
                                            uint32_t acc0) {
    const uint32_t blo = (uint32_t)b0, bhi = (uint32_t)(b0 >> 32);
    asm volatile(
        "{\n\t.reg .pred e, p, one;\n\t.reg .b64 b;\n\t.reg .b32 t, y;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "setp.eq.b32 one, %5, %5;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "mov.b64 b, {%2, %3};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b, %4, p;\n\t"
        "add.u32 t, %1, 8;\n\tadd.u32 y, %2, 128;\n\tmov.b64 b, {y, %3};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, one;\n\t"
        "add.u32 t, %1, 16;\n\tadd.u32 y, %2, 256;\n\tmov.b64 b, {y, %3};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, one;\n\t"
        "add.u32 t, %1, 24;\n\tadd.u32 y, %2, 384;\n\tmov.b64 b, {y, %3};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, one;\n\t"
        "add.u32 t, %1, 32;\n\tadd.u32 y, %2, 512;\n\tmov.b64 b, {y, %3};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, one;\n\t"
        "add.u32 t, %1, 40;\n\tadd.u32 y, %2, 640;\n\tmov.b64 b, {y, %3};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, one;\n\t"
        "add.u32 t, %1, 48;\n\tadd.u32 y, %2, 768;\n\tmov.b64 b, {y, %3};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, one;\n\t"
        "add.u32 t, %1, 56;\n\tadd.u32 y, %2, 896;\n\tmov.b64 b, {y, %3};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, one;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "r"(blo), "r"(bhi), "r"(idesc), "r"(acc0)
        : "memory");
}

// Byte offset of the 16-byte chunk c16 (0..15 along a 128-element bf16
// row) of row r inside such a tile.
__device__ __forceinline__ uint32_t tile_chunk_offset(int r, int c16) {
    return (uint32_t)(c16 >> 3) * kHalfBytes + (uint32_t)r * 128u +
           (uint32_t)(((c16 & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

}  // namespace ptx
}  // namespace arl2

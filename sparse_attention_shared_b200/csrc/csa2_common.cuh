// Device helpers shared by the CSA2 kernels: status reporting, bounded waits,
// mbarriers, bulk copies and the tcgen05 (5th-generation tensor core) wrappers.
// Every wait here is bounded: a wait on an mbarrier (a copy or an MMA of the
// CTA itself) gives up after kSpinBudgetCycles SM cycles; a wait on other CTAs
// (the indexer's group barrier) after a run-time budget that defaults to the
// same and can be shortened by csa2_set_wait_controls. Either records
// CSA2_ERR_TIMEOUT in the status word and lets the caller return.
#pragma once

#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/csa2.h"

namespace csa2 {

// About 2 s at the B200's 1.9 GHz boost clock; longer under a power cap.
constexpr long long kSpinBudgetCycles = 4000000000LL;

__device__ __forceinline__ void report(int32_t* st, int code, int detail) {
    if (st != nullptr) {
        if (atomicCAS(st, 0, code) == 0) atomicExch(st + 1, detail);
    }
}

// Phase-trace build (compiled with -DCSA2_PHASE_TRACE, library libcsa2_trace.so): the
// indexer and attention kernels record, per CTA, the SM clock at numbered phase
// boundaries (CSA2_TRACE) and, per launch, every CTA's start and end on the global
// timer (CSA2_TRACE_END), into buffers the host registers with the csa2_trace_set_*
// entry points of that library. Every record is bounded by the buffer sizes given
// there. In the normal build the macros are empty.
#ifdef CSA2_PHASE_TRACE
static __device__ unsigned long long* g_trace_buf = nullptr;   // [ctas][32]: slot 31 start time, 30 start clock
static __device__ unsigned int g_trace_ncta = 0;               // rows of g_trace_buf
static __device__ int g_trace_on = 0;                          // phase slots on
static __device__ unsigned long long* g_tl_buf = nullptr;      // [cap][4]: kernel kind, CTA, start ns, end ns
static __device__ unsigned int* g_tl_ctr = nullptr;            // records taken (may pass cap)
static __device__ unsigned int g_tl_cap = 0;
__device__ __forceinline__ unsigned long long trace_gtimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ unsigned trace_cta() { return (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x; }
__device__ __forceinline__ bool trace_slot_ok() {
    return threadIdx.x == 0 && g_trace_on && g_trace_buf != nullptr && trace_cta() < g_trace_ncta;
}
#define CSA2_TRACE_INIT()                                                                         \
    const unsigned long long csa2_trace_t0 = ::csa2::trace_gtimer();                            \
    if (::csa2::trace_slot_ok()) {                                                              \
        ::csa2::g_trace_buf[(size_t)::csa2::trace_cta() * 32 + 31] = csa2_trace_t0;              \
        ::csa2::g_trace_buf[(size_t)::csa2::trace_cta() * 32 + 30] = (unsigned long long)clock64(); \
    }
#define CSA2_TRACE(slot)                                                                          \
    if (::csa2::trace_slot_ok())                                                                  \
        ::csa2::g_trace_buf[(size_t)::csa2::trace_cta() * 32 + (slot)] =                          \
            (unsigned long long)clock64() - ::csa2::g_trace_buf[(size_t)::csa2::trace_cta() * 32 + 30];
#define CSA2_TRACE_VAL(slot, v)                                                                   \
    if (::csa2::trace_slot_ok()) ::csa2::g_trace_buf[(size_t)::csa2::trace_cta() * 32 + (slot)] = (unsigned long long)(v);
#define CSA2_TRACE_END(kind)                                                                      \
    if (threadIdx.x == 0 && ::csa2::g_tl_buf != nullptr) {                                        \
        const unsigned csa2_trace_i = atomicAdd(::csa2::g_tl_ctr, 1u);                            \
        if (csa2_trace_i < ::csa2::g_tl_cap) {                                                    \
            ::csa2::g_tl_buf[4 * csa2_trace_i] = (kind);                                          \
            ::csa2::g_tl_buf[4 * csa2_trace_i + 1] = ::csa2::trace_cta();                         \
            ::csa2::g_tl_buf[4 * csa2_trace_i + 2] = csa2_trace_t0;                               \
            ::csa2::g_tl_buf[4 * csa2_trace_i + 3] = ::csa2::trace_gtimer();                      \
        }                                                                                         \
    }
// the host side of one translation unit's trace buffers (each unit has its own copies)
#define CSA2_TRACE_SETTER(name)                                                                   \
    extern "C" int name(void* slots, unsigned ncta, int on, void* tl, void* ctr, unsigned cap) {  \
        if (cudaMemcpyToSymbol(csa2::g_trace_buf, &slots, sizeof(slots)) != cudaSuccess) return 1; \
        if (cudaMemcpyToSymbol(csa2::g_trace_ncta, &ncta, sizeof(ncta)) != cudaSuccess) return 2;  \
        if (cudaMemcpyToSymbol(csa2::g_trace_on, &on, sizeof(on)) != cudaSuccess) return 3;        \
        if (cudaMemcpyToSymbol(csa2::g_tl_buf, &tl, sizeof(tl)) != cudaSuccess) return 4;          \
        if (cudaMemcpyToSymbol(csa2::g_tl_ctr, &ctr, sizeof(ctr)) != cudaSuccess) return 5;        \
        if (cudaMemcpyToSymbol(csa2::g_tl_cap, &cap, sizeof(cap)) != cudaSuccess) return 6;        \
        return 0;                                                                                 \
    }
#else
#define CSA2_TRACE_INIT()
#define CSA2_TRACE(slot)
#define CSA2_TRACE_VAL(slot, v)
#define CSA2_TRACE_END(kind)
#define CSA2_TRACE_SETTER(name)
#endif

// Range-checked build (compiled with -DCSA2_CHECKED, library libcsa2_checked.so): a
// computed shared- or global-memory index is checked before the access it guards; a
// violation is reported as CSA2_ERR_RANGE with `detail` naming the site, and the
// access is skipped. In the normal build the check is the constant true.
// CSA2_GUARD keeps its bound in both builds (an access the normal build skips quietly)
// and reports a violation in the checked one.
#ifdef CSA2_CHECKED
#define CSA2_CHECK(cond, st, detail) (::csa2::checked_ok((cond), (st), (detail)))
#define CSA2_GUARD(cond, st, detail) (::csa2::checked_ok((cond), (st), (detail)))
#else
#define CSA2_CHECK(cond, st, detail) (true)
#define CSA2_GUARD(cond, st, detail) (cond)
#endif

__device__ __forceinline__ bool checked_ok(bool cond, int32_t* st, int detail) {
    if (!cond) report(st, CSA2_ERR_RANGE, detail);
    return cond;
}


// Last global entry a query at position t may read ("CED: Continuing Context with a
// Causal Encoder and Decoder", "What Does the Sequence Compression Rate Reduce?"):
// with compression rate m >= 2, entry j combines positions m j .. m j + m - 1 and
// is read once all of them are <= t (complete groups); with m <= 1 entries are
// positions. Negative for a query that can read no entry yet.
__host__ __device__ __forceinline__ int last_entry(int t, int m) { return m >= 2 ? (t + 1) / m - 1 : t; }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ int ld_relaxed_gpu(const int* p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase. Returns false (and reports) on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* st, int where) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kSpinBudgetCycles) {
            report(st, CSA2_ERR_TIMEOUT, where);
            return false;
        }
    }
    return true;
}

// 3-D tiled TMA load into this CTA's shared memory, completing on `bar`.
// No cluster multicast; the innermost coordinate x must be 16-byte aligned.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* map, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
        "%4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_dsmem(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start before the previous kernel in the stream has finished;
// pdl_wait() blocks until that kernel has completed and its writes are visible
// (it returns at once when there is no such dependency). pdl_launch_dependents()
// lets the next kernel start early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] x B[smem desc], one CTA, kind::f16 (bf16 inputs here).
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A x B with signed int8 operands and int32 accumulation (kind::i8).
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once all tcgen05.mma issued so far by this thread complete.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 32 bits, 8 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, int (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for tcgen05.mma (sm_100 format):
// start address >> 4 in bits [0,14), leading byte offset >> 4 in [16,30),
// stride byte offset >> 4 in [32,46), version 1 in [46,48), base offset 0,
// swizzle mode in [61,64): 2 = 128-byte, 4 = 64-byte, 6 = 32-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t swizzle = 2) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)(swizzle & 7u) << 61;
    return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 accumulation.
// a_mn_major: A stored M-major (1) or K-major (0); B is K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major) {
    return (1u << 4)                          // D format: f32
           | (1u << 7)                        // A format: bf16
           | (1u << 10)                       // B format: bf16
           | ((uint32_t)a_mn_major << 15)     // A major
           | (0u << 16)                       // B major: K
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// The same with f16 A and B.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_mn_major) {
    return idesc_bf16(M, N, a_mn_major) & ~((7u << 7) | (7u << 10));
}

// Instruction descriptor, kind::i8 with signed int8 A/B (both K-major) and int32 accumulation.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
    return (2u << 4)                          // D format: s32
           | (1u << 7)                        // A format: signed 8-bit
           | (1u << 10)                       // B format: signed 8-bit
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Byte offset of the 16-byte chunk `chunk` of row `row` inside a 128-byte-swizzled
// panel whose rows are 128 bytes long (panel base 1024-byte aligned).
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
inline cudaError_t set_smem_once(const void* kern, int bytes) {
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    constexpr int kSlots = 64;
    static const void* kerns[kSlots] = {nullptr};
    static unsigned long long done[kSlots] = {0};   // bit per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    int slot = -1;
    for (int i = 0; i < kSlots; ++i) {
        if (kerns[i] == kern) { slot = i; break; }
        if (kerns[i] == nullptr) { kerns[i] = kern; slot = i; break; }
    }
    if (slot >= 0 && dev < 64 && (done[slot] >> dev) & 1ull) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && slot >= 0 && dev < 64) done[slot] |= 1ull << dev;
    return e;
}

}  // namespace csa2

// dsa_common.cuh -- shared device helpers for the sm_100a kernels of libdsa.
//
// Status word, bounded waits, mbarrier / bulk-copy / TMA / tcgen05 PTX
// wrappers and the order-preserving float key used by the top-k.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/dsa.h"

namespace dsa {

// ---------------------------------------------------------------------------
// Workspace header: the first 256 bytes of every workspace.
// ---------------------------------------------------------------------------
struct WsHeader {
    int status;        // DSA_STATUS_* bits, OR-ed by kernels
    int detail;        // first offending value (bad index) or wait site
    int test_hook;     // DSA_TEST_WITHHOLD_TILE: the TMA producers withhold their first key tile
    int sel_full_rows;  // decode rows whose bin select fell back to the whole row (statistics)
    int sel_max_kept;   // most keys a decode row's bin select kept (statistics)
    int pad[59];
};
static constexpr size_t kWsHeaderBytes = 256;

// True when the host asked the TMA-fed kernels to withhold their first key tile, so that
// every bounded wait on it runs out and the kernel reports DSA_STATUS_TIMEOUT (the test of
// the timeout path; no fault, no unbounded wait).
__device__ __forceinline__ bool test_withhold_tile(const WsHeader* h) {
    return h && *reinterpret_cast<const volatile int*>(&h->test_hook) == DSA_TEST_WITHHOLD_TILE;
}

__device__ __forceinline__ void raise_status(WsHeader* h, int bits, int detail) {
    if (h) {
        atomicOr(&h->status, bits);
        atomicCAS(&h->detail, 0, detail);
    }
}

// Index rows shared by consecutive query rows (multi-token decode): query row i of
// a sequence uses index row i / q_per_idx and skips entries after its own absolute
// position q_pos0 + i.  q_per_idx = 1 without a position limit is the plain case.
struct IdxShare {
    int q_per_idx;
    int q_pos0;    // absolute position of query row 0; ignored when causal == 0
    int causal;
    __host__ __device__ int rows(int n_q) const { return (n_q + q_per_idx - 1) / q_per_idx; }
    __host__ __device__ int limit(int i) const { return causal ? q_pos0 + i : 0x7fffffff; }
};
static constexpr IdxShare kNoShare = {1, 0, 0};

// Paged K/V cache (serving): token t of sequence b lives in row
// table[b * max_pages + t / page_size] * page_size + t % page_size of a
// [num_pages * page_size, ...] pool; lens[b] is the sequence's cache length.
// table == NULL: the contiguous [B, n_kv, ...] layout.
struct KvPages {
    const int* table;
    const int* lens;
    int page_size, max_pages, num_pages;
    int page_shift;  // log2(page_size) when it is a power of two, else -1 (shift / mask instead of divide)
    __device__ __forceinline__ int page_of(int t) const { return page_shift >= 0 ? t >> page_shift : t / page_size; }
    __device__ __forceinline__ int in_page(int t) const {
        return page_shift >= 0 ? t & (page_size - 1) : t % page_size;
    }
};
static constexpr KvPages kContiguous = {nullptr, nullptr, 0, 0, 0, -1};
// log2 of a power-of-two page size, -1 for any other size
inline int page_shift_of(int page_size) {
    if (page_size < 1 || (page_size & (page_size - 1)) != 0) return -1;
    int s = 0;
    while ((1 << s) < page_size) ++s;
    return s;
}

// Top bits of an order-preserving score key that the one-query decode indexer counts into a
// per-row histogram for the bin select that follows it (sign, 8 exponent bits, 4 mantissa bits).
static constexpr int kBinTopkBits = 13;

// Nanoseconds from the global timer.
__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Every device-side wait in this library gives up after this long and
// reports DSA_STATUS_TIMEOUT instead of hanging the GPU.
static constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// ---------------------------------------------------------------------------
// Shared-memory address helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
        "r"(bytes)
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

// As mbar_try_wait, but the thread may stay suspended up to `hint_ns` while
// the phase is incomplete (fewer spin iterations stealing issue slots).
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete; false on timeout
// (the caller then records DSA_STATUS_TIMEOUT and winds down).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
        if ((it & 15u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
}

// ---------------------------------------------------------------------------
// Bulk (non-tensor) async copy global -> shared, completion on an mbarrier.
// Both addresses 16-byte aligned, size a multiple of 16.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                         uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ---------------------------------------------------------------------------
// Order-preserving 32-bit key of an fp32 score: larger float <-> larger key;
// -0.0 and +0.0 map to the same key.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t score_key(float f) {
    // f + 0.0f turns -0.0 into +0.0 (round to nearest) and leaves every other value alone;
    // then negative floats are bit-inverted and non-negative ones get the sign bit set
    const uint32_t u = __float_as_uint(__fadd_rn(f, 0.0f));
    return u ^ (static_cast<uint32_t>(static_cast<int32_t>(u) >> 31) | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// Named barrier over `nthreads` threads (multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace dsa

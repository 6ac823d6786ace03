// tri_internal.cuh -- device helpers shared by the libtri kernels (sm_100a).
//
// Inline PTX wrappers for mbarriers and TMA bulk-tensor loads, the
// order-preserving float -> uint32 map used by the radix select, the device
// flag word, and the constants of the supported shape (head_dim 128).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tri.h"

namespace tri {

constexpr int kD = 128;          // head_dim
constexpr int kF = kD / 2;       // RoPE bands
constexpr int kChunks = 16;      // 16-byte chunks of a bf16 row (4 bands each)
constexpr int kWChunk = 12;      // floats per (head, chunk) weight record: 8 w + 4 c
constexpr int kWHead = kChunks * kWChunk;  // 192 floats per query head
// Place of band f's weights within a head's record.  The record of chunk
// c = f / 4 (bands 4c..4c+3, i = f % 4) is
//   [ReA_0, ReA_1, ImA_0, ImA_1, ReA_2, ReA_3, ImA_2, ImA_3, c_0, c_1, c_2, c_3],
// so a band pair's real parts (and its imaginary parts) are adjacent: the
// score loop multiplies them with (x_i, x_i+1) and (y_i, y_i+1) register
// pairs, the same pairs its packed band-norm products use.
__host__ __device__ constexpr int wrec_re(int f) {
    return (f >> 2) * kWChunk + ((f & 3) >> 1) * 4 + (f & 1);
}
__host__ __device__ constexpr int wrec_im(int f) { return wrec_re(f) + 2; }
__host__ __device__ constexpr int wrec_c(int f) { return (f >> 2) * kWChunk + 8 + (f & 3); }
constexpr int kMaxG = TRI_MAX_GROUP;

// Flag word at the start of every workspace.
struct WsHeader {
    uint32_t flags;
    uint32_t pad[63];
};
constexpr size_t kWsHeader = sizeof(WsHeader);  // 256 bytes

__device__ __forceinline__ void raise_flag(uint32_t* flag, uint32_t bits) {
    if (flag) atomicOr(flag, bits);
}

// Order-preserving 32-bit key of a float: a > b  <=>  key(a) > key(b) for
// numbers; -0.0 and +0.0 share a key; NaN maps to 0, below every number.
__device__ __forceinline__ uint32_t ordered_key(float x) {
    if (x != x) return 0u;
    uint32_t u = __float_as_uint(x);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)::"memory");
    return t;
}

// Wait for the phase with the given parity to complete, giving up after
// kWaitLimitNs nanoseconds (a TMA tile lands in microseconds; the limit only
// exists so that a fault elsewhere can never hang the GPU).  Returns false on
// timeout and raises TRI_FLAG_TIMEOUT.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            raise_flag(flag, TRI_FLAG_TIMEOUT);
            return false;
        }
    }
}

// ---------------------------------------------------------------------------
// TMA (bulk tensor copies, no multicast)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// L2 cache policies for TMA / bulk copies.
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 2-D tile load with an L2 cache policy.
__device__ __forceinline__ void tma_load_2d_hint(void* smem_dst, const CUtensorMap* map,
                                                 uint64_t* bar, int32_t x, int32_t y,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

// 1-D bulk copies (addresses 16-byte aligned, size a multiple of 16).
// global -> shared, completion counted on an mbarrier:
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// global -> shared with an L2 cache policy:
// Ask L2 to fetch [gsrc, gsrc + bytes) ahead of its use (16-byte aligned,
// a multiple of 16 bytes); nothing lands in shared memory.
__device__ __forceinline__ void prefetch_l2_bulk(const void* gsrc, uint32_t bytes, uint64_t policy) {
    asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;" ::"l"(
                     reinterpret_cast<uint64_t>(gsrc)),
                 "r"(bytes), "l"(policy)
                 : "memory");
}

__device__ __forceinline__ void bulk_load_hint(void* smem_dst, const void* gsrc, uint32_t bytes,
                                               uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// shared -> global, tracked by bulk groups of the issuing thread:
__device__ __forceinline__ void bulk_store(void* gdst, const void* smem_src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                     reinterpret_cast<uint64_t>(gdst)),
                 "r"(smem_u32(smem_src)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N committed bulk groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until every committed bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Order this thread's generic-proxy shared-memory accesses before later
// async-proxy (TMA / bulk copy) accesses, and the reverse.
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Streaming 16-byte global load (read once: no L1 allocation) and store
// (evict-first).
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream(uint4* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// 16-byte load that bypasses L1 (data written by other CTAs).
__device__ __forceinline__ uint4 ld_cg_u4(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Copy n16 16-byte words that other CTAs wrote in this launch from global
// memory (through L2, bypassing L1) to shared memory, every thread of the CTA
// keeping up to 8 loads in flight.
__device__ __forceinline__ void copy_l2_to_shared(uint4* dst, const uint4* src, int n16) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    for (int base = 0; base < n16; base += 8 * nthr) {
        uint4 v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int i = base + q * nthr + tid;
            if (i < n16) v[q] = ld_cg_u4(src + i);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int i = base + q * nthr + tid;
            if (i < n16) dst[i] = v[q];
        }
    }
}

// Named barrier among `count` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Approximate IEEE sqrt (max relative error ~2^-23, PTX sqrt.approx).
__device__ __forceinline__ float sqrt_approx(float x) {
    float r;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// bf16 pair in one 32-bit word: low half is the even element.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ int clamp_nvalid(const int32_t* n_valid, int64_t u, int64_t cap,
                                            uint32_t* flag) {
    if (!n_valid) return static_cast<int>(cap);
    int n = n_valid[u];
    if (n < 0 || n > cap) {
        raise_flag(flag, TRI_FLAG_NVALID_RANGE);
        n = n < 0 ? 0 : static_cast<int>(cap);
    }
    return n;
}

// Budget of unit u: the per-unit budget array, clamped to [0, B], or B.
__device__ __forceinline__ int64_t unit_budget(const int32_t* ub, int64_t u, int64_t B) {
    if (!ub) return B;
    const int64_t b = ub[u];
    return b < 0 ? 0 : (b > B ? B : b);
}

}  // namespace tri

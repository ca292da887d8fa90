// common.cuh -- sm_100a helpers shared by the decode kernels: mbarriers,
// bulk (TMA) copies, bounded waits, the device error word.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace attn {

constexpr int kBlockSize = 64;              // tokens per paged cache block

// Device error word bits (read and cleared by attn_decode_last_error).
constexpr unsigned kErrTimeout = 1u;
constexpr unsigned kErrBadBlock = 2u;
constexpr unsigned kErrBadSeqLen = 4u;

// Default bound of every spin-wait: 2 seconds of %globaltimer.
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;

__device__ __forceinline__ void raise_error(unsigned *err, unsigned bits) {
    atomicOr(err, bits);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(count)
                 : "memory");
}

// Make mbarrier initialisation visible to the async proxy (bulk copies).
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    uint64_t state;
    asm volatile("mbarrier.arrive.shared::cta.b64 %0, [%1];"
                 : "=l"(state)
                 : "r"(smem_u32(bar))
                 : "memory");
    (void)state;
}

// One arrival per warp (the barrier counts warps): the lanes' prior memory
// operations are ordered before lane 0's arrival by the warp barrier, so one
// release stands for the whole warp and the barrier word takes 1/32 of the
// atomic traffic.  All 32 lanes must call it.
__device__ __forceinline__ void mbar_arrive_warp(uint64_t *bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar,
                                                      uint32_t bytes) {
    uint64_t state;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 %0, [%1], %2;"
                 : "=l"(state)
                 : "r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
    (void)state;
}

// Waits for the phase for at most about kSuspendNs (the thread sleeps until
// the phase completes or the hint expires), then reports whether it did.
constexpr uint32_t kSuspendNs = 20000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "n"(kSuspendNs)
        : "memory");
    return done != 0;
}

// As mbar_try_wait, with a short suspend hint (kWatchNs), for a waiter that
// has something else to look at between polls.
constexpr uint32_t kWatchNs = 1000;
__device__ __forceinline__ bool mbar_try_wait_short(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "n"(kWatchNs)
        : "memory");
    return done != 0;
}

// Non-blocking probe of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait for the phase of `bar` with the given parity to complete.
// Returns false if it did not within timeout_ns (raising kErrTimeout), or as
// soon as another warp of the CTA has set *abort (then without raising).
// The clock is read only every 64 failed polls: reading %globaltimer is not
// free, and a tight loop of it starves other warps of the same pipe.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          unsigned long long timeout_ns,
                                          unsigned *err,
                                          volatile int *abort = nullptr) {
    if (mbar_try_wait(bar, parity)) return true;
    unsigned long long t0 = 0;
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (abort && *abort) return false;
        if ((it & 63u) == 0) {
            const unsigned long long now = global_timer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > timeout_ns) {
                raise_error(err, kErrTimeout);
                if (abort) *abort = 1;
                return false;
            }
        }
    }
}

// mbar_wait for a whole warp (all 32 lanes call it together) that runs
// `idle()` between polls of at most kWatchNs each.  Same bounds and results
// as mbar_wait; the lanes leave together.
template <typename F>
__device__ __forceinline__ bool mbar_wait_watch(uint64_t *bar, uint32_t parity,
                                                unsigned long long timeout_ns,
                                                unsigned *err, volatile int *abort,
                                                F &&idle) {
    unsigned long long t0 = 0;
    for (uint32_t it = 0;; ++it) {
        if (__any_sync(0xffffffffu, mbar_try_wait_short(bar, parity))) return true;
        if (*abort) return false;
        idle();
        if ((it & 7u) == 7u) {
            const unsigned long long now = global_timer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > timeout_ns) {
                if ((threadIdx.x & 31) == 0) raise_error(err, kErrTimeout);
                *abort = 1;
                return false;
            }
        }
    }
}

// GPU-scope relaxed load and store of a 32-bit word, and an acquire-release
// fence: a relaxed read that observes a value written by another CTA's
// release sequence, followed by the fence, orders this CTA's later reads
// after that CTA's writes.
__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_gpu(unsigned *p, unsigned v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_acq_rel_gpu() {
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Named barrier among `count` threads (multiple of 32), id 1..15.
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ------------------------------------------------------ register split
// Per-warpgroup register budget (all threads of the warpgroup execute it).
template <uint32_t N>
__device__ __forceinline__ void regs_increase() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_decrease() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// --------------------------------------------------------- bulk async copy
// 1-D bulk copy global -> shared, completion counted on `bar` in bytes.
// src and dst 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *dst_smem, const void *src,
                                          uint32_t bytes, uint64_t *bar,
                                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// The same without a cache hint.
__device__ __forceinline__ void bulk_load(void *dst_smem, const void *src,
                                          uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Prefetch `bytes` (multiple of 16, 16-byte aligned) of global memory into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes)
                 : "memory");
}

// L2 policy for data read exactly once (the streamed KV cache).
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t policy;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;"
                 : "=l"(policy));
    return policy;
}

// ------------------------------------------------ programmatic dependent launch
__device__ __forceinline__ void pdl_wait_primary() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------ conversions
// bf16 -> fp32 widening of the low / high half of a packed pair.  A bf16 is
// the top 16 bits of an fp32, so the widening is a shift or a mask; written
// as integer PTX so it stays on the integer pipes (a conversion instruction
// would run on the much narrower XU pipe).
__device__ __forceinline__ float bf16lo(uint32_t w) {
    uint32_t r;
    asm("shl.b32 %0, %1, 16;" : "=r"(r) : "r"(w));
    return __uint_as_float(r);
}
__device__ __forceinline__ float bf16hi(uint32_t w) {
    uint32_t r;
    asm("and.b32 %0, %1, 0xffff0000;" : "=r"(r) : "r"(w));
    return __uint_as_float(r);
}

template <typename T> struct ElemTraits;
template <> struct ElemTraits<float> {
    static constexpr int kBytes = 4;
    static __device__ __forceinline__ float to_float(float x) { return x; }
    static __device__ __forceinline__ float from_float(float x) { return x; }
};
template <> struct ElemTraits<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    static __device__ __forceinline__ float to_float(__nv_bfloat16 x) {
        return __bfloat162float(x);
    }
    static __device__ __forceinline__ __nv_bfloat16 from_float(float x) {
        return __float2bfloat16_rn(x);
    }
};

// Unpack one 16-byte chunk into fp32 values (8 for bf16, 4 for fp32).
template <typename T> struct Chunk;
template <> struct Chunk<__nv_bfloat16> {
    static constexpr int kElems = 8;
    static __device__ __forceinline__ void unpack(const uint4 &v, float *f) {
        f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
        f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
        f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
        f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
    }
};
template <> struct Chunk<float> {
    static constexpr int kElems = 4;
    static __device__ __forceinline__ void unpack(const uint4 &v, float *f) {
        f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
    }
};

}  // namespace attn

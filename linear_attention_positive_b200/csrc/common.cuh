// Device-side building blocks for the sm_100a FAVOR+ kernels: shared-memory barriers with bounded
// waits, TMA tensor and bulk copies, tcgen05 (5th-generation tensor core) MMA issue, tensor-memory
// (TMEM) allocation and load/store, and the descriptor encodings these instructions take.
//
// Every wait in this library is bounded: a wait that does not complete within kWaitLimitNs
// records FAVOR_ERR_TIMEOUT in the device status word and raises the CTA's abort flag, after which
// the kernel drains its own outstanding copies/MMAs (again bounded), frees its TMEM and returns.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/favor.h"

namespace favor {

constexpr int kTile = 128;               // tokens per tile (MMA M for token-major operands)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr unsigned long long kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s per wait

// Device status word (FAVOR_OK or FAVOR_ERR_TIMEOUT), read and cleared by favor_sync_status.
// The library is one translation unit (favor_api.cu includes every kernel file), so this is the
// only definition.
__device__ int g_status = FAVOR_OK;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_status, FAVOR_OK, code); }

// ------------------------------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// (No explicit suspend-time hint: one of 100 us measured 5-7 % slower on the forward kernels, whose
// consumer warps wake on the critical path.)
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

// Waits for the phase with the given parity to complete. Returns false (after recording
// FAVOR_ERR_TIMEOUT and raising *abort) if it does not complete within limit_ns, or at once if
// *abort is already raised by another warp of the CTA.
__device__ __forceinline__ bool mbar_wait_for(uint64_t *bar, uint32_t parity, volatile int *abort,
                                              unsigned long long limit_ns) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(a, parity)) return true;
        if ((it & 63u) == 0) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                record_status(FAVOR_ERR_TIMEOUT);
                *abort = 1;
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    return mbar_wait_for(bar, parity, abort, kWaitLimitNs);
}

// mbar_wait for all lanes of a converged warp, with a warp-uniform result.
__device__ __forceinline__ bool mbar_wait_all(uint64_t *bar, uint32_t parity, volatile int *abort) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}

// mbar_wait for a warp whose wait is off the critical path (producers that run ahead): lane 0
// polls, sleeping between polls so that the shared-memory pipe stays free for the consumers.
__device__ __forceinline__ bool mbar_wait_lazy(uint64_t *bar, uint32_t parity, volatile int *abort) {
    int ok = 1;
    if ((threadIdx.x & 31u) == 0) {
        const uint32_t a = smem_u32(bar);
        if (!mbar_try_wait(a, parity)) {
            const unsigned long long t0 = globaltimer_ns();
            for (uint32_t it = 1;; ++it) {
                __nanosleep(64);
                if (mbar_try_wait(a, parity)) break;
                if ((it & 15u) == 0) {
                    if (*abort) { ok = 0; break; }
                    if (globaltimer_ns() - t0 > kWaitLimitNs) {
                        record_status(FAVOR_ERR_TIMEOUT);
                        *abort = 1;
                        ok = 0;
                        break;
                    }
                }
            }
        }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    // the other lanes observe the completed phase too (acquire for their own later accesses)
    if (ok && (threadIdx.x & 31u) != 0) ok = mbar_try_wait(smem_u32(bar), parity) ? 1 : 0;
    return __all_sync(0xffffffffu, ok != 0);
}

// -------------------------------------------------------------------------------- TMA / bulk copy

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// Plain bulk copy global -> shared (both addresses 16-B aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// Generic-proxy shared-memory writes made visible to the async proxy (tensor core operand reads).
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ------------------------------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Issue forms. Every MMA / commit helper below has a warp-collective "_w" form: all 32 lanes of a
// converged warp execute it and the lane elect.sync picks issues the instruction, predicated inside
// the same asm block. Issued from a branch taken by one lane, a tcgen05.mma stalls the issuing
// thread for about 60-90 cycles (measured on B200); the predicated form issues in a cycle or two and
// leaves the MMAs queued behind each other, so small-N MMA chains run at the tensor pipe's rate.
#define FAVOR_ELECT "elect.sync _|e, 0xffffffff;\n\t"

// D[tmem] (+)= A[smem] * B[smem]; kind::f16 (bf16 operands), fp32 accumulation.
__device__ __forceinline__ void mma_f16_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]; kind::f16 with fp16 operands (A packed two per TMEM column,
// the lower K index in the low half), fp32 accumulation.
__device__ __forceinline__ void mma_f16_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// Chains of kind::f16 MMAs issued from one asm block, so the issuing thread spends a few
// instructions per MMA. Descriptors advance by a fixed number of 16-byte units per K-step of 16
// (the start-address field is the descriptor's low bits; no step crosses its range).
// D (+)= sum_k A_k B_k with A and B in shared memory: 4 K-steps, A/B advancing by a_step/b_step.
__device__ __forceinline__ void mma_ss_x4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc,
                                          uint32_t a_step, uint32_t b_step) {
    const uint64_t a1 = a + a_step, b1 = b + b_step, a2 = a1 + a_step, b2 = b1 + b_step, a3 = a2 + a_step,
                   b3 = b2 + b_step;
    asm volatile(
        "{\n\t.reg .pred p, t;\n\tsetp.ne.b32 p, %9, 0;\n\tsetp.eq.b32 t, %9, %9;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %8, p;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %4, %8, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %6, %8, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %10, %8, t;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "l"(a1), "l"(b1), "l"(a2), "l"(b2), "l"(a3), "r"(idesc), "r"(acc), "l"(b3)
        : "memory");
}

// D (+)= sum_k A_k B_k with A in TMEM (8 columns per K-step of 16 fp16) and B in shared memory:
// 4 K-steps, B advancing by b_step.
__device__ __forceinline__ void mma_ts_x4(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc,
                                          uint32_t b_step) {
    const uint64_t b1 = b + b_step, b2 = b1 + b_step, b3 = b2 + b_step;
    asm volatile(
        "{\n\t.reg .pred p, t;\n\tsetp.ne.b32 p, %6, 0;\n\tsetp.eq.b32 t, %6, %6;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %5, p;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%7], %3, %5, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%8], %4, %5, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%9], %10, %5, t;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "l"(b1), "l"(b2), "r"(idesc), "r"(acc), "r"(a_tmem + 8), "r"(a_tmem + 16),
        "r"(a_tmem + 24), "l"(b3)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]; kind::tf32, fp32 accumulation.
__device__ __forceinline__ void mma_tf32_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]; kind::tf32.
__device__ __forceinline__ void mma_tf32_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05.mma of this thread have completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// ---- warp-collective forms (see "Issue forms" above): call from all 32 lanes of a converged warp.

__device__ __forceinline__ void mma_f16_ss_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\t" FAVOR_ELECT
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_f16_ts_w(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\t" FAVOR_ELECT
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_tf32_ts_w(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\t" FAVOR_ELECT
        "@e tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_tf32_ss_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\t" FAVOR_ELECT
        "@e tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_ss_x4_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc,
                                            uint32_t a_step, uint32_t b_step) {
    const uint64_t a1 = a + a_step, b1 = b + b_step, a2 = a1 + a_step, b2 = b1 + b_step, a3 = a2 + a_step,
                   b3 = b2 + b_step;
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\tsetp.ne.b32 p, %9, 0;\n\tsetp.eq.b32 t, %9, %9;\n\t" FAVOR_ELECT
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %8, p;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %4, %8, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %6, %8, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %10, %8, t;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "l"(a1), "l"(b1), "l"(a2), "l"(b2), "l"(a3), "r"(idesc), "r"(acc), "l"(b3)
        : "memory");
}
__device__ __forceinline__ void mma_ts_x4_w(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc,
                                            uint32_t b_step) {
    const uint64_t b1 = b + b_step, b2 = b1 + b_step, b3 = b2 + b_step;
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\tsetp.ne.b32 p, %6, 0;\n\tsetp.eq.b32 t, %6, %6;\n\t" FAVOR_ELECT
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %5, p;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%7], %3, %5, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%8], %4, %5, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%9], %10, %5, t;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "l"(b1), "l"(b2), "r"(idesc), "r"(acc), "r"(a_tmem + 8), "r"(a_tmem + 16),
        "r"(a_tmem + 24), "l"(b3)
        : "memory");
}
__device__ __forceinline__ void mma_commit_w(uint64_t *bar) {
    asm volatile("{\n\t.reg .pred e;\n\t" FAVOR_ELECT
                 "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

// Instruction descriptor (kind::f16 / kind::tf32): fp32 accumulator, A/B format (1 = bf16,
// 2 = tf32), A/B major (0 = K-major, 1 = MN-major), N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, uint32_t fmt, uint32_t a_mn, uint32_t b_mn) {
    return (1u << 4) | (fmt << 7) | (fmt << 10) | (a_mn << 15) | (b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t kFmtF16 = 0;
constexpr uint32_t kFmtBF16 = 1;
constexpr uint32_t kFmtTF32 = 2;

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version bits. Byte offsets are
// encoded >> 4. K-major: SBO = stride between 8-row groups, LBO unused (1). MN-major: LBO =
// stride between 128-byte-wide blocks along M/N, SBO = stride between 8-row groups along K.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100
    d |= (uint64_t)2 << 61;  // SWIZZLE_128B
    return d;
}

// Shared-memory matrix descriptor without swizzle (interleaved core matrices of 8 rows x 16 bytes,
// each 128 contiguous bytes), K-major: LBO = byte stride between core matrices along K, SBO = byte
// stride between 8-row groups along M/N.
__device__ __forceinline__ uint64_t make_sdesc_interleaved(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100; layout type 0 (no swizzle)
    return d;
}

// fp32 -> bf16 bits, round to nearest even.
__device__ __forceinline__ uint32_t bf16_bits_rn(float x) {
    unsigned short h;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(x));
    return (uint32_t)h;
}

// Byte offset of the 16-byte chunk `chunk` (0..7) of row `row` inside a 128-byte-swizzled tile
// whose rows are 128 bytes long (the layout TMA writes with CU_TENSOR_MAP_SWIZZLE_128B).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

#define FAVOR_REG32(v)                                                                                      \
    "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]),        \
        "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15]), \
        "=f"(v[16]), "=f"(v[17]), "=f"(v[18]), "=f"(v[19]), "=f"(v[20]), "=f"(v[21]), "=f"(v[22]),          \
        "=f"(v[23]), "=f"(v[24]), "=f"(v[25]), "=f"(v[26]), "=f"(v[27]), "=f"(v[28]), "=f"(v[29]),          \
        "=f"(v[30]), "=f"(v[31])
#define FAVOR_RW32(v)                                                                                       \
    "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]), "+f"(v[7]),        \
        "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]), "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]), \
        "+f"(v[16]), "+f"(v[17]), "+f"(v[18]), "+f"(v[19]), "+f"(v[20]), "+f"(v[21]), "+f"(v[22]),          \
        "+f"(v[23]), "+f"(v[24]), "+f"(v[25]), "+f"(v[26]), "+f"(v[27]), "+f"(v[28]), "+f"(v[29]),          \
        "+f"(v[30]), "+f"(v[31])
#define FAVOR_IN32(v)                                                                                        \
    "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),      \
        "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]),       \
        "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]),      \
        "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])

// Loads 32 consecutive fp32 columns of this thread's TMEM lane (warp-collective; the address
// carries the warp's lane quarter in bits 16..). Waits for completion before returning.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : FAVOR_REG32(v)
        : "r"(taddr));
    // The wait names the registers so no use of them can be scheduled before it.
    asm volatile("tcgen05.wait::ld.sync.aligned;" : FAVOR_RW32(v)::"memory");
}

// Loads 32 consecutive fp32 columns of this thread's TMEM lane without waiting (warp-collective).
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, float (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : FAVOR_REG32(v)
        : "r"(taddr));
}
// Waits for this thread's outstanding TMEM loads; names v so no use of it moves above the wait.
__device__ __forceinline__ void tmem_wait_ld32(float (&v)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : FAVOR_RW32(v)::"memory");
}

// Stores 32 consecutive fp32 columns of this thread's TMEM lane (warp-collective; not waited).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        FAVOR_IN32(v)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Stores columns [OFF, OFF + 32) of a 128-value register row to 32 consecutive TMEM columns
// (compile-time offset, so the row stays in registers).
template <int OFF>
__device__ __forceinline__ void tmem_st32_at(uint32_t taddr, const float (&v)[128]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "f"(v[OFF + 0]), "f"(v[OFF + 1]), "f"(v[OFF + 2]), "f"(v[OFF + 3]), "f"(v[OFF + 4]), "f"(v[OFF + 5]),
        "f"(v[OFF + 6]), "f"(v[OFF + 7]), "f"(v[OFF + 8]), "f"(v[OFF + 9]), "f"(v[OFF + 10]), "f"(v[OFF + 11]),
        "f"(v[OFF + 12]), "f"(v[OFF + 13]), "f"(v[OFF + 14]), "f"(v[OFF + 15]), "f"(v[OFF + 16]), "f"(v[OFF + 17]),
        "f"(v[OFF + 18]), "f"(v[OFF + 19]), "f"(v[OFF + 20]), "f"(v[OFF + 21]), "f"(v[OFF + 22]), "f"(v[OFF + 23]),
        "f"(v[OFF + 24]), "f"(v[OFF + 25]), "f"(v[OFF + 26]), "f"(v[OFF + 27]), "f"(v[OFF + 28]), "f"(v[OFF + 29]),
        "f"(v[OFF + 30]), "f"(v[OFF + 31])
        : "memory");
}

#define FAVOR_REG128(v) FAVOR_REG32((&v[0])), FAVOR_REG32((&v[32])), FAVOR_REG32((&v[64])), FAVOR_REG32((&v[96]))

// Loads 128 consecutive fp32 columns of this thread's TMEM lane (two 64-column loads, so that no
// single instruction needs more than 64 destination registers) and waits for them.
#define FAVOR_REG64(v) FAVOR_REG32((&v[0])), FAVOR_REG32((&v[32]))
__device__ __forceinline__ void tmem_ld64_nowait(uint32_t taddr, float *v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
        "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
        "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, "
        "%51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
        : FAVOR_REG64(v)
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, float (&v)[128]) {
    tmem_ld64_nowait(taddr, &v[0]);
    tmem_ld64_nowait(taddr + 64, &v[64]);
    asm volatile("tcgen05.wait::ld.sync.aligned;" : FAVOR_RW32((&v[0])), FAVOR_RW32((&v[32])), FAVOR_RW32((&v[64])),
                 FAVOR_RW32((&v[96]))::"memory");
}

// Loads one fp32 column of this thread's TMEM lane and waits for it.
__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
    float v;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=f"(v) : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+f"(v)::"memory");
    return v;
}

#define FAVOR_U16(h, o)                                                                                        \
    "r"(h[o + 0]), "r"(h[o + 1]), "r"(h[o + 2]), "r"(h[o + 3]), "r"(h[o + 4]), "r"(h[o + 5]), "r"(h[o + 6]),   \
        "r"(h[o + 7]), "r"(h[o + 8]), "r"(h[o + 9]), "r"(h[o + 10]), "r"(h[o + 11]), "r"(h[o + 12]),           \
        "r"(h[o + 13]), "r"(h[o + 14]), "r"(h[o + 15])

// Stores 16 consecutive 32-bit columns of this thread's TMEM lane (warp-collective; not waited).
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&h)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        FAVOR_U16(h, 0)
        : "memory");
}

// Stores 64 consecutive 32-bit columns of this thread's TMEM lane (warp-collective; not waited).
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&h)[64]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, "
        "%35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, "
        "%56, %57, %58, %59, %60, %61, %62, %63, %64};" ::"r"(taddr),
        FAVOR_U16(h, 0), FAVOR_U16(h, 16), FAVOR_U16(h, 32), FAVOR_U16(h, 48)
        : "memory");
}

// Two fp32 values rounded to fp16 (nearest even) and packed, `lo` in the low 16 bits.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// {a0, a1} * {b0, b1} + {c0, c1} on the FMA pipe as one paired instruction.
__device__ __forceinline__ void ffma2(float a0, float a1, float b0, float b1, float c0, float c1, float &r0,
                                      float &r1) {
    uint64_t a, b, c, r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b0), "f"(b1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(c) : "f"(c0), "f"(c1));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r0), "=f"(r1) : "l"(r));
}

// Non-blocking test of an mbarrier phase (true once the phase with this parity has completed).
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Tiled TMA store shared -> global (bulk async-group completion).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(map),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until at most N committed bulk groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Waits until every committed bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_group_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Per-warpgroup register budget changes (all four warps of a warpgroup execute the same one).
template <int N>
__device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// TMEM address of (lane quarter of this warp, column).
__device__ __forceinline__ uint32_t tmem_lane_addr(uint32_t base, uint32_t warp_idx, uint32_t col) {
    return base + (((warp_idx & 3u) * 32u) << 16) + col;
}

// Named barrier among `nthreads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ uint32_t elect_lane0() { return (threadIdx.x & 31u) == 0u; }

// Programmatic dependent launch: let the next kernel on the stream (launched with the programmatic
// serialization attribute) start its prologue once every CTA of this grid has reached this point,
// and, in that next kernel, wait until this grid has completed and its writes are visible before
// reading them.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_prerequisites() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// One lane of a converged warp (elect.sync): the warp runs a producer loop together, so its
// descriptor arithmetic stays warp-uniform, and the elected lane issues the TMA / MMA instruction.
__device__ __forceinline__ bool elect_one() {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r));
    return r != 0;
}

// 2^t for a pair of values on the FMA pipe (no MUFU), t <= 0: Cody-Waite split t = n + f with
// n = round(t) taken from the low bits of t + 1.5*2^23, |f| <= 1/2, a degree-3 polynomial for 2^f
// (this library's own relative-minimax fit on [-1/2, 1/2], max relative error 7.5e-5, below the
// 2^-12 tf32 rounding applied afterwards) and n added to the exponent field. t is clamped at -126
// (results below 2^-126 come out as ~2^-126 instead of 0).
__device__ __forceinline__ void exp2_poly_pair(float t0, float t1, float &r0, float &r1) {
    constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
    t0 = fmaxf(t0, -126.0f);
    t1 = fmaxf(t1, -126.0f);
    uint64_t t, j, n, f, p;
    asm("mov.b64 %0, {%1, %2};" : "=l"(t) : "f"(t0), "f"(t1));
    const uint64_t sh = 0x4B4000004B400000ull, nsh = 0xCB400000CB400000ull;   // {kShift}, {-kShift}
    const uint64_t m1 = 0xBF800000BF800000ull;                                   // {-1}
    const uint64_t c3 = 0x3D61FBAF3D61FBAFull, c2 = 0x3E786F0D3E786F0Dull;      // 2^f ~ c0 + f(c1 + f(c2 + f c3))
    const uint64_t c1 = 0x3F31798D3F31798Dull, c0 = 0x3F7FFB493F7FFB49ull;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(j) : "l"(t), "l"(sh));
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(n) : "l"(j), "l"(nsh));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(f) : "l"(n), "l"(m1), "l"(t));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(c3), "l"(f), "l"(c2));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(c1));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(c0));
    const uint32_t j0 = (uint32_t)j, j1 = (uint32_t)(j >> 32);
    const uint32_t p0 = (uint32_t)p, p1 = (uint32_t)(p >> 32);
    r0 = __uint_as_float(p0 + (j0 << 23));
    r1 = __uint_as_float(p1 + (j1 << 23));
}

// The tensor core reads a tf32 operand as the fp32 value with its low 13 mantissa bits dropped
// (truncation). Sums taken on CUDA cores that must agree with an MMA over the same operand use the
// same truncated value, so both sides carry the same rounding.
__device__ __forceinline__ float tf32_trunc(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

// Rounds an MMA operand to tf32 (nearest, ties away from zero): returns the value to store (the
// bits plus half a tf32 ulp, which the tensor core's truncation turns into the rounded value) and
// sets `used` to that rounded value for sums on CUDA cores that must match the MMA.
__device__ __forceinline__ float tf32_round_store(float x, float &used) {
    const uint32_t u = __float_as_uint(x) + 0x1000u;
    used = __uint_as_float(u & 0xFFFFE000u);
    return __uint_as_float(u);
}

// Stored form of an fp32 value in an MMA operand image: half a tf32 ulp added to the bit pattern,
// so the hardware's truncation yields the value rounded to nearest (ties away). The exact fp32
// value is recovered by subtracting the same integer.
__device__ __forceinline__ float tf32_store(float x) { return __uint_as_float(__float_as_uint(x) + 0x1000u); }
__device__ __forceinline__ float tf32_load(float y) { return __uint_as_float(__float_as_uint(y) - 0x1000u); }

}  // namespace favor

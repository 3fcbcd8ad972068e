// Shared helpers of the paged-decode library: host-side status plumbing and
// thin inline-PTX wrappers for sm_100a (mbarrier, TMA tile loads, warp-level
// matrix moves and bf16 mma).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pa.h"

namespace pa {

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

void count_launch();
int device_sm_count();
// Maps the last CUDA error after a launch to a status.
int launch_status();
// The address a kernel on the current device uses for `p`: device or managed
// memory as is, page-locked host memory through its device mapping.  Host
// memory that is not page-locked (or a pointer CUDA does not know) gives
// PA_ERR_INVALID_ARG, so no kernel is ever handed an address it cannot reach.
int device_address(const void *p, void **dev_ptr);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Largest sequence group of the shared-prefix decode.
constexpr int kMaxGroupSize = 64;

// Shared body of every decode entry point (k_new == nullptr: no cache write;
// prefix_lens != nullptr: groups of group_size sequences share a prefix).
int decode_impl(float *out, const void *q, const void *k_new, const void *v_new, const void *k_cache,
                const void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                const int32_t *seq_lens, int batch, int max_seq_len, int num_q_heads, int num_kv_heads,
                int head_dim, int block_size, int64_t num_blocks, float scale, int partition_tokens,
                void *workspace, size_t workspace_bytes, int32_t *err_flag, void *stream, bool fp8,
                float k_scale, float v_scale, const int32_t *prefix_lens, int group_size);

inline bool supported_shape(int num_q_heads, int num_kv_heads, int head_dim, int block_size) {
    if (num_kv_heads <= 0 || num_q_heads <= 0 || num_q_heads % num_kv_heads) return false;
    const int g = num_q_heads / num_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8) return false;
    if (head_dim != 64 && head_dim != 128) return false;
    if (block_size != 8 && block_size != 16 && block_size != 32 && block_size != 64) return false;
    return true;
}

inline bool supported_block_size(int block_size) {
    return block_size == 8 || block_size == 16 || block_size == 32 || block_size == 64;
}

// ---------------------------------------------------------------------------
// Device side
// ---------------------------------------------------------------------------

// A bounded wait gives up after this many SM clock cycles (about one second).
constexpr long long kWaitLimitCycles = 2000000000LL;

// Wait style: 0 = mbarrier.try_wait (the thread may be suspended by the
// hardware until the phase completes), 1 = mbarrier.test_wait spin.
#ifndef PA_WAIT_SPIN
#define PA_WAIT_SPIN 0
#endif
// try_wait's suspend-time hint in ns (0: none, the hardware's own limit).  A
// waiting thread sleeps until the phase completes or the hint runs out.  A
// tuning knob: on B200 a 10 ms hint made the decode 1-3 % slower.
#ifndef PA_WAIT_SUSPEND_NS
#define PA_WAIT_SUSPEND_NS 0
#endif

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void raise_flag(int32_t *flag, int bits) {
    if (flag) atomicOr(flag, bits);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t *bar, uint32_t parity, uint32_t ns) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity), "r"(ns)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for the phase of `bar` with the given parity to complete.  Returns
// false (and sets PA_FLAG_TIMEOUT) if that takes longer than kWaitLimitCycles
// (give or take one suspend-time hint).  Without a hint the clock is only read
// every 64 polls, so the common case costs one poll.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, int32_t *flag) {
    const long long t0 = clock64();
    for (uint32_t it = 1;; ++it) {
#if PA_WAIT_SPIN
        if (mbar_test_wait(bar, parity)) return true;
#elif PA_WAIT_SUSPEND_NS > 0
        if (mbar_try_wait_suspend(bar, parity, PA_WAIT_SUSPEND_NS)) return true;
        it = 0;  // every poll may have slept: read the clock each time
#else
        if (mbar_try_wait(bar, parity)) return true;
#endif
        if ((it & 63u) == 0 && clock64() - t0 > kWaitLimitCycles) {
            raise_flag(flag, PA_FLAG_TIMEOUT);
            return false;
        }
    }
}

// Order this thread's generic-proxy shared-memory accesses before later
// async-proxy (TMA) accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D TMA tile load (no multicast) into CTA shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar, uint64_t cache_policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::"
        "cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)),
        "l"(cache_policy)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Asynchronous global -> shared copies (no register staging); wait with cp_async_wait_all.
__device__ __forceinline__ void cp_async16(uint32_t smem_dst, const void *gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(smem_dst), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t smem_dst, const void *gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_dst), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                                  uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// D = A(16x16, row) * B(16x8, col) + D, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A(16x16, row) * B(16x8, col) + D, f16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four E4M3 codes (byte 0 first) -> two f16x2 words (exact conversions).
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t four_codes, uint32_t &f01, uint32_t &f23) {
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
        : "=r"(f01), "=r"(f23)
        : "r"(four_codes));
}

// Two E4M3 codes (low byte first) -> two f16 values (exact), as one 32-bit word.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
    uint32_t f01, f23;
    e4m3x4_to_f16x4(two_codes, f01, f23);
    return f01;
}

// Eight bf16 values -> eight E4M3 codes: code = E4M3(x * inv_scale), the product
// in fp32, rounded to nearest even and saturated to the largest finite value.
__device__ __forceinline__ uint2 bf16x8_to_e4m3x8(uint4 v, float inv_scale) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float lo = __fmul_rn(__uint_as_float(w[k] << 16), inv_scale);
        const float hi = __fmul_rn(__uint_as_float(w[k] & 0xffff0000u), inv_scale);
        const uint32_t pair = (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
        out[k >> 1] |= pair << ((k & 1) * 16);
    }
    return make_uint2(out[0], out[1]);
}

// Pack two floats as f16x2 (round to nearest even); `lo` lands in bits 0..15.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

__device__ __forceinline__ float f16_lo_to_float(uint32_t v) {
    return __half2float(__ushort_as_half((unsigned short)(v & 0xffffu)));
}
__device__ __forceinline__ float f16_hi_to_float(uint32_t v) {
    return __half2float(__ushort_as_half((unsigned short)(v >> 16)));
}

// ---- 5th-generation tensor cores (tcgen05): TMEM and single-thread MMA ----

// Allocate `ncols` TMEM columns (a power of two >= 32) for this CTA; the
// address lands in shared memory.  Whole warp; the same warp frees them.
__device__ __forceinline__ void tmem_alloc(uint32_t smem_dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_dst), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Order tcgen05 operations around a thread synchronisation (barrier, mbarrier).
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major operand stored as rows of 128
// bytes with the 128-byte swizzle (the TMA SWIZZLE_128B layout), 8-row groups
// 1024 bytes apart, the group base 1024-byte aligned.  Adding 2 advances the
// start by 32 bytes: the next 32-element K step of an 8-bit operand.
__device__ __forceinline__ uint64_t umma_desc_k_sw128(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3ffffu) >> 4)  // start address, 16-byte units
           | ((uint64_t)1 << 16)                  // leading byte offset (16 B; unused when swizzled)
           | ((uint64_t)(1024 >> 4) << 32)        // stride byte offset: next 8-row group
           | ((uint64_t)1 << 46)                  // descriptor version of sm_100
           | ((uint64_t)2 << 61);                 // 128-byte swizzle
}

// D[tmem] (+)= A * B^T, both operands E4M3 from shared memory (K-major), fp32
// accumulate; issued by one thread.  `accumulate` false overwrites D.
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05.mma this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

// 16 TMEM lanes x 8 fp32 columns into the warp, in the mma.sync accumulator
// layout: lane (g, t) gets (row g, cols 2t, 2t+1) and (row g + 8, cols 2t, 2t+1).
// Waits for the load before returning.
__device__ __forceinline__ void tmem_ld_16x256b(uint32_t taddr, float (&v)[4]) {
    uint32_t r0, r1, r2, r3;
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0, %1, %2, %3}, [%4];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
        : "r"(taddr)
        : "memory");
    v[0] = __uint_as_float(r0);
    v[1] = __uint_as_float(r1);
    v[2] = __uint_as_float(r2);
    v[3] = __uint_as_float(r3);
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Pack two floats as bf16x2 (round to nearest even); `lo` lands in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float bf16_lo_to_float(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi_to_float(uint32_t v) {
    return __uint_as_float(v & 0xffff0000u);
}

}  // namespace pa

// q8_common.cuh -- device helpers shared by the libq8 kernels (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <float.h>
#include <stdint.h>

#include <atomic>

#include "../../include/q8.h"

#ifndef __CUDACC__
#error "q8_common.cuh is CUDA source"
#endif

namespace q8 {

// ---------------------------------------------------------------- exact fp32 steps
// The code-deciding steps are written with explicit round-to-nearest intrinsics so
// that the compiler cannot contract them into fused multiply-adds.

// Activation code: clamp(round(v * inv) + z, -128, 127) with round = ties to even
// (the fake_quant / quantize_per_tensor recipe of the SmolVLM q8 page).  Clamping
// happens in fp32 before the integer conversion, so huge |v| saturate correctly.
__device__ __forceinline__ int act_code(float v, float inv, float zf) {
    float t = __fmul_rn(v, inv);
    float r = __fadd_rn(rintf(t), zf);
    r = fminf(fmaxf(r, -128.0f), 127.0f);
    return __float2int_rn(r);
}

// Asymmetric int8 parameters of a row whose values span [mn, mx] (choose_qparams_affine
// of the executorch 8da4w operator): the range is widened to include 0, s = (mx - mn) / 255
// (at least FLT_EPSILON) and z = -128 - round(mn / s), clamped to [-128, 127].
__device__ __forceinline__ void qparams_from_range(float mn, float mx, float& s, float& zf) {
    mn = fminf(mn, 0.0f);
    mx = fmaxf(mx, 0.0f);
    s = __fdiv_rn(__fsub_rn(mx, mn), 255.0f);
    if (s < FLT_EPSILON) s = FLT_EPSILON;
    zf = __fsub_rn(-128.0f, rintf(__fdiv_rn(mn, s)));
    zf = fminf(fmaxf(zf, -128.0f), 127.0f);
}

// Weight code: clamp(round(w / s), lo, hi) with a true IEEE division.
__device__ __forceinline__ int weight_code(float w, float s, float lo, float hi) {
    float r = rintf(__fdiv_rn(w, s));
    r = fminf(fmaxf(r, lo), hi);
    return __float2int_rn(r);
}

__device__ __forceinline__ uint32_t pack4_s8(int a, int b, int c, int d) {
    return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
           ((uint32_t)(d & 0xFF) << 24);
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---------------------------------------------------------------- memory helpers

// Streaming 16-byte global load through the non-coherent path, not kept in L1.
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16-byte global load through L1 (small operands re-read by many warps).
__device__ __forceinline__ uint4 ldg_keep(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float4 ldg_f4(const float* p) {
    float4 v;
    asm volatile("ld.global.nc.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

// ---------------------------------------------------------------- warp helpers
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---------------------------------------------------------------- int8 -> bf16
// Four int8 codes packed in one word -> two bf16x2 words (low pair, high pair), exact.
// Byte b (two's complement) becomes the fp32 2^23 + (b ^ 0x80) by inserting it into the
// mantissa of 2^23; subtracting 2^23 + 128 leaves the integer b exactly.  An integer with
// |b| <= 128 has at most 8 significant bits, so its bf16 is the high half of its fp32.
__device__ __forceinline__ void s8x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = w ^ 0x80808080u;
    const uint32_t magic = 0x4B000000u;
    uint32_t f0 = __byte_perm(u, magic, 0x7650);
    uint32_t f1 = __byte_perm(u, magic, 0x7651);
    uint32_t f2 = __byte_perm(u, magic, 0x7652);
    uint32_t f3 = __byte_perm(u, magic, 0x7653);
    const float off = 8388736.0f;  // 2^23 + 128
    float a0 = __fsub_rn(__uint_as_float(f0), off);
    float a1 = __fsub_rn(__uint_as_float(f1), off);
    float a2 = __fsub_rn(__uint_as_float(f2), off);
    float a3 = __fsub_rn(__uint_as_float(f3), off);
    lo = __byte_perm(__float_as_uint(a0), __float_as_uint(a1), 0x7632);
    hi = __byte_perm(__float_as_uint(a2), __float_as_uint(a3), 0x7632);
}

// Four int8 codes w = [b0 b1 b2 b3] -> bf16x2 (b0, b2) and (b1, b3), exact, in 7 ALU ops.
// For a byte b in the low half of a 16-bit lane: bf16 bits 0x4300 | (b & 0x7F) are the value
// 128 + (b & 0x7F), and 0x4300 | (b & 0x80) is 128 (b >= 0) or 256 (b < 0); their
// difference is b in both cases and is exact in bf16 (an integer of at most 8 bits).
// The odd bytes are first shifted into the low halves.  The pairing (even, odd) is a
// permutation of k that the caller applies to the other MMA operand as well.
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t mask, uint32_t bits) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(bits));  // (a&b)|c
    return d;
}
__device__ __forceinline__ void s8x4_to_bf16x2_eo(uint32_t w, uint32_t& even, uint32_t& odd) {
    const uint32_t o = w >> 8;
    even = bf16x2_sub(lop_and_or(w, 0x007F007Fu, 0x43004300u),
                      lop_and_or(w, 0x00800080u, 0x43004300u));
    odd = bf16x2_sub(lop_and_or(o, 0x007F007Fu, 0x43004300u),
                     lop_and_or(o, 0x00800080u, 0x43004300u));
}

// ---------------------------------------------------------------- legacy warp MMA
// D(16x8 fp32) += A(16x16 bf16, row) * B(16x8 bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D(16x8 s32) += A(16x32 s8, row) * B(32x8 s8, col)
__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1,
                                             uint32_t a2, uint32_t a3, uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

}  // namespace q8

// ============================================================ TMA / mbarrier (sm_90+)
#include <cuda.h>   // CUtensorMap (type only)

namespace q8 {

// Device status codes written to the caller-visible status word.
constexpr int kStatusWaitTimeout = 1;
constexpr int kStatusNotPositiveDefinite = 2;   // a Cholesky pivot was not positive
// Bounded waits give up after this many nanoseconds of %globaltimer (a correct kernel
// never waits more than microseconds; the limit only turns a logic error into an error
// status instead of a hang).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
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
// Non-blocking test of the same phase.  Measured on B200: a try_wait on an already completed
// phase still costs the issuing thread ~260 cycles, test_wait ~60 -- between the MMAs of a
// single issuing thread that difference halved the tensor-core rate -- so every wait starts
// with test_wait and only falls back to the suspending form.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
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
// The same test, but a thread whose phase is not complete is suspended until it completes
// or `hint_ns` nanoseconds pass.  Waiting threads then take no issue slots from the warps
// that share their scheduler (a hot spin on try_wait slowed a lone MMA-issuing thread
// several-fold), and a completed phase still wakes them at once.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity,
                                                    uint32_t hint_ns) {
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
constexpr uint32_t kWaitSleepNs = 20000;        // longest single suspension of a waiter

// Wait for the phase with the given parity to complete.  Returns false, after recording
// kStatusWaitTimeout in *status and raising the CTA's shared abort flag, if it has not
// completed within kWaitLimitNs -- or at once if the abort flag is already raised (so
// that after one expired wait every other wait of the CTA ends quickly too).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status,
                                          volatile int* abort_flag) {
    if (mbar_test_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
        if ((i & 7u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                atomicExch(status, kStatusWaitTimeout);
                return false;
            }
        }
    }
}
// Same bounded wait with a caller-chosen limit (the self-test uses a short one).
__device__ __forceinline__ bool mbar_wait_limit(uint64_t* bar, uint32_t parity, int* status,
                                                volatile int* abort_flag,
                                                unsigned long long limit_ns) {
    if (mbar_test_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
        if ((i & 7u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                *abort_flag = 1;
                atomicExch(status, kStatusWaitTimeout);
                return false;
            }
        }
    }
}
// Bounded wait used only on exit paths: waits for a phase without touching the abort flag.
// A drain that runs out of time means a logic error; it is recorded in *status if given.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity,
                                           int* status = nullptr) {
    if (mbar_test_wait(bar, parity)) return;
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            if (status) atomicExch(status, kStatusWaitTimeout);
            return;
        }
    }
}
// 2-D tiled TMA load of one box into shared memory; completion is signalled on `bar`
// (transaction bytes).  c0 is the innermost coordinate (bytes for 8-bit elements) and
// must be a multiple of 16.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}
// Same, with an L2 cache-eviction policy (from make_l2_policy_*).
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, int c0, int c1,
                                                 uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
// L2 policies: keep (operands re-read by many tiles) / drop first (read once).
__device__ __forceinline__ uint64_t make_l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t make_l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// Streaming fp32 store (write-once output: evict first from L2).
__device__ __forceinline__ void st_stream_f32(float* p, float v) {
    asm volatile("st.global.cs.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// ---------------------------------------------------------------- host helpers

// Raises kernel K's dynamic shared-memory limit on the current device to at least `bytes`.
// The attribute persists, so it is set once per size increase instead of before every
// launch (a per-call runtime call costs host time on decode-sized launches).
template <auto K>
inline cudaError_t ensure_dyn_smem(int bytes) {
    static std::atomic<int> set_bytes[128];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) {
        cudaGetLastError();
        return cudaErrorInvalidDevice;
    }
    if (set_bytes[dev].load(std::memory_order_relaxed) >= bytes) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(K, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               bytes);
    if (e == cudaSuccess) {
        int cur = set_bytes[dev].load(std::memory_order_relaxed);
        while (cur < bytes && !set_bytes[dev].compare_exchange_weak(cur, bytes)) {
        }
    }
    return e;
}

}  // namespace q8

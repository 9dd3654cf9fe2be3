// q8_common.cuh -- device helpers shared by the libq8 kernels (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

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

// Weight code: clamp(round(w / s), -lim, lim) with a true IEEE division.
__device__ __forceinline__ int weight_code(float w, float s, float lim) {
    float r = rintf(__fdiv_rn(w, s));
    r = fminf(fmaxf(r, -lim), lim);
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

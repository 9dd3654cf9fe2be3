// k_quant.cu -- the quantizers: per-row int8 weight codes, per-row affine activation
// qparams + codes, static per-tensor activation codes (with the two-pass residual),
// the per-tensor min/max observer, and int4 group-symmetric weight codes.
//
// All of them are HBM streams (a few bytes in, fewer out, per element).  Rows are
// handled by one CTA each so that the row reduction and the codes that depend on it
// stay in one place; loads are 16-byte vectors.
#include "q8_kernels.cuh"

#include <float.h>

namespace q8 {

// ------------------------------------------------------------------ block reductions
template <int THREADS>
__device__ __forceinline__ float block_max(float v, float* red) {
    v = warp_max(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    v = (lane < THREADS / 32) ? red[lane] : -FLT_MAX;
    return warp_max(v);
}
template <int THREADS>
__device__ __forceinline__ float block_min(float v, float* red) {
    v = warp_min(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    v = (lane < THREADS / 32) ? red[lane] : FLT_MAX;
    return warp_min(v);
}
template <int THREADS>
__device__ __forceinline__ int block_sum_i(int v, int* red) {
    v = warp_sum_i(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    v = (lane < THREADS / 32) ? red[lane] : 0;
    return warp_sum_i(v);
}

// ------------------------------------------------------------ int8 weight codes (a1)
// One CTA per row n.  Pass 1: absmax.  Pass 2 (row re-read from L1/L2): codes with a
// true division by the scale, the code sum, and 4-byte code stores.
//   full == 0 (ROCm-INT8 quantize_weight): s = amax / 127, codes clamp(rne(w / s), -127, 127);
//             an all-zero row gets s = 1 and zero codes.
//   full == 1 (SmolVLM-Q8 weight_int8, the per-channel symmetric min/max observer):
//             s = max(amax / 127.5, FLT_EPSILON), codes clamp(rne(w / s), -128, 127).
constexpr int QW_THREADS = 256;

__global__ __launch_bounds__(QW_THREADS) void k_quantize_weight(const float* __restrict__ W,
                                                                int K, int full,
                                                                int8_t* __restrict__ q,
                                                                float* __restrict__ s_w,
                                                                int32_t* __restrict__ wsum) {
    __shared__ float redf[QW_THREADS / 32];
    __shared__ int redi[QW_THREADS / 32];
    const int64_t n = blockIdx.x;
    const float* row = W + n * (int64_t)K;
    const int K4 = K >> 2;
    float amax = 0.0f;
    for (int i = threadIdx.x; i < K4; i += QW_THREADS) {
        float4 v = ldg_f4(row + 4 * i);
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    amax = block_max<QW_THREADS>(amax, redf);
    float scale = __fdiv_rn(amax, full ? 127.5f : 127.0f);
    const bool zero = !full && scale == 0.0f;
    if (zero) scale = 1.0f;
    if (full && scale < FLT_EPSILON) scale = FLT_EPSILON;
    const float lo = full ? -128.0f : -127.0f;
    int sum = 0;
    uint32_t* qrow = reinterpret_cast<uint32_t*>(q + n * (int64_t)K);
    for (int i = threadIdx.x; i < K4; i += QW_THREADS) {
        int c0 = 0, c1 = 0, c2 = 0, c3 = 0;
        if (!zero) {
            float4 v = ldg_f4(row + 4 * i);
            c0 = weight_code(v.x, scale, lo, 127.0f);
            c1 = weight_code(v.y, scale, lo, 127.0f);
            c2 = weight_code(v.z, scale, lo, 127.0f);
            c3 = weight_code(v.w, scale, lo, 127.0f);
        }
        sum += c0 + c1 + c2 + c3;
        qrow[i] = pack4_s8(c0, c1, c2, c3);
    }
    if (wsum) sum = block_sum_i<QW_THREADS>(sum, redi);
    if (threadIdx.x == 0) {
        s_w[n] = scale;
        if (wsum) wsum[n] = sum;
    }
}

// ------------------------------------------------- per-row activation qparams (a2)
constexpr int CQ_THREADS = 256;

__global__ __launch_bounds__(CQ_THREADS) void k_choose_qparams(const uint16_t* __restrict__ x,
                                                               int K, float* __restrict__ s_out,
                                                               int32_t* __restrict__ z_out,
                                                               int8_t* __restrict__ xq) {
    // A dependent kernel launched with programmatic serialisation (the 8da4w stream) may
    // start now: it waits for this grid before it reads the codes, scales or zero points.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // One CTA per row.  Rows of up to CQ_REG * 8 * CQ_THREADS values stay in registers
    // between the range pass and the code pass, and all their loads are in flight at once
    // (the kernel is latency-bound: one row is a few KB); longer rows are read twice.
    constexpr int CQ_REG = 4;
    __shared__ float red[2][CQ_THREADS / 32];
    const int64_t m = blockIdx.x;
    const uint16_t* row = x + m * (int64_t)K;
    const int K8 = K >> 3;
    const bool in_regs = K8 <= CQ_REG * CQ_THREADS;
    uint4 v[CQ_REG];
    float mn = 0.0f, mx = 0.0f;                  // the range always includes 0
    auto range = [&](const uint4& u) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float a = bf16lo(w[j]), b = bf16hi(w[j]);
            mn = fminf(mn, fminf(a, b));
            mx = fmaxf(mx, fmaxf(a, b));
        }
    };
    if (in_regs) {
#pragma unroll
        for (int r = 0; r < CQ_REG; ++r) {
            const int i = threadIdx.x + r * CQ_THREADS;
            v[r] = i < K8 ? ldg_keep(row + 8 * i) : make_uint4(0, 0, 0, 0);   // zeros: no effect
        }
#pragma unroll
        for (int r = 0; r < CQ_REG; ++r) range(v[r]);
    } else {
        for (int i = threadIdx.x; i < K8; i += CQ_THREADS) range(ldg_keep(row + 8 * i));
    }
    // min and max over the CTA, one barrier
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if ((threadIdx.x & 31) == 0) {
        red[0][threadIdx.x >> 5] = mn;
        red[1][threadIdx.x >> 5] = mx;
    }
    __syncthreads();
#pragma unroll
    for (int w = 0; w < CQ_THREADS / 32; ++w) {
        mn = fminf(mn, red[0][w]);
        mx = fmaxf(mx, red[1][w]);
    }
    float s, zf;
    qparams_from_range(mn, mx, s, zf);
    if (threadIdx.x == 0) {
        s_out[m] = s;
        z_out[m] = __float2int_rn(zf);
    }
    if (xq == nullptr) return;
    const float inv = __fdiv_rn(1.0f, s);
    uint2* qrow = reinterpret_cast<uint2*>(xq + m * (int64_t)K);
    auto codes = [&](const uint4& u, int i) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        int c[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            c[2 * j] = act_code(bf16lo(w[j]), inv, zf);
            c[2 * j + 1] = act_code(bf16hi(w[j]), inv, zf);
        }
        qrow[i] = make_uint2(pack4_s8(c[0], c[1], c[2], c[3]), pack4_s8(c[4], c[5], c[6], c[7]));
    };
    if (in_regs) {
#pragma unroll
        for (int r = 0; r < CQ_REG; ++r) {
            const int i = threadIdx.x + r * CQ_THREADS;
            if (i < K8) codes(v[r], i);
        }
    } else {
        for (int i = threadIdx.x; i < K8; i += CQ_THREADS) codes(ldg_keep(row + 8 * i), i);
    }
}

// Same qparams, but the codes leave as bf16 integers (xq - z) in [-255, 255] -- the
// activation operand of the tensor-core 8da4w linear (exact in bf16).
__global__ __launch_bounds__(CQ_THREADS) void k_choose_qparams_shifted(
    const uint16_t* __restrict__ x, int K, float* __restrict__ s_out, int32_t* __restrict__ z_out,
    uint16_t* __restrict__ xz) {
    __shared__ float red[CQ_THREADS / 32];
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t m = blockIdx.x;
    const uint16_t* row = x + m * (int64_t)K;
    const int K8 = K >> 3;
    float mn = 0.0f, mx = 0.0f;
    for (int i = threadIdx.x; i < K8; i += CQ_THREADS) {
        uint4 v = ldg_keep(row + 8 * i);
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float a = bf16lo(w[j]), b = bf16hi(w[j]);
            mn = fminf(mn, fminf(a, b));
            mx = fmaxf(mx, fmaxf(a, b));
        }
    }
    mn = block_min<CQ_THREADS>(mn, red);
    mx = block_max<CQ_THREADS>(mx, red);
    float s, zf;
    qparams_from_range(mn, mx, s, zf);
    if (threadIdx.x == 0) {
        s_out[m] = s;
        z_out[m] = __float2int_rn(zf);
    }
    const float inv = __fdiv_rn(1.0f, s);
    const int zi = __float2int_rn(zf);
    uint4* orow = reinterpret_cast<uint4*>(xz + m * (int64_t)K);
    for (int i = threadIdx.x; i < K8; i += CQ_THREADS) {
        uint4 v = ldg_keep(row + 8 * i);
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c0 = act_code(bf16lo(w[j]), inv, zf) - zi;
            const int c1 = act_code(bf16hi(w[j]), inv, zf) - zi;
            o[j] = (__float_as_uint((float)c0) >> 16) | (__float_as_uint((float)c1) & 0xFFFF0000u);
        }
        orow[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// ---------------------------------------------------- static activation codes (a3)
// Elementwise over M*K values (16 per thread per step).
__global__ __launch_bounds__(256) void k_quantize_static(const float* __restrict__ x, int64_t n16,
                                                         float s1, float z1f, int8_t* __restrict__ xq1,
                                                         int has2, float s2, float z2f,
                                                         int8_t* __restrict__ xq2) {
    // the linear launched next may start its set-up (it waits for this kernel's codes)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const float inv1 = __fdiv_rn(1.0f, s1);
    const float inv2 = has2 ? __fdiv_rn(1.0f, s2) : 0.0f;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n16;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float* p = x + 16 * i;
        float v[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float4 f = ldg_f4(p + 4 * j);
            v[4 * j] = f.x; v[4 * j + 1] = f.y; v[4 * j + 2] = f.z; v[4 * j + 3] = f.w;
        }
        uint32_t o1[4], o2[4];
        static_codes16(v, s1, inv1, z1f, has2, inv2, z2f, o1, o2);
        reinterpret_cast<uint4*>(xq1)[i] = make_uint4(o1[0], o1[1], o1[2], o1[3]);
        if (has2) reinterpret_cast<uint4*>(xq2)[i] = make_uint4(o2[0], o2[1], o2[2], o2[3]);
    }
}

// ------------------------------------------------------ per-tensor min/max observer
// Float atomics by integer ordering: for v >= 0 signed-int order equals float order,
// for v < 0 unsigned order is reversed float order.
__device__ __forceinline__ void atomic_max_f(float* a, float v) {
    if (v >= 0.0f) atomicMax(reinterpret_cast<int*>(a), __float_as_int(v));
    else atomicMin(reinterpret_cast<unsigned*>(a), __float_as_uint(v));
}
__device__ __forceinline__ void atomic_min_f(float* a, float v) {
    if (v >= 0.0f) atomicMin(reinterpret_cast<int*>(a), __float_as_int(v));
    else atomicMax(reinterpret_cast<unsigned*>(a), __float_as_uint(v));
}

__global__ void k_minmax_reset(float* mm) {
    mm[0] = __int_as_float(0x7f800000);   // +inf
    mm[1] = __int_as_float(0xff800000);   // -inf
}

// RES = false: min / max of the values themselves (act_observer).
// RES = true:  min / max of the first-pass rounding error r = x - fake_quant(x, s1, z1),
//              the transform the second calibration run observes ([SmolVLM-Q8] calibrate):
//              r = x - (code - z1) * s1 with code = clamp(round(x * (1/s1)) + z1, -128, 127),
//              every step rounded to fp32 exactly as the two-pass quantizer computes it.
template <bool RES>
__device__ __forceinline__ float observed(float v, float s1, float inv1, float z1f) {
    if (!RES) return v;
    const float d1 = __fmul_rn(__fsub_rn((float)act_code(v, inv1, z1f), z1f), s1);
    return __fsub_rn(v, d1);
}

template <bool RES>
__global__ __launch_bounds__(256) void k_observe_minmax(const float* __restrict__ x, int64_t n,
                                                        float s1, float z1f, float* mm) {
    __shared__ float red[8];
    const float inv1 = RES ? __fdiv_rn(1.0f, s1) : 0.0f;
    float lo = FLT_MAX, hi = -FLT_MAX;
    const int64_t n4 = n >> 2;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x) {
        float4 v = ldg_f4(x + 4 * i);
        v.x = observed<RES>(v.x, s1, inv1, z1f);
        v.y = observed<RES>(v.y, s1, inv1, z1f);
        v.z = observed<RES>(v.z, s1, inv1, z1f);
        v.w = observed<RES>(v.w, s1, inv1, z1f);
        lo = fminf(lo, fminf(fminf(v.x, v.y), fminf(v.z, v.w)));
        hi = fmaxf(hi, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
    }
    for (int64_t i = 4 * n4 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float v = observed<RES>(x[i], s1, inv1, z1f);
        lo = fminf(lo, v);
        hi = fmaxf(hi, v);
    }
    lo = block_min<256>(lo, red);
    hi = block_max<256>(hi, red);
    if (threadIdx.x == 0) {
        atomic_min_f(&mm[0], lo);
        atomic_max_f(&mm[1], hi);
    }
}

// ------------------------------------------------------ int4 group weight codes
// One warp per group of G = 32*E consecutive k; lane l holds E consecutive values.
template <int E>
__global__ __launch_bounds__(256) void k_quantize_weight_q4gs(const float* __restrict__ W,
                                                              int64_t groups, int K,
                                                              uint8_t* __restrict__ q4,
                                                              float* __restrict__ gs) {
    constexpr int G = 32 * E;
    const int lane = threadIdx.x & 31;
    const int64_t g = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5);
    if (g >= groups) return;
    const int ng = K / G;
    const int64_t n = g / ng;
    const int gi = (int)(g - n * ng);
    const float* p = W + n * (int64_t)K + (int64_t)gi * G + lane * E;
    float v[E];
    if constexpr (E == 1) {
        v[0] = __ldg(p);
    } else if constexpr (E == 2) {
        float2 f = __ldg(reinterpret_cast<const float2*>(p));
        v[0] = f.x; v[1] = f.y;
    } else {
#pragma unroll
        for (int j = 0; j < E / 4; ++j) {
            float4 f = ldg_f4(p + 4 * j);
            v[4 * j] = f.x; v[4 * j + 1] = f.y; v[4 * j + 2] = f.z; v[4 * j + 3] = f.w;
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < E; ++j) amax = fmaxf(amax, fabsf(v[j]));
    amax = warp_max(amax);
    float scale = __fdiv_rn(amax, 7.0f);
    const bool zero = (scale == 0.0f);
    if (zero) scale = 1.0f;
    int c[E];
#pragma unroll
    for (int j = 0; j < E; ++j) c[j] = zero ? 0 : weight_code(v[j], scale, -7.0f, 7.0f);
    uint8_t* out = q4 + n * (int64_t)(K / 2) + ((int64_t)gi * G + lane * E) / 2;
    if constexpr (E == 1) {
        int other = __shfl_down_sync(0xffffffffu, c[0], 1);
        if ((lane & 1) == 0) *out = (uint8_t)((c[0] & 0xF) | ((other & 0xF) << 4));
    } else {
        uint32_t packed = 0;
#pragma unroll
        for (int j = 0; j < E; ++j) packed |= (uint32_t)(c[j] & 0xF) << (4 * j);
        if constexpr (E == 2) *out = (uint8_t)packed;
        else if constexpr (E == 4) *reinterpret_cast<uint16_t*>(out) = (uint16_t)packed;
        else *reinterpret_cast<uint32_t*>(out) = packed;
    }
    if (lane == 0) gs[g] = scale;
}

// Zero-point fold of the 8da4w weight (pytorch/executorch PR #21229, linear_dq8ca_q4gsw:
// out = s * sum_k (xq - z) * dequant(w), whose zero-point part is z * c[n] with c[n] the
// row sum of the dequantized weight):
//     c[n] = sum_g gs[n,g] * S[n,g],   S[n,g] = sum of the group's signed 4-bit codes.
// One warp per row.  Lane j computes the exact fp64 product for group base + j (24-bit
// scale times a code sum of at most 12 bits); the warp then adds the 32 products in group
// order (every lane runs the same sequential chain), so the fp64 sum runs over g ascending
// and is rounded once to fp32.
__global__ __launch_bounds__(256) void k_q4gs_zero_fold(const uint8_t* __restrict__ q4,
                                                        const float* __restrict__ gs, int G,
                                                        int64_t N, int K,
                                                        float* __restrict__ c) {
    const int lane = threadIdx.x & 31;
    const int64_t n = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5);
    if (n >= N) return;
    const int ng = K / G;
    const uint8_t* row = q4 + n * (int64_t)(K / 2);
    const float* grow = gs + n * (int64_t)ng;
    double acc = 0.0;
    for (int base = 0; base < ng; base += 32) {
        const int g = base + lane;
        double p = 0.0;
        if (g < ng) {
            // G / 2 bytes per group, a multiple of 16: whole 16-byte loads
            const uint4* src = reinterpret_cast<const uint4*>(row + (int64_t)g * (G / 2));
            int S = 0;
            for (int i = 0; i < G / 32; ++i) {
                const uint4 v = __ldg(src + i);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int b = 0; b < 8; ++b)
                        S += (int)(w[j] << (28 - 4 * b)) >> 28;     // sign-extended nibble
            }
            p = (double)__ldg(grow + g) * (double)S;                 // exact
        }
        const int cnt = ng - base < 32 ? ng - base : 32;
        for (int j = 0; j < cnt; ++j) acc = __dadd_rn(acc, __shfl_sync(0xffffffffu, p, j));
    }
    if (lane == 0) c[n] = __double2float_rn(acc);
}

// ---------------------------------------------------------------------- launchers
cudaError_t launch_quantize_weight(const float* W, int64_t N, int K, int full, int8_t* q,
                                   float* s_w, int32_t* wsum, cudaStream_t st) {
    k_quantize_weight<<<(unsigned)N, QW_THREADS, 0, st>>>(W, K, full, q, s_w, wsum);
    return cudaGetLastError();
}

cudaError_t launch_choose_qparams(const uint16_t* x, int64_t M, int K, float* s, int32_t* z,
                                  int8_t* xq, cudaStream_t st) {
    k_choose_qparams<<<(unsigned)M, CQ_THREADS, 0, st>>>(x, K, s, z, xq);
    return cudaGetLastError();
}

cudaError_t launch_choose_qparams_shifted(const uint16_t* x, int64_t M, int K, float* s,
                                          int32_t* z, uint16_t* xz, cudaStream_t st) {
    k_choose_qparams_shifted<<<(unsigned)M, CQ_THREADS, 0, st>>>(x, K, s, z, xz);
    return cudaGetLastError();
}

cudaError_t launch_quantize_static(const float* x, int64_t M, int K, float s1, int z1, int has2,
                                   float s2, int z2, int8_t* xq1, int8_t* xq2, cudaStream_t st,
                                   int num_sms) {
    const int64_t n16 = M * (int64_t)K / 16;
    int64_t blocks = (n16 + 255) / 256;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    k_quantize_static<<<(unsigned)blocks, 256, 0, st>>>(x, n16, s1, (float)z1, xq1, has2, s2,
                                                       (float)z2, xq2);
    return cudaGetLastError();
}

cudaError_t launch_observe_minmax(const float* x, int64_t n, float* mm, int reset, int residual,
                                  float s1, int z1, cudaStream_t st, int num_sms) {
    if (reset) k_minmax_reset<<<1, 1, 0, st>>>(mm);
    if (n > 0) {
        int64_t blocks = (n / 4 + 255) / 256;
        const int64_t cap = (int64_t)num_sms * 4;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        if (residual)
            k_observe_minmax<true><<<(unsigned)blocks, 256, 0, st>>>(x, n, s1, (float)z1, mm);
        else
            k_observe_minmax<false><<<(unsigned)blocks, 256, 0, st>>>(x, n, 1.0f, 0.0f, mm);
    }
    return cudaGetLastError();
}

cudaError_t launch_quantize_weight_q4gs(const float* W, int64_t N, int K, int G, uint8_t* q4,
                                        float* gs, cudaStream_t st) {
    const int64_t groups = N * (int64_t)(K / G);
    const unsigned blocks = (unsigned)((groups + 7) / 8);
    switch (G) {
        case 32: k_quantize_weight_q4gs<1><<<blocks, 256, 0, st>>>(W, groups, K, q4, gs); break;
        case 64: k_quantize_weight_q4gs<2><<<blocks, 256, 0, st>>>(W, groups, K, q4, gs); break;
        case 128: k_quantize_weight_q4gs<4><<<blocks, 256, 0, st>>>(W, groups, K, q4, gs); break;
        case 256: k_quantize_weight_q4gs<8><<<blocks, 256, 0, st>>>(W, groups, K, q4, gs); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_q4gs_zero_fold(const uint8_t* q4, const float* gs, int G, int64_t N, int K,
                                  float* c, cudaStream_t st) {
    k_q4gs_zero_fold<<<(unsigned)((N + 7) / 8), 256, 0, st>>>(q4, gs, G, N, K, c);
    return cudaGetLastError();
}

}  // namespace q8

// k_w4a16.cu -- the NVFP4 weight-only twin of the W8A16 decode linear.
//
// flashrt-structures schemes.py, W4A16Decode: the weight is held as NVFP4 -- E2M1 codes
// packed two per byte plus one scale per 16-element block -- and the activations stay bf16,
// so the decode band streams about half the weight bytes of W8A16.  The page prints no
// quantization rule; the one taken (NVIDIA's NVFP4 layout) is:
//   gsc = amax(W) / (6 * 448)                        per-tensor fp32 (1.0 for W == 0)
//   per block b of 16 consecutive k of a row:
//     sb = amax_b / 6, e = rn_e4m3(sb / gsc), d = e4m3(e) * gsc       (fp32 steps)
//     code = rn_e2m1(W / d)                         (IEEE division; d == 0: codes 0)
//   rounding to the nearest value with ties to the even code, saturating at the largest
//   finite magnitude (6 for E2M1, 448 for E4M3); a value that rounds to 0 gets code +0;
//   byte k/2 of a row holds code k in its low nibble (k even), block scales are bytes
//   [N, K/16].
//   y[m, n] = gsc * sum_k x[m, k] * (e2m1(code[n, k]) * e4m3(e[n, k / 16]))
// The product e2m1 * e4m3 has at most 2 + 4 significant bits and lies within bf16's normal
// range, so the kernels form it exactly in bf16 and run the same bf16 tensor-core MMA as
// W8A16; gsc multiplies the finished sum.
#include "q8_kernels.cuh"

namespace q8 {

// ----------------------------------------------------------------------- quantizer
// Tensor absmax, as the bits of a non-negative float (their integer order is the float
// order, so atomicMax on the bits is the float max; the result does not depend on order).
__global__ __launch_bounds__(256) void k_nvfp4_absmax(const float* __restrict__ W, int64_t n,
                                                      unsigned int* __restrict__ amax_bits) {
    float m = 0.0f;
    const int64_t n4 = n >> 2;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float4 v = ldg_f4(W + 4 * i);
        m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

__device__ __forceinline__ float nvfp4_gsc(float amax) {
    const float g = __fdiv_rn(amax, 2688.0f);         // 6 * 448
    return g == 0.0f ? 1.0f : g;
}

// E4M3 byte -> fp32 (exact): exponent bits 6..3 (bias 7), mantissa bits 2..0, subnormals
// m/8 * 2^-6 (only non-negative scale bytes occur here).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    return e == 0 ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Nearest E4M3 (ties to even, saturating at 448) / E2M1 (ties to even, saturating at 6)
// with the hardware conversions; the same value goes to both halves of the packed result.
__device__ __forceinline__ uint32_t rn_e4m3_sat(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(v));
    return r & 0xFFu;
}
__device__ __forceinline__ uint32_t rn_e2m1_sat(float v) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %1;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r)
        : "f"(v));
    r &= 0xFu;
    return (r & 7u) == 0 ? 0u : r;                   // magnitude 0: code +0
}

// One thread per block of 16 weights.
__global__ __launch_bounds__(256) void k_nvfp4_blocks(const float* __restrict__ W,
                                                      int64_t nblocks,
                                                      const unsigned int* __restrict__ amax_bits,
                                                      uint8_t* __restrict__ q4,
                                                      uint8_t* __restrict__ sf) {
    const int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (b >= nblocks) return;
    const float gsc = nvfp4_gsc(__uint_as_float(*amax_bits));
    float v[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float4 f = ldg_f4(W + 16 * b + 4 * j);
        v[4 * j] = f.x; v[4 * j + 1] = f.y; v[4 * j + 2] = f.z; v[4 * j + 3] = f.w;
    }
    float bmax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) bmax = fmaxf(bmax, fabsf(v[j]));
    const uint32_t e = rn_e4m3_sat(__fdiv_rn(__fdiv_rn(bmax, 6.0f), gsc));
    const float d = __fmul_rn(e4m3_to_f32(e), gsc);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const uint32_t c = d == 0.0f ? 0u : rn_e2m1_sat(__fdiv_rn(v[j], d));
        if (j < 8) lo |= c << (4 * j);
        else hi |= c << (4 * (j - 8));
    }
    *reinterpret_cast<uint2*>(q4 + 8 * b) = make_uint2(lo, hi);
    sf[b] = (uint8_t)e;
}

__global__ void k_nvfp4_gsc(const unsigned int* __restrict__ amax_bits, float* __restrict__ gsc) {
    *gsc = nvfp4_gsc(__uint_as_float(*amax_bits));
}

cudaError_t launch_quantize_weight_nvfp4(const float* W, int64_t N, int K, uint8_t* q4,
                                         uint8_t* sf, float* gsc, cudaStream_t st, int num_sms) {
    // the output scalar holds the absmax bits until the last launch replaces them by gsc
    unsigned int* amax = reinterpret_cast<unsigned int*>(gsc);
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned int), st);
    if (e != cudaSuccess) return e;
    const int64_t n = N * (int64_t)K;
    int64_t grid = (n / 4 + 255) / 256;
    if (grid > (int64_t)num_sms * 8) grid = (int64_t)num_sms * 8;
    k_nvfp4_absmax<<<(unsigned)grid, 256, 0, st>>>(W, n, amax);
    const int64_t nb = n / 16;
    k_nvfp4_blocks<<<(unsigned)((nb + 255) / 256), 256, 0, st>>>(W, nb, amax, q4, sf);
    k_nvfp4_gsc<<<1, 1, 0, st>>>(amax, gsc);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------- the linear
// Eight packed E2M1 codes w (code i in bits 4i..4i+3) times a bf16 block scale s (as
// bf16x2 (s, s)) -> four bf16x2 words of consecutive codes (0,1) (2,3) (4,5) (6,7), exact.
// The bf16 of a magnitude index i comes from two 8-entry byte tables (high and low byte)
// looked up with byte permutes; the sign bit of each code is moved to bit 15 / 31 with
// sign-replicating byte permutes.
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ void e2m1x8_to_bf16x2(uint32_t w, uint32_t s, uint32_t (&o)[4]) {
    // magnitudes 0 .5 1 1.5 2 3 4 6 as bf16: high bytes 00 3F 3F 3F 40 40 40 40,
    // low bytes 00 00 80 C0 00 40 80 C0
    constexpr uint32_t TH0 = 0x3F3F3F00u, TH1 = 0x40404040u;
    constexpr uint32_t TL0 = 0xC0800000u, TL1 = 0xC0804000u;
    const uint32_t m = w & 0x77777777u;
    const uint32_t h0 = __byte_perm(TH0, TH1, m), l0 = __byte_perm(TL0, TL1, m);
    const uint32_t m2 = m >> 16;
    const uint32_t h1 = __byte_perm(TH0, TH1, m2), l1 = __byte_perm(TL0, TL1, m2);
    // signs: code 2j's sign is the top bit of byte j of (w << 4), code 2j+1's of byte j of w
    const uint32_t ws = w << 4;
    o[0] = lop_and_or(__byte_perm(ws, w, 0xC080u), 0x80008000u, __byte_perm(l0, h0, 0x5140u));
    o[1] = lop_and_or(__byte_perm(ws, w, 0xD091u), 0x80008000u, __byte_perm(l0, h0, 0x7362u));
    o[2] = lop_and_or(__byte_perm(ws, w, 0xE0A2u), 0x80008000u, __byte_perm(l1, h1, 0x5140u));
    o[3] = lop_and_or(__byte_perm(ws, w, 0xF0B3u), 0x80008000u, __byte_perm(l1, h1, 0x7362u));
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = bf16x2_mul(o[i], s);
}

// E4M3 scale byte -> bf16x2 (v, v), exact (4 significant bits, within bf16's range).
__device__ __forceinline__ uint32_t e4m3_to_bf16x2(uint32_t b) {
    const uint32_t h = __float_as_uint(e4m3_to_f32(b)) >> 16;
    return h | (h << 16);
}

// Register-streamed GEMV: a CTA of 4 warps owns 16 output channels and all of K, cut into
// chunks of 128 codes (64 bytes per row); warp w takes chunks w, w+4, ...  In a chunk, lane
// (g = lane/4, t = lane%4) loads bytes [16t, 16t+16) -- codes [32t, 32t+32), two scale blocks
// -- of rows n0+g and n0+g+8, and the matching 32 activations of its activation rows.  The
// lane's 32 codes feed its own k slots of 8 MMA steps (m16n8k16): code pairs (4j, 4j+1) and
// (4j+2, 4j+3) go to the slots (2t, 2t+1) and (2t+8, 2t+9) of step j, and the activation
// pairs with the same k go to the same slots of the B fragment, so no data moves between
// lanes.  The four warps' sums are added through shared memory in warp order.
constexpr int W4_THREADS = 128;
constexpr int W4_WARPS = W4_THREADS / 32;

template <int MT, int UNROLL>
__global__ __launch_bounds__(W4_THREADS) void k_w4a16_gemv(
    const uint16_t* __restrict__ x, const uint8_t* __restrict__ q4,
    const uint8_t* __restrict__ sf, const float* __restrict__ gsc, void* __restrict__ y,
    int y_bf16, int M, int N, int K) {
    __shared__ float red[W4_WARPS][MT][32][4];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int n0 = blockIdx.x * 16;
    const int m0 = blockIdx.y * (8 * MT);
    const int nchunks = (K + 127) >> 7;
    const int KB = K >> 4;                              // scale bytes per row

    const int rowa = n0 + g, rowb = n0 + g + 8;
    const bool va = rowa < N, vb = rowb < N;
    const uint8_t* qa = q4 + (int64_t)(va ? rowa : 0) * (K >> 1) + 16 * t;
    const uint8_t* qb = q4 + (int64_t)(vb ? rowb : 0) * (K >> 1) + 16 * t;
    const uint8_t* sa = sf + (int64_t)(va ? rowa : 0) * KB + 2 * t;
    const uint8_t* sb = sf + (int64_t)(vb ? rowb : 0) * KB + 2 * t;
    const uint16_t* xr[MT];
    bool xv[MT];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int m = m0 + mt * 8 + g;
        xv[mt] = m < M;
        xr[mt] = x + (int64_t)(xv[mt] ? m : 0) * K + 32 * t;
    }
    float acc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[mt][i] = 0.0f;

    const uint4 zero4 = make_uint4(0, 0, 0, 0);
    for (int c = warp; c < nchunks; c += W4_WARPS * UNROLL) {
        uint4 wa[UNROLL], wb[UNROLL], xa[UNROLL][MT][4];
        uint32_t ea[UNROLL], eb[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int cc = c + W4_WARPS * u;
            const int kk = cc * 128 + 32 * t;           // first code of this lane
            const bool kin = (cc < nchunks) && (kk < K);   // K % 32 == 0: all 32 or none
            wa[u] = (va && kin) ? ldg_stream(qa + cc * 64) : zero4;
            wb[u] = (vb && kin) ? ldg_stream(qb + cc * 64) : zero4;
            ea[u] = (va && kin) ? (uint32_t)__ldg(reinterpret_cast<const uint16_t*>(sa + cc * 8)) : 0u;
            eb[u] = (vb && kin) ? (uint32_t)__ldg(reinterpret_cast<const uint16_t*>(sb + cc * 8)) : 0u;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const bool ok = xv[mt] && kin;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    xa[u][mt][i] = ok ? ldg_keep(xr[mt] + cc * 128 + 8 * i) : zero4;
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const uint32_t sa0 = e4m3_to_bf16x2(ea[u] & 0xFFu), sa1 = e4m3_to_bf16x2(ea[u] >> 8);
            const uint32_t sb0 = e4m3_to_bf16x2(eb[u] & 0xFFu), sb1 = e4m3_to_bf16x2(eb[u] >> 8);
            const uint32_t wav[4] = {wa[u].x, wa[u].y, wa[u].z, wa[u].w};
            const uint32_t wbv[4] = {wb[u].x, wb[u].y, wb[u].z, wb[u].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {                // word q: codes 8q..8q+7, block q/2
                uint32_t A[4], B[4];
                e2m1x8_to_bf16x2(wav[q], q < 2 ? sa0 : sa1, A);
                e2m1x8_to_bf16x2(wbv[q], q < 2 ? sb0 : sb1, B);
#pragma unroll
                for (int h = 0; h < 2; ++h) {            // MMA step j = 2q + h: codes 4j..4j+3
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        const uint4& xs = xa[u][mt][q];  // activations 8q..8q+7 of the lane
                        const uint32_t b0 = h ? xs.z : xs.x;
                        const uint32_t b1 = h ? xs.w : xs.y;
                        mma_bf16_16816(acc[mt], A[2 * h], B[2 * h], A[2 * h + 1], B[2 * h + 1],
                                       b0, b1);
                    }
                }
            }
        }
    }

#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) red[warp][mt][lane][i] = acc[mt][i];
    __syncthreads();
    const float gs = __ldg(gsc);
    for (int e = threadIdx.x; e < MT * 128; e += W4_THREADS) {
        const int mt = e >> 7, l = (e >> 2) & 31, ci = e & 3;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < W4_WARPS; ++w) v += red[w][mt][l][ci];
        const int m = m0 + mt * 8 + 2 * (l & 3) + (ci & 1);
        const int n = n0 + (l >> 2) + 8 * (ci >> 1);
        if (m < M && n < N) {
            const float r = v * gs;
            if (y_bf16)
                reinterpret_cast<__nv_bfloat16*>(y)[(int64_t)m * N + n] = __float2bfloat16_rn(r);
            else
                reinterpret_cast<float*>(y)[(int64_t)m * N + n] = r;
        }
    }
}

cudaError_t launch_w4a16_nvfp4(const uint16_t* x, const uint8_t* q4, const uint8_t* sf,
                               const float* gsc, void* y, int y_bf16, int64_t M, int64_t N, int K,
                               cudaStream_t st) {
    const unsigned gn = (unsigned)((N + 15) / 16);
    if (M <= 8) {
        k_w4a16_gemv<1, 2><<<dim3(gn, 1), W4_THREADS, 0, st>>>(x, q4, sf, gsc, y, y_bf16, (int)M,
                                                               (int)N, K);
    } else {
        const unsigned gm = (unsigned)((M + 15) / 16);
        k_w4a16_gemv<2, 2><<<dim3(gn, gm), W4_THREADS, 0, st>>>(x, q4, sf, gsc, y, y_bf16,
                                                                (int)M, (int)N, K);
    }
    return cudaGetLastError();
}

}  // namespace q8

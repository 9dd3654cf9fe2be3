// k_gemv.cu -- decode-sized (M <= 16 per block) quantized linears as HBM-streaming GEMVs.
//
// The weight matrix q[N, K] is read exactly once, straight from HBM into registers with
// 16-byte streaming loads; the activations (a few KB) come from L2.  The per-element
// multiply-adds run on the tensor cores through the warp-level MMA, because at M = 16
// there are 16 multiply-adds per weight byte: more than the fp32 pipes can issue at HBM
// speed, while the tensor pipes are nearly idle (a few percent of their peak).  The MMA
// here is only an arithmetic helper for a memory-bound stream; the operands never touch
// shared memory.
//
// Layout of the work.  A CTA of 4 warps owns 16 output channels (rows n0..n0+15 of q) and
// all of K.  K is cut into 64-byte chunks; warp w takes chunks w, w+4, w+8, ...  In a chunk,
// lane (g = lane/4, t = lane%4) loads the 16 bytes [16t, 16t+16) of rows n0+g and n0+g+8,
// and the matching 16 activations of activation row g.  The MMA's k order is immaterial
// to the dot product, so each lane's 16 contiguous k are simply assigned to its own k
// slots of 4 (bf16, k16) or 2 (int8, k32) MMA steps -- no data movement between lanes.
// The four warps' partial sums are added through shared memory and the epilogue applies
// the per-channel scale (and for W8A8 the zero-point term) once.
#include "q8_kernels.cuh"

namespace q8 {

constexpr int GEMV_THREADS = 128;
constexpr int GEMV_WARPS = GEMV_THREADS / 32;

// ------------------------------------------------------------------------- W8A16
// y[m, n] = s_w[n] * sum_k x[m, k] * q[n, k] (+ bias[n]); MT n8-tiles cover 8*MT
// activation rows.
template <int MT, int UNROLL>
__global__ __launch_bounds__(GEMV_THREADS) void k_w8a16_gemv(
    const uint16_t* __restrict__ x, const int8_t* __restrict__ q, const float* __restrict__ s_w,
    const float* __restrict__ bias, void* __restrict__ y, int y_bf16, int M, int N, int K) {
    __shared__ float red[GEMV_WARPS][MT][32][4];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int n0 = blockIdx.x * 16;
    const int m0 = blockIdx.y * (8 * MT);
    const int nchunks = (K + 63) >> 6;

    const int rowa = n0 + g, rowb = n0 + g + 8;
    const bool va = rowa < N, vb = rowb < N;
    const int8_t* qa = q + (int64_t)(va ? rowa : 0) * K + 16 * t;
    const int8_t* qb = q + (int64_t)(vb ? rowb : 0) * K + 16 * t;
    const uint16_t* xr[MT];
    bool xv[MT];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int m = m0 + mt * 8 + g;
        xv[mt] = m < M;
        xr[mt] = x + (int64_t)(xv[mt] ? m : 0) * K + 16 * t;
    }
    float acc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[mt][i] = 0.0f;

    const uint4 zero4 = make_uint4(0, 0, 0, 0);
    for (int c = warp; c < nchunks; c += GEMV_WARPS * UNROLL) {
        uint4 wa[UNROLL], wb[UNROLL], xa[UNROLL][MT][2];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int cc = c + GEMV_WARPS * u;
            const int kk = cc * 64 + 16 * t;
            const bool kin = (cc < nchunks) && (kk < K);
            wa[u] = (va && kin) ? ldg_stream(qa + cc * 64) : zero4;
            wb[u] = (vb && kin) ? ldg_stream(qb + cc * 64) : zero4;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const bool ok = xv[mt] && kin;
                xa[u][mt][0] = ok ? ldg_keep(xr[mt] + cc * 64) : zero4;
                xa[u][mt][1] = ok ? ldg_keep(xr[mt] + cc * 64 + 8) : zero4;
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const uint32_t wav[4] = {wa[u].x, wa[u].y, wa[u].z, wa[u].w};
            const uint32_t wbv[4] = {wb[u].x, wb[u].y, wb[u].z, wb[u].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t alo, ahi, blo, bhi;
                s8x4_to_bf16x4(wav[j], alo, ahi);
                s8x4_to_bf16x4(wbv[j], blo, bhi);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const uint4& xs = xa[u][mt][j >> 1];
                    const uint32_t b0 = (j & 1) ? xs.z : xs.x;
                    const uint32_t b1 = (j & 1) ? xs.w : xs.y;
                    mma_bf16_16816(acc[mt], alo, blo, ahi, bhi, b0, b1);
                }
            }
        }
    }

#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) red[warp][mt][lane][i] = acc[mt][i];
    __syncthreads();
    for (int e = threadIdx.x; e < MT * 128; e += GEMV_THREADS) {
        const int mt = e >> 7, l = (e >> 2) & 31, ci = e & 3;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < GEMV_WARPS; ++w) v += red[w][mt][l][ci];
        const int m = m0 + mt * 8 + 2 * (l & 3) + (ci & 1);
        const int n = n0 + (l >> 2) + 8 * (ci >> 1);
        if (m < M && n < N) {
            const float sv = __ldg(s_w + n);
            const float r = bias ? fmaf(v, sv, __ldg(bias + n)) : v * sv;
            if (y_bf16)
                reinterpret_cast<__nv_bfloat16*>(y)[(int64_t)m * N + n] = __float2bfloat16_rn(r);
            else
                reinterpret_cast<float*>(y)[(int64_t)m * N + n] = r;
        }
    }
}

// -------------------------------------------------------------------------- W8A8
// The static activation codes are computed in the kernel from the fp32 activations
// (SmolVLM-Q8 Q8Linear.forward lowers to one delegated linear_q8ta_q8csw call that takes x
// and its qparams): each lane quantizes exactly the 16 activations it feeds to its own MMA
// k slots, with the fp32 steps of q8_quantize_static (static_codes16), so the codes are the
// same bits without a pass through memory;
// acc = sum_k xq * q (int32, exact) for the first-pass codes (and the residual's);
// y[m, n] = s_w[n] * (s1 * (acc1 - z1 * wsum[n]) + s2 * (acc2 - z2 * wsum[n])) (+ bias[n]).
template <int MT, int UNROLL, bool TWO>
__global__ __launch_bounds__(GEMV_THREADS) void k_w8a8_gemv(
    const float* __restrict__ x, float s1, int z1, float s2, int z2,
    const int8_t* __restrict__ q, const int32_t* __restrict__ wsum,
    const float* __restrict__ s_w, const float* __restrict__ bias, float* __restrict__ y, int M,
    int N, int K) {
    __shared__ int red[GEMV_WARPS][TWO ? 2 : 1][MT][32][4];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int n0 = blockIdx.x * 16;
    const int m0 = blockIdx.y * (8 * MT);
    const int nchunks = (K + 63) >> 6;

    const int rowa = n0 + g, rowb = n0 + g + 8;
    const bool va = rowa < N, vb = rowb < N;
    const int8_t* qa = q + (int64_t)(va ? rowa : 0) * K + 16 * t;
    const int8_t* qb = q + (int64_t)(vb ? rowb : 0) * K + 16 * t;
    int64_t xoff[MT];
    bool xv[MT];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int m = m0 + mt * 8 + g;
        xv[mt] = m < M;
        xoff[mt] = (int64_t)(xv[mt] ? m : 0) * K + 16 * t;
    }
    int acc1[MT][4], acc2[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc1[mt][i] = acc2[mt][i] = 0;

    const float inv1 = __fdiv_rn(1.0f, s1);
    const float inv2 = TWO ? __fdiv_rn(1.0f, s2) : 0.0f;
    const float z1f = (float)z1, z2f = (float)z2;

    // Programmatic dependent launch: the previous kernel on the stream may have written x.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const uint4 zero4 = make_uint4(0, 0, 0, 0);
    for (int c = warp; c < nchunks; c += GEMV_WARPS * UNROLL) {
        uint4 wa[UNROLL], wb[UNROLL], x1[UNROLL][MT], x2[UNROLL][MT];
        float xf[UNROLL][MT][16];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int cc = c + GEMV_WARPS * u;
            const int kk = cc * 64 + 16 * t;
            const bool kin = (cc < nchunks) && (kk < K);
            wa[u] = (va && kin) ? ldg_stream(qa + cc * 64) : zero4;
            wb[u] = (vb && kin) ? ldg_stream(qb + cc * 64) : zero4;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const bool ok = xv[mt] && kin;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 f = ok ? ldg_f4(x + xoff[mt] + cc * 64 + 4 * i)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    xf[u][mt][4 * i] = f.x; xf[u][mt][4 * i + 1] = f.y;
                    xf[u][mt][4 * i + 2] = f.z; xf[u][mt][4 * i + 3] = f.w;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int cc = c + GEMV_WARPS * u;
            const bool kin = (cc < nchunks) && (cc * 64 + 16 * t < K);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                uint32_t o1[4], o2[4];
                static_codes16(xf[u][mt], s1, inv1, z1f, TWO, inv2, z2f, o1, o2);
                // rows past M and k past K contribute nothing (code 0, not z)
                const bool ok = xv[mt] && kin;
                x1[u][mt] = ok ? make_uint4(o1[0], o1[1], o1[2], o1[3]) : zero4;
                if (TWO) x2[u][mt] = ok ? make_uint4(o2[0], o2[1], o2[2], o2[3]) : zero4;
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint32_t a0 = j ? wa[u].z : wa[u].x, a2 = j ? wa[u].w : wa[u].y;
                const uint32_t a1 = j ? wb[u].z : wb[u].x, a3 = j ? wb[u].w : wb[u].y;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const uint32_t b0 = j ? x1[u][mt].z : x1[u][mt].x;
                    const uint32_t b1 = j ? x1[u][mt].w : x1[u][mt].y;
                    mma_s8_16832(acc1[mt], a0, a1, a2, a3, b0, b1);
                    if (TWO) {
                        const uint32_t c0 = j ? x2[u][mt].z : x2[u][mt].x;
                        const uint32_t c1 = j ? x2[u][mt].w : x2[u][mt].y;
                        mma_s8_16832(acc2[mt], a0, a1, a2, a3, c0, c1);
                    }
                }
            }
        }
    }

#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            red[warp][0][mt][lane][i] = acc1[mt][i];
            if (TWO) red[warp][TWO ? 1 : 0][mt][lane][i] = acc2[mt][i];
        }
    __syncthreads();
    for (int e = threadIdx.x; e < MT * 128; e += GEMV_THREADS) {
        const int mt = e >> 7, l = (e >> 2) & 31, ci = e & 3;
        int a1 = 0, a2 = 0;
#pragma unroll
        for (int w = 0; w < GEMV_WARPS; ++w) {
            a1 += red[w][0][mt][l][ci];
            if (TWO) a2 += red[w][TWO ? 1 : 0][mt][l][ci];
        }
        const int m = m0 + mt * 8 + 2 * (l & 3) + (ci & 1);
        const int n = n0 + (l >> 2) + 8 * (ci >> 1);
        if (m < M && n < N) {
            const int ws = __ldg(wsum + n);
            float v = s1 * (float)(a1 - z1 * ws);
            if (TWO) v += s2 * (float)(a2 - z2 * ws);
            y[(int64_t)m * N + n] =
                bias ? fmaf(__ldg(s_w + n), v, __ldg(bias + n)) : __ldg(s_w + n) * v;
        }
    }
}

// ---------------------------------------------------------------------- launchers
cudaError_t launch_w8a16_gemv(const uint16_t* x, const int8_t* q, const float* s_w,
                              const float* bias, void* y, int y_bf16, int64_t M, int64_t N, int K,
                              cudaStream_t st, int num_sms) {
    (void)num_sms;
    const unsigned gx = (unsigned)((N + 15) / 16);
    if (M <= 8) {
        dim3 grid(gx, 1);
        k_w8a16_gemv<1, 4><<<grid, GEMV_THREADS, 0, st>>>(x, q, s_w, bias, y, y_bf16, (int)M,
                                                          (int)N, K);
    } else {
        dim3 grid(gx, (unsigned)((M + 15) / 16));
        k_w8a16_gemv<2, 2><<<grid, GEMV_THREADS, 0, st>>>(x, q, s_w, bias, y, y_bf16, (int)M,
                                                          (int)N, K);
    }
    return cudaGetLastError();
}

template <int MT, int U, bool TWO>
static cudaError_t launch_w8a8_gemv_t(dim3 grid, const float* x, float s1,
                                      int z1, float s2, int z2, const int8_t* q,
                                      const int32_t* wsum, const float* s_w, const float* bias,
                                      float* y, int M, int N, int K, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(GEMV_THREADS);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_w8a8_gemv<MT, U, TWO>, x, s1, z1, s2, z2, q, wsum,
                              s_w, bias, y, M, N, K);
}

cudaError_t launch_w8a8_gemv(const float* x, float s1, int z1, int has2, float s2, int z2,
                             const int8_t* q, const int32_t* wsum, const float* s_w,
                             const float* bias, float* y, int64_t M, int64_t N, int K,
                             cudaStream_t st) {
    const unsigned gx = (unsigned)((N + 15) / 16);
    if (M <= 8) {
        dim3 grid(gx, 1);
        return has2 ? launch_w8a8_gemv_t<1, 4, true>(grid, x, s1, z1, s2, z2, q, wsum, s_w,
                                                     bias, y, (int)M, (int)N, K, st)
                    : launch_w8a8_gemv_t<1, 4, false>(grid, x, s1, z1, s2, z2, q, wsum,
                                                      s_w, bias, y, (int)M, (int)N, K, st);
    }
    dim3 grid(gx, (unsigned)((M + 15) / 16));
    return has2 ? launch_w8a8_gemv_t<2, 2, true>(grid, x, s1, z1, s2, z2, q, wsum, s_w,
                                                 bias, y, (int)M, (int)N, K, st)
                : launch_w8a8_gemv_t<2, 2, false>(grid, x, s1, z1, s2, z2, q, wsum, s_w,
                                                  bias, y, (int)M, (int)N, K, st);
}

}  // namespace q8

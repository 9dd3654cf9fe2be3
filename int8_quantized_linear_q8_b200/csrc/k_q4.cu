// k_q4.cu -- the 8da4w linear (dynamic per-row int8 activations x int4 group weights):
//
//   y[m, n] = s[m] * sum_g gs[n, g] * T_g[m, n],   T_g = sum_{k in g} (xq[m,k] - z[m]) q4[n,k]
//
// (pytorch/executorch PR #21229, linear_dq8ca_q4gsw).  The activation codes, scales and
// zero points come from the per-row qparams kernel (k_choose_qparams) run just before.
//
// Exactness: every group partial T_g is an exact int32 (|T_g| <= G * 255 * 8), the group
// scale is applied to it in fp32 and the groups are summed in fp32 -- the order of the
// page's definition.  The int4 codes enter the integer MMA as 16*q4 (the nibble moved to
// the top of a byte is its exact sign-extended value times 16), so every integer result
// carries a factor 16 that the epilogue removes with an exact power-of-two scale.
//
// Work split (M <= 16 activation rows per block of the grid's y dimension): a CTA of 4
// warps owns 16 weight rows; K is cut into chunks of 128 codes (64 packed bytes) taken
// by the warps in turn.  In a chunk, lane (g, t) reads packed word 4j+t of rows g and
// g+8 for step j = 0..3, so MMA step j covers the 32 consecutive codes [32j, 32j+32) of
// the chunk: a group of 32 is one step, of 64 two, of 128 or more the whole chunk.  The
// code sums sum_{k in g} q4 (for the zero-point term) come from a second MMA against an
// all-ones operand.
#include "q8_kernels.cuh"

namespace q8 {

constexpr int Q4_THREADS = 128;
constexpr int Q4_WARPS = 4;

// 4 packed bytes (8 codes k0..k7, low nibble = even k) -> 16*codes as int8:
// even word = [16k0, 16k2, 16k4, 16k6], odd word = [16k1, 16k3, 16k5, 16k7].
__device__ __forceinline__ void q4x8_to_s8x16(uint32_t w, uint32_t& even, uint32_t& odd) {
    even = (w << 4) & 0xF0F0F0F0u;
    odd = w & 0xF0F0F0F0u;
}

template <int MT>
__global__ __launch_bounds__(Q4_THREADS) void k_q4_gemv(
    const int8_t* __restrict__ xq, const float* __restrict__ s, const int32_t* __restrict__ z,
    const uint8_t* __restrict__ q4, const float* __restrict__ gs, int G, float* __restrict__ y,
    int M, int N, int K) {
    __shared__ float red[Q4_WARPS][MT][32][4];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int n0 = blockIdx.x * 16;
    const int m0 = blockIdx.y * (8 * MT);
    const int nchunks = K >> 7;                 // K % 128 == 0
    const int ngroups = K / G;
    const int seg = G < 128 ? G : 128;          // codes between two scalings
    const int seg_steps = seg >> 5;

    const int rowa = n0 + g, rowb = n0 + g + 8;
    const bool va = rowa < N, vb = rowb < N;
    const uint32_t* wa = reinterpret_cast<const uint32_t*>(q4 + (int64_t)(va ? rowa : 0) * (K / 2));
    const uint32_t* wb = reinterpret_cast<const uint32_t*>(q4 + (int64_t)(vb ? rowb : 0) * (K / 2));
    const float* gsa = gs + (int64_t)(va ? rowa : 0) * ngroups;
    const float* gsb = gs + (int64_t)(vb ? rowb : 0) * ngroups;

    // activation rows this lane feeds (B operand column g) and the zero points of the
    // two accumulator columns it owns (2t, 2t+1)
    int64_t xoff[MT];
    bool xv[MT];
    int zc[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int m = m0 + mt * 8 + g;
        xv[mt] = m < M;
        xoff[mt] = (int64_t)(xv[mt] ? m : 0) * K;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int mc = m0 + mt * 8 + 2 * t + h;
            zc[mt][h] = mc < M ? __ldg(z + mc) : 0;
        }
    }
    float acc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[mt][i] = 0.0f;

    const uint32_t ones = 0x01010101u;
    for (int c = warp; c < nchunks; c += Q4_WARPS) {
        uint32_t wra[4], wrb[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            wra[j] = va ? __ldg(wa + c * 16 + 4 * j + t) : 0u;
            wrb[j] = vb ? __ldg(wb + c * 16 + 4 * j + t) : 0u;
        }
        int p[MT][4], sm[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (j % seg_steps == 0) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) p[mt][i] = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) sm[i] = 0;
            }
            uint32_t ea, oa, eb, ob;
            q4x8_to_s8x16(wra[j], ea, oa);
            q4x8_to_s8x16(wrb[j], eb, ob);
            // k-slots 4t..4t+3 <- even codes, 4t+16..4t+19 <- odd codes of packed word
            mma_s8_16832(sm, ea, eb, oa, ob, ones, ones);
            const int kb = c * 128 + 32 * j + 8 * t;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                uint32_t b0 = 0, b1 = 0;
                if (xv[mt]) {
                    const uint2 v = __ldg(reinterpret_cast<const uint2*>(xq + xoff[mt] + kb));
                    b0 = __byte_perm(v.x, v.y, 0x6420);      // codes k+0, 2, 4, 6
                    b1 = __byte_perm(v.x, v.y, 0x7531);      // codes k+1, 3, 5, 7
                }
                mma_s8_16832(p[mt], ea, eb, oa, ob, b0, b1);
            }
            if ((j + 1) % seg_steps == 0) {
                // end of a scaling segment: T' = 16 * sum (xq - z) q4, exact in int32
                const int gidx = (c * 128 + 32 * j) / G;
                const float ga = va ? __ldg(gsa + gidx) : 0.0f;
                const float gb = vb ? __ldg(gsb + gidx) : 0.0f;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    acc[mt][0] += ga * (float)(p[mt][0] - zc[mt][0] * sm[0]);
                    acc[mt][1] += ga * (float)(p[mt][1] - zc[mt][1] * sm[1]);
                    acc[mt][2] += gb * (float)(p[mt][2] - zc[mt][0] * sm[2]);
                    acc[mt][3] += gb * (float)(p[mt][3] - zc[mt][1] * sm[3]);
                }
            }
        }
    }

#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) red[warp][mt][lane][i] = acc[mt][i];
    __syncthreads();
    for (int e = threadIdx.x; e < MT * 128; e += Q4_THREADS) {
        const int mt = e >> 7, l = (e >> 2) & 31, ci = e & 3;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < Q4_WARPS; ++w) v += red[w][mt][l][ci];
        const int m = m0 + mt * 8 + 2 * (l & 3) + (ci & 1);
        const int n = n0 + (l >> 2) + 8 * (ci >> 1);
        if (m < M && n < N) y[(int64_t)m * N + n] = __ldg(s + m) * (v * 0.0625f);
    }
}

cudaError_t launch_q4_gemv(const int8_t* xq, const float* s, const int32_t* z, const uint8_t* q4,
                           const float* gs, int G, float* y, int64_t M, int64_t N, int K,
                           cudaStream_t st) {
    const unsigned gx = (unsigned)((N + 15) / 16);
    if (M <= 8) {
        k_q4_gemv<1><<<dim3(gx, 1), Q4_THREADS, 0, st>>>(xq, s, z, q4, gs, G, y, (int)M, (int)N, K);
    } else {
        k_q4_gemv<2><<<dim3(gx, (unsigned)((M + 15) / 16)), Q4_THREADS, 0, st>>>(
            xq, s, z, q4, gs, G, y, (int)M, (int)N, K);
    }
    return cudaGetLastError();
}

}  // namespace q8

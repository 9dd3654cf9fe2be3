// k_gemm_tc.cu -- prefill-sized int8 GEMM on the 5th-generation tensor cores.
//
//   acc[m, n] = sum_k a[m, k] * b[n, k]        (int8 x int8 -> int32, exact)
//
// with three epilogues:
//   EPI_S32 : acc itself (the exported int32 GEMM);
//   EPI_W8A8: y = s_w[n] * s1 * (acc1 - z1 * wsum[n])                 (one pass);
//   EPI_TWO : y = s_w[n] * (s1 * (acc1 - z1 wsum[n]) + s2 * (acc2 - z2 wsum[n]))
//   (the two W8A8 forms add bias[n] once, when a bias is given)
//             where acc1 and acc2 come from the two activation-code tensors of the
//             two-pass residual and share every weight tile.
//
// Structure: persistent CTAs (one per SM), 6 warps.
//   warp 0   : TMA producer -- per 128-byte K step, the activation tile(s) (128 rows) and
//              the weight tile (BN rows) land in a 4-stage shared-memory ring, 128-byte
//              swizzled, signalled by an mbarrier with transaction bytes (the whole warp
//              runs the loop, lane 0 issues the copies).
//   warp 1   : allocates all 512 tensor-memory columns, then runs the issuing loop as a
//              whole warp, one elected lane issuing each
//              tcgen05.mma.kind::i8 (M=128, K=32) into an int32 accumulator in tensor
//              memory; tcgen05.commit releases each smem stage and, after the last K
//              step, hands the accumulator to the epilogue.  Accumulators are double-
//              buffered so the epilogue of one tile overlaps the main loop of the next.
//   warps 2-5: epilogue -- tcgen05.ld of 32 columns at a time (each warp reads its
//              32-lane quarter of tensor memory), zero-point term and scales in fp32;
//              each warp's 32 x 32 output chunk goes through a padded shared-memory tile
//              so that every store instruction covers 4 rows x 128 bytes.
// Weight tiles are 256, 160 or 128 rows (BN) for one pass, chosen on the host by rounds of
// tiles over the SMs, and 128 for the two-pass form (two accumulators per tile).
// Every wait is bounded (abort flag + status word), and tensor memory is released only
// after the issuing warp has seen all of its MMAs complete.
#include "q8_kernels.cuh"

namespace q8 {

// EPI_W8A8_N128 / _N160: the one-pass epilogue on 128- or 160-row weight tiles (for grids
// that 256-row tiles would leave unbalanced)
enum { EPI_S32 = 0, EPI_W8A8 = 1, EPI_TWO = 2, EPI_W8A8_N128 = 3, EPI_W8A8_N160 = 4 };

constexpr int TC_BM = 128;          // accumulator rows (= tensor-memory lanes)
constexpr int TC_BK = 128;          // bytes of K per stage (one 128-byte swizzle row)
constexpr int TC_UK = 32;           // K per tcgen05.mma.kind::i8
constexpr int TC_STAGES = 4;
constexpr int TC_THREADS = 192;
constexpr int TC_TMEM_COLS = 512;

template <int EPI>
struct TcCfg {
    static constexpr bool TWO = EPI == EPI_TWO;
    static constexpr int BN =                                  // weight rows per tile
        TWO || EPI == EPI_W8A8_N128 ? 128 : EPI == EPI_W8A8_N160 ? 160 : 256;
    static constexpr int A_TILES = TWO ? 2 : 1;
    static constexpr int A_BYTES = TC_BM * TC_BK;              // 16 KB
    static constexpr int B_BYTES = BN * TC_BK;
    static constexpr int STAGE_BYTES = A_TILES * A_BYTES + B_BYTES;   // 48 KB
    static constexpr int ACC_COLS = TWO ? 2 * BN : BN;         // per accumulator buffer
    static_assert(2 * ACC_COLS <= TC_TMEM_COLS, "tensor memory");
    static_assert(B_BYTES % 1024 == 0 && BN % 32 == 0 && BN <= 256, "tile shape");
    // + control (8 KB) + the epilogue's store-transpose tiles (4 warps x 32 x 36 floats)
    static constexpr size_t SMEM = (size_t)TC_STAGES * STAGE_BYTES + 8192 + 4 * 32 * 36 * 4;
};

struct TcEpi {
    float s1, s2;
    int z1, z2;
    const int32_t* wsum;
    const float* s_w;
    const float* bias;     // nullable
    float* y;
    int32_t* acc;
};

// ------------------------------------------------------------ tcgen05 wrappers
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of 128 bytes
// grouped by 8 (1024 bytes apart).  Leading offset unused for this layout (1), version 1.
__device__ __forceinline__ uint64_t tc_desc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor, kind::i8: signed A and B, int32 accumulator, both K-major.
__host__ __device__ constexpr uint32_t tc_idesc_i8(int M, int N) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
// Called by all 32 lanes of the issuing warp with the same operands (the issuing loop stays
// warp-uniform); one lane, picked by elect.sync, issues the instruction.
__device__ __forceinline__ void tc_mma_i8_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
    const uint32_t z = 0;
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(z), "r"(z),
        "r"(z), "r"(z)
        : "memory");
}
__device__ __forceinline__ void tc_commit_warp(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}"
        ::"r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// -------------------------------------------------------------------- the kernel
// BIAS: the W8A8 epilogues add ep.bias[n] (staged per tile like s_w and wsum).
template <int EPI, bool BIAS>
__global__ __launch_bounds__(TC_THREADS, 1) void k_gemm_tc(
    const __grid_constant__ CUtensorMap amap1, const __grid_constant__ CUtensorMap amap2,
    const __grid_constant__ CUtensorMap bmap, int M, int N, int K, TcEpi ep, int* status) {
    using C = TcCfg<EPI>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte swizzle atoms
    uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* ctrl = smem + (size_t)TC_STAGES * C::STAGE_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
    uint64_t* empty = full + TC_STAGES;
    uint64_t* tfull = empty + TC_STAGES;       // [2]
    uint64_t* tempty = tfull + 2;              // [2]
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* epi_sw = reinterpret_cast<float*>(ctrl + 1024);      // [2][256]
    int* epi_ws = reinterpret_cast<int*>(ctrl + 1024 + 2048);   // [2][256] (ends at 5 KB)
    float* epi_b = reinterpret_cast<float*>(ctrl + 5120);        // [2][256] (ends at 7 KB)
    float* epi_tile = reinterpret_cast<float*>(ctrl + 8192);     // [4 warps][32][36]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_m = (M + TC_BM - 1) / TC_BM;
    const int num_n = (N + C::BN - 1) / C::BN;
    const int tiles = num_m * num_n;
    const int nk = (K + TC_BK - 1) / TC_BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < TC_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TC_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // Programmatic dependent launch: the next kernel may start its set-up now; every
    // global access below waits for the previous kernel (its outputs may be our inputs).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // the whole warp runs the loop (warp-uniform); lane 0 issues the copies
        {
            if (lane == 0) {
                tma_prefetch_desc(&amap1);
                if (C::TWO) tma_prefetch_desc(&amap2);
                tma_prefetch_desc(&bmap);
            }
            int s = 0, it = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int m0 = (t % num_m) * TC_BM, n0 = (t / num_m) * C::BN;
                for (int kb = 0; kb < nk; ++kb) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, status, abort_flag));
                    if (!ok) break;
                    if (lane == 0) {
                        uint8_t* st = smem + (size_t)s * C::STAGE_BYTES;
                        mbar_expect_tx(&full[s], (uint32_t)C::STAGE_BYTES);
                        tma_load_2d(st, &amap1, kb * TC_BK, m0, &full[s]);
                        if (C::TWO) tma_load_2d(st + C::A_BYTES, &amap2, kb * TC_BK, m0, &full[s]);
                        tma_load_2d(st + C::A_TILES * C::A_BYTES, &bmap, kb * TC_BK, n0, &full[s]);
                    }
                    ++it;
                    if (++s == TC_STAGES) { s = 0; ph ^= 1u; }
                }
            }
            for (int i = max(0, it - TC_STAGES); i < it; ++i)
                mbar_drain(&full[i % TC_STAGES], (uint32_t)(i / TC_STAGES) & 1u, status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // the whole warp runs the loop (warp-uniform); one elected lane issues each op
        {
            constexpr uint32_t idesc = tc_idesc_i8(TC_BM, C::BN);
            int s = 0, acc = 0;
            uint32_t ph = 0, acc_ph = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                if (!__all_sync(0xffffffffu, mbar_wait(&tempty[acc], acc_ph ^ 1u, status, abort_flag)))
                    break;
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(acc * C::ACC_COLS);
                for (int kb = 0; kb < nk; ++kb) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&full[s], ph, status, abort_flag));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + (size_t)s * C::STAGE_BYTES);
                    const uint64_t a1 = tc_desc_sw128(st);
                    const uint64_t a2 = tc_desc_sw128(st + C::A_BYTES);
                    const uint64_t b = tc_desc_sw128(st + C::A_TILES * C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < TC_BK / TC_UK; ++k) {
                        // advance 32 bytes of K inside the swizzled rows: +2 in 16-byte units
                        const uint32_t accumulate = (kb | k) != 0;
                        tc_mma_i8_warp(d, a1 + 2 * k, b + 2 * k, idesc, accumulate);
                        if (C::TWO) tc_mma_i8_warp(d + C::BN, a2 + 2 * k, b + 2 * k, idesc, accumulate);
                    }
                    tc_commit_warp(&empty[s]);          // stage free once these MMAs finish
                    if (++s == TC_STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit_warp(&tfull[acc]);            // accumulator ready for the epilogue
                if (++acc == 2) { acc = 0; acc_ph ^= 1u; }
            }
            // all MMAs issued here are complete before tensor memory is released
            tc_commit_warp(mma_done);
            mbar_drain(mma_done, 0, status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                         // tensor-memory lane quarter
        const int row = q * 32 + lane;                  // accumulator row in the tile
        const int et = threadIdx.x - 64;                // 0..127
        int acc = 0;
        uint32_t acc_ph = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
            const int m0 = (t % num_m) * TC_BM, n0 = (t / num_m) * C::BN;
            if (EPI != EPI_S32) {
                // stage this tile's per-channel terms (double-buffered by accumulator)
                for (int i = et; i < C::BN; i += 128) {
                    const int n = n0 + i;
                    epi_sw[acc * 256 + i] = n < N ? __ldg(ep.s_w + n) : 0.0f;
                    epi_ws[acc * 256 + i] = n < N ? __ldg(ep.wsum + n) : 0;
                    if (BIAS) epi_b[acc * 256 + i] = n < N ? __ldg(ep.bias + n) : 0.0f;
                }
                named_bar_sync(2, 128);
            }
            // After an expired wait the loop keeps its shape (the named barrier above needs
            // all four warps) but does no more work.  `live` is warp-uniform because
            // tcgen05.ld is a warp-wide instruction.
            const bool ok = mbar_wait(&tfull[acc], acc_ph, status, abort_flag);
            const bool live = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            tc_fence_after();
            const int m = m0 + row;
            const uint32_t tbase =
                tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::ACC_COLS);
#pragma unroll 1
            for (int c = 0; live && c < C::BN / 32; ++c) {
                uint32_t r1[32];
                tc_ld32(tbase + c * 32, r1);
                const int nb = n0 + c * 32;
                if (EPI == EPI_S32) {
                    if (m < M) {
                        int32_t* out = ep.acc + (int64_t)m * N + nb;
                        if (nb + 32 <= N && (N & 3) == 0) {
#pragma unroll
                            for (int j = 0; j < 32; j += 4)
                                *reinterpret_cast<int4*>(out + j) =
                                    make_int4((int)r1[j], (int)r1[j + 1], (int)r1[j + 2],
                                              (int)r1[j + 3]);
                        } else {
                            for (int j = 0; j < 32; ++j)
                                if (nb + j < N) out[j] = (int)r1[j];
                        }
                    }
                } else {
                    float v[32];
                    const float* sw = epi_sw + acc * 256 + c * 32;
                    const int* ws = epi_ws + acc * 256 + c * 32;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        v[j] = ep.s1 * (float)((int)r1[j] - ep.z1 * ws[j]);
                    if (EPI == EPI_TWO) {
                        uint32_t r2[32];
                        tc_ld32(tbase + C::BN + c * 32, r2);
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            v[j] += ep.s2 * (float)((int)r2[j] - ep.z2 * ws[j]);
                    }
                    if (BIAS) {
                        const float* bb = epi_b + acc * 256 + c * 32;
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = fmaf(v[j], sw[j], bb[j]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] *= sw[j];
                    }
                    // Each thread holds one output row; written directly, every store
                    // instruction would touch 32 rows.  Transpose the warp's 32 x 32 chunk
                    // through shared memory (rows padded to 36 floats: conflict-free
                    // 16-byte accesses) so that each store covers 4 rows x 128 bytes.
                    float* tile = epi_tile + (warp - 2) * (32 * 36);
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4*>(tile + lane * 36 + j) =
                            make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
                    __syncwarp();
                    const int cc = (lane & 7) * 4;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = 4 * i + (lane >> 3);
                        const float4 w = *reinterpret_cast<const float4*>(tile + r * 36 + cc);
                        const int mr = m0 + q * 32 + r;
                        if (mr < M) {
                            float* out = ep.y + (int64_t)mr * N + nb + cc;
                            if (nb + cc + 4 <= N && (N & 3) == 0) {
                                *reinterpret_cast<float4*>(out) = w;
                            } else {
                                const float wv[4] = {w.x, w.y, w.z, w.w};
                                for (int u = 0; u < 4; ++u)
                                    if (nb + cc + u < N) out[u] = wv[u];
                            }
                        }
                    }
                    __syncwarp();                       // the tile is rewritten next chunk
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            if (++acc == 2) { acc = 0; acc_ph ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TC_TMEM_COLS)
                     : "memory");
    }
}

// ----------------------------------------------------------------------- host side
template <int EPI, bool BIAS = false>
static cudaError_t launch_tc(const int8_t* a1, const int8_t* a2, const int8_t* b, int M, int N,
                             int K, const TcEpi& ep, cudaStream_t st, int num_sms, int* status) {
    using C = TcCfg<EPI>;
    CUtensorMap ma1, ma2, mb;
    if (!make_tmap_u8_2d(&ma1, a1, M, K, TC_BK, TC_BM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_tmap_u8_2d(&ma2, a2 ? a2 : a1, M, K, TC_BK, TC_BM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_tmap_u8_2d(&mb, b, N, K, TC_BK, C::BN, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    cudaError_t e = ensure_dyn_smem<k_gemm_tc<EPI, BIAS>>((int)(C::SMEM + 1024));
    if (e != cudaSuccess) return e;
    const int tiles = ((M + TC_BM - 1) / TC_BM) * ((N + C::BN - 1) / C::BN);
    const int grid = tiles < num_sms ? tiles : num_sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = C::SMEM + 1024;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_gemm_tc<EPI, BIAS>, ma1, ma2, mb, M, N, K, ep, status);
}

cudaError_t launch_gemm_s8s8_s32_tc(const int8_t* a, const int8_t* b, int32_t* acc, int64_t M,
                                    int64_t N, int K, cudaStream_t st, int num_sms,
                                    int* status) {
    TcEpi ep = {};
    ep.acc = acc;
    return launch_tc<EPI_S32>(a, nullptr, b, (int)M, (int)N, K, ep, st, num_sms, status);
}

cudaError_t launch_w8a8_tc(const int8_t* xq1, const int8_t* xq2, float s1, int z1, int has2,
                           float s2, int z2, const int8_t* q, const int32_t* wsum,
                           const float* s_w, const float* bias, float* y, int64_t M, int64_t N,
                           int K, cudaStream_t st, int num_sms, int* status) {
    TcEpi ep = {};
    ep.bias = bias;
    ep.s1 = s1;
    ep.z1 = z1;
    ep.s2 = s2;
    ep.z2 = z2;
    ep.wsum = wsum;
    ep.s_w = s_w;
    ep.y = y;
#define TC_W8A8(EPI_, A2_)                                                                  \
    (bias ? launch_tc<EPI_, true>(xq1, A2_, q, (int)M, (int)N, K, ep, st, num_sms, status)  \
          : launch_tc<EPI_, false>(xq1, A2_, q, (int)M, (int)N, K, ep, st, num_sms, status))
    if (has2) return TC_W8A8(EPI_TWO, xq2);
    // Weight-tile rows: 256, 160 or 128, whichever gives the fewest rounds of tiles over
    // the SMs weighted by a tile's cost (taken as its rows plus a fixed part worth 128 rows:
    // pipeline fill and tail).  M = 2048, N = 2560: 160 rows, 2 rounds of 256 tiles instead
    // of 3 rounds of 320 128-row ones; the Llama prefill shapes keep 256 rows.
    const int64_t mt = (M + TC_BM - 1) / TC_BM;
    auto cost = [&](int64_t bn) {
        const int64_t tiles = mt * ((N + bn - 1) / bn);
        return (tiles + num_sms - 1) / num_sms * (bn + 128);
    };
    const int64_t c256 = cost(256), c160 = cost(160), c128 = cost(128);
    if (c256 <= c160 && c256 <= c128) return TC_W8A8(EPI_W8A8, nullptr);
    if (c160 <= c128) return TC_W8A8(EPI_W8A8_N160, nullptr);
    return TC_W8A8(EPI_W8A8_N128, nullptr);
#undef TC_W8A8
}

}  // namespace q8

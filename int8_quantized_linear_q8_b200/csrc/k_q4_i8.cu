// k_q4_i8.cu -- the 8da4w linear for prefill-sized M on the tcgen05 int8 tensor cores.
//
//   y[m, n] = s[m] * sum_g gs[n, g] * T_g[m, n],
//   T_g[m, n] = sum_{k in g} (xq[m,k] - z[m]) q4[n,k]
//             = sum_{k in g} xq[m,k] q4[n,k]  -  z[m] * Q_g[n],   Q_g[n] = sum_{k in g} q4[n,k]
//
// (ET-21229 PR description, linear_dq8ca_q4gsw: dynamic per-row int8 activations folded
// into the 4-bit group-symmetric weight GEMM, the zero-point term applied after the
// integer dot product.)
//
// Operands: A = weights, 16 * q4 as int8 ([-128, 112]), written into shared memory by
// converter warps from the packed nibbles that TMA brings (the low nibble of a byte moved
// to the high half is 16 * code in two's complement, so the expansion is a shift, masks
// and two byte permutes per 8 codes); B = the activation codes xq [M, K] int8 from
// k_choose_qparams, by TMA.  Both 128-byte swizzled, K-major.  tcgen05.mma.kind::i8
// (M = 128 weight rows, N = BN activation rows, K = 32) accumulates
// t = 16 * sum_{k in g} xq q4 per group in tensor memory (int32, |t| <= 2^22 for G <= 256).
// Weight rows are the tensor-memory lanes, so an epilogue thread owns one weight row n and
// its group scale is a per-thread scalar.
//
// Epilogue, per group and element, all exact: f = float(t) by adding t to the bits of
// 1.5 * 2^23 (|t| <= 2^22 keeps the result in [2^23, 2^24], where floats are the integers);
// c = z[m] * 16 * Q_g[n] + 1.5 * 2^23 (an integer below 2^24); 16 * T_g = f - c; then
// acc = fma(gs[n, g] / 16, 16 * T_g, acc), which rounds exactly like fma(gs, T_g, acc): the
// same fp32 result as an epilogue that receives T_g itself.  At the end of a tile
// y = s[m] * acc.  The group sums 16 * Q_g[n] come from k_q4_group_sums16 (one pass over
// the packed codes, launched before the GEMM).
//
// Structure (persistent, one CTA per SM, 16 warps): warp 0 TMA producer (activation codes
// and packed codes of a 128-K stage), warp 1 tensor-memory allocator and MMA issuer (a
// warp-uniform loop; elect.sync picks the lane that issues), warps 2-3 converters (two
// weight rows per thread per stage), warps 4-15 epilogue (three per tensor-memory lane
// quarter, a third of the BN = 192 columns each: two tensor-memory loads per group, and
// three warps per scheduler to overlap their latency).  One group's MMAs go into one of
// NBUF accumulator buffers of BN columns; tcgen05.commit hands a buffer to the epilogue
// and the epilogue's arrival hands it back.
#include "q8_kernels.cuh"

namespace q8 {

constexpr int QI_BM = 128;            // weight rows per tile (MMA M, tensor-memory lanes)
constexpr int QI_BK = 128;            // K per stage: one 128-byte row per operand row
constexpr int QI_UK = 32;             // K per tcgen05.mma.kind::i8
constexpr int QI_CONV_WARPS = 2;
constexpr int QI_EPI_PER_QUARTER = 3;           // epilogue warps per tensor-memory lane quarter
constexpr int QI_EPI_WARPS = 4 * QI_EPI_PER_QUARTER;
constexpr int QI_THREADS = (4 + QI_EPI_WARPS) * 32;

template <int BN>
struct QiCfg {
    static constexpr int A_BYTES = QI_BM * QI_BK;          // 16 KB of int8 weights
    static constexpr int B_BYTES = BN * QI_BK;             // activation codes
    static constexpr int Q_ROW = QI_BK / 2;                // packed bytes per weight row
    static constexpr int Q_BYTES = QI_BM * Q_ROW;          // 8 KB
    static constexpr int STAGE = A_BYTES + B_BYTES + Q_BYTES;
    static constexpr int STAGES = 196608 / STAGE < 6 ? 196608 / STAGE : 6;
    static constexpr int TX = B_BYTES + Q_BYTES;           // bytes the TMA copies deliver
    static constexpr int NBUF = 512 / BN;                  // accumulator buffers
    static constexpr int HC = BN / QI_EPI_PER_QUARTER;     // columns per epilogue warp
    static_assert(HC % 32 == 0, "epilogue column split");
    static constexpr size_t CTRL = 4096;                   // barriers + per-tile constants
    static constexpr size_t SMEM = (size_t)STAGES * STAGE + CTRL;
    static_assert(STAGES >= 2, "ring");
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms");
    static_assert(512 + 8 * BN <= (int)CTRL, "control region");
};

// ------------------------------------------------------------- tcgen05 wrappers

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of 128 bytes
// in groups of 8 (1024 bytes apart); leading offset unused for this layout (1), version 1.
__device__ __forceinline__ uint64_t qi_desc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor, kind::i8: s32 accumulator, A and B signed, K-major, M x N.
__host__ __device__ constexpr uint32_t qi_idesc_s8(int M, int N) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
// Called by all 32 lanes of the issuing warp with the same operands; one lane, picked by
// elect.sync, issues the instruction.
__device__ __forceinline__ void qi_mma_s8_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
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
__device__ __forceinline__ void qi_commit_warp(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}"
        ::"r"(smem_u32(bar))
        : "memory");
}
// 16 consecutive accumulator columns of this warp's lane quarter; waited for separately.
__device__ __forceinline__ void qi_ld_nowait(uint32_t taddr, uint32_t (&u)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
          "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]),
          "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
        : "r"(taddr));
}
// Completes this thread's outstanding tcgen05.ld; the registers are tied to the wait so
// that no use of them is scheduled before it.
__device__ __forceinline__ void qi_wait_ld(uint32_t (&u)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(u[0]), "+r"(u[1]), "+r"(u[2]), "+r"(u[3]), "+r"(u[4]), "+r"(u[5]),
                   "+r"(u[6]), "+r"(u[7]), "+r"(u[8]), "+r"(u[9]), "+r"(u[10]), "+r"(u[11]),
                   "+r"(u[12]), "+r"(u[13]), "+r"(u[14]), "+r"(u[15])::"memory");
}
// (a.x, a.y) = (a.x + b.x * c.x, a.y + b.y * c.y), one packed fp32 instruction, each lane
// rounded once like fmaf.
__device__ __forceinline__ void qi_fma2(float& ax, float& ay, float bx, float by, float cx,
                                        float cy) {
    asm("{\n\t.reg .b64 a, b, c;\n\t"
        "mov.b64 a, {%0, %1};\n\tmov.b64 b, {%2, %3};\n\tmov.b64 c, {%4, %5};\n\t"
        "fma.rn.f32x2 a, b, c, a;\n\tmov.b64 {%0, %1}, a;\n\t}"
        : "+f"(ax), "+f"(ay)
        : "f"(bx), "f"(by), "f"(cx), "f"(cy));
}
// (a.x, a.y) - (b.x, b.y), one packed fp32 instruction (round to nearest).
__device__ __forceinline__ void qi_sub2(float& ax, float& ay, float bx, float by) {
    asm("{\n\t.reg .b64 a, b;\n\t"
        "mov.b64 a, {%0, %1};\n\tmov.b64 b, {%2, %3};\n\t"
        "sub.rn.f32x2 a, a, b;\n\tmov.b64 {%0, %1}, a;\n\t}"
        : "+f"(ax), "+f"(ay)
        : "f"(bx), "f"(by));
}

// Packed word w (codes k..k+7, low nibble first) -> 16 * code as int8, in k order.
__device__ __forceinline__ void q4_word_to_s8x16(uint32_t w, uint32_t& o0, uint32_t& o1) {
    const uint32_t lo = (w << 4) & 0xF0F0F0F0u;    // 16 * codes k, k+2, k+4, k+6
    const uint32_t hi = w & 0xF0F0F0F0u;           // 16 * codes k+1, k+3, k+5, k+7
    o0 = __byte_perm(lo, hi, 0x5140);
    o1 = __byte_perm(lo, hi, 0x7362);
}

constexpr float kQiMagicF = 12582912.0f;          // 1.5 * 2^23
constexpr int kQiMagicI = 0x4B400000;             // its bits

// ------------------------------------------------------------- group sums
// sums16[n, g] = 16 * sum_{k in g} q4[n, k] as fp32 (an integer of magnitude <= 2^15).
__global__ __launch_bounds__(256) void k_q4_group_sums16(const uint8_t* __restrict__ q4,
                                                          int64_t groups, int ngroups, int K,
                                                          int G, float* __restrict__ sums16) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < groups;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = i / ngroups;
        const int g = (int)(i - n * ngroups);
        const uint8_t* p = q4 + n * (int64_t)(K / 2) + (int64_t)g * (G / 2);   // 16-byte aligned
        int acc = 0;
        for (int b = 0; b < G / 2; b += 16) {
            const uint4 v = *reinterpret_cast<const uint4*>(p + b);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t o0, o1;
                q4_word_to_s8x16(w[j], o0, o1);
                acc = __dp4a((int)o0, 0x01010101, acc);
                acc = __dp4a((int)o1, 0x01010101, acc);
            }
        }
        sums16[i] = (float)acc;
    }
}

// ------------------------------------------------------------- the GEMM
template <int BN>
__global__ __launch_bounds__(QI_THREADS, 1) void k_q4_gemm_i8(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap bmap,
    const float* __restrict__ gs, const float* __restrict__ sums16, const float* __restrict__ s,
    const int32_t* __restrict__ z, float* __restrict__ y, int G, int M, int N, int K,
    int* status) {
    using C = QiCfg<BN>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* ctrl = smem + (size_t)C::STAGES * C::STAGE;
    uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);      // TMA bytes (activations, codes)
    uint64_t* aready = full + C::STAGES;                     // int8 weight tile written
    uint64_t* empty = aready + C::STAGES;                    // stage's MMAs complete
    uint64_t* tfull = empty + C::STAGES;                     // [NBUF] group partials ready
    uint64_t* tempty = tfull + C::NBUF;                      // [NBUF] buffer drained
    uint64_t* mma_done = tempty + C::NBUF;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* s_tile = reinterpret_cast<float*>(ctrl + 512);    // [BN] s of the tile's rows
    float* z_tile = s_tile + BN;                             // [BN] z of the tile's rows

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_n = (N + QI_BM - 1) / QI_BM;
    const int num_m = (M + BN - 1) / BN;
    const int tiles = num_n * num_m;
    const int nk = K / QI_BK;                                 // K % 128 == 0
    const int steps_per_group = G / QI_UK;
    const int ngroups = K / G;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&aready[i], QI_CONV_WARPS);
            mbar_init(&empty[i], 1);
        }
        for (int a = 0; a < C::NBUF; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], QI_EPI_WARPS);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem_base = *tmem_slot;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        // the whole warp runs the loop (warp-uniform); lane 0 issues the copies
        if (lane == 0) {
            tma_prefetch_desc(&qmap);
            tma_prefetch_desc(&bmap);
        }
        const uint64_t keep = make_l2_policy_evict_last();   // activation codes: re-read
        int st = 0, it = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            const int n0 = (t / num_m) * QI_BM, m0 = (t % num_m) * BN;
            for (int kb = 0; kb < nk; ++kb) {
                ok = __all_sync(0xffffffffu, mbar_wait(&empty[st], ph ^ 1u, status, abort_flag));
                if (!ok) break;
                if (lane == 0) {
                    uint8_t* base = smem + (size_t)st * C::STAGE;
                    mbar_expect_tx(&full[st], (uint32_t)C::TX);
                    tma_load_2d_hint(base + C::A_BYTES, &bmap, kb * QI_BK, m0, &full[st], keep);
                    tma_load_2d(base + C::A_BYTES + C::B_BYTES, &qmap, kb * C::Q_ROW, n0,
                                &full[st]);
                }
                ++it;
                if (++st == C::STAGES) { st = 0; ph ^= 1u; }
            }
        }
        for (int i = max(0, it - C::STAGES); i < it; ++i)
            mbar_drain(&full[i % C::STAGES], (uint32_t)(i / C::STAGES) & 1u, status);
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        // the whole warp runs the loop; one elected lane issues each tcgen05 op
        constexpr uint32_t idesc = qi_idesc_s8(QI_BM, BN);
        int st = 0, buf = 0;
        uint32_t ph = 0, bph = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            int in_group = 0;                      // MMA step within the current group
            for (int kb = 0; kb < nk && ok; ++kb) {
                ok = __all_sync(0xffffffffu, mbar_wait(&aready[st], ph, status, abort_flag));
                if (!ok) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t base = smem_u32(smem + (size_t)st * C::STAGE);
                const uint64_t a0 = qi_desc_sw128(base);
                const uint64_t b0 = qi_desc_sw128(base + C::A_BYTES);
#pragma unroll
                for (int k = 0; k < QI_BK / QI_UK; ++k) {
                    if (in_group == 0) {
                        ok = __all_sync(0xffffffffu,
                                        mbar_wait(&tempty[buf], bph ^ 1u, status, abort_flag));
                        if (!ok) break;
                        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    }
                    // 32 bytes of K further inside the swizzled rows: +2 in 16-byte units
                    qi_mma_s8_warp(tmem_base + (uint32_t)(buf * BN), a0 + 2 * k, b0 + 2 * k, idesc,
                                   in_group != 0);
                    if (++in_group == steps_per_group) {
                        in_group = 0;
                        qi_commit_warp(&tfull[buf]);
                        if (++buf == C::NBUF) { buf = 0; bph ^= 1u; }
                    }
                }
                qi_commit_warp(&empty[st]);
                if (++st == C::STAGES) { st = 0; ph ^= 1u; }
            }
        }
        // all MMAs issued here are complete before tensor memory is released
        qi_commit_warp(mma_done);
        mbar_drain(mma_done, 0, status);
        __syncwarp();
    } else if (warp < 4) {
        // ---------------------------------------------------------------- converters
        // thread c converts weight rows c and c + 64 of the tile: its 64 packed bytes per row
        // -> 8 chunks of 16 int8 (16 * code), chunk j of row r at position j ^ (r % 8)
        const int c = (warp - 2) * 32 + lane;
        int st = 0;
        uint32_t ph = 0;
        bool live = true;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
            for (int kb = 0; kb < nk; ++kb) {
                const bool okw = mbar_wait(&full[st], ph, status, abort_flag);
                live = live && (__shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0);
                uint8_t* base = smem + (size_t)st * C::STAGE;
                if (live) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int r = c + 64 * h;
                        const uint32_t qrow =
                            smem_u32(base + C::A_BYTES + C::B_BYTES + r * C::Q_ROW);
                        uint4 qw[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) qw[u] = lds128(qrow + 16 * u);
                        const uint32_t arow = smem_u32(base + r * QI_BK);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            // chunk j: packed words 2j, 2j+1 (codes 16j .. 16j+15)
                            const uint4 v = qw[j >> 1];
                            const uint32_t w0 = (j & 1) ? v.z : v.x;
                            const uint32_t w1 = (j & 1) ? v.w : v.y;
                            uint32_t o[4];
                            q4_word_to_s8x16(w0, o[0], o[1]);
                            q4_word_to_s8x16(w1, o[2], o[3]);
                            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(
                                             arow + (uint32_t)((j ^ (r & 7)) << 4)),
                                         "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3])
                                         : "memory");
                        }
                    }
                }
                // make the generic-proxy writes visible to the tensor core, then hand over
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&aready[st]);
                if (++st == C::STAGES) { st = 0; ph ^= 1u; }
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        // warp w (4..15): lane quarter w % 4 of the weight rows, column third (w - 4) / 4
        const int q = warp & 3;
        const int blk = (warp - 4) >> 2;                  // this warp's column block
        const int et = threadIdx.x - 128;                 // 0 .. 32 * QI_EPI_WARPS - 1
        constexpr int HC = C::HC;
        int buf = 0;
        uint32_t bph = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
            const int n0 = (t / num_m) * QI_BM, m0 = (t % num_m) * BN;
            const int n = n0 + q * 32 + lane;             // this thread's weight row
            for (int j = et; j < BN; j += 32 * QI_EPI_WARPS) {
                const bool in = m0 + j < M;
                s_tile[j] = in ? __ldg(s + m0 + j) : 0.f;
                z_tile[j] = in ? (float)__ldg(z + m0 + j) : 0.f;
            }
            named_bar_sync(2, 32 * QI_EPI_WARPS);         // s_tile, z_tile written
            const int64_t rowg = (int64_t)(n < N ? n : 0) * ngroups;
            const float* gsr = gs + rowg;
            const float* qsr = sums16 + rowg;
            const float* zt = z_tile + blk * HC;
            float acc[HC];
#pragma unroll
            for (int j = 0; j < HC; ++j) acc[j] = 0.0f;
            bool live = true;
            // the next group's scale and code sum are loaded while this group is processed
            float gs_next = __ldg(gsr), qs_next = __ldg(qsr);
            for (int g = 0; g < ngroups; ++g) {
                const float gs16 = gs_next * 0.0625f;     // exact: a power-of-two scaling
                const float qsum = qs_next;
                if (g + 1 < ngroups) {
                    gs_next = __ldg(gsr + g + 1);
                    qs_next = __ldg(qsr + g + 1);
                }
                const bool okw = mbar_wait(&tfull[buf], bph, status, abort_flag);
                live = live && (__shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0);
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                if (live) {
                    const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) +
                                           (uint32_t)(buf * BN + blk * HC);
                    // 16-column chunks, double-buffered: the load of chunk c + 1 is in flight
                    // while chunk c is processed, so a group exposes one tensor-memory
                    // latency (two-chunk waits cost the kernel ~2300 cycles per group)
                    constexpr int CW = 16, NC = HC / CW;
                    uint32_t u[2][CW];
                    qi_ld_nowait(taddr, u[0]);
                    qi_wait_ld(u[0]);
#pragma unroll
                    for (int c0 = 0; c0 < NC; ++c0) {
                        if (c0 + 1 < NC) qi_ld_nowait(taddr + (c0 + 1) * CW, u[(c0 + 1) & 1]);
                        const uint32_t(&uc)[CW] = u[c0 & 1];
#pragma unroll
                        for (int j = 0; j < CW; j += 4) {
                            const float4 zz = *reinterpret_cast<const float4*>(zt + c0 * CW + j);
                            // c = z * 16 Q + 1.5 * 2^23, f = 1.5 * 2^23 + t (both exact)
                            float c0x = kQiMagicF, c0y = kQiMagicF, c1x = kQiMagicF,
                                  c1y = kQiMagicF;
                            qi_fma2(c0x, c0y, zz.x, zz.y, qsum, qsum);
                            qi_fma2(c1x, c1y, zz.z, zz.w, qsum, qsum);
                            float f0 = __int_as_float((int)uc[j] + kQiMagicI);
                            float f1 = __int_as_float((int)uc[j + 1] + kQiMagicI);
                            float f2 = __int_as_float((int)uc[j + 2] + kQiMagicI);
                            float f3 = __int_as_float((int)uc[j + 3] + kQiMagicI);
                            qi_sub2(f0, f1, c0x, c0y);          // 16 * T_g, exact
                            qi_sub2(f2, f3, c1x, c1y);
                            const int a = c0 * CW + j;
                            qi_fma2(acc[a], acc[a + 1], gs16, gs16, f0, f1);
                            qi_fma2(acc[a + 2], acc[a + 3], gs16, gs16, f2, f3);
                        }
                        if (c0 + 1 < NC) qi_wait_ld(u[(c0 + 1) & 1]);
                    }
                }
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[buf]);
                if (++buf == C::NBUF) { buf = 0; bph ^= 1u; }
            }
            if (live && n < N) {
#pragma unroll
                for (int j = 0; j < HC; ++j) {
                    const int m = m0 + blk * HC + j;
                    if (m < M) st_stream_f32(y + (int64_t)m * N + n, s_tile[blk * HC + j] * acc[j]);
                }
            }
            named_bar_sync(2, 32 * QI_EPI_WARPS);         // before s_tile is rewritten
        }
    }

    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(512)
                     : "memory");
    }
}

// ----------------------------------------------------------------------- host side


template <int BN>
static cudaError_t launch_qi(const int8_t* xq, const int32_t* z, const float* s,
                             const uint8_t* q4, const float* gs, const float* sums16, float* y,
                             int G, int M, int N, int K, cudaStream_t st, int num_sms,
                             int* status) {
    using C = QiCfg<BN>;
    CUtensorMap mq, mb;
    if (!make_tmap_u8_2d(&mq, q4, N, K / 2, C::Q_ROW, QI_BM, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (!make_tmap_u8_2d(&mb, xq, M, K, QI_BK, BN, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    cudaError_t e = ensure_dyn_smem<k_q4_gemm_i8<BN>>((int)(C::SMEM + 1024));
    if (e != cudaSuccess) return e;
    const int tiles = ((N + QI_BM - 1) / QI_BM) * ((M + BN - 1) / BN);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles < num_sms ? tiles : num_sms);
    cfg.blockDim = dim3(QI_THREADS);
    cfg.dynamicSmemBytes = C::SMEM + 1024;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_q4_gemm_i8<BN>, mq, mb, gs, sums16, s, z, y, G, M, N, K,
                              status);
}

cudaError_t launch_q4_group_sums16(const uint8_t* q4, int64_t N, int K, int G, float* sums16,
                                   cudaStream_t st, int num_sms) {
    const int ngroups = K / G;
    const int64_t groups = N * (int64_t)ngroups;
    int64_t blocks = (groups + 255) / 256;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_q4_group_sums16, q4, groups, ngroups, K, G, sums16);
}

cudaError_t launch_q4_gemm_i8(const int8_t* xq, const int32_t* z, const float* s,
                              const uint8_t* q4, const float* gs, const float* sums16, float* y,
                              int G, int64_t M, int64_t N, int K, cudaStream_t st, int num_sms,
                              int* status) {
    return launch_qi<192>(xq, z, s, q4, gs, sums16, y, G, (int)M, (int)N, K, st, num_sms,
                          status);
}

}  // namespace q8

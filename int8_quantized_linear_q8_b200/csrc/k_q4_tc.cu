// k_q4_tc.cu -- the 8da4w linear for prefill-sized M on the tcgen05 tensor cores.
//
//   y[m, n] = s[m] * sum_g gs[n, g] * T_g[m, n],   T_g = sum_{k in g} (xq[m,k] - z[m]) q4[n,k]
//
// The group scale gs[n, g] multiplies every group partial, so the integer sums must leave
// the tensor core once per group.  From an int8 MMA that costs several ALU operations per
// output element and group (conversion, zero-point term, scale; k_q4_i8.cu does it, and is
// used where it measured faster: few groups per row); here the operands enter a bf16 MMA
// as exact small integers instead -- the codes q4 in [-8, 7] and the shifted activation
// codes (xq - z) in [-255, 255] -- so every product is exact and each group partial is an
// integer below 2^24 (|T_g| <= 256 * 255 * 8), exact in the fp32 accumulator.  The
// epilogue then needs one fp32 multiply-add per element and group.
//
// Operands (prepared by the two kernels below, into the caller's workspace):
//   A = weights  bf16 [N, K]  (each int4 code as a bf16 integer)
//   B = acts     bf16 [M, K]  (xq - z per row, from k_choose_qparams_shifted)
// Swapped roles: the MMA's M dimension is the weight row n (tensor-memory lane), its N
// dimension the activation row m, so an epilogue thread owns one weight row and its
// group scales are per-thread scalars.
//
// Structure (persistent, one CTA per SM, 10 warps): warp 0 TMA producer (128-byte swizzle;
// a ring of 6 boxes of 64 K elements per operand, 128 weight rows and BN activation rows:
// 3 stages of two boxes for G >= 64, so that one barrier round covers 8 MMAs -- a wait
// between MMAs leaves the tensor pipe idle for a few hundred cycles -- or 6 stages of one
// box for G = 32, where a group hand-off comes every 2 MMAs anyway);
// warp 1 tensor-memory allocator and MMA issuer (kind::f16, M = 128, N = BN, K = 16; the
// whole warp runs the issuing loop, one elected lane issues) -- one group's MMAs go into
// one of NBUF accumulator buffers, tcgen05.commit hands it to the epilogue; warps 2-9
// epilogue (two per tensor-memory lane quarter): tcgen05.ld of the
// group partials, fp32 multiply-add with the group scale into per-thread registers, at
// the end of a tile y = s[m] * acc.
#include "q8_kernels.cuh"

namespace q8 {

// ------------------------------------------------------------- operand preparation

// Packed int4 codes [N, K/2] -> bf16 integers [N, K] (16 codes per thread step).
__global__ __launch_bounds__(256) void k_q4_expand_bf16(const uint8_t* __restrict__ q4,
                                                         int64_t n8, uint16_t* __restrict__ wb) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint2 p = __ldg(reinterpret_cast<const uint2*>(q4) + i);   // 16 codes
        const uint32_t w[2] = {p.x, p.y};
        uint32_t o[8];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int byte = (int)((w[h] >> (8 * b)) & 0xFFu);
                const int lo = (byte & 0x8) ? (byte & 0xF) - 16 : (byte & 0xF);
                const int hi = (byte & 0x80) ? ((byte >> 4) & 0xF) - 16 : ((byte >> 4) & 0xF);
                const uint32_t blo = __float_as_uint((float)lo) >> 16;   // exact in bf16
                const uint32_t bhi = __float_as_uint((float)hi) >> 16;
                o[h * 4 + b] = blo | (bhi << 16);
            }
        uint4* dst = reinterpret_cast<uint4*>(wb) + 2 * i;
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

// ----------------------------------------------------------------- the GEMM kernel
constexpr int QT_BM = 128;             // weight rows per tile (tensor-memory lanes)
constexpr int QT_BOXK = 64;            // bf16 K elements per TMA box (one 128-byte swizzle row)
constexpr int QT_RING = 6;             // TMA boxes per operand in flight (the ring's depth)
constexpr int Q4TC_WIDE_M = 2048;      // activation rows from which tiles are 256 rows wide
constexpr int Q4TC_WIDE_G = 64;        // ... for groups of at least this many codes
constexpr int QT_UK = 16;              // K per tcgen05.mma.kind::f16
constexpr int QT_EPI_WARPS = 8;       // two per tensor-memory lane quarter (column halves)
constexpr int QT_THREADS = (2 + QT_EPI_WARPS) * 32;
constexpr int QT_NBUF_MAX = 4;        // group accumulator buffers in tensor memory (<= 512 cols)

// KB boxes per operand and stage: 2 (8 MMAs per barrier round; 3 stages with 128-row
// tiles, 2 with 256) where a group spans at least 4 MMAs -- even with only two stages
// that beats 4 stages of one box (measured, 256-row tiles, G = 128: 576 -> 472 us); with
// G = 32 a group hand-off comes every 2 MMAs anyway and the deeper 6-stage ring of single
// boxes is faster.
// GPB groups per accumulator buffer: side by side (each its own accumulator), handed to
// the epilogue together -- one hand-off per GPB groups (G = 32 with 128-row tiles).
template <int BN, int KB, int GPB = 1>
struct QtCfg {
    static constexpr int KBOX = KB;
    static constexpr int BUFW = BN * GPB;                  // tensor-memory columns per buffer
    static constexpr int BK = QT_BOXK * KB;                // K elements per stage
    static constexpr int STAGE_SZ = (QT_BM + BN) * QT_BOXK * 2 * KB;
    // QT_RING / KB stages, as many as fit next to the control region (192 KB of ring)
    static constexpr int STAGES =
        (QT_RING / KB) * STAGE_SZ <= 196608 ? QT_RING / KB : 196608 / STAGE_SZ;
    static constexpr int A_BOX = QT_BM * QT_BOXK * 2;      // 16 KB
    static constexpr int B_BOX = BN * QT_BOXK * 2;
    static constexpr int A_BYTES = A_BOX * KB;
    static constexpr int B_BYTES = B_BOX * KB;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int NBUF = 512 / BUFW < QT_NBUF_MAX ? 512 / BUFW : QT_NBUF_MAX;
    static constexpr int TMEM_COLS = NBUF * BUFW < 32 ? 32 : NBUF * BUFW;
    static_assert(NBUF >= 2 && NBUF * BUFW <= 512, "tensor memory");
    static constexpr int HALF = BN / 2;                    // columns per epilogue warp
    static constexpr size_t SMEM = (size_t)STAGES * STAGE + 4096;
};

// acc.xy += g * r.xy as one packed fp32x2 multiply-add
__device__ __forceinline__ void ffma2(float& ax, float& ay, float g, float rx, float ry) {
    asm("{\n\t.reg .b64 p, q, c;\n\t"
        "mov.b64 p, {%2, %2};\n\tmov.b64 q, {%3, %4};\n\tmov.b64 c, {%0, %1};\n\t"
        "fma.rn.f32x2 c, p, q, c;\n\tmov.b64 {%0, %1}, c;\n\t}"
        : "+f"(ax), "+f"(ay)
        : "f"(g), "f"(rx), "f"(ry));
}

__host__ __device__ constexpr uint32_t qt_idesc_bf16(int M, int N) {
    // kind::f16: fp32 accumulator (bit 4), A and B bf16 (bits 7 and 10), both K-major
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint64_t qt_desc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// The MMA issuer is a whole warp: all 32 lanes run the issuing loop with the same values
// (its waits, counters and descriptors stay warp-uniform) and call these two with the same
// operands; one lane, picked by elect.sync, issues the instruction.  Run from a single lane
// inside `if (lane == 0)`, the same loop was divergent code and cost ~180 cycles per MMA
// (8 MMAs and their stage's waits took ~2100 cycles; halving the MMAs did not shorten it).
__device__ __forceinline__ void qt_mma_f16_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                uint32_t idesc, uint32_t accumulate) {
    const uint32_t z = 0;
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(z), "r"(z),
        "r"(z), "r"(z)
        : "memory");
}
__device__ __forceinline__ void qt_commit_warp(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}"
        ::"r"(smem_u32(bar))
        : "memory");
}
// Issue a 32-column tensor-memory load; the caller waits once for a batch of them.
__device__ __forceinline__ void qt_ld32_nowait(uint32_t taddr, uint32_t (&u)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
          "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]),
          "=r"(u[13]), "=r"(u[14]), "=r"(u[15]), "=r"(u[16]), "=r"(u[17]), "=r"(u[18]),
          "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]), "=r"(u[24]),
          "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]),
          "=r"(u[31])
        : "r"(taddr));
}
__device__ __forceinline__ void qt_ld32(uint32_t taddr, float (&r)[32]) {
    uint32_t u[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
          "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]),
          "=r"(u[13]), "=r"(u[14]), "=r"(u[15]), "=r"(u[16]), "=r"(u[17]), "=r"(u[18]),
          "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]), "=r"(u[24]),
          "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]),
          "=r"(u[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __uint_as_float(u[i]);
}

template <int BN, int KB, int GPB>
__global__ __launch_bounds__(QT_THREADS, 1) void k_q4_gemm_tc(
    const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
    const float* __restrict__ gs, const float* __restrict__ s, float* __restrict__ y, int G,
    int M, int N, int K, int* status) {
    using C = QtCfg<BN, KB, GPB>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* ctrl = smem + (size_t)C::STAGES * C::STAGE;
    uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;     // [NBUF] group accumulator ready
    uint64_t* tempty = tfull + C::NBUF;      // [NBUF] group accumulator drained
    uint64_t* mma_done = tempty + C::NBUF;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* s_tile = reinterpret_cast<float*>(ctrl + 512);      // [BN] activation-row scales
    static_assert(512 + 4 * BN <= 4096, "control region");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_n = (N + QT_BM - 1) / QT_BM;                  // weight-row tiles
    const int num_m = (M + BN - 1) / BN;                        // activation-row tiles
    const int tiles = num_n * num_m;
    const int nk = K / C::BK;                                   // K % 128 == 0
    const int steps_per_group = G / QT_UK;
    const int ngroups = K / G;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int a = 0; a < C::NBUF; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], QT_EPI_WARPS);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS)
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
        {
            if (lane == 0) {
                tma_prefetch_desc(&amap);
                tma_prefetch_desc(&bmap);
            }
            // Activation tiles are re-read by every weight tile: keep them in L2; weight
            // tiles are re-read only by the next few activation tiles; outputs stream out.
            const uint64_t keep = make_l2_policy_evict_last();
            const uint64_t drop = make_l2_policy_evict_first();
            int st = 0, it = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int n0 = (t / num_m) * QT_BM, m0 = (t % num_m) * BN;
                for (int kb = 0; kb < nk; ++kb) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&empty[st], ph ^ 1u, status, abort_flag));
                    if (!ok) break;
                    if (lane == 0) {
                        uint8_t* base = smem + (size_t)st * C::STAGE;
                        mbar_expect_tx(&full[st], (uint32_t)C::STAGE);
                        // the tensor maps view the bf16 matrices as bytes: K offset in bytes
#pragma unroll
                        for (int h = 0; h < C::KBOX; ++h) {
                            const int kx = (kb * C::BK + h * QT_BOXK) * 2;
                            tma_load_2d_hint(base + h * C::A_BOX, &amap, kx, n0, &full[st], drop);
                            tma_load_2d_hint(base + C::A_BYTES + h * C::B_BOX, &bmap, kx, m0,
                                             &full[st], keep);
                        }
                    }
                    ++it;
                    if (++st == C::STAGES) { st = 0; ph ^= 1u; }
                }
            }
            for (int i = max(0, it - C::STAGES); i < it; ++i)
                mbar_drain(&full[i % C::STAGES], (uint32_t)(i / C::STAGES) & 1u, status);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        // the whole warp runs the loop; one elected lane issues each tcgen05 op
        {
            constexpr uint32_t idesc = qt_idesc_bf16(QT_BM, BN);
            int st = 0, buf = 0;
            uint32_t ph = 0, bph = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                // MMA step within the current group (a running counter: this warp issues
                // every MMA of the CTA, so its loop must stay short -- a modulo per step
                // made the issue loop, not the tensor core, the limit)
                int in_group = 0;
                int gin = 0;                        // group within the current buffer
                for (int kb = 0; kb < nk && ok; ++kb) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&full[st], ph, status, abort_flag));
                    if (!ok) break;
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const uint32_t base = smem_u32(smem + (size_t)st * C::STAGE);
#pragma unroll
                    for (int k = 0; k < C::BK / QT_UK; ++k) {
                        // box k / 4 of each operand, 32-byte K step k % 4 inside its rows
                        constexpr int KPB = QT_BOXK / QT_UK;
                        const uint64_t a = qt_desc_sw128(base + (k / KPB) * C::A_BOX) + 2 * (k % KPB);
                        const uint64_t b =
                            qt_desc_sw128(base + C::A_BYTES + (k / KPB) * C::B_BOX) + 2 * (k % KPB);
                        if (in_group == 0 && gin == 0) {
                            // a new buffer: wait until the epilogue has drained it
                            ok = __all_sync(0xffffffffu,
                                            mbar_wait(&tempty[buf], bph ^ 1u, status, abort_flag));
                            if (!ok) break;
                            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                        }
                        qt_mma_f16_warp(tmem_base + (uint32_t)(buf * C::BUFW + gin * BN), a, b,
                                        idesc, in_group != 0);
                        if (++in_group == steps_per_group) {
                            in_group = 0;
                            if (++gin == GPB) {
                                gin = 0;
                                qt_commit_warp(&tfull[buf]);    // GPB group partials ready
                                if (++buf == C::NBUF) { buf = 0; bph ^= 1u; }
                            }
                        }
                    }
                    qt_commit_warp(&empty[st]);                 // stage free after these MMAs
                    if (++st == C::STAGES) { st = 0; ph ^= 1u; }
                }
            }
            qt_commit_warp(mma_done);
            mbar_drain(mma_done, 0, status);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        // warp w (2..9): lane quarter (w % 4) of the weight rows, column half (w - 2) / 4
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const int et = threadIdx.x - 64;        // 0 .. 32*QT_EPI_WARPS-1
        constexpr int HC = C::HALF;             // columns owned by this warp
        int buf = 0;
        uint32_t bph = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
            const int n0 = (t / num_m) * QT_BM, m0 = (t % num_m) * BN;
            const int n = n0 + q * 32 + lane;   // this thread's weight row
            for (int j = et; j < BN; j += 32 * QT_EPI_WARPS)
                s_tile[j] = (m0 + j < M) ? __ldg(s + m0 + j) : 0.f;
            const float* gsr = gs + (int64_t)(n < N ? n : 0) * ngroups;
            float acc[HC];
#pragma unroll
            for (int j = 0; j < HC; ++j) acc[j] = 0.0f;
            bool live = true;
            // Group scales stream in chunks of 16 groups, one chunk ahead of their use: a
            // group's MMAs take ~10^2 cycles, an L2 round trip several hundred.  With 128
            // columns per warp (256-row tiles, G >= 64: a group's MMAs take >= 512 cycles)
            // one scalar loaded a group ahead does, and leaves the registers to the sums.
            constexpr bool G1 = HC > 64;
            constexpr int GC = G1 ? 1 : 16;
            float gcur[GC], gnxt[GC];
            float gnext1 = G1 ? __ldg(gsr) : 0.f;
            auto load_chunk = [&](float (&dst)[GC], int g0) {
#pragma unroll
                for (int i = 0; i < GC; i += 4) {
                    // rows are 16-byte aligned only when ngroups % 4 == 0
                    if ((ngroups & 3) == 0 && g0 + i + 3 < ngroups) {
                        const float4 v = __ldg(reinterpret_cast<const float4*>(gsr + g0 + i));
                        dst[i] = v.x; dst[i + 1] = v.y; dst[i + 2] = v.z; dst[i + 3] = v.w;
                    } else {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            dst[i + u] = (g0 + i + u < ngroups) ? __ldg(gsr + g0 + i + u) : 0.f;
                    }
                }
            };
            if (!G1) load_chunk(gnxt, 0);
            for (int gb = 0; gb < ngroups; gb += GPB) {      // one hand-off per GPB groups
                const bool okw = mbar_wait(&tfull[buf], bph, status, abort_flag);
                live = live && (__shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0);
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
              for (int sub = 0; sub < GPB; ++sub) {
                const int gi = gb + sub;
                float gsel;
                if (G1) {
                    gsel = gnext1;
                    if (gi + 1 < ngroups) gnext1 = __ldg(gsr + gi + 1);
                } else {
                    if (gi % GC == 0) {
#pragma unroll
                        for (int i = 0; i < GC; ++i) gcur[i] = gnxt[i];
                        if (gi + GC < ngroups) load_chunk(gnxt, gi + GC);
                    }
                    gsel = gcur[0];
#pragma unroll
                    for (int i = 1; i < GC; ++i) gsel = (gi % GC == i) ? gcur[i] : gsel;
                }
                const float gcur_v = gsel;
                if (live) {
                    const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) +
                                           (uint32_t)(buf * C::BUFW + sub * BN + half * HC);
                    // 32-column chunks, up to two per tensor-memory wait (with 128 columns
                    // per warp one at a time: 128 fp32 sums already take the registers)
                    constexpr int NCH = HC / 32;
                    constexpr int LB = NCH <= 2 ? NCH : 1;
#pragma unroll
                    for (int c0 = 0; c0 < NCH; c0 += LB) {
                        uint32_t u[LB][32];
#pragma unroll
                        for (int c = 0; c < LB; ++c) qt_ld32_nowait(taddr + (c0 + c) * 32, u[c]);
                        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                        for (int c = 0; c < LB; ++c)
#pragma unroll
                            for (int j = 0; j < 32; j += 2)
                                ffma2(acc[(c0 + c) * 32 + j], acc[(c0 + c) * 32 + j + 1], gcur_v,
                                      __uint_as_float(u[c][j]), __uint_as_float(u[c][j + 1]));
                    }
                }
              }
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[buf]);
                if (++buf == C::NBUF) { buf = 0; bph ^= 1u; }
            }
            named_bar_sync(2, 32 * QT_EPI_WARPS);   // s_tile written by all epilogue threads
            if (live && n < N) {
#pragma unroll
                for (int j = 0; j < HC; ++j) {
                    const int m = m0 + half * HC + j;
                    if (m < M) st_stream_f32(y + (int64_t)m * N + n, s_tile[half * HC + j] * acc[j]);
                }
            }
            named_bar_sync(2, 32 * QT_EPI_WARPS);   // before s_tile is rewritten
        }
    }

    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(C::TMEM_COLS)
                     : "memory");
    }
}

// ------------------------------------------------- fused variant for small M (M <= 64)
//
// The same GEMM, but the weight operand is built inside the kernel: TMA brings the packed
// int4 rows (128 rows x 32 bytes per 64-K box, 4x fewer bytes than the bf16 matrix), and
// four converter warps write them into the 128-byte-swizzled bf16 A tile (thread r owns
// weight row r).  Each code becomes an exact bf16 integer in three operations per pair:
// the offset nibble v = nibble ^ 8 (= code + 8) is placed in the mantissa of 0x4300
// (bf16 128 + v, exact: the unit in the last place of [128, 256) is 1), and a bf16x2
// subtraction of 136 leaves the code.  The converters fence the async proxy and arrive on
// the stage's "A ready" barrier; the MMA issuer waits only on that barrier (the converters
// waited for the stage's TMA bytes, activations included).  No global bf16 weight copy.
// With few tiles (64 activation rows give N / 128 of them) K is split into S parts per
// tile, S chosen on the host to need the fewest rounds of (tile, part) units over the SMs;
// the parts write their partial sums to the workspace and k_q4_split_reduce, launched
// next, adds them in part order (the same sum on every run) and applies s[m].
constexpr int QF_CONV_WARPS = 4;
constexpr int QF_THREADS = (2 + QF_CONV_WARPS + QT_EPI_WARPS) * 32;

template <int BN, int KB>
struct QfCfg {
    static constexpr int KBOX = KB;
    static constexpr int BK = QT_BOXK * KB;
    static constexpr int A_BOX = QT_BM * QT_BOXK * 2;      // 16 KB of bf16 weight per box
    static constexpr int B_BOX = BN * QT_BOXK * 2;
    static constexpr int A_BYTES = A_BOX * KB;
    static constexpr int B_BYTES = B_BOX * KB;
    static constexpr int Q_ROW = QT_BOXK / 2 * KB;         // packed bytes per weight row
    static constexpr int Q_BYTES = QT_BM * Q_ROW;
    static constexpr int STAGE = A_BYTES + B_BYTES + Q_BYTES;
    static constexpr int STAGES = 196608 / STAGE < 6 ? 196608 / STAGE : 6;
    static constexpr int TX = B_BYTES + Q_BYTES;           // bytes the TMA copies deliver
    static constexpr int NBUF = 512 / BN < QT_NBUF_MAX ? 512 / BN : QT_NBUF_MAX;
    static constexpr int TMEM_COLS = NBUF * BN < 32 ? 32 : NBUF * BN;
    static constexpr int HALF = BN / 2;
    static constexpr size_t SMEM = (size_t)STAGES * STAGE + 4096;
    static_assert(STAGES >= 2, "ring");
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms");
};

// Packed word w (8 codes, low nibble first) -> 4 words of bf16 pairs (codes 2i, 2i+1)
__device__ __forceinline__ void q4_word_to_bf16(uint32_t w, uint32_t (&o)[4]) {
    const uint32_t v = w ^ 0x88888888u;                    // code + 8 per nibble
    const uint32_t lo = v & 0x0F0F0F0Fu, hi = (v >> 4) & 0x0F0F0F0Fu;
    const __nv_bfloat162 off = __halves2bfloat162(__ushort_as_bfloat16((unsigned short)0x4308),
                                                  __ushort_as_bfloat16((unsigned short)0x4308));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        // bytes [lo_i, -, hi_i, -] -> (128 + v) in both halves
        const uint32_t t = (__byte_perm(lo, hi, (uint32_t)(i | (i << 4) | ((4 + i) << 8) |
                                                            ((4 + i) << 12))) &
                            0x00FF00FFu) | 0x43004300u;
        __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&t);
        b = __hsub2(b, off);
        o[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
}

template <int BN, int KB>
__global__ __launch_bounds__(QF_THREADS, 1) void k_q4_gemm_fused(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap bmap,
    const float* __restrict__ gs, const float* __restrict__ s, float* __restrict__ y, int G,
    int M, int N, int K, int S, float* __restrict__ part, int* status) {
    // Work units: (tile, K-part); S parts per tile (K-split for grids with few tiles).  The
    // part boundaries fall on stage and group boundaries.  With S > 1 each unit leaves its
    // partial sums in `part` and k_q4_split_reduce, launched next, adds them in part order.
    using C = QfCfg<BN, KB>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* ctrl = smem + (size_t)C::STAGES * C::STAGE;
    uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);      // TMA bytes (activations, codes)
    uint64_t* aready = full + C::STAGES;                     // bf16 weight tile written
    uint64_t* empty = aready + C::STAGES;                    // stage's MMAs complete
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + C::NBUF;
    uint64_t* mma_done = tempty + C::NBUF;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* s_tile = reinterpret_cast<float*>(ctrl + 512);
    static_assert(512 + 4 * BN <= 4096, "control region");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_n = (N + QT_BM - 1) / QT_BM;
    const int num_m = (M + BN - 1) / BN;
    const int tiles = num_n * num_m;
    const int nk = K / C::BK;                                  // K % 128 == 0
    const int gstep = G > C::BK ? G / C::BK : 1;               // stages per split step
    const int nsplit = nk / gstep;
    const int units = tiles * S;
    // stages [kb0, kb1) of unit u
    auto unit_range = [&](int u, int& tile, int& kb0, int& kb1) {
        tile = u / S;
        const int pp = u - tile * S;
        kb0 = (pp * nsplit / S) * gstep;
        kb1 = ((pp + 1) * nsplit / S) * gstep;
    };
    const int steps_per_group = G / QT_UK;
    const int ngroups = K / G;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&aready[i], QF_CONV_WARPS);
            mbar_init(&empty[i], 1);
        }
        for (int a = 0; a < C::NBUF; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], QT_EPI_WARPS);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS)
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
        {
            if (lane == 0) {
                tma_prefetch_desc(&qmap);
                tma_prefetch_desc(&bmap);
            }
            const uint64_t keep = make_l2_policy_evict_last();   // activations: re-read
            const uint64_t drop = make_l2_policy_evict_first();  // weight codes
            int st = 0, it = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                int t, kb0, kb1;
                unit_range(u, t, kb0, kb1);
                const int n0 = (t / num_m) * QT_BM, m0 = (t % num_m) * BN;
                for (int kb = kb0; kb < kb1; ++kb) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&empty[st], ph ^ 1u, status, abort_flag));
                    if (!ok) break;
                    if (lane == 0) {
                        uint8_t* base = smem + (size_t)st * C::STAGE;
                        mbar_expect_tx(&full[st], (uint32_t)C::TX);
#pragma unroll
                        for (int h = 0; h < C::KBOX; ++h)
                            tma_load_2d_hint(base + C::A_BYTES + h * C::B_BOX, &bmap,
                                             (kb * C::BK + h * QT_BOXK) * 2, m0, &full[st], keep);
                        tma_load_2d_hint(base + C::A_BYTES + C::B_BYTES, &qmap, kb * C::BK / 2, n0,
                                         &full[st], drop);
                    }
                    ++it;
                    if (++st == C::STAGES) { st = 0; ph ^= 1u; }
                }
            }
            for (int i = max(0, it - C::STAGES); i < it; ++i)
                mbar_drain(&full[i % C::STAGES], (uint32_t)(i / C::STAGES) & 1u, status);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        // the whole warp runs the loop; one elected lane issues each tcgen05 op
        {
            constexpr uint32_t idesc = qt_idesc_bf16(QT_BM, BN);
            int st = 0, buf = 0;
            uint32_t ph = 0, bph = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                int t, kb0, kb1;
                unit_range(u, t, kb0, kb1);
                int in_group = 0;                  // MMA step within the current group
                for (int kb = kb0; kb < kb1 && ok; ++kb) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&aready[st], ph, status, abort_flag));
                    if (!ok) break;
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const uint32_t base = smem_u32(smem + (size_t)st * C::STAGE);
                    constexpr int MPS = C::BK / QT_UK;           // MMA steps per stage
                    constexpr int KPB = QT_BOXK / QT_UK;
                    if (KB > 1 && steps_per_group % MPS == 0) {
                        // groups are whole stages: one buffer check and at most one hand-off
                        // per stage, none between the MMAs (single-box stages only serve
                        // G = 32: never)
                        if (in_group == 0) {
                            ok = __all_sync(0xffffffffu,
                                            mbar_wait(&tempty[buf], bph ^ 1u, status, abort_flag));
                            if (!ok) break;
                            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                        }
                        const uint32_t d = tmem_base + (uint32_t)(buf * BN);
#pragma unroll
                        for (int k = 0; k < MPS; ++k) {
                            const uint64_t a =
                                qt_desc_sw128(base + (k / KPB) * C::A_BOX) + 2 * (k % KPB);
                            const uint64_t b =
                                qt_desc_sw128(base + C::A_BYTES + (k / KPB) * C::B_BOX) +
                                2 * (k % KPB);
                            qt_mma_f16_warp(d, a, b, idesc, (in_group | k) != 0);
                        }
                        in_group += MPS;
                        if (in_group == steps_per_group) {
                            in_group = 0;
                            qt_commit_warp(&tfull[buf]);
                            if (++buf == C::NBUF) { buf = 0; bph ^= 1u; }
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < MPS; ++k) {
                            const uint64_t a =
                                qt_desc_sw128(base + (k / KPB) * C::A_BOX) + 2 * (k % KPB);
                            const uint64_t b =
                                qt_desc_sw128(base + C::A_BYTES + (k / KPB) * C::B_BOX) +
                                2 * (k % KPB);
                            if (in_group == 0) {
                                ok = __all_sync(0xffffffffu, mbar_wait(&tempty[buf], bph ^ 1u,
                                                                       status, abort_flag));
                                if (!ok) break;
                                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                            }
                            qt_mma_f16_warp(tmem_base + (uint32_t)(buf * BN), a, b, idesc,
                                            in_group != 0);
                            if (++in_group == steps_per_group) {
                                in_group = 0;
                                qt_commit_warp(&tfull[buf]);
                                if (++buf == C::NBUF) { buf = 0; bph ^= 1u; }
                            }
                        }
                    }
                    qt_commit_warp(&empty[st]);
                    if (++st == C::STAGES) { st = 0; ph ^= 1u; }
                }
            }
            qt_commit_warp(mma_done);
            mbar_drain(mma_done, 0, status);
        }
        __syncwarp();
    } else if (warp < 2 + QF_CONV_WARPS) {
        // ---------------------------------------------------------------- converters
        // thread r: weight row r of the tile, its Q_ROW packed bytes -> 8 * KB 16-byte
        // chunks of bf16 codes, chunk c of box h at row r, position c ^ (r % 8)
        const int r = (warp - 2) * 32 + lane;
        int st = 0;
        uint32_t ph = 0;
        bool live = true;
        for (int u = blockIdx.x; u < units; u += gridDim.x) {
            int t, kb0, kb1;
            unit_range(u, t, kb0, kb1);
            for (int kb = kb0; kb < kb1; ++kb) {
                const bool okw = mbar_wait(&full[st], ph, status, abort_flag);
                live = live && (__shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0);
                uint8_t* base = smem + (size_t)st * C::STAGE;
                if (live) {
                    const uint32_t qrow = smem_u32(base + C::A_BYTES + C::B_BYTES + r * C::Q_ROW);
#pragma unroll
                    for (int h = 0; h < C::KBOX; ++h) {
                        uint4 qw[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u)
                            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                                         : "=r"(qw[u].x), "=r"(qw[u].y), "=r"(qw[u].z), "=r"(qw[u].w)
                                         : "r"(qrow + (uint32_t)(h * 32 + u * 16)));
                        const uint32_t words[8] = {qw[0].x, qw[0].y, qw[0].z, qw[0].w,
                                                   qw[1].x, qw[1].y, qw[1].z, qw[1].w};
                        const uint32_t arow = smem_u32(base + h * C::A_BOX + r * 128);
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            uint32_t o[4];
                            q4_word_to_bf16(words[c], o);
                            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(
                                             arow + (uint32_t)((c ^ (r & 7)) << 4)),
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
        // warp w (6..13): lane quarter w % 4 of the weight rows, column half (w - 6) / 4
        const int q = warp & 3;
        const int half = (warp - 2 - QF_CONV_WARPS) >> 2;
        const int et = threadIdx.x - 32 * (2 + QF_CONV_WARPS);
        constexpr int HC = C::HALF;
        int buf = 0;
        uint32_t bph = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x) {
            int t, kb0, kb1;
            unit_range(u, t, kb0, kb1);
            const int g0 = kb0 * C::BK / G, g1 = kb1 * C::BK / G;
            const int n0 = (t / num_m) * QT_BM, m0 = (t % num_m) * BN;
            const int n = n0 + q * 32 + lane;
            for (int j = et; j < BN; j += 32 * QT_EPI_WARPS)
                s_tile[j] = (m0 + j < M) ? __ldg(s + m0 + j) : 0.f;
            const float* gsr = gs + (int64_t)(n < N ? n : 0) * ngroups;
            float acc[HC];
#pragma unroll
            for (int j = 0; j < HC; ++j) acc[j] = 0.0f;
            bool live = true;
            // the next group's scale is loaded while this group is processed (a group takes
            // longer here than an L2 round trip); kept in scalar registers -- 16-group
            // chunks in arrays went to local memory in this kernel
            float gnext = (g0 < g1) ? __ldg(gsr + g0) : 0.f;
            for (int gi = g0; gi < g1; ++gi) {
                const float gcur_v = gnext;
                if (gi + 1 < g1) gnext = __ldg(gsr + gi + 1);
                const bool okw = mbar_wait(&tfull[buf], bph, status, abort_flag);
                live = live && (__shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0);
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                if (live) {
                    const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) +
                                           (uint32_t)(buf * BN + half * HC);
                    constexpr int NCH = HC / 32;
                    uint32_t u[NCH][32];
#pragma unroll
                    for (int c = 0; c < NCH; ++c) qt_ld32_nowait(taddr + c * 32, u[c]);
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                    for (int c = 0; c < NCH; ++c)
#pragma unroll
                        for (int j = 0; j < 32; j += 2)
                            ffma2(acc[c * 32 + j], acc[c * 32 + j + 1], gcur_v,
                                  __uint_as_float(u[c][j]), __uint_as_float(u[c][j + 1]));
                }
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[buf]);
                if (++buf == C::NBUF) { buf = 0; bph ^= 1u; }
            }
            named_bar_sync(2, 32 * QT_EPI_WARPS);
            const int row = q * 32 + lane;                   // weight row within the tile
            if (S > 1) {
                // this part's sums, [tile][part][column][row] (coalesced by row)
                float* mine = part + ((int64_t)t * S + (u - t * S)) * BN * QT_BM;
#pragma unroll
                for (int j = 0; j < HC; ++j) mine[(half * HC + j) * QT_BM + row] = acc[j];
            }
            if (S == 1 && live && n < N) {
#pragma unroll
                for (int j = 0; j < HC; ++j) {
                    const int m = m0 + half * HC + j;
                    if (m < M) st_stream_f32(y + (int64_t)m * N + n, s_tile[half * HC + j] * acc[j]);
                }
            }
            named_bar_sync(2, 32 * QT_EPI_WARPS);
        }
    }

    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(C::TMEM_COLS)
                     : "memory");
    }
}

// ----------------------------------------------------------------------- host side
static bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, int64_t rows, int64_t cols,
                              int box_cols, int box_rows) {
    // a bf16 [rows, cols] matrix is a uint8 [rows, 2*cols] matrix for the TMA unit
    return make_tmap_u8_2d(map, base, rows, cols * 2, box_cols * 2, box_rows,
                           CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int BN, int KB, int GPB = 1>
static cudaError_t launch_qt(const uint16_t* wb, const uint16_t* xz, const float* gs,
                             const float* s, float* y, int G, int M, int N, int K,
                             cudaStream_t st, int num_sms, int* status) {
    using C = QtCfg<BN, KB, GPB>;
    CUtensorMap ma, mb;
    if (!make_tmap_bf16_2d(&ma, wb, N, K, QT_BOXK, QT_BM)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_2d(&mb, xz, M, K, QT_BOXK, BN)) return cudaErrorInvalidValue;
    cudaError_t e = ensure_dyn_smem<k_q4_gemm_tc<BN, KB, GPB>>((int)(C::SMEM + 1024));
    if (e != cudaSuccess) return e;
    const int tiles = ((N + QT_BM - 1) / QT_BM) * ((M + BN - 1) / BN);
    const int grid = tiles < num_sms ? tiles : num_sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(QT_THREADS);
    cfg.dynamicSmemBytes = C::SMEM + 1024;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_q4_gemm_tc<BN, KB, GPB>, ma, mb, gs, s, y, G, M, N, K, status);
}

// y[m, n] = s[m] * sum over the S parts, in part order, of the fused GEMM's partial sums
// (layout [tile][part][column][row] with 128-row weight tiles and 64-row activation tiles).
__global__ __launch_bounds__(256) void k_q4_split_reduce(const float* __restrict__ part,
                                                          const float* __restrict__ s,
                                                          float* __restrict__ y, int M, int N,
                                                          int S) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int num_m = (M + 63) / 64;
    const int64_t total = (int64_t)M * N;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int m = (int)(i / N), n = (int)(i - (int64_t)m * N);
        const int t = (n / QT_BM) * num_m + m / 64;
        const float* p = part + ((int64_t)t * S * 64 + (m % 64)) * QT_BM + (n % QT_BM);
        float v = 0.0f;
        for (int pp = 0; pp < S; ++pp) v += __ldcg(p + (int64_t)pp * 64 * QT_BM);
        y[i] = __ldg(s + m) * v;
    }
}

// K-parts per tile of the fused GEMM: the count (at most 8) that needs the fewest rounds of
// (tile, part) units over the SMs, measured in whole tiles; ties go to fewer parts.
static int qf_split(int64_t M, int64_t N, int K, int G, int num_sms) {
    const int64_t tiles = ((N + QT_BM - 1) / QT_BM) * ((M + 63) / 64);
    const int bk = QT_BOXK * (G == 32 ? 1 : 2);
    const int nsplit = (K / bk) / (G > bk ? G / bk : 1);
    int best = 1;
    double best_cost = (double)((tiles + num_sms - 1) / num_sms);
    for (int sp = 2; sp <= 8 && sp <= nsplit; ++sp) {
        const double cost = (double)((tiles * sp + num_sms - 1) / num_sms) / sp + 0.02 * sp;
        if (cost < best_cost - 1e-9) { best = sp; best_cost = cost; }
    }
    return best;
}

size_t q4_fused_workspace_bytes(int64_t M, int64_t N, int K, int G, int num_sms) {
    const int sp = qf_split(M, N, K, G, num_sms);
    if (sp == 1) return 0;
    const int64_t tiles = ((N + QT_BM - 1) / QT_BM) * ((M + 63) / 64);
    return (size_t)(tiles * sp * 64 * QT_BM) * sizeof(float);
}

template <int BN, int KB>
static cudaError_t launch_qf(const uint8_t* q4, const uint16_t* xz, const float* gs,
                             const float* s, float* y, int G, int M, int N, int K, int sp,
                             float* part, cudaStream_t st, int num_sms, int* status) {
    using C = QfCfg<BN, KB>;
    CUtensorMap mq, mb;
    if (!make_tmap_u8_2d(&mq, q4, N, K / 2, C::Q_ROW, QT_BM, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (!make_tmap_bf16_2d(&mb, xz, M, K, QT_BOXK, BN)) return cudaErrorInvalidValue;
    cudaError_t e = ensure_dyn_smem<k_q4_gemm_fused<BN, KB>>((int)(C::SMEM + 1024));
    if (e != cudaSuccess) return e;
    const int units = ((N + QT_BM - 1) / QT_BM) * ((M + BN - 1) / BN) * sp;
    const int grid = units < num_sms ? units : num_sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(QF_THREADS);
    cfg.dynamicSmemBytes = C::SMEM + 1024;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_q4_gemm_fused<BN, KB>, mq, mb, gs, s, y, G, M, N, K, sp,
                              part, status);
}

// Up to 64 activation rows the weight is expanded inside the GEMM (no bf16 copy in HBM).
bool q4_tc_fused(int64_t M) { return M <= 64; }

// ws: q4_fused_workspace_bytes() bytes (the K-parts' partial sums).
cudaError_t launch_q4_gemm_fused(const uint8_t* q4, const uint16_t* xz, const float* gs,
                                 const float* s, float* y, int G, int64_t M, int64_t N, int K,
                                 void* ws, cudaStream_t st, int num_sms, int* status) {
    const int sp = qf_split(M, N, K, G, num_sms);
    float* part = (float*)ws;
    cudaError_t e =
        G == 32 ? launch_qf<64, 1>(q4, xz, gs, s, y, G, (int)M, (int)N, K, sp, part, st, num_sms,
                                   status)
                : launch_qf<64, 2>(q4, xz, gs, s, y, G, (int)M, (int)N, K, sp, part, st, num_sms,
                                   status);
    if (e != cudaSuccess || sp == 1) return e;
    cudaLaunchConfig_t cfg = {};
    const int64_t total = M * N;
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_q4_split_reduce, (const float*)part, s, y, (int)M, (int)N,
                              sp);
}

cudaError_t launch_q4_expand_bf16(const uint8_t* q4, int64_t N, int K, uint16_t* wb,
                                  cudaStream_t st, int num_sms) {
    const int64_t n8 = N * (int64_t)K / 16;       // 8-byte groups of packed codes
    int64_t blocks = (n8 + 255) / 256;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    k_q4_expand_bf16<<<(unsigned)blocks, 256, 0, st>>>(q4, n8, wb);
    return cudaGetLastError();
}

cudaError_t launch_q4_gemm_tc(const uint16_t* wb, const uint16_t* xz, const float* gs,
                              const float* s, float* y, int G, int64_t M, int64_t N, int K,
                              cudaStream_t st, int num_sms, int* status) {
    if (M <= 64)
        return G == 32 ? launch_qt<64, 1>(wb, xz, gs, s, y, G, (int)M, (int)N, K, st, num_sms, status)
                       : launch_qt<64, 2>(wb, xz, gs, s, y, G, (int)M, (int)N, K, st, num_sms, status);
    // 256 activation rows per tile where there are enough of them to keep the tiles
    // balanced over the SMs: each MMA does twice the work for the same per-group hand-off.
    // Not for small groups: the epilogue (128 columns per warp, one tensor-memory chunk at
    // a time, registers short) then falls behind the MMAs (G = 32: 1062 -> 1395 us).
    if (M >= Q4TC_WIDE_M && G >= Q4TC_WIDE_G)
        return launch_qt<256, 2>(wb, xz, gs, s, y, G, (int)M, (int)N, K, st, num_sms, status);
    // G = 32: two groups per accumulator buffer (K / 32 groups, a multiple of 4)
    return G == 32
               ? launch_qt<128, 1, 2>(wb, xz, gs, s, y, G, (int)M, (int)N, K, st, num_sms, status)
               : launch_qt<128, 2>(wb, xz, gs, s, y, G, (int)M, (int)N, K, st, num_sms, status);
}

}  // namespace q8

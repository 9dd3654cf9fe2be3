// k_q4_tma.cu -- the decode-sized 8da4w linear as a persistent, TMA-fed HBM stream.
//
//   y[m, n] = s[m] * sum_g gs[n, g] * T_g[m, n],   T_g = sum_{k in g} (xq[m,k] - z[m]) q4[n,k]
//
// (pytorch/executorch PR #21229, linear_dq8ca_q4gsw), for M <= 16 activation rows.  The
// packed int4 weight and its group scales are the large operands; the activation codes,
// scales and zero points come from the per-row qparams kernel launched just before.
//
// Structure (one CTA per SM, persistent over 16-row groups of the weight), as the W8A16
// stream of k_gemv_tma.cu:
//   * warp 8 (producer): one lane streams the CTA's rows through a ring of shared-memory
//     stages with 2-D TMA copies: a stage holds 16 rows x 1 KB of packed codes (2048 codes,
//     8 boxes of 128 bytes) and the same rows' 2048 / G group scales.  Boxes of 128 bytes
//     use the 128-byte swizzle (16-byte chunk c of row r stored at chunk c ^ (r % 8)), so the
//     8 rows a warp reads at once fall in different banks (G <= 64 scales likewise).  The weight
//     does not depend on the qparams kernel (launched without programmatic serialisation,
//     so everything before it has completed), so the stream starts at once; only the
//     consumers wait for the qparams kernel before they read the activation codes.
//   * warps 0-7 (consumers): stage the activation codes in shared memory in MMA-fragment
//     order, then take slabs w and w+8 (64 bytes = 128 codes each) of every stage.  Per MMA
//     step of 32 codes, lane (g, t) holds packed word 4j + t of rows g and g+8; the nibbles
//     become 16 * code as int8 in 3 ALU ops per 8 codes, and the int8 MMA (m16n8k32) gives
//     16 * sum xq * q4 for every 8 activation rows and, against an all-ones operand, 16 *
//     sum q4 for the zero-point term.  Both are exact int32; a group of G codes is one
//     segment of G / 32 steps (one slab for G >= 128), after which its partial is scaled by
//     gs in fp32.  After the last stage of a row group the 8 warps' sums meet in a rotating
//     shared-memory slot; the last warp to arrive applies s[m] / 16 and writes y.
#include "q8_kernels.cuh"

namespace q8 {

constexpr int QS_CONSUMERS = 8;
constexpr int QS_THREADS = (QS_CONSUMERS + 1) * 32;
constexpr int QS_SLABS = 16;                         // 64-byte slabs per stage
constexpr int QS_BOX = 128;                          // q4 box width (bytes), swizzled
constexpr int QS_Q4_BYTES = 16 * 64 * QS_SLABS;      // 16 rows x 1 KB = 2048 codes per row
constexpr int QS_CODES = 2 * 64 * QS_SLABS;          // codes per row and stage
constexpr int QS_SLOTS = 16;
constexpr int QS_MAX_SMEM = 227 * 1024;

struct QsSmem {
    int stages;
    uint32_t gs_bytes;                 // group-scale bytes of a stage (16 rows)
    uint32_t tx_bytes;                 // bytes the TMA copies of a stage deliver
    size_t ring, stage_bytes, xs, red, bars, total;
};

static __host__ __device__ inline QsSmem qs_layout(int M, int K, int G, int MT, int stages) {
    QsSmem L;
    L.stages = stages;
    L.gs_bytes = (uint32_t)(16 * (QS_CODES / G) * 4);
    L.tx_bytes = (uint32_t)QS_Q4_BYTES + L.gs_bytes;
    // stages start on 1024-byte boundaries: the swizzle pattern is tied to address bits
    L.stage_bytes = (size_t)QS_Q4_BYTES + (L.gs_bytes + 1023) / 1024 * 1024;
    L.ring = 0;
    L.xs = (size_t)stages * L.stage_bytes;
    const int nst = (K + QS_CODES - 1) / QS_CODES;
    const size_t xbytes = (size_t)M * nst * QS_CODES;           // one byte per code
    L.red = L.xs + (xbytes + 127) / 128 * 128;
    L.bars = L.red + (size_t)QS_SLOTS * MT * 128 * sizeof(float);
    L.total = L.bars + (size_t)2 * stages * sizeof(uint64_t) + (QS_SLOTS + 4) * sizeof(int);
    return L;
}

// D(16x8 s32) = A(16x32 s8) * B(32x8 s8), no accumulator input
__device__ __forceinline__ void mma_s8_16832_z(int (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    const int z = 0;
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(z));
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}
__device__ __forceinline__ float4 lds128f(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

template <int MT, int SEG>
__global__ __launch_bounds__(QS_THREADS, 1) void k_q4_tma(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap gmap,
    const int8_t* __restrict__ xq, const float* __restrict__ s, const int32_t* __restrict__ z,
    int G, float* __restrict__ y, int M, int N, int K, int stages, int* status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base (the launch adds the slack): swizzled TMA boxes need it
    uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const QsSmem L = qs_layout(M, K, G, MT, stages);
    uint8_t* ring = smem + L.ring;
    float* slots = reinterpret_cast<float*>(smem + L.red);          // [QS_SLOTS][MT][32][4]
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* empty = full + stages;
    int* cnt = reinterpret_cast<int*>(empty + stages);               // [QS_SLOTS]
    volatile int* abort_flag = cnt + QS_SLOTS;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nst = (K + QS_CODES - 1) / QS_CODES;                   // stages per row group
    const int RG = (N + 15) >> 4;
    const int rg0 = (int)((int64_t)RG * blockIdx.x / gridDim.x);
    const int rg1 = (int)((int64_t)RG * (blockIdx.x + 1) / gridDim.x);

    if (threadIdx.x == 0) {
        for (int i = 0; i < stages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], QS_CONSUMERS);
        }
        for (int i = 0; i < QS_SLOTS; ++i) cnt[i] = 0;
        *abort_flag = 0;
        fence_mbar_init();
    }
    for (int i = threadIdx.x; i < QS_SLOTS * MT * 128; i += QS_THREADS) slots[i] = 0.0f;
    __syncthreads();
    // Let the next kernel on the stream start its set-up now.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == QS_CONSUMERS) {
        // ------------------------------------------------------------- producer
        if (lane == 0) {
            tma_prefetch_desc(&qmap);
            tma_prefetch_desc(&gmap);
            const uint64_t pol = make_l2_policy_evict_first();     // weights are read once
            int it = 0, st_i = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int rg = rg0; rg < rg1 && ok; ++rg) {
                for (int st = 0; st < nst; ++st) {
                    if (!mbar_wait(&empty[st_i], ph ^ 1u, status, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* dst = ring + (size_t)st_i * L.stage_bytes;
                    mbar_expect_tx(&full[st_i], L.tx_bytes);
                    const int kb = st * (QS_CODES / 2);              // packed bytes
#pragma unroll
                    for (int j = 0; j < QS_Q4_BYTES / (16 * QS_BOX); ++j)
                        tma_load_2d_hint(dst + j * 16 * QS_BOX, &qmap, kb + j * QS_BOX, rg * 16,
                                         &full[st_i], pol);
                    // group scales: boxes of 128 bytes (swizzled) when a row has that many
                    const int gsr = (int)(L.gs_bytes / 16), gbox = gsr < 128 ? gsr : 128;
                    for (int j = 0; j < gsr / gbox; ++j)
                        tma_load_2d_hint(dst + QS_Q4_BYTES + j * 16 * gbox, &gmap,
                                         st * gsr + j * gbox, rg * 16, &full[st_i], pol);
                    ++it;
                    if (++st_i == stages) { st_i = 0; ph ^= 1u; }
                }
            }
            for (int i = max(0, it - stages); i < it; ++i)
                mbar_drain(&full[i % stages], (uint32_t)(i / stages) & 1u, status);
        }
        return;
    }

    // ----------------------------------------------------------------- consumers
    // The activation codes, scales and zero points are the qparams kernel's output.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int g = lane >> 2, t = lane & 3;
    const uint32_t xs = smem_u32(smem + L.xs);
    const int nsteps = nst * (QS_CODES / 32);                        // 32-code MMA steps
    {
        // xq [M, K] -> per step S, row m, lane t: the 8 codes 32S + 8t .. +8, even ones in
        // the first word and odd ones in the second (the k order of the weight fragments)
        // (batches of 8 loads per thread in flight before their stores)
        const int units = M * nsteps * 4;
        constexpr int UB = 8;
        for (int base = 0; base < units; base += UB * QS_CONSUMERS * 32) {
            uint2 v[UB];
#pragma unroll
            for (int i = 0; i < UB; ++i) {
                const int u = base + threadIdx.x + i * QS_CONSUMERS * 32;
                const int tt = u & 3, m = (u >> 2) % M, S = (u >> 2) / M;
                const int k = 32 * S + 8 * tt;
                v[i] = make_uint2(0u, 0u);
                if (u < units && k < K)
                    v[i] = __ldg(reinterpret_cast<const uint2*>(xq + (int64_t)m * K + k));
            }
#pragma unroll
            for (int i = 0; i < UB; ++i) {
                const int u = base + threadIdx.x + i * QS_CONSUMERS * 32;
                if (u < units) {
                    const uint32_t b0 = __byte_perm(v[i].x, v[i].y, 0x6420);
                    const uint32_t b1 = __byte_perm(v[i].x, v[i].y, 0x7531);
                    asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(xs + (uint32_t)(u * 8)),
                                 "r"(b0), "r"(b1)
                                 : "memory");
                }
            }
        }
    }
    // zero points of this lane's accumulator columns (activation rows 8mt + 2t + {0, 1})
    int zc[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int m = mt * 8 + 2 * t + h;
            zc[mt][h] = m < M ? __ldg(z + m) : 0;
        }
    named_bar_sync(1, QS_CONSUMERS * 32);

    // this lane's activation fragment of step S, row tile mt: xs + ((S*M + 8mt + g)*4 + t)*8
    bool x_live[MT];
    uint32_t x_lane[MT];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int m = mt * 8 + g;
        x_live[mt] = m < M;
        x_lane[mt] = xs + (uint32_t)((((x_live[mt] ? m : 0)) * 4 + t) * 8);
    }
    const uint32_t x_step = (uint32_t)(M * 32);                   // bytes per 32-code step
    constexpr int seg_steps = SEG;                                  // steps per scaling segment
    const uint32_t gs_row = L.gs_bytes / 16;                       // group-scale bytes per row
    const uint32_t ones = 0x01010101u;

    const uint32_t ring_u = smem_u32(ring);
    int st_i = 0, slot = 0;
    uint32_t ph = 0;
    for (int rg = rg0; rg < rg1; ++rg) {
        float acc[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[mt][i] = 0.0f;

        for (int st = 0; st < nst; ++st) {
            mbar_wait(&full[st_i], ph, status, abort_flag);          // on expiry: garbage
            const uint32_t sbase = ring_u + (uint32_t)(st_i * L.stage_bytes);
            // this lane's packed words: slab j (warp, warp+8) is half j%2 of box j/2; rows g
            // and g+8 (same swizzle, g = row % 8), byte 16*step + 4t of the half
            uint32_t wa[2][4], wb[2][4];
            float gsa[2][4], gsb[2][4];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int slab = warp + 8 * jj;
                const uint32_t rowa = sbase + (uint32_t)((slab >> 1) * 16 * QS_BOX + g * QS_BOX + 4 * t);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t chunk = (uint32_t)((((slab & 1) * 4 + j) ^ g) * 16);
                    wa[jj][j] = lds32(rowa + chunk);
                    wb[jj][j] = lds32(rowa + 8 * QS_BOX + chunk);
                }
                // group scales of the slab's segments (one per segment end)
                if (G == 32) {
                    // the slab's 4 groups are one 16-byte chunk of a swizzled 128-byte box
                    const int q = slab * 4;
                    const uint32_t ga = sbase + QS_Q4_BYTES + (uint32_t)((q >> 5) * 16 * 128 +
                                                                         g * 128 +
                                                                         (((q & 31) >> 2) ^ g) * 16);
                    const float4 va = lds128f(ga), vb = lds128f(ga + 8 * 128);
                    gsa[jj][0] = va.x; gsa[jj][1] = va.y; gsa[jj][2] = va.z; gsa[jj][3] = va.w;
                    gsb[jj][0] = vb.x; gsb[jj][1] = vb.y; gsb[jj][2] = vb.z; gsb[jj][3] = vb.w;
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        gsa[jj][j] = gsb[jj][j] = 0.0f;
                        if ((j + 1) % seg_steps == 0) {
                            const int q = (slab * 128 + 32 * j) / G;       // group in stage
                            uint32_t off;
                            if (G == 64)           // one swizzled 128-byte box per row
                                off = (uint32_t)(g * 128 + ((((q & 31) >> 2) ^ g) * 16) + 4 * (q & 3));
                            else                   // plain rows of gs_row bytes
                                off = (uint32_t)(g * gs_row + 4 * q);
                            const uint32_t ga = sbase + QS_Q4_BYTES + off;
                            gsa[jj][j] = lds_f32(ga);
                            gsb[jj][j] = lds_f32(ga + 8 * (G == 64 ? 128u : gs_row));
                        }
                    }
                }
            }
            uint2 xv[2][4][MT];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj)
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        const int S = st * (QS_CODES / 32) + (warp + 8 * jj) * 4 + j;
                        xv[jj][j][mt] = x_live[mt] ? lds64(x_lane[mt] + (uint32_t)S * x_step)
                                                   : make_uint2(0u, 0u);
                    }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st_i]);              // operands are in registers

            // Steps in order, the two slabs interleaved: every MMA accumulates into its
            // own chain (slab x row tile, plus the code sums), so consecutive MMAs do not
            // wait on each other.  A segment of SEG steps starts with a zero accumulator.
            int p[2][MT][4], sm[2][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    // 16 * codes as int8: even codes -> k-slots 4t.., odd codes -> 16 + 4t..
                    const uint32_t ea = (wa[jj][j] << 4) & 0xF0F0F0F0u, oa = wa[jj][j] & 0xF0F0F0F0u;
                    const uint32_t eb = (wb[jj][j] << 4) & 0xF0F0F0F0u, ob = wb[jj][j] & 0xF0F0F0F0u;
                    if (j % SEG == 0) {
                        mma_s8_16832_z(sm[jj], ea, eb, oa, ob, ones, ones);
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt)
                            mma_s8_16832_z(p[jj][mt], ea, eb, oa, ob, xv[jj][j][mt].x,
                                           xv[jj][j][mt].y);
                    } else {
                        mma_s8_16832(sm[jj], ea, eb, oa, ob, ones, ones);
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt)
                            mma_s8_16832(p[jj][mt], ea, eb, oa, ob, xv[jj][j][mt].x,
                                         xv[jj][j][mt].y);
                    }
                }
                if ((j + 1) % SEG == 0) {
                    // end of a segment: 16 * sum (xq - z) q4, exact in int32, times gs
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj)
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            acc[mt][0] += gsa[jj][j] * (float)(p[jj][mt][0] - zc[mt][0] * sm[jj][0]);
                            acc[mt][1] += gsa[jj][j] * (float)(p[jj][mt][1] - zc[mt][1] * sm[jj][1]);
                            acc[mt][2] += gsb[jj][j] * (float)(p[jj][mt][2] - zc[mt][0] * sm[jj][2]);
                            acc[mt][3] += gsb[jj][j] * (float)(p[jj][mt][3] - zc[mt][1] * sm[jj][3]);
                        }
                }
            }
            if (++st_i == stages) { st_i = 0; ph ^= 1u; }
        }

        // the 8 warps' sums meet in a rotating slot; the last warp scales and writes y
        float* sl = slots + (size_t)slot * MT * 128;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) atomicAdd(&sl[(mt * 32 + lane) * 4 + i], acc[mt][i]);
        __threadfence_block();
        __syncwarp();
        int prev = 0;
        if (lane == 0) prev = atomicAdd(&cnt[slot], 1);
        prev = __shfl_sync(0xffffffffu, prev, 0);
        if (prev == QS_CONSUMERS - 1) {
            __threadfence_block();
            float vv[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                volatile float* vp = &sl[(mt * 32 + lane) * 4];
#pragma unroll
                for (int i = 0; i < 4; ++i) vv[mt][i] = vp[i];
#pragma unroll
                for (int i = 0; i < 4; ++i) vp[i] = 0.0f;
            }
            __threadfence_block();
            __syncwarp();
            if (lane == 0) atomicExch(&cnt[slot], 0);
            const int n0 = rg * 16;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int m = mt * 8 + 2 * t + (i & 1);
                    const int n = n0 + g + 8 * (i >> 1);
                    if (m < M && n < N) y[(int64_t)m * N + n] = __ldg(s + m) * (vv[mt][i] * 0.0625f);
                }
        }
        if (++slot == QS_SLOTS) slot = 0;
    }
}

// ----------------------------------------------------------------------- host side

// Whether the stream takes this problem: M <= 16, whole 16-byte rows of group scales
// ((K / G) * 4 a multiple of 16) and the activation codes next to at least 4 stages.
bool q4_tma_fits(int64_t M, int64_t K, int G) {
    if (M < 1 || M > 16 || K % 128 != 0 || K % G != 0 || ((K / G) * 4) % 16 != 0) return false;
    const int MT = M <= 8 ? 1 : 2;
    return qs_layout((int)M, (int)K, G, MT, 4).total + 1024 <= (size_t)QS_MAX_SMEM;
}

template <int MT, int SEG>
static cudaError_t launch_qs(const CUtensorMap& qm, const CUtensorMap& gm, const int8_t* xq,
                             const float* s, const int32_t* z, int G, float* y, int M, int N,
                             int K, cudaStream_t st, int num_sms, int* status) {
    int stages = 8;    // must stay <= QS_SLOTS - 2
    while (stages > 4 && qs_layout(M, K, G, MT, stages).total + 1024 > (size_t)QS_MAX_SMEM)
        --stages;
    const QsSmem L = qs_layout(M, K, G, MT, stages);
    const size_t smem = L.total + 1024;                  // + alignment slack
    cudaError_t e = cudaFuncSetAttribute(k_q4_tma<MT, SEG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int RG = (N + 15) / 16;
    int grid = RG < num_sms ? RG : num_sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(QS_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_q4_tma<MT, SEG>, qm, gm, xq, s, z, G, y, M, N, K, stages,
                              status);
}

cudaError_t launch_q4_tma(const int8_t* xq, const float* s, const int32_t* z, const uint8_t* q4,
                          const float* gs, int G, float* y, int64_t M, int64_t N, int K,
                          cudaStream_t st, int num_sms, int* status) {
    CUtensorMap qm, gm;
    if (!make_tmap_u8_2d(&qm, q4, N, K / 2, QS_BOX, 16, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int gsr = (QS_CODES / G) * 4;                  // group-scale bytes per row and stage
    if (!make_tmap_u8_2d(&gm, gs, N, (int64_t)(K / G) * 4, gsr < 128 ? gsr : 128, 16,
                         gsr >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    // steps of 32 codes per scaling segment: G / 32, at most one slab (4)
    const int m = (int)M, n = (int)N;
    if (M <= 8) {
        if (G == 32) return launch_qs<1, 1>(qm, gm, xq, s, z, G, y, m, n, K, st, num_sms, status);
        if (G == 64) return launch_qs<1, 2>(qm, gm, xq, s, z, G, y, m, n, K, st, num_sms, status);
        return launch_qs<1, 4>(qm, gm, xq, s, z, G, y, m, n, K, st, num_sms, status);
    }
    if (G == 32) return launch_qs<2, 1>(qm, gm, xq, s, z, G, y, m, n, K, st, num_sms, status);
    if (G == 64) return launch_qs<2, 2>(qm, gm, xq, s, z, G, y, m, n, K, st, num_sms, status);
    return launch_qs<2, 4>(qm, gm, xq, s, z, G, y, m, n, K, st, num_sms, status);
}

}  // namespace q8

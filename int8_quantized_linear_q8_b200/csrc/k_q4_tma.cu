// k_q4_tma.cu -- the decode-sized 8da4w linear as a persistent, TMA-fed HBM stream.
//
//   y[m, n] = s[m] * sum_g gs[n, g] * T_g[m, n],   T_g = sum_{k in g} (xq[m,k] - z[m]) q4[n,k]
//
// (pytorch/executorch PR #21229, linear_dq8ca_q4gsw), for M <= 16 activation rows.  The
// packed int4 weight and its group scales are the large operands.  The per-row activation
// qparams (s, z, xq) = choose_qparams(x) are computed inside the kernel for a few rows (QP),
// else by the qparams kernel launched just before.
//
// Structure (one CTA per SM, persistent over 16-row groups of the weight), as the W8A16
// stream of k_gemv_tma.cu, with NC consumer warps (8 for up to 8 activation rows, 16 above):
//   * warp NC (producer): one lane streams the CTA's rows through a ring of shared-memory
//     stages with 2-D TMA copies: a stage holds 16 rows x 1 KB of packed codes (2048 codes,
//     8 boxes of 128 bytes) and the same rows' 2048 / G group scales.  Boxes of 128 bytes
//     use the 128-byte swizzle (16-byte chunk c of row r stored at chunk c ^ (r % 8)), so the
//     8 rows a warp reads at once fall in different banks (G <= 64 scales likewise).  After
//     the qparams kernel (launched normally, so everything before it has completed) the
//     weight cannot be pending, and the stream starts at once; with QP the whole CTA first
//     waits for the previous kernel, which may have written the weight.
//   * warps 0..NC-1 (consumers) stage the activation codes in shared memory in MMA-fragment
//     order.  With QP every CTA quantizes the rows itself: each row is read by 32 NC / M'
//     threads (M' = M rounded up to a power of two), its min and max are reduced, and s, z
//     and the codes follow from the same fp32 steps as the qparams kernel (min and max do not
//     depend on the order of reduction, so the codes are the same bits); CTA 0 also writes
//     s, z and the row-major codes to the caller's workspace.  Without QP the codes are
//     copied from the qparams kernel's output.  Then warp w takes slabs w, w + NC, ... (64
//     bytes = 128 codes each) of every stage.  Per MMA step of 32 codes, lane (g, t) holds
//     packed word 4j + t of rows g and g+8; the nibbles become 16 * code as int8 in 3 ALU
//     ops per 8 codes, and the int8 MMA (m16n8k32) gives 16 * sum xq * q4 for every 8
//     activation rows and, against an all-ones operand, 16 * sum q4 for the zero-point term.
//     Both are exact int32; a group of G codes is one segment of G / 32 steps (one slab for
//     G >= 128), after which its partial is scaled by gs in fp32.  After the last stage of a
//     row group each warp stores its partial sums in a rotating shared-memory slot; the last
//     warp to arrive adds the NC partials in warp order (no float atomics: the result is the
//     same on every run), applies s[m] / 16 and writes y.
#include "q8_kernels.cuh"

namespace q8 {

constexpr int QS_MAX_CONSUMERS = 16;                 // consumer warps: 8 or 16
constexpr int QS_SLABS = 16;                         // 64-byte slabs per stage
constexpr int QS_BOX = 128;                          // q4 box width (bytes), swizzled
constexpr int QS_Q4_BYTES = 16 * 64 * QS_SLABS;      // 16 rows x 1 KB = 2048 codes per row
constexpr int QS_CODES = 2 * 64 * QS_SLABS;          // codes per row and stage
constexpr int QS_SLOTS = 16;
constexpr int QS_MAX_SMEM = 227 * 1024;
// consumer warps: 8 for one 8-row activation tile, 16 for two (more MMAs per stage)
static constexpr int qs_nc(int MT) { return MT == 1 ? 8 : 16; }
constexpr int Q4_QP_MAX_M = 8;                       // rows quantized inside the stream

struct QsSmem {
    int stages;
    int nslots;                        // partial-sum slots (row groups in flight)
    uint32_t gs_bytes;                 // group-scale bytes of a stage (16 rows)
    uint32_t tx_bytes;                 // bytes the TMA copies of a stage deliver
    size_t ring, stage_bytes, xs, red, qp, bars, total;
};

static __host__ __device__ inline QsSmem qs_layout(int M, int K, int G, int MT, int stages,
                                                   int NC) {
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
    // A warp runs at most `stages` stages ahead of the slowest one, so at most
    // ceil(stages / nst) + 2 row groups have partial sums in flight.
    L.nslots = (stages + nst - 1) / nst + 2;
    if (L.nslots > QS_SLOTS) L.nslots = QS_SLOTS;
    L.qp = L.red + (size_t)L.nslots * NC * MT * 128 * sizeof(float);   // row stats, s, z
    L.bars = L.qp + (size_t)(2 * QS_MAX_CONSUMERS + 2 * 16) * sizeof(float);
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

// QP: x is read and (xq, s, z) are written (CTA 0); otherwise (xq, s, z) are read.
// NC consumer warps take 16 / NC slabs of every stage each.
template <int MT, int SEG, bool QP, int NC>
__global__ __launch_bounds__((NC + 1) * 32, 1) void k_q4_tma(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap gmap,
    const uint16_t* __restrict__ x, int8_t* __restrict__ xq, float* __restrict__ s,
    int32_t* __restrict__ z, int G, float* __restrict__ y, int M, int N, int K, int stages,
    int* status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base (the launch adds the slack): swizzled TMA boxes need it
    uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const QsSmem L = qs_layout(M, K, G, MT, stages, NC);
    uint8_t* ring = smem + L.ring;
    float* slots = reinterpret_cast<float*>(smem + L.red);   // [nslots][NC][MT][32][4]
    float* qred = reinterpret_cast<float*>(smem + L.qp);            // [NC][2]
    float* srow = qred + 2 * QS_MAX_CONSUMERS;                      // [16] activation scales
    int* zrow = reinterpret_cast<int*>(srow + 16);                  // [16] zero points
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* empty = full + stages;
    int* cnt = reinterpret_cast<int*>(empty + stages);               // [QS_SLOTS]
    volatile int* abort_flag = cnt + QS_SLOTS;

    constexpr int SPW = QS_SLABS / NC;                               // slabs per warp and stage
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nst = (K + QS_CODES - 1) / QS_CODES;                   // stages per row group
    const int RG = (N + 15) >> 4;
    const int rg0 = (int)((int64_t)RG * blockIdx.x / gridDim.x);
    const int rg1 = (int)((int64_t)RG * (blockIdx.x + 1) / gridDim.x);

    if (threadIdx.x == 0) {
        for (int i = 0; i < stages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], NC);
        }
        for (int i = 0; i < QS_SLOTS; ++i) cnt[i] = 0;
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // Let the next kernel on the stream start its set-up now.  With QP the previous kernel
    // may have written the weight or the activations: wait for it before any global read.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (QP) asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == NC) {
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
    // Without QP the activation codes, scales and zero points are the qparams kernel's output.
    if (!QP) asm volatile("griddepcontrol.wait;" ::: "memory");
    const int g = lane >> 2, t = lane & 3;
    const uint32_t xs = smem_u32(smem + L.xs);
    const int nsteps = nst * (QS_CODES / 32);                        // 32-code MMA steps
    if (QP) {
        // Activation qparams.  Row r belongs to the T = 256 / M' consecutive threads
        // [rT, rT + T); thread lt of them holds the 8-value chunks lt, lt + T, ... of the row.
        const int ctid = threadIdx.x;
        int Mp = 1;
        while (Mp < M) Mp <<= 1;
        const int T = NC * 32 / Mp, row = ctid / T, lt = ctid % T;
        const bool has_row = row < M;
        const int K8 = K >> 3;
        const int per = (K8 + T - 1) / T;                            // chunks per thread
        constexpr int QR = 8;                                        // loads in flight
        const uint16_t* xr = x + (int64_t)(has_row ? row : 0) * K;
        float mn = 0.0f, mx = 0.0f;                                  // the range includes 0
        auto range = [&](const uint4& u) {
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float a = bf16lo(w[j]), b = bf16hi(w[j]);
                mn = fminf(mn, fminf(a, b));
                mx = fmaxf(mx, fmaxf(a, b));
            }
        };
        // batches of QR loads in flight; chunks past the row read as zeros (no effect)
        auto load = [&](uint4 (&v)[QR], int r0) {
#pragma unroll
            for (int r = 0; r < QR; ++r) {
                const int i = lt + (r0 + r) * T;
                v[r] = (has_row && i < K8) ? ldg_keep(xr + 8 * i) : make_uint4(0u, 0u, 0u, 0u);
            }
        };
        uint4 v[QR];
        for (int r0 = 0; r0 < per; r0 += QR) {
            load(v, r0);
#pragma unroll
            for (int r = 0; r < QR; ++r) range(v[r]);
        }
        // reduce over the row's threads: lanes first, then the row's warps (T > 32)
#pragma unroll
        for (int o = 16; o; o >>= 1)
            if (o < T) {
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
        if (T > 32) {
            if (lane == 0) {
                qred[2 * warp] = mn;
                qred[2 * warp + 1] = mx;
            }
            named_bar_sync(1, NC * 32);
            for (int w = row * (T / 32); w < (row + 1) * (T / 32); ++w) {
                mn = fminf(mn, qred[2 * w]);
                mx = fmaxf(mx, qred[2 * w + 1]);
            }
        }
        float sr, zf;
        qparams_from_range(mn, mx, sr, zf);
        const float inv = __fdiv_rn(1.0f, sr);
        if (has_row && lt == 0) {
            srow[row] = sr;
            zrow[row] = __float2int_rn(zf);
            if (blockIdx.x == 0) {
                s[row] = sr;
                z[row] = __float2int_rn(zf);
            }
        }
        // codes of chunk i (k = 8i .. 8i+7) -> fragment unit ((i/4) * M + row) * 4 + i % 4:
        // even codes in the first word, odd ones in the second (the weight fragments' k order)
        auto codes = [&](const uint4& u, int i) {
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
            int c[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                c[2 * j] = act_code(bf16lo(w[j]), inv, zf);
                c[2 * j + 1] = act_code(bf16hi(w[j]), inv, zf);
            }
            const uint32_t unit = (uint32_t)((((i >> 2) * M + row) << 2) + (i & 3));
            asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(xs + unit * 8u),
                         "r"(pack4_s8(c[0], c[2], c[4], c[6])), "r"(pack4_s8(c[1], c[3], c[5], c[7]))
                         : "memory");
            if (blockIdx.x == 0)
                *reinterpret_cast<uint2*>(xq + (int64_t)row * K + 8 * i) =
                    make_uint2(pack4_s8(c[0], c[1], c[2], c[3]), pack4_s8(c[4], c[5], c[6], c[7]));
        };
        if (has_row) {
            if (per <= QR) {
#pragma unroll
                for (int r = 0; r < QR; ++r)
                    if (lt + r * T < K8) codes(v[r], lt + r * T);
            } else {
                for (int r0 = 0; r0 < per; r0 += QR) {
                    load(v, r0);
#pragma unroll
                    for (int r = 0; r < QR; ++r)
                        if (lt + (r0 + r) * T < K8) codes(v[r], lt + (r0 + r) * T);
                }
            }
        }
        // codes of the steps past K (the last stage's tail) are zero: units M*K/8 onwards
        for (int u = M * K8 + ctid; u < M * nsteps * 4; u += NC * 32)
            asm volatile("st.shared.v2.u32 [%0], {%1,%1};" ::"r"(xs + (uint32_t)u * 8u), "r"(0u)
                         : "memory");
    } else {
        // xq [M, K] -> per step S, row m, lane t: the 8 codes 32S + 8t .. +8, even ones in
        // the first word and odd ones in the second (the k order of the weight fragments)
        // (batches of 8 loads per thread in flight before their stores)
        const int units = M * nsteps * 4;
        constexpr int UB = 8;
        for (int base = 0; base < units; base += UB * NC * 32) {
            uint2 v[UB];
#pragma unroll
            for (int i = 0; i < UB; ++i) {
                const int u = base + threadIdx.x + i * NC * 32;
                const int tt = u & 3, m = (u >> 2) % M, S = (u >> 2) / M;
                const int k = 32 * S + 8 * tt;
                v[i] = make_uint2(0u, 0u);
                if (u < units && k < K)
                    v[i] = __ldg(reinterpret_cast<const uint2*>(xq + (int64_t)m * K + k));
            }
#pragma unroll
            for (int i = 0; i < UB; ++i) {
                const int u = base + threadIdx.x + i * NC * 32;
                if (u < units) {
                    const uint32_t b0 = __byte_perm(v[i].x, v[i].y, 0x6420);
                    const uint32_t b1 = __byte_perm(v[i].x, v[i].y, 0x7531);
                    asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(xs + (uint32_t)(u * 8)),
                                 "r"(b0), "r"(b1)
                                 : "memory");
                }
            }
        }
        if (threadIdx.x < M) {
            srow[threadIdx.x] = __ldg(s + threadIdx.x);
            zrow[threadIdx.x] = __ldg(z + threadIdx.x);
        }
    }
    named_bar_sync(1, NC * 32);
    // zero points of this lane's accumulator columns (activation rows 8mt + 2t + {0, 1})
    int zc[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int m = mt * 8 + 2 * t + h;
            zc[mt][h] = m < M ? zrow[m] : 0;
        }

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
            uint32_t wa[SPW][4], wb[SPW][4];
            float gsa[SPW][4], gsb[SPW][4];
#pragma unroll
            for (int jj = 0; jj < SPW; ++jj) {
                const int slab = warp + NC * jj;
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
            uint2 xv[SPW][4][MT];
#pragma unroll
            for (int jj = 0; jj < SPW; ++jj)
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        const int S = st * (QS_CODES / 32) + (warp + NC * jj) * 4 + j;
                        xv[jj][j][mt] = x_live[mt] ? lds64(x_lane[mt] + (uint32_t)S * x_step)
                                                   : make_uint2(0u, 0u);
                    }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st_i]);              // operands are in registers

            // Steps in order, the two slabs interleaved: every MMA accumulates into its
            // own chain (slab x row tile, plus the code sums), so consecutive MMAs do not
            // wait on each other.  A segment of SEG steps starts with a zero accumulator.
            int p[SPW][MT][4], sm[SPW][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int jj = 0; jj < SPW; ++jj) {
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
                    for (int jj = 0; jj < SPW; ++jj)
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

        // The warps' partial sums meet in a rotating slot: each warp stores its own, the
        // last to arrive adds them in warp order (the same sum on every run) and writes y.
        float* sl = slots + (size_t)slot * NC * MT * 128;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
            *reinterpret_cast<float4*>(&sl[((size_t)warp * MT + mt) * 128 + lane * 4]) =
                make_float4(acc[mt][0], acc[mt][1], acc[mt][2], acc[mt][3]);
        __threadfence_block();
        __syncwarp();
        int prev = 0;
        if (lane == 0) prev = atomicAdd(&cnt[slot], 1);
        prev = __shfl_sync(0xffffffffu, prev, 0);
        if (prev == NC - 1) {
            __threadfence_block();
            float vv[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                for (int i = 0; i < 4; ++i) vv[mt][i] = 0.0f;
                for (int w = 0; w < NC; ++w) {
                    const float4 v = lds128f(smem_u32(&sl[((size_t)w * MT + mt) * 128 + lane * 4]));
                    vv[mt][0] += v.x; vv[mt][1] += v.y; vv[mt][2] += v.z; vv[mt][3] += v.w;
                }
            }
            __syncwarp();
            if (lane == 0) atomicExch(&cnt[slot], 0);
            const int n0 = rg * 16;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int m = mt * 8 + 2 * t + (i & 1);
                    const int n = n0 + g + 8 * (i >> 1);
                    if (m < M && n < N) y[(int64_t)m * N + n] = srow[m] * (vv[mt][i] * 0.0625f);
                }
        }
        if (++slot == L.nslots) slot = 0;
    }
}

// ----------------------------------------------------------------------- host side

// Whether the stream quantizes the activation rows itself (one launch) rather than after
// the qparams kernel: every CTA reads all M rows twice, which pays off for a few rows only.
bool q4_tma_quantizes(int64_t M) { return M <= Q4_QP_MAX_M; }

// Whether the stream takes this problem: M <= 16, whole 16-byte rows of group scales
// ((K / G) * 4 a multiple of 16) and the activation codes next to at least 4 stages.
bool q4_tma_fits(int64_t M, int64_t K, int G) {
    if (M < 1 || M > 16 || K % 128 != 0 || K % G != 0 || ((K / G) * 4) % 16 != 0) return false;
    const int MT = M <= 8 ? 1 : 2;
    return qs_layout((int)M, (int)K, G, MT, 4, qs_nc(MT)).total + 1024 <= (size_t)QS_MAX_SMEM;
}

template <int MT, int SEG, bool QP, int NC>
static cudaError_t launch_qs(const CUtensorMap& qm, const CUtensorMap& gm, const uint16_t* x,
                             int8_t* xq, float* s, int32_t* z, int G, float* y, int M, int N,
                             int K, cudaStream_t st, int num_sms, int* status) {
    int stages = 8;    // must stay <= QS_SLOTS - 2
    while (stages > 4 && qs_layout(M, K, G, MT, stages, NC).total + 1024 > (size_t)QS_MAX_SMEM)
        --stages;
    const QsSmem L = qs_layout(M, K, G, MT, stages, NC);
    const size_t smem = L.total + 1024;                  // + alignment slack
    cudaError_t e = ensure_dyn_smem<k_q4_tma<MT, SEG, QP, NC>>((int)smem);
    if (e != cudaSuccess) return e;
    const int RG = (N + 15) / 16;
    int grid = RG < num_sms ? RG : num_sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3((NC + 1) * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_q4_tma<MT, SEG, QP, NC>, qm, gm, x, xq, s, z, G, y, M, N, K,
                              stages, status);
}

cudaError_t launch_q4_tma(const uint16_t* x, int8_t* xq, float* s, int32_t* z, bool qp,
                          const uint8_t* q4, const float* gs, int G, float* y, int64_t M,
                          int64_t N, int K, cudaStream_t st, int num_sms, int* status) {
    CUtensorMap qm, gm;
    if (!make_tmap_u8_2d(&qm, q4, N, K / 2, QS_BOX, 16, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int gsr = (QS_CODES / G) * 4;                  // group-scale bytes per row and stage
    if (!make_tmap_u8_2d(&gm, gs, N, (int64_t)(K / G) * 4, gsr < 128 ? gsr : 128, 16,
                         gsr >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    // steps of 32 codes per scaling segment: G / 32, at most one slab (4)
    const int m = (int)M, n = (int)N;
#define Q4_LAUNCH(MT_, SEG_)                                                                  \
    return qp ? launch_qs<MT_, SEG_, true, qs_nc(MT_)>(qm, gm, x, xq, s, z, G, y, m, n, K,   \
                                                       st, num_sms, status)                  \
              : launch_qs<MT_, SEG_, false, qs_nc(MT_)>(qm, gm, x, xq, s, z, G, y, m, n, K,  \
                                                        st, num_sms, status)
    if (M <= 8) {
        if (G == 32) Q4_LAUNCH(1, 1);
        if (G == 64) Q4_LAUNCH(1, 2);
        Q4_LAUNCH(1, 4);
    }
    if (G == 32) Q4_LAUNCH(2, 1);
    if (G == 64) Q4_LAUNCH(2, 2);
    Q4_LAUNCH(2, 4);
#undef Q4_LAUNCH
}

}  // namespace q8

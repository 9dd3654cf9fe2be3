// k_gemv_tma.cu -- the decode-sized W8A16 linear as a persistent, TMA-fed HBM stream.
//
//   y[m, n] = s_w[n] * sum_k x[m, k] * q[n, k]      (M <= 16 activation rows)
//
// The int8 weight q[N, K] is the only large operand: the kernel exists to move it from
// HBM at full bandwidth and to spend as few instructions as possible per byte.
//
// Structure (one CTA per SM, persistent over 16-row groups of q):
//   * warp 8 (producer): one lane streams the CTA's rows through a ring of shared-memory
//     stages with 2-D TMA copies.  A stage holds 16 rows x 1024 bytes of K, as 4 boxes of
//     [16 rows][256 bytes] (boxes 64 bytes wide stream at about half the rate); stage
//     readiness is an mbarrier with transaction bytes, stage release an mbarrier the
//     consumer warps arrive on.
//   * warps 0-7 (consumers): before the first stage they stage the activations x [M, K]
//     (bf16) in MMA-fragment order, each lane exactly the fragments it will feed to its own
//     MMAs.  When they fit (32 * stages-per-row-group * ceil(M/8) <= 512 columns) they go
//     to tensor memory, which this kernel does not otherwise use: warp w owns TMEM lanes
//     32*(w%4).. and half the columns, and reads its fragments back with tcgen05.ld, so the
//     shared-memory port carries only the weight stream and the whole ring is free for
//     stages.  Otherwise they go to shared memory (at most 128 KB).  Warp w then takes
//     slabs w and w+8 (64 bytes of K each) of every stage, converts the int8 codes to bf16
//     in registers (exact, 7 ALU ops per 4 codes) and accumulates with the warp-level bf16
//     MMA (fp32 accumulate).  After the last stage of a row group the 8 partial sums are
//     added into a rotating shared-memory slot; the last warp to arrive scales, rounds
//     once to the output type and writes y.  No barrier is needed between warps.
//   * partial stages (K not a multiple of 1024) are handled without branches: every box
//     of a stage is always loaded (columns past K read as zeros) and the staged
//     activations are zero-padded to a whole number of stages.
//
// x fragments are stored as two planes of 16-byte pieces in lane order (conflict-free
// loads); weight rows are 256 bytes apart, so a 16-byte load phase (2 rows x 4 lanes) has a
// 2-way bank conflict, well within the shared-memory bandwidth this stream needs.
#include "q8_kernels.cuh"

namespace q8 {

#ifndef WT_CONSUMERS_DEF
#define WT_CONSUMERS_DEF 8
#endif
constexpr int WT_CONSUMERS = WT_CONSUMERS_DEF;          // consumer warps
constexpr int WT_THREADS = (WT_CONSUMERS + 1) * 32;     // + producer warp
constexpr int WT_BOX = 256;                             // TMA box width (bytes of K)
// Stage geometry: a stage is 16 rows x SL slabs of 64 bytes of K (SL = 16 or 32).
#define WT_GEOMETRY(SL_)                                                                   \
    constexpr int WT_SLABS = (SL_);                    /* 64-byte slabs per stage */      \
    constexpr int WT_SPW = WT_SLABS / WT_CONSUMERS;    /* slabs per consumer warp */      \
    constexpr int WT_BOXES = WT_SLABS * 64 / WT_BOX;   /* TMA boxes per stage */          \
    constexpr int WT_STAGE_BYTES = 16 * 64 * WT_SLABS;                                    \
    static_assert(WT_SPW * WT_CONSUMERS == WT_SLABS && WT_CONSUMERS % 4 == 0, "slab split"); \
    (void)WT_SPW;                                                                          \
    (void)WT_BOXES;                                                                        \
    (void)WT_STAGE_BYTES
constexpr int WT_MAX_SMEM = 227 * 1024;
constexpr int WT_SLOTS = 16;                            // most partial-sum slots in flight

struct WtSmem {
    int stages;
    int nslots;                        // partial-sum slots (row groups in flight)
    size_t ring, xs, red, sws, sbias, bars, total;
};

// Rows of q a CTA may own (its s_w slice is staged in shared memory).
constexpr int WT_MAX_ROWS = 1024;

template <int SL>
static __host__ __device__ inline WtSmem wt_layout(int M, int K, int MT, int stages, bool xt,
                                                   bool bias = false) {
    WT_GEOMETRY(SL);
    WtSmem L;
    L.stages = stages;
    L.ring = 0;
    L.xs = (size_t)stages * WT_STAGE_BYTES;
    const int Kpad = (K + WT_SLABS * 64 - 1) / (WT_SLABS * 64) * (WT_SLABS * 64);
    const size_t xbytes = xt ? 0 : (size_t)M * Kpad * 2;
    L.red = L.xs + ((xbytes + 127) / 128) * 128;
    // A warp runs at most `stages` stages ahead of the slowest one, so at most
    // ceil(stages / nst) + 2 row groups (nst stages each) have partial sums in flight;
    // each warp keeps its own partial of a group.
    const int nst = Kpad / (WT_SLABS * 64);
    L.nslots = (stages + nst - 1) / nst + 2;
    if (L.nslots > WT_SLOTS) L.nslots = WT_SLOTS;
    const size_t redbytes = (size_t)L.nslots * WT_CONSUMERS * MT * 32 * 4 * sizeof(float);
    L.sws = L.red + redbytes;
    L.sbias = L.sws + (size_t)WT_MAX_ROWS * sizeof(float);       // bias slice, when given
    L.bars = L.sbias + (bias ? (size_t)WT_MAX_ROWS * sizeof(float) : 0);
    // barriers, slot counters, abort flag, TMEM address
    L.total = L.bars + (size_t)2 * stages * sizeof(uint64_t) + (WT_SLOTS + 4) * sizeof(int);
    return L;
}

// x fragment address: plane h (0/1), chunk c (64 k), activation row m, lane t (0..3):
// the 16-byte piece x[m][64c + 16t + 8h .. +8].  Kpad = K rounded up to whole stages.
__device__ __forceinline__ uint32_t xfrag_addr(uint32_t xs, int M, int Kpad, int c, int m,
                                               int t, int h) {
    return xs + (uint32_t)h * (uint32_t)(M * Kpad) + (uint32_t)(((c * M + m) * 4 + t) * 16);
}

// Tensor-memory columns the staged activations need: every consumer warp holds 8
// columns (32 bytes per lane) per chunk it owns (2 per stage) and per 8 activation rows;
// warps w and w+4 share a lane quarter, so the allocation is twice one warp's share.
template <int SL>
__host__ __device__ inline int wt_tmem_cols(int nst, int MT) { return 2 * SL * nst * MT; }
constexpr int WT_TMEM_MAX_COLS = 512;

__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
        : "memory");
}
__device__ __forceinline__ void tmem_ld_x8(uint32_t taddr, uint32_t (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                   "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr));
}
// Completes this thread's outstanding tcgen05.ld; the registers are tied to the wait so
// that no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_wait_ld_x8(uint32_t (&v)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                   "+r"(v[6]), "+r"(v[7])::"memory");
}

// PF: the producer prefetches the first l2pf stages into L2 before the dependency wait (a
// separate instantiation, so the kernels of short streams are unchanged by it).
template <int MT, bool XT, int SL, bool BIAS, bool PF>
__global__ __launch_bounds__(WT_THREADS, 1) void k_w8a16_tma(
    const __grid_constant__ CUtensorMap wmap, const uint16_t* __restrict__ x,
    const float* __restrict__ s_w, const float* __restrict__ bias, void* __restrict__ y,
    int y_bf16, int M, int N, int K, int stages, int l2pf, int* status) {
    WT_GEOMETRY(SL);
    extern __shared__ __align__(1024) uint8_t smem[];
    const WtSmem L = wt_layout<SL>(M, K, MT, stages, XT, BIAS);
    uint8_t* ring = smem + L.ring;
    float* slots = reinterpret_cast<float*>(smem + L.red);  // [nslots][WT_CONSUMERS][MT][32][4]
    float* sws = reinterpret_cast<float*>(smem + L.sws);          // s_w of this CTA's rows
    float* sbias = reinterpret_cast<float*>(smem + L.sbias);      // and their bias (BIAS)
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* empty = full + stages;
    int* cnt = reinterpret_cast<int*>(empty + stages);               // [WT_SLOTS]
    volatile int* abort_flag = cnt + WT_SLOTS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cnt + WT_SLOTS + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nslab = K >> 6;                              // K % 64 == 0
    const int nst = (nslab + WT_SLABS - 1) / WT_SLABS;     // stages per row group
    const int RG = (N + 15) >> 4;
    const int rg0 = (int)((int64_t)RG * blockIdx.x / gridDim.x);
    const int rg1 = (int)((int64_t)RG * (blockIdx.x + 1) / gridDim.x);
    // power-of-two TMEM allocation (>= 32 columns); the launcher checks it is <= 512
    int tcols = 32;
    if (XT)
        while (tcols < wt_tmem_cols<SL>(nst, MT)) tcols <<= 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], WT_CONSUMERS);
        }
        for (int i = 0; i < WT_SLOTS; ++i) cnt[i] = 0;
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (XT && warp == 0) {
        // One CTA per SM, so the columns are free unless a kernel that ran before this one
        // still holds them; the allocation waits for it.  Done before the dependent launch
        // is released, so no kernel that waits on this one can be holding them.
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(tcols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (XT) asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (XT) asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // Programmatic dependent launch: let the next kernel on the stream start its own
    // set-up now, and wait for the previous one to finish (and its writes to be
    // visible) before the first global-memory access -- any input may be its output.
    // Before that wait, on long streams, the producer asks L2 for the CTA's first l2pf
    // stages of weight boxes.  A prefetch returns nothing to this CTA and L2 is the point of
    // coherence, so if the previous kernel does write the weight, the loads issued after
    // the wait still read its final bytes; otherwise the first stages arrive from L2
    // instead of DRAM while the previous kernel drains.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (PF && warp == WT_CONSUMERS && lane == 0) {
        tma_prefetch_desc(&wmap);
        int rg = rg0, st = 0;
        for (int i = 0; i < l2pf && rg < rg1; ++i) {
#pragma unroll
            for (int j = 0; j < WT_BOXES; ++j)
                asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                                 reinterpret_cast<uint64_t>(&wmap)),
                             "r"(st * WT_SLABS * 64 + j * WT_BOX), "r"(rg * 16)
                             : "memory");
            if (++st == nst) { st = 0; ++rg; }
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == WT_CONSUMERS) {
        // ------------------------------------------------------------- producer
        if (lane == 0) {
            tma_prefetch_desc(&wmap);
            // the weight is read once: let it leave L2 first, so that the activations and
            // scales (of this call and the next ones) stay there
            const uint64_t pol = make_l2_policy_evict_first();
            int it = 0, s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int rg = rg0; rg < rg1 && ok; ++rg) {
                for (int st = 0; st < nst; ++st) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, status, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int k0 = st * WT_SLABS * 64;
                    mbar_expect_tx(&full[s], (uint32_t)WT_STAGE_BYTES);
                    uint8_t* dst = ring + (size_t)s * WT_STAGE_BYTES;
#pragma unroll
                    for (int j = 0; j < WT_BOXES; ++j)     // boxes past K read as zeros
                        tma_load_2d_hint(dst + j * 16 * WT_BOX, &wmap, k0 + j * WT_BOX, rg * 16,
                                         &full[s], pol);
                    ++it;
                    if (++s == stages) { s = 0; ph ^= 1u; }
                }
            }
            // Do not leave while copies issued here may still be landing in shared memory.
            for (int i = max(0, it - stages); i < it; ++i)
                mbar_drain(&full[i % stages], (uint32_t)(i / stages) & 1u, status);
        }
        return;
    }

    // ----------------------------------------------------------------- consumers
    // The producer starts streaming as soon as the previous kernel is done; the consumers
    // stage the scales and the activations meanwhile and then meet at barrier 1.
    {
        // The epilogue must not wait on global loads (a stalled warp holds back the ring):
        // stage this CTA's per-channel scales once.
        const int row0 = rg0 * 16, rows = min(rg1 * 16, N) - row0;
        for (int i = threadIdx.x; i < rows; i += WT_CONSUMERS * 32) {
            sws[i] = __ldg(s_w + row0 + i);
            if (BIAS) sbias[i] = __ldg(bias + row0 + i);
        }
    }
    const int g = lane >> 2, t = lane & 3;
    const int Kpad = nst * WT_SLABS * 64;
    const uint32_t xs = smem_u32(smem + L.xs);
    // this warp's TMEM lanes (its quarter) and columns (share warp / 4 of its quarter)
    const uint32_t tm_warp =
        XT ? *tmem_slot + ((uint32_t)((warp & 3) * 32) << 16) +
                 (uint32_t)((warp >> 2) * (wt_tmem_cols<SL>(nst, MT) / (WT_CONSUMERS / 4)))
           : 0u;
    if (XT) {
        // Lane (g, t) of warp w feeds, for its local chunk lc (chunk c = 16*(lc/2) + w +
        // 8*(lc%2), 64 k) and 8-row tile mt, the 16 elements x[m][64c + 16t .. +16] of row
        // m = 8*mt + g: 8 words in columns (lc*MT + mt)*8 .. +8 of its own lane, element
        // pairs regrouped to the (even, odd) k pairing of s8x4_to_bf16x2_eo; zero for rows
        // past M and chunks past K.  The loads of XB stages are issued together, so the
        // staging costs about nst / XB memory round trips.
        constexpr int XB = (MT == 1 ? 8 : 4) / WT_SPW;
        for (int st0 = 0; st0 < nst; st0 += XB) {
            uint4 v[XB][WT_SPW][MT][2];
#pragma unroll
            for (int b = 0; b < XB; ++b)
#pragma unroll
                for (int jj = 0; jj < WT_SPW; ++jj) {
                    const int c = WT_SLABS * (st0 + b) + warp + WT_CONSUMERS * jj;
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        const int m = mt * 8 + g;
                        v[b][jj][mt][0] = v[b][jj][mt][1] = make_uint4(0, 0, 0, 0);
                        if (m < M && c < nslab) {
                            const uint16_t* src = x + (int64_t)m * K + 64 * c + 16 * t;
                            v[b][jj][mt][0] = ldg_keep(src);
                            v[b][jj][mt][1] = ldg_keep(src + 8);
                        }
                    }
                }
#pragma unroll
            for (int b = 0; b < XB; ++b) {
                if (st0 + b >= nst) break;                   // warp-uniform
#pragma unroll
                for (int jj = 0; jj < WT_SPW; ++jj)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        uint32_t wv[8];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint4 a = v[b][jj][mt][h];
                            wv[4 * h + 0] = __byte_perm(a.x, a.y, 0x5410);
                            wv[4 * h + 1] = __byte_perm(a.x, a.y, 0x7632);
                            wv[4 * h + 2] = __byte_perm(a.z, a.w, 0x5410);
                            wv[4 * h + 3] = __byte_perm(a.z, a.w, 0x7632);
                        }
                        tmem_st_x8(tm_warp +
                                       (uint32_t)(((WT_SPW * (st0 + b) + jj) * MT + mt) * 8),
                                   wv);
                    }
            }
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    } else {
        // x [M, K] -> fragment order (two planes of 16-byte pieces), element pairs
        // regrouped to the (even, odd) k pairing of s8x4_to_bf16x2_eo; zero past K.
        const int units = M * Kpad / 8;
        const int per_row = Kpad / 8;
        for (int u = threadIdx.x; u < units; u += WT_CONSUMERS * 32) {
            const int m = u / per_row, r = u - m * per_row;
            const int c = r >> 3, tt = (r >> 1) & 3, h = r & 1;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (8 * r < K) v = ldg_keep(x + (int64_t)m * K + 8 * r);
            const uint32_t p0 = __byte_perm(v.x, v.y, 0x5410), p1 = __byte_perm(v.x, v.y, 0x7632);
            const uint32_t p2 = __byte_perm(v.z, v.w, 0x5410), p3 = __byte_perm(v.z, v.w, 0x7632);
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(
                             xfrag_addr(xs, M, Kpad, c, m, tt, h)),
                         "r"(p0), "r"(p1), "r"(p2), "r"(p3)
                         : "memory");
        }
    }
    named_bar_sync(1, WT_CONSUMERS * 32);

    // This lane's weight bytes in a stage: slab j (j = warp + WT_CONSUMERS*jj) lives in
    // box j/4, rows g and g+8, bytes (j%4)*64 + 16t .. +16.
    const uint32_t ring_u = smem_u32(ring);
    const uint32_t w_off = (uint32_t)((warp >> 2) * 16 * WT_BOX + g * WT_BOX + (warp & 3) * 64 +
                                      t * 16);
    constexpr uint32_t kSlab2 = WT_CONSUMERS / 4 * 16 * WT_BOX;  // slab j+WT_CONSUMERS
    // Shared-memory staging: activation fragments of chunk c = st*16 + j, plane 0 address;
    // +1024*M bytes per stage; slab j+8 is 8 chunks (8*M*64 bytes) further.
    uint32_t x_lane[MT];
    bool x_live[MT];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int m = mt * 8 + g;
        x_live[mt] = m < M;
        x_lane[mt] = xfrag_addr(xs, M, Kpad, warp, x_live[mt] ? m : 0, t, 0);
    }
    const uint32_t plane = (uint32_t)(M * Kpad);
    const uint32_t x_step = XT ? (uint32_t)(WT_SPW * MT * 8) : (uint32_t)(WT_SLABS * M * 64);
    const uint32_t x_slab2 = (uint32_t)(WT_CONSUMERS * M * 64);

    int s = 0, slot = 0;
    uint32_t ph = 0;
    uint32_t wst = ring_u + w_off;                           // stage s, this lane
    // Independent accumulator chains: consecutive MMAs of a warp go to different
    // accumulators, so they do not wait on each other's results.
    constexpr int CH = WT_SPW == 2 && MT == 1 ? 8 : 4;
    for (int rg = rg0; rg < rg1; ++rg) {
        float acc[CH][MT][4];
#pragma unroll
        for (int c = 0; c < CH; ++c)
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[c][mt][i] = 0.0f;

        uint32_t xst = 0;                   // stage offset into x (TMEM columns or bytes)
        for (int st = 0; st < nst; ++st) {
            // xr[jj][mt]: words 0-3 plane 0 (k 16t..16t+7), words 4-7 plane 1 (+8)
            uint32_t xr[WT_SPW][MT][8];
            if (XT) {
                // the activations do not depend on the stage: read them before waiting
#pragma unroll
                for (int jj = 0; jj < WT_SPW; ++jj)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
                        tmem_ld_x8(tm_warp + xst + (uint32_t)((jj * MT + mt) * 8), xr[jj][mt]);
            }
            mbar_wait(&full[s], ph, status, abort_flag);   // on expiry: finish with garbage
            uint4 w[WT_SPW][2];
#pragma unroll
            for (int jj = 0; jj < WT_SPW; ++jj) {
                w[jj][0] = lds128(wst + jj * kSlab2);
                w[jj][1] = lds128(wst + jj * kSlab2 + 8 * WT_BOX);
            }
            if (XT) {
#pragma unroll
                for (int jj = 0; jj < WT_SPW; ++jj)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) tmem_wait_ld_x8(xr[jj][mt]);
            } else {
#pragma unroll
                for (int jj = 0; jj < WT_SPW; ++jj)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        uint4 a = make_uint4(0, 0, 0, 0), b = a;
                        if (x_live[mt]) {
                            const uint32_t xa_addr = x_lane[mt] + xst + (uint32_t)jj * x_slab2;
                            a = lds128(xa_addr);
                            b = lds128(xa_addr + plane);
                        }
                        xr[jj][mt][0] = a.x; xr[jj][mt][1] = a.y;
                        xr[jj][mt][2] = a.z; xr[jj][mt][3] = a.w;
                        xr[jj][mt][4] = b.x; xr[jj][mt][5] = b.y;
                        xr[jj][mt][6] = b.z; xr[jj][mt][7] = b.w;
                    }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);           // operands are in registers
#pragma unroll
            for (int jj = 0; jj < WT_SPW; ++jj) {
                const uint32_t wav[4] = {w[jj][0].x, w[jj][0].y, w[jj][0].z, w[jj][0].w};
                const uint32_t wbv[4] = {w[jj][1].x, w[jj][1].y, w[jj][1].z, w[jj][1].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t alo, ahi, blo, bhi;       // (even, odd) byte pairs
                    s8x4_to_bf16x2_eo(wav[q], alo, ahi);
                    s8x4_to_bf16x2_eo(wbv[q], blo, bhi);
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
                        mma_bf16_16816(acc[(jj * 4 + q) % CH][mt], alo, blo, ahi, bhi,
                                       xr[jj][mt][2 * q], xr[jj][mt][2 * q + 1]);
                }
            }
            xst += x_step;
            wst += WT_STAGE_BYTES;
            if (++s == stages) { s = 0; ph ^= 1u; wst = ring_u + w_off; }
        }

        // Store this warp's partial sums in the group's slot; the last warp to arrive adds
        // the WT_CONSUMERS partials in warp order (no float atomics, so the sum is the same
        // on every run), scales and writes y.  Slots rotate, so no barrier is needed: a
        // warp can run at most `stages` stages (nslots - 2 groups) ahead of the slowest one.
        float* sl = slots + (size_t)slot * WT_CONSUMERS * MT * 128;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            float v[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[i] = 0.0f;
#pragma unroll
                for (int c = 0; c < CH; ++c) v[i] += acc[c][mt][i];
            }
            *reinterpret_cast<float4*>(&sl[((size_t)warp * MT + mt) * 128 + lane * 4]) =
                make_float4(v[0], v[1], v[2], v[3]);
        }
        __threadfence_block();
        __syncwarp();
        int prev = 0;
        if (lane == 0) prev = atomicAdd(&cnt[slot], 1);
        prev = __shfl_sync(0xffffffffu, prev, 0);
        if (prev == WT_CONSUMERS - 1) {
            __threadfence_block();
            float vv[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                for (int i = 0; i < 4; ++i) vv[mt][i] = 0.0f;
                for (int w = 0; w < WT_CONSUMERS; ++w) {
                    float4 u;
                    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                                 : "=f"(u.x), "=f"(u.y), "=f"(u.z), "=f"(u.w)
                                 : "r"(smem_u32(&sl[((size_t)w * MT + mt) * 128 + lane * 4])));
                    vv[mt][0] += u.x; vv[mt][1] += u.y; vv[mt][2] += u.z; vv[mt][3] += u.w;
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
                    if (m < M && n < N) {
                        const float sv = sws[n - rg0 * 16];
                        const float r = BIAS ? fmaf(vv[mt][i], sv, sbias[n - rg0 * 16])
                                             : vv[mt][i] * sv;
                        if (y_bf16)
                            reinterpret_cast<__nv_bfloat16*>(y)[(int64_t)m * N + n] =
                                __float2bfloat16_rn(r);
                        else
                            reinterpret_cast<float*>(y)[(int64_t)m * N + n] = r;
                    }
                }
        }
        if (++slot == L.nslots) slot = 0;
    }
    if (XT) {
        // every tcgen05.ld of every consumer warp has completed (waited on in the loop)
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        named_bar_sync(1, WT_CONSUMERS * 32);
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (warp == 0)
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(*tmem_slot),
                         "r"(tcols)
                         : "memory");
    }
}

// ----------------------------------------------------------------------- host side

// Tensor-map encoder from the driver, fetched once through the runtime (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    }
    return fn;
}

// 2-D map over a row-major uint8 matrix [rows, cols] (row stride = cols bytes).
bool make_tmap_u8_2d(CUtensorMap* map, const void* base, int64_t rows, int64_t cols,
                     int box_cols, int box_rows, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Whether the activations go to tensor memory (they need at most 512 columns), for
// stages of 16 slabs.  With 9..16 rows they always do: in shared memory they would take
// the room of the ring and double the shared-memory traffic.  With 1..8 rows they do when
// shared memory cannot hold them next to 8 stages, or when each CTA streams at least 512 KB:
// setting up tensor memory costs about half a microsecond more per launch (measured on the
// small shapes), which the lighter shared-memory traffic pays back only on long streams.
static bool wt_use_tmem(int M, int K, int64_t N, int num_sms) {
    WT_GEOMETRY(16);
    const int MT = M <= 8 ? 1 : 2;
    const int nst = (K / 64 + WT_SLABS - 1) / WT_SLABS;
    if (wt_tmem_cols<16>(nst, MT) > WT_TMEM_MAX_COLS) return false;
    if (MT == 2) return true;
    if (wt_layout<16>(M, K, 1, 8, false).total > (size_t)WT_MAX_SMEM) return true;
    const int64_t RG = (N + 15) / 16;
    const int64_t grid = RG < num_sms ? RG : num_sms;
    return (RG + grid - 1) / grid * nst * WT_STAGE_BYTES >= ((int64_t)512 << 10);
}

// Stages of 32 slabs (2 KB of K, 6 in the ring, activations in tensor memory) halve the
// per-stage overhead of the consumers; they pay on long streams (each CTA at least 256 KB)
// when K is a whole number of them, and cost latency on short ones (measured: 4096 x 32000
// -8%, 4096 x 11008 -4%, 2048 x 8192 +3%).
static bool wt_use_wide(int M, int K, int64_t N, int num_sms) {
    const int MT = M <= 8 ? 1 : 2;
    if (K % 2048 != 0 || wt_tmem_cols<32>(K / 2048, MT) > WT_TMEM_MAX_COLS) return false;
    const int64_t RG = (N + 15) / 16;
    const int64_t grid = RG < num_sms ? RG : num_sms;
    return (RG + grid - 1) / grid * 16 * (int64_t)K >= ((int64_t)256 << 10);
}

// Whether the TMA path takes this problem: K % 64 == 0, M <= 16 and the activations fit
// in tensor memory, or in shared memory next to at least 4 ring stages (16-slab stages;
// 32-slab stages are only chosen where they fit too).
bool w8a16_tma_fits(int64_t M, int64_t K, bool bias) {
    WT_GEOMETRY(16);
    if (M < 1 || M > 16 || (K % 64) != 0 || K > (int64_t)1 << 30) return false;
    const int MT = M <= 8 ? 1 : 2;
    const int nst = (int)((K / 64 + WT_SLABS - 1) / WT_SLABS);
    if (wt_tmem_cols<16>(nst, MT) <= WT_TMEM_MAX_COLS) return true;
    // (with 9..16 rows, activations too long for tensor memory do not fit shared memory
    // next to 4 stages either)
    return MT == 1 &&
           wt_layout<16>((int)M, (int)K, 1, 4, false, bias).total <= (size_t)WT_MAX_SMEM;
}

template <int MT, bool XT, int SL, bool BIAS, bool PF>
static cudaError_t launch_wt_pf(const CUtensorMap& map, const uint16_t* x, const float* s_w,
                                const float* bias, void* y, int y_bf16, int M, int N, int K,
                                cudaStream_t st, int grid, int stages, size_t smem,
                                int* status) {
    cudaError_t e = ensure_dyn_smem<k_w8a16_tma<MT, XT, SL, BIAS, PF>>((int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(WT_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_w8a16_tma<MT, XT, SL, BIAS, PF>, map, x, s_w, bias, y,
                              y_bf16, M, N, K, stages, PF ? stages : 0, status);
}

template <int MT, bool XT, int SL, bool BIAS>
static cudaError_t launch_wt(const CUtensorMap& map, const uint16_t* x, const float* s_w,
                             const float* bias, void* y, int y_bf16, int M, int N, int K,
                             cudaStream_t st, int num_sms, int* status) {
    int stages = 8;    // must stay <= WT_SLOTS - 2
    while (stages > 4 && wt_layout<SL>(M, K, MT, stages, XT, BIAS).total > (size_t)WT_MAX_SMEM)
        --stages;
    const WtSmem L = wt_layout<SL>(M, K, MT, stages, XT, BIAS);
    if (L.total > (size_t)WT_MAX_SMEM) return cudaErrorInvalidValue;
    const int RG = (N + 15) / 16;
    int grid = RG < num_sms ? RG : num_sms;
    const int max_rg = WT_MAX_ROWS / 16;                  // rows a CTA may own
    if ((RG + grid - 1) / grid > max_rg) grid = (RG + max_rg - 1) / max_rg;
    // L2 prefetch of the first ring's worth of weight boxes before the dependency wait, for
    // CTAs that stream at least 512 KB (measured on the decode sweep: K = 4096 x N = 32000
    // -0.6 to -1.2 us per call; on shorter streams it only added latency)
    const int64_t cta_bytes = (int64_t)((RG + grid - 1) / grid) * 16 * K;
    if (cta_bytes >= ((int64_t)512 << 10))
        return launch_wt_pf<MT, XT, SL, BIAS, true>(map, x, s_w, bias, y, y_bf16, M, N, K, st,
                                                    grid, stages, L.total, status);
    return launch_wt_pf<MT, XT, SL, BIAS, false>(map, x, s_w, bias, y, y_bf16, M, N, K, st, grid,
                                                 stages, L.total, status);
}

cudaError_t launch_w8a16_tma(const uint16_t* x, const int8_t* q, const float* s_w,
                             const float* bias, void* y, int y_bf16, int64_t M, int64_t N, int K,
                             cudaStream_t st, int num_sms, int* status) {
    CUtensorMap map;
    if (!make_tmap_u8_2d(&map, q, N, K, WT_BOX, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const int m = (int)M, n = (int)N;
#define WT_LAUNCH(MT_, XT_, SL_)                                                            \
    (bias ? launch_wt<MT_, XT_, SL_, true>(map, x, s_w, bias, y, y_bf16, m, n, K, st, num_sms, \
                                           status)                                         \
          : launch_wt<MT_, XT_, SL_, false>(map, x, s_w, bias, y, y_bf16, m, n, K, st,        \
                                            num_sms, status))
    if (wt_use_wide(m, K, N, num_sms))
        return M <= 8 ? WT_LAUNCH(1, true, 32) : WT_LAUNCH(2, true, 32);
    const bool xt = wt_use_tmem(m, K, N, num_sms);
    if (M <= 8) return xt ? WT_LAUNCH(1, true, 16) : WT_LAUNCH(1, false, 16);
    if (!xt) return cudaErrorInvalidValue;             // excluded by w8a16_tma_fits
    return WT_LAUNCH(2, true, 16);
#undef WT_LAUNCH
}

}  // namespace q8

// k_w8a16_tc.cu -- the decode-sized W8A16 linear on the tcgen05 integer tensor cores.
//
//   y[m, n] = s_w[n] * sum_k x[m, k] * q[n, k]        (x bf16 [M, K], q int8 [N, K], M <= 16)
//
// The int8 weight is the only large operand.  This path hands it to tcgen05.mma.kind::i8
// exactly as it lies in HBM (TMA, 128-byte swizzle): no instruction on the CUDA cores per
// weight byte.  The bf16 activations are rewritten once per call as exact int8 digit planes.
//
// Digit planes.  A nonzero finite bf16 value is x = sgn * S * 2^(f - 134), with f >= 1 its
// biased exponent (1 for subnormals) and S its significand as an integer (implicit bit
// included, < 256).  For a base exponent b <= f of its row, I = sgn * S * 2^(f - b) is an
// integer; written in base 128 with signed digits d_j = sgn * ((|I| >> 7j) & 127),
//
//     x[m, k]               = 2^(b_m - 134) * sum_j 128^j d_j[m, k]
//     sum_k x[m, k] q[n, k] = 2^(b_m - 134) * sum_j 128^j P_j[m, n],
//     P_j[m, n]             = sum_k d_j[m, k] q[n, k]   (int32, exact: |P| <= 127*128*K < 2^31)
//
// Every P_j is one column of an int8 GEMM whose B operand is the plane matrix with rows
// (j, m) (row index j*M + m).  The epilogue recombines a row's columns in fp64 (Horner in
// 128, exact while the sum stays below 2^53, else rounded at 2^-53 relative) and scales
// once, so the result is the dot product rounded about once -- tighter than an fp32
// accumulation.  With b_m the smallest exponent of the row, J_m = ceil((8 + f_max - b_m)/7)
// planes represent every element exactly.  A row that would need more planes than the
// tile budget (jcap) raises b_m instead; its elements below 2^(b_m - 134)'s reach, and any
// non-finite element, become residuals: the epilogue adds their products with fp32
// multiplies (exact for bf16 x int8) and fp64 sums, so IEEE infinities and NaNs propagate.
//
// Work split (stream-K).  The weight is cut into 128-row tiles and K into 128-byte
// blocks; a unit is one (tile, block) pair, U = tiles * blocks units in tile-major order,
// and CTA b of G streams the contiguous range [U*b/G, U*(b+1)/G) -- balanced to one unit
// (16 KB of weight).  A tile whose units span several CTAs is finished by the CTA holding
// its first unit (for that CTA it is the last tile of its range); the others write their
// int32 partial accumulators to a workspace slot and raise a flag, which the owner waits
// for before its epilogue.  Flags carry a per-call 64-bit epoch, so they never need
// resetting (the workspace must be zero-filled once before its first use).  The epoch is
// kept on the device, in the workspace (one more than the calls completed on it), so a
// CUDA graph that replays a captured call gets a new epoch on every replay.
//
// CTA structure (6 warps, one CTA per SM):
//   warp 0   : TMA producer.  Weight tiles (128 rows x 128 bytes) start streaming at once;
//              the plane tiles (N rows x 128 bytes, N = 16 * ceil(M * max J / 16)) are
//              added to each stage once the planes exist.
//   warp 1   : allocates 512 TMEM columns; one lane issues tcgen05.mma.kind::i8 (M = 128,
//              N, K = 32) into one of two int32 accumulators (TMEM columns 0 and 256).
//   warps 2-5: first, in CTAs b < min(M, G), the digit planes of activation rows m = b,
//              b + G, ... (written to the workspace, then a row flag); then the epilogue of
//              each tile: tcgen05.ld, cross-CTA partials, fp64 recombination, residuals,
//              scale, store.
// Every wait is bounded (abort flag + status word).
#include "q8_kernels.cuh"

#include <atomic>

namespace q8 {

constexpr int WC_BM = 128;            // weight rows per tile (= TMEM lanes)
constexpr int WC_BK = 128;            // bytes of K per unit (one 128-byte swizzle row)
constexpr int WC_UK = 32;             // K per tcgen05.mma.kind::i8
constexpr int WC_THREADS = 192;
constexpr int WC_TMEM_COLS = 512;
constexpr int WC_ACC_STRIDE = 256;    // TMEM column offset of the second accumulator
constexpr int WC_MAX_M = 16;
constexpr int WC_A_BYTES = WC_BM * WC_BK;   // 16 KB
constexpr int WC_PLANE_ROWS = 256;          // rows of the workspace plane matrix
constexpr int WC_CTRL_BYTES = 2048;

// Tile budget for the plane rows (B operand rows) and the ring depth, by activation rows:
// up to 8 rows, 80 plane rows and 8 stages; above, 160 plane rows and 6 stages.  Rows may
// use up to jcap = nf / M planes each (80 for one row: every finite bf16 row is exact).
struct WcShape {
    int nf, stages, jcap;
};
__host__ __device__ inline WcShape wc_shape(int M) {
    WcShape s;
    s.nf = M <= 8 ? 80 : 160;
    s.stages = M <= 8 ? 8 : 6;
    s.jcap = s.nf / (M > 0 ? M : 1);
    return s;
}
__host__ __device__ inline size_t wc_smem_bytes(int M) {
    const WcShape s = wc_shape(M);
    return (size_t)s.stages * (WC_A_BYTES + (size_t)s.nf * WC_BK) + WC_CTRL_BYTES + 1024;
}

// Per-row plane metadata written by the plane builders.
struct WcMeta {
    int J;        // planes of the row (0: no finite nonzero element)
    int base;     // base exponent b_m
    int nres;     // residual elements
    int pad;
};
struct WcRes {
    int k;        // column of a residual element
    float v;      // its value
};

// Grid-wide state of one call, at the start of the workspace.  Every field but `calls` is
// zero between calls: the flags are compared with the call's epoch, and the counters and
// statistics are returned to zero by the CTA that consumes them.
struct WcHdr {
    unsigned long long stats_flag;     // = epoch once every row's planes count is known
    unsigned long long planes_flag;    // = epoch once every plane and residual is written
    int arrive1, arrive2;              // CTAs done with phase 1 / phase 2 of the build
    int fmax1[WC_MAX_M];               // 1 + largest exponent of the row (0: none yet)
    int fmin1[WC_MAX_M];               // 1000 - smallest exponent (0: none yet)
    int nres[WC_MAX_M];                // residual elements of the row
    int done;                          // CTAs of the current call that have finished
    int pad;
    unsigned long long calls;          // calls completed on this workspace; epoch = calls + 1
};
static_assert(sizeof(WcHdr) <= 256, "the CTA flags start at byte 256");

// Workspace layout (byte offsets), for M activation rows, K columns and G CTAs.  The header
// and the flags come first, at offsets that depend on nothing but G (the device's SM
// count), so that a workspace reused for other sizes never finds other data there.
struct WcPlan {
    size_t hdr, cta_flag, meta, planes, res, slots, bytes;
};
__host__ __device__ inline WcPlan wc_plan(int M, int K, int G) {
    const WcShape s = wc_shape(M);
    auto up = [](size_t v) { return (v + 1023) / 1024 * 1024; };
    WcPlan p;
    p.hdr = 0;
    p.cta_flag = 256;
    p.meta = up(p.cta_flag + (size_t)G * 8);
    p.planes = p.meta + up((size_t)WC_MAX_M * sizeof(WcMeta));
    p.res = p.planes + up((size_t)WC_PLANE_ROWS * K);
    p.slots = p.res + up((size_t)M * K * sizeof(WcRes));
    p.bytes = p.slots + up((size_t)G * WC_BM * s.nf * 4);
    return p;
}

struct WcArgs {
    const uint16_t* x;
    const int8_t* q;
    const float* s_w;
    void* y;
    int y_bf16;
    int M, N, K, KB;          // KB = ceil(K / 128)
    long long U;              // units
    int8_t* planes;
    WcMeta* meta;
    WcRes* res;
    WcHdr* hdr;
    unsigned long long* cta_flag;
    int32_t* slots;
    int* status;
};

// ------------------------------------------------------------------- small helpers
__device__ __forceinline__ uint64_t wc_desc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// kind::i8: signed A and B, int32 accumulator, both K-major; N is a runtime value.
__device__ __forceinline__ uint32_t wc_idesc_i8(int M, int N) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void wc_mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    const uint32_t z = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(z), "r"(z),
        "r"(z), "r"(z)
        : "memory");
}
__device__ __forceinline__ void wc_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void wc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void wc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// 16 consecutive TMEM columns of this warp's 32 lanes, then wait for them.
__device__ __forceinline__ void wc_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    // the registers are tied to the wait, so no use of them is scheduled before it
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])::"memory");
}
// Transaction bytes without an arrival (the stage's arrival comes later, after its
// second copy is issued).
__device__ __forceinline__ void mbar_expect_tx_only(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// Orders this thread's generic-proxy global accesses with its async-proxy (TMA) ones.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Bounded wait for a flag written by another CTA of this grid.
__device__ __forceinline__ bool wait_flag(const unsigned long long* p, unsigned long long epoch,
                                          int* status, volatile int* abort_flag) {
    if (ld_acquire_u64(p) == epoch) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (i > 512) __nanosleep(128);
        if (ld_acquire_u64(p) == epoch) return true;
        if ((i & 15u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                atomicExch(status, kStatusWaitTimeout);
                return false;
            }
        }
    }
}

// CTA holding unit u of U under the split [U*b/G, U*(b+1)/G).
__device__ __forceinline__ int wc_cta_of(long long u, long long U, int G) {
    return (int)(((u + 1) * (long long)G - 1) / U);
}

// Digit j of |I| = S << sh (S < 256, sh >= 0): bits [7j, 7j + 7) of S * 2^sh.
__device__ __forceinline__ int wc_digit(int S, int sh, int j) {
    const int d = sh - 7 * j;
    if (d >= 0) return d >= 7 ? 0 : ((S << d) & 127);
    return -d >= 8 ? 0 : ((S >> -d) & 127);
}

__device__ __forceinline__ void wc_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}
__device__ __forceinline__ uint32_t wc_ld1(uint32_t taddr) {
    uint32_t r;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
    return r;
}
__device__ __forceinline__ void wc_wait_ld16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])::"memory");
}

// Pieces of one bf16 element: significand S (< 256, 0 for zero), exponent f' (>= 1) and
// whether it is finite and nonzero.
__device__ __forceinline__ void wc_split(uint32_t bits, int& S, int& fp, bool& fin_nz) {
    const int f = (int)((bits >> 7) & 0xFFu);
    fp = f > 0 ? f : 1;
    fin_nz = (bits & 0x7FFFu) != 0 && f != 255;
    S = f > 0 ? (int)(128u | (bits & 127u)) : (int)(bits & 127u);
}

// The digit planes are built by every CTA of the grid (its 128 epilogue threads, et), each
// for its slice of the columns (in groups of 8) and all M rows, in two phases separated by
// grid-wide arrivals:
//   1. exponent range of each row over the slice -> shared-memory max/min -> global atomics;
//      the last CTA to arrive turns them into (J, base) per row, zeroes them and raises
//      stats_flag;
//   2. digits of every element of the slice at or above its row's base (residuals below it
//      or non-finite); the last CTA to arrive publishes the residual counts, zeroes the
//      counters and raises planes_flag, which the producers and the epilogues wait for.
// sm: shared scratch of 4 * WC_MAX_M + 1 ints.  Returns false if a wait expired.
__device__ bool wc_build_planes(const WcArgs& a, unsigned long long epoch, int jcap, int et, int* sm,
                                volatile int* abort_flag) {
    const int G = (int)gridDim.x, b = (int)blockIdx.x, K = a.K, M = a.M;
    const int n8 = K >> 3;
    const int c0 = (int)((long long)n8 * b / G), c1 = (int)((long long)n8 * (b + 1) / G);
    const int items = (c1 - c0) * M;                   // (row, 8-column group) pairs
    int* sfmax = sm;                                   // [16]
    int* sfmin = sm + WC_MAX_M;                        // [16]
    int* sJ = sm + 2 * WC_MAX_M;                       // [16]
    int* sBase = sm + 3 * WC_MAX_M;                    // [16]
    int* last = sm + 4 * WC_MAX_M;                     // [1]
    if (et < WC_MAX_M) {
        sfmax[et] = 0;
        sfmin[et] = 0;
    }
    named_bar_sync(3, 128);
    for (int it = et; it < items; it += 128) {
        const int m = it / (c1 - c0), c = c0 + it % (c1 - c0);
        const uint4 v = ldg_keep(a.x + (size_t)m * K + 8 * c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        int fh = 0, fl = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            int S, fp;
            bool ok;
            wc_split((w[e >> 1] >> (16 * (e & 1))) & 0xFFFFu, S, fp, ok);
            if (ok) {
                fh = max(fh, 1 + fp);
                fl = max(fl, 1000 - fp);
            }
        }
        if (fh) {
            atomicMax(&sfmax[m], fh);
            atomicMax(&sfmin[m], fl);
        }
    }
    named_bar_sync(3, 128);
    if (et < M) {
        if (sfmax[et]) {
            atomicMax(&a.hdr->fmax1[et], sfmax[et]);
            atomicMax(&a.hdr->fmin1[et], sfmin[et]);
        }
    }
    __threadfence();
    named_bar_sync(3, 128);
    bool ok = true;
    if (et == 0) {
        if (atomicAdd(&a.hdr->arrive1, 1) == G - 1) {
            // last to arrive: every CTA's contribution is in
            __threadfence();
            for (int m = 0; m < M; ++m) {
                const int fh = atomicExch(&a.hdr->fmax1[m], 0) - 1;
                const int fl = 1000 - atomicExch(&a.hdr->fmin1[m], 0);
                int J = 0, base = 134;
                if (fh >= 1) {
                    const int jfull = (8 + fh - fl + 6) / 7;
                    if (jfull <= jcap) {
                        J = jfull;
                        base = fl;
                    } else {                   // too wide: the lowest elements are residuals
                        J = jcap;
                        base = fh + 8 - 7 * jcap;
                    }
                }
                a.meta[m].J = J;
                a.meta[m].base = base;
            }
            a.hdr->arrive1 = 0;
            __threadfence();
            st_release_u64(&a.hdr->stats_flag, epoch);
        } else {
            ok = wait_flag(&a.hdr->stats_flag, epoch, a.status, abort_flag);
        }
        *last = ok ? 1 : 0;
    }
    named_bar_sync(3, 128);
    ok = *last != 0;
    if (et < M) {
        sJ[et] = ok ? min(max(__ldcg(&a.meta[et].J), 0), jcap) : 0;
        sBase[et] = ok ? __ldcg(&a.meta[et].base) : 134;
    }
    named_bar_sync(3, 128);
    // phase 2: digits and residuals of this slice
    for (int it = et; ok && it < items; it += 128) {
        const int m = it / (c1 - c0), c = c0 + it % (c1 - c0);
        const int J = sJ[m], base = sBase[m];
        const uint4 v = ldg_keep(a.x + (size_t)m * K + 8 * c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        int S[8], sh[8];
        uint32_t neg = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t bits = (w[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
            int Se, fp;
            bool fin_nz;
            wc_split(bits, Se, fp, fin_nz);
            const bool in_planes = fin_nz && fp >= base;
            if ((bits & 0x7FFFu) != 0 && !in_planes) {
                const int idx = atomicAdd(&a.hdr->nres[m], 1);
                WcRes r;
                r.k = 8 * c + e;
                r.v = __uint_as_float(bits << 16);
                a.res[(size_t)m * K + idx] = r;
            }
            S[e] = in_planes ? Se : 0;
            sh[e] = in_planes ? fp - base : 0;
            neg |= (bits >> 15) << e;
        }
        for (int j = 0; j < J; ++j) {
            uint32_t lo = 0, hi = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                int d = wc_digit(S[e], sh[e], j);
                if ((neg >> e) & 1u) d = -d;
                if (e < 4)
                    lo |= ((uint32_t)d & 0xFFu) << (8 * e);
                else
                    hi |= ((uint32_t)d & 0xFFu) << (8 * (e - 4));
            }
            *reinterpret_cast<uint2*>(a.planes + (size_t)(j * M + m) * K + 8 * c) =
                make_uint2(lo, hi);
        }
    }
    fence_proxy_async_global();
    __threadfence();
    named_bar_sync(3, 128);
    if (et == 0 && ok) {
        if (atomicAdd(&a.hdr->arrive2, 1) == G - 1) {
            __threadfence();
            for (int m = 0; m < M; ++m) a.meta[m].nres = atomicExch(&a.hdr->nres[m], 0);
            a.hdr->arrive2 = 0;
            __threadfence();
            st_release_u64(&a.hdr->planes_flag, epoch);
        }
    }
    return ok;
}

// -------------------------------------------------------------------- the kernel
__global__ __launch_bounds__(WC_THREADS, 1) void k_w8a16_tc(
    const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
    const WcArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const WcShape shp = wc_shape(a.M);
    const int S = shp.stages;
    const uint32_t b_stage = (uint32_t)shp.nf * WC_BK;            // bytes of a plane slot
    uint8_t* ringA = smem;
    uint8_t* ringB = smem + (size_t)S * WC_A_BYTES;
    uint8_t* ctrl = ringB + (size_t)S * b_stage;
    uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);            // [S]
    uint64_t* empty = full + S;                                    // [S]
    uint64_t* tfull = empty + S;                                   // [2]
    uint64_t* tempty = tfull + 2;                                  // [2]
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* n_pub = reinterpret_cast<volatile int*>(tmem_slot + 2);
    int* mJ = reinterpret_cast<int*>(ctrl + 512);                  // [16]
    int* mBase = mJ + WC_MAX_M;                                    // [16]
    int* mRes = mBase + WC_MAX_M;                                  // [16]
    int* bsm = reinterpret_cast<int*>(ctrl + 1024);                // plane-builder scratch

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = (int)gridDim.x, b = (int)blockIdx.x;
    const long long U = a.U;
    const long long u0 = U * b / G, u1 = U * (b + 1) / G;
    const int KB = a.KB;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 4);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        *n_pub = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(WC_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    wc_fence_before();
    __syncthreads();
    wc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // Programmatic dependent launch: the next kernel may start its set-up; every global
    // access below waits for the previous kernel (its outputs may be our inputs).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // This call's epoch.  The previous call on the workspace has completed (the wait
    // above), and `calls` only advances once every CTA of this call has read it (the last
    // CTA to finish advances it, below).
    const unsigned long long epoch = ld_acquire_u64(&a.hdr->calls) + 1ull;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&amap);
            tma_prefetch_desc(&bmap);
            const long long nu = u1 - u0;
            const int pre = (int)(nu < S ? nu : S);
            // The weight tiles of the first stages do not wait for the planes.
            for (int i = 0; i < pre; ++i) {
                const long long u = u0 + i;
                mbar_expect_tx_only(&full[i], (uint32_t)WC_A_BYTES);
                tma_load_2d(ringA + (size_t)i * WC_A_BYTES, &amap, (int)(u % KB) * WC_BK,
                            (int)(u / KB) * WC_BM, &full[i]);
            }
            int jmax = 0;
            bool ok = wait_flag(&a.hdr->planes_flag, epoch, a.status, abort_flag);
            fence_proxy_async_global();
            if (ok)
                for (int m = 0; m < a.M; ++m)
                    jmax = max(jmax, min(max(__ldcg(&a.meta[m].J), 0), shp.jcap));
            const int nrows = max(16, (a.M * jmax + 15) / 16 * 16);
            *n_pub = nrows;
            const uint32_t bbytes = (uint32_t)nrows * WC_BK;
            for (int i = 0; i < pre; ++i) {
                const long long u = u0 + i;
                if (ok) {
                    mbar_expect_tx_only(&full[i], bbytes);
                    for (int r = 0; r < nrows; r += 16)
                        tma_load_2d(ringB + (size_t)i * b_stage + (size_t)r * WC_BK, &bmap,
                                    (int)(u % KB) * WC_BK, r, &full[i]);
                }
                mbar_arrive(&full[i]);
            }
            int s = pre % S;
            uint32_t ph = (uint32_t)(pre / S) & 1u;
            long long issued = pre;
            for (long long u = u0 + pre; u < u1 && ok; ++u) {
                if (!mbar_wait(&empty[s], ph ^ 1u, a.status, abort_flag)) {
                    ok = false;
                    break;
                }
                const int kb = (int)(u % KB), t = (int)(u / KB);
                mbar_expect_tx(&full[s], (uint32_t)WC_A_BYTES + bbytes);
                tma_load_2d(ringA + (size_t)s * WC_A_BYTES, &amap, kb * WC_BK, t * WC_BM,
                            &full[s]);
                for (int r = 0; r < nrows; r += 16)
                    tma_load_2d(ringB + (size_t)s * b_stage + (size_t)r * WC_BK, &bmap,
                                kb * WC_BK, r, &full[s]);
                ++issued;
                if (++s == S) { s = 0; ph ^= 1u; }
            }
            // do not leave while copies issued here may still be landing
            for (long long i = issued > S ? issued - S : 0; i < issued; ++i)
                mbar_drain(&full[i % S], (uint32_t)(i / S) & 1u, a.status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int s = 0, acc = 0;
            uint32_t ph = 0, acc_ph = 0, idesc = 0;
            int nrows = 0;
            for (long long u = u0; u < u1; ++u) {
                const int kb = (int)(u % KB);
                const bool first = u == u0 || kb == 0;
                const bool last = u + 1 == u1 || kb == KB - 1;
                if (first) {
                    if (!mbar_wait(&tempty[acc], acc_ph ^ 1u, a.status, abort_flag)) break;
                    wc_fence_after();
                }
                if (!mbar_wait(&full[s], ph, a.status, abort_flag)) break;
                wc_fence_after();
                if (nrows == 0) {
                    nrows = *n_pub;
                    idesc = wc_idesc_i8(WC_BM, nrows);
                }
                const uint32_t d = tmem_base + (uint32_t)(acc * WC_ACC_STRIDE);
                const uint64_t ad = wc_desc_sw128(smem_u32(ringA + (size_t)s * WC_A_BYTES));
                const uint64_t bd = wc_desc_sw128(smem_u32(ringB + (size_t)s * b_stage));
#pragma unroll
                for (int k = 0; k < WC_BK / WC_UK; ++k)      // +32 bytes of K = +2 (16-byte units)
                    wc_mma_i8(d, ad + 2 * k, bd + 2 * k, idesc, (!first || k > 0) ? 1u : 0u);
                wc_commit(&empty[s]);                        // stage free once these finish
                if (++s == S) { s = 0; ph ^= 1u; }
                if (last) {
                    wc_commit(&tfull[acc]);                  // accumulator ready
                    if (++acc == 2) { acc = 0; acc_ph ^= 1u; }
                }
            }
            // every MMA issued here completes before tensor memory is released
            wc_commit(mma_done);
            mbar_drain(mma_done, 0, a.status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ planes, then the epilogue
        const int et = threadIdx.x - 64;                     // 0..127
        const int qd = warp & 3;                             // TMEM lane quarter
        const int row = qd * 32 + lane;                      // tile row of this thread
        bool built = wc_build_planes(a, epoch, shp.jcap, et, bsm, abort_flag);
        if (et == 0) {
            const bool ok = built && wait_flag(&a.hdr->planes_flag, epoch, a.status, abort_flag);
            for (int m = 0; m < WC_MAX_M; ++m) {
                const bool v = ok && m < a.M;
                mJ[m] = v ? min(max(__ldcg(&a.meta[m].J), 0), shp.jcap) : 0;
                mBase[m] = v ? __ldcg(&a.meta[m].base) : 134;
                mRes[m] = v ? min(max(__ldcg(&a.meta[m].nres), 0), a.K) : 0;
            }
        }
        named_bar_sync(3, 128);
        int jmax = 0;
        for (int m = 0; m < WC_MAX_M; ++m) jmax = max(jmax, mJ[m]);
        const int nrows = max(16, (a.M * jmax + 15) / 16 * 16);
        const size_t slot_stride = (size_t)WC_BM * shp.nf;     // int32 per CTA slot

        int acc = 0;
        uint32_t acc_ph = 0;
        const long long tfirst = u0 / KB, tlast = (u1 - 1) / KB;
        for (long long t = tfirst; t <= tlast; ++t) {
            const long long ua = max(u0, t * KB), ub = min(u1, (t + 1) * KB);
            const bool deposit = ua > t * KB;                // tile began in an earlier CTA
            const int last_cta = (!deposit && ub < (t + 1) * KB)
                                     ? wc_cta_of((t + 1) * KB - 1, U, G)
                                     : b;                    // contributors b+1 .. last_cta
            const bool okw = mbar_wait(&tfull[acc], acc_ph, a.status, abort_flag);
            const bool live = __shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0;
            wc_fence_after();
            const uint32_t tb =
                tmem_base + ((uint32_t)(qd * 32) << 16) + (uint32_t)(acc * WC_ACC_STRIDE);
            // A slot holds a CTA's partial tile as [16-column chunk][tile row][16] int32, so
            // that a warp moves 2 KB of contiguous memory per chunk.
            if (deposit) {
                int32_t* slot = a.slots + (size_t)b * slot_stride;
                for (int c = 0; live && c < nrows; c += 16) {
                    uint32_t r[16];
                    wc_ld16(tb + (uint32_t)c, r);
                    int4* o = reinterpret_cast<int4*>(slot + ((size_t)(c >> 4) * WC_BM + row) * 16);
#pragma unroll
                    for (int h = 0; h < 4; ++h)
                        o[h] = make_int4((int)r[4 * h], (int)r[4 * h + 1], (int)r[4 * h + 2],
                                         (int)r[4 * h + 3]);
                }
                __threadfence();
                named_bar_sync(3, 128);
                if (et == 0 && live) st_release_u64(&a.cta_flag[b], epoch);
            } else {
                if (et == 0)
                    for (int c = b + 1; c <= last_cta; ++c)
                        if (!wait_flag(&a.cta_flag[c], epoch, a.status, abort_flag)) break;
                named_bar_sync(3, 128);
                if (live && last_cta > b) {
                    // add the other CTAs' partials into this tile's accumulator, in groups of
                    // up to 5 chunks whose loads are all in flight together
                    constexpr int GRP = 5;
                    const int nch = nrows >> 4;
                    for (int g0 = 0; g0 < nch; g0 += GRP) {
                        for (int cc = b + 1; cc <= last_cta; ++cc) {
                            const int4* src =
                                reinterpret_cast<const int4*>(a.slots + (size_t)cc * slot_stride);
                            int4 v[GRP][4];
#pragma unroll
                            for (int i = 0; i < GRP; ++i)
#pragma unroll
                                for (int h = 0; h < 4; ++h)
                                    v[i][h] = g0 + i < nch
                                                  ? __ldcg(src + ((size_t)(g0 + i) * WC_BM + row) * 4 + h)
                                                  : make_int4(0, 0, 0, 0);
#pragma unroll
                            for (int i = 0; i < GRP; ++i) {
                                if (g0 + i < nch) {                   // warp-uniform
                                    const uint32_t ta = tb + (uint32_t)((g0 + i) * 16);
                                    uint32_t r[16];
                                    wc_ld16(ta, r);
#pragma unroll
                                    for (int h = 0; h < 4; ++h) {
                                        r[4 * h] += (uint32_t)v[i][h].x;
                                        r[4 * h + 1] += (uint32_t)v[i][h].y;
                                        r[4 * h + 2] += (uint32_t)v[i][h].z;
                                        r[4 * h + 3] += (uint32_t)v[i][h].w;
                                    }
                                    wc_st16(ta, r);
                                }
                            }
                            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                        }
                    }
                }
                double T[WC_MAX_M];
#pragma unroll
                for (int m = 0; m < WC_MAX_M; ++m) T[m] = 0.0;
                for (int j = jmax - 1; live && j >= 0; --j) {
                    uint32_t r[WC_MAX_M];
#pragma unroll
                    for (int m = 0; m < WC_MAX_M; ++m)
                        r[m] = m < a.M ? wc_ld1(tb + (uint32_t)(j * a.M + m)) : 0u;
                    wc_wait_ld16(r);
#pragma unroll
                    for (int m = 0; m < WC_MAX_M; ++m) {
                        if (m < a.M && j < mJ[m]) T[m] = fma(T[m], 128.0, (double)(int)r[m]);
                    }
                }
                const long long n = t * WC_BM + row;
                if (live && n < a.N) {
                    const double sw = (double)__ldg(a.s_w + n);
                    const int8_t* qrow = a.q + (size_t)n * a.K;
#pragma unroll
                    for (int m = 0; m < WC_MAX_M; ++m) {
                        if (m < a.M) {
                            double v = ldexp(T[m], mBase[m] - 134);
                            for (int r = 0; r < mRes[m]; ++r) {      // residual elements
                                const WcRes e = a.res[(size_t)m * a.K + r];
                                v += (double)(e.v * (float)__ldg(qrow + e.k));
                            }
                            const float out = (float)(sw * v);
                            if (a.y_bf16)
                                reinterpret_cast<__nv_bfloat16*>(a.y)[(size_t)m * a.N + n] =
                                    __float2bfloat16_rn(out);
                            else
                                reinterpret_cast<float*>(a.y)[(size_t)m * a.N + n] = out;
                        }
                    }
                }
            }
            wc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            if (++acc == 2) { acc = 0; acc_ph ^= 1u; }
        }
    }

    wc_fence_before();
    __syncthreads();
    wc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(WC_TMEM_COLS)
                     : "memory");
    if (threadIdx.x == 0) {
        // every thread of this CTA read the epoch before the barrier above
        __threadfence();
        if (atomicAdd(&a.hdr->done, 1) == G - 1) {
            atomicExch(&a.hdr->done, 0);
            __threadfence();
            atomicAdd(&a.hdr->calls, 1ull);
        }
    }
}

// ----------------------------------------------------------------------- host side
size_t w8a16_tc_workspace_bytes(int64_t M, int64_t K, int num_sms) {
    if (M < 1 || M > WC_MAX_M || K < 16 || K % 16) return 0;
    return wc_plan((int)M, (int)K, num_sms).bytes;
}

cudaError_t launch_w8a16_tc(const uint16_t* x, const int8_t* q, const float* s_w, void* y,
                            int y_bf16, int64_t M, int64_t N, int K, void* ws,
                            cudaStream_t st, int num_sms, int* status) {
    const int KB = (K + WC_BK - 1) / WC_BK;
    const long long T = (N + WC_BM - 1) / WC_BM;
    const long long U = T * KB;
    const int G = (int)(U < num_sms ? U : num_sms);
    const WcPlan p = wc_plan((int)M, K, num_sms);       // slot region sized for num_sms CTAs
    uint8_t* w = static_cast<uint8_t*>(ws);
    CUtensorMap am, bm;
    if (!make_tmap_u8_2d(&am, q, N, K, WC_BK, WC_BM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_tmap_u8_2d(&bm, w + p.planes, WC_PLANE_ROWS, K, WC_BK, 16,
                         CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    WcArgs a;
    a.x = x;
    a.q = q;
    a.s_w = s_w;
    a.y = y;
    a.y_bf16 = y_bf16;
    a.M = (int)M;
    a.N = (int)N;
    a.K = K;
    a.KB = KB;
    a.U = U;
    a.planes = reinterpret_cast<int8_t*>(w + p.planes);
    a.meta = reinterpret_cast<WcMeta*>(w + p.meta);
    a.res = reinterpret_cast<WcRes*>(w + p.res);
    a.hdr = reinterpret_cast<WcHdr*>(w + p.hdr);
    a.cta_flag = reinterpret_cast<unsigned long long*>(w + p.cta_flag);
    a.slots = reinterpret_cast<int32_t*>(w + p.slots);
    a.status = status;
    const size_t smem = wc_smem_bytes((int)M);
    cudaError_t e = ensure_dyn_smem<k_w8a16_tc>((int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(WC_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_w8a16_tc, am, bm, a);
}

}  // namespace q8

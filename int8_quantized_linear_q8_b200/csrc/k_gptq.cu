// k_gptq.cu -- GPTQ on the int8 weight grid and the calibration Hessian, in float64.
//
// [SmolVLM-Q8] gptq_int8 (Frantar et al. 2022) and hessians:
//   H      = sum over calibration batches of x^T x        (x fp32 [R, K], sums in fp64)
//   s[n]   = weight_int8 scale of the ORIGINAL row (observer grid, max(amax/127.5, eps))
//   dead   = diag(H) == 0:  H[k,k] = 1, w[:, k] = 0
//   H     += damp * mean(diag(H)) * I
//   U      = upper Cholesky factor of H^-1 (via L = chol(H), H^-1 = L^-T L^-1, chol again)
//   per block of columns [i1, i2), column by column:
//            q = clamp(round(w / s), -128, 127), e = (w - q s) / U[i,i],
//            w[:, j] -= e U[i, j] for the block's j >= i;
//   after the block, w[:, j] -= sum_t e_t U[t, j] for every j >= i2.
//
// Every float64 sum here runs in ascending index order with one correctly rounded
// operation at a time (explicit _rn intrinsics: no contraction into fused multiply-adds),
// so the results are the same bits as a sequential reference written the same way.  That
// rules out the tensor cores (their accumulation order is fixed by the hardware); the work
// is O(K^3) for the factorisations and O(N K^2) for the updates, offline, once per layer.
//
//   * Cholesky factorisations and the triangular inverse are right-looking: one launch per
//     pivot k finalises the pivot column (row) and updates the whole trailing region.  An entry then receives its subtractions
//     in ascending k -- the order of the left-looking dot products -- while every launch
//     has (K - k)^2 / 2 independent entries instead of a long per-thread chain.
//   * Row n of W is independent of every other row once U exists: the in-block column loop
//     runs one thread per row, the lazy block update one thread per (row, later column).
#include "q8_kernels.cuh"

namespace q8 {

constexpr int GQ_TILE = 32;              // output tile of the Gram kernels (32 x 32)
constexpr int GQ_ROWS = 8;               // thread rows per tile (4 outputs each)
constexpr int GQ_BLOCK_MAX = 256;        // largest GPTQ column block
constexpr int GQ_ROW_THREADS = 32;       // rows per CTA of the in-block column loop

__device__ __forceinline__ double dsub_mul(double t, double a, double b) {
    return __dsub_rn(t, __dmul_rn(a, b));
}

// ------------------------------------------------------------- calibration Hessian
// H[i, j] (= or +=) sum_{r ascending} x[r, i] * x[r, j] for the upper-triangle tiles
// (j-tile >= i-tile), written to both (i, j) and (j, i): the products commute exactly, so
// both triangles equal their sequential sums.
__global__ __launch_bounds__(GQ_TILE * GQ_ROWS) void k_gram_acc(const float* __restrict__ x,
                                                               int64_t R, int K,
                                                               double* __restrict__ H,
                                                               int reset) {
    const int ti = blockIdx.y, tj = blockIdx.x;
    if (tj < ti) return;
    __shared__ float xa[GQ_TILE][GQ_TILE + 1];
    __shared__ float xb[GQ_TILE][GQ_TILE + 1];
    const int tx = threadIdx.x % GQ_TILE, ty = threadIdx.x / GQ_TILE;
    const int i0 = ti * GQ_TILE, j0 = tj * GQ_TILE;
    double acc[GQ_TILE / GQ_ROWS];
#pragma unroll
    for (int m = 0; m < GQ_TILE / GQ_ROWS; ++m) acc[m] = 0.0;
    for (int64_t r0 = 0; r0 < R; r0 += GQ_TILE) {
        // stage 32 calibration rows of the two column tiles (zeros past R or K)
        for (int e = threadIdx.x; e < GQ_TILE * GQ_TILE; e += blockDim.x) {
            const int rr = e / GQ_TILE, cc = e % GQ_TILE;
            const int64_t r = r0 + rr;
            xa[rr][cc] = (r < R && i0 + cc < K) ? x[r * K + i0 + cc] : 0.0f;
            xb[rr][cc] = (r < R && j0 + cc < K) ? x[r * K + j0 + cc] : 0.0f;
        }
        __syncthreads();
        const int rn = (int)((R - r0) < GQ_TILE ? (R - r0) : GQ_TILE);
        for (int rr = 0; rr < rn; ++rr) {
            const double xj = (double)xb[rr][tx];
#pragma unroll
            for (int m = 0; m < GQ_TILE / GQ_ROWS; ++m)
                acc[m] = __dadd_rn(acc[m], __dmul_rn((double)xa[rr][ty + GQ_ROWS * m], xj));
        }
        __syncthreads();
    }
    const int j = j0 + tx;
#pragma unroll
    for (int m = 0; m < GQ_TILE / GQ_ROWS; ++m) {
        const int i = i0 + ty + GQ_ROWS * m;
        if (i >= K || j >= K || i > j) continue;          // (j, i) writes this pair
        const double v = reset ? acc[m] : __dadd_rn(H[(int64_t)i * K + j], acc[m]);
        H[(int64_t)i * K + j] = v;
        if (i != j) H[(int64_t)j * K + i] = v;
    }
}

// ----------------------------------------------------- damped Hessian, dead columns
// A = H with dead diagonal entries set to 1 (off-diagonal copy; the diagonal is written
// by k_gptq_diag).
__global__ void k_gptq_copy(const double* __restrict__ H, int K, double* __restrict__ A) {
    const int64_t n = (int64_t)K * K;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
         e += (int64_t)gridDim.x * blockDim.x)
        A[e] = H[e];
}

// One CTA: dead flags, the diagonal mean (a sequential sum in k, as the reference), the
// damping term damp * mean added to every diagonal entry.
__global__ void k_gptq_diag(const double* __restrict__ H, int K, double damp,
                            double* __restrict__ A, unsigned char* __restrict__ dead) {
    __shared__ double add;
    if (threadIdx.x == 0) {
        double tr = 0.0;
        for (int k = 0; k < K; ++k) {
            const double d = H[(int64_t)k * K + k];
            tr = __dadd_rn(tr, d == 0.0 ? 1.0 : d);
        }
        add = __dmul_rn(damp, __ddiv_rn(tr, (double)K));
    }
    __syncthreads();
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const double d = H[(int64_t)k * K + k];
        dead[k] = d == 0.0;
        A[(int64_t)k * K + k] = __dadd_rn(d == 0.0 ? 1.0 : d, add);
    }
}

// ---------------------------------------------------------------- Cholesky, step k
// T holds A with the subtractions of pivots < k applied (row-major, lower triangle used).
// Step k, one launch over 32 x 32 tiles of the trailing triangle {(i, j): k < j <= i < K}:
//   L[k, k] = d = sqrt(T[k, k]),  L[i, k] = T[i, k] / d   (written by the first tile column)
//   T[i, j] = T[i, j] - L[i, k] * L[j, k]
// Each tile divides its own 32 + 32 entries of column k into shared memory (the same
// correctly rounded divisions wherever they are repeated, so the same bits).  Every entry of
// L is the left-looking sequential formula of the reference: its subtractions arrive in
// ascending k.  Column k of T is only read in step k.
__global__ __launch_bounds__(256) void k_chol_step(double* __restrict__ T, double* __restrict__ L,
                                                   int K, int k, int* status) {
    __shared__ double li[32], lj[32];
    const int i0 = k + 1 + blockIdx.y * 32, j0 = k + 1 + blockIdx.x * 32;
    if (j0 > i0 + 31) return;                            // tile above the diagonal
    const double tkk = T[(int64_t)k * K + k];
    const double d = __dsqrt_rn(tkk);
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
        L[(int64_t)k * K + k] = d;
        if (!(tkk > 0.0) && status) atomicExch(status, kStatusNotPositiveDefinite);
    }
    if (threadIdx.x < 32) {
        const int i = i0 + threadIdx.x;
        if (i < K) {
            li[threadIdx.x] = __ddiv_rn(T[(int64_t)i * K + k], d);
            if (blockIdx.x == 0) L[(int64_t)i * K + k] = li[threadIdx.x];
        }
    } else if (threadIdx.x < 64) {
        const int j = j0 + threadIdx.x - 32;
        if (j < K) lj[threadIdx.x - 32] = __ddiv_rn(T[(int64_t)j * K + k], d);
    }
    __syncthreads();
    const int c = threadIdx.x & 31, j = j0 + c;
    if (j >= K) return;
    for (int r = threadIdx.x >> 5; r < 32; r += 8) {
        const int i = i0 + r;
        if (i < K && j <= i) T[(int64_t)i * K + j] = dsub_mul(T[(int64_t)i * K + j], li[r], lj[c]);
    }
}

// ------------------------------------------------------- inverse of L, step k
// Column-oriented forward substitution for every column j at once.  S holds the running
// sums t[i, j] = 0 - sum_{k' < k} L[i, k'] Li[k', j] (row-major; zero-initialised).
// Step k, one launch over 32 x 32 tiles of {(i, j): k < i < K, j <= k} (at least one tile
// row, so that row k is written even when k = K - 1):
//   Li[k, j] = S[k, j] / L[k, k] (j < k),  Li[k, k] = 1 / L[k, k]  (first tile row writes)
//   S[i, j] = S[i, j] - L[i, k] * Li[k, j]
__global__ __launch_bounds__(256) void k_trinv_step(const double* __restrict__ L,
                                                    double* __restrict__ S,
                                                    double* __restrict__ Li, int K, int k) {
    __shared__ double y[32];
    const int j0 = blockIdx.x * 32, i0 = k + 1 + blockIdx.y * 32;
    const double lkk = L[(int64_t)k * K + k];
    if (threadIdx.x < 32) {
        const int j = j0 + threadIdx.x;
        if (j <= k) {
            y[threadIdx.x] =
                (j == k) ? __ddiv_rn(1.0, lkk) : __ddiv_rn(S[(int64_t)k * K + j], lkk);
            if (blockIdx.y == 0) Li[(int64_t)k * K + j] = y[threadIdx.x];
        }
    }
    __syncthreads();
    const int c = threadIdx.x & 31, j = j0 + c;
    if (j > k) return;
    for (int r = threadIdx.x >> 5; r < 32; r += 8) {
        const int i = i0 + r;
        if (i < K) S[(int64_t)i * K + j] = dsub_mul(S[(int64_t)i * K + j], L[(int64_t)i * K + k], y[c]);
    }
}

// U = LA^T (exact copies), so that the block updates read rows of U: coalesced across the
// later columns j.
__global__ __launch_bounds__(256) void k_transpose(const double* __restrict__ A, int K,
                                                   double* __restrict__ B) {
    __shared__ double t[32][33];
    const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32, c = threadIdx.x & 31;
    for (int r = threadIdx.x >> 5; r < 32; r += 8)
        if (i0 + r < K && j0 + c < K) t[r][c] = A[(int64_t)(i0 + r) * K + j0 + c];
    __syncthreads();
    for (int r = threadIdx.x >> 5; r < 32; r += 8)
        if (j0 + r < K && i0 + c < K) B[(int64_t)(j0 + r) * K + i0 + c] = t[c][r];
}

// -------------------------------------------------------- H^-1 = Li^T Li
// G[i, j] = sum_{k = max(i, j)}^{K-1} Li[k, i] * Li[k, j] (ascending), upper tiles
// computed and mirrored.
__global__ __launch_bounds__(GQ_TILE * GQ_ROWS) void k_inv_gram(const double* __restrict__ Li,
                                                               int K, double* __restrict__ G) {
    const int ti = blockIdx.y, tj = blockIdx.x;
    if (tj < ti) return;
    __shared__ double la[GQ_TILE][GQ_TILE + 1];
    __shared__ double lb[GQ_TILE][GQ_TILE + 1];
    const int tx = threadIdx.x % GQ_TILE, ty = threadIdx.x / GQ_TILE;
    const int i0 = ti * GQ_TILE, j0 = tj * GQ_TILE;
    const int j = j0 + tx;
    double acc[GQ_TILE / GQ_ROWS];
#pragma unroll
    for (int m = 0; m < GQ_TILE / GQ_ROWS; ++m) acc[m] = 0.0;
    for (int k0 = j0; k0 < K; k0 += GQ_TILE) {     // rows k < j0 hold zeros of column j
        for (int e = threadIdx.x; e < GQ_TILE * GQ_TILE; e += blockDim.x) {
            const int kk = e / GQ_TILE, cc = e % GQ_TILE;
            const int k = k0 + kk;
            la[kk][cc] = (k < K && i0 + cc < K) ? Li[(int64_t)k * K + i0 + cc] : 0.0;
            lb[kk][cc] = (k < K && j0 + cc < K) ? Li[(int64_t)k * K + j0 + cc] : 0.0;
        }
        __syncthreads();
        for (int kk = 0; kk < GQ_TILE; ++kk) {
            const int k = k0 + kk;
            if (k >= K) break;
            const double lj = lb[kk][tx];
#pragma unroll
            for (int m = 0; m < GQ_TILE / GQ_ROWS; ++m) {
                const int i = i0 + ty + GQ_ROWS * m;
                if (k >= (i > j ? i : j))
                    acc[m] = __dadd_rn(acc[m], __dmul_rn(la[kk][ty + GQ_ROWS * m], lj));
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int m = 0; m < GQ_TILE / GQ_ROWS; ++m) {
        const int i = i0 + ty + GQ_ROWS * m;
        if (i >= K || j >= K || i > j) continue;
        G[(int64_t)i * K + j] = acc[m];
        G[(int64_t)j * K + i] = acc[m];
    }
}

// ------------------------------------------------------------------ GPTQ passes
// w = the fp64 working copy of W with dead columns zeroed.
__global__ void k_gptq_init_w(const float* __restrict__ W, const unsigned char* __restrict__ dead,
                              int64_t N, int K, double* __restrict__ w) {
    const int64_t n = N * K;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
         e += (int64_t)gridDim.x * blockDim.x)
        w[e] = dead[e % K] ? 0.0 : (double)W[e];
}

// The block [i1, i2): one thread per row, the block's columns in order.  U is the upper
// factor of H^-1 (row-major).  Codes go to q, the scaled errors to err[n, 0..B), and the code
// sum accumulates in wsum (initialised by the first block).
__global__ __launch_bounds__(GQ_ROW_THREADS) void k_gptq_block(
    double* __restrict__ w, const double* __restrict__ U, const float* __restrict__ s_w,
    int64_t N, int K, int i1, int i2, int8_t* __restrict__ q, double* __restrict__ err,
    int32_t* __restrict__ wsum) {
    extern __shared__ double w1s[];                      // [GQ_ROW_THREADS][B + 1]
    const int B = i2 - i1;
    const int64_t n = blockIdx.x * (int64_t)GQ_ROW_THREADS + threadIdx.x;
    if (n >= N) return;
    double* w1 = w1s + threadIdx.x * (B + 1);
    double* wr = w + n * K;
    for (int t = 0; t < B; ++t) w1[t] = wr[i1 + t];
    const double s = (double)s_w[n];
    int sum = 0;
    for (int t = 0; t < B; ++t) {
        const int i = i1 + t;
        const double col = w1[t];
        double qc = rint(__ddiv_rn(col, s));
        qc = fmin(fmax(qc, -128.0), 127.0);
        q[n * K + i] = (int8_t)(int)qc;
        sum += (int)qc;
        const double e = __ddiv_rn(__dsub_rn(col, __dmul_rn(qc, s)), U[(int64_t)i * K + i]);
        for (int u = t; u < B; ++u) w1[u] = dsub_mul(w1[u], e, U[(int64_t)i * K + i1 + u]);
        err[n * GQ_BLOCK_MAX + t] = e;
    }
    if (wsum) wsum[n] = (i1 == 0 ? 0 : wsum[n]) + sum;
}

// w[n, j] -= sum_{t ascending} err[n, t] * U[i1 + t, j] for j >= i2.
__global__ __launch_bounds__(128) void k_gptq_update(double* __restrict__ w,
                                                     const double* __restrict__ U,
                                                     const double* __restrict__ err, int64_t N,
                                                     int K, int i1, int i2) {
    const int j = i2 + blockIdx.x * 128 + threadIdx.x;
    __shared__ double e[GQ_BLOCK_MAX];
    const int B = i2 - i1;
    const double* ut = U + (int64_t)i1 * K + (j < K ? j : 0);    // U[i1 + t, j] at ut[t * K]
    for (int64_t n = blockIdx.y; n < N; n += gridDim.y) {
        __syncthreads();                                 // e[] of the previous row is consumed
        for (int t = threadIdx.x; t < B; t += 128) e[t] = err[n * GQ_BLOCK_MAX + t];
        __syncthreads();
        if (j >= K) continue;
        double p = 0.0;
        for (int t = 0; t < B; ++t) p = __dadd_rn(p, __dmul_rn(e[t], ut[(int64_t)t * K]));
        w[n * K + j] = __dsub_rn(w[n * K + j], p);
    }
}

// ------------------------------------------------------------------- launchers
static unsigned grid_for(int64_t n, int threads, int cap) {
    int64_t b = (n + threads - 1) / threads;
    if (b > cap) b = cap;
    return (unsigned)(b < 1 ? 1 : b);
}

cudaError_t launch_hessian_accumulate(const float* x, int64_t R, int K, double* H, int reset,
                                      cudaStream_t st) {
    const unsigned t = (unsigned)((K + GQ_TILE - 1) / GQ_TILE);
    k_gram_acc<<<dim3(t, t), GQ_TILE * GQ_ROWS, 0, st>>>(x, R, K, H, reset);
    return cudaGetLastError();
}

GptqPlan plan_gptq(int64_t N, int64_t K) {
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    GptqPlan p;
    const size_t kk = (size_t)K * K * sizeof(double);
    p.buf0 = 0;
    p.buf1 = up(p.buf0 + kk);
    p.buf2 = up(p.buf1 + kk);
    p.w = up(p.buf2 + kk);
    p.err = up(p.w + (size_t)N * K * sizeof(double));
    p.dead = up(p.err + (size_t)N * GQ_BLOCK_MAX * sizeof(double));
    p.bytes = up(p.dead + (size_t)K);
    return p;
}

bool gptq_block_ok(int64_t block) { return block >= 1 && block <= GQ_BLOCK_MAX; }

// Lower Cholesky factor of T (consumed) into L: one launch per pivot.
static cudaError_t chol(double* T, double* L, int K, cudaStream_t st, int* status) {
    for (int k = 0; k < K; ++k) {
        const int m = K - k - 1;
        const unsigned t = (unsigned)(m > 0 ? (m + 31) / 32 : 1);
        k_chol_step<<<dim3(t, t), 256, 0, st>>>(T, L, K, k, status);
    }
    return cudaGetLastError();
}

cudaError_t launch_gptq_int8(const float* W, const double* H, int64_t N, int K, double damp,
                             int block, int8_t* q, float* s_w, int32_t* wsum, void* ws,
                             cudaStream_t st, int num_sms, int* status) {
    const GptqPlan p = plan_gptq(N, K);
    uint8_t* base = static_cast<uint8_t*>(ws);
    double* b0 = reinterpret_cast<double*>(base + p.buf0);
    double* b1 = reinterpret_cast<double*>(base + p.buf1);
    double* b2 = reinterpret_cast<double*>(base + p.buf2);
    double* w = reinterpret_cast<double*>(base + p.w);
    double* err = reinterpret_cast<double*>(base + p.err);
    unsigned char* dead = base + p.dead;
    const int64_t kk = (int64_t)K * K;
    const int cap = 8 * num_sms;
    // scales of the original rows (weight_int8's grid); q and wsum are rewritten below
    cudaError_t e = launch_quantize_weight(W, N, K, 1, q, s_w, nullptr, st);
    if (e != cudaSuccess) return e;
    // A = damped H in b0; L = chol(A) in b1 (A is consumed as the trailing matrix)
    k_gptq_copy<<<grid_for(kk, 256, cap), 256, 0, st>>>(H, K, b0);
    k_gptq_diag<<<1, 256, 0, st>>>(H, K, damp, b0, dead);
    if ((e = chol(b0, b1, K, st, status)) != cudaSuccess) return e;
    // Li = L^-1 in b2, running sums in b0 (zeroed)
    if ((e = cudaMemsetAsync(b0, 0, (size_t)kk * sizeof(double), st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(b2, 0, (size_t)kk * sizeof(double), st)) != cudaSuccess) return e;
    for (int k = 0; k < K; ++k) {
        const int rows = K - k - 1;
        k_trinv_step<<<dim3((unsigned)((k + 32) / 32), (unsigned)(rows > 0 ? (rows + 31) / 32 : 1)),
                       256, 0, st>>>(b1, b0, b2, K, k);
    }
    // H^-1 = Li^T Li in b1, then its lower factor LA in b0 (U = LA^T)
    const unsigned t = (unsigned)((K + GQ_TILE - 1) / GQ_TILE);
    k_inv_gram<<<dim3(t, t), GQ_TILE * GQ_ROWS, 0, st>>>(b2, K, b1);
    if ((e = chol(b1, b0, K, st, status)) != cudaSuccess) return e;
    // U = LA^T in b2 (Li is no longer needed)
    k_transpose<<<dim3(t, t), 256, 0, st>>>(b0, K, b2);
    // the column blocks
    k_gptq_init_w<<<grid_for(N * K, 256, cap), 256, 0, st>>>(W, dead, N, K, w);
    const size_t smem = (size_t)GQ_ROW_THREADS * (block + 1) * sizeof(double);
    if ((e = ensure_dyn_smem<k_gptq_block>((int)smem)) != cudaSuccess) return e;
    for (int i1 = 0; i1 < K; i1 += block) {
        const int i2 = i1 + block < K ? i1 + block : K;
        k_gptq_block<<<(unsigned)((N + GQ_ROW_THREADS - 1) / GQ_ROW_THREADS), GQ_ROW_THREADS,
                       smem, st>>>(w, b2, s_w, N, K, i1, i2, q, err, wsum);
        if (i2 < K)
            k_gptq_update<<<dim3((unsigned)((K - i2 + 127) / 128),
                                 (unsigned)(N < 65535 ? N : 65535)),
                            128, 0, st>>>(w, b2, err, N, K, i1, i2);
    }
    return cudaGetLastError();
}

}  // namespace q8

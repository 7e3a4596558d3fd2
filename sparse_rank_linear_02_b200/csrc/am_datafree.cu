// am_datafree.cu -- data-free alternating minimisation W ~ S + U V on the GPU
// (S 2:4 sparse, U V of rank r).
//
// The method (HASSLE-free, section 4, data-free variant; LoSparse, section
// 3.2, for the start): the low-rank block starts from the top-r singular
// subspace of W; then every iteration solves
//   P2: U V = C_r(W - S)          (truncated SVD, HASSLE-free section 4.2.1)
//   P1: S = 2:4 hard threshold of W - U V   (HASSLE-free section 4.1.1).
//
// C_r is computed by subspace iteration on Z = W - S, warm-started from the
// previous iteration's right subspace Q (d_in x r, orthonormal columns):
//   repeat p times:  P = Z Q;  Q = orth(Z^T P)      (Cholesky QR: one pass
//   between power steps, two (CholeskyQR2) on the last)
//   then U = Z Q, V = Q^T, so U V = Z Q Q^T, the best rank-r fit of Z within
//   span(Q), which converges to C_r(Z) as Q converges to the top-r right
//   singular subspace.  The random start Q0 is an input.
//
// Kernels:
//  * the products P = Z Q, Z^T P and U = Z Q run on the tensor cores
//    (tc_gemm_kernel, tc_gemm.cuh) with every operand split into two bf16
//    planes, hi = bf16(x) and lo = bf16(x - hi), and hi*hi + hi*lo + lo*hi
//    accumulated in fp32: about 16 significant bits per operand, so the
//    subspace iteration behaves as in fp32.  Z = W - S is kept as its two
//    planes (written by the P1 product below); Q and P are split before use.
//  * gemm_tn_f32_kernel: C = A^T B in fp32 on CUDA cores, for the small Gram
//    product of the orthonormalisation (Q^T Q, r x r over d_in).
//    128 x 64 output tiles, 16-deep k steps through shared memory, split over
//    k with the partial products summed in a fixed order by
//    reduce_splits_kernel (deterministic).
//  * chol_kernel: one CTA; G = Q^T Q (fp64) -> Cholesky factor L (one
//    barrier per step); solve_rows_kernel: Q <- Q L^-T, one warp per row of
//    Q, so Q has orthonormal columns.
//  * P1 is the same tensor-core product P Q^T (split planes, K = r) with the
//    threshold in its epilogue (tc_gemm_kernel's residual mode): per group of
//    four columns R = W - P Q^T, the two largest |R| kept (ties to the lower
//    index) and written packed (bf16 values, nibble metadata), Z = W - S
//    written as its two bf16 planes for the next subspace iteration, and the
//    CTA's sum of (R - S)^2 as a partial of the objective.
#include <math.h>

#include <algorithm>

#include "tc_gemm.cuh"

namespace slr {

// Error word of the tensor-core products' bounded waits (slr_check_kernel_error).
__device__ unsigned int g_am_error = 0;

namespace {

constexpr int kGT = 256;   // threads of the GEMM kernels
constexpr int kGBM = 128;  // output rows per tile
constexpr int kGBN = 64;   // output columns per tile
constexpr int kGBK = 16;   // k per shared-memory step

// C_part[split] (rows x cols, row-major, ldc = cols) = A^T B over the k range
// of this split: A is kdim x rows (lda), B is kdim x cols (ldb).
__global__ void __launch_bounds__(kGT) gemm_tn_f32_kernel(const float *__restrict__ A, int64_t lda,
                                                          const float *__restrict__ B, int64_t ldb,
                                                          float *__restrict__ Cpart, int64_t rows, int64_t cols,
                                                          int64_t kdim, int64_t k_per_split) {
    __shared__ __align__(16) float As[kGBK][kGBM];
    __shared__ __align__(16) float Bs[kGBK][kGBN];
    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;          // 4 columns x 8 rows per thread
    const int64_t r0 = (int64_t)blockIdx.x * kGBM, c0 = (int64_t)blockIdx.y * kGBN;
    const int64_t k_begin = (int64_t)blockIdx.z * k_per_split;
    int64_t k_end = k_begin + k_per_split;
    if (k_end > kdim) k_end = kdim;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int64_t k0 = k_begin; k0 < k_end; k0 += kGBK) {
        // A tile -> As[k][row]: 16 k (rows of A) x 128 output rows (columns of
        // A), coalesced rows; each thread two 4-wide pieces.
        {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int idx = tid + h * kGT;       // 0..511
                const int kk = idx / 32, cq = (idx % 32) * 4;
                const int64_t gk = k0 + kk, gc = r0 + cq;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (gk < k_end) {
                    if (gc + 3 < rows) {
                        v = *reinterpret_cast<const float4 *>(A + gk * lda + gc);
                    } else {
                        if (gc + 0 < rows) v.x = A[gk * lda + gc + 0];
                        if (gc + 1 < rows) v.y = A[gk * lda + gc + 1];
                        if (gc + 2 < rows) v.z = A[gk * lda + gc + 2];
                    }
                }
                *reinterpret_cast<float4 *>(&As[kk][cq]) = v;
            }
        }
        // B tile -> Bs[k][col]: 16 x 64, one 4-wide piece per thread.
        {
            const int kk = tid / 16, cq = (tid % 16) * 4;
            const int64_t gk = k0 + kk, gc = c0 + cq;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (gk < k_end) {
                if (gc + 3 < cols) {
                    v = *reinterpret_cast<const float4 *>(B + gk * ldb + gc);
                } else {
                    if (gc + 0 < cols) v.x = B[gk * ldb + gc + 0];
                    if (gc + 1 < cols) v.y = B[gk * ldb + gc + 1];
                    if (gc + 2 < cols) v.z = B[gk * ldb + gc + 2];
                }
            }
            *reinterpret_cast<float4 *>(&Bs[kk][cq]) = v;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kGBK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4 *>(&As[kk][ty * 8]);
            const float4 a1 = *reinterpret_cast<const float4 *>(&As[kk][ty * 8 + 4]);
            const float4 b = *reinterpret_cast<const float4 *>(&Bs[kk][tx * 4]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
        }
        __syncthreads();
    }
    float *C = Cpart + (int64_t)blockIdx.z * rows * cols;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t gr = r0 + ty * 8 + i;
        if (gr >= rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t gc = c0 + tx * 4 + j;
            if (gc < cols) C[gr * cols + gc] = acc[i][j];
        }
    }
}

// out = sum over splits of part[s] (n floats each), in split order.
__global__ void reduce_splits_kernel(const float *__restrict__ part, int splits, int64_t n,
                                     float *__restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        float s = 0.f;
        for (int k = 0; k < splits; ++k) s += part[k * n + i];
        out[i] = s;
    }
}

// One CTA: G = sum of `splits` partial r x r Gram matrices (fp64), Cholesky
// G = L L^T (a pivot below 1e-12 of the mean diagonal is raised to it, so a
// rank-deficient block stays finite), written as fp32 L (r x r row-major,
// zero above the diagonal).  Shared memory: the r x r fp64 array with rows
// padded to r + 1 (an odd stride, so column accesses do not collide in one
// bank) and r square roots.  The factorisation is a chain of r steps, so the
// kernel is bound by the barrier between steps; the scaling of each column
// is deferred to keep one barrier per step: for column j (d_j = the current
// A[j][j], floored), A[i][k] -= A[i][j] A[k][j] / d_j for j < k <= i, and at
// the end L[j][j] = sqrt(d_j), L[i][j] = A[i][j] / sqrt(d_j).
__global__ void __launch_bounds__(1024) chol_kernel(const float *__restrict__ gpart, int splits, int r,
                                                   float *__restrict__ Lout) {
    extern __shared__ double A[];  // r rows of ld = r + 1, then r square roots
    __shared__ double floor_pivot;
    const int tid = threadIdx.x, nth = blockDim.x, ld = r + 1;
    const int tx = tid & 31, ty = tid >> 5, ny = nth >> 5;
    double *sq = A + r * ld;
    for (int i = tid; i < r * r; i += nth) {
        double s = 0.0;
        for (int k = 0; k < splits; ++k) s += (double)gpart[(int64_t)k * r * r + i];
        A[(i / r) * ld + i % r] = s;
    }
    __syncthreads();
    if (tid == 0) {
        double tr = 0.0;
        for (int i = 0; i < r; ++i) tr += A[i * ld + i];
        floor_pivot = 1e-12 * (tr > 0.0 ? tr / r : 1.0);
    }
    __syncthreads();
    const double fl = floor_pivot;
    for (int j = 0; j < r; ++j) {
        const double d = A[j * ld + j];
        const double inv2 = 1.0 / (d > fl ? d : fl);
        for (int i = j + 1 + ty; i < r; i += ny) {
            const double f = A[i * ld + j] * inv2;
            for (int k = j + 1 + tx; k <= i; k += 32) A[i * ld + k] -= f * A[k * ld + j];
        }
        __syncthreads();
    }
    for (int j = tid; j < r; j += nth) {
        const double d = A[j * ld + j];
        sq[j] = sqrt(d > fl ? d : fl);
    }
    __syncthreads();
    for (int q = tid; q < r * r; q += nth) {
        const int i = q / r, c = q % r;  // L (fp32, row-major, zero above the diagonal)
        Lout[q] = c < i ? (float)(A[i * ld + c] / sq[c]) : (c == i ? (float)sq[i] : 0.f);
    }
}

// Q <- Q L^-T in place: every row of Q solves x L^T = q by forward
// substitution, x[c] = (q[c] - sum_{k<c} x[k] L[c][k]) / L[c][c].  One warp
// per row: lane l holds x[l], x[l + 32], x[l + 64], x[l + 96] (r <= 128); each
// step's sum is split over the lanes and reduced with shuffles.  L (fp32) is
// read from shared memory (consecutive k across lanes: no bank conflicts).
constexpr int kSolveWarps = 8;
__global__ void __launch_bounds__(kSolveWarps * 32) solve_rows_kernel(float *__restrict__ Q, int64_t n_rows, int r,
                                                                      const float *__restrict__ L) {
    extern __shared__ float Ls[];  // r x r
    for (int i = threadIdx.x; i < r * r; i += kSolveWarps * 32) Ls[i] = L[i];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kSolveWarps + (threadIdx.x >> 5);
    if (row >= n_rows) return;  // warp-uniform; no barrier follows
    float q[4], x[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const int k = lane + 32 * h;
        q[h] = k < r ? Q[row * r + k] : 0.f;
        x[h] = 0.f;
    }
    for (int c = 0; c < r; ++c) {
        const float *lc = Ls + c * r;
        float part = 0.f;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const int k = lane + 32 * h;
            if (k < c) part = fmaf(x[h], lc[k], part);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xFFFFFFFFu, part, o);
        const int h = c >> 5;
        if (lane == (c & 31)) {
            const float qc = h == 0 ? q[0] : (h == 1 ? q[1] : (h == 2 ? q[2] : q[3]));
            const float xc = (qc - part) / lc[c];
            if (h == 0) x[0] = xc;
            else if (h == 1) x[1] = xc;
            else if (h == 2) x[2] = xc;
            else x[3] = xc;
        }
    }
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const int k = lane + 32 * h;
        if (k < r) Q[row * r + k] = x[h];
    }
}

// objective[t] = sqrt(sum of the tile partials), summed in fp64 in tile order.
__global__ void objective_finish_kernel(const float *__restrict__ part, int64_t n, double *__restrict__ out) {
    __shared__ double red[256];
    double s = 0.0;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += (double)part[i];
    red[threadIdx.x] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int k = 0; k < (int)blockDim.x; ++k) t += red[k];
        *out = sqrt(t);
    }
}

// hi = bf16(x), lo = bf16(x - hi), elementwise.
__global__ void split_bf16_kernel(const float *__restrict__ in, int64_t n, uint16_t *__restrict__ hi,
                                  uint16_t *__restrict__ lo) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float x = in[i];
        const uint16_t h = f32_to_bf16_bits(x);
        hi[i] = h;
        lo[i] = f32_to_bf16_bits(x - __uint_as_float((uint32_t)h << 16));
    }
}

// U = bf16(P) [d_out, r]; V[k][j] = bf16(Q[j][k]) [r, d_in].
__global__ void factors_out_kernel(const float *__restrict__ P, const float *__restrict__ Q, int64_t d_out,
                                   int64_t d_in, int r, uint16_t *__restrict__ U, uint16_t *__restrict__ V) {
    const int64_t nu = d_out * r, nv = (int64_t)r * d_in;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nu + nv;
         i += (int64_t)gridDim.x * blockDim.x) {
        if (i < nu) {
            U[i] = f32_to_bf16_bits(P[i]);
        } else {
            const int64_t v = i - nu, k = v / d_in, j = v - k * d_in;
            V[v] = f32_to_bf16_bits(Q[j * r + k]);
        }
    }
}

// U32 = P [d_out, r] and V32[k][j] = Q[j][k] [r, d_in], both fp32 (the
// factors before their rounding to bf16).
__global__ void factors_f32_kernel(const float *__restrict__ P, const float *__restrict__ Q, int64_t d_out,
                                   int64_t d_in, int r, float *__restrict__ U32, float *__restrict__ V32) {
    const int64_t nu = d_out * r, nv = (int64_t)r * d_in;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nu + nv;
         i += (int64_t)gridDim.x * blockDim.x) {
        if (i < nu) {
            if (U32 != nullptr) U32[i] = P[i];
        } else if (V32 != nullptr) {
            const int64_t v = i - nu, k = v / d_in, j = v - k * d_in;
            V32[v] = Q[j * r + k];
        }
    }
}

int grid_cap(int64_t n, int threads) {
    const int64_t b = (n + threads - 1) / threads;
    return (int)(b < 148 * 16 ? (b > 0 ? b : 1) : 148 * 16);
}

}  // namespace

// ----------------------------------------------------------------------------- host driver

AmPlan am_plan(int64_t d_out, int64_t d_in, int64_t r) {
    AmPlan p{};
    // The Gram matrix Q^T Q (r x r, k = d_in) is split over k, 64 rows of Q
    // per CTA (at most 128 CTAs); its partials live in `part`.
    int64_t sg = (d_in + 63) / 64;
    p.split_gram = sg > 128 ? 128 : (sg < 1 ? 1 : sg);
    const int64_t part = p.split_gram * r * r;
    p.tiles_res = ((d_in + 127) / 128) * ((d_out + 127) / 128);  // CTAs of the fused residual product
    auto al = [](int64_t b) { return (b + 255) / 256 * 256; };
    p.off_Z = 0;                                   // Zhi then Zlo, bf16 d_out x d_in each
    p.off_Q = p.off_Z + 2 * al(d_out * d_in * 2);
    p.off_Q2 = p.off_Q + al(d_in * r * 4);
    p.off_P = p.off_Q2 + al(d_in * r * 4);
    p.off_M = p.off_P + al(d_out * r * 4);
    p.off_part = p.off_M + al(r * r * 4);
    p.off_obj = p.off_part + al(part * 4);
    p.off_split = p.off_obj + al(p.tiles_res * 4);  // hi and lo planes of Q or P (bf16, max(d_in, d_out) x r)
    p.off_split2 = p.off_split + 2 * al(std::max(d_in, d_out) * r * 2);  // hi and lo planes of Q (d_in x r)
    p.bytes = p.off_split2 + 2 * al(d_in * r * 2);
    return p;
}

namespace {

// out (rows x cols) = A^T B with A kdim x rows and B kdim x cols, k split over
// `splits` CTAs whose partials are summed in a fixed order.
cudaError_t gemm_tn(const float *A, int64_t lda, const float *B, int64_t ldb, float *out, float *part,
                    int64_t rows, int64_t cols, int64_t kdim, int64_t splits, cudaStream_t st) {
    int64_t kps = (kdim + splits - 1) / splits;
    kps = (kps + kGBK - 1) / kGBK * kGBK;
    const int64_t used = (kdim + kps - 1) / kps;
    dim3 grid((unsigned)((rows + kGBM - 1) / kGBM), (unsigned)((cols + kGBN - 1) / kGBN), (unsigned)used);
    float *dst = used == 1 ? out : part;
    gemm_tn_f32_kernel<<<grid, kGT, 0, st>>>(A, lda, B, ldb, dst, rows, cols, kdim, kps);
    if (used > 1) reduce_splits_kernel<<<grid_cap(rows * cols, 256), 256, 0, st>>>(part, (int)used, rows * cols, out);
    return cudaGetLastError();
}

// Q (d_in x r) <- Q L^-T with L the Cholesky factor of Q^T Q; tmp is d_in x r.
cudaError_t orthonormalise(float *Q, float *tmp, float *M, float *part, int64_t d_in, int r, int64_t split_gram,
                           int passes, cudaStream_t st) {
    for (int pass = 0; pass < passes; ++pass) {  // 2: CholeskyQR2
        // G = Q^T Q into the first r x r floats of tmp (split over d_in, the
        // splits summed in a fixed order), its Cholesky factor L into M, then
        // Q <- Q L^-T by forward substitution on every row.
        cudaError_t e = gemm_tn(Q, r, Q, r, tmp, part, r, r, d_in, split_gram, st);
        if (e != cudaSuccess) return e;
        // 32 warps: each step's trailing update gives a warp one or two rows,
        // which keeps the per-step chain short (the kernel is latency-bound).
        chol_kernel<<<1, 1024, (size_t)r * (r + 2) * sizeof(double), st>>>(tmp, 1, r, M);
        solve_rows_kernel<<<(unsigned)((d_in + kSolveWarps - 1) / kSolveWarps), kSolveWarps * 32,
                            (size_t)r * r * sizeof(float), st>>>(Q, d_in, r, M);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}


// Device address of g_am_error on the current device.
unsigned int *am_err() {
    static unsigned int *addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (addr[dev] == nullptr) {
        void *q = nullptr;
        if (cudaGetSymbolAddress(&q, g_am_error) == cudaSuccess) addr[dev] = static_cast<unsigned int *>(q);
    }
    return addr[dev];
}

// C (rows x r, fp32) = Z B (B: d_in x r) or Z^T B (B: d_out x r) on the tensor
// cores, with Z and B in hi/lo bf16 planes; B (fp32) is split into bh/bl first.
cudaError_t split_product(bool transpose_z, const uint16_t *Zhi, const uint16_t *Zlo, int64_t d_out, int64_t d_in,
                          const float *B, uint16_t *bh, uint16_t *bl, int r, float *C, cudaStream_t st) {
    const int64_t kdim = transpose_z ? d_out : d_in, rows = transpose_z ? d_in : d_out;
    split_bf16_kernel<<<grid_cap(kdim * r, 256), 256, 0, st>>>(B, kdim * r, bh, bl);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (r <= 64)
        return transpose_z ? gemm_tc<true, true, 64, kOutF32, true>(Zhi, Zlo, d_in, bh, bl, r, rows, r, kdim, C, am_err(), st)
                           : gemm_tc<false, true, 64, kOutF32, true>(Zhi, Zlo, d_in, bh, bl, r, rows, r, kdim, C, am_err(), st);
    return transpose_z ? gemm_tc<true, true, 128, kOutF32, true>(Zhi, Zlo, d_in, bh, bl, r, rows, r, kdim, C, am_err(), st)
                       : gemm_tc<false, true, 128, kOutF32, true>(Zhi, Zlo, d_in, bh, bl, r, rows, r, kdim, C, am_err(), st);
}

}  // namespace

cudaError_t launch_am_factors_f32(const uint8_t *ws, int64_t d_out, int64_t d_in, int r, float *U32, float *V32,
                                  cudaStream_t st) {
    const AmPlan p = am_plan(d_out, d_in, r);
    const float *Q = reinterpret_cast<const float *>(ws + p.off_Q);
    const float *P = reinterpret_cast<const float *>(ws + p.off_P);
    factors_f32_kernel<<<grid_cap((d_out + d_in) * r, 256), 256, 0, st>>>(P, Q, d_out, d_in, r, U32, V32);
    return cudaGetLastError();
}

cudaError_t read_and_clear_am_error(unsigned *code) {
    unsigned v = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_am_error, sizeof v);
    if (err != cudaSuccess) return err;
    if (v != 0) {
        const unsigned zero = 0;
        err = cudaMemcpyToSymbol(g_am_error, &zero, sizeof zero);
    }
    *code = v;
    return err;
}

cudaError_t launch_am_datafree(const uint16_t *W, int64_t d_out, int64_t d_in, int r, int iters, int power0,
                               int power, const float *Q0, uint16_t *vals, uint8_t *meta, uint16_t *U, uint16_t *V,
                               double *objective, uint8_t *ws, cudaStream_t st) {
    const AmPlan p = am_plan(d_out, d_in, r);
    uint16_t *Zhi = reinterpret_cast<uint16_t *>(ws + p.off_Z);
    uint16_t *Zlo = Zhi + (p.off_Q - p.off_Z) / 4;  // second half of the Z region
    float *Q = reinterpret_cast<float *>(ws + p.off_Q);
    float *Q2 = reinterpret_cast<float *>(ws + p.off_Q2);
    float *P = reinterpret_cast<float *>(ws + p.off_P);
    float *M = reinterpret_cast<float *>(ws + p.off_M);
    float *part = reinterpret_cast<float *>(ws + p.off_part);
    float *objp = reinterpret_cast<float *>(ws + p.off_obj);
    uint16_t *bh = reinterpret_cast<uint16_t *>(ws + p.off_split);
    uint16_t *bl = bh + (p.off_split2 - p.off_split) / 4;
    uint16_t *qh = reinterpret_cast<uint16_t *>(ws + p.off_split2);
    uint16_t *ql = qh + (p.bytes - p.off_split2) / 4;
    // Set on every call: the attribute belongs to the current device's copy of the kernel.
    cudaError_t e = cudaFuncSetAttribute(chol_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)((size_t)r * (r + 2) * sizeof(double)));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(solve_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)((size_t)r * r * sizeof(float)));
    if (e != cudaSuccess) return e;
    // Start: S = 0, so Z = W (hi = W, lo = 0); Q = orth(Q0).
    e = cudaMemcpyAsync(Zhi, W, (size_t)d_out * d_in * 2, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(Zlo, 0, (size_t)d_out * d_in * 2, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(Q, Q0, (size_t)d_in * r * sizeof(float), cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = orthonormalise(Q, Q2, M, part, d_in, r, p.split_gram, 2, st);
    for (int t = 0; t <= iters && e == cudaSuccess; ++t) {
        // P2: subspace iteration on Z, then U = Z Q.
        const int steps = t == 0 ? power0 : power;
        for (int s = 0; s < steps && e == cudaSuccess; ++s) {
            e = split_product(false, Zhi, Zlo, d_out, d_in, Q, bh, bl, r, P, st);                // P = Z Q
            if (e == cudaSuccess) e = split_product(true, Zhi, Zlo, d_out, d_in, P, bh, bl, r, Q, st);  // Q = Z^T P
            // Between power steps one Cholesky-QR pass keeps the basis well
            // conditioned; the last step's basis, which defines U V = Z Q Q^T,
            // gets the second pass (CholeskyQR2) so that it is orthonormal to
            // working precision.
            if (e == cudaSuccess) e = orthonormalise(Q, Q2, M, part, d_in, r, p.split_gram, s + 1 < steps ? 1 : 2, st);
        }
        if (e == cudaSuccess) e = split_product(false, Zhi, Zlo, d_out, d_in, Q, bh, bl, r, P, st);  // U = Z Q
        if (e != cudaSuccess) break;
        // P1: S = 2:4 threshold of W - U V, Z = W - S, objective: the product
        // P Q^T (both split into bf16 planes) on the tensor cores with the
        // threshold in its epilogue.
        split_bf16_kernel<<<grid_cap(d_out * r, 256), 256, 0, st>>>(P, d_out * r, bh, bl);
        split_bf16_kernel<<<grid_cap(d_in * r, 256), 256, 0, st>>>(Q, d_in * r, qh, ql);
        e = cudaGetLastError();
        if (e == cudaSuccess)
            e = gemm_tc<false, false, 128, kOutResid, true>(bh, bl, r, qh, ql, r, d_out, d_in, r, nullptr, am_err(), st,
                                                             ResidOut{W, vals, meta, Zhi, Zlo, objp});
        if (e == cudaSuccess && objective != nullptr)
            objective_finish_kernel<<<1, 256, 0, st>>>(objp, p.tiles_res, objective + t);
        if (e == cudaSuccess) e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        factors_out_kernel<<<grid_cap((d_out + d_in) * r, 256), 256, 0, st>>>(P, Q, d_out, d_in, r, U, V);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace slr

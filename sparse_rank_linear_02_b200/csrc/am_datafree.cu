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
//   repeat p times:  P = Z Q;  Q = orth(Z^T P)      (CholeskyQR2)
//   then U = Z Q, V = Q^T, so U V = Z Q Q^T, the best rank-r fit of Z within
//   span(Q), which converges to C_r(Z) as Q converges to the top-r right
//   singular subspace.  The random start Q0 is an input.
//
// Kernels (fp32 on CUDA cores; the products are tall and skinny, r <= 128):
//  * gemm_f32_kernel<TRANS_A>: C = A B (A d x k) or C = A^T B, 128 x 64 output
//    tiles, 16-deep k steps through shared memory, 8 x 4 outputs per thread,
//    split over k with the partial products summed in a fixed order by
//    reduce_splits_kernel (deterministic).
//  * chol_inv_kernel: one CTA; G = Q^T Q (from the split partials, in fp64)
//    -> Cholesky factor L -> M = L^-T, so Q M has orthonormal columns.
//  * residual_project_kernel: for a 64 x 128 tile, R = W - P Q^T (K = r
//    through shared memory), then per group of four the two largest |R| are
//    kept (ties to the lower index) and written packed (bf16 values, nibble
//    metadata), Z = W - S is written for the next subspace iteration, and the
//    tile's sum of (R - S)^2 goes to a per-tile partial of the objective.
#include <math.h>

#include <algorithm>

#include "common.cuh"

namespace slr {
namespace {

constexpr int kGT = 256;   // threads of the GEMM kernels
constexpr int kGBM = 128;  // output rows per tile
constexpr int kGBN = 64;   // output columns per tile
constexpr int kGBK = 16;   // k per shared-memory step

// C_part[split] (rows x cols, row-major, ldc = cols) = op(A) B over the k range
// of this split.  TRANS_A == false: A is rows x kdim (lda), C = A B.
// TRANS_A == true: A is kdim x rows (lda), C = A^T B.  B is kdim x cols (ldb).
template <bool TRANS_A>
__global__ void __launch_bounds__(kGT) gemm_f32_kernel(const float *__restrict__ A, int64_t lda,
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
        // A tile -> As[k][row]
        if (!TRANS_A) {
            // 128 rows x 16 k: each thread two 4-wide pieces of a row.
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int idx = tid + h * kGT;       // 0..511
                const int row = idx / 4, kq = (idx % 4) * 4;
                const int64_t gr = r0 + row, gk = k0 + kq;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (gr < rows) {
                    if (gk + 3 < k_end) {
                        v = *reinterpret_cast<const float4 *>(A + gr * lda + gk);
                    } else {
                        if (gk + 0 < k_end) v.x = A[gr * lda + gk + 0];
                        if (gk + 1 < k_end) v.y = A[gr * lda + gk + 1];
                        if (gk + 2 < k_end) v.z = A[gr * lda + gk + 2];
                    }
                }
                As[kq + 0][row] = v.x;
                As[kq + 1][row] = v.y;
                As[kq + 2][row] = v.z;
                As[kq + 3][row] = v.w;
            }
        } else {
            // 16 k (rows of A) x 128 output rows (columns of A): coalesced rows.
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
// rank-deficient block stays finite), then M = L^-T (fp32, r x r row-major).
// Shared memory: one r x r fp64 array; L fills the lower triangle and
// X = L^-1 (also lower triangular) is kept transposed in the strict upper
// triangle (X[i][c] at [c][i]); its diagonal is 1 / L[i][i].  Both phases are
// right-looking, so every step is a parallel update of the trailing block:
//   Cholesky, column j: pivot, scale column j below it, A[i][k] -= L[i][j] L[k][j]
//   for j < k <= i;  inverse, row i: finalise row i of X (divide by L[i][i]),
//   then X[i'][c] -= L[i'][i] X[i][c] for i' > i, c <= i.
__global__ void __launch_bounds__(256) chol_inv_kernel(const float *__restrict__ gpart, int splits, int r,
                                                       float *__restrict__ Mout) {
    extern __shared__ double A[];
    __shared__ double floor_pivot;
    const int tid = threadIdx.x, nth = blockDim.x;
    for (int i = tid; i < r * r; i += nth) {
        double s = 0.0;
        for (int k = 0; k < splits; ++k) s += (double)gpart[(int64_t)k * r * r + i];
        A[i] = s;
    }
    __syncthreads();
    if (tid == 0) {
        double tr = 0.0;
        for (int i = 0; i < r; ++i) tr += A[i * r + i];
        floor_pivot = 1e-12 * (tr > 0.0 ? tr / r : 1.0);
    }
    __syncthreads();
    for (int j = 0; j < r; ++j) {
        if (tid == 0) {
            const double d = A[j * r + j];
            A[j * r + j] = sqrt(d > floor_pivot ? d : floor_pivot);
        }
        __syncthreads();
        const double piv = A[j * r + j];
        for (int i = j + 1 + tid; i < r; i += nth) A[i * r + j] /= piv;
        __syncthreads();
        const int n = r - j - 1;
        for (int q = tid; q < n * n; q += nth) {
            const int ii = q / n, kk = q % n;
            if (kk <= ii) {
                const int i = j + 1 + ii, k = j + 1 + kk;
                A[i * r + k] -= A[i * r + j] * A[k * r + j];
            }
        }
        __syncthreads();
    }
    for (int q = tid; q < r * r; q += nth)
        if (q % r > q / r) A[q] = 0.0;  // strict upper triangle: X starts as the identity
    __syncthreads();
    for (int i = 0; i < r; ++i) {
        const double dinv = 1.0 / A[i * r + i];
        for (int c = tid; c < i; c += nth) A[c * r + i] *= dinv;
        __syncthreads();
        const int n = r - i - 1, m = i + 1;
        for (int q = tid; q < n * m; q += nth) {
            const int ii = i + 1 + q / m, c = q % m;
            const double xic = (c == i) ? dinv : A[c * r + i];
            A[c * r + ii] -= A[ii * r + i] * xic;
        }
        __syncthreads();
    }
    for (int i = tid; i < r * r; i += nth) {
        const int k = i / r, c = i % r;  // M[k][c] = X[c][k]
        float v = 0.f;
        if (c == k) v = (float)(1.0 / A[k * r + k]);
        else if (c > k) v = (float)A[k * r + c];
        Mout[i] = v;
    }
}

// The two positions of a group of four kept by |value| (ties to the lower
// index), from the fp32 magnitudes' bit patterns: the tournament of (0,1) and
// (2,3), the better winner first, then the better of the winning pair's loser
// and the losing pair's winner.  Returns idx0 | idx1 << 2.
__device__ __forceinline__ uint32_t keep_two(float v0, float v1, float v2, float v3) {
    const uint32_t k0 = __float_as_uint(fabsf(v0)), k1 = __float_as_uint(fabsf(v1));
    const uint32_t k2 = __float_as_uint(fabsf(v2)), k3 = __float_as_uint(fabsf(v3));
    const bool b01 = k0 >= k1, b23 = k2 >= k3;
    const uint32_t hi01 = max(k0, k1), lo01 = min(k0, k1), hi23 = max(k2, k3), lo23 = min(k2, k3);
    const uint32_t win01 = b01 ? 0u : 1u, los01 = b01 ? 1u : 0u;
    const uint32_t win23 = b23 ? 2u : 3u, los23 = b23 ? 3u : 2u;
    uint32_t first, second;
    if (hi01 >= hi23) {
        first = win01;
        second = lo01 >= hi23 ? los01 : win23;
    } else {
        first = win23;
        second = hi01 >= lo23 ? win01 : los23;
    }
    return min(first, second) | (max(first, second) << 2);
}

constexpr int kRBM = 64;   // residual tile rows
constexpr int kRBN = 128;  // residual tile columns
constexpr int kRBK = 16;

// R = W - P Q^T on a 64 x 128 tile (P: d_out x r, Q: d_in x r, fp32), then the
// 2:4 projection of R, the packed S, Z = W - S and the tile's sum of (R - S)^2.
// Thread layout: 16 x 16; a thread owns 4 rows x 8 consecutive columns (two
// groups of four per row).  d_in % 128 == 0 is not required (columns are
// guarded); d_in % 8 == 0 is.
__global__ void __launch_bounds__(256) residual_project_kernel(const uint16_t *__restrict__ W,
                                                               const float *__restrict__ P,
                                                               const float *__restrict__ Q, int64_t d_out,
                                                               int64_t d_in, int r, uint16_t *__restrict__ vals,
                                                               uint8_t *__restrict__ meta, float *__restrict__ Z,
                                                               float *__restrict__ obj_part) {
    __shared__ __align__(16) float Ps[kRBK][kRBM];
    __shared__ __align__(16) float Qs[kRBK][kRBN];
    __shared__ float red[8];
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    const int64_t r0 = (int64_t)blockIdx.y * kRBM, c0 = (int64_t)blockIdx.x * kRBN;
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    for (int k0 = 0; k0 < r; k0 += kRBK) {
        // Ps[k][row]: 64 rows x 16 k = 1024 floats, one 16-byte load per
        // thread.  r % 8 == 0, so a 4-wide piece starting below r lies wholly
        // inside the row (and is 16-byte aligned); pieces at or past r are zero.
        {
            const int row = tid / 4, kq = (tid % 4) * 4;
            const int64_t gr = r0 + row;
            const float4 v = (gr < d_out && k0 + kq < r) ? *reinterpret_cast<const float4 *>(P + gr * r + k0 + kq)
                                                         : make_float4(0.f, 0.f, 0.f, 0.f);
            Ps[kq + 0][row] = v.x;
            Ps[kq + 1][row] = v.y;
            Ps[kq + 2][row] = v.z;
            Ps[kq + 3][row] = v.w;
        }
        // Qs[k][col]: 128 cols x 16 k = 2048 floats, two 16-byte loads per thread.
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int idx = tid + h * 256;
            const int col = idx / 4, kq = (idx % 4) * 4;
            const int64_t gc = c0 + col;
            const float4 v = (gc < d_in && k0 + kq < r) ? *reinterpret_cast<const float4 *>(Q + gc * r + k0 + kq)
                                                        : make_float4(0.f, 0.f, 0.f, 0.f);
            Qs[kq + 0][col] = v.x;
            Qs[kq + 1][col] = v.y;
            Qs[kq + 2][col] = v.z;
            Qs[kq + 3][col] = v.w;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kRBK; ++kk) {
            const float4 p = *reinterpret_cast<const float4 *>(&Ps[kk][ty * 4]);
            const float4 q0 = *reinterpret_cast<const float4 *>(&Qs[kk][tx * 8]);
            const float4 q1 = *reinterpret_cast<const float4 *>(&Qs[kk][tx * 8 + 4]);
            const float pa[4] = {p.x, p.y, p.z, p.w};
            const float qa[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(pa[i], qa[j], acc[i][j]);
        }
        __syncthreads();
    }
    float obj = 0.f;
    const int64_t gc = c0 + tx * 8;
    const int64_t meta_row = (d_in / 4 + 1) / 2;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t gr = r0 + ty * 4 + i;
        if (gr >= d_out || gc >= d_in) continue;
        const uint4 w = *reinterpret_cast<const uint4 *>(W + gr * d_in + gc);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        float R[8], S[8];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            R[2 * h] = bf16lo_to_f32(ww[h]) - acc[i][2 * h];
            R[2 * h + 1] = bf16hi_to_f32(ww[h]) - acc[i][2 * h + 1];
        }
        uint32_t byte = 0, kept[2];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            const uint32_t nib = keep_two(R[4 * g], R[4 * g + 1], R[4 * g + 2], R[4 * g + 3]);
            const uint32_t a = nib & 3u, b = nib >> 2;  // a in 0..2, b in 1..3
            uint32_t sv[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                sv[p] = f32_to_bf16_bits(R[4 * g + p]);
                S[4 * g + p] = (p == (int)a || p == (int)b) ? __uint_as_float(sv[p] << 16) : 0.f;
            }
            const uint32_t sa = a == 0u ? sv[0] : (a == 1u ? sv[1] : sv[2]);
            const uint32_t sb = b == 1u ? sv[1] : (b == 2u ? sv[2] : sv[3]);
            kept[g] = sa | (sb << 16);
            byte |= nib << (4 * g);
        }
        *reinterpret_cast<uint2 *>(vals + gr * (d_in / 2) + gc / 2) = make_uint2(kept[0], kept[1]);
        meta[gr * meta_row + gc / 8] = (uint8_t)byte;
        float zr[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const float wv = (p & 1) ? bf16hi_to_f32(ww[p / 2]) : bf16lo_to_f32(ww[p / 2]);
            zr[p] = wv - S[p];
            const float e = R[p] - S[p];
            obj = fmaf(e, e, obj);
        }
        float4 *zp = reinterpret_cast<float4 *>(Z + gr * d_in + gc);
        zp[0] = make_float4(zr[0], zr[1], zr[2], zr[3]);
        zp[1] = make_float4(zr[4], zr[5], zr[6], zr[7]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) obj += __shfl_xor_sync(0xFFFFFFFFu, obj, o);
    if ((tid & 31) == 0) red[tid >> 5] = obj;
    __syncthreads();
    if (tid == 0) {
        float s = 0.f;
        for (int k = 0; k < 8; ++k) s += red[k];
        obj_part[(int64_t)blockIdx.y * gridDim.x + blockIdx.x] = s;
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

__global__ void bf16_to_f32_kernel(const uint16_t *__restrict__ in, int64_t n, float *__restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = __uint_as_float((uint32_t)in[i] << 16);
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

int grid_cap(int64_t n, int threads) {
    const int64_t b = (n + threads - 1) / threads;
    return (int)(b < 148 * 16 ? (b > 0 ? b : 1) : 148 * 16);
}

}  // namespace

// ----------------------------------------------------------------------------- host driver

AmPlan am_plan(int64_t d_out, int64_t d_in, int64_t r) {
    AmPlan p{};
    auto splits_for = [](int64_t tiles, int64_t kdim) {
        // about two CTAs per SM, each split at least 256 deep
        int64_t s = (2 * 148 + tiles - 1) / tiles;
        const int64_t kmax = (kdim + 255) / 256;
        if (s > kmax) s = kmax;
        if (s > 32) s = 32;
        return s < 1 ? int64_t(1) : s;
    };
    const int64_t ctiles = (r + kGBN - 1) / kGBN;
    p.split_nn = splits_for(((d_out + kGBM - 1) / kGBM) * ctiles, d_in);    // P = Z Q
    p.split_tn = splits_for(((d_in + kGBM - 1) / kGBM) * ctiles, d_out);    // Z^T P
    p.split_gram = splits_for(ctiles, d_in);                                  // Q^T Q
    p.split_mul = 1;                                                          // Q M (k = r)
    const int64_t part = std::max({p.split_nn * d_out * r, p.split_tn * d_in * r, p.split_gram * r * r,
                                   d_in * r});
    p.tiles_res = ((d_in + kRBN - 1) / kRBN) * ((d_out + kRBM - 1) / kRBM);
    auto al = [](int64_t b) { return (b + 255) / 256 * 256; };
    p.off_Z = 0;
    p.off_Q = p.off_Z + al(d_out * d_in * 4);
    p.off_Q2 = p.off_Q + al(d_in * r * 4);
    p.off_P = p.off_Q2 + al(d_in * r * 4);
    p.off_M = p.off_P + al(d_out * r * 4);
    p.off_part = p.off_M + al(r * r * 4);
    p.off_obj = p.off_part + al(part * 4);
    p.bytes = p.off_obj + al(p.tiles_res * 4);
    return p;
}

namespace {

cudaError_t gemm(bool trans_a, const float *A, int64_t lda, const float *B, int64_t ldb, float *out, float *part,
                 int64_t rows, int64_t cols, int64_t kdim, int64_t splits, cudaStream_t st) {
    int64_t kps = (kdim + splits - 1) / splits;
    kps = (kps + kGBK - 1) / kGBK * kGBK;
    const int64_t used = (kdim + kps - 1) / kps;
    dim3 grid((unsigned)((rows + kGBM - 1) / kGBM), (unsigned)((cols + kGBN - 1) / kGBN), (unsigned)used);
    float *dst = used == 1 ? out : part;
    if (trans_a)
        gemm_f32_kernel<true><<<grid, kGT, 0, st>>>(A, lda, B, ldb, dst, rows, cols, kdim, kps);
    else
        gemm_f32_kernel<false><<<grid, kGT, 0, st>>>(A, lda, B, ldb, dst, rows, cols, kdim, kps);
    if (used > 1) reduce_splits_kernel<<<grid_cap(rows * cols, 256), 256, 0, st>>>(part, (int)used, rows * cols, out);
    return cudaGetLastError();
}

// Q (d_in x r) <- Q L^-T with L the Cholesky factor of Q^T Q; tmp is d_in x r.
cudaError_t orthonormalise(float *Q, float *tmp, float *M, float *part, int64_t d_in, int r, int64_t split_gram,
                           cudaStream_t st) {
    for (int pass = 0; pass < 2; ++pass) {  // CholeskyQR2
        int64_t kps = (d_in + split_gram - 1) / split_gram;
        kps = (kps + kGBK - 1) / kGBK * kGBK;
        const int64_t used = (d_in + kps - 1) / kps;
        dim3 grid(1, (unsigned)((r + kGBN - 1) / kGBN), (unsigned)used);
        gemm_f32_kernel<true><<<grid, kGT, 0, st>>>(Q, r, Q, r, part, r, r, d_in, kps);
        chol_inv_kernel<<<1, 256, (size_t)r * r * sizeof(double), st>>>(part, (int)used, r, M);
        cudaError_t e = gemm(false, Q, r, M, r, tmp, part, d_in, r, r, 1, st);
        if (e != cudaSuccess) return e;
        e = cudaMemcpyAsync(Q, tmp, (size_t)d_in * r * sizeof(float), cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_am_datafree(const uint16_t *W, int64_t d_out, int64_t d_in, int r, int iters, int power0,
                               int power, const float *Q0, uint16_t *vals, uint8_t *meta, uint16_t *U, uint16_t *V,
                               double *objective, uint8_t *ws, cudaStream_t st) {
    const AmPlan p = am_plan(d_out, d_in, r);
    float *Z = reinterpret_cast<float *>(ws + p.off_Z);
    float *Q = reinterpret_cast<float *>(ws + p.off_Q);
    float *Q2 = reinterpret_cast<float *>(ws + p.off_Q2);
    float *P = reinterpret_cast<float *>(ws + p.off_P);
    float *M = reinterpret_cast<float *>(ws + p.off_M);
    float *part = reinterpret_cast<float *>(ws + p.off_part);
    float *objp = reinterpret_cast<float *>(ws + p.off_obj);
    static bool smem_set = false;
    if (!smem_set) {
        cudaFuncSetAttribute(chol_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 128 * 128 * 8);
        smem_set = true;
    }
    cudaError_t e = cudaSuccess;
    // Start: S = 0, so Z = W; Q = orth(Q0).
    bf16_to_f32_kernel<<<grid_cap(d_out * d_in, 256), 256, 0, st>>>(W, d_out * d_in, Z);
    e = cudaMemcpyAsync(Q, Q0, (size_t)d_in * r * sizeof(float), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
    e = orthonormalise(Q, Q2, M, part, d_in, r, p.split_gram, st);
    const dim3 rgrid((unsigned)((d_in + kRBN - 1) / kRBN), (unsigned)((d_out + kRBM - 1) / kRBM));
    for (int t = 0; t <= iters && e == cudaSuccess; ++t) {
        // P2: subspace iteration on Z, then U = Z Q.
        const int steps = t == 0 ? power0 : power;
        for (int s = 0; s < steps && e == cudaSuccess; ++s) {
            e = gemm(false, Z, d_in, Q, r, P, part, d_out, r, d_in, p.split_nn, st);            // P = Z Q
            if (e == cudaSuccess) e = gemm(true, Z, d_in, P, r, Q, part, d_in, r, d_out, p.split_tn, st);  // Q = Z^T P
            if (e == cudaSuccess) e = orthonormalise(Q, Q2, M, part, d_in, r, p.split_gram, st);
        }
        if (e == cudaSuccess) e = gemm(false, Z, d_in, Q, r, P, part, d_out, r, d_in, p.split_nn, st);  // U = Z Q
        if (e != cudaSuccess) break;
        // P1: S = 2:4 threshold of W - U V, Z = W - S, objective.
        residual_project_kernel<<<rgrid, 256, 0, st>>>(W, P, Q, d_out, d_in, r, vals, meta, Z, objp);
        if (objective != nullptr) objective_finish_kernel<<<1, 256, 0, st>>>(objp, p.tiles_res, objective + t);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        factors_out_kernel<<<grid_cap((d_out + d_in) * r, 256), 256, 0, st>>>(P, Q, d_out, d_in, r, U, V);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace slr

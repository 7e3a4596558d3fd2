// column_norms.cu -- column sums of squares of calibration activations and
// their square roots, the per-column scale of the activation-aware 2:4
// projection.
//
// HASSLE-free, section 4.1.2: the diagonal Hessian approximation keeps only
// diag(X^T X); the square root of entry j, the 2-norm of input column j, is the
// factor by which column j of W is scaled before hard-thresholding (Wanda's
// score).  Section 5.1 builds the Hessian from many token segments, so the sum
// runs over batches: every call adds one batch's squares to a running fp64 sum.
//
// Two kernels, HBM-bound on reading X once (2 bytes per element):
//  (1) partial sums.  Grid = (strips of 256 columns) x (row splits), sized
//      to one wave of 6 resident CTAs on each of 148 SMs.  Lane l of a warp
//      owns 8 columns (one 16-byte load per row, so a warp reads 512
//      contiguous bytes of a row); the 8 warps of a CTA take interleaved rows
//      of the split, kNormRows rows in flight per thread; each thread
//      accumulates its 8 columns in fp32; the 8 warp sums of a column are then
//      added in warp order through shared memory and written to row `split`
//      of the workspace.
//  (2) finish, launched as a programmatic dependent of (1) so that its launch
//      overlaps (1)'s tail.  Four threads per column each add every fourth
//      split in fp64, the four sums are added in a fixed order, the total is
//      added to the running sum and, when asked, the norm is written: the
//      fp64 square root rounded to fp32.
// The split count depends on (M, d_in) only, so the result is deterministic
// and the same on every device.
#include "common.cuh"

namespace slr {
namespace {

constexpr int kNormThreads = 256;     // 8 warps
constexpr int kNormStripCols = 256;   // 32 lanes x 8 columns
constexpr int kNormRows = 4;          // rows in flight per thread
constexpr int kNormCtasPerSm = 6;
constexpr int64_t kNormTargetCtas = 148 * kNormCtasPerSm;  // one wave on B200
constexpr int64_t kNormMinRows = 32;  // one step of 8 warps x kNormRows
constexpr int64_t kNormMaxRows = 512; // caps a thread's serial fp32 sum at 64 terms

__global__ void __launch_bounds__(kNormThreads, kNormCtasPerSm) column_sumsq_partial_kernel(const uint16_t *__restrict__ X,
                                                                            int64_t M, int64_t d_in, int64_t ldx,
                                                                            int64_t rows_per_split,
                                                                            float *__restrict__ partial) {
    // red[w][l * 9 + k]: warp w's sum for column 8 l + k (9 = 8 + 1 pad, so
    // the stores of a warp hit 32 distinct banks).
    __shared__ float red[kNormThreads / 32][32 * 9];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t unit = (int64_t)blockIdx.x * 32 + lane;
    const int64_t r_begin = (int64_t)blockIdx.y * rows_per_split;
    const int64_t r_end = min(M, r_begin + rows_per_split);
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.0f;
    if (unit < d_in / 8) {
        const uint16_t *col = X + 8 * unit;
        for (int64_t r = r_begin + warp; r < r_end; r += 8 * kNormRows) {
            uint4 v[kNormRows];
#pragma unroll
            for (int i = 0; i < kNormRows; ++i) {
                const int64_t rr = r + 8 * i;
                v[i] = rr < r_end ? ld_stream_v4(col + rr * ldx) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < kNormRows; ++i) {
                const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float lo = bf16lo_to_f32(w[h]), hi = bf16hi_to_f32(w[h]);
                    acc[2 * h] = fmaf(lo, lo, acc[2 * h]);
                    acc[2 * h + 1] = fmaf(hi, hi, acc[2 * h + 1]);
                }
            }
        }
    }
    // The finish kernel may be scheduled now; it waits for this grid's
    // completion (and memory flush) before reading the partial sums.
    asm volatile("griddepcontrol.launch_dependents;");
#pragma unroll
    for (int k = 0; k < 8; ++k) red[warp][lane * 9 + k] = acc[k];
    __syncthreads();
    const int t = threadIdx.x;
    const int64_t c = (int64_t)blockIdx.x * kNormStripCols + t;
    if (c < d_in) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kNormThreads / 32; ++w) s += red[w][(t >> 3) * 9 + (t & 7)];
        partial[(int64_t)blockIdx.y * d_in + c] = s;
    }
}

// Block = 64 columns x 4 split classes; thread (q, c) adds splits q, q+4, ...
__global__ void __launch_bounds__(256) column_norms_finish_kernel(const float *__restrict__ partial, int64_t splits,
                                                                  int64_t d_in, double *__restrict__ sumsq,
                                                                  float *__restrict__ norms) {
    __shared__ double red[4][64];
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int q = threadIdx.x >> 6, cl = threadIdx.x & 63;
    const int64_t j = (int64_t)blockIdx.x * 64 + cl;
    double s = 0.0;
    if (j < d_in) {
#pragma unroll 8
        for (int64_t k = q; k < splits; k += 4) s += (double)partial[k * d_in + j];
    }
    red[q][cl] = s;
    __syncthreads();
    if (q == 0 && j < d_in) {
        const double total = sumsq[j] + (((red[0][cl] + red[1][cl]) + red[2][cl]) + red[3][cl]);
        sumsq[j] = total;
        if (norms != nullptr) norms[j] = __double2float_rn(sqrt(total));
    }
}

}  // namespace

NormPlan column_norms_plan(int64_t M, int64_t d_in) {
    NormPlan p{0, 0};
    if (M <= 0 || d_in <= 0) return p;
    const int64_t strips = (d_in + kNormStripCols - 1) / kNormStripCols;
    int64_t rows = (M * strips + kNormTargetCtas - 1) / kNormTargetCtas;
    rows = (rows + kNormMinRows - 1) / kNormMinRows * kNormMinRows;
    rows = rows < kNormMinRows ? kNormMinRows : (rows > kNormMaxRows ? kNormMaxRows : rows);
    const int64_t min_rows = (M + 65534) / 65535;  // the split count is a grid dimension
    if (rows < min_rows) rows = (min_rows + kNormMinRows - 1) / kNormMinRows * kNormMinRows;
    p.rows_per_split = rows;
    p.splits = (M + rows - 1) / rows;
    return p;
}

cudaError_t launch_column_norms(const uint16_t *X, int64_t M, int64_t d_in, int64_t ldx, double *sumsq,
                                float *norms, float *partial, cudaStream_t stream) {
    const NormPlan p = column_norms_plan(M, d_in);
    if (p.splits > 0) {
        const int64_t strips = (d_in + kNormStripCols - 1) / kNormStripCols;
        column_sumsq_partial_kernel<<<dim3((unsigned)strips, (unsigned)p.splits), kNormThreads, 0, stream>>>(
            X, M, d_in, ldx, p.rows_per_split, partial);
    }
    if (p.splits == 0) {
        column_norms_finish_kernel<<<(unsigned)((d_in + 63) / 64), 256, 0, stream>>>(partial, 0, d_in, sumsq, norms);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((d_in + 63) / 64));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, column_norms_finish_kernel, (const float *)partial, p.splits, d_in, sumsq, norms);
}

}  // namespace slr

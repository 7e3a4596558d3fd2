// common.cuh -- internal helpers shared by the kernels of libslr (not exported).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "slr.h"

namespace slr {

// bf16 bit pattern (low 16 bits of x) -> fp32, exact.
__device__ __forceinline__ float bf16lo_to_f32(uint32_t x) { return __uint_as_float(x << 16); }
// bf16 bit pattern (high 16 bits of x) -> fp32, exact.
__device__ __forceinline__ float bf16hi_to_f32(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

// fp32 -> bf16 bits, round to nearest even (the CUDA intrinsic).
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    __nv_bfloat16_raw r = __nv_bfloat16_raw(__float2bfloat16_rn(f));
    return r.x;
}

// Streaming 16-byte load that does not allocate in L1 (weights are read once).
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Loads of data that another grid writes while this one may already run (T
// from the projection kernel, X in a chained launch): ordinary coherent loads
// that bypass L1 (.cg), issued from volatile asm so that the compiler keeps
// them after the griddepcontrol.wait that precedes them.  Read-only loads
// (__ldg, ld.global.nc) must not be used for such data: the compiler treats
// them as invariant and may move them above the wait.
__device__ __forceinline__ float ld_dep_f32(const float *p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ float2 ld_dep_f2(const float *p) {
    float2 v;
    asm volatile("ld.global.cg.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint4 ld_dep_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

// ---------------------------------------------------------------- launchers
// Each returns cudaSuccess or the launch error; arguments were validated by
// the API layer.

cudaError_t launch_pack_2to4(const uint16_t *W, int64_t d_out, int64_t d_in, int64_t ldw,
                             uint16_t *vals, uint8_t *meta, cudaStream_t stream);

// Activation-aware 2:4 projection: as launch_pack_2to4 with the weights of
// column j ranked by |w| * |scale[j]| (fp32).
cudaError_t launch_pack_2to4_scaled(const uint16_t *W, int64_t d_out, int64_t d_in, int64_t ldw,
                                    const float *scale, uint16_t *vals, uint8_t *meta, cudaStream_t stream);

// 2:8 projection; any of the two output pairs may be null (both members of a
// pair together).  vals8 4-byte aligned, vals4 8-byte aligned; d_in % 8 == 0.
cudaError_t launch_pack_2to8(const uint16_t *W, int64_t d_out, int64_t d_in, int64_t ldw, uint16_t *vals8,
                             uint8_t *meta8, uint16_t *vals4, uint8_t *meta4, cudaStream_t stream);

// Small-M streaming forward of a 2:8-packed layer: Y = X S^T + T U^T, T fp32
// [M, r] precomputed (after_projection as for launch_decode_forward).
// d_in % 32 == 0, all pointers 16-byte aligned.
cudaError_t launch_decode28_forward(const uint16_t *X, int64_t M, const uint16_t *vals8, const uint8_t *meta8,
                                    int64_t d_out, int64_t d_in, const uint16_t *U, const float *T32, int64_t r,
                                    uint16_t *Y, bool after_projection, cudaStream_t stream);

// Reads and clears the error word of the decomposition's tensor-core products.
cudaError_t read_and_clear_am_error(unsigned *code);

// Reads and clears the error word of the 2:8 ring kernel's bounded waits.
cudaError_t read_and_clear_decode28_error(unsigned *code);

// Data-free alternating minimisation: workspace layout (byte offsets) and the
// split counts of its products.
struct AmPlan {
    int64_t split_gram;
    int64_t tiles_res;
    int64_t off_Z, off_Q, off_Q2, off_P, off_M, off_part, off_obj, off_split, off_split2, bytes;
};
AmPlan am_plan(int64_t d_out, int64_t d_in, int64_t r);

// W (bf16 d_out x d_in) -> packed 2:4 S (vals, meta), U (bf16 d_out x r),
// V (bf16 r x d_in); objective (device, iters + 1 doubles) may be null.
// Q0: fp32 d_in x r start of the subspace iteration.  ws: am_plan().bytes.
cudaError_t launch_am_datafree(const uint16_t *W, int64_t d_out, int64_t d_in, int r, int iters, int power0,
                               int power, const float *Q0, uint16_t *vals, uint8_t *meta, uint16_t *U, uint16_t *V,
                               double *objective, uint8_t *ws, cudaStream_t st);

// The fp32 factors that the last launch_am_datafree on `ws` (same shape) left
// in its workspace: U32 = P [d_out, r], V32 = Q^T [r, d_in]; either may be null.
cudaError_t launch_am_factors_f32(const uint8_t *ws, int64_t d_out, int64_t d_in, int r, float *U32, float *V32,
                                  cudaStream_t st);

// Gradients of the layer with respect to U and V (S frozen): G = dY U (bf16,
// in ws), dU = dY^T T (fp32 [d_out, r]), dV = G^T X (fp32 [r, d_in]).  T16_in
// is the forward's T = X V^T (bf16 [M, r]) or null (then computed into ws).
// ws: 2 * M * r bf16.  d_in % 64 == 0, d_out % 8 == 0, 8 <= r <= 256, r % 8 == 0.
cudaError_t launch_lora_backward(const uint16_t *X, int64_t M, const uint16_t *dY, int64_t d_out, int64_t d_in,
                                 const uint16_t *U, const uint16_t *V, int64_t r, const uint16_t *T16_in, float *dU,
                                 float *dV, uint16_t *ws, cudaStream_t st);
cudaError_t read_and_clear_backward_error(unsigned *code);

// Row split of the column-norm reduction: `splits` row ranges of
// `rows_per_split` rows, each leaving d_in fp32 partial sums in the workspace.
struct NormPlan {
    int64_t rows_per_split;
    int64_t splits;
};
NormPlan column_norms_plan(int64_t M, int64_t d_in);

// sumsq[j] += sum_m X[m][j]^2; norms[j] = sqrt(sumsq[j]) rounded to fp32 when
// norms is not null.  partial: splits * d_in floats of scratch (d_in >= 1,
// d_in % 8 == 0, ldx % 8 == 0, X 16-byte aligned).
cudaError_t launch_column_norms(const uint16_t *X, int64_t M, int64_t d_in, int64_t ldx, double *sumsq,
                                float *norms, float *partial, cudaStream_t stream);

// T = X * V^T for M tokens, written as fp32 [M, r] (T32, may be null) and/or
// bf16 [M, r] (T16, may be null).  chained: launched as a programmatic
// dependent of whatever precedes it on `stream`; V is prefetched into L2 at
// once, X read and T written only after the wait for the preceding grid.
cudaError_t launch_lowrank_project(const uint16_t *X, int64_t M, const uint16_t *V, int64_t d_in,
                                   int64_t r, float *T32, uint16_t *T16, bool chained, cudaStream_t stream);

// Small-M streaming forward: Y = X S^T + T U^T with T (fp32 [M, r]) precomputed.
// pdl_mode: 0 = ordinary launch; 1 = the projection kernel that writes T32 is
// the kernel launched immediately before on `stream` (programmatic dependent
// launch, waits before reading T32).  Chained launches (2) are not supported
// by this kernel (decode_chain_ok).
// Whether the streaming forward supports chained launches for this M and d_in.
bool decode_chain_ok(int64_t M, int64_t d_in);

cudaError_t launch_decode_forward(const uint16_t *X, int64_t M, const uint16_t *vals,
                                  const uint8_t *meta, int64_t d_out, int64_t d_in,
                                  const uint16_t *U, const float *T32, int64_t r, uint16_t *Y,
                                  int pdl_mode, cudaStream_t stream);

}  // namespace slr

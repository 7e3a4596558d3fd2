// lowrank_project.cu -- the rank-r projection T = X * V^T on CUDA cores.
//
// LoSparse, section 3.2: the low-rank term of the compressed layer is applied
// as (X U) V in the pages' row-vector notation; with W = S + U V stored as
// d_out x d_in here, that product is (X V^T) U^T and this kernel forms the
// first factor T = X V^T (M x r) in fp32.
//
// One CTA per (rank index k, block of 8 tokens).  The 256 threads stride over
// d_in in 16-byte chunks, so V's row k and the 8 rows of X are read with
// coalesced 128-bit loads; partial sums are reduced with warp shuffles and a
// small shared-memory pass.  This is the small-M producer of T; its cost is
// r * d_in * 2 bytes of V plus M * d_in * 2 bytes of X, a few percent of the
// weight bytes the forward streams.
#include "common.cuh"

namespace slr {
namespace {

constexpr int kTokens = 8;
constexpr int kThreads = 256;

__device__ __forceinline__ float dot8(uint4 a, uint4 b, float acc) {
    acc = fmaf(bf16lo_to_f32(a.x), bf16lo_to_f32(b.x), acc);
    acc = fmaf(bf16hi_to_f32(a.x), bf16hi_to_f32(b.x), acc);
    acc = fmaf(bf16lo_to_f32(a.y), bf16lo_to_f32(b.y), acc);
    acc = fmaf(bf16hi_to_f32(a.y), bf16hi_to_f32(b.y), acc);
    acc = fmaf(bf16lo_to_f32(a.z), bf16lo_to_f32(b.z), acc);
    acc = fmaf(bf16hi_to_f32(a.z), bf16hi_to_f32(b.z), acc);
    acc = fmaf(bf16lo_to_f32(a.w), bf16lo_to_f32(b.w), acc);
    acc = fmaf(bf16hi_to_f32(a.w), bf16hi_to_f32(b.w), acc);
    return acc;
}

__global__ void __launch_bounds__(kThreads) lowrank_project_kernel(const uint16_t *__restrict__ X, int64_t M,
                                                                   const uint16_t *__restrict__ V,
                                                                   int64_t d_in, int64_t r,
                                                                   float *__restrict__ T32,
                                                                   uint16_t *__restrict__ T16, int chained) {
    // Let the dependent streaming kernel launch now; it only reads T after
    // its own griddepcontrol.wait, which waits for this grid to complete.
    asm volatile("griddepcontrol.launch_dependents;");
    const int64_t k = blockIdx.x;
    if (chained) {
        // Launched while the preceding grid may still run: V (a weight) is
        // pulled into L2 now; X is read, and T written, only after the wait.
        if (threadIdx.x == 0 && blockIdx.y == 0) {
            const uint8_t *row = reinterpret_cast<const uint8_t *>(V + k * d_in);
            for (int64_t off = 0; off < d_in * 2; off += 32768) {
                const int64_t n = d_in * 2 - off < 32768 ? d_in * 2 - off : 32768;
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(row + off), "r"((uint32_t)n) : "memory");
            }
        }
        asm volatile("griddepcontrol.wait;" ::: "memory");
    }
    const int64_t m0 = (int64_t)blockIdx.y * kTokens;
    const int nt = (int)((M - m0) < kTokens ? (M - m0) : kTokens);
    float acc[kTokens];
#pragma unroll
    for (int t = 0; t < kTokens; ++t) acc[t] = 0.f;

    const int64_t chunks = d_in / 8;
    const uint4 *vrow = reinterpret_cast<const uint4 *>(V + k * d_in);
    for (int64_t c = threadIdx.x; c < chunks; c += kThreads) {
        const uint4 v = __ldg(vrow + c);
#pragma unroll
        for (int t = 0; t < kTokens; ++t) {
            if (t < nt) {
                const uint4 x = ld_dep_v4(reinterpret_cast<const uint4 *>(X + (m0 + t) * d_in) + c);
                acc[t] = dot8(v, x, acc[t]);
            }
        }
    }

    __shared__ float red[kThreads / 32][kTokens];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int t = 0; t < kTokens; ++t) {
        float s = acc[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
        if (lane == 0) red[warp][t] = s;
    }
    __syncthreads();
    if (threadIdx.x < nt) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) s += red[w][threadIdx.x];
        const int64_t m = m0 + threadIdx.x;
        if (T32) T32[m * r + k] = s;
        if (T16) T16[m * r + k] = f32_to_bf16_bits(s);
    }
}

}  // namespace

cudaError_t launch_lowrank_project(const uint16_t *X, int64_t M, const uint16_t *V, int64_t d_in,
                                   int64_t r, float *T32, uint16_t *T16, bool chained, cudaStream_t stream) {
    if (M == 0 || r == 0) return cudaSuccess;
    const int64_t tblocks = (M + kTokens - 1) / kTokens;
    if (tblocks > 65535) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)r, (unsigned)tblocks);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = chained ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, lowrank_project_kernel, X, M, V, d_in, r, T32, T16, (int)(chained ? 1 : 0));
}

}  // namespace slr

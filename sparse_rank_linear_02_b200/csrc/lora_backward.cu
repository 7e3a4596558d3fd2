// lora_backward.cu -- gradients of the layer with respect to its low-rank
// factors (S frozen), on the tensor cores.
//
// Y = X S^T + T U^T with T = X V^T (LoSparse, section 3.2); the low-rank
// factors are what LoRA fine-tuning trains (3BASiL summary page: the low-rank
// components initialise LoRA).  For dY = dL/dY:
//     G  = dY U          (M x r,     bf16)
//     dU = dY^T T        (d_out x r, fp32)
//     dV = G^T X         (r x d_in,  fp32)
// All three are dense products with one small side (r); the weight gradients
// contract over the tokens, which are the outer (row) dimension of dY and X,
// so their operands are read "MN-major" (contiguous along the output
// dimension) straight from the row-major activations: no transposes.
//
// One kernel, tc_gemm_kernel<A_MN, B_MN, RN, OUT>: C (Mc x N, N <= RN) =
// sum_k A(k, m) B(k, n) over K in 64-deep stages.  A is a 128 x 64 tile
// (K-major: 128 rows of 64 K; MN-major: two 64-wide MN panels of 64 K rows),
// B an RN x 64 tile (K-major) or RN/64 panels (MN-major), all loaded by TMA
// with the 128-byte swizzle; tcgen05.mma kind::f16 (bf16 in, fp32 in TMEM)
// with the operand major-ness in the instruction descriptor.  A cluster of KS
// CTAs splits the K stages of one 128-row tile; their fp32 partials meet in
// shared memory and are summed over distributed shared memory (as in the
// rank projection of the forward), then written once: fp32 row-major,
// fp32 transposed (dV), or bf16 row-major (G).  Every wait is bounded.
// dU runs on a second stream beside G and dV (forked and joined with events
// on the caller's stream).
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "tc_forward.cuh"
#include "tc_ptx.cuh"

namespace slr {

// Error word of this file's bounded waits (read by slr_check_kernel_error).
__device__ unsigned int g_bwd_error = 0;

namespace {

using namespace tc;

constexpr int kBM = 128;       // output rows per tile (MMA M)
constexpr int kBThreads = 192;  // producer, MMA, four epilogue warps

enum OutMode { kOutF32 = 0, kOutF32T = 1, kOutBF16 = 2 };

template <int RN>
struct CfgB {
    static constexpr int A_BYTES = kBM * 64 * 2;   // 16 KB
    static constexpr int B_BYTES = RN * 64 * 2;
    static constexpr int STAGE = ((A_BYTES + B_BYTES + 1023) / 1024) * 1024;
    static constexpr int PROW = RN + 4;
    static constexpr int P_BYTES = kBM * PROW * 4;
    static constexpr int NS_FIT = 112640 / STAGE;
    static constexpr int NS = NS_FIT > 8 ? 8 : (NS_FIT < 2 ? 2 : NS_FIT);
    static constexpr int RING = NS * STAGE;
    static constexpr int BAR_OFF = RING > P_BYTES ? RING : P_BYTES;
    static constexpr int SMEM = BAR_OFF + 256 + 1024;
    static constexpr uint32_t TMEM_COLS = RN <= 32 ? 32 : (RN <= 64 ? 64 : (RN <= 128 ? 128 : 256));
    static_assert(RN % 64 == 0 && RN <= 256, "N tile");
    static_assert(SMEM <= 232448, "shared memory budget");
};

// MN-major, 128-byte swizzled operand: rows of 64 elements (128 B) along MN,
// one row per k; 8-row k groups 1024 B apart (SBO), 64-element MN panels
// 8192 B apart (LBO, a panel holds the stage's 64 k rows).
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t addr) { return smem_desc(addr, 8192, 1024, kLayoutSW128); }

template <bool A_MN, bool B_MN, int RN, int OUT>
__global__ void __launch_bounds__(kBThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   void *__restrict__ out, int32_t Mc, int32_t N, int32_t nk_total) {
    using C = CfgB<RN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *empty = full + C::NS;
    uint64_t *acc_full = empty + C::NS;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    volatile uint32_t *fail = tmem_slot + 1;
    float *part = reinterpret_cast<float *>(smem);  // reuses the ring after the K loop

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t ks_n;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(ks_n));
    const uint32_t ks_q = cluster_ctarank();
    const int tile = blockIdx.x / (int)ks_n;
    const int m0 = tile * kBM;
    const int k_begin = (int)(((int64_t)nk_total * ks_q) / ks_n);
    const int k_end = (int)(((int64_t)nk_total * (ks_q + 1)) / ks_n);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        *fail = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (elect_one()) {
            uint32_t s = 0, ph = 0;
            for (int ks = k_begin; ks < k_end; ++ks) {
                if (!mbar_wait(&empty[s], ph ^ 1)) {
                    *fail = 1;
                    atomicOr(&g_bwd_error, 1u);
                    break;
                }
                const uint32_t a = smem_u32(smem + s * C::STAGE), b = a + C::A_BYTES;
                mbar_expect_tx(&full[s], C::A_BYTES + C::B_BYTES);
                if (A_MN) {  // map (inner = MN, outer = K), box 64 x 64
                    tma_load_2d(&tm_a, a, &full[s], m0, ks * 64);
                    tma_load_2d(&tm_a, a + 8192, &full[s], m0 + 64, ks * 64);
                } else {     // map (inner = K, outer = MN), box 64 x 128
                    tma_load_2d(&tm_a, a, &full[s], ks * 64, m0);
                }
                if (B_MN) {  // map (inner = N, outer = K), box 64 x 64
#pragma unroll
                    for (int p = 0; p < RN / 64; ++p) tma_load_2d(&tm_b, b + 8192 * p, &full[s], 64 * p, ks * 64);
                } else {     // map (inner = K, outer = N), box 64 x RN
                    tma_load_2d(&tm_b, b, &full[s], ks * 64, 0);
                }
                if (++s == (uint32_t)C::NS) {
                    s = 0;
                    ph ^= 1;
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issue
        if (elect_one()) {
            constexpr uint32_t kIdesc = idesc_bf16(kBM, RN, false) | (A_MN ? (1u << 15) : 0u) | (B_MN ? (1u << 16) : 0u);
            uint32_t s = 0, ph = 0;
            bool ok = true;
            for (int ks = k_begin; ks < k_end; ++ks) {
                if (!mbar_wait(&full[s], ph)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a = smem_u32(smem + s * C::STAGE), b = a + C::A_BYTES;
#pragma unroll
                for (int c = 0; c < 4; ++c) {  // K = 16 per MMA: 32 B along a K-major row, two 8-row groups MN-major
                    const uint64_t da = A_MN ? desc_mn_sw128(a + 2048 * c) : desc_sw128(a + 32 * c);
                    const uint64_t db = B_MN ? desc_mn_sw128(b + 2048 * c) : desc_sw128(b + 32 * c);
                    mma_dense(tmem_base, da, db, kIdesc, (ks > k_begin) || c);
                }
                mma_commit(&empty[s]);
                if (++s == (uint32_t)C::NS) {
                    s = 0;
                    ph ^= 1;
                }
            }
            if (!ok) {
                *fail = 1;
                atomicOr(&g_bwd_error, 2u);
            }
            mma_commit(acc_full);  // also fires when this CTA had no stages
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue: TMEM -> shared (fp32)
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const bool have = k_end > k_begin;
        if (mbar_wait(acc_full, 0)) {
            tc_fence_after();
#pragma unroll 1
            for (int q = 0; q < RN / 16; ++q) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(q * 16), v);
                float4 *dst = reinterpret_cast<float4 *>(part + row * C::PROW + q * 16);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    dst[j] = have ? make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        } else {
            *fail = 1;
            atomicOr(&g_bwd_error, 4u);
        }
    }
    tc_fence_before();
    cluster_sync_all();  // every CTA's partial is in its shared memory

    // Reduction over the cluster: CTA q owns rows [q*TPC, (q+1)*TPC) of the tile.
    if (warp >= 2) {
        const int tpc = kBM / (int)ks_n;
        const int items = tpc * (RN / 4);
        const uint32_t part_addr = smem_u32(part);
        for (int it = threadIdx.x - 64; it < items; it += 128) {
            const int t = (int)ks_q * tpc + it / (RN / 4);
            const int c = (it % (RN / 4)) * 4;
            const uint32_t off = (uint32_t)((t * C::PROW + c) * 4);
            float4 p[8];
#pragma unroll
            for (uint32_t q = 0; q < 8; ++q)
                p[q] = q < ks_n ? ld_shared_cluster_v4(mapa_shared(part_addr + off, q)) : make_float4(0.f, 0.f, 0.f, 0.f);
            float4 acc = p[0];
#pragma unroll
            for (int q = 1; q < 8; ++q) {
                acc.x += p[q].x;
                acc.y += p[q].y;
                acc.z += p[q].z;
                acc.w += p[q].w;
            }
            const int m = m0 + t;
            if (m < Mc && c < N) {  // N % 8 == 0: the four columns are all in range
                if (OUT == kOutF32) {
                    *reinterpret_cast<float4 *>(static_cast<float *>(out) + (int64_t)m * N + c) = acc;
                } else if (OUT == kOutF32T) {
                    float *o = static_cast<float *>(out);
                    o[(int64_t)(c + 0) * Mc + m] = acc.x;
                    o[(int64_t)(c + 1) * Mc + m] = acc.y;
                    o[(int64_t)(c + 2) * Mc + m] = acc.z;
                    o[(int64_t)(c + 3) * Mc + m] = acc.w;
                } else {
                    uint2 packed;
                    packed.x = (uint32_t)f32_to_bf16_bits(acc.x) | ((uint32_t)f32_to_bf16_bits(acc.y) << 16);
                    packed.y = (uint32_t)f32_to_bf16_bits(acc.z) | ((uint32_t)f32_to_bf16_bits(acc.w) << 16);
                    *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(out) + (int64_t)m * N + c) = packed;
                }
            }
        }
    }
    cluster_sync_all();  // no CTA leaves while its partial may still be read
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
    }
}

constexpr auto kBF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;

// C = sum_k A(k, m) B(k, n).  A_MN: A stored [K][Mc] (row-major, lda elements);
// else [Mc][K].  B_MN: B stored [K][N] (ldb); else [N][K].
template <bool A_MN, bool B_MN, int RN, int OUT>
cudaError_t gemm_tc(const uint16_t *A, int64_t lda, const uint16_t *B, int64_t ldb, int64_t Mc, int64_t N, int64_t K,
                    void *out, cudaStream_t stream) {
    using C = CfgB<RN>;
    CUtensorMap ma, mb;
    const bool ok_a = A_MN ? make_map(&ma, kBF16, A, Mc, K, lda * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)
                           : make_map(&ma, kBF16, A, K, Mc, lda * 2, 64, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
    const bool ok_b = B_MN ? make_map(&mb, kBF16, B, N, K, ldb * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)
                           : make_map(&mb, kBF16, B, K, N, ldb * 2, 64, RN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok_a || !ok_b) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int tiles = (int)((Mc + kBM - 1) / kBM);
    const int nk = (int)((K + 63) / 64);
    int ks = 1;
    while (ks < 8 && ks * 2 <= nk && tiles * ks * 2 <= (ks >= 4 ? sms : 2 * sms)) ks *= 2;
    cudaError_t err = cudaFuncSetAttribute(tc_gemm_kernel<A_MN, B_MN, RN, OUT>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * ks));
    cfg.blockDim = dim3(kBThreads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, tc_gemm_kernel<A_MN, B_MN, RN, OUT>, ma, mb, out, (int32_t)Mc, (int32_t)N,
                              (int32_t)nk);
}

// A second stream per device, so that dU (which needs only dY and T) runs
// beside G and dV; created once, never destroyed (it lives as long as the
// process, like the library's other per-device state).
cudaStream_t side_stream() {
    static std::mutex mu;
    static cudaStream_t streams[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (streams[dev] == nullptr && cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess)
        streams[dev] = nullptr;
    return streams[dev];
}

template <int RN>
cudaError_t backward_rn(const uint16_t *X, int64_t M, const uint16_t *dY, int64_t d_out, int64_t d_in,
                        const uint16_t *U, const uint16_t *T16, uint16_t *G16, int64_t r, float *dU, float *dV,
                        cudaStream_t st) {
    // dU = dY^T T (A = dY [M][d_out] MN-major, K = M; B = T [M][r] MN-major) on
    // the side stream, forked from and joined back into `st` with events, while
    // `st` runs G = dY U (A = dY K-major, K = d_out; B = U [d_out][r] MN-major)
    // and then dV^T = X^T G (A = X [M][d_in] MN-major, B = G [M][r] MN-major,
    // stored transposed as dV [r][d_in]).  Without a side stream, all on `st`.
    cudaStream_t side = side_stream();
    cudaEvent_t fork = nullptr, join = nullptr;
    if (side != nullptr && (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess ||
                            cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess)) {
        if (fork != nullptr) cudaEventDestroy(fork);
        fork = join = nullptr;
        side = nullptr;
    }
    cudaError_t e = cudaSuccess;
    cudaStream_t su = st;
    if (side != nullptr) {
        e = cudaEventRecord(fork, st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(side, fork, 0);
        if (e == cudaSuccess) su = side;
    }
    if (e == cudaSuccess) e = gemm_tc<true, true, RN, kOutF32>(dY, d_out, T16, r, d_out, r, M, dU, su);
    if (e == cudaSuccess && side != nullptr) e = cudaEventRecord(join, side);
    if (e == cudaSuccess) e = gemm_tc<false, true, RN, kOutBF16>(dY, d_out, U, r, M, r, d_out, G16, st);
    if (e == cudaSuccess) e = gemm_tc<true, true, RN, kOutF32T>(X, d_in, G16, r, d_in, r, M, dV, st);
    if (e == cudaSuccess && side != nullptr) e = cudaStreamWaitEvent(st, join, 0);
    if (fork != nullptr) cudaEventDestroy(fork);  // released once the recorded work completes
    if (join != nullptr) cudaEventDestroy(join);
    return e;
}

}  // namespace

cudaError_t launch_lora_backward(const uint16_t *X, int64_t M, const uint16_t *dY, int64_t d_out, int64_t d_in,
                                 const uint16_t *U, const uint16_t *V, int64_t r, const uint16_t *T16_in, float *dU,
                                 float *dV, uint16_t *ws, cudaStream_t st) {
    uint16_t *T16 = ws;                 // M x r (when not given)
    uint16_t *G16 = ws + M * r;         // M x r
    cudaError_t e = cudaSuccess;
    if (T16_in == nullptr) {
        e = launch_tc_project(X, M, V, d_in, r, T16, st);
        T16_in = T16;
    }
    if (e != cudaSuccess) return e;
    if (r <= 64) return backward_rn<64>(X, M, dY, d_out, d_in, U, T16_in, G16, r, dU, dV, st);
    if (r <= 128) return backward_rn<128>(X, M, dY, d_out, d_in, U, T16_in, G16, r, dU, dV, st);
    return backward_rn<256>(X, M, dY, d_out, d_in, U, T16_in, G16, r, dU, dV, st);
}

cudaError_t read_and_clear_backward_error(unsigned *code) {
    unsigned v = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_bwd_error, sizeof v);
    if (err != cudaSuccess) return err;
    if (v != 0) {
        const unsigned zero = 0;
        err = cudaMemcpyToSymbol(g_bwd_error, &zero, sizeof zero);
    }
    *code = v;
    return err;
}

}  // namespace slr

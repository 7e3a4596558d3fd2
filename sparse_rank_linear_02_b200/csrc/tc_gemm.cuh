// tc_gemm.cuh -- a tcgen05 GEMM for products with one small side (internal).
//
// C (Mc x N, N <= RN) = sum_k A(k, m) B(k, n) over K in 64-deep stages, for
// the products whose N is a low rank r (the backward with respect to the
// low-rank factors, the subspace iteration of the data-free decomposition).
// A is a 128 x 64 tile (K-major: 128 rows of 64 K; MN-major: two 64-wide MN
// panels of 64 K rows), B an RN x 64 tile (K-major) or RN/64 panels
// (MN-major), all loaded by TMA with the 128-byte swizzle; tcgen05.mma
// kind::f16 (bf16 in, fp32 in TMEM) with the operand major-ness in the
// instruction descriptor, so row-major activations are read in place whatever
// dimension is contracted.  With SPLIT, each operand comes as two bf16 planes
// (a high part and the bf16 rounding of the remainder) and every k step
// issues hi*hi + hi*lo + lo*hi: three bf16 products that carry about 16
// significant bits of each fp32 operand.  A cluster of KS CTAs splits the K
// stages of one 128-row tile; their fp32 partials meet in shared memory and
// are summed over distributed shared memory, then written once: fp32
// row-major, fp32 transposed, or bf16 row-major.  Every wait is bounded and
// reports to the error word the launcher passes.
//
// Included by one translation unit per user; everything is in an anonymous
// namespace there.
#pragma once

#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "tc_forward.cuh"
#include "tc_ptx.cuh"

namespace slr {
namespace {

using namespace tc;

constexpr int kBM = 128;       // output rows per tile (MMA M)
constexpr int kBThreads = 192;  // producer, MMA, four epilogue warps

// Outputs: fp32 row-major, fp32 transposed, bf16 row-major, or the fused
// residual / 2:4 threshold of the data-free decomposition (ResidOut).
enum OutMode { kOutF32 = 0, kOutF32T = 1, kOutBF16 = 2, kOutResid = 3 };

// kOutResid: C = P Q^T is the rank-r part of W; the epilogue forms R = W - C
// per group of four columns, keeps the two largest |R| (ties to the lower
// index), writes them packed (vals, meta) and Z = W - S as two bf16 planes,
// and leaves the CTA's sum of (R - S)^2 in obj_part[tile].
struct ResidOut {
    const uint16_t *W;  // bf16 [Mc][N]
    uint16_t *vals;     // bf16 [Mc][N / 2]
    uint8_t *meta;      // uint8 [Mc][N / 8]
    uint16_t *Zhi, *Zlo;  // bf16 [Mc][N] each
    float *obj_part;    // one float per CTA
};

// The two positions of a group of four kept by |value| (ties to the lower
// index), from the fp32 magnitudes' bit patterns: the tournament of (0,1) and
// (2,3), the better winner first, then the better of the winning pair's loser
// and the losing pair's winner.  Returns idx0 | idx1 << 2.
__device__ __forceinline__ uint32_t gemm_keep_two(float v0, float v1, float v2, float v3) {
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

template <int RN, bool SPLIT, int NSMAX = 8>
struct CfgB {
    static constexpr int A_BYTES = kBM * 64 * 2;   // 16 KB per plane
    static constexpr int B_BYTES = RN * 64 * 2;
    static constexpr int PLANES = SPLIT ? 2 : 1;
    static constexpr int STAGE = ((PLANES * (A_BYTES + B_BYTES) + 1023) / 1024) * 1024;
    static constexpr int PROW = RN + 4;
    static constexpr int P_BYTES = kBM * PROW * 4;
    static constexpr int NS_FIT = (SPLIT ? 200704 : 112640) / STAGE;
    static constexpr int NS0 = NS_FIT > 8 ? 8 : (NS_FIT < 2 ? 2 : NS_FIT);
    static constexpr int NS = NS0 < NSMAX ? NS0 : NSMAX;
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

template <bool A_MN, bool B_MN, int RN, int OUT, bool SPLIT>
__global__ void __launch_bounds__(kBThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a2,
                   const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_b2,
                   void *__restrict__ out, int32_t Mc, int32_t N, int32_t nk_total, unsigned int *err,
                   ResidOut ro) {
    using C = CfgB<RN, SPLIT, OUT == kOutResid ? 1 : 8>;
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
    const int n0 = blockIdx.y * RN;  // N tiles (the residual mode only; otherwise one)
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

    // Residual mode: each epilogue thread's W values, loaded before the wait for
    // the accumulator so that the loads overlap the tensor-core work (the item
    // loop below has a fixed trip count there, so the indices are static).
    constexpr int kResidItems = RN / 4;  // items per epilogue thread (one CTA per tile)
    uint2 wpre[OUT == kOutResid ? kResidItems : 1];

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (elect_one()) {
            uint32_t s = 0, ph = 0;
            for (int ks = k_begin; ks < k_end; ++ks) {
                if (!mbar_wait(&empty[s], ph ^ 1)) {
                    *fail = 1;
                    atomicOr(err, 1u);
                    break;
                }
                const uint32_t base = smem_u32(smem + s * C::STAGE);
                mbar_expect_tx(&full[s], C::PLANES * (C::A_BYTES + C::B_BYTES));
#pragma unroll
                for (int pl = 0; pl < C::PLANES; ++pl) {
                    const CUtensorMap *ma = pl ? &tm_a2 : &tm_a, *mb = pl ? &tm_b2 : &tm_b;
                    const uint32_t a = base + pl * C::A_BYTES;
                    const uint32_t b = base + C::PLANES * C::A_BYTES + pl * C::B_BYTES;
                    if (A_MN) {  // map (inner = MN, outer = K), box 64 x 64
                        tma_load_2d(ma, a, &full[s], m0, ks * 64);
                        tma_load_2d(ma, a + 8192, &full[s], m0 + 64, ks * 64);
                    } else {     // map (inner = K, outer = MN), box 64 x 128
                        tma_load_2d(ma, a, &full[s], ks * 64, m0);
                    }
                    if (B_MN) {  // map (inner = N, outer = K), box 64 x 64
#pragma unroll
                        for (int p = 0; p < RN / 64; ++p) tma_load_2d(mb, b + 8192 * p, &full[s], n0 + 64 * p, ks * 64);
                    } else {     // map (inner = K, outer = N), box 64 x RN
                        tma_load_2d(mb, b, &full[s], ks * 64, n0);
                    }
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
                const uint32_t a = smem_u32(smem + s * C::STAGE), b = a + C::PLANES * C::A_BYTES;
#pragma unroll
                for (int c = 0; c < 4; ++c) {  // K = 16 per MMA: 32 B along a K-major row, two 8-row groups MN-major
                    const uint32_t ao = A_MN ? 2048 * c : 32 * c, bo = B_MN ? 2048 * c : 32 * c;
                    auto da = [&](int pl) {
                        return A_MN ? desc_mn_sw128(a + pl * C::A_BYTES + ao) : desc_sw128(a + pl * C::A_BYTES + ao);
                    };
                    auto db = [&](int pl) {
                        return B_MN ? desc_mn_sw128(b + pl * C::B_BYTES + bo) : desc_sw128(b + pl * C::B_BYTES + bo);
                    };
                    mma_dense(tmem_base, da(0), db(0), kIdesc, (ks > k_begin) || c);
                    if (SPLIT) {  // hi*lo + lo*hi: the lo*lo term is below the fp32 accumulation error
                        mma_dense(tmem_base, da(0), db(1), kIdesc, 1);
                        mma_dense(tmem_base, da(1), db(0), kIdesc, 1);
                    }
                }
                mma_commit(&empty[s]);
                if (++s == (uint32_t)C::NS) {
                    s = 0;
                    ph ^= 1;
                }
            }
            if (!ok) {
                *fail = 1;
                atomicOr(err, 2u);
            }
            mma_commit(acc_full);  // also fires when this CTA had no stages
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue: TMEM -> shared (fp32)
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const bool have = k_end > k_begin;
        if (OUT == kOutResid) {
#pragma unroll
            for (int k = 0; k < kResidItems; ++k) {
                const int it = threadIdx.x - 64 + 128 * k;
                const int m = m0 + it / (RN / 4), n = n0 + (it % (RN / 4)) * 4;
                wpre[k] = (m < Mc && n < N) ? __ldg(reinterpret_cast<const uint2 *>(ro.W + (int64_t)m * N + n))
                                            : make_uint2(0, 0);
            }
        }
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
            atomicOr(err, 4u);
        }
    }
    tc_fence_before();
    cluster_sync_all();  // every CTA's partial is in its shared memory

    // Reduction over the cluster: CTA q owns rows [q*TPC, (q+1)*TPC) of the tile.
    float obj = 0.f;  // the residual mode's sum of (R - S)^2
    if (OUT == kOutResid && warp >= 2) {
        // One CTA per tile (no K split): item it = row t, columns c..c+3, one
        // group of four; the partner item (the next lane) holds the other
        // group of the same metadata byte.
        const uint32_t part_addr = smem_u32(part);
#pragma unroll
        for (int k = 0; k < kResidItems; ++k) {
            const int it = threadIdx.x - 64 + 128 * k;
            const int t = it / (RN / 4), c = (it % (RN / 4)) * 4;
            const float4 acc = ld_shared_cluster_v4(mapa_shared(part_addr + (uint32_t)((t * C::PROW + c) * 4), 0));
            const int m = m0 + t, n = n0 + c;
            const bool in = m < Mc && n < N;
            uint32_t nib = 0;
            if (in) {
                const uint2 w = wpre[k];
                const float w0 = bf16lo_to_f32(w.x), w1 = bf16hi_to_f32(w.x);
                const float w2 = bf16lo_to_f32(w.y), w3 = bf16hi_to_f32(w.y);
                const float R[4] = {w0 - acc.x, w1 - acc.y, w2 - acc.z, w3 - acc.w};
                const float Wv[4] = {w0, w1, w2, w3};
                nib = gemm_keep_two(R[0], R[1], R[2], R[3]);
                const uint32_t a = nib & 3u, b = nib >> 2;  // a in 0..2, b in 1..3
                uint32_t sv[4], zh[4], zl[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    sv[q] = f32_to_bf16_bits(R[q]);
                    const float sq = (q == (int)a || q == (int)b) ? __uint_as_float(sv[q] << 16) : 0.f;
                    const float z = Wv[q] - sq, e = R[q] - sq;
                    obj = fmaf(e, e, obj);
                    zh[q] = f32_to_bf16_bits(z);
                    zl[q] = f32_to_bf16_bits(z - __uint_as_float(zh[q] << 16));
                }
                const uint32_t sa = a == 0u ? sv[0] : (a == 1u ? sv[1] : sv[2]);
                const uint32_t sb = b == 1u ? sv[1] : (b == 2u ? sv[2] : sv[3]);
                *reinterpret_cast<uint32_t *>(ro.vals + (int64_t)m * (N / 2) + n / 2) = sa | (sb << 16);
                *reinterpret_cast<uint2 *>(ro.Zhi + (int64_t)m * N + n) =
                    make_uint2(zh[0] | (zh[1] << 16), zh[2] | (zh[3] << 16));
                *reinterpret_cast<uint2 *>(ro.Zlo + (int64_t)m * N + n) =
                    make_uint2(zl[0] | (zl[1] << 16), zl[2] | (zl[3] << 16));
            }
            const uint32_t partner = __shfl_down_sync(0xFFFFFFFFu, nib, 1);
            if (in && (c & 4) == 0) ro.meta[(int64_t)m * (N / 8) + n / 8] = (uint8_t)(nib | (partner << 4));
        }
    } else if (warp >= 2) {
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
    if (OUT == kOutResid && warp >= 2) {
        // The four epilogue warps' sums, added in warp order (deterministic).
        float *red = reinterpret_cast<float *>(tmem_slot + 2);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) obj += __shfl_xor_sync(0xFFFFFFFFu, obj, o);
        if (lane == 0) red[warp - 2] = obj;
        named_bar_sync(1, 128);
        if (threadIdx.x == 64) ro.obj_part[blockIdx.y * gridDim.x + blockIdx.x] = ((red[0] + red[1]) + red[2]) + red[3];
    }
    cluster_sync_all();  // no CTA leaves while its partial may still be read
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
    }
}

constexpr auto kBF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;

// C = sum_k A(k, m) B(k, n).  A_MN: A stored [K][Mc] (row-major, lda elements);
// else [Mc][K].  B_MN: B stored [K][N] (ldb); else [N][K].  SPLIT: A = A + A2
// and B = B + B2 (bf16 high and low parts), C = A B + A B2 + A2 B.  err: the
// device word the kernel's bounded waits report to.
template <bool A_MN, bool B_MN, int RN, int OUT, bool SPLIT = false>
cudaError_t gemm_tc(const uint16_t *A, const uint16_t *A2, int64_t lda, const uint16_t *B, const uint16_t *B2,
                    int64_t ldb, int64_t Mc, int64_t N, int64_t K, void *out, unsigned int *err,
                    cudaStream_t stream, ResidOut ro = ResidOut{}) {
    using C = CfgB<RN, SPLIT, OUT == kOutResid ? 1 : 8>;
    if (err == nullptr) return cudaErrorInvalidValue;
    CUtensorMap ma, ma2, mb, mb2;
    auto map_a = [&](CUtensorMap *m, const uint16_t *p) {
        return A_MN ? make_map(m, kBF16, p, Mc, K, lda * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)
                    : make_map(m, kBF16, p, K, Mc, lda * 2, 64, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
    };
    auto map_b = [&](CUtensorMap *m, const uint16_t *p) {
        return B_MN ? make_map(m, kBF16, p, N, K, ldb * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)
                    : make_map(m, kBF16, p, K, N, ldb * 2, 64, RN, CU_TENSOR_MAP_SWIZZLE_128B);
    };
    if (!map_a(&ma, A) || !map_b(&mb, B)) return cudaErrorInvalidValue;
    if (SPLIT ? (!map_a(&ma2, A2) || !map_b(&mb2, B2)) : false) return cudaErrorInvalidValue;
    if (!SPLIT) {
        ma2 = ma;
        mb2 = mb;
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int tiles = (int)((Mc + kBM - 1) / kBM);
    const int nk = (int)((K + 63) / 64);
    int ks = 1;
    while (OUT != kOutResid && ks < 8 && ks * 2 <= nk && tiles * ks * 2 <= (ks >= 4 ? sms : 2 * sms)) ks *= 2;
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<A_MN, B_MN, RN, OUT, SPLIT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * ks), OUT == kOutResid ? (unsigned)((N + RN - 1) / RN) : 1u);
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
    return cudaLaunchKernelEx(&cfg, tc_gemm_kernel<A_MN, B_MN, RN, OUT, SPLIT>, ma, ma2, mb, mb2, out, (int32_t)Mc,
                              (int32_t)N, (int32_t)nk, err, ro);
}


}  // namespace
}  // namespace slr

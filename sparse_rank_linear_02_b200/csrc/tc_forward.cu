// tc_forward.cu -- Y = X S^T + T U^T on the 5th-generation tensor cores (sm_100a).
//
// The compressed layer of LoSparse (section 3.2) evaluates a sparse term and a
// low-rank term side by side; HASSLE-free (section 1, abstract) picks 2:4
// sparsity for S precisely because GPUs accelerate it.  This kernel runs the
// 2:4 term on tcgen05.mma.sp (half the MMA work of the dense product) and
// accumulates the rank-r term into the same TMEM accumulator, so Y is written
// to HBM once.
//
// Operand roles ("swap AB": only operand A of tcgen05.mma.sp may be sparse):
//   A = S tile     128 output rows x 128 logical K (64 stored bf16 / row),
//   B = X tile     BN tokens x 128 K,
//   D = Y^T tile   128 lanes (output rows) x BN fp32 columns in TMEM.
// After the d_in/128 sparse K steps, ceil(r/64) "rank steps" add
//   A = U tile (128 rows x 64 of r), B = T tile (BN tokens x 64 of r)
// with dense tcgen05.mma into the same accumulator.  T = X V^T comes from the
// projection kernel that runs before this one on the stream.
//
// Metadata: the exported format is row-major, one nibble per group of four.
// The tensor core reads sparse metadata from TMEM, one 32-bit column per MMA
// K-step of 32, with lane L = m0 + 8*k1 + 16*m2 holding rows m0+16*m2 and
// m0+8+16*m2 for logical K half k1 (the layout the PTX ISA defines for M=128
// kind::f16 sparse MMA).  A 2 KB tile of row-major metadata is therefore
// permuted in shared memory (a swap of one row bit with one 16-bit-word bit,
// done by the MMA warp with byte permutes) and moved to TMEM with one
// tcgen05.cp 128x128b per stage.
//
// Structure: persistent CTAs (one per SM), 6 warps:
//   warp 0     TMA producer (one lane) filling an NS-stage shared-memory ring,
//   warp 1     TMEM allocator, metadata permute, single-thread MMA issue,
//   warps 2..5 epilogue: tcgen05.ld -> bf16 (RNE) -> smem -> TMA store of Y.
// Two TMEM accumulators let the epilogue of tile i overlap the MMAs of tile
// i+1.  Every mbarrier wait is bounded; on expiry the kernel records an error
// word, leaves its loops, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "tc_forward.cuh"

namespace slr {

__device__ unsigned int g_tc_error = 0;

namespace tc {

constexpr int BM = 128;            // output rows per tile (MMA M)
constexpr int BK = 128;            // logical K per pipeline stage
constexpr int kThreads = 192;      // 6 warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kEcol = 256;    // metadata columns start after two accumulators
constexpr long long kWaitCycles = 2000000000LL;  // ~1 s at the boost clock

template <int BN>
struct Cfg {
    static constexpr int A_BYTES = BM * (BK / 2) * 2;   // 16 KB of packed values
    static constexpr int B_HALF = BN * 64 * 2;          // one 128-byte-wide swizzle panel of X
    static constexpr int B_BYTES = 2 * B_HALF;
    static constexpr int E_BYTES = BM * BK / 8;         // 2 KB of metadata
    static constexpr int STAGE = A_BYTES + B_BYTES + E_BYTES;
    static constexpr int NS = (BN == 128) ? 4 : 6;
    static constexpr int OUT_COLS = 32;                 // tokens per output chunk
    static constexpr int OUT_BYTES = OUT_COLS * BM * 2;
    static constexpr int RING = NS * STAGE;
    static constexpr int BAR_OFF = RING + 2 * OUT_BYTES;
    static constexpr int SMEM = BAR_OFF + 256 + 1024;   // barriers + alignment slack
    static_assert(STAGE % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(SMEM <= 232448, "shared memory budget");
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: false when the phase did not complete within kWaitCycles.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > kWaitCycles) return false;
    }
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap *map, uint32_t dst, uint64_t *bar, int32_t c0,
                                            int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int32_t c0, int32_t c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor (tcgen05 "version 1" format): start address,
// leading/stride byte offsets in 16-byte units, layout type in bits 61..63.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for tcgen05
    d |= (uint64_t)layout << 61;
    return d;
}
constexpr uint32_t kLayoutSW128 = 2;
constexpr uint32_t kLayoutNone = 0;

// K-major, 128-byte swizzled operand tile: 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) { return smem_desc(addr, 16, 1024, kLayoutSW128); }

// Instruction descriptor, kind::f16 with bf16 inputs and fp32 accumulation,
// both operands K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, bool sparse) {
    return (sparse ? (1u << 2) : 0u)       // sparsity flag
           | (1u << 4)                     // D format: f32
           | (1u << 7)                     // A format: bf16
           | (1u << 10)                    // B format: bf16
           | ((uint32_t)(n >> 3) << 17)    // N / 8
           | ((uint32_t)(m >> 4) << 24);   // M / 16
}

__device__ __forceinline__ void mma_sp(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t e_tmem, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.sp.cta_group::1.kind::f16 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(e_tmem), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_dense(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tmem_cp_128x128b(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Permute one 2 KB metadata tile in place from the exported row-major layout
// ([128 rows][16 bytes], byte j = groups 2j, 2j+1) into the tcgen05.cp source
// layout.  Lane handles row pairs p = lane and lane + 32, p = m0 + 8*m2:
// rows A = m0 + 16*m2 and B = A + 8 are read whole and rewritten as
//   row A = [A.w0 B.w0 A.w2 B.w2 A.w4 B.w4 A.w6 B.w6]   (16-bit words)
//   row B = [A.w1 B.w1 A.w3 B.w3 A.w5 B.w5 A.w7 B.w7]
// Rows past d_out arrive zero-filled from TMA, i.e. with the index pair
// (0, 0), which is not a valid 2:4 pattern; rewrite any nibble whose two
// indices are equal to (0, 1).  The values there are zero, so the choice
// does not change the result; it only keeps the hardware on defined input.
__device__ __forceinline__ uint32_t sanitize_nibbles(uint32_t w) {
    const uint32_t lo = w & 0x33333333u, hi = (w >> 2) & 0x33333333u;
    const uint32_t same = ~(lo ^ hi);
    const uint32_t eq = same & (same >> 1) & 0x11111111u;   // one bit per nibble with idx0 == idx1
    return (w & ~(eq * 0xFu)) | (eq * 0x4u);
}

__device__ __forceinline__ void permute_meta_tile(uint8_t *e, int lane) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int p = lane + 32 * h;
        const int rowA = (p & 7) + 16 * (p >> 3);
        uint4 *ra = reinterpret_cast<uint4 *>(e + rowA * 16);
        uint4 *rb = reinterpret_cast<uint4 *>(e + (rowA + 8) * 16);
        uint4 a = *ra, b = *rb;
        a.x = sanitize_nibbles(a.x); a.y = sanitize_nibbles(a.y); a.z = sanitize_nibbles(a.z); a.w = sanitize_nibbles(a.w);
        b.x = sanitize_nibbles(b.x); b.y = sanitize_nibbles(b.y); b.z = sanitize_nibbles(b.z); b.w = sanitize_nibbles(b.w);
        uint4 lo, hi;
        lo.x = __byte_perm(a.x, b.x, 0x5410);
        lo.y = __byte_perm(a.y, b.y, 0x5410);
        lo.z = __byte_perm(a.z, b.z, 0x5410);
        lo.w = __byte_perm(a.w, b.w, 0x5410);
        hi.x = __byte_perm(a.x, b.x, 0x7632);
        hi.y = __byte_perm(a.y, b.y, 0x7632);
        hi.z = __byte_perm(a.z, b.z, 0x7632);
        hi.w = __byte_perm(a.w, b.w, 0x7632);
        *ra = lo;
        *rb = hi;
    }
}

struct Params {
    int32_t M, d_out, d_in, r;
    int32_t n_dtiles, n_tiles, nk, nlr;
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    tc_forward_kernel(const __grid_constant__ CUtensorMap tm_vals, const __grid_constant__ CUtensorMap tm_meta,
                      const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_u,
                      const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_y,
                      const Params prm) {
    using C = Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *empty = full + C::NS;
    uint64_t *acc_full = empty + C::NS;
    uint64_t *acc_empty = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
    volatile uint32_t *fail = tmem_slot + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        *fail = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_vals)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_meta)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_x)) : "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t s = 0, ph = 0;
            for (int tile = blockIdx.x; tile < prm.n_tiles && !*fail; tile += gridDim.x) {
                const int tok0 = (tile / prm.n_dtiles) * BN;
                const int d0 = (tile % prm.n_dtiles) * BM;
                for (int ks = 0; ks < prm.nk + prm.nlr; ++ks) {
                    if (!mbar_wait(&empty[s], ph ^ 1)) {
                        *fail = 1;
                        atomicOr(&g_tc_error, 1u);
                        break;
                    }
                    uint8_t *st = smem + s * C::STAGE;
                    const uint32_t a = smem_u32(st), b = smem_u32(st + C::A_BYTES),
                                   e = smem_u32(st + C::A_BYTES + C::B_BYTES);
                    if (ks < prm.nk) {
                        mbar_expect_tx(&full[s], C::A_BYTES + C::B_BYTES + C::E_BYTES);
                        tma_load_2d(&tm_vals, a, &full[s], ks * 64, d0);
                        tma_load_2d(&tm_x, b, &full[s], ks * BK, tok0);
                        tma_load_2d(&tm_x, b + C::B_HALF, &full[s], ks * BK + 64, tok0);
                        tma_load_2d(&tm_meta, e, &full[s], ks * (BK / 8), d0);
                    } else {
                        const int j = ks - prm.nk;
                        mbar_expect_tx(&full[s], C::A_BYTES + C::B_HALF);
                        tma_load_2d(&tm_u, a, &full[s], j * 64, d0);
                        tma_load_2d(&tm_t, b, &full[s], j * 64, tok0);
                    }
                    if (++s == (uint32_t)C::NS) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue
        constexpr uint32_t kIdescSp = idesc_bf16(BM, BN, true);
        constexpr uint32_t kIdescDense = idesc_bf16(BM, BN, false);
        const uint32_t e_tmem = tmem_base + kEcol;
        uint32_t s = 0, ph = 0;
        int it = 0;
        for (int tile = blockIdx.x; tile < prm.n_tiles && !*fail; tile += gridDim.x, ++it) {
            const int buf = it & 1;
            const uint32_t use = (uint32_t)(it >> 1);
            if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1)) {
                *fail = 1;
                atomicOr(&g_tc_error, 2u);
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
            bool ok = true;
            for (int ks = 0; ks < prm.nk + prm.nlr; ++ks) {
                if (!mbar_wait(&full[s], ph)) {
                    ok = false;
                    break;
                }
                uint8_t *st = smem + s * C::STAGE;
                const uint32_t a = smem_u32(st), b = smem_u32(st + C::A_BYTES);
                if (ks < prm.nk) {
                    permute_meta_tile(st + C::A_BYTES + C::B_BYTES, lane);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tc_fence_after();
                        tmem_cp_128x128b(e_tmem, smem_desc(smem_u32(st + C::A_BYTES + C::B_BYTES), 0, 128, kLayoutNone));
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const uint64_t adesc = desc_sw128(a + 32 * c);
                            const uint64_t bdesc = desc_sw128(b + (c >> 1) * C::B_HALF + (c & 1) * 64);
                            mma_sp(d_tmem, adesc, bdesc, e_tmem + (uint32_t)(c & 2), kIdescSp | (uint32_t)(c & 1),
                                   (ks | c) != 0);
                        }
                        mma_commit(&empty[s]);
                    }
                } else if (lane == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        mma_dense(d_tmem, desc_sw128(a + 32 * c), desc_sw128(b + 32 * c), kIdescDense, 1u);
                    mma_commit(&empty[s]);
                }
                __syncwarp();
                if (++s == (uint32_t)C::NS) {
                    s = 0;
                    ph ^= 1;
                }
            }
            if (!ok) {
                *fail = 1;
                atomicOr(&g_tc_error, 4u);
                break;
            }
            if (lane == 0) mma_commit(&acc_full[buf]);
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;              // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;       // output row within the tile
        const bool leader = (warp == 2 && lane == 0);
        uint8_t *stage_out = smem + C::RING;
        uint32_t chunk = 0;
        int it = 0;
        for (int tile = blockIdx.x; tile < prm.n_tiles && !*fail; tile += gridDim.x, ++it) {
            const int tok0 = (tile / prm.n_dtiles) * BN;
            const int d0 = (tile % prm.n_dtiles) * BM;
            const int buf = it & 1;
            const uint32_t use = (uint32_t)(it >> 1);
            if (!mbar_wait(&acc_full[buf], use & 1)) {
                *fail = 1;
                atomicOr(&g_tc_error, 8u);
                break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int q = 0; q < BN / C::OUT_COLS; ++q) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN + q * 32), v);
                if (q == BN / C::OUT_COLS - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acc_empty[buf]);
                }
                if (tok0 + q * C::OUT_COLS >= prm.M) continue;  // uniform across the epilogue warps
                const uint32_t sb = chunk & 1;
                if (leader) bulk_wait_read1();
                named_bar_sync(1, 128);
                uint16_t *out = reinterpret_cast<uint16_t *>(stage_out + sb * C::OUT_BYTES);
#pragma unroll
                for (int j = 0; j < 32; ++j) out[j * BM + row] = f32_to_bf16_bits(__uint_as_float(v[j]));
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (leader) {
                    tma_store_2d(&tm_y, smem_u32(out), d0, tok0 + q * C::OUT_COLS);
                    bulk_commit();
                }
                ++chunk;
            }
        }
        if (leader) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols));
    }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool make_map(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
cudaError_t launch(const uint16_t *X, int64_t M, const uint16_t *vals, const uint8_t *meta, int64_t d_out,
                   int64_t d_in, const uint16_t *U, const uint16_t *T16, int64_t r, uint16_t *Y,
                   cudaStream_t stream) {
    using C = Cfg<BN>;
    CUtensorMap m_vals, m_meta, m_x, m_u, m_t, m_y;
    memset(&m_u, 0, sizeof m_u);
    memset(&m_t, 0, sizeof m_t);
    const auto BF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    bool ok = make_map(&m_vals, BF16, vals, d_in / 2, d_out, d_in, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&m_meta, CU_TENSOR_MAP_DATA_TYPE_UINT8, meta, d_in / 8, d_out, d_in / 8, 16, BM,
                       CU_TENSOR_MAP_SWIZZLE_NONE) &&
              make_map(&m_x, BF16, X, d_in, M, d_in * 2, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&m_y, BF16, Y, d_out, M, d_out * 2, BM, C::OUT_COLS, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (ok && r > 0)
        ok = make_map(&m_u, BF16, U, r, d_out, r * 2, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&m_t, BF16, T16, r, M, r * 2, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;

    Params prm;
    prm.M = (int32_t)M;
    prm.d_out = (int32_t)d_out;
    prm.d_in = (int32_t)d_in;
    prm.r = (int32_t)r;
    prm.n_dtiles = (int32_t)((d_out + BM - 1) / BM);
    const int64_t n_ttiles = (M + BN - 1) / BN;
    prm.n_tiles = (int32_t)(prm.n_dtiles * n_ttiles);
    prm.nk = (int32_t)(d_in / BK);
    prm.nlr = (int32_t)((r + 63) / 64);

    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t err = cudaFuncSetAttribute(tc_forward_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err != cudaSuccess) return err;
    const int grid = prm.n_tiles < sms ? prm.n_tiles : sms;
    tc_forward_kernel<BN><<<grid, kThreads, C::SMEM, stream>>>(m_vals, m_meta, m_x, m_u, m_t, m_y, prm);
    return cudaGetLastError();
}

}  // namespace tc

cudaError_t launch_tc_forward(const uint16_t *X, int64_t M, const uint16_t *vals, const uint8_t *meta,
                              int64_t d_out, int64_t d_in, const uint16_t *U, const uint16_t *T16, int64_t r,
                              uint16_t *Y, cudaStream_t stream) {
    if (M <= 0) return cudaSuccess;
    if (M > INT32_MAX || d_out > INT32_MAX || d_in > INT32_MAX) return cudaErrorInvalidValue;
    return tc::launch<128>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, stream);
}

cudaError_t read_and_clear_kernel_error(unsigned *code) {
    unsigned v = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_tc_error, sizeof v);
    if (err != cudaSuccess) return err;
    if (v != 0) {
        const unsigned zero = 0;
        err = cudaMemcpyToSymbol(g_tc_error, &zero, sizeof zero);
    }
    *code = v;
    return err;
}

}  // namespace slr

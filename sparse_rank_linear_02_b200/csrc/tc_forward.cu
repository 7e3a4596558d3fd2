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

#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "tc_forward.cuh"
#include "tc_ptx.cuh"

namespace slr {

__device__ unsigned int g_tc_error = 0;

namespace tc {

constexpr int BM = 128;            // output rows per tile (MMA M)
constexpr int BK = 128;            // logical K per pipeline stage
constexpr int kThreads = 192;      // 6 warps

constexpr uint32_t pow2_at_least(uint32_t x) {
    uint32_t p = 32;
    while (p < x) p <<= 1;
    return p;
}

// kSparse: the 2:4 forward (A = packed S tile, 128 logical K per stage, plus
// rank stages).  !kSparse: the dense rank projection T^T = V X^T (A = V tile,
// 64 K per stage, no metadata, no rank stages).
template <int BN, bool kSparse>
struct Cfg {
    static constexpr int A_BYTES = BM * 64 * 2;         // 16 KB: 128 rows x one 128-byte swizzle panel
    static constexpr int B_HALF = BN * 64 * 2;          // BN rows x one 128-byte swizzle panel of X
    static constexpr int B_BYTES = kSparse ? 2 * B_HALF : B_HALF;
    static constexpr int E_BYTES = kSparse ? BM * BK / 8 : 0;   // 2 KB of metadata
    static constexpr int STAGE = ((A_BYTES + B_BYTES + E_BYTES + 1023) / 1024) * 1024;
    static constexpr int OUT_COLS = 32;                 // tokens per output chunk
    static constexpr int OUT_BYTES = OUT_COLS * BM * 2;
    static constexpr int NS_FIT = (232448 - 2 * OUT_BYTES - 2048) / STAGE;
    static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
    static constexpr int K_PER_STAGE = kSparse ? BK : 64;
    static constexpr uint32_t ECOL = 2 * BN;            // metadata columns after two accumulators
    static constexpr uint32_t TMEM_COLS = pow2_at_least(2 * BN + (kSparse ? 4 : 0));
    static constexpr int RING = NS * STAGE;
    static constexpr int BAR_OFF = RING + 2 * OUT_BYTES;
    static constexpr int SMEM = BAR_OFF + 256 + 1024;   // barriers + alignment slack
    static_assert(STAGE % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(NS >= 2, "need at least two stages");
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct Params {
    int32_t M;          // tokens
    int32_t n_ttiles;   // token tiles
    int32_t n_tiles;    // output-row tiles x token tiles
    int32_t nk, nlr;    // K stages, rank stages
};

// Tiles run output-row-tile major: the CTAs resident at one time share a few
// S tiles and all token tiles, so X stays in L2 and S is fetched about once.
template <int BN, bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
    tc_forward_kernel(const __grid_constant__ CUtensorMap tm_vals, const __grid_constant__ CUtensorMap tm_meta,
                      const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_u,
                      const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_y,
                      const Params prm) {
    using C = Cfg<BN, kSparse>;
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
                     "r"(C::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_vals)) : "memory");
        if (kSparse) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_meta)) : "memory");
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
                const int d0 = (tile / prm.n_ttiles) * BM;
                const int tok0 = (tile % prm.n_ttiles) * BN;
                for (int ks = 0; ks < prm.nk + prm.nlr; ++ks) {
                    if (!mbar_wait(&empty[s], ph ^ 1)) {
                        *fail = 1;
                        atomicOr(&g_tc_error, 1u);
                        break;
                    }
                    uint8_t *st = smem + s * C::STAGE;
                    const uint32_t a = smem_u32(st), b = smem_u32(st + C::A_BYTES),
                                   e = smem_u32(st + C::A_BYTES + C::B_BYTES);
                    if (!kSparse) {
                        mbar_expect_tx(&full[s], C::A_BYTES + C::B_HALF);
                        tma_load_2d(&tm_vals, a, &full[s], ks * 64, d0);
                        tma_load_2d(&tm_x, b, &full[s], ks * 64, tok0);
                    } else if (ks < prm.nk) {
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
        const uint32_t e_tmem = tmem_base + C::ECOL;
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
                if (!kSparse) {
                    if (lane == 0) {
                        tc_fence_after();
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            mma_dense(d_tmem, desc_sw128(a + 32 * c), desc_sw128(b + 32 * c), kIdescDense,
                                      (ks | c) != 0);
                        mma_commit(&empty[s]);
                    }
                } else if (ks < prm.nk) {
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
            const int d0 = (tile / prm.n_ttiles) * BM;
            const int tok0 = (tile % prm.n_ttiles) * BN;
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
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
    }
}


// =====================================================================================
// 2-SM variant (cta_group::2).  A cluster of two CTAs on neighbouring SMs computes
// 256-row x n-token pieces of Y^T ("chunks", n <= BN, n a multiple of 16): CTA
// rank q stages rows 128q..128q+127 of the S tile (values and metadata) and
// tokens q*n/2..q*n/2+n/2-1 of the chunk's X rows.  The leader (rank 0) issues
// every tcgen05.cp / tcgen05.mma for the pair; each operand descriptor names the
// same shared-memory offset in both CTAs.  Per 128-K stage each SM moves 16 KB
// of S, 2 KB of metadata and n/2*256 B of X for an M=256 MMA: half the operand
// bytes per MMA cycle of a 1-SM tile.
//
// Work partition (a data-parallel phase, then a balanced tail): the output is
// cut into 256-row tiles and each tile's tokens into 16-token units; a row's
// units form `ttiles` token tiles of near-equal width (<= BN tokens).
//  * Cyclic phase: for `cyc` rounds, round j deals tiles j*P .. j*P+P-1
//    (row-tile major) to the P pairs, rotated by j so that no pair always gets
//    the same token column.  The pairs of one round share a few S row tiles
//    and all of X, so both stay in L2 and S is read from HBM about once.
//  * Tail: the remaining units (between one and two rounds of tiles), in
//    row-tile-major order, are split into contiguous ranges, one per pair,
//    sized on the host so that every pair ends with the same number of
//    units.  A range is cut into chunks of at most BN/16 units that do not
//    cross a row tile (a segment is split into near-equal chunks); even pairs
//    walk their range forwards and odd pairs backwards, so the two pairs that
//    share a row tile at a range boundary read it at about the same time.
// Against whole tiles dealt out in rounds this removes the idle pairs of the
// last round (448 tiles of 256 x 256 on 74 pairs is 7 rounds for 6.05 rounds
// of work on the Llama-3-8B gate/up layer at M = 2048).  X rows are loaded in
// boxes of 64/32/16/8 rows (or one box of BN/2 rows for a full chunk), so a
// narrow chunk moves only its own tokens.
//
// Warps: 0 TMA producer, 1 MMA issue (leader only), 2..5 epilogue, 6 metadata.
// Operand stages: both CTAs' TMA loads of a stage (S values and X, or U and
// T) complete on the LEADER's full[s] barrier (cp.async.bulk.tensor with
// .cta_group::2, no multicast), so the MMA warp learns from one barrier that
// the pair's stage has landed.  Metadata takes a separate, deeper ring: the
// metadata warp of each CTA loads the tile MLEAD sparse stages ahead, permutes
// it into the TMEM layout and signals the leader's mready[m] (the leader with
// an arrive that expects 16 transaction bytes, the follower with a 16-byte
// bulk copy into the leader that completes them), so the permute is off the
// path from a stage's arrival to its MMAs.  The producer and MMA warps walk
// their loops with the whole warp (every branch warp-uniform) and one elected
// lane issues.
//
// Accumulators: two TMEM buffers of BN columns (2*BN + 4 <= 512 columns; the
// metadata takes 4 columns after them), so the epilogue of one chunk overlaps
// the MMAs of the next.
//
// Handshakes (all waits bounded):
//   full[s]      leader: its producer's arrive (both CTAs' bytes) + TMA bytes
//   empty[s]     leader's commit, multicast to both CTAs
//   mfull[m]     local metadata TMA completion (each CTA)
//   mready[m]    leader: its metadata warp (count 1) + follower's 16 bytes
//   mempty[m]    leader's commit after the MMAs that read slot m, multicast
//   acc_full[b]  leader's commit, multicast
//   acc_empty[b] 8 epilogue warps (both CTAs) -> leader: buffer drained
template <int BN>
struct Cfg2 {
    static constexpr int HALF_N = BN / 2;               // most tokens staged per CTA
    static constexpr int CHU = BN / 16;                 // most 16-token units per chunk
    static constexpr int A_BYTES = BM * 64 * 2;         // 16 KB of packed values
    static constexpr int B_HALF = HALF_N * 64 * 2;      // one 128-byte-wide panel of this CTA's tokens
    static constexpr int B_BYTES = 2 * B_HALF;
    static constexpr int E_BYTES = BM * BK / 8;         // 2 KB of metadata
    static constexpr int STAGE = ((A_BYTES + B_BYTES + 1023) / 1024) * 1024;
    static constexpr int MS = 8;                        // metadata slots
    static constexpr int MLEAD = 4;                     // metadata loads ahead of use (even: per-warp parity)
    static constexpr int PF = 12;                       // S tiles prefetched into L2 this many stages ahead
    static constexpr uint32_t TMEM_COLS = 512;
    // Two accumulators when they fit beside the metadata (the epilogue of one
    // chunk then overlaps the MMAs of the next), else one (BN = 256).
    static constexpr int NACC = (2 * BN + 4 <= 512) ? 2 : 1;
    static constexpr uint32_t ACC1 = BN;                // column of accumulator 1
    static constexpr uint32_t ECOL = NACC * BN;         // metadata columns
    static constexpr int OUT_COLS = 32;
    static constexpr int OUT_BYTES = OUT_COLS * BM * 2; // one 32-token piece of this CTA's rows
    static constexpr int FIXED1 = MS * E_BYTES + 1024 + 16 * MS + 16;
    static constexpr int AVAIL = 232448 - 1024 - FIXED1;
    // Two output staging buffers unless dropping one buys another stage.
    static constexpr int NOUT = ((AVAIL - 2 * OUT_BYTES) / STAGE < (AVAIL - OUT_BYTES) / STAGE) ? 1 : 2;
    static constexpr int NS_FIT = (AVAIL - NOUT * OUT_BYTES) / STAGE;
    static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
    static constexpr int RING = NS * STAGE;
    static constexpr int META_OFF = RING;
    static constexpr int OUT_OFF = META_OFF + MS * E_BYTES;
    static constexpr int BAR_OFF = OUT_OFF + NOUT * OUT_BYTES;
    static constexpr int DUMMY_OFF = BAR_OFF + 1024;    // 16-byte signal slots, one per metadata slot
    static constexpr int SMEM = DUMMY_OFF + 16 * MS + 16 + 1024;
    static_assert(BN % 16 == 0 && BN <= 256, "chunk width");
    static_assert(B_HALF % 1024 == 0, "SW128 panels start on 1 KB");
    static_assert(NS >= 2, "need at least two stages");
    static_assert(MLEAD < MS && MLEAD % 2 == 0 && MS % 2 == 0, "metadata lead");
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(ECOL + 4 <= TMEM_COLS, "TMEM budget");
    static_assert((2 * NS + 3 * MS + 4) * 8 + 8 <= 1024, "barrier area");
};

// Tensor maps of the 2-SM kernel.  xs[i] loads box_rows(i) rows of X for both
// 64-element K panels of a stage in one copy (a 3-D view of X: element, row,
// panel), landing as panel 0's rows then panel 1's rows; ts[i] loads
// box_rows(i) rows of T (one panel).  A chunk uses the smallest box that holds
// its rows; rows past the chunk are loaded but not read by the MMA.  Boxes of
// 8, 16, 32 and 64 rows, then `b4` and b4 + 8 rows (the rows of the plan's two
// widths of whole token tiles, so that neither loads padding) and the
// kernel's most (half_n).
struct Maps2 {
    CUtensorMap vals, meta, u, y32, y16;
    CUtensorMap xs[7];
    CUtensorMap ts[7];
    CUtensorMap xt, vt;   // projection phase: X in 128-row boxes, V in RN/2-row boxes (two 64-wide panels)
};

__host__ __device__ constexpr int box_rows(int i, int half_n, int b4) {
    return i < 4 ? (8 << i) : i == 4 ? b4 : i == 5 ? (b4 + 8 < half_n ? b4 + 8 : half_n) : half_n;
}
__host__ __device__ constexpr int pick_box(int rows, int b4) {
    return rows <= 8 ? 0 : rows <= 16 ? 1 : rows <= 32 ? 2 : rows <= 64 ? 3 : rows <= b4 ? 4 : rows <= b4 + 8 ? 5 : 6;
}

constexpr int kMaxPairs = 128;

struct Params2 {
    int32_t M;          // tokens
    int32_t d_out;      // output rows
    int32_t tile_rows;  // output rows per pair tile (256 or 512)
    int32_t nk, nlr;    // K stages, rank stages
    int32_t ut;         // 16-token units per row tile
    int32_t ttiles;     // token tiles per row tile
    int32_t wu, wr;     // token tile tt has wu + (tt < wr) units
    int32_t cyc;        // rounds of the cyclic phase
    int32_t chu;        // most 16-token units per chunk (<= the kernel's BN / 16)
    int32_t box4;       // rows of X box 4: those of the narrower whole token tiles (8 * wu, 64..8 * chu); box 5: 8 more
    int64_t n_tiles;    // tiles dealt in the cyclic phase (a last round may be partial)
    const uint8_t *meta;  // packed metadata [d_out, meta_ld] (copied with cp.async by the 512-row kernel)
    int64_t meta_ld;      // bytes per metadata row (d_in / 8)
    // Projection phase of the 512-row kernel (tp_on): T = X V^T for 256-token
    // tiles, K split tp_ks ways over the first tp_tiles * tp_ks pairs, partial
    // sums in tp_part, reduced by every CTA into T16; tp_count[0] counts the
    // CTAs whose partials are written, tp_count[1] those whose share of T16 is.
    int32_t tp_on, tp_tiles, tp_ks, tp_rn, r;
    float *tp_part;       // [tp_tiles * tp_ks][256][tp_rn] fp32
    uint16_t *tp_t16;     // T [M, r] bf16
    unsigned int *tp_count;
    // K-split last round (ksplit, 512-row kernel): tail[p] = tile << 16 |
    // q << 8 | g when pair p runs K slice q of g of that tile (-1: no tail
    // work); each slice's fp32 partial tile goes to ks_part slot p, and
    // ks_count[i] counts the CTAs whose partial of tail tile i is written.
    int32_t ksplit;
    float *ks_part;       // [pairs][2 CTAs][2 halves][240 / 4 token blocks][128 rows][4] fp32
    unsigned int *ks_count;
    uint16_t *y;          // Y [M, d_out]: the reduction of a K-split tile stores it directly
    // Token-split or whole tail: pair p's tail units are [tail[p], tail[p+1]).
    int64_t tail[kMaxPairs + 1];
};

struct Chunk {
    int32_t d0;         // first output row of the pair's 256-row tile
    int32_t tok0;       // first token
    int32_t n;          // tokens (multiple of 16)
    int32_t k0, k1;     // sparse K stages [k0, k1) of the chunk
    int32_t lr;         // the rank stages follow the sparse ones
    int32_t part;       // a K slice of a tail tile: partial sums, then a share of the reduction
};

// The chunk sequence of one pair; every warp role of the pair walks the same
// sequence.  All partition parameters are copied into registers when the
// iterator is built, so the loops never read the kernel parameters again.
struct ChunkIter {
    int32_t j, cyc, ut, ttiles, wu, wr, pair, npairs, tile_rows, nk, ksplit;
    int64_t n_tiles, lo, hi;

    __host__ __device__ __forceinline__ ChunkIter(const Params2 &prm, int pair_, int npairs_)
        : j(0), cyc(prm.cyc), ut(prm.ut), ttiles(prm.ttiles), wu(prm.wu), wr(prm.wr), pair(pair_), npairs(npairs_),
          tile_rows(prm.tile_rows), nk(prm.nk), ksplit(prm.ksplit), n_tiles(prm.n_tiles), lo(prm.tail[pair_]),
          hi(prm.ksplit ? 0 : prm.tail[pair_ + 1]) {}

    __host__ __device__ __forceinline__ void whole_tile(int64_t tile, Chunk &c) const {
        const int64_t rt = tile / ttiles;
        const int32_t tt = (int32_t)(tile - rt * ttiles);
        const int32_t u0 = tt * wu + (tt < wr ? tt : wr);
        c.d0 = (int32_t)(rt * tile_rows);
        c.tok0 = u0 * 16;
        c.n = (wu + (tt < wr ? 1 : 0)) * 16;
        c.k0 = 0;
        c.k1 = nk;
        c.lr = 1;
        c.part = 0;
    }

    __host__ __device__ __forceinline__ bool next(int32_t chu, Chunk &c) {
        const int64_t tile = (int64_t)j * npairs + (pair + j) % npairs;
        if (j < cyc && tile < n_tiles) {
            whole_tile(tile, c);
            ++j;
            return true;
        }
        if (ksplit) {
            // One K slice of one tail tile (the slices of a tile together
            // cover its K stages once; slice 0 also runs the rank stages).
            if (lo < 0) return false;
            const int64_t t = lo >> 16;
            const int32_t q = (int32_t)((lo >> 8) & 255), g = (int32_t)(lo & 255);
            whole_tile(t, c);
            c.k0 = (int32_t)(((int64_t)nk * q) / g);
            c.k1 = (int32_t)(((int64_t)nk * (q + 1)) / g);
            c.lr = q == 0;
            c.part = g > 1;
            lo = -1;
            return true;
        }
        if (lo >= hi) return false;
        if ((pair & 1) == 0) {
            const int64_t rt = lo / ut;
            const int32_t ui = (int32_t)(lo - rt * ut);
            const int64_t left = hi - lo, to_end = ut - ui;
            const int32_t seg = (int32_t)(left < to_end ? left : to_end);
            const int32_t pieces = (seg + chu - 1) / chu;
            const int32_t nu = (seg + pieces - 1) / pieces;
            c.d0 = (int32_t)(rt * tile_rows);
            c.tok0 = ui * 16;
            c.n = nu * 16;
            lo += nu;
            c.k0 = 0;
            c.k1 = nk;
            c.lr = 1;
            c.part = 0;
        } else {
            const int64_t rt = (hi - 1) / ut;
            const int64_t start = rt * ut;
            const int64_t left = hi - lo, to_start = hi - start;
            const int32_t seg = (int32_t)(left < to_start ? left : to_start);
            const int32_t pieces = (seg + chu - 1) / chu;
            const int32_t nu = (seg + pieces - 1) / pieces;
            c.d0 = (int32_t)(rt * tile_rows);
            c.tok0 = (int32_t)(hi - nu - start) * 16;
            c.n = nu * 16;
            hi -= nu;
            c.k0 = 0;
            c.k1 = nk;
            c.lr = 1;
            c.part = 0;
        }
        return true;
    }
};

// Cursor over a pair's sparse stages (chunk by chunk, stages [k0, k1) each),
// for the metadata warp.
struct SparseCursor {
    ChunkIter iter;
    Chunk ch;
    int32_t ks;
    bool valid;

    __device__ __forceinline__ SparseCursor(const Params2 &prm, int pair, int npairs, int32_t chu)
        : iter(prm, pair, npairs), ks(0) {
        valid = iter.next(chu, ch);
        if (valid) ks = ch.k0;
    }
    __device__ __forceinline__ void advance(int32_t chu) {
        if (++ks == ch.k1) {
            valid = iter.next(chu, ch);
            if (valid) ks = ch.k0;
        }
    }
};

constexpr int kThreads2 = 256;  // 8 warps

template <int BN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads2, 1)
    tc2_forward_kernel(const __grid_constant__ Maps2 maps, const __grid_constant__ Params2 prm) {
    using C = Cfg2<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *empty = full + C::NS;
    uint64_t *mfull = empty + C::NS;
    uint64_t *mready = mfull + C::MS;
    uint64_t *mempty = mready + C::MS;
    uint64_t *acc_full = mempty + C::MS;
    uint64_t *acc_empty = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
    volatile uint32_t *fail = tmem_slot + 1;
    uint8_t *meta_ring = smem + C::META_OFF;
    uint8_t *dummy = smem + C::DUMMY_OFF;   // MS signal slots + 1 source slot

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int nk = prm.nk;
    const int nstages = nk + prm.nlr;
    const int M = prm.M;
    const int d_out = prm.d_out;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int m = 0; m < C::MS; ++m) {
            mbar_init(&mfull[m], 1);
            mbar_init(&mready[m], 1);
            mbar_init(&mempty[m], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);
        }
        *fail = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.vals)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.meta)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.xs[4])) : "memory");
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (each CTA)
        const uint32_t full_leader0 = mapa_shared(smem_u32(&full[0]), 0);
        uint32_t s = 0, ph = 0;
        bool t_ready = false;
        ChunkIter iter(prm, pair, npairs);
        Chunk ch;
        while (!__any_sync(0xFFFFFFFFu, *fail != 0) && iter.next(prm.chu, ch)) {
            const int d0 = ch.d0 + (int)rank * BM;
            const int rows = ch.n / 2;
            const int tok = ch.tok0 + (int)rank * rows;
            const int bi = pick_box(rows, prm.box4);
            const uint32_t brows = (uint32_t)box_rows(bi, C::HALF_N, prm.box4);
            const CUtensorMap *xmap = &maps.xs[bi];
            const CUtensorMap *tmap = &maps.ts[bi];
            for (int ks = 0; ks < nstages; ++ks) {
                if (!__all_sync(0xFFFFFFFFu, mbar_wait_cluster(&empty[s], ph ^ 1))) {
                    if (lane == 0) {
                        *fail = 1;
                        atomicOr(&g_tc_error, 16u);
                    }
                    break;
                }
                uint8_t *st = smem + s * C::STAGE;
                const uint32_t a = smem_u32(st), b = smem_u32(st + C::A_BYTES);
                const uint32_t bar = full_leader0 + s * (uint32_t)sizeof(uint64_t);
                if (ks < nk) {
                    if (elect_one()) {
                        if (leader) mbar_expect_tx(&full[s], 2u * (C::A_BYTES + brows * 256u));
                        tma_load_2d_pair(&maps.vals, a, bar, ks * 64, d0);
                        tma_load_3d_pair(xmap, b, bar, 0, tok, ks * 2);
                        // Bring the S tile of a later stage into L2 now, so that
                        // its load does not wait on HBM.
                        if (ks + C::PF < nk) {
                            tma_prefetch_2d(&maps.vals, (ks + C::PF) * 64, d0);
                            tma_prefetch_2d(&maps.meta, (ks + C::PF) * (BK / 8), d0);
                        }
                    }
                } else {
                    const int j = ks - nk;
                    if (!t_ready) {
                        // T comes from the projection kernel, which may still
                        // be running (programmatic dependent launch).
                        asm volatile("griddepcontrol.wait;" ::: "memory");
                        t_ready = true;
                    }
                    if (elect_one()) {
                        if (leader) mbar_expect_tx(&full[s], 2u * (C::A_BYTES + brows * 128u));
                        tma_load_2d_pair(&maps.u, a, bar, j * 64, d0);
                        tma_load_2d_pair(tmap, b, bar, j * 64, tok);
                    }
                }
                __syncwarp();
                if (++s == (uint32_t)C::NS) {
                    s = 0;
                    ph ^= 1;
                }
            }
        }
    } else if (warp >= 6) {
        // ------------------------------------------------------------ metadata warps (each CTA)
        // Warp 6 takes the even sparse stages, warp 7 the odd ones; each loads
        // its tiles MLEAD stages ahead into slots of its own parity.
        const int par = warp - 6;
        const uint32_t src_slot = smem_u32(dummy + 16 * C::MS);
        SparseCursor ld(prm, pair, npairs, prm.chu), use(prm, pair, npairs, prm.chu);
        if (par) {
            ld.advance(prm.chu);
            use.advance(prm.chu);
        }
        auto issue = [&](int slot) {
            if (elect_one()) {
                mbar_expect_tx(&mfull[slot], C::E_BYTES);
                tma_load_2d(&maps.meta, smem_u32(meta_ring + slot * C::E_BYTES), &mfull[slot], ld.ks * (BK / 8),
                            ld.ch.d0 + (int)rank * BM);
            }
            __syncwarp();
            ld.advance(prm.chu);
            if (ld.valid) ld.advance(prm.chu);
        };
        int64_t n_ld = par;
        for (; n_ld < C::MLEAD && ld.valid; n_ld += 2) issue((int)(n_ld % C::MS));
        int64_t k = par;
        while (use.valid && !__any_sync(0xFFFFFFFFu, *fail != 0)) {
            const int slot = (int)(k % C::MS);
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&mfull[slot], (uint32_t)((k / C::MS) & 1)))) {
                if (lane == 0) {
                    *fail = 1;
                    atomicOr(&g_tc_error, 256u);
                }
                break;
            }
            // Zero-filled rows past d_out carry (0,0) index pairs; only tiles
            // that reach past d_out need them rewritten.
            if (use.ch.d0 + (int)rank * BM + BM > d_out)
                permute_meta_tile<true>(meta_ring + slot * C::E_BYTES, lane);
            else
                permute_meta_tile<false>(meta_ring + slot * C::E_BYTES, lane);
            fence_proxy_async_smem();
            __syncwarp();
            if (elect_one()) {
                if (leader) {
                    mbar_expect_tx(&mready[slot], 16);
                } else {
                    bulk_signal_peer(mapa_shared(smem_u32(dummy + 16 * slot), 0), src_slot + 0,
                                     mapa_shared(smem_u32(&mready[slot]), 0));
                }
            }
            __syncwarp();
            if (ld.valid) {
                // The slot of stage n_ld last held stage n_ld - MS; the MMAs
                // that read it must be done before it is refilled.
                const int s2 = (int)(n_ld % C::MS);
                if (n_ld >= C::MS &&
                    !__all_sync(0xFFFFFFFFu,
                                mbar_wait_cluster(&mempty[s2], (uint32_t)(((n_ld - C::MS) / C::MS) & 1)))) {
                    if (lane == 0) {
                        *fail = 1;
                        atomicOr(&g_tc_error, 512u);
                    }
                    break;
                }
                issue(s2);
                n_ld += 2;
            }
            use.advance(prm.chu);
            if (use.valid) use.advance(prm.chu);
            k += 2;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue (leader CTA)
        if (leader) {
            const uint32_t e_tmem = tmem_base + C::ECOL;
            uint32_t s = 0, ph = 0;
            int it = 0;
            int64_t k = 0;   // sparse stages consumed (metadata slot sequence)
            ChunkIter iter(prm, pair, npairs);
            Chunk ch;
            while (!__any_sync(0xFFFFFFFFu, *fail != 0) && iter.next(prm.chu, ch)) {
                const uint32_t idesc_sp = idesc_bf16(2 * BM, ch.n, true);
                const uint32_t idesc_dense = idesc_bf16(2 * BM, ch.n, false);
                const uint32_t panel = (uint32_t)box_rows(pick_box(ch.n / 2, prm.box4), C::HALF_N, prm.box4) * 128u;
                const int buf = C::NACC == 2 ? (it & 1) : 0;
                const uint32_t use = (uint32_t)(C::NACC == 2 ? (it >> 1) : it);
                bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_cluster(&acc_empty[buf], (use & 1) ^ 1));
                if (!ok) {
                    if (lane == 0) {
                        *fail = 1;
                        atomicOr(&g_tc_error, 32u);
                    }
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (buf ? C::ACC1 : 0u);
                for (int ks = 0; ks < nstages; ++ks) {
                    const bool sparse = ks < nk;
                    const int m = (int)(k % C::MS);
                    bool got = mbar_wait_cluster(&full[s], ph);
                    if (got && sparse) got = mbar_wait_cluster(&mready[m], (uint32_t)((k / C::MS) & 1));
                    if (!__all_sync(0xFFFFFFFFu, got)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t *st = smem + s * C::STAGE;
                    const uint32_t a = smem_u32(st), b = smem_u32(st + C::A_BYTES);
                    if (elect_one()) {
                        if (sparse) {
                            tmem_cp_pair_128x128b(e_tmem,
                                                  smem_desc(smem_u32(meta_ring + m * C::E_BYTES), 0, 128, kLayoutNone));
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const uint64_t adesc = desc_sw128(a + 32 * c);
                                const uint64_t bdesc = desc_sw128(b + (c >> 1) * panel + (c & 1) * 64);
                                mma_sp_pair(d_tmem, adesc, bdesc, e_tmem + (uint32_t)(c & 2),
                                            idesc_sp | (uint32_t)(c & 1), (ks | c) != 0);
                            }
                            mma_commit_pair(&mempty[m]);
                        } else {
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                mma_dense_pair(d_tmem, desc_sw128(a + 32 * c), desc_sw128(b + 32 * c), idesc_dense, 1u);
                        }
                        mma_commit_pair(&empty[s]);
                    }
                    __syncwarp();
                    if (sparse) ++k;
                    if (++s == (uint32_t)C::NS) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (!ok) {
                    if (lane == 0) {
                        *fail = 1;
                        atomicOr(&g_tc_error, 64u);
                    }
                    break;
                }
                if (elect_one()) mma_commit_pair(&acc_full[buf]);
                __syncwarp();
                ++it;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (each CTA, its 128 rows)
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const bool store_thread = (warp == 2 && lane == 0);
        uint8_t *stage_out = smem + C::OUT_OFF;
        const uint32_t empty_leader0 = mapa_shared(smem_u32(&acc_empty[0]), 0);
        uint32_t piece = 0;
        int it = 0;
        ChunkIter iter(prm, pair, npairs);
        Chunk ch;
        while (!*fail && iter.next(prm.chu, ch)) {
            const int d0 = ch.d0 + (int)rank * BM;
            const int buf = C::NACC == 2 ? (it & 1) : 0;
            const uint32_t use = (uint32_t)(C::NACC == 2 ? (it >> 1) : it);
            if (!mbar_wait_cluster(&acc_full[buf], use & 1)) {
                *fail = 1;
                atomicOr(&g_tc_error, 128u);
                break;
            }
            tc_fence_after();
            const uint32_t acc = tmem_base + ((uint32_t)(quarter * 32) << 16) + (buf ? C::ACC1 : 0u);
            const int nq = (ch.n + 31) / 32;
#pragma unroll 1
            for (int q = 0; q < nq; ++q) {
                const bool wide = ch.n - q * 32 >= 32;   // else a 16-token piece
                uint32_t v[32];
                if (wide) {
                    tmem_ld_32x32b_x32(acc + (uint32_t)(q * 32), v);
                } else {
                    uint32_t h[16];
                    tmem_ld_32x32b_x16(acc + (uint32_t)(q * 32), h);
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] = h[j];
                }
                if (q == nq - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote_relaxed(empty_leader0 + (uint32_t)(buf * sizeof(uint64_t)));
                }
                const int tq = ch.tok0 + q * C::OUT_COLS;
                if (tq >= M) continue;  // uniform across the epilogue warps
                const uint32_t sb = C::NOUT == 2 ? (piece & 1) : 0u;
                if (store_thread) {
                    if (C::NOUT == 2)
                        bulk_wait_read1();
                    else
                        bulk_wait_read0();
                }
                named_bar_sync(1, 128);
                uint16_t *out = reinterpret_cast<uint16_t *>(stage_out + sb * C::OUT_BYTES);
                if (wide) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) out[j * BM + row] = f32_to_bf16_bits(__uint_as_float(v[j]));
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) out[j * BM + row] = f32_to_bf16_bits(__uint_as_float(v[j]));
                }
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (store_thread) {
                    tma_store_2d(wide ? &maps.y32 : &maps.y16, smem_u32(out), d0, tq);
                    bulk_commit();
                }
                ++piece;
            }
            ++it;
        }
        if (store_thread) bulk_wait_all();
    }

    tc_fence_before();
    cluster_sync_all();  // the pair's MMAs, signals and stores are done before TMEM is freed
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
    }
}

// =====================================================================================
// Tall 2-SM variant for large M: a pair computes 512 output rows (two 256-row
// halves, each one M=256 cta_group::2 MMA) x n tokens, and both halves read
// the same staged X tile.  Against 256-row pair tiles this halves the number
// of times X crosses from L2 into shared memory (the kernel is bound by that
// traffic: with 256 x 192 tiles on the Llama-3-8B gate/up layer, X is read
// once per 256-row tile, 56 times in all).  CTA rank q stages rows
// 256h + 128q .. +127 of half h of the S tile and tokens q*n/2 .. of X.
//
// TMEM: accumulator h at columns h*BN (2*BN + 8 <= 512, no double
// buffering), metadata of half h at 2*BN + 4h.  The epilogue (8 warps, four
// per half) drains both accumulators after a chunk's last stage; the next
// chunk's MMAs wait for that drain.  Everything else follows the 256-row
// kernel: stage loads of both CTAs complete on the leader's full[s], the
// metadata ring (4 KB per stage: both halves) is loaded MLEAD stages ahead
// and permuted by two warps (even / odd stages), and the producer and MMA
// warps run converged with one elected lane issuing.
template <int BN>
struct CfgT {
    static constexpr int HALF_N = BN / 2;               // most tokens staged per CTA
    static constexpr int CHU = BN / 16;                 // most 16-token units per chunk
    static constexpr int A_BYTES = BM * 64 * 2;         // 16 KB of packed values per half
    static constexpr int B_HALF = HALF_N * 64 * 2;      // one 128-byte-wide panel of this CTA's tokens
    static constexpr int B_BYTES = 2 * B_HALF;
    static constexpr int B_OFF = 2 * A_BYTES;
    static constexpr int E_BYTES = BM * BK / 8;         // 2 KB of metadata per half
    static constexpr int STAGE = ((2 * A_BYTES + B_BYTES + 1023) / 1024) * 1024;
    static constexpr int MS = 5;                        // metadata slots (both halves each)
    static constexpr int MLEAD = 2;                     // metadata loads ahead of use (even: per-warp parity)
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t ECOL = 2 * BN;            // metadata columns (4 per half)
    static constexpr int OUT_COLS = 32;
    static constexpr int OUT_BYTES = OUT_COLS * BM * 2; // one 32-token piece of one half's rows
    static constexpr int FIXED = MS * 2 * E_BYTES + 2 * OUT_BYTES + 1024 + 16 * MS + 16;
    static constexpr int NS_FIT = (232448 - 1024 - FIXED) / STAGE;
    static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
    static constexpr int RING = NS * STAGE;
    static constexpr int META_OFF = RING;
    static constexpr int OUT_OFF = META_OFF + MS * 2 * E_BYTES;
    static constexpr int BAR_OFF = OUT_OFF + 2 * OUT_BYTES;
    static constexpr int DUMMY_OFF = BAR_OFF + 1024;
    static constexpr int SMEM = DUMMY_OFF + 16 * MS + 16 + 1024;
    static_assert(BN % 16 == 0 && 2 * BN + 8 <= 512, "TMEM budget");
    static_assert(B_HALF % 1024 == 0, "SW128 panels start on 1 KB");
    static_assert(NS >= 2, "need at least two stages");
    static_assert(MLEAD < MS && MLEAD % 2 == 0, "metadata lead");
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert((2 * NS + 3 * MS + 6) * 8 + 8 <= 1024, "barrier area");
};

constexpr int kThreadsT = 384;  // 12 warps
static_assert(kKsSlotFloats == 4 * 240 * BM, "K-split slot: 2 CTAs x 2 halves x 240 tokens x 128 rows");
static_assert(kMaxPairs == 128, "fused_pairs_for caps the pairs at 128");

// Bounded spin until *p >= target (acquire, GPU scope); false on expiry.
__device__ __forceinline__ bool spin_count_ge(const unsigned int *p, unsigned int target) {
    const long long t0 = clock64();
    while (true) {
        unsigned int v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
        if (v >= target) return true;
        if (clock64() - t0 > kWaitCycles) return false;
        __nanosleep(64);
    }
}

template <int BN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsT, 1)
    tc2t_forward_kernel(const __grid_constant__ Maps2 maps, const __grid_constant__ Params2 prm) {
    using C = CfgT<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *empty = full + C::NS;
    uint64_t *mfull = empty + C::NS;
    uint64_t *mready = mfull + C::MS;
    uint64_t *mempty = mready + C::MS;
    uint64_t *acc_full = mempty + C::MS;
    uint64_t *acc_empty = acc_full + 1;
    uint64_t *tp_full = acc_empty + 1;    // projection phase: T partial complete in TMEM
    uint64_t *tp_empty = tp_full + 1;     // projection phase: T partial drained (leader)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tp_empty + 1);
    volatile uint32_t *fail = tmem_slot + 1;
    uint8_t *meta_ring = smem + C::META_OFF;
    uint8_t *dummy = smem + C::DUMMY_OFF;   // MS signal slots + 1 source slot

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int nk = prm.nk;
    const int M = prm.M;
    const int d_out = prm.d_out;
    // Projection phase (T = X V^T inside this kernel, LoSparse section 3.2's
    // low-rank term): pair p < tp_tiles * tp_ks computes the partial product
    // of token tile p / tp_ks over the p % tp_ks-th slice of the K stages.
    const bool tp_busy = prm.tp_on && pair < prm.tp_tiles * prm.tp_ks;
    const int tp_tile = tp_busy ? pair / prm.tp_ks : 0, tp_q = tp_busy ? pair % prm.tp_ks : 0;
    const int tp_k0 = tp_busy ? (int)(((int64_t)nk * tp_q) / prm.tp_ks) : 0;
    const int tp_k1 = tp_busy ? (int)(((int64_t)nk * (tp_q + 1)) / prm.tp_ks) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int m = 0; m < C::MS; ++m) {
            mbar_init(&mfull[m], 32);   // one cp.async arrival per lane of the metadata warp
            mbar_init(&mready[m], 1);
            mbar_init(&mempty[m], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 16);
        mbar_init(tp_full, 1);
        mbar_init(tp_empty, 8);
        *fail = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.vals)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.meta)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.xs[4])) : "memory");
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (each CTA)
        const uint32_t full_leader0 = mapa_shared(smem_u32(&full[0]), 0);
        uint32_t s = 0, ph = 0;
        bool t_ready = false;
        // Projection phase: per stage, this CTA's 128 tokens of X (two
        // 128-byte panels, 32 KB) and its tp_rn / 2 rows of V through the
        // same ring as the main loop.
        for (int ks = tp_k0; ks < tp_k1; ++ks) {
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_cluster(&empty[s], ph ^ 1))) {
                if (lane == 0) {
                    *fail = 1;
                    atomicOr(&g_tc_error, 65536u);
                }
                break;
            }
            uint8_t *st = smem + s * C::STAGE;
            const uint32_t a = smem_u32(st), b = smem_u32(st + C::B_OFF);
            const uint32_t bar = full_leader0 + s * (uint32_t)sizeof(uint64_t);
            if (elect_one()) {
                if (leader) mbar_expect_tx(&full[s], 2u * (32768u + (uint32_t)prm.tp_rn * 128u));
                tma_load_3d_pair(&maps.xt, a, bar, 0, tp_tile * 256 + (int)rank * 128, ks * 2);
                tma_load_3d_pair(&maps.vt, b, bar, 0, (int)rank * (prm.tp_rn / 2), ks * 2);
            }
            __syncwarp();
            if (++s == (uint32_t)C::NS) {
                s = 0;
                ph ^= 1;
            }
        }
        ChunkIter iter(prm, pair, npairs);
        Chunk ch;
        while (!__any_sync(0xFFFFFFFFu, *fail != 0) && iter.next(prm.chu, ch)) {
            const int d0 = ch.d0 + (int)rank * BM;        // half 0 rows of this CTA; half 1 at +256
            const int rows = ch.n / 2;
            const int tok = ch.tok0 + (int)rank * rows;
            const int bi = pick_box(rows, prm.box4);
            const uint32_t brows = (uint32_t)box_rows(bi, C::HALF_N, prm.box4);
            const CUtensorMap *xmap = &maps.xs[bi];
            const CUtensorMap *tmap = &maps.ts[bi];
            const int nsp = ch.k1 - ch.k0;
            const int nst = nsp + (ch.lr ? prm.nlr : 0);
            for (int i = 0; i < nst; ++i) {
                if (!__all_sync(0xFFFFFFFFu, mbar_wait_cluster(&empty[s], ph ^ 1))) {
                    if (lane == 0) {
                        *fail = 1;
                        atomicOr(&g_tc_error, 16u);
                    }
                    break;
                }
                uint8_t *st = smem + s * C::STAGE;
                const uint32_t a = smem_u32(st), b = smem_u32(st + C::B_OFF);
                const uint32_t bar = full_leader0 + s * (uint32_t)sizeof(uint64_t);
                if (i < nsp) {
                    const int ks = ch.k0 + i;
                    if (elect_one()) {
                        if (leader) mbar_expect_tx(&full[s], 2u * (2u * C::A_BYTES + brows * 256u));
                        tma_load_2d_pair(&maps.vals, a, bar, ks * 64, d0);
                        tma_load_2d_pair(&maps.vals, a + C::A_BYTES, bar, ks * 64, d0 + 2 * BM);
                        tma_load_3d_pair(xmap, b, bar, 0, tok, ks * 2);
                    }
                } else {
                    const int j = i - nsp;
                    if (!t_ready) {
                        if (prm.tp_on) {
                            // T comes from this grid's projection phase: every
                            // CTA has written its share of T16 (global writes,
                            // then read here through the async proxy).
                            if (!__all_sync(0xFFFFFFFFu, spin_count_ge(prm.tp_count + 1, gridDim.x))) {
                                if (lane == 0) {
                                    *fail = 1;
                                    atomicOr(&g_tc_error, 131072u);
                                }
                                break;
                            }
                            asm volatile("fence.proxy.async.global;" ::: "memory");
                        } else {
                            // T comes from the projection kernel, which may
                            // still be running (programmatic dependent launch).
                            asm volatile("griddepcontrol.wait;" ::: "memory");
                        }
                        t_ready = true;
                    }
                    if (elect_one()) {
                        if (leader) mbar_expect_tx(&full[s], 2u * (2u * C::A_BYTES + brows * 128u));
                        tma_load_2d_pair(&maps.u, a, bar, j * 64, d0);
                        tma_load_2d_pair(&maps.u, a + C::A_BYTES, bar, j * 64, d0 + 2 * BM);
                        tma_load_2d_pair(tmap, b, bar, j * 64, tok);
                    }
                }
                __syncwarp();
                if (++s == (uint32_t)C::NS) {
                    s = 0;
                    ph ^= 1;
                }
            }
        }
    } else if (warp >= 10) {
        // ------------------------------------------------------------ metadata warps (each CTA)
        // Warp 10 takes the even sparse stages, warp 11 the odd ones; a slot
        // holds both halves' tiles (2 x 2 KB).
        const int par = warp - 10;
        const uint32_t src_slot = smem_u32(dummy + 16 * C::MS);
        SparseCursor ld(prm, pair, npairs, prm.chu), use(prm, pair, npairs, prm.chu);
        if (par) {
            ld.advance(prm.chu);
            use.advance(prm.chu);
        }
        // A stage's metadata is 16 bytes per row: as TMA boxes it would cost
        // one copy request per row, as many as the 128-byte rows of the
        // values, on the SM's TMA engine.  The warp's lanes copy the 256 rows
        // (both halves) with 16-byte cp.async instead, eight per lane, and each
        // lane arrives on the slot's barrier when its copies have landed.
        // Rows past d_out are zero-filled, as TMA would.
        auto issue = [&](int slot) {
            uint8_t *e = meta_ring + slot * 2 * C::E_BYTES;
            const int r0 = ld.ch.d0 + (int)rank * BM;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int q = lane + 32 * i;            // 0..255: half q >> 7, row q & 127
                const int row = r0 + (q >> 7) * 2 * BM + (q & 127);
                const bool in = row < d_out;
                const uint8_t *src = prm.meta + (in ? (int64_t)row * prm.meta_ld + (int64_t)ld.ks * (BK / 8) : 0);
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                                 smem_u32(e + (q >> 7) * C::E_BYTES + (q & 127) * 16)),
                             "l"(src), "r"(in ? 16 : 0)
                             : "memory");
            }
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&mfull[slot])) : "memory");
            ld.advance(prm.chu);
            if (ld.valid) ld.advance(prm.chu);
        };
        int64_t n_ld = par;
        for (; n_ld < C::MLEAD && ld.valid; n_ld += 2) issue((int)(n_ld % C::MS));
        int64_t k = par;
        while (use.valid && !__any_sync(0xFFFFFFFFu, *fail != 0)) {
            const int slot = (int)(k % C::MS);
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&mfull[slot], (uint32_t)((k / C::MS) & 1)))) {
                if (lane == 0) {
                    *fail = 1;
                    atomicOr(&g_tc_error, 256u);
                }
                break;
            }
            uint8_t *e = meta_ring + slot * 2 * C::E_BYTES;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // Zero-filled rows past d_out carry (0,0) index pairs; only
                // tiles that reach past d_out need them rewritten.
                if (use.ch.d0 + h * 2 * BM + (int)rank * BM + BM > d_out)
                    permute_meta_tile<true>(e + h * C::E_BYTES, lane);
                else
                    permute_meta_tile<false>(e + h * C::E_BYTES, lane);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (elect_one()) {
                if (leader) {
                    mbar_expect_tx(&mready[slot], 16);
                } else {
                    bulk_signal_peer(mapa_shared(smem_u32(dummy + 16 * slot), 0), src_slot,
                                     mapa_shared(smem_u32(&mready[slot]), 0));
                }
            }
            __syncwarp();
            if (ld.valid) {
                // The slot of stage n_ld last held stage n_ld - MS; the MMAs
                // that read it must be done before it is refilled.
                const int s2 = (int)(n_ld % C::MS);
                if (n_ld >= C::MS &&
                    !__all_sync(0xFFFFFFFFu,
                                mbar_wait_cluster(&mempty[s2], (uint32_t)(((n_ld - C::MS) / C::MS) & 1)))) {
                    if (lane == 0) {
                        *fail = 1;
                        atomicOr(&g_tc_error, 512u);
                    }
                    break;
                }
                issue(s2);
                n_ld += 2;
            }
            use.advance(prm.chu);
            if (use.valid) use.advance(prm.chu);
            k += 2;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue (leader CTA)
        if (leader) {
            const uint32_t e_tmem = tmem_base + C::ECOL;
            uint32_t s = 0, ph = 0;
            int it = 0;
            int64_t k = 0;   // sparse stages consumed (metadata slot sequence)
            if (tp_busy) {
                // Projection phase: D = T partial (M = 256 tokens of the pair,
                // N = tp_rn ranks) in TMEM columns 0..tp_rn-1, dense MMAs with
                // A = the X tile and B = the V tile, K = 16 each.
                const uint32_t idesc_t = idesc_bf16(2 * BM, prm.tp_rn, false);
                const uint32_t vpanel = (uint32_t)prm.tp_rn * 64u;   // tp_rn / 2 rows of 128 bytes
                bool ok = true;
                for (int ks = tp_k0; ks < tp_k1; ++ks) {
                    if (!__all_sync(0xFFFFFFFFu, mbar_wait_cluster(&full[s], ph))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t *st = smem + s * C::STAGE;
                    const uint32_t a = smem_u32(st), b = smem_u32(st + C::B_OFF);
                    if (elect_one()) {
#pragma unroll
                        for (int pn = 0; pn < 2; ++pn)
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                mma_dense_pair(tmem_base, desc_sw128(a + pn * 16384 + 32 * c),
                                               desc_sw128(b + pn * vpanel + 32 * c), idesc_t,
                                               (ks > tp_k0 || pn > 0 || c > 0) ? 1u : 0u);
                        mma_commit_pair(&empty[s]);
                    }
                    __syncwarp();
                    if (++s == (uint32_t)C::NS) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (elect_one()) mma_commit_pair(tp_full);
                __syncwarp();
                // The main loop accumulates into the same TMEM columns: wait
                // until both CTAs have drained the partial.
                if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait_cluster(tp_empty, 0));
                if (!ok) {
                    if (lane == 0) {
                        *fail = 1;
                        atomicOr(&g_tc_error, 262144u);
                    }
                }
                tc_fence_after();
            }
            ChunkIter iter(prm, pair, npairs);
            Chunk ch;
            while (!__any_sync(0xFFFFFFFFu, *fail != 0) && iter.next(prm.chu, ch)) {
                const uint32_t idesc_sp = idesc_bf16(2 * BM, ch.n, true);
                const uint32_t idesc_dense = idesc_bf16(2 * BM, ch.n, false);
                const uint32_t panel = (uint32_t)box_rows(pick_box(ch.n / 2, prm.box4), C::HALF_N, prm.box4) * 128u;
                bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_cluster(acc_empty, (uint32_t)((it & 1) ^ 1)));
                if (!ok) {
                    if (lane == 0) {
                        *fail = 1;
                        atomicOr(&g_tc_error, 32u);
                    }
                    break;
                }
                tc_fence_after();
                const int nsp = ch.k1 - ch.k0;
                const int nst = nsp + (ch.lr ? prm.nlr : 0);
                for (int i = 0; i < nst; ++i) {
                    const bool sparse = i < nsp;
                    const int m = (int)(k % C::MS);
                    bool got = mbar_wait_cluster(&full[s], ph);
                    if (got && sparse) got = mbar_wait_cluster(&mready[m], (uint32_t)((k / C::MS) & 1));
                    if (!__all_sync(0xFFFFFFFFu, got)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t *st = smem + s * C::STAGE;
                    const uint32_t a = smem_u32(st), b = smem_u32(st + C::B_OFF);
                    if (elect_one()) {
                        if (sparse) {
                            const uint32_t e = smem_u32(meta_ring + m * 2 * C::E_BYTES);
                            tmem_cp_pair_128x128b(e_tmem, smem_desc(e, 0, 128, kLayoutNone));
                            tmem_cp_pair_128x128b(e_tmem + 4, smem_desc(e + C::E_BYTES, 0, 128, kLayoutNone));
#pragma unroll
                            for (int h = 0; h < 2; ++h)
#pragma unroll
                                for (int c = 0; c < 4; ++c) {
                                    const uint64_t adesc = desc_sw128(a + h * C::A_BYTES + 32 * c);
                                    const uint64_t bdesc = desc_sw128(b + (c >> 1) * panel + (c & 1) * 64);
                                    mma_sp_pair(tmem_base + h * BN, adesc, bdesc, e_tmem + 4 * h + (uint32_t)(c & 2),
                                                idesc_sp | (uint32_t)(c & 1), (i | c) != 0);
                                }
                            mma_commit_pair(&mempty[m]);
                        } else {
#pragma unroll
                            for (int h = 0; h < 2; ++h)
#pragma unroll
                                for (int c = 0; c < 4; ++c)
                                    mma_dense_pair(tmem_base + h * BN, desc_sw128(a + h * C::A_BYTES + 32 * c),
                                                   desc_sw128(b + 32 * c), idesc_dense, 1u);
                        }
                        mma_commit_pair(&empty[s]);
                    }
                    __syncwarp();
                    if (sparse) ++k;
                    if (++s == (uint32_t)C::NS) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (!ok) {
                    if (lane == 0) {
                        *fail = 1;
                        atomicOr(&g_tc_error, 64u);
                    }
                    break;
                }
                if (elect_one()) mma_commit_pair(acc_full);
                __syncwarp();
                ++it;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..9)
        // Warps 2..5 drain accumulator 0, warps 6..9 accumulator 1; each warp
        // reads the TMEM lanes of its quadrant (warp % 4), one output row per
        // thread.  The drain is on the critical path (the next chunk's MMAs
        // wait for both accumulators), so a thread first moves its row of the
        // chunk from TMEM into registers as packed bf16 (RNE) and releases the
        // accumulators; the stores (32-token pieces staged in shared memory,
        // TMA-stored) then overlap the next chunk's main loop.
        constexpr int kPieces = BN / 16;
        const int grp = (warp - 2) >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const bool store_thread = ((warp - 2) % 4 == 0 && lane == 0);
        uint16_t *out = reinterpret_cast<uint16_t *>(smem + C::OUT_OFF + grp * C::OUT_BYTES);
        const uint32_t empty_leader = mapa_shared(smem_u32(acc_empty), 0);
        if (prm.tp_on) {
            // Projection phase, part 1 (warps 2..5, one per TMEM lane quarter,
            // pairs with a K slice): the fp32 partial of this CTA's 128 tokens
            // goes to tp_part, then the leader learns that TMEM is free.
            const int etid = (int)threadIdx.x - 64;   // 0..255
            if (tp_busy && warp <= 5) {
                const int quarter = warp & 3;
                const int trow = quarter * 32 + lane;
                if (mbar_wait_cluster(tp_full, 0)) {
                    tc_fence_after();
                    float *dst = prm.tp_part +
                                 ((int64_t)(tp_q * prm.tp_tiles + tp_tile) * 256 + (int)rank * 128 + trow) * prm.tp_rn;
                    for (int q = 0; q < prm.tp_rn / 16; ++q) {
                        uint32_t v[16];
                        tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(q * 16), v);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            reinterpret_cast<float4 *>(dst + q * 16)[j] =
                                make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                            __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                    }
                } else {
                    *fail = 1;
                    atomicOr(&g_tc_error, 524288u);
                }
                __threadfence();   // the partial, before the count that publishes it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote_relaxed(mapa_shared(smem_u32(tp_empty), 0));
                named_bar_sync(3, 128);
                if (etid == 0) {
                    __threadfence();
                    atomicAdd(prm.tp_count, 1u);
                }
            }
            // Part 2 (all eight warps of every CTA): once every partial is
            // written, this CTA's share of T = the sum of the tp_ks partials in
            // slice order, rounded to bf16 (RNE) into tp_t16; four ranks per
            // step (r % 8 == 0).
            if (spin_count_ge(prm.tp_count, 2u * (unsigned)(prm.tp_tiles * prm.tp_ks))) {
                const int64_t total = (int64_t)M * prm.r;
                const int64_t per = ((total + gridDim.x - 1) / gridDim.x + 3) / 4 * 4;
                const int64_t e0 = (int64_t)blockIdx.x * per;
                const int64_t e1 = e0 + per < total ? e0 + per : total;
                for (int64_t e = e0 + 4 * etid; e < e1; e += 4 * 256) {
                    const int64_t m = e / prm.r;
                    const int j = (int)(e - m * prm.r);
                    const int tile = (int)(m / 256), trow = (int)(m % 256);
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (int q = 0; q < prm.tp_ks; ++q) {
                        const uint4 p4 = ld_dep_v4(prm.tp_part +
                                                   ((int64_t)(q * prm.tp_tiles + tile) * 256 + trow) * prm.tp_rn + j);
                        acc.x += __uint_as_float(p4.x);
                        acc.y += __uint_as_float(p4.y);
                        acc.z += __uint_as_float(p4.z);
                        acc.w += __uint_as_float(p4.w);
                    }
                    uint2 packed;
                    packed.x = (uint32_t)f32_to_bf16_bits(acc.x) | ((uint32_t)f32_to_bf16_bits(acc.y) << 16);
                    packed.y = (uint32_t)f32_to_bf16_bits(acc.z) | ((uint32_t)f32_to_bf16_bits(acc.w) << 16);
                    *reinterpret_cast<uint2 *>(prm.tp_t16 + e) = packed;
                }
            } else {
                *fail = 1;
                atomicOr(&g_tc_error, 1048576u);
            }
            __threadfence();   // this thread's part of T, before the count that publishes it
            named_bar_sync(4, 256);
            if (etid == 0) {
                __threadfence();
                atomicAdd(prm.tp_count + 1, 1u);
            }
        }
        int it = 0;
        ChunkIter iter(prm, pair, npairs);
        Chunk ch;
        bool part = false;   // the pair's last chunk is a K slice of a tail tile
        while (!*fail && iter.next(prm.chu, ch)) {
            if (ch.part) {
                part = true;
                break;
            }
            const int d0 = ch.d0 + grp * 2 * BM + (int)rank * BM;
            if (!mbar_wait_cluster(acc_full, (uint32_t)(it & 1))) {
                *fail = 1;
                atomicOr(&g_tc_error, 128u);
                break;
            }
            tc_fence_after();
            const uint32_t acc = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(grp * BN);
            uint32_t packed[kPieces * 8];
            // Two 16-column pieces per TMEM round trip (a piece past the
            // chunk re-reads the last valid one; its values are not used).
#pragma unroll
            for (int q = 0; q < kPieces; q += 2) {
                if (q * 16 < ch.n) {
                    const int q2 = (q + 1 < kPieces && (q + 1) * 16 < ch.n) ? q + 1 : q;
                    uint32_t h[32];
                    tmem_ld_32x32b_2x16(acc + (uint32_t)(q * 16), acc + (uint32_t)(q2 * 16), h);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        packed[q * 8 + j] = (uint32_t)f32_to_bf16_bits(__uint_as_float(h[2 * j])) |
                                            ((uint32_t)f32_to_bf16_bits(__uint_as_float(h[2 * j + 1])) << 16);
                    if (q + 1 < kPieces) {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            packed[(q + 1) * 8 + j] = (uint32_t)f32_to_bf16_bits(__uint_as_float(h[16 + 2 * j])) |
                                                      ((uint32_t)f32_to_bf16_bits(__uint_as_float(h[17 + 2 * j])) << 16);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote_relaxed(empty_leader);
#pragma unroll
            for (int p = 0; p < (kPieces + 1) / 2; ++p) {
                const int tq = ch.tok0 + 32 * p;
                if (32 * p < ch.n && tq < M) {          // uniform across the group's warps
                    const bool wide = ch.n - 32 * p >= 32;
                    if (store_thread) bulk_wait_read0();
                    named_bar_sync(1 + grp, 128);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (2 * p + (j >> 4) < kPieces && (wide || j < 16))
                            out[j * BM + row] = (uint16_t)(packed[(2 * p + (j >> 4)) * 8 + ((j & 15) >> 1)] >> (16 * (j & 1)));
                    }
                    fence_proxy_async_smem();
                    named_bar_sync(1 + grp, 128);
                    if (store_thread) {
                        tma_store_2d(wide ? &maps.y32 : &maps.y16, smem_u32(out), d0, tq);
                        bulk_commit();
                    }
                }
            }
            ++it;
        }
        if (part && !*fail) {
            // K slice q of g of tail tile tt (decoded from the plan).  This
            // thread's row of the slice's fp32 partial goes to the pair's slot
            // in blocks of four tokens ([token / 4][row][4]: a warp's 16-byte
            // stores, and the reduction's 16-byte loads, cover 512 consecutive
            // bytes); the accumulators are released; the CTA's count is added
            // once all its threads have written.
            const int64_t e = prm.tail[pair];
            const int cq = (int)((e >> 8) & 255), cg = (int)(e & 255);
            const int tt = (int)((e >> 16) - (int64_t)prm.cyc * npairs);
            const int d0 = ch.d0 + grp * 2 * BM + (int)rank * BM;
            const int64_t sub = ((int)rank * 2 + grp) * (BN * BM);
            bool ok = mbar_wait_cluster(acc_full, (uint32_t)(it & 1));
            if (ok) {
                tc_fence_after();
                const uint32_t acc = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(grp * BN);
                float4 *own = reinterpret_cast<float4 *>(prm.ks_part + (int64_t)pair * kKsSlotFloats + sub) + row;
#pragma unroll 1
                for (int q = 0; q < kPieces && q * 16 < ch.n; ++q) {
                    uint32_t h[16];
                    tmem_ld_32x32b_x16(acc + (uint32_t)(q * 16), h);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        own[(q * 4 + u) * BM] = make_float4(__uint_as_float(h[4 * u]), __uint_as_float(h[4 * u + 1]),
                                                            __uint_as_float(h[4 * u + 2]), __uint_as_float(h[4 * u + 3]));
                }
            } else {
                *fail = 1;
                atomicOr(&g_tc_error, 128u);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote_relaxed(empty_leader);
            __threadfence();
            named_bar_sync(5, 256);
            if (threadIdx.x == 64) {
                __threadfence();
                atomicAdd(prm.ks_count + tt, 1u);
            }
            // Once the 2g CTAs of the tile's slices have written theirs, the
            // pair sums its share of the token blocks of its rows over the g
            // slots in slice order (a fixed order), rounds to bf16 (RNE) and
            // stores them to Y; eight 16-byte loads per thread in flight.
            if (lane == 0) ok = spin_count_ge(prm.ks_count + tt, 2u * (unsigned)cg) && ok;
            ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
            __syncwarp();
            if (!ok) {
                *fail = 1;
                if (lane == 0) atomicOr(&g_tc_error, 2097152u);
            } else {
                const float *first = prm.ks_part + (int64_t)(pair - cq) * kKsSlotFloats + sub + 4 * row;
                const int yrow = d0 + row;
                const int nb = ch.n / 4;
                const int b0 = (nb * cq) / cg, b1 = (nb * (cq + 1)) / cg;
#pragma unroll 1
                for (int b = b0; b < b1; b += 8) {
                    float4 sum[8];
#pragma unroll 1
                    for (int sl = 0; sl < cg; ++sl) {
                        const float *src = first + (int64_t)sl * kKsSlotFloats;
                        uint4 v[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            if (b + u < b1) v[u] = ld_dep_v4(src + (int64_t)(b + u) * (BM * 4));
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            if (b + u < b1) {
                                const float4 f = make_float4(__uint_as_float(v[u].x), __uint_as_float(v[u].y),
                                                             __uint_as_float(v[u].z), __uint_as_float(v[u].w));
                                if (sl == 0) {
                                    sum[u] = f;
                                } else {
                                    sum[u].x += f.x;
                                    sum[u].y += f.y;
                                    sum[u].z += f.z;
                                    sum[u].w += f.w;
                                }
                            }
                        }
                    }
                    if (yrow < d_out) {
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int tok = ch.tok0 + 4 * (b + u);
                            if (b + u < b1) {
                                const float e4[4] = {sum[u].x, sum[u].y, sum[u].z, sum[u].w};
#pragma unroll
                                for (int w = 0; w < 4; ++w)
                                    if (tok + w < M) prm.y[(int64_t)(tok + w) * d_out + yrow] = f32_to_bf16_bits(e4[w]);
                            }
                        }
                    }
                }
            }
        }
        if (store_thread) bulk_wait_all();
    }

    tc_fence_before();
    cluster_sync_all();  // the pair's MMAs, signals and stores are done before TMEM is freed
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
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

// X [M, d_in] bf16 seen as (element in panel, row, panel) with panels of 64
// elements: one copy brings `rows` rows of two adjacent 128-byte panels, laid
// out panel after panel, each in the 128-byte swizzle.
bool make_map_panels(CUtensorMap *map, const void *X, uint64_t d_in, uint64_t M, uint32_t rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[3] = {64, M, d_in / 64};
    const cuuint64_t strides[2] = {d_in * 2, 128};
    const cuuint32_t box[3] = {64, rows, 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(X), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, bool kSparse>
cudaError_t run(const CUtensorMap &m_a, const CUtensorMap &m_meta, const CUtensorMap &m_x, const CUtensorMap &m_u,
                const CUtensorMap &m_t, const CUtensorMap &m_out, int64_t rows, int64_t M, int nk, int nlr,
                cudaStream_t stream) {
    using C = Cfg<BN, kSparse>;
    Params prm;
    prm.M = (int32_t)M;
    prm.n_ttiles = (int32_t)((M + BN - 1) / BN);
    prm.n_tiles = (int32_t)(((rows + BM - 1) / BM) * prm.n_ttiles);
    prm.nk = nk;
    prm.nlr = nlr;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t err =
        cudaFuncSetAttribute(tc_forward_kernel<BN, kSparse>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err != cudaSuccess) return err;
    const int grid = prm.n_tiles < sms ? prm.n_tiles : sms;
    tc_forward_kernel<BN, kSparse><<<grid, kThreads, C::SMEM, stream>>>(m_a, m_meta, m_x, m_u, m_t, m_out, prm);
    return cudaGetLastError();
}

constexpr auto kBF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;

template <int BN>
cudaError_t launch_sparse(const uint16_t *X, int64_t M, const uint16_t *vals, const uint8_t *meta, int64_t d_out,
                          int64_t d_in, const uint16_t *U, const uint16_t *T16, int64_t r, uint16_t *Y,
                          cudaStream_t stream) {
    CUtensorMap m_vals, m_meta, m_x, m_u, m_t, m_y;
    memset(&m_u, 0, sizeof m_u);
    memset(&m_t, 0, sizeof m_t);
    bool ok = make_map(&m_vals, kBF16, vals, d_in / 2, d_out, d_in, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&m_meta, CU_TENSOR_MAP_DATA_TYPE_UINT8, meta, d_in / 8, d_out, d_in / 8, 16, BM,
                       CU_TENSOR_MAP_SWIZZLE_NONE) &&
              make_map(&m_x, kBF16, X, d_in, M, d_in * 2, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&m_y, kBF16, Y, d_out, M, d_out * 2, BM, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (ok && r > 0)
        ok = make_map(&m_u, kBF16, U, r, d_out, r * 2, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&m_t, kBF16, T16, r, M, r * 2, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    return run<BN, true>(m_vals, m_meta, m_x, m_u, m_t, m_y, d_out, M, (int)(d_in / BK), (int)((r + 63) / 64),
                         stream);
}

// T^T = V X^T: A = V (r rows, padded to 128 by TMA zero fill), B = X tile; the
// epilogue stores D (r lanes x tokens) as T [M, r] row-major, the layout the
// rank stages of the sparse kernel read.
template <int BN>
cudaError_t launch_project(const uint16_t *X, int64_t M, const uint16_t *V, int64_t d_in, int64_t r, uint16_t *T16,
                           cudaStream_t stream) {
    CUtensorMap m_v, m_x, m_t, m_none;
    memset(&m_none, 0, sizeof m_none);
    bool ok = make_map(&m_v, kBF16, V, d_in, r, d_in * 2, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&m_x, kBF16, X, d_in, M, d_in * 2, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&m_t, kBF16, T16, r, M, r * 2, BM, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return cudaErrorInvalidValue;
    return run<BN, false>(m_v, m_none, m_x, m_none, m_none, m_t, r, M, (int)(d_in / 64), 0, stream);
}


// Host side of the 2-SM work partition (see the kernel's description): token
// tiles, the cyclic rounds and the tail ranges, sized so that every pair gets
// the same number of units in total when the cyclic phase allows it.
void plan_pairs(int64_t M, int64_t d_out, int64_t d_in, int64_t r, int chu, int tile_rows, int max_pairs,
                int tail_mode, Params2 *prm, int *pairs_out) {
    memset(prm, 0, sizeof *prm);
    prm->M = (int32_t)M;
    prm->d_out = (int32_t)d_out;
    prm->tile_rows = tile_rows;
    prm->chu = chu;
    prm->nk = (int32_t)(d_in / BK);
    prm->nlr = (int32_t)((r + 63) / 64);
    const int64_t ut = (M + 15) / 16;
    const int64_t rows = (d_out + tile_rows - 1) / tile_rows;
    const int64_t units = rows * ut;
    const int64_t ttiles = (ut + chu - 1) / chu;
    prm->ut = (int32_t)ut;
    prm->ttiles = (int32_t)ttiles;
    prm->wu = (int32_t)(ut / ttiles);
    prm->wr = (int32_t)(ut % ttiles);
    {
        int b4 = 8 * prm->wu;
        if (b4 < 64) b4 = 64;
        if (b4 > 8 * chu) b4 = 8 * chu;
        prm->box4 = b4;
    }
    const int P = (int)(units < max_pairs ? units : max_pairs);
    // Whole rounds of tiles first.  tail_mode 0: the last, partial round is
    // dealt as whole tiles too.  1: its tiles are split among all pairs, each
    // pair taking one piece (a run of tokens) of one tile (a piece never
    // crosses a tile, so no pair gets an extra chunk).  2 (512-row kernel
    // with a workspace): its tiles are split along K, each pair taking one
    // slice of the K stages of one tile at the tile's full token width.
    const int64_t T = rows * ttiles;
    prm->n_tiles = T;
    if (tail_mode == 0) {
        prm->cyc = (int32_t)((T + P - 1) / P);
        for (int p = 0; p <= P; ++p) prm->tail[p] = units;
        *pairs_out = P;
        return;
    }
    const int64_t cyc = T / P;
    prm->cyc = (int32_t)cyc;
    const int64_t c_tiles = cyc * P;
    const int64_t rem = T - c_tiles;                   // tiles left, fewer than P
    if (tail_mode == 2) {
        // Pairs [first(i), first(i+1)) share tile c_tiles + i, at most
        // max(1, nk / 4) of them (a slice keeps at least four stages); the
        // others have no tail work.
        prm->ksplit = 1;
        for (int p = 0; p <= kMaxPairs; ++p) prm->tail[p] = -1;
        int gmax = prm->nk / 4;
        gmax = gmax < 1 ? 1 : gmax > 255 ? 255 : gmax;
        for (int64_t i = 0; i < rem; ++i) {
            const int first = (int)(i * P / rem), last = (int)((i + 1) * P / rem);
            const int g = last - first < gmax ? last - first : gmax;
            for (int q = 0; q < g; ++q) prm->tail[first + q] = ((c_tiles + i) << 16) | ((int64_t)q << 8) | g;
        }
        *pairs_out = P;
        return;
    }
    auto tile_u0 = [&](int64_t tile) {                 // first unit of a tile, row-major unit order
        const int64_t rt = tile / ttiles, tt = tile % ttiles;
        return rt * ut + tt * prm->wu + (tt < prm->wr ? tt : prm->wr);
    };
    prm->tail[0] = rem > 0 ? tile_u0(c_tiles) : units;
    if (rem == 0) {
        for (int p = 0; p < P; ++p) prm->tail[p + 1] = units;
    } else {
        // Pairs [first(i), first(i+1)) share tile c_tiles + i.
        int p = 0;
        for (int64_t i = 0; i < rem; ++i) {
            const int first = (int)(i * P / rem), last = (int)((i + 1) * P / rem);
            const int g = last - first;
            const int64_t u0 = tile_u0(c_tiles + i);
            const int64_t nu = (c_tiles + i + 1 < T) ? tile_u0(c_tiles + i + 1) - u0 : units - u0;
            for (int k = 1; k <= g; ++k, ++p) prm->tail[p + 1] = u0 + nu * k / g;
        }
    }
    *pairs_out = P;
}

// Estimated cycles of the slowest pair for a plan: per chunk, its stages at
// the larger of the MMA time and the operand bytes over the shared-memory fill
// rate one SM sustains (about 44 B per cycle measured on B200 for these TMA
// tiles), plus a fixed cost per chunk (the accumulator drain of the 512-row
// kernel is not overlapped).  Only used to rank plans.
double plan_cycles(const Params2 &prm, int pairs, int chu, int half_n, int mode) {
    // mode 0: 256-row tiles, two accumulators; 1: 256-row, one accumulator;
    // 2: 512-row tiles (one accumulator per half).  A K slice of a split tail
    // tile also writes its fp32 partial (256 rows x n tokens per CTA) and
    // reads as many values back in the reduction, at ~32 B per cycle (fitted:
    // on the gate/up prefill the K split and the token split of the last
    // round measured within 1.5%).
    const bool tall = mode == 2;
    const double overhead = mode == 0 ? 800.0 : 3000.0;
    double worst = 0;
    for (int p = 0; p < pairs; ++p) {
        ChunkIter it(prm, p, pairs);
        Chunk ch;
        double cyc = 0;
        while (it.next(chu, ch)) {
            const double brows = box_rows(pick_box(ch.n / 2, prm.box4), half_n, prm.box4);
            const double bytes = tall ? 2.0 * 16384 + brows * 256 + 4096 : 16384 + brows * 256 + 2048;
            const double mma = (tall ? 4.0 : 2.0) * ch.n;
            const int nst = ch.k1 - ch.k0 + (ch.lr ? prm.nlr : 0);
            cyc += nst * (mma > bytes / 44.0 ? mma : bytes / 44.0) + overhead;
            if (ch.part) cyc += 2.0 * 256 * 4 * ch.n / 32.0;
        }
        if (cyc > worst) worst = cyc;
    }
    return worst;
}

// The plan of the pair kernels for one problem shape: kernel kind (0: 256-row
// tiles, chunks of up to 128 tokens; 1: 256-row, 240; 2: 512-row, 240;
// 3: 256-row, 256), chunk width cap and whether the last round is split.
// Chosen by the smallest plan_cycles estimate over the kinds that apply and
// chunk caps of the kind's maximum and up to five units less (narrower token
// tiles can make the tile count fit the pairs better); cached per shape.
struct PlanChoice {
    int kind, chu;
    int tail;   // plan_pairs' tail_mode
};

PlanChoice choose_plan(int64_t M, int64_t d_out, int64_t d_in, int64_t r, int sms, bool allow_ksplit) {
    struct Key {
        int64_t M, d_out, d_in, r;
        int sms;
        bool ks;
    };
    static std::mutex mu;
    static Key keys[64];
    static PlanChoice vals[64];
    static int n_cached = 0, next_slot = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < n_cached; ++i)
            if (keys[i].M == M && keys[i].d_out == d_out && keys[i].d_in == d_in && keys[i].r == r &&
                keys[i].sms == sms && keys[i].ks == allow_ksplit)
                return vals[i];
    }
    const int maxp = sms / 2 < kMaxPairs ? sms / 2 : kMaxPairs;
    PlanChoice best{-1, 0, 1};
    double best_cost = 0;
    for (int kind = 0; kind < 4; ++kind) {
        if (kind == 0 && M >= 192) continue;   // 128-token chunks: below 192 tokens only
        const int cap = kind == 0 ? Cfg2<128>::CHU : kind == 3 ? Cfg2<256>::CHU : Cfg2<240>::CHU;
        const int half_n = cap * 8;
        const int n_modes = kind == 2 && allow_ksplit ? 3 : 2;
        for (int chu = cap; chu >= cap - 5 && chu >= 1; --chu) {
            for (int t = 0; t < n_modes; ++t) {
                const int tm = t == 0 ? 1 : t == 1 ? 0 : 2;   // token split, whole, K split
                Params2 plan;
                int pairs = 0;
                plan_pairs(M, d_out, d_in, r, chu, kind == 2 ? 4 * BM : 2 * BM, maxp, tm, &plan, &pairs);
                const double cost = plan_cycles(plan, pairs, chu, half_n, kind == 2 ? 2 : kind == 3 ? 1 : 0);
                if (best.kind < 0 || cost < best_cost) {
                    best = PlanChoice{kind, chu, tm};
                    best_cost = cost;
                }
            }
        }
    }
    std::lock_guard<std::mutex> lock(mu);
    keys[next_slot] = Key{M, d_out, d_in, r, sms, allow_ksplit};
    vals[next_slot] = best;
    next_slot = (next_slot + 1) % 64;
    if (n_cached < 64) ++n_cached;
    return best;
}

// Host-only check of a pair plan (slr_plan_check): builds the plan as a
// launch would and walks every pair's chunk sequence.  Counts violations:
// each (row tile, 16-token unit, K stage) covered by exactly one chunk, the
// rank stages of each (row tile, unit) by exactly one chunk, chunk rows and
// tokens inside the problem, a K slice only as a pair's last chunk and with
// slice, slot and counter indices in range.  -1 for arguments out of range.
int64_t plan_check(int64_t M, int64_t d_out, int64_t d_in, int64_t r, int kernel, int tail_mode, int max_pairs,
                   int chu) {
    if (M < 1 || M > INT32_MAX || d_out < 1 || d_out > INT32_MAX || d_in < BK || d_in % BK != 0 || r < 0 ||
        r % 8 != 0 || kernel < 0 || kernel > 3 || tail_mode < 0 || tail_mode > 2 || max_pairs < 1 ||
        max_pairs > kMaxPairs || (tail_mode == 2 && kernel != 2))
        return -1;
    const int cap = kernel == 0 ? Cfg2<128>::CHU : kernel == 1 ? Cfg2<240>::CHU : kernel == 3 ? Cfg2<256>::CHU
                                                                                              : CfgT<240>::CHU;
    if (chu <= 0 || chu > cap) chu = cap;
    const int tile_rows = kernel == 2 ? 4 * BM : 2 * BM;
    Params2 prm;
    int P = 0;
    plan_pairs(M, d_out, d_in, r, chu, tile_rows, max_pairs, tail_mode, &prm, &P);
    const int64_t rows = (d_out + tile_rows - 1) / tile_rows, ut = prm.ut, nk = prm.nk;
    if (rows * ut * nk > ((int64_t)1 << 26)) return -1;   // keeps the check's memory bounded
    std::vector<uint8_t> cover((size_t)(rows * ut * nk), 0), rank((size_t)(rows * ut), 0);
    int64_t bad = (P < 1 || P > max_pairs) ? 1 : 0;
    for (int p = 0; p < P; ++p) {
        ChunkIter it(prm, p, P);
        Chunk ch;
        bool part_seen = false;
        int64_t guard = 0;
        while (it.next(chu, ch)) {
            if (++guard > rows * ut + 1) {   // more chunks than units: a loop that does not end
                ++bad;
                break;
            }
            if (part_seen) ++bad;   // a K slice is the pair's last chunk
            if (ch.d0 < 0 || ch.d0 % tile_rows != 0 || ch.d0 / tile_rows >= rows || ch.n <= 0 || ch.n % 16 != 0 ||
                ch.n > 16 * cap || ch.tok0 < 0 || ch.tok0 % 16 != 0 || ch.k0 < 0 || ch.k1 > nk || ch.k0 >= ch.k1) {
                ++bad;
                continue;
            }
            if (ch.part) {
                part_seen = true;
                const int64_t e = prm.tail[p];
                const int q = (int)((e >> 8) & 255), g = (int)(e & 255);
                const int64_t tt = (e >> 16) - (int64_t)prm.cyc * P;
                if (!prm.ksplit || g < 2 || q >= g || p - q < 0 || p - q + g > P || tt < 0 || tt >= P ||
                    64 + 4 * tt + 4 > 1024)
                    ++bad;
            }
            const int64_t rt = ch.d0 / tile_rows;
            for (int64_t u = ch.tok0 / 16; u < (ch.tok0 + ch.n) / 16; ++u) {
                if (u >= ut) {
                    ++bad;
                    continue;
                }
                for (int64_t k = ch.k0; k < ch.k1; ++k) {
                    uint8_t &c = cover[(size_t)((rt * ut + u) * nk + k)];
                    if (c < 255) ++c;
                }
                if (ch.lr) {
                    uint8_t &c = rank[(size_t)(rt * ut + u)];
                    if (c < 255) ++c;
                }
            }
        }
    }
    for (uint8_t c : cover) bad += c != 1;
    for (uint8_t c : rank) bad += c != 1;
    return bad;
}

template <int BN>
cudaError_t launch_sparse_pair(const uint16_t *X, int64_t M, const uint16_t *vals, const uint8_t *meta,
                               int64_t d_out, int64_t d_in, const uint16_t *U, const uint16_t *T16, int64_t r,
                               uint16_t *Y, bool after_projection, int tail_mode, cudaStream_t stream, int chu = 0) {
    using C = Cfg2<BN>;
    if (tail_mode == 2) tail_mode = 1;   // the K split is the 512-row kernel's
    Maps2 maps;
    memset(&maps, 0, sizeof maps);
    bool ok = make_map(&maps.vals, kBF16, vals, d_in / 2, d_out, d_in, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&maps.meta, CU_TENSOR_MAP_DATA_TYPE_UINT8, meta, d_in / 8, d_out, d_in / 8, 16, BM,
                       CU_TENSOR_MAP_SWIZZLE_NONE) &&
              make_map(&maps.y32, kBF16, Y, d_out, M, d_out * 2, BM, 32, CU_TENSOR_MAP_SWIZZLE_NONE) &&
              make_map(&maps.y16, kBF16, Y, d_out, M, d_out * 2, BM, 16, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (ok && r > 0) ok = make_map(&maps.u, kBF16, U, r, d_out, r * 2, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t err = cudaFuncSetAttribute(tc2_forward_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err != cudaSuccess) return err;
    Params2 prm;
    int pairs = 0;
    if (chu <= 0 || chu > C::CHU) chu = C::CHU;
    plan_pairs(M, d_out, d_in, r, chu, 2 * BM, sms / 2 < kMaxPairs ? sms / 2 : kMaxPairs, tail_mode, &prm, &pairs);
    // X and T boxes, now that the plan fixes box 4's rows.
    for (int i = 0; i < 7; ++i) {
        const uint32_t rows_i = (uint32_t)box_rows(i, C::HALF_N, prm.box4);
        if (!make_map_panels(&maps.xs[i], X, d_in, M, rows_i)) return cudaErrorInvalidValue;
        if (r > 0 && !make_map(&maps.ts[i], kBF16, T16, r, M, r * 2, 64, rows_i, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    // Directly after the projection kernel on this stream: programmatic
    // dependent launch (the producer waits before it loads T).  Otherwise an
    // ordinary launch, which must not overlap an unrelated preceding kernel.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(kThreads2);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (after_projection && r > 0) ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, tc2_forward_kernel<BN>, maps, prm);
}

template <int BN>
cudaError_t launch_sparse_tall(const uint16_t *X, int64_t M, const uint16_t *vals, const uint8_t *meta,
                               int64_t d_out, int64_t d_in, const uint16_t *U, const uint16_t *T16, int64_t r,
                               uint16_t *Y, bool after_projection, int tail_mode, cudaStream_t stream, int chu = 0,
                               const uint16_t *V = nullptr, uint8_t *fused_ws = nullptr, size_t ws_bytes = 0) {
    using C = CfgT<BN>;
    // With a fused workspace (single-call forward, r > 0) T lives in its
    // first region; the kernel forms T itself (projection phase) when r <=
    // 128, and the last round may be split along K (partials and counters in
    // the workspace).  Without one the K split falls back to the token split.
    const bool fused = V != nullptr && fused_ws != nullptr && r > 0;
    bool tp = fused && r <= 128;
    if (fused) T16 = reinterpret_cast<const uint16_t *>(fused_ws);
    if (tail_mode == 2 && !fused) tail_mode = 1;
    Maps2 maps;
    memset(&maps, 0, sizeof maps);
    bool ok = make_map(&maps.vals, kBF16, vals, d_in / 2, d_out, d_in, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&maps.meta, CU_TENSOR_MAP_DATA_TYPE_UINT8, meta, d_in / 8, d_out, d_in / 8, 16, BM,
                       CU_TENSOR_MAP_SWIZZLE_NONE) &&
              make_map(&maps.y32, kBF16, Y, d_out, M, d_out * 2, BM, 32, CU_TENSOR_MAP_SWIZZLE_NONE) &&
              make_map(&maps.y16, kBF16, Y, d_out, M, d_out * 2, BM, 16, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (ok && r > 0) ok = make_map(&maps.u, kBF16, U, r, d_out, r * 2, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B);
    const int tp_rn = r <= 64 ? 64 : 128;
    if (ok && tp)
        ok = make_map_panels(&maps.xt, X, d_in, M, 128) && make_map_panels(&maps.vt, V, d_in, r, tp_rn / 2);
    if (!ok) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t err = cudaFuncSetAttribute(tc2t_forward_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err != cudaSuccess) return err;
    Params2 prm;
    int pairs = 0;
    if (chu <= 0 || chu > C::CHU) chu = C::CHU;
    int max_pairs = sms / 2 < kMaxPairs ? sms / 2 : kMaxPairs;
    if (tp || tail_mode == 2) {
        // The projection phase and the K-split reduction wait on counters
        // that other CTAs of the grid advance, so the whole grid must be
        // resident at once: no more pairs than the device holds clusters of
        // this kernel.
        int ncl = 0;
        cudaLaunchConfig_t occ = {};
        occ.gridDim = dim3((unsigned)(2 * max_pairs));
        occ.blockDim = dim3(kThreadsT);
        occ.dynamicSmemBytes = C::SMEM;
        err = cudaOccupancyMaxActiveClusters(&ncl, tc2t_forward_kernel<BN>, &occ);
        if (err != cudaSuccess) return err;
        if (ncl < max_pairs) max_pairs = ncl;
        if (max_pairs < 1) return cudaErrorInvalidConfiguration;
    }
    plan_pairs(M, d_out, d_in, r, chu, 4 * BM, max_pairs, tail_mode, &prm, &pairs);
    const FusedLayout L = fused_layout(M, r, 0);
    if (prm.ksplit && (ws_bytes < L.off_ks_part || (ws_bytes - L.off_ks_part) / (kKsSlotFloats * 4) < (size_t)pairs))
        // A workspace sized for a device with fewer SMs: not enough slots.
        plan_pairs(M, d_out, d_in, r, chu, 4 * BM, max_pairs, 1, &prm, &pairs);
    // X and T boxes, now that the plan fixes box 4's rows.
    for (int i = 0; i < 7; ++i) {
        const uint32_t rows_i = (uint32_t)box_rows(i, C::HALF_N, prm.box4);
        if (!make_map_panels(&maps.xs[i], X, d_in, M, rows_i)) return cudaErrorInvalidValue;
        if (r > 0 && !make_map(&maps.ts[i], kBF16, T16, r, M, r * 2, 64, rows_i, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    // Fewer pairs than 256-token tiles: T from the projection kernel instead.
    if (tp && (M + 255) / 256 > pairs) tp = false;
    prm.meta = meta;
    prm.meta_ld = d_in / 8;
    prm.tp_on = 0;
    prm.r = (int32_t)r;
    prm.tp_rn = tp_rn;
    prm.tp_tiles = (int32_t)((M + 255) / 256);
    prm.tp_ks = 1;
    prm.tp_part = nullptr;
    prm.tp_t16 = const_cast<uint16_t *>(T16);
    prm.tp_count = nullptr;
    prm.ks_part = nullptr;
    prm.ks_count = nullptr;
    prm.y = Y;
    if (tp) {
        // Token tiles of 256 over the pairs, K split as far as the pairs go
        // (every tile has a pair: M <= 256 * pairs).
        const int nk = (int)(d_in / BK);
        int ks = pairs / prm.tp_tiles;
        if (ks > nk) ks = nk;
        prm.tp_on = 1;
        prm.tp_ks = ks < 1 ? 1 : ks;
        prm.tp_count = reinterpret_cast<unsigned int *>(fused_ws + L.off_count);
        prm.tp_part = reinterpret_cast<float *>(fused_ws + L.off_part);
    }
    if (prm.ksplit) {
        prm.ks_count = reinterpret_cast<unsigned int *>(fused_ws + L.off_ks_count);
        prm.ks_part = reinterpret_cast<float *>(fused_ws + L.off_ks_part);
    }
    if (tp || prm.ksplit) {
        // The counters start at zero (the kernel reads, never resets them).
        err = cudaMemsetAsync(fused_ws + L.off_count, 0, 1024, stream);
        if (err != cudaSuccess) return err;
    }
    if (fused && !tp) {
        err = launch_tc_project(X, M, V, d_in, r, const_cast<uint16_t *>(T16), false, stream);
        if (err != cudaSuccess) return err;
        after_projection = true;
    }
    // Directly after the projection kernel on this stream: programmatic
    // dependent launch (the producer waits before it loads T).  Otherwise an
    // ordinary launch, which must not overlap an unrelated preceding kernel.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(kThreadsT);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (after_projection && r > 0 && !tp) ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, tc2t_forward_kernel<BN>, maps, prm);
}


// =====================================================================================
// Rank projection T = X V^T with split K (the first factor of the low-rank term,
// LoSparse section 3.2).  A cluster of KS CTAs (KS <= 8) owns 128 tokens; CTA
// rank q runs the q-th slice of the d_in stages with A = X tile (128 tokens,
// M = 128) and B = V (N = RN >= r, rows past r zero-filled by TMA), so its TMEM
// holds a partial T tile (lane = token, column = rank index).  The epilogue
// warps write the partial to shared memory (fp32, padded rows), the cluster
// synchronises, and each CTA sums its 128/KS tokens over all KS partials through
// distributed shared memory and writes them to T [M, r] in bf16.  One kernel, no
// atomics, no scratch outside shared memory.
template <int RN>
struct CfgP {
    static constexpr int A_BYTES = BM * 64 * 2;          // 16 KB: 128 tokens x 64 K
    static constexpr int B_BYTES = RN * 64 * 2;          // RN rows of V x 64 K
    static constexpr int STAGE = ((A_BYTES + B_BYTES + 1023) / 1024) * 1024;
    static constexpr int PROW = RN + 4;                  // padded fp32 row of the partial tile
    static constexpr int P_BYTES = BM * PROW * 4;
    // Up to ~110 KB of ring so that two CTAs fit on an SM when RN <= 128.
    static constexpr int NS_FIT = (RN <= 128 ? 112640 : 230400) / STAGE;
    static constexpr int NS = NS_FIT > 8 ? 8 : (NS_FIT < 2 ? 2 : NS_FIT);
    static constexpr int RING = NS * STAGE;
    static constexpr int BAR_OFF = (RING > P_BYTES ? RING : P_BYTES);
    static constexpr int SMEM = BAR_OFF + 256 + 1024;
    static constexpr uint32_t TMEM_COLS = pow2_at_least(RN);
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(RN % 16 == 0 && RN <= 256, "MMA N");
};

template <int RN>
__global__ void __launch_bounds__(kThreads, 1)
    tc_project_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_v,
                      uint16_t *__restrict__ T16, int32_t M, int32_t r, int32_t nk_total, int32_t chained) {
    using C = CfgP<RN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *empty = full + C::NS;
    uint64_t *acc_full = empty + C::NS;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    volatile uint32_t *fail = tmem_slot + 1;
    float *part = reinterpret_cast<float *>(smem);      // reuses the ring after the K loop

    // The fused forward kernel that consumes T may launch now (it waits for
    // this grid before its first load of T).
    asm volatile("griddepcontrol.launch_dependents;");
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    uint32_t ks_n, ks_q;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(ks_n));
    ks_q = cluster_ctarank();
    const int tile = blockIdx.x / (int)ks_n;
    const int tok0 = tile * BM;
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
        if (lane == 0) {
            // Chained launch: the preceding grid may still be running.  V is a
            // weight: the first ring's V tiles are requested now; X only after
            // the wait for the preceding grid (which also orders this grid's
            // writes of T after every earlier reader of the workspace).
            const int prologue = chained ? min(k_end - k_begin, C::NS) : 0;
            for (int i = 0; i < prologue; ++i) {
                mbar_expect_tx(&full[i], C::A_BYTES + C::B_BYTES);
                tma_load_2d(&tm_v, smem_u32(smem + i * C::STAGE + C::A_BYTES), &full[i], (k_begin + i) * 64, 0);
            }
            if (chained) asm volatile("griddepcontrol.wait;" ::: "memory");
            for (int i = 0; i < prologue; ++i)
                tma_load_2d(&tm_x, smem_u32(smem + i * C::STAGE), &full[i], (k_begin + i) * 64, tok0);
            uint32_t s = (uint32_t)(prologue % C::NS), ph = prologue == C::NS ? 1u : 0u;
            for (int ks = k_begin + prologue; ks < k_end; ++ks) {
                if (!mbar_wait(&empty[s], ph ^ 1)) {
                    *fail = 1;
                    atomicOr(&g_tc_error, 512u);
                    break;
                }
                uint8_t *st = smem + s * C::STAGE;
                mbar_expect_tx(&full[s], C::A_BYTES + C::B_BYTES);
                tma_load_2d(&tm_x, smem_u32(st), &full[s], ks * 64, tok0);
                tma_load_2d(&tm_v, smem_u32(st + C::A_BYTES), &full[s], ks * 64, 0);
                if (++s == (uint32_t)C::NS) {
                    s = 0;
                    ph ^= 1;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t kIdesc = idesc_bf16(BM, RN, false);
            uint32_t s = 0, ph = 0;
            bool ok = true;
            for (int ks = k_begin; ks < k_end; ++ks) {
                if (!mbar_wait(&full[s], ph)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint8_t *st = smem + s * C::STAGE;
                const uint32_t a = smem_u32(st), b = smem_u32(st + C::A_BYTES);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    mma_dense(tmem_base, desc_sw128(a + 32 * c), desc_sw128(b + 32 * c), kIdesc, (ks > k_begin) || c);
                mma_commit(&empty[s]);
                if (++s == (uint32_t)C::NS) {
                    s = 0;
                    ph ^= 1;
                }
            }
            if (!ok) {
                *fail = 1;
                atomicOr(&g_tc_error, 1024u);
            }
            mma_commit(acc_full);  // also fires when this CTA had no stages
        }
    } else {
        // epilogue: TMEM partial -> shared memory (fp32); an empty K slice
        // contributes zeros
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;   // token within the tile
        const bool have = k_end > k_begin;
        if (mbar_wait(acc_full, 0)) {
            tc_fence_after();
            // 16 columns per load (RN is a multiple of 16)
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
            atomicOr(&g_tc_error, 2048u);
        }
    }
    tc_fence_before();
    cluster_sync_all();  // every CTA's partial is in its shared memory

    // Reduction: CTA q sums tokens [q*TPC, (q+1)*TPC) over the cluster's partials.
    if (warp >= 2) {
        const int tpc = BM / (int)ks_n;
        const int items = tpc * (RN / 4);
        const uint32_t part_addr = smem_u32(part);
        for (int it = threadIdx.x - 64; it < items; it += 128) {
            const int t = (int)ks_q * tpc + it / (RN / 4);
            const int c = (it % (RN / 4)) * 4;
            const uint32_t off = (uint32_t)((t * C::PROW + c) * 4);
            // issue all remote loads before summing, so they are in flight together
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
            const int tok = tok0 + t;
            if (tok < M && c < r) {
                uint2 packed;
                packed.x = (uint32_t)f32_to_bf16_bits(acc.x) | ((uint32_t)f32_to_bf16_bits(acc.y) << 16);
                packed.y = (uint32_t)f32_to_bf16_bits(acc.z) | ((uint32_t)f32_to_bf16_bits(acc.w) << 16);
                *reinterpret_cast<uint2 *>(T16 + (int64_t)tok * r + c) = packed;   // r % 8 == 0: 8-byte aligned
            }
        }
    }
    cluster_sync_all();  // no CTA leaves while its partial may still be read
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
    }
}

template <int RN>
cudaError_t launch_project_splitk(const uint16_t *X, int64_t M, const uint16_t *V, int64_t d_in, int64_t r,
                                  uint16_t *T16, bool chained, cudaStream_t stream) {
    using C = CfgP<RN>;
    CUtensorMap m_x, m_v;
    if (!make_map(&m_x, kBF16, X, d_in, M, d_in * 2, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&m_v, kBF16, V, d_in, r, d_in * 2, 64, RN, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int tiles = (int)((M + BM - 1) / BM);
    const int nk = (int)(d_in / 64);
    // Split K over a cluster of up to 8 CTAs, keeping the grid within one
    // SM's worth of CTAs per SM (clusters of 8 only when few token tiles make
    // the K loop long per CTA).
    int ks = 1;
    while (ks < 8 && ks * 2 <= nk && tiles * ks * 2 <= (ks >= 4 ? sms : 2 * sms)) ks *= 2;
    cudaError_t err = cudaFuncSetAttribute(tc_project_kernel<RN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * ks));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = chained ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, tc_project_kernel<RN>, m_x, m_v, T16, (int32_t)M, (int32_t)r, (int32_t)nk,
                              (int32_t)(chained ? 1 : 0));
}


// =====================================================================================
// Split-K forward for few tokens (BN = 16 .. 128 per tile): Y = X S^T + T U^T
// when the layer is bound by the bytes of S, or has too few row tiles to keep
// the 2-SM pairs busy.  One cluster of KS CTAs (KS <= 4) owns a 128-row x
// BN-token tile and splits its K stages (the 2:4 stages, then the rank stages)
// across its CTAs, so that all SMs stream S at once even when d_out / 128 is
// small; the token tiles of one row tile are neighbouring clusters, which
// stream the same S tile at about the same time (one read from HBM).
// Each CTA accumulates its partial Y^T tile in TMEM (2:4 tcgen05.mma.sp with
// the same metadata permute as the large-M kernels, N = BN), writes it to
// shared memory in fp32, and after a cluster barrier CTA q sums rows
// [q*128/KS, (q+1)*128/KS) over the KS partials through distributed shared
// memory and stores them to Y in bf16 (RNE).
//
// Launch modes (pdl): 0 plain; 1 programmatic dependent of the projection
// kernel that writes T (wait before the first load of T); 2 chained: also
// the preceding work may still run, so S and U are requested first and the
// kernel waits before its first load of X.
//
// CTAs per cluster of the split-K kernel: split K two or four ways while the
// grid stays within two CTAs per SM.
inline int small_cluster(int64_t work, int64_t stages, int sms) {
    int ks = 1;
    while (ks < 4 && ks * 2 <= stages && work * ks * 2 <= 2 * (int64_t)sms) ks *= 2;
    return ks;
}

// Whether the split-K kernel on 128-token tiles is the faster choice for
// M > 64.  It is when the layer has few tiles of 128 rows x 128 tokens (at
// most a quarter of the SM count: the pair kernels then leave pairs idle or
// stream each S tile for short token chunks), or, with a long K (d_in >=
// 8192), when its tiles still fit one CTA per SM.  Measured on B200 with
// r = 64 against the best pair-kernel plan: 4096 x 4096 at M = 65..128 21 vs
// 25 us (64 tiles from M = 160: 28.6 vs 26.7 us, pairs ahead); 1024 x 4096 up
// to M = 512 (32 tiles) 19-22 vs 19-26 us; 4096 x 14336 at M = 65..512 37-64
// vs 60-67 us (160 tiles at M = 640: 106 vs 73 us, pairs ahead); 8192 x 28672
// at M = 65..256 72-115 vs 111-131 us; 14336 x 4096 (112 tiles, short K) and
// 28672 x 8192 (224 tiles) stay on the pair kernels.
inline bool small_wins(int64_t M, int64_t d_out, int64_t d_in, int sms) {
    const int64_t work = ((d_out + BM - 1) / BM) * ((M + 127) / 128);
    return work * 4 <= (int64_t)sms || (d_in >= 8192 && work <= (int64_t)sms);
}

template <int BN>
struct CfgS {
    static constexpr int A_BYTES = BM * 64 * 2;          // 16 KB of packed values (128 logical K)
    static constexpr int B_HALF = BN * 64 * 2;           // BN tokens x one 128-byte panel
    static constexpr int B_BYTES = 2 * B_HALF;
    static constexpr int E_BYTES = BM * BK / 8;          // 2 KB of metadata
    static constexpr int STAGE = ((A_BYTES + B_BYTES + E_BYTES + 1023) / 1024) * 1024;
    static constexpr int PROW = BN + 4;                  // padded fp32 row of the partial tile
    static constexpr int P_BYTES = BM * PROW * 4;
    static constexpr int NS_FIT = 114432 / STAGE;        // two CTAs per SM (114432 + 1280 <= 115712)
    static constexpr int NS = NS_FIT > 8 ? 8 : (NS_FIT < 2 ? 2 : NS_FIT);
    static constexpr int RING = NS * STAGE;
    static constexpr int BAR_OFF = (RING > P_BYTES ? RING : P_BYTES);
    static constexpr int SMEM = BAR_OFF + 256 + 1024;
    static constexpr uint32_t ECOL = BN;
    static constexpr uint32_t TMEM_COLS = pow2_at_least(BN + 4);
    static_assert(SMEM <= 115712, "two CTAs per SM (228 KB less 1 KB reserved per CTA)");
    static_assert(BN % 16 == 0 && BN <= 128, "MMA N");
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 2)
    tc_small_kernel(const __grid_constant__ CUtensorMap tm_vals, const __grid_constant__ CUtensorMap tm_meta,
                    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_u,
                    const __grid_constant__ CUtensorMap tm_t, uint16_t *__restrict__ Y, int32_t M, int32_t d_out,
                    int32_t n_ttiles, int32_t nk, int32_t nlr, int32_t pdl) {
    using C = CfgS<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *empty = full + C::NS;
    uint64_t *acc_full = empty + C::NS;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    float *part = reinterpret_cast<float *>(smem);      // reuses the ring after the K loop

    // The next kernel on the stream may be scheduled now (a chained forward
    // waits for this grid before it reads anything this grid writes).
    asm volatile("griddepcontrol.launch_dependents;");
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    uint32_t ks_n;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(ks_n));
    const uint32_t ks_q = cluster_ctarank();
    const int work = blockIdx.x / (int)ks_n;
    const int d0 = (work / n_ttiles) * BM;
    const int tok0 = (work % n_ttiles) * BN;
    const int total = nk + nlr;
    const int k_begin = (int)(((int64_t)total * ks_q) / ks_n);
    const int k_end = (int)(((int64_t)total * (ks_q + 1)) / ks_n);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    // The producer needs no TMEM: warp 0 arrives on the start barrier and
    // streams at once; the other warps wait there for the TMEM allocation.
    uint32_t tmem_base = 0;
    if (warp == 0) {
        asm volatile("bar.arrive 1, %0;" ::"r"(kThreads) : "memory");
    } else {
        if (warp == 1) {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                         "r"(C::TMEM_COLS));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        }
        tc_fence_before();
        asm volatile("bar.sync 1, %0;" ::"r"(kThreads) : "memory");
        tc_fence_after();
        tmem_base = *tmem_slot;
    }

    if (warp == 0) {
        if (lane == 0) {
            // Chained launch (pdl == 2): the preceding grid may still run.  The
            // first ring's weight operands (S tile and metadata, or a U tile)
            // are requested now; its X / T loads follow the wait.
            const int prologue = pdl == 2 ? min(k_end - k_begin, C::NS) : 0;
            for (int i = 0; i < prologue; ++i) {
                const int ks = k_begin + i;
                uint8_t *st = smem + i * C::STAGE;
                if (ks < nk) {
                    mbar_expect_tx(&full[i], C::A_BYTES + C::B_BYTES + C::E_BYTES);
                    tma_load_2d(&tm_vals, smem_u32(st), &full[i], ks * 64, d0);
                    tma_load_2d(&tm_meta, smem_u32(st + C::A_BYTES + C::B_BYTES), &full[i], ks * (BK / 8), d0);
                } else {
                    mbar_expect_tx(&full[i], C::A_BYTES + C::B_HALF);
                    tma_load_2d(&tm_u, smem_u32(st), &full[i], (ks - nk) * 64, d0);
                }
            }
            if (pdl == 2) asm volatile("griddepcontrol.wait;" ::: "memory");
            for (int i = 0; i < prologue; ++i) {
                const int ks = k_begin + i;
                const uint32_t b = smem_u32(smem + i * C::STAGE + C::A_BYTES);
                if (ks < nk) {
                    tma_load_2d(&tm_x, b, &full[i], ks * BK, tok0);
                    tma_load_2d(&tm_x, b + C::B_HALF, &full[i], ks * BK + 64, tok0);
                } else {
                    tma_load_2d(&tm_t, b, &full[i], (ks - nk) * 64, tok0);
                }
            }
            uint32_t s = (uint32_t)(prologue % C::NS), ph = prologue == C::NS ? 1u : 0u;
            bool t_ready = pdl != 1;
            for (int ks = k_begin + prologue; ks < k_end; ++ks) {
                if (!mbar_wait(&empty[s], ph ^ 1)) {
                    atomicOr(&g_tc_error, 4096u);
                    break;
                }
                uint8_t *st = smem + s * C::STAGE;
                const uint32_t a = smem_u32(st), b = smem_u32(st + C::A_BYTES),
                               e = smem_u32(st + C::A_BYTES + C::B_BYTES);
                if (ks < nk) {
                    mbar_expect_tx(&full[s], C::A_BYTES + C::B_BYTES + C::E_BYTES);
                    tma_load_2d(&tm_vals, a, &full[s], ks * 64, d0);
                    tma_load_2d(&tm_x, b, &full[s], ks * BK, tok0);
                    tma_load_2d(&tm_x, b + C::B_HALF, &full[s], ks * BK + 64, tok0);
                    tma_load_2d(&tm_meta, e, &full[s], ks * (BK / 8), d0);
                } else {
                    if (!t_ready) {
                        // T may still be in production (programmatic dependent launch)
                        asm volatile("griddepcontrol.wait;" ::: "memory");
                        t_ready = true;
                    }
                    const int j = ks - nk;
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
    } else if (warp == 1) {
        constexpr uint32_t kIdescSp = idesc_bf16(BM, BN, true);
        constexpr uint32_t kIdescDense = idesc_bf16(BM, BN, false);
        const uint32_t e_tmem = tmem_base + C::ECOL;
        uint32_t s = 0, ph = 0;
        bool ok = true;
        for (int ks = k_begin; ks < k_end; ++ks) {
            if (!mbar_wait(&full[s], ph)) {
                ok = false;
                break;
            }
            uint8_t *st = smem + s * C::STAGE;
            const uint32_t a = smem_u32(st), b = smem_u32(st + C::A_BYTES);
            const uint32_t first = (ks == k_begin) ? 1u : 0u;
            if (ks < nk) {
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
                        mma_sp(tmem_base, adesc, bdesc, e_tmem + (uint32_t)(c & 2), kIdescSp | (uint32_t)(c & 1),
                               !(first && c == 0));
                    }
                    mma_commit(&empty[s]);
                }
            } else if (lane == 0) {
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    mma_dense(tmem_base, desc_sw128(a + 32 * c), desc_sw128(b + 32 * c), kIdescDense,
                              !(first && c == 0));
                mma_commit(&empty[s]);
            }
            __syncwarp();
            if (++s == (uint32_t)C::NS) {
                s = 0;
                ph ^= 1;
            }
        }
        if (!ok && lane == 0) atomicOr(&g_tc_error, 8192u);
        if (lane == 0) mma_commit(acc_full);  // fires at once when this CTA had no stages
        __syncwarp();
    } else {
        // TMEM partial (lane = output row, column = token) -> shared memory
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const bool have = k_end > k_begin;
        if (mbar_wait(acc_full, 0)) {
            tc_fence_after();
#pragma unroll 1
            for (int q = 0; q < BN / 16; ++q) {
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
            atomicOr(&g_tc_error, 16384u);
        }
    }
    tc_fence_before();
    cluster_sync_all();  // every CTA's partial is in its shared memory

    // CTA q: rows [q*RPC, (q+1)*RPC) of the tile, all BN tokens, summed over
    // the cluster; thread -> (row, group of 4 tokens), rows fastest so that
    // the bf16 stores of one token are contiguous in Y.
    if (warp >= 2) {
        const int rpc = BM / (int)ks_n;
        const int items = rpc * (BN / 4);
        const uint32_t part_addr = smem_u32(part);
        for (int it = threadIdx.x - 64; it < items; it += 128) {
            const int row = (int)ks_q * rpc + it % rpc;
            const int tg = it / rpc;
            const uint32_t off = (uint32_t)((row * C::PROW + 4 * tg) * 4);
            float4 p[4];
#pragma unroll
            for (uint32_t q = 0; q < 4; ++q)
                p[q] = q < ks_n ? ld_shared_cluster_v4(mapa_shared(part_addr + off, q)) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float sum[4] = {p[0].x + p[1].x + p[2].x + p[3].x, p[0].y + p[1].y + p[2].y + p[3].y,
                                  p[0].z + p[1].z + p[2].z + p[3].z, p[0].w + p[1].w + p[2].w + p[3].w};
            const int out_row = d0 + row;
            if (out_row < d_out) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int tok = tok0 + 4 * tg + j;
                    if (tok < M) Y[(int64_t)tok * d_out + out_row] = f32_to_bf16_bits(sum[j]);
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

// pdl: 0 plain launch, 1 after the projection kernel (waits before T), 2
// chained (waits before X and T).
template <int BN>
cudaError_t launch_sparse_small(const uint16_t *X, int64_t M, const uint16_t *vals, const uint8_t *meta,
                                int64_t d_out, int64_t d_in, const uint16_t *U, const uint16_t *T16, int64_t r,
                                uint16_t *Y, int pdl, cudaStream_t stream) {
    using C = CfgS<BN>;
    CUtensorMap m_vals, m_meta, m_x, m_u, m_t;
    memset(&m_u, 0, sizeof m_u);
    memset(&m_t, 0, sizeof m_t);
    bool ok = make_map(&m_vals, kBF16, vals, d_in / 2, d_out, d_in, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&m_meta, CU_TENSOR_MAP_DATA_TYPE_UINT8, meta, d_in / 8, d_out, d_in / 8, 16, BM,
                       CU_TENSOR_MAP_SWIZZLE_NONE) &&
              make_map(&m_x, kBF16, X, d_in, M, d_in * 2, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (ok && r > 0)
        ok = make_map(&m_u, kBF16, U, r, d_out, r * 2, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&m_t, kBF16, T16, r, M, r * 2, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_ttiles = (int)((M + BN - 1) / BN);
    const int work = (int)((d_out + BM - 1) / BM) * n_ttiles;
    const int nk = (int)(d_in / BK), nlr = (int)((r + 63) / 64);
    const int ks = small_cluster(work, nk + nlr, sms);
    cudaError_t err = cudaFuncSetAttribute(tc_small_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(work * ks));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    const int mode = (pdl == 1 && r == 0) ? 0 : pdl;
    cfg.numAttrs = mode != 0 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, tc_small_kernel<BN>, m_vals, m_meta, m_x, m_u, m_t, Y, (int32_t)M,
                              (int32_t)d_out, (int32_t)n_ttiles, (int32_t)nk, (int32_t)nlr, (int32_t)mode);
}

}  // namespace tc

cudaError_t launch_tc_forward(const uint16_t *X, int64_t M, const uint16_t *vals, const uint8_t *meta,
                              int64_t d_out, int64_t d_in, const uint16_t *U, const uint16_t *T16, int64_t r,
                              uint16_t *Y, int pdl, cudaStream_t stream) {
    if (M <= 0) return cudaSuccess;
    if (M > INT32_MAX || d_out > INT32_MAX || d_in > INT32_MAX) return cudaErrorInvalidValue;
    // Chained launches (pdl == 2) exist for the split-K kernel of M <= 64 only.
    if (pdl == 2 && M > kChainMaxM) return cudaErrorInvalidValue;
    const bool after_projection = pdl == 1;
    // SLR_TC_KERNEL=1sm|2sm128[w]|2sm240[w]|2smtall[w]|small forces one kernel
    // (a trailing w deals whole tiles only); used by the tests and for A/B
    // measurements.
    const char *force = getenv("SLR_TC_KERNEL");
    if (force != nullptr) {
        if (strcmp(force, "1sm") == 0) return tc::launch_sparse<128>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, stream);
        const bool whole = force[0] != 0 && force[strlen(force) - 1] == 'w';
        const int tail = whole ? 0 : 1;
        if (strncmp(force, "2sm128", 6) == 0)
            return tc::launch_sparse_pair<128>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, after_projection, tail, stream);
        if (strncmp(force, "2sm256", 6) == 0)
            return tc::launch_sparse_pair<256>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, after_projection, tail, stream);
        if (strncmp(force, "2sm240", 6) == 0)
            return tc::launch_sparse_pair<240>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, after_projection, tail, stream);
        if (strncmp(force, "2smtall", 7) == 0)
            return tc::launch_sparse_tall<240>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, after_projection, tail, stream);
        if (strcmp(force, "small") == 0) {
            if (M <= 16) return tc::launch_sparse_small<16>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, pdl, stream);
            if (M <= 32) return tc::launch_sparse_small<32>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, pdl, stream);
            if (M <= 64) return tc::launch_sparse_small<64>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, pdl, stream);
            return tc::launch_sparse_small<128>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, pdl, stream);
        }
    }
    // Up to 64 tokens the layer streams S: the split-K kernel.  Above, the
    // split-K kernel on 128-token tiles where it wins (few row tiles, one wave,
    // long K per CTA), else 2-SM pairs: on 256-row tiles with chunks of up to
    // 128 tokens (M < 192) or 240 tokens, or on 512-row tiles, which move X
    // into shared memory half as often but drain their accumulators between
    // chunks; each with the last round split among all pairs or dealt as whole
    // tiles.  The pair plan with the smallest estimated time of its slowest
    // pair is launched.
    if (M <= 16) return tc::launch_sparse_small<16>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, pdl, stream);
    if (M <= 32) return tc::launch_sparse_small<32>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, pdl, stream);
    if (M <= 64) return tc::launch_sparse_small<64>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, pdl, stream);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (tc::small_wins(M, d_out, d_in, sms))
        return tc::launch_sparse_small<128>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, pdl, stream);
    const tc::PlanChoice c = tc::choose_plan(M, d_out, d_in, r, sms, false);
    if (c.kind == 0)
        return tc::launch_sparse_pair<128>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, after_projection, c.tail, stream, c.chu);
    if (c.kind == 1)
        return tc::launch_sparse_pair<240>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, after_projection, c.tail, stream, c.chu);
    if (c.kind == 3)
        return tc::launch_sparse_pair<256>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, after_projection, c.tail, stream, c.chu);
    return tc::launch_sparse_tall<240>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, after_projection, c.tail, stream, c.chu);
}

cudaError_t launch_tc_forward_fused(const uint16_t *X, int64_t M, const uint16_t *vals, const uint8_t *meta,
                                    int64_t d_out, int64_t d_in, const uint16_t *U, const uint16_t *V, int64_t r,
                                    uint16_t *Y, uint8_t *ws, size_t ws_bytes, cudaStream_t stream) {
    if (M <= 0) return cudaSuccess;
    if (M > INT32_MAX || d_out > INT32_MAX || d_in > INT32_MAX) return cudaErrorInvalidValue;
    uint16_t *T16 = reinterpret_cast<uint16_t *>(ws);
    // Where the dispatch picks the 512-row kernel (or SLR_TC_KERNEL=
    // 2smtall[w|k] forces it), it runs with the workspace: T formed in its
    // projection phase (r <= 128), and its last round dealt as the plan says
    // (k: split along K).  Otherwise the projection kernel runs first.
    int tail = -1;   // >= 0: the 512-row kernel with this tail mode
    int chu = 0;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const char *force = getenv("SLR_TC_KERNEL");
    if (r > 0) {
        if (force != nullptr) {
            if (strncmp(force, "2smtall", 7) == 0) {
                const char last = force[strlen(force) - 1];
                tail = last == 'w' ? 0 : last == 'k' ? 2 : 1;
            }
        } else if (!tc::small_wins(M, d_out, d_in, sms)) {
            const tc::PlanChoice c = tc::choose_plan(M, d_out, d_in, r, sms, true);
            if (c.kind == 2) {
                tail = c.tail;
                chu = c.chu;
            }
        }
    }
    if (tail >= 0)
        return tc::launch_sparse_tall<240>(X, M, vals, meta, d_out, d_in, U, T16, r, Y, false, tail, stream, chu, V,
                                           ws, ws_bytes);
    cudaError_t err = cudaSuccess;
    if (r > 0) err = launch_tc_project(X, M, V, d_in, r, T16, false, stream);
    if (err == cudaSuccess) err = launch_tc_forward(X, M, vals, meta, d_out, d_in, U, r > 0 ? T16 : nullptr, r, Y, 1, stream);
    return err;
}

cudaError_t launch_tc_project(const uint16_t *X, int64_t M, const uint16_t *V, int64_t d_in, int64_t r,
                              uint16_t *T16, bool chained, cudaStream_t stream) {
    if (M <= 0 || r <= 0) return cudaSuccess;
    if (M > INT32_MAX || d_in > INT32_MAX || r > INT32_MAX) return cudaErrorInvalidValue;
    // Split-K cluster kernel; ranks above 256 fall back to the persistent
    // dense-mode kernel, which tiles r in 128-row steps.
    if (r <= 16) return tc::launch_project_splitk<16>(X, M, V, d_in, r, T16, chained, stream);
    if (r <= 64) return tc::launch_project_splitk<64>(X, M, V, d_in, r, T16, chained, stream);
    if (r <= 128) return tc::launch_project_splitk<128>(X, M, V, d_in, r, T16, chained, stream);
    if (r <= 256) return tc::launch_project_splitk<256>(X, M, V, d_in, r, T16, chained, stream);
    if (M >= 4096) return tc::launch_project<128>(X, M, V, d_in, r, T16, stream);
    if (M >= 1024) return tc::launch_project<64>(X, M, V, d_in, r, T16, stream);
    return tc::launch_project<32>(X, M, V, d_in, r, T16, stream);
}

namespace tc {
// Failure-detection self-test: one thread waits, with the kernels' bounded
// mbarrier wait, on a barrier whose phase nothing completes; when the limit
// expires it sets bit 12 of the error word and the kernel returns.
__global__ void wait_timeout_kernel(long long limit_cycles) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait_for(&bar, 0, limit_cycles)) atomicOr(&g_tc_error, 1u << 12);
}
}  // namespace tc

cudaError_t launch_wait_timeout_selftest(long long limit_cycles, cudaStream_t stream) {
    tc::wait_timeout_kernel<<<1, 32, 0, stream>>>(limit_cycles);
    return cudaGetLastError();
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

// decode28.cu -- small-M forward of a layer whose sparse term is stored in the
// dense 2:8 packing, on CUDA cores.
//
// Y = X S^T + T U^T (LoSparse, section 3.2: the sparse and low-rank terms
// side by side) with S in the 2:8 format (3BASiL summary page: 2:8 plus rank
// 64): two kept bf16 values and one index byte per group of eight weights,
// 0.625 B per weight against 1.125 B for the 2:4 packing.  With one or two
// tokens the layer is bound by the bytes of S, so this path moves about 45%
// fewer bytes than the 2:4 streaming path for the same layer.
//
// Two kernels.
//
// decode28_forward_kernel (the default; any d_in % 32 == 0): a warp owns RW
// rows and its lanes stream 16-byte chunks (4 groups) of each row straight
// from global memory into registers.
//
// decode28_ring_kernel (selectable, d_in % 128 == 0): persistent CTAs, two per SM, each
// owning a contiguous range of row blocks.  One producer lane streams the
// packed rows through a ring of shared-memory stages with untiled bulk
// copies (cp.async.bulk, completion counted on an mbarrier), so the bytes in
// flight come from the ring depth, not from registers.  A stage holds RPS
// rows x SEG columns.  Each of the 256 consumer threads owns one group of
// eight columns (a warp's X loads are 512 contiguous bytes) for RW rows, so
// every X load serves RW rows; per group three byte permutes gather the two
// X values the kept weights multiply.  After a row block's last stage the
// partial sums (rank-r term folded in) are reduced across the threads of
// the block, warp shuffles then shared memory, and Y is written once.
#include "common.cuh"
#include "tc_ptx.cuh"

namespace slr {

// Error word of the ring kernel's bounded waits (read by slr_check_kernel_error).
__device__ unsigned int g_d28_error = 0;

namespace {

constexpr int kWarps28 = 4;
constexpr int kUnrollChunks = 2;  // chunks in flight per lane and row

// One group of eight: kept values vv (idx0 low), index byte b, the eight X
// values of the group in xg.  Byte permutes pick positions idx & 3 from each
// half of xg, then each value from the half its index falls in.
__device__ __forceinline__ float group28_fma(uint32_t vv, uint32_t b, uint4 xg, float acc) {
    const uint32_t sel = ((b & 3u) | ((b & 0x18u) << 5)) * 0x22u + 0x1010u;
    const uint32_t lo = __byte_perm(xg.x, xg.y, sel), hi = __byte_perm(xg.z, xg.w, sel);
    const uint32_t fsel = (b & 4u) * 0x11u + (b & 0x20u) * 0x220u + 0x3210u;
    const uint32_t xs = __byte_perm(lo, hi, fsel);
    acc = fmaf(bf16lo_to_f32(vv), bf16lo_to_f32(xs), acc);
    acc = fmaf(bf16hi_to_f32(vv), bf16hi_to_f32(xs), acc);
    return acc;
}

// The three selectors of group28_fma for every index byte b = idx0 | idx1 << 3
// (only 64 values): low half = the in-half selector, high half = the final
// selector (byte permutes read the low 16 bits of their selector).
__device__ __forceinline__ uint32_t selector_entry(uint32_t b) {
    const uint32_t sel = ((b & 3u) | ((b & 0x18u) << 5)) * 0x22u + 0x1010u;
    const uint32_t fsel = (b & 4u) * 0x11u + (b & 0x20u) * 0x220u + 0x3210u;
    return (sel & 0xFFFFu) | (fsel << 16);
}

// group28_fma with the selectors looked up in the shared table `lut`.
__device__ __forceinline__ float group28_fma_lut(uint32_t vv, uint32_t e, uint4 xg, float acc) {
    const uint32_t lo = __byte_perm(xg.x, xg.y, e), hi = __byte_perm(xg.z, xg.w, e);
    const uint32_t xs = __byte_perm(lo, hi, e >> 16);
    acc = fmaf(bf16lo_to_f32(vv), bf16lo_to_f32(xs), acc);
    acc = fmaf(bf16hi_to_f32(vv), bf16hi_to_f32(xs), acc);
    return acc;
}

// 32 logical columns: v holds the 8 kept values, e the selector entries of the
// 4 groups, x the 32 X values of one token.
__device__ __forceinline__ float chunk28_fma(uint4 v, const uint32_t (&e)[4], const uint4 (&x)[4], float acc) {
    acc = group28_fma_lut(v.x, e[0], x[0], acc);
    acc = group28_fma_lut(v.y, e[1], x[1], acc);
    acc = group28_fma_lut(v.z, e[2], x[2], acc);
    acc = group28_fma_lut(v.w, e[3], x[3], acc);
    return acc;
}

template <int MT, int RW>
__global__ void __launch_bounds__(kWarps28 * 32) decode28_forward_kernel(
    const uint16_t *__restrict__ X, int64_t M, const uint16_t *__restrict__ vals8,
    const uint8_t *__restrict__ meta8, int64_t d_out, int64_t d_in, const uint16_t *__restrict__ U,
    const float *__restrict__ T32, int64_t r, uint16_t *__restrict__ Y) {
    __shared__ uint32_t lut[64];
    if (threadIdx.x < 64) lut[threadIdx.x] = selector_entry(threadIdx.x);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t m0 = (int64_t)blockIdx.y * MT;
    const int nt = (int)((M - m0) < MT ? (M - m0) : MT);
    const int64_t chunks = d_in / 32;
    const int64_t nwarps = (int64_t)gridDim.x * kWarps28;
    const uint16_t *xbase = X + m0 * d_in;
    const bool rk = 2 * lane < r;

    for (int64_t row0 = ((int64_t)blockIdx.x * kWarps28 + (threadIdx.x >> 5)) * RW; row0 < d_out;
         row0 += nwarps * RW) {
        float acc[RW][MT];
        float ur0[RW], ur1[RW];
#pragma unroll
        for (int q = 0; q < RW; ++q) {
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[q][t] = 0.f;
            ur0[q] = ur1[q] = 0.f;
            // U does not depend on the projection kernel: load it now (rank
            // pair 2l, 2l + 1 of row row0 + q; r % 8 == 0 keeps it aligned).
            if (rk && row0 + q < d_out) {
                const uint32_t u2 = __ldg(reinterpret_cast<const unsigned int *>(U + (row0 + q) * r) + lane);
                ur0[q] = bf16lo_to_f32(u2);
                ur1[q] = bf16hi_to_f32(u2);
            }
        }
        float2 tr[MT];
        bool t_loaded = false;
        auto load_t = [&]() {
            t_loaded = true;
            if (r > 0) asm volatile("griddepcontrol.wait;" ::: "memory");
#pragma unroll
            for (int t = 0; t < MT; ++t)
                tr[t] = (rk && t < nt) ? ld_dep_f2(T32 + (m0 + t) * r + 2 * lane)
                                       : make_float2(0.f, 0.f);
        };

        for (int64_t c0 = lane; c0 < chunks; c0 += 32 * kUnrollChunks) {
            uint4 v[kUnrollChunks][RW];
            uint32_t mm[kUnrollChunks][RW];
#pragma unroll
            for (int u = 0; u < kUnrollChunks; ++u) {
                const int64_t c = c0 + 32 * u;
#pragma unroll
                for (int q = 0; q < RW; ++q) {
                    if (c < chunks && row0 + q < d_out) {
                        v[u][q] = ld_stream_v4(vals8 + (row0 + q) * (d_in / 4) + c * 8);
                        mm[u][q] = __ldg(reinterpret_cast<const unsigned int *>(meta8 + (row0 + q) * (d_in / 8)) + c);
                    } else {
                        v[u][q] = make_uint4(0, 0, 0, 0);
                        mm[u][q] = 0x08080808u;  // valid index bytes for the zero padding
                    }
                }
            }
            if (!t_loaded) load_t();  // the first weight chunks are in flight
#pragma unroll
            for (int u = 0; u < kUnrollChunks; ++u) {
                const int64_t c = c0 + 32 * u;
                if (c < chunks) {
                    uint4 x[MT][4];
#pragma unroll
                    for (int t = 0; t < MT; ++t) {
                        const uint4 *xr = reinterpret_cast<const uint4 *>(xbase + t * d_in + c * 32);
#pragma unroll
                        for (int h = 0; h < 4; ++h) x[t][h] = t < nt ? __ldg(xr + h) : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int q = 0; q < RW; ++q) {
                        uint32_t e[4];
#pragma unroll
                        for (int g = 0; g < 4; ++g) e[g] = lut[(mm[u][q] >> (8 * g)) & 0x3Fu];
#pragma unroll
                        for (int t = 0; t < MT; ++t)
                            if (t < nt) acc[q][t] = chunk28_fma(v[u][q], e, x[t], acc[q][t]);
                    }
                }
            }
        }
        if (!t_loaded) load_t();  // lanes that had no weight chunk

        // Rank-r term in the same partial sums; ranks past 64 continue below.
#pragma unroll
        for (int q = 0; q < RW; ++q)
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[q][t] = fmaf(ur1[q], tr[t].y, fmaf(ur0[q], tr[t].x, acc[q][t]));
        for (int64_t k = lane + 64; k < r; k += 32) {
#pragma unroll
            for (int q = 0; q < RW; ++q) {
                if (row0 + q >= d_out) continue;
                const float u = __uint_as_float(
                    (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(U) + (row0 + q) * r + k) << 16);
#pragma unroll
                for (int t = 0; t < MT; ++t)
                    if (t < nt) acc[q][t] = fmaf(u, ld_dep_f32(T32 + (m0 + t) * r + k), acc[q][t]);
            }
        }

#pragma unroll
        for (int q = 0; q < RW; ++q)
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                float s = acc[q][t];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
                acc[q][t] = s;
            }
        // Lane q * MT + t writes (row row0 + q, token m0 + t).
        float out = 0.f;
#pragma unroll
        for (int q = 0; q < RW; ++q)
#pragma unroll
            for (int t = 0; t < MT; ++t)
                if (lane == q * MT + t) out = acc[q][t];
        const int q = lane / MT, t = lane % MT;
        if (lane < RW * MT && t < nt && row0 + q < d_out) Y[(m0 + t) * d_out + row0 + q] = f32_to_bf16_bits(out);
    }
}

// ----------------------------------------------------------------------------- ring kernel

struct Ring28 {
    int64_t M, d_out, d_in, r;
    int64_t n_rb;     // row blocks of rps rows
    int32_t seg;      // columns per stage (divides d_in, multiple of 128)
    int32_t nseg;     // d_in / seg
    int32_t gpr;      // groups of eight per row segment (seg / 8)
    int32_t tg;       // consumer threads per row slot (32..256, divides 256)
    int32_t rps;      // rows per stage: (256 / tg) * RW
    int32_t nst;      // ring stages
    int32_t slot;     // bytes per stage: rps * seg * 5 / 8 (multiple of 16)
};

constexpr int kCWarps = 8;                       // consumer warps
constexpr int kRingThreads = (kCWarps + 1) * 32;  // + one producer warp
constexpr int kRingCtasPerSm = 2;

template <int MT, int RW>
__global__ void __launch_bounds__(kRingThreads, kRingCtasPerSm) decode28_ring_kernel(
    const uint16_t *__restrict__ X, const uint16_t *__restrict__ vals8, const uint8_t *__restrict__ meta8,
    const uint16_t *__restrict__ U, const float *__restrict__ T32, uint16_t *__restrict__ Y, Ring28 p) {
    using namespace tc;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)p.nst * p.slot);
    uint64_t *empty = full + p.nst;
    float *red = reinterpret_cast<float *>(empty + p.nst);          // [kCWarps][RW * MT]
    volatile int *fail = reinterpret_cast<volatile int *>(red + kCWarps * RW * MT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < p.nst; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kCWarps);
        }
        *fail = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    __syncthreads();

    const int64_t m0 = (int64_t)blockIdx.y * MT;
    const int nt = (int)((p.M - m0) < MT ? (p.M - m0) : MT);
    const int64_t rb0 = (int64_t)blockIdx.x * p.n_rb / gridDim.x;
    const int64_t rb1 = ((int64_t)blockIdx.x + 1) * p.n_rb / gridDim.x;
    const int64_t n_stages = (rb1 - rb0) * p.nseg;
    const uint32_t row_vb = (uint32_t)p.seg / 2, row_mb = (uint32_t)p.seg / 8;

    if (warp == kCWarps) {
        // ---------------------------------------------------------------- producer
        if (elect_one()) {
            int64_t issued = 0;
            for (int64_t s = 0; s < n_stages; ++s) {
                const int slot = (int)(s % p.nst);
                const uint32_t ph = (uint32_t)((s / p.nst) & 1);
                if (!mbar_wait(&empty[slot], ph ^ 1u)) {
                    *fail = 1;
                    atomicOr(&g_d28_error, 1u);
                    break;
                }
                if (*fail) break;
                const int64_t row0 = (rb0 + s / p.nseg) * p.rps;
                const int64_t seg = s % p.nseg;
                const int64_t left = p.d_out - row0;
                const int rows = (int)(left < p.rps ? left : p.rps);
                mbar_expect_tx(&full[slot], (uint32_t)rows * (row_vb + row_mb));
                const uint32_t dv = smem_u32(ring + (size_t)slot * p.slot), dm = dv + (uint32_t)p.rps * row_vb;
                if (p.nseg == 1) {  // whole rows: the stage's rows are contiguous in both arrays
                    bulk_load(dv, vals8 + row0 * (p.d_in / 4), (uint32_t)rows * row_vb, &full[slot]);
                    bulk_load(dm, meta8 + row0 * (p.d_in / 8), (uint32_t)rows * row_mb, &full[slot]);
                } else {
                    for (int q = 0; q < rows; ++q) {
                        bulk_load(dv + q * row_vb, vals8 + (row0 + q) * (p.d_in / 4) + seg * (p.seg / 4), row_vb,
                                  &full[slot]);
                        bulk_load(dm + q * row_mb, meta8 + (row0 + q) * (p.d_in / 8) + seg * (p.seg / 8), row_mb,
                                  &full[slot]);
                    }
                }
                issued = s + 1;
            }
            // Copies still in flight land before the CTA may exit: wait (bounded)
            // for the last stages issued (earlier ones were consumed already).
            for (int64_t s = issued > p.nst ? issued - p.nst : 0; s < issued; ++s)
                if (!mbar_wait(&full[s % p.nst], (uint32_t)((s / p.nst) & 1))) atomicOr(&g_d28_error, 4u);
        }
        return;  // the producer warp takes no part in the consumers' named barrier
    }

    // -------------------------------------------------------------------- consumers
    const int ct = threadIdx.x;              // 0..255
    const int rs = ct / p.tg, gi = ct % p.tg;  // row slot, group index
    const bool rk = 2 * gi < p.r;            // this thread's rank pair (2 gi, 2 gi + 1)
    float2 tr[MT];
    bool t_ready = false;
    bool ok = true;
    int64_t s = 0;
    for (int64_t rb = rb0; rb < rb1; ++rb) {
        const int64_t row0 = rb * p.rps + (int64_t)rs * RW;  // this thread's first row
        float acc[RW][MT];
        float ur0[RW], ur1[RW];
#pragma unroll
        for (int j = 0; j < RW; ++j) {
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[j][t] = 0.f;
            ur0[j] = ur1[j] = 0.f;
            if (rk && row0 + j < p.d_out) {
                const uint32_t u2 = __ldg(reinterpret_cast<const unsigned int *>(U + (row0 + j) * p.r) + gi);
                ur0[j] = bf16lo_to_f32(u2);
                ur1[j] = bf16hi_to_f32(u2);
            }
        }
        for (int seg = 0; seg < p.nseg; ++seg, ++s) {
            const int slot = (int)(s % p.nst);
            if (ok && !*fail && !mbar_wait(&full[slot], (uint32_t)((s / p.nst) & 1))) {
                *fail = 1;
                atomicOr(&g_d28_error, 2u);
            }
            ok = ok && !*fail;
            if (ok) {
                const uint32_t *sv = reinterpret_cast<const uint32_t *>(ring + (size_t)slot * p.slot);
                const uint8_t *sm = ring + (size_t)slot * p.slot + (size_t)p.rps * row_vb;
                const uint16_t *xs = X + m0 * p.d_in + (int64_t)seg * p.seg;
                for (int g = gi; g < p.gpr; g += p.tg) {
                    uint32_t vv[RW], bb[RW];
#pragma unroll
                    for (int j = 0; j < RW; ++j) {
                        const int q = rs * RW + j;
                        vv[j] = sv[q * p.gpr + g];
                        bb[j] = sm[q * p.gpr + g];
                    }
#pragma unroll
                    for (int t = 0; t < MT; ++t) {
                        if (t < nt) {
                            const uint4 xg = __ldg(reinterpret_cast<const uint4 *>(xs + t * p.d_in + 8 * g));
#pragma unroll
                            for (int j = 0; j < RW; ++j) acc[j][t] = group28_fma(vv[j], bb[j], xg, acc[j][t]);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
        // Rank-r term: T comes from the projection kernel, which may still run
        // when this grid starts (programmatic dependent launch).
        if (!t_ready) {
            t_ready = true;
            if (p.r > 0) asm volatile("griddepcontrol.wait;" ::: "memory");
#pragma unroll
            for (int t = 0; t < MT; ++t)
                tr[t] = (rk && t < nt) ? ld_dep_f2(T32 + (m0 + t) * p.r + 2 * gi)
                                       : make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < RW; ++j)
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[j][t] = fmaf(ur1[j], tr[t].y, fmaf(ur0[j], tr[t].x, acc[j][t]));
        for (int64_t k = 2 * (gi + (int64_t)p.tg); k < p.r; k += 2 * (int64_t)p.tg) {  // rank > 2 tg
#pragma unroll
            for (int j = 0; j < RW; ++j) {
                if (row0 + j >= p.d_out) continue;
                const uint32_t u2 = __ldg(reinterpret_cast<const unsigned int *>(U + (row0 + j) * p.r + k));
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                    if (t >= nt) continue;
                    const float2 tk = ld_dep_f2(T32 + (m0 + t) * p.r + k);
                    acc[j][t] = fmaf(bf16hi_to_f32(u2), tk.y, fmaf(bf16lo_to_f32(u2), tk.x, acc[j][t]));
                }
            }
        }
        // Reduce over the tg threads of the row slot: shuffles, then the
        // slot's warps through shared memory in warp order.
#pragma unroll
        for (int j = 0; j < RW; ++j)
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                float v = acc[j][t];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                if (lane == 0) red[warp * RW * MT + j * MT + t] = v;
            }
        named_bar_sync(1, kCWarps * 32);
        if (ct < p.rps * MT && ok) {
            const int q = ct / MT, t = ct % MT;
            const int slot_of_q = q / RW, j = q % RW;
            const int w0 = slot_of_q * (p.tg / 32), w1 = w0 + p.tg / 32;
            float v = 0.f;
            for (int w = w0; w < w1; ++w) v += red[w * RW * MT + j * MT + t];
            const int64_t row = rb * p.rps + q;
            if (row < p.d_out && t < nt) Y[(m0 + t) * p.d_out + row] = f32_to_bf16_bits(v);
        }
        named_bar_sync(1, kCWarps * 32);
    }
}

template <int MT, int RW>
cudaError_t launch28(const uint16_t *X, int64_t M, const uint16_t *vals8, const uint8_t *meta8, int64_t d_out,
                     int64_t d_in, const uint16_t *U, const float *T32, int64_t r, uint16_t *Y,
                     bool after_projection, cudaStream_t stream) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // Resident CTAs per SM, asked once per instantiation (a property of the
    // compiled kernel and the sm_100 architecture, the same on every B200).
    static int per_sm = 0;
    if (per_sm == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode28_forward_kernel<MT, RW>, kWarps28 * 32, 0) !=
                cudaSuccess ||
            n < 1)
            n = 1;
        per_sm = n;
    }
    // Row groups of RW rows, one per warp: as many warps as there are groups,
    // up to the resident capacity; with more groups, the fewest whole rounds
    // spread evenly (every warp takes the same number of groups, +-1).
    const int64_t tasks = (d_out + RW - 1) / RW;
    const int64_t capacity = (int64_t)sms * per_sm * kWarps28;
    const int64_t rounds = (tasks + capacity - 1) / capacity;
    const int64_t warps = (tasks + rounds - 1) / rounds;
    const int64_t blocks = (warps + kWarps28 - 1) / kWarps28;
    const int64_t tblocks = (M + MT - 1) / MT;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks, (unsigned)tblocks);
    cfg.blockDim = dim3(kWarps28 * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_projection ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode28_forward_kernel<MT, RW>, X, M, vals8, meta8, d_out, d_in, U, T32, r, Y);
}

// Rows per warp: 4 shares each X load among four rows (the X bytes a warp
// reads from L1 per weight byte fall from 3.2 to 0.8 per token); fewer when
// the layer has too few rows to fill the GPU with groups of four.
int rows_per_warp(int64_t d_out) {
    const char *env = getenv("SLR_DECODE28_RW");
    if (env != nullptr && (env[0] == '1' || env[0] == '2' || env[0] == '4')) return env[0] - '0';
    if (d_out >= 4 * 148 * 16) return 4;
    if (d_out >= 2 * 148 * 16) return 2;
    return 1;
}

template <int MT>
cudaError_t launch_mt28(const uint16_t *X, int64_t M, const uint16_t *vals8, const uint8_t *meta8, int64_t d_out,
                        int64_t d_in, const uint16_t *U, const float *T32, int64_t r, uint16_t *Y,
                        bool after_projection, cudaStream_t stream) {
    switch (rows_per_warp(d_out)) {
        case 4: return launch28<MT, 4>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
        case 2: return launch28<MT, 2>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
        default: return launch28<MT, 1>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
    }
}

// Ring kernel launch: stage geometry from d_in, one or two CTAs per SM.
template <int MT, int RW>
cudaError_t launch_ring28(const uint16_t *X, int64_t M, const uint16_t *vals8, const uint8_t *meta8, int64_t d_out,
                          int64_t d_in, const uint16_t *U, const float *T32, int64_t r, uint16_t *Y,
                          bool after_projection, cudaStream_t stream) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    Ring28 p{};
    p.M = M;
    p.d_out = d_out;
    p.d_in = d_in;
    p.r = r;
    // Whole rows up to 8192 columns (two copies per stage); wider rows in
    // equal segments of at most 8192 columns (two copies per row and stage).
    int64_t seg = d_in;
    if (seg > 8192) {
        seg = 128;
        for (int64_t c = 8192; c >= 128; c -= 128)
            if (d_in % c == 0) {
                seg = c;
                break;
            }
    }
    p.seg = (int32_t)seg;
    p.nseg = (int32_t)(d_in / seg);
    p.gpr = (int32_t)(seg / 8);
    int tg = 256;
    while (tg > 32 && tg > p.gpr) tg /= 2;
    p.tg = tg;
    p.rps = (256 / tg) * RW;
    p.slot = (int32_t)(p.rps * seg * 5 / 8);
    p.n_rb = (d_out + p.rps - 1) / p.rps;
    const int64_t ring_budget = 100 * 1024;
    int64_t nst = ring_budget / p.slot;
    nst = nst < 2 ? 2 : (nst > 16 ? 16 : nst);
    p.nst = (int32_t)nst;
    const size_t smem = (size_t)p.nst * p.slot + 2 * (size_t)p.nst * sizeof(uint64_t) +
                        (size_t)kCWarps * RW * MT * sizeof(float) + 16;
    // Set on every call: the attribute belongs to the current device's copy of the kernel.
    const cudaError_t e = cudaFuncSetAttribute(decode28_ring_kernel<MT, RW>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int64_t grid = (int64_t)sms * kRingCtasPerSm;
    if (grid > p.n_rb) grid = p.n_rb;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, (unsigned)((M + MT - 1) / MT));
    cfg.blockDim = dim3(kRingThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_projection ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode28_ring_kernel<MT, RW>, X, vals8, meta8, U, T32, Y, p);
}

template <int MT>
cudaError_t launch_ring_mt28(const uint16_t *X, int64_t M, const uint16_t *vals8, const uint8_t *meta8,
                             int64_t d_out, int64_t d_in, const uint16_t *U, const float *T32, int64_t r,
                             uint16_t *Y, bool after_projection, cudaStream_t stream) {
    const char *env = getenv("SLR_DECODE28_RW");
    const int rw = (env != nullptr && (env[0] == '1' || env[0] == '2')) ? env[0] - '0' : 4;
    if (rw == 1) return launch_ring28<MT, 1>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
    if (rw == 2) return launch_ring28<MT, 2>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
    return launch_ring28<MT, 4>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
}

// The register kernel is the default: measured on the 70B up projection at
// M = 1 it takes 47.6 us against 86-90 us for the ring kernel, whose
// consumers issue ~44 instructions per group and row (index arithmetic,
// three shared-memory loads, selector arithmetic) and stall on the per-row-
// block barriers.  The ring kernel stays selectable (SLR_DECODE28_KERNEL=ring)
// and tested.
bool use_ring(int64_t d_in) {
    const char *env = getenv("SLR_DECODE28_KERNEL");
    return env != nullptr && env[0] == 'r' && env[1] == 'i' && d_in % 128 == 0;  // "ring"
}

}  // namespace

cudaError_t read_and_clear_decode28_error(unsigned *code) {
    unsigned v = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_d28_error, sizeof v);
    if (err != cudaSuccess) return err;
    if (v != 0) {
        const unsigned zero = 0;
        err = cudaMemcpyToSymbol(g_d28_error, &zero, sizeof zero);
    }
    *code = v;
    return err;
}

cudaError_t launch_decode28_forward(const uint16_t *X, int64_t M, const uint16_t *vals8, const uint8_t *meta8,
                                    int64_t d_out, int64_t d_in, const uint16_t *U, const float *T32, int64_t r,
                                    uint16_t *Y, bool after_projection, cudaStream_t stream) {
    if (use_ring(d_in)) {
        if (M == 1)
            return launch_ring_mt28<1>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
        if (M == 2)
            return launch_ring_mt28<2>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
        return launch_ring_mt28<4>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
    }
    if (M == 1) return launch_mt28<1>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
    if (M == 2) return launch_mt28<2>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
    return launch_mt28<4>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
}

}  // namespace slr

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
// A warp owns RW output rows at a time.  Lane l streams 16-byte chunks of
// each row's packed values (8 kept values = 4 groups = 32 logical columns)
// with non-allocating 128-bit loads plus the chunk's 4 index bytes, and loads
// the matching 64 bytes of every token's X once for the RW rows (X stays in
// L1/L2; it is a few KB per token).  Per group, three byte permutes gather
// the two X values its kept weights multiply.  The rank-r term is folded into
// the same per-lane partial sums before one warp-shuffle reduction per
// (row, token), so Y is written exactly once.  Token blocks of MT tokens go to
// blockIdx.y.
#include "common.cuh"

namespace slr {
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

// 32 logical columns: v holds the 8 kept values, m32 the 4 index bytes, x the
// 32 X values of one token.
__device__ __forceinline__ float chunk28_fma(uint4 v, uint32_t m32, const uint4 (&x)[4], float acc) {
    acc = group28_fma(v.x, m32 & 0xFFu, x[0], acc);
    acc = group28_fma(v.y, (m32 >> 8) & 0xFFu, x[1], acc);
    acc = group28_fma(v.z, (m32 >> 16) & 0xFFu, x[2], acc);
    acc = group28_fma(v.w, m32 >> 24, x[3], acc);
    return acc;
}

template <int MT, int RW>
__global__ void __launch_bounds__(kWarps28 * 32) decode28_forward_kernel(
    const uint16_t *__restrict__ X, int64_t M, const uint16_t *__restrict__ vals8,
    const uint8_t *__restrict__ meta8, int64_t d_out, int64_t d_in, const uint16_t *__restrict__ U,
    const float *__restrict__ T32, int64_t r, uint16_t *__restrict__ Y) {
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
                tr[t] = (rk && t < nt) ? __ldg(reinterpret_cast<const float2 *>(T32 + (m0 + t) * r) + lane)
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
#pragma unroll
                    for (int t = 0; t < MT; ++t) {
                        if (t < nt) {
                            const uint4 *xr = reinterpret_cast<const uint4 *>(xbase + t * d_in + c * 32);
                            const uint4 x[4] = {__ldg(xr), __ldg(xr + 1), __ldg(xr + 2), __ldg(xr + 3)};
#pragma unroll
                            for (int q = 0; q < RW; ++q) acc[q][t] = chunk28_fma(v[u][q], mm[u][q], x, acc[q][t]);
                        }
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
                    if (t < nt) acc[q][t] = fmaf(u, __ldg(T32 + (m0 + t) * r + k), acc[q][t]);
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

template <int MT, int RW>
cudaError_t launch28(const uint16_t *X, int64_t M, const uint16_t *vals8, const uint8_t *meta8, int64_t d_out,
                     int64_t d_in, const uint16_t *U, const float *T32, int64_t r, uint16_t *Y,
                     bool after_projection, cudaStream_t stream) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    static int per_sm = 0;  // resident CTAs per SM, asked once per instantiation
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

}  // namespace

cudaError_t launch_decode28_forward(const uint16_t *X, int64_t M, const uint16_t *vals8, const uint8_t *meta8,
                                    int64_t d_out, int64_t d_in, const uint16_t *U, const float *T32, int64_t r,
                                    uint16_t *Y, bool after_projection, cudaStream_t stream) {
    if (M == 1) return launch_mt28<1>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
    if (M == 2) return launch_mt28<2>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
    return launch_mt28<4>(X, M, vals8, meta8, d_out, d_in, U, T32, r, Y, after_projection, stream);
}

}  // namespace slr

// decode.cu -- small-M (decode) forward on CUDA cores.
//
// Computes Y = X S^T + T U^T (LoSparse, section 3.2: the sparse and the
// low-rank term of the compressed layer evaluated side by side), where S is
// the packed 2:4 matrix and T = X V^T was produced beforehand in fp32.
//
// With a handful of tokens the layer is bound by the bytes of S: 2 B of value
// plus 0.25 B of metadata per kept weight.  Each warp owns one output row at a
// time; lane l streams 16-byte chunks of the row's packed values (8 kept
// weights = 16 logical columns) with non-allocating 128-bit loads, plus the
// chunk's 2 metadata bytes, and multiplies them with the matching 16 columns of
// every token of X (X stays in L1/L2; it is a few KB per token).  The rank-r
// term is folded into the same per-lane partial sums (lanes split the r
// products U[i, k] T[m, k]) before one warp-shuffle reduction per token, so Y
// is written exactly once.  Token blocks of MT tokens go to blockIdx.y.
#include "common.cuh"

namespace slr {
namespace {

constexpr int kWarps = 4;
constexpr int kBlocksPerSm = 7;
// 16-byte chunks in flight per lane: a whole 4096-wide row per round trip for
// one or two tokens; fewer with more tokens (their accumulators and X loads
// need the registers).
template <int MT>
__host__ __device__ constexpr int unroll_for() { return MT == 1 ? 8 : 4; }

// One group of four: kept values (low = lower index) in vv, nibble nib, the
// four X values of the group in x01 (elements 0,1) and x23 (elements 2,3).
// One byte permute gathers the two X values the kept weights multiply (byte
// selectors 2*idx, 2*idx+1 for each index); bf16 -> fp32 is a 16-bit shift
// or a mask.
__device__ __forceinline__ float group_fma(uint32_t vv, uint32_t nib, uint32_t x01, uint32_t x23, float acc) {
    const uint32_t sel = ((nib & 3u) | ((nib & 0xCu) << 6)) * 0x22u + 0x1010u;
    const uint32_t xs = __byte_perm(x01, x23, sel);
    acc = fmaf(bf16lo_to_f32(vv), bf16lo_to_f32(xs), acc);
    acc = fmaf(bf16hi_to_f32(vv), bf16hi_to_f32(xs), acc);
    return acc;
}

// 16 logical columns: 4 groups.  v holds the 8 kept values, m16 the 4 nibbles,
// xa/xb the 16 X values.
__device__ __forceinline__ float chunk_fma(uint4 v, uint32_t m16, uint4 xa, uint4 xb, float acc) {
    acc = group_fma(v.x, m16 & 0xFu, xa.x, xa.y, acc);
    acc = group_fma(v.y, (m16 >> 4) & 0xFu, xa.z, xa.w, acc);
    acc = group_fma(v.z, (m16 >> 8) & 0xFu, xb.x, xb.y, acc);
    acc = group_fma(v.w, (m16 >> 12) & 0xFu, xb.z, xb.w, acc);
    return acc;
}

// 7 resident CTAs of 4 warps per SM (<= 73 registers): 148 x 7 x 4 warps cover
// the 4096 rows of a Llama-3-8B projection, one row per warp, in one wave.
template <int MT>
__global__ void __launch_bounds__(kWarps * 32, kBlocksPerSm) decode_forward_kernel(
    const uint16_t *__restrict__ X, int64_t M, const uint16_t *__restrict__ vals,
    const uint8_t *__restrict__ meta, int64_t d_out, int64_t d_in, const uint16_t *__restrict__ U,
    const float *__restrict__ T32, int64_t r, uint16_t *__restrict__ Y) {
    const int lane = threadIdx.x & 31;
    const int64_t m0 = (int64_t)blockIdx.y * MT;
    const int nt = (int)((M - m0) < MT ? (M - m0) : MT);
    const int64_t chunks = d_in / 16;
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    const uint16_t *xbase = X + m0 * d_in;
    constexpr int kUnroll = unroll_for<MT>();

    for (int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); row < d_out; row += nwarps) {
        float acc[MT];
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[t] = 0.f;
        const uint16_t *vrow = vals + row * (d_in / 2);
        const uint8_t *mrow = meta + row * (d_in / 8);
        // The rank-r operands of this row: U now (it does not depend on the
        // projection), T after griddepcontrol.wait once the first weight
        // chunks are in flight, so neither load adds a round trip at the end.
        // Lane l holds rank pair k = 2l, 2l + 1 (r % 8 == 0, so the pair is
        // 4-byte aligned in U and 8-byte aligned in T): one load each.
        const bool rk = 2 * lane < r;
        float ur0 = 0.f, ur1 = 0.f;
        if (rk) {
            const uint32_t u2 = __ldg(reinterpret_cast<const unsigned int *>(U + row * r) + lane);
            ur0 = bf16lo_to_f32(u2);
            ur1 = bf16hi_to_f32(u2);
        }
        float2 tr[MT];
        bool t_loaded = false;
        auto load_t = [&]() {
            t_loaded = true;
            if (r > 0) asm volatile("griddepcontrol.wait;" ::: "memory");
#pragma unroll
            for (int t = 0; t < MT; ++t)
                tr[t] = (rk && t < nt) ? ld_dep_f2(T32 + (m0 + t) * r + 2 * lane) : make_float2(0.f, 0.f);
        };

        for (int64_t c0 = lane; c0 < chunks; c0 += 32 * kUnroll) {
            uint4 v[kUnroll];
            uint32_t mm[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t c = c0 + 32 * u;
                if (c < chunks) {
                    v[u] = ld_stream_v4(vrow + c * 8);
                    mm[u] = __ldg(reinterpret_cast<const unsigned short *>(mrow + 2 * c));
                } else {
                    v[u] = make_uint4(0, 0, 0, 0);
                    mm[u] = 0x4444u;  // valid nibbles for the zero padding
                }
            }
            if (!t_loaded) load_t();   // the first weight chunks are in flight
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t c = c0 + 32 * u;
                if (c < chunks) {
#pragma unroll
                    for (int t = 0; t < MT; ++t) {
                        if (t < nt) {
                            const uint4 *xr = reinterpret_cast<const uint4 *>(xbase + t * d_in + c * 16);
                            acc[t] = chunk_fma(v[u], mm[u], __ldg(xr), __ldg(xr + 1), acc[t]);
                        }
                    }
                }
            }
        }

        if (!t_loaded) load_t();   // lanes that had no weight chunk
        // Rank-r term: lanes split k, products land in the same partial sums.
        // T comes from the projection kernel, which may still be running when
        // this kernel starts (programmatic dependent launch); it is read after
        // griddepcontrol.wait, with ordered L2 loads (a read-only __ldg load
        // counts as invariant and may be moved above the wait).  Ranks past
        // 64 continue here.
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[t] = fmaf(ur1, tr[t].y, fmaf(ur0, tr[t].x, acc[t]));
        for (int64_t k = lane + 64; k < r; k += 32) {
            const float u = __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(U) + row * r + k) << 16);
#pragma unroll
            for (int t = 0; t < MT; ++t)
                if (t < nt) acc[t] = fmaf(u, ld_dep_f32(T32 + (m0 + t) * r + k), acc[t]);
        }

#pragma unroll
        for (int t = 0; t < MT; ++t) {
            float s = acc[t];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
            acc[t] = s;
        }
        if (lane < nt) {
            float s = acc[0];
#pragma unroll
            for (int t = 1; t < MT; ++t)
                if (lane == t) s = acc[t];
            Y[(m0 + lane) * d_out + row] = f32_to_bf16_bits(s);
        }
    }
}

template <int MT>
cudaError_t launch_mt(const uint16_t *X, int64_t M, const uint16_t *vals, const uint8_t *meta, int64_t d_out,
                      int64_t d_in, const uint16_t *U, const float *T32, int64_t r, uint16_t *Y,
                      bool after_projection, cudaStream_t stream) {
    const int64_t tblocks = (M + MT - 1) / MT;
    if (tblocks > 65535) return cudaErrorInvalidConfiguration;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (d_out + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)sms * kBlocksPerSm;
    if (blocks > cap) blocks = cap;
    // Directly after the projection kernel on the same stream it is launched
    // as a programmatic dependent: it may start streaming S before T is
    // complete (it waits before reading T).  Otherwise it is an ordinary
    // launch (a programmatic launch would also overlap an unrelated
    // preceding kernel, e.g. the producer of X).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks, (unsigned)tblocks);
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_projection ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_forward_kernel<MT>, X, M, vals, meta, d_out, d_in, U, T32, r, Y);
}

}  // namespace

bool decode_chain_ok(int64_t, int64_t) {
    // Seven CTAs of this kernel fill an SM's registers, so a following launch
    // could not start early anyway: chained calls run as ordinary ones here.
    return false;
}

cudaError_t launch_decode_forward(const uint16_t *X, int64_t M, const uint16_t *vals, const uint8_t *meta,
                                  int64_t d_out, int64_t d_in, const uint16_t *U, const float *T32, int64_t r,
                                  uint16_t *Y, int pdl_mode, cudaStream_t stream) {
    const bool pdl = pdl_mode != 0 && r > 0;
    if (M <= 1) return launch_mt<1>(X, M, vals, meta, d_out, d_in, U, T32, r, Y, pdl, stream);
    if (M <= 2) return launch_mt<2>(X, M, vals, meta, d_out, d_in, U, T32, r, Y, pdl, stream);
    if (M <= 4) return launch_mt<4>(X, M, vals, meta, d_out, d_in, U, T32, r, Y, pdl, stream);
    return launch_mt<8>(X, M, vals, meta, d_out, d_in, U, T32, r, Y, pdl, stream);
}

}  // namespace slr

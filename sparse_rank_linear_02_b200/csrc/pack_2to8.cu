// pack_2to8.cu -- 2:8 projection by magnitude, packed densely and/or in the
// 2:4 format.
//
// The 2:8 configuration (3BASiL summary page, "Faster compression and gains
// that survive LoRA": 2:8 sparse plus rank 64) keeps at most two nonzeros in
// every aligned run of eight weights along d_in.  The projection is the same
// hard-thresholding as the 2:4 one (HASSLE-free, section 4.1.1): the two
// largest magnitude keys of each group of eight (bf16 bits without the sign,
// compared as integers), ties to the lower index.
//
// Outputs, each optional:
//  * the dense 2:8 packing: two kept values per group of eight (4 B) and one
//    metadata byte idx0 | idx1 << 3 -- 0.625 B per weight, read by the 2:8
//    streaming forward;
//  * the 2:4 packing of the projected matrix (every half-group of four holds
//    at most two kept positions), bit-identical to packing the unpacked 2:8
//    matrix with the 2:4 rule, for the 2:4 tensor-core forward.
//
// Work unit = one group of eight (16 bytes of W): one 16-byte load, then a
// 4-byte + 1-byte store (2:8) and an 8-byte + 1-byte store (2:4); a warp's
// accesses are contiguous.  HBM-bound at 2 B read + 0.625 B (+ 1.125 B)
// written per weight.
#include "common.cuh"

namespace slr {
namespace {

// Top two of eight keys e_p = (magnitude bits << 3) | (7 - p) (all distinct,
// so a larger magnitude wins and equal magnitudes prefer the lower position):
// top-two of pairs, of quadruples, of the eight, each merge taking
//   first = max(f_a, f_b),  second = max(min(f_a, f_b), max(s_a, s_b)).
// Returns idx0 | idx1 << 3 with idx0 < idx1.
__device__ __forceinline__ uint32_t top_two_of_eight(uint4 w) {
    const uint32_t e0 = ((w.x & 0x7FFFu) << 3) | 7u, e1 = ((w.x >> 13) & 0x3FFF8u) | 6u;
    const uint32_t e2 = ((w.y & 0x7FFFu) << 3) | 5u, e3 = ((w.y >> 13) & 0x3FFF8u) | 4u;
    const uint32_t e4 = ((w.z & 0x7FFFu) << 3) | 3u, e5 = ((w.z >> 13) & 0x3FFF8u) | 2u;
    const uint32_t e6 = ((w.w & 0x7FFFu) << 3) | 1u, e7 = (w.w >> 13) & 0x3FFF8u;
    const uint32_t f01 = max(e0, e1), s01 = min(e0, e1), f23 = max(e2, e3), s23 = min(e2, e3);
    const uint32_t f45 = max(e4, e5), s45 = min(e4, e5), f67 = max(e6, e7), s67 = min(e6, e7);
    const uint32_t f03 = max(f01, f23), s03 = max(min(f01, f23), max(s01, s23));
    const uint32_t f47 = max(f45, f67), s47 = max(min(f45, f67), max(s45, s67));
    const uint32_t first = max(f03, f47), second = max(min(f03, f47), max(s03, s47));
    const uint32_t pa = 7u - (first & 7u), pb = 7u - (second & 7u);
    return min(pa, pb) | (max(pa, pb) << 3);
}

// The two kept bf16 values (idx0 low, idx1 high) of a group of eight held in
// w: one byte permute picks positions idx & 3 from the low pair of words
// (positions 0..3) and from the high pair (4..7); a third takes each value
// from the pair its index falls in.
__device__ __forceinline__ uint32_t gather_two_of_eight(uint4 w, uint32_t b) {
    const uint32_t sel = ((b & 3u) | ((b & 0x18u) << 5)) * 0x22u + 0x1010u;
    const uint32_t lo = __byte_perm(w.x, w.y, sel), hi = __byte_perm(w.z, w.w, sel);
    const uint32_t fsel = (b & 4u) * 0x11u + (b & 0x20u) * 0x220u + 0x3210u;
    return __byte_perm(lo, hi, fsel);
}

// The 2:4 choice on one half-group of four (words w01, w23) in which the
// positions not kept by the 2:8 rule already hold +0: as the 2:4 projection,
// keys (magnitude << 2) | (3 - position), the two largest kept.  Returns the
// nibble; *kept receives the two kept values.
__device__ __forceinline__ uint32_t half_as_2to4(uint32_t w01, uint32_t w23, uint32_t *kept) {
    const uint32_t e0 = ((w01 & 0x7FFFu) << 2) | 3u, e1 = ((w01 >> 14) & 0x1FFFCu) | 2u;
    const uint32_t e2 = ((w23 & 0x7FFFu) << 2) | 1u, e3 = (w23 >> 14) & 0x1FFFCu;
    const uint32_t m01 = max(e0, e1), n01 = min(e0, e1), m23 = max(e2, e3), n23 = min(e2, e3);
    const uint32_t first = max(m01, m23), second = max(min(m01, m23), max(n01, n23));
    const uint32_t pa = 3u - (first & 3u), pb = 3u - (second & 3u);
    const uint32_t i0 = min(pa, pb), i1 = max(pa, pb);
    const uint32_t sel = (i0 * 2u) * 0x11u + 0x10u + (((i1 * 2u) * 0x11u + 0x10u) << 8);
    *kept = __byte_perm(w01, w23, sel);
    return i0 | (i1 << 2);
}

// Zero (to +0) every bf16 of w outside positions idx0, idx1 of the byte b.
__device__ __forceinline__ uint4 mask_to_kept(uint4 w, uint32_t b) {
    const uint32_t keep = (1u << (b & 7u)) | (1u << ((b >> 3) & 7u));
    auto half_mask = [&](int p) -> uint32_t {
        return ((keep >> p) & 1u ? 0x0000FFFFu : 0u) | ((keep >> (p + 1)) & 1u ? 0xFFFF0000u : 0u);
    };
    return make_uint4(w.x & half_mask(0), w.y & half_mask(2), w.z & half_mask(4), w.w & half_mask(6));
}

struct Out28 {
    uint16_t *vals8;  // [d_out, d_in/4] or null
    uint8_t *meta8;   // [d_out, d_in/8] or null
    uint16_t *vals4;  // [d_out, d_in/2] or null
    uint8_t *meta4;   // [d_out, d_in/8] or null
};

__device__ __forceinline__ void emit_group(uint4 w, int64_t row, int64_t g, int64_t d_in, const Out28 &o) {
    const uint32_t b = top_two_of_eight(w);
    if (o.vals8 != nullptr) {
        reinterpret_cast<uint32_t *>(o.vals8 + row * (d_in / 4))[g] = gather_two_of_eight(w, b);
        o.meta8[row * (d_in / 8) + g] = (uint8_t)b;
    }
    if (o.vals4 != nullptr) {
        const uint4 s = mask_to_kept(w, b);
        uint32_t k0, k1;
        const uint32_t n0 = half_as_2to4(s.x, s.y, &k0);
        const uint32_t n1 = half_as_2to4(s.z, s.w, &k1);
        reinterpret_cast<uint2 *>(o.vals4 + row * (d_in / 2))[g] = make_uint2(k0, k1);
        o.meta4[row * (d_in / 8) + g] = (uint8_t)(n0 | (n1 << 4));
    }
}

constexpr int kUnroll28 = 4;

// Vectorised path: W 16-byte aligned with ldw % 8 == 0 (16-byte rows), the
// output pointers aligned for their 4- and 8-byte stores.  Rows over the
// grid; the CTA's threads sweep a row's groups, kUnroll28 loads in flight.
__global__ void __launch_bounds__(256) pack_2to8_v_kernel(const uint16_t *__restrict__ W, int64_t d_out,
                                                          int64_t d_in, int64_t ldw, Out28 o) {
    const int groups = (int)(d_in / 8);
    for (int64_t row = blockIdx.x; row < d_out; row += gridDim.x) {
        const uint16_t *wrow = W + row * ldw;
        for (int g0 = threadIdx.x; g0 < groups; g0 += kUnroll28 * blockDim.x) {
            uint4 w[kUnroll28];
#pragma unroll
            for (int i = 0; i < kUnroll28; ++i) {
                const int g = g0 + i * blockDim.x;
                if (g < groups) w[i] = ld_stream_v4(wrow + (int64_t)g * 8);
            }
#pragma unroll
            for (int i = 0; i < kUnroll28; ++i) {
                const int g = g0 + i * blockDim.x;
                if (g < groups) emit_group(w[i], row, g, d_in, o);
            }
        }
    }
}

// General path: any W alignment or stride (the outputs must still be aligned
// for their 4- and 8-byte stores); one group per thread, scalar loads.
__global__ void __launch_bounds__(256) pack_2to8_any_kernel(const uint16_t *__restrict__ W, int64_t d_out,
                                                            int64_t d_in, int64_t ldw, Out28 o) {
    const int64_t groups = d_in / 8;
    const int64_t total = d_out * groups;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total;
         u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = u / groups, g = u - row * groups;
        const uint16_t *src = W + row * ldw + 8 * g;
        uint4 w;
        w.x = (uint32_t)src[0] | ((uint32_t)src[1] << 16);
        w.y = (uint32_t)src[2] | ((uint32_t)src[3] << 16);
        w.z = (uint32_t)src[4] | ((uint32_t)src[5] << 16);
        w.w = (uint32_t)src[6] | ((uint32_t)src[7] << 16);
        emit_group(w, row, g, d_in, o);
    }
}

}  // namespace

cudaError_t launch_pack_2to8(const uint16_t *W, int64_t d_out, int64_t d_in, int64_t ldw, uint16_t *vals8,
                             uint8_t *meta8, uint16_t *vals4, uint8_t *meta4, cudaStream_t stream) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const Out28 o{vals8, meta8, vals4, meta4};
    const bool v = (ldw % 8 == 0) && ((reinterpret_cast<uintptr_t>(W) & 15) == 0);
    const int64_t cap = (int64_t)sms * 8;
    if (v) {
        const int grid = (int)(d_out < cap ? d_out : cap);
        pack_2to8_v_kernel<<<grid, 256, 0, stream>>>(W, d_out, d_in, ldw, o);
    } else {
        const int64_t units = d_out * (d_in / 8);
        int64_t grid = (units + 255) / 256;
        if (grid > cap) grid = cap;
        pack_2to8_any_kernel<<<(int)(grid > 0 ? grid : 1), 256, 0, stream>>>(W, d_out, d_in, ldw, o);
    }
    return cudaGetLastError();
}

}  // namespace slr

// pack_2to4.cu -- 2:4 projection (plain or activation-aware) and packing
// (values + 2-bit indices).
//
// Hard-thresholding onto the 2:4 pattern (HASSLE-free, section 4.1.1: the
// data-free optimal sparse update keeps the largest magnitudes; 2:4 = two
// nonzeros in each group of four, as on the 3BASiL page).  The magnitude key
// is the bf16 bit pattern with its sign bit cleared, compared as an integer;
// of two equal keys the lower index wins.
//
// The activation-aware variant (HASSLE-free, section 4.1.2: with a diagonal
// Hessian the sparse step hard-thresholds W scaled column-wise by the input
// column norms, Wanda's score) ranks weight w_ij by the fp32 product
// |w_ij| * |scale_j|, NaN products highest, ties again to the lower index.
//
// Work unit = 8 consecutive bf16 of a row (two groups): one 16-byte load, one
// 8-byte store of the four kept values and one metadata byte, so a warp moves
// 512 B in, 256 B + 32 B out, all coalesced.  The kernels are HBM-bound at
// 2 B read + 1.125 B written per weight; the grids keep a few waves of the
// 148 SMs.
#include "common.cuh"

namespace slr {
namespace {

// The two kept positions of a group from the sort keys e_p of its four
// positions, where each key carries (3 - p) in its two low bits so that no two
// keys are equal: a larger score wins and, of two equal scores, the lower
// position.  The two largest keys of four come from a max/min network (max of
// the pair maxima, then the larger of the smaller pair maximum and the larger
// pair minimum).  Returns the nibble idx0 | idx1 << 2 (idx0 < idx1).
template <typename Key>
__device__ __forceinline__ uint32_t top_two_nibble(Key e0, Key e1, Key e2, Key e3) {
    const Key m01 = max(e0, e1), n01 = min(e0, e1);
    const Key m23 = max(e2, e3), n23 = min(e2, e3);
    const Key first = max(m01, m23);
    const Key second = max(min(m01, m23), max(n01, n23));
    const uint32_t pa = 3u - (uint32_t)(first & 3u), pb = 3u - (uint32_t)(second & 3u);
    return min(pa, pb) | (max(pa, pb) << 2);
}

// Gather the two kept bf16 values of a group (held as words w01 = positions
// 0,1 and w23 = positions 2,3) into one word, idx0 low and idx1 high: one byte
// permute, position p sitting in bytes 2p, 2p+1 of (w01, w23).
__device__ __forceinline__ uint32_t gather_kept(uint32_t nib, uint32_t w01, uint32_t w23) {
    const uint32_t i0 = nib & 3u, i1 = nib >> 2;
    const uint32_t sel = (i0 * 2u) * 0x11u + 0x10u + (((i1 * 2u) * 0x11u + 0x10u) << 8);
    return __byte_perm(w01, w23, sel);
}

// Plain projection of one group: the key of position p is
// (magnitude bits << 2) | (3 - p), 17 bits.
__device__ __forceinline__ uint32_t select_group(uint32_t w01, uint32_t w23, uint32_t *kept) {
    const uint32_t e0 = ((w01 & 0x7FFFu) << 2) | 3u;
    const uint32_t e1 = ((w01 >> 14) & 0x1FFFCu) | 2u;
    const uint32_t e2 = ((w23 & 0x7FFFu) << 2) | 1u;
    const uint32_t e3 = (w23 >> 14) & 0x1FFFCu;
    const uint32_t nib = top_two_nibble(e0, e1, e2, e3);
    *kept = gather_kept(nib, w01, w23);
    return nib;
}

// Activation-aware score of a weight (magnitude bits m, already << 16) and a
// non-negative scale a: the bits of the fp32 product |w| * a, rounded to
// nearest (an explicit _rn multiply, never contracted), sign cleared; a NaN
// product takes the largest key 0x7FFFFFFF.  Non-negative floats order like
// their bit patterns, so the keys compare as unsigned integers.
__device__ __forceinline__ uint32_t scaled_key(uint32_t mag_hi, float a) {
    const uint32_t k = __float_as_uint(__fmul_rn(__uint_as_float(mag_hi), a)) & 0x7FFFFFFFu;
    return k > 0x7F800000u ? 0x7FFFFFFFu : k;
}

// Activation-aware projection of one group; a0..a3 are the absolute scales
// of its four columns.  The keys use all 32 bits, so the position tie-break
// is explicit: a tournament of (0,1) and (2,3), where a tie keeps the lower
// position; the overall first is the better of the two pair winners (ties to
// the (0,1) side, whose positions are lower); the second is the better of the
// winning pair's loser and the losing pair's winner (again ties to the lower
// position, which is the one from (0,1)).
__device__ __forceinline__ uint32_t select_group_scaled(uint32_t w01, uint32_t w23, float a0, float a1, float a2,
                                                        float a3, uint32_t *kept) {
    const uint32_t k0 = scaled_key((w01 & 0x7FFFu) << 16, a0);
    const uint32_t k1 = scaled_key(w01 & 0x7FFF0000u, a1);
    const uint32_t k2 = scaled_key((w23 & 0x7FFFu) << 16, a2);
    const uint32_t k3 = scaled_key(w23 & 0x7FFF0000u, a3);
    const bool b01 = k0 >= k1, b23 = k2 >= k3;
    const uint32_t hi01 = max(k0, k1), lo01 = min(k0, k1);
    const uint32_t hi23 = max(k2, k3), lo23 = min(k2, k3);
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
    const uint32_t nib = min(first, second) | (max(first, second) << 2);
    *kept = gather_kept(nib, w01, w23);
    return nib;
}

// Vectorised path: d_in % 8 == 0, ldw % 8 == 0, W 16-byte aligned.  Rows are
// distributed over the grid; the CTA's threads sweep a row in 16-byte units,
// keeping kPackUnroll loads in flight per thread (coalesced across the CTA for
// each step).  No integer division on the index path.
constexpr int kPackUnroll = 4;

__global__ void __launch_bounds__(256) pack_2to4_v8_kernel(const uint16_t *__restrict__ W, int64_t d_out,
                                                           int64_t d_in, int64_t ldw,
                                                           uint16_t *__restrict__ vals,
                                                           uint8_t *__restrict__ meta) {
    const int units = (int)(d_in / 8);
    const int64_t meta_row = (d_in / 4 + 1) / 2;
    for (int64_t row = blockIdx.x; row < d_out; row += gridDim.x) {
        const uint16_t *wrow = W + row * ldw;
        uint2 *vrow = reinterpret_cast<uint2 *>(vals + row * (d_in / 2));
        uint8_t *mrow = meta + row * meta_row;
        for (int c0 = threadIdx.x; c0 < units; c0 += kPackUnroll * blockDim.x) {
            uint4 w[kPackUnroll];
#pragma unroll
            for (int i = 0; i < kPackUnroll; ++i) {
                const int c = c0 + i * blockDim.x;
                if (c < units) w[i] = ld_stream_v4(wrow + (int64_t)c * 8);
            }
#pragma unroll
            for (int i = 0; i < kPackUnroll; ++i) {
                const int c = c0 + i * blockDim.x;
                if (c < units) {
                    uint32_t kept0, kept1;
                    const uint32_t n0 = select_group(w[i].x, w[i].y, &kept0);
                    const uint32_t n1 = select_group(w[i].z, w[i].w, &kept1);
                    vrow[c] = make_uint2(kept0, kept1);
                    mrow[c] = (uint8_t)(n0 | (n1 << 4));
                }
            }
        }
    }
}

// General path: any alignment, d_in % 4 == 0.  Unit = one metadata byte
// (two groups, or one for the last byte of a row with an odd group count).
__global__ void __launch_bounds__(256) pack_2to4_any_kernel(const uint16_t *__restrict__ W, int64_t d_out,
                                                            int64_t d_in, int64_t ldw,
                                                            uint16_t *__restrict__ vals,
                                                            uint8_t *__restrict__ meta) {
    const int64_t groups = d_in / 4;
    const int64_t meta_row = (groups + 1) / 2;
    const int64_t total = d_out * meta_row;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total;
         u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = u / meta_row;
        const int64_t j = u - row * meta_row;
        uint32_t byte = 0;
        for (int h = 0; h < 2; ++h) {
            const int64_t g = 2 * j + h;
            if (g >= groups) break;
            const uint16_t *src = W + row * ldw + 4 * g;
            const uint32_t w01 = (uint32_t)src[0] | ((uint32_t)src[1] << 16);
            const uint32_t w23 = (uint32_t)src[2] | ((uint32_t)src[3] << 16);
            uint32_t kept;
            const uint32_t nib = select_group(w01, w23, &kept);
            uint16_t *dst = vals + row * (d_in / 2) + 2 * g;
            dst[0] = (uint16_t)(kept & 0xFFFFu);
            dst[1] = (uint16_t)(kept >> 16);
            byte |= nib << (4 * h);
        }
        meta[row * meta_row + j] = (uint8_t)byte;
    }
}

// Activation-aware projection, vectorised path (d_in % 8 == 0, ldw % 8 == 0,
// W and scale 16-byte aligned, vals 8-byte aligned).  The grid is
// (column strips of 256 units) x (row blocks): a thread owns one 8-column unit
// for all its rows, so it loads that unit's eight scales once into registers,
// and sweeps rows kScaledRows at a time (one 16-byte load per row in flight
// each; a warp's loads of one row are 512 contiguous bytes).
constexpr int kScaledRows = 4;

__global__ void __launch_bounds__(256) pack_2to4_scaled_v8_kernel(const uint16_t *__restrict__ W, int64_t d_out,
                                                                  int64_t d_in, int64_t ldw,
                                                                  const float *__restrict__ scale,
                                                                  uint16_t *__restrict__ vals,
                                                                  uint8_t *__restrict__ meta) {
    const int64_t units = d_in / 8;
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= units) return;  // no block-wide barrier below
    const int64_t meta_row = (d_in / 4 + 1) / 2;
    const float4 s0 = __ldg(reinterpret_cast<const float4 *>(scale + 8 * c));
    const float4 s1 = __ldg(reinterpret_cast<const float4 *>(scale + 8 * c + 4));
    const float a0 = fabsf(s0.x), a1 = fabsf(s0.y), a2 = fabsf(s0.z), a3 = fabsf(s0.w);
    const float a4 = fabsf(s1.x), a5 = fabsf(s1.y), a6 = fabsf(s1.z), a7 = fabsf(s1.w);
    const int64_t step = (int64_t)gridDim.y * kScaledRows;
    for (int64_t row0 = (int64_t)blockIdx.y * kScaledRows; row0 < d_out; row0 += step) {
        uint4 w[kScaledRows];
#pragma unroll
        for (int i = 0; i < kScaledRows; ++i)
            if (row0 + i < d_out) w[i] = ld_stream_v4(W + (row0 + i) * ldw + 8 * c);
#pragma unroll
        for (int i = 0; i < kScaledRows; ++i) {
            const int64_t row = row0 + i;
            if (row < d_out) {
                uint32_t kept0, kept1;
                const uint32_t n0 = select_group_scaled(w[i].x, w[i].y, a0, a1, a2, a3, &kept0);
                const uint32_t n1 = select_group_scaled(w[i].z, w[i].w, a4, a5, a6, a7, &kept1);
                reinterpret_cast<uint2 *>(vals + row * (d_in / 2))[c] = make_uint2(kept0, kept1);
                meta[row * meta_row + c] = (uint8_t)(n0 | (n1 << 4));
            }
        }
    }
}

// Activation-aware projection, general path: any alignment, d_in % 4 == 0;
// unit = one metadata byte, as in pack_2to4_any_kernel.
__global__ void __launch_bounds__(256) pack_2to4_scaled_any_kernel(const uint16_t *__restrict__ W, int64_t d_out,
                                                                   int64_t d_in, int64_t ldw,
                                                                   const float *__restrict__ scale,
                                                                   uint16_t *__restrict__ vals,
                                                                   uint8_t *__restrict__ meta) {
    const int64_t groups = d_in / 4;
    const int64_t meta_row = (groups + 1) / 2;
    const int64_t total = d_out * meta_row;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total;
         u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = u / meta_row;
        const int64_t j = u - row * meta_row;
        uint32_t byte = 0;
        for (int h = 0; h < 2; ++h) {
            const int64_t g = 2 * j + h;
            if (g >= groups) break;
            const uint16_t *src = W + row * ldw + 4 * g;
            const float *sc = scale + 4 * g;
            const uint32_t w01 = (uint32_t)src[0] | ((uint32_t)src[1] << 16);
            const uint32_t w23 = (uint32_t)src[2] | ((uint32_t)src[3] << 16);
            uint32_t kept;
            const uint32_t nib = select_group_scaled(w01, w23, fabsf(sc[0]), fabsf(sc[1]), fabsf(sc[2]),
                                                     fabsf(sc[3]), &kept);
            uint16_t *dst = vals + row * (d_in / 2) + 2 * g;
            dst[0] = (uint16_t)(kept & 0xFFFFu);
            dst[1] = (uint16_t)(kept >> 16);
            byte |= nib << (4 * h);
        }
        meta[row * meta_row + j] = (uint8_t)byte;
    }
}

int grid_for(int64_t units, int threads) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (units + threads - 1) / threads;
    const int64_t cap = (int64_t)sms * 8;  // 8 resident CTAs of 256 threads per SM
    return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_pack_2to4(const uint16_t *W, int64_t d_out, int64_t d_in, int64_t ldw,
                             uint16_t *vals, uint8_t *meta, cudaStream_t stream) {
    const bool v8 = (d_in % 8 == 0) && (ldw % 8 == 0) && ((reinterpret_cast<uintptr_t>(W) & 15) == 0) &&
                    ((reinterpret_cast<uintptr_t>(vals) & 7) == 0);
    if (v8) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int64_t cap = (int64_t)sms * 8;
        const int grid = (int)(d_out < cap ? d_out : cap);
        pack_2to4_v8_kernel<<<grid, 256, 0, stream>>>(W, d_out, d_in, ldw, vals, meta);
    } else {
        const int64_t units = d_out * ((d_in / 4 + 1) / 2);
        pack_2to4_any_kernel<<<grid_for(units, 256), 256, 0, stream>>>(W, d_out, d_in, ldw, vals, meta);
    }
    return cudaGetLastError();
}

cudaError_t launch_pack_2to4_scaled(const uint16_t *W, int64_t d_out, int64_t d_in, int64_t ldw,
                                    const float *scale, uint16_t *vals, uint8_t *meta, cudaStream_t stream) {
    const bool v8 = (d_in % 8 == 0) && (ldw % 8 == 0) && ((reinterpret_cast<uintptr_t>(W) & 15) == 0) &&
                    ((reinterpret_cast<uintptr_t>(scale) & 15) == 0) &&
                    ((reinterpret_cast<uintptr_t>(vals) & 7) == 0);
    if (v8) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int64_t strips = (d_in / 8 + 255) / 256;
        const int64_t row_blocks = (d_out + kScaledRows - 1) / kScaledRows;
        int64_t gy = ((int64_t)sms * 8 + strips - 1) / strips;  // about 8 CTAs of 256 threads per SM
        if (gy > row_blocks) gy = row_blocks;
        if (gy > 65535) gy = 65535;
        pack_2to4_scaled_v8_kernel<<<dim3((unsigned)strips, (unsigned)gy), 256, 0, stream>>>(W, d_out, d_in, ldw,
                                                                                              scale, vals, meta);
    } else {
        const int64_t units = d_out * ((d_in / 4 + 1) / 2);
        pack_2to4_scaled_any_kernel<<<grid_for(units, 256), 256, 0, stream>>>(W, d_out, d_in, ldw, scale, vals,
                                                                              meta);
    }
    return cudaGetLastError();
}

}  // namespace slr

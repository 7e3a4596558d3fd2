// pack_2to4.cu -- 2:4 projection by magnitude and packing (values + 2-bit indices).
//
// Hard-thresholding onto the 2:4 pattern (HASSLE-free, section 4.1.1: the
// data-free optimal sparse update keeps the largest magnitudes; 2:4 = two
// nonzeros in each group of four, as on the 3BASiL page).  The magnitude key
// is the bf16 bit pattern with its sign bit cleared, compared as an integer;
// of two equal keys the lower index wins.
//
// Work unit = 8 consecutive bf16 of a row (two groups): one 16-byte load, one
// 8-byte store of the four kept values and one metadata byte, so a warp moves
// 512 B in, 256 B + 32 B out, all coalesced.  The kernel is HBM-bound at
// 2 B read + 1.125 B written per weight; a grid-stride loop over
// d_out * d_in / 8 units keeps the grid at a few waves of the 148 SMs.
#include "common.cuh"

namespace slr {
namespace {

// Select the two kept positions of a group given as two 32-bit words holding
// bf16 values 0,1 (w01) and 2,3 (w23).  Returns the nibble idx0 | idx1 << 2 and
// the two kept bit patterns packed low (idx0) / high (idx1).
//
// Each position p gets the sort key (magnitude bits << 2) | (3 - p): a larger
// magnitude wins and, of two equal magnitudes, the lower position.  The two
// largest keys of four come from a max/min network (max of the pair maxima,
// then the larger of the smaller pair maximum and the larger pair minimum),
// and one byte permute gathers the two kept values.
__device__ __forceinline__ uint32_t select_group(uint32_t w01, uint32_t w23, uint32_t *kept) {
    const uint32_t e0 = ((w01 & 0x7FFFu) << 2) | 3u;
    const uint32_t e1 = ((w01 >> 14) & 0x1FFFCu) | 2u;
    const uint32_t e2 = ((w23 & 0x7FFFu) << 2) | 1u;
    const uint32_t e3 = (w23 >> 14) & 0x1FFFCu;
    const uint32_t m01 = max(e0, e1), n01 = min(e0, e1);
    const uint32_t m23 = max(e2, e3), n23 = min(e2, e3);
    const uint32_t first = max(m01, m23);
    const uint32_t second = max(min(m01, m23), max(n01, n23));
    const uint32_t pa = 3u - (first & 3u), pb = 3u - (second & 3u);
    const uint32_t i0 = min(pa, pb), i1 = max(pa, pb);
    // Position p sits in bytes 2p, 2p+1 of (w01, w23).
    const uint32_t sel = (i0 * 2u) * 0x11u + 0x10u + (((i1 * 2u) * 0x11u + 0x10u) << 8);
    *kept = __byte_perm(w01, w23, sel);
    return i0 | (i1 << 2);
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

}  // namespace slr

// tc_forward.cuh -- launcher of the 2:4 tcgen05 tensor-core forward (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace slr {

namespace tc {
// 2-D tiled tensor map of a row-major matrix (inner x outer elements, row
// pitch row_bytes) with the given box and swizzle; false when the driver's
// encoder is unavailable or rejects the arguments.
bool make_map(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);
}  // namespace tc

// Largest M whose tensor-core forward (the split-K kernel) and projection
// support chained launches.
constexpr int64_t kChainMaxM = 64;

// Workspace of the single-call tensor-core forward above kChainMaxM tokens
// (r > 0): T (bf16 [M, r], read by the rank stages), a 1 KB block of counters
// (the projection phase's two at byte 0, one per K-split tail tile from byte
// 64), the fp32 partial products of the 512-row kernel's projection phase (at
// most kFusedMaxParts slices of a 256-token tile, tile rows of up to 128 ranks;
// r <= 128 only), and the fp32 partial tiles of its K-split last round (one
// slot of 2 CTAs x 2 halves x 240 tokens x 128 rows per pair; `pairs` is the
// most pairs a launch may use on the device, fused_pairs_for(SM count)).
constexpr int64_t kFusedMaxParts = 128;
constexpr int64_t kKsSlotFloats = 2 * 2 * 240 * 128;
inline int64_t fused_pairs_for(int sms) {
    const int64_t p = sms / 2;
    return p < 128 ? p : 128;
}
struct FusedLayout {
    size_t off_count, off_ks_count, off_part, off_ks_part, bytes;
};
inline FusedLayout fused_layout(int64_t M, int64_t r, int64_t pairs) {
    const size_t t16 = ((size_t)M * (size_t)r * 2 + 255) / 256 * 256;
    const size_t rn = r <= 64 ? 64 : 128;
    FusedLayout L;
    L.off_count = t16;
    L.off_ks_count = t16 + 64;
    L.off_part = t16 + 1024;
    L.off_ks_part = L.off_part + (r <= 128 ? (size_t)kFusedMaxParts * 256 * rn * 4 : 0);
    L.bytes = L.off_ks_part + (size_t)pairs * kKsSlotFloats * 4;
    return L;
}

// Y = X S^T + T U^T on the tensor cores.  T16 is bf16 [M, r] (may be null when
// r == 0).  Requires d_in % 128 == 0, d_out % 8 == 0, r % 8 == 0.
// pdl: 0 = ordinary launch; 1 = the kernel launched immediately before on
// `stream` is the projection that writes T16 (programmatic dependent launch,
// waits before reading T16); 2 = chained (M <= kChainMaxM): also the work
// before the projection may still be running, so the kernel requests only
// the weights (S, U) before it waits, and reads X and T16 after.
cudaError_t launch_tc_forward(const uint16_t *X, int64_t M, const uint16_t *vals, const uint8_t *meta,
                              int64_t d_out, int64_t d_in, const uint16_t *U, const uint16_t *T16, int64_t r,
                              uint16_t *Y, int pdl, cudaStream_t stream);

// The single-call forward on the tensor cores (M > kChainMaxM): where the
// dispatch picks the 512-row pair kernel, that kernel with its projection phase
// (r <= 128; else after the projection kernel) and its last round split along
// K (one launch after a memset of the counters); otherwise the projection
// kernel followed by launch_tc_forward as its programmatic dependent.
// ws: ws_bytes >= fused_layout(M, r, pairs).bytes for the device's pairs
// (null when r == 0: no projection phase, no K split); with fewer slots than
// a K-split plan needs, the last round is split by tokens instead.
cudaError_t launch_tc_forward_fused(const uint16_t *X, int64_t M, const uint16_t *vals, const uint8_t *meta,
                                    int64_t d_out, int64_t d_in, const uint16_t *U, const uint16_t *V, int64_t r,
                                    uint16_t *Y, uint8_t *ws, size_t ws_bytes, cudaStream_t stream);

// T = X V^T on the tensor cores, written as bf16 [M, r] (dense tcgen05 mode of
// the same kernel).  Requires d_in % 64 == 0, r % 8 == 0.  chained: launched
// as a programmatic dependent of whatever precedes it on `stream` (M <=
// kChainMaxM); it requests V first and waits for the preceding grid before it
// reads X or writes T16.
cudaError_t launch_tc_project(const uint16_t *X, int64_t M, const uint16_t *V, int64_t d_in, int64_t r,
                              uint16_t *T16, bool chained, cudaStream_t stream);

// Host-only check of the pair kernels' work plan (see slr_plan_check in
// slr.h): the number of violations, 0 for a sound plan, -1 for bad arguments.
namespace tc {
int64_t plan_check(int64_t M, int64_t d_out, int64_t d_in, int64_t r, int kernel, int tail_mode, int max_pairs,
                   int chu);
}  // namespace tc

// Launches the failure-detection self-test kernel (a bounded wait that is
// made to expire after limit_cycles SM clock cycles).
cudaError_t launch_wait_timeout_selftest(long long limit_cycles, cudaStream_t stream);

// Reads and clears the device-side error word the tensor-core kernel sets when
// a bounded wait expires (0 = none).  Synchronises the device.
cudaError_t read_and_clear_kernel_error(unsigned *code);

}  // namespace slr

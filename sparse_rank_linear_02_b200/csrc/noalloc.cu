// noalloc.cu -- small-M forward that needs no caller-provided workspace.
//
// The streaming (decode) forward needs scratch for the rank projection
// T = X V^T (M x r fp32) between its two kernels; slr_forward takes that
// scratch from the caller's workspace.  Some callers have no way to provide
// it: an inference engine that reserves the whole device heap at start-up and
// only hands out the tensors it manages, or a latency-critical decode loop in
// which calling cudaMalloc (which can synchronise the device) is not allowed.
// slr_forward_decode_noalloc serves them: it runs the same two kernels, with T
// placed in a fixed array that is part of this library's device image.
//
// Facts a caller must know (also stated in include/slr.h):
//  * Capacity: M * r <= SLR_NOALLOC_MAX_T_ELEMS floats (64 KB).  Larger
//    problems are rejected with SLR_ERR_WORKSPACE before anything is queued.
//  * The array exists once per device that loads the library and stays
//    allocated until the process exits.
//  * The first call on a device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current and caches it; make that
//    first call before any stream capture.
//  * All calls on a device share the one array, which keeps the previous
//    call's contents.  Nothing in it has to start at zero: the projection
//    kernel writes every T entry that the streaming kernel then reads, in
//    stream order.  Calls that can run at the same time on the GPU (different
//    streams, or host threads without ordering between them) race on the
//    array and must be serialised by the caller.
//  * No cudaMalloc, cudaFree or allocating library routine is called.
#include <mutex>

#include "common.cuh"

namespace slr {
namespace {

// The scratch.  In host code `g_noalloc_T` names a host-side stand-in, not a
// device address; only the address returned by cudaGetSymbolAddress may be
// passed to a kernel.
static __device__ __align__(256) float g_noalloc_T[SLR_NOALLOC_MAX_T_ELEMS];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_T on the current device, looked up once per
// device.  Returns SLR_OK and sets *out, or an error status.
slr_status scratch_on_current_device(float **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return SLR_ERR_DEVICE;
    }
    static std::mutex mu;
    static float *addr[kMaxDevices] = {nullptr};
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            cudaGetLastError();
            return SLR_ERR_DEVICE;
        }
        if (major != 10 || minor != 0) return SLR_ERR_DEVICE;
        void *p = nullptr;
        const cudaError_t err = cudaGetSymbolAddress(&p, g_noalloc_T);
        if (err != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return SLR_ERR_CUDA;
        }
        addr[dev] = static_cast<float *>(p);
    }
    *out = addr[dev];
    return SLR_OK;
}

bool is_aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace slr

extern "C" slr_status slr_forward_decode_noalloc(const void *X, int64_t M, const void *vals, const void *meta,
                                                 int64_t d_out, int64_t d_in, const void *U, const void *V,
                                                 int64_t r, void *Y, slr_stream_t stream) {
    if (M < 0 || d_out < 0 || d_in < 0 || r < 0) return SLR_ERR_SHAPE;
    if (M == 0) return SLR_OK;
    if (X == nullptr || vals == nullptr || meta == nullptr || Y == nullptr) return SLR_ERR_NULL;
    if (r > 0 && (U == nullptr || V == nullptr)) return SLR_ERR_NULL;
    if (d_out < 1 || d_in < 128 || d_in % 128 != 0 || r % 8 != 0) return SLR_ERR_SHAPE;
    if (M > INT32_MAX || d_out > INT32_MAX || d_in > INT32_MAX) return SLR_ERR_SHAPE;
    if (r > 0 && M > SLR_NOALLOC_MAX_T_ELEMS / r) return SLR_ERR_WORKSPACE;
    if (!slr::is_aligned16(X) || !slr::is_aligned16(vals) || !slr::is_aligned16(meta) || !slr::is_aligned16(Y))
        return SLR_ERR_ALIGN;
    if (r > 0 && (!slr::is_aligned16(U) || !slr::is_aligned16(V))) return SLR_ERR_ALIGN;
    float *T = nullptr;
    const slr_status st = slr::scratch_on_current_device(&T);
    if (st != SLR_OK) return st;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const uint16_t *x = static_cast<const uint16_t *>(X);
    cudaError_t err = cudaSuccess;
    if (r > 0) err = slr::launch_lowrank_project(x, M, static_cast<const uint16_t *>(V), d_in, r, T, nullptr, false, s);
    if (err == cudaSuccess)
        err = slr::launch_decode_forward(x, M, static_cast<const uint16_t *>(vals), static_cast<const uint8_t *>(meta),
                                         d_out, d_in, static_cast<const uint16_t *>(U), r > 0 ? T : nullptr, r,
                                         static_cast<uint16_t *>(Y), 1, s);
    return err == cudaSuccess ? SLR_OK : SLR_ERR_CUDA;
}

// api.cu -- the exported C ABI (include/slr.h): argument checks, workspace
// layout and path dispatch.  No arithmetic of the layer happens here.
#include <mutex>

#include "common.cuh"
#include "tc_forward.cuh"

namespace slr {
namespace {

constexpr size_t kAlign = 256;
// Largest M whose tensor-core path may take T from the CUDA-core projection,
// and the most bytes of X that projection may re-read.
constexpr int64_t kSmallProjectM = 16;
constexpr double kSmallProjectXBytes = 12.0 * 1024 * 1024;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// sm_100 check, cached per device ordinal.
slr_status check_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        cudaGetLastError();
        return SLR_ERR_DEVICE;
    }
    static std::mutex mu;
    static int device_ok[64] = {0};  // 0 unknown, 1 ok, 2 bad
    if (dev >= 64) return SLR_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(mu);
    if (device_ok[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            cudaGetLastError();
            return SLR_ERR_DEVICE;
        }
        device_ok[dev] = (major == 10 && minor == 0) ? 1 : 2;
    }
    return device_ok[dev] == 1 ? SLR_OK : SLR_ERR_DEVICE;
}

// The CUDA-core streaming path wins only for a single token on layers of up
// to 2^26 weights (measured on B200 with rotating weight copies: 4096 x 4096,
// M = 1: 7.6 us against 11.8 us; M = 2: 12.5 against 11.8 us; 14336 x 4096,
// M = 1: 18.4 against 19.3 us, M = 2: 28.1 against 19.0 us); larger layers
// and two or more tokens stream faster through the split-K tensor-core kernel.
constexpr int64_t kDecodeMaxM = 1;
constexpr int64_t kDecodeMaxWeights = int64_t(1) << 26;

size_t workspace_bytes_for(int64_t M, int64_t r, slr_path path) {
    if (M <= 0 || r <= 0) return 0;
    if (path == SLR_PATH_DECODE) return round_up((size_t)M * r * sizeof(float), kAlign);
    // Above kChainMaxM tokens the single-call forward may run the 512-row
    // kernel with its projection phase and K-split last round: T, counters,
    // partial products and partial tiles.
    if (M > kChainMaxM) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            sms = 148;   // no device: size for a B200
        }
        return round_up(fused_layout(M, r, fused_pairs_for(sms)).bytes, kAlign);
    }
    return round_up((size_t)M * r * sizeof(uint16_t), kAlign);
}

// The tensor-core path stores Y with TMA, whose row pitch must be a multiple
// of 16 bytes (d_out % 8 == 0); other shapes stay on the streaming path.
bool tensor_ok(int64_t d_out) { return d_out % 8 == 0; }

slr_path resolve(slr_path path, int64_t M, int64_t d_out, int64_t d_in) {
    if (path != SLR_PATH_AUTO) return path;
    if (!tensor_ok(d_out)) return SLR_PATH_DECODE;
    return (M <= kDecodeMaxM && d_out * d_in <= kDecodeMaxWeights) ? SLR_PATH_DECODE : SLR_PATH_TENSOR;
}

// Host-side validation shared by the forward entry points.  `need_factors`
// selects which low-rank operands the stage reads.
slr_status validate(const void *X, int64_t M, const void *vals, const void *meta, int64_t d_out, int64_t d_in,
                    const void *U, const void *V, int64_t r, const void *Y, const void *workspace,
                    size_t workspace_bytes, slr_path path, bool need_sparse, bool need_U, bool need_V,
                    slr_path *resolved) {
    if (path != SLR_PATH_AUTO && path != SLR_PATH_DECODE && path != SLR_PATH_TENSOR) return SLR_ERR_ARG;
    if (M < 0 || d_out < 0 || d_in < 0 || r < 0) return SLR_ERR_SHAPE;
    const slr_path p = resolve(path, M, d_out, d_in);
    *resolved = p;
    if (M == 0) return SLR_OK;
    const size_t need = workspace_bytes_for(M, r, p);
    if (X == nullptr) return SLR_ERR_NULL;
    if (need_sparse && (vals == nullptr || meta == nullptr || Y == nullptr)) return SLR_ERR_NULL;
    if (r > 0 && ((need_U && U == nullptr) || (need_V && V == nullptr))) return SLR_ERR_NULL;
    if (need > 0 && workspace == nullptr) return SLR_ERR_NULL;
    if (d_out < 1 || d_in < 128 || d_in % 128 != 0 || r % 8 != 0) return SLR_ERR_SHAPE;
    if (p == SLR_PATH_TENSOR && !tensor_ok(d_out)) return SLR_ERR_SHAPE;
    if (M > INT32_MAX || d_out > INT32_MAX || d_in > INT32_MAX) return SLR_ERR_SHAPE;
    if (!aligned16(X)) return SLR_ERR_ALIGN;
    if (need_sparse && (!aligned16(vals) || !aligned16(meta) || !aligned16(Y))) return SLR_ERR_ALIGN;
    if (r > 0 && ((need_U && !aligned16(U)) || (need_V && !aligned16(V)))) return SLR_ERR_ALIGN;
    if (need > 0 && (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return SLR_ERR_ALIGN;
    if (workspace_bytes < need) return SLR_ERR_WORKSPACE;
    return check_device();
}

// Stage 1: T = X V^T into the workspace, fp32 for the streaming path and bf16
// for the tensor-core path.  chained: see forward_impl.
cudaError_t run_project(const void *X, int64_t M, const void *V, int64_t d_in, int64_t r, void *workspace,
                        slr_path p, bool chained, cudaStream_t stream) {
    if (r == 0) return cudaSuccess;
    const uint16_t *x = static_cast<const uint16_t *>(X);
    const uint16_t *vv = static_cast<const uint16_t *>(V);
    if (p == SLR_PATH_DECODE)
        return launch_lowrank_project(x, M, vv, d_in, r, static_cast<float *>(workspace), nullptr, chained, stream);
    // Up to 16 tokens the CUDA-core projection (r x 1..2 CTAs, fp32 sums
    // rounded to bf16; 2.3-3.6 us on 4096 x 4096 against 6.7 us for the
    // tensor-core projection, which runs on a handful of CTAs there), as long
    // as its CTAs' re-reads of X (each rank index reads the token block's X,
    // r * M * d_in * 2 bytes in all) stay small.
    if (M <= kSmallProjectM && (double)r * (double)M * (double)d_in * 2.0 <= kSmallProjectXBytes)
        return launch_lowrank_project(x, M, vv, d_in, r, nullptr, static_cast<uint16_t *>(workspace), chained, stream);
    return launch_tc_project(x, M, vv, d_in, r, static_cast<uint16_t *>(workspace), chained, stream);
}

// Stage 2: Y = X S^T + T U^T with T read from the workspace.  pdl: 0 ordinary
// launch, 1 right after the projection, 2 chained.
cudaError_t run_combine(const void *X, int64_t M, const void *vals, const void *meta, int64_t d_out, int64_t d_in,
                        const void *U, int64_t r, void *Y, const void *workspace, slr_path p, int pdl,
                        cudaStream_t stream) {
    const uint16_t *x = static_cast<const uint16_t *>(X);
    const uint16_t *v = static_cast<const uint16_t *>(vals);
    const uint8_t *m = static_cast<const uint8_t *>(meta);
    const uint16_t *u = static_cast<const uint16_t *>(U);
    uint16_t *y = static_cast<uint16_t *>(Y);
    if (p == SLR_PATH_DECODE)
        return launch_decode_forward(x, M, v, m, d_out, d_in, u, r > 0 ? static_cast<const float *>(workspace) : nullptr,
                                     r, y, pdl, stream);
    return launch_tc_forward(x, M, v, m, d_out, d_in, u, r > 0 ? static_cast<const uint16_t *>(workspace) : nullptr,
                             r, y, pdl, stream);
}

// Whether a call with SLR_FWD_OVERLAP_PRECEDING runs chained: the small-M
// kernels (the streaming path where it stages X in shared memory, and the
// split-K tensor kernel with its projection up to kChainMaxM tokens and rank
// 256) support it; other calls launch as without the flag, which is also
// correct.
bool chain_supported(slr_path p, int64_t M, int64_t d_in, int64_t r) {
    if (p == SLR_PATH_DECODE) return decode_chain_ok(M, d_in);
    return M <= kChainMaxM && r <= 256;
}

// Chained (flags & SLR_FWD_OVERLAP_PRECEDING, where supported): the
// projection is a programmatic dependent of the work before the call, the
// combine a programmatic dependent of the projection; both request only
// weights (V; S and U) before they wait for the preceding grid, and read X,
// read or write T, and write Y after.  Otherwise the projection is an
// ordinary launch and the combine a programmatic dependent of it that waits
// only before reading T.
slr_status forward_impl(const void *X, int64_t M, const void *vals, const void *meta, int64_t d_out,
                        int64_t d_in, const void *U, const void *V, int64_t r, void *Y, void *workspace,
                        size_t workspace_bytes, slr_path path, uint32_t flags, cudaStream_t stream) {
    slr_path p;
    if ((flags & ~(uint32_t)SLR_FWD_OVERLAP_PRECEDING) != 0) return SLR_ERR_ARG;
    const slr_status st = validate(X, M, vals, meta, d_out, d_in, U, V, r, Y, workspace, workspace_bytes, path,
                                   true, true, true, &p);
    if (st != SLR_OK || M == 0) return st;
    const bool chained = (flags & SLR_FWD_OVERLAP_PRECEDING) != 0 && chain_supported(p, M, d_in, r);
    cudaError_t err = cudaSuccess;
    if (p == SLR_PATH_TENSOR && M > kChainMaxM) {
        // One call: the 512-row kernel with its projection phase where it is
        // the dispatched kernel, else projection then combine.
        err = launch_tc_forward_fused(static_cast<const uint16_t *>(X), M, static_cast<const uint16_t *>(vals),
                                      static_cast<const uint8_t *>(meta), d_out, d_in,
                                      static_cast<const uint16_t *>(U), static_cast<const uint16_t *>(V), r,
                                      static_cast<uint16_t *>(Y), static_cast<uint8_t *>(workspace), workspace_bytes,
                                      stream);
        return err == cudaSuccess ? SLR_OK : SLR_ERR_CUDA;
    }
    err = run_project(X, M, V, d_in, r, workspace, p, chained, stream);
    if (err == cudaSuccess)
        err = run_combine(X, M, vals, meta, d_out, d_in, U, r, Y, workspace, p, chained ? 2 : 1, stream);
    return err == cudaSuccess ? SLR_OK : SLR_ERR_CUDA;
}

}  // namespace
}  // namespace slr

extern "C" {

const char *slr_status_string(slr_status s) {
    switch (s) {
        case SLR_OK: return "SLR_OK";
        case SLR_ERR_NULL: return "SLR_ERR_NULL: a required pointer is NULL";
        case SLR_ERR_SHAPE: return "SLR_ERR_SHAPE: a size is negative or violates a divisibility rule";
        case SLR_ERR_ALIGN: return "SLR_ERR_ALIGN: a pointer is not 16-byte aligned";
        case SLR_ERR_WORKSPACE: return "SLR_ERR_WORKSPACE: workspace too small";
        case SLR_ERR_DEVICE: return "SLR_ERR_DEVICE: no sm_100 CUDA device is current";
        case SLR_ERR_CUDA: return "SLR_ERR_CUDA: a CUDA call or kernel launch failed";
        case SLR_ERR_TIMEOUT: return "SLR_ERR_TIMEOUT: a kernel gave up a bounded wait";
        case SLR_ERR_ARG: return "SLR_ERR_ARG: an enum argument is out of range";
    }
    return "SLR_ERR_UNKNOWN";
}

int slr_version(void) { return 100; }

int64_t slr_meta_row_bytes(int64_t d_in) { return d_in < 0 ? 0 : (d_in / 4 + 1) / 2; }

slr_status slr_pack_2to4(const void *W, int64_t d_out, int64_t d_in, int64_t ldw, void *vals, void *meta,
                         slr_stream_t stream) {
    if (d_out < 0 || d_in < 0 || d_in % 4 != 0 || ldw < d_in) return SLR_ERR_SHAPE;
    if (d_out == 0 || d_in == 0) return SLR_OK;
    if (W == nullptr || vals == nullptr || meta == nullptr) return SLR_ERR_NULL;
    const slr_status dev = slr::check_device();
    if (dev != SLR_OK) return dev;
    const cudaError_t err = slr::launch_pack_2to4(static_cast<const uint16_t *>(W), d_out, d_in, ldw,
                                                  static_cast<uint16_t *>(vals), static_cast<uint8_t *>(meta),
                                                  reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? SLR_OK : SLR_ERR_CUDA;
}

slr_status slr_pack_2to4_scaled(const void *W, int64_t d_out, int64_t d_in, int64_t ldw, const float *scale,
                                void *vals, void *meta, slr_stream_t stream) {
    if (d_out < 0 || d_in < 0 || d_in % 4 != 0 || ldw < d_in) return SLR_ERR_SHAPE;
    if (d_out == 0 || d_in == 0) return SLR_OK;
    if (W == nullptr || scale == nullptr || vals == nullptr || meta == nullptr) return SLR_ERR_NULL;
    const slr_status dev = slr::check_device();
    if (dev != SLR_OK) return dev;
    const cudaError_t err = slr::launch_pack_2to4_scaled(
        static_cast<const uint16_t *>(W), d_out, d_in, ldw, scale, static_cast<uint16_t *>(vals),
        static_cast<uint8_t *>(meta), reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? SLR_OK : SLR_ERR_CUDA;
}

slr_status slr_pack_2to8(const void *W, int64_t d_out, int64_t d_in, int64_t ldw, void *vals8, void *meta8,
                         void *vals4, void *meta4, slr_stream_t stream) {
    if (d_out < 0 || d_in < 0 || d_in % 8 != 0 || ldw < d_in) return SLR_ERR_SHAPE;
    if ((vals8 == nullptr) != (meta8 == nullptr) || (vals4 == nullptr) != (meta4 == nullptr) ||
        (vals8 == nullptr && vals4 == nullptr))
        return SLR_ERR_NULL;
    if (d_out == 0 || d_in == 0) return SLR_OK;
    if (W == nullptr) return SLR_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(vals8) & 3) != 0 || (reinterpret_cast<uintptr_t>(vals4) & 7) != 0)
        return SLR_ERR_ALIGN;
    const slr_status dev = slr::check_device();
    if (dev != SLR_OK) return dev;
    const cudaError_t err = slr::launch_pack_2to8(
        static_cast<const uint16_t *>(W), d_out, d_in, ldw, static_cast<uint16_t *>(vals8),
        static_cast<uint8_t *>(meta8), static_cast<uint16_t *>(vals4), static_cast<uint8_t *>(meta4),
        reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? SLR_OK : SLR_ERR_CUDA;
}

slr_status slr_forward_2to8(const void *X, int64_t M, const void *vals8, const void *meta8, int64_t d_out,
                            int64_t d_in, const void *U, const void *V, int64_t r, void *Y, void *workspace,
                            size_t workspace_bytes, slr_stream_t stream) {
    if (M < 0 || d_out < 0 || d_in < 0 || r < 0) return SLR_ERR_SHAPE;
    if (M == 0) return SLR_OK;
    const size_t need = slr::workspace_bytes_for(M, r, SLR_PATH_DECODE);
    if (X == nullptr || vals8 == nullptr || meta8 == nullptr || Y == nullptr) return SLR_ERR_NULL;
    if (r > 0 && (U == nullptr || V == nullptr)) return SLR_ERR_NULL;
    if (need > 0 && workspace == nullptr) return SLR_ERR_NULL;
    if (d_out < 1 || d_in < 32 || d_in % 32 != 0 || r % 8 != 0) return SLR_ERR_SHAPE;
    if (M >= (int64_t(1) << 18) || d_out > INT32_MAX || d_in > INT32_MAX) return SLR_ERR_SHAPE;
    if (!slr::aligned16(X) || !slr::aligned16(vals8) || !slr::aligned16(meta8) || !slr::aligned16(Y))
        return SLR_ERR_ALIGN;
    if (r > 0 && (!slr::aligned16(U) || !slr::aligned16(V))) return SLR_ERR_ALIGN;
    if (need > 0 && (reinterpret_cast<uintptr_t>(workspace) % slr::kAlign) != 0) return SLR_ERR_ALIGN;
    if (workspace_bytes < need) return SLR_ERR_WORKSPACE;
    const slr_status dev = slr::check_device();
    if (dev != SLR_OK) return dev;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const uint16_t *x = static_cast<const uint16_t *>(X);
    float *T32 = r > 0 ? static_cast<float *>(workspace) : nullptr;
    cudaError_t err = cudaSuccess;
    if (r > 0) err = slr::launch_lowrank_project(x, M, static_cast<const uint16_t *>(V), d_in, r, T32, nullptr, false, st);
    if (err == cudaSuccess)
        err = slr::launch_decode28_forward(x, M, static_cast<const uint16_t *>(vals8),
                                           static_cast<const uint8_t *>(meta8), d_out, d_in,
                                           static_cast<const uint16_t *>(U), T32, r, static_cast<uint16_t *>(Y),
                                           r > 0, st);
    return err == cudaSuccess ? SLR_OK : SLR_ERR_CUDA;
}

size_t slr_lora_backward_workspace_size(int64_t M, int64_t r) {
    if (M <= 0 || r <= 0) return 0;
    return slr::round_up((size_t)4 * M * r, slr::kAlign);
}

slr_status slr_lora_backward(const void *X, int64_t M, const void *dY, int64_t d_out, int64_t d_in, const void *U,
                             const void *V, int64_t r, const void *T, float *dU, float *dV, void *workspace,
                             size_t workspace_bytes, slr_stream_t stream) {
    if (M < 0 || d_out < 8 || d_out % 8 != 0 || d_in < 64 || d_in % 64 != 0 || r < 8 || r > 256 || r % 8 != 0 ||
        M > INT32_MAX || d_out > INT32_MAX || d_in > INT32_MAX)
        return SLR_ERR_SHAPE;
    if (dU == nullptr || dV == nullptr) return SLR_ERR_NULL;
    if (M > 0 && (X == nullptr || dY == nullptr || U == nullptr || V == nullptr || workspace == nullptr))
        return SLR_ERR_NULL;
    if (!slr::aligned16(dU) || !slr::aligned16(dV)) return SLR_ERR_ALIGN;
    if (M > 0 && (!slr::aligned16(X) || !slr::aligned16(dY) || !slr::aligned16(U) || !slr::aligned16(V) ||
                  !slr::aligned16(T) || (reinterpret_cast<uintptr_t>(workspace) % slr::kAlign) != 0))
        return SLR_ERR_ALIGN;
    if (workspace_bytes < slr_lora_backward_workspace_size(M, r)) return SLR_ERR_WORKSPACE;
    const slr_status dev = slr::check_device();
    if (dev != SLR_OK) return dev;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t err;
    if (M == 0) {
        err = cudaMemsetAsync(dU, 0, (size_t)d_out * r * sizeof(float), st);
        if (err == cudaSuccess) err = cudaMemsetAsync(dV, 0, (size_t)r * d_in * sizeof(float), st);
    } else {
        err = slr::launch_lora_backward(static_cast<const uint16_t *>(X), M, static_cast<const uint16_t *>(dY), d_out,
                                        d_in, static_cast<const uint16_t *>(U), static_cast<const uint16_t *>(V), r,
                                        static_cast<const uint16_t *>(T), dU, dV, static_cast<uint16_t *>(workspace),
                                        st);
    }
    return err == cudaSuccess ? SLR_OK : SLR_ERR_CUDA;
}

size_t slr_decompose_workspace_size(int64_t d_out, int64_t d_in, int64_t r) {
    if (d_out < 1 || d_in < 8 || r < 8 || r > 128) return 0;
    return (size_t)slr::am_plan(d_out, d_in, r).bytes;
}

slr_status slr_decompose_datafree(const void *W, int64_t d_out, int64_t d_in, int64_t r, int iters,
                                  int power_first, int power, const float *Q0, void *vals, void *meta, void *U,
                                  void *V, double *objective, void *workspace, size_t workspace_bytes,
                                  slr_stream_t stream) {
    if (d_out < 1 || d_in < 8 || d_in % 8 != 0 || r < 8 || r > 128 || r % 8 != 0 || r > d_out || r > d_in ||
        d_out > INT32_MAX || d_in > INT32_MAX)
        return SLR_ERR_SHAPE;
    if (iters < 0 || iters > 10000 || power_first < 1 || power_first > 1000 || power < 1 || power > 1000)
        return SLR_ERR_ARG;
    if (W == nullptr || Q0 == nullptr || vals == nullptr || meta == nullptr || U == nullptr || V == nullptr ||
        workspace == nullptr)
        return SLR_ERR_NULL;
    if (!slr::aligned16(W) || !slr::aligned16(Q0) || !slr::aligned16(vals) || !slr::aligned16(meta) ||
        !slr::aligned16(U) || !slr::aligned16(V) || !slr::aligned16(workspace) ||
        (reinterpret_cast<uintptr_t>(objective) & 7) != 0)
        return SLR_ERR_ALIGN;
    if (workspace_bytes < slr_decompose_workspace_size(d_out, d_in, r)) return SLR_ERR_WORKSPACE;
    const slr_status dev = slr::check_device();
    if (dev != SLR_OK) return dev;
    const cudaError_t err = slr::launch_am_datafree(
        static_cast<const uint16_t *>(W), d_out, d_in, (int)r, iters, power_first, power, Q0,
        static_cast<uint16_t *>(vals), static_cast<uint8_t *>(meta), static_cast<uint16_t *>(U),
        static_cast<uint16_t *>(V), objective, static_cast<uint8_t *>(workspace),
        reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? SLR_OK : SLR_ERR_CUDA;
}

slr_status slr_decompose_factors_f32(const void *workspace, size_t workspace_bytes, int64_t d_out, int64_t d_in,
                                     int64_t r, float *U32, float *V32, slr_stream_t stream) {
    if (d_out < 1 || d_in < 8 || d_in % 8 != 0 || r < 8 || r > 128 || r % 8 != 0 || r > d_out || r > d_in ||
        d_out > INT32_MAX || d_in > INT32_MAX)
        return SLR_ERR_SHAPE;
    if (workspace == nullptr || (U32 == nullptr && V32 == nullptr)) return SLR_ERR_NULL;
    if (!slr::aligned16(workspace) || !slr::aligned16(U32) || !slr::aligned16(V32)) return SLR_ERR_ALIGN;
    if (workspace_bytes < slr_decompose_workspace_size(d_out, d_in, r)) return SLR_ERR_WORKSPACE;
    const slr_status dev = slr::check_device();
    if (dev != SLR_OK) return dev;
    const cudaError_t err = slr::launch_am_factors_f32(static_cast<const uint8_t *>(workspace), d_out, d_in, (int)r,
                                                       U32, V32, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? SLR_OK : SLR_ERR_CUDA;
}

size_t slr_column_norms_workspace_size(int64_t M, int64_t d_in) {
    if (M <= 0 || d_in <= 0 || d_in % 8 != 0) return 0;
    const slr::NormPlan p = slr::column_norms_plan(M, d_in);
    return slr::round_up((size_t)p.splits * (size_t)d_in * sizeof(float), slr::kAlign);
}

slr_status slr_column_norms(const void *X, int64_t M, int64_t d_in, int64_t ldx, double *sumsq, float *norms,
                            void *workspace, size_t workspace_bytes, slr_stream_t stream) {
    if (M < 0 || d_in < 0 || d_in % 8 != 0 || ldx < d_in || ldx % 8 != 0) return SLR_ERR_SHAPE;
    if (d_in == 0) return SLR_OK;
    if (sumsq == nullptr || (M > 0 && (X == nullptr || workspace == nullptr))) return SLR_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(sumsq) & 7) != 0 || (reinterpret_cast<uintptr_t>(norms) & 3) != 0 ||
        (M > 0 && (!slr::aligned16(X) || !slr::aligned16(workspace))))
        return SLR_ERR_ALIGN;
    if (workspace_bytes < slr_column_norms_workspace_size(M, d_in)) return SLR_ERR_WORKSPACE;
    const slr_status dev = slr::check_device();
    if (dev != SLR_OK) return dev;
    const cudaError_t err = slr::launch_column_norms(static_cast<const uint16_t *>(X), M, d_in, ldx, sumsq, norms,
                                                     static_cast<float *>(workspace),
                                                     reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? SLR_OK : SLR_ERR_CUDA;
}

size_t slr_forward_workspace_size(int64_t M, int64_t d_out, int64_t d_in, int64_t r) {
    (void)d_out;
    (void)d_in;
    const size_t a = slr::workspace_bytes_for(M, r, SLR_PATH_DECODE);
    const size_t b = slr::workspace_bytes_for(M, r, SLR_PATH_TENSOR);
    return a > b ? a : b;
}

slr_path slr_forward_select_path(int64_t M, int64_t d_out, int64_t d_in, int64_t r) {
    (void)d_out;
    (void)d_in;
    (void)r;
    return slr::resolve(SLR_PATH_AUTO, M, d_out, d_in);
}

slr_status slr_check_kernel_error(void) {
    if (slr::check_device() != SLR_OK) return SLR_ERR_DEVICE;
    if (cudaDeviceSynchronize() != cudaSuccess) return SLR_ERR_CUDA;
    unsigned code = 0, code28 = 0, code_bwd = 0, code_am = 0;
    if (slr::read_and_clear_kernel_error(&code) != cudaSuccess) return SLR_ERR_CUDA;
    if (slr::read_and_clear_decode28_error(&code28) != cudaSuccess) return SLR_ERR_CUDA;
    if (slr::read_and_clear_backward_error(&code_bwd) != cudaSuccess) return SLR_ERR_CUDA;
    if (slr::read_and_clear_am_error(&code_am) != cudaSuccess) return SLR_ERR_CUDA;
    return (code | code28 | code_bwd | code_am) ? SLR_ERR_TIMEOUT : SLR_OK;
}

int64_t slr_plan_check(int64_t M, int64_t d_out, int64_t d_in, int64_t r, int32_t kernel, int32_t tail_mode,
                       int32_t max_pairs, int32_t chunk_units) {
    return slr::tc::plan_check(M, d_out, d_in, r, kernel, tail_mode, max_pairs, chunk_units);
}

slr_status slr_selftest_wait_timeout(int64_t limit_cycles, slr_stream_t stream) {
    if (limit_cycles < 1 || limit_cycles > INT32_MAX) return SLR_ERR_ARG;
    if (slr::check_device() != SLR_OK) return SLR_ERR_DEVICE;
    return slr::launch_wait_timeout_selftest((long long)limit_cycles, reinterpret_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? SLR_OK
               : SLR_ERR_CUDA;
}

slr_status slr_forward(const void *X, int64_t M, const void *vals, const void *meta, int64_t d_out, int64_t d_in,
                       const void *U, const void *V, int64_t r, void *Y, void *workspace, size_t workspace_bytes,
                       slr_stream_t stream) {
    return slr::forward_impl(X, M, vals, meta, d_out, d_in, U, V, r, Y, workspace, workspace_bytes, SLR_PATH_AUTO,
                             0u, reinterpret_cast<cudaStream_t>(stream));
}

slr_status slr_forward_project(const void *X, int64_t M, const void *V, int64_t d_out, int64_t d_in, int64_t r,
                               void *workspace, size_t workspace_bytes, slr_path path, slr_stream_t stream) {
    slr_path p;
    const void *dummy = X;
    const slr_status st = slr::validate(X, M, dummy, dummy, d_out, d_in, nullptr, V, r, dummy, workspace,
                                        workspace_bytes, path, false, false, true, &p);
    if (st != SLR_OK || M == 0) return st;
    return slr::run_project(X, M, V, d_in, r, workspace, p, false, reinterpret_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? SLR_OK
               : SLR_ERR_CUDA;
}

slr_status slr_forward_combine(const void *X, int64_t M, const void *vals, const void *meta, int64_t d_out,
                               int64_t d_in, const void *U, int64_t r, void *Y, const void *workspace,
                               size_t workspace_bytes, slr_path path, slr_stream_t stream) {
    slr_path p;
    const slr_status st = slr::validate(X, M, vals, meta, d_out, d_in, U, nullptr, r, Y, workspace, workspace_bytes,
                                        path, true, true, false, &p);
    if (st != SLR_OK || M == 0) return st;
    return slr::run_combine(X, M, vals, meta, d_out, d_in, U, r, Y, workspace, p, 0,
                            reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SLR_OK
               : SLR_ERR_CUDA;
}

slr_status slr_forward_with_path(const void *X, int64_t M, const void *vals, const void *meta, int64_t d_out,
                                 int64_t d_in, const void *U, const void *V, int64_t r, void *Y, void *workspace,
                                 size_t workspace_bytes, slr_path path, slr_stream_t stream) {
    return slr::forward_impl(X, M, vals, meta, d_out, d_in, U, V, r, Y, workspace, workspace_bytes, path, 0u,
                             reinterpret_cast<cudaStream_t>(stream));
}

slr_status slr_forward_ex(const void *X, int64_t M, const void *vals, const void *meta, int64_t d_out, int64_t d_in,
                          const void *U, const void *V, int64_t r, void *Y, void *workspace, size_t workspace_bytes,
                          slr_path path, uint32_t flags, slr_stream_t stream) {
    return slr::forward_impl(X, M, vals, meta, d_out, d_in, U, V, r, Y, workspace, workspace_bytes, path, flags,
                             reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

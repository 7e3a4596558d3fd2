// lora_backward.cu -- gradients of the layer with respect to its low-rank
// factors (S frozen), on the tensor cores.
//
// Y = X S^T + T U^T with T = X V^T (LoSparse, section 3.2); the low-rank
// factors are what LoRA fine-tuning trains (3BASiL summary page: the low-rank
// components initialise LoRA).  For dY = dL/dY:
//     G  = dY U          (M x r,     bf16)
//     dU = dY^T T        (d_out x r, fp32)
//     dV = G^T X         (r x d_in,  fp32)
// All three are dense products with one small side (r); the weight gradients
// contract over the tokens, which are the outer (row) dimension of dY and X,
// so their operands are read "MN-major" (contiguous along the output
// dimension) straight from the row-major activations: no transposes.
//
// The three products run on tc_gemm_kernel (tc_gemm.cuh): bf16 operands,
// fp32 accumulation in TMEM, K- or MN-major operands read in place.
// dU runs on a second stream beside G and dV (forked and joined with events
// on the caller's stream).
#include <cuda.h>

#include <mutex>

#include "tc_gemm.cuh"

namespace slr {

// Error word of this file's bounded waits (read by slr_check_kernel_error).
__device__ unsigned int g_bwd_error = 0;

namespace {

// Device address of this file's error word on the current device.
unsigned int *bwd_err() {
    static unsigned int *addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (addr[dev] == nullptr) {
        void *q = nullptr;
        if (cudaGetSymbolAddress(&q, g_bwd_error) == cudaSuccess) addr[dev] = static_cast<unsigned int *>(q);
    }
    return addr[dev];
}

// A second stream per device, so that dU (which needs only dY and T) runs
// beside G and dV; created once, never destroyed (it lives as long as the
// process, like the library's other per-device state).
cudaStream_t side_stream() {
    static std::mutex mu;
    static cudaStream_t streams[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (streams[dev] == nullptr && cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess)
        streams[dev] = nullptr;
    return streams[dev];
}

template <int RN>
cudaError_t backward_rn(const uint16_t *X, int64_t M, const uint16_t *dY, int64_t d_out, int64_t d_in,
                        const uint16_t *U, const uint16_t *T16, uint16_t *G16, int64_t r, float *dU, float *dV,
                        cudaStream_t st) {
    // dU = dY^T T (A = dY [M][d_out] MN-major, K = M; B = T [M][r] MN-major) on
    // the side stream, forked from and joined back into `st` with events, while
    // `st` runs G = dY U (A = dY K-major, K = d_out; B = U [d_out][r] MN-major)
    // and then dV^T = X^T G (A = X [M][d_in] MN-major, B = G [M][r] MN-major,
    // stored transposed as dV [r][d_in]).  Without a side stream, all on `st`.
    cudaStream_t side = side_stream();
    cudaEvent_t fork = nullptr, join = nullptr;
    if (side != nullptr && (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess ||
                            cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess)) {
        if (fork != nullptr) cudaEventDestroy(fork);
        fork = join = nullptr;
        side = nullptr;
    }
    cudaError_t e = cudaSuccess;
    cudaStream_t su = st;
    if (side != nullptr) {
        e = cudaEventRecord(fork, st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(side, fork, 0);
        if (e == cudaSuccess) su = side;
    }
    if (e == cudaSuccess) e = gemm_tc<true, true, RN, kOutF32>(dY, nullptr, d_out, T16, nullptr, r, d_out, r, M, dU, bwd_err(), su);
    if (e == cudaSuccess && side != nullptr) e = cudaEventRecord(join, side);
    if (e == cudaSuccess) e = gemm_tc<false, true, RN, kOutBF16>(dY, nullptr, d_out, U, nullptr, r, M, r, d_out, G16, bwd_err(), st);
    if (e == cudaSuccess) e = gemm_tc<true, true, RN, kOutF32T>(X, nullptr, d_in, G16, nullptr, r, d_in, r, M, dV, bwd_err(), st);
    if (e == cudaSuccess && side != nullptr) e = cudaStreamWaitEvent(st, join, 0);
    if (fork != nullptr) cudaEventDestroy(fork);  // released once the recorded work completes
    if (join != nullptr) cudaEventDestroy(join);
    return e;
}

}  // namespace

cudaError_t launch_lora_backward(const uint16_t *X, int64_t M, const uint16_t *dY, int64_t d_out, int64_t d_in,
                                 const uint16_t *U, const uint16_t *V, int64_t r, const uint16_t *T16_in, float *dU,
                                 float *dV, uint16_t *ws, cudaStream_t st) {
    uint16_t *T16 = ws;                 // M x r (when not given)
    uint16_t *G16 = ws + M * r;         // M x r
    cudaError_t e = cudaSuccess;
    if (T16_in == nullptr) {
        e = launch_tc_project(X, M, V, d_in, r, T16, false, st);
        T16_in = T16;
    }
    if (e != cudaSuccess) return e;
    if (r <= 64) return backward_rn<64>(X, M, dY, d_out, d_in, U, T16_in, G16, r, dU, dV, st);
    if (r <= 128) return backward_rn<128>(X, M, dY, d_out, d_in, U, T16_in, G16, r, dU, dV, st);
    return backward_rn<256>(X, M, dY, d_out, d_in, U, T16_in, G16, r, dU, dV, st);
}

cudaError_t read_and_clear_backward_error(unsigned *code) {
    unsigned v = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_bwd_error, sizeof v);
    if (err != cudaSuccess) return err;
    if (v != 0) {
        const unsigned zero = 0;
        err = cudaMemcpyToSymbol(g_bwd_error, &zero, sizeof zero);
    }
    *code = v;
    return err;
}

}  // namespace slr

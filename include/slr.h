/*
 * slr.h -- C ABI of the 2:4-sparse + low-rank linear layer library (libslr.so).
 *
 * The layer (LoSparse, arXiv 2306.11222, sections 3 and 3.2; HASSLE-free,
 * arXiv 2502.00899, section 1 and the abstract's 2:4 + rank-64 scheme) stores a
 * weight W (d_out x d_in) as a 2:4 semi-structured sparse matrix S plus a
 * rank-r product U*V, and evaluates the two terms side by side:
 *
 *        Y = X * S^T + (X * V^T) * U^T            (bf16 in, fp32 accumulate, bf16 out)
 *
 * All matrices are row-major with dense rows unless a leading dimension is
 * passed.  Every pointer argument of a compute call is a DEVICE pointer on the
 * current CUDA device; the caller owns all memory (the library allocates
 * nothing and frees nothing).  All work is queued on `stream` and runs
 * asynchronously; no call synchronises.
 *
 * Error behaviour: argument checks (null pointers, shapes, alignment,
 * workspace size, device capability) run on the host before anything is
 * queued, in that order, and return the first failing status with nothing
 * launched.  A launch failure returns SLR_ERR_CUDA.  Faults inside a kernel
 * surface, as usual for CUDA, at the caller's next synchronisation.
 *
 * Threading: calls are safe from several host threads; calls on one stream
 * execute in order.  Outputs must not alias inputs.
 *
 * Per-device state: on its first use on a device the library looks up, and
 * keeps for the life of the process, the device addresses of its own
 * file-scope device arrays (the kernels' error words, the scratch of
 * slr_forward_decode_noalloc).  cudaDeviceReset() unloads the module those
 * addresses belong to, so after a reset of a device this library must not be
 * used on that device again in the same process.
 */
#ifndef SLR_H
#define SLR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SLR_API __attribute__((visibility("default")))
#else
#define SLR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *slr_stream_t;

typedef enum slr_status {
    SLR_OK = 0,
    SLR_ERR_NULL = 1,      /* a required pointer is NULL                         */
    SLR_ERR_SHAPE = 2,     /* a size is negative or violates a divisibility rule */
    SLR_ERR_ALIGN = 3,     /* a pointer is not 16-byte aligned                   */
    SLR_ERR_WORKSPACE = 4, /* workspace smaller than slr_forward_workspace_size  */
    SLR_ERR_DEVICE = 5,    /* no CUDA device, or the current device is not sm_100 */
    SLR_ERR_CUDA = 6,      /* a CUDA runtime/driver call or kernel launch failed */
    SLR_ERR_TIMEOUT = 7,   /* a kernel gave up a bounded wait (see the forward)  */
    SLR_ERR_ARG = 8        /* an enum argument is out of range                   */
} slr_status;

/* Human-readable name of a status code (static string, never NULL). */
SLR_API const char *slr_status_string(slr_status s);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
SLR_API int slr_version(void);

/* --------------------------------------------------------------------------
 * 2:4 projection and packing.
 *
 * Hard-thresholding onto 2:4 (HASSLE-free, section 4.1.1: with an identity
 * Hessian the optimal sparse update keeps the largest-magnitude entries; the
 * 2:4 pattern, "two nonzeros in every four weights", as on the 3BASiL page).
 * For every row i and every aligned group g of four columns 4g..4g+3, the two
 * positions with the largest magnitude are kept (magnitude = the bf16 bits
 * with the sign cleared, compared as integers; equal magnitudes keep the
 * lower index; NaN ranks above Inf).  Exactly two positions are kept per
 * group, even when they hold zeros.
 *
 *   W     device, bf16 [d_out, ldw] (ldw >= d_in), read only.
 *   vals  device, bf16 [d_out, d_in/2], dense rows: the two kept values of
 *         group g at columns 2g, 2g+1, in ascending index order (bit copies).
 *   meta  device, uint8 [d_out, slr_meta_row_bytes(d_in)], dense rows: byte j
 *         of a row holds group 2j in its low nibble and group 2j+1 in its high
 *         nibble; nibble = idx0 | idx1 << 2 with 0 <= idx0 < idx1 <= 3.  When
 *         d_in/4 is odd the last high nibble is 0.
 *
 * Requirements: d_out >= 0, d_in >= 0, d_in % 4 == 0, ldw >= d_in; W, vals and
 * meta non-NULL unless d_out * d_in == 0.  Any alignment is accepted; 16-byte
 * aligned W with d_in and ldw multiples of 8 takes the vectorised path.
 * The result is bit-exact and deterministic.
 * ------------------------------------------------------------------------ */
SLR_API slr_status slr_pack_2to4(const void *W, int64_t d_out, int64_t d_in, int64_t ldw,
                         void *vals, void *meta, slr_stream_t stream);

/* Bytes per metadata row: ceil(d_in / 8). */
SLR_API int64_t slr_meta_row_bytes(int64_t d_in);

/* --------------------------------------------------------------------------
 * Activation-aware 2:4 projection and packing.
 *
 * HASSLE-free, section 4.1.2: with the diagonal Hessian approximation
 * H = diag(X^T X) the sparse step hard-thresholds W D, D = diag of the input
 * column norms, which is Wanda's score.  The weight w_ij is ranked by the
 * fp32 product |w_ij| * |scale[j]| (one IEEE multiply, round to nearest); a
 * NaN product ranks above every number; equal products keep the lower index.
 * The kept values are the unscaled weights; the output format is the one of
 * slr_pack_2to4, so slr_forward consumes it unchanged.  With every scale equal
 * to the same power of two the result equals slr_pack_2to4's.
 *
 *   W      device, bf16 [d_out, ldw] (ldw >= d_in), read only.
 *   scale  device, fp32 [d_in], read only: the column scales (the sign is
 *          ignored), e.g. the norms from slr_column_norms.
 *   vals, meta  as for slr_pack_2to4.
 *
 * Requirements: as slr_pack_2to4, and scale non-NULL unless d_out * d_in == 0.
 * Any alignment is accepted; 16-byte aligned W and scale with d_in and ldw
 * multiples of 8 take the vectorised path.  Bit-exact and deterministic.
 * ------------------------------------------------------------------------ */
SLR_API slr_status slr_pack_2to4_scaled(const void *W, int64_t d_out, int64_t d_in, int64_t ldw,
                                const float *scale, void *vals, void *meta, slr_stream_t stream);

/* --------------------------------------------------------------------------
 * Column norms of calibration activations (the scale of the projection above).
 *
 * HASSLE-free, section 4.1.2 (diagonal Hessian) and section 5.1 (the Hessian
 * is gathered over many token segments): each call adds one batch X
 * (M tokens x d_in) to a running per-column sum of squares and can emit the
 * norms, so a calibration set is streamed batch by batch.
 *
 *   X        device, bf16 [M, ldx] (ldx >= d_in), read only.
 *   sumsq    device, fp64 [d_in], in/out: sumsq[j] += sum_m X[m][j]^2.  Zero it
 *            before the first batch.
 *   norms    device, fp32 [d_in], out, or NULL: norms[j] = sqrt(sumsq[j]) (after
 *            the update; fp64 square root rounded to nearest fp32).
 *   workspace / workspace_bytes: device scratch of at least
 *            slr_column_norms_workspace_size(M, d_in) bytes; clobbered.
 *
 * Arithmetic: squares are summed in fp32 over at most 64 rows per thread and
 * 8 threads per column, partial sums are then added in fp64 in a fixed order
 * (which depends on M and d_in only: deterministic on any device).  Relative
 * error of a batch's sum of squares <= 80 * 2^-24 for M <= 2^25 (tested
 * against fp64).
 *
 * Requirements: M >= 0, d_in >= 0, d_in % 8 == 0, ldx >= d_in, ldx % 8 == 0;
 * when d_in > 0: sumsq non-NULL and 8-byte aligned, norms 4-byte aligned, and
 * when also M > 0: X non-NULL and 16-byte aligned, workspace large enough.
 * M == 0 only (re)writes norms from sumsq; d_in == 0 does nothing.
 * ------------------------------------------------------------------------ */
SLR_API slr_status slr_column_norms(const void *X, int64_t M, int64_t d_in, int64_t ldx, double *sumsq,
                            float *norms, void *workspace, size_t workspace_bytes, slr_stream_t stream);

/* Scratch bytes slr_column_norms needs for a batch of M tokens (0 when none). */
SLR_API size_t slr_column_norms_workspace_size(int64_t M, int64_t d_in);

/* --------------------------------------------------------------------------
 * 2:8 projection and packing.
 *
 * The 2:8 configuration (3BASiL summary page, "Faster compression and gains
 * that survive LoRA": 2:8 sparse plus rank 64): at most two nonzeros in every
 * aligned run of eight weights along d_in, chosen by the same rule as
 * slr_pack_2to4 (largest magnitude bits, ties to the lower index, exactly two
 * positions kept per group).  One pass over W writes either or both of:
 *
 *   vals8  device, bf16 [d_out, d_in/4]: the two kept values of group g
 *          (columns 8g..8g+7) at 2g, 2g+1, lower index first.  4-byte aligned.
 *   meta8  device, uint8 [d_out, d_in/8]: byte g = idx0 | idx1 << 3.
 *   vals4, meta4  the slr_pack_2to4 format of the projected matrix (positions
 *          not kept hold +0), bit-identical to slr_pack_2to4 applied to it;
 *          for slr_forward.  vals4 8-byte aligned.
 *
 * Pass NULL for both members of a pair to skip it (not both pairs).
 * Requirements: d_out >= 0, d_in >= 0, d_in % 8 == 0, ldw >= d_in; W any
 * alignment (16-byte aligned W with ldw % 8 == 0 takes the vectorised path).
 * Bit-exact and deterministic.
 * ------------------------------------------------------------------------ */
SLR_API slr_status slr_pack_2to8(const void *W, int64_t d_out, int64_t d_in, int64_t ldw, void *vals8,
                         void *meta8, void *vals4, void *meta4, slr_stream_t stream);

/* --------------------------------------------------------------------------
 * Forward pass of a 2:8-packed layer (small M).
 *
 * Y = X * S^T + (X * V^T) * U^T with S in the dense 2:8 packing of
 * slr_pack_2to8 (vals8, meta8): 0.625 B per weight instead of 1.125 B, so a
 * single token's forward moves ~45% fewer bytes than slr_forward on the 2:4
 * packing.  CUDA cores, one streaming kernel after the rank projection
 * T = X V^T (fp32).  The kernel is bound by instruction issue rather than by
 * those bytes: on the Llama-3-70B up projection it takes 47.6 us at M = 1
 * against 50.3 us for slr_forward on the 2:4 packing, and is slower from
 * M = 2.  For more than one token use slr_forward on the 2:4 packing of the
 * same matrix (vals4, meta4), which runs on the tensor cores.
 *
 * Arguments as slr_forward, with vals8 [d_out, d_in/4] and meta8
 * [d_out, d_in/8]; workspace of at least slr_forward_workspace_size(M, d_out,
 * d_in, r) bytes.  Arithmetic: fp32 products and sums (T in fp32), one bf16
 * rounding of Y; same accuracy contract as slr_forward.
 *
 * Requirements: 0 <= M < 2^18 (M == 0 returns SLR_OK), d_out >= 1, d_in >= 32
 * with d_in % 32 == 0, r >= 0 with r % 8 == 0, d_out, d_in < 2^31, all
 * pointers 16-byte aligned (workspace 256-byte aligned).
 * ------------------------------------------------------------------------ */
SLR_API slr_status slr_forward_2to8(const void *X, int64_t M, const void *vals8, const void *meta8,
                            int64_t d_out, int64_t d_in, const void *U, const void *V, int64_t r,
                            void *Y, void *workspace, size_t workspace_bytes, slr_stream_t stream);

/* --------------------------------------------------------------------------
 * Backward with respect to the low-rank factors (S frozen), for LoRA-style
 * fine-tuning of U and V (3BASiL summary page: the low-rank components
 * initialise LoRA; LoSparse section 3.2 for the layer).
 *
 * For Y = X S^T + T U^T with T = X V^T and an upstream gradient dY:
 *     dU = dY^T T          dV = (dY U)^T X
 * on the tensor cores (bf16 operands, fp32 accumulation; T and G = dY U are
 * held in bf16 between the products).  The operands are read in place from the
 * row-major X and dY (no transposes).
 *
 *   X       device, bf16 [M, d_in]      (the forward's input).
 *   dY      device, bf16 [M, d_out].
 *   U       device, bf16 [d_out, r];  V  device, bf16 [r, d_in].
 *   T       device, bf16 [M, r], or NULL: the forward's X V^T if the caller
 *           kept it; otherwise it is recomputed.
 *   dU      device, fp32 [d_out, r], out;  dV  device, fp32 [r, d_in], out.
 *   workspace  slr_lora_backward_workspace_size(M, r) bytes, 256-byte aligned.
 *
 * The product dU runs on a library-owned second stream, forked from and joined
 * back into `stream` with events, so the call composes with stream capture
 * like any other work on `stream`.
 *
 * Accuracy contract (tested): relative Frobenius error <= 5e-3 and
 * |err| <= 1e-2 * B + 1e-6 * max(B) per element against the exact gradients of
 * the same bf16 inputs, B = |dY|^T |X| |V|^T for dU and (|dY| |U|)^T |X| for dV.
 *
 * Requirements: M >= 0 (M == 0 writes zero gradients), d_out >= 8 with
 * d_out % 8 == 0, d_in >= 64 with d_in % 64 == 0, 8 <= r <= 256 with r % 8 == 0,
 * M, d_out, d_in < 2^31; all pointers 16-byte aligned.
 * ------------------------------------------------------------------------ */
SLR_API slr_status slr_lora_backward(const void *X, int64_t M, const void *dY, int64_t d_out, int64_t d_in,
                             const void *U, const void *V, int64_t r, const void *T, float *dU, float *dV,
                             void *workspace, size_t workspace_bytes, slr_stream_t stream);

/* Scratch bytes of slr_lora_backward (4 * M * r, rounded up). */
SLR_API size_t slr_lora_backward_workspace_size(int64_t M, int64_t r);

/* --------------------------------------------------------------------------
 * Data-free decomposition W ~ S + U V by alternating minimisation.
 *
 * HASSLE-free, section 4 (data-free variant: identity Hessian), started as in
 * LoSparse, section 3.2 (the low-rank part from the top-r singular subspace
 * of W).  After the start, each of `iters` iterations solves
 *   P2: U V = C_r(W - S)   (rank-r truncated SVD, HASSLE-free section 4.2.1)
 *   P1: S = 2:4 hard threshold of W - U V  (largest |.| of each group of four,
 *       ties to the lower index; HASSLE-free section 4.1.1).
 * C_r is computed by subspace iteration on W - S (power_first steps at the
 * start, from the caller's random Q0, then `power` steps warm-started from the
 * previous subspace, CholeskyQR2 orthonormalisation), in fp32.
 *
 *   W          device, bf16 [d_out, d_in], read only.
 *   Q0         device, fp32 [d_in, r]: the random start (e.g. Gaussian).
 *   vals, meta device: S in the slr_pack_2to4 format (values = W - U V at the
 *              kept positions, rounded to bf16).
 *   U          device, bf16 [d_out, r];  V  device, bf16 [r, d_in].
 *   objective  device, fp64 [iters + 1], or NULL: ||W - S - U V||_F (S as
 *              stored in bf16, U V in fp32) after the start and after every
 *              iteration.
 *   workspace  device scratch of slr_decompose_workspace_size() bytes.
 *
 * Requirements: d_out >= 1, d_in >= 8 with d_in % 8 == 0, 8 <= r <= 128 with
 * r % 8 == 0 and r <= min(d_out, d_in), 0 <= iters <= 10000,
 * 1 <= power_first, power <= 1000; all pointers 16-byte aligned (objective
 * 8-byte aligned).  Deterministic for a given Q0.
 * ------------------------------------------------------------------------ */
SLR_API slr_status slr_decompose_datafree(const void *W, int64_t d_out, int64_t d_in, int64_t r, int iters,
                                  int power_first, int power, const float *Q0, void *vals, void *meta,
                                  void *U, void *V, double *objective, void *workspace,
                                  size_t workspace_bytes, slr_stream_t stream);

/* The factors of the last slr_decompose_datafree call that used `workspace`
 * (same d_out, d_in, r; queued on the same stream before this call), before
 * their rounding to bf16: U32 = fp32 [d_out, r], V32 = fp32 [r, d_in], with
 * U V = U32 V32 up to that rounding (the subspace iteration's Z Q and Q^T,
 * HASSLE-free section 4.2.1).  Either output may be NULL (not both).  The
 * workspace is read only.  Same shape rules as slr_decompose_datafree;
 * SLR_ERR_NULL, SLR_ERR_ALIGN (16 bytes), SLR_ERR_WORKSPACE, SLR_ERR_DEVICE,
 * SLR_ERR_CUDA as there. */
SLR_API slr_status slr_decompose_factors_f32(const void *workspace, size_t workspace_bytes, int64_t d_out,
                                             int64_t d_in, int64_t r, float *U32, float *V32, slr_stream_t stream);

/* Scratch bytes of slr_decompose_datafree (about 4 * d_out * d_in + O((d_out + d_in) * r)). */
SLR_API size_t slr_decompose_workspace_size(int64_t d_out, int64_t d_in, int64_t r);

/* --------------------------------------------------------------------------
 * Forward pass  Y = X * S^T + (X * V^T) * U^T.
 *
 * LoSparse, section 3.2: the compressed layer computes the low-rank and sparse
 * terms in parallel instead of X * W.  Here W' = S + U*V with U d_out x r and
 * V r x d_in; (X V^T) is the rank-r projection T (M x r).
 *
 *   X     device, bf16 [M, d_in]          activations, one token per row.
 *   vals  device, bf16 [d_out, d_in/2]    from slr_pack_2to4.
 *   meta  device, uint8 [d_out, d_in/8]   from slr_pack_2to4.
 *   U     device, bf16 [d_out, r]         (ignored, may be NULL, when r == 0).
 *   V     device, bf16 [r, d_in]          (ignored, may be NULL, when r == 0).
 *   Y     device, bf16 [M, d_out]         output, written once, RNE rounded.
 *   workspace / workspace_bytes: device scratch of at least
 *         slr_forward_workspace_size(M, d_out, d_in, r) bytes, 256-byte
 *         aligned; its contents on entry do not matter and are clobbered.
 *
 * Arithmetic: products of bf16 inputs are accumulated in fp32.  T is kept in
 * fp32 on the small-M path and rounded to bf16 before the second product on
 * the tensor-core path.  Above 64 tokens the 512-row tensor-core kernel forms
 * T in the same launch (a projection phase before its main loop: partial
 * products of 256-token tiles over slices of K, summed in a fixed order), and
 * the other kernels take it from a projection kernel launched just before.
 * When that kernel splits its last round of tiles along K, the slices' fp32
 * partial tiles are summed in slice order before the rounding to bf16: the
 * result does not depend on timing, but may differ in the last bit from an
 * unsplit evaluation of the same tile.  Accuracy contract (tested): relative Frobenius error
 * <= 5e-3 and |err_ij| <= 1e-2 * (|X| |W'|^T)_ij + 1e-3 against the exact
 * result on the same bf16 inputs.
 *
 * Requirements: M >= 0 (M == 0 returns SLR_OK before any pointer is looked
 * at), d_out >= 1, d_in >= 128 with d_in % 128 == 0, r >= 0 with r % 8 == 0,
 * M, d_out, d_in < 2^31, all pointers 16-byte aligned.  The tensor-core path
 * additionally needs d_out % 8 == 0 (SLR_PATH_AUTO avoids it otherwise).
 * ------------------------------------------------------------------------ */
SLR_API slr_status slr_forward(const void *X, int64_t M, const void *vals, const void *meta,
                       int64_t d_out, int64_t d_in, const void *U, const void *V, int64_t r,
                       void *Y, void *workspace, size_t workspace_bytes, slr_stream_t stream);

/* Scratch bytes slr_forward needs for this problem (0 when none): T (fp32
 * [M, r] on the streaming path, bf16 [M, r] on the tensor-core path) and,
 * above 64 tokens with r > 0, 1 KB of counters, room for the partial products
 * with which the 512-row tensor-core kernel forms T itself (r <= 128:
 * 128 x 256 x 64 or 128 fp32 values) and for the fp32 partial tiles of its
 * last round when that round is split along K (one slot of 2 x 2 x 240 x 128
 * fp32 values per SM pair of the current device: 36.4 MB on a 148-SM B200).
 * The size is computed for the current device; a workspace sized on a device
 * with fewer SMs is still valid (that round is then split by tokens).  The
 * counters are zeroed on the stream before each launch that uses them. */
SLR_API size_t slr_forward_workspace_size(int64_t M, int64_t d_out, int64_t d_in, int64_t r);

/* Execution paths of the forward pass. */
typedef enum slr_path {
    SLR_PATH_AUTO = 0,   /* choose by M and layer size (slr_forward_select_path):
                            DECODE for M == 1 on layers of <= 2^26 weights,
                            TENSOR otherwise (and DECODE when d_out % 8 != 0)      */
    SLR_PATH_DECODE = 1, /* CUDA-core streaming kernel over S rows (any M, best
                            for a single token)                                     */
    SLR_PATH_TENSOR = 2  /* 2:4 tcgen05 tensor-core kernels with the rank-r term
                            fused: split-K streaming kernel for M <= 64 and for
                            layers of few 128-row tiles up to a few hundred
                            tokens, 2-SM pairs on 256- or 512-row tiles
                            otherwise (the plan of least estimated time)          */
} slr_path;

/* The path SLR_PATH_AUTO takes for this problem. */
SLR_API slr_path slr_forward_select_path(int64_t M, int64_t d_out, int64_t d_in, int64_t r);

/* slr_forward with an explicit path (for tests and measurement); same
 * arguments, requirements and result contract as slr_forward. */
SLR_API slr_status slr_forward_with_path(const void *X, int64_t M, const void *vals, const void *meta,
                                 int64_t d_out, int64_t d_in, const void *U, const void *V,
                                 int64_t r, void *Y, void *workspace, size_t workspace_bytes,
                                 slr_path path, slr_stream_t stream);

/* Option bits of slr_forward_ex.
 *
 * SLR_FWD_OVERLAP_PRECEDING: the call's kernels may start while the kernel
 * queued just before them on `stream` is still running (programmatic
 * dependent launch).  Before that kernel has completed they only read the
 * layer's weights (vals, meta, U, V); they wait for it before they read X,
 * read or write the workspace, or write Y.  Back-to-back layers of a decode
 * loop then stream the next layer's weights while the previous layer
 * finishes, which hides the launch and ramp-up time of layers of a few tens
 * of MB.  The caller guarantees that the kernel queued immediately before
 * the call does not write vals, meta, U or V (weights written earlier, with
 * at least one other kernel or any copy or event in between, are fine).
 * Honoured for the small-M kernels (the streaming path, and the tensor-core
 * path up to 64 tokens with r <= 256); other calls run as without the flag.
 * The result is the same bits as without the flag. */
#define SLR_FWD_OVERLAP_PRECEDING 1u

/* slr_forward_with_path with option bits (SLR_FWD_*); unknown bits return
 * SLR_ERR_ARG.  flags == 0 is slr_forward_with_path. */
SLR_API slr_status slr_forward_ex(const void *X, int64_t M, const void *vals, const void *meta, int64_t d_out,
                                  int64_t d_in, const void *U, const void *V, int64_t r, void *Y, void *workspace,
                                  size_t workspace_bytes, slr_path path, uint32_t flags, slr_stream_t stream);

/* The two stages of slr_forward, for callers that schedule or time them
 * separately.  slr_forward(...) == slr_forward_project(...) followed on the same
 * stream by slr_forward_combine(...) with the same path and workspace.
 *
 * slr_forward_project: T = X * V^T (the rank-r projection, LoSparse section
 * 3.2) into `workspace`, in the layout the resolved path reads (fp32 [M, r]
 * for SLR_PATH_DECODE, bf16 [M, r] for SLR_PATH_TENSOR).  d_out only selects
 * the path.  vals/meta/U/Y are not read.
 *
 * slr_forward_combine: Y = X * S^T + T * U^T with T taken from `workspace`
 * as written by slr_forward_project for the same (M, d_out, r, path).  V is
 * not read.  Requirements and errors are those of slr_forward restricted to
 * the arguments each stage takes. */
SLR_API slr_status slr_forward_project(const void *X, int64_t M, const void *V, int64_t d_out, int64_t d_in,
                                       int64_t r, void *workspace, size_t workspace_bytes, slr_path path,
                                       slr_stream_t stream);
SLR_API slr_status slr_forward_combine(const void *X, int64_t M, const void *vals, const void *meta,
                                       int64_t d_out, int64_t d_in, const void *U, int64_t r, void *Y,
                                       const void *workspace, size_t workspace_bytes, slr_path path,
                                       slr_stream_t stream);

/* --------------------------------------------------------------------------
 * Small-M forward without a caller workspace.  (The pages have no
 * counterpart to this entry point; it exists for callers of this library.)
 *
 * For callers that cannot allocate device memory where they run the layer,
 * e.g. an inference engine that reserves the whole device heap at start-up
 * and only hands out the tensors it manages, or a latency-critical decode loop
 * that may not call cudaMalloc (which can synchronise the device).  It
 * computes the same result as slr_forward_with_path(..., SLR_PATH_DECODE, ...),
 * with the same argument layouts, but keeps the rank projection T = X V^T in an
 * array built into the library instead of a workspace.
 *
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - Capacity: M * r <= SLR_NOALLOC_MAX_T_ELEMS (fp32 entries, 64 KB); larger
 *     problems return SLR_ERR_WORKSPACE with nothing queued.  r == 0 needs no
 *     scratch and accepts any M.
 *   - The array exists once per device that loads the library and stays
 *     allocated until the process exits.
 *   - The first call on a device does a one-time set-up (it looks up the
 *     array's device address with that device current); make that first call
 *     before any stream capture.
 *   - Every call on a device uses the same array, which keeps the previous
 *     call's contents; nothing in it needs to start at zero because each call
 *     writes every entry it later reads.  Calls that can overlap on the GPU
 *     (different streams, or host threads with no ordering between them) race
 *     on the array: serialise them.
 * Other requirements and errors are those of slr_forward (no workspace
 * arguments).
 * ------------------------------------------------------------------------ */
#define SLR_NOALLOC_MAX_T_ELEMS 16384
SLR_API slr_status slr_forward_decode_noalloc(const void *X, int64_t M, const void *vals, const void *meta,
                                              int64_t d_out, int64_t d_in, const void *U, const void *V,
                                              int64_t r, void *Y, slr_stream_t stream);

/* Synchronises the current device, then reports (and clears) the error word
 * that the tensor-core kernel sets when one of its bounded waits expires:
 * SLR_ERR_TIMEOUT if any launch since the last check gave up, SLR_OK
 * otherwise.  Kernels that time out leave their output incomplete but free
 * their resources and return, so the CUDA context stays usable. */
SLR_API slr_status slr_check_kernel_error(void);

/* Failure-detection self-test (no counterpart on the pages; it checks this
 * library's own error path).  Launches, on `stream`, one thread that waits with
 * the same bounded mbarrier wait the tensor-core kernels use, but with a limit
 * of `limit_cycles` SM clock cycles (1 <= limit_cycles < 2^31; 2e6 is about a
 * millisecond), on a barrier that nothing completes.  The wait expires, the
 * kernel records a timeout in the library's error word and returns, so the
 * next slr_check_kernel_error() reports SLR_ERR_TIMEOUT and the context stays
 * usable.  Returns SLR_ERR_ARG for a limit out of range, SLR_ERR_DEVICE
 * without an sm_100 device, SLR_ERR_CUDA if the launch fails. */
SLR_API slr_status slr_selftest_wait_timeout(int64_t limit_cycles, slr_stream_t stream);

/* Host-only check of the work plan of the 2-SM pair kernels of slr_forward
 * (no device needed, nothing launched).  The layer's product is a sum over
 * the K stages of every output tile (LoSparse, section 3.2); the plan deals
 * the tiles, pieces of tiles (runs of tokens) and K slices of tiles to the
 * pairs.  This builds the plan for a problem shape as a launch would and walks
 * every pair's chunk sequence, counting violations: every (row tile, 16-token
 * unit, K stage) covered by exactly one chunk, the rank stages of every (row
 * tile, unit) by exactly one, chunk rows and tokens inside the problem, a K
 * slice only as a pair's last chunk, with its slice, slot and counter indices
 * in range.
 *
 *   kernel       0: 256-row tiles, chunks of up to 128 tokens; 1: 240;
 *                3: 256; 2: 512-row tiles, 240 tokens.
 *   tail_mode    0: the last round dealt as whole tiles; 1: split by tokens;
 *                2: split along K (kernel 2 only).
 *   max_pairs    1..128 (the device's pairs, e.g. 74 on a 148-SM B200).
 *   chunk_units  most 16-token units per chunk (0: the kernel's maximum).
 *
 * Returns the number of violations (0: the plan is sound), or -1 when an
 * argument is out of range (as for slr_forward, d_in % 128 == 0, r % 8 == 0)
 * or the problem needs more than 2^26 (tile, unit, stage) entries. */
SLR_API int64_t slr_plan_check(int64_t M, int64_t d_out, int64_t d_in, int64_t r, int32_t kernel, int32_t tail_mode,
                               int32_t max_pairs, int32_t chunk_units);

#ifdef __cplusplus
}
#endif

#endif /* SLR_H */

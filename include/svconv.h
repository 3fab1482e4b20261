/*
 * svconv — SparseConv2D on frame-wise pruned ViT tokens, B200 (sm_100a).
 *
 * C ABI of the CUDA library (libsvconv.so).  The operation is the native sparse
 * 3x3 convolution of SV-TAD (papernotes.org, "SV-TAD: Native Sparse Convolutions
 * for Efficient Temporal Action Detection", Method, Key Designs 1 and 2), which
 * convolves a packed, pruned token sequence directly through a neighbour table
 * and never rebuilds the dense H x W grid.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tokens are packed frame by frame: frame t owns packed rows
 *    frame_off[t] .. frame_off[t+1]-1 (frame_off is int32, CSR style, T+1 entries).
 *    coords is int32 [n][3] = (t, y, x) per token.  Within a frame any token
 *    order is accepted.
 *  - Taps j = 0..8 are row-major over (dy, dx) in {-1,0,1}^2: j = (dy+1)*3 + (dx+1).
 *    j = 4 is the token itself and 8-j is the mirrored offset (-dy, -dx).
 *  - The neighbour table nbr is int32 [n][9]; nbr[k][j] is the GLOBAL packed row
 *    of the token at (t, y_k+dy_j, x_k+dx_j), or -1 if that cell was pruned or lies
 *    outside the frame.  Neighbours never cross frames.
 *  - Features are row-major with channels contiguous: X [n][C_in], Y [n][C_out].
 *    Weights are W [C_out][9][C_in] (torch conv2d weight w[o][i][dy+1][dx+1] maps
 *    to W[o][(dy+1)*3+(dx+1)][i]); the operator is a cross-correlation, like conv2d.
 *  - All pointers are DEVICE pointers owned by the caller unless stated otherwise;
 *    the library allocates no device memory and every call is asynchronous on the
 *    given CUDA stream (a cudaStream_t passed as void*; NULL = legacy stream).
 *  - dtype SVCONV_F32: fp32 in/out, fp32 accumulate, CUDA cores.
 *    dtype SVCONV_BF16: bf16 in/out, fp32 accumulate on tcgen05 tensor cores;
 *    requires C_in % 64 == 0 and C_out % 64 == 0 and 16-byte aligned pointers.
 *    Unsupported shapes are rejected with SVCONV_ERR_UNSUPPORTED (no fallback).
 *  - Return value: SVCONV_OK (0) or a negative host-detected error.  Problems found
 *    inside kernels (bad coordinates, an index outside the table, a bounded wait
 *    that ran out) never fault: they set bits in a device status word (see
 *    SVCONV_STATUS_*) and leave the outputs undefined.
 */
#ifndef SVCONV_H_
#define SVCONV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SVCONV_API __attribute__((visibility("default")))
#else
#define SVCONV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* element types */
#define SVCONV_F32 0
#define SVCONV_BF16 1
#define SVCONV_E4M3 2 /* svconv_fwd only: 8-bit float (4 exponent, 3 mantissa bits) X and W */

/* host-side return codes */
#define SVCONV_OK 0
#define SVCONV_ERR_NULL (-1)        /* a required pointer is NULL */
#define SVCONV_ERR_SIZE (-2)        /* negative or too large size / count */
#define SVCONV_ERR_UNSUPPORTED (-3) /* dtype or channel count not supported */
#define SVCONV_ERR_ALIGN (-4)       /* pointer not 16-byte aligned (bf16 paths) */
#define SVCONV_ERR_WORKSPACE (-5)   /* workspace NULL or smaller than the query says */
#define SVCONV_ERR_CUDA (-6)        /* CUDA runtime / launch error */
#define SVCONV_ERR_DEVICE (-7)      /* current device is not an sm_100 GPU */

/* device status bits (OR-ed into an int32 word in device memory) */
#define SVCONV_STATUS_BAD_COORD 1       /* y or x outside the H x W frame */
#define SVCONV_STATUS_DUPLICATE 2       /* two tokens at the same (t, y, x) */
#define SVCONV_STATUS_BAD_FRAME 4       /* coords[k].t differs from the frame holding k */
#define SVCONV_STATUS_BAD_OFFSETS 8     /* frame_off not 0..n and non-decreasing */
#define SVCONV_STATUS_TIMEOUT 16        /* a kernel's bounded wait ran out; it returned early */
#define SVCONV_STATUS_BAD_INDEX 32      /* a neighbour index outside the feature rows; read as 0 */
#define SVCONV_STATUS_CHUNK_OVERFLOW 64 /* adapter chunk holds more rows than max_chunk_rows */

/*
 * Neighbour-index build (Key Design 1: the lookup map M per frame, filled with -1,
 * then M[y_k, x_k] = k; then N[k, j] = M[y_k+dy_j, x_k+dx_j], or -1 when the
 * neighbour was pruned or is out of bounds).  Each CTA keeps the maps of a few
 * consecutive frames in shared memory; nothing returns to the host.
 *   coords     [n][3] int32 device, frame_off [T+1] int32 device.
 *   nbr        [n][9] int32 device, written.
 *   M          [T][H][W] int32 device or NULL; if given, written with the map
 *              (global packed indices, -1 elsewhere).  With duplicate
 *              coordinates the cell holds the largest k and DUPLICATE is set.
 *   dev_status int32 device or NULL; SVCONV_STATUS_BAD_* bits are OR-ed in (the
 *              caller zeroes it).  Rows of tokens with bad coordinates are -1.
 *              Frames are validated independently, so when BAD_OFFSETS is set
 *              other bits may be set as well and nbr / M are undefined.
 *   Limits: H*W <= 16384, T >= 0, 0 <= n <= (2^31 - 1) / 9.
 */
SVCONV_API int svconv_build_index(const int32_t* coords, const int32_t* frame_off, int T, int H, int W, int n,
                       int32_t* nbr, int32_t* M, int32_t* dev_status, void* stream);

/*
 * Forward (Key Design 2: y_k = sum_j W_j x[N[k,j]], N = -1 read as zero padding),
 * plus an optional bias: Y[k][o] = bias[o] + sum_j sum_i W[o][j][i] * X[N[k][j]][i].
 *   X [n][Cin], Y [n][Cout] of dtype; Wt [Cout][9][Cin] of dtype;
 *   bias [Cout] fp32 device or NULL.  Y must not alias X.
 *   fp32 limit: 9*Cin*Cout <= 49152.  bf16: Cin, Cout multiples of 64, Cout <= 4096.
 *   SVCONV_E4M3 (large-channel inference): X [n][Cin] and Wt [Cout][9][Cin] hold e4m3
 *   values (1 byte each), bias fp32, Y is BF16; products are exact and accumulate in
 *   fp32 on the tensor cores (kind::f8f6f4, twice the bf16 rate).  Cin a multiple of
 *   128 and Cout of 256 (both <= 4096); no scaling factors are applied.
 *   bf16 launches: persistent, at most one CTA per SM; output tiles of 256 columns run on
 *   clusters of two CTAs (a pair of SMs shares each 256-row tile), so the device must
 *   allow 2-CTA clusters for those shapes.
 */
SVCONV_API int svconv_fwd(int dtype, const void* X, const int32_t* nbr, int n, int Cin, int Cout, const void* Wt,
               const float* bias, void* Y, void* stream);

/*
 * Backward w.r.t. the input features.  The page names backward kernels but prints
 * no formula; this is the adjoint of svconv_fwd written as a GATHER through the
 * mirrored offset:  dX[k] = sum_j W_j^T dY[N[k][8-j]]  (N[m][j] = k  <=>  N[k][8-j] = m
 * for tokens of one frame), so it is deterministic and uses no atomics.
 *   dY [n][Cout], dX [n][Cin] of dtype; Wt as in svconv_fwd.  dX must not alias dY.
 *   Limits as svconv_fwd.  No workspace.
 */
SVCONV_API int svconv_bwd_data(int dtype, const void* dY, const int32_t* nbr, int n, int Cin, int Cout, const void* Wt,
                    void* dX, void* stream);

/*
 * Backward w.r.t. the weights and bias (adjoint of svconv_fwd):
 *   dW[o][j][i] = sum_k dY[k][o] * X[N[k][j]][i],   db[o] = sum_k dY[k][o].
 * A GEMM over K = n tokens with the gather on the X side, split over token ranges
 * into fp32 partials in the workspace, then reduced in a fixed order: the result
 * is deterministic (bitwise identical across runs) and atomic-free.
 *   dY [n][Cout], X [n][Cin] of dtype; dW [Cout][9][Cin] fp32 and db [Cout] fp32
 *   (db may be NULL) are overwritten.
 *   workspace: device, at least svconv_bwd_weight_workspace_size(...) bytes,
 *   16-byte aligned, no initial contents required.
 */
SVCONV_API int svconv_bwd_weight(int dtype, const void* dY, const void* X, const int32_t* nbr, int n, int Cin, int Cout,
                      float* dW, float* db, void* workspace, size_t ws_bytes, void* stream);
SVCONV_API size_t svconv_bwd_weight_workspace_size(int dtype, int n, int Cin, int Cout);

/*
 * Allocation-free weight / bias gradient.  The paper has no counterpart: this is a
 * convenience for callers that cannot allocate device memory at call time (a
 * service with a fixed memory budget that must not call cudaMalloc after start-up,
 * a plugin that cannot reach its host framework's allocator, a callback where an
 * allocation would synchronise the device).  It computes exactly what
 * svconv_bwd_weight computes, same arguments minus the workspace: the split
 * partials live in a fixed device array of SVCONV_NOALLOC_SCRATCH_BYTES inside the
 * library.  CUDA loads the library's device code on a device lazily, so the array
 * is taken on a device when that happens, at the latest by the first call of this
 * entry point there (an empty call, n = 0, counts), and is then held until the
 * process exits.
 *   - Make the first call on each device at start-up, before any stream capture:
 *     it looks up the array's address and so commits the 16 MiB.
 *   - All calls share the array: calls that overlap on the GPU race.  Serialise them.
 *   - If the usual number of token splits does not fit, fewer are used (a different
 *     summation order, same tolerance); if one split's partials
 *     (640 * Cin / 64 rows of Cout floats for bf16, 9 * Cin + 1 rows for fp32)
 *     exceed the array, it returns SVCONV_ERR_SIZE.
 *   - It calls no cudaMalloc / cudaFree and no allocating library routine.
 */
#define SVCONV_NOALLOC_SCRATCH_BYTES (16u << 20)
SVCONV_API int svconv_bwd_weight_noalloc(int dtype, const void* dY, const void* X, const int32_t* nbr, int n, int Cin,
                                         int Cout, float* dW, float* db, void* stream);

/*
 * Fused backward: the data gradient of svconv_bwd_data and the weight / bias
 * gradients of svconv_bwd_weight in one call (SV-TAD page, Key Design 2: the
 * dedicated backward kernels; both are the adjoints of the forward).
 *   Arguments as in those two calls; dX [n][Cin] of dtype, dW [Cout][9][Cin] and
 *   db [Cout] fp32 (db may be NULL) are overwritten.
 *   workspace: device, at least svconv_bwd_workspace_size(...) bytes, 16-byte
 *   aligned, no initial contents required.
 *   bf16 with C_in = C_out = 64, and bf16 with C_in, C_out multiples of 256 (up to
 *   4096) when a cost model of the two kernels says it is shorter (CTA budgets from
 *   the measured per-stage cycles; at C = 256 and ~49k tokens the data gradient gets
 *   68 SMs and the weight gradient 80): the two gradients run side by side on disjoint
 *   groups of SMs, the weight gradient on a side stream of the library that is
 *   forked from and joined back to `stream` with events, so the call stays ordered
 *   on `stream` and can be captured in a CUDA graph.  Each (device, caller stream)
 *   pair gets its own side stream and events, created by the first such call on
 *   that stream OUTSIDE stream capture; a call made while `stream` is being
 *   captured before it has a side stream (or once 64 caller streams of a device
 *   have one) runs the same two launches one after the other on `stream` instead,
 *   with bitwise the same results.  Calls from several host threads on different
 *   streams, one of them capturing, neither wait on nor enter each other's work.
 *   dX is bitwise identical to svconv_bwd_data's; dW / db use fewer token splits
 *   than svconv_bwd_weight (another fixed summation order: deterministic, same
 *   tolerance; svconv_bwd_workspace_size gives the size for this call's split).
 *   Other shapes and fp32 run the two calls in order on `stream`.
 *   Errors: as the two calls.
 */
SVCONV_API int svconv_bwd(int dtype, const void* dY, const void* X, const int32_t* nbr, int n, int Cin, int Cout,
                          const void* Wt, void* dX, float* dW, float* db, void* workspace, size_t ws_bytes,
                          void* stream);
SVCONV_API size_t svconv_bwd_workspace_size(int dtype, int n, int Cin, int Cout);

/*
 * Both gradients of a bf16 convolution with C_in = C_out = 64 in ONE pass over dY
 * (SV-TAD page, Key Design 2, the dedicated backward kernels): one kernel loads each
 * 128-token tile's dY window once and uses it for the mirrored gather of dX and, in
 * place, as the B operand of the dW MMAs; the 640 x 64 fp32 dW accumulators stay in
 * tensor memory for every tile of a CTA and become that CTA's split partial; a
 * fixed-order reduce over the partials gives dW and db.  Deterministic.  It reads dY
 * and the neighbour table once instead of twice, but on this GPU the side-by-side
 * schedule of svconv_bwd finishes sooner at the workloads measured, so svconv_bwd
 * does not use it.
 *   dY, X [n][64] bf16; Wt [64][9][64] bf16; dX [n][64] bf16; dW [64][9][64] fp32 and
 *   db [64] fp32 (db may be NULL) overwritten; all device, 16-byte aligned.
 *   workspace: >= svconv_bwd_single_pass_workspace_size(n) bytes, no initial contents.
 */
SVCONV_API int svconv_bwd_single_pass(const void* dY, const void* X, const int32_t* nbr, int n, const void* Wt,
                                      void* dX, float* dW, float* db, void* workspace, size_t ws_bytes, void* stream);
SVCONV_API size_t svconv_bwd_single_pass_workspace_size(int n);

/*
 * Chunked bottleneck adapter forward (Key Design 2, "chunked execution" that
 * keeps memory flat in the number of frames; the adapter is the "lightweight
 * bottleneck adapter" with "down-projected" features of the Overall Architecture
 * and Key Design 3).  For each chunk of chunk_T frames, in order:
 *     H1 = bf16(X Wd^T)                         Wd [R][D]
 *     H2 = bf16(GELU(SparseConv3x3(H1) + bc))   Wc [R][9][R], bc [R] fp32 or NULL
 *     X  = bf16(X + H2 Wu^T)   (in place)       Wu [D][R]
 * GELU is the erf form 0.5 x (1 + erf(x / sqrt 2)).  All of X, Wd, Wc, Wu are
 * bf16; accumulation is fp32.
 *   X          [n][D] bf16 device, read and overwritten in place.
 *   nbr        [n][9] global neighbour table (svconv_build_index).
 *   frame_off  [T+1] int32 DEVICE; chunk bounds are read on the device.
 *   max_chunk_rows  upper bound on the tokens of any chunk; a larger chunk sets
 *              SVCONV_STATUS_CHUNK_OVERFLOW and only its first max_chunk_rows rows
 *              are processed.
 *   workspace  >= svconv_adapter_workspace_size(R, max_chunk_rows) bytes.
 *   dev_status int32 device or NULL (status bits are OR-ed in).
 *   Limits: D, R multiples of 64, R <= 4096.
 */
SVCONV_API int svconv_adapter_fwd(void* X, const int32_t* nbr, const int32_t* frame_off, int T, int n, int D, int R,
                       const void* Wd, const void* Wc, const float* bc, const void* Wu, int chunk_T,
                       int max_chunk_rows, void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream);
SVCONV_API size_t svconv_adapter_workspace_size(int R, int max_chunk_rows);

/*
 * Asymmetric cross-attention of auxiliary tokens (SV-TAD page, Key Design 3,
 * "Asymmetric Cross-Attention for Temporal Recombination": auxiliary tokens such as
 * the CLS token are the queries, the down-projected sparse visual features the keys
 * and values, and only the auxiliary tokens are updated).  Per group g (a video) and
 * auxiliary token a, with the R channels split into `heads` heads of d = R / heads:
 *     aux_out[g][a] = aux[g][a] + softmax_r(aux[g][a] . H[r] / sqrt(d)) H[r]
 * over the group's rows r = group_off[g] .. group_off[g+1]-1 (per head); a group
 * with no rows leaves its tokens unchanged.  No extra projections are applied.
 *   H          [n][R] bf16 device (keys = values), 16-byte aligned.
 *   group_off  [G+1] int32 DEVICE (CSR over the rows of H).
 *   max_group_rows  upper bound on any group's rows; a larger group sets
 *              SVCONV_STATUS_CHUNK_OVERFLOW and only its first rows are used.
 *   aux        [G][A][R] bf16 device; aux_out [G][A][R] fp32 device.
 *   workspace  >= svconv_xattn_workspace_size(G, max_group_rows, A) bytes; the
 *              per-block softmax partials (max, sum, weighted row sum) live there
 *              and are merged in a fixed order (bitwise reproducible).
 *   dev_status int32 device or NULL (SVCONV_STATUS_* bits OR-ed in).
 *   Limits: R a multiple of 8, 8 <= R <= 256; 1 <= A <= 16; R / heads a multiple
 *   of 8 with R / heads / 8 a power of two.  CUDA cores (HBM-bound: each row of H
 *   is read once).
 */
SVCONV_API int svconv_xattn_aux(const void* H, int n, int R, const int32_t* group_off, int G, int max_group_rows,
                                const void* aux, int A, int heads, float* aux_out, void* workspace, size_t ws_bytes,
                                int32_t* dev_status, void* stream);
SVCONV_API size_t svconv_xattn_workspace_size(int G, int max_group_rows, int A);

/*
 * The chunked adapter forward of svconv_adapter_fwd with the auxiliary-token
 * cross-attention inside it (Key Design 3: the cross-attention sits in the
 * bottleneck adapter, over the down-projected features).  The whole sequence of T
 * frames is one video: after each chunk's down-projection H1 = bf16(X Wd^T), the
 * auxiliary tokens' softmax partials over that chunk's rows of H1 are taken (H1 is
 * still in L2), and after the last chunk they are merged:
 *     aux_out[a] = aux[a] + softmax_r(aux[a] . H1[r] / sqrt(d)) H1[r]  over all n rows,
 * H1 being the down-projection of the adapter's INPUT X.  X is updated in place
 * exactly as by svconv_adapter_fwd.
 *   aux [A][R] bf16 device, aux_out [A][R] fp32 device; heads as svconv_xattn_aux.
 *   workspace >= svconv_adapter_xattn_workspace_size(T, R, chunk_T, max_chunk_rows, A).
 *   Other arguments and limits as svconv_adapter_fwd and svconv_xattn_aux.
 */
SVCONV_API int svconv_adapter_fwd_xattn(void* X, const int32_t* nbr, const int32_t* frame_off, int T, int n, int D,
                                        int R, const void* Wd, const void* Wc, const float* bc, const void* Wu,
                                        int chunk_T, int max_chunk_rows, const void* aux, int A, int heads,
                                        float* aux_out, void* workspace, size_t ws_bytes, int32_t* dev_status,
                                        void* stream);
SVCONV_API size_t svconv_adapter_xattn_workspace_size(int T, int R, int chunk_T, int max_chunk_rows, int A);

/*
 * The library's own device error word (per device): kernels without a caller
 * status pointer (fwd, bwd_data, bwd_weight) OR SVCONV_STATUS_TIMEOUT and
 * SVCONV_STATUS_BAD_INDEX into it.  Reading it synchronizes the current device,
 * copies the word to *out and clears it.
 */
SVCONV_API int svconv_read_error_word(int32_t* out);

/*
 * Failure-detection check: launches one CTA whose mbarrier wait can never
 * complete (nothing arrives), bounded by timeout_us microseconds.  The kernel
 * gives up, records SVCONV_STATUS_TIMEOUT into *dev_status and returns normally,
 * leaving the context usable.
 */
SVCONV_API int svconv_selftest_timeout(int32_t* dev_status, int timeout_us, void* stream);

/* Static text for a return code or a status bit. */
SVCONV_API const char* svconv_status_str(int code);

/* Library ABI version (major * 100 + minor). */
SVCONV_API int svconv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SVCONV_H_ */

// Fused backward entry point (svconv_bwd): the data gradient and the weight / bias
// gradients of one SparseConv2D in a single call (SV-TAD page, Key Design 2: dedicated
// backward kernels; the formulas are the adjoints of the forward).
//
// Both gradients read the same dY and neighbour table and do not depend on each other.
// At 64 input and output channels both kernels are latency-bound (each CTA waits ~3 us
// for its first operands and carries one or two tiles), so running them side by side on
// disjoint groups of SMs finishes sooner than running them one after the other: the data
// gradient takes about 3/8 of the SMs on the caller's stream, the weight gradient and its
// split reduce the rest on a side stream owned by the library, joined back to the caller's
// stream with events.  Other shapes, and fp32, run the two entry points in order on the
// caller's stream.
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "svconv.h"
#include "svconv_internal.h"

namespace svc {
namespace {

constexpr int kMaxSideStreams = 64;  // per device; further caller streams run the two kernels in order

// One side stream (and its fork / join events) per (device, caller stream).  A side stream is
// forked from and joined back to exactly one caller stream, so a stream capture on one caller
// stream never pulls in, or waits on, work that another caller stream queued, and unrelated
// caller streams are never ordered against each other through the library.
struct SideStream {
  int device = -1;
  cudaStream_t caller = nullptr;
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
std::vector<SideStream> g_side;
std::mutex g_side_mu;  // guards the table and each call's fork / launch / join sequence

bool concurrent_shape(int dtype, int Cin, int Cout) { return dtype == SVCONV_BF16 && Cin == 64 && Cout == 64; }

// CTA budgets: weight gradient 94 of 148 SMs, data gradient the rest (measured best split).
void budgets(int* data_ctas, int* weight_ctas) {
  const int sms = sm_count();
  int w = sms * 94 / 148;
  if (w < 5) w = 5;
  int d = sms - w;
  if (d < 1) d = 1;
  *data_ctas = d;
  *weight_ctas = w;
}

// Side stream of (current device, caller), created on first use (call with g_side_mu held).
// Returns nullptr when none can be used: the caller stream is being captured and has no side
// stream yet (creating one inside a capture is not done), the table is full, or creation failed.
SideStream* side_stream(cudaStream_t caller) {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return nullptr;
  int per_dev = 0;
  for (SideStream& r : g_side) {
    if (r.device != d) continue;
    if (r.caller == caller) return &r;
    ++per_dev;
  }
  if (per_dev >= kMaxSideStreams) return nullptr;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(caller, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) return nullptr;
  SideStream r;
  r.device = d;
  r.caller = caller;
  if (cudaStreamCreateWithFlags(&r.stream, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
  if (cudaEventCreateWithFlags(&r.fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&r.join, cudaEventDisableTiming) != cudaSuccess) {
    if (r.fork) cudaEventDestroy(r.fork);
    cudaStreamDestroy(r.stream);
    return nullptr;
  }
  g_side.push_back(r);
  return &g_side.back();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace svc

using namespace svc;

extern "C" {

size_t svconv_bwd_workspace_size(int dtype, int n, int Cin, int Cout) {
  if (!concurrent_shape(dtype, Cin, Cout) || n <= 0) return svconv_bwd_weight_workspace_size(dtype, n, Cin, Cout);
  int dc, wc, splits, rows_pad, bn;
  budgets(&dc, &wc);
  tc_wgrad_plan_ctas(n, Cin, Cout, wc, &splits, &rows_pad, &bn);
  return (size_t)splits * rows_pad * Cout * sizeof(float);
}

int svconv_bwd(int dtype, const void* dY, const void* X, const int32_t* nbr, int n, int Cin, int Cout,
               const void* Wt, void* dX, float* dW, float* db, void* workspace, size_t ws_bytes, void* stream) {
  if (n < 0 || Cin <= 0 || Cout <= 0) return SVCONV_ERR_SIZE;
  if (!concurrent_shape(dtype, Cin, Cout) || n == 0) {
    const int rc = svconv_bwd_data(dtype, dY, nbr, n, Cin, Cout, Wt, dX, stream);
    if (rc) return rc;
    return svconv_bwd_weight(dtype, dY, X, nbr, n, Cin, Cout, dW, db, workspace, ws_bytes, stream);
  }
  if (!dY || !X || !nbr || !Wt || !dX || !dW) return SVCONV_ERR_NULL;
  int major = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return SVCONV_ERR_CUDA;
  if (major != 10) return SVCONV_ERR_DEVICE;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(Wt) || !aligned16(dX)) return SVCONV_ERR_ALIGN;
  if (!workspace || ws_bytes < svconv_bwd_workspace_size(dtype, n, Cin, Cout)) return SVCONV_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SVCONV_ERR_ALIGN;
  int dc, wc;
  budgets(&dc, &wc);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lk(g_side_mu);
  SideStream* side = side_stream(s);
  if (!side) {
    // no side stream for this caller stream: the same two launches (same CTA budgets, so
    // bitwise the same results) one after the other on the caller's stream
    const int rc = tc_bwd_data(dY, nbr, n, Cin, Cout, Wt, dX, dc, s);
    if (rc) return rc;
    return tc_bwd_weight(dY, X, nbr, n, Cin, Cout, dW, db, static_cast<float*>(workspace), wc, s);
  }
  // fork: the side stream waits for everything before this call on the caller's stream
  if (cudaEventRecord(side->fork, s) != cudaSuccess || cudaStreamWaitEvent(side->stream, side->fork, 0) != cudaSuccess)
    return SVCONV_ERR_CUDA;
  const int rc_data = tc_bwd_data(dY, nbr, n, Cin, Cout, Wt, dX, dc, s);
  const int rc_weight = tc_bwd_weight(dY, X, nbr, n, Cin, Cout, dW, db, static_cast<float*>(workspace), wc,
                                      side->stream);
  // join: the caller's stream waits for the side stream's work (also after a failed launch)
  if (cudaEventRecord(side->join, side->stream) != cudaSuccess || cudaStreamWaitEvent(s, side->join, 0) != cudaSuccess)
    return SVCONV_ERR_CUDA;
  return rc_data ? rc_data : rc_weight;
}

}  // extern "C"

// ---------------------------------------------------------------------------- single pass over dY
// Both gradients at C_in = C_out = 64 from ONE pass over dY (tc_bwd_small_kernel): each
// 128-token tile's dY window is loaded once and feeds the mirrored gather of dX and, in place,
// the MMAs of dW, whose accumulators stay in tensor memory for all tiles of a CTA; then the
// fixed-order split reduce over the CTAs' partials.  It moves the least data, but one CTA does
// both gradients of a tile one stage after the other, and its split partials (one 640 x 64
// block per CTA) make the reduce larger, so svconv_bwd keeps the two kernels side by side.

extern "C" {

size_t svconv_bwd_single_pass_workspace_size(int n) {
  if (n <= 0) return 0;
  int d = 0, major = 0;
  if (cudaGetDevice(&d) != cudaSuccess || cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, d) != cudaSuccess)
    return 0;
  return tc_bwd_small_partial_floats(n) * sizeof(float);
}

int svconv_bwd_single_pass(const void* dY, const void* X, const int32_t* nbr, int n, const void* Wt, void* dX,
                           float* dW, float* db, void* workspace, size_t ws_bytes, void* stream) {
  if (n < 0) return SVCONV_ERR_SIZE;
  if (!dW) return SVCONV_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n == 0) {  // empty sums: zero gradients
    cudaError_t e = cudaMemsetAsync(dW, 0, sizeof(float) * 9 * 64 * 64, s);
    if (e == cudaSuccess && db) e = cudaMemsetAsync(db, 0, sizeof(float) * 64, s);
    return e == cudaSuccess ? SVCONV_OK : SVCONV_ERR_CUDA;
  }
  if (!dY || !X || !nbr || !Wt || !dX) return SVCONV_ERR_NULL;
  int major = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return SVCONV_ERR_CUDA;
  if (major != 10) return SVCONV_ERR_DEVICE;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(Wt) || !aligned16(dX)) return SVCONV_ERR_ALIGN;
  if (!workspace || ws_bytes < svconv_bwd_single_pass_workspace_size(n)) return SVCONV_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SVCONV_ERR_ALIGN;
  const cudaError_t e = launch_tc_bwd_small(dY, X, nbr, n, Wt, dX, static_cast<float*>(workspace), dW, db, s);
  return e == cudaSuccess ? SVCONV_OK : SVCONV_ERR_CUDA;
}

}  // extern "C"

// Fused backward entry point (svconv_bwd): the data gradient and the weight / bias
// gradients of one SparseConv2D in a single call (SV-TAD page, Key Design 2: dedicated
// backward kernels; the formulas are the adjoints of the forward).
//
// Both gradients read the same dY and neighbour table and do not depend on each other, so
// they can run side by side on disjoint groups of SMs: the data gradient on the caller's
// stream, the weight gradient and its split reduce on a side stream owned by the library,
// joined back to the caller's stream with events.
// * 64 input and output channels: both kernels are latency-bound (each CTA waits ~3 us for
//   its first operands and carries one or two tiles); the data gradient takes about 3/8 of
//   the SMs (measured best split).
// * Multiples of 256 channels (CTA-pair kernels): a cost model picks the split.  Each kernel
//   alone on the whole GPU pays its start and end once, and the data gradient's 256-row tiles
//   rarely fill the last wave of 74 clusters; side by side, the data gradient gets the
//   clusters that leave its waves full and the weight gradient a whole number of token
//   splits (fewer partials to reduce).
// Other shapes, and fp32, run the two entry points in order on the caller's stream.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
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

// How svconv_bwd runs the two gradients: side by side with these CTA budgets, or in order.
struct BwdPlan {
  bool side_by_side = false;
  int data_ctas = 0, weight_ctas = 0;
};

// Cost model of the 256-column CTA-pair kernels, in SM cycles of one cluster (per-stage clock
// traces on B200): a data-gradient tile of 256 rows costs ~580 cycles per 64-deep K-block plus
// ~3,300 at its boundary (the epilogue drains the single accumulator); a weight-gradient unit
// ~850 cycles per 64-token block; a kernel ~15,000 cycles of start (first loads) and end (last
// epilogue); the split reduce ~1 cycle per 1,800 bytes of fp32 partials.
constexpr double kDxKbCycles = 580.0, kDxTileCycles = 3300.0, kDwBlockCycles = 850.0, kKernelCycles = 15000.0;
constexpr double kReduceBytesPerCycle = 1800.0;

BwdPlan plan_bwd(int dtype, int n, int Cin, int Cout) {
  BwdPlan p;
  if (dtype != SVCONV_BF16 || n <= 0) return p;
  const int sms = sm_count();
  if (Cin == 64 && Cout == 64) {
    // weight gradient 94 of 148 SMs, data gradient the rest
    int w = sms * 94 / 148;
    if (w < 5) w = 5;
    int d = sms - w;
    if (d < 1) d = 1;
    p.side_by_side = true;
    p.data_ctas = d;
    p.weight_ctas = w;
    return p;
  }
  // (widths the entry points accept: the side-by-side call skips their checks)
  if (Cin % 256 != 0 || Cout % 256 != 0 || Cin > 4096 || Cout > 4096) return p;
  const int clusters = sms / 2;
  const double tiles = (double)((n + 255) / 256) * (Cin / 256);               // data-gradient pair tiles
  const double tile_cycles = 9.0 * Cout / 64 * kDxKbCycles + kDxTileCycles;
  const int units = (Cin / 64) * 5 / 2 * (Cout / 256);                         // weight pair units per split
  const double blocks = (double)((n + 63) / 64);
  const double split_bytes = (double)(Cin / 64) * 5 * 128 * Cout * 4;         // one split's fp32 partial
  auto t_weight = [&](int s) { return std::ceil(blocks / s) * kDwBlockCycles + kKernelCycles + s * split_bytes / kReduceBytesPerCycle; };
  auto t_data = [&](int c) { return std::ceil(tiles / c) * tile_cycles + kKernelCycles; };
  int s_full, rows_pad, bn;
  tc_wgrad_plan(n, Cin, Cout, &s_full, &rows_pad, &bn);
  double best = t_data(clusters) + t_weight(s_full);  // one after the other, each on the whole GPU
  for (int s = 1; units * s < clusters && s <= (int)blocks; ++s) {
    const int cx = clusters - units * s;
    const double t = std::max(t_data(cx), t_weight(s));
    if (t < 0.97 * best) {
      best = t;
      p.side_by_side = true;
      p.data_ctas = 2 * cx;
      p.weight_ctas = 2 * units * s;
    }
  }
  return p;
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
  if (n <= 0 || Cin <= 0 || Cout <= 0) return svconv_bwd_weight_workspace_size(dtype, n, Cin, Cout);
  const BwdPlan plan = plan_bwd(dtype, n, Cin, Cout);
  if (!plan.side_by_side) return svconv_bwd_weight_workspace_size(dtype, n, Cin, Cout);
  int splits, rows_pad, bn;
  tc_wgrad_plan_ctas(n, Cin, Cout, plan.weight_ctas, &splits, &rows_pad, &bn);
  return (size_t)splits * rows_pad * Cout * sizeof(float);
}

int svconv_bwd(int dtype, const void* dY, const void* X, const int32_t* nbr, int n, int Cin, int Cout,
               const void* Wt, void* dX, float* dW, float* db, void* workspace, size_t ws_bytes, void* stream) {
  if (n < 0 || Cin <= 0 || Cout <= 0) return SVCONV_ERR_SIZE;
  const BwdPlan plan = plan_bwd(dtype, n, Cin, Cout);
  if (!plan.side_by_side) {
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
  const int dc = plan.data_ctas, wc = plan.weight_ctas;
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

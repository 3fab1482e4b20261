// Fused backward entry point (svconv_bwd): the data gradient and the weight / bias
// gradients of one SparseConv2D in a single call (SV-TAD page, Key Design 2: dedicated
// backward kernels; the formulas are the adjoints of the forward).
//
// bf16 with C_in = C_out = 64: one kernel makes one pass over dY for both gradients (each
// tile's dY window feeds the mirrored gather of the data gradient and, in place, the weight
// gradient's MMAs; tc_bwd_small_kernel), then the fixed-order split reduce.  At this width
// both gradients are latency-bound, so sharing the loads and the launch is what counts.
// Other shapes, and fp32, run svconv_bwd_data and svconv_bwd_weight in order on the stream.
#include <cuda_runtime.h>

#include "svconv.h"
#include "svconv_internal.h"

namespace svc {
namespace {

bool single_pass_shape(int dtype, int Cin, int Cout) { return dtype == SVCONV_BF16 && Cin == 64 && Cout == 64; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace svc

using namespace svc;

extern "C" {

size_t svconv_bwd_workspace_size(int dtype, int n, int Cin, int Cout) {
  if (!single_pass_shape(dtype, Cin, Cout) || n <= 0) return svconv_bwd_weight_workspace_size(dtype, n, Cin, Cout);
  int d = 0, major = 0;
  if (cudaGetDevice(&d) != cudaSuccess || cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, d) != cudaSuccess)
    return 0;
  return tc_bwd_small_partial_floats(n) * sizeof(float);
}

int svconv_bwd(int dtype, const void* dY, const void* X, const int32_t* nbr, int n, int Cin, int Cout,
               const void* Wt, void* dX, float* dW, float* db, void* workspace, size_t ws_bytes, void* stream) {
  if (n < 0 || Cin <= 0 || Cout <= 0) return SVCONV_ERR_SIZE;
  if (!single_pass_shape(dtype, Cin, Cout) || n == 0) {
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
  const cudaError_t e = launch_tc_bwd_small(dY, X, nbr, n, Wt, dX, static_cast<float*>(workspace), dW, db,
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SVCONV_OK : SVCONV_ERR_CUDA;
}

}  // extern "C"

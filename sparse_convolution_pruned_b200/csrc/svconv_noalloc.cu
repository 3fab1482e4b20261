// Allocation-free variant of the weight / bias gradient (svconv_bwd_weight_noalloc).
//
// The ordinary entry point takes its split-partial workspace from the caller.
// Some callers cannot provide one: code that must not call cudaMalloc after
// start-up (a real-time or fixed-budget service, a plugin running under another
// framework's memory manager that it cannot reach, a callback where an allocation
// would synchronise the device).  This variant keeps the partials in a fixed
// file-scope device array instead, so the caller passes only inputs and outputs.
//
// The array is SVCONV_NOALLOC_SCRATCH_BYTES (16 MiB) per device.  CUDA loads a
// library's device code on a device lazily, so the array is committed on a device
// when the library's module is first loaded there: at the latest by the first call
// of this entry point on that device, which looks up the array's device address
// (cudaGetSymbolAddress, with that device current) before anything else, even for
// an empty input.  From then on it stays until the process exits.  Make that first
// call at start-up, before any stream capture.  All calls share the array: calls whose kernels overlap on
// the GPU (two streams, or two host threads) race and produce wrong gradients;
// serialise them.  No initial contents are needed: every call rewrites every
// partial it later reads.  If the default number of token splits does not fit,
// fewer splits are used (the sum order changes, the result stays within
// tolerance); if even one split does not fit, the call fails with
// SVCONV_ERR_SIZE.  Nothing here allocates memory.
#include <cuda_runtime.h>

#include <mutex>

#include "svconv.h"
#include "svconv_internal.h"

namespace svc {
namespace {

constexpr size_t kScratchFloats = SVCONV_NOALLOC_SCRATCH_BYTES / sizeof(float);
__device__ __align__(256) float g_noalloc_scratch[kScratchFloats];

constexpr int kMaxDev = 64;
float* g_scratch_addr[kMaxDev];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (looked up once per device).
float* scratch_address() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDev) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    g_scratch_addr[d] = static_cast<float*>(p);
  }
  return g_scratch_addr[d];
}

bool sm100_device() {
  int d = 0, major = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, d) != cudaSuccess) return false;
  return major == 10;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace svc

using namespace svc;

extern "C" int svconv_bwd_weight_noalloc(int dtype, const void* dY, const void* X, const int32_t* nbr, int n, int Cin,
                                         int Cout, float* dW, float* db, void* stream) {
  if (n < 0 || Cin <= 0 || Cout <= 0) return SVCONV_ERR_SIZE;
  if (!dW) return SVCONV_ERR_NULL;
  if (dtype != SVCONV_F32 && dtype != SVCONV_BF16) return SVCONV_ERR_UNSUPPORTED;
  if (dtype == SVCONV_BF16 && (Cin % 64 != 0 || Cout % 64 != 0 || Cin > 4096 || Cout > 4096))
    return SVCONV_ERR_UNSUPPORTED;
  if (!sm100_device()) return SVCONV_ERR_DEVICE;
  // Looked up first, so that any first call on a device (an empty one included) loads the
  // library's module there and with it commits the scratch array.
  float* partial = scratch_address();
  if (!partial) return SVCONV_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n == 0) {  // empty sum: zero gradients
    cudaError_t e = cudaMemsetAsync(dW, 0, sizeof(float) * 9 * (size_t)Cin * Cout, s);
    if (e == cudaSuccess && db) e = cudaMemsetAsync(db, 0, sizeof(float) * (size_t)Cout, s);
    return e == cudaSuccess ? SVCONV_OK : SVCONV_ERR_CUDA;
  }
  if (!dY || !X || !nbr) return SVCONV_ERR_NULL;

  int splits = 0, rows_pad = 0, bn = 0;
  if (dtype == SVCONV_BF16) {
    if (!aligned16(dY) || !aligned16(X)) return SVCONV_ERR_ALIGN;
    tc_wgrad_plan(n, Cin, Cout, &splits, &rows_pad, &bn);
  } else {
    splits = (int)f32_wgrad_splits(n);
    rows_pad = 9 * Cin + 1;
  }
  const size_t per_split = (size_t)rows_pad * Cout;  // floats
  const size_t fit = kScratchFloats / per_split;
  if (fit < 1) return SVCONV_ERR_SIZE;  // one split's partial rows exceed the fixed scratch
  if ((size_t)splits > fit) splits = (int)fit;

  cudaError_t e;
  if (dtype == SVCONV_F32) {
    e = launch_f32_wgrad_partials(static_cast<const float*>(dY), static_cast<const float*>(X), nbr, n, Cin, Cout,
                                  partial, splits, rows_pad, s);
  } else {
    TcWgradArgs a{};
    a.dY = dY;
    a.X = X;
    a.nbr = nbr;
    a.n = n;
    a.Cin = Cin;
    a.Cout = Cout;
    a.partial = partial;
    a.splits = splits;
    a.rows_pad = rows_pad;
    e = launch_tc_wgrad_with_splits(a, s);
  }
  if (e != cudaSuccess) return SVCONV_ERR_CUDA;
  e = launch_wgrad_reduce(partial, splits, rows_pad, Cin, Cout, dtype == SVCONV_BF16 ? 1 : 0, dW, db, s);
  return e == cudaSuccess ? SVCONV_OK : SVCONV_ERR_CUDA;
}

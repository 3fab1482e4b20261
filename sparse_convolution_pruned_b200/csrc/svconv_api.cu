// C ABI: argument validation, kernel dispatch and the chunked adapter schedule.
// Every entry point is asynchronous on the caller's stream and allocates no
// device memory (callers pass outputs and workspaces).
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "svconv.h"
#include "svconv_internal.h"

namespace svc {

// One error word per device (each device that loads the library gets its own copy).
__device__ int g_error_word;

namespace {
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
int g_major[kMaxDevices];
int* g_err_ptr[kMaxDevices];
std::mutex g_mu;

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}

// Caches the SM count, compute capability and the error word's address per device.
bool device_info(int d) {
  if (d < 0 || d >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_err_ptr[d]) return true;
  int sms = 0, major = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, d) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, d) != cudaSuccess) return false;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return false;
  g_sm_count[d] = sms;
  g_major[d] = major;
  g_err_ptr[d] = static_cast<int*>(p);
  return true;
}
}  // namespace

int* device_error_word() {
  const int d = current_device();
  return device_info(d) ? g_err_ptr[d] : nullptr;
}

int sm_count() {
  const int d = current_device();
  return device_info(d) ? g_sm_count[d] : 1;
}

static int check_device() {
  const int d = current_device();
  if (!device_info(d)) return SVCONV_ERR_CUDA;
  if (g_major[d] != 10) return SVCONV_ERR_DEVICE;
  return SVCONV_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int cuda_rc(cudaError_t e) { return e == cudaSuccess ? SVCONV_OK : SVCONV_ERR_CUDA; }

static bool bf16_channels_ok(int C) { return C > 0 && C % 64 == 0 && C <= 4096; }

// Output tile width for the tcgen05 conv kernel.
static int conv_bn(int N) { return N % 256 == 0 ? 256 : N % 128 == 0 ? 128 : 64; }

}  // namespace svc

using namespace svc;

namespace svc {
int tc_bwd_data(const void* dY, const int32_t* nbr, int n, int Cin, int Cout, const void* Wt, void* dX, int max_ctas,
                cudaStream_t s) {
  TcConvArgs a{};
  a.A = dY;
  a.lda = Cout;
  a.a_rows = n;
  a.nbr = nbr;
  a.taps = 9;
  a.mirror = 1;
  a.Kc = Cout;
  a.b_mn_major = 1;
  a.M = n;
  a.N = Cin;
  a.out = dX;
  a.ldo = Cin;
  a.out_rows = n;
  a.max_ctas = max_ctas;
  return cuda_rc(launch_tc_conv(a, Wt, 0, 0, conv_bn(Cin), s));
}

int tc_bwd_weight(const void* dY, const void* X, const int32_t* nbr, int n, int Cin, int Cout, float* dW, float* db,
                  float* partial, int ctas, cudaStream_t s) {
  TcWgradArgs a{};
  a.dY = dY;
  a.X = X;
  a.nbr = nbr;
  a.n = n;
  a.Cin = Cin;
  a.Cout = Cout;
  a.partial = partial;
  int bn;
  tc_wgrad_plan_ctas(n, Cin, Cout, ctas > 0 ? ctas : sm_count(), &a.splits, &a.rows_pad, &bn);
  cudaError_t e = launch_tc_wgrad_with_splits(a, s);
  if (e != cudaSuccess) return SVCONV_ERR_CUDA;
  return cuda_rc(launch_wgrad_reduce(partial, a.splits, a.rows_pad, Cin, Cout, 1, dW, db, s));
}
}  // namespace svc

extern "C" {

int svconv_version(void) { return 100; }

const char* svconv_status_str(int code) {
  switch (code) {
    case SVCONV_OK: return "ok";
    case SVCONV_ERR_NULL: return "a required pointer is NULL";
    case SVCONV_ERR_SIZE: return "size or count out of range";
    case SVCONV_ERR_UNSUPPORTED: return "dtype or channel count not supported";
    case SVCONV_ERR_ALIGN: return "pointer not 16-byte aligned";
    case SVCONV_ERR_WORKSPACE: return "workspace missing or too small";
    case SVCONV_ERR_CUDA: return "CUDA runtime or launch error";
    case SVCONV_ERR_DEVICE: return "current device is not sm_100";
    case SVCONV_STATUS_BAD_COORD: return "status: coordinate outside the frame";
    case SVCONV_STATUS_DUPLICATE: return "status: duplicate token coordinate";
    case SVCONV_STATUS_BAD_FRAME: return "status: token frame disagrees with frame_off";
    case SVCONV_STATUS_BAD_OFFSETS: return "status: frame_off not monotone 0..n";
    case SVCONV_STATUS_TIMEOUT: return "status: a bounded wait ran out";
    case SVCONV_STATUS_BAD_INDEX: return "status: neighbour index outside the feature rows";
    case SVCONV_STATUS_CHUNK_OVERFLOW: return "status: adapter chunk larger than max_chunk_rows";
    default: return "unknown code";
  }
}

int svconv_build_index(const int32_t* coords, const int32_t* frame_off, int T, int H, int W, int n, int32_t* nbr,
                       int32_t* M, int32_t* dev_status, void* stream) {
  if (T < 0 || n < 0 || H <= 0 || W <= 0 || (long long)H * W > 16384) return SVCONV_ERR_SIZE;
  if ((long long)n * 9 > 0x7fffffffLL) return SVCONV_ERR_SIZE;  // table entries are indexed with int32
  if (!frame_off || (n > 0 && (!coords || !nbr))) return SVCONV_ERR_NULL;
  int rc = check_device();
  if (rc) return rc;
  return cuda_rc(launch_build_index(coords, frame_off, T, H, W, n, nbr, M, dev_status, (cudaStream_t)stream));
}

int svconv_fwd(int dtype, const void* X, const int32_t* nbr, int n, int Cin, int Cout, const void* Wt,
               const float* bias, void* Y, void* stream) {
  if (n < 0 || Cin <= 0 || Cout <= 0) return SVCONV_ERR_SIZE;
  if (n == 0) return SVCONV_OK;
  if (!X || !nbr || !Wt || !Y) return SVCONV_ERR_NULL;
  if (dtype == SVCONV_E4M3 && (Cin % 128 != 0 || Cin > 4096 || Cout % 256 != 0 || Cout > 4096))
    return SVCONV_ERR_UNSUPPORTED;
  int rc = check_device();
  if (rc) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  if (dtype == SVCONV_F32) {
    if ((long long)9 * Cin * Cout > 49152) return SVCONV_ERR_UNSUPPORTED;
    return cuda_rc(launch_f32_conv(false, static_cast<const float*>(X), nbr, n, Cin, Cout,
                                   static_cast<const float*>(Wt), Cin, Cout, bias, static_cast<float*>(Y), s));
  }
  if (dtype == SVCONV_E4M3) {
    // e4m3 X and W, bf16 Y: the tensor-core gather on CTA pairs with K = 32 per MMA.  The
    // kernel moves bytes, so rows of e4m3 are described as rows of half as many 2-byte units.
    if (!aligned16(X) || !aligned16(Wt) || !aligned16(Y)) return SVCONV_ERR_ALIGN;
    TcConvArgs a{};
    a.A = X;
    a.lda = Cin / 2;
    a.a_rows = n;
    a.nbr = nbr;
    a.taps = 9;
    a.Kc = Cin / 2;
    a.M = n;
    a.N = Cout;
    a.bias = bias;
    a.out = Y;
    a.ldo = Cout;
    a.out_rows = n;
    a.f8 = 1;
    return cuda_rc(launch_tc_conv(a, Wt, Cout, 9 * Cin / 2, 256, s));
  }
  if (dtype != SVCONV_BF16) return SVCONV_ERR_UNSUPPORTED;
  if (!bf16_channels_ok(Cin) || !bf16_channels_ok(Cout)) return SVCONV_ERR_UNSUPPORTED;
  if (!aligned16(X) || !aligned16(Wt) || !aligned16(Y)) return SVCONV_ERR_ALIGN;
  TcConvArgs a{};
  a.A = X;
  a.lda = Cin;
  a.a_rows = n;
  a.nbr = nbr;
  a.taps = 9;
  a.mirror = 0;
  a.Kc = Cin;
  a.b_mn_major = 0;
  a.M = n;
  a.N = Cout;
  a.bias = bias;
  a.out = Y;
  a.ldo = Cout;
  a.out_rows = n;
  return cuda_rc(launch_tc_conv(a, Wt, Cout, 9 * Cin, conv_bn(Cout), s));
}

int svconv_bwd_data(int dtype, const void* dY, const int32_t* nbr, int n, int Cin, int Cout, const void* Wt,
                    void* dX, void* stream) {
  if (n < 0 || Cin <= 0 || Cout <= 0) return SVCONV_ERR_SIZE;
  if (n == 0) return SVCONV_OK;
  if (!dY || !nbr || !Wt || !dX) return SVCONV_ERR_NULL;
  int rc = check_device();
  if (rc) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  if (dtype == SVCONV_F32) {
    if ((long long)9 * Cin * Cout > 49152) return SVCONV_ERR_UNSUPPORTED;
    return cuda_rc(launch_f32_conv(true, static_cast<const float*>(dY), nbr, n, Cout, Cin,
                                   static_cast<const float*>(Wt), Cin, Cout, nullptr, static_cast<float*>(dX), s));
  }
  if (dtype != SVCONV_BF16) return SVCONV_ERR_UNSUPPORTED;
  if (!bf16_channels_ok(Cin) || !bf16_channels_ok(Cout)) return SVCONV_ERR_UNSUPPORTED;
  if (!aligned16(dY) || !aligned16(Wt) || !aligned16(dX)) return SVCONV_ERR_ALIGN;
  return tc_bwd_data(dY, nbr, n, Cin, Cout, Wt, dX, 0, s);
}



size_t svconv_bwd_weight_workspace_size(int dtype, int n, int Cin, int Cout) {
  if (n <= 0 || Cin <= 0 || Cout <= 0) return 0;
  if (dtype == SVCONV_F32) {
    const size_t rows = (size_t)9 * Cin + 1;
    return f32_wgrad_splits(n) * rows * Cout * sizeof(float);
  }
  if (dtype == SVCONV_BF16) {
    if (!bf16_channels_ok(Cin) || !bf16_channels_ok(Cout)) return 0;
    if (check_device()) return 0;
    int splits, rows_pad, bn;
    tc_wgrad_plan(n, Cin, Cout, &splits, &rows_pad, &bn);
    return (size_t)splits * rows_pad * Cout * sizeof(float);
  }
  return 0;
}

int svconv_bwd_weight(int dtype, const void* dY, const void* X, const int32_t* nbr, int n, int Cin, int Cout,
                      float* dW, float* db, void* workspace, size_t ws_bytes, void* stream) {
  if (n < 0 || Cin <= 0 || Cout <= 0) return SVCONV_ERR_SIZE;
  if (!dW) return SVCONV_ERR_NULL;
  int rc = check_device();
  if (rc) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  if (dtype != SVCONV_F32 && dtype != SVCONV_BF16) return SVCONV_ERR_UNSUPPORTED;
  if (dtype == SVCONV_BF16 && (!bf16_channels_ok(Cin) || !bf16_channels_ok(Cout))) return SVCONV_ERR_UNSUPPORTED;
  if (n == 0) {  // empty sum: zero gradients
    cudaError_t e = cudaMemsetAsync(dW, 0, sizeof(float) * 9 * (size_t)Cin * Cout, s);
    if (e == cudaSuccess && db) e = cudaMemsetAsync(db, 0, sizeof(float) * (size_t)Cout, s);
    return cuda_rc(e);
  }
  if (!dY || !X || !nbr) return SVCONV_ERR_NULL;
  const size_t need = svconv_bwd_weight_workspace_size(dtype, n, Cin, Cout);
  if (!workspace || ws_bytes < need) return SVCONV_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SVCONV_ERR_ALIGN;
  float* partial = static_cast<float*>(workspace);
  if (dtype == SVCONV_F32) {
    const int splits = (int)f32_wgrad_splits(n);
    const int rows = 9 * Cin + 1;
    cudaError_t e = launch_f32_wgrad_partials(static_cast<const float*>(dY), static_cast<const float*>(X), nbr, n,
                                              Cin, Cout, partial, splits, rows, s);
    if (e != cudaSuccess) return SVCONV_ERR_CUDA;
    return cuda_rc(launch_wgrad_reduce(partial, splits, rows, Cin, Cout, 0, dW, db, s));
  }
  if (!aligned16(dY) || !aligned16(X)) return SVCONV_ERR_ALIGN;
  return tc_bwd_weight(dY, X, nbr, n, Cin, Cout, dW, db, partial, 0, s);
}

size_t svconv_adapter_workspace_size(int R, int max_chunk_rows) {
  if (R <= 0 || max_chunk_rows <= 0) return 0;
  const size_t rows = ((size_t)max_chunk_rows + 127) / 128 * 128;
  return 2 * rows * (size_t)R * 2;  // H1 and H2, bf16
}

}  // extern "C"

namespace svc {
namespace {

// Auxiliary-token cross-attention riding on the adapter's chunks (nullptr: none).
struct AdapterXattn {
  const void* aux;
  int A, heads;
  float* aux_out;
  float* part;
  int blocks;    // partial slots per chunk
  int n_chunks;
};

int adapter_chunks(void* X, const int32_t* nbr, const int32_t* frame_off, int T, int n, int D, int R,
                   const void* Wd, const void* Wc, const float* bc, const void* Wu, int chunk_T, int max_chunk_rows,
                   void* workspace, int32_t* dev_status, const AdapterXattn* xa, cudaStream_t s) {
  const size_t rows_cap = ((size_t)max_chunk_rows + 127) / 128 * 128;
  void* H1 = workspace;
  void* H2 = static_cast<char*>(workspace) + rows_cap * (size_t)R * 2;
  int32_t* status = dev_status ? dev_status : device_error_word();
  int chunk = 0;
  for (int t0 = 0; t0 < T; t0 += chunk_T, ++chunk) {
    const int t1 = t0 + chunk_T < T ? t0 + chunk_T : T;
    // 1) H1 = X[rows] Wd^T  (dense, one tap)
    TcConvArgs d{};
    d.A = X;
    d.lda = D;
    d.a_rows = n;
    d.nbr = nullptr;
    d.taps = 1;
    d.Kc = D;
    d.M = max_chunk_rows;
    d.row_lo = frame_off + t0;
    d.row_hi = frame_off + t1;
    d.a_abs = 1;
    d.N = R;
    d.out = H1;
    d.ldo = R;
    d.out_rows = max_chunk_rows;
    d.status = status;
    cudaError_t e = launch_tc_conv(d, Wd, R, D, conv_bn(R), s);
    if (e != cudaSuccess) return SVCONV_ERR_CUDA;
    // 1b) auxiliary tokens attend over this chunk's down-projected rows (partials per block)
    if (xa) {
      XattnLaunch x{};
      x.H = H1;
      x.h_rows = max_chunk_rows;
      x.R = R;
      x.heads = xa->heads;
      x.lo = frame_off + t0;
      x.hi = frame_off + t1;
      x.h_sub = frame_off + t0;
      x.G = 1;
      x.max_rows = max_chunk_rows;
      x.aux = xa->aux;
      x.A = xa->A;
      x.part = xa->part;
      x.slot0 = chunk * xa->blocks;
      x.slots_per_group = xa->n_chunks * xa->blocks;
      x.status = status;
      e = launch_xattn_partials(x, s);
      if (e != cudaSuccess) return SVCONV_ERR_CUDA;
    }
    // 2) H2 = GELU(SparseConv(H1) + bc), neighbour rows rebased to the chunk
    TcConvArgs c{};
    c.A = H1;
    c.lda = R;
    c.a_rows = max_chunk_rows;
    c.nbr = nbr;
    c.taps = 9;
    c.Kc = R;
    c.M = max_chunk_rows;
    c.row_lo = frame_off + t0;
    c.row_hi = frame_off + t1;
    c.nbr_abs = 1;
    c.N = R;
    c.bias = bc;
    c.gelu = 1;
    c.out = H2;
    c.ldo = R;
    c.out_rows = max_chunk_rows;
    c.status = status;
    e = launch_tc_conv(c, Wc, R, 9 * R, conv_bn(R), s);
    if (e != cudaSuccess) return SVCONV_ERR_CUDA;
    // 3) X[rows] += H2 Wu^T, in place
    TcConvArgs u{};
    u.A = H2;
    u.lda = R;
    u.a_rows = max_chunk_rows;
    u.nbr = nullptr;
    u.taps = 1;
    u.Kc = R;
    u.M = max_chunk_rows;
    u.row_lo = frame_off + t0;
    u.row_hi = frame_off + t1;
    u.out_abs = 1;
    u.N = D;
    u.residual = X;
    u.out = X;
    u.ldo = D;
    u.out_rows = n;
    u.status = status;
    e = launch_tc_conv(u, Wu, D, R, conv_bn(D), s);
    if (e != cudaSuccess) return SVCONV_ERR_CUDA;
  }
  if (xa)
    return cuda_rc(launch_xattn_combine(xa->part, 1, xa->A, R, xa->n_chunks * xa->blocks, xa->aux, xa->aux_out, s));
  return SVCONV_OK;
}

int adapter_validate(void* X, const int32_t* nbr, const int32_t* frame_off, int T, int n, int D, int R,
                     const void* Wd, const void* Wc, const void* Wu, int chunk_T, int max_chunk_rows,
                     void* workspace, size_t ws_bytes, size_t need) {
  if (T < 0 || n < 0 || chunk_T <= 0 || max_chunk_rows <= 0) return SVCONV_ERR_SIZE;
  if (!bf16_channels_ok(D) || !bf16_channels_ok(R)) return SVCONV_ERR_UNSUPPORTED;
  if (n == 0 || T == 0) return SVCONV_OK;
  if (!X || !nbr || !frame_off || !Wd || !Wc || !Wu) return SVCONV_ERR_NULL;
  if (!aligned16(X) || !aligned16(Wd) || !aligned16(Wc) || !aligned16(Wu) || !aligned16(workspace))
    return SVCONV_ERR_ALIGN;
  if (!workspace || ws_bytes < need) return SVCONV_ERR_WORKSPACE;
  return check_device();
}

}  // namespace
}  // namespace svc

extern "C" {

int svconv_adapter_fwd(void* X, const int32_t* nbr, const int32_t* frame_off, int T, int n, int D, int R,
                       const void* Wd, const void* Wc, const float* bc, const void* Wu, int chunk_T,
                       int max_chunk_rows, void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
  const int rc = adapter_validate(X, nbr, frame_off, T, n, D, R, Wd, Wc, Wu, chunk_T, max_chunk_rows, workspace,
                                  ws_bytes, svconv_adapter_workspace_size(R, max_chunk_rows));
  if (rc || n == 0 || T == 0) return rc;
  return adapter_chunks(X, nbr, frame_off, T, n, D, R, Wd, Wc, bc, Wu, chunk_T, max_chunk_rows, workspace, dev_status,
                        nullptr, (cudaStream_t)stream);
}

size_t svconv_xattn_workspace_size(int G, int max_group_rows, int A) {
  if (G <= 0 || max_group_rows < 0 || A <= 0) return 0;
  return xattn_partial_bytes((size_t)G * xattn_slots(max_group_rows, G), A);
}

int svconv_xattn_aux(const void* H, int n, int R, const int32_t* group_off, int G, int max_group_rows,
                     const void* aux, int A, int heads, float* aux_out, void* workspace, size_t ws_bytes,
                     int32_t* dev_status, void* stream) {
  if (n < 0 || G < 0 || max_group_rows < 0) return SVCONV_ERR_SIZE;
  if (!xattn_shape_ok(R, A, heads)) return SVCONV_ERR_UNSUPPORTED;
  if (G == 0) return SVCONV_OK;
  if (!group_off || !aux || !aux_out || (n > 0 && !H)) return SVCONV_ERR_NULL;
  if (!aligned16(H) || !aligned16(aux) || !aligned16(aux_out) || !aligned16(workspace)) return SVCONV_ERR_ALIGN;
  if (!workspace || ws_bytes < svconv_xattn_workspace_size(G, max_group_rows, A)) return SVCONV_ERR_WORKSPACE;
  int rc = check_device();
  if (rc) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  XattnLaunch x{};
  x.H = H;
  x.h_rows = n;
  x.R = R;
  x.heads = heads;
  x.lo = group_off;
  x.hi = group_off + 1;
  x.h_sub = nullptr;
  x.G = G;
  x.max_rows = max_group_rows;
  x.aux = aux;
  x.A = A;
  x.part = static_cast<float*>(workspace);
  x.slot0 = 0;
  x.slots_per_group = xattn_slots(max_group_rows, G);
  x.status = dev_status ? dev_status : device_error_word();
  cudaError_t e = launch_xattn_partials(x, s);
  if (e != cudaSuccess) return SVCONV_ERR_CUDA;
  return cuda_rc(launch_xattn_combine(x.part, G, A, R, x.slots_per_group, aux, aux_out, s));
}

size_t svconv_adapter_xattn_workspace_size(int T, int R, int chunk_T, int max_chunk_rows, int A) {
  if (T <= 0 || R <= 0 || chunk_T <= 0 || max_chunk_rows <= 0 || A <= 0) return 0;
  const size_t base = (svconv_adapter_workspace_size(R, max_chunk_rows) + 255) / 256 * 256;
  const int n_chunks = (T + chunk_T - 1) / chunk_T;
  return base + xattn_partial_bytes((size_t)n_chunks * xattn_slots(max_chunk_rows, 1), A);
}

int svconv_adapter_fwd_xattn(void* X, const int32_t* nbr, const int32_t* frame_off, int T, int n, int D, int R,
                             const void* Wd, const void* Wc, const float* bc, const void* Wu, int chunk_T,
                             int max_chunk_rows, const void* aux, int A, int heads, float* aux_out, void* workspace,
                             size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (!xattn_shape_ok(R, A, heads)) return SVCONV_ERR_UNSUPPORTED;
  const int rc = adapter_validate(X, nbr, frame_off, T, n, D, R, Wd, Wc, Wu, chunk_T, max_chunk_rows, workspace,
                                  ws_bytes, svconv_adapter_xattn_workspace_size(T, R, chunk_T, max_chunk_rows, A));
  if (rc) return rc;
  if (!aux || !aux_out) return SVCONV_ERR_NULL;
  if (!aligned16(aux) || !aligned16(aux_out)) return SVCONV_ERR_ALIGN;
  cudaStream_t s = (cudaStream_t)stream;
  if (n == 0 || T == 0) {  // no rows: nothing to attend over, the auxiliary tokens are copied unchanged
    const int rc2 = check_device();
    if (rc2) return rc2;
    return cuda_rc(launch_xattn_combine(nullptr, 1, A, R, 0, aux, aux_out, s));
  }
  AdapterXattn xa{};
  xa.aux = aux;
  xa.A = A;
  xa.heads = heads;
  xa.aux_out = aux_out;
  xa.blocks = xattn_slots(max_chunk_rows, 1);
  xa.n_chunks = T > 0 ? (T + chunk_T - 1) / chunk_T : 0;
  const size_t base = (svconv_adapter_workspace_size(R, max_chunk_rows) + 255) / 256 * 256;
  xa.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + base);
  return adapter_chunks(X, nbr, frame_off, T, n, D, R, Wd, Wc, bc, Wu, chunk_T, max_chunk_rows, workspace, dev_status,
                        &xa, s);
}

int svconv_read_error_word(int32_t* out) {
  if (!out) return SVCONV_ERR_NULL;
  int rc = check_device();
  if (rc) return rc;
  if (cudaDeviceSynchronize() != cudaSuccess) return SVCONV_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(int)) != cudaSuccess) return SVCONV_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)) != cudaSuccess) return SVCONV_ERR_CUDA;
  *out = v;
  return SVCONV_OK;
}

int svconv_selftest_timeout(int32_t* dev_status, int timeout_us, void* stream) {
  if (!dev_status) return SVCONV_ERR_NULL;
  if (timeout_us <= 0 || timeout_us > 10000000) return SVCONV_ERR_SIZE;
  int rc = check_device();
  if (rc) return rc;
  return cuda_rc(launch_timeout_selftest(dev_status, (uint64_t)timeout_us * 1000ull, (cudaStream_t)stream));
}

}  // extern "C"

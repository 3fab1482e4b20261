// Internal declarations shared by the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "svconv.h"

namespace svc {

// The library's per-device error word (defined in svconv_api.cu).
int* device_error_word();
int sm_count();

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s for any single bounded wait

// Raise a kernel's dynamic shared-memory limit once per device (the attribute
// call is skipped afterwards, which keeps launches cheap and capturable).
template <typename Kernel>
inline cudaError_t ensure_smem_attr(Kernel kernel, size_t bytes, int* done_bytes /* [64] per device */) {
  int d = 0;
  cudaError_t e = cudaGetDevice(&d);
  if (e != cudaSuccess) return e;
  if (d >= 0 && d < 64 && done_bytes[d] >= (int)bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && d >= 0 && d < 64) done_bytes[d] = (int)bytes;
  return e;
}

// Kernel launch with programmatic stream serialization (the kernel may start while the
// previous kernel on the stream drains; every kernel waits for it with griddepcontrol.wait
// before touching global memory).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// As launch_pdl, with the grid in clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                      unsigned cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------- index build
cudaError_t launch_build_index(const int32_t* coords, const int32_t* frame_off, int T, int H, int W, int n,
                               int32_t* nbr, int32_t* M, int32_t* status, cudaStream_t s);

// ---------------------------------------------------------------- fp32 CUDA-core path
cudaError_t launch_f32_conv(bool mirror_bwd, const float* src, const int32_t* nbr, int n, int Csrc, int Cdst,
                            const float* Wt, int Cin, int Cout, const float* bias, float* dst, cudaStream_t s);
size_t f32_wgrad_splits(int n);
cudaError_t launch_f32_wgrad_partials(const float* dY, const float* X, const int32_t* nbr, int n, int Cin, int Cout,
                                      float* partial, int splits, int rows_pad, cudaStream_t s);
// partial [splits][rows_pad][Cout]; grouped = 0: row m = j*Cin + i (m = 9*Cin holds db);
// grouped = 1 (tensor-core layout): row ((i/64)*10 + j)*64 + i%64, db in row 576
cudaError_t launch_wgrad_reduce(const float* partial, int splits, int rows_pad, int Cin, int Cout, int grouped,
                                float* dW, float* db, cudaStream_t s);

// ---------------------------------------------------------------- tcgen05 bf16 path
struct TcConvArgs {
  // A operand: rows gathered (taps = 9) or read densely (taps = 1)
  const void* A;          // bf16 [rows][lda]
  int lda;
  int a_rows;             // number of valid rows in A (range check for gathered indices)
  const int32_t* nbr;     // [*][9] or nullptr for dense
  int taps;               // 9 or 1
  int mirror;             // gather uses column 8-j
  int Kc;                 // channels per tap (multiple of 64)
  // B operand (weights), described by a TMA tensor map built on the host
  int b_mn_major;         // 0: W[o][j*Kc + c] K-major 2D map; 1: W[c][j][n] MN-major 3D map
  // rows
  int M;                  // rows to compute (upper bound when row pointers are given)
  const int32_t* row_lo;  // device pointers (chunked adapter) or nullptr
  const int32_t* row_hi;
  int a_abs;              // dense A row = lo + r (else r)
  int nbr_abs;            // neighbour table row = lo + r and values are rebased by -lo
  int out_abs;            // output row = lo + r (else r)
  int N;                  // output columns
  // epilogue
  const float* bias;      // [N] or nullptr
  int gelu;
  const void* residual;   // bf16 [rows][ldo] or nullptr (added before the store; may alias out)
  void* out;              // bf16 [rows][ldo]
  int ldo;
  int out_rows;           // rows of out / residual (range check of absolute output rows)
  int32_t* status;        // caller status word or nullptr (library word used otherwise)
  int max_ctas;           // CTA budget (0: one per SM)
  int f8;                 // A and B hold e4m3 values; lda, Kc and the weight columns count PAIRS
                          // of them (2-byte units), so byte offsets match the bf16 path
};
cudaError_t launch_tc_conv(const TcConvArgs& a, const void* Wt, int w_rows, int w_cols, int bn, cudaStream_t s);

struct TcWgradArgs {
  const void* dY;     // bf16 [n][Cout]
  const void* X;      // bf16 [n][Cin]
  const int32_t* nbr; // [n][9]
  int n, Cin, Cout;
  float* partial;     // [splits][rows_pad][Cout], grouped row layout (see launch_wgrad_reduce)
  int splits, rows_pad;
};
void tc_wgrad_plan(int n, int Cin, int Cout, int* splits, int* rows_pad, int* bn);
// the same plan for a budget of `ctas` CTAs (launch with launch_tc_wgrad_with_splits)
void tc_wgrad_plan_ctas(int n, int Cin, int Cout, int ctas, int* splits, int* rows_pad, int* bn);
cudaError_t launch_tc_wgrad(const TcWgradArgs& a, cudaStream_t s);
cudaError_t launch_tc_wgrad_with_splits(const TcWgradArgs& a, cudaStream_t s);

// Single-pass backward at C_in = C_out = 64 (bf16): data gradient, weight-gradient partials
// [tc_bwd_small_grid(n)][640][64] and their fixed-order reduce into dW / db.
int tc_bwd_small_grid(int n);
size_t tc_bwd_small_partial_floats(int n);
cudaError_t launch_tc_bwd_small(const void* dY, const void* X, const int32_t* nbr, int n, const void* Wt, void* dX,
                                float* partial, float* dW, float* db, cudaStream_t s);

// bf16 tensor-core bodies of the data / weight gradients (arguments already validated);
// max_ctas / ctas: CTA budget (0: all SMs).  Return SVCONV_* codes.
int tc_bwd_data(const void* dY, const int32_t* nbr, int n, int Cin, int Cout, const void* Wt, void* dX, int max_ctas,
                cudaStream_t s);
int tc_bwd_weight(const void* dY, const void* X, const int32_t* nbr, int n, int Cin, int Cout, float* dW, float* db,
                  float* partial, int ctas, cudaStream_t s);

// ---------------------------------------------------------------- auxiliary-token cross-attention
constexpr int kXattnMaxQueries = 16;
struct XattnLaunch {
  const void* H;            // bf16 keys / values [h_rows][R]
  int h_rows, R, heads;
  const int32_t* lo;        // device: group g owns rows lo[g] .. hi[g]-1
  const int32_t* hi;
  const int32_t* h_sub;     // device or nullptr: H row = row - *h_sub
  int G, max_rows;          // groups; rows of the largest group (sets the partial blocks per group)
  const void* aux;          // bf16 [G][A][R]
  int A;
  float* part;              // partial records, slot = g * slots_per_group + slot0 + block
  int slot0, slots_per_group;
  int* status;
};
bool xattn_shape_ok(int R, int A, int heads);
size_t xattn_partial_bytes(int slots, int A);
int xattn_slots(int max_rows, int G);  // partial slots (CTAs) per group
cudaError_t launch_xattn_partials(const XattnLaunch& x, cudaStream_t s);
cudaError_t launch_xattn_combine(const float* part, int G, int A, int R, int slots_per_group, const void* aux,
                                 float* out, cudaStream_t s);

// failure-detection self test
cudaError_t launch_timeout_selftest(int32_t* status, uint64_t timeout_ns, cudaStream_t s);

}  // namespace svc

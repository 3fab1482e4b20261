// fp32 path on CUDA cores (exact fp32 arithmetic; TF32 tensor cores would not
// meet an fp32 tolerance), plus the fixed-order split reduction shared by both
// weight-gradient paths.
//
// Sums are compensated: every dot product uses the "Dot2" scheme of Ogita, Rump
// and Oishi ("Accurate sum and dot product", SIAM J. Sci. Comput. 2005): the
// rounding error of each product (recovered exactly with an FMA) and of each
// addition (Knuth's TwoSum) is carried in a second fp32 word.  The result is as
// accurate as if accumulated in about twice the working precision, so outputs
// with heavy cancellation still meet an fp32 tolerance relative to the result.
//
//  * f32_conv_kernel: one thread per (token, output channel).  The 9 x C_src x
//    C_dst weight block sits in shared memory, laid out so that a warp's
//    consecutive output channels read consecutive words (no bank conflicts); the
//    neighbour row of the source features is read once per warp (broadcast).
//    The same kernel computes the forward (gather through N[k][j]) and the data
//    gradient (gather through the mirrored column N[k][8-j] with W_j transposed).
//  * f32_wgrad_partial_kernel: each split of tokens writes its partial dW rows
//    (row m = j*C_in + i, row 9*C_in = db) to the workspace.
//  * wgrad_reduce_kernel: sums the splits in index order (deterministic, and
//    compensated) and transposes to dW[o][j][i] through a 32x32 shared tile.
#include "svconv_internal.h"
#include "svconv_ptx.cuh"

namespace svc {
namespace {

// The _rn intrinsics are never contracted into FMAs, which the error-free
// transformations below rely on.
struct Dot2 {
  float s = 0.0f, c = 0.0f;
  __device__ __forceinline__ void add(float v) {  // TwoSum(s, v), error into c
    const float t = __fadd_rn(s, v);
    const float z = __fsub_rn(t, s);
    c = __fadd_rn(c, __fadd_rn(__fsub_rn(s, __fsub_rn(t, z)), __fsub_rn(v, z)));
    s = t;
  }
  __device__ __forceinline__ void fma(float a, float b) {  // TwoProduct(a, b), then add
    const float p = __fmul_rn(a, b);
    c = __fadd_rn(c, __fmaf_rn(a, b, -p));
    add(p);
  }
  __device__ __forceinline__ float value() const { return __fadd_rn(s, c); }
};

__global__ void __launch_bounds__(256) f32_conv_kernel(const float* __restrict__ src, const int32_t* __restrict__ nbr,
                                                       int n, int Csrc, int Cdst, const float* __restrict__ Wt,
                                                       int Cin, int Cout, int mirror, const float* __restrict__ bias,
                                                       float* __restrict__ dst, int* err) {
  extern __shared__ float sW[];  // [9][Csrc][Cdst]
  const int total_w = 9 * Cin * Cout;
  for (int e = threadIdx.x; e < total_w; e += blockDim.x) {
    const int o = e / (9 * Cin);
    const int j = (e / Cin) % 9;
    const int i = e % Cin;
    const float w = Wt[e];
    if (!mirror)
      sW[((size_t)j * Cin + i) * Cout + o] = w;  // forward: src = X (Cin), dst = Y (Cout)
    else
      sW[((size_t)j * Cout + o) * Cin + i] = w;  // data grad: src = dY (Cout), dst = dX (Cin)
  }
  __syncthreads();
  const long long total = (long long)n * Cdst;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int k = (int)(e / Cdst);
    const int c = (int)(e - (long long)k * Cdst);
    Dot2 acc;
    if (bias) acc.add(bias[c]);
    // the nine neighbour indices first (independent loads), so that the row loads of the
    // taps do not each wait for their own index load
    int mm[9];
#pragma unroll
    for (int j = 0; j < 9; ++j) mm[j] = __ldg(nbr + (size_t)k * 9 + (mirror ? 8 - j : j));
#pragma unroll
    for (int j = 0; j < 9; ++j) {
      const int m = mm[j];
      if (m < 0) continue;
      if (m >= n) {
        atomicOr(err, SVCONV_STATUS_BAD_INDEX);
        continue;
      }
      const float* s = src + (size_t)m * Csrc;
      const float* w = sW + (size_t)j * Csrc * Cdst + c;
      for (int q = 0; q < Csrc; ++q) acc.fma(w[(size_t)q * Cdst], s[q]);
    }
    dst[e] = acc.value();
  }
}

__global__ void __launch_bounds__(256) f32_wgrad_partial_kernel(const float* __restrict__ dY,
                                                                const float* __restrict__ X,
                                                                const int32_t* __restrict__ nbr, int n, int Cin,
                                                                int Cout, float* __restrict__ partial, int splits,
                                                                int rows_pad, int* err) {
  const int sp = blockIdx.y;
  const int k0 = (int)((long long)n * sp / splits), k1 = (int)((long long)n * (sp + 1) / splits);
  const int rows = 9 * Cin + 1;
  const long long total = (long long)rows * Cout;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int m = (int)(e / Cout);
    const int o = (int)(e - (long long)m * Cout);
    Dot2 acc;
    if (m < 9 * Cin) {
      const int j = m / Cin, i = m - j * Cin;
      for (int k = k0; k < k1; ++k) {
        const int nb = nbr[(size_t)k * 9 + j];
        if (nb < 0) continue;
        if (nb >= n) {
          atomicOr(err, SVCONV_STATUS_BAD_INDEX);
          continue;
        }
        acc.fma(dY[(size_t)k * Cout + o], X[(size_t)nb * Cin + i]);
      }
    } else {
      for (int k = k0; k < k1; ++k) acc.add(dY[(size_t)k * Cout + o]);
    }
    partial[((size_t)sp * rows_pad + m) * Cout + o] = acc.value();
  }
}

// One thread per (dW row m = j * Cin + i, output channel o); blocks of 8 rows x 32 output
// channels (about one block per SM at the small-channel size), so that the partial reads
// (along o) are coalesced and many are in flight; the transposed dW writes go through a
// shared-memory tile.  The split sums are issued 16 loads at a time, summed in split order.
// grouped = 0: partial row m (db at 9 Cin); grouped = 1 (tensor-core layout, Cin a
// multiple of 64): partial row ((i / 64) * 10 + j) * 64 + i % 64, db at 9 * 64.
constexpr int kRedRows = 8;
__global__ void __launch_bounds__(256) wgrad_reduce_kernel(const float* __restrict__ partial, int splits,
                                                           int rows_pad, int Cin, int Cout, int grouped,
                                                           float* __restrict__ dW, float* __restrict__ db) {
  __shared__ float tile[kRedRows][33];
  pdl_wait();  // the partials come from the kernel before this one
  pdl_trigger();
  const int rows = 9 * Cin + 1;
  const int m0 = blockIdx.x * kRedRows, o0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  {
    const int m = m0 + ty, o = o0 + tx;
    Dot2 s;
    if (m < rows && o < Cout) {
      int pm = m;
      if (grouped) {
        const int j = m / Cin, i = m - j * Cin;
        pm = m == 9 * Cin ? 9 * 64 : ((i >> 6) * 10 + j) * 64 + (i & 63);
      }
      const size_t stride = (size_t)rows_pad * Cout;
      const float* src = partial + (size_t)pm * Cout + o;
      for (int sp0 = 0; sp0 < splits; sp0 += 16) {
        float v[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) v[q] = (sp0 + q < splits) ? __ldg(src + (size_t)(sp0 + q) * stride) : 0.0f;
#pragma unroll
        for (int q = 0; q < 16; ++q)
          if (sp0 + q < splits) s.add(v[q]);
      }
    }
    tile[ty][tx] = s.value();
  }
  __syncthreads();
  // write: each warp takes 4 output channels, its lanes 8 consecutive rows of each
  {
    const int o = o0 + ty * 4 + (tx >> 3), r = tx & 7, m = m0 + r;
    if (o < Cout) {
      const float v = tile[r][ty * 4 + (tx >> 3)];
      if (m < 9 * Cin)
        dW[(size_t)o * 9 * Cin + m] = v;
      else if (m == 9 * Cin && db)
        db[o] = v;
    }
  }
}

}  // namespace

cudaError_t launch_f32_conv(bool mirror_bwd, const float* src, const int32_t* nbr, int n, int Csrc, int Cdst,
                            const float* Wt, int Cin, int Cout, const float* bias, float* dst, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const size_t smem = sizeof(float) * 9 * (size_t)Cin * Cout;
  static int done[64];
  cudaError_t e = ensure_smem_attr(f32_conv_kernel, smem, done);
  if (e != cudaSuccess) return e;
  long long blocks = ((long long)n * Cdst + 255) / 256;
  const long long cap = (long long)sm_count() * 8;
  if (blocks > cap) blocks = cap;
  f32_conv_kernel<<<(int)blocks, 256, smem, s>>>(src, nbr, n, Csrc, Cdst, Wt, Cin, Cout, mirror_bwd ? 1 : 0, bias,
                                                 dst, device_error_word());
  return cudaGetLastError();
}

// About 16 tokens per split: each thread's token loop is a chain of dependent loads
// (neighbour index, then the feature row), so short loops keep the kernel off the
// load-latency path at small n; at most 128 splits.
size_t f32_wgrad_splits(int n) {
  int sp = (n + 15) / 16;
  if (sp > 128) sp = 128;
  if (sp < 1) sp = 1;
  return (size_t)sp;
}

cudaError_t launch_f32_wgrad_partials(const float* dY, const float* X, const int32_t* nbr, int n, int Cin, int Cout,
                                      float* partial, int splits, int rows_pad, cudaStream_t s) {
  const long long total = (long long)(9 * Cin + 1) * Cout;
  long long bx = (total + 255) / 256;
  if (bx > 64) bx = 64;
  dim3 grid((unsigned)bx, (unsigned)splits);
  f32_wgrad_partial_kernel<<<grid, 256, 0, s>>>(dY, X, nbr, n, Cin, Cout, partial, splits, rows_pad,
                                                device_error_word());
  return cudaGetLastError();
}

// The same reduction with four adjacent output channels per thread (16-byte loads of the
// partials, up to 8 splits in flight per load batch).  The sum is bound by how many bytes
// are in flight, and at one channel per thread the kernel's register use caps it at a few
// MB across the GPU; four channels per thread carry four times as many.  Each element gets
// the same compensated sum over the splits in the same order as in wgrad_reduce_kernel, so
// the results are bitwise identical.  Needs Cout % 4 == 0 (16-byte aligned rows).
template <int CW>  // output channels per block
__global__ void __launch_bounds__(256) wgrad_reduce4_kernel(const float* __restrict__ partial, int splits,
                                                            int rows_pad, int Cin, int Cout, int grouped,
                                                            float* __restrict__ dW, float* __restrict__ db) {
  constexpr int kLanesPerRow = CW / 4;
  constexpr int kRows = 256 / kLanesPerRow;  // partial rows per block
  __shared__ float tile[kRows][CW + 1];
  pdl_wait();  // the partials come from the kernel before this one
  pdl_trigger();
  const int rows = 9 * Cin + 1;
  const int m0 = blockIdx.x * kRows, o0 = blockIdx.y * CW;
  const int r = threadIdx.x / kLanesPerRow, cl = threadIdx.x % kLanesPerRow;
  const int m = m0 + r, o = o0 + 4 * cl;
  Dot2 acc[4];
  if (m < rows && o < Cout) {
    int pm = m;
    if (grouped) {
      const int j = m / Cin, i = m - j * Cin;
      pm = m == 9 * Cin ? 9 * 64 : ((i >> 6) * 10 + j) * 64 + (i & 63);
    }
    const size_t stride4 = (size_t)rows_pad * Cout / 4;
    const float4* src = reinterpret_cast<const float4*>(partial + (size_t)pm * Cout + o);
    for (int sp0 = 0; sp0 < splits; sp0 += 8) {
      float4 v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        v[q] = (sp0 + q < splits) ? __ldg(src + (size_t)(sp0 + q) * stride4) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (sp0 + q < splits) {
          acc[0].add(v[q].x);
          acc[1].add(v[q].y);
          acc[2].add(v[q].z);
          acc[3].add(v[q].w);
        }
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) tile[r][4 * cl + k] = acc[k].value();
  __syncthreads();
  // write: consecutive threads take consecutive rows of one output channel
  for (int e = threadIdx.x; e < CW * kRows; e += 256) {
    const int oc = e / kRows, rr = e - oc * kRows;
    const int oo = o0 + oc, mm = m0 + rr;
    if (oo < Cout) {
      const float v = tile[rr][oc];
      if (mm < 9 * Cin)
        dW[(size_t)oo * 9 * Cin + mm] = v;
      else if (mm == 9 * Cin && db)
        db[oo] = v;
    }
  }
}

cudaError_t launch_wgrad_reduce(const float* partial, int splits, int rows_pad, int Cin, int Cout, int grouped,
                                float* dW, float* db, cudaStream_t s) {
  const int rows = 9 * Cin + 1;
  if (Cout >= 128 && Cout % 4 == 0 && (reinterpret_cast<uintptr_t>(partial) & 15u) == 0) {
    constexpr int kCW = 128, kRows = 256 / (kCW / 4);
    dim3 grid((rows + kRows - 1) / kRows, (Cout + kCW - 1) / kCW);
    return launch_pdl(wgrad_reduce4_kernel<kCW>, grid, dim3(256), 0, s, partial, splits, rows_pad, Cin, Cout, grouped,
                      dW, db);
  }
  dim3 grid((rows + kRedRows - 1) / kRedRows, (Cout + 31) / 32);
  return launch_pdl(wgrad_reduce_kernel, grid, dim3(256), 0, s, partial, splits, rows_pad, Cin, Cout, grouped, dW, db);
}

}  // namespace svc

// Asymmetric cross-attention of auxiliary tokens over the sparse tokens (SV-TAD page, Key
// Design 3, "Asymmetric Cross-Attention for Temporal Recombination"): a few auxiliary tokens
// (a CLS token per video, or landmark tokens) are the queries, the down-projected sparse
// visual features of their video are the keys and the values, and only the auxiliary tokens
// are updated:
//     aux'[a] = aux[a] + softmax_r(aux[a] . H[r] / sqrt(d)) H[r]      (per head of d channels)
//
// With a handful of queries per video this is not a dense contraction: every key row is read
// once and used for A dot products and A weighted sums, 2 A flops per byte, far below the
// tensor-core (and even the CUDA-core) ridge.  So it runs on CUDA cores and is sized for HBM:
//   xattn_partial_kernel  one CTA per block of 256 consecutive rows of a group; each warp
//                         streams rows (one 16-byte piece of a row per lane, four rows in
//                         flight per warp), keeps an online softmax (running max m, sum l,
//                         weighted row sum o) per query in registers, and the CTA merges its
//                         8 warps and writes one partial (m, l, o) per query;
//   xattn_combine_kernel  one CTA per (group, query) merges the group's partials in a fixed
//                         order (deterministic) and adds the result to the auxiliary token.
// Scores are formed in base 2 (the query is prescaled by log2(e) / sqrt(d)), so every
// exponential is one exp2f.
#include <cuda_bf16.h>

#include <cmath>
#include <cstdint>

#include "svconv_internal.h"
#include "svconv_ptx.cuh"

namespace svc {
namespace {

constexpr int kXaRows = 256;    // rows per partial block (one CTA)
constexpr int kXaWarps = 8;     // 256 threads
constexpr int kXaUnroll = 4;    // rows in flight per warp
constexpr int kXaQB = 4;        // queries per pass held in registers
constexpr int kXaRec = 10;      // per lane and query: m, l, o[8]

struct XattnParams {
  const __nv_bfloat16* H;  // keys / values [h_rows][R]
  int h_rows, R;
  int lanes_per_head;      // d / 8 (a power of two)
  const int32_t* lo;       // group g owns rows lo[g] .. hi[g]-1 (row numbers before h_sub)
  const int32_t* hi;
  const int32_t* h_sub;    // nullptr, or H row = row - *h_sub (rows of a chunk stored from 0)
  int rows_cap;            // rows covered per group: gridDim.x * kXaRows
  const __nv_bfloat16* aux;  // [G][A][R]
  int A, q0, qb;           // this pass covers queries q0 .. q0+qb-1
  float qscale;            // log2(e) / sqrt(d)
  float* part;             // [G * slots_per_group][A][kXaRec][32]
  int slot0, slots_per_group;
  int* status;
};

// 16-byte read-only load that does not allocate in L1 (each piece is read once per CTA).
__device__ __forceinline__ uint4 ldg_nc_16(const void* ptr) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(ptr));
  return v;
}

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = __bfloat1622float2(h[i]);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}

// Sum over the lanes of one head (lanes_per_head consecutive lanes, a power of two).
__device__ __forceinline__ float head_sum(float v, int lanes_per_head) {
  for (int o = lanes_per_head >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int QB>
__global__ void __launch_bounds__(kXaWarps * 32) xattn_partial_kernel(const __grid_constant__ XattnParams p) {
  __shared__ float s_state[kXaWarps][QB][kXaRec][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = blockIdx.y, b = blockIdx.x;
  const bool active = lane * 8 < p.R;
  pdl_wait();
  pdl_trigger();

  int lo = p.lo[g], hi = p.hi[g];
  const int sub = p.h_sub ? *p.h_sub : 0;
  int flags = 0;
  if (hi < lo || lo - sub < 0 || hi - sub > p.h_rows) {
    flags |= SVCONV_STATUS_BAD_OFFSETS;
    hi = lo;
  }
  if (hi - lo > p.rows_cap) {
    flags |= SVCONV_STATUS_CHUNK_OVERFLOW;
    hi = lo + p.rows_cap;
  }
  const int r_begin = lo + b * kXaRows;
  const int r_end = min(hi, r_begin + kXaRows);

  // this lane's 8 channels of each query, prescaled so that scores are in base 2
  float q[QB][8];
#pragma unroll
  for (int a = 0; a < QB; ++a) {
    if (active && a < p.qb) {
      const uint4 u = ldg_nc_16(p.aux + ((size_t)g * p.A + p.q0 + a) * p.R + lane * 8);
      unpack8(u, q[a]);
#pragma unroll
      for (int c = 0; c < 8; ++c) q[a][c] *= p.qscale;
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) q[a][c] = 0.f;
    }
  }
  float m[QB], l[QB], o[QB][8];
#pragma unroll
  for (int a = 0; a < QB; ++a) {
    m[a] = -INFINITY;
    l[a] = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) o[a][c] = 0.f;
  }

  const __nv_bfloat16* Hb = p.H + lane * 8;
  for (int r0 = r_begin + warp * kXaUnroll; r0 < r_end; r0 += kXaWarps * kXaUnroll) {
    float h[kXaUnroll][8];
#pragma unroll
    for (int u = 0; u < kXaUnroll; ++u) {
      const int r = r0 + u;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (active && r < r_end) v = ldg_nc_16(Hb + (size_t)(r - sub) * p.R);
      unpack8(v, h[u]);
    }
#pragma unroll
    for (int a = 0; a < QB; ++a) {
      float s[kXaUnroll];
      float mx = m[a];
#pragma unroll
      for (int u = 0; u < kXaUnroll; ++u) {
        float d = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) d = fmaf(q[a][c], h[u][c], d);
        s[u] = head_sum(d, p.lanes_per_head);
        if (r0 + u >= r_end) s[u] = -INFINITY;  // past the block: weight 0
        mx = fmaxf(mx, s[u]);
      }
      if (mx == -INFINITY) continue;  // no row yet (only possible on a block's empty tail)
      const float alpha = exp2f(m[a] - mx);
      float pr[kXaUnroll];
      float lsum = l[a] * alpha;
#pragma unroll
      for (int u = 0; u < kXaUnroll; ++u) {
        pr[u] = exp2f(s[u] - mx);
        lsum += pr[u];
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float acc = o[a][c] * alpha;
#pragma unroll
        for (int u = 0; u < kXaUnroll; ++u) acc = fmaf(pr[u], h[u][c], acc);
        o[a][c] = acc;
      }
      m[a] = mx;
      l[a] = lsum;
    }
  }

#pragma unroll
  for (int a = 0; a < QB; ++a) {
    s_state[warp][a][0][lane] = m[a];
    s_state[warp][a][1][lane] = l[a];
#pragma unroll
    for (int c = 0; c < 8; ++c) s_state[warp][a][2 + c][lane] = o[a][c];
  }
  __syncthreads();
  // merge the warps in a fixed order: thread (a, lane) of the first QB warps
  if (warp < QB && warp < p.qb) {
    const int a = warp;
    float M = -INFINITY;
    for (int w = 0; w < kXaWarps; ++w) M = fmaxf(M, s_state[w][a][0][lane]);
    float L = 0.f, O[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) O[c] = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < kXaWarps; ++w) {
        const float lw = s_state[w][a][1][lane];
        if (lw == 0.f) continue;
        const float f = exp2f(s_state[w][a][0][lane] - M);
        L = fmaf(lw, f, L);
#pragma unroll
        for (int c = 0; c < 8; ++c) O[c] = fmaf(s_state[w][a][2 + c][lane], f, O[c]);
      }
    }
    const size_t slot = (size_t)g * p.slots_per_group + p.slot0 + b;
    float* dst = p.part + ((slot * p.A + p.q0 + a) * kXaRec) * 32 + lane;
    dst[0] = M;
    dst[32] = L;
#pragma unroll
    for (int c = 0; c < 8; ++c) dst[(2 + c) * 32] = O[c];
  }
  if (flags && threadIdx.x == 0 && b == 0) atomicOr(p.status, flags);
}

// Merge of a (group, query)'s partials: one CTA of 8 warps; warp w folds slots w, w + 8, ...
// (four records in flight per lane) into a running (max, sum, weighted sum), then warp 0
// merges the 8 warps in order.  The assignment and the order are fixed: deterministic.
__device__ __forceinline__ void merge_state(float& M, float& L, float (&O)[8], float m, float l, const float (&o)[8]) {
  if (l == 0.f) return;
  const float mx = fmaxf(M, m);
  const float a = exp2f(M - mx), b = exp2f(m - mx);  // M = -inf (nothing yet) gives a = 0
  L = L * a + l * b;
#pragma unroll
  for (int c = 0; c < 8; ++c) O[c] = O[c] * a + o[c] * b;
  M = mx;
}

__global__ void __launch_bounds__(256) xattn_combine_kernel(const float* __restrict__ part, int G, int A, int R,
                                                            int slots_per_group, const __nv_bfloat16* __restrict__ aux,
                                                            float* __restrict__ out) {
  __shared__ float s_state[kXaWarps][kXaRec][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = blockIdx.x / A, a = blockIdx.x - (blockIdx.x / A) * A;
  pdl_wait();
  pdl_trigger();
  float M = -INFINITY, L = 0.f, O[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) O[c] = 0.f;
  const size_t stride = (size_t)A * kXaRec * 32;  // between consecutive slots of the group
  const float* base = part + (((size_t)g * slots_per_group) * A + a) * kXaRec * 32 + lane;
  for (int s0 = warp; s0 < slots_per_group; s0 += 4 * kXaWarps) {
    float m[4], l[4], o[4][8];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int sl = s0 + u * kXaWarps;
      const bool ok = sl < slots_per_group;
      const float* r = base + (size_t)(ok ? sl : 0) * stride;
      m[u] = ok ? r[0] : -INFINITY;
      l[u] = ok ? r[32] : 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) o[u][c] = ok ? r[(2 + c) * 32] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) merge_state(M, L, O, m[u], l[u], o[u]);
  }
  s_state[warp][0][lane] = M;
  s_state[warp][1][lane] = L;
#pragma unroll
  for (int c = 0; c < 8; ++c) s_state[warp][2 + c][lane] = O[c];
  __syncthreads();
  if (warp != 0) return;
  M = -INFINITY, L = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) O[c] = 0.f;
  for (int w = 0; w < kXaWarps; ++w) {
    float o[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) o[c] = s_state[w][2 + c][lane];
    merge_state(M, L, O, s_state[w][0][lane], s_state[w][1][lane], o);
  }
  if (lane * 8 >= R) return;
  float qv[8];
  unpack8(ldg_nc_16(aux + ((size_t)g * A + a) * R + lane * 8), qv);
  float* dst = out + ((size_t)g * A + a) * R + lane * 8;
  const float inv = L > 0.f ? 1.f / L : 0.f;  // a group without rows: aux unchanged
#pragma unroll
  for (int c = 0; c < 8; ++c) dst[c] = qv[c] + O[c] * inv;
}

}  // namespace

bool xattn_shape_ok(int R, int A, int heads) {
  if (R < 8 || R > 256 || R % 8 != 0 || A < 1 || A > kXattnMaxQueries || heads < 1 || R % heads != 0) return false;
  const int lanes = R / heads / 8;
  return lanes >= 1 && (R / heads) % 8 == 0 && (lanes & (lanes - 1)) == 0;
}

size_t xattn_partial_bytes(int slots, int A) { return (size_t)slots * A * kXaRec * 32 * sizeof(float); }

int xattn_blocks(int max_rows) { return max_rows <= 0 ? 1 : (max_rows + kXaRows - 1) / kXaRows; }

cudaError_t launch_xattn_partials(const XattnLaunch& x, cudaStream_t s) {
  XattnParams p{};
  p.H = static_cast<const __nv_bfloat16*>(x.H);
  p.h_rows = x.h_rows;
  p.R = x.R;
  p.lanes_per_head = x.R / x.heads / 8;
  p.lo = x.lo;
  p.hi = x.hi;
  p.h_sub = x.h_sub;
  const int blocks = xattn_blocks(x.max_rows);
  p.rows_cap = blocks * kXaRows;
  p.aux = static_cast<const __nv_bfloat16*>(x.aux);
  p.A = x.A;
  p.qscale = (float)(1.4426950408889634 / std::sqrt((double)(x.R / x.heads)));
  p.part = x.part;
  p.slot0 = x.slot0;
  p.slots_per_group = x.slots_per_group;
  p.status = x.status;
  for (int q0 = 0; q0 < x.A; q0 += kXaQB) {
    p.q0 = q0;
    p.qb = x.A - q0 < kXaQB ? x.A - q0 : kXaQB;
    cudaError_t e;
    const dim3 grid(blocks, x.G);
    if (p.qb == 1)
      e = launch_pdl(xattn_partial_kernel<1>, grid, dim3(kXaWarps * 32), 0, s, p);
    else
      e = launch_pdl(xattn_partial_kernel<kXaQB>, grid, dim3(kXaWarps * 32), 0, s, p);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_xattn_combine(const float* part, int G, int A, int R, int slots_per_group, const void* aux,
                                 float* out, cudaStream_t s) {
  if (G * A == 0) return cudaSuccess;
  return launch_pdl(xattn_combine_kernel, dim3(G * A), dim3(kXaWarps * 32), 0, s, part, G, A, R, slots_per_group,
                    static_cast<const __nv_bfloat16*>(aux), out);
}

}  // namespace svc

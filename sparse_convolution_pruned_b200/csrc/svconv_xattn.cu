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
//   xattn_partial_kernel  one wave of CTAs (3 per SM, >= 128 rows each), each folding every
//                         gridDim.x-th chunk of ~16 KB of consecutive rows of a group; chunks
//                         arrive in shared memory by bulk asynchronous copies, three deep;
//                         each warp keeps an online softmax (running max m, sum l, weighted
//                         row sum o) per query in registers, and the CTA merges its 8 warps
//                         and writes one partial (m, l, o) per query;
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

constexpr int kXaRowsPerCta = 128;  // fewest rows per partial CTA (at most kXaCtaCap CTAs)
constexpr int kXaWarps = 8;     // 256 threads
constexpr int kXaStages = 3;    // staged chunks per CTA
constexpr int kXaStageBytes = 16384;  // about one chunk of rows
constexpr int kXaQB = 4;        // queries per pass held in registers
constexpr int kXaRec = 10;      // per lane and query: m, l, o[8]
constexpr int kXaCtaCap = 444;  // partial CTAs (slots) over all groups: one wave of 3 per SM on 148 SMs
constexpr int kXaCombineWarps = 32;

struct XattnParams {
  const __nv_bfloat16* H;  // keys / values [h_rows][R]
  int h_rows, R;
  int lanes_per_head;      // d / 8 (a power of two)
  const int32_t* lo;       // group g owns rows lo[g] .. hi[g]-1 (row numbers before h_sub)
  const int32_t* hi;
  const int32_t* h_sub;    // nullptr, or H row = row - *h_sub (rows of a chunk stored from 0)
  int rows_cap;            // rows used per group at most (larger groups are flagged and clipped)
  int chunk_rows;          // rows per staged chunk (a multiple of 32)
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

// Fold one (max, sum, weighted sum) state into another (base-2 exponents).
__device__ __forceinline__ void merge_state(float& M, float& L, float (&O)[8], float m, float l, const float (&o)[8]) {
  if (l == 0.f) return;
  const float mx = fmaxf(M, m);
  const float a = exp2f(M - mx), b = exp2f(m - mx);  // M = -inf (nothing yet) gives a = 0
  L = L * a + l * b;
#pragma unroll
  for (int c = 0; c < 8; ++c) O[c] = O[c] * a + o[c] * b;
  M = mx;
}

// Online-softmax update of one query's state with a batch of U rows (h: this lane's 8
// channels of each row, s: the rows' base-2 scores, -inf for rows past the end).
template <int U>
__device__ __forceinline__ void online_update(float& m, float& l, float (&o)[8], const float (&s)[U],
                                              const float (&h)[U][8]) {
  float mx = m;
#pragma unroll
  for (int u = 0; u < U; ++u) mx = fmaxf(mx, s[u]);
  if (mx == -INFINITY) return;  // no valid row in the batch yet
  const float alpha = exp2f(m - mx);
  float lsum = l * alpha;
  float pr[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    pr[u] = exp2f(s[u] - mx);
    lsum += pr[u];
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float acc = o[c] * alpha;
#pragma unroll
    for (int u = 0; u < U; ++u) acc = fmaf(pr[u], h[u][c], acc);
    o[c] = acc;
  }
  m = mx;
  l = lsum;
}

// Lane 0 waits (bounded), the verdict is broadcast: control flow stays warp-uniform.
__device__ __forceinline__ bool xa_warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag, err, kDefaultTimeoutNs);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// CTA x of group g folds the chunks x, x + gridDim.x, ... of the group's rows into one state
// per query and writes it as slot x.  Chunks (chunk_rows consecutive rows, about 16 KB) are
// brought into shared memory by bulk asynchronous copies, kXaStages deep, so each CTA has
// tens of KB in flight at a small register cost; warps then read their rows from shared
// memory (one 16-byte piece per lane, 4 rows per batch: warp w takes rows 32 b + 4 w + u).
template <int QB>
__global__ void __launch_bounds__(kXaWarps * 32) xattn_partial_kernel(const __grid_constant__ XattnParams p) {
  extern __shared__ __align__(16) uint8_t xa_smem[];
  __shared__ __align__(8) uint64_t full[kXaStages];
  __shared__ int abort_flag;
  constexpr int U = 4;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = blockIdx.y;
  const bool active = lane * 8 < p.R;
  const uint32_t row_bytes = (uint32_t)p.R * 2u;
  const uint32_t stage_bytes = (uint32_t)p.chunk_rows * row_bytes;
  int* err = p.status;
  if (threadIdx.x == 0) {
    for (int st = 0; st < kXaStages; ++st) mbar_init(&full[st], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
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
  const int n_chunks = (hi - lo + p.chunk_rows - 1) / p.chunk_rows;
  const int mine = n_chunks > (int)blockIdx.x ? (n_chunks - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
  const uint8_t* Hbytes = reinterpret_cast<const uint8_t*>(p.H);
  auto issue = [&](int i) {  // chunk i of this CTA into stage i % kXaStages (thread 0)
    const int c = (int)blockIdx.x + i * (int)gridDim.x;
    const int r0 = lo + c * p.chunk_rows;
    const int cnt = min(p.chunk_rows, hi - r0);
    const uint32_t bytes = (uint32_t)cnt * row_bytes;
    uint64_t* bar = &full[i % kXaStages];
    mbar_arrive_expect_tx(bar, bytes);
    bulk_copy_g2s(smem_u32(xa_smem) + (uint32_t)(i % kXaStages) * stage_bytes,
                  Hbytes + (size_t)(r0 - sub) * row_bytes, bytes, bar);
  };
  int issued = 0;
  if (threadIdx.x == 0)
    for (; issued < kXaStages && issued < mine; ++issued) issue(issued);

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

  bool aborted = false;
  for (int i = 0; i < mine; ++i) {
    const int st = i % kXaStages;
    // every thread takes the same branch: a warp that passes its wait after another warp gave up
    // must not run ahead into a barrier the others never reach
    const bool ok = xa_warp_wait(&full[st], (uint32_t)((i / kXaStages) & 1), &abort_flag, err);
    if (!__syncthreads_and(ok ? 1 : 0)) {
      aborted = true;
      break;
    }
    const int r0 = lo + ((int)blockIdx.x + i * (int)gridDim.x) * p.chunk_rows;
    const int cnt = min(p.chunk_rows, hi - r0);
    const uint32_t base = smem_u32(xa_smem) + (uint32_t)st * stage_bytes + (uint32_t)lane * 16u;
    for (int b = 0; b < cnt; b += kXaWarps * U) {
      float h[U][8], sc_valid[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int r = b + warp * U + u;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (active && r < cnt) v = ld_shared_16(base + (uint32_t)r * row_bytes);
        unpack8(v, h[u]);
        sc_valid[u] = r < cnt ? 0.f : -INFINITY;
      }
#pragma unroll
      for (int a = 0; a < QB; ++a) {
        float sc[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          float d = 0.f;
#pragma unroll
          for (int c = 0; c < 8; ++c) d = fmaf(q[a][c], h[u][c], d);
          sc[u] = head_sum(d, p.lanes_per_head) + sc_valid[u];  // rows past the chunk: weight 0
        }
        online_update<U>(m[a], l[a], o[a], sc, h);
      }
    }
    __syncthreads();  // every warp is done with stage st
    if (threadIdx.x == 0 && issued < mine) issue(issued++);
  }
  if (aborted) {
    // after a wait ran out: let the copies still in flight land before the CTA exits
    if (threadIdx.x == 0) {
      volatile int never = 0;
      for (int i = 0; i < issued; ++i) mbar_wait(&full[i % kXaStages], (uint32_t)((i / kXaStages) & 1), &never, err,
                                                 kDefaultTimeoutNs);
    }
    __syncthreads();
    return;
  }

  // merge the warps in a fixed order through the (now idle) staging buffer
  float* st_state = reinterpret_cast<float*>(xa_smem);  // [warp][QB][kXaRec][32]
#pragma unroll
  for (int a = 0; a < QB; ++a) {
    float* w0 = st_state + ((warp * QB + a) * kXaRec) * 32 + lane;
    w0[0] = m[a];
    w0[32] = l[a];
#pragma unroll
    for (int c = 0; c < 8; ++c) w0[(2 + c) * 32] = o[a][c];
  }
  __syncthreads();
  if (warp < QB && warp < p.qb) {
    const int a = warp;
    float M = -INFINITY, L = 0.f, O[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) O[c] = 0.f;
    for (int w = 0; w < kXaWarps; ++w) {
      const float* r = st_state + ((w * QB + a) * kXaRec) * 32 + lane;
      float ow[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) ow[c] = r[(2 + c) * 32];
      merge_state(M, L, O, r[0], r[32], ow);
    }
    const size_t slot = (size_t)g * p.slots_per_group + p.slot0 + blockIdx.x;
    float* dst = p.part + ((slot * p.A + p.q0 + a) * kXaRec) * 32 + lane;
    dst[0] = M;
    dst[32] = L;
#pragma unroll
    for (int c = 0; c < 8; ++c) dst[(2 + c) * 32] = O[c];
  }
  if (flags && threadIdx.x == 0 && blockIdx.x == 0) atomicOr(p.status, flags);
}

// Merge of a (group, query)'s partials: one CTA of 32 warps; warp w folds slots w, w + 32, ...
// (four records in flight per lane) into a running (max, sum, weighted sum), then warp 0
// merges the 32 warps in order.  The assignment and the order are fixed: deterministic.
__global__ void __launch_bounds__(kXaCombineWarps * 32) xattn_combine_kernel(
    const float* __restrict__ part, int G, int A, int R, int slots_per_group, const __nv_bfloat16* __restrict__ aux,
    float* __restrict__ out) {
  __shared__ float s_state[kXaCombineWarps][kXaRec][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = blockIdx.x / A, a = blockIdx.x - (blockIdx.x / A) * A;
  pdl_wait();
  pdl_trigger();
  float M = -INFINITY, L = 0.f, O[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) O[c] = 0.f;
  const size_t stride = (size_t)A * kXaRec * 32;  // between consecutive slots of the group
  const float* base = part + (((size_t)g * slots_per_group) * A + a) * kXaRec * 32 + lane;
  for (int s0 = warp; s0 < slots_per_group; s0 += 4 * kXaCombineWarps) {
    float m[4], l[4], o[4][8];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int sl = s0 + u * kXaCombineWarps;
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
  for (int w = 0; w < kXaCombineWarps; ++w) {
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

// CTAs (= partial slots) per group: enough to fill the GPU once (each CTA keeps only its own
// three chunks in flight, so the bytes in flight scale with the CTAs), at most kXaCtaCap over
// all groups and at least 128 rows each.  A fixed number, so the workspace size needs no
// device query.
int xattn_slots(int max_rows, int G) {
  const int cap = G > 0 && kXaCtaCap / G > 0 ? kXaCtaCap / G : 1;
  const int b = max_rows <= 0 ? 1 : (max_rows + kXaRowsPerCta - 1) / kXaRowsPerCta;
  return b < cap ? b : cap;
}

cudaError_t launch_xattn_partials(const XattnLaunch& x, cudaStream_t s) {
  XattnParams p{};
  p.H = static_cast<const __nv_bfloat16*>(x.H);
  p.h_rows = x.h_rows;
  p.R = x.R;
  p.lanes_per_head = x.R / x.heads / 8;
  p.lo = x.lo;
  p.hi = x.hi;
  p.h_sub = x.h_sub;
  p.rows_cap = x.max_rows > 0 ? x.max_rows : 0;
  const int fit = kXaStageBytes / (x.R * 2) / 32 * 32;
  p.chunk_rows = fit > 32 ? fit : 32;
  const int slots = xattn_slots(x.max_rows, x.G);
  size_t smem = (size_t)kXaStages * p.chunk_rows * x.R * 2;
  const size_t state = (size_t)kXaWarps * kXaQB * kXaRec * 32 * sizeof(float);
  if (smem < state) smem = state;
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
    const dim3 grid(slots, x.G);
    // the staged chunks plus the kernel's static barriers exceed the default 48 KB limit
    static int done1[64], done4[64];
    if (p.qb == 1) {
      e = ensure_smem_attr(xattn_partial_kernel<1>, smem, done1);
      if (e == cudaSuccess) e = launch_pdl(xattn_partial_kernel<1>, grid, dim3(kXaWarps * 32), smem, s, p);
    } else {
      e = ensure_smem_attr(xattn_partial_kernel<kXaQB>, smem, done4);
      if (e == cudaSuccess) e = launch_pdl(xattn_partial_kernel<kXaQB>, grid, dim3(kXaWarps * 32), smem, s, p);
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_xattn_combine(const float* part, int G, int A, int R, int slots_per_group, const void* aux,
                                 float* out, cudaStream_t s) {
  if (G * A == 0) return cudaSuccess;
  return launch_pdl(xattn_combine_kernel, dim3(G * A), dim3(kXaCombineWarps * 32), 0, s, part, G, A, R,
                    slots_per_group, static_cast<const __nv_bfloat16*>(aux), out);
}

}  // namespace svc

// Neighbour-index build on the GPU (SV-TAD page, Key Design 1: the per-frame
// lookup map M, filled with -1 and then M[y_k, x_k] = k, and the neighbour table
// N[k, j] = M[y_k + dy_j, x_k + dx_j] or -1).  The page builds both on the CPU;
// here each CTA keeps the maps of a few consecutive frames in shared memory (as many
// frames per CTA as make the launch about one wave), so the table is produced next to
// the features with no host round trip.
//
// Traffic per token: 12 B of coordinates read (twice, the second time from L1/L2)
// and 36 B of N written; the writes are fully coalesced because consecutive
// threads produce consecutive (k, j) entries of the frame's contiguous N rows.
#include "svconv_internal.h"
#include "svconv_ptx.cuh"

namespace svc {
namespace {

constexpr int kIdxMaxFrames = 8;  // frames per CTA at most

// CTA b handles frames t0 = b * F .. t0 + F - 1 (F = frames_per_cta): their maps and token
// cells live in shared memory [F][H*W] each.  A frame whose offsets cannot be trusted is
// treated as empty (and flagged); a frame with more tokens than cells maps its first H*W
// tokens only (and flags DUPLICATE).  All threads of the CTA share the work of all its frames,
// so small frames do not leave most threads idle, and the launch is about one wave.
__global__ void __launch_bounds__(256) build_index_kernel(const int32_t* __restrict__ coords,
                                                          const int32_t* __restrict__ frame_off, int T, int H,
                                                          int W, int n, int frames_per_cta, int32_t* __restrict__ nbr,
                                                          int32_t* __restrict__ Mout, int32_t* status) {
  extern __shared__ int32_t smem[];
  const int HW = H * W;
  const int F = frames_per_cta;
  int32_t* sM = smem;               // [F][HW]
  int32_t* sCell = smem + F * HW;   // [F][HW]: each token's (y << 16 | x), or -1
  __shared__ int s_lo[kIdxMaxFrames], s_cnt[kIdxMaxFrames], s_pre[kIdxMaxFrames + 1];
  __shared__ int s_flags, s_contig;
  __shared__ int32_t sStage[8 * 32 * 9];  // per warp: 32 rows of 9 entries
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * F;
  const int nf = min(F, T - t0);
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) s_flags = 0;
  if (threadIdx.x < nf) {
    const int t = t0 + threadIdx.x;
    int lo = __ldg(frame_off + t), hi = __ldg(frame_off + t + 1);
    int flags = 0;
    if (lo < 0 || hi < lo || hi > n) flags |= SVCONV_STATUS_BAD_OFFSETS;
    if (t == 0 && lo != 0) flags |= SVCONV_STATUS_BAD_OFFSETS;
    if (t == T - 1 && hi != n) flags |= SVCONV_STATUS_BAD_OFFSETS;
    if (flags) lo = hi = 0;  // a segment that cannot be trusted is not touched
    if (hi - lo > HW) flags |= SVCONV_STATUS_DUPLICATE;  // more tokens than cells
    s_lo[threadIdx.x] = lo;
    s_cnt[threadIdx.x] = hi - lo;
    if (flags) atomicOr(&s_flags, flags);
  }
  for (int c = threadIdx.x; c < nf * HW; c += blockDim.x) sM[c] = -1;
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0, contig = 1;
    for (int f = 0; f < nf; ++f) {
      s_pre[f] = acc;
      acc += s_cnt[f];
      if (f > 0 && s_lo[f] != s_lo[f - 1] + s_cnt[f - 1]) contig = 0;
    }
    s_pre[nf] = acc;
    s_contig = contig;
  }
  __syncthreads();
  const int total_tok = s_pre[nf];

  // step 1: M[t][y_k][x_k] = k over all tokens of the CTA's frames.  With duplicates the
  // largest k wins (deterministic).
  for (int i = threadIdx.x; i < total_tok; i += blockDim.x) {
    int f = 0;
    while (f + 1 < nf && s_pre[f + 1] <= i) ++f;
    const int q = i - s_pre[f];
    const int k = s_lo[f] + q;
    const int tt = coords[3 * k], y = coords[3 * k + 1], x = coords[3 * k + 2];
    int cell = -1;
    if (tt != t0 + f) {
      atomicOr(&s_flags, SVCONV_STATUS_BAD_FRAME);
    } else if (y < 0 || y >= H || x < 0 || x >= W) {
      atomicOr(&s_flags, SVCONV_STATUS_BAD_COORD);
    } else {
      atomicMax(&sM[f * HW + y * W + x], k);
      cell = (y << 16) | x;  // kept as (y, x): the lookups below need no division
    }
    if (q < HW) sCell[f * HW + q] = cell;
  }
  __syncthreads();

  // step 2: the 9 lookups, one token per thread (the frame search and the unpacking happen
  // once per token; the taps unroll with constant offsets).  Each warp stages its 32 rows of
  // 9 entries in shared memory (9 is odd, so the staging is free of bank conflicts) and, when
  // the CTA's frames are contiguous in the table, writes them back as 9 coalesced stores.
  int32_t* stage = sStage + warp * 32 * 9;
  const bool contig = s_contig;
  const int row0 = s_lo[0];
  for (int base = warp * 32; base < total_tok; base += (int)blockDim.x) {
    const int i = base + lane;
    int32_t v[9];
    int row = -1;
    if (i < total_tok) {
      int f = 0;
      while (f + 1 < nf && s_pre[f + 1] <= i) ++f;
      const int q = i - s_pre[f];
      row = s_lo[f] + q;
      const int yx = q < HW ? sCell[f * HW + q] : -1;
      if (yx >= 0) {
        const int y = yx >> 16, x = yx & 0xffff;
        const int32_t* Mf = sM + f * HW;
        if (Mf[y * W + x] != row) atomicOr(&s_flags, SVCONV_STATUS_DUPLICATE);
#pragma unroll
        for (int j = 0; j < 9; ++j) {
          const int yy = y + j / 3 - 1, xx = x + j % 3 - 1;
          v[j] = (yy >= 0 && yy < H && xx >= 0 && xx < W) ? Mf[yy * W + xx] : -1;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 9; ++j) v[j] = -1;
      }
    }
    if (contig) {
      if (i < total_tok) {
#pragma unroll
        for (int j = 0; j < 9; ++j) stage[lane * 9 + j] = v[j];
      }
      __syncwarp();
      const int cnt = min(32, total_tok - base) * 9;
      int32_t* dst = nbr + (size_t)(row0 + base) * 9;
#pragma unroll
      for (int m = 0; m < 9; ++m) {
        const int idx = lane + 32 * m;
        if (idx < cnt) dst[idx] = stage[idx];
      }
      __syncwarp();
    } else if (i < total_tok) {
#pragma unroll
      for (int j = 0; j < 9; ++j) nbr[(size_t)row * 9 + j] = v[j];
    }
  }
  if (Mout) {
    for (int c = threadIdx.x; c < nf * HW; c += blockDim.x) Mout[(size_t)t0 * HW + c] = sM[c];
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_flags && status) atomicOr(status, s_flags);
}

}  // namespace

cudaError_t launch_build_index(const int32_t* coords, const int32_t* frame_off, int T, int H, int W, int n,
                               int32_t* nbr, int32_t* M, int32_t* status, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int HW = H * W;
  // frames per CTA: enough that the launch is about one wave (at most 8 CTAs of 256 threads
  // per SM), with the maps in at most 48 KB of shared memory
  const int waves_ctas = 8 * sm_count();
  int F = (T + waves_ctas - 1) / waves_ctas;
  if (F < 1) F = 1;
  if (F > kIdxMaxFrames) F = kIdxMaxFrames;
  while (F > 1 && (size_t)2 * sizeof(int32_t) * HW * F > 32 * 1024) --F;
  const size_t smem = 2 * sizeof(int32_t) * (size_t)HW * F;
  // beyond 48 KB of static (~10 KB) plus dynamic shared memory the kernel must opt in
  if (smem > 36 * 1024) {
    static int done[64];
    cudaError_t e = ensure_smem_attr(build_index_kernel, smem, done);
    if (e != cudaSuccess) return e;
  }
  const int grid = (T + F - 1) / F;
  return launch_pdl(build_index_kernel, dim3(grid), dim3(256), smem, s, coords, frame_off, T, H, W, n, F, nbr, M,
                    status);
}

}  // namespace svc

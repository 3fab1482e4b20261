// Neighbour-index build on the GPU (SV-TAD page, Key Design 1: the per-frame
// lookup map M, filled with -1 and then M[y_k, x_k] = k, and the neighbour table
// N[k, j] = M[y_k + dy_j, x_k + dx_j] or -1).  The page builds both on the CPU;
// here one CTA per frame keeps that frame's M in shared memory, so the table is
// produced next to the features with no host round trip.
//
// Traffic per token: 12 B of coordinates read (twice, the second time from L1/L2)
// and 36 B of N written; the writes are fully coalesced because consecutive
// threads produce consecutive (k, j) entries of the frame's contiguous N rows.
#include "svconv_internal.h"
#include "svconv_ptx.cuh"

namespace svc {
namespace {

__global__ void __launch_bounds__(256) build_index_kernel(const int32_t* __restrict__ coords,
                                                          const int32_t* __restrict__ frame_off, int T, int H,
                                                          int W, int n, int32_t* __restrict__ nbr,
                                                          int32_t* __restrict__ Mout, int32_t* status) {
  // shared: M of this frame [H*W], then each token's packed cell (y*W + x, or -1
  // when its coordinates are invalid) [H*W]; a valid frame holds at most H*W tokens.
  extern __shared__ int32_t smem[];
  const int HW = H * W;
  int32_t* sM = smem;
  int32_t* sCell = smem + HW;
  __shared__ int s_flags;
  const int t = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  // every thread reads the frame's bounds itself (a broadcast load), so no extra barrier
  // round trip is spent handing them out
  int lo = __ldg(frame_off + t), hi = __ldg(frame_off + t + 1);
  int flags = 0;
  if (lo < 0 || hi < lo || hi > n) flags |= SVCONV_STATUS_BAD_OFFSETS;
  if (t == 0 && lo != 0) flags |= SVCONV_STATUS_BAD_OFFSETS;
  if (t == T - 1 && hi != n) flags |= SVCONV_STATUS_BAD_OFFSETS;
  if (flags) lo = hi = 0;  // a segment that cannot be trusted is not touched
  if (hi - lo > HW) flags |= SVCONV_STATUS_DUPLICATE;  // more tokens than cells: only the first HW are mapped
  if (threadIdx.x == 0) s_flags = flags;
  for (int c = threadIdx.x; c < HW; c += blockDim.x) sM[c] = -1;
  __syncthreads();
  const int cnt = hi - lo;

  // step 1: M[y_k][x_k] = k.  With duplicates the largest k wins (deterministic).
  for (int q = threadIdx.x; q < cnt; q += blockDim.x) {
    const int k = lo + q;
    const int tt = coords[3 * k], y = coords[3 * k + 1], x = coords[3 * k + 2];
    int cell = -1;
    if (tt != t) {
      atomicOr(&s_flags, SVCONV_STATUS_BAD_FRAME);
    } else if (y < 0 || y >= H || x < 0 || x >= W) {
      atomicOr(&s_flags, SVCONV_STATUS_BAD_COORD);
    } else {
      cell = y * W + x;
      atomicMax(&sM[cell], k);
    }
    if (q < HW) sCell[q] = cell;
  }
  __syncthreads();

  // step 2: the 9 lookups, one (k, j) entry per thread, coalesced writes.
  const int mapped = cnt < HW ? cnt : HW;
  const int total = cnt * 9;  // cnt <= n < 2^31 / 9 is checked on the host
  int32_t* out = nbr + (size_t)lo * 9;
  for (int e = threadIdx.x; e < total; e += blockDim.x) {
    const int q = e / 9;
    const int j = e - q * 9;
    int32_t v = -1;
    const int cell = q < mapped ? sCell[q] : -1;
    if (cell >= 0) {
      const int y = cell / W, x = cell - y * W;
      if (j == 4 && sM[cell] != lo + q) atomicOr(&s_flags, SVCONV_STATUS_DUPLICATE);
      const int yy = y + j / 3 - 1, xx = x + j % 3 - 1;
      if (yy >= 0 && yy < H && xx >= 0 && xx < W) v = sM[yy * W + xx];
    }
    out[e] = v;
  }
  if (Mout) {
    int32_t* dst = Mout + (size_t)t * HW;
    for (int c = threadIdx.x; c < HW; c += blockDim.x) dst[c] = sM[c];
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_flags && status) atomicOr(status, s_flags);
}

}  // namespace

cudaError_t launch_build_index(const int32_t* coords, const int32_t* frame_off, int T, int H, int W, int n,
                               int32_t* nbr, int32_t* M, int32_t* status, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const size_t smem = 2 * sizeof(int32_t) * (size_t)H * W;
  if (smem > 48 * 1024) {
    static int done[64];
    cudaError_t e = ensure_smem_attr(build_index_kernel, smem, done);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(build_index_kernel, dim3(T), dim3(256), smem, s, coords, frame_off, T, H, W, n, nbr, M, status);
}

}  // namespace svc

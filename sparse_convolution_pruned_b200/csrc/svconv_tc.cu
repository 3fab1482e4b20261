// bf16 SparseConv2D on the 5th-generation tensor cores (tcgen05 + TMEM), fed by TMA.
//
// After the gather, each output tile is a dense contraction (SV-TAD page, Key
// Design 2: y_k = sum_j W_j x[N[k,j]] is a GEMM with K = 9 * C_in whose A rows
// are gathered through the neighbour table), so it runs as a warp-specialised,
// persistent implicit GEMM with every operand moved by the TMA engine:
//
//   warp 4 (producer)    per K-block (tap j, 64 channels): lane l issues one
//                        tile::gather4 TMA load for tile rows 4l..4l+3, i.e. four
//                        128-byte feature-row segments picked by the neighbour
//                        indices; an index of -1 is an out-of-range row, which the
//                        TMA unit fills with zeros (the padding of the page's
//                        equation).  Lane 0 also loads the weight tile B.  All of
//                        it lands in the 128B-swizzled layout tcgen05 reads and
//                        completes on one mbarrier (complete_tx).  The next tile's
//                        neighbour rows are prefetched into registers while the
//                        current tile streams.
//   warp 5 (MMA)         one thread issues tcgen05.mma (M=128, N=BN, K=16) into a
//                        double-buffered fp32 accumulator in TMEM and releases smem
//                        stages with tcgen05.commit.
//   warps 0-3 (epilogue) tcgen05.ld the accumulator (warp w owns TMEM lanes
//                        32w..32w+31 = tile rows), add bias / GELU / residual,
//                        convert to bf16 and store, overlapping the next tile.
//
// The data gradient is the same kernel: the gather goes through the mirrored
// column N[k][8-j] of dY and B = W_j^T is read straight from W[o][j][i] as an
// MN-major operand (3-D TMA box over (i, j, o)), so no transposed copy of W is
// made.  The dense adapter projections are the same kernel with one tap and a
// plain 2-D TMA box for A.
//
// The weight gradient dW^T[(j,i)][o] = sum_k X[N[k,j]][i] dY[k][o] is a GEMM with
// K = tokens: A (gathered X rows, MN-major) and B (dY by TMA, MN-major).  The bias
// gradient comes out of the same MMAs: the A row after the last (j, i) row is
// gathered from a constant [1, 0, ..., 0] row for every valid token, so its
// accumulator row is sum_k dY[k][o].  Token ranges are split over CTAs into fp32
// partials, reduced afterwards in a fixed order.
//
// No TMA multicast is used anywhere.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstring>

#include "svconv_internal.h"
#include "svconv_ptx.cuh"

namespace svc {

constexpr int kBM = 128;                 // tile rows (tokens / dW rows) = TMEM lanes
constexpr int kBK = 64;                  // bf16 elements per K-block (one 128-byte row)
constexpr int kABytes = kBM * kBK * 2;   // 16 KB per A stage
constexpr int kThreads = 6 * 32;         // 4 epilogue warps, 1 producer warp, 1 MMA warp
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kMaxStages = 8;
constexpr int kIdxPerLane = 4 * 9;       // conv: 4 tile rows x 9 taps per producer lane
constexpr int kWgChunk = 8;              // weight gradient: K-blocks whose indices are prefetched together

struct __align__(8) TcBarriers {
  uint64_t full[kMaxStages];    // A and B of the stage landed (arrive.expect_tx + TMA complete_tx)
  uint64_t empty[kMaxStages];   // MMA finished reading the stage (tcgen05.commit)
  uint64_t tfull[2];            // accumulator buffer ready for the epilogue
  uint64_t tempty[2];           // epilogue drained the accumulator buffer (one arrival per epilogue warp)
  uint64_t done;                // final MMA drain before TMEM is released
  uint32_t tmem_base;
  int abort_flag;
};

struct TcConvParams {
  CUtensorMap tmap_a;  // gather: box {64, 1}; dense: box {64, 128}
  CUtensorMap tmap_b;
  const int32_t* nbr;
  const int32_t* row_lo;
  const int32_t* row_hi;
  const float* bias;
  const __nv_bfloat16* residual;
  __nv_bfloat16* out;
  int* status;
  unsigned long long timeout_ns;
  int a_rows, taps, Kc;
  int M, a_abs, nbr_abs, out_abs, N;
  int gelu, ldo, out_rows, stages;
};

struct TcWgradParams {
  CUtensorMap tmap_x;     // X [n][Cin], box {64, 1}
  CUtensorMap tmap_ones;  // [1][64] constant row [1, 0, ..., 0], box {64, 1}
  CUtensorMap tmap_dy;    // dY [n][Cout], box {64, 64}
  const int32_t* nbr;
  float* partial;
  int* status;
  unsigned long long timeout_ns;
  int n, Cin, Cout, splits, rows_pad, stages;
};

// The constant row behind the all-ones A row of the weight gradient (bf16 1.0, then zeros).
__device__ __align__(128) uint16_t kOnesRow[64] = {0x3F80u};

__host__ __device__ constexpr int tmem_cols_for(int bn) {
  return (2 * bn) <= 32 ? 32 : (2 * bn) <= 64 ? 64 : (2 * bn) <= 128 ? 128 : (2 * bn) <= 256 ? 256 : 512;
}

__host__ __device__ constexpr size_t stage_bytes(int bn) { return (size_t)kABytes + (size_t)bn * kBK * 2; }

constexpr size_t kIdxSmemBytes = sizeof(int32_t) * kBM * 9;

static size_t smem_bytes(int bn, int stages) {
  return 1024 /* alignment slack */ + stage_bytes(bn) * stages + kIdxSmemBytes + sizeof(TcBarriers);
}

struct TileCarve {
  uint8_t* a;
  uint8_t* b;
  int32_t* idx;
  TcBarriers* bar;
};

template <int BN>
__device__ __forceinline__ TileCarve carve(uint8_t* smem_raw, int stages) {
  const uint32_t base = smem_u32(smem_raw);
  const uint32_t pad = ((base + 1023u) & ~1023u) - base;
  uint8_t* s = smem_raw + pad;
  TileCarve c;
  c.a = s;
  c.b = s + (size_t)stages * kABytes;
  c.idx = reinterpret_cast<int32_t*>(c.b + (size_t)stages * BN * kBK * 2);
  c.bar = reinterpret_cast<TcBarriers*>(reinterpret_cast<uint8_t*>(c.idx) + kIdxSmemBytes);
  return c;
}

__device__ __forceinline__ void init_barriers(TcBarriers* b, int stages) {
  for (int s = 0; s < stages; ++s) {
    mbar_init(&b->full[s], 1);
    mbar_init(&b->empty[s], 1);
  }
  for (int i = 0; i < 2; ++i) {
    mbar_init(&b->tfull[i], 1);
    mbar_init(&b->tempty[i], 4);
  }
  mbar_init(&b->done, 1);
  b->abort_flag = 0;
  fence_barrier_init();
  fence_proxy_async_smem();
}

// Lane 0 of the warp waits, the verdict is broadcast: control flow stays
// warp-uniform even when a wait gives up.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err,
                                          uint64_t timeout_ns) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag, err, timeout_ns);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Producer exit after an abort: wait (bounded, ignoring the abort flag) until
// every TMA load still in flight has landed, so none writes after the CTA exits.
__device__ __forceinline__ void producer_drain(TcBarriers* bar, uint32_t it, int stages, bool aborted, int* err,
                                               uint64_t timeout_ns) {
  if (aborted && (threadIdx.x & 31) == 0) {
    volatile int never = 0;
    const uint32_t lo = it >= (uint32_t)stages ? it - stages : 0u;
    for (uint32_t q = lo; q < it; ++q) mbar_wait(&bar->full[q % stages], (q / stages) & 1u, &never, err, timeout_ns);
  }
  __syncwarp();
}

// Shared-memory descriptor geometry for the MMA issuer.
// a_step / b_step: byte advance of the descriptors' start address per K=16 step.
struct MmaCfg {
  uint32_t idesc;
  uint32_t a_lbo, a_sbo, a_step;
  uint32_t b_lbo, b_sbo, b_step;
};

// One thread issues the MMAs of one tile (num_kb K-blocks) into accumulator d.
__device__ __forceinline__ bool mma_tile(TcBarriers* bar, const TileCarve& sm, uint32_t b_bytes, int S, uint32_t& it,
                                         int num_kb, uint32_t d, const MmaCfg& c, volatile int* abort_flag, int* err,
                                         uint64_t timeout_ns) {
  for (int kb = 0; kb < num_kb; ++kb, ++it) {
    const int s = it % S;
    const uint32_t ph = (it / S) & 1u;
    if (!mbar_wait(&bar->full[s], ph, abort_flag, err, timeout_ns)) return false;
    tc_fence_after();
    const uint32_t a0 = smem_u32(sm.a + (size_t)s * kABytes);
    const uint32_t b0 = smem_u32(sm.b + (size_t)s * b_bytes);
#pragma unroll
    for (int k = 0; k < kBK / 16; ++k) {
      const uint64_t ad = smem_desc_sw128(a0 + k * c.a_step, c.a_lbo, c.a_sbo);
      const uint64_t bd = smem_desc_sw128(b0 + k * c.b_step, c.b_lbo, c.b_sbo);
      tc_mma_bf16(d, ad, bd, c.idesc, (kb | k) != 0 ? 1u : 0u);
    }
    tc_commit(&bar->empty[s]);
  }
  return true;
}

// ============================================================================ conv / dense GEMM
// MIRROR: gather through column 8-j (data gradient), which always pairs with an
// MN-major weight operand.
template <int BN, bool MIRROR>
__global__ void __launch_bounds__(kThreads, 1) tc_conv_kernel(const __grid_constant__ TcConvParams p) {
  extern __shared__ uint8_t smem_raw[];
  const int S = p.stages;
  TileCarve sm = carve<BN>(smem_raw, S);
  TcBarriers* bar = sm.bar;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* err = p.status;
  constexpr uint32_t kBBytes = BN * kBK * 2;
  constexpr uint32_t kTmemCols = tmem_cols_for(BN);
  constexpr bool B_MN = MIRROR;

  // rows handled by this launch (device-side bounds for the chunked adapter)
  int lo = 0, M = p.M;
  if (p.row_lo) {
    lo = *p.row_lo;
    int m = *p.row_hi - lo;
    if (m > p.M) {
      if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(err, SVCONV_STATUS_CHUNK_OVERFLOW);
      m = p.M;
    }
    M = m < 0 ? 0 : m;
  }
  const int m_tiles = (M + kBM - 1) / kBM;
  const int n_tiles = p.N / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int kb_per_tap = p.Kc / kBK;
  const int num_kb = p.taps * kb_per_tap;
  const bool gather = p.nbr != nullptr;

  if (threadIdx.x == 0) {
    init_barriers(bar, S);
    prefetch_tmap(&p.tmap_a);
    prefetch_tmap(&p.tmap_b);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bar->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bar->tmem_base;
  volatile int* abort_flag = &bar->abort_flag;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    const int nbr_base = p.nbr_abs ? lo : 0;
    const int a_base = p.a_abs ? lo : 0;
    uint32_t it = 0;
    bool aborted = false;
    // Neighbour rows of a tile: raw[i] = entry (lane + 32 i) of the tile's 128 x 9
    // block of N (coalesced loads, all in flight together), then re-read through
    // shared memory as cur[q * 9 + j] = N[m0 + 4*lane + q][j], validated and rebased.
    int raw[kIdxPerLane];
    int cur[kIdxPerLane];
    auto load_raw = [&](int tile) {
      const int m0 = (tile / n_tiles) * kBM;
      const int32_t* src = p.nbr + (size_t)(nbr_base + m0) * 9;
      const int lim = (M - m0) * 9;  // entries of valid rows
#pragma unroll
      for (int i = 0; i < kIdxPerLane; ++i) {
        const int e = lane + 32 * i;
        raw[i] = e < lim ? __ldg(src + e) : -1;
      }
    };
    auto publish_raw = [&]() {
      __syncwarp();
#pragma unroll
      for (int i = 0; i < kIdxPerLane; ++i) {
        int v = raw[i];
        if (v >= 0) {
          v -= nbr_base;
          if ((unsigned)v >= (unsigned)p.a_rows) {
            atomicOr(err, SVCONV_STATUS_BAD_INDEX);
            v = -1;
          }
        }
        sm.idx[lane + 32 * i] = v;
      }
      __syncwarp();
#pragma unroll
      for (int i = 0; i < kIdxPerLane; ++i) cur[i] = sm.idx[lane * kIdxPerLane + i];
    };
    if (gather && (int)blockIdx.x < num_tiles) {
      load_raw(blockIdx.x);
      publish_raw();
    }
    for (int tile = blockIdx.x; tile < num_tiles && !aborted; tile += gridDim.x) {
      const int m0 = (tile / n_tiles) * kBM;
      const int n0 = (tile % n_tiles) * BN;
      const int next = tile + gridDim.x;
      const bool prefetch = gather && next < num_tiles;
      // one K-block: wait for the stage, arm it, load B and A
      auto issue = [&](int j, int cb, int y0, int y1, int y2, int y3) -> bool {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1u;
        if (!warp_wait(&bar->empty[s], ph ^ 1u, abort_flag, err, p.timeout_ns)) return false;
        uint8_t* sb = sm.b + (size_t)s * kBBytes;
        const uint32_t sa = smem_u32(sm.a + (size_t)s * kABytes);
        if (lane == 0) {
          mbar_arrive_expect_tx(&bar->full[s], (uint32_t)kABytes + kBBytes);
          if constexpr (!B_MN) {
            tma_load_2d(smem_u32(sb), &p.tmap_b, &bar->full[s], j * p.Kc + cb * kBK, n0);
          } else {
#pragma unroll
            for (int q = 0; q < BN / 64; ++q)
              tma_load_3d(smem_u32(sb + q * 8192), &p.tmap_b, &bar->full[s], n0 + q * 64, j, cb * kBK);
          }
          if (!gather) tma_load_2d(sa, &p.tmap_a, &bar->full[s], cb * kBK, a_base + m0);
        }
        __syncwarp();
        if (gather) tma_gather4(sa + lane * 512, &p.tmap_a, &bar->full[s], cb * kBK, y0, y1, y2, y3);
        ++it;
        return true;
      };
      if (gather) {
#pragma unroll
        for (int j = 0; j < 9; ++j) {
          const int jj = MIRROR ? 8 - j : j;
          for (int cb = 0; cb < kb_per_tap; ++cb) {
            if (!issue(j, cb, cur[jj], cur[9 + jj], cur[18 + jj], cur[27 + jj])) {
              aborted = true;
              break;
            }
            if (prefetch && j == 0 && cb == 0) load_raw(next);  // overlaps this tile's stream
          }
          if (aborted) break;
        }
        if (!aborted && prefetch) publish_raw();
      } else {
        for (int cb = 0; cb < kb_per_tap; ++cb)
          if (!issue(0, cb, 0, 0, 0, 0)) {
            aborted = true;
            break;
          }
      }
    }
    producer_drain(bar, it, S, aborted, err, p.timeout_ns);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      MmaCfg c;
      c.idesc = idesc_bf16_f32(kBM, BN, 0, B_MN ? 1 : 0);
      c.a_lbo = 16, c.a_sbo = 1024, c.a_step = 32;  // A: K-major, 128-byte rows
      if (B_MN) {
        c.b_lbo = 8192, c.b_sbo = 1024, c.b_step = 2048;  // B: MN-major, 64-wide MN groups 8 KB apart
      } else {
        c.b_lbo = 16, c.b_sbo = 1024, c.b_step = 32;
      }
      uint32_t it = 0, tc = 0;
      bool issued = false;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tc) {
        const uint32_t ab = tc & 1u, aph = (tc >> 1) & 1u;
        if (!mbar_wait(&bar->tempty[ab], aph ^ 1u, abort_flag, err, p.timeout_ns)) break;
        tc_fence_after();
        issued = true;
        if (!mma_tile(bar, sm, kBBytes, S, it, num_kb, tmem_base + ab * BN, c, abort_flag, err, p.timeout_ns)) break;
        tc_commit(&bar->tfull[ab]);
      }
      if (issued) {
        volatile int never = 0;
        tc_commit(&bar->done);
        mbar_wait(&bar->done, 0, &never, err, p.timeout_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-3)
    uint32_t tc = 0;
    const int out_base = p.out_abs ? lo : 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tc) {
      const uint32_t ab = tc & 1u, aph = (tc >> 1) & 1u;
      if (!warp_wait(&bar->tfull[ab], aph, abort_flag, err, p.timeout_ns)) break;
      tc_fence_after();
      const int m0 = (tile / n_tiles) * kBM;
      const int n0 = (tile % n_tiles) * BN;
      const int row = m0 + warp * 32 + lane;
      const int orow_i = out_base + row;
      const bool valid = row < M && orow_i >= 0 && orow_i < p.out_rows;
      const size_t orow = (size_t)orow_i;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(warp * 32) << 16) + ab * BN + c0, v);
        tmem_ld_wait();
        if (valid) {
          float f[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) f[q] = __uint_as_float(v[q]);
          if (p.bias) {
#pragma unroll
            for (int q = 0; q < 32; ++q) f[q] += __ldg(p.bias + n0 + c0 + q);
          }
          if (p.gelu) {
#pragma unroll
            for (int q = 0; q < 32; ++q) f[q] = 0.5f * f[q] * (1.0f + erff(f[q] * 0.70710678118654752f));
          }
          if (p.residual) {
            const uint4* rp = reinterpret_cast<const uint4*>(p.residual + orow * p.ldo + n0 + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 u = rp[q];
              const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float2 x2 = __bfloat1622float2(h[e]);
                f[q * 8 + 2 * e] += x2.x;
                f[q * 8 + 2 * e + 1] += x2.y;
              }
            }
          }
          uint4* op = reinterpret_cast<uint4*>(p.out + orow * p.ldo + n0 + c0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 u;
            __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(f[q * 8 + 2 * e], f[q * 8 + 2 * e + 1]);
            op[q] = u;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->tempty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ============================================================================ weight gradient
template <int BN>
__global__ void __launch_bounds__(kThreads, 1) tc_wgrad_kernel(const __grid_constant__ TcWgradParams p) {
  extern __shared__ uint8_t smem_raw[];
  const int S = p.stages;
  TileCarve sm = carve<BN>(smem_raw, S);
  TcBarriers* bar = sm.bar;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* err = p.status;
  constexpr uint32_t kBBytes = BN * kBK * 2;
  constexpr uint32_t kTmemCols = tmem_cols_for(BN);

  const int m_tiles = p.rows_pad / kBM;
  const int n_tiles = p.Cout / BN;
  const int num_units = m_tiles * n_tiles * p.splits;
  const int kbt = (p.n + kBK - 1) / kBK;  // token blocks in total
  const int wrows = 9 * p.Cin;             // real dW rows; row wrows is db

  if (threadIdx.x == 0) {
    init_barriers(bar, S);
    prefetch_tmap(&p.tmap_x);
    prefetch_tmap(&p.tmap_ones);
    prefetch_tmap(&p.tmap_dy);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bar->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bar->tmem_base;
  volatile int* abort_flag = &bar->abort_flag;

  // unit -> (split, m-tile, n-tile); units of one split run side by side so the
  // tiles of dY and the gathered X rows they share are hot in L2.
  auto decode = [&](int u, int& sp, int& m0, int& n0, int& kb0, int& kb1) {
    const int nt = u % n_tiles;
    const int rest = u / n_tiles;
    const int mt = rest % m_tiles;
    sp = rest / m_tiles;
    m0 = mt * kBM;
    n0 = nt * BN;
    kb0 = (int)((long long)kbt * sp / p.splits);
    kb1 = (int)((long long)kbt * (sp + 1) / p.splits);
  };

  if (warp == kProducerWarp) {
    // Lane l fills 4 token rows (4*(l & 15) .. +3) of A-half (l >> 4); the half is
    // 64 dW rows = one (tap, 64-channel block), the all-ones row, or padding.
    const int h = lane >> 4;
    const int kq = 4 * (lane & 15);
    uint32_t it = 0;
    bool aborted = false;
    for (int u = blockIdx.x; u < num_units && !aborted; u += gridDim.x) {
      int sp, m0, n0, kb0, kb1;
      decode(u, sp, m0, n0, kb0, kb1);
      const int mh = m0 + 64 * h;
      const int kind = mh < wrows ? 0 : (mh == wrows ? 1 : 2);  // 0 gather, 1 ones, 2 padding (not loaded)
      const int jh = kind == 0 ? mh / p.Cin : 0;
      const int i0 = kind == 0 ? mh - jh * p.Cin : 0;
      // padding halves are not loaded: their accumulator rows are never read
      const uint32_t a_bytes = (m0 <= wrows ? 8192u : 0u) + (m0 + 64 <= wrows ? 8192u : 0u);
      int cur[kWgChunk][4], nxt[kWgChunk][4];
      auto load_chunk = [&](int kbc, int (&dst)[kWgChunk][4]) {
#pragma unroll
        for (int c = 0; c < kWgChunk; ++c)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int k = (kbc + c) * kBK + kq + q;
            int v = -1;
            if (kbc + c < kb1 && k < p.n) v = kind == 0 ? __ldg(p.nbr + (size_t)k * 9 + jh) : 0;
            dst[c][q] = v;
          }
      };
      load_chunk(kb0, cur);
      for (int kbc = kb0; kbc < kb1 && !aborted; kbc += kWgChunk) {
        if (kbc + kWgChunk < kb1) load_chunk(kbc + kWgChunk, nxt);
#pragma unroll
        for (int c = 0; c < kWgChunk; ++c) {
          const int kb = kbc + c;
          if (kb >= kb1) break;
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!warp_wait(&bar->empty[s], ph ^ 1u, abort_flag, err, p.timeout_ns)) {
            aborted = true;
            break;
          }
          uint8_t* sb = sm.b + (size_t)s * kBBytes;
          const uint32_t sa = smem_u32(sm.a + (size_t)s * kABytes);
          if (lane == 0) {
            mbar_arrive_expect_tx(&bar->full[s], a_bytes + kBBytes);
#pragma unroll
            for (int q = 0; q < BN / 64; ++q)
              tma_load_2d(smem_u32(sb + q * 8192), &p.tmap_dy, &bar->full[s], n0 + q * 64, kb * kBK);
          }
          __syncwarp();
          int y[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            y[q] = cur[c][q];
            if (kind == 0 && y[q] >= p.n) {
              atomicOr(err, SVCONV_STATUS_BAD_INDEX);
              y[q] = -1;
            }
          }
          const uint32_t dst = sa + h * 8192 + kq * 128;
          if (kind == 0)
            tma_gather4(dst, &p.tmap_x, &bar->full[s], i0, y[0], y[1], y[2], y[3]);
          else if (kind == 1)
            tma_gather4(dst, &p.tmap_ones, &bar->full[s], 0, y[0], y[1], y[2], y[3]);
          ++it;
        }
#pragma unroll
        for (int c = 0; c < kWgChunk; ++c)
#pragma unroll
          for (int q = 0; q < 4; ++q) cur[c][q] = nxt[c][q];
      }
    }
    producer_drain(bar, it, S, aborted, err, p.timeout_ns);
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      MmaCfg c;
      c.idesc = idesc_bf16_f32(kBM, BN, 1, 1);
      c.a_lbo = 8192, c.a_sbo = 1024, c.a_step = 2048;  // both MN-major: 64-wide groups 8 KB apart
      c.b_lbo = 8192, c.b_sbo = 1024, c.b_step = 2048;
      uint32_t it = 0, tc = 0;
      bool issued = false;
      for (int u = blockIdx.x; u < num_units; u += gridDim.x, ++tc) {
        int sp, m0, n0, kb0, kb1;
        decode(u, sp, m0, n0, kb0, kb1);
        const uint32_t ab = tc & 1u, aph = (tc >> 1) & 1u;
        if (!mbar_wait(&bar->tempty[ab], aph ^ 1u, abort_flag, err, p.timeout_ns)) break;
        tc_fence_after();
        issued = true;
        if (!mma_tile(bar, sm, kBBytes, S, it, kb1 - kb0, tmem_base + ab * BN, c, abort_flag, err, p.timeout_ns))
          break;
        tc_commit(&bar->tfull[ab]);
      }
      if (issued) {
        volatile int never = 0;
        tc_commit(&bar->done);
        mbar_wait(&bar->done, 0, &never, err, p.timeout_ns);
      }
    }
    __syncwarp();
  } else {
    uint32_t tc = 0;
    for (int u = blockIdx.x; u < num_units; u += gridDim.x, ++tc) {
      int sp, m0, n0, kb0, kb1;
      decode(u, sp, m0, n0, kb0, kb1);
      const uint32_t ab = tc & 1u, aph = (tc >> 1) & 1u;
      const bool empty_range = kb1 <= kb0;  // no MMA ran for this unit: its partial is zero
      if (!warp_wait(&bar->tfull[ab], aph, abort_flag, err, p.timeout_ns)) break;
      tc_fence_after();
      const int row = m0 + warp * 32 + lane;
      float* dst = p.partial + ((size_t)sp * p.rows_pad + row) * p.Cout + n0;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(warp * 32) << 16) + ab * BN + c0, v);
        tmem_ld_wait();
        float4* o4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 w;
          w.x = empty_range ? 0.f : __uint_as_float(v[4 * q]);
          w.y = empty_range ? 0.f : __uint_as_float(v[4 * q + 1]);
          w.z = empty_range ? 0.f : __uint_as_float(v[4 * q + 2]);
          w.w = empty_range ? 0.f : __uint_as_float(v[4 * q + 3]);
          o4[q] = w;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->tempty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ============================================================================ failure-detection self test
__global__ void timeout_selftest_kernel(int32_t* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // nothing ever arrives
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, (volatile int*)&abort_flag, status, timeout_ns);
}

// ============================================================================ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 tensor map with 128-byte swizzle and zero fill outside the tensor;
// dims / strides innermost first (strides in bytes, rank-1 of them).
static bool make_tmap(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
                      const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides[i];
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// rows x cols (bf16, row-major) with a box of box_rows x 64
static bool make_rows_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {cols * 2};
  const uint32_t box[2] = {64u, box_rows};
  return make_tmap(m, base, 2, dims, strides, box);
}

static int pick_stages(int bn) {
  const size_t budget = 220 * 1024;
  const size_t fixed = 1024 + kIdxSmemBytes + sizeof(TcBarriers);
  int s = (int)((budget - fixed) / stage_bytes(bn));
  if (s > kMaxStages) s = kMaxStages;
  return s;
}

template <int BN, bool MIRROR>
static cudaError_t launch_conv_inst(TcConvParams& prm, int grid, cudaStream_t s) {
  prm.stages = pick_stages(BN);
  const size_t smem = smem_bytes(BN, prm.stages);
  static int done[64];
  cudaError_t e = ensure_smem_attr(tc_conv_kernel<BN, MIRROR>, smem, done);
  if (e != cudaSuccess) return e;
  tc_conv_kernel<BN, MIRROR><<<grid, kThreads, smem, s>>>(prm);
  return cudaGetLastError();
}

cudaError_t launch_tc_conv(const TcConvArgs& a, const void* Wt, int w_rows, int w_cols, int bn, cudaStream_t s) {
  TcConvParams prm;
  memset(&prm, 0, sizeof(prm));
  if (a.mirror != a.b_mn_major) return cudaErrorInvalidValue;  // the data gradient pairs both
  if (a.nbr && a.taps != 9) return cudaErrorInvalidValue;
  // A operand: gathered rows (box 64 x 1) or a dense 128-row box
  if (!make_rows_tmap(&prm.tmap_a, a.A, (uint64_t)a.a_rows, (uint64_t)a.lda, a.nbr ? 1u : (uint32_t)kBM))
    return cudaErrorInvalidValue;
  if (!a.b_mn_major) {
    // W viewed as [w_rows][w_cols] (rows = output channels, K contiguous)
    if (!make_rows_tmap(&prm.tmap_b, Wt, (uint64_t)w_rows, (uint64_t)w_cols, (uint32_t)bn)) return cudaErrorInvalidValue;
  } else {
    // W [Kc rows (o)][9][N cols (i)]: dims (i, j, o), box (64, 1, 64)
    const uint64_t dims[3] = {(uint64_t)a.N, 9u, (uint64_t)a.Kc};
    const uint64_t strides[2] = {(uint64_t)a.N * 2, (uint64_t)a.N * 9 * 2};
    const uint32_t box[3] = {64u, 1u, 64u};
    if (!make_tmap(&prm.tmap_b, Wt, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  prm.nbr = a.nbr;
  prm.row_lo = a.row_lo;
  prm.row_hi = a.row_hi;
  prm.bias = a.bias;
  prm.residual = static_cast<const __nv_bfloat16*>(a.residual);
  prm.out = static_cast<__nv_bfloat16*>(a.out);
  prm.status = a.status ? a.status : device_error_word();
  prm.timeout_ns = kDefaultTimeoutNs;
  prm.a_rows = a.a_rows;
  prm.taps = a.taps;
  prm.Kc = a.Kc;
  prm.M = a.M;
  prm.a_abs = a.a_abs;
  prm.nbr_abs = a.nbr_abs;
  prm.out_abs = a.out_abs;
  prm.N = a.N;
  prm.gelu = a.gelu;
  prm.ldo = a.ldo;
  prm.out_rows = a.out_rows;
  const int tiles = ((a.M + kBM - 1) / kBM) * (a.N / bn);
  if (tiles == 0) return cudaSuccess;
  int grid = sm_count();
  if (grid > tiles) grid = tiles;
  if (bn == 256) return a.mirror ? launch_conv_inst<256, true>(prm, grid, s) : launch_conv_inst<256, false>(prm, grid, s);
  if (bn == 128) return a.mirror ? launch_conv_inst<128, true>(prm, grid, s) : launch_conv_inst<128, false>(prm, grid, s);
  if (bn == 64) return a.mirror ? launch_conv_inst<64, true>(prm, grid, s) : launch_conv_inst<64, false>(prm, grid, s);
  return cudaErrorInvalidValue;
}

static int wgrad_bn(int Cout) { return Cout % 256 == 0 ? 256 : Cout % 128 == 0 ? 128 : 64; }

void tc_wgrad_plan(int n, int Cin, int Cout, int* splits, int* rows_pad, int* bn) {
  const int b = wgrad_bn(Cout);
  const int rp = ((9 * Cin + 1 + kBM - 1) / kBM) * kBM;
  const int base_units = (rp / kBM) * (Cout / b);
  const int kbt = (n + kBK - 1) / kBK;
  int sp = sm_count() / base_units;
  if (sp < 1) sp = 1;
  if (sp > kbt) sp = kbt > 0 ? kbt : 1;
  *splits = sp;
  *rows_pad = rp;
  *bn = b;
}

template <int BN>
static cudaError_t launch_wgrad_inst(TcWgradParams& prm, int grid, cudaStream_t s) {
  prm.stages = pick_stages(BN);
  const size_t smem = smem_bytes(BN, prm.stages);
  static int done[64];
  cudaError_t e = ensure_smem_attr(tc_wgrad_kernel<BN>, smem, done);
  if (e != cudaSuccess) return e;
  tc_wgrad_kernel<BN><<<grid, kThreads, smem, s>>>(prm);
  return cudaGetLastError();
}

static const void* ones_row_address() {
  static const void* addr[64];
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return nullptr;
  if (!addr[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, kOnesRow) != cudaSuccess) return nullptr;
    addr[d] = p;
  }
  return addr[d];
}

cudaError_t launch_tc_wgrad(const TcWgradArgs& a, cudaStream_t s) {
  TcWgradParams prm;
  memset(&prm, 0, sizeof(prm));
  int splits, rows_pad, bn;
  tc_wgrad_plan(a.n, a.Cin, a.Cout, &splits, &rows_pad, &bn);
  if (splits != a.splits || rows_pad != a.rows_pad) return cudaErrorInvalidValue;
  const void* ones = ones_row_address();
  if (!ones) return cudaErrorInvalidValue;
  if (!make_rows_tmap(&prm.tmap_x, a.X, (uint64_t)a.n, (uint64_t)a.Cin, 1u)) return cudaErrorInvalidValue;
  if (!make_rows_tmap(&prm.tmap_ones, ones, 1u, 64u, 1u)) return cudaErrorInvalidValue;
  if (!make_rows_tmap(&prm.tmap_dy, a.dY, (uint64_t)a.n, (uint64_t)a.Cout, 64u)) return cudaErrorInvalidValue;
  prm.nbr = a.nbr;
  prm.partial = a.partial;
  prm.status = device_error_word();
  prm.timeout_ns = kDefaultTimeoutNs;
  prm.n = a.n;
  prm.Cin = a.Cin;
  prm.Cout = a.Cout;
  prm.splits = splits;
  prm.rows_pad = rows_pad;
  const int units = (rows_pad / kBM) * (a.Cout / bn) * splits;
  int grid = sm_count();
  if (grid > units) grid = units;
  if (bn == 256) return launch_wgrad_inst<256>(prm, grid, s);
  if (bn == 128) return launch_wgrad_inst<128>(prm, grid, s);
  return launch_wgrad_inst<64>(prm, grid, s);
}

cudaError_t launch_timeout_selftest(int32_t* status, uint64_t timeout_ns, cudaStream_t s) {
  timeout_selftest_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace svc

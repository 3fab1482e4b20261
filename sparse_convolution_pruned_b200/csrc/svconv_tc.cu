// bf16 SparseConv2D on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// After the gather, each output tile is a dense contraction (SV-TAD page, Key
// Design 2: y_k = sum_j W_j x[N[k,j]] is a GEMM with K = 9 * C_in whose A rows
// are gathered through the neighbour table).  The kernels below run it as a
// warp-specialised, persistent implicit GEMM.
//
// Gathering each neighbour row from global memory once per tap moves 9x the
// unique bytes through L2 in 128-byte pieces, and such row gathers are limited
// by the number of requests an SM can keep in flight.  Instead, the rows a tile
// needs are staged once: tokens are packed frame by frame (the page's packed
// sequence), and within a frame in raster order a neighbour is at most W + 1
// packed rows away, so the neighbours of 128 consecutive tokens lie in one
// short contiguous "halo" range of rows.  The kernels stage the fixed window of
// rows m0 - 32 .. m0 + 127 + 32 around a tile (valid for W <= 31) with a few
// large TMA boxes, issued together with the tile's index entries since the
// window does not depend on them, and assemble the A tile of every tap from it.
// A neighbour outside the window (wider grids, tokens not in raster order) is
// read from global memory instead: the result is the same, only slower.
//
// Warp roles (480 threads):
//   warps 0-3    epilogue: tcgen05.ld the fp32 accumulator (warp w owns TMEM
//                lanes 32w..32w+31 = tile rows), bias / GELU, bf16 boxes staged in
//                shared memory and written by TMA stores (an in-place residual by TMA
//                reduce-adds); rows of a ragged last tile are stored per thread.
//   warps 4-11   A builders (gather): copy each tile row's neighbour segment from the
//                halo (zeros for -1 = padding) straight into the tensor-memory A stage
//                with tcgen05.st; idle in dense mode.
//   warp 12      index / halo loader: cp.async / bulk copy of the tile's neighbour
//                entries and the halo window's TMA boxes (or, for the dense adapter
//                projections, TMA of the A tile itself).
//   warp 13      weight loader: TMA of the B tile (W_j, or W_j^T straight from
//                W[o][j][i] as an MN-major operand for the data gradient).
//   warp 14      MMA issuer: one thread issues tcgen05.mma (K=16) into a TMEM
//                accumulator and tcgen05.commit frees stages.  A gather stage holds two
//                64-deep K-blocks, and A stage s and B stage s share one full / empty
//                barrier pair, so the issuer waits and commits once per 8 MMAs.
//
// 256-column tiles run on CTA pairs (clusters of 2, cta_group::2): M = 256 MMAs over
// both SMs' tensor memory, issued by CTA rank 0; each CTA gathers its own 128 rows and
// loads half of B, and rank 0's barriers count both CTAs' producers.
//
// The data gradient is the same kernel: the gather goes through the mirrored
// column N[k][8-j] of dY.  The weight gradient dW^T[(j,i)][o] = sum_k X[N[k,j]][i]
// dY[k][o] is a GEMM with K = tokens, A (gathered X, transposed into tensor memory,
// assembled from a halo per 64-token block) and B (dY by TMA, MN-major).  The bias
// gradient comes out of the same MMAs: the A row after the last (j, i) row is 1 for
// every valid token, so its accumulator row is sum_k dY[k][o].  Token ranges are split
// over CTAs into fp32 partials, reduced afterwards in a fixed order.
//
// No TMA or bulk load uses cluster multicast; the only multicast is tcgen05.commit's
// arrival on the barriers of both CTAs of a pair.
#include <cuda.h>
#include <cuda_bf16.h>

#include <climits>
#include <cstring>
#include <mutex>

#include "svconv_internal.h"
#include "svconv_ptx.cuh"

namespace svc {

constexpr int kBM = 128;                // tile rows (tokens / dW rows) = TMEM lanes
constexpr int kBK = 64;                 // bf16 elements per K-block (one 128-byte row)
constexpr int kABytes = kBM * kBK * 2;  // 16 KB per A stage
constexpr int kEpiWarps = 4;
constexpr int kProdWarps = 8;
constexpr int kHaloWarp = kEpiWarps + kProdWarps;  // 12
constexpr int kBWarp = kHaloWarp + 1;              // 13
constexpr int kMmaWarp = kBWarp + 1;               // 14
constexpr int kThreads = (kMmaWarp + 1) * 32;      // 480
constexpr int kMaxStages = 8;
constexpr int kHaloBox = 64;                       // rows per halo TMA box
constexpr int kConvPad = 32;                       // conv halo margin: W + 1 <= 32 stays inside
constexpr int kConvHaloRows = kBM + 2 * kConvPad;  // conv halo window (A rows m0 - 32 .. m0 + 159)
constexpr int kWgPad = 32;                         // weight-gradient halo margin: W + 1 <= 32 stays inside
constexpr int kWgHaloRows = kBK + 2 * kWgPad;      // weight-gradient halo window (rows k0 - 32 .. k0 + 95)
// Weight gradient: index + halo slots in flight (one per 64-token block).  8 cover ~2 us of
// load latency at small C.  At 256 columns three builder groups hold three slots and the
// loader runs ahead by two; the 32 KB dY (or dY-pair) stages take the rest of the space.
__host__ __device__ constexpr int wgrad_slots(int bn, bool pair = false) { return bn == 256 ? 5 : 8; }
// Weight gradient on CTA pairs: at most this many two-block stages fit next to the 256-column
// accumulator in tensor memory (2 x 32 columns each).
constexpr int kWgPairStagesMax = 4;
constexpr int kWgTiles = 5;                        // weight gradient: 128-row tiles per 64-channel block
constexpr int kConvIdx = kBM * 9;                  // neighbour entries of a conv tile
constexpr int kWgIdx = kBK * 9;                    // neighbour entries of a 64-token block
__host__ __device__ constexpr int wgrad_a_stages(int bn) { return bn == 256 ? 8 : 4; }  // A stages in TMEM
constexpr int kGatherKb = 2;                       // gather conv: K-blocks (of 64) per pipeline stage
constexpr int kTmemAStageCols = kBK / 2;           // 64 bf16 per row = 32 TMEM columns

struct __align__(16) TcBarriers {
  uint32_t zero16[32];                             // 128 zero bytes (row source for missing neighbours)
  uint64_t afull[kMaxStages], aempty[kMaxStages];  // A stages
  uint64_t bfull[kMaxStages], bempty[kMaxStages];  // B stages
  uint64_t ifull[kMaxStages], iempty[kMaxStages];  // neighbour-row slots (and their halos, weight gradient)
  uint64_t hfull[2], hempty[2];                    // conv halo buffers
  uint64_t tfull[2], tempty[2];                    // TMEM accumulators
  uint64_t done;                                   // final MMA drain before TMEM is released
  uint32_t tmem_base;
  int abort_flag;
};

struct TcConvParams {
  CUtensorMap tmap_a;  // gather: halo boxes {64, 64}; dense: A tile {64, 128}
  CUtensorMap tmap_b;
  CUtensorMap tmap_out;  // out_tma: out [out_rows][N] (row stride ldo), box {64, 32}
  const __nv_bfloat16* A;
  const int32_t* nbr;
  const int32_t* row_lo;
  const int32_t* row_hi;
  const float* bias;
  const __nv_bfloat16* residual;
  __nv_bfloat16* out;
  int* status;
  unsigned long long timeout_ns;
  int lda, a_rows, taps, Kc;
  int M, a_abs, nbr_abs, out_abs, N;
  int gelu, ldo, out_rows, stages_a, stages_b;
  int out_tma;  // 1: the epilogue writes out with TMA stores; 2: adds into out (residual == out) with TMA reduce-adds
  int dense_pair_ring;  // dense, B not resident: A and B stage s on one barrier pair (stages_a == stages_b)
};

struct TcWgradParams {
  CUtensorMap tmap_x;   // X [n][Cin], halo window boxes {64, 128}
  CUtensorMap tmap_dy;  // dY [n][Cout], box {64, 64}
  CUtensorMap tmap_part;  // part_tma: partial [splits * rows_pad][Cout] fp32, box {32, 32}
  const __nv_bfloat16* X;
  const int32_t* nbr;
  float* partial;
  int* status;
  unsigned long long timeout_ns;
  int n, Cin, Cout, splits, rows_pad, stages_a, stages_b;
  int part_tma;  // the last unit of a CTA writes its partial rows with TMA stores
};

__host__ __device__ constexpr int tmem_cols_for(int bn) {
  return (2 * bn) <= 32 ? 32 : (2 * bn) <= 64 ? 64 : (2 * bn) <= 128 ? 128 : (2 * bn) <= 256 ? 256 : 512;
}

// ---------------------------------------------------------------------------- shared memory layout
struct Carve {
  uint8_t* a;      // A ring
  uint8_t* b;      // B ring
  uint8_t* epi;    // dense epilogue staging: 2 boxes of 32 rows x 128 bytes per epilogue warp
  uint8_t* halo;   // conv: 2 halo buffers; weight gradient: 2 slots x 2 halos
  int32_t* idx;    // 2 neighbour-row slots
  float* bias;     // conv: each epilogue warp's copy of the tile's bias columns
  TcBarriers* bar;
};

struct Geometry {
  size_t a_bytes, b_bytes, halo_bytes, idx_bytes, epi_bytes, bias_bytes;
};

__host__ __device__ constexpr size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// a_in_tmem (the gather path): the gathered A stages live in tensor memory, so no shared A
// ring, but two halo buffers and two index slots.  Dense path: an A ring by TMA, no halo.
// epi_stage: the epilogue's staging boxes (TMA stores).
constexpr uint32_t kEpiBoxBytes = 32 * 128;  // 32 rows x 64 bf16 columns
// The epilogue reads the bias from shared memory: at full shared-memory use almost none is
// left as L1, so per-column loads from global memory would wait on L2 with the MMAs stalled.
constexpr int kEpiBiasCols = 256;  // bias columns an epilogue warp holds (the widest tile)
__host__ __device__ inline Geometry conv_geometry(int bn, int sa, int sb, bool a_in_tmem, bool epi_stage, bool bias) {
  return {a_in_tmem ? (size_t)0 : (size_t)sa * kABytes, (size_t)sb * bn * kBK * 2,
          a_in_tmem ? (size_t)2 * kConvHaloRows * 128 : (size_t)0,
          a_in_tmem ? round_up((size_t)2 * kConvIdx * 4, 16) : (size_t)0,
          epi_stage ? (size_t)kEpiWarps * 2 * kEpiBoxBytes : (size_t)0,
          bias ? (size_t)kEpiWarps * kEpiBiasCols * 4 : (size_t)0};
}

// Tensor-memory plan of the conv kernel: accumulator buffers first, then the A stages.
__host__ __device__ constexpr int conv_acc_buffers(int bn, bool a_in_tmem) { return (a_in_tmem && bn == 256) ? 1 : 2; }
__host__ __device__ constexpr uint32_t pow2_cols(uint32_t c) {
  return c <= 32 ? 32 : c <= 64 ? 64 : c <= 128 ? 128 : c <= 256 ? 256 : 512;
}
__host__ __device__ constexpr uint32_t conv_tmem_cols(int bn, bool a_in_tmem, int a_stages) {
  return pow2_cols((uint32_t)(conv_acc_buffers(bn, a_in_tmem) * bn) +
                   (a_in_tmem ? (uint32_t)(a_stages * kGatherKb * kTmemAStageCols) : 0u));
}
// Gather conv: as many stages (kGatherKb K-blocks of A each) in tensor memory as fit next
// to the accumulators, at most kMaxStages.
__host__ __device__ constexpr int conv_tmem_a_stages(int bn) {
  return (512 - conv_acc_buffers(bn, true) * bn) / (int)(kGatherKb * kTmemAStageCols) >= kMaxStages
             ? kMaxStages
             : (512 - conv_acc_buffers(bn, true) * bn) / (int)(kGatherKb * kTmemAStageCols);
}

// Weight gradient: A lives in tensor memory; wgrad_slots(bn) slots of (index entries, halo).
// A dY stage is bn columns of one 64-token block, or on a CTA pair half of them for two blocks:
// the same bytes.
__host__ __device__ inline Geometry wgrad_geometry(int bn, int sb, bool pair = false) {
  return {(size_t)0, (size_t)sb * bn * kBK * 2, (size_t)wgrad_slots(bn, pair) * kWgHaloRows * 128,
          round_up((size_t)wgrad_slots(bn, pair) * kWgIdx * 4, 16)};
}
__host__ __device__ constexpr int wgrad_acc_buffers(int bn) { return bn == 256 ? 1 : 2; }
__host__ __device__ constexpr uint32_t wgrad_tmem_cols(int bn) {
  return pow2_cols((uint32_t)(wgrad_acc_buffers(bn) * bn + wgrad_a_stages(bn) * kTmemAStageCols));
}

__host__ __device__ inline size_t smem_total(const Geometry& g) {
  return 1024 + g.a_bytes + g.b_bytes + g.epi_bytes + g.halo_bytes + g.idx_bytes + g.bias_bytes + sizeof(TcBarriers);
}

__device__ __forceinline__ Carve carve(uint8_t* smem_raw, const Geometry& g) {
  const uint32_t base = smem_u32(smem_raw);
  const uint32_t pad = ((base + 1023u) & ~1023u) - base;
  Carve c;
  c.a = smem_raw + pad;
  c.b = c.a + g.a_bytes;
  c.epi = c.b + g.b_bytes;  // 1024-aligned: the A and B stages are multiples of 1 KB
  c.halo = c.epi + g.epi_bytes;
  c.idx = reinterpret_cast<int32_t*>(c.halo + g.halo_bytes);
  c.bias = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(c.idx) + g.idx_bytes);
  c.bar = reinterpret_cast<TcBarriers*>(reinterpret_cast<uint8_t*>(c.bias) + g.bias_bytes);
  return c;
}

// nslots neighbour-row slots with the given arrival counts; everything else fixed.
__device__ __forceinline__ void init_barriers(TcBarriers* b, int sa, int sb, uint32_t afull_count, int nslots,
                                              uint32_t ifull_count, uint32_t iempty_count,
                                              uint32_t tempty_count = kEpiWarps) {
  for (int i = 0; i < 32; ++i) b->zero16[i] = 0u;
  for (int i = 0; i < nslots; ++i) {
    mbar_init(&b->ifull[i], ifull_count);
    mbar_init(&b->iempty[i], iempty_count);
  }
  for (int s = 0; s < sa; ++s) {
    mbar_init(&b->afull[s], afull_count);
    mbar_init(&b->aempty[s], 1);
  }
  for (int s = 0; s < sb; ++s) {
    mbar_init(&b->bfull[s], 1);
    mbar_init(&b->bempty[s], 1);
  }
  for (int i = 0; i < 2; ++i) {
    mbar_init(&b->hfull[i], 1);
    mbar_init(&b->hempty[i], kProdWarps);
    mbar_init(&b->tfull[i], 1);
    mbar_init(&b->tempty[i], tempty_count);
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

// Phase bookkeeping of a ring slot used for the it-th time.
__device__ __forceinline__ uint32_t ring_parity(uint32_t it, int depth) { return (it / (uint32_t)depth) & 1u; }

// After an abort: wait (bounded, ignoring the abort flag) for the last `count`
// arms of a TMA-fed ring, so that no copy lands after the CTA exits.
__device__ __forceinline__ void drain_ring(uint64_t* full, uint32_t issued, int depth, int* err, uint64_t timeout_ns) {
  if ((threadIdx.x & 31) == 0) {
    volatile int never = 0;
    const uint32_t lo = issued >= (uint32_t)depth ? issued - depth : 0u;
    for (uint32_t q = lo; q < issued; ++q) mbar_wait(&full[q % depth], ring_parity(q, depth), &never, err, timeout_ns);
  }
  __syncwarp();
}

// A warp copies `count` neighbour-table entries (int32) from global src to shared dst and
// accounts for them on `bar`, whose expected arrival count includes all 32 lanes plus one
// expect_tx arrival by lane 0.  With bulk_ok (src 16-byte aligned) the 16-byte-aligned
// prefix goes as one bulk copy on the TMA engine and at most 3 trailing entries by 4-byte
// cp.async; otherwise every entry by 4-byte cp.async.  extra_tx: bytes of other TMA copies
// that lane 0 issues on the same barrier phase (they are declared in the same arrival).
__device__ __forceinline__ void copy_index_entries(uint32_t dst, const int32_t* src, int count, bool bulk_ok,
                                                   uint64_t* bar, uint32_t extra_tx) {
  const int lane = threadIdx.x & 31;
  const int pre = bulk_ok ? (count & ~3) : 0;  // entries covered by the bulk copy (16-byte multiple)
  for (int e = pre + lane; e < count; e += 32) cp_async_4(dst + 4u * e, src + e, 4u);
  cp_async_arrive_noinc(bar);
  if (lane == 0) {
    mbar_arrive_expect_tx(bar, (uint32_t)pre * 4u + extra_tx);
    if (pre > 0) bulk_copy_g2s(dst, src, (uint32_t)pre * 4u, bar);
  }
}

__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ __forceinline__ uint4 ldg_16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Shared-memory descriptor geometry for the MMA issuer.
struct MmaCfg {
  uint32_t idesc;
  uint32_t a_lbo, a_sbo, a_step;  // a_step / b_step: start-address advance per K=16 step
  uint32_t b_lbo, b_sbo, b_step;
};

// Issuer state: descriptors of stage 0 and the per-stage / per-K=16 advances of their
// start-address field (16-byte units), plus ring positions and phases.  The issuing
// thread is on the critical path of the tensor pipe (an MMA of 128x256x16 takes
// ~130 cycles), so its loop avoids divisions and rebuilding descriptors: stage
// indices advance by increment and descriptors by 32-bit adds (the start-address
// field is 14 bits of a 16-byte-granular shared address, so an add never carries
// out of it).
struct MmaIssuer {
  uint32_t a_tmem0;  // A in tensor memory: column address of A stage 0
  uint64_t a_desc0, b_desc0;
  uint32_t a_stage16, b_stage16, a_k16, b_k16;
  uint32_t idesc;
  int SA, SB;
  int sa, sb;
  uint32_t pa, pb;
};

__device__ __forceinline__ MmaIssuer make_issuer(const Carve& sm, uint32_t b_stage_bytes, int SA, int SB,
                                                 const MmaCfg& c) {
  MmaIssuer m;
  m.a_tmem0 = 0;
  m.a_desc0 = smem_desc_sw128(smem_u32(sm.a), c.a_lbo, c.a_sbo);
  m.b_desc0 = smem_desc_sw128(smem_u32(sm.b), c.b_lbo, c.b_sbo);
  m.a_stage16 = (uint32_t)kABytes >> 4;
  m.b_stage16 = b_stage_bytes >> 4;
  m.a_k16 = c.a_step >> 4;
  m.b_k16 = c.b_step >> 4;
  m.idesc = c.idesc;
  m.SA = SA;
  m.SB = SB;
  m.sa = m.sb = 0;
  m.pa = m.pb = 0;
  return m;
}

// One thread issues the MMAs of one tile (num_kb K-blocks) into accumulator d.
// A_TMEM: A stages in tensor memory (written by the builder warps with tcgen05.st).
// GROUP: stages whose barriers are checked back to back before their MMAs are issued.
// The first shared-memory access (an mbarrier wait) after a batch of MMAs stalls until
// those MMAs have read their operands, so checking two stages per batch halves that cost
// when MMAs are short (N = 64); GROUP = 1 keeps the deepest pipelining for long MMAs.
// PAIR: M = 256 MMAs of a CTA pair (issued by rank 0; the stage barriers count both
// CTAs' producers and the commits arrive in both CTAs).
template <bool A_TMEM, int GROUP, bool PAIR = false>
__device__ __forceinline__ bool mma_tile(TcBarriers* bar, MmaIssuer& m, int num_kb, uint32_t d,
                                         volatile int* abort_flag, int* err, uint64_t timeout_ns) {
  for (int kb = 0; kb < num_kb; kb += GROUP) {
    const int cnt = min(GROUP, num_kb - kb);
    int sa[GROUP], sb[GROUP];
    {
      int a = m.sa, b = m.sb;
      uint32_t pa = m.pa, pb = m.pb;
#pragma unroll
      for (int g = 0; g < GROUP; ++g) {
        if (g < cnt) {
          if (!mbar_wait(&bar->afull[a], pa, abort_flag, err, timeout_ns)) return false;
          if (!mbar_wait(&bar->bfull[b], pb, abort_flag, err, timeout_ns)) return false;
        }
        sa[g] = a;
        sb[g] = b;
        if (++a == m.SA) a = 0, pa ^= 1u;
        if (++b == m.SB) b = 0, pb ^= 1u;
      }
    }
    if constexpr (A_TMEM) tc_fence_after();  // the A stages were written to tensor memory by other threads
#pragma unroll
    for (int g = 0; g < GROUP; ++g) {
      if (g >= cnt) break;
      const uint64_t bd = m.b_desc0 + (uint64_t)((uint32_t)sb[g] * m.b_stage16);
      if constexpr (A_TMEM) {
        const uint32_t at = m.a_tmem0 + (uint32_t)sa[g] * kTmemAStageCols;
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          if constexpr (PAIR)
            tc_mma_bf16_ts_pair(d, at + k * 8, bd + (uint64_t)(k * m.b_k16), m.idesc, (kb + g) | k ? 1u : 0u);
          else
            tc_mma_bf16_ts(d, at + k * 8, bd + (uint64_t)(k * m.b_k16), m.idesc, (kb + g) | k ? 1u : 0u);
        }
      } else {
        const uint64_t ad = m.a_desc0 + (uint64_t)((uint32_t)sa[g] * m.a_stage16);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          if constexpr (PAIR)
            tc_mma_bf16_pair(d, ad + (uint64_t)(k * m.a_k16), bd + (uint64_t)(k * m.b_k16), m.idesc,
                             (kb + g) | k ? 1u : 0u);
          else
            tc_mma_bf16(d, ad + (uint64_t)(k * m.a_k16), bd + (uint64_t)(k * m.b_k16), m.idesc,
                        (kb + g) | k ? 1u : 0u);
        }
      }
      if constexpr (PAIR) {
        tc_commit_pair(&bar->aempty[sa[g]]);
        tc_commit_pair(&bar->bempty[sb[g]]);
      } else {
        tc_commit(&bar->aempty[sa[g]]);
        tc_commit(&bar->bempty[sb[g]]);
      }
      if (++m.sa == m.SA) {
        m.sa = 0;
        m.pa ^= 1u;
      }
      if (++m.sb == m.SB) {
        m.sb = 0;
        m.pb ^= 1u;
      }
    }
  }
  return true;
}

// Gather conv: A stage s (tensor memory) and B stage s (shared memory) advance together on
// one full / empty barrier pair (full counts the builder warps and the weight loader), so a
// stage costs the issuing thread one wait and one commit.  The tensor pipe queues only a
// few MMAs, so every cycle the issuing thread spends between MMA bursts is a cycle the pipe
// may sit idle.  GROUP: stages whose barriers are checked before their MMAs are issued.
// A stage holds KBS K-blocks (the last stage of a tile fewer when num_kb is not a
// multiple): A at 32-column steps in tensor memory, B at b_stage16 / KBS steps.
// A_TMEM = false: dense GEMM, A stage s in shared memory as well (one K-block per stage).
template <int GROUP, bool PAIR, int KBS = kGatherKb, bool A_TMEM = true, bool F8 = false>
__device__ __forceinline__ bool mma_tile_unified(TcBarriers* bar, MmaIssuer& m, int num_kb, uint32_t d,
                                                 volatile int* abort_flag, int* err, uint64_t timeout_ns) {
  static_assert(A_TMEM || KBS == 1, "dense stages hold one K-block");
  const int nst = (num_kb + KBS - 1) / KBS;
  const uint32_t b_kb16 = m.b_stage16 / KBS;
  for (int q = 0; q < nst; q += GROUP) {
    const int cnt = min(GROUP, nst - q);
    {
      int st = m.sa;
      uint32_t ps = m.pa;
#pragma unroll
      for (int g = 0; g < GROUP; ++g) {
        if (g < cnt && !mbar_wait(&bar->afull[st], ps, abort_flag, err, timeout_ns)) return false;
        if (++st == m.SA) st = 0, ps ^= 1u;
      }
    }
    if constexpr (A_TMEM) tc_fence_after();  // the A stages were written to tensor memory by other threads
#pragma unroll
    for (int g = 0; g < GROUP; ++g) {
      if (g >= cnt) break;
      const int kb0 = (q + g) * KBS;
#pragma unroll
      for (int h = 0; h < KBS; ++h) {
        if (kb0 + h >= num_kb) break;
        const uint64_t bd = m.b_desc0 + (uint64_t)((uint32_t)m.sa * m.b_stage16 + (uint32_t)h * b_kb16);
        if constexpr (A_TMEM) {
          const uint32_t at = m.a_tmem0 + (uint32_t)(m.sa * KBS + h) * kTmemAStageCols;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            // F8: the same 32 bytes per row and step hold 32 e4m3 values (K = 32 per MMA)
            if constexpr (PAIR && F8)
              tc_mma_f8_ts_pair(d, at + k * 8, bd + (uint64_t)(k * m.b_k16), m.idesc, (kb0 + h) | k ? 1u : 0u);
            else if constexpr (F8)
              tc_mma_f8_ts(d, at + k * 8, bd + (uint64_t)(k * m.b_k16), m.idesc, (kb0 + h) | k ? 1u : 0u);
            else if constexpr (PAIR)
              tc_mma_bf16_ts_pair(d, at + k * 8, bd + (uint64_t)(k * m.b_k16), m.idesc, (kb0 + h) | k ? 1u : 0u);
            else
              tc_mma_bf16_ts(d, at + k * 8, bd + (uint64_t)(k * m.b_k16), m.idesc, (kb0 + h) | k ? 1u : 0u);
          }
        } else {
          const uint64_t ad = m.a_desc0 + (uint64_t)((uint32_t)m.sa * m.a_stage16);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            if constexpr (PAIR)
              tc_mma_bf16_pair(d, ad + (uint64_t)(k * m.a_k16), bd + (uint64_t)(k * m.b_k16), m.idesc,
                               (kb0 + h) | k ? 1u : 0u);
            else
              tc_mma_bf16(d, ad + (uint64_t)(k * m.a_k16), bd + (uint64_t)(k * m.b_k16), m.idesc,
                          (kb0 + h) | k ? 1u : 0u);
          }
        }
      }
      if constexpr (PAIR) {
        tc_commit_pair(&bar->aempty[m.sa]);
      } else {
        tc_commit(&bar->aempty[m.sa]);
      }
      if (++m.sa == m.SA) m.sa = 0, m.pa ^= 1u;
    }
  }
  return true;
}

// Dense GEMM whose whole K extent of B fits in the B stages (num_kb <= SB): a run of
// consecutive tiles of this CTA with the same output columns loads B once and keeps it
// in shared memory.  b_load: first tile of a run (wait for the B stages to fill);
// b_last: last tile of a run (release the B stages after its MMAs).  A streams per tile.
template <bool PAIR = false>
__device__ __forceinline__ bool mma_tile_resident_b(TcBarriers* bar, MmaIssuer& m, int num_kb, uint32_t d,
                                                    bool b_load, bool b_last, volatile int* abort_flag, int* err,
                                                    uint64_t timeout_ns) {
  int b = m.sb;
  uint32_t pb = m.pb;
  for (int kb = 0; kb < num_kb; ++kb) {
    if (!mbar_wait(&bar->afull[m.sa], m.pa, abort_flag, err, timeout_ns)) return false;
    if (b_load && !mbar_wait(&bar->bfull[b], pb, abort_flag, err, timeout_ns)) return false;
    const uint64_t ad = m.a_desc0 + (uint64_t)((uint32_t)m.sa * m.a_stage16);
    const uint64_t bd = m.b_desc0 + (uint64_t)((uint32_t)b * m.b_stage16);
#pragma unroll
    for (int k = 0; k < kBK / 16; ++k) {
      if constexpr (PAIR)
        tc_mma_bf16_pair(d, ad + (uint64_t)(k * m.a_k16), bd + (uint64_t)(k * m.b_k16), m.idesc, kb | k ? 1u : 0u);
      else
        tc_mma_bf16(d, ad + (uint64_t)(k * m.a_k16), bd + (uint64_t)(k * m.b_k16), m.idesc, kb | k ? 1u : 0u);
    }
    if constexpr (PAIR) {
      tc_commit_pair(&bar->aempty[m.sa]);
      if (b_last) tc_commit_pair(&bar->bempty[b]);
    } else {
      tc_commit(&bar->aempty[m.sa]);
      if (b_last) tc_commit(&bar->bempty[b]);
    }
    if (++m.sa == m.SA) {
      m.sa = 0;
      m.pa ^= 1u;
    }
    if (++b == m.SB) b = 0, pb ^= 1u;
  }
  if (b_last) m.sb = b, m.pb = pb;
  return true;
}

// PAIR: the commit always goes out (to both CTAs), so the other CTA's wait on its own
// copy of `done` ends even when no tile was issued.
template <bool PAIR = false>
__device__ __forceinline__ void mma_drain(TcBarriers* bar, bool issued, int* err, uint64_t timeout_ns) {
  if (issued || PAIR) {
    volatile int never = 0;
    if constexpr (PAIR) {
      tc_commit_pair(&bar->done);
    } else {
      tc_commit(&bar->done);
    }
    mbar_wait(&bar->done, 0, &never, err, timeout_ns);
  }
}

// Epilogue of one output tile row: the fp32 accumulator row at TMEM address acc (this
// warp's lane quarter, column 0 of the tile) + bias, GELU, residual -> bf16 row orow,
// columns n0 .. n0 + BN - 1.  Two 32-column loads are in flight per wait.
// GELU in its erf form, x * Phi(x) = x/2 * (1 + erf(x / sqrt 2)), with erf from formula
// 7.1.28 of Abramowitz and Stegun, Handbook of Mathematical Functions (absolute error at
// most 3e-7; in fp32 the GELU stays within ~1e-6 |x| of the exact value, far below bf16
// rounding):
//   erf(z) = 1 - (1 + a1 z + a2 z^2 + a3 z^3 + a4 z^4 + a5 z^5 + a6 z^6)^(-16),  z >= 0,
// odd in z.  It costs one reciprocal, six multiply-adds and four squarings: one special-
// function operation per element instead of the two (reciprocal and exponential) of the
// shorter formula 7.1.26, which made the special-function unit the epilogue's bottleneck
// while the next tile's MMAs wait for the single accumulator.
__device__ __forceinline__ float gelu_erf(float x) {
  const float z = fabsf(x) * 0.70710678118654752f;
  const float p = fmaf(z, fmaf(z, fmaf(z, fmaf(z, fmaf(z, fmaf(z, 0.0000430638f, 0.0002765672f), 0.0001520143f),
                                                 0.0092705272f), 0.0422820123f), 0.0705230784f), 1.0f);
  const float r = __fdividef(1.0f, p);
  const float r2 = r * r, r4 = r2 * r2, r8 = r4 * r4;
  const float erf_abs = 1.0f - r8 * r8;
  return 0.5f * x * (1.0f + copysignf(erf_abs, x));
}

// 32 accumulator columns (raw fp32 bits) + bias[col ..], then GELU when asked.  bias_s: the
// shared-memory address of bias[col] (16-byte aligned), or 0 to read p.bias from global memory.
__device__ __forceinline__ void epi_bias_gelu(const TcConvParams& p, const uint32_t (&v)[32], float (&f)[32], int col,
                                              uint32_t bias_s = 0u) {
#pragma unroll
  for (int q = 0; q < 32; ++q) f[q] = __uint_as_float(v[q]);
  if (bias_s) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint4 b = ld_shared_16(bias_s + 16u * q);  // the same address in every lane: a broadcast
      f[4 * q] += __uint_as_float(b.x), f[4 * q + 1] += __uint_as_float(b.y);
      f[4 * q + 2] += __uint_as_float(b.z), f[4 * q + 3] += __uint_as_float(b.w);
    }
  } else if (p.bias) {
    if ((reinterpret_cast<uintptr_t>(p.bias) & 15u) == 0) {  // col is a multiple of 32
      const float4* b4 = reinterpret_cast<const float4*>(p.bias + col);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 b = __ldg(b4 + q);
        f[4 * q] += b.x, f[4 * q + 1] += b.y, f[4 * q + 2] += b.z, f[4 * q + 3] += b.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 32; ++q) f[q] += __ldg(p.bias + col + q);
    }
  }
  if (p.gelu) {
#pragma unroll
    for (int q = 0; q < 32; ++q) f[q] = gelu_erf(f[q]);
  }
}

template <int BN>
__device__ __forceinline__ void epilogue_rows(const TcConvParams& p, uint32_t acc, bool valid, size_t orow, int n0,
                                              uint32_t bias_s = 0u) {
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 64) {
    uint32_t v[2][32];
    tmem_ld_32x32b_x32(acc + c0, v[0]);
    tmem_ld_32x32b_x32(acc + c0 + 32, v[1]);
    tmem_ld_wait();
    if (!valid) continue;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int c = c0 + 32 * hh;
      float f[32];
      epi_bias_gelu(p, v[hh], f, n0 + c, bias_s ? bias_s + 4u * (uint32_t)c : 0u);
      if (p.residual) {
        const uint4* rp = reinterpret_cast<const uint4*>(p.residual + orow * p.ldo + n0 + c);
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
      uint32_t packed[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(f[2 * q], f[2 * q + 1]);
        packed[q] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      __nv_bfloat16* orow_p = p.out + orow * p.ldo + n0 + c;
      if ((reinterpret_cast<uintptr_t>(orow_p) & 31u) == 0) {  // two 32-byte stores per 32 columns
        st_global_32(orow_p, packed);
        st_global_32(orow_p + 16, packed + 8);
      } else {
        uint4* op = reinterpret_cast<uint4*>(orow_p);
#pragma unroll
        for (int q = 0; q < 4; ++q) op[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
      }
    }
  }
}

// Epilogue through the TMA engine: this warp's 32 tile rows (+ bias, GELU) are rounded
// to bf16 and staged 64 columns at a time in a 128-byte-swizzled box of shared memory
// (two boxes per warp, alternating), and each box goes to out[orow0 .. orow0 + 31]
// [n0 + c0 ..] as one tiled bulk store (REDUCE: a bulk reduce-add into out, which holds
// the residual), so the output leaves the SM in whole lines and a residual never enters
// it.  release() runs once the last accumulator columns are in registers, so the MMAs of
// the next tile may start while the last boxes are still being written.  All 32 rows must
// be rows of out that this tile owns.  q counts the boxes this warp has issued.
template <int BN, bool REDUCE, typename Release>
__device__ __forceinline__ void epilogue_tma(const TcConvParams& p, uint32_t acc, uint32_t boxes, uint32_t& q,
                                             int orow0, int n0, uint32_t bias_s, Release release) {
  const int lane = threadIdx.x & 31;
  const uint32_t row_off = (uint32_t)lane * 128u;
  const uint32_t sw = (uint32_t)(lane & 7);
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 64, ++q) {
    uint32_t v[2][32];
    tmem_ld_32x32b_x32(acc + c0, v[0]);
    tmem_ld_32x32b_x32(acc + c0 + 32, v[1]);
    const uint32_t box = boxes + (q & 1u) * kEpiBoxBytes;
    if (lane == 0) bulk_wait_group_read<1>();  // the copy issued from this box two boxes ago has read it
    __syncwarp();
    tmem_ld_wait();
    if (c0 + 64 >= BN) release();
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float f[32];
      epi_bias_gelu(p, v[hh], f, n0 + c0 + 32 * hh, bias_s ? bias_s + 4u * (uint32_t)(c0 + 32 * hh) : 0u);
      uint32_t packed[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
        packed[e] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      // 16-byte chunk k of the row lands at chunk k ^ (row & 7) (the map's 128-byte swizzle)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t kk = (uint32_t)(4 * hh + k);
        st_shared_16(box + row_off + ((kk ^ sw) << 4), packed[4 * k], packed[4 * k + 1], packed[4 * k + 2],
                     packed[4 * k + 3]);
      }
    }
    fence_proxy_async_smem();  // make the generic-proxy stores visible to the TMA engine
    __syncwarp();
    if (lane == 0) {
      if constexpr (REDUCE)
        tma_reduce_add_2d(&p.tmap_out, box, n0 + c0, orow0);
      else
        tma_store_2d(&p.tmap_out, box, n0 + c0, orow0);
      bulk_commit_group();
    }
  }
}

// ============================================================================ conv / dense GEMM
// MIRROR: gather through column 8-j (data gradient); it always pairs with an
// MN-major weight operand.
// PAIR: a cluster of two CTAs computes 256-row tiles with M = 256 MMAs: each CTA gathers
// (or loads) its own 128 rows of A and holds their accumulator, loads half of the tile's
// B columns, and CTA rank 0 issues the MMAs for both.  Every SM then streams half of B
// per 128 output rows.  Barriers that count both CTAs' producers (A and B stages,
// accumulator release) live in rank 0; the MMA commits arrive in both CTAs.
template <int BN, bool MIRROR, bool PAIR, bool F8 = false>
__global__ void __launch_bounds__(kThreads, 1) tc_conv_kernel(const __grid_constant__ TcConvParams p) {
  static_assert(!PAIR || BN == 256, "CTA pairs run 256-column tiles");
  static_assert(!F8 || !MIRROR, "e4m3 operands: forward gather with a K-major weight only");
  extern __shared__ uint8_t smem_raw[];
  const bool gather = p.nbr != nullptr;  // gathered A lives in tensor memory
  const int SA = p.stages_a, SB = p.stages_b;
  const bool tma_epi = p.out_tma != 0;
  constexpr int kBCols = PAIR ? BN / 2 : BN;  // B columns this CTA loads per stage
  constexpr int kRows = PAIR ? 2 * kBM : kBM;  // output rows per tile
  // gather: a B stage holds kGatherKb K-blocks (geometry counts them as wider stages)
  const Geometry geo = conv_geometry(gather ? kBCols * kGatherKb : kBCols, SA, SB, gather, tma_epi, p.bias != nullptr);
  const Carve sm = carve(smem_raw, geo);
  TcBarriers* bar = sm.bar;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* err = p.status;
  constexpr uint32_t kBBytes = kBCols * kBK * 2;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;  // first tile of this CTA (pair)
  const int units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;    // tile stride
  const int row_off = (int)rank * kBM;                                  // this CTA's rows within a tile
  // rank 0's copy of a barrier (PAIR)
  auto lead = [](uint64_t* b) -> uint32_t { return mapa_shared(smem_u32(b), 0u); };
  const uint32_t tmem_cols = conv_tmem_cols(BN, gather, SA);
  const int n_acc = conv_acc_buffers(BN, gather);
  const uint32_t a_tmem_col = (uint32_t)(n_acc * BN);  // first column of the A stages
  constexpr uint32_t kHaloBufBytes = kConvHaloRows * 128;

  if (threadIdx.x == 0) {
    // afull: one builder group per A stage; ifull: the loader lanes' 32 cp.async arrivals + lane 0's expect_tx
    // gather: afull / aempty serve A and B stage s together (SA == SB); afull counts the
    // builder warps (of both CTAs of a pair) and the weight loader's expect_tx arrival
    // dense with dense_pair_ring: afull counts the A and the B loader's expect_tx arrivals
    init_barriers(bar, SA, SB, gather ? (PAIR ? kProdWarps : kProdWarps / 2) + 1 : (p.dense_pair_ring ? 2 : 1), 2,
                  33, kProdWarps, PAIR ? 2 * kEpiWarps : kEpiWarps);
    prefetch_tmap(&p.tmap_a);
    prefetch_tmap(&p.tmap_b);
  }
  if (warp == kMmaWarp) {
    if constexpr (PAIR) {
      tmem_alloc_pair(&bar->tmem_base, tmem_cols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&bar->tmem_base, tmem_cols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) {
    cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA arrival
  } else {
    __syncthreads();
  }
  tc_fence_after();
  pdl_wait();  // inputs, outputs and the row bounds may come from the kernel before this one
  pdl_trigger();
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
  const int m_tiles = (M + kRows - 1) / kRows;
  const int n_tiles = p.N / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int kb_per_tap = p.Kc / kBK;
  const int taps = p.taps;
  const int num_kb = taps * kb_per_tap;
  const int nbr_base = p.nbr_abs ? lo : 0;
  // dense GEMM with all of K in the B stages: B stays resident across this CTA's tiles
  // with the same output columns (with the stride order, every tile when gridDim.x is a
  // multiple of the column-tile count), so per tile only A crosses into the SM
  const bool res_b = !gather && num_kb <= SB;

  const uint32_t tmem_base = bar->tmem_base;
  volatile int* abort_flag = &bar->abort_flag;

  if (warp == kHaloWarp) {
    // ------------------------------------------------------------ index / halo (or dense A) loader
    if (gather) {
      // The tile's 128 x 9 neighbour entries arrive by cp.async on ifull[slot]; the
      // halo window (A rows m0 - 32 .. m0 + 159) needs none of them, so its TMA boxes
      // are issued right away and both loads are in flight together.
      uint32_t ti = 0, hi = 0, ni = 0;  // ni: index loads issued
      bool aborted = false;
      for (int tile = unit0; tile < num_tiles && !aborted; tile += units, ++ti) {
        const int m0 = (tile / n_tiles) * kRows + row_off;
        const int slot = ti & 1;
        if (!warp_wait(&bar->iempty[slot], ring_parity(ti, 2) ^ 1u, abort_flag, err, p.timeout_ns)) {
          aborted = true;
          break;
        }
        const int32_t* src = p.nbr + (size_t)(nbr_base + m0) * 9;
        const int lim = max(0, min(M - m0, kBM)) * 9;  // PAIR: rank 1's rows may all lie past M
        copy_index_entries(smem_u32(sm.idx + slot * kConvIdx), src, lim,
                           ((reinterpret_cast<uintptr_t>(src) & 15u) == 0), &bar->ifull[slot], 0u);
        __syncwarp();
        ++ni;
        for (int cb = 0; cb < kb_per_tap; ++cb, ++hi) {
          const int hb = hi & 1;
          if (!warp_wait(&bar->hempty[hb], ring_parity(hi, 2) ^ 1u, abort_flag, err, p.timeout_ns)) {
            aborted = true;
            break;
          }
          if (lane == 0) {
            mbar_arrive_expect_tx(&bar->hfull[hb], kHaloBufBytes);
            const uint32_t hdst = smem_u32(sm.halo + hb * kHaloBufBytes);
#pragma unroll
            for (int q = 0; q < kConvHaloRows / kHaloBox; ++q)
              tma_load_2d(hdst + q * kHaloBox * 128, &p.tmap_a, &bar->hfull[hb], cb * kBK,
                          m0 - kConvPad + q * kHaloBox);
          }
          __syncwarp();
        }
      }
      if (aborted) {
        drain_ring(bar->ifull, ni, 2, err, p.timeout_ns);
        drain_ring(bar->hfull, hi, 2, err, p.timeout_ns);
      }
    } else {
      const int a_base = p.a_abs ? lo : 0;
      uint32_t it = 0;
      bool aborted = false;
      for (int tile = unit0; tile < num_tiles && !aborted; tile += units) {
        const int m0 = (tile / n_tiles) * kRows + row_off;
        for (int cb = 0; cb < kb_per_tap; ++cb, ++it) {
          const int sa = it % SA;
          if (!warp_wait(&bar->aempty[sa], ring_parity(it, SA) ^ 1u, abort_flag, err, p.timeout_ns)) {
            aborted = true;
            break;
          }
          if (lane == 0) {
            const uint32_t dst = smem_u32(sm.a + (size_t)sa * kABytes);
            if constexpr (PAIR) {
              if (leader) mbar_arrive_expect_tx(&bar->afull[sa], 2u * (uint32_t)kABytes);  // both CTAs' rows
              tma_load_2d_pair(dst, &p.tmap_a, lead(&bar->afull[sa]), cb * kBK, a_base + m0);
            } else {
              mbar_arrive_expect_tx(&bar->afull[sa], (uint32_t)kABytes);
              tma_load_2d(dst, &p.tmap_a, &bar->afull[sa], cb * kBK, a_base + m0);
            }
          }
          __syncwarp();
        }
      }
      if (aborted && leader && !p.dense_pair_ring) drain_ring(bar->afull, it, SA, err, p.timeout_ns);
      if (aborted && (p.dense_pair_ring || !leader)) {
        // the full barriers also count the other loader (or live in the other CTA): give this
        // warp's copies in flight time to land instead of waiting on a phase
        if (lane == 0) {
          const uint64_t t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < 200000u) {
          }
        }
        __syncwarp();
      }
    }
  } else if (warp == kBWarp && gather) {
    // ------------------------------------------------------------ weight loader (gather)
    // B slab of K-block kb goes to slot kb % kGatherKb of stage q, on the A stages' barrier
    // pair; the full barrier's expect_tx (rank 0) covers all slabs of the stage (both CTAs)
    uint32_t q0 = 0;
    bool aborted = false;
    for (int tile = unit0; tile < num_tiles && !aborted; tile += units) {
      const int n0 = (tile % n_tiles) * BN;
      const int nb = n0 + (int)rank * kBCols;  // this CTA's B columns
      int kb = 0;
      for (int cb = 0; cb < kb_per_tap && !aborted; ++cb)
        for (int j = 0; j < taps; ++j, ++kb) {
          const uint32_t q = q0 + (uint32_t)(kb / kGatherKb);
          const int half = kb % kGatherKb;
          const int st = q % SB;
          if (half == 0) {
            if (!warp_wait(&bar->aempty[st], ring_parity(q, SB) ^ 1u, abort_flag, err, p.timeout_ns)) {
              aborted = true;
              break;
            }
            if (lane == 0 && leader) {
              const uint32_t slabs = (uint32_t)min(kGatherKb, num_kb - kb);
              mbar_arrive_expect_tx(&bar->afull[st], slabs * kBBytes * (PAIR ? 2u : 1u));
            }
          }
          if (lane == 0) {
            const uint32_t dst = smem_u32(sm.b + ((size_t)st * kGatherKb + half) * kBBytes);
            const uint32_t fb = PAIR ? lead(&bar->afull[st]) : smem_u32(&bar->afull[st]);
            if constexpr (!MIRROR) {
              if constexpr (PAIR)
                tma_load_2d_pair(dst, &p.tmap_b, fb, j * p.Kc + cb * kBK, nb);
              else
                tma_load_2d(dst, &p.tmap_b, &bar->afull[st], j * p.Kc + cb * kBK, nb);
            } else {
#pragma unroll
              for (int g = 0; g < kBCols / 64; ++g) {
                if constexpr (PAIR)
                  tma_load_3d_pair(dst + g * 8192, &p.tmap_b, fb, nb + g * 64, j, cb * kBK);
                else
                  tma_load_3d(dst + g * 8192, &p.tmap_b, &bar->afull[st], nb + g * 64, j, cb * kBK);
              }
            }
          }
          __syncwarp();
        }
      q0 += (uint32_t)((num_kb + kGatherKb - 1) / kGatherKb);
    }
    if (aborted) {
      // the full barriers also count the builders (or live in the other CTA): give this
      // warp's copies in flight time to land instead of waiting on a phase
      if (lane == 0) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000u) {
        }
      }
      __syncwarp();
    }
  } else if (warp == kBWarp) {
    // ------------------------------------------------------------ weight loader (dense)
    uint64_t* const bf = p.dense_pair_ring ? bar->afull : bar->bfull;
    uint64_t* const be = p.dense_pair_ring ? bar->aempty : bar->bempty;
    uint32_t it = 0;
    bool aborted = false;
    int prev_nt = -1;
    for (int tile = unit0; tile < num_tiles && !aborted; tile += units) {
      const int nt = tile % n_tiles;
      if (res_b && nt == prev_nt) continue;  // this run's B is still resident
      prev_nt = nt;
      const int n0 = nt * BN;
      for (int cb = 0; cb < kb_per_tap && !aborted; ++cb)
        for (int j = 0; j < taps; ++j, ++it) {
          const int sb = it % SB;
          if (!warp_wait(&be[sb], ring_parity(it, SB) ^ 1u, abort_flag, err, p.timeout_ns)) {
            aborted = true;
            break;
          }
          if (lane == 0) {
            const uint32_t dst = smem_u32(sm.b + (size_t)sb * kBBytes);
            const int nb = n0 + (int)rank * kBCols;  // this CTA's B columns
            if constexpr (PAIR) {
              if (leader) mbar_arrive_expect_tx(&bf[sb], 2u * kBBytes);  // both halves
              const uint32_t fb = lead(&bf[sb]);
              if constexpr (!MIRROR) {
                tma_load_2d_pair(dst, &p.tmap_b, fb, j * p.Kc + cb * kBK, nb);
              } else {
#pragma unroll
                for (int q = 0; q < kBCols / 64; ++q) tma_load_3d_pair(dst + q * 8192, &p.tmap_b, fb, nb + q * 64, j, cb * kBK);
              }
            } else {
              mbar_arrive_expect_tx(&bf[sb], kBBytes);
              if constexpr (!MIRROR) {
                tma_load_2d(dst, &p.tmap_b, &bf[sb], j * p.Kc + cb * kBK, nb);
              } else {
#pragma unroll
                for (int q = 0; q < kBCols / 64; ++q)
                  tma_load_3d(dst + q * 8192, &p.tmap_b, &bf[sb], nb + q * 64, j, cb * kBK);
              }
            }
          }
          __syncwarp();
        }
    }
    if (aborted) {
      if (!leader || p.dense_pair_ring) {
        // the full barriers live in the other CTA or also count the A loader: give this
        // warp's copies in flight time to land instead of waiting on a phase
        if (lane == 0) {
          const uint64_t t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < 200000u) {
          }
        }
        __syncwarp();
      } else {
        drain_ring(bar->bfull, it, SB, err, p.timeout_ns);
      }
    }
  } else if (warp >= kEpiWarps && warp < kHaloWarp) {
    // ------------------------------------------------------------ A builders
    // Two groups of four warps build alternate K-blocks (group g takes the K-blocks
    // with counter parity g, i.e. A stages g and g+2).  Each thread owns one tile row:
    // warp w may only touch TMEM lanes 32*(w%4) .. +31, so thread (w, lane) copies
    // row 32*(w%4) + lane.  It reads the row's neighbour segment from the halo in
    // shared memory (or, for a neighbour outside the halo window, from global
    // memory) and writes it straight
    // into the tensor-memory A stage with tcgen05.st: no shared-memory stores, no
    // proxy fence, and the MMA reads only B from shared memory.
    if (gather) {
      const int grp = (warp - kEpiWarps) >> 2;  // builder group 0 or 1
      const int quarter = warp & 3;             // TMEM lane quarter of this warp
      const int r = quarter * 32 + lane;        // the tile row this thread writes
      const uint32_t a_lane = tmem_base + ((uint32_t)(quarter * 32) << 16) + a_tmem_col;
      const uint32_t zero_row = smem_u32(bar->zero16);
      // stage q (counted over all tiles) holds K-blocks kGatherKb * (q - q0) .. of the tile
      // that starts at stage q0; builder group q & 1 writes it
      uint32_t ti = 0, hi = 0, q0 = 0;
      bool aborted = false;
      for (int tile = unit0; tile < num_tiles && !aborted; tile += units, ++ti) {
        const int slot = ti & 1;
        int kb = 0;  // K-block within the tile
        if (!warp_wait(&bar->ifull[slot], ring_parity(ti, 2), abort_flag, err, p.timeout_ns)) {
          aborted = true;
          break;
        }
        const int m0 = (tile / n_tiles) * kRows + row_off;
        const bool row_ok = m0 + r < M;
        const int hlo = m0 - kConvPad;  // A row of halo row 0
        const uint32_t sidx_s = smem_u32(sm.idx + slot * kConvIdx);
        for (int cb = 0; cb < kb_per_tap && !aborted; ++cb) {
          const int hb = hi & 1;
          if (!warp_wait(&bar->hfull[hb], ring_parity(hi, 2), abort_flag, err, p.timeout_ns)) {
            aborted = true;
            break;
          }
          const uint32_t halo = smem_u32(sm.halo + hb * kHaloBufBytes);
          for (int j = 0; j < 9; ++j, ++kb) {
            const uint32_t q = q0 + (uint32_t)(kb / kGatherKb);
            if ((int)(q & 1u) != grp) continue;
            const int half = kb % kGatherKb;  // slab of the stage
            const bool stage_done = half == kGatherKb - 1 || kb == num_kb - 1;
            const int jj = MIRROR ? 8 - j : j;
            const int sa = q % SA;
            if (half == 0) {
              if (!warp_wait(&bar->aempty[sa], ring_parity(q, SA) ^ 1u, abort_flag, err, p.timeout_ns)) {
                aborted = true;
                break;
              }
              tc_fence_after();  // the MMAs that read this stage are complete
            }
            // branch-free row selection: halo row, or the zero row for a missing neighbour;
            // rows outside the halo window are read from global memory behind a warp vote
            const int raw = row_ok ? ld_shared_s32(sidx_s + 4u * (uint32_t)(r * 9 + jj)) : -1;
            const int rel = raw - nbr_base;
            const bool bad = (raw >= 0) & ((unsigned)rel >= (unsigned)p.a_rows);
            const int idx = ((raw >= 0) & !bad) ? rel : -1;
            const int h = idx - hlo;
            const bool in_win = (idx >= 0) & ((unsigned)h < (unsigned)kConvHaloRows);
            const uint32_t row = in_win ? halo + (uint32_t)h * 128u : zero_row;
            const int sw = in_win ? (h & 7) : 0;
            uint32_t v[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 q = ld_shared_16(row + ((c ^ sw) << 4));
              v[4 * c] = q.x, v[4 * c + 1] = q.y, v[4 * c + 2] = q.z, v[4 * c + 3] = q.w;
            }
            const bool far = (idx >= 0) & !in_win;
            if (__any_sync(0xffffffffu, far | bad)) {
              if (bad) atomicOr(err, SVCONV_STATUS_BAD_INDEX);
              if (far) {
                const __nv_bfloat16* src = p.A + (size_t)idx * p.lda + cb * kBK;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                  const uint4 q = ldg_16(src + c * 8);
                  v[4 * c] = q.x, v[4 * c + 1] = q.y, v[4 * c + 2] = q.z, v[4 * c + 3] = q.w;
                }
              }
            }
            tmem_st_32x32b_x32(a_lane + (uint32_t)(sa * kGatherKb + half) * kTmemAStageCols, v);
            if (stage_done) {
              tmem_st_wait();
              tc_fence_before();
              if (PAIR && !leader) {
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(lead(&bar->afull[sa]));
              } else {
                warp_arrive(&bar->afull[sa]);
              }
            }
          }
          if (!aborted) {
            warp_arrive(&bar->hempty[hb]);
            ++hi;
          }
        }
        q0 += (uint32_t)((num_kb + kGatherKb - 1) / kGatherKb);
        if (!aborted) warp_arrive(&bar->iempty[slot]);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      MmaCfg c;
      c.idesc = F8 ? idesc_e4m3_f32(kRows, BN, 0, 0) : idesc_bf16_f32(kRows, BN, 0, MIRROR ? 1 : 0);
      c.a_lbo = 16, c.a_sbo = 1024, c.a_step = 32;  // smem A (dense): K-major, 128-byte rows
      if (MIRROR) {
        c.b_lbo = 8192, c.b_sbo = 1024, c.b_step = 2048;  // B: MN-major, 64-wide MN groups 8 KB apart
      } else {
        c.b_lbo = 16, c.b_sbo = 1024, c.b_step = 32;
      }
      MmaIssuer mi = make_issuer(sm, gather ? kGatherKb * kBBytes : kBBytes, SA, SB, c);
      mi.a_tmem0 = tmem_base + a_tmem_col;
      uint32_t tc = 0;
      bool issued = false;
      int prev_nt = -1;
      for (int tile = unit0; tile < num_tiles; tile += units, ++tc) {
        const uint32_t ab = tc % (uint32_t)n_acc;
        if (!mbar_wait(&bar->tempty[ab], ring_parity(tc, n_acc) ^ 1u, abort_flag, err, p.timeout_ns)) break;
        tc_fence_after();
        issued = true;
        constexpr int kGroup = 1;
        bool ok;
        if (gather) {
          ok = mma_tile_unified<kGroup, PAIR, kGatherKb, true, F8>(bar, mi, num_kb, tmem_base + ab * BN, abort_flag,
                                                                   err, p.timeout_ns);
        } else if (res_b) {
          const int nt = tile % n_tiles;
          const int next = tile + units;
          const bool b_load = nt != prev_nt;
          const bool b_last = next >= num_tiles || next % n_tiles != nt;
          prev_nt = nt;
          ok = mma_tile_resident_b<PAIR>(bar, mi, num_kb, tmem_base + ab * BN, b_load, b_last, abort_flag, err,
                                         p.timeout_ns);
        } else if (p.dense_pair_ring) {
          ok = mma_tile_unified<1, PAIR, 1, false>(bar, mi, num_kb, tmem_base + ab * BN, abort_flag, err,
                                                   p.timeout_ns);
        } else {
          ok = mma_tile<false, kGroup, PAIR>(bar, mi, num_kb, tmem_base + ab * BN, abort_flag, err, p.timeout_ns);
        }
        if (!ok) break;
        if constexpr (PAIR) {
          tc_commit_pair(&bar->tfull[ab]);
        } else {
          tc_commit(&bar->tfull[ab]);
        }
      }
      mma_drain<PAIR>(bar, issued, err, p.timeout_ns);
    } else if (PAIR && lane == 0) {
      // the other CTA's MMAs read this CTA's tensor and shared memory: wait for them to finish
      volatile int never = 0;
      mbar_wait(&bar->done, 0, &never, err, p.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-3)
    uint32_t tc = 0, nbox = 0;
    const int out_base = p.out_abs ? lo : 0;
    const uint32_t epi_boxes = smem_u32(sm.epi) + (uint32_t)warp * 2u * kEpiBoxBytes;
    // this warp's copy of the tile's bias columns (the data gradient has no bias)
    float* const bias_w = sm.bias + warp * kEpiBiasCols;
    const uint32_t bias_s = (!MIRROR && p.bias) ? smem_u32(bias_w) : 0u;
    int bias_n0 = -1;
    static_assert(BN <= kEpiBiasCols, "bias staging holds one tile's columns");
    for (int tile = unit0; tile < num_tiles; tile += units, ++tc) {
      const uint32_t ab = tc % (uint32_t)n_acc;
      const int m0 = (tile / n_tiles) * kRows + row_off;
      const int n0 = (tile % n_tiles) * BN;
      if (!MIRROR && p.bias && n0 != bias_n0) {
        // while the tile's MMAs run, once every lane is done with the old columns
        __syncwarp();
        for (int c = lane; c < BN; c += 32) bias_w[c] = __ldg(p.bias + n0 + c);
        __syncwarp();
        bias_n0 = n0;
      }
      const int row = m0 + warp * 32 + lane;
      const int orow_i = out_base + row;
      if (p.residual && row < M && orow_i >= 0 && orow_i < p.out_rows) {
        // bring this row's residual segment toward L2 while the tile's MMAs run
        const char* rp = reinterpret_cast<const char*>(p.residual + (size_t)orow_i * p.ldo + n0);
#pragma unroll
        for (int b = 0; b < BN * 2; b += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(rp + b));
      }
      if (!warp_wait(&bar->tfull[ab], ring_parity(tc, n_acc), abort_flag, err, p.timeout_ns)) break;
      tc_fence_after();
      const bool valid = row < M && orow_i >= 0 && orow_i < p.out_rows;
      const uint32_t acc = tmem_base + ((uint32_t)(warp * 32) << 16) + ab * BN;
      // hand the accumulator back to the MMA issuer (at rank 0 of a pair)
      auto release = [&]() {
        tc_fence_before();
        if (PAIR && !leader) {
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(lead(&bar->tempty[ab]));
        } else {
          warp_arrive(&bar->tempty[ab]);
        }
      };
      if (tma_epi && __all_sync(0xffffffffu, valid)) {
        if (p.out_tma == 2)
          epilogue_tma<BN, true>(p, acc, epi_boxes, nbox, orow_i - lane, n0, bias_s, release);
        else
          epilogue_tma<BN, false>(p, acc, epi_boxes, nbox, orow_i - lane, n0, bias_s, release);
      } else {
        epilogue_rows<BN>(p, acc, valid, (size_t)orow_i, n0, bias_s);
        release();
      }
    }
    if (tma_epi && lane == 0) bulk_wait_group<0>();  // bulk copies complete before the CTA exits
  }

  tc_fence_before();
  if constexpr (PAIR) {
    cluster_sync();  // no CTA leaves while the other may still arrive on or read its memory
  } else {
    __syncthreads();
  }
  if (warp == kMmaWarp) {
    tc_fence_after();
    if constexpr (PAIR) {
      tmem_dealloc_pair(tmem_base, tmem_cols);
    } else {
      tmem_dealloc(tmem_base, tmem_cols);
    }
  }
}

// ============================================================================ small-channel conv
// C = 64 on the gathered side and 64 output columns (the small-channel adapter
// conv and its data gradient).  Here an MMA is short (128x64x16) and the per-stage
// handshakes of the general kernel (an mbarrier wait on A and on B before every 4
// MMAs) cost more than the MMAs themselves.  So this kernel keeps all of W (9 taps x
// 64 x 64 bf16 = 72 KB) resident in shared memory, holds all 9 gathered A taps of a
// tile in tensor memory at once (9 x 32 columns next to two 64-column accumulators),
// and synchronises the MMA issuer with the builders twice per tile (one barrier per
// builder group: taps 0-4 and 5-8) instead of twice per tap.  The first two tiles'
// index entries, halo windows and W are requested before the CTA's setup barrier.
constexpr int kSmallTaps0 = 5;                    // builder group 0: taps 0..4, group 1: 5..8
constexpr uint32_t kSmallACol = 128;              // A taps after the two accumulators
constexpr uint32_t kSmallTmemCols = 512;          // 128 + 9 * 32 = 416 columns used
constexpr uint32_t kSmallWBytes = 9 * 64 * 64 * 2;

struct __align__(16) SmallBars {
  uint32_t zero128[32];          // 128 zero bytes (row source for missing neighbours)
  uint64_t wfull;
  uint64_t lfull[2], lempty[2];  // index entries + halo window of a tile
  uint64_t afull[2], aempty[2];  // per builder group
  uint64_t tfull[2], tempty[2];  // accumulators
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
};

__host__ __device__ constexpr size_t small_smem_bytes() {
  return 1024 + kSmallWBytes + 2 * (size_t)kConvHaloRows * 128 + 2 * (size_t)kConvIdx * 4 + sizeof(SmallBars);
}

template <bool MIRROR>
__global__ void __launch_bounds__(kThreads, 1) tc_conv_small_kernel(const __grid_constant__ TcConvParams p) {
  extern __shared__ uint8_t smem_raw[];
  constexpr uint32_t kHaloBufBytes = kConvHaloRows * 128;
  const uint32_t sbase = smem_u32(smem_raw);
  uint8_t* sw = smem_raw + (((sbase + 1023u) & ~1023u) - sbase);
  uint8_t* shalo = sw + kSmallWBytes;
  int32_t* sidx = reinterpret_cast<int32_t*>(shalo + 2 * kHaloBufBytes);
  SmallBars* bar = reinterpret_cast<SmallBars*>(reinterpret_cast<uint8_t*>(sidx) + 2 * kConvIdx * 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* err = p.status;
  const int M = p.M;
  const int num_tiles = (M + kBM - 1) / kBM;

  // index entries (cp.async, one arrival per lane) and the halo window (TMA) of a tile
  auto issue_tile = [&](int tile, int slot) {
    const int m0 = tile * kBM;
    const int32_t* src = p.nbr + (size_t)m0 * 9;
    const int lim = min(M - m0, kBM) * 9;
    copy_index_entries(smem_u32(sidx + slot * kConvIdx), src, lim, ((reinterpret_cast<uintptr_t>(src) & 15u) == 0),
                       &bar->lfull[slot], kHaloBufBytes);
    if (lane == 0) {
      const uint32_t hdst = smem_u32(shalo + slot * kHaloBufBytes);
#pragma unroll
      for (int q = 0; q < kConvHaloRows / kHaloBox; ++q)
        tma_load_2d(hdst + q * kHaloBox * 128, &p.tmap_a, &bar->lfull[slot], 0, m0 - kConvPad + q * kHaloBox);
    }
    __syncwarp();
  };

  // ---- setup: the loaders initialise their own barriers and start their first copies
  uint32_t issued = 0;
  if (warp == kHaloWarp) {
    if (lane == 0) {
      for (int i = 0; i < 2; ++i) {
        mbar_init(&bar->lfull[i], 33);  // 32 cp.async arrivals + the expect_tx arrival
        mbar_init(&bar->lempty[i], kProdWarps);
      }
      fence_barrier_init();
      fence_proxy_async_smem();
      prefetch_tmap(&p.tmap_a);
    }
    __syncwarp();
    pdl_wait();  // the neighbour table and features may come from the kernel before this one
    for (int t = blockIdx.x; t < num_tiles && issued < 2; t += gridDim.x) issue_tile(t, (int)issued++);
  } else if (warp == kBWarp) {
    if (lane == 0) {
      mbar_init(&bar->wfull, 1);
      fence_barrier_init();
      fence_proxy_async_smem();
      pdl_wait();
      mbar_arrive_expect_tx(&bar->wfull, kSmallWBytes);
      const uint32_t dst = smem_u32(sw);
      for (int j = 0; j < 9; ++j) {
        if constexpr (!MIRROR) {
          tma_load_2d(dst + j * 8192, &p.tmap_b, &bar->wfull, j * 64, 0);  // W_j [o][i], K-major
        } else {
          tma_load_3d(dst + j * 8192, &p.tmap_b, &bar->wfull, 0, j, 0);   // W_j^T: [o] rows of i, MN-major
        }
      }
    }
    __syncwarp();
  } else if (threadIdx.x == 0) {
    for (int i = 0; i < 32; ++i) bar->zero128[i] = 0u;
    for (int g = 0; g < 2; ++g) {
      mbar_init(&bar->afull[g], kProdWarps / 2);
      mbar_init(&bar->aempty[g], 1);
      mbar_init(&bar->tfull[g], 1);
      mbar_init(&bar->tempty[g], kEpiWarps);
    }
    mbar_init(&bar->done, 1);
    bar->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bar->tmem_base, kSmallTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  pdl_trigger();
  const uint32_t tmem_base = bar->tmem_base;
  volatile int* abort_flag = &bar->abort_flag;

  if (warp == kHaloWarp) {
    // ------------------------------------------------------------ index / halo loader (tiles 2, 3, ...)
    bool aborted = false;
    uint32_t ti = issued;
    for (int tile = blockIdx.x + (int)issued * gridDim.x; tile < num_tiles; tile += gridDim.x, ++ti) {
      const int slot = ti & 1;
      if (!warp_wait(&bar->lempty[slot], ring_parity(ti, 2) ^ 1u, abort_flag, err, p.timeout_ns)) {
        aborted = true;
        break;
      }
      issue_tile(tile, slot);
      ++issued;
    }
    if (aborted) drain_ring(bar->lfull, issued, 2, err, p.timeout_ns);
  } else if (warp == kBWarp) {
    // W stays resident; make sure its copy has landed before the CTA can exit
    if (lane == 0) {
      volatile int never = 0;
      mbar_wait(&bar->wfull, 0, &never, err, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= kEpiWarps && warp < kHaloWarp) {
    // ------------------------------------------------------------ A builders
    // Thread (w, lane) owns tile row 32 (w % 4) + lane; group 0 writes taps 0-4 and
    // group 1 taps 5-8 of that row into their tensor-memory columns.
    const int grp = (warp - kEpiWarps) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int j0 = grp ? kSmallTaps0 : 0, j1 = grp ? 9 : kSmallTaps0;
    const uint32_t a_lane = tmem_base + ((uint32_t)(quarter * 32) << 16) + kSmallACol;
    const uint32_t zero_row = smem_u32(bar->zero128);
    uint32_t ti = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++ti) {
      const int slot = ti & 1;
      if (!warp_wait(&bar->lfull[slot], ring_parity(ti, 2), abort_flag, err, p.timeout_ns) ||
          !warp_wait(&bar->aempty[grp], (ti & 1u) ^ 1u, abort_flag, err, p.timeout_ns))
        break;
      tc_fence_after();  // the previous tile's MMAs have finished reading these columns
      const int m0 = tile * kBM;
      const bool row_ok = m0 + r < M;
      const int hlo = m0 - kConvPad;
      const uint32_t halo = smem_u32(shalo + slot * kHaloBufBytes);
      const uint32_t si_s = smem_u32(sidx + slot * kConvIdx);
      for (int j = j0; j < j1; ++j) {
        const int jj = MIRROR ? 8 - j : j;
        // branch-free row selection (see the general kernel's builders)
        const int raw = row_ok ? ld_shared_s32(si_s + 4u * (uint32_t)(r * 9 + jj)) : -1;
        const bool bad = (raw >= 0) & ((unsigned)raw >= (unsigned)p.a_rows);
        const int idx = bad ? -1 : raw;
        const int h = idx - hlo;
        const bool in_win = (idx >= 0) & ((unsigned)h < (unsigned)kConvHaloRows);
        const uint32_t row = in_win ? halo + (uint32_t)h * 128u : zero_row;
        const int sw = in_win ? (h & 7) : 0;
        uint32_t v[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 q = ld_shared_16(row + ((c ^ sw) << 4));
          v[4 * c] = q.x, v[4 * c + 1] = q.y, v[4 * c + 2] = q.z, v[4 * c + 3] = q.w;
        }
        const bool far = (idx >= 0) & !in_win;
        if (__any_sync(0xffffffffu, far | bad)) {
          if (bad) atomicOr(err, SVCONV_STATUS_BAD_INDEX);
          if (far) {
            const __nv_bfloat16* src = p.A + (size_t)idx * p.lda;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 q = ldg_16(src + c * 8);
              v[4 * c] = q.x, v[4 * c + 1] = q.y, v[4 * c + 2] = q.z, v[4 * c + 3] = q.w;
            }
          }
        }
        tmem_st_32x32b_x32(a_lane + (uint32_t)j * kTmemAStageCols, v);
      }
      tmem_st_wait();
      tc_fence_before();
      warp_arrive(&bar->afull[grp]);
      warp_arrive(&bar->lempty[slot]);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer: 36 MMAs per tile, 2 waits
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, 64, 0, MIRROR ? 1 : 0);
      const uint64_t b0 = MIRROR ? smem_desc_sw128(smem_u32(sw), 8192, 1024) : smem_desc_sw128(smem_u32(sw), 16, 1024);
      const uint32_t k16 = MIRROR ? (2048u >> 4) : (32u >> 4);  // start-address step per K=16
      bool issued_any = false;
      if (mbar_wait(&bar->wfull, 0, abort_flag, err, p.timeout_ns)) {
        uint32_t tc = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tc) {
          const uint32_t ab = tc & 1u;
          if (!mbar_wait(&bar->tempty[ab], ring_parity(tc, 2) ^ 1u, abort_flag, err, p.timeout_ns)) break;
          const uint32_t d = tmem_base + ab * 64;
          bool ok = true;
          for (int g = 0; g < 2 && ok; ++g) {
            if (!mbar_wait(&bar->afull[g], tc & 1u, abort_flag, err, p.timeout_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issued_any = true;
            const int j0 = g ? kSmallTaps0 : 0, j1 = g ? 9 : kSmallTaps0;
            for (int j = j0; j < j1; ++j) {
              const uint64_t bd = b0 + (uint64_t)((uint32_t)j * (8192u >> 4));
              const uint32_t at = tmem_base + kSmallACol + (uint32_t)j * kTmemAStageCols;
#pragma unroll
              for (int k = 0; k < 4; ++k)
                tc_mma_bf16_ts(d, at + k * 8, bd + (uint64_t)(k * k16), idesc, (j | k) != 0 ? 1u : 0u);
            }
            tc_commit(&bar->aempty[g]);
          }
          if (!ok) break;
          tc_commit(&bar->tfull[ab]);
        }
      }
      if (issued_any) {
        volatile int never = 0;
        tc_commit(&bar->done);
        mbar_wait(&bar->done, 0, &never, err, p.timeout_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-3)
    uint32_t tc = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tc) {
      const uint32_t ab = tc & 1u;
      if (!warp_wait(&bar->tfull[ab], ring_parity(tc, 2), abort_flag, err, p.timeout_ns)) break;
      tc_fence_after();
      const int row = tile * kBM + warp * 32 + lane;
      epilogue_rows<64>(p, tmem_base + ((uint32_t)(warp * 32) << 16) + ab * 64, row < M, (size_t)row, 0);
      tc_fence_before();
      warp_arrive(&bar->tempty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kSmallTmemCols);
  }
}

// ============================================================================ weight gradient
// dW^T[(j,i)][o] = sum_k X[N[k,j]][i] dY[k][o] (SV-TAD page, Key Design 2: the
// weight gradient is the transposed contraction over kept tokens), db[o] = sum_k dY[k][o].
//
// M (accumulator rows) runs over (64-channel block cb, tap j, channel c): each
// block cb owns 10 half-tiles of 64 rows, taps 0..8 then one extra half that holds
// the all-ones row for db (block 0) or padding (other blocks), so a 128-row tile
// covers two taps of ONE channel block and needs a single halo.  Partial row of
// (j, i): ((i / 64) * 10 + j) * 64 + i % 64; db is row 9 * 64.
//
// K runs over tokens in blocks of 64.  The halo of a block is the fixed window
// of X rows k0 - 32 .. k0 + 95 (a neighbour is at most W + 1 packed rows away), so
// its TMA is issued together with the block's index entries, without waiting for
// them; an entry outside the window (W > 31, or tokens out of raster order) is
// read from global memory instead.  A lives in tensor memory: the builders read
// 8 x 8 (token x channel) pieces of the halo with ldmatrix.trans, which yields
// exactly the (channel lane, token-pair column) order of tcgen05.st.16x128b, so A
// is transposed and gathered on the way in, with no shared-memory stores.  B is
// dY by TMA (MN-major).
//
// PAIR (256 columns, an even number of 128-row tiles): a cluster of two CTAs takes two
// adjacent row tiles with M = 256 MMAs, each CTA building its own tile's A in its tensor
// memory and loading half of the dY columns, so a dY tile crosses into the SMs once per
// 256 rows instead of once per 128.  CTA rank 0 issues the MMAs; the A / B full barriers
// and the accumulator release count both CTAs and live in rank 0; the MMA commits arrive
// in both CTAs.  Halo and index slots stay per CTA.  A pair's stage holds two token blocks
// (A: 2 x 32 tensor-memory columns; B: both blocks' dY halves) on ONE full / empty barrier
// pair, as in the gather conv, so the issuing thread waits and commits once per 8 MMAs.
// Weight-gradient builder, rare path (kept out of line so the builders' loop stays small):
// the 16 registers of a 16-channel piece hold zeros for entries outside the halo window;
// fetch those elements from global memory.
struct Regs16 {
  uint32_t v[16];
};
__device__ __noinline__ Regs16 wgrad_patch_far(Regs16 R, uint32_t sidx_s, const uint16_t* X16, int n, int Cin, int k0,
                                               int hlo, int j, int ch0, int win = kWgHaloRows) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const int k4 = r >> 2, m = r & 3;
    const int ch = ch0 + 8 * (m & 1) + (lane >> 2);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int tk = 16 * k4 + 8 * (m >> 1) + 2 * (lane & 3) + e;
      const int x = k0 + tk < n ? ld_shared_s32(sidx_s + 4u * (uint32_t)(tk * 9 + j)) : -1;
      if (x >= 0 && x < n && (unsigned)(x - hlo) >= (unsigned)win) {
        const uint32_t v = __ldg(X16 + (size_t)x * Cin + ch);
        R.v[r] = e == 0 ? ((R.v[r] & 0xFFFF0000u) | v) : ((R.v[r] & 0x0000FFFFu) | (v << 16));
      }
    }
  }
  return R;
}

template <int BN, bool PAIR = false>
__global__ void __launch_bounds__(kThreads, 1) tc_wgrad_kernel(const __grid_constant__ TcWgradParams p) {
  static_assert(!PAIR || BN == 256, "CTA pairs run 256-column tiles");
  extern __shared__ uint8_t smem_raw[];
  const int SB = p.stages_b;
  const Geometry geo = wgrad_geometry(BN, SB, PAIR);
  const Carve sm = carve(smem_raw, geo);
  TcBarriers* bar = sm.bar;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* err = p.status;
  constexpr int kBCols = PAIR ? BN / 2 : BN;  // dY columns this CTA loads per stage
  constexpr uint32_t kBBytes = kBCols * kBK * 2;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;  // first unit of this CTA (pair)
  const int ustride = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;  // unit stride
  // rank 0's copy of a barrier (PAIR)
  auto lead = [](uint64_t* b) -> uint32_t { return mapa_shared(smem_u32(b), 0u); };
  constexpr int kAcc = wgrad_acc_buffers(BN);
  constexpr uint32_t kTmemCols = wgrad_tmem_cols(BN);
  constexpr uint32_t kACol = (uint32_t)(kAcc * BN);  // first column of the A stages
  constexpr uint32_t kHaloBufBytes = kWgHaloRows * 128;
  constexpr int kSlots = wgrad_slots(BN, PAIR);
  // PAIR: stages of kKbs = 2 token blocks, A and B on one barrier pair (p.stages_a == p.stages_b)
  constexpr int kKbs = PAIR ? 2 : 1;
  const int kAStages = p.stages_a;
  // Builder groups of four warps.  At 256 columns a CTA usually carries one unit, so its four
  // epilogue warps would idle until the very end: they build A stages as a third group.
  constexpr int kGroups = BN == 256 ? 3 : 2;

  const int m_tiles = p.rows_pad / kBM;
  const int m_units = PAIR ? m_tiles / 2 : m_tiles;  // row tiles (PAIR: pairs of adjacent tiles)
  const int n_tiles = p.Cout / BN;
  const int num_units = m_units * n_tiles * p.splits;
  const int kbt = (p.n + kBK - 1) / kBK;  // token blocks in total

  if (threadIdx.x == 0) {
    // ifull: 32 cp.async arrivals of the loader lanes + its expect_tx arrival
    // afull: one builder group of four warps (of each CTA of a pair); tempty: the epilogue warps (of both)
    // PAIR: afull also counts the weight loader's expect_tx arrival (rank 0)
    init_barriers(bar, kAStages, PAIR ? 0 : SB, PAIR ? 2 * (kProdWarps / 2) + 1 : kProdWarps / 2, kSlots, 33,
                  kProdWarps / 2, (PAIR ? 2 : 1) * kEpiWarps);
    prefetch_tmap(&p.tmap_x);
    prefetch_tmap(&p.tmap_dy);
  }
  if (warp == kMmaWarp) {
    if constexpr (PAIR) {
      tmem_alloc_pair(&bar->tmem_base, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&bar->tmem_base, kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) {
    cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA arrival
  } else {
    __syncthreads();
  }
  tc_fence_after();
  pdl_wait();  // inputs and outputs may belong to the kernel before this one
  pdl_trigger();
  const uint32_t tmem_base = bar->tmem_base;
  volatile int* abort_flag = &bar->abort_flag;

  // unit -> (split, m-tile, n-tile); units of one split run side by side so the
  // tiles of dY and the X rows they share are hot in L2.  PAIR: this CTA's tile of the pair.
  auto decode = [&](int u, int& sp, int& mt, int& n0, int& kb0, int& kb1) {
    const int nt = u % n_tiles;
    const int rest = u / n_tiles;
    mt = PAIR ? 2 * (rest % m_units) + (int)rank : rest % m_units;
    sp = rest / m_units;
    n0 = nt * BN;
    kb0 = (int)((long long)kbt * sp / p.splits);
    kb1 = (int)((long long)kbt * (sp + 1) / p.splits);
  };

  // Builds the A stages of unit u whose running stage index qs satisfies qs % kGroups == grp
  // (qs counts every stage of the CTA and qb every token block, so the groups stay in step);
  // false when a wait gave up.
  auto build_unit = [&](int u, uint32_t& qs, uint32_t& qb, int grp) -> bool {
    const int quarter = warp & 3;
    const int half = quarter >> 1;
    const int cq = (quarter & 1) * 32;
    const uint32_t zero_addr = smem_u32(bar->zero16);
    const uint16_t* X16 = reinterpret_cast<const uint16_t*>(p.X);
    int sp, mt, n0, kb0, kb1;
    decode(u, sp, mt, n0, kb0, kb1);
    const int cb = mt / kWgTiles;
    const int j = 2 * (mt % kWgTiles) + half;        // tap of this warp's half (9: the extra half)
    const int kind = j < 9 ? 0 : (cb == 0 ? 1 : 2);  // gathered X, ones row, padding
    for (int kbs = kb0; kbs < kb1; kbs += kKbs, ++qs) {
      const int nb = min(kKbs, kb1 - kbs);  // token blocks in this stage
      if ((int)(qs % (uint32_t)kGroups) != grp) {
        qb += (uint32_t)nb;
        continue;
      }
      const int sa = (int)(qs % (uint32_t)kAStages);
      if (!warp_wait(&bar->aempty[sa], ring_parity(qs, kAStages) ^ 1u, abort_flag, err, p.timeout_ns)) return false;
      tc_fence_after();  // the MMAs that read this A stage are complete
      for (int hb = 0; hb < nb; ++hb, ++qb) {
        const int kb = kbs + hb;
        const int slot = (int)(qb % kSlots);
        if (!warp_wait(&bar->ifull[slot], ring_parity(qb, kSlots), abort_flag, err, p.timeout_ns)) return false;
        const int k0 = kb * kBK;
        const uint32_t a_col = tmem_base + kACol + (uint32_t)(sa * kKbs + hb) * kTmemAStageCols;
        if (kind == 0) {
          const uint32_t sidx_s = smem_u32(sm.idx + slot * kWgIdx);
          const uint32_t halo = smem_u32(sm.halo + (size_t)slot * kHaloBufBytes);
          const int hlo = k0 - kWgPad;
          const int mi = lane >> 3;
  #pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            const int c16 = cq + 16 * sub;  // first channel of these 16 lanes
            uint32_t R[16];
            bool far = false, bad = false;
            const int chunk = (c16 >> 3) + (mi & 1);
  #pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              // branch-free: entries of tokens past n (stale slot contents) count as missing
              const int tk = 16 * k4 + 8 * (mi >> 1) + (lane & 7);
              const int raw = ld_shared_s32(sidx_s + 4u * (uint32_t)(tk * 9 + j));
              const bool tok_ok = k0 + tk < p.n;
              bad |= tok_ok & (raw >= p.n);
              const int x = (tok_ok & (raw < p.n)) ? raw : -1;
              const int h = x - hlo;
              const bool in_win = (x >= 0) & ((unsigned)h < (unsigned)kWgHaloRows);
              far |= (x >= 0) & !in_win;
              const uint32_t addr =
                  in_win ? halo + (uint32_t)h * 128u + ((uint32_t)(chunk ^ (h & 7)) << 4) : zero_addr;
              ldmatrix_x4_trans(addr, R[4 * k4], R[4 * k4 + 1], R[4 * k4 + 2], R[4 * k4 + 3]);
            }
            if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(err, SVCONV_STATUS_BAD_INDEX);
            if (__any_sync(0xffffffffu, far)) {
              // entries outside the halo window read as zero above: fetch them from global memory
              Regs16 rr;
  #pragma unroll
              for (int r = 0; r < 16; ++r) rr.v[r] = R[r];
              rr = wgrad_patch_far(rr, sidx_s, X16, p.n, p.Cin, k0, hlo, j, cb * kBK + c16);
  #pragma unroll
              for (int r = 0; r < 16; ++r) R[r] = rr.v[r];
            }
            tmem_st_16x128b_x8(a_col + ((uint32_t)(32 * quarter + 16 * sub) << 16), R);
          }
        } else if (kind == 1) {
          // row 0 of the extra half is 1 for every valid token: its accumulator row is db
  #pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            uint32_t R[16];
  #pragma unroll
            for (int r = 0; r < 16; ++r) R[r] = 0u;
            if ((quarter & 1) == 0 && sub == 0 && lane < 4) {
  #pragma unroll
              for (int k = 0; k < 8; ++k) {
                const int tk = k0 + 8 * k + 2 * lane;
                R[2 * k] = (tk < p.n ? 0x3F80u : 0u) | (tk + 1 < p.n ? 0x3F800000u : 0u);
              }
            }
            tmem_st_16x128b_x8(a_col + ((uint32_t)(32 * quarter + 16 * sub) << 16), R);
          }
        }
        // (padding halves are not written: their accumulator rows are never read)
        warp_arrive(&bar->iempty[slot]);  // the halo and index rows are in registers / tensor memory
      }
      tmem_st_wait();
      tc_fence_before();
      if (PAIR && !leader) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lead(&bar->afull[sa]));
      } else {
        warp_arrive(&bar->afull[sa]);
      }
    }
    return true;
  };

  if (warp == kHaloWarp) {
    // ------------------------------------------------------------ index entries + halo window, per token block
    uint32_t q = 0;
    bool aborted = false;
    for (int u = unit0; u < num_units && !aborted; u += ustride) {
      int sp, mt, n0, kb0, kb1;
      decode(u, sp, mt, n0, kb0, kb1);
      const int cb = mt / kWgTiles;
      for (int kb = kb0; kb < kb1; ++kb, ++q) {
        const int slot = (int)(q % kSlots);
        if (!warp_wait(&bar->iempty[slot], ring_parity(q, kSlots) ^ 1u, abort_flag, err, p.timeout_ns)) {
          aborted = true;
          break;
        }
        const int k0 = kb * kBK;
        const int lim = min(p.n - k0, kBK) * 9;
        const int32_t* src = p.nbr + (size_t)k0 * 9;
        copy_index_entries(smem_u32(sm.idx + slot * kWgIdx), src, lim, ((reinterpret_cast<uintptr_t>(src) & 15u) == 0),
                           &bar->ifull[slot], kHaloBufBytes);
        if (lane == 0) {
          const uint32_t hb = smem_u32(sm.halo + (size_t)slot * kHaloBufBytes);
          // the whole window in one box: the loader's issue time per block, not bytes, paced
          // the kernel (one copy fewer per block measured 3% faster)
          tma_load_2d(hb, &p.tmap_x, &bar->ifull[slot], cb * kBK, k0 - kWgPad);
        }
        __syncwarp();
      }
    }
    if (aborted) drain_ring(bar->ifull, q, kSlots, err, p.timeout_ns);
  } else if (warp == kBWarp) {
    // ------------------------------------------------------------ dY tiles
    uint32_t it = 0;
    bool aborted = false;
    for (int u = unit0; u < num_units && !aborted; u += ustride) {
      int sp, mt, n0, kb0, kb1;
      decode(u, sp, mt, n0, kb0, kb1);
      for (int kb = kb0; kb < kb1; kb += kKbs, ++it) {
        const int sb = (int)(it % (uint32_t)SB);
        uint64_t* const empty = PAIR ? bar->aempty : bar->bempty;  // PAIR: one ring with the A stages
        if (!warp_wait(&empty[sb], ring_parity(it, SB) ^ 1u, abort_flag, err, p.timeout_ns)) {
          aborted = true;
          break;
        }
        if (lane == 0) {
          const uint32_t dst = smem_u32(sm.b + (size_t)sb * kKbs * kBBytes);
          if constexpr (PAIR) {
            // this CTA's half of the columns of the stage's blocks, counted on rank 0's full barrier
            const int nb = min(kKbs, kb1 - kb);
            if (leader) mbar_arrive_expect_tx(&bar->afull[sb], 2u * (uint32_t)nb * kBBytes);
            const uint32_t fb = lead(&bar->afull[sb]);
            for (int h = 0; h < nb; ++h) {
#pragma unroll
              for (int q = 0; q < kBCols / 64; ++q)
                tma_load_2d_pair(dst + h * kBBytes + q * 8192, &p.tmap_dy, fb, n0 + (int)rank * kBCols + q * 64,
                                 (kb + h) * kBK);
            }
          } else {
            mbar_arrive_expect_tx(&bar->bfull[sb], kBBytes);
#pragma unroll
            for (int q = 0; q < BN / 64; ++q)
              tma_load_2d(dst + q * 8192, &p.tmap_dy, &bar->bfull[sb], n0 + q * 64, kb * kBK);
          }
        }
        __syncwarp();
      }
    }
    if (aborted) {
      if (PAIR) {
        // the full barriers live in rank 0 and also count the builders: give this warp's
        // copies in flight time to land instead of waiting on a phase
        if (lane == 0) {
          const uint64_t t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < 200000u) {
          }
        }
        __syncwarp();
      } else {
        drain_ring(bar->bfull, it, SB, err, p.timeout_ns);
      }
    }
  } else if (warp >= kEpiWarps && warp < kHaloWarp) {
    // ------------------------------------------------------------ A builders (tensor memory)
    // Groups of four warps take turns over the token blocks (two groups, plus the epilogue
    // warps as a third at 256 columns).  Warp w writes TMEM lanes
    // 32 (w % 4) .. + 31: half (w % 4) / 2 of the tile, channels 32 (w % 2) .. + 31 of
    // that half's tap, as two 16-lane pieces of 16 channels x 64 tokens.  For one
    // piece, ldmatrix k4 (k4 = 0..3) covers tokens 16 k4 .. + 15: lane i supplies the
    // halo row of token 16 k4 + 8 (i / 16) + i % 8, channels +8 ((i / 8) % 2); its four
    // registers are then registers 4 k4 .. 4 k4 + 3 of the 16x128b.x8 store.
    const int grp = (warp - kEpiWarps) >> 2;
    uint32_t qs = 0, qb = 0;
    for (int u = unit0; u < num_units; u += ustride)
      if (!build_unit(u, qs, qb, grp)) break;
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      MmaCfg c;
      c.idesc = idesc_bf16_f32(PAIR ? 2 * kBM : kBM, BN, 0, 1);  // A from tensor memory, B (dY) MN-major
      c.a_lbo = 0, c.a_sbo = 0, c.a_step = 0;
      c.b_lbo = 8192, c.b_sbo = 1024, c.b_step = 2048;  // 64-wide N groups 8 KB apart, 16 K rows per step
      MmaIssuer mi = make_issuer(sm, kKbs * kBBytes, kAStages, SB, c);
      mi.a_tmem0 = tmem_base + kACol;
      uint32_t tc = 0;
      bool issued = false;
      for (int u = unit0; u < num_units; u += ustride, ++tc) {
        int sp, mt, n0, kb0, kb1;
        decode(u, sp, mt, n0, kb0, kb1);
        const uint32_t ab = tc % (uint32_t)kAcc;
        if (!mbar_wait(&bar->tempty[ab], ring_parity(tc, kAcc) ^ 1u, abort_flag, err, p.timeout_ns)) break;
        tc_fence_after();
        issued = true;
        bool ok;
        if constexpr (PAIR) {
          ok = mma_tile_unified<1, true, kKbs>(bar, mi, kb1 - kb0, tmem_base + ab * BN, abort_flag, err, p.timeout_ns);
        } else {
          ok = mma_tile<true, 2>(bar, mi, kb1 - kb0, tmem_base + ab * BN, abort_flag, err, p.timeout_ns);
        }
        if (!ok) break;
        if constexpr (PAIR) {
          tc_commit_pair(&bar->tfull[ab]);
        } else {
          tc_commit(&bar->tfull[ab]);
        }
      }
      mma_drain<PAIR>(bar, issued, err, p.timeout_ns);
    } else if (PAIR && lane == 0) {
      // the other CTA's MMAs read this CTA's tensor and shared memory: wait for them to finish
      volatile int never = 0;
      mbar_wait(&bar->done, 0, &never, err, p.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue: fp32 partial rows
    uint32_t tc = 0;
    uint32_t qes = 0, qeb = 0;  // stage and block counters of the third builder group
    for (int u = unit0; u < num_units; u += ustride, ++tc) {
      if constexpr (kGroups == 3) {
        if (!build_unit(u, qes, qeb, 2)) break;
      }
      int sp, mt, n0, kb0, kb1;
      decode(u, sp, mt, n0, kb0, kb1);
      const uint32_t ab = tc % (uint32_t)kAcc;
      const bool empty_range = kb1 <= kb0;  // no MMA ran for this unit: its partial is zero
      if (!warp_wait(&bar->tfull[ab], ring_parity(tc, kAcc), abort_flag, err, p.timeout_ns)) break;
      tc_fence_after();
      const int row = mt * kBM + warp * 32 + lane;
      float* dst = p.partial + ((size_t)sp * p.rows_pad + row) * p.Cout + n0;
      // The CTA's last unit: its MMAs are done and no dY tile will be loaded any more, so the
      // dY ring is free and stages the partial rows for TMA stores (whole lines, no per-thread
      // row stores); other units store their rows directly.
      if (p.part_tma && u + ustride >= num_units) {
        const uint32_t boxes = smem_u32(sm.b) + (uint32_t)warp * 2u * 4096u;
        const uint32_t sw = (uint32_t)(lane & 7);
        const int prow0 = sp * p.rows_pad + mt * kBM + warp * 32;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(warp * 32) << 16) + ab * BN + c0, v);
          const uint32_t box = boxes + (uint32_t)((c0 / 32) & 1) * 4096u;
          if (lane == 0) bulk_wait_group_read<1>();  // the store issued from this box two boxes ago has read it
          __syncwarp();
          tmem_ld_wait();
          // row `lane` of the box: 16-byte chunk k lands at chunk k ^ (lane & 7) (128-byte swizzle)
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t a0 = empty_range ? 0u : v[4 * k], a1 = empty_range ? 0u : v[4 * k + 1];
            const uint32_t a2 = empty_range ? 0u : v[4 * k + 2], a3 = empty_range ? 0u : v[4 * k + 3];
            st_shared_16(box + (uint32_t)lane * 128u + (((uint32_t)k ^ sw) << 4), a0, a1, a2, a3);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&p.tmap_part, box, n0 + c0, prow0);
            bulk_commit_group();
          }
        }
      } else {
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
      }
      // hand the accumulator back to the MMA issuer (at rank 0 of a pair)
      tc_fence_before();
      if (PAIR && !leader) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lead(&bar->tempty[ab]));
      } else {
        warp_arrive(&bar->tempty[ab]);
      }
    }
    if (p.part_tma && lane == 0) bulk_wait_group<0>();  // partial-row stores complete before the CTA exits
  }

  tc_fence_before();
  if constexpr (PAIR) {
    cluster_sync();  // no CTA leaves while the other may still arrive on or read its memory
  } else {
    __syncthreads();
  }
  if (warp == kMmaWarp) {
    tc_fence_after();
    if constexpr (PAIR) {
      tmem_dealloc_pair(tmem_base, kTmemCols);
    } else {
      tmem_dealloc(tmem_base, kTmemCols);
    }
  }
}

// ============================================================================ single-pass backward, 64 channels
// Both gradients of a C_in = C_out = 64 convolution in ONE pass over dY (SV-TAD page, Key
// Design 2: the dedicated backward kernels; both are adjoints of the forward):
//   dX[k]          = sum_j W_j^T dY[N[k][8-j]]                (mirrored gather, as tc_conv_small)
//   dW^T[(j,i)][o] += sum_{k in tile} X[N[k][j]][i] dY[k][o]  (gathered X transposed, as tc_wgrad)
// For each 128-token tile the loader brings the dY halo window (rows m0-32 .. m0+159), the X
// halo window over the same rows and the tile's neighbour entries once.  The dY window feeds
// the data gradient's gather AND, read in place as the MN-major B operand (its rows 32..159
// are the tile's own tokens), the weight gradient's MMAs; so dY crosses L2 -> SM once.
// The 640 x 64 fp32 weight-gradient accumulators (taps 0..8 and the db half, as in tc_wgrad)
// stay in tensor memory for all tiles of the CTA and are written once at the end as the
// CTA's split partial; the fixed-order split reduce turns them into dW and db.
// Tensor memory: dW^T accumulators (5 x 64 columns), the dX accumulator (64), and a ring of
// four 32-column A stages shared by both kinds of stage (19 per tile: 9 taps, 10 blocks).
constexpr int kFbStages = 4;
constexpr int kFbMTiles = 5;
constexpr int kFbStagesPerTile = 9 + 2 * kFbMTiles;
constexpr uint32_t kFbDxCol = kFbMTiles * 64;        // 320
constexpr uint32_t kFbACol = kFbDxCol + 64;          // 384
constexpr uint32_t kFbTmemCols = 512;
constexpr uint32_t kFbHaloBytes = kConvHaloRows * 128;
constexpr int kFbRowsPad = kFbMTiles * kBM;          // 640 partial rows

struct FbParams {
  CUtensorMap tmap_dy;  // dY [n][64], boxes {64, 64}
  CUtensorMap tmap_x;   // X [n][64], boxes {64, 64}
  CUtensorMap tmap_w;   // W as (i, j, o), box (64, 1, 64): W_j^T, MN-major
  const __nv_bfloat16* dY;
  const __nv_bfloat16* X;
  const int32_t* nbr;
  __nv_bfloat16* dX;
  float* partial;       // [gridDim.x][640][64]
  int* status;
  unsigned long long timeout_ns;
  int n;
};

struct __align__(16) FbBars {
  uint32_t zero128[32];  // 128 zero bytes
  uint64_t wfull;
  uint64_t lfull[2], lempty[2];                   // tile slots: index entries + both halos
  uint64_t afull[kFbStages], aempty[kFbStages];   // A stages in tensor memory
  uint64_t tfull, tempty;                         // dX accumulator
  uint64_t dwfull;                                // all weight-gradient MMAs of the CTA done
  uint32_t tmem_base;
  int abort_flag;
};

__host__ __device__ constexpr size_t fb_smem_bytes() {
  return 1024 + kSmallWBytes + 4 * (size_t)kFbHaloBytes + 2 * (size_t)kConvIdx * 4 + sizeof(FbBars);
}

__global__ void __launch_bounds__(kThreads, 1) tc_bwd_small_kernel(const __grid_constant__ FbParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  uint8_t* sw = smem_raw + (((sbase + 1023u) & ~1023u) - sbase);
  uint8_t* shalo = sw + kSmallWBytes;  // slot s: dY window at 2 s H, X window at (2 s + 1) H
  int32_t* sidx = reinterpret_cast<int32_t*>(shalo + 4 * kFbHaloBytes);
  FbBars* bar = reinterpret_cast<FbBars*>(reinterpret_cast<uint8_t*>(sidx) + 2 * kConvIdx * 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* err = p.status;
  const int M = p.n;
  const int num_tiles = (M + kBM - 1) / kBM;
  auto dy_win = [&](int slot) { return smem_u32(shalo + (size_t)(2 * slot) * kFbHaloBytes); };
  auto x_win = [&](int slot) { return smem_u32(shalo + (size_t)(2 * slot + 1) * kFbHaloBytes); };

  auto issue_tile = [&](int tile, int slot) {
    const int m0 = tile * kBM;
    const int32_t* src = p.nbr + (size_t)m0 * 9;
    const int lim = min(M - m0, kBM) * 9;
    copy_index_entries(smem_u32(sidx + slot * kConvIdx), src, lim, ((reinterpret_cast<uintptr_t>(src) & 15u) == 0),
                       &bar->lfull[slot], 2 * kFbHaloBytes);
    if (lane == 0) {
#pragma unroll
      for (int q = 0; q < kConvHaloRows / kHaloBox; ++q) {
        tma_load_2d(dy_win(slot) + q * kHaloBox * 128, &p.tmap_dy, &bar->lfull[slot], 0, m0 - kConvPad + q * kHaloBox);
        tma_load_2d(x_win(slot) + q * kHaloBox * 128, &p.tmap_x, &bar->lfull[slot], 0, m0 - kConvPad + q * kHaloBox);
      }
    }
    __syncwarp();
  };

  // ---- setup
  uint32_t issued = 0;
  if (warp == kHaloWarp) {
    if (lane == 0) {
      for (int i = 0; i < 2; ++i) {
        mbar_init(&bar->lfull[i], 33);              // 32 cp.async arrivals + the expect_tx arrival
        mbar_init(&bar->lempty[i], kProdWarps + 1);  // the builder warps + the MMAs that read dY in place
      }
      fence_barrier_init();
      fence_proxy_async_smem();
      prefetch_tmap(&p.tmap_dy);
      prefetch_tmap(&p.tmap_x);
    }
    __syncwarp();
    pdl_wait();
    for (int t = blockIdx.x; t < num_tiles && issued < 2; t += gridDim.x) issue_tile(t, (int)issued++);
  } else if (warp == kBWarp) {
    if (lane == 0) {
      mbar_init(&bar->wfull, 1);
      fence_barrier_init();
      fence_proxy_async_smem();
      pdl_wait();
      mbar_arrive_expect_tx(&bar->wfull, kSmallWBytes);
      const uint32_t dst = smem_u32(sw);
      for (int j = 0; j < 9; ++j) tma_load_3d(dst + j * 8192, &p.tmap_w, &bar->wfull, 0, j, 0);
    }
    __syncwarp();
  } else if (threadIdx.x == 0) {
    for (int i = 0; i < 32; ++i) bar->zero128[i] = 0u;
    for (int s = 0; s < kFbStages; ++s) {
      mbar_init(&bar->afull[s], kProdWarps / 2);
      mbar_init(&bar->aempty[s], 1);
    }
    mbar_init(&bar->tfull, 1);
    mbar_init(&bar->tempty, kEpiWarps);
    mbar_init(&bar->dwfull, 1);
    bar->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bar->tmem_base, kFbTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  pdl_trigger();
  const uint32_t tmem_base = bar->tmem_base;
  volatile int* abort_flag = &bar->abort_flag;

  if (warp == kHaloWarp) {
    // ------------------------------------------------------------ loader (tiles 2, 3, ...)
    bool aborted = false;
    uint32_t ti = issued;
    for (int tile = blockIdx.x + (int)issued * gridDim.x; tile < num_tiles; tile += gridDim.x, ++ti) {
      const int slot = ti & 1;
      if (!warp_wait(&bar->lempty[slot], ring_parity(ti, 2) ^ 1u, abort_flag, err, p.timeout_ns)) {
        aborted = true;
        break;
      }
      issue_tile(tile, slot);
      ++issued;
    }
    if (aborted) drain_ring(bar->lfull, issued, 2, err, p.timeout_ns);
  } else if (warp == kBWarp) {
    if (lane == 0) {  // W stays resident; its copy must land before the CTA can exit
      volatile int never = 0;
      mbar_wait(&bar->wfull, 0, &never, err, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= kEpiWarps && warp < kHaloWarp) {
    // ------------------------------------------------------------ A builders
    // Stage q of the CTA (19 per tile) goes to ring slot q % 4 and is built by the group of
    // four warps q % 2.  Taps 0..8: thread (quarter, lane) writes token row 32 quarter + lane
    // of dY[N[k][8-j]] (32x32b store).  Weight-gradient block (mt, tb): the transposed gather
    // of tc_wgrad over tokens m0 + 64 tb .. + 63, half (quarter / 2) of M-tile mt, channels
    // 32 (quarter % 2) .. + 31 (16x128b stores).
    const int grp = (warp - kEpiWarps) >> 2;
    const int quarter = warp & 3;
    const uint32_t zero_row = smem_u32(bar->zero128);
    const uint16_t* X16 = reinterpret_cast<const uint16_t*>(p.X);
    uint32_t q = 0, ti = 0;
    bool aborted = false;
    for (int tile = blockIdx.x; tile < num_tiles && !aborted; tile += gridDim.x, ++ti, q += kFbStagesPerTile) {
      const int slot = ti & 1;
      if (!warp_wait(&bar->lfull[slot], ring_parity(ti, 2), abort_flag, err, p.timeout_ns)) break;
      const int m0 = tile * kBM;
      const int hlo = m0 - kConvPad;
      const uint32_t si_s = smem_u32(sidx + slot * kConvIdx);
      for (int t = 0; t < kFbStagesPerTile; ++t) {
        const uint32_t qq = q + (uint32_t)t;
        if ((int)(qq & 1u) != grp) continue;
        const int st = (int)(qq % kFbStages);
        if (!warp_wait(&bar->aempty[st], ring_parity(qq, kFbStages) ^ 1u, abort_flag, err, p.timeout_ns)) {
          aborted = true;
          break;
        }
        tc_fence_after();  // the MMAs that read this stage are complete
        const uint32_t a_col = tmem_base + kFbACol + (uint32_t)st * kTmemAStageCols;
        if (t < 9) {
          const int j = t;
          const int r = quarter * 32 + lane;
          const bool row_ok = m0 + r < M;
          const uint32_t halo = dy_win(slot);
          const int raw = row_ok ? ld_shared_s32(si_s + 4u * (uint32_t)(r * 9 + (8 - j))) : -1;
          const bool bad = (raw >= 0) & ((unsigned)raw >= (unsigned)M);
          const int idx = bad ? -1 : raw;
          const int h = idx - hlo;
          const bool in_win = (idx >= 0) & ((unsigned)h < (unsigned)kConvHaloRows);
          const uint32_t row = in_win ? halo + (uint32_t)h * 128u : zero_row;
          const int swz = in_win ? (h & 7) : 0;
          uint32_t v[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 u = ld_shared_16(row + ((c ^ swz) << 4));
            v[4 * c] = u.x, v[4 * c + 1] = u.y, v[4 * c + 2] = u.z, v[4 * c + 3] = u.w;
          }
          const bool far = (idx >= 0) & !in_win;
          if (__any_sync(0xffffffffu, far | bad)) {
            if (bad) atomicOr(err, SVCONV_STATUS_BAD_INDEX);
            if (far) {
              const __nv_bfloat16* src = p.dY + (size_t)idx * 64;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const uint4 u = ldg_16(src + c * 8);
                v[4 * c] = u.x, v[4 * c + 1] = u.y, v[4 * c + 2] = u.z, v[4 * c + 3] = u.w;
              }
            }
          }
          tmem_st_32x32b_x32(a_col + ((uint32_t)(quarter * 32) << 16), v);
        } else {
          const int mt = (t - 9) >> 1, tb = (t - 9) & 1;
          const int half = quarter >> 1;
          const int cq = (quarter & 1) * 32;
          const int j = 2 * mt + half;  // 9: the extra half (its row 0 gives db)
          const int k0 = m0 + tb * kBK;
          const uint32_t sidx_b = si_s + 4u * (uint32_t)(tb * kBK * 9);
          if (j < 9) {
            const uint32_t halo = x_win(slot);
            const int mi = lane >> 3;
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
              const int c16 = cq + 16 * sub;
              uint32_t R[16];
              bool far = false, bad = false;
              const int chunk = (c16 >> 3) + (mi & 1);
#pragma unroll
              for (int k4 = 0; k4 < 4; ++k4) {
                const int tk = 16 * k4 + 8 * (mi >> 1) + (lane & 7);
                const int raw = ld_shared_s32(sidx_b + 4u * (uint32_t)(tk * 9 + j));
                const bool tok_ok = k0 + tk < M;
                bad |= tok_ok & (raw >= M);
                const int x = (tok_ok & (raw < M)) ? raw : -1;
                const int h = x - hlo;
                const bool in_win = (x >= 0) & ((unsigned)h < (unsigned)kConvHaloRows);
                far |= (x >= 0) & !in_win;
                const uint32_t addr =
                    in_win ? halo + (uint32_t)h * 128u + ((uint32_t)(chunk ^ (h & 7)) << 4) : zero_row;
                ldmatrix_x4_trans(addr, R[4 * k4], R[4 * k4 + 1], R[4 * k4 + 2], R[4 * k4 + 3]);
              }
              if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(err, SVCONV_STATUS_BAD_INDEX);
              if (__any_sync(0xffffffffu, far)) {
                Regs16 rr;
#pragma unroll
                for (int r2 = 0; r2 < 16; ++r2) rr.v[r2] = R[r2];
                rr = wgrad_patch_far(rr, sidx_b, X16, M, 64, k0, hlo, j, c16, kConvHaloRows);
#pragma unroll
                for (int r2 = 0; r2 < 16; ++r2) R[r2] = rr.v[r2];
              }
              tmem_st_16x128b_x8(a_col + ((uint32_t)(32 * quarter + 16 * sub) << 16), R);
            }
          } else {
            // row 0 of the extra half is 1 for every valid token: its accumulator row is db
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
              uint32_t R[16];
#pragma unroll
              for (int r2 = 0; r2 < 16; ++r2) R[r2] = 0u;
              if ((quarter & 1) == 0 && sub == 0 && lane < 4) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                  const int tk = k0 + 8 * k + 2 * lane;
                  R[2 * k] = (tk < M ? 0x3F80u : 0u) | (tk + 1 < M ? 0x3F800000u : 0u);
                }
              }
              tmem_st_16x128b_x8(a_col + ((uint32_t)(32 * quarter + 16 * sub) << 16), R);
            }
          }
        }
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(&bar->afull[st]);
      }
      if (aborted) break;
      warp_arrive(&bar->lempty[slot]);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer: 36 + 40 MMAs per tile
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, 64, 0, 1);  // A from tensor memory, B MN-major (W^T and dY)
      const uint64_t bw0 = smem_desc_sw128(smem_u32(sw), 8192, 1024);
      constexpr uint32_t k16 = 2048u >> 4;  // 16 K rows of an MN-major operand per MMA
      bool ok = true;
      if (mbar_wait(&bar->wfull, 0, abort_flag, err, p.timeout_ns)) {
        uint32_t q = 0, ti = 0;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++ti) {
          const int slot = ti & 1;
          if (!mbar_wait(&bar->tempty, (ti & 1u) ^ 1u, abort_flag, err, p.timeout_ns)) break;
          const uint64_t bdy0 = smem_desc_sw128(dy_win(slot) + kConvPad * 128u, 8192, 1024);
          for (int t = 0; t < kFbStagesPerTile; ++t, ++q) {
            const int st = (int)(q % kFbStages);
            if (!mbar_wait(&bar->afull[st], ring_parity(q, kFbStages), abort_flag, err, p.timeout_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t at = tmem_base + kFbACol + (uint32_t)st * kTmemAStageCols;
            if (t < 9) {
              const uint64_t bd = bw0 + (uint64_t)((uint32_t)t * (8192u >> 4));
#pragma unroll
              for (int k = 0; k < 4; ++k)
                tc_mma_bf16_ts(tmem_base + kFbDxCol, at + k * 8, bd + (uint64_t)(k * k16), idesc, (t | k) != 0 ? 1u : 0u);
            } else {
              const int mt = (t - 9) >> 1, tb = (t - 9) & 1;
              const uint64_t bd = bdy0 + (uint64_t)((uint32_t)tb * (8192u >> 4));
              const bool first = ti == 0 && tb == 0;  // the CTA's first block of this M-tile overwrites
#pragma unroll
              for (int k = 0; k < 4; ++k)
                tc_mma_bf16_ts(tmem_base + (uint32_t)mt * 64u, at + k * 8, bd + (uint64_t)(k * k16), idesc,
                               (first && k == 0) ? 0u : 1u);
            }
            tc_commit(&bar->aempty[st]);
            if (t == 8) tc_commit(&bar->tfull);
          }
          if (ok) tc_commit(&bar->lempty[slot]);  // the dW MMAs have read this slot's dY window
        }
      }
      // every issued MMA (the weight-gradient accumulators in particular) is complete before
      // the epilogue reads them and before tensor memory is released
      tc_commit(&bar->dwfull);
      volatile int never = 0;
      mbar_wait(&bar->dwfull, 0, &never, err, p.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-3)
    uint32_t ti = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++ti) {
      if (!warp_wait(&bar->tfull, ti & 1u, abort_flag, err, p.timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int row = tile * kBM + warp * 32 + lane;
      uint32_t v[2][32];
      const uint32_t acc = tmem_base + ((uint32_t)(warp * 32) << 16) + kFbDxCol;
      tmem_ld_32x32b_x32(acc, v[0]);
      tmem_ld_32x32b_x32(acc + 32, v[1]);
      tmem_ld_wait();
      tc_fence_before();
      warp_arrive(&bar->tempty);
      if (row < M) {
        uint32_t packed[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int hh = e >> 4, c = (e & 15) * 2;
          const __nv_bfloat162 h2 =
              __floats2bfloat162_rn(__uint_as_float(v[hh][c]), __uint_as_float(v[hh][c + 1]));
          packed[e] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        uint4* op = reinterpret_cast<uint4*>(p.dX + (size_t)row * 64);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          op[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
      }
    }
    // the CTA's weight-gradient partial: 5 M-tiles x 64 columns, this warp's 32 lanes of each
    if (ok && warp_wait(&bar->dwfull, 0, abort_flag, err, p.timeout_ns)) {
      tc_fence_after();
      float* base = p.partial + (size_t)blockIdx.x * kFbRowsPad * 64;
#pragma unroll 1
      for (int mt = 0; mt < kFbMTiles; ++mt) {
        uint32_t v[2][32];
        const uint32_t acc = tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)mt * 64u;
        tmem_ld_32x32b_x32(acc, v[0]);
        tmem_ld_32x32b_x32(acc + 32, v[1]);
        tmem_ld_wait();
        float4* dst = reinterpret_cast<float4*>(base + (size_t)(mt * kBM + warp * 32 + lane) * 64);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int hh = e >> 3, c = (e & 7) * 4;
          dst[e] = make_float4(__uint_as_float(v[hh][c]), __uint_as_float(v[hh][c + 1]), __uint_as_float(v[hh][c + 2]),
                               __uint_as_float(v[hh][c + 3]));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kFbTmemCols);
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
                      const uint32_t* box, CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides[i];
  auto encode = [&]() {
    return fn(m, dt, (cuuint32_t)rank, const_cast<void*>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  };
  CUresult r = encode();
  if (r != CUDA_SUCCESS) {
    // The encoder needs a current context.  A host thread whose first CUDA work is this call
    // has none yet (device queries do not bind one): bind the current device's primary
    // context to the thread and try once more.
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || cudaSetDevice(d) != cudaSuccess) return false;
    r = encode();
  }
  return r == CUDA_SUCCESS;
}

// rows x cols (bf16, row-major) with a box of box_rows x 64
static bool make_rows_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {cols * 2};
  const uint32_t box[2] = {64u, box_rows};
  return make_tmap(m, base, 2, dims, strides, box);
}

// Stage counts for the dense path (about 220 KB of shared memory).  When all num_kb
// K-blocks of B fit, take that many B stages (B then stays resident across a CTA's tiles
// with the same columns) and as many A stages (2-4) as remain; otherwise up to 4 A stages
// (short latency) and as many B stages (TMA from L2) as fit.
static void pick_stages(int bn, int num_kb, bool epi, bool bias, int* sa, int* sb) {
  const size_t budget = 224 * 1024;
  if (num_kb <= kMaxStages) {
    for (int a = 4; a >= 2; --a) {
      const int b = num_kb < 2 ? 2 : num_kb;
      if (smem_total(conv_geometry(bn, a, b, false, epi, bias)) <= budget) {
        *sa = a;
        *sb = b;
        return;
      }
    }
  }
  for (int a = 4; a >= 2; a -= 2) {
    int b_best = 0;
    for (int b = 2; b <= kMaxStages; ++b) {
      const Geometry g = conv_geometry(bn, a, b, false, epi, bias);
      if (smem_total(g) <= budget) b_best = b;
    }
    if (b_best >= 3 || (a == 2 && b_best >= 2)) {
      *sa = a;
      *sb = b_best;
      return;
    }
  }
  *sa = 2;
  *sb = 2;
}

// grid: CTAs (PAIR: an even number, two per cluster).
// A persistent kernel on clusters of two loops over its tiles, so it gets no more clusters
// than can be resident at once: *grid (CTAs, even) is clamped to twice that number.  Per
// kernel and device the count is queried once for a shared-memory size (host threads may
// launch concurrently).
template <auto kernel>
static cudaError_t clamp_pair_grid(size_t smem, int* grid) {
  static int occ_smem[64], occ_clusters[64];
  static std::mutex occ_mu;
  int d = 0;
  cudaError_t e = cudaGetDevice(&d);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(occ_mu);
  int n = (d >= 0 && d < 64 && occ_smem[d] == (int)smem) ? occ_clusters[d] : 0;
  if (n == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(*grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
    if (e != cudaSuccess) return e;
    if (n < 1) return cudaErrorInvalidConfiguration;
    if (d >= 0 && d < 64) occ_smem[d] = (int)smem, occ_clusters[d] = n;
  }
  if (*grid > 2 * n) *grid = 2 * n;
  return cudaSuccess;
}

template <int BN, bool MIRROR, bool PAIR, bool F8 = false>
static cudaError_t launch_conv_inst(TcConvParams& prm, int grid, cudaStream_t s) {
  const bool a_in_tmem = prm.nbr != nullptr;
  const bool has_bias = prm.bias != nullptr;  // the epilogue warps' bias copies
  constexpr int kBCols = PAIR ? BN / 2 : BN;  // B columns per CTA
  if (a_in_tmem) {
    // A stage s in tensor memory and B stage s in shared memory advance together: as many
    // stages as both the free tensor-memory columns and the shared-memory budget allow
    int sb = 2;
    for (int b = 2; b <= kMaxStages; ++b)
      if (smem_total(conv_geometry(kBCols * kGatherKb, 0, b, true, prm.out_tma != 0, has_bias)) <= 224 * 1024) sb = b;
    prm.stages_a = prm.stages_b = conv_tmem_a_stages(BN) < sb ? conv_tmem_a_stages(BN) : sb;
  } else {
    const int num_kb = prm.taps * (prm.Kc / kBK);
    pick_stages(kBCols, num_kb, prm.out_tma != 0, has_bias, &prm.stages_a, &prm.stages_b);
    if (num_kb > prm.stages_b) {
      // B streams: A stage s and B stage s on one barrier pair, as many stages as fit
      int st = 2;
      for (int b = 2; b <= kMaxStages; ++b)
        if (smem_total(conv_geometry(kBCols, b, b, false, prm.out_tma != 0, has_bias)) <= 224 * 1024) st = b;
      prm.stages_a = prm.stages_b = st;
      prm.dense_pair_ring = 1;
    }
  }
  // (the same geometry the kernel carves: gather B stages hold kGatherKb K-blocks)
  const size_t smem = smem_total(conv_geometry(a_in_tmem ? kBCols * kGatherKb : kBCols, prm.stages_a, prm.stages_b,
                                               a_in_tmem, prm.out_tma != 0, has_bias));
  static int done[64];
  cudaError_t e = ensure_smem_attr(tc_conv_kernel<BN, MIRROR, PAIR, F8>, smem, done);
  if (e != cudaSuccess) return e;
  if constexpr (PAIR) {
    e = clamp_pair_grid<tc_conv_kernel<BN, MIRROR, PAIR, F8>>(smem, &grid);
    if (e != cudaSuccess) return e;
    return launch_pdl_cluster(tc_conv_kernel<BN, MIRROR, PAIR, F8>, dim3(grid), dim3(kThreads), smem, s, 2u, prm);
  } else
    return launch_pdl(tc_conv_kernel<BN, MIRROR, PAIR, F8>, dim3(grid), dim3(kThreads), smem, s, prm);
}

template <bool MIRROR>
static cudaError_t launch_small_inst(const TcConvParams& prm, int grid, cudaStream_t s) {
  const size_t smem = small_smem_bytes();
  static int done[64];
  cudaError_t e = ensure_smem_attr(tc_conv_small_kernel<MIRROR>, smem, done);
  if (e != cudaSuccess) return e;
  return launch_pdl(tc_conv_small_kernel<MIRROR>, dim3(grid), dim3(kThreads), smem, s, prm);
}

cudaError_t launch_tc_conv(const TcConvArgs& a, const void* Wt, int w_rows, int w_cols, int bn, cudaStream_t s) {
  TcConvParams prm;
  memset(&prm, 0, sizeof(prm));
  if (a.mirror != a.b_mn_major) return cudaErrorInvalidValue;  // the data gradient pairs both
  // e4m3 operands: the forward gather on CTA pairs only (lda, Kc and w_cols count pairs of
  // e4m3 values, i.e. 2-byte units, so every byte offset below is unchanged)
  if (a.f8 && (a.mirror || !a.nbr || bn != 256 || a.max_ctas == 1)) return cudaErrorInvalidValue;
  if (a.nbr && a.taps != 9) return cudaErrorInvalidValue;
  // A operand: halo boxes of 64 rows (gather) or the 128-row tile itself (dense)
  if (!make_rows_tmap(&prm.tmap_a, a.A, (uint64_t)a.a_rows, (uint64_t)a.lda, a.nbr ? (uint32_t)kHaloBox : (uint32_t)kBM))
    return cudaErrorInvalidValue;
  // 256-column tiles run on CTA pairs (each CTA loads 128 of the B columns) unless the
  // CTA budget is below two
  const bool pair = bn == 256 && a.max_ctas != 1;
  if (!a.b_mn_major) {
    // W viewed as [w_rows][w_cols] (rows = output channels, K contiguous)
    if (!make_rows_tmap(&prm.tmap_b, Wt, (uint64_t)w_rows, (uint64_t)w_cols, (uint32_t)(pair ? bn / 2 : bn)))
      return cudaErrorInvalidValue;
  } else {
    // W [Kc rows (o)][9][N cols (i)]: dims (i, j, o), box (64, 1, 64)
    const uint64_t dims[3] = {(uint64_t)a.N, 9u, (uint64_t)a.Kc};
    const uint64_t strides[2] = {(uint64_t)a.N * 2, (uint64_t)a.N * 9 * 2};
    const uint32_t box[3] = {64u, 1u, 64u};
    if (!make_tmap(&prm.tmap_b, Wt, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  // Output through TMA stores (boxes of 32 rows x 64 columns of out [out_rows][N], row
  // stride ldo); an in-place residual (residual == out) through TMA reduce-adds.  A
  // residual elsewhere keeps the per-thread epilogue.
  if ((!a.residual || a.residual == a.out) && a.N % 64 == 0 && a.out_rows > 0 && (a.ldo * 2) % 16 == 0 &&
      (reinterpret_cast<uintptr_t>(a.out) & 15u) == 0) {
    const uint64_t dims[2] = {(uint64_t)a.N, (uint64_t)a.out_rows};
    const uint64_t strides[1] = {(uint64_t)a.ldo * 2};
    const uint32_t box[2] = {64u, 32u};
    if (make_tmap(&prm.tmap_out, a.out, 2, dims, strides, box)) prm.out_tma = a.residual ? 2 : 1;
  }
  prm.A = static_cast<const __nv_bfloat16*>(a.A);
  prm.nbr = a.nbr;
  prm.row_lo = a.row_lo;
  prm.row_hi = a.row_hi;
  prm.bias = a.bias;
  prm.residual = static_cast<const __nv_bfloat16*>(a.residual);
  prm.out = static_cast<__nv_bfloat16*>(a.out);
  prm.status = a.status ? a.status : device_error_word();
  prm.timeout_ns = kDefaultTimeoutNs;
  prm.lda = a.lda;
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
  if (a.max_ctas > 0 && grid > a.max_ctas) grid = a.max_ctas;
  if (grid > tiles) grid = tiles;
  // 64 gathered channels and 64 output columns, whole-table rows: W-resident small-channel kernel
  if (a.nbr && a.Kc == 64 && a.N == 64 && bn == 64 && !a.row_lo && !a.a_abs && !a.nbr_abs && !a.out_abs && !a.f8)
    return a.mirror ? launch_small_inst<true>(prm, grid, s) : launch_small_inst<false>(prm, grid, s);
  if (pair) {
    // one cluster per 256-row tile, at most one CTA per SM
    const int pair_tiles = ((a.M + 2 * kBM - 1) / (2 * kBM)) * (a.N / bn);
    int clusters = sm_count() / 2;
    if (a.max_ctas > 0 && clusters > a.max_ctas / 2) clusters = a.max_ctas / 2;
    if (clusters > pair_tiles) clusters = pair_tiles;
    if (clusters < 1) clusters = 1;
    if (a.f8) return launch_conv_inst<256, false, true, true>(prm, 2 * clusters, s);
    return a.mirror ? launch_conv_inst<256, true, true>(prm, 2 * clusters, s)
                    : launch_conv_inst<256, false, true>(prm, 2 * clusters, s);
  }
  if (bn == 256)
    return a.mirror ? launch_conv_inst<256, true, false>(prm, grid, s) : launch_conv_inst<256, false, false>(prm, grid, s);
  if (bn == 128)
    return a.mirror ? launch_conv_inst<128, true, false>(prm, grid, s) : launch_conv_inst<128, false, false>(prm, grid, s);
  if (bn == 64)
    return a.mirror ? launch_conv_inst<64, true, false>(prm, grid, s) : launch_conv_inst<64, false, false>(prm, grid, s);
  return cudaErrorInvalidValue;
}

// Single-pass backward at 64 channels: as many CTAs as make every CTA carry the same number
// of tiles (each CTA's partial covers its tiles; fewer CTAs, fewer partials to reduce).
int tc_bwd_small_grid(int n) {
  const int tiles = (n + kBM - 1) / kBM;
  if (tiles <= 0) return 0;
  const int sms = sm_count();
  const int per = (tiles + sms - 1) / sms;
  return (tiles + per - 1) / per;
}

size_t tc_bwd_small_partial_floats(int n) { return (size_t)tc_bwd_small_grid(n) * kFbRowsPad * 64; }

cudaError_t launch_tc_bwd_small(const void* dY, const void* X, const int32_t* nbr, int n, const void* Wt, void* dX,
                                float* partial, float* dW, float* db, cudaStream_t s) {
  const int grid = tc_bwd_small_grid(n);
  if (grid == 0) return cudaSuccess;
  FbParams prm;
  memset(&prm, 0, sizeof(prm));
  if (!make_rows_tmap(&prm.tmap_dy, dY, (uint64_t)n, 64, (uint32_t)kHaloBox) ||
      !make_rows_tmap(&prm.tmap_x, X, (uint64_t)n, 64, (uint32_t)kHaloBox))
    return cudaErrorInvalidValue;
  {
    // W [o][j][i]: dims (i, j, o), box (64, 1, 64): tap j as an MN-major W_j^T
    const uint64_t dims[3] = {64u, 9u, 64u};
    const uint64_t strides[2] = {64u * 2, 64u * 9 * 2};
    const uint32_t box[3] = {64u, 1u, 64u};
    if (!make_tmap(&prm.tmap_w, Wt, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  prm.dY = static_cast<const __nv_bfloat16*>(dY);
  prm.X = static_cast<const __nv_bfloat16*>(X);
  prm.nbr = nbr;
  prm.dX = static_cast<__nv_bfloat16*>(dX);
  prm.partial = partial;
  prm.status = device_error_word();
  prm.timeout_ns = kDefaultTimeoutNs;
  prm.n = n;
  const size_t smem = fb_smem_bytes();
  static int done[64];
  cudaError_t e = ensure_smem_attr(tc_bwd_small_kernel, smem, done);
  if (e != cudaSuccess) return e;
  e = launch_pdl(tc_bwd_small_kernel, dim3(grid), dim3(kThreads), smem, s, prm);
  if (e != cudaSuccess) return e;
  return launch_wgrad_reduce(partial, grid, kFbRowsPad, 64, 64, 1, dW, db, s);
}

static int wgrad_bn(int Cout) { return Cout % 256 == 0 ? 256 : Cout % 128 == 0 ? 128 : 64; }

void tc_wgrad_plan(int n, int Cin, int Cout, int* splits, int* rows_pad, int* bn) {
  tc_wgrad_plan_ctas(n, Cin, Cout, sm_count(), splits, rows_pad, bn);
}

void tc_wgrad_plan_ctas(int n, int Cin, int Cout, int ctas, int* splits, int* rows_pad, int* bn) {
  const int b = wgrad_bn(Cout);
  const int rp = (Cin / kBK) * kWgTiles * kBM;  // 10 half-tiles of 64 rows per 64-channel block
  const int base_units = (rp / kBM) * (Cout / b);
  const int kbt = (n + kBK - 1) / kBK;
  int sp = ctas / base_units;
  if (sp < 1) sp = 1;
  if (sp > kbt) sp = kbt > 0 ? kbt : 1;
  *splits = sp;
  *rows_pad = rp;
  *bn = b;
}

template <int BN, bool PAIR = false>
static cudaError_t launch_wgrad_inst(TcWgradParams& prm, int grid, cudaStream_t s) {
  // partial rows [splits * rows_pad][Cout] fp32 through TMA stores (boxes of 32 rows x 32 columns)
  if ((reinterpret_cast<uintptr_t>(prm.partial) & 15u) == 0 && prm.Cout % 32 == 0) {
    const uint64_t dims[2] = {(uint64_t)prm.Cout, (uint64_t)prm.splits * prm.rows_pad};
    const uint64_t strides[1] = {(uint64_t)prm.Cout * 4};
    const uint32_t box[2] = {32u, 32u};
    prm.part_tma = make_tmap(&prm.tmap_part, prm.partial, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT32) ? 1 : 0;
  }
  prm.stages_b = 2;
  for (int b = 2; b <= kMaxStages; ++b)
    if (smem_total(wgrad_geometry(BN, b, PAIR)) <= 226 * 1024) prm.stages_b = b;
  if constexpr (PAIR) {
    // one ring: A (tensor memory) and dY (shared memory) stages advance together
    if (prm.stages_b > kWgPairStagesMax) prm.stages_b = kWgPairStagesMax;
    prm.stages_a = prm.stages_b;
  } else {
    prm.stages_a = wgrad_a_stages(BN);
    // the issuer checks two stages of each ring before it issues (and releases) either
    if (prm.stages_b < 2) return cudaErrorInvalidConfiguration;
  }
  const size_t smem = smem_total(wgrad_geometry(BN, prm.stages_b, PAIR));
  static int done[64];
  cudaError_t e = ensure_smem_attr(tc_wgrad_kernel<BN, PAIR>, smem, done);
  if (e != cudaSuccess) return e;
  if constexpr (PAIR) {
    e = clamp_pair_grid<tc_wgrad_kernel<BN, PAIR>>(smem, &grid);
    if (e != cudaSuccess) return e;
    return launch_pdl_cluster(tc_wgrad_kernel<BN, PAIR>, dim3(grid), dim3(kThreads), smem, s, 2u, prm);
  } else {
    return launch_pdl(tc_wgrad_kernel<BN, PAIR>, dim3(grid), dim3(kThreads), smem, s, prm);
  }
}

// Grid and instantiation for a plan: 256 columns over an even number of row tiles run on
// CTA pairs (one cluster per pair of row tiles and split), otherwise one CTA per unit.
static cudaError_t launch_wgrad_plan(TcWgradParams& prm, int bn, cudaStream_t s) {
  const int m_tiles = prm.rows_pad / kBM;
  if (bn == 256 && m_tiles % 2 == 0) {
    const int pair_units = (m_tiles / 2) * (prm.Cout / bn) * prm.splits;
    int clusters = sm_count() / 2;
    if (clusters > pair_units) clusters = pair_units;
    if (clusters < 1) clusters = 1;
    return launch_wgrad_inst<256, true>(prm, 2 * clusters, s);
  }
  const int units = m_tiles * (prm.Cout / bn) * prm.splits;
  int grid = sm_count();
  if (grid > units) grid = units;
  if (bn == 256) return launch_wgrad_inst<256>(prm, grid, s);
  if (bn == 128) return launch_wgrad_inst<128>(prm, grid, s);
  return launch_wgrad_inst<64>(prm, grid, s);
}

cudaError_t launch_tc_wgrad(const TcWgradArgs& a, cudaStream_t s) {
  TcWgradParams prm;
  memset(&prm, 0, sizeof(prm));
  int splits, rows_pad, bn;
  tc_wgrad_plan(a.n, a.Cin, a.Cout, &splits, &rows_pad, &bn);
  if (splits != a.splits || rows_pad != a.rows_pad) return cudaErrorInvalidValue;
  if (!make_rows_tmap(&prm.tmap_x, a.X, (uint64_t)a.n, (uint64_t)a.Cin, (uint32_t)kWgHaloRows))
    return cudaErrorInvalidValue;
  if (!make_rows_tmap(&prm.tmap_dy, a.dY, (uint64_t)a.n, (uint64_t)a.Cout, 64u)) return cudaErrorInvalidValue;
  prm.X = static_cast<const __nv_bfloat16*>(a.X);
  prm.nbr = a.nbr;
  prm.partial = a.partial;
  prm.status = device_error_word();
  prm.timeout_ns = kDefaultTimeoutNs;
  prm.n = a.n;
  prm.Cin = a.Cin;
  prm.Cout = a.Cout;
  prm.splits = splits;
  prm.rows_pad = rows_pad;
  return launch_wgrad_plan(prm, bn, s);
}

// Same kernel with a caller-chosen number of token splits (1 <= splits <= token
// blocks); used by the allocation-free entry point, whose scratch is fixed.
cudaError_t launch_tc_wgrad_with_splits(const TcWgradArgs& a, cudaStream_t s) {
  TcWgradParams prm;
  memset(&prm, 0, sizeof(prm));
  int plan_splits, rows_pad, bn;
  tc_wgrad_plan(a.n, a.Cin, a.Cout, &plan_splits, &rows_pad, &bn);
  const int kbt = (a.n + kBK - 1) / kBK;
  if (a.splits < 1 || a.splits > kbt || rows_pad != a.rows_pad) return cudaErrorInvalidValue;
  if (!make_rows_tmap(&prm.tmap_x, a.X, (uint64_t)a.n, (uint64_t)a.Cin, (uint32_t)kWgHaloRows))
    return cudaErrorInvalidValue;
  if (!make_rows_tmap(&prm.tmap_dy, a.dY, (uint64_t)a.n, (uint64_t)a.Cout, 64u)) return cudaErrorInvalidValue;
  prm.X = static_cast<const __nv_bfloat16*>(a.X);
  prm.nbr = a.nbr;
  prm.partial = a.partial;
  prm.status = device_error_word();
  prm.timeout_ns = kDefaultTimeoutNs;
  prm.n = a.n;
  prm.Cin = a.Cin;
  prm.Cout = a.Cout;
  prm.splits = a.splits;
  prm.rows_pad = rows_pad;
  return launch_wgrad_plan(prm, bn, s);
}

cudaError_t launch_timeout_selftest(int32_t* status, uint64_t timeout_ns, cudaStream_t s) {
  timeout_selftest_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace svc

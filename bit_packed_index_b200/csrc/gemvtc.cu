// gemvtc.cu -- batched decode (batch 2..16) on the tcgen05 tensor cores, for
// layers with one 2^16-entry, d = 8 codebook, and for layers whose books fit
// shared memory (at most 2^12 + 2^12 entries, d = 6 or 8), in row or tiled
// index order.
//
// y[b][o] = sum_k x[b][k] * W_hat[o][k] ("VPTQ Guide", section "Step 3";
// "Vector Quantization for LLM Weights in Production", section "1. Prefill vs.
// Decode Bottlenecks": decode at B = 1 to 8 is memory bound; the dequantised
// vectors feed "GEMV / Tensor Core Dot Products").  With a 2^16-entry book
// every index costs one random 16-byte centroid gather from L2, whatever the
// batch; the multiply-adds grow with the batch.  So the products go to the
// tensor cores and the kernel is built to keep the gathers flowing:
//
//  * A CTA owns 128 rows of W (the MMA's M) and a range of the input
//    dimension in steps of 64 (eight vectors, one 128-byte swizzled row of a
//    K-major tile).  Four producer warps, one thread per row, read the row's
//    eight indices of a step and issue eight 16-byte cp.async gathers of the
//    centroids straight into the swizzled A tile: no register staging, three
//    steps of gathers in flight per thread, three CTAs per SM.
//  * x, scaled per batch row by a power of two into fp16 (so no value
//    overflows and the products stay exact), is the N = 16 operand (the batch
//    padded with zero rows), brought in by TMA per step.
//  * One thread issues four tcgen05.mma (M = 128, N = 16, K = 16) per step
//    into a 16-column fp32 accumulator in tensor memory; the producer warps
//    then read it back (tcgen05.ld) and apply y = s[o] * acc * 2^e_b +
//    t[o] * sum_k x[b][k].
//  * Narrow layers split the input dimension across CTAs; fp32 partials go to
//    the workspace and a second kernel adds them in split order.
//  * Every wait is bounded: a wait that runs out records VQ_ERR_TIMEOUT in
//    the workspace's status word and the block drains and ends.
#include <algorithm>
#include <cstdlib>

#include "sm100.cuh"

namespace vqk {
namespace {

using namespace sm100;

constexpr int kTcRows = 128;                     // W rows per CTA (MMA M)
constexpr int kTcN = 16;                         // batch rows (MMA N; zero rows past the batch)
constexpr int kTcK = 64;                         // halves per step: 8 vectors of d = 8
constexpr int kTcATile = kTcRows * kTcK * 2;     // 16 KB
constexpr int kTcXTile = kTcN * kTcK * 2;        // 2 KB
constexpr int kTcStage = kTcATile + kTcXTile;    // 18 KB (a multiple of 1024)
#ifndef VQ_TC_STAGES
#define VQ_TC_STAGES 4
#define VQ_TC_LAG 2
#define VQ_TC_PER_SM 3
#endif
constexpr int kTcStages = VQ_TC_STAGES;
constexpr int kTcLag = VQ_TC_LAG;                // gather steps a producer keeps in flight
constexpr int kTcThreads = 256;                  // warp 0: x loads, warp 1: MMA, warps 4-7: rows
constexpr int kTcProducer0 = 128;
constexpr int kTcSmem = 2048 + kTcStages * kTcStage;   // control block + alignment slack + stages
constexpr int kTcPerSm = VQ_TC_PER_SM;

struct TcCtrl {
  uint64_t full[kTcStages];    // the producers' gathers of a stage landed
  uint64_t xfull[kTcStages];   // the stage's x tile landed (TMA)
  uint64_t empty[kTcStages];
  uint64_t acc;
  uint64_t accf[2];            // small-book kernel: accumulator b complete
  uint64_t acce[2];            //   accumulator b read by the epilogue
  uint64_t xf[16];             //   x ring: tile landed (TMA)
  uint64_t xe[16];             //   x ring: tile consumed by the MMAs
  uint32_t tmem;
  int abort;
};

static_assert(sizeof(TcCtrl) <= 1024, "control block");

struct TcArgs {
  Layer L;
  int num_kt;             // steps of the whole input dimension
  int kt_per_split;
  int batch;
  const float* xe;        // 2^e of each batch row (x' = x * 2^-e)
  const float* xsum;      // sum_k x[b][k]
  void* y;
  vq_dtype yt;
  int64_t ldy;
  float* part;            // [nsplit][batch][N] when the input dimension is split
  int* status;
  long long budget;
  int tiles, nitems;      // small-book kernel: work items (row tile, split), split-major
  int xs;                 // small-book kernel: slots of the x ring
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// The 128 bits holding the eight 16-bit indices of row o for vectors
// 8*kt .. 8*kt+7 (word i: vectors 8kt + 2i and 8kt + 2i + 1).
template <int LAYOUT>
__device__ __forceinline__ uint4 step_words(const Layer& L, int64_t o, int kt) {
  if constexpr (LAYOUT == VQ_IDX_TILE4) {
    // tiles 2kt and 2kt+1, row o's 64-bit record in each (the second tile may
    // lie past the last vector)
    const int ntile = (L.nvec + 3) / 4;
    const uint2 a = __ldg(reinterpret_cast<const uint2*>(L.idx[0] + (2 * kt) * L.rw[0] + 2 * o));
    const uint2 b = 2 * kt + 1 < ntile
                        ? __ldg(reinterpret_cast<const uint2*>(L.idx[0] + (2 * kt + 1) * L.rw[0] + 2 * o))
                        : make_uint2(0u, 0u);
    return make_uint4(a.x, a.y, b.x, b.y);
  } else {
    // 16 bytes of row o (rows are 16-byte aligned and cover every step)
    return __ldg(reinterpret_cast<const uint4*>(L.idx[0] + o * L.rw[0] + 4 * kt));
  }
}

template <int LAYOUT>
__global__ void __launch_bounds__(kTcThreads) gemv_tc_kernel(const __grid_constant__ CUtensorMap xmap, TcArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  TcCtrl* ctrl = reinterpret_cast<TcCtrl*>(base);
  uint8_t* stages = base + 1024;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Layer& L = g.L;
  const int row0 = blockIdx.x * kTcRows;
  const int split = blockIdx.y;
  const int kt0 = split * g.kt_per_split;
  const int nkt = min(g.num_kt, kt0 + g.kt_per_split) - kt0;   // >= 1 by construction
  volatile int* abort_flag = &ctrl->abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&ctrl->full[s], kTcRows / 32);   // one arrival per producer warp
      mbar_init(&ctrl->xfull[s], 1);             // the x load
      mbar_init(&ctrl->empty[s], 1);
    }
    mbar_init(&ctrl->acc, 1);
    ctrl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctrl->tmem, 32);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) tma_prefetch(&xmap);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem;

  if (warp == 0) {
    if (lane == 0) {                                   // x tiles by TMA
      int issued = 0;
      for (int i = 0; i < nkt; ++i) {
        const int s = i % kTcStages;
        const uint32_t ph = (i / kTcStages) & 1;
        if (!bounded_wait(&ctrl->empty[s], ph ^ 1, abort_flag, g.status, g.budget)) break;
        mbar_arrive_expect_tx(&ctrl->xfull[s], kTcXTile);
        tma_load_2d(stages + s * kTcStage + kTcATile, &xmap, &ctrl->xfull[s], (kt0 + i) * kTcK, 0);
        issued = i + 1;
      }
      if (*abort_flag) {   // let loads already in flight land before the block exits
        for (int i = max(0, issued - kTcStages); i < issued; ++i)
          drain_phase(&ctrl->xfull[i % kTcStages], (i / kTcStages) & 1, 4000000000LL);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {                                   // MMA issuer
      const uint32_t idesc = f16_idesc(kTcRows, kTcN);
      int issued = 0;
      for (int i = 0; i < nkt; ++i) {
        const int s = i % kTcStages;
        const uint32_t ph = (i / kTcStages) & 1;
        if (!bounded_wait(&ctrl->full[s], ph, abort_flag, g.status, g.budget)) break;
        if (!bounded_wait(&ctrl->xfull[s], ph, abort_flag, g.status, g.budget)) break;
        fence_proxy_async_smem();                      // gathered rows were written by cp.async
        tc_fence_after();
        const uint32_t a = smem_addr(stages + s * kTcStage);
        const uint32_t b = a + kTcATile;
#pragma unroll
        for (int kk = 0; kk < kTcK / 16; ++kk)
          umma_f16(tmem, sw128_kmajor_desc(a + kk * 32), sw128_kmajor_desc(b + kk * 32), idesc, (i | kk) != 0);
        umma_commit(&ctrl->empty[s]);
        issued = i + 1;
      }
      if (issued > 0) {
        umma_commit(&ctrl->acc);
        // every product issued has finished before tensor memory is freed,
        // even when the epilogue gave up waiting for it
        drain_phase(&ctrl->acc, 0, 4000000000LL);
      }
    }
  } else if (warp >= 4) {
    // Producers: thread r gathers row row0 + r (rows past N repeat row N-1,
    // whose results are never stored).
    const int r = threadIdx.x - kTcProducer0;
    const int64_t o = min(row0 + r, L.n - 1);
    const uint16_t* book = L.book[0];
    int published = 0;
    // the index words of the next three steps are always in flight
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    uint4 w0 = nkt > 0 ? step_words<LAYOUT>(L, o, kt0) : z;
    uint4 w1 = nkt > 1 ? step_words<LAYOUT>(L, o, kt0 + 1) : z;
    uint4 w2 = nkt > 2 ? step_words<LAYOUT>(L, o, kt0 + 2) : z;
    for (int i = 0; i < nkt; ++i) {
      const int s = i % kTcStages;
      const uint32_t ph = (i / kTcStages) & 1;
      // warp-uniform: the warp publishes its steps with one arrival
      if (!__all_sync(0xffffffffu, bounded_wait(&ctrl->empty[s], ph ^ 1, abort_flag, g.status, g.budget))) break;
      const uint32_t wd[4] = {w0.x, w0.y, w0.z, w0.w};
      w0 = w1;
      w1 = w2;
      w2 = i + 3 < nkt ? step_words<LAYOUT>(L, o, kt0 + i + 3) : z;
      uint8_t* at = stages + s * kTcStage;
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const uint32_t f = (wd[v >> 1] >> (16 * (v & 1))) & 0xFFFFu;
        cp_async16(at + sw128_off(r, v), book + static_cast<size_t>(f) * 8);
      }
      cp_async_commit();
      if (i >= kTcLag) {                               // step i - kTcLag has landed: publish it
        cp_async_wait<kTcLag>();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->full[(i - kTcLag) % kTcStages]);
        published = i - kTcLag + 1;
      }
    }
    cp_async_wait<0>();                                // nothing of ours may land after the exit
    fence_proxy_async_smem();
    __syncwarp();
    if (__all_sync(0xffffffffu, !*abort_flag) && lane == 0)
      for (int i = published; i < nkt; ++i) mbar_arrive(&ctrl->full[i % kTcStages]);
    // Epilogue: lane quarter warp & 3, one output row per thread.
    if (bounded_wait(&ctrl->acc, 0, abort_flag, g.status, g.budget)) {
      tc_fence_after();
      uint32_t acc[16];
      tmem_ld16(tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16), acc);
      tmem_wait_ld();
      const int row = row0 + r;
      if (row < L.n) {
        const float sc = L.scale ? h2f(L.scale[row]) : 1.0f;
        const float tb = (L.bias && split == 0) ? h2f(L.bias[row]) : 0.0f;
        const float ob = split == 0 ? out_bias_of(L.ob, row) : 0.0f;
        for (int b = 0; b < g.batch; ++b) {
          const float v = sc * (__uint_as_float(acc[b]) * g.xe[b]) + tb * g.xsum[b] + ob;
          if (g.part) g.part[(static_cast<int64_t>(split) * g.batch + b) * L.n + row] = v;
          else store_out(g.y, g.yt, b * g.ldy + row, v);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
}

// ---------------------------------------------------------------------------
// Small books (the 8B and 405B layers: a 2^12-entry main book plus a 2^4 or
// 2^8 residual, d = 6 or 8).  Both books fit shared memory, so no gather
// leaves the SM: the books are staged once per CTA as 16-byte rows (d = 6
// rows zero-padded to 8 halves), and the producer warps -- two or four
// threads per row, each with its share of a step's eight vectors -- read a vector's two centroids
// from shared memory, add them (one fp16 rounding of c1 + c2, the rounding
// W_hat itself carries) and store the sum into the swizzled A tile.  x' puts
// vector j at columns 8 j .. 8 j + 7 (gemv_tc_prep), so the MMA, the x loads
// and the epilogue are those of the kernel above.
// ---------------------------------------------------------------------------
// Producer threads per row: four in the tiled order (a warp's loads of a
// tile's records are contiguous), two in row order (each thread's index
// words come from its own row, so fewer, longer reads measured faster).
template <int LAYOUT>
struct TsShape {
  static constexpr int per_row = LAYOUT == VQ_IDX_TILE4 ? 4 : 2;
  static constexpr int vpt = 8 / per_row;                  // vectors of a step per producer thread
  static constexpr int producers = kTcRows * per_row;
  static constexpr int threads = kTcProducer0 + producers;   // warps 4..: producers
};
#ifndef VQ_TS_NACC
#define VQ_TS_NACC 4
#endif
constexpr int kTsNacc = VQ_TS_NACC;              // accumulators per item: the K slices of a step alternate
constexpr int kTsTmemCols = 2 * 16 * kTsNacc < 32 ? 32 : 2 * 16 * kTsNacc;
#ifndef VQ_TS_PF
#define VQ_TS_PF 4
#endif
constexpr int kTsPf = VQ_TS_PF;                  // steps of index words a producer keeps in flight
constexpr int kTsMaxEntries = 8192;              // K1 + K2 staged (128 KB)
// The x ring: per slot the step's x tile (2 KB) and, in the tiled order,
// the step's index records of the CTA's 128 rows (two tiles of each book,
// 64 b bytes per tile and book: at most 3 KB), brought in by bulk copies on
// the same barrier.  As many slots as shared memory leaves, 4..12.
constexpr int kTsSlot = 5 * 1024;
constexpr int kTsXsMin = 4, kTsXsMax = 12;
constexpr int kTsFixed = 2048 + kTcStages * kTcATile;   // control, slack, A ring; x ring and books follow

// Words holding the TsShape<LAYOUT>::vpt fields of book m for vectors 8 kt + TsShape<LAYOUT>::vpt p ..
// of row o, and the bit position of the first (fields are b bits, LSB
// first).
template <int LAYOUT>
__device__ __forceinline__ void tcs_words(const Layer& L, int m, int64_t o, int kt, int p, uint32_t (&w)[3],
                                          int& sh) {
  const int b = L.b[m];
  const uint32_t* src;
  int64_t w0, avail;
  if constexpr (LAYOUT == VQ_IDX_TILE4) {
    const int t = 2 * kt + (TsShape<LAYOUT>::vpt * p) / 4;
    if (t >= (L.nvec + 3) / 4) {                     // a tile past the last vector
      w[0] = w[1] = w[2] = 0u;
      sh = 0;
      return;
    }
    const int64_t bit0 = o * 4 * b + ((TsShape<LAYOUT>::vpt * p) % 4) * b;
    src = L.idx[m] + static_cast<int64_t>(t) * L.rw[m];
    w0 = bit0 >> 5;
    sh = static_cast<int>(bit0 & 31);
  } else {
    const int64_t bit0 = static_cast<int64_t>(8 * kt + TsShape<LAYOUT>::vpt * p) * b;
    src = L.idx[m] + o * L.rw[m];
    w0 = bit0 >> 5;
    sh = static_cast<int>(bit0 & 31);
  }
  avail = L.rw[m] - w0;                              // words of the row (tile) left
#pragma unroll
  for (int i = 0; i < 3; ++i) w[i] = i < avail ? __ldg(src + w0 + i) : 0u;
}

__device__ __forceinline__ uint32_t tcs_field(const uint32_t (&w)[3], int bit, uint32_t mask) {
  const int q = bit >> 5, s = bit & 31;
  const uint32_t lo = q == 0 ? w[0] : (q == 1 ? w[1] : w[2]);
  const uint32_t hi = q == 0 ? w[1] : (q == 1 ? w[2] : 0u);
  return __funnelshift_r(lo, hi, s) & mask;
}

__device__ __forceinline__ uint32_t hadd2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Persistent: one CTA per SM stages the books once and takes work items
// (row tile, split) in turn; the stage ring and its phases run on across
// items, and two 16-column accumulators alternate so that the epilogue of
// one item overlaps the products of the next.
template <int LAYOUT>
__global__ void __launch_bounds__(TsShape<LAYOUT>::threads, 1) gemv_tcs_kernel(const __grid_constant__ CUtensorMap xmap, TcArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  TcCtrl* ctrl = reinterpret_cast<TcCtrl*>(base);
  uint8_t* stages = base + 1024;
  uint8_t* xring = stages + kTcStages * kTcATile;   // g.xs slots of kTsSlot bytes
  uint8_t* books = xring + g.xs * kTsSlot;          // [K1][16 B], then [K2][16 B]
  const int xs = g.xs;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Layer& L = g.L;
  // index records of a slot (tiled order): book 1 tiles 0 and 1, then book 2's
  const int rb1 = 64 * L.b[0], rb2 = L.nb == 2 ? 64 * L.b[1] : 0;
  volatile int* abort_flag = &ctrl->abort;
  const int k1 = 1 << L.b[0];
  const int k2 = L.nb == 2 ? 1 << L.b[1] : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&ctrl->full[s], TsShape<LAYOUT>::producers / 32);   // one arrival per producer warp
      mbar_init(&ctrl->xfull[s], 1);             // the x load
      mbar_init(&ctrl->empty[s], 1);
    }
    mbar_init(&ctrl->acc, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctrl->accf[b], 1);
      mbar_init(&ctrl->acce[b], 4);              // the four epilogue warps
    }
    for (int q = 0; q < xs; ++q) {
      mbar_init(&ctrl->xf[q], 1);
      mbar_init(&ctrl->xe[q], 1);
    }
    ctrl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctrl->tmem, kTsTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) tma_prefetch(&xmap);
  // Stage the books: entry k of book m as 8 halves (d of them from the book,
  // zeros after).
  for (int i = threadIdx.x; i < k1 + k2; i += TsShape<LAYOUT>::threads) {
    const int m = i < k1 ? 0 : 1;
    const int k = i - m * k1;
    const uint16_t* c = L.book[m] + static_cast<int64_t>(k) * L.d;
    uint4 v;
    if (L.d == 8) {
      v = __ldg(reinterpret_cast<const uint4*>(c));
    } else {                                         // d = 6: 12 bytes, 4-byte aligned
      const uint32_t* c32 = reinterpret_cast<const uint32_t*>(c);
      v = make_uint4(__ldg(c32), __ldg(c32 + 1), __ldg(c32 + 2), 0u);
    }
    *reinterpret_cast<uint4*>(books + static_cast<size_t>(i) * 16) = v;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem;

  if (warp == 0) {
    if (lane == 0) {                                   // x tiles by TMA
      int gs = 0;                                      // steps issued over all items
      bool stop = false;
      for (int item = blockIdx.x; item < g.nitems && !stop; item += gridDim.x) {
        const int kt0 = (item / g.tiles) * g.kt_per_split;
        const int nkt = min(g.num_kt, kt0 + g.kt_per_split) - kt0;
        const int row0 = (item % g.tiles) * kTcRows;
        for (int i = 0; i < nkt; ++i, ++gs) {
          const int q = gs % xs;
          const uint32_t ph = (gs / xs) & 1;
          if (!bounded_wait(&ctrl->xe[q], ph ^ 1, abort_flag, g.status, g.budget)) {
            stop = true;
            break;
          }
          uint8_t* slot = xring + q * kTsSlot;
          // the records of tiles 2 kt and 2 kt + 1 for rows row0 .. row0+127
          // (fewer bytes at the end of a tile; none past the last tile)
          uint32_t bytes[2][2] = {{0u, 0u}, {0u, 0u}};
          const uint32_t* src[2][2] = {{nullptr, nullptr}, {nullptr, nullptr}};
          if (LAYOUT == VQ_IDX_TILE4) {
            const int ntile = (L.nvec + 3) / 4;
#pragma unroll
            for (int m = 0; m < 2; ++m) {
              if (m >= L.nb) break;
              const int64_t off = static_cast<int64_t>(row0) * L.b[m] / 8;   // words before row0's record
              const int64_t avail = (L.rw[m] - off) * 4;
#pragma unroll
              for (int tt = 0; tt < 2; ++tt) {
                const int t = 2 * (kt0 + i) + tt;
                if (t >= ntile) continue;
                bytes[m][tt] = static_cast<uint32_t>(avail < 64 * L.b[m] ? avail : 64 * L.b[m]);
                src[m][tt] = L.idx[m] + static_cast<int64_t>(t) * L.rw[m] + off;
              }
            }
          }
          mbar_arrive_expect_tx(&ctrl->xf[q], kTcXTile + bytes[0][0] + bytes[0][1] + bytes[1][0] + bytes[1][1]);
          tma_load_2d(slot, &xmap, &ctrl->xf[q], (kt0 + i) * kTcK, 0);
#pragma unroll
          for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int tt = 0; tt < 2; ++tt)
              if (bytes[m][tt])
                bulk_load(slot + kTcXTile + (m == 0 ? tt * rb1 : 2 * rb1 + tt * rb2), src[m][tt], bytes[m][tt],
                          &ctrl->xf[q]);
        }
      }
      if (*abort_flag) {   // let loads already in flight land before the block exits
        for (int i = max(0, gs - xs); i < gs; ++i)
          drain_phase(&ctrl->xf[i % xs], (i / xs) & 1, 4000000000LL);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {                                   // MMA issuer
      const uint32_t idesc = f16_idesc(kTcRows, kTcN);
      int gs = 0, it = 0;
      bool any = false, stop = false;
      for (int item = blockIdx.x; item < g.nitems && !stop; item += gridDim.x, ++it) {
        const int kt0 = (item / g.tiles) * g.kt_per_split;
        const int nkt = min(g.num_kt, kt0 + g.kt_per_split) - kt0;
        const int buf = it & 1;
        // the epilogue has read what this accumulator held two items ago
        if (it >= 2 && !bounded_wait(&ctrl->acce[buf], ((it >> 1) & 1) ^ 1, abort_flag, g.status, g.budget))
          break;
        tc_fence_after();
        for (int i = 0; i < nkt; ++i, ++gs) {
          const int s = gs % kTcStages;
          const uint32_t ph = (gs / kTcStages) & 1;
          const int xq = gs % xs;
          if (!bounded_wait(&ctrl->full[s], ph, abort_flag, g.status, g.budget) ||
              !bounded_wait(&ctrl->xf[xq], (gs / xs) & 1, abort_flag, g.status, g.budget)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_addr(stages + s * kTcATile);
          const uint32_t b = smem_addr(xring + xq * kTsSlot);
          // consecutive products go to different accumulators, so none waits
          // for the previous one to finish accumulating
#pragma unroll
          for (int kk = 0; kk < kTcK / 16; ++kk)
            umma_f16(tmem + 16 * (kTsNacc * buf + kk % kTsNacc), sw128_kmajor_desc(a + kk * 32),
                     sw128_kmajor_desc(b + kk * 32), idesc, (i != 0) || (kk >= kTsNacc));
          umma_commit(&ctrl->empty[s]);
          umma_commit(&ctrl->xe[xq]);
          any = true;
        }
        if (!stop) umma_commit(&ctrl->accf[buf]);
      }
      if (any) {
        // every product issued has finished before tensor memory is freed
        umma_commit(&ctrl->acc);
        drain_phase(&ctrl->acc, 0, 4000000000LL);
      }
    }
  } else if (warp >= 4) {
    // Producers: thread (r, p) builds vectors TsShape<LAYOUT>::vpt p .. of each step of
    // row row0 + r (rows past N repeat row N-1, whose results are never
    // stored); warps 4-7 (p = 0) then run the item's epilogue.
    const int pr = threadIdx.x - kTcProducer0;
    const int r = pr & (kTcRows - 1), p = pr >> 7;
    const uint32_t m1 = (1u << L.b[0]) - 1u, m2 = L.nb == 2 ? (1u << L.b[1]) - 1u : 0u;
    const int b1 = L.b[0], b2 = L.nb == 2 ? L.b[1] : 0;
    const uint8_t* book2 = books + static_cast<size_t>(k1) * 16;
    int gs = 0, it = 0;
    bool stop = false;
    for (int item = blockIdx.x; item < g.nitems && !stop; item += gridDim.x, ++it) {
      const int split = item / g.tiles;
      const int row0 = (item - split * g.tiles) * kTcRows;
      const int kt0 = split * g.kt_per_split;
      const int nkt = min(g.num_kt, kt0 + g.kt_per_split) - kt0;
      const int64_t o = min(row0 + r, L.n - 1);
      // Row order: index words of the next kTsPf steps in flight in
      // registers (a window that slides by one step per iteration).  Tiled
      // order: the step's records arrive with x in the x ring (bulk copies).
      constexpr bool kRec = LAYOUT == VQ_IDX_TILE4;
      constexpr int PF = kRec ? 1 : kTsPf;
      constexpr int VPT = TsShape<LAYOUT>::vpt;
      uint32_t pw[PF][2][3];
      int psh[PF][2];
#pragma unroll
      for (int q = 0; q < PF; ++q) {
        pw[q][0][0] = pw[q][0][1] = pw[q][0][2] = 0u;
        pw[q][1][0] = pw[q][1][1] = pw[q][1][2] = 0u;
        psh[q][0] = psh[q][1] = 0;
        if (!kRec && q < nkt) {
          tcs_words<LAYOUT>(L, 0, o, kt0 + q, p, pw[q][0], psh[q][0]);
          if (L.nb == 2) tcs_words<LAYOUT>(L, 1, o, kt0 + q, p, pw[q][1], psh[q][1]);
        }
      }
      for (int i = 0; i < nkt; ++i, ++gs) {
        const int s = gs % kTcStages;
        const uint32_t ph = (gs / kTcStages) & 1;
        uint32_t f1[VPT], f2[VPT];
        if constexpr (kRec) {
          const int q = gs % xs;
          if (!__all_sync(0xffffffffu, bounded_wait(&ctrl->xf[q], (gs / xs) & 1, abort_flag, g.status, g.budget))) {
            stop = true;
            break;
          }
          // this thread's VPT fields of row r: tile (VPT p) / 4 of the step,
          // starting at field (VPT p) % 4 of the row's record
          const uint8_t* slot = xring + q * kTsSlot + kTcXTile;
          const int tt = (VPT * p) >> 2, f0 = (VPT * p) & 3;
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            if (m == 1 && L.nb != 2) break;
            const int bm = m == 0 ? b1 : b2;
            const uint32_t* rec =
                reinterpret_cast<const uint32_t*>(slot + (m == 0 ? tt * rb1 : 2 * rb1 + tt * rb2));
            const int bit = r * 4 * bm + f0 * bm;
            uint32_t w3[3];
            w3[0] = rec[bit >> 5];
            w3[1] = (bit & 31) + VPT * bm > 32 ? rec[(bit >> 5) + 1] : 0u;
            w3[2] = 0u;
#pragma unroll
            for (int v = 0; v < VPT; ++v) {
              const uint32_t f = tcs_field(w3, (bit & 31) + v * bm, m == 0 ? m1 : m2);
              if (m == 0) f1[v] = f;
              else f2[v] = f;
            }
          }
          if (L.nb != 2) {
#pragma unroll
            for (int v = 0; v < VPT; ++v) f2[v] = 0u;
          }
        } else {
#pragma unroll
          for (int v = 0; v < VPT; ++v) {
            f1[v] = tcs_field(pw[0][0], psh[0][0] + v * b1, m1);
            f2[v] = L.nb == 2 ? tcs_field(pw[0][1], psh[0][1] + v * b2, m2) : 0u;
          }
#pragma unroll
          for (int q = 0; q + 1 < PF; ++q) {
#pragma unroll
            for (int m = 0; m < 2; ++m) {
              pw[q][m][0] = pw[q + 1][m][0];
              pw[q][m][1] = pw[q + 1][m][1];
              pw[q][m][2] = pw[q + 1][m][2];
              psh[q][m] = psh[q + 1][m];
            }
          }
          if (i + PF < nkt) {
            tcs_words<LAYOUT>(L, 0, o, kt0 + i + PF, p, pw[PF - 1][0], psh[PF - 1][0]);
            if (L.nb == 2) tcs_words<LAYOUT>(L, 1, o, kt0 + i + PF, p, pw[PF - 1][1], psh[PF - 1][1]);
          }
        }
        uint4 c[TsShape<LAYOUT>::vpt];
#pragma unroll
        for (int v = 0; v < TsShape<LAYOUT>::vpt; ++v) {
          c[v] = *reinterpret_cast<const uint4*>(books + static_cast<size_t>(f1[v]) * 16);
          if (L.nb == 2) {
            const uint4 c2 = *reinterpret_cast<const uint4*>(book2 + static_cast<size_t>(f2[v]) * 16);
            c[v] = make_uint4(hadd2_u32(c[v].x, c2.x), hadd2_u32(c[v].y, c2.y), hadd2_u32(c[v].z, c2.z),
                              hadd2_u32(c[v].w, c2.w));
          }
        }
        // warp-uniform: the warp publishes its rows of a step with one arrival
        if (!__all_sync(0xffffffffu, bounded_wait(&ctrl->empty[s], ph ^ 1, abort_flag, g.status, g.budget))) {
          stop = true;
          break;
        }
        uint8_t* at = stages + s * kTcATile;
#pragma unroll
        for (int v = 0; v < TsShape<LAYOUT>::vpt; ++v) *reinterpret_cast<uint4*>(at + sw128_off(r, TsShape<LAYOUT>::vpt * p + v)) = c[v];
        fence_proxy_async_smem();                      // visible to the tensor cores
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->full[s]);
      }
      if (stop || p != 0) continue;
      // Epilogue (warps 4-7): lane quarter warp & 3, one output row per thread.
      const int buf = it & 1;
      if (!__all_sync(0xffffffffu, bounded_wait(&ctrl->accf[buf], (it >> 1) & 1, abort_flag, g.status, g.budget))) {
        stop = true;
        continue;
      }
      tc_fence_after();
      uint32_t acc[16];
      float accs[16];
      tmem_ld16(tmem + 16 * kTsNacc * buf + (static_cast<uint32_t>(32 * (warp & 3)) << 16), acc);
      tmem_wait_ld();
#pragma unroll
      for (int b = 0; b < 16; ++b) accs[b] = __uint_as_float(acc[b]);
#pragma unroll
      for (int q = 1; q < kTsNacc; ++q) {
        tmem_ld16(tmem + 16 * (kTsNacc * buf + q) + (static_cast<uint32_t>(32 * (warp & 3)) << 16), acc);
        tmem_wait_ld();
#pragma unroll
        for (int b = 0; b < 16; ++b) accs[b] += __uint_as_float(acc[b]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->acce[buf]);
      const int row = row0 + r;
      if (row < L.n) {
        const float sc = L.scale ? h2f(L.scale[row]) : 1.0f;
        const float tb = (L.bias && split == 0) ? h2f(L.bias[row]) : 0.0f;
        const float ob = split == 0 ? out_bias_of(L.ob, row) : 0.0f;
#pragma unroll
        for (int b = 0; b < kTcN; ++b) {
          if (b < g.batch) {
            const float v = sc * (accs[b] * g.xe[b]) + tb * g.xsum[b] + ob;
            if (g.part) g.part[(static_cast<int64_t>(split) * g.batch + b) * L.n + row] = v;
            else store_out(g.y, g.yt, b * g.ldy + row, v);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTsTmemCols);
  }
}

// x' = x * 2^-e_b in fp16 [16][kp] (zero past kin and for rows b >= batch),
// 2^e_b and sum_k x[b][k].  e_b puts max_k |x[b][k]| in [2^14, 2^15), so no
// value overflows fp16 and values above max * 2^-29 stay exact.  x' holds
// vector j of the layer (d elements) at columns 8 j .. 8 j + d - 1 and zeros
// in the rest of its 8 columns (d = 8: x' is x itself, scaled).
// Grid (16, kPrepChunks): every block of row b reads the whole row for its
// maximum and sum (the same order in each, so the same result), then writes
// its share of the row's columns, 8 at a time; block (b, 0) stores 2^e_b and
// the sum.  vec: x is 16-byte aligned with ldx a multiple of 8.
constexpr int kPrepChunks = 8;

__global__ void __launch_bounds__(256) gemv_tc_prep(const uint16_t* __restrict__ x, int x_fp16, int64_t ldx,
                                                    int kin, int kp, int batch, int d, int vec,
                                                    uint16_t* __restrict__ xh, float* __restrict__ xe,
                                                    float* __restrict__ xsum) {
  __shared__ float s_max[8], s_sum[8];
  const int b = blockIdx.x, c = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool live = b < batch;
  const uint16_t* xr = x + static_cast<int64_t>(b) * ldx;
  auto val = [&](uint16_t u) { return x_fp16 ? h2f(u) : bf2f(u); };
  float mx = 0.0f, sm = 0.0f;
  if (live) {
    if (vec) {
      for (int k = 8 * tid; k < kin; k += 8 * 256) {
        if (k + 8 <= kin) {
          const uint4 q = __ldg(reinterpret_cast<const uint4*>(xr + k));
          const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float lo = val(static_cast<uint16_t>(w[i] & 0xFFFFu)), hi = val(static_cast<uint16_t>(w[i] >> 16));
            mx = fmaxf(mx, fmaxf(fabsf(lo), fabsf(hi)));
            sm += lo;
            sm += hi;
          }
        } else {
          for (int i = k; i < kin; ++i) {
            const float v = val(xr[i]);
            mx = fmaxf(mx, fabsf(v));
            sm += v;
          }
        }
      }
    } else {
      for (int k = tid; k < kin; k += 256) {
        const float v = val(xr[k]);
        mx = fmaxf(mx, fabsf(v));
        sm += v;
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    sm += __shfl_xor_sync(0xffffffffu, sm, off);
  }
  if (lane == 0) { s_max[warp] = mx; s_sum[warp] = sm; }
  __syncthreads();
  mx = 0.0f;
  sm = 0.0f;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    mx = fmaxf(mx, s_max[w]);
    sm += s_sum[w];
  }
  // max = m * 2^E with 0.5 <= m < 1; e = E - 15, kept in [-126, 127] (values
  // below 2^-111 scale to fp16 subnormals or zero).
  int e = 0;
  if (mx > 0.0f && mx < INFINITY) e = max(-126, min(127, static_cast<int>(__float_as_uint(mx) >> 23) - 126 - 15));
  const float f1 = __uint_as_float(static_cast<uint32_t>(127 - e / 2) << 23);
  const float f2 = __uint_as_float(static_cast<uint32_t>(127 - (e - e / 2)) << 23);
  // this block's columns: groups of 8 (one vector of the layer each)
  const int ngroups = kp / 8;
  const int g0 = c * ngroups / kPrepChunks, g1 = (c + 1) * ngroups / kPrepChunks;
  for (int g = g0 + tid; g < g1; g += 256) {
    uint32_t h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v2[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int e8 = 2 * i + q;
        const int src = g * d + e8;                  // element of x in column 8 g + e8
        v2[q] = (live && e8 < d && src < kin) ? val(xr[src]) * f1 * f2 : 0.0f;
      }
      h[i] = f2h(v2[0]) | (static_cast<uint32_t>(f2h(v2[1])) << 16);
    }
    *reinterpret_cast<uint4*>(xh + static_cast<int64_t>(b) * kp + 8 * g) = make_uint4(h[0], h[1], h[2], h[3]);
  }
  if (c == 0 && tid == 0) {
    xe[b] = live ? __uint_as_float(static_cast<uint32_t>(127 + e) << 23) : 0.0f;
    xsum[b] = live ? sm : 0.0f;
  }
}

// y[b][o] = sum over splits of part[s][b][o], in split order.
__global__ void gemv_tc_finalize(const float* __restrict__ part, int nsplit, int batch, int n, void* __restrict__ y,
                                 vq_dtype yt, int64_t ldy) {
  const int64_t total = static_cast<int64_t>(batch) * n;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = i / n, o = i - b * n;
    float v = 0.0f;
    for (int s = 0; s < nsplit; ++s) v += part[(s * static_cast<int64_t>(batch) + b) * n + o];
    store_out(y, yt, b * ldy + o, v);
  }
}

struct TcLayout {
  int tiles, nsplit, kt_per_split, num_kt, kp;
  size_t off_status, off_xh, off_xe, off_part, total;
};

// The 2^16-book kernel runs three CTAs per SM and splits the input dimension
// so that the grid fills about one wave of them; the small-book kernel runs
// one CTA per SM and picks the split (up to 8) that wastes the least of the
// last wave.
TcLayout tc_layout(const Layer& L, int batch, bool small) {
  TcLayout t{};
  t.tiles = (L.n + kTcRows - 1) / kTcRows;
  t.num_kt = (L.nvec + 7) / 8;
  t.kp = t.num_kt * kTcK;
  int nsplit = 1;
  if (!small) {
    const int target = kTcPerSm * device_sm_count();
    nsplit = std::max(1, std::min(t.num_kt, (target + t.tiles / 2) / t.tiles));
  } else {
    const int sms = device_sm_count();
    double best = -1.0;
    for (int ns = 1; ns <= std::min(8, t.num_kt); ++ns) {
      const int64_t ctas = static_cast<int64_t>(t.tiles) * ns;
      const int64_t waves = (ctas + sms - 1) / sms;
      const double score = static_cast<double>(ctas) / static_cast<double>(waves * sms) - 0.005 * (ns - 1);
      if (score > best + 1e-9) {
        best = score;
        nsplit = ns;
      }
    }
  }
  t.kt_per_split = (t.num_kt + nsplit - 1) / nsplit;
  t.nsplit = (t.num_kt + t.kt_per_split - 1) / t.kt_per_split;
  auto r256 = [](size_t b) { return (b + 255) / 256 * 256; };
  t.off_status = 0;
  t.off_xh = 256;
  t.off_xe = t.off_xh + r256(static_cast<size_t>(kTcN) * t.kp * 2);
  t.off_part = t.off_xe + 256;
  t.total = t.off_part + (t.nsplit > 1 ? r256(static_cast<size_t>(t.nsplit) * batch * L.n * 4) : 0);
  return t;
}

// Smallest batch the kernels serve (VQ_TC_MIN_BATCH and VQ_TCS_MIN_BATCH
// override, for measurements).
int tc_min_batch() {
  if (const char* env = std::getenv("VQ_TC_MIN_BATCH")) return std::atoi(env);
  return 2;
}
int tcs_min_batch() {
  if (const char* env = std::getenv("VQ_TCS_MIN_BATCH")) return std::atoi(env);
  return 3;
}

bool tcs_supported(const Layer& L) {
  if (!(L.d == 6 || L.d == 8) || L.b[0] > 12 || (L.nb == 2 && L.b[1] > 12)) return false;
  return (1 << L.b[0]) + (L.nb == 2 ? 1 << L.b[1] : 0) <= kTsMaxEntries;
}
// x-ring slots that fit beside the books (0 when fewer than kTsXsMin do).
int tcs_slots(const Layer& L) {
  const int books = ((1 << L.b[0]) + (L.nb == 2 ? 1 << L.b[1] : 0)) * 16;
  const int room = device_smem_optin() - kTsFixed - books;
  const int xs = std::min(kTsXsMax, room / kTsSlot);
  return xs >= kTsXsMin ? xs : 0;
}
int tcs_smem(const Layer& L) {
  return kTsFixed + tcs_slots(L) * kTsSlot + ((1 << L.b[0]) + (L.nb == 2 ? 1 << L.b[1] : 0)) * 16;
}

long long tc_wait_budget() {
  if (const char* env = std::getenv("VQ_WAIT_BUDGET")) return std::atoll(env);
  return 4000000000LL;
}

}  // namespace

bool plan_gemv_tc(const Layer& L, int batch, size_t ws_cap, GemvPlan* p) {
  if (!(L.layout == VQ_IDX_ROWS || L.layout == VQ_IDX_TILE4) || L.n < 1 || L.nvec < 1 || batch > kTcN) return false;
  const bool big = L.nb == 1 && L.d == 8 && L.b[0] == 16;
  const bool small = !big && tcs_supported(L) && tcs_slots(L) > 0;
  if (!big && !small) return false;
  if (batch < std::max(1, big ? tc_min_batch() : tcs_min_batch())) return false;
  const int smem = big ? kTcSmem : tcs_smem(L);
  if (device_smem_optin() < smem) return false;
  const TcLayout t = tc_layout(L, batch, small);
  if (t.total > ws_cap) return false;
  *p = GemvPlan{};
  p->fast = big ? 7 : 8;
  p->bt = batch;
  p->nsplit = t.nsplit;
  p->grid_x = t.tiles;
  p->smem = smem;
  p->ws_bytes = t.total;
  return true;
}

vq_status launch_gemv_tc(const Layer& L, const GemvPlan& p, const void* x, bool x_fp16, int batch, int64_t ldx,
                         void* y, vq_dtype yt, int64_t ldy, void* ws, cudaStream_t stream) {
  const bool small = p.fast == 8;
  const TcLayout t = tc_layout(L, batch, small);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* xh = reinterpret_cast<uint16_t*>(w + t.off_xh);
  float* xe = reinterpret_cast<float*>(w + t.off_xe);
  float* xsum = xe + kTcN;
  int* status = reinterpret_cast<int*>(w + t.off_status);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), stream);
  if (e != cudaSuccess) return cuda_status(e);
  count_launch();
  const int vec = aligned(x, 16) && ldx % 8 == 0;
  gemv_tc_prep<<<dim3(kTcN, kPrepChunks), 256, 0, stream>>>(static_cast<const uint16_t*>(x), x_fp16 ? 1 : 0, ldx,
                                                            L.kin, t.kp, batch, L.d, vec, xh, xe, xsum);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  CUtensorMap xmap;
  if (!make_map_f16_sw128(&xmap, xh, t.kp, kTcN, t.kp, kTcN)) return VQ_ERR_CUDA;
  TcArgs g{};
  g.L = L;
  g.num_kt = t.num_kt;
  g.kt_per_split = t.kt_per_split;
  g.batch = batch;
  g.xe = xe;
  g.xsum = xsum;
  g.y = y;
  g.yt = yt;
  g.ldy = ldy;
  g.part = t.nsplit > 1 ? reinterpret_cast<float*>(w + t.off_part) : nullptr;
  g.status = status;
  g.budget = tc_wait_budget();
  auto k = small ? (L.layout == VQ_IDX_TILE4 ? gemv_tcs_kernel<VQ_IDX_TILE4> : gemv_tcs_kernel<VQ_IDX_ROWS>)
                 : (L.layout == VQ_IDX_TILE4 ? gemv_tc_kernel<VQ_IDX_TILE4> : gemv_tc_kernel<VQ_IDX_ROWS>);
  const int threads = small ? (L.layout == VQ_IDX_TILE4 ? TsShape<VQ_IDX_TILE4>::threads
                                                      : TsShape<VQ_IDX_ROWS>::threads)
                            : kTcThreads;
  if ((e = set_func_attr(reinterpret_cast<const void*>(k), cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem)) != cudaSuccess)
    return cuda_status(e);
  g.tiles = t.tiles;
  g.nitems = t.tiles * t.nsplit;
  g.xs = small ? tcs_slots(L) : 0;
  const dim3 grid = small ? dim3(std::min(g.nitems, device_sm_count())) : dim3(t.tiles, t.nsplit);
  count_launch();
  k<<<grid, threads, p.smem, stream>>>(xmap, g);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  if (t.nsplit > 1) {
    const int64_t total = static_cast<int64_t>(batch) * L.n;
    const int grid = static_cast<int>(std::min<int64_t>((total + 255) / 256, 4LL * device_sm_count()));
    count_launch();
    gemv_tc_finalize<<<grid, 256, 0, stream>>>(g.part, t.nsplit, batch, L.n, y, yt, ldy);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  return VQ_OK;
}

}  // namespace vqk

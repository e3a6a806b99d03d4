// gemm.cu -- vq_gemm: prefill y = x . W_hat^T on the tcgen05 tensor cores.
//
// The pages place prefill in the compute-bound regime, where table lookups
// compete with the matrix multiply ("Vector Quantization for LLM Weights in
// Production", section "1. Prefill vs. Decode Bottlenecks"; its dequantisation
// diagram feeds dequantised fp16/bf16 vectors to "GEMV / Tensor Core Dot
// Products").  The B200 design:
//
//  * One CTA per 128 x 256 output tile, K in steps of 64 (fp16 operands, 128-
//    byte rows, 128-byte swizzle), a multi-stage shared-memory pipeline driven
//    by mbarriers, one elected thread issuing tcgen05.mma (M=128, N=256, K=16)
//    into an fp32 accumulator in tensor memory, and a tcgen05.ld epilogue.
//  * A tiles (activations) arrive by TMA from an fp16 copy of x that a small
//    pre-pass writes into the workspace, together with the row sums of x.
//    bf16 -> fp16 is exact for |x| in [2^-14, 65504].
//  * B tiles (weights) come from one of two sources:
//      - fused: eight producer warps unpack the index streams, gather the
//        centroids (shared memory for small books, L1/L2 for 2^16-entry
//        books), add the residual centroid in fp16 and write the swizzled
//        tile directly; W_hat never reaches global memory.  Scale and bias
//        are applied in the epilogue: y = s[n] * acc + t[n] * sum_k x[m][k].
//      - staged: vq_dequant writes W_hat (fp16, bit-exact) into the
//        workspace once and TMA streams its tiles; the epilogue is y = acc.
//    Each W_hat element costs one centroid gather per 128 rows of x in the
//    fused form but one gather in total in the staged form, so the staged
//    form wins when gathers are served from L2 and M is large.
//  * Every mbarrier wait is bounded; a wait that runs out of budget raises
//    the block's abort flag, records VQ_ERR_TIMEOUT in the workspace's status
//    word and lets every warp fall through to the teardown.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "codebook.cuh"
#include "sm100.cuh"

namespace vqk {
namespace {

using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 64;       // one MMA: M = 128, N <= 256, K = 16
constexpr int kATile = BM * BK * 2;             // 16 KB per 128-row A sub-tile
constexpr int kBTile = BN * BK * 2;             // 32 KB
// A CTA covers MSUB (1 or 2) A sub-tiles of 128 rows that share each B tile:
// two sub-tiles halve the weight-tile bytes (and, fused, the gathers) per FLOP.
__host__ __device__ constexpr int stage_bytes(int msub) { return msub * kATile + kBTile; }
constexpr int kThreads = 384;                   // 12 warps
constexpr int kProducerThread0 = 128;           // warps 4..11 produce B tiles
constexpr int kProducers = 256;
constexpr int kCtrlBytes = 4096;                // barriers, flags, scale/bias staging
constexpr long long kWaitBudget = 4000000000LL; // SM clocks (about 2 s)
constexpr int kMaxStages = 8;

enum Mode { kFused = 0, kStaged = 1 };

struct GemmArgs {
  Layer L;
  int m;
  int num_kt;
  int stages;
  int smem_mask;
  int book_bytes;
  int bn;                 // tile width along N (multiple of 32, <= BN)
  uint32_t idesc;         // tcgen05 instruction descriptor for M = 128, N = bn
  const float* rowsum;
  const float* rowscale;  // 2^e_m of each row of x (its fp16 copy is x * 2^-e_m), or null for 1
  void* y;
  vq_dtype yt;
  int64_t ldy;
  int* status;
  long long budget;       // SM clocks a wait may take (VQ_WAIT_BUDGET overrides about 2 s)
};

// Control block at the start of (1024-aligned) dynamic shared memory.
struct Ctrl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
  float sb[3 * BN];   // per-column scale, bias and output bias of this tile
};
static_assert(sizeof(Ctrl) <= kCtrlBytes, "control block");

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

// Eight consecutive B-bit fields starting at field j0 (a multiple of 8, so
// the first bit is word aligned for B in {4, 8, 12, 16}).  Words past the row
// are read as zero (their fields lie past the last vector and are masked).
template <int B>
__device__ __forceinline__ void fields8(const uint32_t* __restrict__ row, int64_t rw, int j0,
                                        uint32_t (&f)[8]) {
  constexpr int NW = (8 * B) / 32;
  const int64_t w0 = (static_cast<int64_t>(j0) * B) >> 5;
  uint32_t w[NW + 1];
  if (B == 16 && w0 + 4 <= rw) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(row + w0));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if (B == 8 && w0 + 2 <= rw) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(row + w0));
    w[0] = v.x; w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < NW; ++i) w[i] = (w0 + i < rw) ? __ldg(row + w0 + i) : 0u;
  }
  w[NW] = 0u;
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    constexpr uint32_t mask = (1u << B) - 1u;
    const int bit = v * B;
    f[v] = __funnelshift_r(w[bit >> 5], w[(bit >> 5) + 1], bit & 31) & mask;
  }
}

__device__ __forceinline__ uint4 hadd8(uint4 a, uint4 b) {
  uint4 r;
  const __half2* x = reinterpret_cast<const __half2*>(&a);
  const __half2* y = reinterpret_cast<const __half2*>(&b);
  __half2* z = reinterpret_cast<__half2*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) z[i] = __hadd2(x[i], y[i]);
  return r;
}

__device__ __forceinline__ uint4 zero_tail8(uint4 v, int valid) {   // keep `valid` of 8 halves
  uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (2 * i >= valid) w[i] = 0u;
    else if (2 * i + 1 >= valid) w[i] &= 0xFFFFu;
  }
  return v;
}

// Fused B-tile rows at d = 8 with compile-time index widths (B2 = 0: one
// book), split in three steps so a producer can keep the next stage's index
// loads and centroid gathers in flight while it waits for a free stage:
// the 8 index fields of row n for K-step kt, the 8 centroid rows (fp16 sum of
// both books), and the swizzled 16-byte stores into the tile.
template <int B1, int B2>
__device__ __forceinline__ void d8_fields(const Layer& L, int n, int kt, uint32_t (&f1)[8],
                                          uint32_t (&f2)[8]) {
  const int j0 = kt * 8;
  fields8<B1>(L.idx[0] + static_cast<int64_t>(n) * L.rw[0], L.rw[0], j0, f1);
  if constexpr (B2 > 0) fields8<B2>(L.idx[1] + static_cast<int64_t>(n) * L.rw[1], L.rw[1], j0, f2);
}

template <int B2>
__device__ __forceinline__ void d8_gather(const BookView (&bv)[2], const uint32_t (&f1)[8],
                                          const uint32_t (&f2)[8], uint4 (&c)[8]) {
#pragma unroll
  for (int v = 0; v < 8; ++v) c[v] = *reinterpret_cast<const uint4*>(bv[0].base + static_cast<size_t>(f1[v]) * 8);
  if constexpr (B2 > 0) {
#pragma unroll
    for (int v = 0; v < 8; ++v)
      c[v] = hadd8(c[v], *reinterpret_cast<const uint4*>(bv[1].base + static_cast<size_t>(f2[v]) * 8));
  }
}

__device__ __forceinline__ void d8_store(const Layer& L, bool live, int kt, const uint4 (&c)[8],
                                         uint8_t* btile, int r) {
  const int k0 = kt * BK;
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    const int valid = live ? L.kin - (k0 + 8 * v) : 0;
    uint4 x = c[v];
    if (valid < 8) x = zero_tail8(x, valid < 0 ? 0 : valid);
    *reinterpret_cast<uint4*>(btile + sw128_off(r, v)) = x;
  }
}

// Fused B-tile row, any d <= 8 and any index widths.
template <int NB>
__device__ __forceinline__ void produce_row_generic(const Layer& L, const BookView (&bv)[2], int n,
                                                    int kt, uint8_t* btile, int r) {
  const int k0 = kt * BK;
  if (n >= L.n || k0 + BK > L.kin) {
#pragma unroll
    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(btile + sw128_off(r, c)) = make_uint4(0, 0, 0, 0);
    if (n >= L.n) return;
  }
  const int d = L.d;
  const int j_lo = k0 / d;
  const int j_hi = min(L.nvec - 1, (k0 + BK - 1) / d);
  const uint32_t* row0 = L.idx[0] + static_cast<int64_t>(n) * L.rw[0];
  const uint32_t* row1 = L.idx[1] + static_cast<int64_t>(n) * L.rw[1];
  for (int j = j_lo; j <= j_hi; ++j) {
    const uint32_t i1 = load_field(row0, static_cast<int64_t>(j) * L.b[0], L.b[0]);
    const uint16_t* c1 = bv[0].base + static_cast<size_t>(i1) * bv[0].stride;
    const uint16_t* c2 = nullptr;
    if (NB == 2) {
      const uint32_t i2 = load_field(row1, static_cast<int64_t>(j) * L.b[1], L.b[1]);
      c2 = bv[1].base + static_cast<size_t>(i2) * bv[1].stride;
    }
    for (int e = 0; e < d; ++e) {
      const int k = j * d + e;
      if (k < k0 || k >= k0 + BK || k >= L.kin) continue;
      __half h = __ushort_as_half(c1[e]);
      if (NB == 2) h = __hadd(h, __ushort_as_half(c2[e]));
      const int kk = k - k0;
      *reinterpret_cast<__half*>(btile + sw128_off(r, kk >> 3) + (kk & 7) * 2) = h;
    }
  }
}

template <int MODE, int B1, int B2, int MSUB>
__global__ void __launch_bounds__(kThreads, 1)
    vq_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                   const __grid_constant__ CUtensorMap tmap_b, GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem);
  uint8_t* stages = smem + kCtrlBytes + (1024 - kCtrlBytes % 1024) % 1024;
  constexpr int kStage = stage_bytes(MSUB);
  uint16_t* books = reinterpret_cast<uint16_t*>(stages + g.stages * kStage);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t kTmemCols = 256 * MSUB;      // one 256-column fp32 accumulator per sub-tile
  const int bn = g.bn;
  const int m0 = blockIdx.x * BM * MSUB, n0 = blockIdx.y * bn;
  const Layer& L = g.L;
  volatile int* abort_flag = &ctrl->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < g.stages; ++s) {
      mbar_init(&ctrl->full[s], MODE == kFused ? kProducers + 1 : 1);
      mbar_init(&ctrl->empty[s], 1);
    }
    mbar_init(&ctrl->acc_full, 1);
    ctrl->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctrl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tmap_a);
    if (MODE == kStaged) tma_prefetch(&tmap_b);
  }
  // Per-column scale and bias of this tile (fused form applies them; the
  // staged form's W_hat already holds them) and the output bias (both forms).
  for (int i = threadIdx.x; i < BN; i += kThreads) {
    const int n = n0 + i;
    float s = 1.0f, t = 0.0f;
    if (MODE == kFused && n < L.n) {
      if (L.scale) s = h2f(L.scale[n]);
      if (L.bias) t = h2f(L.bias[n]);
    }
    ctrl->sb[i] = s;
    ctrl->sb[BN + i] = t;
    ctrl->sb[2 * BN + i] = n < L.n ? out_bias_of(L.ob, n) : 0.0f;
  }
  BookView bv[2];
  if (MODE == kFused) {
    size_t off = 0;
    for (int m = 0; m < L.nb; ++m) {
      if (g.smem_mask & (1 << m)) {
        uint16_t* dst = books + off / 2;
        stage_book(dst, L.book[m], 1 << L.b[m], L.d, 8);
        bv[m] = {dst, 8};
        off += padded_book_bytes(L.b[m], L.d);
      } else {
        bv[m] = {L.book[m], L.d};
      }
    }
    if (L.nb == 1) bv[1] = bv[0];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  // As a programmatic dependent (the staged form's slabs), the weight tiles
  // come from the launch before: wait for it; then let the next launch (the
  // next slab's dequantisation) be scheduled.  No-ops for a plain launch.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    if (lane == 0) {                                   // TMA producer
      int issued = 0;
      for (int kt = 0; kt < g.num_kt; ++kt) {
        const int s = kt % g.stages;
        const uint32_t ph = (kt / g.stages) & 1;
        if (!bounded_wait(&ctrl->empty[s], ph ^ 1, abort_flag, g.status, g.budget)) break;
        uint8_t* a = stages + s * kStage;
        mbar_arrive_expect_tx(&ctrl->full[s], MODE == kStaged ? MSUB * kATile + bn * BK * 2 : MSUB * kATile);
#pragma unroll
        for (int sub = 0; sub < MSUB; ++sub)
          tma_load_2d(a + sub * kATile, &tmap_a, &ctrl->full[s], kt * BK, m0 + sub * BM);
        if (MODE == kStaged) tma_load_2d(a + MSUB * kATile, &tmap_b, &ctrl->full[s], kt * BK, n0);
        issued = kt + 1;
      }
      if (*abort_flag) {   // let loads already in flight land before the block exits
        // (with fused tiles a stage also waits for the producers, who may have
        // given up: then the time bound, far above a load's latency, ends it)
        for (int kt = max(0, issued - g.stages); kt < issued; ++kt)
          drain_phase(&ctrl->full[kt % g.stages], (kt / g.stages) & 1, kWaitBudget / 64);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {                                   // MMA issuer
      const uint32_t idesc = g.idesc;
      for (int kt = 0; kt < g.num_kt; ++kt) {
        const int s = kt % g.stages;
        const uint32_t ph = (kt / g.stages) & 1;
        if (!bounded_wait(&ctrl->full[s], ph, abort_flag, g.status, g.budget)) break;
        tc_fence_after();
        const uint32_t a = smem_addr(stages + s * kStage);
        const uint32_t b = a + MSUB * kATile;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
#pragma unroll
          for (int sub = 0; sub < MSUB; ++sub)
            umma_f16(tmem + sub * 256, sw128_kmajor_desc(a + sub * kATile + kk * 32),
                     sw128_kmajor_desc(b + kk * 32), idesc, (kt | kk) != 0);
        umma_commit(&ctrl->empty[s]);
      }
      umma_commit(&ctrl->acc_full);
      // every product issued has finished before tensor memory is freed, even
      // when the epilogue gave up waiting for it
      drain_phase(&ctrl->acc_full, 0, kWaitBudget);
    }
  } else if (warp >= 4) {
    if (MODE == kFused && B1 > 0) {                    // B-tile producers, d = 8 fast path
      // Software pipeline: while waiting for stage kt to be free, the index
      // loads of kt+2 and the centroid gathers of kt+1 are in flight.
      const int r = threadIdx.x - kProducerThread0;
      const int n = n0 + r;
      const bool live = r < bn && n < L.n;
      uint32_t fa[8], fb[8], ga[8], gb[8];
      uint4 cur[8], nxt[8];
#pragma unroll
      for (int v = 0; v < 8; ++v) { fa[v] = fb[v] = ga[v] = gb[v] = 0u; }
      if (live && g.num_kt > 0) d8_fields<B1, B2>(L, n, 0, fa, fb);
      if (live && g.num_kt > 0) d8_gather<B2>(bv, fa, fb, nxt);
      if (live && g.num_kt > 1) d8_fields<B1, B2>(L, n, 1, ga, gb);
      for (int kt = 0; kt < g.num_kt; ++kt) {
#pragma unroll
        for (int v = 0; v < 8; ++v) cur[v] = nxt[v];
        if (live && kt + 1 < g.num_kt) {
          d8_gather<B2>(bv, ga, gb, nxt);
          if (kt + 2 < g.num_kt) d8_fields<B1, B2>(L, n, kt + 2, ga, gb);
        }
        const int s = kt % g.stages;
        const uint32_t ph = (kt / g.stages) & 1;
        if (!bounded_wait(&ctrl->empty[s], ph ^ 1, abort_flag, g.status, g.budget)) break;
        if (r < bn) d8_store(L, live, kt, cur, stages + s * kStage + MSUB * kATile, r);
        fence_proxy_async_smem();
        mbar_arrive(&ctrl->full[s]);
      }
    } else if (MODE == kFused) {                       // B-tile producers, any d <= 8
      const int r = threadIdx.x - kProducerThread0;
      for (int kt = 0; kt < g.num_kt; ++kt) {
        const int s = kt % g.stages;
        const uint32_t ph = (kt / g.stages) & 1;
        if (!bounded_wait(&ctrl->empty[s], ph ^ 1, abort_flag, g.status, g.budget)) break;
        uint8_t* btile = stages + s * kStage + MSUB * kATile;
        if (r < bn) {                                  // rows past the tile width stay idle
          if (L.nb == 2) produce_row_generic<2>(L, bv, n0 + r, kt, btile, r);
          else produce_row_generic<1>(L, bv, n0 + r, kt, btile, r);
        }
        fence_proxy_async_smem();
        mbar_arrive(&ctrl->full[s]);
      }
    }
    if (warp < 4 + 4 * MSUB) {                         // epilogue: warp & 3 = TMEM lane quarter
      const int q = warp & 3;
      const int sub = (warp - 4) >> 2;                 // which 128-row sub-tile
      if (bounded_wait(&ctrl->acc_full, 0, abort_flag, g.status, g.budget)) {
        tc_fence_after();
        const int row = m0 + sub * BM + q * 32 + lane;
        const float rs = (MODE == kFused && L.bias && row < g.m) ? g.rowsum[row] : 0.0f;
        const float rsc = (g.rowscale && row < g.m) ? g.rowscale[row] : 1.0f;
        const size_t es = g.yt == VQ_FP32 ? 4 : 2;
        for (int c = 0; c < bn / 32; ++c) {
          uint32_t acc[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + sub * 256 + c * 32, acc);
          tmem_wait_ld();
          const int nb = n0 + c * 32;
          if (row >= g.m || nb >= L.n) continue;
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            v[i] = ctrl->sb[c * 32 + i] * (__uint_as_float(acc[i]) * rsc) + ctrl->sb[BN + c * 32 + i] * rs +
                   ctrl->sb[2 * BN + c * 32 + i];
          const int ncols = min(32, L.n - nb);
          uint8_t* dst = reinterpret_cast<uint8_t*>(g.y) + (static_cast<int64_t>(row) * g.ldy + nb) * es;
          if (ncols == 32 && aligned(dst, 16)) {
            if (g.yt == VQ_FP32) {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                reinterpret_cast<float4*>(dst)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            } else {
              uint32_t p[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const uint16_t lo = g.yt == VQ_FP16 ? f2h(v[2 * i]) : f2bf(v[2 * i]);
                const uint16_t hi = g.yt == VQ_FP16 ? f2h(v[2 * i + 1]) : f2bf(v[2 * i + 1]);
                p[i] = lo | (static_cast<uint32_t>(hi) << 16);
              }
#pragma unroll
              for (int i = 0; i < 4; ++i)
                reinterpret_cast<uint4*>(dst)[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
            }
          } else {
            for (int i = 0; i < ncols; ++i) store_out(dst, g.yt, i, v[i]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Per row of bf16 activations: 2^e with max_k |x[m][k]| * 2^-e in [2^14, 2^15)
// (e kept in [-126, 127]; 1 for an all-zero row), and the row sum of x.  The
// fp16 operand copy holds x * 2^-e, so no bf16 value overflows fp16 and every
// value above 2^-29 of its row's largest stays exact; the epilogue multiplies
// the accumulator by 2^e.  (For typical rows the scaling changes no bit of y:
// a power of two commutes with every fp32 rounding of the products.)
__global__ void gemm_rowscale(const uint16_t* __restrict__ x, int m, int kin, int64_t ldx,
                              float* __restrict__ rowscale, float* __restrict__ rowsum) {
  const int warps = blockDim.x >> 5;
  const int row = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= m) return;
  const uint16_t* r = x + static_cast<int64_t>(row) * ldx;
  float mx = 0.0f, s = 0.0f;
  for (int k = lane; k < kin; k += 32) {
    const float v = bf2f(r[k]);
    mx = fmaxf(mx, fabsf(v));
    s += v;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    s += __shfl_xor_sync(0xffffffffu, s, off);
  }
  if (lane == 0) {
    int e = 0;
    if (mx > 0.0f && mx < INFINITY) e = max(-126, min(127, static_cast<int>(__float_as_uint(mx) >> 23) - 126 - 15));
    rowscale[row] = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
    rowsum[row] = s;
  }
}

// x -> fp16 copy [m][kp] (zeros past kin), each row times 1 / rowscale[row]
// (an exact power of two, applied as two factors so each stays a normal
// float) when rowscale is given: one 8-element chunk per thread, 16-byte
// loads and stores when x rows are 16-byte aligned.
__global__ void gemm_convert(const uint16_t* __restrict__ x, int x_fp16, int m, int kin,
                             int64_t ldx, int vec, uint16_t* __restrict__ x16, int kp,
                             const float* __restrict__ rowscale) {
  const int cpr = kp / 8;                                   // chunks per row
  const int64_t total = static_cast<int64_t>(m) * cpr;
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < total;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = q / cpr;
    const int k = static_cast<int>(q - row * cpr) * 8;
    const uint16_t* xr = x + row * ldx;
    float v[8];
    if (vec && k + 8 <= kin) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(xr + k));
      const uint16_t* h = reinterpret_cast<const uint16_t*>(&u);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = x_fp16 ? h2f(h[i]) : bf2f(h[i]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = (k + i < kin) ? (x_fp16 ? h2f(xr[k + i]) : bf2f(xr[k + i])) : 0.0f;
    }
    if (rowscale) {
      const int e = static_cast<int>(__float_as_uint(rowscale[row]) >> 23) - 127;
      const float f1 = __uint_as_float(static_cast<uint32_t>(127 - e / 2) << 23);
      const float f2 = __uint_as_float(static_cast<uint32_t>(127 - (e - e / 2)) << 23);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = v[i] * f1 * f2;
    }
    uint32_t p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      p[i] = f2h(v[2 * i]) | (static_cast<uint32_t>(f2h(v[2 * i + 1])) << 16);
    *reinterpret_cast<uint4*>(x16 + row * kp + k) = make_uint4(p[0], p[1], p[2], p[3]);
  }
}

// fp32 row sums of the fp16 operand rows a[m][lda] (first kin columns): the
// bias term of the fused epilogue.  One warp per row.
__global__ void gemm_rowsum(const uint16_t* __restrict__ a, int m, int kin, int64_t lda,
                            float* __restrict__ rowsum) {
  const int warps = blockDim.x >> 5;
  const int row = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= m) return;
  const uint16_t* r = a + static_cast<int64_t>(row) * lda;
  float s = 0.0f;
  for (int k = lane; k < kin; k += 32) s += h2f(r[k]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) rowsum[row] = s;
}

// ---- host side ---------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D fp16 tensor [rows][cols] with row stride ld elements, box {64, box_rows},
// 128-byte swizzle; reads past cols / rows return zeros.
bool make_map(CUtensorMap* map, const void* base, int64_t cols, int64_t rows, int64_t ld,
              int box_rows) {
  return make_map_f16_sw128(map, base, cols, rows, ld, box_rows);
}

}  // namespace

bool make_map_f16_sw128(CUtensorMap* map, const void* base, int64_t cols, int64_t rows, int64_t ld,
                        int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// SM clocks a bounded wait may take: about 2 s, or VQ_WAIT_BUDGET (tests use
// a few clocks to make the waits give up).
long long wait_budget() {
  if (const char* env = std::getenv("VQ_WAIT_BUDGET")) return std::atoll(env);
  return kWaitBudget;
}

struct GemmLayout {
  int mode;
  int kp;
  bool copy_x;       // bf16 activations (or misaligned fp16) need an fp16 copy
  size_t off_rowsum, off_rowscale, off_x16, off_w, total;
};

bool fused_fast_path(const Layer& L) {
  if (L.d != 8) return false;
  const int b1 = L.b[0], b2 = L.nb == 2 ? L.b[1] : 0;
  return (b1 == 16 && (b2 == 0 || b2 == 8)) || (b1 == 12 && b2 == 8) || (b1 == 8 && b2 == 8);
}

int choose_mode(const Layer& L, int m) {
  // The fused producers read row-order records; a tiled layer is dequantised
  // by its own kernel into the workspace.
  if (L.layout == VQ_IDX_TILE4) return kStaged;
  const char* env = std::getenv("VQ_GEMM_MODE");
  if (env && std::strcmp(env, "fused") == 0) return kFused;
  if (env && std::strcmp(env, "staged") == 0) return kStaged;
  // The staged form gathers each centroid once; the fused form once per
  // 128-256 rows of x.  Fused only where its producers have a vectorised
  // path and the gathers stay cheap: shared-memory books, or few rows.
  bool l2_book = false;
  for (int i = 0; i < L.nb; ++i) l2_book |= L.b[i] > 12;
  if (!fused_fast_path(L)) return kStaged;
  return (l2_book && m > 256) || m >= 2048 ? kStaged : kFused;
}

GemmLayout layout_for(const Layer& L, int m, bool x_fp16) {
  GemmLayout g;
  g.mode = choose_mode(L, m);
  g.kp = (L.kin + 7) / 8 * 8;
  g.copy_x = !x_fp16;   // fp16 activations are read in place (16-byte aligned, ldx % 8 == 0)
  g.off_rowsum = 256;
  g.off_rowscale = g.off_rowsum + round256(static_cast<size_t>(m) * 4);
  g.off_x16 = g.off_rowscale + (g.copy_x ? round256(static_cast<size_t>(m) * 4) : 0);
  g.off_w = g.off_x16 + (g.copy_x ? round256(static_cast<size_t>(m) * g.kp * 2) : 0);
  g.total = g.off_w + (g.mode == kStaged ? round256(static_cast<size_t>(L.n) * g.kp * 2) : 0);
  return g;
}

template <int MODE, int B1, int B2, int MSUB>
cudaError_t launch_kernel(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& g,
                          size_t smem, dim3 grid, cudaStream_t stream, bool pdl = false) {
  auto k = vq_gemm_kernel<MODE, B1, B2, MSUB>;
  cudaError_t e = set_func_attr(reinterpret_cast<const void*>(k), cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  count_launch();
  if (pdl) return launch_pdl(k, grid, kThreads, smem, stream, ma, mb, g);
  k<<<grid, kThreads, smem, stream>>>(ma, mb, g);
  return cudaGetLastError();
}

// Tile shape: two 128-row sub-tiles per CTA when that still gives about one
// tile per SM; then the N width (a multiple of 32, 128..256) that wastes the
// least of the last wave: cost ~ waves * (width + 64), the 64 standing for
// the activation bytes every tile loads whatever its width.
void choose_tiles(int m, int n, int sms, int* msub, int* bn) {
  const int tiles2 = ((m + 2 * BM - 1) / (2 * BM)) * ((n + BN - 1) / BN);
  *msub = tiles2 * 5 >= sms * 4 ? 2 : 1;
  const int mt = (m + BM * *msub - 1) / (BM * *msub);
  long best = -1;
  for (int w = BN; w >= 128; w -= 32) {
    const long tiles = static_cast<long>(mt) * ((n + w - 1) / w);
    const long waves = (tiles + sms - 1) / sms;
    const long cost = waves * (w + 64);
    if (best < 0 || cost < best) { best = cost; *bn = w; }
  }
}

template <int MSUB>
cudaError_t dispatch(const Layer& L, int mode, const CUtensorMap& ma, const CUtensorMap& mb,
                     const GemmArgs& g, size_t smem, dim3 grid, cudaStream_t stream, bool pdl = false) {
  if (mode == kStaged) return launch_kernel<kStaged, 0, 0, MSUB>(ma, mb, g, smem, grid, stream, pdl);
  if (L.d == 8 && L.nb == 1 && L.b[0] == 16)
    return launch_kernel<kFused, 16, 0, MSUB>(ma, mb, g, smem, grid, stream);
  if (L.d == 8 && L.nb == 2 && L.b[0] == 16 && L.b[1] == 8)
    return launch_kernel<kFused, 16, 8, MSUB>(ma, mb, g, smem, grid, stream);
  if (L.d == 8 && L.nb == 2 && L.b[0] == 12 && L.b[1] == 8)
    return launch_kernel<kFused, 12, 8, MSUB>(ma, mb, g, smem, grid, stream);
  if (L.d == 8 && L.nb == 2 && L.b[0] == 8 && L.b[1] == 8)
    return launch_kernel<kFused, 8, 8, MSUB>(ma, mb, g, smem, grid, stream);
  return launch_kernel<kFused, 0, 0, MSUB>(ma, mb, g, smem, grid, stream);
}

// ---------------------------------------------------------------------------
// Hessian collection: H = X^T X on the same tcgen05 pipeline (staged form,
// A = B = X^T with the tokens as the contraction), then the normalisation
// and damping of "VPTQ Guide", section "Step 1: Hessian Matrix Collection":
// h = 2 H / n, h[i][i] += 0.01 * mean_i h[i][i].
// ---------------------------------------------------------------------------

// xt[i][t] = x[t][i] (t < n, i < d), through 32 x 32 shared-memory tiles.
__global__ void hess_transpose(const uint16_t* __restrict__ x, int64_t ldx, int n, int d,
                               uint16_t* __restrict__ xt, int64_t ldt) {
  __shared__ uint16_t tile[32][33];
  const int t0 = blockIdx.x * 32, i0 = blockIdx.y * 32;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int t = t0 + r, i = i0 + threadIdx.x;
    tile[r][threadIdx.x] = (t < n && i < d) ? x[static_cast<int64_t>(t) * ldx + i] : static_cast<uint16_t>(0);
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int i = i0 + r, t = t0 + threadIdx.x;
    if (i < d && t < n) xt[static_cast<int64_t>(i) * ldt + t] = tile[threadIdx.x][r];
  }
}

// damp = 0.01 * mean_i (2 / n) h[i][i], in fp64 (one block).
__global__ void hess_damp(const float* __restrict__ h, int64_t ldh, int d, double two_over_n,
                          double* __restrict__ damp) {
  __shared__ double red[256];
  double s = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) s += static_cast<double>(h[static_cast<int64_t>(i) * ldh + i]);
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *damp = 0.01 * (red[0] * two_over_n / d);
}

// h[i][j] = fp32((2 / n) h[i][j] + (i == j ? damp : 0)), one rounding.
__global__ void hess_scale(float* __restrict__ h, int64_t ldh, int d, double two_over_n,
                           const double* __restrict__ damp) {
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k >= static_cast<int64_t>(d) * d) return;
  const int i = static_cast<int>(k / d), j = static_cast<int>(k % d);
  float* p = h + static_cast<int64_t>(i) * ldh + j;
  *p = static_cast<float>(static_cast<double>(*p) * two_over_n + (i == j ? *damp : 0.0));
}

// Instruction descriptor for kind::f16 with bf16 A and B (atype = btype = 1).
constexpr uint32_t bf16_idesc(int m, int n) { return f16_idesc(m, n) | (1u << 7) | (1u << 10); }

struct HessLayout {
  int64_t ldt;
  size_t off_xt, off_damp, total;
};

HessLayout hess_layout(int n, int d) {
  HessLayout h;
  h.ldt = (static_cast<int64_t>(n) + 7) / 8 * 8;
  h.off_xt = 256;
  h.off_damp = h.off_xt + round256(static_cast<size_t>(d) * h.ldt * 2);
  h.total = h.off_damp + 256;
  return h;
}

}  // namespace

size_t gemm_workspace_bytes(const Layer& L, int m, bool x_fp16) {
  return layout_for(L, m, x_fp16).total;
}

// Closes the staged form's chain of dependent launches.  A slab's product
// waits only for its own dequantisation, so products can finish out of
// order; this plain launch starts after all of them, so whatever the stream
// runs next sees the whole of y.
__global__ void gemm_join() {}

// Slabs of the staged form.  One by default: splitting measured slower at
// every size tried (8192^2, M = 2048: 299 us in one slab, 355 / 421 / 736 in
// 2 / 4 / 8), because a product's CTAs hold most of an SM's shared memory,
// so the next slab's product cannot share SMs with the running one and the
// slabs run one after another, each on a partial wave.  VQ_GEMM_SLABS sets
// the count, for measurements (each slab a whole number of tile widths).
int gemm_slabs(int n, int bn) {
  const int tiles = (n + bn - 1) / bn;
  int s = 1;
  if (const char* env = std::getenv("VQ_GEMM_SLABS")) s = std::max(1, std::atoi(env));
  return std::max(1, std::min(s, tiles / 2));
}

vq_status launch_gemm(const Layer& L, const void* x, bool x_fp16, int m, int64_t ldx, void* y,
                      vq_dtype yt, int64_t ldy, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (L.kin == 0) return launch_empty_rows(L, y, yt, ldy, m, stream);
  const GemmLayout lay = layout_for(L, m, x_fp16);
  if (ws_bytes < lay.total) return VQ_ERR_WORKSPACE;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(w8);
  float* rowsum = reinterpret_cast<float*>(w8 + lay.off_rowsum);
  float* rowscale = reinterpret_cast<float*>(w8 + lay.off_rowscale);
  uint16_t* x16 = reinterpret_cast<uint16_t*>(w8 + lay.off_x16);
  uint16_t* what = reinterpret_cast<uint16_t*>(w8 + lay.off_w);

  {
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), stream);
    if (e != cudaSuccess) return cuda_status(e);
    if (lay.copy_x) {
      // bf16 activations: per-row power-of-two scale (and the row sums), then
      // the scaled fp16 copy
      const int warps = 8;
      count_launch();
      gemm_rowscale<<<(m + warps - 1) / warps, warps * 32, 0, stream>>>(static_cast<const uint16_t*>(x), m,
                                                                         L.kin, ldx, rowscale, rowsum);
      if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
      const int vec = aligned(x, 16) && ldx % 8 == 0;
      const int64_t chunks = static_cast<int64_t>(m) * (lay.kp / 8);
      const int blocks = static_cast<int>(std::min<int64_t>((chunks + 255) / 256, 16 * device_sm_count()));
      count_launch();
      gemm_convert<<<blocks, 256, 0, stream>>>(static_cast<const uint16_t*>(x), x_fp16 ? 1 : 0, m,
                                              L.kin, ldx, vec, x16, lay.kp, rowscale);
      if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
    } else if (lay.mode == kFused && L.bias != nullptr) {   // row sums feed the fused bias term only
      const int warps = 8;
      count_launch();
      gemm_rowsum<<<(m + warps - 1) / warps, warps * 32, 0, stream>>>(static_cast<const uint16_t*>(x), m, L.kin,
                                                                       ldx, rowsum);
      if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
    }
  }
  int msub = 1, bn = BN;
  choose_tiles(m, L.n, device_sm_count(), &msub, &bn);
  // Staged form: W_hat is written in slabs of output rows (one by default,
  // see gemm_slabs).  Each slab's product is launched as a programmatic
  // dependent of its dequantisation, and the next slab's dequantisation as a
  // dependent of that product, so that the two may run side by side.
  const int nslab = lay.mode == kStaged ? gemm_slabs(L.n, bn) : 1;
  const int slab_rows = lay.mode == kStaged ? ((L.n + nslab - 1) / nslab + bn - 1) / bn * bn : L.n;
  if (lay.mode == kStaged) {
    vq_status st = launch_dequant(layer_rows(L, 0, std::min(L.n, slab_rows)), what, lay.kp, stream);
    if (st != VQ_OK) return st;
  }
  CUtensorMap ma, mb;
  if (lay.copy_x) {
    if (!make_map(&ma, x16, L.kin, m, lay.kp, BM)) return VQ_ERR_CUDA;
  } else {
    if (!make_map(&ma, x, L.kin, m, ldx, BM)) return VQ_ERR_CUDA;
  }
  if (lay.mode != kStaged) mb = ma;

  GemmArgs g{};
  g.L = L;
  g.m = m;
  g.num_kt = (L.kin + BK - 1) / BK;
  g.rowsum = rowsum;
  g.rowscale = lay.copy_x ? rowscale : nullptr;
  g.y = y;
  g.yt = yt;
  g.ldy = ldy;
  g.status = status;
  g.budget = wait_budget();
  g.smem_mask = 0;
  g.book_bytes = 0;
  const int optin = device_smem_optin();
  const int kStageBytes = stage_bytes(msub);
  const size_t fixed = 1024 + kCtrlBytes;   // alignment slack + control block
  if (lay.mode == kFused) {
    // Stage the books that fit next to at least three pipeline stages.
    const size_t budget = static_cast<size_t>(optin) - fixed - 2 * kStageBytes;
    int mask = 0;
    size_t used = 0;
    for (int i = 0; i < L.nb; ++i) {
      const size_t b = padded_book_bytes(L.b[i], L.d);
      if (used + b <= budget) { used += b; mask |= 1 << i; }
    }
    g.smem_mask = mask;
    g.book_bytes = static_cast<int>(used);
  }
  g.stages = static_cast<int>(std::min<size_t>(kMaxStages, (optin - fixed - g.book_bytes) / kStageBytes));
  g.stages = std::min(g.stages, 4);
  const size_t smem = fixed + static_cast<size_t>(g.stages) * kStageBytes + g.book_bytes;
  g.bn = bn;
  g.idesc = f16_idesc(BM, bn);
  if (lay.mode != kStaged) {
    dim3 grid((m + BM * msub - 1) / (BM * msub), (L.n + bn - 1) / bn);
    return cuda_status(msub == 2 ? dispatch<2>(L, lay.mode, ma, mb, g, smem, grid, stream)
                                 : dispatch<1>(L, lay.mode, ma, mb, g, smem, grid, stream));
  }
  for (int n0 = 0; n0 < L.n; n0 += slab_rows) {
    const int n1 = std::min(L.n, n0 + slab_rows);
    GemmArgs gs = g;
    gs.L = layer_rows(L, n0, n1);
    gs.y = static_cast<uint8_t*>(y) + static_cast<size_t>(n0) * (yt == VQ_FP32 ? 4 : 2);
    uint16_t* wslab = what + static_cast<size_t>(n0) * lay.kp;
    if (!make_map(&mb, wslab, L.kin, n1 - n0, lay.kp, bn)) return VQ_ERR_CUDA;
    dim3 grid((m + BM * msub - 1) / (BM * msub), (n1 - n0 + bn - 1) / bn);
    cudaError_t e = msub == 2 ? dispatch<2>(gs.L, kStaged, ma, mb, gs, smem, grid, stream, true)
                              : dispatch<1>(gs.L, kStaged, ma, mb, gs, smem, grid, stream, true);
    if (e != cudaSuccess) return cuda_status(e);
    if (n1 < L.n) {
      vq_status st = launch_dequant(layer_rows(L, n1, std::min(L.n, n1 + slab_rows)),
                                    what + static_cast<size_t>(n1) * lay.kp, lay.kp, stream, true);
      if (st != VQ_OK) return st;
    }
  }
  if (nslab > 1) {
    count_launch();
    gemm_join<<<1, 32, 0, stream>>>();
    return cuda_status(cudaGetLastError());
  }
  return VQ_OK;
}

}  // namespace vqk


namespace vqk {

size_t hessian_workspace_bytes(int n, int d) { return (n < 1 || d < 1) ? 0 : hess_layout(n, d).total; }

vq_status launch_hessian(const void* x, bool x_fp16, int n, int d, int64_t ldx, float* h, int64_t ldh,
                         void* ws, size_t ws_bytes, cudaStream_t stream) {
  const HessLayout lay = hess_layout(n, d);
  if (ws_bytes < lay.total) return VQ_ERR_WORKSPACE;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(w8);
  uint16_t* xt = reinterpret_cast<uint16_t*>(w8 + lay.off_xt);
  double* damp = reinterpret_cast<double*>(w8 + lay.off_damp);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), stream);
  if (e != cudaSuccess) return cuda_status(e);
  count_launch();
  hess_transpose<<<dim3((n + 31) / 32, (d + 31) / 32), dim3(32, 8), 0, stream>>>(
      static_cast<const uint16_t*>(x), ldx, n, d, xt, lay.ldt);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);

  int msub = 1, bn = BN;
  choose_tiles(d, d, device_sm_count(), &msub, &bn);
  CUtensorMap ma, mb;
  if (!make_map(&ma, xt, n, d, lay.ldt, BM) || !make_map(&mb, xt, n, d, lay.ldt, bn)) return VQ_ERR_CUDA;
  GemmArgs g{};
  g.L.n = d;
  g.L.kin = n;
  g.m = d;
  g.num_kt = (n + BK - 1) / BK;
  g.rowsum = nullptr;
  g.y = h;
  g.yt = VQ_FP32;
  g.ldy = ldh;
  g.status = status;
  g.budget = wait_budget();
  const int optin = device_smem_optin();
  const int kStageBytes = stage_bytes(msub);
  const size_t fixed = 1024 + kCtrlBytes;
  g.stages = std::min(4, static_cast<int>((optin - fixed) / kStageBytes));
  const size_t smem = fixed + static_cast<size_t>(g.stages) * kStageBytes;
  g.bn = bn;
  g.idesc = x_fp16 ? f16_idesc(BM, bn) : bf16_idesc(BM, bn);
  dim3 grid((d + BM * msub - 1) / (BM * msub), (d + bn - 1) / bn);
  e = msub == 2 ? launch_kernel<kStaged, 0, 0, 2>(ma, mb, g, smem, grid, stream)
                : launch_kernel<kStaged, 0, 0, 1>(ma, mb, g, smem, grid, stream);
  if (e != cudaSuccess) return cuda_status(e);
  const double two_over_n = 2.0 / static_cast<double>(n);
  count_launch();
  hess_damp<<<1, 256, 0, stream>>>(h, ldh, d, two_over_n, damp);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  const int64_t cnt = static_cast<int64_t>(d) * d;
  count_launch();
  hess_scale<<<static_cast<unsigned>((cnt + 255) / 256), 256, 0, stream>>>(h, ldh, d, two_over_n, damp);
  return cuda_status(cudaGetLastError());
}

}  // namespace vqk

// gemvb.cu -- batched decode (2 <= batch <= 16) fast path of vq_gemv.
//
// Same shape as the single-row kernel (gemv1.cu): a warp owns a chunk of the
// input dimension, keeps that chunk of x in registers and walks many output
// rows, gathering one centroid row per packed index.  With a batch the
// multiply-adds grow B-fold while the gathers stay the same, so:
//
//  * the chunk shrinks with the batch so x stays in registers: G vectors per
//    lane with G*d*B <= 64 values for B <= 4 and <= 128 above (G = 4, 2, 2, 1
//    for B = 2, 4, 8, 16 at d = 8), with 4 or 2 rows in flight per warp;
//  * the products use packed fp32x2 FMAs (two batch rows per instruction);
//  * per row the B partial dot products of a warp are reduced with a
//    reduce-scatter (B/2 + B/4 + ... shuffles instead of 5 per value), and
//    the chunks of a row are combined with shared-memory atomic adds;
//  * the block finishes with y[b][o] = s[o] * dot + t[o] * sum_k x[b][k].
// Narrow layers are split along the input dimension as in gemv1.cu, with
// fp32 partials in the workspace summed in split order by gemv_finalize.
#include <algorithm>

#include "gemv_common.cuh"

namespace vqk {
namespace {

using namespace dec;

constexpr int kThreadsB = 256;
constexpr int kWarpsB = kThreadsB / 32;
constexpr int kRowsB = 128;            // rows per block, at most

// Vectors per lane: the largest power of two with G*d*B <= 64 x values for
// B <= 4 (two rows in flight) or <= 128 for B >= 8 (one row in flight).
__host__ __device__ constexpr int vectors_per_lane(int d, int bt) {
  const int budget = bt <= 4 ? 64 : 128;
  return d * bt * 8 <= budget ? 8 : d * bt * 4 <= budget ? 4 : d * bt * 2 <= budget ? 2 : 1;
}

// Rows in flight per warp: enough that a lane keeps G*R >= 4 gathers and
// their index loads outstanding while it computes.
__host__ __device__ constexpr int rows_in_flight(int bt) { return bt <= 4 ? 4 : 2; }

template <int D, int BT> struct ShapeB {
  static constexpr int G = vectors_per_lane(D, BT);
  static constexpr int R = rows_in_flight(BT);
};

// (a0, a1) += c * (x0, x1), one packed fp32x2 FMA (round to nearest).
__device__ __forceinline__ void fma2(float& a0, float& a1, float c, float x0, float x1) {
  unsigned long long acc, xv, cc;
  asm("mov.b64 %0, {%1, %2};" : "=l"(acc) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(xv) : "f"(x0), "f"(x1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(cc) : "f"(c));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(cc), "l"(xv));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(acc));
}

// Reduce-scatter of N values across the warp: afterwards every lane holds the
// full warp sum of value (lane >> (5 - log2 N)) & (N - 1) in v[0].
template <int N, int OFF>
struct ReduceScatter {
  static __device__ __forceinline__ void run(float* v, int lane) {
    if constexpr (OFF == 0) {
      return;
    } else if constexpr (N > 1) {
      constexpr int H = N / 2;
      const bool upper = (lane & OFF) != 0;
#pragma unroll
      for (int i = 0; i < H; ++i) {
        const float send = upper ? v[i] : v[i + H];
        const float keep = upper ? v[i + H] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
      }
      ReduceScatter<H, OFF / 2>::run(v, lane);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], OFF);
      ReduceScatter<1, OFF / 2>::run(v, lane);
    }
  }
};

template <int N> constexpr int log2c() { return N <= 1 ? 0 : 1 + log2c<N / 2>(); }

template <int D, int B1, int B2, bool SM1, bool SM2, int BT>
__global__ void __launch_bounds__(kThreadsB, 1) gemvb_kernel(
    Layer L, const uint16_t* __restrict__ x, int x_fp16, int batch, int64_t ldx, int x_vec,
    int chunks_per_split, int rpb, int smem_mask, int book_bytes, void* __restrict__ y,
    vq_dtype yt, int64_t ldy, float* __restrict__ ws) {
  constexpr int G = ShapeB<D, BT>::G;
  constexpr int R = ShapeB<D, BT>::R;
  constexpr int CH = 32 * G;                       // vectors per warp chunk
  constexpr bool NB2 = B2 > 0;
  constexpr int SHIFT = 5 - log2c<BT>();
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const uint16_t* book1 = L.book[0];
  const uint16_t* book2 = L.book[1];
  {
    size_t off = 0;
    if (smem_mask & 1) {
      uint16_t* dst = reinterpret_cast<uint16_t*>(smem);
      stage_book(dst, L.book[0], 1 << B1, D, 8);
      book1 = dst;
      off += padded_book_bytes(B1, D);
    }
    if (NB2 && (smem_mask & 2)) {
      uint16_t* dst = reinterpret_cast<uint16_t*>(smem + off);
      stage_book(dst, L.book[1], 1 << B2, D, 8);
      book2 = dst;
    }
  }
  const int nchunks_total = (L.nvec + CH - 1) / CH;
  const int split = blockIdx.y;
  const int c0 = split * chunks_per_split;
  const int nck = min(chunks_per_split, nchunks_total - c0);
  float* part = reinterpret_cast<float*>(smem + book_bytes);   // [rpb][BT]
  float* xsum = part + kRowsB * BT;                               // [BT]

  // Sum of each x row over this split's columns.
  {
    const int64_t k0 = static_cast<int64_t>(c0) * CH * D;
    const int64_t kend = static_cast<int64_t>(c0 + nck) * CH * D;
    const int64_t k1 = L.kin < kend ? static_cast<int64_t>(L.kin) : kend;
    for (int b = warp; b < BT; b += kWarpsB) {
      float s = 0.0f;
      if (b < batch)
        for (int64_t k = k0 + lane; k < k1; k += 32) s += x_fp16 ? h2f(x[b * ldx + k]) : bf2f(x[b * ldx + k]);
      s = warp_sum(s);
      if (lane == 0) xsum[b] = s;
    }
  }

  const int nrb = (L.n + rpb - 1) / rpb;
  const int pairs = rpb / R;
  const int items = nck * pairs;
  const int per_warp = (items + kWarpsB - 1) / kWarpsB;
  const int it_begin = warp * per_warp;
  const int it_end = min(items, it_begin + per_warp);

  for (int rb = blockIdx.x; rb < nrb; rb += gridDim.x) {
    const int o0 = rb * rpb;
    for (int i = tid; i < rpb * BT; i += kThreadsB) part[i] = 0.0f;
    __syncthreads();

    int cur_chunk = -1;
    bool lane_live = false;
    float xr[G][D][BT];
    uint32_t f1n[R][G], f2n[R][G];

    auto load_item = [&](int it, uint32_t (&a)[R][G], uint32_t (&b)[R][G]) {
      const int ch = c0 + it / pairs;
      const int vbase = ch * CH + lane * G;
      const bool live = vbase < L.nvec;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int o = min(o0 + (it % pairs) * R + r, L.n - 1);
        if (live) {
          load_fields<G, B1>(L.idx[0] + static_cast<int64_t>(o) * L.rw[0], L.rw[0], vbase, a[r]);
          if constexpr (NB2)
            load_fields<G, NB2 ? B2 : 4>(L.idx[1] + static_cast<int64_t>(o) * L.rw[1], L.rw[1], vbase, b[r]);
        } else {
#pragma unroll
          for (int v = 0; v < G; ++v) { a[r][v] = 0u; b[r][v] = 0u; }
        }
      }
    };

    if (it_begin < it_end) load_item(it_begin, f1n, f2n);
    for (int it = it_begin; it < it_end; ++it) {
      uint32_t f1[R][G], f2[R][G];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int v = 0; v < G; ++v) { f1[r][v] = f1n[r][v]; f2[r][v] = f2n[r][v]; }
      if (it + 1 < it_end) load_item(it + 1, f1n, f2n);

      const int ch = c0 + it / pairs;
      if (ch != cur_chunk) {                      // this lane's G vectors of x, zero past Kin / batch
        cur_chunk = ch;
        const int v0 = ch * CH + lane * G;
        lane_live = v0 < L.nvec;
#pragma unroll
        for (int v = 0; v < G; ++v) {
          const int64_t k0 = static_cast<int64_t>(v0 + v) * D;
#pragma unroll
          for (int b = 0; b < BT; ++b) {
            const uint16_t* xp = x + b * ldx + k0;
            if (D == 8 && x_vec && b < batch && k0 + 8 <= L.kin) {
              const uint4 u = __ldg(reinterpret_cast<const uint4*>(xp));
              const uint16_t* h = reinterpret_cast<const uint16_t*>(&u);
#pragma unroll
              for (int e = 0; e < D; ++e) xr[v][e][b] = x_fp16 ? h2f(h[e]) : bf2f(h[e]);
            } else {
#pragma unroll
              for (int e = 0; e < D; ++e)
                xr[v][e][b] = (b < batch && k0 + e < L.kin) ? (x_fp16 ? h2f(xp[e]) : bf2f(xp[e])) : 0.0f;
            }
          }
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float acc[BT];
#pragma unroll
        for (int b = 0; b < BT; ++b) acc[b] = 0.0f;
        if (lane_live) {
#pragma unroll
          for (int v = 0; v < G; ++v) {
            float c[D];
            centroid<D, SM1>(book1, f1[r][v], c);
            if constexpr (NB2) {
              float c2[D];
              centroid<D, SM2>(book2, f2[r][v], c2);
#pragma unroll
              for (int e = 0; e < D; ++e) c[e] += c2[e];
            }
#pragma unroll
            for (int e = 0; e < D; ++e)
#pragma unroll
              for (int b = 0; b < BT; b += 2) fma2(acc[b], acc[b + 1], c[e], xr[v][e][b], xr[v][e][b + 1]);
          }
        }
        ReduceScatter<BT, 16>::run(acc, lane);
        if ((lane & ((1 << SHIFT) - 1)) == 0) {
          const int rl = (it % pairs) * R + r;
          atomicAdd(&part[rl * BT + ((lane >> SHIFT) & (BT - 1))], acc[0]);
        }
      }
    }
    __syncthreads();
    for (int i = tid; i < rpb * batch; i += kThreadsB) {
      const int rl = i / batch, b = i - rl * batch;
      const int o = o0 + rl;
      if (o >= L.n) continue;
      const float sc = L.scale ? h2f(L.scale[o]) : 1.0f;
      const float t = L.bias ? h2f(L.bias[o]) : 0.0f;
      float val = sc * part[rl * BT + b] + t * xsum[b];
      if (split == 0) val += out_bias_of(L.ob, o);   // once, with split 0's part
      if (ws) ws[(static_cast<int64_t>(split) * batch + b) * L.n + o] = val;
      else store_out(y, yt, b * ldy + o, val);
    }
    __syncthreads();
  }
}

template <int D, int B1, int B2, bool SM1, bool SM2, int BT>
cudaError_t launchb(const Layer& L, const GemvPlan& p, const void* x, bool xf, int batch,
                    int64_t ldx, void* y, vq_dtype yt, int64_t ldy, float* ws, cudaStream_t stream) {
  auto k = gemvb_kernel<D, B1, B2, SM1, SM2, BT>;
  cudaError_t e = set_func_attr(reinterpret_cast<const void*>(k), cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem);
  if (e != cudaSuccess) return e;
  if (!SM1) {   // L2-served book: keep shared memory small so L1 is as large as possible
    e = set_func_attr(reinterpret_cast<const void*>(k), cudaFuncAttributePreferredSharedMemoryCarveout, 10);
    if (e != cudaSuccess) return e;
  }
  const int x_vec = aligned(x, 16) && ldx % 8 == 0;
  dim3 grid(p.grid_x, p.nsplit);
  count_launch();
  k<<<grid, kThreadsB, p.smem, stream>>>(L, static_cast<const uint16_t*>(x), xf ? 1 : 0, batch, ldx,
                                         x_vec, p.vps / (32 * ShapeB<D, BT>::G), p.rpb,
                                         p.books_in_smem, p.book_bytes, y, yt, ldy,
                                         p.nsplit > 1 ? ws : nullptr);
  return cudaGetLastError();
}

template <int D, int B1, int B2, bool SM1, bool SM2>
cudaError_t launchb_bt(const Layer& L, const GemvPlan& p, const void* x, bool xf, int batch,
                       int64_t ldx, void* y, vq_dtype yt, int64_t ldy, float* ws, cudaStream_t s) {
  switch (p.bt) {   // batch tiles of 4 are left to the generic kernel (see gemvb_supported)
    case 2: return launchb<D, B1, B2, SM1, SM2, 2>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
    case 8: return launchb<D, B1, B2, SM1, SM2, 8>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
    case 16: return launchb<D, B1, B2, SM1, SM2, 16>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

// Where this kernel beats the generic one (gemv.cu), as measured on B200:
// shared-memory books at every batch except 3..4, and the L2-served 2^16 book
// at batch 2 only (beyond that its few gathers in flight per lane leave the
// L2 latency exposed, and the generic kernel's higher occupancy wins).
bool gemvb_supported(const Layer& L, int batch) {
  if (batch < 2 || batch > kMaxBatch) return false;
  if (!dec::decode_fast_path(L.d, L.b[0], L.nb == 2 ? L.b[1] : 0)) return false;
  int bt = 2;
  while (bt < batch) bt <<= 1;
  if (bt == 4) return false;
  if (L.b[0] > 12 && batch > 2) return false;
  return true;
}

void plan_gemvb(const Layer& L, int batch, GemvPlan* p) {
  int bt = 2;
  while (bt < batch) bt <<= 1;
  const int chunk = 32 * vectors_per_lane(L.d, bt);
  int mask = 0;
  size_t books = 0;
  for (int m = 0; m < L.nb; ++m) {
    if (L.b[m] <= 12) {
      mask |= 1 << m;
      books += padded_book_bytes(L.b[m], L.d);
    }
  }
  const int nchunks = (L.nvec + chunk - 1) / chunk;
  const int slots = device_sm_count();
  int nsplit = 1;
  while (nsplit < nchunks && ((L.n + kRowsB - 1) / kRowsB) * nsplit < slots) nsplit *= 2;
  nsplit = std::min(nsplit, nchunks);
  const int cps = (nchunks + nsplit - 1) / nsplit;
  nsplit = (nchunks + cps - 1) / cps;
  const int R = rows_in_flight(bt);
  const int grid_x = std::max(1, slots / nsplit);
  const int rounds = std::max(1, (L.n + grid_x * kRowsB - 1) / (grid_x * kRowsB));
  int rpb = (L.n + grid_x * rounds - 1) / (grid_x * rounds);
  rpb = std::min(kRowsB, std::max(R, (rpb + R - 1) / R * R));
  const int nrb = (L.n + rpb - 1) / rpb;
  p->bt = bt;
  p->nsplit = nsplit;
  p->vps = cps * chunk;
  p->rpb = rpb;
  p->books_in_smem = mask;
  p->book_bytes = static_cast<int>(books);
  p->smem = static_cast<int>(books + sizeof(float) * (kRowsB * bt + bt));
  p->grid_x = std::max(1, std::min(nrb, grid_x));
  p->ws_bytes = nsplit > 1 ? static_cast<size_t>(nsplit) * batch * L.n * sizeof(float) : 0;
  p->fast = 2;
}

cudaError_t launch_gemvb(const Layer& L, const GemvPlan& p, const void* x, bool xf, int batch,
                         int64_t ldx, void* y, vq_dtype yt, int64_t ldy, float* ws, cudaStream_t s) {
  const int b1 = L.b[0], b2 = L.nb == 2 ? L.b[1] : 0;
  if (L.d == 8 && b1 == 16 && b2 == 0) return launchb_bt<8, 16, 0, false, false>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
  if (L.d == 8 && b1 == 16 && b2 == 8) return launchb_bt<8, 16, 8, false, true>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
  if (L.d == 8 && b1 == 12 && b2 == 8) return launchb_bt<8, 12, 8, true, true>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
  if (L.d == 8 && b1 == 8 && b2 == 8) return launchb_bt<8, 8, 8, true, true>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
  if (L.d == 8 && b1 == 8 && b2 == 0) return launchb_bt<8, 8, 0, true, false>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
  if (L.d == 6 && b1 == 12 && b2 == 4) return launchb_bt<6, 12, 4, true, true>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
  if (L.d == 6 && b1 == 12 && b2 == 0) return launchb_bt<6, 12, 0, true, false>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
  return cudaErrorNotSupported;
}

}  // namespace vqk

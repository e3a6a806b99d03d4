// gemv1.cu -- single-row decode (batch 1) fast path of vq_gemv.
//
// The decode GEMV of the pages ("VPTQ Guide: Extreme 2-Bit Vector
// Quantization", section "Step 3": a warp loads indices, looks up the
// codebook, dot product in registers) is bound on B200 by how fast random
// 16-byte centroid rows can be gathered, not by HBM: a 2^16-entry book
// (1 MiB) lives in L2 and every lookup is a separate L1 tag lookup.  This
// kernel is shaped around that:
//
//  * A warp owns one 256-vector chunk of the input dimension (2048 columns at
//    d = 8) and keeps that chunk of x in registers (8 vectors per lane), then
//    walks many output rows: per row each lane loads its 8 packed indices
//    (one aligned 4-16 byte load), gathers 8 centroid rows, and accumulates
//    8*d products.  Two rows are in flight per warp and the next pair's index
//    words are loaded before the current pair is consumed.
//  * Index words are read with L1::no_allocate and L2-served centroid rows
//    with L1::evict_last, so L1 holds codebook rows rather than the index
//    stream; the kernel asks for the smallest shared-memory carveout so L1 is
//    as large as possible.  Books of up to 2^12 entries are staged in shared
//    memory instead.
//  * Per row, each chunk's dot product is reduced across the warp with
//    shuffles and parked in shared memory; the block then sums the chunks of
//    each row in order and applies the scale and bias (y = s * dot + t *
//    sum(x)).  Narrow layers are split along the input dimension into several
//    blocks whose partial results go to the workspace and are summed in split
//    order by the finalize kernel of gemv.cu.
#include <algorithm>

#include "codebook.cuh"

namespace vqk {
namespace {

constexpr int kG = 8;                  // vectors per lane per chunk
constexpr int kChunk = 32 * kG;        // vectors per warp chunk
constexpr int kThreads1 = 256;
constexpr int kWarps1 = kThreads1 / 32;
constexpr int kRows1 = 128;            // rows per work item (block)
constexpr int kR = 2;                  // rows in flight per warp

template <int B> struct Words { static constexpr int n = (kG * B) / 32; };

// The kG index fields of one lane: kG*B bits starting at bit v0*B, which is
// word aligned because kG*B is a multiple of 32 for B in {4, 8, 12, 16}.
// Words at or past the row end read as zero.
template <int B>
__device__ __forceinline__ void load_words(const uint32_t* __restrict__ row, int64_t rw, int v0,
                                           uint32_t (&w)[Words<B>::n]) {
  constexpr int NW = Words<B>::n;
  const int64_t w0 = (static_cast<int64_t>(v0) * B) >> 5;
  const uint32_t* p = row + w0;
  if (w0 + NW <= rw) {
    if constexpr (NW == 4) {
      asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "l"(p));
    } else if constexpr (NW == 2) {
      asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                   : "=r"(w[0]), "=r"(w[1]) : "l"(p));
    } else {
#pragma unroll
      for (int i = 0; i < NW; ++i)
        asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(w[i]) : "l"(p + i));
    }
  } else {
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      w[i] = 0u;
      if (w0 + i < rw)
        asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(w[i]) : "l"(p + i));
    }
  }
}

template <int B>
__device__ __forceinline__ uint32_t field_of(const uint32_t (&w)[Words<B>::n], int v) {
  constexpr int NW = Words<B>::n;
  const int bit = v * B;                       // compile-time after unrolling
  const int q = bit >> 5, s = bit & 31;
  const uint32_t lo = w[q];
  const uint32_t hi = (q + 1 < NW) ? w[q + 1] : 0u;
  return __funnelshift_r(lo, hi, s) & ((1u << B) - 1u);
}

// Centroid row k as fp32.  SMEM: staged book with 16-byte rows.  Otherwise a
// global book with d-half rows, read through L1 with evict-last priority.
template <int D, bool SMEM>
__device__ __forceinline__ void centroid(const uint16_t* base, uint32_t k, float (&c)[D]) {
  if constexpr (SMEM) {
    const uint4 v = *reinterpret_cast<const uint4*>(base + static_cast<size_t>(k) * 8);
    float t[8];
    unpack8(v, t);
#pragma unroll
    for (int e = 0; e < D; ++e) c[e] = t[e];
  } else if constexpr (D == 8) {
    uint4 v;
    asm volatile("ld.global.nc.L1::evict_last.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(base + static_cast<size_t>(k) * 8));
    float t[8];
    unpack8(v, t);
#pragma unroll
    for (int e = 0; e < 8; ++e) c[e] = t[e];
  } else {
    static_assert(D % 2 == 0, "global books need an even d");
    const uint32_t* p = reinterpret_cast<const uint32_t*>(base + static_cast<size_t>(k) * D);
#pragma unroll
    for (int q = 0; q < D / 2; ++q) {
      uint32_t w;
      asm volatile("ld.global.nc.L1::evict_last.u32 %0, [%1];" : "=r"(w) : "l"(p + q));
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
      c[2 * q] = f.x;
      c[2 * q + 1] = f.y;
    }
  }
}

__device__ __forceinline__ float warp_sum1(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

template <int D, int B1, int B2, bool SM1, bool SM2>
__global__ void __launch_bounds__(kThreads1, 1) gemv1_kernel(
    Layer L, const uint16_t* __restrict__ x, int x_fp16, int chunks_per_split, int rpb,
    int smem_mask, int book_bytes, void* __restrict__ y, vq_dtype yt, float* __restrict__ ws) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr bool NB2 = B2 > 0;

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
  const int nchunks_total = (L.nvec + kChunk - 1) / kChunk;
  const int split = blockIdx.y;
  const int c0 = split * chunks_per_split;
  const int nck = min(chunks_per_split, nchunks_total - c0);
  float* part = reinterpret_cast<float*>(smem + book_bytes);   // [rpb][nck]
  float* xsum_s = part + kRows1 * chunks_per_split;

  // Sum of x over this split's columns.
  if (warp == 0) {
    const int64_t k0 = static_cast<int64_t>(c0) * kChunk * D;
    const int64_t kend = static_cast<int64_t>(c0 + nck) * kChunk * D;
    const int64_t k1 = L.kin < kend ? static_cast<int64_t>(L.kin) : kend;
    float s = 0.0f;
    for (int64_t k = k0 + lane; k < k1; k += 32) s += x_fp16 ? h2f(x[k]) : bf2f(x[k]);
    s = warp_sum1(s);
    if (lane == 0) *xsum_s = s;
  }
  __syncthreads();

  const int nrb = (L.n + rpb - 1) / rpb;
  // Work items: (chunk, pair of rows) in chunk-major order; each warp takes a
  // contiguous range, so it stays on one chunk (one load of x) almost always.
  const int kPairs = rpb / kR;
  const int items = nck * kPairs;
  const int per_warp = (items + kWarps1 - 1) / kWarps1;
  const int it_begin = warp * per_warp;
  const int it_end = min(items, it_begin + per_warp);
  for (int rb = blockIdx.x; rb < nrb; rb += gridDim.x) {
    const int o0 = rb * rpb;
    int cur_chunk = -1;
    float xr[kG][D];
    bool lane_live = false;
    uint32_t w1n[kR][Words<B1>::n], w2n[kR][Words<NB2 ? B2 : 4>::n];

    auto load_item = [&](int it, uint32_t (&a)[kR][Words<B1>::n],
                         uint32_t (&b)[kR][Words<NB2 ? B2 : 4>::n]) {
      const int ch = c0 + it / kPairs;
      const int vbase = ch * kChunk + lane * kG;
      const bool live = vbase < L.nvec;
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        const int o = min(o0 + (it % kPairs) * kR + r, L.n - 1);
        if (live) {
          load_words<B1>(L.idx[0] + static_cast<int64_t>(o) * L.rw[0], L.rw[0], vbase, a[r]);
          if constexpr (NB2)
            load_words<B2>(L.idx[1] + static_cast<int64_t>(o) * L.rw[1], L.rw[1], vbase, b[r]);
        } else {
#pragma unroll
          for (int i = 0; i < Words<B1>::n; ++i) a[r][i] = 0u;
          if constexpr (NB2) {
#pragma unroll
            for (int i = 0; i < Words<NB2 ? B2 : 4>::n; ++i) b[r][i] = 0u;
          }
        }
      }
    };

    if (it_begin < it_end) load_item(it_begin, w1n, w2n);
    for (int it = it_begin; it < it_end; ++it) {
      uint32_t w1[kR][Words<B1>::n], w2[kR][Words<NB2 ? B2 : 4>::n];
#pragma unroll
      for (int r = 0; r < kR; ++r) {
#pragma unroll
        for (int i = 0; i < Words<B1>::n; ++i) w1[r][i] = w1n[r][i];
        if constexpr (NB2) {
#pragma unroll
          for (int i = 0; i < Words<NB2 ? B2 : 4>::n; ++i) w2[r][i] = w2n[r][i];
        }
      }
      if (it + 1 < it_end) load_item(it + 1, w1n, w2n);

      const int ch = c0 + it / kPairs;
      if (ch != cur_chunk) {                      // x of this lane's 8 vectors, zero past Kin
        cur_chunk = ch;
        const int v0 = ch * kChunk + lane * kG;
        lane_live = v0 < L.nvec;
#pragma unroll
        for (int v = 0; v < kG; ++v)
#pragma unroll
          for (int e = 0; e < D; ++e) {
            const int64_t k = static_cast<int64_t>(v0 + v) * D + e;
            xr[v][e] = (k < L.kin) ? (x_fp16 ? h2f(x[k]) : bf2f(x[k])) : 0.0f;
          }
      }
      float acc[kR];
#pragma unroll
      for (int r = 0; r < kR; ++r) acc[r] = 0.0f;
      if (lane_live) {
#pragma unroll
        for (int r = 0; r < kR; ++r) {
          float c[kG][D];
#pragma unroll
          for (int v = 0; v < kG; ++v) centroid<D, SM1>(book1, field_of<B1>(w1[r], v), c[v]);
          if constexpr (NB2) {
#pragma unroll
            for (int v = 0; v < kG; ++v) {
              float c2[D];
              centroid<D, SM2>(book2, field_of<NB2 ? B2 : 4>(w2[r], v), c2);
#pragma unroll
              for (int e = 0; e < D; ++e) c[v][e] += c2[e];
            }
          }
#pragma unroll
          for (int v = 0; v < kG; ++v)
#pragma unroll
            for (int e = 0; e < D; ++e) acc[r] = fmaf(c[v][e], xr[v][e], acc[r]);
        }
      }
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        const float s = warp_sum1(acc[r]);
        const int rl = (it % kPairs) * kR + r;
        if (lane == 0) part[rl * chunks_per_split + (ch - c0)] = s;
      }
    }
    __syncthreads();
    for (int rl = tid; rl < rpb; rl += kThreads1) {
      const int o = o0 + rl;
      if (o >= L.n) continue;
      float dot = 0.0f;
      for (int c = 0; c < nck; ++c) dot += part[rl * chunks_per_split + c];
      const float sc = L.scale ? h2f(L.scale[o]) : 1.0f;
      const float t = L.bias ? h2f(L.bias[o]) : 0.0f;
      float val = sc * dot + t * (*xsum_s);
      if (split == 0) val += out_bias_of(L.ob, o);   // once, with split 0's part
      if (ws) ws[static_cast<int64_t>(split) * L.n + o] = val;
      else store_out(y, yt, o, val);
    }
    __syncthreads();
  }
}

template <int D, int B1, int B2, bool SM1, bool SM2>
cudaError_t launch1(const Layer& L, const GemvPlan& p, const void* x, bool xf, void* y,
                    vq_dtype yt, float* ws, cudaStream_t stream) {
  auto k = gemv1_kernel<D, B1, B2, SM1, SM2>;
  cudaError_t e = set_func_attr(reinterpret_cast<const void*>(k), cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem);
  if (e != cudaSuccess) return e;
  if (!SM1) {   // L2-served book: keep shared memory small so L1 is as large as possible
    e = set_func_attr(reinterpret_cast<const void*>(k), cudaFuncAttributePreferredSharedMemoryCarveout, 10);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(p.grid_x, p.nsplit);
  count_launch();
  k<<<grid, kThreads1, p.smem, stream>>>(L, static_cast<const uint16_t*>(x), xf ? 1 : 0, p.vps / kChunk,
                                         p.rpb, p.books_in_smem, p.book_bytes, y, yt,
                                         p.nsplit > 1 ? ws : nullptr);
  return cudaGetLastError();
}

}  // namespace

// The single-row kernel covers d in {6, 8} with the index widths of the named
// workloads; returns cudaErrorNotSupported (and launches nothing) otherwise.
bool gemv1_supported(const Layer& L) {
  if (L.d != 8 && L.d != 6) return false;
  const int b1 = L.b[0], b2 = L.nb == 2 ? L.b[1] : 0;
  if (L.d == 8 && b1 == 16 && b2 == 0) return true;
  if (L.d == 8 && b1 == 16 && b2 == 8) return true;
  if (L.d == 8 && b1 == 12 && b2 == 8) return true;
  if (L.d == 8 && b1 == 8 && (b2 == 8 || b2 == 0)) return true;
  if (L.d == 6 && b1 == 12 && (b2 == 4 || b2 == 0)) return true;
  return false;
}

void plan_gemv1(const Layer& L, GemvPlan* p) {
  int mask = 0;
  // Books of up to 2^12 entries go to shared memory; a 2^16-entry book stays in L2.
  size_t books = 0;
  for (int m = 0; m < L.nb; ++m) {
    if (L.b[m] <= 12) {
      mask |= 1 << m;
      books += padded_book_bytes(L.b[m], L.d);
    }
  }
  const int nchunks = (L.nvec + kChunk - 1) / kChunk;
  // One block per SM (the kernel is register-heavy).  Split the input
  // dimension only when there are too few 128-row blocks to fill the SMs.
  const int slots = device_sm_count();
  int nsplit = 1;
  while (nsplit < nchunks && ((L.n + kRows1 - 1) / kRows1) * nsplit < slots) nsplit *= 2;
  nsplit = std::min(nsplit, nchunks);
  const int cps = (nchunks + nsplit - 1) / nsplit;
  nsplit = (nchunks + cps - 1) / cps;
  // Rows per block: every block of a split handles the same number of row
  // blocks (`rounds`), each at most 128 rows, so no SM idles in a last wave.
  const int grid_x = std::max(1, slots / nsplit);
  const int rounds = std::max(1, (L.n + grid_x * kRows1 - 1) / (grid_x * kRows1));
  int rpb = (L.n + grid_x * rounds - 1) / (grid_x * rounds);
  rpb = std::min(kRows1, std::max(kR, (rpb + kR - 1) / kR * kR));
  const int nrb = (L.n + rpb - 1) / rpb;
  p->bt = 1;
  p->nsplit = nsplit;
  p->vps = cps * kChunk;
  p->rpb = rpb;
  p->books_in_smem = mask;
  p->book_bytes = static_cast<int>(books);
  p->smem = static_cast<int>(books + sizeof(float) * (kRows1 * cps + 4));
  p->grid_x = std::max(1, std::min(nrb, grid_x));
  p->ws_bytes = nsplit > 1 ? static_cast<size_t>(nsplit) * L.n * sizeof(float) : 0;
  p->fast = 1;
}

cudaError_t launch_gemv1(const Layer& L, const GemvPlan& p, const void* x, bool xf, void* y,
                         vq_dtype yt, float* ws, cudaStream_t s) {
  const int b1 = L.b[0], b2 = L.nb == 2 ? L.b[1] : 0;
  const bool s1 = p.books_in_smem & 1, s2 = (p.books_in_smem & 2) != 0;
  if (L.d == 8 && b1 == 16 && b2 == 0) return launch1<8, 16, 0, false, false>(L, p, x, xf, y, yt, ws, s);
  if (L.d == 8 && b1 == 16 && b2 == 8) return launch1<8, 16, 8, false, true>(L, p, x, xf, y, yt, ws, s);
  if (L.d == 8 && b1 == 12 && b2 == 8 && s1 && s2) return launch1<8, 12, 8, true, true>(L, p, x, xf, y, yt, ws, s);
  if (L.d == 8 && b1 == 8 && b2 == 8) return launch1<8, 8, 8, true, true>(L, p, x, xf, y, yt, ws, s);
  if (L.d == 8 && b1 == 8 && b2 == 0) return launch1<8, 8, 0, true, false>(L, p, x, xf, y, yt, ws, s);
  if (L.d == 6 && b1 == 12 && b2 == 4) return launch1<6, 12, 4, true, true>(L, p, x, xf, y, yt, ws, s);
  if (L.d == 6 && b1 == 12 && b2 == 0) return launch1<6, 12, 0, true, false>(L, p, x, xf, y, yt, ws, s);
  return cudaErrorNotSupported;
}

}  // namespace vqk

// gemv.cu -- vq_gemv: decode-time y = x . W_hat^T for batch <= 16, fused
// unpack -> centroid gather -> multiply-accumulate, W_hat never leaves
// registers.  The general split-K kernel here reads either index order; the
// batch-1 fast paths are gemv1.cu (row order) and tile4.cu (tiled order).
//
// The pages describe the kernel shape this follows ("VPTQ Guide: Extreme
// 2-Bit Vector Quantization", section "Step 3: Fused Low-Bit VPTQ Linear
// Layer": each warp loads indices from memory, looks up the on-chip codebook
// and does the dot product in registers; "Vector Quantization for LLM Weights
// in Production", section "2. Lookup Table (LUT) Overhead vs. Bit-Shifting":
// small codebooks in shared memory, large ones served by the cache
// hierarchy).  The B200 design:
//
//  * Work item = (group of R output rows) x (K split).  A warp owns the R
//    rows; lane l takes vectors v = l, l+32, ... of the split, so the index
//    reads of a warp are contiguous and its activation reads hit 32 distinct
//    banks.
//  * Activations of the split are staged once per block in shared memory as
//    fp32 in a [batch][e][v] layout (element e of vector v), zero past Kin.
//  * Codebooks that fit are staged in shared memory with 16-byte rows; the
//    2^16-entry books are read through L1/L2.
//  * Scale and bias are factored out of the inner loop: per row the kernel
//    accumulates <C1[i1] + C2[i2], x_j> and finishes with s * dot + t * sum(x).
//  * Lanes reduce with warp shuffles.  With several K splits each split
//    writes fp32 partials to the workspace and a second kernel sums them in
//    split order (deterministic), then converts to the output type.
#include <algorithm>

#include "codebook.cuh"

namespace vqk {
namespace {

constexpr int kGvThreads = 256;
constexpr int kGvWarps = kGvThreads / 32;
constexpr size_t kGvSmemBooks = 96 * 1024;   // stage books up to this size
constexpr size_t kGvSmemBlock = 110 * 1024;  // per-block budget: two blocks per SM

template <int BT> struct RowsPerWarp { static constexpr int value = BT >= 4 ? 4 : 2; };

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// TILED: the index streams are in the tiled order (VQ_IDX_TILE4): field
// (o, j) is slot j % 4 of row o's record in tile j / 4.
template <int D, int NB, int BT, bool TILED>
__global__ void __launch_bounds__(kGvThreads) gemv_kernel(
    Layer L, const uint16_t* __restrict__ x, int x_fp16, int batch, int64_t ldx, int vps, int rpb,
    int smem_mask, int book_bytes, void* __restrict__ y, vq_dtype yt, int64_t ldy,
    float* __restrict__ ws) {
  constexpr int R = RowsPerWarp<BT>::value;
  constexpr int DM = D > 0 ? D : kMaxVecDim;
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = D > 0 ? D : L.d;

  BookView bv[2];
  {
    size_t off = 0;
#pragma unroll
    for (int m = 0; m < NB; ++m) {
      if (smem_mask & (1 << m)) {
        const int pad = L.d <= 8 ? 8 : 16;
        uint16_t* dst = reinterpret_cast<uint16_t*>(smem + off);
        stage_book(dst, L.book[m], 1 << L.b[m], L.d, pad);
        bv[m] = {dst, pad};
        off += (static_cast<size_t>(1) << L.b[m]) * pad * sizeof(uint16_t);
      } else {
        bv[m] = {L.book[m], L.d};
      }
    }
  }

  // Activations of this split: xs[b][e][v] (fp32), then their sums.
  const int split = blockIdx.y;
  const int j0 = split * vps;
  const int nv = max(0, min(L.nvec, j0 + vps) - j0);
  float* xs = reinterpret_cast<float*>(smem + book_bytes);
  float* xsum = xs + BT * d * vps;
  for (int i = tid; i < BT * d * vps; i += kGvThreads) {
    const int b = i / (d * vps);
    const int rem = i - b * d * vps;
    const int e = rem / vps, v = rem - e * vps;
    const int64_t k = static_cast<int64_t>(j0 + v) * d + e;
    float val = 0.0f;
    if (b < batch && v < nv && k < L.kin) {
      const uint16_t h = x[b * ldx + k];
      val = x_fp16 ? h2f(h) : bf2f(h);
    }
    xs[i] = val;
  }
  __syncthreads();
  for (int b = warp; b < BT; b += kGvWarps) {
    float s = 0.0f;
    for (int i = lane; i < d * vps; i += 32) s += xs[b * d * vps + i];
    s = warp_sum(s);
    if (lane == 0) xsum[b] = s;
  }
  __syncthreads();

  const int nrb = (L.n + rpb - 1) / rpb;
  for (int rb = blockIdx.x; rb < nrb; rb += gridDim.x) {
    const int o_end = min(L.n, rb * rpb + rpb);
    for (int o = rb * rpb + warp * R; o < o_end; o += kGvWarps * R) {
      const uint32_t* row0[R];
      const uint32_t* row1[R];
      int64_t orows[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int64_t orow = min(o + r, o_end - 1);     // clamp: results of extra rows are dropped
        orows[r] = orow;
        row0[r] = L.idx[0] + orow * L.rw[0];
        row1[r] = (NB == 2) ? L.idx[1] + orow * L.rw[NB - 1] : nullptr;
      }
      // Field j of row r, book m, in either storage order.
      auto field = [&](int m, int r, int64_t j) -> uint32_t {
        if constexpr (TILED)
          return load_field(L.idx[m] + (j >> 2) * L.rw[m], (orows[r] * 4 + (j & 3)) * L.b[m], L.b[m]);
        else
          return load_field(m == 0 ? row0[r] : row1[r], j * L.b[m], L.b[m]);
      };
      float acc[R][BT];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < BT; ++b) acc[r][b] = 0.0f;

#pragma unroll 2
      for (int v = lane; v < nv; v += 32) {
        const int64_t j = j0 + v;
        float wv[R][DM];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          load_centroid<D>(bv[0], field(0, r, j), d, wv[r]);
          if constexpr (NB == 2) {
            float c2[DM];
            load_centroid<D>(bv[1], field(1, r, j), d, c2);
#pragma unroll
            for (int e = 0; e < DM; ++e) wv[r][e] += c2[e];
          }
        }
#pragma unroll
        for (int b = 0; b < BT; ++b) {
          float xv[DM];
#pragma unroll
          for (int e = 0; e < DM; ++e) xv[e] = (e < d) ? xs[(b * d + e) * vps + v] : 0.0f;
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int e = 0; e < DM; ++e)
              if (e < d) acc[r][b] = fmaf(wv[r][e], xv[e], acc[r][b]);
        }
      }

#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int orow = o + r;
#pragma unroll
        for (int b = 0; b < BT; ++b) {
          const float dot = warp_sum(acc[r][b]);
          if (lane == 0 && orow < o_end && b < batch) {
            const float sc = L.scale ? h2f(L.scale[orow]) : 1.0f;
            const float t = L.bias ? h2f(L.bias[orow]) : 0.0f;
            float val = sc * dot + t * xsum[b];
            if (split == 0) val += out_bias_of(L.ob, orow);   // once, with split 0's part
            if (ws) ws[(static_cast<int64_t>(split) * batch + b) * L.n + orow] = val;
            else store_out(y, yt, b * ldy + orow, val);
          }
        }
      }
    }
  }
}

// Sum the K-split partials in split order and convert.
__global__ void gemv_finalize(const float* __restrict__ ws, int nsplit, int batch, int n,
                              void* __restrict__ y, vq_dtype yt, int64_t ldy) {
  const int64_t total = static_cast<int64_t>(batch) * n;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = i / n, o = i - b * n;
    float v = 0.0f;
    for (int s = 0; s < nsplit; ++s) v += ws[(s * static_cast<int64_t>(batch) + b) * n + o];
    store_out(y, yt, b * ldy + o, v);
  }
}

// y[b][o] = out_bias[o] for every row b of y (a layer with no inputs).
__global__ void fill_out_bias(const uint16_t* __restrict__ ob, int rows, int n, void* __restrict__ y,
                              vq_dtype yt, int64_t ldy) {
  const int64_t total = static_cast<int64_t>(rows) * n;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = i / n, o = i - b * n;
    store_out(y, yt, b * ldy + o, h2f(ob[o]));
  }
}

template <int D, int NB, int BT>
cudaError_t launch_bt(const Layer& L, const GemvPlan& p, const void* x, bool x_fp16, int batch,
                      int64_t ldx, void* y, vq_dtype yt, int64_t ldy, float* ws,
                      cudaStream_t stream) {
  auto k = L.layout == VQ_IDX_TILE4 ? gemv_kernel<D, NB, BT, true> : gemv_kernel<D, NB, BT, false>;
  cudaError_t e = set_func_attr(reinterpret_cast<const void*>(k), cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.grid_x, p.nsplit);
  count_launch();
  k<<<grid, kGvThreads, p.smem, stream>>>(L, static_cast<const uint16_t*>(x), x_fp16 ? 1 : 0, batch,
                                          ldx, p.vps, p.rpb, p.books_in_smem, p.book_bytes, y, yt,
                                          ldy, p.nsplit > 1 ? ws : nullptr);
  return cudaGetLastError();
}

template <int D, int NB>
cudaError_t launch_d(const Layer& L, const GemvPlan& p, const void* x, bool xf, int batch,
                     int64_t ldx, void* y, vq_dtype yt, int64_t ldy, float* ws, cudaStream_t s) {
  switch (p.bt) {
    case 1: return launch_bt<D, NB, 1>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
    case 2: return launch_bt<D, NB, 2>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
    case 4: return launch_bt<D, NB, 4>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
    case 8: return launch_bt<D, NB, 8>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
    default: return launch_bt<D, NB, 16>(L, p, x, xf, batch, ldx, y, yt, ldy, ws, s);
  }
}

}  // namespace

vq_status plan_gemv(const Layer& L, int batch, GemvPlan* p, size_t ws_cap) {
  if (L.layout == VQ_IDX_TILE4) {
    // small batches: the lookup-table kernels; larger batches of 2^16-book
    // layers: the tensor-core kernel; everything else: the split-K gather
    // kernel below, reading the tiled records
    if (plan_gemv_lut(L, batch, ws_cap, p)) return VQ_OK;
    if (plan_gemv_tc(L, batch, ws_cap, p)) return VQ_OK;
  } else {
    if (batch >= 2 && plan_gemv_tc(L, batch, ws_cap, p)) return VQ_OK;
    if (batch == 1 && gemv1_supported(L)) {
      plan_gemv1(L, p);
      if (p->smem <= device_smem_optin()) return VQ_OK;
    }
    if (gemvb_supported(L, batch)) {
      plan_gemvb(L, batch, p);
      if (p->smem <= device_smem_optin()) return VQ_OK;
    }
  }
  *p = GemvPlan{};
  p->fast = 0;
  int bt = 1;
  while (bt < batch) bt <<= 1;
  p->bt = bt;
  int mask = 0;
  const size_t books = stage_plan(L, kGvSmemBooks, &mask);
  p->books_in_smem = mask;
  p->book_bytes = static_cast<int>(books);
  const size_t x_budget = std::max<size_t>(16 * 1024, kGvSmemBlock - std::min(books, kGvSmemBlock));
  const size_t per_vec = static_cast<size_t>(bt) * L.d * sizeof(float);
  int vps_max = static_cast<int>(x_budget / per_vec) / 32 * 32;
  vps_max = std::max(32, vps_max);
  const int nvec = std::max(1, L.nvec);
  const int nsplit_min = (nvec + vps_max - 1) / vps_max;
  p->rpb = 64;
  const int nrb = std::max(1, (L.n + p->rpb - 1) / p->rpb);
  const int sms = device_sm_count();
  const int target = 2 * sms;
  int nsplit = std::max(nsplit_min, std::min((target + nrb - 1) / nrb, (nvec + 31) / 32));
  int vps = ((nvec + nsplit - 1) / nsplit + 31) / 32 * 32;
  nsplit = (nvec + vps - 1) / vps;
  p->nsplit = nsplit;
  p->vps = vps;
  p->smem = static_cast<int>(books + sizeof(float) * (static_cast<size_t>(bt) * L.d * vps + bt));
  const int blocks_per_sm = std::max(1, static_cast<int>((228 * 1024) / (p->smem + 1024)));
  const int resident = sms * std::min(blocks_per_sm, 8);
  p->grid_x = std::max(1, std::min(nrb, (resident + nsplit - 1) / nsplit));
  p->ws_bytes = nsplit > 1 ? static_cast<size_t>(nsplit) * batch * L.n * sizeof(float) : 0;
  if (p->smem > device_smem_optin()) return VQ_ERR_UNSUPPORTED;
  return VQ_OK;
}

vq_status launch_empty_rows(const Layer& L, void* y, vq_dtype yt, int64_t ldy, int rows,
                            cudaStream_t stream) {
  if (!L.ob) {   // y = 0: all-zero bits in every output type
    const size_t es = yt == VQ_FP32 ? 4 : 2;
    return cuda_status(cudaMemset2DAsync(y, ldy * es, 0, L.n * es, rows, stream));
  }
  const int64_t total = static_cast<int64_t>(rows) * L.n;
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 4 * device_sm_count()));
  count_launch();
  fill_out_bias<<<blocks, 256, 0, stream>>>(L.ob, rows, L.n, y, yt, ldy);
  return cuda_status(cudaGetLastError());
}

vq_status launch_gemv(const Layer& L, const GemvPlan& p, const void* x, bool x_fp16, int batch,
                      int64_t ldx, void* y, vq_dtype yt, int64_t ldy, float* ws,
                      cudaStream_t stream) {
  if (L.n == 0 || batch == 0) return VQ_OK;
  if (L.kin == 0) return launch_empty_rows(L, y, yt, ldy, batch, stream);
  const int D = (L.d == 8) ? 8 : (L.d == 6 ? 6 : 0);
  cudaError_t e;
  if (p.fast == 7 || p.fast == 8) {
    return launch_gemv_tc(L, p, x, x_fp16, batch, ldx, y, yt, ldy, ws, stream);
  } else if (p.fast >= 3) {
    return cuda_status(launch_gemv_lut(L, p, x, x_fp16, batch, ldx, y, yt, ldy, ws, stream));
  } else if (p.fast == 1) {
    e = launch_gemv1(L, p, x, x_fp16, y, yt, ws, stream);
  } else if (p.fast == 2) {
    e = launch_gemvb(L, p, x, x_fp16, batch, ldx, y, yt, ldy, ws, stream);
  } else if (L.nb == 1) {
    e = D == 8 ? launch_d<8, 1>(L, p, x, x_fp16, batch, ldx, y, yt, ldy, ws, stream)
      : D == 6 ? launch_d<6, 1>(L, p, x, x_fp16, batch, ldx, y, yt, ldy, ws, stream)
               : launch_d<0, 1>(L, p, x, x_fp16, batch, ldx, y, yt, ldy, ws, stream);
  } else {
    e = D == 8 ? launch_d<8, 2>(L, p, x, x_fp16, batch, ldx, y, yt, ldy, ws, stream)
      : D == 6 ? launch_d<6, 2>(L, p, x, x_fp16, batch, ldx, y, yt, ldy, ws, stream)
               : launch_d<0, 2>(L, p, x, x_fp16, batch, ldx, y, yt, ldy, ws, stream);
  }
  if (e == cudaSuccess && p.nsplit > 1) {
    const int64_t total = static_cast<int64_t>(batch) * L.n;
    const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 4 * device_sm_count()));
    count_launch();
    gemv_finalize<<<blocks, 256, 0, stream>>>(ws, p.nsplit, batch, L.n, y, yt, ldy);
    e = cudaGetLastError();
  }
  return cuda_status(e);
}

}  // namespace vqk

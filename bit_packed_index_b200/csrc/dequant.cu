// dequant.cu -- vq_dequant: W_hat = fp16((C1[i1] + C2[i2]) * s + t), bit-exact.
//
// Follows "VPTQ Guide: Extreme 2-Bit Vector Quantization", section "Step 2"
// (dequantize: gather both codebooks, add, reshape to (out, in)) with the
// per-row scale and bias of the layer, in the fixed fp32 order documented in
// include/vq.h.  Every fp32 operation is an explicitly rounded intrinsic
// (__fadd_rn / __fmul_rn), so no multiply-add contraction can change a bit.
//
// Work split: persistent blocks loop over output rows; each thread owns whole
// d-vectors (consecutive threads -> consecutive vectors, so index reads and
// W_hat stores are coalesced).  Books that fit are staged once per block in
// shared memory; 2^16-entry books are read through L1/L2.  For d = 8 with an
// aligned destination a vector is written with one 16-byte store.
#include <algorithm>

#include "codebook.cuh"

namespace vqk {
namespace {

constexpr int kDqThreads = 256;
constexpr size_t kDqSmemBooks = 96 * 1024;   // stage books up to this size

template <int D, int NB>
__global__ void __launch_bounds__(kDqThreads) dequant_kernel(Layer L, uint16_t* __restrict__ w,
                                                             int64_t ldw, int smem_mask,
                                                             int vec_store) {
  extern __shared__ __align__(16) uint8_t smem[];
  // reads only the layer: a programmatic dependent may be scheduled at once
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
    if (smem_mask) __syncthreads();
  }
  const int d = (D > 0) ? D : L.d;
  // Centroid row k of book m: staged rows from shared memory; for an
  // L2-served d = 8 book an evict-last load keeps its rows in L1.
  auto fetch = [&](int m, uint32_t k, float* c) {
    if (D == 8 && !(smem_mask & (1 << m))) {
      uint4 v;
      asm volatile("ld.global.nc.L1::evict_last.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                   : "l"(bv[m].base + static_cast<size_t>(k) * 8));
      unpack8(v, c);
    } else {
      load_centroid<D>(bv[m], k, d, c);
    }
  };
  for (int64_t o = blockIdx.x; o < L.n; o += gridDim.x) {
    const bool has_s = L.scale != nullptr, has_t = L.bias != nullptr;
    const float s = has_s ? h2f(L.scale[o]) : 1.0f;
    const float t = has_t ? h2f(L.bias[o]) : 0.0f;
    const uint32_t* row0 = L.idx[0] + o * L.rw[0];
    const uint32_t* row1 = (NB == 2) ? L.idx[1] + o * L.rw[1] : nullptr;
    uint16_t* wrow = w + o * ldw;
    // Two vectors per thread per step: both index fields and both gathers are
    // issued before either result is used.
    for (int j0 = threadIdx.x; j0 < L.nvec; j0 += 2 * blockDim.x) {
      const int jv[2] = {j0, j0 + static_cast<int>(blockDim.x)};
      const bool ok1 = jv[1] < L.nvec;
      uint32_t i1[2], i2[2] = {0u, 0u};
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int j = ok1 || u == 0 ? jv[u] : jv[0];
        i1[u] = load_field(row0, static_cast<int64_t>(j) * L.b[0], L.b[0]);
        if constexpr (NB == 2) i2[u] = load_field(row1, static_cast<int64_t>(j) * L.b[1], L.b[1]);
      }
      float c[2][kMaxVecDim];
#pragma unroll
      for (int u = 0; u < 2; ++u) fetch(0, i1[u], c[u]);
      if constexpr (NB == 2) {
        float c2[2][kMaxVecDim];
#pragma unroll
        for (int u = 0; u < 2; ++u) fetch(1, i2[u], c2[u]);
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int e = 0; e < kMaxVecDim; ++e)
            if (e < d) c[u][e] = __fadd_rn(c[u][e], c2[u][e]);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (u == 1 && !ok1) break;
        uint16_t h[kMaxVecDim];
#pragma unroll
        for (int e = 0; e < kMaxVecDim; ++e) {
          if (e < d) {
            float v = c[u][e];
            if (has_s) v = __fmul_rn(v, s);
            if (has_t) v = __fadd_rn(v, t);
            h[e] = f2h(v);
          }
        }
        const int64_t k0 = static_cast<int64_t>(jv[u]) * d;
        if (D == 8 && vec_store && k0 + 8 <= L.kin) {
          uint4 v;
          v.x = h[0] | (static_cast<uint32_t>(h[1]) << 16);
          v.y = h[2] | (static_cast<uint32_t>(h[3]) << 16);
          v.z = h[4] | (static_cast<uint32_t>(h[5]) << 16);
          v.w = h[6] | (static_cast<uint32_t>(h[7]) << 16);
          *reinterpret_cast<uint4*>(wrow + k0) = v;
        } else {
#pragma unroll
          for (int e = 0; e < kMaxVecDim; ++e)
            if (e < d && k0 + e < L.kin) wrow[k0 + e] = h[e];
        }
      }
    }
  }
}

// One wave of persistent blocks: as many as the SMs hold at once (registers
// bound this kernel: 40-44 per thread leave room for 5-6 blocks of 256, not
// 8), at most one per row.
template <int D, int NB>
cudaError_t launch_dq(const Layer& L, uint16_t* w, int64_t ldw, int smem_mask, size_t smem,
                      int vec_store, cudaStream_t stream, bool pdl) {
  auto k = dequant_kernel<D, NB>;
  if (smem > 48 * 1024) {
    cudaError_t e = set_func_attr(reinterpret_cast<const void*>(k), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const int per_sm = std::min(8, resident_blocks_per_sm(reinterpret_cast<const void*>(k), kDqThreads, smem));
  const int grid = static_cast<int>(std::min<int64_t>(L.n, static_cast<int64_t>(device_sm_count()) * per_sm));
  count_launch();
  if (pdl) return launch_pdl(k, grid, kDqThreads, smem, stream, L, w, ldw, smem_mask, vec_store);
  k<<<grid, kDqThreads, smem, stream>>>(L, w, ldw, smem_mask, vec_store);
  return cudaGetLastError();
}

}  // namespace

vq_status launch_dequant(const Layer& L, uint16_t* w, int64_t ldw, cudaStream_t stream, bool pdl) {
  if (L.n == 0 || L.kin == 0) return VQ_OK;
  if (L.layout == VQ_IDX_TILE4) return launch_dequant_tile4(L, w, ldw, stream, pdl);
  int smem_mask = 0;
  const size_t smem = stage_plan(L, std::min<size_t>(kDqSmemBooks, device_smem_optin()), &smem_mask);
  const int vec_store = aligned(w, 16) && (ldw % 8 == 0);
  cudaError_t e;
  const int D = (L.d == 8) ? 8 : (L.d == 6 ? 6 : 0);
  if (L.nb == 1) {
    e = D == 8 ? launch_dq<8, 1>(L, w, ldw, smem_mask, smem, vec_store, stream, pdl)
      : D == 6 ? launch_dq<6, 1>(L, w, ldw, smem_mask, smem, vec_store, stream, pdl)
               : launch_dq<0, 1>(L, w, ldw, smem_mask, smem, vec_store, stream, pdl);
  } else {
    e = D == 8 ? launch_dq<8, 2>(L, w, ldw, smem_mask, smem, vec_store, stream, pdl)
      : D == 6 ? launch_dq<6, 2>(L, w, ldw, smem_mask, smem, vec_store, stream, pdl)
               : launch_dq<0, 2>(L, w, ldw, smem_mask, smem, vec_store, stream, pdl);
  }
  return cuda_status(e);
}

Layer layer_rows(const Layer& L, int n0, int n1) {
  Layer v = L;
  v.n = n1 - n0;
  for (int m = 0; m < 2; ++m) {
    if (L.layout == VQ_IDX_TILE4)   // records of row o start at bit 4 o b of every tile
      v.idx[m] = L.idx[m] + static_cast<int64_t>(n0) * 4 * L.b[m] / 32;
    else
      v.idx[m] = L.idx[m] + static_cast<int64_t>(n0) * L.rw[m];
  }
  if (L.scale) v.scale = L.scale + n0;
  if (L.bias) v.bias = L.bias + n0;
  if (L.ob) v.ob = L.ob + n0;
  return v;
}

}  // namespace vqk

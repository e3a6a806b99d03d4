// rht.cu -- the randomized Hadamard transform of QuIP#-style incoherence
// processing (vq_rht) and the decode product of a layer stored in the
// transformed basis (vq_gemv_rht): W~ = U W V^T is what the index streams
// encode, so y = W x = U^T (W~ (V x)).  "Vector Quantization for LLM Weights
// in Production", section "1. QuIP#: Incoherence Processing and Lattice
// Codebooks" (W~ = U W V^T, x~ = V x, U and V randomized Walsh-Hadamard
// matrices); "Sub-4-Bit Quantization", section "QuIP#: Incoherence
// Processing" (Hadamard plus random signs, O(d log d)).
//
// A row of length n is transformed in blocks of b = the largest power of two
// dividing n (at most 2^15): forward y = H_b diag(s) x / sqrt(b), inverse
// y = diag(s) H_b x / sqrt(b), H_b Sylvester's Hadamard matrix, s = -1 where
// the sign bit is set.  One thread block per (row, block): the b values are
// staged in shared memory as fp32 and go through log2(b) butterfly stages
// (the fast Walsh-Hadamard transform, natural order), fp32 throughout.
#include <algorithm>
#include <cmath>

#include <cooperative_groups.h>

#include "vq_internal.cuh"

namespace vqk {
namespace {

namespace cg = cooperative_groups;

constexpr int kRhtMaxBlock = 32768;

int rht_block(int64_t n) {
  if (n <= 0) return 0;
  int b = 1;
  while (b < kRhtMaxBlock && n % (2 * static_cast<int64_t>(b)) == 0) b *= 2;
  return b;
}

__device__ __forceinline__ float rht_load(const void* p, int t, int64_t i) {
  if (t == VQ_FP32) return static_cast<const float*>(p)[i];
  const uint16_t u = static_cast<const uint16_t*>(p)[i];
  return t == VQ_FP16 ? h2f(u) : bf2f(u);
}

__device__ __forceinline__ float rht_sign(const uint32_t* __restrict__ signs, int64_t t) {
  return (__ldg(signs + (t >> 5)) >> (t & 31)) & 1u ? -1.0f : 1.0f;
}

// grid (n / b, rows); dynamic shared memory b floats.  `add` (fp16 [n], may
// be null) is added to every output row after the transform.
__global__ void rht_kernel(const void* __restrict__ in, int in_t, int64_t ld_in, int b,
                           const uint32_t* __restrict__ signs, int inverse, float scale,
                           void* __restrict__ out, int out_t, int64_t ld_out, const uint16_t* __restrict__ add) {
  extern __shared__ float hv[];
  // launched as a programmatic dependent (launch_pdl): the input may be the
  // previous kernel's output
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t row = blockIdx.y;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * b;
  for (int i = threadIdx.x; i < b; i += blockDim.x) {
    float v = rht_load(in, in_t, row * ld_in + k0 + i);
    if (!inverse) v *= rht_sign(signs, k0 + i);
    hv[i] = v;
  }
  __syncthreads();
  for (int lh = 0; (1 << lh) < b; ++lh) {
    const int h = 1 << lh;
    for (int p = threadIdx.x; p < b / 2; p += blockDim.x) {
      const int i = ((p >> lh) << (lh + 1)) | (p & (h - 1));
      const float a = hv[i], c = hv[i + h];
      hv[i] = a + c;
      hv[i + h] = a - c;
    }
    __syncthreads();
  }
  for (int i = threadIdx.x; i < b; i += blockDim.x) {
    float v = hv[i] * scale;
    if (inverse) v *= rht_sign(signs, k0 + i);
    v += out_bias_of(add, static_cast<int>(k0 + i));
    store_out(out, static_cast<vq_dtype>(out_t), row * ld_out + k0 + i, v);
  }
}

// Blocks of b >= 256: T = min(1024, b / 8) threads, E = b / T consecutive
// elements per thread.  Stages h < E run in registers, E <= h < 32 E between
// the lanes of a warp (shuffles), the rest through shared memory.
template <int E>
__global__ void __launch_bounds__(1024) rht_big_kernel(const void* __restrict__ in, int in_t, int64_t ld_in,
                                                       int b, const uint32_t* __restrict__ signs, int inverse,
                                                       float scale, void* __restrict__ out, int out_t,
                                                       int64_t ld_out, const uint16_t* __restrict__ add) {
  extern __shared__ float hv[];
  asm volatile("griddepcontrol.wait;" ::: "memory");      // as rht_kernel
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int t = threadIdx.x, T = blockDim.x;
  const int64_t row = blockIdx.y;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * b;
  const int64_t base = k0 + static_cast<int64_t>(t) * E;
  float v[E];
#pragma unroll
  for (int r = 0; r < E; ++r) {
    v[r] = rht_load(in, in_t, row * ld_in + base + r);
    if (!inverse) v[r] *= rht_sign(signs, base + r);
  }
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int r = 0; r < E; ++r) {
      if ((r & h) == 0) {
        const float a = v[r], c = v[r + h];
        v[r] = a + c;
        v[r + h] = a - c;
      }
    }
  }
#pragma unroll
  for (int m = 1; m < 32 && m * E < b; m <<= 1) {   // partner thread t ^ m, same register
    const bool upper = (t & m) != 0;
#pragma unroll
    for (int r = 0; r < E; ++r) {
      const float o = __shfl_xor_sync(0xffffffffu, v[r], m);
      v[r] = upper ? o - v[r] : v[r] + o;
    }
  }
  if (32 * E < b) {
#pragma unroll
    for (int r = 0; r < E; ++r) hv[t * E + r] = v[r];
    __syncthreads();
    for (int lh = 0; (1 << lh) < b; ++lh) {
      const int h = 1 << lh;
      if (h < 32 * E) continue;
      for (int p = t; p < b / 2; p += T) {
        const int i = ((p >> lh) << (lh + 1)) | (p & (h - 1));
        const float a = hv[i], c = hv[i + h];
        hv[i] = a + c;
        hv[i + h] = a - c;
      }
      __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < E; ++r) v[r] = hv[t * E + r];
  }
#pragma unroll
  for (int r = 0; r < E; ++r) {
    float y = v[r] * scale;
    if (inverse) y *= rht_sign(signs, base + r);
    y += out_bias_of(add, static_cast<int>(base + r));
    store_out(out, static_cast<vq_dtype>(out_t), row * ld_out + base + r, y);
  }
}

// Blocks of b = 1024 C (C = 2, 4 or 8): a cluster of C CTAs transforms one
// block, 1024 elements per CTA (128 threads x 8).  Stages h < 1024 run
// inside each CTA as in rht_big_kernel (registers, shuffles, two through
// shared memory); the last log2(C) stages pair CTA r with CTA r ^ (h / 1024)
// and read the partner's elements through distributed shared memory, from a
// second buffer so no CTA overwrites what its partner still reads.  One
// thread block per Hadamard block leaves one SM to do all the work at batch 1
// (8192 elements: 10.6 us); the cluster spreads it over C SMs.
constexpr int kRhtClThreads = 128;
constexpr int kRhtClElems = 1024;

template <int C>
__global__ void __cluster_dims__(C, 1, 1) __launch_bounds__(kRhtClThreads)
    rht_cluster_kernel(const void* __restrict__ in, int in_t, int64_t ld_in, const uint32_t* __restrict__ signs,
                       int inverse, float scale, void* __restrict__ out, int out_t, int64_t ld_out,
                       const uint16_t* __restrict__ add) {
  constexpr int E = 8;
  __shared__ float hv[2][kRhtClElems];
  asm volatile("griddepcontrol.wait;" ::: "memory");      // as rht_kernel
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int t = threadIdx.x;
  const int64_t row = blockIdx.y;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x / C) * (C * kRhtClElems) + static_cast<int64_t>(rank) * kRhtClElems;
  const int64_t base = k0 + static_cast<int64_t>(t) * E;
  float v[E];
#pragma unroll
  for (int r = 0; r < E; ++r) {
    v[r] = rht_load(in, in_t, row * ld_in + base + r);
    if (!inverse) v[r] *= rht_sign(signs, base + r);
  }
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int r = 0; r < E; ++r) {
      if ((r & h) == 0) {
        const float a = v[r], c = v[r + h];
        v[r] = a + c;
        v[r + h] = a - c;
      }
    }
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {                 // h = 8 .. 128
    const bool upper = (t & m) != 0;
#pragma unroll
    for (int r = 0; r < E; ++r) {
      const float o = __shfl_xor_sync(0xffffffffu, v[r], m);
      v[r] = upper ? o - v[r] : v[r] + o;
    }
  }
  // h = 256 and 512 through shared memory (element i at hv[0][i])
#pragma unroll
  for (int r = 0; r < E; ++r) hv[0][t * E + r] = v[r];
  __syncthreads();
#pragma unroll
  for (int lh = 8; lh < 10; ++lh) {
    const int h = 1 << lh;
#pragma unroll
    for (int q = 0; q < kRhtClElems / 2 / kRhtClThreads; ++q) {
      const int p = t + q * kRhtClThreads;
      const int i = ((p >> lh) << (lh + 1)) | (p & (h - 1));
      const float a = hv[0][i], c = hv[0][i + h];
      hv[0][i] = a + c;
      hv[0][i + h] = a - c;
    }
    __syncthreads();
  }
  // h = 1024 C' for C' < C: across the cluster
  int cur = 0;
#pragma unroll
  for (int q = 1; q < C; q <<= 1) {
    cluster.sync();                                   // every CTA's buffer `cur` is complete
    const float* peer = cluster.map_shared_rank(&hv[cur][0], rank ^ q);
    const bool upper = (rank & q) != 0;
#pragma unroll
    for (int r = 0; r < E; ++r) {
      const int i = t * E + r;
      const float mine = hv[cur][i], other = peer[i];
      hv[cur ^ 1][i] = upper ? other - mine : mine + other;
    }
    cur ^= 1;
  }
  cluster.sync();                                     // no CTA exits while a peer still reads it
#pragma unroll
  for (int r = 0; r < E; ++r) {
    float y = hv[cur][t * E + r] * scale;
    if (inverse) y *= rht_sign(signs, base + r);
    y += out_bias_of(add, static_cast<int>(base + r));
    store_out(out, static_cast<vq_dtype>(out_t), row * ld_out + base + r, y);
  }
}

template <int C>
cudaError_t launch_rht_cluster(const void* in, vq_dtype in_t, int rows, int n, int64_t ld_in,
                               const uint32_t* signs, bool inverse, void* out, vq_dtype out_t, int64_t ld_out,
                               cudaStream_t stream, const uint16_t* add) {
  const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(C * kRhtClElems)));
  count_launch();
  return launch_pdl(rht_cluster_kernel<C>, dim3(n / kRhtClElems, rows), kRhtClThreads, 0, stream, in,
                    static_cast<int>(in_t), ld_in, signs, inverse ? 1 : 0, scale, out, static_cast<int>(out_t),
                    ld_out, add);
}

cudaError_t launch_rht(const void* in, vq_dtype in_t, int rows, int n, int64_t ld_in, const uint32_t* signs,
                       bool inverse, void* out, vq_dtype out_t, int64_t ld_out, cudaStream_t stream,
                       const uint16_t* add = nullptr) {
  const int b = rht_block(n);
  // Few rows: spread each block over a cluster (rows * n / 1024 CTAs)
  if (rows <= 16 && (b == 2048 || b == 4096 || b == 8192)) {
    if (b == 2048) return launch_rht_cluster<2>(in, in_t, rows, n, ld_in, signs, inverse, out, out_t, ld_out, stream, add);
    if (b == 4096) return launch_rht_cluster<4>(in, in_t, rows, n, ld_in, signs, inverse, out, out_t, ld_out, stream, add);
    return launch_rht_cluster<8>(in, in_t, rows, n, ld_in, signs, inverse, out, out_t, ld_out, stream, add);
  }
  if (b >= 256) {
    const int T = std::min(1024, b / 8), E = b / T;
    const int smem = 32 * E < b ? b * static_cast<int>(sizeof(float)) : 0;
    const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(b)));
    auto k = E == 8 ? rht_big_kernel<8> : E == 16 ? rht_big_kernel<16> : rht_big_kernel<32>;
    cudaError_t e = set_func_attr(reinterpret_cast<const void*>(k), cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    count_launch();
    return launch_pdl(k, dim3(n / b, rows), T, smem, stream, in, static_cast<int>(in_t), ld_in, b, signs,
                      inverse ? 1 : 0, scale, out, static_cast<int>(out_t), ld_out, add);
  }
  const int smem = b * static_cast<int>(sizeof(float));
  cudaError_t e = set_func_attr(reinterpret_cast<const void*>(rht_kernel), cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int threads = std::min(1024, std::max(32, b / 2));
  const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(b)));
  count_launch();
  return launch_pdl(rht_kernel, dim3(n / b, rows), threads, smem, stream, in, static_cast<int>(in_t), ld_in, b,
                    signs, inverse ? 1 : 0, scale, out, static_cast<int>(out_t), ld_out, add);
}

size_t rht_round256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace of vq_gemv_rht: x~ (fp16 [batch][ldt]), y~ (fp32 [batch][N]),
// then the GEMV's own workspace.
struct RhtLayout {
  int64_t ldt;
  size_t off_y, off_g, gemv_bytes, total;
};

vq_status rht_layout(const vq_layer_desc* layer, const Layer& L, int32_t batch, RhtLayout* r) {
  r->ldt = (static_cast<int64_t>(L.kin) + 7) / 8 * 8;
  r->off_y = rht_round256(static_cast<size_t>(batch) * r->ldt * 2);
  r->off_g = r->off_y + rht_round256(static_cast<size_t>(batch) * L.n * 4);
  vq_status st = gemv_workspace_bytes(layer, batch, ~static_cast<size_t>(0), &r->gemv_bytes);
  if (st != VQ_OK) return st;
  r->total = r->off_g + r->gemv_bytes;
  return VQ_OK;
}

}  // namespace
}  // namespace vqk

using namespace vqk;

extern "C" {

vq_status vq_rht(const void* in, vq_dtype in_dtype, int32_t rows, int32_t n, int64_t ld_in, const uint32_t* signs,
                 int32_t inverse, void* out, vq_dtype out_dtype, int64_t ld_out, void* stream) {
  if (rows < 0 || n < 0 || ld_in < n || ld_out < n) return VQ_ERR_INVALID_ARG;
  if (in_dtype != VQ_BF16 && in_dtype != VQ_FP16 && in_dtype != VQ_FP32) return VQ_ERR_INVALID_ARG;
  if (out_dtype != VQ_BF16 && out_dtype != VQ_FP16 && out_dtype != VQ_FP32) return VQ_ERR_INVALID_ARG;
  if (rows == 0 || n == 0) return VQ_OK;
  if (rows > 65535) return VQ_ERR_UNSUPPORTED;
  if (!in || !out || !signs) return VQ_ERR_INVALID_ARG;
  const size_t ei = in_dtype == VQ_FP32 ? 4 : 2, eo = out_dtype == VQ_FP32 ? 4 : 2;
  if (!aligned(in, ei) || !aligned(out, eo) || !aligned(signs, 4)) return VQ_ERR_ALIGNMENT;
  return cuda_status(launch_rht(in, in_dtype, rows, n, ld_in, signs, inverse != 0, out, out_dtype, ld_out,
                                static_cast<cudaStream_t>(stream)));
}

vq_status vq_gemv_rht_workspace_size(const vq_layer_desc* layer, int32_t batch, size_t* bytes) {
  if (!bytes) return VQ_ERR_INVALID_ARG;
  Layer L;
  vq_status st = check_layer(layer, &L);
  if (st != VQ_OK) return st;
  if (batch < 0) return VQ_ERR_INVALID_ARG;
  if (batch > kMaxBatch) return VQ_ERR_UNSUPPORTED;
  if (batch == 0 || L.n == 0) {
    *bytes = 0;
    return VQ_OK;
  }
  RhtLayout r;
  st = rht_layout(layer, L, batch, &r);
  if (st != VQ_OK) return st;
  *bytes = r.total;
  return VQ_OK;
}

vq_status vq_gemv_rht(const vq_layer_desc* layer, const uint32_t* signs_in, const uint32_t* signs_out,
                      const void* x, vq_dtype x_dtype, int32_t batch, int64_t ldx, void* y, vq_dtype y_dtype,
                      int64_t ldy, void* workspace, size_t workspace_bytes, void* stream_) {
  Layer L;
  vq_status st = check_layer(layer, &L);
  if (st != VQ_OK) return st;
  if (batch < 0 || (x_dtype != VQ_BF16 && x_dtype != VQ_FP16)) return VQ_ERR_INVALID_ARG;
  if (y_dtype != VQ_BF16 && y_dtype != VQ_FP16 && y_dtype != VQ_FP32) return VQ_ERR_INVALID_ARG;
  if (batch > kMaxBatch) return VQ_ERR_UNSUPPORTED;
  if (ldx < L.kin || ldy < L.n) return VQ_ERR_INVALID_ARG;
  if (batch == 0 || L.n == 0) return VQ_OK;
  if (!y || !signs_out || (L.kin > 0 && (!x || !signs_in))) return VQ_ERR_INVALID_ARG;
  RhtLayout r;
  st = rht_layout(layer, L, batch, &r);
  if (st != VQ_OK) return st;
  if (!workspace || workspace_bytes < r.total) return VQ_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return VQ_ERR_ALIGNMENT;
  if (!aligned(x, 2) || !aligned(y, y_dtype == VQ_FP32 ? 4 : 2) || !aligned(signs_out, 4) ||
      (signs_in && !aligned(signs_in, 4)))
    return VQ_ERR_ALIGNMENT;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* xt = reinterpret_cast<uint16_t*>(ws);
  float* yt = reinterpret_cast<float*>(ws + r.off_y);
  if (L.kin > 0) {
    cudaError_t e = launch_rht(x, x_dtype, batch, L.kin, ldx, signs_in, false, xt, VQ_FP16, r.ldt, stream);
    if (e != cudaSuccess) return cuda_status(e);
  }
  // The output bias belongs to y, not to y~: the inverse transform adds it.
  vq_layer_desc inner = *layer;
  inner.out_bias = nullptr;
  st = gemv_run(&inner, xt, VQ_FP16, batch, r.ldt, yt, VQ_FP32, L.n, r.gemv_bytes ? ws + r.off_g : nullptr,
                r.gemv_bytes, ~static_cast<size_t>(0), stream);
  if (st != VQ_OK) return st;
  return cuda_status(launch_rht(yt, VQ_FP32, batch, L.n, L.n, signs_out, true, y, y_dtype, ldy, stream, L.ob));
}

}  // extern "C"

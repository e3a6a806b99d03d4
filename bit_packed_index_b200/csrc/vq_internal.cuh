// vq_internal.cuh -- shared pieces of libvq's kernels and host entry points.
//
// The storage format, the layer description and what each call computes are
// documented in include/vq.h.  This header holds the validated, by-value copy
// of a layer that kernels receive, the index-field extraction, and the fp16 /
// bf16 conversions (CUDA's own intrinsics).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "vq.h"

namespace vqk {

constexpr int kMaxVecDim = 16;
constexpr int kMaxBatch = 16;

// A validated layer, passed to kernels by value.
struct Layer {
  int n;            // out_features
  int kin;          // in_features
  int d;            // vector length
  int nb;           // number of codebooks (1 or 2)
  int nvec;         // ceil(kin / d)
  int b[2];         // index width per book
  int64_t rw[2];    // stream row (row order) or tile (tiled order) stride, 32-bit words
  const uint32_t* idx[2];
  const uint16_t* book[2];
  const uint16_t* scale;  // may be null
  const uint16_t* bias;   // may be null
  const uint16_t* ob;     // output bias added to y after the product, may be null
  int layout;             // VQ_IDX_ROWS or VQ_IDX_TILE4
};

// ---------------------------------------------------------------------------
// Host helpers (vq_api.cu).
// ---------------------------------------------------------------------------
vq_status check_layer(const vq_layer_desc* desc, Layer* out);
// The GEMV entry points, with the largest workspace the caller can give
// (vq_gemv: unlimited; vq_gemv_noalloc: its fixed scratch array).
vq_status gemv_workspace_bytes(const vq_layer_desc* layer, int32_t batch, size_t cap, size_t* bytes);
vq_status gemv_run(const vq_layer_desc* layer, const void* x, vq_dtype x_dtype, int32_t batch,
                   int64_t ldx, void* y, vq_dtype y_dtype, int64_t ldy, void* workspace,
                   size_t workspace_bytes, size_t cap, cudaStream_t stream);
vq_status cuda_status(cudaError_t e);  // records e, returns VQ_ERR_CUDA (or VQ_OK)
void count_launch(int n = 1);          // adds to the process-wide kernel launch counter
int device_sm_count();
// cudaFuncSetAttribute, remembered per (device, kernel, attribute): a call
// that would not change the value launches nothing and costs a table lookup.
cudaError_t set_func_attr(const void* func, cudaFuncAttribute attr, int value);
int device_smem_optin();               // max dynamic shared memory per block, bytes
// Blocks of `func` (threads per block, dynamic shared memory) that one SM
// holds at once, from the occupancy calculator (registers, shared memory,
// threads), remembered per (device, kernel, shape); at least 1.  A
// grid-stride kernel sized past SMs x this runs a partial second wave.
int resident_blocks_per_sm(const void* func, int threads, size_t smem);

__host__ __device__ inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Launch `kernel` as a programmatic dependent of the previous work on the
// stream: it may start while that kernel drains, and must execute
// griddepcontrol.wait before it reads what that kernel wrote or writes what
// that kernel reads.  (Without a trigger in the previous kernel it starts
// when that kernel completes, as a plain launch would.)
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// Kernel launchers (one per .cu file).
// ---------------------------------------------------------------------------
// pdl: launched as a programmatic dependent (it reads only the layer, so it
// may overlap the kernel before it; that kernel must not read w).
vq_status launch_dequant(const Layer& L, uint16_t* w, int64_t ldw, cudaStream_t stream, bool pdl = false);
// Rows n0 .. n1-1 of L as a layer of their own (n0 a multiple of 32).
Layer layer_rows(const Layer& L, int n0, int n1);
// y of a layer without inputs (Kin = 0): its output bias, else zeros (gemv.cu).
vq_status launch_empty_rows(const Layer& L, void* y, vq_dtype yt, int64_t ldy, int rows,
                            cudaStream_t stream);

// Tiled index order (tile4.cu).
vq_status launch_repack_tile4(const Layer& src, uint32_t* const dst[2], const int64_t tile_words[2],
                              cudaStream_t stream);
vq_status launch_dequant_tile4(const Layer& L, uint16_t* w, int64_t ldw, cudaStream_t stream, bool pdl = false);

struct GemvPlan {
  int bt;        // batch tile (power of two >= batch)
  int nsplit;    // K splits
  int vps;       // vectors per split (multiple of 32)
  int rpb;       // rows per work item
  int grid_x;    // blocks per split
  int smem;      // dynamic shared memory bytes
  int books_in_smem;  // bit m set: book m staged in shared memory
  int book_bytes;     // shared memory taken by the staged books
  size_t ws_bytes;
  int fast = 0;       // 0: split-K gather kernel (gemv.cu, either index order),
                      // 1: single-row kernel (gemv1.cu), 2: batched kernel (gemvb.cu),
                      // 3: lookup-table kernel (2^16 book), 5: lookup-table kernel for
                      // books of <= 2^12 entries (tile4.cu, tiled order, batch 1),
                      // 7: tensor-core batched decode, 2^16 book (gemvtc.cu),
                      // 8: the same for books staged in shared memory
};
// ws_cap: largest workspace the caller can provide (plans that need more
// either shrink, for the tiled kernels, or are reported by their ws_bytes).
vq_status plan_gemv(const Layer& L, int batch, GemvPlan* plan, size_t ws_cap = ~static_cast<size_t>(0));
// Lookup-table plans (tiled order; a batch runs one table pass per row of x,
// up to a per-layer limit); false when no table kernel applies.
bool plan_gemv_lut(const Layer& L, int batch, size_t ws_cap, GemvPlan* plan);
// Hessian of a layer's inputs on the tensor cores (gemm.cu).
size_t hessian_workspace_bytes(int n_tokens, int d);
vq_status launch_hessian(const void* x, bool x_fp16, int n_tokens, int d, int64_t ldx, float* h, int64_t ldh,
                         void* workspace, size_t workspace_bytes, cudaStream_t stream);

// Layers sharing x in one table launch (tiled 2^16 books, batch 1).
struct LutMultiPlan {
  int grid;
  int rb8;      // row-sum batches of all layers (power of two)
  int lb;       // batches per layer (power of two)
  int kind;     // 0: 2^16-book kernel, 1: paired-row small-book kernel
  int smem;     // dynamic shared memory of the table kernel
  size_t ws_bytes;
};
bool plan_gemv_lut_multi(const Layer* layers, int n_layers, int batch, size_t ws_cap, LutMultiPlan* plan);
cudaError_t launch_gemv_lut_multi(const Layer* layers, int n_layers, const LutMultiPlan& plan, const void* x,
                                  bool x_fp16, void* const* y, vq_dtype y_dtype, float* ws, cudaStream_t stream);
cudaError_t launch_gemv_lut(const Layer& L, const GemvPlan& plan, const void* x, bool x_fp16, int batch,
                            int64_t ldx, void* y, vq_dtype y_dtype, int64_t ldy, float* ws,
                            cudaStream_t stream);
bool gemv1_supported(const Layer& L);
bool gemvb_supported(const Layer& L, int batch);
void plan_gemvb(const Layer& L, int batch, GemvPlan* plan);
cudaError_t launch_gemvb(const Layer& L, const GemvPlan& plan, const void* x, bool x_fp16, int batch,
                         int64_t ldx, void* y, vq_dtype y_dtype, int64_t ldy, float* ws,
                         cudaStream_t stream);
void plan_gemv1(const Layer& L, GemvPlan* plan);
cudaError_t launch_gemv1(const Layer& L, const GemvPlan& plan, const void* x, bool x_fp16, void* y,
                         vq_dtype y_dtype, float* ws, cudaStream_t stream);
vq_status launch_gemv(const Layer& L, const GemvPlan& plan, const void* x, bool x_fp16, int batch,
                      int64_t ldx, void* y, vq_dtype y_dtype, int64_t ldy, float* ws,
                      cudaStream_t stream);

// TMA map of a 2-D fp16 tensor [rows][cols] (row stride ld elements), box
// {64, box_rows}, 128-byte swizzle, zero fill past the edges (gemm.cu).
bool make_map_f16_sw128(CUtensorMap* map, const void* base, int64_t cols, int64_t rows, int64_t ld,
                        int box_rows);

// Batched decode on the tensor cores (gemvtc.cu): layers with one 2^16-entry
// d = 8 book, row or tiled order.
bool plan_gemv_tc(const Layer& L, int batch, size_t ws_cap, GemvPlan* plan);
vq_status launch_gemv_tc(const Layer& L, const GemvPlan& plan, const void* x, bool x_fp16, int batch,
                         int64_t ldx, void* y, vq_dtype y_dtype, int64_t ldy, void* ws, cudaStream_t stream);

size_t gemm_workspace_bytes(const Layer& L, int m, bool x_fp16);
vq_status launch_gemm(const Layer& L, const void* x, bool x_fp16, int m, int64_t ldx, void* y,
                      vq_dtype y_dtype, int64_t ldy, void* ws, size_t ws_bytes,
                      cudaStream_t stream);

// ---------------------------------------------------------------------------
// Device helpers.
// ---------------------------------------------------------------------------

// Field j of a stream row: bits [j*b, j*b+b), LSB-first in 32-bit words.  A
// field of b <= 16 bits spans at most two words; the second is read only
// when the field crosses into it, so no read goes past the row.
__device__ __forceinline__ uint32_t load_field(const uint32_t* __restrict__ row, int64_t bit, int b) {
  const int64_t w = bit >> 5;
  const int sh = static_cast<int>(bit & 31);
  const uint32_t lo = __ldg(row + w);
  const uint32_t hi = (sh + b > 32) ? __ldg(row + w + 1) : 0u;
  return __funnelshift_r(lo, hi, sh) & ((1u << b) - 1u);
}

__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }
// Output bias of row o (0 without one).
__device__ __forceinline__ float out_bias_of(const uint16_t* ob, int o) { return ob ? h2f(ob[o]) : 0.0f; }
__device__ __forceinline__ float bf2f(uint16_t h) {
  return __bfloat162float(__ushort_as_bfloat16(h));
}
__device__ __forceinline__ uint16_t f2h(float f) { return __half_as_ushort(__float2half_rn(f)); }
__device__ __forceinline__ uint16_t f2bf(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ void store_out(void* y, vq_dtype t, int64_t i, float v) {
  if (t == VQ_FP32) reinterpret_cast<float*>(y)[i] = v;
  else if (t == VQ_FP16) reinterpret_cast<uint16_t*>(y)[i] = f2h(v);
  else reinterpret_cast<uint16_t*>(y)[i] = f2bf(v);
}

// Copy codebook m into shared memory with rows padded to `pad` halves
// (8 for d <= 8, 16 above), zeros in the padding.
__device__ __forceinline__ void stage_book(uint16_t* dst, const uint16_t* __restrict__ src, int k,
                                           int d, int pad) {
  const int total = k * pad;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int r = i / pad, e = i - r * pad;
    dst[i] = (e < d) ? src[static_cast<int64_t>(r) * d + e] : static_cast<uint16_t>(0);
  }
}

}  // namespace vqk

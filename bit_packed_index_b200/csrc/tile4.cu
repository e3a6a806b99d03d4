// tile4.cu -- kernels for the tiled index order (VQ_IDX_TILE4, include/vq.h):
// the repack from row order, W_hat from a tiled layer, and the decode
// lookup-table GEMVs (batch 1) that the order exists for.  Other batches and
// layers run gemv.cu's split-K kernel, which reads either order.
//
// The lookup-table GEMV ("Vector Quantization for LLM Weights in Production",
// section "2. Lookup Table (LUT) Overhead vs. Bit-Shifting": codebook lookups
// feeding the accumulation; "VPTQ Guide", section "Step 3": y = x . W_hat^T)
// reorders the sum y[o] = sum_j <x_j, C[i(o, j)]> around the codebook instead
// of around the rows.  For a group of four vectors j (one tile) and a slice
// of the 2^16 centroids k (24576, 24576, then 16384) it forms
// T[k][j] = <x_j, C[k]> once -- one 16 x 8 x 16 tensor-core product per 32
// centroids, two centroids per A row -- stores T in shared memory as fp16,
// and then every row adds the entries its four indices select.  A row's
// indices sit side by side in the tiled order and consecutive rows follow one
// another, so each thread reads one 8-byte record per row and a warp reads
// 256 contiguous bytes.  Each (group, slice) is one task; a block owns every
// row of the layer for the tasks it runs, and keeps its per-row sums in
// tensor memory (TMEM) across tasks.  Several layers that read the same x
// run as one task list, each layer's rows in their own TMEM batches.  A
// second kernel, launched as a programmatic dependent, adds the per-block
// sums and applies scale and bias.  Books of at most 2^12 entries use whole
// tables per group (no slices): gemv_lut_small_kernel and, for 12-bit main
// books, gemv_lut_pair_kernel.
#include <algorithm>
#include <cstdlib>

#include "codebook.cuh"
#include "sm100.cuh"

namespace vqk {
namespace {

// ---------------------------------------------------------------------------
// Repack: row order -> tiled order.  One thread per output word; the word's 32
// bits collect every field that overlaps them.  Works for any field width.
// ---------------------------------------------------------------------------
__global__ void repack_tile4_kernel(const uint32_t* __restrict__ src, int64_t src_rw, int b, int n,
                                    int nvec, uint32_t* __restrict__ dst, int64_t tw) {
  const int ntile = (nvec + 3) / 4;
  const int64_t total = static_cast<int64_t>(ntile) * tw;
  const int64_t nbits = static_cast<int64_t>(n) * 4 * b;   // record bits per tile
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / tw;
    const int64_t bit0 = (i - t * tw) * 32;
    uint32_t out = 0;
    if (bit0 < nbits) {
      const int64_t q0 = bit0 / b;
      const int64_t q1 = min((nbits - 1) / b, (bit0 + 31) / b);
      for (int64_t q = q0; q <= q1; ++q) {          // field q = record q/4, slot q%4
        const int64_t o = q >> 2;
        const int64_t j = t * 4 + (q & 3);
        if (j >= nvec) continue;
        const uint32_t v = load_field(src + o * src_rw, j * b, b);
        const int64_t pos = q * b - bit0;            // in (-b, 32)
        out |= pos >= 0 ? (v << pos) : (v >> (-pos));
      }
    }
    dst[i] = out;
  }
}

// ---------------------------------------------------------------------------
// W_hat from a tiled layer.  Work unit = (row, tile): the row's four vectors
// of that tile.  Four consecutive threads take four consecutive tiles of one
// row, so a warp writes 8 rows x 256 contiguous bytes (d = 8) and reads 8
// consecutive records from each of 4 tiles.  Books that fit are staged in
// shared memory as in vq_dequant's row-order kernel.  The fp32 operations and
// their order are that kernel's (centroid sum, times scale, plus bias, one
// fp16 rounding).
// ---------------------------------------------------------------------------
template <int D, int NB>
__global__ void dequant_tile4_kernel(Layer L, uint16_t* __restrict__ w, int64_t ldw, int vec_store,
                                     int smem_mask) {
  // reads only the layer: a programmatic dependent may be scheduled at once
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(16) uint8_t smem[];
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
  const int ntile = (L.nvec + 3) / 4;
  const int ntb = (ntile + 3) / 4;                        // groups of four tiles
  const int64_t total = static_cast<int64_t>(ntb) * L.n * 4;
  const int d = D > 0 ? D : L.d;
  const bool has_s = L.scale != nullptr, has_t = L.bias != nullptr;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t rest = i >> 2;
    const int64_t tb = rest / L.n, o = rest - tb * L.n;
    const int64_t t = tb * 4 + (i & 3);
    if (t >= ntile) continue;
    const float s = has_s ? h2f(L.scale[o]) : 1.0f;
    const float tbias = has_t ? h2f(L.bias[o]) : 0.0f;
    const uint32_t* tile0 = L.idx[0] + t * L.rw[0];
    const uint32_t* tile1 = L.idx[1] + t * L.rw[1];
    uint16_t* wrow = w + o * ldw;
    // The record's four fields and their centroids first (all gathers in
    // flight), then the arithmetic and the stores.
    uint32_t f0[4], f1[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      f0[jj] = load_field(tile0, (o * 4 + jj) * L.b[0], L.b[0]);
      if constexpr (NB == 2) f1[jj] = load_field(tile1, (o * 4 + jj) * L.b[1], L.b[1]);
    }
    constexpr int DM = D > 0 ? D : kMaxVecDim;
    float c[4][DM];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      load_centroid<D>(bv[0], f0[jj], d, c[jj]);
      if constexpr (NB == 2) {
        float c2[DM];
        load_centroid<D>(bv[1], f1[jj], d, c2);
#pragma unroll
        for (int e = 0; e < DM; ++e)
          if (e < d) c[jj][e] = __fadd_rn(c[jj][e], c2[e]);
      }
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int64_t j = t * 4 + jj;
      if (j >= L.nvec) break;
      const int64_t k0 = j * d;
      uint16_t h[DM];
#pragma unroll
      for (int e = 0; e < DM; ++e) {
        if (e < d) {
          float v = c[jj][e];
          if (has_s) v = __fmul_rn(v, s);
          if (has_t) v = __fadd_rn(v, tbias);
          h[e] = f2h(v);
        }
      }
      if (D == 8 && vec_store == 2 && k0 + 8 <= L.kin) {      // one 16-byte store
        *reinterpret_cast<uint4*>(wrow + k0) =
            make_uint4(h[0] | (static_cast<uint32_t>(h[1]) << 16), h[2] | (static_cast<uint32_t>(h[3]) << 16),
                       h[4] | (static_cast<uint32_t>(h[5]) << 16), h[6] | (static_cast<uint32_t>(h[7]) << 16));
      } else if (D == 6 && vec_store >= 1 && k0 + 6 <= L.kin) {  // three 4-byte stores
#pragma unroll
        for (int e = 0; e < 6; e += 2)
          *reinterpret_cast<uint32_t*>(wrow + k0 + e) = h[e] | (static_cast<uint32_t>(h[e + 1]) << 16);
      } else {
#pragma unroll
        for (int e = 0; e < DM; ++e)
          if (e < d && k0 + e < L.kin) wrow[k0 + e] = h[e];
      }
    }
  }
}

constexpr size_t kDq4SmemBooks = 96 * 1024;   // stage books up to this size

template <int D, int NB>
cudaError_t launch_dq4(const Layer& L, uint16_t* w, int64_t ldw, cudaStream_t stream, bool pdl) {
  int smem_mask = 0;
  const size_t smem = stage_plan(L, std::min<size_t>(kDq4SmemBooks, device_smem_optin()), &smem_mask);
  auto k = dequant_tile4_kernel<D, NB>;
  if (smem > 48 * 1024) {
    cudaError_t e = set_func_attr(reinterpret_cast<const void*>(k), cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  // one wave: a grid-stride loop past what the SMs hold runs a partial second wave
  const int per_sm = std::min(8, resident_blocks_per_sm(reinterpret_cast<const void*>(k), 256, smem));
  const int64_t total = static_cast<int64_t>((((L.nvec + 3) / 4) + 3) / 4) * L.n * 4;
  const int grid = static_cast<int>(std::min<int64_t>((total + 255) / 256,
                                                      static_cast<int64_t>(device_sm_count()) * per_sm));
  // 2: 16-byte rows of 8 halves aligned; 1: 4-byte pairs aligned (rows of even length)
  const int vec_store = (aligned(w, 16) && ldw % 8 == 0) ? 2 : (aligned(w, 4) && ldw % 2 == 0) ? 1 : 0;
  count_launch();
  if (pdl) return launch_pdl(k, grid, 256, smem, stream, L, w, ldw, vec_store, smem_mask);
  k<<<grid, 256, smem, stream>>>(L, w, ldw, vec_store, smem_mask);
  return cudaGetLastError();
}

}  // namespace

vq_status launch_repack_tile4(const Layer& L, uint32_t* const dst[2], const int64_t tw[2],
                              cudaStream_t stream) {
  for (int m = 0; m < L.nb; ++m) {
    const int64_t total = static_cast<int64_t>((L.nvec + 3) / 4) * tw[m];
    const int grid = static_cast<int>(std::min<int64_t>((total + 255) / 256, 16LL * device_sm_count()));
    count_launch();
    repack_tile4_kernel<<<grid, 256, 0, stream>>>(L.idx[m], L.rw[m], L.b[m], L.n, L.nvec, dst[m], tw[m]);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e);
  }
  return VQ_OK;
}

vq_status launch_dequant_tile4(const Layer& L, uint16_t* w, int64_t ldw, cudaStream_t stream, bool pdl) {
  if (L.n == 0 || L.kin == 0) return VQ_OK;
  cudaError_t e;
  if (L.nb == 1)
    e = L.d == 8 ? launch_dq4<8, 1>(L, w, ldw, stream, pdl)
      : L.d == 6 ? launch_dq4<6, 1>(L, w, ldw, stream, pdl) : launch_dq4<0, 1>(L, w, ldw, stream, pdl);
  else
    e = L.d == 8 ? launch_dq4<8, 2>(L, w, ldw, stream, pdl)
      : L.d == 6 ? launch_dq4<6, 2>(L, w, ldw, stream, pdl) : launch_dq4<0, 2>(L, w, ldw, stream, pdl);
  return cuda_status(e);
}


namespace {

__device__ __forceinline__ float x_at(const uint16_t* __restrict__ x, int x_fp16, int64_t i) {
  const uint16_t u = __ldg(x + i);
  return x_fp16 ? h2f(u) : bf2f(u);
}

}  // namespace


namespace {

// ---------------------------------------------------------------------------
// Decode lookup-table GEMV (batch 1; one book; d = 8; 16-bit indices).
// ---------------------------------------------------------------------------
constexpr int kLutThreads = 1024;
constexpr int kLutNJ = 4;                           // vectors per task: one tile
constexpr int kLutS = 24576;                        // centroids per slice (the last: 16384)
constexpr int kLutSlices = (65536 + kLutS - 1) / kLutS;   // 3 slices of the 2^16 book
constexpr int kLutSmem = kLutS * kLutNJ * 2;        // T[S][4] in fp16: 192 KB
constexpr int kLutPD = 4;                           // 32-centroid tiles per load batch

__device__ __forceinline__ uint2 ldg_stream64(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// The table products of a 2^16 book run as m16n8k16 with two centroids per A
// row: row r of a 32-centroid tile is centroids 2r and 2r+1 (16 consecutive
// halves), B column n < 4 holds x'_n against the even centroid and n >= 4
// x'_(n-4) against the odd one, so all eight output columns are table entries
// and every lane stores.  Any permutation of k serves if A and B share it: lane
// (n = lane/4, t = lane%4) takes k = {2t, 2t+1} and {2t+8, 2t+9} from the four
// consecutive halves 4t..4t+3 of its row, one 8-byte load.  Those halves are
// components 4(t%2)..+3 of the even (t < 2) or odd (t >= 2) centroid, so the
// lane's B pair is x' of vector n%4 at those components when t/2 == n/4, zero
// otherwise.  x' = x * 2^-e with ||x'_j||_1 < 1 for the group's four vectors,
// so no product overflows fp16; the return value is 2^e.  *xpart gets the
// lane's share of the group's sum of x (each element counted once per warp).
__device__ __forceinline__ float lut_pair_bfrag(const uint16_t* __restrict__ x, int x_fp16, int kin, int g,
                                                int lane, uint32_t (&bf)[2], float* xpart) {
  const int n = lane >> 2, t = lane & 3;
  const int k0 = (g * kLutNJ + (n & 3)) * 8 + 4 * (t & 1);
  float v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint16_t u = k0 + i < kin ? __ldg(x + k0 + i) : static_cast<uint16_t>(0);
    v[i] = x_fp16 ? h2f(u) : bf2f(u);
  }
  float l1 = (fabsf(v[0]) + fabsf(v[1])) + (fabsf(v[2]) + fabsf(v[3]));
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);       // the vector's other half
  float mx = l1;
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  // e: the exponent with mx = m * 2^e, 0.5 <= m < 1, read from the bits
  // (-126 for a subnormal mx, which only makes x' smaller); 0 when mx is
  // zero or not finite.  2^-e is applied as two factors 2^-(e/2) and
  // 2^-(e - e/2), each a normal float for every e in [-126, 128], so x' is
  // the exactly scaled x (or rounds to zero only where fp16 would anyway).
  int e = 0;
  if (mx > 0.0f && mx < INFINITY) e = static_cast<int>(__float_as_uint(mx) >> 23) - 126;
  const float f1 = __uint_as_float(static_cast<uint32_t>(127 - e / 2) << 23);
  const float f2 = __uint_as_float(static_cast<uint32_t>(127 - (e - e / 2)) << 23);
  const bool on = (t >> 1) == (n >> 2);
  const __half2 h0 = __floats2half2_rn(on ? v[0] * f1 * f2 : 0.0f, on ? v[1] * f1 * f2 : 0.0f);
  const __half2 h1 = __floats2half2_rn(on ? v[2] * f1 * f2 : 0.0f, on ? v[3] * f1 * f2 : 0.0f);
  bf[0] = *reinterpret_cast<const uint32_t*>(&h0);
  bf[1] = *reinterpret_cast<const uint32_t*>(&h1);
  *xpart = (n < 4 && t < 2) ? (v[0] + v[1]) + (v[2] + v[3]) : 0.0f;
  return __uint_as_float(static_cast<uint32_t>(127 + e) << 23);   // 2^e (inf for e = 128)
}

// e with mx = m * 2^e, 0.5 <= m < 1, from the float bits (-126 for a
// subnormal mx; 0 when mx is zero or not finite), and x * 2^-e as two exact
// power-of-two factors (each a normal float for e in [-126, 128]).
__device__ __forceinline__ int lut_exp(float mx) {
  return (mx > 0.0f && mx < INFINITY) ? static_cast<int>(__float_as_uint(mx) >> 23) - 126 : 0;
}
__device__ __forceinline__ float lut_scale_down(float v, int e) {
  const float f1 = __uint_as_float(static_cast<uint32_t>(127 - e / 2) << 23);
  const float f2 = __uint_as_float(static_cast<uint32_t>(127 - (e - e / 2)) << 23);
  return v * f1 * f2;
}
__device__ __forceinline__ float lut_pow2(int e) {               // 2^e (inf for e = 128)
  return __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
}

// One 32-centroid tile: D = A x B (fp32), A = afr (rows g and g+8 of the
// tile, each an 8-byte load), then the eight table entries of this lane in
// fp16.  Lane (n, t) owns T[32*tile + 2n + t/2][2(t%2), +1] and the same for
// row n+8; a warp's two stores are 128 contiguous bytes each.
__device__ __forceinline__ void lut_pair_mma_store(const uint32_t (&afr)[4], const uint32_t (&bf)[2],
                                                   uint16_t* __restrict__ lut, int tile, int lane) {
  float d0, d1, d2, d3;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %11, %12, %13};"
      : "=f"(d0), "=f"(d1), "=f"(d2), "=f"(d3)
      : "r"(afr[0]), "r"(afr[1]), "r"(afr[2]), "r"(afr[3]), "r"(bf[0]), "r"(bf[1]), "f"(0.0f), "f"(0.0f),
        "f"(0.0f), "f"(0.0f));
  uint16_t* p = lut + tile * 32 * kLutNJ + 2 * lane;   // = T[32 tile + 2n + t/2][2(t%2)]
  *reinterpret_cast<__half2*>(p) = __floats2half2_rn(d0, d1);
  *reinterpret_cast<__half2*>(p + 16 * kLutNJ) = __floats2half2_rn(d2, d3);
}

// A operand of one 32-centroid tile read from the book (rows n and n+8 of
// the tile: centroids 32 tile + 2n, +1 and 32 tile + 2n + 16, +17).
__device__ __forceinline__ void lut_pair_afr(const uint16_t* __restrict__ bslice, int tile, int lane,
                                             uint32_t (&afr)[4]) {
  const uint16_t* c = bslice + tile * 32 * 8 + 4 * lane;
  const uint2 r0 = ldg_stream64(c);
  const uint2 r1 = ldg_stream64(c + 16 * 8);
  afr[0] = r0.x;   // row n,   k = 2t, 2t+1
  afr[1] = r1.x;   // row n+8, k = 2t, 2t+1
  afr[2] = r0.y;   // row n,   k = 2t+8, 2t+9
  afr[3] = r1.y;   // row n+8, k = 2t+8, 2t+9
}

// One or more layers that share x (the projections of one block), run as one
// task list.  Layer l's rows occupy the 8192-row batches l*LB .. l*LB+LB-1 of
// the block's row sums, so a batch never mixes layers.
constexpr int kLutMaxLayers = 4;
struct LutSet {
  Layer L[kLutMaxLayers];
  int nl;
  int row0[kLutMaxLayers + 1];   // first row of each layer in the partial sums; row0[nl] = rows
};

// RB8 batches of 8 rows per thread (all layers together): a block covers
// 8 * RB8 * 1024 rows; thread (warp w, lane l) keeps its row sums in TMEM lane
// 32*(w%4)+l, columns (w/4)*8*RB8 .. +8*RB8 (warps may only touch their own
// quarter of the lanes).  Tasks: (group of four vectors, layer, slice), the
// three slices of one layer and group consecutive.
template <int RB8, int LB>
__global__ void __launch_bounds__(kLutThreads, 1) gemv_lut_kernel(LutSet S, const uint16_t* __restrict__ x,
                                                                  int x_fp16, float* __restrict__ part,
                                                                  float* __restrict__ xpart) {
  constexpr int CPW = 8 * RB8;                      // TMEM columns per group of 4 warps
  constexpr int TCOLS = 8 * CPW;                    // 64 .. 512, a power of two
  constexpr int NBATCH = kLutS / 32 / (kLutThreads / 32) / kLutPD;   // batches, full slice
  static_assert(kLutS % (32 * (kLutThreads / 32) * kLutPD) == 0 &&
                (65536 % kLutS) % (32 * (kLutThreads / 32) * kLutPD) == 0,
                "every slice splits into whole load batches per warp");
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* lut = reinterpret_cast<uint16_t*>(smem);   // T[k - slice base][kLutNJ vectors]
  __shared__ uint32_t s_tmem;
  __shared__ float s_scale;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr bool MULTI = LB < RB8;                  // several layers, LB batches each
  const int kin = S.L[0].kin;
  const int nl = MULTI ? S.nl : 1;
  const int ntot = S.row0[nl];                       // rows of the block's partial sums
  const int ntasks = ((S.L[0].nvec + kLutNJ - 1) / kLutNJ) * nl * kLutSlices;

  if (warp == 0) {
    sm100::tmem_alloc(&s_tmem, TCOLS);
    sm100::tmem_relinquish();
  }
  // The reduction launch may be scheduled now; it waits for this grid's
  // completion (griddepcontrol.wait) before reading anything.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tbase = s_tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) +
                         static_cast<uint32_t>((warp >> 2) * CPW);
  {
    float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int b = 0; b < RB8; ++b) sm100::tmem_st8(tbase + 8 * b, z);
    sm100::tmem_wait_st();
  }
  // Launched as a programmatic dependent: x may come from the kernel before
  // (a transform of it); everything above overlapped that kernel's tail.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float xs_acc = 0.0f;   // warp 0: sum of x, one group per slice-0 task

  // Work items: the tasks of the whole rounds, then the last partial round's
  // tasks split by 8192-row batches over the blocks that would idle (each
  // piece builds the task's table, then does its share of the lookups).
  const int full = (ntasks / static_cast<int>(gridDim.x)) * static_cast<int>(gridDim.x);
  const int tail = ntasks - full;
  int nbat_max = 1;
  for (int l = 0; l < nl; ++l) nbat_max = max(nbat_max, (S.L[l].n + 8 * kLutThreads - 1) / (8 * kLutThreads));
  const int parts = tail > 0 ? max(1, min(nbat_max, static_cast<int>(gridDim.x) / tail)) : 1;
  const int nitems = full + tail * parts;
  for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
    int task = item, part = 0, nparts = 1;
    if (item >= full) {
      const int q = item - full;
      part = q % parts;
      nparts = parts;
      task = full + q / parts;
    }
    const int g = task / (nl * kLutSlices);
    const int ls = task - g * nl * kLutSlices;
    const int l = MULTI ? ls / kLutSlices : 0, s = ls - l * kLutSlices;
    const Layer& L = S.L[l];
    const int n = L.n;
    // this layer's LB row-sum batches (rows past n unused)
    const int bb0 = l * LB;
    constexpr int nbat = LB;
    const int nb_used = MULTI ? (n + 8 * kLutThreads - 1) / (8 * kLutThreads) : nbat_max;
    const int b_lo = part * nb_used / nparts, b_hi = (part + 1) * nb_used / nparts;
    // Phase A operands of the first load batch go out before the activations
    // are read, so the two latencies overlap.
    const uint16_t* bslice = L.book[0] + static_cast<size_t>(s) * kLutS * 8;
    const int slice_n = min(kLutS, 65536 - s * kLutS);
    const int tpw = slice_n / 32 / (kLutThreads / 32);        // tiles per warp
    const int nb = tpw / kLutPD;                                // load batches
    const int t0w = warp * tpw;
    uint32_t afr[2][kLutPD][4];
#pragma unroll
    for (int p = 0; p < kLutPD; ++p) lut_pair_afr(bslice, t0w + p, lane, afr[0][p]);
    uint32_t bfrag[2];
    {
      float xp;
      const float sc = lut_pair_bfrag(x, x_fp16, kin, g, lane, bfrag, &xp);
      if (tid == 0) s_scale = sc;
      if (warp == 0 && s == 0 && l == 0 && part == 0) {   // each group of x once
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) xp += __shfl_xor_sync(0xffffffffu, xp, off);
        xs_acc += xp;
      }
    }
    // Phase A: T for this slice.  Warp w builds its share of the slice's
    // 32-centroid tiles, the A operands read straight from the codebook, two
    // load batches in flight.
    {
#pragma unroll
      for (int bt = 0; bt < NBATCH; ++bt) {
        if (bt >= nb) break;                        // uniform: the slice's own size
        const int cur = bt & 1;
        if (bt + 1 < nb) {
#pragma unroll
          for (int p = 0; p < kLutPD; ++p) lut_pair_afr(bslice, t0w + (bt + 1) * kLutPD + p, lane, afr[cur ^ 1][p]);
        }
#pragma unroll
        for (int p = 0; p < kLutPD; ++p) lut_pair_mma_store(afr[cur][p], bfrag, lut, t0w + bt * kLutPD + p, lane);
      }
    }
    __syncthreads();   // T complete
    // Phase B: every row adds the T entries its four indices select from this
    // slice; the records come straight from global memory, two batches of 8
    // rows in flight, and the running sums live in TMEM.
    {
      const float sc = s_scale;
      const uint2* trow = reinterpret_cast<const uint2*>(L.idx[0] + static_cast<int64_t>(g) * L.rw[0]);
      uint2 w[2][8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int o = r * kLutThreads + tid;
        w[0][r] = o < n ? ldg_stream64(trow + o) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int b = 0; b < RB8; ++b) {               // b: this layer's batch
        if (b >= nbat) break;                        // uniform
        const int cur = b & 1;
        if (b + 1 < nbat) {
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const int o = ((b + 1) * 8 + r) * kLutThreads + tid;
            w[cur ^ 1][r] = o < n ? ldg_stream64(trow + o) : make_uint2(0u, 0u);
          }
        }
        if (b < b_lo || b >= b_hi) continue;         // uniform: another piece's rows
        const uint32_t tb = tbase + 8 * (bb0 + b);
        float acc[8];
        sm100::tmem_ld8(tb, acc);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          // uniform: no thread has this row (a 28672-row layer's last batch
          // is half empty; its lookups would be an eighth of the work).  Not
          // compiled for one-batch layers: the test alone slowed the 8192-row
          // down_proj by 3 %, which has no such rows.
          if constexpr (LB > 1)
            if ((b * 8 + r) * kLutThreads >= n) break;
          float v = 0.0f;
#pragma unroll
          for (int jj = 0; jj < kLutNJ; ++jj) {
            const uint32_t k = ((jj < 2 ? w[cur][r].x : w[cur][r].y) >> (16 * (jj & 1))) & 0xFFFFu;
            const uint32_t t = k - static_cast<uint32_t>(s * kLutS);   // wraps when below
            if (t < static_cast<uint32_t>(kLutS)) v += h2f(lut[t * kLutNJ + jj]);
          }
          acc[r] = fmaf(v, sc, acc[r]);
        }
        sm100::tmem_st8(tb, acc);
      }
      sm100::tmem_wait_st();
    }
    __syncthreads();   // all lookups done before the next task rewrites T
  }

  // Partial sums of every row of every layer, layers one after another.
  for (int l = 0; l < nl; ++l) {
    const int n = S.L[l].n;
    float* dst = part + static_cast<int64_t>(blockIdx.x) * ntot + S.row0[l];
#pragma unroll
    for (int b = 0; b < LB; ++b) {
      float acc[8];
      sm100::tmem_ld8(tbase + 8 * (l * LB + b), acc);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int o = (b * 8 + r) * kLutThreads + tid;
        if (o < n) dst[o] = acc[r];
      }
    }
  }
  if (tid == 0) xpart[blockIdx.x] = xs_acc;
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  if (warp == 0) sm100::tmem_dealloc(s_tmem, TCOLS);
}

// ---------------------------------------------------------------------------
// Lookup-table GEMV for small books (batch 1; d = 6 or 8; one or two books of
// at most 2^12 centroids each).  The whole table of a group of four vectors
// fits in shared memory -- T_m[k][4] for each book, at most 64 KB -- so a task
// is one group, each index is looked up exactly once and there is no slice
// test.  Records of 4 fields are 4*b_m bits wide and read with a bit-exact
// funnel (consecutive rows share words, so the loads go through L1).  The
// rest is the 2^16 kernel's structure: tensor-core table products, row sums in
// TMEM, per-block sums added by gemv_lut_finalize.
// ---------------------------------------------------------------------------
constexpr int kLutSmallMaxTiles = 8;                 // 16-centroid tiles per warp: K <= 4096

// The 4*b-bit record of row o in a tiled stream (b <= 12: at most 48 bits,
// spread over up to three words; only words holding record bits are read).
__device__ __forceinline__ uint64_t load_record(const uint32_t* __restrict__ tile, int64_t o, int b) {
  const int64_t p = o * 4 * b;
  const uint32_t* w = tile + (p >> 5);
  const int sh = static_cast<int>(p & 31);
  const int nbits = 4 * b;
  const uint64_t lo = __ldg(w);
  const uint64_t mid = (sh + nbits > 32) ? __ldg(w + 1) : 0u;
  uint64_t r = ((mid << 32) | lo) >> sh;
  if (sh + nbits > 64) r |= static_cast<uint64_t>(__ldg(w + 2)) << (64 - sh);
  return r;
}

// Table of one book for the task's four vectors: T[k][j] = <x'_j, C[k]>, in
// two planes of K 4-byte words (plane p, word k: T[k][2p], T[k][2p+1]) that
// start small_plane(K) halves apart.  A lookup instruction's lanes (one j,
// random k) then spread over all 32 banks -- one 8-byte row T[k][0..3] per
// centroid would put a given j in only 16 of them -- and a warp's stores
// (8 consecutive words in each plane) hit 16 distinct banks.
__device__ __forceinline__ int small_plane(int K) { return 2 * K + 32; }

template <int D>
__device__ __forceinline__ void build_small_table(const uint16_t* __restrict__ book, int K, uint32_t bfrag,
                                                  uint16_t* __restrict__ tab, int warp, int lane) {
  const int tiles = (K + 15) / 16;
  const int g = lane >> 2, t = lane & 3;
  uint32_t a[kLutSmallMaxTiles][2];
#pragma unroll
  for (int i = 0; i < kLutSmallMaxTiles; ++i) {
    const int tile = warp + 32 * i;
    const int r0 = tile * 16 + g, r1 = r0 + 8;
    const bool cok = 2 * t < D;                       // d = 6: components 6, 7 are zero
    a[i][0] = (tile < tiles && r0 < K && cok) ? __ldg(reinterpret_cast<const uint32_t*>(book + r0 * D + 2 * t)) : 0u;
    a[i][1] = (tile < tiles && r1 < K && cok) ? __ldg(reinterpret_cast<const uint32_t*>(book + r1 * D + 2 * t)) : 0u;
  }
#pragma unroll
  for (int i = 0; i < kLutSmallMaxTiles; ++i) {
    const int tile = warp + 32 * i;
    if (tile >= tiles) break;                          // uniform per warp
    float d0, d1, d2, d3;
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
        "{%7, %8, %9, %10};"
        : "=f"(d0), "=f"(d1), "=f"(d2), "=f"(d3)
        : "r"(a[i][0]), "r"(a[i][1]), "r"(bfrag), "f"(0.0f), "f"(0.0f), "f"(0.0f), "f"(0.0f));
    const int r0 = tile * 16 + g;
    if (t < 2) {
      uint16_t* plane = tab + t * small_plane(K);
      if (r0 < K) *reinterpret_cast<__half2*>(plane + r0 * 2) = __floats2half2_rn(d0, d1);
      if (r0 + 8 < K) *reinterpret_cast<__half2*>(plane + (r0 + 8) * 2) = __floats2half2_rn(d2, d3);
    }
  }
}

// The same table as fp32, one array per vector (T[j][k], K entries apart), for
// the paired-row kernel: a lookup is one 4-byte load, and lanes that read the
// same vector's array spread over all 32 banks.
template <int D>
__device__ __forceinline__ void build_small_table_f32(const uint16_t* __restrict__ book, int K, uint32_t bfrag,
                                                      float* __restrict__ tab, int warp, int lane) {
  const int tiles = (K + 15) / 16;
  const int g = lane >> 2, t = lane & 3;
  uint32_t a[kLutSmallMaxTiles][2];
#pragma unroll
  for (int i = 0; i < kLutSmallMaxTiles; ++i) {
    const int tile = warp + 32 * i;
    const int r0 = tile * 16 + g, r1 = r0 + 8;
    const bool cok = 2 * t < D;
    a[i][0] = (tile < tiles && r0 < K && cok) ? __ldg(reinterpret_cast<const uint32_t*>(book + r0 * D + 2 * t)) : 0u;
    a[i][1] = (tile < tiles && r1 < K && cok) ? __ldg(reinterpret_cast<const uint32_t*>(book + r1 * D + 2 * t)) : 0u;
  }
#pragma unroll
  for (int i = 0; i < kLutSmallMaxTiles; ++i) {
    const int tile = warp + 32 * i;
    if (tile >= tiles) break;
    float d0, d1, d2, d3;
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
        "{%7, %8, %9, %10};"
        : "=f"(d0), "=f"(d1), "=f"(d2), "=f"(d3)
        : "r"(a[i][0]), "r"(a[i][1]), "r"(bfrag), "f"(0.0f), "f"(0.0f), "f"(0.0f), "f"(0.0f));
    const int r0 = tile * 16 + g;
    if (t < 2) {
      if (r0 < K) {
        tab[(2 * t) * K + r0] = d0;
        tab[(2 * t + 1) * K + r0] = d1;
      }
      if (r0 + 8 < K) {
        tab[(2 * t) * K + r0 + 8] = d2;
        tab[(2 * t + 1) * K + r0 + 8] = d3;
      }
    }
  }
}

template <int RB8, int D, int NB>
__global__ void __launch_bounds__(kLutThreads, 1) gemv_lut_small_kernel(Layer L, const uint16_t* __restrict__ x,
                                                                        int x_fp16, float* __restrict__ part,
                                                                        float* __restrict__ xpart) {
  constexpr int CPW = 8 * RB8;
  constexpr int TCOLS = 8 * CPW;
  extern __shared__ __align__(128) uint8_t smem[];
  const int K1 = 1 << L.b[0], K2 = NB == 2 ? (1 << L.b[1]) : 0;
  uint16_t* tab1 = reinterpret_cast<uint16_t*>(smem);   // T1, two planes
  uint16_t* tab2 = tab1 + 2 * small_plane(K1);           // T2, two planes
  __shared__ uint32_t s_tmem;
  __shared__ float s_scale;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = L.n, kin = L.kin;
  const int ntasks = (L.nvec + 3) / 4;

  if (warp == 0) {
    sm100::tmem_alloc(&s_tmem, TCOLS);
    sm100::tmem_relinquish();
  }
  // The reduction launch may be scheduled now; it waits for this grid's
  // completion (griddepcontrol.wait) before reading anything.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tbase = s_tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) +
                         static_cast<uint32_t>((warp >> 2) * CPW);
  {
    float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int b = 0; b < RB8; ++b) sm100::tmem_st8(tbase + 8 * b, z);
    sm100::tmem_wait_st();
  }
  // Launched as a programmatic dependent: x may come from the kernel before
  // (a transform of it); everything above overlapped that kernel's tail.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float xs_acc = 0.0f;

  for (int g = blockIdx.x; g < ntasks; g += gridDim.x) {
    uint32_t bfrag;
    {
      const int jj = lane >> 2, t = lane & 3;
      const int64_t k = (static_cast<int64_t>(g) * 4 + jj) * D + 2 * t;
      float a = 0.0f, b = 0.0f;
      if (jj < 4 && 2 * t < D) {
        if (k < kin) a = x_at(x, x_fp16, k);
        if (k + 1 < kin) b = x_at(x, x_fp16, k + 1);
      }
      float l1 = fabsf(a) + fabsf(b);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      float mx = l1;
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const int e = lut_exp(mx);
      const __half2 h = __floats2half2_rn(lut_scale_down(a, e), lut_scale_down(b, e));
      bfrag = *reinterpret_cast<const uint32_t*>(&h);
      if (tid == 0) s_scale = lut_pow2(e);
      if (warp == 0) {
        float v = a + b;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        xs_acc += v;
      }
    }
    build_small_table<D>(L.book[0], K1, bfrag, tab1, warp, lane);
    if constexpr (NB == 2) build_small_table<D>(L.book[1], K2, bfrag, tab2, warp, lane);
    __syncthreads();   // tables complete
    {
      const float sc = s_scale;
      const uint32_t* tile1 = L.idx[0] + static_cast<int64_t>(g) * L.rw[0];
      const uint32_t* tile2 = L.idx[1] + static_cast<int64_t>(g) * L.rw[1];
      const int b1 = L.b[0], b2 = L.b[1];
      const uint32_t m1 = (1u << b1) - 1u, m2 = (1u << b2) - 1u;
#pragma unroll 1
      for (int b = 0; b < RB8; ++b) {
        if (b * 8 * kLutThreads >= n) break;          // uniform: no row of this batch exists
        // Every record of the batch is requested before any is used (rows past
        // N read row N-1 and are never stored), so the loads overlap.
        uint64_t rec1[8], rec2[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int o = min((b * 8 + r) * kLutThreads + tid, n - 1);
          rec1[r] = load_record(tile1, o, b1);
          if constexpr (NB == 2) rec2[r] = load_record(tile2, o, b2);
        }
        float acc[8];
        sm100::tmem_ld8(tbase + 8 * b, acc);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          if ((b * 8 + r) * kLutThreads >= n) break;  // uniform: no thread has this row
          float v = 0.0f;
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const uint16_t* p1 = tab1 + (jj >> 1) * small_plane(K1) + (jj & 1);
            float u = h2f(p1[(static_cast<uint32_t>(rec1[r] >> (jj * b1)) & m1) * 2]);
            if constexpr (NB == 2) {
              const uint16_t* p2 = tab2 + (jj >> 1) * small_plane(K2) + (jj & 1);
              u += h2f(p2[(static_cast<uint32_t>(rec2[r] >> (jj * b2)) & m2) * 2]);
            }
            v += u;
          }
          acc[r] = fmaf(v, sc, acc[r]);
        }
        sm100::tmem_st8(tbase + 8 * b, acc);
      }
      sm100::tmem_wait_st();
    }
    __syncthreads();   // all lookups done before the next task rewrites the tables
  }

#pragma unroll
  for (int b = 0; b < RB8; ++b) {
    float acc[8];
    sm100::tmem_ld8(tbase + 8 * b, acc);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int o = (b * 8 + r) * kLutThreads + tid;
      if (o < n) part[static_cast<int64_t>(blockIdx.x) * n + o] = acc[r];
    }
  }
  if (tid == 0) xpart[blockIdx.x] = xs_acc;
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  if (warp == 0) sm100::tmem_dealloc(s_tmem, TCOLS);
}

// Rows in pairs, for 12-bit main books (with no second book, or a 4- or
// 8-bit one): two 48-bit records are exactly three words, so every field of
// the pair sits at a fixed bit position and its table byte offset (index * 4)
// takes one shift and one mask.  The tables are fp32, one array per vector
// (build_small_table_f32); a thread's batch is four pairs (8 rows, 8 TMEM
// columns).
template <int B, int Q, int NW>
__device__ __forceinline__ uint32_t field_off(const uint32_t (&w)[NW]) {
  constexpr int bit = Q * B, wi = bit >> 5, sh = bit & 31;
  uint32_t v;
  if constexpr (sh + B <= 32) {
    v = w[wi] >> sh;
  } else {
    v = __funnelshift_r(w[wi], w[wi + 1], sh);
  }
  return (v & ((1u << B) - 1u)) << 2;
}

template <int B, int H, int NW>
__device__ __forceinline__ float row_lookup(const uint32_t (&w)[NW], const uint8_t* tab) {
  // fields 4H .. 4H+3 of the pair: the four vectors of row 2p + H, each in its
  // own array of 2^B floats
  constexpr int stride = 4 << B;
  const float a = *reinterpret_cast<const float*>(tab + field_off<B, 4 * H + 0>(w));
  const float b = *reinterpret_cast<const float*>(tab + field_off<B, 4 * H + 1>(w) + stride);
  const float c = *reinterpret_cast<const float*>(tab + field_off<B, 4 * H + 2>(w) + 2 * stride);
  const float d = *reinterpret_cast<const float*>(tab + field_off<B, 4 * H + 3>(w) + 3 * stride);
  return (a + b) + (c + d);
}

// Layers of one set (S.nl of them, LB batches of 8192 rows each in the row
// sums; one layer: LB = RB8) share x; a task is (group, layer).
template <int RB8, int D, int B2, int LB>
__global__ void __launch_bounds__(kLutThreads, 1) gemv_lut_pair_kernel(LutSet S, const uint16_t* __restrict__ x,
                                                                       int x_fp16, float* __restrict__ part,
                                                                       float* __restrict__ xpart) {
  constexpr bool MULTI = LB < RB8;
  constexpr int B1 = 12;
  constexpr int NB = B2 > 0 ? 2 : 1;
  constexpr int W2 = B2 == 8 ? 2 : 1;               // words per pair of book-2 records
  constexpr int CPW = 8 * RB8;
  constexpr int TCOLS = 8 * CPW;
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int K1 = 1 << B1, K2 = B2 > 0 ? (1 << B2) : 0;
  float* tab1 = reinterpret_cast<float*>(smem);          // T1[4][K1]
  float* tab2 = tab1 + K1 * 4;                           // T2[4][K2]
  __shared__ uint32_t s_tmem;
  __shared__ float s_scale;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kin = S.L[0].kin;
  const int nl = MULTI ? S.nl : 1;
  const int ntot = S.row0[nl];
  const int ntasks = ((S.L[0].nvec + 3) / 4) * nl;

  if (warp == 0) {
    sm100::tmem_alloc(&s_tmem, TCOLS);
    sm100::tmem_relinquish();
  }
  // The reduction launch may be scheduled now; it waits for this grid's
  // completion (griddepcontrol.wait) before reading anything.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tbase = s_tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) +
                         static_cast<uint32_t>((warp >> 2) * CPW);
  {
    float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int b = 0; b < RB8; ++b) sm100::tmem_st8(tbase + 8 * b, z);
    sm100::tmem_wait_st();
  }
  // Launched as a programmatic dependent: x may come from the kernel before
  // (a transform of it); everything above overlapped that kernel's tail.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float xs_acc = 0.0f;

  for (int task = blockIdx.x; task < ntasks; task += gridDim.x) {
    const int g = MULTI ? task / nl : task, l = MULTI ? task - g * nl : 0;
    const Layer& L = S.L[l];
    const int n = L.n;
    const int npairs = (n + 1) / 2;
    const int64_t nw1 = (static_cast<int64_t>(n) * 4 * B1 + 31) / 32;   // words holding records
    const int64_t nw2 = (static_cast<int64_t>(n) * 4 * (B2 > 0 ? B2 : 1) + 31) / 32;
    uint32_t bfrag;
    {
      const int jj = lane >> 2, t = lane & 3;
      const int64_t k = (static_cast<int64_t>(g) * 4 + jj) * D + 2 * t;
      float a = 0.0f, b = 0.0f;
      if (jj < 4 && 2 * t < D) {
        if (k < kin) a = x_at(x, x_fp16, k);
        if (k + 1 < kin) b = x_at(x, x_fp16, k + 1);
      }
      float l1 = fabsf(a) + fabsf(b);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      float mx = l1;
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const int e = lut_exp(mx);
      const __half2 h = __floats2half2_rn(lut_scale_down(a, e), lut_scale_down(b, e));
      bfrag = *reinterpret_cast<const uint32_t*>(&h);
      if (tid == 0) s_scale = lut_pow2(e);
      if (warp == 0 && l == 0) {                    // each group of x once
        float v = a + b;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        xs_acc += v;
      }
    }
    build_small_table_f32<D>(L.book[0], K1, bfrag, tab1, warp, lane);
    if constexpr (NB == 2) build_small_table_f32<D>(L.book[1], K2, bfrag, tab2, warp, lane);
    __syncthreads();   // tables complete
    {
      const float sc = s_scale;
      const uint32_t* tile1 = L.idx[0] + static_cast<int64_t>(g) * L.rw[0];
      const uint32_t* tile2 = L.idx[1] + static_cast<int64_t>(g) * L.rw[1];
      const uint8_t* t1 = reinterpret_cast<const uint8_t*>(tab1);
      const uint8_t* t2 = reinterpret_cast<const uint8_t*>(tab2);
#pragma unroll 1
      for (int b = 0; b < LB; ++b) {
        if (b * 8 * kLutThreads >= n) break;          // uniform: no row of this batch exists
        const uint32_t tb = tbase + 8 * (l * LB + b);
        uint32_t w1[4][3], w2[4][W2];
#pragma unroll
        for (int r = 0; r < 4; ++r) {                 // all loads of the batch first
          const int64_t pi = static_cast<int64_t>(b * 4 + r) * kLutThreads + tid;
#pragma unroll
          for (int i = 0; i < 3; ++i) w1[r][i] = 3 * pi + i < nw1 ? __ldg(tile1 + 3 * pi + i) : 0u;
          if constexpr (NB == 2) {
#pragma unroll
            for (int i = 0; i < W2; ++i) w2[r][i] = W2 * pi + i < nw2 ? __ldg(tile2 + W2 * pi + i) : 0u;
          }
        }
        float acc[8];
        sm100::tmem_ld8(tb, acc);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if ((b * 4 + r) * kLutThreads >= npairs) break;   // uniform: no thread has this pair
          float va = row_lookup<B1, 0>(w1[r], t1);
          float vb = row_lookup<B1, 1>(w1[r], t1);
          if constexpr (NB == 2) {
            va += row_lookup<B2, 0>(w2[r], t2);
            vb += row_lookup<B2, 1>(w2[r], t2);
          }
          acc[2 * r] = fmaf(va, sc, acc[2 * r]);
          acc[2 * r + 1] = fmaf(vb, sc, acc[2 * r + 1]);
        }
        sm100::tmem_st8(tb, acc);
      }
      sm100::tmem_wait_st();
    }
    __syncthreads();   // all lookups done before the next task rewrites the tables
  }

  for (int l = 0; l < nl; ++l) {
    const int n = S.L[l].n;
    float* dst = part + static_cast<int64_t>(blockIdx.x) * ntot + S.row0[l];
#pragma unroll 1
    for (int b = 0; b < LB; ++b) {
      float acc[8];
      sm100::tmem_ld8(tbase + 8 * (l * LB + b), acc);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int64_t o = 2 * (static_cast<int64_t>(b * 4 + (r >> 1)) * kLutThreads + tid) + (r & 1);
        if (o < n) dst[o] = acc[r];
      }
    }
  }
  if (tid == 0) xpart[blockIdx.x] = xs_acc;
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  if (warp == 0) sm100::tmem_dealloc(s_tmem, TCOLS);
}

// y[o] = s[o] * sum_b part[b][o] + t[o] * sum_b xpart[b], in a fixed order.
// 32 rows per block: lane = row, the 8 warps stride the per-block sums with
// every load of a thread in flight at once.  The reduction is bound by load
// latency, so the block is capped at 32 registers per thread: 8 blocks per SM
// and one wave for the 70B layers (896 blocks).
constexpr int kFinU = 20;

// Outputs of a table launch: layer l's rows are rows row0[l] .. row0[l+1]-1
// of the partial sums.
struct LutOut {
  int nl;
  int row0[kLutMaxLayers + 1];
  const uint16_t* scale[kLutMaxLayers];
  const uint16_t* bias[kLutMaxLayers];
  const uint16_t* ob[kLutMaxLayers];     // output bias, may be null
  void* y[kLutMaxLayers];
};

LutOut lut_out_single(const Layer& L, void* y) {
  LutOut o{};
  o.nl = 1;
  o.row0[0] = 0;
  o.row0[1] = L.n;
  o.scale[0] = L.scale;
  o.bias[0] = L.bias;
  o.ob[0] = L.ob;
  o.y[0] = y;
  return o;
}

// y_l[o] = s_l[o] * sum_b part[b][row0_l + o] + t_l[o] * sum_b xpart[b]
// + ob_l[o], the partial sums added in a fixed order.
__global__ void __launch_bounds__(256, 8) gemv_lut_finalize(const float* __restrict__ part,
                                                            const float* __restrict__ xpart, int nparts,
                                                            int ntot, LutOut out, vq_dtype yt) {
  // Launched as a programmatic dependent of the table kernel: wait for that
  // grid to complete and its writes to be visible (a no-op otherwise).  The
  // next launch may then be scheduled (it waits for this grid the same way).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float red[8][33];
  __shared__ float s_xsum;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int v = blockIdx.x * 32 + lane;
  if (warp == 0) {
    float t = 0.0f;
    for (int i = lane; i < nparts; i += 32) t += xpart[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    if (lane == 0) s_xsum = t;
  }
  float acc = 0.0f;
  if (v < ntot) {
    const float* col = part + v;
    for (int b0 = warp; b0 < nparts; b0 += 8 * kFinU) {
      float u[kFinU];
#pragma unroll
      for (int i = 0; i < kFinU; ++i) {
        const int b = b0 + 8 * i;
        u[i] = b < nparts ? col[static_cast<int64_t>(b) * ntot] : 0.0f;
      }
#pragma unroll
      for (int i = 0; i < kFinU; ++i) acc += u[i];
    }
  }
  red[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && v < ntot) {
    float t = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[w][lane];
    int l = 0;
    while (l + 1 < out.nl && v >= out.row0[l + 1]) ++l;
    const int o = v - out.row0[l];
    const float sc = out.scale[l] ? h2f(out.scale[l][o]) : 1.0f;
    const float tb = out.bias[l] ? h2f(out.bias[l][o]) : 0.0f;
    store_out(out.y[l], yt, o, sc * t + tb * s_xsum + out_bias_of(out.ob[l], o));
  }
}

// The reduction of a table launch, as a programmatic dependent launch: its
// blocks are scheduled while the table kernel drains, instead of after it.
cudaError_t launch_finalize(const float* part, const float* xpart, int nparts, int ntot, const LutOut& out,
                            vq_dtype yt, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((ntot + 31) / 32);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, gemv_lut_finalize, part, xpart, nparts, ntot, out, yt);
}

// The layers of S share x; their partial sums take S.row0[S.nl] rows per block.
template <int RB8, int LB>
cudaError_t launch_lut_set(const LutSet& S, const LutOut& out, int grid, const void* x, bool x_fp16,
                           vq_dtype yt, float* ws, cudaStream_t stream) {
  auto k = gemv_lut_kernel<RB8, LB>;
  cudaError_t e = set_func_attr(reinterpret_cast<const void*>(k), cudaFuncAttributeMaxDynamicSharedMemorySize, kLutSmem);
  if (e != cudaSuccess) return e;
  const int ntot = S.row0[S.nl];
  float* part = ws;
  float* xpart = ws + static_cast<int64_t>(grid) * ntot;
  count_launch();
  e = launch_pdl(k, grid, kLutThreads, kLutSmem, stream, S, static_cast<const uint16_t*>(x), x_fp16 ? 1 : 0, part,
                 xpart);
  if (e != cudaSuccess) return e;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_finalize(part, xpart, grid, ntot, out, yt, stream);
}

LutSet lut_set_single(const Layer& L) {
  LutSet S{};
  S.L[0] = L;
  S.nl = 1;
  S.row0[0] = 0;
  S.row0[1] = L.n;
  return S;
}

template <int RB8>
cudaError_t launch_lut(const Layer& L, const GemvPlan& p, const void* x, bool x_fp16, void* y,
                       vq_dtype yt, float* ws, cudaStream_t stream) {
  return launch_lut_set<RB8, RB8>(lut_set_single(L), lut_out_single(L, y), p.grid_x, x, x_fp16, yt, ws, stream);
}

template <int RB8, int D, int NB>
cudaError_t launch_lut_small_t(const Layer& L, const GemvPlan& p, const void* x, bool x_fp16, float* ws,
                               cudaStream_t stream) {
  auto k = gemv_lut_small_kernel<RB8, D, NB>;
  cudaError_t e = set_func_attr(reinterpret_cast<const void*>(k), cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem);
  if (e != cudaSuccess) return e;
  count_launch();
  return launch_pdl(k, p.grid_x, kLutThreads, p.smem, stream, L, static_cast<const uint16_t*>(x), x_fp16 ? 1 : 0,
                    ws, ws + static_cast<int64_t>(p.grid_x) * L.n);
}

bool lut_pair_path(const Layer& L) {
  const int b2 = L.nb == 2 ? L.b[1] : 0;
  return L.b[0] == 12 && (b2 == 0 || b2 == 4 || b2 == 8);
}

template <int RB8, int D, int B2, int LB>
cudaError_t launch_lut_pair_set(const LutSet& S, int grid, int smem, const void* x, bool x_fp16, float* ws,
                                cudaStream_t stream) {
  auto k = gemv_lut_pair_kernel<RB8, D, B2, LB>;
  cudaError_t e = set_func_attr(reinterpret_cast<const void*>(k), cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  count_launch();
  return launch_pdl(k, grid, kLutThreads, smem, stream, S, static_cast<const uint16_t*>(x), x_fp16 ? 1 : 0, ws,
                    ws + static_cast<int64_t>(grid) * S.row0[S.nl]);
}

template <int RB8, int D, int B2>
cudaError_t launch_lut_pair_t(const Layer& L, const GemvPlan& p, const void* x, bool x_fp16, float* ws,
                              cudaStream_t stream) {
  return launch_lut_pair_set<RB8, D, B2, RB8>(lut_set_single(L), p.grid_x, p.smem, x, x_fp16, ws, stream);
}

template <int RB8>
cudaError_t launch_lut_small(const Layer& L, const GemvPlan& p, const void* x, bool x_fp16, void* y,
                             vq_dtype yt, float* ws, cudaStream_t stream) {
  cudaError_t e;
  const int b2 = L.nb == 2 ? L.b[1] : 0;
  if (lut_pair_path(L)) {                                       // rows in pairs, fixed offsets
    if (L.d == 8)
      e = b2 == 0 ? launch_lut_pair_t<RB8, 8, 0>(L, p, x, x_fp16, ws, stream)
        : b2 == 4 ? launch_lut_pair_t<RB8, 8, 4>(L, p, x, x_fp16, ws, stream)
                  : launch_lut_pair_t<RB8, 8, 8>(L, p, x, x_fp16, ws, stream);
    else
      e = b2 == 0 ? launch_lut_pair_t<RB8, 6, 0>(L, p, x, x_fp16, ws, stream)
        : b2 == 4 ? launch_lut_pair_t<RB8, 6, 4>(L, p, x, x_fp16, ws, stream)
                  : launch_lut_pair_t<RB8, 6, 8>(L, p, x, x_fp16, ws, stream);
  } else if (L.d == 8) {
    e = L.nb == 1 ? launch_lut_small_t<RB8, 8, 1>(L, p, x, x_fp16, ws, stream)
                  : launch_lut_small_t<RB8, 8, 2>(L, p, x, x_fp16, ws, stream);
  } else {
    e = L.nb == 1 ? launch_lut_small_t<RB8, 6, 1>(L, p, x, x_fp16, ws, stream)
                  : launch_lut_small_t<RB8, 6, 2>(L, p, x, x_fp16, ws, stream);
  }
  if (e != cudaSuccess) return e;
  return launch_finalize(ws, ws + static_cast<int64_t>(p.grid_x) * L.n, p.grid_x, L.n, lut_out_single(L, y), yt,
                         stream);
}

// Tables of the small-book kernels: fp16 [K][4] per book in two padded
// planes (small_plane), or fp32 [4][K] on the paired-row path.
size_t lut_small_smem(const Layer& L) {
  const size_t k = (static_cast<size_t>(1) << L.b[0]) + (L.nb == 2 ? (static_cast<size_t>(1) << L.b[1]) : 0);
  return lut_pair_path(L) ? k * 4 * 4 : k * 4 * 2 + 2 * 128;
}

bool lut_small_supported(const Layer& L) {
  return L.layout == VQ_IDX_TILE4 && (L.d == 6 || L.d == 8) && L.b[0] <= 12 &&
         (L.nb == 1 || L.b[1] <= 12) && L.n >= 1 && L.n <= 8 * 8 * kLutThreads && L.nvec >= 1 &&
         lut_small_smem(L) + 1024 <= static_cast<size_t>(device_smem_optin());
}

bool lut_supported(const Layer& L) {
  return L.layout == VQ_IDX_TILE4 && L.nb == 1 && L.d == 8 && L.b[0] == 16 && L.n >= 1 &&
         L.n <= 8 * 8 * kLutThreads && L.nvec >= 1 && device_smem_optin() >= kLutSmem + 1024;
}

}  // namespace

cudaError_t launch_gemv_lut_row(const Layer& L, const GemvPlan& p, const void* x, bool x_fp16, void* y,
                                vq_dtype yt, float* ws, cudaStream_t stream);
// Measured crossovers against the tensor-core batched kernels (gemvtc.cu) on
// tiled layers (B200, L2 flushed): the table pass costs about the same per
// row of x whatever the batch, the tensor-core kernels about the same per
// call.  A 2^16 book pays up to batch 2 (70B gate: 169 us at B = 2; the
// tensor-core kernel 190 at any batch).  Books of <= 2^12 entries: up to
// batch 3 on short rows (8B up, 512 vectors per row: 73 us at B = 3 against
// 80) and batch 5 on long ones (405B q, 2731 vectors: 62 us per row of x
// against 309; 405B gate: 136 per row against 856).
constexpr int kLutMaxBatchBig = 2;
constexpr int kLutMaxBatchSmallShort = 3;
constexpr int kLutMaxBatchSmallLong = 5;

// Largest batch served by running the batch-1 table kernel once per row of x
// (each run reads the index streams again); larger batches take the
// tensor-core kernels, else the split-K gather kernel.  Environment override
// for measurements: VQ_LUT_MAX_BATCH.
int lut_batch_limit(const Layer& L, bool big) {
  if (const char* env = std::getenv("VQ_LUT_MAX_BATCH")) return std::atoi(env);
  if (big) return kLutMaxBatchBig;
  return L.nvec > 1024 ? kLutMaxBatchSmallLong : kLutMaxBatchSmallShort;
}

bool plan_gemv_lut(const Layer& L, int batch, size_t ws_cap, GemvPlan* p) {
  const bool big = lut_supported(L), small = !big && lut_small_supported(L);
  if (!(big || small) || batch < 1 || batch > lut_batch_limit(L, big)) return false;
  const int ntasks = ((L.nvec + 3) / 4) * (big ? kLutSlices : 1);
  const size_t per_block = (static_cast<size_t>(L.n) + 1) * sizeof(float);
  int grid = std::min(device_sm_count(), ntasks);
  if (ws_cap / per_block < static_cast<size_t>(grid)) grid = static_cast<int>(ws_cap / per_block);
  if (grid < 1) return false;
  int rb8 = 1;
  while (static_cast<int64_t>(rb8) * 8 * kLutThreads < L.n) rb8 <<= 1;
  *p = GemvPlan{};
  p->nsplit = 1;
  p->fast = big ? 3 : 5;
  p->grid_x = grid;
  p->bt = rb8;
  p->smem = big ? kLutSmem : static_cast<int>(lut_small_smem(L));
  p->ws_bytes = per_block * grid;
  return true;
}

// Several tiled 2^16-book layers that share x, at batch 1: one table launch
// over all their tasks (one reduction launch) when 2..4 layers qualify and
// their rows fit the block's row sums (8 batches of 8192).
bool plan_gemv_lut_multi(const Layer* L, int nl, int batch, size_t ws_cap, LutMultiPlan* p) {
  if (nl < 2 || nl > kLutMaxLayers || batch != 1) return false;
  // All layers 2^16 books (the sliced kernel), or all on the paired-row path
  // with the same vector length and books (d = 6 with 2^12 + 2^4, or d = 8
  // with 2^12 + 2^8: the shapes of the 405B and 8B layers).
  bool big = true, pair = true;
  for (int l = 0; l < nl; ++l) {
    if (L[l].kin != L[0].kin) return false;
    big = big && lut_supported(L[l]);
    pair = pair && lut_small_supported(L[l]) && lut_pair_path(L[l]) && L[l].nb == 2 && L[l].d == L[0].d &&
           L[l].b[1] == L[0].b[1] && ((L[l].d == 6 && L[l].b[1] == 4) || (L[l].d == 8 && L[l].b[1] == 8));
  }
  if (!big && !pair) return false;
  int lb = 1;
  int64_t rows = 0;
  for (int l = 0; l < nl; ++l) {
    while (static_cast<int64_t>(lb) * 8 * kLutThreads < L[l].n) lb <<= 1;
    rows += L[l].n;
  }
  int rb8 = 1;
  while (rb8 < nl * lb) rb8 <<= 1;
  if (pair) rb8 = std::max(rb8, 4);                  // the compiled paired-row shapes
  if (rb8 > 8 || (pair && !((rb8 == 4 && lb <= 2) || (rb8 == 8 && lb == 2)))) return false;
  const int ntasks = ((L[0].nvec + kLutNJ - 1) / kLutNJ) * nl * (big ? kLutSlices : 1);
  const size_t per_block = (static_cast<size_t>(rows) + 1) * sizeof(float);
  int grid = std::min(device_sm_count(), ntasks);
  if (ws_cap / per_block < static_cast<size_t>(grid)) grid = static_cast<int>(ws_cap / per_block);
  if (grid < 1) return false;
  p->grid = grid;
  p->rb8 = rb8;
  p->lb = lb;
  p->kind = big ? 0 : 1;
  p->smem = big ? kLutSmem : static_cast<int>(lut_small_smem(L[0]));
  p->ws_bytes = per_block * grid;
  return true;
}

cudaError_t launch_gemv_lut_multi(const Layer* L, int nl, const LutMultiPlan& p, const void* x, bool x_fp16,
                                  void* const* y, vq_dtype yt, float* ws, cudaStream_t stream) {
  LutSet S{};
  LutOut out{};
  S.nl = out.nl = nl;
  for (int l = 0; l < nl; ++l) {
    S.L[l] = L[l];
    S.row0[l + 1] = out.row0[l + 1] = S.row0[l] + L[l].n;
    out.scale[l] = L[l].scale;
    out.bias[l] = L[l].bias;
    out.ob[l] = L[l].ob;
    out.y[l] = y[l];
  }
  if (p.kind == 1) {                                 // paired-row small-book kernel
    const bool d6 = L[0].d == 6;
    cudaError_t e;
    if (p.rb8 == 8)
      e = d6 ? launch_lut_pair_set<8, 6, 4, 2>(S, p.grid, p.smem, x, x_fp16, ws, stream)
             : launch_lut_pair_set<8, 8, 8, 2>(S, p.grid, p.smem, x, x_fp16, ws, stream);
    else if (p.lb == 2)
      e = d6 ? launch_lut_pair_set<4, 6, 4, 2>(S, p.grid, p.smem, x, x_fp16, ws, stream)
             : launch_lut_pair_set<4, 8, 8, 2>(S, p.grid, p.smem, x, x_fp16, ws, stream);
    else
      e = d6 ? launch_lut_pair_set<4, 6, 4, 1>(S, p.grid, p.smem, x, x_fp16, ws, stream)
             : launch_lut_pair_set<4, 8, 8, 1>(S, p.grid, p.smem, x, x_fp16, ws, stream);
    if (e != cudaSuccess) return e;
    const int ntot = S.row0[nl];
    return launch_finalize(ws, ws + static_cast<int64_t>(p.grid) * ntot, p.grid, ntot, out, yt, stream);
  }
  if (p.rb8 == 2) return launch_lut_set<2, 1>(S, out, p.grid, x, x_fp16, yt, ws, stream);
  if (p.rb8 == 4) return p.lb == 1 ? launch_lut_set<4, 1>(S, out, p.grid, x, x_fp16, yt, ws, stream)
                                   : launch_lut_set<4, 2>(S, out, p.grid, x, x_fp16, yt, ws, stream);
  return p.lb == 2 ? launch_lut_set<8, 2>(S, out, p.grid, x, x_fp16, yt, ws, stream)
                   : launch_lut_set<8, 4>(S, out, p.grid, x, x_fp16, yt, ws, stream);
}

cudaError_t launch_gemv_lut(const Layer& L, const GemvPlan& p, const void* x, bool x_fp16, int batch,
                            int64_t ldx, void* y, vq_dtype yt, int64_t ldy, float* ws, cudaStream_t stream) {
  // One batch-1 table pass per row of x, in stream order (the workspace is
  // reused by each pass).
  const size_t ysz = yt == VQ_FP32 ? 4 : 2;
  for (int b = 0; b < batch; ++b) {
    cudaError_t e = launch_gemv_lut_row(L, p, static_cast<const uint16_t*>(x) + b * ldx, x_fp16,
                                        static_cast<char*>(y) + b * ldy * ysz, yt, ws, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_gemv_lut_row(const Layer& L, const GemvPlan& p, const void* x, bool x_fp16, void* y,
                                vq_dtype yt, float* ws, cudaStream_t stream) {
  if (p.fast == 3) {
    switch (p.bt) {
      case 1: return launch_lut<1>(L, p, x, x_fp16, y, yt, ws, stream);
      case 2: return launch_lut<2>(L, p, x, x_fp16, y, yt, ws, stream);
      case 4: return launch_lut<4>(L, p, x, x_fp16, y, yt, ws, stream);
      default: return launch_lut<8>(L, p, x, x_fp16, y, yt, ws, stream);
    }
  }
  switch (p.bt) {
    case 1: return launch_lut_small<1>(L, p, x, x_fp16, y, yt, ws, stream);
    case 2: return launch_lut_small<2>(L, p, x, x_fp16, y, yt, ws, stream);
    case 4: return launch_lut_small<4>(L, p, x, x_fp16, y, yt, ws, stream);
    default: return launch_lut_small<8>(L, p, x, x_fp16, y, yt, ws, stream);
  }
}

}  // namespace vqk

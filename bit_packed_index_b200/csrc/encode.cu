// encode.cu -- the nearest-centroid encoder (vq_encode in include/vq.h):
// idx[o][j] = argmin_k ||v - C[k]||^2 for every vector of a weight matrix,
// ties to the lowest k, equal to the exact (fp64) definition; with two books
// the second stage encodes the residual of the first (greedy cascade).
// Follows "VPTQ Guide: Extreme 2-Bit Vector Quantization", section "The
// Information-Theoretic Superiority of Vector Quantization" (q = argmin) and
// section "2. Multi-Stage Residual Vector Quantization (RVQ)".
//
// Design:
//  * ||v - c||^2 = ||v||^2 + (||c||^2 - 2<v, c>), and only the bracket depends
//    on c.  The bracket is one dot product of length d + 2 <= 16: A row =
//    [v~, 1, 1, 0...], B row = [-2 c~, hi, lo, 0...] with hi + lo = ||c~||^2
//    split into two fp16 values, so a single tcgen05 MMA (M = 128 vectors,
//    N = 256 centroids, K = 16, fp16 x fp16 -> fp32 in tensor memory) gives the
//    whole bracket for 32768 pairs.  v~ and c~ are v and c times one power of
//    two per book, chosen so that max ||c~||^2 lies in [2^8, 2^10): the
//    argmin does not change and every operand stays well inside fp16.
//  * The prepared book ([-2c~, hi, lo] rows, 32 bytes per centroid) is laid
//    out in global memory exactly as the 128-byte-swizzled K-major operand the
//    MMA reads -- four centroids of different 256-row groups share a 128-byte
//    row -- so 1024 centroids arrive with one 32 KB bulk copy and the four
//    MMAs of that block address it with a 32-byte column offset.
//  * Sixteen epilogue warps read the accumulators (two TMEM buffers of 256
//    columns, so the MMA of the next tile overlaps) and keep, per vector and
//    column quarter, the smallest value, its column and the second smallest:
//    a 32-column chunk costs 31 min operations and one compare, and only a
//    chunk that holds a new minimum is scanned again.
//  * A vector whose second smallest value exceeds the smallest by more than
//    twice a bound on the arithmetic error (fp32 accumulation, the hi/lo
//    split, fp16 rounding of a residual) has the exact argmin in hand.  Every
//    other vector -- near-ties, partial last vectors, values fp16 cannot hold
//    -- is decided by an fp64 pass over the whole book that repeats the
//    definition operation by operation, so the output equals the definition.
//  * Hessian-weighted form ("VPTQ Guide", section "1. Second-Order
//    Hessian-Weighted Optimization": D_H(v, c) = (v - c)^T H_v (v - c), H_v
//    the sub-matrix of H on the vector's channels).  D_H = v^T H v + (c^T H_v
//    c - 2 c^T H_s v) with H_s = (H_v + H_v^T) / 2, and again only the bracket
//    depends on c.  A block holds 128 rows of one block of channels j, so all
//    its vectors share H_j: the A row is z = H_s v (scaled, split into fp16 hi
//    and lo halves), the B row [-2 c~, -2 c~] (the same for every j), and the
//    epilogue adds nc[j][k] = c~^T H_j c~ (a table of fp32 values per block
//    of channels, made once per call) with one fma per value.  The exact
//    paths evaluate (v - c)^T H_v (v - c) as the definition does.
//  * Every mbarrier wait is bounded; a wait that runs out of budget raises
//    the block's abort flag, records VQ_ERR_TIMEOUT in the workspace's status
//    word and lets every warp fall through to the teardown.
#include <climits>
#include <cmath>

#include "sm100.cuh"
#include "vq_internal.cuh"

namespace vqk {
namespace {

using namespace sm100;

constexpr int kEncM = 128;                          // vectors per block (MMA M)
constexpr int kEncN = 256;                          // centroids per MMA (N)
constexpr int kEncBlockK = 1024;                    // centroids per staged block: 4 MMAs
constexpr int kEncBlockBytes = kEncBlockK / 4 * 128;   // 256 rows x 128 B = 32 KB
constexpr int kEncStages = 3;
constexpr int kEncEpiWarps = 16;                    // 4 lane quarters x 4 column quarters
constexpr int kEncThreads = (4 + kEncEpiWarps) * 32;
constexpr int kEncATile = kEncM * 128;              // 16 KB: rows of 128 B, first 32 B used
constexpr long long kEncWaitBudget = 4000000000LL;  // SM clocks (about 2 s)
constexpr float kEncPadNorm = 30000.0f;             // hi = lo of padding centroids
constexpr int kEncMaxD = 14;                        // d + 2 <= 16
constexpr int kEncHMaxD = 8;                        // Hessian-weighted form: 2 d <= 16
constexpr int kEncExactThreads = 256;

struct EncCtrl {
  uint64_t full[kEncStages];
  uint64_t empty[kEncStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort_flag;
  float eps[kEncM];              // error bound of each vector's bracket values
  int flag[kEncM];               // 0: decide here, 1: exact pass, 2: no vector
  float best[4][kEncM];          // per column quarter: smallest bracket value,
  float second[4][kEncM];        //   smallest chunk minimum of the other chunks,
  int chunk[4][kEncM];           //   first centroid of the chunk holding the smallest
  double v[kEncM][kEncMaxD];     // the vectors, exactly (fp64)
  double vnorm[kEncM];           // ||v||^2 (fp64); v^T H v in the weighted form
  // Hessian-weighted form only:
  float zsc[kEncM];              // 2^u: the vector's scale of z = H_s v~
  double slack[kEncM];           // size of the fp64 rounding in its exact distances
  double hj[kEncHMaxD][kEncHMaxD];   // H on this block's channels (fp64)
  float ncw[kEncEpiWarps][64];   // each epilogue warp's nc values of the current tile
};

// Workspace control words (first 256 bytes).
struct EncWsCtrl {
  int status;
  int list_count[2];             // vectors left to the exact pass, per stage
  unsigned cmax_bits[2];         // max_k ||C_m[k]||^2 (fp32 bits; non-negative)
};

__device__ __forceinline__ uint8_t* enc_align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled operand.
__device__ __forceinline__ uint32_t enc_sw128(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

// Power-of-two exponent s with cmax * 4^s in [2^8, 2^10) (s = 0 for a zero or
// non-finite cmax; a subnormal cmax is treated as 2^-127).
__device__ __forceinline__ int enc_scale_exp(float cmax) {
  if (!(cmax > 0.0f) || !(cmax < INFINITY)) return 0;
  const int e = static_cast<int>((__float_as_uint(cmax) >> 23) & 0xffu) - 127;
  return (9 - e) >> 1;                               // floor((9 - e) / 2)
}
__device__ __forceinline__ float enc_pow2(int s) {  // 2^s, s in [-126, 127]
  return __uint_as_float(static_cast<uint32_t>(127 + s) << 23);
}

// Plain bulk copy global -> shared (no multicast), completing on bar.
__device__ __forceinline__ void enc_bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// Book preparation.
// ---------------------------------------------------------------------------
__global__ void enc_book_norm_kernel(const uint16_t* __restrict__ book, int K, int d,
                                     unsigned* __restrict__ cmax_bits) {
  float m = 0.0f;
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < K; k += gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int e = 0; e < d; ++e) {
      const float c = h2f(book[static_cast<int64_t>(k) * d + e]);
      s = fmaf(c, c, s);
    }
    m = fmaxf(m, s);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) atomicMax(cmax_bits, __float_as_uint(m));   // m >= 0: bits order as values
}

// Prepared book: centroid k = 1024 q + 256 sl + r sits in block q (32 KB),
// row r, 16-half column slot sl, 128-byte swizzled; halves [-2 c~ (d), hi,
// lo, 0...], c~ = fp16(c * 2^s), hi + lo = ||c~||^2.  Centroids k >= K (the
// padding up to a whole block) get hi = lo = kEncPadNorm and zero c~.  The
// Hessian-weighted form (hw) stores [-2 c~ (d), -2 c~ (d), 0...] instead (the
// two copies multiply the two fp16 halves of z) and zero for the padding,
// whose c^T H c term is infinite.
__global__ void enc_book_prep_kernel(const uint16_t* __restrict__ book, int K, int d, int kp,
                                     const unsigned* __restrict__ cmax_bits, uint8_t* __restrict__ bprep,
                                     int hw) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= kp) return;
  const float f = enc_pow2(enc_scale_exp(__uint_as_float(*cmax_bits)));
  uint16_t h[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) h[i] = 0;
  if (hw) {
    if (k < K)
      for (int e = 0; e < d; ++e) {
        const float c = h2f(f2h(h2f(book[static_cast<int64_t>(k) * d + e]) * f));
        h[e] = h[d + e] = f2h(-2.0f * c);
      }
  } else if (k < K) {
    float nrm = 0.0f;
    for (int e = 0; e < d; ++e) {
      const float c = h2f(f2h(h2f(book[static_cast<int64_t>(k) * d + e]) * f));
      h[e] = f2h(-2.0f * c);
      nrm = __fadd_rn(nrm, __fmul_rn(c, c));
    }
    const uint16_t hi = f2h(nrm);
    h[d] = hi;
    h[d + 1] = f2h(nrm - h2f(hi));
  } else {
    h[d] = f2h(kEncPadNorm);
    h[d + 1] = f2h(kEncPadNorm);
  }
  const int q = k / kEncBlockK, rem = k % kEncBlockK, sl = rem / kEncN, r = rem % kEncN;
  uint8_t* base = bprep + static_cast<size_t>(q) * kEncBlockBytes;
  uint4 c0, c1;
  c0.x = h[0] | (static_cast<uint32_t>(h[1]) << 16);
  c0.y = h[2] | (static_cast<uint32_t>(h[3]) << 16);
  c0.z = h[4] | (static_cast<uint32_t>(h[5]) << 16);
  c0.w = h[6] | (static_cast<uint32_t>(h[7]) << 16);
  c1.x = h[8] | (static_cast<uint32_t>(h[9]) << 16);
  c1.y = h[10] | (static_cast<uint32_t>(h[11]) << 16);
  c1.z = h[12] | (static_cast<uint32_t>(h[13]) << 16);
  c1.w = h[14] | (static_cast<uint32_t>(h[15]) << 16);
  *reinterpret_cast<uint4*>(base + enc_sw128(r, 2 * sl)) = c0;
  *reinterpret_cast<uint4*>(base + enc_sw128(r, 2 * sl + 1)) = c1;
}

// Hessian-weighted form: nc[j][k] = c~_k^T H_j c~_k in fp32 for every block j
// of d channels (j < nfull) and centroid k < kp, with c~ = fp16(c 2^s) as in
// the prepared book and H_j the d x d block of h on channels j d .. j d + d - 1;
// +infinity for the padding k >= K.  Also ncabs[j] = max_k |c~_k|^T |H_j|
// |c~_k| (as fp32 bits; zero on entry), the scale of nc's rounding error.
// Grid (kp / 256, nfull).
__global__ void enc_nc_kernel(const uint16_t* __restrict__ book, int K, int d, int kp,
                              const unsigned* __restrict__ cmax_bits, const float* __restrict__ h,
                              int64_t ldh, float* __restrict__ nc, unsigned* __restrict__ ncabs) {
  __shared__ float hs[kEncHMaxD * kEncHMaxD];
  __shared__ float red[8];
  const int j = blockIdx.y;
  if (threadIdx.x < d * d) {
    const int e = threadIdx.x / d, g = threadIdx.x % d;
    hs[threadIdx.x] = h[static_cast<int64_t>(j * d + e) * ldh + j * d + g];
  }
  __syncthreads();
  const int k = blockIdx.x * blockDim.x + threadIdx.x;   // kp is a multiple of 256: always < kp
  float v = INFINITY, va = 0.0f;
  if (k < K) {
    const float f = enc_pow2(enc_scale_exp(__uint_as_float(*cmax_bits)));
    float c[kEncHMaxD];
#pragma unroll
    for (int e = 0; e < kEncHMaxD; ++e)
      c[e] = e < d ? h2f(f2h(h2f(book[static_cast<int64_t>(k) * d + e]) * f)) : 0.0f;
    v = 0.0f;
#pragma unroll
    for (int e = 0; e < kEncHMaxD; ++e) {
      if (e < d) {
        float g = 0.0f, ga = 0.0f;
#pragma unroll
        for (int q = 0; q < kEncHMaxD; ++q)
          if (q < d) {
            g = fmaf(hs[e * d + q], c[q], g);
            ga = fmaf(fabsf(hs[e * d + q]), fabsf(c[q]), ga);
          }
        v = fmaf(c[e], g, v);
        va = fmaf(fabsf(c[e]), ga, va);
      }
    }
  }
  nc[static_cast<int64_t>(j) * kp + k] = v;
  // the block's largest |c|^T |H| |c| (non-negative, so the bits order as the values)
  va *= 1.0f + 0x1p-20f;                               // covers the rounding of va itself
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) va = fmaxf(va, __shfl_xor_sync(0xffffffffu, va, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = va;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.0f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
    atomicMax(ncabs + j, __float_as_uint(m));
  }
}

// The book in fp64 (exact), for the exact distances.
__global__ void enc_book64_kernel(const uint16_t* __restrict__ book, int64_t count, double* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < count) out[i] = static_cast<double>(h2f(book[i]));
}

// ---------------------------------------------------------------------------
// The tensor-core pass.
// ---------------------------------------------------------------------------
struct EncArgs {
  const uint16_t* w;
  int64_t ldw;
  int n, kin, d, nfull, nvec;    // nfull = kin / d whole vectors per row
  int64_t nv_full;               // n * nfull
  const uint8_t* bprep;
  int kp, K;                     // padded and real book size
  const unsigned* cmax_bits;
  const double* book64;          // the book in fp64 [K][d]
  const uint16_t* book1;         // second stage: v = w - C_1[idx1] (else null)
  const uint32_t* idx1;
  uint32_t* idx_out;             // [n][nvec]
  int* list;                     // vector ids o * nvec + j left to the exact pass
  int* list_count;
  int* status;
  // Hessian-weighted form: a block's 128 vectors are rows o0 .. o0+127 of one
  // block of channels j (mt blocks per j), nc = c~^T H_j c~ [nfull][kp].
  const float* h;
  int64_t ldh;
  const float* nc;
  const unsigned* ncabs;         // max_k |c~_k|^T |H_j| |c~_k| per block j (fp32 bits)
  int mt;
};

// sum_e (v_e - c_e)^2 with each difference, square and sum rounded once in
// fp64, e ascending: the distance of the definition.
__device__ __forceinline__ double enc_dist64(const double* v, const double* c, int d) {
  double dist = 0.0;
  for (int e = 0; e < d; ++e) {
    const double t = __dsub_rn(v[e], c[e]);
    dist = __dadd_rn(dist, __dmul_rn(t, t));
  }
  return dist;
}

// (v - c)^T H (v - c) with t_e = v_e - c_e, g_e = sum_f H[e][f] t_f (f
// ascending), the sum over e ascending, every operation rounded once in
// fp64: the weighted distance of the definition.
__device__ __forceinline__ double enc_dist64h(const double* v, const double* c,
                                              const double (*hj)[kEncHMaxD], int d) {
  double t[kEncHMaxD];
#pragma unroll
  for (int e = 0; e < kEncHMaxD; ++e) t[e] = e < d ? __dsub_rn(v[e], c[e]) : 0.0;
  double dist = 0.0;
#pragma unroll
  for (int e = 0; e < kEncHMaxD; ++e) {
    if (e < d) {
      double g = 0.0;
#pragma unroll
      for (int f = 0; f < kEncHMaxD; ++f)
        if (f < d) g = __dadd_rn(g, __dmul_rn(hj[e][f], t[f]));
      dist = __dadd_rn(dist, __dmul_rn(t[e], g));
    }
  }
  return dist;
}

// One 32-column chunk of bracket values for centroids k0 .. k0+31: the
// running smallest value, the first centroid of the chunk that holds it, and
// the smallest chunk minimum among all other chunks.  Which column of the
// best chunk holds the minimum is settled later, exactly.
__device__ __forceinline__ float enc_min3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ void enc_chunk(const uint32_t (&r)[32], int k0, float& best, float& second,
                                          int& chunk) {
  float m[12];
#pragma unroll
  for (int i = 0; i < 10; ++i)
    m[i] = enc_min3(__uint_as_float(r[3 * i]), __uint_as_float(r[3 * i + 1]), __uint_as_float(r[3 * i + 2]));
  m[10] = __uint_as_float(r[30]);
  m[11] = __uint_as_float(r[31]);
  const float mn = fminf(enc_min3(enc_min3(m[0], m[1], m[2]), enc_min3(m[3], m[4], m[5]), enc_min3(m[6], m[7], m[8])),
                         enc_min3(m[9], m[10], m[11]));
  const bool p = mn < best;
  second = p ? best : fminf(second, mn);
  best = p ? mn : best;
  chunk = p ? k0 : chunk;
}

// HW: the Hessian-weighted form (see EncArgs).  The plain form's blocks take
// 128 consecutive vectors in (row, vector) order.
template <bool HW>
__global__ void __launch_bounds__(kEncThreads, 1) enc_tc_kernel(EncArgs a) {
  extern __shared__ __align__(1024) uint8_t enc_smem[];
  EncCtrl* ctrl = reinterpret_cast<EncCtrl*>(enc_smem);
  uint8_t* atile = enc_align1024(enc_smem + sizeof(EncCtrl));
  uint8_t* stages = atile + kEncATile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &ctrl->abort_flag;
  const int64_t v0 = HW ? 0 : static_cast<int64_t>(blockIdx.x) * kEncM;
  const int hblk = HW ? static_cast<int>(blockIdx.x / a.mt) : 0;          // block of channels
  const int obase = HW ? static_cast<int>(blockIdx.x % a.mt) * kEncM : 0;  // its first row

  if (threadIdx.x == 0) {
    for (int s = 0; s < kEncStages; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctrl->acc_full[b], 1);
      mbar_init(&ctrl->acc_empty[b], kEncEpiWarps);
    }
    ctrl->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctrl->tmem_base, 512);
    tmem_relinquish();
  }
  if (HW) {                                            // H on this block's channels, in fp64
    if (threadIdx.x < kEncHMaxD * kEncHMaxD) {
      const int e = threadIdx.x / kEncHMaxD, g = threadIdx.x % kEncHMaxD;
      ctrl->hj[e][g] = (e < a.d && g < a.d)
                           ? static_cast<double>(a.h[static_cast<int64_t>(hblk * a.d + e) * a.ldh + hblk * a.d + g])
                           : 0.0;
    }
    __syncthreads();
  }

  // A operand: row t = [v~ (d halves), 1, 1, 0...] of vector v0 + t, and the
  // vector's error bound.  With s the book's exponent and v~ = fp16(v 2^s),
  // the MMA returns D(k) = sum_e v~_e (-2 c~_ke) + hi_k + lo_k, and
  //   |D(k) - (||c_k||^2 - 2<v, c_k>) 4^s|
  //     <= 2^-18 (||v~||^2 + 2 C + 1)      fp32 accumulation, hi/lo split
  //      + 2^-22 ||v~||_1 (1 + sqrt C)     fp16 rounding of tiny c~ components
  //      + 2 delta (sqrt C + 1)            v~ against v 2^s (delta: its L1 error)
  // with C = max_k ||c~_k||^2 < 2^10; the terms are loose by design.
  //
  // Weighted form: row t = [z~ hi (d halves), z~ lo (d halves), 0...] with
  // z = H_s v 2^s (fp32), z~ = z 2^u (u puts max |z~| in [2^13, 2^14)) split
  // into two fp16 halves; the MMA returns -2<z~, c~> and the epilogue adds
  // nc_k 2^u, so D(k) approximates (c~^T H c~ - 2 c~^T H_s v~) 2^u =
  // (D_H(v, c) - v^T H v) 4^s 2^u.  The bound (eps) sums, each with a factor
  // of four to spare: fp32 rounding of nc (d + 2 roundings of terms up to
  // Hmax d C), of z (d + 2 roundings of |H_s| |v~|), of the MMA's sums and
  // the epilogue's fma, the fp16 hi/lo split of z~ (2^-22 relative, 2^-25
  // absolute) and the fp16 rounding of tiny c~ components (2^-25 absolute).
  if (threadIdx.x < kEncM) {
    const int t = threadIdx.x;
    const float cmax = __uint_as_float(*a.cmax_bits);
    const int se = enc_scale_exp(cmax);
    const float f = enc_pow2(se);
    uint16_t h[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) h[i] = 0;
    float eps = 0.0f;
    int flag = 2;
    if (HW) {
      const int o = obase + t, j = hblk;
      if (o < a.n) {
        flag = 0;
        const uint16_t* wr = a.w + static_cast<int64_t>(o) * a.ldw + static_cast<int64_t>(j) * a.d;
        const uint16_t* c1 = a.book1 ? a.book1 + static_cast<int64_t>(a.idx1[static_cast<int64_t>(o) * a.nvec + j]) * a.d
                                     : nullptr;
        double vd[kEncHMaxD];
        float vs[kEncHMaxD];
#pragma unroll
        for (int e = 0; e < kEncHMaxD; ++e) {
          vd[e] = 0.0;
          vs[e] = 0.0f;
          if (e < a.d) {
            double ve = static_cast<double>(h2f(wr[e]));
            if (c1) ve = __dsub_rn(ve, static_cast<double>(h2f(c1[e])));
            vd[e] = ve;
            ctrl->v[t][e] = ve;
            float v = h2f(wr[e]);
            if (c1) v = __fsub_rn(v, h2f(c1[e]));
            vs[e] = v * f;                             // a power-of-two scale
          }
        }
        // v^T H v in fp64 (the definition's order), |v|^T |H| |v|, ||v||^2, max |H|
        double vhv = 0.0, vha = 0.0, vn = 0.0;
        float hmax = 0.0f;
#pragma unroll
        for (int e = 0; e < kEncHMaxD; ++e) {
          if (e < a.d) {
            double g = 0.0, ga = 0.0;
#pragma unroll
            for (int q = 0; q < kEncHMaxD; ++q) {
              if (q < a.d) {
                const double hv = ctrl->hj[e][q];
                g = __dadd_rn(g, __dmul_rn(hv, vd[q]));
                ga += fabs(hv) * fabs(vd[q]);
                hmax = fmaxf(hmax, fabsf(static_cast<float>(hv)));
              }
            }
            vhv = __dadd_rn(vhv, __dmul_rn(vd[e], g));
            vha += fabs(vd[e]) * ga;
            vn += vd[e] * vd[e];
          }
        }
        // z = H_s v~ in fp32, and the 2-norm of the terms' magnitudes (|H_s| |v~|)
        float z[kEncHMaxD], hv2 = 0.0f, zmax = 0.0f;
#pragma unroll
        for (int e = 0; e < kEncHMaxD; ++e) {
          z[e] = 0.0f;
          if (e < a.d) {
            float ha = 0.0f;
#pragma unroll
            for (int q = 0; q < kEncHMaxD; ++q) {
              if (q < a.d) {
                const float hs = 0.5f * (static_cast<float>(ctrl->hj[e][q]) + static_cast<float>(ctrl->hj[q][e]));
                z[e] = fmaf(hs, vs[q], z[e]);
                ha += fabsf(hs) * fabsf(vs[q]);
              }
            }
            hv2 += ha * ha;
            zmax = fmaxf(zmax, fabsf(z[e]));
          }
        }
        hv2 = sqrtf(hv2) * 1.001f;
        float zs = 1.0f;
        if (zmax > 0.0f && zmax < INFINITY) {
          const int ez = static_cast<int>((__float_as_uint(zmax) >> 23) & 0xffu) - 127;
          zs = enc_pow2(max(-126, min(127, 13 - ez)));
        }
        float z2 = 0.0f, zmx = 0.0f;
#pragma unroll
        for (int e = 0; e < kEncHMaxD; ++e) {
          if (e < a.d) {
            const float zt = z[e] * zs;
            const uint16_t hi = f2h(zt);
            const uint16_t lo = f2h(zt - h2f(hi));
            h[e] = hi;
            h[a.d + e] = lo;
            z2 += zt * zt;
            zmx = fmaxf(zmx, fabsf(zt));
          }
        }
        z2 = sqrtf(z2) * 1.001f;
        const float dd = static_cast<float>(a.d);
        const float cs = cmax * f * f;
        const float rc = sqrtf(cs) * 1.001f;           // >= |c~_k| for every k
        const float na = __uint_as_float(a.ncabs[j]) * zs;   // >= |c~|^T |H_j| |c~| 2^u
        const float hm = hmax * zs, hv = hv2 * zs;
        // nc's fp32 sums (2 d roundings), the epilogue's fma, the MMA's fp32
        // sums of 2 d products (|sum| <= 2 rc ||z~||), z's own rounding and
        // fp16 split, and the fp16 rounding of tiny c~ components
        eps = 2.0f * ((2.0f * dd + 2.0f) * 0x1p-24f * na + 0x1p-24f * (na + 2.0f * rc * z2) +
                      (2.0f * dd + 1.0f) * 0x1p-24f * 2.0f * rc * z2 +
                      2.0f * rc * ((dd + 2.0f) * 0x1p-24f * hv + 0x1p-22f * z2 + 3.0f * 0x1p-25f) +
                      0x1p-23f * dd * (hm * dd * rc + zmx));
        if (!(eps < INFINITY) || !(fabs(vhv) < INFINITY) || !(zmx < 16384.0f)) flag = 1;
        ctrl->vnorm[t] = vhv;
        ctrl->zsc[t] = zs;
        // fp64 rounding of the exact distances and of v^T H v, before scaling
        ctrl->slack[t] = 0x1p-36 * (vha + 2.0 * static_cast<double>(hmax) * a.d * (vn + static_cast<double>(cmax)));
      }
    } else {
      const int64_t gv = v0 + t;
      if (gv < a.nv_full) {
        flag = 0;
        const int o = static_cast<int>(gv / a.nfull), j = static_cast<int>(gv % a.nfull);
        const uint16_t* wr = a.w + static_cast<int64_t>(o) * a.ldw + static_cast<int64_t>(j) * a.d;
        const uint16_t* c1 = a.book1 ? a.book1 + static_cast<int64_t>(a.idx1[static_cast<int64_t>(o) * a.nvec + j]) * a.d
                                     : nullptr;
        float n2 = 0.0f, l1 = 0.0f, dl = 0.0f;
        double vn = 0.0;
        for (int e = 0; e < a.d; ++e) {
          double ve = static_cast<double>(h2f(wr[e]));
          if (c1) ve = __dsub_rn(ve, static_cast<double>(h2f(c1[e])));
          ctrl->v[t][e] = ve;
          vn = __dadd_rn(vn, __dmul_rn(ve, ve));
          float v = h2f(wr[e]);
          if (c1) v = __fsub_rn(v, h2f(c1[e]));
          const float vs = v * f;                      // exact: a power-of-two scale in range
          const uint16_t hv = f2h(vs);
          const float vt = h2f(hv);
          if (!(fabsf(vt) <= 65504.0f)) flag = 1;      // overflow or NaN: exact pass
          h[e] = hv;
          n2 = fmaf(vt, vt, n2);
          l1 += fabsf(vt);
          dl += fabsf(vt - vs) + fabsf(vs) * 0x1p-22f + 0x1p-24f;
        }
        ctrl->vnorm[t] = vn;
        h[a.d] = 0x3C00u;                              // 1.0 (times hi)
        h[a.d + 1] = 0x3C00u;                          // 1.0 (times lo)
        const float cs = cmax * f * f;
        const float rc = sqrtf(cs);
        eps = 0x1p-18f * (n2 + 2.0f * cs + 1.0f) + 0x1p-22f * l1 * (1.0f + rc) + 2.0f * dl * (rc + 1.0f);
        if (!(eps < INFINITY)) flag = 1;
      }
    }
    ctrl->eps[t] = eps;
    ctrl->flag[t] = flag;
    uint4 c0, c1v;
    c0.x = h[0] | (static_cast<uint32_t>(h[1]) << 16);
    c0.y = h[2] | (static_cast<uint32_t>(h[3]) << 16);
    c0.z = h[4] | (static_cast<uint32_t>(h[5]) << 16);
    c0.w = h[6] | (static_cast<uint32_t>(h[7]) << 16);
    c1v.x = h[8] | (static_cast<uint32_t>(h[9]) << 16);
    c1v.y = h[10] | (static_cast<uint32_t>(h[11]) << 16);
    c1v.z = h[12] | (static_cast<uint32_t>(h[13]) << 16);
    c1v.w = h[14] | (static_cast<uint32_t>(h[15]) << 16);
    *reinterpret_cast<uint4*>(atile + enc_sw128(t, 0)) = c0;
    *reinterpret_cast<uint4*>(atile + enc_sw128(t, 1)) = c1v;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  const int nq = a.kp / kEncBlockK;
  const int ntiles = nq * 4;

  if (warp == 0) {
    if (lane == 0) {                                   // staged-book loader
      int issued = 0;
      for (int q = 0; q < nq; ++q) {
        const int s = q % kEncStages;
        const uint32_t ph = (q / kEncStages) & 1;
        if (!bounded_wait(&ctrl->empty[s], ph ^ 1, abort_flag, a.status, kEncWaitBudget)) break;
        mbar_arrive_expect_tx(&ctrl->full[s], kEncBlockBytes);
        enc_bulk_load(stages + s * kEncBlockBytes, a.bprep + static_cast<size_t>(q) * kEncBlockBytes,
                      kEncBlockBytes, &ctrl->full[s]);
        issued = q + 1;
      }
      if (*abort_flag) {   // let copies already in flight land before the block exits
        for (int q = max(0, issued - kEncStages); q < issued; ++q)
          drain_phase(&ctrl->full[q % kEncStages], (q / kEncStages) & 1, kEncWaitBudget / 8);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {                                   // MMA issuer
      const uint32_t idesc = f16_idesc(kEncM, kEncN);
      const uint64_t adesc = sw128_kmajor_desc(smem_addr(atile));
      for (int t = 0; t < ntiles; ++t) {
        const int q = t >> 2, sl = t & 3, s = q % kEncStages;
        if (sl == 0 && !bounded_wait(&ctrl->full[s], (q / kEncStages) & 1, abort_flag, a.status, kEncWaitBudget))
          break;
        const int ab = t & 1;
        if (!bounded_wait(&ctrl->acc_empty[ab], ((t >> 1) & 1) ^ 1, abort_flag, a.status, kEncWaitBudget)) break;
        tc_fence_after();
        const uint32_t b = smem_addr(stages + s * kEncBlockBytes) + sl * 32;
        umma_f16(tmem + ab * kEncN, adesc, sw128_kmajor_desc(b), idesc, 0);
        umma_commit(&ctrl->acc_full[ab]);
        if (sl == 3) umma_commit(&ctrl->empty[s]);
      }
    }
  } else if (warp >= 4) {                              // epilogue
    const int lq = warp & 3, cq = (warp - 4) >> 2;
    const int row = lq * 32 + lane;
    float best = INFINITY, second = INFINITY;
    int chunk = 0;
    // Weighted form: this warp's 64 values of nc for the next tile, fetched a
    // tile ahead (two per lane) and passed through its own shared-memory row.
    const float* ncr = HW ? a.nc + static_cast<int64_t>(hblk) * a.kp : nullptr;
    float p0 = 0.0f, p1 = 0.0f, zs = 1.0f;
    if (HW) {
      p0 = ncr[cq * 64 + lane];
      p1 = ncr[cq * 64 + 32 + lane];
      zs = ctrl->zsc[row];
    }
    for (int t = 0; t < ntiles; ++t) {
      const int ab = t & 1;
      if (!bounded_wait(&ctrl->acc_full[ab], (t >> 1) & 1, abort_flag, a.status, kEncWaitBudget)) break;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      const uint32_t ta = tmem + (static_cast<uint32_t>(lq * 32) << 16) + ab * kEncN + cq * 64;
      tmem_ld32(ta, r0);
      tmem_ld32(ta + 32, r1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->acc_empty[ab]);
      const int k0 = (t >> 2) * kEncBlockK + (t & 3) * kEncN + cq * 64;
      if (HW) {
        float* ns = ctrl->ncw[warp - 4];
        ns[lane] = p0;
        ns[32 + lane] = p1;
        __syncwarp();
        if (t + 1 < ntiles) {
          const int k1 = ((t + 1) >> 2) * kEncBlockK + ((t + 1) & 3) * kEncN + cq * 64;
          p0 = ncr[k1 + lane];
          p1 = ncr[k1 + 32 + lane];
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          r0[i] = __float_as_uint(fmaf(ns[i], zs, __uint_as_float(r0[i])));
          r1[i] = __float_as_uint(fmaf(ns[32 + i], zs, __uint_as_float(r1[i])));
        }
        __syncwarp();
      }
      enc_chunk(r0, k0, best, second, chunk);
      enc_chunk(r1, k0 + 32, best, second, chunk);
    }
    ctrl->best[cq][row] = best;
    ctrl->second[cq][row] = second;
    ctrl->chunk[cq][row] = chunk;
  }
  tc_fence_before();
  __syncthreads();

  // Merge the four column quarters: the best chunk overall and the smallest
  // value outside it (quarter order breaks ties; a tie leaves no margin).
  const bool live = !*abort_flag;
  if (threadIdx.x < kEncM && live && ctrl->flag[threadIdx.x] == 0) {
    const int t = threadIdx.x;
    float b = ctrl->best[0][t], s2 = ctrl->second[0][t];
    int c0 = ctrl->chunk[0][t];
#pragma unroll
    for (int q = 1; q < 4; ++q) {
      const float bq = ctrl->best[q][t];
      if (bq < b) {
        s2 = fminf(fminf(s2, b), ctrl->second[q][t]);
        b = bq;
        c0 = ctrl->chunk[q][t];
      } else {
        s2 = fminf(fminf(s2, bq), ctrl->second[q][t]);
      }
    }
    ctrl->second[0][t] = s2;
    ctrl->chunk[0][t] = c0;
  }
  __syncthreads();
  // The 32 centroids of each vector's best chunk, exactly (fp64, the
  // definition's operation order); the staged-book buffers hold the results.
  double* ex = reinterpret_cast<double*>(stages);       // [kEncM][32]
  if (live) {
    for (int p = threadIdx.x; p < kEncM * 32; p += kEncThreads) {
      const int t = p >> 5, c = p & 31;
      double e = INFINITY;
      if (ctrl->flag[t] == 0) {
        const int k = ctrl->chunk[0][t] + c;
        if (k < a.K)
          e = HW ? enc_dist64h(ctrl->v[t], a.book64 + static_cast<int64_t>(k) * a.d, ctrl->hj, a.d)
                 : enc_dist64(ctrl->v[t], a.book64 + static_cast<int64_t>(k) * a.d, a.d);
      }
      ex[p] = e;
    }
  }
  __syncthreads();
  // Decide: if every centroid outside the chunk is provably farther than the
  // chunk's exact minimum, that minimum (lowest k on ties) is the answer.
  //   outside:  D(k) >= second  =>  exact bracket >= second - eps
  //   inside:   exact bracket of the best = (dist - ||v||^2) 4^s
  //             (weighted: (dist - v^T H v) 4^s 2^u)
  if (threadIdx.x < kEncM && live) {
    const int t = threadIdx.x;
    const int flag = ctrl->flag[t];
    if (flag != 2) {
      int o, j;
      if (HW) {
        o = obase + t;
        j = hblk;
      } else {
        const int64_t gv = v0 + t;
        o = static_cast<int>(gv / a.nfull);
        j = static_cast<int>(gv % a.nfull);
      }
      const int64_t vid = static_cast<int64_t>(o) * a.nvec + j;
      bool done = false;
      if (flag == 0) {
        double emin = INFINITY;
        int kmin = -1;
        for (int c = 0; c < 32; ++c) {
          const double e = ex[t * 32 + c];
          if (e < emin) {
            emin = e;
            kmin = ctrl->chunk[0][t] + c;
          }
        }
        if (kmin >= 0) {
          const int se2 = 2 * enc_scale_exp(__uint_as_float(*a.cmax_bits));   // 4^s as a double
          double sc = __longlong_as_double(static_cast<long long>(1023 + se2) << 52);
          if (HW) sc *= static_cast<double>(ctrl->zsc[t]);
          const double dex = (emin - ctrl->vnorm[t]) * sc;
          double slack = 0x1p-40 * (fabs(emin) + fabs(ctrl->vnorm[t])) * sc;
          if (HW) slack += ctrl->slack[t] * sc;
          if (static_cast<double>(ctrl->second[0][t]) - dex > static_cast<double>(ctrl->eps[t]) + slack) {
            a.idx_out[vid] = static_cast<uint32_t>(kmin);
            done = true;
          }
        }
      }
      if (!done) {
        const int pos = atomicAdd(a.list_count, 1);
        a.list[pos] = static_cast<int>(vid);
      }
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// The exact pass: the definition, operation by operation, in fp64.
// ---------------------------------------------------------------------------
struct EncExactArgs {
  const uint16_t* w;
  int64_t ldw;
  int n, kin, d, nvec;
  const double* book64;          // the book in fp64 [K][d]
  int K;
  const uint16_t* book1;         // second stage: v = w - C_1[idx1] in fp64 (else null)
  const uint32_t* idx1;
  uint32_t* idx_out;
  const int* list;
  const int* list_count;
  int partial_rows;              // n when the last vector of every row is partial, else 0
  const float* h;                // weighted form: the Hessian (else null)
  int64_t ldh;
};

// Work items: the listed vectors, then the partial last vector of every row.
// A block takes eight items, one per warp, and streams the book through
// shared memory in tiles of 512 fp64 centroids (stored component-major, so a
// warp's loads are consecutive) that all eight warps scan, the lanes of a
// warp striding over the tile.  dist(k) = sum_e (v_e - c_e)^2 with
// every difference, square and sum rounded once in fp64, e ascending; the
// smallest dist wins, ties to the lowest k; a NaN distance never wins and a
// vector with no finite distance gets index 0.
constexpr int kEncExactTile = 512;

// The weighted form (HW) takes (v - c)^T H_v (v - c) instead, H_v read once
// per vector into registers (fp64), in the order of enc_dist64h.
template <bool HW>
__global__ void __launch_bounds__(kEncExactThreads) enc_exact_kernel(EncExactArgs a) {
  constexpr int NW = kEncExactThreads / 32;
  extern __shared__ double tile[];                 // [d][kEncExactTile]
  const int nlist = *a.list_count;
  const int nitems = nlist + a.partial_rows;
  const int ngroups = (nitems + NW - 1) / NW;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int grp = blockIdx.x; grp < ngroups; grp += gridDim.x) {
    const int item = grp * NW + warp;
    const bool has = item < nitems;
    int o = 0, j = 0;
    if (has) {
      if (item < nlist) {
        const int vid = a.list[item];
        o = vid / a.nvec;
        j = vid % a.nvec;
      } else {
        o = item - nlist;
        j = a.nvec - 1;
      }
    }
    const int dv = has ? min(a.d, a.kin - j * a.d) : 0;
    const int64_t vid = static_cast<int64_t>(o) * a.nvec + j;
    double v[kEncMaxD];
#pragma unroll
    for (int e = 0; e < kEncMaxD; ++e) {
      v[e] = 0.0;
      if (e < dv) {
        v[e] = static_cast<double>(h2f(a.w[static_cast<int64_t>(o) * a.ldw + static_cast<int64_t>(j) * a.d + e]));
        if (a.book1)
          v[e] = __dsub_rn(v[e], static_cast<double>(h2f(a.book1[static_cast<int64_t>(a.idx1[vid]) * a.d + e])));
      }
    }
    double hr[HW ? kEncHMaxD : 1][HW ? kEncHMaxD : 1];
    if (HW) {
#pragma unroll
      for (int e = 0; e < (HW ? kEncHMaxD : 1); ++e)
#pragma unroll
        for (int g = 0; g < (HW ? kEncHMaxD : 1); ++g)
          hr[e][g] = (e < dv && g < dv)
                         ? static_cast<double>(a.h[static_cast<int64_t>(j * a.d + e) * a.ldh + j * a.d + g])
                         : 0.0;
    }
    double best = INFINITY;
    int arg = INT_MAX;
    for (int k0 = 0; k0 < a.K; k0 += kEncExactTile) {
      const int nk = min(kEncExactTile, a.K - k0);
      __syncthreads();                             // the previous tile is consumed
      for (int i = threadIdx.x; i < nk * a.d; i += kEncExactThreads)   // transposed: tile[e][kk]
        tile[(i % a.d) * kEncExactTile + i / a.d] = a.book64[static_cast<int64_t>(k0) * a.d + i];
      __syncthreads();
      if (has) {
        for (int kk = lane; kk < nk; kk += 32) {
          double dist = 0.0;
          if (HW) {
            double t[kEncHMaxD];
#pragma unroll
            for (int e = 0; e < kEncHMaxD; ++e) t[e] = e < dv ? __dsub_rn(v[e], tile[e * kEncExactTile + kk]) : 0.0;
#pragma unroll
            for (int e = 0; e < (HW ? kEncHMaxD : 1); ++e) {
              if (e < dv) {
                double g = 0.0;
#pragma unroll
                for (int f = 0; f < (HW ? kEncHMaxD : 1); ++f)
                  if (f < dv) g = __dadd_rn(g, __dmul_rn(hr[e][f], t[f]));
                dist = __dadd_rn(dist, __dmul_rn(t[e], g));
              }
            }
          } else {
#pragma unroll
            for (int e = 0; e < kEncMaxD; ++e) {
              if (e < dv) {
                const double t = __dsub_rn(v[e], tile[e * kEncExactTile + kk]);
                dist = __dadd_rn(dist, __dmul_rn(t, t));
              }
            }
          }
          if (dist < best) {       // k ascends per lane: the first minimum
            best = dist;
            arg = k0 + kk;
          }
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, best, off);
      const int ok = __shfl_xor_sync(0xffffffffu, arg, off);
      if (ob < best || (ob == best && ok < arg)) {
        best = ob;
        arg = ok;
      }
    }
    if (has && lane == 0) a.idx_out[vid] = arg == INT_MAX ? 0u : static_cast<uint32_t>(arg);
  }
}

// Row o's stream word t: the fields j whose bits [j b, j b + b) overlap
// [32 t, 32 t + 32), LSB first; zero past the last field.
__global__ void enc_pack_kernel(const uint32_t* __restrict__ idx, int n, int nvec, int b,
                                uint32_t* __restrict__ out, int64_t rw) {
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= static_cast<int64_t>(n) * rw) return;
  const int64_t o = gid / rw, t = gid % rw;
  const int64_t bit0 = t * 32;
  const uint32_t mask = b >= 32 ? 0xffffffffu : ((1u << b) - 1u);
  uint32_t word = 0;
  for (int64_t j = bit0 / b; j < nvec && j * b < bit0 + 32; ++j) {
    const uint32_t f = idx[o * nvec + j] & mask;
    const int64_t p = j * b - bit0;
    word |= p >= 0 ? (f << p) : (f >> (-p));
  }
  out[o * rw + t] = word;
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
static_assert(sizeof(vq_encode_desc) == 104, "vq_encode_desc layout");

struct EncPlan {
  int n, kin, d, nb, nvec, nfull;
  int b[2], K[2], kp[2];
  int64_t nv_full;
  bool hw;                       // Hessian-weighted form
  int mt;                        // weighted form: blocks of 128 rows
  size_t off_bprep[2], off_book64[2], off_idx[2], off_nc[2], off_ncabs[2], off_list, total;
};

size_t enc_round256(size_t x) { return (x + 255) / 256 * 256; }

// Sizes and strides always; pointers only when `ptrs` (the size query takes
// a description whose buffers do not exist yet).
vq_status enc_check(const vq_encode_desc* e, EncPlan* p, bool ptrs) {
  if (!e) return VQ_ERR_INVALID_ARG;
  if (e->out_features < 0 || e->in_features < 0 || e->vec_dim < 1 || e->vec_dim > kEncMaxD ||
      e->n_books < 1 || e->n_books > 2)
    return VQ_ERR_INVALID_ARG;
  p->n = e->out_features;
  p->kin = e->in_features;
  p->d = e->vec_dim;
  p->nb = e->n_books;
  p->nvec = (p->kin + p->d - 1) / p->d;
  p->nfull = p->kin / p->d;
  p->nv_full = static_cast<int64_t>(p->n) * p->nfull;
  if (static_cast<int64_t>(p->n) * p->nvec >= (int64_t{1} << 31)) return VQ_ERR_UNSUPPORTED;
  const bool data = ptrs && p->n > 0 && p->nvec > 0;
  if (e->ldw < p->kin) return VQ_ERR_INVALID_ARG;
  if (data && !e->w) return VQ_ERR_INVALID_ARG;
  if (data && !aligned(e->w, 2)) return VQ_ERR_ALIGNMENT;
  p->hw = e->h != nullptr;
  p->mt = (p->n + kEncM - 1) / kEncM;
  if (p->hw) {
    if (p->d > kEncHMaxD) return VQ_ERR_UNSUPPORTED;
    if (e->ldh < p->kin) return VQ_ERR_INVALID_ARG;
    if (!aligned(e->h, 4)) return VQ_ERR_ALIGNMENT;
    if (static_cast<int64_t>(p->nfull) * p->mt >= (int64_t{1} << 31) || p->nfull > 65535)
      return VQ_ERR_UNSUPPORTED;
  }
  size_t off = 256;
  for (int m = 0; m < p->nb; ++m) {
    if (e->log2k[m] < 1 || e->log2k[m] > 16) return VQ_ERR_INVALID_ARG;
    p->b[m] = e->log2k[m];
    p->K[m] = 1 << p->b[m];
    p->kp[m] = (p->K[m] + kEncBlockK - 1) / kEncBlockK * kEncBlockK;
    const int64_t need = (static_cast<int64_t>(p->nvec) * p->b[m] + 127) / 128 * 4;
    if (e->idx_row_words[m] < need || e->idx_row_words[m] % 4 != 0) return VQ_ERR_INVALID_ARG;
    if (data) {
      if (!e->codebook[m] || !e->idx[m]) return VQ_ERR_INVALID_ARG;
      if (!aligned(e->codebook[m], 2)) return VQ_ERR_ALIGNMENT;
      if (!aligned(e->idx[m], 16)) return VQ_ERR_ALIGNMENT;
    }
    p->off_bprep[m] = off;
    off = enc_round256(off + static_cast<size_t>(p->kp[m]) * 32);
    p->off_book64[m] = off;
    off = enc_round256(off + static_cast<size_t>(p->K[m]) * p->d * 8);
  }
  const size_t nv = static_cast<size_t>(p->n) * p->nvec;
  for (int m = 0; m < p->nb; ++m) {
    p->off_idx[m] = off;
    off = enc_round256(off + nv * 4);
  }
  for (int m = 0; m < p->nb; ++m) {   // weighted form: c~^T H_j c~ per block and centroid,
    p->off_nc[m] = off;                 // then its error scale per block
    if (p->hw) off = enc_round256(off + static_cast<size_t>(p->nfull) * p->kp[m] * 4);
    p->off_ncabs[m] = off;
    if (p->hw) off = enc_round256(off + static_cast<size_t>(p->nfull) * 4);
  }
  p->off_list = off;
  off = enc_round256(off + nv * 4);
  p->total = (p->n > 0 && p->nvec > 0) ? off : 0;
  return VQ_OK;
}

}  // namespace
}  // namespace vqk

using namespace vqk;

extern "C" {

vq_status vq_encode_workspace_size(const vq_encode_desc* desc, size_t* bytes) {
  if (!bytes) return VQ_ERR_INVALID_ARG;
  EncPlan p;
  vq_status st = enc_check(desc, &p, false);
  if (st != VQ_OK) return st;
  *bytes = p.total;
  return VQ_OK;
}

vq_status vq_encode(const vq_encode_desc* desc, void* workspace, size_t workspace_bytes, void* stream_) {
  EncPlan p;
  vq_status st = enc_check(desc, &p, true);
  if (st != VQ_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (p.n == 0) return VQ_OK;
  if (p.nvec == 0) {                 // empty rows: the streams hold only padding
    for (int m = 0; m < p.nb; ++m) {
      if (desc->idx_row_words[m] == 0) continue;
      if (!desc->idx[m]) return VQ_ERR_INVALID_ARG;
      cudaError_t e = cudaMemset2DAsync(desc->idx[m], desc->idx_row_words[m] * 4, 0,
                                        desc->idx_row_words[m] * 4, p.n, stream);
      if (e != cudaSuccess) return cuda_status(e);
    }
    return VQ_OK;
  }
  if (!workspace || workspace_bytes < p.total) return VQ_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return VQ_ERR_ALIGNMENT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  EncWsCtrl* wc = reinterpret_cast<EncWsCtrl*>(ws);
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, stream);
  if (e != cudaSuccess) return cuda_status(e);

  for (int m = 0; m < p.nb; ++m) {
    count_launch();
    enc_book_norm_kernel<<<std::min(256, (p.K[m] + 255) / 256), 256, 0, stream>>>(
        desc->codebook[m], p.K[m], p.d, &wc->cmax_bits[m]);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
    count_launch();
    enc_book_prep_kernel<<<(p.kp[m] + 255) / 256, 256, 0, stream>>>(
        desc->codebook[m], p.K[m], p.d, p.kp[m], &wc->cmax_bits[m], ws + p.off_bprep[m], p.hw ? 1 : 0);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
    if (p.hw && p.nfull > 0) {
      e = cudaMemsetAsync(ws + p.off_ncabs[m], 0, static_cast<size_t>(p.nfull) * 4, stream);
      if (e != cudaSuccess) return cuda_status(e);
      count_launch();
      enc_nc_kernel<<<dim3(p.kp[m] / 256, p.nfull), 256, 0, stream>>>(
          desc->codebook[m], p.K[m], p.d, p.kp[m], &wc->cmax_bits[m], desc->h, desc->ldh,
          reinterpret_cast<float*>(ws + p.off_nc[m]), reinterpret_cast<unsigned*>(ws + p.off_ncabs[m]));
      if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
    }
    const int64_t cnt = static_cast<int64_t>(p.K[m]) * p.d;
    count_launch();
    enc_book64_kernel<<<static_cast<unsigned>((cnt + 255) / 256), 256, 0, stream>>>(
        desc->codebook[m], cnt, reinterpret_cast<double*>(ws + p.off_book64[m]));
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }

  const int smem = static_cast<int>(sizeof(EncCtrl)) + 1024 + kEncATile + kEncStages * kEncBlockBytes;
  auto tck = p.hw ? enc_tc_kernel<true> : enc_tc_kernel<false>;
  e = set_func_attr(reinterpret_cast<const void*>(tck), cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_status(e);
  int* list = reinterpret_cast<int*>(ws + p.off_list);
  for (int m = 0; m < p.nb; ++m) {
    uint32_t* idx_out = reinterpret_cast<uint32_t*>(ws + p.off_idx[m]);
    const uint32_t* idx1 = m == 1 ? reinterpret_cast<const uint32_t*>(ws + p.off_idx[0]) : nullptr;
    const uint16_t* book1 = m == 1 ? desc->codebook[0] : nullptr;
    if (p.nv_full > 0) {
      EncArgs a;
      a.w = desc->w;
      a.ldw = desc->ldw;
      a.n = p.n;
      a.kin = p.kin;
      a.d = p.d;
      a.nfull = p.nfull;
      a.nvec = p.nvec;
      a.nv_full = p.nv_full;
      a.bprep = ws + p.off_bprep[m];
      a.kp = p.kp[m];
      a.K = p.K[m];
      a.cmax_bits = &wc->cmax_bits[m];
      a.book64 = reinterpret_cast<const double*>(ws + p.off_book64[m]);
      a.book1 = book1;
      a.idx1 = idx1;
      a.idx_out = idx_out;
      a.list = list;
      a.list_count = &wc->list_count[m];
      a.status = &wc->status;
      a.h = desc->h;
      a.ldh = desc->ldh;
      a.nc = p.hw ? reinterpret_cast<const float*>(ws + p.off_nc[m]) : nullptr;
      a.ncabs = p.hw ? reinterpret_cast<const unsigned*>(ws + p.off_ncabs[m]) : nullptr;
      a.mt = p.mt;
      const int64_t grid = p.hw ? static_cast<int64_t>(p.nfull) * p.mt : (p.nv_full + kEncM - 1) / kEncM;
      count_launch();
      tck<<<static_cast<unsigned>(grid), kEncThreads, smem, stream>>>(a);
      if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
    }
    EncExactArgs x;
    x.w = desc->w;
    x.ldw = desc->ldw;
    x.n = p.n;
    x.kin = p.kin;
    x.d = p.d;
    x.nvec = p.nvec;
    x.book64 = reinterpret_cast<const double*>(ws + p.off_book64[m]);
    x.K = p.K[m];
    x.book1 = book1;
    x.idx1 = idx1;
    x.idx_out = idx_out;
    x.list = list;
    x.list_count = &wc->list_count[m];
    x.partial_rows = p.nfull < p.nvec ? p.n : 0;
    x.h = desc->h;
    x.ldh = desc->ldh;
    count_launch();
    const int xsmem = kEncExactTile * p.d * static_cast<int>(sizeof(double));
    auto xk = p.hw ? enc_exact_kernel<true> : enc_exact_kernel<false>;
    if (m == 0) {
      e = set_func_attr(reinterpret_cast<const void*>(xk), cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kEncExactTile * kEncMaxD * static_cast<int>(sizeof(double)));
      if (e != cudaSuccess) return cuda_status(e);
    }
    xk<<<2 * device_sm_count(), kEncExactThreads, xsmem, stream>>>(x);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  for (int m = 0; m < p.nb; ++m) {
    const int64_t words = static_cast<int64_t>(p.n) * desc->idx_row_words[m];
    count_launch();
    enc_pack_kernel<<<static_cast<unsigned>((words + 255) / 256), 256, 0, stream>>>(
        reinterpret_cast<const uint32_t*>(ws + p.off_idx[m]), p.n, p.nvec, p.b[m], desc->idx[m],
        desc->idx_row_words[m]);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  return VQ_OK;
}

}  // extern "C"

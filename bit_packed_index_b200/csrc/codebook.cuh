// codebook.cuh -- centroid loads for libvq's kernels.
//
// A codebook is read either from shared memory, where it was staged with rows
// padded to 8 (d <= 8) or 16 halves, or straight from global memory with rows
// of d halves (the large 2^16-entry books, served by L1/L2).  Both cases are
// described by a generic pointer and a row stride in halves, so one load
// routine serves both; the stride also fixes the vector width of the load.
#pragma once

#include "vq_internal.cuh"

namespace vqk {

struct BookView {
  const uint16_t* base;  // generic address: shared or global
  int stride;            // halves between rows
};

__device__ __forceinline__ void unpack8(const uint4& v, float* c) {
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&v.y));
  const float2 e = __half22float2(*reinterpret_cast<const __half2*>(&v.z));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&v.w));
  c[0] = a.x; c[1] = a.y; c[2] = b.x; c[3] = b.y;
  c[4] = e.x; c[5] = e.y; c[6] = f.x; c[7] = f.y;
}

// c[0..d) = fp32 values of row k.  D is 8, 6 or 0 (any d <= 16).
template <int D>
__device__ __forceinline__ void load_centroid(const BookView& bv, uint32_t k, int d, float* c) {
  const uint16_t* row = bv.base + static_cast<size_t>(k) * bv.stride;
  if constexpr (D == 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(row);   // stride 8: 16-byte rows
    unpack8(v, c);
  } else if constexpr (D == 6) {
    if (bv.stride == 8) {
      const uint4 v = *reinterpret_cast<const uint4*>(row);
      float t[8];
      unpack8(v, t);
#pragma unroll
      for (int e = 0; e < 6; ++e) c[e] = t[e];
    } else {                                                  // stride 6: 12-byte rows
      const uint32_t* r = reinterpret_cast<const uint32_t*>(row);
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const uint32_t w = r[q];
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
        c[2 * q] = f.x;
        c[2 * q + 1] = f.y;
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < kMaxVecDim; ++e) c[e] = (e < d) ? h2f(row[e]) : 0.0f;
  }
}

// Shared-memory bytes to stage a book with padded rows.
__host__ __device__ inline size_t padded_book_bytes(int b, int d) {
  return (static_cast<size_t>(1) << b) * (d <= 8 ? 8 : 16) * sizeof(uint16_t);
}

// Which books to stage in shared memory: book m is staged (bit m of *mask)
// while the running total stays within `budget` bytes.  Returns the bytes.
inline size_t stage_plan(const Layer& L, size_t budget, int* mask) {
  size_t used = 0;
  *mask = 0;
  for (int m = 0; m < L.nb; ++m) {
    const size_t b = padded_book_bytes(L.b[m], L.d);
    if (used + b <= budget) {
      used += b;
      *mask |= 1 << m;
    }
  }
  return used;
}

}  // namespace vqk

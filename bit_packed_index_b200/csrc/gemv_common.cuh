// gemv_common.cuh -- index and centroid loads shared by the decode kernels
// (gemv1.cu: batch 1; gemvb.cu: batch 2..16).
//
// Index words are read with L1::no_allocate (each is used once) and
// L2-served centroid rows with L1::evict_last, so L1 keeps codebook rows.
#pragma once

#include "codebook.cuh"

namespace vqk {
namespace dec {

__device__ __forceinline__ uint32_t ld_na(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// f[v] = index field v0 + v (v < G) of a stream row of rw words.  When G*B is
// a multiple of 32 a lane's fields start on a word boundary (v0 is a multiple
// of G) and are read with one 4-16 byte load; otherwise field by field.
// Words at or past the row end read as zero (their fields lie past the last
// vector and are never used).
template <int G, int B>
__device__ __forceinline__ void load_fields(const uint32_t* __restrict__ row, int64_t rw, int v0,
                                            uint32_t (&f)[G]) {
  constexpr uint32_t mask = (1u << B) - 1u;
  if constexpr ((G * B) % 32 == 0) {
    constexpr int NW = (G * B) / 32;
    const int64_t w0 = (static_cast<int64_t>(v0) * B) >> 5;
    const uint32_t* p = row + w0;
    uint32_t w[NW + 1];
    if (w0 + NW <= rw) {
      if constexpr (NW == 4) {
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "l"(p));
      } else if constexpr (NW == 2) {
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                     : "=r"(w[0]), "=r"(w[1]) : "l"(p));
      } else {
#pragma unroll
        for (int i = 0; i < NW; ++i) w[i] = ld_na(p + i);
      }
    } else {
#pragma unroll
      for (int i = 0; i < NW; ++i) w[i] = (w0 + i < rw) ? ld_na(p + i) : 0u;
    }
    w[NW] = 0u;
#pragma unroll
    for (int v = 0; v < G; ++v) {
      const int bit = v * B;                   // compile-time after unrolling
      f[v] = __funnelshift_r(w[bit >> 5], w[(bit >> 5) + 1], bit & 31) & mask;
    }
  } else {
#pragma unroll
    for (int v = 0; v < G; ++v) {
      const int64_t bit = static_cast<int64_t>(v0 + v) * B;
      const int64_t wi = bit >> 5;
      const int sh = static_cast<int>(bit & 31);
      const uint32_t lo = wi < rw ? ld_na(row + wi) : 0u;
      const uint32_t hi = (sh + B > 32 && wi + 1 < rw) ? ld_na(row + wi + 1) : 0u;
      f[v] = __funnelshift_r(lo, hi, sh) & mask;
    }
  }
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

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// The (d, index widths) pairs the decode kernels specialise for.
__host__ __device__ inline bool decode_fast_path(int d, int b1, int b2) {
  if (d == 8 && b1 == 16 && (b2 == 0 || b2 == 8)) return true;
  if (d == 8 && b1 == 12 && b2 == 8) return true;
  if (d == 8 && b1 == 8 && (b2 == 8 || b2 == 0)) return true;
  if (d == 6 && b1 == 12 && (b2 == 4 || b2 == 0)) return true;
  return false;
}

}  // namespace dec
}  // namespace vqk

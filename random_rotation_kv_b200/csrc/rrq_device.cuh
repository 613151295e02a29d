// rrq_device.cuh — device building blocks shared by the rrq kernels (sm_100a).
//
// Lane layout.  A vector of D coordinates is owned by a group of G consecutive
// lanes of a warp (32/G vectors per warp).  The vector is cut into chunks of 8
// consecutive coordinates (16 bytes of fp16/bf16); chunk q lives in lane
// h = q mod G, slot s = q / G, so one 16-byte load instruction of the warp
// reads G·16 contiguous bytes of every vector it touches (fully used
// sectors).  Lane h therefore holds C = D/G values v[r], r = s·8 + e, for
// coordinate i = (s·G + h)·8 + e.  In the bits of i: bits 0..2 are e (local),
// bits 3..3+log2(G)−1 are the lane bits h, the rest are s (local).
//
// Walsh–Hadamard transform.  The unnormalised transform y = H·v with
// H_ij = (−1)^popcount(i&j) factors into one butterfly (a, b) → (a+b, a−b)
// per bit of i, in any order.  Local bits are butterflies between registers;
// lane bits are one __shfl_xor_sync per value, the lower lane adding and the
// upper lane subtracting.  ("Random-rotation quantization" page, section "Why
// rotation works": the randomized Hadamard transform, O(d log d).)
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "rrq_params.h"

namespace rrq {

constexpr unsigned kFull = 0xffffffffu;

// ----------------------------------------------------------------- SplitMix64
// Output number c of SplitMix64 seeded with `seed` (Steele, Lea & Flood 2014;
// constants of the public reference implementation).
__host__ __device__ __forceinline__ uint64_t splitmix64_at(uint64_t seed, uint64_t c) {
  uint64_t z = seed + (c + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Rotation sign of coordinate i: 1 (negative) when bit 63 of output i is set.
__host__ __device__ __forceinline__ uint32_t sign_bit(uint64_t seed, int i) {
  return uint32_t(splitmix64_at(seed, uint64_t(i)) >> 63);
}

// ------------------------------------------------------------ element types
template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kDtype = RRQ_F32;
  static constexpr int kBytes = 4;
};
template <> struct Elem<__half> {
  static constexpr int kDtype = RRQ_F16;
  static constexpr int kBytes = 2;
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int kDtype = RRQ_BF16;
  static constexpr int kBytes = 2;
};

// Sign-flip masks in shared memory, one 32-bit XOR word per pair of 16-bit
// elements (sign bits 15 and 31) or per fp32 element (bit 31).
template <typename T> struct SignMask {
  static constexpr int kWordsPerChunk = (Elem<T>::kBytes == 2) ? 4 : 8;
  template <int D> static constexpr int words() { return D / 8 * kWordsPerChunk; }
};

template <typename T, int D>
__device__ __forceinline__ void build_sign_mask(uint32_t* smask, uint64_t seed) {
  if constexpr (Elem<T>::kBytes == 2) {
    for (int k = threadIdx.x; k < D / 2; k += blockDim.x) {
      smask[k] = (sign_bit(seed, 2 * k) << 15) | (sign_bit(seed, 2 * k + 1) << 31);
    }
  } else {
    for (int i = threadIdx.x; i < D; i += blockDim.x) smask[i] = sign_bit(seed, i) << 31;
  }
}

// ----------------------------------------------------- 16-byte memory helpers
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void st_stream(void* p, uint4 v) {
  __stcs(reinterpret_cast<uint4*>(p), v);
}
__device__ __forceinline__ uint4 xor4(uint4 a, uint4 b) {
  return make_uint4(a.x ^ b.x, a.y ^ b.y, a.z ^ b.z, a.w ^ b.w);
}

// 2 packed 16-bit elements -> 2 floats (exact)
template <typename T> __device__ __forceinline__ float2 unpack2(uint32_t w);
template <> __device__ __forceinline__ float2 unpack2<__half>(uint32_t w) {
  __half2 h = *reinterpret_cast<__half2*>(&w);
  return __half22float2(h);
}
template <> __device__ __forceinline__ float2 unpack2<__nv_bfloat16>(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// 2 floats -> 2 packed 16-bit elements, round to nearest even
template <typename T> __device__ __forceinline__ uint32_t pack2(float a, float b);
template <> __device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------- lane layout
template <int D, int G> struct Layout {
  static_assert(D % (8 * G) == 0, "D must be a multiple of 8*G");
  static constexpr int C = D / G;     // values per lane
  static constexpr int S = C / 8;     // chunks per lane
  static constexpr int VPW = 32 / G;  // vectors per warp
  __host__ __device__ static constexpr int chunk(int s, int h) { return s * G + h; }
};

// Sum over the G lanes of a group.
template <int G>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int m = 1; m < G; m <<= 1) x += __shfl_xor_sync(kFull, x, m);
  return x;
}

// ---------------------------------------------------------- packed fp32 pairs
// sm_100 issues two fp32 additions / multiplies per instruction (f32x2).  All
// of these round each component once, exactly like the scalar operation.
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.f, -1.f), a);  // a − b (b·(−1) is exact)
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Unnormalised Walsh–Hadamard transform on packed pairs: w[k] holds values
// r = 2k and 2k+1 of the lane (same coordinate map as fwht above).  Bit 0 of r
// is a butterfly inside each pair; the other local bits pair whole registers.
template <int D, int G>
__device__ __forceinline__ void fwht2(float2 (&w)[D / G / 2], int h) {
  constexpr int P = D / G / 2;
#pragma unroll
  for (int k = 0; k < P; ++k) {
    const float a = w[k].x, b = w[k].y;
    w[k] = make_float2(a + b, a - b);
  }
#pragma unroll
  for (int mm = 1; mm < P; mm <<= 1) {
#pragma unroll
    for (int k = 0; k < P; ++k) {
      if ((k & mm) == 0) {
        const float2 a = w[k], b = w[k | mm];
        w[k] = add2(a, b);
        w[k | mm] = sub2(a, b);
      }
    }
  }
#pragma unroll
  for (int m = 1; m < G; m <<= 1) {
    const float sg = (h & m) ? -1.f : 1.f;
    const float2 sgn = make_float2(sg, sg);
#pragma unroll
    for (int k = 0; k < P; ++k) {
      const float2 t = make_float2(__shfl_xor_sync(kFull, w[k].x, m), __shfl_xor_sync(kFull, w[k].y, m));
      w[k] = fma2(w[k], sgn, t);  // lower lane: w + t; upper lane: t − w
    }
  }
}

// One chunk (8 elements) of raw input words -> 4 packed pairs, sign masks applied.
template <typename T, bool FLIP>
__device__ __forceinline__ void chunk_to_pairs(const uint4* raw, const uint4* mask, float2* w) {
  if constexpr (Elem<T>::kBytes == 2) {
    uint4 r = raw[0];
    if constexpr (FLIP) r = xor4(r, mask[0]);
    w[0] = unpack2<T>(r.x); w[1] = unpack2<T>(r.y); w[2] = unpack2<T>(r.z); w[3] = unpack2<T>(r.w);
  } else {
    uint4 r0 = raw[0], r1 = raw[1];
    if constexpr (FLIP) { r0 = xor4(r0, mask[0]); r1 = xor4(r1, mask[1]); }
    w[0] = make_float2(__uint_as_float(r0.x), __uint_as_float(r0.y));
    w[1] = make_float2(__uint_as_float(r0.z), __uint_as_float(r0.w));
    w[2] = make_float2(__uint_as_float(r1.x), __uint_as_float(r1.y));
    w[3] = make_float2(__uint_as_float(r1.z), __uint_as_float(r1.w));
  }
}

// Raw 16-byte words of one vector owned by a lane (S chunks; 2 words per chunk for fp32).
template <typename T, int D, int G> struct RawVec {
  static constexpr int kWordsPerChunk = Elem<T>::kBytes == 2 ? 1 : 2;
  static constexpr int N = Layout<D, G>::S * kWordsPerChunk;
  uint4 r[N];
  __device__ __forceinline__ void load(const T* __restrict__ row, bool valid, int h) {
#pragma unroll
    for (int s = 0; s < Layout<D, G>::S; ++s) {
      const int q = Layout<D, G>::chunk(s, h);
#pragma unroll
      for (int c = 0; c < kWordsPerChunk; ++c)
        r[s * kWordsPerChunk + c] =
            valid ? ld_stream(row + q * 8 + c * 4) : make_uint4(0, 0, 0, 0);
    }
  }
};

// Lanes per vector for a head dimension: 2 up to d = 128, then 64 values a lane.
template <int D> struct GroupOf { static constexpr int value = D <= 128 ? 2 : D / 64; };

}  // namespace rrq

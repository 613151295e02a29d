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

// Load chunk-by-chunk (optionally XOR-ing the sign masks of D first) into v.
// `row` points at the vector's first element; `valid` false yields zeros.
template <typename T, int D, int G, bool FLIP>
__device__ __forceinline__ void load_vector(const T* __restrict__ row, bool valid, int h,
                                            const uint32_t* smask, float (&v)[D / G]) {
  using L = Layout<D, G>;
#pragma unroll
  for (int s = 0; s < L::S; ++s) {
    const int q = L::chunk(s, h);
    if constexpr (Elem<T>::kBytes == 2) {
      uint4 raw = valid ? ld_stream(row + q * 8) : make_uint4(0, 0, 0, 0);
      if constexpr (FLIP) raw = xor4(raw, reinterpret_cast<const uint4*>(smask)[q]);
      const float2 a = unpack2<T>(raw.x), b = unpack2<T>(raw.y);
      const float2 c = unpack2<T>(raw.z), d = unpack2<T>(raw.w);
      v[s * 8 + 0] = a.x; v[s * 8 + 1] = a.y; v[s * 8 + 2] = b.x; v[s * 8 + 3] = b.y;
      v[s * 8 + 4] = c.x; v[s * 8 + 5] = c.y; v[s * 8 + 6] = d.x; v[s * 8 + 7] = d.y;
    } else {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint4 raw = valid ? ld_stream(row + q * 8 + half * 4) : make_uint4(0, 0, 0, 0);
        if constexpr (FLIP) raw = xor4(raw, reinterpret_cast<const uint4*>(smask)[q * 2 + half]);
        v[s * 8 + half * 4 + 0] = __uint_as_float(raw.x);
        v[s * 8 + half * 4 + 1] = __uint_as_float(raw.y);
        v[s * 8 + half * 4 + 2] = __uint_as_float(raw.z);
        v[s * 8 + half * 4 + 3] = __uint_as_float(raw.w);
      }
    }
  }
}

// Store v (times `scale`) chunk-by-chunk as T, optionally XOR-ing sign masks.
template <typename T, int D, int G, bool FLIP>
__device__ __forceinline__ void store_vector(T* __restrict__ row, bool valid, int h,
                                             const uint32_t* smask, const float (&v)[D / G],
                                             float scale) {
  using L = Layout<D, G>;
#pragma unroll
  for (int s = 0; s < L::S; ++s) {
    const int q = L::chunk(s, h);
    if constexpr (Elem<T>::kBytes == 2) {
      uint4 w;
      w.x = pack2<T>(v[s * 8 + 0] * scale, v[s * 8 + 1] * scale);
      w.y = pack2<T>(v[s * 8 + 2] * scale, v[s * 8 + 3] * scale);
      w.z = pack2<T>(v[s * 8 + 4] * scale, v[s * 8 + 5] * scale);
      w.w = pack2<T>(v[s * 8 + 6] * scale, v[s * 8 + 7] * scale);
      if constexpr (FLIP) w = xor4(w, reinterpret_cast<const uint4*>(smask)[q]);
      if (valid) st_stream(row + q * 8, w);
    } else {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint4 w;
        w.x = __float_as_uint(v[s * 8 + half * 4 + 0] * scale);
        w.y = __float_as_uint(v[s * 8 + half * 4 + 1] * scale);
        w.z = __float_as_uint(v[s * 8 + half * 4 + 2] * scale);
        w.w = __float_as_uint(v[s * 8 + half * 4 + 3] * scale);
        if constexpr (FLIP) w = xor4(w, reinterpret_cast<const uint4*>(smask)[q * 2 + half]);
        if (valid) st_stream(row + q * 8 + half * 4, w);
      }
    }
  }
}

// Unnormalised Walsh–Hadamard transform of the group's D values.
template <int D, int G>
__device__ __forceinline__ void fwht(float (&v)[D / G], int h) {
  constexpr int C = D / G;
#pragma unroll
  for (int m = 1; m < C; m <<= 1) {
#pragma unroll
    for (int r = 0; r < C; ++r) {
      if ((r & m) == 0) {
        const float a = v[r], b = v[r | m];
        v[r] = a + b;
        v[r | m] = a - b;
      }
    }
  }
#pragma unroll
  for (int m = 1; m < G; m <<= 1) {
    const float sgn = (h & m) ? -1.f : 1.f;
#pragma unroll
    for (int r = 0; r < C; ++r) {
      const float t = __shfl_xor_sync(kFull, v[r], m);
      v[r] = fmaf(v[r], sgn, t);  // lower lane: v + t; upper lane: t − v
    }
  }
}

// Sum over the G lanes of a group.
template <int G>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int m = 1; m < G; m <<= 1) x += __shfl_xor_sync(kFull, x, m);
  return x;
}

// Lanes per vector for a head dimension: 2 up to d = 128, then 64 values a lane.
template <int D> struct GroupOf { static constexpr int value = D <= 128 ? 2 : D / 64; };

}  // namespace rrq

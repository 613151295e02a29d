// quant_kernels.cuh — encode / decode / rotate kernels (templates).
//
// "Random-rotation quantization" page (brain.bigb.es):
//   scheme steps 1–3: rotate by Π, quantise each rotated coordinate with one
//   fixed codebook, decode and apply Πᵀ;
//   "History", EDEN bullet: normalise to ≈N(0,1), Lloyd–Max codebook;
//   TurboQuant bullet: one constant scale per vector;
//   "Three decoders, one rotation", MSE decoder: nearest of 2^b centroids.
//
// Per vector (one group of G lanes, see rrq_device.cuh):
//   encode: 16 B loads (issued one grid-stride iteration ahead) → XOR rotation
//           signs on the raw elements → ν² = Σx² (fp32 pairs, group shuffle
//           sum) → unnormalised FWHT y' = H·D·x = √d·Πx → code_i = #{k : y'_i >
//           ν·τ_k}, the same decision as u_i = y'_i/ν > τ_k with the scale
//           folded into the thresholds once per vector → b-bit packing.
//   decode: codes (loaded one iteration ahead) → levels c[code] → FWHT →
//           × ν/d → round to the output type → XOR rotation signs → 16 B stores.
//   rotate: y = Πx (signs, FWHT, × 1/√d) or y = Πᵀx (FWHT, × 1/√d, signs).
// Instruction economy matters more than anything else here: the kernels are
// issue-bound before they are HBM-bound, so arithmetic runs on packed fp32
// pairs and the codebook search is a branch-free binary search.
#pragma once

#include "rrq_device.cuh"

namespace rrq {

constexpr int kThreads = 256;

// ------------------------------------------------------------- code search
// Number of thresholds t[0..2^K−2] (ascending) strictly below a, by a K-level
// branch-free binary search: the predicate of each level picks the next
// threshold with a select, so a 16-level codebook costs 3 compares.
template <int K>
__device__ __forceinline__ uint32_t count_below(float a, const float (&t)[(1 << K) > 1 ? (1 << K) - 1 : 1]) {
  if constexpr (K == 0) {
    return 0u;
  } else if constexpr (K == 1) {
    return a > t[0] ? 1u : 0u;
  } else if constexpr (K == 2) {
    const bool p1 = a > t[1];
    const bool p0 = a > (p1 ? t[2] : t[0]);
    return (p1 ? 2u : 0u) + (p0 ? 1u : 0u);
  } else {
    static_assert(K == 3, "bits <= 4");
    const bool p2 = a > t[3];
    const bool p1 = a > (p2 ? t[5] : t[1]);
    const float hi = p2 ? t[6] : t[2];
    const float lo = p2 ? t[4] : t[0];
    const bool p0 = a > (p1 ? hi : lo);
    return (p2 ? 4u : 0u) + (p1 ? 2u : 0u) + (p0 ? 1u : 0u);
  }
}

// Code of one rotated value y' for an exactly symmetric codebook with L levels:
// T[j] = ν·τ_{L/2+j} (the positive thresholds; τ_{L/2−1} = 0).
//   y' > 0:  code = L/2 + #{j : |y'| > T_j}
//   y' ≤ 0:  code = L/2 − 1 − #{j : |y'| > T_j}
// The second line takes ties |y'| = T_j to the upper code where the exact rule
// (strict u > τ) takes the lower one; such values lie on a threshold, inside the
// band where codes are allowed to differ.  y' = ±0 gives L/2 − 1 exactly.
// With m' = (L/2 − 1) − m = m ^ (L/2 − 1): code = pos ? m' ^ (L − 1) : m'.
template <int B>
__device__ __forceinline__ uint32_t code_sym(float y, const float (&T)[(1 << (B - 1)) > 1 ? (1 << (B - 1)) - 1 : 1]) {
  constexpr uint32_t L = 1u << B;
  const uint32_t m = count_below<B - 1>(fabsf(y), T);
  const uint32_t mm = m ^ (L / 2 - 1);
  return y > 0.f ? (mm ^ (L - 1)) : mm;
}

// Any ascending codebook: code = #{k : y' > T_k}, T_k = ν·τ_k.
template <int L>
__device__ __forceinline__ uint32_t code_generic(float y, const float (&tg)[L - 1]) {
  uint32_t m = 0;
#pragma unroll
  for (int k = 0; k < L - 1; ++k) m += (y > tg[k]) ? 1u : 0u;
  return m;
}

// Chunk q of a packed row: 8 codes of B bits = B bytes at byte offset q·B,
// little endian (code e at bits [e·B, (e+1)·B)).
template <int B>
__device__ __forceinline__ void store_chunk(uint8_t* __restrict__ row, int q, uint32_t w) {
  if constexpr (B == 4) {
    reinterpret_cast<uint32_t*>(row)[q] = w;
  } else if constexpr (B == 2) {
    reinterpret_cast<uint16_t*>(row)[q] = uint16_t(w);
  } else if constexpr (B == 1) {
    row[q] = uint8_t(w);
  } else {
    row[3 * q + 0] = uint8_t(w);
    row[3 * q + 1] = uint8_t(w >> 8);
    row[3 * q + 2] = uint8_t(w >> 16);
  }
}

template <int B>
__device__ __forceinline__ uint32_t load_chunk(const uint8_t* __restrict__ row, int q) {
  if constexpr (B == 4) {
    return __ldcs(reinterpret_cast<const uint32_t*>(row) + q);
  } else if constexpr (B == 2) {
    return __ldcs(reinterpret_cast<const uint16_t*>(row) + q);
  } else if constexpr (B == 1) {
    return __ldcs(row + q);
  } else {
    return uint32_t(__ldcs(row + 3 * q)) | (uint32_t(__ldcs(row + 3 * q + 1)) << 8) |
           (uint32_t(__ldcs(row + 3 * q + 2)) << 16);
  }
}

// Packed pairs of one lane -> stored row (times `scale`), optional sign XOR.
template <typename T, int D, int G, bool FLIP>
__device__ __forceinline__ void store_pairs(T* __restrict__ row, bool valid, int h,
                                            const uint32_t* smask, const float2 (&w)[D / G / 2],
                                            float scale) {
  using Lay = Layout<D, G>;
  const float2 s2 = make_float2(scale, scale);
#pragma unroll
  for (int s = 0; s < Lay::S; ++s) {
    const int q = Lay::chunk(s, h);
    const float2 a = mul2(w[s * 4 + 0], s2), b = mul2(w[s * 4 + 1], s2);
    const float2 c = mul2(w[s * 4 + 2], s2), d = mul2(w[s * 4 + 3], s2);
    if constexpr (Elem<T>::kBytes == 2) {
      uint4 o = make_uint4(pack2<T>(a.x, a.y), pack2<T>(b.x, b.y), pack2<T>(c.x, c.y),
                           pack2<T>(d.x, d.y));
      if constexpr (FLIP) o = xor4(o, reinterpret_cast<const uint4*>(smask)[q]);
      if (valid) st_stream(row + q * 8, o);
    } else {
      uint4 o0 = make_uint4(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(b.x),
                            __float_as_uint(b.y));
      uint4 o1 = make_uint4(__float_as_uint(c.x), __float_as_uint(c.y), __float_as_uint(d.x),
                            __float_as_uint(d.y));
      if constexpr (FLIP) {
        o0 = xor4(o0, reinterpret_cast<const uint4*>(smask)[q * 2]);
        o1 = xor4(o1, reinterpret_cast<const uint4*>(smask)[q * 2 + 1]);
      }
      if (valid) {
        st_stream(row + q * 8, o0);
        st_stream(row + q * 8 + 4, o1);
      }
    }
  }
}

// Raw words -> packed pairs, with optional sign XOR.
template <typename T, int D, int G, bool FLIP>
__device__ __forceinline__ void raw_to_pairs(const RawVec<T, D, G>& raw, int h,
                                             const uint32_t* smask, float2 (&w)[D / G / 2]) {
  using Lay = Layout<D, G>;
  constexpr int WPC = RawVec<T, D, G>::kWordsPerChunk;
#pragma unroll
  for (int s = 0; s < Lay::S; ++s) {
    const int q = Lay::chunk(s, h);
    chunk_to_pairs<T, FLIP>(&raw.r[s * WPC], reinterpret_cast<const uint4*>(smask) + q * WPC,
                            &w[s * 4]);
  }
}

// ------------------------------------------------------------------ encode
template <typename T, int D, int B, bool SYM>
__global__ void __launch_bounds__(kThreads)
encode_kernel(const T* __restrict__ x, int64_t n, uint8_t* __restrict__ codes,
              float* __restrict__ norms, const QuantParams p) {
  constexpr int G = GroupOf<D>::value;
  using Lay = Layout<D, G>;
  constexpr int P = Lay::C / 2, S = Lay::S, VPW = Lay::VPW;
  constexpr int L = 1 << B;
  constexpr int CB = D * B / 8;  // code bytes per vector
  __shared__ __align__(16) uint32_t smask[SignMask<T>::template words<D>()];
  build_sign_mask<T, D>(smask, p.seed);
  __syncthreads();

  const int lane = threadIdx.x & 31, h = lane & (G - 1), vsub = lane / G;
  const int64_t gwarp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t stride = ((int64_t(gridDim.x) * blockDim.x) >> 5) * VPW;

  int64_t vec = gwarp * VPW + vsub;
  RawVec<T, D, G> nxt;
  nxt.load(x + vec * D, vec < n, h);
  for (int64_t base = gwarp * VPW; base < n; base += stride, vec += stride) {
    const bool valid = vec < n;
    float2 w[P];
    raw_to_pairs<T, D, G, true>(nxt, h, smask, w);
    nxt.load(x + (vec + stride) * D, vec + stride < n, h);  // next iteration, in flight now

    float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < P; ++k) ss2 = fma2(w[k], w[k], ss2);
    const float nu = sqrtf(group_sum<G>(ss2.x + ss2.y));
    fwht2<D, G>(w, h);
    const float ns = nu > 0.f ? nu : 1.f;  // ν = 0: y' = 0, u = 0 against the plain thresholds
    uint8_t* crow = codes + vec * CB;
    if constexpr (SYM) {
      float tp[L / 2 > 1 ? L / 2 - 1 : 1];
#pragma unroll
      for (int j = 0; j < L / 2 - 1; ++j) tp[j] = ns * p.thr[L / 2 + j];
#pragma unroll
      for (int s = 0; s < S; ++s) {
        uint32_t cw = 0;
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const float2 y = w[s * 4 + e / 2];
          cw |= code_sym<B>(y.x, tp) << (e * B);
          cw |= code_sym<B>(y.y, tp) << ((e + 1) * B);
        }
        if (valid) store_chunk<B>(crow, Lay::chunk(s, h), cw);
      }
    } else {
      float tg[L - 1];
#pragma unroll
      for (int k = 0; k < L - 1; ++k) tg[k] = ns * p.thr[k];
#pragma unroll
      for (int s = 0; s < S; ++s) {
        uint32_t cw = 0;
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const float2 y = w[s * 4 + e / 2];
          cw |= code_generic<L>(y.x, tg) << (e * B);
          cw |= code_generic<L>(y.y, tg) << ((e + 1) * B);
        }
        if (valid) store_chunk<B>(crow, Lay::chunk(s, h), cw);
      }
    }
    if (valid && h == 0) norms[vec] = nu;
  }
}

// ------------------------------------------------------------------ decode
template <typename T, int D, int B>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ norms, int64_t n,
              T* __restrict__ out, const QuantParams p) {
  constexpr int G = GroupOf<D>::value;
  using Lay = Layout<D, G>;
  constexpr int P = Lay::C / 2, S = Lay::S, VPW = Lay::VPW;
  constexpr int L = 1 << B;
  constexpr int CB = D * B / 8;
  __shared__ __align__(16) uint32_t smask[SignMask<T>::template words<D>()];
  __shared__ float slev[L];
  build_sign_mask<T, D>(smask, p.seed);
  if (threadIdx.x < L) slev[threadIdx.x] = p.levels[threadIdx.x];
  __syncthreads();

  const int lane = threadIdx.x & 31, h = lane & (G - 1), vsub = lane / G;
  const int64_t gwarp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t stride = ((int64_t(gridDim.x) * blockDim.x) >> 5) * VPW;

  int64_t vec = gwarp * VPW + vsub;
  uint32_t cw_next[S];
  float nu_next = 0.f;
  auto fetch = [&](int64_t v) {
    const bool ok = v < n;
    const uint8_t* crow = codes + v * CB;
#pragma unroll
    for (int s = 0; s < S; ++s) cw_next[s] = ok ? load_chunk<B>(crow, Lay::chunk(s, h)) : 0u;
    nu_next = ok ? __ldcs(norms + v) : 0.f;
  };
  fetch(vec);
  for (int64_t base = gwarp * VPW; base < n; base += stride, vec += stride) {
    const bool valid = vec < n;
    uint32_t cw[S];
#pragma unroll
    for (int s = 0; s < S; ++s) cw[s] = cw_next[s];
    const float nu = nu_next;
    fetch(vec + stride);  // next iteration, in flight now

    float2 w[P];
#pragma unroll
    for (int s = 0; s < S; ++s) {
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        w[s * 4 + e / 2] = make_float2(slev[(cw[s] >> (e * B)) & (L - 1)],
                                       slev[(cw[s] >> ((e + 1) * B)) & (L - 1)]);
      }
    }
    fwht2<D, G>(w, h);
    store_pairs<T, D, G, true>(out + vec * D, valid, h, smask, w, nu * p.inv_d);
  }
}

// ------------------------------------------------------------------ rotate
template <typename T, int D, bool INV>
__global__ void __launch_bounds__(kThreads)
rotate_kernel(const T* __restrict__ x, int64_t n, float* __restrict__ y, uint64_t seed,
              float inv_sqrt_d) {
  constexpr int G = GroupOf<D>::value;
  using Lay = Layout<D, G>;
  constexpr int P = Lay::C / 2, VPW = Lay::VPW;
  __shared__ __align__(16) uint32_t smask_in[SignMask<T>::template words<D>()];
  __shared__ __align__(16) uint32_t smask_out[SignMask<float>::template words<D>()];
  if constexpr (!INV) build_sign_mask<T, D>(smask_in, seed);
  else build_sign_mask<float, D>(smask_out, seed);
  __syncthreads();

  const int lane = threadIdx.x & 31, h = lane & (G - 1), vsub = lane / G;
  const int64_t gwarp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t stride = ((int64_t(gridDim.x) * blockDim.x) >> 5) * VPW;
  int64_t vec = gwarp * VPW + vsub;
  RawVec<T, D, G> nxt;
  nxt.load(x + vec * D, vec < n, h);
  for (int64_t base = gwarp * VPW; base < n; base += stride, vec += stride) {
    const bool valid = vec < n;
    float2 w[P];
    raw_to_pairs<T, D, G, !INV>(nxt, h, smask_in, w);
    nxt.load(x + (vec + stride) * D, vec + stride < n, h);
    fwht2<D, G>(w, h);
    store_pairs<float, D, G, INV>(y + vec * D, valid, h, smask_out, w, inv_sqrt_d);
  }
}

// ---------------------------------------------------------------- launchers
constexpr int vectors_per_block(int d) { return (kThreads / 32) * (32 / (d <= 128 ? 2 : d / 64)); }

template <typename T, int D, int B>
cudaError_t encode_db(const T* x, int64_t n, const QuantParams& p, uint8_t* codes, float* norms,
                      cudaStream_t stream) {
  const int64_t work = (n + vectors_per_block(D) - 1) / vectors_per_block(D);
  if (p.sym) {
    auto k = encode_kernel<T, D, B, true>;
    const int grid = grid_for(reinterpret_cast<const void*>(k), kThreads, 0, work);
    k<<<grid, kThreads, 0, stream>>>(x, n, codes, norms, p);
  } else {
    auto k = encode_kernel<T, D, B, false>;
    const int grid = grid_for(reinterpret_cast<const void*>(k), kThreads, 0, work);
    k<<<grid, kThreads, 0, stream>>>(x, n, codes, norms, p);
  }
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t encode_d(const T* x, int64_t n, const QuantParams& p, uint8_t* codes, float* norms,
                     cudaStream_t stream) {
  switch (p.bits) {
    case 1: return encode_db<T, D, 1>(x, n, p, codes, norms, stream);
    case 2: return encode_db<T, D, 2>(x, n, p, codes, norms, stream);
    case 3: return encode_db<T, D, 3>(x, n, p, codes, norms, stream);
    case 4: return encode_db<T, D, 4>(x, n, p, codes, norms, stream);
  }
  return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t encode_typed(const T* x, int64_t n, int d, const QuantParams& p, uint8_t* codes,
                         float* norms, cudaStream_t stream) {
  switch (d) {
    case 64: return encode_d<T, 64>(x, n, p, codes, norms, stream);
    case 128: return encode_d<T, 128>(x, n, p, codes, norms, stream);
    case 256: return encode_d<T, 256>(x, n, p, codes, norms, stream);
    case 512: return encode_d<T, 512>(x, n, p, codes, norms, stream);
  }
  return cudaErrorInvalidValue;
}

template <typename T, int D, int B>
cudaError_t decode_db(const uint8_t* codes, const float* norms, int64_t n, const QuantParams& p,
                      T* out, cudaStream_t stream) {
  const int64_t work = (n + vectors_per_block(D) - 1) / vectors_per_block(D);
  auto k = decode_kernel<T, D, B>;
  const int grid = grid_for(reinterpret_cast<const void*>(k), kThreads, 0, work);
  k<<<grid, kThreads, 0, stream>>>(codes, norms, n, out, p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t decode_d(const uint8_t* codes, const float* norms, int64_t n, const QuantParams& p,
                     T* out, cudaStream_t stream) {
  switch (p.bits) {
    case 1: return decode_db<T, D, 1>(codes, norms, n, p, out, stream);
    case 2: return decode_db<T, D, 2>(codes, norms, n, p, out, stream);
    case 3: return decode_db<T, D, 3>(codes, norms, n, p, out, stream);
    case 4: return decode_db<T, D, 4>(codes, norms, n, p, out, stream);
  }
  return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t decode_typed(const uint8_t* codes, const float* norms, int64_t n, int d,
                         const QuantParams& p, T* out, cudaStream_t stream) {
  switch (d) {
    case 64: return decode_d<T, 64>(codes, norms, n, p, out, stream);
    case 128: return decode_d<T, 128>(codes, norms, n, p, out, stream);
    case 256: return decode_d<T, 256>(codes, norms, n, p, out, stream);
    case 512: return decode_d<T, 512>(codes, norms, n, p, out, stream);
  }
  return cudaErrorInvalidValue;
}

template <typename T, int D>
cudaError_t rotate_d(const T* x, int64_t n, uint64_t seed, int inverse, float inv_sqrt_d, float* y,
                     cudaStream_t stream) {
  const int64_t work = (n + vectors_per_block(D) - 1) / vectors_per_block(D);
  if (inverse) {
    auto k = rotate_kernel<T, D, true>;
    const int grid = grid_for(reinterpret_cast<const void*>(k), kThreads, 0, work);
    k<<<grid, kThreads, 0, stream>>>(x, n, y, seed, inv_sqrt_d);
  } else {
    auto k = rotate_kernel<T, D, false>;
    const int grid = grid_for(reinterpret_cast<const void*>(k), kThreads, 0, work);
    k<<<grid, kThreads, 0, stream>>>(x, n, y, seed, inv_sqrt_d);
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t rotate_typed(const T* x, int64_t n, int d, uint64_t seed, int inverse, float inv_sqrt_d,
                         float* y, cudaStream_t stream) {
  switch (d) {
    case 64: return rotate_d<T, 64>(x, n, seed, inverse, inv_sqrt_d, y, stream);
    case 128: return rotate_d<T, 128>(x, n, seed, inverse, inv_sqrt_d, y, stream);
    case 256: return rotate_d<T, 256>(x, n, seed, inverse, inv_sqrt_d, y, stream);
    case 512: return rotate_d<T, 512>(x, n, seed, inverse, inv_sqrt_d, y, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rrq

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
//   encode: load 16 B chunks → XOR rotation signs on the raw elements →
//           ν² = Σx² (fp32, group shuffle sum) → unnormalised FWHT
//           y' = H·D·x = √d·Πx → code_i = #{k : y'_i > ν·τ_k} (the same
//           decision as u_i = y'_i/ν > τ_k, with the scale folded into the
//           thresholds once per vector) → b-bit packing → store codes and ν.
//   decode: codes → levels c[code] → FWHT → × ν/d → round to the output type
//           → XOR rotation signs → 16 B stores.
//   rotate: y = Πx (signs, FWHT, × 1/√d) or y = Πᵀx (FWHT, × 1/√d, signs).
#pragma once

#include "rrq_device.cuh"

namespace rrq {

constexpr int kThreads = 256;

// Code of one rotated value y' against the per-vector scaled thresholds, for an
// exactly symmetric codebook.  tb[j] = bits of ν·τ_{L/2+j} (positive, ascending).
// y' > 0:  code = L/2 + #{j : |y'| > T_j};
// y' ≤ 0:  code = L/2 − 1 − #{j : |y'| ≥ T_j}.
// For non-negative floats the bit patterns order like the values, and
// |y'| ≥ T ⇔ nextup(|y'|) > T ⇔ bits(|y'|) + 1 > bits(T), so both sides use
// one unsigned compare per threshold.  y' = ±0 gives L/2 − 1.
template <int L>
__device__ __forceinline__ uint32_t code_sym(float y, const uint32_t (&tb)[L / 2 > 1 ? L / 2 - 1 : 1]) {
  const uint32_t bits = __float_as_uint(y);
  const bool pos = int32_t(bits) > 0;
  const uint32_t key = (bits & 0x7fffffffu) + (pos ? 0u : 1u);
  uint32_t m = 0;
  if constexpr (L > 2) {
#pragma unroll
    for (int j = 0; j < L / 2 - 1; ++j) m += (key > tb[j]) ? 1u : 0u;
  }
  return pos ? uint32_t(L / 2) + m : uint32_t(L / 2 - 1) - m;
}

// Generic (any ascending codebook): code = #{k : y' > T_k}, T_k = ν·τ_k.
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
    return __ldg(reinterpret_cast<const uint32_t*>(row) + q);
  } else if constexpr (B == 2) {
    return __ldg(reinterpret_cast<const uint16_t*>(row) + q);
  } else if constexpr (B == 1) {
    return __ldg(row + q);
  } else {
    return uint32_t(__ldg(row + 3 * q)) | (uint32_t(__ldg(row + 3 * q + 1)) << 8) |
           (uint32_t(__ldg(row + 3 * q + 2)) << 16);
  }
}

// ------------------------------------------------------------------ encode
template <typename T, int D, int B, bool SYM>
__global__ void __launch_bounds__(kThreads)
encode_kernel(const T* __restrict__ x, int64_t n, uint8_t* __restrict__ codes,
              float* __restrict__ norms, const QuantParams p) {
  constexpr int G = GroupOf<D>::value;
  using Lay = Layout<D, G>;
  constexpr int C = Lay::C, S = Lay::S, VPW = Lay::VPW;
  constexpr int L = 1 << B;
  constexpr int CB = D * B / 8;  // code bytes per vector
  __shared__ __align__(16) uint32_t smask[SignMask<T>::template words<D>()];
  build_sign_mask<T, D>(smask, p.seed);
  __syncthreads();

  const int lane = threadIdx.x & 31, h = lane & (G - 1), vsub = lane / G;
  const int64_t gwarp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarp = (int64_t(gridDim.x) * blockDim.x) >> 5;

  for (int64_t base = gwarp * VPW; base < n; base += nwarp * VPW) {
    const int64_t vec = base + vsub;
    const bool valid = vec < n;
    float v[C];
    load_vector<T, D, G, true>(x + vec * D, valid, h, smask, v);
    float ss = 0.f;
#pragma unroll
    for (int r = 0; r < C; ++r) ss = fmaf(v[r], v[r], ss);
    const float nu = sqrtf(group_sum<G>(ss));
    fwht<D, G>(v, h);
    const float ns = nu > 0.f ? nu : 1.f;  // ν = 0: y' = 0, u = 0 against the plain thresholds
    uint8_t* crow = codes + vec * CB;
    if constexpr (SYM) {
      uint32_t tb[L / 2 > 1 ? L / 2 - 1 : 1];
#pragma unroll
      for (int j = 0; j < L / 2 - 1; ++j) tb[j] = __float_as_uint(ns * p.thr[L / 2 + j]);
#pragma unroll
      for (int s = 0; s < S; ++s) {
        uint32_t w = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) w |= code_sym<L>(v[s * 8 + e], tb) << (e * B);
        if (valid) store_chunk<B>(crow, Lay::chunk(s, h), w);
      }
    } else {
      float tg[L - 1];
#pragma unroll
      for (int k = 0; k < L - 1; ++k) tg[k] = ns * p.thr[k];
#pragma unroll
      for (int s = 0; s < S; ++s) {
        uint32_t w = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) w |= code_generic<L>(v[s * 8 + e], tg) << (e * B);
        if (valid) store_chunk<B>(crow, Lay::chunk(s, h), w);
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
  constexpr int C = Lay::C, S = Lay::S, VPW = Lay::VPW;
  constexpr int L = 1 << B;
  constexpr int CB = D * B / 8;
  __shared__ __align__(16) uint32_t smask[SignMask<T>::template words<D>()];
  __shared__ float slev[L];
  build_sign_mask<T, D>(smask, p.seed);
  if (threadIdx.x < L) slev[threadIdx.x] = p.levels[threadIdx.x];
  __syncthreads();

  const int lane = threadIdx.x & 31, h = lane & (G - 1), vsub = lane / G;
  const int64_t gwarp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarp = (int64_t(gridDim.x) * blockDim.x) >> 5;

  for (int64_t base = gwarp * VPW; base < n; base += nwarp * VPW) {
    const int64_t vec = base + vsub;
    const bool valid = vec < n;
    const uint8_t* crow = codes + vec * CB;
    float v[C];
#pragma unroll
    for (int s = 0; s < S; ++s) {
      const uint32_t w = valid ? load_chunk<B>(crow, Lay::chunk(s, h)) : 0u;
#pragma unroll
      for (int e = 0; e < 8; ++e) v[s * 8 + e] = slev[(w >> (e * B)) & (L - 1)];
    }
    const float nu = valid ? __ldg(norms + vec) : 0.f;
    fwht<D, G>(v, h);
    store_vector<T, D, G, true>(out + vec * D, valid, h, smask, v, nu * p.inv_d);
  }
}

// ------------------------------------------------------------------ rotate
template <typename T, int D, bool INV>
__global__ void __launch_bounds__(kThreads)
rotate_kernel(const T* __restrict__ x, int64_t n, float* __restrict__ y, uint64_t seed,
              float inv_sqrt_d) {
  constexpr int G = GroupOf<D>::value;
  using Lay = Layout<D, G>;
  constexpr int C = Lay::C, VPW = Lay::VPW;
  __shared__ __align__(16) uint32_t smask_in[SignMask<T>::template words<D>()];
  __shared__ __align__(16) uint32_t smask_out[SignMask<float>::template words<D>()];
  if constexpr (!INV) build_sign_mask<T, D>(smask_in, seed);
  else build_sign_mask<float, D>(smask_out, seed);
  __syncthreads();

  const int lane = threadIdx.x & 31, h = lane & (G - 1), vsub = lane / G;
  const int64_t gwarp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarp = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t base = gwarp * VPW; base < n; base += nwarp * VPW) {
    const int64_t vec = base + vsub;
    const bool valid = vec < n;
    float v[C];
    load_vector<T, D, G, !INV>(x + vec * D, valid, h, smask_in, v);
    fwht<D, G>(v, h);
    store_vector<float, D, G, INV>(y + vec * D, valid, h, smask_out, v, inv_sqrt_d);
  }
}

// ---------------------------------------------------------------- launchers
template <typename K>
inline int vectors_per_block(int d) {
  const int g = d <= 128 ? 2 : d / 64;
  return (kThreads / 32) * (32 / g);
}

template <typename T, int D, int B>
cudaError_t encode_db(const T* x, int64_t n, const QuantParams& p, uint8_t* codes, float* norms,
                      cudaStream_t stream) {
  const int64_t work = (n + vectors_per_block<T>(D) - 1) / vectors_per_block<T>(D);
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
  const int64_t work = (n + vectors_per_block<T>(D) - 1) / vectors_per_block<T>(D);
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
  const int64_t work = (n + vectors_per_block<T>(D) - 1) / vectors_per_block<T>(D);
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

// q4_0.cu — "Attn-rot" (TurboQuant lite): randomized Hadamard rotation, then
// q4_0 blocks of 32, and the inverse.
//
// "Attn-rot (TurboQuant lite) in llama.cpp" page: rotate K and V before an
// ordinary block format, q4_0 first of all.  The page names q4_0 without
// defining it; the public llama.cpp q4_0 block is used, kept identical for
// interoperability:
//   m = block element of largest |y| (first on ties), Δ = m/−8 (fp32),
//   q_j = min(15, ⌊fp32(fp32(y_j·inv) + 8.5)⌋), inv = fp32(1/Δ) (0 when Δ = 0),
//   18 bytes: fp16(Δ) little endian, then byte j = q_j | q_{j+16} << 4;
//   decode: (q_j − 8)·fp16(Δ).
// With rotation y = Πx = H·D·x/√d, decode applies Πᵀ = D·H/√d.
//
// Layout: the encoder's (64 values per lane, sectors of 16 interleaved over
// G = d/64 lanes, see rrq_device.cuh).  A block is two consecutive sectors;
// for G ≥ 2 they sit in lanes h and h^1 at the same slot, for G = 1 in one
// lane.  A warp always covers 64 blocks = 1152 bytes of output, staged in
// shared memory and written with 16-byte stores (decode reads the same way).
#include "rrq_device.cuh"

namespace rrq {
namespace {

constexpr int kQThreads = 128;
constexpr int kBlockBytes = 18;
constexpr int kWarpBytes = 64 * kBlockBytes;  // 1152

template <int D> struct QLay {
  static constexpr int C = D < 64 ? D : 64;
  using L = Layout<D, C>;
};

// Interleave two words of 8 nibbles: byte j = lo_j | hi_j << 4 (little endian).
__device__ __forceinline__ uint2 interleave_nibbles(uint32_t lo, uint32_t hi) {
  auto spread = [](uint32_t v) -> uint64_t {  // nibble j -> bits [8j, 8j+4)
    uint64_t x = v;
    x = (x | (x << 16)) & 0x0000FFFF0000FFFFull;
    x = (x | (x << 8)) & 0x00FF00FF00FF00FFull;
    x = (x | (x << 4)) & 0x0F0F0F0F0F0F0F0Full;
    return x;
  };
  const uint64_t r = spread(lo) | (spread(hi) << 4);
  return make_uint2(uint32_t(r), uint32_t(r >> 32));
}

// Largest |value| of 16 values (first index on ties): returns the signed value.
__device__ __forceinline__ float sector_absmax(const float2* w, float& amax) {
  float best = w[0].x, ba = fabsf(w[0].x);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float a0 = fabsf(w[k].x), a1 = fabsf(w[k].y);
    if (k > 0 && a0 > ba) { ba = a0; best = w[k].x; }
    if (a1 > ba) { ba = a1; best = w[k].y; }
  }
  amax = ba;
  return best;
}

// 16 codes of a sector as 8-nibble words (codes 0..7, 8..15).
__device__ __forceinline__ uint2 sector_codes_q4(const float2* w, float inv) {
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    // fp32 y·inv, then + 8.5, each rounded (no fused multiply-add), as the
    // format's reference arithmetic
    const int q0 = min(15, max(0, int(floorf(__fadd_rn(__fmul_rn(w[k].x, inv), 8.5f)))));
    const int q1 = min(15, max(0, int(floorf(__fadd_rn(__fmul_rn(w[k].y, inv), 8.5f)))));
    out[k / 4] |= (uint32_t(q0) << (8 * (k % 4))) | (uint32_t(q1) << (8 * (k % 4) + 4));
  }
  return make_uint2(out[0], out[1]);
}

__device__ __forceinline__ void st_u16(uint8_t* p, uint32_t v) { *reinterpret_cast<uint16_t*>(p) = uint16_t(v); }
__device__ __forceinline__ uint32_t ld_u16(const uint8_t* p) { return *reinterpret_cast<const uint16_t*>(p); }

// Copy `bytes` (a multiple of 2) of a warp's staging buffer to global memory.
__device__ __forceinline__ void warp_copy_out(uint8_t* __restrict__ dst, const uint8_t* src, int bytes,
                                              int lane) {
  const int full = bytes / 16;
  for (int i = lane; i < full; i += 32)
    reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(src)[i];
  for (int i = full * 8 + lane; i < bytes / 2; i += 32)
    reinterpret_cast<uint16_t*>(dst)[i] = reinterpret_cast<const uint16_t*>(src)[i];
}

__device__ __forceinline__ void warp_copy_in(uint8_t* dst, const uint8_t* __restrict__ src, int bytes,
                                             int lane) {
  const int full = bytes / 16;
  for (int i = lane; i < full; i += 32)
    reinterpret_cast<uint4*>(dst)[i] = __ldcs(reinterpret_cast<const uint4*>(src) + i);
  for (int i = full * 8 + lane; i < bytes / 2; i += 32)
    reinterpret_cast<uint16_t*>(dst)[i] = reinterpret_cast<const uint16_t*>(src)[i];
}

template <typename T, int D, bool ROT>
__global__ void __launch_bounds__(kQThreads) q4_encode_kernel(const T* __restrict__ x, int64_t n,
                                                              uint8_t* __restrict__ blocks,
                                                              uint64_t seed, float inv_sqrt_d) {
  pdl_release();
  using Lay = typename QLay<D>::L;
  constexpr int C = QLay<D>::C;
  constexpr int G = Lay::G, P = Lay::P, SEC = Lay::SEC, VPW = Lay::VPW;
  constexpr int OB = D / 32 * kBlockBytes;  // bytes per vector
  __shared__ __align__(16) uint32_t smask[mask_words<T, D>()];
  __shared__ __align__(16) uint8_t stage[kQThreads / 32][kWarpBytes];
  if constexpr (ROT) build_sign_mask<T, D>(smask, seed);
  __syncthreads();
  pdl_wait();  // from here on, global memory

  const int lane = threadIdx.x & 31, h = lane & (G - 1), vsub = lane / G;
  uint8_t* buf = stage[threadIdx.x >> 5];
  const int64_t gwarp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t stride = ((int64_t(gridDim.x) * blockDim.x) >> 5) * VPW;
  int64_t vec = gwarp * VPW + vsub;
  RawVec<T, D, C> nxt;
  nxt.load(x + vec * D, vec < n, h);
  for (int64_t base = gwarp * VPW; base < n; base += stride, vec += stride) {
    float2 w[P];
    raw_to_pairs<T, D, C, ROT>(nxt, h, smask, w);
    nxt.load(x + (vec + stride) * D, vec + stride < n, h);
    if constexpr (ROT) {
      fwht2<D, C>(w, h);
      const float2 s2 = make_float2(inv_sqrt_d, inv_sqrt_d);
#pragma unroll
      for (int k = 0; k < P; ++k) w[k] = mul2(w[k], s2);
    }
    uint8_t* vb = buf + vsub * OB;
    if constexpr (G == 1) {
#pragma unroll
      for (int b = 0; b < SEC / 2; ++b) {  // block b = sectors 2b, 2b+1
        float a0, a1;
        const float m0 = sector_absmax(&w[16 * b], a0);
        const float m1 = sector_absmax(&w[16 * b + 8], a1);
        const float m = a1 > a0 ? m1 : m0;
        const float delta = m * -0.125f;
        const float inv = delta != 0.f ? 1.f / delta : 0.f;
        // lo: codes 0..15 of the block, hi: codes 16..31 (nibble k of .x = code k, of .y = code 8+k)
        const uint2 lo = sector_codes_q4(&w[16 * b], inv), hi = sector_codes_q4(&w[16 * b + 8], inv);
        const uint2 b0 = interleave_nibbles(lo.x, hi.x), b1 = interleave_nibbles(lo.y, hi.y);
        uint8_t* blk = vb + b * kBlockBytes;
        st_u16(blk, __half_as_ushort(__float2half_rn(delta)));
        st_u16(blk + 2, b0.x); st_u16(blk + 4, b0.x >> 16); st_u16(blk + 6, b0.y); st_u16(blk + 8, b0.y >> 16);
        st_u16(blk + 10, b1.x); st_u16(blk + 12, b1.x >> 16); st_u16(blk + 14, b1.y); st_u16(blk + 16, b1.y >> 16);
      }
    } else {
#pragma unroll
      for (int s = 0; s < SEC; ++s) {  // sector q = s·G + h; block q/2 shared with lane h^1
        float am;
        const float mm = sector_absmax(&w[8 * s], am);
        const float pm = __shfl_xor_sync(kFull, mm, 1), pa = __shfl_xor_sync(kFull, am, 1);
        // the even lane holds the block's first half: the odd half wins only if strictly larger
        const float m = (h & 1) ? (am > pa ? mm : pm) : (pa > am ? pm : mm);
        const float delta = m * -0.125f;
        const float inv = delta != 0.f ? 1.f / delta : 0.f;
        const uint2 c = sector_codes_q4(&w[8 * s], inv);
        // even lane: needs partner's codes 0..7 (bytes 0..7); odd lane: partner's 8..15
        const uint32_t send = (h & 1) ? c.x : c.y;
        const uint32_t recv = __shfl_xor_sync(kFull, send, 1);
        const int q = Lay::sector(s, h);
        uint8_t* blk = vb + (q >> 1) * kBlockBytes;
        if ((h & 1) == 0) {
          const uint2 b0 = interleave_nibbles(c.x, recv);  // bytes 0..7
          st_u16(blk, __half_as_ushort(__float2half_rn(delta)));
          st_u16(blk + 2, b0.x); st_u16(blk + 4, b0.x >> 16); st_u16(blk + 6, b0.y); st_u16(blk + 8, b0.y >> 16);
        } else {
          const uint2 b1 = interleave_nibbles(recv, c.y);  // bytes 8..15
          st_u16(blk + 10, b1.x); st_u16(blk + 12, b1.x >> 16); st_u16(blk + 14, b1.y); st_u16(blk + 16, b1.y >> 16);
        }
      }
    }
    __syncwarp();
    const int64_t nvalid = n - base < VPW ? n - base : VPW;
    warp_copy_out(blocks + base * OB, buf, int(nvalid) * OB, lane);
    __syncwarp();
  }
}

template <typename T, int D, bool ROT>
__global__ void __launch_bounds__(kQThreads) q4_decode_kernel(const uint8_t* __restrict__ blocks,
                                                              int64_t n, T* __restrict__ out,
                                                              uint64_t seed, float inv_sqrt_d) {
  pdl_release();
  using Lay = typename QLay<D>::L;
  constexpr int C = QLay<D>::C;
  constexpr int G = Lay::G, P = Lay::P, SEC = Lay::SEC, VPW = Lay::VPW;
  constexpr int OB = D / 32 * kBlockBytes;
  __shared__ __align__(16) uint32_t smask[mask_words<T, D>()];
  __shared__ __align__(16) uint8_t stage[kQThreads / 32][kWarpBytes];
  if constexpr (ROT) build_sign_mask<T, D>(smask, seed);
  __syncthreads();
  pdl_wait();  // from here on, global memory

  const int lane = threadIdx.x & 31, h = lane & (G - 1), vsub = lane / G;
  uint8_t* buf = stage[threadIdx.x >> 5];
  const int64_t gwarp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t stride = ((int64_t(gridDim.x) * blockDim.x) >> 5) * VPW;
  int64_t vec = gwarp * VPW + vsub;
  for (int64_t base = gwarp * VPW; base < n; base += stride, vec += stride) {
    const int64_t nvalid = n - base < VPW ? n - base : VPW;
    warp_copy_in(buf, blocks + base * OB, int(nvalid) * OB, lane);
    __syncwarp();
    const uint8_t* vb = buf + vsub * OB;
    float2 w[P];
#pragma unroll
    for (int s = 0; s < SEC; ++s) {
      const int q = Lay::sector(s, h);  // sector q: block q/2, half q&1
      const uint8_t* blk = vb + (q >> 1) * kBlockBytes;
      const float delta = __half2float(__ushort_as_half(uint16_t(ld_u16(blk))));
      const int sh = (q & 1) ? 4 : 0;
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const uint32_t two = ld_u16(blk + 2 + j);  // bytes j, j+1
        const float c0 = float(int((two >> sh) & 15u) - 8), c1 = float(int((two >> (8 + sh)) & 15u) - 8);
        w[8 * s + j / 2] = make_float2(c0 * delta, c1 * delta);
      }
    }
    __syncwarp();
    if constexpr (ROT) {
      fwht2<D, C>(w, h);
      store_pairs<T, D, C, true>(out + vec * D, vec < n, h, smask, w, inv_sqrt_d);
    } else {
      store_pairs<T, D, C, false>(out + vec * D, vec < n, h, smask, w, 1.f);
    }
  }
}

template <typename T, int D>
cudaError_t q4_enc_d(const T* x, int64_t n, uint64_t seed, int rotate, float isd, uint8_t* blocks,
                     cudaStream_t stream) {
  constexpr int vpb = (kQThreads / 32) * QLay<D>::L::VPW;
  const int64_t work = (n + vpb - 1) / vpb;
  if (rotate) {
    auto k = q4_encode_kernel<T, D, true>;
    const int grid = grid_for(reinterpret_cast<const void*>(k), kQThreads, 0, work);
    const cudaError_t e = launch_pdl(k, grid, kQThreads, 0, stream, x, n, blocks, seed, isd);
    if (e != cudaSuccess) return e;
  } else {
    auto k = q4_encode_kernel<T, D, false>;
    const int grid = grid_for(reinterpret_cast<const void*>(k), kQThreads, 0, work);
    const cudaError_t e = launch_pdl(k, grid, kQThreads, 0, stream, x, n, blocks, seed, isd);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t q4_dec_d(const uint8_t* blocks, int64_t n, uint64_t seed, int rotate, float isd, T* out,
                     cudaStream_t stream) {
  constexpr int vpb = (kQThreads / 32) * QLay<D>::L::VPW;
  const int64_t work = (n + vpb - 1) / vpb;
  if (rotate) {
    auto k = q4_decode_kernel<T, D, true>;
    const int grid = grid_for(reinterpret_cast<const void*>(k), kQThreads, 0, work);
    const cudaError_t e = launch_pdl(k, grid, kQThreads, 0, stream, blocks, n, out, seed, isd);
    if (e != cudaSuccess) return e;
  } else {
    auto k = q4_decode_kernel<T, D, false>;
    const int grid = grid_for(reinterpret_cast<const void*>(k), kQThreads, 0, work);
    const cudaError_t e = launch_pdl(k, grid, kQThreads, 0, stream, blocks, n, out, seed, isd);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t q4_enc_t(const void* x, int64_t n, int d, uint64_t seed, int rotate, float isd, void* blocks,
                     cudaStream_t s) {
  const T* xx = static_cast<const T*>(x);
  uint8_t* b = static_cast<uint8_t*>(blocks);
  switch (d) {
    case 64: return q4_enc_d<T, 64>(xx, n, seed, rotate, isd, b, s);
    case 128: return q4_enc_d<T, 128>(xx, n, seed, rotate, isd, b, s);
    case 256: return q4_enc_d<T, 256>(xx, n, seed, rotate, isd, b, s);
    case 512: return q4_enc_d<T, 512>(xx, n, seed, rotate, isd, b, s);
  }
  return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t q4_dec_t(const void* blocks, int64_t n, int d, uint64_t seed, int rotate, float isd, void* out,
                     cudaStream_t s) {
  const uint8_t* b = static_cast<const uint8_t*>(blocks);
  T* o = static_cast<T*>(out);
  switch (d) {
    case 64: return q4_dec_d<T, 64>(b, n, seed, rotate, isd, o, s);
    case 128: return q4_dec_d<T, 128>(b, n, seed, rotate, isd, o, s);
    case 256: return q4_dec_d<T, 256>(b, n, seed, rotate, isd, o, s);
    case 512: return q4_dec_d<T, 512>(b, n, seed, rotate, isd, o, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_q4_0(const void* x, int dtype, int64_t n, int d, uint64_t seed, int rotate,
                        float inv_sqrt_d, void* blocks, cudaStream_t stream) {
  switch (dtype) {
    case RRQ_F16: return q4_enc_t<__half>(x, n, d, seed, rotate, inv_sqrt_d, blocks, stream);
    case RRQ_BF16: return q4_enc_t<__nv_bfloat16>(x, n, d, seed, rotate, inv_sqrt_d, blocks, stream);
    case RRQ_F32: return q4_enc_t<float>(x, n, d, seed, rotate, inv_sqrt_d, blocks, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_q4_0_decode(const void* blocks, int64_t n, int d, uint64_t seed, int rotate,
                               float inv_sqrt_d, void* out, int out_dtype, cudaStream_t stream) {
  switch (out_dtype) {
    case RRQ_F16: return q4_dec_t<__half>(blocks, n, d, seed, rotate, inv_sqrt_d, out, stream);
    case RRQ_BF16: return q4_dec_t<__nv_bfloat16>(blocks, n, d, seed, rotate, inv_sqrt_d, out, stream);
    case RRQ_F32: return q4_dec_t<float>(blocks, n, d, seed, rotate, inv_sqrt_d, out, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rrq

// q4_0.cu — "Attn-rot" (TurboQuant lite): randomized Hadamard rotation, then
// q4_0 blocks of 32, and the inverse.
//
// "Attn-rot (TurboQuant lite) in llama.cpp" page: rotate K and V before an
// ordinary block format, q4_0 first of all.  The page names q4_0 without
// defining it; the public llama.cpp q4_0 block is used, kept identical for
// interoperability:
//   m = block element of largest |y| (first on ties, +0 for a block of zeros),
//   Δ = m/−8 (fp32), q_j = min(15, ⌊fp32(fp32(y_j·inv) + 8.5)⌋), inv = fp32(1/Δ)
//   (0 when Δ = 0); 18 bytes: fp16(Δ) little endian, then byte j = q_j | q_{j+16} << 4;
//   decode: (q_j − 8)·fp16(Δ).
// With rotation y = Πx = H·D·x/√d, decode applies Πᵀ = D·H/√d.
//
// The encoder is the block-type kernel of ggml_blocks.cu.  The decoder here
// works in the encoder's lane layout (64 values per lane, sectors of 16
// interleaved over G = d/64 lanes, see rrq_device.cuh): a block is two
// consecutive sectors, for G ≥ 2 in lanes h and h^1 at the same slot, for G = 1
// in one lane.  A warp reads 64 blocks = 1152 bytes with 16-byte loads into
// shared memory and each lane decodes its own sectors from there.
#include "ggml_blocks.h"
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

__device__ __forceinline__ uint32_t ld_u16(const uint8_t* p) { return *reinterpret_cast<const uint16_t*>(p); }

__device__ __forceinline__ void warp_copy_in(uint8_t* dst, const uint8_t* __restrict__ src, int bytes,
                                             int lane) {
  const int full = bytes / 16;
  for (int i = lane; i < full; i += 32)
    reinterpret_cast<uint4*>(dst)[i] = __ldcs(reinterpret_cast<const uint4*>(src) + i);
  for (int i = full * 8 + lane; i < bytes / 2; i += 32)
    reinterpret_cast<uint16_t*>(dst)[i] = reinterpret_cast<const uint16_t*>(src)[i];
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
  return launch_ggml_blocks(x, dtype, n, d, seed, rotate, RRQ_GGML_Q4_0, inv_sqrt_d, blocks, stream);
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

// ggml_blocks.cu — "Attn-rot" with the GGML block types: randomized Hadamard
// rotation, then q4_0, q4_1, q5_0, q5_1 or q8_0 blocks of 32, and back (the q4_0
// decoder in q4_0.cu is used for q4_0 blocks; it reads them faster).
//
// "Attn-rot (TurboQuant lite) in llama.cpp" page, section "How to use it":
// besides q4_0, the cache types q4_1, q5_0 and q5_1 (and q8_0).  The page names
// them without defining them; the public llama.cpp blocks are used, kept
// identical for interoperability, with every decision in fp32 (each product,
// sum and quotient rounded, no fused multiply-add):
//   q4_0 (18 B): m = first element of largest |y| (+0 for a block of zeros),
//        Δ = m/−8, q = min(15, ⌊y·inv + 8.5⌋); fp16 Δ, 16 bytes q_j | q_{j+16} << 4.
//   q4_1 (20 B): lo/hi = first min/max in index order, Δ = (hi − lo)/15,
//        q = min(15, ⌊(y − lo)·inv + 0.5⌋); fp16 Δ, fp16 lo, 16 nibble bytes.
//   q5_0 (22 B): m = first element of largest |y| (+0 for a block of zeros),
//        Δ = m/−16, q = min(31, ⌊y·inv + 16.5⌋); fp16 Δ, a 32-bit word with bit j
//        = bit 4 of q_j, 16 bytes (q_j & 15) | (q_{j+16} & 15) << 4.
//   q5_1 (24 B): as q4_1 with 31 steps; fp16 Δ, fp16 lo, the high-bit word, nibbles.
//   q8_0 (34 B): Δ = max|y|/127, q = round(y·inv) (halves away from zero), int8.
// inv = fp32(1/Δ), 0 when Δ = 0.  Decode: q·Δ + lo, (q − 16)·Δ or q·Δ with the
// stored fp16 values, then Πᵀ when the vector was rotated.
//
// Layout.  The rotation runs in the encoder's lane layout (64 values per lane,
// sectors of 16 interleaved over G = d/64 lanes, see rrq_device.cuh).  A warp
// pass covers 32 × 64 = 2048 values = 64 blocks; the rotated values go through
// a per-warp shared tile with a row stride of 33 floats, and each lane then
// quantises whole blocks (lane and lane + 32), reading its block's 32 values
// without bank conflicts.  Block bytes are staged per warp and leave in 16-byte
// stores; the decoder runs the same way backwards.
#include "batch_kernels.cuh"
#include "ggml_blocks.h"
#include "rrq_device.cuh"
#include "tensor_map.h"

namespace rrq {
namespace {

constexpr int kBThreads = 128;
constexpr int kWarpBlocks = 64;  // blocks of 32 per warp pass (2048 values)
constexpr int kRow = 33;         // shared row stride of a block, in floats

template <int F> struct BlockType;
template <> struct BlockType<RRQ_GGML_Q4_0> { static constexpr int kBytes = 18; };
template <> struct BlockType<RRQ_GGML_Q4_1> { static constexpr int kBytes = 20; };
template <> struct BlockType<RRQ_GGML_Q5_0> { static constexpr int kBytes = 22; };
template <> struct BlockType<RRQ_GGML_Q5_1> { static constexpr int kBytes = 24; };
template <> struct BlockType<RRQ_GGML_Q8_0> { static constexpr int kBytes = 34; };

template <int D> using BLayout = Layout<D, 64>;

__device__ __forceinline__ void st16(uint8_t* p, uint32_t v) { *reinterpret_cast<uint16_t*>(p) = uint16_t(v); }
__device__ __forceinline__ uint32_t ld16(const uint8_t* p) { return *reinterpret_cast<const uint16_t*>(p); }
__device__ __forceinline__ uint32_t half_bits(float v) { return __half_as_ushort(__float2half_rn(v)); }
__device__ __forceinline__ float half_val(uint32_t b) { return __half2float(__ushort_as_half(uint16_t(b))); }

// 16 bytes, byte j = (q_j & 15) | (q_{j+16} & 15) << 4, as 8 little-endian 16-bit stores.
__device__ __forceinline__ void put_nibbles(uint8_t* p, const int (&q)[32]) {
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    const uint32_t b0 = uint32_t(q[j] & 15) | (uint32_t(q[j + 16] & 15) << 4);
    const uint32_t b1 = uint32_t(q[j + 1] & 15) | (uint32_t(q[j + 17] & 15) << 4);
    st16(p + j, b0 | (b1 << 8));
  }
}

__device__ __forceinline__ void put_high_bits(uint8_t* p, const int (&q)[32]) {
  uint32_t w = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) w |= uint32_t((q[j] >> 4) & 1) << j;
  st16(p, w);
  st16(p + 2, w >> 16);
}

// Quantise one block of 32 fp32 values into `out`; v(j) returns value j (a
// shared row, or registers: every j is a compile-time constant after unrolling).
template <int F, typename Get>
__device__ __forceinline__ void encode_block(Get v, uint8_t* out) {
  int q[32];
  if constexpr (F == RRQ_GGML_Q4_1 || F == RRQ_GGML_Q5_1) {
    constexpr int kTop = F == RRQ_GGML_Q4_1 ? 15 : 31;
    float lo = v(0), hi = v(0);
#pragma unroll
    for (int j = 1; j < 32; ++j) {  // strict: the first extreme in index order stays
      if (v(j) < lo) lo = v(j);
      if (v(j) > hi) hi = v(j);
    }
    const float dlt = __fdiv_rn(__fsub_rn(hi, lo), float(kTop));
    const float inv = dlt != 0.f ? __frcp_rn(dlt) : 0.f;  // 1/Δ, correctly rounded
#pragma unroll
    for (int j = 0; j < 32; ++j)
      q[j] = min(kTop, int(__fadd_rn(__fmul_rn(__fsub_rn(v(j), lo), inv), 0.5f)));
    st16(out, half_bits(dlt));
    st16(out + 2, half_bits(lo));
    if constexpr (F == RRQ_GGML_Q5_1) {
      put_high_bits(out + 4, q);
      put_nibbles(out + 8, q);
    } else {
      put_nibbles(out + 4, q);
    }
  } else if constexpr (F == RRQ_GGML_Q4_0 || F == RRQ_GGML_Q5_0) {
    constexpr float kHalf = F == RRQ_GGML_Q4_0 ? 8.f : 16.f;
    constexpr int kTop = F == RRQ_GGML_Q4_0 ? 15 : 31;
    float amax = 0.f, m = 0.f;  // m stays +0 for a block of zeros
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float a = fabsf(v(j));
      if (amax < a) { amax = a; m = v(j); }
    }
    const float dlt = __fmul_rn(m, -1.f / kHalf);  // m/−8 or m/−16: exact
    const float inv = dlt != 0.f ? __frcp_rn(dlt) : 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) q[j] = min(kTop, int(__fadd_rn(__fmul_rn(v(j), inv), kHalf + 0.5f)));
    st16(out, half_bits(dlt));
    if constexpr (F == RRQ_GGML_Q5_0) {
      put_high_bits(out + 2, q);
      put_nibbles(out + 6, q);
    } else {
      put_nibbles(out + 2, q);
    }
  } else {
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v(j)));
    const float dlt = __fdiv_rn(amax, 127.f);
    const float inv = dlt != 0.f ? __frcp_rn(dlt) : 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) q[j] = int(roundf(__fmul_rn(v(j), inv)));
    st16(out, half_bits(dlt));
#pragma unroll
    for (int j = 0; j < 32; j += 2) st16(out + 2 + j, uint32_t(q[j] & 255) | (uint32_t(q[j + 1] & 255) << 8));
  }
}

// One block's 32 values from its bytes, into shared row v.
template <int F>
__device__ __forceinline__ void decode_block(const uint8_t* in, float* v) {
  const float dlt = half_val(ld16(in));
  if constexpr (F == RRQ_GGML_Q8_0) {
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const uint32_t two = ld16(in + 2 + j);
      v[j] = float(int(int8_t(two & 255))) * dlt;
      v[j + 1] = float(int(int8_t(two >> 8))) * dlt;
    }
  } else {
    constexpr bool kMin = F == RRQ_GGML_Q4_1 || F == RRQ_GGML_Q5_1;
    constexpr bool kHigh = F == RRQ_GGML_Q5_0 || F == RRQ_GGML_Q5_1;
    const float lo = kMin ? half_val(ld16(in + 2)) : 0.f;
    const uint8_t* p = in + (kMin ? 4 : 2);
    uint32_t high = 0;
    if constexpr (kHigh) {
      high = ld16(p) | (ld16(p + 2) << 16);
      p += 4;
    }
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      const uint32_t two = ld16(p + j);  // bytes j, j+1
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t byte = (two >> (8 * u)) & 255;
        int q0 = int(byte & 15), q1 = int(byte >> 4);  // elements j+u and j+u+16
        if constexpr (kHigh) {
          q0 |= int((high >> (j + u)) & 1) << 4;
          q1 |= int((high >> (j + u + 16)) & 1) << 4;
        }
        if constexpr (kMin) {
          v[j + u] = fmaf(float(q0), dlt, lo);
          v[j + u + 16] = fmaf(float(q1), dlt, lo);
        } else {
          v[j + u] = float(q0 - 16) * dlt;
          v[j + u + 16] = float(q1 - 16) * dlt;
        }
      }
    }
  }
}

// Copy `bytes` (a multiple of 2) between a warp's staging buffer and global memory.
__device__ __forceinline__ void copy_out(uint8_t* __restrict__ dst, const uint8_t* src, int bytes, int lane) {
  const int full = bytes / 16;
  for (int i = lane; i < full; i += 32)
    reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(src)[i];
  for (int i = full * 8 + lane; i < bytes / 2; i += 32)
    reinterpret_cast<uint16_t*>(dst)[i] = reinterpret_cast<const uint16_t*>(src)[i];
}

__device__ __forceinline__ void copy_in(uint8_t* dst, const uint8_t* __restrict__ src, int bytes, int lane) {
  const int full = bytes / 16;
  for (int i = lane; i < full; i += 32)
    reinterpret_cast<uint4*>(dst)[i] = __ldcs(reinterpret_cast<const uint4*>(src) + i);
  for (int i = full * 8 + lane; i < bytes / 2; i += 32)
    reinterpret_cast<uint16_t*>(dst)[i] = reinterpret_cast<const uint16_t*>(src)[i];
}

template <typename T, int D, int F, bool ROT>
__global__ void __launch_bounds__(kBThreads) blocks_encode_kernel(const T* __restrict__ x, int64_t n,
                                                                  uint8_t* __restrict__ blocks,
                                                                  uint64_t seed, float inv_sqrt_d) {
  pdl_release();
  using Lay = BLayout<D>;
  constexpr int C = 64, G = Lay::G, P = Lay::P, SEC = Lay::SEC, VPW = Lay::VPW;
  constexpr int BY = BlockType<F>::kBytes, NB = D / 32, OB = NB * BY;
  static_assert(VPW * NB == kWarpBlocks, "a warp pass covers 64 blocks");
  __shared__ __align__(16) uint32_t smask[mask_words<T, D>()];
  __shared__ float vals[kBThreads / 32][kWarpBlocks * kRow];
  __shared__ __align__(16) uint8_t stage[kBThreads / 32][kWarpBlocks * BY];
  if constexpr (ROT) build_sign_mask<T, D>(smask, seed);
  __syncthreads();
  pdl_wait();  // from here on, global memory

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, h = lane & (G - 1), vsub = lane / G;
  float* wv = vals[warp];
  uint8_t* buf = stage[warp];
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
#pragma unroll
    for (int s = 0; s < SEC; ++s) {  // sector q = 16 values: block q/2, half q&1
      const int q = Lay::sector(s, h);
      float* row = wv + (vsub * NB + (q >> 1)) * kRow + (q & 1) * 16;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        row[2 * e] = w[8 * s + e].x;
        row[2 * e + 1] = w[8 * s + e].y;
      }
    }
    __syncwarp();
#pragma unroll
    for (int b = lane; b < kWarpBlocks; b += 32) {
      const float* row = wv + b * kRow;
      encode_block<F>([row](int j) { return row[j]; }, buf + b * BY);
    }
    __syncwarp();
    const int64_t nvalid = n - base < VPW ? n - base : VPW;
    copy_out(blocks + base * OB, buf, int(nvalid) * OB, lane);
    __syncwarp();
  }
}

template <typename T, int D, int F, bool ROT>
__global__ void __launch_bounds__(kBThreads) blocks_decode_kernel(const uint8_t* __restrict__ blocks,
                                                                  int64_t n, T* __restrict__ out,
                                                                  uint64_t seed, float inv_sqrt_d) {
  pdl_release();
  using Lay = BLayout<D>;
  constexpr int C = 64, G = Lay::G, P = Lay::P, SEC = Lay::SEC, VPW = Lay::VPW;
  constexpr int BY = BlockType<F>::kBytes, NB = D / 32, OB = NB * BY;
  __shared__ __align__(16) uint32_t smask[mask_words<T, D>()];
  __shared__ float vals[kBThreads / 32][kWarpBlocks * kRow];
  __shared__ __align__(16) uint8_t stage[kBThreads / 32][kWarpBlocks * BY];
  if constexpr (ROT) build_sign_mask<T, D>(smask, seed);
  __syncthreads();
  pdl_wait();  // from here on, global memory

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, h = lane & (G - 1), vsub = lane / G;
  float* wv = vals[warp];
  uint8_t* buf = stage[warp];
  const int64_t gwarp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t stride = ((int64_t(gridDim.x) * blockDim.x) >> 5) * VPW;
  int64_t vec = gwarp * VPW + vsub;
  for (int64_t base = gwarp * VPW; base < n; base += stride, vec += stride) {
    const int64_t nvalid = n - base < VPW ? n - base : VPW;
    copy_in(buf, blocks + base * OB, int(nvalid) * OB, lane);
    __syncwarp();
    // blocks of vectors past n decode stale staging bytes; those rows are not stored
#pragma unroll
    for (int b = lane; b < kWarpBlocks; b += 32) decode_block<F>(buf + b * BY, wv + b * kRow);
    __syncwarp();
    float2 w[P];
#pragma unroll
    for (int s = 0; s < SEC; ++s) {
      const int q = Lay::sector(s, h);
      const float* row = wv + (vsub * NB + (q >> 1)) * kRow + (q & 1) * 16;
#pragma unroll
      for (int e = 0; e < 8; ++e) w[8 * s + e] = make_float2(row[2 * e], row[2 * e + 1]);
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

// ------------------------------------------- one lane per vector (16-bit, d ≤ 128)
// Used for q4_0 and q8_0 with rotation (see enc_dtf).
// The batch encoder's structure: a warp takes 32 consecutive vectors, TMA boxes
// bring their rows into a 128-byte-swizzled stage (two per warp), each lane
// builds its vector's transform in registers (first butterfly from the 16-bit
// pairs, packed fp32 stages), scales it by 1/√d and quantises its d/32 blocks
// straight from the registers into its row of a per-warp output tile, which
// leaves in one bulk copy (two tiles per warp, alternating).
template <int D, int F> struct BlkBatch {
  static_assert(D == 64 || D == 128, "d = 64 or 128");
  static constexpr int ROW = D * 2;                      // input row bytes (16-bit)
  static constexpr int BOXES = ROW / 128;
  static constexpr int NS = 2;
  static constexpr int STAGE = 32 * ROW;
  static constexpr int OB = D / 32 * BlockType<F>::kBytes;  // block bytes per vector
  static constexpr int OTILE = (32 * OB + 127) / 128 * 128;
  static constexpr int WARP_BYTES = (NS * STAGE + 2 * OTILE + 1023) / 1024 * 1024;
  static constexpr int WARPS = 8;
  static constexpr int THREADS = WARPS * 32;
  static constexpr int MASK = D / 2 * 4;
  static constexpr int BARS = WARPS * NS * 8;
  static constexpr int HEAD = (MASK + BARS + 1023) / 1024 * 1024;
  static constexpr size_t total() { return 1024 + size_t(HEAD) + size_t(WARPS) * WARP_BYTES; }
  static_assert(total() <= 227 * 1024, "shared memory");
};

template <typename T, int D, int F>
__global__ void __launch_bounds__(BlkBatch<D, F>::THREADS, 1)
blocks_batch_kernel(const __grid_constant__ CUtensorMap xmap, int64_t n, uint8_t* __restrict__ blocks,
                    uint64_t seed, float inv_sqrt_d) {
  pdl_release();
  using SM = BlkBatch<D, F>;
  constexpr int P = D / 2, NS = SM::NS, NB = D / 32, BY = BlockType<F>::kBytes, OB = SM::OB;
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = dsm_raw + ((1024u - (smem_addr(dsm_raw) & 1023u)) & 1023u);
  uint32_t* smask = reinterpret_cast<uint32_t*>(dsm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(dsm + SM::MASK);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* wmem = dsm + SM::HEAD + warp * SM::WARP_BYTES;
  build_sign_mask<T, D>(smask, seed);
  if (lane == 0) {
    for (int st = 0; st < NS; ++st) mbarrier_init(smem_addr(&bars[warp * NS + st]), 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  pdl_wait();  // from here on, global memory

  const int64_t nb = (n + 31) >> 5;
  const int64_t tw = int64_t(gridDim.x) * SM::WARPS;
  const int64_t gw = int64_t(warp) * gridDim.x + blockIdx.x;  // warp-major: equal batches per SM
  const uint32_t bar0 = smem_addr(&bars[warp * NS]);
  const uint32_t stage0 = smem_addr(wmem);
  uint8_t* otile0 = wmem + NS * SM::STAGE;
  uint32_t pending = 0;
  auto issue = [&](int st, int64_t b) {
    if (b >= nb) return;
    if (lane == 0) {
      const uint32_t bar = bar0 + 8 * st;
      mbarrier_expect_tx(bar, SM::STAGE);
#pragma unroll
      for (int h = 0; h < SM::BOXES; ++h)
        tma_load_2d(stage0 + st * SM::STAGE + h * 4096, &xmap, h * 64, int(b << 5), bar);
    }
    pending |= 1u << st;
  };
#pragma unroll
  for (int st = 0; st < NS; ++st) issue(st, gw + st * tw);

  uint32_t parity = 0;
  int st = 0, ot = 0;
  bool failed = false;
  int64_t b = gw;
  for (; b < nb; b += tw) {
    if (!mbarrier_wait(bar0 + 8 * st, (parity >> st) & 1u)) {
      failed = true;
      break;
    }
    parity ^= 1u << st;
    pending &= ~(1u << st);
    const int64_t v0 = b << 5;
    const int nv = int(min(int64_t(32), n - v0));

    float2 w[P];
    const uint8_t* stage = wmem + st * SM::STAGE;
#pragma unroll
    for (int c = 0; c < SM::ROW / 16; ++c) {
      const uint4 r = *reinterpret_cast<const uint4*>(stage + (c >> 3) * 4096 + swz128(lane, c & 7));
      const uint4 m = reinterpret_cast<const uint4*>(smask)[c];
      w[4 * c + 0] = first_butterfly<T>(r.x ^ m.x);
      w[4 * c + 1] = first_butterfly<T>(r.y ^ m.y);
      w[4 * c + 2] = first_butterfly<T>(r.z ^ m.z);
      w[4 * c + 3] = first_butterfly<T>(r.w ^ m.w);
    }
    __syncwarp();  // every lane holds its row: the stage may be refilled
    fence_proxy_async_smem();
    issue(st, b + NS * tw);
#pragma unroll
    for (int mm = 1; mm < P; mm <<= 1) {
#pragma unroll
      for (int k = 0; k < P; ++k) {
        if ((k & mm) == 0) {
          const float2 a0 = w[k], a1 = w[k | mm];
          w[k] = add2(a0, a1);
          w[k | mm] = sub2(a0, a1);
        }
      }
    }
    const float2 s2 = make_float2(inv_sqrt_d, inv_sqrt_d);
#pragma unroll
    for (int k = 0; k < P; ++k) w[k] = mul2(w[k], s2);  // y = Πx

    uint8_t* tile = otile0 + ot * SM::OTILE;
    if (lane == 0) bulk_wait_read_1();  // the store from this tile two batches ago has read it
    __syncwarp();
    uint8_t* row = tile + lane * OB;
#pragma unroll
    for (int bb = 0; bb < NB; ++bb)
      encode_block<F>([&](int j) { return (j & 1) ? w[16 * bb + (j >> 1)].y : w[16 * bb + (j >> 1)].x; },
                      row + bb * BY);
    __syncwarp();
    const uint32_t bytes = uint32_t(nv) * OB;
    if (bytes % 16 == 0) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) bulk_store(blocks + v0 * OB, smem_addr(tile), bytes);
    } else {
      for (uint32_t i = lane; i < bytes / 2; i += 32)
        reinterpret_cast<uint16_t*>(blocks + v0 * OB)[i] = reinterpret_cast<const uint16_t*>(tile)[i];
    }
    ot ^= 1;
    st = (st + 1 == NS) ? 0 : st + 1;
  }
  if (failed) {
    // A stage never completed: give every block this warp still owns a NaN scale
    // (fp16 0x7E00 in its first two bytes), and wait (bounded) for the copies in flight.
    for (; b < nb; b += tw) {
      const int64_t v0 = b << 5;
      if (lane < n - v0)
        for (int bb = 0; bb < NB; ++bb) st16(blocks + (v0 + lane) * OB + bb * BY, 0x7E00u);
    }
#pragma unroll
    for (int s2i = 0; s2i < NS; ++s2i)
      if (pending & (1u << s2i)) mbarrier_wait(bar0 + 8 * s2i, (parity >> s2i) & 1u);
  }
  if (lane == 0) bulk_wait_all();
}

// cudaErrorNotSupported when no tensor map can be made (the caller then uses the tile kernel).
template <typename T, int D, int F>
cudaError_t launch_blocks_batch(const T* x, int64_t n, uint64_t seed, float isd, uint8_t* blocks,
                                cudaStream_t stream) {
  using SM = BlkBatch<D, F>;
  CUtensorMap xmap;
  if (!row_tensor_map(&xmap, x, n, D, 2, 32)) return cudaErrorNotSupported;
  auto k = blocks_batch_kernel<T, D, F>;
  constexpr size_t smem = SM::total();
  const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int64_t batches = (n + 31) / 32;
  const int grid = grid_for(reinterpret_cast<const void*>(k), SM::THREADS, smem,
                            (batches + SM::WARPS - 1) / SM::WARPS);
  return launch_pdl(k, grid, SM::THREADS, smem, stream, xmap, n, blocks, seed, isd);
}

template <typename T, int D, int F>
cudaError_t enc_dtf(const T* x, int64_t n, uint64_t seed, int rotate, float isd, uint8_t* blocks,
                    cudaStream_t stream) {
  // one lane per vector pays for q4_0 and q8_0 (measured 113.5 → 107 and 109 → 100 µs on
  // 1M vectors); the min/max types keep the tile kernel, whose 13 warps per SM hide
  // their longer per-block arithmetic better (118 vs 122, 126 vs 136 µs)
  if constexpr (Elem<T>::kBytes == 2 && D <= 128 && (F == RRQ_GGML_Q4_0 || F == RRQ_GGML_Q8_0)) {
    if (rotate) {
      const cudaError_t e = launch_blocks_batch<T, D, F>(x, n, seed, isd, blocks, stream);
      if (e != cudaErrorNotSupported) return e;
    }
  }
  constexpr int vpb = (kBThreads / 32) * BLayout<D>::VPW;
  const int64_t work = (n + vpb - 1) / vpb;
  auto k = rotate ? blocks_encode_kernel<T, D, F, true> : blocks_encode_kernel<T, D, F, false>;
  const int grid = grid_for(reinterpret_cast<const void*>(k), kBThreads, 0, work);
  return launch_pdl(k, grid, kBThreads, 0, stream, x, n, blocks, seed, isd);
}

template <typename T, int D, int F>
cudaError_t dec_dtf(const uint8_t* blocks, int64_t n, uint64_t seed, int rotate, float isd, T* out,
                    cudaStream_t stream) {
  constexpr int vpb = (kBThreads / 32) * BLayout<D>::VPW;
  const int64_t work = (n + vpb - 1) / vpb;
  auto k = rotate ? blocks_decode_kernel<T, D, F, true> : blocks_decode_kernel<T, D, F, false>;
  const int grid = grid_for(reinterpret_cast<const void*>(k), kBThreads, 0, work);
  return launch_pdl(k, grid, kBThreads, 0, stream, blocks, n, out, seed, isd);
}

template <typename T, int F>
cudaError_t enc_tf(const void* x, int64_t n, int d, uint64_t seed, int rotate, float isd, void* blocks,
                   cudaStream_t s) {
  const T* xx = static_cast<const T*>(x);
  uint8_t* b = static_cast<uint8_t*>(blocks);
  switch (d) {
    case 64: return enc_dtf<T, 64, F>(xx, n, seed, rotate, isd, b, s);
    case 128: return enc_dtf<T, 128, F>(xx, n, seed, rotate, isd, b, s);
    case 256: return enc_dtf<T, 256, F>(xx, n, seed, rotate, isd, b, s);
    case 512: return enc_dtf<T, 512, F>(xx, n, seed, rotate, isd, b, s);
  }
  return cudaErrorInvalidValue;
}

template <typename T, int F>
cudaError_t dec_tf(const void* blocks, int64_t n, int d, uint64_t seed, int rotate, float isd, void* out,
                   cudaStream_t s) {
  const uint8_t* b = static_cast<const uint8_t*>(blocks);
  T* o = static_cast<T*>(out);
  switch (d) {
    case 64: return dec_dtf<T, 64, F>(b, n, seed, rotate, isd, o, s);
    case 128: return dec_dtf<T, 128, F>(b, n, seed, rotate, isd, o, s);
    case 256: return dec_dtf<T, 256, F>(b, n, seed, rotate, isd, o, s);
    case 512: return dec_dtf<T, 512, F>(b, n, seed, rotate, isd, o, s);
  }
  return cudaErrorInvalidValue;
}

template <int F>
cudaError_t enc_f(const void* x, int dtype, int64_t n, int d, uint64_t seed, int rotate, float isd,
                  void* blocks, cudaStream_t s) {
  switch (dtype) {
    case RRQ_F16: return enc_tf<__half, F>(x, n, d, seed, rotate, isd, blocks, s);
    case RRQ_BF16: return enc_tf<__nv_bfloat16, F>(x, n, d, seed, rotate, isd, blocks, s);
    case RRQ_F32: return enc_tf<float, F>(x, n, d, seed, rotate, isd, blocks, s);
  }
  return cudaErrorInvalidValue;
}

template <int F>
cudaError_t dec_f(const void* blocks, int64_t n, int d, uint64_t seed, int rotate, float isd, void* out,
                  int out_dtype, cudaStream_t s) {
  switch (out_dtype) {
    case RRQ_F16: return dec_tf<__half, F>(blocks, n, d, seed, rotate, isd, out, s);
    case RRQ_BF16: return dec_tf<__nv_bfloat16, F>(blocks, n, d, seed, rotate, isd, out, s);
    case RRQ_F32: return dec_tf<float, F>(blocks, n, d, seed, rotate, isd, out, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_ggml_blocks(const void* x, int dtype, int64_t n, int d, uint64_t seed, int rotate,
                               int type, float inv_sqrt_d, void* blocks, cudaStream_t stream) {
  switch (type) {
    case RRQ_GGML_Q4_0: return enc_f<RRQ_GGML_Q4_0>(x, dtype, n, d, seed, rotate, inv_sqrt_d, blocks, stream);
    case RRQ_GGML_Q4_1: return enc_f<RRQ_GGML_Q4_1>(x, dtype, n, d, seed, rotate, inv_sqrt_d, blocks, stream);
    case RRQ_GGML_Q5_0: return enc_f<RRQ_GGML_Q5_0>(x, dtype, n, d, seed, rotate, inv_sqrt_d, blocks, stream);
    case RRQ_GGML_Q5_1: return enc_f<RRQ_GGML_Q5_1>(x, dtype, n, d, seed, rotate, inv_sqrt_d, blocks, stream);
    case RRQ_GGML_Q8_0: return enc_f<RRQ_GGML_Q8_0>(x, dtype, n, d, seed, rotate, inv_sqrt_d, blocks, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_ggml_blocks_decode(const void* blocks, int type, int64_t n, int d, uint64_t seed,
                                      int rotate, float inv_sqrt_d, void* out, int out_dtype,
                                      cudaStream_t stream) {
  switch (type) {
    case RRQ_GGML_Q4_1: return dec_f<RRQ_GGML_Q4_1>(blocks, n, d, seed, rotate, inv_sqrt_d, out, out_dtype, stream);
    case RRQ_GGML_Q5_0: return dec_f<RRQ_GGML_Q5_0>(blocks, n, d, seed, rotate, inv_sqrt_d, out, out_dtype, stream);
    case RRQ_GGML_Q5_1: return dec_f<RRQ_GGML_Q5_1>(blocks, n, d, seed, rotate, inv_sqrt_d, out, out_dtype, stream);
    case RRQ_GGML_Q8_0: return dec_f<RRQ_GGML_Q8_0>(blocks, n, d, seed, rotate, inv_sqrt_d, out, out_dtype, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rrq

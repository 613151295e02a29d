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
//   encode: 32 B loads (issued one grid-stride iteration ahead) → XOR rotation
//           signs on the raw elements → ν² = Σx² (packed fp32, group shuffle
//           sum) → unnormalised FWHT y' = H·D·x = √d·Πx → code_i =
//           #{k : y'_i > ν·τ_k}, the same decision as u_i = y'_i/ν > τ_k with
//           the scale folded into the thresholds once per vector → packing.
//   decode: codes (loaded one iteration ahead) → levels c[code] from shared
//           memory → FWHT → × ν/d → round to the output type → XOR rotation
//           signs → 32 B stores.
//   rotate: y = Πx (signs, FWHT, × 1/√d) or y = Πᵀx (FWHT, × 1/√d, signs).
//
// The kernels are issue-bound before they are HBM-bound, so the code search
// is split between the two arithmetic pipes: half of the coordinates take a
// branch-free compare/select binary search (integer/logic pipe), the other
// half an equivalent search built from saturating FMAs (FMA pipe).
#pragma once

#include <type_traits>

#include "rrq_device.cuh"

namespace rrq {

constexpr int kThreads = 128;
constexpr int kMinBlocks = 3;  // resident blocks per SM the register budget must allow

// Values per lane: 64 for the encoder (the raw input of the next iteration is
// held in registers too), 128 for the decoder (so a d ≤ 128 vector is one
// lane and the transform needs no shuffles).
template <int D> struct EncC { static constexpr int value = D < 64 ? D : 64; };
template <int D> struct DecC { static constexpr int value = D < 128 ? D : 128; };

// ------------------------------------------------------------- code search
// Number of thresholds t[0..2^K−2] (ascending) strictly below a, by a K-level
// branch-free binary search: each level's predicate selects the next threshold.
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

// Code of one rotated value y' for an exactly symmetric codebook with 2^B
// levels; T[j] = ν·τ_{L/2+j} (the positive thresholds; τ_{L/2−1} = 0):
//   y' > 0:  code = L/2 + #{j : |y'| > T_j}
//   y' ≤ 0:  code = L/2 − 1 − #{j : |y'| > T_j}
// The second line takes a tie |y'| = T_j to the upper code where the exact
// rule (strict u > τ) takes the lower one; such a value lies on a threshold,
// inside the band where codes may differ.  y' = ±0 gives L/2 − 1 exactly.
// With m' = (L/2 − 1) − m = m ^ (L/2 − 1): code = pos ? m' ^ (L − 1) : m'.
template <int B>
__device__ __forceinline__ uint32_t code_sym(float y, const float (&T)[(1 << (B - 1)) > 1 ? (1 << (B - 1)) - 1 : 1]) {
  constexpr uint32_t L = 1u << B;
  const uint32_t mm = count_below<B - 1>(fabsf(y), T) ^ (L / 2 - 1);
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

// The same 4-bit symmetric search on the FMA pipe.  With big = 2^k chosen so
// that ulp(T_0)·big = 1, every scaled threshold tb_j = T_j·big is an integer
// and a·big is an integer whenever a ≥ T_0, so sat(a·big − tb) is exactly 1
// when a > T and exactly 0 otherwise (a < T_0 gives a negative argument).
// Thresholds of later levels are picked by arithmetic on the 0/1 results
// (integer-valued, hence exact to within an ulp of the scaled threshold —
// far inside the boundary band).
struct Sym4 {
  float t[7];   // T_j, for the compare/select path
  float big;    // power of two, ulp(T_0)·big = 1
  float tb[7];  // T_j·big
  float d51, c1, c2, c3;

  __device__ __forceinline__ void init(float ns, const QuantParams& p) {
#pragma unroll
    for (int j = 0; j < 7; ++j) t[j] = ns * p.thr[8 + j];
    const uint32_t be = (__float_as_uint(t[0]) >> 23) & 0xffu;
    const int bb = min(254, max(1, 277 - int(be)));
    big = __uint_as_float(uint32_t(bb) << 23);
#pragma unroll
    for (int j = 0; j < 7; ++j) tb[j] = t[j] * big;
    d51 = tb[5] - tb[1];
    c1 = tb[2] - tb[0];
    c2 = tb[4] - tb[0];
    c3 = (tb[6] - tb[4]) - c1;
  }

  // code as an exact small integer in a float
  __device__ __forceinline__ float code_fma(float y) const {
    const float a = fabsf(y);
    const float p2 = __saturatef(fmaf(a, big, -tb[3]));
    const float tb1 = fmaf(p2, d51, tb[1]);
    const float p1 = __saturatef(fmaf(a, big, -tb1));
    const float tb0 = fmaf(p1, fmaf(p2, c3, c1), fmaf(p2, c2, tb[0]));
    const float p0 = __saturatef(fmaf(a, big, -tb0));
    const float m = fmaf(p2, 4.f, fmaf(p1, 2.f, p0));
    const float ps = y > 0.f ? 1.f : 0.f;
    return fmaf(ps, fmaf(m, 2.f, 1.f), 7.f - m);  // pos: 8 + m, else 7 − m
  }
};

// 16 codes of one sector (4 bits each) -> two words; coordinates 0..3 and
// 8..11 take the compare/select path, 4..7 and 12..15 the FMA path.
__device__ __forceinline__ uint2 sector_codes4(const float2* w, const Sym4& k) {
  uint32_t out[2];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const float2* v = w + 4 * half;
    const uint32_t lo = code_sym<4>(v[0].x, k.t) | (code_sym<4>(v[0].y, k.t) << 4) |
                        (code_sym<4>(v[1].x, k.t) << 8) | (code_sym<4>(v[1].y, k.t) << 12);
    float f = k.code_fma(v[3].y);
    f = fmaf(f, 16.f, k.code_fma(v[3].x));
    f = fmaf(f, 16.f, k.code_fma(v[2].y));
    f = fmaf(f, 16.f, k.code_fma(v[2].x));  // exact integer < 2^16
    const uint32_t hi = __float_as_uint(f + 8388608.f);  // low 16 bits = f
    out[half] = __byte_perm(lo, hi, 0x5410);
  }
  return make_uint2(out[0], out[1]);
}

// Number of positive thresholds of a symmetric codebook at B bits (≥ 1 slot).
template <int B> constexpr int npos() { return (1 << (B - 1)) > 1 ? (1 << (B - 1)) - 1 : 1; }

// 16 codes of one sector at B bits (B·16 bits, little endian) on the
// compare/select path.
template <int B, bool SYM>
__device__ __forceinline__ uint64_t sector_codes(const float2* w, const float (&tp)[npos<B>()],
                                                 const float (&tg)[(1 << B) - 1]) {
  uint64_t acc = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t c0, c1;
    if constexpr (SYM) {
      c0 = code_sym<B>(w[j].x, tp);
      c1 = code_sym<B>(w[j].y, tp);
    } else {
      c0 = code_generic<1 << B>(w[j].x, tg);
      c1 = code_generic<1 << B>(w[j].y, tg);
    }
    acc |= uint64_t(c0 | (c1 << B)) << (2 * j * B);
  }
  return acc;
}

// ------------------------------------------------------- packed code rows
// A lane's code bits: for G = 1 the whole row (contiguous); otherwise only the
// lane's sectors, each 2B bytes at byte offset q·2B of the row.
template <int NB>  // NB = bytes
__device__ __forceinline__ void store_bytes(uint8_t* __restrict__ p, const uint32_t* words) {
  if constexpr (NB % 32 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 32; ++i) {
      W8 v;
#pragma unroll
      for (int j = 0; j < 8; ++j) v.w[j] = words[i * 8 + j];
      st256(p + 32 * i, v);
    }
  } else if constexpr (NB % 16 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 16; ++i)
      reinterpret_cast<uint4*>(p)[i] =
          make_uint4(words[4 * i], words[4 * i + 1], words[4 * i + 2], words[4 * i + 3]);
  } else {
    static_assert(NB % 8 == 0, "code rows are a multiple of 8 bytes");
#pragma unroll
    for (int i = 0; i < NB / 8; ++i)
      reinterpret_cast<uint2*>(p)[i] = make_uint2(words[2 * i], words[2 * i + 1]);
  }
}

template <int NB>
__device__ __forceinline__ void load_bytes(const uint8_t* __restrict__ p, bool valid, uint32_t* words) {
  if constexpr (NB % 32 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 32; ++i) {
      W8 v;
      if (valid) {
        v = ld256(p + 32 * i);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v.w[j] = 0u;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) words[i * 8 + j] = v.w[j];
    }
  } else if constexpr (NB % 16 == 0) {
#pragma unroll
    for (int i = 0; i < NB / 16; ++i) {
      const uint4 v = valid ? __ldcs(reinterpret_cast<const uint4*>(p) + i) : make_uint4(0, 0, 0, 0);
      words[4 * i] = v.x; words[4 * i + 1] = v.y; words[4 * i + 2] = v.z; words[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < NB / 8; ++i) {
      const uint2 v = valid ? __ldcs(reinterpret_cast<const uint2*>(p) + i) : make_uint2(0, 0);
      words[2 * i] = v.x; words[2 * i + 1] = v.y;
    }
  }
}

// One sector (2B bytes) of a row at byte offset q·2B (G > 1 layouts).
template <int B>
__device__ __forceinline__ void store_sector_codes(uint8_t* __restrict__ row, int q, uint64_t v) {
  if constexpr (B == 4) {
    reinterpret_cast<uint2*>(row)[q] = make_uint2(uint32_t(v), uint32_t(v >> 32));
  } else if constexpr (B == 2) {
    reinterpret_cast<uint32_t*>(row)[q] = uint32_t(v);
  } else if constexpr (B == 1) {
    reinterpret_cast<uint16_t*>(row)[q] = uint16_t(v);
  } else {
    uint16_t* p = reinterpret_cast<uint16_t*>(row) + 3 * q;
    p[0] = uint16_t(v); p[1] = uint16_t(v >> 16); p[2] = uint16_t(v >> 32);
  }
}

template <int B>
__device__ __forceinline__ uint64_t load_sector_codes(const uint8_t* __restrict__ row, int q) {
  if constexpr (B == 4) {
    const uint2 v = __ldcs(reinterpret_cast<const uint2*>(row) + q);
    return uint64_t(v.x) | (uint64_t(v.y) << 32);
  } else if constexpr (B == 2) {
    return __ldcs(reinterpret_cast<const uint32_t*>(row) + q);
  } else if constexpr (B == 1) {
    return __ldcs(reinterpret_cast<const uint16_t*>(row) + q);
  } else {
    const uint16_t* p = reinterpret_cast<const uint16_t*>(row) + 3 * q;
    return uint64_t(__ldcs(p)) | (uint64_t(__ldcs(p + 1)) << 16) | (uint64_t(__ldcs(p + 2)) << 32);
  }
}

// ------------------------------------------------------------------ encode
template <typename T, int D, int B, bool SYM>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
encode_kernel(const T* __restrict__ x, int64_t n, uint8_t* __restrict__ codes,
              float* __restrict__ norms, const QuantParams p) {
  pdl_release();
  constexpr int C = EncC<D>::value;
  using Lay = Layout<D, C>;
  constexpr int G = Lay::G, P = Lay::P, SEC = Lay::SEC, VPW = Lay::VPW;
  constexpr int L = 1 << B;
  constexpr int CB = D * B / 8;  // code bytes per vector
  __shared__ __align__(16) uint32_t smask[mask_words<T, D>()];
  build_sign_mask<T, D>(smask, p.seed);
  __syncthreads();
  pdl_wait();  // from here on, global memory

  const int lane = threadIdx.x & 31, h = lane & (G - 1), vsub = lane / G;
  const int64_t gwarp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t stride = ((int64_t(gridDim.x) * blockDim.x) >> 5) * VPW;

  int64_t vec = gwarp * VPW + vsub;
  RawVec<T, D, C> nxt;
  nxt.load(x + vec * D, vec < n, h);
  for (int64_t base = gwarp * VPW; base < n; base += stride, vec += stride) {
    const bool valid = vec < n;
    float2 w[P];
    raw_to_pairs<T, D, C, true>(nxt, h, smask, w);
    nxt.load(x + (vec + stride) * D, vec + stride < n, h);  // next iteration, in flight now

    float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < P; ++k) ss2 = fma2(w[k], w[k], ss2);
    const float ss = group_sum<G>(ss2.x + ss2.y);  // ‖x‖₂²
    const float nu = sqrtf(ss);
    fwht2<D, C>(w, h);
    float stored = nu;
    if constexpr (B == 1) {
      if (p.norm_mode != 0) {  // DRIVE scale × √d (QuantParams::norm_mode)
        float2 l1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < P; ++k) l1 = add2(l1, make_float2(fabsf(w[k].x), fabsf(w[k].y)));
        const float s1 = group_sum<G>(l1.x + l1.y);  // ‖y'‖₁
        stored = p.norm_mode == 1 ? s1 * p.inv_d
                                  : (s1 > 0.f ? __fdiv_rn(ss * float(D), s1) : 0.f);
      }
    }
    const float ns = nu > 0.f ? nu : 1.f;  // ν = 0: y' = 0, u = 0 against the plain thresholds
    uint8_t* crow = codes + vec * CB;

    uint64_t sec[SEC];
    if constexpr (SYM && B == 4) {
      Sym4 k4;
      k4.init(ns, p);
#pragma unroll
      for (int s = 0; s < SEC; ++s) {
        const uint2 v = sector_codes4(&w[s * 8], k4);
        sec[s] = uint64_t(v.x) | (uint64_t(v.y) << 32);
      }
    } else {
      float tp[npos<B>()] = {};
      float tg[L - 1] = {};
      if constexpr (SYM) {
#pragma unroll
        for (int j = 0; j < L / 2 - 1; ++j) tp[j] = ns * p.thr[L / 2 + j];
      } else {
#pragma unroll
        for (int k = 0; k < L - 1; ++k) tg[k] = ns * p.thr[k];
      }
#pragma unroll
      for (int s = 0; s < SEC; ++s) sec[s] = sector_codes<B, SYM>(&w[s * 8], tp, tg);
    }
    if constexpr (G == 1) {
      uint32_t words[CB / 4];
#pragma unroll
      for (int i = 0; i < CB / 4; ++i) words[i] = 0u;
#pragma unroll
      for (int s = 0; s < SEC; ++s) {
        // sector s at bit s·16B
        if constexpr (B == 4) { words[2 * s] = uint32_t(sec[s]); words[2 * s + 1] = uint32_t(sec[s] >> 32); }
        else if constexpr (B == 2) { words[s] = uint32_t(sec[s]); }
        else if constexpr (B == 1) { words[s / 2] |= uint32_t(sec[s]) << (16 * (s & 1)); }
        else {  // B == 3: 48 bits at bit 48·s
          const int pos = 48 * s, wi = pos / 32, off = pos % 32;
          words[wi] |= uint32_t(sec[s] << off);
          words[wi + 1] |= uint32_t(sec[s] >> (32 - off));
          if (off > 16) words[wi + 2] |= uint32_t(sec[s] >> (64 - off));
        }
      }
      if (valid) store_bytes<CB>(crow, words);
    } else {
#pragma unroll
      for (int s = 0; s < SEC; ++s)
        if (valid) store_sector_codes<B>(crow, Lay::sector(s, h), sec[s]);
    }
    if (valid && h == 0) norms[vec] = stored;
  }
}

// ------------------------------------------------------------------ decode
// d ≤ 128: one lane per vector, batches of 32 consecutive vectors per warp.
// Global traffic moves in whole lines while the arithmetic stays per lane:
//  * codes and norms of batch k+NS−1 are copied (cp.async, 8 vectors = 512
//    contiguous bytes per instruction) into a per-warp ring of padded rows
//    (80 B for d·b/8 = 64: conflict-free 128-bit reads by the owning lane);
//  * each lane writes its reconstructed row into a padded shared tile
//    (row stride ≡ 16 mod 128 B: conflict-free) and issues a bulk (TMA) copy
//    of that row to global memory.
// d > 128: several lanes per vector (shuffle stages); codes read straight
// from global memory, 32-byte stores.
constexpr int kDecodeStages = 3;

// 4-bit codes and fp16 outputs: look up a byte (two codes) at once.  Entry
// e = lo | hi << 4 holds (c_lo + c_hi, c_lo − c_hi) in fp16 — the first
// butterfly of the transform already applied.  The fp16 rounding (2^-12
// relative) is below the fp16 output's own rounding; bf16 and fp32 outputs use
// exact fp32 levels.  The table is replicated per lane (word e·32 + lane), so
// every lane reads its own bank.
template <typename T, int B>
constexpr bool use_pair_table() { return B == 4 && std::is_same<T, __half>::value; }
constexpr int kPairTableWords = 256 * 32;

template <typename T, int D, int B> struct DecodeSmem {
  static constexpr int CB = D * B / 8;
  static constexpr int CBP = (CB + 15) / 16 * 16;       // codes, padded
  static constexpr int RR = CBP + 16;                    // ring row: codes | norm | pad
  static constexpr int UNIT = (CB % 16 == 0) ? 16 : 8;  // cp.async unit
  static constexpr int UPV = CB / UNIT;
  static constexpr int ROW = D * Elem<T>::kBytes;        // output row bytes
  static constexpr int TROW = ROW + 16;                  // padded tile row
  static constexpr int RING = kDecodeStages * 32 * RR;
  static constexpr int WARP = RING + 32 * TROW;          // per warp
  static constexpr bool ONE_LANE = DecC<D>::value == D;
  static constexpr int TABLE = use_pair_table<T, B>() ? kPairTableWords * 4 : 0;
  // One block per SM holding as many warps as shared memory allows (≤ 12,
  // which the 168-register budget also allows); the warps share one table.
  static constexpr int kMaxBlockSmem = 227 * 1024;
  static constexpr int WARPS_BY_SMEM = ONE_LANE ? (kMaxBlockSmem - TABLE) / WARP : 12;
  static constexpr int WARPS = WARPS_BY_SMEM < 12 ? WARPS_BY_SMEM : 12;
  static constexpr int THREADS = WARPS * 32;
  static constexpr size_t total() { return (ONE_LANE ? size_t(WARPS) * WARP : 0) + TABLE; }
};

template <typename T, int D, int B>
__global__ void __launch_bounds__(DecodeSmem<T, D, B>::THREADS, 1)
decode_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ norms, int64_t n,
              T* __restrict__ out, const QuantParams p) {
  pdl_release();
  constexpr int C = DecC<D>::value;
  using Lay = Layout<D, C>;
  using SM = DecodeSmem<T, D, B>;
  constexpr int G = Lay::G, P = Lay::P, SEC = Lay::SEC, VPW = Lay::VPW;
  constexpr int L = 1 << B;
  constexpr int CB = SM::CB;
  constexpr int NW = (G == 1) ? CB / 4 : SEC * 2;  // code words held per lane
  constexpr int NS = kDecodeStages;
  constexpr bool PAIR = use_pair_table<T, B>();
  __shared__ __align__(16) uint32_t smask[mask_words<T, D>()];
  __shared__ float slev[L];
  extern __shared__ __align__(16) uint8_t dyn_smem[];
  uint32_t* ptab = reinterpret_cast<uint32_t*>(dyn_smem);  // pair table (PAIR only)
  uint8_t* warp_mem = dyn_smem + (PAIR ? kPairTableWords * 4 : 0) + (threadIdx.x >> 5) * SM::WARP;
  build_sign_mask<T, D>(smask, p.seed);
  if (threadIdx.x < L) slev[threadIdx.x] = p.levels[threadIdx.x];
  if constexpr (PAIR) {
    for (int i = threadIdx.x; i < kPairTableWords; i += blockDim.x) {
      const int e = i >> 5;
      const float lo = p.levels[e & 15], hi = p.levels[e >> 4];
      const __half2 v = __floats2half2_rn(lo + hi, lo - hi);
      ptab[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
  }
  __syncthreads();
  pdl_wait();  // from here on, global memory

  const int lane = threadIdx.x & 31, h = lane & (G - 1), vsub = lane / G;
  const int64_t gwarp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t stride = ((int64_t(gridDim.x) * blockDim.x) >> 5) * VPW;
  const uint32_t* lane_tab = ptab + lane;

  // codes -> levels (in pairs) -> transform; w holds the lane's values
  auto expand = [&](const uint32_t* cw, float2 (&w)[P]) {
#pragma unroll
    for (int s = 0; s < SEC; ++s) {
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        if constexpr (PAIR) {
          const int bytepos = G == 1 ? (s * 16 + e) * 4 : 64 * s + e * 4;
          const uint32_t pv = lane_tab[get_bits(cw, bytepos, 8) << 5];
          w[s * 8 + e / 2] = __half22float2(*reinterpret_cast<const __half2*>(&pv));
        } else {
          uint32_t c0, c1;
          if constexpr (G == 1) {
            c0 = get_bits(cw, (s * 16 + e) * B, B);
            c1 = get_bits(cw, (s * 16 + e + 1) * B, B);
          } else {
            c0 = get_bits(cw + 2 * s, e * B, B);
            c1 = get_bits(cw + 2 * s, (e + 1) * B, B);
          }
          w[s * 8 + e / 2] = make_float2(slev[c0], slev[c1]);
        }
      }
    }
    fwht2<D, C, PAIR>(w, h);
  };

  if constexpr (G == 1) {
    uint8_t* ring = warp_mem;
    uint8_t* tile_row = warp_mem + SM::RING + lane * SM::TROW;
    // warp-cooperative copy of batch `bvec` (32 vectors from bvec) into stage
    auto issue = [&](int stage, int64_t bvec) {
      uint8_t* st = ring + stage * 32 * SM::RR;
#pragma unroll
      for (int i = 0; i < SM::UPV; ++i) {
        const int t = lane + 32 * i;  // unit t of the batch
        const int v = t / SM::UPV, u = t % SM::UPV;
        const bool ok = bvec + v < n;
        const uint8_t* src = codes + (ok ? (bvec + v) * CB + u * SM::UNIT : 0);
        const uint32_t dst = smem_addr(st + v * SM::RR + u * SM::UNIT);
        if constexpr (SM::UNIT == 16) cp_async16(dst, src, ok ? 16 : 0);
        else cp_async8(dst, src, ok ? 8 : 0);
      }
      const bool ok = bvec + lane < n;
      cp_async4(smem_addr(st + lane * SM::RR + SM::CBP), norms + (ok ? bvec + lane : 0), ok ? 4 : 0);
    };
    const int64_t wbase = gwarp * 32;
#pragma unroll
    for (int k = 0; k < NS - 1; ++k) {
      issue(k, wbase + k * stride);
      cp_async_commit();
    }
    int stage = 0;
    for (int64_t base = wbase; base < n; base += stride) {
      cp_async_wait<NS - 2>();
      __syncwarp();
      const uint8_t* row = ring + stage * 32 * SM::RR + lane * SM::RR;
      uint32_t cw[NW];
#pragma unroll
      for (int i = 0; i < CB / 4; i += (SM::UNIT / 4)) {
        if constexpr (SM::UNIT == 16) {
          const uint4 v = *reinterpret_cast<const uint4*>(row + 4 * i);
          cw[i] = v.x; cw[i + 1] = v.y; cw[i + 2] = v.z; cw[i + 3] = v.w;
        } else {
          const uint2 v = *reinterpret_cast<const uint2*>(row + 4 * i);
          cw[i] = v.x; cw[i + 1] = v.y;
        }
      }
      const float nu = *reinterpret_cast<const float*>(row + SM::CBP);
      __syncwarp();  // every lane has read this stage before it is refilled
      issue((stage + NS - 1) % NS, base + (NS - 1) * stride);
      cp_async_commit();
      stage = (stage + 1) % NS;

      float2 w[P];
      expand(cw, w);
      const int64_t vec = base + lane;
      bulk_wait_read_all();  // the previous bulk store has read this lane's tile row
      store_pairs_smem<T, D>(tile_row, smask, w, nu * p.inv_d);
      fence_proxy_async_smem();
      if (vec < n) bulk_store(out + vec * D, smem_addr(tile_row), SM::ROW);
    }
    cp_async_wait<0>();
    bulk_wait_all();
  } else {
    int64_t vec = gwarp * VPW + vsub;
    for (int64_t base = gwarp * VPW; base < n; base += stride, vec += stride) {
      const bool ok = vec < n;
      uint32_t cw[NW];
      const uint8_t* crow = codes + (ok ? vec : 0) * CB;
#pragma unroll
      for (int s = 0; s < SEC; ++s) {
        const uint64_t c = ok ? load_sector_codes<B>(crow, Lay::sector(s, h)) : 0ull;
        cw[2 * s] = uint32_t(c);
        cw[2 * s + 1] = uint32_t(c >> 32);
      }
      const float nu = ok ? __ldcs(norms + vec) : 0.f;
      float2 w[P];
      expand(cw, w);
      store_pairs<T, D, C, true>(out + vec * D, ok, h, smask, w, nu * p.inv_d);
    }
  }
}

// ------------------------------------------------------------------ rotate
template <typename T, int D, bool INV>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
rotate_kernel(const T* __restrict__ x, int64_t n, float* __restrict__ y, uint64_t seed,
              float inv_sqrt_d) {
  pdl_release();
  constexpr int C = EncC<D>::value;
  using Lay = Layout<D, C>;
  constexpr int G = Lay::G, P = Lay::P, VPW = Lay::VPW;
  __shared__ __align__(16) uint32_t smask_in[mask_words<T, D>()];
  __shared__ __align__(16) uint32_t smask_out[mask_words<float, D>()];
  if constexpr (!INV) build_sign_mask<T, D>(smask_in, seed);
  else build_sign_mask<float, D>(smask_out, seed);
  __syncthreads();
  pdl_wait();  // from here on, global memory

  const int lane = threadIdx.x & 31, h = lane & (G - 1), vsub = lane / G;
  const int64_t gwarp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t stride = ((int64_t(gridDim.x) * blockDim.x) >> 5) * VPW;
  int64_t vec = gwarp * VPW + vsub;
  RawVec<T, D, C> nxt;
  nxt.load(x + vec * D, vec < n, h);
  for (int64_t base = gwarp * VPW; base < n; base += stride, vec += stride) {
    const bool valid = vec < n;
    float2 w[P];
    raw_to_pairs<T, D, C, !INV>(nxt, h, smask_in, w);
    nxt.load(x + (vec + stride) * D, vec + stride < n, h);
    fwht2<D, C>(w, h);
    store_pairs<float, D, C, INV>(y + vec * D, valid, h, smask_out, w, inv_sqrt_d);
  }
}

// ---------------------------------------------------------------- launchers
template <int C_>
constexpr int vectors_per_block(int d) { return (kThreads / 32) * (32 / (d / (d < C_ ? d : C_))); }

// One-lane-per-vector encoder for d ≤ 128 and 16-bit inputs (batch_kernels.cuh).
template <typename T, int D, int B>
cudaError_t launch_encode_batch(const T* x, int64_t n, const QuantParams& p, uint8_t* codes,
                                float* norms, cudaStream_t stream);

template <typename T, int D, int B>
cudaError_t encode_db(const T* x, int64_t n, const QuantParams& p, uint8_t* codes, float* norms,
                      cudaStream_t stream) {
  if constexpr (Elem<T>::kBytes == 2 && D <= 128) {
    if (p.cell.cells > 0 || p.norm_mode != 0) {  // DRIVE codes need no table
      const cudaError_t e = launch_encode_batch<T, D, B>(x, n, p, codes, norms, stream);
      if (e != cudaErrorNotSupported) return e;
    }
  }
  constexpr int vpb = vectors_per_block<EncC<D>::value>(D);
  const int64_t work = (n + vpb - 1) / vpb;
  if (p.sym) {
    auto k = encode_kernel<T, D, B, true>;
    const int grid = grid_for(reinterpret_cast<const void*>(k), kThreads, 0, work);
    const cudaError_t e = launch_pdl(k, grid, kThreads, 0, stream, x, n, codes, norms, p);
    if (e != cudaSuccess) return e;
  } else {
    auto k = encode_kernel<T, D, B, false>;
    const int grid = grid_for(reinterpret_cast<const void*>(k), kThreads, 0, work);
    const cudaError_t e = launch_pdl(k, grid, kThreads, 0, stream, x, n, codes, norms, p);
    if (e != cudaSuccess) return e;
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

// One-lane-per-vector decoder for 4-bit codes and d ≤ 128 (batch_kernels.cuh).
template <typename T, int D>
cudaError_t launch_decode_batch(const uint8_t* codes, const float* norms, int64_t n,
                                const QuantParams& p, T* out, cudaStream_t stream);

template <typename T, int D, int B>
cudaError_t decode_db(const uint8_t* codes, const float* norms, int64_t n, const QuantParams& p,
                      T* out, cudaStream_t stream) {
  if constexpr (B == 4 && D <= 128) {
    const cudaError_t e = launch_decode_batch<T, D>(codes, norms, n, p, out, stream);
    if (e != cudaErrorNotSupported) return e;
  }
  using SM = DecodeSmem<T, D, B>;
  constexpr int vpb = SM::WARPS * (32 / (D / DecC<D>::value));
  const int64_t work = (n + vpb - 1) / vpb;
  auto k = decode_kernel<T, D, B>;
  constexpr size_t smem = DecodeSmem<T, D, B>::total();
  if constexpr (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
  }
  const int grid = grid_for(reinterpret_cast<const void*>(k), SM::THREADS, smem, work);
  const cudaError_t e = launch_pdl(k, grid, SM::THREADS, smem, stream, codes, norms, n, out, p);
  if (e != cudaSuccess) return e;
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
  constexpr int vpb = vectors_per_block<EncC<D>::value>(D);
  const int64_t work = (n + vpb - 1) / vpb;
  if (inverse) {
    auto k = rotate_kernel<T, D, true>;
    const int grid = grid_for(reinterpret_cast<const void*>(k), kThreads, 0, work);
    const cudaError_t e = launch_pdl(k, grid, kThreads, 0, stream, x, n, y, seed, inv_sqrt_d);
    if (e != cudaSuccess) return e;
  } else {
    auto k = rotate_kernel<T, D, false>;
    const int grid = grid_for(reinterpret_cast<const void*>(k), kThreads, 0, work);
    const cudaError_t e = launch_pdl(k, grid, kThreads, 0, stream, x, n, y, seed, inv_sqrt_d);
    if (e != cudaSuccess) return e;
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

// batch_kernels.cuh — one-lane-per-vector encoder for d ≤ 128 and 16-bit
// inputs (the KV-cache case).
//
// "Random-rotation quantization" page: scheme steps 1–2 (rotate by Π, then
// quantise every rotated coordinate with one fixed codebook); "History", EDEN
// bullet (normalise to ≈N(0,1), Lloyd–Max codebook); TurboQuant bullet (one
// constant scale per vector).
//
// Work unit: a batch of 32 consecutive vectors, one per lane of a warp, so the
// whole transform runs in one lane's registers with no shuffles.
//  * Staging.  One lane per warp moves a whole batch (32 rows, contiguous in
//    global memory) with TMA tensor copies of 32 × 128-byte boxes, completing
//    on the stage's mbarrier; two stages per warp (an optional L2 prefetch of
//    later batches measured slower, and is off).  The boxes land 128-byte swizzled (tensor_map.h),
//    so each lane reads its own row in 16-byte chunks without bank conflicts,
//    and rows past the end of the array arrive as zeros.  (A bulk copy per
//    lane would do the same work, but bulk and tensor copies take warp-uniform
//    operands: 32 different addresses cost a 32-step issue loop.)
//  * Arithmetic.  Rotation signs are an XOR of the element sign bits; the
//    first butterfly is a mixed-precision add/sub straight from the 16-bit
//    elements; the remaining log2(d) − 1 butterfly stages run on packed fp32
//    pairs; ν² = Σ x² comes from the first-stage outputs
//    ((a+b)² + (a−b)² = 2a² + 2b²).
//  * Code search (CellTable): s = sat(y'·A/ν + 1/2); the cell index
//    round(s·N) selects, from a lane-replicated table, the code of the cell's
//    lower end and the one threshold inside it; code = lo + (s > thr).  This is
//    exactly #{k : s > t_k}, the rule code = #{k : u > τ_k} evaluated on
//    s = u·A + 1/2.
//  * Output.  Codes go to a per-warp shared tile laid out as in global memory
//    and leave in one bulk store per batch; norms are plain coalesced stores.
#pragma once

#include "quant_kernels.cuh"
#include "tensor_map.h"
#include "mma_encode.cuh"
#include "mma_decode.cuh"
#include "tc_encode.cuh"

namespace rrq {

// (x_lo + x_hi, x_lo − x_hi) in fp32 from one word of two 16-bit elements:
// each result is the exact sum rounded once to fp32.
template <typename T> __device__ __forceinline__ float2 first_butterfly(uint32_t w);
// The result is produced as one 64-bit register pair, the operand form of the
// packed fp32 instructions that follow.
template <> __device__ __forceinline__ float2 first_butterfly<__half>(uint32_t w) {
  const float hi = __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
  uint64_t r;
  asm("{\n\t.reg .b16 l, h;\n\t.reg .f32 s, d;\n\tmov.b32 {l, h}, %1;\n\t"
      "add.rn.f32.f16 s, l, %2;\n\tsub.rn.f32.f16 d, l, %2;\n\tmov.b64 %0, {s, d};\n\t}"
      : "=l"(r)
      : "r"(w), "f"(hi));
  return *reinterpret_cast<float2*>(&r);
}
template <> __device__ __forceinline__ float2 first_butterfly<__nv_bfloat16>(uint32_t w) {
  const float hi = __uint_as_float(w & 0xffff0000u);
  uint64_t r;
  asm("{\n\t.reg .b16 l, h;\n\t.reg .f32 s, d;\n\tmov.b32 {l, h}, %1;\n\t"
      "add.rn.f32.bf16 s, l, %2;\n\tsub.rn.f32.bf16 d, l, %2;\n\tmov.b64 %0, {s, d};\n\t}"
      : "=l"(r)
      : "r"(w), "f"(hi));
  return *reinterpret_cast<float2*>(&r);
}


// OR code c (B bits) of coordinate i into a little-endian word array.
template <int B>
__device__ __forceinline__ void put_code(uint32_t* words, int i, uint32_t c) {
  const int bit = i * B, wi = bit >> 5, off = bit & 31;
  words[wi] |= c << off;
  if (off + B > 32) words[wi + 1] |= c >> (32 - off);
}

template <typename T, int D, int B, int WARPS_ = 8, int NS_ = 2, int PF_ = 0> struct EncBatch {
  static_assert(D <= 128 && D % 64 == 0 && Elem<T>::kBytes == 2,
                "batch encoder: d = 64 or 128, 16-bit inputs");
  static constexpr int ROW = D * 2;            // input row bytes
  static constexpr int BOXES = ROW / 128;      // 128-byte boxes per row
  static constexpr int NS = NS_;               // shared-memory stages per warp
  static constexpr int PF = PF_;               // further batches prefetched into L2 (measured: none is best)
  static constexpr int CB = D * B / 8;         // code bytes per vector
  static constexpr int STAGE = 32 * ROW;       // BOXES boxes of 32 × 128 bytes (1024-aligned)
  static constexpr int CTILE = 32 * CB;        // one batch of codes, as in global memory
  static constexpr int WARP_BYTES = (NS * STAGE + 2 * CTILE + 1023) / 1024 * 1024;
  static constexpr int TABLE = (kMaxCells + 1) * 32 * 8;  // lane-replicated (thr, lo) pairs
  static constexpr int MASK = D / 2 * 4;
  static constexpr int WARPS = WARPS_;
  static constexpr int THREADS = WARPS * 32;
  static constexpr int BARS = WARPS * NS * 8;
  static constexpr int HEAD = (TABLE + MASK + BARS + 1023) / 1024 * 1024;
  // + 1024: the dynamic shared memory base is rounded up to a 1024-byte boundary
  static constexpr size_t total() { return 1024 + size_t(HEAD) + size_t(WARPS) * WARP_BYTES; }
  static_assert(total() <= 227 * 1024, "shared memory");
};

// DRV: DRIVE's one-bit encoder (B = 1, ±1 codebook): code = (y' > 0) and the
// stored value is the scale that p.norm_mode selects (QuantParams::norm_mode).
template <typename T, int D, int B, int WARPS_ = 8, int NS_ = 2, int PF_ = 0, bool DRV = false>
__global__ void __launch_bounds__(EncBatch<T, D, B, WARPS_, NS_, PF_>::THREADS, 1)
encode_batch_kernel(const __grid_constant__ CUtensorMap xmap, int64_t n, uint8_t* __restrict__ codes,
                    float* __restrict__ norms, const QuantParams p) {
  using SM = EncBatch<T, D, B, WARPS_, NS_, PF_>;
  constexpr int P = D / 2, CB = SM::CB, NW = (CB + 3) / 4, NS = SM::NS;
  pdl_release();
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = dsm_raw + ((1024u - (smem_addr(dsm_raw) & 1023u)) & 1023u);
  float2* tab = reinterpret_cast<float2*>(dsm);
  uint32_t* smask = reinterpret_cast<uint32_t*>(dsm + SM::TABLE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(dsm + SM::TABLE + SM::MASK);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* wmem = dsm + SM::HEAD + warp * SM::WARP_BYTES;

  const int N = p.cell.cells;
  for (int i = threadIdx.x; i < (N + 1) * 32; i += blockDim.x)
    tab[i] = make_float2(p.cell.thr[i >> 5], __uint_as_float(p.cell.lo[i >> 5]));
  build_sign_mask<T, D>(smask, p.seed);
  if (lane == 0) {
    for (int s = 0; s < NS; ++s) mbarrier_init(smem_addr(&bars[warp * NS + s]), 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  pdl_wait();  // the shared tables are built: from here on, global memory

  const int64_t nb = (n + 31) >> 5;
  const int64_t tw = int64_t(gridDim.x) * SM::WARPS;
  // warp-major numbering: consecutive batches go to consecutive SMs, so every
  // SM gets the same number of batches (±1) whatever the warps per CTA
  const int64_t gw = int64_t(warp) * gridDim.x + blockIdx.x;
  const uint32_t bar0 = smem_addr(&bars[warp * NS]);
  const uint32_t stage0 = smem_addr(wmem);
  const uint32_t tab_lane = smem_addr(tab) + lane * 8;
  uint8_t* ctile = wmem + NS * SM::STAGE;
  uint32_t pending = 0;  // bit s: a load into stage s is in flight

  // Boxes past the end of the array are zero-filled and still count their full
  // size toward the transaction bytes.
  auto issue = [&](int s, int64_t b) {
    if (b >= nb) return;
    if (lane == 0) {
      const uint32_t bar = bar0 + 8 * s;
      mbarrier_expect_tx(bar, SM::STAGE);
#pragma unroll
      for (int h = 0; h < SM::BOXES; ++h)
        tma_load_2d(stage0 + s * SM::STAGE + h * 4096, &xmap, h * 64, int(b << 5), bar);
    }
    pending |= 1u << s;
  };
  auto prefetch = [&](int64_t b) {
    if (lane == 0 && b < nb) {
#pragma unroll
      for (int h = 0; h < SM::BOXES; ++h) tma_prefetch_2d(&xmap, h * 64, int(b << 5));
    }
  };

#pragma unroll
  for (int s = 0; s < NS; ++s) issue(s, gw + s * tw);
#pragma unroll
  for (int k = NS; k < NS + SM::PF; ++k) prefetch(gw + k * tw);

  const float Nf = float(N);
  const float A = p.cell.a;
  uint32_t parity = 0;  // bit s: phase parity to wait for on stage s
  int s = 0, ct = 0;
  bool failed = false;
  int64_t b = gw;
  for (; b < nb; b += tw) {
    if (!mbarrier_wait(bar0 + 8 * s, (parity >> s) & 1u)) {
      failed = true;
      break;
    }
    parity ^= 1u << s;
    pending &= ~(1u << s);
    const int64_t v0 = b << 5;
    const int nv = int(min(int64_t(32), n - v0));
    const bool valid = lane < nv;

    // row -> signs -> first butterfly -> fp32 pairs
    float2 w[P];
    const uint8_t* stage = wmem + s * SM::STAGE;
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
    issue(s, b + NS * tw);
    prefetch(b + (NS + SM::PF) * tw);

    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                     make_float2(0.f, 0.f)};
#pragma unroll
    for (int k = 0; k < P; ++k) acc[k & 3] = fma2(w[k], w[k], acc[k & 3]);
    const float2 a01 = add2(acc[0], acc[1]), a23 = add2(acc[2], acc[3]);
    const float2 a4 = add2(a01, a23);
    const float ss = 0.5f * (a4.x + a4.y);  // ‖x‖₂² (the butterfly doubled it)
    const float nu = sqrtf(ss);

#pragma unroll
    for (int mm = 1; mm < P; mm <<= 1) {
#pragma unroll
      for (int k = 0; k < P; ++k) {
        if ((k & mm) == 0) {
          const float2 a = w[k], c = w[k | mm];
          w[k] = add2(a, c);
          w[k | mm] = sub2(a, c);
        }
      }
    }

    uint32_t words[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) words[i] = 0u;
    float stored = nu;
    if constexpr (DRV) {
      static_assert(B == 1, "DRIVE codes are one bit");
      float2 l1[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int k = 0; k < P; ++k) {
        l1[k & 1] = add2(l1[k & 1], make_float2(fabsf(w[k].x), fabsf(w[k].y)));
        put_code<1>(words, 2 * k, w[k].x > 0.f ? 1u : 0u);
        put_code<1>(words, 2 * k + 1, w[k].y > 0.f ? 1u : 0u);
      }
      const float2 l = add2(l1[0], l1[1]);
      const float s1 = l.x + l.y;  // ‖y'‖₁ = √d·‖Πx‖₁
      stored = p.norm_mode == 1 ? s1 * p.inv_d : (s1 > 0.f ? __fdiv_rn(ss * float(D), s1) : 0.f);
    }
    const float sc = nu > 0.f ? __fdiv_rn(A, nu) : 0.f;  // s = sat(y'·A/ν + 1/2)
#pragma unroll
    for (int k = 0; k < (DRV ? 0 : P); ++k) {
      const float sx = __saturatef(fmaf(w[k].x, sc, 0.5f));
      const float sy = __saturatef(fmaf(w[k].y, sc, 0.5f));
      const float2 f = fma2(make_float2(sx, sy), make_float2(Nf, Nf), make_float2(8388608.f, 8388608.f));
      // the float bits are 0x4B000000 + round(s·N); ·256 drops the exponent
      const float2 ex = lds_f2(tab_lane + (__float_as_uint(f.x) << 8));
      const float2 ey = lds_f2(tab_lane + (__float_as_uint(f.y) << 8));
      const uint32_t cx = __float_as_uint(ex.y) + (sx > ex.x ? 1u : 0u);
      const uint32_t cy = __float_as_uint(ey.y) + (sy > ey.x ? 1u : 0u);
      if constexpr (B == 4) {
        const uint32_t byte = cx + (cy << 4);  // coordinates 2k (low nibble), 2k+1
        words[k >> 2] = (k & 3) == 0 ? byte : words[k >> 2] + (byte << (8 * (k & 3)));
      } else {
        put_code<B>(words, 2 * k, cx);
        put_code<B>(words, 2 * k + 1, cy);
      }
    }

    uint8_t* tile = ctile + ct * SM::CTILE;
    if (lane == 0) bulk_wait_read_1();  // the store from this tile two batches ago has read it
    __syncwarp();
    const bool bulk = (nv * CB) % 16 == 0;
    if (valid) {
      uint8_t* dst = bulk ? tile + lane * CB : codes + (v0 + lane) * CB;
      if constexpr (CB % 16 == 0) {
#pragma unroll
        for (int i = 0; i < CB / 16; ++i)
          reinterpret_cast<uint4*>(dst)[i] =
              make_uint4(words[4 * i], words[4 * i + 1], words[4 * i + 2], words[4 * i + 3]);
      } else {
#pragma unroll
        for (int i = 0; i < CB / 8; ++i)
          reinterpret_cast<uint2*>(dst)[i] = make_uint2(words[2 * i], words[2 * i + 1]);
      }
      norms[v0 + lane] = stored;
    }
    if (bulk) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) bulk_store(codes + v0 * CB, smem_addr(tile), uint32_t(nv * CB));
    }
    ct ^= 1;
    s = (s + 1 == NS) ? 0 : s + 1;
  }

  if (failed) {
    // A stage never completed: mark every vector this warp still owns with a
    // NaN norm, and wait (bounded) for the copies still in flight.
    for (; b < nb; b += tw) {
      const int64_t v0 = b << 5;
      if (lane < n - v0) norms[v0 + lane] = __uint_as_float(0x7fc00000u);
    }
#pragma unroll
    for (int st = 0; st < NS; ++st)
      if (pending & (1u << st)) mbarrier_wait(bar0 + 8 * st, (parity >> st) & 1u);
  }
  if (lane == 0) bulk_wait_all();
}

// cudaErrorNotSupported when no tensor map can be made (the caller then uses
// the general encoder).
template <typename T, int D, int B>
cudaError_t launch_encode_batch(const T* x, int64_t n, const QuantParams& p, uint8_t* codes,
                                float* norms, cudaStream_t stream) {
  if constexpr (D == 128 && B == 4) {
    if (p.norm_mode == 0) {
      cudaError_t e = launch_encode_tc<T>(x, n, p, codes, norms, stream);
      if (e != cudaErrorNotSupported) return e;
      e = launch_encode_mma<T>(x, n, p, codes, norms, stream);
      if (e != cudaErrorNotSupported) return e;
    }
  }
  using SM = EncBatch<T, D, B>;
  CUtensorMap xmap;
  if (!row_tensor_map(&xmap, x, n, D, 2, 32)) return cudaErrorNotSupported;
  auto k = encode_batch_kernel<T, D, B>;
  if constexpr (B == 1) {
    if (p.norm_mode != 0) k = encode_batch_kernel<T, D, 1, 8, 2, 0, true>;
  }
  constexpr size_t smem = SM::total();
  const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int64_t batches = (n + 31) / 32;
  const int grid = grid_for(reinterpret_cast<const void*>(k), SM::THREADS, smem,
                            (batches + SM::WARPS - 1) / SM::WARPS);
  return launch_pdl(k, grid, SM::THREADS, smem, stream, xmap, n, codes, norms, p);
}

}  // namespace rrq

namespace rrq {

// ------------------------------------------------------------------ decode
// One-lane-per-vector decoder for 4-bit codes and d ≤ 128 ("Random-rotation
// quantization" page, scheme step 3: dequantise, then apply Πᵀ).
//  * Codes and norms of the next batch stream into a per-warp cp.async ring
//    (80-byte rows: conflict-free 16-byte reads by the owning lane); the
//    batches after it are prefetched into L2.
//  * Each code byte (coordinates 2j, 2j+1) indexes a lane-replicated table of
//    fp32 pairs (c_lo + c_hi, c_lo − c_hi): level lookup and the first
//    butterfly at once.  The byte and the lane's table column are merged by
//    one byte permute into the table offset byte·256 + lane·8.
//  * log2(d) − 1 butterfly stages on packed fp32 pairs, × ν/d, rounding to
//    the output type, rotation signs (XOR of the sign bits).
//  * Rows go to a 128-byte-swizzled shared tile (conflict-free 16-byte
//    stores) and leave in TMA tensor stores, 32 rows × 128 bytes per box;
//    the store clips rows past the end of the array.
template <typename T, int D, int WARPS_, int NS_ = 2, int PF_ = 2> struct DecBatch {
  static_assert(D == 64 || D == 128, "batch decoder: d = 64 or 128");
  static constexpr int CB = D / 2;                 // 4-bit codes per vector
  static constexpr int RR = CB + 16;               // ring row: codes | norm | pad
  static constexpr int NS = NS_;                   // ring stages
  static constexpr int PF = PF_;                   // further batches prefetched into L2
  static constexpr int RING = NS * 32 * RR;
  static constexpr int ROW = D * Elem<T>::kBytes;  // output row bytes
  static constexpr int BOXES = ROW / 128;
  static constexpr int TILE = 32 * ROW;            // 1024-aligned output tile
  static constexpr int TABLE = 256 * 32 * 8;       // (lo + hi, lo − hi) per byte and lane
  static constexpr int MASK = mask_words<T, D>() * 4;
  static constexpr int HEAD = (TABLE + MASK + 1023) / 1024 * 1024;
  static constexpr int WARPS = WARPS_;
  static constexpr int THREADS = WARPS * 32;
  // [table | mask] [tiles of every warp] [rings of every warp]
  static constexpr size_t total() {
    return 1024 + size_t(HEAD) + size_t(WARPS) * TILE + size_t(WARPS) * RING;
  }
  static_assert(total() <= 227 * 1024, "shared memory");
};

template <typename T> constexpr int dec_batch_warps() { return Elem<T>::kBytes == 4 ? 6 : 12; }

template <typename T, int D, int WARPS_, int NS_ = 2, int PF_ = 2>
__global__ void __launch_bounds__(WARPS_ * 32, 1)
decode_batch_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ norms, int64_t n,
                    const __grid_constant__ CUtensorMap omap, const QuantParams p) {
  using SM = DecBatch<T, D, WARPS_, NS_, PF_>;
  constexpr int P = D / 2, CB = SM::CB, NS = SM::NS;
  pdl_release();
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = dsm_raw + ((1024u - (smem_addr(dsm_raw) & 1023u)) & 1023u);
  float2* tab = reinterpret_cast<float2*>(dsm);
  uint32_t* smask = reinterpret_cast<uint32_t*>(dsm + SM::TABLE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* tile = dsm + SM::HEAD + warp * SM::TILE;
  uint8_t* ring = dsm + SM::HEAD + SM::WARPS * SM::TILE + warp * SM::RING;

  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
    const int e = i >> 5;
    const float lo = p.levels[e & 15], hi = p.levels[e >> 4];
    tab[i] = make_float2(lo + hi, lo - hi);
  }
  build_sign_mask<T, D>(smask, p.seed);
  __syncthreads();
  pdl_wait();  // the shared tables are built: from here on, global memory

  const int64_t nb = (n + 31) >> 5;
  const int64_t tw = int64_t(gridDim.x) * SM::WARPS;
  // warp-major numbering: consecutive batches go to consecutive SMs, so every
  // SM gets the same number of batches (±1) whatever the warps per CTA
  const int64_t gw = int64_t(warp) * gridDim.x + blockIdx.x;
  const char* lane_tab = reinterpret_cast<const char*>(tab);
  const uint32_t lane8 = uint32_t(lane) * 8u;

  // batch b's codes and norms into ring stage st (16-byte units, coalesced)
  auto issue = [&](int st, int64_t b) {
    if (b < nb) {
      const int64_t v0 = b << 5;
      uint8_t* sb = ring + st * 32 * SM::RR;
#pragma unroll
      for (int i = 0; i < CB / 16; ++i) {
        const int t = lane + 32 * i, v = t / (CB / 16), u = t % (CB / 16);
        const bool ok = v0 + v < n;
        cp_async16(smem_addr(sb + v * SM::RR + u * 16), codes + (ok ? (v0 + v) * CB + u * 16 : 0),
                   ok ? 16 : 0);
      }
      const bool ok = v0 + lane < n;
      cp_async4(smem_addr(sb + lane * SM::RR + CB), norms + (ok ? v0 + lane : 0), ok ? 4 : 0);
    }
    cp_async_commit();
  };
  auto prefetch = [&](int64_t b) {
    if (lane == 0 && b < nb) {
      const int64_t v0 = b << 5;
      const uint32_t nv = uint32_t(min(int64_t(32), n - v0));
      prefetch_l2(codes + v0 * CB, nv * CB);
      if (nv * 4 % 16 == 0 && (reinterpret_cast<uintptr_t>(norms + v0) & 15) == 0)
        prefetch_l2(norms + v0, nv * 4);
    }
  };
#pragma unroll
  for (int k = 0; k < NS - 1; ++k) issue(k, gw + k * tw);
#pragma unroll
  for (int k = NS - 1; k < NS - 1 + SM::PF; ++k) prefetch(gw + k * tw);

  int st = 0;
  for (int64_t b = gw; b < nb; b += tw) {
    cp_async_wait<NS - 2>();
    __syncwarp();
    const uint8_t* row = ring + st * 32 * SM::RR + lane * SM::RR;
    uint32_t cw[CB / 4];
#pragma unroll
    for (int i = 0; i < CB / 16; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(row + 16 * i);
      cw[4 * i] = v.x; cw[4 * i + 1] = v.y; cw[4 * i + 2] = v.z; cw[4 * i + 3] = v.w;
    }
    const float nu = *reinterpret_cast<const float*>(row + CB);
    __syncwarp();  // every lane has read this stage before it is refilled
    issue((st + NS - 1) % NS, b + (NS - 1) * tw);
    prefetch(b + (NS - 1 + SM::PF) * tw);
    st = (st + 1 == NS) ? 0 : st + 1;

    float2 w[P];
#pragma unroll
    for (int j = 0; j < P; ++j) {
      // table offset: code byte j at bits 8..15, the lane's column at bits 0..7
      const uint32_t off = __byte_perm(cw[j >> 2], lane8, 0x5504u | ((j & 3) << 4));
      w[j] = *reinterpret_cast<const float2*>(lane_tab + off);
    }
    fwht2<D, D, true>(w, 0);

    if (lane == 0) bulk_wait_read_all();  // the previous batch's stores have read the tile
    __syncwarp();
    const float2 s2 = make_float2(nu * p.inv_d, nu * p.inv_d);
    if constexpr (Elem<T>::kBytes == 2) {
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {  // chunk c: values 8c .. 8c+7
        const uint4 m = reinterpret_cast<const uint4*>(smask)[c];
        uint4 o;
        o.x = pack2<T>(mul2(w[4 * c + 0], s2)) ^ m.x;
        o.y = pack2<T>(mul2(w[4 * c + 1], s2)) ^ m.y;
        o.z = pack2<T>(mul2(w[4 * c + 2], s2)) ^ m.z;
        o.w = pack2<T>(mul2(w[4 * c + 3], s2)) ^ m.w;
        *reinterpret_cast<uint4*>(tile + (c >> 3) * 4096 + swz128(lane, c & 7)) = o;
      }
    } else {
#pragma unroll
      for (int c = 0; c < D / 4; ++c) {  // chunk c: values 4c .. 4c+3
        const uint4 m = reinterpret_cast<const uint4*>(smask)[c];
        const float2 a = mul2(w[2 * c], s2), bb = mul2(w[2 * c + 1], s2);
        *reinterpret_cast<uint4*>(tile + (c >> 3) * 4096 + swz128(lane, c & 7)) =
            make_uint4(__float_as_uint(a.x) ^ m.x, __float_as_uint(a.y) ^ m.y,
                       __float_as_uint(bb.x) ^ m.z, __float_as_uint(bb.y) ^ m.w);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < SM::BOXES; ++h)
        tma_store_2d(&omap, h * (128 / Elem<T>::kBytes), int(b << 5), smem_addr(tile + h * 4096));
      bulk_commit();
    }
  }
  cp_async_wait<0>();
  if (lane == 0) bulk_wait_all();
}

// cudaErrorNotSupported when no tensor map can be made (the caller then uses
// the general decoder).
template <typename T, int D>
cudaError_t launch_decode_batch(const uint8_t* codes, const float* norms, int64_t n,
                                const QuantParams& p, T* out, cudaStream_t stream) {
  if constexpr (D == 128 && std::is_same<T, __half>::value) {
    const cudaError_t e = launch_decode_mma<T>(codes, norms, n, p, out, stream);
    if (e != cudaErrorNotSupported) return e;
  }
  constexpr int W = dec_batch_warps<T>();
  using SM = DecBatch<T, D, W>;
  CUtensorMap omap;
  if (!row_tensor_map(&omap, out, n, D, Elem<T>::kBytes, 32)) return cudaErrorNotSupported;
  auto k = decode_batch_kernel<T, D, W>;
  constexpr size_t smem = SM::total();
  const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int64_t batches = (n + 31) / 32;
  const int grid = grid_for(reinterpret_cast<const void*>(k), SM::THREADS, smem,
                            (batches + SM::WARPS - 1) / SM::WARPS);
  return launch_pdl(k, grid, SM::THREADS, smem, stream, codes, norms, n, omap, p);
}

}  // namespace rrq

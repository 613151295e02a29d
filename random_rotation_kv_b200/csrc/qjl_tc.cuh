// qjl_tc.cuh — MSE encode fused with the QJL sketch of the residual for
// 16-bit inputs at d = 128: both contractions on tcgen05, warp-specialised.
//
// "Random-rotation quantization" page, "History": QJL — a one-bit sketch of
// the residual made unbiased; TurboQuant — a (b−1)-bit MSE quantiser followed
// by the unbiased one-bit stage.  Per vector:
//     y' = H_128·D·x,  ν = ‖x‖ = ‖y'‖/√d,  code_i = the Lloyd–Max cell of y'_i/ν,
//     r = (y' − ν·c[code])/√d   (Πx − x̂ in the rotated domain),  ρ = ‖r‖,
//     v = S·r,  bit_i = [v_i > 0].
// One CTA per SM, 128-row tiles:
//  * a producer warp loads each tile with two TMA boxes (128-byte swizzle) and
//    issues the two products: Y = X·(D·H_128)ᵀ (8 × tcgen05.mma, M = N = 128,
//    K = 16, the input's own 16-bit type against the ±1 table — exact
//    products, fp32 sums) into one of two tensor-memory buffers, and later
//    V = R·Sᵀ from the residual tile R that the workers leave in shared memory
//    (16 products: R = R_hi + R_lo, two fp16 parts of the residual scaled by a
//    power of two, against S in fp16) into another pair of buffers;
//  * eight worker warps: tensor-memory lane r (tile row r) is read by warps w
//    and w + 4, each taking 64 coordinates; the halves of ‖y'‖² and ‖r‖² meet
//    through shared memory at a 64-thread named barrier; codes are byte 2 of
//    bits(f) + off_j (FixedSearch, mma_encode.cuh) and the level c[code] a
//    lane-replicated load from the unused half of the same table rows (for
//    b = 2 one 8-byte load per coordinate pair); the
//    signs of tile k − 1 are read while tile k's residual waits for its turn,
//    so neither the workers nor the tensor pipe wait on each other in steady
//    state.
// Every wait is bounded; after a timeout the remaining rows' residual norms
// are NaN, the copies and products in flight are waited for (bounded) and the
// tensor memory is freed.
#pragma once

#include "mma_encode.cuh"
#include "tc_encode.cuh"
#include "tcgen05.cuh"

namespace rrq {

struct QjlTc {
  static constexpr int D = 128, TILE = 128;
  // shared addresses (the dynamic base is checked to be kBase)
  static constexpr uint32_t kBase = 0x400;
  static constexpr uint32_t HT = 0x400;       // ±1 rotation table, 32 KB (as in tc_encode.cuh)
  static constexpr uint32_t SMASK = 0x8400;   // 128 sign bits
  static constexpr uint32_t BARS = 0x8410;    // in_full, y_done[2], v_done, a2_full
  static constexpr uint32_t TSLOT = 0x8440;
  static constexpr uint32_t FLAGS = 0x8444;
  static constexpr uint32_t PSUM = 0x8800;    // [tile parity][ν², ρ²][part][row], ≤ 8 KB
  static constexpr uint32_t kTable = 0x10000; // off_j at kTable + j·256 + lane·4
  static constexpr uint32_t kLev = 0x10080;   // c[code] at kLev + code·256 + lane·4 (b = 2: pairs)
  static constexpr uint32_t SB = 0x18000;     // S in fp16, K-major core matrices, 32 KB
  static constexpr uint32_t A2H = 0x20000;    // residual tile, high parts, 32 KB
  static constexpr uint32_t A2L = 0x28000;    // low parts, 32 KB
  static constexpr uint32_t IN = 0x30000;     // input tile: two 16 KB boxes
  static constexpr uint32_t kEnd = 0x38000;
  static constexpr size_t kTotal = size_t(kEnd) - kBase;
  static_assert(PSUM + 2 * 2 * 4 * TILE * 4 <= kTable && kTotal <= 227 * 1024, "layout");
  static constexpr uint32_t idesc(bool bf16) {  // kind::f16, fp32 accumulation, M = N = 128
    return (1u << 4) | (bf16 ? (1u << 7) | (1u << 10) : 0u) | ((128u / 8) << 17) | ((128u / 16) << 24);
  }
};

struct QjlTcArgs {
  int64_t n;
  const uint16_t* S;  // bf16 bits [128][128], row i = projection i
  uint8_t* codes;
  float* norms;
  uint8_t* qbits;
  float* rnorm;
  float rbound;  // 1 + max|c|/√d: |r_i| ≤ ν·rbound
};

// Byte offset of 16-byte chunk kb (8 k values) of row `row` in a [128 × 128]
// 16-bit K-major core-matrix tile (no swizzle).
__device__ __forceinline__ uint32_t qjl_cm(int row, int kb) {
  return uint32_t(row >> 3) * 2048u + uint32_t(kb) * 128u + uint32_t(row & 7) * 16u;
}

// Codes of coordinates 16g + [0, 16) of a thread's part of a row (byte 2 of
// each cv), b bits each LSB first, into the part's words; for b = 2 also the
// code pairs of coordinates (2t, 2t + 1) as bytes, the index of their levels.
template <int B, int NW>
__device__ __forceinline__ void pack16(const uint32_t (&cv)[16], int g, uint32_t (&w)[NW], uint32_t (&pairs)[2]) {
  // byte t of the result: the codes of cv[2t] (low) and cv[2t + 1], for 8 entries
  auto pair8 = [&](int o, int shift) {
    const uint32_t ev = __byte_perm(__byte_perm(cv[o], cv[o + 2], 0x0062u), __byte_perm(cv[o + 4], cv[o + 6], 0x6200u), 0x7610u);
    const uint32_t od = __byte_perm(__byte_perm(cv[o + 1], cv[o + 3], 0x0062u), __byte_perm(cv[o + 5], cv[o + 7], 0x6200u), 0x7610u);
    return ev + (od << shift);
  };
  if constexpr (B == 4) {
    w[2 * g] = pair8(0, 4);
    w[2 * g + 1] = pair8(8, 4);
  } else if constexpr (B == 2) {
    const uint32_t a = pair8(0, 2), b = pair8(8, 2);
    w[g] = __byte_perm(a, b, 0x6420u) + (__byte_perm(a, b, 0x7531u) << 4);
    pairs[0] = a;  // byte t: code(2t) | code(2t + 1) << 2, coordinates 0..7
    pairs[1] = b;  // the same for coordinates 8..15
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t c = __byte_perm(cv[j], 0u, 0x4442u);
      const int bit = (16 * g + j) * B, wi = bit >> 5, off = bit & 31;
      w[wi] |= c << off;
      if (off + B > 32) w[wi + 1] |= c >> (32 - off);
    }
  }
}

template <typename T, int B, int QS>
__global__ void __launch_bounds__(32 * (4 * QS + 1), 1)
qjl_tc_kernel(const __grid_constant__ CUtensorMap xmap, const QjlTcArgs a, const QuantParams p,
              const __grid_constant__ FixedSearch fs) {
  using L = QjlTc;
  constexpr int WORKERS = 4 * QS;        // QS threads per row (warps w, w + 4, ...)
  constexpr int CW = L::D / QS;          // coordinates per thread
  constexpr int CBH = CW * B / 8;        // code bytes per thread
  constexpr int NW = (CW * B + 31) / 32; // code words per thread
  extern __shared__ __align__(1024) uint8_t dsm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool producer = warp == WORKERS;
  const int h = warp >> 2, q = warp & 3;  // workers: row part, lane quarter
  const int row = 32 * q + lane;
  const int64_t ntiles = (a.n + L::TILE - 1) / L::TILE;
  const int64_t my_tiles = blockIdx.x < ntiles ? (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  auto tile_row0 = [&](int64_t k) { return (int64_t(blockIdx.x) + k * gridDim.x) * L::TILE; };
  pdl_release();
  if (smem_addr(dsm) != L::kBase) {
    // not the layout the launch assumed: this CTA's vectors get NaN residual norms
    pdl_wait();
    for (int64_t k = 0; k < my_tiles && !producer && h == 0; ++k) {
      const int64_t r = tile_row0(k) + row;
      if (r < a.n) a.rnorm[r] = __uint_as_float(0x7fc00000u);
    }
    return;
  }
  auto at = [&](uint32_t addr) { return dsm + (addr - L::kBase); };
  uint32_t* smask = reinterpret_cast<uint32_t*>(at(L::SMASK));
  uint64_t* bars = reinterpret_cast<uint64_t*>(at(L::BARS));
  uint64_t* in_full = bars + 0;
  uint64_t* y_done = bars + 1;  // [buffer]
  uint64_t* v_done = bars + 3;
  uint64_t* a2_full = bars + 4;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(at(L::TSLOT));
  volatile int* gfail = reinterpret_cast<volatile int*>(at(L::FLAGS));
  float* psum = reinterpret_cast<float*>(at(L::PSUM));
  uint32_t* tab = reinterpret_cast<uint32_t*>(at(L::kTable));

  // ---- tables, barriers, tensor memory (512 columns: Y[0], Y[1], V[0], V[1])
  if (warp < L::D / 32) {
    const uint32_t m = __ballot_sync(kFull, sign_bit(p.seed, 32 * warp + lane) != 0);
    if (lane == 0) smask[warp] = m;
  }
  for (int i = tid; i < 128 * 32; i += blockDim.x) tab[(i >> 5) * 64 + (i & 31)] = fs.off[i >> 5];
  if constexpr (B == 2) {
    // (c[e & 3], c[e >> 2]) for a code pair e in the second half of rows 0..15,
    // 16 copies of 8 bytes
    for (int i = tid; i < 16 * 16; i += blockDim.x) {
      const int e = i >> 4, l = i & 15;
      tab[e * 64 + 32 + 2 * l] = __float_as_uint(p.levels[e & 3]);
      tab[e * 64 + 32 + 2 * l + 1] = __float_as_uint(p.levels[e >> 2]);
    }
  } else {
    for (int i = tid; i < 16 * 32; i += blockDim.x)  // c[code] in the second half of rows 0..15
      tab[(i >> 5) * 64 + 32 + (i & 31)] = __float_as_uint((i >> 5) < (1 << B) ? p.levels[i >> 5] : 0.f);
  }
  if (tid == 0) {
    mbar_init(in_full, 1);
    mbar_init(&y_done[0], 1);
    mbar_init(&y_done[1], 1);
    mbar_init(v_done, 1);
    mbar_init(a2_full, WORKERS);
    gfail[0] = 0;
    fence_mbarrier_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tslot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  // the ±1 rotation table B^T[n][k] = s_k·(−1)^popc(n & k), as in tc_encode.cuh
  for (int i = tid; i < L::D * L::D / 8; i += blockDim.x) {
    const int m = i & 7, kb = (i >> 3) & 15, nn = ((i >> 7) << 3) | m;
    uint32_t e = (m & 1 ? 0xAAu : 0u) ^ (m & 2 ? 0xCCu : 0u) ^ (m & 4 ? 0xF0u : 0u);
    e ^= (smask[kb >> 2] >> (8 * (kb & 3))) & 0xFFu;
    e ^= (__popc(nn & (kb << 3)) & 1) ? 0xFFu : 0u;
    constexpr uint32_t one2 = uint32_t(MmaType<T>::kOne) * 0x10001u;
    uint32_t w[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) w[t] = one2 | (((e >> (2 * t)) & 1u) << 15) | (((e >> (2 * t + 1)) & 1u) << 31);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(L::HT + qjl_cm(nn, kb)), "r"(w[0]), "r"(w[1]),
                 "r"(w[2]), "r"(w[3])
                 : "memory");
  }
  pdl_wait();  // S and x may come from the previous kernel
  // S in fp16 (bf16 → fp16 is exact but for entries below 2^-14, which move by < 2^-25)
  for (int c = tid; c < L::D * 16; c += blockDim.x) {
    const int r = c >> 4, kb = c & 15;
    const uint4 v = *reinterpret_cast<const uint4*>(a.S + r * L::D + kb * 8);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2 hh = __floats2half2_rn(__uint_as_float(wv[j] << 16), __uint_as_float(wv[j] & 0xffff0000u));
      o[j] = *reinterpret_cast<const uint32_t*>(&hh);
    }
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(L::SB + qjl_cm(r, kb)), "r"(o[0]), "r"(o[1]),
                 "r"(o[2]), "r"(o[3])
                 : "memory");
  }
  fence_proxy_async_smem();  // the tables are visible to the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (producer) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && my_tiles > 0) {
      constexpr uint32_t IDESC1 = L::idesc(MmaType<T>::kOne == 0x3F80u);
      constexpr uint32_t IDESC2 = L::idesc(false);
      bool ok = true;
      bool copy_pending = false;
      uint32_t copy_phase = 0;
      int64_t n_mma1 = 0, n_mma2 = 0;  // products Y and V issued
      // one input stage: tile k + 1 is loaded once tile k's Y is done, so the
      // tiles two and three ahead are prefetched into L2 to hide the DRAM latency
      auto prefetch = [&](int64_t k) {
        if (k < my_tiles) {
          tma_prefetch_2d(&xmap, 0, int(tile_row0(k)));
          tma_prefetch_2d(&xmap, 64, int(tile_row0(k)));
        }
      };
      auto copy = [&](int64_t k) {
        prefetch(k + 2);
        mbarrier_expect_tx(smem_addr(in_full), 2 * 16384);
        tma_load_2d(L::IN, &xmap, 0, int(tile_row0(k)), smem_addr(in_full));
        tma_load_2d(L::IN + 16384, &xmap, 64, int(tile_row0(k)), smem_addr(in_full));
        copy_pending = true;
        copy_phase = uint32_t(k & 1);
      };
      auto mma1 = [&](int64_t k) {  // Y[k & 1] = X_k·(D·H)ᵀ
        const uint32_t d = tmem + uint32_t(k & 1) * 128u;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc_mma_f16(d, smem_desc_sw128(L::IN + (ks >> 2) * 16384 + (ks & 3) * 32),
                     smem_desc(L::HT + uint32_t(ks) * 256, 128, 2048), IDESC1, uint32_t(ks));
        mma_commit(&y_done[k & 1]);
        n_mma1 = k + 1;
      };
      auto mma2 = [&](int64_t k) {  // V[k & 1] = (R_hi + R_lo)·Sᵀ
        const uint32_t d = tmem + 256u + uint32_t(k & 1) * 128u;
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            tc_mma_f16(d, smem_desc((part ? L::A2L : L::A2H) + uint32_t(ks) * 256, 128, 2048),
                       smem_desc(L::SB + uint32_t(ks) * 256, 128, 2048), IDESC2, uint32_t(part | ks));
        mma_commit(v_done);
        ++n_mma2;
      };
      // Step k: tile k's copy landed → its Y; the workers' residual of tile
      // k − 1 → its V; tile k's Y done → the stage is free for tile k + 1.  Y[k & 1]
      // last held tile k − 2, read before the workers arrived on a2_full for tile
      // k − 2 (waited at step k − 1); V[(k − 1) & 1] last held tile k − 3, read
      // before their arrival for tile k − 1 (waited here).
      prefetch(1);
      copy(0);
      for (int64_t k = 0; k <= my_tiles && ok; ++k) {
        if (k < my_tiles) {
          ok = tc_wait(in_full, uint32_t(k & 1));
          if (!ok) break;
          copy_pending = false;
          tc_fence_after();
          mma1(k);
        }
        if (k >= 1) {
          ok = tc_wait(a2_full, uint32_t((k - 1) & 1));
          if (!ok) break;
          tc_fence_after();
          mma2(k - 1);
        }
        if (k + 1 < my_tiles) {
          ok = tc_wait(&y_done[k & 1], uint32_t((k >> 1) & 1));
          if (!ok) break;
          copy(k + 1);
        }
      }
      if (!ok) gfail[0] = 1;
      // after a failure: copies and products in flight end before the CTA exits
      if (copy_pending) tc_wait(in_full, copy_phase);
      if (n_mma1 > 0) tc_wait(&y_done[(n_mma1 - 1) & 1], uint32_t(((n_mma1 - 1) >> 1) & 1));
      if (n_mma2 > 0) tc_wait(v_done, uint32_t((n_mma2 - 1) & 1));
    }
  } else {
    // ----------------------------------------------------------------- workers
    const uint32_t row_bar = uint32_t(1 + q);  // the QS warps of lane quarter q
    constexpr uint32_t NROW = 32 * QS;
    const uint32_t lane_off = L::kTable | uint32_t(lane) * 4u;
    const uint32_t lane_lev = L::kLev | uint32_t(lane) * 4u;
    const uint32_t lane_pair = L::kLev | uint32_t(lane & 15) * 8u;
    const float2 bias2 = make_float2(fs.bias, fs.bias);
    const uint32_t tl = tmem + (uint32_t(32 * q) << 16) + uint32_t(CW * h);
    float rho_part = 0.f, sc_prev = 1.f;  // tile k − 1: this part's Σ rs², its scale
    // psum: [tile parity][ν², ρ²][part][row]
    auto pslot = [&](int64_t kk, int kind, int part) { return psum + ((int(kk & 1) * 2 + kind) * QS + part) * L::TILE + row; };
    auto part_sum = [&](int64_t kk, int kind) {  // the same order in every part
      float t = *pslot(kk, kind, 0);
#pragma unroll
      for (int i = 1; i < QS; ++i) t += *pslot(kk, kind, i);
      return t;
    };
    int64_t k = 0;
    auto signs = [&](int64_t kk, uint32_t (&bits)[CW / 32]) {  // tile kk's bits from V
#pragma unroll
      for (int c = 0; c < CW / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tl + 256u + uint32_t(kk & 1) * 128u + uint32_t(32 * c), v);
        tmem_ld_wait();
        uint32_t neg = 0;
#pragma unroll
        for (int j = 31; j >= 0; --j) neg = (neg << 1) | (v[j] >> 31);
        bits[c] = ~neg;
      }
    };
    auto store_bits = [&](int64_t kk, const uint32_t (&bits)[CW / 32], float rho) {
      const int64_t rp = tile_row0(kk) + row;
      if (rp < a.n) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(a.qbits + rp * 16) + (CW / 32) * h;
#pragma unroll
        for (int c = 0; c < CW / 32; ++c) dst[c] = rho > 0.f ? bits[c] : 0u;
        if (h == 0) a.rnorm[rp] = rho;
      }
    };
    for (; k < my_tiles; ++k) {
      const int s = int(k & 1);
      if (!bar_and(row_bar, NROW, gfail[0] == 0 && tc_wait(&y_done[s], uint32_t((k >> 1) & 1)))) break;
      tc_fence_after();
      // ---- y'[CW·h + c] of tile row `row`
      uint32_t y[CW / 16][16];
#pragma unroll
      for (int i = 0; i < CW / 16; ++i) tmem_ld16(tl + uint32_t(s * 128 + 16 * i), y[i]);
      tmem_ld_wait();
      float2 acc = make_float2(0.f, 0.f), acc2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < CW / 16; ++i)
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          const float2 u = make_float2(__uint_as_float(y[i][2 * j]), __uint_as_float(y[i][2 * j + 1]));
          const float2 w = make_float2(__uint_as_float(y[i][2 * j + 2]), __uint_as_float(y[i][2 * j + 3]));
          acc = fma2(u, u, acc);
          acc2 = fma2(w, w, acc2);
        }
      const float2 qa = add2(acc, acc2);
      *pslot(k, 0, h) = qa.x + qa.y;
      *pslot(k - 1, 1, h) = rho_part;
      bar_named(row_bar, NROW);
      const float nu2 = part_sum(k, 0) * p.inv_d;
      const float rho_prev = sqrtf(part_sum(k - 1, 1)) / sc_prev;
      const float nu = sqrtf(nu2);
      const float scs = nu2 > 0.f ? fs.num * rsqrtf(nu2) : 0.f;  // 2^18/ν
      // sc = 2^(10 − e) with ν·rbound < 2^e (ν·rbound is a normal float when ν > 0):
      // |r·sc| ≤ 2^10
      const int ex = max(int((__float_as_uint(nu * a.rbound) >> 23) & 0xFFu) - 126, -100);
      const float sc = nu > 0.f ? __uint_as_float(uint32_t(127 + 10 - ex) << 23) : 1.f;
      const float k1 = sc * p.inv_sqrt_d, k2 = -nu * k1;

      // ---- per 16 coordinates: codes (cv = bits(f) + off_j, the code in byte
      // 2), the level c[code], the residual scaled by sc and split in two fp16
      // parts, kept in registers until the residual tile is free
      uint32_t words[NW], hi[CW / 2], lo[CW / 2];
#pragma unroll
      for (int i = 0; i < NW; ++i) words[i] = 0u;
      float2 racc = make_float2(0.f, 0.f);
#pragma unroll
      for (int g16 = 0; g16 < CW / 16; ++g16) {
        uint32_t cv[16];
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          const float2 f = fma2(make_float2(__uint_as_float(y[g16][j]), __uint_as_float(y[g16][j + 1])),
                                make_float2(scs, scs), bias2);
          const uint32_t fx = __float_as_uint(f.x), fy = __float_as_uint(f.y);
          cv[j] = fx + lds_u32(__byte_perm(fx, lane_off, 0x7624u));
          cv[j + 1] = fy + lds_u32(__byte_perm(fy, lane_off, 0x7624u));
        }
        uint32_t pairs[2];
        pack16<B, NW>(cv, g16, words, pairs);
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          float cx, cy;
          if constexpr (B == 2) {
            const float2 c2 = lds_f2(__byte_perm(pairs[j >> 3], lane_pair, 0x7604u | (((j >> 1) & 3) << 4)));
            cx = c2.x;
            cy = c2.y;
          } else {
            cx = __uint_as_float(lds_u32(__byte_perm(cv[j], lane_lev, 0x7624u)));
            cy = __uint_as_float(lds_u32(__byte_perm(cv[j + 1], lane_lev, 0x7624u)));
          }
          const float2 yv = make_float2(__uint_as_float(y[g16][j]), __uint_as_float(y[g16][j + 1]));
          const float2 r = fma2(make_float2(cx, cy), make_float2(k2, k2), mul2(yv, make_float2(k1, k1)));
          racc = fma2(r, r, racc);
          const __half2 hh = __float22half2_rn(r);
          const __half2 ll = __float22half2_rn(sub2(r, __half22float2(hh)));
          hi[8 * g16 + j / 2] = *reinterpret_cast<const uint32_t*>(&hh);
          lo[8 * g16 + j / 2] = *reinterpret_cast<const uint32_t*>(&ll);
        }
      }
      const int64_t r0 = tile_row0(k) + row;
      if (r0 < a.n) {
        uint8_t* dst = a.codes + r0 * (QS * CBH) + h * CBH;
        if constexpr (CBH % 16 == 0) {
#pragma unroll
          for (int i = 0; i < CBH / 16; ++i)
            reinterpret_cast<uint4*>(dst)[i] = make_uint4(words[4 * i], words[4 * i + 1], words[4 * i + 2], words[4 * i + 3]);
        } else if constexpr (CBH % 8 == 0) {
#pragma unroll
          for (int i = 0; i < CBH / 8; ++i) reinterpret_cast<uint2*>(dst)[i] = make_uint2(words[2 * i], words[2 * i + 1]);
        } else {
#pragma unroll
          for (int i = 0; i < CBH / 4; ++i) reinterpret_cast<uint32_t*>(dst)[i] = words[i];
        }
        if (h == 0) a.norms[r0] = nu;
      }

      // ---- tile k − 1: its product V is the last reader of the residual tile
      if (k >= 1) {
        const bool vok = tc_wait(v_done, uint32_t((k - 1) & 1));
        if (!vok) gfail[0] = 1;
        tc_fence_after();
        uint32_t bits[CW / 32];
        signs(k - 1, bits);
        store_bits(k - 1, bits, vok ? rho_prev : __uint_as_float(0x7fc00000u));
      }

      // ---- residual tile: this thread's row, K chunks (CW/8)·h + kb
#pragma unroll
      for (int kb = 0; kb < CW / 8; ++kb) {
        const uint32_t off = qjl_cm(row, (CW / 8) * h + kb);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(L::A2H + off), "r"(hi[4 * kb]),
                     "r"(hi[4 * kb + 1]), "r"(hi[4 * kb + 2]), "r"(hi[4 * kb + 3])
                     : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(L::A2L + off), "r"(lo[4 * kb]),
                     "r"(lo[4 * kb + 1]), "r"(lo[4 * kb + 2]), "r"(lo[4 * kb + 3])
                     : "memory");
      }
      rho_part = racc.x + racc.y;
      sc_prev = sc;
      fence_proxy_async_smem();  // the residual tile is visible to the tensor cores
      tc_fence_before();          // and this warp's tensor-memory reads are done
      __syncwarp();
      if (lane == 0) mbar_arrive(a2_full);
    }
    if (k < my_tiles) {
      // a wait gave up: the rest of the rows (from tile k − 1 on) get NaN
      gfail[0] = 1;
      for (int64_t kk = k > 0 ? k - 1 : 0; kk < my_tiles && h == 0; ++kk) {
        const int64_t r = tile_row0(kk) + row;
        if (r < a.n) a.rnorm[r] = __uint_as_float(0x7fc00000u);
      }
    } else if (my_tiles > 0) {
      // the last tile's signs and residual norm
      const bool ok = tc_wait(v_done, uint32_t((my_tiles - 1) & 1));
      tc_fence_after();
      uint32_t bits[CW / 32];
      signs(my_tiles - 1, bits);
      *pslot(my_tiles - 1, 1, h) = rho_part;
      bar_named(row_bar, NROW);
      const float rho = ok ? sqrtf(part_sum(my_tiles - 1, 1)) / sc_prev : __uint_as_float(0x7fc00000u);
      store_bits(my_tiles - 1, bits, rho);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
  }
}

// cudaErrorNotSupported when this kernel cannot serve the call (the caller then
// uses another QJL kernel): norm mode, codebook, layout or tensor map.
template <typename T, int B, int QS = 2>
cudaError_t launch_qjl_tc(const void* x, int64_t n, const QuantParams& p, const uint16_t* S, uint8_t* codes,
                          float* norms, uint8_t* qbits, float* rnorm, cudaStream_t stream) {
  if (p.norm_mode != 0) return cudaErrorNotSupported;
  const FixedSearch fs = make_fixed_search(p);
  if (!fs.ok) return cudaErrorNotSupported;
  int dev = 0, reserved = 0, sms = 1;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      uint32_t(reserved) != QjlTc::kBase)
    return cudaErrorNotSupported;
  CUtensorMap xmap;
  if (!row_tensor_map(&xmap, x, n, 128, 2, QjlTc::TILE)) return cudaErrorNotSupported;
  QjlTcArgs a;
  a.n = n;
  a.S = S;
  a.codes = codes;
  a.norms = norms;
  a.qbits = qbits;
  a.rnorm = rnorm;
  float cmax = 0.f;
  for (int k = 0; k < (1 << B); ++k) cmax = std::fmax(cmax, std::fabs(p.levels[k]));
  a.rbound = 1.f + cmax * p.inv_sqrt_d;
  auto k = qjl_tc_kernel<T, B, QS>;
  constexpr size_t smem = QjlTc::kTotal;
  const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int64_t tiles = (n + QjlTc::TILE - 1) / QjlTc::TILE;
  const int grid = int(tiles < sms ? tiles : sms);
  return launch_pdl(k, grid, 32 * (4 * QS + 1), smem, stream, xmap, a, p, fs);
}

}  // namespace rrq

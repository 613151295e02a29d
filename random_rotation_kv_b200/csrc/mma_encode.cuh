// mma_encode.cuh — encoder for d = 128, 4-bit codes and 16-bit inputs (the
// KV-cache case) with the Hadamard transform on tensor-core tiles.
//
// "Random-rotation quantization" page: scheme steps 1–2 (rotate by Π, then
// quantise every rotated coordinate with one fixed codebook); "Why rotation
// works" (the randomized Hadamard transform); "History", EDEN bullet
// (normalise to ≈N(0,1), Lloyd–Max codebook) and TurboQuant bullet (one
// constant scale per vector).
//
// The rotation y' = H·D·x is a dense product with a ±1 matrix, and H factors
// as H_128 = H_4 ⊗ H_32 over the split of a coordinate c = 32a + b (block a,
// offset b): H_128[c, c'] = H_4[a, a']·H_32[b, b'].  So
//     z[a, b] = Σ_b' H_32[b, b']·s_{32a+b'}·x_{32a+b'}     (one 32×32 product per block),
//     y'[32a + b] = Σ_a' H_4[a, a']·z[a', b]               (two butterfly stages).
// A warp takes a batch of 32 vectors (rows).  The first step is, per block, the
// product X_a[32 × 32]·B_a[32 × 32] with B_a[k][n] = s_{32a+k}·H_32[π(n), k]: the
// rotation signs sit in the ±1 table, exact in fp16/bf16, so the inputs go to
// the tensor cores untouched (mma.sync m16n8k16, fp16/bf16 operands as stored,
// fp32 accumulation).  Each thread then holds, for 4 rows, the same 32 column
// positions of all 4 blocks, and the H_4 stages run in its registers on packed
// fp32 pairs.  The column order π (bit fields 1–2 and 3–4 of the column index
// swapped) makes thread c of a quad own coordinates 32a + 8c + [0, 8) of each
// block, i.e. the 4-byte code words 4a + c of its rows.
//
// Per batch that is 64 MMAs, 16 ldmatrix loads of the inputs and 16 of the
// tables and 128 packed butterfly operations, where the one-lane-per-vector
// kernel (batch_kernels.cuh) spends 64 sign XORs, 192 conversion-and-first-
// stage operations and 384 packed butterfly operations on the transform:
//  * inputs arrive as TMA tensor boxes (32 rows × 128 bytes, 128-byte swizzle,
//    zero fill past the end), one stage per warp: the stage is refilled as soon
//    as the warp's fragments are in registers, and 12 warps per SM cover the
//    copy latency;
//  * ν² = ‖y'‖²/d from the thread's 32 values per row and two quad shuffles;
//    each thread of a quad computes ν and 2^18/ν of one of its 4 rows and shares
//    the scale by shuffles;
//  * the code search is the fixed-point table search below (FixedSearch);
//  * codes go to a per-warp 32 × 64-byte tile in the 64-byte swizzle (the
//    quad-strided word stores are conflict-free in it) and leave in one TMA
//    tensor store per batch, which clips rows past the end.
// The shared layout is fixed (the dynamic base must be shared address 0x400;
// the launch checks the device's reserved shared memory and the kernel checks
// the address): the search table sits at 0x10000, the warps' buffers below
// and above it.
#pragma once

#include <cmath>
#include <cstdlib>
#include <type_traits>

#include "tensor_map.h"

namespace rrq {

template <typename T> struct MmaType;
template <> struct MmaType<__half> {
  static constexpr uint16_t kOne = 0x3C00u, kMinusOne = 0xBC00u;
};
template <> struct MmaType<__nv_bfloat16> {
  static constexpr uint16_t kOne = 0x3F80u, kMinusOne = 0xBF80u;
};

// d += A·B for one m16n8k16 tile, 16-bit operands of type T, fp32 accumulators.
template <typename T>
__device__ __forceinline__ void mma_t(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1);
template <>
__device__ __forceinline__ void mma_t<__half>(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
template <>
__device__ __forceinline__ void mma_t<__nv_bfloat16>(float (&d)[4], const uint32_t (&a)[4],
                                                     uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four 8×8 16-bit matrices from shared memory; lane l gives the address of row
// l mod 8 of matrix l / 8, and register j receives matrix j.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Fixed-point code search.  The kernel forms I = round(u·2^18) for the
// normalised coordinate u = y'/ν as the integer bits of one fp32 FMA,
//     f = y'·(2^18/ν) + 1.5·2^23,   bits(f) = 0x4B400000 + I   (|I| < 2^22),
// so the cell j = ⌊I / 2^16⌋ (a quarter of a unit of u wide) is byte 2 of
// bits(f) minus 0x40, and the decision u > τ_k is the integer comparison
// I > T_k with T_k = ⌊τ_k·2^18⌋ (exact, from the levels in double on the host).
// I resolves u to 2^-18 ≈ 3.8·10^-6, inside the 10^-5 band of the decision
// rule.  |u| ≤ √d = 11.3 keeps j within ±46, so a 128-row table holds every
// reachable cell.  Byte 2 of bits(f) and the lane's column are merged by one
// byte permute into the address of the lane-replicated entry (thr_j, lo_j) at
// shared address 0x10000 + byte·256 + lane·8:
//     code = lo_j + (I > thr_j),   thr_j = the one T_k in cell j (or none),
// the comparison being the carry of I − (thr_j + 1) added to lo_j,
// with no saturation and no separate s.  A codebook with two thresholds within
// one cell of the reachable range (closer than 1/4) takes another encoder.
// The same decision in one integer add: with off_j chosen so that
//     bits(f) + off_j ≡ (lo_j + 1)·2^16 + (I − thr_j − 1)   (cell with a threshold)
//     bits(f) + off_j ≡  lo_j·2^16      + (I − 2^16·j)      (cell without one)
// modulo 2^24, byte 2 of bits(f) + off_j is the code itself: in the first case
// I − thr_j − 1 lies in [−2^16, 2^16) and borrows from byte 2 exactly when
// I ≤ thr_j; in the second it lies in [0, 2^16).
struct FixedSearch {
  int ok;            // 0: the table cannot serve this codebook (another encoder runs)
  float num;         // 2^18 (scaled by 1/ν per vector)
  float bias;        // 1.5·2^23
  uint2 rows[128];   // row r = cell r − 64: (biased threshold inside it + 1, or 2^32 − 1; lo)
  uint32_t off[128]; // row r: off_j above (mod 2^32)
};

// Host: the fixed-point parameters for a codebook (levels ascending, L = 2^bits)
// at d = 128, or ok = 0 when two thresholds share a reachable cell.
inline FixedSearch make_fixed_search(const QuantParams& p) {
  FixedSearch fs{};
  const int L = 1 << p.bits, nthr = L - 1;
  const double G = 262144.0;
  int32_t T[kMaxLevels];
  for (int k = 0; k < nthr; ++k) {
    const double tau = (double(p.levels[k]) + double(p.levels[k + 1])) * 0.5;
    // |I| < 2^22 always, so clamping far thresholds at ±2^23 keeps every decision
    const double t = std::floor(tau * G);
    T[k] = int32_t(t < -8388608.0 ? -8388608.0 : (t > 8388608.0 ? 8388608.0 : t));
  }
  for (int k = 1; k < nthr; ++k) {
    const bool reachable = T[k] >= -(64 << 16) && T[k - 1] < (64 << 16);
    if (reachable && (T[k] >> 16) == (T[k - 1] >> 16)) return fs;
  }
  fs.ok = 1;
  fs.num = float(G);
  fs.bias = float(1.5 * 8388608.0);
  for (int r = 0; r < 128; ++r) {
    const int64_t edge = int64_t(r - 64) * 65536;  // I at the cell's lower end
    uint32_t lo = 0, thr = 0xFFFFFFFFu;
    int64_t anchor = edge;  // the I that lands on a whole multiple of 2^16: edge, or thr_j + 1
    for (int k = 0; k < nthr; ++k) {
      if (T[k] < edge) {
        ++lo;
      } else if (T[k] < edge + 65536) {
        thr = uint32_t(int32_t(0x4B400000) + T[k]) + 1u;
        anchor = int64_t(T[k]) + 1;
      }
    }
    fs.rows[r] = make_uint2(thr, lo);
    const int64_t target = int64_t(lo + (thr == 0xFFFFFFFFu ? 0u : 1u)) << 16;
    fs.off[r] = uint32_t(uint64_t(target - (int64_t(0x4B400000) + anchor)));
  }
  return fs;
}

// Code of one coordinate from its biased fixed-point value f and the address of
// its cell's entry (thr + 1, lo): lo plus the carry of f − (thr + 1), i.e.
// lo + (f > thr), in one subtract-with-carry and one add-carry.
__device__ __forceinline__ uint32_t code_at(uint32_t f, uint32_t addr) {
  uint32_t thr1, lo, c;
  asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(thr1), "=r"(lo) : "r"(addr));
  asm("{\n\t.reg .u32 t;\n\tsub.cc.u32 t, %1, %2;\n\taddc.u32 %0, %3, 0;\n\t}"
      : "=r"(c)
      : "r"(f), "r"(thr1), "r"(lo));
  return c;
}

template <int WARPS_, int NS_, int CT_> struct EncMma {
  static constexpr int D = 128, NB = 4, ROW = 256, BOXES = 2, CB = 64;
  static constexpr int NS = NS_, CT = CT_, WARPS = WARPS_, THREADS = WARPS * 32;
  static constexpr int STAGE = 32 * ROW, CTILE = 32 * CB;
  static constexpr int WB = (NS * STAGE + CT * CTILE + 1023) / 1024 * 1024;
  static constexpr uint32_t kBase = 0x400;      // dynamic shared memory base (checked)
  static constexpr uint32_t kTable = 0x10000;   // lane-replicated entries, rows 0..127
  static constexpr uint32_t kTableEnd = kTable + 128 * 256;
  static constexpr int HROW = 80, HTAB = NB * 32 * HROW;
  static constexpr uint32_t HT = 0, SIGNS = HTAB, BARS = SIGNS + D;  // offsets from kBase
  static constexpr uint32_t FRONT = kBase + (BARS + WARPS * NS * 8 + 1023) / 1024 * 1024;
  static constexpr int NFRONT = (kTable - FRONT) / WB < WARPS ? int((kTable - FRONT) / WB) : WARPS;
  static constexpr uint32_t warp_base(int w) {  // shared address of warp w's buffers
    return w < NFRONT ? FRONT + uint32_t(w) * WB : kTableEnd + uint32_t(w - NFRONT) * WB;
  }
  static constexpr size_t total() { return size_t(warp_base(WARPS)) - kBase; }
  static_assert(total() <= 227 * 1024, "shared memory");
  static_assert(FRONT % 1024 == 0 && kTableEnd % 1024 == 0, "1024-aligned stages");
};

template <typename T, int WARPS_, int NS_, int CT_, bool SPLIT>
__global__ void __launch_bounds__(WARPS_ * 32, 1)
encode_mma_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap cmap,
                   int64_t n, float* __restrict__ norms, const QuantParams p,
                   const __grid_constant__ FixedSearch fs) {
  using SM = EncMma<WARPS_, NS_, CT_>;
  constexpr int NB = SM::NB, NS = SM::NS;
  pdl_release();
  extern __shared__ __align__(1024) uint8_t dsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_addr(dsm) != SM::kBase) {
    // not the layout the launch assumed: mark every norm of this CTA's batches NaN
    pdl_wait();
    for (int64_t b = int64_t(warp) * gridDim.x + blockIdx.x; b < (n + 31) >> 5;
         b += int64_t(gridDim.x) * SM::WARPS)
      if ((b << 5) + lane < n) norms[(b << 5) + lane] = __uint_as_float(0x7fc00000u);
    return;
  }
  uint8_t* htab = dsm + SM::HT;
  uint8_t* signs = dsm + SM::SIGNS;
  uint64_t* bars = reinterpret_cast<uint64_t*>(dsm + SM::BARS);
  uint2* tab = reinterpret_cast<uint2*>(dsm + (SM::kTable - SM::kBase));

  for (int i = threadIdx.x; i < SM::D; i += blockDim.x) signs[i] = uint8_t(sign_bit(p.seed, i));
  for (int i = threadIdx.x; i < 128 * 32; i += blockDim.x) tab[i] = fs.rows[i >> 5];
  if (lane == 0) {
    for (int st = 0; st < NS; ++st) mbarrier_init(smem_addr(&bars[warp * NS + st]), 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  for (int i = threadIdx.x; i < NB * 32 * 32; i += blockDim.x) {
    const int k = i & 31, nn = (i >> 5) & 31, a = i >> 10;
    const int pn = (nn & 1) | (((nn >> 3) & 3) << 1) | (((nn >> 1) & 3) << 3);
    const int neg = (signs[32 * a + k] ^ __popc(pn & k)) & 1;
    reinterpret_cast<uint16_t*>(htab + (a * 32 + nn) * SM::HROW)[k] =
        neg ? MmaType<T>::kMinusOne : MmaType<T>::kOne;
  }
  __syncthreads();
  pdl_wait();

  const int64_t nb = (n + 31) >> 5;
  const int64_t tw = int64_t(gridDim.x) * SM::WARPS;
  const int64_t gw = int64_t(warp) * gridDim.x + blockIdx.x;
  const uint32_t wbase = SM::warp_base(warp);
  const uint32_t bar0 = smem_addr(&bars[warp * NS]);
  const uint32_t stage0 = wbase;
  const uint32_t ctile0 = wbase + NS * SM::STAGE;
  const int qr = lane >> 2, qc = lane & 3;
  const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8, a_chunk = lane >> 4;
  const uint32_t h_lane = smem_addr(htab) + uint32_t((lane & 7) * SM::HROW + (lane >> 3) * 16);
  const uint32_t lane_word = SM::kTable | uint32_t(lane) * 8u;  // bytes 0 and 2 of the address
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

  const float num = fs.num, bias = fs.bias;
  // codes of a coordinate pair: byte = code(v.x) | code(v.y) << 4
  auto pair_code = [&](float2 v, float sc) -> uint32_t {
    const float2 f = fma2(v, make_float2(sc, sc), make_float2(bias, bias));
    const uint32_t fx = __float_as_uint(f.x), fy = __float_as_uint(f.y);
    return code_at(fx, __byte_perm(fx, lane_word, 0x7624u)) +
           (code_at(fy, __byte_perm(fy, lane_word, 0x7624u)) << 4);
  };

  uint32_t parity = 0;
  int st = 0, ct = 0;
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
    const uint32_t sbase = stage0 + st * SM::STAGE;
    if (lane == 0 && CT_ == 2) bulk_wait_read_1();
    if (lane == 0 && CT_ == 1) bulk_wait_read_all();
    const uint32_t tile = ctile0 + (CT_ == 2 ? ct : 0) * SM::CTILE;
    const uint32_t swz = uint32_t((qr >> 1) & 3);
    float my_nu = 0.f;

    // one m-tile of 16 rows (mt), or both at once
    auto run = [&](auto mts) {
      constexpr int M0 = decltype(mts)::value >= 2 ? 0 : decltype(mts)::value;
      constexpr int MN = decltype(mts)::value >= 2 ? 2 : 1;
      float acc[NB][MN][4][4];
#pragma unroll
      for (int a = 0; a < NB; ++a) {
        uint32_t bf[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) ldsm_x4(bf[nt], h_lane + uint32_t((a * 32 + 8 * nt) * SM::HROW));
#pragma unroll
        for (int m = 0; m < MN; ++m) {
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) acc[a][m][nt][0] = acc[a][m][nt][1] = acc[a][m][nt][2] = acc[a][m][nt][3] = 0.f;
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const int colb = 64 * a + 32 * ks + 16 * a_chunk;
            uint32_t af[4];
            ldsm_x4(af, sbase + (colb >> 7) * 4096 + swz128(16 * (M0 + m) + a_row, (colb & 127) >> 4));
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) mma_t<T>(acc[a][m][nt], af, bf[nt][2 * ks], bf[nt][2 * ks + 1]);
          }
        }
      }
      if (M0 + MN == 2) {  // every fragment of the stage is in registers: refill it
        __syncwarp();
        fence_proxy_async_smem();
        issue(st, b + NS * tw);
      }
      // H_4 over the blocks, ν² per row (r = h + 2m)
      float2 q2[2 * MN];
#pragma unroll
      for (int r = 0; r < 2 * MN; ++r) q2[r] = make_float2(0.f, 0.f);
#pragma unroll
      for (int m = 0; m < MN; ++m)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float2 z[NB];
#pragma unroll
            for (int a = 0; a < NB; ++a) z[a] = make_float2(acc[a][m][nt][2 * h], acc[a][m][nt][2 * h + 1]);
#pragma unroll
            for (int mm = 1; mm < NB; mm <<= 1)
#pragma unroll
              for (int a = 0; a < NB; ++a)
                if ((a & mm) == 0) {
                  const float2 u = z[a], w = z[a | mm];
                  z[a] = add2(u, w);
                  z[a | mm] = sub2(u, w);
                }
#pragma unroll
            for (int a = 0; a < NB; ++a) {
              acc[a][m][nt][2 * h] = z[a].x;
              acc[a][m][nt][2 * h + 1] = z[a].y;
              q2[h + 2 * m] = fma2(z[a], z[a], q2[h + 2 * m]);
            }
          }
      float ss[2 * MN];
#pragma unroll
      for (int r = 0; r < 2 * MN; ++r) {
        ss[r] = q2[r].x + q2[r].y;
        ss[r] += __shfl_xor_sync(kFull, ss[r], 1);
        ss[r] += __shfl_xor_sync(kFull, ss[r], 2);
      }
      // thread qc: ν of local row qc mod 2·MN; rows are qr + 8(h + 2(M0 + m))
      float mine = ss[0];
#pragma unroll
      for (int r = 1; r < 2 * MN; ++r) mine = (qc % (2 * MN)) == r ? ss[r] : mine;
      const float nu = sqrtf(mine * p.inv_d);
      const float msc = nu > 0.f ? __fdiv_rn(num, nu) : 0.f;
      if (MN == 2 || (qc >> 1) == M0) my_nu = nu;
      float sc[2 * MN];
#pragma unroll
      for (int r = 0; r < 2 * MN; ++r) sc[r] = __shfl_sync(kFull, msc, (lane & ~3) | r);
#pragma unroll
      for (int m = 0; m < MN; ++m)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = qr + 8 * (h + 2 * (M0 + m));
#pragma unroll
          for (int a = 0; a < NB; ++a) {
            uint32_t word = 0;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
              word += pair_code(make_float2(acc[a][m][nt][2 * h], acc[a][m][nt][2 * h + 1]), sc[h + 2 * m])
                      << (8 * nt);
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(tile + uint32_t(row * 64) + ((uint32_t(a) ^ swz) << 4) +
                                                             uint32_t(qc * 4)),
                         "r"(word)
                         : "memory");
          }
        }
    };
    if constexpr (SPLIT) {
      run(std::integral_constant<int, 0>());
      run(std::integral_constant<int, 1>());
    } else {
      run(std::integral_constant<int, 2>());
    }
    if (v0 + qr + 8 * qc < n) norms[v0 + qr + 8 * qc] = my_nu;
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(&cmap, 0, int(v0), tile);
      bulk_commit();
    }
    ct ^= 1;
    st = (st + 1 == NS) ? 0 : st + 1;
  }

  if (failed) {
    for (; b < nb; b += tw) {
      const int64_t v0 = b << 5;
      if (lane < n - v0) norms[v0 + lane] = __uint_as_float(0x7fc00000u);
    }
#pragma unroll
    for (int s2 = 0; s2 < NS; ++s2)
      if (pending & (1u << s2)) mbarrier_wait(bar0 + 8 * s2, (parity >> s2) & 1u);
  }
  if (lane == 0) bulk_wait_all();
}

template <typename T, int W, int NS, int CT, bool SPLIT>
cudaError_t launch_encode_mma_v(const CUtensorMap& xmap, const CUtensorMap& cmap, int64_t n,
                                 const QuantParams& p, const FixedSearch& fs, float* norms,
                                 cudaStream_t stream) {
  using SM = EncMma<W, NS, CT>;
  auto k = encode_mma_kernel<T, W, NS, CT, SPLIT>;
  constexpr size_t smem = SM::total();
  const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int64_t batches = (n + 31) / 32;
  const int grid = grid_for(reinterpret_cast<const void*>(k), SM::THREADS, smem, (batches + W - 1) / W);
  return launch_pdl(k, grid, SM::THREADS, smem, stream, xmap, cmap, n, norms, p, fs);
}

template <typename T>
cudaError_t launch_encode_mma(const T* x, int64_t n, const QuantParams& p, uint8_t* codes,
                               float* norms, cudaStream_t stream) {
  const FixedSearch fs = make_fixed_search(p);
  if (!fs.ok) return cudaErrorNotSupported;
  int dev = 0, reserved = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
      uint32_t(reserved) != EncMma<12, 1, 2>::kBase)
    return cudaErrorNotSupported;
  CUtensorMap xmap, cmap;
  if (!row_tensor_map(&xmap, x, n, 128, 2, 32)) return cudaErrorNotSupported;
  if (!code_tensor_map(&cmap, codes, n, 64, 32)) return cudaErrorNotSupported;
  return launch_encode_mma_v<T, 12, 1, 2, false>(xmap, cmap, n, p, fs, norms, stream);
}

}  // namespace rrq

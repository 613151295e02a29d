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
// tables, 128 packed butterfly operations and the code search, against 64 sign
// XORs, 192 conversion-and-first-stage operations and 384 packed butterfly
// operations of the one-lane-per-vector kernel (batch_kernels.cuh), whose
// staging, code search and output this kernel keeps:
//  * inputs arrive as TMA tensor boxes (32 rows × 128 bytes, 128-byte swizzle,
//    two stages per warp, zero fill past the end);
//  * ν² = ‖y'‖²/d from the thread's 32 values per row and two quad shuffles;
//    each thread of a quad computes ν and A/ν of one of its 4 rows and shares
//    A/ν by shuffles;
//  * the cell table decides each code (code = lo + (s > thr), s = sat(u·A + 1/2));
//  * codes go to a per-warp 32 × 64-byte tile in the 64-byte swizzle (the
//    quad-strided word stores are conflict-free in it) and leave in one TMA
//    tensor store per batch, which clips rows past the end.
#pragma once

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

template <typename T, int WARPS_ = 8, int NS_ = 2> struct EncMma {
  static constexpr int D = 128, NB = D / 32;   // four 32-coordinate blocks
  static constexpr int ROW = D * 2;            // input row bytes
  static constexpr int BOXES = ROW / 128;      // 128-byte boxes per row
  static constexpr int NS = NS_;               // input stages per warp
  static constexpr int CB = D / 2;             // code bytes per vector (4-bit codes)
  static constexpr int STAGE = 32 * ROW;       // 1024-aligned
  static constexpr int CTILE = 32 * CB;        // one batch of codes, 64-byte swizzle
  static constexpr int WARP_BYTES = (NS * STAGE + 2 * CTILE + 1023) / 1024 * 1024;
  static constexpr int TABLE = (kMaxCells + 1) * 32 * 8;  // lane-replicated (thr, lo) pairs
  static constexpr int HROW = 80;              // bytes per row of a block table (64 + 16 padding)
  static constexpr int HTAB = NB * 32 * HROW;  // B_a^T, rows n, 32 columns k each
  static constexpr int SIGNS = D;              // one byte per coordinate (set-up only)
  static constexpr int WARPS = WARPS_;
  static constexpr int THREADS = WARPS * 32;
  static constexpr int BARS = WARPS * NS * 8;
  static constexpr int HEAD = (TABLE + HTAB + SIGNS + BARS + 1023) / 1024 * 1024;
  // + 1024: the dynamic shared memory base is rounded up to a 1024-byte boundary
  static constexpr size_t total() { return 1024 + size_t(HEAD) + size_t(WARPS) * WARP_BYTES; }
  static_assert(total() <= 227 * 1024, "shared memory");
};

template <typename T, int WARPS_ = 8, int NS_ = 2>
__global__ void __launch_bounds__(EncMma<T, WARPS_, NS_>::THREADS, 1)
encode_mma_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap cmap,
                  int64_t n, float* __restrict__ norms, const QuantParams p) {
  using SM = EncMma<T, WARPS_, NS_>;
  constexpr int NB = SM::NB, NS = SM::NS;
  pdl_release();
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = dsm_raw + ((1024u - (smem_addr(dsm_raw) & 1023u)) & 1023u);
  float2* tab = reinterpret_cast<float2*>(dsm);
  uint8_t* htab = dsm + SM::TABLE;
  uint8_t* signs = htab + SM::HTAB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(signs + SM::SIGNS);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* wmem = dsm + SM::HEAD + warp * SM::WARP_BYTES;

  const int N = p.cell.cells;
  for (int i = threadIdx.x; i < (N + 1) * 32; i += blockDim.x)
    tab[i] = make_float2(p.cell.thr[i >> 5], __uint_as_float(p.cell.lo[i >> 5]));
  for (int i = threadIdx.x; i < SM::D; i += blockDim.x) signs[i] = uint8_t(sign_bit(p.seed, i));
  if (lane == 0) {
    for (int s = 0; s < NS; ++s) mbarrier_init(smem_addr(&bars[warp * NS + s]), 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  // B_a^T[n][k] = s_{32a+k}·H_32[π(n), k], π swapping bit fields 1–2 and 3–4 of n
  for (int i = threadIdx.x; i < NB * 32 * 32; i += blockDim.x) {
    const int k = i & 31, nn = (i >> 5) & 31, a = i >> 10;
    const int pn = (nn & 1) | (((nn >> 3) & 3) << 1) | (((nn >> 1) & 3) << 3);
    const int neg = (signs[32 * a + k] ^ __popc(pn & k)) & 1;
    reinterpret_cast<uint16_t*>(htab + (a * 32 + nn) * SM::HROW)[k] =
        neg ? MmaType<T>::kMinusOne : MmaType<T>::kOne;
  }
  __syncthreads();
  pdl_wait();  // the shared tables are built: from here on, global memory

  const int64_t nb = (n + 31) >> 5;
  const int64_t tw = int64_t(gridDim.x) * SM::WARPS;
  // warp-major numbering: every SM gets the same number of batches (±1)
  const int64_t gw = int64_t(warp) * gridDim.x + blockIdx.x;
  const uint32_t bar0 = smem_addr(&bars[warp * NS]);
  const uint32_t stage0 = smem_addr(wmem);
  const uint32_t tab_lane = smem_addr(tab) + lane * 8;
  const uint32_t ctile0 = smem_addr(wmem + NS * SM::STAGE);
  const int qr = lane >> 2, qc = lane & 3;
  // ldmatrix row addresses: A rows 16mt + (l mod 8) + 8·bit3(l), 16-byte column
  // chunk bit4(l); table rows 8nt + (l mod 8), 16-byte column chunk l / 8
  const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8, a_chunk = lane >> 4;
  const uint32_t h_lane = smem_addr(htab) + uint32_t((lane & 7) * SM::HROW + (lane >> 3) * 16);
  uint32_t pending = 0;  // bit s: a load into stage s is in flight

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
#pragma unroll
  for (int s = 0; s < NS; ++s) issue(s, gw + s * tw);

  const float Nf = float(N);
  const float A = p.cell.a;
  uint32_t parity = 0;
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

    // z[a] = X_a · B_a on m16n8k16 tiles: acc[a][mt][nt] covers rows
    // 16mt + {qr, qr + 8}, columns 8nt + 2qc + {0, 1} of block a
    float acc[NB][2][4][4];
    const uint32_t st = stage0 + s * SM::STAGE;
#pragma unroll
    for (int a = 0; a < NB; ++a) {
      uint32_t bf[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) ldsm_x4(bf[nt], h_lane + uint32_t((a * 32 + 8 * nt) * SM::HROW));
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) acc[a][mt][nt][0] = acc[a][mt][nt][1] = acc[a][mt][nt][2] = acc[a][mt][nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const int colb = 64 * a + 32 * ks + 16 * a_chunk;  // byte within the 256-byte row
          uint32_t af[4];
          ldsm_x4(af, st + (colb >> 7) * 4096 + swz128(16 * mt + a_row, (colb & 127) >> 4));
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) mma_t<T>(acc[a][mt][nt], af, bf[nt][2 * ks], bf[nt][2 * ks + 1]);
        }
      }
    }
    __syncwarp();  // every lane's fragments are in registers: the stage may be refilled
    fence_proxy_async_smem();
    issue(s, b + NS * tw);

    // y'[32a + b] = Σ_a' H_4[a, a']·z[a', b] on packed pairs, and ν² per row:
    // row index r = h + 2mt is row qr + 8r of the batch
    float2 y[NB][2][4][2];
    float2 q2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                    make_float2(0.f, 0.f)};
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float2 z[NB];
#pragma unroll
          for (int a = 0; a < NB; ++a) z[a] = make_float2(acc[a][mt][nt][2 * h], acc[a][mt][nt][2 * h + 1]);
#pragma unroll
          for (int m = 1; m < NB; m <<= 1)
#pragma unroll
            for (int a = 0; a < NB; ++a)
              if ((a & m) == 0) {
                const float2 u = z[a], v = z[a | m];
                z[a] = add2(u, v);
                z[a | m] = sub2(u, v);
              }
#pragma unroll
          for (int a = 0; a < NB; ++a) {
            y[a][mt][nt][h] = z[a];
            q2[h + 2 * mt] = fma2(z[a], z[a], q2[h + 2 * mt]);
          }
        }
    float ss[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      ss[r] = q2[r].x + q2[r].y;
      ss[r] += __shfl_xor_sync(kFull, ss[r], 1);
      ss[r] += __shfl_xor_sync(kFull, ss[r], 2);
    }
    // thread qc of the quad: ν and A/ν of row qr + 8qc (‖y'‖² = d·‖x‖²)
    const float my_ss = qc == 0 ? ss[0] : qc == 1 ? ss[1] : qc == 2 ? ss[2] : ss[3];
    const float nu = sqrtf(my_ss * p.inv_d);
    const float my_sc = nu > 0.f ? __fdiv_rn(A, nu) : 0.f;  // s = sat(y'·A/ν + 1/2)
    float sc[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) sc[r] = __shfl_sync(kFull, my_sc, (lane & ~3) | r);

    // codes: row qr + 8r, word 4a + qc holds coordinates 32a + 8qc + [0, 8)
    if (lane == 0) bulk_wait_read_1();  // the store from this tile two batches ago has read it
    __syncwarp();
    const uint32_t tile = ctile0 + ct * SM::CTILE;
    const uint32_t swz = uint32_t((qr >> 1) & 3);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = h + 2 * mt;
        const float scr = sc[r];
#pragma unroll
        for (int a = 0; a < NB; ++a) {
          uint32_t word = 0;
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            const float2 v = y[a][mt][nt][h];
            const float sx = __saturatef(fmaf(v.x, scr, 0.5f));
            const float sy = __saturatef(fmaf(v.y, scr, 0.5f));
            const float2 f = fma2(make_float2(sx, sy), make_float2(Nf, Nf), make_float2(8388608.f, 8388608.f));
            // the float bits are 0x4B000000 + round(s·N); ·256 drops the exponent
            const float2 ex = lds_f2(tab_lane + (__float_as_uint(f.x) << 8));
            const float2 ey = lds_f2(tab_lane + (__float_as_uint(f.y) << 8));
            const uint32_t cx = __float_as_uint(ex.y) + (sx > ex.x ? 1u : 0u);
            const uint32_t cy = __float_as_uint(ey.y) + (sy > ey.x ? 1u : 0u);
            word |= (cx + (cy << 4)) << (8 * nt);
          }
          const int row = qr + 8 * r;
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(tile + uint32_t(row * 64) + ((uint32_t(a) ^ swz) << 4) +
                                                           uint32_t(qc * 4)),
                       "r"(word)
                       : "memory");
        }
      }
    if (v0 + qr + 8 * qc < n) norms[v0 + qr + 8 * qc] = nu;
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(&cmap, 0, int(v0), tile);
      bulk_commit();
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
// another encoder).
template <typename T>
cudaError_t launch_encode_mma(const T* x, int64_t n, const QuantParams& p, uint8_t* codes,
                              float* norms, cudaStream_t stream) {
  using SM = EncMma<T>;
  CUtensorMap xmap, cmap;
  if (!row_tensor_map(&xmap, x, n, SM::D, 2, 32)) return cudaErrorNotSupported;
  if (!code_tensor_map(&cmap, codes, n, SM::CB, 32)) return cudaErrorNotSupported;
  auto k = encode_mma_kernel<T>;
  constexpr size_t smem = SM::total();
  const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int64_t batches = (n + 31) / 32;
  const int grid = grid_for(reinterpret_cast<const void*>(k), SM::THREADS, smem,
                            (batches + SM::WARPS - 1) / SM::WARPS);
  return launch_pdl(k, grid, SM::THREADS, smem, stream, xmap, cmap, n, norms, p);
}

}  // namespace rrq

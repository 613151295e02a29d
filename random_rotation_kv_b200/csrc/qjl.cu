// qjl.cu — MSE encode fused with the QJL 1-bit sketch of the residual, with
// the d×d projection on the 5th-generation tensor cores (tcgen05).
//
// "Random-rotation quantization" page, "History": QJL — a DRIVE-style one-bit
// construction for attention keys made unbiased through residuals;
// TurboQuant — a (b−1)-bit biased MSE quantiser followed by an unbiased 1-bit
// one.  "Bias vs unbiasedness": the residual chain removes the MSE shrinkage.
// For each vector:
//     r = Πx − ŷ (rotated domain, ŷ = (ν/√d)·c[code]),  ρ = ‖r‖₂,
//     v = S·r (S: d×d, bf16-valued Gaussian),  bit_i = [v_i > 0].
//
// Two kernels.  For 16-bit inputs (the usual case) `qjl_batch_kernel` below:
// two 4-warp groups per CTA with their own tiles, TMA-staged inputs, the
// batch encoder's arithmetic, and the residual in two fp16 parts (two MMA
// passes).  For fp32 inputs, or codebooks the cell table cannot hold, the
// one-group kernel described here:
//
// Tile of 128 vectors per CTA iteration (one thread per vector, d = 128):
//  1. the input tile arrives by cp.async in padded shared rows (prefetched one
//     tile ahead);
//  2. each thread runs the MSE encoder on its vector (codes and ν to global
//     memory), forms r in fp32 and splits it exactly into three bf16 parts
//     r = r_hi + r_mid + r_lo (8 significant bits each: together the 24 of
//     fp32), written into three A operand tiles [128 × 128] (K-major, no
//     swizzle: 8×16-byte core matrices);
//  3. one thread issues 3 × 8 tcgen05.mma (M = 128, N = 128, K = 16,
//     bf16 × bf16 → fp32) against S (B operand, resident for the whole
//     kernel), accumulating V = R·Sᵀ in tensor memory; products are exact and
//     only the fp32 accumulation rounds;
//  4. tcgen05.commit arrives on an mbarrier; each warp reads its 32 TMEM lanes
//     (one lane = one vector's 128 outputs) and packs the signs.
// Every wait is bounded; on a timeout the tile's residual norms are set to
// NaN, the CTA drains its copies, frees its tensor memory and returns.
#include <cstring>

#include "batch_kernels.cuh"
#include "qjl_tc.cuh"
#include "tcgen05.cuh"

namespace rrq {
namespace {

constexpr int kQjlD = 128;
constexpr int kQjlTile = 128;
constexpr int kQjlThreads = 128;
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kWaitLimit = 1u << 24;  // try_wait polls before giving up

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major,
// N = 128 (bits 17..22 = N/8), M = 128 (bits 24..28 = M/16).
constexpr uint32_t kIdescBf16M128N128 =
    (1u << 4) | (1u << 7) | (1u << 10) | ((128u / 8) << 17) | ((128u / 16) << 24);

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kIdescBf16M128N128), "r"(accumulate)
      : "memory");
}
// Byte offset of element (row, k) in a [128 × 128] bf16 K-major core-matrix tile.
constexpr uint32_t kLbo = 128;   // next 8 k
constexpr uint32_t kSbo = 2048;  // next 8 rows
__device__ __forceinline__ uint32_t cm_offset(int row, int kb) {  // kb = k/8, 16-byte chunk
  return uint32_t(row >> 3) * kSbo + uint32_t(kb) * kLbo + uint32_t(row & 7) * 16;
}

template <typename T>
struct QjlSmem {
  static constexpr int ROWB = kQjlD * Elem<T>::kBytes;       // input row bytes
  static constexpr int ROWP = ROWB + 16;                      // padded
  static constexpr int STAGES = Elem<T>::kBytes == 2 ? 2 : 1;
  static constexpr int OPER = kQjlTile * kQjlD * 2;          // one bf16 operand tile (32 KB)
  static constexpr int S_OFF = 0;
  static constexpr int A_OFF = S_OFF + OPER;                  // 3 parts
  static constexpr int IN_OFF = A_OFF + 3 * OPER;
  static constexpr int IN_BYTES = STAGES * kQjlTile * ROWP;
  static constexpr int TOTAL = IN_OFF + IN_BYTES;
};

struct QjlArgs {
  CUtensorMap xmap;  // 16-bit inputs, two-group kernel: boxes of 64 elements × 128 rows
  const void* x;
  int64_t n;
  const uint16_t* S;  // bf16 bits [128][128]
  uint8_t* codes;
  float* norms;
  uint8_t* qbits;
  float* rnorm;
  QuantParams p;
};

template <typename T, int B, bool SYM>
__global__ void __launch_bounds__(kQjlThreads, 1) qjl_encode_kernel(const QjlArgs a) {
  pdl_release();
  pdl_wait();  // the prologue reads S: wait for the previous kernel first
  using Sm = QjlSmem<T>;
  constexpr int D = kQjlD, P = D / 2, SEC = D / 16, L = 1 << B, CB = D * B / 8;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(16) uint32_t smask[mask_words<T, D>()];
  __shared__ float slev[L];
  __shared__ __align__(8) uint64_t mbar;
  __shared__ uint32_t tmem_base;
  __shared__ int tile_ok;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const QuantParams& p = a.p;
  const T* x = static_cast<const T*>(a.x);
  build_sign_mask<T, D>(smask, p.seed);
  if (tid < L) slev[tid] = p.levels[tid];
  // S -> B operand tile (core-matrix layout), 16-byte chunks
  for (int c = tid; c < kQjlD * 16; c += kQjlThreads) {
    const int row = c >> 4, kb = c & 15;
    const uint4 v = *reinterpret_cast<const uint4*>(a.S + row * kQjlD + kb * 8);
    *reinterpret_cast<uint4*>(smem + Sm::S_OFF + cm_offset(row, kb)) = v;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(&tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) mbar_init(&mbar, 1);
  fence_proxy_async_smem();  // S tile and barrier visible to the async proxy
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  const int64_t ntiles = (a.n + kQjlTile - 1) / kQjlTile;
  // input tile t -> stage: 128 rows, 16-byte units, coalesced, padded rows
  auto issue = [&](int stage, int64_t t) {
    uint8_t* st = smem + Sm::IN_OFF + stage * kQjlTile * Sm::ROWP;
    constexpr int UPR = Sm::ROWB / 16;  // units per row
    for (int u = tid; u < kQjlTile * UPR; u += kQjlThreads) {
      const int row = u / UPR, c = u % UPR;
      const int64_t v = t * kQjlTile + row;
      const bool ok = t < ntiles && v < a.n;
      const uint8_t* src = static_cast<const uint8_t*>(a.x) + (ok ? v * Sm::ROWB + c * 16 : 0);
      cp_async16(smem_addr(st + row * Sm::ROWP + c * 16), src, ok ? 16 : 0);
    }
  };
  int64_t t = blockIdx.x;
  if constexpr (Sm::STAGES == 2) issue(0, t);
  cp_async_commit();
  uint32_t phase = 0;
  bool failed = false;
  for (int it = 0; t < ntiles; ++it, t += gridDim.x) {
    const int stage = Sm::STAGES == 2 ? (it & 1) : 0;
    if constexpr (Sm::STAGES == 2) {
      issue(stage ^ 1, t + gridDim.x);  // next tile, in flight now
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      issue(0, t);
      cp_async_commit();
      cp_async_wait<0>();
    }
    __syncthreads();

    // ---- MSE encode of vector `vec` by this thread
    const int64_t vec = t * kQjlTile + tid;
    const bool valid = vec < a.n;
    const uint8_t* row = smem + Sm::IN_OFF + stage * kQjlTile * Sm::ROWP + tid * Sm::ROWP;
    float2 w[P];
#pragma unroll
    for (int s = 0; s < SEC; ++s) {
      uint32_t raw[sector_words<T>()];
#pragma unroll
      for (int c = 0; c < sector_words<T>() / 4; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + s * 16 * Elem<T>::kBytes + c * 16);
        raw[4 * c] = v.x; raw[4 * c + 1] = v.y; raw[4 * c + 2] = v.z; raw[4 * c + 3] = v.w;
      }
      sector_to_pairs<T, true>(raw, smask + s * sector_words<T>(), &w[s * 8]);
    }
    float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < P; ++k) ss2 = fma2(w[k], w[k], ss2);
    const float nu = sqrtf(ss2.x + ss2.y);
    fwht2<D, D>(w, 0);
    const float ns = nu > 0.f ? nu : 1.f;
    uint64_t sec[SEC];
    {
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
    {
      uint32_t words[CB / 4];
#pragma unroll
      for (int i = 0; i < CB / 4; ++i) words[i] = 0u;
#pragma unroll
      for (int s = 0; s < SEC; ++s) {  // sector s at bit s·16B
        const int pos = s * 16 * B, wi = pos / 32, off = pos % 32;
        words[wi] |= uint32_t(sec[s] << off);
        if (off + 16 * B > 32) words[wi + 1] |= uint32_t(sec[s] >> (32 - off));
        if (off + 16 * B > 64) words[wi + 2] |= uint32_t(sec[s] >> (64 - off));
      }
      if (valid) {
        store_bytes<CB>(a.codes + vec * CB, words);
        a.norms[vec] = nu;
      }
    }

    // ---- residual r = (y' − ν·c[code])/√d, split into three bf16 parts
    float rr = 0.f;
#pragma unroll
    for (int s = 0; s < SEC; ++s) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {  // 8 values = one 16-byte chunk per part
        uint32_t hi[4], mid[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int e = half * 8 + 2 * j;  // value index within the sector
          const uint32_t c0 = uint32_t(sec[s] >> (e * B)) & (L - 1);
          const uint32_t c1 = uint32_t(sec[s] >> ((e + 1) * B)) & (L - 1);
          const float2 y = w[s * 8 + half * 4 + j];
          float r0 = (y.x - nu * slev[c0]) * p.inv_sqrt_d;
          float r1 = (y.y - nu * slev[c1]) * p.inv_sqrt_d;
          if (!valid) { r0 = 0.f; r1 = 0.f; }
          rr = fmaf(r0, r0, fmaf(r1, r1, rr));
          const __nv_bfloat162 h = __floats2bfloat162_rn(r0, r1);
          const float2 hf = __bfloat1622float2(h);
          const float m0 = r0 - hf.x, m1 = r1 - hf.y;  // exact
          const __nv_bfloat162 md = __floats2bfloat162_rn(m0, m1);
          const float2 mf = __bfloat1622float2(md);
          const __nv_bfloat162 l = __floats2bfloat162_rn(m0 - mf.x, m1 - mf.y);  // exact
          hi[j] = *reinterpret_cast<const uint32_t*>(&h);
          mid[j] = *reinterpret_cast<const uint32_t*>(&md);
          lo[j] = *reinterpret_cast<const uint32_t*>(&l);
        }
        const uint32_t off = cm_offset(tid, s * 2 + half);
        *reinterpret_cast<uint4*>(smem + Sm::A_OFF + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(smem + Sm::A_OFF + Sm::OPER + off) =
            make_uint4(mid[0], mid[1], mid[2], mid[3]);
        *reinterpret_cast<uint4*>(smem + Sm::A_OFF + 2 * Sm::OPER + off) =
            make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    const float rho = sqrtf(rr);

    // ---- V = R·Sᵀ on the tensor cores
    fence_proxy_async_smem();  // A tiles visible to the tensor cores
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t s_base = smem_addr(smem + Sm::S_OFF);
      uint32_t acc = 0;
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        const uint32_t a_base = smem_addr(smem + Sm::A_OFF + part * Sm::OPER);
#pragma unroll
        for (int ks = 0; ks < kQjlD / 16; ++ks) {
          mma_bf16(tmem, smem_desc(a_base + ks * 2 * kLbo, kLbo, kSbo),
                   smem_desc(s_base + ks * 2 * kLbo, kLbo, kSbo), acc);
          acc = 1;
        }
      }
      mma_commit(&mbar);
      bool ok = false;
      for (uint32_t i = 0; i < kWaitLimit && !ok; ++i) ok = mbar_try_wait(&mbar, phase);
      tile_ok = ok ? 1 : 0;
    }
    __syncthreads();
    phase ^= 1u;
    if (!tile_ok) {
      if (valid) a.rnorm[vec] = __int_as_float(0x7fc00000);  // NaN marks the failure
      failed = true;
      break;
    }
    tc_fence_after();

    // ---- signs: warp w reads TMEM lanes 32w..32w+31 (this thread's vector)
    uint32_t bits[4];
#pragma unroll
    for (int cchunk = 0; cchunk < 4; ++cchunk) {
      uint32_t v[32];
      tmem_ld32(tmem + (uint32_t(warp * 32) << 16) + uint32_t(cchunk * 32), v);
      tmem_ld_wait();
      uint32_t b = 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) b |= (__uint_as_float(v[j]) > 0.f ? 1u : 0u) << j;
      bits[cchunk] = b;
    }
    if (valid) {
      reinterpret_cast<uint4*>(a.qbits + vec * (kQjlD / 8))[0] = make_uint4(bits[0], bits[1], bits[2], bits[3]);
      a.rnorm[vec] = rho;
    }
    tc_fence_before();
    __syncthreads();  // TMEM read and A tiles free before the next tile
  }
  cp_async_wait<0>();
  tc_fence_before();
  __syncthreads();
  (void)failed;
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------- two-group kernel (16-bit x)
// Two groups of 4 warps per CTA, each with its own 128-vector tiles, input
// stage, A operands and 128 TMEM columns, so one group's tensor-core work
// overlaps the other's CUDA-core work.  The CUDA-core part is the batch
// encoder's (first butterfly from the 16-bit elements, packed fp32 stages,
// cell-table code search).  The residual is scaled per vector by a power of
// two (signs of S·r do not change) into [−2¹⁰, 2¹⁰] and split exactly enough
// into two fp16 parts r = r_hi + r_lo (22 significant bits); S is taken in
// fp16, rounded from bf16, which moves no entry by more than 2⁻²⁵.  Each part
// error bounds |Δ(S·r)_i| well below 10⁻⁵·ρ.  Two fp16 MMAs per K-step.
constexpr int kQ2Groups = 2;
constexpr int kQ2Threads = kQ2Groups * kQjlTile;  // 256
constexpr uint32_t kQ2TmemCols = 256;
constexpr int kQ2MaxCells = 32;                    // cell table copies fit for N ≤ 32

// Instruction descriptor, kind::f16: D fp32, A and B fp16, K-major, M = N = 128.
constexpr uint32_t kIdescF16M128N128 = (1u << 4) | ((128u / 8) << 17) | ((128u / 16) << 24);

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kIdescF16M128N128), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "r"(kQjlTile) : "memory");
}

struct Qjl2Smem {
  static constexpr int IN = kQjlTile * kQjlD * 2;            // one group's input tile: 2 swizzled boxes
  static constexpr int OPER = kQjlTile * kQjlD * 2;          // one fp16 operand tile
  static constexpr int IN_OFF = 0;
  static constexpr int S_OFF = IN_OFF + kQ2Groups * IN;
  static constexpr int A_OFF = S_OFF + OPER;                 // [group][part]
  static constexpr int TAB_OFF = A_OFF + kQ2Groups * 2 * OPER;
  static constexpr int TAB = (kQ2MaxCells + 1) * 64;        // 8 copies × 8 bytes per cell
  static constexpr int MASK_OFF = TAB_OFF + TAB;
  static constexpr int LEV_OFF = MASK_OFF + kQjlD / 2 * 4;
  static constexpr int BAR_OFF = LEV_OFF + kMaxLevels * 4;   // barriers, tmem base, flags
  static constexpr int TOTAL = BAR_OFF + 64;
  static_assert(TOTAL <= 227 * 1024, "shared memory");
};

template <typename T, int B>
__global__ void __launch_bounds__(kQ2Threads, 1) qjl_batch_kernel(const __grid_constant__ QjlArgs a) {
  pdl_release();
  pdl_wait();  // the prologue reads S: wait for the previous kernel first
  using Sm = Qjl2Smem;
  constexpr int D = kQjlD, P = D / 2, CB = D * B / 8, NW = (CB + 3) / 4;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint32_t* smask = reinterpret_cast<uint32_t*>(smem + Sm::MASK_OFF);
  float* slev = reinterpret_cast<float*>(smem + Sm::LEV_OFF);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + Sm::BAR_OFF);       // MMA done [group]
  uint64_t* ibar = reinterpret_cast<uint64_t*>(smem + Sm::BAR_OFF + 16);  // input landed [group]
  uint32_t* tmem_base = reinterpret_cast<uint32_t*>(smem + Sm::BAR_OFF + 32);
  int* tile_ok = reinterpret_cast<int*>(smem + Sm::BAR_OFF + 40);         // [group]
  int* in_ok = reinterpret_cast<int*>(smem + Sm::BAR_OFF + 48);           // [group]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = tid / kQjlTile, gt = tid % kQjlTile;  // group, vector row in the tile
  const QuantParams& p = a.p;
  const uint8_t* xb = static_cast<const uint8_t*>(a.x);
  constexpr int ROWB = D * 2;

  // ---- prologue: sign mask, levels, cell table (8 copies), S in fp16, TMEM, barriers
  build_sign_mask<T, D>(smask, p.seed);
  if (tid < kMaxLevels) slev[tid] = p.levels[tid];
  const int N = p.cell.cells;
  for (int i = tid; i < (N + 1) * 8; i += kQ2Threads)
    reinterpret_cast<float2*>(smem + Sm::TAB_OFF)[i] =
        make_float2(p.cell.thr[i >> 3], __uint_as_float(p.cell.lo[i >> 3]));
  for (int c = tid; c < D * 16; c += kQ2Threads) {  // S row r, 8 elements per chunk
    const int row = c >> 4, kb = c & 15;
    const uint4 v = *reinterpret_cast<const uint4*>(a.S + row * D + kb * 8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2 h = __floats2half2_rn(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xffff0000u));
      o[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(smem + Sm::S_OFF + cm_offset(row, kb)) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_base)),
                 "r"(kQ2TmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid < kQ2Groups) {
    mbar_init(&mbar[tid], 1);
    mbar_init(&ibar[tid], 1);
    fence_mbarrier_init();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base + uint32_t(g * kQjlTile);  // this group's 128 columns

  // ---- tiles of this group: warp-major over the grid, so SMs get equal counts
  const int64_t ntiles = (a.n + kQjlTile - 1) / kQjlTile;
  const int64_t tstride = int64_t(gridDim.x) * kQ2Groups;
  uint8_t* in = smem + Sm::IN_OFF + g * Sm::IN;
  // this group's input tile t: two TMA boxes (columns 0..63, 64..127) of 128 rows;
  // rows past the end arrive as zeros and count toward the transaction bytes
  auto issue = [&](int64_t t) {
    if (t < ntiles && gt == 0) {
      fence_proxy_async_smem();
      mbarrier_expect_tx(smem_addr(&ibar[g]), Sm::IN);
#pragma unroll
      for (int h = 0; h < 2; ++h)
        tma_load_2d(smem_addr(in + h * (Sm::IN / 2)), &a.xmap, h * 64, int(t * kQjlTile), smem_addr(&ibar[g]));
    }
  };
  // cell j, copy (lane & 7) at TAB + j·64 + (lane & 7)·8.  The index arrives as the
  // float bits 0x4B000000 + j; (bits << 6) keeps 0x4B000000 << 6 ≡ 0xC0000000
  // (mod 2³²) of the exponent, which the base takes off again.
  const uint32_t tab_lane = smem_addr(smem + Sm::TAB_OFF) + uint32_t(lane & 7) * 8u - (0x4B000000u << 6);
  const float Nf = float(N), A = p.cell.a;
  const uint32_t a_hi = smem_addr(smem + Sm::A_OFF + (g * 2 + 0) * Sm::OPER);
  const uint32_t a_lo = smem_addr(smem + Sm::A_OFF + (g * 2 + 1) * Sm::OPER);
  const uint32_t s_base = smem_addr(smem + Sm::S_OFF);
  // level bound for the residual scale: |r_i| ≤ ν·(1 + max|c|/√d)
  float cmax = 0.f;
#pragma unroll
  for (int k = 0; k < kMaxLevels; ++k)
    if (k < (1 << B)) cmax = fmaxf(cmax, fabsf(p.levels[k]));
  const float rbound = 1.f + cmax * p.inv_sqrt_d;

  uint32_t phase = 0, iphase = 0;
  int64_t t = int64_t(g) * gridDim.x + blockIdx.x;
  bool pending = t < ntiles;  // an input copy of this group is in flight
  issue(t);
  for (; t < ntiles; t += tstride) {
    // one thread waits (bounded) and tells the group, so all threads agree
    if (gt == 0) in_ok[g] = mbarrier_wait(smem_addr(&ibar[g]), iphase) ? 1 : 0;
    group_sync(g);  // the tile is in shared memory for every thread of the group
    iphase ^= 1u;
    const int64_t vec = t * kQjlTile + gt;
    const bool valid = vec < a.n;
    if (!in_ok[g]) {
      if (valid) a.rnorm[vec] = __int_as_float(0x7fc00000);  // NaN marks the failure
      break;
    }
    pending = false;

    float2 w[P];
#pragma unroll
    for (int c = 0; c < ROWB / 16; ++c) {
      const uint4 r = *reinterpret_cast<const uint4*>(in + (c >> 3) * (Sm::IN / 2) + swz128(gt, c & 7));
      const uint4 m = reinterpret_cast<const uint4*>(smask)[c];
      w[4 * c + 0] = first_butterfly<T>(r.x ^ m.x);
      w[4 * c + 1] = first_butterfly<T>(r.y ^ m.y);
      w[4 * c + 2] = first_butterfly<T>(r.z ^ m.z);
      w[4 * c + 3] = first_butterfly<T>(r.w ^ m.w);
    }
    group_sync(g);  // every row read: the stage may be refilled
    issue(t + tstride);
    pending = t + tstride < ntiles;

    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                     make_float2(0.f, 0.f)};
#pragma unroll
    for (int k = 0; k < P; ++k) acc[k & 3] = fma2(w[k], w[k], acc[k & 3]);
    const float2 a4 = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
    const float nu = sqrtf(0.5f * (a4.x + a4.y));
#pragma unroll
    for (int mm = 1; mm < P; mm <<= 1) {
#pragma unroll
      for (int k = 0; k < P; ++k) {
        if ((k & mm) == 0) {
          const float2 x0 = w[k], x1 = w[k | mm];
          w[k] = add2(x0, x1);
          w[k | mm] = sub2(x0, x1);
        }
      }
    }

    // codes (cell table) and the scaled residual rs = (y' − ν·c)·sc/√d, split in fp16
    const float scs = nu > 0.f ? __fdiv_rn(A, nu) : 0.f;
    int ex = 0;
    frexpf(nu * rbound, &ex);
    const float sc = nu > 0.f ? ldexpf(1.f, 10 - max(ex, -100)) : 1.f;  // |rs| ≤ 2^10
    const float k1 = sc * p.inv_sqrt_d, k2 = nu * k1;
    uint32_t words[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) words[i] = 0u;
    float2 rr2 = make_float2(0.f, 0.f);
    const float2 k1x2 = make_float2(k1, k1), nk2x2 = make_float2(-k2, -k2);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {  // 8 coordinates = one 16-byte chunk per part
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = 4 * c + j;
        const float sx = __saturatef(fmaf(w[k].x, scs, 0.5f));
        const float sy = __saturatef(fmaf(w[k].y, scs, 0.5f));
        const float2 f = fma2(make_float2(sx, sy), make_float2(Nf, Nf), make_float2(8388608.f, 8388608.f));
        const float2 ex0 = lds_f2(tab_lane + (__float_as_uint(f.x) << 6));
        const float2 ey0 = lds_f2(tab_lane + (__float_as_uint(f.y) << 6));
        const uint32_t cx = __float_as_uint(ex0.y) + (sx > ex0.x ? 1u : 0u);
        const uint32_t cy = __float_as_uint(ey0.y) + (sy > ey0.x ? 1u : 0u);
        put_code<B>(words, 2 * k, cx);
        put_code<B>(words, 2 * k + 1, cy);
        // rows past n arrive zero-filled with ν = 0, so their residual is 0
        const float2 r = fma2(w[k], k1x2, mul2(make_float2(slev[cx], slev[cy]), nk2x2));
        rr2 = fma2(r, r, rr2);
        const __half2 h = __float22half2_rn(r);
        const __half2 l = __float22half2_rn(sub2(r, __half22float2(h)));
        hi[j] = *reinterpret_cast<const uint32_t*>(&h);
        lo[j] = *reinterpret_cast<const uint32_t*>(&l);
      }
      const uint32_t off = cm_offset(gt, c);
      *reinterpret_cast<uint4*>(smem + Sm::A_OFF + (g * 2 + 0) * Sm::OPER + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(smem + Sm::A_OFF + (g * 2 + 1) * Sm::OPER + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    if (valid) {
      store_bytes<CB>(a.codes + vec * CB, words);
      a.norms[vec] = nu;
    }
    const float rho = sqrtf(rr2.x + rr2.y) / sc;  // ‖r‖ from the scaled residual

    // ---- V = R·Sᵀ on the tensor cores (one thread of the group issues)
    fence_proxy_async_smem();  // A tiles visible to the tensor cores
    tc_fence_before();
    group_sync(g);
    if (gt == 0) {
      tc_fence_after();
      uint32_t accf = 0;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t ab = part == 0 ? a_hi : a_lo;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          mma_f16(tmem, smem_desc(ab + ks * 2 * kLbo, kLbo, kSbo), smem_desc(s_base + ks * 2 * kLbo, kLbo, kSbo), accf);
          accf = 1;
        }
      }
      mma_commit(&mbar[g]);
      bool ok = false;
      for (uint32_t i = 0; i < kWaitLimit && !ok; ++i) ok = mbar_try_wait(&mbar[g], phase);
      tile_ok[g] = ok ? 1 : 0;
    }
    group_sync(g);
    phase ^= 1u;
    if (!tile_ok[g]) {
      if (valid) a.rnorm[vec] = __int_as_float(0x7fc00000);  // NaN marks the failure
      break;
    }
    tc_fence_after();

    // ---- signs: each warp reads its 32 TMEM lanes (its vectors), 4 × 32 columns
    uint32_t bits[4];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t v[32];
      tmem_ld32(tmem + (uint32_t((warp & 3) * 32) << 16) + uint32_t(cc * 32), v);
      tmem_ld_wait();
      // bit j = [v_j > 0] from the sign bits (an exact +0 only arises with r = 0,
      // handled below; elsewhere it lies far inside the sign exemption band)
      uint32_t neg = 0;
#pragma unroll
      for (int j = 31; j >= 0; --j) neg = (neg << 1) | (v[j] >> 31);
      bits[cc] = rho > 0.f ? ~neg : 0u;
    }
    if (valid) {
      reinterpret_cast<uint4*>(a.qbits + vec * (D / 8))[0] = make_uint4(bits[0], bits[1], bits[2], bits[3]);
      a.rnorm[vec] = rho;
    }
    tc_fence_before();  // TMEM reads done before the next MMA of this group
  }
  // after a failure: wait (bounded) for an input copy still in flight
  if (pending && gt == 0) mbarrier_wait(smem_addr(&ibar[g]), iphase);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(*tmem_base), "r"(kQ2TmemCols)
                 : "memory");
  }
}

template <typename T, int B>
cudaError_t launch_qjl_tb(const QjlArgs& a, cudaStream_t stream) {
  if constexpr (Elem<T>::kBytes == 2) {
    const cudaError_t e = launch_qjl_tc<T, B>(a.x, a.n, a.p, a.S, a.codes, a.norms, a.qbits, a.rnorm, stream);
    if (e != cudaErrorNotSupported) return e;
  }
  if constexpr (Elem<T>::kBytes == 2) {
    // the swizzled input boxes need a 1024-byte-aligned start of dynamic shared
    // memory, which follows from the per-block reservation before it
    int dev = 0, reserved = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    QjlArgs a2 = a;
    if (a.p.cell.cells > 0 && a.p.cell.cells <= kQ2MaxCells && reserved % 1024 == 0 &&
        row_tensor_map(&a2.xmap, a.x, a.n, kQjlD, 2, kQjlTile)) {
      auto k2 = qjl_batch_kernel<T, B>;
      constexpr int smem2 = Qjl2Smem::TOTAL;
      cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k2),
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem2);
      if (e != cudaSuccess) return e;
      const int64_t ntiles = (a.n + kQjlTile - 1) / kQjlTile;
      int sms = 1;
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      const int64_t want = (ntiles + kQ2Groups - 1) / kQ2Groups;
      const int grid = int(want < sms ? want : sms);  // persistent: one CTA per SM
      return launch_pdl(k2, grid, kQ2Threads, smem2, stream, a2);
    }
  }
  auto k = a.p.sym ? qjl_encode_kernel<T, B, true> : qjl_encode_kernel<T, B, false>;
  constexpr int smem = QjlSmem<T>::TOTAL;
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = (a.n + kQjlTile - 1) / kQjlTile;
  int dev = 0, sms = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = int(ntiles < sms ? ntiles : sms);  // persistent: one CTA per SM
  return launch_pdl(k, grid, kQjlThreads, smem, stream, a);
}

template <typename T>
cudaError_t launch_qjl_t(const QjlArgs& a, cudaStream_t stream) {
  switch (a.p.bits) {
    case 1: return launch_qjl_tb<T, 1>(a, stream);
    case 2: return launch_qjl_tb<T, 2>(a, stream);
    case 3: return launch_qjl_tb<T, 3>(a, stream);
    case 4: return launch_qjl_tb<T, 4>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_encode_qjl(const void* x, int dtype, int64_t n, int d, const QuantParams& p,
                              const uint16_t* S, uint8_t* codes, float* norms, uint8_t* qjl_bits,
                              float* qjl_rnorm, cudaStream_t stream) {
  if (d != kQjlD) return cudaErrorInvalidValue;
  QjlArgs a;
  std::memset(&a.xmap, 0, sizeof(a.xmap));
  a.x = x;
  a.n = n;
  a.S = S;
  a.codes = codes;
  a.norms = norms;
  a.qbits = qjl_bits;
  a.rnorm = qjl_rnorm;
  a.p = p;
  switch (dtype) {
    case RRQ_F16: return launch_qjl_t<__half>(a, stream);
    case RRQ_BF16: return launch_qjl_t<__nv_bfloat16>(a, stream);
    case RRQ_F32: return launch_qjl_t<float>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rrq

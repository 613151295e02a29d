// tc_encode.cuh — encoder for d = 128, 4-bit codes and 16-bit inputs (the
// KV-cache case) with the rotation on tcgen05 and the accumulators in tensor
// memory.
//
// "Random-rotation quantization" page: scheme steps 1–2, "Why rotation works"
// (the randomized Hadamard transform), "History", EDEN and TurboQuant bullets.
// The rotated vector y' = H_128·D·x is formed as one dense product per tile:
// the ±1 matrix B^T[n][k] = s_k·H_128[n, k] (Sylvester order, the seeded signs
// folded in) is exact in fp16 and bf16, so tcgen05.mma (M = 128 rows, N = 128,
// K = 16, operands as stored, fp32 accumulation) gives every y'_n of a row
// with no butterfly left on the CUDA cores, which bound this kernel; the tensor
// pipe runs a few per cent busy.  A CTA has two groups of eight warps; each
// group owns 128-row tiles:
//  * one elected thread of the group loads a tile with two TMA boxes (128 rows
//    × 128 bytes, 128-byte swizzle) and issues its eight products into one of
//    the group's two 128-column tensor-memory buffers, so the next tile's
//    products run while the warps finish this one;
//  * tensor-memory lane r (row r of the tile) is read by two threads, warp
//    w and w + 4 of the group: thread half h takes coordinates [64h, 64h + 64),
//    i.e. bytes [32h, 32h + 32) of the code row; the two halves of ‖y'‖²
//    meet through shared memory and a 64-thread named barrier (ν² = ‖y'‖²/d),
//    summed in one order by both;
//  * the code of a coordinate is byte 2 of bits(f) + off_j, one lane-replicated
//    table load and one add (FixedSearch, mma_encode.cuh), and eight codes go
//    into a word by byte permutes;
//  * codes leave through a per-warp 32 × 32-byte tile in the 32-byte swizzle
//    (conflict-free for row-per-thread stores) and a TMA tensor store.
// Every wait is bounded, and each pair of warps takes its go/stop decision
// for a tile together (a barrier reduction), so a pair never splits at its
// named barrier; after a timeout the tile's norms are NaN, the copies and
// products still in flight are waited for (bounded) and the tensor memory is
// freed.
#pragma once

#include "mma_encode.cuh"
#include "tcgen05.cuh"

namespace rrq {

struct EncTc {
  static constexpr int D = 128, TILE = 128, GROUPS = 2, WARPS = 16, THREADS = WARPS * 32;
  // shared addresses (the dynamic base is checked to be kBase)
  static constexpr uint32_t kBase = 0x400;
  static constexpr uint32_t HT = 0x400;       // B^T: 16 n-groups × 16 k-groups of 8×8 core matrices, 32 KB
  static constexpr uint32_t SIGNS = 0x8400;   // 128 sign bits, bit k of word k / 32
  static constexpr uint32_t BARS = 0x8480;    // [group][stage]: in_full, mma_done, tmem_free
  static constexpr uint32_t TSLOT = 0x84E0;
  static constexpr uint32_t FLAGS = 0x84F0;   // [group] failure flags
  static constexpr uint32_t PSUM = 0x8800;    // [group][tile parity][half][row] partial ‖y'‖², 4 KB
  static constexpr uint32_t CTILE = 0x9800;   // 16 warps × 1 KB code tiles
  static constexpr uint32_t kTable = 0x10000; // off_j at kTable + j·256 + lane·4
  static constexpr uint32_t kStages = 0x18000;
  static constexpr uint32_t STAGE = TILE * D * 2;   // 32 KB: two boxes of 16 KB
  static constexpr size_t kTotal = size_t(kStages + GROUPS * 2 * STAGE) - kBase;
  static_assert(HT + D * D * 2 <= SIGNS && BARS + GROUPS * 2 * 3 * 8 <= TSLOT && FLAGS + 16 <= PSUM, "head");
  static_assert(PSUM + GROUPS * 2 * 2 * TILE * 4 <= CTILE && CTILE + WARPS * 1024 <= kTable, "code tiles");
  static_assert(kTotal <= 227 * 1024, "shared memory");
  // instruction descriptor, kind::f16: D fp32, A and B fp16 (or both bf16),
  // K-major, N = 128, M = 128
  static constexpr uint32_t idesc(bool bf16) {
    return (1u << 4) | (bf16 ? (1u << 7) | (1u << 10) : 0u) | ((128u / 8) << 17) | ((128u / 16) << 24);
  }
};

// Bounded wait: up to 2^24 polls of the phase (a few seconds in all).
constexpr uint32_t kTcWaitLimit = 1u << 24;

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kTcWaitLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// AND of `v` over the `nthreads` threads (whole warps) meeting at named barrier `id`.
__device__ __forceinline__ bool bar_and(uint32_t id, uint32_t nthreads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(v)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bar_named(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <typename T>
__global__ void __launch_bounds__(EncTc::THREADS, 1)
encode_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap cmap,
                 int64_t n, float* __restrict__ norms, const QuantParams p,
                 const __grid_constant__ FixedSearch fs) {
  using L = EncTc;
  pdl_release();
  extern __shared__ __align__(1024) uint8_t dsm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = warp >> 3, h = (warp >> 2) & 1, q = warp & 3;  // group, row half, lane quarter
  const int64_t ntiles = (n + L::TILE - 1) / L::TILE;
  const int64_t tstride = int64_t(L::GROUPS) * gridDim.x;
  const int64_t t0 = int64_t(g) * gridDim.x + blockIdx.x;
  const int64_t my_tiles = t0 < ntiles ? (ntiles - t0 + tstride - 1) / tstride : 0;
  if (smem_addr(dsm) != L::kBase) {
    // not the layout the launch assumed: this CTA's vectors get NaN norms
    pdl_wait();
    for (int64_t k = 0; k < my_tiles && h == 0; ++k) {
      const int64_t r = (t0 + k * tstride) * L::TILE + 32 * q + lane;
      if (r < n) norms[r] = __uint_as_float(0x7fc00000u);
    }
    return;
  }
  auto at = [&](uint32_t addr) { return dsm + (addr - L::kBase); };
  uint32_t* smask = reinterpret_cast<uint32_t*>(at(L::SIGNS));
  uint64_t* bars = reinterpret_cast<uint64_t*>(at(L::BARS));
  uint32_t* tslot = reinterpret_cast<uint32_t*>(at(L::TSLOT));
  volatile int* gfail = reinterpret_cast<volatile int*>(at(L::FLAGS));
  float* psum = reinterpret_cast<float*>(at(L::PSUM));
  uint32_t* tab = reinterpret_cast<uint32_t*>(at(L::kTable));
  auto in_full = [&](int s) { return &bars[(g * 2 + s) * 3 + 0]; };
  auto mma_done = [&](int s) { return &bars[(g * 2 + s) * 3 + 1]; };
  auto tmem_free = [&](int s) { return &bars[(g * 2 + s) * 3 + 2]; };

  // ---- tables, barriers, tensor memory
  if (warp < L::D / 32) {
    const uint32_t m = __ballot_sync(kFull, sign_bit(p.seed, 32 * warp + lane) != 0);
    if (lane == 0) smask[warp] = m;
  }
  for (int i = tid; i < 128 * 32; i += blockDim.x) tab[(i >> 5) * 64 + (i & 31)] = fs.off[i >> 5];
  if (tid == 0) {
    for (int i = 0; i < L::GROUPS * 2; ++i) {
      mbar_init(&bars[i * 3 + 0], 1);
      mbar_init(&bars[i * 3 + 1], 1);
      mbar_init(&bars[i * 3 + 2], 8);
    }
    gfail[0] = gfail[1] = 0;
    fence_mbarrier_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tslot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  // B^T[n][k] = s_k·(−1)^popc(n & k), K-major, no swizzle: core matrix (n/8, k/8)
  // of 8 n × 8 k at 2048·(n/8) + 128·(k/8), row n % 8 at 16·(n % 8), one
  // 16-byte row per item.  For k = 8kb + j the sign bit is s_k ⊕ parity(n & 8kb)
  // ⊕ parity((n mod 8) & j); the last term over j = 0..7 is the byte
  // 0xAA·n₀ ⊕ 0xCC·n₁ ⊕ 0xF0·n₂ (n_i the bits of n mod 8).
  for (int i = tid; i < L::D * L::D / 8; i += blockDim.x) {
    const int m = i & 7, kb = (i >> 3) & 15, nn = ((i >> 7) << 3) | m;
    uint32_t e = (m & 1 ? 0xAAu : 0u) ^ (m & 2 ? 0xCCu : 0u) ^ (m & 4 ? 0xF0u : 0u);
    e ^= (smask[kb >> 2] >> (8 * (kb & 3))) & 0xFFu;
    e ^= (__popc(nn & (kb << 3)) & 1) ? 0xFFu : 0u;
    constexpr uint32_t one2 = uint32_t(MmaType<T>::kOne) * 0x10001u;  // −1 = 1 with bit 15 set
    uint32_t w[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) w[t] = one2 | (((e >> (2 * t)) & 1u) << 15) | (((e >> (2 * t + 1)) & 1u) << 31);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(L::HT + uint32_t((nn >> 3) * 2048 + kb * 128 + m * 16)),
                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                 : "memory");
  }
  fence_proxy_async_smem();  // the table is visible to the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot + uint32_t(g * 2 * 128);  // this group's two 128-column buffers
  pdl_wait();  // from here on, global memory

  const bool leader = tid == 256 * g;  // lane 0 of the group's first warp
  const uint32_t stage0 = L::kStages + uint32_t(g * 2) * L::STAGE;
  constexpr uint32_t IDESC = L::idesc(MmaType<T>::kOne == 0x3F80u);
  auto issue_tma = [&](int64_t k) {
    const int s = int(k & 1);
    const int row = int((t0 + k * tstride) * L::TILE);
    mbarrier_expect_tx(smem_addr(in_full(s)), L::STAGE);
    tma_load_2d(stage0 + s * L::STAGE, &xmap, 0, row, smem_addr(in_full(s)));
    tma_load_2d(stage0 + s * L::STAGE + L::STAGE / 2, &xmap, 64, row, smem_addr(in_full(s)));
  };
  auto issue_mma = [&](int64_t k) {
    const int s = int(k & 1);
    const uint32_t st = stage0 + s * L::STAGE;
#pragma unroll
    for (int ks = 0; ks < L::D / 16; ++ks)
      tc_mma_f16(tmem + uint32_t(s * 128), smem_desc_sw128(st + (ks >> 2) * (L::STAGE / 2) + (ks & 3) * 32),
                 smem_desc(L::HT + uint32_t(ks) * 256, 128, 2048), IDESC, uint32_t(ks));
    mma_commit(mma_done(s));
  };

  // prologue: the first two tiles' copies, the first tile's products
  uint32_t pending = 0;  // leader: bit s = a copy into stage s is in flight, bit 2 + s its phase
  int64_t issued = 0;    // leader: tiles whose products have been issued
  auto copy = [&](int64_t kk) {
    issue_tma(kk);
    const int s = int(kk & 1);
    pending = (pending & ~(5u << s)) | (1u << s) | (uint32_t((kk >> 1) & 1) << (2 + s));
  };
  if (leader && my_tiles > 0) {
    copy(0);
    if (my_tiles > 1) copy(1);
    if (tc_wait(in_full(0), 0)) {
      pending &= ~1u;
      tc_fence_after();
      issue_mma(0);
      issued = 1;
    } else {
      gfail[g] = 1;
    }
  }

  const uint32_t pair_bar = uint32_t(1 + 4 * g + q);  // warps (g, 0, q) and (g, 1, q)
  const uint32_t tile = L::CTILE + uint32_t(warp) * 1024;
  const uint32_t swz = uint32_t((lane >> 2) & 1);
  const float2 bias2 = make_float2(fs.bias, fs.bias);
  const float num = fs.num;
  const uint32_t lane_word = L::kTable | uint32_t(lane) * 4u;
  const int row = 32 * q + lane;
  int64_t k = 0;
  for (; k < my_tiles; ++k) {
    const int s = int(k & 1);
    const uint32_t ph = uint32_t(k >> 1) & 1u;
    if (!bar_and(pair_bar, 64, gfail[g] == 0 && tc_wait(mma_done(s), ph))) break;
    tc_fence_after();
    if (leader) {
      // the next tile's products into the other buffer, once its copy has
      // landed and the warps have read that buffer's previous tile
      if (k + 1 < my_tiles) {
        const int s1 = s ^ 1;
        const bool ok = tc_wait(in_full(s1), uint32_t((k + 1) >> 1) & 1u) &&
                        (k < 1 || tc_wait(tmem_free(s1), uint32_t((k - 1) >> 1) & 1u));
        if (ok) {
          pending &= ~(1u << s1);
          tc_fence_after();
          issue_mma(k + 1);
          issued = k + 2;
        } else {
          gfail[g] = 1;
        }
      }
      // stage s has been read by this tile's products: refill it
      if (k + 2 < my_tiles) copy(k + 2);
    }
    __syncwarp();

    // ---- y'[64h + c], c < 64, of tile row `row` (tensor-memory lane), buffer s
    uint32_t v[4][16];
    const uint32_t tb = tmem + (uint32_t(32 * q) << 16) + uint32_t(s * 128 + 64 * h);
#pragma unroll
    for (int i = 0; i < 4; ++i) tmem_ld16(tb + uint32_t(16 * i), v[i]);
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(tmem_free(s));
    float2 acc = make_float2(0.f, 0.f), acc2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float2 a = make_float2(__uint_as_float(v[i][2 * j]), __uint_as_float(v[i][2 * j + 1]));
        const float2 b = make_float2(__uint_as_float(v[i][2 * j + 2]), __uint_as_float(v[i][2 * j + 3]));
        acc = fma2(a, a, acc);
        acc2 = fma2(b, b, acc2);
      }
    const float2 qa = add2(acc, acc2);
    float* ps = psum + (g * 2 + s) * 2 * L::TILE;
    ps[h * L::TILE + row] = qa.x + qa.y;
    bar_named(pair_bar, 64);
    const float nu2 = (ps[row] + ps[L::TILE + row]) * p.inv_d;  // the same order in both halves
    const float nu = sqrtf(nu2);
    // 2^18/ν to a few ulp: moves I by a fraction of a unit, inside the decision band
    const float sc = nu2 > 0.f ? num * rsqrtf(nu2) : 0.f;
    const float2 sc2 = make_float2(sc, sc);

    // codes: word w holds coordinates 64h + 8w + [0, 8)
    uint32_t words[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t cv[8];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int c = 8 * w + 2 * t;
        const float2 f = fma2(make_float2(__uint_as_float(v[c >> 4][c & 15]), __uint_as_float(v[c >> 4][(c & 15) + 1])),
                              sc2, bias2);
        const uint32_t fx = __float_as_uint(f.x), fy = __float_as_uint(f.y);
        cv[2 * t] = fx + lds_u32(__byte_perm(fx, lane_word, 0x7624u));
        cv[2 * t + 1] = fy + lds_u32(__byte_perm(fy, lane_word, 0x7624u));
      }
      // byte 2 of each cv is a code: gather the even and the odd coordinates'
      const uint32_t ev =
          __byte_perm(__byte_perm(cv[0], cv[2], 0x0062u), __byte_perm(cv[4], cv[6], 0x6200u), 0x7610u);
      const uint32_t od =
          __byte_perm(__byte_perm(cv[1], cv[3], 0x0062u), __byte_perm(cv[5], cv[7], 0x6200u), 0x7610u);
      words[w] = ev + (od << 4);
    }

    const int64_t row0 = (t0 + k * tstride) * L::TILE + 32 * q;
    if (lane == 0) bulk_wait_read_all();  // the previous tile's store has read the code tile
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 2; ++c)
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(tile + uint32_t(lane * 32) + ((uint32_t(c) ^ swz) << 4)),
                   "r"(words[4 * c]), "r"(words[4 * c + 1]), "r"(words[4 * c + 2]), "r"(words[4 * c + 3])
                   : "memory");
    if (h == 0 && row0 + lane < n) norms[row0 + lane] = nu;
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(&cmap, 32 * h, int(row0), tile);
      bulk_commit();
    }
  }
  if (k < my_tiles) {
    // a wait gave up: the rest of this thread's rows get NaN norms
    gfail[g] = 1;
    for (; k < my_tiles && h == 0; ++k) {
      const int64_t r = (t0 + k * tstride) * L::TILE + 32 * q + lane;
      if (r < n) norms[r] = __uint_as_float(0x7fc00000u);
    }
  }
  if (leader) {
    // copies and products still in flight (after a failure) end before the
    // stages and the tensor memory are given up
    for (int st = 0; st < 2; ++st)
      if (pending & (1u << st)) tc_wait(in_full(st), (pending >> (2 + st)) & 1u);
    if (issued > 0) tc_wait(mma_done(int((issued - 1) & 1)), uint32_t((issued - 1) >> 1) & 1u);
  }
  if (lane == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(*tslot), "r"(512) : "memory");
  }
}

// cudaErrorNotSupported when the layout, the search table or a tensor map cannot
// be had (the caller then uses another encoder).
template <typename T>
cudaError_t launch_encode_tc(const T* x, int64_t n, const QuantParams& p, uint8_t* codes,
                             float* norms, cudaStream_t stream) {
  const FixedSearch fs = make_fixed_search(p);
  if (!fs.ok) return cudaErrorNotSupported;
  int dev = 0, reserved = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
      uint32_t(reserved) != EncTc::kBase)
    return cudaErrorNotSupported;
  CUtensorMap xmap, cmap;
  if (!row_tensor_map(&xmap, x, n, 128, 2, EncTc::TILE)) return cudaErrorNotSupported;
  if (!code_box32_tensor_map(&cmap, codes, n, 64, 32)) return cudaErrorNotSupported;
  auto k = encode_tc_kernel<T>;
  constexpr size_t smem = EncTc::kTotal;
  const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int64_t tiles = (n + EncTc::TILE - 1) / EncTc::TILE;
  const int grid = grid_for(reinterpret_cast<const void*>(k), EncTc::THREADS, smem,
                            (tiles + EncTc::GROUPS - 1) / EncTc::GROUPS);
  return launch_pdl(k, grid, EncTc::THREADS, smem, stream, xmap, cmap, n, norms, p, fs);
}

}  // namespace rrq

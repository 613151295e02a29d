// tc_encode.cuh — encoder for d = 128, 4-bit codes and 16-bit inputs (the
// KV-cache case) with the 32×32 Hadamard blocks on tcgen05 and the
// accumulators in tensor memory.
//
// "Random-rotation quantization" page: scheme steps 1–2, "Why rotation works"
// (the randomized Hadamard transform), "History", EDEN and TurboQuant bullets.
// As in mma_encode.cuh, H_128 = H_4 ⊗ H_32 over c = 32a + b:
//     z[a, b] = Σ_b' H_32[b, b']·s_{32a+b'}·x_{32a+b'},   y'[32a + b] = Σ_a' H_4[a, a']·z[a', b].
// A CTA has two groups of eight warps; each group owns 128-row tiles:
//  * one elected thread of the group loads a tile with two TMA boxes (128 rows
//    × 128 bytes, 128-byte swizzle) and issues, per block a, two
//    tcgen05.mma (M = 128, N = 32, K = 16, fp16/bf16 operands as stored, fp32
//    accumulation) of the tile's K slice against B_a = the ±1 table with the
//    rotation signs folded in; the accumulators are 4 × 32 columns of tensor
//    memory, two buffers per group, so the next tile's products run while the
//    warps finish this one;
//  * tensor-memory lane r (row r of the tile) is read by two threads, warp
//    w and w + 4 of the group: both sum all 128 z² (ν² = ‖y'‖²/d = 4·Σ z²/d),
//    then read the row again in column quarters and form y' and the codes
//    of blocks 2h and 2h + 1 only (thread half h), i.e. bytes [32h, 32h + 32)
//    of the code row; registers hold at most 64 z values at a time;
//  * the code of a coordinate is byte 2 of bits(f) + off_j, one lane-replicated
//    table load and one add (FixedSearch, mma_encode.cuh), and eight codes go
//    into a word by byte permutes;
//  * codes leave through a per-warp 32 × 32-byte tile in the 32-byte swizzle
//    (conflict-free for row-per-thread stores) and a TMA tensor store.
// Every wait is bounded; after a timeout the tile's norms are NaN, the copies
// and products still in flight are waited for (bounded) and the tensor memory
// is freed.
#pragma once

#include "mma_encode.cuh"
#include "tcgen05.cuh"

namespace rrq {

struct EncTc {
  static constexpr int D = 128, NB = 4, TILE = 128, GROUPS = 2, WARPS = 16, THREADS = WARPS * 32;
  static constexpr uint32_t kBase = 0x400;       // dynamic shared memory base (checked)
  static constexpr uint32_t HT = 0;              // 4 blocks × [32 n × 32 k] core matrices, 2 KB each
  static constexpr uint32_t SIGNS = HT + NB * 2048;
  static constexpr uint32_t BARS = SIGNS + D;    // [group][stage]: in_full, mma_done, tmem_free
  static constexpr uint32_t TSLOT = BARS + GROUPS * 2 * 3 * 8;
  static constexpr uint32_t FLAGS = TSLOT + 16;  // [group] failure flags
  static constexpr uint32_t CTILE = 0x3000;      // shared address: 16 warps × 2 × 1 KB code tiles
  static constexpr uint32_t kTable = 0x10000;    // off_j at kTable + j·256 + lane·4
  static constexpr uint32_t kStages = 0x18000;
  static constexpr uint32_t STAGE = TILE * D * 2;   // 32 KB: two boxes of 16 KB
  static constexpr size_t kTotal = size_t(kStages + GROUPS * 2 * STAGE) - kBase;
  static_assert(kBase + FLAGS + 16 <= CTILE, "head");
  static_assert(CTILE + WARPS * 2 * 1024 <= kTable, "code tiles");
  static_assert(kTotal <= 227 * 1024, "shared memory");
  // instruction descriptor, kind::f16: D fp32, A and B fp16 (or both bf16),
  // K-major, N = 32, M = 128
  static constexpr uint32_t idesc(bool bf16) {
    return (1u << 4) | (bf16 ? (1u << 7) | (1u << 10) : 0u) | ((32u / 8) << 17) | ((128u / 16) << 24);
  }
};

constexpr uint32_t kTcWaitLimit = 1u << 24;  // try_wait polls before a wait gives up

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kTcWaitLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

template <typename T>
__global__ void __launch_bounds__(EncTc::THREADS, 1)
encode_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap cmap,
                 int64_t n, float* __restrict__ norms, const QuantParams p,
                 const __grid_constant__ FixedSearch fs) {
  using L = EncTc;
  constexpr int NB = L::NB;
  pdl_release();
  extern __shared__ __align__(1024) uint8_t dsm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = warp >> 3, h = (warp >> 2) & 1, q = warp & 3;  // group, block half, lane quarter
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
  uint8_t* htab = dsm + L::HT;
  uint8_t* signs = dsm + L::SIGNS;
  uint64_t* bars = reinterpret_cast<uint64_t*>(dsm + L::BARS);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(dsm + L::TSLOT);
  volatile int* gfail = reinterpret_cast<volatile int*>(dsm + L::FLAGS);
  uint32_t* tab = reinterpret_cast<uint32_t*>(dsm + (L::kTable - L::kBase));
  auto in_full = [&](int s) { return &bars[(g * 2 + s) * 3 + 0]; };
  auto mma_done = [&](int s) { return &bars[(g * 2 + s) * 3 + 1]; };
  auto tmem_free = [&](int s) { return &bars[(g * 2 + s) * 3 + 2]; };

  // ---- tables, barriers, tensor memory
  for (int i = tid; i < L::D; i += blockDim.x) signs[i] = uint8_t(sign_bit(p.seed, i));
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
  // B_a^T[n][k] = s_{32a+k}·H_32[n, k] in the no-swizzle core-matrix layout
  // (8 n × 8 k per 128 bytes; 128 bytes between k groups, 512 between n groups)
  for (int i = tid; i < NB * 32 * 32; i += blockDim.x) {
    const int k = i & 31, nn = (i >> 5) & 31, a = i >> 10;
    const int neg = (signs[32 * a + k] ^ __popc(nn & k)) & 1;
    const uint32_t off = uint32_t(a * 2048 + (nn >> 3) * 512 + (k >> 3) * 128 + (nn & 7) * 16 + (k & 7) * 2);
    *reinterpret_cast<uint16_t*>(htab + off) = neg ? MmaType<T>::kMinusOne : MmaType<T>::kOne;
  }
  fence_proxy_async_smem();  // the tables are visible to the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot + uint32_t(g * 2 * 128);  // this group's two 128-column buffers
  pdl_wait();  // from here on, global memory

  const bool leader = tid == 256 * g;  // lane 0 of the group's first warp
  const uint32_t stage0 = L::kStages + uint32_t(g * 2) * L::STAGE;
  const uint32_t ht0 = smem_addr(htab);
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
    for (int a = 0; a < NB; ++a)
#pragma unroll
      for (int ks = 0; ks < 2; ++ks)
        tc_mma_f16(tmem + uint32_t(s * 128 + a * 32),
                   smem_desc_sw128(st + (a >> 1) * (L::STAGE / 2) + (a & 1) * 64 + ks * 32),
                   smem_desc(ht0 + a * 2048 + ks * 256, 128, 512), IDESC, uint32_t(ks));
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

  const uint32_t ctile0 = L::CTILE + uint32_t(warp) * 2 * 1024;
  const uint32_t swz = uint32_t((lane >> 2) & 1);
  const float2 bias2 = make_float2(fs.bias, fs.bias);
  const float num = fs.num;
  const float hsign = h ? -1.f : 1.f;  // y'[32(2h)+b] = p0 + (±p1), y'[32(2h+1)+b] = m0 + (±m1)
  const uint32_t lane_word = L::kTable | uint32_t(lane) * 4u;
  int ct = 0;
  int64_t k = 0;
  for (; k < my_tiles; ++k) {
    const int s = int(k & 1);
    const uint32_t ph = uint32_t(k >> 1) & 1u;
    if (!__all_sync(kFull, gfail[g] == 0 && tc_wait(mma_done(s), ph))) break;
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

    // ---- row 32q + lane of the tile (tensor-memory lane), buffer s.  First
    // Σ z² over all 128 columns, then, per column quarter b ∈ [8c, 8c + 8),
    // the H_4 rows 2h + ab on packed pairs (coordinates 2j, 2j + 1) and their
    // codes: word 4ab + c holds coordinates 32(2h + ab) + 8c + [0, 8)
    const uint32_t tb = tmem + (uint32_t(32 * q) << 16) + uint32_t(s * 128);
    float2 acc = make_float2(0.f, 0.f), acc2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t v[2][16];
      tmem_ld16(tb + uint32_t(32 * c), v[0]);
      tmem_ld16(tb + uint32_t(32 * c + 16), v[1]);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 z0 = make_float2(__uint_as_float(v[0][2 * j]), __uint_as_float(v[0][2 * j + 1]));
        const float2 z1 = make_float2(__uint_as_float(v[1][2 * j]), __uint_as_float(v[1][2 * j + 1]));
        acc = fma2(z0, z0, acc);
        acc2 = fma2(z1, z1, acc2);
      }
    }
    const float2 qa = add2(acc, acc2);
    const float nu = sqrtf(((qa.x + qa.y) * 4.f) * p.inv_d);  // ‖y'‖² = 4·Σ z² = d·‖x‖²
    const float sc = nu > 0.f ? __fdiv_rn(num, nu) : 0.f;
    const float2 sc2 = make_float2(sc, sc);
    const float2 hs2 = make_float2(hsign, hsign);

    uint32_t words[8];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t v[NB][8];
#pragma unroll
      for (int a = 0; a < NB; ++a) tmem_ld8(tb + uint32_t(a * 32 + 8 * c), v[a]);
      tmem_ld_wait();
      if (c == 3) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tmem_free(s));
      }
#pragma unroll
      for (int ab = 0; ab < 2; ++ab) {
        uint32_t cv[8];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          float2 z[NB];
#pragma unroll
          for (int a = 0; a < NB; ++a) z[a] = make_float2(__uint_as_float(v[a][2 * t]), __uint_as_float(v[a][2 * t + 1]));
          const float2 u = ab ? sub2(z[0], z[1]) : add2(z[0], z[1]);
          const float2 w = ab ? sub2(z[2], z[3]) : add2(z[2], z[3]);
          const float2 f = fma2(fma2(w, hs2, u), sc2, bias2);
          const uint32_t fx = __float_as_uint(f.x), fy = __float_as_uint(f.y);
          cv[2 * t] = fx + lds_u32(__byte_perm(fx, lane_word, 0x7624u));
          cv[2 * t + 1] = fy + lds_u32(__byte_perm(fy, lane_word, 0x7624u));
        }
        // byte 2 of each cv is a code: gather the even and the odd coordinates'
        const uint32_t ev =
            __byte_perm(__byte_perm(cv[0], cv[2], 0x0062u), __byte_perm(cv[4], cv[6], 0x6200u), 0x7610u);
        const uint32_t od =
            __byte_perm(__byte_perm(cv[1], cv[3], 0x0062u), __byte_perm(cv[5], cv[7], 0x6200u), 0x7610u);
        words[4 * ab + c] = ev + (od << 4);
      }
    }

    const int64_t row0 = (t0 + k * tstride) * L::TILE + 32 * q;
    const uint32_t tile = ctile0 + uint32_t(ct) * 1024;
    if (lane == 0) bulk_wait_read_1();  // the store from this tile two tiles ago has read it
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
    ct ^= 1;
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

// mma_decode.cuh — decoder for d = 128, 4-bit codes and fp16 outputs (the
// KV-cache case) with the inverse Hadamard transform on tensor-core tiles.
//
// "Random-rotation quantization" page, scheme step 3 (dequantise, then apply
// Πᵀ) and "Three decoders, one rotation" (the MSE decoder):
//     x̂ = Πᵀ·(ν/√d)·c[code] = D·H·c[code]·(ν/d),   H = H_4 ⊗ H_32.
// With coordinates c = 32a + b:
//     z[a', b] = Σ_b' H_32[b, b']·c[code_{32a'+b'}]    (per block a', on the tensor cores),
//     x̂[32a + b] = s_{32a+b}·(ν/d)·Σ_a' H_4[a, a']·z[a', b]   (two butterfly stages in registers).
// A warp takes a batch of 32 vectors.  The A operand of block a' (32 rows ×
// 32 levels) is looked up from the codes in fp16: one lane-replicated table of
// level pairs, one entry per code byte, at shared address 0x10000 + byte·256 +
// lane·4, so the byte permute that picks a code byte out of its word is the
// load address.  The k order of the product is permuted (σ: k bit fields
// [e, c, h, s] → coordinate bits [e, h, s, c]) so that quad thread c reads
// exactly code word 4a' + c of each of its rows; the ±1 table B = H_32 with
// rows σ and columns π (as in the encoder) is the same for every block and sits
// in 16 registers.  The output columns π give quad thread c the coordinates
// 32a + 8c + [0, 8): one 16-byte fp16 chunk per row and block.
//  * codes and norms of the next batch stream into a per-warp cp.async ring
//    (80-byte rows), and one ldmatrix per 8 rows hands every quad thread its
//    code words without bank conflicts;
//  * after the H_4 stages: × ν/d, rounding to the output type, and the rotation
//    signs as an XOR of the sign bits;
//  * rows go to a per-warp tile of four 64-byte-wide boxes (one per block) in
//    the 64-byte swizzle, conflict-free for the quad layout, and leave in TMA
//    tensor stores that clip rows past the end of the array.
// Levels are fp16 (2^-12 relative), accumulation fp32.  With fp16 outputs the
// rounding of the levels stays below that of the output itself (ulp 2^-10);
// bf16 outputs (ulp 2^-7) would flip enough roundings against the exact
// reconstruction to approach the 2e-3 tolerance, so they keep the fp32-level
// decoder.
#pragma once

#include "mma_encode.cuh"

namespace rrq {

template <int WARPS_, int NS_, bool SPLIT> struct DecMma {
  static constexpr int D = 128, NB = 4, CB = 64, RR = 80;
  static constexpr int NS = NS_, WARPS = WARPS_, THREADS = WARPS * 32;
  static constexpr int RING = NS * 32 * RR;
  static constexpr int TROWS = SPLIT ? 16 : 32;   // rows per output tile
  static constexpr int TILE = TROWS * 256;        // four boxes of TROWS × 64 bytes
  static constexpr int WB = (TILE + RING + 1023) / 1024 * 1024;
  static constexpr uint32_t kBase = 0x400;        // dynamic shared memory base (checked)
  static constexpr uint32_t kTable = 0x10000, kTableEnd = 0x20000;
  static constexpr uint32_t FRONT = kBase;        // 1024-aligned
  static constexpr int NFRONT = (kTable - FRONT) / WB < WARPS ? int((kTable - FRONT) / WB) : WARPS;
  static constexpr uint32_t warp_base(int w) {
    return w < NFRONT ? FRONT + uint32_t(w) * WB : kTableEnd + uint32_t(w - NFRONT) * WB;
  }
  static constexpr size_t total() { return size_t(warp_base(WARPS)) - kBase; }
  static_assert(total() <= 227 * 1024, "shared memory");
};

template <typename T, int WARPS_, int NS_, bool SPLIT>
__global__ void __launch_bounds__(WARPS_ * 32, 1)
decode_mma_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ norms, int64_t n,
                  const __grid_constant__ CUtensorMap omap, T* __restrict__ out, const QuantParams p) {
  using SM = DecMma<WARPS_, NS_, SPLIT>;
  constexpr int NB = SM::NB, NS = SM::NS, CB = SM::CB;
  pdl_release();
  extern __shared__ __align__(1024) uint8_t dsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qr = lane >> 2, qc = lane & 3;
  const int64_t nb = (n + 31) >> 5;
  const int64_t tw = int64_t(gridDim.x) * SM::WARPS;
  const int64_t gw = int64_t(warp) * gridDim.x + blockIdx.x;
  if (smem_addr(dsm) != SM::kBase) {
    // not the layout the launch assumed: this CTA's rows become NaN (0xFFFF
    // is a NaN in fp16 and in bf16)
    pdl_wait();
    for (int64_t b = gw; b < nb; b += tw) {
      const int64_t row = (b << 5) + lane;
      if (row < n)
        for (int c = 0; c < SM::D; c += 8)
          *reinterpret_cast<uint4*>(out + row * SM::D + c) = make_uint4(~0u, ~0u, ~0u, ~0u);
    }
    return;
  }
  uint32_t* tab = reinterpret_cast<uint32_t*>(dsm + (SM::kTable - SM::kBase));
  // the 128 rotation signs as 4 bit words, in the unused half of the table's first row
  uint32_t* sbits = tab + 32;
  if (warp == 0) {
#pragma unroll
    for (int a = 0; a < NB; ++a) {
      const uint32_t w = __ballot_sync(kFull, sign_bit(p.seed, 32 * a + lane) != 0);
      if (lane == 0) sbits[a] = w;
    }
  }
  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
    const int e = i >> 5;
    const __half2 v = __floats2half2_rn(p.levels[e & 15], p.levels[e >> 4]);
    tab[e * 64 + (i & 31)] = *reinterpret_cast<const uint32_t*>(&v);
  }
  // B fragments: b[nt][ks][j] holds H_32[π(8nt + qr)][σ(16ks + 2qc + 8j + e)] for e = 0, 1
  uint32_t bfr[4][2][2];
  {
    const int pn_lo = (qr & 1) | (((qr >> 1) & 3) << 3);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int ks = 0; ks < 2; ++ks)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int pn = pn_lo | (nt << 1);
          uint32_t w = 0;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int sk = e | (j << 1) | (ks << 2) | (qc << 3);
            w |= uint32_t((__popc(pn & sk) & 1) ? 0xBC00u : 0x3C00u) << (16 * e);
          }
          bfr[nt][ks][j] = w;
        }
  }
  __syncthreads();
  // sign masks of the output words: coordinates 32a + 8qc + 2nt + {0, 1}
  uint32_t smask[NB][4];
#pragma unroll
  for (int a = 0; a < NB; ++a) {
    const uint32_t w = sbits[a] >> (8 * qc);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
      smask[a][nt] = (((w >> (2 * nt)) & 1u) << 15) | (((w >> (2 * nt + 1)) & 1u) << 31);
  }
  pdl_wait();

  const uint32_t wbase = SM::warp_base(warp);
  const uint32_t tile = wbase;
  const uint32_t ring = wbase + SM::TILE;
  const uint32_t lane_word = SM::kTable | uint32_t(lane) * 4u;
  const uint32_t swz = uint32_t((qr >> 1) & 3);
  const float inv_d = p.inv_d;

  // batch b's codes and norms into ring stage st (16-byte units, coalesced)
  auto issue = [&](int st, int64_t b) {
    if (b < nb) {
      const int64_t v0 = b << 5;
      const uint32_t sb = ring + uint32_t(st * 32 * SM::RR);
#pragma unroll
      for (int i = 0; i < CB / 16; ++i) {
        const int t = lane + 32 * i, v = t / (CB / 16), u = t % (CB / 16);
        const bool ok = v0 + v < n;
        cp_async16(sb + uint32_t(v * SM::RR + u * 16), codes + (ok ? (v0 + v) * CB + u * 16 : 0), ok ? 16 : 0);
      }
      const bool ok = v0 + lane < n;
      cp_async4(sb + uint32_t(lane * SM::RR + CB), norms + (ok ? v0 + lane : 0), ok ? 4 : 0);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int k = 0; k < NS - 1; ++k) issue(k, gw + k * tw);

  int st = 0;
  for (int64_t b = gw; b < nb; b += tw) {
    cp_async_wait<NS - 2>();
    __syncwarp();
    const int64_t v0 = b << 5;
    // this lane's code words (rows qr + 8r, words 4a + qc) and norms
    uint32_t cw[4][NB];
    float sc[4];
    {
      const uint32_t sb = ring + uint32_t(st * 32 * SM::RR);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        // matrix a of the load: rows 8r + [0, 8), bytes [16a, 16a + 16): the
        // quad thread c receives word 4a + c of row 8r + qr
        ldsm_x4(cw[r], sb + uint32_t((8 * r + (lane & 7)) * SM::RR + (lane >> 3) * 16));
        float nu;
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(nu) : "r"(sb + uint32_t((qr + 8 * r) * SM::RR + CB)));
        sc[r] = nu * inv_d;
      }
    }
    __syncwarp();  // every lane has read this stage before it is refilled
    issue((st + NS - 1) % NS, b + (NS - 1) * tw);
    st = (st + 1 == NS) ? 0 : st + 1;

    auto run = [&](auto mts) {
      constexpr int M0 = decltype(mts)::value >= 2 ? 0 : decltype(mts)::value;
      constexpr int MN = decltype(mts)::value >= 2 ? 2 : 1;
      float acc[NB][MN][4][4];
#pragma unroll
      for (int a = 0; a < NB; ++a)
#pragma unroll
        for (int m = 0; m < MN; ++m) {
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) acc[a][m][nt][0] = acc[a][m][nt][1] = acc[a][m][nt][2] = acc[a][m][nt][3] = 0.f;
          const uint32_t w0 = cw[2 * (M0 + m)][a], w1 = cw[2 * (M0 + m) + 1][a];
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            uint32_t af[4];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint32_t sel = 0x7604u | uint32_t((2 * ks + j) << 4);
              asm("ld.shared.b32 %0, [%1];" : "=r"(af[2 * j]) : "r"(__byte_perm(w0, lane_word, sel)));
              asm("ld.shared.b32 %0, [%1];" : "=r"(af[2 * j + 1]) : "r"(__byte_perm(w1, lane_word, sel)));
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) mma_t<__half>(acc[a][m][nt], af, bfr[nt][ks][0], bfr[nt][ks][1]);
          }
        }
      if (lane == 0) bulk_wait_read_all();  // the previous stores have read the tile
      __syncwarp();
#pragma unroll
      for (int m = 0; m < MN; ++m)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = h + 2 * (M0 + m);  // row qr + 8r of the batch
          const float2 s2 = make_float2(sc[r], sc[r]);
          uint32_t ow[NB][4];
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
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
            for (int a = 0; a < NB; ++a) ow[a][nt] = pack2<T>(mul2(z[a], s2)) ^ smask[a][nt];
          }
          const int trow = qr + 8 * h + (SPLIT ? 0 : 16 * m);
#pragma unroll
          for (int a = 0; a < NB; ++a) {
            const uint32_t addr = tile + uint32_t(a * SM::TROWS * 64 + trow * 64) + ((uint32_t(qc) ^ swz) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(ow[a][0]), "r"(ow[a][1]),
                         "r"(ow[a][2]), "r"(ow[a][3])
                         : "memory");
          }
        }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int a = 0; a < NB; ++a)
          tma_store_2d(&omap, 32 * a, int(v0 + (SPLIT ? 16 * M0 : 0)), tile + uint32_t(a * SM::TROWS * 64));
        bulk_commit();
      }
    };
    if constexpr (SPLIT) {
      run(std::integral_constant<int, 0>());
      run(std::integral_constant<int, 1>());
    } else {
      run(std::integral_constant<int, 2>());
    }
  }
  cp_async_wait<0>();
  if (lane == 0) bulk_wait_all();
}

template <typename T, int W, int NS, bool SPLIT>
cudaError_t launch_decode_mma_v(const uint8_t* codes, const float* norms, int64_t n,
                                const CUtensorMap& omap, T* out, const QuantParams& p,
                                cudaStream_t stream) {
  using SM = DecMma<W, NS, SPLIT>;
  auto k = decode_mma_kernel<T, W, NS, SPLIT>;
  constexpr size_t smem = SM::total();
  const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int64_t batches = (n + 31) / 32;
  const int grid = grid_for(reinterpret_cast<const void*>(k), SM::THREADS, smem, (batches + W - 1) / W);
  return launch_pdl(k, grid, SM::THREADS, smem, stream, codes, norms, n, omap, out, p);
}

// cudaErrorNotSupported when the layout or the tensor map cannot be had (the
// caller then uses another decoder).
template <typename T>
cudaError_t launch_decode_mma(const uint8_t* codes, const float* norms, int64_t n,
                              const QuantParams& p, T* out, cudaStream_t stream) {
  int dev = 0, reserved = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
      uint32_t(reserved) != DecMma<12, 3, true>::kBase)
    return cudaErrorNotSupported;
  CUtensorMap omap;
  if (!half_box64_tensor_map(&omap, out, n, 128, DecMma<12, 3, true>::TROWS)) return cudaErrorNotSupported;
  return launch_decode_mma_v<T, 12, 3, true>(codes, norms, n, omap, out, p, stream);
}

}  // namespace rrq

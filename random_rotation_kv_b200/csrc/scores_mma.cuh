// scores_mma.cuh — the tensor-core score kernel for b ∈ {1, 2, 3, 4} and
// d ∈ {64, 128, 256, 512}, included by scores.cu (ScoreArgs, rotate_queries).
//
// "Random-rotation quantization" page, "Three decoders, one rotation",
// inner-product decoder: s[h,t] = scale·(ν/d)·Σ_i q'_{h,i}·c[code_i], q' = H·D·q.
// For one kv head g the scores of a 32-token unit are a [32 × d]·[d × G]
// product of the code levels and the group's rotated queries, run as
// mma.sync m16n8k16 tiles (fp16 operands, fp32 accumulation): tokens are M
// (two 16-row tiles), the group's query heads N (zero columns pad G to 8), d
// is K.  The dot product sums over coordinates, so any assignment of
// coordinates to K positions serves as long as the query operand (B) uses the
// same one:
//  * The row is cut into chunks of CS = min(d, 128) coordinates; in chunk c,
//    quad thread qc owns coordinates c·CS + qc·CC + [0, CC), CC = CS/4, i.e. a
//    contiguous slice of CC·b/8 bytes, and in the chunk's k-step kk its A
//    columns 2qc, 2qc + 1 hold "pair" 2kk and columns 2qc + 8, 2qc + 9 pair
//    2kk + 1 of that slice.
//  * b = 4: pair p is code byte p (coordinates 2p, 2p + 1); b = 2: the nibble
//    p; b = 3: the six bits at 6p: each becomes its fp16 level pair with one
//    load from a lane-replicated table at shared address 0x10000 (rows of 256
//    bytes: byte·256 | half·128 | lane·4, so a byte permute builds the address
//    for b = 4 and 2).
//  * b = 1: pair p is coordinates (p, p + CC/2), whose bits sit 16 apart in a
//    32-bit word, so one shift and one logic operation give the fp16 pair
//    (±1, ±1) with no table; with c = m ± h (m the midpoint, h the half gap of
//    the two levels) the score is (ν/d)·(h·Σ q'·(±1) + m·Σ q').
//  * The thread's tokens are 4qr + j (j = 2mt + h is row qr + 8h of m-tile mt),
//    so its norms and its scores of a head are 16-byte accesses.
//  * Units u = tile·hkv + g are taken warp-strided (u = w, w + nw, …): the
//    warps working at one moment read whole token rows together, and with nw a
//    multiple of hkv a warp keeps one kv head, whose B fragments stay in
//    registers.  A unit's code rows and norms stream through a per-warp
//    cp.async ring whose rows are padded so the quads' slice loads are
//    conflict-free.
#pragma once

namespace rrq {
namespace {

template <int D, int B, int W> struct ScoreMmaCfg {
  static constexpr int CS = D < 128 ? D : 128;       // coordinates per chunk
  static constexpr int NCH = D / CS;                 // chunks per row
  static constexpr int CC = CS / 4;                  // coordinates per thread per chunk
  static constexpr int SB = CC * B / 8;              // slice bytes per thread per chunk
  static constexpr int KC = CC / 4;                  // k-steps per chunk
  static constexpr int KK = NCH * KC;                // k-steps per row (= d/16)
  static constexpr int CB = D * B / 8;               // code bytes per key-head
  // ring row: CB bytes padded so that 4·RS spreads the quads' slices over the
  // banks (16-byte slices: RS ≡ 16, 8-byte: ≡ 8, else ≡ 4 modulo 32)
  static constexpr int PADT = SB >= 16 ? 16 : SB >= 8 ? 8 : 4;
  static constexpr int RS = CB + ((PADT - CB % 32) % 32 + 32) % 32;
  static constexpr int CP = RS % 16 == 0 ? 16 : RS % 8 == 0 ? 8 : 4;  // cp.async bytes
  static constexpr int NS = D >= 512 ? 2 : 3;        // ring stages
  static constexpr int STAGE = (32 * RS + 32 * 4 + 15) / 16 * 16;
  static constexpr int RING = NS * STAGE;
  static constexpr bool TABLE = B != 1;
  static constexpr uint32_t kBase = 0x400, kTable = 0x10000;
  static constexpr uint32_t TABLE_BYTES = B == 3 ? 64 * 256 : B == 1 ? 0 : 256 * 256;
  static constexpr int SW = (SB + 3) / 4;            // slice words per chunk
  // [inv | qsum | front rings] below 0x10000, the table, [back rings] (qf
  // aliases the back region in the prologue)
  __host__ __device__ static size_t inv(int hq) { return (size_t(hq) * 8 + 15) / 16 * 16; }
  __host__ __device__ static size_t head(int hq, int hkv) { return (void)hkv, inv(hq); }
  __host__ __device__ static size_t qf(int hq) { return size_t(hq) * D * 4; }
  __host__ __device__ static size_t front(int hq, int hkv) {
    const size_t start = (head(hq, hkv) + 15) / 16 * 16, room = kTable - kBase;
    const size_t n = start < room ? (room - start) / RING : 0;
    return n < size_t(W) ? n : size_t(W);
  }
  __host__ __device__ static size_t back0() {
    return kTable - kBase + (TABLE_BYTES > 0 ? TABLE_BYTES : 0);
  }
  __host__ __device__ static size_t ring(int hq, int hkv, int w) {
    const size_t nf = front(hq, hkv);
    return size_t(w) < nf ? (head(hq, hkv) + 15) / 16 * 16 + size_t(w) * RING
                          : back0() + (size_t(w) - nf) * RING;
  }
  __host__ __device__ static size_t total(int hq, int hkv) {
    if (head(hq, hkv) > kTable - kBase) return ~size_t(0);
    const size_t back = (size_t(W) - front(hq, hkv)) * RING;
    return back0() + (qf(hq) > back ? qf(hq) : back);
  }
};

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// The two coordinates of pair p of a thread's chunk slice (offsets within it).
template <int B, int CC> __host__ __device__ constexpr int pair_coord(int p, int e) {
  return B == 1 ? p + e * (CC / 2) : 2 * p + e;
}

// A register of pair p (compile-time after unrolling) of a slice held in
// words w[]: b = 1: nw holds the negated slice word(s) (see below).
template <int B, int CC>
__device__ __forceinline__ uint32_t a_reg(const uint32_t* w, int p, uint32_t col, uint32_t col2) {
  if constexpr (B == 4) {
    return lds32(__byte_perm(w[p >> 2], col, 0x7604u | ((p & 3) << 4)));
  } else if constexpr (B == 2) {
    return lds32(__byte_perm(w[p >> 3], (p & 1) ? col2 : col, 0x7604u | (((p >> 1) & 3) << 4)));
  } else if constexpr (B == 3) {
    const int o = 6 * p, wi = o >> 5, sh = o & 31;
    // the six bits at bits 8..13, then the row offset
    uint32_t v;
    if (sh <= 8) v = w[wi] << (8 - sh);
    else if (sh + 6 <= 32) v = w[wi] >> (sh - 8);
    else v = __funnelshift_r(w[wi], w[wi + 1], sh - 8);
    return lds32((v & 0x3F00u) | col);
  } else {
    // coordinates p and p + CC/2 at bits p and p + 16 of the (negated, spread)
    // slice word: into the sign bits of an fp16 pair of ±1
    return ((w[0] << (15 - p)) & 0x80008000u) | 0x3C003C00u;
  }
}

template <int D, int B, int G, int W>
__global__ void __launch_bounds__(W * 32, 1) qk_scores_mma_kernel(const ScoreArgs a) {
  pdl_release();
  using Cf = ScoreMmaCfg<D, B, W>;
  constexpr int CB = Cf::CB, KK = Cf::KK, KC = Cf::KC, NCH = Cf::NCH, CC = Cf::CC, SB = Cf::SB;
  constexpr int SW = Cf::SW, NS = Cf::NS;
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const QuantParams& p = a.p;
  if (smem_addr(smem) != Cf::kBase) {
    // not the layout the launch assumed: mark every score as invalid
    pdl_wait();
    for (int64_t i = int64_t(blockIdx.x) * W * 32 + tid; i < int64_t(a.hq) * a.T; i += int64_t(gridDim.x) * W * 32)
      a.scores[i] = __int_as_float(0x7fc00000);
    return;
  }
  float* inv_s = reinterpret_cast<float*>(smem);
  float* qsum = inv_s + a.hq;  // Σ_i q'_{h,i} (1-bit codes)
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem + (Cf::kTable - Cf::kBase));
  float* qf = reinterpret_cast<float*>(smem + Cf::back0());
  uint8_t* ring = smem + Cf::ring(a.hq, a.hkv, warp);

  // ---- level table (lane-replicated pairs; half 1 of a row for b = 2's high nibble)
  if constexpr (Cf::TABLE) {
    constexpr int E = B == 3 ? 64 : 256;
    constexpr uint32_t M = (1u << B) - 1u;
    for (int i = tid; i < E * 64; i += W * 32) {
      const int e = i >> 6, h = (i >> 5) & 1;
      uint32_t lo, hi;
      if constexpr (B == 2) {
        const uint32_t nib = (uint32_t(e) >> (4 * h)) & 15u;
        lo = nib & M;
        hi = nib >> 2;
      } else {
        lo = uint32_t(e) & M;
        hi = uint32_t(e) >> B;
      }
      const __half2 v = __floats2half2_rn(p.levels[lo], p.levels[hi]);
      tab[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
  }
  pdl_wait();  // from here on, global memory
  rotate_queries<D>(a, qf, inv_s, warp, lane, W);
  __syncthreads();
  if constexpr (B == 1) {
    // Σ_i q'_{h,i} of the unscaled q' (qf holds q'·s_h)
    for (int h = warp; h < a.hq; h += W) {
      float acc = 0.f;
      for (int i = lane; i < D; i += 32) acc += qf[h * D + i];
#pragma unroll
      for (int m = 16; m > 0; m >>= 1) acc += __shfl_xor_sync(kFull, acc, m);
      if (lane == 0) qsum[h] = acc * inv_s[h];
    }
  }
  // ---- units u = tile·hkv + g, warp-strided (the launch makes nw a multiple of hkv)
  const int lg_hkv = __ffs(a.hkv) - 1;  // hkv is a power of two
  const int64_t nbt = (a.T + 31) >> 5;
  const int64_t nw = int64_t(gridDim.x) * W, gw = int64_t(blockIdx.x) * W + warp;
  const int g = int(gw & (a.hkv - 1));
  const int64_t tile0 = gw >> lg_hkv, TS = nw >> lg_hkv;
  const int64_t my_units = tile0 < nbt ? (nbt - tile0 + TS - 1) / TS : 0;
  const uint32_t col = Cf::kTable | uint32_t(lane) * 4u, col2 = col | 128u;
  const int qc = lane & 3, qr = lane >> 2;

  // this lane's B fragments (the kv head is fixed): head qr of group g (zero for
  // qr ≥ G); in chunk ch, k-step kc, b0 holds pair 2kc and b1 pair 2kc + 1 of
  // quad thread qc's slice
  uint32_t bfr[KK][2];
#pragma unroll
  for (int kk = 0; kk < KK; ++kk) {
    const int ch = kk / KC, kc = kk % KC;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      __half2 v = __floats2half2_rn(0.f, 0.f);
      if (qr < G) {
        const float* qh = qf + (g * G + qr) * D + ch * Cf::CS + qc * CC;
        const int pr = 2 * kc + j;
        v = __floats2half2_rn(qh[pair_coord<B, CC>(pr, 0)], qh[pair_coord<B, CC>(pr, 1)]);
      }
      bfr[kk][j] = *reinterpret_cast<const uint32_t*>(&v);
    }
  }
  __syncthreads();  // qf is dead: its space becomes the back rings

  // copy k of a unit (k < CPR) moves chunk i % CPR of row i / CPR, i = lane + 32k
  constexpr int CPR = CB / Cf::CP;  // copies per row = copies per lane
  const int64_t row_bytes = int64_t(a.hkv) * CB;
  const int64_t unit_step = TS * 32;
  const uint8_t* src_next = a.codes + (tile0 * 32 * a.hkv + g) * CB;
  const float* nrm_next = a.norms + (tile0 * 32 + lane) * a.hkv + g;
  int64_t t_next = tile0 * 32;
  const uint32_t ring0 = smem_addr(ring);
  auto copy = [&](uint32_t dst, const uint8_t* src, bool ok) {
    if constexpr (Cf::CP == 16) cp_async16(dst, ok ? src : a.codes, ok ? 16 : 0);
    else if constexpr (Cf::CP == 8) cp_async8(dst, ok ? src : a.codes, ok ? 8 : 0);
    else cp_async4(dst, ok ? src : a.codes, ok ? 4 : 0);
  };
  int64_t issued = 0;
  auto issue = [&](int stage) {
    if (issued < my_units) {
      const uint32_t sbase = ring0 + uint32_t(stage * Cf::STAGE);
      if (t_next + 32 <= a.T) {
#pragma unroll
        for (int k = 0; k < CPR; ++k) {
          const int i = lane + 32 * k, row = i / CPR, c = i % CPR;
          copy(sbase + uint32_t(row * Cf::RS + c * Cf::CP), src_next + row * row_bytes + c * Cf::CP, true);
        }
      } else {
#pragma unroll
        for (int k = 0; k < CPR; ++k) {
          const int i = lane + 32 * k, row = i / CPR, c = i % CPR;
          copy(sbase + uint32_t(row * Cf::RS + c * Cf::CP), src_next + row * row_bytes + c * Cf::CP,
               t_next + row < a.T);
        }
      }
      const bool ok = t_next + lane < a.T;
      cp_async4(sbase + 32 * Cf::RS + lane * 4, ok ? nrm_next : a.norms, ok ? 4 : 0);
      ++issued;
      src_next += unit_step * row_bytes;
      nrm_next += unit_step * a.hkv;
      t_next += unit_step;
    }
    cp_async_commit();
  };
#pragma unroll
  for (int k = 0; k < NS - 1; ++k) issue(k);

  // head scales of the lane's two accumulator columns
  float hsc[2], hoff[2];  // scale·inv_d/s_h (× h for b = 1) and scale·inv_d·m·Σq'
  {
    const float cm = 0.5f * (p.levels[0] + p.levels[1]), ch = 0.5f * (p.levels[1] - p.levels[0]);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = g * G + 2 * qc + e;
      const bool ok = 2 * qc + e < G;
      hsc[e] = ok ? a.scale * p.inv_d * inv_s[h] * (B == 1 ? ch : 1.f) : 0.f;
      hoff[e] = ok && B == 1 ? a.scale * p.inv_d * cm * qsum[h] : 0.f;
    }
  }
  const bool vec_out = (a.T & 3) == 0;  // 16-byte score stores stay aligned
  float* out_next = a.scores + int64_t(g * G + 2 * qc) * a.T + tile0 * 32 + 4 * qr;
  int64_t t0 = tile0 * 32;

  int stage = 0;
  for (int64_t k = 0; k < my_units; ++k) {
    cp_async_wait<NS - 2>();
    __syncwarp();
    const uint8_t* st = ring + stage * Cf::STAGE;
    const float4 nu = *reinterpret_cast<const float4*>(st + 32 * Cf::RS + 16 * qr);
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
      // slice words of the four rows (tokens 4qr + j) in chunk ch
      uint32_t sw[4][SW];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint8_t* src = st + (4 * qr + j) * Cf::RS + ch * 4 * SB + qc * SB;
        if constexpr (SB == 16) {
          const uint4 v = *reinterpret_cast<const uint4*>(src);
          sw[j][0] = v.x; sw[j][1] = v.y; sw[j][2] = v.z; sw[j][3] = v.w;
        } else if constexpr (SB == 8) {
          const uint2 v = *reinterpret_cast<const uint2*>(src);
          sw[j][0] = v.x; sw[j][1] = v.y;
        } else if constexpr (SB % 4 == 0) {
#pragma unroll
          for (int i = 0; i < SW; ++i) sw[j][i] = reinterpret_cast<const uint32_t*>(src)[i];
        } else {  // 2 or 6 bytes (d = 64, b = 1 or 3): 16-bit loads
          const uint16_t* s16 = reinterpret_cast<const uint16_t*>(src);
#pragma unroll
          for (int i = 0; i < SW; ++i)
            sw[j][i] = uint32_t(s16[2 * i]) | (2 * i + 1 < SB / 2 ? uint32_t(s16[2 * i + 1]) << 16 : 0u);
        }
        if constexpr (B == 1) {
          // with 16 coordinates per slice, copy bits 8..15 to 16..23 so that
          // coordinates p and p + 8 sit 16 bits apart; then negate (a set bit is +1)
          if constexpr (CC == 16) sw[j][0] = sw[j][0] | (sw[j][0] << 8);
          sw[j][0] = ~sw[j][0];
        }
      }
      if (ch == NCH - 1) {
        __syncwarp();  // every lane has read this stage before it is refilled
        issue(stage == 0 ? NS - 1 : stage - 1);
        stage = (stage + 1 == NS) ? 0 : stage + 1;
      }
#pragma unroll
      for (int kc = 0; kc < KC; ++kc) {
        const int kk = ch * KC + kc;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const uint32_t* lo = sw[2 * mt];
          const uint32_t* hi = sw[2 * mt + 1];
          mma_16816(acc[mt], a_reg<B, CC>(lo, 2 * kc, col, col2), a_reg<B, CC>(hi, 2 * kc, col, col2),
                    a_reg<B, CC>(lo, 2 * kc + 1, col, col2), a_reg<B, CC>(hi, 2 * kc + 1, col, col2),
                    bfr[kk][0], bfr[kk][1]);
        }
      }
    }

    // accumulator i of tile mt: token 4qr + 2mt + (i >> 1), head 2qc + (i & 1)
    const bool full = vec_out && t0 + 32 <= a.T;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (2 * qc + e < G) {
        float* out = out_next + int64_t(e) * a.T;
        const float2 hs2 = make_float2(hsc[e], hsc[e]);
        float2 v01, v23;
        if constexpr (B == 1) {  // ν·(h·acc/s + m·Σq')·scale/d
          const float2 ho2 = make_float2(hoff[e], hoff[e]);
          v01 = mul2(make_float2(nu.x, nu.y), fma2(make_float2(acc[0][e], acc[0][2 + e]), hs2, ho2));
          v23 = mul2(make_float2(nu.z, nu.w), fma2(make_float2(acc[1][e], acc[1][2 + e]), hs2, ho2));
        } else {  // ν·acc/s·scale/d
          v01 = mul2(make_float2(acc[0][e], acc[0][2 + e]), mul2(make_float2(nu.x, nu.y), hs2));
          v23 = mul2(make_float2(acc[1][e], acc[1][2 + e]), mul2(make_float2(nu.z, nu.w), hs2));
        }
        if (full) {
          *reinterpret_cast<float4*>(out) = make_float4(v01.x, v01.y, v23.x, v23.y);
        } else {
          const float vv[4] = {v01.x, v01.y, v23.x, v23.y};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (t0 + 4 * qr + j < a.T) out[j] = vv[j];
        }
      }
    }
    out_next += unit_step;
    t0 += unit_step;
  }
  cp_async_wait<0>();
}

template <int D, int B, int G, int W>
cudaError_t launch_scores_mma_w(const ScoreArgs& a, cudaStream_t stream) {
  using Cf = ScoreMmaCfg<D, B, W>;
  auto k = qk_scores_mma_kernel<D, B, G, W>;
  const size_t smem = Cf::total(a.hq, a.hkv);
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int64_t units = ((a.T + 31) / 32) * a.hkv;
  int grid = grid_for(reinterpret_cast<const void*>(k), W * 32, smem, (units + W - 1) / W);
  // the kernel needs the warp count grid·W to be a multiple of hkv (a power of
  // two): round the grid to a multiple of hkv/W when hkv exceeds W
  if (a.hkv > W) {
    const int m = a.hkv / W;
    grid = grid < m ? m : grid / m * m;
  }
  return launch_pdl(k, grid, W * 32, smem, stream, a);
}

// Warps of the tensor-core kernel for (d, b, hq, hkv): 16 for d ≤ 128, 8 for
// d ≥ 256, as long as the shared layout fits; 0 when it does not apply (a
// group above 8 or not a power of two, a device whose reserved shared memory
// is not the 1 KB the fixed layout assumes).
template <int D, int B>
int mma_score_warps(int hq, int hkv) {
  const int group = hq / hkv;
  if (group > 8 || (group & (group - 1))) return 0;
  int dev = 0, reserved = 0;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) == cudaSuccess &&
      uint32_t(reserved) != ScoreMmaCfg<D, B, 16>::kBase)
    return 0;
  if (D <= 128 && ScoreMmaCfg<D, B, 16>::total(hq, hkv) <= 227 * 1024) return 16;
  if (ScoreMmaCfg<D, B, 8>::total(hq, hkv) <= 227 * 1024) return 8;
  return 0;
}

template <int D, int B, int G>
cudaError_t launch_scores_mma_g(const ScoreArgs& a, cudaStream_t stream) {
  if constexpr (D <= 128) {
    if (mma_score_warps<D, B>(a.hq, a.hkv) == 16) return launch_scores_mma_w<D, B, G, 16>(a, stream);
  }
  return launch_scores_mma_w<D, B, G, 8>(a, stream);
}

template <int D, int B>
cudaError_t launch_scores_mma(const ScoreArgs& a, cudaStream_t stream) {
  switch (a.group) {
    case 1: return launch_scores_mma_g<D, B, 1>(a, stream);
    case 2: return launch_scores_mma_g<D, B, 2>(a, stream);
    case 4: return launch_scores_mma_g<D, B, 4>(a, stream);
    case 8: return launch_scores_mma_g<D, B, 8>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace
}  // namespace rrq

// scores_qjl.cu — unbiased decode-time attention scores on TurboQuant-style
// keys: b-bit MSE codes plus the one-bit QJL sketch of the residual, in one pass.
//
// "Random-rotation quantization" page: "History", TurboQuant bullet (a biased
// MSE quantiser followed by an unbiased one-bit stage on the residual) and QJL
// bullet; "Three decoders, one rotation", inner-product decoder; "Bias vs
// unbiasedness".  With q' = H·D·q = √d·Πq, v = S·q' and g = ⌊h·hkv/hq⌋:
//     s[h][t] = scale · ( (ν_{t,g}/d)·Σ_i q'_{h,i}·c[code_{t,g,i}]
//                         + √(π/2)·ρ_{t,g}/(d·√d) · Σ_i v_{h,i}·sign_{t,g,i} ),
// the first term scale·<q_h, x̂_{t,g}>, the second the residual estimate
// √(π/2)/d·ρ·<S·Πq_h, sign> (sign_i = +1 for a set bit, −1 otherwise).
//
// Work split.  A CTA serves one kv head g and its GQA group of G query heads,
// so its prologue rotates only those G queries and projects them by S (G×d²
// multiply-adds, S read from L2).  Both are kept as fp16 pairs, each head
// scaled by a power of two to |·| ≤ 1 (undone in fp32).  Warps then take
// units of 32 consecutive tokens of that kv head, and each unit's two dot
// products are mma.sync m16n8k16 tiles (fp16 operands, fp32 accumulation):
// tokens are M, the group's heads N (zero columns pad G to 8), coordinates K.
// Thread quad position c owns coordinates [32c, 32c + 32) of its rows, so it
// loads B code words and one sign word per row (the next unit's while it works
// on this one).  Each A register of the code product is one load from a
// lane-replicated table of fp16 level pairs (coordinates 2j, 2j + 1).  The
// sign product pairs coordinates j and j + 16 of a sign word instead: their
// bits are 16 apart, so one shift and one logic operation place both (negated)
// into the sign bits of an fp16 pair of ±1, with no table.  The query operand
// of each product uses its product's coordinate order.
#include <cmath>

#include "rrq_device.cuh"
#include "scores_qjl.h"

namespace rrq {
namespace {

constexpr int kSD = 128;              // head dimension served
constexpr int kSWarps = 16;
constexpr int kSThreads = kSWarps * 32;

// Level table of the b-bit codes, lane-replicated, at a shared address aligned
// to its size so that entry | lane column | base is one OR.  An entry is 256
// bytes: the 32 lanes' copies of its first level pair, then (b ≤ 2) of its
// second, so each half2 is one 32-bit load:
//   b = 1: a code nibble (two coordinate pairs), 16 entries;
//   b = 2: a code byte (two pairs), 256 entries;
//   b = 3: six bits (one pair), 64 entries of 128 B;
//   b = 4: a code byte (one pair), 256 entries (the second half unused: the
//     byte permute places the byte at bits 8..15).
template <int B> struct LevelTable {
  static constexpr uint32_t kEntries = B == 1 ? 16 : B == 3 ? 64 : 256;
  static constexpr uint32_t kStride = B == 3 ? 128 : 256;
  static constexpr uint32_t kBytes = kEntries * kStride;
  static constexpr bool kTwoPairs = B <= 2;  // an entry holds pairs 2kk and 2kk+1
};

// Shared memory, as offsets from the dynamic base at shared address `base`
// (the host computes it for the device's reserved shared memory; the kernel
// checks it):
//   bf   B fragments of q'' and v'', [2][4][32] × 16 B;
//   qf   q' and v in fp32 (prologue), [2][G][128];
//   sc   1/s_q, 1/s_v and max|v| bits per head;
//   tab  the level table, aligned to its size.
struct QjlLayout {
  uint32_t bf, qf, sc, tab, total;
};
template <int B, int G>
__host__ __device__ constexpr QjlLayout qjl_layout(uint32_t base) {
  const uint32_t tb = LevelTable<B>::kBytes;
  const uint32_t bf = (base + 15u) / 16u * 16u;
  const uint32_t qf = bf + 2u * 4u * 32u * 16u;
  const uint32_t sc = qf + 2u * G * kSD * 4u;
  const uint32_t end = (sc + 3u * G * 4u + 15u) / 16u * 16u;
  const uint32_t tab = (end + tb - 1u) / tb * tb;
  return QjlLayout{bf - base, qf - base, sc - base, tab - base, tab + tb - base};
}

// The slice of one key row that quad position c owns: coordinate pairs
// [16c, 16c + 16), i.e. code words [B·c, B·c + B) and sign word c.
template <int B> struct RowSlice {
  uint32_t c[B];
  uint32_t s;
  float nu, rho;
};

template <int B>
__device__ __forceinline__ void load_slice(RowSlice<B>& r, const QjlScoreArgs& a, int64_t n, bool ok,
                                           int qc) {
  if (ok) {
    const uint32_t* cw = reinterpret_cast<const uint32_t*>(a.codes + n * (16 * B)) + B * qc;
    if constexpr (B == 4) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4*>(cw));
      r.c[0] = v.x; r.c[1] = v.y; r.c[2] = v.z; r.c[3] = v.w;
    } else if constexpr (B == 2) {
      const uint2 v = __ldcs(reinterpret_cast<const uint2*>(cw));
      r.c[0] = v.x; r.c[1] = v.y;
    } else {
#pragma unroll
      for (int k = 0; k < B; ++k) r.c[k] = __ldcs(cw + k);
    }
    r.s = __ldcs(reinterpret_cast<const uint32_t*>(a.bits + n * 16) + qc);
    r.nu = __ldcs(a.norms + n);
    r.rho = __ldcs(a.rnorm + n);
  } else {
#pragma unroll
    for (int k = 0; k < B; ++k) r.c[k] = 0u;
    r.s = 0u;
    r.nu = 0.f;
    r.rho = 0.f;
  }
}

// Nibble kk of w at bits 8..11 (kk compile-time after unrolling).
__device__ __forceinline__ uint32_t nibble_bits(uint32_t w, int kk) {
  const uint32_t t = kk <= 2 ? (w << (8 - 4 * kk)) : (w >> (4 * kk - 8));
  return t & 0xF00u;
}

// fp16 pair (±1, ±1) from bits j and j + 16 of the negated sign word nw (a set
// bit of the sign word is +1): the two bits moved to bits 15 and 31, the rest
// of both halves the pattern of 1.0.
__device__ __forceinline__ uint32_t sign_pair(uint32_t nw, int j) {
  return ((nw << (15 - j)) & 0x80008000u) | 0x3C003C00u;
}

__device__ __forceinline__ uint32_t lds1(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// d += A·B for one m16n8k16 tile: fp16 A (row-major) and B (column-major)
// fragments, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Level pairs of coordinate pairs 2kk (x) and 2kk + 1 (y) of a row slice;
// col addresses the entry's first half, col2 = col | 128 its second.
template <int B>
__device__ __forceinline__ uint2 level_pairs(const uint32_t (&c)[B], int kk, uint32_t col, uint32_t col2) {
  if constexpr (B == 1) {
    const uint32_t t = nibble_bits(c[0], kk);
    return make_uint2(lds1(t | col), lds1(t | col2));
  } else if constexpr (B == 2) {
    const uint32_t sel = 0x7604u | ((kk & 3) << 4);
    return make_uint2(lds1(__byte_perm(c[kk >> 2], col, sel)), lds1(__byte_perm(c[kk >> 2], col2, sel)));
  } else if constexpr (B == 4) {
    const uint32_t w = c[kk >> 1], pos = 2 * (kk & 1);
    return make_uint2(lds1(__byte_perm(w, col, 0x7604u | (pos << 4))),
                      lds1(__byte_perm(w, col, 0x7604u | ((pos + 1) << 4))));
  } else {  // B == 3: six bits per pair, possibly across a word boundary
    uint32_t e[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int o = 6 * (2 * kk + hh), wi = o >> 5, sh = o & 31;
      const uint32_t v = sh + 6 <= 32 ? (c[wi] >> sh) : __funnelshift_r(c[wi], c[wi + 1], sh);
      e[hh] = lds1(((v & 63u) << 7) | col);
    }
    return make_uint2(e[0], e[1]);
  }
}

template <int B, int G>
__global__ void __launch_bounds__(kSThreads, 1) qk_scores_qjl_kernel(const QjlScoreArgs a, uint32_t base) {
  pdl_release();
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = blockIdx.x % a.hkv;
  const QjlLayout lay = qjl_layout<B, G>(base);
  if (smem_addr(smem) != base) {
    // not the layout the launch assumed: mark this CTA's scores as invalid
    pdl_wait();
    const int cpg = gridDim.x / a.hkv;
    for (int64_t t = int64_t(blockIdx.x / a.hkv) * kSThreads + tid; t < a.T; t += int64_t(cpg) * kSThreads)
      for (int j = 0; j < G; ++j) a.scores[int64_t(g * G + j) * a.T + t] = __int_as_float(0x7fc00000);
    return;
  }
  uint32_t* bf = reinterpret_cast<uint32_t*>(smem + lay.bf);
  float* qf = reinterpret_cast<float*>(smem + lay.qf);
  float* vf = qf + G * kSD;
  float* inv_sq = reinterpret_cast<float*>(smem + lay.sc);
  float* inv_sv = inv_sq + G;
  unsigned* vmax = reinterpret_cast<unsigned*>(inv_sv + G);
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem + lay.tab);
  const QuantParams& p = a.p;

  // ---- tables from the parameters alone
  using LT = LevelTable<B>;
  constexpr uint32_t M = (1u << B) - 1u;
  for (uint32_t i = tid; i < LT::kBytes / 4; i += kSThreads) {
    const uint32_t e = i / (LT::kStride / 4), wv = i % (LT::kStride / 4);
    float lo, hi;
    if constexpr (LT::kTwoPairs) {  // word wv = 32·hh + lane: pair hh of the entry
      const uint32_t pr = (e >> (2 * B * (wv >> 5))) & ((1u << (2 * B)) - 1u);
      lo = p.levels[pr & M];
      hi = p.levels[pr >> B];
    } else {
      lo = p.levels[e & M];
      hi = p.levels[e >> B];
    }
    const __half2 v = __floats2half2_rn(lo, hi);
    tab[i] = *reinterpret_cast<const uint32_t*>(&v);
  }
  if (tid < G) vmax[tid] = 0u;
  pdl_wait();  // from here on, global memory

  // ---- q' = H·D·q for the group's heads (one warp per head, 4 coordinates per lane)
  for (int j = warp; j < G; j += kSWarps) {
    const int h = g * G + j;
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = lane * 4 + k;
      const float x = __half2float(a.q[int64_t(h) * kSD + i]);
      v[k] = sign_bit(p.seed, i) ? -x : x;
    }
#pragma unroll
    for (int m = 1; m < 4; m <<= 1)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if ((k & m) == 0) {
          const float x0 = v[k], x1 = v[k | m];
          v[k] = x0 + x1;
          v[k | m] = x0 - x1;
        }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const float sg = (lane & m) ? -1.f : 1.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = fmaf(v[k], sg, __shfl_xor_sync(kFull, v[k], m));
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) qf[j * kSD + lane * 4 + k] = v[k];
  }
  __syncthreads();

  // ---- v = S·q' (row i of S against each head's q'), fp32
  for (int o = tid; o < G * kSD; o += kSThreads) {
    const int j = o / kSD, i = o % kSD;
    const uint4* srow = reinterpret_cast<const uint4*>(a.S + int64_t(i) * kSD);
    const float* qj = qf + j * kSD;
    float acc = 0.f;
#pragma unroll 4
    for (int kc = 0; kc < kSD / 8; ++kc) {
      const uint4 w = __ldg(srow + kc);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float s0 = __uint_as_float(ww[u] << 16), s1 = __uint_as_float(ww[u] & 0xFFFF0000u);
        acc = fmaf(s0, qj[kc * 8 + 2 * u], acc);
        acc = fmaf(s1, qj[kc * 8 + 2 * u + 1], acc);
      }
    }
    vf[o] = acc;
    atomicMax(&vmax[j], __float_as_uint(fabsf(acc)));
  }
  if (warp < G) {  // max|q'| of head `warp`
    float mx = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) mx = fmaxf(mx, fabsf(qf[warp * kSD + lane * 4 + k]));
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
    if (lane == 0) {
      int ex = 0;
      frexpf(mx, &ex);  // mx = f·2^ex, 0.5 ≤ f < 1
      inv_sq[warp] = mx > 0.f ? ldexpf(1.f, ex) : 1.f;
    }
  }
  __syncthreads();
  if (tid < G) {
    const float mx = __uint_as_float(vmax[tid]);
    int ex = 0;
    frexpf(mx, &ex);
    inv_sv[tid] = mx > 0.f ? ldexpf(1.f, ex) : 1.f;
  }
  __syncthreads();
  // B fragment word w = 2kk + hh of lane l (quad position c, column n), zero
  // for n ≥ G: part 0, head n's q'' at coordinates 2β, 2β + 1 with the pair
  // β = 16c + 2kk + hh; part 1, head n's v'' at coordinates 32c + 2kk + hh and
  // that + 16 (the sign product's order).
  for (int i = tid; i < 2 * 4 * 32 * 4; i += kSThreads) {
    const int comp = i & 3, l = (i >> 2) & 31, j = (i >> 7) & 3, part = i >> 9;
    const int w = 4 * j + comp, kk = w >> 1, hh = w & 1, c = l & 3, n = l >> 2;
    __half2 v = __floats2half2_rn(0.f, 0.f);
    if (n < G) {
      const float* src = (part ? vf : qf) + n * kSD;
      const float s = 1.f / (part ? inv_sv[n] : inv_sq[n]);  // a power of two
      const int i0 = part ? 32 * c + 2 * kk + hh : 2 * (16 * c + 2 * kk + hh);
      const int i1 = part ? i0 + 16 : i0 + 1;
      v = __floats2half2_rn(src[i0] * s, src[i1] * s);
    }
    bf[i] = *reinterpret_cast<const uint32_t*>(&v);
  }
  __syncthreads();

  const int qc = lane & 3, qr = lane >> 2;  // quad position, row in an 8-row group
  uint32_t bq[16], bv[16];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 x = reinterpret_cast<const uint4*>(bf)[j * 32 + lane];
    const uint4 y = reinterpret_cast<const uint4*>(bf)[(4 + j) * 32 + lane];
    bq[4 * j] = x.x; bq[4 * j + 1] = x.y; bq[4 * j + 2] = x.z; bq[4 * j + 3] = x.w;
    bv[4 * j] = y.x; bv[4 * j + 1] = y.y; bv[4 * j + 2] = y.z; bv[4 * j + 3] = y.w;
  }
  // per accumulator column e (head 2·qc + e): scale·inv_d/s_q and scale·cq/s_v
  const float cq = sqrtf(0.5f * float(M_PI)) / (float(kSD) * sqrtf(float(kSD)));
  float km[2], ks[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int h = 2 * qc + e;
    km[e] = h < G ? a.scale * p.inv_d * inv_sq[h] : 0.f;
    ks[e] = h < G ? a.scale * cq * inv_sv[h] : 0.f;
  }
  const uint32_t col_t = (base + lay.tab) | uint32_t(lane) * 4u;
  const uint32_t col_t2 = col_t | 128u;

  // ---- units of 32 tokens of kv head g, warp-major over the CTAs of g; rows
  // qr + 8m (m = 0..3) per thread
  const int cpg = gridDim.x / a.hkv;
  const int64_t ntile = (a.T + 31) / 32;
  const int64_t stride = int64_t(cpg) * kSWarps;
  int64_t tile = int64_t(warp) * cpg + blockIdx.x / a.hkv;  // warp-major: equal tiles per CTA
  RowSlice<B> cur[4], nxt[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int64_t t = tile * 32 + qr + 8 * m;
    load_slice<B>(cur[m], a, t * a.hkv + g, t < a.T, qc);
  }
  for (; tile < ntile; tile += stride) {
    const int64_t t0 = tile * 32;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int64_t t = t0 + stride * 32 + qr + 8 * m;
      load_slice<B>(nxt[m], a, t * a.hkv + g, t < a.T, qc);
    }
    float am[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float as[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    uint32_t nsw[4];  // negated sign words of the four rows
#pragma unroll
    for (int m = 0; m < 4; ++m) nsw[m] = ~cur[m].s;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint2 lo = level_pairs<B>(cur[2 * mt].c, kk, col_t, col_t2);
        const uint2 hi = level_pairs<B>(cur[2 * mt + 1].c, kk, col_t, col_t2);
        mma16816(am[mt], lo.x, hi.x, lo.y, hi.y, bq[2 * kk], bq[2 * kk + 1]);
        // A columns 2qc, 2qc + 1: coordinates 2kk, 2kk + 16; columns 2qc + 8,
        // 2qc + 9: coordinates 2kk + 1, 2kk + 17 of the thread's sign word
        mma16816(as[mt], sign_pair(nsw[2 * mt], 2 * kk), sign_pair(nsw[2 * mt + 1], 2 * kk),
                 sign_pair(nsw[2 * mt], 2 * kk + 1), sign_pair(nsw[2 * mt + 1], 2 * kk + 1),
                 bv[2 * kk], bv[2 * kk + 1]);
      }
    }
    // accumulator i of tile mt: row qr + 8·(i >> 1) + 16·mt, head 2·qc + (i & 1)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * qc + e;
      if (h < G) {
        float* out = a.scores + int64_t(g * G + h) * a.T + t0 + qr;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float v = fmaf(cur[m].nu * km[e], am[m >> 1][2 * (m & 1) + e],
                               cur[m].rho * ks[e] * as[m >> 1][2 * (m & 1) + e]);
          if (t0 + qr + 8 * m < a.T) out[8 * m] = v;
        }
      }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) cur[m] = nxt[m];
  }
}

template <int B, int G>
cudaError_t launch_bg(const QjlScoreArgs& a, cudaStream_t stream) {
  auto k = qk_scores_qjl_kernel<B, G>;
  int dev = 0, reserved = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  const uint32_t base = uint32_t(reserved);
  const QjlLayout lay = qjl_layout<B, G>(base);
  const int smem = int(lay.total);
  const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t ntile = (a.T + 31) / 32;
  const int resident = grid_for(reinterpret_cast<const void*>(k), kSThreads, smem, int64_t(1) << 40);
  int64_t cpg = resident / a.hkv;
  const int64_t need = (ntile + kSWarps - 1) / kSWarps;
  if (cpg > need) cpg = need;
  if (cpg < 1) cpg = 1;
  const int grid = int(cpg * a.hkv);
  return launch_pdl(k, grid, kSThreads, size_t(smem), stream, a, base);
}

template <int B>
cudaError_t launch_b(const QjlScoreArgs& a, cudaStream_t stream) {
  switch (a.group) {
    case 1: return launch_bg<B, 1>(a, stream);
    case 2: return launch_bg<B, 2>(a, stream);
    case 4: return launch_bg<B, 4>(a, stream);
    case 8: return launch_bg<B, 8>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_qk_scores_qjl(const QjlScoreArgs& a, cudaStream_t stream) {
  switch (a.p.bits) {
    case 1: return launch_b<1>(a, stream);
    case 2: return launch_b<2>(a, stream);
    case 3: return launch_b<3>(a, stream);
    case 4: return launch_b<4>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rrq

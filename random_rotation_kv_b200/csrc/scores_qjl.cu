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
// multiply-adds, S read from L2).  Both are kept as fp16 pairs, pair-major, each
// head scaled by a power of two to |·| ≤ 1 (undone in fp32).  Warps then take
// tiles of 32 consecutive tokens of that kv head, one token per lane: the lane
// loads its code row, sign row, norm and residual norm (16-byte loads, the next
// tile's while it works on this one), looks up each pair of codes in a
// lane-replicated table of fp16 level pairs and each pair of sign bits in a
// lane-replicated table of (±1, ±1), and accumulates both dot products for the
// G heads with packed fp16 FMAs, folded into fp32 every 16 pairs.
#include <cmath>

#include "rrq_device.cuh"
#include "scores_qjl.h"

namespace rrq {
namespace {

constexpr int kSD = 128;              // head dimension served
constexpr int kSP = kSD / 2;          // coordinate pairs
constexpr int kSWarps = 8;
constexpr int kSThreads = kSWarps * 32;

template <int B, int G> struct QSLayout {
  static constexpr int E = 1 << (2 * B);        // pair-table entries (two codes)
  static constexpr int TAB = 0;                 // [E][32] half2 level pairs
  static constexpr int SGN = TAB + E * 32 * 4;  // [4][32] half2 (±1, ±1)
  static constexpr int QH = SGN + 4 * 32 * 4;   // [kSP][G] half2 q'' pairs
  static constexpr int VH = QH + kSP * G * 4;   // [kSP][G] half2 v'' pairs
  static constexpr int QF = VH + kSP * G * 4;   // [G][kSD] fp32 q' (prologue)
  static constexpr int VF = QF + G * kSD * 4;   // [G][kSD] fp32 v (prologue)
  static constexpr int SC = VF + G * kSD * 4;   // [G] 1/s_q, [G] 1/s_v, [G] max|v| bits
  static constexpr int TOTAL = SC + 3 * G * 4;
};

// Bits [o, o + n) of a little-endian word array (o, n compile-time after unrolling).
template <int NW>
__device__ __forceinline__ uint32_t bit_field(const uint32_t (&w)[NW], int o, int n) {
  const int wi = o >> 5, sh = o & 31;
  const uint32_t lo = w[wi];
  const uint32_t hi = (wi + 1 < NW) ? w[wi + 1] : 0u;
  const uint32_t v = sh + n <= 32 ? (lo >> sh) : __funnelshift_r(lo, hi, sh);
  return v & ((1u << n) - 1u);
}

template <int B>
struct KeyRow {
  static constexpr int NW = 4 * B;  // code words (16·B bytes)
  uint32_t c[NW];
  uint32_t s[4];  // sign bits
  float nu, rho;
};

template <int B>
__device__ __forceinline__ void load_row(KeyRow<B>& r, const QjlScoreArgs& a, int64_t t, int g) {
  if (t < a.T) {
    const int64_t n = t * a.hkv + g;
    const uint4* cp = reinterpret_cast<const uint4*>(a.codes + n * (16 * B));
#pragma unroll
    for (int k = 0; k < B; ++k) {
      const uint4 v = __ldcs(cp + k);
      r.c[4 * k] = v.x; r.c[4 * k + 1] = v.y; r.c[4 * k + 2] = v.z; r.c[4 * k + 3] = v.w;
    }
    const uint4 sv = __ldcs(reinterpret_cast<const uint4*>(a.bits + n * 16));
    r.s[0] = sv.x; r.s[1] = sv.y; r.s[2] = sv.z; r.s[3] = sv.w;
    r.nu = __ldcs(a.norms + n);
    r.rho = __ldcs(a.rnorm + n);
  } else {
#pragma unroll
    for (int k = 0; k < KeyRow<B>::NW; ++k) r.c[k] = 0u;
#pragma unroll
    for (int k = 0; k < 4; ++k) r.s[k] = 0u;
    r.nu = 0.f;
    r.rho = 0.f;
  }
}

template <int B, int G>
__global__ void __launch_bounds__(kSThreads) qk_scores_qjl_kernel(const QjlScoreArgs a) {
  pdl_release();
  using L = QSLayout<B, G>;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem + L::TAB);
  uint32_t* sgn = reinterpret_cast<uint32_t*>(smem + L::SGN);
  __half2* qh = reinterpret_cast<__half2*>(smem + L::QH);
  __half2* vh = reinterpret_cast<__half2*>(smem + L::VH);
  float* qf = reinterpret_cast<float*>(smem + L::QF);
  float* vf = reinterpret_cast<float*>(smem + L::VF);
  float* inv_sq = reinterpret_cast<float*>(smem + L::SC);
  float* inv_sv = inv_sq + G;
  unsigned* vmax = reinterpret_cast<unsigned*>(inv_sv + G);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const QuantParams& p = a.p;
  const int g = blockIdx.x % a.hkv;

  // ---- tables from the parameters alone
  for (int i = tid; i < L::E * 32; i += kSThreads) {
    const int e = i >> 5;
    const __half2 v = __floats2half2_rn(p.levels[e & ((1 << B) - 1)], p.levels[e >> B]);
    tab[i] = *reinterpret_cast<const uint32_t*>(&v);
  }
  if (tid < 128) {
    const int e = tid >> 5;
    const __half2 v = __floats2half2_rn((e & 1) ? 1.f : -1.f, (e & 2) ? 1.f : -1.f);
    sgn[tid] = *reinterpret_cast<const uint32_t*>(&v);
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
    float mx = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) mx = fmaxf(mx, fabsf(v[k]));
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
    int ex = 0;
    frexpf(mx, &ex);
    const float s = mx > 0.f ? ldexpf(1.f, -ex) : 1.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) qf[j * kSD + lane * 4 + k] = v[k];
    qh[(2 * lane) * G + j] = __floats2half2_rn(v[0] * s, v[1] * s);
    qh[(2 * lane + 1) * G + j] = __floats2half2_rn(v[2] * s, v[3] * s);
    if (lane == 0) inv_sq[j] = 1.f / s;
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
  __syncthreads();
  for (int o = tid; o < G * kSP; o += kSThreads) {
    const int j = o / kSP, pr = o % kSP;
    const float mx = __uint_as_float(vmax[j]);
    int ex = 0;
    frexpf(mx, &ex);
    const float s = mx > 0.f ? ldexpf(1.f, -ex) : 1.f;
    vh[pr * G + j] = __floats2half2_rn(vf[j * kSD + 2 * pr] * s, vf[j * kSD + 2 * pr + 1] * s);
    if (pr == 0) inv_sv[j] = 1.f / s;
  }
  __syncthreads();

  // ---- tiles of 32 tokens of kv head g, one token per lane
  const int cpg = gridDim.x / a.hkv;
  const int64_t ntile = (a.T + 31) / 32;
  const int64_t stride = int64_t(cpg) * kSWarps;
  int64_t tile = int64_t(warp) * cpg + blockIdx.x / a.hkv;  // warp-major: equal tiles per CTA
  const float cq = sqrtf(0.5f * float(M_PI)) / (float(kSD) * sqrtf(float(kSD)));
  const uint32_t* tab_l = tab + lane;
  const uint32_t* sgn_l = sgn + lane;
  KeyRow<B> cur, nxt;
  load_row<B>(cur, a, tile * 32 + lane, g);
  for (; tile < ntile; tile += stride) {
    const int64_t t = tile * 32 + lane;
    load_row<B>(nxt, a, t + stride * 32, g);
    float accm[G], accq[G];
#pragma unroll
    for (int j = 0; j < G; ++j) accm[j] = accq[j] = 0.f;
#pragma unroll
    for (int f = 0; f < kSP / 16; ++f) {
      __half2 hm[G], hs[G];
#pragma unroll
      for (int j = 0; j < G; ++j) hm[j] = hs[j] = __float2half2_rn(0.f);
#pragma unroll
      for (int pp = 0; pp < 16; ++pp) {
        const int pr = f * 16 + pp;
        const uint32_t e = bit_field(cur.c, 2 * B * pr, 2 * B);
        const uint32_t sb = (cur.s[pr >> 4] >> ((2 * pr) & 31)) & 3u;
        const uint32_t cw = tab_l[e << 5], sw = sgn_l[sb << 5];
        const __half2 c2 = *reinterpret_cast<const __half2*>(&cw);
        const __half2 s2 = *reinterpret_cast<const __half2*>(&sw);
#pragma unroll
        for (int j = 0; j < G; ++j) {
          hm[j] = __hfma2(qh[pr * G + j], c2, hm[j]);
          hs[j] = __hfma2(vh[pr * G + j], s2, hs[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float2 m2 = __half22float2(hm[j]), s2 = __half22float2(hs[j]);
        accm[j] += m2.x + m2.y;
        accq[j] += s2.x + s2.y;
      }
    }
    if (t < a.T) {
      const float mse = cur.nu * p.inv_d, res = cur.rho * cq;
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float sc = a.scale * (mse * inv_sq[j] * accm[j] + res * inv_sv[j] * accq[j]);
        a.scores[int64_t(g * G + j) * a.T + t] = sc;
      }
    }
    cur = nxt;
  }
}

template <int B, int G>
cudaError_t launch_bg(const QjlScoreArgs& a, cudaStream_t stream) {
  auto k = qk_scores_qjl_kernel<B, G>;
  constexpr int smem = QSLayout<B, G>::TOTAL;
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t ntile = (a.T + 31) / 32;
  const int resident = grid_for(reinterpret_cast<const void*>(k), kSThreads, smem, int64_t(1) << 40);
  int64_t cpg = resident / a.hkv;
  const int64_t need = (ntile + kSWarps - 1) / kSWarps;
  if (cpg > need) cpg = need;
  if (cpg < 1) cpg = 1;
  const int grid = int(cpg * a.hkv);
  return launch_pdl(k, grid, kSThreads, smem, stream, a);
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

// attention.cu — one decode step of attention over a fully quantised K/V cache:
// scores from the packed K codes, softmax, and the weighted sum of the packed V
// codes, in one kernel.
//
// "Attn-rot (TurboQuant lite) in llama.cpp" page, "What kind of beast is
// Attn-rot": keys and values are both quantised after a rotation.
// "Random-rotation quantization" page, "Three decoders, one rotation": the MSE
// decoder for KV-cache compression, x̃ = Πᵀ(ν/√d · c[code]).  With g = ⌊h·hkv/hq⌋:
//     s[h,t] = scale · (ν^K_{t,g}/d) · Σ_i q'_{h,i}·c_K[code^K_{t,g,i}],   q' = H·D_K·q,
//     p[h,t] = softmax_t(s[h,·]),
//     out[h] = Σ_t p[h,t]·v̂_{t,g} = Πᵀ_V ( Σ_t p[h,t]·(ν^V_{t,g}/√d)·c_V[code^V_{t,g}] ),
// so the values are summed in their rotated domain and rotated back once per head.
//
// Work split.  The cache of kv head g is cut into S token ranges, one 16-warp
// CTA each (grid hkv × S, one CTA per SM); a CTA serves the GQA group of G query
// heads of its kv head, and its warps take tiles of 32 consecutive tokens.  Both
// contractions of a tile run as mma.sync m16n8k16 tiles (fp16 operands, fp32
// accumulation; the group padded to 8 columns), their A fragments looked up from
// lane-replicated tables of level pairs; the online softmax runs on the score
// fragments in base 2, and the value weights reach the value product through a
// per-warp transpose buffer (attention_decode_kernel says how).
//
// Range of the value weights.  The value product takes fp16 weights.  Rather
// than p·ν^V (which flushes to zero for small value norms and overflows for
// large ones), a weight is 2^(z − M + kWBias) with z = s·log2(e) + log2(ν^V) and
// M the running maximum of z: the token with the largest p·ν^V weighs
// 2^kWBias, no weight overflows, and only terms below 2^-(24 + kWBias) of the
// largest one flush, at any scale of the value norms.  The softmax denominator
// Σ 2^(s·log2(e) − m) keeps its own running maximum m, in fp32; the two meet
// once, in the final factor 2^(M − m − kWBias)/Σ.
// The warps' states merge within the CTA (shared-memory atomics after a common
// rescaling); each CTA writes its state (max, sum, G×128 partial sums) to the
// caller's workspace and counts itself in its kv head's counter there.  The
// last CTA of a kv head merges the S states, applies Πᵀ (a 128-point transform
// per head), writes the output and sets the counter back to zero.  No CTA waits
// for another.
#include <cmath>
#include <mutex>

#include "attention.h"
#include "rrq_device.cuh"

namespace rrq {
namespace {

constexpr int kAD = 128;
constexpr int kAWarps = 16;
constexpr int kAThreads = kAWarps * 32;
constexpr int kWRow = 40;  // fp16 weights per head row of a warp's transpose buffer (padded)
constexpr float kWBias = 14.f;  // log2 of the largest value weight (fp16 holds up to 65504)
constexpr float kLog2e = 1.4426950408889634f;

// 2^x and log2(x) (the SFU approximations; relative error about 2^-22).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Shared memory, as offsets from the dynamic base at shared address kBase (the
// launch checks the device's reserved shared memory; the kernel checks the
// address).  The two level tables sit at 64 KB-aligned addresses so that a byte
// permute of a code byte and the lane column (byte·256 | lane·4 | table) is the
// load address itself.
template <int G> struct ALayout {
  static constexpr uint32_t kBase = 0x400;
  static constexpr uint32_t KTAB = 0x10000 - kBase;              // [256][64] half2, K level pairs
  static constexpr uint32_t VTAB = 0x20000 - kBase;              // [256][64] half2, V level pairs
  static constexpr uint32_t BF = 0;                              // [4][32] uint4 B fragments of q''
  static constexpr uint32_t QF = BF + 4 * 32 * 16;               // [G][kAD] fp32 q' (prologue)
  static constexpr uint32_t INV = QF + G * kAD * 4;              // [G] 1/s
  static constexpr uint32_t WBUF = (INV + G * 4 + 15) / 16 * 16; // per warp: [8][kWRow] fp16 weights
  static constexpr uint32_t WM = WBUF + kAWarps * 8 * kWRow * 2; // [kAWarps][2G] warp maxima m, M
  static constexpr int PART_FLOATS = 3 * G + G * kAD;           // [G] m, [G] l, [G] M, [G][kAD] o
  static constexpr uint32_t PART = WM + kAWarps * 2 * G * 4;     // the CTA's partial state
  static constexpr uint32_t FLAG = PART + PART_FLOATS * 4;       // "this CTA merges its kv head"
  static constexpr uint32_t FIN = (FLAG + 16 + 15) / 16 * 16;    // the merging CTA's sums [G][kAD], [G] l, [G] M − m
  static constexpr uint32_t END = FIN + G * (kAD + 2) * 4;
  static constexpr uint32_t TOTAL = VTAB + 256 * 256;
  static_assert(END <= KTAB, "the small buffers fit below the K table");
  static_assert(TOTAL <= 227 * 1024, "shared memory");
};

// d += A·B for one m16n8k16 tile: fp16 A (row-major) and B (column-major)
// fragments, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Level pair of code byte `pos` of w: one load at byte·256 | col.
__device__ __forceinline__ uint32_t pair_at(uint32_t w, int pos, uint32_t col) {
  uint32_t v;
  asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(__byte_perm(w, col, 0x7604u | (pos << 4))));
  return v;
}
__device__ __forceinline__ uint32_t word4(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}
__device__ __forceinline__ uint32_t word2(const uint2& v, int i) { return i == 0 ? v.x : v.y; }

// 128-point unnormalised Walsh–Hadamard transform of v (4 values per lane, lane-major).
__device__ __forceinline__ void fwht128(float (&v)[4], int lane) {
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
}

// Per 32-token tile of kv head g, in each warp (qr = lane / 4, qc = lane % 4):
//  A. scores S[32 tokens × 8] = levels(K codes)·q'' as in the score kernel:
//     rows qr + 8m (m = 0..3) are the thread's tokens, its code slice is bytes
//     [16qc, 16qc + 16), columns 2qc, 2qc + 1 its heads.
//  B. the online softmax per head on those fragments (maxima and sum over the
//     tile by shuffles across the 8 lanes of equal qc); the value weights
//     2^(z − M + kWBias) go to the warp's transpose buffer as fp16 [head][token].
//  C. O^T[128 × 8] += levels(V codes)^T·W^T: coordinates are M, heads N,
//     tokens K.  Row qr of m-tile mt is coordinate 2(8qr + mt) and row qr + 8
//     coordinate 2(8qr + mt) + 1, so both come from V byte 8qr + mt; for the
//     token pair of a fragment column the two bytes' level pairs are looked up
//     and regrouped per coordinate with two byte permutes.  The output
//     columns are the same heads 2qc, 2qc + 1 as the score columns, so the
//     softmax rescaling touches only the thread's own accumulators.
template <int G>
__global__ void __launch_bounds__(kAThreads, 1) attention_decode_kernel(const AttnArgs a) {
  pdl_release();
  using L = ALayout<G>;
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = a.splits;
  const int g = blockIdx.x / S, sidx = blockIdx.x % S;
  if (smem_addr(smem) != L::kBase) {
    // not the layout the launch assumed: this CTA's kv head gets NaN outputs
    pdl_wait();
    if (sidx == 0)
      for (int i = tid; i < G * kAD; i += kAThreads) a.out[int64_t(g * G) * kAD + i] = __int_as_float(0x7fc00000);
    return;
  }
  uint32_t* ktab = reinterpret_cast<uint32_t*>(smem + L::KTAB);
  uint32_t* vtab = reinterpret_cast<uint32_t*>(smem + L::VTAB);
  uint32_t* bf = reinterpret_cast<uint32_t*>(smem + L::BF);
  float* qf = reinterpret_cast<float*>(smem + L::QF);
  float* inv_s = reinterpret_cast<float*>(smem + L::INV);
  __half* wbuf = reinterpret_cast<__half*>(smem + L::WBUF) + warp * 8 * kWRow;
  float* wmax = reinterpret_cast<float*>(smem + L::WM);
  float* part = reinterpret_cast<float*>(smem + L::PART);
  int* last_flag = reinterpret_cast<int*>(smem + L::FLAG);
  float* fin = reinterpret_cast<float*>(smem + L::FIN);

  // ---- level tables from the parameters alone: entry e at e·256 + lane·4
  for (int i = tid; i < 256 * 64; i += kAThreads) {
    const int e = i >> 6;
    const __half2 kv = __floats2half2_rn(a.pk.levels[e & 15], a.pk.levels[e >> 4]);
    const __half2 vv = __floats2half2_rn(a.pv.levels[e & 15], a.pv.levels[e >> 4]);
    ktab[i] = *reinterpret_cast<const uint32_t*>(&kv);
    vtab[i] = *reinterpret_cast<const uint32_t*>(&vv);
  }
  // weight rows of the padding heads (G..7) stay zero
  for (int i = lane; i < 8 * kWRow; i += 32) wbuf[i] = __float2half_rn(0.f);
  for (int i = tid; i < L::PART_FLOATS; i += kAThreads) part[i] = 0.f;
  pdl_wait();  // from here on, global memory

  // ---- q' = H·D_K·q for the group's heads, scaled per head to |q''| ≤ 1
  for (int j = warp; j < G; j += kAWarps) {
    const int h = g * G + j;
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = lane * 4 + k;
      const float x = __half2float(a.q[int64_t(h) * kAD + i]);
      v[k] = sign_bit(a.pk.seed, i) ? -x : x;
    }
    fwht128(v, lane);
    float mx = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) mx = fmaxf(mx, fabsf(v[k]));
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
    int ex = 0;
    frexpf(mx, &ex);
    const float s = mx > 0.f ? ldexpf(1.f, -ex) : 1.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) qf[j * kAD + lane * 4 + k] = v[k] * s;
    if (lane == 0) inv_s[j] = 1.f / s;
  }
  __syncthreads();
  // B fragment word w = 2kk + hh of lane l (quad position c, column n): the
  // pair β = 16c + 2kk + hh of head n's q'', zero for n ≥ G.
  for (int i = tid; i < 4 * 32 * 4; i += kAThreads) {
    const int comp = i & 3, l = (i >> 2) & 31, j = i >> 7;
    const int w = 4 * j + comp, kk = w >> 1, hh = w & 1, c = l & 3, n = l >> 2;
    const int beta = 16 * c + 2 * kk + hh;
    __half2 v = __floats2half2_rn(0.f, 0.f);
    if (n < G) v = __floats2half2_rn(qf[n * kAD + 2 * beta], qf[n * kAD + 2 * beta + 1]);
    bf[i] = *reinterpret_cast<const uint32_t*>(&v);
  }
  __syncthreads();

  const int qc = lane & 3, qr = lane >> 2;
  // this lane's B fragment words, read per k-step (registers are the scarce resource)
  const uint2* bq = reinterpret_cast<const uint2*>(bf) + lane * 2;
  float kse[2];  // log2(e)·scale·inv_d/s of heads 2qc + e: scores in base 2
#pragma unroll
  for (int e = 0; e < 2; ++e)
    kse[e] = 2 * qc + e < G ? kLog2e * a.scale * a.pk.inv_d * inv_s[2 * qc + e] : 0.f;
  const uint32_t kcol = 0x10000u | uint32_t(lane) * 4u;
  const uint32_t vcol = 0x20000u | uint32_t(lane) * 4u;

  // ---- token tiles of kv head g (warp-major over the S CTAs' warps)
  const int64_t ntile = (a.T + 31) / 32;
  const int64_t stride = int64_t(S) * kAWarps;
  // per head: score maximum m, denominator l, maximum M of z = s + log2 ν^V
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f}, M_run[2] = {-INFINITY, -INFINITY};
  float o[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  for (int64_t tile = int64_t(warp) * S + sidx; tile < ntile; tile += stride) {
    const int64_t t0 = tile * 32;
    // K slices of tokens qr + 8m, V bytes [8qr, 8qr + 8) of tokens 2qc + {0, 1, 8, 9} + 16ks
    uint4 kc[4];
    uint2 vc[2][4];
    float kn[4], vn[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int64_t t = t0 + qr + 8 * m;
      const bool ok = t < a.T;
      const int64_t n = ok ? t * a.hkv + g : 0;
      kc[m] = ok ? __ldcs(reinterpret_cast<const uint4*>(a.k_codes + n * 64) + qc) : make_uint4(0u, 0u, 0u, 0u);
      kn[m] = ok ? __ldcs(a.k_norms + n) : 0.f;
      vn[m] = ok ? __ldcs(a.v_norms + n) : 0.f;
    }
#pragma unroll
    for (int ks = 0; ks < 2; ++ks)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t t = t0 + 16 * ks + 2 * qc + (j & 1) + 8 * (j >> 1);
        const bool ok = t < a.T;
        vc[ks][j] = ok ? __ldcs(reinterpret_cast<const uint2*>(a.v_codes + (t * a.hkv + g) * 64) + qr)
                       : make_uint2(0u, 0u);
      }

    // A. scores
    float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int wi = kk >> 1, pos = 2 * (kk & 1);
      const uint2 b = bq[(kk >> 1) * 64 + (kk & 1)];  // words 2kk, 2kk + 1 of the lane's fragment
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint32_t lo = word4(kc[2 * mt], wi), hi = word4(kc[2 * mt + 1], wi);
        mma16816(sacc[mt], pair_at(lo, pos, kcol), pair_at(hi, pos, kcol), pair_at(lo, pos + 1, kcol),
                 pair_at(hi, pos + 1, kcol), b.x, b.y);
      }
    }

    // B. online softmax per head (base 2); value weights to the transpose buffer
    float lv[4];  // log2 ν^V: −inf for a zero norm and for a token past T
#pragma unroll
    for (int m = 0; m < 4; ++m) lv[m] = lg2(vn[m]);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * qc + e;
      float s[4], z[4];
      float mt = -INFINITY, zt = -INFINITY;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const bool ok = t0 + qr + 8 * m < a.T;
        s[m] = ok ? kse[e] * kn[m] * sacc[m >> 1][2 * (m & 1) + e] : -INFINITY;
        z[m] = s[m] + lv[m];
        mt = fmaxf(mt, s[m]);
        zt = fmaxf(zt, z[m]);
      }
#pragma unroll
      for (int sh = 4; sh < 32; sh <<= 1) {
        mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, sh));
        zt = fmaxf(zt, __shfl_xor_sync(kFull, zt, sh));
      }
      const float mn = fmaxf(m_run[e], mt);  // finite: the tile holds a valid token
      const float zn = fmaxf(M_run[e], zt);  // −inf while every value norm so far is 0
      const bool live = zn != -INFINITY;
      const float alpha = ex2(m_run[e] - mn);            // 0 on the first tile
      const float beta = live ? ex2(M_run[e] - zn) : 0.f;
      const float zb = zn - kWBias;
      float ps = 0.f;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        ps += ex2(s[m] - mn);  // 0 for a token past T
        const float w = live ? ex2(z[m] - zb) : 0.f;
        if (h < G) wbuf[h * kWRow + qr + 8 * m] = __float2half_rn(w);
      }
#pragma unroll
      for (int sh = 4; sh < 32; sh <<= 1) ps += __shfl_xor_sync(kFull, ps, sh);
      l_run[e] = l_run[e] * alpha + ps;
      m_run[e] = mn;
      M_run[e] = zn;
#pragma unroll
      for (int mt2 = 0; mt2 < 8; ++mt2) {
        o[mt2][e] *= beta;
        o[mt2][2 + e] *= beta;
      }
    }
    __syncwarp();

    // C. O^T += levels(V)^T · W^T
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const uint32_t* wr = reinterpret_cast<const uint32_t*>(wbuf + qr * kWRow + 16 * ks + 2 * qc);
      const uint32_t b0 = wr[0], b1 = wr[4];  // tokens 16ks + 2qc, +1 and +8, +9 of head qr
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int wi = mt >> 2, pos = mt & 3;
        const uint32_t p0 = pair_at(word2(vc[ks][0], wi), pos, vcol);  // token 2qc
        const uint32_t p1 = pair_at(word2(vc[ks][1], wi), pos, vcol);  // token 2qc + 1
        const uint32_t p8 = pair_at(word2(vc[ks][2], wi), pos, vcol);  // token 2qc + 8
        const uint32_t p9 = pair_at(word2(vc[ks][3], wi), pos, vcol);  // token 2qc + 9
        mma16816(o[mt], __byte_perm(p0, p1, 0x5410u), __byte_perm(p0, p1, 0x7632u),
                 __byte_perm(p8, p9, 0x5410u), __byte_perm(p8, p9, 0x7632u), b0, b1);
      }
    }
    __syncwarp();  // the buffer is read before the next tile writes it
  }

  // ---- merge the warps' states: CTA maxima per head, then rescaled sums by
  // shared-memory atomics.  Accumulator o[mt][i]: coordinate 16qr + 2mt + (i >> 1),
  // head 2qc + (i & 1).
  if (qr == 0) {
#pragma unroll
    for (int e = 0; e < 2; ++e)
      if (2 * qc + e < G) {
        wmax[warp * 2 * G + 2 * qc + e] = m_run[e];
        wmax[warp * 2 * G + G + 2 * qc + e] = M_run[e];
      }
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int h = 2 * qc + e;
    if (h < G) {
      float mx = -INFINITY, zx = -INFINITY;
      for (int w = 0; w < kAWarps; ++w) {
        mx = fmaxf(mx, wmax[w * 2 * G + h]);
        zx = fmaxf(zx, wmax[w * 2 * G + G + h]);
      }
      const float fl = m_run[e] == -INFINITY ? 0.f : ex2(m_run[e] - mx);
      const float fo = M_run[e] == -INFINITY ? 0.f : ex2(M_run[e] - zx);
      float* oh = part + 3 * G + h * kAD + 16 * qr;
      if (fo > 0.f) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          atomicAdd(oh + 2 * mt, fo * o[mt][e]);
          atomicAdd(oh + 2 * mt + 1, fo * o[mt][2 + e]);
        }
      }
      if (fl > 0.f && qr == 0) atomicAdd(part + G + h, fl * l_run[e]);
      if (warp == 0 && qr == 0) {
        part[h] = mx;
        part[2 * G + h] = zx;
      }
    }
  }
  __syncthreads();

  // ---- this CTA's state to the workspace; the kv head's last CTA merges them all
  unsigned* counter = a.counters + g;
  float* states = a.states + int64_t(g) * S * L::PART_FLOATS;
  for (int i = tid; i < L::PART_FLOATS; i += kAThreads) __stcg(states + sidx * L::PART_FLOATS + i, part[i]);
  __threadfence();  // the state is visible device-wide before the count says so
  __syncthreads();
  if (tid == 0) *last_flag = atomicAdd(counter, 1u) == unsigned(S - 1) ? 1 : 0;
  __syncthreads();
  if (*last_flag == 0) return;
  __threadfence();
  for (int idx = tid; idx < G * (kAD + 1); idx += kAThreads) {
    const int j = idx / (kAD + 1), c = idx % (kAD + 1);
    // the sums of the value product (c < kAD) carry the maximum M, the softmax
    // denominator (c = kAD) the maximum m.  Unrolled so that each batch of loads
    // is in flight at once (the order of the additions is unchanged).
    const int mo = c < kAD ? 2 * G + j : j;
    float mx = -INFINITY;
#pragma unroll 8
    for (int r = 0; r < S; ++r) mx = fmaxf(mx, __ldcg(states + r * L::PART_FLOATS + mo));
    float acc = 0.f;
#pragma unroll 8
    for (int r = 0; r < S; ++r) {
      const float* pr = states + r * L::PART_FLOATS;
      const float m = __ldcg(pr + mo);
      const float f = m == -INFINITY ? 0.f : ex2(m - mx);
      acc += f * __ldcg(c < kAD ? pr + 3 * G + j * kAD + c : pr + G + j);
    }
    if (c < kAD) {
      fin[j * kAD + c] = acc;  // Σ over every token of the rotated-domain sum
    } else {
      float zx = -INFINITY;
#pragma unroll 8
      for (int r = 0; r < S; ++r) zx = fmaxf(zx, __ldcg(states + r * L::PART_FLOATS + 2 * G + j));
      fin[G * kAD + j] = acc;                // the softmax denominator
      fin[G * kAD + G + j] = zx == -INFINITY ? 0.f : ex2(zx - mx - kWBias);  // 2^(M − m − kWBias)
    }
  }
  if (tid == 0) *counter = 0u;  // every CTA of this kv head has counted: ready for the next call
  __syncthreads();
  for (int j = warp; j < G; j += kAWarps) {
    const float lsum = fin[G * kAD + j];
    const float inv = lsum > 0.f ? fin[G * kAD + G + j] / lsum : 0.f;
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = fin[j * kAD + lane * 4 + k] * inv;
    fwht128(v, lane);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = lane * 4 + k;
      const float y = v[k] * a.pv.inv_d;  // 1/√d of the reconstruction, 1/√d of Πᵀ
      a.out[int64_t(g * G + j) * kAD + i] = sign_bit(a.pv.seed, i) ? -y : y;
    }
  }
}

template <int G>
cudaError_t launch_g(const AttnArgs& a, cudaStream_t stream) {
  auto k = attention_decode_kernel<G>;
  int dev = 0, reserved = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  if (e != cudaSuccess) return e;
  if (uint32_t(reserved) != ALayout<G>::kBase) return cudaErrorNotSupported;
  constexpr int smem = ALayout<G>::TOTAL;
  e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k), cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, a.hkv * a.splits, kAThreads, smem, stream, a);
}

}  // namespace

int attention_splits(int hkv, int group, int64_t T) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  (void)group;  // one CTA per SM for every group
  // rounded down: one CTA more than the SMs hold would run as a second wave and
  // double the kernel's time
  int64_t s = int64_t(sms) / hkv;
  const int64_t ntile = (T + 31) / 32;
  const int64_t most = (ntile + kAWarps - 1) / kAWarps;  // every CTA gets a tile per warp
  if (s > most) s = most;
  return int(s < 1 ? 1 : s);
}

size_t attention_workspace_bytes(int hq, int hkv, int64_t T) {
  const int s = attention_splits(hkv, hq / hkv, T);
  const size_t counters = (size_t(hkv) * 4 + 255) / 256 * 256;
  return counters + size_t(hq) * s * (kAD + 3) * 4;
}

// ------------------------------------------------ allocation-free variant
// Scratch of the allocation-free entry point: a fixed array in the library's own
// device image, present on every GPU that loads the library until the process
// exits.  Host code reaches it only through the address cudaGetSymbolAddress
// reports for the current device (the array's name in host code is a stand-in).
static __device__ __align__(256) uint8_t g_attention_scratch[kAttentionScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// The array's address on the current device, looked up once per device.
cudaError_t attention_scratch(void** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attention_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return cudaSuccess;
}

cudaError_t launch_attention_decode_in_scratch(AttnArgs a, cudaStream_t stream) {
  void* base = nullptr;
  cudaError_t e = attention_scratch(&base);
  if (e != cudaSuccess) return e;
  const size_t counters = (size_t(a.hkv) * 4 + 255) / 256 * 256;
  // the counters must start at zero; the previous call's partial states need not
  e = cudaMemsetAsync(base, 0, counters, stream);
  if (e != cudaSuccess) return e;
  a.counters = static_cast<unsigned*>(base);
  a.states = reinterpret_cast<float*>(static_cast<uint8_t*>(base) + counters);
  return launch_attention_decode(a, stream);
}

cudaError_t launch_attention_decode(const AttnArgs& a, cudaStream_t stream) {
  switch (a.group) {
    case 1: return launch_g<1>(a, stream);
    case 2: return launch_g<2>(a, stream);
    case 4: return launch_g<4>(a, stream);
    case 8: return launch_g<8>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rrq

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
// M a running maximum of z (moved only when a tile exceeds it by more than
// one, which spares most tiles the rescaling of the value sums): every weight
// is below 2^(kWBias + 1), none overflows, and only terms below 2^-(23 + kWBias)
// of the largest one flush, at any scale of the value norms.  The softmax denominator
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
constexpr int kAWarps = 12;
constexpr int kAThreads = kAWarps * 32;
constexpr int kWRow = 40;  // fp16 weights per head row of a warp's transpose buffer (padded)
constexpr int kRS = 80;    // ring row: 64 code bytes + 16 bytes of padding (conflict-free reads)
constexpr int kNS = 2;     // ring stages per warp
constexpr int kMaxSplits = 160;  // token ranges per kv head: at most one per SM
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
// address).  The level-pair table sits at the 64 KB-aligned address 0x10000, K
// pairs in the first 128 bytes of each 256-byte row and V pairs in the second,
// so that a byte permute of a code byte and the lane column (byte·256 |
// lane·4 | table, + 128 for V) is the load address itself.  The warps' rings
// and transpose buffers fill the space below and above the table.
template <int G> struct ALayout {
  static constexpr uint32_t kBase = 0x400;
  static constexpr uint32_t kTable = 0x10000, kTableEnd = 0x20000;
  static constexpr uint32_t QF = 0;                              // [G][kAD] fp32 q' (prologue)
  static constexpr uint32_t INV = QF + G * kAD * 4;              // [G] 1/s
  static constexpr uint32_t WM = (INV + G * 4 + 15) / 16 * 16;   // [kAWarps][2G] warp maxima m, M
  static constexpr int PART_FLOATS = 3 * G + G * kAD;           // [G] m, [G] l, [G] M, [G][kAD] o
  static constexpr uint32_t PART = WM + kAWarps * 2 * G * 4;     // the CTA's partial state
  static constexpr uint32_t FLAG = PART + PART_FLOATS * 4;       // "this CTA merges its kv head"
  static constexpr uint32_t FIN = (FLAG + 16 + 15) / 16 * 16;    // the merging CTA's sums [G][kAD], [G] l, [G] M − m, [2][G] maxima
  static constexpr uint32_t HEAD_END = FIN + (G * (kAD + 2) + 2 * G) * 4;
  // per warp: kNS ring stages (K rows, V rows, K norms, V norms), then the
  // transpose buffer [8][kWRow] fp16
  static constexpr uint32_t KROW = 0, VROW = 32 * kRS, KN = 64 * kRS, VN = KN + 128;
  static constexpr uint32_t STAGE = VN + 128;
  static constexpr uint32_t WBUF = kNS * STAGE;
  static constexpr uint32_t WB = (WBUF + 8 * kWRow * 2 + 127) / 128 * 128;
  static constexpr uint32_t FRONT = (kBase + HEAD_END + 127) / 128 * 128;
  static constexpr int NFRONT = (kTable - FRONT) / WB < uint32_t(kAWarps) ? int((kTable - FRONT) / WB) : kAWarps;
  static constexpr uint32_t warp_base(int w) {  // shared address of warp w's buffers
    return w < NFRONT ? FRONT + uint32_t(w) * WB : kTableEnd + uint32_t(w - NFRONT) * WB;
  }
  static constexpr uint32_t TOTAL = (warp_base(kAWarps) > kTableEnd ? warp_base(kAWarps) : kTableEnd) - kBase;
  static_assert(WB >= 2 * kMaxSplits * G * 4, "the merge's per-state values fit warp 0's buffers");
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
//  0. The tile's K and V code rows and norms arrive in the warp's cp.async ring
//     (kNS stages, 80-byte rows), loaded one tile ahead.
//  A. scores S[32 tokens × 8] = levels(K codes)·q'' as in the score kernel:
//     the thread's tokens are 4qr + j (j = 2mt + h is row qr + 8h of m-tile
//     mt), its code slice is bytes [16qc, 16qc + 16), columns 2qc, 2qc + 1 its
//     heads.
//  B. the online softmax per head on those fragments, in base 2 (maxima and
//     sum over the tile by shuffles across the 8 lanes of equal qc); the value
//     weights 2^(z − M + kWBias) go to the warp's transpose buffer as fp16
//     [head][token], four tokens in one 8-byte store.
//  C. O^T[128 × 8] += levels(V codes)^T·W^T: coordinates are M, heads N,
//     tokens K.  Row qr of m-tile mt is coordinate 2(8qr + mt) and row qr + 8
//     coordinate 2(8qr + mt) + 1, so both come from V byte 8qr + mt; for the
//     token pair of a fragment column the two bytes are first merged nibble by
//     nibble (the two tokens' codes of one coordinate in one byte), so each A
//     register is one level-pair lookup.  The output
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
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem + (L::kTable - L::kBase));
  float* qf = reinterpret_cast<float*>(smem + L::QF);
  float* inv_s = reinterpret_cast<float*>(smem + L::INV);
  float* wmax = reinterpret_cast<float*>(smem + L::WM);
  float* part = reinterpret_cast<float*>(smem + L::PART);
  int* last_flag = reinterpret_cast<int*>(smem + L::FLAG);
  float* fin = reinterpret_cast<float*>(smem + L::FIN);
  const uint32_t wbase = L::warp_base(warp);
  __half* wbuf = reinterpret_cast<__half*>(smem + (wbase - L::kBase) + L::WBUF);

  // ---- level tables from the parameters alone: K entry e at e·256 + lane·4,
  // V entry at e·256 + 128 + lane·4
  for (int i = tid; i < 256 * 32; i += kAThreads) {
    const int e = i >> 5, l = i & 31;
    const __half2 kv = __floats2half2_rn(a.pk.levels[e & 15], a.pk.levels[e >> 4]);
    const __half2 vv = __floats2half2_rn(a.pv.levels[e & 15], a.pv.levels[e >> 4]);
    tab[e * 64 + l] = *reinterpret_cast<const uint32_t*>(&kv);
    tab[e * 64 + 32 + l] = *reinterpret_cast<const uint32_t*>(&vv);
  }
  // weight rows of the padding heads (G..7) stay zero
  for (int i = lane; i < 8 * kWRow; i += 32) wbuf[i] = __float2half_rn(0.f);
  for (int i = tid; i < L::PART_FLOATS; i += kAThreads) part[i] = 0.f;
  pdl_wait();  // from here on, global memory

  // ---- tiles of kv head g: tile = warp·S + sidx + k·S·kAWarps, so all
  // addresses advance by constant steps; the ring runs one tile ahead
  const int64_t ntile = (a.T + 31) / 32;
  const int64_t tstride = int64_t(S) * kAWarps;
  const int64_t tile0 = int64_t(warp) * S + sidx;
  const int64_t my_tiles = tile0 < ntile ? (ntile - tile0 + tstride - 1) / tstride : 0;
  const int64_t row_bytes = int64_t(a.hkv) * 64;  // between tokens
  const int lt = lane >> 2, lc = lane & 3;        // copy k: row lt + 8k, 16-byte chunk lc
  const int64_t step_rows = tstride * 32;
  const uint8_t* ksrc = a.k_codes + (tile0 * 32 + lt) * row_bytes + g * 64 + lc * 16;
  const uint8_t* vsrc = a.v_codes + (tile0 * 32 + lt) * row_bytes + g * 64 + lc * 16;
  const float* knsrc = a.k_norms + (tile0 * 32 + lane) * a.hkv + g;
  const float* vnsrc = a.v_norms + (tile0 * 32 + lane) * a.hkv + g;
  int64_t t_next = tile0 * 32;
  int64_t issued = 0;
  const uint32_t lane_dst = uint32_t(lt * kRS + lc * 16);
  auto issue = [&](int stage) {
    if (issued < my_tiles) {
      const uint32_t sb = wbase + uint32_t(stage) * L::STAGE;
      if (t_next + 32 <= a.T) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          cp_async16(sb + L::KROW + lane_dst + k * 8 * kRS, ksrc + k * 8 * row_bytes, 16);
          cp_async16(sb + L::VROW + lane_dst + k * 8 * kRS, vsrc + k * 8 * row_bytes, 16);
        }
        cp_async4(sb + L::KN + lane * 4, knsrc, 4);
        cp_async4(sb + L::VN + lane * 4, vnsrc, 4);
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const bool ok = t_next + lt + 8 * k < a.T;
          cp_async16(sb + L::KROW + lane_dst + k * 8 * kRS, ok ? ksrc + k * 8 * row_bytes : a.k_codes, ok ? 16 : 0);
          cp_async16(sb + L::VROW + lane_dst + k * 8 * kRS, ok ? vsrc + k * 8 * row_bytes : a.v_codes, ok ? 16 : 0);
        }
        const bool ok = t_next + lane < a.T;
        cp_async4(sb + L::KN + lane * 4, ok ? knsrc : a.k_norms, ok ? 4 : 0);
        cp_async4(sb + L::VN + lane * 4, ok ? vnsrc : a.v_norms, ok ? 4 : 0);
      }
      ++issued;
      ksrc += step_rows * row_bytes;
      vsrc += step_rows * row_bytes;
      knsrc += step_rows * a.hkv;
      vnsrc += step_rows * a.hkv;
      t_next += step_rows;
    }
    cp_async_commit();
  };
#pragma unroll
  for (int k = 0; k < kNS - 1; ++k) issue(k);

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

  const int qc = lane & 3, qr = lane >> 2;
  // this lane's B fragments: k-step kk, word j is the pair β = 16qc + 2kk + j of
  // head qr's q'' (zero for qr ≥ G)
  uint32_t bq[8][2];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int beta = 16 * qc + 2 * kk + j;
      __half2 v = __floats2half2_rn(0.f, 0.f);
      if (qr < G) v = __floats2half2_rn(qf[qr * kAD + 2 * beta], qf[qr * kAD + 2 * beta + 1]);
      bq[kk][j] = *reinterpret_cast<const uint32_t*>(&v);
    }
  float kse[2];  // log2(e)·scale·inv_d/s of heads 2qc + e: scores in base 2
#pragma unroll
  for (int e = 0; e < 2; ++e)
    kse[e] = 2 * qc + e < G ? kLog2e * a.scale * a.pk.inv_d * inv_s[2 * qc + e] : 0.f;
  const uint32_t kcol = L::kTable | uint32_t(lane) * 4u;
  const uint32_t vcol = kcol | 128u;

  // per head: score maximum m, denominator l, maximum M of z = s + log2 ν^V
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f}, M_run[2] = {-INFINITY, -INFINITY};
  float o[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  int stage = 0;
  int64_t t0 = tile0 * 32;
  for (int64_t k = 0; k < my_tiles; ++k) {
    cp_async_wait<kNS - 2>();
    __syncwarp();
    const uint8_t* st = smem + (wbase - L::kBase) + stage * L::STAGE;
    // K slices of tokens 4qr + j; V bytes [8qr, 8qr + 8) of tokens 2qc + {0, 1, 8, 9} + 16ks
    uint4 kc[4];
    uint2 vc[2][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) kc[j] = *reinterpret_cast<const uint4*>(st + L::KROW + (4 * qr + j) * kRS + 16 * qc);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        vc[ks][j] = *reinterpret_cast<const uint2*>(st + L::VROW + (16 * ks + 2 * qc + (j & 1) + 8 * (j >> 1)) * kRS + 8 * qr);
    const float4 kn4 = *reinterpret_cast<const float4*>(st + L::KN + 16 * qr);
    const float4 vn4 = *reinterpret_cast<const float4*>(st + L::VN + 16 * qr);
    __syncwarp();  // every lane has read this stage before it is refilled
    issue(stage == 0 ? kNS - 1 : stage - 1);
    stage = (stage + 1 == kNS) ? 0 : stage + 1;

    // A. scores
    float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int wi = kk >> 1, pos = 2 * (kk & 1);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint32_t lo = word4(kc[2 * mt], wi), hi = word4(kc[2 * mt + 1], wi);
        mma16816(sacc[mt], pair_at(lo, pos, kcol), pair_at(hi, pos, kcol), pair_at(lo, pos + 1, kcol),
                 pair_at(hi, pos + 1, kcol), bq[kk][0], bq[kk][1]);
      }
    }

    // B. online softmax per head (base 2); value weights to the transpose buffer
    const float kn[4] = {kn4.x, kn4.y, kn4.z, kn4.w};
    float lv[4] = {lg2(vn4.x), lg2(vn4.y), lg2(vn4.z), lg2(vn4.w)};  // −inf for a zero norm
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * qc + e;
      float s[4], z[4];
      float mt = -INFINITY, zt = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool ok = t0 + 4 * qr + j < a.T;
        s[j] = ok ? kse[e] * kn[j] * sacc[j >> 1][2 * (j & 1) + e] : -INFINITY;
        z[j] = s[j] + lv[j];
        mt = fmaxf(mt, s[j]);
        zt = fmaxf(zt, z[j]);
      }
#pragma unroll
      for (int sh = 4; sh < 32; sh <<= 1) {
        mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, sh));
        zt = fmaxf(zt, __shfl_xor_sync(kFull, zt, sh));
      }
      const float mn = fmaxf(m_run[e], mt);  // finite: the tile holds a valid token
      // M moves (and the value sums are rescaled) only when the tile's maximum
      // exceeds it by more than one: the weights then stay below 2^(kWBias + 1)
      const bool moved = zt > M_run[e] + 1.f || M_run[e] == -INFINITY;
      const float zn = moved ? fmaxf(M_run[e], zt) : M_run[e];  // −inf while every norm so far is 0
      const bool live = zn != -INFINITY;
      const float alpha = ex2(m_run[e] - mn);  // 0 on the first tile
      const float zb = zn - kWBias;
      float ps = 0.f;
      __half w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        ps += ex2(s[j] - mn);  // 0 for a token past T
        w[j] = __float2half_rn(live ? ex2(z[j] - zb) : 0.f);
      }
      if (h < G) {
        const __half2 w01 = __halves2half2(w[0], w[1]), w23 = __halves2half2(w[2], w[3]);
        *reinterpret_cast<uint2*>(wbuf + h * kWRow + 4 * qr) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&w01), *reinterpret_cast<const uint32_t*>(&w23));
      }
#pragma unroll
      for (int sh = 4; sh < 32; sh <<= 1) ps += __shfl_xor_sync(kFull, ps, sh);
      l_run[e] = l_run[e] * alpha + ps;
      m_run[e] = mn;
      if (moved) {
        const float beta = live ? ex2(M_run[e] - zn) : 0.f;  // 0 on the first move
#pragma unroll
        for (int mt2 = 0; mt2 < 8; ++mt2) {
          o[mt2][e] *= beta;
          o[mt2][2 + e] *= beta;
        }
      }
      M_run[e] = zn;
    }
    __syncwarp();

    // C. O^T += levels(V)^T · W^T
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const uint32_t* wr = reinterpret_cast<const uint32_t*>(wbuf + qr * kWRow + 16 * ks + 2 * qc);
      const uint32_t b0 = wr[0], b1 = wr[4];  // tokens 16ks + 2qc, +1 and +8, +9 of head qr
      // byte b of lo[i] (hi[i]) holds the low (high) nibbles of byte b of the two
      // tokens 2qc + 8i and 2qc + 8i + 1: the codes of coordinate 2(4w + b)
      // (+1) for the token pair, looked up as one level pair = one A register
      uint32_t lo[2][2], hi[2][2];
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const uint32_t t0w = word2(vc[ks][2 * i], w), t1w = word2(vc[ks][2 * i + 1], w);
          lo[i][w] = (t0w & 0x0F0F0F0Fu) | ((t1w << 4) & 0xF0F0F0F0u);
          hi[i][w] = ((t0w >> 4) & 0x0F0F0F0Fu) | (t1w & 0xF0F0F0F0u);
        }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int wi = mt >> 2, pos = mt & 3;
        mma16816(o[mt], pair_at(lo[0][wi], pos, vcol), pair_at(hi[0][wi], pos, vcol),
                 pair_at(lo[1][wi], pos, vcol), pair_at(hi[1][wi], pos, vcol), b0, b1);
      }
    }
    __syncwarp();  // the buffer is read before the next tile writes it
    t0 += step_rows;
  }
  cp_async_wait<0>();

  // ---- merge the warps' states: CTA maxima per head; each warp writes its sums,
  // rescaled to them, into its own (now idle) buffers; then every thread adds a
  // column over the warps.  Accumulator o[mt][i]: coordinate 16qr + 2mt + (i >> 1),
  // head 2qc + (i & 1).  (Shared-memory float atomics here serialised the lanes:
  // ≈ 7 µs of a 60 µs launch.)
  if (qr == 0) {
#pragma unroll
    for (int e = 0; e < 2; ++e)
      if (2 * qc + e < G) {
        wmax[warp * 2 * G + 2 * qc + e] = m_run[e];
        wmax[warp * 2 * G + G + 2 * qc + e] = M_run[e];
      }
  }
  __syncthreads();
  {
    // this warp's [G][kAD] rescaled sums, then [G] rescaled denominators
    float* ws = reinterpret_cast<float*>(smem + (L::warp_base(warp) - L::kBase));
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
        float* oh = ws + h * kAD + 16 * qr;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
          *reinterpret_cast<float2*>(oh + 2 * mt) = make_float2(fo * o[mt][e], fo * o[mt][2 + e]);
        if (qr == 0) ws[G * kAD + h] = fl * l_run[e];
        if (warp == 0 && qr == 0) {
          part[h] = mx;
          part[2 * G + h] = zx;
        }
      }
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * (kAD + 1); idx += kAThreads) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kAWarps; ++w)
      acc += reinterpret_cast<const float*>(smem + (L::warp_base(w) - L::kBase))[idx];
    if (idx < G * kAD) part[3 * G + idx] = acc;  // rotated-domain sums
    else part[G + idx - G * kAD] = acc;          // softmax denominators
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
  // The merge, in three short passes over shared memory and one over the
  // states: (1) every state's maxima m_r, M_r; (2) the heads' maxima; (3) the
  // factors 2^(m_r − m) and 2^(M_r − M); then every sum (the 128 rotated-domain
  // sums carry M, the denominator m) as one batch of independent loads per
  // thread.  Warp 0's buffers, idle now, hold the per-state values.
  float* mm = reinterpret_cast<float*>(smem + (L::warp_base(0) - L::kBase));  // [S][G] m_r, then factors
  float* zz = mm + S * G;                                                    // [S][G] M_r, then factors
  float* hx = fin + G * (kAD + 2);  // [2][G] head maxima (after the FIN sums)
  for (int i = tid; i < S * G; i += kAThreads) {
    const int r = i / G, j = i % G;
    mm[i] = __ldcg(states + r * L::PART_FLOATS + j);
    zz[i] = __ldcg(states + r * L::PART_FLOATS + 2 * G + j);
  }
  __syncthreads();
  if (tid < 2 * G) {
    const float* src = tid < G ? mm : zz;
    const int j = tid % G;
    float mx = -INFINITY;
    for (int r = 0; r < S; ++r) mx = fmaxf(mx, src[r * G + j]);
    hx[tid] = mx;
  }
  __syncthreads();
  for (int i = tid; i < S * G; i += kAThreads) {
    const int j = i % G;
    mm[i] = mm[i] == -INFINITY ? 0.f : ex2(mm[i] - hx[j]);
    zz[i] = zz[i] == -INFINITY ? 0.f : ex2(zz[i] - hx[G + j]);
  }
  __syncthreads();
  for (int idx = tid; idx < G * (kAD + 1); idx += kAThreads) {
    const int j = idx / (kAD + 1), c = idx % (kAD + 1);
    const float* fac = c < kAD ? zz : mm;
    const float* src = states + (c < kAD ? 3 * G + j * kAD + c : G + j);
    float acc = 0.f;
#pragma unroll 16
    for (int r = 0; r < S; ++r) acc += fac[r * G + j] * __ldcg(src + r * L::PART_FLOATS);
    if (c < kAD) {
      fin[j * kAD + c] = acc;  // Σ over every token of the rotated-domain sum
    } else {
      fin[G * kAD + j] = acc;  // the softmax denominator
      const float zx = hx[G + j];
      fin[G * kAD + G + j] = zx == -INFINITY ? 0.f : ex2(zx - hx[j] - kWBias);  // 2^(M − m − kWBias)
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
  if (s > kMaxSplits) s = kMaxSplits;
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

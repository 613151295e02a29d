// attention_gen.cu — decode attention over a quantised K/V cache for the shapes
// the fused kernel (attention.cu, d = 128 with 4-bit K and V) does not take:
// d ∈ {64, 128, 256, 512}, 1- to 4-bit K and V codes, GQA group ∈ {1, 2, 4, 8}.
//
// "Attn-rot (TurboQuant lite) in llama.cpp" page, "What kind of beast is
// Attn-rot": keys and values both quantised after a rotation;
// "Random-rotation quantization" page, "Three decoders, one rotation": the MSE
// decoder, x̃ = Πᵀ(ν/√d · c[code]).  With g = ⌊h·hkv/hq⌋ and Πᵀ = D·H/√d:
//     s[h,t]  = scale · ⟨q_h, k̂_{t,g}⟩,
//     out[h]  = Σ_t p[h,t]·v̂_{t,g} = D·H·( Σ_t e^{s[h,t] − M}·ν^V_t·c_V[code_t] ) / (d·Σ_t e^{s[h,t] − M}),
// with M any common shift (the largest score of the head here), so the values
// are summed in their rotated domain and rotated back once per head.
//
// Two launches.  The scores are the score kernel's (rrq_qk_scores: tensor-core
// tiles on the packed K codes, every d and bit width), written to the
// workspace.  Then one CTA per (kv head, token range): the range's per-head
// maximum of the scores; each warp walks its tokens in batches of 32 (lane j
// computes token j's weights e^{s − m}·ν for the group's heads and puts them in
// the warp's shared-memory buffer), lane l owning coordinates [l·d/32,
// (l + 1)·d/32) of every row — it reads the 32-bit words that hold its b·d/32
// code bits (the loads of 32 rows, 16 for wide 3-bit rows, issued before any is
// used, no branch between them), takes each level from the lane that holds it
// (one shuffle) and each row's weights from the buffer (one broadcast read), and
// adds w·c into its fp32 sums; the bit width is a template parameter, so every
// shift is a constant.  Warps meet through shared-memory atomics, the CTA writes its state
// (m, Σ e^{s−m}, d sums per head) to the workspace and counts itself in its kv
// head's counter; the CTA that counts last merges the ranges, applies D·H (a
// shared-memory Walsh–Hadamard transform per head), writes the output and sets
// the counter back to zero.  No CTA waits for another.  Everything is fp32.
#include <cmath>

#include "attention.h"
#include "rrq_device.cuh"

namespace rrq {
namespace {

constexpr int kGWarps = 8;
constexpr int kGThreads = kGWarps * 32;
constexpr int kGMaxSplits = 444;  // token ranges per kv head: at most three CTAs per SM in all

// Words of a V row that lane `lane` reads: its B·CPL code bits start at bit
// lane·B·CPL of the row (bit i of the row = bit i mod 8 of byte i / 8,
// coordinate j at bits [j·B, (j + 1)·B)).  kWin words hold them once shifted
// down by `off`; a 3-bit lane's bits may start inside a word and end inside the
// next, so it reads one word more, the word index kept inside the row (a word
// past the lane's bits only fills bits above them).
// Rows whose loads are in flight together: 32, or 16 where the words of 32 rows
// and the G × CPL sums would not fit the 128 registers of two CTAs per SM.
template <int G, int B, int CPL> struct VRow {
  static constexpr int kRowWords = B * CPL;                 // 32-bit words of a row
  static constexpr int kWin = (B * CPL + 31) / 32;          // words of the lane's bits
  static constexpr int kNW = kWin + (B == 3 ? 1 : 0);       // words read per row
  static constexpr int kRows = kNW == 1 && G * CPL <= 32 ? 32 : 16;
};

template <int G, int CPL, int B>
__global__ void __launch_bounds__(kGThreads) attention_value_kernel(const AttnGenArgs a) {
  using R = VRow<G, B, CPL>;
  constexpr int D = 32 * CPL;
  __shared__ float s_acc[G * D];     // the CTA's sums, then the merged sums
  __shared__ __align__(16) float s_w[kGWarps][32][G];  // a warp's batch of weights, token-major
  __shared__ float s_max[kGWarps][G];
  __shared__ float s_f[kGMaxSplits * G];  // the merge's per-range maxima, then factors
  __shared__ float s_m[G], s_l[G];
  __shared__ int s_last;
  pdl_release();
  pdl_wait();  // the scores come from the previous launch
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = blockIdx.x / a.splits, r = blockIdx.x % a.splits;
  const int64_t per = (a.T + a.splits - 1) / a.splits;
  const int64_t t0 = int64_t(r) * per, t1 = t0 + per < a.T ? t0 + per : a.T;
  const float* sc = a.scores + int64_t(g) * G * a.T;  // [G][T] of this kv head's heads
  for (int i = tid; i < G * D; i += kGThreads) s_acc[i] = 0.f;
  if (tid < G) s_l[tid] = 0.f;

  // ---- the range's largest score per head
  float mh[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float m = -INFINITY;
#pragma unroll 4
    for (int64_t t = t0 + tid; t < t1; t += kGThreads) m = fmaxf(m, sc[int64_t(h) * a.T + t]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    if (lane == 0) s_max[warp][h] = m;
  }
  __syncthreads();
  if (tid < G) {
    float m = s_max[0][tid];
    for (int w = 1; w < kGWarps; ++w) m = fmaxf(m, s_max[w][tid]);
    s_m[tid] = m;
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < G; ++h) mh[h] = s_m[h];

  // ---- Σ_t e^{s − m}·ν·c over the warp's tokens, coordinates [lane·CPL, +CPL)
  // Lane i holds level i mod 2^B, so a shuffle whose source lane has the code in
  // its low B bits (whatever lies above them) fetches that code's level.
  const float lev = a.pv.levels[lane & ((1 << B) - 1)];
  const int bit0 = lane * B * CPL;
  const int w0 = bit0 >> 5, off = bit0 & 31;
  int wo[R::kNW];  // the lane's word offsets within a row
#pragma unroll
  for (int k = 0; k < R::kNW; ++k) wo[k] = (w0 + k < R::kRowWords ? w0 + k : R::kRowWords - 1);
  const int stride = a.hkv * R::kRowWords;  // words from one token's row to the next
  const uint32_t* vrows = reinterpret_cast<const uint32_t*>(a.v_codes) + int64_t(g) * R::kRowWords;
  float acc[G][CPL];
  float lsum[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    lsum[h] = 0.f;
#pragma unroll
    for (int j = 0; j < CPL; ++j) acc[h][j] = 0.f;
  }
  // batches of 32 tokens per warp: lane j takes token j's scores and norm
  // (coalesced) and puts its weights in the warp's buffer; every lane reads its
  // words of the batch's rows, all loads of a group of rows issued before any of
  // them is used.  Rows past the range's end repeat its last row with weight 0.
  for (int64_t tb = t0 + int64_t(warp) * 32; tb < t1; tb += int64_t(kGWarps) * 32) {
    const int nt = int(t1 - tb < 32 ? t1 - tb : 32);
    const bool mine = lane < nt;
    const int64_t t = tb + lane;
    float sv[G];
#pragma unroll
    for (int h = 0; h < G; ++h) sv[h] = mine ? sc[int64_t(h) * a.T + t] : -INFINITY;
    const float nu = mine ? __ldg(a.v_norms + t * a.hkv + g) : 0.f;
    const uint32_t* rows = vrows + tb * stride;
    float wl[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      wl[h] = mine ? __expf(sv[h] - mh[h]) : 0.f;
      lsum[h] += wl[h];
      wl[h] *= nu;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) s_w[warp][lane][h] = wl[h];
    __syncwarp();
#pragma unroll
    for (int j0 = 0; j0 < 32; j0 += R::kRows) {
      uint32_t cw[R::kRows][R::kNW];
#pragma unroll
      for (int j = 0; j < R::kRows; ++j) {
        const int row = j0 + j < nt ? j0 + j : nt - 1;
#pragma unroll
        for (int k = 0; k < R::kNW; ++k) cw[j][k] = __ldg(rows + row * stride + wo[k]);
      }
#pragma unroll
      for (int j = 0; j < R::kRows; ++j) {
        float w[G];
#pragma unroll
        for (int h = 0; h < G; ++h) w[h] = s_w[warp][j0 + j][h];
        uint32_t u[R::kWin + 1];  // the lane's bits from bit 0 on
#pragma unroll
        for (int k = 0; k < R::kWin; ++k) {
          if constexpr (B == 3) u[k] = __funnelshift_r(cw[j][k], cw[j][k + 1], off);
          else if constexpr (R::kWin == 1) u[k] = cw[j][0] >> off;
          else u[k] = cw[j][k];  // B·CPL ≥ 32: the lane's bits start at a word
        }
        u[R::kWin] = 0u;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          constexpr int kB = B;
          const int bit = c * kB, k = bit >> 5, sh = bit & 31;
          const uint32_t code = sh + kB > 32 ? __funnelshift_r(u[k], u[k + 1], sh) : u[k] >> sh;
          const float lv = __shfl_sync(kFull, lev, int(code));  // lane = code mod 32
#pragma unroll
          for (int h = 0; h < G; ++h) acc[h][c] = fmaf(w[h], lv, acc[h][c]);
        }
      }
    }
    __syncwarp();  // the buffer is rewritten by the next batch
  }
  // the lanes' shares of the softmax sums
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lsum[h] += __shfl_xor_sync(kFull, lsum[h], o);
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int j = 0; j < CPL; ++j) atomicAdd(&s_acc[h * D + lane * CPL + j], acc[h][j]);
    if (lane == 0) atomicAdd(&s_l[h], lsum[h]);
  }
  __syncthreads();

  // ---- this range's state: [G] m, [G] l, [G][D] sums
  float* st = a.states + (int64_t(g) * a.splits + r) * G * (D + 2);
  for (int i = tid; i < G * (D + 2); i += kGThreads)
    st[i] = i < G ? s_m[i] : i < 2 * G ? s_l[i - G] : s_acc[i - 2 * G];
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(a.counters + g, 1u) == unsigned(a.splits - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- the last range of kv head g: merge the ranges' states, in three short
  // passes over shared memory and one over the states: every state's maxima,
  // the heads' maxima (warp h reduces head h), the factors e^{m_q − m}; then each
  // thread's sums (and the denominators) as batches of independent loads
  const int S = a.splits;
  const int64_t sstride = int64_t(G) * (D + 2);
  const float* st0 = a.states + int64_t(g) * S * sstride;
  for (int i = tid; i < S * G; i += kGThreads) s_f[i] = __ldcg(st0 + (i / G) * sstride + i % G);
  __syncthreads();
  if (warp < G) {
    float m = -INFINITY;
    for (int q = lane; q < S; q += 32) m = fmaxf(m, s_f[q * G + warp]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    if (lane == 0) s_m[warp] = m;
  }
  __syncthreads();
  for (int i = tid; i < S * G; i += kGThreads) {
    const float mq = s_f[i];
    s_f[i] = mq == -INFINITY ? 0.f : __expf(mq - s_m[i % G]);  // an empty range adds nothing
  }
  __syncthreads();
  for (int idx = tid; idx < G * (D + 1); idx += kGThreads) {
    const int h = idx / (D + 1), c = idx % (D + 1);
    const float* src = st0 + (c < D ? 2 * G + h * D + c : G + h);
    float v = 0.f;
#pragma unroll 16
    for (int q = 0; q < S; ++q) v = fmaf(s_f[q * G + h], __ldcg(src + q * sstride), v);
    if (c < D) s_acc[h * D + c] = v;
    else s_l[h] = v;
  }
  __syncthreads();
  // H (unnormalised, Sylvester order) per head, in place
  for (int len = 1; len < D; len <<= 1) {
    for (int i = tid; i < G * D / 2; i += kGThreads) {
      const int h = i / (D / 2), k = i % (D / 2);
      const int p0 = h * D + (k / len) * 2 * len + (k % len), p1 = p0 + len;
      const float x0 = s_acc[p0], x1 = s_acc[p1];
      s_acc[p0] = x0 + x1;
      s_acc[p1] = x0 - x1;
    }
    __syncthreads();
  }
  for (int i = tid; i < G * D; i += kGThreads) {
    const int h = i / D, c = i % D;
    const float l = s_l[h];
    const float y = l > 0.f ? s_acc[i] / (float(D) * l) : 0.f;
    a.out[int64_t(g * G + h) * D + c] = sign_bit(a.pv.seed, c) ? -y : y;
  }
  if (tid == 0) a.counters[g] = 0u;  // ready for the next call
}

using ValueKernel = void (*)(AttnGenArgs);

// The value kernel for (G, d, V bits), or null where none is built.
template <int G, int B> ValueKernel value_kernel_d(int d) {
  switch (d) {
    case 64: return attention_value_kernel<G, 2, B>;
    case 128: return attention_value_kernel<G, 4, B>;
    case 256: return attention_value_kernel<G, 8, B>;
    case 512:
      if constexpr (G <= 4) return attention_value_kernel<G, 16, B>;
      break;
  }
  return nullptr;
}
template <int G> ValueKernel value_kernel_g(int d, int bits) {
  switch (bits) {
    case 1: return value_kernel_d<G, 1>(d);
    case 2: return value_kernel_d<G, 2>(d);
    case 3: return value_kernel_d<G, 3>(d);
    case 4: return value_kernel_d<G, 4>(d);
  }
  return nullptr;
}
ValueKernel value_kernel(int group, int d, int bits) {
  switch (group) {
    case 1: return value_kernel_g<1>(d, bits);
    case 2: return value_kernel_g<2>(d, bits);
    case 4: return value_kernel_g<4>(d, bits);
    case 8: return value_kernel_g<8>(d, bits);
  }
  return nullptr;
}

// CTAs of the value kernel for (group, d, V bits) that one SM holds at once, at most three
int value_ctas_per_sm(int group, int d, int v_bits) {
  const ValueKernel k = value_kernel(group, d, v_bits);
  int n = 1;
  if (k == nullptr ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, reinterpret_cast<const void*>(k), kGThreads, 0) !=
          cudaSuccess ||
      n < 1)
    n = 1;
  return n > 3 ? 3 : n;
}

}  // namespace

int attention_general_splits(int hkv, int group, int d, int v_bits, int64_t T) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // as many CTAs as the SMs hold at once (at most three each), so the grid is one wave
  int64_t s = int64_t(value_ctas_per_sm(group, d, v_bits)) * sms / hkv;
  if (s > kGMaxSplits) s = kGMaxSplits;
  const int64_t most = (T + 4 * kGWarps - 1) / (4 * kGWarps);  // at least 4 tokens per warp
  if (s > most) s = most;
  return int(s < 1 ? 1 : s);
}

bool attention_general_supported(int d, int k_bits, int hq, int hkv) {
  const int group = hkv > 0 ? hq / hkv : 0;
  if (group != 1 && group != 2 && group != 4 && group != 8) return false;
  if (d != 64 && d != 128 && d != 256 && d != 512) return false;
  if (d == 512 && group == 8) return false;  // 8 × 16 sums per lane exceed the registers
  return qk_scores_supported(d, k_bits, hq, hkv);
}

// counters (padded to 256 bytes) | states hkv × splits × G × (d + 2) floats
// (padded to 256 bytes) | scores hq × T floats
size_t attention_general_workspace_bytes(int hq, int hkv, int d, int v_bits, int64_t T) {
  const int s = attention_general_splits(hkv, hkv > 0 ? hq / hkv : 1, d, v_bits, T);
  const size_t counters = (size_t(hkv) * 4 + 255) / 256 * 256;
  const size_t states = (size_t(hq) * s * (d + 2) * 4 + 255) / 256 * 256;
  return counters + states + size_t(hq) * size_t(T) * 4;
}

cudaError_t launch_attention_general(AttnGenArgs a, void* workspace, cudaStream_t stream) {
  a.splits = attention_general_splits(a.hkv, a.group, a.d, a.pv.bits, a.T);
  const size_t counters = (size_t(a.hkv) * 4 + 255) / 256 * 256;
  const size_t states = (size_t(a.hq) * a.splits * (a.d + 2) * 4 + 255) / 256 * 256;
  a.counters = static_cast<unsigned*>(workspace);
  a.states = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + counters);
  a.scores = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + counters + states);
  cudaError_t e = launch_qk_scores(a.q, a.hq, a.k_codes, a.k_norms, a.T, a.hkv, a.d, a.pk, a.scale, a.scores,
                                   stream);
  if (e != cudaSuccess) return e;
  const ValueKernel k = value_kernel(a.group, a.d, a.pv.bits);
  if (k == nullptr) return cudaErrorNotSupported;
  return launch_pdl(k, a.hkv * a.splits, kGThreads, 0, stream, a);
}

}  // namespace rrq

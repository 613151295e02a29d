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
// computes token j's weights e^{s − m}·ν for the group's heads), lane l owning
// coordinates [l·d/32, (l + 1)·d/32) of every row — it reads the 32-bit words
// that hold its b·d/32 code bits (a batch's 32 rows in flight at once), takes each
// level from the lane that holds it (one shuffle) and each weight from the
// token's lane, and adds w·c into its fp32 sums; warps meet through shared-memory atomics, the CTA writes its state
// (m, Σ e^{s−m}, d sums per head) to the workspace and counts itself in its kv
// head's counter; the CTA that counts last merges the ranges, applies D·H (a
// shared-memory Walsh–Hadamard transform per head), writes the output and sets
// the counter back to zero.  No CTA waits for another.  Everything is fp32.
#include <cmath>
#include <type_traits>

#include "attention.h"
#include "rrq_device.cuh"

namespace rrq {
namespace {

constexpr int kGWarps = 8;
constexpr int kGThreads = kGWarps * 32;
constexpr int kGMaxSplits = 296;  // token ranges per kv head: at most two CTAs per SM in all

// The lane's b·CPL code bits of row `row` (bit i of the row = bit i mod 8 of byte
// i / 8, coordinate j at bits [j·b, (j + 1)·b)), as the low bits of a 64-bit word.
template <int CPL>
__device__ __forceinline__ uint64_t lane_bits(const uint8_t* __restrict__ row, int lane, int b) {
  const int start = lane * CPL * b;            // first bit of the lane
  const int w0 = start >> 5, off = start & 31;  // its 32-bit word and the offset in it
  const int nbits = CPL * b;                    // ≤ 64
  const uint32_t* rw = reinterpret_cast<const uint32_t*>(row);
  uint64_t v = __ldg(rw + w0);
  if (off + nbits > 32) v |= uint64_t(__ldg(rw + w0 + 1)) << 32;
  v >>= off;
  if (off + nbits > 64) v |= uint64_t(__ldg(rw + w0 + 2)) << (64 - off);
  return v;
}

template <int G, int CPL>
__global__ void __launch_bounds__(kGThreads) attention_value_kernel(const AttnGenArgs a) {
  constexpr int D = 32 * CPL;
  __shared__ float s_acc[G * D];     // the CTA's sums, then the merged sums
  __shared__ float s_max[kGWarps][G];
  __shared__ float s_m[G], s_l[G];
  __shared__ int s_last;
  pdl_release();
  pdl_wait();  // the scores come from the previous launch
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = blockIdx.x / a.splits, r = blockIdx.x % a.splits;
  const int64_t per = (a.T + a.splits - 1) / a.splits;
  const int64_t t0 = int64_t(r) * per, t1 = t0 + per < a.T ? t0 + per : a.T;
  const int bv = a.pv.bits;
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
  const float lev = a.pv.levels[lane & 15];  // lane i < 2^b holds level i
  const uint64_t mask = (uint64_t(1) << bv) - 1;
  const int64_t rowbytes = int64_t(D) * bv / 8;
  float acc[G][CPL];
  float lsum[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    lsum[h] = 0.f;
#pragma unroll
    for (int j = 0; j < CPL; ++j) acc[h][j] = 0.f;
  }
  // batches of 32 tokens per warp: lane j takes token j's scores and norm (coalesced)
  // and every lane its code bits of all 32 rows, all loads of a batch issued
  // before any of them is used
  for (int64_t tb = t0 + int64_t(warp) * 32; tb < t1; tb += int64_t(kGWarps) * 32) {
    const int nt = int(t1 - tb < 32 ? t1 - tb : 32);
    const bool mine = lane < nt;
    const int64_t t = tb + lane;
    float sv[G];
#pragma unroll
    for (int h = 0; h < G; ++h) sv[h] = mine ? sc[int64_t(h) * a.T + t] : -INFINITY;
    const float nu = mine ? __ldg(a.v_norms + t * a.hkv + g) : 0.f;
    uint64_t cw[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
      cw[j] = j < nt ? lane_bits<CPL>(a.v_codes + ((tb + j) * a.hkv + g) * rowbytes, lane, bv) : 0;
    float wl[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      wl[h] = mine ? __expf(sv[h] - mh[h]) : 0.f;
      lsum[h] += wl[h];
      wl[h] *= nu;
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j >= nt) break;
      float w[G];
#pragma unroll
      for (int h = 0; h < G; ++h) w[h] = __shfl_sync(kFull, wl[h], j);
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const float lv = __shfl_sync(kFull, lev, int((cw[j] >> (c * bv)) & mask));
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h][c] = fmaf(w[h], lv, acc[h][c]);
      }
    }
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

  // ---- the last range of kv head g: merge the ranges' states
  const float* st0 = a.states + int64_t(g) * a.splits * G * (D + 2);
  if (tid < G) {
    float m = -INFINITY;
    for (int q = 0; q < a.splits; ++q) m = fmaxf(m, __ldcg(st0 + int64_t(q) * G * (D + 2) + tid));
    float l = 0.f;
    for (int q = 0; q < a.splits; ++q) {
      const float* sq = st0 + int64_t(q) * G * (D + 2);
      const float mq = __ldcg(sq + tid);
      if (mq != -INFINITY) l += __ldcg(sq + G + tid) * __expf(mq - m);
    }
    s_m[tid] = m;
    s_l[tid] = l;
  }
  __syncthreads();
  for (int i = tid; i < G * D; i += kGThreads) {
    const int h = i / D;
    float v = 0.f;
    for (int q = 0; q < a.splits; ++q) {
      const float* sq = st0 + int64_t(q) * G * (D + 2);
      const float mq = __ldcg(sq + h);
      if (mq != -INFINITY) v = fmaf(__ldcg(sq + 2 * G + i), __expf(mq - s_m[h]), v);
    }
    s_acc[i] = v;
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

template <int G>
cudaError_t launch_value_g(const AttnGenArgs& a, cudaStream_t stream) {
  const int grid = a.hkv * a.splits;
  switch (a.d) {
    case 64: return launch_pdl(attention_value_kernel<G, 2>, grid, kGThreads, 0, stream, a);
    case 128: return launch_pdl(attention_value_kernel<G, 4>, grid, kGThreads, 0, stream, a);
    case 256: return launch_pdl(attention_value_kernel<G, 8>, grid, kGThreads, 0, stream, a);
    case 512:
      if constexpr (G <= 4) return launch_pdl(attention_value_kernel<G, 16>, grid, kGThreads, 0, stream, a);
      break;
  }
  return cudaErrorNotSupported;
}

// CTAs of the value kernel for (group, d) that one SM holds at once
int value_ctas_per_sm(int group, int d) {
  const void* k = nullptr;
  auto pick = [&](auto g) {
    constexpr int G = decltype(g)::value;
    switch (d) {
      case 64: k = reinterpret_cast<const void*>(attention_value_kernel<G, 2>); break;
      case 128: k = reinterpret_cast<const void*>(attention_value_kernel<G, 4>); break;
      case 256: k = reinterpret_cast<const void*>(attention_value_kernel<G, 8>); break;
      case 512:
        if constexpr (G <= 4) k = reinterpret_cast<const void*>(attention_value_kernel<G, 16>);
        break;
    }
  };
  switch (group) {
    case 1: pick(std::integral_constant<int, 1>()); break;
    case 2: pick(std::integral_constant<int, 2>()); break;
    case 4: pick(std::integral_constant<int, 4>()); break;
    case 8: pick(std::integral_constant<int, 8>()); break;
  }
  int n = 1;
  if (k == nullptr || cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kGThreads, 0) != cudaSuccess || n < 1)
    n = 1;
  return n > 2 ? 2 : n;
}

}  // namespace

int attention_general_splits(int hkv, int group, int d, int64_t T) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // as many CTAs as the SMs hold at once (at most two each), so the grid is one wave
  int64_t s = int64_t(value_ctas_per_sm(group, d)) * sms / hkv;
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
size_t attention_general_workspace_bytes(int hq, int hkv, int d, int64_t T) {
  const int s = attention_general_splits(hkv, hkv > 0 ? hq / hkv : 1, d, T);
  const size_t counters = (size_t(hkv) * 4 + 255) / 256 * 256;
  const size_t states = (size_t(hq) * s * (d + 2) * 4 + 255) / 256 * 256;
  return counters + states + size_t(hq) * size_t(T) * 4;
}

cudaError_t launch_attention_general(AttnGenArgs a, void* workspace, cudaStream_t stream) {
  a.splits = attention_general_splits(a.hkv, a.group, a.d, a.T);
  const size_t counters = (size_t(a.hkv) * 4 + 255) / 256 * 256;
  const size_t states = (size_t(a.hq) * a.splits * (a.d + 2) * 4 + 255) / 256 * 256;
  a.counters = static_cast<unsigned*>(workspace);
  a.states = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + counters);
  a.scores = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + counters + states);
  cudaError_t e = launch_qk_scores(a.q, a.hq, a.k_codes, a.k_norms, a.T, a.hkv, a.d, a.pk, a.scale, a.scores,
                                   stream);
  if (e != cudaSuccess) return e;
  switch (a.group) {
    case 1: return launch_value_g<1>(a, stream);
    case 2: return launch_value_g<2>(a, stream);
    case 4: return launch_value_g<4>(a, stream);
    case 8: return launch_value_g<8>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rrq

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
// Work split.  The cache of kv head g is cut into S token ranges, one CTA each
// (grid hkv × S, about two CTAs per SM); a CTA serves the GQA group of G query
// heads of its kv head, and its warps take tiles of 32 consecutive tokens:
//  A. one token per lane: the lane loads its K row (64 B), scores the G heads
//     with packed fp16 FMAs on a lane-replicated table of level pairs (as the
//     score kernel), and the warp updates its running softmax state (max, sum)
//     per head; the lane writes its weights w_h = p_h·ν^V/√d to the warp buffer.
//  B. four coordinates per lane: the warp reads the tile's V rows (two bytes
//     per lane per token, 64 contiguous bytes per token, all 32 loads in flight
//     at once), looks each byte up in a table of fp32 level pairs (16 copies,
//     one per lane of a half-warp) and accumulates w_h times them into fp32
//     partial sums (packed FMAs).
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
constexpr int kAP = kAD / 2;
constexpr int kAWarps = 8;
constexpr int kAThreads = kAWarps * 32;

template <int G> struct ALayout {
  static constexpr int KTAB = 0;                               // [256][32] half2 (K level pairs)
  static constexpr int VTAB = KTAB + 256 * 32 * 4;             // [256][16] float2 (V level pairs)
  static constexpr int QH = VTAB + 256 * 16 * 8;               // [kAP][G] half2 q''
  static constexpr int INV = QH + kAP * G * 4;                 // [G] 1/s
  static constexpr int WBUF = (INV + G * 4 + 15) / 16 * 16;    // per warp: weights [32][G]
  static constexpr int WM = WBUF + kAWarps * 32 * G * 4;       // [kAWarps][G] warp maxima
  static constexpr int PART_FLOATS = 2 * G + G * kAD;         // [G] m, [G] l, [G][kAD] o
  static constexpr int PART = WM + kAWarps * G * 4;            // the CTA's partial state
  static constexpr int FLAG = PART + PART_FLOATS * 4;          // "this CTA merges its kv head"
  static constexpr int TOTAL = FLAG + 16;
  static constexpr int FIN = KTAB;  // the last CTA's merged sums reuse the level tables
  static_assert(G * (kAD + 1) * 4 <= VTAB, "merged sums fit over the K table");
  static_assert(TOTAL <= 110 * 1024, "two CTAs per SM");
};

struct KRow {
  uint4 k[4];
  float kn, vn;
};

__device__ __forceinline__ void load_krow(KRow& r, const AttnArgs& a, int64_t t, int g) {
  if (t < a.T) {
    const int64_t n = t * a.hkv + g;
    const uint4* kp = reinterpret_cast<const uint4*>(a.k_codes + n * 64);
#pragma unroll
    for (int i = 0; i < 4; ++i) r.k[i] = __ldcs(kp + i);
    r.kn = __ldcs(a.k_norms + n);
    r.vn = __ldcs(a.v_norms + n);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) r.k[i] = make_uint4(0u, 0u, 0u, 0u);
    r.kn = r.vn = 0.f;
  }
}

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

// Two CTAs per SM (≤ 128 registers) where the group's accumulators allow it.
template <int G> constexpr int attention_min_blocks() { return G <= 4 ? 2 : 1; }

template <int G>
__global__ void __launch_bounds__(kAThreads, attention_min_blocks<G>()) attention_decode_kernel(const AttnArgs a) {
  pdl_release();
  using L = ALayout<G>;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* ktab = reinterpret_cast<uint32_t*>(smem + L::KTAB);
  float2* vtab = reinterpret_cast<float2*>(smem + L::VTAB);
  __half2* qh = reinterpret_cast<__half2*>(smem + L::QH);
  float* inv_s = reinterpret_cast<float*>(smem + L::INV);
  float* part = reinterpret_cast<float*>(smem + L::PART);
  float* fin = reinterpret_cast<float*>(smem + L::FIN);
  int* last_flag = reinterpret_cast<int*>(smem + L::FLAG);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = a.splits;
  const int g = blockIdx.x / S, sidx = blockIdx.x % S;
  float* wbuf = reinterpret_cast<float*>(smem + L::WBUF) + warp * 32 * G;
  float* wmax = reinterpret_cast<float*>(smem + L::WM);

  // ---- level tables from the parameters alone
  for (int i = tid; i < 256 * 32; i += kAThreads) {
    const int e = i >> 5;
    const __half2 kv = __floats2half2_rn(a.pk.levels[e & 15], a.pk.levels[e >> 4]);
    ktab[i] = *reinterpret_cast<const uint32_t*>(&kv);
  }
  // 16 copies suffice for the fp32 pairs: a 64-bit shared load serves each half-warp
  // in its own pass, so lanes l and l + 16 never meet in one
  for (int i = tid; i < 256 * 16; i += kAThreads)
    vtab[i] = make_float2(a.pv.levels[(i >> 4) & 15], a.pv.levels[i >> 8]);
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
    qh[(2 * lane) * G + j] = __floats2half2_rn(v[0] * s, v[1] * s);
    qh[(2 * lane + 1) * G + j] = __floats2half2_rn(v[2] * s, v[3] * s);
    if (lane == 0) inv_s[j] = 1.f / s;
  }
  __syncthreads();

  // ---- token tiles of kv head g (warp-major over the S CTAs' warps)
  const int64_t ntile = (a.T + 31) / 32;
  const int64_t stride = int64_t(S) * kAWarps;
  int64_t tile = int64_t(warp) * S + sidx;
  const float kscale = a.scale * a.pk.inv_d;
  const float vscale = a.pv.inv_sqrt_d;
  const uint32_t* ktab_l = ktab + lane;
  const float2* vtab_l = vtab + (lane & 15);
  float m_run[G], l_run[G];
  float2 o[G][2];  // coordinates 4·lane .. 4·lane+3 of each head's rotated-domain sum
#pragma unroll
  for (int j = 0; j < G; ++j) {
    m_run[j] = -INFINITY;
    l_run[j] = 0.f;
    o[j][0] = o[j][1] = make_float2(0.f, 0.f);
  }
  for (; tile < ntile; tile += stride) {
    const int64_t t = tile * 32 + lane;
    KRow cur;
    load_krow(cur, a, t, g);
    // the tile's V code bytes for this lane's four coordinates, all in flight now
    uint32_t vb[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int64_t tu = tile * 32 + u;
      vb[u] = tu < a.T ? uint32_t(__ldcs(reinterpret_cast<const uint16_t*>(
                             a.v_codes + (tu * a.hkv + g) * 64) + lane))
                       : 0u;
    }
    // A. scores of this lane's token
    const uint32_t* kw = reinterpret_cast<const uint32_t*>(cur.k);
    float sc[G];
#pragma unroll
    for (int j = 0; j < G; ++j) sc[j] = 0.f;
#pragma unroll
    for (int f = 0; f < kAP / 16; ++f) {
      __half2 hs[G];
#pragma unroll
      for (int j = 0; j < G; ++j) hs[j] = __float2half2_rn(0.f);
#pragma unroll
      for (int pp = 0; pp < 16; ++pp) {
        const int pr = f * 16 + pp;
        const uint32_t byte = (kw[pr >> 2] >> (8 * (pr & 3))) & 255u;
        const uint32_t cw = ktab_l[byte << 5];
        const __half2 c2 = *reinterpret_cast<const __half2*>(&cw);
#pragma unroll
        for (int j = 0; j < G; ++j) hs[j] = __hfma2(qh[pr * G + j], c2, hs[j]);
      }
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float2 s2 = __half22float2(hs[j]);
        sc[j] += s2.x + s2.y;
      }
    }
    const bool valid = t < a.T;
    float alpha[G];
#pragma unroll
    for (int j = 0; j < G; ++j) {
      const float s = valid ? kscale * cur.kn * inv_s[j] * sc[j] : -INFINITY;
      float mt = s;
#pragma unroll
      for (int m = 16; m > 0; m >>= 1) mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, m));
      const float mn = fmaxf(m_run[j], mt);  // finite: the tile holds a valid token
      alpha[j] = __expf(m_run[j] - mn);
      const float pj = valid ? __expf(s - mn) : 0.f;
      float ps = pj;
#pragma unroll
      for (int m = 16; m > 0; m >>= 1) ps += __shfl_xor_sync(kFull, ps, m);
      l_run[j] = l_run[j] * alpha[j] + ps;
      m_run[j] = mn;
      wbuf[lane * G + j] = pj * cur.vn * vscale;
    }
#pragma unroll
    for (int j = 0; j < G; ++j) {
      o[j][0] = make_float2(o[j][0].x * alpha[j], o[j][0].y * alpha[j]);
      o[j][1] = make_float2(o[j][1].x * alpha[j], o[j][1].y * alpha[j]);
    }
    __syncwarp();
    // B. weighted sum of the tile's V rows, four coordinates per lane
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const float2 c0 = vtab_l[(vb[u] & 255u) << 4], c1 = vtab_l[(vb[u] >> 8) << 4];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float w = wbuf[u * G + j];
        o[j][0] = __ffma2_rn(c0, make_float2(w, w), o[j][0]);
        o[j][1] = __ffma2_rn(c1, make_float2(w, w), o[j][1]);
      }
    }
    __syncwarp();
  }

  // ---- merge the warps' states: CTA maximum per head, then rescaled sums by
  // shared-memory atomics
  if (lane == 0) {
#pragma unroll
    for (int jj = 0; jj < G; ++jj) wmax[warp * G + jj] = m_run[jj];
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < G; ++j) {
    float mx = -INFINITY;
    for (int w = 0; w < kAWarps; ++w) mx = fmaxf(mx, wmax[w * G + j]);
    const float f = m_run[j] == -INFINITY ? 0.f : __expf(m_run[j] - mx);
    float* oj = part + 2 * G + j * kAD + 4 * lane;
    if (f > 0.f) {
      atomicAdd(oj, f * o[j][0].x);
      atomicAdd(oj + 1, f * o[j][0].y);
      atomicAdd(oj + 2, f * o[j][1].x);
      atomicAdd(oj + 3, f * o[j][1].y);
      if (lane == 0) atomicAdd(part + G + j, f * l_run[j]);
    }
    if (tid == 0) part[j] = mx;
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
    float mx = -INFINITY;
    for (int r = 0; r < S; ++r) mx = fmaxf(mx, __ldcg(states + r * L::PART_FLOATS + j));
    float acc = 0.f;
    for (int r = 0; r < S; ++r) {
      const float* pr = states + r * L::PART_FLOATS;
      const float m = __ldcg(pr + j);
      const float f = m == -INFINITY ? 0.f : __expf(m - mx);
      acc += f * __ldcg(c < kAD ? pr + 2 * G + j * kAD + c : pr + G + j);
    }
    if (c < kAD) fin[j * kAD + c] = acc;  // Σ over every token of the rotated-domain sum
    else fin[G * kAD + j] = acc;        // the softmax denominator
  }
  if (tid == 0) *counter = 0u;  // every CTA of this kv head has counted: ready for the next call
  __syncthreads();
  for (int j = warp; j < G; j += kAWarps) {
    const float lsum = fin[G * kAD + j];
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = fin[j * kAD + lane * 4 + k] * inv;
    fwht128(v, lane);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = lane * 4 + k;
      const float y = v[k] * a.pv.inv_sqrt_d;
      a.out[int64_t(g * G + j) * kAD + i] = sign_bit(a.pv.seed, i) ? -y : y;
    }
  }
}

template <int G>
cudaError_t launch_g(const AttnArgs& a, cudaStream_t stream) {
  auto k = attention_decode_kernel<G>;
  constexpr int smem = ALayout<G>::TOTAL;
  const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, a.hkv * a.splits, kAThreads, smem, stream, a);
}

}  // namespace

int attention_splits(int hkv, int group, int64_t T) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int per_sm = group <= 4 ? 2 : 1;  // the CTAs an SM holds (registers)
  int64_t s = (int64_t(per_sm) * sms + hkv - 1) / hkv;
  const int64_t ntile = (T + 31) / 32;
  const int64_t most = (ntile + kAWarps - 1) / kAWarps;  // every CTA gets a tile per warp
  if (s > most) s = most;
  return int(s < 1 ? 1 : s);
}

size_t attention_workspace_bytes(int hq, int hkv, int64_t T) {
  const int s = attention_splits(hkv, hq / hkv, T);
  const size_t counters = (size_t(hkv) * 4 + 255) / 256 * 256;
  return counters + size_t(hq) * s * (kAD + 2) * 4;
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

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
// Work split.  A cluster of C CTAs serves one kv head g and its GQA group of G
// query heads; its warps take tiles of 32 consecutive tokens.  Per tile:
//  A. one token per lane: the lane loads its K row (64 B), scores the G heads
//     with packed fp16 FMAs on a lane-replicated table of level pairs (as the
//     score kernel), and the warp updates its running softmax state (max, sum)
//     per head; the lane writes its weights w_h = p_h·ν^V/√d to the warp buffer.
//  B. four coordinates per lane: the warp reads the tile's V rows (two bytes
//     per lane per token, 64 contiguous bytes per token, all 32 loads in flight
//     at once), looks each byte up in a table of fp32 level pairs (16 copies,
//     one per lane of a half-warp) and accumulates w_h times them into fp32
//     partial sums (packed FMAs).
// At the end the warps' states merge within the CTA (shared-memory atomics after
// a common rescaling), and the CTAs' within the cluster through distributed
// shared memory: rank 0 reads every CTA's partial sums, normalises, applies Πᵀ
// (a 128-point transform per head) and writes out.  16 warps and under 96 KB of
// shared memory per CTA, so that 16-CTA clusters of every kv head are resident
// together.
#include <cooperative_groups.h>

#include <cmath>
#include <mutex>

#include "attention.h"
#include "rrq_device.cuh"

namespace cg = cooperative_groups;

namespace rrq {
namespace {

constexpr int kAD = 128;
constexpr int kAP = kAD / 2;
constexpr int kAWarps = 16;
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
  static constexpr int FIN = PART + PART_FLOATS * 4;           // rank 0: [G][kAD] sums, [G] denominators
  static constexpr int TOTAL = FIN + G * (kAD + 1) * 4;
  static_assert(TOTAL <= 96 * 1024, "two CTAs per SM, so 16-CTA clusters of 8 kv heads fit");
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

template <int G>
__global__ void __launch_bounds__(kAThreads, 1) attention_decode_kernel(const AttnArgs a) {
  pdl_release();
  using L = ALayout<G>;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* ktab = reinterpret_cast<uint32_t*>(smem + L::KTAB);
  float2* vtab = reinterpret_cast<float2*>(smem + L::VTAB);
  __half2* qh = reinterpret_cast<__half2*>(smem + L::QH);
  float* inv_s = reinterpret_cast<float*>(smem + L::INV);
  float* part = reinterpret_cast<float*>(smem + L::PART);
  float* fin = reinterpret_cast<float*>(smem + L::FIN);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  cg::cluster_group cluster = cg::this_cluster();
  const int C = int(cluster.num_blocks()), rank = int(cluster.block_rank());
  const int g = blockIdx.x / C;
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

  // ---- token tiles of kv head g (warp-major over the cluster's warps)
  const int64_t ntile = (a.T + 31) / 32;
  const int64_t stride = int64_t(C) * kAWarps;
  int64_t tile = int64_t(warp) * C + rank;
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
  // shared-memory atomics; then the CTAs' states across the cluster
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
  cluster.sync();
  if (rank == 0) {
    for (int idx = tid; idx < G * (kAD + 1); idx += kAThreads) {
      const int j = idx / (kAD + 1), c = idx % (kAD + 1);
      float mx = -INFINITY;
      for (int r = 0; r < C; ++r) mx = fmaxf(mx, cluster.map_shared_rank(part, r)[j]);
      float acc = 0.f;
      for (int r = 0; r < C; ++r) {
        const float* pr = cluster.map_shared_rank(part, r);
        const float f = mx == -INFINITY ? 0.f : __expf(pr[j] - mx);
        acc += f * (c < kAD ? pr[2 * G + j * kAD + c] : pr[G + j]);
      }
      if (c < kAD) fin[j * kAD + c] = acc;  // Σ over every token of the rotated-domain sum
      else fin[G * kAD + j] = acc;        // the softmax denominator
    }
  }
  cluster.sync();  // the other CTAs' shared memory stays alive until rank 0 has read it
  if (rank == 0) {
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
}

// Cluster sizes found for (group size, device, hkv), a fixed table (no heap
// memory); 0 = not yet known.  When the table is full a choice is simply
// searched again on the next call.
struct ClusterChoice {
  int g, dev, hkv, c;
};
constexpr int kClusterChoices = 64;
std::mutex g_cluster_mu;
ClusterChoice g_cluster_choices[kClusterChoices];
int g_cluster_count = 0;

int cached_cluster_size(int g, int dev, int hkv) {
  std::lock_guard<std::mutex> lock(g_cluster_mu);
  for (int i = 0; i < g_cluster_count; ++i) {
    const ClusterChoice& c = g_cluster_choices[i];
    if (c.g == g && c.dev == dev && c.hkv == hkv) return c.c;
  }
  return 0;
}

void remember_cluster_size(int g, int dev, int hkv, int c) {
  std::lock_guard<std::mutex> lock(g_cluster_mu);
  if (g_cluster_count < kClusterChoices) g_cluster_choices[g_cluster_count++] = {g, dev, hkv, c};
}

template <int G>
cudaError_t launch_g(const AttnArgs& a, cudaStream_t stream) {
  auto k = attention_decode_kernel<G>;
  constexpr int smem = ALayout<G>::TOTAL;
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                           cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  // cluster size: the largest C ≤ 16 for which the clusters of every kv head can
  // be resident together (one wave), found once per (device, hkv) by occupancy
  // queries, and no larger than the cache needs
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int cmax = cached_cluster_size(G, dev, a.hkv);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  auto configure = [&](int c) {
    cfg.gridDim = dim3(unsigned(a.hkv * c));
    cfg.blockDim = dim3(kAThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(c);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  };
  if (cmax == 0) {
    int fallback = 0;
    for (int c = 16; c >= 1; --c) {
      configure(c);
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, reinterpret_cast<const void*>(k), &cfg) !=
          cudaSuccess) {
        (void)cudaGetLastError();
        continue;
      }
      if (fallback == 0 && clusters > 0) fallback = c;  // the largest that runs at all
      if (clusters >= a.hkv) {                            // every kv head at once
        cmax = c;
        break;
      }
    }
    if (cmax == 0) cmax = fallback;
    if (cmax == 0) return cudaErrorInvalidConfiguration;
    remember_cluster_size(G, dev, a.hkv, cmax);
  }
  const int64_t ntile = (a.T + 31) / 32;
  int C = cmax;
  while (C > 1 && int64_t(C - 1) * kAWarps >= ntile) --C;  // no idle CTAs on short caches
  configure(C);
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k, a);
}

}  // namespace

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

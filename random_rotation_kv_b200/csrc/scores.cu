// scores.cu — decode-time attention scores straight from packed codes.
//
// "Random-rotation quantization" page, "Three decoders, one rotation",
// inner-product decoder: <q, x> is recovered from <Πq, code(Πx)> and a
// normalising scalar.  With q' = H·D·q = √d·Πq:
//     s[h][t] = scale · (ν_{t,g}/d) · Σ_i q'_{h,i} · c[code_{t,g,i}],  g = ⌊h·hkv/hq⌋,
// which equals scale·<q_h, x̂_{t,g}> without ever forming x̂.
//
// Layout.  Each lane owns 32 consecutive coordinates of a key-head row
// (d/32 lanes per key-head; KPW = 1024/d key-heads per warp iteration).  A
// lane's GQA group of GQ query heads is fixed for the whole kernel, so its
// slice of the rotated queries lives in registers as fp16 pairs, scaled per
// head by a power of two so |q''| ≤ 1 (the scale is undone in fp32).
// Per key-head the lane looks up its 16 code pairs in a table of fp16 level
// pairs (c_lo, c_hi), replicated per lane so every lane reads its own bank,
// and accumulates GQ dot products with packed fp16 FMAs, folding into fp32
// every 8 pairs.  The d/32 partial sums are combined with shuffles.
//
// Data movement.  Each warp streams its rows through a cp.async ring (one
// iteration = KPW contiguous rows, 32 lanes × 16 B per instruction); scores
// of a tile of TT tokens × hq heads are staged in shared memory and written
// head-major with 16-byte stores.
#include <type_traits>

#include "rrq_device.cuh"

namespace rrq {
namespace {

constexpr int kScoreWarps = 8;
constexpr int kScoreThreads = kScoreWarps * 32;
constexpr int kScoreTile = 128;  // tokens per CTA tile
constexpr int kScoreStages = 4;  // ring depth

struct ScoreArgs {
  const __half* q;
  const uint8_t* codes;
  const float* norms;
  float* scores;
  int64_t T;
  int hq, hkv, group;
  float scale;
  QuantParams p;
};

template <int D, int B>
struct ScoreGeom {
  static constexpr int LPK = D / 32;               // lanes per key-head
  static constexpr int KPW = 32 / LPK;             // key-heads per warp iteration
  static constexpr int CB = D * B / 8;             // code bytes per key-head
  static constexpr int LB = 4 * B;                 // code bytes per lane (32 codes)
  static constexpr int IT_BYTES = KPW * CB;        // codes per iteration (= 128·B)
  static constexpr int NPAIR = 16;                 // code pairs per lane
  static constexpr int TABLE_WORDS = (1 << (2 * B)) * 32;
  static constexpr int RING_STAGE = (IT_BYTES + KPW * 4 + 15) / 16 * 16;  // codes | norms
};

// Shared memory: pair table | q'' (fp16 pairs) | inverse head scales | score tile | rings
template <int D, int B>
struct ScoreSmem {
  using Gm = ScoreGeom<D, B>;
  __host__ __device__ static constexpr size_t table() { return size_t(Gm::TABLE_WORDS) * 4; }
  __host__ __device__ static size_t q(int hq) { return size_t(hq) * D * 2; }
  __host__ __device__ static size_t inv(int hq) { return (size_t(hq) * 4 + 15) / 16 * 16; }
  __host__ __device__ static size_t tile(int hq) { return size_t(hq) * kScoreTile * 4; }
  __host__ __device__ static constexpr size_t ring() { return size_t(kScoreWarps) * kScoreStages * Gm::RING_STAGE; }
  __host__ __device__ static size_t qf(int hq) { return size_t(hq) * D * 4; }  // fp32 q' (prologue; aliases tile+ring)
  __host__ __device__ static size_t total(int hq) {
    const size_t main = tile(hq) + ring();
    return table() + q(hq) + inv(hq) + (qf(hq) > main ? qf(hq) : main);
  }
};

template <int D, int B, int GQ>
__global__ void __launch_bounds__(kScoreThreads, 1) qk_scores_kernel(const ScoreArgs a) {
  using Gm = ScoreGeom<D, B>;
  using Sm = ScoreSmem<D, B>;
  constexpr int LPK = Gm::LPK, KPW = Gm::KPW, CB = Gm::CB;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* ptab = reinterpret_cast<uint32_t*>(smem);
  uint32_t* qh = reinterpret_cast<uint32_t*>(smem + Sm::table());  // [hq][D/2] half2
  float* inv_s = reinterpret_cast<float*>(smem + Sm::table() + Sm::q(a.hq));
  uint8_t* work = smem + Sm::table() + Sm::q(a.hq) + Sm::inv(a.hq);
  float* qf = reinterpret_cast<float*>(work);      // prologue only
  float* tile = reinterpret_cast<float*>(work);    // [hq][kScoreTile]
  uint8_t* rings = work + Sm::tile(a.hq);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const QuantParams& p = a.p;

  // ---- pair table: entry e = lo | hi << B  ->  half2(c_lo, c_hi), per lane
  for (int i = tid; i < Gm::TABLE_WORDS; i += kScoreThreads) {
    const int e = i >> 5;
    const __half2 v = __floats2half2_rn(p.levels[e & ((1 << B) - 1)], p.levels[e >> B]);
    ptab[i] = *reinterpret_cast<const uint32_t*>(&v);
  }

  // ---- rotate the queries: q' = H·D·q (fp32), one warp per head
  {
    constexpr int QC = D / 32;  // values per lane
    for (int h = warp; h < a.hq; h += kScoreWarps) {
      float v[QC];
#pragma unroll
      for (int j = 0; j < QC; ++j) {
        const int i = lane * QC + j;
        const float x = __half2float(a.q[int64_t(h) * D + i]);
        v[j] = sign_bit(p.seed, i) ? -x : x;
      }
#pragma unroll
      for (int m = 1; m < QC; m <<= 1)
#pragma unroll
        for (int j = 0; j < QC; ++j)
          if ((j & m) == 0) {
            const float x0 = v[j], x1 = v[j | m];
            v[j] = x0 + x1;
            v[j | m] = x0 - x1;
          }
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        const float sg = (lane & m) ? -1.f : 1.f;
#pragma unroll
        for (int j = 0; j < QC; ++j) v[j] = fmaf(v[j], sg, __shfl_xor_sync(kFull, v[j], m));
      }
      float mx = 0.f;
#pragma unroll
      for (int j = 0; j < QC; ++j) mx = fmaxf(mx, fabsf(v[j]));
#pragma unroll
      for (int m = 16; m > 0; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
      // power-of-two scale with max·s ≤ 1 (s = 1 for an all-zero head)
      int ex = 0;
      frexpf(mx, &ex);  // mx = f·2^ex, 0.5 ≤ f < 1
      const float s = mx > 0.f ? ldexpf(1.f, -ex) : 1.f;
#pragma unroll
      for (int j = 0; j < QC; ++j) qf[h * D + lane * QC + j] = v[j] * s;
      if (lane == 0) inv_s[h] = 1.f / s;
    }
  }
  __syncthreads();
  for (int i = tid; i < a.hq * D / 2; i += kScoreThreads) {
    const __half2 v = __floats2half2_rn(qf[2 * i], qf[2 * i + 1]);
    qh[i] = *reinterpret_cast<const uint32_t*>(&v);
  }
  __syncthreads();  // qf is dead from here on (its space becomes tile + rings)

  // ---- warp work assignment
  // slot = lane / LPK (key-head within the iteration), part = lane % LPK
  const int slot = lane / LPK, part = lane % LPK;
  const int HB = a.hkv > KPW ? a.hkv / KPW : 1;   // head blocks
  const int TPI = a.hkv > KPW ? 1 : KPW / a.hkv;  // tokens per iteration
  const int hb = warp % HB;                        // this warp's head block
  const int wgroup = warp / HB, nwg = kScoreWarps / HB;
  const int g = a.hkv > KPW ? hb * KPW + slot : slot % a.hkv;  // lane's kv head
  const int tok_in_it = a.hkv > KPW ? 0 : slot / a.hkv;         // token offset within iteration

  // lane's query slices: heads g·group + j0 + j, coordinates [32·part, 32·part + 32)
  uint32_t qr[GQ][16];
  float qscale[GQ];

  uint8_t* ring = rings + warp * kScoreStages * Gm::RING_STAGE;
  const uint32_t* lane_tab = ptab + lane;
  const int its_per_tile = kScoreTile / TPI;
  const int64_t ntiles = (a.T + kScoreTile - 1) / kScoreTile;

  // iteration k of this warp within a tile covers tokens t0 + (wgroup + k·nwg)·TPI ...
  auto iter_row0 = [&](int64_t t0, int it) -> int64_t {
    const int64_t t = t0 + int64_t(it) * TPI;
    return t * a.hkv + (a.hkv > KPW ? hb * KPW : 0);
  };
  const int64_t nrows = a.T * a.hkv;
  auto issue = [&](int stage, int64_t row0, bool ok_it) {
    uint8_t* st = ring + stage * Gm::RING_STAGE;
    // codes: IT_BYTES contiguous bytes from row0·CB (zero-filled past the end)
#pragma unroll
    for (int c = 0; c < (Gm::IT_BYTES + 511) / 512; ++c) {
      const int off = c * 512 + lane * 16;
      if (off < Gm::IT_BYTES) {
        const int64_t left = ok_it ? nrows * CB - (row0 * CB + off) : 0;
        const int nb = left <= 0 ? 0 : (left >= 16 ? 16 : int(left));
        cp_async16(smem_addr(st + off), a.codes + (nb ? row0 * CB + off : 0), nb);
      }
    }
    // norms: KPW floats from row0
    if (lane < KPW) {
      const bool ok = ok_it && row0 + lane < nrows;
      cp_async4(smem_addr(st + Gm::IT_BYTES + lane * 4), a.norms + (ok ? row0 + lane : 0), ok ? 4 : 0);
    }
  };

  for (int pass = 0; pass < (a.group + GQ - 1) / GQ; ++pass) {
    const int j0 = pass * GQ;
#pragma unroll
    for (int j = 0; j < GQ; ++j) {
      const int h = g * a.group + j0 + j;
      const bool hv = j0 + j < a.group;
#pragma unroll
      for (int k = 0; k < 16; ++k) qr[j][k] = hv ? qh[h * (D / 2) + part * 16 + k] : 0u;
      qscale[j] = hv ? inv_s[h] * a.scale * p.inv_d : 0.f;
    }
    for (int64_t tile_i = blockIdx.x; tile_i < ntiles; tile_i += gridDim.x) {
      const int64_t t0 = tile_i * kScoreTile;
      // iterations of this warp: it = wgroup + k·nwg < its_per_tile
      const int nit = (its_per_tile - wgroup + nwg - 1) / nwg;
#pragma unroll 1
      for (int k = 0; k < kScoreStages - 1; ++k) {
        const int it = wgroup + k * nwg;
        issue(k, iter_row0(t0, it < its_per_tile ? it : 0), k < nit);
        cp_async_commit();
      }
      for (int k = 0; k < nit; ++k) {
        const int stage = k % kScoreStages;
        cp_async_wait<kScoreStages - 2>();
        __syncwarp();
        const uint8_t* st = ring + stage * Gm::RING_STAGE;
        uint32_t cw[B];
#pragma unroll
        for (int i = 0; i < B; ++i)
          cw[i] = reinterpret_cast<const uint32_t*>(st + slot * CB + part * Gm::LB)[i];
        const float nu = reinterpret_cast<const float*>(st + Gm::IT_BYTES)[slot];
        __syncwarp();
        {
          const int kn = k + kScoreStages - 1;
          const int itn = wgroup + kn * nwg;
          issue(kn % kScoreStages, iter_row0(t0, itn < its_per_tile ? itn : 0), kn < nit);
          cp_async_commit();
        }
        // dot products with the GQ query slices
        float dot[GQ];
#pragma unroll
        for (int j = 0; j < GQ; ++j) dot[j] = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          __half2 acc[GQ];
#pragma unroll
          for (int j = 0; j < GQ; ++j) acc[j] = __float2half2_rn(0.f);
#pragma unroll
          for (int k2 = 0; k2 < 8; ++k2) {
            const int pr = half * 8 + k2;  // pair index: codes 2pr, 2pr+1
            const uint32_t e = get_bits(cw, pr * 2 * B, 2 * B);
            const uint32_t cv = lane_tab[e << 5];
            const __half2 c = *reinterpret_cast<const __half2*>(&cv);
#pragma unroll
            for (int j = 0; j < GQ; ++j)
              acc[j] = __hfma2(*reinterpret_cast<const __half2*>(&qr[j][pr]), c, acc[j]);
          }
#pragma unroll
          for (int j = 0; j < GQ; ++j) {
            const float2 f = __half22float2(acc[j]);
            dot[j] += f.x + f.y;
          }
        }
#pragma unroll
        for (int m = 1; m < LPK; m <<= 1)
#pragma unroll
          for (int j = 0; j < GQ; ++j) dot[j] += __shfl_xor_sync(kFull, dot[j], m);
        const int it = wgroup + k * nwg;
        const int tt = it * TPI + tok_in_it;  // token within the tile
#pragma unroll
        for (int j = 0; j < GQ; ++j)
          if (part == j % LPK && j0 + j < a.group)
            tile[(g * a.group + j0 + j) * kScoreTile + tt] = dot[j] * nu * qscale[j];
      }
      cp_async_wait<0>();
      __syncthreads();
      // write the tile: hq rows of up to kScoreTile scores, head-major
      const int64_t tvalid = a.T - t0 < kScoreTile ? a.T - t0 : kScoreTile;
      if (tvalid == kScoreTile && (a.T % 4) == 0) {
        for (int i = tid; i < a.hq * kScoreTile / 4; i += kScoreThreads) {
          const int h = i / (kScoreTile / 4), c = i % (kScoreTile / 4);
          const int64_t hbase = int64_t(h) * a.T + t0;
          if (j0 <= h % a.group && h % a.group < j0 + GQ)
            reinterpret_cast<float4*>(a.scores + hbase)[c] =
                reinterpret_cast<const float4*>(tile + h * kScoreTile)[c];
        }
      } else {
        for (int i = tid; i < a.hq * kScoreTile; i += kScoreThreads) {
          const int h = i / kScoreTile, c = i % kScoreTile;
          if (c < tvalid && j0 <= h % a.group && h % a.group < j0 + GQ)
            a.scores[int64_t(h) * a.T + t0 + c] = tile[h * kScoreTile + c];
        }
      }
      __syncthreads();
    }
  }
}

template <int D, int B, int GQ>
cudaError_t launch_scores_dbg(const ScoreArgs& a, cudaStream_t stream) {
  auto k = qk_scores_kernel<D, B, GQ>;
  const size_t smem = ScoreSmem<D, B>::total(a.hq);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int64_t ntiles = (a.T + kScoreTile - 1) / kScoreTile;
  const int grid = grid_for(reinterpret_cast<const void*>(k), kScoreThreads, smem, ntiles);
  k<<<grid, kScoreThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int D, int B>
cudaError_t launch_scores_db(const ScoreArgs& a, cudaStream_t stream) {
  switch (a.group) {
    case 1: return launch_scores_dbg<D, B, 1>(a, stream);
    case 2: return launch_scores_dbg<D, B, 2>(a, stream);
    default: return launch_scores_dbg<D, B, 4>(a, stream);  // 4, and 8 in two passes
  }
}

template <int D>
cudaError_t launch_scores_d(const ScoreArgs& a, cudaStream_t stream) {
  switch (a.p.bits) {
    case 1: return launch_scores_db<D, 1>(a, stream);
    case 2: return launch_scores_db<D, 2>(a, stream);
    case 3: return launch_scores_db<D, 3>(a, stream);
    case 4: return launch_scores_db<D, 4>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool qk_scores_supported(int d, int bits, int hq, int hkv) {
  if (hkv & (hkv - 1)) return false;  // the kv-head count must be a power of two
  const int kpw = 1024 / d;
  const int hb = hkv > kpw ? hkv / kpw : 1;
  if (hb > kScoreWarps) return false;
  size_t smem = 0;
  switch (d * 10 + bits) {
#define RRQ_SM(DD, BB) case DD * 10 + BB: smem = ScoreSmem<DD, BB>::total(hq); break;
    RRQ_SM(64, 1) RRQ_SM(64, 2) RRQ_SM(64, 3) RRQ_SM(64, 4)
    RRQ_SM(128, 1) RRQ_SM(128, 2) RRQ_SM(128, 3) RRQ_SM(128, 4)
    RRQ_SM(256, 1) RRQ_SM(256, 2) RRQ_SM(256, 3) RRQ_SM(256, 4)
    RRQ_SM(512, 1) RRQ_SM(512, 2) RRQ_SM(512, 3) RRQ_SM(512, 4)
#undef RRQ_SM
    default: return false;
  }
  return smem <= 227 * 1024;
}

cudaError_t launch_qk_scores(const void* q, int hq, const uint8_t* codes, const float* norms,
                             int64_t T, int hkv, int d, const QuantParams& p, float scale,
                             float* scores, cudaStream_t stream) {
  ScoreArgs a;
  a.q = static_cast<const __half*>(q);
  a.codes = codes;
  a.norms = norms;
  a.scores = scores;
  a.T = T;
  a.hq = hq;
  a.hkv = hkv;
  a.group = hq / hkv;
  a.scale = scale;
  a.p = p;
  switch (d) {
    case 64: return launch_scores_d<64>(a, stream);
    case 128: return launch_scores_d<128>(a, stream);
    case 256: return launch_scores_d<256>(a, stream);
    case 512: return launch_scores_d<512>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rrq

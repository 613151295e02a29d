// scores.cu — decode-time attention scores straight from packed codes.
//
// "Random-rotation quantization" page, "Three decoders, one rotation",
// inner-product decoder: <q, x> is recovered from <Πq, code(Πx)> and a
// normalising scalar.  With q' = H·D·q = √d·Πq:
//     s[h][t] = scale · (ν_{t,g}/d) · Σ_i q'_{h,i} · c[code_{t,g,i}],  g = ⌊h·hkv/hq⌋,
// which equals scale·<q_h, x̂_{t,g}> without ever forming x̂.
//
// 4-bit codes at d ≤ 128 with a power-of-two group ≤ 8 (the KV-cache case) take
// the tensor-core kernel further down (qk_scores_mma_kernel); the rest of this
// header describes the general kernel, for every other width and d.
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
// Data movement.  A warp owns whole tiles of kScoreTile tokens (for its
// head block when hkv exceeds one iteration's key-heads) and works through a
// tile U iterations per step (one iteration = KPW key-head rows).  Codes and
// norms stream through a per-warp cp.async ring that runs on across tiles, so
// the pipeline never drains; the tile's scores (its heads × kScoreTile) are
// staged in the warp's own shared buffer and leave as 128-byte coalesced rows,
// with no synchronisation beyond the warp.
// For 4-bit codes the table offset of a code byte is built by one byte
// permute (byte·256 + lane·4: one 128-byte row of lane copies per entry,
// padded to 256 bytes); other widths extract the bits and index the table.
#include <type_traits>

#include "rrq_device.cuh"

namespace rrq {
namespace {

constexpr int kScoreTile = 32;   // tokens per warp tile
constexpr int kScoreStages = 3;  // ring depth (steps)
template <int W> constexpr int score_u() { return W >= 16 ? 2 : 4; }  // iterations per step

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

// q' = H·D·q for every query head (fp32, one warp per head), scaled per head
// by a power of two s with max|q'·s| ≤ 1 (s = 1 for an all-zero head);
// qf[h·D + i] = q'_{h,i}·s and inv_s[h] = 1/s.
template <int D>
__device__ void rotate_queries(const ScoreArgs& a, float* qf, float* inv_s, int warp, int lane,
                               int nwarps) {
  constexpr int QC = D / 32;  // values per lane
  const QuantParams& p = a.p;
  for (int h = warp; h < a.hq; h += nwarps) {
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
    int ex = 0;
    frexpf(mx, &ex);  // mx = f·2^ex, 0.5 ≤ f < 1
    const float s = mx > 0.f ? ldexpf(1.f, -ex) : 1.f;
#pragma unroll
    for (int j = 0; j < QC; ++j) qf[h * D + lane * QC + j] = v[j] * s;
    if (lane == 0) inv_s[h] = 1.f / s;
  }
}

template <int D, int B>
struct ScoreGeom {
  static constexpr int LPK = D / 32;               // lanes per key-head
  static constexpr int KPW = 32 / LPK;             // key-heads per warp iteration
  static constexpr int CB = D * B / 8;             // code bytes per key-head
  static constexpr int LB = 4 * B;                 // code bytes per lane (32 codes)
  static constexpr int IT_BYTES = KPW * CB;        // codes per iteration (= 128·B)
  static constexpr int NPAIR = 16;                 // code pairs per lane
  static constexpr bool PRMT = B == 4;             // byte-permute table offsets
  static constexpr int ROW_WORDS = PRMT ? 64 : 32; // table words per entry
  static constexpr int TABLE_WORDS = (1 << (2 * B)) * ROW_WORDS;
  static constexpr int IT_STRIDE = (IT_BYTES + KPW * 4 + 15) / 16 * 16;  // codes | norms
};

// Shared memory: pair table | q'' (fp16 pairs) | inverse head scales | warp tiles | rings
template <int D, int B, int W>
struct ScoreSmem {
  using Gm = ScoreGeom<D, B>;
  static constexpr int RING_STAGE = score_u<W>() * Gm::IT_STRIDE;
  __host__ __device__ static constexpr size_t table() { return size_t(Gm::TABLE_WORDS) * 4; }
  __host__ __device__ static size_t q(int hq) { return size_t(hq) * D * 2; }
  __host__ __device__ static size_t inv(int hq) { return (size_t(hq) * 4 + 15) / 16 * 16; }
  // q heads of one head block: the rows of a warp tile
  __host__ __device__ static int bheads(int hq, int hkv) {
    return (hkv > Gm::KPW ? Gm::KPW : hkv) * (hq / hkv);
  }
  __host__ __device__ static size_t tile(int hq, int hkv) { return size_t(W) * bheads(hq, hkv) * kScoreTile * 4; }
  __host__ __device__ static constexpr size_t ring() { return size_t(W) * kScoreStages * RING_STAGE; }
  __host__ __device__ static size_t qf(int hq) { return size_t(hq) * D * 4; }  // fp32 q' (prologue; aliases tiles+rings)
  __host__ __device__ static size_t total(int hq, int hkv) {
    const size_t main = tile(hq, hkv) + ring();
    return table() + q(hq) + inv(hq) + (qf(hq) > main ? qf(hq) : main);
  }
};

template <int D, int B, int GQ, int W>
__global__ void __launch_bounds__(W * 32, 1) qk_scores_kernel(const ScoreArgs a) {
  pdl_release();
  constexpr int kScoreWarps = W, kScoreThreads = W * 32, kScoreU = score_u<W>();
  using Gm = ScoreGeom<D, B>;
  using Sm = ScoreSmem<D, B, W>;
  constexpr int LPK = Gm::LPK, KPW = Gm::KPW, CB = Gm::CB;
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* ptab = reinterpret_cast<uint32_t*>(smem);
  uint32_t* qh = reinterpret_cast<uint32_t*>(smem + Sm::table());  // [hq][D/2] half2
  float* inv_s = reinterpret_cast<float*>(smem + Sm::table() + Sm::q(a.hq));
  uint8_t* work = smem + Sm::table() + Sm::q(a.hq) + Sm::inv(a.hq);
  float* qf = reinterpret_cast<float*>(work);      // prologue only
  float* tiles = reinterpret_cast<float*>(work);   // per warp: [heads of its block][kScoreTile]
  uint8_t* rings = work + Sm::tile(a.hq, a.hkv);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const QuantParams& p = a.p;

  // ---- pair table: entry e = lo | hi << B  ->  half2(c_lo, c_hi), per lane
  for (int i = tid; i < Gm::TABLE_WORDS; i += kScoreThreads) {
    const int e = i / Gm::ROW_WORDS;
    const __half2 v = __floats2half2_rn(p.levels[e & ((1 << B) - 1)], p.levels[e >> B]);
    ptab[i] = *reinterpret_cast<const uint32_t*>(&v);
  }

  pdl_wait();  // from here on, global memory
  rotate_queries<D>(a, qf, inv_s, warp, lane, kScoreWarps);
  __syncthreads();
  for (int i = tid; i < a.hq * D / 2; i += kScoreThreads) {
    const __half2 v = __floats2half2_rn(qf[2 * i], qf[2 * i + 1]);
    qh[i] = *reinterpret_cast<const uint32_t*>(&v);
  }
  __syncthreads();  // qf is dead from here on (its space becomes tile + rings)

  // ---- warp work assignment
  // slot = lane / LPK (key-head within the iteration), part = lane % LPK
  const int slot = lane / LPK, part = lane % LPK;
  const int HB = a.hkv > KPW ? a.hkv / KPW : 1;   // head blocks (divides kScoreWarps)
  const int TPI = a.hkv > KPW ? 1 : KPW / a.hkv;  // tokens per iteration
  const int hb = warp % HB;                        // this warp's head block (fixed)
  const int g = a.hkv > KPW ? hb * KPW + slot : slot % a.hkv;  // lane's kv head
  const int tok_in_it = a.hkv > KPW ? 0 : slot / a.hkv;         // token offset within iteration
  const int g0 = a.hkv > KPW ? hb * KPW : 0;                   // first kv head of the block
  const int bheads = (a.hkv > KPW ? KPW : a.hkv) * a.group;    // q heads of the block

  // lane's query slices: heads g·group + j0 + j, coordinates [32·part, 32·part + 32)
  uint32_t qr[GQ][16];
  float qscale[GQ];

  uint8_t* ring = rings + warp * kScoreStages * Sm::RING_STAGE;
  float* tile = tiles + warp * Sm::bheads(a.hq, a.hkv) * kScoreTile;
  const uint32_t* lane_tab = ptab + lane;
  const char* tab_bytes = reinterpret_cast<const char*>(ptab);
  const uint32_t lane4 = uint32_t(lane) * 4u;
  // Token range of this warp: the warps of a head block split the tokens
  // evenly, in units of one iteration (TPI tokens); the range is worked in
  // chunks of kScoreTile tokens (icp iterations), one warp tile each.
  const int icp = kScoreTile / TPI;                 // iterations per chunk
  const int64_t units = (a.T + TPI - 1) / TPI;
  const int64_t nwh = int64_t(gridDim.x) * kScoreWarps / HB;  // warps per head block
  const int64_t wi = (int64_t(blockIdx.x) * kScoreWarps + warp) / HB;
  const int64_t it_begin = units * wi / nwh, it_end = units * (wi + 1) / nwh;
  const int64_t n_it = it_end - it_begin;           // iterations of this warp
  const int64_t nsteps = (n_it + kScoreU - 1) / kScoreU;
  const int64_t nrows = a.T * a.hkv;

  // row of the first key-head of this warp's iteration `it`
  auto iter_row0 = [&](int64_t it) -> int64_t { return (it_begin + it) * TPI * a.hkv + g0; };
  // step q (iterations q·U .. q·U + U − 1) into ring stage `stage`
  auto issue = [&](int stage, int64_t q) {
    if (q < nsteps) {
      const int64_t i0 = q * kScoreU;
      // all U iterations present and inside the array: no per-copy bounds
      const bool full = i0 + kScoreU <= n_it && iter_row0(i0 + kScoreU - 1) + KPW <= nrows;
#pragma unroll
      for (int u = 0; u < kScoreU; ++u) {
        uint8_t* st = ring + stage * Sm::RING_STAGE + u * Gm::IT_STRIDE;
        const bool ok_it = i0 + u < n_it;
        const int64_t row0 = ok_it ? iter_row0(i0 + u) : 0;
        if (full) {
#pragma unroll
          for (int c = 0; c < (Gm::IT_BYTES + 511) / 512; ++c) {
            const int off = c * 512 + lane * 16;
            if (off < Gm::IT_BYTES) cp_async16(smem_addr(st + off), a.codes + row0 * CB + off, 16);
          }
          if (lane < KPW) cp_async4(smem_addr(st + Gm::IT_BYTES + lane * 4), a.norms + row0 + lane, 4);
        } else {
#pragma unroll
          for (int c = 0; c < (Gm::IT_BYTES + 511) / 512; ++c) {
            const int off = c * 512 + lane * 16;
            if (off < Gm::IT_BYTES) {
              const int64_t left = ok_it ? nrows * CB - (row0 * CB + off) : 0;
              const int nb = left <= 0 ? 0 : (left >= 16 ? 16 : int(left));
              cp_async16(smem_addr(st + off), a.codes + (nb ? row0 * CB + off : 0), nb);
            }
          }
          if (lane < KPW) {
            const bool ok = ok_it && row0 + lane < nrows;
            cp_async4(smem_addr(st + Gm::IT_BYTES + lane * 4), a.norms + (ok ? row0 + lane : 0), ok ? 4 : 0);
          }
        }
      }
    }
    cp_async_commit();
  };

  for (int pass = 0; pass < (a.group + GQ - 1) / GQ; ++pass) {
    const int j0 = pass * GQ;
    // tile row of (kv head g, query head j0 + j) is (g − g0)·group + j0 + j
    float* tile_lane = tile + ((g - g0) * a.group + j0) * kScoreTile;
#pragma unroll
    for (int j = 0; j < GQ; ++j) {
      const int h = g * a.group + j0 + j;
      const bool hv = j0 + j < a.group;
#pragma unroll
      for (int k = 0; k < 16; ++k) qr[j][k] = hv ? qh[h * (D / 2) + part * 16 + k] : 0u;
      qscale[j] = hv ? inv_s[h] * a.scale * p.inv_d : 0.f;
    }
    float qscale_own = 0.f;  // the scale of head j0 + part (reduce-scatter layout)
#pragma unroll
    for (int j = 0; j < GQ; ++j)
      if (j == part) qscale_own = qscale[j];

#pragma unroll 1
    for (int k = 0; k < kScoreStages - 1; ++k) issue(k, k);
    int stage = 0;
    int ic = 0;  // iteration within the current chunk
    for (int64_t q = 0; q < nsteps; ++q) {
      const int64_t i0 = q * kScoreU;
      cp_async_wait<kScoreStages - 2>();
      __syncwarp();
      const uint8_t* stb = ring + stage * Sm::RING_STAGE;
      uint32_t cw[kScoreU][B];
      float nu[kScoreU];
#pragma unroll
      for (int u = 0; u < kScoreU; ++u) {
        const uint8_t* st = stb + u * Gm::IT_STRIDE;
        if constexpr (B == 4) {
          const uint4 v = *reinterpret_cast<const uint4*>(st + slot * CB + part * Gm::LB);
          cw[u][0] = v.x; cw[u][1] = v.y; cw[u][2] = v.z; cw[u][3] = v.w;
        } else {
#pragma unroll
          for (int i = 0; i < B; ++i)
            cw[u][i] = reinterpret_cast<const uint32_t*>(st + slot * CB + part * Gm::LB)[i];
        }
        nu[u] = reinterpret_cast<const float*>(st + Gm::IT_BYTES)[slot];
      }
      __syncwarp();  // every lane has read this stage before it is refilled
      issue(stage == 0 ? kScoreStages - 1 : stage - 1, q + kScoreStages - 1);
      stage = (stage + 1 == kScoreStages) ? 0 : stage + 1;

#pragma unroll
      for (int u = 0; u < kScoreU; ++u) {
        // dot products of this key-head slice with the GQ query slices: 16
        // code pairs accumulated in fp16 (|q''| ≤ 1), then one fold to fp32
        __half2 acc[GQ];
#pragma unroll
        for (int j = 0; j < GQ; ++j) acc[j] = __float2half2_rn(0.f);
#pragma unroll
        for (int pr = 0; pr < 16; ++pr) {  // pair index: codes 2pr, 2pr+1
          uint32_t cv;
          if constexpr (Gm::PRMT) {
            const uint32_t off = __byte_perm(cw[u][pr >> 2], lane4, 0x5504u | ((pr & 3) << 4));
            cv = *reinterpret_cast<const uint32_t*>(tab_bytes + off);
          } else {
            cv = lane_tab[get_bits(cw[u], pr * 2 * B, 2 * B) << 5];
          }
          const __half2 c = *reinterpret_cast<const __half2*>(&cv);
#pragma unroll
          for (int j = 0; j < GQ; ++j)
            acc[j] = __hfma2(*reinterpret_cast<const __half2*>(&qr[j][pr]), c, acc[j]);
        }
        float dot[GQ];
#pragma unroll
        for (int j = 0; j < GQ; ++j) {
          const float2 f = __half22float2(acc[j]);
          dot[j] = f.x + f.y;
        }
        const int tt = (ic + u) * TPI + tok_in_it;  // token within the chunk
        if constexpr (GQ == LPK) {
          // reduce-scatter over the LPK lanes of a key-head: at lane bit m each
          // lane keeps the heads whose bit m equals its own and sends the rest,
          // so lane `part` ends with the full dot product of head `part`
          float r[GQ];
#pragma unroll
          for (int j = 0; j < GQ; ++j) r[j] = dot[j];
#pragma unroll
          for (int m = 1, n = GQ; m < LPK; m <<= 1, n >>= 1) {
            const bool up = (part & m) != 0;
#pragma unroll
            for (int i = 0; i < n / 2; ++i) {
              // pair (r[2i], r[2i+1]) holds heads differing in bit m
              const float keep = up ? r[2 * i + 1] : r[2 * i];
              const float send = up ? r[2 * i] : r[2 * i + 1];
              r[i] = keep + __shfl_xor_sync(kFull, send, m);
            }
          }
          if (i0 + u < n_it && j0 + part < a.group)
            tile_lane[part * kScoreTile + tt] = r[0] * nu[u] * qscale_own;
        } else {
#pragma unroll
          for (int m = 1; m < LPK; m <<= 1)
#pragma unroll
            for (int j = 0; j < GQ; ++j) dot[j] += __shfl_xor_sync(kFull, dot[j], m);
          if (i0 + u < n_it) {
#pragma unroll
            for (int j = 0; j < GQ; ++j)
              if (part == j % LPK && j0 + j < a.group) tile_lane[j * kScoreTile + tt] = dot[j] * nu[u] * qscale[j];
          }
        }
      }

      ic += kScoreU;
      if (ic == icp || i0 + kScoreU >= n_it) {  // chunk complete: write its rows out
        __syncwarp();
        const int64_t ct0 = (it_begin + i0 + kScoreU - ic) * TPI;  // first token of the chunk
        const int64_t tt = ct0 + lane;                             // kScoreTile == 32
        const int ctok = int(min(int64_t(ic) * TPI, (it_begin + n_it) * TPI - ct0));
        const int nrow = min(GQ, a.group - j0);
        if (lane < ctok && tt < a.T) {
          for (int gr = 0; gr < bheads / a.group; ++gr)
            for (int j = j0; j < j0 + nrow; ++j) {
              const int r = gr * a.group + j;
              a.scores[int64_t(g0 * a.group + r) * a.T + tt] = tile[r * kScoreTile + lane];
            }
        }
        __syncwarp();
        ic = 0;
      }
    }
    cp_async_wait<0>();
  }
}

template <int D, int B, int GQ, int W>
cudaError_t launch_scores_dbgw(const ScoreArgs& a, cudaStream_t stream) {
  auto k = qk_scores_kernel<D, B, GQ, W>;
  const size_t smem = ScoreSmem<D, B, W>::total(a.hq, a.hkv);
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int64_t ntiles = (a.T + kScoreTile - 1) / kScoreTile;
  const int hb = a.hkv > ScoreGeom<D, B>::KPW ? a.hkv / ScoreGeom<D, B>::KPW : 1;
  const int grid = grid_for(reinterpret_cast<const void*>(k), W * 32, smem, (ntiles * hb + W - 1) / W);
  return launch_pdl(k, grid, W * 32, smem, stream, a);
}

// The largest warp count whose tiles and rings fit in one CTA's shared memory.
template <int D, int B>
int score_warps(int hq, int hkv) {
  constexpr size_t kMax = 227 * 1024;
  constexpr int KPW = ScoreGeom<D, B>::KPW;
  const int hb = hkv > KPW ? hkv / KPW : 1;
  const int icp = kScoreTile / (hkv > KPW ? 1 : KPW / hkv);  // iterations per chunk
  // a step (score_u iterations) must not straddle chunks
  auto ok = [&](int w) { return icp % (w >= 16 ? 2 : 4) == 0 && w % hb == 0; };
  if (ok(12) && ScoreSmem<D, B, 12>::total(hq, hkv) <= kMax) return 12;
  if (ok(16) && ScoreSmem<D, B, 16>::total(hq, hkv) <= kMax) return 16;
  if (ok(8) && ScoreSmem<D, B, 8>::total(hq, hkv) <= kMax) return 8;
  if (ok(4) && ScoreSmem<D, B, 4>::total(hq, hkv) <= kMax) return 4;
  return 0;
}

template <int D, int B, int GQ>
cudaError_t launch_scores_dbg(const ScoreArgs& a, cudaStream_t stream) {
  switch (score_warps<D, B>(a.hq, a.hkv)) {
    case 16: return launch_scores_dbgw<D, B, GQ, 16>(a, stream);
    case 12: return launch_scores_dbgw<D, B, GQ, 12>(a, stream);
    case 8: return launch_scores_dbgw<D, B, GQ, 8>(a, stream);
    case 4: return launch_scores_dbgw<D, B, GQ, 4>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace
}  // namespace rrq

#include "scores_mma.cuh"

namespace rrq {
namespace {

template <int D, int B>
cudaError_t launch_scores_db(const ScoreArgs& a, cudaStream_t stream) {
  if (mma_score_warps<D, B>(a.hq, a.hkv) > 0) return launch_scores_mma<D, B>(a, stream);
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
  int w = 0;
  switch (d * 10 + bits) {
#define RRQ_SM(DD, BB) case DD * 10 + BB: w = score_warps<DD, BB>(hq, hkv); break;
    RRQ_SM(64, 1) RRQ_SM(64, 2) RRQ_SM(64, 3) RRQ_SM(64, 4)
    RRQ_SM(128, 1) RRQ_SM(128, 2) RRQ_SM(128, 3) RRQ_SM(128, 4)
    RRQ_SM(256, 1) RRQ_SM(256, 2) RRQ_SM(256, 3) RRQ_SM(256, 4)
    RRQ_SM(512, 1) RRQ_SM(512, 2) RRQ_SM(512, 3) RRQ_SM(512, 4)
#undef RRQ_SM
    default: return false;
  }
  (void)hb;
  if (w > 0) return true;  // a warp's head block is fixed: head blocks divide the warps
  switch (d * 10 + bits) {
#define RRQ_MW(DD, BB) case DD * 10 + BB: return mma_score_warps<DD, BB>(hq, hkv) > 0;
    RRQ_MW(64, 1) RRQ_MW(64, 2) RRQ_MW(64, 3) RRQ_MW(64, 4)
    RRQ_MW(128, 1) RRQ_MW(128, 2) RRQ_MW(128, 3) RRQ_MW(128, 4)
    RRQ_MW(256, 1) RRQ_MW(256, 2) RRQ_MW(256, 3) RRQ_MW(256, 4)
    RRQ_MW(512, 1) RRQ_MW(512, 2) RRQ_MW(512, 3) RRQ_MW(512, 4)
#undef RRQ_MW
  }
  return false;
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

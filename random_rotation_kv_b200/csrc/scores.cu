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

constexpr int kScoreWarpsMax = 16;  // warps per CTA: 16, or 8 / 4 when the tiles do not fit
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

// ------------------------------------------------ tensor-core tiles, 4-bit codes
// 4-bit codes, d = 64 or 128, GQA group G ∈ {1, 2, 4, 8}.  For one kv head g
// the scores of a 32-token unit are a [32 × d]·[d × G] product of the code
// levels and the group's rotated queries, run as mma.sync m16n8k16 tiles
// (fp16 operands, fp32 accumulation): tokens are M (two 16-row tiles), the
// group's query heads are N (zero columns pad G to 8), d is K.
//  * Because the dot product sums over coordinates, any assignment of code
//    pairs to K positions serves, as long as the query operand uses the same
//    one.  Thread quad position c owns code bytes [c·d/8, (c+1)·d/8) of a row
//    (one 16- or 8-byte load per row), and in k-step kk its A-fragment columns
//    2c, 2c+1 hold code byte 2kk of that slice and columns 2c+8, 2c+9 byte
//    2kk+1.  Each byte becomes its fp16 level pair with one byte permute and
//    one load from a lane-replicated table, which is the A register itself.
//  * The B fragments (query pairs in the same order) are built once per CTA in
//    shared memory, [g][j][lane] 16-byte words, so a unit loads them with
//    d/32 conflict-free 16-byte loads.
//  * A unit's codes (32 rows of d/2 bytes, hkv rows apart) and norms stream
//    through a per-warp cp.async ring of unpadded rows; each 16-byte
//    (8-byte) fragment load of a quarter (half) warp covers 128 contiguous
//    bytes, so it is conflict-free.  The warps split the units evenly.
//  * Epilogue: each accumulator is scaled by ν_t·scale/d and the head's
//    power-of-two factor and stored; for a head, eight lanes write 32
//    consecutive bytes.
template <int D, int W>
struct MmaScoreSmem {
  static constexpr int CB = D / 2;          // code bytes per key-head
  static constexpr int KK = CB / 8;         // k-steps of 16 coordinates
  static constexpr int CW = CB / 16;        // words of a thread's row slice
  static constexpr int NS = 3;              // ring stages
  // ring rows padded so the quads' slice loads (tokens 4r + j, r = 0..7) are
  // conflict-free: 80 bytes at d = 128 (16-byte copies), 40 at d = 64 (8-byte)
  // ring rows padded so the quads' slice loads (tokens 4r + j, r = 0..7) are
  // conflict-free: 80 bytes at d = 128 (16-byte copies), 40 at d = 64 (8-byte)
  static constexpr int RS = D == 128 ? CB + 16 : CB + 8;
  static constexpr int CP = D == 128 ? 16 : 8;  // cp.async chunk bytes
  static constexpr int STAGE = 32 * RS + 32 * 4;
  static constexpr int RING = NS * STAGE;   // per warp
  __host__ __device__ static constexpr size_t table() { return 256 * 64 * 4; }  // entry e at byte e·256 + lane·4
  __host__ __device__ static size_t bq(int hkv) { return size_t(hkv) * 32 * CB; }  // B fragments
  __host__ __device__ static size_t inv(int hq) { return (size_t(hq) * 4 + 15) / 16 * 16; }
  __host__ __device__ static size_t qf(int hq) { return size_t(hq) * D * 4; }  // prologue only (aliases rings)
  __host__ __device__ static constexpr size_t rings() { return size_t(W) * RING; }
  __host__ __device__ static size_t head(int hq, int hkv) { return bq(hkv) + inv(hq); }
  // Plain layout: [table | B fragments | inv | rings (qf aliased)].
  __host__ __device__ static size_t total(int hq, int hkv) {
    return table() + head(hq, hkv) + (qf(hq) > rings() ? qf(hq) : rings());
  }
  // Folded layout, for a dynamic base at shared address kFoldBase: the table
  // sits at shared address 0x10000 so that the byte-permuted offset
  // 0x10000 | byte·256 | lane·4 is the load address itself.  Below it: the B
  // fragments, inv and the first `front` rings; above it: the other rings
  // (qf aliased).
  static constexpr uint32_t kFoldBase = 0x400, kFoldTable = 0x10000;
  __host__ __device__ static size_t fold_front_rings(int hq, int hkv) {
    const size_t start = head(hq, hkv);
    const size_t room = kFoldTable - kFoldBase;
    const size_t n = start < room ? (room - start) / RING : 0;
    return n < size_t(W) ? n : size_t(W);
  }
  __host__ __device__ static size_t fold_back() { return kFoldTable - kFoldBase + table(); }
  __host__ __device__ static size_t fold_ring(int hq, int hkv, int w) {
    const size_t nf = fold_front_rings(hq, hkv);
    return size_t(w) < nf ? head(hq, hkv) + size_t(w) * RING : fold_back() + (size_t(w) - nf) * RING;
  }
  __host__ __device__ static size_t fold_total(int hq, int hkv) {
    const size_t back = (size_t(W) - fold_front_rings(hq, hkv)) * RING;
    return head(hq, hkv) <= kFoldTable - kFoldBase ? fold_back() + (qf(hq) > back ? qf(hq) : back)
                                                   : ~size_t(0);
  }
};

// d += A·B for one m16n8k16 tile: fp16 A (row-major) and B (column-major)
// fragments, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}
__device__ __forceinline__ uint32_t word_of(const uint2& v, int i) { return i == 0 ? v.x : v.y; }

template <int D, int G, int W, bool FOLD>
__global__ void __launch_bounds__(W * 32, 1) qk_scores_mma_kernel(const ScoreArgs a) {
  pdl_release();
  using Sm = MmaScoreSmem<D, W>;
  constexpr int CB = Sm::CB, KK = Sm::KK, NS = Sm::NS;
  using Chunk = std::conditional_t<D == 128, uint4, uint2>;  // a thread's slice of a row
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const QuantParams& p = a.p;
  uint32_t* ptab;
  uint4* bq;
  float* inv_s;
  float* qf;
  uint8_t* ring;
  if constexpr (FOLD) {
    if (smem_addr(smem) != Sm::kFoldBase) {
      // not the layout the launch assumed: mark every score as invalid
      pdl_wait();
      for (int64_t i = int64_t(blockIdx.x) * W * 32 + tid; i < int64_t(a.hq) * a.T; i += int64_t(gridDim.x) * W * 32)
        a.scores[i] = __int_as_float(0x7fc00000);
      return;
    }
    bq = reinterpret_cast<uint4*>(smem);
    inv_s = reinterpret_cast<float*>(smem + Sm::bq(a.hkv));
    ptab = reinterpret_cast<uint32_t*>(smem + (Sm::kFoldTable - Sm::kFoldBase));
    qf = reinterpret_cast<float*>(smem + Sm::fold_back());
    ring = smem + Sm::fold_ring(a.hq, a.hkv, warp);
  } else {
    ptab = reinterpret_cast<uint32_t*>(smem);
    bq = reinterpret_cast<uint4*>(smem + Sm::table());
    inv_s = reinterpret_cast<float*>(smem + Sm::table() + Sm::bq(a.hkv));
    uint8_t* work = smem + Sm::table() + Sm::head(a.hq, a.hkv);
    qf = reinterpret_cast<float*>(work);  // prologue only
    ring = work + warp * Sm::RING;
  }

  for (int i = tid; i < 256 * 64; i += W * 32) {
    const int e = i >> 6;
    const __half2 v = __floats2half2_rn(p.levels[e & 15], p.levels[e >> 4]);
    ptab[i] = *reinterpret_cast<const uint32_t*>(&v);
  }
  pdl_wait();  // from here on, global memory
  rotate_queries<D>(a, qf, inv_s, warp, lane, W);
  __syncthreads();
  // B fragment word w = 2kk + hh of lane l (quad position c, column n): the
  // rotated pair β = c·d/8 + 2kk + hh of head g·G + n, zero for n ≥ G.
  {
    uint32_t* bw = reinterpret_cast<uint32_t*>(bq);
    for (int i = tid; i < a.hkv * 32 * 2 * KK; i += W * 32) {
      const int comp = i & 3, l = (i >> 2) & 31, j = (i >> 7) % (KK / 2), g = (i >> 7) / (KK / 2);
      const int w = 4 * j + comp, kk = w >> 1, hh = w & 1, c = l & 3, n = l >> 2;
      const int beta = c * (CB / 4) + 2 * kk + hh;
      __half2 v = __floats2half2_rn(0.f, 0.f);
      if (n < G) {
        const float* qh = qf + (g * G + n) * D;
        v = __floats2half2_rn(qh[2 * beta], qh[2 * beta + 1]);
      }
      bw[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
  }
  __syncthreads();  // qf is dead: its space becomes the rings

  // units u = tile·hkv + g (token-major); warp w takes u = w, w + nw, w + 2nw, …
  // so the warps working at one moment read whole token rows of the cache
  // together.  The launch makes nw a multiple of hkv, so all units of a warp
  // have the same kv head g (its B fragments stay in registers) and consecutive
  // units are TS = nw/hkv tiles apart: every address advances by a constant.
  const int lg_hkv = __ffs(a.hkv) - 1;  // hkv is a power of two
  const int64_t nbt = (a.T + 31) >> 5;
  const int64_t nw = int64_t(gridDim.x) * W, gw = int64_t(blockIdx.x) * W + warp;
  const int g = int(gw & (a.hkv - 1));
  const int64_t tile0 = gw >> lg_hkv, TS = nw >> lg_hkv;
  const int64_t my_units = tile0 < nbt ? (nbt - tile0 + TS - 1) / TS : 0;
  // FOLD: byte 2 of the permute's second operand is the table's address bit 16
  const char* tab_bytes = reinterpret_cast<const char*>(ptab);
  const uint32_t lane4 = uint32_t(lane) * 4u | (FOLD ? Sm::kFoldTable : 0u);
  const int qc = lane & 3, qr = lane >> 2;  // quad position, token group 4qr .. 4qr + 3

  // Copy k of a unit moves chunk c = lane % CPR of row t = lane / CPR + k·(32 / CPR)
  constexpr int CPR = CB / Sm::CP;  // copies per row
  const int lt = lane / CPR, lc = lane % CPR;
  const int64_t row_bytes = int64_t(a.hkv) * CB;  // global stride between tokens
  const int64_t unit_step = TS * 32;              // tokens between consecutive units
  const int64_t src_step = unit_step * row_bytes;
  const uint8_t* src_next = a.codes + (tile0 * 32 * a.hkv + g) * CB + lt * row_bytes + lc * Sm::CP;
  const float* nrm_next = a.norms + (tile0 * 32 + lane) * a.hkv + g;
  int64_t t_next = tile0 * 32;  // first token of the next unit to load
  const uint32_t ring0 = smem_addr(ring);
  const uint32_t lane_dst = uint32_t(lt * Sm::RS + lc * Sm::CP);
  auto copy = [&](uint32_t dst, const uint8_t* src, bool ok) {
    if constexpr (Sm::CP == 16) cp_async16(dst, ok ? src : a.codes, ok ? 16 : 0);
    else cp_async8(dst, ok ? src : a.codes, ok ? 8 : 0);
  };
  int64_t issued = 0;
  auto issue = [&](int stage) {
    if (issued < my_units) {
      const uint32_t sbase = ring0 + uint32_t(stage * Sm::STAGE);
      if (t_next + 32 <= a.T) {
#pragma unroll
        for (int k = 0; k < CPR; ++k)
          copy(sbase + lane_dst + k * (32 / CPR) * Sm::RS, src_next + k * (32 / CPR) * row_bytes, true);
        cp_async4(sbase + 32 * Sm::RS + lane * 4, nrm_next, 4);
      } else {
#pragma unroll
        for (int k = 0; k < CPR; ++k)
          copy(sbase + lane_dst + k * (32 / CPR) * Sm::RS, src_next + k * (32 / CPR) * row_bytes,
               t_next + lt + k * (32 / CPR) < a.T);
        const bool ok = t_next + lane < a.T;
        cp_async4(sbase + 32 * Sm::RS + lane * 4, ok ? nrm_next : a.norms, ok ? 4 : 0);
      }
      ++issued;
      src_next += src_step;
      nrm_next += unit_step * a.hkv;
      t_next += unit_step;
    }
    cp_async_commit();
  };
#pragma unroll
  for (int k = 0; k < NS - 1; ++k) issue(k);

  auto level_pair = [&](uint32_t word, int pos) -> uint32_t {
    uint32_t cv;
    if constexpr (FOLD) {  // address 0x10000 | byte·256 | lane·4
      const uint32_t addr = __byte_perm(word, lane4, 0x7604u | (pos << 4));
      asm("ld.shared.b32 %0, [%1];" : "=r"(cv) : "r"(addr));
    } else {
      const uint32_t off = __byte_perm(word, lane4, 0x5504u | (pos << 4));
      cv = *reinterpret_cast<const uint32_t*>(tab_bytes + off);
    }
    return cv;
  };

  // the lane's B fragments (k-step kk: words 2kk, 2kk + 1) and head scales
  uint32_t bfr[KK][2];
#pragma unroll
  for (int j = 0; j < KK / 2; ++j) {
    const uint4 v = bq[(g * (KK / 2) + j) * 32 + lane];
    bfr[2 * j][0] = v.x;
    bfr[2 * j][1] = v.y;
    bfr[2 * j + 1][0] = v.z;
    bfr[2 * j + 1][1] = v.w;
  }
  float hsc[2];
#pragma unroll
  for (int e = 0; e < 2; ++e)
    hsc[e] = 2 * qc + e < G ? a.scale * p.inv_d * inv_s[g * G + 2 * qc + e] : 0.f;
  const bool vec_out = (a.T & 3) == 0;  // 16-byte score stores stay aligned
  const int h0 = g * G + 2 * qc;        // the lane's first head
  float* out_next = a.scores + int64_t(h0) * a.T + tile0 * 32 + 4 * qr;
  int64_t t0 = tile0 * 32;

  int stage = 0;
  for (int64_t k = 0; k < my_units; ++k) {
    cp_async_wait<NS - 2>();
    __syncwarp();
    const uint8_t* st = ring + stage * Sm::STAGE;
    // token 4qr + j (j = 2mt + h) is row qr + 8h of m-tile mt
    Chunk cw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) cw[j] = *reinterpret_cast<const Chunk*>(st + (4 * qr + j) * Sm::RS + qc * (CB / 4));
    const float4 nu = *reinterpret_cast<const float4*>(st + 32 * Sm::RS + 16 * qr);
    __syncwarp();  // every lane has read this stage before it is refilled
    issue(stage == 0 ? NS - 1 : stage - 1);
    stage = (stage + 1 == NS) ? 0 : stage + 1;

    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < KK; ++kk) {
      const int wi = kk >> 1, pos = 2 * (kk & 1);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint32_t lo = word_of(cw[2 * mt], wi), hi = word_of(cw[2 * mt + 1], wi);
        mma_16816(acc[mt], level_pair(lo, pos), level_pair(hi, pos), level_pair(lo, pos + 1),
                  level_pair(hi, pos + 1), bfr[kk][0], bfr[kk][1]);
      }
    }

    // accumulator i of tile mt: token 4qr + 2mt + (i >> 1), head 2qc + (i & 1)
    const bool full = vec_out && t0 + 32 <= a.T;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (2 * qc + e < G) {
        float* out = out_next + int64_t(e) * a.T;
        const float2 hs2 = make_float2(hsc[e], hsc[e]);
        const float2 s01 = mul2(make_float2(nu.x, nu.y), hs2), s23 = mul2(make_float2(nu.z, nu.w), hs2);
        const float2 v01 = mul2(make_float2(acc[0][e], acc[0][2 + e]), s01);
        const float2 v23 = mul2(make_float2(acc[1][e], acc[1][2 + e]), s23);
        const float4 v = make_float4(v01.x, v01.y, v23.x, v23.y);
        if (full) {
          *reinterpret_cast<float4*>(out) = v;
        } else {
          const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (t0 + 4 * qr + j < a.T) out[j] = vv[j];
        }
      }
    }
    out_next += TS * 32;
    t0 += TS * 32;
  }
  cp_async_wait<0>();
}

template <int D, int G, int W>
cudaError_t launch_scores_mma_w(const ScoreArgs& a, cudaStream_t stream) {
  using Sm = MmaScoreSmem<D, W>;
  int dev = 0, reserved = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  const bool fold = reserved == int(Sm::kFoldBase) && Sm::fold_total(a.hq, a.hkv) <= 227 * 1024;
  auto k = fold ? qk_scores_mma_kernel<D, G, W, true> : qk_scores_mma_kernel<D, G, W, false>;
  const size_t smem = fold ? Sm::fold_total(a.hq, a.hkv) : Sm::total(a.hq, a.hkv);
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int64_t units = ((a.T + 31) / 32) * a.hkv;
  int grid = grid_for(reinterpret_cast<const void*>(k), W * 32, smem, (units + W - 1) / W);
  // the kernel needs the warp count grid·W to be a multiple of hkv (a power of
  // two): round the grid to a multiple of hkv/W when hkv exceeds W
  if (a.hkv > W) {
    const int m = a.hkv / W;
    grid = grid < m ? m : grid / m * m;
  }
  return launch_pdl(k, grid, W * 32, smem, stream, a);
}

// The tensor-core kernel applies (4-bit codes, d ≤ 128, a power-of-two group
// ≤ 8, and its shared memory fits with 16 or 8 warps); returns its warps or 0.
template <int D>
int mma_score_warps(int bits, int hq, int hkv) {
  const int group = hq / hkv;
  if (bits != 4 || (D != 64 && D != 128) || group > 8 || (group & (group - 1))) return 0;
  if (MmaScoreSmem<D, 16>::total(hq, hkv) <= 227 * 1024) return 16;
  if (MmaScoreSmem<D, 8>::total(hq, hkv) <= 227 * 1024) return 8;
  return 0;
}

template <int D, int G>
cudaError_t launch_scores_mma_g(const ScoreArgs& a, cudaStream_t stream) {
  if (mma_score_warps<D>(4, a.hq, a.hkv) == 16) return launch_scores_mma_w<D, G, 16>(a, stream);
  return launch_scores_mma_w<D, G, 8>(a, stream);
}

template <int D>
cudaError_t launch_scores_mma(const ScoreArgs& a, cudaStream_t stream) {
  switch (a.group) {
    case 1: return launch_scores_mma_g<D, 1>(a, stream);
    case 2: return launch_scores_mma_g<D, 2>(a, stream);
    case 4: return launch_scores_mma_g<D, 4>(a, stream);
    case 8: return launch_scores_mma_g<D, 8>(a, stream);
  }
  return cudaErrorInvalidValue;
}

template <int D, int B>
cudaError_t launch_scores_db(const ScoreArgs& a, cudaStream_t stream) {
  if constexpr (B == 4 && D <= 128) {
    if (mma_score_warps<D>(B, a.hq, a.hkv) > 0) return launch_scores_mma<D>(a, stream);
  }
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
  if (d == 64) return mma_score_warps<64>(bits, hq, hkv) > 0;
  if (d == 128) return mma_score_warps<128>(bits, hq, hkv) > 0;
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

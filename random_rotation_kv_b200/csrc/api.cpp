// api.cpp — the C ABI of librrq.so: argument validation, the default codebook,
// per-call parameter blocks, and dispatch to the kernel launchers.
//
// Every entry point validates all arguments before touching the device and
// returns RRQ_ERR_INVALID on the first violation; nothing is launched then.
#include <cmath>
#include <cstdint>
#include <cstring>

#include "rrq.h"
#include "attention.h"
#include "ggml_blocks.h"
#include "scores_qjl.h"
#include "rrq_params.h"

namespace {

constexpr double kInvSqrt2Pi = 0.39894228040143267794;

bool d_ok(int d) { return d == 64 || d == 128 || d == 256 || d == 512; }
bool bits_ok(int b) { return b >= 1 && b <= 4; }
bool dtype_ok(int t) { return t == RRQ_F32 || t == RRQ_F16 || t == RRQ_BF16; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool arr_ok(const void* p, int64_t n, uintptr_t a) { return n == 0 || (p != nullptr && aligned(p, a)); }

int status_of(cudaError_t e) { return e == cudaSuccess ? RRQ_OK : RRQ_ERR_CUDA; }
cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// ---------------------------------------------------------------- codebook
// Lloyd–Max quantiser for N(0,1) ("Random-rotation quantization" page,
// section "History", EDEN bullet).  Lloyd's alternation on the positive half
// of a symmetric codebook: thresholds at midpoints of neighbouring levels
// (0 between the two innermost), levels at the centroid of their cell,
//   c = (φ(a) − φ(b)) / (Q(a) − Q(b)),  Q(x) = P(X > x) = erfc(x/√2)/2,
// iterated until no level moves by more than 1e-15; the negative half is the
// mirror image, so the codebook is exactly symmetric after rounding to float.
double phi(double x) { return std::isinf(x) ? 0.0 : kInvSqrt2Pi * std::exp(-0.5 * x * x); }
double upper_tail(double x) { return std::isinf(x) ? 0.0 : 0.5 * std::erfc(x / std::sqrt(2.0)); }

struct DefaultCodebooks {
  float levels[5][rrq::kMaxLevels];
  DefaultCodebooks() {
    std::memset(levels, 0, sizeof(levels));
    for (int bits = 1; bits <= 4; ++bits) {
      const int half = 1 << (bits - 1);
      double c[8];
      for (int j = 0; j < half; ++j) c[j] = 2.5 * (2 * j + 1) / (2.0 * half);
      for (int it = 0; it < 200000; ++it) {
        double moved = 0.0;
        double nc[8];
        for (int j = 0; j < half; ++j) {
          const double a = j == 0 ? 0.0 : 0.5 * (c[j - 1] + c[j]);
          const double b = j == half - 1 ? INFINITY : 0.5 * (c[j] + c[j + 1]);
          nc[j] = (phi(a) - phi(b)) / (upper_tail(a) - upper_tail(b));
          moved = std::fmax(moved, std::fabs(nc[j] - c[j]));
        }
        std::memcpy(c, nc, sizeof(double) * half);
        if (moved < 1e-15) break;
      }
      const int L = 2 * half;
      for (int j = 0; j < half; ++j) {
        levels[bits][half + j] = static_cast<float>(c[j]);
        levels[bits][half - 1 - j] = -static_cast<float>(c[j]);
      }
      (void)L;
    }
  }
};

const DefaultCodebooks& default_codebooks() {
  static const DefaultCodebooks cb;  // built once, thread-safe initialisation
  return cb;
}

// Fill the per-call parameter block; returns RRQ_ERR_INVALID for a bad codebook.
// Cell table of the batch encoder's code search (see rrq::CellTable): the
// smallest N in {16, 32, 64} whose closed cells [(j − 1/2)/N, (j + 1/2)/N]
// each hold at most one threshold t_k = fp32(τ_k·A + 1/2); cells = 0 if none.
// All quantities are exact binary fractions except t_k, which is rounded
// exactly as stored, so the table decides #{k : s > t_k} with no error.
void make_cell_table(const float* thr, int nthr, rrq::CellTable* ct) {
  float tmax = 0.f;
  for (int k = 0; k < nthr; ++k) tmax = std::fmax(tmax, std::fabs(thr[k]));
  float R = 1.f;
  while (!(R > tmax)) R *= 2.f;
  if (!std::isfinite(R) || R > 1048576.f) {
    ct->cells = 0;
    return;
  }
  const float A = 0.5f / R;  // exact: R is a power of two
  float t[rrq::kMaxLevels];
  for (int k = 0; k < nthr; ++k) t[k] = thr[k] * A + 0.5f;  // τ·A exact; one rounding
  for (int N = 16; N <= rrq::kMaxCells; N *= 2) {
    bool ok = true;
    for (int j = 0; j <= N && ok; ++j) {
      const double lo = (j - 0.5) / N, hi = (j + 0.5) / N;
      int inside = 0, below = 0;
      float tin = 2.f;
      for (int k = 0; k < nthr; ++k) {
        if (t[k] < lo) ++below;
        else if (t[k] <= hi) { ++inside; tin = t[k]; }
      }
      if (inside > 1) ok = false;
      ct->thr[j] = tin;
      ct->lo[j] = static_cast<uint32_t>(below);
    }
    if (ok) {
      ct->cells = N;
      ct->a = A;
      return;
    }
  }
  ct->cells = 0;
}

int make_params(int bits, const float* codebook, uint64_t seed, int d, rrq::QuantParams* p) {
  std::memset(p, 0, sizeof(*p));
  const int L = 1 << bits;
  const float* c = codebook ? codebook : default_codebooks().levels[bits];
  for (int k = 0; k < L; ++k) {
    if (!std::isfinite(c[k])) return RRQ_ERR_INVALID;
    if (k > 0 && !(c[k] > c[k - 1])) return RRQ_ERR_INVALID;
    p->levels[k] = c[k];
  }
  for (int k = 0; k + 1 < L; ++k)
    p->thr[k] = static_cast<float>((static_cast<double>(c[k]) + static_cast<double>(c[k + 1])) * 0.5);
  int sym = 1;
  for (int k = 0; k < L; ++k) sym &= (c[k] == -c[L - 1 - k]) ? 1 : 0;
  p->sym = sym;
  p->bits = bits;
  p->seed = seed;
  p->inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  p->inv_d = 1.0f / static_cast<float>(d);
  make_cell_table(p->thr, L - 1, &p->cell);
  return RRQ_OK;
}

}  // namespace

extern "C" {

int rrq_format_version(void) { return RRQ_FORMAT_VERSION; }

const char* rrq_strerror(int status) {
  switch (status) {
    case RRQ_OK: return "ok";
    case RRQ_ERR_INVALID: return "invalid argument (checked before launch; nothing was run)";
    case RRQ_ERR_CUDA: return "CUDA launch or runtime error";
    case RRQ_ERR_UNSUPPORTED: return "valid request that the library does not implement";
    case RRQ_ERR_SCRATCH:
      return "request needs more scratch than the 4 MiB of rrq_attention_decode_noalloc "
             "(use rrq_attention_decode with a workspace)";
  }
  return "unknown status";
}

int rrq_codebook(int bits, float* levels) {
  if (!bits_ok(bits) || levels == nullptr) return RRQ_ERR_INVALID;
  std::memcpy(levels, default_codebooks().levels[bits], sizeof(float) * (1u << bits));
  return RRQ_OK;
}

int rrq_rotate(const void* x, int x_dtype, int64_t n, int d, uint64_t seed, int inverse, float* y,
               void* stream) {
  if (n < 0 || !d_ok(d) || !dtype_ok(x_dtype) || (inverse != 0 && inverse != 1))
    return RRQ_ERR_INVALID;
  if (!arr_ok(x, n, 32) || !arr_ok(y, n, 32)) return RRQ_ERR_INVALID;
  if (n == 0) return RRQ_OK;
  const float inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  return status_of(rrq::launch_rotate(x, x_dtype, n, d, seed, inverse, inv_sqrt_d, y,
                                      as_stream(stream)));
}

int rrq_encode(const void* x, int x_dtype, int64_t n, int d, int bits, uint64_t seed,
               const float* codebook, uint8_t* codes, float* norms, const uint16_t* qjl_S,
               uint8_t* qjl_bits, float* qjl_rnorm, void* stream) {
  if (n < 0 || !d_ok(d) || !bits_ok(bits) || !dtype_ok(x_dtype)) return RRQ_ERR_INVALID;
  if (!arr_ok(x, n, 32) || !arr_ok(codes, n, 32) || !arr_ok(norms, n, 4)) return RRQ_ERR_INVALID;
  if (qjl_S != nullptr) {
    if (!aligned(qjl_S, 16) || !arr_ok(qjl_bits, n, 16) || !arr_ok(qjl_rnorm, n, 4))
      return RRQ_ERR_INVALID;
  }
  rrq::QuantParams p;
  if (make_params(bits, codebook, seed, d, &p) != RRQ_OK) return RRQ_ERR_INVALID;
  if (n == 0) return RRQ_OK;
  if (qjl_S != nullptr) {
    if (d != 128) return RRQ_ERR_UNSUPPORTED;
    return status_of(rrq::launch_encode_qjl(x, x_dtype, n, d, p, qjl_S, codes, norms, qjl_bits,
                                            qjl_rnorm, as_stream(stream)));
  }
  return status_of(rrq::launch_encode(x, x_dtype, n, d, p, codes, norms, as_stream(stream)));
}

int rrq_decode(const uint8_t* codes, const float* norms, int64_t n, int d, int bits, uint64_t seed,
               const float* codebook, void* out, int out_dtype, void* stream) {
  if (n < 0 || !d_ok(d) || !bits_ok(bits) || !dtype_ok(out_dtype)) return RRQ_ERR_INVALID;
  if (!arr_ok(codes, n, 32) || !arr_ok(norms, n, 4) || !arr_ok(out, n, 32)) return RRQ_ERR_INVALID;
  rrq::QuantParams p;
  if (make_params(bits, codebook, seed, d, &p) != RRQ_OK) return RRQ_ERR_INVALID;
  if (n == 0) return RRQ_OK;
  return status_of(rrq::launch_decode(codes, norms, n, d, p, out, out_dtype, as_stream(stream)));
}

int rrq_drive_encode(const void* x, int x_dtype, int64_t n, int d, uint64_t seed, int unbiased,
                     uint8_t* codes, float* scales, void* stream) {
  if (n < 0 || !d_ok(d) || !dtype_ok(x_dtype) || (unbiased != 0 && unbiased != 1))
    return RRQ_ERR_INVALID;
  if (!arr_ok(x, n, 32) || !arr_ok(codes, n, 32) || !arr_ok(scales, n, 4)) return RRQ_ERR_INVALID;
  static const float kSigns[2] = {-1.0f, 1.0f};
  rrq::QuantParams p;
  if (make_params(1, kSigns, seed, d, &p) != RRQ_OK) return RRQ_ERR_INVALID;
  p.norm_mode = 1 + unbiased;
  if (n == 0) return RRQ_OK;
  return status_of(rrq::launch_encode(x, x_dtype, n, d, p, codes, scales, as_stream(stream)));
}

int rrq_qk_scores(const void* q, int hq, const uint8_t* codes, const float* norms, int64_t T,
                  int hkv, int d, int bits, uint64_t seed, const float* codebook, float scale,
                  float* scores, void* stream) {
  if (T < 0 || !d_ok(d) || !bits_ok(bits) || hq < 1 || hkv < 1 || hq % hkv != 0 ||
      !std::isfinite(scale))
    return RRQ_ERR_INVALID;
  if (q == nullptr || !aligned(q, 16)) return RRQ_ERR_INVALID;
  if (!arr_ok(codes, T, 16) || !arr_ok(norms, T, 4) || !arr_ok(scores, T, 16))
    return RRQ_ERR_INVALID;
  const int group = hq / hkv;
  if (group != 1 && group != 2 && group != 4 && group != 8) return RRQ_ERR_UNSUPPORTED;
  if (!rrq::qk_scores_supported(d, bits, hq, hkv)) return RRQ_ERR_UNSUPPORTED;
  rrq::QuantParams p;
  if (make_params(bits, codebook, seed, d, &p) != RRQ_OK) return RRQ_ERR_INVALID;
  if (T == 0) return RRQ_OK;
  return status_of(rrq::launch_qk_scores(q, hq, codes, norms, T, hkv, d, p, scale, scores,
                                         as_stream(stream)));
}

int rrq_qk_scores_qjl(const void* q, int hq, const uint8_t* codes, const float* norms,
                      const uint8_t* qjl_bits, const float* qjl_rnorm, const uint16_t* qjl_S,
                      int64_t T, int hkv, int d, int bits, uint64_t seed, const float* codebook,
                      float scale, float* scores, void* stream) {
  if (T < 0 || !d_ok(d) || !bits_ok(bits) || hq < 1 || hkv < 1 || hq % hkv != 0 ||
      !std::isfinite(scale))
    return RRQ_ERR_INVALID;
  if (q == nullptr || !aligned(q, 16) || qjl_S == nullptr || !aligned(qjl_S, 16))
    return RRQ_ERR_INVALID;
  if (!arr_ok(codes, T, 16) || !arr_ok(norms, T, 4) || !arr_ok(qjl_bits, T, 16) ||
      !arr_ok(qjl_rnorm, T, 4) || !arr_ok(scores, T, 16))
    return RRQ_ERR_INVALID;
  const int group = hq / hkv;
  if (d != 128 || (group != 1 && group != 2 && group != 4 && group != 8)) return RRQ_ERR_UNSUPPORTED;
  rrq::QjlScoreArgs a;
  if (make_params(bits, codebook, seed, d, &a.p) != RRQ_OK) return RRQ_ERR_INVALID;
  if (T == 0) return RRQ_OK;
  a.q = static_cast<const __half*>(q);
  a.codes = codes;
  a.norms = norms;
  a.bits = qjl_bits;
  a.rnorm = qjl_rnorm;
  a.S = reinterpret_cast<const __nv_bfloat16*>(qjl_S);
  a.scores = scores;
  a.T = T;
  a.hq = hq;
  a.hkv = hkv;
  a.group = group;
  a.scale = scale;
  return status_of(rrq::launch_qk_scores_qjl(a, as_stream(stream)));
}

namespace {
// Whether the fused kernel (d = 128, 4-bit K and V) serves the shape.
bool attention_fused(int d, int k_bits, int v_bits) { return d == 128 && k_bits == 4 && v_bits == 4; }
size_t attention_ws(int hq, int hkv, int d, int k_bits, int v_bits, int64_t T) {
  return attention_fused(d, k_bits, v_bits) ? rrq::attention_workspace_bytes(hq, hkv, T)
                                            : rrq::attention_general_workspace_bytes(hq, hkv, d, v_bits, T);
}
// Validation shared by the two attention entries: RRQ_OK, or the status to return.
int attention_check(const void* q, int hq, const uint8_t* k_codes, const float* k_norms,
                    const uint8_t* v_codes, const float* v_norms, int64_t T, int hkv, int d, int k_bits,
                    int v_bits, float scale, const float* out) {
  if (T < 1 || !d_ok(d) || !bits_ok(k_bits) || !bits_ok(v_bits) || hq < 1 || hkv < 1 ||
      hq % hkv != 0 || !std::isfinite(scale))
    return RRQ_ERR_INVALID;
  if (q == nullptr || !aligned(q, 16) || out == nullptr || !aligned(out, 16)) return RRQ_ERR_INVALID;
  if (!arr_ok(k_codes, T, 16) || !arr_ok(k_norms, T, 4) || !arr_ok(v_codes, T, 16) ||
      !arr_ok(v_norms, T, 4))
    return RRQ_ERR_INVALID;
  const int group = hq / hkv;
  if (group != 1 && group != 2 && group != 4 && group != 8) return RRQ_ERR_UNSUPPORTED;
  if (!attention_fused(d, k_bits, v_bits) && !rrq::attention_general_supported(d, k_bits, hq, hkv))
    return RRQ_ERR_UNSUPPORTED;
  return RRQ_OK;
}
// The general path's launch with its workspace (counters zero on entry).
int attention_general(const void* q, int hq, const uint8_t* k_codes, const float* k_norms,
                      const uint8_t* v_codes, const float* v_norms, int64_t T, int hkv, int d,
                      const rrq::QuantParams& pk, const rrq::QuantParams& pv, float scale, void* workspace,
                      float* out, cudaStream_t stream) {
  rrq::AttnGenArgs g;
  g.q = q;
  g.k_codes = k_codes;
  g.k_norms = k_norms;
  g.v_codes = v_codes;
  g.v_norms = v_norms;
  g.out = out;
  g.T = T;
  g.hq = hq;
  g.hkv = hkv;
  g.group = hq / hkv;
  g.d = d;
  g.scale = scale;
  g.pk = pk;
  g.pv = pv;
  const cudaError_t e = rrq::launch_attention_general(g, workspace, stream);
  return e == cudaErrorNotSupported ? RRQ_ERR_UNSUPPORTED : status_of(e);
}
}  // namespace

size_t rrq_attention_workspace_bytes(int hq, int hkv, int d, int k_bits, int v_bits, int64_t T) {
  if (T < 1 || !d_ok(d) || !bits_ok(k_bits) || !bits_ok(v_bits) || hq < 1 || hkv < 1 || hq % hkv != 0)
    return 0;
  return attention_ws(hq, hkv, d, k_bits, v_bits, T);
}

int rrq_attention_decode_noalloc(const void* q, int hq, const uint8_t* k_codes,
                                 const float* k_norms, const uint8_t* v_codes,
                                 const float* v_norms, int64_t T, int hkv, int d, int k_bits,
                                 uint64_t k_seed, const float* k_codebook, int v_bits,
                                 uint64_t v_seed, const float* v_codebook, float scale,
                                 float* out, void* stream) {
  const int chk = attention_check(q, hq, k_codes, k_norms, v_codes, v_norms, T, hkv, d, k_bits, v_bits,
                                  scale, out);
  if (chk != RRQ_OK) return chk;
  if (attention_ws(hq, hkv, d, k_bits, v_bits, T) > rrq::kAttentionScratchBytes) return RRQ_ERR_SCRATCH;
  rrq::QuantParams pk, pv;
  if (make_params(k_bits, k_codebook, k_seed, d, &pk) != RRQ_OK ||
      make_params(v_bits, v_codebook, v_seed, d, &pv) != RRQ_OK)
    return RRQ_ERR_INVALID;
  if (!attention_fused(d, k_bits, v_bits)) {
    void* base = nullptr;
    cudaError_t e = rrq::attention_scratch(&base);
    if (e != cudaSuccess) return status_of(e);
    // the counters must start at zero; the rest is overwritten before it is read
    e = cudaMemsetAsync(base, 0, (size_t(hkv) * 4 + 255) / 256 * 256, as_stream(stream));
    if (e != cudaSuccess) return status_of(e);
    return attention_general(q, hq, k_codes, k_norms, v_codes, v_norms, T, hkv, d, pk, pv, scale, base, out,
                             as_stream(stream));
  }
  rrq::AttnArgs a;
  a.pk = pk;
  a.pv = pv;
  a.q = static_cast<const __half*>(q);
  a.k_codes = k_codes;
  a.k_norms = k_norms;
  a.v_codes = v_codes;
  a.v_norms = v_norms;
  a.out = out;
  a.T = T;
  a.hq = hq;
  a.hkv = hkv;
  a.group = hq / hkv;
  a.splits = rrq::attention_splits(hkv, a.group, T);
  a.scale = scale;
  const cudaError_t e = rrq::launch_attention_decode_in_scratch(a, as_stream(stream));
  return e == cudaErrorNotSupported ? RRQ_ERR_UNSUPPORTED : status_of(e);
}

int rrq_attention_decode(const void* q, int hq, const uint8_t* k_codes, const float* k_norms,
                         const uint8_t* v_codes, const float* v_norms, int64_t T, int hkv, int d,
                         int k_bits, uint64_t k_seed, const float* k_codebook, int v_bits,
                         uint64_t v_seed, const float* v_codebook, float scale, void* workspace,
                         size_t workspace_bytes, float* out, void* stream) {
  const int chk = attention_check(q, hq, k_codes, k_norms, v_codes, v_norms, T, hkv, d, k_bits, v_bits,
                                  scale, out);
  if (chk != RRQ_OK) return chk;
  if (workspace == nullptr || !aligned(workspace, 256) ||
      workspace_bytes < attention_ws(hq, hkv, d, k_bits, v_bits, T))
    return RRQ_ERR_INVALID;
  rrq::QuantParams pk, pv;
  if (make_params(k_bits, k_codebook, k_seed, d, &pk) != RRQ_OK ||
      make_params(v_bits, v_codebook, v_seed, d, &pv) != RRQ_OK)
    return RRQ_ERR_INVALID;
  if (!attention_fused(d, k_bits, v_bits))
    return attention_general(q, hq, k_codes, k_norms, v_codes, v_norms, T, hkv, d, pk, pv, scale, workspace,
                             out, as_stream(stream));
  rrq::AttnArgs a;
  a.pk = pk;
  a.pv = pv;
  a.q = static_cast<const __half*>(q);
  a.k_codes = k_codes;
  a.k_norms = k_norms;
  a.v_codes = v_codes;
  a.v_norms = v_norms;
  a.out = out;
  a.T = T;
  a.hq = hq;
  a.hkv = hkv;
  a.group = hq / hkv;
  a.splits = rrq::attention_splits(hkv, a.group, T);
  a.scale = scale;
  a.counters = static_cast<unsigned*>(workspace);
  a.states = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                      (size_t(hkv) * 4 + 255) / 256 * 256);
  const cudaError_t e = rrq::launch_attention_decode(a, as_stream(stream));
  return e == cudaErrorNotSupported ? RRQ_ERR_UNSUPPORTED : status_of(e);
}

int rrq_q4_0_rot(const void* x, int x_dtype, int64_t n, int d, uint64_t seed, int rotate,
                 void* blocks, void* stream) {
  if (n < 0 || !d_ok(d) || !dtype_ok(x_dtype) || (rotate != 0 && rotate != 1))
    return RRQ_ERR_INVALID;
  if (!arr_ok(x, n, 32) || !arr_ok(blocks, n, 16)) return RRQ_ERR_INVALID;
  if (n == 0) return RRQ_OK;
  const float inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  return status_of(rrq::launch_q4_0(x, x_dtype, n, d, seed, rotate, inv_sqrt_d, blocks,
                                    as_stream(stream)));
}

int rrq_ggml_block_bytes(int type) {
  switch (type) {
    case RRQ_GGML_Q4_0: return 18;
    case RRQ_GGML_Q4_1: return 20;
    case RRQ_GGML_Q5_0: return 22;
    case RRQ_GGML_Q5_1: return 24;
    case RRQ_GGML_Q8_0: return 34;
  }
  return 0;
}

int rrq_ggml_rot(const void* x, int x_dtype, int64_t n, int d, uint64_t seed, int rotate, int type,
                 void* blocks, void* stream) {
  if (n < 0 || !d_ok(d) || !dtype_ok(x_dtype) || (rotate != 0 && rotate != 1) ||
      rrq_ggml_block_bytes(type) == 0)
    return RRQ_ERR_INVALID;
  if (!arr_ok(x, n, 32) || !arr_ok(blocks, n, 16)) return RRQ_ERR_INVALID;
  if (n == 0) return RRQ_OK;
  const float inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  if (type == RRQ_GGML_Q4_0)
    return status_of(rrq::launch_q4_0(x, x_dtype, n, d, seed, rotate, inv_sqrt_d, blocks,
                                      as_stream(stream)));
  return status_of(rrq::launch_ggml_blocks(x, x_dtype, n, d, seed, rotate, type, inv_sqrt_d, blocks,
                                           as_stream(stream)));
}

int rrq_ggml_rot_decode(const void* blocks, int type, int64_t n, int d, uint64_t seed, int rotate,
                        void* out, int out_dtype, void* stream) {
  if (n < 0 || !d_ok(d) || !dtype_ok(out_dtype) || (rotate != 0 && rotate != 1) ||
      rrq_ggml_block_bytes(type) == 0)
    return RRQ_ERR_INVALID;
  if (!arr_ok(blocks, n, 16) || !arr_ok(out, n, 32)) return RRQ_ERR_INVALID;
  if (n == 0) return RRQ_OK;
  const float inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  if (type == RRQ_GGML_Q4_0)
    return status_of(rrq::launch_q4_0_decode(blocks, n, d, seed, rotate, inv_sqrt_d, out, out_dtype,
                                             as_stream(stream)));
  return status_of(rrq::launch_ggml_blocks_decode(blocks, type, n, d, seed, rotate, inv_sqrt_d, out,
                                                  out_dtype, as_stream(stream)));
}

int rrq_q4_0_rot_decode(const void* blocks, int64_t n, int d, uint64_t seed, int rotate, void* out,
                        int out_dtype, void* stream) {
  if (n < 0 || !d_ok(d) || !dtype_ok(out_dtype) || (rotate != 0 && rotate != 1))
    return RRQ_ERR_INVALID;
  if (!arr_ok(blocks, n, 16) || !arr_ok(out, n, 32)) return RRQ_ERR_INVALID;
  if (n == 0) return RRQ_OK;
  const float inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  return status_of(rrq::launch_q4_0_decode(blocks, n, d, seed, rotate, inv_sqrt_d, out, out_dtype,
                                           as_stream(stream)));
}

// QJL projection on the host: Box–Muller from two SplitMix64 outputs per entry,
// rounded to bf16 (nearest even) directly from double.
int rrq_qjl_matrix(uint64_t seed, int d, uint16_t* S) {
  if (!d_ok(d) || S == nullptr) return RRQ_ERR_INVALID;
  auto out = [seed](uint64_t c) {
    uint64_t z = seed + (c + 1ull) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  };
  const double two_pi = 6.283185307179586476925286766559;
  const int64_t total = int64_t(d) * d;
  for (int64_t e = 0; e < total; ++e) {
    const double u1 = double(out(2 * uint64_t(e)) >> 11) * (1.0 / 9007199254740992.0);
    const double u2 = double(out(2 * uint64_t(e) + 1) >> 11) * (1.0 / 9007199254740992.0);
    const double z = std::sqrt(-2.0 * std::log(1.0 - u1)) * std::cos(two_pi * u2);
    // round to bf16: keep 8 significant bits, ties to even (exact in double)
    int ex = 0;
    const double m = std::frexp(z, &ex);  // z = m·2^ex, 0.5 ≤ |m| < 1
    const double r = std::nearbyint(std::ldexp(m, 8));
    const float f = static_cast<float>(std::ldexp(r, ex - 8));  // exact in float
    uint32_t bits;
    std::memcpy(&bits, &f, 4);
    S[e] = static_cast<uint16_t>(bits >> 16);
  }
  return RRQ_OK;
}

}  // extern "C"

/*
 * rrq.h — random-rotation vector quantisation for KV-cache and embedding vectors
 * on NVIDIA B200 (sm_100a).  C ABI of librrq.so.
 *
 * The method ("Random-rotation quantization" page, brain.bigb.es, intro "the
 * scheme", steps 1–3): rotate each vector by a random orthogonal Π, quantise
 * every rotated coordinate independently with one fixed codebook computed once
 * for the post-rotation marginal, and at decode time dequantise and apply Πᵀ.
 * Π is the randomized Hadamard transform (section "Why rotation works";
 * "TurboQuant and per-layer outlier-aware K" page, section "TurboQuant 2026":
 * the FWHT):
 *
 *     Π = H·D/√d,  D = diag(s_0 .. s_{d-1}),  s_i = ±1,
 *     H = Sylvester–Hadamard matrix of order d in natural order,
 *     H_ij = (−1)^popcount(i & j).
 *
 * s_i = −1 exactly when bit 63 of SplitMix64 output number i is set, where
 * output c of a generator seeded with `seed` is mix(seed + (c+1)·0x9E3779B97F4A7C15)
 * (Steele, Lea & Flood 2014).  One D per call, shared by every vector.
 *
 * Common conventions
 * ------------------
 *  - Every data pointer is a DEVICE pointer owned by the caller, except where
 *    an argument says "host".  The library allocates no device memory and
 *    keeps no per-call state; it never synchronises the stream.
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).  Inputs and outputs must not alias.
 *  - Vectors are rows of a dense row-major [n × d] array; a KV tensor
 *    [tokens × heads × d] is n = tokens·heads rows, row t·heads + h.
 *  - d is a power of two in [64, 512]; bits in 1..4; n ≥ 0 (n = 0 is a
 *    no-op returning RRQ_OK).
 *  - Vector and code arrays must be 32-byte aligned (the kernels move whole
 *    32-byte sectors); norm arrays 4-byte; other alignments are stated per
 *    entry point.
 *  - Element types: RRQ_F32 (float), RRQ_F16 (IEEE binary16), RRQ_BF16.
 *  - Arguments are validated before any launch; an invalid call returns
 *    RRQ_ERR_INVALID and touches no memory.  A failed launch returns
 *    RRQ_ERR_CUDA.  Non-finite inputs give unspecified codes (no fault).
 *  - fp32 / bf16 inputs need 1e-18 < ‖x‖₂ < 1e18 (the squared norm is
 *    accumulated in fp32); fp16 inputs have no range restriction.
 *
 * Codebook (`codebook` arguments)
 * -------------------------------
 *  A HOST pointer to 2^bits strictly ascending finite floats, copied by value
 *  at the call, or NULL for the Lloyd–Max codebook of N(0,1) ("Random-rotation
 *  quantization" page, section "History", EDEN bullet: 1-bit ±√(2/π),
 *  2-bit ±0.453, ±1.510).  Decision thresholds are the midpoints
 *  τ_k = (c_k + c_{k+1})/2 (nearest-centroid cells; section "Three decoders,
 *  one rotation", MSE decoder).  A codebook that is exactly symmetric
 *  (c_k = −c_{L−1−k}) takes a faster path; any ascending codebook is accepted.
 *
 * Packed code format (RRQ_FORMAT_VERSION 1)
 * -----------------------------------------
 *  Per vector d·bits/8 bytes; coordinate i occupies bits [i·bits, (i+1)·bits)
 *  of the byte string, least significant bit first (bits = 4: coordinate 2j
 *  in the low nibble of byte j).  Code k means level c_k (code 0 = most
 *  negative).  The per-vector scale is a separate fp32 array: ν = ‖x‖₂.
 */
#ifndef RRQ_H
#define RRQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RRQ_FORMAT_VERSION 1

/* status codes */
#define RRQ_OK 0
#define RRQ_ERR_INVALID 1     /* bad argument, detected before any launch       */
#define RRQ_ERR_CUDA 2        /* a CUDA launch or runtime call failed           */
#define RRQ_ERR_UNSUPPORTED 3 /* valid request the library does not implement  */
#define RRQ_ERR_SCRATCH 4     /* request larger than the fixed scratch of
                                 rrq_attention_decode_noalloc                   */

/* element types */
#define RRQ_F32 0
#define RRQ_F16 1
#define RRQ_BF16 2

/* GGML block types for rrq_ggml_rot (the numbers of ggml's own type enumeration) */
#define RRQ_GGML_Q4_0 2
#define RRQ_GGML_Q4_1 3
#define RRQ_GGML_Q5_0 6
#define RRQ_GGML_Q5_1 7
#define RRQ_GGML_Q8_0 8

/* Packed-format version this library writes and reads. */
int rrq_format_version(void);

/* Static, NUL-terminated description of a status code (never NULL). */
const char* rrq_strerror(int status);

/*
 * rrq_codebook — the default codebook: ascending Lloyd–Max levels for N(0,1).
 * "Random-rotation quantization" page, section "History", EDEN bullet.
 * Computed on the host in double by Lloyd's iteration (centroid of each
 * nearest-level cell under the normal density, thresholds at midpoints) and
 * rounded to float; exactly symmetric.
 *   bits    1..4
 *   levels  HOST, float[2^bits], written in ascending order
 * Returns RRQ_OK or RRQ_ERR_INVALID.  Thread-safe; no CUDA call.
 */
int rrq_codebook(int bits, float* levels);

/*
 * rrq_rotate — y = Πx (inverse = 0) or y = Πᵀx (inverse = 1), fp32 output.
 * "Random-rotation quantization" page, scheme steps 1 and 3, and section
 * "Why rotation works" (randomized Hadamard transform).
 *   x      [n × d] of x_dtype
 *   y      [n × d] float
 * Errors: RRQ_ERR_INVALID (d, dtype, n, null or misaligned pointer),
 * RRQ_ERR_CUDA.
 */
int rrq_rotate(const void* x, int x_dtype, int64_t n, int d, uint64_t seed, int inverse,
               float* y, void* stream);

/*
 * rrq_encode — quantise n vectors.
 * "Random-rotation quantization" page: scheme steps 1–2; "History", EDEN
 * bullet (normalise to ≈N(0,1), Lloyd–Max codebook) and TurboQuant bullet
 * (constant per-vector scale); "Three decoders, one rotation", MSE decoder.
 * For each vector x:
 *     ν = ‖x‖₂,  u = √d·Πx/ν  (u = 0 when ν = 0),
 *     code_i = #{k : u_i > τ_k}   (a value on a threshold takes the lower code),
 * codes are packed as described above and ν is stored as fp32.
 *
 * Optional QJL stage ("History", QJL and TurboQuant bullets: a 1-bit sign
 * sketch of the residual makes inner products unbiased; "Bias vs
 * unbiasedness"): when qjl_S is non-NULL, also
 *     r = Πx − ŷ,  ŷ = (ν/√d)·c[code]  (the decoder's rotated-domain value),
 *     qjl_bits bit i = [ (S·r)_i > 0 ],  qjl_rnorm = ‖r‖₂,
 * with S the d×d matrix at qjl_S (bf16, row-major, see rrq_qjl_matrix).
 * The product S·r runs on the tensor cores (tcgen05): for fp32 x with r split
 * exactly into three bf16 parts (an fp32-accurate product); for 16-bit x with
 * r scaled by a power of two and split into two fp16 parts and S rounded to
 * fp16 (the sign of an output can differ only where |(S·r)_i| < 1e-5·‖r‖₂).
 *   x          [n × d] of x_dtype
 *   codes      [n × d·bits/8] bytes (output)
 *   norms      [n] float (output)
 *   qjl_S      bf16 [d × d] or NULL (no QJL; then qjl_bits/qjl_rnorm ignored)
 *   qjl_bits   [n × d/8] bytes (output, with qjl_S)
 *   qjl_rnorm  [n] float (output, with qjl_S)
 * Errors: RRQ_ERR_INVALID (bad d / bits / dtype / codebook, null or
 * misaligned pointer), RRQ_ERR_UNSUPPORTED (QJL with d other than 128),
 * RRQ_ERR_CUDA.
 */
int rrq_encode(const void* x, int x_dtype, int64_t n, int d, int bits, uint64_t seed,
               const float* codebook, uint8_t* codes, float* norms,
               const uint16_t* qjl_S, uint8_t* qjl_bits, float* qjl_rnorm, void* stream);

/*
 * rrq_decode — reconstruct n vectors from codes and norms.
 * "Random-rotation quantization" page, scheme step 3 and "Three decoders,
 * one rotation", MSE decoder:
 *     ŷ_i = (ν/√d)·c[code_i],   x̂ = Πᵀŷ = (ν/d)·D·H·c[code],
 * computed in fp32 and rounded to out_dtype (round to nearest even).
 *   codes  [n × d·bits/8] bytes;  norms [n] float
 *   out    [n × d] of out_dtype
 * Errors: RRQ_ERR_INVALID, RRQ_ERR_CUDA.
 */
int rrq_decode(const uint8_t* codes, const float* norms, int64_t n, int d, int bits,
               uint64_t seed, const float* codebook, void* out, int out_dtype, void* stream);

/*
 * rrq_drive_encode — DRIVE's one-bit encoder.
 * "Random-rotation quantization" page, "History", DRIVE bullet (one bit per
 * coordinate, sign(R(x)), plus one scale; ‖R(x)‖₁/d is the biased, MSE-optimal
 * choice and ‖x‖₂²/‖R(x)‖₁ the unbiased one), and "Three decoders, one
 * rotation", mean decoder x̂ = S·Πᵀ·sign(Πx).  For each vector x:
 *     bit_i = [ (Πx)_i > 0 ]   (0 decodes to −1, 1 to +1),
 *     S = ‖Πx‖₁/d (unbiased = 0) or ‖x‖₂²/‖Πx‖₁ (unbiased = 1; 0 when x = 0),
 *     scales = fp32(S·√d).
 * Bits are packed as rrq_encode's one-bit codes, and the stored value is what
 * rrq_decode and rrq_qk_scores read as the norm, so rrq_decode(bits = 1,
 * codebook {−1, +1}) returns S·Πᵀ·sign(Πx) and rrq_qk_scores with the same
 * codebook returns scale·S·⟨Πq, sign(Πx)⟩.
 *   x       [n × d] of x_dtype
 *   codes   [n × d/8] bytes (output);  scales [n] float (output)
 * Errors: RRQ_ERR_INVALID (d, dtype, unbiased not 0/1, null or misaligned
 * pointer), RRQ_ERR_CUDA.
 */
int rrq_drive_encode(const void* x, int x_dtype, int64_t n, int d, uint64_t seed, int unbiased,
                     uint8_t* codes, float* scales, void* stream);

/*
 * rrq_qk_scores — decode-time attention scores against a quantised K cache,
 * without decoding it.  "Random-rotation quantization" page, "Three decoders,
 * one rotation", inner-product decoder: <q, x> is recovered from <Πq, code(Πx)>
 * and a normalising scalar.  With q' = Πq (rotated once per call):
 *     scores[h][t] = scale · (ν_{t,g}/√d) · Σ_i q'_{h,i} · c[code_{t,g,i}]
 *                  = scale · <q_h, x̂_{t,g}>,    g = ⌊h·hkv/hq⌋ (GQA groups).
 *   q       [hq × d] half (unrotated query heads)
 *   codes   [T·hkv × d·bits/8] bytes, row t·hkv + g;  norms [T·hkv] float
 *   scores  [hq × T] float (output)
 * hq must be a multiple of hkv with hq/hkv in {1, 2, 4, 8}.
 * Accuracy: fp16 query values (each head scaled by a power of two) times fp16
 * levels, summed in fp32 (tensor-core tiles for 4-bit codes at d ≤ 128, fp16 pairs
 * with fp32 partial sums otherwise); the error is far below 1e-3·‖q‖·‖x̂‖ for
 * bits ≤ 4.
 * Errors: RRQ_ERR_INVALID, RRQ_ERR_UNSUPPORTED (group size), RRQ_ERR_CUDA.
 */
int rrq_qk_scores(const void* q, int hq, const uint8_t* codes, const float* norms, int64_t T,
                  int hkv, int d, int bits, uint64_t seed, const float* codebook, float scale,
                  float* scores, void* stream);

/*
 * rrq_qk_scores_qjl — unbiased decode-time attention scores on keys stored as
 * b-bit MSE codes plus the QJL one-bit residual sketch (rrq_encode with qjl_S).
 * "Random-rotation quantization" page: "History", TurboQuant bullet (a biased
 * MSE quantiser followed by an unbiased one-bit stage on the residual) and QJL
 * bullet; "Three decoders, one rotation", inner-product decoder; "Bias vs
 * unbiasedness".  With g = ⌊h·hkv/hq⌋:
 *     scores[h][t] = scale · ( <q_h, x̂_{t,g}>
 *                              + √(π/2)/d · ρ_{t,g} · <S·Π·q_h, sign_{t,g}> ),
 * x̂ the b-bit MSE reconstruction (as rrq_qk_scores), sign_i = +1 where QJL bit i
 * is set and −1 elsewhere, ρ the stored residual norm.  Averaged over the
 * Gaussian S the score is unbiased for scale·<q_h, x_{t,g}>.
 *   q          [hq × d] fp16 (unrotated)
 *   codes      [T·hkv × d·bits/8] bytes, row t·hkv + g;  norms [T·hkv] float
 *   qjl_bits   [T·hkv × d/8] bytes;  qjl_rnorm [T·hkv] float (as rrq_encode writes)
 *   qjl_S      bf16 [d × d] (the S given to rrq_encode)
 *   scores     [hq × T] float (output)
 * d must be 128; hq a multiple of hkv with hq/hkv in {1, 2, 4, 8}.
 * Accuracy: both dot products as fp16 × fp16 products summed in fp32 (tensor-core
 * tiles), each head's query and projected query scaled by a power of two.
 * Errors: RRQ_ERR_INVALID, RRQ_ERR_UNSUPPORTED (d other than 128, group size),
 * RRQ_ERR_CUDA.
 */
int rrq_qk_scores_qjl(const void* q, int hq, const uint8_t* codes, const float* norms,
                      const uint8_t* qjl_bits, const float* qjl_rnorm, const uint16_t* qjl_S,
                      int64_t T, int hkv, int d, int bits, uint64_t seed, const float* codebook,
                      float scale, float* scores, void* stream);

/*
 * rrq_attention_decode — one decode step of attention over a quantised K/V cache.
 * "Attn-rot (TurboQuant lite) in llama.cpp" page, "What kind of beast is
 * Attn-rot" (keys and values both quantised after a rotation);
 * "Random-rotation quantization" page, "Three decoders, one rotation" (the MSE
 * decoder is the one for KV-cache compression).  With g = ⌊h·hkv/hq⌋:
 *     s[h][t] = scale · <q_h, k̂_{t,g}>         (as rrq_qk_scores, K codebook and seed),
 *     p[h][t] = exp(s[h][t] − max_t s[h][·]) / Σ_t exp(s[h][t] − max_t s[h][·]),
 *     out[h]  = Σ_t p[h][t] · v̂_{t,g}          (v̂ as rrq_decode, V codebook and seed).
 * The values are summed in their rotated domain and rotated back once per head.
 *   q          [hq × d] fp16
 *   k_codes    [T·hkv × d·k_bits/8] bytes, row t·hkv + g;  k_norms [T·hkv] float
 *   v_codes    [T·hkv × d·v_bits/8] bytes;                 v_norms [T·hkv] float
 *   k_codebook, v_codebook: HOST float[2^bits] or NULL (the default codebook)
 *   workspace  device scratch of workspace_bytes ≥ rrq_attention_workspace_bytes(
 *              hq, hkv, d, k_bits, v_bits, T), 256-byte aligned, owned by the caller,
 *              and ZERO before its first use: each call leaves its counters at zero
 *              again.  Calls that share a workspace must not overlap on the GPU.
 *   out        [hq × d] float (output)
 * d ∈ {64, 128, 256, 512}, K and V codes of 1 to 4 bits; hq a multiple of hkv
 * with hq/hkv in {1, 2, 4, 8} (at most 4 for d = 512); T ≥ 1.  Scores as
 * rrq_qk_scores (fp16 operands, fp32 sums); softmax in fp32.  d = 128 with 4-bit
 * K and V runs as one fused kernel whose value sums take fp16 levels and fp16
 * weights with fp32 accumulation; the weights are p·ν relative to the largest
 * p·ν of the head (exponent and log2 ν added before the one exponential), so any
 * finite value norm keeps its precision.  Every other shape writes the scores
 * to the workspace (hq × T floats) and sums the values in fp32.  Either way, per
 * head the output is within 2e-3·Σ_t p_t·‖v̂_t‖ of the exact softmax-weighted sum
 * of the reconstructions.
 * Errors: RRQ_ERR_INVALID (incl. a workspace that is too small), RRQ_ERR_UNSUPPORTED
 * (d, bits, group size; for d = 128 with 4-bit codes also a device whose
 * per-block reserved shared memory is not the 1 KB the fused kernel's shared
 * layout assumes), RRQ_ERR_CUDA.
 */
int rrq_attention_decode(const void* q, int hq, const uint8_t* k_codes, const float* k_norms,
                         const uint8_t* v_codes, const float* v_norms, int64_t T, int hkv, int d,
                         int k_bits, uint64_t k_seed, const float* k_codebook, int v_bits,
                         uint64_t v_seed, const float* v_codebook, float scale, void* workspace,
                         size_t workspace_bytes, float* out, void* stream);

/*
 * rrq_attention_decode_noalloc — rrq_attention_decode without a workspace argument
 * and without allocating anything.  The pages have no counterpart: this entry is
 * for callers that cannot allocate device memory at the point of the call, such
 * as a serving loop whose memory is reserved up front by its own allocator (a
 * cudaMalloc there would synchronise the device and fragment the pool) or code
 * deep in a call chain that has no workspace to pass down.
 * Its scratch is a fixed 4 MiB array inside the library's device image, so every
 * GPU that loads the library holds those 4 MiB until the process exits.  Requests
 * whose workspace (rrq_attention_workspace_bytes) exceeds 4 MiB are rejected with
 * RRQ_ERR_SCRATCH before anything is launched.
 * The first call on a device looks up the array's address on that device (once)
 * and keeps it for the life of the process; make that first call before any
 * stream capture.  A cudaDeviceReset() of that device invalidates the kept
 * address: do not call this entry on a device after resetting it.  Each call clears the array's
 * counters on `stream` before its kernel runs.  All calls share the one array:
 * calls whose GPU work overlaps (other streams, other host threads) race and
 * give wrong results; calls ordered on one stream are safe.
 * Arguments, outputs and the other errors as rrq_attention_decode.
 */
int rrq_attention_decode_noalloc(const void* q, int hq, const uint8_t* k_codes,
                                 const float* k_norms, const uint8_t* v_codes,
                                 const float* v_norms, int64_t T, int hkv, int d, int k_bits,
                                 uint64_t k_seed, const float* k_codebook, int v_bits,
                                 uint64_t v_seed, const float* v_codebook, float scale,
                                 float* out, void* stream);

/*
 * rrq_attention_workspace_bytes — the workspace rrq_attention_decode needs for
 * (hq, hkv, d, k_bits, v_bits, T) on the current device (it depends on the SM
 * count and, for the shapes other than d = 128 with 4-bit K and V, on how many
 * CTAs of the value kernel for that d and V width one SM holds), or 0 for an
 * invalid shape.  d = 128 with 4-bit K and V needs the counters and partial
 * states only (well under 1 MB for 32 query heads); every other shape adds
 * hq × T floats of scores.  No CUDA work beyond reading the device's attributes
 * and the kernels' occupancy.
 */
size_t rrq_attention_workspace_bytes(int hq, int hkv, int d, int k_bits, int v_bits, int64_t T);

/*
 * rrq_q4_0_rot — "Attn-rot" (TurboQuant lite): rotate, then q4_0.
 * "Attn-rot (TurboQuant lite) in llama.cpp" page: rotate K/V before an
 * ordinary block format, q4_0 first of all.  With y = Πx (rotate = 1) or
 * y = x (rotate = 0), per block of 32 consecutive coordinates:
 *     m = the element of largest |y| (first on ties), Δ = m/−8 (fp32),
 *     q_j = min(15, ⌊fp32(fp32(y_j·inv) + 8.5)⌋),  inv = fp32(1/Δ) (0 when Δ = 0),
 * stored as 18 bytes: fp16(Δ) little endian, then byte j = q_j | q_{j+16}<<4
 * (the public llama.cpp q4_0 block, kept identical for interoperability).
 *   x       [n × d] of x_dtype (d a multiple of 32 within [64, 512])
 *   blocks  [n × d/32 × 18] bytes (output; 16-byte aligned)
 * Errors: RRQ_ERR_INVALID, RRQ_ERR_CUDA.
 */
int rrq_q4_0_rot(const void* x, int x_dtype, int64_t n, int d, uint64_t seed, int rotate,
                 void* blocks, void* stream);

/*
 * rrq_q4_0_rot_decode — inverse of rrq_q4_0_rot: ŷ_j = (q_j − 8)·fp16(Δ), then
 * x̂ = Πᵀŷ when rotate = 1; fp32 arithmetic, rounded to out_dtype.
 *   blocks  [n × d/32 × 18] bytes;  out [n × d] of out_dtype
 */
int rrq_q4_0_rot_decode(const void* blocks, int64_t n, int d, uint64_t seed, int rotate,
                        void* out, int out_dtype, void* stream);

/*
 * rrq_ggml_block_bytes — bytes of one block of 32 values of a GGML block type:
 * 18 (q4_0), 20 (q4_1), 22 (q5_0), 24 (q5_1), 34 (q8_0); 0 for any other type.
 */
int rrq_ggml_block_bytes(int type);

/*
 * rrq_ggml_rot — "Attn-rot" with any of the GGML block types the page lists:
 * rotate (rotate = 1: y = Πx, orthonormal; rotate = 0: y = x), then blocks of 32.
 * "Attn-rot (TurboQuant lite) in llama.cpp" page, "How to use it": q4_0 first of
 * all, also q4_1, q5_0, q5_1 (and q8_0).  The page names the types without
 * defining them; the public llama.cpp blocks are used, kept identical for
 * interoperability, with every decision in fp32 (y rounded to fp32, each
 * product, sum and quotient rounded, no fused multiply-add), inv = fp32(1/Δ),
 * 0 when Δ = 0:
 *   q4_0  as rrq_q4_0_rot (18 bytes);
 *   q4_1  lo, hi = first min / max in index order, Δ = (hi − lo)/15,
 *         q_j = min(15, ⌊(y_j − lo)·inv + 0.5⌋); 20 bytes: fp16 Δ, fp16 lo, then
 *         byte j = q_j | q_{j+16} << 4;
 *   q5_0  m = first element of largest |y| (+0 for a block of zeros), Δ = m/−16,
 *         q_j = min(31, ⌊y_j·inv + 16.5⌋); 22 bytes: fp16 Δ, a little-endian
 *         32-bit word whose bit j is bit 4 of q_j, then byte j = (q_j & 15) |
 *         (q_{j+16} & 15) << 4;
 *   q5_1  as q4_1 with Δ = (hi − lo)/31 and no clamp; 24 bytes: fp16 Δ, fp16 lo,
 *         the high-bit word, the nibble bytes;
 *   q8_0  Δ = max|y|/127, q_j = round(y_j·inv) (halves away from zero); 34
 *         bytes: fp16 Δ, then q_j as signed bytes.
 *   x       [n × d] of x_dtype (d in {64, 128, 256, 512})
 *   type    RRQ_GGML_Q4_0 / _Q4_1 / _Q5_0 / _Q5_1 / _Q8_0
 *   blocks  [n × d/32 × rrq_ggml_block_bytes(type)] bytes (output; 16-byte aligned)
 * Errors: RRQ_ERR_INVALID (type, d, dtype, rotate, null or misaligned pointer),
 * RRQ_ERR_CUDA.
 */
int rrq_ggml_rot(const void* x, int x_dtype, int64_t n, int d, uint64_t seed, int rotate, int type,
                 void* blocks, void* stream);

/*
 * rrq_ggml_rot_decode — inverse of rrq_ggml_rot: with the stored fp16 values,
 * ŷ_j = q_j·Δ + lo (q4_1, q5_1), (q_j − 16)·Δ (q5_0), q_j·Δ (q8_0), (q_j − 8)·Δ
 * (q4_0); then x̂ = Πᵀŷ when rotate = 1.  fp32 arithmetic (q·Δ + lo as one fused
 * multiply-add), rounded to out_dtype.
 *   blocks  [n × d/32 × rrq_ggml_block_bytes(type)] bytes;  out [n × d] of out_dtype
 * Errors: RRQ_ERR_INVALID, RRQ_ERR_CUDA.
 */
int rrq_ggml_rot_decode(const void* blocks, int type, int64_t n, int d, uint64_t seed, int rotate,
                        void* out, int out_dtype, void* stream);

/*
 * rrq_qjl_matrix — the QJL projection S for a seed, on the HOST.
 * Entry e = i·d + j: u1, u2 = top 53 bits of SplitMix64 outputs 2e, 2e+1 as
 * uniforms in [0,1); z = sqrt(−2 ln(1 − u1))·cos(2π·u2) (Box–Muller);
 * S[i][j] = bf16(z) (nearest even).  Written as bf16 bit patterns; the
 * caller copies S to the device once and passes it to rrq_encode.
 *   S  HOST, uint16_t[d × d]
 * d a power of two in [64, 512].  Errors: RRQ_ERR_INVALID.
 */
int rrq_qjl_matrix(uint64_t seed, int d, uint16_t* S);

#ifdef __cplusplus
}
#endif

#endif /* RRQ_H */

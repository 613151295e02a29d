// rrq_device.cuh — device building blocks shared by the rrq kernels (sm_100a).
//
// Lane layout.  A vector of D coordinates is owned by a group of G = D/C
// consecutive lanes of a warp, each lane holding C coordinates (C ≤ 128, a
// per-kernel choice; 32/G vectors per warp).  The vector is cut into sectors
// of 16 consecutive coordinates (32 bytes of fp16/bf16, one DRAM sector);
// sector q lives in lane h = q mod G, slot s = q / G.  Each lane moves whole
// sectors with 256-bit loads and stores (sm_100 `ld/st.global.v8.b32`), and
// for G > 1 the G lanes of a vector read G adjacent sectors in one
// instruction.  Lane h holds values v[r], r = s·16 + e, of coordinate
// i = (s·G + h)·16 + e: bits 0..3 of i are e (local), bits 4..4+log2(G)−1 are
// the lane bits h, the remaining bits are s (local).
//
// Walsh–Hadamard transform.  The unnormalised transform y = H·v with
// H_ij = (−1)^popcount(i&j) factors into one butterfly (a, b) → (a+b, a−b)
// per bit of i, in any order.  Local bits are butterflies between registers
// (on packed fp32 pairs: sm_100 issues two fp32 additions per instruction);
// lane bits are one __shfl_xor_sync per value, the lower lane adding and the
// upper lane subtracting.  ("Random-rotation quantization" page, section "Why
// rotation works": the randomized Hadamard transform, O(d log d).)
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <utility>

#include "rrq_params.h"

namespace rrq {

// ------------------------------------------------ programmatic dependent launch
// Every rrq kernel is launched with programmatic stream serialization allowed
// (`launch_pdl`), so when the kernel before it in the stream lets its
// dependents start, this kernel's CTAs launch early and build their
// shared-memory tables while that kernel drains.  `pdl_wait()` blocks until
// the previous kernel has completed and its memory is visible; every kernel
// calls it before its first global-memory access (read or write).  Launched
// without a dependency, it returns at once.  `pdl_release()` lets the next
// kernel in the stream launch; its CTAs still wait for this kernel's
// completion before touching memory.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch `kernel` on `stream` with programmatic stream serialization allowed.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

constexpr unsigned kFull = 0xffffffffu;

// ----------------------------------------------------------------- SplitMix64
// Output number c of SplitMix64 seeded with `seed` (Steele, Lea & Flood 2014;
// constants of the public reference implementation).
__host__ __device__ __forceinline__ uint64_t splitmix64_at(uint64_t seed, uint64_t c) {
  uint64_t z = seed + (c + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Rotation sign of coordinate i: 1 (negative) when bit 63 of output i is set.
__host__ __device__ __forceinline__ uint32_t sign_bit(uint64_t seed, int i) {
  return uint32_t(splitmix64_at(seed, uint64_t(i)) >> 63);
}

// ------------------------------------------------------------ element types
template <typename T> struct Elem;
template <> struct Elem<float> { static constexpr int kBytes = 4; };
template <> struct Elem<__half> { static constexpr int kBytes = 2; };
template <> struct Elem<__nv_bfloat16> { static constexpr int kBytes = 2; };

// 32-bit words per 16-coordinate sector of T.
template <typename T> constexpr int sector_words() { return 16 * Elem<T>::kBytes / 4; }

// Sign-flip masks in shared memory: one XOR word per element word of a sector
// (sign bits 15 and 31 for a pair of 16-bit elements, bit 31 for fp32).
template <typename T, int D> constexpr int mask_words() { return D / 16 * sector_words<T>(); }

template <typename T, int D>
__device__ __forceinline__ void build_sign_mask(uint32_t* smask, uint64_t seed) {
  if constexpr (Elem<T>::kBytes == 2) {
    for (int k = threadIdx.x; k < D / 2; k += blockDim.x)
      smask[k] = (sign_bit(seed, 2 * k) << 15) | (sign_bit(seed, 2 * k + 1) << 31);
  } else {
    for (int i = threadIdx.x; i < D; i += blockDim.x) smask[i] = sign_bit(seed, i) << 31;
  }
}

// -------------------------------------------------------- 256-bit accesses
struct alignas(32) W8 {
  uint32_t w[8];
};

// Streaming 32-byte load (read once: no L1 allocation).
__device__ __forceinline__ W8 ld256(const void* p) {
  W8 r;
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3]), "=r"(r.w[4]),
                 "=r"(r.w[5]), "=r"(r.w[6]), "=r"(r.w[7])
               : "l"(p));
  return r;
}

// Streaming 32-byte store (evict-first).
__device__ __forceinline__ void st256(void* p, const W8& v) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v.w[0]),
               "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]), "r"(v.w[6]),
               "r"(v.w[7])
               : "memory");
}

// ------------------------------------------------- asynchronous smem copies
// cp.async (global -> shared, bypassing registers).  src_bytes < size
// zero-fills the rest; callers pass an in-bounds source address always.
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Bulk (TMA) copy of a shared-memory range to global memory; the issuing
// thread later waits for the source to be read before reusing it.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void bulk_store(void* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc),
               "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ------------------------------------------------ mbarriers and bulk copies
// Bounded waits: try_wait polls (each suspends for a short hardware-defined
// time) before a wait gives up and the caller reports a failure.
constexpr uint32_t kMbarPolls = 1u << 22;

__device__ __forceinline__ void mbarrier_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
// Makes initialised mbarriers visible to the asynchronous (bulk copy) proxy.
__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbarrier_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbarrier_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for phase `parity` of the mbarrier to complete; false after the
// poll limit.
__device__ __forceinline__ bool mbarrier_wait(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < kMbarPolls; ++i)
    if (mbarrier_try_wait(bar, parity)) return true;
  return false;
}
// Bulk copy global -> shared; completion counted in bytes on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t sdst, const void* gsrc, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          sdst),
      "l"(gsrc), "r"(bytes), "r"(bar)
      : "memory");
}
// Hint: bring a global range into L2 ahead of its bulk copy.
__device__ __forceinline__ void prefetch_l2(const void* gsrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(gsrc), "r"(bytes) : "memory");
}
// TMA tile copies through a tensor map (a __grid_constant__ kernel parameter).
// Load: box at element (x, y) into shared memory, completion in bytes on
// `bar`; store: box from shared memory to element (x, y), one bulk group.
__device__ __forceinline__ void tma_load_2d(uint32_t sdst, const void* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(sdst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_store_2d(const void* map, int x, int y, uint32_t ssrc) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   map),
               "r"(x), "r"(y), "r"(ssrc)
               : "memory");
}
__device__ __forceinline__ void tma_prefetch_2d(const void* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(x),
               "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Byte offset of 16-byte chunk c of 128-byte line r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t swz128(int r, int c) { return uint32_t(r * 128 + ((c ^ (r & 7)) << 4)); }

// Two fp32 values from shared memory (8-byte aligned address).
__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

// One 32-bit word from shared memory.
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// Waits until at most one committed bulk store still reads shared memory.
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// 2 packed 16-bit elements -> 2 floats (exact)
template <typename T> __device__ __forceinline__ float2 unpack2(uint32_t w);
template <> __device__ __forceinline__ float2 unpack2<__half>(uint32_t w) {
  __half2 h = *reinterpret_cast<__half2*>(&w);
  return __half22float2(h);
}
template <> __device__ __forceinline__ float2 unpack2<__nv_bfloat16>(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// 2 floats -> 2 packed 16-bit elements, round to nearest even
template <typename T> __device__ __forceinline__ uint32_t pack2(float2 v);
template <> __device__ __forceinline__ uint32_t pack2<__half>(float2 v) {
  __half2 h = __float22half2_rn(v);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float2 v) {
  __nv_bfloat162 h = __float22bfloat162_rn(v);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------- packed fp32 pairs
// Each component is rounded once, exactly like the scalar operation.
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.f, -1.f), a);  // a − b: b·(−1) is exact
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// ---------------------------------------------------------------- lane layout
template <int D, int C> struct Layout {
  static_assert(C % 16 == 0 && D % C == 0, "C must be a multiple of 16 dividing D");
  static constexpr int G = D / C;       // lanes per vector
  static constexpr int SEC = C / 16;    // sectors per lane
  static constexpr int P = C / 2;       // packed pairs per lane
  static constexpr int VPW = 32 / G;    // vectors per warp
  __host__ __device__ static constexpr int sector(int s, int h) { return s * G + h; }
};

// One sector of raw words -> 8 packed pairs, with optional sign XOR from smem.
template <typename T, bool FLIP>
__device__ __forceinline__ void sector_to_pairs(const uint32_t* raw, const uint32_t* mask,
                                                float2* w) {
  if constexpr (Elem<T>::kBytes == 2) {
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = unpack2<T>(FLIP ? raw[j] ^ mask[j] : raw[j]);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      w[j] = make_float2(__uint_as_float(FLIP ? raw[2 * j] ^ mask[2 * j] : raw[2 * j]),
                         __uint_as_float(FLIP ? raw[2 * j + 1] ^ mask[2 * j + 1] : raw[2 * j + 1]));
  }
}

// The lane's raw input words of one vector.
template <typename T, int D, int C> struct RawVec {
  static constexpr int SW = sector_words<T>();  // 8 (16-bit) or 16 (fp32)
  static constexpr int N = Layout<D, C>::SEC * SW;
  uint32_t r[N];
  __device__ __forceinline__ void load(const T* __restrict__ row, bool valid, int h) {
#pragma unroll
    for (int s = 0; s < Layout<D, C>::SEC; ++s) {
      const T* src = row + Layout<D, C>::sector(s, h) * 16;
#pragma unroll
      for (int c = 0; c < SW / 8; ++c) {
        W8 v;
        if (valid) {
          v = ld256(src + c * (32 / Elem<T>::kBytes));
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) v.w[j] = 0u;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) r[s * SW + c * 8 + j] = v.w[j];
      }
    }
  }
};

template <typename T, int D, int C, bool FLIP>
__device__ __forceinline__ void raw_to_pairs(const RawVec<T, D, C>& raw, int h,
                                             const uint32_t* smask, float2 (&w)[C / 2]) {
  using Lay = Layout<D, C>;
  constexpr int SW = sector_words<T>();
#pragma unroll
  for (int s = 0; s < Lay::SEC; ++s)
    sector_to_pairs<T, FLIP>(&raw.r[s * SW], smask + Lay::sector(s, h) * SW, &w[s * 8]);
}

// Packed pairs of one lane -> stored row (times `scale`), optional sign XOR.
template <typename T, int D, int C, bool FLIP>
__device__ __forceinline__ void store_pairs(T* __restrict__ row, bool valid, int h,
                                            const uint32_t* smask, const float2 (&w)[C / 2],
                                            float scale) {
  using Lay = Layout<D, C>;
  constexpr int SW = sector_words<T>();
  const float2 s2 = make_float2(scale, scale);
#pragma unroll
  for (int s = 0; s < Lay::SEC; ++s) {
    const int q = Lay::sector(s, h);
    const uint32_t* m = smask + q * SW;
#pragma unroll
    for (int c = 0; c < SW / 8; ++c) {
      W8 o;
      if constexpr (Elem<T>::kBytes == 2) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t p = pack2<T>(mul2(w[s * 8 + j], s2));
          o.w[j] = FLIP ? p ^ m[j] : p;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 v = mul2(w[s * 8 + c * 4 + j], s2);
          o.w[2 * j] = FLIP ? __float_as_uint(v.x) ^ m[c * 8 + 2 * j] : __float_as_uint(v.x);
          o.w[2 * j + 1] =
              FLIP ? __float_as_uint(v.y) ^ m[c * 8 + 2 * j + 1] : __float_as_uint(v.y);
        }
      }
      if (valid) st256(row + q * 16 + c * (32 / Elem<T>::kBytes), o);
    }
  }
}

// One lane's whole row (G = 1) times `scale`, sign XOR applied, into shared
// memory at `dst` (16-byte stores, 16-byte aligned).
template <typename T, int D>
__device__ __forceinline__ void store_pairs_smem(uint8_t* dst, const uint32_t* smask,
                                                 const float2 (&w)[D / 2], float scale) {
  const float2 s2 = make_float2(scale, scale);
  if constexpr (Elem<T>::kBytes == 2) {
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {  // chunk c: values 8c .. 8c+7
      const uint4 m = reinterpret_cast<const uint4*>(smask)[c];
      uint4 o;
      o.x = pack2<T>(mul2(w[4 * c + 0], s2)) ^ m.x;
      o.y = pack2<T>(mul2(w[4 * c + 1], s2)) ^ m.y;
      o.z = pack2<T>(mul2(w[4 * c + 2], s2)) ^ m.z;
      o.w = pack2<T>(mul2(w[4 * c + 3], s2)) ^ m.w;
      reinterpret_cast<uint4*>(dst)[c] = o;
    }
  } else {
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {  // chunk c: values 4c .. 4c+3
      const uint4 m = reinterpret_cast<const uint4*>(smask)[c];
      const float2 a = mul2(w[2 * c], s2), b = mul2(w[2 * c + 1], s2);
      reinterpret_cast<uint4*>(dst)[c] =
          make_uint4(__float_as_uint(a.x) ^ m.x, __float_as_uint(a.y) ^ m.y,
                     __float_as_uint(b.x) ^ m.z, __float_as_uint(b.y) ^ m.w);
    }
  }
}

// Unnormalised Walsh–Hadamard transform on packed pairs: w[k] holds values
// r = 2k and 2k+1 of the lane.  Bit 0 of r is a butterfly inside each pair;
// the other local bits pair whole registers; lane bits use shuffles.
// PAIRED = true: the butterfly inside each pair was already applied.
template <int D, int C, bool PAIRED = false>
__device__ __forceinline__ void fwht2(float2 (&w)[C / 2], int h) {
  constexpr int P = C / 2, G = D / C;
  if constexpr (!PAIRED) {
#pragma unroll
    for (int k = 0; k < P; ++k) {
      const float a = w[k].x, b = w[k].y;
      w[k] = make_float2(a + b, a - b);
    }
  }
#pragma unroll
  for (int mm = 1; mm < P; mm <<= 1) {
#pragma unroll
    for (int k = 0; k < P; ++k) {
      if ((k & mm) == 0) {
        const float2 a = w[k], b = w[k | mm];
        w[k] = add2(a, b);
        w[k | mm] = sub2(a, b);
      }
    }
  }
#pragma unroll
  for (int m = 1; m < G; m <<= 1) {
    const float sg = (h & m) ? -1.f : 1.f;
    const float2 sgn = make_float2(sg, sg);
#pragma unroll
    for (int k = 0; k < P; ++k) {
      const float2 t =
          make_float2(__shfl_xor_sync(kFull, w[k].x, m), __shfl_xor_sync(kFull, w[k].y, m));
      w[k] = fma2(w[k], sgn, t);  // lower lane: w + t; upper lane: t − w
    }
  }
}

// Bits [pos, pos+nb) of a little-endian word array (nb ≤ 8; pos and nb are
// constants after unrolling, so the array stays in registers).
__device__ __forceinline__ uint32_t get_bits(const uint32_t* words, int pos, int nb) {
  const int wi = pos >> 5, off = pos & 31;
  uint32_t v = words[wi] >> off;
  if (off + nb > 32) v |= words[wi + 1] << (32 - off);
  return v & ((1u << nb) - 1u);
}

// Sum over the G lanes of a group.
template <int G>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int m = 1; m < G; m <<= 1) x += __shfl_xor_sync(kFull, x, m);
  return x;
}

}  // namespace rrq

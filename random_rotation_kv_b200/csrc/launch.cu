// launch.cu — element-type dispatch for the encode/decode/rotate launchers and
// the occupancy-based grid sizing shared by every grid-stride kernel.
#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "quant_kernels.cuh"

namespace rrq {

extern template cudaError_t encode_typed<__half>(const __half*, int64_t, int, const QuantParams&,
                                                 uint8_t*, float*, cudaStream_t);
extern template cudaError_t encode_typed<__nv_bfloat16>(const __nv_bfloat16*, int64_t, int,
                                                        const QuantParams&, uint8_t*, float*,
                                                        cudaStream_t);
extern template cudaError_t encode_typed<float>(const float*, int64_t, int, const QuantParams&,
                                                uint8_t*, float*, cudaStream_t);
extern template cudaError_t decode_typed<__half>(const uint8_t*, const float*, int64_t, int,
                                                 const QuantParams&, __half*, cudaStream_t);
extern template cudaError_t decode_typed<__nv_bfloat16>(const uint8_t*, const float*, int64_t, int,
                                                        const QuantParams&, __nv_bfloat16*,
                                                        cudaStream_t);
extern template cudaError_t decode_typed<float>(const uint8_t*, const float*, int64_t, int,
                                                const QuantParams&, float*, cudaStream_t);
extern template cudaError_t rotate_typed<__half>(const __half*, int64_t, int, uint64_t, int, float,
                                                 float*, cudaStream_t);
extern template cudaError_t rotate_typed<__nv_bfloat16>(const __nv_bfloat16*, int64_t, int,
                                                        uint64_t, int, float, float*, cudaStream_t);
extern template cudaError_t rotate_typed<float>(const float*, int64_t, int, uint64_t, int, float,
                                                float*, cudaStream_t);

int grid_for(const void* kernel, int threads, size_t smem, int64_t work_blocks) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> per_sm_cache;
  static std::map<int, int> sm_count;
  int dev = 0;
  cudaGetDevice(&dev);
  int per_sm = 1, sms = 1;
  {
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_pair(kernel, dev);
    auto it = per_sm_cache.find(key);
    if (it == per_sm_cache.end()) {
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) !=
              cudaSuccess ||
          per_sm < 1)
        per_sm = 1;
      per_sm_cache[key] = per_sm;
    } else {
      per_sm = it->second;
    }
    auto is = sm_count.find(dev);
    if (is == sm_count.end()) {
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
          sms < 1)
        sms = 1;
      sm_count[dev] = sms;
    } else {
      sms = is->second;
    }
  }
  const int64_t cap = int64_t(per_sm) * sms;
  return int(std::max<int64_t>(1, std::min<int64_t>(work_blocks, cap)));
}

cudaError_t launch_encode(const void* x, int dtype, int64_t n, int d, const QuantParams& p,
                          uint8_t* codes, float* norms, cudaStream_t stream) {
  switch (dtype) {
    case RRQ_F16:
      return encode_typed<__half>(static_cast<const __half*>(x), n, d, p, codes, norms, stream);
    case RRQ_BF16:
      return encode_typed<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x), n, d, p, codes,
                                         norms, stream);
    case RRQ_F32:
      return encode_typed<float>(static_cast<const float*>(x), n, d, p, codes, norms, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const uint8_t* codes, const float* norms, int64_t n, int d,
                          const QuantParams& p, void* out, int out_dtype, cudaStream_t stream) {
  switch (out_dtype) {
    case RRQ_F16:
      return decode_typed<__half>(codes, norms, n, d, p, static_cast<__half*>(out), stream);
    case RRQ_BF16:
      return decode_typed<__nv_bfloat16>(codes, norms, n, d, p,
                                         static_cast<__nv_bfloat16*>(out), stream);
    case RRQ_F32:
      return decode_typed<float>(codes, norms, n, d, p, static_cast<float*>(out), stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_rotate(const void* x, int dtype, int64_t n, int d, uint64_t seed, int inverse,
                          float inv_sqrt_d, float* y, cudaStream_t stream) {
  switch (dtype) {
    case RRQ_F16:
      return rotate_typed<__half>(static_cast<const __half*>(x), n, d, seed, inverse, inv_sqrt_d, y,
                                  stream);
    case RRQ_BF16:
      return rotate_typed<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x), n, d, seed, inverse,
                                         inv_sqrt_d, y, stream);
    case RRQ_F32:
      return rotate_typed<float>(static_cast<const float*>(x), n, d, seed, inverse, inv_sqrt_d, y,
                                 stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rrq

// FP8 E4M3 quantization of a BF16 pool: the lossy comparator of the summary's
// chapter "Lossless or FP8" (FP8 halves the cache but changes the values).
// code = E4M3 nearest to value * inv_scale (single-precision product, round
// to nearest even, saturating at +-448), one scale per pool.
#include <cuda_runtime.h>

#include <cstdint>

#include "zf_device.cuh"
#include "zf_internal.h"

namespace zf {
namespace {

__global__ void __launch_bounds__(256) fp8_quantize_kernel(const uint4* __restrict__ src, int64_t n8,
                                                           float inv_scale, uint2* __restrict__ dst) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const uint4 w = __ldcs(src + i);  // eight bf16 values
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    uint32_t c[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t lo = f32x2_to_e4m3x2(bf16_lo_to_f32(ww[2 * k]) * inv_scale, bf16_hi_to_f32(ww[2 * k]) * inv_scale);
      const uint32_t hi =
          f32x2_to_e4m3x2(bf16_lo_to_f32(ww[2 * k + 1]) * inv_scale, bf16_hi_to_f32(ww[2 * k + 1]) * inv_scale);
      c[k] = (lo & 0xFFFFu) | (hi << 16);
    }
    __stcs(dst + i, make_uint2(c[0], c[1]));
  }
}

}  // namespace
}  // namespace zf

using namespace zf;

extern "C" {

zf_status zf_fp8_quantize(const uint16_t* src, int64_t n_values, float inv_scale, uint8_t* dst,
                          zf_stream_t stream) {
  if (n_values < 0 || n_values % 8 != 0) return ZF_ERR_INVALID_ARG;
  if (!(inv_scale > 0.f) || inv_scale > 3.0e38f) return ZF_ERR_INVALID_ARG;
  if (n_values == 0) return ZF_OK;
  if (!src || !dst || !aligned(src, 16) || !aligned(dst, 8)) return ZF_ERR_INVALID_ARG;
  const int sms = current_sm_count();
  if (sms <= 0) return ZF_ERR_CUDA;
  const int64_t n8 = n_values / 8;
  int64_t blocks = (n8 + 255) / 256;
  if (blocks > int64_t(sms) * 8) blocks = int64_t(sms) * 8;
  fp8_quantize_kernel<<<static_cast<unsigned>(blocks), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint4*>(src), n8, inv_scale, reinterpret_cast<uint2*>(dst));
  return cuda_status(cudaGetLastError());
}

}  // extern "C"

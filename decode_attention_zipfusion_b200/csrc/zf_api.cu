// Small C-ABI calls: version, status names, the device error word.
#include <cuda_runtime.h>

#include "zf_internal.h"

extern "C" {

int zf_version(void) { return 100; }  // 0.1.0

const char* zf_status_string(zf_status s) {
  switch (s) {
    case ZF_OK: return "ZF_OK";
    case ZF_ERR_INVALID_ARG: return "ZF_ERR_INVALID_ARG";
    case ZF_ERR_UNSUPPORTED: return "ZF_ERR_UNSUPPORTED";
    case ZF_ERR_WORKSPACE: return "ZF_ERR_WORKSPACE";
    case ZF_ERR_CUDA: return "ZF_ERR_CUDA";
    case ZF_ERR_BAD_INPUT: return "ZF_ERR_BAD_INPUT";
    case ZF_ERR_TIMEOUT: return "ZF_ERR_TIMEOUT";
  }
  return "ZF_ERR_UNKNOWN";
}

zf_status zf_clear_device_error(void* ws, zf_stream_t stream) {
  if (!ws || !zf::aligned(ws, 4)) return ZF_ERR_INVALID_ARG;
  return zf::cuda_status(cudaMemsetAsync(ws, 0, sizeof(uint32_t), reinterpret_cast<cudaStream_t>(stream)));
}

zf_status zf_get_device_error(const void* ws, int* host_code) {
  if (!ws || !host_code || !zf::aligned(ws, 4)) return ZF_ERR_INVALID_ARG;
  uint32_t v = 0;
  if (cudaMemcpy(&v, ws, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return ZF_ERR_CUDA;
  *host_code = static_cast<int>(v);
  if (v & ZF_DEVERR_TIMEOUT) return ZF_ERR_TIMEOUT;
  return v ? ZF_ERR_BAD_INPUT : ZF_OK;
}

}  // extern "C"

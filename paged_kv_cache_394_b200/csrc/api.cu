// api.cu — version, status strings and the per-thread CUDA error record.
#include "host_common.h"

namespace pkv {
namespace {
thread_local int g_last_cuda_error = 0;
}

pkv_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return PKV_OK;
  g_last_cuda_error = static_cast<int>(e);
  return PKV_ERR_CUDA;
}

}  // namespace pkv

extern "C" const char* pkv_version(void) { return "pagedkv 0.1.0 sm_100a"; }

extern "C" const char* pkv_status_string(int status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID_ARG: return "invalid argument";
    case PKV_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case PKV_ERR_WORKSPACE: return "workspace or staging buffer too small";
    case PKV_ERR_CUDA: return "CUDA runtime error";
    case PKV_ERR_OUT_OF_BLOCKS: return "out of KV-cache blocks";
    default: return "unknown status";
  }
}

extern "C" int pkv_last_cuda_error(void) { return pkv::g_last_cuda_error; }

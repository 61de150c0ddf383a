// Status names and version of the liboda C ABI.
#include <cuda_runtime_api.h>

#include "oda.h"

namespace oda {
namespace {
thread_local int g_last_cuda_error = 0;
}
void note_cuda_error(int err) {
  if (err != 0) g_last_cuda_error = err;
}
}  // namespace oda

extern "C" const char* oda_last_cuda_error(void) {
  const int e = oda::g_last_cuda_error;
  if (e == 0) return "no CUDA error recorded";
  return cudaGetErrorString(static_cast<cudaError_t>(e));
}

extern "C" const char* oda_status_string(int code) {
  switch (code) {
    case ODA_OK: return "ODA_OK";
    case ODA_ERR_INVALID_ARG: return "ODA_ERR_INVALID_ARG";
    case ODA_ERR_UNSUPPORTED_SHAPE: return "ODA_ERR_UNSUPPORTED_SHAPE";
    case ODA_ERR_WORKSPACE_TOO_SMALL: return "ODA_ERR_WORKSPACE_TOO_SMALL";
    case ODA_ERR_CUDA: return "ODA_ERR_CUDA";
    case ODA_ERR_NOT_IMPLEMENTED: return "ODA_ERR_NOT_IMPLEMENTED";
    case ODA_DEV_BAD_BLOCK: return "ODA_DEV_BAD_BLOCK";
    case ODA_DEV_BAD_LEN: return "ODA_DEV_BAD_LEN";
    case ODA_DEV_BAD_KEEP_LIST: return "ODA_DEV_BAD_KEEP_LIST";
    case ODA_DEV_TIMEOUT: return "ODA_DEV_TIMEOUT";
    case ODA_DEV_BAD_DA: return "ODA_DEV_BAD_DA";
    default: return "ODA_UNKNOWN_STATUS";
  }
}

extern "C" int oda_version(void) { return 101; }

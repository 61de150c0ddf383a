// Status names and version of the liboda C ABI.
#include <cuda_runtime_api.h>

#include <atomic>

#include "oda.h"

namespace oda {
namespace {
thread_local int g_last_cuda_error = 0;
constexpr unsigned long long kDefaultWaitNs = 1000000000ull;  // 1 s
std::atomic<unsigned long long> g_wait_ns{kDefaultWaitNs};
std::atomic<int> g_stall{ODA_STALL_NONE};
std::atomic<int> g_local_shape{-1};
}  // namespace
void note_cuda_error(int err) {
  if (err != 0) g_last_cuda_error = err;
}
unsigned long long test_wait_ns() { return g_wait_ns.load(std::memory_order_relaxed); }
int test_stall() { return g_stall.load(std::memory_order_relaxed); }
int test_local_shape() { return g_local_shape.load(std::memory_order_relaxed); }
}  // namespace oda

extern "C" int oda_debug_set_wait_limit(unsigned long long ns) {
  oda::g_wait_ns.store(ns == 0 ? oda::kDefaultWaitNs : ns, std::memory_order_relaxed);
  return ODA_OK;
}

extern "C" int oda_debug_set_local_shape(int index) {
  if (index < -1 || index > 3) return ODA_ERR_INVALID_ARG;
  oda::g_local_shape.store(index, std::memory_order_relaxed);
  return ODA_OK;
}

extern "C" int oda_debug_set_stall(int kind) {
  if (kind < ODA_STALL_NONE || kind > ODA_STALL_LOCAL_PUSH) return ODA_ERR_INVALID_ARG;
  oda::g_stall.store(kind, std::memory_order_relaxed);
  return ODA_OK;
}

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

// Full decode that allocates nothing and takes no workspace from the caller.
//
// Some callers of this library cannot allocate device memory: code that runs while a CUDA
// graph is being captured in a mode that forbids allocation calls, plugins whose host
// framework owns every device allocation (a serving runtime's memory arena), and callers
// that must not risk an allocation failure or the device-wide synchronisation a fresh
// cudaMalloc can imply in the middle of a decode step. For them, the split partials and
// merge tickets of the Full decode live in one file-scope device array. Every GPU that
// loads this library holds that array (2 MiB) until the process exits.
#include "oda_decode.cuh"

namespace oda {
namespace {

constexpr size_t kStaticWsBytes = size_t(2) << 20;  // 2 MiB of scratch per device
__device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

// Device address of g_static_ws in the current device's context. In host code the symbol
// itself is only a host-side stand-in: passing it to a kernel would fault, or silently touch
// the wrong memory where the GPU can reach host memory, so only this looked-up address is
// ever handed to the kernel. It is looked up on every call (a cheap host call once the module
// is loaded) rather than cached: a cache would go stale if the context were torn down and
// created again (the module, and the array, could then sit elsewhere), and a cache shared by
// host threads would need its own synchronisation.
int static_ws_address(void** ptr) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) return ODA_ERR_CUDA;
  *ptr = p;
  return ODA_OK;
}

}  // namespace
}  // namespace oda

extern "C" int oda_decode_full_noalloc(const oda_kv* kv, const void* q, int32_t num_q_heads,
                                       float scale, const int32_t* gate, const void* k_new,
                                       const void* v_new, void* out, int32_t out_dtype,
                                       float* lse, void* stream) {
  int rc = oda::check_kv(kv);
  if (rc != ODA_OK) return rc;
  if (kv->batch == 0) return ODA_OK;
  size_t total = 0, ticket_off = 0;
  if ((rc = oda::decode_ws_layout(kv->batch, kv->num_kv_heads, num_q_heads, &total,
                                  &ticket_off)) != ODA_OK)
    return rc;
  if (total > oda::kStaticWsBytes) return ODA_ERR_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  if ((rc = oda::static_ws_address(&ws)) != ODA_OK) return rc;
  oda_visibility vis = oda::visibility(ODA_MODE_FULL);
  vis.gate = gate;
  // Every host-side check of the launch first, so that a rejected call queues no work at all
  // (no stray write to the shared array, no stray node in a graph being captured).
  oda::DecodeParams p;
  if ((rc = oda::decode_params(kv, vis, q, num_q_heads, scale, k_new, v_new, out, out_dtype, lse,
                               ws, oda::kStaticWsBytes, &p)) != ODA_OK)
    return rc;
  // The array keeps whatever the previous call left; the merge tickets must start at zero.
  if (cudaMemsetAsync(static_cast<unsigned char*>(ws) + ticket_off, 0, total - ticket_off,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ODA_ERR_CUDA;
  return oda::launch_decode(kv, vis, q, num_q_heads, scale, k_new, v_new, out, out_dtype, lse,
                            ws, oda::kStaticWsBytes, stream, 0, 0);
}

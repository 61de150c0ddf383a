// K1: commit of the step's K/V into slot t of the paged cache ([ODA] 접근 방법: the selected
// path's current-position K/V joins the fully retained history). One warp per (sequence,
// KV head): lanes 0-15 move the 256-byte K row, lanes 16-31 the V row, 16 bytes each.
#include "oda_common.cuh"
#include "oda_internal.h"

namespace oda {

__global__ void append_kernel(__nv_bfloat16* k_cache, __nv_bfloat16* v_cache,
                              const int32_t* block_table, const int32_t* seq_lens,
                              int max_blocks, int num_blocks, int hkv,
                              const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                              const int32_t* gate, int* status) {
  const int b = blockIdx.x;
  const int g = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (gate != nullptr && gate[b] == 0) return;
  const int len = seq_lens[b];
  if (len < 1 || len > max_blocks * kPage) {
    if (threadIdx.x == 0) report(status, ODA_DEV_BAD_LEN);
    return;
  }
  const int t = len - 1;
  const int pb = block_table[(size_t)b * max_blocks + t / kPage];
  if (pb < 0 || pb >= num_blocks) {
    if (threadIdx.x == 0) report(status, ODA_DEV_BAD_BLOCK);
    return;
  }
  const bool isk = lane < 16;
  const int li = lane & 15;
  const uint4 v = *reinterpret_cast<const uint4*>((isk ? k_new : v_new) +
                                                  ((size_t)b * hkv + g) * kHeadDim + 8 * li);
  __nv_bfloat16* dst = (isk ? k_cache : v_cache) +
                       (((size_t)pb * hkv + g) * kPage + t % kPage) * kHeadDim + 8 * li;
  *reinterpret_cast<uint4*>(dst) = v;
}

}  // namespace oda

using namespace oda;

extern "C" int oda_kv_append(const oda_kv* kv, const void* k_new, const void* v_new,
                             const int32_t* gate, void* stream) {
  int rc = check_kv(kv);
  if (rc != ODA_OK) return rc;
  if (kv->num_kv_heads > 32) return ODA_ERR_UNSUPPORTED_SHAPE;
  if (kv->batch == 0) return ODA_OK;
  if (k_new == nullptr || v_new == nullptr) return ODA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new)) & 15u)
    return ODA_ERR_INVALID_ARG;
  if (!aligned_or_null(gate, 4)) return ODA_ERR_INVALID_ARG;
  append_kernel<<<kv->batch, 32 * kv->num_kv_heads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<__nv_bfloat16*>(kv->k_cache), static_cast<__nv_bfloat16*>(kv->v_cache),
      kv->block_table, kv->seq_lens, kv->max_blocks_per_seq, kv->num_blocks, kv->num_kv_heads,
      static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new), gate,
      kv->dev_status);
  return cuda_status(cudaGetLastError());
}

// Random gate schedule: the ablation baseline of [ODA] 주요 결과 (learned timing matters),
// which calls Full at the same realised rate as ODA but at random steps. The uniform
// variates are drawn by the caller and passed in; the kernel compares, counts and opens the
// step graph's conditional Full pass exactly as the recall head does.
#include "oda_common.cuh"
#include "oda_internal.h"

namespace oda {

constexpr int kSchedThreads = 256;

__global__ void __launch_bounds__(kSchedThreads)
    gate_schedule_kernel(const float* u, int batch, float rho, int32_t* gate_out,
                         unsigned long long* full_count, cudaGraphConditionalHandle cond,
                         int use_cond) {
  __shared__ unsigned s_count;
  if (threadIdx.x == 0) s_count = 0u;
  __syncthreads();
  unsigned n = 0;
  for (int b = threadIdx.x; b < batch; b += kSchedThreads) {
    const int g = u[b] < rho ? 1 : 0;
    gate_out[b] = g;
    n += g;
  }
  n = __reduce_add_sync(0xffffffffu, n);
  if ((threadIdx.x & 31) == 0 && n) atomicAdd(&s_count, n);
  __syncthreads();
  if (threadIdx.x == 0) {
    if (full_count != nullptr && s_count) {
      atomicAdd(&full_count[0], (unsigned long long)s_count);
      atomicAdd(&full_count[1], 1ull);
    }
    if (use_cond) cudaGraphSetConditional(cond, s_count ? 1u : 0u);
  }
}

int launch_gate_schedule(const float* u, int batch, float rho, int32_t* gate_out,
                         unsigned long long* full_count, unsigned long long graph_cond_handle,
                         void* stream) {
  if (batch < 0 || !(rho >= 0.f && rho <= 1.f)) return ODA_ERR_INVALID_ARG;
  if (batch == 0) return ODA_OK;
  if (u == nullptr || gate_out == nullptr) return ODA_ERR_INVALID_ARG;
  if (!aligned_or_null(u, 4) || !aligned_or_null(gate_out, 4) || !aligned_or_null(full_count, 8))
    return ODA_ERR_INVALID_ARG;
  gate_schedule_kernel<<<1, kSchedThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      u, batch, rho, gate_out, full_count,
      static_cast<cudaGraphConditionalHandle>(graph_cond_handle), graph_cond_handle != 0ull);
  return cuda_status(cudaGetLastError());
}

}  // namespace oda

extern "C" int oda_gate_schedule(const float* u, int32_t batch, float rho, int32_t* gate_out,
                                 unsigned long long* full_count,
                                 unsigned long long graph_cond_handle, void* stream) {
  return oda::launch_gate_schedule(u, batch, rho, gate_out, full_count, graph_cond_handle, stream);
}

// LSE merge of decode partials computed over disjoint position ranges (context-parallel Full:
// every GPU attends its shard of the history, the (O, LSE) pairs are gathered, and this
// kernel combines them). The merge is the usual log-sum-exp rescaling: each part is weighted
// by e^(lse_r - M) with M the largest part normaliser, parts are summed in index order.
#include <math.h>

#include "oda_common.cuh"
#include "oda_internal.h"

namespace oda {

constexpr int kMergeThreads = kHeadDim;  // one thread per output dim
constexpr int kMaxParts = 64;

struct MergeParams {
  const float* o_parts;
  const float* lse_parts;
  int parts, batch, hq;
  const int32_t* gate;
  void* out;
  int out_bf16;
  float* lse;
};

// One CTA per (sequence, query head).
__global__ void __launch_bounds__(kMergeThreads) merge_partials_kernel(const MergeParams p) {
  const int row = blockIdx.x;  // b * hq + h
  const int b = row / p.hq;
  const int tid = threadIdx.x;
  if (p.gate != nullptr && p.gate[b] == 0) return;
  const size_t rows = (size_t)p.batch * p.hq;
  __shared__ float s_w[kMaxParts];
  __shared__ float s_m, s_sum;
  if (tid < 32) {
    float m = -INFINITY;
    for (int r = tid; r < p.parts; r += 32) m = fmaxf(m, p.lse_parts[r * rows + row]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = 0.f;
    for (int r = tid; r < p.parts; r += 32) {
      const float l = p.lse_parts[r * rows + row];
      const float w = (l == -INFINITY) ? 0.f : expf(l - m);
      s_w[r] = w;
      sum += w;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (tid == 0) {
      s_m = m;
      s_sum = sum;
    }
  }
  __syncthreads();
  float o = 0.f, l = -INFINITY;
  if (s_m != -INFINITY) {
    float a = 0.f;
    for (int r = 0; r < p.parts; ++r)
      a = fmaf(s_w[r], __ldg(&p.o_parts[(r * rows + row) * kHeadDim + tid]), a);
    o = a / s_sum;
    l = s_m + logf(s_sum);
  }
  if (p.out_bf16)
    reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)row * kHeadDim + tid] = __float2bfloat16_rn(o);
  else
    reinterpret_cast<float*>(p.out)[(size_t)row * kHeadDim + tid] = o;
  if (p.lse != nullptr && tid == 0) p.lse[row] = l;
}

}  // namespace oda

using namespace oda;

extern "C" int oda_merge_partials(const float* o_parts, const float* lse_parts, int32_t num_parts,
                                  int32_t batch, int32_t num_q_heads, const int32_t* gate,
                                  void* out, int32_t out_dtype, float* lse, void* stream) {
  if (num_parts < 1 || num_parts > kMaxParts || batch < 0 || num_q_heads < 1)
    return ODA_ERR_INVALID_ARG;
  if (out_dtype != ODA_F32 && out_dtype != ODA_BF16) return ODA_ERR_INVALID_ARG;
  if ((long long)batch * num_q_heads >= (1ll << 31) / kHeadDim / kMaxParts)
    return ODA_ERR_UNSUPPORTED_SHAPE;
  if (batch == 0) return ODA_OK;
  if (o_parts == nullptr || lse_parts == nullptr || out == nullptr) return ODA_ERR_INVALID_ARG;
  if (!aligned_or_null(o_parts, 4) || !aligned_or_null(lse_parts, 4) ||
      !aligned_or_null(gate, 4) || !aligned_or_null(out, out_dtype == ODA_BF16 ? 2 : 4) ||
      !aligned_or_null(lse, 4))
    return ODA_ERR_INVALID_ARG;
  MergeParams p;
  p.o_parts = o_parts;
  p.lse_parts = lse_parts;
  p.parts = num_parts;
  p.batch = batch;
  p.hq = num_q_heads;
  p.gate = gate;
  p.out = out;
  p.out_bf16 = out_dtype == ODA_BF16;
  p.lse = lse;
  merge_partials_kernel<<<batch * num_q_heads, kMergeThreads, 0,
                          static_cast<cudaStream_t>(stream)>>>(p);
  return cuda_status(cudaGetLastError());
}

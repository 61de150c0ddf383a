// Recall-head training objective and gradient ([ODA] 핵심 기여 / 접근 방법: the head is trained
// by Huber regression, delta = 1, of q_t on the signed-log target y_t = sign(d_t) log(1 +
// |d_t|), d_t = g_t - lambda, with the backbone frozen). For a batch of B rows:
//   z = W1^T x + b1,  a = GELU(z),  q = w2 . a + b2,  r = q - y,  loss = mean_b Huber(r)
//   dq_b = clip(r_b, -delta, delta) / B,  dw2 = sum_b dq_b a_b,  db2 = sum_b dq_b,
//   dz_b = dq_b w2 * GELU'(z_b),  db1 = sum_b dz_b,  dW1 = sum_b x_b dz_b^T.
// Two launches:
//   1. train_z_kernel     (slab, column tile) CTAs stream W1 once: partial z per slab; the
//                         last slab CTA of each column tile (acquire-release ticket) forms
//                         z, a and q partials for its columns; the last tile then forms q,
//                         the targets, the loss, dq and db2;
//   2. train_grad_kernel  one CTA per 32-row block of W1: dz for every column (recomputed
//                         from z and dq), then its rows of dW1 written once, coalesced; the
//                         first CTA also writes db1 and dw2.
// dW1 (3 hidden x mlp fp32) is written once and W1 read once: the pair bounds the time.
// Every sum runs in a fixed order, so results are bitwise reproducible.
#include <math.h>

#include "oda_common.cuh"
#include "oda_internal.h"
#include "oda_recall.cuh"

namespace oda {

constexpr int kGradRows = 32;   // W1 rows per gradient CTA
constexpr int kMaxTrainBatch = 1024;

struct TrainWs {
  size_t z_part_off, z_off, q_part_off, dq_off, ticket_off, total;
  int slabs, tiles;
};

static size_t align_t(size_t x) { return (x + 255) / 256 * 256; }

static TrainWs train_ws(int batch, int hidden, int mlp) {
  TrainWs w;
  w.slabs = (3 * hidden + kRows - 1) / kRows;
  w.tiles = mlp / kColTile;
  w.z_part_off = 0;
  w.z_off = align_t((size_t)w.slabs * batch * mlp * sizeof(float));
  w.q_part_off = w.z_off + align_t((size_t)batch * mlp * sizeof(float));
  w.dq_off = w.q_part_off + align_t((size_t)w.tiles * batch * sizeof(float));
  w.ticket_off = w.dq_off + align_t((size_t)batch * sizeof(float));
  w.total = w.ticket_off + align_t((size_t)(w.tiles + 1) * sizeof(unsigned));
  return w;
}

struct TrainParams {
  RecallInputs in;
  int batch, hidden, mlp;
  const float* w1;
  const float* b1;
  const float* w2;
  float b2;
  const float* gain;   // [batch] g_t
  float lambda, delta;
  float* q_out;        // nullable [batch]
  float* loss_out;     // [1]
  float* dw1;          // [3 hidden][mlp]
  float* db1;          // [mlp]
  float* dw2;          // [mlp]
  float* db2;          // [1]
  float* z_part;       // [slabs][batch][mlp]
  float* z;            // [batch][mlp], b1 included
  float* q_part;       // [tiles][batch]
  float* dq;           // [batch]
  unsigned* tickets;   // [tiles + 1]
};

__device__ __forceinline__ float gelu_erf_grad(float z) {
  return 0.5f * (1.f + erff(z * 0.70710678118654752f)) +
         z * expf(-0.5f * z * z) * 0.39894228040143268f;  // Phi(z) + z phi(z)
}

__global__ void __launch_bounds__(kRThreads) train_z_kernel(const TrainParams p) {
  __shared__ float xs[kBTile][kRows];
  __shared__ float red[kRowGroups][kBTile][kColTile];
  __shared__ float qs[kRowGroups][2];
  __shared__ int s_last;
  __shared__ float s_h[kMaxTrainBatch], s_dq[kMaxTrainBatch];
  const int tid = threadIdx.x;
  const int rg = tid / kColTile, col = tid % kColTile;
  const int slab = blockIdx.x, tile = blockIdx.y;
  const int slabs = gridDim.x, tiles = gridDim.y;
  const int r0 = slab * kRows;
  const int nrows = min(kRows, 3 * p.hidden - r0);
  const int gcol = tile * kColTile + col;
  float wv[kRowsPerThread];
  load_w1_slab(p.w1, p.mlp, r0, nrows, gcol, rg, wv);
  slab_partial_z(p.in, wv, p.batch, p.mlp, slab, r0, nrows, gcol, xs, red, p.z_part);

  // ---- last slab of this column tile: z (stored for the gradient), GELU, w2 ----
  if (tid == 0) s_last = ticket_arrive(&p.tickets[tile]) == (unsigned)(slabs - 1);
  __syncthreads();
  if (!s_last) return;
  const int bl = tid / kColTile;
  for (int b0 = 0; b0 < p.batch; b0 += kRowGroups) {
    const int b = b0 + bl;
    float v = 0.f;
    if (b < p.batch) {
      const float z = sum_slabs(p.z_part, b, gcol, p.batch, p.mlp, slabs) + p.b1[gcol];
      p.z[(size_t)b * p.mlp + gcol] = z;
      v = gelu_erf(z) * p.w2[gcol];
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((tid & 31) == 0) qs[bl][(tid >> 5) & 1] = v;
    __syncthreads();
    if (tid < kRowGroups && b0 + tid < p.batch)
      p.q_part[(size_t)tile * p.batch + b0 + tid] = qs[tid][0] + qs[tid][1];
    __syncthreads();
  }
  if (tid == 0) p.tickets[tile] = 0u;

  // ---- last column tile: q, the loss and dq ----
  if (tid == 0) s_last = ticket_arrive(&p.tickets[tiles]) == (unsigned)(tiles - 1);
  __syncthreads();
  if (!s_last) return;
  const float inv_b = 1.f / (float)p.batch;
  for (int b = tid; b < p.batch; b += kRThreads) {
    float q = 0.f;
    for (int t = 0; t < tiles; ++t) q += __ldcg(&p.q_part[(size_t)t * p.batch + b]);
    q += p.b2;
    const float d = p.gain[b] - p.lambda;
    const float y = copysignf(log1pf(fabsf(d)), d);
    const float r = q - y;
    const float ar = fabsf(r);
    s_h[b] = ar <= p.delta ? 0.5f * r * r : p.delta * (ar - 0.5f * p.delta);
    const float dq = fminf(fmaxf(r, -p.delta), p.delta) * inv_b;
    s_dq[b] = dq;
    p.dq[b] = dq;
    if (p.q_out != nullptr) p.q_out[b] = q;
  }
  __syncthreads();
  if (tid == 0) {
    float loss = 0.f, db2 = 0.f;
    for (int b = 0; b < p.batch; ++b) {
      loss += s_h[b];
      db2 += s_dq[b];
    }
    *p.loss_out = loss * inv_b;
    *p.db2 = db2;
    p.tickets[tiles] = 0u;  // leave the workspace as found
  }
}

__global__ void __launch_bounds__(kRThreads) train_grad_kernel(const TrainParams p) {
  __shared__ float xs[kBTile][kGradRows];
  const int tid = threadIdx.x;
  const int r0 = blockIdx.x * kGradRows;
  const int nrows = min(kGradRows, 3 * p.hidden - r0);
  for (int c0 = 0; c0 < p.mlp; c0 += kRThreads) {
    const int c = c0 + tid;
    const bool has_c = c < p.mlp;
    const float w2c = has_c ? p.w2[c] : 0.f;
    float acc[kGradRows];
#pragma unroll
    for (int i = 0; i < kGradRows; ++i) acc[i] = 0.f;
    float db1 = 0.f, dw2 = 0.f;
    for (int b0 = 0; b0 < p.batch; b0 += kBTile) {
      const int nb = min(kBTile, p.batch - b0);
      // this column's z and every dq of the tile, all loads issued together (clamped
      // indices; rows past the batch are never used)
      float zv[kBTile], dqv[kBTile];
#pragma unroll
      for (int bb = 0; bb < kBTile; ++bb) {
        const int b = b0 + min(bb, nb - 1);
        zv[bb] = has_c ? __ldcg(&p.z[(size_t)b * p.mlp + c]) : 0.f;
        dqv[bb] = __ldcg(&p.dq[b]);
      }
      __syncthreads();
      {  // one x value per thread: kBTile x kGradRows = 256
        const int bb = tid / kGradRows, i = tid % kGradRows;
        xs[bb][i] = (bb < nb && i < nrows) ? x_at(p.in, b0 + bb, r0 + i) : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int bb = 0; bb < kBTile; ++bb) {
        if (bb < nb && has_c) {
          const float z = zv[bb];
          const float dq = dqv[bb];
          const float dz = dq * w2c * gelu_erf_grad(z);
          db1 += dz;
          dw2 = fmaf(dq, gelu_erf(z), dw2);
#pragma unroll
          for (int i = 0; i < kGradRows; ++i) acc[i] = fmaf(xs[bb][i], dz, acc[i]);
        }
      }
    }
    if (has_c) {
#pragma unroll
      for (int i = 0; i < kGradRows; ++i)
        if (i < nrows) p.dw1[(size_t)(r0 + i) * p.mlp + c] = acc[i];
      if (blockIdx.x == 0) {
        p.db1[c] = db1;
        p.dw2[c] = dw2;
      }
    }
  }
}

}  // namespace oda

using namespace oda;

extern "C" int oda_recall_train_workspace_size(int32_t batch, int32_t hidden, int32_t mlp,
                                               size_t* bytes) {
  if (bytes == nullptr || batch < 0 || batch > kMaxTrainBatch || hidden < 1 || mlp < kColTile ||
      mlp % kColTile != 0)
    return ODA_ERR_INVALID_ARG;
  *bytes = train_ws(batch, hidden, mlp).total;
  return ODA_OK;
}

extern "C" int oda_recall_loss_grad(const float* h_prev, const float* emb, const void* h_local,
                                    int32_t h_local_dtype, int32_t batch, int32_t hidden,
                                    int32_t mlp, const float* w1, const float* b1,
                                    const float* w2, float b2, const float* gain, float lambda,
                                    float delta, float* q_out, float* loss_out, float* dw1,
                                    float* db1, float* dw2, float* db2, void* ws,
                                    size_t ws_bytes, void* stream) {
  if (batch < 0 || batch > kMaxTrainBatch || hidden < 1 || mlp < kColTile ||
      mlp % kColTile != 0)
    return ODA_ERR_INVALID_ARG;
  if (h_local_dtype != ODA_F32 && h_local_dtype != ODA_BF16) return ODA_ERR_INVALID_ARG;
  if (!(delta > 0.f) || !isfinite(delta) || !isfinite(lambda)) return ODA_ERR_INVALID_ARG;
  if (batch == 0) return ODA_OK;
  if (!h_prev || !emb || !h_local || !w1 || !b1 || !w2 || !gain || !loss_out || !dw1 || !db1 ||
      !dw2 || !db2 || !ws)
    return ODA_ERR_INVALID_ARG;
  for (const void* f : {static_cast<const void*>(h_prev), static_cast<const void*>(emb),
                        static_cast<const void*>(w1), static_cast<const void*>(b1),
                        static_cast<const void*>(w2), static_cast<const void*>(gain),
                        static_cast<const void*>(q_out), static_cast<const void*>(loss_out),
                        static_cast<const void*>(dw1), static_cast<const void*>(db1),
                        static_cast<const void*>(dw2), static_cast<const void*>(db2)})
    if (!aligned_or_null(f, 4)) return ODA_ERR_INVALID_ARG;
  if (!aligned_or_null(h_local, h_local_dtype == ODA_BF16 ? 2 : 4) || !aligned_or_null(ws, 16))
    return ODA_ERR_INVALID_ARG;
  const TrainWs wl = train_ws(batch, hidden, mlp);
  if (ws_bytes < wl.total) return ODA_ERR_WORKSPACE_TOO_SMALL;
  TrainParams p;
  p.in.h_prev = h_prev;
  p.in.emb = emb;
  p.in.h_local = h_local;
  p.in.h_local_bf16 = h_local_dtype == ODA_BF16;
  p.in.hidden = hidden;
  p.batch = batch;
  p.hidden = hidden;
  p.mlp = mlp;
  p.w1 = w1;
  p.b1 = b1;
  p.w2 = w2;
  p.b2 = b2;
  p.gain = gain;
  p.lambda = lambda;
  p.delta = delta;
  p.q_out = q_out;
  p.loss_out = loss_out;
  p.dw1 = dw1;
  p.db1 = db1;
  p.dw2 = dw2;
  p.db2 = db2;
  unsigned char* w = static_cast<unsigned char*>(ws);
  p.z_part = reinterpret_cast<float*>(w + wl.z_part_off);
  p.z = reinterpret_cast<float*>(w + wl.z_off);
  p.q_part = reinterpret_cast<float*>(w + wl.q_part_off);
  p.dq = reinterpret_cast<float*>(w + wl.dq_off);
  p.tickets = reinterpret_cast<unsigned*>(w + wl.ticket_off);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  train_z_kernel<<<dim3(wl.slabs, wl.tiles), kRThreads, 0, st>>>(p);
  train_grad_kernel<<<(3 * hidden + kGradRows - 1) / kGradRows, kRThreads, 0, st>>>(p);
  return cuda_status(cudaGetLastError());
}

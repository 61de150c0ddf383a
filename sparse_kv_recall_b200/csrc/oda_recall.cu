// K4: recall head, gate, Full-rate counter and graph condition ([ODA] 접근 방법: the recall
// head scores the step from h_{t-1}, E(x_t) and the current Local final hidden h^L_t, and
// Full is recomputed iff q_t > theta; 개발자 관점: evaluated in FP32 on the GPU, inside the
// same execution stream as Local and the conditional Full pass).
//
// q = w2 . GELU(W1^T x + b1) + b2 with x = [h_prev; emb; h_local] (3 * hidden rows of W1).
// The 3*hidden x mlp weight matrix is split into 256-row slabs x 64-column tiles, one CTA
// each, so the whole GPU streams W1 once per call for every sequence of the batch; each
// thread holds its 64 W1 values in registers, all loads in flight at once. Per column tile,
// the last slab CTA to finish (atomic ticket) sums the slabs' partial z in fixed order, one
// (sequence, column) per thread with 24 loads in flight, and applies b1, GELU and w2; the
// last column tile then forms q, the gate, the counters and the graph condition. For up to
// four sequences one ticket over all CTAs replaces the two levels: the last CTA sums every
// slab of every column itself. Fixed orders make every result bitwise reproducible.
#include <math.h>

#include "oda_common.cuh"
#include "oda_internal.h"
#include "oda_recall.cuh"

namespace oda {

struct RecallWs {
  size_t z_off, q_off, ticket_off, total;
  int slabs, tiles;
};

static size_t align_up_r(size_t x, size_t a) { return (x + a - 1) / a * a; }

static RecallWs recall_ws(int batch, int hidden, int mlp) {
  RecallWs w;
  w.slabs = (3 * hidden + kRows - 1) / kRows;
  w.tiles = mlp / kColTile;
  w.z_off = 0;
  w.q_off = align_up_r((size_t)w.slabs * batch * mlp * sizeof(float), 256);
  w.ticket_off = w.q_off + align_up_r((size_t)w.tiles * batch * sizeof(float), 256);
  w.total = w.ticket_off + align_up_r((size_t)(w.tiles + 1) * sizeof(unsigned), 256);
  return w;
}

struct RecallParams {
  RecallInputs in;
  int batch, hidden, mlp;
  const float* w1;
  const float* b1;
  const float* w2;
  float b2, theta;
  float* q_out;
  int32_t* gate_out;
  unsigned long long* full_count;
  cudaGraphConditionalHandle cond;
  int use_cond;
  float* z_part;      // [slabs][batch][mlp]
  float* q_part;      // [tiles][batch]
  unsigned* tickets;  // [tiles + 1]
};

constexpr int kSmallBatch = 4;  // up to this many sequences: one ticket level (see below)

// Gate, Full-call counters and the graph condition from this thread's q of sequence b.
__device__ __forceinline__ void gate_one(const RecallParams& p, int b, float q,
                                         unsigned* s_count) {
  const int gate = q > p.theta ? 1 : 0;
  p.q_out[b] = q;
  p.gate_out[b] = gate;
  if (gate) atomicAdd(s_count, 1u);
}
__device__ __forceinline__ void publish_gate(const RecallParams& p, unsigned count) {
  if (p.full_count != nullptr && count) {
    atomicAdd(&p.full_count[0], (unsigned long long)count);
    atomicAdd(&p.full_count[1], 1ull);
  }
  if (p.use_cond) cudaGraphSetConditional(p.cond, count ? 1u : 0u);
}

// At most 104 registers: two Local CTAs and one recall CTA fit on an SM together, so the
// recall head can start (programmatic dependent launch) while the last Local layer runs.
__global__ void __maxnreg__(104) recall_kernel(const RecallParams p) {
  __shared__ float xs[kBTile][kRows];
  __shared__ float red[kRowGroups][kBTile][kColTile];
  __shared__ float qs[kRowGroups][2];
  __shared__ int s_last;
  __shared__ unsigned s_count;
  __shared__ float s_red[kRThreads / 32][kSmallBatch];

  const int tid = threadIdx.x;
  const int rg = tid / kColTile, col = tid % kColTile;
  const int slab = blockIdx.x, tile = blockIdx.y;
  const int slabs = gridDim.x, tiles = gridDim.y;
  const int r0 = slab * kRows;
  const int nrows = min(kRows, 3 * p.hidden - r0);
  const int gcol = tile * kColTile + col;

  float wv[kRowsPerThread];  // this thread's W1 column over its rows, all loads in flight
  load_w1_slab(p.w1, p.mlp, r0, nrows, gcol, rg, wv);
  // the final reduction's constants for column tid, in case this CTA ends up doing it
  const float b1_own = tid < p.mlp ? __ldg(&p.b1[tid]) : 0.f;
  const float w2_own = tid < p.mlp ? __ldg(&p.w2[tid]) : 0.f;
  // W1 is constant, so its loads above may overlap the previous kernel (the last Local
  // layer, which writes h_local); slabs that read h_local rows wait for it only now.
  if (r0 + nrows > 2 * p.hidden) griddep_wait();
  griddep_launch_dependents();

  // ---- partial z of this slab for every sequence ----
  slab_partial_z(p.in, wv, p.batch, p.mlp, slab, r0, nrows, gcol, xs, red, p.z_part);

  // ---- small batches: one ticket over every CTA; the last one sums every slab of every
  // column (all loads of a thread in flight together) and reduces q in the CTA, one global
  // round trip shorter than the two-level reduction below ----
  if (p.batch <= kSmallBatch) {
    __syncthreads();  // the CTA's partials are written; thread 0 publishes them (release)
    if (tid == 0) {
      s_last = ticket_arrive(&p.tickets[tiles]) == (unsigned)(slabs * tiles - 1);
      s_count = 0u;
    }
    __syncthreads();  // ... and the last CTA's thread 0 acquired everyone's partials
    if (!s_last) return;
#pragma unroll 1
    for (int b = 0; b < p.batch; ++b) {
      float v = 0.f;
      for (int c = tid; c < p.mlp; c += kRThreads) {
        const bool first = c == tid;  // this column's b1, w2 were fetched before the wait
        v += gelu_erf(sum_slabs(p.z_part, b, c, p.batch, p.mlp, slabs) +
                      (first ? b1_own : p.b1[c])) * (first ? w2_own : p.w2[c]);
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if ((tid & 31) == 0) s_red[tid >> 5][b] = v;
    }
    __syncthreads();
    if (tid < p.batch) {
      float q = 0.f;
#pragma unroll
      for (int w = 0; w < kRThreads / 32; ++w) q += s_red[w][tid];
      gate_one(p, tid, q + p.b2, &s_count);
    }
    __syncthreads();
    if (tid == 0) {
      publish_gate(p, s_count);
      p.tickets[tiles] = 0u;
    }
    return;
  }

  // ---- last slab of this column tile: z, GELU, w2 (summed over the tile's columns) ----
  __syncthreads();
  if (tid == 0) s_last = ticket_arrive(&p.tickets[tile]) == (unsigned)(slabs - 1);
  __syncthreads();
  if (!s_last) return;
  // Thread (bl, col) sums column gcol of sequence b0 + bl over every slab, kSlabChunk
  // independent loads in flight at a time, in fixed slab order.
  const int bl = tid / kColTile;
  for (int b0 = 0; b0 < p.batch; b0 += kRowGroups) {
    const int b = b0 + bl;
    float v = 0.f;
    if (b < p.batch) {
      const float z = sum_slabs(p.z_part, b, gcol, p.batch, p.mlp, slabs);
      v = gelu_erf(z + p.b1[gcol]) * p.w2[gcol];
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

  // ---- last column tile: q, gate, counters, condition ----
  __syncthreads();
  if (tid == 0) {
    s_last = ticket_arrive(&p.tickets[tiles]) == (unsigned)(tiles - 1);
    s_count = 0u;
  }
  __syncthreads();
  if (!s_last) return;
  for (int b = tid; b < p.batch; b += kRThreads) {
    float q = 0.f;
    for (int t = 0; t < tiles; ++t) q += __ldcg(&p.q_part[(size_t)t * p.batch + b]);
    gate_one(p, b, q + p.b2, &s_count);
  }
  __syncthreads();
  if (tid == 0) {
    publish_gate(p, s_count);
    p.tickets[tiles] = 0u;
  }
}

// ---------------------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------------------
int launch_recall(const float* h_prev, const float* emb, const void* h_local, int h_local_dtype,
                  int batch, int hidden, int mlp, const float* w1, const float* b1,
                  const float* w2, float b2, float theta, float* q_out, int32_t* gate_out,
                  unsigned long long* full_count, unsigned long long graph_cond_handle,
                  void* ws, size_t ws_bytes, void* stream, int pdl) {
  if (batch < 0 || hidden < 1 || mlp < kColTile || mlp % kColTile != 0) return ODA_ERR_INVALID_ARG;
  if (h_local_dtype != ODA_F32 && h_local_dtype != ODA_BF16) return ODA_ERR_INVALID_ARG;
  if (batch == 0) return ODA_OK;
  if (!h_prev || !emb || !h_local || !w1 || !b1 || !w2 || !q_out || !gate_out || !ws)
    return ODA_ERR_INVALID_ARG;
  for (const void* f : {static_cast<const void*>(h_prev), static_cast<const void*>(emb),
                        static_cast<const void*>(w1), static_cast<const void*>(b1),
                        static_cast<const void*>(w2), static_cast<const void*>(q_out),
                        static_cast<const void*>(gate_out)})
    if (!aligned_or_null(f, 4)) return ODA_ERR_INVALID_ARG;
  if (!aligned_or_null(h_local, h_local_dtype == ODA_BF16 ? 2 : 4) ||
      !aligned_or_null(full_count, 8) || !aligned_or_null(ws, 16))
    return ODA_ERR_INVALID_ARG;
  const RecallWs wl = recall_ws(batch, hidden, mlp);
  if (ws_bytes < wl.total) return ODA_ERR_WORKSPACE_TOO_SMALL;
  RecallParams p;
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
  p.theta = theta;
  p.q_out = q_out;
  p.gate_out = gate_out;
  p.full_count = full_count;
  p.cond = static_cast<cudaGraphConditionalHandle>(graph_cond_handle);
  p.use_cond = graph_cond_handle != 0ull;
  unsigned char* w = static_cast<unsigned char*>(ws);
  p.z_part = reinterpret_cast<float*>(w + wl.z_off);
  p.q_part = reinterpret_cast<float*>(w + wl.q_off);
  p.tickets = reinterpret_cast<unsigned*>(w + wl.ticket_off);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(wl.slabs, wl.tiles);
  cfg.blockDim = dim3(kRThreads);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cuda_status(cudaLaunchKernelEx(&cfg, recall_kernel, p));
}

}  // namespace oda

using namespace oda;

namespace oda {
int recall_ws_tickets(int batch, int hidden, int mlp, size_t* ticket_off, int* tiles) {
  if (batch < 0 || hidden < 1 || mlp < kColTile || mlp % kColTile != 0) return ODA_ERR_INVALID_ARG;
  const RecallWs w = recall_ws(batch, hidden, mlp);
  *ticket_off = w.ticket_off;
  *tiles = w.tiles;
  return ODA_OK;
}
}  // namespace oda

extern "C" int oda_recall_workspace_size(int32_t batch, int32_t hidden, int32_t mlp,
                                         size_t* bytes) {
  if (bytes == nullptr || batch < 0 || hidden < 1 || mlp < kColTile || mlp % kColTile != 0)
    return ODA_ERR_INVALID_ARG;
  *bytes = recall_ws(batch, hidden, mlp).total;
  return ODA_OK;
}

extern "C" int oda_recall_score(const float* h_prev, const float* emb, const void* h_local,
                                int32_t h_local_dtype, int32_t batch, int32_t hidden,
                                int32_t mlp, const float* w1, const float* b1, const float* w2,
                                float b2, float theta, float* q_out, int32_t* gate_out,
                                unsigned long long* full_count,
                                unsigned long long graph_cond_handle, void* ws, size_t ws_bytes,
                                void* stream) {
  return launch_recall(h_prev, emb, h_local, h_local_dtype, batch, hidden, mlp, w1, b1, w2, b2,
                       theta, q_out, gate_out, full_count, graph_cond_handle, ws, ws_bytes,
                       stream, 0);
}

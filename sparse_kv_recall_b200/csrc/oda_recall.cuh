// Pieces shared by the recall head (oda_recall.cu) and its training gradient (oda_train.cu):
// the recall input x = [h_prev; emb; h_local] read row by row, and the split of
// z = W1^T x over 256-row slabs x 64-column tiles of W1 (one CTA each), with the slabs'
// partial sums combined in fixed order.
#pragma once

#include <math.h>

#include "oda_common.cuh"

namespace oda {

constexpr int kRThreads = 256;
constexpr int kColTile = 64;
constexpr int kRowGroups = kRThreads / kColTile;  // 4
constexpr int kRows = 256;                        // rows of W1 per CTA
constexpr int kRowsPerThread = kRows / kRowGroups;
constexpr int kBTile = 8;                         // sequences per pass over the slab
constexpr int kSlabChunk = 24;                    // slab partials in flight per thread

__device__ __forceinline__ float gelu_erf(float z) {
  return 0.5f * z * (1.f + erff(z * 0.70710678118654752f));
}

struct RecallInputs {
  const float* h_prev;   // fp32 [batch][hidden]
  const float* emb;      // fp32 [batch][hidden]
  const void* h_local;   // fp32 or bf16 [batch][hidden]
  int h_local_bf16;
  int hidden;
};

// Row r of sequence b's recall input.
__device__ __forceinline__ float x_at(const RecallInputs& in, int b, int r) {
  const int H = in.hidden;
  if (r < H) return in.h_prev[(size_t)b * H + r];
  if (r < 2 * H) return in.emb[(size_t)b * H + r - H];
  const size_t i = (size_t)b * H + (r - 2 * H);
  if (in.h_local_bf16) return __bfloat162float(static_cast<const __nv_bfloat16*>(in.h_local)[i]);
  return static_cast<const float*>(in.h_local)[i];
}

// This thread's W1 column gcol over its rows rg, rg + 4, ... of the slab starting at row r0,
// all loads issued at once.
__device__ __forceinline__ void load_w1_slab(const float* w1, int mlp, int r0, int nrows,
                                             int gcol, int rg, float (&wv)[kRowsPerThread]) {
#pragma unroll
  for (int i = 0; i < kRowsPerThread; ++i) {
    const int r = rg + i * kRowGroups;
    wv[i] = r < nrows ? __ldg(&w1[(size_t)(r0 + r) * mlp + gcol]) : 0.f;
  }
}

// Partial z of one slab for every sequence: z_part[slab][b][gcol] = sum over the slab's rows
// of x_b[r] W1[r][gcol]. xs / red are the CTA's shared scratch; thread (rg, col) = (tid / 64,
// tid % 64). Ends with a CTA barrier.
__device__ __forceinline__ void slab_partial_z(const RecallInputs& in,
                                               const float (&wv)[kRowsPerThread], int batch,
                                               int mlp, int slab, int r0, int nrows, int gcol,
                                               float (*xs)[kRows], float (*red)[kBTile][kColTile],
                                               float* z_part) {
  const int tid = threadIdx.x;
  const int rg = tid / kColTile, col = tid % kColTile;
  static_assert(kRows == kRThreads, "each thread stages one row of the slab");
  for (int b0 = 0; b0 < batch; b0 += kBTile) {
    const int nb = min(kBTile, batch - b0);
    // thread tid stages row tid of every sequence of the tile, all loads in flight together
    float xv[kBTile];
#pragma unroll
    for (int bb = 0; bb < kBTile; ++bb)
      xv[bb] = (bb < nb && tid < nrows) ? x_at(in, b0 + bb, r0 + tid) : 0.f;
#pragma unroll
    for (int bb = 0; bb < kBTile; ++bb) xs[bb][tid] = xv[bb];
    __syncthreads();
    // only the nb sequences present (a batch of one does 1/8 of the FMAs of a full tile)
#pragma unroll
    for (int bb = 0; bb < kBTile; ++bb) {
      if (bb < nb) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i)
          acc = fmaf(xs[bb][rg + i * kRowGroups], wv[i], acc);
        red[rg][bb][col] = acc;
      }
    }
    __syncthreads();
    if (rg == 0) {
      for (int bb = 0; bb < nb; ++bb) {
        const float z = red[0][bb][col] + red[1][bb][col] + red[2][bb][col] + red[3][bb][col];
        z_part[((size_t)slab * batch + b0 + bb) * mlp + gcol] = z;
      }
    }
    __syncthreads();
  }
}

// z of (sequence b, column gcol) summed over every slab in fixed order, kSlabChunk loads in
// flight at a time.
__device__ __forceinline__ float sum_slabs(const float* z_part, int b, int gcol, int batch,
                                           int mlp, int slabs) {
  const float* zp = z_part + (size_t)b * mlp + gcol;
  const size_t sstride = (size_t)batch * mlp;
  float z = 0.f;
  for (int s0 = 0; s0 < slabs; s0 += kSlabChunk) {
    // every load unconditional (a clamped slab index past the end), so all of them issue
    // back to back; the out-of-range ones are dropped from the sum
    float part[kSlabChunk];
#pragma unroll
    for (int u = 0; u < kSlabChunk; ++u)
      part[u] = __ldcg(zp + (size_t)min(s0 + u, slabs - 1) * sstride);
#pragma unroll
    for (int u = 0; u < kSlabChunk; ++u) z += (s0 + u < slabs) ? part[u] : 0.f;
  }
  return z;
}

}  // namespace oda

// Library-internal launch paths shared between translation units (not part of the C ABI).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "oda.h"

namespace oda {

// Remember the most recent CUDA error seen by this thread (reported by oda_last_cuda_error).
void note_cuda_error(int err);

// True when p is null or a multiple of `bytes` (a power of two): every pointer a kernel
// reads or writes as a typed, vector or atomic access is checked on the host with this.
inline bool aligned_or_null(const void* p, size_t bytes) {
  return (reinterpret_cast<uintptr_t>(p) & (bytes - 1)) == 0;
}

// Attribute setup for every decode kernel instantiation on the current device; call before
// stream capture so that nothing but launches is recorded.
int prepare_decode_kernels();

// Decode launch with optional programmatic dependent launch: pdl = 1 lets the kernel start
// while the previous kernel of the stream finishes; wait_first = 1 makes it wait for that
// kernel before reading anything (needed when the previous kernel writes the gate).
int launch_decode(const oda_kv* kv, const oda_visibility& vis, const void* q, int hq,
                  float scale, const void* k_new, const void* v_new, void* out, int out_dtype,
                  float* lse, void* ws, size_t ws_bytes, void* stream, int pdl, int wait_first);

// A visibility rule with every field zero but `mode` (and window = 1).
oda_visibility visibility(int mode);

// Host checks of a visibility rule against the cache it is applied to.
int check_visibility(const oda_kv* kv, const oda_visibility* v);

// oda_kv checks shared by every entry point (ODA_OK or an ODA_ERR_* code).
int check_kv(const oda_kv* kv);

// Decode workspace size and the offset of its merge tickets on the current device.
int decode_ws_layout(int batch, int hkv, int hq, size_t* total, size_t* ticket_off);

// Recall head launch; pdl = 1 lets the part of W1 that reads h_prev and emb run while the
// previous kernel (the last Local layer, which writes h_local) finishes.
int launch_recall(const float* h_prev, const float* emb, const void* h_local, int h_local_dtype,
                  int batch, int hidden, int mlp, const float* w1, const float* b1,
                  const float* w2, float b2, float theta, float* q_out, int32_t* gate_out,
                  unsigned long long* full_count, unsigned long long graph_cond_handle,
                  void* ws, size_t ws_bytes, void* stream, int pdl);

// Random gate schedule (gate = u < rho), counters and graph condition as the recall head.
int launch_gate_schedule(const float* u, int batch, float rho, int32_t* gate_out,
                         unsigned long long* full_count, unsigned long long graph_cond_handle,
                         void* stream);

}  // namespace oda

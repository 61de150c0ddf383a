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

// Test hooks (oda_debug_set_wait_limit / oda_debug_set_stall): the limit every bounded
// device wait of later launches uses, and which wait, if any, later launches make run out.
unsigned long long test_wait_ns();
int test_stall();
int test_local_shape();  // -1: the persistent Local kernel picks its shape

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

// Decode workspace size and the offset of the persistent step kernels' counters (256 bytes:
// the Local kernel's four words, then the Full kernel's four).
int decode_ws_chain_offset(int batch, int hkv, int hq, size_t* total, size_t* chain_off);

// Recall workspace: offset of its tickets and the number of column tiles (the fused recall
// head of the persistent Local kernel uses its partial area and ticket [tiles]).
int recall_ws_tickets(int batch, int hidden, int mlp, size_t* ticket_off, int* tiles);

// Persistent step kernels (oda_chain.cu). prepare_chain_kernels: once per device, before any
// stream capture. launch_local_chain: Local at every layer with the commit, then (phases
// holding ODA_PHASE_RECALL) the gate -- the fused recall head or the random schedule --
// setting the graph condition when cond != 0; ODA_ERR_NOT_IMPLEMENTED when the step's shape
// does not fit the kernel (the caller then launches per layer). launch_full_chain: gated
// Full at every layer with the gated commit, returning at once when no sequence is gated.
struct LocalChainPlan {
  int usable = 0;      // the persistent Local kernel serves this step
  int gate_fused = 0;  // ... with the gate (recall head or random schedule) inside it
  int clusters = 0;
  int shape = 0;       // index of the (CTAs per cluster, warps per CTA) shape
  size_t smem = 0;
};
int prepare_chain_kernels();
// Outside stream capture: whether (and how) the persistent Local kernel serves a step.
int plan_local_chain(const oda_step_desc* d, int phases, LocalChainPlan* plan);
int launch_local_chain(const oda_step_desc* d, const LocalChainPlan& plan, int phases,
                       unsigned long long cond, void* stream);
int launch_full_chain(const oda_step_desc* d, void* stream);
// Clusters of the persistent Local kernel the current device holds at once for a group size,
// batch and recall width (fused head), and whether its launches are cooperative.
int step_kernel_limits(int G, int batch, int mlp, int* clusters, int* cooperative);

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

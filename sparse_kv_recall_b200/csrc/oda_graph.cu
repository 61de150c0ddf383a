// Step runtime: a whole ODA decode step as one CUDA graph ([ODA] 개발자 관점: Local, the FP32
// recall head and the conditional Full recompute run in one GPU execution stream, e.g. CUDA
// Graphs, so that routing needs no host synchronisation).
//
// Top-level graph:  [ev0] Local+commit x L  [ev1] recall  [ev2] IF(any gate) [ev3]
// (with the random gate source the recall head is replaced by the gate schedule kernel)
// IF body:          Full+gated commit for every layer
// A layer outside the Local restriction (hybrid backbones, [ODA] 개발자 관점: the runtime
// restricts only some layers to Local) attends its whole history in the Local pass as well.
// The recall kernel sets the IF node's condition from the device on every step (1 iff any
// sequence is gated), so a step whose sequences are all Local skips the body entirely, and
// a step with some gated sequences runs Full kernels that skip the ungated ones on-device.
#include <stdlib.h>

#include <new>

#include "oda_common.cuh"
#include "oda_internal.h"

struct oda_step_graph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  cudaStream_t cap = nullptr;
  cudaStream_t cap_body = nullptr;
  cudaEvent_t placeholder[4] = {nullptr, nullptr, nullptr, nullptr};
  cudaGraphNode_t ev_node[4] = {nullptr, nullptr, nullptr, nullptr};
  bool timing = false;
  int timing_mode = 0;          // desc->timing_events: 1 every phase boundary, 2 see oda.h
  int launches[3] = {0, 0, 0};  // kernels per step: Local, gate, Full
  oda::LocalChainPlan lplan;    // the persistent Local kernel's plan (decided before capture)
};

namespace {

void release(oda_step_graph* g) {
  if (g == nullptr) return;
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  for (auto& e : g->placeholder)
    if (e) cudaEventDestroy(e);
  if (g->cap) cudaStreamDestroy(g->cap);
  if (g->cap_body) cudaStreamDestroy(g->cap_body);
  delete g;
}

// Record a timing event as a graph node and remember the node.
int record_event_node(oda_step_graph* g, int i) {
  if (cudaEventRecordWithFlags(g->placeholder[i], g->cap, cudaEventRecordExternal) != cudaSuccess)
    return ODA_ERR_CUDA;
  cudaStreamCaptureStatus st;
  const cudaGraphNode_t* deps = nullptr;
  size_t n = 0;
  if (cudaStreamGetCaptureInfo(g->cap, &st, nullptr, nullptr, &deps, &n) != cudaSuccess || n != 1)
    return ODA_ERR_CUDA;
  g->ev_node[i] = deps[0];
  return ODA_OK;
}

int layer_sink(const oda_step_desc* d, int l) { return d->sinks ? d->sinks[l] : d->sink; }
int layer_window(const oda_step_desc* d, int l) { return d->windows ? d->windows[l] : d->window; }

int capture_step(const oda_step_desc* d, oda_step_graph* g, cudaGraphConditionalHandle cond) {
  const int L = d->num_layers;
  const int phases = d->phases ? d->phases : (ODA_PHASE_LOCAL | ODA_PHASE_RECALL | ODA_PHASE_FULL);
  const bool persistent = d->step_kernels != ODA_STEP_PER_LAYER;  // (Full; Local: the plan)
  const unsigned long long cond_u64 = d->use_conditional ? (unsigned long long)cond : 0ull;
  int rc;
  if (g->timing && (rc = record_event_node(g, 0)) != ODA_OK) return rc;

  // Local (and, fused into the same launch, the gate) as one persistent kernel when the step's
  // shape fits it; otherwise one launch per layer and a separate gate kernel.
  bool gate_done = false;
  bool local_done = !(phases & ODA_PHASE_LOCAL);
  if (!local_done && persistent && g->lplan.usable) {
    // with the gate fused if its shape allows, else Local alone and the gate kernel after it
    rc = oda::launch_local_chain(d, g->lplan, phases, cond_u64, g->cap);
    if (rc != ODA_OK) return rc;
    local_done = true;
    gate_done = g->lplan.gate_fused && (phases & ODA_PHASE_RECALL) != 0;
    g->launches[0] = 1;
  }
  // Programmatic dependent launch between consecutive kernels: each Local layer after the
  // first, the recall head after the last Local layer and each Full layer after the first
  // may start while its predecessor finishes (see the kernels for what they do before
  // waiting). Kernels next to a timing-event node keep ordinary launches.
  for (int l = 0; l < L && !local_done; ++l) {
    const bool restricted = d->local_layers == nullptr || d->local_layers[l] != 0;
    oda_visibility vis = oda::visibility(restricted ? ODA_MODE_LOCAL : ODA_MODE_FULL);
    vis.sink = layer_sink(d, l);
    vis.window = layer_window(d, l);
    rc = oda::launch_decode(&d->layers[l], vis, d->q_local[l], d->num_q_heads, d->scale,
                            d->k_local[l], d->v_local[l], d->out[l], ODA_F32,
                            d->lse ? d->lse[l] : nullptr, d->decode_ws, d->decode_ws_bytes,
                            g->cap, l > 0 ? 1 : 0, 0);
    if (rc != ODA_OK) return rc;
    ++g->launches[0];
  }
  const bool lean_events = g->timing_mode == 2 && (phases & ODA_PHASE_RECALL);
  if (g->timing && !lean_events && (rc = record_event_node(g, 1)) != ODA_OK) return rc;
  if (!(phases & ODA_PHASE_RECALL)) {
    if (g->timing)
      for (int i = 2; i < 4; ++i)
        if ((rc = record_event_node(g, i)) != ODA_OK) return rc;
    return ODA_OK;
  }
  if (!gate_done) {
    if (d->gate_source == ODA_GATE_RANDOM) {
      rc = oda::launch_gate_schedule(d->gate_u, d->layers[0].batch, d->rho, d->gate_out,
                                     d->full_count, cond_u64, g->cap);
    } else {
      const int hidden = d->num_q_heads * d->layers[0].head_dim;
      rc = oda::launch_recall(d->h_prev, d->emb, d->out[L - 1], ODA_F32, d->layers[0].batch,
                              hidden, d->mlp, d->w1, d->b1, d->w2, d->b2, d->theta, d->q_out,
                              d->gate_out, d->full_count, cond_u64, d->recall_ws,
                              d->recall_ws_bytes, g->cap, g->timing && !lean_events ? 0 : 1);
    }
    if (rc != ODA_OK) return rc;
    g->launches[1] = 1;
  }
  if (lean_events && (rc = record_event_node(g, 1)) != ODA_OK) return rc;
  if (g->timing && (rc = record_event_node(g, 2)) != ODA_OK) return rc;

  if (!(phases & ODA_PHASE_FULL)) {
    if (g->timing && (rc = record_event_node(g, 3)) != ODA_OK) return rc;
    return ODA_OK;
  }
  cudaStream_t full_stream = g->cap;
  cudaGraph_t body = nullptr;
  if (d->use_conditional) {
    cudaStreamCaptureStatus st;
    cudaGraph_t capg = nullptr;
    const cudaGraphNode_t* deps = nullptr;
    size_t n = 0;
    if (cudaStreamGetCaptureInfo(g->cap, &st, nullptr, &capg, &deps, &n) != cudaSuccess)
      return ODA_ERR_CUDA;
    cudaGraphNodeParams cp = {};
    cp.type = cudaGraphNodeTypeConditional;
    cp.conditional.handle = cond;
    cp.conditional.type = cudaGraphCondTypeIf;
    cp.conditional.size = 1;
    cudaGraphNode_t cnode;
    if (cudaGraphAddNode(&cnode, capg, deps, n, &cp) != cudaSuccess) return ODA_ERR_CUDA;
    body = cp.conditional.phGraph_out[0];
    if (cudaStreamUpdateCaptureDependencies(g->cap, &cnode, 1, cudaStreamSetCaptureDependencies) !=
        cudaSuccess)
      return ODA_ERR_CUDA;
    if (cudaStreamBeginCaptureToGraph(g->cap_body, body, nullptr, nullptr, 0,
                                      cudaStreamCaptureModeThreadLocal) != cudaSuccess)
      return ODA_ERR_CUDA;
    full_stream = g->cap_body;
  }
  // Full at every layer: one persistent launch that returns at once when no sequence is gated
  // (the device-side early exit), or one launch per layer that skips ungated sequences.
  rc = persistent ? oda::launch_full_chain(d, full_stream) : ODA_ERR_NOT_IMPLEMENTED;
  if (rc == ODA_OK) g->launches[2] = 1;
  if (rc == ODA_ERR_NOT_IMPLEMENTED) {
    rc = ODA_OK;
    for (int l = 0; l < L; ++l) {
      // The first Full kernel reads the gate the gate kernel just wrote: inside the IF body it
      // is the body's first node; without the IF node it waits for the gate kernel at once.
      int pdl = 1, wait_first = 0;
      if (l == 0) {
        pdl = (!d->use_conditional && !g->timing && !gate_done) ? 1 : 0;
        wait_first = 1;
      }
      oda_visibility vis = oda::visibility(ODA_MODE_FULL);
      vis.gate = d->gate_out;
      rc = oda::launch_decode(&d->layers[l], vis, d->q_full[l], d->num_q_heads, d->scale,
                              d->k_full[l], d->v_full[l], d->out[l], ODA_F32,
                              d->lse ? d->lse[l] : nullptr,
                              d->decode_ws, d->decode_ws_bytes, full_stream, pdl, wait_first);
      if (rc != ODA_OK) break;
      ++g->launches[2];
    }
  }
  if (d->use_conditional) {
    cudaGraph_t done = nullptr;
    const cudaError_t e = cudaStreamEndCapture(g->cap_body, &done);
    if (rc != ODA_OK) return rc;
    if (e != cudaSuccess) return ODA_ERR_CUDA;
  }
  if (rc != ODA_OK) return rc;
  if (g->timing && (rc = record_event_node(g, 3)) != ODA_OK) return rc;
  return ODA_OK;
}

int check_desc(const oda_step_desc* d) {
  if (d == nullptr || d->num_layers < 1 || d->layers == nullptr) return ODA_ERR_INVALID_ARG;
  if (!d->q_local || !d->k_local || !d->v_local || !d->q_full || !d->k_full || !d->v_full ||
      !d->out)
    return ODA_ERR_INVALID_ARG;
  const oda_kv& k0 = d->layers[0];
  for (int l = 1; l < d->num_layers; ++l) {
    const oda_kv& k = d->layers[l];
    if (k.batch != k0.batch || k.num_kv_heads != k0.num_kv_heads || k.seq_lens != k0.seq_lens ||
        k.block_table != k0.block_table || k.max_blocks_per_seq != k0.max_blocks_per_seq)
      return ODA_ERR_INVALID_ARG;
  }
  if (k0.batch < 1) return ODA_ERR_INVALID_ARG;
  for (int l = 0; l < d->num_layers; ++l)
    if (layer_sink(d, l) < 0 || layer_window(d, l) < 1) return ODA_ERR_INVALID_ARG;
  if (d->gate_source != ODA_GATE_RECALL && d->gate_source != ODA_GATE_RANDOM)
    return ODA_ERR_INVALID_ARG;
  if (d->gate_source == ODA_GATE_RANDOM &&
      (d->gate_u == nullptr || !(d->rho >= 0.f && d->rho <= 1.f)))
    return ODA_ERR_INVALID_ARG;
  if (d->step_kernels != ODA_STEP_FULL_PERSISTENT && d->step_kernels != ODA_STEP_PER_LAYER &&
      d->step_kernels != ODA_STEP_PERSISTENT)
    return ODA_ERR_INVALID_ARG;
  if (d->timing_events < 0 || d->timing_events > 2) return ODA_ERR_INVALID_ARG;
  return ODA_OK;
}

}  // namespace

extern "C" int oda_step_graph_create(const oda_step_desc* desc, void* stream,
                                     oda_step_graph** graph) {
  (void)stream;
  if (graph == nullptr) return ODA_ERR_INVALID_ARG;
  *graph = nullptr;
  int rc = check_desc(desc);
  if (rc != ODA_OK) return rc;
  if ((rc = oda::prepare_decode_kernels()) != ODA_OK) return rc;
  if ((rc = oda::prepare_chain_kernels()) != ODA_OK) return rc;
  oda_step_graph* g = new (std::nothrow) oda_step_graph();
  if (g == nullptr) return ODA_ERR_CUDA;
  g->timing = desc->timing_events != 0;
  g->timing_mode = desc->timing_events;
  if (cudaStreamCreateWithFlags(&g->cap, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&g->cap_body, cudaStreamNonBlocking) != cudaSuccess ||
      cudaGraphCreate(&g->graph, 0) != cudaSuccess) {
    release(g);
    return ODA_ERR_CUDA;
  }
  if (g->timing)
    for (auto& e : g->placeholder)
      if (cudaEventCreate(&e) != cudaSuccess) {
        release(g);
        return ODA_ERR_CUDA;
      }
  cudaGraphConditionalHandle cond = 0;
  const int phases = desc->phases ? desc->phases : ODA_PHASE_FULL;
  if (desc->use_conditional && (phases & ODA_PHASE_FULL) &&
      cudaGraphConditionalHandleCreate(&cond, g->graph, 0, 0) !=
          cudaSuccess) {
    release(g);
    return ODA_ERR_CUDA;
  }
  const int all = ODA_PHASE_LOCAL | ODA_PHASE_RECALL | ODA_PHASE_FULL;
  if ((rc = oda::plan_local_chain(desc, desc->phases ? desc->phases : all, &g->lplan)) != ODA_OK) {
    release(g);
    return rc;
  }
  if (cudaStreamBeginCaptureToGraph(g->cap, g->graph, nullptr, nullptr, 0,
                                    cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    release(g);
    return ODA_ERR_CUDA;
  }
  rc = capture_step(desc, g, cond);
  cudaGraph_t captured = nullptr;
  const cudaError_t e = cudaStreamEndCapture(g->cap, &captured);
  if (rc == ODA_OK && e != cudaSuccess) rc = ODA_ERR_CUDA;
  if (rc == ODA_OK && cudaGraphInstantiate(&g->exec, g->graph, 0) != cudaSuccess) rc = ODA_ERR_CUDA;
  if (rc != ODA_OK) {
    oda::note_cuda_error(cudaGetLastError());
    release(g);
    return rc;
  }
  *graph = g;
  return ODA_OK;
}

extern "C" int oda_step_graph_launch(oda_step_graph* graph, void* stream) {
  if (graph == nullptr || graph->exec == nullptr) return ODA_ERR_INVALID_ARG;
  return oda::cuda_status(cudaGraphLaunch(graph->exec, static_cast<cudaStream_t>(stream)));
}

extern "C" int oda_step_graph_set_events(oda_step_graph* graph, void* ev_start, void* ev_local,
                                         void* ev_recall, void* ev_end) {
  if (graph == nullptr || !graph->timing) return ODA_ERR_INVALID_ARG;
  void* evs[4] = {ev_start, ev_local, ev_recall, ev_end};
  for (int i = 0; i < 4; ++i) {
    if (evs[i] == nullptr) return ODA_ERR_INVALID_ARG;
    if (cudaGraphExecEventRecordNodeSetEvent(graph->exec, graph->ev_node[i],
                                             static_cast<cudaEvent_t>(evs[i])) != cudaSuccess)
      return ODA_ERR_CUDA;
  }
  return ODA_OK;
}

extern "C" int oda_step_graph_kernels(const oda_step_graph* graph, int32_t* local_launches,
                                      int32_t* gate_launches, int32_t* full_launches) {
  if (graph == nullptr || local_launches == nullptr || gate_launches == nullptr ||
      full_launches == nullptr)
    return ODA_ERR_INVALID_ARG;
  *local_launches = graph->launches[0];
  *gate_launches = graph->launches[1];
  *full_launches = graph->launches[2];
  return ODA_OK;
}

extern "C" void oda_step_graph_destroy(oda_step_graph* graph) { release(graph); }

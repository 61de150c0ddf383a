// Persistent step kernels: the Local pass over every layer, with the recall head fused at its
// end, and the Full recompute over every layer, each as ONE launch ([ODA] 접근 방법: each
// decode step attends Local at every layer, scores the step from the final Local hidden,
// and only then, iff q_t > theta, recomputes every layer with Full; 개발자 관점: Local, the
// FP32 recall head and the conditional Full pass run on the GPU with no routing sync).
//
// Why one launch per phase. Each layer's query depends on the previous layer's output, so a
// step is a chain of dependent layers. At batch 1 a Local layer streams only 8.4 MB, far too
// little to hide a kernel boundary (grid completion, then the next grid's wait), which cost
// about 1.5 us of a 6 us layer; Full at 128K streams 0.54 GB per layer and loses little there.
//
// local_chain_kernel: one thread-block cluster of 16 CTAs x 9 warps per (sequence, KV head),
// two CTAs per SM, resident for the whole step. Each warp owns one page of its (b, g)'s Local
// list at every layer; as soon as it has attended layer l's page it requests layer l + 1's
// into the same stage (a history page that no layer of this step writes), so the copy runs
// while the CTAs merge and wait. The CTAs of a cluster merge their partials in rank 0's
// shared memory; rank 0
// writes the layer's output and adds one to a launch-wide layer count with release
// semantics; every CTA waits (acquire, bounded) for the count of layer l - 1 before it reads
// layer l's query and K/V row. After the last layer the CTAs evaluate the recall head:
// W1's h_prev / emb rows were applied at the start (their inputs are known then), the h^L
// rows (requested into the page buffer once the last layer's pages are consumed) once the
// last layer's count is complete; the
// partial z vectors are summed in each cluster's rank 0, then across clusters by the last to
// arrive on a ticket, which applies b1, GELU, w2, b2, the gate, the counters and the graph
// condition. Every sum runs in a fixed order, so results are bitwise reproducible.
//
// full_chain_kernel: the split decode pass (oda_decode.cuh) of every layer in one launch of
// two CTAs per SM; a grid-wide count between layers takes the place of the kernel boundary
// (each CTA requests its first pages of layer l before it waits for layer l - 1). When the
// gate selects no sequence every CTA returns at once: the device-side early exit that makes
// a graph conditional node unnecessary.
//
// Both kernels run as cooperative launches (every CTA resident at once), every wait gives up
// after a limit (ODA_DEV_TIMEOUT, then a launch-wide abort word stops the others), and each
// kernel's last CTA to finish resets its counters, so the workspace is reusable in stream
// order.
#include <math.h>

#include "oda_decode.cuh"
#include "oda_recall.cuh"

namespace oda {

constexpr int kMaxChainLayers = 40;
constexpr int kChainMaxBatch = 8;     // sequences per launch of the fused recall head
constexpr int kChainMaxClusters = 16; // clusters of the Local kernel with the fused recall head
constexpr int kChainXs = 1024;        // [h_prev; emb] recall inputs a CTA stages (all sequences)
constexpr int kChainMaxHl = 64;       // h^L rows per CTA: 128 G / C, rounded up
// Shapes of the Local kernel: C CTAs per cluster (one cluster per (sequence, KV head)) of W
// warps, one page per warp, so C x W pages per (sequence, KV head) at most. The 16 x 9 shape
// runs two CTAs per SM; the shorter clusters run one CTA per SM (their shared memory is
// padded to make sure), so that no cluster's page steps and merges share an SM's issue slots.
// The 8 x 18 shape (576 threads, so at most 112 registers a thread) serves one and two query
// heads per KV head only.

// Floats of the in-CTA merge scratch: the warps' softmax states of G heads (max, sum, 128
// accumulators each).
template <int W>
__host__ __device__ constexpr int chain_scratch_floats(int G) {
  return G == 1 ? cluster_scratch_floats<1, false, W>()
                : (G == 2 ? cluster_scratch_floats<2, true, W>()
                          : cluster_scratch_floats<4, true, W>());
}

// Launch-wide counters in the decode workspace (see ws_layout): [0] layer / barrier count,
// [1] CTAs that have finished, [2] abort word.
enum { kCtrCount = 0, kCtrExit = 1, kCtrAbort = 2, kCtrWords = 4 };

struct ChainLayer {
  const __nv_bfloat16* k_cache;
  const __nv_bfloat16* v_cache;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_new;  // nullable: commit at slot t
  const __nv_bfloat16* v_new;
  float* out;                  // fp32 [batch][hq][128]
  float* lse;                  // nullable
  int sink, window;            // Local rule of this layer
};

struct LocalChainParams {
  ChainLayer layer[kMaxChainLayers];
  int L, batch, hkv, hq;
  const int32_t* seq_lens;
  const int32_t* block_table;
  int max_blocks, num_blocks;
  float scale_log2;
  int* status;
  unsigned long long* stats;
  unsigned* ctr;               // kCtrWords launch-wide counters
  unsigned long long wait_ns;
  int test_stall;              // 1: cluster 0 withholds its layer-0 count (test hook)
  // fused gate: 0 none (Local only), 1 recall head, 2 random schedule
  int gate_mode;
  const float* h_prev;         // fp32 [batch][hidden]
  const float* emb;
  const float* w1;             // fp32 [3 hidden][mlp]
  const float* b1;
  const float* w2;
  float b2, theta;
  int hidden, mlp;
  int rows_pre, rows_hl;       // W1 rows per CTA of the [h_prev; emb] and h^L sections
  const float* gate_u;         // random schedule: fp32 [batch]
  float rho;
  float* q_out;
  int32_t* gate_out;
  unsigned long long* full_count;
  cudaGraphConditionalHandle cond;
  int use_cond;
  float* z_clusters;           // [clusters][batch][mlp]
  unsigned* recall_ticket;
};

struct FullChainParams {
  ChainLayer layer[kMaxChainLayers];  // sink / window unused
  DecodeParams base;                  // plan (Full, gated), shapes, workspace, hooks
  int L;
  unsigned* ctr;
  int test_stall;                     // 1: CTA 0 withholds its layer-0 arrival (test hook)
};

// W1 is read once per step by the fused recall head; keep it in L2 across steps.
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ float ld_keep(const float* p, uint64_t pol) {
  float v;
  asm volatile("ld.global.nc.L2::cache_hint.f32 %0, [%1], %2;" : "=f"(v) : "l"(p), "l"(pol));
  return v;
}

// Thread 0 waits for the launch-wide count to reach `target`; on a timeout it reports
// ODA_DEV_TIMEOUT and raises the abort word. Returns the answer to every thread of the CTA.
__device__ __forceinline__ bool cta_wait_count(unsigned* ctr, unsigned target,
                                               unsigned long long limit_ns, int* status,
                                               int* s_flag) {
  if (threadIdx.x == 0) {
    const int ok = counter_wait(&ctr[kCtrCount], target, &ctr[kCtrAbort], limit_ns);
    if (!ok && counter_acquire_load(&ctr[kCtrAbort]) == 0u) {
      report(status, ODA_DEV_TIMEOUT);
      atomicExch(&ctr[kCtrAbort], 1u);
    }
    *s_flag = ok;
  }
  __syncthreads();
  return *s_flag != 0;
}

// Every CTA calls this last. The CTA that finishes last resets the launch's counters for the
// next launch (its arrival acquired every other CTA's last use of them); if the launch was
// abandoned it also zeroes the n merge tickets an interrupted merge may have left behind.
__device__ __forceinline__ void cta_exit(unsigned* ctr, unsigned* tickets, int n, int* s_flag) {
  __syncthreads();
  if (threadIdx.x == 0) *s_flag = ticket_arrive(&ctr[kCtrExit]) == gridDim.x - 1;
  __syncthreads();
  if (*s_flag) {
    if (__ldcg(&ctr[kCtrAbort]) != 0u)
      for (int i = threadIdx.x; i < n; i += blockDim.x) tickets[i] = 0u;
    if (threadIdx.x == 0) {
      ctr[kCtrCount] = 0u;
      ctr[kCtrAbort] = 0u;
      ctr[kCtrExit] = 0u;
    }
  }
}

// ---------------------------------------------------------------------------------------
// Local over every layer + recall head.
//
// Handshakes inside a cluster, per layer: every CTA ships its partial into rank 0's inbox
// (one bulk copy completing on rank 0's `ibar`); rank 0 waits for all of them, arms `ibar`
// for the next layer, merges, then arrives on every CTA's `obar`: the inbox may be refilled
// and each sender's `mypart` written again. A CTA waits on its `obar` before it writes
// `mypart` for the next layer, so no CTA runs more than one layer ahead of its rank 0, and
// every copy into the inbox comes after rank 0 armed the phase it completes.
//
// Error path. A CTA whose wait runs out (or that sees the abort word) turns "dead" for the
// rest of the launch -- the same answer in all its threads -- but still steps through every
// remaining layer's cluster phase with an empty partial and no global write, so the CTAs of
// a cluster always arrive on the same barrier phases and none leaves while another may still
// store into its shared memory. A dead CTA requests no further copies and waits (bounded) for
// those already requested, including a page whose wait ran out.
// ---------------------------------------------------------------------------------------
template <int G, int C, int W>
__global__ void __launch_bounds__(W * 32, (C == 16 && G != 4) ? 2 : 1)
    local_chain_kernel(const LocalChainParams p) {
  constexpr int kThreadsC = W * 32;
  constexpr int kBufBytes = W * kStageBytes;
  constexpr bool kMma = MmaScores<G>::value;  // page scores on the tensor cores (G = 2, 4)
  constexpr int VPL = ClusterStates<G, kMma, W>::VPL;
  constexpr int kPs = 18 * G;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* buf = smem;                                            // [warp][kStageBytes]
  float* scratch = reinterpret_cast<float*>(smem + kBufBytes);          // in-CTA merge
  uint64_t* bars = reinterpret_cast<uint64_t*>(scratch + chain_scratch_floats<W>(G));
  uint64_t* wbar = bars + W;                                            // W1 rows
  uint64_t* ibar = wbar + 1;                                            // rank 0: inbox filled
  uint64_t* obar = ibar + 1;                                            // rank 0 merged: mypart free
  float* pscratch = reinterpret_cast<float*>(obar + 1);                 // [warp][kPs]
  float* inbox = align16(pscratch + W * kPs);                           // rank 0: [C][stride]
  __shared__ float xs[kChainXs];      // [h_prev; emb] inputs of this CTA's W1 rows, per sequence
  __shared__ __align__(16) float xh[kChainMaxHl];  // h^L inputs of this CTA's W1 rows
  __shared__ int s_flag;
  __shared__ unsigned long long s_rows, s_pages;
  __shared__ float s_red[W][kChainMaxBatch];
  __shared__ unsigned s_count;

  if (p.L == 0) return;  // nothing to do (also the shape of the launch probe)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int li = lane & 15;
  const unsigned rank = cluster_ctarank();
  const int cl = blockIdx.x / C;
  const int ncl = gridDim.x / C;
  const int b = cl / p.hkv, g = cl % p.hkv;
  const int B = p.batch;
  // inbox slots: a CTA partial or, with the fused recall head, the batch's partial z (B x mlp,
  // a multiple of 64 floats); both multiples of 4 floats
  const int stride = max(ClusterPart<G>::value, p.gate_mode == 1 ? B * p.mlp : 0);
  float* mypart = inbox + C * stride;  // this CTA's partial, shipped to rank 0's inbox
  const uint32_t slot_bytes = (uint32_t)stride * sizeof(float);
  const int j = (int)rank * W + warp;  // this warp's entry of the page list
  const size_t head_off = (size_t)g * (kPage * kHeadDim);
  const size_t page_stride = (size_t)p.hkv * kPage * kHeadDim;
  unsigned char* st = buf + warp * kStageBytes;

  PlanArgs pa;
  pa.seq_lens = p.seq_lens;
  pa.block_table = p.block_table;
  pa.max_blocks = p.max_blocks;
  pa.num_blocks = p.num_blocks;
  pa.mode = ODA_MODE_LOCAL;
  pa.sink = 0;
  pa.window = 1;
  pa.gate = nullptr;
  pa.keep_blocks = nullptr;
  pa.keep_counts = nullptr;
  pa.max_keep = 0;
  pa.da_modes = nullptr;
  pa.da_offsets = nullptr;
  pa.da_focus_len = pa.da_recent = pa.da_local_len = 0;
  pa.pos_lo = pa.pos_hi = 0;
  auto plan_of = [&](int l) {
    PlanArgs a = pa;
    a.sink = p.layer[l].sink;
    a.window = p.layer[l].window;
    return make_plan(a, b);
  };

  if (tid == 0) {
    s_rows = 0;
    s_pages = 0;
  }
  if (lane == 0) {
    mbar_init(&bars[warp], 1);
    if (warp == 0) {
      mbar_init(wbar, 1);
      mbar_init(ibar, 1);
      mbar_init(obar, 1);
    }
    fence_barrier_init();
  }
  // rank 0's inbox barrier expects every CTA's partial of layer 0
  if (rank == 0 && tid == 0) mbar_arrive_expect_tx(ibar, (uint32_t)C * slot_bytes);
  __syncthreads();
  // every CTA's barriers are initialised before any copy of the cluster may signal them
  cluster_arrive();
  cluster_wait();

  // The recall head's rows of W1 for this CTA. The h^L section: this cluster's heads g G ..
  // g G + G - 1 of sequence b are 128 G rows, rows_hl of them per CTA in rank order, so the
  // inputs of those rows are exactly what this cluster's rank 0 computes at the last layer.
  // The [h_prev; emb] section (inputs known at the start) is spread over the CTAs other than
  // rank 0, which apply it after the first layer, while rank 0 merges.
  const int hl0 = (g * G) * kHeadDim + (int)rank * p.rows_hl;  // within sequence b's h^L
  const int nhl = max(0, min(p.rows_hl, G * kHeadDim - (int)rank * p.rows_hl));
  const int nworkers = ncl * (C - 1);
  const int worker = cl * (C - 1) + (int)rank - 1;  // -1 for rank 0
  const int pre0 = rank == 0 ? 0 : min(worker * p.rows_pre, 2 * p.hidden);
  const int npre = rank == 0 ? 0 : max(0, min(p.rows_pre, 2 * p.hidden - pre0));
  (void)nworkers;
  const uint64_t keep = l2_evict_last_policy();
  const uint64_t stream_pol = l2_evict_first_policy();

  // Layer l's plan and this warp's page of it (every lane: they read only the lengths and the
  // page table, which no kernel of the step writes), computed when the page is requested, a
  // layer ahead, so that nothing but the query and the step's K/V row is read after a wait.
  struct WarpPage {
    SeqPlan sp;
    PageRef r;
    bool has;  // the warp attends a page of this layer
  };
  auto page_of = [&](int l) {
    WarpPage w;
    w.sp = plan_of(l);
    w.has = !w.sp.skip && w.sp.err == 0 && j < w.sp.npages;
    w.r.err = 1;
    w.r.lp = 0;
    w.r.pb = 0;
    if (w.has) w.r = page_ref(pa, w.sp, b, j);
    return w;
  };
  // Lane 0 requests the page into this warp's stage. Every warp arms its barrier at every
  // layer (a plain arrive when it has no page), so its phases stay in step with the layers.
  auto issue_page = [&](int l, const WarpPage& w) {
    if (lane != 0) return;
    if (w.has && w.r.err == 0) {
      const size_t src = (size_t)w.r.pb * page_stride + head_off;
      mbar_arrive_expect_tx(&bars[warp], kStageBytes);
      bulk_load(st, p.layer[l].k_cache + src, kPageBytes, &bars[warp], stream_pol);
      bulk_load(st + kPageBytes, p.layer[l].v_cache + src, kPageBytes, &bars[warp], stream_pol);
    } else {
      if (w.has) report(p.status, w.r.err);
      mbar_arrive(&bars[warp]);
    }
  };
  WarpPage cur = page_of(0);
  issue_page(0, cur);
  int issued = 0;          // highest layer whose page copy was requested
  bool w1_issued = false;

  if (rank == 0 && g == 0 && tid == 0 && cur.sp.err != 0) report(p.status, cur.sp.err);

  // The random schedule needs no Local output: decide it at once.
  if (p.gate_mode == 2 && blockIdx.x == 0) {
    if (tid == 0) s_count = 0u;
    __syncthreads();
    for (int bb = tid; bb < B; bb += kThreadsC) {
      const int gate = p.gate_u[bb] < p.rho ? 1 : 0;
      p.gate_out[bb] = gate;
      if (gate) atomicAdd(&s_count, 1u);
    }
    __syncthreads();
    if (tid == 0) {
      if (p.full_count != nullptr && s_count) {
        atomicAdd(&p.full_count[0], (unsigned long long)s_count);
        atomicAdd(&p.full_count[1], 1ull);
      }
      if (p.use_cond) cudaGraphSetConditional(p.cond, s_count ? 1u : 0u);
    }
  }

  // ---- Local, layer by layer ----
  float zpre[kChainMaxBatch];  // this CTA's partial z of the recall head, per sequence
#pragma unroll
  for (int bb = 0; bb < kChainMaxBatch; ++bb) zpre[bb] = 0.f;
  unsigned rows_vis = 0, pages_read = 0;
  bool dead = false;
  int stuck = -1;  // the layer whose page wait (this warp's) ran out
  for (int l = 0; l < p.L; ++l) {
    const ChainLayer& ly = p.layer[l];
    const bool last = l + 1 == p.L;
    if (l > 0 && !dead && !cta_wait_count(p.ctr, (unsigned)(ncl * l), p.wait_ns, p.status, &s_flag))
      dead = true;
    const SeqPlan sp = cur.sp;
    const PageRef r = cur.r;
    const bool has = !dead && cur.has && r.err == 0;
    const bool commit = has && ly.k_new != nullptr && r.lp == sp.t / kPage;
    float m_run[VPL], l_run[VPL];
    f2_t acc[G][4];
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      m_run[u] = -INFINITY;
      l_run[u] = 0.f;
    }
#pragma unroll
    for (int gg = 0; gg < G; ++gg)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) acc[gg][jj] = f2_pack(0.f, 0.f);
    // The layer's query and, for the warp whose page holds slot t, the step's K/V row: both
    // requested together, the only reads after the wait.
    f2_t q2[G][4];
    uint4 qv[4];
    uint4 kvrow = make_uint4(0u, 0u, 0u, 0u);
    if (has) {
      if constexpr (kMma) load_q_mma<G>(ly.q + ((size_t)b * p.hq + g * G) * kHeadDim, lane, qv);
      else load_q_scaled<G>(ly.q, p.hq, b, g, p.scale_log2, li, q2);
      if (commit)
        kvrow = *reinterpret_cast<const uint4*>((lane < 16 ? ly.k_new : ly.v_new) +
                                                ((size_t)b * p.hkv + g) * kHeadDim + 8 * li);
    }
    // this layer's page (requested unless the CTA turned dead a layer ago)
    const bool landed = l > issued ||
        __all_sync(0xffffffffu, mbar_wait(&bars[warp], l & 1u, p.wait_ns));
    if (!landed) {
      stuck = l;  // its copy may still land: waited for again before leaving
    } else if (has) {
      if (commit) {
        // the step's K/V take slot t, in the cache and in this page's copy
        const int row = sp.t % kPage;
        const bool isk = lane < 16;
        *reinterpret_cast<uint4*>(st + (isk ? 0 : kPageBytes) + row * kRowBytes + 16 * li) = kvrow;
        __nv_bfloat16* dst = const_cast<__nv_bfloat16*>(isk ? ly.k_cache : ly.v_cache) +
                             (size_t)r.pb * page_stride + head_off + row * kHeadDim + 8 * li;
        *reinterpret_cast<uint4*>(dst) = kvrow;
        __syncwarp();
      }
      if constexpr (kMma)
        page_step_mma<G>(st, qv, p.scale_log2, m_run, l_run, acc, pscratch + warp * kPs, sp,
                         r.lp, lane, rows_vis);
      else
        page_step<G>(st, q2, m_run, l_run, acc, pscratch + warp * kPs, sp, r.lp, lane, rows_vis);
      ++pages_read;
    }
    fence_proxy_async_smem();  // the commit wrote the stage through the generic proxy
    // Before `mypart` is written again: rank 0 has merged the previous layer (its copy of
    // `mypart` has landed). A page or handshake wait that ran out makes the CTA dead.
    const bool lost =
        __syncthreads_or((lane == 0 && !landed) ||
                         (tid == 0 && l > 0 && !mbar_wait_cluster(obar, (l - 1) & 1u, p.wait_ns)));
    if (lost) {
      if (tid == 0) {
        report(p.status, ODA_DEV_TIMEOUT);
        atomicExch(&p.ctr[kCtrAbort], 1u);
      }
      dead = true;
    }
    cluster_push_partial<G, kMma, W, true>(m_run, l_run, acc, scratch, mypart, stride, rank);
    // (every page of this layer is consumed: the barrier inside the push saw to it)
    fence_proxy_async_smem();  // the partial was written through the generic proxy ...
    __syncthreads();
    if (tid == 0) {            // ... and leaves by one bulk copy into rank 0's inbox slot
      bulk_to_cluster(cluster_addr(inbox + rank * stride, 0), mypart, slot_bytes,
                      cluster_addr(ibar, 0));
    }
    // Off the critical path now (every CTA waits for rank 0 next): the next layer's page into
    // this warp's stage, or, after the last layer, this CTA's W1 rows of the h^L section into
    // the page buffer (one bulk copy).
    if (!dead && !last) {
      // the next layer's plan and page are this layer's when its rule is the same (no read)
      if (p.layer[l + 1].sink != ly.sink || p.layer[l + 1].window != ly.window)
        cur = page_of(l + 1);
      issue_page(l + 1, cur);
      issued = l + 1;
    }
    if (last && !dead && p.gate_mode == 1) {
      if (tid == 0) {
        if (nhl > 0) {
          const uint32_t bytes = (uint32_t)nhl * p.mlp * sizeof(float);
          mbar_arrive_expect_tx(wbar, bytes);
          bulk_load(buf, p.w1 + ((size_t)2 * p.hidden + hl0) * p.mlp, bytes, wbar, keep);
        } else {
          mbar_arrive(wbar);
        }
      }
      w1_issued = true;
    }
    if (rank == 0) {
      // every CTA's partial has landed in this CTA's inbox (a CTA that turned dead still sends
      // one, so the barrier's phases stay in step with the layers)
      if (__syncthreads_or(mbar_wait_cluster(ibar, l & 1u, p.wait_ns) ? 0 : 1)) {
        if (tid == 0) {
          report(p.status, ODA_DEV_TIMEOUT);
          atomicExch(&p.ctr[kCtrAbort], 1u);
        }
        dead = true;
      }
      if (!last && tid == 0) mbar_arrive_expect_tx(ibar, (uint32_t)C * slot_bytes);  // next layer
      // The merge of the C CTA partials, in rank order: one thread per (head, partial)
      // weighs it against the head's maximum, then one thread per (head, dim) sums.
      float* wsm = scratch;                 // [G][C] weights (the CTA merge is done with it)
      float* msm = scratch + C * G;         // [G] maxima
      constexpr int kOut = ClusterPart<G>::kOut;
      if (tid < C * G) {
        const int gg = tid / C, cc = tid % C;
        float M = -INFINITY;
#pragma unroll
        for (int c2 = 0; c2 < C; ++c2) M = fmaxf(M, inbox[c2 * stride + kOut + gg]);
        const float lc = inbox[cc * stride + kOut + gg];
        wsm[tid] = (lc == -INFINITY) ? 0.f : ex2_fast(lc - M);
        if (cc == 0) msm[gg] = M;
      }
      __syncthreads();
      for (int o4 = tid; o4 < kOut / 4 && !dead; o4 += kThreadsC) {
        const int o = 4 * o4, gg = o / kHeadDim, d = o % kHeadDim;  // 4 dims of head gg
        const float M = msm[gg];
        float ov[4] = {0.f, 0.f, 0.f, 0.f};
        float l2 = -INFINITY;
        if (M != -INFINITY) {
          float Ls = 0.f;
#pragma unroll
          for (int cc = 0; cc < C; ++cc) {
            const float wc = wsm[gg * C + cc];
            const float4 av = *reinterpret_cast<const float4*>(inbox + cc * stride + o);
            Ls += wc;
            ov[0] = fmaf(wc, av.x, ov[0]);
            ov[1] = fmaf(wc, av.y, ov[1]);
            ov[2] = fmaf(wc, av.z, ov[2]);
            ov[3] = fmaf(wc, av.w, ov[3]);
          }
          const float rL = rcp_fast(Ls);
#pragma unroll
          for (int k = 0; k < 4; ++k) ov[k] *= rL;
          l2 = M + lg2_fast(Ls);
        }
        const size_t h = (size_t)b * p.hq + g * G + gg;
        float* dst = ly.out + h * kHeadDim + d;
        if ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
          *reinterpret_cast<float4*>(dst) = make_float4(ov[0], ov[1], ov[2], ov[3]);
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = ov[k];
        }
        if (ly.lse != nullptr && d == 0)
          ly.lse[h] = (l2 == -INFINITY) ? -INFINITY : l2 * 0.69314718055994531f;
        if (last && p.gate_mode == 1) {
          // h^L rows o .. o + 3 of this cluster go to the CTA whose W1 rows they meet
          if (p.rows_hl % 4 == 0) {
            dsmem_st4(&xh[o % p.rows_hl], (unsigned)(o / p.rows_hl),
                      make_float4(ov[0], ov[1], ov[2], ov[3]));
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              dsmem_st(&xh[(o + k) % p.rows_hl], (unsigned)((o + k) / p.rows_hl), ov[k]);
          }
        }
      }
      __syncthreads();  // the layer's output is written, the inbox read
      if (tid < C) mbar_arrive_remote(cluster_addr(obar, (unsigned)tid));  // (dead or not)
      if (!dead && tid == 0 && !last && !(p.test_stall && l == 0 && cl == 0))
        counter_release_add(&p.ctr[kCtrCount], 1u);  // this (b, g)'s layer-l output is written
    } else if (l == 0 && p.gate_mode == 1) {
      // [h_prev; emb] rows of W1 while rank 0 merges: inputs known since the start
      for (int i = tid; i < B * npre; i += kThreadsC) {
        const int bb = i / npre, rr = pre0 + i % npre;
        xs[bb * npre + i % npre] = rr < p.hidden ? p.h_prev[(size_t)bb * p.hidden + rr]
                                                 : p.emb[(size_t)bb * p.hidden + rr - p.hidden];
      }
      __syncthreads();
      if (tid < p.mlp) {
        for (int i0 = 0; i0 < npre; i0 += 16) {
          float wv[16];  // all of a chunk's loads in flight together
#pragma unroll
          for (int u = 0; u < 16; ++u)
            wv[u] = i0 + u < npre ? ld_keep(p.w1 + (size_t)(pre0 + i0 + u) * p.mlp + tid, keep)
                                  : 0.f;
#pragma unroll
          for (int bb = 0; bb < kChainMaxBatch; ++bb)
            if (bb < B)
#pragma unroll
              for (int u = 0; u < 16; ++u)
                if (i0 + u < npre) zpre[bb] = fmaf(wv[u], xs[bb * npre + i0 + u], zpre[bb]);
        }
      }
    }
  }
  // (ranks other than 0 still owe the wait of the last layer's cluster phase)

  // ---- recall head: this cluster's h^L rows arrive through distributed shared memory ----
  if (p.gate_mode == 1) {
    cluster_arrive();               // rank 0 arrives after its h^L stores (release) ...
    cluster_wait();                 // ... which every CTA then sees (acquire)
    const bool w1_ok =
        !w1_issued || __syncthreads_and(mbar_wait(wbar, 0u, p.wait_ns) ? 1 : 0) != 0;
    const bool use = !dead && w1_ok && w1_issued;
    if (use && tid < p.mlp) {
      const float* w1s = reinterpret_cast<const float*>(buf);
      float z = 0.f;
      for (int i = 0; i < nhl; ++i) z = fmaf(w1s[i * p.mlp + tid], xh[i], z);
#pragma unroll
      for (int bb = 0; bb < kChainMaxBatch; ++bb)
        if (bb == b) zpre[bb] += z;
    }
    if (!w1_ok && tid == 0) {
      report(p.status, ODA_DEV_TIMEOUT);
      atomicExch(&p.ctr[kCtrAbort], 1u);
    }
    // cluster sum of the CTAs' partial z, in rank order: every 4th lane gathers its
    // neighbours' columns and pushes them as one 16-byte store
#pragma unroll
    for (int bb = 0; bb < kChainMaxBatch; ++bb) {
      if (bb < B) {
        const float z0 = zpre[bb];
        const float z1 = __shfl_down_sync(0xffffffffu, z0, 1);
        const float z2 = __shfl_down_sync(0xffffffffu, z0, 2);
        const float z3 = __shfl_down_sync(0xffffffffu, z0, 3);
        if (tid < p.mlp && (tid & 3) == 0)
          dsmem_st4(inbox + rank * stride + bb * p.mlp + tid, 0, make_float4(z0, z1, z2, z3));
      }
    }
    cluster_arrive();
    if (rank == 0) {
      cluster_wait();  // every CTA's partial z is in this CTA's inbox
      if (use && tid < p.mlp)
        for (int bb = 0; bb < B; ++bb) {
          float z = 0.f;
#pragma unroll
          for (int cc = 0; cc < C; ++cc) z += inbox[cc * stride + bb * p.mlp + tid];
          __stcg(&p.z_clusters[((size_t)cl * B + bb) * p.mlp + tid], z);
        }
      __syncthreads();  // the cluster's z is written; thread 0 publishes it (release)
      if (tid == 0) s_flag = use && ticket_arrive(p.recall_ticket) == (unsigned)(ncl - 1);
      __syncthreads();
      if (s_flag) {  // the last cluster: z over every cluster in fixed order, then the gate
        if (tid == 0) s_count = 0u;
        for (int bb = 0; bb < B; ++bb) {
          float v = 0.f;
          if (tid < p.mlp) {
            float zc[kChainMaxClusters];
#pragma unroll
            for (int cc = 0; cc < kChainMaxClusters; ++cc)
              zc[cc] = cc < ncl ? __ldcg(&p.z_clusters[((size_t)cc * B + bb) * p.mlp + tid]) : 0.f;
            float z = 0.f;
#pragma unroll
            for (int cc = 0; cc < kChainMaxClusters; ++cc) z += zc[cc];
            v = gelu_erf(z + p.b1[tid]) * p.w2[tid];
          }
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0) s_red[warp][bb] = v;
        }
        __syncthreads();
        if (tid < B) {
          float q = 0.f;
#pragma unroll
          for (int w = 0; w < W; ++w) q += s_red[w][tid];
          q += p.b2;
          const int gate = q > p.theta ? 1 : 0;
          p.q_out[tid] = q;
          p.gate_out[tid] = gate;
          if (gate) atomicAdd(&s_count, 1u);
        }
        __syncthreads();
        if (tid == 0) {
          if (p.full_count != nullptr && s_count) {
            atomicAdd(&p.full_count[0], (unsigned long long)s_count);
            atomicAdd(&p.full_count[1], 1ull);
          }
          if (p.use_cond) cudaGraphSetConditional(p.cond, s_count ? 1u : 0u);
          *p.recall_ticket = 0u;
        }
      }
    }
  }

  // ---- leave: the last cluster phase, counters ----
  if (p.stats != nullptr && lane == 0 && pages_read) {
    atomicAdd(&s_rows, (unsigned long long)rows_vis);
    atomicAdd(&s_pages, (unsigned long long)pages_read);
  }
  // Every CTA arrives on every cluster phase and waits before leaving, so no CTA exits while
  // another may still store or copy into its shared memory: rank 0 arrives on the last one
  // after every partial of the last layer has landed in its inbox. A page whose wait ran out
  // gets one more bounded wait.
  if (rank != 0 && p.gate_mode == 1) cluster_wait();  // the recall head's last phase
  if (lane == 0 && stuck >= 0) mbar_wait(&bars[warp], (unsigned)stuck & 1u, p.wait_ns);
  cluster_arrive();
  cluster_wait();
  if (p.stats != nullptr && tid == 0) {
    if (s_rows) atomicAdd(&p.stats[ODA_STAT_ROWS], s_rows);
    if (s_pages) atomicAdd(&p.stats[ODA_STAT_PAGES], s_pages);
  }
  cta_exit(p.ctr, p.recall_ticket, p.gate_mode == 1 ? 1 : 0, &s_flag);
}

// ---------------------------------------------------------------------------------------
// Full over every layer.
// ---------------------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) full_chain_kernel(const FullChainParams cp) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_align, s_last, s_flag;
  __shared__ unsigned long long s_rows, s_pages;
  if (cp.L == 0) return;
  const int tid = threadIdx.x;
  const int B = cp.base.batch;

  // Device-side early exit: no gated sequence, nothing to recompute.
  int any = cp.base.plan.gate == nullptr ? 1 : 0;
  if (!any)
    for (int bb = tid; bb < B; bb += kThreads) any |= cp.base.plan.gate[bb] != 0;
  if (!__syncthreads_or(any)) return;

  const SplitSmem sm = split_smem<G>(smem, &s_align, &s_last, &s_rows, &s_pages);
  const long long T = split_prologue(cp.base.plan, B, cp.base.hkv, sm, cp.base.status);
  RingState rs{0u, false, false};
  const unsigned P = gridDim.x;
  for (int l = 0; l < cp.L; ++l) {
    DecodeParams p = cp.base;
    const ChainLayer& ly = cp.layer[l];
    p.k_cache = ly.k_cache;
    p.v_cache = ly.v_cache;
    p.k_cache_w = const_cast<__nv_bfloat16*>(ly.k_cache);
    p.v_cache_w = const_cast<__nv_bfloat16*>(ly.v_cache);
    p.q = ly.q;
    p.k_new = ly.k_new;
    p.v_new = ly.v_new;
    p.out = ly.out;
    p.lse = ly.lse;
    bool waited = l == 0, ok = true;
    auto wait = [&]() {
      if (!waited) {
        ok = cta_wait_count(cp.ctr, P * (unsigned)l, p.wait_ns, p.status, &s_flag);
        waited = true;
      }
      return ok;
    };
    decode_pass<G>(p, sm, T, rs, wait);
    if (rs.aborted) break;
    __syncthreads();  // this CTA's layer-l writes (outputs, merges, tickets) are done
    if (tid == 0 && !(cp.test_stall && l == 0 && blockIdx.x == 0))
      counter_release_add(&cp.ctr[kCtrCount], 1u);
  }
  cta_exit(cp.ctr, cp.base.ws_ticket, B * cp.base.hkv, &s_flag);
}

// ---------------------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------------------
// A shape of the Local kernel: C CTAs per cluster, W warps per CTA.
struct ChainShape {
  int C, W;
};
constexpr ChainShape kChainShapes[] = {{16, 9}, {14, 10}, {12, 11}, {8, 18}};
constexpr int kNumChainShapes = 4;
// Shapes tried in this order (the first whose clusters are all resident at once is used).
constexpr int kChainPrefer[kNumChainShapes] = {3, 1, 2, 0};

// Dynamic shared memory of the Local kernel: page buffer, merge scratch, barriers, per-warp
// softmax exchange, rank 0's inbox; for the one-CTA-per-SM shapes at least kOneCtaSmem.
constexpr size_t kOneCtaSmem = 118 * 1024;
static size_t local_chain_smem(int G, ChainShape sh, int inbox_stride) {
  const int scratch = sh.W == 9    ? chain_scratch_floats<9>(G)
                      : sh.W == 10 ? chain_scratch_floats<10>(G)
                      : sh.W == 11 ? chain_scratch_floats<11>(G)
                                   : chain_scratch_floats<18>(G);
  size_t n = (size_t)sh.W * kStageBytes + (size_t)scratch * sizeof(float) +
             (sh.W + 3) * sizeof(uint64_t) + (size_t)sh.W * 18 * G * sizeof(float) + 16 +
             (size_t)(sh.C + 1) * inbox_stride * sizeof(float);
  if (sh.C != 16 && n < kOneCtaSmem) n = kOneCtaSmem;
  return n;
}
struct ChainDeviceFacts {
  bool done = false;
  bool local_coop = false;  // cooperative cluster launches accepted
  bool full_ok[kMaxGroup + 1] = {false, false, false, false, false};
  // dynamic shared memory limit of the Local kernel, by group size and shape
  int max_dyn[kMaxGroup + 1][kNumChainShapes] = {};
  // clusters of the Local kernel resident at once, by group size, shape and shared memory
  int occ_g[32] = {0}, occ_s[32] = {0}, occ_n[32] = {0};
  size_t occ_smem[32] = {0};
  int occ_used = 0;
};
static ChainDeviceFacts g_chain[64];

template <int G, int C, int W>
static cudaError_t launch_local_chain_kernel(const LocalChainParams& p, int clusters,
                                             size_t smem, cudaStream_t st, bool coop) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(clusters * C);
  cfg.blockDim = dim3(W * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = coop ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, local_chain_kernel<G, C, W>, p);
}

template <int G>
static cudaError_t launch_full_chain_kernel(const FullChainParams& p, int grid, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = split_smem_bytes(G);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, full_chain_kernel<G>, p);
}

template <int G, int C, int W>
static int occupancy_clusters(size_t smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C);
  cfg.blockDim = dim3(W * 32);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, local_chain_kernel<G, C, W>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  return n;
}

// Attributes of one Local kernel instance: the dynamic shared memory it may ask for (the
// per-block maximum less its static shared memory) and the non-portable cluster size.
template <int G, int C, int W>
static cudaError_t local_attrs(int optin, int* max_dyn) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, local_chain_kernel<G, C, W>);
  if (e != cudaSuccess) return e;
  *max_dyn = optin > (int)fa.sharedSizeBytes ? optin - (int)fa.sharedSizeBytes : 0;
  if ((e = cudaFuncSetAttribute(local_chain_kernel<G, C, W>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, *max_dyn)) !=
      cudaSuccess)
    return e;
  return cudaFuncSetAttribute(local_chain_kernel<G, C, W>,
                              cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
}

// The instances by (group size, shape index): one dispatch per operation.
#define ODA_LOCAL_INSTANCES(X) \
  X(1, 0, 16, 9) X(1, 1, 14, 10) X(1, 2, 12, 11) X(1, 3, 8, 18) \
  X(2, 0, 16, 9) X(2, 1, 14, 10) X(2, 2, 12, 11) X(2, 3, 8, 18) \
  X(4, 0, 16, 9) X(4, 1, 14, 10) X(4, 2, 12, 11)
static bool local_has(int G, int si) {
#define ODA_X(g, i, c, w) \
  if (G == g && si == i) return true;
  ODA_LOCAL_INSTANCES(ODA_X)
#undef ODA_X
  return false;
}

static cudaError_t local_launch(int G, int si, const LocalChainParams& p, int clusters,
                                size_t smem, cudaStream_t st, bool coop) {
#define ODA_X(g, i, c, w) \
  if (G == g && si == i) return launch_local_chain_kernel<g, c, w>(p, clusters, smem, st, coop);
  ODA_LOCAL_INSTANCES(ODA_X)
#undef ODA_X
  return cudaErrorInvalidValue;
}
static int local_occupancy(int G, int si, size_t smem) {
#define ODA_X(g, i, c, w) \
  if (G == g && si == i) return occupancy_clusters<g, c, w>(smem);
  ODA_LOCAL_INSTANCES(ODA_X)
#undef ODA_X
  return 0;
}
static cudaError_t local_set_attrs(int G, int si, int optin, int* max_dyn) {
#define ODA_X(g, i, c, w) \
  if (G == g && si == i) return local_attrs<g, c, w>(optin, max_dyn);
  ODA_LOCAL_INSTANCES(ODA_X)
#undef ODA_X
  return cudaErrorInvalidValue;
}

template <int G>
static int prepare_full_g(ChainDeviceFacts& f) {
  const cudaError_t e = cudaFuncSetAttribute(
      full_chain_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)split_smem_bytes(G));
  if (e != cudaSuccess) return cuda_status(e);
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, full_chain_kernel<G>, kThreads,
                                                    split_smem_bytes(G)) != cudaSuccess) {
    cudaGetLastError();
    per_sm = 0;
  }
  f.full_ok[G] = per_sm >= kCtasPerSm;
  return ODA_OK;
}

// Attributes, the Full kernel's residency and whether cooperative cluster launches are
// accepted, once per device, outside any stream capture (the probe launches the Local kernel
// with no layer, which returns at once).
int prepare_chain_kernels() {
  DeviceInfo di;
  int rc = current_device_info(&di);
  if (rc != ODA_OK) return rc;
  ChainDeviceFacts& f = g_chain[di.device];
  if (f.done) return ODA_OK;
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                         di.device);
  if (e != cudaSuccess) return cuda_status(e);
  for (int G : {1, 2, 4})
    for (int si = 0; si < kNumChainShapes; ++si)
      if (local_has(G, si) && (e = local_set_attrs(G, si, optin, &f.max_dyn[G][si])) != cudaSuccess)
        return cuda_status(e);
  if ((rc = prepare_full_g<1>(f)) != ODA_OK) return rc;
  if ((rc = prepare_full_g<2>(f)) != ODA_OK) return rc;
  if ((rc = prepare_full_g<4>(f)) != ODA_OK) return rc;
  f.local_coop = false;
  const size_t probe_smem = local_chain_smem(2, kChainShapes[0], ClusterPart<2>::value);
  static_assert(ClusterPart<2>::value % 4 == 0, "inbox slots hold 16-byte stores");
  if (probe_smem <= (size_t)f.max_dyn[2][0] && local_occupancy(2, 0, probe_smem) > 0) {
    cudaStream_t s = nullptr;
    if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) == cudaSuccess) {
      LocalChainParams probe = {};
      probe.L = 0;
      e = local_launch(2, 0, probe, 1, probe_smem, s, true);
      f.local_coop = e == cudaSuccess && cudaStreamSynchronize(s) == cudaSuccess;
      cudaGetLastError();
      cudaStreamDestroy(s);
    }
  }
  f.done = true;
  return ODA_OK;
}

// Clusters of the Local kernel the device holds at once (queried once per group size, shape
// and shared memory; outside stream capture).
static int local_clusters(int dev, int G, int si, size_t smem) {
  ChainDeviceFacts& f = g_chain[dev];
  if (smem > (size_t)f.max_dyn[G][si]) return 0;
  for (int i = 0; i < f.occ_used; ++i)
    if (f.occ_g[i] == G && f.occ_s[i] == si && f.occ_smem[i] == smem) return f.occ_n[i];
  const int n = local_occupancy(G, si, smem);
  if (f.occ_used < 32) {
    f.occ_g[f.occ_used] = G;
    f.occ_s[f.occ_used] = si;
    f.occ_smem[f.occ_used] = smem;
    f.occ_n[f.occ_used] = n;
    ++f.occ_used;
  }
  return n;
}

// Shared memory of the Local kernel for a step: the inbox rows hold a CTA partial or, with
// the fused recall head, the batch's partial z.
static size_t local_chain_smem_for(int G, ChainShape sh, int B, int mlp, bool fused) {
  const int part = (G * kHeadDim + G + 3) / 4 * 4;  // ClusterPart<G>::value
  const int stride = fused && B * mlp > part ? B * mlp : part;
  return local_chain_smem(G, sh, stride);
}

// Whether the fused recall head can serve this step (shapes and the recall workspace).
static bool recall_fusable(const oda_step_desc* d, int B, int G, ChainShape sh, int hidden,
                           int clusters) {
  if (d->gate_source != ODA_GATE_RECALL) return true;
  if (B > kChainMaxBatch || d->mlp > sh.W * 32 || d->mlp % 64 != 0 || d->mlp < 64)
    return false;
  if (!aligned_or_null(d->w1, 16)) return false;  // the h^L rows arrive by one bulk copy
  const int workers = clusters * (sh.C - 1);
  const int rows_pre = (2 * hidden + workers - 1) / workers;
  const int rows_hl = (G * kHeadDim + sh.C - 1) / sh.C;
  if ((long long)rows_pre * B > kChainXs || rows_hl > kChainMaxHl ||
      (size_t)rows_hl * d->mlp * sizeof(float) > (size_t)sh.W * kStageBytes ||
      clusters > kChainMaxClusters)
    return false;
  size_t rbytes = 0;
  if (oda_recall_workspace_size(B, hidden, d->mlp, &rbytes) != ODA_OK) return false;
  const int slabs = (3 * hidden + kRows - 1) / kRows;
  return clusters <= slabs && d->recall_ws != nullptr && d->recall_ws_bytes >= rbytes;
}

int plan_local_chain(const oda_step_desc* d, int phases, LocalChainPlan* pl) {
  *pl = LocalChainPlan{};
  if (!(phases & ODA_PHASE_LOCAL) || d->step_kernels != ODA_STEP_PERSISTENT) return ODA_OK;
  DeviceInfo di;
  int rc = current_device_info(&di);
  if (rc != ODA_OK) return rc;
  const ChainDeviceFacts& f = g_chain[di.device];
  const oda_kv& k0 = d->layers[0];
  const int B = k0.batch, hkv = k0.num_kv_heads, hq = d->num_q_heads;
  if (!f.done || hq % hkv != 0 || d->num_layers > kMaxChainLayers) return ODA_OK;
  const int G = hq / hkv;
  if (G != 1 && G != 2 && G != 4) return ODA_OK;
  long long max_pages = 0;
  for (int l = 0; l < d->num_layers; ++l) {
    if (d->local_layers != nullptr && d->local_layers[l] == 0) return ODA_OK;
    const int s = d->sinks ? d->sinks[l] : d->sink, w = d->windows ? d->windows[l] : d->window;
    const long long pages = (s + kPage - 1) / kPage + (long long)(w - 1) / kPage + 2;
    if (pages > max_pages) max_pages = pages;
    const oda_kv& k = d->layers[l];
    if (k.num_blocks != k0.num_blocks || k.dev_status != k0.dev_status || k.stats != k0.stats)
      return ODA_OK;
  }
  const int ncl = B * hkv;
  const bool want_gate = (phases & ODA_PHASE_RECALL) != 0;
  // shapes in order of preference (one CTA per SM first), or the one a tuning hook names
  const int forced = test_local_shape();
  for (int k = 0; k < kNumChainShapes; ++k) {
    const int si = forced >= 0 ? forced : kChainPrefer[k];
    if (forced >= 0 && k > 0) break;
    const ChainShape sh = kChainShapes[si];
    if (max_pages > (long long)sh.C * sh.W) continue;
    const bool fusable = want_gate && recall_fusable(d, B, G, sh, hq * kHeadDim, ncl);
    for (int fuse = fusable ? 1 : 0; fuse >= 0; --fuse) {
      const size_t smem = local_chain_smem_for(G, sh, B, d->mlp, fuse != 0);
      if (local_clusters(di.device, G, si, smem) < ncl) continue;
      pl->usable = 1;
      pl->gate_fused = fuse;
      pl->clusters = ncl;
      pl->shape = si;
      pl->smem = smem;
      return ODA_OK;
    }
  }
  return ODA_OK;
}

int launch_local_chain(const oda_step_desc* d, const LocalChainPlan& pl, int phases,
                       unsigned long long cond, void* stream) {
  if (!pl.usable) return ODA_ERR_NOT_IMPLEMENTED;
  const oda_kv& k0 = d->layers[0];
  const int B = k0.batch, hkv = k0.num_kv_heads, hq = d->num_q_heads;
  const int G = hq / hkv;
  DeviceInfo di;
  int rc = current_device_info(&di);
  if (rc != ODA_OK) return rc;
  const int L = d->num_layers;
  const int hidden = hq * kHeadDim;
  const int gate_mode = !(phases & ODA_PHASE_RECALL) || !pl.gate_fused ? 0
                        : (d->gate_source == ODA_GATE_RANDOM ? 2 : 1);
  LocalChainParams p = {};
  p.L = L;
  p.batch = B;
  p.hkv = hkv;
  p.hq = hq;
  p.seq_lens = k0.seq_lens;
  p.block_table = k0.block_table;
  p.max_blocks = k0.max_blocks_per_seq;
  p.num_blocks = k0.num_blocks;
  p.scale_log2 = d->scale * 1.4426950408889634f;
  p.status = k0.dev_status;
  p.stats = k0.stats;
  p.wait_ns = test_wait_ns();
  p.test_stall = test_stall() == ODA_STALL_LOCAL_CHAIN ? 1 : 0;
  for (int l = 0; l < L; ++l) {
    const oda_kv& k = d->layers[l];
    if ((rc = check_kv(&k)) != ODA_OK) return rc;
    if (!aligned_or_null(d->q_local[l], 16) || !aligned_or_null(d->k_local[l], 16) ||
        !aligned_or_null(d->v_local[l], 16) || !aligned_or_null(d->out[l], 4) ||
        d->q_local[l] == nullptr || d->out[l] == nullptr ||
        (d->k_local[l] == nullptr) != (d->v_local[l] == nullptr) ||
        (d->lse != nullptr && !aligned_or_null(d->lse[l], 4)))
      return ODA_ERR_INVALID_ARG;
    ChainLayer& c = p.layer[l];
    c.k_cache = static_cast<const __nv_bfloat16*>(k.k_cache);
    c.v_cache = static_cast<const __nv_bfloat16*>(k.v_cache);
    c.q = static_cast<const __nv_bfloat16*>(d->q_local[l]);
    c.k_new = static_cast<const __nv_bfloat16*>(d->k_local[l]);
    c.v_new = static_cast<const __nv_bfloat16*>(d->v_local[l]);
    c.out = static_cast<float*>(d->out[l]);
    c.lse = d->lse ? d->lse[l] : nullptr;
    c.sink = d->sinks ? d->sinks[l] : d->sink;
    c.window = d->windows ? d->windows[l] : d->window;
  }
  if (!(d->scale > 0.f) || !isfinite(d->scale)) return ODA_ERR_INVALID_ARG;
  p.gate_mode = gate_mode;
  p.hidden = hidden;
  p.mlp = d->mlp;
  const ChainShape sh = kChainShapes[pl.shape];
  if (gate_mode == 1) {
    for (const void* f : {static_cast<const void*>(d->h_prev), static_cast<const void*>(d->emb),
                          static_cast<const void*>(d->b1), static_cast<const void*>(d->w2),
                          static_cast<const void*>(d->q_out), static_cast<const void*>(d->gate_out)})
      if (f == nullptr || !aligned_or_null(f, 4)) return ODA_ERR_INVALID_ARG;
    if (d->w1 == nullptr || !aligned_or_null(d->full_count, 8)) return ODA_ERR_INVALID_ARG;
    // h^L rows: each cluster's heads (128 G rows of its sequence), 8 G per CTA in rank order;
    // [h_prev; emb] rows: spread over the CTAs other than each cluster's rank 0
    const int workers = pl.clusters * (sh.C - 1);
    p.rows_pre = (2 * hidden + workers - 1) / workers;
    p.rows_hl = (G * kHeadDim + sh.C - 1) / sh.C;
    // The recall workspace holds the z partials of its slabs first (at least as many slabs as
    // clusters here) and its tickets after them; ticket [tiles] is the one-level ticket.
    size_t ticket_off = 0;
    int tiles = 0;
    if ((rc = recall_ws_tickets(B, hidden, d->mlp, &ticket_off, &tiles)) != ODA_OK) return rc;
    unsigned char* w = static_cast<unsigned char*>(d->recall_ws);
    p.z_clusters = reinterpret_cast<float*>(w);
    p.recall_ticket = reinterpret_cast<unsigned*>(w + ticket_off) + tiles;
    p.h_prev = d->h_prev;
    p.emb = d->emb;
    p.w1 = d->w1;
    p.b1 = d->b1;
    p.w2 = d->w2;
    p.b2 = d->b2;
    p.theta = d->theta;
  } else if (gate_mode == 2) {
    if (d->gate_u == nullptr || !aligned_or_null(d->gate_u, 4) || d->gate_out == nullptr ||
        !aligned_or_null(d->gate_out, 4) || !aligned_or_null(d->full_count, 8))
      return ODA_ERR_INVALID_ARG;
    p.gate_u = d->gate_u;
    p.rho = d->rho;
  }
  p.q_out = d->q_out;
  p.gate_out = d->gate_out;
  p.full_count = d->full_count;
  p.cond = static_cast<cudaGraphConditionalHandle>(cond);
  p.use_cond = gate_mode != 0 && cond != 0ull;
  size_t total = 0, chain_off = 0;
  if ((rc = decode_ws_chain_offset(B, hkv, hq, &total, &chain_off)) != ODA_OK) return rc;
  if (d->decode_ws == nullptr || !aligned_or_null(d->decode_ws, 16) || d->decode_ws_bytes < total)
    return ODA_ERR_WORKSPACE_TOO_SMALL;
  p.ctr = reinterpret_cast<unsigned*>(static_cast<unsigned char*>(d->decode_ws) + chain_off);
  const bool coop = g_chain[di.device].local_coop;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(local_launch(G, pl.shape, p, pl.clusters, pl.smem, st, coop));
}

int launch_full_chain(const oda_step_desc* d, void* stream) {
  const oda_kv& k0 = d->layers[0];
  const int B = k0.batch, hkv = k0.num_kv_heads, hq = d->num_q_heads;
  if (hq % hkv != 0) return ODA_ERR_UNSUPPORTED_SHAPE;
  const int G = hq / hkv;
  if (G != 1 && G != 2 && G != 4) return ODA_ERR_UNSUPPORTED_SHAPE;
  DeviceInfo di;
  int rc = current_device_info(&di);
  if (rc != ODA_OK) return rc;
  if (!g_chain[di.device].full_ok[G] || d->num_layers > kMaxChainLayers)
    return ODA_ERR_NOT_IMPLEMENTED;
  const int L = d->num_layers;
  FullChainParams cp = {};
  cp.L = L;
  for (int l = 0; l < L; ++l) {
    const oda_kv& k = d->layers[l];
    if (k.num_blocks != k0.num_blocks || k.dev_status != k0.dev_status || k.stats != k0.stats)
      return ODA_ERR_NOT_IMPLEMENTED;
    if ((rc = check_kv(&k)) != ODA_OK) return rc;
    if (d->q_full[l] == nullptr || d->out[l] == nullptr || !aligned_or_null(d->q_full[l], 16) ||
        !aligned_or_null(d->k_full[l], 16) || !aligned_or_null(d->v_full[l], 16) ||
        (d->k_full[l] == nullptr) != (d->v_full[l] == nullptr) ||
        !aligned_or_null(d->out[l], 4) || (d->lse != nullptr && !aligned_or_null(d->lse[l], 4)))
      return ODA_ERR_INVALID_ARG;
    ChainLayer& c = cp.layer[l];
    c.k_cache = static_cast<const __nv_bfloat16*>(k.k_cache);
    c.v_cache = static_cast<const __nv_bfloat16*>(k.v_cache);
    c.q = static_cast<const __nv_bfloat16*>(d->q_full[l]);
    c.k_new = static_cast<const __nv_bfloat16*>(d->k_full[l]);
    c.v_new = static_cast<const __nv_bfloat16*>(d->v_full[l]);
    c.out = static_cast<float*>(d->out[l]);
    c.lse = d->lse ? d->lse[l] : nullptr;
  }
  // The base parameters are those of a gated Full decode of layer 0 (same checks).
  oda_visibility vis = visibility(ODA_MODE_FULL);
  vis.gate = d->gate_out;
  DecodeParams base;
  if ((rc = decode_params(&k0, vis, d->q_full[0], hq, d->scale, d->k_full[0], d->v_full[0],
                          d->out[0], ODA_F32, d->lse ? d->lse[0] : nullptr, d->decode_ws,
                          d->decode_ws_bytes, &base)) != ODA_OK)
    return rc;
  cp.base = base;
  size_t total = 0, chain_off = 0;
  if ((rc = decode_ws_chain_offset(B, hkv, hq, &total, &chain_off)) != ODA_OK) return rc;
  cp.ctr = reinterpret_cast<unsigned*>(static_cast<unsigned char*>(d->decode_ws) + chain_off) +
           kCtrWords;
  cp.test_stall = test_stall() == ODA_STALL_FULL_CHAIN ? 1 : 0;
  const int grid = di.sms * kCtasPerSm;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (G) {
    case 1: e = launch_full_chain_kernel<1>(cp, grid, st); break;
    case 2: e = launch_full_chain_kernel<2>(cp, grid, st); break;
    default: e = launch_full_chain_kernel<4>(cp, grid, st); break;
  }
  return cuda_status(e);
}

int step_kernel_limits(int G, int batch, int mlp, int* clusters, int* cooperative) {
  DeviceInfo di;
  int rc = current_device_info(&di);
  if (rc != ODA_OK) return rc;
  if ((rc = prepare_chain_kernels()) != ODA_OK) return rc;
  if (G != 1 && G != 2 && G != 4) return ODA_ERR_UNSUPPORTED_SHAPE;
  int best = 0;  // the most clusters any shape fits (a step takes the first shape that fits)
  for (int si = 0; si < kNumChainShapes; ++si) {
    const int n = local_clusters(di.device, G, si,
                                 local_chain_smem_for(G, kChainShapes[si], batch, mlp, mlp > 0));
    if (n > best) best = n;
  }
  *clusters = best;
  *cooperative = g_chain[di.device].local_coop ? 1 : 0;
  return ODA_OK;
}

}  // namespace oda

using namespace oda;

extern "C" int oda_step_kernel_limits(int32_t group, int32_t batch, int32_t mlp,
                                      int32_t* max_clusters, int32_t* cooperative) {
  if (max_clusters == nullptr || cooperative == nullptr || batch < 1 || mlp < 0)
    return ODA_ERR_INVALID_ARG;
  int n = 0, c = 0;
  const int rc = step_kernel_limits(group, batch, mlp, &n, &c);
  if (rc != ODA_OK) return rc;
  *max_clusters = n;
  *cooperative = c;
  return ODA_OK;
}

// K2 + K3: paged decode attention for Local, Full, keep-page, DA and shard visibility, split
// over the whole GPU and merged inside the same launch (decode_kernel: one split pass, see
// oda_decode.cuh), and the short-window cluster kernel for Local at small batch.
#include <math.h>

#include "oda_decode.cuh"

namespace oda {

template <int G>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_align, s_last;
  __shared__ unsigned long long s_rows, s_pages;
  const SplitSmem sm = split_smem<G>(smem, &s_align, &s_last, &s_rows, &s_pages);

  // Programmatic dependent launch: before griddep_wait this kernel only reads data that no
  // kernel still in flight writes (lengths, page tables, keep lists, history pages) and fills
  // shared memory; every global write and every read of q / k_new / v_new comes after it.
  bool waited = false;
  auto dep_wait = [&]() {
    if (!waited) {
      griddep_wait();
      griddep_launch_dependents();
      waited = true;
    }
    return true;
  };
  if (p.wait_first) dep_wait();
  const long long T = split_prologue(p.plan, p.batch, p.hkv, sm, p.status);
  RingState rs{0u, false, false};
  decode_pass<G>(p, sm, T, rs, dep_wait);
}

// ---------------------------------------------------------------------------------------
// Short-window kernel (Local at small batch). The split above ends a short launch with a
// chain of global round trips: every CTA's partial to global memory, an acquire-release
// ticket, the last CTA reading every partial back. Here one thread-block cluster of
// kLocalCtas CTAs takes one (sequence, KV head). Ranks 1 .. kLocalCtas - 1 hold the pages,
// one per warp (kLocalClusterPages at most); each forms its CTA partial and sends it straight
// into rank 0's shared memory by st.async stores that complete on rank 0's inbox mbarrier, and
// leaves. Rank 0 holds no page: its stage memory is that inbox; once the barrier phase shows
// every partial landed it merges them in rank order and writes the output. No CTA waits for
// another except rank 0 for the partials (the cluster barrier is only split around the
// launch, to publish the mbarrier's initialisation before the first remote store), so a
// CTA's SM slot frees as soon as its partial is sent, for the next layer's clusters. The page
// step (tensor-core scores for G = 2 and 4), the commit of slot t and the in-CTA merge are
// those of the split pass and the persistent Local kernel.
// ---------------------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(kLocalThreads, kLocalCtasPerSm)
    cluster_decode_kernel(const DecodeParams p) {
  constexpr bool kMma = MmaScores<G>::value;
  constexpr int VPL = ClusterStates<G, kMma>::VPL;
  constexpr int kPs = 18 * G;
  constexpr int kPart = ClusterPart<G>::value;
  static_assert(kLocalCtas * kPart * sizeof(float) <= kLocalWarps * kStageBytes,
                "rank 0's inbox lives in its stage memory");
  static_assert(cluster_scratch_floats<G, kMma, kLocalWarps>() * sizeof(float) <=
                    kLocalWarps * kStageBytes,
                "the in-CTA merge reuses the stage memory");
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* stages = smem;  // [warp][kStageBytes]: one page per warp (ranks >= 1)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kLocalWarps * kStageBytes);
  float* pscratch = reinterpret_cast<float*>(bars + kLocalWarps);  // [warp][kPs]
  // rank 0: [kLocalCtas][kPart] partials (slot r from rank r; slot 0 unused)
  float* inbox = reinterpret_cast<float*>(stages);
  __shared__ unsigned long long s_rows, s_pages;
  __shared__ __align__(8) uint64_t s_inbar;  // rank 0: every partial has landed
  constexpr uint32_t kPartBytes = (ClusterPart<G>::kOut + G) * sizeof(float);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int li = lane & 15;
  const unsigned rank = cluster_ctarank();
  const int bg = blockIdx.x / kLocalCtas;
  const int b = bg / p.hkv, g = bg % p.hkv;
  if (tid == 0) {
    s_rows = 0;
    s_pages = 0;
  }
  if (lane == 0) {
    mbar_init(&bars[warp], 1);
    if (tid == 0 && rank == 0) {
      mbar_init(&s_inbar, 1);
      mbar_arrive_expect_tx(&s_inbar, (kLocalCtas - 1) * kPartBytes);
    }
    fence_barrier_init();
  }
  __syncwarp();
  cluster_arrive_relaxed();  // rank 0's inbox barrier is initialised (waited for before a push)
  // The next kernel (the next layer, or the recall head) may launch as soon as every CTA of
  // this one is resident: its own pre-wait reads touch nothing this one writes.
  griddep_launch_dependents();
  if (p.wait_first) griddep_wait();

  // Before the dependency wait: the plan and this warp's page copy (history pages only).
  const SeqPlan sp = make_plan(p.plan, b);
  if (rank == 0 && g == 0 && tid == 0 && sp.err != 0) report(p.status, sp.err);
  const int j = ((int)rank - 1) * kLocalWarps + warp;
  const bool has = rank != 0 && !sp.skip && j < sp.npages;
  const size_t head_off = (size_t)g * (kPage * kHeadDim);
  const size_t page_stride = (size_t)p.hkv * kPage * kHeadDim;
  unsigned char* st = stages + warp * kStageBytes;
  PageRef r;
  r.err = 0;
  r.lp = 0;
  r.pb = 0;
  if (has) {
    r = page_ref(p.plan, sp, b, j);
    if (lane == 0) {
      if (r.err == 0) {
        const uint64_t policy = l2_evict_first_policy();
        const size_t src = (size_t)r.pb * page_stride + head_off;
        mbar_arrive_expect_tx(&bars[warp], kStageBytes);
        bulk_load(st, p.k_cache + src, kPageBytes, &bars[warp], policy);
        bulk_load(st + kPageBytes, p.v_cache + src, kPageBytes, &bars[warp], policy);
      } else {
        report(p.status, r.err);
      }
    }
  }
  __syncwarp();
  if (!p.wait_first) griddep_wait();

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
  unsigned rows_vis = 0, pages_read = 0;
  if (has && r.err == 0) {
    f2_t q2[G][4];
    uint4 qv[4];
    if constexpr (kMma) load_q_mma<G>(p.q + ((size_t)b * p.hq + g * G) * kHeadDim, lane, qv);
    else load_q_scaled<G>(p.q, p.hq, b, g, p.scale_log2, li, q2);
    if (!__all_sync(0xffffffffu, mbar_wait(&bars[warp], 0u, p.wait_ns))) {
      if (lane == 0) report(p.status, ODA_DEV_TIMEOUT);
    } else {
      if (p.k_new != nullptr && r.lp == sp.t / kPage)
        commit_slot(st, p.k_new, p.v_new, p.k_cache_w, p.v_cache_w, b, p.hkv, g, sp.t, r.pb,
                    lane);
      if constexpr (kMma)
        page_step_mma<G>(st, qv, p.scale_log2, m_run, l_run, acc, pscratch + warp * kPs, sp,
                         r.lp, lane, rows_vis);
      else
        page_step<G>(st, q2, m_run, l_run, acc, pscratch + warp * kPs, sp, r.lp, lane,
                     rows_vis);
      pages_read = 1;
    }
  }

  // ---- merge the CTA's warp states, push to rank 0 ----
  if (p.stats != nullptr && lane == 0 && pages_read) {
    atomicAdd(&s_rows, (unsigned long long)rows_vis);
    atomicAdd(&s_pages, (unsigned long long)pages_read);
  }
  __syncthreads();  // every warp is done with its page: stage memory becomes merge scratch
  if (p.stats != nullptr && tid == 0) {
    if (s_rows) atomicAdd(&p.stats[ODA_STAT_ROWS], s_rows);
    if (s_pages) atomicAdd(&p.stats[ODA_STAT_PAGES], s_pages);
  }
  cluster_wait();  // (long since complete: every CTA arrived at its start)
  if (rank != 0) {
    if (!(p.test_stall == 2 && bg == 0 && rank == 1))  // (test hook: withhold this partial)
      cluster_push_partial<G, kMma, kLocalWarps, false, true>(
          m_run, l_run, acc, reinterpret_cast<float*>(stages), inbox, kPart, rank,
          cluster_addr(&s_inbar, 0));
  } else if (tid < kHeadDim) {
    if (!mbar_wait_cluster(&s_inbar, 0u, p.wait_ns)) {
      if (tid == 0) report(p.status, ODA_DEV_TIMEOUT);
    } else if (!sp.skip) {
      float o[G], l2[G];
      cluster_merge_inbox<G, 1, kLocalCtas>(inbox, kPart, o, l2);
      write_final<G>(p, b, g, o, l2);
    }
  }
}

// Debug export of the same plan: mask[b][p] = 1 for every visible position p < max_tokens.
__global__ void visible_mask_kernel(PlanArgs a, uint8_t* mask, int max_tokens, int* status) {
  const int b = blockIdx.x;
  uint8_t* row = mask + (size_t)b * max_tokens;
  for (int i = threadIdx.x; i < max_tokens; i += blockDim.x) row[i] = 0;
  __syncthreads();
  const SeqPlan sp = make_plan(a, b);
  if (sp.err != 0) report(status, sp.err);
  if (sp.skip || sp.err != 0) return;
  for (int idx = threadIdx.x; idx < sp.npages * kPage; idx += blockDim.x) {
    const int j = idx / kPage, r = idx % kPage;
    const PageRef pr = page_ref(a, sp, b, j);
    if (pr.err != 0) {
      report(status, pr.err);
      continue;
    }
    const int pos = pr.lp * kPage + r;
    if (pos < max_tokens && row_visible(sp, pos)) row[pos] = 1;
  }
}

// ---------------------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------------------
static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The CTAs of a Local cluster on distinct SMs where the hardware can: their page steps are
// bound by instruction issue, so two of one cluster on one SM take turns.
constexpr cudaClusterSchedulingPolicy kLocalClusterPolicy = cudaClusterSchedulingPolicySpread;

static size_t decode_smem_bytes(int G) { return split_smem_bytes(G); }

// Decode workspace: split partials (O and log-sums, one slot per CTA and per (b, g)), the
// merge tickets, and the launch-wide counters of the persistent step kernels.
struct WsLayout {
  size_t o_off, lse_off, ticket_off, chain_off, total;
};

static WsLayout ws_layout(int batch, int hkv, int G, int grid) {
  const size_t slots = (size_t)grid + (size_t)batch * hkv;
  WsLayout w;
  w.o_off = 0;
  w.lse_off = align_up(slots * G * kHeadDim * sizeof(float), 256);
  w.ticket_off = w.lse_off + align_up(slots * G * sizeof(float), 256);
  w.chain_off = w.ticket_off + align_up((size_t)batch * hkv * sizeof(unsigned), 256);
  w.total = w.chain_off + 256;
  return w;
}

// Stages (rank 0: the inbox), one mbarrier and the softmax exchange per warp (73.3 KB at
// G = 2, 74.6 KB at G = 4), padded to kLocalSmemFloor: two CTAs per SM.
static size_t cluster_smem_bytes(int G) {
  const size_t need = (size_t)kLocalWarps * kStageBytes +
                      (size_t)kLocalWarps * sizeof(uint64_t) +
                      (size_t)kLocalWarps * 18 * G * sizeof(float);
  return need > kLocalSmemFloor ? need : kLocalSmemFloor;
}

// Clusters of the short-window kernel the device can hold at once, per device and group
// size (0: the cluster shape cannot be scheduled here, e.g. under a partitioned GPU).
static int g_max_clusters[64][kMaxGroup + 1];

template <int G>
static int prepare_decode_kernel(int device) {
  static bool done[64] = {false};
  if (device < 0 || device >= 64) return ODA_ERR_CUDA;
  if (done[device]) return ODA_OK;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(decode_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)decode_smem_bytes(G))) != cudaSuccess ||
      (e = cudaFuncSetAttribute(cluster_decode_kernel<G>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)cluster_smem_bytes(G))) != cudaSuccess ||
      (e = cudaFuncSetAttribute(cluster_decode_kernel<G>,
                                cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) != cudaSuccess)
    return cuda_status(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kLocalCtas);
  cfg.blockDim = dim3(kLocalThreads);
  cfg.dynamicSmemBytes = cluster_smem_bytes(G);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kLocalCtas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
  attr[1].val.clusterSchedulingPolicyPreference = kLocalClusterPolicy;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, cluster_decode_kernel<G>, &cfg) != cudaSuccess) {
    cudaGetLastError();  // not fatal: the split kernel serves every launch
    n = 0;
  }
  g_max_clusters[device][G] = n;
  done[device] = true;
  return ODA_OK;
}

static int grid_size(const DeviceInfo& di) { return di.sms * kCtasPerSm; }

int current_device_info(DeviceInfo* info) {
  static DeviceInfo cache[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ODA_ERR_CUDA;
  if (cache[dev].device != dev) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ODA_ERR_CUDA;
    cache[dev].sms = sms;
    cache[dev].device = dev;
  }
  *info = cache[dev];
  return ODA_OK;
}

// Called before graph capture so that no attribute call happens while capturing.
int prepare_decode_kernels() {
  DeviceInfo di;
  int rc = current_device_info(&di);
  if (rc != ODA_OK) return rc;
  if ((rc = prepare_decode_kernel<1>(di.device)) != ODA_OK) return rc;
  if ((rc = prepare_decode_kernel<2>(di.device)) != ODA_OK) return rc;
  return prepare_decode_kernel<4>(di.device);
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_kv(const oda_kv* kv) {
  if (kv == nullptr) return ODA_ERR_INVALID_ARG;
  if (kv->batch < 0 || kv->num_kv_heads < 1 || kv->max_blocks_per_seq < 1 || kv->num_blocks < 1)
    return ODA_ERR_INVALID_ARG;
  if (kv->head_dim != kHeadDim || kv->block_size != kPage) return ODA_ERR_UNSUPPORTED_SHAPE;
  if (kv->batch > kMaxBatch) return ODA_ERR_UNSUPPORTED_SHAPE;
  if ((long long)kv->batch * kv->max_blocks_per_seq * kv->num_kv_heads >= (1ll << 31))
    return ODA_ERR_UNSUPPORTED_SHAPE;
  if (kv->batch > 0 && (kv->k_cache == nullptr || kv->v_cache == nullptr ||
                        kv->block_table == nullptr || kv->seq_lens == nullptr))
    return ODA_ERR_INVALID_ARG;
  if (!aligned16(kv->k_cache) || !aligned16(kv->v_cache)) return ODA_ERR_INVALID_ARG;
  if (!aligned_or_null(kv->block_table, 4) || !aligned_or_null(kv->seq_lens, 4) ||
      !aligned_or_null(kv->dev_status, 4) || !aligned_or_null(kv->stats, 8))
    return ODA_ERR_INVALID_ARG;
  return ODA_OK;
}

static int group_of(const oda_kv* kv, int hq, int* G) {
  if (hq < 1 || hq % kv->num_kv_heads != 0) return ODA_ERR_UNSUPPORTED_SHAPE;
  const int g = hq / kv->num_kv_heads;
  if (g != 1 && g != 2 && g != 4) return ODA_ERR_UNSUPPORTED_SHAPE;
  *G = g;
  return ODA_OK;
}

template <int G>
static cudaError_t launch_decode_kernel(const DecodeParams& p, int grid, size_t smem,
                                        cudaStream_t st, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, decode_kernel<G>, p);
}

template <int G>
static cudaError_t launch_cluster_kernel(const DecodeParams& p, int grid, cudaStream_t st,
                                         bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kLocalThreads);
  cfg.dynamicSmemBytes = cluster_smem_bytes(G);
  cfg.stream = st;
  cudaLaunchAttribute attr[3];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kLocalCtas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
  attr[1].val.clusterSchedulingPolicyPreference = kLocalClusterPolicy;
  attr[2].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[2].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 3 : 2;
  return cudaLaunchKernelEx(&cfg, cluster_decode_kernel<G>, p);
}

// The short-window kernel takes a launch when the rule bounds every sequence's page list by
// one cluster's warps (Local: sink pages + window pages) and one cluster per (sequence, KV
// head) fits the GPU in one wave at two CTAs per SM.
static bool use_cluster_kernel(const oda_kv* kv, const oda_visibility& vis, const DeviceInfo& di,
                               int G) {
  if (vis.mode != ODA_MODE_LOCAL) return false;
  const long long pages = (vis.sink + kPage - 1) / kPage + (long long)(vis.window - 1) / kPage + 2;
  const long long clusters = (long long)kv->batch * kv->num_kv_heads;
  return pages <= kLocalClusterPages && clusters * kLocalCtas <= 2ll * di.sms &&
         clusters <= g_max_clusters[di.device][G];
}

int check_visibility(const oda_kv* kv, const oda_visibility* v) {
  if (v == nullptr) return ODA_ERR_INVALID_ARG;
  if (!aligned_or_null(v->gate, 4) || !aligned_or_null(v->keep_blocks, 4) ||
      !aligned_or_null(v->keep_counts, 4) || !aligned_or_null(v->da_modes, 4) ||
      !aligned_or_null(v->da_focus_offsets, 4))
    return ODA_ERR_INVALID_ARG;
  switch (v->mode) {
    case ODA_MODE_LOCAL:
      return (v->sink < 0 || v->window < 1) ? ODA_ERR_INVALID_ARG : ODA_OK;
    case ODA_MODE_FULL:
      return ODA_OK;
    case ODA_MODE_KEEP:
      return (v->keep_blocks == nullptr || v->keep_counts == nullptr || v->max_keep < 0 ||
              v->max_keep > kv->max_blocks_per_seq)
                 ? ODA_ERR_INVALID_ARG
                 : ODA_OK;
    case ODA_MODE_DA:
      return (v->da_modes == nullptr || v->da_focus_offsets == nullptr || v->da_focus_len < 1 ||
              v->da_recent < 1 || v->da_local_len < 1)
                 ? ODA_ERR_INVALID_ARG
                 : ODA_OK;
    case ODA_MODE_SHARD:
      return (v->pos_lo < 0 || v->pos_hi <= v->pos_lo || v->pos_lo % kPage != 0 ||
              v->pos_hi % kPage != 0)
                 ? ODA_ERR_INVALID_ARG
                 : ODA_OK;
    default:
      return ODA_ERR_INVALID_ARG;
  }
}

static PlanArgs plan_args(const oda_kv* kv, const oda_visibility& v) {
  PlanArgs a;
  a.seq_lens = kv->seq_lens;
  a.block_table = kv->block_table;
  a.max_blocks = kv->max_blocks_per_seq;
  a.num_blocks = kv->num_blocks;
  a.mode = v.mode;
  a.sink = v.sink;
  a.window = v.window;
  a.gate = (v.mode == ODA_MODE_FULL || v.mode == ODA_MODE_SHARD) ? v.gate : nullptr;
  a.keep_blocks = v.keep_blocks;
  a.keep_counts = v.keep_counts;
  a.max_keep = v.max_keep;
  a.da_modes = v.da_modes;
  a.da_offsets = v.da_focus_offsets;
  a.da_focus_len = v.da_focus_len;
  a.da_recent = v.da_recent;
  a.da_local_len = v.da_local_len;
  a.pos_lo = v.pos_lo;
  a.pos_hi = v.pos_hi;
  return a;
}

oda_visibility visibility(int mode) {
  oda_visibility v = {};
  v.mode = mode;
  v.window = 1;
  return v;
}

int decode_params(const oda_kv* kv, const oda_visibility& vis, const void* q, int hq,
                  float scale, const void* k_new, const void* v_new, void* out, int out_dtype,
                  float* lse, void* ws, size_t ws_bytes, DecodeParams* pp) {
  int rc = check_kv(kv);
  if (rc != ODA_OK) return rc;
  if ((rc = check_visibility(kv, &vis)) != ODA_OK) return rc;
  int G = 0;
  if ((rc = group_of(kv, hq, &G)) != ODA_OK) return rc;
  if (out_dtype != ODA_F32 && out_dtype != ODA_BF16) return ODA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return ODA_ERR_INVALID_ARG;
  if ((k_new == nullptr) != (v_new == nullptr)) return ODA_ERR_INVALID_ARG;
  if (k_new != nullptr && (vis.mode == ODA_MODE_KEEP || vis.mode == ODA_MODE_DA))
    return ODA_ERR_INVALID_ARG;  // a kept set need not hold slot t
  if (kv->batch == 0) return ODA_OK;
  if (q == nullptr || out == nullptr || ws == nullptr) return ODA_ERR_INVALID_ARG;
  if (!aligned16(q) || (k_new && (!aligned16(k_new) || !aligned16(v_new))))
    return ODA_ERR_INVALID_ARG;
  if (!aligned16(ws) || !aligned_or_null(out, out_dtype == ODA_BF16 ? 2 : 4) ||
      !aligned_or_null(lse, 4))
    return ODA_ERR_INVALID_ARG;
  DeviceInfo di;
  if ((rc = current_device_info(&di)) != ODA_OK) return rc;
  const int grid = grid_size(di);
  const WsLayout wl = ws_layout(kv->batch, kv->num_kv_heads, G, grid);
  if (ws_bytes < wl.total) return ODA_ERR_WORKSPACE_TOO_SMALL;

  DecodeParams& p = *pp;
  p.plan = plan_args(kv, vis);
  p.k_cache = static_cast<const __nv_bfloat16*>(kv->k_cache);
  p.v_cache = static_cast<const __nv_bfloat16*>(kv->v_cache);
  p.k_cache_w = static_cast<__nv_bfloat16*>(kv->k_cache);
  p.v_cache_w = static_cast<__nv_bfloat16*>(kv->v_cache);
  p.batch = kv->batch;
  p.hkv = kv->num_kv_heads;
  p.hq = hq;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = out;
  p.out_bf16 = out_dtype == ODA_BF16;
  p.lse = lse;
  unsigned char* w = static_cast<unsigned char*>(ws);
  p.ws_o = reinterpret_cast<float*>(w + wl.o_off);
  p.ws_lse = reinterpret_cast<float*>(w + wl.lse_off);
  p.ws_ticket = reinterpret_cast<unsigned*>(w + wl.ticket_off);
  p.status = kv->dev_status;
  p.stats = kv->stats;
  p.wait_first = 0;
  p.wait_ns = test_wait_ns();
  p.test_stall = test_stall() == ODA_STALL_DECODE_RING ? 1
                 : test_stall() == ODA_STALL_LOCAL_PUSH ? 2
                                                         : 0;
  return ODA_OK;
}

int launch_decode(const oda_kv* kv, const oda_visibility& vis, const void* q, int hq,
                  float scale, const void* k_new, const void* v_new, void* out, int out_dtype,
                  float* lse, void* ws, size_t ws_bytes, void* stream, int pdl, int wait_first) {
  DecodeParams p;
  int rc = decode_params(kv, vis, q, hq, scale, k_new, v_new, out, out_dtype, lse, ws, ws_bytes,
                         &p);
  if (rc != ODA_OK || kv->batch == 0) return rc;
  p.wait_first = wait_first;
  const int G = hq / kv->num_kv_heads;
  DeviceInfo di;
  if ((rc = current_device_info(&di)) != ODA_OK) return rc;
  const int grid = grid_size(di);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t smem = decode_smem_bytes(G);
  switch (G) {  // attributes and the cluster capacity first
    case 1: rc = prepare_decode_kernel<1>(di.device); break;
    case 2: rc = prepare_decode_kernel<2>(di.device); break;
    default: rc = prepare_decode_kernel<4>(di.device); break;
  }
  if (rc != ODA_OK) return rc;
  const bool cluster = use_cluster_kernel(kv, vis, di, G);
  const int cgrid = kv->batch * kv->num_kv_heads * kLocalCtas;
  cudaError_t e;
  switch (G) {
    case 1:
      e = cluster ? launch_cluster_kernel<1>(p, cgrid, st, pdl != 0)
                  : launch_decode_kernel<1>(p, grid, smem, st, pdl != 0);
      break;
    case 2:
      e = cluster ? launch_cluster_kernel<2>(p, cgrid, st, pdl != 0)
                  : launch_decode_kernel<2>(p, grid, smem, st, pdl != 0);
      break;
    default:
      e = cluster ? launch_cluster_kernel<4>(p, cgrid, st, pdl != 0)
                  : launch_decode_kernel<4>(p, grid, smem, st, pdl != 0);
      break;
  }
  return cuda_status(e);
}

}  // namespace oda

using namespace oda;

namespace oda {
int decode_ws_layout(int batch, int hkv, int hq, size_t* total, size_t* ticket_off) {
  if (batch < 0 || hkv < 1 || hq < 1 || hq % hkv != 0 || hq / hkv > kMaxGroup)
    return ODA_ERR_UNSUPPORTED_SHAPE;
  DeviceInfo di;
  const int rc = current_device_info(&di);
  if (rc != ODA_OK) return rc;
  const WsLayout wl = ws_layout(batch, hkv, hq / hkv, grid_size(di));
  *total = wl.total;
  *ticket_off = wl.ticket_off;
  return ODA_OK;
}

int decode_ws_chain_offset(int batch, int hkv, int hq, size_t* total, size_t* chain_off) {
  if (batch < 0 || hkv < 1 || hq < 1 || hq % hkv != 0 || hq / hkv > kMaxGroup)
    return ODA_ERR_UNSUPPORTED_SHAPE;
  DeviceInfo di;
  const int rc = current_device_info(&di);
  if (rc != ODA_OK) return rc;
  const WsLayout wl = ws_layout(batch, hkv, hq / hkv, grid_size(di));
  *total = wl.total;
  *chain_off = wl.chain_off;
  return ODA_OK;
}
}  // namespace oda

extern "C" int oda_decode_workspace_size(int32_t batch, int32_t num_kv_heads,
                                         int32_t num_q_heads, size_t* bytes) {
  if (bytes == nullptr || batch < 0 || num_kv_heads < 1 || num_q_heads < 1)
    return ODA_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads != 0) return ODA_ERR_UNSUPPORTED_SHAPE;
  const int G = num_q_heads / num_kv_heads;
  if (G > kMaxGroup) return ODA_ERR_UNSUPPORTED_SHAPE;
  DeviceInfo di;
  const int rc = current_device_info(&di);
  if (rc != ODA_OK) return rc;
  *bytes = ws_layout(batch, num_kv_heads, G, grid_size(di)).total;
  return ODA_OK;
}

extern "C" int oda_decode(const oda_kv* kv, const oda_visibility* vis, const void* q,
                          int32_t num_q_heads, float scale, const void* k_new, const void* v_new,
                          void* out, int32_t out_dtype, float* lse, void* ws, size_t ws_bytes,
                          void* stream) {
  if (vis == nullptr) return ODA_ERR_INVALID_ARG;
  return launch_decode(kv, *vis, q, num_q_heads, scale, k_new, v_new, out, out_dtype, lse, ws,
                       ws_bytes, stream, 0, 0);
}

extern "C" int oda_decode_local(const oda_kv* kv, const void* q, int32_t num_q_heads,
                                int32_t sink, int32_t window, float scale, const void* k_new,
                                const void* v_new, void* out, int32_t out_dtype, float* lse,
                                void* ws, size_t ws_bytes, void* stream) {
  oda_visibility v = visibility(ODA_MODE_LOCAL);
  v.sink = sink;
  v.window = window;
  return launch_decode(kv, v, q, num_q_heads, scale, k_new, v_new, out, out_dtype, lse, ws,
                       ws_bytes, stream, 0, 0);
}

extern "C" int oda_decode_full(const oda_kv* kv, const void* q, int32_t num_q_heads, float scale,
                               const int32_t* gate, const void* k_new, const void* v_new,
                               void* out, int32_t out_dtype, float* lse, void* ws,
                               size_t ws_bytes, void* stream) {
  oda_visibility v = visibility(ODA_MODE_FULL);
  v.gate = gate;
  return launch_decode(kv, v, q, num_q_heads, scale, k_new, v_new, out, out_dtype, lse, ws,
                       ws_bytes, stream, 0, 0);
}

extern "C" int oda_decode_blockmask(const oda_kv* kv, const void* q, int32_t num_q_heads,
                                    float scale, const int32_t* keep_blocks,
                                    const int32_t* keep_counts, int32_t max_keep, void* out,
                                    int32_t out_dtype, float* lse, void* ws, size_t ws_bytes,
                                    void* stream) {
  oda_visibility v = visibility(ODA_MODE_KEEP);
  v.keep_blocks = keep_blocks;
  v.keep_counts = keep_counts;
  v.max_keep = max_keep;
  return launch_decode(kv, v, q, num_q_heads, scale, nullptr, nullptr, out, out_dtype, lse, ws,
                       ws_bytes, stream, 0, 0);
}

extern "C" int oda_visible_mask_ex(const oda_kv* kv, const oda_visibility* vis, uint8_t* mask,
                                   int32_t max_tokens, void* stream) {
  int rc = check_kv(kv);
  if (rc != ODA_OK) return rc;
  if ((rc = check_visibility(kv, vis)) != ODA_OK) return rc;
  if (max_tokens < 0 || (max_tokens > 0 && kv->batch > 0 && mask == nullptr))
    return ODA_ERR_INVALID_ARG;
  if (kv->batch == 0 || max_tokens == 0) return ODA_OK;
  visible_mask_kernel<<<kv->batch, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      plan_args(kv, *vis), mask, max_tokens, kv->dev_status);
  return cuda_status(cudaGetLastError());
}

extern "C" int oda_visible_mask(const oda_kv* kv, int32_t mode, int32_t sink, int32_t window,
                                const int32_t* gate, const int32_t* keep_blocks,
                                const int32_t* keep_counts, int32_t max_keep, uint8_t* mask,
                                int32_t max_tokens, void* stream) {
  if (mode != ODA_MODE_LOCAL && mode != ODA_MODE_FULL && mode != ODA_MODE_KEEP)
    return ODA_ERR_INVALID_ARG;
  oda_visibility v = visibility(mode);
  v.sink = sink;
  v.window = window;
  v.gate = gate;
  v.keep_blocks = keep_blocks;
  v.keep_counts = keep_counts;
  v.max_keep = max_keep;
  return oda_visible_mask_ex(kv, &v, mask, max_tokens, stream);
}

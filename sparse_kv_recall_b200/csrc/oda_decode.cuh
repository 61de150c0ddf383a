// Device pieces of the paged decode kernels (oda_decode.cu, oda_chain.cu): the split
// work plan, the page step (CUDA-core or tensor-core scores, online softmax, P.V), the commit
// of slot t, the merges, and the whole split decode pass over one layer.
//
// Lane layout for a 16 x 128 page: lane = 16 * half + li; lane li owns dims [8 li, 8 li + 8)
// of rows 2k + half, k = 0..7, for P.V. The CUDA-core scores (the cluster kernels, and
// decode_pass<1>) are reduced over the 16 lanes of a half by a reduce-scatter butterfly,
// after which lane li holds row 2 (li / 2) + half for heads (li % 2) * G / 2 + u;
// decode_pass<2> and <4> form the scores on the tensor cores (page_step_mma).
#pragma once

#include <math.h>

#include "oda_internal.h"
#include "oda_plan.cuh"

namespace oda {
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;   // == kHeadDim: merges map one thread to one dim
constexpr int kStages = 3;
constexpr int kStageBytes = 2 * kPageBytes;
constexpr int kCtasPerSm = 2;
constexpr int kMaxBatch = 1024;
constexpr int kMaxGroup = 4;
constexpr int kMinShare = 4;            // units per CTA at least (one page per warp)

static_assert(kThreads == kHeadDim, "merge maps one thread per output dim");

struct DecodeParams {
  PlanArgs plan;
  const __nv_bfloat16* k_cache;
  const __nv_bfloat16* v_cache;
  __nv_bfloat16* k_cache_w;
  __nv_bfloat16* v_cache_w;
  int batch, hkv, hq;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_new;  // nullable: commit at slot t
  const __nv_bfloat16* v_new;
  float scale_log2;            // scale * log2(e): scores are kept in base-2 units
  void* out;
  int out_bf16;
  float* lse;
  float* ws_o;                 // [slots][G][128]
  float* ws_lse;               // [slots][G], base-2 log-sum
  unsigned int* ws_ticket;     // [batch * hkv]
  int* status;
  unsigned long long* stats;
  int wait_first;              // 1: the previous kernel may still write the gate: wait at once
  unsigned long long wait_ns;  // limit of every bounded wait (kWaitNs unless a test sets it)
  int test_stall;              // test hook: 1 = CTA 0's warp 0 arms its first stage for bytes
                               // that no copy delivers, so that its bounded wait runs out;
                               // 2 = the Local cluster kernel's first cluster's rank 1
                               // withholds its partial, so that rank 0's inbox wait runs out
};

// ---- reduce-scatter of C values over the 16 lanes of a half-warp ------------------------
// After the call, v[0 .. max(C/16, 1)) of lane li hold the sums of the original value
// indices li * (C / 16) + u (for C < 16 the last steps are plain all-reduces).
template <int C, int O>
__device__ __forceinline__ void reduce_scatter(float* v, int lane) {
  if constexpr (O >= 1) {
    if constexpr (C > 1) {
      const bool up = (lane & O) != 0;
#pragma unroll
      for (int j = 0; j < C / 2; ++j) {
        const float send = up ? v[j] : v[j + C / 2];
        const float keep = up ? v[j + C / 2] : v[j];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, O);
      }
      reduce_scatter<C / 2, O / 2>(v, lane);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
      reduce_scatter<1, O / 2>(v, lane);
    }
  }
}

template <int G>
struct Vpl {
  static constexpr int value = G >= 2 ? G / 2 : 1;  // softmax values each lane owns
};

// Packed fp32 pairs: sm_100's fma.rn.f32x2 / mul.rn.f32x2 run two independent fp32 lanes per
// instruction, each rounded exactly as fmaf / __fmul_rn would round it.
typedef unsigned long long f2_t;

__device__ __forceinline__ f2_t f2_pack(float lo, float hi) {
  f2_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(f2_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f2_t f2_fma(f2_t a, f2_t b, f2_t c) {
  f2_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f2_t f2_mul(f2_t a, f2_t b) {
  f2_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// A bf16 pair (low half = lower index) widened exactly to an fp32 pair.
__device__ __forceinline__ f2_t bf16x2_widen(uint32_t w) {
  return f2_pack(bf16lo(w), bf16hi(w));
}

// One page: scores, online-softmax update, P.V accumulation. q2[gg][j] holds the scaled
// query dims (8 li + 2j, 8 li + 2j + 1) of head gg; acc[gg][j] the same dims of its P.V sum.
template <int G>
__device__ __forceinline__ void page_step(const unsigned char* stage, const f2_t (&q2)[G][4],
                                          float (&m_run)[Vpl<G>::value],
                                          float (&l_run)[Vpl<G>::value], f2_t (&acc)[G][4],
                                          float* ps, const SeqPlan& sp, int lp, int lane,
                                          unsigned& rows_vis) {
  constexpr int VPL = Vpl<G>::value;
  const int half = lane >> 4, li = lane & 15;
  const uint4* K = reinterpret_cast<const uint4*>(stage);
  const uint4* V = reinterpret_cast<const uint4*>(stage + kPageBytes);

  float sc[8 * G];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint4 kw = K[(2 * k + half) * 16 + li];
    const f2_t kp[4] = {bf16x2_widen(kw.x), bf16x2_widen(kw.y), bf16x2_widen(kw.z),
                        bf16x2_widen(kw.w)};
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      // even and odd dims accumulate in the two lanes of a pair, then add
      f2_t s2 = f2_mul(q2[gg][0], kp[0]);
#pragma unroll
      for (int j = 1; j < 4; ++j) s2 = f2_fma(q2[gg][j], kp[j], s2);
      float lo, hi;
      f2_unpack(s2, lo, hi);
      sc[k * G + gg] = lo + hi;
    }
  }
  reduce_scatter<8 * G, 8>(sc, lane);

  const int myk = li >> 1;
  const bool vis = row_visible(sp, lp * kPage + 2 * myk + half);
  rows_vis += __popc(__ballot_sync(0xffffffffu, vis) & 0x55555555u);

  float* pshare = ps;                 // [2 halves][8 rows][G]
  float* ashare = ps + 16 * G;        // [2 halves][G]
#pragma unroll
  for (int u = 0; u < VPL; ++u) {
    const float v = vis ? sc[u] : -INFINITY;
    float mx = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mnew = fmaxf(m_run[u], mx);
    const float pr = (v == -INFINITY) ? 0.f : ex2_fast(v - mnew);
    const float al = (m_run[u] == mnew) ? 1.f : ex2_fast(m_run[u] - mnew);
    l_run[u] = l_run[u] * al + pr;
    m_run[u] = mnew;
    const int gh = (G >= 2) ? ((li & 1) * (G / 2) + u) : 0;
    if (G >= 2 || (li & 1) == 0) {
      pshare[(half * 8 + myk) * G + gh] = pr;
      if (myk == 0) ashare[half * G + gh] = al;
    }
  }
  __syncwarp();

#pragma unroll
  for (int gg = 0; gg < G; ++gg) {
    const float al = ashare[half * G + gg];
    const f2_t al2 = f2_pack(al, al);
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[gg][j] = f2_mul(acc[gg][j], al2);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint4 vw = V[(2 * k + half) * 16 + li];
    const f2_t vp[4] = {bf16x2_widen(vw.x), bf16x2_widen(vw.y), bf16x2_widen(vw.z),
                        bf16x2_widen(vw.w)};
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      const float pk = pshare[(half * 8 + k) * G + gg];
      const f2_t pp = f2_pack(pk, pk);
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[gg][j] = f2_fma(pp, vp[j], acc[gg][j]);
    }
  }
  __syncwarp();
}

// ---- G = 2, 4: page scores on the tensor cores -----------------------------------------
// With four query heads per KV head the CUDA-core page step above is bound by instruction
// issue (about twice the FMAs of G = 2 and a 32-value reduce-scatter), so decode_kernel<4>
// and decode_kernel<2> form the scores with mma.sync m16n8k16 (bf16 operands, fp32
// accumulation; the products of two bf16 values are exact in fp32): A = the page's 16 K rows,
// B = the group's query heads as 8 columns (columns G..7 zero), C = 16 tokens x 8 heads,
// eight k-steps of 16 dims.
// Lane (gid = lane / 4, tig = lane % 4) supplies tokens gid and gid + 8 and the 16-byte dim
// chunks tig + 4 j (j < 4) of them. Inside a chunk the k order is chosen so that each A and B
// register is one 32-bit word of those chunks: k-step 2 j + h takes words 2 h and 2 h + 1 of
// chunk tig + 4 j (rows gid and gid + 8 for A, head gid for B). No shuffles or transposes;
// the 16-byte shared loads of a quarter-warp hit at most two lanes per bank group. The lane
// then holds the scores of tokens gid and gid + 8 for heads 2 tig and 2 tig + 1; softmax
// weights go to the same shared exchange as above and P.V stays on the CUDA cores.
template <int G>
struct MmaScores {
  static constexpr bool value = G == 4 || G == 2;
};

__device__ __forceinline__ void mma_16816_bf16(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The query of head gid of group (b, g) as B fragments: chunks tig + 4 j, zero for gid >= G.
template <int G>
__device__ __forceinline__ void load_q_mma(const __nv_bfloat16* q, int lane, uint4 (&qv)[4]) {
  const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    qv[j] = gid < G ? *reinterpret_cast<const uint4*>(q + gid * kHeadDim + 8 * (tig + 4 * j))
                    : make_uint4(0u, 0u, 0u, 0u);
}

// A group's running maximum is raised only when a score exceeds it by more than this many
// base-2 units, so the rescale of the accumulators is rare; unnormalised weights stay below
// 2^kLazyMax, far inside fp32 range. (m, l, acc) keep their meaning: acc and l are sums of
// 2^(s - m) with m the same for every lane that holds a head.
constexpr float kLazyMax = 8.f;

// One page for G = 2 or 4. m_run[u], l_run[u] belong to head 2 tig + u (l_run: this lane's
// tokens only; lanes with 2 tig >= G hold no head); acc is the half-warp P.V layout of
// page_step.
template <int G>
__device__ __forceinline__ void page_step_mma(const unsigned char* stage, const uint4 (&qv)[4],
                                              float scale_log2, float (&m_run)[2],
                                              float (&l_run)[2], f2_t (&acc)[G][4], float* ps,
                                              const SeqPlan& sp, int lp, int lane,
                                              unsigned& rows_vis) {
  static_assert(G == 4 || G == 2, "tensor-core scores serve two or four heads per KV head");
  const int gid = lane >> 2, tig = lane & 3;
  const unsigned char* k0 = stage + gid * kRowBytes + 16 * tig;
  const unsigned char* k1 = k0 + 8 * kRowBytes;
  float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 ka = *reinterpret_cast<const uint4*>(k0 + 64 * j);
    const uint4 kb = *reinterpret_cast<const uint4*>(k1 + 64 * j);
    mma_16816_bf16(c, ka.x, kb.x, ka.y, kb.y, qv[j].x, qv[j].y);
    mma_16816_bf16(c, ka.z, kb.z, ka.w, kb.w, qv[j].z, qv[j].w);
  }
  const bool v0 = row_visible(sp, lp * kPage + gid);
  const bool v1 = row_visible(sp, lp * kPage + gid + 8);
  rows_vis += __popc(__ballot_sync(0xffffffffu, v0) & 0x11111111u) +
              __popc(__ballot_sync(0xffffffffu, v1) & 0x11111111u);
  const bool head_ok = 2 * tig < G;  // columns 2 tig, 2 tig + 1 are real heads
  float s[2][2];                     // [token gid, gid + 8][head 2 tig + u]
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    s[0][u] = v0 ? c[u] * scale_log2 : -INFINITY;
    s[1][u] = v1 ? c[2 + u] * scale_log2 : -INFINITY;
  }
  float* pshare = ps;           // [2 halves][8 rows][G], as page_step
  float* ashare = ps + 16 * G;  // [G] rescale factors (written when a maximum is raised)
  bool raise = false;
#pragma unroll
  for (int u = 0; u < 2; ++u) raise |= head_ok && fmaxf(s[0][u], s[1][u]) > m_run[u] + kLazyMax;
  const bool raised = __any_sync(0xffffffffu, raise);
  if (raised) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float mx = fmaxf(s[0][u], s[1][u]);  // page maximum of the head over the 8 gid lanes
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const bool up = mx > m_run[u] + kLazyMax;
      const float al = !up ? 1.f : (m_run[u] == -INFINITY ? 0.f : ex2_fast(m_run[u] - mx));
      if (up) m_run[u] = mx;
      l_run[u] *= al;
      if (head_ok && gid == 0) ashare[2 * tig + u] = al;
    }
  }
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int r = gid + 8 * t;
    const int slot = (r & 1) * 8 + (r >> 1);  // page_step's [half][k] order of row r
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float pr = (s[t][u] == -INFINITY) ? 0.f : ex2_fast(s[t][u] - m_run[u]);
      l_run[u] += pr;
      if (head_ok) pshare[slot * G + 2 * tig + u] = pr;
    }
  }
  __syncwarp();

  const int half = lane >> 4, li = lane & 15;
  if (raised) {
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      const float al = ashare[gg];
      const f2_t al2 = f2_pack(al, al);
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[gg][j] = f2_mul(acc[gg][j], al2);
    }
  }
  const uint4* V = reinterpret_cast<const uint4*>(stage + kPageBytes);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint4 vw = V[(2 * k + half) * 16 + li];
    const f2_t vp[4] = {bf16x2_widen(vw.x), bf16x2_widen(vw.y), bf16x2_widen(vw.z),
                        bf16x2_widen(vw.w)};
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      const float pk = pshare[(half * 8 + k) * G + gg];
      const f2_t pp = f2_pack(pk, pk);
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[gg][j] = f2_fma(pp, vp[j], acc[gg][j]);
    }
  }
  __syncwarp();
}

__device__ __forceinline__ void store_out(const DecodeParams& p, size_t idx, float v) {
  if (p.out_bf16)
    reinterpret_cast<__nv_bfloat16*>(p.out)[idx] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(p.out)[idx] = v;
}

// Final output of query heads g*G .. g*G+G-1 of sequence b; thread tid writes dim tid.
template <int G>
__device__ __forceinline__ void write_final(const DecodeParams& p, int b, int g,
                                            const float (&o)[G], const float (&lse2)[G]) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int gg = 0; gg < G; ++gg) {
    const size_t h = (size_t)b * p.hq + g * G + gg;
    store_out(p, h * kHeadDim + tid, o[gg]);
    if (p.lse != nullptr && tid == 0)
      p.lse[h] = (lse2[gg] == -INFINITY) ? -INFINITY : lse2[gg] * 0.69314718055994531f;
  }
}

// CTA whose share contains flattened unit x (shares are [c*T/P, (c+1)*T/P), P <= T).
__device__ __forceinline__ int cta_of(long long x, long long T, int P) {
  return (int)(((x + 1) * P - 1) / T);
}

// ---------------------------------------------------------------------------------------
// The split decode pass over one layer (decode_kernel runs one, full_chain_kernel one per
// layer on the same rings).
//
// Work decomposition. Every sequence b contributes npages(b) visible pages per KV head; the
// flattened list of (b, KV head g, page j) units is cut into equal contiguous shares, one per
// CTA. A share may cover part of one (b, g) or the ends of several. Inside a CTA each of the
// 4 warps streams every 4th page of the current (b, g) piece through its own 3-stage ring of
// shared-memory stages filled by 1-D bulk copies (TMA engine, 4 KB K page + 4 KB V page per
// stage), and keeps an online softmax for all G = Hq / Hkv query heads that share the KV
// head, so each page is read from HBM once for the whole group. A piece's 8 half-warp states
// are merged in shared memory; if the (b, g) spans several CTAs, each writes its normalised
// partial (O, log2-sum) to the workspace and the last to arrive (atomic ticket) merges them
// in fixed order.
// ---------------------------------------------------------------------------------------

// Shared memory of a split-decode CTA.
struct SplitSmem {
  unsigned char* stages;      // [kWarps][kStages][kStageBytes]; merge scratch between pieces
  uint64_t* bars;             // [kWarps][kStages]
  float* pscratch;            // [kWarps][18 G]: per-warp softmax exchange
  int* pre;                   // [batch + 1]: prefix of unit counts per sequence
  int* s_align;               // CTA-count granularity that keeps shares inside one (b, g)
  int* s_last;
  unsigned long long* s_rows; // counter updates gathered per piece
  unsigned long long* s_pages;
};

constexpr size_t split_smem_bytes(int G) {
  return (size_t)kWarps * kStages * kStageBytes + (size_t)kWarps * kStages * sizeof(uint64_t) +
         (size_t)kWarps * 18 * G * sizeof(float) + (size_t)(kMaxBatch + 1) * sizeof(int);
}

template <int G>
__device__ __forceinline__ SplitSmem split_smem(unsigned char* smem, int* s_align, int* s_last,
                                                unsigned long long* s_rows,
                                                unsigned long long* s_pages) {
  SplitSmem sm;
  sm.stages = smem;
  sm.bars = reinterpret_cast<uint64_t*>(smem + kWarps * kStages * kStageBytes);
  sm.pscratch = reinterpret_cast<float*>(sm.bars + kWarps * kStages);
  sm.pre = reinterpret_cast<int*>(sm.pscratch + kWarps * 18 * G);
  sm.s_align = s_align;
  sm.s_last = s_last;
  sm.s_rows = s_rows;
  sm.s_pages = s_pages;
  return sm;
}

// Ring barriers (once per launch) and the per-sequence prefix of visible units with the
// share alignment (once per plan). Ends with a CTA barrier; returns the total unit count.
__device__ __forceinline__ long long split_prologue(const PlanArgs& plan, int B, int Hkv,
                                                    const SplitSmem& sm, int* status) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) mbar_init(&sm.bars[warp * kStages + s], 1);
    fence_barrier_init();
  }
  if (tid == 0) {
    *sm.s_rows = 0;
    *sm.s_pages = 0;
    sm.pre[0] = 0;
  }
  for (int b = tid; b < B; b += kThreads) {
    const SeqPlan sp = make_plan(plan, b);
    sm.pre[b + 1] = sp.npages * Hkv;
    if (blockIdx.x == 0 && sp.err != 0) report(status, sp.err);
  }
  __syncthreads();
  if (warp == 0) {  // inclusive scan of the per-sequence unit counts
    int carry = 0;
    unsigned vmin = 0xffffffffu, vmax = 0u, active = 0u;
    for (int base = 0; base < B; base += 32) {
      const int i = base + lane;
      int v = i < B ? sm.pre[i + 1] : 0;
      const unsigned nz = (i < B && v > 0) ? (unsigned)v : 0u;
      vmin = min(vmin, __reduce_min_sync(0xffffffffu, nz ? nz : 0xffffffffu));
      vmax = max(vmax, __reduce_max_sync(0xffffffffu, nz));
      active += __popc(__ballot_sync(0xffffffffu, nz != 0u));
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
      }
      v += carry;
      if (i < B) sm.pre[i + 1] = v;
      carry = __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) *sm.s_align = (active > 0 && vmin == vmax) ? (int)active * Hkv : 0;
  }
  __syncthreads();
  return sm.pre[B];
}

// Ring position a CTA carries from one pass to the next, and whether a bounded wait gave up.
struct RingState {
  unsigned wcount;  // pages this warp has consumed, over all pieces and passes
  bool dead;        // stop touching the ring
  bool aborted;     // dep_wait() answered false: the pass was left (uniform over the CTA)
};

// One decode pass of this CTA over its share of the T units. dep_wait() is called (it must be
// idempotent) after the first pages of the first piece are requested and before anything
// reads q / k_new / v_new, the gate or writes global memory; it returns false (the same
// answer in every thread of the CTA) when the launch is being abandoned, and the pass then
// returns with rs.aborted set.
template <int G, class Wait>
__device__ __forceinline__ void decode_pass(const DecodeParams& p, const SplitSmem& sm,
                                            long long T, RingState& rs, Wait& dep_wait) {
  constexpr int VPL = MmaScores<G>::value ? 2 : Vpl<G>::value;  // softmax states per lane
  constexpr int kPs = 18 * G;  // per-warp softmax exchange: 16 G weights + 2 G rescales
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int li = lane & 15;
  const int B = p.batch, Hkv = p.hkv;
  const int P = gridDim.x, c = blockIdx.x;
  const int* pre = sm.pre;
  unsigned char* stages = sm.stages;

  const uint64_t policy = l2_evict_first_policy();
  unsigned char* wst = stages + warp * kStages * kStageBytes;
  uint64_t* wbar = sm.bars + warp * kStages;
  float* ps = sm.pscratch + warp * kPs;
  unsigned rows_vis = 0, pages_read = 0;

  // Shares go to the first Pe <= min(P, ceil(T / kMinShare)) CTAs only, so that every CTA
  // holding a share has at least one unit (and the CTAs that touch a (b, g) form a contiguous
  // index range), and small launches do not fan a (b, g) out over more CTAs than they need.
  int Pe = (int)min((long long)P, (T + kMinShare - 1) / kMinShare);
  // When every non-empty sequence has the same page count, a multiple of (non-empty
  // sequences x Hkv) CTAs makes every share fall inside one (b, g), so no CTA has to finish
  // one piece before it can start streaming the next. Rounding up (when the grid has the
  // CTAs) rather than down keeps the largest share at ceil(T / Pe) <= kMinShare units, i.e.
  // at most one page per warp, so no warp of a short launch holds up its (b, g)'s merge.
  // Rounding up never exceeds T: T = s_align x (pages per sequence).
  const int s_align = *sm.s_align;
  if (s_align > 0) {
    const int up = (Pe + s_align - 1) / s_align * s_align;
    if (up <= P) Pe = up;
    else if (Pe >= s_align) Pe -= Pe % s_align;
  }
  long long x = c < Pe ? (T * c) / Pe : 0;
  const long long x_end = c < Pe ? (T * (c + 1)) / Pe : 0;
  while (x < x_end) {
    int lo = 0, hi = B - 1;  // largest b with pre[b] <= x
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= x) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int npg = (pre[b + 1] - pre[b]) / Hkv;
    const long long off = x - pre[b];
    const int g = (int)(off / npg);
    const int j0 = (int)(off - (long long)g * npg);
    const long long seg0 = pre[b] + (long long)g * npg;
    const long long seg1 = seg0 + npg;
    const long long xe = min(x_end, seg1);
    const int j1 = j0 + (int)(xe - x);
    const SeqPlan sp = make_plan(p.plan, b);
    const int bg = b * Hkv + g;
    const size_t head_off = (size_t)g * (kPage * kHeadDim);
    const size_t page_stride = (size_t)Hkv * kPage * kHeadDim;

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
      for (int j = 0; j < 4; ++j) acc[gg][j] = f2_pack(0.f, 0.f);

    const int first = j0 + warp;
    const int cnt = first < j1 ? (j1 - first + kWarps - 1) / kWarps : 0;
    const unsigned wcount = rs.wcount;

    // lane 0 starts page n of this piece into stage (wcount + n) % kStages
    auto issue = [&](int n) {
      const int j = first + n * kWarps;
      const PageRef r = page_ref(p.plan, sp, b, j);
      uint64_t* bar = &wbar[(wcount + n) % kStages];
      unsigned char* dst = wst + ((wcount + n) % kStages) * kStageBytes;
      if (p.test_stall == 1 && c == 0 && warp == 0 && wcount + n == 0) {
        mbar_arrive_expect_tx(bar, 16u);  // test hook: bytes that never arrive
      } else if (r.err == 0) {
        const size_t src = (size_t)r.pb * page_stride + head_off;
        mbar_arrive_expect_tx(bar, kStageBytes);
        bulk_load(dst, p.k_cache + src, kPageBytes, bar, policy);
        bulk_load(dst + kPageBytes, p.v_cache + src, kPageBytes, bar, policy);
      } else {
        report(p.status, r.err);
        mbar_arrive(bar);
      }
    };

    if (!rs.dead && lane == 0)
      for (int n = 0; n < min(cnt, kStages); ++n) issue(n);
    __syncwarp();
    if (!dep_wait()) {
      // The launch is being abandoned (a persistent kernel's wait ran out; the answer is the
      // same for the whole CTA): let the copies just issued land, then leave the pass.
      if (!rs.dead)
        for (int n = 0; n < min(cnt, kStages); ++n)
          mbar_wait(&wbar[(wcount + n) % kStages], ((wcount + n) / kStages) & 1u, p.wait_ns);
      rs.dead = true;
      rs.aborted = true;
      return;
    }

    f2_t q2[G][4];  // CUDA-core scores: scaled query dims 8 li .. 8 li + 7 of every head
    uint4 qv[4];    // tensor-core scores: B fragments
    if constexpr (MmaScores<G>::value) {
      load_q_mma<G>(p.q + ((size_t)b * p.hq + g * G) * kHeadDim, lane, qv);
    } else {
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        const uint4 qw = *reinterpret_cast<const uint4*>(
            p.q + ((size_t)b * p.hq + g * G + gg) * kHeadDim + 8 * li);
        float qf[8];
        unpack8(qw, qf);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          q2[gg][j] = f2_pack(qf[2 * j] * p.scale_log2, qf[2 * j + 1] * p.scale_log2);
      }
    }

    for (int n = 0; n < cnt && !rs.dead; ++n) {
      const unsigned k = wcount + n;
      const int stage = k % kStages;
      const PageRef r = page_ref(p.plan, sp, b, first + n * kWarps);
      if (!__all_sync(0xffffffffu, mbar_wait(&wbar[stage], (k / kStages) & 1u, p.wait_ns))) {
        if (lane == 0) report(p.status, ODA_DEV_TIMEOUT);
        // let the copies already started into the other stages land, then stop
        for (int m = n + 1; m < min(cnt, n + kStages); ++m) {
          const unsigned km = wcount + m;
          mbar_wait(&wbar[km % kStages], (km / kStages) & 1u, p.wait_ns);
        }
        rs.dead = true;
        break;
      }
      if (r.err == 0) {
        unsigned char* st = wst + stage * kStageBytes;
        if (p.k_new != nullptr && r.lp == sp.t / kPage) {
          // Commit: the step's K/V take slot t, in the cache and in this page's copy.
          const int row = sp.t % kPage;
          const bool isk = lane < 16;
          const uint4 v = *reinterpret_cast<const uint4*>(
              (isk ? p.k_new : p.v_new) + ((size_t)b * Hkv + g) * kHeadDim + 8 * li);
          *reinterpret_cast<uint4*>(st + (isk ? 0 : kPageBytes) + row * kRowBytes + 16 * li) = v;
          __nv_bfloat16* dst = (isk ? p.k_cache_w : p.v_cache_w) + (size_t)r.pb * page_stride +
                               head_off + row * kHeadDim + 8 * li;
          *reinterpret_cast<uint4*>(dst) = v;
          fence_proxy_async_smem();  // this stage is refilled by a bulk copy later
          __syncwarp();
        }
        if constexpr (MmaScores<G>::value)
          page_step_mma<G>(st, qv, p.scale_log2, m_run, l_run, acc, ps, sp, r.lp, lane, rows_vis);
        else
          page_step<G>(st, q2, m_run, l_run, acc, ps, sp, r.lp, lane, rows_vis);
        ++pages_read;
      }
      __syncwarp();
      if (lane == 0 && n + kStages < cnt) issue(n + kStages);
      __syncwarp();
    }
    rs.wcount = wcount + cnt;

    // ---- merge the 8 half-warp states of this piece ----
    // State (warp, half) covers the page rows of parity `half`. Its softmax sum is spread over
    // the lanes that scored those rows: li bits 1..3 of a half (CUDA-core scores), or gid bits
    // 1..2 at a fixed gid parity and tig (tensor-core scores).
    float lsum[VPL];
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      float v = l_run[u];
      if constexpr (MmaScores<G>::value) {
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
      } else {
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
      }
      lsum[u] = v;
    }
    if (p.stats != nullptr && lane == 0 && (rows_vis | pages_read)) {
      atomicAdd(sm.s_rows, (unsigned long long)rows_vis);
      atomicAdd(sm.s_pages, (unsigned long long)pages_read);
    }
    rows_vis = 0;
    pages_read = 0;
    __syncthreads();  // every warp is done with its stages: reuse them as merge scratch
    if (p.stats != nullptr && tid == 0) {
      // issued now, so that the counter updates complete while the merge runs
      if (*sm.s_rows) atomicAdd(&p.stats[ODA_STAT_ROWS], *sm.s_rows);
      if (*sm.s_pages) atomicAdd(&p.stats[ODA_STAT_PAGES], *sm.s_pages);
      *sm.s_rows = 0;
      *sm.s_pages = 0;
    }
    float* Mw = reinterpret_cast<float*>(stages);  // [2 * kWarps][G]
    float* Lw = Mw + 2 * kWarps * G;               // [2 * kWarps][G]
    float* Aw = Lw + 2 * kWarps * G;               // [2 * kWarps][G][128]
    const int half = lane >> 4;
    const int sidx = warp * 2 + half;
    if constexpr (MmaScores<G>::value) {
      const int gid = lane >> 2, tig = lane & 3;  // lane gid < 2 holds rows of parity gid
      if (gid < 2 && 2 * tig < G) {
#pragma unroll
        for (int u = 0; u < VPL; ++u) {
          Mw[(warp * 2 + gid) * G + 2 * tig + u] = m_run[u];
          Lw[(warp * 2 + gid) * G + 2 * tig + u] = lsum[u];
        }
      }
    } else if (li < 2 && (G >= 2 || li == 0)) {
#pragma unroll
      for (int u = 0; u < VPL; ++u) {
        const int gh = (G >= 2) ? ((li & 1) * (G / 2) + u) : 0;
        Mw[sidx * G + gh] = m_run[u];
        Lw[sidx * G + gh] = lsum[u];
      }
    }
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      float4* dst = reinterpret_cast<float4*>(Aw + (sidx * G + gg) * kHeadDim + 8 * li);
      float a[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) f2_unpack(acc[gg][j], a[2 * j], a[2 * j + 1]);
      dst[0] = make_float4(a[0], a[1], a[2], a[3]);
      dst[1] = make_float4(a[4], a[5], a[6], a[7]);
    }
    __syncthreads();
    float o[G], l2[G];
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      float M = -INFINITY;
#pragma unroll
      for (int s = 0; s < 2 * kWarps; ++s) M = fmaxf(M, Mw[s * G + gg]);
      if (M == -INFINITY) {
        o[gg] = 0.f;
        l2[gg] = -INFINITY;
      } else {
        float L = 0.f, a = 0.f;
#pragma unroll
        for (int s = 0; s < 2 * kWarps; ++s) {
          const float ms = Mw[s * G + gg];
          const float w = (ms == -INFINITY) ? 0.f : ex2_fast(ms - M);
          L = fmaf(w, Lw[s * G + gg], L);
          a = fmaf(w, Aw[(s * G + gg) * kHeadDim + tid], a);
        }
        o[gg] = a * rcp_fast(L);
        l2[gg] = M + lg2_fast(L);
      }
    }

    const int c_first = cta_of(seg0, T, Pe);
    const int n_contrib = cta_of(seg1 - 1, T, Pe) - c_first + 1;
    if (n_contrib == 1) {
      write_final<G>(p, b, g, o, l2);
    } else {
      const size_t slot = (size_t)c + bg;
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        p.ws_o[(slot * G + gg) * kHeadDim + tid] = o[gg];
        if (tid == 0) p.ws_lse[slot * G + gg] = l2[gg];
      }
      __syncthreads();  // the CTA's partial is written; thread 0 publishes it (release)
      if (tid == 0) *sm.s_last = ticket_arrive(&p.ws_ticket[bg]) == (unsigned)(n_contrib - 1);
      __syncthreads();  // ... and the last CTA's thread 0 acquired everyone's partials
      if (*sm.s_last) {
        // Merge the n_contrib partials in fixed order: log-sums into shared memory (stage
        // memory is free again), per-head max and weights by one warp per head, then every
        // thread sums its dim over the partials with independent loads in flight. Partials
        // are staged through shared memory, as many at a time as the stage memory holds
        // (every one of a short launch's partials at once), by 16-byte asynchronous copies
        // all in flight together; the first chunk is requested along with the log-sums, so
        // one L2 round trip brings both.
        const size_t s0 = (size_t)c_first + bg;
        float* sw = reinterpret_cast<float*>(stages);  // [n_contrib][G] log-sums -> weights
        float* sml = sw + n_contrib * G;                // [G] max, [G] weight sum
        float* so = sml + 2 * G + (4 - (n_contrib * G + 2 * G) % 4) % 4;  // float4-aligned
        const int chunk = (int)((kWarps * kStages * kStageBytes -
                                 (size_t)(so - sw) * sizeof(float)) / (G * kHeadDim * sizeof(float)));
        const float4* src = reinterpret_cast<const float4*>(p.ws_o + s0 * G * kHeadDim);
        float4* dst4 = reinterpret_cast<float4*>(so);
        auto stage_chunk = [&](int s_lo) {  // issue only; cp_async_wait_all completes it
          const int n4 = min(chunk, n_contrib - s_lo) * G * kHeadDim / 4;
          const float4* src_c = src + (size_t)s_lo * G * kHeadDim / 4;
          for (int i = tid; i < n4; i += kThreads) cp_async16(dst4 + i, src_c + i);
        };
        stage_chunk(0);
        for (int i = tid; i < n_contrib * G; i += kThreads) sw[i] = __ldcg(&p.ws_lse[s0 * G + i]);
        cp_async_wait_all();
        __syncthreads();
        if (warp < G) {
          float m = -INFINITY;
          for (int s = lane; s < n_contrib; s += 32) m = fmaxf(m, sw[s * G + warp]);
#pragma unroll
          for (int o2 = 16; o2 >= 1; o2 >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o2));
          float sum = 0.f;
          for (int s = lane; s < n_contrib; s += 32) {
            const float ls = sw[s * G + warp];
            const float wgt = (ls == -INFINITY) ? 0.f : ex2_fast(ls - m);
            sw[s * G + warp] = wgt;
            sum += wgt;
          }
#pragma unroll
          for (int o2 = 16; o2 >= 1; o2 >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o2);
          if (lane == 0) {
            sml[warp] = m;
            sml[G + warp] = sum;
          }
        }
        __syncthreads();  // weights and the first chunk are in shared memory
        float a[G];
#pragma unroll
        for (int gg = 0; gg < G; ++gg) a[gg] = 0.f;
        for (int s_lo = 0; s_lo < n_contrib; s_lo += chunk) {
          const int ns = min(chunk, n_contrib - s_lo);
          if (s_lo > 0) {
            __syncthreads();  // everyone is done with the previous chunk
            stage_chunk(s_lo);
            cp_async_wait_all();
            __syncthreads();
          }
          for (int s = 0; s < ns; ++s)
#pragma unroll
            for (int gg = 0; gg < G; ++gg)
              a[gg] = fmaf(sw[(s_lo + s) * G + gg], so[(s * G + gg) * kHeadDim + tid], a[gg]);
        }
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
          const float M = sml[gg], L = sml[G + gg];
          if (M == -INFINITY) {
            o[gg] = 0.f;
            l2[gg] = -INFINITY;
          } else {
            o[gg] = a[gg] * rcp_fast(L);
            l2[gg] = M + lg2_fast(L);
          }
        }
        write_final<G>(p, b, g, o, l2);
        if (tid == 0) p.ws_ticket[bg] = 0u;  // leave the workspace zeroed
      }
    }
    fence_proxy_async_smem();  // merge scratch is the next piece's stage memory
    __syncthreads();
    x = xe;
  }

  // Sequences with nothing visible (bad length, empty keep list) but not gated off.
  if (!dep_wait()) {
    rs.aborted = true;
    return;
  }
  for (int bg = c; bg < B * Hkv; bg += P) {
    const int b = bg / Hkv;
    if (pre[b + 1] == pre[b] && !(p.plan.gate != nullptr && p.plan.gate[b] == 0)) {
      float o[G], l2[G];
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        o[gg] = 0.f;
        l2[gg] = -INFINITY;
      }
      write_final<G>(p, b, bg % Hkv, o, l2);
    }
  }
}

// Host (oda_decode.cu): the parameters of a decode launch after every host-side check of the
// public entry points (ODA_OK, or the ODA_ERR_* code they would return).
int decode_params(const oda_kv* kv, const oda_visibility& vis, const void* q, int hq,
                  float scale, const void* k_new, const void* v_new, void* out, int out_dtype,
                  float* lse, void* ws, size_t ws_bytes, DecodeParams* p);

// ---------------------------------------------------------------------------------------
// Cluster pieces (cluster_decode_kernel and local_chain_kernel): one thread-block cluster of
// kClusterCtas CTAs x kClusterWarps warps per (sequence, KV head), one page per warp, the
// CTAs' partials merged in cluster rank 0's shared memory.
// ---------------------------------------------------------------------------------------
constexpr int kClusterCtas = 16;  // a non-portable cluster size (B200 supports 16)
constexpr int kClusterWarps = 9;
constexpr int kClusterThreads = kClusterWarps * 32;
constexpr int kClusterPages = kClusterCtas * kClusterWarps;  // pages per (b, g) at most
// The per-layer cluster kernel: rank 0 holds no page (its stage memory is the inbox); two CTAs
// per SM (its shared memory is padded to kLocalSmemFloor so that a third does not fit: with
// three, every cluster of the next layer is resident early, but the layer itself was measured
// slower, 5.50 against 5.28 us at 28 layers x 8 KV heads x 2,052 tokens).
constexpr int kLocalCtas = 16;
constexpr int kLocalWarps = 9;
constexpr int kLocalThreads = kLocalWarps * 32;
constexpr int kLocalClusterPages = (kLocalCtas - 1) * kLocalWarps;
constexpr int kLocalCtasPerSm = 2;
constexpr size_t kLocalSmemFloor = 80 * 1024;  // > 228 KB per SM / 3 - 1 KB reserved per CTA

// Floats of one CTA partial in rank 0's inbox: G * 128 outputs + G log-sums, padded to a
// multiple of 4 so that every slot starts 16-byte aligned (the partials arrive by 16-byte
// remote stores).
template <int G>
struct ClusterPart {
  static constexpr int kOut = G * kHeadDim;
  static constexpr int value = (kOut + G + 3) / 4 * 4;
};

// `p` rounded up to a 16-byte boundary (shared-memory carve-outs that take 16-byte accesses;
// their size computations reserve 16 bytes of slack for it).
__device__ __forceinline__ float* align16(float* p) {
  return reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(p) + 15) & ~uintptr_t(15));
}

// Query of heads g G .. g G + G - 1 of sequence b, scaled into base-2 score units, in the
// half-warp layout of page_step (lane li: dims 8 li .. 8 li + 7).
template <int G>
__device__ __forceinline__ void load_q_scaled(const __nv_bfloat16* q, int hq, int b, int g,
                                              float scale_log2, int li, f2_t (&q2)[G][4]) {
#pragma unroll
  for (int gg = 0; gg < G; ++gg) {
    const uint4 qv =
        *reinterpret_cast<const uint4*>(q + ((size_t)b * hq + g * G + gg) * kHeadDim + 8 * li);
    float qf[8];
    unpack8(qv, qf);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
      q2[gg][jj] = f2_pack(qf[2 * jj] * scale_log2, qf[2 * jj + 1] * scale_log2);
  }
}

// Commit of slot t by the warp that holds its page: the step's K/V row into the cache and
// into the page's shared-memory copy (lanes 0-15 the K row, 16-31 the V row).
__device__ __forceinline__ void commit_slot(unsigned char* st, const __nv_bfloat16* k_new,
                                            const __nv_bfloat16* v_new, __nv_bfloat16* k_cache_w,
                                            __nv_bfloat16* v_cache_w, int b, int hkv, int g,
                                            int t, int pb, int lane) {
  const int li = lane & 15;
  const int row = t % kPage;
  const bool isk = lane < 16;
  const uint4 v = *reinterpret_cast<const uint4*>((isk ? k_new : v_new) +
                                                  ((size_t)b * hkv + g) * kHeadDim + 8 * li);
  *reinterpret_cast<uint4*>(st + (isk ? 0 : kPageBytes) + row * kRowBytes + 16 * li) = v;
  __nv_bfloat16* dst = (isk ? k_cache_w : v_cache_w) + (size_t)pb * hkv * kPage * kHeadDim +
                       (size_t)g * (kPage * kHeadDim) + row * kHeadDim + 8 * li;
  *reinterpret_cast<uint4*>(dst) = v;
  __syncwarp();
}

// Softmax states a warp contributes to its CTA's merge: two (one per row parity) with the
// CUDA-core page step, whose halves keep their own maxima; one with the tensor-core page step
// (page_step_mma), whose maxima are shared by the whole warp, so the halves simply add.
template <int G, bool kMma, int W = kClusterWarps>
struct ClusterStates {
  static constexpr int VPL = kMma ? 2 : Vpl<G>::value;  // softmax values per lane
  static constexpr int per_warp = kMma ? 1 : 2;
  static constexpr int value = per_warp * W;            // W warps per CTA
};

// Floats of the in-CTA merge scratch for ClusterStates<G, kMma, W>::value states.
template <int G, bool kMma, int W = kClusterWarps>
__host__ __device__ constexpr int cluster_scratch_floats() {
  return ClusterStates<G, kMma, W>::value * G * (kHeadDim + 2);
}

// The CTA partial of a cluster CTA: merges its warps' states (through `scratch`, at least
// cluster_scratch_floats<G, kMma>() floats, which a CTA barrier before the call must separate
// from earlier reads of it), normalises, and stores the result and its log2-sum into slot
// `rank` (slots `stride` floats apart) of cluster rank 0's inbox (`inbox` is the local
// address of the inbox; every CTA of the cluster has one at the same offset), the caller's
// cluster barrier publishing the stores -- or, with kAsync, by st.async stores that complete
// on rank 0's mbarrier `inbar` (a cluster address), (G * 128 + G) * 4 bytes per CTA -- or, with
// kLocal, into this CTA's own buffer `inbox` for the caller to ship. Contains a CTA barrier
// before the states are read.
template <int G, bool kMma = false, int W = kClusterWarps, bool kLocal = false,
          bool kAsync = false>
__device__ __forceinline__ void cluster_push_partial(
    const float (&m_run)[ClusterStates<G, kMma, W>::VPL],
    const float (&l_run)[ClusterStates<G, kMma, W>::VPL], f2_t (&acc)[G][4], float* scratch,
    float* inbox, int stride, unsigned rank, uint32_t inbar = 0u) {
  constexpr int VPL = ClusterStates<G, kMma, W>::VPL;
  constexpr int kStates = ClusterStates<G, kMma, W>::value;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = lane >> 4, li = lane & 15;
  float* Mw = scratch;           // [kStates][G]
  float* Lw = Mw + kStates * G;  // [kStates][G]
  float* Aw = Lw + kStates * G;  // [kStates][G][128]
  if constexpr (kMma) {
    // lane (gid, tig) summed its own tokens of heads 2 tig + u: add over gid; the halves'
    // P.V sums (rows of each parity) add too, the maxima being the warp's
    const int tig = lane & 3;
    float lsum[VPL];
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      float v = l_run[u];
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      lsum[u] = v;
    }
    if (lane < 4 && 2 * tig < G) {
#pragma unroll
      for (int u = 0; u < VPL; ++u) {
        Mw[warp * G + 2 * tig + u] = m_run[u];
        Lw[warp * G + 2 * tig + u] = lsum[u];
      }
    }
#pragma unroll
    for (int gg = 0; gg < G; ++gg)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float lo, hi, olo, ohi;
        f2_unpack(acc[gg][j], lo, hi);
        olo = __shfl_xor_sync(0xffffffffu, lo, 16);
        ohi = __shfl_xor_sync(0xffffffffu, hi, 16);
        acc[gg][j] = f2_pack(lo + olo, hi + ohi);
      }
    if (half == 0) {
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        float a[8];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) f2_unpack(acc[gg][jj], a[2 * jj], a[2 * jj + 1]);
        float4* dst = reinterpret_cast<float4*>(Aw + (warp * G + gg) * kHeadDim + 8 * li);
        dst[0] = make_float4(a[0], a[1], a[2], a[3]);
        dst[1] = make_float4(a[4], a[5], a[6], a[7]);
      }
    }
  } else {
    float lsum[VPL];
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      float v = l_run[u];
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      lsum[u] = v;
    }
    const int sidx = warp * 2 + half;
    if (li < 2 && (G >= 2 || li == 0)) {
#pragma unroll
      for (int u = 0; u < VPL; ++u) {
        const int gh = (G >= 2) ? ((li & 1) * (G / 2) + u) : 0;
        Mw[sidx * G + gh] = m_run[u];
        Lw[sidx * G + gh] = lsum[u];
      }
    }
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      float a[8];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) f2_unpack(acc[gg][jj], a[2 * jj], a[2 * jj + 1]);
      float4* dst = reinterpret_cast<float4*>(Aw + (sidx * G + gg) * kHeadDim + 8 * li);
      dst[0] = make_float4(a[0], a[1], a[2], a[3]);
      dst[1] = make_float4(a[4], a[5], a[6], a[7]);
    }
  }
  __syncthreads();
  // One thread per (head, 4 dims) reads every state's max and sum (broadcast shared loads),
  // weighs the states once, sums its 4 dims and pushes the normalised result (one 16-byte
  // store) and, for dim 0, the log-sum straight into rank 0's shared memory: few, wide remote
  // stores, since the inbox's SM takes them from every CTA of the cluster at once.
  constexpr int kOut = ClusterPart<G>::kOut;
  float* slot = inbox + rank * stride;  // 16-byte aligned: inbox and stride are
  for (int o4 = tid; o4 < kOut / 4; o4 += blockDim.x) {
    const int gg = (4 * o4) / kHeadDim, d = (4 * o4) % kHeadDim;
    float M = -INFINITY;
#pragma unroll
    for (int s2 = 0; s2 < kStates; ++s2) M = fmaxf(M, Mw[s2 * G + gg]);
    float4 oval = make_float4(0.f, 0.f, 0.f, 0.f);
    float l2 = -INFINITY;
    if (M != -INFINITY) {
      float L = 0.f;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int s2 = 0; s2 < kStates; ++s2) {
        const float ms = Mw[s2 * G + gg];
        const float w = (ms == -INFINITY) ? 0.f : ex2_fast(ms - M);
        L = fmaf(w, Lw[s2 * G + gg], L);
        const float4 av = *reinterpret_cast<const float4*>(Aw + (s2 * G + gg) * kHeadDim + d);
        a.x = fmaf(w, av.x, a.x);
        a.y = fmaf(w, av.y, a.y);
        a.z = fmaf(w, av.z, a.z);
        a.w = fmaf(w, av.w, a.w);
      }
      const float rL = rcp_fast(L);
      oval = make_float4(a.x * rL, a.y * rL, a.z * rL, a.w * rL);
      l2 = M + lg2_fast(L);
    }
    if constexpr (kLocal) {  // into this CTA's own slot (`inbox`), shipped by the caller
      *reinterpret_cast<float4*>(inbox + 4 * o4) = oval;
      if (d == 0) inbox[kOut + gg] = l2;
    } else if constexpr (kAsync) {
      st_async4(cluster_addr(slot + 4 * o4, 0), oval, inbar);
      if (d == 0) st_async1(cluster_addr(slot + kOut + gg, 0), l2, inbar);
    } else {
      dsmem_st4(slot + 4 * o4, 0, oval);
      if (d == 0) dsmem_st(slot + kOut + gg, 0, l2);
    }
  }
}

// Rank 0's merge of the partials in slots kFirst .. C - 1 of its inbox (slots `stride` floats
// apart), in rank order: dim `tid` (< 128) of every head of the group.
template <int G, int kFirst = 0, int C = kClusterCtas>
__device__ __forceinline__ void cluster_merge_inbox(const float* inbox, int stride, float (&o)[G],
                                                    float (&l2)[G]) {
  constexpr int kOut = ClusterPart<G>::kOut;
  constexpr int kN = C - kFirst;
  const int kPart = stride;
  const int tid = threadIdx.x;
  float ls[G][kN], os[G][kN];
#pragma unroll
  for (int gg = 0; gg < G; ++gg)
#pragma unroll
    for (int c = 0; c < kN; ++c) {
      ls[gg][c] = inbox[(c + kFirst) * kPart + kOut + gg];
      os[gg][c] = inbox[(c + kFirst) * kPart + gg * kHeadDim + tid];
    }
#pragma unroll
  for (int gg = 0; gg < G; ++gg) {
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < kN; ++c) M = fmaxf(M, ls[gg][c]);
    if (M == -INFINITY) {
      o[gg] = 0.f;
      l2[gg] = -INFINITY;
    } else {
      float L = 0.f, a = 0.f;
#pragma unroll
      for (int c = 0; c < kN; ++c) {
        const float w = (ls[gg][c] == -INFINITY) ? 0.f : ex2_fast(ls[gg][c] - M);
        L += w;
        a = fmaf(w, os[gg][c], a);
      }
      o[gg] = a * rcp_fast(L);
      l2[gg] = M + lg2_fast(L);
    }
  }
}

}  // namespace oda

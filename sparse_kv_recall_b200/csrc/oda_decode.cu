// K2 + K3: paged decode attention for Local, Full and keep-page visibility, split over the
// whole GPU and merged inside the same launch.
//
// Work decomposition. Every sequence b contributes npages(b) visible pages per KV head; the
// flattened list of (b, KV head g, page j) units is cut into gridDim.x equal contiguous
// shares, one per CTA (grid = 2 CTAs per SM, one wave, no tail). A share may cover part of
// one (b, g) or the ends of several. Inside a CTA each of the 4 warps streams every 4th page
// of the current (b, g) piece through its own 3-stage ring of shared-memory stages filled by
// 1-D bulk copies (TMA engine, 4 KB K page + 4 KB V page per stage), and keeps an online
// softmax for all G = Hq / Hkv query heads that share the KV head, so each page is read
// from HBM once for the whole group. A piece's 8 half-warp states are merged in shared
// memory; if the (b, g) spans several CTAs, each writes its normalised partial (O, log2-sum)
// to the workspace and the last to arrive (atomic ticket) merges them in fixed order.
//
// Short windows at small batch (Local) take cluster_decode_kernel instead: one thread-block
// cluster per (b, g), one page per warp, partials merged in distributed shared memory (see
// that kernel). Both kernels share the plan, the P.V step and the commit of slot t.
//
// Lane layout for a 16 x 128 page: lane = 16 * half + li; lane li owns dims [8 li, 8 li + 8)
// of rows 2k + half, k = 0..7, for P.V. The CUDA-core scores (cluster_decode_kernel, and
// decode_kernel<1>) are reduced over the 16 lanes of a half by a reduce-scatter butterfly,
// after which lane li holds row 2 (li / 2) + half for heads (li % 2) * G / 2 + u;
// decode_kernel<2> and <4> form the scores on the tensor cores (page_step_mma).
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
    const float pr = (v == -INFINITY) ? 0.f : exp2f(v - mnew);
    const float al = (m_run[u] == mnew) ? 1.f : exp2f(m_run[u] - mnew);
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
      const float al = !up ? 1.f : (m_run[u] == -INFINITY ? 0.f : exp2f(m_run[u] - mx));
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
      const float pr = (s[t][u] == -INFINITY) ? 0.f : exp2f(s[t][u] - m_run[u]);
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

template <int G>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_kernel(const DecodeParams p) {
  constexpr int VPL = MmaScores<G>::value ? 2 : Vpl<G>::value;  // softmax states per lane
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* stages = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kStages * kStageBytes);
  float* pscratch = reinterpret_cast<float*>(bars + kWarps * kStages);
  constexpr int kPs = 18 * G;  // per-warp softmax exchange: 16 G weights + 2 G rescales
  int* pre = reinterpret_cast<int*>(pscratch + kWarps * kPs);  // [batch + 1] prefix of units
  __shared__ int s_last;
  __shared__ unsigned long long s_rows, s_pages;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = lane >> 4, li = lane & 15;
  const int B = p.batch, Hkv = p.hkv;
  const int P = gridDim.x, c = blockIdx.x;

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
  };
  if (p.wait_first) dep_wait();
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[warp * kStages + s], 1);
    fence_barrier_init();
  }
  if (tid == 0) {
    s_rows = 0;
    s_pages = 0;
    pre[0] = 0;
  }
  for (int b = tid; b < B; b += kThreads) {
    const SeqPlan sp = make_plan(p.plan, b);
    pre[b + 1] = sp.npages * Hkv;
    if (c == 0 && sp.err != 0) report(p.status, sp.err);
  }
  __syncthreads();
  __shared__ int s_align;  // CTA-count granularity that keeps shares inside one (b, g)
  if (warp == 0) {  // inclusive scan of the per-sequence unit counts
    int carry = 0;
    unsigned vmin = 0xffffffffu, vmax = 0u, active = 0u;
    for (int base = 0; base < B; base += 32) {
      const int i = base + lane;
      int v = i < B ? pre[i + 1] : 0;
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
      if (i < B) pre[i + 1] = v;
      carry = __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) s_align = (active > 0 && vmin == vmax) ? (int)active * Hkv : 0;
  }
  __syncthreads();
  const long long T = pre[B];

  const uint64_t policy = l2_evict_first_policy();
  unsigned char* wst = stages + warp * kStages * kStageBytes;
  uint64_t* wbar = bars + warp * kStages;
  float* ps = pscratch + warp * kPs;
  unsigned wcount = 0;       // pages this warp has consumed, over all pieces
  bool dead = false;         // a bounded wait gave up: stop touching the ring
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

    // lane 0 starts page n of this piece into stage (wcount + n) % kStages
    auto issue = [&](int n) {
      const int j = first + n * kWarps;
      const PageRef r = page_ref(p.plan, sp, b, j);
      uint64_t* bar = &wbar[(wcount + n) % kStages];
      unsigned char* dst = wst + ((wcount + n) % kStages) * kStageBytes;
      if (r.err == 0) {
        const size_t src = (size_t)r.pb * page_stride + head_off;
        mbar_arrive_expect_tx(bar, kStageBytes);
        bulk_load(dst, p.k_cache + src, kPageBytes, bar, policy);
        bulk_load(dst + kPageBytes, p.v_cache + src, kPageBytes, bar, policy);
      } else {
        report(p.status, r.err);
        mbar_arrive(bar);
      }
    };

    if (!dead && lane == 0)
      for (int n = 0; n < min(cnt, kStages); ++n) issue(n);
    __syncwarp();
    dep_wait();

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

    for (int n = 0; n < cnt && !dead; ++n) {
      const unsigned k = wcount + n;
      const int stage = k % kStages;
      const PageRef r = page_ref(p.plan, sp, b, first + n * kWarps);
      if (!__all_sync(0xffffffffu, mbar_wait(&wbar[stage], (k / kStages) & 1u))) {
        if (lane == 0) report(p.status, ODA_DEV_TIMEOUT);
        // let the copies already started into the other stages land, then stop
        for (int m = n + 1; m < min(cnt, n + kStages); ++m) {
          const unsigned km = wcount + m;
          mbar_wait(&wbar[km % kStages], (km / kStages) & 1u);
        }
        dead = true;
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
    wcount += cnt;

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
      atomicAdd(&s_rows, (unsigned long long)rows_vis);
      atomicAdd(&s_pages, (unsigned long long)pages_read);
    }
    rows_vis = 0;
    pages_read = 0;
    __syncthreads();  // every warp is done with its stages: reuse them as merge scratch
    if (p.stats != nullptr && tid == 0) {
      // issued now, so that the counter updates complete while the merge runs
      if (s_rows) atomicAdd(&p.stats[ODA_STAT_ROWS], s_rows);
      if (s_pages) atomicAdd(&p.stats[ODA_STAT_PAGES], s_pages);
      s_rows = 0;
      s_pages = 0;
    }
    float* Mw = reinterpret_cast<float*>(stages);  // [2 * kWarps][G]
    float* Lw = Mw + 2 * kWarps * G;               // [2 * kWarps][G]
    float* Aw = Lw + 2 * kWarps * G;               // [2 * kWarps][G][128]
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
          const float w = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
          L = fmaf(w, Lw[s * G + gg], L);
          a = fmaf(w, Aw[(s * G + gg) * kHeadDim + tid], a);
        }
        o[gg] = a / L;
        l2[gg] = M + log2f(L);
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
      if (tid == 0) s_last = ticket_arrive(&p.ws_ticket[bg]) == (unsigned)(n_contrib - 1);
      __syncthreads();  // ... and the last CTA's thread 0 acquired everyone's partials
      if (s_last) {
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
            const float wgt = (ls == -INFINITY) ? 0.f : exp2f(ls - m);
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
            o[gg] = a[gg] / L;
            l2[gg] = M + log2f(L);
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
  dep_wait();
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

// ---------------------------------------------------------------------------------------
// Short-window kernel (Local at small batch). The split above ends a short launch with a
// chain of global round trips: every CTA's partial to global memory, an acquire-release
// ticket, the last CTA reading every partial back. Here one thread-block cluster of
// kClusterCtas CTAs takes one (sequence, KV head); each of its kClusterCtas x kClusterWarps
// warps attends at most one page, and the CTAs' partials are merged through distributed
// shared memory by cluster rank 0 between two cluster barriers. The page step, the commit
// of slot t and the in-CTA merge are those of decode_kernel.
// ---------------------------------------------------------------------------------------
constexpr int kClusterCtas = 16;  // a non-portable cluster size (B200 supports 16)
constexpr int kClusterWarps = 9;
constexpr int kClusterThreads = kClusterWarps * 32;
constexpr int kClusterPages = kClusterCtas * kClusterWarps;  // pages per (b, g) at most

template <int G>
__global__ void __launch_bounds__(kClusterThreads, 2) cluster_decode_kernel(const DecodeParams p) {
  constexpr int VPL = Vpl<G>::value;
  constexpr int kPs = 18 * G;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* stages = smem;  // [warp][kStageBytes]: one page per warp
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kClusterWarps * kStageBytes);
  float* pscratch = reinterpret_cast<float*>(bars + kClusterWarps);  // [warp][kPs]
  // rank 0's copy gathers every CTA's partial: [kClusterCtas][G * 128 outputs + G log-sums]
  float* part = pscratch + kClusterWarps * kPs;
  __shared__ unsigned long long s_rows, s_pages;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = lane >> 4, li = lane & 15;
  const unsigned rank = cluster_ctarank();
  const int bg = blockIdx.x / kClusterCtas;
  const int b = bg / p.hkv, g = bg % p.hkv;
  if (tid == 0) {
    s_rows = 0;
    s_pages = 0;
  }
  if (lane == 0) {
    mbar_init(&bars[warp], 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (p.wait_first) griddep_wait();

  // Before the dependency wait: the plan and this warp's page copy (history pages only).
  const SeqPlan sp = make_plan(p.plan, b);
  if (rank == 0 && g == 0 && tid == 0 && sp.err != 0) report(p.status, sp.err);
  const int j = (int)rank * kClusterWarps + warp;
  const bool has = !sp.skip && j < sp.npages;
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
  griddep_launch_dependents();

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
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      const uint4 qv = *reinterpret_cast<const uint4*>(
          p.q + ((size_t)b * p.hq + g * G + gg) * kHeadDim + 8 * li);
      float qf[8];
      unpack8(qv, qf);
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
        q2[gg][jj] = f2_pack(qf[2 * jj] * p.scale_log2, qf[2 * jj + 1] * p.scale_log2);
    }
    if (!__all_sync(0xffffffffu, mbar_wait(&bars[warp], 0u))) {
      if (lane == 0) report(p.status, ODA_DEV_TIMEOUT);
    } else {
      if (p.k_new != nullptr && r.lp == sp.t / kPage) {
        // Commit: the step's K/V take slot t, in the cache and in this page's copy.
        const int row = sp.t % kPage;
        const bool isk = lane < 16;
        const uint4 v = *reinterpret_cast<const uint4*>(
            (isk ? p.k_new : p.v_new) + ((size_t)b * p.hkv + g) * kHeadDim + 8 * li);
        *reinterpret_cast<uint4*>(st + (isk ? 0 : kPageBytes) + row * kRowBytes + 16 * li) = v;
        __nv_bfloat16* dst = (isk ? p.k_cache_w : p.v_cache_w) + (size_t)r.pb * page_stride +
                             head_off + row * kHeadDim + 8 * li;
        *reinterpret_cast<uint4*>(dst) = v;
        __syncwarp();
      }
      page_step<G>(st, q2, m_run, l_run, acc, pscratch + warp * kPs, sp, r.lp, lane, rows_vis);
      pages_read = 1;
    }
  }

  // ---- merge the CTA's 2 x kClusterWarps half-warp states ----
  float lsum[VPL];
#pragma unroll
  for (int u = 0; u < VPL; ++u) {
    float v = l_run[u];
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    lsum[u] = v;
  }
  if (p.stats != nullptr && lane == 0 && pages_read) {
    atomicAdd(&s_rows, (unsigned long long)rows_vis);
    atomicAdd(&s_pages, (unsigned long long)pages_read);
  }
  __syncthreads();  // every warp is done with its page: stage memory becomes merge scratch
  if (p.stats != nullptr && tid == 0) {
    if (s_rows) atomicAdd(&p.stats[ODA_STAT_ROWS], s_rows);
    if (s_pages) atomicAdd(&p.stats[ODA_STAT_PAGES], s_pages);
  }
  constexpr int kStates = 2 * kClusterWarps;
  float* Mw = reinterpret_cast<float*>(stages);  // [kStates][G]
  float* Lw = Mw + kStates * G;                  // [kStates][G]
  float* Aw = Lw + kStates * G;                  // [kStates][G][128]
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
  __syncthreads();
  // The CTA partial: one thread per (head, dim) output reads every state's max and sum
  // (broadcast shared loads), weighs the states and pushes the normalised result and the
  // log-sum straight into rank 0's shared memory.
  constexpr int kOut = G * kHeadDim;
  constexpr int kPart = kOut + G;
  float* slot = part + rank * kPart;
  for (int o = tid; o < kOut; o += kClusterThreads) {
    const int gg = o / kHeadDim, d = o % kHeadDim;
    float M = -INFINITY;
#pragma unroll
    for (int s2 = 0; s2 < kStates; ++s2) M = fmaxf(M, Mw[s2 * G + gg]);
    float oval = 0.f, l2 = -INFINITY;
    if (M != -INFINITY) {
      float L = 0.f, a = 0.f;
#pragma unroll
      for (int s2 = 0; s2 < kStates; ++s2) {
        const float ms = Mw[s2 * G + gg];
        const float w = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
        L = fmaf(w, Lw[s2 * G + gg], L);
        a = fmaf(w, Aw[(s2 * G + gg) * kHeadDim + d], a);
      }
      oval = a / L;
      l2 = M + log2f(L);
    }
    dsmem_st(slot + o, 0, oval);
    if (d == 0) dsmem_st(slot + kOut + gg, 0, l2);
  }
  cluster_sync();  // every CTA's partial has landed in rank 0's shared memory
  if (rank == 0 && !sp.skip && tid < kHeadDim) {
    float ls[G][kClusterCtas], os[G][kClusterCtas];
#pragma unroll
    for (int gg = 0; gg < G; ++gg)
#pragma unroll
      for (int c = 0; c < kClusterCtas; ++c) {
        ls[gg][c] = part[c * kPart + kOut + gg];
        os[gg][c] = part[c * kPart + gg * kHeadDim + tid];
      }
    float o[G], l2[G];
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      float M = -INFINITY;
#pragma unroll
      for (int c = 0; c < kClusterCtas; ++c) M = fmaxf(M, ls[gg][c]);
      if (M == -INFINITY) {
        o[gg] = 0.f;
        l2[gg] = -INFINITY;
      } else {
        float L = 0.f, a = 0.f;
#pragma unroll
        for (int c = 0; c < kClusterCtas; ++c) {
          const float w = (ls[gg][c] == -INFINITY) ? 0.f : exp2f(ls[gg][c] - M);
          L += w;
          a = fmaf(w, os[gg][c], a);
        }
        o[gg] = a / L;
        l2[gg] = M + log2f(L);
      }
    }
    write_final<G>(p, b, g, o, l2);
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

static size_t decode_smem_bytes(int G) {
  return (size_t)kWarps * kStages * kStageBytes + (size_t)kWarps * kStages * sizeof(uint64_t) +
         (size_t)kWarps * 18 * G * sizeof(float) + (size_t)(kMaxBatch + 1) * sizeof(int);
}

struct WsLayout {
  size_t o_off, lse_off, ticket_off, total;
};

static WsLayout ws_layout(int batch, int hkv, int G, int grid) {
  const size_t slots = (size_t)grid + (size_t)batch * hkv;
  WsLayout w;
  w.o_off = 0;
  w.lse_off = align_up(slots * G * kHeadDim * sizeof(float), 256);
  w.ticket_off = w.lse_off + align_up(slots * G * sizeof(float), 256);
  w.total = w.ticket_off + align_up((size_t)batch * hkv * sizeof(unsigned), 256);
  return w;
}

static size_t cluster_smem_bytes(int G) {
  return (size_t)kClusterWarps * kStageBytes + (size_t)kClusterWarps * sizeof(uint64_t) +
         (size_t)kClusterWarps * 18 * G * sizeof(float) +
         (size_t)kClusterCtas * (G * kHeadDim + G) * sizeof(float);
}

// Clusters of the short-window kernel the device can hold at once, per device and group
// size (0: the cluster shape cannot be scheduled here, e.g. under a partitioned GPU).
static int g_max_clusters[64][kMaxGroup + 1];

template <int G>
static int prepare_decode_kernel(int device) {
  static bool done[64] = {false};
  if (device < 0 || device >= 64) return ODA_ERR_CUDA;
  if (done[device]) return ODA_OK;
  if (cudaFuncSetAttribute(decode_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)decode_smem_bytes(G)) != cudaSuccess ||
      cudaFuncSetAttribute(cluster_decode_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)cluster_smem_bytes(G)) != cudaSuccess ||
      cudaFuncSetAttribute(cluster_decode_kernel<G>,
                           cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
    return ODA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kClusterCtas);
  cfg.blockDim = dim3(kClusterThreads);
  cfg.dynamicSmemBytes = cluster_smem_bytes(G);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kClusterCtas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
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
  cfg.blockDim = dim3(kClusterThreads);
  cfg.dynamicSmemBytes = cluster_smem_bytes(G);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kClusterCtas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
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
  return pages <= kClusterPages && clusters * kClusterCtas <= 2ll * di.sms &&
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

int launch_decode(const oda_kv* kv, const oda_visibility& vis, const void* q, int hq,
                  float scale, const void* k_new, const void* v_new, void* out, int out_dtype,
                  float* lse, void* ws, size_t ws_bytes, void* stream, int pdl, int wait_first) {
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

  DecodeParams p;
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
  p.wait_first = wait_first;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t smem = decode_smem_bytes(G);
  switch (G) {  // attributes and the cluster capacity first
    case 1: rc = prepare_decode_kernel<1>(di.device); break;
    case 2: rc = prepare_decode_kernel<2>(di.device); break;
    default: rc = prepare_decode_kernel<4>(di.device); break;
  }
  if (rc != ODA_OK) return rc;
  const bool cluster = use_cluster_kernel(kv, vis, di, G);
  const int cgrid = kv->batch * kv->num_kv_heads * kClusterCtas;
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

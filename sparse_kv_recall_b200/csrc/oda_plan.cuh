// Visibility plan: which KV pages a sequence streams and which rows of them it attends.
//
// Local  ([ODA] 접근 방법; 주요 결과, last item): the first `sink` positions and the `window`
//        most recent ones, the current position included, as a set union.
// Full   ([ODA] 접근 방법): positions 0..t.
// Keep   ([DA] section 3): the kept logical pages, up to position t.
// DA     ([DA] section 3): a declared mode per sequence -- global, focus or local -- compiled
//        here into ascending runs of kept pages (every page a region touches is kept).
// Shard  positions [pos_lo, pos_hi) of 0..t: one GPU's part of a context-parallel Full.
//
// Every rule but Keep becomes at most kMaxRuns ascending runs of logical pages plus a row
// predicate (row_lo <= p <= row_hi, outside Local's sink/window gap); Keep reads its page
// list from memory. Both the attention kernel and the plan export use these functions.
#pragma once

#include "oda_common.cuh"

namespace oda {

constexpr int kMaxRuns = 3;

struct SeqPlan {
  int t;                    // current position (seq_len - 1)
  int npages;               // pages in the visible list (0: nothing to read)
  int err;                  // ODA_DEV_* of a bad length or keep / DA spec (then npages = 0)
  bool skip;                // gated off: write nothing
  int nruns;                // page runs (0 in Keep mode: the list is in memory)
  int first0, first1, first2;  // logical first page of each run, ascending, disjoint; held
  int len0, len1, len2;        // as scalars (an array member would put the plan in local memory)
  int row_lo, row_hi;       // visible rows: row_lo <= p <= row_hi ...
  int gap_lo, gap_hi;       // ... and not gap_lo <= p < gap_hi (Local's sink/window gap)
};
static_assert(kMaxRuns == 3, "SeqPlan holds three runs");

// Run i of a plan; i is a compile-time constant wherever these are called (unrolled loops).
__host__ __device__ __forceinline__ int& run_first(SeqPlan& s, int i) {
  return i == 0 ? s.first0 : (i == 1 ? s.first1 : s.first2);
}
__host__ __device__ __forceinline__ int& run_len(SeqPlan& s, int i) {
  return i == 0 ? s.len0 : (i == 1 ? s.len1 : s.len2);
}
__host__ __device__ __forceinline__ int run_first(const SeqPlan& s, int i) {
  return i == 0 ? s.first0 : (i == 1 ? s.first1 : s.first2);
}
__host__ __device__ __forceinline__ int run_len(const SeqPlan& s, int i) {
  return i == 0 ? s.len0 : (i == 1 ? s.len1 : s.len2);
}

struct PlanArgs {
  const int32_t* seq_lens;
  const int32_t* block_table;
  int max_blocks;
  int num_blocks;
  int mode;                    // ODA_MODE_*
  int sink, window;            // Local
  const int32_t* gate;         // nullable (Full, Shard)
  const int32_t* keep_blocks;  // Keep: [batch][max_keep]
  const int32_t* keep_counts;
  int max_keep;
  const int32_t* da_modes;     // DA: [batch] ODA_DA_*
  const int32_t* da_offsets;   // DA: [batch] first position of the focused region
  int da_focus_len, da_recent, da_local_len;
  int pos_lo, pos_hi;          // Shard
};

// Append logical pages [first, last] to the run list; runs arrive in ascending order of
// `first`, and a run that touches or overlaps the previous one extends it. Every index is a
// compile-time constant, so the plan stays in registers.
__host__ __device__ __forceinline__ void add_run(SeqPlan& s, int first, int last) {
  if (last < first) return;
  bool merged = false;
#pragma unroll
  for (int i = 0; i < kMaxRuns; ++i) {
    if (i == s.nruns - 1) {
      const int prev_last = run_first(s, i) + run_len(s, i) - 1;
      if (first <= prev_last + 1) {
        run_len(s, i) = max(prev_last, last) - run_first(s, i) + 1;
        merged = true;
      }
    }
  }
  if (merged) return;
#pragma unroll
  for (int i = 0; i < kMaxRuns; ++i) {
    if (i == s.nruns) {
      run_first(s, i) = first;
      run_len(s, i) = last - first + 1;
    }
  }
  ++s.nruns;
}

__host__ __device__ __forceinline__ SeqPlan make_plan(const PlanArgs& a, int b) {
  SeqPlan s;
  s.npages = 0;
  s.err = 0;
  s.skip = false;
  s.nruns = 0;
  s.first0 = s.first1 = s.first2 = 0;
  s.len0 = s.len1 = s.len2 = 0;
  s.gap_lo = 0;
  s.gap_hi = 0;
  const int len = a.seq_lens[b];
  s.t = len - 1;
  s.row_lo = 0;
  s.row_hi = s.t;
  if (a.gate != nullptr && a.gate[b] == 0) {
    s.skip = true;
    return s;
  }
  if (len < 1 || len > a.max_blocks * kPage) {
    s.err = ODA_DEV_BAD_LEN;
    return s;
  }
  const int t = s.t;
  const int last_page = t / kPage;
  if (a.mode == ODA_MODE_KEEP) {
    const int c = a.keep_counts[b];
    if (c < 0 || c > a.max_keep) {
      s.err = ODA_DEV_BAD_KEEP_LIST;
      return s;
    }
    s.npages = c;
    return s;
  }
  if (a.mode == ODA_MODE_LOCAL) {
    const int sink_end = min(max(a.sink, 0), t + 1);
    const int win_start = max(0, t - max(a.window, 0) + 1);
    if (win_start <= sink_end) {  // the union is the whole history
      add_run(s, 0, last_page);
    } else {
      s.gap_lo = sink_end;
      s.gap_hi = win_start;
      add_run(s, 0, (sink_end + kPage - 1) / kPage - 1);
      add_run(s, win_start / kPage, last_page);
    }
  } else if (a.mode == ODA_MODE_DA) {
    const int m = a.da_modes[b];
    if (m == ODA_DA_GLOBAL) {
      add_run(s, 0, last_page);
    } else if (m == ODA_DA_LOCAL) {
      add_run(s, max(0, t - a.da_local_len + 1) / kPage, last_page);
    } else if (m == ODA_DA_FOCUS && a.da_offsets[b] >= 0) {
      // sink page, focused region, recent tokens; a focus region that starts after the
      // recent run's first page lies inside that run and adds nothing
      const int off = a.da_offsets[b];
      const long long f_end = min((long long)t, (long long)off + a.da_focus_len - 1);
      const int r_first = max(0, t - a.da_recent + 1) / kPage;
      add_run(s, 0, 0);
      if (off <= f_end && off / kPage <= r_first) add_run(s, off / kPage, (int)(f_end / kPage));
      add_run(s, r_first, last_page);
    } else {
      s.err = ODA_DEV_BAD_DA;
      return s;
    }
  } else if (a.mode == ODA_MODE_SHARD) {
    s.row_lo = a.pos_lo;
    s.row_hi = min(t, a.pos_hi - 1);
    if (s.row_lo <= s.row_hi) add_run(s, s.row_lo / kPage, s.row_hi / kPage);
  } else {  // Full
    add_run(s, 0, last_page);
  }
  s.npages = s.len0 + s.len1 + s.len2;
  return s;
}

// Row predicate on absolute position p of a listed page.
__host__ __device__ __forceinline__ bool row_visible(const SeqPlan& s, int p) {
  return p >= s.row_lo && p <= s.row_hi && !(p >= s.gap_lo && p < s.gap_hi);
}

struct PageRef {
  int lp;   // logical page
  int pb;   // physical page
  int err;  // 0, or the ODA_DEV_* code that makes this page unusable
};

// Logical and physical page of list entry j of sequence b.
__host__ __device__ __forceinline__ PageRef page_ref(const PlanArgs& a, const SeqPlan& s, int b, int j) {
  PageRef r;
  r.err = 0;
  if (a.mode == ODA_MODE_KEEP) {
    const int32_t* kb = a.keep_blocks + (size_t)b * a.max_keep;
    r.lp = kb[j];
    if (r.lp < 0 || r.lp > s.t / kPage || (j > 0 && kb[j - 1] >= r.lp)) {
      r.err = ODA_DEV_BAD_KEEP_LIST;
      r.pb = -1;
      return r;
    }
  } else {
    int before = 0;
    r.lp = -1;
#pragma unroll
    for (int i = 0; i < kMaxRuns; ++i) {  // the run holding entry j
      if (r.lp < 0 && j - before < run_len(s, i)) r.lp = run_first(s, i) + (j - before);
      before += run_len(s, i);
    }
    if (r.lp < 0) {  // j beyond the list: callers never ask, but never read table[-1]
      r.err = ODA_DEV_BAD_BLOCK;
      r.pb = -1;
      return r;
    }
  }
  r.pb = a.block_table[(size_t)b * a.max_blocks + r.lp];
  if (r.pb < 0 || r.pb >= a.num_blocks) r.err = ODA_DEV_BAD_BLOCK;
  return r;
}

}  // namespace oda

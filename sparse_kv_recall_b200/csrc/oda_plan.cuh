// Visibility plan: which KV pages a sequence streams and which rows of them it attends.
//
// Local  ([ODA] 접근 방법; 주요 결과, last item): the first `sink` positions and the `window`
//        most recent ones, the current position included, as a set union.
// Full   ([ODA] 접근 방법): positions 0..t.
// Keep   ([DA] section 3): the kept logical pages, up to position t.
//
// Each rule becomes an ordered list of logical pages j = 0..npages-1 plus a row predicate.
// Local's list is the sink pages [0, head_pages) followed by the window pages
// [tail_first, t/16]; when the two touch, it is simply pages 0..t/16 and the row predicate
// removes the gap. Both the attention kernel and the plan export use these functions.
#pragma once

#include "oda_common.cuh"

namespace oda {

struct SeqPlan {
  int t;           // current position (seq_len - 1)
  int npages;      // pages in the visible list (0: nothing to read)
  int head_pages;  // list entries j < head_pages are logical page j
  int tail_first;  // list entry j >= head_pages is logical page tail_first + j - head_pages
  int sink_end;    // Local row rule: p < sink_end or p >= win_start (and p <= t)
  int win_start;
  bool skip;       // gated off: write nothing
  bool bad_len;    // seq_len outside [1, max_blocks * 16]
  bool bad_keep;   // keep count outside [0, max_keep]
};

struct PlanArgs {
  const int32_t* seq_lens;
  const int32_t* block_table;
  int max_blocks;
  int num_blocks;
  int mode;                    // ODA_MODE_*
  int sink, window;
  const int32_t* gate;         // nullable (Full)
  const int32_t* keep_blocks;  // Keep: [batch][max_keep]
  const int32_t* keep_counts;
  int max_keep;
};

__host__ __device__ __forceinline__ SeqPlan make_plan(const PlanArgs& a, int b) {
  SeqPlan s;
  s.skip = false;
  s.bad_len = false;
  s.bad_keep = false;
  s.npages = 0;
  s.head_pages = 0;
  s.tail_first = 0;
  s.sink_end = 0;
  s.win_start = 0;
  const int len = a.seq_lens[b];
  s.t = len - 1;
  if (a.gate != nullptr && a.gate[b] == 0) {
    s.skip = true;
    return s;
  }
  if (len < 1 || len > a.max_blocks * kPage) {
    s.bad_len = true;
    return s;
  }
  const int t = s.t;
  const int last_page = t / kPage;
  s.sink_end = t + 1;
  s.win_start = 0;
  if (a.mode == ODA_MODE_KEEP) {
    const int c = a.keep_counts[b];
    s.bad_keep = c < 0 || c > a.max_keep;
    s.npages = s.bad_keep ? 0 : c;
    s.head_pages = 0;
  } else if (a.mode == ODA_MODE_LOCAL) {
    const int sink_end = min(max(a.sink, 0), t + 1);
    const int win_start = max(0, t - max(a.window, 0) + 1);
    if (win_start <= sink_end) {  // the union is the whole history
      s.npages = last_page + 1;
      s.head_pages = s.npages;
    } else {
      s.sink_end = sink_end;
      s.win_start = win_start;
      const int head = (sink_end + kPage - 1) / kPage;
      const int first = win_start / kPage;
      if (first <= head) {  // window's first page touches the sink pages: one run
        s.npages = last_page + 1;
        s.head_pages = s.npages;
      } else {
        s.head_pages = head;
        s.tail_first = first;
        s.npages = head + (last_page - first + 1);
      }
    }
  } else {  // Full
    s.npages = last_page + 1;
    s.head_pages = s.npages;
  }
  return s;
}

// Row predicate on absolute position p of a listed page.
__host__ __device__ __forceinline__ bool row_visible(const SeqPlan& s, int p) {
  return p <= s.t && (p < s.sink_end || p >= s.win_start);
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
    r.lp = j < s.head_pages ? j : s.tail_first + (j - s.head_pages);
  }
  r.pb = a.block_table[(size_t)b * a.max_blocks + r.lp];
  if (r.pb < 0 || r.pb >= a.num_blocks) r.err = ODA_DEV_BAD_BLOCK;
  return r;
}

}  // namespace oda

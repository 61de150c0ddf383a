// Host-side driver for the library's visibility plan (oda_plan.cuh is __host__ __device__):
// reads one case per line on stdin and prints the visible positions the decode kernel's
// plan produces, so that tests can compare them with the oracle's set definitions without
// a GPU. Input lines (whitespace separated):
//   L t sink window            Local
//   F t                        Full
//   K t n id0 .. id{n-1}       Keep list
//   D t mode offset focus_len recent local_len
//   S t lo hi                  Shard
// Output per case: "err npages p0 p1 ..." (visible positions in list order), or "bad" when a
// page id is out of order / range.
#include <cstdio>
#include <string>
#include <vector>

#include "oda_plan.cuh"

using namespace oda;

int main() {
  const int maxb = 1 << 16;
  std::vector<int32_t> table(maxb);
  for (int i = 0; i < maxb; ++i) table[i] = (int)((i * 7919ll) % maxb);  // any permutation
  char kind;
  while (std::scanf(" %c", &kind) == 1) {
    int t = 0;
    if (std::scanf("%d", &t) != 1) return 2;
    int32_t len = t + 1;
    std::vector<int32_t> keep;
    int32_t keep_count = 0;
    int32_t da_mode = 0, da_off = 0;
    PlanArgs a = {};
    a.seq_lens = &len;
    a.block_table = table.data();
    a.max_blocks = maxb;
    a.num_blocks = maxb;
    a.window = 1;
    if (kind == 'L') {
      a.mode = ODA_MODE_LOCAL;
      if (std::scanf("%d %d", &a.sink, &a.window) != 2) return 2;
    } else if (kind == 'F') {
      a.mode = ODA_MODE_FULL;
    } else if (kind == 'K') {
      a.mode = ODA_MODE_KEEP;
      if (std::scanf("%d", &keep_count) != 1) return 2;
      keep.resize(keep_count > 0 ? keep_count : 1);
      for (int i = 0; i < keep_count; ++i)
        if (std::scanf("%d", &keep[i]) != 1) return 2;
      a.keep_blocks = keep.data();
      a.keep_counts = &keep_count;
      a.max_keep = keep_count;
    } else if (kind == 'D') {
      a.mode = ODA_MODE_DA;
      if (std::scanf("%d %d %d %d %d", &da_mode, &da_off, &a.da_focus_len, &a.da_recent,
                     &a.da_local_len) != 5)
        return 2;
      a.da_modes = &da_mode;
      a.da_offsets = &da_off;
    } else if (kind == 'S') {
      a.mode = ODA_MODE_SHARD;
      if (std::scanf("%d %d", &a.pos_lo, &a.pos_hi) != 2) return 2;
    } else {
      return 2;
    }
    const SeqPlan sp = make_plan(a, 0);
    std::string line = std::to_string(sp.err) + " " + std::to_string(sp.npages);
    bool bad = false;
    int prev = -1;
    for (int j = 0; j < sp.npages && !bad; ++j) {
      const PageRef r = page_ref(a, sp, 0, j);
      if (r.err != 0 || r.lp <= prev || r.pb != table[r.lp]) bad = true;
      prev = r.lp;
      for (int row = 0; row < kPage && !bad; ++row) {
        const int p = r.lp * kPage + row;
        if (row_visible(sp, p)) line += " " + std::to_string(p);
      }
    }
    std::puts(bad ? "bad" : line.c_str());
  }
  return 0;
}

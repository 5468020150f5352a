// Host-side check of the chunk plan: every (sequence, kv head, unit, key block) is
// covered by exactly one chunk, where the key blocks of a sequence are its 128-key
// prefix blocks followed by its tree block; chunk ids are dense, and the per-sequence
// chunk ranges that the combine kernel uses agree with locate_chunk.
// Usage: plan_check B Hq Hkv T C uniform_n L_0 ... L_{B-1}   (exit 0 = pass); with
// PLAN_CHECK_NO_TREE set, the key lists hold the prefix blocks only; with
// PLAN_CHECK_WINDOW=W, a sliding window of W positions: the attended range must start on
// a block boundary at or before the root's first visible key, L + 1 - W, and the per-row
// cut must land exactly on L + depth + 1 - W.
#include <cstdio>
#include <cstdlib>
#include <map>
#include <tuple>
#include <vector>

#include "ls_plan.cuh"

int main(int argc, char** argv) {
  if (argc < 7) return 2;
  ls::Plan p{};
  p.B = atoi(argv[1]);
  p.Hq = atoi(argv[2]);
  p.Hkv = atoi(argv[3]);
  p.T = atoi(argv[4]);
  p.C = atoi(argv[5]);
  p.uniform_n = atoi(argv[6]);
  p.d = 128;
  p.g = p.Hq / p.Hkv;
  p.rows = p.T * p.g;
  p.tpu = ls::kUnitRows / p.g;
  p.rg = ls::ceil_div(p.T, p.tpu);
  p.with_tree = getenv("PLAN_CHECK_NO_TREE") ? 0 : 1;  // prefix-only plans (cross-attention)
  p.window = getenv("PLAN_CHECK_WINDOW") ? atoi(getenv("PLAN_CHECK_WINDOW")) : 0;
  if (argc != 7 + p.B) return 2;
  std::vector<int32_t> cu(p.B + 1, 0);
  for (int b = 0; b < p.B; ++b) cu[b + 1] = cu[b] + atoi(argv[7 + b]);
  int32_t total = 0, first = 0, per = 0;
  ls::sequence_chunks(p, cu.data(), 0, &first, &per, &total);
  p.n_chunks = total;
  std::map<std::tuple<int, int, int, int>, int> seen;  // (b, kh, rg, block) -> count
  for (int cid = 0; cid < total; ++cid) {
    ls::ChunkCoord c = ls::locate_chunk(p, cu.data(), cid);
    if (!c.valid) { printf("chunk %d invalid\n", cid); return 1; }
    int32_t f, n, t;
    ls::sequence_chunks(p, cu.data(), c.b, &f, &n, &t);
    const int expect = f + (c.kh * p.rg + c.rgi) * n + c.split;
    if (expect != cid) { printf("chunk %d: combine index %d\n", cid, expect); return 1; }
    if (c.key_end > c.key_begin && c.key_begin % ls::kBlockN) { printf("chunk %d unaligned start\n", cid); return 1; }
    const int nblk = ls::ceil_div(c.key_end - c.key_begin, ls::kBlockN) + (c.has_tree ? 1 : 0);
    if (nblk > p.C) { printf("chunk %d too long\n", cid); return 1; }
    const int Lb = cu[c.b + 1] - cu[c.b];
    const int s0 = ls::window_start(p, Lb);
    if (c.seq_offset != cu[c.b] + s0 || c.key_skip != s0) { printf("chunk %d offset\n", cid); return 1; }
    for (int k = c.key_begin; k < c.key_end; k += ls::kBlockN)
      seen[std::make_tuple(c.b, c.kh, c.rgi, k / ls::kBlockN)]++;
    // the tree block is block number prefix_blocks(L) of the sequence's list
    if (c.has_tree) seen[std::make_tuple(c.b, c.kh, c.rgi, ls::prefix_blocks(ls::attended_len(p, Lb)))]++;
  }
  if (ls::locate_chunk(p, cu.data(), total).valid) { printf("chunk past the end is valid\n"); return 1; }
  for (int b = 0; b < p.B; ++b) {
    const int L = cu[b + 1] - cu[b];
    const int s0 = ls::window_start(p, L);
    if (ls::attended_len(p, L) != (L > 0 ? L - s0 : 0)) return 1;
    if (p.window > 0 && L > 0) {
      const int first = L + 1 - p.window > 0 ? L + 1 - p.window : 0;  // root's first visible key
      if (s0 % ls::kBlockN || s0 > first || first - s0 >= ls::kBlockN) { printf("window start %d\n", s0); return 1; }
      for (int dep = 0; dep < p.T; ++dep) {
        const int want = L + dep + 1 - p.window;  // first visible key of a row at this depth
        const int cut = ls::window_cut(p, L, dep);
        if (s0 + cut != (want > s0 ? want : s0)) { printf("cut at depth %d\n", dep); return 1; }
      }
    } else if (s0 != 0 || ls::window_cut(p, L, 3) != 0) {
      return 1;
    }
    for (int kh = 0; kh < p.Hkv; ++kh)
      for (int r = 0; r < p.rg; ++r)
        for (int k = 0; k < ls::prefix_blocks(ls::attended_len(p, L)) + p.with_tree; ++k) {
          auto it = seen.find(std::make_tuple(b, kh, r, k));
          if (it == seen.end() || it->second != 1) {
            printf("block (%d,%d,%d,%d) covered %d times\n", b, kh, r, k,
                   it == seen.end() ? 0 : it->second);
            return 1;
          }
        }
  }
  printf("ok %d chunks\n", total);
  return 0;
}

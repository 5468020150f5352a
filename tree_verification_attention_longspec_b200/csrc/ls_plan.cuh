// Work split and workspace layout shared by the host launcher and the kernels.
//
// The attention work is cut into chunks. A chunk is one (sequence b, kv head kh, unit
// u, range of key blocks) and becomes one CTA of the partials kernel. The query rows of
// a kv head are its T*g (tree node i, head-in-group j) pairs; a unit holds the rows of
// tpu = floor(256 / g) consecutive tree nodes, so its rows are whole nodes (at most 256
// of them, row (i - u*tpu)*g + j of the unit) and one TMA box brings them in.
// The keys of sequence b form ceil(L_b / 128) prefix blocks ("Cached-Teil", no mask)
// followed by one block of its T <= 128 tree keys ("Speculative-Teil", tree mask).
// A sequence's list is cut into n = ceil(blocks / C) chunks of consecutive blocks, as
// even as possible, so the chunk that holds the tree block also attends the last prefix
// keys, and a sequence without prefix still has one chunk. The chunk grid follows from
// the prefix lengths and C alone, and the device recomputes it from cu_seqlens without
// any table in memory.
// Trees may differ in size per sequence (cu_tree): the grid is then planned for T, the
// largest tree allowed, and units past a sequence's own tree have no rows.
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define LS_HD __host__ __device__ __forceinline__
#else
#define LS_HD inline
#endif

namespace ls {

constexpr int kBlockN = 128;       // keys per block of the prefix loop
constexpr int kUnitRows = 256;     // query rows per prefix chunk (two 128-row MMA tiles)
constexpr int kMaxTree = 128;      // largest supported tree (one key block)
constexpr int kMergeRows = 4;      // output rows per CTA of the combine kernel (a warp each)
constexpr int kPlanCu = 33;        // host lengths carried in the plan for batches up to 32

// device-side status bits (combined into one LS_ERR_* by ls_verify_attn_check)
constexpr uint32_t kErrBadTree = 1u;
constexpr uint32_t kErrLengths = 2u;
constexpr uint32_t kErrTimeout = 4u;
constexpr uint32_t kErrIndex = 8u;  // index-checking (LS_DEBUG) builds: an address outside its extent

// The index checks of the LS_DEBUG build: every TMA coordinate and global index the
// kernels form is checked against the extent of the tensor it addresses, and a failed
// check records kErrIndex in `flag` (reported through the call's status). Release
// builds compile the checks away.
#if defined(LS_DEBUG)
#define LS_DCHECK(flag, ok)                    \
  do {                                         \
    if (!(ok)) (flag) |= ::ls::kErrIndex;      \
  } while (0)
#else
#define LS_DCHECK(flag, ok) \
  do {                      \
  } while (0)
#endif

struct Plan {
  int32_t B, Hq, Hkv, d, T, g;  // T: tree nodes per sequence (the largest, with cu_tree)
  int32_t N;           // tree nodes of the batch: B * T, or cu_tree[B]
  int32_t rope;        // 1: q and k_tree are rotated (RoPE) by the tree kernel first
  int32_t window;      // > 0: sliding window of this many positions; 0: the whole prefix
  int32_t rows;        // T * g query rows per (sequence, kv head)
  int32_t tpu;         // tree nodes per unit: floor(kUnitRows / g)
  int32_t rg;          // units per (sequence, kv head): ceil(T / tpu)
  int32_t C;           // 128-key blocks per chunk
  int32_t with_tree;   // 1: every key list ends with the tree block; 0: prefix keys only
  int32_t uniform_n;   // >= 0: chunks per unit for every sequence; -1: from L_b
  int32_t n_chunks;    // partials-kernel CTAs
  int32_t n_combine;   // combine CTAs = ceil(B * T * Hq / kMergeRows), or B * T * Hq when wide
  int32_t combine_wide;  // 1: one output row per combine CTA, its warps splitting the row's partials
  float scale;         // softmax scale
  float scale_log2;    // softmax scale * log2(e)
  // The host copy of cu_seqlens, when the caller gave one and B < kPlanCu: the kernels
  // address keys with it (kernel parameters, no memory round trip at start-up); the
  // combine checks that the device array agrees. cu_n = 0: the device array is used.
  int32_t cu_n;
  int32_t cu_host[kPlanCu];
  // Longest time any bounded device-side wait of the partials kernel may take before the
  // call gives up and reports kErrTimeout (nanoseconds of %globaltimer).
  int64_t wait_ns;
};

// The offsets the kernels address keys with: the plan's host copy, else the device array.
LS_HD const int32_t* plan_cu(const Plan& p, const int32_t* cu_dev) { return p.cu_n ? p.cu_host : cu_dev; }

LS_HD int32_t ceil_div(int32_t a, int32_t b) { return (a + b - 1) / b; }

// 128-key blocks of a prefix of L keys
LS_HD int32_t prefix_blocks(int32_t L) { return L > 0 ? ceil_div(L, kBlockN) : 0; }

// Sliding window (draft self-attention; LongSpec, gist.science summary, section 2A): a
// query at position P sees the keys at positions P - window + 1 .. P. Node i sits at
// position L + depth(i) and prefix key j at position j, so the root sees the prefix keys
// from L + 1 - window on and deeper nodes fewer (a per-row cut, `window_cut`). The
// attended range [window_start, L) is what every row of the sequence may need, started
// on a 128-key boundary (so that a block never straddles two pages of a paged cache);
// the keys before the exact start are cut for every row. window = 0: the whole prefix.
LS_HD int32_t window_start(const Plan& p, int32_t L) {
  if (p.window <= 0 || L <= 0) return 0;
  const int32_t s = L + 1 - p.window;
  return s <= 0 ? 0 : s / kBlockN * kBlockN;
}

// prefix keys of a sequence of L keys that its rows may attend
LS_HD int32_t attended_len(const Plan& p, int32_t L) {
  if (L <= 0) return 0;
  return L - window_start(p, L);
}

// The first attended key (index into [window_start, L)) that a row at tree depth `depth`
// may see; 0 without a window.
LS_HD int32_t window_cut(const Plan& p, int32_t L, int32_t depth) {
  if (p.window <= 0 || L <= 0) return 0;
  const int32_t c = L + depth + 1 - p.window - window_start(p, L);
  return c > 0 ? c : 0;
}

// chunks of one (sequence, kv head, unit) for a prefix of L keys: its attended prefix
// blocks and (with_tree) the tree block, C per chunk
LS_HD int32_t chunks_per_unit(const Plan& p, int32_t L) {
  if (p.uniform_n >= 0) return p.uniform_n;
  return ceil_div(prefix_blocks(attended_len(p, L)) + p.with_tree, p.C);
}

// Tree nodes of sequence b: rows [*base, *base + *n) of q, k_tree, v_tree, tree_parent,
// out and lse. Without cu_tree every sequence has T nodes. A cu_tree entry that does
// not describe a packed layout (cu_tree[0] = 0, non-decreasing, cu_tree[B] = N, at most
// T nodes a tree) gives the sequence no node and returns false.
LS_HD bool tree_range(const Plan& p, const int32_t* cu_tree, int32_t b, int32_t* base, int32_t* n) {
  if (cu_tree == nullptr) {
    *base = b * p.T;
    *n = p.T;
    return true;
  }
  const int32_t s = cu_tree[b], e = cu_tree[b + 1];
  const bool ok = s >= 0 && e >= s && e <= p.N && e - s <= p.T && (b > 0 || s == 0) && (b < p.B - 1 || e == p.N);
  *base = ok ? s : 0;
  *n = ok ? e - s : 0;
  return ok;
}

// A unit of at most 128 existing rows is run with both query tiles on its rows, taking
// alternate key blocks, and leaves two partials per chunk (rows r and r + 128 of the
// chunk's slot).
LS_HD bool unit_alternates(int32_t rows_here) { return rows_here <= 128; }

// Unit and row inside the unit of query row (tree node i, head-in-group j).
LS_HD void unit_row(const Plan& p, int32_t i, int32_t j, int32_t* unit, int32_t* row) {
  *unit = i / p.tpu;
  *row = (i - *unit * p.tpu) * p.g + j;
}

struct ChunkCoord {
  int32_t b, kh, rgi, split, n_split;  // sequence, kv head, unit, split index, splits of unit
  int32_t key_begin, key_end;          // attended key range of the chunk (from window_start)
  int32_t key_skip;                    // window_start: prefix keys before the attended range
  int32_t seq_offset;                  // cu_seqlens[b] + key_skip
  bool has_tree;                       // the chunk also attends the tree block
  bool valid;
};

// Finds chunk `cid` by walking the sequences in order (B is small).
LS_HD ChunkCoord locate_chunk(const Plan& p, const int32_t* cu, int32_t cid) {
  ChunkCoord c{};
  c.valid = false;
  int32_t base = 0;
  const int32_t units = p.Hkv * p.rg;
  for (int32_t b = 0; b < p.B; ++b) {
    const int32_t L = cu[b + 1] - cu[b];
    const int32_t n = chunks_per_unit(p, L);
    const int32_t nb = n * units;
    if (cid < base + nb) {
      const int32_t local = cid - base;
      const int32_t u = local / n;
      c.b = b;
      c.kh = u / p.rg;
      c.rgi = u % p.rg;
      c.split = local % n;
      c.n_split = n;
      c.key_skip = window_start(p, L);
      c.seq_offset = cu[b] + c.key_skip;
      const int32_t Lc = attended_len(p, L);
      // The key list's blocks are cut into n runs of consecutive blocks as even as
      // possible (their lengths differ by at most one, none longer than C): blocks [v0, v1).
      const int32_t nbl = prefix_blocks(Lc) + p.with_tree;
      const int32_t v0 = (int32_t)((int64_t)c.split * nbl / n), v1 = (int32_t)((int64_t)(c.split + 1) * nbl / n);
      const int32_t kb = v0 * kBlockN, ke = v1 * kBlockN;
      c.key_begin = kb < Lc ? kb : Lc;
      c.key_end = ke < Lc ? ke : Lc;
      const int32_t tree_block = prefix_blocks(Lc);
      c.has_tree = p.with_tree && v0 <= tree_block && tree_block < v1;
      c.valid = true;
      return c;
    }
    base += nb;
  }
  return c;
}

// First chunk id of sequence b's units and the chunks per unit; also the total.
LS_HD void sequence_chunks(const Plan& p, const int32_t* cu, int32_t b, int32_t* first,
                           int32_t* per_unit, int32_t* total) {
  int32_t base = 0, f = 0, n_b = 0;
  const int32_t units = p.Hkv * p.rg;
  for (int32_t s = 0; s < p.B; ++s) {
    const int32_t n = chunks_per_unit(p, cu[s + 1] - cu[s]);
    if (s == b) { f = base; n_b = n; }
    base += n * units;
  }
  *first = f;
  *per_unit = n_b;
  *total = base;
}

// Workspace layout (byte offsets, each 256-aligned). The combine's status words come
// first, so that their place depends on the output rows alone, not on the chunk plan.
struct Layout {
  uint64_t status;        // u32   [n_combine]
  uint64_t o_part;        // float [n_chunks][kUnitRows][d]   partial out, normalised
  uint64_t lse_part;      // float [n_chunks][kUnitRows]      partial lse, log2 domain
  uint64_t chunk_status;  // u32   [n_chunks]
  uint64_t q_rot;         // bf16  [N][Hq][d]    rotated queries (rope only)
  uint64_t k_rot;         // bf16  [N][Hkv][d]   rotated tree keys (rope only)
  uint64_t rope_status;   // u32   [B*T]         index-check result of each tree-kernel CTA (rope only)
  uint64_t total;
};

LS_HD uint64_t align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

LS_HD Layout make_layout(const Plan& p) {
  Layout l{};
  uint64_t off = 0;
  l.status = off;
  off = align256(off + (uint64_t)p.n_combine * 4);
  l.o_part = off;
  off = align256(off + (uint64_t)p.n_chunks * kUnitRows * p.d * 4);
  l.lse_part = off;
  off = align256(off + (uint64_t)p.n_chunks * kUnitRows * 4);
  l.chunk_status = off;
  off = align256(off + (uint64_t)p.n_chunks * 4);
  const uint64_t nq = p.rope ? (uint64_t)p.N * p.Hq * p.d * 2 : 0, nk = p.rope ? (uint64_t)p.N * p.Hkv * p.d * 2 : 0;
  l.q_rot = off;
  off = align256(off + nq);
  l.k_rot = off;
  off = align256(off + nk);
  l.rope_status = off;
  off = align256(off + (p.rope ? (uint64_t)p.B * p.T * 4 : 0));
  l.total = off;
  return l;
}

}  // namespace ls

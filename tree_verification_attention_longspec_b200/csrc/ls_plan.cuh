// Work split and workspace layout shared by the host launcher and the kernels.
//
// The prefix ("Cached-Teil") work is cut into chunks. A chunk is one
// (sequence b, kv head kh, unit u, key range) and becomes one CTA of the prefix
// kernel. The query rows of a kv head are its T*g (tree node i, head-in-group j)
// pairs; a unit holds the rows of tpu = floor(256 / g) consecutive tree nodes, so its
// rows are whole nodes (at most 256 of them, row (i - u*tpu)*g + j of the unit) and
// one TMA box brings them in. Every chunk of a sequence covers C consecutive 128-key
// blocks (the last one fewer), so the chunk grid follows from the prefix lengths and
// C alone, and the device recomputes it from cu_seqlens without any table in memory.
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
constexpr int kMaxTree = 128;      // largest supported tree

// device-side status bits (combined into one LS_ERR_* by ls_verify_attn_check)
constexpr uint32_t kErrBadTree = 1u;
constexpr uint32_t kErrLengths = 2u;
constexpr uint32_t kErrTimeout = 4u;

struct Plan {
  int32_t B, Hq, Hkv, d, T, g;
  int32_t rows;        // T * g query rows per (sequence, kv head)
  int32_t tpu;         // tree nodes per unit: floor(kUnitRows / g)
  int32_t rg;          // units per (sequence, kv head): ceil(T / tpu)
  int32_t C;           // 128-key blocks per chunk
  int32_t uniform_n;   // >= 0: chunks per unit for every sequence; -1: from L_b
  int32_t n_chunks;    // prefix CTAs
  int32_t n_combine;   // tree/combine CTAs = B * T * Hkv
  float scale;         // softmax scale
  float scale_log2;    // softmax scale * log2(e)
};

LS_HD int32_t ceil_div(int32_t a, int32_t b) { return (a + b - 1) / b; }

// chunks of one (sequence, kv head, unit) for a prefix of L keys
LS_HD int32_t chunks_per_unit(const Plan& p, int32_t L) {
  if (p.uniform_n >= 0) return p.uniform_n;
  if (L <= 0) return 0;
  return ceil_div(ceil_div(L, kBlockN), p.C);
}

// Unit and row inside the unit of query row (tree node i, head-in-group j).
LS_HD void unit_row(const Plan& p, int32_t i, int32_t j, int32_t* unit, int32_t* row) {
  *unit = i / p.tpu;
  *row = (i - *unit * p.tpu) * p.g + j;
}

struct ChunkCoord {
  int32_t b, kh, rgi, split, n_split;  // sequence, kv head, unit, split index, splits of unit
  int32_t key_begin, key_end;          // key range inside the sequence's prefix
  int32_t seq_offset;                  // cu_seqlens[b]
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
      c.seq_offset = cu[b];
      const int32_t Lc = L < 0 ? 0 : L;
      int32_t kb = c.split * p.C * kBlockN;
      int32_t ke = kb + p.C * kBlockN;
      c.key_begin = kb < Lc ? kb : Lc;
      c.key_end = ke < Lc ? ke : Lc;
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

// Workspace layout (byte offsets, each 256-aligned).
struct Layout {
  uint64_t o_part;        // float [n_chunks][kUnitRows][d]   prefix partial out, normalised
  uint64_t lse_part;      // float [n_chunks][kUnitRows]      prefix partial lse, log2 domain
  uint64_t chunk_status;  // u32   [n_chunks]
  uint64_t status;        // u32   [n_combine]
  uint64_t total;
};

LS_HD uint64_t align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

LS_HD Layout make_layout(const Plan& p) {
  Layout l{};
  uint64_t off = 0;
  l.o_part = off;
  off = align256(off + (uint64_t)p.n_chunks * kUnitRows * p.d * 4);
  l.lse_part = off;
  off = align256(off + (uint64_t)p.n_chunks * kUnitRows * 4);
  l.chunk_status = off;
  off = align256(off + (uint64_t)p.n_chunks * 4);
  l.status = off;
  off = align256(off + (uint64_t)p.n_combine * 4);
  l.total = off;
  return l;
}

}  // namespace ls

// Attention partials on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// LongSpec, gist.science summary, section 2C: the cached prefix is attended with no
// mask ("Cached-Teil"), the speculative tree tokens under the tree mask
// ("Speculative-Teil"), and the partial results are joined by log-sum-exp
// ("Aggregation"). With grouped-query attention the T*g (tree node, head-in-group) rows
// of one kv head share every key, so each part is a dense contraction: S = Q K^T and
// O += P V. One CTA handles one chunk: a 256-row unit of one (sequence, kv head), as two
// 128-row query tiles, against a run of 128-key blocks; the chunk that ends the
// sequence's key list also takes the block of its T <= 128 tree keys, with every score
// outside the row's ancestor-or-self set masked. A masked block is one more step of the
// same online softmax, which is the log-sum-exp join itself. The CTA leaves its partial
// (out normalised by its own sum; lse in the log2 domain) for the combine kernel.
//
// Ping-pong. Each query tile t has one softmax warpgroup, one score buffer S_t and one
// output accumulator O_t in TMEM. The MMA thread walks the key blocks and, per block j,
// issues O_0 += P_0(j) V(j), S_0(j+1) = Q_0 K(j+1)^T, then the same for tile 1. While
// the tensor core works for one tile, the other tile's warpgroup runs its softmax, so
// the exponentials of one tile overlap the other tile's MMAs, and the special-function
// unit (MUFU), which bounds the softmax, is shared by two warpgroups that are out of
// phase. Every K/V tile staged in shared memory serves both query tiles.
//
// Alternate blocks. When a unit has at most 128 query rows (a small tree, a single draft
// query, the last nodes of a tree), the second tile would hold only padding. Both tiles then take
// the same rows and alternate key blocks: tile 0 the even blocks of the chunk, tile 1 the
// odd ones, each with its own S, O and running max, so two chains advance through one
// key range; their results are two partials of the chunk (rows 0..127 and 128..255 of
// its slot), merged by the combine like any other.
//
// Warp roles (320 threads, one CTA per SM):
//   warps 0-3  softmax of tile 0, warps 4-7 of tile 1: one thread per query row (= TMEM
//              lane) holding the block's 128 scores. P is computed against the running
//              max m in one pass; only when a block's maximum exceeds m by more than 2^8
//              is m raised and O_t rescaled in TMEM. P (bf16) overwrites the scores in
//              two halves of 64 keys, each announced on its own barrier, so the MMA
//              thread starts on the first half while the second is computed.
//   warp 8     TMA producer: Q, then 128-key K and V blocks (prefix, then tree) into a
//              ring of slots.
//   warp 9     MMA issuer (one thread): S = Q K^T (shared-memory operands, N = 128) and
//              O += P V (P from TMEM, N = d), tcgen05.commit to mbarriers.
// TMEM columns (512 allocated): S_t at 128 t, O_t at 256 + d t.
// Every wait is bounded (the call's wait limit, 4 s by default): on a timeout the CTA
// raises an abort flag, all roles drain their in-flight copies and MMAs, TMEM is freed,
// and the chunk status reports it.
#include <cudaTypedefs.h>

#include "ls_device.cuh"
#include "sm100.cuh"

namespace ls {
namespace {
using namespace sm100;

constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kMaxSlots = 12;
constexpr int kTiles = 2;  // 128-row query tiles per CTA
constexpr int kHalf = 64;  // keys per P half
// Draining after an abort waits for copies and MMAs that were issued and always
// complete; its own bound is fixed (the call's wait limit may be far shorter).
constexpr uint64_t kDrainNs = 4000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
static_assert(kUnitRows == kTiles * 128, "a unit is two 128-row tiles");

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kPanelBytes = 128 * 128;             // 128 rows x 64 bf16, 128B-swizzled
  static constexpr int kTileBytes = kPanels * kPanelBytes;  // 128 rows x D bf16
  static constexpr int kSlots = D == 128 ? 5 : 12;
  // Q: [panel][kUnitRows rows][128 B]; tile t is rows [128 t, 128 t + 128) of each panel
  static constexpr int kQPanelBytes = kUnitRows * 128;
  static constexpr int kQOff = 0;
  static constexpr int kSlotOff = kPanels * kQPanelBytes;
  static constexpr int kBarOff = kSlotOff + kSlots * kTileBytes;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;    // S_t / P_t at 128 t
  static constexpr uint32_t kColO = 256;  // O_t at 256 + D t
  static_assert(kSlots <= kMaxSlots, "slots");
  static_assert(kPanels * kQPanelBytes >= 128 * D * 4 && kSlots * kTileBytes >= 128 * D * 4, "epilogue staging");
};

struct alignas(64) TcParams {
  CUtensorMap tmap_q;
  CUtensorMap tmap_k;   // prefix keys
  CUtensorMap tmap_v;
  CUtensorMap tmap_kt;  // tree keys
  CUtensorMap tmap_vt;
  CUtensorMap tmap_o;   // o_part as [n_chunks * 256 rows][d] fp32, stores of 128 rows x 32 floats
  PartialsArgs a;
};

struct Bars {
  uint64_t q_full;  // the unit's Q rows are in shared memory
  uint64_t full[kMaxSlots];
  uint64_t empty[kMaxSlots];
  uint64_t s_full[kTiles];     // S_t(j) is in TMEM (and O_t holds every PV before it)
  uint64_t p_full[kTiles][2];  // half h of P_t(j) is in TMEM
  uint64_t o_full[kTiles];     // every MMA of tile t finished
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t tree_err;          // a parent link that is not a rooted tree's
  uint32_t dbg;               // index-checking builds: kErrIndex once a check failed
  int16_t parent[kMaxTree];   // the sequence's tree (chunks that hold the tree block)
};

// The kernel asks for the dynamic window of a CTA less 1 KB and aligns its layout up to
// 1024 bytes inside it (the 128-byte
// swizzle atom repeats every 1024 bytes).
constexpr int kSmemWindow = 232448 - 1024;
template <int D>
constexpr int smem_need() {
  return Cfg<D>::kBarOff + (int)sizeof(Bars) + 1024;
}
static_assert(smem_need<128>() <= kSmemWindow && smem_need<64>() <= kSmemWindow, "shared memory");

// AND of `pred` over the `n` threads that meet at named barrier `id`.
__device__ __forceinline__ bool bar_and(uint32_t id, uint32_t n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// Waits only on time (used to drain in-flight work after an abort).
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  uint32_t never = 0;
  return mbar_wait_bounded(bar, parity, &never, kDrainNs);
}

// P = 2^(s*cs - m) for 64 scores, packed to bf16 pairs; adds the values to (sum0, sum1)
// and their bf16 roundings, the weights the PV product uses, to (rsum0, rsum1). The
// output is normalised by the rounded sum, so that it is a convex combination of the
// values with exactly those weights (their rounding, relative 2^-9 each, then cancels
// where the values agree); the lse keeps the exact sum. EMU of every 4 pairs use the
// FMA-pipe exponential. Every block takes this one path,
// masked or not (one copy of the loop keeps the softmax's code small; a second, MUFU-only
// copy for masked blocks cost 6% in time): a masked score (-inf) gives 0 on the MUFU
// and 2^-125 on the FMA pipe, which clamps its input there, and 2^-125 is nothing next
// to the row's own maximum term, 1 (or, in a row with no visible key yet, m stays -inf
// and a later raise multiplies the sums by 2^-inf = 0).
template <int EMU>
__device__ __forceinline__ void make_p(const float (&s)[kHalf], float cs, float m, uint32_t (&pk)[kHalf / 2],
                                       float& sum0, float& sum1, float& rsum0, float& rsum1) {
  const float nm = -m;
#pragma unroll
  for (int e = 0; e < kHalf / 2; ++e) {
    float x0, x1, p0, p1;
    fma2_bc(x0, x1, s[2 * e], s[2 * e + 1], cs, nm);
    if ((e & 3) < EMU) {
      exp2_poly_x2(x0, x1, p0, p1);
    } else {
      p0 = ex2_approx(x0);
      p1 = ex2_approx(x1);
    }
    add2(sum0, sum1, p0, p1);
    pk[e] = pack_bf16x2(p0, p1);
    add_bf16x2_to_f32(rsum0, rsum1, pk[e]);
  }
}

// Tree mask (LongSpec, gist.science summary, section 2C, "Baum-Maskierung") on the
// scores of the tree block in this thread's TMEM lane: key x (tree node x) stays visible
// when x is the row's node or one of its ancestors, found by following parent links.
// Every link is checked (node 0 is the root with parent -1, any other node's parent
// lies below it), so the walk ends; a failed check raises `bad`. node < 0 (a padding
// row) masks every key. The scores go back to TMEM as -inf where masked.
__device__ __forceinline__ bool mask_tree_scores(const int16_t* parent, uint32_t tS, int node) {
  uint32_t am[4] = {0u, 0u, 0u, 0u};
  bool bad = false;
  if (node >= 0) {
    int x = node;
    for (int step = 0; step <= kMaxTree; ++step) {
      const uint32_t bit = 1u << (x & 31);
      const int w = x >> 5;
      am[0] |= w == 0 ? bit : 0u;
      am[1] |= w == 1 ? bit : 0u;
      am[2] |= w == 2 ? bit : 0u;
      am[3] |= w == 3 ? bit : 0u;
      const int pp = parent[x];
      if (x == 0) {
        bad = pp != -1;
        break;
      }
      if (pp < 0 || pp >= x) {
        bad = true;
        break;
      }
      x = pp;
    }
  }
  __syncwarp();  // the TMEM accesses below are warp-collective
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t r[32];
    tmem_ld32(tS + 32 * q, r);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (!((am[q] >> e) & 1u)) r[e] = __float_as_uint(-INFINITY);
    tmem_st32(tS + 32 * q, r);
  }
  tmem_wait_st();
  return bad;
}

// GENERAL = false: the instance for a packed cache and the whole prefix; the paged and
// sliding-window paths are compiled out of it, which keeps the code the block loop
// fetches smaller (2% on the Qwen-7B layer). GENERAL = true: every path, chosen at run
// time. Both wait for the tree kernel when it rotates q and k_tree first.
template <int D, int EMU, bool GENERAL>
__global__ void __launch_bounds__(kThreads, 1) partials_tc_kernel(const __grid_constant__ TcParams P) {
  using C = Cfg<D>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kBarOff);
  const PartialsArgs& a = P.a;
  const Plan& p = a.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint64_t wait_ns = (uint64_t)p.wait_ns;  // limit of every bounded wait below

  const int32_t* cu = plan_cu(p, a.cu);  // kernel parameters when the host gave lengths
  const ChunkCoord c = locate_chunk(p, cu, blockIdx.x);
  if (!c.valid) return;  // more CTAs than the device lengths need: the combine reports it
  const int n_keys = c.key_end - c.key_begin;
  const int nb = (n_keys + kBlockN - 1) / kBlockN;  // prefix blocks
  // The last prefix block of a packed cache is loaded as the box that ends at the
  // sequence end (its leading tail_shift columns are earlier keys, masked); in a paged
  // cache it is loaded from its aligned start, page by page, and its columns from
  // tail_end on lie past the sequence end (masked).
  const bool paged = GENERAL && a.page_table != nullptr;
  const int tail_shift = paged ? 0 : nb * kBlockN - n_keys;
  const int tail_end = paged ? n_keys - (nb - 1) * kBlockN : kBlockN;
  const bool has_tree = c.has_tree;
  const int nbt = nb + (has_tree ? 1 : 0);  // blocks, the tree block (block nb) last
  const int seq_len = cu[c.b + 1] - cu[c.b];
  // sliding window: a row at depth d sees the attended keys from window_cut(d) on, which
  // is below 2 * 128, so only the chunks that start there cut rows individually
  const bool win_rows = GENERAL && p.window > 0 && nb > 0 && c.key_begin < 2 * kBlockN;
  int tree_base, tree_n;  // the sequence's tree nodes (none if cu_tree is bad: the combine reports it)
  tree_range(p, a.cu_tree, c.b, &tree_base, &tree_n);
  const int tok0 = c.rgi * p.tpu;                       // first tree node of the unit
  const int rows_here = min(p.tpu, tree_n - tok0) * p.g;  // rows of the unit that exist
  const bool alt = unit_alternates(rows_here);             // both tiles on these rows
  if (rows_here <= 0) {  // a unit past the sequence's tree: nothing to attend for
    if (tid == 0) a.chunk_status[blockIdx.x] = 0u;
    return;
  }
  if (nbt == 0) {  // empty key range: an empty partial (two of them when the tiles alternate)
    for (int r = tid; r < rows_here; r += kThreads) {
      a.lse_part[(size_t)blockIdx.x * kUnitRows + r] = -INFINITY;
      if (alt) a.lse_part[(size_t)blockIdx.x * kUnitRows + 128 + r] = -INFINITY;
    }
    if (tid == 0) a.chunk_status[blockIdx.x] = 0u;
    return;
  }

  volatile uint32_t* abort = &bars->abort;
  // ------------------------------------------------------------------ TMA producer state
  // Ring order = consumption order: K(0), V(0), K(1), V(1), ... The whole warp walks the
  // blocks; lane 0 arms the barriers and issues whole-block boxes, and for a paged cache
  // the lanes issue the block's page boxes (and read their page-table entries) at once.
  // The producer sets up the barriers and issues Q and K(0) before the CTA-wide barrier,
  // so that the first tiles are in flight while the other warps set up.
  // Q: one box per 64-column panel, tpu nodes x g heads of kv head kh (rows past the
  // batch's last node read as zeros)
  auto load_q = [&]() {
#if defined(LS_DEBUG)
    // the unit's existing nodes lie inside q (the box rows after them read zeros)
    if (lane == 0 && !(tok0 >= 0 && tok0 < tree_n && tree_base >= 0 && tree_base + tree_n <= p.N)) bars->dbg = kErrIndex;
#endif
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars->q_full, C::kPanels * 128 * p.g * p.tpu);
#pragma unroll
      for (int pn = 0; pn < C::kPanels; ++pn)
        tma_load_4d(smem + C::kQOff + pn * C::kQPanelBytes, &P.tmap_q, &bars->q_full, pn * 64, 0, c.kh,
                    tree_base + tok0);
    }
  };
  // When the tree kernel writes q and k_tree (rotated), this grid may start before
  // that grid ends: the prefix loads go ahead, Q and the tree block wait for it.
  bool prior_done = !a.after_prep;
  auto wait_prior = [&]() {
    if (!prior_done) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      prior_done = true;
    }
  };
  bool q_loaded = false;
  // a page box is bh rows (the page, or 128 rows of a larger page); lane l issues box
  // l / kPanels, panel l % kPanels
  const int bh = paged ? (a.page_size < kBlockN ? a.page_size : kBlockN) : kBlockN;
  const int n_boxes = (kBlockN / bh) * C::kPanels;
  const int n_pages = paged ? (seq_len + a.page_size - 1) / a.page_size : 0;
  int issued = 0, slot = 0, use = 0;
  // the MMA thread's order: K(j), V(j) for j = 0, 1, ...; with alternate blocks K(0),
  // K(1), then V(j) and K(j + 2) for j = 0, 1, ... (no K past the last block)
  const int n_loads = 2 * nbt;
  const int pro = nbt < 2 ? nbt : 2, pairs = nbt > 2 ? nbt - 2 : 0;
  // Issues load `ld` of the ring once its slot is free; false if the wait gave up.
  auto issue_load = [&](int ld) -> bool {
    int j, kv;
    if (!alt) {
      j = ld >> 1;
      kv = ld & 1;
    } else if (ld < pro) {
      j = ld;
      kv = 0;
    } else if (ld - pro < 2 * pairs) {
      const int r = ld - pro;
      j = (r >> 1) + ((r & 1) ? 2 : 0);
      kv = (r & 1) ? 0 : 1;
    } else {
      j = pairs + (ld - pro - 2 * pairs);
      kv = 1;
    }
    // prefix block j, or the tree block: the sequence's nodes (the rows after them
    // belong to the next sequence or lie past the tensor, read as zeros; masked)
    const bool tree = j == nb;
    int row = c.seq_offset + c.key_begin + j * kBlockN;
    if (j == nb - 1) row -= tail_shift;  // the box ends at the sequence end
    if (tree) {
      row = tree_base;
      wait_prior();
    }
    const bool pieces = paged && !tree;  // the block's rows come page by page
    // this lane's page box of the block: a page-table entry is only a TMA coordinate,
    // so a bad one reads zeros or another page, never outside the cache; boxes past
    // the sequence end read its last page (masked)
    int prow = 0;
    const int pc = lane / C::kPanels, pn_l = lane % C::kPanels;
    if (pieces && lane < n_boxes) {
      const int key = c.key_skip + c.key_begin + j * kBlockN + pc * bh;
      int lp = key / a.page_size;
      if (lp >= n_pages) lp = n_pages - 1;
      if (lp >= a.max_pages) lp = a.max_pages - 1;
      prow = a.page_table[(size_t)c.b * a.max_pages + lp] * a.page_size + key % a.page_size;
    }
#if defined(LS_DEBUG)
    {
      // the rows of the block that are not masked must lie inside the sequence (inside the
      // tree for the tree block) and every box inside the tensor's data
      uint32_t bad = 0u;
      if (tree) {
        LS_DCHECK(bad, tree_base >= 0 && tree_base + tree_n <= p.N);
      } else if (!pieces) {
        const int lo = j == nb - 1 ? tail_shift : 0;
        LS_DCHECK(bad, j >= 0 && j < nb);
        LS_DCHECK(bad, row + lo >= c.seq_offset && row + kBlockN <= cu[c.b + 1]);
        LS_DCHECK(bad, row + kBlockN <= cu[p.B] && (int64_t)row + kBlockN <= a.kv_rows);
      } else if (lane < n_boxes) {
        const int key = c.key_skip + c.key_begin + j * kBlockN + pc * bh;
        if (key < c.key_skip + c.key_end) {  // a box with keys of the sequence (else masked)
          const int lp = key / a.page_size;
          LS_DCHECK(bad, lp < n_pages && lp < a.max_pages && c.b < p.B);
          const int32_t pe = a.page_table[(size_t)c.b * a.max_pages + lp];
          LS_DCHECK(bad, pe >= 0 && (int64_t)pe * a.page_size + bh <= a.kv_rows);
        }
      }
      bad = __reduce_or_sync(0xffffffffu, bad);
      if (lane == 0 && bad) bars->dbg = kErrIndex;
    }
#endif
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars->empty[slot], (use & 1) ^ 1, abort, wait_ns)))
      return false;
    if (lane == 0) mbar_arrive_expect_tx(&bars->full[slot], C::kTileBytes);
    __syncwarp();
    uint8_t* dst = smem + C::kSlotOff + slot * C::kTileBytes;
    const CUtensorMap* map = tree ? (kv ? &P.tmap_vt : &P.tmap_kt) : (kv ? &P.tmap_v : &P.tmap_k);
    if (!pieces) {
      if (lane == 0) {
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d(dst + pn * C::kPanelBytes, map, &bars->full[slot], pn * 64, c.kh, row);
      }
    } else if (lane < n_boxes) {
      tma_load_3d(dst + pn_l * C::kPanelBytes + pc * bh * 128, map, &bars->full[slot], pn_l * 64, c.kh, prow);
    }
    ++issued;
    if (++slot == C::kSlots) {
      slot = 0;
      ++use;
    }
    return true;
  };

  if (warp == kProducerWarp) {
    if (lane == 0) {
      mbar_init(&bars->q_full, 1);
      for (int s = 0; s < C::kSlots; ++s) {
        mbar_init(&bars->full[s], 1);
        mbar_init(&bars->empty[s], 1);
      }
      for (int t = 0; t < kTiles; ++t) {
        mbar_init(&bars->s_full[t], 1);
        mbar_init(&bars->p_full[t][0], 128);
        mbar_init(&bars->p_full[t][1], 128);
      }
      mbar_init(&bars->o_full[0], 1);
      mbar_init(&bars->o_full[1], 1);
      bars->abort = 0u;
      bars->tree_err = 0u;
      bars->dbg = 0u;
      fence_mbar_init();
      tma_prefetch_map(&P.tmap_q);
      tma_prefetch_map(&P.tmap_k);
      tma_prefetch_map(&P.tmap_v);
      tma_prefetch_map(&P.tmap_o);
      if (has_tree) {
        tma_prefetch_map(&P.tmap_kt);
        tma_prefetch_map(&P.tmap_vt);
      }
    }
    __syncwarp();
    // K(0) first, then Q (unless Q waits for the tree kernel): at start-up every CTA asks
    // for just these two, so they arrive quickly instead of sharing the memory system with
    // the whole ring's fill. A fresh barrier never makes the first wait give up.
    issue_load(0);
    if (prior_done) {
      load_q();
      q_loaded = true;
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tbase = bars->tmem_base;
  // the tree/combine kernel may start its own prologue now; it waits for this grid's
  // results before it reads them
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == kProducerWarp) {
    {
      bool ok = true;
      if (!q_loaded) {
        wait_prior();
        load_q();
        q_loaded = true;
      }
      // the rest of the ring once K(0) has landed
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars->full[0], 0, abort, wait_ns))) ok = false;
      for (int ld = 1; ld < n_loads && ok; ++ld) ok = issue_load(ld);
      // make sure no copy is still writing shared memory when the CTA ends
      if (lane == 0) {
        drain_wait(&bars->q_full, 0);
        const int first = issued > C::kSlots ? issued - C::kSlots : 0;
        for (int seq = first; seq < issued; ++seq)
          drain_wait(&bars->full[seq % C::kSlots], (seq / C::kSlots) & 1);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ Q padding (warps 0-7)
    // The TMA box fills rows [0, tpu*g) of each Q panel; the (fewer than g) rows after
    // it are zeroed here so that no stale shared memory enters an MMA.
    if (warp < 8) {
      const int pad0 = p.tpu * p.g;
      const int n16 = (kUnitRows - pad0) * 8;  // 16-byte chunks per panel
      for (int idx = tid; idx < C::kPanels * n16; idx += 256) {
        const int pn = idx / n16, k = idx % n16;
        *reinterpret_cast<uint4*>(smem + C::kQOff + pn * C::kQPanelBytes + pad0 * 128 + k * 16) =
            make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      // the tree of the sequence, for the tree mask; a parent outside [-1, T) is stored
      // as a value that fails the walk's checks
      if (has_tree || win_rows) {
        for (int x = tid; x < tree_n; x += 256) {
#if defined(LS_DEBUG)
          if (!(tree_base + x < p.N)) bars->dbg = kErrIndex;
#endif
          const int32_t pp = a.parent[(size_t)tree_base + x];
          bars->parent[x] = (int16_t)(pp >= -1 && pp < tree_n ? pp : kMaxTree);
        }
      }
    }
    // the padding and the tree are in shared memory: warps 0-7 and the MMA warp meet at
    // barrier 1
    if (warp < 8 || warp == kMmaWarp) asm volatile("bar.sync 1, 288;" ::: "memory");

    if (warp == kMmaWarp) {
      if (lane == 0) {
        // -------------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc_qk = umma_idesc_bf16(128, kBlockN, false);
        constexpr uint32_t idesc_pv = umma_idesc_bf16(128, D, true);
        // A descriptor differs from another of the same kind only in its start-address
        // field (address >> 4 in the low 14 bits; shared addresses stay below 256 KB, so
        // adding an offset never carries out of it): build the bases once, add offsets.
        const uint64_t dq0 = umma_sdesc_sw128(smem_u32(smem + C::kQOff), 16, 1024);
        constexpr uint32_t kQPanel16 = C::kQPanelBytes >> 4, kQTile16 = (128 * 128) >> 4;
        const uint64_t dk0 = umma_sdesc_sw128(smem_u32(smem + C::kSlotOff), 16, 1024);
        const uint64_t dv0 = umma_sdesc_sw128(smem_u32(smem + C::kSlotOff), C::kPanelBytes, 1024);
        constexpr uint32_t kTile16 = C::kTileBytes >> 4, kPanel16 = C::kPanelBytes >> 4;
        // S_t = Q_t K^T into tile t's score buffer; K sits in ring slot `slot`
        auto issue_qk = [&](int t, int slot) {
          const uint64_t dq = dq0 + (uint64_t)((alt ? 0 : t) * kQTile16);  // both tiles read tile 0's Q rows when alternating
          const uint64_t dk = dk0 + (uint64_t)(slot * kTile16);
          const uint32_t tS = tbase + C::kColS + t * kBlockN;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk & 3) * 2;  // 32 bytes per K step inside a panel (16-byte units)
            umma_ss(tS, dq + (kk >> 2) * kQPanel16 + koff, dk + (kk >> 2) * kPanel16 + koff, idesc_qk,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars->s_full[t]);
        };
        // O_t += P_t V over keys [64h, 64h+64) of block j: four K = 16 steps, P from TMEM
        auto issue_pv = [&](int t, int slot, int j, int h) {
          const uint64_t dv = dv0 + (uint64_t)(slot * kTile16);
          const uint32_t tP = tbase + C::kColS + t * kBlockN;
          const uint32_t tO = tbase + C::kColO + t * D;
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int kk = 4 * h + k4;
            umma_ts(tO, tP + kk * 8, dv + kk * (2048 / 16), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          }
        };
        // P written by the softmax warps' tcgen05.st: their wait::st, fence and arrive pair
        // with this wait and the fence after it before an MMA reads P
        auto wait = [&](uint64_t* bar, uint32_t parity) {
          const bool got = mbar_wait_bounded(bar, parity, abort, wait_ns);
          if (got) tc_fence_after_sync();
          return got;
        };
        // Q, K, V written by TMA: the barrier's transaction count completes once the bytes
        // are in shared memory, where the MMAs read them; no tcgen05 fence is needed
        auto wait_tma = [&](uint64_t* bar, uint32_t parity) { return mbar_wait_bounded(bar, parity, abort, wait_ns); };
        int slot = 0, use = 0;  // ring position of the next tile, in consumption order
        auto advance = [&]() {
          if (++slot == C::kSlots) {
            slot = 0;
            use ^= 1;
          }
        };
        bool ok = wait_tma(&bars->q_full, 0);
        if (alt) {
          // alternate blocks: tile t takes blocks t, t + 2, ...; S_t = Q K(t)^T first, then
          // for j = 0, 1, ...: PV of block j for tile j % 2 and that tile's next QK^T
          for (int t = 0; t < kTiles && t < nbt && ok; ++t) {
            ok = wait_tma(&bars->full[slot], use);
            if (!ok) break;
            issue_qk(t, slot);
            umma_commit(&bars->empty[slot]);
            advance();
          }
          for (int j = 0; j < nbt && ok; ++j) {
            const int t = j & 1, i = j >> 1;  // tile and its own block count
            ok = wait_tma(&bars->full[slot], use);  // V(j)
            if (!ok) break;
            const int sv = slot;
            advance();
            ok = wait(&bars->p_full[t][0], i & 1);
            if (!ok) break;
            issue_pv(t, sv, i, 0);
            ok = wait(&bars->p_full[t][1], i & 1);
            if (!ok) break;
            issue_pv(t, sv, i, 1);
            umma_commit(&bars->empty[sv]);
            if (j + 2 < nbt) {
              ok = wait_tma(&bars->full[slot], use);  // K(j + 2)
              if (!ok) break;
              issue_qk(t, slot);
              umma_commit(&bars->empty[slot]);
              advance();
            } else if (t == 0) {
              umma_commit(&bars->o_full[0]);  // tile 0's last PV; no QK^T follows it
            }
          }
        }
        if (ok && !alt) {
          ok = wait_tma(&bars->full[slot], use);  // K(0)
          if (ok) {
            issue_qk(0, slot);
            issue_qk(1, slot);
            umma_commit(&bars->empty[slot]);
            advance();
          }
        }
        for (int j = 0; j < nbt && ok && !alt; ++j) {
          const int sv = slot, uv = use;  // V(j)
          advance();
          const bool more = j + 1 < nbt;
          const int sk = slot, uk = use;  // K(j+1), when there is one
          const uint32_t pp = j & 1;
          ok = wait_tma(&bars->full[sv], uv);
          for (int t = 0; t < kTiles && ok; ++t) {
            ok = wait(&bars->p_full[t][0], pp);
            if (!ok) break;
            issue_pv(t, sv, j, 0);
            ok = wait(&bars->p_full[t][1], pp);
            if (!ok) break;
            issue_pv(t, sv, j, 1);
            // V(j) is free once both tiles' PV have read it: released before the next QK^T,
            // so that its refill (a few microseconds in flight) starts that much earlier
            if (t == 1) umma_commit(&bars->empty[sv]);
            if (!more && t == 0) umma_commit(&bars->o_full[0]);  // tile 0's epilogue may start
            if (more) {
              if (t == 0) ok = wait_tma(&bars->full[sk], uk);
              if (!ok) break;
              issue_qk(t, sk);
            }
          }
          if (!ok) break;
          if (more) {
            umma_commit(&bars->empty[sk]);
            advance();
          }
        }
        // tile 0's last PV precedes tile 1's in issue order, so o_full[1] completes last
        umma_commit(&bars->o_full[1]);
        drain_wait(&bars->o_full[1], 0);
      }
      __syncwarp();
    } else {
      // ---------------------------------------------------------------- softmax / epilogue
      const int t = warp >> 2;                 // query tile
      const int row = (warp & 3) * 32 + lane;  // row of the tile = TMEM lane
      const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
      const uint32_t tS = tbase + lane_base + C::kColS + t * kBlockN;
      const uint32_t tO = tbase + lane_base + C::kColO + t * D;
      const float cs = p.scale_log2;
      // running max (log2 units) of this row, its sum of weights and the sum of their
      // bf16 roundings (the weights in O_t)
      float m = -INFINITY, l = 0.f, lr = 0.f;
      const int ur = alt ? row : t * 128 + row;  // row of the unit (both tiles' rows when alternating)
      const bool has_row = ur < rows_here;
      const int node = tok0 + ur / p.g;   // its tree node
      int cut = 0;                        // window: first attended key this row sees
      if (win_rows && has_row) {
        int x = node, depth = 0;
        for (int step = 0; step < kMaxTree && x > 0; ++step) {
          const int pp = bars->parent[x];
          if (pp < 0 || pp >= x) break;  // not a rooted tree: the tree block's chunk reports it
          x = pp;
          ++depth;
        }
        cut = window_cut(p, seq_len, depth);
      }
      bool ok = true;
      // blocks of this tile: all of them, or every other one (from block t) when alternating
      const int n_mine = alt ? (nbt - t + 1) / 2 : nbt;
      for (int i = 0; i < n_mine; ++i) {
        const int j = alt ? 2 * i + t : i;  // the block
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->s_full[t], i & 1, abort, wait_ns));
        if (!ok) break;
        tc_fence_after_sync();
        int shift = j == nb - 1 ? tail_shift : 0;          // masked leading columns (this row)
        if (win_rows && j < nb) {
          const int kb = c.key_begin + j * kBlockN - shift;  // attended key of column 0
          shift = max(shift, min(cut - kb, kBlockN));
        }
        const int lim = j == nb - 1 ? tail_end : kBlockN;  // columns from here on are masked
        const bool tree_blk = j == nb;                      // keys = the sequence's tree nodes
        if (tree_blk && mask_tree_scores(bars->parent, tS, has_row ? node : -1)) bars->tree_err = 1u;
        // All 128 scores for the row maximum, kept in registers for both halves of P (P
        // goes to columns 0..63, whose scores are in registers by then; d = 64 reads keys
        // 64..127 again below).
        float lo[kHalf];
        float hi[kHalf];
        float mx;
        {
          uint32_t r[4][32];
#pragma unroll
          for (int q = 0; q < 4; ++q) tmem_ld32(tS + 32 * q, r[q]);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < kHalf; ++e) {
            lo[e] = __uint_as_float(r[e >> 5][e & 31]);
            hi[e] = __uint_as_float(r[2 + (e >> 5)][e & 31]);
          }
          if (shift > 0 || lim < kBlockN) {  // the sequence's last prefix block
#pragma unroll
            for (int e = 0; e < kHalf; ++e) {
              if (e < shift || e >= lim) lo[e] = -INFINITY;
              if (e + kHalf < shift || e + kHalf >= lim) hi[e] = -INFINITY;
            }
          }
          float m0 = fmaxf(lo[0], hi[0]), m1 = fmaxf(lo[1], hi[1]);
          float m2 = fmaxf(lo[2], hi[2]), m3 = fmaxf(lo[3], hi[3]);
#pragma unroll
          for (int e = 4; e < kHalf; e += 4) {
            m0 = fmax3(m0, lo[e], hi[e]);
            m1 = fmax3(m1, lo[e + 1], hi[e + 1]);
            m2 = fmax3(m2, lo[e + 2], hi[e + 2]);
            m3 = fmax3(m3, lo[e + 3], hi[e + 3]);
          }
          mx = fmax3(m0, m1, fmaxf(m2, m3)) * cs;
        }
        const bool raise = mx > m + kRescaleThreshold;
        const bool any_raise = __any_sync(0xffffffffu, raise);
        const float m_new = raise ? mx : m;
        // a row that has seen no visible key yet (a padding row of a tree-only chunk)
        // keeps m = -inf; its P is 0 against any finite reference
        const float m_ref = m_new == -INFINITY ? 0.f : m_new;
        float sum0 = 0.f, sum1 = 0.f, rsum0 = 0.f, rsum1 = 0.f;
        {
          uint32_t pk[kHalf / 2];
          make_p<EMU>(lo, cs, m_ref, pk, sum0, sum1, rsum0, rsum1);
          if (any_raise) {
            // the maximum moved up: rescale what O_t and l hold. O_t is idle: every PV of
            // this tile issued before S_t(j) has completed (s_full), and PV_t(j) waits for
            // this warpgroup's P. f = 1 where m is unchanged, 0 before the first block.
            const float f = m == m_new ? 1.f : ex2_approx(m - m_new);
            if (i > 0) {
#pragma unroll
              for (int q = 0; q < D / 16; ++q) {
                uint32_t o[16];
                tmem_ld16(tO + 16 * q, o);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                tmem_st16(tO + 16 * q, o);
              }
            }
            l *= f;
            lr *= f;
            m = m_new;
          }
          tmem_st32(tS, pk);  // P over keys 0..63 -> columns 0..31
          tmem_wait_st();
          tc_fence_before_sync();
          mbar_arrive(&bars->p_full[t][0]);
        }
        if constexpr (D != 128) {
          // d = 64 would spill with both halves live: its keys 64..127 are read again (P
          // took columns 0..31 only, so their scores are intact)
          uint32_t r[2][32];
          tmem_ld32(tS + 64, r[0]);
          tmem_ld32(tS + 96, r[1]);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < kHalf; ++e) hi[e] = __uint_as_float(r[e >> 5][e & 31]);
          if (shift > kHalf || lim < kBlockN) {
#pragma unroll
            for (int e = 0; e < kHalf; ++e)
              if (e + kHalf < shift || e + kHalf >= lim) hi[e] = -INFINITY;
          }
        }
        {
          uint32_t pk[kHalf / 2];
          make_p<EMU>(hi, cs, m_ref, pk, sum0, sum1, rsum0, rsum1);
          tmem_st32(tS + 32, pk);  // keys 64..127 -> columns 32..63
          tmem_wait_st();
          tc_fence_before_sync();
          mbar_arrive(&bars->p_full[t][1]);
        }
        l += sum0 + sum1;
        lr += rsum0 + rsum1;
      }
      // -------------------------------------------------------------- epilogue
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->o_full[t], 0, abort, wait_ns));
      // Each warpgroup stages its normalised 128 x D tile in shared memory as D/32 panels
      // of 128 rows x 128 B, swizzled like the tensor map (16-byte chunk q of row r at
      // q ^ (r & 7): conflict-free for the per-row writes), and one thread stores the
      // panels to o_part with TMA. Tile 0 finishes while tile 1's last PV may still read
      // V from the slot ring, so it stages over the Q tiles (every QK has completed by
      // o_full[0]); tile 1, last of all, stages over the ring. Rows past the unit's last
      // row are stored too: they stay inside the chunk's 256-row slot, which no one reads.
      const bool ok_all = bar_and(2 + t, 128, ok);
      if (ok_all) {
        tc_fence_after_sync();
        constexpr int kOPanels = D / 32;  // 128-byte panels of an fp32 row
        uint8_t* stage = smem + (t == 0 ? C::kQOff : C::kSlotOff);
        const float inv = 1.f / lr;
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {  // panel q = columns [32 q, 32 q + 32)
          uint32_t r[32];
          tmem_ld32(tO + 32 * q, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e)
            *reinterpret_cast<float4*>(stage + q * (128 * 128) + row * 128 + ((e ^ (row & 7)) << 4)) =
                make_float4(__uint_as_float(r[4 * e]) * inv, __uint_as_float(r[4 * e + 1]) * inv,
                            __uint_as_float(r[4 * e + 2]) * inv, __uint_as_float(r[4 * e + 3]) * inv);
        }
        // this tile's partial: rows [128 t, 128 t + 128) of the chunk's slot
#if defined(LS_DEBUG)
        // the partial's rows stay inside the chunk's slot of o_part / lse_part
        if (!((int64_t)blockIdx.x < p.n_chunks && t * 128 + row < kUnitRows)) bars->dbg = kErrIndex;
#endif
        if (has_row) a.lse_part[(size_t)blockIdx.x * kUnitRows + t * 128 + row] = m + log2f(l);
        fence_proxy_async_smem();  // the staged tile is read by the TMA unit
        asm volatile("bar.sync %0, 128;" ::"r"(2 + t) : "memory");
        if ((warp & 3) == 0 && lane == 0 && (alt || t * 128 < rows_here)) {
#pragma unroll
          for (int q = 0; q < kOPanels; ++q)
            tma_store_2d(&P.tmap_o, stage + q * (128 * 128), 32 * q, (int)blockIdx.x * kUnitRows + t * 128);
          bulk_commit();
          bulk_wait_all();  // the shared memory must stay until the TMA has read it
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tbase, C::kTmemCols);
  }
  if (tid == 0)
    a.chunk_status[blockIdx.x] = (bars->abort ? kErrTimeout : 0u) | (bars->tree_err ? kErrBadTree : 0u) | bars->dbg;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// K or V cache viewed as [rows][H_kv][D] bf16; boxes of 128 rows x 64 elements of one head.
bool make_kv_map(CUtensorMap* map, const void* base, int D, int Hkv, int64_t rows, int box_rows = 128) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Q viewed as [B*T nodes][H_kv][g][D] bf16; a box is 64 elements x g heads x one kv
// head x tpu nodes, which lands as tpu*g consecutive 128-byte rows, node-major.
bool make_q_map(CUtensorMap* map, const void* base, int D, const Plan& p) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)p.g, (cuuint64_t)p.Hkv, (cuuint64_t)(p.N > 0 ? p.N : 1)};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)p.g * D * 2, (cuuint64_t)p.Hq * D * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)p.g, 1, (cuuint32_t)p.tpu};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// o_part viewed as [n_chunks * 256 rows][D] fp32; boxes of 128 rows x 32 floats (128 B),
// 128B-swizzled like the kernel's staging.
bool make_o_map(CUtensorMap* map, float* base, int D, int64_t rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)D * 4};
  cuuint32_t box[2] = {32, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int EMU, bool GENERAL>
cudaError_t launch_d(const PartialsArgs& a, int64_t kv_rows, cudaStream_t stream) {
  TcParams P;
  P.a = a;
  const int64_t tree_rows = a.p.N > 0 ? a.p.N : 1;
  // a paged cache is read in boxes of one page (at most 128 rows)
  const int box_rows = a.page_table != nullptr && a.page_size < kBlockN ? a.page_size : kBlockN;
  if (!make_q_map(&P.tmap_q, a.q, D, a.p) || !make_kv_map(&P.tmap_k, a.k_cache, D, a.p.Hkv, kv_rows, box_rows) ||
      !make_kv_map(&P.tmap_v, a.v_cache, D, a.p.Hkv, kv_rows, box_rows) ||
      !make_kv_map(&P.tmap_kt, a.k_tree, D, a.p.Hkv, tree_rows) ||
      !make_kv_map(&P.tmap_vt, a.v_tree, D, a.p.Hkv, tree_rows) ||
      !make_o_map(&P.tmap_o, a.o_part, D, (int64_t)a.p.n_chunks * kUnitRows))
    return cudaErrorInvalidValue;
  const int smem = kSmemWindow;
  // opt in to the large shared-memory carve-out once per device
  static bool configured[64] = {};  // per template instance
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(partials_tc_kernel<D, EMU, GENERAL>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  if (!a.after_prep) {
    partials_tc_kernel<D, EMU, GENERAL><<<a.p.n_chunks, kThreads, smem, stream>>>(P);
    return cudaGetLastError();
  }
  // a programmatic dependent of the tree kernel (see the producer's wait_prior)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.p.n_chunks);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, partials_tc_kernel<D, EMU, GENERAL>, P);
}

}  // namespace

cudaError_t launch_partials(const PartialsArgs& a, int64_t kv_rows, cudaStream_t stream) {
  if (a.p.n_chunks == 0) return cudaSuccess;
  // One pair of scores in four takes the FMA-pipe exponential: a quarter of the
  // softmax's exponentials move off the special-function unit (MUFU), which is as busy
  // as the tensor pipe at d = 128 and busier at d = 64. More than a quarter makes the
  // FMA pipe the slower one.
  const bool general = a.page_table != nullptr || a.p.window > 0;
  if (a.p.d == 64) return general ? launch_d<64, 1, true>(a, kv_rows, stream) : launch_d<64, 1, false>(a, kv_rows, stream);
  return general ? launch_d<128, 1, true>(a, kv_rows, stream) : launch_d<128, 1, false>(a, kv_rows, stream);
}

}  // namespace ls

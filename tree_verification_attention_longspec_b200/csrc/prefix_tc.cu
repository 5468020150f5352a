// Prefix partial attention on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// LongSpec, gist.science summary, section 2C: the cached prefix is attended with no
// mask, and it carries most of the work, so it runs on the fastest path. With grouped-
// query attention the T*g (tree node, head-in-group) rows of one kv head share every
// key, so the prefix step is a dense contraction: S = Q K^T and O += P V. One CTA handles
// one chunk: a 128-row tile of one (sequence, kv head) against a range of 128-key
// blocks, and leaves its partial (out normalised by its own sum, lse in the log2
// domain) for the combine kernel.
//
// Pipeline. The scores of key block j go to one of two 128-column TMEM buffers (j % 2),
// so the tensor core computes S(j+1) = Q K(j+1)^T while the softmax works on S(j).
// The two softmax warpgroups split every block's columns: warpgroup x owns keys
// [64x, 64x+64) of each block and keeps its own running max m_x, sum l_x and output
// accumulator O_x += P_x V_x in TMEM, so the halves never wait for each other; they are
// merged by log-sum-exp once, at the end. P_x (bf16) is written over the scores it came
// from and read by the PV product straight from TMEM.
//
// Warp roles (320 threads, one CTA per SM):
//   warps 0-3  softmax of key half 0, warps 4-7 of key half 1: one thread per query
//              row (= TMEM lane). P is computed against the current m_x in one pass;
//              only when a block's maximum exceeds m_x by more than 2^8 is m_x raised,
//              O_x rescaled in TMEM and P recomputed.
//   warp 8     TMA producer: streams 128-key K and V blocks into a ring of slots.
//   warp 9     MMA issuer (one thread): S = Q K^T (shared-memory operands, N = 128) and
//              O_x += P_x V_x (P from TMEM, K = 64, N = d), tcgen05.commit to mbarriers.
//              It waits once per block and then issues the block's 16 MMAs back to back:
//              MMA issue is throttled to the tensor pipe's pace, so every pause of this
//              thread is idle tensor time.
// TMEM columns (512 allocated): score buffer u at 128u, O_x at 256 + d*x.
// Every wait is bounded: on a timeout the CTA raises an abort flag, all roles drain
// their in-flight copies and MMAs, TMEM is freed, and the chunk status reports it.
#include <cudaTypedefs.h>

#include <cstdlib>

#include "ls_device.cuh"
#include "sm100.cuh"

namespace ls {
namespace {
using namespace sm100;

constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kMaxSlots = 12;
constexpr int kHalf = 64;  // keys of a block owned by one softmax warpgroup
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kPanelBytes = 128 * 128;             // 128 rows x 64 bf16, 128B-swizzled
  static constexpr int kTileBytes = kPanels * kPanelBytes;  // 128 rows x D bf16
  static constexpr int kSlots = D == 128 ? 6 : 12;
  static constexpr int kQOff = 0;
  static constexpr int kSlotOff = kTileBytes;
  static constexpr int kBarOff = kSlotOff + kSlots * kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 1024 + 1024;  // barriers + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColO = 256;
  static_assert(kSlots <= kMaxSlots, "slots");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

struct alignas(64) TcParams {
  CUtensorMap tmap_k;
  CUtensorMap tmap_v;
  PrefixArgs a;
};

struct Bars {
  uint64_t full[kMaxSlots];
  uint64_t empty[kMaxSlots];
  uint64_t s_full[2];     // [buffer]: S(j) of buffer j%2 is in TMEM
  uint64_t p_full[2][2];  // [half][buffer]: P_x(j) is in TMEM
  uint64_t pv_last;       // O += P(nb-2) V(nb-2) finished (lets the last block rescale O)
  uint64_t o_full;
  uint32_t tmem_base;
  uint32_t abort;
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

// Waits only on time (used to drain in-flight work after an abort).
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  uint32_t never = 0;
  return mbar_wait_bounded(bar, parity, &never, kTimeoutNs);
}

// P = 2^(s*cs - m) for the 64 scores this thread holds, packed to bf16 pairs; adds the
// values to (sum0, sum1). EMU of every 4 pairs use the FMA-pipe exponential.
template <int EMU>
__device__ __forceinline__ void make_p(const float (&s)[kHalf], float cs, float m, uint32_t (&pk)[kHalf / 2],
                                       float& sum0, float& sum1) {
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
  }
}

template <int D, int EMU>
__global__ void __launch_bounds__(kThreads, 1) prefix_tc_kernel(const __grid_constant__ TcParams P) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kBarOff);
  const PrefixArgs& a = P.a;
  const Plan& p = a.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const ChunkCoord c = locate_chunk(p, a.cu, blockIdx.x);
  if (!c.valid) return;  // more CTAs than the device lengths need: the combine reports it
  const int n_keys = c.key_end - c.key_begin;
  const int nb = (n_keys + kBlockN - 1) / kBlockN;
  const int tail_shift = nb * kBlockN - n_keys;  // masked leading columns of the last block
  const int row0 = c.rgi * kUnitRows;
  const int rows_here = min(kUnitRows, p.rows - row0);

  if (nb == 0) {  // empty key range: an empty partial
    if (tid < rows_here) a.lse_part[(size_t)blockIdx.x * kUnitRows + tid] = -INFINITY;
    if (tid == 0) a.chunk_status[blockIdx.x] = 0u;
    return;
  }

  if (tid == 0) {
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(&bars->s_full[u], 1);
      mbar_init(&bars->p_full[0][u], 128);
      mbar_init(&bars->p_full[1][u], 128);
    }
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->pv_last, 1);
    bars->abort = 0u;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_map(&P.tmap_k);
    tma_prefetch_map(&P.tmap_v);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tbase = bars->tmem_base;
  volatile uint32_t* abort = &bars->abort;
  // the tree/combine kernel may start its own prologue now; it waits for this grid's
  // results before it reads them
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < nb; ++j) {
        int key0 = c.key_begin + j * kBlockN;
        if (j == nb - 1) key0 -= tail_shift;  // the box ends at the sequence end
        const int grow = c.seq_offset + key0;
        bool ok = true;
        for (int kv = 0; kv < 2; ++kv) {
          const int seq = 2 * j + kv, slot = seq % C::kSlots, use = seq / C::kSlots;
          if (!mbar_wait_bounded(&bars->empty[slot], (use & 1) ^ 1, abort, kTimeoutNs)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->full[slot], C::kTileBytes);
          uint8_t* dst = smem + C::kSlotOff + slot * C::kTileBytes;
          const CUtensorMap* map = kv ? &P.tmap_v : &P.tmap_k;
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_3d(dst + pn * C::kPanelBytes, map, &bars->full[slot], pn * 64, c.kh, grow);
          ++issued;
        }
        if (!ok) break;
      }
      // make sure no copy is still writing shared memory when the CTA ends
      const int first = issued > C::kSlots ? issued - C::kSlots : 0;
      for (int seq = first; seq < issued; ++seq)
        drain_wait(&bars->full[seq % C::kSlots], (seq / C::kSlots) & 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ load Q (warps 0-7)
    if (warp < 8) {
      const int chunks_per_row = D / 8;  // 16-byte chunks
      const int total = 128 * chunks_per_row;
      for (int idx = tid; idx < total; idx += 256) {
        const int r = idx / chunks_per_row, ch = idx % chunks_per_row;
        const int rg = row0 + r;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (rg < p.rows) {
          const int i = rg / p.g, jh = rg % p.g;
          const uint16_t* src = a.q + ((size_t)(c.b * p.T + i) * p.Hq + c.kh * p.g + jh) * D + ch * 8;
          v = *reinterpret_cast<const uint4*>(src);
        }
        const int pn = ch >> 3, cc = ch & 7;
        uint8_t* dst = smem + C::kQOff + pn * C::kPanelBytes + r * 128 + ((cc ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = v;
      }
      fence_proxy_async_smem();
    }
    // Q is in shared memory: warps 0-7 and the MMA warp meet at named barrier 1
    if (warp < 8 || warp == kMmaWarp) asm volatile("bar.sync 1, 288;" ::: "memory");

    if (warp == kMmaWarp) {
      if (lane == 0) {
        // -------------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc_qk = umma_idesc_bf16(128, kBlockN, false);
        constexpr uint32_t idesc_pv = umma_idesc_bf16(128, D, true);
        // A descriptor differs from another of the same kind only in its start-address
        // field (address >> 4 in the low 14 bits; shared addresses stay below 256 KB, so
        // adding an offset never carries out of it): build the bases once, add offsets.
        const uint64_t dq = umma_sdesc_sw128(smem_u32(smem + C::kQOff), 16, 1024);
        const uint64_t dk0 = umma_sdesc_sw128(smem_u32(smem + C::kSlotOff), 16, 1024);
        const uint64_t dv0 = umma_sdesc_sw128(smem_u32(smem + C::kSlotOff), C::kPanelBytes, 1024);
        constexpr uint32_t kTile16 = C::kTileBytes >> 4, kPanel16 = C::kPanelBytes >> 4;
        // K block j is sequence 2j of the slot ring, V block j is sequence 2j+1
        auto wait_full = [&](int seq) {
          return mbar_wait_bounded(&bars->full[seq % C::kSlots], (seq / C::kSlots) & 1, abort, kTimeoutNs);
        };
        // S(j) = Q K(j)^T into score buffer j%2; K(j) sits in ring slot `slot`
        auto issue_qk = [&](int j, int slot) {
          const uint64_t dk = dk0 + (uint64_t)(slot * kTile16);
          const uint32_t tS = tbase + C::kColS + (j & 1) * kBlockN;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kPanel16 + (kk & 3) * 2;  // 16-byte units
            umma_ss(tS, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars->s_full[j & 1]);
        };
        // O_x += P_x(j) V_x(j): K = 64 keys of half x, P from TMEM, V rows of that half;
        // V(j) sits in ring slot `slot`
        auto issue_pv = [&](int x, int j, int slot) {
          const uint64_t dv = dv0 + (uint64_t)(slot * kTile16 + x * (kHalf * 128 / 16));
          const uint32_t tP = tbase + C::kColS + (j & 1) * kBlockN + x * kHalf;
          const uint32_t tO = tbase + C::kColO + x * D;
#pragma unroll
          for (int kk = 0; kk < kHalf / 16; ++kk)
            umma_ts(tO, tP + kk * 8, dv + kk * (2048 / 16), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        };
        bool ok = wait_full(0);
        if (ok) {
          tc_fence_after_sync();
          issue_qk(0, 0);
          umma_commit(&bars->empty[0]);
          if (nb > 1) {
            ok = wait_full(2);
            if (ok) {
              tc_fence_after_sync();
              issue_qk(1, 2 % C::kSlots);
              umma_commit(&bars->empty[2 % C::kSlots]);
            }
          }
        }
        // One wait point per block, then all of the block's MMAs back to back:
        // O_x += P_x(j) V_x(j) for both halves, then S(j+2) into buffer j%2 (whose P(j)
        // has just been consumed). Three commits per block: V(j)'s slot, S(j+2) and
        // K(j+2)'s slot. Slot indices and phases advance incrementally (V(j) is sequence
        // 2j+1, K(j+2) is sequence 2j+4 of the ring).
        int sv = 1 % C::kSlots, uv = 1 / C::kSlots;  // V(j): slot and use count parity
        int sk = 4 % C::kSlots, uk = 4 / C::kSlots;  // K(j+2)
        for (int j = 0; j < nb && ok; ++j) {
          const bool more = j + 2 < nb;
          uint64_t* bk = more ? &bars->full[sk] : &bars->full[sv];  // no K(j+2): test V twice
          const uint32_t pk = more ? (uk & 1) : (uv & 1);
          const uint32_t pp = (j >> 1) & 1;
          if (!mbar_try_wait4(&bars->full[sv], uv & 1, bk, pk, &bars->p_full[0][j & 1], pp,
                              &bars->p_full[1][j & 1], pp)) {
            ok = mbar_wait_bounded(&bars->full[sv], uv & 1, abort, kTimeoutNs) &&
                 mbar_wait_bounded(bk, pk, abort, kTimeoutNs) &&
                 mbar_wait_bounded(&bars->p_full[0][j & 1], pp, abort, kTimeoutNs) &&
                 mbar_wait_bounded(&bars->p_full[1][j & 1], pp, abort, kTimeoutNs);
            if (!ok) break;
          }
          tc_fence_after_sync();
          issue_pv(0, j, sv);
          issue_pv(1, j, sv);
          umma_commit(&bars->empty[sv]);
          if (j == nb - 2) umma_commit(&bars->pv_last);
          if (more) {
            issue_qk(j + 2, sk);
            umma_commit(&bars->empty[sk]);
          }
          sv += 2;
          if (sv >= C::kSlots) { sv -= C::kSlots; uv ^= 1; }
          sk += 2;
          if (sk >= C::kSlots) { sk -= C::kSlots; uk ^= 1; }
        }
        umma_commit(&bars->o_full);
        drain_wait(&bars->o_full, 0);
      }
      __syncwarp();
    } else {
      // ---------------------------------------------------------------- softmax / epilogue
      const int x = warp >> 2;  // key half
      const int row = (warp & 3) * 32 + lane;
      const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
      const uint32_t tS0 = tbase + lane_base + C::kColS + x * kHalf;
      const uint32_t tOx = tbase + lane_base + C::kColO + x * D;
      const float cs = p.scale_log2;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nb; ++j) {
        const int u = j & 1;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->s_full[u], (j >> 1) & 1, abort, kTimeoutNs));
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t tS = tS0 + u * kBlockN;
        float s[kHalf];
        {
          uint32_t r0[32], r1[32];
          tmem_ld32(tS, r0);
          tmem_ld32(tS + 32, r1);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            s[e] = __uint_as_float(r0[e]);
            s[32 + e] = __uint_as_float(r1[e]);
          }
        }
        // the sequence's last block: columns before tail_shift belong to earlier keys
        const int shift = j == nb - 1 ? tail_shift - x * kHalf : 0;
        if (shift > 0) {
#pragma unroll
          for (int e = 0; e < kHalf; ++e)
            if (e < shift) s[e] = -INFINITY;
        }
        float mx;
        {
          float m0 = s[0], m1 = s[1], m2 = s[2], m3 = s[3];
#pragma unroll
          for (int e = 4; e < kHalf; e += 8) {
            m0 = fmax3(m0, s[e], s[e + 1]);
            m1 = fmax3(m1, s[e + 2], s[e + 3]);
            m2 = fmax3(m2, s[e + 4], s[e + 5]);
            m3 = fmax3(m3, s[e + 6], s[e + 7]);
          }
          mx = fmax3(m0, m1, fmaxf(m2, m3)) * cs;  // -inf if the whole half is masked
        }
        uint32_t pk[kHalf / 2];
        float sum0 = 0.f, sum1 = 0.f;
        const bool raise = mx > m + kRescaleThreshold;
        if (__any_sync(0xffffffffu, raise)) {
          // the maximum moved up: rescale what O_x and l hold (once the previous PV has
          // landed) and compute P against the new maximum
          const float m_new = raise ? mx : m;
          if (j > 0) {
            // O_x must hold all of PV(j-1) before it is rescaled. QK(j+1) was issued after
            // PV(j-1), so S(j+1) being ready implies it; the last block has no S(j+1) and
            // waits for the commit issued after PV(nb-2) instead.
            ok = __all_sync(0xffffffffu, j + 1 < nb ? mbar_wait_bounded(&bars->s_full[(j + 1) & 1], ((j + 1) >> 1) & 1,
                                                                        abort, kTimeoutNs)
                                                    : mbar_wait_bounded(&bars->pv_last, 0, abort, kTimeoutNs));
            if (!ok) break;
            tc_fence_after_sync();
            // f = 1 where m is unchanged; 0 where nothing was accumulated yet (m = -inf)
            const float f = m == m_new ? 1.f : ex2_approx(m - m_new);
#pragma unroll
            for (int q4 = 0; q4 < D / 32; ++q4) {
              uint32_t r[32];
              tmem_ld32(tOx + q4 * 32, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
              tmem_st32(tOx + q4 * 32, r);
            }
            l *= f;
          }
          m = m_new;
        }
        // masked columns (-inf) and the rare blocks above take the MUFU-only path; while
        // nothing has been seen yet (m = -inf, everything so far masked) every P is 0
        if (EMU == 0 || shift > 0 || m == -INFINITY || __any_sync(0xffffffffu, raise)) {
          make_p<0>(s, cs, m == -INFINITY ? 0.f : m, pk, sum0, sum1);
        } else {
          make_p<EMU>(s, cs, m, pk, sum0, sum1);
        }
        l += sum0 + sum1;
        tmem_st32(tS, pk);
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(&bars->p_full[x][u]);
      }
      // -------------------------------------------------------------- epilogue
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->o_full, 0, abort, kTimeoutNs));
      // every MMA has finished (o_full), so the Q tile's shared memory is free: it carries
      // both halves' (m, l) of every row to the other warpgroup
      float* xm = reinterpret_cast<float*>(smem + C::kQOff);  // [2][128]
      float* xl = xm + 256;                                   // [2][128]
      xm[x * 128 + row] = ok ? m : -INFINITY;
      xl[x * 128 + row] = ok ? l : 0.f;
      asm volatile("bar.sync 2, 256;" ::: "memory");
      if (ok) {
        tc_fence_after_sync();
        const float ma = xm[row], mb = xm[128 + row];
        const float M = fmaxf(ma, mb);
        const float wa = ma == -INFINITY ? 0.f : ex2_approx(ma - M);
        const float wb = mb == -INFINITY ? 0.f : ex2_approx(mb - M);
        const float Ls = wa * xl[row] + wb * xl[128 + row];
        const float inv = 1.f / Ls;
        const float ca = wa * inv, cb = wb * inv;
        const bool valid = row < rows_here;
        // this warpgroup writes output columns [x*D/2, (x+1)*D/2) of its rows
        float* dst = a.o_part + ((size_t)blockIdx.x * kUnitRows + row) * D + x * (D / 2);
        const uint32_t tOa = tbase + lane_base + C::kColO + x * (D / 2);
        const uint32_t tOb = tOa + D;
#pragma unroll
        for (int q4 = 0; q4 < D / 64; ++q4) {
          uint32_t ra[32], rb[32];
          tmem_ld32(tOa + q4 * 32, ra);
          tmem_ld32(tOb + q4 * 32, rb);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              float4 v;
              v.x = fmaf(ca, __uint_as_float(ra[e]), cb * __uint_as_float(rb[e]));
              v.y = fmaf(ca, __uint_as_float(ra[e + 1]), cb * __uint_as_float(rb[e + 1]));
              v.z = fmaf(ca, __uint_as_float(ra[e + 2]), cb * __uint_as_float(rb[e + 2]));
              v.w = fmaf(ca, __uint_as_float(ra[e + 3]), cb * __uint_as_float(rb[e + 3]));
              *reinterpret_cast<float4*>(dst + q4 * 32 + e) = v;
            }
          }
        }
        if (valid && x == 0) a.lse_part[(size_t)blockIdx.x * kUnitRows + row] = M + log2f(Ls);
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tbase, C::kTmemCols);
  }
  if (tid == 0) a.chunk_status[blockIdx.x] = bars->abort ? kErrTimeout : 0u;
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
bool make_kv_map(CUtensorMap* map, const void* base, int D, int Hkv, int64_t rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int EMU>
cudaError_t launch_d(const PrefixArgs& a, int64_t kv_rows, cudaStream_t stream) {
  TcParams P;
  P.a = a;
  if (!make_kv_map(&P.tmap_k, a.k_cache, D, a.p.Hkv, kv_rows) ||
      !make_kv_map(&P.tmap_v, a.v_cache, D, a.p.Hkv, kv_rows))
    return cudaErrorInvalidValue;
  const int smem = Cfg<D>::kSmemBytes;
  // opt in to the large shared-memory carve-out once per device
  static bool configured[64] = {};  // per template instance
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(prefix_tc_kernel<D, EMU>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  prefix_tc_kernel<D, EMU><<<a.p.n_chunks, kThreads, smem, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefix_tc(const PrefixArgs& a, int64_t kv_rows, cudaStream_t stream) {
  if (a.p.n_chunks == 0) return cudaSuccess;
  const char* env = getenv("LS_EMU");
  const int emu = env ? atoi(env) : 0;
  if (a.p.d == 64) return launch_d<64, 0>(a, kv_rows, stream);
  switch (emu) {
    case 1: return launch_d<128, 1>(a, kv_rows, stream);
    case 2: return launch_d<128, 2>(a, kv_rows, stream);
    default: return launch_d<128, 0>(a, kv_rows, stream);
  }
}

}  // namespace ls

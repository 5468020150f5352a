// Prefix partial attention on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// LongSpec, gist.science summary, section 2C: the cached prefix is attended with no
// mask, and it carries most of the work, so it runs on the fastest path. With grouped-
// query attention the T*g (tree node, head-in-group) rows of one kv head share every
// key, so the prefix step is a dense contraction: S = Q K^T and O += P V per 128-key
// block. One CTA handles one chunk: 256 query rows (two 128-row tiles) of one
// (sequence, kv head) against a range of 128-key blocks, and leaves its partial
// (out normalised by its own sum, lse in the log2 domain) for the combine kernel.
//
// Warp roles (320 threads, one CTA per SM):
//   warps 0-3  softmax for tile 0, warps 4-7 softmax for tile 1: one thread per query
//              row (= TMEM lane). Reads S from TMEM, keeps the running max m and sum l,
//              writes P (bf16) back over S in TMEM, rescales O in TMEM when m moves up
//              by more than 2^8, and writes the normalised partial at the end.
//   warp 8     TMA producer: streams K and V blocks into a ring of shared-memory slots.
//   warp 9     MMA issuer (one thread): S_t = Q_t K^T (both operands in shared memory)
//              and O_t += P_t V (P from TMEM, V in shared memory), tcgen05.commit to
//              mbarriers.
// A softmax thread never holds a whole score row: it reads S from TMEM twice, once in
// 32-column chunks for the row maximum and once to turn each chunk into P, which keeps
// it far below the 168 registers a thread has at 320 threads per SM.
// TMEM columns: S/P of tile t at 128*t, O of tile t at 256 + D*t (512 allocated).
// Every wait is bounded: on a timeout the CTA raises an abort flag, all roles drain
// their in-flight copies and MMAs, TMEM is freed, and the chunk status reports it.
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
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kPanelBytes = 128 * 128;             // 128 rows x 64 bf16, 128B-swizzled
  static constexpr int kTileBytes = kPanels * kPanelBytes;  // 128 rows x D bf16
  static constexpr int kSlots = D == 128 ? 5 : 12;
  static constexpr int kQOff = 0;
  static constexpr int kSlotOff = 2 * kTileBytes;
  static constexpr int kBarOff = kSlotOff + kSlots * kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 512 + 1024;   // barriers + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColO = 256;
  static_assert(kSlots <= kMaxSlots, "slots");
};

struct alignas(64) TcParams {
  CUtensorMap tmap_k;
  CUtensorMap tmap_v;
  PrefixArgs a;
};

struct Bars {
  uint64_t full[kMaxSlots];
  uint64_t empty[kMaxSlots];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full;
  uint32_t tmem_base;
  uint32_t abort;
};

// Waits only on time (used to drain in-flight work after an abort).
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  uint32_t never = 0;
  return mbar_wait_bounded(bar, parity, &never, kTimeoutNs);
}

template <int D>
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
  const int nt = rows_here > 128 ? 2 : 1;

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
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 128);
    }
    mbar_init(&bars->o_full, 1);
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
      const int total = nt * 128 * chunks_per_row;
      for (int idx = tid; idx < total; idx += 256) {
        const int r = idx / chunks_per_row, ch = idx % chunks_per_row;
        const int rg = row0 + r;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (rg < p.rows) {
          const int i = rg / p.g, jh = rg % p.g;
          const uint16_t* src = a.q + ((size_t)(c.b * p.T + i) * p.Hq + c.kh * p.g + jh) * D + ch * 8;
          v = *reinterpret_cast<const uint4*>(src);
        }
        const int t = r >> 7, rr = r & 127, pn = ch >> 3, cc = ch & 7;
        uint8_t* dst = smem + C::kQOff + t * C::kTileBytes + pn * C::kPanelBytes + rr * 128 + ((cc ^ (rr & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = v;
      }
      fence_proxy_async_smem();
    }
    // Q is in shared memory: warps 0-7 and the MMA warp meet at named barrier 1
    if (warp < 8 || warp == kMmaWarp) asm volatile("bar.sync 1, 288;" ::: "memory");

    if (warp == kMmaWarp) {
      if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc_qk = umma_idesc_bf16(128, 128, false);
        constexpr uint32_t idesc_pv = umma_idesc_bf16(128, D, true);
        const uint32_t q_base = smem_u32(smem + C::kQOff);
        const uint32_t slot_base = smem_u32(smem + C::kSlotOff);
        bool ok = true;
        for (int j = 0; j <= nb && ok; ++j) {
          const int sk = (2 * j) % C::kSlots, uk = (2 * j) / C::kSlots;
          const int sv = (2 * j - 1 + 2 * C::kSlots) % C::kSlots, uv = (2 * j - 1) / C::kSlots;
          if (j < nb) {
            ok = mbar_wait_bounded(&bars->full[sk], uk & 1, abort, kTimeoutNs);
            if (!ok) break;
            tc_fence_after_sync();
          }
          for (int t = 0; t < nt; ++t) {
            if (j > 0) {
              // O_t += P_t(j-1) V(j-1)
              if (t == 0) {
                ok = mbar_wait_bounded(&bars->full[sv], uv & 1, abort, kTimeoutNs);
                if (!ok) break;
              }
              ok = mbar_wait_bounded(&bars->p_full[t], (j - 1) & 1, abort, kTimeoutNs);
              if (!ok) break;
              tc_fence_after_sync();
              const uint32_t vaddr = slot_base + sv * C::kTileBytes;
              const uint32_t tP = tbase + C::kColS + t * 128;
              const uint32_t tO = tbase + C::kColO + t * D;
#pragma unroll
              for (int kk = 0; kk < kBlockN / 16; ++kk)
                umma_ts(tO, tP + kk * 8, umma_sdesc_sw128(vaddr + kk * 2048, C::kPanelBytes, 1024), idesc_pv,
                        (j > 1 || kk > 0) ? 1u : 0u);
            }
            if (j < nb) {
              // S_t = Q_t K(j)^T
              const uint32_t kaddr = slot_base + sk * C::kTileBytes;
              const uint32_t qaddr = q_base + t * C::kTileBytes;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
                umma_ss(tbase + C::kColS + t * 128, umma_sdesc_sw128(qaddr + off, 16, 1024),
                        umma_sdesc_sw128(kaddr + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
              }
              umma_commit(&bars->s_full[t]);
            }
          }
          if (!ok) break;
          if (j < nb) umma_commit(&bars->empty[sk]);
          if (j > 0) umma_commit(&bars->empty[sv]);
        }
        umma_commit(&bars->o_full);
        drain_wait(&bars->o_full, 0);
      }
      __syncwarp();
    } else {
      // ---------------------------------------------------------------- softmax / epilogue
      const int t = warp >> 2;
      if (t < nt) {
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tbase + lane_base + C::kColS + t * 128;
        const uint32_t tO = tbase + lane_base + C::kColO + t * D;
        const float cs = p.scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nb; ++j) {
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->s_full[t], j & 1, abort, kTimeoutNs));
          if (!ok) break;
          const int shift = j == nb - 1 ? tail_shift : 0;
          tc_fence_after_sync();
          // pass 1: row maximum of the raw scores (masked leading columns excluded)
          float mx = -INFINITY;
#pragma unroll
          for (int q4 = 0; q4 < kBlockN / 32; ++q4) {
            uint32_t r[32];
            tmem_ld32(tS + q4 * 32, r);
            tmem_wait_ld();
            float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const bool k0 = q4 * 32 + e >= shift, k1 = q4 * 32 + e + 1 >= shift;
              m0 = fmaxf(m0, k0 ? __uint_as_float(r[e]) : -INFINITY);
              m1 = fmaxf(m1, k1 ? __uint_as_float(r[e + 1]) : -INFINITY);
            }
            mx = fmaxf(mx, fmaxf(m0, m1));
          }
          const float m_new = fmaxf(m, mx * cs);
          const bool need = m_new > m + kRescaleThreshold;
          if (j > 0 && __any_sync(0xffffffffu, need)) {
            const float f = need ? ex2_approx(m - m_new) : 1.f;
#pragma unroll
            for (int q4 = 0; q4 < D / 32; ++q4) {
              uint32_t r[32];
              tmem_ld32(tO + q4 * 32, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
              tmem_st32(tO + q4 * 32, r);
            }
            l *= f;
          }
          if (need) m = m_new;
          const float nm = -m;
          // pass 2: P = 2^(s*scale*log2e - m) as bf16, written over the part of S already read
          float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
          for (int q4 = 0; q4 < kBlockN / 32; ++q4) {
            uint32_t r[32];
            tmem_ld32(tS + q4 * 32, r);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const bool k0 = q4 * 32 + 2 * e >= shift, k1 = q4 * 32 + 2 * e + 1 >= shift;
              const float p0 = k0 ? ex2_approx(fmaf(__uint_as_float(r[2 * e]), cs, nm)) : 0.f;
              const float p1 = k1 ? ex2_approx(fmaf(__uint_as_float(r[2 * e + 1]), cs, nm)) : 0.f;
              sum0 += p0;
              sum1 += p1;
              pk[e] = pack_bf16x2(p0, p1);
            }
            tmem_st16(tS + q4 * 16, pk);
          }
          l += sum0 + sum1;
          tmem_wait_st();
          tc_fence_before_sync();
          mbar_arrive(&bars->p_full[t]);
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->o_full, 0, abort, kTimeoutNs));
        if (ok) {
          tc_fence_after_sync();
          const int r_local = t * 128 + (warp & 3) * 32 + lane;
          const bool valid = r_local < rows_here;
          const float inv = 1.f / l;
          float* dst = a.o_part + ((size_t)blockIdx.x * kUnitRows + r_local) * D;
#pragma unroll
          for (int q4 = 0; q4 < D / 32; ++q4) {
            uint32_t r[32];
            tmem_ld32(tO + q4 * 32, r);
            tmem_wait_ld();
            if (valid) {
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4*>(dst + q4 * 32 + e) =
                    make_float4(__uint_as_float(r[e]) * inv, __uint_as_float(r[e + 1]) * inv,
                                __uint_as_float(r[e + 2]) * inv, __uint_as_float(r[e + 3]) * inv);
            }
          }
          if (valid) a.lse_part[(size_t)blockIdx.x * kUnitRows + r_local] = m + log2f(l);
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

template <int D>
cudaError_t launch_d(const PrefixArgs& a, int64_t kv_rows, cudaStream_t stream) {
  TcParams P;
  P.a = a;
  if (!make_kv_map(&P.tmap_k, a.k_cache, D, a.p.Hkv, kv_rows) ||
      !make_kv_map(&P.tmap_v, a.v_cache, D, a.p.Hkv, kv_rows))
    return cudaErrorInvalidValue;
  const int smem = Cfg<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(prefix_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  prefix_tc_kernel<D><<<a.p.n_chunks, kThreads, smem, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefix_tc(const PrefixArgs& a, int64_t kv_rows, cudaStream_t stream) {
  if (a.p.n_chunks == 0) return cudaSuccess;
  return a.p.d == 64 ? launch_d<64>(a, kv_rows, stream) : launch_d<128>(a, kv_rows, stream);
}

}  // namespace ls

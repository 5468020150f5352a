// Log-sum-exp combine of the attention partials.
//
// LongSpec, gist.science summary, section 2C ("Aggregation"): the partial results are
// joined by a log-sum-exp step into one exact softmax. Every chunk of the partials
// kernel left, for each row of its unit, its output normalised by its own sum (o_part)
// and its lse in the log2 domain (lse_part); the chunks of one unit cover its prefix
// blocks and its tree block once each. For a row with partials (o_x, l_x):
//   M = max_x l_x,  w_x = 2^(l_x - M),  out = sum_x w_x o_x / sum_x w_x,
//   lse = (M + log2 sum_x w_x) * ln 2   (natural log, scale included).
// One warp per output row (tree node i of sequence b, query head h); lanes split the
// head dimension. Rows are enumerated as if every sequence had T nodes; with
// per-sequence trees (cu_tree) the rows past a sequence's own tree have no output. The kernel is launched as a programmatic dependent of the partials
// kernel and waits for its results with griddepcontrol.wait: its CTAs are launched onto
// the SMs the partials grid leaves free (and onto each SM as a partials CTA leaves; the
// partials CTA's registers keep them apart while it runs), do their row bookkeeping and
// wait there.
#include "ls_device.cuh"

namespace ls {
namespace {

// The merge's exponentials, reciprocal and logarithm by the special-function unit's
// approximate instructions (relative error about 2^-22, far below the bf16 result's 2^-9):
// the accurate library versions lengthened each row's dependent chain measurably.
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_fast(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_fast(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr int kPrefetch = 20;  // partials in flight per warp (the headline has 18 per row)

template <int D, bool WIDE>
__global__ void __maxnreg__(112) combine_kernel(const __grid_constant__ CombineArgs a) {
  constexpr int E = D / 32;  // head-dim elements per lane
  const Plan& p = a.p;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ uint32_t err_s;
  if (threadIdx.x == 0) err_s = 0u;
  __syncthreads();

  // Everything that does not depend on the partials is done before the wait: the row's
  // sequence, its chunk range (from cu_seqlens, an input) and the length check.
  const int64_t n_rows = (int64_t)p.B * p.T * p.Hq;
  constexpr bool wide = WIDE;  // the CTA's warps share one row
  const int64_t row = wide ? (int64_t)blockIdx.x : (int64_t)blockIdx.x * kMergeRows + warp;
  const bool has_row = row < n_rows;
  int n = 0, cbase = 0, rl = 0;
  bool alt = false;  // the row's unit ran with alternating tiles: two partials per chunk
  int64_t out_row = 0;
  bool lengths_ok = false, writes = false;
  uint32_t err = 0u;
  if (has_row) {
    const int tok = (int)(row / p.Hq), h = (int)(row % p.Hq);
    const int b = tok / p.T, i = tok % p.T;
    const int kh = h / p.g, j = h % p.g;
    int tree_base = 0, tree_n = 0;
    if (!tree_range(p, a.cu_tree, b, &tree_base, &tree_n)) err |= kErrLengths;
    writes = i < tree_n;  // the node exists in sequence b's tree
    out_row = (int64_t)(tree_base + i) * p.Hq + h;
    int first = 0, total = 0;
    const int32_t* cu = plan_cu(p, a.cu);
    sequence_chunks(p, cu, b, &first, &n, &total);
    const int32_t L = a.cu[b + 1] - a.cu[b];
    // the device lengths must give the chunk grid the host planned (else some keys were
    // never attended): same chunk count, a uniform plan long enough for this L, and the
    // very lengths the kernels addressed keys with when they came with the plan
    lengths_ok = L >= 0 && total == p.n_chunks &&
                 (p.uniform_n < 0 || (int64_t)prefix_blocks(attended_len(p, L)) + p.with_tree <= (int64_t)p.uniform_n * p.C) &&
                 (p.cu_n == 0 || (a.cu[b] == cu[b] && a.cu[b + 1] == cu[b + 1]));
    int32_t u, r;
    unit_row(p, i, j, &u, &r);
    rl = r;
    alt = unit_alternates(min(p.tpu, tree_n - u * p.tpu) * p.g);
    cbase = first + (kh * p.rg + u) * n;
    // the row's chunks, its output row and (with RoPE) the tree kernel's word of its node
    LS_DCHECK(err, b < p.B && kh < p.Hkv && u < p.rg && r < kUnitRows);
    LS_DCHECK(err, !(writes && lengths_ok) || (cbase >= 0 && cbase + n <= p.n_chunks));
    LS_DCHECK(err, !writes || (tree_base + i < p.N && out_row < (int64_t)p.N * p.Hq));
#if defined(LS_DEBUG)
    if (writes && a.rope_status != nullptr) err |= a.rope_status[(size_t)b * p.T + i];
#endif
  }
  // the partials kernel may still be running: wait for its grid to finish
  asm volatile("griddepcontrol.wait;" ::: "memory");

  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float M = -INFINITY, Lsum = 0.f;  // running max of the lse and sum of weights 2^(l - M)
  if (writes) {
    if (lengths_ok) {
      // the row's partials: one per chunk, or two (rows rl and rl + 128 of the chunk's
      // slot) when the partials kernel's tiles alternated key blocks
      const int sh = alt ? 1 : 0;
      const int n_parts = n << sh;
      const size_t row0 = (size_t)cbase * kUnitRows + rl;
      auto part_row = [&](int k) -> size_t {  // row of partial k in o_part / lse_part
        return row0 + (uint32_t)((k >> sh) * kUnitRows + ((k & sh) << 7));
      };
      // a wide CTA's warp w takes the batches w, w + 4, ...
      const int first_batch = wide ? warp * kPrefetch : 0, stride = wide ? kMergeRows * kPrefetch : kPrefetch;
      for (int x0 = first_batch; x0 < n_parts; x0 += stride) {
        const int nx = min(kPrefetch, n_parts - x0);
        // every lane one partial's lse and status; up to kPrefetch outputs in flight
        float lx = -INFINITY;
        if (lane < nx) {
          LS_DCHECK(err, cbase + ((x0 + lane) >> sh) < p.n_chunks &&
                             part_row(x0 + lane) < (size_t)p.n_chunks * kUnitRows);
          lx = a.lse_part[part_row(x0 + lane)];
          err |= a.chunk_status[cbase + ((x0 + lane) >> sh)];
        }
        float ov[kPrefetch][E];
#pragma unroll
        for (int x = 0; x < kPrefetch; ++x) {
          if (x < nx) {
            const float* op = a.o_part + part_row(x0 + x) * D + lane * E;
            if constexpr (E == 4) {
              const float4 v = *reinterpret_cast<const float4*>(op);
              ov[x][0] = v.x;
              ov[x][1] = v.y;
              ov[x][2] = v.z;
              ov[x][3] = v.w;
            } else {
              const float2 v = *reinterpret_cast<const float2*>(op);
              ov[x][0] = v.x;
              ov[x][1] = v.y;
            }
          }
        }
        float mx = lx;
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
        const float Mn = fmaxf(M, mx);
        const float corr = M == Mn ? 1.f : ex2_fast(M - Mn);       // M = -inf before any weight: 0
        const float wl = lx == -INFINITY ? 0.f : ex2_fast(lx - Mn);  // this lane's chunk weight
        Lsum = Lsum * corr + warp_sum(wl);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] *= corr;
        M = Mn;
#pragma unroll
        for (int x = 0; x < kPrefetch; ++x) {
          const float w = __shfl_sync(0xffffffffu, wl, x);
          if (x < nx && w > 0.f) {  // an empty partial has weight 0 (its output slot is not read)
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = fmaf(w, ov[x][e], acc[e]);
          }
        }
      }
    } else {
      err |= kErrLengths;
    }
  }
  if constexpr (WIDE) {
    // the warps' merges of their batches, joined by warp 0 in the same way (only the wide
    // instance holds this scratch)
    __shared__ float w_m[kMergeRows], w_l[kMergeRows], w_acc[kMergeRows][D];
    if (lane == 0) {
      w_m[warp] = M;
      w_l[warp] = Lsum;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) w_acc[warp][lane * E + e] = acc[e];
    __syncthreads();
    if (warp == 0) {
      float Mt = -INFINITY;
      for (int w = 0; w < kMergeRows; ++w)
        if (w_l[w] > 0.f) Mt = fmaxf(Mt, w_m[w]);
      Lsum = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = 0.f;
      for (int w = 0; w < kMergeRows; ++w) {
        if (!(w_l[w] > 0.f)) continue;  // a warp without partials
        const float f = ex2_fast(w_m[w] - Mt);
        Lsum = fmaf(w_l[w], f, Lsum);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(w_acc[w][lane * E + e], f, acc[e]);
      }
      M = Mt;
    }
  }
  if (writes && (!wide || warp == 0)) {
    const float inv = Lsum > 0.f ? rcp_fast(Lsum) : 0.f;
    uint16_t* dst = a.out + out_row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const uint32_t lo = f32_to_bf16(acc[e] * inv), hi = f32_to_bf16(acc[e + 1] * inv);
      *reinterpret_cast<uint32_t*>(dst + e) = lo | (hi << 16);
    }
    if (lane == 0) a.lse[out_row] = Lsum > 0.f ? (M + lg2_fast(Lsum)) * kLn2 : -INFINITY;
  }
#pragma unroll
  for (int o2 = 16; o2 > 0; o2 >>= 1) err |= __shfl_xor_sync(0xffffffffu, err, o2);
  if (lane == 0 && err) atomicOr(&err_s, err);
  __syncthreads();
  if (threadIdx.x == 0) a.status[blockIdx.x] = err_s;
}

template <int D, bool WIDE>
cudaError_t launch_d(const CombineArgs& a, cudaStream_t stream) {
  // a programmatic dependent of the partials kernel: its CTAs may be scheduled while
  // that grid runs and wait in griddepcontrol.wait
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.p.n_combine);
  cfg.blockDim = dim3(32 * kMergeRows);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.after_partials ? 1 : 0;  // else an ordinary launch (it reads cu before its wait)
  return cudaLaunchKernelEx(&cfg, combine_kernel<D, WIDE>, a);
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
  if (a.p.n_combine == 0) return cudaSuccess;
  if (a.p.combine_wide) return a.p.d == 64 ? launch_d<64, true>(a, stream) : launch_d<128, true>(a, stream);
  return a.p.d == 64 ? launch_d<64, false>(a, stream) : launch_d<128, false>(a, stream);
}

}  // namespace ls

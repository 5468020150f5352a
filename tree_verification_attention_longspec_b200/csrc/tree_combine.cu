// Tree partial attention fused with the log-sum-exp combine.
//
// LongSpec, gist.science summary, section 2C: the speculative tree tokens are
// attended under the tree mask ("Speculative-Teil ... Baum-Maskierung"), and the
// partial results are joined by a log-sum-exp step into one exact softmax
// ("Aggregation").
//
// One CTA per (tree node i of sequence b, kv head kh); one warp per query head of
// the group, lanes split the head dimension. The work is arranged in few dependent
// rounds of global loads:
//   1. the tree's parent array (into shared memory), the prefix lengths and the query
//      row of the warp's first head;
//   2. thread 0 follows parent links in shared memory to list node i's visible set (i
//      and its ancestors), validating every link (node 0 is the root with parent -1,
//      every other node's parent lies in [0, c), so the walk ends after at most i+1
//      steps); then all threads stage the visible nodes' keys and values in shared
//      memory;
//   3. each warp runs the online softmax over the staged tree keys of its head, then
//      waits for the prefix kernel (this kernel is launched as its programmatic
//      dependent, so rounds 1-3 overlap the prefix kernel's tail), loads its row's prefix
//      partials (every lane one chunk's lse, up to 16 chunk outputs in flight), merges
//      everything by log-sum-exp and writes bf16 `out` and the natural-log `lse`.
#include "ls_device.cuh"

namespace ls {
namespace {

constexpr int kPrefetch = 16;  // prefix partials in flight per warp

template <int D>
__global__ void __launch_bounds__(256) tree_combine_kernel(CombineArgs a) {
  constexpr int E = D / 32;  // head-dim elements per lane
  extern __shared__ __align__(16) uint8_t dsmem[];
  __shared__ int par_s[kMaxTree];
  __shared__ int anc[kMaxTree];
  __shared__ int n_anc;
  __shared__ uint32_t err_s;
  const Plan& p = a.p;
  const int T = p.T;
  uint16_t* kt_s = reinterpret_cast<uint16_t*>(dsmem);  // [T][D] keys of the visible nodes
  uint16_t* vt_s = kt_s + (size_t)T * D;                 // [T][D] values
  const int tok = blockIdx.x;  // b*T + i
  const int kh = blockIdx.y;
  const int b = tok / T, i = tok % T;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;

  // ---- round 1
  for (int x = threadIdx.x; x < T; x += blockDim.x) par_s[x] = a.parent[(size_t)b * T + x];
  int chunk_first = 0, chunk_per_unit = 0, total = 0;
  sequence_chunks(p, a.cu, b, &chunk_first, &chunk_per_unit, &total);
  const int L = a.cu[b + 1] - a.cu[b];
  const bool use_prefix =
      !(L < 0 || total != p.n_chunks || (p.uniform_n >= 0 && (long long)L > (long long)p.uniform_n * p.C * kBlockN));
  float q_first[E];
  if (warp < p.g) {
    const size_t row = (size_t)tok * p.Hq + kh * p.g + warp;
#pragma unroll
    for (int e = 0; e < E; ++e) q_first[e] = bf16_to_f32(a.q[row * D + lane * E + e]);
  }
  if (threadIdx.x == 0) err_s = use_prefix ? 0u : kErrLengths;
  __syncthreads();

  // ---- round 2
  if (threadIdx.x == 0) {
    int node = i, n = 0;
    bool bad = false;
    while (true) {
      anc[n++] = node;
      const int pp = par_s[node];
      if (node == 0) {
        bad = pp != -1;
        break;
      }
      if (pp < 0 || pp >= node) {
        bad = true;
        break;
      }
      node = pp;
    }
    n_anc = n;
    if (bad) err_s |= kErrBadTree;
  }
  __syncthreads();
  const int na = n_anc;
  {
    constexpr int kPieces = D / 8;  // 16-byte pieces per row
    for (int idx = threadIdx.x; idx < 2 * na * kPieces; idx += blockDim.x) {
      const int kv = idx / (na * kPieces), rem = idx % (na * kPieces);
      const int x = rem / kPieces, pc = rem % kPieces;
      const uint16_t* src = (kv ? a.v_tree : a.k_tree) + ((size_t)(b * T + anc[x]) * p.Hkv + kh) * D + pc * 8;
      uint16_t* dst = (kv ? vt_s : kt_s) + (size_t)x * D + pc * 8;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    }
  }
  __syncthreads();

  // ---- round 3: tree part per head, then (once the prefix kernel has finished) its
  // prefix partials
  uint32_t err_w = 0;
  for (int j = warp; j < p.g; j += nwarps) {
    const size_t row = (size_t)tok * p.Hq + kh * p.g + j;
    int32_t rgi, rl;
    unit_row(p, i, j, &rgi, &rl);
    const int cbase = chunk_first + (kh * p.rg + rgi) * chunk_per_unit;
    const int n_chunks = use_prefix ? chunk_per_unit : 0;

    // issue the first batch of prefix-partial loads
    float lx = -INFINITY;
    float ov[kPrefetch][E];
    auto issue = [&](int x0) {
      const int nx = min(kPrefetch, n_chunks - x0);
      lx = -INFINITY;
      if (lane < nx) {
        lx = a.lse_part[(size_t)(cbase + x0 + lane) * kUnitRows + rl];
        err_w |= a.chunk_status[cbase + x0 + lane];
      }
      const float* base = a.o_part + ((size_t)(cbase + x0) * kUnitRows + rl) * D + lane * E;
#pragma unroll
      for (int x = 0; x < kPrefetch; ++x) {
        if (x < nx) {
          const float* op = base + (size_t)x * kUnitRows * D;
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
    };
    float qv[E], o[E];
    if (j == warp) {
#pragma unroll
      for (int e = 0; e < E; ++e) qv[e] = q_first[e];
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) qv[e] = bf16_to_f32(a.q[row * D + lane * E + e]);
    }
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] = 0.f;
    // tree part: online softmax over node i and its ancestors (log2 domain), four keys
    // at a time so that their warp reductions overlap
    float m = -INFINITY, l = 0.f;
    for (int x0 = 0; x0 < na; x0 += 4) {
      float d4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        d4[u] = 0.f;
        if (x0 + u < na) {
          const uint16_t* kr = kt_s + (size_t)(x0 + u) * D + lane * E;
#pragma unroll
          for (int e = 0; e < E; ++e) d4[u] = fmaf(qv[e], bf16_to_f32(kr[e]), d4[u]);
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
        for (int u = 0; u < 4; ++u) d4[u] += __shfl_xor_sync(0xffffffffu, d4[u], off);
      }
      float mn = m;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        d4[u] = x0 + u < na ? d4[u] * p.scale_log2 : -INFINITY;
        mn = fmaxf(mn, d4[u]);
      }
      const float corr = exp2f(m - mn);  // m = -inf on the first group: 0
      l *= corr;
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] *= corr;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (x0 + u < na) {
          const float w = exp2f(d4[u] - mn);
          l += w;
          const uint16_t* vr = vt_s + (size_t)(x0 + u) * D + lane * E;
#pragma unroll
          for (int e = 0; e < E; ++e) o[e] = fmaf(w, bf16_to_f32(vr[e]), o[e]);
        }
      }
      m = mn;
    }
    // The prefix kernel may still be running (programmatic dependent launch): wait for
    // it, then fold in its partials. The tree part above overlapped its tail.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    issue(0);
    // merge: the tree part is (lse M, normalised out acc); each chunk adds (lx, ov)
    float M = m + log2f(l);
    float acc[E];
    const float inv_l = 1.f / l;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = o[e] * inv_l;
    float Lsum = 1.f;  // sum of weights relative to 2^M
    for (int x0 = 0; x0 < n_chunks; x0 += kPrefetch) {
      if (x0 > 0) issue(x0);
      const int nx = min(kPrefetch, n_chunks - x0);
      float mx = lx;
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
      const float Mn = fmaxf(M, mx);
      const float corr = exp2f(M - Mn);
      const float wl = lx == -INFINITY ? 0.f : exp2f(lx - Mn);  // this lane's chunk weight
      Lsum = Lsum * corr + warp_sum(wl);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] *= corr;
      M = Mn;
#pragma unroll
      for (int x = 0; x < kPrefetch; ++x) {
        const float w = __shfl_sync(0xffffffffu, wl, x);
        if (x < nx && w > 0.f) {  // an empty chunk leaves its output slot unwritten
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] = fmaf(w, ov[x][e], acc[e]);
        }
      }
    }
    const float inv = 1.f / Lsum;
    uint16_t* dst = a.out + row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const uint32_t lo = f32_to_bf16(acc[e] * inv), hi = f32_to_bf16(acc[e + 1] * inv);
      *reinterpret_cast<uint32_t*>(dst + e) = lo | (hi << 16);
    }
    if (lane == 0) a.lse[row] = (M + log2f(Lsum)) * kLn2;
  }
  if (err_w) atomicOr(&err_s, err_w);
  __syncthreads();
  if (threadIdx.x == 0) a.status[(size_t)blockIdx.y * gridDim.x + blockIdx.x] = err_s;
}

template <int D>
cudaError_t launch_d(const CombineArgs& a, cudaStream_t stream) {
  const int warps = a.p.g < 8 ? a.p.g : 8;
  dim3 grid(a.p.B * a.p.T, a.p.Hkv);
  const size_t smem = (size_t)2 * a.p.T * D * sizeof(uint16_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(tree_combine_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  // launched as a programmatic dependent of the prefix kernel: its first two rounds
  // (the tree) overlap the prefix kernel's tail; it waits for the prefix partials with
  // griddepcontrol.wait
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(32 * warps);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tree_combine_kernel<D>, a);
}

}  // namespace

cudaError_t launch_tree_combine(const CombineArgs& a, cudaStream_t stream) {
  return a.p.d == 64 ? launch_d<64>(a, stream) : launch_d<128>(a, stream);
}

}  // namespace ls

// Tree partial attention fused with the log-sum-exp combine.
//
// LongSpec, gist.science summary, section 2C: the speculative tree tokens are
// attended under the tree mask ("Speculative-Teil ... Baum-Maskierung"), and the
// partial results are joined by a log-sum-exp step into one exact softmax
// ("Aggregation").
//
// One CTA per (tree node i of sequence b, kv head kh); one warp per query head of
// the group, lanes split the head dimension. Thread 0 builds node i's visible set
// (i and its ancestors) by following parent links, validating each link (node 0 is
// the root with parent -1, otherwise parent[c] lies in [0, c), so the walk ends after
// at most i+1 steps). Each warp then runs an online softmax over the visible tree
// keys and folds in every prefix chunk's (lse, out) partial of its row, and writes
// bf16 `out` and the natural-log `lse`.
#include "ls_device.cuh"

namespace ls {
namespace {

template <int D>
__global__ void __launch_bounds__(256) tree_combine_kernel(CombineArgs a) {
  constexpr int E = D / 32;  // head-dim elements per lane
  __shared__ int anc[kMaxTree];
  __shared__ int n_anc;
  __shared__ int chunk_first, chunk_per_unit;
  __shared__ uint32_t err_s;
  const Plan& p = a.p;
  const int tok = blockIdx.x;  // b*T + i
  const int kh = blockIdx.y;
  const int b = tok / p.T, i = tok % p.T;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;

  if (threadIdx.x == 0) {
    uint32_t err = 0;
    const int32_t* par = a.parent + (size_t)b * p.T;
    int node = i, n = 0;
    while (true) {
      anc[n++] = node;
      const int pp = par[node];
      if (node == 0) {
        if (pp != -1) err |= kErrBadTree;
        break;
      }
      if (pp < 0 || pp >= node) {
        err |= kErrBadTree;
        break;
      }
      node = pp;
    }
    n_anc = n;
    int first = 0, per_unit = 0, total = 0;
    sequence_chunks(p, a.cu, b, &first, &per_unit, &total);
    const int L = a.cu[b + 1] - a.cu[b];
    if (L < 0 || total != p.n_chunks) err |= kErrLengths;
    if (p.uniform_n >= 0 && (long long)L > (long long)p.uniform_n * p.C * kBlockN) err |= kErrLengths;
    chunk_first = first;
    chunk_per_unit = per_unit;
    err_s = err;
  }
  __syncthreads();
  const bool use_prefix = (err_s & kErrLengths) == 0;
  uint32_t err_w = 0;

  for (int j = warp; j < p.g; j += nwarps) {
    const size_t row = (size_t)tok * p.Hq + kh * p.g + j;
    float qv[E], o[E];
    {
      const uint16_t* qp = a.q + row * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        qv[e] = bf16_to_f32(qp[e]);
        o[e] = 0.f;
      }
    }
    float m = -INFINITY, l = 0.f;
    // tree part: node i and its ancestors
    for (int x = 0; x < n_anc; ++x) {
      const size_t kr = ((size_t)(b * p.T + anc[x]) * p.Hkv + kh) * D + lane * E;
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) dot = fmaf(qv[e], bf16_to_f32(a.k_tree[kr + e]), dot);
      const float s = warp_sum(dot) * p.scale_log2;
      const float mn = fmaxf(m, s);
      const float corr = exp2f(m - mn), w = exp2f(s - mn);
      l = l * corr + w;
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = fmaf(w, bf16_to_f32(a.v_tree[kr + e]), o[e] * corr);
      m = mn;
    }
    // prefix partials of this row's unit, each (normalised out, log2 lse)
    if (use_prefix) {
      const int r = i * p.g + j;
      const int rgi = r / kUnitRows, rl = r % kUnitRows;
      const int cbase = chunk_first + (kh * p.rg + rgi) * chunk_per_unit;
      for (int x = 0; x < chunk_per_unit; ++x) {
        const size_t slot = (size_t)(cbase + x) * kUnitRows + rl;
        if (lane == 0) err_w |= a.chunk_status[cbase + x];
        const float lx = a.lse_part[slot];
        if (lx == -INFINITY) continue;
        const float mn = fmaxf(m, lx);
        const float corr = exp2f(m - mn), w = exp2f(lx - mn);
        l = l * corr + w;
        const float* op = a.o_part + slot * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = fmaf(w, op[e], o[e] * corr);
        m = mn;
      }
    }
    const float inv = 1.f / l;
    uint16_t* dst = a.out + row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const uint32_t lo = f32_to_bf16(o[e] * inv), hi = f32_to_bf16(o[e + 1] * inv);
      *reinterpret_cast<uint32_t*>(dst + e) = lo | (hi << 16);
    }
    if (lane == 0) a.lse[row] = (m + log2f(l)) * kLn2;
  }
  if (err_w) atomicOr(&err_s, err_w);
  __syncthreads();
  if (threadIdx.x == 0) a.status[(size_t)blockIdx.y * gridDim.x + blockIdx.x] = err_s;
}

template <int D>
cudaError_t launch_d(const CombineArgs& a, cudaStream_t stream) {
  const int warps = a.p.g < 8 ? a.p.g : 8;
  dim3 grid(a.p.B * a.p.T, a.p.Hkv);
  tree_combine_kernel<D><<<grid, 32 * warps, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tree_combine(const CombineArgs& a, cudaStream_t stream) {
  return a.p.d == 64 ? launch_d<64>(a, stream) : launch_d<128>(a, stream);
}

}  // namespace ls

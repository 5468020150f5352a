// Tree positions and rotary embedding of the tree's queries and keys.
//
// A draft tree's nodes are new tokens: node i of sequence b follows the L_b cached
// tokens at depth(i) steps below the root, so its position is L_b + depth(i) (the root,
// depth 0, is the token right after the prefix; siblings share a position). The
// attention uses rotary position embedding (RoFormer, listed under "Builds on" on the
// mlsanity page; the evaluated Llama and Qwen models use it): q and k of a token at
// position m are rotated pair by pair, pair e = (x[e], x[e + d/2]) (the half-split
// pairing of those models' reference code, `rotate_half`) by the angle m * theta_e,
// theta_e = base^(-2e/d). The cached keys were rotated when they were written; this
// kernel rotates the tree's queries and keys, so that the attention kernels read them as
// if the caller had done it. Results are rounded to bf16 like the caller's tensors.
//
// One CTA per (sequence, node slot); nodes past a sequence's tree do nothing. The CTA
// first issues the loads of its node's q and k_tree rows (they do not depend on the
// position), then finds the depth: every thread takes one node of the sequence and the
// parent links are followed by pointer jumping in shared memory (after round r each
// node knows its ancestor 2^r levels up and its distance to it, so seven rounds cover
// 128 levels); a link that is not a rooted tree's stops the jumping there (the attention
// kernel reports that tree). The angle is reduced modulo 2 pi in double precision and
// its sine and cosine taken in float, so that large positions (10^5 and more) keep their
// precision.
#include "ls_device.cuh"

namespace ls {
namespace {

constexpr int kRopeThreads = 256;
constexpr int kPrefetch = 2;  // (head, 8-pair group) items per thread loaded up front

__device__ __forceinline__ void rotate8(const uint4& lo, const uint4& hi, const float* cos_s, const float* sin_s,
                                        int e0, uint4& olo, uint4& ohi) {
  const uint32_t lw[4] = {lo.x, lo.y, lo.z, lo.w}, hw[4] = {hi.x, hi.y, hi.z, hi.w};
  uint32_t ol[4], oh[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t rl = 0u, rh = 0u;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int e = e0 + 2 * w + k;
      const float x1 = bf16_to_f32((uint16_t)(lw[w] >> (16 * k)));
      const float x2 = bf16_to_f32((uint16_t)(hw[w] >> (16 * k)));
      const float c = cos_s[e], s = sin_s[e];
      const float y1 = fmaf(x1, c, -x2 * s);  // first of the pair
      const float y2 = fmaf(x2, c, x1 * s);   // second of the pair
      rl |= (uint32_t)f32_to_bf16(y1) << (16 * k);
      rh |= (uint32_t)f32_to_bf16(y2) << (16 * k);
    }
    ol[w] = rl;
    oh[w] = rh;
  }
  olo = make_uint4(ol[0], ol[1], ol[2], ol[3]);
  ohi = make_uint4(oh[0], oh[1], oh[2], oh[3]);
}

__global__ void __launch_bounds__(kRopeThreads) tree_rope_kernel(TreeRopeArgs a) {
  const Plan& p = a.p;
  // the attention kernel may begin its prefix loads now; it waits for this grid before
  // it reads q_rot and k_rot
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int b = blockIdx.x / p.T, i = blockIdx.x % p.T;
  int base = 0, n = 0;
  tree_range(p, a.cu_tree, b, &base, &n);
  if (i >= n) {  // a node slot past the sequence's tree
#if defined(LS_DEBUG)
    if (threadIdx.x == 0) a.rope_status[blockIdx.x] = 0u;
#endif
    return;
  }
  const int tid = threadIdx.x;
  const int half = p.d / 2;
  const int groups = half / 8;  // items: (head, group of 8 pairs); q heads first, then k_tree's
  const int items = (p.Hq + p.Hkv) * groups;
  const size_t node = (size_t)base + i;
  auto src_of = [&](int it) -> const uint16_t* {
    const int hh = it / groups, e0 = (it % groups) * 8;
    return hh < p.Hq ? a.q + (node * p.Hq + hh) * p.d + e0 : a.k_tree + (node * p.Hkv + (hh - p.Hq)) * p.d + e0;
  };
  auto dst_of = [&](int it) -> uint16_t* {
    const int hh = it / groups, e0 = (it % groups) * 8;
    return hh < p.Hq ? a.q_rot + (node * p.Hq + hh) * p.d + e0 : a.k_rot + (node * p.Hkv + (hh - p.Hq)) * p.d + e0;
  };
  uint32_t bad = 0u;  // index-checking builds: this CTA's failed checks
  LS_DCHECK(bad, b < p.B && node < (size_t)p.N);
  uint4 lo[kPrefetch], hi[kPrefetch];
#pragma unroll
  for (int k = 0; k < kPrefetch; ++k) {
    const int it = tid + k * kRopeThreads;
    if (it < items) {
      LS_DCHECK(bad, it / groups < p.Hq + p.Hkv && (it % groups) * 8 + 8 <= half);
      lo[k] = *reinterpret_cast<const uint4*>(src_of(it));
      hi[k] = *reinterpret_cast<const uint4*>(src_of(it) + half);
    }
  }

  __shared__ int32_t anc[2][kMaxTree], dist[2][kMaxTree];
  __shared__ float cos_s[64], sin_s[64];
  if (tid < n) {
    LS_DCHECK(bad, base + tid < p.N);
    const int32_t pp = a.parent[(size_t)base + tid];
    const bool link = tid > 0 && pp >= 0 && pp < tid;  // a valid link one level up
    anc[0][tid] = link ? pp : tid;                     // the root (or a bad link) points at itself
    dist[0][tid] = link ? 1 : 0;
  }
  __syncthreads();
  int cur = 0;
  for (int r = 0; r < 7; ++r) {  // 2^7 = 128 >= any depth
    if (tid < n) {
      const int up = anc[cur][tid];
      anc[cur ^ 1][tid] = anc[cur][up];
      dist[cur ^ 1][tid] = dist[cur][tid] + (up != tid ? dist[cur][up] : 0);
    }
    cur ^= 1;
    __syncthreads();
  }
  const int depth = dist[cur][i];
  const int32_t L = max(a.cu[b + 1] - a.cu[b], 0);
  const double pos = (double)L + (double)depth;
  if (tid < half) {
    // theta_e = base^(-2e/d); the angle pos * theta_e reduced to [-pi, pi]
    const double inv_freq = exp2(-(2.0 * tid / p.d) * a.log2_theta);
    const double ang = pos * inv_freq;
    constexpr double kTwoPiHi = 6.283185307179586232;     // 2 pi rounded to double
    constexpr double kTwoPiLo = 2.4492935982947064e-16;   // 2 pi - kTwoPiHi
    const double k = rint(ang * 0.15915494309189533577);  // ang / (2 pi), rounded
    const double r = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, ang));
    float s, c;
    sincosf((float)r, &s, &c);
    cos_s[tid] = c;
    sin_s[tid] = s;
  }
  __syncthreads();

#pragma unroll
  for (int k = 0; k < kPrefetch; ++k) {
    const int it = tid + k * kRopeThreads;
    if (it < items) {
      uint4 olo, ohi;
      rotate8(lo[k], hi[k], cos_s, sin_s, (it % groups) * 8, olo, ohi);
      *reinterpret_cast<uint4*>(dst_of(it)) = olo;
      *reinterpret_cast<uint4*>(dst_of(it) + half) = ohi;
    }
  }
  for (int it = tid + kPrefetch * kRopeThreads; it < items; it += kRopeThreads) {  // large head counts
    LS_DCHECK(bad, it / groups < p.Hq + p.Hkv);
    const uint4 l1 = *reinterpret_cast<const uint4*>(src_of(it));
    const uint4 h1 = *reinterpret_cast<const uint4*>(src_of(it) + half);
    uint4 olo, ohi;
    rotate8(l1, h1, cos_s, sin_s, (it % groups) * 8, olo, ohi);
    *reinterpret_cast<uint4*>(dst_of(it)) = olo;
    *reinterpret_cast<uint4*>(dst_of(it) + half) = ohi;
  }
#if defined(LS_DEBUG)
  // one word per node slot, read by the combine for the rows of this node
  bad = __syncthreads_or(bad) ? kErrIndex : 0u;
  if (tid == 0) a.rope_status[blockIdx.x] = bad;
#endif
}

}  // namespace

cudaError_t launch_tree_rope(const TreeRopeArgs& a, cudaStream_t stream) {
  const int64_t grid = (int64_t)a.p.B * a.p.T;
  if (grid == 0) return cudaSuccess;
  tree_rope_kernel<<<(unsigned)grid, kRopeThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace ls

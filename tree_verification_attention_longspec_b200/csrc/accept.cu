// Greedy acceptance of a verified draft tree.
//
// After the target model has run the tree (the attention of this library is its
// verification step; LongSpec, gist.science summary, section 2C), each tree node i has a
// row of logits: the target's distribution for the token after node i. Greedy decoding
// is lossless when the accepted tokens are exactly the ones the target would have chosen
// itself: starting at the root (the last token already accepted), the walk moves to a
// child whose draft token equals the argmax of the current node's logits, and stops when
// no child does; the argmax at the last node is the next token (the "bonus" token), so a
// step yields accepted + 1 tokens (the acceptance length tau of section 3). Ties are
// broken by the smallest index, both in the argmax (first maximal entry, NaN never
// chosen) and among matching siblings. The argmax is the first index of the largest
// value above -inf (NaN entries are skipped); a row with no such value gives index 0.
//
// Two kernels. argmax_part_kernel: the logits matrix is the only large input (nodes x
// vocabulary, HBM-bound), so every row is cut into S segments and each CTA finds the
// (max, first index) of one segment with 16-byte loads. accept_walk_kernel, one CTA per
// sequence and a programmatic dependent of the first, merges the segments of its nodes,
// marks for every node the smallest child whose token matches, and walks from the root.
#include <algorithm>

#include "ls_device.cuh"
#include "ls_verify_attn.h"

namespace ls {

struct AcceptArgs {
  const void* logits;      // [N][V] bf16 or fp32
  const int32_t* tokens;   // [N]
  const int32_t* parent;   // [N], local indices
  const int32_t* cu_tree;  // [B+1] or nullptr (T nodes each)
  int32_t* accept_len;     // [B]
  int32_t* accept_path;    // [B][T]
  int32_t* next_token;     // [B]
  float* part_val;         // [N][S]
  int32_t* part_idx;       // [N][S]
  int32_t B, T, N, V, S, seg, fp32, vec;
};

namespace {

constexpr int kArgmaxThreads = 256;
constexpr int kUnroll = 8;  // 16-byte loads in flight per thread
constexpr int kWalkThreads = kMaxTree;
constexpr int kMergeBatch = 16;  // segment results loaded together by the walk kernel

// (v, i) beats (w, j): larger value, or equal value and smaller index; NaN never wins
__device__ __forceinline__ bool beats(float v, int i, float w, int j) { return v > w || (v == w && i < j); }

__device__ __forceinline__ void take(float x, int i, float& bv, int& bi) {
  if (x > bv) {  // indices arrive in increasing order per thread: keep the first maximum
    bv = x;
    bi = i;
  }
}

__global__ void __launch_bounds__(kArgmaxThreads) argmax_part_kernel(AcceptArgs a) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int row = blockIdx.x / a.S, sg = blockIdx.x % a.S;
  const int64_t lo = (int64_t)sg * a.seg;
  const int64_t hi = min(lo + (int64_t)a.seg, (int64_t)a.V);
  float bv = -INFINITY;
  int bi = INT32_MAX;
  const int tid = threadIdx.x;
  if (a.fp32) {
    const float* r = static_cast<const float*>(a.logits) + (int64_t)row * a.V;
    if (a.vec) {  // lo, hi multiples of 4 elements (16 bytes) except hi = V, V % 4 == 0
      constexpr int kStep = 4 * kArgmaxThreads;
      for (int64_t e0 = lo + 4 * tid; e0 < hi; e0 += kUnroll * kStep) {
        float4 v[kUnroll];  // kUnroll loads in flight before any is used
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
          if (e0 + u * kStep < hi) v[u] = *reinterpret_cast<const float4*>(r + e0 + u * kStep);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int e = (int)(e0 + u * kStep);
          if (e < hi) {
            take(v[u].x, e, bv, bi);
            take(v[u].y, e + 1, bv, bi);
            take(v[u].z, e + 2, bv, bi);
            take(v[u].w, e + 3, bv, bi);
          }
        }
      }
    } else {
      for (int64_t e = lo + tid; e < hi; e += kArgmaxThreads) take(r[e], (int)e, bv, bi);
    }
  } else {
    const uint16_t* r = static_cast<const uint16_t*>(a.logits) + (int64_t)row * a.V;
    if (a.vec) {  // lo, hi multiples of 8 elements (16 bytes) except hi = V, V % 8 == 0
      constexpr int kStep = 8 * kArgmaxThreads;
      for (int64_t e0 = lo + 8 * tid; e0 < hi; e0 += kUnroll * kStep) {
        uint4 v[kUnroll];  // kUnroll loads in flight before any is used
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
          if (e0 + u * kStep < hi) v[u] = *reinterpret_cast<const uint4*>(r + e0 + u * kStep);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int e = (int)(e0 + u * kStep);
          if (e < hi) {
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              take(__uint_as_float(w[k] << 16), e + 2 * k, bv, bi);
              take(__uint_as_float(w[k] & 0xffff0000u), e + 2 * k + 1, bv, bi);
            }
          }
        }
      }
    } else {
      for (int64_t e = lo + tid; e < hi; e += kArgmaxThreads) take(bf16_to_f32(r[e]), (int)e, bv, bi);
    }
  }
  // warp, then block: the best (value, index) pair
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (beats(ov, oi, bv, bi)) {
      bv = ov;
      bi = oi;
    }
  }
  __shared__ float sv[kArgmaxThreads / 32];
  __shared__ int si[kArgmaxThreads / 32];
  const int warp = tid >> 5, lane = tid & 31;
  if (lane == 0) {
    sv[warp] = bv;
    si[warp] = bi;
  }
  __syncthreads();
  if (tid == 0) {
    for (int w = 1; w < kArgmaxThreads / 32; ++w)
      if (beats(sv[w], si[w], bv, bi)) {
        bv = sv[w];
        bi = si[w];
      }
    a.part_val[(int64_t)row * a.S + sg] = bv;
    a.part_idx[(int64_t)row * a.S + sg] = bi;
  }
}

__global__ void __launch_bounds__(kWalkThreads) accept_walk_kernel(AcceptArgs a) {
  const int b = blockIdx.x, tid = threadIdx.x;
  Plan p{};
  p.B = a.B;
  p.T = a.T;
  p.N = a.N;
  int base = 0, n = 0;
  bool ok = tree_range(p, a.cu_tree, b, &base, &n);
  __shared__ int32_t am[kMaxTree], par[kMaxTree], tok[kMaxTree], first_match[kMaxTree];
  // inputs that the first kernel does not write: read before waiting for it
  if (tid < n) {
    par[tid] = a.parent[base + tid];
    tok[tid] = a.tokens[base + tid];
  }
  first_match[tid] = INT32_MAX;
  const bool bad_link = tid < n && (tid == 0 ? par[tid] != -1 : (par[tid] < 0 || par[tid] >= tid));
  ok = ok && n > 0 && !__syncthreads_or(bad_link);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (ok && tid < n) {
    float bv = -INFINITY;
    int bi = INT32_MAX;
    const float* pv = a.part_val + (int64_t)(base + tid) * a.S;
    const int32_t* pi = a.part_idx + (int64_t)(base + tid) * a.S;
    for (int s0 = 0; s0 < a.S; s0 += kMergeBatch) {
      float v[kMergeBatch];  // a batch of segment results in flight before any is compared
      int i[kMergeBatch];
#pragma unroll
      for (int k = 0; k < kMergeBatch; ++k) {
        v[k] = s0 + k < a.S ? pv[s0 + k] : -INFINITY;
        i[k] = s0 + k < a.S ? pi[s0 + k] : INT32_MAX;
      }
#pragma unroll
      for (int k = 0; k < kMergeBatch; ++k)
        if (beats(v[k], i[k], bv, bi)) {
          bv = v[k];
          bi = i[k];
        }
    }
    am[tid] = bi == INT32_MAX ? 0 : bi;  // no value above -inf: index 0
  }
  __syncthreads();
  // the smallest child of every node whose draft token is that node's argmax
  if (ok && tid > 0 && tid < n && tok[tid] == am[par[tid]]) atomicMin(&first_match[par[tid]], tid);
  __syncthreads();
  if (tid == 0) {
    int32_t* path = a.accept_path + (int64_t)b * a.T;
    if (!ok) {
      a.accept_len[b] = -1;
      a.next_token[b] = -1;
    } else {
      int cur = 0, len = 0;
      path[0] = 0;
      while (first_match[cur] < n) {  // children lie above their parent: the walk ends
        cur = first_match[cur];
        path[++len] = cur;
      }
      a.accept_len[b] = len;
      a.next_token[b] = am[cur];
    }
  }
}

}  // namespace

}  // namespace ls

namespace {

int accept_plan(const ls_accept_dims* d, int32_t total_nodes, int* S, int* seg, size_t* bytes) {
  if (d == nullptr || d->batch < 1 || d->tree_size < 1 || d->vocab < 1) return LS_ERR_INVALID_ARG;
  if (d->tree_size > ls::kMaxTree) return LS_ERR_UNSUPPORTED;
  if (d->logits_dtype != LS_DTYPE_BF16 && d->logits_dtype != LS_DTYPE_F32) return LS_ERR_INVALID_ARG;
  if (total_nodes < 0 || (int64_t)total_nodes > (int64_t)d->batch * d->tree_size) return LS_ERR_INVALID_ARG;
  const int N = total_nodes;
  // segments: about 4 CTAs per SM of a 148-SM part in all, each at least 4096 entries,
  // a multiple of 8 entries (16 bytes of bf16)
  const int64_t target = 4 * 148;
  int64_t s = N > 0 ? (target + N - 1) / N : 1;
  s = std::max<int64_t>(1, std::min<int64_t>(s, (d->vocab + 4095) / 4096));
  int64_t sl = (d->vocab + s - 1) / s;
  sl = (sl + 7) / 8 * 8;
  s = (d->vocab + sl - 1) / sl;
  *S = (int)s;
  *seg = (int)sl;
  const uint64_t nv = (uint64_t)std::max(N, 1) * s;
  *bytes = ls::align256(nv * 4) + ls::align256(nv * 4);
  return LS_OK;
}

}  // namespace

extern "C" {

size_t ls_tree_accept_workspace_size(const ls_accept_dims* dims, int32_t total_nodes) {
  int S, seg;
  size_t bytes;
  if (accept_plan(dims, total_nodes, &S, &seg, &bytes) != LS_OK) return 0;
  return bytes;
}

int ls_tree_accept_greedy(const void* logits, const int32_t* tree_tokens, const int32_t* tree_parent,
                          const int32_t* cu_tree, int32_t total_nodes, int32_t* accept_len, int32_t* accept_path,
                          int32_t* next_token, const ls_accept_dims* dims, void* workspace, size_t workspace_bytes,
                          void* stream) {
  if (dims != nullptr && cu_tree == nullptr) total_nodes = dims->batch * dims->tree_size;
  int S, seg;
  size_t bytes;
  int rc = accept_plan(dims, total_nodes, &S, &seg, &bytes);
  if (rc != LS_OK) return rc;
  auto al4 = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 3u) == 0; };
  if (logits == nullptr || tree_tokens == nullptr || tree_parent == nullptr || accept_len == nullptr ||
      accept_path == nullptr || next_token == nullptr)
    return LS_ERR_INVALID_ARG;
  if (!al4(tree_tokens) || !al4(tree_parent) || !al4(accept_len) || !al4(accept_path) || !al4(next_token) ||
      (cu_tree != nullptr && !al4(cu_tree)))
    return LS_ERR_INVALID_ARG;
  const bool f32 = dims->logits_dtype == LS_DTYPE_F32;
  if ((reinterpret_cast<uintptr_t>(logits) & (f32 ? 3u : 1u)) != 0) return LS_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < bytes)
    return LS_ERR_WORKSPACE;
  ls::AcceptArgs a;
  a.logits = logits;
  a.tokens = tree_tokens;
  a.parent = tree_parent;
  a.cu_tree = cu_tree;
  a.accept_len = accept_len;
  a.accept_path = accept_path;
  a.next_token = next_token;
  const int N = total_nodes;
  const uint64_t nv = (uint64_t)std::max(N, 1) * S;
  a.part_val = static_cast<float*>(workspace);
  a.part_idx = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + ls::align256(nv * 4));
  a.B = dims->batch;
  a.T = dims->tree_size;
  a.N = N;
  a.V = dims->vocab;
  a.S = S;
  a.seg = seg;
  a.fp32 = f32 ? 1 : 0;
  // 16-byte loads when every row starts on a 16-byte boundary
  a.vec = (reinterpret_cast<uintptr_t>(logits) & 15u) == 0 && (f32 ? dims->vocab % 4 == 0 : dims->vocab % 8 == 0);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  (void)cudaGetLastError();
  if (N > 0) {
    ls::argmax_part_kernel<<<(unsigned)((int64_t)N * S), ls::kArgmaxThreads, 0, st>>>(a);
    if (cudaGetLastError() != cudaSuccess) return LS_ERR_CUDA;
  }
  // the walk is a programmatic dependent of the argmax kernel (it reads the tokens and
  // parents before waiting for that grid); without that kernel, an ordinary launch
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(dims->batch);
  cfg.blockDim = dim3(ls::kWalkThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = N > 0 ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, ls::accept_walk_kernel, a) != cudaSuccess) return LS_ERR_CUDA;
  return LS_OK;
}

}  // extern "C"

// C-ABI entry points: argument checks, the work split, workspace layout and launches.
// Declared and documented in include/ls_verify_attn.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <vector>

#include "ls_device.cuh"
#include "ls_verify_attn.h"

namespace {

using ls::Plan;

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultWaitNs = 4000000000ull;  // 4 s
constexpr uint64_t kMaxWaitNs = 60000000000ull;     // 60 s
int g_sm_count[kMaxDevices];  // 0 = not queried yet; a benign race writes the same value
int g_cc_major[kMaxDevices];

int device_info(int* sm_count, int* cc_major) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return LS_ERR_CUDA;
  if (dev < kMaxDevices && g_sm_count[dev] > 0) {
    *sm_count = g_sm_count[dev];
    *cc_major = g_cc_major[dev];
    return LS_OK;
  }
  int sms = 0, major = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return LS_ERR_CUDA;
  if (dev < kMaxDevices) {
    g_cc_major[dev] = major;
    g_sm_count[dev] = sms;
  }
  *sm_count = sms;
  *cc_major = major;
  return LS_OK;
}

int check_dims(const ls_verify_dims* d) {
  if (d == nullptr) return LS_ERR_INVALID_ARG;
  if (d->batch < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1 || d->tree_size < 1 ||
      d->max_prefix_len < 0)
    return LS_ERR_INVALID_ARG;
  if (d->num_q_heads % d->num_kv_heads != 0) return LS_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return LS_ERR_UNSUPPORTED;
  if (d->tree_size > ls::kMaxTree) return LS_ERR_UNSUPPORTED;
  // index arithmetic stays in int32 for rows and in size_t for element offsets
  const long long rows = (long long)d->batch * d->tree_size * d->num_q_heads;
  if (rows > (1ll << 30)) return LS_ERR_UNSUPPORTED;
  if (d->cu_seqlens_host != nullptr) {
    const int32_t* cu = d->cu_seqlens_host;
    if (cu[0] != 0) return LS_ERR_INVALID_ARG;
    for (int b = 0; b < d->batch; ++b)
      if (cu[b + 1] < cu[b]) return LS_ERR_INVALID_ARG;
  }
  return LS_OK;
}

// Checks the per-sequence tree options; nullptr means uniform trees, no RoPE.
int check_tree(const ls_verify_dims* d, const ls_tree_opts* t) {
  if (t == nullptr) return LS_OK;
  if (t->cu_tree != nullptr) {
    if ((reinterpret_cast<uintptr_t>(t->cu_tree) & 3u) != 0) return LS_ERR_INVALID_ARG;
    if (t->total_nodes < 0 || (long long)t->total_nodes > (long long)d->batch * d->tree_size)
      return LS_ERR_INVALID_ARG;
  }
  // a window shorter than the tree would also cut tree keys: not offered
  if (t->window < 0 || (t->window > 0 && t->window < d->tree_size)) return LS_ERR_INVALID_ARG;
  if (!(t->rope_theta >= 0.0) || !std::isfinite(t->rope_theta)) return LS_ERR_INVALID_ARG;
  if (t->rope_theta > 0.0 && t->rope_theta <= 1.0) return LS_ERR_INVALID_ARG;  // a base above 1
  if (t->wait_limit_ns > kMaxWaitNs) return LS_ERR_INVALID_ARG;
  return LS_OK;
}

// Chooses the chunk length C (in 128-key blocks) that minimises the estimated time of
// the partials kernel: waves of `slots` CTAs, each wave as long as its longest chunk
// plus a fixed per-chunk cost for loading Q and writing the partial. A sequence's key
// list is its prefix blocks plus one tree block, cut into ceil(blocks / C) chunks of
// nearly equal length (none longer than C). The estimate is closed-form: the plan is
// made on every call, so it must cost microseconds, not the milliseconds that simulating
// the grid's schedule would.
int make_plan(const ls_verify_dims* d, Plan* p, bool with_tree = true, const ls_tree_opts* tree = nullptr) {
  int rc = check_dims(d);
  if (rc != LS_OK) return rc;
  rc = check_tree(d, tree);
  if (rc != LS_OK) return rc;
  int sms = 0, major = 0;
  rc = device_info(&sms, &major);
  if (rc != LS_OK) return rc;
  if (major != 10) return LS_ERR_UNSUPPORTED;

  Plan q{};
  q.B = d->batch;
  q.Hq = d->num_q_heads;
  q.Hkv = d->num_kv_heads;
  q.d = d->head_dim;
  q.T = d->tree_size;
  q.g = q.Hq / q.Hkv;
  q.rows = q.T * q.g;
  q.N = tree != nullptr && tree->cu_tree != nullptr ? tree->total_nodes : q.B * q.T;
  q.rope = with_tree && tree != nullptr && tree->rope_theta > 0.0 ? 1 : 0;
  q.window = with_tree && tree != nullptr ? tree->window : 0;
  q.wait_ns = (int64_t)(tree != nullptr && tree->wait_limit_ns > 0 ? tree->wait_limit_ns : kDefaultWaitNs);
  if (q.g > ls::kUnitRows) return LS_ERR_UNSUPPORTED;
  q.tpu = ls::kUnitRows / q.g;
  q.rg = ls::ceil_div(q.T, q.tpu);
  q.scale = d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / std::sqrt((float)q.d);
  q.scale_log2 = (float)((double)q.scale * 1.4426950408889634074);
  // few output rows (a draft query or a small tree): one row per combine CTA, whose warps
  // split the row's partials, so that more warps share the merge
  const long long out_rows = (long long)q.B * q.T * q.Hq;
  q.combine_wide = out_rows < 4LL * sms ? 1 : 0;
  q.n_combine = (int32_t)(q.combine_wide ? out_rows : (out_rows + ls::kMergeRows - 1) / ls::kMergeRows);

  std::vector<int32_t> blocks(q.B);
  int32_t max_blocks = 0;
  for (int b = 0; b < q.B; ++b) {
    const int32_t L = d->cu_seqlens_host ? d->cu_seqlens_host[b + 1] - d->cu_seqlens_host[b]
                                         : d->max_prefix_len;
    blocks[b] = ls::prefix_blocks(ls::attended_len(q, L)) + (with_tree ? 1 : 0);  // prefix blocks, tree block
    if (blocks[b] > max_blocks) max_blocks = blocks[b];
  }
  const long long units = (long long)q.Hkv * q.rg;
  const long long slots = sms;  // one prefix CTA per SM
  const long long overhead = 2;  // per-chunk cost in blocks (Q load, partial store)
  int32_t best_C = max_blocks > 0 ? max_blocks : 1;
  long long best_cost = -1, best_n = 0;
  for (int32_t C = 1; C <= max_blocks; ++C) {
    long long n = 0;
    for (int b = 0; b < q.B; ++b) n += units * ls::ceil_div(blocks[b], C);
    const long long waves = (n + slots - 1) / slots;
    const long long cost = waves * (C + overhead);
    if (best_cost < 0 || cost < best_cost || (cost == best_cost && n < best_n)) {
      best_cost = cost;
      best_C = C;
      best_n = n;
    }
  }
  q.C = best_C;
  q.cu_n = 0;
  if (d->cu_seqlens_host != nullptr && q.B < ls::kPlanCu) {
    q.cu_n = q.B + 1;
    for (int b = 0; b <= q.B; ++b) q.cu_host[b] = d->cu_seqlens_host[b];
  }
  q.with_tree = with_tree ? 1 : 0;
  if (d->cu_seqlens_host) {
    q.uniform_n = -1;
  } else {
    q.uniform_n = max_blocks > 0 ? ls::ceil_div(max_blocks, q.C) : 0;
  }
  long long n = 0;
  for (int b = 0; b < q.B; ++b)
    n += units * (q.uniform_n >= 0 ? q.uniform_n : ls::ceil_div(blocks[b], q.C));
  if (n > (1ll << 30)) return LS_ERR_UNSUPPORTED;
  q.n_chunks = (int32_t)n;
  *p = q;
  return LS_OK;
}

bool aligned16(const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15u) == 0; }
bool aligned4(const void* x) { return (reinterpret_cast<uintptr_t>(x) & 3u) == 0; }

bool workspace_ok(const void* ws, size_t bytes, const ls::Layout& lay) {
  return ws != nullptr && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0 && bytes >= lay.total;
}

}  // namespace

extern "C" {

size_t ls_verify_attn_workspace_size(const ls_verify_dims* dims) {
  Plan p;
  if (make_plan(dims, &p) != LS_OK) return 0;
  return (size_t)ls::make_layout(p).total;
}

int ls_verify_attn_plan(const ls_verify_dims* dims, int32_t* partials_ctas, int32_t* blocks_per_chunk,
                        int32_t* combine_ctas) {
  Plan p;
  const int rc = make_plan(dims, &p);
  if (rc != LS_OK) return rc;
  if (partials_ctas) *partials_ctas = p.n_chunks;
  if (blocks_per_chunk) *blocks_per_chunk = p.C;
  if (combine_ctas) *combine_ctas = p.n_combine;
  return LS_OK;
}

}  // extern "C"

namespace {

// The partials stage for a packed (pg == nullptr) or paged K/V cache, after the tree
// kernel when RoPE is asked for; arguments checked.
int run_partials(const void* q, const void* k_cache, const void* v_cache, const void* k_tree, const void* v_tree,
                 const int32_t* tree_parent, const int32_t* cu_seqlens, const ls_verify_dims* dims,
                 const ls_paged_kv* pg, void* workspace, size_t workspace_bytes, void* stream,
                 bool with_tree = true, const ls_tree_opts* tree = nullptr, const Plan* planned = nullptr) {
  // the caller's plan for these arguments when it made one already (one plan per call)
  Plan p;
  if (planned != nullptr) {
    p = *planned;
  } else {
    const int rc0 = make_plan(dims, &p, with_tree, tree);
    if (rc0 != LS_OK) return rc0;
  }
  if (q == nullptr || !aligned16(q) || cu_seqlens == nullptr || !aligned4(cu_seqlens)) return LS_ERR_INVALID_ARG;
  if (with_tree) {
    if (k_tree == nullptr || v_tree == nullptr || !aligned16(k_tree) || !aligned16(v_tree))
      return LS_ERR_INVALID_ARG;
    if (tree_parent == nullptr || !aligned4(tree_parent)) return LS_ERR_INVALID_ARG;
  }
  const bool any_prefix =
      dims->cu_seqlens_host ? dims->cu_seqlens_host[dims->batch] > 0 : dims->max_prefix_len > 0;
  int64_t kv_rows = dims->cu_seqlens_host ? (int64_t)dims->cu_seqlens_host[dims->batch]
                                          : (int64_t)dims->batch * dims->max_prefix_len;
  if (pg != nullptr) {
    // pages of 16, 32 or 64 keys, or a multiple of 128 (a 128-key block never straddles
    // two pages then); enough table columns for the longest planned sequence
    const int32_t ps = pg->page_size;
    if (!(ps == 16 || ps == 32 || ps == 64 || (ps >= 128 && ps % 128 == 0 && ps <= (1 << 20))))
      return LS_ERR_UNSUPPORTED;
    if (pg->page_table == nullptr || !aligned4(pg->page_table) || pg->max_pages_per_seq < 1 || pg->num_pages < 1)
      return LS_ERR_INVALID_ARG;
    int64_t max_len = dims->max_prefix_len;
    if (dims->cu_seqlens_host)
      for (int b = 0; b < dims->batch; ++b)
        max_len = std::max<int64_t>(max_len, dims->cu_seqlens_host[b + 1] - dims->cu_seqlens_host[b]);
    if ((max_len + ps - 1) / ps > pg->max_pages_per_seq) return LS_ERR_INVALID_ARG;
    if (pg->num_pages * (int64_t)ps >= (int64_t)1 << 31) return LS_ERR_UNSUPPORTED;  // rows stay int32
    kv_rows = pg->num_pages * (int64_t)ps;
  }
  if (k_cache == nullptr || v_cache == nullptr || !aligned16(k_cache) || !aligned16(v_cache)) {
    // a call without prefix keys may pass null caches
    if (any_prefix || (k_cache != nullptr && !aligned16(k_cache)) || (v_cache != nullptr && !aligned16(v_cache)))
      return LS_ERR_INVALID_ARG;
  }
  if (!with_tree && p.n_chunks == 0) return LS_OK;  // no key at all: the combine writes the empty result
  const ls::Layout lay = ls::make_layout(p);
  if (!workspace_ok(workspace, workspace_bytes, lay)) return LS_ERR_WORKSPACE;
  char* ws = static_cast<char*>(workspace);
  (void)cudaGetLastError();  // clear a stale, non-sticky error from unrelated work
  ls::PartialsArgs pa;
  pa.q = static_cast<const uint16_t*>(q);
  // the tensor maps need an address even where no row is ever read through them
  pa.k_cache = static_cast<const uint16_t*>(k_cache ? k_cache : k_tree);
  pa.v_cache = static_cast<const uint16_t*>(v_cache ? v_cache : v_tree);
  pa.k_tree = static_cast<const uint16_t*>(with_tree ? k_tree : k_cache);
  pa.v_tree = static_cast<const uint16_t*>(with_tree ? v_tree : v_cache);
  pa.parent = tree_parent;
  pa.cu = cu_seqlens;
  pa.cu_tree = tree != nullptr ? tree->cu_tree : nullptr;
  pa.after_prep = 0;
  pa.page_table = pg ? pg->page_table : nullptr;
  pa.page_size = pg ? pg->page_size : 0;
  pa.max_pages = pg ? pg->max_pages_per_seq : 0;
  pa.o_part = reinterpret_cast<float*>(ws + lay.o_part);
  pa.lse_part = reinterpret_cast<float*>(ws + lay.lse_part);
  pa.chunk_status = reinterpret_cast<uint32_t*>(ws + lay.chunk_status);
  pa.p = p;
  // rows of the K/V tensors that the TMA descriptors may address (an upper bound is
  // enough: no block is ever read past the tensor)
  if (k_cache == nullptr) kv_rows = p.N;
  if (p.rope) {
    // rotate q and k_tree into the workspace; the partials kernel reads them from there
    ls::TreeRopeArgs ra;
    ra.q = pa.q;
    ra.k_tree = pa.k_tree;
    ra.parent = tree_parent;
    ra.cu = cu_seqlens;
    ra.cu_tree = pa.cu_tree;
    ra.q_rot = reinterpret_cast<uint16_t*>(ws + lay.q_rot);
    ra.k_rot = reinterpret_cast<uint16_t*>(ws + lay.k_rot);
    ra.rope_status = reinterpret_cast<uint32_t*>(ws + lay.rope_status);
    ra.log2_theta = std::log2(tree->rope_theta);
    ra.p = p;
    if (ls::launch_tree_rope(ra, static_cast<cudaStream_t>(stream)) != cudaSuccess) return LS_ERR_CUDA;
    pa.q = ra.q_rot;
    pa.k_tree = ra.k_rot;
    pa.after_prep = 1;
  }
  pa.kv_rows = kv_rows;
  const cudaError_t e = ls::launch_partials(pa, kv_rows, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return LS_ERR_CUDA;
  return LS_OK;
}

}  // namespace

extern "C" {

int ls_verify_attn_partials(const void* q, const void* k_cache, const void* v_cache, const void* k_tree,
                            const void* v_tree, const int32_t* tree_parent, const int32_t* cu_seqlens,
                            const ls_verify_dims* dims, void* workspace, size_t workspace_bytes, void* stream) {
  return run_partials(q, k_cache, v_cache, k_tree, v_tree, tree_parent, cu_seqlens, dims, nullptr, workspace,
                      workspace_bytes, stream);
}

}  // extern "C"

namespace {

int run_combine(const int32_t* cu_seqlens, void* out, float* lse, const ls_verify_dims* dims, void* workspace,
                size_t workspace_bytes, void* stream, bool with_tree, const ls_tree_opts* tree = nullptr,
                const Plan* planned = nullptr) {
  Plan p;
  if (planned != nullptr) {
    p = *planned;
  } else {
    const int rc0 = make_plan(dims, &p, with_tree, tree);
    if (rc0 != LS_OK) return rc0;
  }
  if (out == nullptr || !aligned16(out)) return LS_ERR_INVALID_ARG;
  if (cu_seqlens == nullptr || lse == nullptr || !aligned4(cu_seqlens) || !aligned4(lse)) return LS_ERR_INVALID_ARG;
  const ls::Layout lay = ls::make_layout(p);
  if (!workspace_ok(workspace, workspace_bytes, lay)) return LS_ERR_WORKSPACE;
  char* ws = static_cast<char*>(workspace);
  (void)cudaGetLastError();
  ls::CombineArgs ca;
  ca.cu = cu_seqlens;
  ca.cu_tree = tree != nullptr ? tree->cu_tree : nullptr;
  ca.o_part = reinterpret_cast<const float*>(ws + lay.o_part);
  ca.lse_part = reinterpret_cast<const float*>(ws + lay.lse_part);
  ca.chunk_status = reinterpret_cast<const uint32_t*>(ws + lay.chunk_status);
  ca.out = static_cast<uint16_t*>(out);
  ca.lse = lse;
  ca.status = reinterpret_cast<uint32_t*>(ws + lay.status);
  ca.rope_status = p.rope ? reinterpret_cast<const uint32_t*>(ws + lay.rope_status) : nullptr;
  // the partials kernel ran just before unless a prefix-only call had no key at all
  ca.after_partials = with_tree || p.n_chunks > 0 ? 1 : 0;
  ca.p = p;
  if (ls::launch_combine(ca, static_cast<cudaStream_t>(stream)) != cudaSuccess) return LS_ERR_CUDA;
  return LS_OK;
}

}  // namespace

extern "C" {

int ls_verify_attn_combine(const int32_t* cu_seqlens, void* out, float* lse, const ls_verify_dims* dims,
                           void* workspace, size_t workspace_bytes, void* stream) {
  return run_combine(cu_seqlens, out, lse, dims, workspace, workspace_bytes, stream, true);
}

size_t ls_cross_attn_workspace_size(const ls_verify_dims* dims) {
  Plan p;
  if (make_plan(dims, &p, false) != LS_OK) return 0;
  return (size_t)ls::make_layout(p).total;
}

int ls_cross_attn(const void* q, const void* k_cache, const void* v_cache, const int32_t* cu_seqlens, void* out,
                  float* lse, const ls_verify_dims* dims, void* workspace, size_t workspace_bytes, void* stream) {
  Plan p;
  int rc = make_plan(dims, &p, false);
  if (rc != LS_OK) return rc;
  if (out == nullptr || !aligned16(out) || lse == nullptr || !aligned4(lse)) return LS_ERR_INVALID_ARG;
  rc = run_partials(q, k_cache, v_cache, nullptr, nullptr, nullptr, cu_seqlens, dims, nullptr, workspace,
                    workspace_bytes, stream, false, nullptr, &p);
  if (rc != LS_OK) return rc;
  return run_combine(cu_seqlens, out, lse, dims, workspace, workspace_bytes, stream, false, nullptr, &p);
}

int ls_verify_attn(const void* q, const void* k_cache, const void* v_cache, const void* k_tree,
                   const void* v_tree, const int32_t* tree_parent, const int32_t* cu_seqlens,
                   void* out, float* lse, const ls_verify_dims* dims, void* workspace,
                   size_t workspace_bytes, void* stream) {
  // check every argument of both stages before launching the first
  Plan p;
  int rc = make_plan(dims, &p);
  if (rc != LS_OK) return rc;
  if (out == nullptr || !aligned16(out) || lse == nullptr || !aligned4(lse)) return LS_ERR_INVALID_ARG;
  rc = run_partials(q, k_cache, v_cache, k_tree, v_tree, tree_parent, cu_seqlens, dims, nullptr, workspace,
                    workspace_bytes, stream, true, nullptr, &p);
  if (rc != LS_OK) return rc;
  return run_combine(cu_seqlens, out, lse, dims, workspace, workspace_bytes, stream, true, nullptr, &p);
}

int ls_verify_attn_paged(const void* q, const void* k_pages, const void* v_pages, const ls_paged_kv* paged,
                         const void* k_tree, const void* v_tree, const int32_t* tree_parent,
                         const int32_t* cu_seqlens, void* out, float* lse, const ls_verify_dims* dims,
                         void* workspace, size_t workspace_bytes, void* stream) {
  Plan p;
  int rc = make_plan(dims, &p);
  if (rc != LS_OK) return rc;
  if (paged == nullptr) return LS_ERR_INVALID_ARG;
  if (out == nullptr || !aligned16(out) || lse == nullptr || !aligned4(lse)) return LS_ERR_INVALID_ARG;
  rc = run_partials(q, k_pages, v_pages, k_tree, v_tree, tree_parent, cu_seqlens, dims, paged, workspace,
                    workspace_bytes, stream, true, nullptr, &p);
  if (rc != LS_OK) return rc;
  return run_combine(cu_seqlens, out, lse, dims, workspace, workspace_bytes, stream, true, nullptr, &p);
}

size_t ls_verify_attn_ex_workspace_size(const ls_verify_dims* dims, const ls_tree_opts* tree) {
  Plan p;
  if (make_plan(dims, &p, true, tree) != LS_OK) return 0;
  return (size_t)ls::make_layout(p).total;
}

int ls_verify_attn_ex(const void* q, const void* k_cache, const void* v_cache, const ls_paged_kv* paged,
                      const void* k_tree, const void* v_tree, const int32_t* tree_parent, const int32_t* cu_seqlens,
                      const ls_tree_opts* tree, void* out, float* lse, const ls_verify_dims* dims, void* workspace,
                      size_t workspace_bytes, void* stream) {
  Plan p;
  int rc = make_plan(dims, &p, true, tree);
  if (rc != LS_OK) return rc;
  if (out == nullptr || !aligned16(out) || lse == nullptr || !aligned4(lse)) return LS_ERR_INVALID_ARG;
  rc = run_partials(q, k_cache, v_cache, k_tree, v_tree, tree_parent, cu_seqlens, dims, paged, workspace,
                    workspace_bytes, stream, true, tree, &p);
  if (rc != LS_OK) return rc;
  return run_combine(cu_seqlens, out, lse, dims, workspace, workspace_bytes, stream, true, tree, &p);
}

int ls_verify_attn_check(const ls_verify_dims* dims, const void* workspace, void* stream) {
  Plan p;
  int rc = make_plan(dims, &p);
  if (rc != LS_OK) return rc;
  if (workspace == nullptr) return LS_ERR_WORKSPACE;
  const ls::Layout lay = ls::make_layout(p);
  std::vector<uint32_t> st(p.n_combine);
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return LS_ERR_CUDA;
  if (cudaMemcpy(st.data(), static_cast<const char*>(workspace) + lay.status,
                 st.size() * sizeof(uint32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LS_ERR_CUDA;
  uint32_t all = 0;
  for (uint32_t v : st) all |= v;
  if (all & ls::kErrLengths) return LS_ERR_LENGTHS;
  if (all & ls::kErrBadTree) return LS_ERR_BAD_TREE;
  if (all & ls::kErrTimeout) return LS_ERR_TIMEOUT;
  if (all & ls::kErrIndex) return LS_ERR_INDEX;
  return LS_OK;
}

const char* ls_status_string(int status) {
  switch (status) {
    case LS_OK: return "ok";
    case LS_ERR_INVALID_ARG: return "invalid argument";
    case LS_ERR_UNSUPPORTED: return "unsupported shape or device";
    case LS_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case LS_ERR_CUDA: return "CUDA launch or copy failed";
    case LS_ERR_BAD_TREE: return "tree_parent is not a rooted tree with parent[i] < i";
    case LS_ERR_TIMEOUT: return "a device-side wait timed out";
    case LS_ERR_LENGTHS: return "device cu_seqlens disagrees with the planned lengths";
    case LS_ERR_INDEX: return "an index check of the index-checking build failed";
    default: return "unknown status";
  }
}

}  // extern "C"

// Device-side helpers and kernel argument blocks.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "ls_plan.cuh"

namespace ls {

constexpr float kLn2 = 0.693147180559945309417f;

// The partials kernel: every chunk's prefix blocks and, for the chunk that holds it,
// the masked tree block.
struct PartialsArgs {
  const uint16_t* q;
  const uint16_t* k_cache;
  const uint16_t* v_cache;
  const uint16_t* k_tree;
  const uint16_t* v_tree;
  const int32_t* parent;
  const int32_t* cu;
  const int32_t* cu_tree;  // per-sequence tree offsets; nullptr: T nodes each
  // paged K/V cache: page_table[b * max_pages + i] is the physical page of keys
  // [i * page_size, (i + 1) * page_size) of sequence b; nullptr = keys packed by cu
  const int32_t* page_table;
  int32_t page_size;
  int32_t max_pages;
  float* o_part;
  float* lse_part;
  uint32_t* chunk_status;
  int32_t after_prep;  // q and k_tree are written by the tree kernel launched just before
  int64_t kv_rows;     // rows of k_cache / v_cache (of the pages, for a paged cache)
  Plan p;
};

// The tree kernel: every node's depth, and q and k_tree rotated (RoPE) to the node's
// position prefix length + depth.
struct TreeRopeArgs {
  const uint16_t* q;
  const uint16_t* k_tree;
  const int32_t* parent;
  const int32_t* cu;
  const int32_t* cu_tree;
  uint16_t* q_rot;
  uint16_t* k_rot;
  uint32_t* rope_status;  // index-checking builds: one word per CTA (node slot b * T + i)
  double log2_theta;  // log2 of the RoPE base
  Plan p;
};

// The combine kernel: the log-sum-exp merge of every chunk's partial.
struct CombineArgs {
  const int32_t* cu;
  const int32_t* cu_tree;
  const float* o_part;
  const float* lse_part;
  const uint32_t* chunk_status;
  uint16_t* out;
  float* lse;
  uint32_t* status;
  const uint32_t* rope_status;  // index-checking builds, with RoPE: the tree kernel's words
  int32_t after_partials;  // launched right after the partials kernel: a programmatic dependent
  Plan p;
};

__device__ __forceinline__ float bf16_to_f32(uint16_t bits) {
  return __uint_as_float(static_cast<uint32_t>(bits) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&h);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace ls

// Launchers (defined in the kernel files, called by the host API).
namespace ls {
cudaError_t launch_partials(const PartialsArgs& a, int64_t kv_rows, cudaStream_t stream);  // kv_rows: rows of the K/V tensors
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream);
cudaError_t launch_tree_rope(const TreeRopeArgs& a, cudaStream_t stream);
}  // namespace ls

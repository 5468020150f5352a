// ls_verify_attn_static: tree-verification attention for callers that cannot allocate
// device memory.
//
// ls_verify_attn needs a caller-provided workspace for the attention partials. Some
// callers only ever receive their input and output buffers and have no way to obtain
// more device memory: for example an operator plugin running inside an inference
// engine that owns the whole device heap and exposes no allocator to its plugins, or
// code that must not call cudaMalloc because it would synchronise the device or break
// the host application's memory accounting. This entry point serves them: its scratch
// is a fixed array in the library's own device memory, so the call allocates nothing.
//
// The array is a file-scope __device__ variable of kStaticScratchBytes. Every GPU
// that loads this library holds it until the process exits, and every call on that
// GPU shares it.
#include <cuda_runtime.h>

#include <cstdint>

#include "ls_verify_attn.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int kMaxDevices = 64;

// The scratch itself. Host code must not use its name as a pointer: on the host it is
// only a stand-in for the symbol, so its device address is looked up below.
static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

// Device address of g_scratch, per device, looked up once and kept for the life of the
// process. cudaDeviceReset unloads this library's device code and a later call may find
// the array elsewhere, so after a reset the process must not call this entry again.
void* g_scratch_addr[kMaxDevices];

}  // namespace

extern "C" {

LS_API int ls_verify_attn_static(const void* q, const void* k_cache, const void* v_cache, const void* k_tree,
                                 const void* v_tree, const int32_t* tree_parent, const int32_t* cu_seqlens,
                                 void* out, float* lse, const ls_verify_dims* dims, void* stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LS_ERR_CUDA;
  if (g_scratch_addr[dev] == nullptr) {
    // first call on this device: find where the array lives in its memory
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_scratch) != cudaSuccess || ptr == nullptr) return LS_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
  }
  const size_t need = ls_verify_attn_workspace_size(dims);
  if (need == 0) {
    // invalid or unsupported dims: let the regular entry point name the reason
    return ls_verify_attn(q, k_cache, v_cache, k_tree, v_tree, tree_parent, cu_seqlens, out, lse, dims,
                          nullptr, 0, stream);
  }
  if (need > kStaticScratchBytes) return LS_ERR_WORKSPACE;
  return ls_verify_attn(q, k_cache, v_cache, k_tree, v_tree, tree_parent, cu_seqlens, out, lse, dims,
                        g_scratch_addr[dev], kStaticScratchBytes, stream);
}

}  // extern "C"

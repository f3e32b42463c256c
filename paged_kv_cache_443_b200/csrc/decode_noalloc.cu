// decode_noalloc.cu -- pa_decode_noalloc: decode attention for callers that
// cannot allocate device memory.
//
// pa_decode needs scratch space for its split-K partials, which the caller
// passes in.  Some callers have no way to provide it: a serving runtime that
// has already handed all free device memory to its KV-cache pool (a later
// cudaMalloc fails or fragments that pool), plain C host code that links only
// this library and owns no device allocator, and latency-critical loops that
// cannot afford cudaMalloc's implicit device synchronisation.  This entry point
// takes the scratch from a fixed array in this file instead, so it allocates
// nothing.
//
// The array lives in every GPU that loads the library, until the process
// exits.  In host code its name is only a host-side stand-in, so the kernels
// are given the device address that cudaGetSymbolAddress returns for the
// current device; that lookup runs on the first call made on each device.
#include <cuda_runtime.h>

#include <mutex>

#include "pa_internal.h"
#include "pagedkv.h"

namespace {

// Largest split-K workspace this entry point serves: 32 MiB.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

__device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
float* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device (looked up once
// per device, with that device current).  nullptr on a CUDA error.
float* scratch_address() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    pa::fail(PA_ERR_CUDA, "pa_decode_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev]) return g_scratch_addr[dev];
  float* ptr = nullptr;
  e = cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_noalloc_scratch);
  if (e != cudaSuccess || ptr == nullptr) {
    pa::fail(PA_ERR_CUDA, "pa_decode_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    return nullptr;
  }
  g_scratch_addr[dev] = ptr;
  return ptr;
}

}  // namespace

extern "C" pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* block_tables,
                                       int max_blocks_per_seq, const int32_t* context_lens,
                                       int num_seqs, int num_heads, int num_kv_heads,
                                       int head_size, int block_size, int num_blocks, float scale,
                                       pa_dtype dtype, int partition_size, int max_context_len,
                                       void* stream) {
  if (pa_decode_num_partitions(max_context_len, partition_size) < 0)
    return pa::fail(PA_ERR_INVALID, "pa_decode_noalloc: bad partition_size %d", partition_size);
  const size_t need = pa_decode_workspace_bytes(num_seqs, num_heads, head_size, max_context_len,
                                                partition_size);
  if (need > kNoAllocScratchBytes)
    return pa::fail(PA_ERR_UNSUPPORTED,
                    "pa_decode_noalloc: this batch needs %zu bytes of split-K scratch, more than "
                    "the fixed %zu-byte array; use pa_decode with a caller-provided workspace, or "
                    "fewer sequences / a larger partition_size",
                    need, kNoAllocScratchBytes);
  float* scratch = nullptr;
  if (need > 0 && num_seqs > 0) {
    scratch = scratch_address();
    if (!scratch) return PA_ERR_CUDA;
  }
  return pa_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                   num_seqs, num_heads, num_kv_heads, head_size, block_size, num_blocks, scale,
                   dtype, partition_size, max_context_len, scratch,
                   scratch ? kNoAllocScratchBytes : 0, stream);
}

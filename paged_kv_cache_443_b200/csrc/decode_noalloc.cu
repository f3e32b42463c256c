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
// current device; that lookup runs on the first call made on each device, and
// again whenever the device's current context is not the one the address was
// looked up in (after cudaDeviceReset the module is loaded anew, possibly at
// another address).
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "pa_internal.h"
#include "pagedkv.h"

namespace {

// Largest split-K workspace this entry point serves: 32 MiB.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

__device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
struct ScratchAddr {
  float* ptr = nullptr;
  unsigned long long ctx_id = 0;  // context the address belongs to (0: unknown)
};
ScratchAddr g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context; false when there is
// none yet or the driver does not offer the query.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS && *id != 0;
}

// Device address of g_noalloc_scratch in the current device's current context
// (looked up with that device current, and cached per device and context).
// nullptr on a CUDA error.
float* scratch_address() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    pa::fail(PA_ERR_CUDA, "pa_decode_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
    return nullptr;
  }
  unsigned long long ctx = 0;
  const bool known = current_context_id(&ctx);
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchAddr& c = g_scratch[dev];
  if (c.ptr && known && c.ctx_id == ctx) return c.ptr;
  float* ptr = nullptr;
  e = cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_noalloc_scratch);
  if (e != cudaSuccess || ptr == nullptr) {
    pa::fail(PA_ERR_CUDA, "pa_decode_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    return nullptr;
  }
  // the lookup made the device's primary context current if none was; without
  // a context id every call looks the address up again
  c.ptr = ptr;
  c.ctx_id = current_context_id(&ctx) ? ctx : 0;
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

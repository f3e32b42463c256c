// api.cpp -- the C ABI of libpagedkv.so for the device calls: argument checks
// (all before any launch, so a rejected call has no side effect), workspace
// sizing and dispatch to the kernel launchers.  See include/pagedkv.h for the
// contract of every entry point.
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "pa_internal.h"
#include "pagedkv.h"

namespace {

constexpr const char* kVersion = "pagedkv-b200 0.1.0 (sm_100a)";

bool supported_head(int d) { return d == 64 || d == 128; }
bool supported_block(int bs) { return bs == 8 || bs == 16 || bs == 32; }
bool supported_group(int g) { return g == 1 || g == 2 || g == 4 || g == 8; }

int resolve_partition(int partition_size) {
  if (partition_size == 0) return pa::kDefaultPartition;
  if (partition_size < 0 || partition_size % pa::kStageTokens != 0) return -1;
  return partition_size;
}

int64_t num_partitions(int max_context_len, int P) {
  if (max_context_len <= 0) return 1;
  return (static_cast<int64_t>(max_context_len) + P - 1) / P;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

// Partition length pa_decode (and pa_decode_fp8) use for partition_size = 0.
// Every CTA pays a fixed set-up and pipeline fill, so the partitions are as
// long as still gives at least 8 CTAs per SM at the longest context: for the
// tensor-core kernels (fp16/bf16 queries, head size 128, 4 or 8 query heads per
// kv head; 16-bit or E4M3 caches, which also stream several partitions per
// CTA) the longest of 4096 / 2048 / 1024 tokens; for the CUDA-core kernel 1024
// (2048 measured slower at opt13b: fewer, longer CTAs leave the last wave
// thin); else the default.
int auto_partition(int num_seqs, int num_heads, int num_kv_heads, int head_size, pa_dtype dtype,
                   int max_context_len) {
  const int G = num_kv_heads > 0 ? num_heads / num_kv_heads : 0;
  const bool tc = (dtype == PA_F16 || dtype == PA_BF16) && head_size == 128 && (G == 4 || G == 8);
  const int64_t want = 8ll * num_sms();
  for (int P : {4096, 2048, 1024}) {
    if (!tc && P > 1024) continue;
    const int64_t ctas = static_cast<int64_t>(num_seqs) * num_kv_heads * num_partitions(max_context_len, P);
    if (ctas >= want) return P;
  }
  return pa::kDefaultPartition;
}

size_t workspace_bytes(int64_t B, int64_t Hq, int64_t D, int64_t NP) {
  if (NP <= 1 || B <= 0) return 0;
  const size_t raw = static_cast<size_t>(B * Hq * NP * (D + 2) * 4);
  return (raw + 255) / 256 * 256;
}

// Shared checks of pa_decode / pa_decode_partitions / pa_decode_reduce.
pa_status check_decode(const char* fn, int num_seqs, int num_heads, int num_kv_heads,
                       int head_size, pa_dtype dtype, int partition_size, int max_context_len,
                       int* P_out, int64_t* NP_out) {
  if (pa::elem_size(dtype) == 0) return pa::fail(PA_ERR_INVALID, "%s: unknown dtype %d", fn, dtype);
  if (dtype == PA_FP8_E4M3)
    return pa::fail(PA_ERR_UNSUPPORTED,
                    "%s: E4M3 is a cache type only; q and out must be f32, f16 or bf16 (the "
                    "*_fp8 calls take an E4M3 cache)", fn);
  if (num_seqs < 0) return pa::fail(PA_ERR_INVALID, "%s: num_seqs < 0", fn);
  if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0)
    return pa::fail(PA_ERR_INVALID, "%s: num_heads (%d) must be a positive multiple of num_kv_heads (%d)",
                    fn, num_heads, num_kv_heads);
  if (num_kv_heads > 65535) return pa::fail(PA_ERR_UNSUPPORTED, "%s: num_kv_heads > 65535", fn);
  if (!supported_group(num_heads / num_kv_heads))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: query heads per kv head must be 1, 2, 4 or 8 (got %d)",
                    fn, num_heads / num_kv_heads);
  if (head_size <= 0) return pa::fail(PA_ERR_INVALID, "%s: head_size <= 0", fn);
  if (!supported_head(head_size))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: head_size must be 64 or 128 (got %d)", fn, head_size);
  const int P = resolve_partition(partition_size);
  if (P < 0)
    return pa::fail(PA_ERR_INVALID, "%s: partition_size must be 0 or a positive multiple of %d",
                    fn, pa::kStageTokens);
  if (max_context_len < 0) return pa::fail(PA_ERR_INVALID, "%s: max_context_len < 0", fn);
  const int64_t NP = num_partitions(max_context_len, P);
  if (NP > 65535) return pa::fail(PA_ERR_UNSUPPORTED, "%s: more than 65535 partitions", fn);
  *P_out = P;
  *NP_out = NP;
  return PA_OK;
}

pa_status check_decode_full(const char* fn, void* out, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* block_tables,
                            int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                            int num_heads, int num_kv_heads, int head_size, int block_size,
                            int num_blocks, float scale, pa_dtype dtype, int partition_size,
                            int max_context_len, void* workspace, size_t workspace_bytes_in,
                            pa::DecodeArgs* a) {
  int P = 0;
  int64_t NP = 0;
  pa_status st = check_decode(fn, num_seqs, num_heads, num_kv_heads, head_size, dtype,
                              partition_size, max_context_len, &P, &NP);
  if (st != PA_OK) return st;
  if (block_size <= 0) return pa::fail(PA_ERR_INVALID, "%s: block_size <= 0", fn);
  if (!supported_block(block_size))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: block_size must be 8, 16 or 32 (got %d)", fn, block_size);
  if (num_blocks <= 0) return pa::fail(PA_ERR_INVALID, "%s: num_blocks <= 0", fn);
  if (max_blocks_per_seq <= 0) return pa::fail(PA_ERR_INVALID, "%s: max_blocks_per_seq <= 0", fn);
  if (static_cast<int64_t>(max_context_len) > static_cast<int64_t>(max_blocks_per_seq) * block_size)
    return pa::fail(PA_ERR_INVALID, "%s: max_context_len %d exceeds max_blocks_per_seq * block_size",
                    fn, max_context_len);
  if (!std::isfinite(scale)) return pa::fail(PA_ERR_INVALID, "%s: scale is not finite", fn);
  if (num_seqs > 0) {
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
      return pa::fail(PA_ERR_INVALID, "%s: NULL device pointer", fn);
    if (!pa::aligned16(out) || !pa::aligned16(q) || !pa::aligned16(k_cache) ||
        !pa::aligned16(v_cache))
      return pa::fail(PA_ERR_INVALID, "%s: out, q and the caches must be 16-byte aligned", fn);
    if ((reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
        (reinterpret_cast<uintptr_t>(context_lens) & 3u))
      return pa::fail(PA_ERR_INVALID, "%s: block_tables / context_lens must be 4-byte aligned", fn);
  }
  const size_t need = workspace_bytes(num_seqs, num_heads, head_size, NP);
  if (need > 0) {
    if (!workspace || workspace_bytes_in < need)
      return pa::fail(PA_ERR_INVALID, "%s: workspace of %zu bytes needed (got %zu%s)", fn, need,
                      workspace_bytes_in, workspace ? "" : ", NULL");
    if (!pa::aligned16(workspace))
      return pa::fail(PA_ERR_INVALID, "%s: workspace must be 16-byte aligned", fn);
  }
  a->out = out;
  a->q = q;
  a->k_cache = k_cache;
  a->v_cache = v_cache;
  a->block_tables = block_tables;
  a->context_lens = context_lens;
  a->workspace = need > 0 ? static_cast<float*>(workspace) : nullptr;
  a->max_blocks = max_blocks_per_seq;
  a->num_seqs = num_seqs;
  a->Hq = num_heads;
  a->Hkv = num_kv_heads;
  a->D = head_size;
  a->block_size = block_size;
  a->num_blocks = num_blocks;
  a->partition_size = P;
  a->num_partitions = static_cast<int>(NP);
  a->scale = scale;
  a->dtype = dtype;
  a->kv_dtype = dtype;
  a->k_scale = a->v_scale = 1.f;
  return PA_OK;
}

bool valid_kv_scale(float s) { return std::isfinite(s) && s > 0.f; }

// pa_decode_fp8 / pa_decode_partitions_fp8: the pa_decode checks with q's
// dtype, then the E4M3 cache and its scales.
pa_status check_decode_fp8(const char* fn, void* out, const void* q, const void* k_cache,
                           const void* v_cache, const int32_t* block_tables,
                           int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                           int num_heads, int num_kv_heads, int head_size, int block_size,
                           int num_blocks, float scale, pa_dtype dtype, float k_scale,
                           float v_scale, int partition_size, int max_context_len,
                           void* workspace, size_t workspace_bytes_in, pa::DecodeArgs* a) {
  if (!valid_kv_scale(k_scale) || !valid_kv_scale(v_scale))
    return pa::fail(PA_ERR_INVALID, "%s: k_scale and v_scale must be finite and > 0", fn);
  pa_status st = check_decode_full(fn, out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                   context_lens, num_seqs, num_heads, num_kv_heads, head_size,
                                   block_size, num_blocks, scale, dtype, partition_size,
                                   max_context_len, workspace, workspace_bytes_in, a);
  if (st != PA_OK) return st;
  a->kv_dtype = PA_FP8_E4M3;
  a->k_scale = k_scale;
  a->v_scale = v_scale;
  return PA_OK;
}

int launch_partitions(const pa::DecodeArgs& a, unsigned int* status, void* stream) {
  if (pa::decode_tc8_supported(a)) return pa::launch_decode_partitions_tc8(a, status, stream);
  if (a.kv_dtype == a.dtype && pa::decode_tc_supported(a)) return pa::launch_decode_partitions_tc(a, status, stream);
  return pa::launch_decode_partitions(a, status, stream);
}

pa_status launch_status(const char* fn, int err, int n_launched) {
  if (err != cudaSuccess)
    return pa::fail(PA_ERR_CUDA, "%s: launch failed: %s", fn,
                    cudaGetErrorString(static_cast<cudaError_t>(err)));
  pa::count_launch(n_launched);
  return PA_OK;
}

}  // namespace

extern "C" const char* pa_version(void) { return kVersion; }

extern "C" int pa_decode_default_partition_size(void) { return pa::kDefaultPartition; }

extern "C" int pa_decode_num_partitions(int max_context_len, int partition_size) {
  const int P = resolve_partition(partition_size);
  if (P < 0) return -1;
  const int64_t np = num_partitions(max_context_len, P);
  return np > 0x7fffffff ? -1 : static_cast<int>(np);
}

extern "C" size_t pa_decode_workspace_bytes(int num_seqs, int num_heads, int head_size,
                                            int max_context_len, int partition_size) {
  const int P = resolve_partition(partition_size);
  if (P < 0 || num_seqs < 0 || num_heads < 0 || head_size < 0) return 0;
  return workspace_bytes(num_seqs, num_heads, head_size, num_partitions(max_context_len, P));
}

extern "C" pa_status pa_decode_partitions(void* out, const void* q, const void* k_cache,
                                          const void* v_cache, const int32_t* block_tables,
                                          int max_blocks_per_seq, const int32_t* context_lens,
                                          int num_seqs, int num_heads, int num_kv_heads,
                                          int head_size, int block_size, int num_blocks,
                                          float scale, pa_dtype dtype, int partition_size,
                                          int max_context_len, void* workspace,
                                          size_t workspace_bytes_in, void* stream) {
  pa::DecodeArgs a;
  pa_status st = check_decode_full("pa_decode_partitions", out, q, k_cache, v_cache, block_tables,
                                   max_blocks_per_seq, context_lens, num_seqs, num_heads,
                                   num_kv_heads, head_size, block_size, num_blocks, scale, dtype,
                                   partition_size, max_context_len, workspace, workspace_bytes_in,
                                   &a);
  if (st != PA_OK || num_seqs == 0) return st;
  unsigned int* status = pa::device_status_word();
  if (!status) return PA_ERR_CUDA;
  return launch_status("pa_decode_partitions", launch_partitions(a, status, stream), 1);
}

extern "C" pa_status pa_decode_reduce(void* out, const int32_t* context_lens, int num_seqs,
                                      int num_heads, int head_size, pa_dtype dtype,
                                      int partition_size, int max_context_len,
                                      const void* workspace, size_t workspace_bytes_in,
                                      void* stream) {
  int P = 0;
  int64_t NP = 0;
  // the kv-head count does not matter here; pass num_heads for both
  pa_status st = check_decode("pa_decode_reduce", num_seqs, num_heads, num_heads, head_size, dtype,
                              partition_size, max_context_len, &P, &NP);
  if (st != PA_OK) return st;
  const size_t need = workspace_bytes(num_seqs, num_heads, head_size, NP);
  if (need == 0 || num_seqs == 0) return PA_OK;
  if (!out || !context_lens || !workspace)
    return pa::fail(PA_ERR_INVALID, "pa_decode_reduce: NULL device pointer");
  if (workspace_bytes_in < need)
    return pa::fail(PA_ERR_INVALID, "pa_decode_reduce: workspace of %zu bytes needed (got %zu)",
                    need, workspace_bytes_in);
  if (!pa::aligned16(out) || !pa::aligned16(workspace))
    return pa::fail(PA_ERR_INVALID, "pa_decode_reduce: out and workspace must be 16-byte aligned");
  pa::DecodeArgs a{};
  a.out = out;
  a.context_lens = context_lens;
  a.workspace = const_cast<float*>(static_cast<const float*>(workspace));
  a.num_seqs = num_seqs;
  a.Hq = num_heads;
  a.Hkv = num_heads;
  a.D = head_size;
  a.partition_size = P;
  a.num_partitions = static_cast<int>(NP);
  a.dtype = dtype;
  return launch_status("pa_decode_reduce", pa::launch_decode_reduce(a, nullptr, stream), 1);
}

extern "C" int pa_decode_auto_partition_size(int num_seqs, int num_heads, int num_kv_heads,
                                             int head_size, pa_dtype dtype, int max_context_len) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
      head_size <= 0 || pa::elem_size(dtype) == 0 || max_context_len < 0)
    return -1;
  return auto_partition(num_seqs, num_heads, num_kv_heads, head_size, dtype, max_context_len);
}

extern "C" int pa_decode_fp8_auto_partition_size(int num_seqs, int num_heads, int num_kv_heads,
                                                 int head_size, pa_dtype dtype,
                                                 int max_context_len) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
      head_size <= 0 || pa::elem_size(dtype) == 0 || dtype == PA_FP8_E4M3 || max_context_len < 0)
    return -1;
  return auto_partition(num_seqs, num_heads, num_kv_heads, head_size, dtype, max_context_len);
}

extern "C" pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* context_lens, int num_seqs, int num_heads,
                               int num_kv_heads, int head_size, int block_size, int num_blocks,
                               float scale, pa_dtype dtype, int partition_size,
                               int max_context_len, void* workspace, size_t workspace_bytes_in,
                               void* stream) {
  // 0 = the automatic length; it never needs more workspace than the default
  // (a longer partition means fewer partials), which is what
  // pa_decode_workspace_bytes(..., 0) sized
  if (partition_size == 0 && num_heads > 0 && num_kv_heads > 0)
    partition_size =
        auto_partition(num_seqs, num_heads, num_kv_heads, head_size, dtype, max_context_len);
  pa::DecodeArgs a;
  pa_status st = check_decode_full("pa_decode", out, q, k_cache, v_cache, block_tables,
                                   max_blocks_per_seq, context_lens, num_seqs, num_heads,
                                   num_kv_heads, head_size, block_size, num_blocks, scale, dtype,
                                   partition_size, max_context_len, workspace, workspace_bytes_in,
                                   &a);
  if (st != PA_OK || num_seqs == 0) return st;
  unsigned int* status = pa::device_status_word();
  if (!status) return PA_ERR_CUDA;
  st = launch_status("pa_decode", launch_partitions(a, status, stream), 1);
  if (st != PA_OK || a.num_partitions <= 1) return st;
  return launch_status("pa_decode", pa::launch_decode_reduce(a, status, stream), 1);
}

extern "C" pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                          void* v_cache, const int64_t* slot_mapping,
                                          int num_tokens, int num_kv_heads, int head_size,
                                          int block_size, int num_blocks, pa_dtype dtype,
                                          void* stream) {
  const char* fn = "pa_reshape_and_cache";
  const int es = pa::elem_size(dtype);
  if (es == 0) return pa::fail(PA_ERR_INVALID, "%s: unknown dtype %d", fn, dtype);
  if (num_tokens < 0) return pa::fail(PA_ERR_INVALID, "%s: num_tokens < 0", fn);
  if (num_kv_heads <= 0 || head_size <= 0 || block_size <= 0 || num_blocks <= 0)
    return pa::fail(PA_ERR_INVALID, "%s: sizes must be positive", fn);
  if (!supported_head(head_size))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: head_size must be 64 or 128", fn);
  if (!supported_block(block_size))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: block_size must be 8, 16 or 32", fn);
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping)
    return pa::fail(PA_ERR_INVALID, "%s: NULL device pointer", fn);
  if (!pa::aligned16(key) || !pa::aligned16(value) || !pa::aligned16(k_cache) ||
      !pa::aligned16(v_cache) || (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return pa::fail(PA_ERR_INVALID, "%s: key/value/caches must be 16-byte aligned, slots 8", fn);
  unsigned int* status = pa::device_status_word();
  if (!status) return PA_ERR_CUDA;
  return launch_status(fn,
                       pa::launch_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping,
                                                    num_tokens, num_kv_heads, head_size,
                                                    block_size, num_blocks, es, status, stream),
                       1);
}

extern "C" pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_pairs,
                                    int num_pairs, int num_kv_heads, int head_size,
                                    int block_size, int num_blocks, pa_dtype dtype,
                                    void* stream) {
  const char* fn = "pa_copy_blocks";
  const int es = pa::elem_size(dtype);
  if (es == 0) return pa::fail(PA_ERR_INVALID, "%s: unknown dtype %d", fn, dtype);
  if (num_pairs < 0) return pa::fail(PA_ERR_INVALID, "%s: num_pairs < 0", fn);
  if (num_kv_heads <= 0 || head_size <= 0 || block_size <= 0 || num_blocks <= 0)
    return pa::fail(PA_ERR_INVALID, "%s: sizes must be positive", fn);
  if (!supported_head(head_size))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: head_size must be 64 or 128", fn);
  if (!supported_block(block_size))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: block_size must be 8, 16 or 32", fn);
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !block_pairs)
    return pa::fail(PA_ERR_INVALID, "%s: NULL device pointer", fn);
  if (!pa::aligned16(k_cache) || !pa::aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(block_pairs) & 7u))
    return pa::fail(PA_ERR_INVALID, "%s: caches must be 16-byte aligned, pairs 8", fn);
  unsigned int* status = pa::device_status_word();
  if (!status) return PA_ERR_CUDA;
  return launch_status(fn,
                       pa::launch_copy_blocks(k_cache, v_cache, k_cache, v_cache, block_pairs,
                                              num_pairs, num_kv_heads, head_size, block_size,
                                              num_blocks, num_blocks, es, status, stream),
                       1);
}

extern "C" pa_status pa_swap_blocks(void* dst_k_cache, void* dst_v_cache, int dst_num_blocks,
                                    const void* src_k_cache, const void* src_v_cache,
                                    int src_num_blocks, const int64_t* block_pairs, int num_pairs,
                                    int num_kv_heads, int head_size, int block_size,
                                    pa_dtype dtype, void* stream) {
  const char* fn = "pa_swap_blocks";
  const int es = pa::elem_size(dtype);
  if (es == 0) return pa::fail(PA_ERR_INVALID, "%s: unknown dtype %d", fn, dtype);
  if (num_pairs < 0) return pa::fail(PA_ERR_INVALID, "%s: num_pairs < 0", fn);
  if (num_kv_heads <= 0 || head_size <= 0 || block_size <= 0 || dst_num_blocks <= 0 ||
      src_num_blocks <= 0)
    return pa::fail(PA_ERR_INVALID, "%s: sizes must be positive", fn);
  if (!supported_head(head_size))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: head_size must be 64 or 128", fn);
  if (!supported_block(block_size))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: block_size must be 8, 16 or 32", fn);
  if (num_pairs == 0) return PA_OK;
  if (!dst_k_cache || !dst_v_cache || !src_k_cache || !src_v_cache || !block_pairs)
    return pa::fail(PA_ERR_INVALID, "%s: NULL pointer", fn);
  if (!pa::aligned16(dst_k_cache) || !pa::aligned16(dst_v_cache) || !pa::aligned16(src_k_cache) ||
      !pa::aligned16(src_v_cache) || (reinterpret_cast<uintptr_t>(block_pairs) & 7u))
    return pa::fail(PA_ERR_INVALID, "%s: caches must be 16-byte aligned, pairs 8", fn);
  unsigned int* status = pa::device_status_word();
  if (!status) return PA_ERR_CUDA;
  return launch_status(fn,
                       pa::launch_copy_blocks(dst_k_cache, dst_v_cache, src_k_cache, src_v_cache,
                                              block_pairs, num_pairs, num_kv_heads, head_size,
                                              block_size, src_num_blocks, dst_num_blocks, es,
                                              status, stream),
                       1);
}

extern "C" pa_status pa_decode_partitions_fp8(void* out, const void* q, const void* k_cache,
                                              const void* v_cache, const int32_t* block_tables,
                                              int max_blocks_per_seq, const int32_t* context_lens,
                                              int num_seqs, int num_heads, int num_kv_heads,
                                              int head_size, int block_size, int num_blocks,
                                              float scale, pa_dtype dtype, float k_scale,
                                              float v_scale, int partition_size,
                                              int max_context_len, void* workspace,
                                              size_t workspace_bytes_in, void* stream) {
  const char* fn = "pa_decode_partitions_fp8";
  pa::DecodeArgs a;
  pa_status st = check_decode_fp8(fn, out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                  context_lens, num_seqs, num_heads, num_kv_heads, head_size,
                                  block_size, num_blocks, scale, dtype, k_scale, v_scale,
                                  partition_size, max_context_len, workspace, workspace_bytes_in,
                                  &a);
  if (st != PA_OK || num_seqs == 0) return st;
  unsigned int* status = pa::device_status_word();
  if (!status) return PA_ERR_CUDA;
  return launch_status(fn, launch_partitions(a, status, stream), 1);
}

extern "C" pa_status pa_decode_fp8(void* out, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* block_tables,
                                   int max_blocks_per_seq, const int32_t* context_lens,
                                   int num_seqs, int num_heads, int num_kv_heads, int head_size,
                                   int block_size, int num_blocks, float scale, pa_dtype dtype,
                                   float k_scale, float v_scale, int partition_size,
                                   int max_context_len, void* workspace,
                                   size_t workspace_bytes_in, void* stream) {
  const char* fn = "pa_decode_fp8";
  if (partition_size == 0 && num_heads > 0 && num_kv_heads > 0)   // as pa_decode
    partition_size =
        auto_partition(num_seqs, num_heads, num_kv_heads, head_size, dtype, max_context_len);
  pa::DecodeArgs a;
  pa_status st = check_decode_fp8(fn, out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                  context_lens, num_seqs, num_heads, num_kv_heads, head_size,
                                  block_size, num_blocks, scale, dtype, k_scale, v_scale,
                                  partition_size, max_context_len, workspace, workspace_bytes_in,
                                  &a);
  if (st != PA_OK || num_seqs == 0) return st;
  unsigned int* status = pa::device_status_word();
  if (!status) return PA_ERR_CUDA;
  st = launch_status(fn, launch_partitions(a, status, stream), 1);
  if (st != PA_OK || a.num_partitions <= 1) return st;
  return launch_status(fn, pa::launch_decode_reduce(a, status, stream), 1);
}

extern "C" pa_status pa_reshape_and_cache_fp8(const void* key, const void* value, void* k_cache,
                                              void* v_cache, const int64_t* slot_mapping,
                                              int num_tokens, int num_kv_heads, int head_size,
                                              int block_size, int num_blocks, pa_dtype dtype,
                                              float k_scale, float v_scale, void* stream) {
  const char* fn = "pa_reshape_and_cache_fp8";
  if (pa::elem_size(dtype) == 0) return pa::fail(PA_ERR_INVALID, "%s: unknown dtype %d", fn, dtype);
  if (dtype == PA_FP8_E4M3)
    return pa::fail(PA_ERR_INVALID, "%s: key/value must be f32, f16 or bf16", fn);
  if (!valid_kv_scale(k_scale) || !valid_kv_scale(v_scale))
    return pa::fail(PA_ERR_INVALID, "%s: k_scale and v_scale must be finite and > 0", fn);
  if (num_tokens < 0) return pa::fail(PA_ERR_INVALID, "%s: num_tokens < 0", fn);
  if (num_kv_heads <= 0 || head_size <= 0 || block_size <= 0 || num_blocks <= 0)
    return pa::fail(PA_ERR_INVALID, "%s: sizes must be positive", fn);
  if (!supported_head(head_size))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: head_size must be 64 or 128", fn);
  if (!supported_block(block_size))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: block_size must be 8, 16 or 32", fn);
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping)
    return pa::fail(PA_ERR_INVALID, "%s: NULL device pointer", fn);
  if (!pa::aligned16(key) || !pa::aligned16(value) || !pa::aligned16(k_cache) ||
      !pa::aligned16(v_cache) || (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return pa::fail(PA_ERR_INVALID, "%s: key/value/caches must be 16-byte aligned, slots 8", fn);
  unsigned int* status = pa::device_status_word();
  if (!status) return PA_ERR_CUDA;
  return launch_status(fn,
                       pa::launch_reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping,
                                                        num_tokens, num_kv_heads, head_size,
                                                        block_size, num_blocks, dtype, k_scale,
                                                        v_scale, status, stream),
                       1);
}

// Partition length pa_decode_multi uses for partition_size = 0.  The
// query-major kernel (many query tokens; two query tiles of kMqRows rows per
// CTA) holds one CTA per SM, so the keys are
// split only as far as it takes to give at least two CTAs per SM: a prefill
// chunk of hundreds of tokens needs no split at all, and every split costs
// fp32 partials for all of its query rows.  Few queries per sequence (the
// token-major decode kernel) take pa_decode's rule with q_groups CTAs per
// sequence.  Never below the default 512, so the default's workspace size
// always suffices.
int auto_partition_multi(int num_seqs, int num_heads, int num_kv_heads, int max_query_len,
                         pa_dtype dtype, int max_context_len) {
  const int G = num_heads / num_kv_heads;
  const int P0 = pa::kDefaultPartition;
  if (max_context_len <= P0) return P0;
  if (G >= 4 && max_query_len * G <= 64) {           // token-major
    const int nq = pa::tc_query_tokens_per_cta(G, max_query_len);
    const int q_groups = (max_query_len + nq - 1) / nq;
    const int P = auto_partition(num_seqs * q_groups, num_heads, num_kv_heads, 128, dtype,
                                 max_context_len);
    return P < P0 ? P0 : P;
  }
  const int64_t qblocks = (max_query_len + pa::kMqRows / G - 1) / (pa::kMqRows / G);
  const int64_t base = static_cast<int64_t>(num_seqs) * num_kv_heads *
                       ((qblocks + pa::kMqTiles - 1) / pa::kMqTiles);   // CTAs per key range
  const int64_t want = 2ll * num_sms();
  int64_t np = base >= want ? 1 : (want + base - 1) / base;
  const int64_t np_max = (max_context_len + P0 - 1) / P0;
  if (np > np_max) np = np_max;
  int64_t P = (max_context_len + np - 1) / np;
  P = (P + 127) / 128 * 128;
  return static_cast<int>(P < P0 ? P0 : P);
}

extern "C" size_t pa_decode_multi_workspace_bytes(int total_q, int num_heads, int head_size,
                                                  int max_context_len, int partition_size) {
  const int P = resolve_partition(partition_size);
  if (P < 0 || P % 128 != 0 || total_q < 0 || num_heads < 0 || head_size < 0) return 0;
  return workspace_bytes(total_q, num_heads, head_size, num_partitions(max_context_len, P));
}

extern "C" pa_status pa_decode_multi(void* out, const void* q, const void* k_cache,
                                     const void* v_cache, const int32_t* block_tables,
                                     int max_blocks_per_seq, const int32_t* context_lens,
                                     const int32_t* query_start_loc, int num_seqs, int total_q,
                                     int max_query_len, int num_heads, int num_kv_heads,
                                     int head_size, int block_size, int num_blocks, float scale,
                                     pa_dtype dtype, int partition_size, int max_context_len,
                                     void* workspace, size_t workspace_bytes_in, void* stream) {
  const char* fn = "pa_decode_multi";
  if (partition_size == 0 && num_heads > 0 && num_kv_heads > 0 && num_heads % num_kv_heads == 0 &&
      max_query_len > 0 && num_seqs >= 0)
    partition_size = auto_partition_multi(num_seqs, num_heads, num_kv_heads, max_query_len, dtype,
                                          max_context_len);
  if (pa::elem_size(dtype) == 0) return pa::fail(PA_ERR_INVALID, "%s: unknown dtype %d", fn, dtype);
  if (dtype != PA_F16 && dtype != PA_BF16)
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: q, out and the caches must be f16 or bf16", fn);
  if (num_seqs < 0 || total_q < 0) return pa::fail(PA_ERR_INVALID, "%s: negative count", fn);
  if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0)
    return pa::fail(PA_ERR_INVALID, "%s: num_heads must be a positive multiple of num_kv_heads", fn);
  if (!supported_group(num_heads / num_kv_heads))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: query heads per kv head must be 1, 2, 4 or 8", fn);
  if (num_kv_heads > 65535) return pa::fail(PA_ERR_UNSUPPORTED, "%s: num_kv_heads > 65535", fn);
  if (head_size != 128) return pa::fail(PA_ERR_UNSUPPORTED, "%s: head_size must be 128", fn);
  if (block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0)
    return pa::fail(PA_ERR_INVALID, "%s: sizes must be positive", fn);
  if (!supported_block(block_size))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: block_size must be 8, 16 or 32", fn);
  const int P = resolve_partition(partition_size);
  if (P < 0 || P % 128 != 0)
    return pa::fail(PA_ERR_INVALID, "%s: partition_size must be 0 or a positive multiple of 128", fn);
  if (max_context_len < 0 ||
      static_cast<int64_t>(max_context_len) > static_cast<int64_t>(max_blocks_per_seq) * block_size)
    return pa::fail(PA_ERR_INVALID, "%s: max_context_len out of range", fn);
  if (total_q > 0 && (max_query_len < 1 || max_query_len > total_q || max_query_len > max_context_len))
    return pa::fail(PA_ERR_INVALID, "%s: max_query_len must be in [1, min(total_q, max_context_len)]", fn);
  if (!std::isfinite(scale)) return pa::fail(PA_ERR_INVALID, "%s: scale is not finite", fn);
  const int64_t NP = num_partitions(max_context_len, P);
  const int G = num_heads / num_kv_heads;
  const int64_t qblocks = total_q > 0 ? (max_query_len + pa::kMqRows / G - 1) / (pa::kMqRows / G) : 0;
  const int64_t qpairs = (qblocks + pa::kMqTiles - 1) / pa::kMqTiles;
  if (qpairs * NP > 65535) return pa::fail(PA_ERR_UNSUPPORTED, "%s: too many query blocks x partitions", fn);
  if (num_seqs == 0 || total_q == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start_loc)
    return pa::fail(PA_ERR_INVALID, "%s: NULL device pointer", fn);
  if (!pa::aligned16(out) || !pa::aligned16(q) || !pa::aligned16(k_cache) || !pa::aligned16(v_cache))
    return pa::fail(PA_ERR_INVALID, "%s: out, q and the caches must be 16-byte aligned", fn);
  if ((reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(context_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(query_start_loc) & 3u))
    return pa::fail(PA_ERR_INVALID, "%s: int32 arrays must be 4-byte aligned", fn);
  if (static_cast<int64_t>(num_blocks) * num_kv_heads * block_size >= (int64_t(1) << 31))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: cache larger than 2^31 rows", fn);
  const size_t need = workspace_bytes(total_q, num_heads, head_size, NP);
  if (need > 0 && (!workspace || workspace_bytes_in < need || !pa::aligned16(workspace)))
    return pa::fail(PA_ERR_INVALID, "%s: a 16-byte aligned workspace of %zu bytes is needed", fn, need);
  if (!pa::tmap_available())
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: the driver's tensor-map encoder is unavailable", fn);
  pa::MqArgs a;
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.query_start = query_start_loc;
  a.workspace = need > 0 ? static_cast<float*>(workspace) : nullptr;
  a.max_blocks = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.total_q = total_q;
  a.max_query_len = max_query_len;
  a.Hq = num_heads;
  a.Hkv = num_kv_heads;
  a.D = head_size;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.partition_size = P;
  a.num_partitions = static_cast<int>(NP);
  a.scale = scale;
  a.dtype = dtype;
  unsigned int* status = pa::device_status_word();
  if (!status) return PA_ERR_CUDA;
  // few queries per sequence: token-major (tokens as the MMA's M, query tokens x
  // heads as its N); else query-major, as a prefill kernel
  // The token-major kernel writes a sequence's outputs directly exactly when
  // its whole context fits one partition (all its query tokens form one run);
  // the query-major kernel decides per block of kMqRows / G query tokens.
  const bool token_major = pa::decode_mq_tc_supported(a);
  a.direct_qblock = token_major ? max_query_len : pa::kMqTiles * (pa::kMqRows / G);
  const int err = token_major ? pa::launch_decode_mq_tc(a, status, stream)
                              : pa::launch_decode_mq(a, status, stream);
  pa_status st = launch_status(fn, err, 1);
  if (st != PA_OK || NP <= 1) return st;
  return launch_status(fn, pa::launch_decode_mq_reduce(a, stream), 1);
}

// ---- shared-prefix groups ----

namespace {

// pa_decode_grouped runs the groups' spans on a library-owned stream of the
// device (at its highest priority) next to the rest of the sequences on the
// caller's stream: a fork
// event recorded on the caller's stream, then a join event the caller's stream
// waits on before the reduce.  Created on first use; the mutex keeps the
// record / wait / launch sequence of concurrent host threads apart (an event's
// wait binds the record before it, so reusing the two events is safe).
struct AuxStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxAuxDevices = 64;
AuxStream g_aux[kMaxAuxDevices];
std::mutex g_aux_mu;

AuxStream* aux_stream(int dev) {
  if (dev < 0 || dev >= kMaxAuxDevices) return nullptr;
  AuxStream& x = g_aux[dev];
  if (!x.stream) {
    cudaStream_t st = nullptr;
    cudaEvent_t f = nullptr, j = nullptr;
    // the highest priority of the device: the spans' CTAs (few, long) are
    // placed before the rest's (many, short), which then fill the SMs the
    // spans' last wave leaves idle instead of pushing that wave to the end
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&st, cudaStreamNonBlocking, greatest) != cudaSuccess)
      return nullptr;
    if (cudaEventCreateWithFlags(&f, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&j, cudaEventDisableTiming) != cudaSuccess) {
      if (f) cudaEventDestroy(f);
      cudaStreamDestroy(st);
      return nullptr;
    }
    x.stream = st;
    x.fork = f;
    x.join = j;
  }
  return &x;
}

int64_t grouped_span_partitions(int max_shared_len, int P) {
  return max_shared_len > 0 ? (static_cast<int64_t>(max_shared_len) + P - 1) / P : 0;
}

}  // namespace

extern "C" size_t pa_decode_grouped_workspace_bytes(int num_seqs, int num_heads, int head_size,
                                                    int max_context_len, int max_shared_len,
                                                    int partition_size) {
  const int P = resolve_partition(partition_size);
  if (P < 0 || num_seqs < 0 || num_heads < 0 || head_size < 0 || max_shared_len < 0) return 0;
  const int64_t NPg = grouped_span_partitions(max_shared_len, P);
  const int64_t NPs = num_partitions(max_context_len, P);
  if (NPg == 0) return workspace_bytes(num_seqs, num_heads, head_size, NPs);
  // with a shared span every row is reduced, even one with a single partial
  const size_t raw = static_cast<size_t>(static_cast<int64_t>(num_seqs) * num_heads * (NPg + NPs) *
                                         (head_size + 2) * 4);
  return (raw + 255) / 256 * 256;
}

namespace {

// pa_decode_grouped and pa_decode_grouped_fp8 (E4M3 caches: fp8 set, the
// cache's scales given): the same checks, groups and launches, with the plain
// decode of the cache type where nothing is shared or no kernel serves spans.
pa_status decode_grouped(const char* fn, void* out, const void* q, const void* k_cache,
                         const void* v_cache, const int32_t* block_tables, int max_blocks_per_seq,
                         const int32_t* context_lens, const int32_t* group_start,
                         const int32_t* shared_lens, int num_groups, int max_group_size,
                         int max_shared_len, int num_seqs, int num_heads, int num_kv_heads,
                         int head_size, int block_size, int num_blocks, float scale,
                         pa_dtype dtype, bool fp8, float k_scale, float v_scale,
                         int partition_size, int max_context_len, void* workspace,
                         size_t workspace_bytes_in, void* stream) {
  if (partition_size == 0 && num_heads > 0 && num_kv_heads > 0)   // as pa_decode
    partition_size =
        auto_partition(num_seqs, num_heads, num_kv_heads, head_size, dtype, max_context_len);
  auto plain = [&]() {
    return fp8 ? pa_decode_fp8(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                               context_lens, num_seqs, num_heads, num_kv_heads, head_size,
                               block_size, num_blocks, scale, dtype, k_scale, v_scale,
                               partition_size, max_context_len, workspace, workspace_bytes_in,
                               stream)
               : pa_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                           context_lens, num_seqs, num_heads, num_kv_heads, head_size, block_size,
                           num_blocks, scale, dtype, partition_size, max_context_len, workspace,
                           workspace_bytes_in, stream);
  };
  const int P = resolve_partition(partition_size);
  if (num_groups < 0 || max_shared_len < 0 || max_group_size < 0)
    return pa::fail(PA_ERR_INVALID, "%s: negative group count or size", fn);
  if (num_groups > num_seqs)
    return pa::fail(PA_ERR_INVALID, "%s: more groups (%d) than sequences (%d)", fn, num_groups,
                    num_seqs);
  if (max_shared_len > max_context_len)
    return pa::fail(PA_ERR_INVALID, "%s: max_shared_len exceeds max_context_len", fn);
  if (block_size > 0 && max_shared_len % block_size != 0)
    return pa::fail(PA_ERR_INVALID, "%s: max_shared_len must be a multiple of block_size", fn);
  if (num_groups > 0 && max_shared_len > 0 &&
      (!group_start || !shared_lens || max_group_size < 1 || max_group_size > num_seqs))
    return pa::fail(PA_ERR_INVALID, "%s: group_start / shared_lens / max_group_size missing", fn);
  const int64_t NPg = P > 0 ? grouped_span_partitions(max_shared_len, P) : 0;
  if (num_groups == 0 || NPg == 0) return plain();   // nothing shared
  // the checks of the plain decode, with the workspace sized for the grouped layout
  pa::DecodeArgs a;
  const size_t need = pa_decode_grouped_workspace_bytes(num_seqs, num_heads, head_size,
                                                        max_context_len, max_shared_len, P);
  pa_status st =
      fp8 ? check_decode_fp8(fn, out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                             context_lens, num_seqs, num_heads, num_kv_heads, head_size,
                             block_size, num_blocks, scale, dtype, k_scale, v_scale,
                             partition_size, max_context_len, workspace, workspace_bytes_in, &a)
          : check_decode_full(fn, out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                              context_lens, num_seqs, num_heads, num_kv_heads, head_size,
                              block_size, num_blocks, scale, dtype, partition_size,
                              max_context_len, workspace, workspace_bytes_in, &a);
  if (st != PA_OK) return st;
  if (!workspace || workspace_bytes_in < need || !pa::aligned16(workspace))
    return pa::fail(PA_ERR_INVALID, "%s: a 16-byte aligned workspace of %zu bytes is needed", fn,
                    need);
  const int64_t NP = NPg + a.num_partitions;
  if (NP > 65535) return pa::fail(PA_ERR_UNSUPPORTED, "%s: more than 65535 partitions", fn);
  if ((reinterpret_cast<uintptr_t>(group_start) & 3u) || (reinterpret_cast<uintptr_t>(shared_lens) & 3u))
    return pa::fail(PA_ERR_INVALID, "%s: group_start / shared_lens must be 4-byte aligned", fn);
  a.workspace = static_cast<float*>(workspace);
  if (!(fp8 ? pa::decode_group_tc8_supported(a) : pa::decode_group_tc_supported(a)))
    return plain();   // same result without the sharing
  const int G = num_heads / num_kv_heads;
  const int64_t member_runs = (max_group_size + (16 / G) - 1) / (16 / G);
  if (static_cast<int64_t>(num_groups) * member_runs + num_seqs > 0x7fffffff)
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: too many groups", fn);
  unsigned int* status = pa::device_status_word();
  if (!status) return PA_ERR_CUDA;
  a.num_partitions = static_cast<int>(NP);
  a.slot_base = static_cast<int>(NPg);
  a.seq_shift = shared_lens;
  a.group_start = group_start;
  a.num_groups = num_groups;
  a.max_group_size = max_group_size;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return pa::fail(PA_ERR_CUDA, "%s: cudaGetDevice", fn);
  cudaStream_t st_main = static_cast<cudaStream_t>(stream);
  {
    std::lock_guard<std::mutex> lk(g_aux_mu);
    AuxStream* aux = aux_stream(dev);
    if (aux == nullptr)   // no second stream: the spans first, then the rest
      return pa::fail(PA_ERR_CUDA, "%s: could not create the library's auxiliary stream", fn);
    // fork: the spans on the auxiliary stream, the rest on the caller's
    if (cudaEventRecord(aux->fork, st_main) != cudaSuccess ||
        cudaStreamWaitEvent(aux->stream, aux->fork, 0) != cudaSuccess)
      return pa::fail(PA_ERR_CUDA, "%s: fork to the auxiliary stream failed", fn);
    st = launch_status(fn,
                       fp8 ? pa::launch_decode_group_tc8(a, status, aux->stream)
                           : pa::launch_decode_group_tc(a, status, aux->stream),
                       1);
    const pa_status st_rest = launch_status(fn, launch_partitions(a, status, stream), 1);
    // join, whatever happened, so that the caller's stream never runs ahead
    // of work left on the auxiliary one
    const bool joined = cudaEventRecord(aux->join, aux->stream) == cudaSuccess &&
                        cudaStreamWaitEvent(st_main, aux->join, 0) == cudaSuccess;
    if (st != PA_OK) return st;
    if (st_rest != PA_OK) return st_rest;
    if (!joined) return pa::fail(PA_ERR_CUDA, "%s: join with the auxiliary stream failed", fn);
  }
  return launch_status(fn, pa::launch_decode_reduce(a, status, stream), 1);
}

}  // namespace

extern "C" pa_status pa_decode_grouped(void* out, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* block_tables,
                                       int max_blocks_per_seq, const int32_t* context_lens,
                                       const int32_t* group_start, const int32_t* shared_lens,
                                       int num_groups, int max_group_size, int max_shared_len,
                                       int num_seqs, int num_heads, int num_kv_heads,
                                       int head_size, int block_size, int num_blocks,
                                       float scale, pa_dtype dtype, int partition_size,
                                       int max_context_len, void* workspace,
                                       size_t workspace_bytes_in, void* stream) {
  return decode_grouped("pa_decode_grouped", out, q, k_cache, v_cache, block_tables,
                        max_blocks_per_seq, context_lens, group_start, shared_lens, num_groups,
                        max_group_size, max_shared_len, num_seqs, num_heads, num_kv_heads,
                        head_size, block_size, num_blocks, scale, dtype, false, 1.f, 1.f,
                        partition_size, max_context_len, workspace, workspace_bytes_in, stream);
}

extern "C" pa_status pa_decode_grouped_fp8(void* out, const void* q, const void* k_cache,
                                           const void* v_cache, const int32_t* block_tables,
                                           int max_blocks_per_seq, const int32_t* context_lens,
                                           const int32_t* group_start, const int32_t* shared_lens,
                                           int num_groups, int max_group_size,
                                           int max_shared_len, int num_seqs, int num_heads,
                                           int num_kv_heads, int head_size, int block_size,
                                           int num_blocks, float scale, pa_dtype dtype,
                                           float k_scale, float v_scale, int partition_size,
                                           int max_context_len, void* workspace,
                                           size_t workspace_bytes_in, void* stream) {
  return decode_grouped("pa_decode_grouped_fp8", out, q, k_cache, v_cache, block_tables,
                        max_blocks_per_seq, context_lens, group_start, shared_lens, num_groups,
                        max_group_size, max_shared_len, num_seqs, num_heads, num_kv_heads,
                        head_size, block_size, num_blocks, scale, dtype, true, k_scale, v_scale,
                        partition_size, max_context_len, workspace, workspace_bytes_in, stream);
}

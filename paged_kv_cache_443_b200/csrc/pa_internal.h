// pa_internal.h -- declarations shared by the library's translation units
// (host side only; nothing here is part of the public ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <utility>

#include <cuda_runtime.h>

#include "pagedkv.h"

namespace pa {

// Records a message for pa_last_error() and returns `st`.
pa_status fail(pa_status st, const char* fmt, ...)
#if defined(__GNUC__)
    __attribute__((format(printf, 2, 3)))
#endif
    ;

// Counts successful kernel launches (pa_launch_count).
void count_launch(uint64_t n = 1);

// Device address of the current device's status word (cached per device).
// Returns nullptr (and records a message) if CUDA fails.
unsigned int* device_status_word();

// Element size of a dtype, 0 if invalid.
inline int elem_size(pa_dtype dt) {
  switch (dt) {
    case PA_F32: return 4;
    case PA_F16: return 2;
    case PA_BF16: return 2;
    case PA_FP8_E4M3: return 1;
    default: return 0;
  }
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kDefaultPartition = 512;  // tokens per split-K partition
constexpr int kStageTokens = 32;        // tokens per pipeline stage of the decode kernel

// ---- decode launch description (validated on the host) ----
struct DecodeArgs {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* workspace;  // may be null when num_partitions == 1
  int64_t max_blocks;
  int num_seqs, Hq, Hkv, D, block_size, num_blocks;
  int partition_size, num_partitions;
  float scale;
  pa_dtype dtype;      // q and out (and the caches unless kv_dtype says otherwise)
  pa_dtype kv_dtype;   // the caches: dtype, or PA_FP8_E4M3
  float k_scale = 1.f, v_scale = 1.f;  // per-cache scales of E4M3 codes
  // Shared-prefix groups (pa_decode_grouped).  num_partitions is then the
  // workspace's slots per (sequence, head): the groups' span partitions first,
  // then the rest of each sequence's from slot_base.  seq_shift[b] (device,
  // nullable) is the number of leading tokens of sequence b its group serves.
  const int32_t* seq_shift = nullptr;
  int slot_base = 0;          // first slot of the partition launch (and rest of the reduce)
  // the group launch: members group_start[i] .. group_start[i+1]-1 (device)
  const int32_t* group_start = nullptr;
  int num_groups = 0, max_group_size = 0;
};

// Kernel launchers (kernels.cu).  They return cudaError_t as int.
int launch_decode_partitions(const DecodeArgs& a, unsigned int* status, void* stream);
int launch_decode_reduce(const DecodeArgs& a, unsigned int* status, void* stream);
// Tensor-core partition kernel (decode_tc.cu): fp16/bf16, head size 128, 4 or 8
// query heads per kv head, partition length a multiple of 128.
bool decode_tc_supported(const DecodeArgs& a);
int launch_decode_partitions_tc(const DecodeArgs& a, unsigned int* status, void* stream);
// Consecutive partitions one CTA of a tensor-core decode kernel streams (1, 2,
// 4 or 8) when ctas_without CTAs would each serve one partition of n_parts.
int tc_parts_per_cta(const DecodeArgs& a);
// rows: CTAs per partition index (sequences x kv heads); other_ctas: CTAs of
// other work in the same grid.
int tc_parts_per_cta(int64_t rows, int partition_size, int n_parts, int64_t other_ctas);
// pa_decode_grouped's partition phase on the tcgen05 kernel in one launch (f16
// / bf16, head size 128, G in {1, 2, 4, 8}): the groups' shared spans
// (partials into slots [0, a.slot_base) of every member's row) and the rest of
// every sequence (slots from a.slot_base).
bool decode_group_tc_supported(const DecodeArgs& a);
int launch_decode_group_tc(const DecodeArgs& a, unsigned int* status, void* stream);
// Tensor-core partition kernel over an E4M3 cache (decode_tc8.cu): f16/bf16
// queries, head size 128, 4 or 8 query heads per kv head, partition length a
// multiple of 128.
bool decode_tc8_supported(const DecodeArgs& a);  // needs tmap_available()
int launch_decode_partitions_tc8(const DecodeArgs& a, unsigned int* status, void* stream);
// The groups' shared spans over an E4M3 cache (pa_decode_grouped_fp8), G = 1, 2, 4, 8.
bool decode_group_tc8_supported(const DecodeArgs& a);  // needs tmap_available()
int launch_decode_group_tc8(const DecodeArgs& a, unsigned int* status, void* stream);
// A TMA tensor map of 16-bit elements (bytes for PA_FP8_E4M3) with the 128-byte swizzle: `rank` dims
// (innermost first), byte strides of dims 1..rank-1, a box; `map` points at a
// CUtensorMap.  False if encoding fails.
bool make_tmap(void* map, const void* base, int rank, const int64_t* dims,
               const int64_t* strides_bytes, const int* box, pa_dtype dt);
// Whether the driver entry point that encodes tensor maps could be found.
bool tmap_available();

// ---- several query tokens per sequence (decode_mq.cu) ----
struct MqArgs {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start;
  float* workspace;  // may be null when num_partitions == 1
  int64_t max_blocks;
  int num_seqs, total_q, max_query_len, Hq, Hkv, D, block_size, num_blocks;
  int partition_size, num_partitions;
  float scale;
  pa_dtype dtype;
  // Set by the partition launcher for the reduce: the partition kernel groups a
  // sequence's query tokens in runs of this many (from the first) and writes a
  // run's outputs directly, with no partials, when its last query token's last
  // key lies in the first partition.
  int direct_qblock = 0;
};
constexpr int kMqRows = 128;  // (query token, head) rows per query tile of the multi-query kernel
constexpr int kMqTiles = 2;   // query tiles per CTA of the multi-query kernel
int launch_decode_mq(const MqArgs& a, unsigned int* status, void* stream);
// Few query tokens per sequence (max_query_len * G <= 64, G = 4 or 8): the
// token-major tcgen05 decode kernel with per-column causal limits, 16 / G query
// tokens per CTA (decode_tc.cu).
bool decode_mq_tc_supported(const MqArgs& a);
// Query tokens one CTA of the token-major kernel serves for G query heads per kv
// head: 2 (G * 2 <= 16 columns), 4 at G = 4 (16 columns), else 32 / G (the
// N = 32 variant: 4 at G = 8, 8 at G = 4).
inline int tc_query_tokens_per_cta(int G, int max_query_len) {
  if (max_query_len <= 2) return 2;
  if (G == 4 && max_query_len <= 4) return 4;
  return 32 / G;
}
int launch_decode_mq_tc(const MqArgs& a, unsigned int* status, void* stream);
int launch_decode_mq_reduce(const MqArgs& a, void* stream);

int launch_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                             const int64_t* slot_mapping, int num_tokens, int Hkv, int D,
                             int block_size, int num_blocks, int esize, unsigned int* status,
                             void* stream);
// Append into an E4M3 cache; key/value of `dtype` (f32 / f16 / bf16).
int launch_reshape_and_cache_fp8(const void* key, const void* value, void* k_cache,
                                 void* v_cache, const int64_t* slot_mapping, int num_tokens,
                                 int Hkv, int D, int block_size, int num_blocks, pa_dtype dtype,
                                 float k_scale, float v_scale, unsigned int* status, void* stream);
int launch_copy_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                       const int64_t* pairs, int num_pairs, int Hkv, int D, int block_size,
                       int src_blocks, int dst_blocks, int esize, unsigned int* status,
                       void* stream);

// Launches `kernel` on `stream` allowing it to overlap the tail of the previous
// kernel on the stream (programmatic stream serialisation); the kernel must
// call grid_dependency_wait() before it reads anything an earlier launch wrote.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_overlapped(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                     cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace pa

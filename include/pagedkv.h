/*
 * pagedkv.h -- C ABI of libpagedkv.so: the decode hot path of PagedAttention
 * (attention over a KV cache kept in fixed-size physical blocks) for NVIDIA
 * B200 (sm_100a), plus the host-side block manager that produces its block
 * tables.
 *
 * Sources (three web pages on vLLM / PagedAttention):
 *   [P1] supersilo.blog, "vLLM" summary of the PagedAttention paper:
 *        "자기회귀 생성과 KV 캐시" (attention scores q.k_j / sqrt(d_k),
 *        softmax over valid past positions, weighted sum of V);
 *        "PagedAttention의 설계" (fixed-size blocks, block table from logical to
 *        physical blocks, kernel gathers K/V through the table in logical
 *        order with one softmax over all valid tokens, unused slots in the last
 *        block, block manager allocating and reclaiming blocks);
 *        "블록 공유" (parallel samples / beams share prompt blocks, copy when
 *        modified).
 *   [P2] blog.aqudi.me, "3. vLLM: KV cache를 블록 단위로 관리하기" (a new block
 *        when the current one fills; copy-on-write of shared prompt blocks).
 *   [P3] hjr-study-book Day 3, "1. KV 캐시란" (each decode step stores the new
 *        token's K and V), "4.2 PagedAttention의 접근" (block-table example) and
 *        "5. Prefix Caching" (the KV blocks of a repeated prompt prefix are
 *        reused across requests).
 *
 * Conventions for every call below:
 *   - Shapes use B = num_seqs, Hq = num_heads (query heads), Hkv = num_kv_heads,
 *     D = head_size, bs = block_size, NB = num_blocks.  All arrays are dense,
 *     row-major (C order), with the element type given by `dtype`.
 *   - KV cache layout: k_cache and v_cache are each [NB][Hkv][bs][D]; token j of
 *     a sequence b lives in physical block block_tables[b][j / bs] at slot
 *     offset j % bs.  A slot index is physical_block * bs + offset.
 *   - Grouped-query attention: query head h reads kv head h / (Hq / Hkv).
 *   - Device pointers are owned by the caller; the library allocates no device
 *     memory on any of these paths (scratch space is passed in).  Device calls
 *     are asynchronous on `stream` (a cudaStream_t passed as void*, NULL = the
 *     legacy default stream) on the current CUDA device, and never synchronise
 *     the host.
 *   - Every shape, dtype, alignment and size check runs on the host before any
 *     launch; a failed check returns PA_ERR_INVALID (or PA_ERR_UNSUPPORTED for a
 *     shape the kernels do not implement) with no side effect, and
 *     pa_last_error() describes it.  A failed launch returns PA_ERR_CUDA.
 *   - Checks that need device data (block ids in block_tables, context lengths,
 *     slots, copy pairs) run inside the kernels: an out-of-range value is never
 *     dereferenced; the kernel skips that access and sets a bit in a per-device
 *     status word read by pa_device_status().  The output of that call is then
 *     unspecified.  No kernel traps or asserts.
 *   - Supported: dtype f32 / f16 / bf16; D in {64, 128}; bs in {8, 16, 32};
 *     Hq / Hkv in {1, 2, 4, 8}.
 */
#ifndef PAGEDKV_H_
#define PAGEDKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = 1,     /* bad argument; nothing was done */
  PA_ERR_OOM = 2,         /* block manager: not enough free blocks; nothing was done */
  PA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  PA_ERR_UNSUPPORTED = 4  /* valid request outside the implemented shapes */
} pa_status;

/*
 * Element types.  PA_FP8_E4M3 is a cache storage type only: one byte per
 * element, an OCP E4M3 code (1 sign, 4 exponent bits with bias 7, 3 fraction
 * bits, largest finite 448) standing for code * scale with one scale per cache
 * ([P2] "4. 이 밖의 기법들": quantization lowers the KV cache's precision to save
 * memory and bandwidth; the format and per-cache scale are this library's
 * reading).  It is accepted by pa_copy_blocks, pa_swap_blocks and
 * pa_reshape_and_cache (codes moved as bytes) and as the cache type of the
 * *_fp8 calls; as a query / output type it is PA_ERR_UNSUPPORTED.
 */
typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2, PA_FP8_E4M3 = 3 } pa_dtype;

/* Bits of the per-device status word (see pa_device_status). */
#define PA_DEVERR_TABLE 0x1u    /* a block-table entry outside [0, NB) was met */
#define PA_DEVERR_CONTEXT 0x2u  /* a context length < 0, beyond the table, or beyond max_context_len */
#define PA_DEVERR_SLOT 0x4u     /* a slot_mapping entry >= NB * bs */
#define PA_DEVERR_PAIR 0x8u     /* a copy pair with an id outside [0, NB) */
#define PA_DEVERR_TIMEOUT 0x10u /* an internal pipeline wait gave up (about one second) */

/* Message for the last non-OK status returned on this host thread. */
const char* pa_last_error(void);

/* Library version string. */
const char* pa_version(void);

/* Number of kernels this library has launched in this process (all devices). */
uint64_t pa_launch_count(void);

/*
 * Reads the status word of the current device into *flags_out (PA_DEVERR_*
 * bits; 0 = no device-side problem seen) and clears it if `clear` is non-zero.
 * Synchronises the current device.
 */
pa_status pa_device_status(unsigned int* flags_out, int clear);

/*
 * Checks the kernels' bounded-wait mechanism (no counterpart on the pages: a
 * robustness test).  Launches one CTA on the current device that waits, with a
 * 20 ms limit, on a shared-memory barrier that nothing will complete; the wait
 * gives up and sets PA_DEVERR_TIMEOUT.  On return *flags_out holds the status
 * word that launch produced (PA_DEVERR_TIMEOUT expected) and the device is
 * usable as before; bits already pending are kept for pa_device_status.
 * Synchronises the current device.
 */
pa_status pa_selftest_wait_timeout(unsigned int* flags_out);

/* ------------------------------------------------------------------------ */
/* Decode attention ([P1] "자기회귀 생성과 KV 캐시", "PagedAttention의 설계")  */

/*
 * The split-K partition length used when partition_size = 0 is passed
 * (tokens; a multiple of 32).
 */
int pa_decode_default_partition_size(void);

/*
 * The partition length pa_decode uses when it is given partition_size = 0
 * (tokens; 512, 1024, 2048 or 4096): the longest P that still gives
 * num_seqs * num_kv_heads * ceil(max_context_len / P) >= 8 * (number of SMs)
 * CTAs, among 4096 / 2048 / 1024 with 4 or 8 query heads per kv head in
 * fp16/bf16 and head size 128 (the tensor-core kernel), among 1024 otherwise;
 * the default (512) when none does.  Pass it explicitly to
 * pa_decode_partitions / pa_decode_reduce to reproduce pa_decode's automatic
 * choice.  Returns -1 for invalid arguments.
 */
int pa_decode_auto_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_size,
                                  pa_dtype dtype, int max_context_len);

/*
 * The partition length pa_decode_fp8 uses when it is given partition_size = 0:
 * the rule of pa_decode_auto_partition_size, with dtype the queries' type (f32,
 * f16 or bf16).  Returns -1 for invalid arguments (PA_FP8_E4M3 as dtype
 * included).
 */
int pa_decode_fp8_auto_partition_size(int num_seqs, int num_heads, int num_kv_heads,
                                      int head_size, pa_dtype dtype, int max_context_len);

/*
 * Number of split-K partitions per sequence for a batch whose longest context
 * is max_context_len: ceil(max_context_len / P), P = the partition size (0 =
 * default).  Returns -1 for an invalid partition size.
 */
int pa_decode_num_partitions(int max_context_len, int partition_size);

/*
 * Bytes of scratch `workspace` pa_decode needs: 0 when every sequence fits one
 * partition, else B * Hq * num_partitions * (D + 2) * 4 rounded up to 256 (the
 * split-K partials).
 */
size_t pa_decode_workspace_bytes(int num_seqs, int num_heads, int head_size, int max_context_len,
                                 int partition_size);

/*
 * Single-query attention for every sequence b < B and query head h < Hq:
 *
 *   out[b][h][:] = sum_j w_j V_b[j][:],  w = softmax_j(scale * q[b][h] . K_b[j]),
 *
 * over the valid positions j < context_lens[b] only, where K_b[j] / V_b[j] is
 * row j % bs of kv head h / G in physical block block_tables[b][j / bs] of
 * k_cache / v_cache.  The softmax is normalised jointly over all of a
 * sequence's tokens (a running max and sum carried across blocks and
 * partitions), never as per-block softmaxes added up; unused slots of the last
 * block are never read into the result, whatever they hold.  The plain reading
 * of [P1] gives scale = 1 / sqrt(D).
 *
 *   out           [B][Hq][D] dtype, written (16-byte aligned)
 *   q             [B][Hq][D] dtype (16-byte aligned)
 *   k_cache, v_cache  [NB][Hkv][bs][D] dtype (16-byte aligned)
 *   block_tables  [B][max_blocks_per_seq] int32; entries past a sequence's
 *                 last block are never read (any value, e.g. -1)
 *   context_lens  [B] int32, each in [0, max_context_len] and
 *                 <= max_blocks_per_seq * bs; a length of 0 gives a zero row
 *   partition_size  0 = automatic (pa_decode_auto_partition_size), else a
 *                 multiple of 32 tokens: contexts longer than this are split
 *                 into partitions reduced by a second kernel
 *   max_context_len  an upper bound of context_lens (sizes the launch grid and
 *                 the workspace)
 *   workspace     device scratch of at least pa_decode_workspace_bytes(...)
 *                 bytes, 16-byte aligned; may be NULL when that is 0.  Its
 *                 contents need no initialisation and are clobbered; calls
 *                 that share a workspace must not overlap on the GPU.
 *
 * pa_decode_workspace_bytes(..., partition_size = 0, ...) bytes always suffice
 * for the automatic length.
 *
 * Precision: products and sums in fp32; the result is rounded to dtype once.
 * With 4 or 8 query heads per kv head in fp16/bf16 (head size 128, partition a
 * multiple of 128) the products run on the tensor cores, whose operands share
 * one type: the probabilities are rounded to dtype before they weight V.
 * Exactly pa_decode_partitions followed (when the workspace size is not 0) by
 * pa_decode_reduce on the same stream, with the same partition length (for
 * partition_size = 0: pa_decode_auto_partition_size(...), passed to both).
 */
pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int max_blocks_per_seq,
                    const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                    int head_size, int block_size, int num_blocks, float scale, pa_dtype dtype,
                    int partition_size, int max_context_len, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * First phase of pa_decode (same arguments; partition_size = 0 means the
 * default 512 here): one CTA per (sequence, kv head, partition).  Sequences that fit one partition get their final `out` rows;
 * the others leave per-partition (max, sum, unnormalised output) partials in
 * the workspace.  A kernel that covers several consecutive partitions with
 * one softmax (the tensor-core kernels do, for partitions shorter than 2048
 * tokens) writes the merged partial to the first partition's slot and empty
 * partials (max -inf, sum 0, output 0) to the others; pa_decode_reduce gives
 * them weight 0, so the result is the same joint softmax.
 */
pa_status pa_decode_partitions(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* context_lens, int num_seqs, int num_heads,
                               int num_kv_heads, int head_size, int block_size, int num_blocks,
                               float scale, pa_dtype dtype, int partition_size,
                               int max_context_len, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * Second phase of pa_decode: merges the partials of every multi-partition
 * sequence into `out` with one global max and normaliser ([P1] "PagedAttention의
 * 설계": one softmax over all valid tokens).  A no-op returning PA_OK when the
 * workspace size for these arguments is 0.
 */
pa_status pa_decode_reduce(void* out, const int32_t* context_lens, int num_seqs, int num_heads,
                           int head_size, pa_dtype dtype, int partition_size, int max_context_len,
                           const void* workspace, size_t workspace_bytes, void* stream);

/*
 * pa_decode for callers that cannot allocate device memory.  The pages have no
 * counterpart: this is an interface convenience, not part of the method.
 *
 * Same arguments and result as pa_decode, without the workspace: the split-K
 * scratch comes from a fixed 32 MiB array compiled into the library, which
 * every GPU that loads the library holds until the process exits.  No call
 * allocates (no cudaMalloc / cudaFree or allocating library routine).  Meant
 * for callers whose device memory is all committed to a KV-cache pool, plain C
 * hosts without a device allocator, and loops that cannot take cudaMalloc's
 * implicit device synchronisation.
 *
 *   - A batch whose pa_decode_workspace_bytes(...) exceeds 32 MiB is rejected
 *     with PA_ERR_UNSUPPORTED (and a message) before any launch.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is looked up again when the
 *     device's current context is a different one (after cudaDeviceReset the
 *     library's device code is loaded anew); make the first call after such a
 *     reset before any capture as well.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents.  Nothing in it needs to start at zero (each call writes every
 *     partial it reads), but calls that overlap on the GPU -- on different
 *     streams, or from different host threads -- race on it and give wrong
 *     results; order them on one stream.
 */
pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, int max_blocks_per_seq,
                            const int32_t* context_lens, int num_seqs, int num_heads,
                            int num_kv_heads, int head_size, int block_size, int num_blocks,
                            float scale, pa_dtype dtype, int partition_size, int max_context_len,
                            void* stream);

/*
 * Decode of sequences that share leading blocks ([P1] "블록 공유": parallel
 * samples of one prompt, or requests with a common prefix, point at the same
 * physical blocks).  The result is that of pa_decode on the same arguments;
 * what changes is the work: the shared span of a group is read once for all
 * its members, whose queries form the columns of one tensor-core tile (each
 * column a (member, query head) pair: 16 / G members per CTA, or 8 / G when
 * every group has at most that many), instead of once
 * per member.  Each member's remaining tokens are decoded as in pa_decode, and
 * a reduce merges both parts with one softmax over all of the sequence's
 * tokens ([P1] "PagedAttention의 설계").
 *
 *   group_start   [num_groups + 1] int32 (device): group i is sequences
 *                 group_start[i] .. group_start[i+1]-1 (consecutive in the
 *                 batch); 0 = group_start[0] <= ... <= group_start[num_groups]
 *                 = num_seqs
 *   shared_lens   [num_seqs] int32 (device): for each sequence, the tokens at
 *                 its start that all members of its group share: a multiple of
 *                 block_size, at most every member's context length, equal for
 *                 all members of a group, and the table entries of those
 *                 blocks the same physical blocks for all members (0: nothing
 *                 shared)
 *   max_group_size, max_shared_len  upper bounds of the group sizes and of
 *                 shared_lens (size the grid and the workspace)
 *   workspace     pa_decode_grouped_workspace_bytes(...) bytes, 16-byte aligned
 * Other arguments as pa_decode (partition_size 0 = its automatic length).
 * pa_build_groups computes the groups from host block tables.  Device-side
 * checks: inconsistent groups (offsets out of order, members whose shared_lens
 * differ or exceed their context, a length not a multiple of block_size) set
 * PA_DEVERR_CONTEXT.  With max_shared_len = 0 or num_groups = 0 this is
 * pa_decode; so it is for f32 / head size 64, where no tensor-core kernel
 * serves the shared span.  Three launches: the groups' spans run on a stream
 * the library creates per device on first use (with two events), forked from
 * and joined back to `stream`, next to the rest of every sequence on `stream`;
 * then the reduce on `stream`.  Everything stays ordered on `stream` for the
 * caller (and inside a stream capture).  Calls from several host threads are
 * serialised around that fork and join.
 */
size_t pa_decode_grouped_workspace_bytes(int num_seqs, int num_heads, int head_size,
                                         int max_context_len, int max_shared_len,
                                         int partition_size);
pa_status pa_decode_grouped(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, int max_blocks_per_seq,
                            const int32_t* context_lens, const int32_t* group_start,
                            const int32_t* shared_lens, int num_groups, int max_group_size,
                            int max_shared_len, int num_seqs, int num_heads, int num_kv_heads,
                            int head_size, int block_size, int num_blocks, float scale,
                            pa_dtype dtype, int partition_size, int max_context_len,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * pa_decode_grouped over an E4M3 cache: q and out of type `dtype` (f16 or
 * bf16 for the shared spans' tensor-core kernel), cache elements standing for
 * code * k_scale (keys) and code * v_scale (values), as pa_decode_fp8.  The
 * result is that of pa_decode_fp8 on the same arguments; group arguments,
 * workspace, launches and device-side checks are those of pa_decode_grouped.
 * With nothing shared, f32 queries or head size 64 this is pa_decode_fp8.
 */
pa_status pa_decode_grouped_fp8(void* out, const void* q, const void* k_cache,
                                const void* v_cache, const int32_t* block_tables,
                                int max_blocks_per_seq, const int32_t* context_lens,
                                const int32_t* group_start, const int32_t* shared_lens,
                                int num_groups, int max_group_size, int max_shared_len,
                                int num_seqs, int num_heads, int num_kv_heads, int head_size,
                                int block_size, int num_blocks, float scale, pa_dtype dtype,
                                float k_scale, float v_scale, int partition_size,
                                int max_context_len, void* workspace, size_t workspace_bytes,
                                void* stream);

/* ------------------------------------------------------------------------ */
/* Cache updates                                                           */

/*
 * Append ([P3] "1. KV 캐시란": each decode step stores the new token's K and
 * V): for every t < num_tokens with s = slot_mapping[t] >= 0,
 *   k_cache[s / bs][h][s % bs][:] = key[t][h][:]  and the same for value, all h.
 * A negative slot is skipped (padding).  Bytes are copied exactly.
 *
 *   key, value    [num_tokens][Hkv][D] dtype (16-byte aligned)
 *   k_cache, v_cache  [NB][Hkv][bs][D] dtype (16-byte aligned), updated in place
 *   slot_mapping  [num_tokens] int64 (device)
 * Two tokens given the same slot race (one of them wins).
 */
pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                               const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                               int head_size, int block_size, int num_blocks, pa_dtype dtype,
                               void* stream);

/*
 * Copy-on-write ([P1] "블록 공유", [P2] copy-on-write bullet): for each pair p,
 * physical block block_pairs[p][1] of both caches becomes a byte copy of block
 * block_pairs[p][0] (all kv heads, all slots).
 *
 *   block_pairs  [num_pairs][2] int64 (device): (src, dst)
 * The destinations must be distinct and must not appear as a source of the
 * same call (true of the pairs the block manager emits); otherwise the result
 * is unspecified.
 */
pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_pairs, int num_pairs,
                         int num_kv_heads, int head_size, int block_size, int num_blocks,
                         pa_dtype dtype, void* stream);

/*
 * Several new query tokens per sequence: chunked prefill and speculative
 * verification ([P2] "4. 이 밖의 기법들": a long prefill is cut into chunks run
 * between decode steps; several proposed tokens are checked at once).  The
 * attention is that of pa_decode ([P1] "자기회귀 생성과 KV 캐시"), with this
 * library's reading of the position of each query: sequence b's query tokens
 * are rows query_start_loc[b] .. query_start_loc[b+1]-1 of q, they are the
 * LAST Q_b = query_start_loc[b+1] - query_start_loc[b] of its context_lens[b]
 * tokens (their K/V already appended), and query token i attends to positions
 * 0 .. context_lens[b] - Q_b + i (causal among the new tokens):
 *
 *   out[t][h] = sum_{j <= pos(t)} softmax_j(scale * q[t][h] . K_b[j]) V_b[j].
 *
 *   q, out          [total_q][Hq][D], dtype f16 or bf16
 *   query_start_loc [num_seqs + 1] int32 (device): 0, then non-decreasing,
 *                   ending at total_q; max_query_len >= every Q_b
 *   k_cache, v_cache, block_tables, context_lens, max_context_len: as pa_decode
 * Supported: f16/bf16, head_size 128, Hq/Hkv in {1, 2, 4, 8}, bs in {8, 16,
 * 32}, partition_size a multiple of 128, or 0 for an automatic length of at
 * least 512: with many query tokens (a prefill chunk) the keys are split only
 * as far as needed for two CTAs per SM, with few (verification) pa_decode's
 * rule applies.  The workspace holds the split-K partials when
 * max_context_len exceeds the partition length (pa_decode_multi_workspace_bytes;
 * with partition_size 0 it returns the size for 512, which suffices for the
 * automatic length).  Offsets that are not non-decreasing, or
 * Q_b > context_lens[b], set PA_DEVERR_CONTEXT and the sequence is skipped.
 * One or two launches on `stream`.
 */
size_t pa_decode_multi_workspace_bytes(int total_q, int num_heads, int head_size,
                                       int max_context_len, int partition_size);
pa_status pa_decode_multi(void* out, const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, int max_blocks_per_seq,
                          const int32_t* context_lens, const int32_t* query_start_loc,
                          int num_seqs, int total_q, int max_query_len, int num_heads,
                          int num_kv_heads, int head_size, int block_size, int num_blocks,
                          float scale, pa_dtype dtype, int partition_size, int max_context_len,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * E4M3 KV cache ([P2] "4. 이 밖의 기법들", quantization; format and scales as
 * described at pa_dtype).
 *
 * pa_reshape_and_cache_fp8: as pa_reshape_and_cache, but key/value are f32 /
 * f16 / bf16 (`dtype`) and the caches hold E4M3 codes:
 *   k_cache[s / bs][h][s % bs][d] = E4M3(fp32(key[t][h][d]) / k_scale)
 * (the quotient rounded once in fp32, then to the nearest E4M3 value with ties
 * to an even fraction, magnitudes above 448 saturating to 448); value alike
 * with v_scale.  Scales must be finite and > 0.
 *
 * pa_decode_fp8 / pa_decode_partitions_fp8: as pa_decode / pa_decode_partitions
 * with q and out of type `dtype` (f32 / f16 / bf16) and caches of E4M3 codes,
 * each standing for code * k_scale (keys) or code * v_scale (values).  The
 * workspace and pa_decode_reduce (with `dtype`) are the same as for pa_decode;
 * partition_size 0 means the default length.
 */
pa_status pa_reshape_and_cache_fp8(const void* key, const void* value, void* k_cache,
                                   void* v_cache, const int64_t* slot_mapping, int num_tokens,
                                   int num_kv_heads, int head_size, int block_size,
                                   int num_blocks, pa_dtype dtype, float k_scale, float v_scale,
                                   void* stream);

pa_status pa_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* block_tables, int max_blocks_per_seq,
                        const int32_t* context_lens, int num_seqs, int num_heads,
                        int num_kv_heads, int head_size, int block_size, int num_blocks,
                        float scale, pa_dtype dtype, float k_scale, float v_scale,
                        int partition_size, int max_context_len, void* workspace,
                        size_t workspace_bytes, void* stream);

pa_status pa_decode_partitions_fp8(void* out, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* block_tables,
                                   int max_blocks_per_seq, const int32_t* context_lens,
                                   int num_seqs, int num_heads, int num_kv_heads, int head_size,
                                   int block_size, int num_blocks, float scale, pa_dtype dtype,
                                   float k_scale, float v_scale, int partition_size,
                                   int max_context_len, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * Swap ([P1] "적용 범위와 관련 연구": when GPU memory runs short a sequence's KV
 * blocks move to CPU memory and come back later): for each pair p, physical
 * block block_pairs[p][1] of the destination caches becomes a byte copy of
 * block block_pairs[p][0] of the source caches (all kv heads, all slots).
 * One cache pair is device memory, the other may be device memory or pinned
 * host memory the GPU can address (cudaHostAlloc / cudaHostRegister with
 * unified addressing); the copy runs as a kernel on `stream`, so one call moves
 * any number of scattered blocks.
 *
 *   dst_k_cache, dst_v_cache  [dst_num_blocks][Hkv][bs][D] dtype (16-byte aligned)
 *   src_k_cache, src_v_cache  [src_num_blocks][Hkv][bs][D] dtype (16-byte aligned)
 *   block_pairs  [num_pairs][2] int64 (src, dst), device or GPU-addressable host memory
 * Pairs with an id outside their pool are skipped (PA_DEVERR_PAIR).  The
 * destinations must be distinct and must not overlap the sources.
 */
pa_status pa_swap_blocks(void* dst_k_cache, void* dst_v_cache, int dst_num_blocks,
                         const void* src_k_cache, const void* src_v_cache, int src_num_blocks,
                         const int64_t* block_pairs, int num_pairs, int num_kv_heads,
                         int head_size, int block_size, pa_dtype dtype, void* stream);

/* ------------------------------------------------------------------------ */
/* Block manager (host memory; [P1] "PagedAttention의 설계", "블록 공유";     */
/* [P2] section 3; [P3] "4.2 PagedAttention의 접근").  Not thread-safe: use one */
/* handle per thread or lock around calls.                                 */

typedef struct pa_allocator pa_allocator;

/*
 * Creates a manager of num_blocks blocks of block_size tokens.  Free blocks are
 * a LIFO stack: initial_free_order (num_blocks distinct ids; the LAST entry is
 * handed out first) or, if NULL, [num_blocks-1, ..., 1, 0].  *out receives the
 * handle (free with pa_alloc_destroy).
 */
pa_status pa_alloc_create(int num_blocks, int block_size, const int32_t* initial_free_order,
                          pa_allocator** out);
void pa_alloc_destroy(pa_allocator* a);

/* Blocks an allocation can take: the free stack plus, with prefix caching, the
 * evictable cached blocks; -1 for a NULL handle. */
int pa_alloc_num_free(const pa_allocator* a);

/* Reference count of a block (number of sequences using it); -1 if out of range. */
int pa_alloc_refcount(const pa_allocator* a, int32_t block);

/* Copies the free stack, bottom to top, into out[0..capacity); *n_out = its size. */
pa_status pa_alloc_free_stack(const pa_allocator* a, int32_t* out, int capacity, int* n_out);

/* New empty sequence; PA_ERR_INVALID if the id exists. */
pa_status pa_seq_add(pa_allocator* a, int64_t seq_id);

/* The child shares all of the parent's blocks (each block's count + 1). */
pa_status pa_seq_fork(pa_allocator* a, int64_t parent, int64_t child);

/*
 * Reserves slots for n_tokens new tokens of the sequence and writes them to
 * slots_out[0..n_tokens).  A new block is taken only when the current last
 * block is full.  If the first new token lands in a partly filled last block
 * that other sequences share, that block is replaced by a fresh one and the
 * pair (old, new) is written to cow_pair_out[0..2) with *n_cow = 1: the caller
 * must run pa_copy_blocks on it before writing the new tokens; otherwise
 * *n_cow = 0.  The copy block is taken first, then new blocks in logical order.
 * PA_ERR_OOM (nothing changed) when the free stack is too short.
 */
pa_status pa_seq_append(pa_allocator* a, int64_t seq_id, int n_tokens, int64_t* slots_out,
                        int64_t* cow_pair_out, int* n_cow);

/* Drops the sequence; its blocks lose one reference each, in logical order, and
 * blocks reaching zero are pushed on the free stack (cached blocks of a prefix
 * cache go to the back of the evictable list instead). */
pa_status pa_seq_free(pa_allocator* a, int64_t seq_id);

/*
 * Prefix caching ([P3] "5. Prefix Caching"; [P2] "4. 이 밖의 기법들": the KV
 * blocks of a prompt prefix that repeats across requests are reused).  The
 * pages give no mechanism; this library's:
 *   - each full block of a committed sequence is keyed by its content chain,
 *     (key of the previous block or none, the block's block_size token ids),
 *     compared exactly (no hash aliasing);
 *   - pa_seq_add_cached creates a sequence holding the cached blocks of the
 *     longest run of its leading full blocks whose keys are cached, stopping at
 *     the first miss and leaving at least one token uncached; *num_cached
 *     receives the tokens covered (a multiple of block_size).  The caller then
 *     appends the remaining tokens with pa_seq_append and writes their K/V;
 *   - pa_seq_commit registers the full blocks among the sequence's first
 *     num_tokens tokens (token_ids from the start of the sequence); a key that
 *     already has a block keeps it, and a block keeps its first key;
 *   - a cached block whose count reaches zero stays cached as evictable; an
 *     allocation takes the free stack first, then the least recently released
 *     evictable block, whose key is dropped.
 * pa_alloc_enable_prefix_cache turns this on (before or after blocks are in
 * use); without it pa_seq_add_cached behaves as pa_seq_add (*num_cached = 0)
 * and pa_seq_commit does nothing.  pa_alloc_evictable copies the evictable
 * list, first to be evicted first, into out[0..capacity); *n_out = its size.
 */
pa_status pa_alloc_enable_prefix_cache(pa_allocator* a);
pa_status pa_alloc_evictable(const pa_allocator* a, int32_t* out, int capacity, int* n_out);
pa_status pa_seq_add_cached(pa_allocator* a, int64_t seq_id, const int32_t* token_ids,
                            int num_tokens, int* num_cached);
pa_status pa_seq_commit(pa_allocator* a, int64_t seq_id, const int32_t* token_ids,
                        int num_tokens);

/*
 * Moves sequences from manager `src` to manager `dst` (same block size), e.g.
 * to a pinned host pool when GPU memory runs short and back again ([P1]
 * "적용 범위와 관련 연구").  Sharing among the sequences moved together is kept:
 * walking seq_ids in order and each one's blocks in logical order, a source
 * block met for the first time takes a fresh destination block (as an
 * allocation in dst) and the pair (src block, dst block) is appended to
 * pairs_out [pairs_capacity][2]; every later holder shares that block.  The
 * token counts move unchanged; then each sequence is freed in `src` in caller
 * order (as pa_seq_free).  The caller runs pa_swap_blocks on the *n_pairs pairs
 * before any block freed in `src` is written again (stream order suffices).
 * Errors change nothing: PA_ERR_OOM when dst has fewer free blocks than the
 * distinct blocks; PA_ERR_INVALID for an unknown id, an id already in dst, a
 * repeated id, differing block sizes, src == dst, or pairs_capacity below
 * the number of distinct blocks (at most the sum of the sequences' blocks).
 */
pa_status pa_seq_move(pa_allocator* src, pa_allocator* dst, const int64_t* seq_ids, int num_seqs,
                      int64_t* pairs_out, int pairs_capacity, int* n_pairs);

/* Tokens held by the sequence. */
pa_status pa_seq_num_tokens(const pa_allocator* a, int64_t seq_id, int* out);

/*
 * Host block tables for a decode batch: row b of block_tables_out
 * [num_seqs][max_blocks_per_seq] holds the physical blocks of seq_ids[b] in
 * logical order, padded with -1; context_lens_out[b] its token count.
 * PA_ERR_INVALID if a sequence is unknown or has more blocks than a row holds.
 */
pa_status pa_build_tables(const pa_allocator* a, const int64_t* seq_ids, int num_seqs,
                          int max_blocks_per_seq, int32_t* block_tables_out,
                          int32_t* context_lens_out);

/*
 * Shared-prefix groups of a decode batch for pa_decode_grouped, from its host
 * block tables (the rows pa_build_tables writes) and context lengths.
 * Consecutive sequences whose first block is the same physical block (and
 * holds a whole block of each one's tokens) form a group; its shared length
 * is the longest run of leading table entries all members have in common,
 * within the whole blocks every member's context covers, times block_size.  A
 * group of one shares nothing (0).  Host memory only:
 *   group_start_out [num_seqs + 1], shared_lens_out [num_seqs];
 *   *num_groups_out, *max_group_size_out, *max_shared_len_out.
 * PA_ERR_INVALID for a context length outside [0, max_blocks_per_seq * bs].
 */
pa_status pa_build_groups(const int32_t* block_tables, int num_seqs, int max_blocks_per_seq,
                          const int32_t* context_lens, int block_size, int32_t* group_start_out,
                          int32_t* shared_lens_out, int* num_groups_out, int* max_group_size_out,
                          int* max_shared_len_out);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H_ */

// decode_tc.cu -- paged decode attention on the 5th-generation tensor cores
// (tcgen05 + TMEM) for grouped-query heads (G = Hq/Hkv in {4, 8}), fp16/bf16,
// head size 128; the same kernel with (member, head) columns serves the shared
// spans of sequence families at G = 1, 2, 4, 8, and with (query token, head)
// columns a few query tokens per sequence.
//
// Same contract and split-K partials as decode.cu ("자기회귀 생성과 KV 캐시" and
// "PagedAttention의 설계", supersilo.blog vLLM summary: scores q.k/sqrt(d_k),
// softmax over all valid tokens with one running max/sum across blocks and
// partitions, unused tail slots masked).  When G query heads share a kv head the
// per-token work is a real dense contraction, so the two products run on the
// tensor cores with tokens as the MMA's M dimension:
//
//   S^T [128 tokens x 16] = K [128 x 128] . Q^T [128 x 16]     (heads padded to 16)
//   O^T [128 dims   x 16] += V^T [128 x 128] . P^T [128 x 16]     (both MN-major)
//
// Roles in a CTA of 6 warps, one CTA per (sequence, kv head, run of partitions):
//   warp 0   producer: block-table lookups, one TMA load per physical block of
//            its K (or V) rows into a ring of 32 KB slots (three; two in the
//            three-CTA layout) holding K_0, V_0, K_1, V_1, ...  The cache is viewed as a 4-D tensor (64 columns, 8
//            rows, 2 column halves, 8-row groups), so a block lands as
//            [8-row group][half][8 rows x 128 B] with the 128-byte swizzle: the
//            canonical K-major layout of K and MN-major layout of V^T, with
//            8-row groups 2 KB apart and halves 1 KB apart;
//   warp 1   TMEM owner and MMA issuer (one thread): S = K Q^T into one of two
//            TMEM score buffers, O += V^T P^T into the TMEM output buffer;
//   warps 2-5  softmax: each thread owns one token row of S (its TMEM lane),
//            masks invalid tokens, keeps a running max that is raised only when
//            a score exceeds it by 2^8 (then O and the partial sums are
//            rescaled), writes P (cache dtype) into shared memory for the
//            second MMA, zeroes the V rows of invalid tokens of a final tile, and
//            at the end reads its row of O from TMEM and writes the output or the
//            split-K partial.
// About 109 KB of shared memory (113 KB with 32 columns), so two CTAs share an
// SM and hide each other's pipeline fill; the group spans of families at
// G = 1, 2 use a 72 KB layout with three CTAs per SM.  Every mbarrier wait is bounded;
// block ids outside the pool are skipped and flagged.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>
#include <type_traits>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "tc_common.cuh"

namespace pa {

namespace {

using namespace tc;

constexpr unsigned FULL = 0xffffffffu;
constexpr int TOK = 128;                     // tokens per tile (M of the first MMA)
constexpr int DH = 128;                      // head size
constexpr int SLOT_BYTES = TOK * 256;        // one tile of K (or V): 32 KB
constexpr int GROUP_BYTES = 2048;            // 8 token rows, both 64-column halves
constexpr int HALF_OFF = 1024;               // second 64-column half of a group
// Threads of a CTA: producer, MMA issuer and 4 softmax warps; at N = 32
// columns 8 softmax warps, two threads per token row with 16 columns each.
template <int NP>
__host__ __device__ constexpr int tc_threads() {
  return NP == 32 ? 64 + 256 : 64 + 128;
}
constexpr float RESCALE_THRESHOLD = 8.0f;    // log2 units: raise the max past 2^8 growth
// The running max before any score: finite, so that 2^(s - m) needs no mask
// test (a masked score is -inf and gives exactly 0) and the first raise gives
// 2^(M_NONE - max) = 0; a partial that saw no score is written with max -inf.
constexpr float M_NONE = -1.0e30f;

// 2^x by the hardware's approximate base-2 exponential (flushes subnormals).
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// P^T is stored MN-major without swizzle: a 16-byte row holds 8 columns
// (heads) of one token, 128 tokens make a 2 KB chunk of 8 columns, and the
// chunks of columns 8-15 (and 16-31) follow at P_CHUNK strides.
constexpr int P_CHUNK = TOK * 16;

// Shared-memory matrix descriptor without swizzle (the interleaved layout):
// core matrices of 8 rows of 16 bytes, 128 contiguous bytes each.  For an
// MN-major operand in this layout the leading offset (lbo) steps to the next
// 8 rows along K and the stride offset (sbo) to the next 16 bytes along MN
// (the swizzled MN-major layouts use them the other way round).
__device__ __forceinline__ uint64_t smem_desc_plain(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

// Two floats rounded to T and packed (the first in the low half), one cvt.
template <typename T>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
  } else {
    const __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
  }
}

// Shared-memory and TMEM layout for N = NP columns (16, or 32 for 32 query
// tokens x heads) and CTAS CTAs per SM.  The 1024-byte aligned part holds a
// ring of K/V tiles, the Q^T operand and PBUF P^T buffers of NP columns: for
// two CTAs per SM three tiles and two P buffers at N = 16, one at N = 32 (so
// that two CTAs still share an SM); for three CTAs per SM two tiles and one P
// buffer (72 KB at N = 16).  The barriers, the TMEM address
// and the 4-warp reduction buffer live in the 1 KB the allocation adds for
// aligning the base: in front of the aligned part where the base's offset
// leaves room, behind it otherwise (small_layout).
// TMEM: S0 [0, NP), S1 [NP, 2NP), O [2NP, 3NP).
template <int NP, int CTAS = 2>
struct Lay {
  static constexpr int NPAD = NP;
  static constexpr int SLOTS = CTAS >= 3 ? 2 : 3;
  static constexpr int PBUF = (NP <= 16 && CTAS < 3) ? 2 : 1;
  static constexpr int OPB_BYTES = 2 * NP * 128;   // Q^T (K-major) or P^T (MN-major): NP x 128 16-bit
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_Q = OFF_RING + SLOTS * SLOT_BYTES;
  static constexpr int OFF_P = OFF_Q + OPB_BYTES;
  static constexpr int ALIGNED_BYTES = OFF_P + PBUF * OPB_BYTES;
  // ring full/empty, S full/free, P full/free, Q ready
  static constexpr int NBARS = 2 * SLOTS + 4 + 2 * PBUF + 1;
  static constexpr int RED_BYTES = 4 * NP * 4;
  static constexpr int MISC_BYTES = (NBARS * 8 + 16 + 15) / 16 * 16;   // barriers, TMEM address
  static constexpr int SMEM_BYTES = ALIGNED_BYTES + 1024;
  static constexpr int TMEM_COLS = 3 * NP <= 64 ? 64 : 128;
  // small_layout's placement always fits when these hold
  static_assert(RED_BYTES <= 512 && RED_BYTES + 2 * MISC_BYTES <= 1024, "small buffers");
  static_assert(CTAS * (SMEM_BYTES + 1024) <= 228 * 1024, "CTAS CTAs per SM");
  static_assert(CTAS * TMEM_COLS <= 512, "TMEM of CTAS CTAs");
};

// Where the small buffers go, given the dynamic allocation's base: f bytes
// lie in front of the aligned part and 1024 - f behind it (f a multiple of 16).
// The reduction buffer goes in front if it fits there, else behind (1024 - f >
// 512 >= its size); the barriers take whichever side still has room, which
// RED_BYTES + 2 * MISC_BYTES <= 1024 guarantees.
template <int NP, int CTAS>
struct SmemPtrs {
  uint8_t* aligned;
  float* red;
  uint8_t* misc;
};
template <int NP, int CTAS>
__device__ __forceinline__ SmemPtrs<NP, CTAS> small_layout(uint8_t* raw) {
  using Y = Lay<NP, CTAS>;
  const uintptr_t b = reinterpret_cast<uintptr_t>(raw);
  const uint32_t f = static_cast<uint32_t>(((b + 1023) & ~static_cast<uintptr_t>(1023)) - b);
  SmemPtrs<NP, CTAS> r;
  r.aligned = raw + f;
  uint8_t* back = r.aligned + Y::ALIGNED_BYTES;
  if (f >= static_cast<uint32_t>(Y::RED_BYTES)) {
    r.red = reinterpret_cast<float*>(raw);
    r.misc = f - Y::RED_BYTES >= static_cast<uint32_t>(Y::MISC_BYTES) ? raw + Y::RED_BYTES : back;
  } else {
    r.red = reinterpret_cast<float*>(back);
    r.misc = 1024 - f - Y::RED_BYTES >= static_cast<uint32_t>(Y::MISC_BYTES) ? back + Y::RED_BYTES
                                                                               : raw;
  }
  return r;
}

struct TcParams {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* ws_o;
  float* ws_m;
  float* ws_l;
  unsigned int* status;
  int64_t max_blocks;
  int Hq, Hkv, num_blocks, block_size, partition_size, num_partitions;
  int parts_per_cta;  // consecutive partitions one CTA streams through
  float scale_log2;
  // several query tokens per sequence (NQ > 1): q / out rows are tokens; a
  // sequence's queries are served in groups of NQ by q_groups adjacent CTAs
  const int32_t* query_start;
  int total_q;
  int q_groups;
  // Shared-prefix groups (pa_decode_grouped).  seq_shift[b]: tokens at the
  // start of sequence b that the members of its group share (a multiple of the
  // block size; nullable = 0).  With group_start set (NQ > 1) a CTA serves the
  // shared span of group blockIdx.x / q_groups for NQ of its members, each
  // column a (member, head) pair; otherwise a CTA serves the tokens of its
  // sequence past seq_shift[b].  Partials go to workspace slots from slot_base.
  const int32_t* seq_shift;
  const int32_t* group_start;
  int slot_base;
  // One launch serves both parts of a grouped decode: blockIdx.x < span_x are
  // the groups' span CTAs (span_ppc partitions each, partials from slot 0),
  // the others sequence blockIdx.x - span_x past its shift (parts_per_cta
  // partitions each, partials from slot_base).
  int span_x;
  int span_ppc;
};

// NQ > 1 serves several query tokens per sequence (speculative verification):
// column c of S / O is query token c / G (one of the sequence's last Qb <= NQ
// context tokens) with head c % G, and a key counts for it only up to that
// token's own position.  NQ = 1 is the decode step and compiles as before.
template <typename T, int G, int NQ = 1, int NP = 16, int CTAS = 2>
__global__ void __launch_bounds__(tc_threads<NP>(), CTAS)
    decode_partition_tc_kernel(const TcParams p, const __grid_constant__ CUtensorMap tmap_k,
                               const __grid_constant__ CUtensorMap tmap_v) {
  using Y = Lay<NP, CTAS>;
  constexpr int NPAD = NP, SLOTS = Y::SLOTS, PBUF = Y::PBUF, OPB_BYTES = Y::OPB_BYTES;
  constexpr int OFF_RING = Y::OFF_RING, OFF_Q = Y::OFF_Q, OFF_P = Y::OFF_P;
  constexpr int TMEM_COLS = Y::TMEM_COLS;
  extern __shared__ uint8_t smem_raw[];
  const SmemPtrs<NP, CTAS> sp = small_layout<NP, CTAS>(smem_raw);
  uint8_t* smem = sp.aligned;
  uint8_t* ring = smem + OFF_RING;
  uint8_t* qop = smem + OFF_Q;
  uint8_t* pop = smem + OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sp.misc);
  uint64_t* ring_full = bars;
  uint64_t* ring_empty = bars + SLOTS;
  uint64_t* s_full = bars + 2 * SLOTS;      // [2]
  uint64_t* s_free = s_full + 2;            // [2]
  uint64_t* p_full = s_free + 2;            // [PBUF]
  uint64_t* p_free = p_full + PBUF;         // [PBUF]
  uint64_t* q_ready = p_free + PBUF;        // Q^T operand staged
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sp.misc + Y::NBARS * 8);
  float* red = sp.red;

  // A CTA covers parts_per_cta consecutive partitions with one softmax, so
  // short partitions do not each pay the pipeline's fill and drain: its partial
  // goes to the first one's slot and the others' slots get empty partials (max
  // -inf, sum 0, output 0), which the reduce weighs by exactly 0.
  // this CTA's work: a group's shared span, several query tokens of one
  // sequence, or (the decode) one sequence past its shift
  const bool grouped = NQ > 1 && p.group_start != nullptr && blockIdx.x < p.span_x;
  const bool multi = NQ > 1 && p.query_start != nullptr;
  int b = multi ? blockIdx.x / p.q_groups : blockIdx.x - p.span_x;
  const int ppc = grouped ? p.span_ppc : p.parts_per_cta;
  const int g = blockIdx.y, part = blockIdx.z * ppc;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NC = G * NQ;                // S / O columns in use
  static_assert(NC <= NPAD, "query tokens x heads must fit the MMA's N");
  constexpr int NSPL = NP == 32 ? 2 : 1;    // softmax threads per token row
  constexpr int NSW = 4 * NSPL;             // softmax warps
  constexpr int NCH = NC / NSPL;            // S / O columns per softmax thread in use
  constexpr int NLD = NPAD / NSPL;          // ... and loaded (whole 16-column TMEM loads)
  static_assert(NLD % 16 == 0 && NCH <= NLD, "16-column TMEM loads per softmax thread");
  static_assert(NC % (8 * NSPL) == 0 || NSPL == 1, "whole P chunks per softmax thread");
  constexpr int KTHREADS = tc_threads<NP>();

  grid_dependency_wait();   // the appended tokens of the previous kernel are in the cache
  allow_dependents();       // the reduce kernel may start launching
  const int bs = p.block_size;
  int gs = 0, ge = 0;       // group mode: the group's members gs .. ge - 1 (gs's table row)
  if (grouped) {
    gs = p.group_start[blockIdx.x / p.q_groups];
    ge = p.group_start[blockIdx.x / p.q_groups + 1];
    if (gs < 0 || ge < gs || ge > p.total_q) {      // total_q = num_seqs here
      if (threadIdx.x == 0 && blockIdx.z == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
      return;
    }
    if (gs == ge) return;
    if (ge - gs > p.q_groups * NQ && blockIdx.x % p.q_groups == 0 && threadIdx.x == 0 &&
        blockIdx.z == 0 && g == 0)
      atomicOr(p.status, PA_DEVERR_CONTEXT);    // more members than max_group_size
    b = gs;
  }
  int L = p.context_lens[b];
  // this CTA's query tokens: q0 .. q0 + Qb - 1, at positions L - Qall + qoff + c / G
  int q0 = b, Qb = 1, Qall = 1, qoff = 0;
  int shift = 0;            // tokens of the sequence skipped (served by its group)
  if (grouped) {
    // members m0 .. m0 + Qb - 1 of the group, all attending to the whole
    // shared span [0, S) of the first member's table (Qall = 1, qoff = 0 put
    // every column's causal limit at the span's last token)
    const int m0 = gs + (blockIdx.x % p.q_groups) * NQ;
    Qb = min(NQ, ge - m0);
    if (Qb <= 0) return;
    const int S = p.seq_shift[gs];
    bool bad = S < 0 || S % bs != 0 || S > L;
    for (int m = m0; m < m0 + Qb; ++m)
      bad |= p.seq_shift[m] != S || p.context_lens[m] < S;
    if (bad) {
      if (threadIdx.x == 0 && blockIdx.z == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
      return;
    }
    q0 = m0;
    L = S;
  } else if (multi) {
    const int qg = blockIdx.x % p.q_groups;
    const int qs = p.query_start[b];
    Qall = p.query_start[b + 1] - qs;
    if (Qall < 0 || Qall > L || Qall > NQ * p.q_groups || qs < 0 || qs + Qall > p.total_q) {
      if (threadIdx.x == 0 && blockIdx.z == 0 && g == 0 && qg == 0)
        atomicOr(p.status, PA_DEVERR_CONTEXT);
      return;
    }
    qoff = qg * NQ;
    q0 = qs + qoff;
    Qb = min(NQ, Qall - qoff);
    if (Qb <= 0) return;
  }
  const int P = p.partition_size;
  int64_t cap = p.max_blocks * p.block_size;
  if (L < 0 || L > cap) {
    if (threadIdx.x == 0 && part == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
    L = L < 0 ? 0 : static_cast<int>(cap);
  }
  if (!grouped && !multi && p.seq_shift != nullptr) {
    // the tokens past the sequence's shared span (its group serves the span)
    shift = p.seq_shift[b];
    if (shift < 0 || shift % bs != 0 || shift > L) {
      if (threadIdx.x == 0 && part == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
      shift = 0;
    }
    L -= shift;
  }
  const int slot0 = grouped ? 0 : p.slot_base;        // this CTA's first workspace slot
  const int64_t grid_cap = static_cast<int64_t>(p.num_partitions - slot0) * P;
  if (L > grid_cap) {
    if (threadIdx.x == 0 && part == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
    L = static_cast<int>(grid_cap);
  }
  const int start = part * P;
  if (L == 0) {
    if (!grouped && !multi && part == 0 && shift == 0) {
      T* o = static_cast<T*>(p.out) + (static_cast<int64_t>(b) * p.Hq + g * G) * DH;
      for (int i = threadIdx.x; i < G * DH; i += KTHREADS) o[i] = Elem<T>::from_float(0.f);
    }
    return;
  }
  if (start >= L) return;
  const int end = static_cast<int>(
      min(static_cast<int64_t>(L), start + static_cast<int64_t>(P) * ppc));
  const int n_tiles = (end - start + TOK - 1) / TOK;
  // the output directly, or partials for the reduce (always for a group's span
  // and for a sequence whose first tokens its group served)
  const bool single = (L <= P) && !grouped && shift == 0;
  const int n_slots = min(ppc, (L + P - 1) / P - part);   // partials this CTA writes

  // ---- set-up: the producer starts streaming right after the barrier, while
  // the softmax warps stage Q^T and the MMA issuer waits for it ----
  const int bpt = TOK / bs;                              // blocks per tile: 4, 8 or 16
  const int first_blk = start / bs;
  const int last_blk = (end + bs - 1) / bs;
  const int32_t* trow = p.block_tables + static_cast<int64_t>(b) * p.max_blocks + shift / bs;
  int pb_first = -1;                                     // tile 0's table entries, read early
  if (warp == 0) {
    if (lane < min(bpt, last_blk - first_blk)) pb_first = __ldg(trow + first_blk + lane);
    if (lane == 0) {
      for (int s = 0; s < SLOTS; ++s) {
        mbar_init(&ring_full[s], 1);
        mbar_init(&ring_empty[s], 1);
      }
      for (int j = 0; j < 2; ++j) {
        mbar_init(&s_full[j], 1);
        mbar_init(&s_free[j], NSW);
      }
      for (int j = 0; j < PBUF; ++j) {
        mbar_init(&p_full[j], NSW);
        mbar_init(&p_free[j], 1);
      }
      mbar_init(q_ready, NSW);
      fence_mbar_init();
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_v)) : "memory");
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 2) {
    // Q^T operand (16 rows = heads, 128 columns = dims, two swizzled 64-column
    // blocks), rows >= G zero; both P buffers zeroed (their rows >= G stay 0).
    const int t = threadIdx.x - 64;
    for (int i = t; i < NPAD * (DH / 8); i += 32 * NSW) {   // one 16-byte chunk each
      const int h = i / (DH / 8);                      // column: query token h / G, head h % G
      const int c = i % (DH / 8);                      // chunk of 8 dims
      uint4 v = make_uint4(0, 0, 0, 0);
      if (h < NC && h / G < Qb) {
        const T* qrow = static_cast<const T*>(p.q) +
                        ((static_cast<int64_t>(q0) + h / G) * p.Hq + g * G + h % G) * DH;
        v = __ldg(reinterpret_cast<const uint4*>(qrow + c * 8));
      }
      const uint32_t off = (c / 8) * (NPAD * 128) + sw128(h, (c % 8) * 8);
      *reinterpret_cast<uint4*>(qop + off) = v;
    }
    for (int i = t; i < PBUF * OPB_BYTES / 16; i += 32 * NSW)
      reinterpret_cast<uint4*>(pop)[i] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(q_ready);
  }

  if (warp == 0) {
    // ================= producer =================
    const int row_stride = p.Hkv * bs;                   // rows of one physical block
    bool ok = true;
    int issued = 0;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int b0 = first_blk + i * bpt;
      const int nb = min(bpt, last_blk - b0);
      int pb = pb_first;
      if (i > 0) pb = lane < nb ? __ldg(trow + b0 + lane) : -1;
      const bool mine = lane < nb;
      const bool valid = mine && pb >= 0 && pb < p.num_blocks;
      if (mine && !valid) atomicOr(p.status, PA_DEVERR_TABLE);
      const unsigned vmask = __ballot_sync(FULL, valid);
      const uint32_t bytes = __popc(vmask) * 2u * static_cast<uint32_t>(bs) * 128u;
      const int grp = valid ? (pb * row_stride + g * bs) / 8 : 0;   // first 8-row group
      for (int kv = 0; kv < 2; ++kv) {                   // 0: K, 1: V
        const int u = 2 * i + kv;
        const int s = u % SLOTS;
        if (u >= SLOTS && !mbar_wait(&ring_empty[s], ((u / SLOTS) - 1) & 1, p.status)) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(&ring_full[s], bytes);
        __syncwarp();
        if (valid) {
          uint8_t* dst = ring + s * SLOT_BYTES + lane * bs * 256;
          const CUtensorMap* map = kv == 0 ? &tmap_k : &tmap_v;
          tma_load_4d(dst, map, 0, 0, 0, grp, &ring_full[s]);
        }
        issued = u + 1;
      }
    }
    if (!ok) {
      for (int u = issued - SLOTS < 0 ? 0 : issued - SLOTS; u < issued; ++u)
        mbar_wait(&ring_full[u % SLOTS], (u / SLOTS) & 1, p.status);
    }
    return;
  }

  if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      const uint32_t id_qk = instr_desc<T, NPAD>(false);
      const uint32_t id_pv = instr_desc<T, NPAD>(true) | (1u << 16);   // V^T and P^T MN-major
      const uint32_t ring_a = smem_addr(ring), q_a = smem_addr(qop), p_a = smem_addr(pop);
      bool ok = true;
      auto issue_qk = [&](int i) -> bool {
        const int u = 2 * i, s = u % SLOTS;
        if (!mbar_wait(&ring_full[s], (u / SLOTS) & 1, p.status)) return false;
        if (i >= 2 && !mbar_wait(&s_free[i & 1], ((i >> 1) - 1) & 1, p.status)) return false;
        tc_fence_after();
        const uint32_t d = tmem + (i & 1) * NPAD;
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const uint32_t koff = (k >> 2) * HALF_OFF + (k & 3) * 32;
          const uint64_t a = smem_desc(ring_a + s * SLOT_BYTES + koff, 16, GROUP_BYTES);
          const uint64_t bq = smem_desc(q_a + (k >> 2) * (NPAD * 128) + (k & 3) * 32, 16, 1024);
          mma_f16(d, a, bq, id_qk, k > 0);
        }
        mma_commit(&s_full[i & 1]);
        mma_commit(&ring_empty[s]);
        return true;
      };
      auto issue_pv = [&](int i) -> bool {
        const int u = 2 * i + 1, s = u % SLOTS;
        if (!mbar_wait(&ring_full[s], (u / SLOTS) & 1, p.status)) return false;
        if (!mbar_wait(&p_full[i % PBUF], (i / PBUF) & 1, p.status)) return false;
        const bool first = i == 0;                     // O starts at 0
        tc_fence_after();
        const uint32_t d = tmem + 2 * NPAD;
#pragma unroll
        for (int k = 0; k < TOK / 16; ++k) {
          const uint64_t a =
              smem_desc(ring_a + s * SLOT_BYTES + k * 2 * GROUP_BYTES, HALF_OFF, GROUP_BYTES);
          const uint64_t bp = smem_desc_plain(p_a + (i % PBUF) * OPB_BYTES + k * 16 * 16, 128, P_CHUNK);
          mma_f16(d, a, bp, id_pv, (!first || k > 0) ? 1u : 0u);
        }
        mma_commit(&ring_empty[s]);
        mma_commit(&p_free[i % PBUF]);
        return true;
      };
      ok = mbar_wait(q_ready, 0, p.status) && issue_qk(0);
      for (int i = 0; i < n_tiles && ok; ++i) {
        if (i + 1 < n_tiles) ok = issue_qk(i + 1);
        if (ok) ok = issue_pv(i);
      }
    }
    __syncwarp();
  } else {
    // ================= softmax warps =================
    // NSPL threads per token row: the warps of half hf (NCH columns from c0)
    // meet on named barrier 1 + 2 hf.
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int hf = NSPL == 1 ? 0 : (warp - 2) >> 2;   // column half (a constant 0 when NSPL = 1)
    const int c0 = hf * NCH;                   // first S / O column of this thread
    const int sbar = 1 + 2 * hf;
    const int r = quad * 32 + lane;            // token row of the tile / dim row of O
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    float m_run[NCH], l_part[NCH];
#pragma unroll
    for (int h = 0; h < NCH; ++h) {
      m_run[h] = M_NONE;
      l_part[h] = 0.f;
    }
    // A failed (timed-out) wait makes `ok` false for the whole warp; later waits
    // are then skipped, but every named barrier is still joined so the
    // softmax warps never wait on each other forever.
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (ok) ok = mbar_wait(bar, parity, p.status);
      ok = __all_sync(FULL, ok);
      return ok;
    };
    // Row r of O^T (dim r, this thread's columns) and the sums of the CTA's
    // span, whose last tile is i: the output, or the split-K partial of
    // partition part (and empty partials for the span's other partitions).
    auto flush = [&](int i) {
      wait(&p_free[i % PBUF], (i / PBUF) & 1);
      tc_fence_after();
      float o[NLD];
      tmem_ld_cols<NLD>(tmem + lane_base + 2 * NPAD + c0, o);
      tc_fence_before();
      __syncwarp();
#pragma unroll
      for (int h = 0; h < NCH; ++h) {
        float x = l_part[h];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
        l_part[h] = x;
      }
      named_sync(sbar, 128);
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < NCH; ++h) red[quad * NPAD + c0 + h] = l_part[h];
      }
      named_sync(sbar, 128);
      if (ok) {
#pragma unroll
        for (int h = 0; h < NCH; ++h) {
          const int hg = c0 + h;                 // column: query row hg / G, head hg % G
          const float Ls = red[hg] + red[NPAD + hg] + red[2 * NPAD + hg] + red[3 * NPAD + hg];
          const int64_t hq = (static_cast<int64_t>(q0) + hg / G) * p.Hq + g * G + hg % G;
          if (NQ > 1 && hg / G >= Qb) continue;
          if (single) {
            static_cast<T*>(p.out)[hq * DH + r] = Elem<T>::from_float(o[h] / Ls);
          } else {
            const int64_t slot = hq * p.num_partitions + slot0 + part;
            p.ws_o[slot * DH + r] = o[h];
            if (r == 0) {
              p.ws_m[slot] = Ls > 0.f ? m_run[h] : -INFINITY;
              p.ws_l[slot] = Ls;
            }
            for (int e = 1; e < n_slots; ++e) {
              p.ws_o[(slot + e) * DH + r] = 0.f;
              if (r == 0) {
                p.ws_m[slot + e] = -INFINITY;
                p.ws_l[slot + e] = 0.f;
              }
            }
          }
        }
      }
    };
    for (int i = 0; i < n_tiles; ++i) {
      const int n_valid = min(TOK, end - (start + i * TOK));
      const bool valid = r < n_valid;
      float sv[NLD];
      if (wait(&s_full[i & 1], (i >> 1) & 1)) {
        tc_fence_after();
        tmem_ld_cols<NLD>(tmem + lane_base + (i & 1) * NPAD + c0, sv);
      } else {
#pragma unroll
        for (int h = 0; h < NLD; ++h) sv[h] = 0.f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[i & 1]);
      float s[NCH];
      bool need = false;
#pragma unroll
      for (int h = 0; h < NCH; ++h) {
        bool ok_h = valid;
        if constexpr (NQ > 1) {  // causal: up to query token hg / G's own position
          const int hg = c0 + h;
          ok_h = ok_h && hg / G < Qb && start + i * TOK + r <= L - Qall + qoff + hg / G;
        }
        s[h] = ok_h ? sv[h] * p.scale_log2 : -INFINITY;
        need |= s[h] > m_run[h] + RESCALE_THRESHOLD;
      }
      if (bar_or(sbar, 128, need)) {
        // raise the running max to this tile's max (the half's 128 threads agree)
#pragma unroll
        for (int h = 0; h < NCH; ++h) {
          float x = s[h];
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) x = fmaxf(x, __shfl_xor_sync(FULL, x, off));
          if (lane == 0) red[quad * NPAD + c0 + h] = x;
        }
        named_sync(sbar, 128);
        float alpha[NCH];
#pragma unroll
        for (int h = 0; h < NCH; ++h) {
          const int hg = c0 + h;
          const float tmax =
              fmaxf(fmaxf(red[hg], red[NPAD + hg]), fmaxf(red[2 * NPAD + hg], red[3 * NPAD + hg]));
          const float mnew = fmaxf(m_run[h], tmax);
          alpha[h] = ex2_fast(m_run[h] - mnew);   // 0 after M_NONE
          m_run[h] = mnew;
          l_part[h] *= alpha[h];
        }
        named_sync(sbar, 128);
        // O must hold every earlier tile before it is rescaled (at the first
        // tile O starts from zero instead)
        if (i > 0 && wait(&p_free[(i - 1) % PBUF], ((i - 1) / PBUF) & 1)) {
          tc_fence_after();
          float o[NLD];
          tmem_ld_cols<NLD>(tmem + lane_base + 2 * NPAD + c0, o);
#pragma unroll
          for (int h = 0; h < NCH; ++h) o[h] *= alpha[h];
          tmem_st_cols<NLD>(tmem + lane_base + 2 * NPAD + c0, o);
        }
      }
      float pr[NCH];
#pragma unroll
      for (int h = 0; h < NCH; ++h) {
        pr[h] = ex2_fast(s[h] - m_run[h]);        // masked: 2^-inf = 0
        l_part[h] += pr[h];
      }
      if (i >= PBUF) wait(&p_free[i % PBUF], ((i / PBUF) - 1) & 1);   // P buffer read
      // token r's columns are 16-byte rows of the MN-major P^T operand: heads
      // 8c .. 8c + 7 at chunk c (columns >= NC stay 0)
      uint8_t* pb = pop + (i % PBUF) * OPB_BYTES + r * 16;
#pragma unroll
      for (int c = 0; c < (NCH + 7) / 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h = 8 * c + 2 * e;
          w[e] = pack2<T>(h < NCH ? pr[h < NCH ? h : 0] : 0.f,
                          h + 1 < NCH ? pr[h + 1 < NCH ? h + 1 : 0] : 0.f);
        }
        *reinterpret_cast<uint4*>(pb + (c0 / 8 + c) * P_CHUNK) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      if (n_valid < TOK && hf == 0) {
        // the last tile: zero the V rows of tokens past the end, so that
        // whatever they hold (unused slots, stale data) adds 0 * 0 to O (one
        // half's warps do it; the MMA waits for every softmax warp)
        const int u = 2 * i + 1, s_ = u % SLOTS;
        // The parity wait below is only sound once the slot's previous load
        // has landed.  With three slots that is K of tile i - 1, which S of
        // tile i - 1 needed; with two it is V of tile i - 1, which may still be
        // in flight (tile i's fewer blocks can land first) — wait for the MMA
        // that read it, or the zeroing could come before tile i's V lands and
        // bring back whatever the cache holds past the context.
        if (SLOTS == 2 && i > 0) wait(&p_free[(i - 1) % PBUF], ((i - 1) / PBUF) & 1);
        if (wait(&ring_full[s_], (u / SLOTS) & 1) && !valid) {
          uint8_t* row = ring + s_ * SLOT_BYTES + (r >> 3) * GROUP_BYTES + (r & 7) * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            *reinterpret_cast<uint4*>(row + c * 16) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(row + HALF_OFF + c * 16) = make_uint4(0, 0, 0, 0);
          }
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[i % PBUF]);
    }
    flush(n_tiles - 1);
  }

  // ---- teardown: warps 1 .. (all but the producer) meet, warp 1 frees TMEM ----
  tc_fence_before();
  named_sync(2, KTHREADS - 32);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

// ---- host side ----

template <typename T, int G>
cudaError_t launch_tc_t(const DecodeArgs& a, unsigned int* status, cudaStream_t stream) {
  const int ppc = tc_parts_per_cta(a);
  auto kern = decode_partition_tc_kernel<T, G>;
  constexpr int SMEM_BYTES = Lay<16>::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e == cudaSuccess)   // all of the SM's 228 KB as shared memory: two CTAs of up to 113 KB
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  // the cache [NB][Hkv][bs][128] as a 4-D tensor: 64 columns (stride 2 B),
  // 8 rows (256 B), 2 column halves (128 B), NB*Hkv*bs/8 row groups (2 KB); a
  // box is one physical block: 64 x 8 x 2 x bs/8, stored with the 128-byte swizzle
  CUtensorMap mk, mv;
  const int64_t groups = static_cast<int64_t>(a.num_blocks) * a.Hkv * a.block_size / 8;
  const int64_t dims[4] = {64, 8, 2, groups};
  const int64_t strides[3] = {DH * 2, 128, 8 * DH * 2};
  const int box[4] = {64, 8, 2, a.block_size / 8};
  if (!make_tmap(&mk, a.k_cache, 4, dims, strides, box, a.dtype) ||
      !make_tmap(&mv, a.v_cache, 4, dims, strides, box, a.dtype))
    return cudaErrorInvalidValue;
  TcParams p;
  p.out = a.out;
  p.q = a.q;
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  const int64_t nrows = static_cast<int64_t>(a.num_seqs) * a.Hq * a.num_partitions;
  p.ws_o = a.workspace;
  p.ws_m = a.workspace ? a.workspace + nrows * DH : nullptr;
  p.ws_l = a.workspace ? a.workspace + nrows * (DH + 1) : nullptr;
  p.status = status;
  p.max_blocks = a.max_blocks;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.num_blocks = a.num_blocks;
  p.block_size = a.block_size;
  p.partition_size = a.partition_size;
  p.num_partitions = a.num_partitions;
  p.parts_per_cta = ppc;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.query_start = nullptr;
  p.total_q = a.num_seqs;
  p.q_groups = 1;
  p.seq_shift = a.seq_shift;
  p.group_start = nullptr;
  p.slot_base = a.slot_base;
  p.span_x = 0;
  p.span_ppc = 1;
  const int np = a.num_partitions - a.slot_base;
  dim3 grid(a.num_seqs, a.Hkv, (np + p.parts_per_cta - 1) / p.parts_per_cta);
  return launch_overlapped(kern, grid, dim3(tc_threads<16>()), SMEM_BYTES, stream, p, mk, mv);
}

// The groups' shared spans, with NQ = 16 / G: each CTA serves NQ members of a
// group (column = (member, head)), one CTA per (group, run of NQ members, kv
// head, run of span partitions), partials into slots [0, a.slot_base) of every
// member's row.  (The kernel can also take the rest of every sequence in the
// same grid, blockIdx.x >= span_x; launched alone, the rest keeps its own
// kernel and N, which measured faster.)
template <typename T, int G, int CTAS = 2, int NQ = 16 / G>
cudaError_t launch_group_tc_t(const DecodeArgs& a, unsigned int* status, cudaStream_t stream) {
  auto kern = decode_partition_tc_kernel<T, G, NQ, 16, CTAS>;
  constexpr int SMEM_BYTES = Lay<16, CTAS>::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e == cudaSuccess)   // all of the SM's 228 KB as shared memory
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  CUtensorMap mk, mv;
  const int64_t groups = static_cast<int64_t>(a.num_blocks) * a.Hkv * a.block_size / 8;
  const int64_t dims[4] = {64, 8, 2, groups};
  const int64_t strides[3] = {DH * 2, 128, 8 * DH * 2};
  const int box[4] = {64, 8, 2, a.block_size / 8};
  if (!make_tmap(&mk, a.k_cache, 4, dims, strides, box, a.dtype) ||
      !make_tmap(&mv, a.v_cache, 4, dims, strides, box, a.dtype))
    return cudaErrorInvalidValue;
  TcParams p;
  p.out = a.out;
  p.q = a.q;
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  const int64_t nrows = static_cast<int64_t>(a.num_seqs) * a.Hq * a.num_partitions;
  p.ws_o = a.workspace;
  p.ws_m = a.workspace + nrows * DH;
  p.ws_l = a.workspace + nrows * (DH + 1);
  p.status = status;
  p.max_blocks = a.max_blocks;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.num_blocks = a.num_blocks;
  p.block_size = a.block_size;
  p.partition_size = a.partition_size;
  p.num_partitions = a.num_partitions;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.query_start = nullptr;
  p.total_q = a.num_seqs;
  p.q_groups = (a.max_group_size + NQ - 1) / NQ;
  p.seq_shift = a.seq_shift;
  p.group_start = a.group_start;
  p.slot_base = a.slot_base;                       // = the groups' span partitions
  const int span_parts = a.slot_base;
  const int rest_parts = a.num_partitions - a.slot_base;
  p.span_x = a.num_groups * p.q_groups;
  // streaming by the decode kernel's rule, counting the rest's CTAs, which run
  // at the same time on the caller's stream
  const int64_t span_rows = static_cast<int64_t>(p.span_x) * a.Hkv;
  const int64_t rest_rows = static_cast<int64_t>(a.num_seqs) * a.Hkv;
  p.parts_per_cta = 1;
  p.span_ppc = tc_parts_per_cta(span_rows, a.partition_size, span_parts, rest_rows * rest_parts);
  dim3 grid(p.span_x, a.Hkv, (span_parts + p.span_ppc - 1) / p.span_ppc);
  return launch_overlapped(kern, grid, dim3(tc_threads<16>()), SMEM_BYTES, stream, p, mk, mv);
}

}  // namespace

static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

// Consecutive partitions per CTA (one softmax over them): for partitions
// shorter than 2048 tokens, the most of 8 / 4 / 2 that keeps a CTA's span
// within 4096 tokens and still leaves at least 8 CTAs per SM.
int tc_parts_per_cta(int64_t rows, int partition_size, int n_parts, int64_t other_ctas) {
  if (partition_size >= 2048 || n_parts <= 0) return 1;
  const int64_t want = 8ll * sm_count();
  for (int c : {8, 4, 2}) {
    const int64_t ctas = rows * ((n_parts + c - 1) / c) + other_ctas;
    if (static_cast<int64_t>(partition_size) * c <= 4096 && n_parts >= c && ctas >= want) return c;
  }
  return 1;
}

int tc_parts_per_cta(const DecodeArgs& a) {
  return tc_parts_per_cta(static_cast<int64_t>(a.num_seqs) * a.Hkv, a.partition_size,
                          a.num_partitions - a.slot_base, 0);
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}
}  // namespace

bool make_tmap(void* map, const void* base, int rank, const int64_t* dims,
               const int64_t* strides_bytes, const int* box, pa_dtype dt) {
  auto fn = encode_fn();
  if (!fn || rank < 1 || rank > 5) return false;
  cuuint64_t gdim[5], gstride[4];
  cuuint32_t bdim[5], estr[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = static_cast<cuuint64_t>(dims[i]);
    bdim[i] = static_cast<cuuint32_t>(box[i]);
    estr[i] = 1u;
    if (i + 1 < rank) gstride[i] = static_cast<cuuint64_t>(strides_bytes[i]);
  }
  const CUtensorMapDataType t = dt == PA_BF16       ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                : dt == PA_FP8_E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return fn(static_cast<CUtensorMap*>(map), t, static_cast<cuuint32_t>(rank),
            const_cast<void*>(base), gdim, gstride, bdim, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tmap_available() { return encode_fn() != nullptr; }

namespace {

template <typename T, int G, int NQ, int NP = 16>
cudaError_t launch_tcq_t(const MqArgs& m, unsigned int* status, cudaStream_t stream) {
  const int q_groups = (m.max_query_len + NQ - 1) / NQ;
  const int ppc = tc_parts_per_cta(static_cast<int64_t>(m.num_seqs) * q_groups * m.Hkv,
                                   m.partition_size, m.num_partitions, 0);
  auto kern = decode_partition_tc_kernel<T, G, NQ, NP>;
  constexpr int SMEM_BYTES = Lay<NP>::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e == cudaSuccess)   // all of the SM's 228 KB as shared memory: two CTAs of up to 113 KB
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  CUtensorMap mk, mv;
  const int64_t groups = static_cast<int64_t>(m.num_blocks) * m.Hkv * m.block_size / 8;
  const int64_t dims[4] = {64, 8, 2, groups};
  const int64_t strides[3] = {DH * 2, 128, 8 * DH * 2};
  const int box[4] = {64, 8, 2, m.block_size / 8};
  if (!make_tmap(&mk, m.k_cache, 4, dims, strides, box, m.dtype) ||
      !make_tmap(&mv, m.v_cache, 4, dims, strides, box, m.dtype))
    return cudaErrorInvalidValue;
  TcParams p;
  p.out = m.out;
  p.q = m.q;
  p.block_tables = m.block_tables;
  p.context_lens = m.context_lens;
  const int64_t nrows = static_cast<int64_t>(m.total_q) * m.Hq * m.num_partitions;
  p.ws_o = m.workspace;
  p.ws_m = m.workspace ? m.workspace + nrows * DH : nullptr;
  p.ws_l = m.workspace ? m.workspace + nrows * (DH + 1) : nullptr;
  p.status = status;
  p.max_blocks = m.max_blocks;
  p.Hq = m.Hq;
  p.Hkv = m.Hkv;
  p.num_blocks = m.num_blocks;
  p.block_size = m.block_size;
  p.partition_size = m.partition_size;
  p.num_partitions = m.num_partitions;
  p.parts_per_cta = ppc;
  p.scale_log2 = m.scale * 1.4426950408889634f;
  p.query_start = m.query_start;
  p.total_q = m.total_q;
  p.q_groups = q_groups;
  p.seq_shift = nullptr;
  p.group_start = nullptr;
  p.slot_base = 0;
  p.span_x = 0;
  p.span_ppc = 1;
  dim3 grid(m.num_seqs * p.q_groups, m.Hkv, (m.num_partitions + ppc - 1) / ppc);
  return launch_overlapped(kern, grid, dim3(tc_threads<NP>()), SMEM_BYTES, stream, p, mk, mv);
}

// Query tokens per CTA (tc_query_tokens_per_cta): up to 16 columns on the
// N = 16 kernel, else 32 columns on the N = 32 kernel, so 4 tokens at G = 8
// (or 8 at G = 4) share one read of the sequence's K/V.
template <typename T>
cudaError_t launch_tcq_g(const MqArgs& m, unsigned int* status, cudaStream_t stream) {
  const int G = m.Hq / m.Hkv;
  const int nq = tc_query_tokens_per_cta(G, m.max_query_len);
  if (G == 8) {
    return nq == 2 ? launch_tcq_t<T, 8, 2>(m, status, stream)
                   : launch_tcq_t<T, 8, 4, 32>(m, status, stream);
  }
  return nq == 2 ? launch_tcq_t<T, 4, 2>(m, status, stream)
       : nq == 4 ? launch_tcq_t<T, 4, 4>(m, status, stream)
                 : launch_tcq_t<T, 4, 8, 32>(m, status, stream);
}

}  // namespace

bool decode_mq_tc_supported(const MqArgs& m) {
  const int G = m.Hkv > 0 ? m.Hq / m.Hkv : 0;
  // up to 64 (query token, head) columns, in one or two CTAs per sequence;
  // longer query runs are prefill-like
  return (m.dtype == PA_F16 || m.dtype == PA_BF16) && m.D == DH && (G == 4 || G == 8) &&
         m.max_query_len >= 1 && m.max_query_len * G <= 64 && m.partition_size % TOK == 0 &&
         static_cast<int64_t>(m.num_blocks) * m.Hkv * m.block_size < (int64_t(1) << 31) &&
         encode_fn() != nullptr;
}

int launch_decode_mq_tc(const MqArgs& m, unsigned int* status, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return m.dtype == PA_BF16 ? launch_tcq_g<__nv_bfloat16>(m, status, st)
                            : launch_tcq_g<__half>(m, status, st);
}

bool decode_tc_supported(const DecodeArgs& a) {
  const int G = a.Hq / a.Hkv;
  return (a.dtype == PA_F16 || a.dtype == PA_BF16) && a.D == DH && (G == 4 || G == 8) &&
         a.partition_size % TOK == 0 &&
         static_cast<int64_t>(a.num_blocks) * a.Hkv * a.block_size < (int64_t(1) << 31) &&
         encode_fn() != nullptr;
}

bool decode_group_tc_supported(const DecodeArgs& a) {
  const int G = a.Hq / a.Hkv;
  return (a.dtype == PA_F16 || a.dtype == PA_BF16) && a.kv_dtype == a.dtype && a.D == DH &&
         (G == 1 || G == 2 || G == 4 || G == 8) && a.partition_size % TOK == 0 &&
         static_cast<int64_t>(a.num_blocks) * a.Hkv * a.block_size < (int64_t(1) << 31) &&
         encode_fn() != nullptr;
}

// Members per span CTA: 16 / G fill the MMA's 16 columns; when every family
// has at most 8 / G members, 8 / G of them (8 columns in use) halve the
// softmax's per-column work on every tile at the same CTA count (the MMA still
// computes 16 columns, which costs nothing that shows).
template <typename T, int G, int CTAS>
int launch_group_g(const DecodeArgs& a, unsigned int* status, cudaStream_t stream) {
  if constexpr (G <= 4) {
    if (static_cast<int64_t>(a.max_group_size) * G <= 8)
      return launch_group_tc_t<T, G, CTAS, 8 / G>(a, status, stream);
  }
  return launch_group_tc_t<T, G, CTAS>(a, status, stream);
}

// G = 1, 2 (families of parallel samples: each span is a prompt's own blocks,
// read from HBM by few CTAs of a few tiles each) take the layout with rings of
// two tiles and one P buffer, three CTAs per SM: more spans in flight at once
// (llama13b_ps decode 131 -> 127 us).  G = 4, 8 keep three tiles and two CTAs
// per SM (a long prefix served from L2: 0.5 % faster).
int launch_decode_group_tc(const DecodeArgs& a, unsigned int* status, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = a.Hq / a.Hkv;
  if (a.dtype == PA_BF16) {
    switch (G) {
      case 1: return launch_group_g<__nv_bfloat16, 1, 3>(a, status, st);
      case 2: return launch_group_g<__nv_bfloat16, 2, 3>(a, status, st);
      case 4: return launch_group_g<__nv_bfloat16, 4, 2>(a, status, st);
      default: return launch_group_g<__nv_bfloat16, 8, 2>(a, status, st);
    }
  }
  switch (G) {
    case 1: return launch_group_g<__half, 1, 3>(a, status, st);
    case 2: return launch_group_g<__half, 2, 3>(a, status, st);
    case 4: return launch_group_g<__half, 4, 2>(a, status, st);
    default: return launch_group_g<__half, 8, 2>(a, status, st);
  }
}

int launch_decode_partitions_tc(const DecodeArgs& a, unsigned int* status, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = a.Hq / a.Hkv;
  if (a.dtype == PA_BF16) {
    return G == 8 ? launch_tc_t<__nv_bfloat16, 8>(a, status, st)
                  : launch_tc_t<__nv_bfloat16, 4>(a, status, st);
  }
  return G == 8 ? launch_tc_t<__half, 8>(a, status, st) : launch_tc_t<__half, 4>(a, status, st);
}

}  // namespace pa

// decode_mq.cu -- paged attention for several new query tokens per sequence
// (chunked prefill, speculative verification) on the tensor cores: fp16/bf16,
// head size 128, G = Hq/Hkv in {1, 2, 4, 8}.
//
// What is computed ("자기회귀 생성과 KV 캐시" and "PagedAttention의 설계",
// supersilo.blog; chunked prefill and speculative decoding in "4. 이 밖의
// 기법들", blog.aqudi.me): sequence b's last Q_b context tokens are its query
// tokens (rows query_start[b] .. query_start[b+1]-1 of q); query token i sits
// at position L_b - Q_b + i and attends, through the block table, to
// positions 0 .. L_b - Q_b + i with one softmax over them.
//
// With many query rows the work is query-major, as in a prefill kernel: a CTA
// serves one (sequence, kv head, pair of blocks of 128/G query tokens,
// partition of keys); each block's 128 rows are (query token, query head)
// pairs of that kv head, and per tile of 128 keys, for each of the two blocks
//
//   S [128 rows x 128 keys] = Q [128 x 128] . K^T          (K K-major)
//   O [128 rows x 128 dims] += P [128 x 128 keys] . V      (P from TMEM, V MN-major)
//
// run on tcgen05 (kind::f16, fp32 accumulation in TMEM).  K and V tiles are
// the TMA boxes of decode_tc.cu (one 4-D box per physical block, 128-byte
// swizzle).  The MMA issuer alternates between the two blocks, so the tensor
// core runs one block's products while the softmax threads work on the
// other's.  A row's running max, sum and causal limit belong to its two
// softmax threads (one per 64-column half of each tile and of O); a warp
// rescales its half of its 32 rows of O in TMEM when one of their maxima grows
// by more than 2^8.  P goes back into the TMEM columns of the S it came from
// and feeds the second product from there.
//
// Roles (18 warps): warp 0 TMA producer, warp 1 TMEM owner and MMA issuer,
// warps 2-9 the first block's Q staging, softmax and epilogue, warps 10-17 the
// second block's.  A ring of three K/V tiles and the two Q blocks, about 167
// KB of shared memory, and all 512 TMEM columns: one CTA per SM.  Every wait
// is bounded; block ids outside the pool are skipped and flagged;
// inconsistent query offsets are flagged (PA_DEVERR_CONTEXT) and their
// sequence skipped.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "tc_common.cuh"

namespace pa {

namespace {

using namespace tc;

constexpr unsigned FULL = 0xffffffffu;
constexpr int TOK = 128;                   // keys per tile
constexpr int MR = 128;                    // query rows per query block
constexpr int DH = 128;
constexpr int SLOTS = 3;
constexpr int SLOT_BYTES = TOK * 256;      // K or V tile (as in decode_tc.cu): 32 KB
constexpr int GROUP_BYTES = 2048;
constexpr int HALF_OFF = 1024;
constexpr int OPA_BYTES = MR * 256;        // a 128 x 128 16-bit row-major operand: 32 KB
constexpr int OPA_HALF = MR * 128;         // its second 64-column half
constexpr int TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;

// ---- the query-major kernel with two query tiles per CTA (decode_mq_kernel) ----
// TMEM: S of tile X at X * 128, O of tile X at 256 + X * 128; P of tile X
// (bf16/f16 pairs) overwrites the S columns it was computed from.
constexpr int NT = kMqTiles;                  // query tiles per CTA
constexpr int THREADS2 = 64 + NT * 256;       // producer, MMA, 8 softmax warps per tile
constexpr int OFF2_Q = SLOTS * SLOT_BYTES;
constexpr int OFF2_BAR = OFF2_Q + NT * OPA_BYTES;
constexpr int NBARS2 = 2 * SLOTS + 3 * NT + 1;  // ring full/empty, s_full, p_full, p_free, q_ready
constexpr int OFF2_TMEM = OFF2_BAR + NBARS2 * 8;
constexpr int OFF2_RMAX = (OFF2_TMEM + 16 + 15) / 16 * 16;  // [2 tiles parity][NT][2 halves][MR]
constexpr int OFF2_RSUM = OFF2_RMAX + 2 * NT * 2 * MR * 4;   // [NT][2 halves][MR]
constexpr int SMEM2_USED = OFF2_RSUM + NT * 2 * MR * 4;
constexpr int SMEM2_BYTES = SMEM2_USED + 1024;
static_assert(SMEM2_BYTES <= 227 * 1024, "shared memory");
static_assert(NT == 2, "two query tiles: TMEM holds 2 x (S, O) of 128 columns");

// kind::f16 instruction descriptor, fp32 accumulation, M = 128, N = 128;
// A K-major; B K-major (S) or MN-major (O).
template <typename T>
__device__ __forceinline__ constexpr uint32_t idesc_mq(bool b_mn_major) {
  constexpr uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
  return (1u << 4) | (fmt << 7) | (fmt << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

// MMA with the A operand in TMEM (M = 128 lanes, K along the columns: two
// 16-bit elements per 32-bit column) and B from shared memory.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16 32-bit words into 16 consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t* w) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
      "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 2^x by the SFU's approximation (relative error about 2^-22; 2^-inf = +0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

// Byte offset of the 16-byte chunk c (elements 8c..8c+7) of row r of a
// 128 x 128 16-bit operand stored as two 64-column halves with the 128-byte
// swizzle (the canonical K-major layout).
__device__ __forceinline__ uint32_t opa_chunk(int r, int c) {
  return (c >> 3) * OPA_HALF + r * 128 + ((((c & 7) ^ (r & 7)) & 7) << 4);
}

struct MqParams {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start;
  float* ws_o;
  float* ws_m;
  float* ws_l;
  unsigned int* status;
  int64_t max_blocks;
  int num_seqs, total_q, Hq, Hkv, num_blocks, block_size, partition_size, num_partitions;
  float scale_log2;
};

// Query-major multi-query kernel with two query tiles per CTA: a CTA serves
// (sequence, kv head, pair of query blocks of 128 / G tokens, key partition).
// Per 128-key tile the MMA issuer alternates between the tiles (S_A, S_B, then
// O_A += P_A V and O_B += P_B V as each tile's softmax finishes), so the tensor
// core works on one tile while the softmax threads work on the other.  Each
// row has two softmax threads (warps of the same TMEM lane quadrant, one per
// 64-column half, as in decode_mq_kernel); tile X has its own 8 warps.  P is
// written back into the TMEM columns of the S it came from (half h's 64 keys as
// 32 columns of 16-bit pairs at h * 64) and is the A operand of the second MMA
// straight from TMEM, so no shared memory holds P.  Warps 0 and 1: producer
// and MMA issuer; warps 2 + 8X .. 9 + 8X: tile X.  Shared memory: the K/V ring
// and the two Q tiles (~167 KB); all 512 TMEM columns.
template <typename T, int G>
__global__ void __launch_bounds__(THREADS2, 1)
    decode_mq_kernel(const MqParams p, const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v) {
  constexpr int QB = MR / G;                        // query tokens per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint8_t* qop = smem + OFF2_Q;                     // NT tiles of OPA_BYTES
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF2_BAR);
  uint64_t* ring_full = bars;
  uint64_t* ring_empty = bars + SLOTS;
  uint64_t* s_full = bars + 2 * SLOTS;              // [NT]
  uint64_t* p_full = s_full + NT;                   // [NT]
  uint64_t* p_free = p_full + NT;                   // [NT]
  uint64_t* q_ready = p_free + NT;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF2_TMEM);
  float* rmax = reinterpret_cast<float*>(smem + OFF2_RMAX);
  float* rsum = reinterpret_cast<float*>(smem + OFF2_RSUM);

  const int n_pairs = gridDim.z / p.num_partitions;
  const int b = blockIdx.x, g = blockIdx.y;
  const int pair = blockIdx.z % n_pairs, part = blockIdx.z / n_pairs;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  grid_dependency_wait();
  allow_dependents();
  // ---- this CTA's query rows and key range (validated) ----
  const int q0 = p.query_start[b];
  const int Qb = p.query_start[b + 1] - q0;
  int L = p.context_lens[b];
  const int P = p.partition_size;
  int64_t cap = p.max_blocks * p.block_size;
  const int64_t grid_cap = static_cast<int64_t>(p.num_partitions) * P;
  cap = cap < grid_cap ? cap : grid_cap;
  if (L < 0 || L > cap || Qb < 0 || Qb > L || q0 < 0 || q0 + Qb > p.total_q) {
    if (threadIdx.x == 0 && pair == 0 && part == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
    return;
  }
  if (pair == 0 && part == 0 && g == 0 && threadIdx.x == 0 && Qb > n_pairs * NT * QB)
    atomicOr(p.status, PA_DEVERR_CONTEXT);          // max_query_len below this Q_b
  const int qb0 = pair * NT;                        // the CTA's first query block
  if (qb0 * QB >= Qb) return;                       // no query tokens here
  const int i_last = min(Qb, (qb0 + NT) * QB) - 1;  // the CTA's last query token
  const int pmax = L - Qb + i_last;                 // its position: the last key needed
  const int kstart = part * P;
  if (kstart > pmax) return;
  const int kend = min(kstart + P, pmax + 1);
  const int n_tiles = (kend - kstart + TOK - 1) / TOK;
  const bool single = (pmax < P);

  const int bs = p.block_size;
  const int bpt = TOK / bs;
  const int first_blk = kstart / bs;
  const int last_blk = (kend + bs - 1) / bs;
  const int32_t* trow = p.block_tables + static_cast<int64_t>(b) * p.max_blocks;
  if (threadIdx.x == 0) {
    for (int s = 0; s < SLOTS; ++s) {
      mbar_init(&ring_full[s], 1);
      mbar_init(&ring_empty[s], 1);
    }
    for (int x = 0; x < NT; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 8);
      mbar_init(&p_free[x], 1);
    }
    mbar_init(q_ready, 8 * NT);
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_v)) : "memory");
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

  if (warp == 0) {
    // ================= producer (as in decode_mq_kernel) =================
    const int row_stride = p.Hkv * bs;
    bool ok = true;
    int issued = 0;
    auto table = [&](int i) {
      const int b0 = first_blk + i * bpt;
      return (i < n_tiles && lane < min(bpt, last_blk - b0)) ? __ldg(trow + b0 + lane) : -1;
    };
    int pb_next = table(0);
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int b0 = first_blk + i * bpt;
      const int nb = min(bpt, last_blk - b0);
      const int pb = pb_next;
      pb_next = table(i + 1);
      const bool mine = lane < nb;
      const bool valid = mine && pb >= 0 && pb < p.num_blocks;
      if (mine && !valid) atomicOr(p.status, PA_DEVERR_TABLE);
      const unsigned vmask = __ballot_sync(FULL, valid);
      const uint32_t bytes = __popc(vmask) * 2u * static_cast<uint32_t>(bs) * 128u;
      const int grp = valid ? (pb * row_stride + g * bs) / 8 : 0;
      for (int kv = 0; kv < 2; ++kv) {
        const int u = 2 * i + kv;
        const int s = u % SLOTS;
        if (u >= SLOTS && !mbar_wait(&ring_empty[s], ((u / SLOTS) - 1) & 1, p.status)) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(&ring_full[s], bytes);
        __syncwarp();
        if (valid)
          tma_load_4d(ring + s * SLOT_BYTES + lane * bs * 256, kv == 0 ? &tmap_k : &tmap_v, 0, 0,
                      0, grp, &ring_full[s]);
        issued = u + 1;
      }
    }
    if (!ok) {
      for (int u = issued - SLOTS < 0 ? 0 : issued - SLOTS; u < issued; ++u)
        mbar_wait(&ring_full[u % SLOTS], (u / SLOTS) & 1, p.status);
    }
    return;
  }

  // softmax thread: tile X, row r (TMEM lane), key / dim half `half`
  const int lw = warp - 2;                          // 0 .. 8 NT - 1 for softmax warps
  const int X = lw >> 3;
  const int half = (lw >> 2) & 1;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  const int il = r / G, hl = r % G;
  const int qtok = (qb0 + X) * QB + il;             // query token of the row within the sequence
  const bool row_valid = warp >= 2 && qtok < Qb;
  const int64_t t = static_cast<int64_t>(q0) + qtok;
  const int pos = L - Qb + qtok;
  const int pair_bar = 3 + X * 4 + quad;            // named barrier of this row's two threads

  if (warp >= 2) {
    // Q operand of tile X: row r = q[t][g*G + hl][:] (this thread its 8 of
    // the 16 chunks), zero for rows past the sequence's query tokens
    const T* src = static_cast<const T*>(p.q) + (t * p.Hq + g * G + hl) * DH;
    uint4 v[DH / 16];
#pragma unroll
    for (int c = 0; c < DH / 16; ++c)
      v[c] = row_valid ? __ldg(reinterpret_cast<const uint4*>(src + (half * 8 + c) * 8))
                       : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int c = 0; c < DH / 16; ++c)
      *reinterpret_cast<uint4*>(qop + X * OPA_BYTES + opa_chunk(r, half * 8 + c)) = v[c];
    fence_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(q_ready);
  }

  if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      const uint32_t id_s = idesc_mq<T>(false);
      const uint32_t id_o = idesc_mq<T>(true);
      const uint32_t ring_a = smem_addr(ring), q_a = smem_addr(qop);
      bool ok = true;
      auto issue_s = [&](int x, int i) {           // S_x = Q_x . K_i^T
        const int s = (2 * i) % SLOTS;
        const uint32_t d = tmem + x * 128;
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const uint64_t a =
              smem_desc(q_a + x * OPA_BYTES + (k >> 2) * OPA_HALF + (k & 3) * 32, 16, 1024);
          const uint64_t bk =
              smem_desc(ring_a + s * SLOT_BYTES + (k >> 2) * HALF_OFF + (k & 3) * 32, 16, GROUP_BYTES);
          mma_f16(d, a, bk, id_s, k > 0);
        }
        mma_commit(&s_full[x]);
      };
      auto issue_pv = [&](int x, int i) {          // O_x += P_x . V_i, P_x in TMEM
        const int s = (2 * i + 1) % SLOTS;
        const uint32_t d = tmem + 256 + x * 128;
#pragma unroll
        for (int k = 0; k < TOK / 16; ++k) {
          // keys 16k .. 16k + 15: half k / 4's P columns
          const uint32_t a = tmem + x * 128 + (k >> 2) * 64 + (k & 3) * 8;
          const uint64_t bv =
              smem_desc(ring_a + s * SLOT_BYTES + k * 2 * GROUP_BYTES, HALF_OFF, GROUP_BYTES);
          mma_f16_ts(d, a, bv, id_o, (i > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(&p_free[x]);
      };
      auto ring_wait = [&](int u) { return mbar_wait(&ring_full[u % SLOTS], (u / SLOTS) & 1, p.status); };
      ok = mbar_wait(q_ready, 0, p.status) && ring_wait(0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        mma_commit(&ring_empty[0]);
      }
      for (int i = 0; i < n_tiles && ok; ++i) {
        ok = ring_wait(2 * i + 1) && mbar_wait(&p_full[0], i & 1, p.status);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, i);
        const bool more = i + 1 < n_tiles;
        if (more) {
          ok = ring_wait(2 * i + 2);
          if (!ok) break;
          tc_fence_after();
          issue_s(0, i + 1);                       // after O_0 += P_0 V_i read P_0's columns
        }
        ok = mbar_wait(&p_full[1], i & 1, p.status);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, i);
        mma_commit(&ring_empty[(2 * i + 1) % SLOTS]);
        if (more) {
          issue_s(1, i + 1);
          mma_commit(&ring_empty[(2 * i + 2) % SLOTS]);
        }
      }
    }
    __syncwarp();
  } else if (warp >= 2) {
    // ================= softmax of tile X, two threads per row =================
    const bool warp_active = __any_sync(FULL, row_valid);
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t s_col = tmem + lane_base + X * 128 + half * 64;      // my 64 S columns
    const uint32_t o_col = tmem + lane_base + 256 + X * 128 + half * 64; // my 64 dims of O
    const int col0 = half * 64;
    float m_run = -INFINITY, l_half = 0.f;
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (ok) ok = mbar_wait(bar, parity, p.status);
      ok = __all_sync(FULL, ok);
      return ok;
    };
    for (int i = 0; i < n_tiles; ++i) {
      const int tile0 = kstart + i * TOK;
      const int n_valid = min(TOK, kend - tile0);
      wait(&s_full[X], i & 1);
      tc_fence_after();
      if (warp_active) {
        const int lim = row_valid ? min(pos - tile0, n_valid - 1) : -1;  // last key column
        const bool open = __all_sync(FULL, col0 + 63 <= lim);
        // pass 1: the row's maximum over this half (raw scores when open)
        float pm[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) pm[k] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float sv[32];
          if (ok) tmem_ld32(s_col + c * 32, sv);
          else
#pragma unroll
            for (int j = 0; j < 32; ++j) sv[j] = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float x = open ? sv[j] : (col0 + c * 32 + j <= lim ? sv[j] : -INFINITY);
            pm[j & 7] = fmaxf(pm[j & 7], x);
          }
        }
        float tmax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                           fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
        tmax = tmax == -INFINITY ? tmax : tmax * p.scale_log2;
        rmax[(((i & 1) * NT + X) * 2 + half) * MR + r] = tmax;
        named_sync(pair_bar, 64);
        tmax = fmaxf(tmax, rmax[(((i & 1) * NT + X) * 2 + (half ^ 1)) * MR + r]);
        const bool need = tmax > m_run + RESCALE_THRESHOLD;
        if (__any_sync(FULL, need)) {              // the same for both warps of the pair
          const float mnew = fmaxf(m_run, tmax);
          const float alpha = (m_run == -INFINITY) ? 0.f : exp2f(m_run - mnew);
          m_run = mnew;
          l_half *= alpha;
          // O must hold every earlier tile before it is rescaled
          if (i > 0 && wait(&p_free[X], (i - 1) & 1)) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
              float o[32];
              tmem_ld32(o_col + c * 32, o);
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] *= alpha;
              tmem_st32(o_col + c * 32, o);
            }
          }
        }
        // pass 2: P = 2^(scale * s - m) into the first 32 of my S columns
        const float neg_m = -m_run;
        float ps[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) ps[k] = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float sv[32];
          if (ok) tmem_ld32(s_col + c * 32, sv);
          else
#pragma unroll
            for (int j = 0; j < 32; ++j) sv[j] = 0.f;
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int j0 = 2 * e, j1 = 2 * e + 1;
            float p0, p1;
            if (open) {
              p0 = ex2_approx(fmaf(sv[j0], p.scale_log2, neg_m));
              p1 = ex2_approx(fmaf(sv[j1], p.scale_log2, neg_m));
            } else {
              const bool v0 = col0 + c * 32 + j0 <= lim && m_run != -INFINITY;
              const bool v1 = col0 + c * 32 + j1 <= lim && m_run != -INFINITY;
              p0 = v0 ? ex2_approx(fmaf(sv[j0], p.scale_log2, neg_m)) : 0.f;
              p1 = v1 ? ex2_approx(fmaf(sv[j1], p.scale_log2, neg_m)) : 0.f;
            }
            ps[(2 * e) & 7] += p0;
            ps[(2 * e + 1) & 7] += p1;
            w[e] = pack2<T>(p0, p1);
          }
          tmem_st16u(s_col + c * 16, w);
        }
        l_half += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      } else {
        // no query row in this warp: its P rows are 0
        uint32_t z[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) z[e] = 0u;
        tmem_st16u(s_col, z);
        tmem_st16u(s_col + 16, z);
      }
      if (X == 0 && n_valid < TOK) {
        // the last tile: zero the V rows of keys past the range (this thread
        // its 64-dim half of row r), so that whatever they hold adds 0 to O
        const int u = 2 * i + 1, s_ = u % SLOTS;
        if (wait(&ring_full[s_], (u / SLOTS) & 1) && r >= n_valid) {
          uint8_t* row = ring + s_ * SLOT_BYTES + (r >> 3) * GROUP_BYTES + (r & 7) * 128 + half * HALF_OFF;
#pragma unroll
          for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(row + c * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[X]);
    }
    // ---- epilogue: row r of O_X, dims col0..col0+63; the row's sum over both halves ----
    rsum[(X * 2 + half) * MR + r] = l_half;
    named_sync(pair_bar, 64);
    const float l_sum = l_half + rsum[(X * 2 + (half ^ 1)) * MR + r];
    wait(&p_free[X], (n_tiles - 1) & 1);
    tc_fence_after();
    const int64_t hq = t * p.Hq + g * G + hl;
#pragma unroll 1
    for (int c = 0; c < (warp_active ? 2 : 0); ++c) {
      float o[32];
      tmem_ld32(o_col + c * 32, o);
      if (ok && row_valid) {
        if (single) {
          const float inv = 1.f / l_sum;
          T* dst = static_cast<T*>(p.out) + hq * DH + col0 + c * 32;
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) w[e] = pack2<T>(o[j + 2 * e] * inv, o[j + 2 * e + 1] * inv);
            *reinterpret_cast<uint4*>(dst + j) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          const int64_t slot = hq * p.num_partitions + part;
          float* dst = p.ws_o + slot * DH + col0 + c * 32;
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(dst + j) = make_float4(o[j], o[j + 1], o[j + 2], o[j + 3]);
          if (c == 0 && half == 0) {
            p.ws_m[slot] = m_run;
            p.ws_l[slot] = l_sum;
          }
        }
      }
    }
  }

  // ---- teardown: warps 1 .. 1 + 8 NT meet, warp 1 frees TMEM ----
  tc_fence_before();
  named_sync(2, THREADS2 - 32);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

struct MqReduceParams {
  void* out;
  const int32_t* context_lens;
  const int32_t* query_start;
  const float* ws_o;
  const float* ws_m;
  const float* ws_l;
  int num_seqs, total_q, Hq, partition_size, num_partitions;
  int direct_qblock;  // query-token run length of the partition launcher (MqArgs)
};

// One warp per (query token, head) whose block spanned several partitions.
template <typename T>
__global__ void __launch_bounds__(128) decode_mq_reduce_kernel(const MqReduceParams p) {
  constexpr int DPL = DH / 32;
  grid_dependency_wait();
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<int64_t>(p.total_q) * p.Hq) return;
  const int t = static_cast<int>(row / p.Hq);
  // the sequence of token t: the last b with query_start[b] <= t
  int lo = 0, hi = p.num_seqs;                      // invariant: qs[lo] <= t < qs[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.query_start[mid] <= t) lo = mid; else hi = mid;
  }
  const int b = lo;
  const int Qb = p.query_start[b + 1] - p.query_start[b];
  const int L = p.context_lens[b];
  const int i = t - p.query_start[b];
  if (Qb <= 0 || Qb > L || i < 0 || i >= Qb) return;   // flagged by the partition kernel
  // the run of query tokens token i was served in (the partition launcher's
  // grouping), and that run's last key position
  const int QB = p.direct_qblock;
  const int i_last = min(Qb, (i / QB + 1) * QB) - 1;
  const int pmax = L - Qb + i_last;
  if (pmax < p.partition_size) return;              // written directly
  const int pos = L - Qb + i;
  const int np = min(pos / p.partition_size + 1, p.num_partitions);
  const int64_t base = row * p.num_partitions;
  float M = -INFINITY;
  for (int k = lane; k < np; k += 32) M = fmaxf(M, p.ws_m[base + k]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, off));
  float Ls = 0.f;
  for (int k = lane; k < np; k += 32) Ls += p.ws_l[base + k] * exp2f(p.ws_m[base + k] - M);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) Ls += __shfl_xor_sync(FULL, Ls, off);
  float acc[DPL];
#pragma unroll
  for (int k = 0; k < DPL; ++k) acc[k] = 0.f;
  for (int k = 0; k < np; ++k) {
    const float f = exp2f(p.ws_m[base + k] - M);
    const float* src = p.ws_o + (base + k) * DH + lane * DPL;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = fmaf(f, src[e], acc[e]);
  }
  T* dst = static_cast<T*>(p.out) + row * DH + lane * DPL;
  const float inv = 1.f / Ls;
#pragma unroll
  for (int e = 0; e < DPL; ++e) dst[e] = Elem<T>::from_float(acc[e] * inv);
}

template <typename T, int G>
cudaError_t launch_mq_t(const MqArgs& a, unsigned int* status, cudaStream_t stream) {
  auto kern = decode_mq_kernel<T, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM2_BYTES);
  if (e != cudaSuccess) return e;
  CUtensorMap mk, mv;
  const int64_t groups = static_cast<int64_t>(a.num_blocks) * a.Hkv * a.block_size / 8;
  const int64_t dims[4] = {64, 8, 2, groups};
  const int64_t strides[3] = {DH * 2, 128, 8 * DH * 2};
  const int box[4] = {64, 8, 2, a.block_size / 8};
  if (!make_tmap(&mk, a.k_cache, 4, dims, strides, box, a.dtype) ||
      !make_tmap(&mv, a.v_cache, 4, dims, strides, box, a.dtype))
    return cudaErrorInvalidValue;
  MqParams p;
  p.out = a.out;
  p.q = a.q;
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.query_start = a.query_start;
  const int64_t nrows = static_cast<int64_t>(a.total_q) * a.Hq * a.num_partitions;
  p.ws_o = a.workspace;
  p.ws_m = a.workspace ? a.workspace + nrows * DH : nullptr;
  p.ws_l = a.workspace ? a.workspace + nrows * (DH + 1) : nullptr;
  p.status = status;
  p.max_blocks = a.max_blocks;
  p.num_seqs = a.num_seqs;
  p.total_q = a.total_q;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.num_blocks = a.num_blocks;
  p.block_size = a.block_size;
  p.partition_size = a.partition_size;
  p.num_partitions = a.num_partitions;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  const int qblocks = (a.max_query_len + MR / G - 1) / (MR / G);
  const int pairs = (qblocks + NT - 1) / NT;
  dim3 grid(a.num_seqs, a.Hkv, pairs * a.num_partitions);
  return launch_overlapped(kern, grid, dim3(THREADS2), SMEM2_BYTES, stream, p, mk, mv);
}

template <typename T>
cudaError_t launch_mq_reduce_t(const MqArgs& a, cudaStream_t stream) {
  MqReduceParams p;
  p.out = a.out;
  p.context_lens = a.context_lens;
  p.query_start = a.query_start;
  const int64_t nrows = static_cast<int64_t>(a.total_q) * a.Hq * a.num_partitions;
  p.ws_o = a.workspace;
  p.ws_m = a.workspace + nrows * DH;
  p.ws_l = a.workspace + nrows * (DH + 1);
  p.num_seqs = a.num_seqs;
  p.total_q = a.total_q;
  p.Hq = a.Hq;
  p.direct_qblock = a.direct_qblock > 0 ? a.direct_qblock : NT * (MR / (a.Hq / a.Hkv));
  p.partition_size = a.partition_size;
  p.num_partitions = a.num_partitions;
  const int64_t warps = static_cast<int64_t>(a.total_q) * a.Hq;
  const unsigned grid = static_cast<unsigned>((warps + 3) / 4);
  return launch_overlapped(decode_mq_reduce_kernel<T>, dim3(grid), dim3(128), 0, stream, p);
}

template <typename T>
cudaError_t launch_mq_g(const MqArgs& a, unsigned int* status, cudaStream_t stream) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_mq_t<T, 1>(a, status, stream);
    case 2: return launch_mq_t<T, 2>(a, status, stream);
    case 4: return launch_mq_t<T, 4>(a, status, stream);
    case 8: return launch_mq_t<T, 8>(a, status, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int launch_decode_mq(const MqArgs& a, unsigned int* status, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return a.dtype == PA_BF16 ? launch_mq_g<__nv_bfloat16>(a, status, st)
                            : launch_mq_g<__half>(a, status, st);
}

int launch_decode_mq_reduce(const MqArgs& a, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return a.dtype == PA_BF16 ? launch_mq_reduce_t<__nv_bfloat16>(a, st)
                            : launch_mq_reduce_t<__half>(a, st);
}

}  // namespace pa

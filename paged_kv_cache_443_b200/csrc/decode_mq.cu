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
// serves one (sequence, kv head, block of 128/G query tokens, partition of
// keys); its 128 rows are (query token, query head) pairs of that kv head, and
// per tile of 128 keys
//
//   S [128 rows x 128 keys] = Q [128 x 128] . K^T          (K K-major)
//   O [128 rows x 128 dims] += P [128 x 128 keys] . V      (V MN-major)
//
// run on tcgen05 (kind::f16, fp32 accumulation in TMEM).  K and V tiles are
// the TMA boxes of decode_tc.cu (one 4-D box per physical block, 128-byte
// swizzle).  A row's running max, sum and causal limit belong to its two
// softmax threads, and a warp rescales its half of its 32 rows of O in TMEM
// when one of their maxima grows by more than 2^8.
//
// Roles (10 warps): warp 0 TMA producer, warp 1 TMEM owner and MMA issuer,
// warps 2-9 Q staging, softmax and epilogue, two threads per row: the warps
// w and w + 4 share a TMEM lane quadrant, one takes key columns 0-63 of each
// tile (and dims 0-63 of O), the other 64-127, and the pair agrees on each
// row's maximum through shared memory and a named barrier.  A ring of three
// K/V tiles, about 196 KB of shared memory and all 512 TMEM columns: one CTA
// per SM.  Every wait is bounded; block ids
// outside the pool are skipped and flagged; inconsistent query offsets are
// flagged (PA_DEVERR_CONTEXT) and their sequence skipped.
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
constexpr int MR = 128;                    // query rows per CTA
constexpr int DH = 128;
constexpr int SLOTS = 3;
constexpr int SLOT_BYTES = TOK * 256;      // K or V tile (as in decode_tc.cu): 32 KB
constexpr int GROUP_BYTES = 2048;
constexpr int HALF_OFF = 1024;
constexpr int OPA_BYTES = MR * 256;        // a 128 x 128 16-bit row-major operand: 32 KB
constexpr int OPA_HALF = MR * 128;         // its second 64-column half
constexpr int OFF_RING = 0;
constexpr int OFF_Q = OFF_RING + SLOTS * SLOT_BYTES;
constexpr int OFF_P = OFF_Q + OPA_BYTES;   // two P buffers
constexpr int OFF_BAR = OFF_P + 2 * OPA_BYTES;
constexpr int NBARS = 2 * SLOTS + 9;
constexpr int OFF_TMEM = OFF_BAR + NBARS * 8;
constexpr int OFF_RMAX = (OFF_TMEM + 16 + 15) / 16 * 16;   // [2 tiles][2 halves][MR] row maxima
constexpr int OFF_RSUM = OFF_RMAX + 2 * 2 * MR * 4;          // [2 halves][MR] row sums
constexpr int SMEM_USED = OFF_RSUM + 2 * MR * 4;
constexpr int SMEM_BYTES = SMEM_USED + 1024;
constexpr int THREADS = 320;                 // producer, MMA, 8 softmax warps
constexpr int NSOFT = 256;                   // softmax threads: two per row
constexpr int TMEM_COLS = 512;             // S0 [0,128), S1 [128,256), O [256,384)
constexpr int O_COL = 256;
constexpr float RESCALE_THRESHOLD = 8.0f;

static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");

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

// One TMEM load of 128 consecutive 32-bit columns of this thread's lane, one wait.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, float* v) {
  uint32_t r[128];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 128; ++i) v[i] = __uint_as_float(r[i]);
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

template <typename T, int G>
__global__ void __launch_bounds__(THREADS, 1)
    decode_mq_kernel(const MqParams p, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v) {
  constexpr int QB = MR / G;                        // query tokens per CTA
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem + OFF_RING;
  uint8_t* qop = smem + OFF_Q;
  uint8_t* pop = smem + OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* ring_full = bars;
  uint64_t* ring_empty = bars + SLOTS;
  uint64_t* s_full = bars + 2 * SLOTS;      // [2]
  uint64_t* s_free = s_full + 2;            // [2]
  uint64_t* p_full = s_free + 2;            // [2]
  uint64_t* p_free = p_full + 2;            // [2]
  uint64_t* q_ready = p_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_TMEM);

  // the query blocks of one (sequence, kv head, key partition) are adjacent in
  // the grid, so they run together and read that partition's K/V from L2
  const int n_qb = gridDim.z / p.num_partitions;
  const int b = blockIdx.x, g = blockIdx.y;
  const int qb = blockIdx.z % n_qb, part = blockIdx.z / n_qb;
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
    if (threadIdx.x == 0 && qb == 0 && part == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
    return;
  }
  if (qb == 0 && part == 0 && g == 0 && threadIdx.x == 0 &&
      Qb > static_cast<int>(gridDim.z / p.num_partitions) * QB)
    atomicOr(p.status, PA_DEVERR_CONTEXT);          // max_query_len below this Q_b
  if (qb * QB >= Qb) return;                        // no query tokens in this block
  const int i_last = min(Qb, (qb + 1) * QB) - 1;    // last query token of the block
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
    for (int j = 0; j < 2; ++j) {
      mbar_init(&s_full[j], 1);
      mbar_init(&s_free[j], 8);
      mbar_init(&p_full[j], 8);
      mbar_init(&p_free[j], 1);
    }
    mbar_init(q_ready, 8);
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
    // ================= producer (as in decode_tc.cu) =================
    const int row_stride = p.Hkv * bs;
    bool ok = true;
    int issued = 0;
    auto table = [&](int i) {                       // lane j: block j of tile i, read a tile ahead
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

  // rows of this CTA: r = il * G + hl  (query token il of the block, head hl).
  // Each row has two softmax threads in two warps of the same TMEM lane
  // quadrant: `half` 0 takes key columns 0-63 of a tile (and dims 0-63 of O),
  // half 1 columns 64-127 (dims 64-127).
  const int quad = warp & 3;
  const int half = warp >= 6 ? 1 : 0;
  const int r = quad * 32 + lane;
  const int il = r / G, hl = r % G;
  const bool row_valid = warp >= 2 && qb * QB + il < Qb;
  const int64_t t = static_cast<int64_t>(q0) + qb * QB + il;          // query token index
  const int pos = L - Qb + qb * QB + il;                               // its position
  float* rmax = reinterpret_cast<float*>(smem + OFF_RMAX);            // [2][2][MR]
  float* rsum = reinterpret_cast<float*>(smem + OFF_RSUM);            // [2][MR]

  if (warp >= 2) {
    // Q operand: row r = q[t][g*G + hl][:] (this thread its half of the 16
    // chunks), zero for rows past the block's tokens
    const T* src = static_cast<const T*>(p.q) + (t * p.Hq + g * G + hl) * DH;
    uint4 v[DH / 16];
#pragma unroll
    for (int c = 0; c < DH / 16; ++c)
      v[c] = row_valid ? __ldg(reinterpret_cast<const uint4*>(src + (half * 8 + c) * 8))
                       : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int c = 0; c < DH / 16; ++c) *reinterpret_cast<uint4*>(qop + opa_chunk(r, half * 8 + c)) = v[c];
    fence_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(q_ready);
  }

  if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      const uint32_t id_s = idesc_mq<T>(false);
      const uint32_t id_o = idesc_mq<T>(true);
      const uint32_t ring_a = smem_addr(ring), q_a = smem_addr(qop), p_a = smem_addr(pop);
      bool ok = true;
      auto issue_s = [&](int i) -> bool {
        const int u = 2 * i, s = u % SLOTS;
        if (!mbar_wait(&ring_full[s], (u / SLOTS) & 1, p.status)) return false;
        if (i >= 2 && !mbar_wait(&s_free[i & 1], ((i >> 1) - 1) & 1, p.status)) return false;
        tc_fence_after();
        const uint32_t d = tmem + (i & 1) * 128;
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const uint64_t a = smem_desc(q_a + (k >> 2) * OPA_HALF + (k & 3) * 32, 16, 1024);
          const uint64_t bk =
              smem_desc(ring_a + s * SLOT_BYTES + (k >> 2) * HALF_OFF + (k & 3) * 32, 16, GROUP_BYTES);
          mma_f16(d, a, bk, id_s, k > 0);
        }
        mma_commit(&s_full[i & 1]);
        mma_commit(&ring_empty[s]);
        return true;
      };
      auto issue_o = [&](int i) -> bool {
        const int u = 2 * i + 1, s = u % SLOTS;
        if (!mbar_wait(&ring_full[s], (u / SLOTS) & 1, p.status)) return false;
        if (!mbar_wait(&p_full[i & 1], (i >> 1) & 1, p.status)) return false;
        tc_fence_after();
        const uint32_t d = tmem + O_COL;
#pragma unroll
        for (int k = 0; k < TOK / 16; ++k) {
          const uint64_t a =
              smem_desc(p_a + (i & 1) * OPA_BYTES + (k >> 2) * OPA_HALF + (k & 3) * 32, 16, 1024);
          const uint64_t bv =
              smem_desc(ring_a + s * SLOT_BYTES + k * 2 * GROUP_BYTES, HALF_OFF, GROUP_BYTES);
          mma_f16(d, a, bv, id_o, (i > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(&ring_empty[s]);
        mma_commit(&p_free[i & 1]);
        return true;
      };
      ok = mbar_wait(q_ready, 0, p.status) && issue_s(0);
      for (int i = 0; i < n_tiles && ok; ++i) {
        if (i + 1 < n_tiles) ok = issue_s(i + 1);
        if (ok) ok = issue_o(i);
      }
    }
    __syncwarp();
  } else if (warp >= 2) {
    // ================= softmax: two threads per row =================
    // A warp whose 32 rows hold no query token (few queries per sequence) only
    // keeps pace with the barriers and zeroes V rows; its P rows stay zero.
    // The two threads of a row meet at a named barrier of their warp pair
    // (id 3 + quad) to agree on the row's maximum each tile.
    const bool warp_active = __any_sync(FULL, row_valid);
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int col0 = half * 64;                        // this thread's key / dim columns
    float m_run = -INFINITY, l_half = 0.f;
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (ok) ok = mbar_wait(bar, parity, p.status);
      ok = __all_sync(FULL, ok);
      return ok;
    };
    if (!warp_active) {
#pragma unroll
      for (int buf = 0; buf < 2; ++buf)
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(pop + buf * OPA_BYTES + opa_chunk(r, half * 8 + c)) =
              make_uint4(0, 0, 0, 0);
    }
    for (int i = 0; i < n_tiles; ++i) {
      const int tile0 = kstart + i * TOK;
      const int n_valid = min(TOK, kend - tile0);
      wait(&s_full[i & 1], (i >> 1) & 1);
      if (warp_active) {
        const int lim = row_valid ? min(pos - tile0, n_valid - 1) : -1;  // last key column
        float sv[64];
        if (ok) {
          tc_fence_after();
          tmem_ld32(tmem + lane_base + (i & 1) * 128 + col0, sv);
          tmem_ld32(tmem + lane_base + (i & 1) * 128 + col0 + 32, sv + 32);
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j) sv[j] = 0.f;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[i & 1]);
        // Every column of this thread's half visible to every row of the warp
        // (all but the diagonal and last tiles): no mask, and the scale (> 0)
        // moves into the exponent's FMA below, so the scores stay raw here.
        const bool open = __all_sync(FULL, col0 + 63 <= lim);
        float pm[8];                                   // 8 independent partial maxima
#pragma unroll
        for (int k = 0; k < 8; ++k) pm[k] = -INFINITY;
        if (open) {
#pragma unroll
          for (int j = 0; j < 64; ++j) pm[j & 7] = fmaxf(pm[j & 7], sv[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            sv[j] = col0 + j <= lim ? sv[j] * p.scale_log2 : -INFINITY;
            pm[j & 7] = fmaxf(pm[j & 7], sv[j]);
          }
        }
        float tmax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                           fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
        if (open) tmax *= p.scale_log2;
        // the row's maximum over both halves (the buffer alternates by tile, so
        // a partner a tile ahead never overwrites what this thread still reads)
        rmax[((i & 1) * 2 + half) * MR + r] = tmax;
        named_sync(3 + quad, 64);
        tmax = fmaxf(tmax, rmax[((i & 1) * 2 + (half ^ 1)) * MR + r]);
        const bool need = tmax > m_run + RESCALE_THRESHOLD;
        if (__any_sync(FULL, need)) {                  // the same for both warps of the pair
          const float mnew = fmaxf(m_run, tmax);
          const float alpha = (m_run == -INFINITY) ? 0.f : exp2f(m_run - mnew);
          m_run = mnew;
          l_half *= alpha;
          // O must hold every earlier tile before it is rescaled (its dims col0..col0+63)
          if (i > 0 && wait(&p_free[(i - 1) & 1], ((i - 1) >> 1) & 1)) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
              float o[32];
              tmem_ld32(tmem + lane_base + O_COL + col0 + c * 32, o);
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] *= alpha;
              tmem_st32(tmem + lane_base + O_COL + col0 + c * 32, o);
            }
          }
        }
        if (i >= 2) wait(&p_free[i & 1], ((i >> 1) - 1) & 1);
        uint8_t* pb = pop + (i & 1) * OPA_BYTES;
        float ps[8];                                   // 8 independent partial sums
#pragma unroll
        for (int k = 0; k < 8; ++k) ps[k] = 0.f;
        // P = 2^(scale * s - m): one FMA and one ex2 per column when open
        const float neg_m = -m_run;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float s0 = sv[8 * c + 2 * e], s1 = sv[8 * c + 2 * e + 1];
            float p0, p1;
            if (open) {
              p0 = ex2_approx(fmaf(s0, p.scale_log2, neg_m));
              p1 = ex2_approx(fmaf(s1, p.scale_log2, neg_m));
            } else {
              p0 = s0 == -INFINITY ? 0.f : ex2_approx(s0 + neg_m);
              p1 = s1 == -INFINITY ? 0.f : ex2_approx(s1 + neg_m);
            }
            ps[2 * e] += p0;
            ps[2 * e + 1] += p1;
            w[e] = pack2<T>(p0, p1);
          }
          *reinterpret_cast<uint4*>(pb + opa_chunk(r, half * 8 + c)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        l_half += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      } else {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[i & 1]);
      }
      if (n_valid < TOK) {
        // the last tile: zero the V rows of keys past the range (this thread
        // its 64-dim half of row r), so that whatever they hold adds 0 * 0 to O
        const int u = 2 * i + 1, s_ = u % SLOTS;
        if (wait(&ring_full[s_], (u / SLOTS) & 1) && r >= n_valid) {
          uint8_t* row = ring + s_ * SLOT_BYTES + (r >> 3) * GROUP_BYTES + (r & 7) * 128 + half * HALF_OFF;
#pragma unroll
          for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(row + c * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[i & 1]);
    }
    // ---- epilogue: row r of O, dims col0..col0+63; the row's sum over both halves ----
    rsum[half * MR + r] = l_half;
    named_sync(3 + quad, 64);
    const float l_sum = l_half + rsum[(half ^ 1) * MR + r];
    wait(&p_free[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1);
    tc_fence_after();
    const int64_t hq = t * p.Hq + g * G + hl;
#pragma unroll 1
    for (int c = 0; c < (warp_active ? 2 : 0); ++c) {
      float o[32];
      tmem_ld32(tmem + lane_base + O_COL + col0 + c * 32, o);
      if (ok && row_valid) {
        if (single) {
          const float inv = 1.f / l_sum;
          T* dst = static_cast<T*>(p.out) + hq * DH + col0 + c * 32;
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = static_cast<uint32_t>(to_bits<T>(o[j + 2 * e] * inv)) |
                     (static_cast<uint32_t>(to_bits<T>(o[j + 2 * e + 1] * inv)) << 16);
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

  // ---- teardown: warps 1-9 meet, warp 1 frees TMEM ----
  tc_fence_before();
  named_sync(2, THREADS - 32);
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
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
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
  dim3 grid(a.num_seqs, a.Hkv, qblocks * a.num_partitions);
  return launch_overlapped(kern, grid, dim3(THREADS), SMEM_BYTES, stream, p, mk, mv);
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
  p.direct_qblock = a.direct_qblock > 0 ? a.direct_qblock : MR / (a.Hq / a.Hkv);
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

// decode_tc8.cu -- paged decode attention on the tensor cores over an E4M3 KV
// cache, head size 128, f16 or bf16 queries and outputs, G = Hq/Hkv query
// heads per kv head 4 or 8 (the code holds for 1 and 2 as well, where the
// CUDA-core kernel of decode.cu is the faster one).
//
// What is computed is that of decode_tc.cu ("자기회귀 생성과 KV 캐시" and
// "PagedAttention의 설계", supersilo.blog vLLM summary), with the cache's
// elements standing for code * k_scale and code * v_scale (E4M3 codes: the
// reading of "quantization" in "4. 이 밖의 기법들", blog.aqudi.me).  Tokens are
// the MMA's M dimension for S and the reduction dimension for O; both products
// run on kind::f8f6f4 with the cache codes as they are in shared memory:
//
//   S^T [128 tokens x 16] = K [128 x 128] . Q^T [128 x 16]         K-major K
//   O^T [128 dims   x 16] += V^T [128 x 128] . P^T [128 x 16]      MN-major V^T, P^T
//
// * Q: split into E4M3 terms, Q * 2^e = Q1 + Q2 (+ Q3) (each the nearest E4M3
//   value of what the previous terms left; e a per-head power of two putting
//   the head's largest |q| in [2^7, 2^8)), and S accumulates their products.
//   Each term takes the next 4 significant bits: three terms for an f16 query
//   (11 bits), two for a bf16 one (8 bits), so the split is exact for every
//   component at least 2^-6 of the head's largest; 2^-e and k_scale are
//   folded into the softmax scale.
// * P: the running max is raised as soon as a score passes it by 2 (base 2),
//   so P <= 4; P * 2^6 (<= 256, inside E4M3's range) is split into two E4M3
//   terms the same way, P1 + P2, which keeps P to about 2^-8 of its value for
//   P >= 2^-12 (and to 2^-16 absolutely below that).  The partial sums l add
//   the fp32 P; 2^-6 and v_scale are applied to O.
// * Each physical block's K and V codes arrive in one TMA load each, rows of
//   128 codes stored with the 128-byte swizzle: the canonical K-major layout of
//   K and, unchanged, the MN-major layout of V^T (8-token groups 1 KB apart).
//
// Roles in a CTA of 6 warps, one CTA per (sequence, kv head, run of partitions):
//   warp 0     producer: block-table lookups; per tile one TMA load per block
//              of its K codes and one of its V codes into two rings of three
//              16 KB tiles;
//   warp 1     TMEM owner and MMA issuer;
//   warps 2-5  query terms, then softmax (as in decode_tc.cu), P as two E4M3
//              terms; they zero the V rows of tokens past the end of a final
//              tile.
// About 113 KB of shared memory (two CTAs per SM) for f16 queries; for bf16
// queries two query terms, rings of two tiles and one P buffer, about 73 KB,
// so three CTAs share an SM.  Every wait is bounded;
// block ids outside the pool are skipped and flagged.
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
constexpr int TOK = 128;                    // tokens per tile
constexpr int NPAD = 16;                    // MMA N (heads padded)
constexpr int DH = 128;                     // head size
constexpr int PTERM = 2;                    // E4M3 terms of P
constexpr int TILE_BYTES = TOK * DH;        // one tile of codes: 16 KB
constexpr int QT_BYTES = NPAD * DH;         // one query term: 16 rows x 128 codes
constexpr int PT_BYTES = NPAD * TOK;        // one P term: 128 tokens x 16 heads (MN-major)
constexpr int PB_BYTES = PTERM * PT_BYTES;  // one P buffer (both terms)
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 64;               // S0 [0,16), S1 [16,32), O [32,48)
constexpr float RESCALE_THRESHOLD = 2.0f;   // P <= 2^2
constexpr float P_UP = 64.0f;               // P * 2^6 <= 256 < 448
constexpr float P_DOWN = 1.0f / 64.0f;

// 2^x by the hardware's approximate base-2 exponential (flushes subnormals).
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Shared-memory layout for NTERM query terms, SLOTS tiles per ring (one ring
// for K codes, one for V codes) and PBUF P buffers.  Two layouts are built:
//   3 terms, 3 + 3 slots, 2 P buffers (~113 KB): two CTAs per SM, for f16
//     queries (11 significant bits: three 4-bit terms);
//   2 terms, 2 + 2 slots, 1 P buffer (~73 KB): three CTAs per SM, for bf16
//     queries (8 significant bits: two 4-bit terms are exact).  A third CTA's
//     pipeline hides more of each tile's serial chain than a third slot does.
template <int NTERM_, int SLOTS_, int PBUF_>
struct Lay8 {
  static constexpr int NTERM = NTERM_, SLOTS = SLOTS_, PBUF = PBUF_;
  static constexpr int OFF_KR = 0;
  static constexpr int OFF_VR = OFF_KR + SLOTS * TILE_BYTES;
  static constexpr int OFF_Q = OFF_VR + SLOTS * TILE_BYTES;
  static constexpr int OFF_P = OFF_Q + NTERM * QT_BYTES;
  static constexpr int OFF_BAR = OFF_P + PBUF * PB_BYTES;
  static constexpr int NBARS = 4 * SLOTS + 4 + 2 * PBUF + 1;
  static constexpr int OFF_TMEM = (OFF_BAR + NBARS * 8 + 15) / 16 * 16;
  static constexpr int OFF_RED = OFF_TMEM + 16;      // 4 warps x 16 floats
  static constexpr int OFF_QS = OFF_RED + 4 * NPAD * 4;
  static constexpr int SMEM_USED = OFF_QS + NPAD * 4;
  static constexpr int SMEM_BYTES = SMEM_USED + 1024;
  static constexpr int CTAS_PER_SM = (228 * 1024) / (SMEM_BYTES + 1024);
  static_assert(OFF_VR % 1024 == 0 && OFF_Q % 1024 == 0 && OFF_P % 1024 == 0 &&
                    QT_BYTES % 1024 == 0 && PT_BYTES % 1024 == 0,
                "swizzled operands on 1 KB boundaries");
};
using LayF16 = Lay8<3, 3, 2>;
using LayBF16 = Lay8<2, 2, 1>;
static_assert(LayF16::CTAS_PER_SM >= 2, "two CTAs per SM");
static_assert(LayBF16::CTAS_PER_SM >= 3, "three CTAs per SM");
static_assert(3 * TMEM_COLS <= 512, "TMEM of three CTAs");

// Instruction descriptor of kind::f8f6f4: E4M3 x E4M3 (format 0 for both),
// fp32 accumulation, M = 128, N = 16; A K-major (S) or MN-major (O), B K-major.
constexpr uint32_t kIdescE4M3 = (1u << 4) | (static_cast<uint32_t>(NPAD >> 3) << 17) |
                                (static_cast<uint32_t>(128 >> 4) << 24);
constexpr uint32_t kIdescE4M3_AMN = kIdescE4M3 | (1u << 15);
// O += V^T P^T with V^T and P^T both MN-major (bits 15 and 16).
constexpr uint32_t kIdescE4M3_AMN_BMN = kIdescE4M3_AMN | (1u << 16);

// Shared-memory matrix descriptor without swizzle (the interleaved layout):
// 16-byte core rows, 8 rows of a core matrix 16 bytes apart.  For the MN-major
// P^T operand: each token's 16 head codes are one 16-byte row, so a core
// matrix is 8 consecutive tokens (128 contiguous bytes); the leading offset
// steps to the next 8 tokens (128 bytes on) and the stride offset, the step to
// the next 16 heads, is never used at N = 16.
__device__ __forceinline__ uint64_t smem_desc_plain(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct Tc8Params {
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
  float scale_log2;  // scale * log2(e) * k_scale
  float v_scale;
  // Shared-prefix groups (pa_decode_grouped_fp8), as in decode_tc.cu:
  // seq_shift[b] leading tokens of sequence b are its group's shared span
  // (nullable = 0).  NQ = 1: a CTA serves sequence blockIdx.x past its shift,
  // partials from workspace slot slot_base.  NQ > 1 (group_start set): a CTA
  // serves the shared span of group blockIdx.x / q_groups for NQ of its
  // members (column = (member, head)), partials from slot 0.
  const int32_t* seq_shift;
  const int32_t* group_start;
  int slot_base;
  int total_q;       // num_seqs
  int q_groups;      // CTAs per group along x (members / NQ, rounded up)
};

// Four E4M3 codes (one 32-bit word, code i in byte i) -> two f16x2 words
// (codes 0,1 and 2,3, lower code in the lower half), exactly.
__device__ __forceinline__ void widen4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// Nearest E4M3 codes of two floats (saturating; the first in the low byte).
__device__ __forceinline__ uint32_t to_e4m3x2(float a, float b) {
  return static_cast<uint32_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}
// The exact values of two codes in the low 16 bits of c.
__device__ __forceinline__ float2 from_e4m3x2(uint32_t c) {
  uint32_t lo, hi;
  widen4(c, lo, hi);
  return __half22float2(*reinterpret_cast<const __half2*>(&lo));
}

// NQ = 1 is the decode (one sequence per CTA, its G heads the columns); NQ > 1
// serves a group's shared span for NQ members at once (G * NQ <= 16 columns).
template <typename T, int G, typename Y, int NQ = 1>
__global__ void __launch_bounds__(THREADS, Y::CTAS_PER_SM)
    decode_partition_tc8_kernel(const Tc8Params p, const __grid_constant__ CUtensorMap tmap_k,
                                const __grid_constant__ CUtensorMap tmap_v) {
  constexpr int NTERM = Y::NTERM, SLOTS = Y::SLOTS, PBUF = Y::PBUF;
  constexpr int OFF_KR = Y::OFF_KR, OFF_VR = Y::OFF_VR, OFF_Q = Y::OFF_Q, OFF_P = Y::OFF_P;
  constexpr int OFF_BAR = Y::OFF_BAR, OFF_TMEM = Y::OFF_TMEM, OFF_RED = Y::OFF_RED;
  constexpr int OFF_QS = Y::OFF_QS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* kring = smem + OFF_KR;
  uint8_t* vring = smem + OFF_VR;
  uint8_t* qop = smem + OFF_Q;
  uint8_t* pop = smem + OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* kr_full = bars;                  // [SLOTS]
  uint64_t* kr_empty = kr_full + SLOTS;      // [SLOTS]
  uint64_t* vr_full = kr_empty + SLOTS;      // [SLOTS]
  uint64_t* vr_empty = vr_full + SLOTS;      // [SLOTS]
  uint64_t* s_full = vr_empty + SLOTS;       // [2]
  uint64_t* s_free = s_full + 2;             // [2]
  uint64_t* p_full = s_free + 2;             // [PBUF]
  uint64_t* p_free = p_full + PBUF;          // [PBUF]
  uint64_t* q_ready = p_free + PBUF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_TMEM);
  float* red = reinterpret_cast<float*>(smem + OFF_RED);
  float* qs = reinterpret_cast<float*>(smem + OFF_QS);

  // a CTA covers parts_per_cta consecutive partitions with one softmax (as in
  // decode_tc.cu): its partial goes to the first one's slot, the others' slots
  // get empty partials (max -inf, sum 0, output 0), which the reduce weighs by 0
  constexpr bool grouped = NQ > 1;
  constexpr int NC = G * NQ;                // S / O columns in use: (member, head)
  static_assert(NC <= NPAD, "members x heads must fit the MMA's N");
  int b = blockIdx.x;
  const int g = blockIdx.y, part = blockIdx.z * p.parts_per_cta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  grid_dependency_wait();
  allow_dependents();
  const int bs = p.block_size;
  // this CTA's query rows: sequences q0 .. q0 + Qb - 1 (columns h / G)
  int q0 = b, Qb = 1;
  int L = 0, shift = 0;
  if constexpr (grouped) {
    const int grp = blockIdx.x / p.q_groups;
    const int gs = p.group_start[grp], ge = p.group_start[grp + 1];
    if (gs < 0 || ge < gs || ge > p.total_q) {
      if (threadIdx.x == 0 && blockIdx.z == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
      return;
    }
    if (gs == ge) return;
    if (ge - gs > p.q_groups * NQ && blockIdx.x % p.q_groups == 0 && threadIdx.x == 0 &&
        blockIdx.z == 0 && g == 0)
      atomicOr(p.status, PA_DEVERR_CONTEXT);    // more members than max_group_size
    const int m0 = gs + (blockIdx.x % p.q_groups) * NQ;
    Qb = min(NQ, ge - m0);
    if (Qb <= 0) return;
    // every member attends to the whole shared span [0, S) of the first
    // member's table
    const int S = p.seq_shift[gs];
    bool bad = S < 0 || S % bs != 0 || S > p.context_lens[gs];
    for (int m = m0; m < m0 + Qb; ++m) bad |= p.seq_shift[m] != S || p.context_lens[m] < S;
    if (bad) {
      if (threadIdx.x == 0 && blockIdx.z == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
      return;
    }
    b = gs;
    q0 = m0;
    L = S;
  } else {
    L = p.context_lens[b];
  }
  const int P = p.partition_size;
  const int64_t cap = p.max_blocks * p.block_size;
  if (L < 0 || L > cap) {
    if (threadIdx.x == 0 && part == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
    L = L < 0 ? 0 : static_cast<int>(cap);
  }
  if (!grouped && p.seq_shift != nullptr) {
    // the tokens past the sequence's shared span (its group serves the span)
    shift = p.seq_shift[b];
    if (shift < 0 || shift % bs != 0 || shift > L) {
      if (threadIdx.x == 0 && part == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
      shift = 0;
    }
    L -= shift;
  }
  const int slot0 = grouped ? 0 : p.slot_base;          // this CTA's first workspace slot
  const int64_t grid_cap = static_cast<int64_t>(p.num_partitions - slot0) * P;
  if (L > grid_cap) {
    if (threadIdx.x == 0 && part == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
    L = static_cast<int>(grid_cap);
  }
  const int start = part * P;
  if (L == 0) {
    if (!grouped && part == 0 && shift == 0) {
      T* o = static_cast<T*>(p.out) + (static_cast<int64_t>(b) * p.Hq + g * G) * DH;
      for (int i = threadIdx.x; i < G * DH; i += THREADS) o[i] = Elem<T>::from_float(0.f);
    }
    return;
  }
  if (start >= L) return;
  const int end = static_cast<int>(
      min(static_cast<int64_t>(L), start + static_cast<int64_t>(P) * p.parts_per_cta));
  const int n_tiles = (end - start + TOK - 1) / TOK;
  // the output directly, or partials for the reduce (always for a group's span
  // and for a sequence whose first tokens its group served)
  const bool single = (L <= P) && !grouped && shift == 0;
  const int n_slots = min(p.parts_per_cta, (L + P - 1) / P - part);   // partials this CTA writes

  const int first_blk = start / bs;
  const int last_blk = (end + bs - 1) / bs;
  const int32_t* trow = p.block_tables + static_cast<int64_t>(b) * p.max_blocks + shift / bs;
  if (threadIdx.x == 0) {
    for (int s = 0; s < SLOTS; ++s) {
      mbar_init(&kr_full[s], 1);
      mbar_init(&kr_empty[s], 1);
      mbar_init(&vr_full[s], 1);
      mbar_init(&vr_empty[s], 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&s_full[j], 1);
      mbar_init(&s_free[j], 4);
    }
    for (int j = 0; j < PBUF; ++j) {
      mbar_init(&p_full[j], 4);
      mbar_init(&p_free[j], 1);
    }
    mbar_init(q_ready, 4);
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
    // ================= producer =================
    const uint32_t blk_bytes = static_cast<uint32_t>(bs) * DH;       // one (block, head) run
    const int bpt = TOK / bs;                 // blocks per tile (4, 8 or 16)
    bool ok = true;
    int issued = 0;                           // tiles whose K and V loads are out
    auto table = [&](int i) {                 // lane j: block j of tile i (read one tile ahead)
      const int b0 = first_blk + i * bpt;
      return (i < n_tiles && lane < min(bpt, last_blk - b0)) ? __ldg(trow + b0 + lane) : -1;
    };
    int pb_next = table(0);
    for (int i = 0; i < n_tiles; ++i) {
      const int b0 = first_blk + i * bpt;
      const int pb_l = pb_next;
      pb_next = table(i + 1);
      const int nbt = min(bpt, last_blk - b0);
      const bool mine_t = lane < nbt;
      const bool valid_t = mine_t && pb_l >= 0 && pb_l < p.num_blocks;
      if (mine_t && !valid_t) atomicOr(p.status, PA_DEVERR_TABLE);
      const unsigned vmask = __ballot_sync(FULL, valid_t);
      const int row = (pb_l * p.Hkv + g) * bs;
      const int s = i % SLOTS;
      // K, then V: the tile's blocks straight into the swizzled operands
      if (i >= SLOTS && !mbar_wait(&kr_empty[s], ((i / SLOTS) - 1) & 1, p.status)) ok = false;
      if (!__all_sync(FULL, ok)) break;
      if (lane == 0) mbar_arrive_expect_tx(&kr_full[s], __popc(vmask) * blk_bytes);
      __syncwarp();
      if (valid_t) tma_load_2d(kring + s * TILE_BYTES + lane * blk_bytes, &tmap_k, 0, row, &kr_full[s]);
      if (i >= SLOTS && !mbar_wait(&vr_empty[s], ((i / SLOTS) - 1) & 1, p.status)) ok = false;
      if (!__all_sync(FULL, ok)) {
        issued = -(i + 1);                    // K of tile i is out, V is not
        break;
      }
      if (lane == 0) mbar_arrive_expect_tx(&vr_full[s], __popc(vmask) * blk_bytes);
      __syncwarp();
      if (valid_t) tma_load_2d(vring + s * TILE_BYTES + lane * blk_bytes, &tmap_v, 0, row, &vr_full[s]);
      issued = i + 1;
    }
    if (!ok) {  // wait (bounded) for our own copies still in flight
      const int k_out = issued < 0 ? -issued : issued;
      const int v_out = issued < 0 ? -issued - 1 : issued;
      for (int i = k_out - SLOTS < 0 ? 0 : k_out - SLOTS; i < k_out; ++i)
        mbar_wait(&kr_full[i % SLOTS], (i / SLOTS) & 1, p.status);
      for (int i = v_out - SLOTS < 0 ? 0 : v_out - SLOTS; i < v_out; ++i)
        mbar_wait(&vr_full[i % SLOTS], (i / SLOTS) & 1, p.status);
    }
    return;
  }

  if (warp >= 2) {
    // Query terms: thread t covers column h = t / 8 (query row q0 + h / G,
    // head h % G) and its codes 16c..16c+15 (c = t % 8); a column's 8 threads
    // are consecutive lanes.  P buffers zeroed.
    const int t = threadIdx.x - 64;
    const int h = t >> 3, c = t & 7;
    float f[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) f[e] = 0.f;
    if (h < NC && h / G < Qb) {
      const T* src = static_cast<const T*>(p.q) +
                     ((static_cast<int64_t>(q0) + h / G) * p.Hq + g * G + h % G) * DH + c * 16;
      Elem<T>::unpack(__ldg(reinterpret_cast<const uint4*>(src)), f);
      Elem<T>::unpack(__ldg(reinterpret_cast<const uint4*>(src + 8)), f + 8);
    }
    float mx = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(f[e]));
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, off));
    int ex = 0;
    if (mx > 0.f) {
      const int be = static_cast<int>((__float_as_uint(mx) >> 23) & 0xffu);
      ex = 7 - (be == 0 ? -126 : be - 127);
      ex = max(-126, min(126, ex));
    }
    const float up = __uint_as_float(static_cast<uint32_t>(ex + 127) << 23);
    if (c == 0) qs[h] = __uint_as_float(static_cast<uint32_t>(127 - ex) << 23);
#pragma unroll
    for (int e = 0; e < 16; ++e) f[e] *= up;
    const uint32_t row_off = h * 128 + (((c ^ (h & 7)) & 7) << 4);
#pragma unroll
    for (int term = 0; term < NTERM; ++term) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t c01 = to_e4m3x2(f[4 * k], f[4 * k + 1]);
        const uint32_t c23 = to_e4m3x2(f[4 * k + 2], f[4 * k + 3]);
        const float2 v01 = from_e4m3x2(c01), v23 = from_e4m3x2(c23);
        f[4 * k] -= v01.x;        // what the next term takes (exact)
        f[4 * k + 1] -= v01.y;
        f[4 * k + 2] -= v23.x;
        f[4 * k + 3] -= v23.y;
        w[k] = c01 | (c23 << 16);
      }
      *reinterpret_cast<uint4*>(qop + term * QT_BYTES + row_off) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    for (int i = t; i < PBUF * PB_BYTES / 16; i += 128)
      reinterpret_cast<uint4*>(pop)[i] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(q_ready);
    named_sync(1, 128);   // qs[] visible to all softmax warps
  }

  if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      const uint32_t k_a = smem_addr(kring), v_a = smem_addr(vring);
      const uint32_t q_a = smem_addr(qop), p_a = smem_addr(pop);
      bool ok = true;
      auto issue_qk = [&](int i) -> bool {
        const int s = i % SLOTS;
        if (!mbar_wait(&kr_full[s], (i / SLOTS) & 1, p.status)) return false;
        if (i >= 2 && !mbar_wait(&s_free[i & 1], ((i >> 1) - 1) & 1, p.status)) return false;
        tc_fence_after();
        const uint32_t d = tmem + (i & 1) * NPAD;
#pragma unroll
        for (int term = 0; term < NTERM; ++term) {
#pragma unroll
          for (int k = 0; k < DH / 32; ++k) {   // 32 codes (32 bytes) per MMA
            const uint64_t a = smem_desc(k_a + s * TILE_BYTES + k * 32, 16, 1024);
            const uint64_t bq = smem_desc(q_a + term * QT_BYTES + k * 32, 16, 1024);
            mma_e4m3(d, a, bq, kIdescE4M3, (term > 0 || k > 0) ? 1u : 0u);
          }
        }
        mma_commit(&s_full[i & 1]);
        mma_commit(&kr_empty[s]);
        return true;
      };
      auto issue_pv = [&](int i) -> bool {
        const int s = i % SLOTS;
        if (!mbar_wait(&vr_full[s], (i / SLOTS) & 1, p.status)) return false;
        if (!mbar_wait(&p_full[i % PBUF], (i / PBUF) & 1, p.status)) return false;
        const bool first = i == 0;             // O starts at 0
        tc_fence_after();
        const uint32_t d = tmem + 2 * NPAD;
#pragma unroll
        for (int term = 0; term < PTERM; ++term) {
#pragma unroll
          for (int k = 0; k < TOK / 32; ++k) {  // 32 tokens per MMA: four 8-token groups
            const uint64_t a = smem_desc(v_a + s * TILE_BYTES + k * 4096, 1024, 1024);
            const uint64_t bp =
                smem_desc_plain(p_a + (i % PBUF) * PB_BYTES + term * PT_BYTES + k * 32 * NPAD, 128, 128);
            mma_e4m3(d, a, bp, kIdescE4M3_AMN_BMN, (!first || term > 0 || k > 0) ? 1u : 0u);
          }
        }
        mma_commit(&vr_empty[s]);
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
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    float m_run[NC], l_part[NC], sc[NC];
#pragma unroll
    for (int h = 0; h < NC; ++h) {
      m_run[h] = -INFINITY;
      l_part[h] = 0.f;
      sc[h] = p.scale_log2 * qs[h];
    }
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (ok) ok = mbar_wait(bar, parity, p.status);
      ok = __all_sync(FULL, ok);
      return ok;
    };
    // row r of O^T and the sums of the CTA's span, whose last tile is i
    auto flush = [&](int i) {
      wait(&p_free[i % PBUF], (i / PBUF) & 1);
      tc_fence_after();
      float o[16];
      tmem_ld16(tmem + lane_base + 2 * NPAD, o);
      tc_fence_before();
      __syncwarp();
#pragma unroll
      for (int h = 0; h < NC; ++h) {
        float x = l_part[h];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
        l_part[h] = x;
      }
      named_sync(1, 128);
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < NC; ++h) red[quad * NPAD + h] = l_part[h];
      }
      named_sync(1, 128);
      if (ok) {
        const float oscale = p.v_scale * P_DOWN;
#pragma unroll
        for (int h = 0; h < NC; ++h) {
          if (h / G >= Qb) continue;
          const float Ls = red[h] + red[NPAD + h] + red[2 * NPAD + h] + red[3 * NPAD + h];
          const float O = o[h] * oscale;
          const int64_t hq = (static_cast<int64_t>(q0) + h / G) * p.Hq + g * G + h % G;
          if (single) {
            static_cast<T*>(p.out)[hq * DH + r] = Elem<T>::from_float(O / Ls);
          } else {
            const int64_t slot = hq * p.num_partitions + slot0 + part;
            p.ws_o[slot * DH + r] = O;
            if (r == 0) {
              p.ws_m[slot] = m_run[h];
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
      float sv[16];
      if (wait(&s_full[i & 1], (i >> 1) & 1)) {
        tc_fence_after();
        tmem_ld16(tmem + lane_base + (i & 1) * NPAD, sv);
      } else {
#pragma unroll
        for (int h = 0; h < 16; ++h) sv[h] = 0.f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[i & 1]);
      float s[NC];
      bool need = false;
#pragma unroll
      for (int h = 0; h < NC; ++h) {
        s[h] = valid && h / G < Qb ? sv[h] * sc[h] : -INFINITY;
        need |= s[h] > m_run[h] + RESCALE_THRESHOLD;
      }
      if (bar_or(1, 128, need)) {
#pragma unroll
        for (int h = 0; h < NC; ++h) {
          float x = s[h];
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) x = fmaxf(x, __shfl_xor_sync(FULL, x, off));
          if (lane == 0) red[quad * NPAD + h] = x;
        }
        named_sync(1, 128);
        float alpha[NC];
#pragma unroll
        for (int h = 0; h < NC; ++h) {
          const float tmax =
              fmaxf(fmaxf(red[h], red[NPAD + h]), fmaxf(red[2 * NPAD + h], red[3 * NPAD + h]));
          const float mnew = fmaxf(m_run[h], tmax);
          alpha[h] = (m_run[h] == -INFINITY) ? 0.f : ex2_fast(m_run[h] - mnew);
          m_run[h] = mnew;
          l_part[h] *= alpha[h];
        }
        named_sync(1, 128);
        if (i > 0 && wait(&p_free[(i - 1) % PBUF], ((i - 1) / PBUF) & 1)) {
          tc_fence_after();
          float o[16];
          tmem_ld16(tmem + lane_base + 2 * NPAD, o);
#pragma unroll
          for (int h = 0; h < NC; ++h) o[h] *= alpha[h];
          tmem_st16(tmem + lane_base + 2 * NPAD, o);
        }
      }
      float pr[NC];
#pragma unroll
      for (int h = 0; h < NC; ++h) {
        pr[h] = s[h] != -INFINITY ? ex2_fast(s[h] - m_run[h]) : 0.f;
        l_part[h] += pr[h];
      }
      if (i >= PBUF) wait(&p_free[i % PBUF], ((i / PBUF) - 1) & 1);
      // P * 2^6 = P1 + P2, two E4M3 codes per head (heads h, h+1 in one pair);
      // token r's 16 head codes of each term are one 16-byte row of the
      // MN-major P^T operand (columns >= NC are 0)
      uint32_t w1[4] = {0u, 0u, 0u, 0u}, w2[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int h = 0; h < NC; h += 2) {
        const float x0 = pr[h] * P_UP;
        const float x1 = (h + 1 < NC) ? pr[h + 1] * P_UP : 0.f;
        const uint32_t c1 = to_e4m3x2(x0, x1);
        const float2 d1 = from_e4m3x2(c1);
        const uint32_t c2 = to_e4m3x2(x0 - d1.x, x1 - d1.y);
        w1[h >> 2] |= c1 << ((h & 2) * 8);
        w2[h >> 2] |= c2 << ((h & 2) * 8);
      }
      uint8_t* pb = pop + (i % PBUF) * PB_BYTES + r * NPAD;
      *reinterpret_cast<uint4*>(pb) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
      *reinterpret_cast<uint4*>(pb + PT_BYTES) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
      if (n_valid < TOK) {
        // the last tile: zero the V rows of tokens past the end, so that
        // whatever they hold (unused slots, stale data) adds 0 * 0 to O
        const int s_ = i % SLOTS;
        if (wait(&vr_full[s_], (i / SLOTS) & 1) && !valid) {
          uint4* row = reinterpret_cast<uint4*>(vring + s_ * TILE_BYTES + r * DH);
#pragma unroll
          for (int c = 0; c < 8; ++c) row[c] = make_uint4(0, 0, 0, 0);
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[i % PBUF]);
    }
    flush(n_tiles - 1);
  }

  // ---- teardown: warps 1-5 meet, warp 1 frees TMEM ----
  tc_fence_before();
  named_sync(2, 160);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

constexpr int kMaxSpan = 4096;   // tokens one CTA may stream through
constexpr int kStreamBelow = 2048;  // only partitions shorter than this are streamed

int sm_count8() {
  static int n = 0;
  if (n == 0) {
    int dev = 0, v = 0;
    n = (cudaGetDevice(&dev) == cudaSuccess &&
         cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            ? v
            : 148;
  }
  return n;
}

// Consecutive partitions per CTA: for partitions shorter than kStreamBelow
// tokens, the most of 8 / 4 / 2 that keeps a CTA's span within kMaxSpan tokens
// and still leaves at least 8 CTAs per SM (a tile of E4M3 codes is half the
// bytes of a 16-bit one, so a CTA streams longer before its fixed costs are
// paid back; two partitions of 2048 were slower than one).
// rows: CTAs along x and y; other_ctas: CTAs of a kernel running beside it
// (the rest of a grouped decode, for the groups' spans).
int tc8_parts_per_cta(int64_t rows, int partition_size, int n_parts, int64_t other_ctas) {
  if (partition_size >= kStreamBelow || n_parts <= 0) return 1;
  const int64_t want = 8ll * sm_count8();
  for (int c : {8, 4, 2}) {
    const int64_t ctas = rows * ((n_parts + c - 1) / c) + other_ctas;
    if (static_cast<int64_t>(partition_size) * c <= kMaxSpan && n_parts >= c && ctas >= want)
      return c;
  }
  return 1;
}

// NQ = 1: the decode, or the rest of every sequence past its shift (partials
// from a.slot_base).  NQ = 16 / G: the groups' shared spans, one CTA per
// (group, run of NQ members, kv head, run of span partitions), partials into
// slots [0, a.slot_base) of every member's row.
template <typename T, int G, int NQ>
cudaError_t launch_tc8_t(const DecodeArgs& a, unsigned int* status, cudaStream_t stream) {
  using Y = typename std::conditional<std::is_same<T, __nv_bfloat16>::value, LayBF16, LayF16>::type;
  constexpr int SMEM_BYTES = Y::SMEM_BYTES;
  constexpr bool grouped = NQ > 1;
  const int q_groups = grouped ? (a.max_group_size + NQ - 1) / NQ : 1;
  const int64_t xs = grouped ? static_cast<int64_t>(a.num_groups) * q_groups : a.num_seqs;
  const int n_parts = grouped ? a.slot_base : a.num_partitions - a.slot_base;
  int64_t other = 0;      // the rest's CTAs next to the spans: one per (sequence, head, partition)
  if (grouped) other = static_cast<int64_t>(a.num_seqs) * a.Hkv * (a.num_partitions - a.slot_base);
  const int ppc = tc8_parts_per_cta(xs * a.Hkv, a.partition_size, n_parts, other);
  auto kern = decode_partition_tc8_kernel<T, G, Y, NQ>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // each cache [NB][Hkv][bs][128] as rows of 128 codes; a box is the bs rows of
  // one (block, head), stored with the 128-byte swizzle
  CUtensorMap mk, mv;
  const int64_t rows = static_cast<int64_t>(a.num_blocks) * a.Hkv * a.block_size;
  const int64_t dims[2] = {DH, rows};
  const int64_t strides[1] = {DH};
  const int box[2] = {DH, a.block_size};
  if (!make_tmap(&mk, a.k_cache, 2, dims, strides, box, PA_FP8_E4M3) ||
      !make_tmap(&mv, a.v_cache, 2, dims, strides, box, PA_FP8_E4M3))
    return cudaErrorInvalidValue;
  Tc8Params p;
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
  p.scale_log2 = a.scale * 1.4426950408889634f * a.k_scale;
  p.v_scale = a.v_scale;
  p.seq_shift = a.seq_shift;
  p.group_start = grouped ? a.group_start : nullptr;
  p.slot_base = grouped ? 0 : a.slot_base;
  p.total_q = a.num_seqs;
  p.q_groups = q_groups;
  if (xs <= 0 || xs > 0x7fffffff) return cudaErrorInvalidValue;
  dim3 grid(static_cast<unsigned>(xs), a.Hkv, (n_parts + ppc - 1) / ppc);
  return launch_overlapped(kern, grid, dim3(THREADS), SMEM_BYTES, stream, p, mk, mv);
}

}  // namespace

bool decode_tc8_supported(const DecodeArgs& a) {
  const int G = a.Hq / a.Hkv;
  return a.kv_dtype == PA_FP8_E4M3 && (a.dtype == PA_F16 || a.dtype == PA_BF16) && a.D == DH &&
         (G == 4 || G == 8) && a.partition_size % TOK == 0 &&
         static_cast<int64_t>(a.num_blocks) * a.Hkv * a.block_size < (int64_t(1) << 31) &&
         tmap_available();
}

int launch_decode_partitions_tc8(const DecodeArgs& a, unsigned int* status, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = a.Hq / a.Hkv;
  if (a.dtype == PA_BF16) {
    return G == 8 ? launch_tc8_t<__nv_bfloat16, 8, 1>(a, status, st)
                  : launch_tc8_t<__nv_bfloat16, 4, 1>(a, status, st);
  }
  return G == 8 ? launch_tc8_t<__half, 8, 1>(a, status, st)
                : launch_tc8_t<__half, 4, 1>(a, status, st);
}

bool decode_group_tc8_supported(const DecodeArgs& a) {
  const int G = a.Hkv > 0 ? a.Hq / a.Hkv : 0;
  return a.kv_dtype == PA_FP8_E4M3 && (a.dtype == PA_F16 || a.dtype == PA_BF16) && a.D == DH &&
         (G == 1 || G == 2 || G == 4 || G == 8) && a.partition_size % TOK == 0 &&
         static_cast<int64_t>(a.num_blocks) * a.Hkv * a.block_size < (int64_t(1) << 31) &&
         tmap_available();
}

namespace {
// 8 / G members per span CTA when every family fits (half the softmax's
// per-column work; as in decode_tc.cu), else 16 / G
template <typename T, int G>
int launch_group8_g(const DecodeArgs& a, unsigned int* status, cudaStream_t stream) {
  if constexpr (G <= 4) {
    if (static_cast<int64_t>(a.max_group_size) * G <= 8)
      return launch_tc8_t<T, G, 8 / G>(a, status, stream);
  }
  return launch_tc8_t<T, G, 16 / G>(a, status, stream);
}
}  // namespace

int launch_decode_group_tc8(const DecodeArgs& a, unsigned int* status, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = a.Hq / a.Hkv;
  if (a.dtype == PA_BF16) {
    switch (G) {
      case 1: return launch_group8_g<__nv_bfloat16, 1>(a, status, st);
      case 2: return launch_group8_g<__nv_bfloat16, 2>(a, status, st);
      case 4: return launch_group8_g<__nv_bfloat16, 4>(a, status, st);
      default: return launch_group8_g<__nv_bfloat16, 8>(a, status, st);
    }
  }
  switch (G) {
    case 1: return launch_group8_g<__half, 1>(a, status, st);
    case 2: return launch_group8_g<__half, 2>(a, status, st);
    case 4: return launch_group8_g<__half, 4>(a, status, st);
    default: return launch_group8_g<__half, 8>(a, status, st);
  }
}

}  // namespace pa

// decode_tc8.cu -- paged decode attention on the tensor cores over an E4M3 KV
// cache, for grouped-query heads (G = Hq/Hkv in {4, 8}), head size 128, f16 or
// bf16 queries and outputs.
//
// What is computed is that of decode_tc.cu ("자기회귀 생성과 KV 캐시" and
// "PagedAttention의 설계", supersilo.blog vLLM summary), with the cache's
// elements standing for code * k_scale and code * v_scale (E4M3 codes: the
// reading of "quantization" in "4. 이 밖의 기법들", blog.aqudi.me).  Tokens are
// the MMA's M dimension:
//
//   S^T [128 tokens x 16] = K [128 x 128] . Q^T [128 x 16]     kind::f8f6f4
//   O^T [128 dims   x 16] += V^T [128 x 128] . P^T [128 x 16]   kind::f16
//
// * S: the K codes feed the tensor cores as they are, K-major, straight from
//   a TMA load per physical block (rows of 128 codes, 128-byte swizzle).  The
//   query is split into three E4M3 terms, Q * 2^e = Q1 + Q2 + Q3 (each the
//   nearest E4M3 value of what the previous terms left; e a per-head power of
//   two putting the head's largest |q| in [2^7, 2^8)), and S accumulates the
//   three products.  An f16 or bf16 query has at most 11 significant bits, and
//   each term takes the next 4, so the split is exact for every component at
//   least 2^-6 of the head's largest (smaller ones are off by under 2^-10 in
//   the scaled units); 2^-e and k_scale are folded into the softmax scale.
// * O: P keeps f16's range (the lazily raised running max can leave P far
//   below E4M3's smallest value), so V is widened to f16 (exact: every E4M3
//   value is an f16 value) by converter warps into the MN-major layout of V^T;
//   v_scale is applied to the output.
//
// Roles in a CTA of 10 warps, one CTA per (sequence, kv head, partition):
//   warp 0     producer: block-table lookups; per tile one TMA load per block
//              of its K codes into a ring of three 16 KB tiles, and one 1-D bulk
//              copy per block of its V codes into a ring of two 8 KB slots;
//   warp 1     TMEM owner and MMA issuer;
//   warps 2-5  query terms, then softmax (as in decode_tc.cu), P as f16;
//   warps 6-9  converters: a tile's V codes into registers (the slots go back
//              at once), then the f16 V^T tile, zeros for tokens past the end.
// About 111 KB of shared memory: two CTAs per SM.  Every wait is bounded;
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
constexpr int NTERM = 3;                    // E4M3 terms of the query
constexpr int KR_SLOTS = 3;
constexpr int KR_BYTES = TOK * DH;          // one tile of K codes: 16 KB
constexpr int HALF_TOK = 64;                // tokens per V staging slot
constexpr int ST_SLOTS = 2;
constexpr int ST_BYTES = HALF_TOK * DH;     // 8 KB of V codes
constexpr int VOP_BYTES = TOK * DH * 2;     // the f16 V^T tile: 32 KB
constexpr int GROUP_BYTES = 2048;           // f16 tile: 8 token rows, both 64-column halves
constexpr int HALF_OFF = 1024;
constexpr int QT_BYTES = NPAD * DH;         // one query term: 16 rows x 128 codes
constexpr int OPB_BYTES = 2 * NPAD * 128;   // f16 16-row operand (P): 4 KB
constexpr int OFF_KR = 0;
constexpr int OFF_VOP = OFF_KR + KR_SLOTS * KR_BYTES;
constexpr int OFF_ST = OFF_VOP + VOP_BYTES;
constexpr int OFF_Q = OFF_ST + ST_SLOTS * ST_BYTES;
constexpr int OFF_P = OFF_Q + NTERM * QT_BYTES;   // two P buffers
constexpr int OFF_BAR = OFF_P + 2 * OPB_BYTES;
constexpr int NBARS = 2 * KR_SLOTS + 2 * ST_SLOTS + 2 + 8 + 2;
constexpr int OFF_TMEM = (OFF_BAR + NBARS * 8 + 15) / 16 * 16;
constexpr int OFF_RED = OFF_TMEM + 16;      // 4 warps x 16 floats
constexpr int OFF_QS = OFF_RED + 4 * NPAD * 4;
constexpr int SMEM_USED = OFF_QS + NPAD * 4;
constexpr int SMEM_BYTES = SMEM_USED + 1024;
constexpr int THREADS = 320;
constexpr int TMEM_COLS = 64;               // S0 [0,16), S1 [16,32), O [32,48)
constexpr float RESCALE_THRESHOLD = 8.0f;

static_assert(SMEM_BYTES * 2 + 2048 <= 228 * 1024, "two CTAs per SM");
static_assert(OFF_VOP % 1024 == 0 && OFF_Q % 1024 == 0 && OFF_P % 1024 == 0 &&
                  QT_BYTES % 1024 == 0,
              "swizzled operands on 1 KB boundaries");

// Instruction descriptor of kind::f8f6f4: E4M3 x E4M3 (format 0 for both),
// fp32 accumulation, both operands K-major, M = 128, N = 16.
constexpr uint32_t kIdescE4M3 = (1u << 4) | (static_cast<uint32_t>(NPAD >> 3) << 17) |
                                (static_cast<uint32_t>(128 >> 4) << 24);

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
  const uint8_t* v_cache;
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
};

// Four E4M3 codes (one 32-bit word, code i in byte i) -> two f16x2 words
// (codes 0,1 and 2,3, lower code in the lower half), exactly.
__device__ __forceinline__ void widen4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

__device__ __forceinline__ void widen16(const uint4& c, uint4& lo, uint4& hi) {
  widen4(c.x, lo.x, lo.y);
  widen4(c.y, lo.z, lo.w);
  widen4(c.z, hi.x, hi.y);
  widen4(c.w, hi.z, hi.w);
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

template <typename T, int G, bool MULTI>
__global__ void __launch_bounds__(THREADS, 2)
    decode_partition_tc8_kernel(const Tc8Params p, const __grid_constant__ CUtensorMap tmap_k) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* kring = smem + OFF_KR;
  uint8_t* vop = smem + OFF_VOP;
  uint8_t* stage = smem + OFF_ST;
  uint8_t* qop = smem + OFF_Q;
  uint8_t* pop = smem + OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* kr_full = bars;                  // [KR_SLOTS]
  uint64_t* kr_empty = kr_full + KR_SLOTS;   // [KR_SLOTS]
  uint64_t* st_full = kr_empty + KR_SLOTS;   // [ST_SLOTS]
  uint64_t* st_empty = st_full + ST_SLOTS;   // [ST_SLOTS]
  uint64_t* vop_full = st_empty + ST_SLOTS;
  uint64_t* vop_empty = vop_full + 1;
  uint64_t* s_full = vop_empty + 1;          // [2]
  uint64_t* s_free = s_full + 2;             // [2]
  uint64_t* p_full = s_free + 2;             // [2]
  uint64_t* p_free = p_full + 2;             // [2]
  uint64_t* q_ready = p_free + 2;
  uint64_t* o_free = q_ready + 1;            // a partition's O has been read out
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_TMEM);
  float* red = reinterpret_cast<float*>(smem + OFF_RED);
  float* qs = reinterpret_cast<float*>(smem + OFF_QS);

  // a CTA streams parts_per_cta consecutive partitions (as in decode_tc.cu)
  const int b = blockIdx.x, g = blockIdx.y, part = MULTI ? blockIdx.z * p.parts_per_cta : blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  grid_dependency_wait();
  allow_dependents();
  int L = p.context_lens[b];
  const int P = p.partition_size;
  int64_t cap = p.max_blocks * p.block_size;
  const int64_t grid_cap = static_cast<int64_t>(p.num_partitions) * P;
  cap = cap < grid_cap ? cap : grid_cap;
  if (L < 0 || L > cap) {
    if (threadIdx.x == 0 && part == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
    L = L < 0 ? 0 : static_cast<int>(cap);
  }
  const int start = part * P;
  if (L == 0) {
    if (part == 0) {
      T* o = static_cast<T*>(p.out) + (static_cast<int64_t>(b) * p.Hq + g * G) * DH;
      for (int i = threadIdx.x; i < G * DH; i += THREADS) o[i] = Elem<T>::from_float(0.f);
    }
    return;
  }
  if (start >= L) return;
  const int end = MULTI ? static_cast<int>(min(static_cast<int64_t>(L),
                                               start + static_cast<int64_t>(P) * p.parts_per_cta))
                        : min(L, start + P);
  const int n_tiles = (end - start + TOK - 1) / TOK;
  const int tpp = MULTI ? P / TOK : (1 << 30);                    // tiles per partition
  const bool single = (L <= P);

  const int bs = p.block_size;
  const int first_blk = start / bs;
  const int last_blk = (end + bs - 1) / bs;
  const int32_t* trow = p.block_tables + static_cast<int64_t>(b) * p.max_blocks;
  if (threadIdx.x == 0) {
    for (int s = 0; s < KR_SLOTS; ++s) {
      mbar_init(&kr_full[s], 1);
      mbar_init(&kr_empty[s], 1);
    }
    for (int s = 0; s < ST_SLOTS; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 4);
    }
    mbar_init(vop_full, 4);
    mbar_init(vop_empty, 1);
    for (int j = 0; j < 2; ++j) {
      mbar_init(&s_full[j], 1);
      mbar_init(&s_free[j], 4);
      mbar_init(&p_full[j], 4);
      mbar_init(&p_free[j], 1);
    }
    mbar_init(q_ready, 4);
    mbar_init(o_free, 4);
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)) : "memory");
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
    const int64_t blk_stride = static_cast<int64_t>(p.Hkv) * blk_bytes;
    const uint8_t* vbase = p.v_cache + static_cast<int64_t>(g) * blk_bytes;
    const int bpt = TOK / bs;                 // blocks per tile (4, 8 or 16)
    const int bph = HALF_TOK / bs;            // blocks per V staging slot (2, 4 or 8)
    bool ok = true;
    int k_issued = 0, v_issued = 0;
    auto table = [&](int i) {                 // lane j: block j of tile i (read one tile ahead)
      const int b0 = first_blk + i * bpt;
      return (i < n_tiles && lane < min(bpt, last_blk - b0)) ? __ldg(trow + b0 + lane) : -1;
    };
    int pb_next = table(0);
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int b0 = first_blk + i * bpt;
      const int pb_l = pb_next;
      pb_next = table(i + 1);
      const int nbt = min(bpt, last_blk - b0);
      const bool mine_t = lane < nbt;
      const bool valid_t = mine_t && pb_l >= 0 && pb_l < p.num_blocks;
      if (mine_t && !valid_t) atomicOr(p.status, PA_DEVERR_TABLE);
      // K: the tile's blocks straight into the swizzled K-major operand
      {
        const int s = i % KR_SLOTS;
        if (i >= KR_SLOTS && !mbar_wait(&kr_empty[s], ((i / KR_SLOTS) - 1) & 1, p.status)) {
          ok = false;
          break;
        }
        const unsigned vmask = __ballot_sync(FULL, valid_t);
        if (lane == 0) mbar_arrive_expect_tx(&kr_full[s], __popc(vmask) * blk_bytes);
        __syncwarp();
        if (valid_t)
          tma_load_2d(kring + s * KR_BYTES + lane * blk_bytes, &tmap_k, 0,
                      (pb_l * p.Hkv + g) * bs, &kr_full[s]);
        k_issued = i + 1;
      }
      // V: two staging slots of 64 tokens
      for (int hh = 0; hh < 2; ++hh) {
        const int u = 2 * i + hh;
        const int s = u % ST_SLOTS;
        if (u >= ST_SLOTS && !mbar_wait(&st_empty[s], ((u / ST_SLOTS) - 1) & 1, p.status)) {
          ok = false;
          break;
        }
        const int j0 = hh * bph;
        const int nb = max(0, min(bph, last_blk - (b0 + j0)));
        const int pb = __shfl_sync(FULL, pb_l, (j0 + (lane < bph ? lane : 0)) & 31);
        const bool valid = lane < nb && pb >= 0 && pb < p.num_blocks;
        const unsigned vmask = __ballot_sync(FULL, valid);
        if (lane == 0) mbar_arrive_expect_tx(&st_full[s], __popc(vmask) * blk_bytes);
        __syncwarp();
        if (valid)
          bulk_load(stage + s * ST_BYTES + lane * blk_bytes,
                    vbase + static_cast<int64_t>(pb) * blk_stride, blk_bytes, &st_full[s]);
        v_issued = u + 1;
      }
    }
    if (!ok) {  // wait (bounded) for our own copies still in flight
      for (int i = k_issued - KR_SLOTS < 0 ? 0 : k_issued - KR_SLOTS; i < k_issued; ++i)
        mbar_wait(&kr_full[i % KR_SLOTS], (i / KR_SLOTS) & 1, p.status);
      for (int u = v_issued - ST_SLOTS < 0 ? 0 : v_issued - ST_SLOTS; u < v_issued; ++u)
        mbar_wait(&st_full[u % ST_SLOTS], (u / ST_SLOTS) & 1, p.status);
    }
    return;
  }

  if (warp >= 6) {
    // ================= converters: V codes -> the f16 V^T operand =================
    const int ct = threadIdx.x - 192;         // 0..127
    const int c = ct & 7;                     // 16-code chunk of a 128-byte row
    const int r0 = ct >> 3;                   // 0..15
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (ok) ok = mbar_wait(bar, parity, p.status);
      ok = __all_sync(FULL, ok);
      return ok;
    };
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int n_valid = min(TOK, end - (start + i * TOK));
      uint4 cw[2][4];
      for (int hh = 0; hh < 2; ++hh) {
        const int u = 2 * i + hh;
        const int s = u % ST_SLOTS;
        if (!wait(&st_full[s], (u / ST_SLOTS) & 1)) break;
        const uint8_t* src = stage + s * ST_BYTES;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int rr = r0 + 16 * j;
          cw[hh][j] = (hh * HALF_TOK + rr < n_valid)
                          ? *reinterpret_cast<const uint4*>(src + rr * DH + c * 16)
                          : make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&st_empty[s]);
      }
      if (!ok) break;
      if (i >= 1 && !wait(vop_empty, (i - 1) & 1)) break;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int R = hh * HALF_TOK + r0 + 16 * j;     // token row within the tile
          uint4 lo, hi;
          widen16(cw[hh][j], lo, hi);                    // zero codes widen to +0
          const uint32_t rb = (R >> 3) * GROUP_BYTES + (R & 7) * 128;
          const int c0 = 2 * c, c1 = 2 * c + 1;          // 8-dim chunks of the f16 row
          *reinterpret_cast<uint4*>(vop + rb + (c0 >> 3) * HALF_OFF + (((c0 & 7) ^ (R & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(vop + rb + (c1 >> 3) * HALF_OFF + (((c1 & 7) ^ (R & 7)) << 4)) = hi;
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(vop_full);
    }
    return;
  }

  if (warp >= 2) {
    // Query terms: thread t covers head h = t / 8 and its codes 16c..16c+15
    // (c = t % 8); a head's 8 threads are consecutive lanes.  P buffers zeroed.
    const int t = threadIdx.x - 64;
    const int h = t >> 3, c = t & 7;
    float f[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) f[e] = 0.f;
    if (h < G) {
      const T* src =
          static_cast<const T*>(p.q) + (static_cast<int64_t>(b) * p.Hq + g * G + h) * DH + c * 16;
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
    for (int i = t; i < 2 * OPB_BYTES / 16; i += 128)
      reinterpret_cast<uint4*>(pop)[i] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(q_ready);
    named_sync(1, 128);   // qs[] visible to all softmax warps
  }

  if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      const uint32_t id_pv = instr_desc<__half>(true);
      const uint32_t k_a = smem_addr(kring), v_a = smem_addr(vop);
      const uint32_t q_a = smem_addr(qop), p_a = smem_addr(pop);
      bool ok = true;
      auto issue_qk = [&](int i) -> bool {
        const int s = i % KR_SLOTS;
        if (!mbar_wait(&kr_full[s], (i / KR_SLOTS) & 1, p.status)) return false;
        if (i >= 2 && !mbar_wait(&s_free[i & 1], ((i >> 1) - 1) & 1, p.status)) return false;
        tc_fence_after();
        const uint32_t d = tmem + (i & 1) * NPAD;
#pragma unroll
        for (int term = 0; term < NTERM; ++term) {
#pragma unroll
          for (int k = 0; k < DH / 32; ++k) {   // 32 codes (32 bytes) per MMA
            const uint64_t a = smem_desc(k_a + s * KR_BYTES + k * 32, 16, 1024);
            const uint64_t bq = smem_desc(q_a + term * QT_BYTES + k * 32, 16, 1024);
            mma_e4m3(d, a, bq, kIdescE4M3, (term > 0 || k > 0) ? 1u : 0u);
          }
        }
        mma_commit(&s_full[i & 1]);
        mma_commit(&kr_empty[s]);
        return true;
      };
      auto issue_pv = [&](int i) -> bool {
        if (!mbar_wait(vop_full, i & 1, p.status)) return false;
        if (!mbar_wait(&p_full[i & 1], (i >> 1) & 1, p.status)) return false;
        const bool first = (i % tpp) == 0;     // a partition starts: O restarts at 0
        if (MULTI && first && i > 0 && !mbar_wait(o_free, ((i / tpp) - 1) & 1, p.status)) return false;
        tc_fence_after();
        const uint32_t d = tmem + 2 * NPAD;
#pragma unroll
        for (int k = 0; k < TOK / 16; ++k) {
          const uint64_t a = smem_desc(v_a + k * 2 * GROUP_BYTES, HALF_OFF, GROUP_BYTES);
          const uint64_t bp =
              smem_desc(p_a + (i & 1) * OPB_BYTES + (k >> 2) * (NPAD * 128) + (k & 3) * 32, 16, 1024);
          mma_f16(d, a, bp, id_pv, (!first || k > 0) ? 1u : 0u);
        }
        mma_commit(vop_empty);
        mma_commit(&p_free[i & 1]);
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
    float m_run[G], l_part[G], sc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
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
    // row r of O^T and the sums of the partition ending at tile i
    auto flush = [&](int i) {
      wait(&p_free[i & 1], (i >> 1) & 1);
      tc_fence_after();
      float o[16];
      tmem_ld16(tmem + lane_base + 2 * NPAD, o);
      tc_fence_before();
      __syncwarp();
      if (MULTI && lane == 0) mbar_arrive(o_free);      // the next partition may reuse O
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float x = l_part[h];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
        l_part[h] = x;
      }
      named_sync(1, 128);
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) red[quad * NPAD + h] = l_part[h];
      }
      named_sync(1, 128);
      if (ok) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float Ls = red[h] + red[NPAD + h] + red[2 * NPAD + h] + red[3 * NPAD + h];
          const float O = o[h] * p.v_scale;
          const int64_t hq = static_cast<int64_t>(b) * p.Hq + g * G + h;
          if (single) {
            static_cast<T*>(p.out)[hq * DH + r] = Elem<T>::from_float(O / Ls);
          } else {
            const int64_t slot = hq * p.num_partitions + part + i / tpp;
            p.ws_o[slot * DH + r] = O;
            if (r == 0) {
              p.ws_m[slot] = m_run[h];
              p.ws_l[slot] = Ls;
            }
          }
        }
      }
    };
    for (int i = 0; i < n_tiles; ++i) {
      const int n_valid = min(TOK, end - (start + i * TOK));
      const bool valid = r < n_valid;
      const bool first = (i % tpp) == 0;
      if (MULTI && first && i > 0) {                    // a new partition: a new softmax
#pragma unroll
        for (int h = 0; h < G; ++h) {
          m_run[h] = -INFINITY;
          l_part[h] = 0.f;
        }
      }
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
      float s[G];
      bool need = false;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        s[h] = valid ? sv[h] * sc[h] : -INFINITY;
        need |= s[h] > m_run[h] + RESCALE_THRESHOLD;
      }
      if (bar_or(1, 128, need)) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float x = s[h];
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) x = fmaxf(x, __shfl_xor_sync(FULL, x, off));
          if (lane == 0) red[quad * NPAD + h] = x;
        }
        named_sync(1, 128);
        float alpha[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float tmax =
              fmaxf(fmaxf(red[h], red[NPAD + h]), fmaxf(red[2 * NPAD + h], red[3 * NPAD + h]));
          const float mnew = fmaxf(m_run[h], tmax);
          alpha[h] = (m_run[h] == -INFINITY) ? 0.f : exp2f(m_run[h] - mnew);
          m_run[h] = mnew;
          l_part[h] *= alpha[h];
        }
        named_sync(1, 128);
        if (!first && wait(&p_free[(i - 1) & 1], ((i - 1) >> 1) & 1)) {
          tc_fence_after();
          float o[16];
          tmem_ld16(tmem + lane_base + 2 * NPAD, o);
#pragma unroll
          for (int h = 0; h < G; ++h) o[h] *= alpha[h];
          tmem_st16(tmem + lane_base + 2 * NPAD, o);
        }
      }
      float pr[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        pr[h] = valid ? exp2f(s[h] - m_run[h]) : 0.f;
        l_part[h] += pr[h];
      }
      if (i >= 2) wait(&p_free[i & 1], ((i >> 1) - 1) & 1);
      uint8_t* pb = pop + (i & 1) * OPB_BYTES + (r >> 6) * (NPAD * 128);
#pragma unroll
      for (int h = 0; h < G; ++h)
        *reinterpret_cast<uint16_t*>(pb + sw128(h, r & 63)) = to_bits<__half>(pr[h]);
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[i & 1]);
      if (MULTI && (i + 1) % tpp == 0 && i + 1 < n_tiles) flush(i);   // a partition ends mid-CTA
    }
    flush(n_tiles - 1);                                       // the CTA's last partition
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

template <typename T, int G>
cudaError_t launch_tc8_t(const DecodeArgs& a, unsigned int* status, cudaStream_t stream) {
  const int ppc = tc_parts_per_cta(a);
  // one partition per CTA compiles without the partition-streaming logic
  auto kern = ppc > 1 ? decode_partition_tc8_kernel<T, G, true> : decode_partition_tc8_kernel<T, G, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // the K cache [NB][Hkv][bs][128] as rows of 128 codes; a box is the bs rows of
  // one (block, head), stored with the 128-byte swizzle
  CUtensorMap mk;
  const int64_t rows = static_cast<int64_t>(a.num_blocks) * a.Hkv * a.block_size;
  const int64_t dims[2] = {DH, rows};
  const int64_t strides[1] = {DH};
  const int box[2] = {DH, a.block_size};
  if (!make_tmap(&mk, a.k_cache, 2, dims, strides, box, PA_FP8_E4M3)) return cudaErrorInvalidValue;
  Tc8Params p;
  p.out = a.out;
  p.q = a.q;
  p.v_cache = static_cast<const uint8_t*>(a.v_cache);
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
  dim3 grid(a.num_seqs, a.Hkv, (a.num_partitions + p.parts_per_cta - 1) / p.parts_per_cta);
  return launch_overlapped(kern, grid, dim3(THREADS), SMEM_BYTES, stream, p, mk);
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
    return G == 8 ? launch_tc8_t<__nv_bfloat16, 8>(a, status, st)
                  : launch_tc8_t<__nv_bfloat16, 4>(a, status, st);
  }
  return G == 8 ? launch_tc8_t<__half, 8>(a, status, st) : launch_tc8_t<__half, 4>(a, status, st);
}

}  // namespace pa

// decode.cu -- paged decode attention for sm_100a: the split-K partition kernel
// and the partition-reduce kernel.
//
// What is computed ("자기회귀 생성과 KV 캐시" and "PagedAttention의 설계" of the
// supersilo.blog vLLM summary): for sequence b and query head h,
//   out[b][h] = sum_j softmax_j(scale * q[b][h] . K_b[j]) V_b[j],  j < context_lens[b],
// where K_b[j] / V_b[j] are fetched through the block table in logical order and
// one softmax spans all of the sequence's tokens: a running max m and sum l are
// carried across blocks inside a partition, and across partitions by the
// reduce kernel (never per-block softmaxes summed).  Unused slots of a last
// block are masked out and never reach the result.
//
// Design (B200):
//   * one CTA per (sequence, kv head, partition of P tokens); all G = Hq/Hkv
//     query heads of the kv head are served by the same CTA, so every K/V byte
//     is read from HBM once;
//   * warp 0 is the producer: it reads the block table (32 entries per
//     coalesced load) and moves each physical (block, kv head) K and V tile --
//     a contiguous bs*D run -- into shared memory with 1-D bulk copies on the
//     TMA engine, into a ring of S stages (32 KB in flight per CTA for 16-bit
//     caches, six CTAs per SM; 64 KB of E4M3 codes) tracked by mbarriers with
//     transaction counts;
//   * NCW consumer warps each own 8 tokens of a stage (16 for E4M3 codes at
//     G <= 2): q (pre-scaled by scale*log2 e, or raw f16 pairs over E4M3)
//     sits in registers, a lane owns one 16-byte chunk of a K/V row,
//     dot products are finished with a butterfly reduce-scatter across the lanes
//     of a row, softmax runs in base 2 on the warp's scores in shared memory,
//     and P.V accumulates in fp32 registers;
//   * at the end the consumer warps merge their (m, l, o) states; a sequence that
//     fits one partition gets its normalised output directly, otherwise the
//     partial (m, l, o) goes to the workspace for the reduce kernel.
//   Every mbarrier wait is bounded (pa_device.cuh); a block id outside the pool
//   is never dereferenced (the copy is skipped and PA_DEVERR_TABLE set).
//
// E4M3 caches ("quantization" in "4. 이 밖의 기법들", blog.aqudi.me): the K/V
// type TK is separate from the query/output type TQ.  A lane loads 16 codes (16
// bytes; 8 at G > 2); k_scale is folded into the score scale and v_scale into the partial
// output.  Every E4M3 value is an f16 value and the hardware converts a code
// pair to an f16x2 pair exactly.  With f16 queries the products q_e k_e and
// p v_e are then taken by the mixed-precision FMA (two f16 operands, an fp32
// addend and result: the product of two f16 values is exact in fp32, so this
// is fmaf of the widened operands without the widening); with bf16 or fp32
// queries the codes are widened to fp32 and the loops are those of the 16-bit
// caches.  Half the bytes per token means twice the tokens per stage (and
// twice the consumer warps) for the same bytes in flight.
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr unsigned FULL_MASK = 0xffffffffu;

constexpr int cmax(int a, int b) { return a > b ? a : b; }
constexpr int cmin(int a, int b) { return a < b ? a : b; }
constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }
constexpr float RESCALE_LOG2 = 8.0f;   // raise the running max past 2^8 growth

// 2^x by the hardware's approximate base-2 exponential (flushes subnormals).
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <typename T, int D, int G, int NCW, int BUDGET = 65536, int TPW_ = 8>
struct Cfg {
  static constexpr int ES = sizeof(T);
  // elements a lane loads at once: one 16-byte chunk (8 codes at G > 2, where
  // the query and output registers grow with G)
  static constexpr int EPL = ES == 1 ? (G <= 2 ? 16 : 8) : Elem<T>::EPL;
  static constexpr int LPR = D / EPL;          // lanes per K/V row
  static constexpr int RPW = 32 / LPR;         // rows a warp covers per iteration
  static constexpr int TOK = NCW * TPW_;       // tokens per stage (TPW_ per consumer warp)
  static constexpr int TPW = TOK / NCW;        // tokens per consumer warp per stage
  static constexpr int ITERS = TPW / RPW;
  static constexpr int ROW_BYTES = D * ES;
  static constexpr int TILE_BYTES = TOK * ROW_BYTES;  // K (or V) part of a stage
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int S = cmin(8, cmax(2, BUDGET / STAGE_BYTES));   // stages in flight
  static constexpr int NV = G * ITERS;         // partial dots per lane per stage
  static constexpr int NSM = G * TPW;          // scores per warp per stage
  static constexpr int NPASS = (NSM + 31) / 32;
  static constexpr int SC_BYTES = round_up(NCW * NSM * 4, 128);
  static constexpr int HDR_BYTES = 128 + SC_BYTES;
  static constexpr int SMEM = HDR_BYTES + S * STAGE_BYTES;
  static constexpr int THREADS = 32 * (NCW + 1);
  static constexpr int CB_STRIDE = D + 2;      // combine buffer row: o[D], m, l
  static_assert(LPR >= 1 && LPR <= 32 && (32 % LPR) == 0, "row must map onto a warp");
  static_assert(TPW % RPW == 0 && ITERS >= 1, "warp tokens must be whole iterations");
  static_assert(TPW <= 32 && (TPW & (TPW - 1)) == 0, "score segment must fit a warp");
  static_assert(NCW * G * CB_STRIDE * 4 <= S * STAGE_BYTES, "combine buffer must fit the stages");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(TOK % kStageTokens == 0 && TOK <= 256, "a stage is whole table words of blocks");
};

// (d0, d1) += (a0 * b0, a1 * b1) as one paired fp32 FMA (each half rounded
// as fmaf would round it).
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 d, {%0, %1};\n\t"
      "fma.rn.f32x2 d, a, b, d;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// fmaf(a, b, c) for f16 a, b (raw bits) and fp32 c: the mixed-precision FMA.
__device__ __forceinline__ float fma_h(uint16_t a, uint16_t b, float c) {
  float d;
  asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint16_t lo16(uint32_t x) { return static_cast<uint16_t>(x & 0xffffu); }
__device__ __forceinline__ uint16_t hi16(uint32_t x) { return static_cast<uint16_t>(x >> 16); }

// 16 E4M3 codes (one 16-byte chunk in shared memory) as 8 f16x2 pairs, code
// 2i in the low half of h[i].
__device__ __forceinline__ void codes_to_f16x2(const void* src, uint32_t* h) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>((w[i] >> (16 * j)) & 0xffffu), __NV_E4M3);
      h[2 * i + j] = static_cast<uint32_t>(r.x) | (static_cast<uint32_t>(r.y) << 16);
    }
  }
}

// EPL elements of a K/V row chunk in shared memory widened to fp32: 16 E4M3
// codes, or one 16-byte chunk of a 16/32-bit type.
template <typename TK, int EPL>
__device__ __forceinline__ void load_row(const TK* src, float* f) {
  if constexpr (sizeof(TK) == 1 && EPL == 16) {
    uint32_t h[8];
    codes_to_f16x2(src, h);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&h[i]));
      f[2 * i] = v.x;
      f[2 * i + 1] = v.y;
    }
  } else {
    static_assert(EPL == Elem<TK>::EPL, "one load of the element type");
    Elem<TK>::load(src, f);
  }
}

// q row chunk of EPL elements of TQ (global memory, read-only path) to fp32.
template <typename TQ, int EPL>
__device__ __forceinline__ void load_q(const TQ* src, float* f) {
  constexpr int PER = Elem<TQ>::EPL;  // elements of one 16-byte load
  static_assert(EPL % PER == 0, "q chunk must be whole 16-byte loads");
#pragma unroll
  for (int i = 0; i < EPL / PER; ++i) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(src + i * PER));
    Elem<TQ>::unpack(u, f + i * PER);
  }
}

// Butterfly reduce-scatter of N values over the lanes of a row (lane bits
// below LPR): each halving step keeps one half of the values and adds the
// partner's copy of it; once one value is left the remaining steps all-reduce.
template <int N, int OFF>
__device__ __forceinline__ void reduce_scatter(float* v, int lane) {
  if constexpr (OFF >= 1) {
    if constexpr (N >= 2) {
      constexpr int H = N / 2;
      const bool upper = (lane & OFF) != 0;
#pragma unroll
      for (int i = 0; i < H; ++i) {
        const float send = upper ? v[i] : v[i + H];
        const float keep = upper ? v[i + H] : v[i];
        v[i] = keep + __shfl_xor_sync(FULL_MASK, send, OFF);
      }
      reduce_scatter<H, OFF / 2>(v, lane);
    } else {
      v[0] += __shfl_xor_sync(FULL_MASK, v[0], OFF);
      reduce_scatter<1, OFF / 2>(v, lane);
    }
  }
}

// Index (in the original array) of v[0] after reduce_scatter<N, OFF>.
template <int N, int OFF>
__device__ __forceinline__ int reduce_scatter_base(int lane) {
  if constexpr (OFF >= 1 && N >= 2) {
    return ((lane & OFF) ? N / 2 : 0) + reduce_scatter_base<N / 2, OFF / 2>(lane);
  } else {
    return 0;
  }
}

struct PartitionParams {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* ws_o;  // [B][Hq][NP][D]
  float* ws_m;  // [B][Hq][NP]
  float* ws_l;  // [B][Hq][NP]
  unsigned int* status;
  int64_t max_blocks;
  int Hq, Hkv, num_blocks, block_size, partition_size, num_partitions;
  float scale_log2;  // scale * log2(e) (* k_scale for E4M3 caches)
  float v_scale;     // E4M3 caches: the value scale (1 otherwise, unused)
  // shared-prefix groups: seq_shift[b] leading tokens of sequence b are served
  // by its group (nullable = 0); this launch's partials start at slot_base
  const int32_t* seq_shift;
  int slot_base;
};

template <typename TQ, typename TK, int D, int G, int NCW, int BUDGET, int TPW_>
__global__ void __launch_bounds__(Cfg<TK, D, G, NCW, BUDGET, TPW_>::THREADS)
    decode_partition_kernel(const PartitionParams p) {
  using C = Cfg<TK, D, G, NCW, BUDGET, TPW_>;
  using E = Elem<TK>;
  using EQ = Elem<TQ>;
  constexpr bool kCoded = sizeof(TK) == 1;  // E4M3 codes
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + C::S;
  float* scores = reinterpret_cast<float*>(smem + 128);
  uint8_t* stages = smem + C::HDR_BYTES;

  const int b = blockIdx.x;
  const int g = blockIdx.y;
  const int part = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  grid_dependency_wait();   // the appended tokens of the previous kernel are in the cache
  allow_dependents();       // the reduce kernel may start launching
  // ---- this partition's token range (validated) ----
  int L = p.context_lens[b];
  const int P = p.partition_size;
  // longest context this launch can serve: the table row and the partition grid
  const int64_t cap = p.max_blocks * p.block_size;
  if (L < 0 || L > cap) {
    if (threadIdx.x == 0 && part == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
    L = L < 0 ? 0 : static_cast<int>(cap);
  }
  int shift = 0;           // leading tokens its group serves
  if (p.seq_shift != nullptr) {
    shift = p.seq_shift[b];
    if (shift < 0 || shift % p.block_size != 0 || shift > L) {
      if (threadIdx.x == 0 && part == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
      shift = 0;
    }
    L -= shift;
  }
  const int64_t grid_cap = static_cast<int64_t>(p.num_partitions - p.slot_base) * P;
  if (L > grid_cap) {
    if (threadIdx.x == 0 && part == 0 && g == 0) atomicOr(p.status, PA_DEVERR_CONTEXT);
    L = static_cast<int>(grid_cap);
  }
  const int start = part * P;
  if (L == 0) {
    if (part == 0 && shift == 0) {
      TQ* o = static_cast<TQ*>(p.out) + (static_cast<int64_t>(b) * p.Hq + g * G) * D;
      for (int i = threadIdx.x; i < G * D; i += C::THREADS) o[i] = EQ::from_float(0.f);
    }
    return;
  }
  if (start >= L) return;
  const int end = min(L, start + P);
  const int n_tiles = (end - start + C::TOK - 1) / C::TOK;
  const bool single = (L <= P) && shift == 0;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < C::S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ================= producer =================
    const int bs = p.block_size;
    const int bpt = C::TOK / bs;                      // blocks per stage
    const int first_blk = start / bs;
    const int last_blk = (end + bs - 1) / bs;         // exclusive
    const uint32_t blk_bytes = static_cast<uint32_t>(bs) * C::ROW_BYTES;
    const int64_t head_off = static_cast<int64_t>(g) * blk_bytes;
    const int64_t blk_stride = static_cast<int64_t>(p.Hkv) * blk_bytes;
    const int32_t* trow =
        p.block_tables + static_cast<int64_t>(b) * p.max_blocks + shift / p.block_size;
    const char* kbase = static_cast<const char*>(p.k_cache) + head_off;
    const char* vbase = static_cast<const char*>(p.v_cache) + head_off;
    int cached = -1;
    int issued = 0;
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      const int s = t % C::S;
      if (t >= C::S && !mbar_wait(&empty[s], ((t / C::S) - 1) & 1, p.status)) {
        ok = false;
        break;
      }
      const int rel = t * bpt;                        // block index within the partition
      if ((rel & 31) == 0) {
        const int lb = first_blk + rel + lane;
        cached = lb < last_blk ? __ldg(trow + lb) : -1;
      }
      const int nb = min(bpt, last_blk - (first_blk + rel));
      const int src_lane = (rel & 31) + (lane < nb ? lane : 0);
      const int pb = __shfl_sync(FULL_MASK, cached, src_lane);
      const bool mine = lane < nb;
      const bool valid = mine && pb >= 0 && pb < p.num_blocks;
      if (mine && !valid) atomicOr(p.status, PA_DEVERR_TABLE);
      const unsigned vmask = __ballot_sync(FULL_MASK, valid);
      if (lane == 0) mbar_arrive_expect_tx(&full[s], __popc(vmask) * 2u * blk_bytes);
      __syncwarp();
      if (valid) {
        uint8_t* kdst = stages + s * C::STAGE_BYTES + lane * blk_bytes;
        uint8_t* vdst = kdst + C::TILE_BYTES;
        const int64_t off = static_cast<int64_t>(pb) * blk_stride;
        bulk_load(kdst, kbase + off, blk_bytes, &full[s]);
        bulk_load(vdst, vbase + off, blk_bytes, &full[s]);
      }
      issued = t + 1;
    }
    if (!ok) {
      // a consumer stopped: wait (bounded) for our own copies still in flight
      for (int t = issued - C::S < 0 ? 0 : issued - C::S; t < issued; ++t)
        mbar_wait(&full[t % C::S], (t / C::S) & 1, p.status);
    }
    return;
  }

  // ================= consumers =================
  const int w = warp - 1;
  const int r = lane / C::LPR;      // row group within the warp
  const int c = lane % C::LPR;      // 16-byte chunk of the row this lane owns
  float* sc = scores + w * C::NSM;  // [G][TPW]

  // f16 queries over 16-code chunks keep q as raw f16x2 pairs (the scale is
  // applied to the finished dot); otherwise q is fp32, pre-scaled
  constexpr bool kMixed = kCoded && std::is_same<TQ, __half>::value && C::EPL == 16;
  constexpr int QW = kMixed ? C::EPL / 2 : 1;
  float qf[G][kMixed ? 1 : C::EPL];
  uint32_t qh[G][QW];
  {
    const TQ* qrow = static_cast<const TQ*>(p.q) + (static_cast<int64_t>(b) * p.Hq + g * G) * D;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      if constexpr (kMixed) {
#pragma unroll
        for (int i = 0; i < QW / 4; ++i) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(qrow + h * D + c * C::EPL) + i);
          qh[h][4 * i] = u.x;
          qh[h][4 * i + 1] = u.y;
          qh[h][4 * i + 2] = u.z;
          qh[h][4 * i + 3] = u.w;
        }
      } else {
        load_q<TQ, C::EPL>(qrow + h * D + c * C::EPL, qf[h]);
#pragma unroll
        for (int e = 0; e < C::EPL; ++e) qf[h][e] *= p.scale_log2;
      }
    }
  }
  float m[G], l[G], o[G][C::EPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < C::EPL; ++e) o[h][e] = 0.f;
  }

  bool ok = true;
  for (int t = 0; t < n_tiles; ++t) {
    const int s = t % C::S;
    if (!mbar_wait(&full[s], (t / C::S) & 1, p.status)) {
      ok = false;
      break;
    }
    const TK* Ks = reinterpret_cast<const TK*>(stages + s * C::STAGE_BYTES);
    const TK* Vs = reinterpret_cast<const TK*>(stages + s * C::STAGE_BYTES + C::TILE_BYTES);
    const int n_valid = min(C::TOK, end - (start + t * C::TOK));

    // ---- scores: partial dots over this lane's chunk, then across the row ----
    float part_dot[C::NV];
#pragma unroll
    for (int it = 0; it < C::ITERS; ++it) {
      const int row = w * C::TPW + it * C::RPW + r;
      if constexpr (kMixed) {
        uint32_t kh[C::EPL / 2];
        codes_to_f16x2(Ks + row * D + c * C::EPL, kh);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          // even and odd elements in two accumulators, as below
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int i = 0; i < C::EPL / 2; ++i) {
            a0 = fma_h(lo16(qh[h][i]), lo16(kh[i]), a0);
            a1 = fma_h(hi16(qh[h][i]), hi16(kh[i]), a1);
          }
          part_dot[h * C::ITERS + it] = (a0 + a1) * p.scale_log2;
        }
      } else {
        float kf[C::EPL];
        load_row<TK, C::EPL>(Ks + row * D + c * C::EPL, kf);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          // even and odd elements in the two halves of a paired FMA
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int e = 0; e < C::EPL; e += 2) fma2(a0, a1, qf[h][e], qf[h][e + 1], kf[e], kf[e + 1]);
          part_dot[h * C::ITERS + it] = a0 + a1;
        }
      }
    }
    reduce_scatter<C::NV, C::LPR / 2>(part_dot, lane);
    {
      constexpr int NF = C::NV >= C::LPR ? C::NV / C::LPR : 1;
      constexpr int REP = C::NV >= C::LPR ? 1 : C::LPR / C::NV;
      const int base = reduce_scatter_base<C::NV, C::LPR / 2>(lane);
      if ((c % REP) == 0) {
#pragma unroll
        for (int i = 0; i < NF; ++i) {
          const int idx = base + i;
          const int h = idx / C::ITERS;
          const int it = idx % C::ITERS;
          const int row_local = it * C::RPW + r;
          const bool valid = (w * C::TPW + row_local) < n_valid;
          sc[h * C::TPW + row_local] = valid ? part_dot[i] : -INFINITY;
        }
      }
    }
    __syncwarp();

    // ---- online softmax (base 2) over the warp's tokens, per head ----
    float sv[C::NPASS], seg[C::NPASS];
#pragma unroll
    for (int ps = 0; ps < C::NPASS; ++ps) {
      const int idx = ps * 32 + lane;
      sv[ps] = idx < C::NSM ? sc[idx] : -INFINITY;
      float x = sv[ps];
#pragma unroll
      for (int off = C::TPW / 2; off >= 1; off >>= 1) x = fmaxf(x, __shfl_xor_sync(FULL_MASK, x, off));
      seg[ps] = x;
    }
    // The running max is raised only when a score passes it by 2^8 (base 2),
    // so O is rarely rescaled; P <= 2^8 meanwhile.  tmax is the same in every
    // lane, so `raise` is warp-uniform.
    float mnew[G], alpha[G];
    bool raise = false;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float tmax = __shfl_sync(FULL_MASK, seg[(h * C::TPW) / 32], (h * C::TPW) % 32);
      const bool up = tmax > m[h] + RESCALE_LOG2;
      mnew[h] = up ? tmax : m[h];
      alpha[h] = !up ? 1.f : (m[h] == -INFINITY) ? 0.f : ex2_fast(m[h] - tmax);
      raise |= up;
    }
#pragma unroll
    for (int ps = 0; ps < C::NPASS; ++ps) {
      const int idx = ps * 32 + lane;
      const int hh = idx / C::TPW;
      float mh = -INFINITY;
#pragma unroll
      for (int h = 0; h < G; ++h) mh = (h == hh) ? mnew[h] : mh;
      const float pr = (sv[ps] == -INFINITY) ? 0.f : ex2_fast(sv[ps] - mh);
      if (idx < C::NSM) sc[idx] = pr;
      float x = pr;
#pragma unroll
      for (int off = C::TPW / 2; off >= 1; off >>= 1) x += __shfl_xor_sync(FULL_MASK, x, off);
      seg[ps] = x;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float tsum = __shfl_sync(FULL_MASK, seg[(h * C::TPW) / 32], (h * C::TPW) % 32);
      l[h] = l[h] * alpha[h] + tsum;
      m[h] = mnew[h];
      if (raise) {
#pragma unroll
        for (int e = 0; e < C::EPL; ++e) o[h][e] *= alpha[h];
      }
    }
    __syncwarp();

    // ---- P.V over the warp's valid rows ----
#pragma unroll
    for (int it = 0; it < C::ITERS; ++it) {
      const int row_local = it * C::RPW + r;
      const int row = w * C::TPW + row_local;
      if (row < n_valid) {
        if constexpr (kMixed) {
          // P rounded to f16 (as the tensor-core kernels round it to the
          // operand type), V exact
          uint32_t vh[C::EPL / 2];
          codes_to_f16x2(Vs + row * D + c * C::EPL, vh);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const uint16_t ph = __half_as_ushort(__float2half_rn(sc[h * C::TPW + row_local]));
#pragma unroll
            for (int i = 0; i < C::EPL / 2; ++i) {
              o[h][2 * i] = fma_h(ph, lo16(vh[i]), o[h][2 * i]);
              o[h][2 * i + 1] = fma_h(ph, hi16(vh[i]), o[h][2 * i + 1]);
            }
          }
        } else {
          float vf[C::EPL];
          load_row<TK, C::EPL>(Vs + row * D + c * C::EPL, vf);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float pr = sc[h * C::TPW + row_local];
#pragma unroll
            for (int e = 0; e < C::EPL; e += 2) fma2(o[h][e], o[h][e + 1], pr, pr, vf[e], vf[e + 1]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // ---- merge row groups of the warp, then the consumer warps ----
#pragma unroll
  for (int off = C::LPR; off < 32; off <<= 1) {
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < C::EPL; ++e) o[h][e] += __shfl_xor_sync(FULL_MASK, o[h][e], off);
  }
  named_sync(1, NCW * 32);  // every consumer is done with the stages
  float* cb = reinterpret_cast<float*>(stages);
  if (r == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < C::EPL; ++e) cb[(w * G + h) * C::CB_STRIDE + c * C::EPL + e] = o[h][e];
  }
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      cb[(w * G + h) * C::CB_STRIDE + D] = m[h];
      cb[(w * G + h) * C::CB_STRIDE + D + 1] = l[h];
    }
  }
  named_sync(1, NCW * 32);
  if (!ok) return;  // status already records the failure

  const int tid = threadIdx.x - 32;
  for (int idx = tid; idx < G * D; idx += NCW * 32) {
    const int h = idx / D;
    const int d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int ww = 0; ww < NCW; ++ww) M = fmaxf(M, cb[(ww * G + h) * C::CB_STRIDE + D]);
    float Ls = 0.f, O = 0.f;
#pragma unroll
    for (int ww = 0; ww < NCW; ++ww) {
      const float mw = cb[(ww * G + h) * C::CB_STRIDE + D];
      const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
      Ls = fmaf(cb[(ww * G + h) * C::CB_STRIDE + D + 1], f, Ls);
      O = fmaf(cb[(ww * G + h) * C::CB_STRIDE + d], f, O);
    }
    const int64_t hq = static_cast<int64_t>(b) * p.Hq + g * G + h;
    if constexpr (kCoded) O *= p.v_scale;
    if (single) {
      static_cast<TQ*>(p.out)[hq * D + d] = EQ::from_float(O / Ls);
    } else {
      const int64_t slot = hq * p.num_partitions + p.slot_base + part;
      p.ws_o[slot * D + d] = O;
      if (d == 0) {
        p.ws_m[slot] = M;
        p.ws_l[slot] = Ls;
      }
    }
  }
}

struct ReduceParams {
  void* out;
  const int32_t* context_lens;
  const float* ws_o;
  const float* ws_m;
  const float* ws_l;
  int64_t table_cap;  // tokens a block-table row holds (max_blocks * block_size), or INT64_MAX
  int num_seqs, Hq, partition_size, num_partitions;
  // shared-prefix groups: sequence b's first seq_shift[b] tokens were served
  // by its group, whose partials fill slots [0, ceil(shift / P)); the rest of
  // the sequence's partials start at slot_rest (nullable: no groups, 0)
  const int32_t* seq_shift;
  int slot_rest;
};

// One warp per (sequence, query head) with more than one partition:
// out = sum_p o_p 2^(m_p - M) / sum_p l_p 2^(m_p - M),  M = max_p m_p.
template <typename T, int D>
__global__ void __launch_bounds__(128) decode_reduce_kernel(const ReduceParams p) {
  using E = Elem<T>;
  constexpr int DPL = D / 32;  // dims per lane
  grid_dependency_wait();   // every partial of the partition kernel is written
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<int64_t>(p.num_seqs) * p.Hq) return;
  const int b = static_cast<int>(row / p.Hq);
  int L = p.context_lens[b];
  L = L < 0 ? 0 : L;
  // the partition kernels serve at most min(table row, partition grid) tokens
  // (longer contexts are flagged there); read only the partials they wrote
  if (L > p.table_cap) L = static_cast<int>(p.table_cap);
  int S = p.seq_shift ? p.seq_shift[b] : 0;   // tokens its group served
  if (S < 0 || S > L) S = 0;                  // flagged by the partition kernel
  const int P = p.partition_size;
  int64_t rest = L - S;
  const int64_t cap = static_cast<int64_t>(p.num_partitions - p.slot_rest) * P;
  if (rest > cap) rest = cap;
  const int np_a = (S + P - 1) / P;           // the group's partials of the shared span
  const int np = np_a + static_cast<int>((rest + P - 1) / P);
  if (S == 0 && np <= 1) return;  // written directly by the partition kernel
  // partial i of the row: the group's span first, then the rest of the sequence
  auto slot = [&](int i) { return i < np_a ? i : p.slot_rest + (i - np_a); };
  const int64_t base = row * p.num_partitions;
  float M = -INFINITY;
  for (int i = lane; i < np; i += 32) M = fmaxf(M, p.ws_m[base + slot(i)]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL_MASK, M, off));
  float Ls = 0.f;
  for (int i = lane; i < np; i += 32)
    Ls += p.ws_l[base + slot(i)] * exp2f(p.ws_m[base + slot(i)] - M);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) Ls += __shfl_xor_sync(FULL_MASK, Ls, off);
  // The weighted outputs, in partition order.  Only partials with a finite
  // max carry weight: a CTA that streamed several partitions left empty ones
  // (max -inf, sum 0, output 0) in the other slots of its span, whose terms
  // would add exactly 0, so they are skipped and their outputs never read.
  // A warp takes 32 slots at a time, finds the live ones with a ballot and
  // loads up to four of them together.
  using V = typename std::conditional<DPL == 4, float4, float2>::type;
  static_assert(DPL == 4 || DPL == 2, "head size 128 or 64");
  float acc[DPL];
#pragma unroll
  for (int k = 0; k < DPL; ++k) acc[k] = 0.f;
  for (int i0 = 0; i0 < np; i0 += 32) {
    const int i = i0 + lane;
    const float mi = i < np ? p.ws_m[base + slot(i)] : -INFINITY;
    const float fi = exp2f(mi - M);
    unsigned live = __ballot_sync(FULL_MASK, mi != -INFINITY);
    while (live) {                      // warp-uniform
      int ks[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        ks[u] = live ? __ffs(live) - 1 : -1;
        live = live ? (live & (live - 1)) : 0u;
      }
      V v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (ks[u] >= 0)
          v[u] = *reinterpret_cast<const V*>(p.ws_o + (base + slot(i0 + ks[u])) * D + lane * DPL);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (ks[u] < 0) break;
        const float f = __shfl_sync(FULL_MASK, fi, ks[u]);
        const float* x = reinterpret_cast<const float*>(&v[u]);
#pragma unroll
        for (int k = 0; k < DPL; ++k) acc[k] = fmaf(f, x[k], acc[k]);
      }
    }
  }
  T* dst = static_cast<T*>(p.out) + row * D + lane * DPL;
  const float inv = 1.f / Ls;
#pragma unroll
  for (int k = 0; k < DPL; ++k) dst[k] = E::from_float(acc[k] * inv);
}

// Consumer warps: 4 (32-token stages); E4M3 caches with up to 2 query heads
// per kv head use 8 (64-token stages, the same bytes per stage).
template <typename TK, int G>
constexpr int consumer_warps() {
  return (sizeof(TK) == 1 && G <= 2) ? 8 : 4;
}

// Shared memory for the stages in flight: 32 KB for 16-bit and fp32 caches
// (two 16 KB stages at D = 128, so that six CTAs share an SM; against four
// stages and three CTAs, the same bytes in flight per SM but twice the
// independent pipelines: opt13b 0.94 -> 0.96, llama13b_ps' short per-sample
// rests 0.62 -> 0.68), 64 KB for E4M3 codes (its 288-thread CTAs are held to
// four per SM by registers anyway, and opt13b_fp8 measured 1.5 % slower).
template <typename TK>
constexpr int stage_budget() {
  return sizeof(TK) == 1 ? 65536 : 32768;
}

// Tokens per consumer warp per stage: 16 for E4M3 codes at G <= 2 (128-token
// stages of 32 KB, two in flight: each warp's fixed per-stage work -- the
// barrier waits, the scores' round trip through shared memory, the softmax
// shuffles -- is spread over twice the bytes; opt13b_fp8 0.765 -> 0.800), 8
// otherwise (16-bit caches keep two 16 KB stages and six CTAs per SM).
template <typename TK, int G>
constexpr int warp_tokens() {
  return (sizeof(TK) == 1 && G <= 2) ? 16 : 8;
}

template <typename TQ, typename TK, int D, int G, int BUDGET = stage_budget<TK>(), int TPW_ = 8>
cudaError_t launch_partition_t(const DecodeArgs& a, unsigned int* status, cudaStream_t stream) {
  constexpr int NCW = consumer_warps<TK, G>();
  using C = Cfg<TK, D, G, NCW, BUDGET, TPW_>;
  auto kern = decode_partition_kernel<TQ, TK, D, G, NCW, BUDGET, TPW_>;
  // opt in to > 48 KB of dynamic shared memory (idempotent, cheap)
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  PartitionParams p;
  p.out = a.out;
  p.q = a.q;
  p.k_cache = a.k_cache;
  p.v_cache = a.v_cache;
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  const int64_t rows = static_cast<int64_t>(a.num_seqs) * a.Hq * a.num_partitions;
  p.ws_o = a.workspace;
  p.ws_m = a.workspace ? a.workspace + rows * D : nullptr;
  p.ws_l = a.workspace ? a.workspace + rows * (D + 1) : nullptr;
  p.status = status;
  p.max_blocks = a.max_blocks;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.num_blocks = a.num_blocks;
  p.block_size = a.block_size;
  p.partition_size = a.partition_size;
  p.num_partitions = a.num_partitions;
  p.scale_log2 = a.scale * 1.4426950408889634f * a.k_scale;
  p.v_scale = a.v_scale;
  p.seq_shift = a.seq_shift;
  p.slot_base = a.slot_base;
  dim3 grid(a.num_seqs, a.Hkv, a.num_partitions - a.slot_base);
  return launch_overlapped(kern, grid, dim3(C::THREADS), C::SMEM, stream, p);
}

template <typename TQ, typename TK, int D>
cudaError_t launch_partition_g(const DecodeArgs& a, unsigned int* status, cudaStream_t stream) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_partition_t<TQ, TK, D, 1, stage_budget<TK>(), warp_tokens<TK, 1>()>(a, status, stream);
    case 2: return launch_partition_t<TQ, TK, D, 2, stage_budget<TK>(), warp_tokens<TK, 2>()>(a, status, stream);
    case 4: return launch_partition_t<TQ, TK, D, 4>(a, status, stream);
    case 8: return launch_partition_t<TQ, TK, D, 8>(a, status, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename TQ, typename TK>
cudaError_t launch_partition_d(const DecodeArgs& a, unsigned int* status, cudaStream_t stream) {
  switch (a.D) {
    case 64: return launch_partition_g<TQ, TK, 64>(a, status, stream);
    case 128: return launch_partition_g<TQ, TK, 128>(a, status, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename TQ>
cudaError_t launch_partition_kv(const DecodeArgs& a, unsigned int* status, cudaStream_t stream) {
  if (a.kv_dtype == PA_FP8_E4M3) return launch_partition_d<TQ, __nv_fp8_e4m3>(a, status, stream);
  if (a.kv_dtype != a.dtype) return cudaErrorInvalidValue;
  return launch_partition_d<TQ, TQ>(a, status, stream);
}

template <typename T>
cudaError_t launch_reduce_t(const DecodeArgs& a, cudaStream_t stream) {
  ReduceParams p;
  p.out = a.out;
  p.context_lens = a.context_lens;
  const int64_t rows = static_cast<int64_t>(a.num_seqs) * a.Hq * a.num_partitions;
  p.ws_o = a.workspace;
  p.ws_m = a.workspace + rows * a.D;
  p.ws_l = a.workspace + rows * (a.D + 1);
  p.table_cap = a.max_blocks > 0 ? a.max_blocks * a.block_size : INT64_MAX;
  p.seq_shift = a.seq_shift;
  p.slot_rest = a.slot_base;
  p.num_seqs = a.num_seqs;
  p.Hq = a.Hq;
  p.partition_size = a.partition_size;
  p.num_partitions = a.num_partitions;
  const int64_t warps = static_cast<int64_t>(a.num_seqs) * a.Hq;
  const unsigned grid = static_cast<unsigned>((warps + 3) / 4);
  if (a.D == 64) return launch_overlapped(decode_reduce_kernel<T, 64>, dim3(grid), dim3(128), 0, stream, p);
  return launch_overlapped(decode_reduce_kernel<T, 128>, dim3(grid), dim3(128), 0, stream, p);
}

}  // namespace

int launch_decode_partitions(const DecodeArgs& a, unsigned int* status, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (a.dtype) {
    case PA_F32: return launch_partition_kv<float>(a, status, st);
    case PA_F16: return launch_partition_kv<__half>(a, status, st);
    case PA_BF16: return launch_partition_kv<__nv_bfloat16>(a, status, st);
    default: return cudaErrorInvalidValue;
  }
}

int launch_decode_reduce(const DecodeArgs& a, unsigned int* /*status*/, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (a.dtype) {
    case PA_F32: return launch_reduce_t<float>(a, st);
    case PA_F16: return launch_reduce_t<__half>(a, st);
    case PA_BF16: return launch_reduce_t<__nv_bfloat16>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pa

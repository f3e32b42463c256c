// pa_device.cuh -- device helpers: element unpacking, shared-memory barriers
// with bounded waits, 1-D bulk copies (TMA engine, no tensor map), and the
// device status bits.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pagedkv.h"

namespace pa {

// Give up an mbarrier wait after this long (a healthy pipeline waits microseconds).
constexpr unsigned long long kWaitTimeoutNs = 1000000000ull;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits for the phase of `bar` with the given parity to complete.  Bounded:
// after `limit_ns` (or 2^31 polls) it sets PA_DEVERR_TIMEOUT in *status and
// returns false, so a broken pipeline ends the kernel instead of hanging it.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned int* status,
                                          unsigned long long limit_ns = kWaitTimeoutNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1; i < 0x80000000u; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 127u) == 0 && global_ns() - t0 > limit_ns) break;
  }
  atomicOr(status, PA_DEVERR_TIMEOUT);
  return false;
}

// 1-D bulk copy global -> shared through the TMA engine; completion is
// signalled as transaction bytes on `bar`.  dst, src 16-byte aligned; bytes a
// multiple of 16.  The source is this GPU's own memory; no multicast.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Same with an L2 eviction-priority hint (a policy from createpolicy).
__device__ __forceinline__ void bulk_load_hint(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                               uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], "
      "%2, [%3], %4;" ::"r"(smem_addr(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Programmatic dependent launch: a kernel launched right after another on the
// same stream (with programmatic stream serialisation) may start before that
// one finishes; grid_dependency_wait() blocks until it has completed and its
// memory is visible (a no-op when there is no such dependency), and
// allow_dependents() lets the next kernel of the stream begin launching.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Named barrier over `nthreads` threads (a multiple of 32) with id `id` (1..15).
__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---- element types ----
// Elem<T>: a lane's load of EPL elements (one 16-byte chunk; 8 bytes for E4M3)
// widened to fp32 (load), unpack of a 16-byte chunk, and rounding fp32 to T.
template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int EPL = 4;
  __device__ __forceinline__ static void load(const void* p, float* f) {
    unpack(*reinterpret_cast<const uint4*>(p), f);
  }
  __device__ __forceinline__ static void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
  __device__ __forceinline__ static float from_float(float x) { return x; }
};

template <>
struct Elem<__half> {
  static constexpr int EPL = 8;
  __device__ __forceinline__ static void load(const void* p, float* f) {
    unpack(*reinterpret_cast<const uint4*>(p), f);
  }
  __device__ __forceinline__ static void unpack(const uint4& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h2 = *reinterpret_cast<const __half2*>(&w[i]);
      float2 v = __half22float2(h2);
      f[2 * i] = v.x;
      f[2 * i + 1] = v.y;
    }
  }
  __device__ __forceinline__ static __half from_float(float x) { return __float2half_rn(x); }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int EPL = 8;
  __device__ __forceinline__ static void load(const void* p, float* f) {
    unpack(*reinterpret_cast<const uint4*>(p), f);
  }
  __device__ __forceinline__ static void unpack(const uint4& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // a bfloat16 is the upper half of an fp32 bit pattern
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ static __nv_bfloat16 from_float(float x) {
    return __float2bfloat16_rn(x);
  }
};

// OCP E4M3 codes (a cache type only; the value is code * the cache's scale,
// applied by the caller).  Every E4M3 value is an fp16 value, so the hardware
// conversion to f16x2 and the widening to fp32 are exact.  Byte i of the
// loaded word becomes f[i].
template <>
struct Elem<__nv_fp8_e4m3> {
  static constexpr int EPL = 8;
  __device__ __forceinline__ static void load(const void* p, float* f) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const uint32_t w[2] = {u.x, u.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const __nv_fp8x2_storage_t pair =
            static_cast<__nv_fp8x2_storage_t>((w[i] >> (16 * j)) & 0xffffu);
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
        const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&hr));
        f[4 * i + 2 * j] = v.x;
        f[4 * i + 2 * j + 1] = v.y;
      }
    }
  }
};

}  // namespace pa

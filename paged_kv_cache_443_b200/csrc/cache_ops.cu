// cache_ops.cu -- KV-cache updates: the append of new tokens' K/V at their
// slots and the copy-on-write block copy.
//
// Append: "1. KV 캐시란" (hjr-study-book Day 3) -- every decode step stores the
// new token's K and V; the slot arithmetic (physical block * block_size +
// offset) is that of the block-table example of "4.2 PagedAttention의 접근".
// Copy-on-write: "블록 공유" (supersilo.blog) and section 3 of the blog.aqudi.me
// write-up -- a block shared by several sequences is copied before one writes.
// Swap: "적용 범위와 관련 연구" (supersilo.blog) -- when GPU memory is short a
// sequence's blocks move to CPU memory and back; the same copy kernel moves
// blocks between a device cache and a pinned host cache the GPU can address.
//
// Append and copy are pure data movement in 16-byte chunks: loads are coalesced along
// the source, stores along a D-element cache row (append) or a whole
// contiguous [Hkv][bs][D] block (copy).  Out-of-range slots or block ids are
// skipped and flagged in the status word, never dereferenced.
#include <cuda_runtime.h>

#include <cstdint>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

// One thread per 16-byte chunk of key/value [N][Hkv][D].
__global__ void __launch_bounds__(256)
    reshape_and_cache_kernel(const uint4* __restrict__ key, const uint4* __restrict__ value,
                             uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                             const int64_t* __restrict__ slot_mapping, int64_t total_chunks,
                             int Hkv, int chunks_per_row, int log2_bs, int64_t num_slots,
                             unsigned int* status) {
  allow_dependents();   // the decode kernels may start launching (they wait for us)
  const int64_t per_token = static_cast<int64_t>(Hkv) * chunks_per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total_chunks;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_token;
    const int64_t rem = i - t * per_token;  // h * chunks_per_row + chunk
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      atomicOr(status, PA_DEVERR_SLOT);
      continue;
    }
    const int64_t blk = slot >> log2_bs;
    const int64_t off = slot & ((1 << log2_bs) - 1);
    const int64_t h = rem / chunks_per_row;
    const int64_t chunk = rem - h * chunks_per_row;
    const int64_t dst = (((blk * Hkv + h) << log2_bs) + off) * chunks_per_row + chunk;
    k_cache[dst] = __ldg(key + i);
    v_cache[dst] = __ldg(value + i);
  }
}

// Append into E4M3 caches ("quantization" in "4. 이 밖의 기법들",
// blog.aqudi.me): one thread per 16 elements of key/value [N][Hkv][D] of type
// T; code = E4M3(x / scale) with the quotient correctly rounded in fp32 and the
// hardware conversion rounding to nearest-even, saturating at 448; one 16-byte
// store per cache.
template <typename T>
__global__ void __launch_bounds__(256)
    reshape_and_cache_fp8_kernel(const T* __restrict__ key, const T* __restrict__ value,
                                 uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                                 const int64_t* __restrict__ slot_mapping, int64_t total_chunks,
                                 int Hkv, int chunks_per_row, int log2_bs, int64_t num_slots,
                                 float k_scale, float v_scale, unsigned int* status) {
  allow_dependents();
  constexpr int PER = Elem<T>::EPL;  // elements per 16-byte load of T
  const int64_t per_token = static_cast<int64_t>(Hkv) * chunks_per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total_chunks;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_token;
    const int64_t rem = i - t * per_token;
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      atomicOr(status, PA_DEVERR_SLOT);
      continue;
    }
    float kf[16], vf[16];
#pragma unroll
    for (int j = 0; j < 16 / PER; ++j) {
      Elem<T>::unpack(__ldg(reinterpret_cast<const uint4*>(key + i * 16 + j * PER)), kf + j * PER);
      Elem<T>::unpack(__ldg(reinterpret_cast<const uint4*>(value + i * 16 + j * PER)), vf + j * PER);
    }
    uint32_t kw[4], vw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t kk = 0, vv = 0;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float2 kp = make_float2(__fdiv_rn(kf[4 * j + 2 * e], k_scale),
                                      __fdiv_rn(kf[4 * j + 2 * e + 1], k_scale));
        const float2 vp = make_float2(__fdiv_rn(vf[4 * j + 2 * e], v_scale),
                                      __fdiv_rn(vf[4 * j + 2 * e + 1], v_scale));
        kk |= static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(kp, __NV_SATFINITE, __NV_E4M3))
              << (16 * e);
        vv |= static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(vp, __NV_SATFINITE, __NV_E4M3))
              << (16 * e);
      }
      kw[j] = kk;
      vw[j] = vv;
    }
    const int64_t blk = slot >> log2_bs;
    const int64_t off = slot & ((1 << log2_bs) - 1);
    const int64_t h = rem / chunks_per_row;
    const int64_t chunk = rem - h * chunks_per_row;
    const int64_t dst = (((blk * Hkv + h) << log2_bs) + off) * chunks_per_row + chunk;
    k_cache[dst] = make_uint4(kw[0], kw[1], kw[2], kw[3]);
    v_cache[dst] = make_uint4(vw[0], vw[1], vw[2], vw[3]);
  }
}

// Block pairs[p][1] of the destination caches := block pairs[p][0] of the source
// caches.  The caches may be the same (copy-on-write) or live in different
// memories, e.g. device and pinned host (swap).  grid.y strides over pairs;
// grid.x * blockDim.x threads stride over one block.
__global__ void __launch_bounds__(256)
    copy_blocks_kernel(uint4* __restrict__ dst_k, uint4* __restrict__ dst_v,
                       const uint4* __restrict__ src_k, const uint4* __restrict__ src_v,
                       const int64_t* __restrict__ pairs, int num_pairs, int64_t chunks_per_block,
                       int64_t src_blocks, int64_t dst_blocks, unsigned int* status) {
  allow_dependents();
  for (int pr = blockIdx.y; pr < num_pairs; pr += gridDim.y) {
    const int64_t src = __ldg(pairs + 2 * pr);
    const int64_t dst = __ldg(pairs + 2 * pr + 1);
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
      if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(status, PA_DEVERR_PAIR);
      continue;
    }
    const uint4* ks = src_k + src * chunks_per_block;
    const uint4* vs = src_v + src * chunks_per_block;
    uint4* kd = dst_k + dst * chunks_per_block;
    uint4* vd = dst_v + dst * chunks_per_block;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < chunks_per_block;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      kd[i] = ks[i];
      vd[i] = vs[i];
    }
  }
}

int ilog2(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}

int num_sms() {
  static thread_local int cached_dev = -1, cached_sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev != cached_dev) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
      cached_sms = n;
    cached_dev = dev;
  }
  return cached_sms;
}

}  // namespace

int launch_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                             const int64_t* slot_mapping, int num_tokens, int Hkv, int D,
                             int block_size, int num_blocks, int esize, unsigned int* status,
                             void* stream) {
  const int chunks_per_row = D * esize / 16;
  const int64_t total = static_cast<int64_t>(num_tokens) * Hkv * chunks_per_row;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  reshape_and_cache_kernel<<<static_cast<unsigned>(blocks), threads, 0,
                             static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(key), static_cast<const uint4*>(value),
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), slot_mapping, total, Hkv,
      chunks_per_row, ilog2(block_size), static_cast<int64_t>(num_blocks) * block_size, status);
  return cudaGetLastError();
}

int launch_reshape_and_cache_fp8(const void* key, const void* value, void* k_cache,
                                 void* v_cache, const int64_t* slot_mapping, int num_tokens,
                                 int Hkv, int D, int block_size, int num_blocks, pa_dtype dtype,
                                 float k_scale, float v_scale, unsigned int* status,
                                 void* stream) {
  const int chunks_per_row = D / 16;  // 16 codes = 16 bytes per chunk
  const int64_t total = static_cast<int64_t>(num_tokens) * Hkv * chunks_per_row;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const dim3 grid(static_cast<unsigned>(blocks));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t slots = static_cast<int64_t>(num_blocks) * block_size;
  const int lb = ilog2(block_size);
  uint4* kc = static_cast<uint4*>(k_cache);
  uint4* vc = static_cast<uint4*>(v_cache);
  switch (dtype) {
    case PA_F32:
      reshape_and_cache_fp8_kernel<float><<<grid, threads, 0, st>>>(
          static_cast<const float*>(key), static_cast<const float*>(value), kc, vc, slot_mapping,
          total, Hkv, chunks_per_row, lb, slots, k_scale, v_scale, status);
      break;
    case PA_F16:
      reshape_and_cache_fp8_kernel<__half><<<grid, threads, 0, st>>>(
          static_cast<const __half*>(key), static_cast<const __half*>(value), kc, vc,
          slot_mapping, total, Hkv, chunks_per_row, lb, slots, k_scale, v_scale, status);
      break;
    case PA_BF16:
      reshape_and_cache_fp8_kernel<__nv_bfloat16><<<grid, threads, 0, st>>>(
          static_cast<const __nv_bfloat16*>(key), static_cast<const __nv_bfloat16*>(value), kc,
          vc, slot_mapping, total, Hkv, chunks_per_row, lb, slots, k_scale, v_scale, status);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

int launch_copy_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                       const int64_t* pairs, int num_pairs, int Hkv, int D, int block_size,
                       int src_blocks, int dst_blocks, int esize, unsigned int* status,
                       void* stream) {
  const int64_t chunks = static_cast<int64_t>(Hkv) * block_size * D * esize / 16;
  const int threads = 256;
  int64_t gx = (chunks + threads * 4 - 1) / (threads * 4);  // ~4 chunks per thread per cache
  if (gx < 1) gx = 1;
  if (gx > 1024) gx = 1024;
  const int gy = num_pairs < 65535 ? num_pairs : 65535;
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  copy_blocks_kernel<<<grid, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v), static_cast<const uint4*>(src_k),
      static_cast<const uint4*>(src_v), pairs, num_pairs, chunks, src_blocks, dst_blocks, status);
  return cudaGetLastError();
}

}  // namespace pa

// Slot-mapped KV write and copy-on-write block copy: bandwidth-bound scatter and copy kernels.
//
// pa_cache_write follows page "vllm" (cnblogs) section 2.2 Decode (each step stores the new
// token's K and V in the cache) with the token's place given by its block and offset ("PagedAttention
// 原理", "实现一个虚拟内存").  pa_copy_blocks is step 2 of the copy-on-write list ("PagedAttention原理",
// "解决COW"): copy the shared block's contents into the newly allocated block.
//
// Both move 16-byte vectors with consecutive threads on consecutive addresses.  One row (token,
// kv head) of d elements is d*e/16 vectors; a whole block of Hk*B*d elements is contiguous in the
// [n_blocks][Hk][B][d] layout, so a block copy is one long contiguous run per cache.
#include <cuda_runtime.h>

#include "pa_internal.h"

namespace {

constexpr int kThreads = 256;
constexpr int kVecPerThread = 4;  // independent 16-byte loads in flight per thread

// One thread per (token, kv head, 16-byte chunk) of key and of value.
__global__ void __launch_bounds__(kThreads) cache_write_kernel(uint4* __restrict__ kc, uint4* __restrict__ vc,
                                                               const uint4* __restrict__ key,
                                                               const uint4* __restrict__ value,
                                                               const int64_t* __restrict__ slot_mapping,
                                                               long long total, int Hk, int chunks, int B,
                                                               int n_blocks) {
  const long long per_token = static_cast<long long>(Hk) * chunks;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long n = i / per_token;
    const long long rest = i - n * per_token;  // kh * chunks + c
    const int64_t slot = __ldg(slot_mapping + n);
    if (slot < 0) continue;  // padding token
    const int64_t blk = slot / B, off = slot - blk * B;
    if (blk >= n_blocks) continue;
    const int kh = static_cast<int>(rest / chunks), c = static_cast<int>(rest - static_cast<long long>(kh) * chunks);
    const long long dst = ((blk * Hk + kh) * B + off) * chunks + c;
    const uint4 kv = __ldg(key + i), vv = __ldg(value + i);
    kc[dst] = kv;
    vc[dst] = vv;
  }
}

// Grid-stride over (pair, cache, vector) with several independent vectors per thread.
// With n_pairs_dev set, the pair count is read on the device (at most P).
__global__ void __launch_bounds__(kThreads) copy_blocks_kernel(uint4* __restrict__ kc, uint4* __restrict__ vc,
                                                               const int32_t* __restrict__ pairs, int P,
                                                               const int32_t* __restrict__ n_pairs_dev,
                                                               long long vec_per_block, int n_blocks) {
  if (n_pairs_dev) P = min(max(*n_pairs_dev, 0), P);
  const long long per_pair = 2 * vec_per_block;
  const long long total = per_pair * P;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x * kVecPerThread;
  for (long long base = (blockIdx.x * static_cast<long long>(blockDim.x)) * kVecPerThread + threadIdx.x;
       base < total; base += stride) {
    uint4 buf[kVecPerThread];
    long long dst_idx[kVecPerThread];
    uint4* dst_ptr[kVecPerThread];
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const long long i = base + static_cast<long long>(u) * blockDim.x;
      dst_ptr[u] = nullptr;
      if (i >= total) continue;
      const int p = static_cast<int>(i / per_pair);
      long long r = i - static_cast<long long>(p) * per_pair;
      uint4* cache = kc;
      if (r >= vec_per_block) {
        cache = vc;
        r -= vec_per_block;
      }
      const int src = __ldg(pairs + 2 * p), dst = __ldg(pairs + 2 * p + 1);
      if (src < 0 || src >= n_blocks || dst < 0 || dst >= n_blocks) continue;
      buf[u] = cache[static_cast<long long>(src) * vec_per_block + r];
      dst_idx[u] = static_cast<long long>(dst) * vec_per_block + r;
      dst_ptr[u] = cache;
    }
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u)
      if (dst_ptr[u]) dst_ptr[u][dst_idx[u]] = buf[u];
  }
}

// Whole-block copies between two pools with the same block layout (one of them usually pinned
// host memory, reached over the host link).  Eight independent 16-byte vectors per thread keep
// enough bytes in flight to cover the link's latency.
constexpr int kSwapVec = 8;

__global__ void __launch_bounds__(kThreads) swap_blocks_kernel(uint4* __restrict__ dk, uint4* __restrict__ dv,
                                                               const uint4* __restrict__ sk,
                                                               const uint4* __restrict__ sv,
                                                               const int32_t* __restrict__ pairs, int P,
                                                               long long vec_per_block, int n_dst, int n_src) {
  const long long per_pair = 2 * vec_per_block;
  const long long total = per_pair * P;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x * kSwapVec;
  for (long long base = (blockIdx.x * static_cast<long long>(blockDim.x)) * kSwapVec + threadIdx.x; base < total;
       base += stride) {
    uint4 buf[kSwapVec];
    uint4* dst_ptr[kSwapVec];
#pragma unroll
    for (int u = 0; u < kSwapVec; ++u) {
      const long long i = base + static_cast<long long>(u) * blockDim.x;
      dst_ptr[u] = nullptr;
      if (i >= total) continue;
      const int p = static_cast<int>(i / per_pair);
      long long r = i - static_cast<long long>(p) * per_pair;
      const bool is_v = r >= vec_per_block;
      if (is_v) r -= vec_per_block;
      const int src = __ldg(pairs + 2 * p), dst = __ldg(pairs + 2 * p + 1);
      if (src < 0 || src >= n_src || dst < 0 || dst >= n_dst) continue;
      buf[u] = (is_v ? sv : sk)[static_cast<long long>(src) * vec_per_block + r];
      dst_ptr[u] = (is_v ? dv : dk) + static_cast<long long>(dst) * vec_per_block + r;
    }
#pragma unroll
    for (int u = 0; u < kSwapVec; ++u)
      if (dst_ptr[u]) *dst_ptr[u] = buf[u];
  }
}

int grid_for(long long work_items, int per_block) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (work_items + per_block - 1) / per_block;
  const long long cap = static_cast<long long>(sms) * 8;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

pa_status check_common(const void* kc, const void* vc, int Hk, int d, int B, int n_blocks, pa_dtype dtype,
                       const char* who) {
  if (!kc || !vc) return pa::fail(PA_ERR_INVALID_ARG, "%s: null cache pointer", who);
  if (!pa::aligned16(kc) || !pa::aligned16(vc)) return pa::fail(PA_ERR_INVALID_ARG, "%s: caches must be 16-byte aligned", who);
  if (!pa::valid_dtype(dtype)) return pa::fail(PA_ERR_INVALID_ARG, "%s: unknown dtype %d", who, static_cast<int>(dtype));
  if (Hk <= 0 || d <= 0 || B <= 0 || n_blocks <= 0) return pa::fail(PA_ERR_INVALID_ARG, "%s: sizes must be positive", who);
  if ((static_cast<size_t>(d) * pa::elem_size(dtype)) % 16 != 0)
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: d * element size must be a multiple of 16 bytes", who);
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_cache_write(void* k_cache, void* v_cache, const void* key, const void* value,
                                    const int64_t* slot_mapping, int T, int Hk, int d, int B, int n_blocks,
                                    pa_dtype dtype, void* stream) {
  pa_status st = check_common(k_cache, v_cache, Hk, d, B, n_blocks, dtype, "pa_cache_write");
  if (st != PA_OK) return st;
  if (T < 0) return pa::fail(PA_ERR_INVALID_ARG, "pa_cache_write: T < 0");
  if (T == 0) return pa::ok();
  if (!key || !value || !slot_mapping) return pa::fail(PA_ERR_INVALID_ARG, "pa_cache_write: null input");
  if (!pa::aligned16(key) || !pa::aligned16(value)) return pa::fail(PA_ERR_INVALID_ARG, "pa_cache_write: key/value must be 16-byte aligned");
  const int chunks = static_cast<int>(static_cast<size_t>(d) * pa::elem_size(dtype) / 16);
  const long long total = static_cast<long long>(T) * Hk * chunks;
  cache_write_kernel<<<grid_for(total, kThreads), kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), static_cast<const uint4*>(key),
      static_cast<const uint4*>(value), slot_mapping, total, Hk, chunks, B, n_blocks);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_cache_write: launch failed: %s", cudaGetErrorString(e));
  return pa::ok();
}

extern "C" pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs, int P, int Hk, int d,
                                    int B, int n_blocks, pa_dtype dtype, void* stream) {
  pa_status st = check_common(k_cache, v_cache, Hk, d, B, n_blocks, dtype, "pa_copy_blocks");
  if (st != PA_OK) return st;
  if (P < 0) return pa::fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: P < 0");
  if (P == 0) return pa::ok();
  if (!pairs) return pa::fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: null pairs");
  const long long vec_per_block = static_cast<long long>(Hk) * B * d * static_cast<long long>(pa::elem_size(dtype)) / 16;
  const long long total = 2 * vec_per_block * P;
  copy_blocks_kernel<<<grid_for(total, kThreads * kVecPerThread), kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), pairs, P, nullptr, vec_per_block, n_blocks);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_copy_blocks: launch failed: %s", cudaGetErrorString(e));
  return pa::ok();
}

pa_status pa::copy_blocks_counted(void* k_cache, void* v_cache, const int32_t* pairs, const int32_t* n_pairs_dev,
                                  int max_pairs, int Hk, int d, int B, int n_blocks, pa_dtype dtype, void* stream) {
  pa_status st = check_common(k_cache, v_cache, Hk, d, B, n_blocks, dtype, "copy_blocks_counted");
  if (st != PA_OK) return st;
  if (max_pairs <= 0) return pa::ok();
  if (!pairs || !n_pairs_dev) return pa::fail(PA_ERR_INVALID_ARG, "copy_blocks_counted: null pairs");
  const long long vec_per_block = static_cast<long long>(Hk) * B * d * static_cast<long long>(pa::elem_size(dtype)) / 16;
  const long long total = 2 * vec_per_block * max_pairs;
  copy_blocks_kernel<<<grid_for(total, kThreads * kVecPerThread), kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), pairs, max_pairs, n_pairs_dev, vec_per_block,
      n_blocks);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "copy_blocks_counted: launch failed: %s", cudaGetErrorString(e));
  return pa::ok();
}

extern "C" pa_status pa_swap_blocks(void* dst_k, void* dst_v, int n_dst_blocks, const void* src_k, const void* src_v,
                                    int n_src_blocks, const int32_t* pairs, int P, int Hk, int d, int B,
                                    pa_dtype dtype, void* stream) {
  pa_status st = check_common(dst_k, dst_v, Hk, d, B, n_dst_blocks, dtype, "pa_swap_blocks");
  if (st != PA_OK) return st;
  if (!src_k || !src_v || !pa::aligned16(src_k) || !pa::aligned16(src_v) || n_src_blocks <= 0)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_swap_blocks: bad source pool");
  if (P < 0) return pa::fail(PA_ERR_INVALID_ARG, "pa_swap_blocks: P < 0");
  if (P == 0) return pa::ok();
  if (!pairs) return pa::fail(PA_ERR_INVALID_ARG, "pa_swap_blocks: null pairs");
  const long long vec_per_block = static_cast<long long>(Hk) * B * d * static_cast<long long>(pa::elem_size(dtype)) / 16;
  const long long total = 2 * vec_per_block * P;
  swap_blocks_kernel<<<grid_for(total, kThreads * kSwapVec), kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v), static_cast<const uint4*>(src_k),
      static_cast<const uint4*>(src_v), pairs, P, vec_per_block, n_dst_blocks, n_src_blocks);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_swap_blocks: launch failed: %s", cudaGetErrorString(e));
  return pa::ok();
}

// Slot-mapped KV write and copy-on-write block copy: bandwidth-bound scatter and copy kernels.
//
// pa_cache_write follows page "vllm" (cnblogs) section 2.2 Decode (each step stores the new
// token's K and V in the cache) with the token's place given by its block and offset ("PagedAttention
// 原理", "实现一个虚拟内存").  pa_copy_blocks is step 2 of the copy-on-write list ("PagedAttention原理",
// "解决COW"): copy the shared block's contents into the newly allocated block.
//
// Both move 16-byte vectors with consecutive threads on consecutive addresses.  One row (token,
// kv head) of d elements is d*e/16 vectors; a whole block of Hk*B*d elements is contiguous in the
// [n_blocks][Hk][B][d] layout, so a block copy is one long contiguous run per cache.  Each thread
// issues several independent loads before its stores, which is what keeps HBM busy here.
#include <cuda_runtime.h>

#include "pa_internal.h"

namespace {

constexpr int kThreads = 256;
constexpr int kWriteVec = 4;  // 16-byte vectors of key (and of value) in flight per lane
constexpr int kCopyVec = 8;   // 16-byte vectors in flight per thread of a block copy

// One warp per (new token, part of its rows): the token's slot is read once, then the lanes move
// their share of its Hk rows of key and of value (per_token = Hk * chunks vectors each; row kh goes
// to ((blk * Hk + kh) * B + off) * chunks), all loads of a round issued before its stores.  A
// token is split into `splits` parts of per_part vectors only when there are too few tokens to
// give every SM several warps (decode steps write one token per sequence).
__global__ void __launch_bounds__(kThreads) cache_write_kernel(uint4* __restrict__ kc, uint4* __restrict__ vc,
                                                               const uint4* __restrict__ key,
                                                               const uint4* __restrict__ value,
                                                               const int64_t* __restrict__ slot_mapping, int T,
                                                               int Hk, int chunks, int B, int n_blocks, int splits,
                                                               int per_part) {
  const int per_token = Hk * chunks;
  const int lane = threadIdx.x & 31;
  const long long items = static_cast<long long>(T) * splits;
  const long long n_warps = static_cast<long long>(gridDim.x) * (kThreads / 32);
  for (long long item = static_cast<long long>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5); item < items;
       item += n_warps) {
    const long long n = item / splits;
    const int part = static_cast<int>(item - n * splits);
    const int64_t slot = __ldg(slot_mapping + n);
    if (slot < 0) continue;  // padding token
    const int64_t blk = slot / B, off = slot - blk * B;
    if (blk >= n_blocks) continue;
    const uint4* ks = key + n * per_token;
    const uint4* vs = value + n * per_token;
    uint4* kd = kc + (blk * Hk * B + off) * chunks;
    uint4* vd = vc + (blk * Hk * B + off) * chunks;
    const int v_end = min(per_token, (part + 1) * per_part);
    for (int v0 = part * per_part; v0 < v_end; v0 += 32 * kWriteVec) {
      uint4 kb[kWriteVec], vb[kWriteVec];
#pragma unroll
      for (int u = 0; u < kWriteVec; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < v_end) {
          kb[u] = __ldg(ks + v);
          vb[u] = __ldg(vs + v);
        }
      }
#pragma unroll
      for (int u = 0; u < kWriteVec; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < v_end) {
          const int kh = v / chunks, c = v - kh * chunks;
          const long long o = static_cast<long long>(kh) * B * chunks + c;
          kd[o] = kb[u];
          vd[o] = vb[u];
        }
      }
    }
  }
}

// One CTA per (pair, cache) at a time: a block is one contiguous run of vec_per_block vectors in
// each cache, copied in rounds of kThreads * kCopyVec vectors with every load of a round in flight
// before its stores.  With n_pairs_dev set, the pair count is read on the device (at most P).
__global__ void __launch_bounds__(kThreads) copy_blocks_kernel(uint4* __restrict__ kc, uint4* __restrict__ vc,
                                                               const int32_t* __restrict__ pairs, int P,
                                                               const int32_t* __restrict__ n_pairs_dev,
                                                               long long vec_per_block, int n_blocks) {
  if (n_pairs_dev) P = min(max(*n_pairs_dev, 0), P);
  const long long items = 2LL * P;
  for (long long it = blockIdx.x; it < items; it += gridDim.x) {
    const int p = static_cast<int>(it >> 1);
    uint4* cache = (it & 1) ? vc : kc;
    const int src = __ldg(pairs + 2 * p), dst = __ldg(pairs + 2 * p + 1);
    if (src < 0 || src >= n_blocks || dst < 0 || dst >= n_blocks) continue;
    const uint4* sp = cache + static_cast<long long>(src) * vec_per_block;
    uint4* dp = cache + static_cast<long long>(dst) * vec_per_block;
    for (long long v0 = 0; v0 < vec_per_block; v0 += static_cast<long long>(kThreads) * kCopyVec) {
      uint4 b[kCopyVec];
#pragma unroll
      for (int u = 0; u < kCopyVec; ++u) {
        const long long v = v0 + u * kThreads + threadIdx.x;
        if (v < vec_per_block) b[u] = sp[v];
      }
#pragma unroll
      for (int u = 0; u < kCopyVec; ++u) {
        const long long v = v0 + u * kThreads + threadIdx.x;
        if (v < vec_per_block) dp[v] = b[u];
      }
    }
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

// Grid for a grid-stride loop over work_items, per_block of them per CTA and round: at most 8 CTAs
// per SM, and, when that takes several rounds, the smallest grid that needs the same number of
// rounds, so that every CTA does the same number (2048 block copies on 1184 CTAs would leave half
// of them idle for the second round; on 1024 CTAs each does two).
int grid_for(long long work_items, int per_block) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (work_items + per_block - 1) / per_block;
  const long long cap = static_cast<long long>(sms) * 8;
  if (want <= cap) return static_cast<int>(want < 1 ? 1 : want);
  const long long rounds = (want + cap - 1) / cap;
  return static_cast<int>((want + rounds - 1) / rounds);
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
  if (static_cast<long long>(Hk) * chunks > (1LL << 30))
    return pa::fail(PA_ERR_UNSUPPORTED, "pa_cache_write: Hk * d too large");
  // parts per token: enough warps for 32 per SM, each part a multiple of 32 vectors
  const int per_token = Hk * chunks;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (32LL * sms + T - 1) / T;
  const int max_splits = (per_token + 31) / 32;
  const int splits = static_cast<int>(want < 1 ? 1 : (want > max_splits ? max_splits : want));
  const int per_part = ((per_token + splits - 1) / splits + 31) / 32 * 32;
  cache_write_kernel<<<grid_for(static_cast<long long>(T) * splits, kThreads / 32), kThreads, 0,
                       static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), static_cast<const uint4*>(key),
      static_cast<const uint4*>(value), slot_mapping, T, Hk, chunks, B, n_blocks, splits, per_part);
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
  copy_blocks_kernel<<<grid_for(2LL * P, 1), kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
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
  copy_blocks_kernel<<<grid_for(2LL * max_pairs, 1), kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
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

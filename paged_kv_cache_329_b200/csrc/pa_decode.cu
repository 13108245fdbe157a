// Paged decode attention for sm_100a.
//
// What is computed ("PagedAttention原理", "为什么会有 KV cache", eq. o_t = softmax(q_t K^T/sqrt(d)) V,
// and "实现一个虚拟内存", eqs. K_j, V_j, A_ij, o_i): for each sequence and query head, the scores of
// the query against the c cached keys, their softmax, and the softmax-weighted sum of the cached
// values, where token t lives in physical block block_tables[s][t / B] at offset t % B.  The
// denominator of A_ij is a sum over blocks, so it is accumulated block by block with a running
// maximum (online softmax) and, across partitions of the context, merged by log-sum-exp.
//
// Design (one B200, HBM-bound: each cached token of each kv head is read once per step):
//   * Work unit = (sequence, kv head, partition of P tokens).  A plan kernel lists the units
//     (whole partitions first, then the tails); a persistent grid pulls them from an atomic
//     counter, so long and short sequences balance across the 148 SMs.
//   * Per CTA one producer warp streams 64-token tiles of K and V into shared memory with TMA
//     loads (one box per physical block holding all its 128-byte column panels, 128-byte
//     swizzle), into a ring of stages guarded by full/empty mbarriers.  The q rows of the unit's head group come in with
//     the first tile by a 1-D bulk copy.  Each block is located through the block table, so the
//     kernel never touches a slot past the sequence's length.
//   * Four consumer warps share every loaded tile across the g = H/Hk query heads of the group.
//     q.k: each group of L lanes covers one token row (one 16-byte chunk per lane, q for that
//     chunk held in registers), partial dot products are reduce-scattered across the L lanes so
//     each lane ends with whole scores.  Online softmax in fp32 (log2 domain), then p.V: the same
//     lanes own the same chunks of V and accumulate g output rows.
//   * At the end of a unit the four warps merge their (max, sum, accumulator) states in shared
//     memory in a fixed order, then write the final row (single-partition sequences) or the
//     partial state for the combine kernel.  All summation orders depend only on logical token
//     positions, so outputs do not change when blocks move to other physical ids.
//   * pa_decode_step puts a step's copy-on-write copies, slot writes and the plan into one
//     prologue kernel ahead of the decode grid ("PagedAttention原理", "解决COW": copy, then write,
//     then read), and pa_prefill hands its one-token sequences to these kernels (rows q_start[s]).
#include <atomic>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace {

using pa::ChunkTraits;

constexpr int kTileTokens = 64;     // tokens per pipeline stage
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kPlanThreads = 1024;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Workspace header words.
constexpr int kHdrCounter = 0;
constexpr int kHdrNumItems = 1;
constexpr int kHdrError = 2;
constexpr size_t kHdrBytes = 256;

enum : int { kFirst = 1, kLast = 2, kDone = 4, kSingle = 8 };

struct __align__(16) StageMeta {
  int s, kh, part, ntok, flags, orow, pad1, pad2;  // orow: the sequence's row of query and out
};

struct DecodeArgs {
  const void* q;
  void* out;
  int out_dtype;
  const int32_t* bt;
  const int32_t* lens;
  int S, H, Hk, max_blocks, n_blocks, B, P;
  int max_c;         // context lengths are clamped to this (max_context_len)
  float scale_log2;  // scale * log2(e)
  const int2* items;
  int* hdr;
  int* err;               // error word (the header's, or another call's when decode serves it)
  const int32_t* q_rows;  // row of query / out for sequence s (null: row s)
  float* part_o;
  float* part_m;
  float* part_l;
  int max_parts;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- workspace layout ---------------------------------------------------------------------------

struct WsLayout {
  size_t items, part_m, part_l, part_o, total;
};

WsLayout ws_layout(int S, int H, int Hk, int d, int max_parts) {
  WsLayout w;
  size_t off = kHdrBytes;
  w.items = off;
  off = align_up(off + sizeof(int2) * static_cast<size_t>(S) * Hk * max_parts, 256);
  w.part_m = off;
  off = align_up(off + sizeof(float) * static_cast<size_t>(S) * H * max_parts, 256);
  w.part_l = off;
  off = align_up(off + sizeof(float) * static_cast<size_t>(S) * H * max_parts, 256);
  w.part_o = off;
  off = align_up(off + sizeof(float) * static_cast<size_t>(S) * H * max_parts * d, 256);
  w.total = off;
  return w;
}

// ---- plan: list the work units -----------------------------------------------------------------
// Units are (sequence, kv head, partition); n_parts(s) = max(1, ceil(c / P)) and c = 0 still gets
// one unit, which writes zeros.  Units are listed longest first (by 64-token tiles, in at most
// kBuckets groups): every whole partition, then the last partitions from longest to shortest, so
// the persistent grid ends on short units.  Positions inside a group come from atomic cursors;
// the order of units does not change any result (each unit's arithmetic is independent of it, and
// partitions are merged in index order).
constexpr int kBuckets = 128;

__device__ __forceinline__ int tile_bucket(int ntok, int P) {
  const int tiles = (ntok + kTileTokens - 1) / kTileTokens;  // 0 .. P/64
  const int max_tiles = P / kTileTokens;
  const int nb = max_tiles < kBuckets ? max_tiles : kBuckets;
  return tiles <= 1 ? 0 : ((tiles - 1) * nb) / max_tiles;    // 0 .. nb-1, monotone in ntok
}

constexpr int kPlanCache = 4096;  // lengths kept in shared memory between the two passes

constexpr int kPlanLong = 1024;   // sequences whose whole-partition items a warp writes

struct PlanSmem {
  int count[kBuckets], cursor[kBuckets];
  int c_cache[kPlanCache];
  int2 long_seq[kPlanLong];
  int n_long;
};

// Lists the units of one decode launch into items[] and resets the workspace header; run by one
// whole CTA (any block size that is a multiple of 32).  Each bucket's start is an exclusive
// prefix sum over the buckets from the longest down, taken by the first warp; a thread per
// sequence then writes its items, except that a warp writes the whole-partition items of a
// sequence that has more than 32 of them.
__device__ __forceinline__ void build_plan(PlanSmem& sm, const int32_t* __restrict__ lens, int S, int Hk, int P,
                                           int max_c, int2* __restrict__ items, int* __restrict__ hdr,
                                           const int32_t* __restrict__ q_start = nullptr, int* err = nullptr) {
  // With q_start, only sequences with exactly one query token (q_start[s+1] - q_start[s] == 1) get
  // units (the others are some other kernel's), and a cut length is or-ed into *err instead of
  // resetting the header's error word.
  const int tid = threadIdx.x, nt = blockDim.x;
  const int nb = min(P / kTileTokens, kBuckets);
  for (int b = tid; b < kBuckets; b += nt) sm.count[b] = 0;
  __syncthreads();
  bool clamped = false;
  for (int s = tid; s < S; s += nt) {
    const bool mine = !q_start || q_start[s + 1] - q_start[s] == 1;
    const int raw = lens[s];
    clamped |= mine && raw > max_c;
    const int c = mine ? min(max(raw, 0), max_c) : -1;  // -1: not listed
    if (s < kPlanCache) sm.c_cache[s] = c;
    if (!mine) continue;
    const int f = max(1, (c + P - 1) / P) - 1;  // whole partitions before the last one
    if (f > 0) atomicAdd(&sm.count[nb - 1], f * Hk);
    atomicAdd(&sm.count[tile_bucket(c - f * P, P)], Hk);
  }
  __syncthreads();
  if (tid < 32) {
    // buckets nb-1, nb-2, ..., 0 in that order: lane l owns positions 4l .. 4l+3 of it
    constexpr int kPer = kBuckets / 32;
    int v[kPer], run = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int pos = tid * kPer + i;
      v[i] = pos < nb ? sm.count[nb - 1 - pos] : 0;
      run += v[i];
    }
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (tid >= o) incl += y;
    }
    int excl = incl - run;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int pos = tid * kPer + i;
      if (pos < nb) sm.cursor[nb - 1 - pos] = excl;
      excl += v[i];
    }
    if (tid == 31) {
      hdr[kHdrCounter] = 0;
      hdr[kHdrNumItems] = incl;
    }
  }
  if (tid == 0) sm.n_long = 0;
  __syncthreads();
  // A thread per sequence takes its places and writes its last-partition items; a sequence with
  // more than 32 whole-partition items leaves those to a warp (below).
  for (int s = tid; s < S; s += nt) {
    const int c = s < kPlanCache ? sm.c_cache[s]
                                 : ((!q_start || q_start[s + 1] - q_start[s] == 1) ? min(max(lens[s], 0), max_c) : -1);
    if (c < 0) continue;
    const int f = max(1, (c + P - 1) / P) - 1;
    if (f > 0) {
      const int base = atomicAdd(&sm.cursor[nb - 1], f * Hk);
      if (f * Hk <= 32 || s >= kPlanCache) {
        for (int i = 0; i < f * Hk; ++i) items[base + i] = make_int2(s, ((i % Hk) << 16) | (i / Hk));
      } else {
        const int k = atomicAdd(&sm.n_long, 1);
        if (k < kPlanLong) {
          sm.long_seq[k] = make_int2(s, base);
        } else {  // more long sequences than the list holds: this thread writes them itself
          atomicSub(&sm.n_long, 1);
          for (int i = 0; i < f * Hk; ++i) items[base + i] = make_int2(s, ((i % Hk) << 16) | (i / Hk));
        }
      }
    }
    const int base = atomicAdd(&sm.cursor[tile_bucket(c - f * P, P)], Hk);
    for (int kh = 0; kh < Hk; ++kh) items[base + kh] = make_int2(s, (kh << 16) | f);
  }
  __syncthreads();
  const int lane = tid & 31;
  for (int k = tid >> 5; k < sm.n_long; k += nt >> 5) {
    const int s = sm.long_seq[k].x, base = sm.long_seq[k].y;
    const int f = max(1, (sm.c_cache[s] + P - 1) / P) - 1;
    for (int i = lane; i < f * Hk; i += 32) items[base + i] = make_int2(s, ((i % Hk) << 16) | (i / Hk));
  }
  const int any_clamped = __syncthreads_or(clamped);
  if (tid == 0) {
    if (err) {
      if (any_clamped) atomicOr(err, pa::kErrBadLength);
    } else {
      hdr[kHdrError] = any_clamped ? pa::kErrBadLength : 0;
    }
  }
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ lens, int S, int Hk, int P,
                                                            int max_c, int2* __restrict__ items, int* __restrict__ hdr,
                                                            const int32_t* __restrict__ q_start, int* err) {
  // Let the decode grid start its set-up now; wait for earlier work on the stream (it may have
  // written the lengths) before reading anything.
  pa::grid_dependency_launch();
  pa::grid_dependency_wait();
  __shared__ PlanSmem sm;
  build_plan(sm, lens, S, Hk, P, max_c, items, hdr, q_start, err);
}

// ---- step prologue: copy-on-write copies, slot writes and the plan in one launch ---------------
// "解决COW" orders a shared block's copy before the write into the copy, and the decode reads the
// cache after both.  CTA 0 builds the decode plan (it reads only the lengths).  Every other CTA
// takes copy pairs p = blockIdx.x - 1, ... in steps of gridDim.x - 1: it copies the pair's K and
// V block and then itself writes every new token whose slot lies in the destination block, so the
// write follows the copy within one CTA.  Tokens whose block is no copy destination are written by
// any CTA, one warp per token.  The decode kernels wait for this whole grid (griddepcontrol.wait).
constexpr int kPrologueThreads = 256;
using pa::kMaxStepPairs;

struct PrologueArgs {
  uint4* kc;
  uint4* vc;
  const uint4* key;
  const uint4* value;
  const int64_t* slots;
  const int32_t* pairs;
  const int32_t* n_pairs_dev;  // count on the device, or null: max_pairs
  int T, max_pairs, Hk, chunks, B, n_blocks;
  long long vec_per_block;     // 16-byte vectors per block and cache (Hk * B * d * e / 16)
};

// The rows of token n (slot = blk * B + off, blk in range) of key and value, by the given threads.
__device__ __forceinline__ void write_token(const PrologueArgs& w, int n, long long blk, int off, int t0, int nt) {
  const int per_token = w.Hk * w.chunks;
  const uint4* ks = w.key + static_cast<long long>(n) * per_token;
  const uint4* vs = w.value + static_cast<long long>(n) * per_token;
  uint4* kd = w.kc + (blk * w.Hk * w.B + off) * w.chunks;
  uint4* vd = w.vc + (blk * w.Hk * w.B + off) * w.chunks;
  for (int v0 = t0; v0 < per_token; v0 += 4 * nt) {
    uint4 kb[4], vb[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = v0 + u * nt;
      if (v < per_token) {
        kb[u] = __ldg(ks + v);
        vb[u] = __ldg(vs + v);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = v0 + u * nt;
      if (v < per_token) {
        const int kh = v / w.chunks, c = v - kh * w.chunks;
        const long long o = static_cast<long long>(kh) * w.B * w.chunks + c;
        kd[o] = kb[u];
        vd[o] = vb[u];
      }
    }
  }
}

__global__ void __launch_bounds__(kPrologueThreads) step_prologue_kernel(PrologueArgs w, const int32_t* __restrict__ lens,
                                                                         int S, int Hk, int P, int max_c,
                                                                         int2* __restrict__ items, int* __restrict__ hdr) {
  // The previous step's kernels may still read blocks this step overwrites (a freed block can be
  // a copy destination now), and its decode reads the workspace: wait for them before any write.
  pa::grid_dependency_wait();
  pa::grid_dependency_launch();
  __shared__ union {
    PlanSmem plan;
    int32_t dst[kMaxStepPairs];
  } sm;
  __shared__ int n_mine;
  __shared__ int mine[kPrologueThreads];
  if (blockIdx.x == 0) {
    build_plan(sm.plan, lens, S, Hk, P, max_c, items, hdr);
    return;
  }
  const int n_pairs = w.n_pairs_dev ? min(max(*w.n_pairs_dev, 0), w.max_pairs) : w.max_pairs;
  for (int i = threadIdx.x; i < n_pairs; i += blockDim.x) sm.dst[i] = __ldg(w.pairs + 2 * i + 1);
  __syncthreads();
  const int workers = gridDim.x - 1, wid = blockIdx.x - 1;
  // (a) block copies, each followed by the writes into its destination
  for (int p = wid; p < n_pairs; p += workers) {
    const int src = __ldg(w.pairs + 2 * p), dst = sm.dst[p];
    if (src >= 0 && src < w.n_blocks && dst >= 0 && dst < w.n_blocks) {
#pragma unroll 1
      for (int cache = 0; cache < 2; ++cache) {
        const uint4* sp = (cache ? w.vc : w.kc) + static_cast<long long>(src) * w.vec_per_block;
        uint4* dp = (cache ? w.vc : w.kc) + static_cast<long long>(dst) * w.vec_per_block;
        for (long long v0 = 0; v0 < w.vec_per_block; v0 += 8LL * kPrologueThreads) {
          uint4 b[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const long long v = v0 + u * kPrologueThreads + threadIdx.x;
            if (v < w.vec_per_block) b[u] = sp[v];
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const long long v = v0 + u * kPrologueThreads + threadIdx.x;
            if (v < w.vec_per_block) dp[v] = b[u];
          }
        }
      }
    }
    if (threadIdx.x == 0) n_mine = 0;
    __syncthreads();  // the copy is complete (and visible to the CTA) before the writes below
    for (int n = threadIdx.x; n < w.T; n += blockDim.x) {
      const int64_t slot = __ldg(w.slots + n);
      if (slot >= 0 && slot / w.B == dst) {
        const int k = atomicAdd(&n_mine, 1);
        if (k < kPrologueThreads) mine[k] = n;
      }
    }
    __syncthreads();
    const int cnt = min(n_mine, kPrologueThreads);
    if (dst >= 0 && dst < w.n_blocks) {
      for (int i = 0; i < cnt; ++i) {
        const int n = mine[i];
        const int64_t slot = __ldg(w.slots + n);
        write_token(w, n, slot / w.B, static_cast<int>(slot % w.B), threadIdx.x, blockDim.x);
      }
    }
    __syncthreads();
  }
  // (b) the other tokens, one warp each
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_warps = workers * (kPrologueThreads / 32);
  for (int n = wid * (kPrologueThreads / 32) + warp; n < w.T; n += n_warps) {
    const int64_t slot = __ldg(w.slots + n);
    if (slot < 0) continue;
    const int64_t blk = slot / w.B;
    if (blk >= w.n_blocks) continue;
    bool copied = false;
    for (int i = lane; i < n_pairs && !copied; i += 32) copied = sm.dst[i] == blk;
    if (__any_sync(0xffffffffu, copied)) continue;  // written by the CTA that copied its block
    write_token(w, n, blk, static_cast<int>(slot - blk * w.B), lane, 32);
  }
}

// ---- the decode kernel --------------------------------------------------------------------------

template <class T, int D, int G>
struct Cfg {
  static constexpr int kES = sizeof(T);
  static constexpr int kE = ChunkTraits<T>::kElems;          // elements per 16-byte chunk
  static constexpr int kCH = D / kE;                          // chunks per row
  static constexpr int kPanelElems = 128 / kES;               // elements per 128-byte panel row
  static constexpr int kNPanel = D / kPanelElems;             // panels per row
  static constexpr int kKVBytes = kTileTokens * D * kES;     // K (or V) tile
  static constexpr int kStageBytes = 2 * kKVBytes;
  static constexpr int kStages = kNPanel == 1 ? 6 : 3;
  static constexpr int kQBytes = G * D * kES;
  static constexpr int kQSlot = (kQBytes + 127) / 128 * 128;
  static constexpr int kL = kCH < 16 ? kCH : 16;              // lanes per token row
  static constexpr int kCPL = kCH / kL;                       // chunks per lane
  static constexpr int kNG = 32 / kL;                         // token groups per warp
  static constexpr int kR = (G >= 8 || kL < 16) ? 4 : 8;      // tokens per group per pass
  static constexpr int kTPW = kNG * kR;                       // tokens per warp per pass
  static constexpr int kPasses = kTileTokens / (kConsumerWarps * kTPW);
  static constexpr int kAcc = kCPL * kE;                      // accumulator floats per head per lane
  // shared memory carve-up (offsets from a 1024-byte aligned base)
  static constexpr int kOffQ = kStages * kStageBytes;
  static constexpr int kOffMeta = kOffQ + kStages * kQSlot;
  static constexpr int kOffBar = kOffMeta + kStages * static_cast<int>(sizeof(StageMeta));
  static constexpr int kOffML = (kOffBar + (2 * kStages + 1) * 8 + 127) / 128 * 128;
  static constexpr int kOffMerge = (kOffML + kConsumerWarps * G * 2 * 4 + 127) / 128 * 128;
  static constexpr int kSmemBytes = kOffMerge + 2 * G * D * 4 + 1024;  // + alignment slack
  static_assert(kPasses >= 1 && kTileTokens % (kConsumerWarps * kTPW) == 0, "tile/mapping mismatch");
  static_assert(kCH % kL == 0, "chunks must split evenly over lanes");
  static_assert(kQBytes % 16 == 0, "q rows must be whole 16-byte chunks");
};

// Shared-memory place of tile row t (0..63), 16-byte chunk c of a K or V tile.  A tile holds its
// 64/B blocks one after the other; each block is one TMA box of B rows laid out panel by panel
// (a panel = 128 bytes of every row, so d = 128 at 16 bits has 2 panels), and the 128-byte
// swizzle puts chunk c of row t at chunk (c % 8) ^ (t % 8) of its 128-byte line, which keeps the
// 8 rows that one ldmatrix phase reads on distinct banks.
struct TileAddr {
  int panel_stride;  // B * 128: from one panel of a block to the next
  int blk_extra;     // B * 128 * (panels - 1): what a block adds beyond its B rows of 128 bytes
  int log2b;
  __device__ __forceinline__ TileAddr(int B, int n_panel) {
    panel_stride = B * 128;
    blk_extra = B * 128 * (n_panel - 1);
    log2b = B == 8 ? 3 : (B == 16 ? 4 : 5);
  }
  __device__ __forceinline__ int row(int t) const { return t * 128 + (t >> log2b) * blk_extra; }
  __device__ __forceinline__ int chunk(int t, int c) const {
    return (c >> 3) * panel_stride + (((c & 7) ^ (t & 7)) << 4);
  }
};

// Reduce-scatter of partial dot products over the L lanes of a token group: at each level with
// N > 1 tokens, a lane keeps half of them and adds its partner's partials for that half; once a
// lane holds one token, the remaining levels add the partner's partial for the same token.
template <int G, int R, int MSK, int N>
__device__ __forceinline__ void reduce_scatter(float (&part)[G][R], int l) {
  if constexpr (MSK >= 1) {
    if constexpr (N > 1) {
      constexpr int HALF = N / 2;
      const bool up = (l & MSK) != 0;
#pragma unroll
      for (int j = 0; j < HALF; ++j)
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float send = up ? part[h][j] : part[h][j + HALF];
          const float keep = up ? part[h][j + HALF] : part[h][j];
          part[h][j] = keep + __shfl_xor_sync(0xffffffffu, send, MSK);
        }
      reduce_scatter<G, R, MSK / 2, HALF>(part, l);
    } else {
#pragma unroll
      for (int h = 0; h < G; ++h) part[h][0] += __shfl_xor_sync(0xffffffffu, part[h][0], MSK);
      reduce_scatter<G, R, MSK / 2, 1>(part, l);
    }
  }
}

// Token (0..R-1) whose score lane l of a group holds after reduce_scatter, and the inverse.
template <int L, int R>
__device__ __forceinline__ int token_of_lane(int l) {
  int t = 0, n = R;
#pragma unroll
  for (int msk = L / 2; msk >= 1; msk >>= 1)
    if (n > 1) {
      n >>= 1;
      if (l & msk) t += n;
    }
  return t;
}

template <int L, int R>
__device__ __forceinline__ int lane_of_token(int t) {
  int l = 0, n = R;
#pragma unroll
  for (int msk = L / 2; msk >= 1; msk >>= 1)
    if (n > 1) {
      n >>= 1;
      if (t & n) l |= msk;
    }
  return l;
}

// Lanes that hold a duplicate score (set bits at the all-reduce levels) do not add to the sum.
template <int L, int R>
__device__ __forceinline__ bool primary_lane(int l) {
  int n = R, dup = 0;
#pragma unroll
  for (int msk = L / 2; msk >= 1; msk >>= 1) {
    if (n > 1) n >>= 1;
    else dup |= msk;
  }
  return (l & dup) == 0;
}

template <class OutT, int D, int G, int AC, int L, int CPL, int E>
__device__ __forceinline__ void write_rows(OutT* base, const float (&acc)[G][AC], const float* mul, int l) {
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      float v[E];
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = acc[h][k * E + e] * mul[h];
      pa::store_floats<OutT, E>(base + static_cast<size_t>(h) * D + (k * L + l) * E, v);
    }
}


// ---- tensor-core consumers (16-bit caches) ---------------------------------------------------------
// Each consumer warp owns 16 token rows of every 64-token tile.  With tokens in M and the head group
// in N (g <= 8 heads, zero-padded to 8):
//   S^T[16 tok x 8 heads]  = K[16 tok x d] * Q^T[d x 8]          (d/16 mma.m16n8k16, K by ldmatrix)
//   O^T[d x 8 heads]      += V^T[d x 16 tok] * P^T[16 tok x 8]   (d/16 m-tiles, V by ldmatrix.trans)
// P^T comes from the S^T accumulator layout by an 8x8 register transpose (movmatrix) and is fed as a
// 16-bit pair hi + lo (hi = p rounded, lo = p - hi rounded), so the weights keep ~16 bits of
// precision; scores, maxima, sums and the output accumulate in fp32.  Tokens past the sequence's
// length get score -inf and their V elements are zeroed in registers (the shared tile may hold
// stale data or unused slots there).
template <class T, int D, int G, class C>
__device__ __forceinline__ void consume_mma(uint8_t* stages, uint8_t* qslots, StageMeta* meta, uint64_t* full,
                                            uint64_t* empty, uint64_t* epi, float* ml, float* merge,
                                            const DecodeArgs& a, int warp, int lane) {
  using M = pa::Mma<T>;
  constexpr int KS = D / 16;  // k-steps of q.k and m-tiles of p.V
  constexpr int NF4 = G * D / 4;
  constexpr int NMINE = (NF4 + kConsumerWarps * 32 - 1) / (kConsumerWarps * 32);
  const int gq = lane >> 2, tq = lane & 3;  // mma groupID / thread-in-group
  const int tid = warp * 32 + lane;
  uint32_t bq[KS][2];
  float acc[KS][4];
  float m_run[2], l_run[2];
#pragma unroll
  for (int k = 0; k < KS; ++k) {
    bq[k][0] = bq[k][1] = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[k][e] = 0.f;
  }
  m_run[0] = m_run[1] = -INFINITY;
  l_run[0] = l_run[1] = 0.f;

  int stage = 0;
  uint32_t phase = 0, epi_phase = 0;
  auto epi_sync = [&]() -> bool {
    pa::mbar_arrive(epi);
    const bool done = pa::mbar_wait(epi, epi_phase);
    epi_phase ^= 1;
    if (!done && lane == 0) atomicOr(a.err, pa::kErrWaitTimeout);
    return done;
  };
  // ldmatrix row/chunk assignment of this lane (tile index = lane / 8)
  const int ld_row = ((lane >> 3) & 1) * 8 + (lane & 7);      // q.k: tiles (tok 0-7, tok 8-15) x (lo, hi dims)
  const int ld_hi = lane >> 4;
  const int ldt_row = (lane >> 4) * 8 + (lane & 7);            // p.V: tiles (lo, hi dims) x (tok 0-7, tok 8-15)
  const int ldt_hi = (lane >> 3) & 1;
  const TileAddr ta(a.B, C::kNPanel);
  const int k_row = warp * 16 + ld_row, v_row = warp * 16 + ldt_row;
  const int k_row_off = ta.row(k_row), v_row_off = ta.row(v_row);

  while (true) {
    if (!pa::mbar_wait(&full[stage], phase)) {
      if (lane == 0) atomicOr(a.err, pa::kErrWaitTimeout);
      return;
    }
    const StageMeta mt = meta[stage];
    if (mt.flags & kDone) break;
    const uint8_t* ks = stages + stage * C::kStageBytes;
    const uint8_t* vs = ks + C::kKVBytes;
    const int ntok = mt.ntok;

    if (mt.flags & kFirst) {
      const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qslots + stage * C::kQSlot);
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        bq[k][0] = gq < G ? q32[(gq * D + k * 16 + 2 * tq) >> 1] : 0u;
        bq[k][1] = gq < G ? q32[(gq * D + k * 16 + 8 + 2 * tq) >> 1] : 0u;
      }
      m_run[0] = m_run[1] = -INFINITY;
      l_run[0] = l_run[1] = 0.f;
#pragma unroll
      for (int k = 0; k < KS; ++k)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[k][e] = 0.f;
    }

    const int r0 = warp * 16;
    if (r0 < ntok) {
      // ---- scores S^T = K Q^T ----
      float sacc[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t kbase = pa::smem_addr(ks);
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const int row = r0 + ld_row, c = 2 * k + ld_hi;
        uint32_t af[4];
        pa::ldsm_x4(af, kbase + k_row_off + ta.chunk(row, c));
        M::run(sacc, af, bq[k]);
      }
      // ---- online softmax; this lane holds tokens gq, gq+8 for heads 2tq, 2tq+1 ----
      const bool v0 = r0 + gq < ntok, v1 = r0 + gq + 8 < ntok;
      float x[4];
      x[0] = v0 ? sacc[0] * a.scale_log2 : -INFINITY;
      x[1] = v0 ? sacc[1] * a.scale_log2 : -INFINITY;
      x[2] = v1 ? sacc[2] * a.scale_log2 : -INFINITY;
      x[3] = v1 ? sacc[3] * a.scale_log2 : -INFINITY;
      float mx[2] = {fmaxf(x[0], x[2]), fmaxf(x[1], x[3])};
#pragma unroll
      for (int msk = 4; msk <= 16; msk <<= 1) {
        mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], msk));
        mx[1] = fmaxf(mx[1], __shfl_xor_sync(0xffffffffu, mx[1], msk));
      }
      float alpha[2], mn[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        mn[j] = fmaxf(m_run[j], mx[j]);
        alpha[j] = (mn[j] == -INFINITY) ? 1.f : exp2f(m_run[j] - mn[j]);
        m_run[j] = mn[j];
      }
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) p[e] = (mn[e & 1] == -INFINITY) ? 0.f : exp2f(x[e] - mn[e & 1]);
      l_run[0] = l_run[0] * alpha[0] + (p[0] + p[2]);
      l_run[1] = l_run[1] * alpha[1] + (p[1] + p[3]);
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        acc[k][0] *= alpha[0];
        acc[k][1] *= alpha[1];
        acc[k][2] *= alpha[0];
        acc[k][3] *= alpha[1];
      }
      // ---- P^T fragments (hi and lo parts) ----
      float r[4];
      const uint32_t h01 = M::pack(p[0], p[1], r[0], r[1]);
      const uint32_t h23 = M::pack(p[2], p[3], r[2], r[3]);
      float dummy0, dummy1;
      const uint32_t l01 = M::pack(p[0] - r[0], p[1] - r[1], dummy0, dummy1);
      const uint32_t l23 = M::pack(p[2] - r[2], p[3] - r[3], dummy0, dummy1);
      const uint32_t bh[2] = {pa::movmatrix_trans(h01), pa::movmatrix_trans(h23)};
      const uint32_t bl[2] = {pa::movmatrix_trans(l01), pa::movmatrix_trans(l23)};
      // ---- O^T += V^T P^T ----
      const bool partial = r0 + 16 > ntok;
      uint32_t mask01 = 0xffffffffu, mask23 = 0xffffffffu;
      if (partial) {
        const int t0 = r0 + 2 * tq;
        mask01 = (t0 < ntok ? 0x0000ffffu : 0u) | (t0 + 1 < ntok ? 0xffff0000u : 0u);
        mask23 = (t0 + 8 < ntok ? 0x0000ffffu : 0u) | (t0 + 9 < ntok ? 0xffff0000u : 0u);
      }
      const uint32_t vbase = pa::smem_addr(vs);
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const int row = r0 + ldt_row, c = 2 * k + ldt_hi;
        uint32_t af[4];
        pa::ldsm_x4_trans(af, vbase + v_row_off + ta.chunk(row, c));
        af[0] &= mask01;
        af[1] &= mask01;
        af[2] &= mask23;
        af[3] &= mask23;
        M::run(acc[k], af, bh);
        M::run(acc[k], af, bl);
      }
    }

    __syncwarp();
    if (lane == 0) pa::mbar_arrive(&empty[stage]);

    if (mt.flags & kLast) {
      // ---- merge the four warps in a fixed order: (w0 + w2) + (w1 + w3) ----
      float lsum[2] = {l_run[0], l_run[1]};
#pragma unroll
      for (int msk = 4; msk <= 16; msk <<= 1) {
        lsum[0] += __shfl_xor_sync(0xffffffffu, lsum[0], msk);
        lsum[1] += __shfl_xor_sync(0xffffffffu, lsum[1], msk);
      }
      if (gq == 0) {
#pragma unroll
        for (int j = 0; j < 2; ++j)
          if (2 * tq + j < G) {
            ml[(warp * G + 2 * tq + j) * 2] = m_run[j];
            ml[(warp * G + 2 * tq + j) * 2 + 1] = lsum[j];
          }
      }
      if (!epi_sync()) return;
      // weights of this warp's heads, and 1/den (or M, den) for the heads this thread writes out
      float wmine[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int h = 2 * tq + j;
        wmine[j] = 0.f;
        if (h < G) {
          float mxh = -INFINITY;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) mxh = fmaxf(mxh, ml[(w * G + h) * 2]);
          wmine[j] = (m_run[j] == -INFINITY) ? 0.f : exp2f(m_run[j] - mxh);
        }
      }
      float outM[NMINE], outDen[NMINE];
#pragma unroll
      for (int i = 0; i < NMINE; ++i) {
        const int f = tid + i * kConsumerWarps * 32;
        const int h = f < NF4 ? (f * 4) / D : 0;
        float mxh = -INFINITY, den = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) mxh = fmaxf(mxh, ml[(w * G + h) * 2]);
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float mw = ml[(w * G + h) * 2];
          if (mw != -INFINITY) den += exp2f(mw - mxh) * ml[(w * G + h) * 2 + 1];
        }
        outM[i] = mxh;
        outDen[i] = den;
      }
      // this thread's accumulator elements: dims 16k + gq (+8), heads 2tq, 2tq+1
      auto put = [&](float* buf, bool add) {
#pragma unroll
        for (int k = 0; k < KS; ++k)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int h = 2 * tq + (e & 1);
            if (h < G) {
              float* dst = buf + h * D + 16 * k + gq + (e >> 1) * 8;
              *dst = add ? *dst + acc[k][e] * wmine[e & 1] : acc[k][e] * wmine[e & 1];
            }
          }
      };
      if (warp >= 2) put(merge + (warp - 2) * G * D, false);
      if (!epi_sync()) return;
      if (warp < 2) put(merge + warp * G * D, true);
      if (!epi_sync()) return;
      const size_t row = static_cast<size_t>(mt.orow) * a.H + static_cast<size_t>(mt.kh) * G;   // out
      const size_t prow = static_cast<size_t>(mt.s) * a.H + static_cast<size_t>(mt.kh) * G;   // partials
#pragma unroll
      for (int i = 0; i < NMINE; ++i) {
        const int f = tid + i * kConsumerWarps * 32;
        if (f < NF4) {
          const int h = (f * 4) / D, dd = (f * 4) % D;
          const float4 x0 = *reinterpret_cast<const float4*>(merge + f * 4);
          const float4 x1 = *reinterpret_cast<const float4*>(merge + G * D + f * 4);
          float v[4] = {x0.x + x1.x, x0.y + x1.y, x0.z + x1.z, x0.w + x1.w};
          if (mt.flags & kSingle) {
            const float inv = outDen[i] > 0.f ? 1.f / outDen[i] : 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] *= inv;
            if (a.out_dtype == PA_F32)
              pa::store_floats<float, 4>(static_cast<float*>(a.out) + (row + h) * D + dd, v);
            else if (a.out_dtype == PA_F16)
              pa::store_floats<__half, 4>(static_cast<__half*>(a.out) + (row + h) * D + dd, v);
            else
              pa::store_floats<__nv_bfloat16, 4>(static_cast<__nv_bfloat16*>(a.out) + (row + h) * D + dd, v);
          } else {
            const size_t pidx = (prow + h) * a.max_parts + mt.part;
            pa::store_floats<float, 4>(a.part_o + pidx * D + dd, v);
            if (dd == 0) {
              a.part_m[pidx] = outM[i] == -INFINITY ? -INFINITY : outM[i] * kLn2;
              a.part_l[pidx] = outDen[i];
            }
          }
        }
      }
      m_run[0] = m_run[1] = -INFINITY;
      l_run[0] = l_run[1] = 0.f;
#pragma unroll
      for (int k = 0; k < KS; ++k)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[k][e] = 0.f;
    }

    if (++stage == C::kStages) {
      stage = 0;
      phase ^= 1;
    }
  }
}

template <class T, int D, int G, bool kMma>
__global__ void __launch_bounds__(kThreads) decode_kernel(const __grid_constant__ CUtensorMap tmK,
                                                          const __grid_constant__ CUtensorMap tmV,
                                                          const DecodeArgs a) {
  using C = Cfg<T, D, G>;
  constexpr int E = C::kE, L = C::kL, CPL = C::kCPL, R = C::kR, AC = C::kAcc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* qslots = smem + C::kOffQ;
  StageMeta* meta = reinterpret_cast<StageMeta*>(smem + C::kOffMeta);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + C::kStages;
  uint64_t* epi = empty + C::kStages;  // consumer-only barrier for the end-of-unit merge
  float* ml = reinterpret_cast<float*>(smem + C::kOffML);        // [warp][G][2] (max, sum)
  float* merge = reinterpret_cast<float*>(smem + C::kOffMerge);  // [2][G][D]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      pa::mbar_init(&full[i], 1);
      pa::mbar_init(&empty[i], kConsumerWarps);
    }
    pa::mbar_init(epi, kConsumerWarps * 32);
    pa::fence_barrier_init();
  }
  __syncthreads();
  // The plan kernel (and everything before it on the stream) must be complete from here on.
  pa::grid_dependency_wait();

  if (warp == kConsumerWarps) {
    // ================================ producer warp ==========================================
    if (lane == 0) {
      pa::prefetch_tmap(&tmK);
      pa::prefetch_tmap(&tmV);
    }
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;  // stages filled so far (for draining after a timeout)
    const int n_items = a.hdr[kHdrNumItems];
    bool ok = true;
    while (ok) {
      int k = 0;
      if (lane == 0) k = atomicAdd(a.hdr + kHdrCounter, 1);
      k = __shfl_sync(0xffffffffu, k, 0);
      if (k >= n_items) {
        if (lane == 0) pa::grid_dependency_launch();  // the combine grid may start launching
        if (!pa::mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
        if (lane == 0) {
          meta[stage].flags = kDone;
          pa::mbar_arrive(&full[stage]);
        }
        break;
      }
      const int2 it = a.items[k];
      const int s = it.x, kh = it.y >> 16, part = it.y & 0xffff;
      const int orow = a.q_rows ? a.q_rows[s] : s;
      const int c = min(max(a.lens[s], 0), a.max_c);
      const int n_parts = max(1, (c + a.P - 1) / a.P);
      const int t0 = part * a.P;
      const int t1 = min(t0 + a.P, c);
      const int ntok_item = max(t1 - t0, 0);
      const int ntiles = max(1, (ntok_item + kTileTokens - 1) / kTileTokens);
      const int32_t* bt_row = a.bt + static_cast<size_t>(s) * a.max_blocks;
      for (int tile = 0; tile < ntiles; ++tile) {
        if (!pa::mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
        const int tok0 = t0 + tile * kTileTokens;
        const int ntok = max(0, min(kTileTokens, t1 - tok0));
        const int nblk = (ntok + a.B - 1) / a.B;
        const int j0 = tok0 / a.B;
        int phys = -1;
        if (lane < nblk) {
          phys = __ldg(bt_row + j0 + lane);
          if (phys < 0 || phys >= a.n_blocks) {
            atomicOr(a.err, pa::kErrBadBlock);
            phys = -1;  // a fully out-of-range box: the TMA unit fills it with zeros
          }
        }
        const uint32_t bytes = static_cast<uint32_t>(nblk) * a.B * D * C::kES * 2u + (tile == 0 ? C::kQBytes : 0u);
        if (lane == 0) {
          StageMeta m;
          m.s = s;
          m.kh = kh;
          m.part = part;
          m.ntok = ntok;
          m.flags = (tile == 0 ? kFirst : 0) | (tile == ntiles - 1 ? kLast : 0) | (n_parts == 1 ? kSingle : 0);
          m.orow = orow;
          meta[stage] = m;
          pa::mbar_arrive_expect_tx(&full[stage], bytes);
        }
        __syncwarp();
        uint8_t* kdst = stages + stage * C::kStageBytes;
        uint8_t* vdst = kdst + C::kKVBytes;
        if (lane < nblk) {
          // one box per (block, K or V): B rows x every panel (a 3-D box when there are several)
          const int y = (phys * a.Hk + kh) * a.B;
          const int off = lane * a.B * D * C::kES;
          if constexpr (C::kNPanel == 1) {
            pa::tma_load_2d(kdst + off, &tmK, 0, y, &full[stage]);
            pa::tma_load_2d(vdst + off, &tmV, 0, y, &full[stage]);
          } else {
            pa::tma_load_3d(kdst + off, &tmK, 0, y, 0, &full[stage]);
            pa::tma_load_3d(vdst + off, &tmV, 0, y, 0, &full[stage]);
          }
        }
        if (tile == 0 && lane == 0) {
          const uint8_t* qsrc = static_cast<const uint8_t*>(a.q) +
                                (static_cast<size_t>(orow) * a.H + static_cast<size_t>(kh) * G) * D * C::kES;
          pa::bulk_load(qslots + stage * C::kQSlot, qsrc, C::kQBytes, &full[stage]);
        }
        ++issued;
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok) {
      if (lane == 0) atomicOr(a.err, pa::kErrWaitTimeout);
      // Let every copy this warp started land before the CTA can exit.
      int st = stage;
      uint32_t ph = phase;
      for (int i = 0; i < C::kStages && i < issued; ++i) {
        if (--st < 0) {
          st = C::kStages - 1;
          ph ^= 1;
        }
        pa::mbar_wait(&full[st], ph);
      }
    }
    return;
  }

  // ================================== consumer warps ============================================
  if constexpr (kMma) {
    consume_mma<T, D, G, C>(stages, qslots, meta, full, empty, epi, ml, merge, a, warp, lane);
  } else {
  const int grp = lane / L, l = lane % L;
  const TileAddr ta(a.B, C::kNPanel);
  const int my_tok = token_of_lane<L, R>(l);
  const bool primary = primary_lane<L, R>(l);
  float qf[G][AC];
  float acc[G][AC];
  float m_run[G], l_lane[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m_run[h] = -INFINITY;
    l_lane[h] = 0.f;
#pragma unroll
    for (int e = 0; e < AC; ++e) acc[h][e] = 0.f, qf[h][e] = 0.f;
  }

  int stage = 0;
  uint32_t phase = 0, epi_phase = 0;
  // All 128 consumer threads arrive; a wait that runs out of time abandons the kernel.
  auto epi_sync = [&]() -> bool {
    pa::mbar_arrive(epi);
    const bool done = pa::mbar_wait(epi, epi_phase);
    epi_phase ^= 1;
    if (!done && lane == 0) atomicOr(a.err, pa::kErrWaitTimeout);
    return done;
  };
  while (true) {
    if (!pa::mbar_wait(&full[stage], phase)) {
      if (lane == 0) atomicOr(a.err, pa::kErrWaitTimeout);
      return;
    }
    const StageMeta mt = meta[stage];
    if (mt.flags & kDone) break;
    const uint8_t* ks = stages + stage * C::kStageBytes;
    const uint8_t* vs = ks + C::kKVBytes;
    const int ntok = mt.ntok;

    if (mt.flags & kFirst) {
      const T* qsm = reinterpret_cast<const T*>(qslots + stage * C::kQSlot);
#pragma unroll
      for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
          const uint4 raw = *reinterpret_cast<const uint4*>(qsm + h * D + (k * L + l) * E);
          ChunkTraits<T>::to_float(raw, &qf[h][k * E]);
        }
#pragma unroll
        for (int e = 0; e < AC; ++e) qf[h][e] *= a.scale_log2;
        m_run[h] = -INFINITY;
        l_lane[h] = 0.f;
#pragma unroll
        for (int e = 0; e < AC; ++e) acc[h][e] = 0.f;
      }
    }

#pragma unroll
    for (int pass = 0; pass < C::kPasses; ++pass) {
      const int row0 = pass * (kConsumerWarps * C::kTPW) + warp * C::kTPW + grp * R;
      // ---- scores: partial dot products over this lane's chunks, then reduce-scatter ----
      float part[G][R];
#pragma unroll
      for (int i = 0; i < R; ++i) {
#pragma unroll
        for (int h = 0; h < G; ++h) part[h][i] = 0.f;
        const int row = row0 + i;
        if (row < ntok) {
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            const int c = k * L + l;
            const uint4 raw =
                pa::lds128(ks + ta.row(row) + ta.chunk(row, c));
            float kv[E];
            ChunkTraits<T>::to_float(raw, kv);
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
              for (int e = 0; e < E; ++e) part[h][i] = fmaf(qf[h][k * E + e], kv[e], part[h][i]);
          }
        }
      }
      reduce_scatter<G, R, L / 2, R>(part, l);

      // ---- online softmax (scores are in log2 units) ----
      const bool valid = row0 + my_tok < ntok;
      float sc[G], mt_[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        sc[h] = valid ? part[h][0] : -INFINITY;
        mt_[h] = sc[h];
      }
#pragma unroll
      for (int msk = 16; msk >= 1; msk >>= 1) {
        // lanes that differ only in all-reduce bits hold the same score; skip those levels
        const bool dup_level = (msk < L) && (msk < L / R);
        if (!dup_level) {
#pragma unroll
          for (int h = 0; h < G; ++h) mt_[h] = fmaxf(mt_[h], __shfl_xor_sync(0xffffffffu, mt_[h], msk));
        }
      }
      float p[G];
      bool rescale = false;
      float alpha[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mn = fmaxf(m_run[h], mt_[h]);
        alpha[h] = (mn == -INFINITY) ? 1.f : exp2f(m_run[h] - mn);
        p[h] = (mn == -INFINITY) ? 0.f : exp2f(sc[h] - mn);
        rescale |= (mn != m_run[h]);
        m_run[h] = mn;
        l_lane[h] = l_lane[h] * alpha[h] + (primary ? p[h] : 0.f);
      }
      if (rescale) {
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int e = 0; e < AC; ++e) acc[h][e] *= alpha[h];
      }

      // ---- p.V over the group's R tokens ----
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const int src = grp * L + lane_of_token<L, R>(i);
        float pi[G];
#pragma unroll
        for (int h = 0; h < G; ++h) pi[h] = __shfl_sync(0xffffffffu, p[h], src);
        const int row = row0 + i;
        if (row < ntok) {
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            const int c = k * L + l;
            const uint4 raw =
                pa::lds128(vs + ta.row(row) + ta.chunk(row, c));
            float vv[E];
            ChunkTraits<T>::to_float(raw, vv);
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
              for (int e = 0; e < E; ++e) acc[h][k * E + e] = fmaf(pi[h], vv[e], acc[h][k * E + e]);
          }
        }
      }
    }

    __syncwarp();
    if (lane == 0) pa::mbar_arrive(&empty[stage]);

    if (mt.flags & kLast) {
      // ---- merge the four warps' states in a fixed order and write the result ----
      float lw[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float v = l_lane[h];
#pragma unroll
        for (int msk = 16; msk >= 1; msk >>= 1) v += __shfl_xor_sync(0xffffffffu, v, msk);
        lw[h] = v;
      }
#pragma unroll
      for (int msk = L; msk < 32; msk <<= 1)
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int e = 0; e < AC; ++e) acc[h][e] += __shfl_xor_sync(0xffffffffu, acc[h][e], msk);
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          ml[(warp * G + h) * 2] = m_run[h];
          ml[(warp * G + h) * 2 + 1] = lw[h];
        }
      }
      if (!epi_sync()) return;
      float M[G], den[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, ml[(w * G + h) * 2]);
        float dsum = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float mw = ml[(w * G + h) * 2];
          if (mw != -INFINITY) dsum += exp2f(mw - mx) * ml[(w * G + h) * 2 + 1];
        }
        M[h] = mx;
        den[h] = dsum;
        const float mine = (m_run[h] == -INFINITY) ? 0.f : exp2f(m_run[h] - mx);
#pragma unroll
        for (int e = 0; e < AC; ++e) acc[h][e] *= mine;
      }
      // tree sum: (w0 + w2) + (w1 + w3), then w0 + w1; lanes of group 0 hold the warp's sums
      const bool writer = grp == 0;
      constexpr unsigned kWriterMask = L == 32 ? 0xffffffffu : ((1u << L) - 1u);
      if (warp >= 2 && writer) {
        float* buf = merge + (warp - 2) * G * D;
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int k = 0; k < CPL; ++k)
#pragma unroll
            for (int e = 0; e < E; e += 4)
              *reinterpret_cast<float4*>(buf + h * D + (k * L + l) * E + e) =
                  make_float4(acc[h][k * E + e], acc[h][k * E + e + 1], acc[h][k * E + e + 2], acc[h][k * E + e + 3]);
      }
      if (!epi_sync()) return;
      if (warp < 2 && writer) {
        float* buf = merge + warp * G * D;
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int k = 0; k < CPL; ++k)
#pragma unroll
            for (int e = 0; e < E; e += 4) {
              const float4 v = *reinterpret_cast<const float4*>(buf + h * D + (k * L + l) * E + e);
              acc[h][k * E + e] += v.x;
              acc[h][k * E + e + 1] += v.y;
              acc[h][k * E + e + 2] += v.z;
              acc[h][k * E + e + 3] += v.w;
            }
        if (warp == 1) {
          __syncwarp(kWriterMask);  // only the writer lanes are here
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int k = 0; k < CPL; ++k)
#pragma unroll
              for (int e = 0; e < E; e += 4)
                *reinterpret_cast<float4*>(buf + h * D + (k * L + l) * E + e) = make_float4(
                    acc[h][k * E + e], acc[h][k * E + e + 1], acc[h][k * E + e + 2], acc[h][k * E + e + 3]);
        }
      }
      if (!epi_sync()) return;
      if (warp == 0 && writer) {
        const float* buf = merge + G * D;
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int k = 0; k < CPL; ++k)
#pragma unroll
            for (int e = 0; e < E; e += 4) {
              const float4 v = *reinterpret_cast<const float4*>(buf + h * D + (k * L + l) * E + e);
              acc[h][k * E + e] += v.x;
              acc[h][k * E + e + 1] += v.y;
              acc[h][k * E + e + 2] += v.z;
              acc[h][k * E + e + 3] += v.w;
            }
        const size_t row = static_cast<size_t>(mt.orow) * a.H + static_cast<size_t>(mt.kh) * G;  // out
        const size_t prow = static_cast<size_t>(mt.s) * a.H + static_cast<size_t>(mt.kh) * G;  // partials
        if (mt.flags & kSingle) {
          float inv[G];
#pragma unroll
          for (int h = 0; h < G; ++h) inv[h] = den[h] > 0.f ? 1.f / den[h] : 0.f;
          if (a.out_dtype == PA_F32)
            write_rows<float, D, G, AC, L, CPL, E>(static_cast<float*>(a.out) + row * D, acc, inv, l);
          else if (a.out_dtype == PA_F16)
            write_rows<__half, D, G, AC, L, CPL, E>(static_cast<__half*>(a.out) + row * D, acc, inv, l);
          else
            write_rows<__nv_bfloat16, D, G, AC, L, CPL, E>(static_cast<__nv_bfloat16*>(a.out) + row * D, acc, inv,
                                                           l);
        } else {
          float one[G];
#pragma unroll
          for (int h = 0; h < G; ++h) one[h] = 1.f;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const size_t pidx = (prow + h) * a.max_parts + mt.part;
            float acc_h[1][AC];
#pragma unroll
            for (int e = 0; e < AC; ++e) acc_h[0][e] = acc[h][e];
            write_rows<float, D, 1, AC, L, CPL, E>(a.part_o + pidx * D, acc_h, one, l);
            if (l == 0) {
              a.part_m[pidx] = M[h] == -INFINITY ? -INFINITY : M[h] * kLn2;
              a.part_l[pidx] = den[h];
            }
          }
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m_run[h] = -INFINITY;
        l_lane[h] = 0.f;
#pragma unroll
        for (int e = 0; e < AC; ++e) acc[h][e] = 0.f;
      }
    }

    if (++stage == C::kStages) {
      stage = 0;
      phase ^= 1;
    }
  }
  }  // consumers
}

// ---- log-sum-exp combine -----------------------------------------------------------------------
// WPR warps per (sequence, query head); lane owns D/32 consecutive dims.  q_rows is null, or the
// q_start of a mixed batch whose one-token sequences are merged here (output row q_start[s]).  With WPR > 1 the warps of
// a row take interleaved batches of 32 partitions (batch b to warp b % WPR) and their sums are
// added in a fixed order through shared memory, so that rows with many partitions keep more loads
// in flight.  Sequences with fewer than min_parts partitions are skipped (the decode kernel
// already wrote them).
constexpr int kCombineThreads = 256;

template <class OutT, int D, int WPR>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(OutT* __restrict__ out, const float* __restrict__ part_o,
                                                                  const float* __restrict__ part_m,
                                                                  const float* __restrict__ part_l,
                                                                  const int32_t* __restrict__ lens, int S, int H,
                                                                  int max_parts, int P, int min_parts,
                                                                  const int32_t* __restrict__ q_rows) {
  // Partitions past max_parts are never read: a length that needs more is cut to max_parts * P.
  pa::grid_dependency_wait();  // launched right behind the decode grid: its partials must be complete
  constexpr int PER = D / 32;
  constexpr int kRowsPerCta = kCombineThreads / 32 / WPR;
  __shared__ float red_acc[WPR > 1 ? kRowsPerCta * (WPR - 1) * D : 1];
  __shared__ float red_den[WPR > 1 ? kRowsPerCta * (WPR - 1) : 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_in_cta = warp / WPR, sub = warp % WPR;
  const long long gw = static_cast<long long>(blockIdx.x) * kRowsPerCta + row_in_cta;
  bool write = false;  // this row's output is written here (by sub-warp 0)
  int np = 0;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float den = 0.f;
  if (gw < static_cast<long long>(S) * H) {
    const int s = static_cast<int>(gw / H);
    const int c = max(lens[s], 0);
    np = min((c + P - 1) / P, max_parts);
    // empty context: zeros (the decode kernel already wrote them when min_parts > 1)
    write = np == 0 ? min_parts <= 1 : np >= min_parts;
    // q_rows is a mixed batch's q_start: only its one-token sequences are this launch's
    if (q_rows && q_rows[s + 1] - q_rows[s] != 1) write = false;
  }
  if (write && np > 0) {
    const float* pm = part_m + gw * max_parts;
    const float* pl = part_l + gw * max_parts;
    float mx = -INFINITY;
    for (int p = lane; p < np; p += 32) mx = fmaxf(mx, pm[p]);
#pragma unroll
    for (int msk = 16; msk >= 1; msk >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, msk));
    if (mx != -INFINITY) {
      // 32 partitions at a time: lane j computes partition (base + j)'s weight, then every lane
      // accumulates its dims over the 32 with independent loads in flight.
      for (int base = sub * 32; base < np; base += 32 * WPR) {
        const int p = base + lane;
        float w = 0.f;
        if (p < np) {
          const float mp = pm[p];
          w = mp == -INFINITY ? 0.f : expf(mp - mx);
          den = fmaf(w, pl[p], den);
        }
        const int cnt = min(32, np - base);
        const float* src = part_o + (gw * max_parts + base) * D + lane * PER;
#pragma unroll 8
        for (int j = 0; j < cnt; ++j) {
          const float wj = __shfl_sync(0xffffffffu, w, j);
#pragma unroll
          for (int e = 0; e < PER; e += 2) {
            const float2 v = *reinterpret_cast<const float2*>(src + static_cast<size_t>(j) * D + e);
            acc[e] = fmaf(wj, v.x, acc[e]);
            acc[e + 1] = fmaf(wj, v.y, acc[e + 1]);
          }
        }
      }
#pragma unroll
      for (int msk = 16; msk >= 1; msk >>= 1) den += __shfl_xor_sync(0xffffffffu, den, msk);
    }
  }
  if constexpr (WPR > 1) {
    // sub-warps 1 .. WPR-1 hand their sums to sub-warp 0, which adds them in index order
    if (sub > 0) {
      float* dst = red_acc + (row_in_cta * (WPR - 1) + sub - 1) * D + lane * PER;
#pragma unroll
      for (int e = 0; e < PER; ++e) dst[e] = acc[e];
      if (lane == 0) red_den[row_in_cta * (WPR - 1) + sub - 1] = den;
    }
    __syncthreads();
    if (sub > 0) return;
#pragma unroll
    for (int k = 0; k < WPR - 1; ++k) {
      const float* src = red_acc + (row_in_cta * (WPR - 1) + k) * D + lane * PER;
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] += src[e];
      den += red_den[row_in_cta * (WPR - 1) + k];
    }
  }
  if (!write) return;
  const long long orow = q_rows ? static_cast<long long>(q_rows[gw / H]) * H + gw % H : gw;
  OutT* o = out + orow * D + lane * PER;
  const float inv = den > 0.f ? 1.f / den : 0.f;
  float res[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) res[e] = acc[e] * inv;
  pa::store_pairs<OutT, PER>(o, res);
}



// ---- host side ----------------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Tensor map over a cache viewed as [n_blocks*Hk*B rows][d].  One box is the B rows of one
// (block, kv head) with every 128-byte panel of them: with a single panel (d * element size = 128)
// a 2-D box {128 bytes, B rows}; otherwise a 3-D view {128 bytes, row, panel} whose panel stride
// (128 bytes) is smaller than its row stride (d * element size), so that the box lands panel by
// panel ([panel][B rows][128 bytes]), the order the 128-byte swizzle needs for conflict-free
// ldmatrix.  Every element the view addresses lies inside the cache.
bool make_cache_map(CUtensorMap* map, const void* base, pa_dtype dt, int d, long long rows, int B) {
  auto enc = get_encoder();
  if (!enc) return false;
  const CUtensorMapDataType t = dt == PA_F32   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                : dt == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                               : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int es = static_cast<int>(pa::elem_size(dt));
  const int panel_elems = 128 / es, n_panel = d / panel_elems;
  if (n_panel == 1) {
    cuuint64_t gdim[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
    cuuint64_t gstride[1] = {static_cast<cuuint64_t>(d) * es};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(panel_elems), static_cast<cuuint32_t>(B)};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, t, 2, const_cast<void*>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  cuuint64_t gdim[3] = {static_cast<cuuint64_t>(panel_elems), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(n_panel)};
  cuuint64_t gstride[2] = {static_cast<cuuint64_t>(d) * es, 128};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(panel_elems), static_cast<cuuint32_t>(B),
                       static_cast<cuuint32_t>(n_panel)};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, t, 3, const_cast<void*>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch with programmatic stream serialisation: the grid may start while the previous kernel on
// the stream finishes; the kernel itself waits (griddepcontrol.wait) before touching its inputs.
template <class... KArgs, class... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int D, int WPR>
cudaError_t launch_combine_w(void* out, pa_dtype out_dtype, const float* po, const float* pm, const float* pl,
                             const int32_t* lens, int S, int H, int max_parts, int P, int min_parts,
                             const int32_t* q_rows, cudaStream_t st) {
  constexpr int kRowsPerCta = kCombineThreads / 32 / WPR;
  const long long rows = static_cast<long long>(S) * H;
  const dim3 grid(static_cast<unsigned>((rows + kRowsPerCta - 1) / kRowsPerCta)), block(kCombineThreads);
  if (grid.x == 0) return cudaSuccess;
  if (out_dtype == PA_F32)
    return launch_pdl(combine_kernel<float, D, WPR>, grid, block, 0, st, static_cast<float*>(out), po, pm, pl, lens, S,
                      H, max_parts, P, min_parts, q_rows);
  if (out_dtype == PA_F16)
    return launch_pdl(combine_kernel<__half, D, WPR>, grid, block, 0, st, static_cast<__half*>(out), po, pm, pl, lens,
                      S, H, max_parts, P, min_parts, q_rows);
  return launch_pdl(combine_kernel<__nv_bfloat16, D, WPR>, grid, block, 0, st, static_cast<__nv_bfloat16*>(out), po,
                    pm, pl, lens, S, H, max_parts, P, min_parts, q_rows);
}

// Rows with many partitions (more than two batches of 32) get four warps each.
template <int D>
cudaError_t launch_combine(void* out, pa_dtype out_dtype, const float* po, const float* pm, const float* pl,
                           const int32_t* lens, int S, int H, int max_parts, int P, int min_parts,
                           cudaStream_t st, const int32_t* q_rows = nullptr) {
  return max_parts > 64
             ? launch_combine_w<D, 4>(out, out_dtype, po, pm, pl, lens, S, H, max_parts, P, min_parts, q_rows, st)
             : launch_combine_w<D, 1>(out, out_dtype, po, pm, pl, lens, S, H, max_parts, P, min_parts, q_rows, st);
}

struct DeviceInfo {
  int sms = 0;
};

DeviceInfo device_info() {
  DeviceInfo di;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
  if (di.sms <= 0) di.sms = 148;
  return di;
}

template <class T, int D, int G, bool kMma>
cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a, int max_units,
                          cudaStream_t st) {
  using C = Cfg<T, D, G>;
  // the shared-memory attribute belongs to the current context (each device keeps its own, a device
  // reset drops it): set again whenever the context differs from the one it was set in
  static std::atomic<unsigned long long> ready_ctx{0};
  static std::atomic<int> occupancy{1};
  cudaError_t e = cudaSuccess;
  const unsigned long long ctx = pa::current_context_id();
  if (ctx == 0 || ready_ctx.load(std::memory_order_acquire) != ctx) {
    e = cudaFuncSetAttribute(decode_kernel<T, D, G, kMma>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernel<T, D, G, kMma>, kThreads, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    occupancy.store(occ < 1 ? 1 : occ, std::memory_order_relaxed);
    ready_ctx.store(pa::current_context_id(), std::memory_order_release);
  }
  const DeviceInfo di = device_info();
  long long grid = static_cast<long long>(di.sms) * occupancy.load(std::memory_order_relaxed);
  if (grid > max_units) grid = max_units;
  if (grid < 1) grid = 1;
  return launch_pdl(decode_kernel<T, D, G, kMma>, dim3(static_cast<unsigned>(grid)), dim3(kThreads), C::kSmemBytes,
                    st, tk, tv, a);
}

// Tensor-core consumers for 16-bit caches unless PA_DECODE_CONSUMER=cuda_core; fp32 caches always
// use the CUDA-core consumers.
bool use_tensor_cores() {
  const char* v = std::getenv("PA_DECODE_CONSUMER");
  return !(v && std::strcmp(v, "cuda_core") == 0);
}

template <class T, int D, bool kMma>
cudaError_t dispatch_g(int g, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a, int max_units,
                       cudaStream_t st) {
  switch (g) {
    case 1: return launch_decode<T, D, 1, kMma>(tk, tv, a, max_units, st);
    case 2: return launch_decode<T, D, 2, kMma>(tk, tv, a, max_units, st);
    case 4: return launch_decode<T, D, 4, kMma>(tk, tv, a, max_units, st);
    default: return launch_decode<T, D, 8, kMma>(tk, tv, a, max_units, st);
  }
}

template <class T, bool kMma>
cudaError_t dispatch_d(int d, int g, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a,
                       int max_units, cudaStream_t st) {
  return d == 64 ? dispatch_g<T, 64, kMma>(g, tk, tv, a, max_units, st)
                 : dispatch_g<T, 128, kMma>(g, tk, tv, a, max_units, st);
}

template <class T>
cudaError_t dispatch_16bit(int d, int g, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a,
                           int max_units, cudaStream_t st) {
  return use_tensor_cores() ? dispatch_d<T, true>(d, g, tk, tv, a, max_units, st)
                            : dispatch_d<T, false>(d, g, tk, tv, a, max_units, st);
}

int default_partition(int S, int Hk, int max_context_len) {
  // Longer partitions mean fewer partial states to write and merge and fewer unit start-ups; the
  // longest-first unit order keeps the persistent grid balanced while there are enough units per
  // CTA.  The count below is an upper bound (every sequence at max_context_len), so the bar is six
  // per SM.  Measured on B200 (fraction of the HBM copy peak): gqa8k 0.956 / 0.980 / 0.991 / 1.009
  // at P = 1024 / 2048 / 4096 / 8192; long-context (16 seqs, 16-32 k tokens, B 16) 0.939 / 0.953 /
  // 0.976 at 1024 / 2048 / 4096 but 0.813 at 8192 (about 384 actual units for 296 CTAs).
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  // No longer than the smallest of them that holds the longest context: beyond it nothing splits
  // any more, and the shared-prefix workload (contexts ~1.1-1.4 k) measured 0.995 at 2048 but 0.98
  // at 8192.
  const long long pairs = static_cast<long long>(S) * Hk;
  for (int P : {8192, 4096, 2048, 1024, 512, 256})
    if (pairs * ((max_context_len + P - 1) / P) >= 6LL * sms && (P / 2 < max_context_len || P == 256)) return P;
  return 128;
}

int max_parts_for(int max_context_len, int P) {
  const int n = (max_context_len + P - 1) / P;
  return n < 1 ? 1 : n;
}

}  // namespace

unsigned long long pa::current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}


extern "C" int pa_decode_default_partition(int S, int Hk, int max_context_len) {
  return default_partition(S, Hk, max_context_len);
}

extern "C" size_t pa_decode_workspace_size(int S, int H, int Hk, int d, int max_context_len, int partition_size) {
  if (S < 0 || H <= 0 || Hk <= 0 || d <= 0 || max_context_len < 0) return 0;
  const int P = partition_size > 0 ? partition_size : default_partition(S, Hk, max_context_len);
  return ws_layout(S, H, Hk, d, max_parts_for(max_context_len, P)).total;
}

extern "C" pa_status pa_workspace_error(const void* workspace, int* flags, void* stream) {
  if (!workspace || !flags) return pa::fail(PA_ERR_INVALID_ARG, "pa_workspace_error: null argument");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess)
    e = cudaMemcpy(flags, static_cast<const int*>(workspace) + kHdrError, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_workspace_error: %s", cudaGetErrorString(e));
  return pa::ok();
}

namespace {

// Everything a decode launch needs, validated: kernel arguments, tensor maps and sizes.
struct DecodePlan {
  DecodeArgs a;
  CUtensorMap tk, tv;
  WsLayout wl;
  int g, d, P, max_parts, max_units;
  pa_dtype kv_dtype, out_dtype;
};

pa_status prepare_decode(DecodePlan& dp, const char* who, void* out, pa_dtype out_dtype, const void* query,
                         const void* k_cache, const void* v_cache, const int32_t* block_tables,
                         const int32_t* context_lens, int S, int H, int Hk, int d, int B, int n_blocks,
                         int max_blocks_per_seq, int max_context_len, float scale, pa_dtype kv_dtype,
                         int partition_size, void* workspace, size_t workspace_bytes) {
  if (S < 0 || H <= 0 || Hk <= 0 || n_blocks <= 0 || max_blocks_per_seq < 0 || max_context_len < 0)
    return pa::fail(PA_ERR_INVALID_ARG, "%s: bad sizes (S=%d H=%d Hk=%d n_blocks=%d)", who, S, H, Hk, n_blocks);
  if (H % Hk != 0) return pa::fail(PA_ERR_INVALID_ARG, "%s: H (%d) must be a multiple of Hk (%d)", who, H, Hk);
  const int g = H / Hk;
  if (g != 1 && g != 2 && g != 4 && g != 8) return pa::fail(PA_ERR_UNSUPPORTED, "%s: H/Hk = %d not in {1,2,4,8}", who, g);
  if (d != 64 && d != 128) return pa::fail(PA_ERR_UNSUPPORTED, "%s: d = %d not in {64,128}", who, d);
  if (B != 8 && B != 16 && B != 32) return pa::fail(PA_ERR_UNSUPPORTED, "%s: B = %d not in {8,16,32}", who, B);
  if (!pa::valid_dtype(kv_dtype) || !pa::valid_dtype(out_dtype)) return pa::fail(PA_ERR_INVALID_ARG, "%s: unknown dtype", who);
  if (!std::isfinite(scale)) return pa::fail(PA_ERR_INVALID_ARG, "%s: scale must be finite", who);
  const int P = partition_size > 0 ? partition_size : default_partition(S, Hk, max_context_len);
  if (P % kTileTokens != 0 || P > (1 << 24))
    return pa::fail(PA_ERR_INVALID_ARG, "%s: partition_size %d must be a positive multiple of 64", who, P);
  const int max_parts = max_parts_for(max_context_len, P);
  if (max_parts > 0xffff) return pa::fail(PA_ERR_UNSUPPORTED, "%s: more than 65535 partitions per sequence", who);
  if (static_cast<long long>(max_blocks_per_seq) * B < max_context_len)
    return pa::fail(PA_ERR_INVALID_ARG, "%s: max_blocks_per_seq * B < max_context_len", who);
  const long long rows = static_cast<long long>(n_blocks) * Hk * B;
  if (rows >= (1ll << 31) || static_cast<long long>(S) * Hk * max_parts > (1ll << 31))
    return pa::fail(PA_ERR_UNSUPPORTED, "%s: problem too large for 32-bit indices", who);
  dp.g = g;
  dp.d = d;
  dp.P = P;
  dp.max_parts = max_parts;
  dp.kv_dtype = kv_dtype;
  dp.out_dtype = out_dtype;
  if (S == 0) return PA_OK;
  if (!out || !query || !k_cache || !v_cache || !block_tables || !context_lens || !workspace)
    return pa::fail(PA_ERR_INVALID_ARG, "%s: null pointer", who);
  if (!pa::aligned16(out) || !pa::aligned16(query) || !pa::aligned16(k_cache) || !pa::aligned16(v_cache))
    return pa::fail(PA_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", who);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return pa::fail(PA_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
  dp.wl = ws_layout(S, H, Hk, d, max_parts);
  if (workspace_bytes < dp.wl.total)
    return pa::fail(PA_ERR_INVALID_ARG, "%s: workspace of %zu bytes < %zu needed", who, workspace_bytes, dp.wl.total);
  if (!make_cache_map(&dp.tk, k_cache, kv_dtype, d, rows, B) || !make_cache_map(&dp.tv, v_cache, kv_dtype, d, rows, B))
    return pa::fail(PA_ERR_CUDA, "%s: could not encode the cache tensor maps", who);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeArgs& a = dp.a;
  a.q = query;
  a.out = out;
  a.out_dtype = out_dtype;
  a.bt = block_tables;
  a.lens = context_lens;
  a.S = S;
  a.H = H;
  a.Hk = Hk;
  a.max_blocks = max_blocks_per_seq;
  a.n_blocks = n_blocks;
  a.B = B;
  a.P = P;
  a.max_c = max_context_len;
  a.scale_log2 = scale * kLog2e;
  a.items = reinterpret_cast<const int2*>(ws + dp.wl.items);
  a.hdr = reinterpret_cast<int*>(ws);
  a.err = a.hdr + kHdrError;
  a.q_rows = nullptr;
  a.part_o = reinterpret_cast<float*>(ws + dp.wl.part_o);
  a.part_m = reinterpret_cast<float*>(ws + dp.wl.part_m);
  a.part_l = reinterpret_cast<float*>(ws + dp.wl.part_l);
  a.max_parts = max_parts;
  const long long units = static_cast<long long>(S) * Hk * max_parts;
  dp.max_units = static_cast<int>(units < (1ll << 30) ? units : (1ll << 30));
  return PA_OK;
}

// The decode kernel and, for split sequences, the combine; both behind the plan with PDL.
pa_status launch_decode_and_combine(const DecodePlan& dp, const char* who, cudaStream_t st) {
  const DecodeArgs& a = dp.a;
  cudaError_t e;
  if (dp.kv_dtype == PA_F32) e = dispatch_d<float, false>(dp.d, dp.g, dp.tk, dp.tv, a, dp.max_units, st);
  else if (dp.kv_dtype == PA_F16) e = dispatch_16bit<__half>(dp.d, dp.g, dp.tk, dp.tv, a, dp.max_units, st);
  else e = dispatch_16bit<__nv_bfloat16>(dp.d, dp.g, dp.tk, dp.tv, a, dp.max_units, st);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "%s: decode launch failed: %s", who, cudaGetErrorString(e));
  if (dp.max_parts > 1) {
    e = dp.d == 64 ? launch_combine<64>(a.out, dp.out_dtype, a.part_o, a.part_m, a.part_l, a.lens, a.S, a.H,
                                        dp.max_parts, dp.P, 2, st, a.q_rows)
                   : launch_combine<128>(a.out, dp.out_dtype, a.part_o, a.part_m, a.part_l, a.lens, a.S, a.H,
                                         dp.max_parts, dp.P, 2, st, a.q_rows);
    if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "%s: combine launch failed: %s", who, cudaGetErrorString(e));
  }
  return pa::ok();
}

}  // namespace

extern "C" pa_status pa_decode(void* out, pa_dtype out_dtype, const void* query, const void* k_cache,
                               const void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                               int S, int H, int Hk, int d, int B, int n_blocks, int max_blocks_per_seq,
                               int max_context_len, float scale, pa_dtype kv_dtype, int partition_size,
                               void* workspace, size_t workspace_bytes, void* stream) {
  DecodePlan dp;
  const pa_status ps = prepare_decode(dp, "pa_decode", out, out_dtype, query, k_cache, v_cache, block_tables,
                                      context_lens, S, H, Hk, d, B, n_blocks, max_blocks_per_seq, max_context_len,
                                      scale, kv_dtype, partition_size, workspace, workspace_bytes);
  if (ps != PA_OK) return ps;
  if (S == 0) return pa::ok();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = launch_pdl(plan_kernel, dim3(1), dim3(kPlanThreads), 0, st, context_lens, S, Hk, dp.P,
                                   max_context_len, reinterpret_cast<int2*>(const_cast<int2*>(dp.a.items)), dp.a.hdr,
                                   static_cast<const int32_t*>(nullptr), static_cast<int*>(nullptr));
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_decode: plan launch failed: %s", cudaGetErrorString(e));
  return launch_decode_and_combine(dp, "pa_decode", st);
}

// ---- decode of the one-token sequences of a mixed batch (for pa_prefill) ---------------------------
// The sequences with exactly one query token are decoded by the kernels above: their query and
// output rows are q_start[s], their units come from a plan that skips every other sequence, and
// errors are or-ed into the caller's error word.

namespace {
int single_rows_partition(int S, int Hk, int max_context_len) {
  const int P = default_partition(S, Hk, max_context_len);
  return P > 1024 ? 1024 : P;
}
}  // namespace

size_t pa::decode_single_rows_workspace(int S, int H, int Hk, int d, int max_context_len) {
  return pa_decode_workspace_size(S, H, Hk, d, max_context_len, single_rows_partition(S, Hk, max_context_len));
}

pa_status pa::decode_single_rows(void* out, pa_dtype out_dtype, const void* query, const int32_t* q_start,
                                 const void* k_cache, const void* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, int S, int H, int Hk, int d, int B, int n_blocks,
                                 int max_blocks_per_seq, int max_context_len, float scale, pa_dtype kv_dtype,
                                 void* workspace, size_t workspace_bytes, int* err, void* stream) {
  // A mixed batch's decode rows are usually a minority of its sequences, so the unit count that
  // the default partition assumes (every sequence at max_context_len) overstates their work and
  // the longest of them would be the grid's tail: partitions of at most 1024 tokens.
  DecodePlan dp;
  const pa_status ps = prepare_decode(dp, "pa_prefill (one-token rows)", out, out_dtype, query, k_cache, v_cache,
                                      block_tables, context_lens, S, H, Hk, d, B, n_blocks, max_blocks_per_seq,
                                      max_context_len, scale, kv_dtype, single_rows_partition(S, Hk, max_context_len),
                                      workspace, workspace_bytes);
  if (ps != PA_OK || S == 0) return ps;
  dp.a.q_rows = q_start;
  dp.a.err = err;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = launch_pdl(plan_kernel, dim3(1), dim3(kPlanThreads), 0, st, context_lens, S, Hk, dp.P,
                                   max_context_len, reinterpret_cast<int2*>(const_cast<int2*>(dp.a.items)), dp.a.hdr,
                                   q_start, err);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_prefill: plan launch failed: %s", cudaGetErrorString(e));
  return launch_decode_and_combine(dp, "pa_prefill (one-token rows)", st);
}

extern "C" pa_status pa_decode_step(void* out, pa_dtype out_dtype, const void* query, void* k_cache, void* v_cache,
                                    const int32_t* block_tables, const int32_t* context_lens, const void* key,
                                    const void* value, const int64_t* slot_mapping, int T, const int32_t* pairs,
                                    const int32_t* n_pairs, int max_pairs, int S, int H, int Hk, int d, int B,
                                    int n_blocks, int max_blocks_per_seq, int max_context_len, float scale,
                                    pa_dtype kv_dtype, int partition_size, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  DecodePlan dp;
  const pa_status ps = prepare_decode(dp, "pa_decode_step", out, out_dtype, query, k_cache, v_cache, block_tables,
                                      context_lens, S, H, Hk, d, B, n_blocks, max_blocks_per_seq, max_context_len,
                                      scale, kv_dtype, partition_size, workspace, workspace_bytes);
  if (ps != PA_OK) return ps;
  if (T < 0 || max_pairs < 0 || max_pairs > kMaxStepPairs)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_decode_step: need T >= 0 and 0 <= max_pairs <= %d (T=%d, max_pairs=%d)",
                    kMaxStepPairs, T, max_pairs);
  if ((T > 0 && (!key || !value || !slot_mapping)) || (max_pairs > 0 && !pairs) || !k_cache || !v_cache)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_decode_step: null pointer");
  if (!pa::aligned16(k_cache) || !pa::aligned16(v_cache) || (T > 0 && (!pa::aligned16(key) || !pa::aligned16(value))))
    return pa::fail(PA_ERR_INVALID_ARG, "pa_decode_step: caches, key and value must be 16-byte aligned");
  const int es = static_cast<int>(pa::elem_size(kv_dtype));
  PrologueArgs w;
  w.kc = static_cast<uint4*>(k_cache);
  w.vc = static_cast<uint4*>(v_cache);
  w.key = static_cast<const uint4*>(key);
  w.value = static_cast<const uint4*>(value);
  w.slots = slot_mapping;
  w.pairs = pairs;
  w.n_pairs_dev = n_pairs;
  w.T = T;
  w.max_pairs = max_pairs;
  w.Hk = Hk;
  w.chunks = d * es / 16;
  w.B = B;
  w.n_blocks = n_blocks;
  w.vec_per_block = static_cast<long long>(Hk) * B * d * es / 16;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (S == 0) {
    // nothing to decode: the copies and writes alone, in their order
    pa_status s2 = max_pairs > 0 ? (n_pairs ? pa::copy_blocks_counted(k_cache, v_cache, pairs, n_pairs, max_pairs, Hk,
                                                                       d, B, n_blocks, kv_dtype, stream)
                                            : pa_copy_blocks(k_cache, v_cache, pairs, max_pairs, Hk, d, B, n_blocks,
                                                             kv_dtype, stream))
                                 : PA_OK;
    if (s2 == PA_OK) s2 = pa_cache_write(k_cache, v_cache, key, value, slot_mapping, T, Hk, d, B, n_blocks, kv_dtype, stream);
    return s2;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // one CTA for the plan, then workers: one per pair (the count on the device may be smaller) and
  // enough warps for the tokens, at most four per SM
  long long workers = max_pairs;
  const long long for_tokens = (static_cast<long long>(T) + kPrologueThreads / 32 - 1) / (kPrologueThreads / 32);
  if (workers < for_tokens) workers = for_tokens;
  if (workers > 4LL * sms) workers = 4LL * sms;
  if (workers < 1) workers = 1;
  cudaError_t e = launch_pdl(step_prologue_kernel, dim3(static_cast<unsigned>(1 + workers)), dim3(kPrologueThreads), 0,
                             st, w, context_lens, S, Hk, dp.P, max_context_len,
                             reinterpret_cast<int2*>(const_cast<int2*>(dp.a.items)), dp.a.hdr);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_decode_step: prologue launch failed: %s", cudaGetErrorString(e));
  return launch_decode_and_combine(dp, "pa_decode_step", st);
}

extern "C" pa_status pa_combine(void* out, pa_dtype out_dtype, const float* part_o, const float* part_m,
                                const float* part_l, const int32_t* context_lens, int S, int H, int d, int max_parts,
                                int partition_size, void* stream) {
  if (S < 0 || H <= 0 || max_parts <= 0 || partition_size <= 0)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_combine: bad sizes");
  if (d != 64 && d != 128) return pa::fail(PA_ERR_UNSUPPORTED, "pa_combine: d = %d not in {64,128}", d);
  if (!pa::valid_dtype(out_dtype)) return pa::fail(PA_ERR_INVALID_ARG, "pa_combine: unknown dtype");
  if (S == 0) return pa::ok();
  if (!out || !part_o || !part_m || !part_l || !context_lens) return pa::fail(PA_ERR_INVALID_ARG, "pa_combine: null pointer");
  if (!pa::aligned16(out) || !pa::aligned16(part_o)) return pa::fail(PA_ERR_INVALID_ARG, "pa_combine: out/part_o must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e =
      d == 64 ? launch_combine<64>(out, out_dtype, part_o, part_m, part_l, context_lens, S, H, max_parts, partition_size, 1, st)
              : launch_combine<128>(out, out_dtype, part_o, part_m, part_l, context_lens, S, H, max_parts, partition_size, 1, st);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_combine: launch failed: %s", cudaGetErrorString(e));
  return pa::ok();
}

// ---- decode without any device allocation --------------------------------------------------------
// The decode workspace of pa_decode_noalloc lives in this file-scope device array instead of
// caller memory.  Every GPU that loads the library holds it until the process exits.  In host
// code `g_noalloc_scratch` only names a host-side stand-in, so its device address is fetched with
// cudaGetSymbolAddress (with the device current) and passed to the kernels.  The address belongs
// to the device's current context: it is looked up once per device and looked up again when that
// context has changed (a device reset destroys the context, and the module holding the array is
// loaded again, possibly elsewhere, in the next one).  Contexts are told apart by the driver's
// context id, which is never reused within a process.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
struct NoAllocSlot {
  void* ptr = nullptr;
  unsigned long long ctx_id = 0;
};
NoAllocSlot g_noalloc[kMaxDevices];

cudaError_t noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoAllocSlot& slot = g_noalloc[dev];
  const unsigned long long ctx_id = pa::current_context_id();  // 0 before the runtime has made one current
  if (!slot.ptr || ctx_id == 0 || slot.ctx_id != ctx_id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // makes the device's context current if needed
    if (e != cudaSuccess) return e;
    slot.ptr = p;
    slot.ctx_id = pa::current_context_id();
  }
  *ptr = slot.ptr;
  return cudaSuccess;
}

}  // namespace

extern "C" pa_status pa_decode_noalloc(void* out, pa_dtype out_dtype, const void* query, const void* k_cache,
                                       const void* v_cache, const int32_t* block_tables,
                                       const int32_t* context_lens, int S, int H, int Hk, int d, int B,
                                       int n_blocks, int max_blocks_per_seq, int max_context_len, float scale,
                                       pa_dtype kv_dtype, int partition_size, void* stream) {
  const size_t need = pa_decode_workspace_size(S, H, Hk, d, max_context_len, partition_size);
  if (need == 0) return pa::fail(PA_ERR_INVALID_ARG, "pa_decode_noalloc: bad sizes");
  if (need > kNoAllocScratchBytes)
    return pa::fail(PA_ERR_INVALID_ARG,
                    "pa_decode_noalloc: these sizes need %zu bytes of scratch; the built-in scratch holds %zu "
                    "(use pa_decode with a caller-provided workspace, or a larger partition_size)",
                    need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  const cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess)
    return pa::fail(PA_ERR_CUDA, "pa_decode_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
  return pa_decode(out, out_dtype, query, k_cache, v_cache, block_tables, context_lens, S, H, Hk, d, B, n_blocks,
                   max_blocks_per_seq, max_context_len, scale, kv_dtype, partition_size, scratch,
                   kNoAllocScratchBytes, stream);
}

// ---- self-test of the bounded pipeline wait -------------------------------------------------------
namespace {

// Waits, with the same helper the decode pipeline uses, for a barrier phase that nothing completes;
// the wait gives up after limit_ns and the kernel reports it instead of spinning.
__global__ void wait_probe_kernel(unsigned long long limit_ns, int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    pa::mbar_init(&bar, 1);
    pa::fence_barrier_init();
  }
  __syncthreads();
  const bool done = pa::mbar_wait(&bar, 0, limit_ns);
  if (threadIdx.x == 0) *status = done ? 0 : pa::kErrWaitTimeout;
}

}  // namespace

extern "C" pa_status pa_selftest_wait_timeout(unsigned int limit_us, int* status, void* stream) {
  if (!status || limit_us == 0 || limit_us > 10000000u)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_selftest_wait_timeout: need a status pointer and 0 < limit_us <= 1e7");
  wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(1000ull * limit_us, status);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_selftest_wait_timeout: %s", cudaGetErrorString(e));
  return pa::ok();
}

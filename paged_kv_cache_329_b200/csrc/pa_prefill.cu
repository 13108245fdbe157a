// Paged attention for several query tokens per sequence: chunked prefill, and batches that mix
// prefill chunks with decode tokens.
//
// What is computed: sequence s has n_s query tokens, the last n_s of its c_s context tokens
// (already written to the cache); the token at position p attends causally to positions 0..p,
// o = softmax(scale * q K[0..p]^T) V[0..p] -- the decode definition ("PagedAttention原理",
// "为什么会有 KV cache", eq. o_t; "实现一个虚拟内存", eqs. A_ij, o_i) per query token.  Prefill
// processes a prompt's tokens together ("vllm" 2.1 Prefill); batching prefill and decode tokens of
// different requests, with only attention aware of each token's request and phase, is Orca's
// selective batching ("Paged Attention&Orca Paper笔记与解读").  Decode is n_s = 1.
//
// Design: a work unit is (sequence, kv head, 112 query rows), a row being one (token, head) pair of
// the head group, so a unit covers 112/g tokens and all g heads that share the kv head.  One
// producer warp streams the unit's key range [0, last position] in 64-token tiles with 2-D TMA loads
// (the same tensor maps as decode); seven consumer warps own 16 rows each (their query rows staged
// once per unit in shared memory) and run
// S = Q K^T and O += P V on tensor cores (mma.sync m16n8k16, fp32 accumulators), P fed back as a
// 16-bit hi + lo pair, with the online softmax per row in fp32.  Causal masking compares each
// key's position with the row's own position.  Every warp finishes its rows alone, so there is
// no cross-warp merge; units are listed longest key range first.
#include <atomic>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <utility>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace {

constexpr int kTile = 64;     // key tokens per stage
constexpr int kCW = 7;        // consumer warps (with the producer: 8 warps, 256 threads)
constexpr int kThreads = (kCW + 1) * 32;
constexpr int kRows = kCW * 16;  // query rows per unit
constexpr int kPlanThreads = 1024;
constexpr int kBuckets = 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kHdrCounter = 0, kHdrNumItems = 1, kHdrError = 2;
constexpr size_t kHdrBytes = 256;

enum : int { kFirst = 1, kLast = 2, kDone = 4 };

struct __align__(16) Meta {
  int s, kh, q_row0, qpos0, nq, tile_pos, ntok, flags;
};

struct Args {
  const void* q;
  void* out;
  int out_dtype;
  const int32_t* q_start;
  const int32_t* bt;
  const int32_t* lens;
  int S, H, Hk, max_blocks, n_blocks, B, max_c, max_q, QT;
  int route_single;  // sequences with one query token are left to the decode kernels
  float scale_log2;
  const int2* items;
  int* hdr;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int tokens_per_unit(int g) { return kRows / g; }  // the smaller of the two unit sizes

size_t max_units(int S, int Hk, int g, int max_q_len) {
  const int QT = tokens_per_unit(g);
  return static_cast<size_t>(S) * Hk * static_cast<size_t>((max_q_len + QT - 1) / QT);
}

// Length of query chunk and context of sequence s, checked: 0 <= n <= min(c, max_q), c <= max_c.
// Out-of-range values are cut to the bounds (and reported), so no index leaves its buffer.
__device__ __forceinline__ void seq_sizes(const Args& a, int s, int& n, int& c, bool& bad) {
  n = a.q_start[s + 1] - a.q_start[s];
  c = a.lens[s];
  bad = n < 0 || c > a.max_c || n > c || n > a.max_q || a.q_start[s] < 0;
  if (a.q_start[s] < 0) n = 0;  // a negative row offset would index below the query buffer
  c = min(max(c, 0), a.max_c);
  n = min(min(max(n, 0), c), a.max_q);
}

__device__ __forceinline__ int bucket_of(int kv_end, int max_c) {
  const int tiles = (kv_end + kTile - 1) / kTile, max_tiles = max(1, (max_c + kTile - 1) / kTile);
  const int nb = min(max_tiles, kBuckets);
  return tiles <= 1 ? 0 : min(nb - 1, ((tiles - 1) * nb) / max_tiles);
}

// Units (s, kh, q-tile), longest key range first (64 buckets of key tiles, atomic cursors).
__global__ void __launch_bounds__(kPlanThreads) prefill_plan_kernel(Args a, int2* __restrict__ items) {
  pa::grid_dependency_launch();
  pa::grid_dependency_wait();
  __shared__ int count[kBuckets], cursor[kBuckets];
  const int tid = threadIdx.x;
  const int max_tiles = max(1, (a.max_c + kTile - 1) / kTile), nb = min(max_tiles, kBuckets);
  for (int b = tid; b < kBuckets; b += kPlanThreads) count[b] = 0;
  __syncthreads();
  bool bad_any = false;
  for (int s = tid; s < a.S; s += kPlanThreads) {
    int n, c;
    bool bad;
    seq_sizes(a, s, n, c, bad);
    bad_any |= bad;
    if (a.route_single && n == 1) continue;
    for (int t0 = 0; t0 < n; t0 += a.QT) atomicAdd(&count[bucket_of(c - n + min(t0 + a.QT, n), a.max_c)], a.Hk);
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int b = nb - 1; b >= 0; --b) {
      cursor[b] = run;
      run += count[b];
    }
    a.hdr[kHdrCounter] = 0;
    a.hdr[kHdrNumItems] = run;
  }
  __syncthreads();
  for (int s = tid; s < a.S; s += kPlanThreads) {
    int n, c;
    bool bad;
    seq_sizes(a, s, n, c, bad);
    if (a.route_single && n == 1) continue;
    for (int t0 = 0, qt = 0; t0 < n; t0 += a.QT, ++qt) {
      const int base = atomicAdd(&cursor[bucket_of(c - n + min(t0 + a.QT, n), a.max_c)], a.Hk);
      for (int kh = 0; kh < a.Hk; ++kh) items[base + kh] = make_int2(s, (kh << 16) | qt);
    }
  }
  const int any = __syncthreads_or(bad_any);
  if (tid == 0) a.hdr[kHdrError] = any ? pa::kErrBadLength : 0;
}

template <int D>
struct PCfg {
  static constexpr int kNPanel = D / 64;  // 128-byte panels of 16-bit elements
  static constexpr int kPanelBytes = kTile * 128;
  static constexpr int kKVBytes = kNPanel * kPanelBytes;
  static constexpr int kStageBytes = 2 * kKVBytes;
  static constexpr int kStages = kNPanel == 1 ? 6 : 3;
  static constexpr int kOffQ = kStages * kStageBytes;      // [4 warps][16 rows][D], 16-byte chunks
  static constexpr int kQWarpBytes = 16 * D * 2;           // swizzled by row: chunk ^ (row & 7)
  static constexpr int kOffMeta = kOffQ + kCW * kQWarpBytes;
  static constexpr int kOffBar = kOffMeta + kStages * static_cast<int>(sizeof(Meta));
  static constexpr int kSmemBytes = kOffBar + 2 * kStages * 8 + 1024;
};

template <class OutT>
__device__ __forceinline__ void store_pair(OutT* p, float x0, float x1) {
  if constexpr (sizeof(OutT) == 4) {
    *reinterpret_cast<float2*>(p) = make_float2(x0, x1);
  } else {
    OutT t[2] = {pa::from_float<OutT>(x0), pa::from_float<OutT>(x1)};
    *reinterpret_cast<uint32_t*>(p) = *reinterpret_cast<const uint32_t*>(t);
  }
}

// The producer warp: pulls units, streams each unit's causal key range [0, last position] in
// 64-token tiles (one 2-D TMA box per block and 128-byte panel, for K and for V) into the stage
// ring, with the unit's geometry in the stage's Meta; signals kDone when the units run out.
template <int D, class C>
__device__ __forceinline__ void produce_units(uint8_t* smem, Meta* meta, uint64_t* full, uint64_t* empty,
                                              const CUtensorMap& tmK, const CUtensorMap& tmV, const Args& a,
                                              int lane) {
  int stage = 0, issued = 0;
  uint32_t phase = 0;
  const int n_items = a.hdr[kHdrNumItems];
  bool ok = true;
  while (ok) {
    int k = 0;
    if (lane == 0) k = atomicAdd(a.hdr + kHdrCounter, 1);
    k = __shfl_sync(0xffffffffu, k, 0);
    if (k >= n_items) {
      if (!pa::mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
      if (lane == 0) {
        meta[stage].flags = kDone;
        pa::mbar_arrive(&full[stage]);
      }
      break;
    }
    const int2 it = a.items[k];
    const int s = it.x, kh = it.y >> 16, qt = it.y & 0xffff;
    int n, c;
    bool bad;
    seq_sizes(a, s, n, c, bad);
    const int tok0 = qt * a.QT, tok1 = min(tok0 + a.QT, n);
    const int kv_end = c - n + tok1;  // keys 0 .. kv_end-1
    const int ntiles = max(1, (kv_end + kTile - 1) / kTile);
    const int32_t* bt_row = a.bt + static_cast<size_t>(s) * a.max_blocks;
    for (int tile = 0; tile < ntiles; ++tile) {
      if (!pa::mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
      const int pos0 = tile * kTile;
      const int ntok = max(0, min(kTile, kv_end - pos0));
      const int nblk = (ntok + a.B - 1) / a.B;
      const int j0 = pos0 / a.B;
      int phys = -1;
      if (lane < nblk) {
        phys = __ldg(bt_row + j0 + lane);
        if (phys < 0 || phys >= a.n_blocks) {
          atomicOr(a.hdr + kHdrError, pa::kErrBadBlock);
          phys = -1;
        }
      }
      if (lane == 0) {
        Meta m;
        m.s = s;
        m.kh = kh;
        m.q_row0 = a.q_start[s] + tok0;
        m.qpos0 = c - n + tok0;
        m.nq = tok1 - tok0;
        m.tile_pos = pos0;
        m.ntok = ntok;
        m.flags = (tile == 0 ? kFirst : 0) | (tile == ntiles - 1 ? kLast : 0);
        meta[stage] = m;
        pa::mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(nblk) * a.B * D * 2u * 2u);
      }
      __syncwarp();
      uint8_t* kdst = smem + stage * C::kStageBytes;
      uint8_t* vdst = kdst + C::kKVBytes;
      if (lane < nblk) {
        const int y = (phys * a.Hk + kh) * a.B;
#pragma unroll
        for (int p = 0; p < C::kNPanel; ++p) {
          pa::tma_load_2d(kdst + p * C::kPanelBytes + lane * a.B * 128, &tmK, p * 64, y, &full[stage]);
          pa::tma_load_2d(vdst + p * C::kPanelBytes + lane * a.B * 128, &tmV, p * 64, y, &full[stage]);
        }
      }
      ++issued;
      if (++stage == C::kStages) {
        stage = 0;
        phase ^= 1;
      }
    }
  }
  if (!ok) {
    if (lane == 0) atomicOr(a.hdr + kHdrError, pa::kErrWaitTimeout);
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
}

template <class T, int D, int G>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(const __grid_constant__ CUtensorMap tmK,
                                                           const __grid_constant__ CUtensorMap tmV, const Args a) {
  using C = PCfg<D>;
  using M = pa::Mma<T>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Meta* meta = reinterpret_cast<Meta*>(smem + C::kOffMeta);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + C::kStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      pa::mbar_init(&full[i], 1);
      pa::mbar_init(&empty[i], kCW);
    }
    pa::fence_barrier_init();
  }
  __syncthreads();
  pa::grid_dependency_wait();

  if (warp == kCW) {
    produce_units<D, C>(smem, meta, full, empty, tmK, tmV, a, lane);
    return;
  }

  // ================================== consumer warps ============================================
  constexpr int KS = D / 16;  // k-steps of q.k
  constexpr int DN = D / 8;   // 8-wide dim tiles of the output
  const int gq = lane >> 2, tq = lane & 3;
  // this thread's two rows (r, r + 8) of the warp's 16; row = token * G + head
  const int ra = warp * 16 + gq, rb = ra + 8;
  const int tok_a = ra / G, h_a = ra % G, tok_b = rb / G, h_b = rb % G;
  float o[DN][4];
  uint8_t* qw = smem + C::kOffQ + warp * C::kQWarpBytes;  // this warp's 16 query rows
  float m_run[2], l_run[2];
  int qpos_a = 0, qpos_b = 0, row_a = -1, row_b = -1, warp_qmax = -1;
  const int ld_tok = ((lane >> 4) << 3) + (lane & 7), ld_hi = (lane >> 3) & 1;   // K: (tok 0-7|8-15) x (lo|hi)
  const int ldv_tok = (((lane >> 3) & 1) << 3) + (lane & 7), ldv_hi = lane >> 4;  // V: (tok lo|hi) x (dim c|c+1)

  int stage = 0;
  uint32_t phase = 0;
  while (true) {
    if (!pa::mbar_wait(&full[stage], phase)) {
      if (lane == 0) atomicOr(a.hdr + kHdrError, pa::kErrWaitTimeout);
      return;
    }
    const Meta mt = meta[stage];
    if (mt.flags & kDone) break;
    const uint8_t* ks = smem + stage * C::kStageBytes;
    const uint8_t* vs = ks + C::kKVBytes;

    if (mt.flags & kFirst) {
      const bool va = tok_a < mt.nq, vb = tok_b < mt.nq;
      qpos_a = mt.qpos0 + tok_a;
      qpos_b = mt.qpos0 + tok_b;
      row_a = va ? (mt.q_row0 + tok_a) * a.H + mt.kh * G + h_a : -1;
      row_b = vb ? (mt.q_row0 + tok_b) * a.H + mt.kh * G + h_b : -1;
      warp_qmax = -1;
      if (warp * 16 / G < mt.nq) warp_qmax = mt.qpos0 + min(mt.nq - 1, (warp * 16 + 15) / G);
      // stage the warp's 16 query rows in shared memory (zeros for rows past the chunk)
      {
        constexpr int CH = D / 8;  // 16-byte chunks per row
        const uint4* q16 = static_cast<const uint4*>(a.q);
        for (int i = lane; i < 16 * CH; i += 32) {
          const int r = i / CH, c = i % CH;
          const int rr = warp * 16 + r, tok = rr / G;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (tok < mt.nq) v = __ldg(q16 + (static_cast<size_t>((mt.q_row0 + tok) * a.H + mt.kh * G + rr % G) * D) / 8 + c);
          *reinterpret_cast<uint4*>(qw + r * (D * 2) + ((c ^ (r & 7)) << 4)) = v;
        }
        __syncwarp();
      }
#pragma unroll
      for (int i = 0; i < DN; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
      m_run[0] = m_run[1] = -INFINITY;
      l_run[0] = l_run[1] = 0.f;
    }

    // skip tiles wholly after this warp's last query position (or warps with no rows)
    if (warp_qmax >= mt.tile_pos && mt.ntok > 0) {
      // ---- S = Q K^T for 16 rows x 64 keys ----
      float sacc[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[j][e] = 0.f;
      const uint32_t kbase = pa::smem_addr(ks);
      const uint32_t qbase = pa::smem_addr(qw);
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        uint32_t aq[4];  // A fragment: (rows 0-7 | 8-15) x (dims lo | hi) of this k-step
        {
          const int r = ((lane >> 3) & 1) * 8 + (lane & 7), c = 2 * k + (lane >> 4);
          pa::ldsm_x4(aq, qbase + r * (D * 2) + ((c ^ (r & 7)) << 4));
        }
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          const int row = np * 16 + ld_tok, c = 2 * k + ld_hi;
          uint32_t bf[4];
          pa::ldsm_x4(bf, kbase + (c >> 3) * C::kPanelBytes + row * 128 + (((c & 7) ^ (row & 7)) << 4));
          const uint32_t b0[2] = {bf[0], bf[1]}, b1[2] = {bf[2], bf[3]};
          M::run(sacc[2 * np], aq, b0);
          M::run(sacc[2 * np + 1], aq, b1);
        }
      }
      // ---- causal mask, online softmax (rows a: e = 0,1; b: e = 2,3) ----
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = j * 8 + 2 * tq + (e & 1);
          const int kp = mt.tile_pos + t;
          const bool ok = t < mt.ntok && kp <= ((e < 2) ? qpos_a : qpos_b) && ((e < 2) ? row_a : row_b) >= 0;
          sacc[j][e] = ok ? sacc[j][e] * a.scale_log2 : -INFINITY;
          mx[e >> 1] = fmaxf(mx[e >> 1], sacc[j][e]);
        }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      }
      float alpha[2], mn[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mn[r] = fmaxf(m_run[r], mx[r]);
        alpha[r] = (mn[r] == -INFINITY) ? 1.f : exp2f(m_run[r] - mn[r]);
        m_run[r] = mn[r];
        l_run[r] *= alpha[r];
      }
#pragma unroll
      for (int i = 0; i < DN; ++i) {
        o[i][0] *= alpha[0];
        o[i][1] *= alpha[0];
        o[i][2] *= alpha[1];
        o[i][3] *= alpha[1];
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float mr = mn[e >> 1];
          sacc[j][e] = mr == -INFINITY ? 0.f : exp2f(sacc[j][e] - mr);
          l_run[e >> 1] += sacc[j][e];
        }
      // ---- O += P V, P as a 16-bit hi + lo pair ----
      const bool partial = mt.ntok < kTile;
      const uint32_t vbase = pa::smem_addr(vs);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t ph[4], pl[4];
        float r0, r1, d0, d1;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float* src = sacc[2 * kk + (q >> 1)] + (q & 1) * 2;  // a0: row a lo toks, a1: row b, a2/a3: hi toks
          ph[q] = M::pack(src[0], src[1], r0, r1);
          pl[q] = M::pack(src[0] - r0, src[1] - r1, d0, d1);
        }
        uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
        if (partial) {
          const int t0 = kk * 16 + 2 * tq;
          mlo = (t0 < mt.ntok ? 0x0000ffffu : 0u) | (t0 + 1 < mt.ntok ? 0xffff0000u : 0u);
          mhi = (t0 + 8 < mt.ntok ? 0x0000ffffu : 0u) | (t0 + 9 < mt.ntok ? 0xffff0000u : 0u);
        }
#pragma unroll
        for (int dn = 0; dn < DN; dn += 2) {
          const int row = kk * 16 + ldv_tok, c = dn + ldv_hi;
          uint32_t vf[4];
          pa::ldsm_x4_trans(vf, vbase + (c >> 3) * C::kPanelBytes + row * 128 + (((c & 7) ^ (row & 7)) << 4));
          const uint32_t b0[2] = {vf[0] & mlo, vf[1] & mhi}, b1[2] = {vf[2] & mlo, vf[3] & mhi};
          M::run(o[dn], ph, b0);
          M::run(o[dn], pl, b0);
          M::run(o[dn + 1], ph, b1);
          M::run(o[dn + 1], pl, b1);
        }
      }
    }

    __syncwarp();
    if (lane == 0) pa::mbar_arrive(&empty[stage]);

    if (mt.flags & kLast) {
      float l[2] = {l_run[0], l_run[1]};
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
      }
      const float inv_a = l[0] > 0.f ? 1.f / l[0] : 0.f, inv_b = l[1] > 0.f ? 1.f / l[1] : 0.f;
#pragma unroll
      for (int dn = 0; dn < DN; ++dn) {
        const int col = dn * 8 + 2 * tq;
        if (a.out_dtype == PA_F32) {
          if (row_a >= 0) store_pair(static_cast<float*>(a.out) + static_cast<size_t>(row_a) * D + col, o[dn][0] * inv_a, o[dn][1] * inv_a);
          if (row_b >= 0) store_pair(static_cast<float*>(a.out) + static_cast<size_t>(row_b) * D + col, o[dn][2] * inv_b, o[dn][3] * inv_b);
        } else if (a.out_dtype == PA_F16) {
          if (row_a >= 0) store_pair(static_cast<__half*>(a.out) + static_cast<size_t>(row_a) * D + col, o[dn][0] * inv_a, o[dn][1] * inv_a);
          if (row_b >= 0) store_pair(static_cast<__half*>(a.out) + static_cast<size_t>(row_b) * D + col, o[dn][2] * inv_b, o[dn][3] * inv_b);
        } else {
          if (row_a >= 0) store_pair(static_cast<__nv_bfloat16*>(a.out) + static_cast<size_t>(row_a) * D + col, o[dn][0] * inv_a, o[dn][1] * inv_a);
          if (row_b >= 0) store_pair(static_cast<__nv_bfloat16*>(a.out) + static_cast<size_t>(row_b) * D + col, o[dn][2] * inv_b, o[dn][3] * inv_b);
        }
      }
    }
    if (++stage == C::kStages) {
      stage = 0;
      phase ^= 1;
    }
  }
}


// ---- tcgen05 consumers -------------------------------------------------------------------------------
// 256 query rows per unit in two 128-row halves A and B (one TMEM lane per row in each half).
// Warps 0-3 own the rows of half A, warps 4-7 those of half B (softmax, P, output); warp 8 is the
// TMA producer; one lane each of warps 9 and 10 issues the S MMAs of halves A and B, one lane each
// of warps 11 and 12 their P.V MMAs.  A single thread issues one tcgen05.mma about every 126-134
// cycles with A in shared memory and 166-186 with A in tensor memory, whatever its N up to 128
// (measured on B200), and separate issuing warps add up: four issuers keep up with the tensor core
// where one per half (about 2400 issue cycles per 64-key tile) did not.  Warp 9 also allocates TMEM.
// Per 64-key tile j and half h, in the TMEM buffer b = j mod 2 of that half:
//   S_h,b[128 x 64] = Q_h K_j^T              d/16 tcgen05.mma, A = Q tile, B = K tile (K-major)
//   the rows of h read S out of the buffer, mask causally, and write P (hi and lo 16-bit parts) back
//   into the same 64 columns
//   O_h[128 x d]  += P_hi V_j + P_lo V_j      A = P from TMEM, B = V tile (MN-major: d contiguous)
// The halves are independent pipelines that share the K/V ring.  With two buffers per half the
// rows never wait for a P.V product before writing P (P(j) replaces S(j), which they have just
// read); S(j+2) waits until P.V(j) has read P(j) out of buffer b, so S(j+1) is ready while the rows
// still work on tile j.  The running maximum is updated lazily: O_h (in TMEM) is rescaled only when
// a row's maximum grows by more than 2^8, which keeps every exponent bounded; only then do the rows
// wait for P.V(j-1).
constexpr int kURows = 128;                  // rows per half (TMEM lanes)
constexpr int kUHalves = 2;
constexpr int kUUnitRows = kURows * kUHalves;
constexpr int kUProducer = 8;
constexpr int kUMmaS = 9;                    // S issuers: warps 9 (half A) and 10 (half B)
constexpr int kUMmaPV = 11;                  // P.V issuers: warps 11 (half A) and 12 (half B)
constexpr int kUThreads = 16 * 32;          // four warpgroups: rows (2), producer + issuers, issuer + idle
// Registers: the CTA launches with 512 x 128.  The row warpgroups raise theirs to kRegsRows and the
// two others lower theirs to kRegsOther; 2 x 128 x (kRegsRows + kRegsOther) must not exceed
// 512 x 128, or the raise would wait for registers that are never released.
constexpr uint32_t kRegsRows = 200, kRegsOther = 56;
static_assert(2 * 128 * (kRegsRows + kRegsOther) <= 512 * 128, "register split exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;          // S/P buffers 64 (2h + b).., O_A 256.., O_B 256 + d..
constexpr uint32_t kTmemO = 256;             // P in a buffer: 32 columns of packed hi pairs, then 32 of lo pairs

template <int D>
struct UCfg {
  static constexpr int kNPanel = D / 64;
  static constexpr int kPanelBytes = kTile * 128;
  static constexpr int kKVBytes = kNPanel * kPanelBytes;
  static constexpr int kStageBytes = 2 * kKVBytes;
  static constexpr int kStages = kNPanel == 1 ? 8 : 5;
  static constexpr int kQPanelBytes = kURows * 128;
  static constexpr int kQHalfBytes = kNPanel * kQPanelBytes;
  static constexpr int kOffQ = kStages * kStageBytes;
  static constexpr int kOffMeta = kOffQ + kUHalves * kQHalfBytes;
  static constexpr int kOffBar = kOffMeta + kStages * static_cast<int>(sizeof(Meta));
  // full[S], empty[S], q_ready[2], then per (half, buffer): s_full, p_full, o_done; then teardown
  static constexpr int kNBars = 2 * kStages + kUHalves + 3 * 2 * kUHalves + 1;
  static constexpr int kOffTmem = kOffBar + kNBars * 8;
  static constexpr int kSmemBytes = kOffTmem + 16 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kTmemO + kUHalves * D <= static_cast<int>(kTmemCols), "TMEM columns: four S/P buffers and two O tiles");
};

template <class T, int D, int G>
__global__ void __launch_bounds__(kUThreads, 1) prefill_umma_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                    const __grid_constant__ CUtensorMap tmV,
                                                                    const Args a) {
  using C = UCfg<D>;
  constexpr bool kBF16 = sizeof(T) == 2 && !std::is_same<T, __half>::value;
  constexpr uint32_t kIdescS = pa::umma_idesc(kBF16, kURows, kTile, false, false);
  constexpr uint32_t kIdescO = pa::umma_idesc(kBF16, kURows, D, false, true);
  constexpr int KS = D / 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Meta* meta = reinterpret_cast<Meta*>(smem + C::kOffMeta);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + C::kStages;
  // per (half h, buffer b) at index 2h + b: barriers of one buffer complete once every two tiles,
  // so no waiter can fall two phases behind (tile j + 2 of a buffer needs tile j's P.V first)
  uint64_t* q_ready = empty + C::kStages;      // [2]
  uint64_t* s_full = q_ready + kUHalves;       // [4]: S(j) is in the buffer
  uint64_t* p_full = s_full + 2 * kUHalves;    // [4]: the rows have written P(j) into it
  uint64_t* o_done = p_full + 2 * kUHalves;    // [4]: P.V(j) has run (the buffer is free, O is current)
  uint64_t* teardown = o_done + 2 * kUHalves;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffTmem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      pa::mbar_init(&full[i], 1);
      pa::mbar_init(&empty[i], 2 * kUHalves);  // one tcgen05.commit per tile from each of the 4 issuers
    }
    for (int h = 0; h < kUHalves; ++h) pa::mbar_init(&q_ready[h], kURows);
    for (int i = 0; i < 2 * kUHalves; ++i) {
      pa::mbar_init(&s_full[i], 1);
      pa::mbar_init(&p_full[i], kURows);
      pa::mbar_init(&o_done[i], 1);
    }
    pa::mbar_init(teardown, kUUnitRows);
    pa::fence_barrier_init();
  }
  if (warp == kUMmaS) {
    pa::tmem_alloc(tmem_slot, kTmemCols);
    pa::tmem_relinquish();
  }
  pa::tc_fence_before();
  __syncthreads();
  pa::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pa::grid_dependency_wait();
  if (warp >= 8) {
    // every path of warps 8-15 ends in a return below: the row code after this block runs with the
    // raised budget only
    pa::setmaxnreg_dec<kRegsOther>();
    if (warp > kUMmaPV + 1) return;  // warps 13-15 only complete the last warpgroup

    if (warp == kUProducer) {
      produce_units<D, C>(smem, meta, full, empty, tmK, tmV, a, lane);
      return;
    }

    if (warp >= kUMmaS && warp < kUMmaS + 2) {
      // ================================ S issuers (one per half) ================================
      const int h = warp - kUMmaS;
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0, q_ph = 0;
        const uint32_t q_base = pa::smem_addr(smem + C::kOffQ) + h * C::kQHalfBytes;
        bool ok = true, active = false;
        // S = Q_h K^T over d in K = 16 steps, into buffer b of this half
        auto s_tile = [&](int st, int b) {
          const uint32_t kb = pa::smem_addr(smem + st * C::kStageBytes);
  #pragma unroll
          for (int k = 0; k < KS; ++k) {
            const uint64_t da = pa::sw128_desc(q_base + (k >> 2) * C::kQPanelBytes + (k & 3) * 32, 16, 1024);
            const uint64_t db = pa::sw128_desc(kb + (k >> 2) * C::kPanelBytes + (k & 3) * 32, 16, 1024);
            pa::umma_f16_ss(tmem + 64 * (2 * h + b), da, db, kIdescS, k > 0 ? 1u : 0u);
          }
        };
        // n counts this half's tiles over all units of the CTA; tile n uses buffer n & 1
        for (uint32_t n = 0;; ++n) {
          if (!pa::mbar_wait(&full[stage], phase)) { ok = false; break; }
          const Meta mt = meta[stage];
          if (mt.flags & kDone) break;
          if (mt.flags & kFirst) {
            // the unit's Q, staged by the rows once they have read the previous unit's last S
            if (!pa::mbar_wait(&q_ready[h], q_ph)) { ok = false; break; }
            q_ph ^= 1;
            // a half whose rows hold no query (a short unit, a ragged chunk end) gets no MMAs, but
            // its barriers are committed all the same so that both sides count the same phases
            active = h == 0 || mt.nq * G > kURows;
          }
          const int b = static_cast<int>(n & 1u);
          // the buffer is free once P.V(n - 2) has read its P
          if (n >= 2 && !pa::mbar_wait(&o_done[2 * h + b], ((n - 2) >> 1) & 1u)) { ok = false; break; }
          pa::tc_fence_after();
          if (active) s_tile(stage, b);
          pa::umma_commit(&s_full[2 * h + b]);
          pa::umma_commit(&empty[stage]);  // this half is done with the stage's K once S has run
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) atomicOr(a.hdr + kHdrError, pa::kErrWaitTimeout);
      }
      if (h == 1) return;
      __syncwarp();
      // free TMEM once the row threads are done with it (they wait for every MMA's result)
      pa::mbar_wait(teardown, 0);
      pa::tc_fence_after();
      pa::tmem_dealloc(tmem, kTmemCols);
      return;
    }

    if (warp >= kUMmaPV && warp < kUMmaPV + 2) {
      // ================================ P.V issuers (one per half) ==============================
      const int h = warp - kUMmaPV;
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        constexpr int kPV = 2 * (kTile / 16);
        for (uint32_t n = 0;; ++n) {
          if (!pa::mbar_wait(&full[stage], phase)) { ok = false; break; }
          const Meta mt = meta[stage];
          if (mt.flags & kDone) break;
          const bool active = h == 0 || mt.nq * G > kURows;
          const bool first = (mt.flags & kFirst) != 0;
          const int b = static_cast<int>(n & 1u);
          // O_h += P V: i over the hi keys, then the lo keys, in K = 16 steps; A = P from buffer b
          if (!pa::mbar_wait(&p_full[2 * h + b], (n >> 1) & 1u)) { ok = false; break; }
          pa::tc_fence_after();
          if (active) {
            const uint32_t vb = pa::smem_addr(smem + stage * C::kStageBytes) + C::kKVBytes;
  #pragma unroll
            for (int i = 0; i < kPV; ++i) {
              const int part = i / (kTile / 16), kk = i % (kTile / 16);
              const uint64_t db = pa::sw128_desc(vb + kk * 16 * 128, C::kPanelBytes, 1024);
              pa::umma_f16_tmem_a(tmem + kTmemO + D * h, tmem + 64 * (2 * h + b) + part * 32 + kk * 8, db, kIdescO,
                                  (first && i == 0) ? 0u : 1u);
            }
          }
          pa::umma_commit(&o_done[2 * h + b]);
          pa::umma_commit(&empty[stage]);  // and with the stage's V once P V has run
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) atomicOr(a.hdr + kHdrError, pa::kErrWaitTimeout);
      }
      return;
    }

    return;
  }  // warps 8-15

  // ================================== row threads (warps 0-7) =====================================
  pa::setmaxnreg_inc<kRegsRows>();
  const int half = warp >> 2;                         // 0: rows 0..127, 1: rows 128..255
  const int hr = (warp & 3) * 32 + lane;              // row within the half = TMEM lane
  const int r = half * kURows + hr;                   // row within the unit
  const int warp_row0 = half * kURows + (warp & 3) * 32;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t tSP = tmem + 64 * (2 * half), tO = tmem + kTmemO + D * half;
  uint8_t* qs = smem + C::kOffQ + half * C::kQHalfBytes;
  uint64_t* my_q_ready = &q_ready[half];
  int stage = 0;
  uint32_t phase = 0;
  float m_used = -INFINITY, l = 0.f;
  int row_global = -1, qpos = 0;
  bool ok = true, warp_active = false;
  const float sl2 = a.scale_log2 == 0.f ? 1.f : fabsf(a.scale_log2);
  // n counts this half's tiles over all units of the CTA, as the issuers do: tile n is in buffer
  // b = n & 1, whose barriers complete for the (n >> 1)-th time
  // Only a unit's first tile needs the producer's meta: the rows derive the others' position,
  // length and last-tile flag from it, and wait for a stage's data only where they write into it
  // (the zeroed V rows of a ragged last tile).
  Meta mt;
  mt.flags = kLast;  // the next tile starts a unit
  for (uint32_t n = 0;; ++n) {
    const int b = static_cast<int>(n & 1u);
    const uint32_t nph = (n >> 1) & 1u;
    if (mt.flags & kLast) {
      if (!pa::mbar_wait(&full[stage], phase)) { ok = false; break; }
      mt = meta[stage];
    } else {
      mt.tile_pos += kTile;
      const int kv_end = mt.qpos0 + mt.nq;  // keys 0 .. kv_end-1 for the unit's queries
      mt.ntok = min(kTile, kv_end - mt.tile_pos);
      mt.flags = mt.tile_pos + kTile >= kv_end ? kLast : 0;
      if (mt.ntok < kTile && !pa::mbar_wait(&full[stage], phase)) { ok = false; break; }
    }
    if (mt.flags & kDone) break;
    if (mt.flags & kFirst) {
      const int tok = r / G, h = r % G;
      const bool valid = tok < mt.nq;
      qpos = mt.qpos0 + tok;
      row_global = valid ? (mt.q_row0 + tok) * a.H + mt.kh * G + h : -1;
      // a warp none of whose rows holds a query skips the arithmetic (its S, P and O are unused)
      // but keeps to the barrier protocol
      warp_active = mt.nq * G > warp_row0;
      const uint4* src = static_cast<const uint4*>(a.q) + static_cast<size_t>(valid ? row_global : 0) * (D / 8);
      // the scale's sign is carried by q (exact: a sign flip, or zero for scale 0), so that the
      // row maximum can be taken before scaling by sl2 >= 0
      const uint32_t q_flip = a.scale_log2 < 0.f ? 0x80008000u : 0u;
      const bool q_keep = valid && a.scale_log2 != 0.f;
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        uint4 v = q_keep ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
        v.x ^= q_flip;
        v.y ^= q_flip;
        v.z ^= q_flip;
        v.w ^= q_flip;
        *reinterpret_cast<uint4*>(qs + (c >> 3) * C::kQPanelBytes + hr * 128 + (((c & 7) ^ (hr & 7)) << 4)) = v;
      }
      pa::fence_proxy_async_smem();
      pa::mbar_arrive(my_q_ready);
      m_used = -INFINITY;
      l = 0.f;
    }
    // keys past the tile's valid ones get p = 0; zero their V rows, which may hold stale or unused
    // data.  Each half does it before its own P.V product is issued (the two write the same zeros),
    // and makes the writes visible to the tensor core.
    if (mt.ntok < kTile) {
      uint8_t* vs = smem + stage * C::kStageBytes + C::kKVBytes;
      for (int i = hr; i < (kTile - mt.ntok) * (D / 8); i += kURows) {
        const int row = mt.ntok + i / (D / 8), c = i % (D / 8);
        *reinterpret_cast<uint4*>(vs + (c >> 3) * C::kPanelBytes + row * 128 + (((c & 7) ^ (row & 7)) << 4)) =
            make_uint4(0u, 0u, 0u, 0u);
      }
      pa::fence_proxy_async_smem();
    }
    if (!pa::mbar_wait(&s_full[2 * half + b], nph)) { ok = false; break; }
    pa::tc_fence_after();
    float sv[kTile];
    if (warp_active) pa::tmem_ld64(tSP + 64 * b + lane_base, sv);  // waits for the load: P may replace S
    uint32_t hi[kTile / 2], lo[kTile / 2];
    float f = 1.f;
    bool rescale = false;
    if (warp_active) {
      // causal and length masking only on tiles that reach past the unit's first query position
      // or past the context (the same decision for the whole unit)
      if (mt.ntok < kTile || mt.tile_pos + kTile - 1 > mt.qpos0) {
        const int cut = row_global < 0 ? 0 : min(qpos - mt.tile_pos + 1, mt.ntok);
#pragma unroll
        for (int c = 0; c < kTile; ++c) sv[c] = c < cut ? sv[c] : -INFINITY;
      }
      // row maximum with three-input max: 64 -> 22 -> 8 -> 3 -> 1
      float m22[22];
#pragma unroll
      for (int i = 0; i < 21; ++i) m22[i] = pa::max3(sv[3 * i], sv[3 * i + 1], sv[3 * i + 2]);
      m22[21] = sv[63];
      float m8[8];
#pragma unroll
      for (int i = 0; i < 7; ++i) m8[i] = pa::max3(m22[3 * i], m22[3 * i + 1], m22[3 * i + 2]);
      m8[7] = m22[21];
      const float mx = pa::max3(pa::max3(m8[0], m8[1], m8[2]), pa::max3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])) * sl2;
      // the running maximum moves only when it grows by more than 2^8; O is then rescaled by f
      // (below, once P.V(j-1) is done), decided per warp because tcgen05.ld/st are warp-collective
      if (mx > m_used + 8.f) {
        if (m_used != -INFINITY) f = pa::ex2(m_used - mx);
        l *= f;
        m_used = mx;
      }
      rescale = !(mt.flags & kFirst) && __any_sync(0xffffffffu, f != 1.f);
      // p = 2^(s * sl2 - m); with no visible key so far every s is -inf and p = 0
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      // two keys per packed instruction for the scaling, the row sum and the lo parts
      const uint64_t sc2 = pa::f2_pack(sl2, sl2), nm2 = pa::f2_pack(neg_m, neg_m);
      uint64_t ls2[2] = {pa::f2_pack(0.f, 0.f), pa::f2_pack(0.f, 0.f)};
#pragma unroll
      for (int k2 = 0; k2 < kTile / 2; ++k2) {
        float x0, x1;
        pa::f2_unpack(pa::f2_fma(pa::f2_pack(sv[2 * k2], sv[2 * k2 + 1]), sc2, nm2), x0, x1);
        const float p0 = pa::ex2(x0), p1 = pa::ex2(x1);
        const uint64_t p2 = pa::f2_pack(p0, p1);
        ls2[k2 & 1] = pa::f2_add(ls2[k2 & 1], p2);
        pa::Split2<T>::run(p0, p1, p2, hi[k2], lo[k2]);
      }
      float l0, l1, l2v, l3;
      pa::f2_unpack(ls2[0], l0, l1);
      pa::f2_unpack(ls2[1], l2v, l3);
      l += (l0 + l1) + (l2v + l3);
    }
    // O is rescaled once P.V(n-1) has added to it (a warp-uniform decision; a warp with nothing to
    // rescale does not wait)
    if (rescale) {
      if (!pa::mbar_wait(&o_done[2 * half + (b ^ 1)], ((n - 1) >> 1) & 1u)) { ok = false; break; }
      pa::tc_fence_after();
    }
    if (warp_active) {
      if (rescale) {
#pragma unroll 1
        for (int j = 0; j < D / 16; ++j) {
          float t[16];
          pa::tmem_ld16(tO + lane_base + 16 * j, t);
#pragma unroll
          for (int e = 0; e < 16; ++e) t[e] *= f;
          pa::tmem_st16(tO + lane_base + 16 * j, t);
        }
      }
      pa::tmem_st32(tSP + 64 * b + lane_base, hi);
      pa::tmem_st32(tSP + 64 * b + lane_base + 32, lo);
      pa::tmem_wait_st();
    }
    pa::tc_fence_before();
    pa::mbar_arrive(&p_full[2 * half + b]);
    if (mt.flags & kLast) {
      if (!pa::mbar_wait(&o_done[2 * half + b], nph)) { ok = false; break; }
      pa::tc_fence_after();
      if (warp_active) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
        for (int j = 0; j < D / 16; ++j) {
          float t[16];
          pa::tmem_ld16(tO + lane_base + 16 * j, t);
#pragma unroll
          for (int e = 0; e < 16; ++e) t[e] *= inv;
          if (row_global >= 0) {
            const size_t off = static_cast<size_t>(row_global) * D + 16 * j;
            if (a.out_dtype == PA_F32) pa::store_floats<float, 16>(static_cast<float*>(a.out) + off, t);
            else if (a.out_dtype == PA_F16) pa::store_floats<__half, 16>(static_cast<__half*>(a.out) + off, t);
            else pa::store_floats<__nv_bfloat16, 16>(static_cast<__nv_bfloat16*>(a.out) + off, t);
          }
        }
      }
    }
    if (++stage == C::kStages) {
      stage = 0;
      phase ^= 1;
    }
  }
  if (!ok && lane == 0) atomicOr(a.hdr + kHdrError, pa::kErrWaitTimeout);
  pa::tc_fence_before();
  pa::mbar_arrive(teardown);
}

// ---- host side ----------------------------------------------------------------------------------

template <class... KArgs, class... Args2>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args2&&... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args2>(args)...);
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
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

bool cache_map(CUtensorMap* map, const void* base, pa_dtype dt, int d, long long rows, int B) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t gdim[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  cuuint64_t gstride[1] = {static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(B)};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, dt == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
             const_cast<void*>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class T, int D, int G>
cudaError_t launch(const CUtensorMap& tk, const CUtensorMap& tv, const Args& a, long long units, cudaStream_t st) {
  using C = PCfg<D>;
  // per context: the shared-memory attribute is kept per device and lost with a device reset
  static std::atomic<unsigned long long> ready_ctx{0};
  static std::atomic<int> occupancy{1};
  const unsigned long long ctx = pa::current_context_id();
  if (ctx == 0 || ready_ctx.load(std::memory_order_acquire) != ctx) {
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, prefill_kernel<T, D, G>, kThreads, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    occupancy.store(occ < 1 ? 1 : occ, std::memory_order_relaxed);
    ready_ctx.store(pa::current_context_id(), std::memory_order_release);
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long grid = static_cast<long long>(sms) * occupancy.load(std::memory_order_relaxed);
  if (grid > units) grid = units;
  if (grid < 1) grid = 1;
  return launch_pdl(prefill_kernel<T, D, G>, dim3(static_cast<unsigned>(grid)), dim3(kThreads), C::kSmemBytes, st,
                    tk, tv, a);
}

template <class T, int D, int G>
cudaError_t launch_umma(const CUtensorMap& tk, const CUtensorMap& tv, const Args& a, long long units, cudaStream_t st) {
  using C = UCfg<D>;
  static std::atomic<unsigned long long> ready_ctx{0};  // per context, as in launch()
  const unsigned long long ctx = pa::current_context_id();
  if (ctx == 0 || ready_ctx.load(std::memory_order_acquire) != ctx) {
    cudaError_t e = cudaFuncSetAttribute(prefill_umma_kernel<T, D, G>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    // The warpgroups' register split must fit in what the CTA is launched with, or the row
    // warpgroups' setmaxnreg.inc would wait for ever: refuse to launch otherwise.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, prefill_umma_kernel<T, D, G>);
    if (e != cudaSuccess) return e;
    if (static_cast<long long>(fa.numRegs) * kUThreads < 2LL * 128 * (kRegsRows + kRegsOther))
      return cudaErrorInvalidConfiguration;
    ready_ctx.store(pa::current_context_id(), std::memory_order_release);
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long grid = sms;  // one CTA per SM: its shared memory and TMEM allocation are sized for that
  if (grid > units) grid = units;
  if (grid < 1) grid = 1;
  return launch_pdl(prefill_umma_kernel<T, D, G>, dim3(static_cast<unsigned>(grid)), dim3(kUThreads),
                    C::kSmemBytes, st, tk, tv, a);
}

// tcgen05 consumers unless PA_PREFILL_CONSUMER=mma_sync.
bool use_umma() {
  const char* v = std::getenv("PA_PREFILL_CONSUMER");
  return !(v && std::strcmp(v, "mma_sync") == 0);
}

int rows_per_unit() { return use_umma() ? kUUnitRows : kRows; }

template <class T, int D>
cudaError_t dispatch(int g, const CUtensorMap& tk, const CUtensorMap& tv, const Args& a, long long units, cudaStream_t st) {
  if (use_umma()) {
    switch (g) {
      case 1: return launch_umma<T, D, 1>(tk, tv, a, units, st);
      case 2: return launch_umma<T, D, 2>(tk, tv, a, units, st);
      case 4: return launch_umma<T, D, 4>(tk, tv, a, units, st);
      default: return launch_umma<T, D, 8>(tk, tv, a, units, st);
    }
  }
  switch (g) {
    case 1: return launch<T, D, 1>(tk, tv, a, units, st);
    case 2: return launch<T, D, 2>(tk, tv, a, units, st);
    case 4: return launch<T, D, 4>(tk, tv, a, units, st);
    default: return launch<T, D, 8>(tk, tv, a, units, st);
  }
}

// The prefill kernel's header and unit list, then the decode workspace of the one-token sequences.
size_t prefill_part_bytes(int S, int H, int Hk, int max_q_len) {
  return align_up(kHdrBytes + sizeof(int2) * max_units(S, Hk, H / Hk, max_q_len), 256);
}

}  // namespace

extern "C" size_t pa_prefill_workspace_size(int S, int H, int Hk, int d, int max_context_len, int max_q_len) {
  if (S < 0 || H <= 0 || Hk <= 0 || H % Hk != 0 || max_q_len < 0 || max_context_len < 0 || d <= 0) return 0;
  return prefill_part_bytes(S, H, Hk, max_q_len) + pa::decode_single_rows_workspace(S, H, Hk, d, max_context_len);
}

extern "C" pa_status pa_prefill(void* out, pa_dtype out_dtype, const void* query, const int32_t* q_start,
                                const void* k_cache, const void* v_cache, const int32_t* block_tables,
                                const int32_t* context_lens, int S, int H, int Hk, int d, int B, int n_blocks,
                                int max_blocks_per_seq, int max_context_len, int max_q_len, float scale,
                                pa_dtype kv_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  if (S < 0 || H <= 0 || Hk <= 0 || n_blocks <= 0 || max_blocks_per_seq < 0 || max_context_len < 0 || max_q_len < 0)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_prefill: bad sizes");
  if (H % Hk != 0) return pa::fail(PA_ERR_INVALID_ARG, "pa_prefill: H (%d) must be a multiple of Hk (%d)", H, Hk);
  const int g = H / Hk;
  if (g != 1 && g != 2 && g != 4 && g != 8) return pa::fail(PA_ERR_UNSUPPORTED, "pa_prefill: H/Hk = %d not in {1,2,4,8}", g);
  if (d != 64 && d != 128) return pa::fail(PA_ERR_UNSUPPORTED, "pa_prefill: d = %d not in {64,128}", d);
  if (B != 8 && B != 16 && B != 32) return pa::fail(PA_ERR_UNSUPPORTED, "pa_prefill: B = %d not in {8,16,32}", B);
  if (kv_dtype != PA_F16 && kv_dtype != PA_BF16) return pa::fail(PA_ERR_UNSUPPORTED, "pa_prefill: caches must be fp16 or bf16");
  if (!pa::valid_dtype(out_dtype)) return pa::fail(PA_ERR_INVALID_ARG, "pa_prefill: unknown output type");
  if (!std::isfinite(scale)) return pa::fail(PA_ERR_INVALID_ARG, "pa_prefill: scale must be finite");
  if (static_cast<long long>(max_blocks_per_seq) * B < max_context_len)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_prefill: max_blocks_per_seq * B < max_context_len");
  const long long rows = static_cast<long long>(n_blocks) * Hk * B;
  const long long units = static_cast<long long>(max_units(S, Hk, g, max_q_len));
  if (rows >= (1ll << 31) || units >= (1ll << 30) || (max_q_len + tokens_per_unit(g) - 1) / tokens_per_unit(g) > 0xffff)
    return pa::fail(PA_ERR_UNSUPPORTED, "pa_prefill: problem too large for 32-bit indices");
  if (S == 0 || max_q_len == 0) return pa::ok();
  if (!out || !query || !q_start || !k_cache || !v_cache || !block_tables || !context_lens || !workspace)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_prefill: null pointer");
  if (!pa::aligned16(out) || !pa::aligned16(query) || !pa::aligned16(k_cache) || !pa::aligned16(v_cache))
    return pa::fail(PA_ERR_INVALID_ARG, "pa_prefill: tensors must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return pa::fail(PA_ERR_INVALID_ARG, "pa_prefill: workspace must be 256-byte aligned");
  const size_t need = pa_prefill_workspace_size(S, H, Hk, d, max_context_len, max_q_len);
  if (workspace_bytes < need) return pa::fail(PA_ERR_INVALID_ARG, "pa_prefill: workspace of %zu bytes < %zu needed", workspace_bytes, need);
  CUtensorMap tk, tv;
  if (!cache_map(&tk, k_cache, kv_dtype, d, rows, B) || !cache_map(&tv, v_cache, kv_dtype, d, rows, B))
    return pa::fail(PA_ERR_CUDA, "pa_prefill: could not encode the cache tensor maps");
  Args a;
  a.q = query;
  a.out = out;
  a.out_dtype = out_dtype;
  a.q_start = q_start;
  a.bt = block_tables;
  a.lens = context_lens;
  a.S = S;
  a.H = H;
  a.Hk = Hk;
  a.max_blocks = max_blocks_per_seq;
  a.n_blocks = n_blocks;
  a.B = B;
  a.max_c = max_context_len;
  a.max_q = max_q_len;
  a.QT = rows_per_unit() / g;  // the workspace is sized for the smaller unit (more units)
  a.scale_log2 = scale * kLog2e;
  a.route_single = 1;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.hdr = reinterpret_cast<int*>(ws);
  a.items = reinterpret_cast<const int2*>(ws + kHdrBytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_pdl(prefill_plan_kernel, dim3(1), dim3(kPlanThreads), 0, st, a,
                             reinterpret_cast<int2*>(ws + kHdrBytes));
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_prefill: plan launch failed: %s", cudaGetErrorString(e));
  if (max_q_len > 1) {  // with at most one query token per sequence the decode kernels do all of it
    if (kv_dtype == PA_F16)
      e = d == 64 ? dispatch<__half, 64>(g, tk, tv, a, units, st) : dispatch<__half, 128>(g, tk, tv, a, units, st);
    else
      e = d == 64 ? dispatch<__nv_bfloat16, 64>(g, tk, tv, a, units, st)
                  : dispatch<__nv_bfloat16, 128>(g, tk, tv, a, units, st);
    if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_prefill: launch failed: %s", cudaGetErrorString(e));
  }
  // The sequences with one query token (decode rows of a mixed batch): the decode kernels, which
  // stream their context at the HBM rate instead of spending a 128-row tensor-core tile on g rows.
  const size_t off = prefill_part_bytes(S, H, Hk, max_q_len);
  return pa::decode_single_rows(out, out_dtype, query, q_start, k_cache, v_cache, block_tables, context_lens, S, H, Hk,
                                d, B, n_blocks, max_blocks_per_seq, max_context_len, scale, kv_dtype, ws + off,
                                workspace_bytes - off, a.hdr + kHdrError, stream);
}

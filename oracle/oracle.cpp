// Oracle for paged decode attention and its companion paths -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, obviously correct fp64 CPU restatement of what the pages define.  Only the
// tests, the smoke check and the benchmark's CPU-baseline leg may load this library; the
// product path never does.  It shares no source with the CUDA library: element decoding,
// indexing and the attention arithmetic are all written out again here.
//
// Sources (page title, section, equation):
//   [P2-KV]    "PagedAttention原理", section "为什么会有 KV cache", eq. o_t = softmax(q_t K^T/sqrt(d)) V
//   [P2-BLK]   "PagedAttention原理", section "实现一个虚拟内存", eqs. K_j, V_j, A_ij, o_i
//   [P2-TABLE] "PagedAttention原理", section "实现一个虚拟内存", block-table figure caption
//              (each logical block maps to a physical block and records how many slots it fills)
//   [P2-COW]   "PagedAttention原理", section "解决COW", five-step copy-on-write list
//   [P4-DEC]   "vllm" (cnblogs), section 2.2 Decode: each decode step stores the new token's K,V
//
// Readings taken where the pages leave a step open:
//   * query head h reads kv head h / g with g = H / Hk (grouped-query attention, contiguous groups);
//   * the last block of a sequence holds c - (nb-1)*B valid tokens; only t < c contributes;
//   * the score scale is passed in (1/sqrt(d) by default);
//   * c = 0 gives an all-zero output and reads no block table entry;
//   * a slot id < 0 in a slot mapping means "padding, write nothing".
//
// Element types are coded 0 = fp32, 1 = fp16, 2 = bf16.  Every element is converted to double
// exactly, so the only rounding is that of the fp64 arithmetic itself.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---- exact element decoding --------------------------------------------------------------

double half_bits_to_double(uint16_t h) {
  // IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
  const int sign = (h >> 15) & 1;
  const int expo = (h >> 10) & 0x1f;
  const int frac = h & 0x3ff;
  double mag;
  if (expo == 0) {
    mag = std::ldexp(static_cast<double>(frac), -24);  // subnormal: frac * 2^-24
  } else if (expo == 31) {
    mag = frac ? std::nan("") : INFINITY;
  } else {
    mag = std::ldexp(static_cast<double>(1024 + frac), expo - 25);  // (1 + frac/1024) * 2^(e-15)
  }
  return sign ? -mag : mag;
}

double bf16_bits_to_double(uint16_t b) {
  // bfloat16 is the top half of an IEEE binary32.
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

double load_elem(const void* base, int dtype, size_t idx) {
  if (dtype == 0) {
    float f;
    std::memcpy(&f, static_cast<const char*>(base) + idx * 4, 4);
    return static_cast<double>(f);
  }
  uint16_t bits;
  std::memcpy(&bits, static_cast<const char*>(base) + idx * 2, 2);
  return dtype == 1 ? half_bits_to_double(bits) : bf16_bits_to_double(bits);
}

size_t elem_bytes(int dtype) { return dtype == 0 ? 4 : 2; }

// Runs fn(u) for u in [0, n) on up to n_threads threads (n_threads <= 0: all hardware threads).
template <class Fn>
void parallel_for(long n, int n_threads, Fn fn) {
  if (n_threads <= 0) n_threads = static_cast<int>(std::thread::hardware_concurrency());
  if (n_threads < 1) n_threads = 1;
  if (n_threads == 1 || n <= 1) {
    for (long u = 0; u < n; ++u) fn(u);
    return;
  }
  std::atomic<long> next{0};
  std::vector<std::thread> pool;
  for (int t = 0; t < n_threads; ++t)
    pool.emplace_back([&] {
      for (long u = next.fetch_add(1); u < n; u = next.fetch_add(1)) fn(u);
    });
  for (auto& th : pool) th.join();
}

// Physical row of token t of sequence s for kv head kh in a cache laid out as
// [n_blocks][Hk][B][d]: the block table gives the physical block of logical block t / B
// [P2-TABLE], and the token sits at offset t % B inside it [P2-BLK, K_j].
bool token_row(const int32_t* bt, int max_blocks, int n_blocks, int s, int t, int Hk, int kh, int B,
               size_t* row) {
  const int j = t / B;
  if (j >= max_blocks) return false;
  const int32_t phys = bt[static_cast<size_t>(s) * max_blocks + j];
  if (phys < 0 || phys >= n_blocks) return false;
  *row = (static_cast<size_t>(phys) * Hk + kh) * B + (t % B);
  return true;
}

}  // namespace

extern "C" {

int oracle_hardware_threads() { return static_cast<int>(std::thread::hardware_concurrency()); }

double oracle_elem_to_double(const void* base, int dtype, long idx) { return load_elem(base, dtype, idx); }

// [P2-KV] Plain definition: for each sequence s and query head h, gather the c = context_lens[s]
// cached keys and values into contiguous [c][d] arrays, then o = softmax(scale * q K^T) V with the
// textbook softmax (the maximum is subtracted first, which leaves the value unchanged).
// out: [S][H][d] doubles.  Returns 0, or -1 if a needed block-table entry is out of range.
int oracle_decode(double* out, const void* q, int q_dtype, const void* k_cache, const void* v_cache,
                  int kv_dtype, const int32_t* block_tables, const int32_t* context_lens, int S, int H,
                  int Hk, int d, int B, int n_blocks, int max_blocks_per_seq, double scale,
                  int n_threads) {
  if (S < 0 || H <= 0 || Hk <= 0 || H % Hk != 0 || d <= 0 || B <= 0) return -2;
  const int g = H / Hk;
  std::atomic<int> bad{0};
  parallel_for(static_cast<long>(S) * H, n_threads, [&](long u) {
    const int s = static_cast<int>(u / H), h = static_cast<int>(u % H);
    const int kh = h / g;
    double* o = out + (static_cast<size_t>(s) * H + h) * d;
    const int c = context_lens[s];
    for (int i = 0; i < d; ++i) o[i] = 0.0;
    if (c <= 0) return;
    // gather K_s, V_s (contiguous copies, as in a non-paged cache)
    std::vector<double> K(static_cast<size_t>(c) * d), V(static_cast<size_t>(c) * d), qv(d);
    for (int i = 0; i < d; ++i) qv[i] = load_elem(q, q_dtype, (static_cast<size_t>(s) * H + h) * d + i);
    for (int t = 0; t < c; ++t) {
      size_t row;
      if (!token_row(block_tables, max_blocks_per_seq, n_blocks, s, t, Hk, kh, B, &row)) {
        bad = 1;
        return;
      }
      for (int i = 0; i < d; ++i) {
        K[static_cast<size_t>(t) * d + i] = load_elem(k_cache, kv_dtype, row * d + i);
        V[static_cast<size_t>(t) * d + i] = load_elem(v_cache, kv_dtype, row * d + i);
      }
    }
    // scores x_t = scale * <q, k_t>
    std::vector<double> x(c);
    double mx = -INFINITY;
    for (int t = 0; t < c; ++t) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += qv[i] * K[static_cast<size_t>(t) * d + i];
      x[t] = scale * acc;
      if (x[t] > mx) mx = x[t];
    }
    // softmax weights and the weighted sum of values
    double z = 0.0;
    for (int t = 0; t < c; ++t) {
      x[t] = std::exp(x[t] - mx);
      z += x[t];
    }
    for (int t = 0; t < c; ++t)
      for (int i = 0; i < d; ++i) o[i] += x[t] * V[static_cast<size_t>(t) * d + i];
    for (int i = 0; i < d; ++i) o[i] /= z;
  });
  return bad ? -1 : 0;
}

// [P2-BLK] The block-wise rewrite, taken literally: with K_j, V_j the j-th block of B tokens,
//   A_ij = exp(q^T K_j * scale) / sum_{t=1..ceil(c/B)} sum_{tokens of block t} exp(q^T k * scale)
//   o    = sum_j V_j A_ij^T
// The denominator sums exp over every token of every block (the pages' K_t is a block, so the
// term is a B-vector and the plain reading sums its entries).  No maximum is subtracted, exactly
// as printed.  The last block holds only c - (nb-1)*B tokens.  This is the formulation the
// method computes; the test suite checks it against oracle_decode.
int oracle_decode_blockwise(double* out, const void* q, int q_dtype, const void* k_cache,
                            const void* v_cache, int kv_dtype, const int32_t* block_tables,
                            const int32_t* context_lens, int S, int H, int Hk, int d, int B,
                            int n_blocks, int max_blocks_per_seq, double scale) {
  if (S < 0 || H <= 0 || Hk <= 0 || H % Hk != 0 || d <= 0 || B <= 0) return -2;
  const int g = H / Hk;
  for (int s = 0; s < S; ++s) {
    const int c = context_lens[s];
    const int nb = (c + B - 1) / B;
    for (int h = 0; h < H; ++h) {
      const int kh = h / g;
      double* o = out + (static_cast<size_t>(s) * H + h) * d;
      for (int i = 0; i < d; ++i) o[i] = 0.0;
      if (c <= 0) continue;
      if (nb > max_blocks_per_seq) return -1;
      std::vector<double> qv(d);
      for (int i = 0; i < d; ++i) qv[i] = load_elem(q, q_dtype, (static_cast<size_t>(s) * H + h) * d + i);
      // exp(q^T K_j scale) for every block j, one entry per token of the block
      std::vector<std::vector<double>> e(nb);
      double denom = 0.0;
      for (int j = 0; j < nb; ++j) {
        const int32_t phys = block_tables[static_cast<size_t>(s) * max_blocks_per_seq + j];
        if (phys < 0 || phys >= n_blocks) return -1;
        const int filled = (j == nb - 1) ? c - j * B : B;
        e[j].resize(filled);
        for (int r = 0; r < filled; ++r) {
          const size_t row = (static_cast<size_t>(phys) * Hk + kh) * B + r;
          double dot = 0.0;
          for (int i = 0; i < d; ++i) dot += qv[i] * load_elem(k_cache, kv_dtype, row * d + i);
          e[j][r] = std::exp(dot * scale);
          denom += e[j][r];
        }
      }
      // o = sum_j V_j A_ij^T, with A_ij = e_j / denom
      for (int j = 0; j < nb; ++j) {
        const int32_t phys = block_tables[static_cast<size_t>(s) * max_blocks_per_seq + j];
        for (int r = 0; r < static_cast<int>(e[j].size()); ++r) {
          const size_t row = (static_cast<size_t>(phys) * Hk + kh) * B + r;
          const double a = e[j][r] / denom;
          for (int i = 0; i < d; ++i) o[i] += a * load_elem(v_cache, kv_dtype, row * d + i);
        }
      }
    }
  }
  return 0;
}

// Partial state over the token range [t0, t1) of one (sequence, query head): the unnormalised
// weighted sum o~ = sum_t exp(x_t - m) v_t, the maximum score m and l = sum_t exp(x_t - m).
// This is the denominator of [P2-BLK] restricted to a subset of blocks; merging the subsets
// (oracle_combine) gives the whole sum back.  Empty ranges give m = -inf, l = 0, o~ = 0.
// part_o: [S][H][n_parts][d], part_m/part_l: [S][H][n_parts] doubles; part p covers
// [p*P, min((p+1)*P, c)).
int oracle_partials(double* part_o, double* part_m, double* part_l, int n_parts, int P,
                    const void* q, int q_dtype, const void* k_cache, const void* v_cache, int kv_dtype,
                    const int32_t* block_tables, const int32_t* context_lens, int S, int H, int Hk,
                    int d, int B, int n_blocks, int max_blocks_per_seq, double scale) {
  if (S < 0 || H <= 0 || Hk <= 0 || H % Hk != 0 || d <= 0 || B <= 0 || P <= 0) return -2;
  const int g = H / Hk;
  for (int s = 0; s < S; ++s)
    for (int h = 0; h < H; ++h) {
      const int kh = h / g, c = context_lens[s];
      std::vector<double> qv(d);
      for (int i = 0; i < d; ++i) qv[i] = load_elem(q, q_dtype, (static_cast<size_t>(s) * H + h) * d + i);
      for (int p = 0; p < n_parts; ++p) {
        const size_t pi = (static_cast<size_t>(s) * H + h) * n_parts + p;
        double* o = part_o + pi * d;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        part_m[pi] = -INFINITY;
        part_l[pi] = 0.0;
        const int t0 = p * P, t1 = (p + 1) * P < c ? (p + 1) * P : c;
        if (t0 >= t1) continue;
        std::vector<double> x(t1 - t0);
        std::vector<size_t> rows(t1 - t0);
        double mx = -INFINITY;
        for (int t = t0; t < t1; ++t) {
          if (!token_row(block_tables, max_blocks_per_seq, n_blocks, s, t, Hk, kh, B, &rows[t - t0]))
            return -1;
          double dot = 0.0;
          for (int i = 0; i < d; ++i) dot += qv[i] * load_elem(k_cache, kv_dtype, rows[t - t0] * d + i);
          x[t - t0] = scale * dot;
          if (x[t - t0] > mx) mx = x[t - t0];
        }
        double l = 0.0;
        for (int t = t0; t < t1; ++t) {
          const double w = std::exp(x[t - t0] - mx);
          l += w;
          for (int i = 0; i < d; ++i) o[i] += w * load_elem(v_cache, kv_dtype, rows[t - t0] * d + i);
        }
        part_m[pi] = mx;
        part_l[pi] = l;
      }
    }
  return 0;
}

// Merges partial states: with M = max_p m_p and w_p = exp(m_p - M),
//   o = sum_p w_p o~_p / sum_p w_p l_p.
// Parts with m_p = -inf (empty) carry no weight; if every part is empty the output is zero.
// Inputs may be fp32 (in_f32 != 0; part arrays are float) or double.  out: [S][H][d] doubles.
void oracle_combine(double* out, const void* part_o, const void* part_m, const void* part_l,
                    int in_f32, int S, int H, int n_parts, int d) {
  auto rd = [&](const void* base, size_t idx) {
    return in_f32 ? static_cast<double>(static_cast<const float*>(base)[idx])
                  : static_cast<const double*>(base)[idx];
  };
  for (int s = 0; s < S; ++s)
    for (int h = 0; h < H; ++h) {
      const size_t base = (static_cast<size_t>(s) * H + h) * n_parts;
      double* o = out + (static_cast<size_t>(s) * H + h) * d;
      double M = -INFINITY;
      for (int p = 0; p < n_parts; ++p) M = rd(part_m, base + p) > M ? rd(part_m, base + p) : M;
      for (int i = 0; i < d; ++i) o[i] = 0.0;
      if (M == -INFINITY) continue;
      double den = 0.0;
      for (int p = 0; p < n_parts; ++p) {
        const double mp = rd(part_m, base + p);
        if (mp == -INFINITY) continue;
        const double w = std::exp(mp - M);
        den += w * rd(part_l, base + p);
        for (int i = 0; i < d; ++i) o[i] += w * rd(part_o, (base + p) * d + i);
      }
      for (int i = 0; i < d; ++i) o[i] /= den;
    }
}

// [P4-DEC] Slot-mapped write of new tokens: token n's key and value for kv head kh go to
// physical block slot / B at offset slot % B.  Elements are copied bit for bit.
// key/value: [T][Hk][d]; caches [n_blocks][Hk][B][d].  Returns -1 on an out-of-range slot.
int oracle_cache_write(void* k_cache, void* v_cache, const void* key, const void* value,
                       const int64_t* slot_mapping, int T, int Hk, int d, int B, int n_blocks,
                       int dtype) {
  const size_t e = elem_bytes(dtype);
  for (int n = 0; n < T; ++n) {
    const int64_t slot = slot_mapping[n];
    if (slot < 0) continue;  // padding token
    const int64_t blk = slot / B, off = slot % B;
    if (blk >= n_blocks) return -1;
    for (int kh = 0; kh < Hk; ++kh)
      for (int i = 0; i < d; ++i) {
        const size_t src = (static_cast<size_t>(n) * Hk + kh) * d + i;
        const size_t dst = ((static_cast<size_t>(blk) * Hk + kh) * B + off) * d + i;
        std::memcpy(static_cast<char*>(k_cache) + dst * e, static_cast<const char*>(key) + src * e, e);
        std::memcpy(static_cast<char*>(v_cache) + dst * e, static_cast<const char*>(value) + src * e, e);
      }
  }
  return 0;
}

// [P2-COW] step 2, "copy the shared block's contents to the new block": for each (src, dst)
// pair, the whole physical block (all kv heads, all B slots) of the key cache and of the value
// cache is copied.  pairs: [P][2].  Returns -1 on an out-of-range id.
int oracle_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs, int P, int Hk, int d, int B,
                       int n_blocks, int dtype) {
  const size_t bytes = static_cast<size_t>(Hk) * B * d * elem_bytes(dtype);
  for (int p = 0; p < P; ++p) {
    const int32_t src = pairs[2 * p], dst = pairs[2 * p + 1];
    if (src < 0 || src >= n_blocks || dst < 0 || dst >= n_blocks) return -1;
    std::memcpy(static_cast<char*>(k_cache) + dst * bytes, static_cast<const char*>(k_cache) + src * bytes, bytes);
    std::memcpy(static_cast<char*>(v_cache) + dst * bytes, static_cast<const char*>(v_cache) + src * bytes, bytes);
  }
  return 0;
}

// Chunked prefill and mixed batches ("Paged Attention&Orca Paper笔记与解读", selective batching:
// prefill and decode tokens of different requests are batched, and only attention needs to know
// each token's request and phase; "vllm" 2.1 Prefill: the prompt's tokens are processed together).
// Sequence s has n_s = q_start[s+1] - q_start[s] query tokens, the last n_s of its c_s context
// tokens (already in the cache); the token at position p = c_s - n_s + i attends to positions
// 0..p (causal), i.e. o = softmax(scale * q K[0..p]^T) V[0..p] -- the decode definition applied
// to each query token with the context cut at its own position.  Decode is n_s = 1.
// query: [T][H][d]; out: [T][H][d] doubles.  Returns -1 on a bad table entry or n_s > c_s.
int oracle_prefill(double* out, const void* q, int q_dtype, const int32_t* q_start, const void* k_cache,
                   const void* v_cache, int kv_dtype, const int32_t* block_tables, const int32_t* context_lens,
                   int S, int H, int Hk, int d, int B, int n_blocks, int max_blocks_per_seq, double scale,
                   int n_threads) {
  if (S < 0 || H <= 0 || Hk <= 0 || H % Hk != 0 || d <= 0 || B <= 0) return -2;
  const int g = H / Hk;
  const int T = S > 0 ? q_start[S] : 0;
  std::atomic<int> bad{0};
  parallel_for(static_cast<long>(T) * H, n_threads, [&](long u) {
    const int row = static_cast<int>(u / H), h = static_cast<int>(u % H), kh = h / g;
    int s = 0;
    while (s + 1 <= S && q_start[s + 1] <= row) ++s;  // the sequence this query token belongs to
    const int n = q_start[s + 1] - q_start[s], c = context_lens[s];
    double* o = out + (static_cast<size_t>(row) * H + h) * d;
    for (int i = 0; i < d; ++i) o[i] = 0.0;
    if (n > c) {
      bad = 1;
      return;
    }
    const int pos = c - n + (row - q_start[s]);  // this token's position; it sees 0..pos
    std::vector<double> qv(d), x(pos + 1);
    for (int i = 0; i < d; ++i) qv[i] = load_elem(q, q_dtype, (static_cast<size_t>(row) * H + h) * d + i);
    double mx = -INFINITY;
    std::vector<size_t> rows(pos + 1);
    for (int t = 0; t <= pos; ++t) {
      if (!token_row(block_tables, max_blocks_per_seq, n_blocks, s, t, Hk, kh, B, &rows[t])) {
        bad = 1;
        return;
      }
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += qv[i] * load_elem(k_cache, kv_dtype, rows[t] * d + i);
      x[t] = scale * acc;
      if (x[t] > mx) mx = x[t];
    }
    double z = 0.0;
    for (int t = 0; t <= pos; ++t) {
      x[t] = std::exp(x[t] - mx);
      z += x[t];
    }
    for (int t = 0; t <= pos; ++t)
      for (int i = 0; i < d; ++i) o[i] += x[t] * load_elem(v_cache, kv_dtype, rows[t] * d + i);
    for (int i = 0; i < d; ++i) o[i] /= z;
  });
  return bad ? -1 : 0;
}

// Preemption by swapping ("PagedAttention原理", "抢占与恢复", swap: a preempted sequence's blocks move
// to CPU memory and come back before it runs again): for each (src, dst) pair, block dst of the
// destination pool becomes a copy of block src of the source pool, for K and V.  The two pools
// have the same [n][Hk][B][d] layout and may differ in size.  Returns -1 on an out-of-range id.
int oracle_swap_blocks(void* dst_k, void* dst_v, int n_dst, const void* src_k, const void* src_v, int n_src,
                       const int32_t* pairs, int P, int Hk, int d, int B, int dtype) {
  const size_t bytes = static_cast<size_t>(Hk) * B * d * elem_bytes(dtype);
  for (int p = 0; p < P; ++p) {
    const int32_t src = pairs[2 * p], dst = pairs[2 * p + 1];
    if (src < 0 || src >= n_src || dst < 0 || dst >= n_dst) return -1;
    std::memcpy(static_cast<char*>(dst_k) + dst * bytes, static_cast<const char*>(src_k) + src * bytes, bytes);
    std::memcpy(static_cast<char*>(dst_v) + dst * bytes, static_cast<const char*>(src_v) + src * bytes, bytes);
  }
  return 0;
}

}  // extern "C"

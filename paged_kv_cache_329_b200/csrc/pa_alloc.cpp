// Host block manager of libpa: reference-counted physical blocks, sequences with block tables,
// slot reservation with copy-on-write, and block-table packing.
//
// Rules (page "PagedAttention原理"): blocks of B tokens are taken one at a time as a sequence grows
// ("从虚拟内存的启发"); the block table maps each logical block to a physical block and knows how
// full it is ("实现一个虚拟内存"); each physical block has a reference count and is released at 0
// ("解决共享prompt"); a write into a shared block goes through the five copy-on-write steps
// ("解决COW"), while a block with room and a single owner is appended to in place ("COW 区别").
// Forked sequences share all blocks, as in parallel sampling and beam search (page "Paged
// Attention&Orca Paper笔记与解读").
#include <new>
#include <unordered_map>
#include <vector>

#include "pa_internal.h"

struct pa_alloc {
  struct Seq {
    std::vector<int32_t> table;  // logical block j -> physical block
    int64_t n_tokens = 0;        // filled slots; the last block holds n_tokens - (nb-1)*B
  };
  int n_blocks = 0;
  int B = 0;
  std::vector<int32_t> ref;   // reference count per physical block (0 = free)
  std::vector<int32_t> free;  // LIFO stack of free ids; back() is handed out next
  using SeqMap = std::unordered_map<int32_t, Seq>;
  SeqMap seqs;
  std::vector<SeqMap::node_type> spare;  // freed sequences' map nodes (with their table storage)
  int32_t next_seq = 0;
};

namespace {

bool allocated(const pa_alloc* a, int32_t b) { return b >= 0 && b < a->n_blocks && a->ref[b] > 0; }

int32_t take_block(pa_alloc* a) {  // caller checked that the stack is not empty
  const int32_t b = a->free.back();
  a->free.pop_back();
  a->ref[b] = 1;
  return b;
}

void release(pa_alloc* a, int32_t b) {  // caller checked allocated(a, b)
  if (--a->ref[b] == 0) a->free.push_back(b);
}

// Inserts a new sequence `id` with an empty table and returns it.  The map node and the table
// storage of a freed sequence are reused when there is one: a serving loop forks and frees a batch
// of sequences every step, and once as many sequences have been freed as are created per step, a
// step allocates neither nodes nor tables (the map's bucket array grows only when the number of
// live sequences exceeds every earlier count).
pa_alloc::Seq& insert_seq(pa_alloc* a, int32_t id) {
  if (a->spare.empty()) return a->seqs.emplace(id, pa_alloc::Seq{}).first->second;
  pa_alloc::SeqMap::node_type node = std::move(a->spare.back());
  a->spare.pop_back();
  node.key() = id;
  node.mapped().table.clear();
  node.mapped().n_tokens = 0;
  return a->seqs.insert(std::move(node)).position->second;
}

}  // namespace

extern "C" {

pa_alloc* pa_alloc_create(int n_blocks, int B) {
  if (n_blocks <= 0 || B <= 0) {
    pa::fail(PA_ERR_INVALID_ARG, "pa_alloc_create: n_blocks (%d) and B (%d) must be positive", n_blocks, B);
    return nullptr;
  }
  pa_alloc* a = new (std::nothrow) pa_alloc;
  if (!a) {
    pa::fail(PA_ERR_INVALID_ARG, "pa_alloc_create: out of host memory");
    return nullptr;
  }
  a->n_blocks = n_blocks;
  a->B = B;
  a->ref.assign(n_blocks, 0);
  a->seqs.reserve(1024);
  a->free.resize(n_blocks);
  for (int i = 0; i < n_blocks; ++i) a->free[i] = n_blocks - 1 - i;  // back() == 0
  pa::ok();
  return a;
}

void pa_alloc_destroy(pa_alloc* a) { delete a; }

pa_status pa_alloc_block(pa_alloc* a, int32_t* block_id) {
  if (!a || !block_id) return pa::fail(PA_ERR_INVALID_ARG, "pa_alloc_block: null argument");
  if (a->free.empty()) return pa::fail(PA_ERR_NO_FREE_BLOCK, "pa_alloc_block: pool of %d blocks exhausted", a->n_blocks);
  *block_id = take_block(a);
  return pa::ok();
}

pa_status pa_block_incref(pa_alloc* a, int32_t b) {
  if (!a || !allocated(a, b)) return pa::fail(PA_ERR_INVALID_ARG, "pa_block_incref: block %d is not allocated", b);
  ++a->ref[b];
  return pa::ok();
}

pa_status pa_block_decref(pa_alloc* a, int32_t b) {
  if (!a || !allocated(a, b)) return pa::fail(PA_ERR_INVALID_ARG, "pa_block_decref: block %d is not allocated", b);
  release(a, b);
  return pa::ok();
}

int pa_block_refcount(const pa_alloc* a, int32_t b) {
  if (!a || b < 0 || b >= a->n_blocks) return -1;
  return a->ref[b];
}

int pa_alloc_num_free(const pa_alloc* a) { return a ? static_cast<int>(a->free.size()) : -1; }

pa_status pa_seq_create(pa_alloc* a, int32_t* seq_id) {
  if (!a || !seq_id) return pa::fail(PA_ERR_INVALID_ARG, "pa_seq_create: null argument");
  const int32_t id = a->next_seq++;
  insert_seq(a, id);
  *seq_id = id;
  return pa::ok();
}

pa_status pa_seq_fork(pa_alloc* a, int32_t parent, int32_t* child) {
  if (!a || !child) return pa::fail(PA_ERR_INVALID_ARG, "pa_seq_fork: null argument");
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end()) return pa::fail(PA_ERR_INVALID_ARG, "pa_seq_fork: unknown sequence %d", parent);
  const int32_t id = a->next_seq++;
  // the parent's entry stays valid: unordered_map references survive insertion (rehash included)
  const pa_alloc::Seq& parent_seq = it->second;
  pa_alloc::Seq& s = insert_seq(a, id);
  s.table.assign(parent_seq.table.begin(), parent_seq.table.end());
  s.n_tokens = parent_seq.n_tokens;
  for (int32_t b : s.table) ++a->ref[b];
  *child = id;
  return pa::ok();
}

pa_status pa_seq_free(pa_alloc* a, int32_t seq_id) {
  if (!a) return pa::fail(PA_ERR_INVALID_ARG, "pa_seq_free: null handle");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return pa::fail(PA_ERR_INVALID_ARG, "pa_seq_free: unknown sequence %d", seq_id);
  for (int32_t b : it->second.table) release(a, b);
  if (a->spare.size() < 4096) a->spare.push_back(a->seqs.extract(it));
  else a->seqs.erase(it);
  return pa::ok();
}

pa_status pa_seq_fork_batch(pa_alloc* a, const int32_t* parents, int n, int32_t* children) {
  if (!a || n < 0 || (n > 0 && (!parents || !children)))
    return pa::fail(PA_ERR_INVALID_ARG, "pa_seq_fork_batch: bad arguments");
  for (int i = 0; i < n; ++i) {
    const pa_status st = pa_seq_fork(a, parents[i], children + i);
    if (st != PA_OK) return st;
  }
  return pa::ok();
}

pa_status pa_seq_free_batch(pa_alloc* a, const int32_t* seq_ids, int n) {
  if (!a || n < 0 || (n > 0 && !seq_ids)) return pa::fail(PA_ERR_INVALID_ARG, "pa_seq_free_batch: bad arguments");
  for (int i = 0; i < n; ++i) {
    const pa_status st = pa_seq_free(a, seq_ids[i]);
    if (st != PA_OK) return st;
  }
  return pa::ok();
}

int pa_seq_len(const pa_alloc* a, int32_t seq_id) {
  if (!a) return -1;
  auto it = a->seqs.find(seq_id);
  return it == a->seqs.end() ? -1 : static_cast<int>(it->second.n_tokens);
}

int pa_seq_num_blocks(const pa_alloc* a, int32_t seq_id) {
  if (!a) return -1;
  auto it = a->seqs.find(seq_id);
  return it == a->seqs.end() ? -1 : static_cast<int>(it->second.table.size());
}

pa_status pa_seq_reserve_slots(pa_alloc* a, int32_t seq_id, int n_new, int64_t* slots,
                               int32_t* cow_pairs, int* n_cow) {
  if (!a || n_new < 0 || (n_new > 0 && !slots) || !n_cow)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_seq_reserve_slots: bad arguments");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return pa::fail(PA_ERR_INVALID_ARG, "pa_seq_reserve_slots: unknown sequence %d", seq_id);
  pa_alloc::Seq& s = it->second;
  const int64_t B = a->B;
  int64_t n = s.n_tokens;
  // Count every block the reservation needs before touching any state, so a failure is atomic.
  const bool cow = n_new > 0 && n % B != 0 && a->ref[s.table.back()] > 1;
  const int64_t fresh = (n + n_new + B - 1) / B - static_cast<int64_t>(s.table.size());
  if ((cow ? 1 : 0) + fresh > static_cast<int64_t>(a->free.size()))
    return pa::fail(PA_ERR_NO_FREE_BLOCK, "pa_seq_reserve_slots: needs %lld blocks, %zu free",
                    static_cast<long long>((cow ? 1 : 0) + fresh), a->free.size());
  if (cow && !cow_pairs) return pa::fail(PA_ERR_INVALID_ARG, "pa_seq_reserve_slots: cow_pairs is null");
  *n_cow = 0;
  for (int i = 0; i < n_new; ++i, ++n) {
    if (n % B == 0) {
      s.table.push_back(take_block(a));  // last block full or none: fresh block, nothing copied
    } else if (a->ref[s.table.back()] > 1) {
      const int32_t old_b = s.table.back();
      const int32_t new_b = take_block(a);   // (1) allocate a new physical block
      cow_pairs[2 * *n_cow] = old_b;         // (2) the caller copies old -> new
      cow_pairs[2 * *n_cow + 1] = new_b;
      ++*n_cow;
      s.table.back() = new_b;                // (3) remap the logical block
      release(a, old_b);                     // (4) decrement the old block's count
    }
    slots[i] = static_cast<int64_t>(s.table[n / B]) * B + n % B;  // (5) write lands in the new block
  }
  s.n_tokens = n;
  return pa::ok();
}

pa_status pa_seq_reserve_slots_batch(pa_alloc* a, const int32_t* seq_ids, int S, int n_new, int64_t* slots,
                                     int32_t* cow_pairs, int* n_cow, int* n_done) {
  if (!a || S < 0 || n_new < 0 || (S > 0 && (!seq_ids || (n_new > 0 && !slots))) || !n_cow || !n_done)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_seq_reserve_slots_batch: bad arguments");
  *n_cow = 0;
  *n_done = 0;
  for (int i = 0; i < S; ++i) {
    int c = 0;
    const pa_status st = pa_seq_reserve_slots(a, seq_ids[i], n_new, slots + static_cast<size_t>(i) * n_new,
                                              cow_pairs ? cow_pairs + 2 * *n_cow : nullptr, &c);
    if (st != PA_OK) return st;
    *n_cow += c;
    *n_done = i + 1;
  }
  return pa::ok();
}

pa_status pa_build_block_tables(const pa_alloc* a, const int32_t* seq_ids, int S, int32_t* tables,
                                int max_blocks_per_seq, int32_t* context_lens) {
  if (!a || S < 0 || (S > 0 && (!seq_ids || !tables || !context_lens)) || max_blocks_per_seq < 0)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_build_block_tables: bad arguments");
  for (int i = 0; i < S; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end())
      return pa::fail(PA_ERR_INVALID_ARG, "pa_build_block_tables: unknown sequence %d", seq_ids[i]);
    if (static_cast<int>(it->second.table.size()) > max_blocks_per_seq)
      return pa::fail(PA_ERR_INVALID_ARG, "pa_build_block_tables: sequence %d has %zu blocks > %d",
                      seq_ids[i], it->second.table.size(), max_blocks_per_seq);
    if (it->second.n_tokens > INT32_MAX)
      return pa::fail(PA_ERR_INVALID_ARG, "pa_build_block_tables: sequence %d too long", seq_ids[i]);
  }
  for (int i = 0; i < S; ++i) {
    const pa_alloc::Seq& s = a->seqs.find(seq_ids[i])->second;
    int32_t* row = tables + static_cast<size_t>(i) * max_blocks_per_seq;
    const int nb = static_cast<int>(s.table.size());
    for (int j = 0; j < max_blocks_per_seq; ++j) row[j] = j < nb ? s.table[j] : -1;
    context_lens[i] = static_cast<int32_t>(s.n_tokens);
  }
  return pa::ok();
}

}  // extern "C"

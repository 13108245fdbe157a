/*
 * pa.h -- C ABI of libpa: paged decode attention on NVIDIA B200 (sm_100a).
 *
 * The library computes the decode step of attention over a KV cache that is stored in fixed-size
 * physical blocks, and carries the two data-parallel paths that keep such a cache up to date
 * (the slot-mapped write of new tokens and the copy-on-write block copy), plus a host-side block
 * manager with reference counts that produces the block tables, slot mappings and copy pairs.
 *
 * Sources (page title, section, equation or list):
 *   "PagedAttention原理" (scmmm.top), "为什么会有 KV cache": o_t = softmax(q_t K^T / sqrt(d)) V
 *   "PagedAttention原理", "实现一个虚拟内存": K_j = (k_{(j-1)B+1} .. k_{jB}), V_j likewise,
 *       A_ij = exp(q_i^T K_j / sqrt(d)) / sum_t exp(q_i^T K_t / sqrt(d)),  o_i = sum_j V_j A_ij^T;
 *       the block table records, per logical block, its physical block and its fill count.
 *   "PagedAttention原理", "从虚拟内存的启发": blocks of B tokens requested one at a time.
 *   "PagedAttention原理", "解决共享prompt" and "解决COW": per-block reference counts and the five
 *       copy-on-write steps; "COW 区别": a block with free slots is appended to without copying.
 *   "vllm" (cnblogs), section 2.2 Decode: each decode step appends the new token's K and V.
 *
 * Conventions for every entry point below.
 *   - Tensors are dense, row-major, contiguous.  "device" pointers point to memory the caller
 *     allocated on the current CUDA device; "host" pointers to host memory.  The library never
 *     takes ownership of a caller's buffer and allocates no device buffers (scratch is a
 *     caller-provided workspace; pa_step_create creates CUDA streams, events and graphs only).
 *   - Device pointers must be 16-byte aligned.
 *   - Device work is enqueued on `stream` (a cudaStream_t; NULL is the legacy default stream) and
 *     runs asynchronously: a return of PA_OK means the arguments were valid and the kernels were
 *     launched.  Faults inside a kernel surface at the caller's next synchronisation.
 *   - No C++ exception crosses this boundary.  On failure an entry point returns a pa_status
 *     other than PA_OK and pa_last_error() returns a message (per host thread).
 *   - Shapes: S sequences, H query heads, Hk kv heads (H % Hk == 0; query head h reads kv head
 *     h / (H / Hk)), head dimension d, block size B (tokens per block), n_blocks physical blocks.
 *   - Supported: d in {64, 128}; B in {8, 16, 32}; H / Hk in {1, 2, 4, 8}; element types
 *     PA_F32, PA_F16, PA_BF16 (query and caches share one type).
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,   /* bad shape, type, pointer, alignment or size */
  PA_ERR_NO_FREE_BLOCK = 2, /* block pool exhausted; the call changed nothing */
  PA_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed */
  PA_ERR_UNSUPPORTED = 4    /* valid request outside the supported set above */
} pa_status;

typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2 } pa_dtype;

/* Message for the last failure on the calling host thread ("" if none).  The string is owned by
 * the library and stays valid until the thread's next call into it. */
const char* pa_last_error(void);

/* Library version string, static storage. */
const char* pa_version(void);

/* ---------------------------------------------------------------------------------------------
 * Paged decode attention.
 *
 * For every sequence s (context length c = context_lens[s], which counts the token written in
 * this step) and query head h with kv head kh = h / (H / Hk):
 *     x_t = scale * <query[s][h], k_t>          for t = 0 .. c-1,
 *     out[s][h] = sum_t softmax(x)_t * v_t,
 * where k_t = k_cache[block_tables[s][t / B]][kh][t % B] and v_t likewise ("实现一个虚拟内存",
 * eqs. A_ij, o_i; "为什么会有 KV cache", eq. o_t).  Only the c valid tokens are read: slots past
 * c in the last block and table entries past ceil(c / B) are never used.  c = 0 gives zeros.
 * Scores, the softmax and the weighted sum are computed in fp32.
 *
 * The context is cut into partitions of `partition_size` tokens (a multiple of 64; 0 = chosen by
 * the library from S, Hk and max_context_len).  Each (sequence, kv head, partition) is one unit of
 * work; partitions of one sequence are merged by the log-sum-exp combine (pa_combine's rule).
 * For a fixed partition size the result is a deterministic function of the logical contents:
 * repeating a call, or moving blocks to other physical ids and updating the table, gives
 * bit-identical output.
 *
 *   out            device, [S][H][d] of out_dtype (any of the three types)
 *   query          device, [S][H][d] of kv_dtype
 *   k_cache        device, [n_blocks][Hk][B][d] of kv_dtype
 *   v_cache        device, [n_blocks][Hk][B][d] of kv_dtype
 *   block_tables   device, [S][max_blocks_per_seq] int32 physical block ids
 *   context_lens   device, [S] int32, each in [0, max_context_len]
 *   max_context_len  host bound on every context_lens[s] (sizes the partition grid)
 *   scale          score scale, normally 1/sqrt(d)
 *   workspace      device scratch of at least pa_decode_workspace_size(...) bytes, 256-byte
 *                  aligned, owned by the caller; its contents need no initialisation and are
 *                  overwritten.  Calls that overlap on the GPU must not share a workspace.
 * A block-table entry outside [0, n_blocks) reads as zeros and sets the error word read by
 * pa_workspace_error().
 */
size_t pa_decode_workspace_size(int S, int H, int Hk, int d, int max_context_len, int partition_size);

pa_status pa_decode(void* out, pa_dtype out_dtype, const void* query, const void* k_cache,
                    const void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                    int S, int H, int Hk, int d, int B, int n_blocks, int max_blocks_per_seq,
                    int max_context_len, float scale, pa_dtype kv_dtype, int partition_size,
                    void* workspace, size_t workspace_bytes, void* stream);

/* One decode step on device-resident inputs: the copy-on-write block copies, then the slot-mapped
 * write of the new tokens, then paged decode attention -- the order the pages give ("解决COW":
 * copy the shared block before writing into the copy; "vllm" 2.2 Decode: the new token's K and V
 * are stored, then attended over).  The result equals
 *     pa_copy_blocks(k_cache, v_cache, pairs, n);  pa_cache_write(..., key, value, slot_mapping, T);
 *     pa_decode(out, ...);
 * in fewer launches: one kernel makes the copies, the writes and the decode's work plan (a block
 * copy and every write into the copied block are made by the same CTA, copy first), and the
 * decode kernels follow it by programmatic dependent launch and wait for all of it.
 *
 *   key, value     device [T][Hk][d] of kv_dtype: the new tokens
 *   slot_mapping   device [T] int64, slot = block * B + offset (< 0: padding, skipped)
 *   pairs          device [max_pairs][2] int32 (src, dst), destinations distinct and no
 *                  destination also a source (as the block manager emits them)
 *   n_pairs        device pointer to the number of pairs used (clamped to [0, max_pairs]), read by
 *                  the kernel -- so one capture serves steps with different counts -- or NULL to
 *                  use all max_pairs; max_pairs <= 8192
 *   everything else: as pa_decode (workspace of pa_decode_workspace_size(...) bytes).
 * Out-of-range block ids in pairs or slots are skipped as in pa_copy_blocks / pa_cache_write. */
pa_status pa_decode_step(void* out, pa_dtype out_dtype, const void* query, void* k_cache, void* v_cache,
                         const int32_t* block_tables, const int32_t* context_lens, const void* key,
                         const void* value, const int64_t* slot_mapping, int T, const int32_t* pairs,
                         const int32_t* n_pairs, int max_pairs, int S, int H, int Hk, int d, int B,
                         int n_blocks, int max_blocks_per_seq, int max_context_len, float scale,
                         pa_dtype kv_dtype, int partition_size, void* workspace, size_t workspace_bytes,
                         void* stream);

/* Paged decode attention that allocates nothing and takes no workspace.  The pages have no
 * counterpart to this entry point; it exists for callers that cannot call cudaMalloc: plugins
 * whose host process owns the whole device-memory budget and forbids allocations by libraries,
 * and serving loops that must not let an allocation (which can synchronise the device or fail
 * under memory pressure) happen on the decode path.
 *
 * Arguments and results are those of pa_decode without `workspace` / `workspace_bytes`; the
 * caller still passes every input and the output.  The workspace instead lives in one file-scope
 * device array of 32 MiB (33554432 bytes) inside libpa, which every GPU that loads the library
 * holds until the process exits.  Sizes whose pa_decode_workspace_size(...) exceeds 32 MiB are
 * rejected with PA_ERR_INVALID_ARG and a message naming both sizes (a larger partition_size, or
 * pa_decode with a caller-provided workspace, serves them).
 *
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
 * that device current) and caches it for the device's current context; make that first call
 * before any stream capture.  After a device reset (a new context) the next call looks the
 * address up again, so that call too should come before any stream capture.  Every
 * call uses the same array, which keeps the last call's contents; the only fields that must
 * start from known values (the unit counter, the unit count and the error word) are reset by the
 * call's own first kernel.  Calls that overlap on the GPU (different streams, or different host
 * threads on one device) race on the array: serialise them.  The error word of the array cannot
 * be read through pa_workspace_error. */
pa_status pa_decode_noalloc(void* out, pa_dtype out_dtype, const void* query, const void* k_cache,
                            const void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                            int S, int H, int Hk, int d, int B, int n_blocks, int max_blocks_per_seq,
                            int max_context_len, float scale, pa_dtype kv_dtype, int partition_size,
                            void* stream);

/* Partition size (tokens) that pa_decode uses for these arguments when given 0: the largest of
 * 8192, 4096, ..., 256 with at least six units per SM of the current device when every sequence
 * is max_context_len long, and no larger than the power of two that holds max_context_len
 * (else 128). */
int pa_decode_default_partition(int S, int Hk, int max_context_len);

/* Copies the error word of a decode workspace to *flags (host) after synchronising `stream`.
 * 0 = no error; bit 0 = a block-table entry was out of range (read as zeros); bit 1 = a pipeline
 * wait timed out (the kernel gave up); bit 2 = a context length exceeded max_context_len (cut to it). */
pa_status pa_workspace_error(const void* workspace, int* flags, void* stream);

/* Self-test of the kernels' bounded waits: launches one CTA that waits, with the same wait the
 * decode pipeline uses, on a barrier phase that nothing completes.  After limit_us microseconds
 * (0 < limit_us <= 1e7) the wait gives up and the kernel writes the timeout bit (2) to *status
 * (device int) instead of hanging; the context stays usable.  Used by the tests. */
pa_status pa_selftest_wait_timeout(unsigned int limit_us, int* status, void* stream);

/* ---------------------------------------------------------------------------------------------
 * Log-sum-exp merge of per-partition partial states ("实现一个虚拟内存", eq. A_ij: its denominator
 * is a sum over blocks, so it can be accumulated over any partition of the blocks and merged).
 *
 * Partition p of sequence s covers tokens [p*P, min((p+1)*P, c)), with P = partition_size and
 * n_parts(s) = ceil(c / P) (c = context_lens[s]).  For each (s, h) and p < n_parts(s):
 *   part_m[s][h][p]  = max score m_p over the partition (natural-log units, scores scale*q.k)
 *   part_l[s][h][p]  = sum over the partition of exp(x_t - m_p)
 *   part_o[s][h][p]  = sum over the partition of exp(x_t - m_p) * v_t        (d floats)
 * and the output is  out[s][h] = sum_p w_p part_o_p / sum_p w_p part_l_p,  w_p = exp(m_p - max m).
 * Entries with p >= n_parts(s) are not read.  c = 0 gives zeros.
 *
 *   out      device [S][H][d] of out_dtype
 *   part_o   device [S][H][max_parts][d] float32
 *   part_m   device [S][H][max_parts] float32
 *   part_l   device [S][H][max_parts] float32
 *   context_lens  device [S] int32, ceil(c / P) <= max_parts
 */
pa_status pa_combine(void* out, pa_dtype out_dtype, const float* part_o, const float* part_m,
                     const float* part_l, const int32_t* context_lens, int S, int H, int d,
                     int max_parts, int partition_size, void* stream);

/* ---------------------------------------------------------------------------------------------
 * Slot-mapped cache write ("vllm" 2.2 Decode: after each step the new token's K,V go into the
 * cache; "实现一个虚拟内存": a token's place is its block and its offset in the block).
 * For every token n with slot = slot_mapping[n] >= 0 and every kv head kh:
 *     k_cache[slot / B][kh][slot % B][:] = key[n][kh][:],   v_cache likewise from value.
 * slot < 0 marks a padding token and writes nothing.  Copies are bit-exact.  Two tokens with the
 * same slot race (the result is one of them).  slot / B must be < n_blocks: out-of-range slots are
 * skipped on the device and reported by nothing else, so validate slot mappings on the host when
 * they do not come from the block manager below.
 *
 *   k_cache, v_cache  device [n_blocks][Hk][B][d] of dtype
 *   key, value        device [T][Hk][d] of dtype
 *   slot_mapping      device [T] int64
 */
pa_status pa_cache_write(void* k_cache, void* v_cache, const void* key, const void* value,
                         const int64_t* slot_mapping, int T, int Hk, int d, int B, int n_blocks,
                         pa_dtype dtype, void* stream);

/* ---------------------------------------------------------------------------------------------
 * Copy-on-write block copy ("解决COW", step 2: copy the shared block's contents into the new
 * block).  For each pair p: block pairs[p][1] of k_cache and of v_cache becomes a bit copy of
 * block pairs[p][0] (all Hk heads, all B slots).  Destinations must be distinct and no
 * destination may also be a source in the same call (the block manager's pairs satisfy this);
 * otherwise the result is undefined.  Out-of-range ids are skipped on the device.
 *
 *   pairs   device [P][2] int32 (src, dst)
 */
pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs, int P, int Hk, int d,
                         int B, int n_blocks, pa_dtype dtype, void* stream);

/* ---------------------------------------------------------------------------------------------
 * Paged attention for several query tokens per sequence: chunked prefill, and batches that mix
 * prefill chunks with decode tokens ("vllm" 2.1 Prefill: the prompt's tokens are processed
 * together; "Paged Attention&Orca Paper笔记与解读", selective batching: tokens of requests in
 * different phases are batched and only attention separates them).
 *
 * Sequence s has n_s = q_start[s+1] - q_start[s] query tokens (rows q_start[s] .. q_start[s+1]-1 of
 * query), which are the LAST n_s of its c_s = context_lens[s] tokens and are already in the cache
 * (pa_cache_write first).  The token at position p = c_s - n_s + i attends to positions 0 .. p:
 *     out[row][h] = softmax(scale * q K[0..p]^T) V[0..p]      (kv head h / (H/Hk)),
 * the decode definition with the context cut at the token's own position; n_s = 1 is exactly
 * pa_decode.  Needs n_s <= c_s, n_s <= max_q_len, c_s <= max_context_len; values outside
 * are cut to those bounds and set bit 2 of the workspace error word.
 *
 *   out           device [T][H][d] of out_dtype, T = q_start[S]
 *   query         device [T][H][d] of kv_dtype (fp16 or bf16 only)
 *   q_start       device [S+1] int32, non-decreasing, q_start[0] = 0
 *   k_cache, v_cache, block_tables, context_lens, B, n_blocks, max_blocks_per_seq: as pa_decode
 *   max_q_len     host bound on every n_s
 *   scale         any finite value (usually 1/sqrt(d))
 *   workspace     device scratch of pa_prefill_workspace_size(...) bytes, 256-byte aligned; its
 *                 error word (pa_workspace_error) has bit 1 set if a bounded wait gave up and
 *                 bit 2 if a size was cut to its bound
 *
 * Kernels: sequences with two or more query tokens run on tcgen05 tensor cores with the S and O
 * accumulators and P in tensor memory (default; the environment variable
 * PA_PREFILL_CONSUMER=mma_sync selects the mma.sync kernel instead; both give the same results
 * within the tolerance, P being carried as two 16-bit parts).  Sequences with exactly one query
 * token -- the decode rows of a mixed batch -- are computed by pa_decode's kernels in the same call
 * (the decode definition is the n_s = 1 case), which stream their context at the HBM rate.
 */
size_t pa_prefill_workspace_size(int S, int H, int Hk, int d, int max_context_len, int max_q_len);

pa_status pa_prefill(void* out, pa_dtype out_dtype, const void* query, const int32_t* q_start,
                     const void* k_cache, const void* v_cache, const int32_t* block_tables,
                     const int32_t* context_lens, int S, int H, int Hk, int d, int B, int n_blocks,
                     int max_blocks_per_seq, int max_context_len, int max_q_len, float scale,
                     pa_dtype kv_dtype, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * Block swap for preemption by swapping ("PagedAttention原理", "抢占与恢复", swap: a preempted
 * sequence's blocks move to CPU memory and are moved back before it runs again; the CPU pool is at
 * most as large as the GPU pool).  For each pair p: block pairs[p][1] of the destination pool
 * becomes a bit copy of block pairs[p][0] of the source pool, for K and for V.  Both pools have the
 * [n][Hk][B][d] layout of the caches; one is normally the device cache and the other pinned host
 * memory (cudaHostAlloc / cudaHostRegister), which the kernel reads or writes over the host link.
 * Destination blocks must be distinct.  Out-of-range ids are skipped.
 *
 *   dst_k, dst_v  [n_dst_blocks][Hk][B][d], device or pinned host
 *   src_k, src_v  [n_src_blocks][Hk][B][d], device or pinned host
 *   pairs         [P][2] int32 (src, dst), device or pinned host
 */
pa_status pa_swap_blocks(void* dst_k, void* dst_v, int n_dst_blocks, const void* src_k, const void* src_v,
                         int n_src_blocks, const int32_t* pairs, int P, int Hk, int d, int B, pa_dtype dtype,
                         void* stream);

/* ---------------------------------------------------------------------------------------------
 * A whole decode step as one replayable CUDA graph.
 *
 * One step of serving, in stream order: copy the step's inputs from pinned host buffers to the
 * device, pa_copy_blocks on the step's copy-on-write pairs, pa_cache_write of one new token per
 * sequence, pa_decode, and copy the output back to the host.  pa_step_create captures this once
 * into a CUDA graph over the fixed buffers named in the descriptor; pa_step_run replays it, so a
 * step costs one graph launch instead of a dozen API calls (the copy-on-write count, which varies
 * from step to step, travels in pinned memory with the other inputs).  The caller refills the host
 * buffers (e.g. with pa_seq_reserve_slots_batch and pa_build_block_tables) before each run.  Host
 * inputs that are laid out like their device buffers (same offsets from one host block and one
 * device block, gaps up to 4 KiB) are copied with a single transfer.
 */
typedef struct {
  /* pinned host buffers (cudaHostAlloc / cudaHostRegister memory), read or written by each run */
  const void* h_query;          /* [S][H][d] kv_dtype */
  const void* h_key;            /* [S][Hk][d] kv_dtype: the new token of each sequence */
  const void* h_value;          /* [S][Hk][d] kv_dtype */
  const int64_t* h_slots;       /* [S] slot of each new token (< 0: no token) */
  const int32_t* h_pairs;       /* [max_pairs][2] copy-on-write (src, dst) pairs */
  const int32_t* h_n_pairs;     /* one int: pairs used this step, 0 .. max_pairs */
  const int32_t* h_tables;      /* [S][max_blocks_per_seq] */
  const int32_t* h_lens;        /* [S] context lengths including the new token */
  void* h_out;                  /* [S][H][d] out_dtype, written by each run */
  /* device buffers (the same sizes), plus the caches and a decode workspace */
  void* d_query;
  void* d_key;
  void* d_value;
  int64_t* d_slots;
  int32_t* d_pairs;             /* [max_pairs][2] followed by one int (the count): 8*max_pairs+16 bytes */
  int32_t* d_tables;
  int32_t* d_lens;
  void* d_out;
  void* k_cache;
  void* v_cache;
  void* workspace;
  size_t workspace_bytes;
  /* sizes */
  int S, H, Hk, d, B, n_blocks, max_blocks_per_seq, max_context_len, max_pairs, partition_size;
  float scale;
  pa_dtype kv_dtype, out_dtype;
} pa_step_desc;

typedef struct pa_step pa_step;

/* Validates the descriptor, captures the step into a graph (on a private stream of the current
 * device) and instantiates it.  The capture itself runs nothing.  Every host buffer must be pinned.
 * NULL on failure (pa_last_error() says why). */
pa_step* pa_step_create(const pa_step_desc* desc);

/* Launches the captured step on `stream` and waits for it (the output is in h_out on return). */
pa_status pa_step_run(pa_step* step, void* stream);

/* Launches the captured step on `stream` and returns at once; the output is in h_out once the
 * stream has reached this point.  With two steps (two sets of buffers) a caller can prepare the
 * next step's inputs on the host while the GPU runs the current one. */
pa_status pa_step_launch(pa_step* step, void* stream);

/* Pipelined form of pa_step_launch: returns at once, and the step's transfers overlap the kernels
 * of neighbouring steps.  The host->device copy of the inputs runs on a copy stream of the step
 * (after this step's previous kernels are done with its device inputs); the kernels (copy-on-write
 * copy, cache write, decode; captured once as a graph) run on `stream` once that copy has landed
 * and this step's previous output copy has left d_out; the device->host copy of the output runs on
 * a second copy stream once the kernels are done.  All kernels of all steps launched on one
 * `stream` run in launch order, so the caches see the steps in order.  The caller may refill this
 * step's host inputs, and read h_out, only after pa_step_wait(step).  With two steps (two sets of
 * buffers) launched alternately, step i+1's input copy and step i-1's output copy overlap step i's
 * kernels. */
pa_status pa_step_launch_async(pa_step* step, void* stream);

/* Blocks until the output copy of this step's last pa_step_launch_async has completed (at once if
 * there was none). */
pa_status pa_step_wait(pa_step* step);

void pa_step_destroy(pa_step* step);

/* ---------------------------------------------------------------------------------------------
 * Host block manager ("从虚拟内存的启发", "解决共享prompt", "解决COW", "COW 区别").  Pure CPU; a handle
 * must not be used by two threads at once.  Policies (the pages leave them open):
 *   - free blocks form a LIFO stack that starts as [n_blocks-1, ..., 1, 0]: the first allocation
 *     returns 0 and the most recently freed block is handed out next;
 *   - sequence ids are 0, 1, 2, ... in creation order and are never reused;
 *   - freeing a sequence releases its blocks in logical order;
 *   - a reservation that cannot get every block it needs fails with PA_ERR_NO_FREE_BLOCK and
 *     leaves all state unchanged.
 */
typedef struct pa_alloc pa_alloc;

/* New manager over n_blocks physical blocks of B tokens; NULL on bad arguments. */
pa_alloc* pa_alloc_create(int n_blocks, int B);
void pa_alloc_destroy(pa_alloc* a);

/* Take one free block with reference count 1. */
pa_status pa_alloc_block(pa_alloc* a, int32_t* block_id);
/* Reference counting of an allocated block; decref releases the block when the count hits 0. */
pa_status pa_block_incref(pa_alloc* a, int32_t block_id);
pa_status pa_block_decref(pa_alloc* a, int32_t block_id);
/* Current count (0 = free), or -1 for an id out of range. */
int pa_block_refcount(const pa_alloc* a, int32_t block_id);
int pa_alloc_num_free(const pa_alloc* a);

/* Sequences: an empty sequence; a fork that shares every block of the parent (each block's count
 * goes up by one; the child has the parent's length); free (every block's count goes down by
 * one).  Parallel sampling and beam search build on fork ("Paged Attention&Orca Paper笔记与解读",
 * parallel sampling and beam search items). */
pa_status pa_seq_create(pa_alloc* a, int32_t* seq_id);
pa_status pa_seq_fork(pa_alloc* a, int32_t parent, int32_t* child);
pa_status pa_seq_free(pa_alloc* a, int32_t seq_id);
/* Batched forms for a serving step (beam search re-parenting): fork each of parents[0..n) in
 * order (children[i] receives the new id; a parent may appear several times), or free each of
 * seq_ids[0..n) in order.  They stop at the first unknown id and return its status; the forks or
 * frees before it stay done. */
pa_status pa_seq_fork_batch(pa_alloc* a, const int32_t* parents, int n, int32_t* children);
pa_status pa_seq_free_batch(pa_alloc* a, const int32_t* seq_ids, int n);

/* Length (tokens) of a sequence, or -1 if unknown. */
int pa_seq_len(const pa_alloc* a, int32_t seq_id);

/* Reserve the slots of the next n_new tokens of a sequence.
 * For each new token, in order:
 *   - the last block is full (or there is none): take a fresh block; nothing is copied, even if
 *     the full block is shared;
 *   - the last block has room and count 1: write in place;
 *   - the last block has room and count > 1: copy-on-write -- (1) take a new block, (2) emit the
 *     pair (old, new) for pa_copy_blocks, (3) map the logical block to the new block,
 *     (4) decrement the old block's count, (5) the token's slot is in the new block.
 * slots      host [n_new] int64: slot = physical_block * B + offset, for pa_cache_write.
 * cow_pairs  host [>= 1][2] int32 (src, dst), filled with *n_cow pairs (0 or 1 per call).
 * The caller copies first (pa_copy_blocks), then writes (pa_cache_write), then decodes. */
pa_status pa_seq_reserve_slots(pa_alloc* a, int32_t seq_id, int n_new, int64_t* slots,
                               int32_t* cow_pairs, int* n_cow);

/* One decode step of a batch: reserves n_new slots for each of seq_ids[0..S), in order, exactly as
 * S calls of pa_seq_reserve_slots would.  slots: host [S * n_new] int64 (sequence i's slots at
 * i*n_new).  cow_pairs: host [S][2] int32, filled with *n_cow pairs.  Each sequence's reservation
 * is atomic; on the first failure the call stops, sets *n_done to the number of sequences already
 * reserved (their slots and pairs are valid) and returns that failure's status.  On success
 * *n_done = S. */
pa_status pa_seq_reserve_slots_batch(pa_alloc* a, const int32_t* seq_ids, int S, int n_new, int64_t* slots,
                                     int32_t* cow_pairs, int* n_cow, int* n_done);

/* Number of blocks in a sequence's table, or -1 if unknown. */
int pa_seq_num_blocks(const pa_alloc* a, int32_t seq_id);

/* Pack the block tables of seq_ids[0..S) into host tables [S][max_blocks_per_seq] (unused entries
 * -1) and their lengths into host context_lens [S].  PA_ERR_INVALID_ARG if a sequence is unknown
 * or has more than max_blocks_per_seq blocks (nothing is written then). */
pa_status pa_build_block_tables(const pa_alloc* a, const int32_t* seq_ids, int S, int32_t* tables,
                                int max_blocks_per_seq, int32_t* context_lens);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */

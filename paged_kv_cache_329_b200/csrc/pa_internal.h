// Host-side helpers shared by the translation units of libpa (not part of the public ABI).
#pragma once
#include <cstdarg>
#include <cstddef>
#include <cstdint>

#include "pa.h"

namespace pa {

// Records a printf-style message for pa_last_error() and returns `st`.
pa_status fail(pa_status st, const char* fmt, ...);
// Clears the message and returns PA_OK.
pa_status ok();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t elem_size(pa_dtype t) { return t == PA_F32 ? 4 : 2; }
inline bool valid_dtype(int t) { return t == PA_F32 || t == PA_F16 || t == PA_BF16; }

// Id of the calling thread's current CUDA context, 0 if there is none or it cannot be had.  The
// driver never reuses an id within a process, so a set-up that belongs to a context (a kernel's
// shared-memory size attribute, kept per device and lost with a device reset) can be keyed on it.
unsigned long long current_context_id();

// Most copy pairs pa_decode_step takes (their destinations are held in shared memory).
constexpr int kMaxStepPairs = 8192;

// pa_copy_blocks whose pair count is read on the device from *n_pairs_dev (clamped to max_pairs);
// the grid is sized for max_pairs so the launch can be captured once and replayed.
pa_status copy_blocks_counted(void* k_cache, void* v_cache, const int32_t* pairs, const int32_t* n_pairs_dev,
                              int max_pairs, int Hk, int d, int B, int n_blocks, pa_dtype dtype, void* stream);

// Decode attention of the sequences of a mixed batch that have exactly one query token
// (q_start[s+1] - q_start[s] == 1): query and output row q_start[s], the decode kernels of
// pa_decode, a cut length or a kernel error or-ed into *err (a device int).  The workspace is
// decode_single_rows_workspace(...) bytes, 256-byte aligned.
size_t decode_single_rows_workspace(int S, int H, int Hk, int d, int max_context_len);
pa_status decode_single_rows(void* out, pa_dtype out_dtype, const void* query, const int32_t* q_start,
                             const void* k_cache, const void* v_cache, const int32_t* block_tables,
                             const int32_t* context_lens, int S, int H, int Hk, int d, int B, int n_blocks,
                             int max_blocks_per_seq, int max_context_len, float scale, pa_dtype kv_dtype,
                             void* workspace, size_t workspace_bytes, int* err, void* stream);

}  // namespace pa

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

// Most copy pairs pa_decode_step takes (their destinations are held in shared memory).
constexpr int kMaxStepPairs = 8192;

// pa_copy_blocks whose pair count is read on the device from *n_pairs_dev (clamped to max_pairs);
// the grid is sized for max_pairs so the launch can be captured once and replayed.
pa_status copy_blocks_counted(void* k_cache, void* v_cache, const int32_t* pairs, const int32_t* n_pairs_dev,
                              int max_pairs, int Hk, int d, int B, int n_blocks, pa_dtype dtype, void* stream);

}  // namespace pa

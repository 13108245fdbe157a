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

}  // namespace pa

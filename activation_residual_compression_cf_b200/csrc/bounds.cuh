// bounds.cuh -- index checks of the bounds-checked debug build.
//
// Built with -DCF_DEBUG_BOUNDS (build.build(debug=True) -> libcf_debug.so),
// CF_IN(cond) states, at a global or shared-memory access, that the index
// arithmetic keeps the access inside its array: `cond` is evaluated, and if
// it is false the first failure's source location is recorded in this
// translation unit's g_bounds_hit word and the guarded access is skipped.
// Nothing traps.  The release build compiles every CF_IN to `true`, so the
// guarded code is the shipped code with the checks removed.
//
// A failure is recorded as (file tag << 16) | line, the tag a 15-bit hash
// of the file name (bounds_file_tag) that the host side reproduces.
#pragma once

#include <stdint.h>

namespace cf {

// FNV-1a of the file's base name (the part after the last '/'), folded to
// 15 bits, so a tag does not depend on where the sources were built.
__host__ __device__ constexpr uint32_t bounds_file_tag(const char *s) {
    const char *b = s;
    for (const char *q = s; *q; ++q)
        if (*q == '/') b = q + 1;
    uint32_t h = 2166136261u;
    while (*b) h = (h ^ (uint8_t)*b++) * 16777619u;
    return (h ^ (h >> 15)) & 0x7fffu;
}

#ifdef CF_DEBUG_BOUNDS

// One word per translation unit (no relocatable device code); the host side
// of each unit reads and clears its own (bounds_take_* in the .cu files).
static __device__ int32_t g_bounds_hit = 0;

__device__ __forceinline__ bool bounds_ok(bool ok, uint32_t tag, int line) {
    if (!ok) atomicCAS(&g_bounds_hit, 0, (int32_t)((tag << 16) | (uint32_t)line));
    return ok;
}

#define CF_IN(cond)                                                                        \
    (::cf::bounds_ok((cond), ::cf::BoundsTag<::cf::bounds_file_tag(__FILE__)>::value, __LINE__))
template <uint32_t V>
struct BoundsTag {  // forces the tag to a compile-time constant
    static constexpr uint32_t value = V;
};
constexpr bool kBoundsChecked = true;

#else

#define CF_IN(cond) true
constexpr bool kBoundsChecked = false;

#endif

}  // namespace cf

// check.cuh -- the bounds-checked debug build: compiled with -DDF11_CHECK=1
// (libdf11_check.so), the decode kernels check every shared-memory index and
// every global access against its buffer or section before making it; an
// access outside is skipped and DF11_DEV_ERR_BOUNDS is ORed into the
// launch's error word.  Nothing traps.  The normal build compiles every check
// away.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "df11.h"

#ifndef DF11_CHECK
#define DF11_CHECK 0
#endif

namespace df11 {
namespace {

// [off, off + len) inside [0, cap)?  Always true in the normal build; in the
// check build a violation sets DF11_DEV_ERR_BOUNDS in err.
__device__ __forceinline__ bool in_bounds(uint64_t off, uint64_t len, uint64_t cap, uint32_t &err) {
#if DF11_CHECK
    if (off <= cap && len <= cap - off) return true;
    err |= DF11_DEV_ERR_BOUNDS;
    return false;
#else
    (void)off;
    (void)len;
    (void)cap;
    (void)err;
    return true;
#endif
}

// The same for an access that may be empty (an empty one is always inside).
__device__ __forceinline__ bool in_bounds_or_empty(uint64_t off, uint64_t len, uint64_t cap, uint32_t &err) {
    return len == 0 || in_bounds(off, len, cap, err);
}

}  // namespace
}  // namespace df11

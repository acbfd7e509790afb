// Index predicate of the bounds-checked build (compile with -DRACE_BOUNDS_CHECK): plain
// C++, so that the host tests exercise the same function the kernels call.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define RACE_HD __host__ __device__ __forceinline__
#else
#define RACE_HD inline
#endif

namespace race {

// True when 0 <= i < n.  The unsigned comparison covers negative i (any i < 0 becomes a
// value >= 2^63 > n) and n <= 0 (no index is in range).
RACE_HD bool index_in_range(int64_t i, int64_t n) {
  return n > 0 && (uint64_t)i < (uint64_t)n;
}

}  // namespace race

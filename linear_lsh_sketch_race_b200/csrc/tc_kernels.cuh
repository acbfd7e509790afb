// Tensor-core (tcgen05) kernels of RACE attention.
#pragma once

#include "common.cuh"

namespace race {
namespace tc {

inline bool supported(const race_args_t*) { return false; }
inline size_t forward_workspace(const race_args_t*) { return 0; }
inline race_status_t forward(const race_args_t*, const void*, const void*, const void*,
                             const float*, void*, char*, cudaStream_t) {
  return RACE_ERR_UNSUPPORTED;
}

}  // namespace tc
}  // namespace race

// Shared device/host helpers of the RACE attention library.
//
// Source tags used in comments across csrc/:
//   [JA]  "RACE Attention: 長系列トレーニングのための厳密な線形時間アテンションの技術的概要"
//         (gist.science, Japanese technical overview of arXiv 2510.04008)
//   [IT]  "RACE Attention: A Strictly Linear-Time Attention for Long-Sequence Training"
//         (gist.science, Italian technical summary)
//   [KO]  the same title on gist.science, Korean technical summary
//   [ABS] "Replacing Softmax Similarity with a Sharpened Angular Similarity: Theory and
//         Practice of Scaling To Billion-Context Attention" (arXiv abstract)
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bounds.h"
#include "race_attn.h"

namespace race {

constexpr int kD = 64;          // head dimension handled by every kernel
constexpr int kDV = kD + 1;     // [v | 1]: value columns plus the mass column
constexpr int kNumStride = 68;  // row stride (floats) of [num | den] scratch rows
constexpr float kEpsNorm = 1e-12f;

// Device status flag bits (race_device_status).
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBounds = 2u;

// The library is a single translation unit; this is its only definition.
__device__ uint32_t g_device_status = 0;

__device__ __forceinline__ void raise_status(uint32_t bits) {
  atomicOr(&g_device_status, bits);
}

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// RACE_IN_RANGE(i, n): in the bounds-checked build (-DRACE_BOUNDS_CHECK) false, with the
// bounds bit of the device status flag raised, when i is outside [0, n); the caller then
// skips the access (no trap, no early return, so no barrier is left waiting).  In the
// normal build the condition is the constant true and costs nothing.
#ifdef RACE_BOUNDS_CHECK
__device__ __forceinline__ bool checked_index(int64_t i, int64_t n) {
  if (index_in_range(i, n)) return true;
  raise_status(kStatusBounds);
  return false;
}
#define RACE_IN_RANGE(i, n) (::race::checked_index((int64_t)(i), (int64_t)(n)))
#else
#define RACE_IN_RANGE(i, n) true
#endif

// ---------------------------------------------------------------- element access
template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Logistic function of +-z evaluated without cancellation: returns
// (1/(1+exp(-z)), 1/(1+exp(z))).  With z = 2u/tau these are the two corner
// probabilities of one hyperplane: the softmax over the 2^P corners factorises into
// one such pair per plane, since sum_p c_bp u_p splits over planes.
__device__ __forceinline__ void logistic_pair(float z, float &sp, float &sm) {
  float e = expf(-fabsf(z));          // in (0, 1]
  float big = 1.0f / (1.0f + e);      // sigma(|z|)
  float small = e * big;              // sigma(-|z|) = e / (1 + e)
  if (z >= 0.f) { sp = big; sm = small; } else { sp = small; sm = big; }
}

// Problem sizes shared by host planning and kernels.
struct Dims {
  int64_t N;
  int H, L, P, R;
  float tau;
  int causal;
  int64_t w_hs;   // floats between the hash planes of consecutive heads (0: shared W)
};

}  // namespace race

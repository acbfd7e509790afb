// Classic RACE with hard hashes (the tau -> 0 limit of the soft estimator): repeated
// arrays of counts ([JA] §2.1: count estimators, bucket aggregation; [KO] §2: L tables of
// P-bit buckets).  Integer and memory-bound work on CUDA cores:
//
//   k_hard_ids    bucket ids h_l(x) = sum_p [W_l[:,p] . x >= 0] 2^p, uint8 [H][N][L]
//   k_hard_seg    per (head, table, segment): key counts C[b] (int32) and value sums
//                 V[b][64] (float32) of the segment, in shared memory, then to global
//   k_hard_scan   exclusive prefix (causal) or total (non-causal) of the segments, with
//                 counts in int64-free int32 (a head holds fewer than 2^31 tokens)
//   k_hard_sweep  per (head, table, segment): the running arrays start from the scanned
//                 prefix; per chunk of 128 queries, each query reads C and V at its bucket
//                 (plus the keys j <= i of its chunk in that bucket, causal), then the
//                 chunk's keys are added; per-table results are summed over tables into
//                 num[h][n][0..63] (float32 atomics) and cnt[h][n] (int32 atomics)
//   k_hard_normalize  o = num / cnt, 0 where no key collides (cnt = 0)
//
// The sign decision x . W_l[:,p] >= 0 is taken in float32 on the unnormalised x (the same
// sign as for x / |x|; x = 0 gives all bits set, as x / max(|x|, eps) = 0 does).
#pragma once

#include "common.cuh"

namespace race {
namespace hard {

constexpr int kHT = 256;     // threads per CTA
constexpr int kHC = 128;     // tokens per chunk of the sweep

// ids[h][n][l] for 32 tokens per CTA; W of the head (w_hs floats apart when per head).
template <typename T>
__global__ void __launch_bounds__(kHT) k_hard_ids(const T* __restrict__ x,
                                                  const float* __restrict__ W,
                                                  uint8_t* __restrict__ ids, int64_t N,
                                                  int L, int P, int64_t w_hs) {
  __shared__ float xs[32][kD + 1];
  const int h = blockIdx.y;
  const int64_t n0 = (int64_t)blockIdx.x * 32;
  const T* xh = x + ((size_t)h * N + n0) * kD;
  const float* Wh = W + (size_t)h * w_hs;
  for (int e = threadIdx.x; e < 32 * kD; e += kHT) {
    const int t = e / kD, c = e % kD;
    xs[t][c] = (n0 + t < N) ? to_f(xh[(size_t)t * kD + c]) : 0.f;
  }
  __syncthreads();
  const int t = threadIdx.x & 31;
  if (n0 + t >= N) return;
  for (int l = threadIdx.x >> 5; l < L; l += kHT / 32) {
    const float* Wl = Wh + (size_t)l * kD * P;
    uint32_t id = 0;
    for (int p = 0; p < P; ++p) {
      float u = 0.f;
#pragma unroll 8
      for (int c = 0; c < kD; ++c) u = fmaf(xs[t][c], Wl[c * P + p], u);
      id |= (u >= 0.f ? 1u : 0u) << p;
    }
    ids[((size_t)h * N + n0 + t) * L + l] = (uint8_t)id;
  }
}

// Segment arrays of one (head, table, segment): cnt[b] and val[b][64].
template <typename T>
__global__ void __launch_bounds__(kHT) k_hard_seg(const uint8_t* __restrict__ kid,
                                                  const T* __restrict__ v,
                                                  int* __restrict__ cseg,
                                                  float* __restrict__ vseg, int64_t N, int L,
                                                  int R, int G, int64_t seg_len) {
  extern __shared__ float hsm[];
  float* V = hsm;                                   // [R][64]
  int* C = reinterpret_cast<int*>(V + (size_t)R * kD);
  const int g = blockIdx.x, l = blockIdx.y, h = blockIdx.z;
  for (int e = threadIdx.x; e < R * kD; e += kHT) V[e] = 0.f;
  for (int e = threadIdx.x; e < R; e += kHT) C[e] = 0;
  __syncthreads();
  const int64_t s0 = (int64_t)g * seg_len, s1 = min64(N, s0 + seg_len);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t j = s0 + warp; j < s1; j += kHT / 32) {   // one warp per key
    const int b = kid[((size_t)h * N + j) * L + l];
    if (!RACE_IN_RANGE(b, R)) continue;   // bounds-checked build: a corrupt id is skipped
    const T* vj = v + ((size_t)h * N + j) * kD;
    atomicAdd(&V[b * kD + lane], to_f(vj[lane]));
    atomicAdd(&V[b * kD + lane + 32], to_f(vj[lane + 32]));
    if (lane == 0) atomicAdd(&C[b], 1);
  }
  __syncthreads();
  const size_t o = (((size_t)h * L + l) * G + g) * R;
  for (int e = threadIdx.x; e < R * kD; e += kHT) vseg[o * kD + e] = V[e];
  for (int e = threadIdx.x; e < R; e += kHT) cseg[o + e] = C[e];
}

// Exclusive prefix (mode 0) or total (mode 2) over the segments, in fixed order; one thread
// per (bucket, column) of one (head, table): column 64 is the count.
__global__ void k_hard_scan(const int* __restrict__ cseg, const float* __restrict__ vseg,
                            int* __restrict__ cinit, float* __restrict__ vinit, int R, int G,
                            int mode) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;    // over R * 65
  if (e >= R * kDV) return;
  const size_t unit = blockIdx.y;                          // head * L + table
  const int b = e / kDV, c = e % kDV;
  if (c < kD) {
    const size_t base = unit * G * R * kD + (size_t)b * kD + c;
    float run = 0.f, tot = 0.f;
    for (int g = 0; g < G; ++g) tot += vseg[base + (size_t)g * R * kD];
    for (int g = 0; g < G; ++g) {
      vinit[base + (size_t)g * R * kD] = mode == 2 ? tot : run;
      run += vseg[base + (size_t)g * R * kD];
    }
  } else {
    const size_t base = unit * G * R + b;
    int run = 0, tot = 0;
    for (int g = 0; g < G; ++g) tot += cseg[base + (size_t)g * R];
    for (int g = 0; g < G; ++g) {
      cinit[base + (size_t)g * R] = mode == 2 ? tot : run;
      run += cseg[base + (size_t)g * R];
    }
  }
}

// The sweep of one (head, table, segment); num[h][n][64] and cnt[h][n] receive the sum
// over tables (zeroed by the caller).
template <typename T>
__global__ void __launch_bounds__(kHT) k_hard_sweep(
    const uint8_t* __restrict__ qid, const uint8_t* __restrict__ kid,
    const T* __restrict__ v, const int* __restrict__ cinit, const float* __restrict__ vinit,
    float* __restrict__ num, int* __restrict__ cnt, int64_t N, int L, int R, int G,
    int64_t seg_len, int causal, int have_init) {
  extern __shared__ float hsm[];
  float* V = hsm;                                    // [R][64] running value sums
  int* C = reinterpret_cast<int*>(V + (size_t)R * kD);   // [R] running counts
  int* kb = C + R;                                   // [kHC] bucket of the chunk's keys
  float* vc = reinterpret_cast<float*>(kb + kHC);   // [kHC][64] the chunk's values
  const int g = blockIdx.x, l = blockIdx.y, h = blockIdx.z;
  const size_t o = (((size_t)h * L + l) * G + g) * R;
  for (int e = threadIdx.x; e < R * kD; e += kHT) V[e] = have_init ? vinit[o * kD + e] : 0.f;
  for (int e = threadIdx.x; e < R; e += kHT) C[e] = have_init ? cinit[o + e] : 0;
  __syncthreads();
  const int64_t s0 = (int64_t)g * seg_len, s1 = min64(N, s0 + seg_len);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t c0 = s0; c0 < s1; c0 += kHC) {
    const int nt = (int)min64(kHC, s1 - c0);
    if (causal) {   // the chunk's keys: buckets and values
      for (int e = threadIdx.x; e < nt; e += kHT) kb[e] = kid[((size_t)h * N + c0 + e) * L + l];
      for (int e = threadIdx.x; e < nt * kD; e += kHT)
        vc[e] = to_f(v[((size_t)h * N + c0) * kD + e]);
      __syncthreads();
    }
    // queries: one warp each, two value columns per lane
    for (int t = warp; t < nt; t += kHT / 32) {
      const int64_t i = c0 + t;
      const int b = qid[((size_t)h * N + i) * L + l];
      if (!RACE_IN_RANGE(b, R)) continue;
      float a0 = V[b * kD + lane], a1 = V[b * kD + lane + 32];
      int n = C[b];
      if (causal) {
        for (int j = 0; j <= t; ++j)
          if (kb[j] == b) {
            a0 += vc[j * kD + lane];
            a1 += vc[j * kD + lane + 32];
            ++n;
          }
      }
      if (n > 0) {
        float* dst = num + ((size_t)h * N + i) * kD;
        atomicAdd(dst + lane, a0);
        atomicAdd(dst + lane + 32, a1);
        if (lane == 0) atomicAdd(cnt + (size_t)h * N + i, n);
      }
    }
    if (causal) {   // the chunk's keys join the running arrays
      __syncthreads();
      for (int t = warp; t < nt; t += kHT / 32) {
        const int b = kb[t];
        if (!RACE_IN_RANGE(b, R)) continue;
        atomicAdd(&V[b * kD + lane], vc[t * kD + lane]);
        atomicAdd(&V[b * kD + lane + 32], vc[t * kD + lane + 32]);
        if (lane == 0) atomicAdd(&C[b], 1);
      }
      __syncthreads();
    }
  }
}

template <typename TO>
__global__ void k_hard_normalize(const float* __restrict__ num, const int* __restrict__ cnt,
                                 TO* __restrict__ out, int64_t rows) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= rows * kD) return;
  const int n = cnt[e / kD];
  out[e] = from_f<TO>(n > 0 ? num[e] / (float)n : 0.f);
}

inline size_t seg_smem(int R) { return (size_t)R * kD * sizeof(float) + (size_t)R * sizeof(int); }
inline size_t sweep_smem(int R) {
  return seg_smem(R) + kHC * sizeof(int) + (size_t)kHC * kD * sizeof(float);
}

}  // namespace hard
}  // namespace race

// CUDA-core ("SIMT") kernels of RACE attention: every dtype, every size, forward
// and backward.  They are the float32 path (tensor cores cannot meet a 1e-5
// relative tolerance) and the second GPU implementation the tensor-core kernels are
// checked against.  Tiles of 32 tokens; one CTA per (segment, table, head).
//
// Internal scaling: kernels work with the unscaled softmax blocks p_l instead of
// phi = p_l/sqrt(L), so a'_ij = sum_l p_l(q_i).p_l(k_j) = L * a_ij.  The factor
// cancels in o = num/den; den and the gradients are rescaled where they leave.
//
// Soft hash ([JA] §2.1 soft bucketization; [IT] §2 item 2): the softmax over the
// 2^P corners of <c_b,u>/tau equals prod_p sigma(2 c_bp u_p / tau) exactly, so one
// logistic pair per plane gives every corner probability by P products.
#pragma once

#include "common.cuh"

namespace race {
namespace simt {

constexpr int TT = 32;     // tokens per tile
constexpr int NT = 256;    // threads per CTA
constexpr int XS = kD + 1; // padded row of the x tile

// Shared-memory carve-up of one CTA (floats).  R <= 256, P <= 8.
struct Layout {
  int R, P;
  int off_W, off_xs, off_inv, off_sp, off_sm, off_phia, off_phib, off_vals, off_gpp,
      off_S, off_a, off_b, off_dP, off_dW, total;
  __host__ __device__ Layout(int R_, int P_) : R(R_), P(P_) {
    int o = 0;
    off_W = o;    o += kD * 8;
    off_xs = o;   o += TT * XS;
    off_inv = o;  o += TT;
    off_sp = o;   o += TT * 8;
    off_sm = o;   o += TT * 8;
    off_phia = o; o += TT * R;
    off_phib = o; o += TT * R;
    off_vals = o; o += TT * kNumStride;
    off_gpp = o;  o += TT * kNumStride;
    off_S = o;    o += R * kDV;
    off_a = o;    o += TT * (TT + 1);
    off_b = o;    o += TT * (TT + 1);
    off_dP = o;   o += TT * R;
    off_dW = o;   o += kD * 8;
    total = o;
  }
  __host__ __device__ size_t bytes() const { return size_t(total) * sizeof(float); }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// W_l [d][P] of table l into shared memory as Ws[c*P + p].
__device__ __forceinline__ void load_W(const float* __restrict__ W, int l, int P,
                                       float* Ws) {
  for (int e = threadIdx.x; e < kD * P; e += blockDim.x) Ws[e] = W[(size_t)l * kD * P + e];
}

// Soft hash of a tile of `ntok` rows of x (rows tok0.. of one head):
// xs <- x, inv <- 1/max(|x|,eps), (sp, sm) <- logistic pair of 2u/tau per plane,
// phi[t][b] <- prod_p (bit p of b ? sp : sm).  Rows t >= ntok get phi = 0.
template <typename T>
__device__ void tile_soft_hash(const T* __restrict__ x, int64_t tok0, int ntok,
                               const float* Ws, int P, int R, float two_over_tau,
                               float* xs, float* inv, float* sp, float* sm, float* phi) {
  for (int e = threadIdx.x; e < TT * kD; e += blockDim.x) {
    int t = e / kD, c = e % kD;
    xs[t * XS + c] = (t < ntok) ? to_f(x[(tok0 + t) * kD + c]) : 0.f;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t = warp; t < TT; t += blockDim.x >> 5) {
    float a = xs[t * XS + lane], b = xs[t * XS + lane + 32];
    float s = warp_sum(a * a + b * b);
    if (lane == 0) inv[t] = 1.0f / fmaxf(sqrtf(s), kEpsNorm);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < TT * P; e += blockDim.x) {
    int t = e / P, p = e % P;
    float u = 0.f;
#pragma unroll 8
    for (int c = 0; c < kD; ++c) u = fmaf(xs[t * XS + c], Ws[c * P + p], u);
    u *= inv[t];
    logistic_pair(two_over_tau * u, sp[t * 8 + p], sm[t * 8 + p]);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < TT * R; e += blockDim.x) {
    int t = e / R, b = e - t * R;
    float f = 1.f;
    for (int p = 0; p < P; ++p) f *= ((b >> p) & 1) ? sp[t * 8 + p] : sm[t * 8 + p];
    phi[e] = (t < ntok) ? f : 0.f;
  }
  __syncthreads();
}

// vals[t][0..63] <- v rows, vals[t][64] <- 1 (0 for padding rows).
template <typename T>
__device__ void tile_values(const T* __restrict__ v, int64_t tok0, int ntok, float* vals) {
  for (int e = threadIdx.x; e < TT * kDV; e += blockDim.x) {
    int t = e / kDV, c = e % kDV;
    float val = 0.f;
    if (t < ntok) val = (c < kD) ? to_f(v[(tok0 + t) * kD + c]) : 1.f;
    vals[t * kNumStride + c] = val;
  }
}

// rows[t][0..64] <- src rows (float, stride kNumStride), 0 for padding rows.
__device__ void tile_rows65(const float* __restrict__ src, int64_t tok0, int ntok,
                            float* rows) {
  for (int e = threadIdx.x; e < TT * kDV; e += blockDim.x) {
    int t = e / kDV, c = e % kDV;
    rows[t * kNumStride + c] = (t < ntok) ? src[(tok0 + t) * kNumStride + c] : 0.f;
  }
}

// S[b][c] += sum_t phi[t][b] * rows[t][c]   (bucket aggregation, [JA] §2.1)
__device__ void state_update(float* S, const float* phi, const float* rows, int R) {
  for (int e = threadIdx.x; e < R * kDV; e += blockDim.x) {
    int b = e / kDV, c = e - b * kDV;
    float acc = S[e];
#pragma unroll 8
    for (int t = 0; t < TT; ++t) acc = fmaf(phi[t * R + b], rows[t * kNumStride + c], acc);
    S[e] = acc;
  }
}

// --------------------------------------------------------------------------- //
// race_hash: phi dump
// --------------------------------------------------------------------------- //
template <typename T, typename TO>
__global__ void __launch_bounds__(NT) k_hash(const T* __restrict__ x,
                                             const float* __restrict__ W,
                                             TO* __restrict__ phi_out, Dims dm) {
  extern __shared__ float sm_[];
  Layout ly(dm.R, dm.P);
  const int h = blockIdx.y;
  const int64_t tok0 = (int64_t)blockIdx.x * TT;
  const int ntok = (int)min64(TT, dm.N - tok0);
  const T* xh = x + (size_t)h * dm.N * kD;
  const float scale = rsqrtf((float)dm.L);
  const int LR = dm.L * dm.R;
  for (int l = 0; l < dm.L; ++l) {
    load_W(W + (size_t)h * dm.w_hs, l, dm.P, sm_ + ly.off_W);
    __syncthreads();
    tile_soft_hash(xh, tok0, ntok, sm_ + ly.off_W, dm.P, dm.R, 2.f / dm.tau,
                   sm_ + ly.off_xs, sm_ + ly.off_inv, sm_ + ly.off_sp, sm_ + ly.off_sm,
                   sm_ + ly.off_phia);
    for (int e = threadIdx.x; e < ntok * dm.R; e += blockDim.x) {
      int t = e / dm.R, b = e - t * dm.R;
      phi_out[((size_t)h * dm.N + tok0 + t) * LR + (size_t)l * dm.R + b] =
          from_f<TO>(sm_[ly.off_phia + e] * scale);
    }
    __syncthreads();
  }
}

// --------------------------------------------------------------------------- //
// Segment sums of the sketch: seg[h][l][g] = sum_{t in segment g} p_l(x_t) rows_t^T.
// MODE 0: x = k, rows = [v | 1]  (forward state S|z)
// MODE 1: x = q, rows = g''      (backward suffix state T|-t)
// --------------------------------------------------------------------------- //
template <typename T, int MODE>
__global__ void __launch_bounds__(NT) k_build(const T* __restrict__ x,
                                              const T* __restrict__ v,
                                              const float* __restrict__ gpp,
                                              const float* __restrict__ W,
                                              float* __restrict__ seg, Dims dm, int G,
                                              int64_t seg_len) {
  extern __shared__ float sm_[];
  Layout ly(dm.R, dm.P);
  const int g = blockIdx.x, l = blockIdx.y, h = blockIdx.z;
  const int64_t s0 = (int64_t)g * seg_len, s1 = min64(dm.N, s0 + seg_len);
  float* S = sm_ + ly.off_S;
  for (int e = threadIdx.x; e < dm.R * kDV; e += blockDim.x) S[e] = 0.f;
  load_W(W + (size_t)h * dm.w_hs, l, dm.P, sm_ + ly.off_W);
  __syncthreads();
  const T* xh = x + (size_t)h * dm.N * kD;
  for (int64_t t0 = s0; t0 < s1; t0 += TT) {
    int ntok = (int)min64(TT, s1 - t0);
    tile_soft_hash(xh, t0, ntok, sm_ + ly.off_W, dm.P, dm.R, 2.f / dm.tau,
                   sm_ + ly.off_xs, sm_ + ly.off_inv, sm_ + ly.off_sp, sm_ + ly.off_sm,
                   sm_ + ly.off_phia);
    if (MODE == 0)
      tile_values(v + (size_t)h * dm.N * kD, t0, ntok, sm_ + ly.off_vals);
    else
      tile_rows65(gpp + (size_t)h * dm.N * kNumStride, t0, ntok, sm_ + ly.off_vals);
    __syncthreads();
    state_update(S, sm_ + ly.off_phia, sm_ + ly.off_vals, dm.R);
    __syncthreads();
  }
  float* out = seg + (((size_t)h * dm.L + l) * G + g) * dm.R * kDV;
  for (int e = threadIdx.x; e < dm.R * kDV; e += blockDim.x) out[e] = S[e];
}

// Prefix of segment sums along the sequence, in fixed order ([JA] §2.2 prefix sums).
// mode 0: exclusive prefix, 1: exclusive suffix, 2: total (written to every g).
__global__ void k_scan(const float* __restrict__ seg, float* __restrict__ init, int RD,
                       int G, int mode) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= RD) return;
  const size_t base = (size_t)blockIdx.y * G * RD + e;
  if (mode == 2) {
    float tot = 0.f;
    for (int g = 0; g < G; ++g) tot += seg[base + (size_t)g * RD];
    for (int g = 0; g < G; ++g) init[base + (size_t)g * RD] = tot;
  } else if (mode == 0) {
    float run = 0.f;
    for (int g = 0; g < G; ++g) {
      float s = seg[base + (size_t)g * RD];
      init[base + (size_t)g * RD] = run;
      run += s;
    }
  } else {
    float run = 0.f;
    for (int g = G - 1; g >= 0; --g) {
      float s = seg[base + (size_t)g * RD];
      init[base + (size_t)g * RD] = run;
      run += s;
    }
  }
}

// The same prefix with a carried state (streaming): unit u = (head, row group) holds
// `rows` sketch rows of `ncols` columns (65 used) per segment; carry_in / carry_out are the
// public state [H][L*R][65] (sketch row = row group * rows + row).  Segment g starts from
// carry_in plus the sum of segments before it (causal) or from carry_in plus the total
// (mode 2); carry_out receives carry_in plus the total.  carry_in may be null (zeros) and
// may equal carry_out (each element is read before it is written, by the same thread).
__global__ void k_scan_carry(const float* __restrict__ seg, float* __restrict__ init,
                             const float* carry_in, float* carry_out, int rows, int ncols,
                             int units_per_head, int64_t LR, int G, int mode) {
  const int RD = rows * ncols;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= RD) return;
  const int u = blockIdx.y;
  const int r = e / ncols, c = e % ncols;
  const int64_t h = u / units_per_head, rgx = u % units_per_head;
  const int64_t pub = (h * LR + rgx * rows + r) * kDV + c;
  const size_t base = (size_t)u * G * RD + e;
  const float b0 = (c < kDV && carry_in) ? carry_in[pub] : 0.f;
  float tot = 0.f;
  for (int g = 0; g < G; ++g) tot += seg[base + (size_t)g * RD];
  if (mode == 2) {
    for (int g = 0; g < G; ++g) init[base + (size_t)g * RD] = b0 + tot;
  } else {
    float run = b0;
    for (int g = 0; g < G; ++g) {
      const float sg = seg[base + (size_t)g * RD];
      init[base + (size_t)g * RD] = run;
      run += sg;
    }
  }
  if (c < kDV && carry_out) carry_out[pub] = b0 + tot;
}

// Start state of a sweep: init[h][l][g] when there is one, else zeros.
__device__ void load_state(float* S, const float* init, int h, int l, int g, int G,
                           int R, bool have) {
  const float* src = init + (((size_t)h * gridDim.y + l) * G + g) * R * kDV;
  for (int e = threadIdx.x; e < R * kDV; e += blockDim.x) S[e] = have ? src[e] : 0.f;
}

// --------------------------------------------------------------------------- //
// Forward sweep.  Per tile: num_i += p(q_i).S (+ masked in-tile term), then (causal)
// S += p(k)^T [v|1].  The sum over tables goes to num[h][i][0..64] by atomics.
// Reconstruction: [JA] §2.1; causal prefix: [JA] §2.2.
// --------------------------------------------------------------------------- //
template <typename T>
__global__ void __launch_bounds__(NT) k_fwd_sweep(const T* __restrict__ q,
                                                  const T* __restrict__ k,
                                                  const T* __restrict__ v,
                                                  const float* __restrict__ W,
                                                  const float* __restrict__ init,
                                                  float* __restrict__ num, Dims dm, int G,
                                                  int64_t seg_len, int have_init) {
  extern __shared__ float sm_[];
  Layout ly(dm.R, dm.P);
  const int g = blockIdx.x, l = blockIdx.y, h = blockIdx.z;
  const int R = dm.R;
  const int64_t s0 = (int64_t)g * seg_len, s1 = min64(dm.N, s0 + seg_len);
  float* S = sm_ + ly.off_S;
  float* phq = sm_ + ly.off_phia;
  float* phk = sm_ + ly.off_phib;
  float* vals = sm_ + ly.off_vals;
  float* A = sm_ + ly.off_a;
  load_state(S, init, h, l, g, G, R, have_init != 0);
  load_W(W + (size_t)h * dm.w_hs, l, dm.P, sm_ + ly.off_W);
  __syncthreads();
  const size_t hoff = (size_t)h * dm.N * kD;
  for (int64_t t0 = s0; t0 < s1; t0 += TT) {
    int ntok = (int)min64(TT, s1 - t0);
    tile_soft_hash(q + hoff, t0, ntok, sm_ + ly.off_W, dm.P, R, 2.f / dm.tau,
                   sm_ + ly.off_xs, sm_ + ly.off_inv, sm_ + ly.off_sp, sm_ + ly.off_sm, phq);
    if (dm.causal)
      tile_soft_hash(k + hoff, t0, ntok, sm_ + ly.off_W, dm.P, R, 2.f / dm.tau,
                     sm_ + ly.off_xs, sm_ + ly.off_inv, sm_ + ly.off_sp, sm_ + ly.off_sm,
                     phk);
    tile_values(v + hoff, t0, ntok, vals);
    __syncthreads();
    if (dm.causal) {
      for (int e = threadIdx.x; e < TT * TT; e += blockDim.x) {
        int i = e / TT, j = e % TT;
        float acc = 0.f;
        if (j <= i)
          for (int b = 0; b < R; ++b) acc = fmaf(phq[i * R + b], phk[j * R + b], acc);
        A[i * (TT + 1) + j] = acc;
      }
      __syncthreads();
    }
    for (int e = threadIdx.x; e < ntok * kDV; e += blockDim.x) {
      int i = e / kDV, c = e - i * kDV;
      float acc = 0.f;
      for (int b = 0; b < R; ++b) acc = fmaf(phq[i * R + b], S[b * kDV + c], acc);
      if (dm.causal)
        for (int j = 0; j <= i; ++j) acc = fmaf(A[i * (TT + 1) + j], vals[j * kNumStride + c], acc);
      atomicAdd(num + ((size_t)h * dm.N + t0 + i) * kNumStride + c, acc);
    }
    if (dm.causal) {
      __syncthreads();
      state_update(S, phk, vals, R);
    }
    __syncthreads();
  }
}

// o = num / den  and  den_out = den / L  (den includes the factor L, see top).
template <typename TO>
__global__ void k_normalize(const float* __restrict__ num, TO* __restrict__ out,
                            float* __restrict__ den_out, int64_t rows, float inv_L) {
  const int64_t i = (int64_t)blockIdx.x * (blockDim.x / kD) + threadIdx.x / kD;
  const int c = threadIdx.x % kD;
  if (i >= rows) return;
  const float* r = num + i * kNumStride;
  const float den = r[kD];
  out[i * kD + c] = from_f<TO>(r[c] / den);
  if (den_out && c == 0) den_out[i] = den * inv_L;
}

// Eight consecutive outputs of a row, 16-byte aligned destination.
__device__ __forceinline__ void store8(float* dst, const float* v) {
  __stcs(reinterpret_cast<float4*>(dst), make_float4(v[0], v[1], v[2], v[3]));
  __stcs(reinterpret_cast<float4*>(dst) + 1, make_float4(v[4], v[5], v[6], v[7]));
}
__device__ __forceinline__ void store8(__nv_bfloat16* dst, const float* v) {
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
    w[e] = *reinterpret_cast<const uint32_t*>(&p);
  }
  __stcs(reinterpret_cast<uint4*>(dst), make_uint4(w[0], w[1], w[2], w[3]));
}

// k_normalize with one thread per eight outputs (vector loads and stores, streaming
// cache hints); num rows and out rows must be 16-byte aligned.  Grid-stride loop.
template <typename TO>
__global__ void k_normalize8(const float* __restrict__ num, TO* __restrict__ out,
                             float* __restrict__ den_out, int64_t rows, float inv_L) {
  const int64_t n8 = rows * (kD / 8);
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n8;
       g += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = g >> 3;
    const int part = (int)(g & 7);
    const float* r = num + i * kNumStride;
    const float4 a = __ldcs(reinterpret_cast<const float4*>(r + part * 8));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(r + part * 8) + 1);
    const float den = r[kD];
    const float o[8] = {a.x / den, a.y / den, a.z / den, a.w / den,
                        b.x / den, b.y / den, b.z / den, b.w / den};
    store8(out + i * kD + part * 8, o);
    if (den_out && part == 0) den_out[i] = den * inv_L;
  }
}

// --------------------------------------------------------------------------- //
// backward
// g''_i = [g_i / den'_i , -(g_i . o_i) / den'_i]  with den' = L * den.
// --------------------------------------------------------------------------- //
template <typename T, typename TO>
__global__ void k_gpp(const T* __restrict__ dout, const TO* __restrict__ out,
                      const float* __restrict__ num, const float* __restrict__ den_in,
                      float* __restrict__ gpp, int64_t rows, float L) {
  const int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= rows) return;
  const float den = den_in ? den_in[i] * L : num[i * kNumStride + kD];
  const float inv = 1.0f / den;
  float g0 = to_f(dout[i * kD + lane]), g1 = to_f(dout[i * kD + lane + 32]);
  float o0 = to_f(out[i * kD + lane]), o1 = to_f(out[i * kD + lane + 32]);
  float c = warp_sum(g0 * o0 + g1 * o1);
  float* r = gpp + i * kNumStride;
  r[lane] = g0 * inv;
  r[lane + 32] = g1 * inv;
  if (lane == 0) r[kD] = -c * inv;
}

// Chain rule through the soft hash for one tile and one table (warp per token):
// dlogit_b = p_b (dP_b - <p, dP>); du_p = (1/tau) sum_b c_bp dlogit_b
//          = (1/tau) [sum_b c_bp p_b dP_b - tanh(u_p/tau) sum_b p_b dP_b];
// dxhat += W_l du (atomics into dxh[h][tok][:]); dW_l += xhat du^T (shared atomics).
__device__ void tile_hash_backward(const float* phi, const float* dP, const float* sp,
                                   const float* sm, const float* xs, const float* inv,
                                   const float* Ws, float* dWs, float* __restrict__ dxh,
                                   int64_t tok0, int ntok, int P, int R, float inv_tau) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t = warp; t < ntok; t += blockDim.x >> 5) {
    float sums[9];
#pragma unroll
    for (int p = 0; p < 9; ++p) sums[p] = 0.f;
    for (int b = lane; b < R; b += 32) {
      float w = phi[t * R + b] * dP[t * R + b];
      sums[8] += w;
#pragma unroll
      for (int p = 0; p < 8; ++p)
        if (p < P) sums[p] += ((b >> p) & 1) ? w : -w;
    }
    float du[8];
    float tot = warp_sum(sums[8]);
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      du[p] = 0.f;
      if (p < P) {
        float cs = warp_sum(sums[p]);
        float tnh = sp[t * 8 + p] - sm[t * 8 + p];
        du[p] = inv_tau * (cs - tnh * tot);
      }
    }
    for (int c = lane; c < kD; c += 32) {
      float acc = 0.f;
      for (int p = 0; p < P; ++p) acc = fmaf(Ws[c * P + p], du[p], acc);
      atomicAdd(dxh + (tok0 + t) * kD + c, acc);
      float xh = xs[t * XS + c] * inv[t];
      for (int p = 0; p < P; ++p) atomicAdd(&dWs[c * P + p], xh * du[p]);
    }
  }
}

// Forward-direction backward sweep: dP(q_i) = U_i g''_i (+ in-tile term), then the
// hash backward of q.  U is the same prefix state [S | z] as the forward.
template <typename T>
__global__ void __launch_bounds__(NT) k_bwd_q(const T* __restrict__ q,
                                              const T* __restrict__ k,
                                              const T* __restrict__ v,
                                              const float* __restrict__ W,
                                              const float* __restrict__ init,
                                              const float* __restrict__ gpp,
                                              float* __restrict__ dxq,
                                              float* __restrict__ dWpart, Dims dm, int G,
                                              int64_t seg_len, int have_init) {
  extern __shared__ float sm_[];
  Layout ly(dm.R, dm.P);
  const int g = blockIdx.x, l = blockIdx.y, h = blockIdx.z;
  const int R = dm.R, P = dm.P;
  const int64_t s0 = (int64_t)g * seg_len, s1 = min64(dm.N, s0 + seg_len);
  float* S = sm_ + ly.off_S;
  float* phq = sm_ + ly.off_phia;
  float* phk = sm_ + ly.off_phib;
  float* vals = sm_ + ly.off_vals;
  float* gt = sm_ + ly.off_gpp;
  float* B = sm_ + ly.off_b;
  float* dP = sm_ + ly.off_dP;
  float* dWs = sm_ + ly.off_dW;
  float* spq = sm_ + ly.off_sp;   // q factors stay here: k's hash reuses the x tile only
  float* smq = sm_ + ly.off_sm;
  load_state(S, init, h, l, g, G, R, have_init != 0);
  load_W(W + (size_t)h * dm.w_hs, l, P, sm_ + ly.off_W);
  for (int e = threadIdx.x; e < kD * 8; e += blockDim.x) dWs[e] = 0.f;
  __syncthreads();
  const size_t hoff = (size_t)h * dm.N * kD;
  __shared__ float spk[TT * 8], smk[TT * 8];
  for (int64_t t0 = s0; t0 < s1; t0 += TT) {
    int ntok = (int)min64(TT, s1 - t0);
    if (dm.causal)
      tile_soft_hash(k + hoff, t0, ntok, sm_ + ly.off_W, P, R, 2.f / dm.tau,
                     sm_ + ly.off_xs, sm_ + ly.off_inv, spk, smk, phk);
    tile_soft_hash(q + hoff, t0, ntok, sm_ + ly.off_W, P, R, 2.f / dm.tau,
                   sm_ + ly.off_xs, sm_ + ly.off_inv, spq, smq, phq);
    tile_values(v + hoff, t0, ntok, vals);
    tile_rows65(gpp + (size_t)h * dm.N * kNumStride, t0, ntok, gt);
    __syncthreads();
    if (dm.causal) {
      for (int e = threadIdx.x; e < TT * TT; e += blockDim.x) {
        int i = e / TT, j = e % TT;
        float acc = 0.f;
        if (j <= i)
          for (int c = 0; c < kDV; ++c) acc = fmaf(gt[i * kNumStride + c], vals[j * kNumStride + c], acc);
        B[i * (TT + 1) + j] = acc;
      }
      __syncthreads();
    }
    for (int e = threadIdx.x; e < TT * R; e += blockDim.x) {
      int i = e / R, b = e - i * R;
      float acc = 0.f;
      for (int c = 0; c < kDV; ++c) acc = fmaf(gt[i * kNumStride + c], S[b * kDV + c], acc);
      if (dm.causal)
        for (int j = 0; j <= i; ++j) acc = fmaf(phk[j * R + b], B[i * (TT + 1) + j], acc);
      dP[e] = acc;
    }
    __syncthreads();
    tile_hash_backward(phq, dP, spq, smq, sm_ + ly.off_xs, sm_ + ly.off_inv,
                       sm_ + ly.off_W, dWs, dxq + hoff, t0, ntok, P, R, 1.f / dm.tau);
    __syncthreads();
    if (dm.causal) {
      state_update(S, phk, vals, R);
      __syncthreads();
    }
  }
  float* o = dWpart + (((size_t)h * dm.L + l) * G + g) * kD * P;
  for (int e = threadIdx.x; e < kD * P; e += blockDim.x) o[e] = dWs[e];
}

// Reverse-direction backward sweep with the suffix state Q' = sum_{i later} p(q_i) g''_i^T:
// dP(k_j) = Q' [v_j;1] (+ in-tile term), dv_j = Q'^T p(k_j) restricted to value columns
// (+ in-tile term), then the hash backward of k.
template <typename T>
__global__ void __launch_bounds__(NT) k_bwd_kv(const T* __restrict__ q,
                                               const T* __restrict__ k,
                                               const T* __restrict__ v,
                                               const float* __restrict__ W,
                                               const float* __restrict__ init,
                                               const float* __restrict__ gpp,
                                               float* __restrict__ dxk,
                                               float* __restrict__ dvacc,
                                               float* __restrict__ dWpart, Dims dm, int G,
                                               int64_t seg_len, int have_init) {
  extern __shared__ float sm_[];
  Layout ly(dm.R, dm.P);
  const int g = blockIdx.x, l = blockIdx.y, h = blockIdx.z;
  const int R = dm.R, P = dm.P;
  const int64_t s0 = (int64_t)g * seg_len, s1 = min64(dm.N, s0 + seg_len);
  float* S = sm_ + ly.off_S;
  float* phq = sm_ + ly.off_phia;
  float* phk = sm_ + ly.off_phib;
  float* vals = sm_ + ly.off_vals;
  float* gt = sm_ + ly.off_gpp;
  float* A = sm_ + ly.off_a;
  float* B = sm_ + ly.off_b;
  float* dP = sm_ + ly.off_dP;
  float* dWs = sm_ + ly.off_dW;
  float* spk = sm_ + ly.off_sp;
  float* smk = sm_ + ly.off_sm;
  load_state(S, init, h, l, g, G, R, have_init != 0);
  load_W(W + (size_t)h * dm.w_hs, l, P, sm_ + ly.off_W);
  for (int e = threadIdx.x; e < kD * 8; e += blockDim.x) dWs[e] = 0.f;
  __syncthreads();
  const size_t hoff = (size_t)h * dm.N * kD;
  __shared__ float spq[TT * 8], smq[TT * 8];
  const int64_t ntile = (s1 - s0 + TT - 1) / TT;
  for (int64_t it = ntile - 1; it >= 0; --it) {
    const int64_t t0 = s0 + it * TT;
    int ntok = (int)min64(TT, s1 - t0);
    tile_soft_hash(q + hoff, t0, ntok, sm_ + ly.off_W, P, R, 2.f / dm.tau,
                   sm_ + ly.off_xs, sm_ + ly.off_inv, spq, smq, phq);
    tile_soft_hash(k + hoff, t0, ntok, sm_ + ly.off_W, P, R, 2.f / dm.tau,
                   sm_ + ly.off_xs, sm_ + ly.off_inv, spk, smk, phk);
    tile_values(v + hoff, t0, ntok, vals);
    tile_rows65(gpp + (size_t)h * dm.N * kNumStride, t0, ntok, gt);
    __syncthreads();
    if (dm.causal) {
      for (int e = threadIdx.x; e < TT * TT; e += blockDim.x) {
        int i = e / TT, j = e % TT;
        float a = 0.f, bb = 0.f;
        if (j <= i) {
          for (int b = 0; b < R; ++b) a = fmaf(phq[i * R + b], phk[j * R + b], a);
          for (int c = 0; c < kDV; ++c) bb = fmaf(gt[i * kNumStride + c], vals[j * kNumStride + c], bb);
        }
        A[i * (TT + 1) + j] = a;
        B[i * (TT + 1) + j] = bb;
      }
      __syncthreads();
    }
    for (int e = threadIdx.x; e < TT * R; e += blockDim.x) {
      int j = e / R, b = e - j * R;
      float acc = 0.f;
      for (int c = 0; c < kDV; ++c) acc = fmaf(S[b * kDV + c], vals[j * kNumStride + c], acc);
      if (dm.causal)
        for (int i = j; i < TT; ++i) acc = fmaf(phq[i * R + b], B[i * (TT + 1) + j], acc);
      dP[e] = acc;
    }
    for (int e = threadIdx.x; e < ntok * kD; e += blockDim.x) {
      int j = e / kD, c = e - j * kD;
      float acc = 0.f;
      for (int b = 0; b < R; ++b) acc = fmaf(phk[j * R + b], S[b * kDV + c], acc);
      if (dm.causal)
        for (int i = j; i < TT; ++i) acc = fmaf(A[i * (TT + 1) + j], gt[i * kNumStride + c], acc);
      atomicAdd(dvacc + (hoff + (t0 + j) * kD + c), acc);
    }
    __syncthreads();
    tile_hash_backward(phk, dP, spk, smk, sm_ + ly.off_xs, sm_ + ly.off_inv,
                       sm_ + ly.off_W, dWs, dxk + hoff, t0, ntok, P, R, 1.f / dm.tau);
    __syncthreads();
    if (dm.causal) {
      state_update(S, phq, gt, R);
      __syncthreads();
    }
  }
  float* o = dWpart + (((size_t)h * dm.L + l) * G + g) * kD * P;
  for (int e = threadIdx.x; e < kD * P; e += blockDim.x) o[e] = dWs[e];
}

// dx = (dxhat - xhat (xhat . dxhat)) / |x|  (dxhat / eps when |x| <= eps); warp per row.
template <typename T, typename TG>
__global__ void k_finalize_dx(const T* __restrict__ x, const float* __restrict__ dxh,
                              TG* __restrict__ dx, int64_t rows) {
  const int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= rows) return;
  float x0 = to_f(x[i * kD + lane]), x1 = to_f(x[i * kD + lane + 32]);
  float n = sqrtf(warp_sum(x0 * x0 + x1 * x1));
  float d0 = dxh[i * kD + lane], d1 = dxh[i * kD + lane + 32];
  if (n > kEpsNorm) {
    float inv = 1.f / n;
    float xh0 = x0 * inv, xh1 = x1 * inv;
    float dot = warp_sum(xh0 * d0 + xh1 * d1);
    dx[i * kD + lane] = from_f<TG>((d0 - xh0 * dot) * inv);
    dx[i * kD + lane + 32] = from_f<TG>((d1 - xh1 * dot) * inv);
  } else {
    dx[i * kD + lane] = from_f<TG>(d0 / kEpsNorm);
    dx[i * kD + lane + 32] = from_f<TG>(d1 / kEpsNorm);
  }
}

template <typename T>
__global__ void k_convert(const float* __restrict__ src, T* __restrict__ dst, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = from_f<T>(src[i]);
}

// dW[l][c][p] = sum over heads and segments of both partial buffers, in fixed order;
// with per-head planes dW[h][l][c][p] sums over the segments of head h only.
__global__ void k_dw_reduce(const float* __restrict__ pq, const float* __restrict__ pk,
                            float* __restrict__ dW, int H, int L, int G, int P,
                            int per_head) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int per = kD * P;
  const int n_out = (per_head ? H : 1) * L * per;
  if (e >= n_out) return;
  const int hh = e / (L * per), l = (e / per) % L, r = e % per;
  const int h0 = per_head ? hh : 0, h1 = per_head ? hh + 1 : H;
  float acc = 0.f;
  for (int h = h0; h < h1; ++h)
    for (int g = 0; g < G; ++g) {
      size_t o = (((size_t)h * L + l) * G + g) * per + r;
      acc += pq[o] + pk[o];
    }
  dW[e] = acc;
}

}  // namespace simt
}  // namespace race

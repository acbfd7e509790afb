// Tensor-core (tcgen05 / TMEM / TMA) kernels of RACE attention, bf16 operands with
// float32 accumulation.
//
// Work decomposition.  The sketch of one head has L*R rows (table, bucket) and 65
// value columns [v | 1] (padded to 80).  A CTA owns a row group of 256 rows (one
// table at R = 256, 256/R tables below) for one segment of the sequence and keeps
// its part of the state S = sum_j p(k_j) [v_j | 1]^T in tensor memory as two
// 128 x 80 float32 accumulators.  Per chunk of 128 tokens:
//
//   TMA      q, k, v tiles (128 x 64 bf16, 128-byte swizzle) into shared memory
//   MMA      u = x W_l (projections; W split in bf16 hi + lo, both accumulated)
//   CUDA     soft hash ([JA] §2.1; softmax over corners = product of logistic
//   cores    factors, one pair per plane): expand p(q), p(k) rows to bf16 tiles
//   MMA      QK = p(q) p(k)^T over the CTA's rows           (causal in-chunk term)
//   CUDA     mask j > i, round to bf16, store to TMEM as an A operand
//   MMA      num = p(q) S_bf16 + mask(QK) [v | 1]            (readout, [JA] §2.1)
//   MMA      S  += p(k)^T [v | 1]                            (bucket aggregation)
//   CUDA     num rows -> global float32 accumulators (sum over row groups);
//            S -> bf16 copy in shared memory for the next chunk's readout
//
// The same kernel, by MODE, also builds segment sums (no readout) and runs the
// non-causal readout against a fixed state.  An optional per-key factor kscale[h][n]
// multiplies p(k_n) (the backward's dv pass uses the keys' 1/den').  Segments of one sweep start from the
// exclusive prefix of the segment sums ([JA] §2.2, prefix sums for causal masking).
#pragma once

#include <cudaTypedefs.h>

#include "common.cuh"
#include "simt_kernels.cuh"
#include "tc_ptx.cuh"

namespace race {
namespace tc {

constexpr int kC = 128;          // tokens per chunk: the M of the token-major MMAs
constexpr int kNV = 80;          // state columns: 64 of v, 16 of ones (mass z)
constexpr int kThreads = 160;    // warps 0-3: CUDA-core work (one TMEM lane each); warp 4: issuer
constexpr int kAlu = 128;

enum Mode { kSweep = 0, kBuild = 1, kReadout = 2 };

struct Params {
  int64_t N;
  int H, L, R;
  int rows;          // sketch rows per CTA (128 or 256)
  int tables;        // tables per CTA = rows / R
  int np;            // projection columns, tables * P padded to a multiple of 16
  int n_rg;          // row groups per head = L * R / rows
  int G;             // segments
  int64_t seg_len;   // tokens per segment (multiple of kC)
  float two_over_tau;
  int have_init;
  int lps;           // backward: row stride (elements) of the per-plane gradient arrays
  int64_t w_hs;      // floats between the hash planes of consecutive heads (0: shared W)
};

// Shared-memory map (bytes from a 1024-aligned base).
struct Smem {
  static constexpr uint32_t q = 0;          // 128 x 64 bf16 TMA tile, 128B swizzle
  static constexpr uint32_t k = 16384;
  static constexpr uint32_t v = 32768;
  static constexpr uint32_t phq = 49152;    // 128 tokens x 256 rows bf16, core-matrix layout
  static constexpr uint32_t phk = 114688;
  static constexpr uint32_t sbf = 180224;   // 256 rows x 80 bf16 (readout B operand)
  static constexpr uint32_t whi = 221184;   // 64 x 32 bf16 (projection B operand)
  static constexpr uint32_t wlo = 225280;
  static constexpr uint32_t ones = 229376;  // 16 x 16 bf16 ones
  static constexpr uint32_t bars = 229888;  // 8 mbarriers + TMEM base address
  static constexpr uint32_t total = 230016;
  static constexpr uint32_t alloc = total + 1024;
};

// Tensor-memory columns (float32 accumulators unless noted).
struct Tm {
  static constexpr uint32_t S0 = 0, S1 = 96, num = 192, qk = 288, pq = 288, pk = 320,
                            intra = 416;  // intra: bf16 A operand, 64 columns
};

// One step of the Kronecker tree over planes: entries [0, HALF) become the products
// with the "bit clear" factor and [HALF, 2*HALF) with the "bit set" factor.  A template
// so every index is a compile-time constant (the array stays in registers).
template <int HALF>
__device__ __forceinline__ void kron_step(float* v, float set, float clear) {
#pragma unroll
  for (int c = 0; c < HALF; ++c) {
    v[c + HALF] = v[c] * set;
    v[c] = v[c] * clear;
  }
}

// v[c] for c < 2^(P-FIRST): product over planes FIRST..P-1 of set (bit p-FIRST of c set)
// or clear factors, times v[0] on entry.
template <int FIRST, int P>
__device__ __forceinline__ void kron_tree(float* v, const float* set, const float* clear) {
  if constexpr (FIRST < P) {
    kron_tree<FIRST, P - 1>(v, set, clear);
    kron_step<(1 << (P - 1 - FIRST))>(v, set[P - 1], clear[P - 1]);
  }
}

// --------------------------------------------------------------------------- helpers
__device__ __forceinline__ void logistic_fast(float z, float& sp, float& sm) {
  const float e = __expf(-fabsf(z));
  const float big = __fdividef(1.0f, 1.0f + e);
  const float small = e * big;
  sp = z >= 0.f ? big : small;
  sm = z >= 0.f ? small : big;
}

// Soft-hash rows of one token for `tables` consecutive tables into the core-matrix
// tile at `tile` (K-major, no swizzle: core (token/8, row/8) at
// (token/8)*rows*16 + (row/8)*128, token row within it at (token%8)*16).
// u[j*P + p] are the raw projections x.W of table j, plane p; every value is multiplied
// by `factor` (0 for tokens past the end) before its bf16 rounding.
template <int P>
__device__ __forceinline__ void write_phi_rows(uint32_t tile, int t, int rows, int tables,
                                               const float* u, float scale, float factor) {
  constexpr int R = 1 << P;
  constexpr int NHI = R / 8;
  const uint32_t base = tile + (t >> 3) * (rows * 16) + (t & 7) * 16;
  for (int j = 0; j < tables; ++j) {
    float sp[P], sm[P];
#pragma unroll
    for (int p = 0; p < P; ++p) logistic_fast(u[j * P + p] * scale, sp[p], sm[p]);
    float lo[8];
#pragma unroll
    for (int b = 0; b < 8; ++b)
      lo[b] = ((b & 1) ? sp[0] : sm[0]) * ((b & 2) ? sp[1] : sm[1]) * ((b & 4) ? sp[2] : sm[2]);
    float hi[NHI];
    hi[0] = factor;
    kron_tree<3, P>(hi, sp, sm);
#pragma unroll
    for (int c = 0; c < NHI; ++c) {
      const uint32_t addr = base + (uint32_t)((j * R) / 8 + c) * 128;
      st_shared_v4(addr, pack_bf16(hi[c] * lo[0], hi[c] * lo[1]),
                   pack_bf16(hi[c] * lo[2], hi[c] * lo[3]),
                   pack_bf16(hi[c] * lo[4], hi[c] * lo[5]),
                   pack_bf16(hi[c] * lo[6], hi[c] * lo[7]));
    }
  }
}

// 1/max(|x|, eps) of token row t of a 128-byte-swizzled 128 x 64 bf16 tile (the
// chunk order inside a row does not matter for a sum of squares).  Thread t starts at
// chunk t % 8, so eight consecutive rows (128 bytes apart) read eight different banks
// groups in each step.
__device__ __forceinline__ float row_inv_norm(const uint8_t* tile, int t) {
  const uint4* row = reinterpret_cast<const uint4*>(tile + t * 128);
  float s[4] = {0.f, 0.f, 0.f, 0.f};   // four independent sums: short dependency chains
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 w = row[c ^ (t & 7)];
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&ws[e]);
      float2 f = __bfloat1622float2(b2);
      s[e] = fmaf(f.x, f.x, fmaf(f.y, f.y, s[e]));
    }
  }
  return 1.0f / fmaxf(sqrtf((s[0] + s[1]) + (s[2] + s[3])), kEpsNorm);
}

// bf16 copy of one 80-column state row into the readout B operand (MN-major, no
// swizzle: core (row/8, col/8) at (row/8)*1280 + (col/8)*128, row within at (row%8)*16).
__device__ __forceinline__ void store_state_row_bf16(uint32_t sbf, int row, const float* v) {
  const uint32_t base = sbf + (row >> 3) * 1280 + (row & 7) * 16;
#pragma unroll
  for (int nc = 0; nc < 10; ++nc)
    st_shared_v4(base + nc * 128, pack_bf16(v[nc * 8 + 0], v[nc * 8 + 1]),
                 pack_bf16(v[nc * 8 + 2], v[nc * 8 + 3]),
                 pack_bf16(v[nc * 8 + 4], v[nc * 8 + 5]),
                 pack_bf16(v[nc * 8 + 6], v[nc * 8 + 7]));
}

// 80 consecutive columns of this thread's lane: five loads in flight, one wait.
__device__ __forceinline__ void tmem_ld80(uint32_t taddr, float* v) {
  uint32_t r[80];
#pragma unroll
  for (int b = 0; b < 5; ++b) tmem_ld16(taddr + b * 16, r + b * 16);
  tmem_ld_wait();
#pragma unroll
  for (int e = 0; e < 80; ++e) v[e] = __uint_as_float(r[e]);
}

// --------------------------------------------------------------------------- kernel
template <int P, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    k_sketch(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
             const __grid_constant__ CUtensorMap tv, const float* __restrict__ W,
             const float* __restrict__ init, float* __restrict__ seg_out,
             float* __restrict__ num, const float* __restrict__ kscale, Params prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Smem::bars);
  uint64_t* bar_tma = bars + 0;
  uint64_t* bar_proj = bars + 1;
  uint64_t* bar_phi = bars + 2;
  uint64_t* bar_qk = bars + 3;
  uint64_t* bar_intra = bars + 4;
  uint64_t* bar_mma = bars + 5;
  uint64_t* bar_free = bars + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 7);
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, rg = blockIdx.y, h = blockIdx.z;
  const int rows = prm.rows, tables = prm.tables, np = prm.np;
  const int mtiles = rows / 128;
  const int64_t s0 = (int64_t)g * prm.seg_len;
  const int64_t s1 = min64(prm.N, s0 + prm.seg_len);
  const int nchunks = (int)((s1 - s0 + kC - 1) / kC);
  const int l0 = rg * tables;
  W += (size_t)h * prm.w_hs;   // this head's hash planes

  if (threadIdx.x == 0) {
    for (int i = 0; i < 7; ++i) mbar_init(bars + i, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }

  // ---- setup by the CUDA-core warps: projection operands, ones, initial state
  if (threadIdx.x < kAlu) {
    const int t = threadIdx.x;
    for (int e = t; e < 64 * np; e += kAlu) {
      const int n = e / 64, kd = e % 64;
      float w = 0.f;
      if (n < tables * P) w = W[((size_t)(l0 + n / P) * 64 + kd) * P + (n % P)];
      const __nv_bfloat16 hi = __float2bfloat16_rn(w);
      const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
      const uint32_t off = (n >> 3) * 1024 + (kd >> 3) * 128 + (n & 7) * 16 + (kd & 7) * 2;
      *reinterpret_cast<__nv_bfloat16*>(sm + Smem::whi + off) = hi;
      *reinterpret_cast<__nv_bfloat16*>(sm + Smem::wlo + off) = lo;
    }
    for (int e = t; e < 256; e += kAlu)
      reinterpret_cast<__nv_bfloat16*>(sm + Smem::ones)[e] = __float2bfloat16_rn(1.0f);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const float* init_cta =
      init + (((size_t)h * prm.n_rg + rg) * prm.G + g) * (size_t)rows * kNV;
  if (threadIdx.x < kAlu) {
    const int t = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    if (MODE != kReadout) {
      for (int mt = 0; mt < mtiles; ++mt) {
        float vals[kNV];
#pragma unroll
        for (int c = 0; c < kNV; ++c)
          vals[c] = prm.have_init ? init_cta[(size_t)(mt * 128 + t) * kNV + c] : 0.f;
        uint32_t r[16];
#pragma unroll
        for (int b = 0; b < 5; ++b) {
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(vals[b * 16 + e]);
          tmem_st16(tmem + lane_off + (mt ? Tm::S1 : Tm::S0) + b * 16, r);
        }
        if (MODE == kSweep) store_state_row_bf16(sb + Smem::sbf, mt * 128 + t, vals);
      }
      tmem_st_wait();
    } else {
      for (int row = t; row < rows; row += kAlu) {
        float vals[kNV];
#pragma unroll
        for (int c = 0; c < kNV; ++c) vals[c] = init_cta[(size_t)row * kNV + c];
        store_state_row_bf16(sb + Smem::sbf, row, vals);
      }
    }
    fence_proxy_async();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 4) {
    // ================================================================ issuer
    if (lane == 0) {
      prefetch_tmap(&tq);
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
      const uint32_t id_proj = idesc_bf16(128, np, 0, 0);
      const uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
      const uint32_t id_read = idesc_bf16(128, kNV, 0, 1);
      const uint32_t id_av = idesc_bf16(128, 64, 0, 1);
      const uint32_t id_av1 = idesc_bf16(128, 16, 0, 1);
      const uint32_t id_up = idesc_bf16(128, 64, 1, 1);
      const uint32_t id_up1 = idesc_bf16(128, 16, 1, 1);
      const uint64_t d_ones = sdesc(sb + Smem::ones, 256, 128, kSwizzleNone);
      for (int i = 0; i < nchunks; ++i) {
        const int t0 = (int)(s0 + (int64_t)i * kC);
        uint32_t bytes = 0;
        if (MODE != kBuild) bytes += 16384;
        if (MODE != kReadout) bytes += 32768;
        mbar_arrive_expect_tx(bar_tma, bytes);
        if (MODE != kBuild) tma_load_3d(sm + Smem::q, &tq, 0, t0, h, bar_tma);
        if (MODE != kReadout) {
          tma_load_3d(sm + Smem::k, &tk, 0, t0, h, bar_tma);
          tma_load_3d(sm + Smem::v, &tv, 0, t0, h, bar_tma);
        }
        if (!mbar_wait(bar_tma, i & 1)) { s_abort = 1; break; }
        tc_fence_after();
        // projections u = x (W_hi + W_lo)
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t bh = sdesc(sb + Smem::whi + s * 256, 128, 1024, kSwizzleNone);
          const uint64_t bl = sdesc(sb + Smem::wlo + s * 256, 128, 1024, kSwizzleNone);
          if (MODE != kBuild) {
            const uint64_t a = sdesc(sb + Smem::q + s * 32, 16, 1024, kSwizzle128B);
            umma_ss(tmem + Tm::pq, a, bh, id_proj, s > 0);
            umma_ss(tmem + Tm::pq, a, bl, id_proj, 1);
          }
          if (MODE != kReadout) {
            const uint64_t a = sdesc(sb + Smem::k + s * 32, 16, 1024, kSwizzle128B);
            umma_ss(tmem + Tm::pk, a, bh, id_proj, s > 0);
            umma_ss(tmem + Tm::pk, a, bl, id_proj, 1);
          }
        }
        umma_commit(bar_proj);
        if (!mbar_wait(bar_phi, i & 1)) { s_abort = 1; break; }
        tc_fence_after();
        const int ksteps = rows / 16;
        if (MODE == kSweep) {
          for (int s = 0; s < ksteps; ++s)
            umma_ss(tmem + Tm::qk, sdesc(sb + Smem::phq + s * 256, 128, rows * 16, kSwizzleNone),
                    sdesc(sb + Smem::phk + s * 256, 128, rows * 16, kSwizzleNone), id_qk, s > 0);
          umma_commit(bar_qk);
          if (!mbar_wait(bar_intra, i & 1)) { s_abort = 1; break; }
          tc_fence_after();
        }
        if (MODE != kBuild) {
          for (int s = 0; s < ksteps; ++s)
            umma_ss(tmem + Tm::num, sdesc(sb + Smem::phq + s * 256, 128, rows * 16, kSwizzleNone),
                    sdesc(sb + Smem::sbf + s * 2560, 1280, 128, kSwizzleNone), id_read, s > 0);
        }
        if (MODE == kSweep) {
          for (int s = 0; s < kC / 16; ++s) {
            const uint64_t bv = sdesc(sb + Smem::v + s * 2048, 8192, 1024, kSwizzle128B);
            umma_ts(tmem + Tm::num, tmem + Tm::intra + s * 8, bv, id_av, 1);
            umma_ts(tmem + Tm::num + 64, tmem + Tm::intra + s * 8, d_ones, id_av1, 1);
          }
        }
        if (MODE != kReadout) {
          for (int mt = 0; mt < mtiles; ++mt) {
            const uint32_t dS = tmem + (mt ? Tm::S1 : Tm::S0);
            for (int s = 0; s < kC / 16; ++s) {
              const uint64_t a = sdesc(sb + Smem::phk + mt * 2048 + s * 32 * rows, rows * 16,
                                       128, kSwizzleNone);
              const uint64_t bv = sdesc(sb + Smem::v + s * 2048, 8192, 1024, kSwizzle128B);
              umma_ss(dS, a, bv, id_up, 1);
              umma_ss(dS + 64, a, d_ones, id_up1, 1);
            }
          }
        }
        umma_commit(bar_mma);
        if (!mbar_wait(bar_free, i & 1)) { s_abort = 1; break; }
      }
    }
  } else {
    // ================================================================ CUDA-core warps
    const int t = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float* num_h = num + (size_t)h * prm.N * kNumStride;
    for (int i = 0; i < nchunks; ++i) {
      if (s_abort) break;
      const int64_t t0 = s0 + (int64_t)i * kC;
      const bool valid = (t0 + t) < s1;
      if (!mbar_wait(bar_proj, i & 1)) { s_abort = 1; break; }
      tc_fence_after();
      float u[32];
      uint32_t r[16];
      if (MODE != kBuild) {
        const float sc = row_inv_norm(sm + Smem::q, t) * prm.two_over_tau;
        for (int b = 0; b < np / 16; ++b) {
          tmem_ld16(tmem + lane_off + Tm::pq + b * 16, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) u[b * 16 + e] = __uint_as_float(r[e]);
        }
        write_phi_rows<P>(sb + Smem::phq, t, rows, tables, u, sc, valid ? 1.f : 0.f);
      }
      if (MODE != kReadout) {
        const float sc = row_inv_norm(sm + Smem::k, t) * prm.two_over_tau;
        for (int b = 0; b < np / 16; ++b) {
          tmem_ld16(tmem + lane_off + Tm::pk + b * 16, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) u[b * 16 + e] = __uint_as_float(r[e]);
        }
        const float kf =
            valid ? (kscale ? kscale[(size_t)h * prm.N + t0 + t] : 1.f) : 0.f;
        write_phi_rows<P>(sb + Smem::phk, t, rows, tables, u, sc, kf);
      }
      fence_proxy_async();
      tc_fence_before();
      named_bar(1, kAlu);
      if (t == 0) mbar_arrive(bar_phi);

      if (MODE == kSweep) {
        if (!mbar_wait(bar_qk, i & 1)) { s_abort = 1; break; }
        tc_fence_after();
        for (int cb = 0; cb < kC / 16; ++cb) {
          tmem_ld16(tmem + lane_off + Tm::qk + cb * 16, r);
          tmem_ld_wait();
          uint32_t pk8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j0 = cb * 16 + 2 * e;
            const float a0 = (j0 <= t) ? __uint_as_float(r[2 * e]) : 0.f;
            const float a1 = (j0 + 1 <= t) ? __uint_as_float(r[2 * e + 1]) : 0.f;
            pk8[e] = pack_bf16(a0, a1);
          }
          tmem_st8(tmem + lane_off + Tm::intra + cb * 8, pk8);
        }
        tmem_st_wait();
        tc_fence_before();
        named_bar(1, kAlu);
        if (t == 0) mbar_arrive(bar_intra);
      }

      if (!mbar_wait(bar_mma, i & 1)) { s_abort = 1; break; }
      tc_fence_after();
      if (MODE != kBuild) {
        float acc[kNV];
        tmem_ld80(tmem + lane_off + Tm::num, acc);   // warp-collective: every lane loads
        if (valid) {
          float* dst = num_h + (t0 + t) * kNumStride;
#pragma unroll
          for (int c = 0; c < 64; c += 4)
            red_add_v4(dst + c, acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
          atomicAdd(dst + 64, acc[64]);
        }
      }
      if (MODE == kSweep) {
        for (int mt = 0; mt < mtiles; ++mt) {
          float vals[kNV];
          tmem_ld80(tmem + lane_off + (mt ? Tm::S1 : Tm::S0), vals);
          store_state_row_bf16(sb + Smem::sbf, mt * 128 + t, vals);
        }
        fence_proxy_async();
      }
      tc_fence_before();
      named_bar(1, kAlu);
      if (t == 0) mbar_arrive(bar_free);
    }
    if (MODE == kBuild && !s_abort) {
      float* out = seg_out + (((size_t)h * prm.n_rg + rg) * prm.G + g) * (size_t)rows * kNV;
      for (int mt = 0; mt < mtiles; ++mt) {
        float vals[kNV];
        tmem_ld80(tmem + lane_off + (mt ? Tm::S1 : Tm::S0), vals);
        float4* o4 = reinterpret_cast<float4*>(out + (size_t)(mt * 128 + t) * kNV);
#pragma unroll
        for (int c = 0; c < kNV / 4; ++c)
          o4[c] = make_float4(vals[4 * c], vals[4 * c + 1], vals[4 * c + 2], vals[4 * c + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// =========================================================================== host
struct Plan {
  Params prm;
  int P;
  size_t off_num, off_seg, off_init, off_inv, bytes;
  int64_t inv_stride;
};

inline bool supported(const race_args_t* a) {
  if (a->d != kD || a->dtype != RACE_BF16) return false;
  if (a->P < 6 || a->P > 8) return false;
  const int64_t LR = (int64_t)a->L << a->P;
  if (LR % 128 != 0) return false;
  if (a->N > (int64_t)INT32_MAX - kC) return false;
  return true;
}

inline Plan make_plan(const race_args_t* a) {
  Plan pl;
  Params& p = pl.prm;
  pl.P = a->P;
  p.N = a->N;
  p.H = a->H;
  p.L = a->L;
  p.R = 1 << a->P;
  const int LR = a->L * p.R;
  p.rows = (LR % 256 == 0) ? 256 : 128;   // divides L*R; a multiple of R (R <= 256)
  p.tables = p.rows / p.R;
  p.np = ((p.tables * a->P + 15) / 16) * 16;
  p.n_rg = LR / p.rows;
  const int64_t units = (int64_t)a->H * p.n_rg;
  const int64_t tiles = (a->N + kC - 1) / kC;
  int64_t G;
  if (a->causal)
    G = std::max<int64_t>(1, 148 / units);
  else
    G = std::max<int64_t>(1, (4 * 148 + units - 1) / units);
  G = std::min<int64_t>(G, tiles);
  const int64_t seg_tiles = (tiles + G - 1) / G;
  p.seg_len = seg_tiles * kC;
  p.G = (int)((a->N + p.seg_len - 1) / p.seg_len);
  p.two_over_tau = 2.0f / a->tau;
  p.have_init = 0;
  p.lps = 0;
  p.w_hs = a->w_per_head ? (int64_t)a->L * kD * a->P : 0;
  const size_t st = (size_t)a->H * p.n_rg * p.G * p.rows * kNV * sizeof(float);
  size_t o = 0;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  pl.off_num = o;  o = al(o + (size_t)a->H * a->N * kNumStride * sizeof(float));
  pl.off_seg = o;  o = al(o + st);
  pl.off_init = o; o = al(o + st);
  pl.inv_stride = ((a->N + kC - 1) / kC) * kC;  // per-head row stride: whole chunks
  pl.off_inv = o;  o = al(o + 2 * (size_t)a->H * pl.inv_stride * sizeof(float));
  pl.bytes = o;
  return pl;
}

inline size_t forward_workspace(const race_args_t* a) { return make_plan(a).bytes; }

// cuTensorMapEncodeTiled through the runtime's driver entry-point query, looked up once
// (a function-local static: initialised thread-safely, never modified afterwards).
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

inline bool encode_tmap(CUtensorMap* m, const void* base, int64_t N, int H) {
  const auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)N, (cuuint64_t)H};
  cuuint64_t strides[2] = {128, (cuuint64_t)N * 128};
  cuuint32_t box[3] = {64, (cuuint32_t)kC, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D view [H][N][68] of the float32 output accumulators for TMA reductions: boxes of
// 64 rows x 68 columns, rows beyond N of a head are dropped.
inline bool encode_num_tmap(CUtensorMap* m, void* base, int64_t N, int H) {
  const auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kNumStride, (cuuint64_t)N, (cuuint64_t)H};
  cuuint64_t strides[2] = {(cuuint64_t)kNumStride * 4, (cuuint64_t)N * kNumStride * 4};
  cuuint32_t box[3] = {(cuuint32_t)kNumStride, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace race

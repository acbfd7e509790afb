// Tensor-core (tcgen05) backward of RACE attention for row groups of 256 sketch rows
// (one table at R = 256, 256/R tables below).
//
// Notation (kernel units: p = unscaled corner probabilities, den' = L * den):
//   g'_i  = [g_i , -(g_i . o_i)]                          (80 wide: g_i is the upstream
//                                                          gradient exactly as given, the
//                                                          last entry a bf16 hi + lo pair)
//   r_i   = 1 / den'_i                                    (float32)
//   dw_ij = r_i g'_i . [v_j ; 1]                          (gradient of the weight w_ij)
//   dP(q_i) = sum_{j <= i} dw_ij p(k_j) = r_i S_i g'_i     S_i = sum_{j <= i} p(k_j)[v_j;1]^T
//   dP(k_j) = sum_{i >= j} dw_ij p(q_i) = T_j [v_j ; 1]    T_j = sum_{i >= j} r_i p(q_i) g'_i^T
// The per-row factor r_i is never applied to g (a bf16 rounding of g / den' would cost
// up to 2^-8, the bf16 unit roundoff, of every gradient entry): on the q side it scales
// the per-plane gradients in float32, on the k side it scales p(q_i) before its own
// bf16 rounding.
// Both sides are the same computation with the roles exchanged and the sweep reversed:
// a side "a" whose corner gradients are wanted, with 80-wide features X, and a side "b"
// with features Y whose p(b), times an optional row factor rb, builds the state:
//   dP_a = ra (X S^T + mask(X Y^T) p~(b)),   S += p~(b)^T Y,   p~(b) = rb p(b)
//   q pass: a = q, X = g', ra = r, b = k, Y = [v | 1]; forward order, keys j <= i
//   k pass: a = k, X = [v | 1], b = q, Y = g', rb = r; reverse order, queries i >= j
// The soft hash backward then gives, per table and plane ([JA] §2.1 soft
// bucketization; the softmax over corners factorises into logistic pairs),
//   du_p = (2/tau) (sum_{b: bit p of b set} p_b dP_b - s_p sum_b p_b dP_b),
//   s_p = sigma(2 u_p / tau),
// written per token to du[h][n][L*P]; the projection transposes and the
// normalisation Jacobian run in k_bwd_finalize.
//
// One CTA sweeps one segment of one row group of one head: TMA loads the x tiles
// (128B swizzle) and the feature tiles (32-byte swizzle, 4 boxes of 16 columns plus a
// fifth atom holding the extra column); tcgen05 computes the projections, X Y^T, the
// corner gradients (two halves of 128 rows) and the state update; the CUDA-core warps
// expand p(b), mask and round X Y^T, run the hash backward and keep the bf16 copy of S.
#pragma once

#include "tc_kernels.cuh"

namespace race {
namespace tc {

constexpr int kBwThreads = 160;  // warps 0-3: CUDA-core work (TMEM lane = token row); warp 4: issuer

struct BwSmem {
  static constexpr uint32_t xa = 0;        // 128 x 64 bf16, 128B swizzle (TMA)
  static constexpr uint32_t xb = 16384;
  static constexpr uint32_t fa = 32768;    // 5 atoms of 128 rows x 32 B, 32B swizzle
  static constexpr uint32_t fb = 53248;
  static constexpr uint32_t phb = 73728;   // p(b): 128 tokens x 256 rows, core-matrix layout
  static constexpr uint32_t sbf = 139264;  // state as bf16 hi, 256 x 80, core-matrix layout
  static constexpr uint32_t sbl = 180224;  // and the bf16 rest (S - hi)
  static constexpr uint32_t whi = 221184;  // projection operand, up to 32 x 64 bf16
  static constexpr uint32_t wlo = 225280;
  static constexpr uint32_t bars = 229376;
  static constexpr uint32_t total = bars + 16 * 8;
  static constexpr uint32_t alloc = total + 1024;
};
static_assert(BwSmem::alloc <= 232448, "shared memory budget of one CTA");

// Tensor-memory columns.  dw (float32, 128 keys) is rounded in place to the bf16 A
// operand intra (64 columns).
struct BwTm {
  static constexpr uint32_t S0 = 0, S1 = 80, dp = 160, dw = 288, intra = 288, pa = 416,
                            pb = 448;
};

enum BwBar : int {
  kbTMAX = 0, kbTMAF, kbPROJ, kbPHI, kbDW, kbINTRA, kbDP, kbDPFREE, kbUP, kbCOUNT
};

// Extra feature columns of token row t in atom 4 of a 32B-swizzled feature tile.  The
// 16 columns 64..79 are [e_hi, e_lo, 0, ...] with e = e_hi + e_lo split into two bf16
// values on the g'' side, and [1, 1, 0, ...] on the [v | 1] side, so that their product
// keeps -(g . o)/den' to about 16 bits: it nearly cancels g . v / den' in dw_ij.  Zero
// for tokens past the end.  The two 16-byte halves of a 32-byte row are swapped on rows
// 4-7 of each 8-row group.
// x: the extra value of the token on the g'' side (loaded ahead by the caller); ones:
// the [v | 1] side.
__device__ __forceinline__ void store_extra_cols(uint32_t tile, int t, float x, bool ones,
                                                 bool valid) {
  float c0 = 0.f, c1 = 0.f;
  if (valid) {
    if (!ones) {
      c0 = __bfloat162float(__float2bfloat16_rn(x));
      c1 = x - c0;
    } else {
      c0 = c1 = 1.f;
    }
  }
  const uint32_t row = tile + 4 * 4096 + t * 32;
  const uint32_t first = ((t >> 2) & 1) << 4;
  st_shared_v4(row + first, pack_bf16(c0, c1), 0u, 0u, 0u);
  st_shared_v4(row + (first ^ 16), 0u, 0u, 0u, 0u);
}

// State row r as bf16 hi and bf16 lo = row - hi (X S^T adds both: the products with
// g'' cancel to a small fraction of the state's size, so one bf16 rounding is too coarse).
// Each pair is rounded once (one packed conversion); hi is widened back exactly by bit
// moves, and lo = v - hi is exact in float32 before its own rounding.
__device__ __forceinline__ void store_state_row_split(uint32_t hi_base, uint32_t lo_base, int r,
                                                      const float* v) {
  const uint32_t hb = hi_base + (r >> 3) * 1280 + (r & 7) * 16;
  const uint32_t lb = lo_base + (r >> 3) * 1280 + (r & 7) * 16;
#pragma unroll
  for (int nc = 0; nc < 10; ++nc) {
    uint32_t hp[4], lp[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = v[nc * 8 + 2 * e], b = v[nc * 8 + 2 * e + 1];
      hp[e] = pack_bf16(a, b);
      lp[e] = pack_bf16(a - __uint_as_float(hp[e] << 16), b - __uint_as_float(hp[e] & 0xffff0000u));
    }
    st_shared_v4(hb + nc * 128, hp[0], hp[1], hp[2], hp[3]);
    st_shared_v4(lb + nc * 128, lp[0], lp[1], lp[2], lp[3]);
  }
}

// Hash-backward partial sums of one token over the 128 sketch rows of half HALF.
// dp[r] = dP of row HALF*128 + r; lo/hi: corner factors of every table of the row group
// (table j: lo[8j..8j+7], hi[(R/8)j ..]); Ts[j] = sum_b p_b dP_b, As[j*P + p] = sum over
// corners with bit p set.
// write_phi_rows for 256 sketch rows with the loop over groups of four high corners kept
// rolled (a smaller instruction footprint for the sweep's CUDA-core warps): corner
// c = 4g + jj has high factor p34[jj] (planes 3-4) times the product over planes 5.. chosen
// by the bits of g.  Every value is multiplied by `factor` (0 for tokens past the end)
// before its bf16 rounding.
template <int P, int TABLES>
__device__ __forceinline__ void write_phi_rows_rolled(uint32_t tile, int t, const float* u,
                                                      float scale, float factor) {
  constexpr int R = 1 << P;
  constexpr int NG = R / 32;
  const uint32_t base = tile + (t >> 3) * (256 * 16) + (t & 7) * 16;
#pragma unroll
  for (int j = 0; j < TABLES; ++j) {
    float sp[P], sm[P];
#pragma unroll
    for (int p = 0; p < P; ++p) logistic_fast(u[j * P + p] * scale, sp[p], sm[p]);
    float lo[8], p34[4];
#pragma unroll
    for (int b = 0; b < 8; ++b)
      lo[b] = ((b & 1) ? sp[0] : sm[0]) * ((b & 2) ? sp[1] : sm[1]) * ((b & 4) ? sp[2] : sm[2]);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
      p34[jj] = factor * ((jj & 1) ? sp[3] : sm[3]) * ((jj & 2) ? sp[4] : sm[4]);
#pragma unroll 1
    for (int g = 0; g < NG; ++g) {
      float hg = 1.f;
#pragma unroll
      for (int p = 5; p < P; ++p) hg *= ((g >> (p - 5)) & 1) ? sp[p] : sm[p];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
        store_chunk(base + (uint32_t)((j * R) / 8 + 4 * g + jj) * 128, hg * p34[jj], lo);
    }
  }
}

template <int P, int HALF>
__device__ __forceinline__ void hash_bwd_half(const float* dp, const float* lo, const float* hi,
                                              float* Ts, float* As) {
  constexpr int R = 1 << P;
  constexpr int NHI = R / 8;
#pragma unroll
  for (int g8 = 0; g8 < 16; ++g8) {
    const int row0 = HALF * 128 + g8 * 8;
    const int j = row0 / R;              // table
    const int c = (row0 % R) / 8;        // high corner index within the table
    float m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = lo[8 * j + e] * dp[g8 * 8 + e];
    const float z = ((m[0] + m[1]) + (m[2] + m[3])) + ((m[4] + m[5]) + (m[6] + m[7]));
    const float hz = hi[NHI * j + c];
    Ts[j] = fmaf(hz, z, Ts[j]);
    As[j * P + 0] = fmaf(hz, (m[1] + m[3]) + (m[5] + m[7]), As[j * P + 0]);
    As[j * P + 1] = fmaf(hz, (m[2] + m[3]) + (m[6] + m[7]), As[j * P + 1]);
    As[j * P + 2] = fmaf(hz, (m[4] + m[5]) + (m[6] + m[7]), As[j * P + 2]);
    const float w = hz * z;
#pragma unroll
    for (int p = 3; p < P; ++p)
      if ((c >> (p - 3)) & 1) As[j * P + p] += w;
  }
}

template <int P, int MODE, bool REV>
__global__ void __launch_bounds__(kBwThreads, 1)
    k_bwd_phi(const __grid_constant__ CUtensorMap txa, const __grid_constant__ CUtensorMap txb,
              const __grid_constant__ CUtensorMap tfa, const __grid_constant__ CUtensorMap tfb,
              const float* __restrict__ ea, const float* __restrict__ eb,
              const float* __restrict__ ra, const float* __restrict__ rb,
              const float* __restrict__ W, const float* __restrict__ init,
              float* __restrict__ seg_out, __nv_bfloat16* __restrict__ du_out, Params prm) {
  constexpr bool HAS_A = MODE != kBuild;      // corner gradients of side a
  constexpr bool HAS_B = MODE != kReadout;    // state built from side b
  constexpr bool CAUSAL = MODE == kSweep;
  constexpr int R = 1 << P;
  constexpr int TABLES = 256 / R;
  constexpr int NP = ((TABLES * P + 15) / 16) * 16;
  static_assert((TABLES * P) % 2 == 0, "per-plane gradients are stored as bf16 pairs");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + BwSmem::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + kbCOUNT);
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, rg = blockIdx.y, h = blockIdx.z;
  const int64_t s0 = (int64_t)g * prm.seg_len;
  const int64_t s1 = min64(prm.N, s0 + prm.seg_len);
  const int nchunks = (int)((s1 - s0 + kC - 1) / kC);
  const int l0 = rg * TABLES;
  W += (size_t)h * prm.w_hs;   // this head's hash planes

  if (threadIdx.x == 0) {
    for (int i = 0; i < kbCOUNT; ++i) mbar_init(bar + i, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (threadIdx.x < kAlu) {
    // projection operand [K = 64 dims][N = NP], W split into bf16 hi + lo
    for (int e = threadIdx.x; e < 64 * NP; e += kAlu) {
      const int n = e / 64, kd = e % 64;
      float w = 0.f;
      if (n < TABLES * P) w = W[((size_t)(l0 + n / P) * 64 + kd) * P + (n % P)];
      const __nv_bfloat16 hi = __float2bfloat16_rn(w);
      const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
      const uint32_t off = (n >> 3) * 1024 + (kd >> 3) * 128 + (n & 7) * 16 + (kd & 7) * 2;
      *reinterpret_cast<__nv_bfloat16*>(sm + BwSmem::whi + off) = hi;
      *reinterpret_cast<__nv_bfloat16*>(sm + BwSmem::wlo + off) = lo;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- initial state: TMEM accumulators (HAS_B) and/or the bf16 copy (HAS_A)
  const float* init_cta = init + (((size_t)h * prm.n_rg + rg) * prm.G + g) * (size_t)256 * kNV;
  if (threadIdx.x < kAlu) {
    const int t = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    for (int mt = 0; mt < 2; ++mt) {
      float vals[kNV];
#pragma unroll
      for (int c = 0; c < kNV; ++c)
        vals[c] = prm.have_init ? init_cta[(size_t)(mt * 128 + t) * kNV + c] : 0.f;
      if (HAS_B) {
        uint32_t r[16];
#pragma unroll
        for (int b = 0; b < 5; ++b) {
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(vals[b * 16 + e]);
          tmem_st16(tmem + lane_off + (mt ? BwTm::S1 : BwTm::S0) + b * 16, r);
        }
      }
      if (HAS_A) store_state_row_split(sb + BwSmem::sbf, sb + BwSmem::sbl, mt * 128 + t, vals);
    }
    if (HAS_B) tmem_st_wait();
    fence_proxy_async();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 4) {
    // ================================================================ issuer
    // The whole warp runs the loop (waits included, with a warp-uniform outcome); TMA
    // copies, MMAs and commits are issued by one elected lane (the same one every time).
    if (elect_one()) {
      if (HAS_A) { prefetch_tmap(&txa); prefetch_tmap(&tfa); }
      if (HAS_B) { prefetch_tmap(&txb); prefetch_tmap(&tfb); }
    }
    __syncwarp();
    const uint32_t id_proj = idesc_bf16(128, NP, 0, 0);
    const uint32_t id_128 = idesc_bf16(128, 128, 0, 0);   // X Y^T and X S^T
    const uint32_t id_d3 = idesc_bf16(128, 128, 0, 1);    // A tmem, B MN-major
    const uint32_t id_up = idesc_bf16(128, kNV, 1, 1);    // A, B MN-major
    bool ok = true;
    auto wait = [&](int b, uint32_t par) {
      if (ok && !mbar_wait(bar + b, par)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      if (!ok && lane == 0) s_abort = 1;
      return ok;
    };
    // x tiles of sweep step i (read by PROJ(i) and by the CUDA-core warps' 1/|x| before
    // PHI(i)) and feature tiles (read by the MMAs of step i up to UPD(i)); one elected lane
    auto step_t0 = [&](int i) { return (int)(s0 + (int64_t)(REV ? nchunks - 1 - i : i) * kC); };
    auto load_x = [&](int i) {
      const int t0 = step_t0(i);
      mbar_arrive_expect_tx(bar + kbTMAX, (HAS_A ? 16384u : 0u) + (HAS_B ? 16384u : 0u));
      if (HAS_A) tma_load_3d(sm + BwSmem::xa, &txa, 0, t0, h, bar + kbTMAX);
      if (HAS_B) tma_load_3d(sm + BwSmem::xb, &txb, 0, t0, h, bar + kbTMAX);
    };
    auto load_f = [&](int i) {
      const int t0 = step_t0(i);
      mbar_arrive_expect_tx(bar + kbTMAF, (HAS_A ? 16384u : 0u) + (HAS_B ? 16384u : 0u));
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        if (HAS_A) tma_load_3d(sm + BwSmem::fa + a * 4096, &tfa, a * 16, t0, h, bar + kbTMAF);
        if (HAS_B) tma_load_3d(sm + BwSmem::fb + a * 4096, &tfb, a * 16, t0, h, bar + kbTMAF);
      }
    };
    // projections of the step whose x tiles are in shared memory
    auto proj = [&]() {
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t bh = sdesc(sb + BwSmem::whi + s * 256, 128, 1024, kSwizzleNone);
          const uint64_t bl = sdesc(sb + BwSmem::wlo + s * 256, 128, 1024, kSwizzleNone);
          if (HAS_A) {
            const uint64_t a = sdesc(sb + BwSmem::xa + s * 32, 16, 1024, kSwizzle128B);
            umma_ss(tmem + BwTm::pa, a, bh, id_proj, s > 0);
            umma_ss(tmem + BwTm::pa, a, bl, id_proj, 1);
          }
          if (HAS_B) {
            const uint64_t a = sdesc(sb + BwSmem::xb + s * 32, 16, 1024, kSwizzle128B);
            umma_ss(tmem + BwTm::pb, a, bh, id_proj, s > 0);
            umma_ss(tmem + BwTm::pb, a, bl, id_proj, 1);
          }
        }
        umma_commit(bar + kbPROJ);
      }
      __syncwarp();
    };
    if (nchunks > 0) {
      if (elect_one()) {
        load_x(0);
        load_f(0);
      }
      __syncwarp();
      if (wait(kbTMAX, 0)) proj();
    }
    // Step i in tensor-core order: X Y^T, UPD (while the CUDA-core warps mask X Y^T),
    // dP half 0, dP half 1, PROJ(i+1).  The x tiles of step i+1 are loaded once the
    // warps have read the projections and x tiles of step i (PHI); PROJ(i+1) follows
    // every MMA of step i, and its completion frees the feature tiles for step i+1.
    for (int i = 0; i < nchunks && ok; ++i) {
      BW_TRACE(i, 0);
      if (!wait(kbPHI, i & 1)) break;
      BW_TRACE(i, 2);
      if (i + 1 < nchunks && elect_one()) load_x(i + 1);
      __syncwarp();
      if (!wait(kbTMAF, i & 1)) break;
      BW_TRACE(i, 1);
      tc_fence_after();
      if (CAUSAL) {
        // X Y^T: rows of side a x tokens of side b, K = 80 feature columns
        if (elect_one()) {
#pragma unroll
          for (int s = 0; s < 5; ++s)
            umma_ss(tmem + BwTm::dw, sdesc(sb + BwSmem::fa + s * 4096, 16, 256, kSwizzle32B),
                    sdesc(sb + BwSmem::fb + s * 4096, 16, 256, kSwizzle32B), id_128, s > 0);
          umma_commit(bar + kbDW);
        }
        __syncwarp();
      }
      if (HAS_B) {
        // S += p(b)^T Y, both halves of the sketch rows (K = 128 tokens); it runs while
        // the CUDA-core warps mask X Y^T.  dP(i) reads the bf16 copy of the state before
        // step i, which the warps rewrite only after dP(i) (and this update) are done.
        tc_fence_after();
        if (elect_one()) {
          for (int half = 0; half < 2; ++half)
#pragma unroll
            for (int s = 0; s < 8; ++s)
              umma_ss(tmem + (half ? BwTm::S1 : BwTm::S0),
                      sdesc(sb + BwSmem::phb + half * 2048 + s * 8192, 4096, 128, kSwizzleNone),
                      sdesc(sb + BwSmem::fb + s * 512, 4096, 256, kSwizzle32B), id_up, 1);
          umma_commit(bar + kbUP);
        }
        __syncwarp();
      }
      if (CAUSAL) {
        if (!wait(kbINTRA, i & 1)) break;
        BW_TRACE(i, 3);
        tc_fence_after();
      }
      if (HAS_A) {
        for (int half = 0; half < 2 && ok; ++half) {
          if (elect_one()) {
            // X S^T over sketch rows half*128 .. +127 (K = 80)
#pragma unroll
            for (int s = 0; s < 5; ++s) {
              const uint64_t xd = sdesc(sb + BwSmem::fa + s * 4096, 16, 256, kSwizzle32B);
              umma_ss(tmem + BwTm::dp, xd,
                      sdesc(sb + BwSmem::sbf + half * 20480 + s * 256, 128, 1280, kSwizzleNone),
                      id_128, s > 0);
              umma_ss(tmem + BwTm::dp, xd,
                      sdesc(sb + BwSmem::sbl + half * 20480 + s * 256, 128, 1280, kSwizzleNone),
                      id_128, 1);
            }
            if (CAUSAL) {
              // + mask(X Y^T) p(b): K = 128 tokens of side b
#pragma unroll
              for (int s = 0; s < 8; ++s)
                umma_ts(tmem + BwTm::dp, tmem + BwTm::intra + s * 8,
                        sdesc(sb + BwSmem::phb + half * 2048 + s * 8192, 4096, 128, kSwizzleNone),
                        id_d3, 1);
            }
            umma_commit(bar + kbDP);
          }
          __syncwarp();
          // the second half overwrites dP once the warps have read the first; the next
          // step's first half comes after its PHI, i.e. after the warps read this one's
          // second half
          if (half == 0) {
            if (!wait(kbDPFREE, 0)) break;
            BW_TRACE(i, 4);
            tc_fence_after();
          }
        }
        if (!ok) break;
      }
      if (i + 1 < nchunks) {
        if (!wait(kbTMAX, (i + 1) & 1)) break;
        proj();
        BW_TRACE(i, 5);
        // PROJ(i+1) follows every MMA of step i, so its completion frees the feature
        // tiles of step i (the CUDA-core warps wait on the same barrier)
        if (!wait(kbPROJ, (i + 1) & 1)) break;
        BW_TRACE(i, 6);
        if (elect_one()) load_f(i + 1);
        __syncwarp();
      }
    }
  } else if (warp < 4) {
    // ================================================================ CUDA-core warps
    const int t = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    // the g' extra value of this thread's token, one step ahead (a global load); at most
    // one side is the g' side (ea or eb non-null), the other is [v | 1]
    const float* ex_src = HAS_A && ea ? ea : (HAS_B ? eb : nullptr);
    // the row factors of both sides, [H][N] float32 (null: 1)
    const float* ra_src = HAS_A ? ra : nullptr;
    const float* rb_src = HAS_B ? rb : nullptr;
    auto row_of = [&](int i) { return s0 + (int64_t)(REV ? nchunks - 1 - i : i) * kC + t; };
    auto load_ex = [&](int i) {
      const int64_t row = row_of(i);
      return (ex_src && row < s1) ? ex_src[(size_t)h * prm.N + row] : 0.f;
    };
    auto load_rf = [&](const float* src, int i) {
      const int64_t row = row_of(i);
      return row < s1 ? (src ? src[(size_t)h * prm.N + row] : 1.f) : 0.f;
    };
    float ex_next = nchunks > 0 ? load_ex(0) : 0.f;
    float ra_next = nchunks > 0 ? load_rf(ra_src, 0) : 0.f;
    float rb_next = nchunks > 0 ? load_rf(rb_src, 0) : 0.f;
    for (int i = 0; i < nchunks; ++i) {
      if (s_abort) break;
      const int c = REV ? nchunks - 1 - i : i;
      const int64_t t0 = s0 + (int64_t)c * kC;
      const bool valid = (t0 + t) < s1;
      const float ex = ex_next;
      const float fa = ra_next, fb = rb_next;   // row factors (0 past the end)
      if (i + 1 < nchunks) {
        ex_next = load_ex(i + 1);
        ra_next = load_rf(ra_src, i + 1);
        rb_next = load_rf(rb_src, i + 1);
      }
      if (!mbar_wait(bar + kbPROJ, i & 1)) { s_abort = 1; break; }
      if (t == 0) BW_TRACE(i, 10);
      tc_fence_after();
      float ua[NP], ub[NP];
      float inv_a = 0.f;
      {   // both sides' projections: all loads in flight, one wait
        uint32_t ra[NP], rb[NP];
#pragma unroll
        for (int b = 0; b < NP / 16; ++b) {
          if (HAS_A) tmem_ld16(tmem + lane_off + BwTm::pa + b * 16, ra + b * 16);
          if (HAS_B) tmem_ld16(tmem + lane_off + BwTm::pb + b * 16, rb + b * 16);
        }
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < NP; ++e) {
          ua[e] = HAS_A ? __uint_as_float(ra[e]) : 0.f;
          ub[e] = HAS_B ? __uint_as_float(rb[e]) : 0.f;
        }
      }
      if (HAS_A) {
        inv_a = row_inv_norm(sm + BwSmem::xa, t);
        store_extra_cols(sb + BwSmem::fa, t, ex, ea == nullptr, valid);
      }
      if (HAS_B) {
        const float sc = row_inv_norm(sm + BwSmem::xb, t) * prm.two_over_tau;
        write_phi_rows_rolled<P, TABLES>(sb + BwSmem::phb, t, ub, sc, fb);
        store_extra_cols(sb + BwSmem::fb, t, ex, eb == nullptr, valid);
      }
      fence_proxy_async();
      tc_fence_before();
      named_bar(1, kAlu);
      if (t == 0) mbar_arrive(bar + kbPHI);
      if (t == 0) BW_TRACE(i, 11);

      if (CAUSAL) {
        // mask X Y^T (b tokens j <= t, or j >= t in the reverse sweep), round to bf16
        if (!mbar_wait(bar + kbDW, i & 1)) { s_abort = 1; break; }
        if (t == 0) BW_TRACE(i, 12);
        tc_fence_after();
        // key blocks in pairs: blocks 0-1 (fp32 columns 0-63) are loaded, masked and
        // rounded, and their bf16 pairs land in columns 0-31, which held keys already
        // loaded; then blocks 2-3 (columns 64-127), whose pairs land in columns 32-63
#pragma unroll 1
        for (int kp = 0; kp < 2; ++kp) {
          uint32_t x[64], o[32];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            tmem_ld16(tmem + lane_off + BwTm::dw + kp * 64 + q * 16, x + q * 16);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int j0 = kp * 64 + 2 * e;
            const bool k0 = REV ? (j0 >= t) : (j0 <= t);
            const bool k1 = REV ? (j0 + 1 >= t) : (j0 + 1 <= t);
            o[e] = pack_bf16(k0 ? __uint_as_float(x[2 * e]) : 0.f,
                             k1 ? __uint_as_float(x[2 * e + 1]) : 0.f);
          }
          tmem_st16(tmem + lane_off + BwTm::intra + kp * 32, o);
          tmem_st16(tmem + lane_off + BwTm::intra + kp * 32 + 16, o + 16);
        }
        tmem_st_wait();
        tc_fence_before();
        named_bar(1, kAlu);
        if (t == 0) mbar_arrive(bar + kbINTRA);
        if (t == 0) BW_TRACE(i, 13);
      }

      if (HAS_A) {
        // ---- soft hash backward of side a
        float sp[TABLES * P], lo[TABLES * 8], hi[TABLES * (R / 8)];
        const float sc = inv_a * prm.two_over_tau;
#pragma unroll
        for (int j = 0; j < TABLES; ++j) {
          float spj[P], smj[P];
#pragma unroll
          for (int p = 0; p < P; ++p) {
            logistic_fast(ua[j * P + p] * sc, spj[p], smj[p]);
            sp[j * P + p] = spj[p];
          }
#pragma unroll
          for (int b = 0; b < 8; ++b)
            lo[8 * j + b] = ((b & 1) ? spj[0] : smj[0]) * ((b & 2) ? spj[1] : smj[1]) *
                            ((b & 4) ? spj[2] : smj[2]);
          float hj[R / 8];
          hj[0] = 1.f;
          kron_tree<3, P>(hj, spj, smj);
#pragma unroll
          for (int cc = 0; cc < R / 8; ++cc) hi[(R / 8) * j + cc] = hj[cc];
        }
        float Ts[TABLES], As[TABLES * P];
#pragma unroll
        for (int j = 0; j < TABLES; ++j) Ts[j] = 0.f;
#pragma unroll
        for (int e = 0; e < TABLES * P; ++e) As[e] = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!mbar_wait(bar + kbDP, half)) { s_abort = 1; break; }
          if (t == 0) BW_TRACE(i, 14 + 2 * half);
          tc_fence_after();
          float dp[128];
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            uint32_t x[64];
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) tmem_ld16(tmem + lane_off + BwTm::dp + hb * 64 + cb * 16, x + cb * 16);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 64; ++e) dp[hb * 64 + e] = __uint_as_float(x[e]);
          }
          tc_fence_before();
          named_bar(1, kAlu);
          if (t == 0) mbar_arrive(bar + kbDPFREE);
          if (t == 0) BW_TRACE(i, 15 + 2 * half);
          if (half == 0) hash_bwd_half<P, 0>(dp, lo, hi, Ts, As);
          else hash_bwd_half<P, 1>(dp, lo, hi, Ts, As);
        }
        if (s_abort) break;
        const size_t off = ((size_t)h * prm.N + t0 + t) * prm.lps + (size_t)l0 * P;
        if (valid && RACE_IN_RANGE(off + TABLES * P - 1, (int64_t)prm.H * prm.N * prm.lps)) {
          // du' = du / max(|x|, eps) as a bf16 hi + lo pair (about 16 significant bits):
          // the finalize then multiplies by W and by the unnormalised x tile directly
          __nv_bfloat16* dh = du_out + off;
          __nv_bfloat16* dl = du_out + (size_t)prm.H * prm.N * prm.lps + off;
          const float sc = prm.two_over_tau * fa * inv_a;
          uint32_t hp[(TABLES * P) / 2], lp[(TABLES * P) / 2];
#pragma unroll
          for (int e = 0; e < TABLES * P; e += 2) {
            const int j0 = e / P, p0 = e % P, j1 = (e + 1) / P, p1 = (e + 1) % P;
            const float d0 = sc * (As[j0 * P + p0] - sp[j0 * P + p0] * Ts[j0]);
            const float d1 = sc * (As[j1 * P + p1] - sp[j1 * P + p1] * Ts[j1]);
            hp[e / 2] = pack_bf16(d0, d1);
            lp[e / 2] = pack_bf16(d0 - __uint_as_float(hp[e / 2] << 16),
                                  d1 - __uint_as_float(hp[e / 2] & 0xffff0000u));
          }
          if ((TABLES * P) % 8 == 0) {   // the slice is then 16-byte aligned
#pragma unroll
            for (int e = 0; e < (TABLES * P) / 2; e += 4) {
              *reinterpret_cast<uint4*>(dh + 2 * e) = make_uint4(hp[e], hp[e + 1], hp[e + 2], hp[e + 3]);
              *reinterpret_cast<uint4*>(dl + 2 * e) = make_uint4(lp[e], lp[e + 1], lp[e + 2], lp[e + 3]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < (TABLES * P) / 2; ++e) {
              reinterpret_cast<uint32_t*>(dh)[e] = hp[e];
              reinterpret_cast<uint32_t*>(dl)[e] = lp[e];
            }
          }
        }
      }

      if (HAS_B) {
        if (!mbar_wait(bar + kbUP, i & 1)) { s_abort = 1; break; }
        if (t == 0) BW_TRACE(i, 19);
        tc_fence_after();
        if (CAUSAL) {
#pragma unroll 1
          for (int mt = 0; mt < 2; ++mt) {
            float vals[kNV];
            tmem_ld80(tmem + lane_off + (mt ? BwTm::S1 : BwTm::S0), vals);
            store_state_row_split(sb + BwSmem::sbf, sb + BwSmem::sbl, mt * 128 + t, vals);
          }
          fence_proxy_async();
        }
      }
      tc_fence_before();
      named_bar(1, kAlu);
      if (t == 0) BW_TRACE(i, 20);
    }
    if (MODE == kBuild && !s_abort) {
      float* out = seg_out + (((size_t)h * prm.n_rg + rg) * prm.G + g) * (size_t)256 * kNV;
      for (int mt = 0; mt < 2; ++mt) {
        float vals[kNV];
        tmem_ld80(tmem + lane_off + (mt ? BwTm::S1 : BwTm::S0), vals);
        float4* o4 = reinterpret_cast<float4*>(out + (size_t)(mt * 128 + t) * kNV);
#pragma unroll
        for (int cc = 0; cc < kNV / 4; ++cc)
          o4[cc] = make_float4(vals[4 * cc], vals[4 * cc + 1], vals[4 * cc + 2], vals[4 * cc + 3]);
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

// --------------------------------------------------------------------------- helpers
// Per row of the upstream gradient: gdot_i = -(g_i . o_i) (the extra feature column of
// g'_i) and r_i = 1/den'_i, both float32 (one warp per row).  den' comes from the
// caller's saved den (times L) or from forward accumulators.
template <typename T, typename TO>
__global__ void k_bwd_prep(const T* __restrict__ dout, const TO* __restrict__ out,
                           const float* __restrict__ num, const float* __restrict__ den_in,
                           float* __restrict__ gdot, float* __restrict__ rinv, int64_t rows,
                           float L) {
  // eight lanes per row (8 elements each), four rows per warp per pass, grid-stride
  const int lane = threadIdx.x & 31, sub = lane & 7;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t i = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 4 + (lane >> 3);
       i - (lane >> 3) < rows; i += warps * 4) {
    const bool valid = i < rows;
    float c = 0.f;
    if (valid) {
      float g[8], o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        g[e] = to_f(dout[i * kD + sub * 8 + e]);
        o[e] = to_f(out[i * kD + sub * 8 + e]);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) c = fmaf(g[e], o[e], c);
    }
    c += __shfl_xor_sync(0xffffffffu, c, 1);
    c += __shfl_xor_sync(0xffffffffu, c, 2);
    c += __shfl_xor_sync(0xffffffffu, c, 4);
    if (valid && sub == 0) {
      const float den = den_in ? den_in[i] * L : num[i * kNumStride + kD];
      gdot[i] = -c;
      rinv[i] = 1.0f / den;
    }
  }
}

// dst[h][N-1-n] = src[h][n] for float32 [H][N] rows.
__global__ void k_reverse_vec(const float* __restrict__ src, float* __restrict__ dst,
                              int64_t N, int H) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)H * N) return;
  const int64_t h = e / N, n = e % N;
  dst[h * N + (N - 1 - n)] = src[e];
}

// dst[h][N-1-n] = src[h][n] for 64-wide bf16 rows.
__global__ void k_reverse_rows(const __nv_bfloat16* __restrict__ src,
                               __nv_bfloat16* __restrict__ dst, int64_t N, int H) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // one 16-byte piece
  if (e >= (int64_t)H * N * 8) return;
  const int64_t row = e >> 3;
  const int piece = (int)(e & 7);
  const int64_t h = row / N, n = row % N;
  const uint4* s = reinterpret_cast<const uint4*>(src + row * kD) + piece;
  uint4* d = reinterpret_cast<uint4*>(dst + (h * N + (N - 1 - n)) * kD) + piece;
  *d = *s;
}

// dv[h][n] = first 64 accumulators of row n (reversed rows: N-1-n) of the anti-causal
// sweep.
template <typename T>
__global__ void k_dv_out(const float* __restrict__ num, T* __restrict__ dv, int64_t N, int H,
                         int reversed) {
  // grid (row blocks, H): sixteen threads per row, four columns (one float4) each
  const int h = blockIdx.y;
  const int64_t n = (int64_t)blockIdx.x * (blockDim.x >> 4) + (threadIdx.x >> 4);
  const int c4 = (threadIdx.x & 15) * 4;
  if (n >= N) return;
  const int64_t src = (int64_t)h * N + (reversed ? N - 1 - n : n);
  const float4 v = *reinterpret_cast<const float4*>(num + src * kNumStride + c4);
  T* d = dv + ((int64_t)h * N + n) * kD + c4;
  d[0] = from_f<T>(v.x);
  d[1] = from_f<T>(v.y);
  d[2] = from_f<T>(v.z);
  d[3] = from_f<T>(v.w);
}

// Hash backward, last steps, per token x (a row of q or k) on CUDA cores, for L * P above
// what the tensor-core finalize (tc_finalize.cuh) covers.  Input du' = (dL/du)/max(|x|,eps)
// as bf16 hi + lo arrays [rows][lps]: dxh' = W du' (projection transpose),
// dx = dxh' - xhat (xhat . dxh') (normalisation Jacobian), and dW partials x du'^T summed
// over the tokens of each block (x unnormalised: x du' = xhat du).
// Grid (blocks, H): head h's rows are h*N .. h*N + N - 1 and its planes W + h * w_hs; the
// partials go to part[h][block][L*P][64].
// 256 threads, 64 tokens per tile, LP padded to LPP = 16 * MT with zero columns.
// Register tiles: dxh' as 4 tokens x 4 dims per thread over K = LPP in steps of 4; dW as
// MT consecutive rows x 4 dims per thread over the 64 tokens of the tile.
constexpr int kMaxLP = 256;
constexpr int kFinTok = 64;
template <typename T, int MT, typename TG>
__global__ void __launch_bounds__(256) k_bwd_finalize(const T* __restrict__ x,
                                                     const __nv_bfloat16* __restrict__ du,
                                                     const float* __restrict__ W,
                                                     TG* __restrict__ dx, float* __restrict__ part,
                                                     int64_t N, int L, int P, int lps,
                                                     int64_t w_hs) {
  constexpr int LPP = 16 * MT;
  constexpr int LDS = LPP + 4;          // row stride of the du tile (16-byte aligned rows)
  extern __shared__ float4 fsm4[];
  float* fsm = reinterpret_cast<float*>(fsm4);
  const int LP = L * P;
  const int h = blockIdx.y;
  const __nv_bfloat16* du_lo = du + (size_t)gridDim.y * N * lps;
  W += (size_t)h * w_hs;
  // this head's rows
  x += (size_t)h * N * kD;
  du += (size_t)h * N * lps;
  du_lo += (size_t)h * N * lps;
  dx += (size_t)h * N * kD;
  const int64_t rows = N;
  float* Wt = fsm;                       // [LPP][64]: row lp = plane p of table l
  float* dus = Wt + LPP * 64;            // [64 tokens][LDS]
  float* xs = dus + kFinTok * LDS;       // [64 tokens][68]: x
  float* ninv = xs + kFinTok * 68;       // [64]: 1 / max(|x|, eps), 0 for padding rows
  const int tid = threadIdx.x;
  for (int e = tid; e < LPP * 64; e += 256) {
    const int lp = e / 64, d = e % 64;
    Wt[e] = lp < LP ? W[((size_t)(lp / P) * 64 + d) * P + (lp % P)] : 0.f;
  }
  const int tg = tid >> 4, dg = (tid & 15) * 4;   // dxh': tokens tg + 16 i, dims dg..dg+3
  const int rg = (tid >> 4) * MT;                 // dW: rows rg..rg+MT-1, dims dg..dg+3
  float acc[MT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[m][e] = 0.f;
  for (int64_t base = (int64_t)blockIdx.x * kFinTok; base < rows;
       base += (int64_t)gridDim.x * kFinTok) {
    __syncthreads();
    const int ntok = (int)min64(kFinTok, rows - base);
    for (int e = tid; e < kFinTok * LPP; e += 256) {
      const int tt = e / LPP, lp = e % LPP;
      float val = 0.f;
      if (tt < ntok && lp < LP) {
        const size_t o = (size_t)(base + tt) * lps + lp;
        val = __bfloat162float(du[o]) + __bfloat162float(du_lo[o]);
      }
      dus[tt * LDS + lp] = val;
    }
    {   // x and 1/|x|: 4 threads per token, 16 dims each
      const int tok = tid >> 2, qd = (tid & 3) * 16;
      const bool live = tok < ntok;
      float xv[16], ss = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        xv[e] = live ? to_f(x[(base + tok) * kD + qd + e]) : 0.f;
        ss = fmaf(xv[e], xv[e], ss);
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      const float inv = 1.0f / fmaxf(sqrtf(ss), kEpsNorm);
#pragma unroll
      for (int e = 0; e < 16; ++e) xs[tok * 68 + qd + e] = xv[e];
      if ((tid & 3) == 0) ninv[tok] = live ? inv : 0.f;
    }
    __syncthreads();
    // ---- dxh' = W du' for tokens tg + 16 i
    float dxh[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) dxh[i][e] = 0.f;
#pragma unroll 2
    for (int k = 0; k < LPP; k += 4) {
      float4 w[4], u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = *reinterpret_cast<const float4*>(Wt + (k + j) * 64 + dg);
#pragma unroll
      for (int i = 0; i < 4; ++i) u[i] = *reinterpret_cast<const float4*>(dus + (tg + 16 * i) * LDS + k);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float uu[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          dxh[i][0] = fmaf(w[j].x, uu[j], dxh[i][0]);
          dxh[i][1] = fmaf(w[j].y, uu[j], dxh[i][1]);
          dxh[i][2] = fmaf(w[j].z, uu[j], dxh[i][2]);
          dxh[i][3] = fmaf(w[j].w, uu[j], dxh[i][3]);
        }
      }
    }
    // ---- dx = dxh' - x inv^2 (x . dxh'); the 16 threads of a token are 16 lanes
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tok = tg + 16 * i;
      const float4 xv = *reinterpret_cast<const float4*>(xs + tok * 68 + dg);
      float dot = xv.x * dxh[i][0] + xv.y * dxh[i][1] + xv.z * dxh[i][2] + xv.w * dxh[i][3];
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      dot += __shfl_xor_sync(0xffffffffu, dot, 2);
      dot += __shfl_xor_sync(0xffffffffu, dot, 4);
      dot += __shfl_xor_sync(0xffffffffu, dot, 8);
      const float inv = ninv[tok];
      const float f = dot * inv * inv;
      if (tok < ntok) {
        TG* o = dx + (base + tok) * kD + dg;
        o[0] = from_f<TG>(dxh[i][0] - xv.x * f);
        o[1] = from_f<TG>(dxh[i][1] - xv.y * f);
        o[2] = from_f<TG>(dxh[i][2] - xv.z * f);
        o[3] = from_f<TG>(dxh[i][3] - xv.w * f);
      }
    }
    // ---- dW partials: rows rg..rg+MT-1 (table l, plane p), dims dg..dg+3
#pragma unroll 2
    for (int tt = 0; tt < kFinTok; ++tt) {
      const float4 xv = *reinterpret_cast<const float4*>(xs + tt * 68 + dg);
      float u[MT];
#pragma unroll
      for (int m = 0; m < MT; m += 4) {
        if (m + 4 <= MT) {
          const float4 u4 = *reinterpret_cast<const float4*>(dus + tt * LDS + rg + m);
          u[m] = u4.x; u[m + 1] = u4.y; u[m + 2] = u4.z; u[m + 3] = u4.w;
        } else {
#pragma unroll
          for (int mm = m; mm < MT; ++mm) u[mm] = dus[tt * LDS + rg + mm];
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        acc[m][0] = fmaf(xv.x, u[m], acc[m][0]);
        acc[m][1] = fmaf(xv.y, u[m], acc[m][1]);
        acc[m][2] = fmaf(xv.z, u[m], acc[m][2]);
        acc[m][3] = fmaf(xv.w, u[m], acc[m][3]);
      }
    }
  }
  float* o = part + ((size_t)h * gridDim.x + blockIdx.x) * LP * 64;
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const int lp = rg + m;
    if (lp < LP)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[lp * 64 + dg + e] = acc[m][e];
  }
}

inline int finalize_mt(int LP) { return (LP + 15) / 16; }
inline size_t finalize_smem(int LP) {
  const int LPP = 16 * finalize_mt(LP);
  return ((size_t)LPP * 64 + (size_t)kFinTok * (LPP + 4) + (size_t)kFinTok * 68 + kFinTok) *
         sizeof(float);
}

// dW[l][d][p] = sum of the partials [H][blocks][L*P][64] of both sides over heads and
// blocks, in fixed order; with per-head planes dW[h][l][d][p] sums head h's blocks only.
__global__ void k_bwd_dw_reduce(const float* __restrict__ pq, const float* __restrict__ pk,
                                int H, int nblocks, int per_head, float* __restrict__ dW,
                                int L, int P) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;   // over (H or 1) * L*64*P, W layout
  const int per = L * 64 * P;
  if (e >= (per_head ? H : 1) * per) return;
  const int hh = e / per, r = e % per;
  const int l = r / (64 * P), d = (r / P) % 64, p = r % P;
  const int LP = L * P;
  const size_t off = (size_t)(l * P + p) * 64 + d;
  const int h0 = per_head ? hh : 0, h1 = per_head ? hh + 1 : H;
  float acc = 0.f;
  for (int h = h0; h < h1; ++h)
    for (int b = 0; b < nblocks; ++b) acc += pq[((size_t)h * nblocks + b) * LP * 64 + off];
  for (int h = h0; h < h1; ++h)
    for (int b = 0; b < nblocks; ++b) acc += pk[((size_t)h * nblocks + b) * LP * 64 + off];
  dW[e] = acc;
}

// 3-D view [H][N][64] bf16 of a feature tensor for the 32B-swizzled loads: boxes of
// 16 columns x 128 rows.
inline bool encode_feat_tmap(CUtensorMap* m, const void* base, int64_t N, int H) {
  const auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)N, (cuuint64_t)H};
  cuuint64_t strides[2] = {128, (cuuint64_t)N * 128};
  cuuint32_t box[3] = {16, (cuuint32_t)kC, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace race

// Pipelined corner-gradient sweep of the backward for R = 256 buckets (P = 8), causal:
// the same arithmetic as k_bwd_phi<8, kSweep, REV> (notation there), with the CUDA-core
// work of step i+1 overlapping the MMAs of step i.
//
// A CTA owns half a table (128 sketch rows: the buckets whose plane-7 bit is the CTA's
// rank in its 2-CTA cluster) for one segment of one head.  The two halves of a table form
// a cluster: each computes the per-plane gradient sums of its 128 corners, the upper half
// sends them to the lower half through distributed shared memory, and the lower half adds
// the two and stores du' = (dL/du) / |x| as a bf16 hi + lo pair ([JA] §2.2: the soft
// assignment is differentiable; the per-plane split follows from the softmax over corners
// factorising into logistic pairs, [JA] §2.1).
//
// The scaled projections z = (x . W_l[:,p]) (2/tau) / |x| of every token, table and plane
// come from a tensor-core pre-pass (k_bwd_zproj), one 4 KB bulk copy per side and step.
//
// Per step i (128 tokens of side a and of side b):
//   warp 16 (issuer A): dP(i) = X S^T (state hi + lo) + mask(XY) p(b) into one of two dP
//                       buffers, with UPD(i): S += p(b)^T Y issued between the two parts
//                       (the first needs no mask); XY(i+1) = X Y^T (-> DW)
//   warp 17 (issuer B): the copies of features and projections
//   warps 0-3   (EXP):  p(b) of step i into one of two tiles
//   warps 4-7, 12-15 (MASK + STAGE, one 64-key block and part of the state per warp):
//                       after dP(i-1), S_{i-1} from tensor memory into its bf16 hi + lo
//                       copy for dP(i); mask(XY(i)) rounded to bf16 in place (the A
//                       operand of dP(i))
//   warps 8-11  (HASH): side-a logistic factors; reads dP(i), per-plane sums over the half
//                       table, exchange, du' store
// Every producer/consumer pair has its own mbarrier, every wait is bounded, and no
// barrier can complete a phase twice ahead of one of its waiters (two-slot resources
// have one barrier per slot).
#pragma once

#include "tc_backward.cuh"
#include "tc_sweep256.cuh"
#include "tc_sweep_pipe.cuh"

namespace race {
namespace tc {

constexpr int kBPThreads = 576;

enum BPBar : int {
  bp_FA0 = 0, bp_FA1, bp_FB0, bp_FB1, bp_Z0, bp_Z1, bp_ZREAD0, bp_ZREAD1, bp_PB0, bp_PB1,
  bp_PBU0, bp_PBU1, bp_PBD0, bp_PBD1, bp_XY0, bp_XY1, bp_INTRA0, bp_INTRA1, bp_DP0, bp_DP1,
  bp_DPFREE0, bp_DPFREE1, bp_SBF, bp_XFULL, bp_XFREE, bp_COUNT
};

struct BPSmem {
  static constexpr uint32_t fa0 = 0, fa1 = 20480;                // X feature tiles
  static constexpr uint32_t fb0 = 40960, fb1 = 61440;            // Y feature tiles
  static constexpr uint32_t pb0 = 81920, pb1 = 114688;           // p(b): 128 tokens x 128 rows
  static constexpr uint32_t shi = 147456, slo = 167936;          // state hi / lo, 128 x 80
  static constexpr uint32_t z = 188416;                          // [slot][side] 128 x 8 float
  static constexpr uint32_t inva = 204800;                       // 1/|x| of side a, two slots
  static constexpr uint32_t xch = 205824;                        // exchange, 128 x 8 float
  static constexpr uint32_t bars = 209920;
  static constexpr uint32_t tmem_slot = bars + 8 * bp_COUNT;
  static constexpr uint32_t total = tmem_slot + 16;
  static constexpr uint32_t alloc = total + 1024;
};
static_assert(BPSmem::alloc <= 232448, "shared memory budget of one CTA");

struct BPTm {   // tensor-memory columns
  static constexpr uint32_t S = 0, DW = 80, DP0 = 208, DP1 = 336;
};

// 128-row p(b) tile in the 128B-swizzled layout of the forward sweep's p(k) tile (two
// atoms of 64 rows, 16 KB each; token t's 128-byte row at (t/8) * 1024 + (t%8) * 128; the
// 16-byte chunk of rows 8c..8c+7 at index (c%8) XOR (t%8)): the rows of half `hb` of a
// 256-bucket table, bucket = hb * 128 + row, as products of the corner factors.
__device__ __forceinline__ void expand_half128(uint32_t tile, int t, const Corners& k, int hb) {
  const uint32_t base = tile + (t >> 3) * 1024 + (t & 7) * 128;
#pragma unroll 1
  for (int gg = 0; gg < 4; ++gg) {
    const float h5 = corners_h5(k, 4 * hb + gg);   // planes 5-7 (plane 7 = hb)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = 4 * gg + j;                     // rows 8c .. 8c+7 of the half
      const uint64_t hh = bcast_f32x2(h5 * k.p34[j]);
      st_shared_v4(base + (uint32_t)(c >> 3) * 16384 + ((uint32_t)((c & 7) ^ (t & 7)) << 4),
                   mul_pack_bf16(k.lo2[0], hh), mul_pack_bf16(k.lo2[1], hh),
                   mul_pack_bf16(k.lo2[2], hh), mul_pack_bf16(k.lo2[3], hh));
    }
  }
}

// Byte offset of columns 8m .. 8m+7 of state row r in a K-major 32B-swizzled copy (atom
// m/2 of 16 columns at (m/2) * 4 KB, rows of 32 B, the two 16-byte halves swapped on rows
// 4-7 of each 8-row group): the layout of the feature tiles, as the B operand of X S^T.
__device__ __forceinline__ uint32_t state_sw32_off(int r, int m) {
  return (uint32_t)(m >> 1) * 4096 + (uint32_t)r * 32 + ((uint32_t)((m & 1) ^ ((r >> 2) & 1)) << 4);
}

// Extra feature columns 64..79 of the [v | 1] side, [1, 1, 0, ...] on every row, written
// once into atom 4 of a 32B-swizzled feature tile (the two 16-byte halves of a row are
// swapped on rows 4-7 of each 8-row group).  Rows past the end of the sequence keep the
// ones: their v columns are zero, and where they meet the other side their corner
// probabilities are zero.
__device__ __forceinline__ void store_ones_atom(uint32_t tile, int t) {
  const uint32_t row = tile + 4 * 4096 + t * 32;
  const uint32_t first = ((t >> 2) & 1) << 4;
  st_shared_v4(row + first, pack_bf16(1.f, 1.f), 0u, 0u, 0u);
  st_shared_v4(row + (first ^ 16), 0u, 0u, 0u, 0u);
}

// Eight state values as bf16 hi and lo = value - hi (four packed pairs each).
__device__ __forceinline__ void split_state8(const uint32_t* r, uint32_t* hi, uint32_t* lo) {
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float a = __uint_as_float(r[2 * e]), b = __uint_as_float(r[2 * e + 1]);
    hi[e] = pack_bf16(a, b);
    lo[e] = pack_bf16(a - __uint_as_float(hi[e] << 16), b - __uint_as_float(hi[e] & 0xffff0000u));
  }
}

__device__ __forceinline__ void ld_shared_v4f(uint32_t addr, float* v) {
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3])
               : "r"(addr)
               : "memory");
}

// REV = false (q side): side a = q with features X = g', side b = k with Y = [v | 1];
// REV = true (k side, reverse sweep): side a = k with X = [v | 1], side b = q with Y = g'.
// tge: the extra feature columns of g' ([e_hi, e_lo, 0, ...], e = -(g . o), 16 bf16 per
// row); rinv: the row factor 1/den' of the g' side.  za, zb: scaled projections of the
// two sides, [H][L][zstride][8] float32; inv_a: 1/|x| of side a, [H][zstride].
template <bool REV>
__global__ void __launch_bounds__(kBPThreads, 1) __cluster_dims__(1, 2, 1)
    k_bwd_pipe(const __grid_constant__ CUtensorMap tfa, const __grid_constant__ CUtensorMap tfb,
               const __grid_constant__ CUtensorMap tge, const float* __restrict__ rinv,
               const float* __restrict__ za, const float* __restrict__ zb,
               const float* __restrict__ inv_a, int64_t zstride,
               const float* __restrict__ init, __nv_bfloat16* __restrict__ du_out, Params prm) {
  constexpr int P = 8;
  constexpr bool A_IS_G = !REV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + BPSmem::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + BPSmem::tmem_slot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, h = blockIdx.z;
  const int l = blockIdx.y >> 1;                    // table
  const int hb = (int)cluster_rank();               // half of the table (plane-7 bit)
  const int64_t s0 = (int64_t)g * prm.seg_len;
  const int64_t s1 = min64(prm.N, s0 + prm.seg_len);
  const int n = (int)((s1 - s0 + kC - 1) / kC);

  if (threadIdx.x == 0) {
    for (int i = 0; i < bp_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i == bp_PB0 || i == bp_PB1 || i == bp_DPFREE0 || i == bp_DPFREE1) cnt = 4;
      if (i == bp_ZREAD0 || i == bp_ZREAD1) cnt = 8;   // EXP and HASH warps
      if (i == bp_INTRA0 || i == bp_INTRA1 || i == bp_SBF) cnt = 8;   // MASK + STAGE warps
      if (i == bp_XFREE) cnt = 128;                    // one arrival per thread of the peer
      mbar_init(bar + i, cnt);
    }
    fence_mbar_init();
    // the lower half expects the upper half's 128 x 32 bytes of step 0 (asynchronous
    // stores completing on XFULL); each later step's expectation is posted after the
    // previous step's exchange
    if (hb == 0) mbar_arrive_expect_tx(bar + bp_XFULL, 128 * 32);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (threadIdx.x >= 256 && threadIdx.x < 384) {
    // the [v | 1] side's extra columns: constant, written once
    const int t = threadIdx.x - 256;
    if (A_IS_G) {
      store_ones_atom(sb + BPSmem::fb0, t);
      store_ones_atom(sb + BPSmem::fb1, t);
    } else {
      store_ones_atom(sb + BPSmem::fa0, t);
      store_ones_atom(sb + BPSmem::fa1, t);
    }
    fence_proxy_async();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // initial state of the half table: tensor memory and its bf16 hi + lo copy
  if (threadIdx.x < 128) {
    const int t = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float* src = init + (((size_t)h * prm.n_rg + l) * prm.G + g) * 256 * kNV +
                       (size_t)(hb * 128 + t) * kNV;
    float vals[kNV];
#pragma unroll
    for (int c = 0; c < kNV; ++c) vals[c] = prm.have_init ? src[c] : 0.f;
    uint32_t r[16];
#pragma unroll
    for (int b = 0; b < 5; ++b) {
#pragma unroll
      for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(vals[b * 16 + e]);
      tmem_st16(tmem + lane_off + BPTm::S + b * 16, r);
    }
    tmem_st_wait();
#pragma unroll
    for (int m = 0; m < 10; ++m) {
      uint32_t hp[4], lp[4];
      uint32_t rr[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) rr[e] = __float_as_uint(vals[8 * m + e]);
      split_state8(rr, hp, lp);
      st_shared_v4(sb + BPSmem::shi + state_sw32_off(t, m), hp[0], hp[1], hp[2], hp[3]);
      st_shared_v4(sb + BPSmem::slo + state_sw32_off(t, m), lp[0], lp[1], lp[2], lp[3]);
    }
    fence_proxy_async();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();   // both halves have initialised their barriers before any remote access

  bool ok = true;
  auto wait = [&](int b, uint32_t par) {
    if (ok && !mbar_wait(bar + b, par)) ok = false;
    ok = __all_sync(0xffffffffu, ok);
    return ok;
  };
  auto chunk_of = [&](int i) { return REV ? n - 1 - i : i; };
  auto t0_of = [&](int i) { return (int)(s0 + (int64_t)chunk_of(i) * kC); };
  // row factor of one side's token (the g' side: 1/den'; the other: 1), 0 past the end
  auto row_factor = [&](bool g_side, int i, int t) {
    const int64_t row = s0 + (int64_t)chunk_of(i) * kC + t;
    return row < s1 ? (g_side ? rinv[(size_t)h * prm.N + row] : 1.f) : 0.f;
  };
  const size_t zrow0 = ((size_t)h * prm.L + l) * zstride;   // this table's projections

  if (warp >= 16) {
    // ================================================================ issuers
    const uint32_t id_128 = idesc_bf16(128, 128, 0, 0);   // XY and X S^T
    const uint32_t id_d3 = idesc_bf16(128, 128, 0, 1);    // A tmem, B MN-major
    const uint32_t id_up = idesc_bf16(128, kNV, 1, 1);    // A, B MN-major
    auto load_z = [&](int i) {   // projections of both sides and 1/|x_a| of step i
      const int st = i & 1;
      const int t0 = t0_of(i);
      mbar_arrive_expect_tx(bar + bp_Z0 + st, 2 * 4096 + 512);
      bulk_load(sm + BPSmem::z + st * 8192, za + (zrow0 + t0) * 8, 4096, bar + bp_Z0 + st);
      bulk_load(sm + BPSmem::z + st * 8192 + 4096, zb + (zrow0 + t0) * 8, 4096,
                bar + bp_Z0 + st);
      bulk_load(sm + BPSmem::inva + st * 512, inv_a + (size_t)h * zstride + t0, 512,
                bar + bp_Z0 + st);
    };
    auto load_fa = [&](int i) {   // X feature tile of step i into slot i % 2
      const int st = i & 1;
      const int t0 = t0_of(i);
      uint8_t* dst = sm + (st ? BPSmem::fa1 : BPSmem::fa0);
      mbar_arrive_expect_tx(bar + bp_FA0 + st, A_IS_G ? 20480 : 16384);
#pragma unroll
      for (int a = 0; a < 4; ++a) tma_load_3d(dst + a * 4096, &tfa, a * 16, t0, h, bar + bp_FA0 + st);
      if (A_IS_G) tma_load_3d(dst + 4 * 4096, &tge, 0, t0, h, bar + bp_FA0 + st);
    };
    auto load_fb = [&](int i) {   // Y feature tile of step i into slot i % 2
      const int st = i & 1;
      const int t0 = t0_of(i);
      uint8_t* dst = sm + (st ? BPSmem::fb1 : BPSmem::fb0);
      mbar_arrive_expect_tx(bar + bp_FB0 + st, A_IS_G ? 16384 : 20480);
#pragma unroll
      for (int a = 0; a < 4; ++a) tma_load_3d(dst + a * 4096, &tfb, a * 16, t0, h, bar + bp_FB0 + st);
      if (!A_IS_G) tma_load_3d(dst + 4 * 4096, &tge, 0, t0, h, bar + bp_FB0 + st);
    };
    if (warp == 16) {
      // ---------------------------------------------------------- issuer A: XY, UPD, dP
      // Tensor-core order: ... X S^T(i), UPD(i), intra(i), XY(i+1), X S^T(i+1), ...  MMAs
      // issued by one thread execute in issue order, so XY(i+1) overwrites DW only after
      // dP(i) has read it; X S^T(i+1) and UPD(i+1) run while XY(i+1) is masked.
      auto xy = [&](int i) {
        const int st = i & 1;
        const uint32_t fa = sb + (st ? BPSmem::fa1 : BPSmem::fa0);
        const uint32_t fb = sb + (st ? BPSmem::fb1 : BPSmem::fb0);
        if (lane == 0) BW_TRACE(i, 27);
        if (!wait(bp_FA0 + st, (uint32_t)(i >> 1) & 1)) return false;
        if (lane == 0) BW_TRACE(i, 28);
        if (!wait(bp_FB0 + st, (uint32_t)(i >> 1) & 1)) return false;
        if (lane == 0) BW_TRACE(i, 2);
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int s = 0; s < 5; ++s)
            umma_ss(tmem + BPTm::DW, sdesc(fa + s * 4096, 16, 256, kSwizzle32B),
                    sdesc(fb + s * 4096, 16, 256, kSwizzle32B), id_128, s > 0);
          umma_commit(bar + bp_XY0 + st);
        }
        __syncwarp();
        return true;
      };
      if (n > 0) xy(0);
      for (int i = 0; i < n && ok; ++i) {
        if (lane == 0) BW_TRACE(i, 0);
        const int st = i & 1;
        const uint32_t fa = sb + (st ? BPSmem::fa1 : BPSmem::fa0);
        const uint32_t fb = sb + (st ? BPSmem::fb1 : BPSmem::fb0);
        const uint32_t pbt = sb + (st ? BPSmem::pb1 : BPSmem::pb0);
        // dP(i) in two parts: X S_{i-1}^T (hi + lo copy) as soon as the copy exists and
        // dP buffer st was read two steps ago, then the state update, then the in-chunk
        // term mask(XY(i)) p(b) once the MASK warps have rounded XY(i): the tensor core
        // works on the first two while XY(i) is masked.
        if (!wait(bp_PB0 + st, (uint32_t)(i >> 1) & 1)) break;
        if (i > 0 && !wait(bp_SBF, (uint32_t)(i - 1) & 1)) break;
        if (i > 1 && !wait(bp_DPFREE0 + st, (uint32_t)((i - 2) >> 1) & 1)) break;
        if (lane == 0) BW_TRACE(i, 4);
        tc_fence_after();
        if (elect_one()) {
          const uint32_t dP = tmem + (st ? BPTm::DP1 : BPTm::DP0);
#pragma unroll
          for (int s = 0; s < 5; ++s) {
            const uint64_t xd = sdesc(fa + s * 4096, 16, 256, kSwizzle32B);
            umma_ss(dP, xd, sdesc(sb + BPSmem::shi + s * 4096, 16, 256, kSwizzle32B), id_128,
                    s > 0);
            umma_ss(dP, xd, sdesc(sb + BPSmem::slo + s * 4096, 16, 256, kSwizzle32B), id_128, 1);
          }
          // state update with p(b) of step i (S_{i-1} was copied out: SBF above)
          const uint64_t dpb = sdesc(pbt, 16384, 1024, kSwizzle128B);
#pragma unroll
          for (int s = 0; s < 8; ++s)
            umma_ss(tmem + BPTm::S, dpb + 128 * s, sdesc(fb + s * 512, 4096, 256, kSwizzle32B),
                    id_up, 1);
          umma_commit(bar + bp_PBU0 + st);
        }
        __syncwarp();
        if (!wait(bp_INTRA0 + st, (uint32_t)(i >> 1) & 1)) break;
        if (lane == 0) BW_TRACE(i, 3);
        tc_fence_after();
        if (elect_one()) {
          const uint32_t dP = tmem + (st ? BPTm::DP1 : BPTm::DP0);
          const uint64_t dpb = sdesc(pbt, 16384, 1024, kSwizzle128B);
#pragma unroll
          for (int s = 0; s < 8; ++s)   // keys 16 s ..: block s/4, packed columns 8 (s % 4)
            umma_ts(dP, tmem + BPTm::DW + (s >> 2) * 64 + (s & 3) * 8, dpb + 128 * s, id_d3, 1);
          umma_commit(bar + bp_DP0 + st);
          umma_commit(bar + bp_PBD0 + st);
        }
        __syncwarp();
        if (i + 1 < n && !xy(i + 1)) break;
        // the X slot of step i is refilled with step i+2 once dP(i) has read it
        if (i + 2 < n) {
          if (!wait(bp_DP0 + st, (uint32_t)(i >> 1) & 1)) break;
          if (lane == 0) BW_TRACE(i, 1);
          if (elect_one()) load_fa(i + 2);
          __syncwarp();
        }
      }
    } else {
      // ---------------------------------------------------------- issuer B: copies
      if (n > 0) {
        if (elect_one()) {
          prefetch_tmap(&tfa);
          prefetch_tmap(&tfb);
          prefetch_tmap(&tge);
          load_z(0);
          load_fa(0);
          load_fb(0);
          if (n > 1) {
            load_z(1);
            load_fa(1);
            load_fb(1);
          }
        }
        __syncwarp();
      }
      for (int i = 0; i + 2 < n && ok; ++i) {
        const int st = i & 1;
        const uint32_t par = (uint32_t)(i >> 1) & 1;
        // projections of step i+2 once both sides have read step i's
        if (!wait(bp_ZREAD0 + st, par)) break;
        if (lane == 0) BW_TRACE(i, 5);
        if (elect_one()) load_z(i + 2);
        __syncwarp();
        // Y of step i+2 once XY(i) and UPD(i) have read step i's
        if (!wait(bp_XY0 + st, par) || !wait(bp_PBU0 + st, par)) break;
        if (lane == 0) BW_TRACE(i, 6);
        if (elect_one()) load_fb(i + 2);
        __syncwarp();
      }
    }
  } else if (warp < 4) {
    // ================================================================ EXP: p(b)
    const int t = warp * 32 + lane;
    float fb_next = n > 0 ? row_factor(!A_IS_G, 0, t) : 0.f;
    for (int i = 0; i < n; ++i) {
      const int st = i & 1;
      const float fb = fb_next;   // row factor (0 past the end), loaded a step ahead
      if (i + 1 < n) fb_next = row_factor(!A_IS_G, i + 1, t);
      if (!wait(bp_Z0 + st, (uint32_t)(i >> 1) & 1)) break;
      if (t == 0) BW_TRACE(i, 9);
      float z[P];
      ld_shared_v4f(sb + BPSmem::z + st * 8192 + 4096 + t * 32, z);
      ld_shared_v4f(sb + BPSmem::z + st * 8192 + 4096 + t * 32 + 16, z + 4);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + bp_ZREAD0 + st);
      float sp[P], smv[P];
#pragma unroll
      for (int p = 0; p < P; ++p) logistic_fast(z[p], sp[p], smv[p]);
      Corners k;
      corners_of(sp, smv, fb, k);
      // p(b) tile slot free once UPD(i-2) and dP(i-2) have read it; the expansion runs
      // after MASK(i-1), alongside dP(i-1), off the CUDA-core work between dP(i-1) and dP(i)
      if (i > 1 && (!wait(bp_PBU0 + st, (uint32_t)((i - 2) >> 1) & 1) ||
                    !wait(bp_PBD0 + st, (uint32_t)((i - 2) >> 1) & 1)))
        break;
      if (i > 0 && !wait(bp_INTRA0 + ((i - 1) & 1), (uint32_t)((i - 1) >> 1) & 1)) break;
      if (t == 0) BW_TRACE(i, 10);
      expand_half128(sb + (st ? BPSmem::pb1 : BPSmem::pb0), t, k, hb);
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + bp_PB0 + st);
      if (t == 0) BW_TRACE(i, 11);
    }
  } else if (warp >= 8 && warp < 12) {
    // ================================================================ HASH (side a)
    const int q4 = warp - 8;
    const int t = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t peer = (uint32_t)(hb ^ 1);
    const uint32_t xch = sb + BPSmem::xch + t * 32;
    float fa_next = n > 0 ? row_factor(A_IS_G, 0, t) : 0.f;
    for (int i = 0; i < n; ++i) {
      const int st = i & 1;
      const int64_t row = s0 + (int64_t)chunk_of(i) * kC + t;
      const bool valid = row < s1;
      const float fa = fa_next;   // row factor (0 past the end), loaded a step ahead
      if (i + 1 < n) fa_next = row_factor(A_IS_G, i + 1, t);
      if (t == 0) BW_TRACE(i, 26);
      // projections and logistic factors of side a
      if (!wait(bp_Z0 + st, (uint32_t)(i >> 1) & 1)) break;
      if (t == 0) BW_TRACE(i, 15);
      float z[P];
      ld_shared_v4f(sb + BPSmem::z + st * 8192 + t * 32, z);
      ld_shared_v4f(sb + BPSmem::z + st * 8192 + t * 32 + 16, z + 4);
      const float inv = valid ? reinterpret_cast<const float*>(sm + BPSmem::inva + st * 512)[t] : 0.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + bp_ZREAD0 + st);
      // corner factors: low corners e (planes 0-2), and the high corner c = 4 q + g of the
      // half as p34[g] (planes 3-4) times p567[q] (planes 5-6 and plane 7 = hb)
      float sp[P], lo[8], p34[4], p567[4];
      {
        float sm_[P];
#pragma unroll
        for (int p = 0; p < P; ++p) logistic_fast(z[p], sp[p], sm_[p]);
#pragma unroll
        for (int b = 0; b < 8; ++b)
          lo[b] = ((b & 1) ? sp[0] : sm_[0]) * ((b & 2) ? sp[1] : sm_[1]) * ((b & 4) ? sp[2] : sm_[2]);
        const float f7 = hb ? sp[7] : sm_[7];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          p34[g] = ((g & 1) ? sp[3] : sm_[3]) * ((g & 2) ? sp[4] : sm_[4]);
          p567[g] = ((g & 1) ? sp[5] : sm_[5]) * ((g & 2) ? sp[6] : sm_[6]) * f7;
        }
      }
      // per-plane sums over this half's 128 corners, after MASK(i+1): alongside dP(i+1),
      // off the CUDA-core work between dP(i) and dP(i+1)
      if (!wait(bp_DP0 + st, (uint32_t)(i >> 1) & 1)) break;
      if (i + 1 < n && !wait(bp_INTRA0 + ((i + 1) & 1), (uint32_t)((i + 1) >> 1) & 1)) break;
      if (t == 0) BW_TRACE(i, 16);
      tc_fence_after();
      // Packed pairs over the 8 low corners e of each group of 8 rows: with
      // m_e = lo_e dP_e, S1 = (m0+m2, m1+m3), S2 = (m4+m6, m5+m7), T = S1 + S2 and
      // U = (m2+m6, m3+m7): sum_e m_e = T.x + T.y, plane 0 = T.y, plane 1 = U.x + U.y,
      // plane 2 = S2.x + S2.y; planes 3-6 take hi_c T where bit p-3 of the group c is set.
      uint64_t accT = 0, accU = 0, accS2 = 0, acc3 = 0, acc4 = 0, acc5 = 0, acc6 = 0;
      const uint64_t lo01 = pair_f32x2(lo[0], lo[1]), lo23 = pair_f32x2(lo[2], lo[3]);
      const uint64_t lo45 = pair_f32x2(lo[4], lo[5]), lo67 = pair_f32x2(lo[6], lo[7]);
      const uint32_t dpc = tmem + lane_off + (st ? BPTm::DP1 : BPTm::DP0);
      // 16 columns per piece; the load of piece q+1 is in flight while piece q is summed
      uint32_t xb[2][16];
      tmem_ld16(dpc, xb[0]);
      tmem_ld_wait();
#pragma unroll
      for (int qq = 0; qq < 8; ++qq) {
        if (qq + 1 < 8) tmem_ld16(dpc + (qq + 1) * 16, xb[(qq + 1) & 1]);
        const uint32_t* x = xb[qq & 1];
#pragma unroll
        for (int g8 = 0; g8 < 2; ++g8) {
          const int c = qq * 2 + g8;                  // high corner index (planes 3-6)
          const uint32_t* xg = x + g8 * 8;
          const uint64_t m01 = mul_f32x2(lo01, pair_u32x2(xg[0], xg[1]));
          const uint64_t m23 = mul_f32x2(lo23, pair_u32x2(xg[2], xg[3]));
          const uint64_t m45 = mul_f32x2(lo45, pair_u32x2(xg[4], xg[5]));
          const uint64_t m67 = mul_f32x2(lo67, pair_u32x2(xg[6], xg[7]));
          const uint64_t s2 = add_f32x2(m45, m67);
          const uint64_t tt = add_f32x2(add_f32x2(m01, m23), s2);
          const uint64_t uu = add_f32x2(m23, m67);
          const uint64_t hz = bcast_f32x2(p34[c & 3] * p567[c >> 2]);
          const uint64_t ht = mul_f32x2(hz, tt);
          accT = add_f32x2(accT, ht);
          accU = fma_f32x2(hz, uu, accU);
          accS2 = fma_f32x2(hz, s2, accS2);
          if (c & 1) acc3 = add_f32x2(acc3, ht);
          if (c & 2) acc4 = add_f32x2(acc4, ht);
          if (c & 4) acc5 = add_f32x2(acc5, ht);
          if (c & 8) acc6 = add_f32x2(acc6, ht);
        }
        if (qq + 1 < 8) tmem_ld_wait();
      }
      float Ts, As[P];
      {
        const float2 vt = unpack_f32x2(accT), vu = unpack_f32x2(accU), vs = unpack_f32x2(accS2);
        const float2 v3 = unpack_f32x2(acc3), v4 = unpack_f32x2(acc4);
        const float2 v5 = unpack_f32x2(acc5), v6 = unpack_f32x2(acc6);
        Ts = vt.x + vt.y;
        As[0] = vt.y;
        As[1] = vu.x + vu.y;
        As[2] = vs.x + vs.y;
        As[3] = v3.x + v3.y;
        As[4] = v4.x + v4.y;
        As[5] = v5.x + v5.y;
        As[6] = v6.x + v6.y;
        As[7] = 0.f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + bp_DPFREE0 + st);
      if (t == 0) BW_TRACE(i, 17);
      if (hb) As[7] = Ts;                            // every corner of the upper half has bit 7
      const float sc = prm.two_over_tau * fa * inv;
      float d[P];
#pragma unroll
      for (int p = 0; p < P; ++p) d[p] = sc * (As[p] - sp[p] * Ts);
      // ---- the two halves' sums meet in the lower half (one exchange slot)
      if (t == 0) BW_TRACE(i, 18);
      if (hb) {
        if (i > 0 && !mbar_wait_cluster(bar + bp_XFREE, (uint32_t)(i - 1) & 1)) { ok = false; }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const uint32_t dst = map_to_rank(xch, peer);
        const uint32_t rbar = map_to_rank(smem_u32(bar + bp_XFULL), peer);
        st_async_v4(dst, d[0], d[1], d[2], d[3], rbar);
        st_async_v4(dst + 16, d[4], d[5], d[6], d[7], rbar);
      } else {
        if (!mbar_wait_cluster(bar + bp_XFULL, (uint32_t)i & 1)) { ok = false; }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (t == 0) BW_TRACE(i, 19);
        // the next step's data cannot arrive before this thread's XFREE arrival below
        if (t == 0 && i + 1 < n) mbar_arrive_expect_tx(bar + bp_XFULL, 128 * 32);
        float o[8];
        ld_shared_v4f(xch, o);
        ld_shared_v4f(xch + 16, o + 4);
#pragma unroll
        for (int p = 0; p < P; ++p) d[p] += o[p];
        // the slot's values are in registers (used above): the peer may refill it
        asm volatile("" ::"f"(d[0]), "f"(d[1]), "f"(d[2]), "f"(d[3]), "f"(d[4]), "f"(d[5]),
                     "f"(d[6]), "f"(d[7]));
        mbar_arrive_remote_relaxed(map_to_rank(smem_u32(bar + bp_XFREE), peer));
        if (t == 0) BW_TRACE(i, 20);
        const size_t off = ((size_t)h * prm.N + row) * prm.lps + (size_t)l * P;
        if (valid && RACE_IN_RANGE(off + P - 1, (int64_t)prm.H * prm.N * prm.lps)) {
          uint32_t hp[4], lp[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            hp[e] = pack_bf16(d[2 * e], d[2 * e + 1]);
            lp[e] = pack_bf16(d[2 * e] - __uint_as_float(hp[e] << 16),
                              d[2 * e + 1] - __uint_as_float(hp[e] & 0xffff0000u));
          }
          *reinterpret_cast<uint4*>(du_out + off) = make_uint4(hp[0], hp[1], hp[2], hp[3]);
          *reinterpret_cast<uint4*>(du_out + (size_t)prm.H * prm.N * prm.lps + off) =
              make_uint4(lp[0], lp[1], lp[2], lp[3]);
        }
        if (t == 0) BW_TRACE(i, 25);
      }
    }
  } else {
    // ================================================================ MASK + STAGE
    // Warps 4-7 and 12-15: lane quarter q4 = warp % 4, key block kb = warp / 12 (keys
    // 64 kb .. 64 kb + 63; state columns 40 kb .. 40 kb + 39).  Per step i: STAGE(i-1) after
    // dP(i-1), which also covers UPD(i-1) issued before it by the same thread: S_{i-1}
    // from tensor memory into its bf16 hi + lo copy read by dP(i); then MASK(i): the
    // key block of XY(i), masked and rounded to bf16 pairs in place, in the first 32
    // columns of the block (the A operand of dP(i)).
    const int q4 = warp & 3, kb = warp >= 12 ? 1 : 0;
    const int t = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const int m0 = kb * 5;                         // state columns 8 m0 .. 8 m0 + 39
    const int j_lo = kb * 64, j_hi = kb * 64 + 63, t_lo = q4 * 32, t_hi = q4 * 32 + 31;
    const bool all_kept = REV ? (j_lo >= t_hi) : (j_hi <= t_lo);
    const bool all_dropped = REV ? (j_hi < t_lo) : (j_lo > t_hi);
    for (int i = 0; i < n; ++i) {
      if (i > 0) {
        if (!wait(bp_DP0 + ((i - 1) & 1), (uint32_t)((i - 1) >> 1) & 1)) break;
        if (t == 0) BW_TRACE(i - 1, 23);
        tc_fence_after();
        // this warp's 40 state columns (8-column groups m0 .. m0+4) in one round of loads
        uint32_t r[40];
#pragma unroll
        for (int j = 0; j < 5; ++j) tmem_ld8(tmem + lane_off + BPTm::S + (m0 + j) * 8, r + 8 * j);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 5; ++j) {
          uint32_t hi[4], lo[4];
          split_state8(r + 8 * j, hi, lo);
          const uint32_t o = state_sw32_off(t, m0 + j);
          st_shared_v4(sb + BPSmem::shi + o, hi[0], hi[1], hi[2], hi[3]);
          st_shared_v4(sb + BPSmem::slo + o, lo[0], lo[1], lo[2], lo[3]);
        }
        tc_fence_before();
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar + bp_SBF);
        if (t == 0) BW_TRACE(i - 1, 24);
      }
      if (!wait(bp_XY0 + (i & 1), (uint32_t)(i >> 1) & 1)) break;
      if (t == 0) BW_TRACE(i, 12);
      tc_fence_after();
      // two halves of 32 keys: fp32 columns 64 kb + 32 h .. -> bf16 pairs in 64 kb + 16 h ..,
      // which this warp has already read
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t x[32];
        if (all_dropped) {
#pragma unroll
          for (int e = 0; e < 16; ++e) x[e] = 0u;
        } else {
          tmem_ld16(tmem + lane_off + BPTm::DW + kb * 64 + hh * 32, x);
          tmem_ld16(tmem + lane_off + BPTm::DW + kb * 64 + hh * 32 + 16, x + 16);
          tmem_ld_wait();
          if (all_kept) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              x[e] = pack_bf16(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1]));
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int j0 = kb * 64 + hh * 32 + 2 * e;
              const bool k0 = REV ? (j0 >= t) : (j0 <= t);
              const bool k1 = REV ? (j0 + 1 >= t) : (j0 + 1 <= t);
              x[e] = pack_bf16(k0 ? __uint_as_float(x[2 * e]) : 0.f,
                               k1 ? __uint_as_float(x[2 * e + 1]) : 0.f);
            }
          }
        }
        tmem_st16(tmem + lane_off + BPTm::DW + kb * 64 + hh * 16, x);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + bp_INTRA0 + (i & 1));
      if (t == 0) BW_TRACE(i, 13);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // no remote access to either half is pending past this point
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------------------- pre-pass
// Scaled projections of every row of q (side 0) and k (side 1) on every plane of every
// table, z[side][h][l][n][p] = (x_n . W_l[:,p]) (2/tau) / max(|x_n|, eps) (float32, rows
// padded to zstride, zero past N), and inv[side][h][n] = 1 / max(|x_n|, eps).
// One 128-row tile per iteration: TMA x tile (128B swizzle, two slots: the next tile loads
// while this one's epilogue runs) -> tcgen05 (A = x, B = W as a bf16 hi + lo pair in the
// 16 columns of each table, N = 16 L in tiles of at most 256) -> tensor memory -> 128
// threads, one row each, four tables per round of loads.  160 threads; warp 4 issues.
constexpr int kZpThreads = 160;

__host__ __device__ inline int zproj_cols(int L) { return 16 * L <= 256 ? 256 : 512; }
inline size_t zproj_smem(int L) {
  const size_t need = 2 * 16384 + (size_t)64 * 16 * L * 2 + 64 + 1024;
  // at most 512 / cols CTAs per SM, so that tensor-memory allocation never waits
  const size_t one_per_sm = 232448 / 2 + 1024;
  return zproj_cols(L) == 512 ? std::max(need, one_per_sm) : std::max(need, (size_t)232448 / 3 + 1024);
}

__global__ void __launch_bounds__(kZpThreads, 1)
    k_bwd_zproj(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const float* __restrict__ W, int64_t w_hs, float* __restrict__ z,
                float* __restrict__ inv, int64_t N, int H, int L, int64_t zstride,
                float two_over_tau) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  constexpr uint32_t kX = 0, kW = 32768;                   // x: two 16 KB slots
  const int NC = 16 * L;                                   // B columns
  const uint32_t bars = kW + (uint32_t)64 * NC * 2;
  // 0, 1: x tile slots; 2: MMA done; 3: epilogue done reading (tensor memory, x slot)
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + bars + 32);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, side = blockIdx.z;
  const int cols = zproj_cols(L);
  W += (size_t)h * w_hs;
  if (threadIdx.x == 0) {
    mbar_init(bar + 0, 1);
    mbar_init(bar + 1, 1);
    mbar_init(bar + 2, 1);
    mbar_init(bar + 3, 4);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, cols);
    tmem_relinquish();
  }
  // B operand [K = 64][N = 16 L], K-major core matrices: column 16 l + p = W_hi, 16 l + 8 + p
  // = W_lo of plane p of table l
  for (int e = threadIdx.x; e < 64 * NC; e += kZpThreads) {
    const int nn = e / 64, kd = e % 64;
    const int ll = nn >> 4, p = nn & 7;
    const float wv = W[((size_t)ll * 64 + kd) * 8 + p];
    const __nv_bfloat16 hi = __float2bfloat16_rn(wv);
    const __nv_bfloat16 v = (nn & 8) ? __float2bfloat16_rn(wv - __bfloat162float(hi)) : hi;
    const uint32_t off = (nn >> 3) * 1024 + (kd >> 3) * 128 + (nn & 7) * 16 + (kd & 7) * 2;
    *reinterpret_cast<__nv_bfloat16*>(sm + kW + off) = v;
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t tiles = (N + kC - 1) / kC;
  const CUtensorMap* tx = side ? &tk : &tq;
  const int64_t first = blockIdx.x, step = gridDim.x;
  const int its = first < tiles ? (int)((tiles - 1 - first) / step + 1) : 0;
  bool ok = true;
  if (warp == 4) {
    auto load = [&](int it) {
      if (elect_one()) {
        mbar_arrive_expect_tx(bar + (it & 1), 16384);
        tma_load_3d(sm + kX + (it & 1) * 16384, tx, 0, (int)((first + (int64_t)it * step) * kC),
                    h, bar + (it & 1));
      }
      __syncwarp();
    };
    if (its > 0) load(0);
    for (int it = 0; it < its && ok; ++it) {
      // the epilogue of tile it-1 has read the tensor memory and x slot (it+1) % 2
      if (it >= 1) {
        ok = mbar_wait(bar + 3, (uint32_t)(it - 1) & 1);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      if (it + 1 < its) load(it + 1);
      ok = mbar_wait(bar + (it & 1), (uint32_t)(it >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t xs = sb + kX + (it & 1) * 16384;
        for (int nt = 0; nt < NC; nt += 256) {
          const int nw = NC - nt < 256 ? NC - nt : 256;
          const uint32_t id = idesc_bf16(128, nw, 0, 0);
#pragma unroll
          for (int s = 0; s < 4; ++s)
            umma_ss(tmem + nt, sdesc(xs + s * 32, 16, 1024, kSwizzle128B),
                    sdesc(sb + kW + nt * 128 + s * 256, 128, 1024, kSwizzleNone), id, s > 0);
        }
        umma_commit(bar + 2);
      }
      __syncwarp();
    }
  } else {
    const int t = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    for (int it = 0; it < its; ++it) {
      const int64_t row = (first + (int64_t)it * step) * kC + t;
      // the x tile (TMA) for the norms, the projections (MMA) in tensor memory
      if (!mbar_wait(bar + (it & 1), (uint32_t)(it >> 1) & 1) ||
          !mbar_wait(bar + 2, (uint32_t)it & 1))
        break;
      tc_fence_after();
      const float iv = row_inv_norm(sm + kX + (it & 1) * 16384, t);
      const float sc = iv * two_over_tau;
      for (int l4 = 0; l4 < L; l4 += 4) {   // four tables per round of loads
        uint32_t r[4][16];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (l4 + j < L) tmem_ld16(tmem + lane_off + (l4 + j) * 16, r[j]);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (l4 + j < L) {
            float o[8];
#pragma unroll
            for (int p = 0; p < 8; ++p)
              o[p] = (__uint_as_float(r[j][p]) + __uint_as_float(r[j][8 + p])) * sc;
            float4* dst = reinterpret_cast<float4*>(
                z + ((((size_t)side * H + h) * L + l4 + j) * zstride + row) * 8);
            dst[0] = make_float4(o[0], o[1], o[2], o[3]);
            dst[1] = make_float4(o[4], o[5], o[6], o[7]);
          }
        }
      }
      inv[((size_t)side * H + h) * zstride + row] = iv;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + 3);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, cols);
  }
}

// 3-D view [H][N][16] of the extra feature columns of g' (bf16, 32-byte rows): boxes of
// 16 columns x 128 rows, 32-byte swizzle (atom 4 of a feature tile); rows past N read 0.
inline bool encode_gext_tmap(CUtensorMap* m, const void* base, int64_t N, int H) {
  const auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[3] = {16, (cuuint64_t)N, (cuuint64_t)H};
  cuuint64_t strides[2] = {32, (cuuint64_t)N * 32};
  cuuint32_t box[3] = {16, (cuuint32_t)kC, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// gext[h][n] = [e_hi, e_lo, 0, ...] with e = gdot[h][n] = e_hi + e_lo (two bf16 values).
__global__ void k_bwd_gext(const float* __restrict__ gdot, __nv_bfloat16* __restrict__ gext,
                           int64_t rows) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows) return;
  const float e = gdot[i];
  const float e_hi = __bfloat162float(__float2bfloat16_rn(e));
  uint4* dst = reinterpret_cast<uint4*>(gext + i * 16);
  dst[0] = make_uint4(pack_bf16(e_hi, e - e_hi), 0u, 0u, 0u);
  dst[1] = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace tc
}  // namespace race

// Pipelined non-causal readout for R < 256 (P = 6, 7): the same arithmetic as
// k_sketch<P, kReadout> (num += p(q) S over a 256-row group, S the totals of the sequence,
// [JA] §2.1 reconstruction; [IT] §3 non-causal kernel), with the corner expansion of chunk
// c+1 on CUDA cores overlapping the readout MMA of chunk c and the output of chunk c-1.
//
// One CTA per (segment, 256-row group, head), 448 threads:
//   warp 12 (issuer P): TMA copies of the q tiles (two slots) and PROJ(c) = q (W_hi + W_lo)
//            into one of two tensor-memory slots
//   warp 13 (issuer R): RO(c) = p(q) S_bf16 into one of two NUM accumulators
//   warps 0-7  (EXP): warp w expands the tables of half w / 4 of the row group for the 32
//            tokens of lane quarter w % 4 into one of two p(q) tiles
//   warps 8-11 (OUT): NUM rows of chunk c added to the float32 accumulators of the head
//            (the sum over row groups), columns 0-64
// Every producer/consumer pair has its own mbarrier, two-slot resources have a barrier per
// slot, and every wait is bounded.
#pragma once

#include "tc_kernels.cuh"

namespace race {
namespace tc {

constexpr int kRPipeThreads = 448;

enum RdBar : int {
  rd_Q0 = 0, rd_Q1, rd_PROJ0, rd_PROJ1, rd_PRD0, rd_PRD1, rd_PHI0, rd_PHI1, rd_RO0, rd_RO1,
  rd_NF0, rd_NF1, rd_COUNT
};

struct RdSmem {
  static constexpr uint32_t q = 0;            // two 128 x 64 bf16 tiles, 128B swizzle
  static constexpr uint32_t p = 32768;        // two 128 tokens x 256 rows, core-matrix layout
  static constexpr uint32_t sbf = 163840;     // S as bf16, 256 x 80, core-matrix layout
  static constexpr uint32_t whi = 204800;     // 64 x 32 bf16 projection operand
  static constexpr uint32_t wlo = 208896;
  static constexpr uint32_t bars = 212992;
  static constexpr uint32_t tmem_slot = bars + 8 * rd_COUNT;
  static constexpr uint32_t total = tmem_slot + 16;
  static constexpr uint32_t alloc = total + 1024;
};
static_assert(RdSmem::alloc <= 232448, "shared memory budget of one CTA");

struct RdTm {   // tensor-memory columns
  static constexpr uint32_t NUM = 0, PJ = 192;   // NUM: two slots of 96; PJ: two of 32
};

template <int P>
__global__ void __launch_bounds__(kRPipeThreads, 1)
    k_readout_pipe(const __grid_constant__ CUtensorMap tq, const float* __restrict__ W,
                   const float* __restrict__ init, float* __restrict__ num, Params prm) {
  constexpr int R = 1 << P;
  constexpr int TABLES = 256 / R;
  constexpr int TH = TABLES / 2;                    // tables per half of the row group
  static_assert(TH >= 1, "two halves of whole tables");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + RdSmem::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + RdSmem::tmem_slot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, rg = blockIdx.y, h = blockIdx.z;
  const int np = prm.np;
  const int64_t s0 = (int64_t)g * prm.seg_len;
  const int64_t s1 = min64(prm.N, s0 + prm.seg_len);
  const int n = (int)((s1 - s0 + kC - 1) / kC);
  const int l0 = rg * TABLES;
  W += (size_t)h * prm.w_hs;

  if (threadIdx.x == 0) {
    for (int i = 0; i < rd_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i >= rd_PRD0 && i <= rd_PHI1) cnt = 8;     // EXP warps
      if (i == rd_NF0 || i == rd_NF1) cnt = 4;       // OUT warps
      mbar_init(bar + i, cnt);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  // projection operand [K = 64][N = np], W split into bf16 hi + lo
  for (int e = threadIdx.x; e < 64 * np; e += kRPipeThreads) {
    const int nn = e / 64, kd = e % 64;
    float w = 0.f;
    if (nn < TABLES * P) w = W[((size_t)(l0 + nn / P) * 64 + kd) * P + (nn % P)];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
    const uint32_t off = (nn >> 3) * 1024 + (kd >> 3) * 128 + (nn & 7) * 16 + (kd & 7) * 2;
    *reinterpret_cast<__nv_bfloat16*>(sm + RdSmem::whi + off) = hi;
    *reinterpret_cast<__nv_bfloat16*>(sm + RdSmem::wlo + off) = lo;
  }
  // the totals of the row group as the bf16 B operand of the readout
  {
    const float* init_cta = init + (((size_t)h * prm.n_rg + rg) * prm.G + g) * (size_t)256 * kNV;
    for (int row = threadIdx.x; row < 256; row += kRPipeThreads) {
      float vals[kNV];
#pragma unroll
      for (int c = 0; c < kNV; ++c) vals[c] = init_cta[(size_t)row * kNV + c];
      store_state_row_bf16(sb + RdSmem::sbf, row, vals);
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  bool ok = true;
  auto wait = [&](int b, uint32_t par) {
    if (ok && !mbar_wait(bar + b, par)) ok = false;
    ok = __all_sync(0xffffffffu, ok);
    return ok;
  };
  auto t0_of = [&](int c) { return (int)(s0 + (int64_t)c * kC); };

  if (warp == 12) {
    // ================================================================ issuer P
    const uint32_t id_proj = idesc_bf16(128, np, 0, 0);
    auto load_q = [&](int c) {
      const int st = c & 1;
      mbar_arrive_expect_tx(bar + rd_Q0 + st, 16384);
      tma_load_3d(sm + RdSmem::q + st * 16384, &tq, 0, t0_of(c), h, bar + rd_Q0 + st);
    };
    if (n > 0 && elect_one()) {
      prefetch_tmap(&tq);
      load_q(0);
      if (n > 1) load_q(1);
    }
    __syncwarp();
    for (int c = 0; c < n && ok; ++c) {
      const int st = c & 1;
      // PROJ(c), once the EXP warps have read PROJ(c-2) from the same slot
      if (!wait(rd_Q0 + st, (uint32_t)(c >> 1) & 1)) break;
      if (c >= 2 && !wait(rd_PRD0 + st, (uint32_t)((c - 2) >> 1) & 1)) break;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t qt = sb + RdSmem::q + st * 16384;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t a = sdesc(qt + s * 32, 16, 1024, kSwizzle128B);
          umma_ss(tmem + RdTm::PJ + st * 32, a,
                  sdesc(sb + RdSmem::whi + s * 256, 128, 1024, kSwizzleNone), id_proj, s > 0);
          umma_ss(tmem + RdTm::PJ + st * 32, a,
                  sdesc(sb + RdSmem::wlo + s * 256, 128, 1024, kSwizzleNone), id_proj, 1);
        }
        umma_commit(bar + rd_PROJ0 + st);
      }
      __syncwarp();
      // q of chunk c+1 into the slot of chunk c-1 once the EXP warps have read that tile
      if (c >= 1 && c + 1 < n) {
        if (!wait(rd_PRD0 + ((c - 1) & 1), (uint32_t)((c - 1) >> 1) & 1)) break;
        if (elect_one()) load_q(c + 1);
        __syncwarp();
      }
    }
  } else if (warp == 13) {
    // ================================================================ issuer R
    const uint32_t id_read = idesc_bf16(128, kNV, 0, 1);
    for (int c = 0; c < n && ok; ++c) {
      const int st = c & 1;
      if (!wait(rd_PHI0 + st, (uint32_t)(c >> 1) & 1)) break;
      if (c >= 2 && !wait(rd_NF0 + st, (uint32_t)((c - 2) >> 1) & 1)) break;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t pt = sb + RdSmem::p + st * 65536;
#pragma unroll
        for (int s = 0; s < 16; ++s)
          umma_ss(tmem + RdTm::NUM + st * 96, sdesc(pt + s * 256, 128, 256 * 16, kSwizzleNone),
                  sdesc(sb + RdSmem::sbf + s * 2560, 1280, 128, kSwizzleNone), id_read, s > 0);
        umma_commit(bar + rd_RO0 + st);
      }
      __syncwarp();
    }
  } else if (warp < 8) {
    // ================================================================ EXP
    const int q4 = warp & 3, hw = warp >> 2;
    const int t = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    for (int c = 0; c < n; ++c) {
      const int st = c & 1;
      const float valid = (s0 + (int64_t)c * kC + t) < s1 ? 1.f : 0.f;
      if (!wait(rd_PROJ0 + st, (uint32_t)(c >> 1) & 1)) break;
      tc_fence_after();
      // this half's TH tables of projections, register-indexed (hw selects, no local array)
      float u[TH * P];
      {
        uint32_t r[32];
        tmem_ld16(tmem + lane_off + RdTm::PJ + st * 32, r);
        if (np > 16) tmem_ld16(tmem + lane_off + RdTm::PJ + st * 32 + 16, r + 16);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < TH * P; ++e)
          u[e] = __uint_as_float(hw ? r[(TH * P + e) & 31] : r[e]);
      }
      const float sc = row_inv_norm(sm + RdSmem::q + st * 16384, t) * prm.two_over_tau;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + rd_PRD0 + st);
      // p(q) tile slot free once RO(c-2) has read it
      if (c > 1 && !wait(rd_RO0 + st, (uint32_t)((c - 2) >> 1) & 1)) break;
      const uint32_t tile = sb + RdSmem::p + st * 65536 + (uint32_t)((hw * TH * R) / 8) * 128;
      write_phi_rows<P>(tile, t, 256, TH, u, sc, valid);
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + rd_PHI0 + st);
    }
  } else {
    // ================================================================ OUT
    const int q4 = warp - 8;
    const int t = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    float* num_h = num + (size_t)h * prm.N * kNumStride;
    for (int c = 0; c < n; ++c) {
      const int st = c & 1;
      const int64_t row = s0 + (int64_t)c * kC + t;
      if (!wait(rd_RO0 + st, (uint32_t)(c >> 1) & 1)) break;
      tc_fence_after();
      float acc[kNV];
      tmem_ld80(tmem + lane_off + RdTm::NUM + st * 96, acc);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + rd_NF0 + st);
      if (row < s1 && RACE_IN_RANGE(row, prm.N)) {
        float* dst = num_h + row * kNumStride;
#pragma unroll
        for (int cc = 0; cc < 64; cc += 4)
          red_add_v4(dst + cc, acc[cc], acc[cc + 1], acc[cc + 2], acc[cc + 3]);
        atomicAdd(dst + 64, acc[64]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace tc
}  // namespace race

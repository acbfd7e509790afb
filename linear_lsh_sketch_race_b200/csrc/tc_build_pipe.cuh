// Pipelined segment sums of the sketch state for R < 256 (P = 6, 7): the same arithmetic as
// k_sketch<P, kBuild> (S = sum over a segment's keys of p(k)^T [v | 1], two accumulators
// of 128 sketch rows, [JA] §2.1 aggregation; segments feed the prefix scan of the causal
// sweep or the totals of the non-causal readout, [JA] §2.2), with the corner expansion of
// chunk c+1 on CUDA cores overlapping the state update of chunk c on the tensor core.
//
// One CTA per (segment, 256-row group, head), 320 threads:
//   warp 8 (issuer U): UPD(c): S_h += p_h(k)^T [v | 1] for the two halves h of the row group
//   warp 9 (issuer P): TMA copies (k tiles in two slots, v tiles in three) and PROJ(c+1) =
//            k (W_hi + W_lo) into one of two tensor-memory slots; its waits for free
//            slots never hold up the state updates
//   warps 0-7 (EXP): warp w expands the tables of half w / 4 of the row group for the 32
//            tokens of lane quarter w % 4 into one of two p(k) tiles; warps 0-3 then write
//            the segment's state to global memory
// Every producer/consumer pair has its own mbarrier, two- and three-slot resources have a
// barrier per slot, and every wait is bounded.
#pragma once

#include "tc_kernels.cuh"

namespace race {
namespace tc {

constexpr int kBPipeThreads = 320;

enum BldBar : int {
  bl_K0 = 0, bl_K1, bl_V0, bl_V1, bl_V2, bl_VF0, bl_VF1, bl_VF2, bl_PROJ0, bl_PROJ1, bl_PRD0,
  bl_PRD1, bl_PHI0, bl_PHI1, bl_UPD0, bl_UPD1, bl_FIN, bl_COUNT
};

struct BldSmem {
  static constexpr uint32_t k = 0;            // two 128 x 64 bf16 tiles, 128B swizzle
  static constexpr uint32_t v = 32768;        // three
  static constexpr uint32_t p = 81920;        // two 128 tokens x 256 rows, core-matrix layout
  static constexpr uint32_t whi = 212992;     // 64 x 32 bf16 projection operand
  static constexpr uint32_t wlo = 217088;
  static constexpr uint32_t ones = 221184;    // 16 x 16 bf16 ones
  static constexpr uint32_t bars = 221696;
  static constexpr uint32_t tmem_slot = bars + 8 * bl_COUNT;
  static constexpr uint32_t total = tmem_slot + 16;
  static constexpr uint32_t alloc = total + 1024;
};
static_assert(BldSmem::alloc <= 232448, "shared memory budget of one CTA");

struct BldTm {   // tensor-memory columns
  static constexpr uint32_t S0 = 0, S1 = 96, PJ = 192;   // PJ: two slots of 32 columns
};

template <int P>
__global__ void __launch_bounds__(kBPipeThreads, 1)
    k_build_pipe(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                 const float* __restrict__ W, float* __restrict__ seg_out,
                 const float* __restrict__ kscale, Params prm) {
  constexpr int R = 1 << P;
  constexpr int TABLES = 256 / R;
  constexpr int TH = TABLES / 2;                    // tables per half of the row group
  static_assert(TH >= 1, "two halves of whole tables");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + BldSmem::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + BldSmem::tmem_slot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, rg = blockIdx.y, h = blockIdx.z;
  const int np = prm.np;
  const int64_t s0 = (int64_t)g * prm.seg_len;
  const int64_t s1 = min64(prm.N, s0 + prm.seg_len);
  const int n = (int)((s1 - s0 + kC - 1) / kC);
  const int l0 = rg * TABLES;
  W += (size_t)h * prm.w_hs;

  if (threadIdx.x == 0) {
    for (int i = 0; i < bl_COUNT; ++i)
      mbar_init(bar + i, (i >= bl_PRD0 && i <= bl_PHI1) ? 8 : 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  // projection operand [K = 64][N = np], W split into bf16 hi + lo; a 16 x 16 ones block
  for (int e = threadIdx.x; e < 64 * np; e += kBPipeThreads) {
    const int nn = e / 64, kd = e % 64;
    float w = 0.f;
    if (nn < TABLES * P) w = W[((size_t)(l0 + nn / P) * 64 + kd) * P + (nn % P)];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
    const uint32_t off = (nn >> 3) * 1024 + (kd >> 3) * 128 + (nn & 7) * 16 + (kd & 7) * 2;
    *reinterpret_cast<__nv_bfloat16*>(sm + BldSmem::whi + off) = hi;
    *reinterpret_cast<__nv_bfloat16*>(sm + BldSmem::wlo + off) = lo;
  }
  for (int e = threadIdx.x; e < 256; e += kBPipeThreads)
    reinterpret_cast<__nv_bfloat16*>(sm + BldSmem::ones)[e] = __float2bfloat16_rn(1.0f);
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the segment sums start from zero
  if (warp < 4) {
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    uint32_t z[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) z[e] = 0u;
#pragma unroll
    for (int b = 0; b < 5; ++b) {
      tmem_st16(tmem + lane_off + BldTm::S0 + b * 16, z);
      tmem_st16(tmem + lane_off + BldTm::S1 + b * 16, z);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  bool ok = true;
  auto wait = [&](int b, uint32_t par) {
    if (ok && !mbar_wait(bar + b, par)) ok = false;
    ok = __all_sync(0xffffffffu, ok);
    return ok;
  };
  auto t0_of = [&](int c) { return (int)(s0 + (int64_t)c * kC); };

  auto load_k = [&](int c) {   // one elected thread
    const int st = c & 1;
    mbar_arrive_expect_tx(bar + bl_K0 + st, 16384);
    tma_load_3d(sm + BldSmem::k + st * 16384, &tk, 0, t0_of(c), h, bar + bl_K0 + st);
  };
  auto load_v = [&](int c) {
    const int sv = c % 3;
    mbar_arrive_expect_tx(bar + bl_V0 + sv, 16384);
    tma_load_3d(sm + BldSmem::v + sv * 16384, &tv, 0, t0_of(c), h, bar + bl_V0 + sv);
  };
  if (warp == 9) {
    // ================================================================ issuer P
    const uint32_t id_proj = idesc_bf16(128, np, 0, 0);
    auto proj = [&](int c) {   // PROJ(c) into tensor-memory slot c % 2
      const int st = c & 1;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t kt = sb + BldSmem::k + st * 16384;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t a = sdesc(kt + s * 32, 16, 1024, kSwizzle128B);
          umma_ss(tmem + BldTm::PJ + st * 32, a,
                  sdesc(sb + BldSmem::whi + s * 256, 128, 1024, kSwizzleNone), id_proj, s > 0);
          umma_ss(tmem + BldTm::PJ + st * 32, a,
                  sdesc(sb + BldSmem::wlo + s * 256, 128, 1024, kSwizzleNone), id_proj, 1);
        }
        umma_commit(bar + bl_PROJ0 + st);
      }
      __syncwarp();
    };
    if (n > 0 && elect_one()) {
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
      for (int c = 0; c < 3 && c < n; ++c) load_v(c);
      load_k(0);
      if (n > 1) load_k(1);
    }
    __syncwarp();
    for (int c = 0; c < n && ok; ++c) {
      const int st = c & 1;
      // PROJ(c), once the EXP warps have read PROJ(c-2) from the same slot
      if (!wait(bl_K0 + st, (uint32_t)(c >> 1) & 1)) break;
      if (c >= 2 && !wait(bl_PRD0 + st, (uint32_t)((c - 2) >> 1) & 1)) break;
      proj(c);
      // k of chunk c+1 into the slot of chunk c-1 once the EXP warps have read that tile
      if (c >= 1 && c + 1 < n) {
        if (!wait(bl_PRD0 + ((c - 1) & 1), (uint32_t)((c - 1) >> 1) & 1)) break;
        if (elect_one()) load_k(c + 1);
        __syncwarp();
      }
      // v of chunk c+2 into the slot of chunk c-1 once UPD(c-1) has read it
      if (c >= 1 && c + 2 < n) {
        if (!wait(bl_VF0 + ((c - 1) % 3), (uint32_t)((c - 1) / 3) & 1)) break;
        if (elect_one()) load_v(c + 2);
        __syncwarp();
      }
    }
  } else if (warp == 8) {
    // ================================================================ issuer U
    const uint32_t id_up = idesc_bf16(128, 64, 1, 1);
    const uint32_t id_up1 = idesc_bf16(128, 16, 1, 1);
    const uint64_t d_ones = sdesc(sb + BldSmem::ones, 256, 128, kSwizzleNone);
    for (int c = 0; c < n && ok; ++c) {
      const int st = c & 1, sv = c % 3;
      if (!wait(bl_V0 + sv, (uint32_t)(c / 3) & 1) || !wait(bl_PHI0 + st, (uint32_t)(c >> 1) & 1))
        break;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t pt = sb + BldSmem::p + st * 65536;
        const uint32_t vt = sb + BldSmem::v + sv * 16384;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const uint32_t dS = tmem + (mt ? BldTm::S1 : BldTm::S0);
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            const uint64_t a = sdesc(pt + mt * 2048 + s * 32 * 256, 256 * 16, 128, kSwizzleNone);
            umma_ss(dS, a, sdesc(vt + s * 2048, 8192, 1024, kSwizzle128B), id_up, 1);
            umma_ss(dS + 64, a, d_ones, id_up1, 1);
          }
        }
        umma_commit(bar + bl_UPD0 + st);
        umma_commit(bar + bl_VF0 + sv);
        if (c + 1 == n) umma_commit(bar + bl_FIN);
      }
      __syncwarp();
    }
  } else {
    // ================================================================ EXP
    const int q4 = warp & 3, hw = warp >> 2;
    const int t = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    auto kfac = [&](int c) {   // row factor of the key (0 past the end)
      const int64_t row = s0 + (int64_t)c * kC + t;
      return row < s1 ? (kscale ? kscale[(size_t)h * prm.N + row] : 1.f) : 0.f;
    };
    float kf_next = n > 0 ? kfac(0) : 0.f;
    for (int c = 0; c < n; ++c) {
      const int st = c & 1;
      const float kf = kf_next;
      if (c + 1 < n) kf_next = kfac(c + 1);
      if (!wait(bl_PROJ0 + st, (uint32_t)(c >> 1) & 1)) break;
      tc_fence_after();
      // this half's TH tables of projections, register-indexed (hw selects, no local array)
      float u[TH * P];
      {
        uint32_t r[32];
        tmem_ld16(tmem + lane_off + BldTm::PJ + st * 32, r);
        if (np > 16) tmem_ld16(tmem + lane_off + BldTm::PJ + st * 32 + 16, r + 16);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < TH * P; ++e)
          u[e] = __uint_as_float(hw ? r[(TH * P + e) & 31] : r[e]);
      }
      const float sc = row_inv_norm(sm + BldSmem::k + st * 16384, t) * prm.two_over_tau;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + bl_PRD0 + st);
      // p(k) tile slot free once UPD(c-2) has read it
      if (c > 1 && !wait(bl_UPD0 + st, (uint32_t)((c - 2) >> 1) & 1)) break;
      const uint32_t tile = sb + BldSmem::p + st * 65536 + (uint32_t)((hw * TH * R) / 8) * 128;
      write_phi_rows<P>(tile, t, 256, TH, u, sc, kf);
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + bl_PHI0 + st);
    }
    if (warp < 4 && ok) {
      if (n == 0 || wait(bl_FIN, 0)) {   // an empty segment writes zeros
        tc_fence_after();
        float* out = seg_out + (((size_t)h * prm.n_rg + rg) * prm.G + g) * (size_t)256 * kNV;
        for (int mt = 0; mt < 2; ++mt) {
          float vals[kNV];
          tmem_ld80(tmem + lane_off + (mt ? BldTm::S1 : BldTm::S0), vals);
          float4* o4 = reinterpret_cast<float4*>(out + (size_t)(mt * 128 + t) * kNV);
#pragma unroll
          for (int cc = 0; cc < kNV / 4; ++cc)
            o4[cc] = make_float4(vals[4 * cc], vals[4 * cc + 1], vals[4 * cc + 2], vals[4 * cc + 3]);
        }
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

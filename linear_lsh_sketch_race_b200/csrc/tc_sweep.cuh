// Pipelined causal sweep on tensor cores (one CTA per head, 256-row group of the
// sketch and segment of the sequence).  Same arithmetic as k_sketch<..., kSweep>;
// what changes is the schedule:
//
//   * warps 0-3 hash q and warps 4-7 hash k (one token per thread, TMEM lane = token);
//     warp 8 issues TMA copies and tcgen05 MMAs from one thread;
//   * the 256 sketch rows are handled as two halves of 128 rows with their own
//     barriers, so the MMAs of one half (in-chunk QK, readout, state update) run
//     while the CUDA cores expand the other half;
//   * the q/k tiles of the next chunk are fetched as soon as the projections and
//     norms of the current chunk have been read; the v tile once the last MMA that
//     reads it has completed;
//   * the readout accumulator is released by the output epilogue and the bf16
//     state halves by the restage step, each through its own barrier.
//
// Causal prefix state ([JA] §2.2 prefix sums), bucket aggregation and readout
// ([JA] §2.1), soft hash as products of per-plane logistic factors.
#pragma once

#include "tc_kernels.cuh"

namespace race {
namespace tc {

constexpr int kSwThreads = 288;

// Optional phase timeline of CTA (0,0,0), compiled in with -DRACE_SWEEP_TRACE: clock64
// stamps per chunk and event, read back through race_sweep_trace_read().
#ifdef RACE_SWEEP_TRACE
constexpr int kTraceChunks = 512, kTraceEvents = 40;
// rows 0-511: forward sweep; rows 512-1023: backward sweep steps
__device__ unsigned long long g_sweep_trace[2 * kTraceChunks * kTraceEvents];
#define SW_TRACE(c, ev)                                                                 \
  do {                                                                                  \
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && (c) < kTraceChunks)    \
      g_sweep_trace[(c) * kTraceEvents + (ev)] = clock64();                              \
  } while (0)
// Per-CTA record in row = linear CTA index: 25 SM id, 26/27 global timer at start/end,
// 38/39 clock64 at start/end.
__device__ __forceinline__ void sw_trace_cta(bool end) {
  const int row = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  if (threadIdx.x != 0 || row >= kTraceChunks) return;
  unsigned long long gt;
  unsigned int sm;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(gt));
  asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
  unsigned long long* r = g_sweep_trace + row * kTraceEvents;
  r[end ? 27 : 26] = gt;
  r[end ? 39 : 38] = clock64();
  r[25] = sm;
}
#define SW_TRACE_CTA(end) sw_trace_cta(end)
#define BW_TRACE(c, ev)                                                                 \
  do {                                                                                  \
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && (c) < kTraceChunks)    \
      g_sweep_trace[(kTraceChunks + (c)) * kTraceEvents + (ev)] = clock64();             \
  } while (0)
#else
#define SW_TRACE(c, ev) \
  do {                  \
  } while (0)
#define SW_TRACE_CTA(end) \
  do {                    \
  } while (0)
#define BW_TRACE(c, ev) \
  do {                  \
  } while (0)
#endif

enum SwBar : int {
  kB_QKFULL = 0, kB_VFULL, kB_PROJ, kB_QKFREE, kB_PHQ0, kB_PHQ1, kB_PHK0, kB_PHK1,
  kB_HALF0, kB_HALF1, kB_QKDONE, kB_INTRA, kB_AV, kB_SBF0, kB_SBF1, kB_NUMFREE, kB_COUNT
};

// Shared memory: the k_sketch map up to its barriers; 16 barriers and the TMEM base
// address follow.
struct SwSmem {
  static constexpr uint32_t bars = Smem::bars;
  static constexpr uint32_t tmem_slot = bars + 8 * kB_COUNT;
  static constexpr uint32_t total = tmem_slot + 16;
  static constexpr uint32_t alloc = total + 1024;
};
static_assert(SwSmem::alloc <= 232448, "shared memory budget of one CTA");

struct SwTm {
  static constexpr uint32_t S0 = 0, S1 = 80, num = 160, qk = 256, pq = 384, pk = 416,
                            intra = 448;
};

// 1/max(|x|, eps) of token row t of a 128-byte-swizzled 128 x 64 bf16 tile.  Thread t
// starts at chunk t % 8 so that the eight threads of a shared-memory phase touch
// eight different 16-byte bank groups.
__device__ __forceinline__ float row_inv_norm_rot(const uint8_t* tile, int t) {
  const uint4* row = reinterpret_cast<const uint4*>(tile + t * 128);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint4 w = row[(i + t) & 7];
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ws[e]));
      s = fmaf(f.x, f.x, fmaf(f.y, f.y, s));
    }
  }
  return 1.0f / fmaxf(sqrtf(s), kEpsNorm);
}

__device__ __forceinline__ void store_chunk(uint32_t addr, float h, const float* lo) {
  st_shared_v4(addr, pack_bf16(h * lo[0], h * lo[1]), pack_bf16(h * lo[2], h * lo[3]),
               pack_bf16(h * lo[4], h * lo[5]), pack_bf16(h * lo[6], h * lo[7]));
}

// Expand sketch rows [128*HALF, 128*HALF + 128) of one token into the core-matrix tile
// (256 rows: core (token/8, row/8) at (token/8)*4096 + (row/8)*128).  sp/sm hold the
// logistic pair of every plane of the CTA's tables; a row's value is the product over
// planes of sp (bit set) or sm (bit clear).
template <int P, int TABLES, int HALF>
__device__ __forceinline__ void expand_half(uint32_t tile, int t, const float* sp,
                                            const float* sm, float valid) {
  constexpr int R = 1 << P;
  const uint32_t base = tile + (t >> 3) * 4096 + (t & 7) * 16 + HALF * 16 * 128;
  if constexpr (TABLES == 1) {
    // R = 256: the half is fixed by the top plane (plane 7)
    float lo[8];
#pragma unroll
    for (int b = 0; b < 8; ++b)
      lo[b] = ((b & 1) ? sp[0] : sm[0]) * ((b & 2) ? sp[1] : sm[1]) * ((b & 4) ? sp[2] : sm[2]);
    float hi[16];
    hi[0] = valid * (HALF ? sp[P - 1] : sm[P - 1]);
    kron_tree<3, P - 1>(hi, sp, sm);
#pragma unroll
    for (int c = 0; c < 16; ++c) store_chunk(base + c * 128, hi[c], lo);
  } else {
    constexpr int TH = TABLES / 2;  // whole tables per half
#pragma unroll
    for (int jj = 0; jj < TH; ++jj) {
      const int j = HALF * TH + jj;
      const float* a = sp + j * P;
      const float* b_ = sm + j * P;
      float lo[8];
#pragma unroll
      for (int b = 0; b < 8; ++b)
        lo[b] = ((b & 1) ? a[0] : b_[0]) * ((b & 2) ? a[1] : b_[1]) * ((b & 4) ? a[2] : b_[2]);
      float hi[R / 8];
      hi[0] = valid;
      kron_tree<3, P>(hi, a, b_);
#pragma unroll
      for (int c = 0; c < R / 8; ++c) store_chunk(base + (jj * (R / 8) + c) * 128, hi[c], lo);
    }
  }
}

template <int P, int TABLES>
__global__ void __launch_bounds__(kSwThreads, 1)
    k_sweep(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
            const __grid_constant__ CUtensorMap tv, const float* __restrict__ W,
            const float* __restrict__ init, float* __restrict__ num,
            const float* __restrict__ kscale, Params prm) {
  constexpr int R = 1 << P;
  constexpr int NPL = TABLES * P;               // planes of the CTA
  constexpr int NP = ((NPL + 15) / 16) * 16;    // projection columns
  static_assert(R * TABLES == 256, "k_sweep handles 256-row groups");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + SwSmem::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SwSmem::tmem_slot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, rg = blockIdx.y, h = blockIdx.z;
  const int64_t s0 = (int64_t)g * prm.seg_len;
  const int64_t s1 = min64(prm.N, s0 + prm.seg_len);
  const int nchunks = (int)((s1 - s0 + kC - 1) / kC);
  const int l0 = rg * TABLES;
  W += (size_t)h * prm.w_hs;   // this head's hash planes

  if (threadIdx.x == 0) {
    for (int i = 0; i < kB_COUNT; ++i)
      mbar_init(bar + i, (i == kB_QKFREE || i == kB_INTRA || i == kB_NUMFREE) ? 2 : 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (threadIdx.x < 256) {
    const int t = threadIdx.x;
    for (int e = t; e < 64 * NP; e += 256) {
      const int n = e / 64, kd = e % 64;
      float w = 0.f;
      if (n < NPL) w = W[((size_t)(l0 + n / P) * 64 + kd) * P + (n % P)];
      const __nv_bfloat16 hi = __float2bfloat16_rn(w);
      const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
      const uint32_t off = (n >> 3) * 1024 + (kd >> 3) * 128 + (n & 7) * 16 + (kd & 7) * 2;
      *reinterpret_cast<__nv_bfloat16*>(sm + Smem::whi + off) = hi;
      *reinterpret_cast<__nv_bfloat16*>(sm + Smem::wlo + off) = lo;
    }
    for (int e = t; e < 256; e += 256)
      reinterpret_cast<__nv_bfloat16*>(sm + Smem::ones)[e] = __float2bfloat16_rn(1.0f);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // initial state: warps 0-3 own state rows 0-127 (S0), warps 4-7 rows 128-255 (S1)
  if (threadIdx.x < 256) {
    const int hf = warp >> 2;
    const int t = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float* src = init + (((size_t)h * prm.n_rg + rg) * prm.G + g) * 256 * kNV +
                       (size_t)(hf * 128 + t) * kNV;
    float vals[kNV];
#pragma unroll
    for (int c = 0; c < kNV; ++c) vals[c] = prm.have_init ? src[c] : 0.f;
    uint32_t r[16];
#pragma unroll
    for (int b = 0; b < 5; ++b) {
#pragma unroll
      for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(vals[b * 16 + e]);
      tmem_st16(tmem + lane_off + (hf ? SwTm::S1 : SwTm::S0) + b * 16, r);
    }
    tmem_st_wait();
    store_state_row_bf16(sb + Smem::sbf, hf * 128 + t, vals);
    fence_proxy_async();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {  // phase 0 of the "state staged" and "accumulator free" barriers
    mbar_arrive(bar + kB_SBF0);
    mbar_arrive(bar + kB_SBF1);
    mbar_arrive(bar + kB_NUMFREE);
    mbar_arrive(bar + kB_NUMFREE);
  }

  if (warp == 8) {
    // ================================================================ issuer
    if (lane == 0) {
      prefetch_tmap(&tq);
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
      const uint32_t id_proj = idesc_bf16(128, NP, 0, 0);
      const uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
      const uint32_t id_read = idesc_bf16(128, kNV, 0, 1);
      const uint32_t id_av = idesc_bf16(128, 64, 0, 1);
      const uint32_t id_av1 = idesc_bf16(128, 16, 0, 1);
      const uint32_t id_up = idesc_bf16(128, 64, 1, 1);
      const uint32_t id_up1 = idesc_bf16(128, 16, 1, 1);
      const uint64_t d_ones = sdesc(sb + Smem::ones, 256, 128, kSwizzleNone);
      bool ok = true;
      if (nchunks > 0) {
        mbar_arrive_expect_tx(bar + kB_QKFULL, 32768);
        tma_load_3d(sm + Smem::q, &tq, 0, (int)s0, h, bar + kB_QKFULL);
        tma_load_3d(sm + Smem::k, &tk, 0, (int)s0, h, bar + kB_QKFULL);
        mbar_arrive_expect_tx(bar + kB_VFULL, 16384);
        tma_load_3d(sm + Smem::v, &tv, 0, (int)s0, h, bar + kB_VFULL);
      }
      auto wait = [&](int b, uint32_t par) {
        if (ok && !mbar_wait(bar + b, par)) ok = false;
        return ok;
      };
      for (int c = 0; c < nchunks && ok; ++c) {
        const uint32_t par = c & 1;
        const int t0 = (int)(s0 + (int64_t)c * kC);
        SW_TRACE(c, 0);
        if (!wait(kB_QKFULL, par)) break;
        SW_TRACE(c, 1);
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t bh = sdesc(sb + Smem::whi + s * 256, 128, 1024, kSwizzleNone);
          const uint64_t bl = sdesc(sb + Smem::wlo + s * 256, 128, 1024, kSwizzleNone);
          const uint64_t aq = sdesc(sb + Smem::q + s * 32, 16, 1024, kSwizzle128B);
          const uint64_t ak = sdesc(sb + Smem::k + s * 32, 16, 1024, kSwizzle128B);
          umma_ss(tmem + SwTm::pq, aq, bh, id_proj, s > 0);
          umma_ss(tmem + SwTm::pq, aq, bl, id_proj, 1);
          umma_ss(tmem + SwTm::pk, ak, bh, id_proj, s > 0);
          umma_ss(tmem + SwTm::pk, ak, bl, id_proj, 1);
        }
        umma_commit(bar + kB_PROJ);
        if (c > 0) {  // the v tile of chunk c-1 is free once its last reader (AV) completed
          if (!wait(kB_AV, par ^ 1)) break;
          SW_TRACE(c, 2);
          mbar_arrive_expect_tx(bar + kB_VFULL, 16384);
          tma_load_3d(sm + Smem::v, &tv, 0, t0, h, bar + kB_VFULL);
        }
        // ---------------- half 0: rows 0-127
        if (!wait(kB_PHQ0, par) || !wait(kB_PHK0, par)) break;
        SW_TRACE(c, 3);
        if (!wait(kB_SBF0, par) || !wait(kB_NUMFREE, par)) break;
        SW_TRACE(c, 4);
        if (!wait(kB_VFULL, par)) break;
        SW_TRACE(c, 5);
        tc_fence_after();
        for (int s = 0; s < 8; ++s)
          umma_ss(tmem + SwTm::qk, sdesc(sb + Smem::phq + s * 256, 128, 4096, kSwizzleNone),
                  sdesc(sb + Smem::phk + s * 256, 128, 4096, kSwizzleNone), id_qk, s > 0);
        for (int s = 0; s < 8; ++s)
          umma_ss(tmem + SwTm::num, sdesc(sb + Smem::phq + s * 256, 128, 4096, kSwizzleNone),
                  sdesc(sb + Smem::sbf + s * 2560, 1280, 128, kSwizzleNone), id_read, s > 0);
        for (int s = 0; s < 8; ++s) {
          const uint64_t a = sdesc(sb + Smem::phk + s * 8192, 4096, 128, kSwizzleNone);
          const uint64_t bv = sdesc(sb + Smem::v + s * 2048, 8192, 1024, kSwizzle128B);
          umma_ss(tmem + SwTm::S0, a, bv, id_up, 1);
          umma_ss(tmem + SwTm::S0 + 64, a, d_ones, id_up1, 1);
        }
        umma_commit(bar + kB_HALF0);
        // q/k tiles of chunk c are free once projections and norms were read
        if (!wait(kB_QKFREE, par)) break;
        SW_TRACE(c, 6);
        if (c + 1 < nchunks) {
          mbar_arrive_expect_tx(bar + kB_QKFULL, 32768);
          tma_load_3d(sm + Smem::q, &tq, 0, t0 + kC, h, bar + kB_QKFULL);
          tma_load_3d(sm + Smem::k, &tk, 0, t0 + kC, h, bar + kB_QKFULL);
        }
        // ---------------- half 1: rows 128-255
        if (!wait(kB_PHQ1, par) || !wait(kB_PHK1, par)) break;
        SW_TRACE(c, 7);
        if (!wait(kB_SBF1, par)) break;
        SW_TRACE(c, 8);
        tc_fence_after();
        for (int s = 8; s < 16; ++s)
          umma_ss(tmem + SwTm::qk, sdesc(sb + Smem::phq + s * 256, 128, 4096, kSwizzleNone),
                  sdesc(sb + Smem::phk + s * 256, 128, 4096, kSwizzleNone), id_qk, 1);
        umma_commit(bar + kB_QKDONE);
        for (int s = 8; s < 16; ++s)
          umma_ss(tmem + SwTm::num, sdesc(sb + Smem::phq + s * 256, 128, 4096, kSwizzleNone),
                  sdesc(sb + Smem::sbf + s * 2560, 1280, 128, kSwizzleNone), id_read, 1);
        for (int s = 0; s < 8; ++s) {
          const uint64_t a = sdesc(sb + Smem::phk + 2048 + s * 8192, 4096, 128, kSwizzleNone);
          const uint64_t bv = sdesc(sb + Smem::v + s * 2048, 8192, 1024, kSwizzle128B);
          umma_ss(tmem + SwTm::S1, a, bv, id_up, 1);
          umma_ss(tmem + SwTm::S1 + 64, a, d_ones, id_up1, 1);
        }
        umma_commit(bar + kB_HALF1);
        // ---------------- masked in-chunk term
        if (!wait(kB_INTRA, par)) break;
        SW_TRACE(c, 9);
        tc_fence_after();
        for (int s = 0; s < 8; ++s) {
          const uint64_t bv = sdesc(sb + Smem::v + s * 2048, 8192, 1024, kSwizzle128B);
          umma_ts(tmem + SwTm::num, tmem + SwTm::intra + s * 8, bv, id_av, 1);
          umma_ts(tmem + SwTm::num + 64, tmem + SwTm::intra + s * 8, d_ones, id_av1, 1);
        }
        umma_commit(bar + kB_AV);
      }
      if (ok && nchunks > 0) wait(kB_AV, (nchunks - 1) & 1);
    }
  } else {
    // ================================================================ CUDA-core warps
    const int grp = warp >> 2;                 // 0: q side, 1: k side
    const int t = (warp & 3) * 32 + lane;      // token row = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int nbar = 1 + grp;                  // named barrier of this group
    const uint8_t* tile = sm + (grp ? Smem::k : Smem::q);
    const uint32_t ph_tile = sb + (grp ? Smem::phk : Smem::phq);
    const uint32_t tm_proj = tmem + lane_off + (grp ? SwTm::pk : SwTm::pq);
    float* num_h = num + (size_t)h * prm.N * kNumStride;
    bool ok = true;
    auto wait = [&](int b, uint32_t par) {
      if (ok && !mbar_wait(bar + b, par)) ok = false;
      return ok;
    };
    for (int c = 0; c < nchunks && ok; ++c) {
      const uint32_t par = c & 1;
      const int64_t t0 = s0 + (int64_t)c * kC;
      const float valid = (t0 + t) < s1 ? 1.f : 0.f;
      // factor of the expanded corner probabilities: 0 past the end; on the k side the
      // optional per-key factor
      const float fac = (grp && kscale && valid != 0.f) ? kscale[(size_t)h * prm.N + t0 + t]
                                                       : valid;
      // ---- projections and norms
      [[maybe_unused]] const int eb = 10 + 15 * grp;   // trace events of this group
      if (t == 0) SW_TRACE(c, eb + 0);
      if (!wait(kB_PROJ, par)) break;
      if (t == 0) SW_TRACE(c, eb + 1);
      tc_fence_after();
      const float scale = row_inv_norm_rot(tile, t) * prm.two_over_tau;
      float u[NP];
      uint32_t r[16];
#pragma unroll
      for (int b = 0; b < NP / 16; ++b) {
        tmem_ld16(tm_proj + b * 16, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) u[b * 16 + e] = __uint_as_float(r[e]);
      }
      tc_fence_before();
      named_bar(nbar, 128);
      if (t == 0) mbar_arrive(bar + kB_QKFREE);
      float sp[NPL], sm_[NPL];
#pragma unroll
      for (int n = 0; n < NPL; ++n) logistic_fast(u[n] * scale, sp[n], sm_[n]);
      // ---- soft-hash rows, half by half
      if (t == 0) SW_TRACE(c, eb + 2);
      if (c > 0 && !wait(kB_HALF0, par ^ 1)) break;
      if (t == 0) SW_TRACE(c, eb + 3);
      expand_half<P, TABLES, 0>(ph_tile, t, sp, sm_, fac);
      fence_proxy_async();
      named_bar(nbar, 128);
      if (t == 0) mbar_arrive(bar + (grp ? kB_PHK0 : kB_PHQ0));
      if (t == 0) SW_TRACE(c, eb + 4);
      if (c > 0 && !wait(kB_HALF1, par ^ 1)) break;
      if (t == 0) SW_TRACE(c, eb + 5);
      expand_half<P, TABLES, 1>(ph_tile, t, sp, sm_, fac);
      fence_proxy_async();
      named_bar(nbar, 128);
      if (t == 0) mbar_arrive(bar + (grp ? kB_PHK1 : kB_PHQ1));
      // ---- masked in-chunk weights: key columns [64*grp, 64*grp + 64)
      if (t == 0) SW_TRACE(c, eb + 6);
      if (!wait(kB_QKDONE, par)) break;
      if (t == 0) SW_TRACE(c, eb + 7);
      tc_fence_after();
#pragma unroll
      for (int cb = 4 * grp; cb < 4 * grp + 4; ++cb) {
        tmem_ld16(tmem + lane_off + SwTm::qk + cb * 16, r);
        tmem_ld_wait();
        uint32_t pk8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j0 = cb * 16 + 2 * e;
          const float a0 = (j0 <= t) ? __uint_as_float(r[2 * e]) : 0.f;
          const float a1 = (j0 + 1 <= t) ? __uint_as_float(r[2 * e + 1]) : 0.f;
          pk8[e] = pack_bf16(a0, a1);
        }
        tmem_st8(tmem + lane_off + SwTm::intra + cb * 8, pk8);
      }
      tmem_st_wait();
      tc_fence_before();
      named_bar(nbar, 128);
      if (t == 0) mbar_arrive(bar + kB_INTRA);
      // ---- bf16 copy of state half grp for the next chunk's readout
      if (t == 0) SW_TRACE(c, eb + 8);
      if (!wait(grp ? kB_HALF1 : kB_HALF0, par)) break;
      if (t == 0) SW_TRACE(c, eb + 9);
      tc_fence_after();
      {
        float vals[kNV];
        tmem_ld80(tmem + lane_off + (grp ? SwTm::S1 : SwTm::S0), vals);
        store_state_row_bf16(sb + Smem::sbf, grp * 128 + t, vals);
      }
      fence_proxy_async();
      tc_fence_before();
      named_bar(nbar, 128);
      if (t == 0) mbar_arrive(bar + (grp ? kB_SBF1 : kB_SBF0));
      // ---- output rows: sum over row groups in global float32 accumulators
      if (t == 0) SW_TRACE(c, eb + 10);
      if (!wait(kB_AV, par)) break;
      if (t == 0) SW_TRACE(c, eb + 11);
      tc_fence_after();
      {
        float acc[40];
        uint32_t rr[16];
        const uint32_t col = SwTm::num + grp * 40;
        tmem_ld16(tmem + lane_off + col, rr);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = __uint_as_float(rr[e]);
        tmem_ld16(tmem + lane_off + col + 16, rr);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[16 + e] = __uint_as_float(rr[e]);
        tmem_ld8(tmem + lane_off + col + 32, rr);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[32 + e] = __uint_as_float(rr[e]);
        tc_fence_before();
        named_bar(nbar, 128);
        if (t == 0) mbar_arrive(bar + kB_NUMFREE);
        if (valid != 0.f) {
          float* dst = num_h + (t0 + t) * kNumStride + grp * 40;
          if (grp == 0) {
#pragma unroll
            for (int e = 0; e < 40; e += 4)
              red_add_v4(dst + e, acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
          } else {
#pragma unroll
            for (int e = 0; e < 24; e += 4)
              red_add_v4(dst + e, acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
            atomicAdd(dst + 24, acc[24]);
          }
        }
      }
      if (t == 0) SW_TRACE(c, eb + 12);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace race

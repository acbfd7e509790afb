// Causal sweep with the CUDA-core work of chunk c + 1 overlapping the MMAs of chunk c;
// one table per CTA (R = 256 buckets, P = 8 planes), the shape of the long-context
// workload.  Soft bucketization, bucket aggregation and readout: [JA] §2.1; causal
// prefix state: [JA] §2.2.
//
// Tensor-core work of chunk c, in two streams issued by two warps (one elected lane each):
//
//   warp 16: QK(c)        p(q) p(k)^T over 256 buckets   -> QK   (A: p(q) in tensor memory)
//            RO(c)        p(q) S_bf16                     -> NUM  (then p(q) is free)
//            AV(c)        mask(QK) [v | 1]                -> NUM
//   warp 17: PROJ_Q(c+1)  u_q = x_q (W_hi + W_lo)        -> PROJ (16 tensor-memory columns)
//            UPD(c)       S_h += p(k)_h^T [v | 1], h = 0, 1 -> S0, S1
//            PROJ_K(c+2)  u_k                             -> PROJ
//
// The waits and bookkeeping of one stream are covered by the other's MMAs: the tensor
// core's queue holds only a few tens of cycles of work ahead of a single issuer.
//
// CUDA-core warp groups (one warp per tensor-memory lane quadrant each):
//   warps 0-3   expand p(q) of chunk c+1 into tensor memory once RO(c) has read p(q);
//   warps 4-7   expand p(k) of chunk c+1 into one of three 32 KB half-buffers
//               (bucket halves; a half-buffer is free once both QK and the state update
//               that read it have completed);
//   warps 8-11  mask QK(c) and round it to bf16 in place; bf16 copy of S for RO(c+1);
//   warps 12-15 move NUM rows to the float32 output accumulators (TMA reduce-add).
// Every producer/consumer pair has its own mbarrier; a producer can be at most one
// phase ahead of its consumer, so parity waits stay unambiguous.  An optional per-key
// factor kscale[h][n] multiplies p(k_n) (the backward's dv pass uses the keys' 1/den').
//
// NVC is the width of the value side of every MMA: 80 = the 64 value columns and an atom
// of ones whose first column accumulates the mass z (the forward, which needs the
// denominator), or 64 = the values alone (the dv pass, which reads only the numerator;
// its denominator column is written as zero).
#pragma once

#include "tc_sweep256.cuh"

namespace race {
namespace tc {

constexpr int kSPThreads = 576;

enum SPBar : int {
  sp_QT = 0, sp_KT, sp_VT0, sp_VT1,
  sp_PROJK_FULL, sp_PROJK_READ, sp_PROJQ_FULL, sp_PROJQ_READ,
  sp_PHQ0, sp_PHQ1, sp_PHK0, sp_PHK1, sp_PHK2, sp_KFREE0, sp_KFREE1, sp_KFREE2,
  sp_KFREEA0, sp_KFREEA1, sp_KFREEA2,
  sp_QK_FULL, sp_CONV, sp_PQ_FREE, sp_UPD0, sp_UPD1, sp_SREAD0, sp_SREAD1, sp_SBF,
  sp_AV_DONE, sp_NUMFREE, sp_RO_ISSUED,
  sp_COUNT
};

struct SPSmem {
  static constexpr uint32_t qt = 0, kt = 16384;            // x tiles, 128 x 64 bf16, 128B swizzle
  static constexpr uint32_t vt0 = 32768, vt1 = 49152;      // v tiles (two stages)
  static constexpr uint32_t pk = 65536;                     // 3 half-buffers of p(k), 32 KB each
  static constexpr uint32_t sbf = 163840;                   // state bf16, 32B swizzle, 40 KB
  static constexpr uint32_t w = 204800;                     // [64 x 16] bf16 hi | lo
  static constexpr uint32_t ones = 206848;                  // second atom of [v | 1]
  static constexpr uint32_t invq = 208896, invk = 209408;   // 1/|x| of the chunk's rows
  static constexpr uint32_t stage = 209920;                 // 64 rows x 68 f32
  static constexpr uint32_t bars = 227328;
  static constexpr uint32_t tmem_slot = bars + 8 * sp_COUNT;
  static constexpr uint32_t total = tmem_slot + 16;
  static constexpr uint32_t alloc = total + 1024;
};
static_assert(SPSmem::alloc <= 232448, "shared memory budget of one CTA");
static_assert(SPSmem::stage + 64 * kNumStride * 4 <= SPSmem::bars, "staging overlaps barriers");

// Tensor-memory columns.  QK (fp32, 128 keys) is rounded in place to bf16 pairs in its
// first 64 columns, the A operand of AV.  p(q) holds bucket pairs (2i, 2i+1) in column i.
struct SPTm {
  static constexpr uint32_t S0 = 0, S1 = 80, num = 160, qk = 240, pq = 368, proj = 496;
};


// bf16 copy of the NVC-column state row held in tensor-memory lane (this thread) at
// column `col`: two batches of loads (48 + NVC - 48 columns), one wait each, packed to
// NVC / 2 bf16 pairs.  After this returns the tensor-memory row may be overwritten.
template <int NVC>
__device__ __forceinline__ void restage_load(uint32_t taddr, uint32_t* pk) {
  static_assert(NVC == 64 || NVC == 80, "value width");
  uint32_t v[48];
  tmem_ld16(taddr, v);
  tmem_ld16(taddr + 16, v + 16);
  tmem_ld16(taddr + 32, v + 32);
  tmem_ld_wait();
#pragma unroll
  for (int e = 0; e < 24; ++e) pk[e] = pack_bf16(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
#pragma unroll
  for (int b = 0; b < (NVC - 48) / 16; ++b) tmem_ld16(taddr + 48 + 16 * b, v + 16 * b);
  tmem_ld_wait();
#pragma unroll
  for (int e = 0; e < (NVC - 48) / 2; ++e)
    pk[24 + e] = pack_bf16(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
}

// Row r of the 32B-swizzled readout operand (see store_state_row_sw32) from NVC / 2 bf16
// pairs (one 16-column atom per 8 pairs).
template <int NVC>
__device__ __forceinline__ void restage_store(uint32_t sbf, int r, const uint32_t* pk) {
  const uint32_t rb = sbf + (r >> 3) * 256 + (r & 7) * 32;
  const uint32_t flip = (r >> 2) & 1;
#pragma unroll
  for (int a = 0; a < NVC / 16; ++a)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const uint32_t* x = pk + a * 8 + hh * 4;
      st_shared_v4(rb + a * 8192 + ((hh ^ flip) << 4), x[0], x[1], x[2], x[3]);
    }
}

// Corner probabilities of one token in factored form: bucket b = 8c + e, c = 4g + j,
// p_b = lo[e] * p34[j] * h5(g), with lo over planes 0-2, p34 over planes 3-4 and h5 over
// planes 5-7 chosen by the bits of g (the product over planes of the logistic factor of
// the corner's side of each plane).  Loops over g stay rolled, which keeps the code of the
// expanding warps small.
struct Corners {
  float lo[8];
  float p34[4];
  float f5[2], f6[2], f7[2];
  uint64_t lo2[4];   // float pairs (lo[2e], lo[2e+1]) in one 64-bit register
};

__device__ __forceinline__ void corners_of(const float* sp, const float* sm, float valid,
                                           Corners& k) {
#pragma unroll
  for (int b = 0; b < 8; ++b)
    k.lo[b] = ((b & 1) ? sp[0] : sm[0]) * ((b & 2) ? sp[1] : sm[1]) * ((b & 4) ? sp[2] : sm[2]);
#pragma unroll
  for (int j = 0; j < 4; ++j) k.p34[j] = valid * ((j & 1) ? sp[3] : sm[3]) * ((j & 2) ? sp[4] : sm[4]);
  k.f5[0] = sm[5]; k.f5[1] = sp[5];
  k.f6[0] = sm[6]; k.f6[1] = sp[6];
  k.f7[0] = sm[7]; k.f7[1] = sp[7];
#pragma unroll
  for (int e = 0; e < 4; ++e) k.lo2[e] = pair_f32x2(k.lo[2 * e], k.lo[2 * e + 1]);
}
__device__ __forceinline__ float corners_h5(const Corners& k, int g) {
  return ((g & 1) ? k.f5[1] : k.f5[0]) * ((g & 2) ? k.f6[1] : k.f6[0]) *
         ((g & 4) ? k.f7[1] : k.f7[0]);
}

template <int NVC>
__global__ void __launch_bounds__(kSPThreads, 1)
    k_sweep_pipe(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                 const __grid_constant__ CUtensorMap tv, const float* __restrict__ W,
                 const float* __restrict__ init, const float* __restrict__ inv_norms,
                 int64_t inv_stride, const __grid_constant__ CUtensorMap tnum,
                 float* __restrict__ num, const float* __restrict__ kscale, Params prm) {
  constexpr int P = 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + SPSmem::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SPSmem::tmem_slot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, l0 = blockIdx.y, h = blockIdx.z;
  const int64_t s0 = (int64_t)g * prm.seg_len;
  const int64_t s1 = min64(prm.N, s0 + prm.seg_len);
  const int n = (int)((s1 - s0 + kC - 1) / kC);
  W += (size_t)h * prm.w_hs;   // this head's hash planes

  if (threadIdx.x == 0) {
    for (int i = 0; i < sp_COUNT; ++i) {
      const bool by_warps = i == sp_PHQ0 ||
                            i == sp_PHQ1 || (i >= sp_PHK0 && i <= sp_PHK2) || i == sp_CONV ||
                            i == sp_SBF || i == sp_NUMFREE || i == sp_SREAD0 ||
                            i == sp_SREAD1;
      mbar_init(bar + i, by_warps ? 4 : 1);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (threadIdx.x < 256) {
    // projection operand [K = 64 dims][N = 16]: columns 0-7 W_hi planes, 8-15 W_lo planes
    for (int e = threadIdx.x; e < 64 * 16; e += 256) {
      const int nn = e / 64, kd = e % 64;
      const float w = W[((size_t)l0 * 64 + kd) * P + (nn & 7)];
      const __nv_bfloat16 hi = __float2bfloat16_rn(w);
      const __nv_bfloat16 v = nn < 8 ? hi : __float2bfloat16_rn(w - __bfloat162float(hi));
      const uint32_t off = (nn >> 3) * 1024 + (kd >> 3) * 128 + (nn & 7) * 16 + (kd & 7) * 2;
      *reinterpret_cast<__nv_bfloat16*>(sm + SPSmem::w + off) = v;
    }
    for (int e = threadIdx.x; e < 1024; e += 256)
      reinterpret_cast<__nv_bfloat16*>(sm + SPSmem::ones)[e] = __float2bfloat16_rn(1.0f);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (threadIdx.x < 256) {  // initial state: warps 0-3 rows 0-127 (S0), warps 4-7 rows 128-255
    const int hf = warp >> 2;
    const int t = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float* src = init + (((size_t)h * prm.n_rg + l0) * prm.G + g) * 256 * kNV +
                       (size_t)(hf * 128 + t) * kNV;
    float vals[kNV];
#pragma unroll
    for (int c = 0; c < kNV; ++c) vals[c] = prm.have_init ? src[c] : 0.f;
    uint32_t r[16];
#pragma unroll
    for (int b = 0; b < 5; ++b) {
#pragma unroll
      for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(vals[b * 16 + e]);
      tmem_st16(tmem + lane_off + (hf ? SPTm::S1 : SPTm::S0) + b * 16, r);
    }
    tmem_st_wait();
    store_state_row_sw32(sb + SPSmem::sbf, hf * 128 + t, vals);
    fence_proxy_async();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  SW_TRACE_CTA(false);
  bool ok = true;
  // Warp-uniform bounded wait: a timeout anywhere in the warp ends the warp's loop.
  auto wait = [&](int b, uint32_t par) {
    if (ok && !mbar_wait(bar + b, par)) ok = false;
    ok = __all_sync(0xffffffffu, ok);
    return ok;
  };
  const uint32_t pk_base = sb + SPSmem::pk;

  // TMA copies: q/k tiles (with their 1/|x|) of chunk x+1 are issued by the q/k side
  // once it has read chunk x's projections (single buffer each); v tiles of chunk x+2 by
  // the masking warps once UPD(x) and AV(x) have completed (two stages).
  const float* inv_q = inv_norms + (size_t)h * inv_stride;
  const float* inv_k = inv_norms + ((size_t)prm.H + h) * inv_stride;
  auto t0_of = [&](int c) { return (int)(s0 + (int64_t)c * kC); };
  auto load_q = [&](int c) {   // one thread
    mbar_arrive_expect_tx(bar + sp_QT, 16384 + 512);
    tma_load_3d(sm + SPSmem::qt, &tq, 0, t0_of(c), h, bar + sp_QT);
    bulk_load(sm + SPSmem::invq, inv_q + t0_of(c), 512, bar + sp_QT);
    if (c + 3 < n) tma_prefetch_3d(&tq, 0, t0_of(c + 3), h);
  };
  auto load_k = [&](int c) {   // one thread
    mbar_arrive_expect_tx(bar + sp_KT, 16384 + 512);
    tma_load_3d(sm + SPSmem::kt, &tk, 0, t0_of(c), h, bar + sp_KT);
    bulk_load(sm + SPSmem::invk, inv_k + t0_of(c), 512, bar + sp_KT);
    if (c + 3 < n) tma_prefetch_3d(&tk, 0, t0_of(c + 3), h);
  };
  auto load_v = [&](int c) {   // one thread
    const int st = c & 1;
    mbar_arrive_expect_tx(bar + sp_VT0 + st, 16384);
    tma_load_3d(sm + (st ? SPSmem::vt1 : SPSmem::vt0), &tv, 0, t0_of(c), h, bar + sp_VT0 + st);
    if (c + 3 < n) tma_prefetch_3d(&tv, 0, t0_of(c + 3), h);
  };

  if (warp >= 16) {
    // ================================================================ issuers
    // Two warps issue two independent MMA streams, so that each one's waits and
    // bookkeeping between issue blocks are covered by the other's MMAs (the MMA queue
    // holds only a few tens of cycles of work ahead of a single issuer):
    //   warp 16: QK(c) over the two bucket halves, RO(c), AV(c)       (p(q) side)
    //   warp 17: PROJ_Q(c+1), UPD(c) over the two halves, PROJ_K(c+2) (state, projections)
    // A p(k) half-buffer is free once both QK (warp 16) and UPD (warp 17) have read it;
    // the bf16 state is rewritten only after RO(c) has read it, and UPD(c+1) of a bucket
    // half starts once that half of the state after chunk c has been read out.
    const uint32_t id_proj = idesc_bf16(128, 16, 0, 0);
    const uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
    const uint32_t id_ro = idesc_bf16(128, NVC, 0, 1);   // A tmem (K-major), B MN-major
    const uint32_t id_up = idesc_bf16(128, NVC, 1, 1);   // A MN-major smem, B MN-major
    // Start addresses stay below 2^18 bytes, so adding (bytes >> 4) to a descriptor
    // never carries out of its 14-bit field.
    const uint64_t d_w = sdesc(sb + SPSmem::w, 128, 1024, kSwizzleNone);
    const uint64_t d_ro = sdesc(sb + SPSmem::sbf, 8192, 256, kSwizzle32B);
    const uint64_t d_xq = sdesc(sb + SPSmem::qt, 16, 1024, kSwizzle128B);
    const uint64_t d_xk = sdesc(sb + SPSmem::kt, 16, 1024, kSwizzle128B);
    const uint64_t d_vone0 = sdesc(sb + SPSmem::vt0, SPSmem::ones - SPSmem::vt0, 1024, kSwizzle128B);
    const uint64_t d_vone1 = sdesc(sb + SPSmem::vt1, SPSmem::ones - SPSmem::vt1, 1024, kSwizzle128B);
    const uint64_t vstep = (uint64_t)(2048 >> 4) - ((uint64_t)(2048 >> 4) << 16);
    auto proj = [&](uint64_t dx, int done) {
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int s = 0; s < 4; ++s)
          umma_ss(tmem + SPTm::proj, dx + 2 * s, d_w + 16 * s, id_proj, s > 0);
        umma_commit(bar + done);
      }
      __syncwarp();
    };
    if (warp == 16) {
      for (int c = 0; c < n && ok; ++c) {
        const uint32_t par = c & 1;
        const int i0 = 2 * c, i1 = 2 * c + 1;
        const int b0 = i0 % 3, b1 = i1 % 3;
        const uint32_t m0 = (uint32_t)(i0 / 3), m1 = (uint32_t)(i1 / 3);
        const uint64_t d_vone = (c & 1) ? d_vone1 : d_vone0;
        SW_TRACE(c, 0);
        // ---- in-chunk QK over the two bucket halves
        if (!wait(sp_PHQ0, par) || !wait(sp_PHK0 + b0, m0 & 1)) break;
        SW_TRACE(c, 1);
        tc_fence_after();
        if (elect_one()) {
          const uint64_t d_qk = sdesc(pk_base + b0 * 32768, 16, 1024, kSwizzle128B);
#pragma unroll
          for (int s = 0; s < 8; ++s)
            umma_ts(tmem + SPTm::qk, tmem + SPTm::pq + s * 8,
                    d_qk + (uint64_t)((s >> 2) * 1024 + (s & 3) * 2), id_qk, s > 0);
          umma_commit(bar + sp_KFREEA0 + b0);
        }
        __syncwarp();
        if (!wait(sp_PHQ1, par) || !wait(sp_PHK0 + b1, m1 & 1)) break;
        SW_TRACE(c, 2);
        tc_fence_after();
        if (elect_one()) {
          const uint64_t d_qk = sdesc(pk_base + b1 * 32768, 16, 1024, kSwizzle128B);
#pragma unroll
          for (int s = 0; s < 8; ++s)
            umma_ts(tmem + SPTm::qk, tmem + SPTm::pq + 64 + s * 8,
                    d_qk + (uint64_t)((s >> 2) * 1024 + (s & 3) * 2), id_qk, 1);
          umma_commit(bar + sp_QK_FULL);
          umma_commit(bar + sp_KFREEA0 + b1);
        }
        __syncwarp();
        // ---- readout against the state before the chunk; then p(q) is free
        if (c > 0 && (!wait(sp_SBF, (c - 1) & 1) || !wait(sp_NUMFREE, (c - 1) & 1))) break;
        SW_TRACE(c, 3);
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int s = 0; s < 16; ++s)
            umma_ts(tmem + SPTm::num, tmem + SPTm::pq + s * 8, d_ro + 32 * s, id_ro, s > 0);
          umma_commit(bar + sp_PQ_FREE);
          mbar_arrive(bar + sp_RO_ISSUED);
        }
        __syncwarp();
        // ---- masked in-chunk weights times [v | 1]
        if (!wait(sp_CONV, par) || !wait(sp_VT0 + (c & 1), (c >> 1) & 1)) break;
        SW_TRACE(c, 5);
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int s = 0; s < 8; ++s)
            umma_ts(tmem + SPTm::num, tmem + SPTm::qk + s * 8, d_vone + vstep * s, id_ro, 1);
          umma_commit(bar + sp_AV_DONE);
        }
        __syncwarp();
      }
    } else {
      if (n > 0) {
        if (elect_one()) {
          prefetch_tmap(&tq);
          prefetch_tmap(&tk);
          prefetch_tmap(&tv);
          for (int c = 1; c < 3 && c < n; ++c) {
            tma_prefetch_3d(&tq, 0, t0_of(c), h);
            tma_prefetch_3d(&tk, 0, t0_of(c), h);
            tma_prefetch_3d(&tv, 0, t0_of(c), h);
          }
          load_k(0);
          load_q(0);
          load_v(0);
          if (n > 1) load_v(1);
        }
        __syncwarp();
        // PROJ holds, in turn, PROJ_K(0), PROJ_Q(0), PROJ_K(1), PROJ_Q(1), ...; each fill
        // waits until the previous one was read.
        if (wait(sp_KT, 0)) proj(d_xk, sp_PROJK_FULL);
        if (wait(sp_PROJK_READ, 0) && wait(sp_QT, 0)) proj(d_xq, sp_PROJQ_FULL);
        if (n > 1 && wait(sp_PROJQ_READ, 0) && wait(sp_KT, 1)) proj(d_xk, sp_PROJK_FULL);
      }
      for (int c = 0; c < n && ok; ++c) {
        const int i0 = 2 * c, i1 = 2 * c + 1;
        const int b0 = i0 % 3, b1 = i1 % 3;
        const uint32_t m0 = (uint32_t)(i0 / 3), m1 = (uint32_t)(i1 / 3);
        const uint64_t d_vone = (c & 1) ? d_vone1 : d_vone0;
        // ---- q projections of chunk c+1
        if (c + 1 < n) {
          if (!wait(sp_PROJK_READ, (c + 1) & 1) || !wait(sp_QT, (c + 1) & 1)) break;
          proj(d_xq, sp_PROJQ_FULL);
        }
        // ---- state update, one bucket half per accumulator
        if (!wait(sp_PHK0 + b0, m0 & 1) || !wait(sp_PHK0 + b1, m1 & 1) ||
            !wait(sp_VT0 + (c & 1), (c >> 1) & 1))
          break;
        if (c > 0 && !wait(sp_SREAD0, (c - 1) & 1)) break;
        // the state update queues behind QK(c) and RO(c), which lie on the critical chains
        if (!wait(sp_RO_ISSUED, c & 1)) break;
        SW_TRACE(c, 4);
        tc_fence_after();
        if (elect_one()) {
          const uint64_t d_up0 = sdesc(pk_base + b0 * 32768, 16384, 1024, kSwizzle128B);
#pragma unroll
          for (int s = 0; s < 8; ++s)
            umma_ss(tmem + SPTm::S0, d_up0 + 128 * s, d_vone + vstep * s, id_up, 1);
          umma_commit(bar + sp_UPD0);
          umma_commit(bar + sp_KFREE0 + b0);
        }
        __syncwarp();
        if (c > 0 && !wait(sp_SREAD1, (c - 1) & 1)) break;
        tc_fence_after();
        if (elect_one()) {
          const uint64_t d_up1 = sdesc(pk_base + b1 * 32768, 16384, 1024, kSwizzle128B);
#pragma unroll
          for (int s = 0; s < 8; ++s)
            umma_ss(tmem + SPTm::S1, d_up1 + 128 * s, d_vone + vstep * s, id_up, 1);
          umma_commit(bar + sp_UPD1);
          umma_commit(bar + sp_KFREE0 + b1);
        }
        __syncwarp();
        // ---- k projections of chunk c+2
        if (c + 2 < n) {
          if (!wait(sp_PROJQ_READ, (c + 1) & 1) || !wait(sp_KT, c & 1)) break;
          proj(d_xk, sp_PROJK_FULL);
        }
        SW_TRACE(c, 6);
      }
    }
  } else if (warp < 4) {
    // ================================================================ p(q) of chunk x
    const int t = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    for (int x = 0; x < n; ++x) {
      const uint32_t par = x & 1;
      const bool valid = s0 + (int64_t)x * kC + t < s1;
      if (!wait(sp_QT, par) || !wait(sp_PROJQ_FULL, par)) break;
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(tmem + lane_off + SPTm::proj, r);
      tmem_ld_wait();
      const float inv = reinterpret_cast<const float*>(sm + SPSmem::invq)[t];
      tc_fence_before();
      named_bar(2, 128);            // all four q warps read PROJ and 1/|x| of chunk x
      if (warp == 0 && elect_one()) {
        mbar_arrive(bar + sp_PROJQ_READ);
        if (x + 1 < n) load_q(x + 1);
      }
      __syncwarp();
      if (t == 0) SW_TRACE(x, 10);
      const float scale = valid ? inv * prm.two_over_tau : 0.f;
      float sp[P], smv[P];
#pragma unroll
      for (int p = 0; p < P; ++p)
        logistic_fast((__uint_as_float(r[p]) + __uint_as_float(r[8 + p])) * scale, sp[p], smv[p]);
      Corners k;
      corners_of(sp, smv, valid ? 1.f : 0.f, k);
      if (x > 0 && !wait(sp_PQ_FREE, (x - 1) & 1)) break;
      if (t == 0) SW_TRACE(x, 11);
      tc_fence_after();
      // group g = buckets 32g..32g+31 = tensor-memory columns 16g..16g+15
#pragma unroll 1
      for (int g = 0; g < 8; ++g) {
        const float h5 = corners_h5(k, g);
        uint32_t v16[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t hh = bcast_f32x2(h5 * k.p34[j]);
#pragma unroll
          for (int e = 0; e < 4; ++e) v16[j * 4 + e] = mul_pack_bf16(k.lo2[e], hh);
        }
        tmem_st16(tmem + lane_off + SPTm::pq + 16 * g, v16);
        if ((g & 3) == 3) {        // a bucket half is complete
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar + sp_PHQ0 + (g >> 2));
          if (t == 0) SW_TRACE(x, 12 + (g >> 2));
        }
      }
    }
  } else if (warp < 8) {
    // ================================================================ p(k) of chunk x
    const int t = (warp - 4) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp - 4) * 32) << 16;
    for (int x = 0; x < n; ++x) {
      const uint32_t par = x & 1;
      const bool valid = s0 + (int64_t)x * kC + t < s1;
      // factor of the corner probabilities: 0 past the end, else the optional per-key
      // factor (loaded before the waits, so its latency overlaps them)
      const float kf = valid ? (kscale ? kscale[(size_t)h * prm.N + s0 + (int64_t)x * kC + t]
                                       : 1.f)
                             : 0.f;
      if (!wait(sp_KT, par) || !wait(sp_PROJK_FULL, par)) break;
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(tmem + lane_off + SPTm::proj, r);
      tmem_ld_wait();
      const float inv = reinterpret_cast<const float*>(sm + SPSmem::invk)[t];
      tc_fence_before();
      named_bar(3, 128);            // all four k warps read PROJ and 1/|x| of chunk x
      if (warp == 4 && elect_one()) {
        mbar_arrive(bar + sp_PROJK_READ);
        if (x + 1 < n) load_k(x + 1);
      }
      __syncwarp();
      if (t == 0) SW_TRACE(x, 20);
      const float scale = valid ? inv * prm.two_over_tau : 0.f;
      float sp[P], smv[P];
#pragma unroll
      for (int p = 0; p < P; ++p)
        logistic_fast((__uint_as_float(r[p]) + __uint_as_float(r[8 + p])) * scale, sp[p], smv[p]);
      Corners k;
      corners_of(sp, smv, kf, k);
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const int i = 2 * x + half;
        const int b = i % 3;
        const int m = i / 3;
        if (m >= 1 && (!wait(sp_KFREE0 + b, (uint32_t)(m - 1) & 1) ||
                       !wait(sp_KFREEA0 + b, (uint32_t)(m - 1) & 1)))
          break;
        if (t == 0) SW_TRACE(x, 21 + 2 * half);
        const uint32_t base = pk_base + b * 32768;
#pragma unroll 1
        for (int gg = 0; gg < 4; ++gg) {
          const float h5 = corners_h5(k, 4 * half + gg);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t hh = bcast_f32x2(h5 * k.p34[j]);
            st_shared_v4(phk_addr(base, t, 4 * gg + j), mul_pack_bf16(k.lo2[0], hh),
                         mul_pack_bf16(k.lo2[1], hh), mul_pack_bf16(k.lo2[2], hh),
                         mul_pack_bf16(k.lo2[3], hh));
          }
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar + sp_PHK0 + b);
        if (t == 0) SW_TRACE(x, 22 + 2 * half);
      }
      if (!ok) break;
    }
  } else if (warp < 12) {
    // ================================================================ mask, restage
    const int q4 = warp - 8;
    const int t = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    for (int x = 0; x < n; ++x) {
      const uint32_t par = x & 1;
      if (!wait(sp_QK_FULL, par)) break;
      if (t == 0) SW_TRACE(x, 30);
      tc_fence_after();
      // key block b (keys 32b..32b+31): blocks above this warp's rows are all zero
#pragma unroll 1
      for (int b = 0; b < 4; ++b) {
        uint32_t o[16];
        if (b <= q4) {
          uint32_t f[32];
          tmem_ld16(tmem + lane_off + SPTm::qk + 32 * b, f);
          tmem_ld16(tmem + lane_off + SPTm::qk + 32 * b + 16, f + 16);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int j0 = 32 * b + 2 * e;
            const float a0 = (j0 <= t) ? __uint_as_float(f[2 * e]) : 0.f;
            const float a1 = (j0 + 1 <= t) ? __uint_as_float(f[2 * e + 1]) : 0.f;
            o[e] = pack_bf16(a0, a1);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = 0u;
        }
        tmem_st16(tmem + lane_off + SPTm::qk + 16 * b, o);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + sp_CONV);
      if (t == 0) SW_TRACE(x, 31);
      // State halves: read into registers as soon as UPD(x) has written them (then UPD(x+1)
      // may accumulate again), write the bf16 copy once RO(x) has read the previous one.
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        if (!wait(sp_UPD0 + hf, par)) break;
        tc_fence_after();
        uint32_t pk[NVC / 2];
        restage_load<NVC>(tmem + lane_off + (hf ? SPTm::S1 : SPTm::S0), pk);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar + sp_SREAD0 + hf);
        if (hf == 0 && !wait(sp_PQ_FREE, par)) break;   // RO(x) read the state of chunk x-1
        restage_store<NVC>(sb + SPSmem::sbf, 128 * hf + t, pk);
        if (t == 0) SW_TRACE(x, 32 + hf);
      }
      if (!ok) break;
      fence_proxy_async();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + sp_SBF);
      // v(x) was read by UPD(x) (waited above) and AV(x); v(x+2) takes its stage.  AV(x+1)
      // needs this warp group's CONV(x+1), so AV_DONE cannot run a phase ahead here.
      if (warp == 8 && x + 2 < n) {
        if (!wait(sp_AV_DONE, par)) break;
        if (elect_one()) load_v(x + 2);
        __syncwarp();
      }
    }
  } else {
    // ================================================================ output rows
    // NUM rows go through a 64-row staging buffer and are added to the float32
    // accumulators by TMA tensor reductions (the sum over the tables of a head).
    const int t = (warp - 12) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp - 12) * 32) << 16;
    float* stg = reinterpret_cast<float*>(sm + SPSmem::stage);
    const bool leader = (warp == 12 && lane == 0);
    for (int x = 0; x < n; ++x) {
      const int t0 = (int)(s0 + (int64_t)x * kC);
      if (!wait(sp_AV_DONE, x & 1)) break;
      if (t == 0) SW_TRACE(x, 35);
      tc_fence_after();
      uint32_t acc[72];
#pragma unroll
      for (int b = 0; b < 4; ++b) tmem_ld16(tmem + lane_off + SPTm::num + b * 16, acc + b * 16);
      if (NVC == 80) tmem_ld8(tmem + lane_off + SPTm::num + 64, acc + 64);
      else acc[64] = 0u;   // no denominator column: the dv pass reads the numerator only
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + sp_NUMFREE);
      if (t == 0) SW_TRACE(x, 36);
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        if ((t >> 6) == half) {
          float4* row = reinterpret_cast<float4*>(stg + (t & 63) * kNumStride);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            row[e] = make_float4(__uint_as_float(acc[4 * e]), __uint_as_float(acc[4 * e + 1]),
                                 __uint_as_float(acc[4 * e + 2]), __uint_as_float(acc[4 * e + 3]));
          row[16] = make_float4(__uint_as_float(acc[64]), 0.f, 0.f, 0.f);
          fence_proxy_async();
        }
        named_bar(1, 128);
        if (leader) {
          tma_reduce_add_3d(&tnum, 0, t0 + half * 64, h, stg);
          bulk_commit();
          bulk_wait_read0();
        }
        named_bar(1, 128);
      }
      if (t == 0) SW_TRACE(x, 37);
    }
    if (leader) bulk_wait0();
  }
  tc_fence_before();
  __syncthreads();
  SW_TRACE_CTA(true);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace race

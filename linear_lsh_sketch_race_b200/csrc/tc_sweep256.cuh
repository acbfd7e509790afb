// Causal sweep for one full table per CTA (R = 256 buckets, P = 8 planes): the shape of
// the long-context headline workload.  Differences from k_sweep (tc_sweep.cuh):
//
//   * p(q) lives in tensor memory and is the A operand of the readout MMA (no shared-
//     memory copy, no shared-memory operand reads for it);
//   * the in-chunk QK = p(q) p(k)^T reads p(q) from tensor memory and p(k) from shared
//     memory; its fp32 result is masked and rounded to bf16 in place in tensor memory
//     (each warp group converts the key columns it later owns, so no group overwrites
//     columns the other still has to read);
//   * q/k/v tiles are double-buffered (two TMA stages);
//   * 1/|x| comes from a pre-pass (k_inv_norms) and travels with the q/k tiles as a
//     bulk copy;
//   * a separate warp group moves output rows to the global accumulators, so the
//     hashing warps never wait on the atomics.
//
// Warps 0-3: q side (hash q, expand p(q) into TMEM, in-chunk weights of keys 0-63,
// bf16 copy of state half 0).  Warps 4-7: k side (hash k, expand p(k) into shared
// memory, in-chunk weights of keys 64-127, state half 1).  Warps 8-11: output epilogue.
// Warp 12: TMA and tcgen05 issue (one thread).
// Soft bucketization and aggregation: [JA] §2.1; causal prefix: [JA] §2.2.
#pragma once

#include "tc_sweep.cuh"

namespace race {
namespace tc {

constexpr int kS8Threads = 416;

enum S8Bar : int {
  k8_QKFULL0 = 0, k8_QKFULL1, k8_VFULL0, k8_VFULL1, k8_PROJ, k8_PROJFREE, k8_PHQ, k8_PHK0,
  k8_PHK1, k8_QKDONE, k8_CONV, k8_HALF0, k8_HALF1, k8_AV, k8_SBF0, k8_SBF1, k8_NUMFREE,
  k8_COUNT
};

struct S8Smem {
  static constexpr uint32_t q0 = 0, k0 = 16384, v0 = 32768;       // stage 0 tiles
  static constexpr uint32_t q1 = 49152, k1 = 65536, v1 = 81920;   // stage 1 tiles
  static constexpr uint32_t phk = 98304;    // p(k): 4 atoms (64 buckets) x 128 tokens x 128 B, 128B swizzle
  static constexpr uint32_t sbf = 163840;   // state bf16, 5 atoms (16 columns) x 256 rows x 32 B, 32B swizzle
  static constexpr uint32_t w = 204800;     // [64 x 16] bf16 hi|lo
  static constexpr uint32_t ones = 206848;  // 16 rows x 128 B of bf16 ones (second atom of [v | 1])
  static constexpr uint32_t inv0 = 208896;  // [2][128] f32, stage 0
  static constexpr uint32_t inv1 = 209920;  // stage 1
  static constexpr uint32_t stage = 210944; // 64 output rows x 68 f32 (TMA reduce source)
  static constexpr uint32_t bars = 228352;
  static constexpr uint32_t tmem_slot = bars + 8 * k8_COUNT;
  static constexpr uint32_t total = tmem_slot + 16;
  static constexpr uint32_t alloc = total + 1024;
};
static_assert(S8Smem::alloc <= 232448, "shared memory budget of one CTA");

// Tensor memory.  qk holds the in-chunk QK (fp32, 128 columns); after masking, keys
// 0-63 become bf16 A-operand columns qk+0..31 and keys 64-127 columns qk+64..95.  The
// projections of the next chunk land in the last 32 columns of the p(q) region (rows
// 192-255 of p(q)) as soon as the QK of this chunk has read p(q); the q side writes
// those rows of the next p(q) only after both sides have read the projections.
struct S8Tm {
  static constexpr uint32_t S0 = 0, S1 = 80, num = 160, phq = 240, pq = 336, pk = 352,
                            qk = 368, intraA = 368, intraB = 432;
};

// 1/max(|x|, eps) of every row of q and k into out[side][h][stride] (side 0: q, 1: k);
// grid (ceil(N/256), 2*H).  Entries stride - N .. of each head are never written and
// never used (they pad the last chunk so it can be bulk-copied whole).
__global__ void k_inv_norms(const __nv_bfloat16* __restrict__ q,
                            const __nv_bfloat16* __restrict__ k, float* __restrict__ out,
                            int64_t N, int H, int64_t stride) {
  const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int sh = blockIdx.y;                 // side * H + head
  if (n >= N) return;
  const int side = sh >= H, h = sh - side * H;
  const __nv_bfloat16* x = (side ? k : q) + ((size_t)h * N + n) * kD;
  const uint4* r = reinterpret_cast<const uint4*>(x);
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 w = __ldg(r + c);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ws[e]));
      s = fmaf(f.x, f.x, fmaf(f.y, f.y, s));
    }
  }
  out[(size_t)sh * stride + n] = 1.0f / fmaxf(sqrtf(s), kEpsNorm);
}

// Expand the 256 corner probabilities of one token: bucket b = 8*c + e has value
// hi[c] * lo[e], with lo over planes 0-2 and hi over planes 3-7.
__device__ __forceinline__ void corner_factors(const float* sp, const float* sm, float valid,
                                               float* lo, float* hi) {
#pragma unroll
  for (int b = 0; b < 8; ++b)
    lo[b] = ((b & 1) ? sp[0] : sm[0]) * ((b & 2) ? sp[1] : sm[1]) * ((b & 4) ? sp[2] : sm[2]);
  hi[0] = valid;
  kron_tree<3, 8>(hi, sp, sm);
}

// p(k) chunk c (buckets 8c..8c+7) of token t in the 128B-swizzled tile: atom c/8 of
// 64 buckets, 8-token groups of 1 KB, 16-byte chunk index XOR token%8.
__device__ __forceinline__ uint32_t phk_addr(uint32_t base, int t, int c) {
  return base + (c >> 3) * 16384 + (t >> 3) * 1024 + (t & 7) * 128 +
         ((((c & 7) ^ (t & 7))) << 4);
}

// bf16 copy of state row r (80 columns) as the readout B operand: MN-major with 32-byte
// swizzle, atom a = columns 16a..16a+15 at a*8 KB, 8-row groups of 256 B, the two 16-byte
// halves of a 32-byte row swapped on rows 4-7 of each group.
__device__ __forceinline__ void store_state_row_sw32(uint32_t sbf, int r, const float* v) {
  const uint32_t rb = sbf + (r >> 3) * 256 + (r & 7) * 32;
  const uint32_t flip = (r >> 2) & 1;
#pragma unroll
  for (int a = 0; a < 5; ++a)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const float* x = v + a * 16 + hh * 8;
      st_shared_v4(rb + a * 8192 + ((hh ^ flip) << 4), pack_bf16(x[0], x[1]),
                   pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
    }
}

__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, int x, int y, int z,
                                                  const void* src) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%1, %2, %3}], [%4];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(z), "r"(smem_u32(src))
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__global__ void __launch_bounds__(kS8Threads, 1)
    k_sweep256(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, const float* __restrict__ W,
               const float* __restrict__ init, const float* __restrict__ inv_norms,
               int64_t inv_stride, const __grid_constant__ CUtensorMap tnum, Params prm) {
  constexpr int P = 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + S8Smem::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + S8Smem::tmem_slot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, l0 = blockIdx.y, h = blockIdx.z;
  const int64_t s0 = (int64_t)g * prm.seg_len;
  const int64_t s1 = min64(prm.N, s0 + prm.seg_len);
  const int nchunks = (int)((s1 - s0 + kC - 1) / kC);

  if (threadIdx.x == 0) {
    for (int i = 0; i < k8_COUNT; ++i)
      mbar_init(bar + i, (i == k8_PROJFREE || i == k8_CONV) ? 2 : 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (threadIdx.x < 256) {
    // projection operand [K = 64 dims][N = 16]: columns 0-7 W_hi planes, 8-15 W_lo planes
    for (int e = threadIdx.x; e < 64 * 16; e += 256) {
      const int n = e / 64, kd = e % 64;
      const float w = W[((size_t)l0 * 64 + kd) * P + (n & 7)];
      const __nv_bfloat16 hi = __float2bfloat16_rn(w);
      const __nv_bfloat16 v = n < 8 ? hi : __float2bfloat16_rn(w - __bfloat162float(hi));
      const uint32_t off = (n >> 3) * 1024 + (kd >> 3) * 128 + (n & 7) * 16 + (kd & 7) * 2;
      *reinterpret_cast<__nv_bfloat16*>(sm + S8Smem::w + off) = v;
    }
    for (int e = threadIdx.x; e < 1024; e += 256)
      reinterpret_cast<__nv_bfloat16*>(sm + S8Smem::ones)[e] = __float2bfloat16_rn(1.0f);
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
      tmem_st16(tmem + lane_off + (hf ? S8Tm::S1 : S8Tm::S0) + b * 16, r);
    }
    tmem_st_wait();
    store_state_row_sw32(sb + S8Smem::sbf, hf * 128 + t, vals);
    fence_proxy_async();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    mbar_arrive(bar + k8_SBF0);
    mbar_arrive(bar + k8_SBF1);
  }

  if (warp == 12) {
    // ================================================================ issuer
    // The whole warp runs this loop (waits included); TMA copies, MMAs and commits are
    // issued by one elected lane (the same lane every time).
    {
      if (elect_one()) {
        prefetch_tmap(&tq);
        prefetch_tmap(&tk);
        prefetch_tmap(&tv);
      }
      __syncwarp();
      const uint32_t id_proj = idesc_bf16(128, 16, 0, 0);
      const uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
      const uint32_t id_ro = idesc_bf16(128, kNV, 0, 1);   // A tmem (K-major), B MN-major
      const uint32_t id_up = idesc_bf16(128, kNV, 1, 1);   // A MN-major smem, B MN-major
      // Descriptor bases; per K-step only the start address (and for [v|1] the leading
      // offset) moves, by constants.  Start addresses stay below 2^18 bytes, so adding
      // (bytes >> 4) to the descriptor never carries out of its 14-bit field.
      const uint64_t d_w = sdesc(sb + S8Smem::w, 128, 1024, kSwizzleNone);
      const uint64_t d_qk = sdesc(sb + S8Smem::phk, 16, 1024, kSwizzle128B);
      const uint64_t d_ro = sdesc(sb + S8Smem::sbf, 8192, 256, kSwizzle32B);
      const uint64_t d_up0 = sdesc(sb + S8Smem::phk, 16384, 1024, kSwizzle128B);
      const uint64_t d_up1 = sdesc(sb + S8Smem::phk + 32768, 16384, 1024, kSwizzle128B);
      // [v | 1] for K-step s: start v + s*2048, second atom (the ones block) at leading
      // offset ones - (v + s*2048)
      const uint64_t d_vone0 = sdesc(sb + S8Smem::v0, S8Smem::ones - S8Smem::v0, 1024, kSwizzle128B);
      const uint64_t d_vone1 = sdesc(sb + S8Smem::v1, S8Smem::ones - S8Smem::v1, 1024, kSwizzle128B);
      const uint64_t vstep = (uint64_t)(2048 >> 4) - ((uint64_t)(2048 >> 4) << 16);
      const float* inv_q = inv_norms + (size_t)h * inv_stride;
      const float* inv_k = inv_norms + ((size_t)prm.H + h) * inv_stride;
      bool ok = true;
      auto wait = [&](int b, uint32_t par) {   // warp-uniform outcome
        if (ok && !mbar_wait(bar + b, par)) ok = false;
        ok = __all_sync(0xffffffffu, ok);
        return ok;
      };
      auto load_qk = [&](int c) {
        const int st = c & 1;
        const int t0 = (int)(s0 + (int64_t)c * kC);
        if (elect_one()) {
          mbar_arrive_expect_tx(bar + k8_QKFULL0 + st, 32768 + 1024);
          tma_load_3d(sm + (st ? S8Smem::q1 : S8Smem::q0), &tq, 0, t0, h, bar + k8_QKFULL0 + st);
          tma_load_3d(sm + (st ? S8Smem::k1 : S8Smem::k0), &tk, 0, t0, h, bar + k8_QKFULL0 + st);
          uint8_t* inv = sm + (st ? S8Smem::inv1 : S8Smem::inv0);
          bulk_load(inv, inv_q + t0, 512, bar + k8_QKFULL0 + st);
          bulk_load(inv + 512, inv_k + t0, 512, bar + k8_QKFULL0 + st);
        }
        __syncwarp();
      };
      auto load_v = [&](int c) {
        const int st = c & 1;
        const int t0 = (int)(s0 + (int64_t)c * kC);
        if (elect_one()) {
          mbar_arrive_expect_tx(bar + k8_VFULL0 + st, 16384);
          tma_load_3d(sm + (st ? S8Smem::v1 : S8Smem::v0), &tv, 0, t0, h, bar + k8_VFULL0 + st);
        }
        __syncwarp();
      };
      auto issue_proj = [&](int c) {
        const int st = c & 1;
        const uint64_t dq = sdesc(sb + (st ? S8Smem::q1 : S8Smem::q0), 16, 1024, kSwizzle128B);
        const uint64_t dk = sdesc(sb + (st ? S8Smem::k1 : S8Smem::k0), 16, 1024, kSwizzle128B);
        if (elect_one()) {
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            umma_ss(tmem + S8Tm::pq, dq + 2 * s, d_w + 16 * s, id_proj, s > 0);
            umma_ss(tmem + S8Tm::pk, dk + 2 * s, d_w + 16 * s, id_proj, s > 0);
          }
          umma_commit(bar + k8_PROJ);
        }
        __syncwarp();
      };
      if (nchunks > 0) {
        load_qk(0);
        load_v(0);
        if (nchunks > 1) {
          load_qk(1);
          load_v(1);
        }
        if (wait(k8_QKFULL0, 0)) {
          tc_fence_after();
          issue_proj(0);
        }
      }
      for (int c = 0; c < nchunks && ok; ++c) {
        const uint32_t par = c & 1;
        const int st = c & 1;
        const uint32_t spar = (c >> 1) & 1;
        const uint64_t d_vone = st ? d_vone1 : d_vone0;
        // stage st (q/k tiles, 1/|x|) is free once the projections completed and both
        // hashing groups read their results
        if (!wait(k8_PROJ, par) || !wait(k8_PROJFREE, par)) break;
        SW_TRACE(c, 0);
        if (c + 2 < nchunks) load_qk(c + 2);
        // ---- half 0 of the rows: QK (keys x rows 0-127), readout, state update
        if (!wait(k8_PHQ, par) || !wait(k8_PHK0, par)) break;
        SW_TRACE(c, 1);
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int s = 0; s < 8; ++s)
            umma_ts(tmem + S8Tm::qk, tmem + S8Tm::phq + s * 8,
                    d_qk + (uint64_t)((s >> 2) * 1024 + (s & 3) * 2), id_qk, s > 0);
        }
        __syncwarp();
        if (!wait(k8_SBF0, par) || !wait(k8_SBF1, par)) break;
        if (c > 0 && !wait(k8_NUMFREE, par ^ 1)) break;
        SW_TRACE(c, 2);
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int s = 0; s < 16; ++s)
            umma_ts(tmem + S8Tm::num, tmem + S8Tm::phq + s * 8, d_ro + 32 * s, id_ro, s > 0);
        }
        __syncwarp();
        if (!wait(k8_VFULL0 + st, spar)) break;
        SW_TRACE(c, 3);
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int s = 0; s < 8; ++s)
            umma_ss(tmem + S8Tm::S0, d_up0 + 128 * s, d_vone + vstep * s, id_up, 1);
          umma_commit(bar + k8_HALF0);
        }
        __syncwarp();
        // ---- half 1
        if (!wait(k8_PHK1, par)) break;
        SW_TRACE(c, 4);
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int s = 8; s < 16; ++s)
            umma_ts(tmem + S8Tm::qk, tmem + S8Tm::phq + s * 8,
                    d_qk + (uint64_t)((s >> 2) * 1024 + (s & 3) * 2), id_qk, 1);
          umma_commit(bar + k8_QKDONE);    // QK complete; p(q) of this chunk no longer read
        }
        __syncwarp();
        // next chunk's projections go into the p(q) columns just released (in issue
        // order after the last MMA that reads p(q) of this chunk)
        if (c + 1 < nchunks) {
          if (!wait(k8_QKFULL0 + (st ^ 1), ((c + 1) >> 1) & 1)) break;
          tc_fence_after();
          issue_proj(c + 1);
        }
        if (elect_one()) {
#pragma unroll
          for (int s = 0; s < 8; ++s)
            umma_ss(tmem + S8Tm::S1, d_up1 + 128 * s, d_vone + vstep * s, id_up, 1);
          umma_commit(bar + k8_HALF1);
        }
        __syncwarp();
        // ---- masked in-chunk weights are ready in tensor memory
        if (!wait(k8_CONV, par)) break;
        SW_TRACE(c, 5);
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int s = 0; s < 8; ++s)
            umma_ts(tmem + S8Tm::num,
                    tmem + (s < 4 ? S8Tm::intraA + s * 8 : S8Tm::intraB + (s - 4) * 8),
                    d_vone + vstep * s, id_ro, 1);
          umma_commit(bar + k8_AV);
        }
        __syncwarp();
        if (c + 2 < nchunks) {       // v tile of stage st: AV was its last reader
          if (!wait(k8_AV, par)) break;
          SW_TRACE(c, 7);
          load_v(c + 2);
        }
      }
      if (ok && nchunks > 0) wait(k8_AV, (nchunks - 1) & 1);
    }
  } else if (warp >= 8) {
    // ================================================================ output epilogue
    // Rows leave tensor memory, go through a 64-row staging buffer and are added to the
    // global float32 accumulators by TMA tensor reductions (sum over the row groups of
    // a head), half a chunk at a time.
    const int t = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    float* stg = reinterpret_cast<float*>(sm + S8Smem::stage);
    const bool leader = (warp == 8 && lane == 0);
    for (int c = 0; c < nchunks; ++c) {
      const int t0 = (int)(s0 + (int64_t)c * kC);
      if (t == 0) SW_TRACE(c, 30);
      if (!mbar_wait(bar + k8_AV, c & 1)) break;
      if (t == 0) SW_TRACE(c, 31);
      tc_fence_after();
      float acc[kNV];
      tmem_ld80(tmem + lane_off + S8Tm::num, acc);
      tc_fence_before();
      named_bar(3, 128);
      if (t == 0) mbar_arrive(bar + k8_NUMFREE);
      if (t == 0) SW_TRACE(c, 32);
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        if ((t >> 6) == half) {
          float4* row = reinterpret_cast<float4*>(stg + (t & 63) * kNumStride);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            row[e] = make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]);
          row[16] = make_float4(acc[64], 0.f, 0.f, 0.f);
          fence_proxy_async();
        }
        named_bar(3, 128);
        if (leader) {
          tma_reduce_add_3d(&tnum, 0, t0 + half * 64, h, stg);
          bulk_commit();
          bulk_wait_read0();
        }
        named_bar(3, 128);
        if (t == 0) SW_TRACE(c, 33 - half * 0);
      }
    }
    if (leader) bulk_wait0();
  } else {
    // ================================================================ hashing warps
    const int grp = warp >> 2;                 // 0: q side, 1: k side
    const int t = (warp & 3) * 32 + lane;      // token row = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int nb = 1 + grp;
    bool ok = true;
    auto wait = [&](int b, uint32_t par) {
      if (ok && !mbar_wait(bar + b, par)) ok = false;
      return ok;
    };
    for (int c = 0; c < nchunks && ok; ++c) {
      const uint32_t par = c & 1;
      const int st = c & 1;
      const int64_t t0 = s0 + (int64_t)c * kC;
      const bool tv_ = (t0 + t) < s1;
      const float valid = tv_ ? 1.f : 0.f;
      // ---- projections (hi + lo halves) and 1/|x|
      const int eb = 10 + 10 * grp;
      if (t == 0) SW_TRACE(c, eb);
      if (!wait(k8_QKFULL0 + st, (c >> 1) & 1) || !wait(k8_PROJ, par)) break;
      if (t == 0) SW_TRACE(c, eb + 1);
      tc_fence_after();
      const float inv = reinterpret_cast<const float*>(
          sm + (st ? S8Smem::inv1 : S8Smem::inv0))[grp * 128 + t];
      const float scale = tv_ ? inv * prm.two_over_tau : 0.f;
      uint32_t r[16];
      tmem_ld16(tmem + lane_off + (grp ? S8Tm::pk : S8Tm::pq), r);
      tmem_ld_wait();
      if (lane == 0 && grp == 0) SW_TRACE(c, 34 + (warp & 3));
      tc_fence_before();
      named_bar(nb, 128);
      if (t == 0) mbar_arrive(bar + k8_PROJFREE);
      if (t == 0) SW_TRACE(c, eb + 8);
      float sp[P], smv[P];
#pragma unroll
      for (int p = 0; p < P; ++p) {
        const float u = __uint_as_float(r[p]) + __uint_as_float(r[8 + p]);
        logistic_fast(u * scale, sp[p], smv[p]);
      }
      float lo[8], hi[32];
      corner_factors(sp, smv, valid, lo, hi);
      if (grp == 0) {
        // ---- p(q) into tensor memory: column c holds rows 2c (low half) and 2c+1
        if (t == 0) SW_TRACE(c, 38);
        if (c > 0 && !wait(k8_QKDONE, par ^ 1)) break;
        if (t == 0) SW_TRACE(c, eb + 2);
        tc_fence_after();
#pragma unroll
        for (int blk = 0; blk < 8; ++blk) {
          if (blk == 6 && !wait(k8_PROJFREE, par)) break;   // rows 192-255 hold projections
          uint32_t v16[16];
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const float hv = hi[blk * 4 + cc];
#pragma unroll
            for (int e = 0; e < 4; ++e) v16[cc * 4 + e] = pack_bf16(hv * lo[2 * e], hv * lo[2 * e + 1]);
          }
          tmem_st16(tmem + lane_off + S8Tm::phq + blk * 16, v16);
        }
        tmem_st_wait();
        tc_fence_before();
        named_bar(nb, 128);
        if (t == 0) mbar_arrive(bar + k8_PHQ);
        if (t == 0) SW_TRACE(c, eb + 3);
      } else {
        // ---- p(k) rows into shared memory (core-matrix layout, 256 rows)
        const uint32_t base = sb + S8Smem::phk;
        if (t == 0) SW_TRACE(c, 39);
        if (c > 0 && !wait(k8_HALF0, par ^ 1)) break;
        if (t == 0) SW_TRACE(c, eb + 2);
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) store_chunk(phk_addr(base, t, cc), hi[cc], lo);
        fence_proxy_async();
        named_bar(nb, 128);
        if (t == 0) mbar_arrive(bar + k8_PHK0);
        if (t == 0) SW_TRACE(c, eb + 3);
        if (c > 0 && !wait(k8_HALF1, par ^ 1)) break;
        if (t == 0) SW_TRACE(c, eb + 4);
#pragma unroll
        for (int cc = 16; cc < 32; ++cc) store_chunk(phk_addr(base, t, cc), hi[cc], lo);
        fence_proxy_async();
        named_bar(nb, 128);
        if (t == 0) mbar_arrive(bar + k8_PHK1);
        if (t == 0) SW_TRACE(c, eb + 5);
      }
      // ---- mask QK (keys j <= row t) and round to bf16, in place: group 0 owns keys
      //      0-63 (written to qk+0..31), group 1 keys 64-127 (written to qk+64..95)
      if (t == 0) SW_TRACE(c, eb + 6);
      if (!wait(k8_QKDONE, par)) break;
      if (t == 0) SW_TRACE(c, eb + 7);
      tc_fence_after();
      const uint32_t src = tmem + lane_off + S8Tm::qk + grp * 64;
      const uint32_t dst = tmem + lane_off + (grp ? S8Tm::intraB : S8Tm::intraA);
      uint32_t out32[32], qk64[64];
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) tmem_ld16(src + cb * 16, qk64 + cb * 16);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int j0 = grp * 64 + 2 * e;
        const float a0 = (j0 <= t) ? __uint_as_float(qk64[2 * e]) : 0.f;
        const float a1 = (j0 + 1 <= t) ? __uint_as_float(qk64[2 * e + 1]) : 0.f;
        out32[e] = pack_bf16(a0, a1);
      }
      tmem_st16(dst, out32);
      tmem_st16(dst + 16, out32 + 16);
      tmem_st_wait();
      tc_fence_before();
      named_bar(nb, 128);
      if (t == 0) mbar_arrive(bar + k8_CONV);
      // ---- bf16 copy of state half grp for the next chunk's readout
      if (!wait(grp ? k8_HALF1 : k8_HALF0, par)) break;
      if (t == 0) SW_TRACE(c, eb + 9);
      tc_fence_after();
      {
        float vals[kNV];
        tmem_ld80(tmem + lane_off + (grp ? S8Tm::S1 : S8Tm::S0), vals);
        store_state_row_sw32(sb + S8Smem::sbf, grp * 128 + t, vals);
      }
      fence_proxy_async();
      tc_fence_before();
      named_bar(nb, 128);
      if (t == 0) mbar_arrive(bar + (grp ? k8_SBF1 : k8_SBF0));
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

// Last steps of the soft-hash backward on tensor cores: from the per-plane gradients
// du' = (dL/du) / max(|x|, eps) of every token of one side (q or k) to
//   dx  = dxh' - xhat (xhat . dxh'),   dxh' = du' W^T          (projection transpose and
//                                                              normalisation Jacobian)
//   dW += du'^T x = du^T xhat                                  (per-CTA partial sums)
// which is the chain rule through u = W^T xhat, xhat = x / max(|x|, eps) ([JA] §2.2:
// the soft assignment is differentiable end to end).
//
// Operands (bf16, float32 accumulation in tensor memory):
//   du' is stored by the corner-gradient sweep as a hi + lo pair of bf16 arrays
//   [rows][lps] (about 16 significant bits); W^T is split the same way in shared memory;
//   x is the bf16 input itself, exact.  dxh' takes three products (hi.hi, lo.hi, hi.lo),
//   dW two (hi.x, lo.x).
// Grid (blocks, H): the CTAs of head h are persistent over its tiles of 128 tokens (the
// tensor maps are [H][N][cols], so a tile never reaches into the next head), two TMA
// stages.  Warps 0-3 (thread = token = tensor-memory lane) compute 1/|x| from the x tile,
// read dxh' and write dx; warp 4 issues TMA copies and MMAs from an elected lane.
// L * P <= 128: one accumulator of 128 lanes holds dW (lane = table * P + plane), and the
// du' tile is two boxes of 64.  W is this head's planes (offset w_hs per head, 0 when
// shared); the partial sums go to part[h][block][L*P][64].
#pragma once

#include "tc_kernels.cuh"

namespace race {
namespace tc {

constexpr int kFzThreads = 160;
constexpr int kFzMaxLP = 128;

struct FzSmem {
  static constexpr uint32_t stage = 81920;                 // bytes per TMA stage
  static constexpr uint32_t duh = 0, dul = 32768, x = 65536;  // offsets within a stage
  static constexpr uint32_t wth = 2 * stage;               // W^T hi: 2 boxes [64 dims][64 lp]
  static constexpr uint32_t wtl = wth + 16384;             // W^T lo
  static constexpr uint32_t bars = wtl + 16384;
  static constexpr uint32_t total = bars + 128;
  static constexpr uint32_t alloc = total + 1024;
};
static_assert(FzSmem::alloc <= 232448, "shared memory budget of one CTA");

enum FzBar : int {
  fz_FULL0 = 0, fz_FULL1, fz_MMA0, fz_MMA1, fz_READ0, fz_READ1, fz_DX, fz_DXFREE, fz_COUNT
};

template <typename TG>
__global__ void __launch_bounds__(kFzThreads, 1)
    k_bwd_finalize_tc(const __grid_constant__ CUtensorMap tduh,
                      const __grid_constant__ CUtensorMap tdul,
                      const __grid_constant__ CUtensorMap tx, const float* __restrict__ W,
                      TG* __restrict__ dx, float* __restrict__ part, int64_t N, int L,
                      int P, int64_t w_hs) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + FzSmem::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + fz_COUNT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int LP = L * P;
  const int h = blockIdx.y;
  W += (size_t)h * w_hs;
  const int64_t ntiles = (N + 127) / 128;
  const int my_tiles =
      blockIdx.x < ntiles ? (int)((ntiles - 1 - blockIdx.x) / gridDim.x) + 1 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < fz_COUNT; ++i)
      mbar_init(bar + i, (i == fz_READ0 || i == fz_READ1 || i == fz_DXFREE) ? 4 : 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  // W^T [dim][lp] as hi + lo bf16 in two 128B-swizzled boxes of 64 lp (zero past L*P)
  for (int e = threadIdx.x; e < 64 * kFzMaxLP; e += blockDim.x) {
    const int d = e / kFzMaxLP, lp = e % kFzMaxLP;
    const float w = lp < LP ? W[((size_t)(lp / P) * 64 + d) * P + (lp % P)] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
    const uint32_t off = (lp >> 6) * 8192 + d * 128 + ((((lp & 63) >> 3) ^ (d & 7)) << 4) +
                         (lp & 7) * 2;
    *reinterpret_cast<__nv_bfloat16*>(sm + FzSmem::wth + off) = hi;
    *reinterpret_cast<__nv_bfloat16*>(sm + FzSmem::wtl + off) = lo;
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t TM_DX = 0, TM_DW = 64;
  bool ok = true;
  auto wait = [&](int b, uint32_t par) {
    if (ok && !mbar_wait(bar + b, par)) ok = false;
    ok = __all_sync(0xffffffffu, ok);
    return ok;
  };
  auto tile_row0 = [&](int k) { return (int)((blockIdx.x + (int64_t)k * gridDim.x) * 128); };

  if (warp == 4) {
    // ================================================================ issuer
    const uint32_t id_dx = idesc_bf16(128, 64, 0, 0);   // A du' K-major, B W^T K-major
    const uint32_t id_dw = idesc_bf16(128, 64, 1, 1);   // A du'^T MN-major, B x MN-major
    auto load = [&](int k) {
      const int st = k & 1;
      const uint32_t base = st * FzSmem::stage;
      const int r0 = tile_row0(k);
      mbar_arrive_expect_tx(bar + fz_FULL0 + st, FzSmem::stage);
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        tma_load_3d(sm + base + FzSmem::duh + b * 16384, &tduh, 64 * b, r0, h, bar + fz_FULL0 + st);
        tma_load_3d(sm + base + FzSmem::dul + b * 16384, &tdul, 64 * b, r0, h, bar + fz_FULL0 + st);
      }
      tma_load_3d(sm + base + FzSmem::x, &tx, 0, r0, h, bar + fz_FULL0 + st);
    };
    if (elect_one()) {
      prefetch_tmap(&tduh);
      prefetch_tmap(&tdul);
      prefetch_tmap(&tx);
      if (my_tiles > 0) load(0);
      if (my_tiles > 1) load(1);
    }
    __syncwarp();
    for (int k = 0; k < my_tiles && ok; ++k) {
      const int st = k & 1;
      const uint32_t ph = (uint32_t)(k >> 1) & 1;
      const uint32_t base = sb + st * FzSmem::stage;
      if (!wait(fz_FULL0 + st, ph)) break;
      if (k > 0 && !wait(fz_DXFREE, (uint32_t)(k - 1) & 1)) break;
      tc_fence_after();
      if (elect_one()) {
        // dxh' = du' W^T over K = 128 lp (two boxes of 64, four K-steps of 16 each)
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint32_t ko = (s >> 2) * 16384 + (s & 3) * 32;
          const uint32_t kw = (s >> 2) * 8192 + (s & 3) * 32;
          const uint64_t ah = sdesc(base + FzSmem::duh + ko, 16, 1024, kSwizzle128B);
          const uint64_t al = sdesc(base + FzSmem::dul + ko, 16, 1024, kSwizzle128B);
          const uint64_t bh = sdesc(sb + FzSmem::wth + kw, 16, 1024, kSwizzle128B);
          const uint64_t bl = sdesc(sb + FzSmem::wtl + kw, 16, 1024, kSwizzle128B);
          umma_ss(tmem + TM_DX, ah, bh, id_dx, s > 0);
          umma_ss(tmem + TM_DX, al, bh, id_dx, 1);
          umma_ss(tmem + TM_DX, ah, bl, id_dx, 1);
        }
        umma_commit(bar + fz_DX);
        // dW += du'^T x over K = 128 tokens (K-steps of 16 rows = 2 KB)
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint64_t ah = sdesc(base + FzSmem::duh + s * 2048, 16384, 1024, kSwizzle128B);
          const uint64_t al = sdesc(base + FzSmem::dul + s * 2048, 16384, 1024, kSwizzle128B);
          const uint64_t bx = sdesc(base + FzSmem::x + s * 2048, 8192, 1024, kSwizzle128B);
          umma_ss(tmem + TM_DW, ah, bx, id_dw, (k > 0 || s > 0) ? 1u : 0u);
          umma_ss(tmem + TM_DW, al, bx, id_dw, 1);
        }
        umma_commit(bar + fz_MMA0 + st);
      }
      __syncwarp();
      // stage st takes tile k+2 once its MMAs and the CUDA-core reads of x are done
      if (k + 2 < my_tiles) {
        if (!wait(fz_MMA0 + st, ph) || !wait(fz_READ0 + st, ph)) break;
        if (elect_one()) load(k + 2);
        __syncwarp();
      }
    }
  } else {
    // ================================================================ CUDA-core warps
    const int t = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    for (int k = 0; k < my_tiles; ++k) {
      const int st = k & 1;
      const uint32_t ph = (uint32_t)(k >> 1) & 1;
      const uint8_t* xt = sm + st * FzSmem::stage + FzSmem::x;
      if (!wait(fz_FULL0 + st, ph)) break;
      // this token's x row and 1 / max(|x|, eps).  In the 128-byte-swizzled tile, chunk
      // c of row t sits at position c ^ (t % 8); reading position c ^ (t % 8) in step c
      // makes the eight rows of a shared-memory phase hit eight different bank groups.
      float xr[64];
      float ss[4] = {0.f, 0.f, 0.f, 0.f};
      {
        const uint4* row = reinterpret_cast<const uint4*>(xt + t * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 w = row[c ^ (t & 7)];
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ws[e]));
            xr[c * 8 + 2 * e] = f.x;
            xr[c * 8 + 2 * e + 1] = f.y;
            ss[e] = fmaf(f.x, f.x, fmaf(f.y, f.y, ss[e]));
          }
        }
      }
      const float inv = 1.0f / fmaxf(sqrtf((ss[0] + ss[1]) + (ss[2] + ss[3])), kEpsNorm);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + fz_READ0 + st);
      if (!wait(fz_DX, (uint32_t)k & 1)) break;
      tc_fence_after();
      uint32_t r[64];
#pragma unroll
      for (int b = 0; b < 4; ++b) tmem_ld16(tmem + lane_off + TM_DX + b * 16, r + b * 16);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + fz_DXFREE);
      // dx = dxh' - xhat (xhat . dxh') = dxh' - x (inv^2 (x . dxh'))
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) dot = fmaf(xr[c], __uint_as_float(r[c]), dot);
      const float f = dot * inv * inv;
      const int64_t row = (int64_t)tile_row0(k) + t;
      if (row < N) {
        TG* o = dx + ((size_t)h * N + row) * kD;
        if constexpr (sizeof(TG) == 4) {
#pragma unroll
          for (int c = 0; c < 64; c += 4)
            *reinterpret_cast<float4*>(o + c) =
                make_float4(fmaf(-xr[c], f, __uint_as_float(r[c])),
                            fmaf(-xr[c + 1], f, __uint_as_float(r[c + 1])),
                            fmaf(-xr[c + 2], f, __uint_as_float(r[c + 2])),
                            fmaf(-xr[c + 3], f, __uint_as_float(r[c + 3])));
        } else {
#pragma unroll
          for (int c = 0; c < 64; c += 8)
            *reinterpret_cast<uint4*>(o + c) = make_uint4(
                pack_bf16(fmaf(-xr[c], f, __uint_as_float(r[c])),
                          fmaf(-xr[c + 1], f, __uint_as_float(r[c + 1]))),
                pack_bf16(fmaf(-xr[c + 2], f, __uint_as_float(r[c + 2])),
                          fmaf(-xr[c + 3], f, __uint_as_float(r[c + 3]))),
                pack_bf16(fmaf(-xr[c + 4], f, __uint_as_float(r[c + 4])),
                          fmaf(-xr[c + 5], f, __uint_as_float(r[c + 5]))),
                pack_bf16(fmaf(-xr[c + 6], f, __uint_as_float(r[c + 6])),
                          fmaf(-xr[c + 7], f, __uint_as_float(r[c + 7]))));
        }
      }
    }
    // the CTA's dW partial: lane = table * P + plane, 64 columns = dims
    if (ok && my_tiles > 0) {
      const int last = my_tiles - 1;
      if (wait(fz_MMA0 + (last & 1), (uint32_t)(last >> 1) & 1)) {
        tc_fence_after();
        uint32_t r[64];
#pragma unroll
        for (int b = 0; b < 4; ++b) tmem_ld16(tmem + lane_off + TM_DW + b * 16, r + b * 16);
        tmem_ld_wait();
        if (t < LP) {
          float* o = part + (((size_t)h * gridDim.x + blockIdx.x) * LP + t) * 64;
#pragma unroll
          for (int c = 0; c < 64; c += 4)
            *reinterpret_cast<float4*>(o + c) =
                make_float4(__uint_as_float(r[c]), __uint_as_float(r[c + 1]),
                            __uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]));
        }
      }
    } else if (t < LP) {
      float* o = part + (((size_t)h * gridDim.x + blockIdx.x) * LP + t) * 64;
      for (int c = 0; c < 64; ++c) o[c] = 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// 3-D bf16 view [H][N][inner] with the given row stride (elements), for 128B-swizzled
// boxes of 64 elements x 128 rows of one head.
inline bool encode_rows_bf16(CUtensorMap* m, const void* base, int64_t inner, int64_t N, int H,
                             int64_t row_stride_elems) {
  const auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)N, (cuuint64_t)H};
  cuuint64_t strides[2] = {(cuuint64_t)row_stride_elems * 2,
                           (cuuint64_t)row_stride_elems * 2 * (cuuint64_t)N};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace race

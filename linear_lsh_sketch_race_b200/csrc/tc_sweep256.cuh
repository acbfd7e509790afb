// Helpers of the one-table-per-CTA causal sweep (R = 256 buckets, P = 8 planes): the
// 1/|x| pre-pass over q and k, the corner-factor expansion, the 128B-swizzled p(k) tile
// addressing, the 32B-swizzled bf16 state operand, and TMA / bulk-copy wrappers for the
// output reductions.  The sweep kernel itself is k_sweep_pipe (tc_sweep_pipe.cuh).
// Soft bucketization and aggregation: [JA] §2.1; causal prefix: [JA] §2.2.
#pragma once

#include "tc_sweep.cuh"

namespace race {
namespace tc {

// 1/max(|x|, eps) of every row of q and k into out[side][h][stride] (side 0: q, 1: k);
// grid (ceil(N/128), 2*H), 256 threads: eight threads per row, one 16-byte load each, so
// a warp reads four whole rows per load; each thread covers four rows 32 apart (four
// loads in flight).  The squares are summed over the eight lanes of a row with shuffles.
// Entries stride - N .. of each head are never written and never used (they pad the
// last chunk so it can be bulk-copied whole).
__global__ void k_inv_norms(const __nv_bfloat16* __restrict__ q,
                            const __nv_bfloat16* __restrict__ k, float* __restrict__ out,
                            int64_t N, int H, int64_t stride) {
  const int part = threadIdx.x & 7;
  const int sh = blockIdx.y;                 // side * H + head
  const int side = sh >= H, h = sh - side * H;
  const __nv_bfloat16* x = (side ? k : q) + (size_t)h * N * kD + part * 8;
  const int64_t n0 = (int64_t)blockIdx.x * 128 + (threadIdx.x >> 3);
  uint4 w[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t n = n0 + 32 * r;
    w[r] = n < N ? __ldg(reinterpret_cast<const uint4*>(x + n * kD)) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const uint32_t ws[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ws[e]));
      s = fmaf(f.x, f.x, fmaf(f.y, f.y, s));
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    const int64_t n = n0 + 32 * r;
    if (n < N && part == 0) out[(size_t)sh * stride + n] = 1.0f / fmaxf(sqrtf(s), kEpsNorm);
  }
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

}  // namespace tc
}  // namespace race

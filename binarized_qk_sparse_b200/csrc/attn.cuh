// attn.cuh -- the parity export of the integer scores from packed bits
// (k_scores_int) on warp-level mma.sync fragments: 64-row CTA tiles of 4 warps,
// cp.async staging.  A kernel of its own, independent of the hot path, which
// runs on tcgen05 (attn_tc.cuh).
#pragma once

#include "common.cuh"

namespace had {

constexpr int kQT = 64;             // query rows per CTA
constexpr int kKT = 64;             // keys per tile
constexpr int kAttnThreads = 128;   // 4 warps

enum { KMAP_NATURAL = 0, KMAP_U8 = 1 };

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gmem_src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Tile-local key index of score column `col` (0..7) of n-block `nb` (0..7).
// KMAP_NATURAL: natural order.  KMAP_U8: each 32-key chunk interleaves four
// n-blocks so that lane q's C-fragment scores form the A-fragment bytes
// (keys 4q..4q+3 and 16+4q..16+4q+3) of an m16n8k32 u8 x s8 MMA.
template <int MODE>
__device__ __forceinline__ int key_of(int nb, int col) {
  if (MODE == KMAP_NATURAL) return nb * 8 + col;
  int cc = nb >> 2, x = nb & 3;
  return cc * 32 + ((x >> 1) << 4) + ((col >> 1) << 2) + ((x & 1) << 1) + (col & 1);
}

}  // namespace had

namespace had {

// Debug export of the integer scores from packed bits, on legacy mma.sync
// m16n8k32 s8 fragments (a kernel of its own, independent of k_attn_tc, whose
// scores the EXP_SCORES export reads from tensor memory):
// S[i][j] = q~_i . k~_j = d - 2*popcount(q XOR k) for i, j < L, 0 elsewhere.
// The K~ tile is expanded from packed bits in smem.
template <int MODE>
__global__ void __launch_bounds__(kAttnThreads) k_scores_int(const uint32_t* __restrict__ qbits,
                                                             const uint32_t* __restrict__ kbits, int H, int n,
                                                             const int32_t* seqlens, int32_t* __restrict__ S,
                                                             unsigned* status) {
  __shared__ __align__(16) int8_t kt[kKT * kD];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
  const int bh = blockIdx.y, b = bh / H;
  const int q0 = blockIdx.x * kQT;
  const int L = valid_len(seqlens, b, n, status);
  const int i0 = q0 + warp * 16 + g, i1 = i0 + 8;
  uint32_t qa[2][4];
  {
    auto field = [&](int i) -> uint32_t {
      if (i >= L) return 0u;
      const uint2 w = *reinterpret_cast<const uint2*>(qbits + ((size_t)bh * n + i) * kW);
      return (((q < 2) ? w.x : w.y) >> ((q & 1) * 16)) & 0xFFFFu;
    };
    const uint32_t f0 = field(i0), f1 = field(i1);
    qa[0][0] = expand_nibble_pm1(f0 & 15u);
    qa[0][1] = expand_nibble_pm1(f1 & 15u);
    qa[0][2] = expand_nibble_pm1((f0 >> 4) & 15u);
    qa[0][3] = expand_nibble_pm1((f1 >> 4) & 15u);
    qa[1][0] = expand_nibble_pm1((f0 >> 8) & 15u);
    qa[1][1] = expand_nibble_pm1((f1 >> 8) & 15u);
    qa[1][2] = expand_nibble_pm1((f0 >> 12) & 15u);
    qa[1][3] = expand_nibble_pm1((f1 >> 12) & 15u);
  }
  const int ntiles = (n + kKT - 1) / kKT;
  for (int t = 0; t < ntiles; ++t) {
    __syncthreads();
    // expand 64 keys x 64 channels: thread -> (key, 32 channels)
    {
      const int r = tid >> 1, half = tid & 1, j = t * kKT + r;
      uint32_t word = (j < L) ? kbits[((size_t)bh * n + j) * kW + half] : 0u;
      uint32_t* dst = reinterpret_cast<uint32_t*>(kt + r * kD + half * 32);
#pragma unroll
      for (int u = 0; u < 8; ++u) dst[u] = expand_nibble_pm1((word >> (4 * u)) & 15u);
    }
    __syncthreads();
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      const uint4 kb = *reinterpret_cast<const uint4*>(kt + key_of<MODE>(nb, g) * kD + q * 16);
      int sc[4] = {0, 0, 0, 0};
      mma_s8_16x8x32(sc, qa[0], kb.x, kb.y);
      mma_s8_16x8x32(sc, qa[1], kb.z, kb.w);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = (e < 2) ? i0 : i1;
        const int j = t * kKT + key_of<MODE>(nb, 2 * q + (e & 1));
        if (i < n && j < n) S[((size_t)bh * n + i) * n + j] = (i < L && j < L) ? sc[e] : 0;
      }
    }
  }
}

}  // namespace had

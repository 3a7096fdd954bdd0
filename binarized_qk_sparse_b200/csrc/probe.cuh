// probe.cuh -- tensor-pipe throughput probe for the roofline of the score
// contraction.  The score s = Q~ K~^T of BinaryAttention §2.2 runs as a +-1
// int8 tcgen05.mma (kind::i8); the bf16 kind (kind::f16) carries the float A.V.
// This kernel measures what those two MMA kinds sustain on this GPU: one CTA per
// SM issues back-to-back M=128, N=256 MMAs into one tensor-memory accumulator
// from operands resident in shared memory (no loads in the loop), so the rate is
// the tensor pipe's own.  Included once, by had_lib.cu.
#pragma once

#include "sm100.cuh"

namespace had {
namespace probe {

using namespace had::sm100;

constexpr int kM = 128, kN = 256;
constexpr int kThreads = 128;
// Operand bytes per K-step row: 32 int8 or 16 bf16 elements (32 B).  A and B
// tiles are 64 B per row (two K-steps), 64-byte swizzled K-major, as in the
// attention kernel.
constexpr int kRowBytes = 64;
constexpr int kSmemA = kM * kRowBytes, kSmemB = kN * kRowBytes;
constexpr int kSmemTotal = kSmemA + kSmemB + 64 + 1024;

// kind: 0 = kind::i8 (s8 x s8 -> s32), 1 = kind::f16 (bf16 x bf16 -> f32).
// Each CTA issues `iters` MMAs of K = 32 (i8) or K = 16 (bf16) elements.
__global__ void __launch_bounds__(kThreads, 1) k_probe_mma(int kind, int iters, unsigned* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sA = sm;
  uint8_t* sB = sm + kSmemA;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kSmemA + kSmemB);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kSmemA + kSmemB + 8);
  const int tid = threadIdx.x, warp = tid >> 5;
  // operands: +-1 (int8) or +-1.0 (bf16) patterns, as the score operands are
  for (int e = tid; e < (kSmemA + kSmemB) / 4; e += kThreads) {
    const uint32_t hsh = (uint32_t)e * 2654435761u + 0x9E3779B9u * (uint32_t)blockIdx.x;
    uint32_t v;
    if (kind == 0) v = 0x01010101u | ((hsh & 0x01010101u) * 0xFEu);
    else v = ((hsh & 1u) ? 0xBF80u : 0x3F80u) | (((hsh & 2u) ? 0xBF80u : 0x3F80u) << 16);
    reinterpret_cast<uint32_t*>(sm)[e] = v;
  }
  if (warp == 0) {
    tmem_alloc(tslot, 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  if (tid == 0) {
    const uint32_t id = kind == 0 ? idesc_i8(kM, kN, true, true, false) : idesc_bf16(kM, kN, false);
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    for (int it = 0; it < iters; ++it) {
      const uint32_t ks = (uint32_t)(it & 1) * 32u;
      const uint64_t ad = sdesc(a0 + ks, 16, 512, kSwizzle64B), bd = sdesc(b0 + ks, 16, 512, kSwizzle64B);
      if (kind == 0) mma_i8_ss(tmem, ad, bd, id, it > 0 ? 1u : 0u);
      else mma_f16_ss(tmem, ad, bd, id, it > 0 ? 1u : 0u);
    }
    mma_commit(bar);
    // bounded: a probe of `iters` MMAs takes far less than this many clocks
    if (!mbar_wait(bar, 0, 4000000000LL)) raise_status(status, kDevErrTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace probe
}  // namespace had

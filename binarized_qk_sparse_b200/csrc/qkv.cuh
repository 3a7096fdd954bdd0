// qkv.cuh -- the projection that precedes the attention path, fused with its
// binarization.  From BinaryAttention §2.2 (the scaled binarization
// X~ = sign(X - mu) of Q and K) and its Table 8, which counts the separate
// Q/K/V quantization step against the kernel: here that step happens in the
// epilogue of the projection GEMM itself.
//
// The means come first, without the projected tensors: the mean of a linear
// map's outputs is the map of the mean input, so
//   mu_Q[b][h][c] = (1/L_b) sum_{i<L_b} (X_i W_Q^T)[h*d + c] = xbar_b . W_Q[h*d + c],
// with xbar_b the mean of the valid tokens of X (k_xsum: fp64 token sums per
// 256-token chunk; k_mu: one warp per output channel, fp64 dot product, one
// rounding to fp32).  Then k_qkv_tc runs the projection on the tensor cores and
// compares each fp32 result with its mean in the epilogue:
//   - Q columns: the 64 sign bits of a token (bit 1 = below the mean), in the
//     attention workspace's packed layout;
//   - K columns: the +-1 row of a token (int8, or e4m3 for the fp8 score path),
//     rows past L (and up to n_pad) +1;
//   - V columns: the bf16 row of V, the attention's V input.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace had {
namespace qkv {

using namespace had::sm100;

constexpr int kXsumChunk = 256;    // tokens per partial sum of X
constexpr int kXsumThreads = 128;  // features per k_xsum CTA
constexpr int kMuWarps = 8;        // output channels per k_mu CTA

// Token sums of X over the valid tokens of each 256-token chunk: part[b][ch][k], fp64.
__global__ void __launch_bounds__(kXsumThreads) k_xsum(const __nv_bfloat16* __restrict__ X, int n, int Dm,
                                                       const int32_t* seqlens, int nch, double* __restrict__ part) {
  const int k = blockIdx.x * kXsumThreads + threadIdx.x, ch = blockIdx.y, b = blockIdx.z;
  if (k >= Dm) return;
  const int L = valid_len(seqlens, b, n, nullptr);
  const int i0 = ch * kXsumChunk, i1 = min(i0 + kXsumChunk, L);
  double s = 0.0;
  for (int i = i0; i < i1; ++i) s += (double)__bfloat162float(X[((size_t)b * n + i) * Dm + k]);
  part[((size_t)b * nch + ch) * Dm + k] = s;
}

// mu[t][b][h][c] for t in {Q, K}: one warp per output channel o = t*H*64 + h*64 + c,
// the fp64 dot product of the token sum of X with W's row o, divided by L.
__global__ void __launch_bounds__(kMuWarps * 32) k_mu(const __nv_bfloat16* __restrict__ W,
                                                      const double* __restrict__ part, int nch, int n, int B, int H,
                                                      int Dm, const int32_t* seqlens, unsigned* status,
                                                      float* __restrict__ mu) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o = blockIdx.x * kMuWarps + warp, b = blockIdx.y;
  if (o >= 2 * H * 64) return;
  const int L = valid_len(seqlens, b, n, status);
  const int nv = (L + kXsumChunk - 1) / kXsumChunk;
  double acc = 0.0;
  for (int k = lane; k < Dm; k += 32) {
    double xs = 0.0;
    for (int c = 0; c < nv; ++c) xs += part[((size_t)b * nch + c) * Dm + k];
    acc += xs * (double)__bfloat162float(W[(size_t)o * Dm + k]);
  }
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    const int t = o / (H * 64), r = o - t * H * 64;  // r = h * 64 + c
    mu[((size_t)t * B + b) * H * 64 + r] = (L > 0) ? (float)(acc / (double)L) : 0.0f;
  }
}

// ---------------------------------------------------------------------------- the fused projection

constexpr int kM = 128;        // tokens per CTA (TMEM lanes)
constexpr int kN = 64;         // output channels per CTA: one head's d = 64 channels of Q, K or V
constexpr int kK = 64;         // features per panel (128 bytes of bf16: one 128-byte swizzle row)
constexpr int kStages = 4;
constexpr int kThreads = 192;  // warps 0-3: epilogue (TMEM lane quadrants); 4: MMA; 5: TMA
constexpr int kMmaWarp = 4, kProdWarp = 5;
constexpr uint32_t kTmemCols = 64;
constexpr long long kWaitCycles = 2000000000LL;  // bound of a pipeline wait: about one second

struct QkvArgs {
  CUtensorMap tm_x;   // X [B*n][Dm] bf16, box {64, 128}, 128-byte swizzle
  CUtensorMap tm_w;   // W [3*H*64][Dm] bf16, box {64, 64}, 128-byte swizzle
  int B, H, n, n_pad, Dm;
  const int32_t* seqlens;
  const float* mu;    // [2][B][H][64]: the means of Q, then of K
  uint32_t* qbits;    // [B*H][n][2]
  int8_t* kpm;        // [B*H][n_pad][64] +-1 rows of K
  int k_e4m3;         // the +-1 rows as e4m3 (0x38 / 0xB8) instead of int8 (0x01 / 0xFF)
  __nv_bfloat16* V;   // [B][H][n][64]
  unsigned* status;
};

struct QkvSmem {
  static constexpr int kA = 0;                          // kStages x [128 tokens][64 features] bf16
  static constexpr int kB = kA + kStages * kM * kK * 2;  // kStages x [64 channels][64 features] bf16
  static constexpr int kBar = kB + kStages * kN * kK * 2;
  static constexpr int kNumBars = 2 * kStages + 2;       // full, empty, accumulator done, final
  static constexpr int kMu = kBar + kNumBars * 8;        // 64 means
  static constexpr int kMisc = kMu + kN * 4;             // [0] TMEM base, [1] abort
  static constexpr int kTotal = kMisc + 16 + 1024;       // + alignment slack
};

__global__ void __launch_bounds__(kThreads, 1) k_qkv_tc(const __grid_constant__ QkvArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + QkvSmem::kBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_bar = bars + 2 * kStages;
  uint64_t* fin_bar = bars + 2 * kStages + 1;
  float* smu = reinterpret_cast<float*>(sm + QkvSmem::kMu);
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + QkvSmem::kMisc);
  volatile uint32_t* abort_flag = misc + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kM, b = blockIdx.y, j = blockIdx.z;
  const int t = j / a.H, h = j - t * a.H;  // tensor (0 Q, 1 K, 2 V) and head of this CTA's 64 columns
  const int L = valid_len(a.seqlens, b, a.n, a.status);
  const int npanel = a.Dm / kK;

  if (warp == kMmaWarp) {
    tmem_alloc(misc, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProdWarp && lane == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(acc_bar, 1);
    mbar_init(fin_bar, 1);
    misc[1] = 0;
    fence_barrier_init();
    prefetch_tensormap(&a.tm_x);
    prefetch_tensormap(&a.tm_w);
  }
  if (tid < kN) smu[tid] = (t < 2) ? a.mu[(((size_t)t * a.B + b) * a.H + h) * kN + tid] : 0.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  auto bounded_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity, kWaitCycles)) return true;
    *abort_flag = 1u;
    raise_status(a.status, kDevErrTimeout);
    return false;
  };

  int par[kStages];  // producer: parity of the last load per stage (-1 none)
#pragma unroll
  for (int s = 0; s < kStages; ++s) par[s] = -1;
  if (warp == kProdWarp && lane == 0) {
    for (int p = 0; p < npanel; ++p) {
      const int st = p % kStages;
      if (p >= kStages && !bounded_wait(&empty[st], ((p / kStages) - 1) & 1)) break;
      if (*abort_flag) break;
      mbar_arrive_expect_tx(&full[st], (uint32_t)(kM + kN) * kK * 2);
      tma_load_2d(sm + QkvSmem::kA + st * kM * kK * 2, &a.tm_x, p * kK, b * a.n + m0, &full[st]);
      tma_load_2d(sm + QkvSmem::kB + st * kN * kK * 2, &a.tm_w, p * kK, j * kN, &full[st]);
      par[st] = (p / kStages) & 1;
    }
  } else if (warp == kMmaWarp && lane == 0) {
    // D[128 tokens][64 channels] += X panel [128][64] x W panel [64][64]^T: 4 K-steps of 16
    const uint32_t idesc = idesc_bf16(kM, kN, false);
    for (int p = 0; p < npanel; ++p) {
      const int st = p % kStages;
      if (!bounded_wait(&full[st], (p / kStages) & 1)) break;
      tc_fence_after();
      const uint32_t sa = smem_u32(sm + QkvSmem::kA + st * kM * kK * 2);
      const uint32_t sb = smem_u32(sm + QkvSmem::kB + st * kN * kK * 2);
#pragma unroll
      for (int ks = 0; ks < kK / 16; ++ks)
        mma_f16_ss(tmem, sdesc(sa + 32 * ks, 16, 1024, kSwizzle128B), sdesc(sb + 32 * ks, 16, 1024, kSwizzle128B),
                   idesc, (p | ks) > 0 ? 1u : 0u);
      mma_commit(&empty[st]);
    }
    mma_commit(acc_bar);
  } else if (warp < 4) {
    // epilogue: thread (warp w, lane l) owns token m0 + 32 w + l, TMEM lane 32 w + l
    const bool ok = __all_sync(0xffffffffu, bounded_wait(acc_bar, 0));
    tc_fence_after();
    uint32_t v0[32], v1[32];
    const uint32_t tl = tmem + ((uint32_t)(32 * warp) << 16);
    tmem_ld32(tl, v0);
    tmem_ld32(tl + 32, v1);
    tmem_wait_ld();
    const int r = m0 + 32 * warp + lane;
    const size_t bh = (size_t)b * a.H + h;
    if (ok && t < 2) {
      uint32_t w0 = 0u, w1 = 0u;
      if (r < L) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          w0 |= (__uint_as_float(v0[c]) < smu[c] ? 1u : 0u) << c;
          w1 |= (__uint_as_float(v1[c]) < smu[32 + c] ? 1u : 0u) << c;
        }
      }
      if (t == 0) {
        if (r < a.n) *reinterpret_cast<uint2*>(a.qbits + (bh * a.n + r) * 2) = make_uint2(w0, w1);
      } else if (r < a.n_pad) {
        uint4* dst = reinterpret_cast<uint4*>(a.kpm + (bh * a.n_pad + r) * kN);
        const bool e4 = a.k_e4m3 != 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t f = (q < 2 ? w0 : w1) >> ((q & 1) * 16);
          dst[q] = make_uint4(expand_nibble_pm(f & 15u, e4), expand_nibble_pm((f >> 4) & 15u, e4),
                              expand_nibble_pm((f >> 8) & 15u, e4), expand_nibble_pm((f >> 12) & 15u, e4));
        }
      }
    } else if (ok && r < a.n) {
      // V: the bf16 row
      uint4* dst = reinterpret_cast<uint4*>(a.V + (bh * a.n + r) * kN);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t* src = q < 4 ? &v0[8 * q] : &v1[8 * (q - 4)];
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) pk[e] = pack_bf16x2(__uint_as_float(src[2 * e]), __uint_as_float(src[2 * e + 1]));
        dst[q] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
  }

  // teardown: loads still in flight land, every tcgen05 operation completes, TMEM is freed
  if (warp == kProdWarp && lane == 0 && *abort_flag)
    for (int s = 0; s < kStages; ++s)
      if (par[s] >= 0) mbar_wait(&full[s], (uint32_t)par[s], 200000000LL);
  if (warp == kMmaWarp && lane == 0) {
    mma_commit(fin_bar);
    mbar_wait(fin_bar, 0, 200000000LL);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace qkv
}  // namespace had

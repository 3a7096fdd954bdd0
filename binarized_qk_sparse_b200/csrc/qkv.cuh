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
// 32-token chunk; k_mu: the means from those sums, then their fp64 product with
// W in feature slices, added in order and rounded once to fp32 by k_qkv_tc).  Then k_qkv_tc runs the projection on the tensor cores and
// compares each fp32 result with its mean in the epilogue:
//   - Q columns: the 64 sign bits of a token (bit 1 = below the mean), in the
//     attention workspace's packed layout;
//   - K columns: the +-1 row of a token (int8, or e4m3 for the fp8 score path),
//     rows past L (and up to n_pad) +1;
//   - V columns: the bf16 row of V, the attention's V input, and in the uint8
//     modes V's column absmax per head (atomic maxima), from which the
//     quantization of V takes its scales without a statistics pass.
// A CTA takes 128 tokens and 256 output channels (four heads' column blocks): one
// M128 N256 K16 MMA per K-step, so that each X tile serves four blocks.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "prep.cuh"
#include "sm100.cuh"

namespace had {
namespace qkv {

using namespace had::sm100;

constexpr int kXsumChunk = 32;     // tokens per partial sum of X
constexpr int kXsumThreads = 128;  // k_xsum: feature threads (8 features each) per token group
constexpr int kMuB = 16, kMuK = 64;  // k_mu: batches per CTA, features per staged chunk

// Token sums of X over the valid tokens of each 32-token chunk: part[b][ch][k], fp64.
// Thread (g, f) of a CTA adds 8 adjacent features over the g-th 8 tokens of the
// chunk (eight 16-byte loads issued together); the four groups' sums are then
// added in group order.
constexpr int kXsumGroups = kXsumChunk / 8;
__global__ void __launch_bounds__(kXsumThreads * kXsumGroups) k_xsum(const __nv_bfloat16* __restrict__ X, int n,
                                                                     int Dm, int H, const int32_t* seqlens, int nch,
                                                                     double* __restrict__ part,
                                                                     uint32_t* __restrict__ vamax) {
  __shared__ double red[kXsumGroups - 1][8][kXsumThreads];
  if (vamax && blockIdx.x == 0 && blockIdx.y == 0)  // V's column absmax of batch b, raised later by the projection
    for (int e = threadIdx.x; e < H * 64; e += blockDim.x) vamax[(size_t)blockIdx.z * H * 64 + e] = 0u;
  const int ft = threadIdx.x % kXsumThreads, tg = threadIdx.x / kXsumThreads;
  const int k0 = (blockIdx.x * kXsumThreads + ft) * 8, ch = blockIdx.y, b = blockIdx.z;
  const bool act = k0 < Dm;
  const int L = valid_len(seqlens, b, n, nullptr);
  const int i0 = ch * kXsumChunk + tg * 8, i1 = min(i0 + 8, L);
  double s[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) s[u] = 0.0;
  if (act && i0 < i1) {
    // rows past the group's end re-read its last row and are zeroed after the load
    uint4 x[8];
#pragma unroll
    for (int t = 0; t < 8; ++t)
      x[t] = __ldg(reinterpret_cast<const uint4*>(X + ((size_t)b * n + min(i0 + t, i1 - 1)) * Dm + k0));
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (i0 + t >= i1) x[t] = make_uint4(0u, 0u, 0u, 0u);
      const uint32_t w[4] = {x[t].x, x[t].y, x[t].z, x[t].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        s[2 * u] += (double)__uint_as_float(w[u] << 16);
        s[2 * u + 1] += (double)__uint_as_float(w[u] & 0xFFFF0000u);
      }
    }
  }
  if (tg > 0) {
#pragma unroll
    for (int u = 0; u < 8; ++u) red[tg - 1][u][ft] = s[u];
  }
  __syncthreads();
  if (tg == 0 && act) {
#pragma unroll
    for (int g = 0; g < kXsumGroups - 1; ++g)
#pragma unroll
      for (int u = 0; u < 8; ++u) s[u] += red[g][u][ft];
    double* dst = part + ((size_t)b * nch + ch) * Dm + k0;
#pragma unroll
    for (int u = 0; u < 8; u += 2) *reinterpret_cast<double2*>(dst + u) = make_double2(s[u], s[u + 1]);
  }
}

// Partial dot products of the means with W: mupart[z][t][b][h][c] = sum over the
// z-th of kMuSplit feature slices of xbar[b][k] W[o][k], o = t*H*64 + h*64 + c, in
// fp64 on the tensor cores (mma.sync m8n8k4 f64: an 8 x 4 block of means times a
// 4 x 8 block of W per instruction).  k_qkv_tc adds the kMuSplit partials in slice
// order and rounds once to fp32.  A CTA of 8 warps takes 16 batches and 128
// channels of one slice, 64 features at a time: it stages the 16 batches' means
// (the chunk sums of k_xsum added in chunk order, divided by L) in shared memory,
// and warp w takes channels 16w .. 16w + 15 as two 8 x 8 output blocks per batch
// group.  Inside a 32-feature step, the lane with k-slot q (lane % 4) supplies
// features 8q .. 8q + 7 to the step's eight MMAs, one per MMA, for the means and
// for W alike, so that its W piece is one 16-byte load.
constexpr int kMuThreads = 256;
constexpr int kMuO = 128;    // channels per CTA
constexpr int kMuSplit = 8;  // feature slices

__device__ __forceinline__ void dmma_8x8x4(double (&c)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(c[0]), "+d"(c[1])
               : "d"(a), "d"(b));
}

__global__ void __launch_bounds__(kMuThreads) k_mu(const __nv_bfloat16* __restrict__ W,
                                                   const double* __restrict__ part, int nch, int n,
                                                   const int32_t* seqlens, int B, int H, int Dm,
                                                   double* __restrict__ mupart) {
  __shared__ __align__(16) double xs[kMuB][kMuK + 2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int o0 = blockIdx.x * kMuO + 16 * warp, b0 = blockIdx.y * kMuB;
  const int no = 2 * H * 64;
  const int slice = Dm / kMuSplit;  // a multiple of 8 (Dm is a multiple of 64)
  const int kbeg = blockIdx.z * slice, kend = kbeg + slice;
  double acc[2][2][2];  // [batch group][channel group][the lane's two outputs]
#pragma unroll
  for (int mg = 0; mg < 2; ++mg)
#pragma unroll
    for (int ng = 0; ng < 2; ++ng) acc[mg][ng][0] = acc[mg][ng][1] = 0.0;
  for (int k0 = kbeg; k0 < kend; k0 += kMuK) {
    const int kn = min(kMuK, kend - k0);  // a multiple of 8
    // this chunk's W pieces: two 32-feature steps x two channel groups, issued before the staging
    uint4 wv[kMuK / 32][2];
#pragma unroll
    for (int st = 0; st < kMuK / 32; ++st)
#pragma unroll
      for (int ng = 0; ng < 2; ++ng) {
        const int o = o0 + 8 * ng + g, kk = 32 * st + 8 * q;
        wv[st][ng] = (o < no && kk < kn) ? __ldg(reinterpret_cast<const uint4*>(W + (size_t)o * Dm + k0 + kk))
                                         : make_uint4(0u, 0u, 0u, 0u);
      }
    __syncthreads();  // the previous chunk's reads of xs are done
    // the means: the chunk sums of k_xsum added in chunk order, divided by L
    for (int e = threadIdx.x; e < kMuB * kMuK / 2; e += kMuThreads) {
      const int br = e / (kMuK / 2), cc = (e % (kMuK / 2)) * 2, b = b0 + br;
      double2 m = make_double2(0.0, 0.0);
      if (b < B && cc < kn) {
        const int L = valid_len(seqlens, b, n, nullptr);  // the projection reports bad lengths
        const int nv = (L + kXsumChunk - 1) / kXsumChunk;
        for (int c = 0; c < nv; ++c) {
          const double2 p = *reinterpret_cast<const double2*>(part + ((size_t)b * nch + c) * Dm + k0 + cc);
          m.x += p.x;
          m.y += p.y;
        }
        if (L > 0) m = make_double2(m.x / (double)L, m.y / (double)L);
      }
      *reinterpret_cast<double2*>(&xs[br][cc]) = m;
    }
    __syncthreads();
#pragma unroll
    for (int st = 0; st < kMuK / 32; ++st) {
      if (32 * st >= kn) break;  // uniform over the CTA
      double wb[2][8];
#pragma unroll
      for (int ng = 0; ng < 2; ++ng) {
        const uint32_t u[4] = {wv[st][ng].x, wv[st][ng].y, wv[st][ng].z, wv[st][ng].w};
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          wb[ng][2 * v] = (double)__uint_as_float(u[v] << 16);
          wb[ng][2 * v + 1] = (double)__uint_as_float(u[v] & 0xFFFF0000u);
        }
      }
#pragma unroll
      for (int mg = 0; mg < 2; ++mg) {
        double xa[8];
        const double2* xp = reinterpret_cast<const double2*>(&xs[8 * mg + g][32 * st + 8 * q]);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const double2 x2 = xp[v];
          xa[2 * v] = x2.x;
          xa[2 * v + 1] = x2.y;
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
#pragma unroll
          for (int ng = 0; ng < 2; ++ng) dmma_8x8x4(acc[mg][ng], xa[jj], wb[ng][jj]);
      }
    }
  }
  // lane (g, q) holds outputs (batch 8 mg + g, channels 8 ng + 2q, 8 ng + 2q + 1)
#pragma unroll
  for (int mg = 0; mg < 2; ++mg)
#pragma unroll
    for (int ng = 0; ng < 2; ++ng)
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const int b = b0 + 8 * mg + g, o = o0 + 8 * ng + 2 * q + v;
        if (b >= B || o >= no) continue;
        const int t = o / (H * 64), r = o - t * H * 64;  // r = h * 64 + c
        mupart[(((size_t)blockIdx.z * 2 + t) * B + b) * H * 64 + r] = acc[mg][ng][v];
      }
}

// V's codes from the projection's bf16 V and the epilogue's column absmax, as the
// prepare stage makes them (scale absmax/qmax, 1 if the absmax is 0; codes
// rint(V/scale) clamped to +-qmax, 0 past L), transposed to V^T: int8
// [B*H][64][n_pad], or packed 4-bit [B*H][64][n_pad/2] with key 2k in the low
// nibble of byte k.  A CTA takes 64 tokens of one head: each thread reads four
// channels of four tokens, writes their codes into a [64 channels][64 tokens] byte
// tile four tokens at a time, and the tile's rows leave as 16-byte (int8) or
// 8-byte (4-bit) stores.
constexpr int kVcThreads = 256;
__global__ void __launch_bounds__(kVcThreads) k_vcodes(const __nv_bfloat16* __restrict__ V,
                                                       const uint32_t* __restrict__ vamax, int H, int n,
                                                       int n_pad, const int32_t* seqlens, int vbits,
                                                       int8_t* __restrict__ vqT, float* __restrict__ vscale) {
  __shared__ float sc[64], rsc[64];
  __shared__ __align__(16) uint8_t tile[64][64 + 16];
  const int bh = blockIdx.y, i0 = blockIdx.x * 64, tid = threadIdx.x;
  const int L = valid_len(seqlens, bh / H, n, nullptr);  // the projection reported bad lengths
  const float qmax = vbits == 4 ? 7.0f : 127.0f;
  if (tid < 64) {
    const float m = __uint_as_float(vamax[(size_t)bh * 64 + tid]);
    const float s = m > 0.0f ? __fdiv_rn(m, qmax) : 1.0f;
    sc[tid] = s;
    rsc[tid] = 1.0f / s;
    if (blockIdx.x == 0) vscale[(size_t)bh * 64 + tid] = s;
  }
  __syncthreads();
  {
    // thread (channel quad cq, token quad tq): tokens 4tq .. 4tq + 3, channels 4cq .. 4cq + 3 (8-byte
    // loads), then one 4-byte store of four tokens' codes per channel
    const int cq = tid & 15, tq = tid >> 4;
    uint2 x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + 4 * tq + u;
      x[u] = i < L ? __ldg(reinterpret_cast<const uint2*>(V + ((size_t)bh * n + i) * 64 + 4 * cq)) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int c = 4 * cq + v;
      uint32_t w = 0u;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t pr = (v < 2) ? x[u].x : x[u].y;
        const float xv = __uint_as_float((v & 1) ? (pr & 0xFFFF0000u) : (pr << 16));
        w |= ((uint32_t)quant_v(xv, sc[c], rsc[c], qmax) & 0xFFu) << (8 * u);
      }
      // 16-byte chunk k of row c sits at chunk k ^ (c / 4 % 4): the 32 lanes' stores hit 16 banks
      *reinterpret_cast<uint32_t*>(&tile[c][16 * ((tq >> 2) ^ (cq & 3)) + 4 * (tq & 3)]) = w;
    }
  }
  __syncthreads();
  const int c = tid >> 2, seg = tid & 3;  // channel row c, 16 of its 64 tokens
  const uint4 w = *reinterpret_cast<const uint4*>(&tile[c][16 * (seg ^ ((c >> 2) & 3))]);
  if (vbits == 4) {
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
    uint32_t out[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      uint32_t o = 0u;
#pragma unroll
      for (int b = 0; b < 4; ++b) {  // byte b of word k: keys 8k + 2b (low nibble) and 8k + 2b + 1
        const uint32_t wd = in[2 * k + (b >> 1)], sh = (b & 1) * 16;
        o |= (((wd >> sh) & 15u) | (((wd >> (sh + 8)) & 15u) << 4)) << (8 * b);
      }
      out[k] = o;
    }
    uint8_t* dst = reinterpret_cast<uint8_t*>(vqT) + ((size_t)bh * 64 + c) * (n_pad / 2) + i0 / 2 + 8 * seg;
    *reinterpret_cast<uint2*>(dst) = make_uint2(out[0], out[1]);
  } else {
    *reinterpret_cast<uint4*>(vqT + ((size_t)bh * 64 + c) * n_pad + i0 + 16 * seg) = w;
  }
}

// ---------------------------------------------------------------------------- the fused projection

constexpr int kM = 128;        // tokens per CTA (TMEM lanes)
constexpr int kHd = 64;        // a head's channels: one column block of Q, K or V
constexpr int kNB = 4;         // column blocks per CTA
constexpr int kN = kHd * kNB;  // output channels per CTA (one M128 N256 MMA per K-step)
constexpr int kK = 64;         // features per panel (128 bytes of bf16: one 128-byte swizzle row)
constexpr int kStages = 2;     // 2 x 48 KB: two CTAs per SM, so one's epilogue overlaps the other's main loop
constexpr int kThreads = 192;  // warps 0-3: epilogue (TMEM lane quadrants); 4: MMA; 5: TMA
constexpr int kMmaWarp = 4, kProdWarp = 5;
constexpr uint32_t kTmemCols = kN;
constexpr long long kWaitCycles = 2000000000LL;  // bound of a pipeline wait: about one second

struct QkvArgs {
  CUtensorMap tm_x;   // X [B*n][Dm] bf16, box {64, 128}, 128-byte swizzle
  CUtensorMap tm_w;   // W [3*H*64][Dm] bf16, box {64, 256}, 128-byte swizzle
  int B, H, n, n_pad, Dm;
  const int32_t* seqlens;
  const double* mupart;  // [kMuSplit][2][B][H][64]: partial means of Q, then of K (k_mu)
  uint32_t* qbits;    // [B*H][n][2]
  int8_t* kpm;        // [B*H][n_pad][64] +-1 rows of K
  int k_e4m3;         // the +-1 rows as e4m3 (0x38 / 0xB8) instead of int8 (0x01 / 0xFF)
  __nv_bfloat16* V;   // [B][H][n][64]
  uint32_t* vamax;    // [B*H][64] float bits: V's column absmax over the valid tokens (or null)
  unsigned* status;
};

struct QkvSmem {
  static constexpr int kA = 0;                          // kStages x [128 tokens][64 features] bf16
  static constexpr int kB = kA + kStages * kM * kK * 2;  // kStages x [256 channels][64 features] bf16
  static constexpr int kBar = kB + kStages * kN * kK * 2;
  static constexpr int kNumBars = 2 * kStages + 2;       // full, empty, accumulator done, final
  static constexpr int kMu = kBar + kNumBars * 8;        // the 256 columns' means
  static constexpr int kMisc = kMu + kN * 4;             // [0] TMEM base, [1] abort
  static constexpr int kTotal = kMisc + 16 + 1024;       // + alignment slack
};

__global__ void __launch_bounds__(kThreads, 2) k_qkv_tc(const __grid_constant__ QkvArgs a) {
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
  const int m0 = blockIdx.x * kM, b = blockIdx.y, j0 = blockIdx.z * kNB;  // first column block
  const int nblk = 3 * a.H;  // column blocks of Q, K and V: block j is tensor j / H, head j % H
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
      tma_load_2d(sm + QkvSmem::kB + st * kN * kK * 2, &a.tm_w, p * kK, j0 * kHd, &full[st]);
      par[st] = (p / kStages) & 1;
    }
  } else if (warp == kMmaWarp && lane == 0) {
    // D[128 tokens][256 channels] += X panel [128][64] x W panel [256][64]^T: 4 K-steps of 16
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
    // epilogue: thread (warp w, lane l) owns token m0 + 32 w + l, TMEM lane 32 w + l, and
    // takes the CTA's column blocks one after the other.  First the means of the CTA's Q and K
    // columns (the partials added in slice order, one rounding), while the main loop runs
    for (int e = tid; e < kN; e += 128) {
      const int j = j0 + e / kHd, t = j / a.H, h = j - t * a.H;
      double m = 0.0;
      if (j < nblk && t < 2)
        for (int z = 0; z < kMuSplit; ++z)
          m += a.mupart[((((size_t)z * 2 + t) * a.B + b) * a.H + h) * kHd + (e % kHd)];
      smu[e] = (float)m;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
    const bool ok = __all_sync(0xffffffffu, bounded_wait(acc_bar, 0));
    tc_fence_after();
    const uint32_t tl = tmem + ((uint32_t)(32 * warp) << 16);
    const int r = m0 + 32 * warp + lane;
    for (int jb = 0; jb < kNB; ++jb) {
      const int j = j0 + jb;
      if (j >= nblk) break;  // uniform over the CTA
      const int t = j / a.H, h = j - t * a.H;
      uint32_t v0[32], v1[32];
      tmem_ld32(tl + jb * kHd, v0);
      tmem_ld32(tl + jb * kHd + 32, v1);
      tmem_wait_ld();
      const float* mu = smu + jb * kHd;
      const size_t bh = (size_t)b * a.H + h;
      if (ok && t < 2) {
        uint32_t w0 = 0u, w1 = 0u;
        if (r < L) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            w0 |= (__uint_as_float(v0[c]) < mu[c] ? 1u : 0u) << c;
            w1 |= (__uint_as_float(v1[c]) < mu[32 + c] ? 1u : 0u) << c;
          }
        }
        if (t == 0) {
          if (r < a.n) *reinterpret_cast<uint2*>(a.qbits + (bh * a.n + r) * 2) = make_uint2(w0, w1);
        } else if (r < a.n_pad) {
          uint4* dst = reinterpret_cast<uint4*>(a.kpm + (bh * a.n_pad + r) * kHd);
          const bool e4 = a.k_e4m3 != 0;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t f = (q < 2 ? w0 : w1) >> ((q & 1) * 16);
            dst[q] = make_uint4(expand_nibble_pm(f & 15u, e4), expand_nibble_pm((f >> 4) & 15u, e4),
                                expand_nibble_pm((f >> 8) & 15u, e4), expand_nibble_pm((f >> 12) & 15u, e4));
          }
        }
      } else if (ok) {
        // V: the bf16 row
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const uint32_t* src = e < 16 ? &v0[2 * e] : &v1[2 * (e - 16)];
          pk[e] = pack_bf16x2(__uint_as_float(src[0]), __uint_as_float(src[1]));
        }
        if (r < a.n) {
          uint4* dst = reinterpret_cast<uint4*>(a.V + (bh * a.n + r) * kHd);
#pragma unroll
          for (int q = 0; q < 8; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
        if (a.vamax) {
          // the column absmax of the bf16 values over this warp's valid tokens: the warp's 32 rows go
          // through shared memory (the first stage buffer is free once the accumulator is done; 4 KB
          // per warp, 16-byte chunks swizzled by row), then lane l scans columns 2l and 2l + 1 down
          // the rows (magnitude bits, whose order is the values' order) and raises their maxima
          uint32_t* tile = reinterpret_cast<uint32_t*>(sm + QkvSmem::kA) + warp * 32 * 32;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4*>(tile + lane * 32 + ((q ^ (lane & 7)) << 2)) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          __syncwarp();
          const int nvalid = min(32, L - (m0 + 32 * warp));  // rows of this warp below L
          uint32_t mlo = 0u, mhi = 0u;
          for (int rr = 0; rr < nvalid; ++rr) {
            const uint32_t wv = tile[rr * 32 + ((((lane >> 2) ^ (rr & 7)) << 2) | (lane & 3))];
            mlo = max(mlo, wv & 0x7FFFu);
            mhi = max(mhi, (wv >> 16) & 0x7FFFu);
          }
          __syncwarp();
          if (mlo) atomicMax(a.vamax + bh * kHd + 2 * lane, mlo << 16);
          if (mhi) atomicMax(a.vamax + bh * kHd + 2 * lane + 1, mhi << 16);
        }
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

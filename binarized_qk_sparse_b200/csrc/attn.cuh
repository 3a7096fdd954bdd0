// attn.cuh -- the fused binarized-QK top-N attention kernel (sm_100a).
//
// One CTA = one (batch, head) and a tile of 64 query rows (4 warps x 16 rows).
// Keys stream through shared memory in tiles of 64 (double-buffered cp.async):
// the +-1 int8 K~ rows (64 B/key) and, for the A.V pass, the V tile (bf16,
// XOR-swizzled for conflict-free ldmatrix.trans) or the int8 V^T tile.
//
// Score  : s = q~ . k~ on the int8 tensor cores (mma.sync m16n8k32 s8.s8.s32,
//          two k-steps for d = 64).  For +-1 vectors this is exactly
//          d - 2*popcount(q XOR k) (BinaryAttention §2.1/§2.2).
// Logit  : l = fmaf(s, c, b_ij) (BinaryAttention §2.3), bias from the
//          relative-position table (one gather per score).
// Top-N  : (HAD, top-N per query, ties to the lower key index)
//   no bias  -> pass 1 builds, per row, a histogram of the 65 score levels
//               (lane-private counters, conflict-free smem atomics); the
//               threshold level F and the number r_F of keys to keep at F
//               follow from prefix counts.
//   bias     -> pass 1 histogram of score levels bounds the threshold to a
//               band [fmaf(s_N,c,bmin), fmaf(s_max,c,bmax)]; then radix passes
//               over the order-preserving uint32 key of l (256 bins) narrow it
//               until the threshold bin holds <= 64 keys, which are collected
//               and ranked exactly.
//   Keys with l > F are kept; keys with l == F are kept in key order while
//   their rank among the ties is < r_F (a quad-lane prefix count in pass 2).
// Softmax: exp2 on the MUFU; float mode normalizes at the end, uint8 mode needs
//          the normalizer first (A = floor(255 p + 0.5), BinaryAttention §2.4).
// A.V    : float -> bf16 P x bf16 V (mma.sync m16n8k16, fp32 accumulate;
//          fp32 V uses a hi/lo bf16 split, 3 MMAs); uint8 -> u8 A x s8 V
//          (mma.sync m16n8k32 u8.s8.s32, exact int32 accumulate), dequantized
//          by the per-channel V scale / 255.
#pragma once

#include "common.cuh"

namespace had {

constexpr int kQT = 64;             // query rows per CTA
constexpr int kKT = 64;             // keys per tile
constexpr int kAttnThreads = 128;   // 4 warps
constexpr int kRadixBins = 256;
constexpr int kCandCap = 64;        // candidates collected per row in the final radix step

enum { SEL_DENSE = 0, SEL_TOPN_INT = 1, SEL_TOPN_FLOAT = 2 };
enum { MODE_F = 0, MODE_Q = 1 };
enum { EXP_NONE = 0, EXP_IDX = 1, EXP_CODES = 2 };

struct AttnArgs {
  const uint32_t* qbits;   // [BH][n][2]
  const int8_t* kpm;       // [BH][n_pad][64] +-1 int8
  const void* V;           // [BH][n][64] bf16 / fp32   (float mode)
  const int8_t* vqT;       // [BH][64][n_pad]           (uint8 mode)
  const float* vscale;     // [BH][64]
  const float* table;      // [H][th][tw] or null
  int gh, gw, prefix, th, tw;
  const float* bminmax;    // [H][2]
  const int32_t* seqlens;
  void* O;
  int o_bf16;
  int32_t* idx;            // EXP_IDX  [BH][n][N]
  uint8_t* codes;          // EXP_CODES [BH][row_end-row_begin][n]
  int row_begin, row_end;
  int B, H, n, n_pad, N;
  unsigned* status;
  float c_head[kMaxHeads];
};

// Shared-memory layout (bytes) for one CTA.
template <int MODE, bool V_F32>
struct SmemLayout {
  static constexpr int kK = kKT * kD;                                      // K~ tile
  static constexpr int kV = (MODE == MODE_Q) ? kD * kKT : (V_F32 ? 2 : 1) * kKT * kD * 2;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + 2 * kK;
  static constexpr int kOffKoff = kOffV + 2 * kV;
  static constexpr int kOffRow = kOffKoff + 2 * kKT * 4;
  static constexpr int kRowFields = 12;
  static constexpr int kOffHist = kOffRow + kQT * kRowFields * 4;
  static constexpr int kHistBytes = 65 * kQT * 4 * 4;                       // [65 levels][64 rows x 4 lanes]
  static constexpr int kTotalDense = kOffHist;
  static constexpr int kTotalTopN = kOffHist + kHistBytes;
  static_assert(kQT * kRadixBins * 4 <= kHistBytes, "radix histogram must fit in the level histogram area");
  static_assert(kQT * kCandCap * 8 <= kHistBytes, "candidate buffer must fit in the level histogram area");
};

// Per-row state kept in shared memory between passes.
enum {
  RF_F = 0,       // float threshold F
  RF_M,           // softmax shift m
  RF_SCALE,       // 255/l (uint8 mode) or 1/l (float, top-N int)
  RF_RF,          // int: keys to keep among l == F
  RF_CUT,         // int: 1 if the ties at F must be cut by key order
  RF_UHI,         // radix: upper key
  RF_SPAN,        // radix: span (u_hi - u_lo)
  RF_SHIFT,       // radix: shift
  RF_RANK,        // radix: 1-based rank still to find inside the range
  RF_STATE,       // radix: 0 done, 1 refine, 2 collect
  RF_BIN,         // radix: target bin
  RF_L            // float: sum of e over kept (pass 1d)
};

__device__ __forceinline__ float rowf(const uint8_t* smem, int off, int field, int r) {
  return reinterpret_cast<const float*>(smem + off)[field * kQT + r];
}
__device__ __forceinline__ int rowi(const uint8_t* smem, int off, int field, int r) {
  return reinterpret_cast<const int*>(smem + off)[field * kQT + r];
}
__device__ __forceinline__ float* rowfp(uint8_t* smem, int off, int field) {
  return reinterpret_cast<float*>(smem + off) + field * kQT;
}
__device__ __forceinline__ int* rowip(uint8_t* smem, int off, int field) {
  return reinterpret_cast<int*>(smem + off) + field * kQT;
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gmem_src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Tile-local key index of score column `col` (0..7) of n-block `nb` (0..7).
// Float mode: natural order.  Uint8 mode: each 32-key chunk interleaves four
// n-blocks so that lane q's C-fragment scores form the A-fragment bytes
// (keys 4q..4q+3 and 16+4q..16+4q+3) of the u8 x s8 MMA.
template <int MODE>
__device__ __forceinline__ int key_of(int nb, int col) {
  if (MODE == MODE_F) return nb * 8 + col;
  int cc = nb >> 2, x = nb & 3;
  return cc * 32 + ((x >> 1) << 4) + ((col >> 1) << 2) + ((x & 1) << 1) + (col & 1);
}

// Order of a key inside its prefix group ("group" = keys whose scores the 4
// lanes of a quad hold as contiguous runs): float mode groups are one n-block
// (lane q holds 2 keys), uint8 mode groups are two n-blocks (lane q holds 4 keys).
template <int MODE>
struct Groups {
  static constexpr int kNBPerGroup = (MODE == MODE_F) ? 1 : 2;
  static constexpr int kGroups = 8 / kNBPerGroup;
  static constexpr int kPerLane = 2 * kNBPerGroup;
  // score slot (nb_in_group, col bit) of the lane's u-th key (key order)
  __device__ static __forceinline__ int nb_of(int g, int u) {
    if (MODE == MODE_F) return g;
    // group g covers n-blocks {A,B} (g even) or {C,D} (g odd) of chunk g>>1
    return (g >> 1) * 4 + ((g & 1) << 1) + (u >> 1);
  }
};

template <int SEL, int MODE, bool HAS_BIAS, bool V_F32, int EXPORT>
__global__ void __launch_bounds__(kAttnThreads) k_attn(const __grid_constant__ AttnArgs a) {
  using SL = SmemLayout<MODE, V_F32>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int q0 = blockIdx.x * kQT;
  const int L = valid_len(a.seqlens, b, a.n, a.status);
  const float c = a.c_head[h];
  const int lr0 = warp * 16 + g, lr1 = lr0 + 8;
  const int i0 = q0 + lr0, i1 = q0 + lr1;
  const bool row_ok0 = i0 < L, row_ok1 = i1 < L;
  const int keff = (a.N == 0 || a.N >= L) ? L : a.N;

  // ---- rows past the valid length: zero output (and -1 indices / zero codes)
  if (q0 >= L) {
    if (EXPORT == EXP_NONE) {
      for (int e = tid; e < kQT * kD; e += kAttnThreads) {
        int r = q0 + e / kD, ch = e % kD;
        if (r < a.n) {
          size_t o = ((size_t)bh * a.n + r) * kD + ch;
          if (a.o_bf16) reinterpret_cast<__nv_bfloat16*>(a.O)[o] = __float2bfloat16(0.0f);
          else reinterpret_cast<float*>(a.O)[o] = 0.0f;
        }
      }
    } else if (EXPORT == EXP_IDX) {
      for (int e = tid; e < kQT * a.N; e += kAttnThreads) {
        int r = q0 + e / a.N;
        if (r < a.n) a.idx[((size_t)bh * a.n + r) * a.N + e % a.N] = -1;
      }
    } else {
      int rows = a.row_end - a.row_begin;
      for (int e = tid; e < kQT * a.n; e += kAttnThreads) {
        int r = q0 + e / a.n;
        if (r >= a.row_begin && r < a.row_end && r < a.n)
          a.codes[((size_t)bh * rows + (r - a.row_begin)) * a.n + e % a.n] = 0;
      }
    }
    return;
  }

  // ---- Q~ A-fragments from the packed bits (+-1 int8, lane q holds channels 16q..16q+15)
  uint32_t qa[2][4];
  {
    auto field = [&](int i) -> uint32_t {
      if (i >= L) return 0u;
      const uint2 w = __ldg(reinterpret_cast<const uint2*>(a.qbits + ((size_t)bh * a.n + i) * kW));
      uint32_t word = (q < 2) ? w.x : w.y;
      return (word >> ((q & 1) * 16)) & 0xFFFFu;
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

  // ---- relative-position bias: b_ij = table[h][rowbase_i - keyoff_j] (0 for prefix tokens)
  const float* tab = HAS_BIAS ? a.table + (size_t)h * a.th * a.tw : nullptr;
  int rb0 = -1, rb1 = -1;  // -1: row is a prefix token (bias 0)
  if (HAS_BIAS) {
    if (i0 >= a.prefix && i0 < a.n) {
      int t = i0 - a.prefix, y = t / a.gw, x = t % a.gw;
      rb0 = (y + a.gh - 1) * a.tw + (x + a.gw - 1);
    }
    if (i1 >= a.prefix && i1 < a.n) {
      int t = i1 - a.prefix, y = t / a.gw, x = t % a.gw;
      rb1 = (y + a.gh - 1) * a.tw + (x + a.gw - 1);
    }
  }

  const int ntiles = (L + kKT - 1) / kKT;
  const int8_t* kpm = a.kpm + (size_t)bh * a.n_pad * kD;

  // ---- tile loader (cp.async, 16-byte chunks)
  auto load_tile = [&](int buf, int t, bool with_v) {
    const int j0 = t * kKT;
    int8_t* kt = reinterpret_cast<int8_t*>(smem + SL::kOffK + buf * SL::kK);
    for (int e = tid; e < kKT * kD / 16; e += kAttnThreads) {
      int r = e >> 2, ch = e & 3;
      cp_async16(kt + r * kD + ch * 16, kpm + (size_t)(j0 + r) * kD + ch * 16);
    }
    if (HAS_BIAS && tid < kKT) {
      int j = j0 + tid, off = INT_MIN;
      if (j >= a.prefix && j < a.n) {
        int tt = j - a.prefix, y = tt / a.gw, x = tt % a.gw;
        off = y * a.tw + x;
      }
      reinterpret_cast<int*>(smem + SL::kOffKoff)[buf * kKT + tid] = off;
    }
    if (with_v) {
      uint8_t* vt = smem + SL::kOffV + buf * SL::kV;
      if (MODE == MODE_Q) {
        const int8_t* src = a.vqT + (size_t)bh * kD * a.n_pad + j0;
        for (int e = tid; e < kD * kKT / 16; e += kAttnThreads) {
          int chn = e >> 2, seg = e & 3;
          int phys = seg ^ ((chn >> 1) & 3);
          cp_async16(vt + chn * kKT + phys * 16, src + (size_t)chn * a.n_pad + seg * 16);
        }
      } else if (!V_F32) {
        const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(a.V) + (size_t)bh * a.n * kD;
        for (int e = tid; e < kKT * 8; e += kAttnThreads) {
          int r = e >> 3, seg = e & 7;
          uint8_t* dst = vt + r * 128 + ((seg ^ (r & 7)) * 16);
          if (j0 + r < L) cp_async16(dst, src + (size_t)(j0 + r) * kD + seg * 8);
          else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
      } else {
        const float* src = reinterpret_cast<const float*>(a.V) + (size_t)bh * a.n * kD;
        uint8_t* vlo = vt + kKT * kD * 2;
        for (int e = tid; e < kKT * 8; e += kAttnThreads) {
          int r = e >> 3, seg = e & 7;
          float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f), x1 = x0;
          if (j0 + r < L) {
            x0 = __ldg(reinterpret_cast<const float4*>(src + (size_t)(j0 + r) * kD + seg * 8));
            x1 = __ldg(reinterpret_cast<const float4*>(src + (size_t)(j0 + r) * kD + seg * 8 + 4));
          }
          float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            __nv_bfloat162 hv = __floats2bfloat162_rn(xs[2 * u], xs[2 * u + 1]);
            float2 hf = __bfloat1622float2(hv);
            __nv_bfloat162 lv = __floats2bfloat162_rn(xs[2 * u] - hf.x, xs[2 * u + 1] - hf.y);
            hi[u] = *reinterpret_cast<uint32_t*>(&hv);
            lo[u] = *reinterpret_cast<uint32_t*>(&lv);
          }
          const int off = r * 128 + ((seg ^ (r & 7)) * 16);
          *reinterpret_cast<uint4*>(vt + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(vlo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
    }
    cp_async_commit();
  };

  // ---- scores of one tile: sc[nb][0..3] for rows lr0 (0,1) and lr1 (2,3)
  auto tile_scores = [&](int buf, int (&sc)[8][4]) {
    const int8_t* kt = reinterpret_cast<const int8_t*>(smem + SL::kOffK + buf * SL::kK);
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      const uint4 kb = *reinterpret_cast<const uint4*>(kt + key_of<MODE>(nb, g) * kD + q * 16);
      sc[nb][0] = sc[nb][1] = sc[nb][2] = sc[nb][3] = 0;
      mma_s8_16x8x32(sc[nb], qa[0], kb.x, kb.y);
      mma_s8_16x8x32(sc[nb], qa[1], kb.z, kb.w);
    }
  };

  // logit of score slot e (0..3) in n-block nb of tile t
  auto logit = [&](int buf, int nb, int e, int s) -> float {
    if (!HAS_BIAS) return (float)s * c;
    const int koff = reinterpret_cast<const int*>(smem + SL::kOffKoff)[buf * kKT + key_of<MODE>(nb, 2 * q + (e & 1))];
    const int rb = (e < 2) ? rb0 : rb1;
    float bval = 0.0f;
    if (rb >= 0 && koff != INT_MIN) bval = __ldg(tab + (rb - koff));
    return __fmaf_rn((float)s, c, bval);
  };

  float* rF = rowfp(smem, SL::kOffRow, RF_F);
  float* rM = rowfp(smem, SL::kOffRow, RF_M);
  float* rS = rowfp(smem, SL::kOffRow, RF_SCALE);
  int* rR = rowip(smem, SL::kOffRow, RF_RF);
  int* rC = rowip(smem, SL::kOffRow, RF_CUT);
  const float kLog2e = 1.4426950408889634f;

  // =========================================================================
  // Pass 1 (top-N): histogram of score levels per row
  // =========================================================================
  if (SEL != SEL_DENSE) {
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + SL::kOffHist);
    for (int e = tid; e < 65 * kQT * 4; e += kAttnThreads) hist[e] = 0u;
    __syncthreads();
    // hist[level][row*4 + lane] with level = (64 - s) / 2; byte address = base - s * 512
    const uint32_t hb = (uint32_t)__cvta_generic_to_shared(hist);
    const uint32_t base0 = hb + (uint32_t)(lr0 * 4 + q) * 4u + 32u * 1024u;
    const uint32_t base1 = hb + (uint32_t)(lr1 * 4 + q) * 4u + 32u * 1024u;
    load_tile(0, 0, false);
    for (int t = 0; t < ntiles; ++t) {
      if (t + 1 < ntiles) { load_tile((t + 1) & 1, t + 1, false); cp_async_wait<1>(); }
      else cp_async_wait<0>();
      __syncthreads();
      int sc[8][4];
      tile_scores(t & 1, sc);
      const bool full = (t + 1) * kKT <= L;
#pragma unroll
      for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = t * kKT + key_of<MODE>(nb, 2 * q + (e & 1));
          const bool ok = (e < 2 ? row_ok0 : row_ok1) && (full || j < L);
          if (ok) {
            uint32_t addr = (e < 2 ? base0 : base1) - (uint32_t)(sc[nb][e] * 512);
            asm volatile("red.shared.add.u32 [%0], 1;\n" ::"r"(addr));
          }
        }
      }
      __syncthreads();
    }
    // ---- per-row threshold from the level histogram (one thread per row)
    if (tid < kQT) {
      const int r = tid, i = q0 + r;
      float F = -INFINITY, m = 0.0f, scale = 1.0f;
      int rfv = 0, cut = 0;
      int state = 0;
      if (i < L) {
        auto cnt = [&](int lev) -> int {
          const uint32_t* hrow = hist + lev * (kQT * 4) + r * 4;
          return (int)(hrow[0] + hrow[1] + hrow[2] + hrow[3]);
        };
        int hmin = 0;
        while (hmin < 64 && cnt(hmin) == 0) ++hmin;
        int cum = 0, hN = 64;
        for (int lev = 0; lev <= 64; ++lev) {
          cum += cnt(lev);
          if (cum >= keff) { hN = lev; break; }
        }
        const int smax = 64 - 2 * hmin, sN = 64 - 2 * hN;
        if (SEL == SEL_TOPN_INT) {
          F = (float)sN * c;
          int gt = 0, eq = 0;
          for (int lev = 0; lev <= 64; ++lev) {
            const float lv = (float)(64 - 2 * lev) * c;
            const int k = cnt(lev);
            if (lv > F) gt += k;
            else if (lv == F) eq += k;
          }
          rfv = keff - gt;
          cut = rfv < eq ? 1 : 0;
          m = (float)smax * c;
          float lsum = 0.0f;
          for (int lev = 0; lev <= 64; ++lev) {
            const float lv = (float)(64 - 2 * lev) * c;
            if (lv > F) lsum += (float)cnt(lev) * fast_exp2((lv - m) * kLog2e);
          }
          lsum += (float)rfv * fast_exp2((F - m) * kLog2e);
          scale = (MODE == MODE_Q) ? 255.0f / lsum : 1.0f / lsum;
        } else {
          // band for the float radix select
          const float bmin = a.bminmax[2 * h], bmax = a.bminmax[2 * h + 1];
          const float lo = __fmaf_rn((float)sN, c, bmin);
          const float hi = __fmaf_rn((float)smax, c, bmax);
          const uint32_t ulo = float_order_key(lo), uhi = float_order_key(hi);
          const uint32_t span = uhi - ulo;
          int shift = 0;
          while ((span >> shift) >= (uint32_t)kRadixBins) ++shift;
          rowip(smem, SL::kOffRow, RF_UHI)[r] = (int)uhi;
          rowip(smem, SL::kOffRow, RF_SPAN)[r] = (int)span;
          rowip(smem, SL::kOffRow, RF_SHIFT)[r] = shift;
          rowip(smem, SL::kOffRow, RF_RANK)[r] = keff;
          m = hi;
          state = 1;
        }
      }
      rF[r] = F; rM[r] = m; rS[r] = scale; rR[r] = rfv; rC[r] = cut;
      rowip(smem, SL::kOffRow, RF_STATE)[r] = state;
    }
    __syncthreads();

    // =========================================================================
    // Pass 1b / 1c (top-N with bias): radix refinement over order-preserving keys
    // =========================================================================
    if (SEL == SEL_TOPN_FLOAT) {
      int* rUhi = rowip(smem, SL::kOffRow, RF_UHI);
      int* rSpan = rowip(smem, SL::kOffRow, RF_SPAN);
      int* rShift = rowip(smem, SL::kOffRow, RF_SHIFT);
      int* rRank = rowip(smem, SL::kOffRow, RF_RANK);
      int* rState = rowip(smem, SL::kOffRow, RF_STATE);
      int* rBin = rowip(smem, SL::kOffRow, RF_BIN);
      uint32_t* rh = reinterpret_cast<uint32_t*>(smem + SL::kOffHist);       // [64 rows][256]
      uint2* cand = reinterpret_cast<uint2*>(smem + SL::kOffHist);           // [64 rows][64] (u, j)
      for (int iter = 0; iter < 6; ++iter) {
        const int any_refine = __syncthreads_or(tid < kQT && rState[tid] == 1);
        if (!any_refine) break;
        for (int e = tid; e < kQT * kRadixBins; e += kAttnThreads) rh[e] = 0u;
        __syncthreads();
        const bool act0 = row_ok0 && rState[lr0] == 1, act1 = row_ok1 && rState[lr1] == 1;
        const uint32_t uhi0 = (uint32_t)rUhi[lr0], uhi1 = (uint32_t)rUhi[lr1];
        const uint32_t sp0 = (uint32_t)rSpan[lr0], sp1 = (uint32_t)rSpan[lr1];
        const int sh0 = rShift[lr0], sh1 = rShift[lr1];
        const bool warp_act = __any_sync(0xffffffffu, act0 || act1);
        load_tile(0, 0, false);
        for (int t = 0; t < ntiles; ++t) {
          if (t + 1 < ntiles) { load_tile((t + 1) & 1, t + 1, false); cp_async_wait<1>(); }
          else cp_async_wait<0>();
          __syncthreads();
          if (warp_act) {
            int sc[8][4];
            tile_scores(t & 1, sc);
#pragma unroll
            for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = t * kKT + key_of<MODE>(nb, 2 * q + (e & 1));
                const bool act = (e < 2) ? act0 : act1;
                if (act && j < L) {
                  const uint32_t u = float_order_key(logit(t & 1, nb, e, sc[nb][e]));
                  const uint32_t dd = ((e < 2) ? uhi0 : uhi1) - u;
                  if (dd <= ((e < 2) ? sp0 : sp1)) {
                    const uint32_t bin = dd >> ((e < 2) ? sh0 : sh1);
                    atomicAdd(&rh[((e < 2) ? lr0 : lr1) * kRadixBins + bin], 1u);
                  }
                }
              }
            }
          }
          __syncthreads();
        }
        // choose the bin holding the target rank; refine, finish, or collect
        if (tid < kQT && rState[tid] == 1) {
          const int r = tid;
          int rank = rRank[r], cum = 0, bsel = kRadixBins - 1;
          for (int bb = 0; bb < kRadixBins; ++bb) {
            const int k = (int)rh[r * kRadixBins + bb];
            if (cum + k >= rank) { bsel = bb; break; }
            cum += k;
          }
          const int kbin = (int)rh[r * kRadixBins + bsel];
          rank -= cum;
          const int shift = rShift[r];
          const uint32_t uhi = (uint32_t)rUhi[r] - ((uint32_t)bsel << shift);
          if (shift == 0) {
            // a single float value: F known, keep the first `rank` of its `kbin` ties
            const uint32_t uF = uhi;
            const uint32_t bits = (uF & 0x80000000u) ? (uF & 0x7FFFFFFFu) : ~uF;
            rF[r] = __uint_as_float(bits);
            rR[r] = rank;
            rC[r] = rank < kbin ? 1 : 0;
            rState[r] = 0;
          } else if (kbin <= kCandCap) {
            rBin[r] = bsel;
            rRank[r] = rank;
            rState[r] = 2;
          } else {
            const int nshift = shift > 8 ? shift - 8 : 0;
            const uint32_t span_left = (uint32_t)rSpan[r] - ((uint32_t)bsel << shift);
            rUhi[r] = (int)uhi;
            rSpan[r] = (int)min(((uint32_t)1 << shift) - 1u, span_left);
            rShift[r] = nshift;
            rRank[r] = rank;
          }
        }
      }
      // ---- collect the candidates of rows in state 2 and rank them exactly
      const int any_collect = __syncthreads_or(tid < kQT && rState[tid] == 2);
      if (any_collect) {
        int* ccount = rowip(smem, SL::kOffRow, RF_L);
        if (tid < kQT) ccount[tid] = 0;
        __syncthreads();
        const bool act0 = row_ok0 && rState[lr0] == 2, act1 = row_ok1 && rState[lr1] == 2;
        const uint32_t uhi0 = (uint32_t)rUhi[lr0], uhi1 = (uint32_t)rUhi[lr1];
        const uint32_t sp0 = (uint32_t)rSpan[lr0], sp1 = (uint32_t)rSpan[lr1];
        const int sh0 = rShift[lr0], sh1 = rShift[lr1];
        const uint32_t bin0 = (uint32_t)rBin[lr0], bin1 = (uint32_t)rBin[lr1];
        const bool warp_act = __any_sync(0xffffffffu, act0 || act1);
        load_tile(0, 0, false);
        for (int t = 0; t < ntiles; ++t) {
          if (t + 1 < ntiles) { load_tile((t + 1) & 1, t + 1, false); cp_async_wait<1>(); }
          else cp_async_wait<0>();
          __syncthreads();
          if (warp_act) {
            int sc[8][4];
            tile_scores(t & 1, sc);
#pragma unroll
            for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = t * kKT + key_of<MODE>(nb, 2 * q + (e & 1));
                const bool act = (e < 2) ? act0 : act1;
                if (act && j < L) {
                  const uint32_t u = float_order_key(logit(t & 1, nb, e, sc[nb][e]));
                  const uint32_t dd = ((e < 2) ? uhi0 : uhi1) - u;
                  if (dd <= ((e < 2) ? sp0 : sp1) && (dd >> ((e < 2) ? sh0 : sh1)) == ((e < 2) ? bin0 : bin1)) {
                    const int r = (e < 2) ? lr0 : lr1;
                    const int pos = atomicAdd(&ccount[r], 1);
                    if (pos < kCandCap) cand[r * kCandCap + pos] = make_uint2(u, (uint32_t)j);
                  }
                }
              }
            }
          }
          __syncthreads();
        }
        if (tid < kQT && rState[tid] == 2) {
          const int r = tid;
          const int nc = min(ccount[r], kCandCap);
          if (ccount[r] > kCandCap) raise_status(a.status, kDevErrCapacity);
          const int rank = rRank[r];
          // the rank-th element of (u desc, j asc): count how many precede each candidate
          uint32_t uF = 0u;
          for (int x = 0; x < nc; ++x) {
            const uint2 cx = cand[r * kCandCap + x];
            int before = 0;
            for (int y = 0; y < nc; ++y) {
              const uint2 cy = cand[r * kCandCap + y];
              before += (cy.x > cx.x || (cy.x == cx.x && cy.y < cx.y)) ? 1 : 0;
            }
            if (before == rank - 1) uF = cx.x;
          }
          int gt = 0, eq = 0;
          for (int x = 0; x < nc; ++x) {
            const uint32_t ux = cand[r * kCandCap + x].x;
            gt += ux > uF ? 1 : 0;
            eq += ux == uF ? 1 : 0;
          }
          const uint32_t bits = (uF & 0x80000000u) ? (uF & 0x7FFFFFFFu) : ~uF;
          rF[r] = __uint_as_float(bits);
          rR[r] = rank - gt;
          rC[r] = (rank - gt) < eq ? 1 : 0;
          rState[r] = 0;
        }
        __syncthreads();
      }
    }
  }

  // ---- quad prefix helper: exclusive prefix and total of (cnt0 | cnt1 << 16) over lanes q = 0..3
  auto quad_scan = [&](uint32_t v, uint32_t& excl, uint32_t& total) {
    uint32_t incl = v;
    uint32_t t1 = __shfl_up_sync(0xffffffffu, incl, 1, 4);
    if (q >= 1) incl += t1;
    uint32_t t2 = __shfl_up_sync(0xffffffffu, incl, 2, 4);
    if (q >= 2) incl += t2;
    total = __shfl_sync(0xffffffffu, incl, 3, 4);
    excl = incl - v;
  };

  // keep mask of a tile for rows lr0/lr1 in key order, maintaining the per-row tie counters
  // kept[nb][e]: 1 if kept; logits in lg[nb][e]
  float F0 = -INFINITY, F1 = -INFINITY;
  int rf0 = 0, rf1 = 0, cut0 = 0, cut1 = 0;
  float m0 = 0.0f, m1 = 0.0f, sc0 = 1.0f, sc1 = 1.0f;
  if (SEL != SEL_DENSE) {
    F0 = rF[lr0]; F1 = rF[lr1];
    rf0 = rR[lr0]; rf1 = rR[lr1];
    cut0 = rC[lr0]; cut1 = rC[lr1];
    m0 = rM[lr0]; m1 = rM[lr1];
    sc0 = rS[lr0]; sc1 = rS[lr1];
  }
  const bool warp_cut = __any_sync(0xffffffffu, (cut0 && row_ok0) || (cut1 && row_ok1));
  uint32_t tie_run = 0;   // ties at F seen so far, row lr0 in bits 0..15, lr1 in 16..31
  uint32_t kept_run = 0;  // kept keys so far (index export)

  auto keep_tile = [&](int t, const float (&lg)[8][4], uint32_t (&keep)[8]) {
    const bool full = (t + 1) * kKT <= L;
    using G = Groups<MODE>;
#pragma unroll
    for (int gi = 0; gi < G::kGroups; ++gi) {
      // per lane: G::kPerLane keys per row, in key order u = 0.. (nb_of(gi,u), col bit u&1)
      uint32_t tie0 = 0, tie1 = 0, kp0 = 0, kp1 = 0;
#pragma unroll
      for (int u = 0; u < G::kPerLane; ++u) {
        const int nb = G::nb_of(gi, u);
        const int col = u & 1;
        const int j = t * kKT + key_of<MODE>(nb, 2 * q + col);
        const bool vj = full || j < L;
        const float l0 = lg[nb][col], l1 = lg[nb][2 + col];
        if (SEL == SEL_DENSE) {
          kp0 |= (vj ? 1u : 0u) << u;
          kp1 |= (vj ? 1u : 0u) << u;
        } else {
          kp0 |= (vj && l0 > F0 ? 1u : 0u) << u;
          kp1 |= (vj && l1 > F1 ? 1u : 0u) << u;
          tie0 |= (vj && l0 == F0 ? 1u : 0u) << u;
          tie1 |= (vj && l1 == F1 ? 1u : 0u) << u;
        }
      }
      if (SEL != SEL_DENSE) {
        if (warp_cut) {
          uint32_t excl, total;
          quad_scan((uint32_t)__popc(tie0) | ((uint32_t)__popc(tie1) << 16), excl, total);
          int base0 = (int)(tie_run & 0xFFFFu) + (int)(excl & 0xFFFFu);
          int base1 = (int)(tie_run >> 16) + (int)(excl >> 16);
#pragma unroll
          for (int u = 0; u < G::kPerLane; ++u) {
            if ((tie0 >> u) & 1u) { if (!cut0 || base0 < rf0) kp0 |= 1u << u; ++base0; }
            if ((tie1 >> u) & 1u) { if (!cut1 || base1 < rf1) kp1 |= 1u << u; ++base1; }
          }
          tie_run += total;
        } else {
          kp0 |= tie0;
          kp1 |= tie1;
        }
      }
      if (!row_ok0) kp0 = 0;
      if (!row_ok1) kp1 = 0;
      keep[gi] = kp0 | (kp1 << 16);
    }
  };

  // =========================================================================
  // Dense uint8 (or top-N-with-bias uint8): normalizer pass
  // =========================================================================
  if (MODE == MODE_Q && (SEL == SEL_DENSE || SEL == SEL_TOPN_FLOAT)) {
    float mx0 = -INFINITY, mx1 = -INFINITY, s0 = 0.0f, s1 = 0.0f;
    if (SEL == SEL_TOPN_FLOAT) { mx0 = m0; mx1 = m1; }
    uint32_t tie_save = tie_run;
    load_tile(0, 0, false);
    for (int t = 0; t < ntiles; ++t) {
      if (t + 1 < ntiles) { load_tile((t + 1) & 1, t + 1, false); cp_async_wait<1>(); }
      else cp_async_wait<0>();
      __syncthreads();
      int sc[8][4];
      tile_scores(t & 1, sc);
      float lg[8][4];
#pragma unroll
      for (int nb = 0; nb < 8; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) lg[nb][e] = logit(t & 1, nb, e, sc[nb][e]);
      uint32_t keep[8];
      keep_tile(t, lg, keep);
      using G = Groups<MODE>;
      if (SEL == SEL_DENSE) {
        float tm0 = -INFINITY, tm1 = -INFINITY;
#pragma unroll
        for (int gi = 0; gi < G::kGroups; ++gi)
#pragma unroll
          for (int u = 0; u < G::kPerLane; ++u) {
            const int nb = G::nb_of(gi, u), col = u & 1;
            if ((keep[gi] >> u) & 1u) tm0 = fmaxf(tm0, lg[nb][col]);
            if ((keep[gi] >> (16 + u)) & 1u) tm1 = fmaxf(tm1, lg[nb][2 + col]);
          }
        if (tm0 > mx0) { s0 *= fast_exp2((mx0 - tm0) * kLog2e); mx0 = tm0; }
        if (tm1 > mx1) { s1 *= fast_exp2((mx1 - tm1) * kLog2e); mx1 = tm1; }
      }
#pragma unroll
      for (int gi = 0; gi < G::kGroups; ++gi)
#pragma unroll
        for (int u = 0; u < G::kPerLane; ++u) {
          const int nb = G::nb_of(gi, u), col = u & 1;
          if ((keep[gi] >> u) & 1u) s0 += fast_exp2((lg[nb][col] - mx0) * kLog2e);
          if ((keep[gi] >> (16 + u)) & 1u) s1 += fast_exp2((lg[nb][2 + col] - mx1) * kLog2e);
        }
      __syncthreads();
    }
    // combine the 4 lanes of each row
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
      float om0 = __shfl_xor_sync(0xffffffffu, mx0, o), os0 = __shfl_xor_sync(0xffffffffu, s0, o);
      float om1 = __shfl_xor_sync(0xffffffffu, mx1, o), os1 = __shfl_xor_sync(0xffffffffu, s1, o);
      float nm0 = fmaxf(mx0, om0), nm1 = fmaxf(mx1, om1);
      s0 = (mx0 == -INFINITY ? 0.0f : s0 * fast_exp2((mx0 - nm0) * kLog2e)) +
           (om0 == -INFINITY ? 0.0f : os0 * fast_exp2((om0 - nm0) * kLog2e));
      s1 = (mx1 == -INFINITY ? 0.0f : s1 * fast_exp2((mx1 - nm1) * kLog2e)) +
           (om1 == -INFINITY ? 0.0f : os1 * fast_exp2((om1 - nm1) * kLog2e));
      mx0 = nm0; mx1 = nm1;
    }
    m0 = mx0; m1 = mx1;
    sc0 = 255.0f / s0; sc1 = 255.0f / s1;
    tie_run = tie_save;
  }

  // =========================================================================
  // Pass 2: keep mask, softmax weights and A.V (or the exports)
  // =========================================================================
  float of[8][4];
  int oi[8][4];
#pragma unroll
  for (int cb = 0; cb < 8; ++cb)
#pragma unroll
    for (int e = 0; e < 4; ++e) { of[cb][e] = 0.0f; oi[cb][e] = 0; }
  float lsum0 = 0.0f, lsum1 = 0.0f;           // float mode: sum of e over kept keys (per lane)
  float run_m0 = -INFINITY, run_m1 = -INFINITY;  // dense float: online max
  const bool online = (MODE == MODE_F && SEL == SEL_DENSE);
  const bool need_v = (EXPORT == EXP_NONE);

  load_tile(0, 0, need_v);
  for (int t = 0; t < ntiles; ++t) {
    if (t + 1 < ntiles) { load_tile((t + 1) & 1, t + 1, need_v); cp_async_wait<1>(); }
    else cp_async_wait<0>();
    __syncthreads();
    const int buf = t & 1;
    int sc[8][4];
    tile_scores(buf, sc);
    float lg[8][4];
#pragma unroll
    for (int nb = 0; nb < 8; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) lg[nb][e] = logit(buf, nb, e, sc[nb][e]);
    uint32_t keep[8];
    keep_tile(t, lg, keep);
    using G = Groups<MODE>;

    if (EXPORT == EXP_IDX) {
#pragma unroll
      for (int gi = 0; gi < G::kGroups; ++gi) {
        const uint32_t k0 = keep[gi] & 0xFFFFu, k1 = keep[gi] >> 16;
        uint32_t excl, total;
        quad_scan((uint32_t)__popc(k0) | ((uint32_t)__popc(k1) << 16), excl, total);
        int p0 = (int)(kept_run & 0xFFFFu) + (int)(excl & 0xFFFFu);
        int p1 = (int)(kept_run >> 16) + (int)(excl >> 16);
#pragma unroll
        for (int u = 0; u < G::kPerLane; ++u) {
          const int nb = G::nb_of(gi, u), col = u & 1;
          const int j = t * kKT + key_of<MODE>(nb, 2 * q + col);
          if ((k0 >> u) & 1u) { if (p0 < a.N) a.idx[((size_t)bh * a.n + i0) * a.N + p0] = j; ++p0; }
          if ((k1 >> u) & 1u) { if (p1 < a.N) a.idx[((size_t)bh * a.n + i1) * a.N + p1] = j; ++p1; }
        }
        kept_run += total;
      }
      __syncthreads();
      continue;
    }

    // softmax weights e = exp(l - m) of kept keys (0 elsewhere)
    float pw[8][4];
    if (online) {
      float tm0 = -INFINITY, tm1 = -INFINITY;
#pragma unroll
      for (int gi = 0; gi < G::kGroups; ++gi)
#pragma unroll
        for (int u = 0; u < G::kPerLane; ++u) {
          const int nb = G::nb_of(gi, u), col = u & 1;
          if ((keep[gi] >> u) & 1u) tm0 = fmaxf(tm0, lg[nb][col]);
          if ((keep[gi] >> (16 + u)) & 1u) tm1 = fmaxf(tm1, lg[nb][2 + col]);
        }
      tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, 1));
      tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, 2));
      tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, 1));
      tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, 2));
      const float nm0 = fmaxf(run_m0, tm0), nm1 = fmaxf(run_m1, tm1);
      const float al0 = (run_m0 == -INFINITY) ? 0.0f : fast_exp2((run_m0 - nm0) * kLog2e);
      const float al1 = (run_m1 == -INFINITY) ? 0.0f : fast_exp2((run_m1 - nm1) * kLog2e);
      if (nm0 != run_m0) {
        lsum0 *= al0;
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) { of[cb][0] *= al0; of[cb][1] *= al0; }
      }
      if (nm1 != run_m1) {
        lsum1 *= al1;
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) { of[cb][2] *= al1; of[cb][3] *= al1; }
      }
      run_m0 = nm0; run_m1 = nm1;
      m0 = nm0; m1 = nm1;
    }
#pragma unroll
    for (int nb = 0; nb < 8; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) pw[nb][e] = 0.0f;
#pragma unroll
    for (int gi = 0; gi < G::kGroups; ++gi)
#pragma unroll
      for (int u = 0; u < G::kPerLane; ++u) {
        const int nb = G::nb_of(gi, u), col = u & 1;
        if ((keep[gi] >> u) & 1u) pw[nb][col] = fast_exp2((lg[nb][col] - m0) * kLog2e);
        if ((keep[gi] >> (16 + u)) & 1u) pw[nb][2 + col] = fast_exp2((lg[nb][2 + col] - m1) * kLog2e);
      }

    if (MODE == MODE_F) {
#pragma unroll
      for (int nb = 0; nb < 8; ++nb) { lsum0 += pw[nb][0] + pw[nb][1]; lsum1 += pw[nb][2] + pw[nb][3]; }
      const uint8_t* vt = smem + SL::kOffV + buf * SL::kV;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t pa[4];
        pa[0] = pack_bf16x2(pw[2 * ks][0], pw[2 * ks][1]);
        pa[1] = pack_bf16x2(pw[2 * ks][2], pw[2 * ks][3]);
        pa[2] = pack_bf16x2(pw[2 * ks + 1][0], pw[2 * ks + 1][1]);
        pa[3] = pack_bf16x2(pw[2 * ks + 1][2], pw[2 * ks + 1][3]);
        uint32_t pl[4];
        if (V_F32) {
          // residuals of the bf16 rounding of P
          const float* pp[4] = {&pw[2 * ks][0], &pw[2 * ks][2], &pw[2 * ks + 1][0], &pw[2 * ks + 1][2]};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            __nv_bfloat162 hv = *reinterpret_cast<__nv_bfloat162*>(&pa[u]);
            float2 hf = __bfloat1622float2(hv);
            pl[u] = pack_bf16x2(pp[u][0] - hf.x, pp[u][1] - hf.y);
          }
        }
        const int mi = lane >> 3, rr = lane & 7;
        const int key = ks * 16 + (mi & 1) * 8 + rr;
#pragma unroll
        for (int cbp = 0; cbp < 4; ++cbp) {
          const int chunk = 2 * cbp + (mi >> 1);
          const int off = key * 128 + ((chunk ^ (key & 7)) * 16);
          uint32_t vb[4];
          ldmatrix_x4_trans(vb, vt + off);
          mma_bf16_16x8x16(of[2 * cbp], pa, vb[0], vb[1]);
          mma_bf16_16x8x16(of[2 * cbp + 1], pa, vb[2], vb[3]);
          if (V_F32) {
            uint32_t vl[4];
            ldmatrix_x4_trans(vl, vt + kKT * kD * 2 + off);
            mma_bf16_16x8x16(of[2 * cbp], pa, vl[0], vl[1]);
            mma_bf16_16x8x16(of[2 * cbp + 1], pa, vl[2], vl[3]);
            mma_bf16_16x8x16(of[2 * cbp], pl, vb[0], vb[1]);
            mma_bf16_16x8x16(of[2 * cbp + 1], pl, vb[2], vb[3]);
          }
        }
      }
    } else {
      // uint8 codes A = floor(255 p + 0.5), p = e * (1/l)
      uint32_t aq[8][4];
#pragma unroll
      for (int nb = 0; nb < 8; ++nb) {
        aq[nb][0] = (uint32_t)min(255, (int)floorf(__fmaf_rn(pw[nb][0], sc0, 0.5f)));
        aq[nb][1] = (uint32_t)min(255, (int)floorf(__fmaf_rn(pw[nb][1], sc0, 0.5f)));
        aq[nb][2] = (uint32_t)min(255, (int)floorf(__fmaf_rn(pw[nb][2], sc1, 0.5f)));
        aq[nb][3] = (uint32_t)min(255, (int)floorf(__fmaf_rn(pw[nb][3], sc1, 0.5f)));
      }
      if (EXPORT == EXP_CODES) {
        const int rows = a.row_end - a.row_begin;
#pragma unroll
        for (int nb = 0; nb < 8; ++nb)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = (e < 2) ? i0 : i1;
            const int j = t * kKT + key_of<MODE>(nb, 2 * q + (e & 1));
            if (i >= a.row_begin && i < a.row_end && i < a.n && j < a.n)
              a.codes[((size_t)bh * rows + (i - a.row_begin)) * a.n + j] = (uint8_t)aq[nb][e];
          }
        __syncthreads();
        continue;
      }
      const uint8_t* vt = smem + SL::kOffV + buf * SL::kV;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int A = cc * 4, Bn = A + 1, C = A + 2, Dn = A + 3;
        uint32_t pa[4];
        pa[0] = aq[A][0] | (aq[A][1] << 8) | (aq[Bn][0] << 16) | (aq[Bn][1] << 24);
        pa[1] = aq[A][2] | (aq[A][3] << 8) | (aq[Bn][2] << 16) | (aq[Bn][3] << 24);
        pa[2] = aq[C][0] | (aq[C][1] << 8) | (aq[Dn][0] << 16) | (aq[Dn][1] << 24);
        pa[3] = aq[C][2] | (aq[C][3] << 8) | (aq[Dn][2] << 16) | (aq[Dn][3] << 24);
        const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int cbp = 0; cbp < 4; ++cbp) {
          const int chn = (2 * cbp + (mi >> 1)) * 8 + rr;
          const int seg = 2 * cc + (mi & 1);
          const int off = chn * kKT + ((seg ^ ((chn >> 1) & 3)) * 16);
          uint32_t vb[4];
          ldmatrix_x4(vb, vt + off);
          mma_u8s8_16x8x32(oi[2 * cbp], pa, vb[0], vb[1]);
          mma_u8s8_16x8x32(oi[2 * cbp + 1], pa, vb[2], vb[3]);
        }
      }
    }
    __syncthreads();
  }

  if (EXPORT == EXP_IDX) {
    // pad each row's list with -1 after its kept keys
    if (q == 0) {
      const int k0 = (int)(kept_run & 0xFFFFu), k1 = (int)(kept_run >> 16);
      if (i0 < a.n)
        for (int p = row_ok0 ? k0 : 0; p < a.N; ++p) a.idx[((size_t)bh * a.n + i0) * a.N + p] = -1;
      if (i1 < a.n)
        for (int p = row_ok1 ? k1 : 0; p < a.N; ++p) a.idx[((size_t)bh * a.n + i1) * a.N + p] = -1;
    }
    return;
  }
  if (EXPORT == EXP_CODES) {
    // columns j in [L, n) of the exported rows are zero
    const int rows = a.row_end - a.row_begin;
    for (int rr = 0; rr < 2; ++rr) {
      const int i = rr ? i1 : i0;
      if (i >= a.row_begin && i < a.row_end && i < a.n)
        for (int j = ntiles * kKT + q; j < a.n; j += 4) a.codes[((size_t)bh * rows + (i - a.row_begin)) * a.n + j] = 0;
      if (i >= a.row_begin && i < a.row_end && i < a.n && i >= L)
        for (int j = q; j < min(a.n, ntiles * kKT); j += 4) a.codes[((size_t)bh * rows + (i - a.row_begin)) * a.n + j] = 0;
    }
    return;
  }

  // ---- epilogue: normalize / dequantize and store O (rows past L are 0)
  float out0[16], out1[16];
  if (MODE == MODE_F) {
    lsum0 += __shfl_xor_sync(0xffffffffu, lsum0, 1);
    lsum0 += __shfl_xor_sync(0xffffffffu, lsum0, 2);
    lsum1 += __shfl_xor_sync(0xffffffffu, lsum1, 1);
    lsum1 += __shfl_xor_sync(0xffffffffu, lsum1, 2);
    const float inv0 = row_ok0 ? 1.0f / lsum0 : 0.0f, inv1 = row_ok1 ? 1.0f / lsum1 : 0.0f;
#pragma unroll
    for (int cb = 0; cb < 8; ++cb) {
      out0[2 * cb] = of[cb][0] * inv0; out0[2 * cb + 1] = of[cb][1] * inv0;
      out1[2 * cb] = of[cb][2] * inv1; out1[2 * cb + 1] = of[cb][3] * inv1;
    }
  } else {
    const float* vs = a.vscale + (size_t)bh * kD;
#pragma unroll
    for (int cb = 0; cb < 8; ++cb) {
      const float d0 = __fdiv_rn(vs[8 * cb + 2 * q], 255.0f), d1 = __fdiv_rn(vs[8 * cb + 2 * q + 1], 255.0f);
      out0[2 * cb] = row_ok0 ? (float)oi[cb][0] * d0 : 0.0f;
      out0[2 * cb + 1] = row_ok0 ? (float)oi[cb][1] * d1 : 0.0f;
      out1[2 * cb] = row_ok1 ? (float)oi[cb][2] * d0 : 0.0f;
      out1[2 * cb + 1] = row_ok1 ? (float)oi[cb][3] * d1 : 0.0f;
    }
  }
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int i = rr ? i1 : i0;
    if (i >= a.n) continue;
    const float* src = rr ? out1 : out0;
    const size_t o = ((size_t)bh * a.n + i) * kD;
#pragma unroll
    for (int cb = 0; cb < 8; ++cb) {
      const int ch = 8 * cb + 2 * q;
      if (a.o_bf16) {
        *reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(a.O) + o + ch) =
            pack_bf16x2(src[2 * cb], src[2 * cb + 1]);
      } else {
        *reinterpret_cast<float2*>(reinterpret_cast<float*>(a.O) + o + ch) = make_float2(src[2 * cb], src[2 * cb + 1]);
      }
    }
  }
}

}  // namespace had

namespace had {

// Debug export of the integer scores through the same +-1 int8 tensor-core
// fragments as k_attn: S[i][j] = q~_i . k~_j = d - 2*popcount(q XOR k) for
// i, j < L, 0 elsewhere.  The K~ tile is expanded from packed bits in smem.
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

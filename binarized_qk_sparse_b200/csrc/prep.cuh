// prep.cuh -- per-head statistics, sign+pack and V quantization kernels.
//
//   k_stats : per (chunk of 64 tokens, batch*head, tensor) partial fp64 channel
//             sums of Q and K over the valid tokens, and fp32 channel absmax of V
//             (BinaryAttention §2.2 "mu = mean over tokens"; §2.4 per-channel V scale).
//   k_pack  : reduces the partials in a fixed order -> mu (fp64 sum / L, rounded
//             once to fp32) or the V scale (absmax / 127), then packs sign bits
//             (bit 1 <=> x < mu, word w bit j <=> channel 32w+j) with 128-bit
//             loads and lane shuffles, or writes int8 V transposed to
//             [channel][token] for the uint8 x int8 A.V tiles.
//
// Both kernels read each input element once with 16-byte loads; a CTA covers
// 64 tokens x 64 channels, so the grid is B*H*ceil(n/64) CTAs per tensor.
#pragma once

#include "common.cuh"

namespace had {

constexpr int kChunk = 64;         // tokens per stats/pack CTA
constexpr int kPrepThreads = 256;

template <typename T>
struct LoadTraits;
template <>
struct LoadTraits<__nv_bfloat16> {
  static constexpr int kEPT = 8;  // elements per 16-byte load
  __device__ static void load(const void* base, size_t elem, float (&x)[8]) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + elem));
    x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x); x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
    x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z); x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
  }
};
template <>
struct LoadTraits<float> {
  static constexpr int kEPT = 4;
  __device__ static void load(const void* base, size_t elem, float (&x)[8]) {
    float4 v = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem));
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
};

struct PrepArgs {
  const void* X[3];     // tensors 0,1 -> sums (Q, K); tensor 2 -> absmax (V)
  int ntens;            // tensors handled by this launch (blockIdx.z < ntens)
  int first_tensor;     // tensor id of blockIdx.z == 0 (lets a launch do only V, or only one of Q/K)
  int B, H, n, nchunks;
  const int32_t* seqlens;
  double* sums;         // [2][BH][nchunks][D]
  float* amax;          // [BH][nchunks][D]
  unsigned* status;
};

// Head dims D in {32, 64, 128}: a token row is D / EPT threads of one 16-byte load each.
template <typename T, int D>
__global__ void __launch_bounds__(kPrepThreads) k_stats(const PrepArgs a) {
  constexpr int kD = D;
  constexpr int EPT = LoadTraits<T>::kEPT;
  constexpr int TPT = kD / EPT;                 // threads per token row
  constexpr int TPP = kPrepThreads / TPT;       // tokens per pass
  const int chunk = blockIdx.x, bh = blockIdx.y, tz = a.first_tensor + blockIdx.z;
  const int b = bh / a.H;
  const int L = valid_len(a.seqlens, b, a.n, a.status);
  const int cg = threadIdx.x % TPT, tok = threadIdx.x / TPT;
  const int i0 = chunk * kChunk, i1 = min(i0 + kChunk, L);
  const size_t head = (size_t)bh * a.n * kD;
  __shared__ double red[TPP][kD];
  __shared__ float redf[TPP][kD];
  if (tz < 2) {
    double acc[EPT];
#pragma unroll
    for (int u = 0; u < EPT; ++u) acc[u] = 0.0;
    for (int i = i0 + tok; i < i1; i += TPP) {
      float x[8];
      LoadTraits<T>::load(a.X[tz], head + (size_t)i * kD + cg * EPT, x);
#pragma unroll
      for (int u = 0; u < EPT; ++u) acc[u] += (double)x[u];
    }
#pragma unroll
    for (int u = 0; u < EPT; ++u) red[tok][cg * EPT + u] = acc[u];
    __syncthreads();
    if (threadIdx.x < kD) {
      double s = 0.0;
      for (int t = 0; t < TPP; ++t) s += red[t][threadIdx.x];
      a.sums[(((size_t)tz * gridDim.y + bh) * a.nchunks + chunk) * kD + threadIdx.x] = s;
    }
  } else {
    float m[EPT];
#pragma unroll
    for (int u = 0; u < EPT; ++u) m[u] = 0.0f;
    for (int i = i0 + tok; i < i1; i += TPP) {
      float x[8];
      LoadTraits<T>::load(a.X[tz], head + (size_t)i * kD + cg * EPT, x);
#pragma unroll
      for (int u = 0; u < EPT; ++u) m[u] = fmaxf(m[u], fabsf(x[u]));
    }
#pragma unroll
    for (int u = 0; u < EPT; ++u) redf[tok][cg * EPT + u] = m[u];
    __syncthreads();
    if (threadIdx.x < kD) {
      float s = 0.0f;
      for (int t = 0; t < TPP; ++t) s = fmaxf(s, redf[t][threadIdx.x]);
      a.amax[((size_t)bh * a.nchunks + chunk) * kD + threadIdx.x] = s;
    }
  }
}

// The per-head statistic from the chunk partials, once per (b, h, channel): the
// mean of Q or K (fp64 sum of the partials in chunk order, one rounding to fp32,
// stored back as a double in chunk 0's slot) or the V absmax (chunk 0's slot).
// k_pack then reads chunk 0 instead of every CTA reducing all of the head's chunks.
template <int D>
__global__ void __launch_bounds__(128) k_stats_final(const PrepArgs a) {
  const int bh = blockIdx.x, tz = a.first_tensor + blockIdx.y, c = threadIdx.x;
  if (c >= D) return;
  const int L = valid_len(a.seqlens, bh / a.H, a.n, nullptr);  // k_stats already reported bad lengths
  const int nv = (L + kChunk - 1) / kChunk;
  constexpr int kBatch = 64;  // loads in flight; the adds still run in chunk order
  if (tz < 2) {
    double* col = a.sums + ((size_t)tz * gridDim.x + bh) * a.nchunks * D + c;
    double s = 0.0;
    for (int k0 = 0; k0 < nv; k0 += kBatch) {
      double v[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) v[k] = k0 + k < nv ? col[(size_t)(k0 + k) * D] : 0.0;
#pragma unroll
      for (int k = 0; k < kBatch; ++k) if (k0 + k < nv) s += v[k];
    }
    col[0] = (double)((L > 0) ? __double2float_rn(s / (double)L) : 0.0f);
  } else {
    float* col = a.amax + (size_t)bh * a.nchunks * D + c;
    float m = 0.0f;
    for (int k0 = 0; k0 < nv; k0 += kBatch) {
      float v[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) v[k] = k0 + k < nv ? col[(size_t)(k0 + k) * D] : 0.0f;
#pragma unroll
      for (int k = 0; k < kBatch; ++k) m = fmaxf(m, v[k]);
    }
    col[0] = m;
  }
}

struct PackArgs {
  const void* X[3];
  int ntens, first_tensor;
  int B, H, n, nchunks, n_pad;
  const int32_t* seqlens;
  const double* sums;     // from k_stats (unused when mu_in != nullptr)
  const float* amax;      // V's column absmax of head bh at amax[bh * amax_ld + c]
  int amax_ld;
  const float* mu_in[2];  // optional caller means per tensor 0/1
  float* mu_out[2];       // optional mean outputs per tensor 0/1
  uint32_t* bits[2];      // [BH][n][D/32] per tensor 0/1 (or null)
  int8_t* pm[2];          // [BH][n_pad][D] +-1 rows per tensor 0/1 (or null); +1 past L
  int pm_e4m3;            // the +-1 rows as e4m3 bytes (0x38 / 0xB8) instead of int8 (0x01 / 0xFF)
  int8_t* vqT;            // [BH][D][n_pad] int8, or [BH][D][n_pad / 2] packed 4-bit (key 2k in the low nibble of byte k)
  float* vscale;          // [BH][D]
  int v_bits;             // 8: int8 V, scale absmax/127; 4: 4-bit V, scale absmax/7
  unsigned* status;
};

// Integer code of x at scale sc: rint(x / sc) clamped to +-qmax (127 or 7), with
// x / sc the correctly rounded fp32 quotient.  For |x / sc| <= 128 the product
// x * (1/sc) is within 2^-15 of that quotient, so both round to the same integer
// unless the product lies within 2^-12 of a half-integer; only then is the
// quotient computed.
__device__ __forceinline__ int quant_v(float x, float sc, float rsc, float qmax) {
  const float y = x * rsc;
  float q = rintf(y);
  if (fabsf(y - q) > 0.5f - 0x1p-12f) q = rintf(__fdiv_rn(x, sc));
  return (int)fminf(fmaxf(q, -qmax), qmax);
}

template <typename T, int D>
__global__ void __launch_bounds__(kPrepThreads) k_pack(const PackArgs a) {
  constexpr int kD = D;
  constexpr int kW = D / 32;
  constexpr int EPT = LoadTraits<T>::kEPT;
  constexpr int TPT = kD / EPT;
  constexpr int TPP = kPrepThreads / TPT;
  constexpr int TPW = 32 / EPT;                 // threads contributing to one 32-bit word
  const int chunk = blockIdx.x, bh = blockIdx.y, tz = a.first_tensor + blockIdx.z;
  const int b = bh / a.H;
  const int L = valid_len(a.seqlens, b, a.n, nullptr);  // k_stats already reported bad lengths
  const int cg = threadIdx.x % TPT, tok = threadIdx.x / TPT;
  const int i0 = chunk * kChunk;
  const size_t head = (size_t)bh * a.n * kD;
  __shared__ float stat[kD], rstat[kD];
  __shared__ __align__(16) int8_t vt[kD][kChunk];
  if (threadIdx.x < kD) {
    const int c = threadIdx.x;
    if (tz < 2) {
      float mu;
      if (a.mu_in[tz]) {
        mu = a.mu_in[tz][(size_t)bh * kD + c];
      } else {  // the mean k_stats_final left in chunk 0's slot
        mu = (float)a.sums[((size_t)tz * gridDim.y + bh) * a.nchunks * kD + c];
      }
      stat[c] = mu;
      if (chunk == 0 && a.mu_out[tz]) a.mu_out[tz][(size_t)bh * kD + c] = mu;
    } else {
      const float m = a.amax[(size_t)bh * a.amax_ld + c];  // k_stats_final's (chunk 0 slot) or the caller's
      const float qmax = a.v_bits == 4 ? 7.0f : 127.0f;
      float s = (m > 0.0f) ? __fdiv_rn(m, qmax) : 1.0f;
      stat[c] = s;
      rstat[c] = 1.0f / s;
      if (chunk == 0) a.vscale[(size_t)bh * kD + c] = s;
    }
  }
  __syncthreads();
  if (tz < 2) {
    uint32_t* out = a.bits[tz] ? a.bits[tz] + (size_t)bh * a.n * kW : nullptr;
    int8_t* pmo = a.pm[tz] ? a.pm[tz] + (size_t)bh * a.n_pad * kD : nullptr;
    const int lane = threadIdx.x & 31;
    for (int t = tok; t < kChunk; t += TPP) {
      const int i = i0 + t;
      uint32_t v = 0;
      if (i < L) {
        float x[8];
        LoadTraits<T>::load(a.X[tz], head + (size_t)i * kD + cg * EPT, x);
#pragma unroll
        for (int u = 0; u < EPT; ++u) v |= (x[u] < stat[cg * EPT + u] ? 1u : 0u) << u;
      }
      if (pmo && i < a.n_pad) {
        // +-1 copy of the same signs (bit 1 -> -1): int8 0xFF / 0x01, or e4m3 0xB8 / 0x38
        uint32_t w0 = expand_nibble_pm(v & 15u, a.pm_e4m3);
        if (EPT == 8) {
          uint32_t w1 = expand_nibble_pm((v >> 4) & 15u, a.pm_e4m3);
          *reinterpret_cast<uint2*>(pmo + (size_t)i * kD + cg * EPT) = make_uint2(w0, w1);
        } else {
          *reinterpret_cast<uint32_t*>(pmo + (size_t)i * kD + cg * EPT) = w0;
        }
      }
      v <<= (cg * EPT) & 31;
      // OR together the TPW lanes that share a word (they are adjacent lanes)
#pragma unroll
      for (int o = 1; o < TPW; o <<= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
      if (out && i < a.n && (lane % TPW) == 0) out[(size_t)i * kW + (cg * EPT) / 32] = v;
    }
  } else {
    for (int t = tok; t < kChunk; t += TPP) {
      const int i = i0 + t;
      float x[8];
      if (i < L) {
        LoadTraits<T>::load(a.X[tz], head + (size_t)i * kD + cg * EPT, x);
      } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = 0.0f;
      }
      const float qmax = a.v_bits == 4 ? 7.0f : 127.0f;
#pragma unroll
      for (int u = 0; u < EPT; ++u)
        vt[cg * EPT + u][t] = (int8_t)quant_v(x[u], stat[cg * EPT + u], rstat[cg * EPT + u], qmax);
    }
    __syncthreads();
    if (a.v_bits == 4) {
      // the D x 64 block of packed 4-bit V^T: row c, bytes [i0/2, i0/2 + 32), 16 bytes per thread and step
      uint8_t* dst = reinterpret_cast<uint8_t*>(a.vqT) + (size_t)bh * kD * (a.n_pad / 2);
      for (int e = threadIdx.x; e < kD * 2; e += kPrepThreads) {
        const int c = e >> 1, seg = e & 1;
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t v = 0;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int t0 = seg * 32 + 8 * k + 2 * b;
            v |= ((((uint32_t)(uint8_t)vt[c][t0]) & 15u) | ((((uint32_t)(uint8_t)vt[c][t0 + 1]) & 15u) << 4)) << (8 * b);
          }
          w[k] = v;
        }
        *reinterpret_cast<uint4*>(dst + (size_t)c * (a.n_pad / 2) + i0 / 2 + seg * 16) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
      // write the D x 64 int8 block of V^T: row c, tokens [i0, i0+64) -- 16 bytes per thread and step
      int8_t* dst = a.vqT + (size_t)bh * kD * a.n_pad;
      for (int e = threadIdx.x; e < kD * 4; e += kPrepThreads) {
        const int c = e >> 2, seg = e & 3;
        if (i0 + seg * 16 < a.n_pad)
          *reinterpret_cast<uint4*>(dst + (size_t)c * a.n_pad + i0 + seg * 16) =
              *reinterpret_cast<const uint4*>(&vt[c][seg * 16]);
      }
    }
  }
}

}  // namespace had

namespace had {

// ---------------------------------------------------------------------------- one-pass prep for short heads
//
// k_prep_head: one CTA per (batch*head, tensor) when the head's valid tokens fit
// in shared memory.  The head is read from HBM once (16-byte cp.async chunks),
// then from shared memory: channel sums in fp64 (Q, K) or channel absmax (V),
// the mean (or scale), and the packed outputs -- Q sign bits, K as +-1 int8
// rows, V as int8 V^T.  Same definitions as k_stats + k_pack.

// Threads of a short-head CTA: 128 for heads up to kHeadSmallBytes (more CTAs per
// SM, so more heads' loads overlap), 256 above.
constexpr int kHeadSmallBytes = 48 * 1024;
constexpr int kHeadMaxBytes = 128 * 1024;   // staged head: n * 64 * sizeof(T)

struct HeadArgs {
  const void* X[3];
  int first_tensor;
  int B, H, n, n_pad;
  const int32_t* seqlens;
  uint32_t* qbits;     // tensor 0 -> [BH][n][2]
  int8_t* kpm;         // tensor 1 -> [BH][n_pad][64]
  int kpm_e4m3;        // K~ as e4m3 bytes (see PackArgs::pm_e4m3)
  int8_t* vqT;         // tensor 2 -> [BH][64][n_pad] int8, or [BH][64][n_pad / 2] packed 4-bit
  float* vscale;       // [BH][64]
  int v_bits;          // 8 or 4 (see PackArgs)
  unsigned* status;
  int bias_slice;      // grid slice y == bias_slice computes the bias tables (if launched)
};

// Per-head bias range (0 included when class tokens exist: their pairs have bias
// 0) and the two extended tables (see RelposExt, DenseExt) the attention kernel
// reads: the bias itself (class pairs 0, keys past L -inf) and exp(b - b_max)
// (class pairs exp(-b_max), keys past L 0).  One CTA per head (relative-position
// tables; dense matrices below).
struct BiasArgs {
  const float* table;  // [H][2gh-1][2gw-1], or [H][n][n] when dense, or null
  int gh, gw, prefix;
  int dense, n;        // dense: a bias matrix over the n x n pairs
  float* bminmax;      // [H][2]
  float* bext;         // [H][E]
  float* expb;         // [H][E]
};

// The extended tables of head h, entries [e0, e1), given the table maximum mx.
__device__ __forceinline__ void relpos_fill(const BiasArgs& a, int h, float mx, int e0, int e1) {
  const RelposExt x = relpos_ext(a.gh, a.gw);
  const int tw = 2 * a.gw - 1;
  const float* t = a.table + (size_t)h * (2 * a.gh - 1) * tw;
  const float kLog2e = 1.4426950408889634f;
  const float e_class = exp2f((0.0f - mx) * kLog2e);
  float* be = a.bext + (size_t)h * x.E;
  float* ee = a.expb + (size_t)h * x.E;
  const int z0 = 2 * x.T + 2 * x.Kx;
  for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    float b, w;
    if (e < x.T) {  // table row e / S, column e % S (columns past 2gw-2 are padding)
      const int dy = e / x.S, dx = e - dy * x.S;
      b = dx < tw ? t[dy * tw + dx] : 0.0f;
      w = exp2f((b - mx) * kLog2e);
    }
    else if (e < z0) { b = 0.0f; w = e_class; }
    else { b = -INFINITY; w = 0.0f; }
    be[e] = b;
    ee[e] = w;
  }
}

// The range of head h's table (0 included when class tokens exist) into bminmax,
// then, with `fill`, its extended tables.
__device__ __forceinline__ void bias_tables_block(const BiasArgs& a, int h, bool fill = true) {
  __shared__ float smn[32], smx[32];
  const RelposExt x = relpos_ext(a.gh, a.gw);
  const int tw = 2 * a.gw - 1;
  const size_t cells = (size_t)(2 * a.gh - 1) * tw;
  const float* t = a.table + (size_t)h * cells;
  float mn = INFINITY, mx = -INFINITY;
  constexpr int kInFlight = 8;
  for (size_t e0 = threadIdx.x; e0 < cells; e0 += (size_t)kInFlight * blockDim.x) {
    float v[kInFlight];
#pragma unroll
    for (int k = 0; k < kInFlight; ++k) {
      const size_t e = e0 + (size_t)k * blockDim.x;
      v[k] = e < cells ? t[e] : t[e0];
    }
#pragma unroll
    for (int k = 0; k < kInFlight; ++k) { mn = fminf(mn, v[k]); mx = fmaxf(mx, v[k]); }
  }
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if ((threadIdx.x & 31) == 0) { smn[threadIdx.x >> 5] = mn; smx[threadIdx.x >> 5] = mx; }
  __syncthreads();
  mn = smn[0]; mx = smx[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) { mn = fminf(mn, smn[w]); mx = fmaxf(mx, smx[w]); }
  if (a.prefix > 0) { mn = fminf(mn, 0.0f); mx = fmaxf(mx, 0.0f); }
  if (threadIdx.x == 0) { a.bminmax[2 * h] = mn; a.bminmax[2 * h + 1] = mx; }
  if (fill) relpos_fill(a, h, mx, 0, x.E);
}

__global__ void __launch_bounds__(256) k_bias_tables(const BiasArgs a) { bias_tables_block(a, blockIdx.x); }

// Long sequences: one CTA per head takes the range (k_bias_range), then the tables,
// up to 2.4 MB per head at 128 x 128 patches, are written by many CTAs per head
// (k_bias_fill, grid (entries / kBiasFillPerCta, H)).
constexpr int kBiasFillPerCta = 8192;
constexpr int kBiasRangeThreads = 1024;
__global__ void __launch_bounds__(kBiasRangeThreads) k_bias_range(const BiasArgs a) { bias_tables_block(a, blockIdx.x, false); }
__global__ void __launch_bounds__(256) k_bias_fill(const BiasArgs a) {
  const int h = blockIdx.y, e0 = blockIdx.x * kBiasFillPerCta;
  relpos_fill(a, h, a.bminmax[2 * h + 1], e0, min(e0 + kBiasFillPerCta, relpos_ext(a.gh, a.gw).E));
}

// A dense bias matrix has n^2 entries per head, too many for one CTA per head to
// turn into tables quickly: one CTA per head takes the range, then the tables
// are written by many CTAs per head (grid (entries / kDenseTabPerCta, H)).
constexpr int kDenseTabPerCta = 4096;

constexpr int kDenseRangeThreads = 1024;

__global__ void __launch_bounds__(kDenseRangeThreads) k_dense_bias_range(const BiasArgs a) {
  constexpr int kWarps = kDenseRangeThreads / 32, kInFlight = 8;  // loads in flight per thread
  __shared__ float smn[kWarps], smx[kWarps];
  const int h = blockIdx.x;
  const size_t cells = (size_t)a.n * a.n;
  const float* t = a.table + (size_t)h * cells;
  float mn = INFINITY, mx = -INFINITY;
  for (size_t e0 = threadIdx.x; e0 < cells; e0 += (size_t)kInFlight * kDenseRangeThreads) {
    float v[kInFlight];
#pragma unroll
    for (int k = 0; k < kInFlight; ++k) {
      const size_t e = e0 + (size_t)k * kDenseRangeThreads;
      v[k] = e < cells ? __ldg(t + e) : t[e0];
    }
#pragma unroll
    for (int k = 0; k < kInFlight; ++k) { mn = fminf(mn, v[k]); mx = fmaxf(mx, v[k]); }
  }
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if ((threadIdx.x & 31) == 0) { smn[threadIdx.x >> 5] = mn; smx[threadIdx.x >> 5] = mx; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kWarps; ++w) { mn = fminf(mn, smn[w]); mx = fmaxf(mx, smx[w]); }
    a.bminmax[2 * h] = mn;
    a.bminmax[2 * h + 1] = mx;
  }
}

__global__ void __launch_bounds__(256) k_dense_bias_tables(const BiasArgs a) {
  const int h = blockIdx.y;
  const DenseExt dx = dense_ext(a.n);
  const float* t = a.table + (size_t)h * a.n * a.n;
  const float mx = a.bminmax[2 * h + 1];
  const float kLog2e = 1.4426950408889634f;
  float* be = a.bext + (size_t)h * dx.E;
  float* ee = a.expb + (size_t)h * dx.E;
  const int e1 = min(dx.E, (int)(blockIdx.x + 1) * kDenseTabPerCta);
  for (int e = blockIdx.x * kDenseTabPerCta + threadIdx.x; e < e1; e += blockDim.x) {
    const int i = e / dx.S, j = e - i * dx.S;  // row i at i * S, the sentinel in column n, padding 0
    float b = 0.0f, w = 0.0f;
    if (i < a.n && j < a.n) {
      b = t[(size_t)i * a.n + j];
      w = exp2f((b - mx) * kLog2e);
    } else if (i < a.n && j == a.n) {
      b = -INFINITY;
    }
    be[e] = b;
    ee[e] = w;
  }
}

template <typename T, int kHeadThreads>
__global__ void __launch_bounds__(kHeadThreads) k_prep_head(const HeadArgs a, const BiasArgs ba) {
  if ((int)blockIdx.y == a.bias_slice) {  // the bias slice: one CTA per head
    if ((int)blockIdx.x < a.H) bias_tables_block(ba, blockIdx.x);
    return;
  }
  // The head's valid tokens, 16-byte chunk c of token i stored at chunk c ^ (i & 7)
  // of its row, so that one thread per token (and one warp per token row) reads
  // shared memory without bank conflicts.
  extern __shared__ __align__(16) uint8_t xs[];
  constexpr int kGroups = kHeadThreads / 32;
  __shared__ double part[kGroups][kD];
  __shared__ __align__(16) float stat[kD];
  const int bh = blockIdx.x, tz = a.first_tensor + blockIdx.y, b = bh / a.H;
  const int L = valid_len(a.seqlens, b, a.n, a.status);
  const int tid = threadIdx.x;
  constexpr int kRow = kD * (int)sizeof(T);  // bytes per token
  constexpr int kChunks = kRow / 16;
  const uint8_t* src = static_cast<const uint8_t*>(a.X[tz]) + (size_t)bh * a.n * kRow;
  for (int e = tid; e < L * kChunks; e += kHeadThreads) {
    const int i = e / kChunks, c = e % kChunks;
    uint32_t d = (uint32_t)__cvta_generic_to_shared(xs + i * kRow + ((c ^ (i & 7)) * 16));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src + (size_t)e * 16));
  }
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
  __syncthreads();
  // byte offset of channels 2p, 2p+1 inside a row whose token index is = k (mod 8)
  auto pair_off = [&](int p, int k) -> int {
    const int byte = 2 * p * (int)sizeof(T);
    return (((byte >> 4) ^ k) << 4) + (byte & 15);
  };
  auto pair_load = [&](const uint8_t* q) -> float2 {
    if (sizeof(T) == 2) {
      const uint32_t u = *reinterpret_cast<const uint32_t*>(q);
      return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    }
    return *reinterpret_cast<const float2*>(q);
  };
  // ---- channel statistic: warp g covers tokens g, g + kGroups, ...; lane p channels 2p, 2p+1
  // (with 8 warps every token of a warp is = g mod 8, so its swizzled column is fixed)
  {
    const int p = tid & 31, g = tid >> 5;
    const uint8_t* col = xs + pair_off(p, g);
    if (tz < 2) {
      double s0 = 0.0, s1 = 0.0;
      for (int i = g; i < L; i += kGroups) {
        const float2 x = pair_load((kGroups % 8 == 0 ? col : xs + pair_off(p, i & 7)) + i * kRow);
        s0 += (double)x.x;
        s1 += (double)x.y;
      }
      part[g][2 * p] = s0;
      part[g][2 * p + 1] = s1;
    } else {
      float m0 = 0.0f, m1 = 0.0f;
      for (int i = g; i < L; i += kGroups) {
        const float2 x = pair_load((kGroups % 8 == 0 ? col : xs + pair_off(p, i & 7)) + i * kRow);
        m0 = fmaxf(m0, fabsf(x.x));
        m1 = fmaxf(m1, fabsf(x.y));
      }
      part[g][2 * p] = (double)m0;
      part[g][2 * p + 1] = (double)m1;
    }
  }
  __syncthreads();
  if (tid < kD) {
    if (tz < 2) {
      double s = 0.0;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) s += part[g][tid];
      stat[tid] = (L > 0) ? __double2float_rn(s / (double)L) : 0.0f;
    } else {
      float mx = 0.0f;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) mx = fmaxf(mx, (float)part[g][tid]);
      const float sc = (mx > 0.0f) ? __fdiv_rn(mx, a.v_bits == 4 ? 7.0f : 127.0f) : 1.0f;
      stat[tid] = sc;
      a.vscale[(size_t)bh * kD + tid] = sc;
    }
  }
  __syncthreads();
  if (tz < 2) {
    // one thread per token: 64 sign bits against the means (bit 1: x < mu)
    const int ntok = (tz == 0) ? a.n : a.n_pad;
    for (int i = tid; i < ntok; i += kHeadThreads) {
      uint32_t w[2] = {0u, 0u};
      if (i < L) {
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(xs + i * kRow + ((c ^ (i & 7)) << 4));
          const uint32_t u[4] = {v.x, v.y, v.z, v.w};
          if (sizeof(T) == 2) {
            const float4 m0 = *reinterpret_cast<const float4*>(stat + 8 * c);
            const float4 m1 = *reinterpret_cast<const float4*>(stat + 8 * c + 4);
            const float mu[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float x = (e & 1) ? __uint_as_float(u[e >> 1] & 0xFFFF0000u) : __uint_as_float(u[e >> 1] << 16);
              const int ch = 8 * c + e;
              w[ch >> 5] |= (x < mu[e] ? 1u : 0u) << (ch & 31);
            }
          } else {
            const float4 m0 = *reinterpret_cast<const float4*>(stat + 4 * c);
            const float mu[4] = {m0.x, m0.y, m0.z, m0.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int ch = 4 * c + e;
              w[ch >> 5] |= (__uint_as_float(u[e]) < mu[e] ? 1u : 0u) << (ch & 31);
            }
          }
        }
      }
      if (tz == 0) {
        *reinterpret_cast<uint2*>(a.qbits + ((size_t)bh * a.n + i) * kW) = make_uint2(w[0], w[1]);
      } else {
        // +-1 row of K (bit 1 -> -1), int8 or e4m3; rows past L are +1
        uint4* dst = reinterpret_cast<uint4*>(a.kpm + ((size_t)bh * a.n_pad + i) * kD);
        const bool e4 = a.kpm_e4m3 != 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t f = w[q >> 1] >> ((q & 1) * 16);
          dst[q] = make_uint4(expand_nibble_pm(f & 15u, e4), expand_nibble_pm((f >> 4) & 15u, e4),
                              expand_nibble_pm((f >> 8) & 15u, e4), expand_nibble_pm((f >> 12) & 15u, e4));
        }
      }
    }
  } else {
    // thread (channel pair, block of 16 tokens): two V^T row segments of 16 int8
    // codes (16 bytes) or 16 packed 4-bit codes (8 bytes)
    const int p = tid & 31;
    const float sc0 = stat[2 * p], sc1 = stat[2 * p + 1];
    const float r0 = 1.0f / sc0, r1 = 1.0f / sc1;
    const bool v4 = a.v_bits == 4;
    const float qmax = v4 ? 7.0f : 127.0f;
    int off[8];  // token u of a block is = u (mod 8)
#pragma unroll
    for (int k = 0; k < 8; ++k) off[k] = pair_off(p, k);
    for (int blk = tid >> 5; blk * 16 < a.n_pad; blk += kGroups) {
      uint32_t w0[4] = {0u, 0u, 0u, 0u}, w1[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int i = blk * 16 + u;
        if (i < L) {
          const float2 x = pair_load(xs + i * kRow + off[u & 7]);
          const uint32_t q0 = (uint32_t)quant_v(x.x, sc0, r0, qmax), q1 = (uint32_t)quant_v(x.y, sc1, r1, qmax);
          if (v4) {
            w0[u >> 3] |= (q0 & 15u) << (4 * (u & 7));
            w1[u >> 3] |= (q1 & 15u) << (4 * (u & 7));
          } else {
            w0[u >> 2] |= (q0 & 0xFFu) << (8 * (u & 3));
            w1[u >> 2] |= (q1 & 0xFFu) << (8 * (u & 3));
          }
        }
      }
      if (v4) {
        uint8_t* base = reinterpret_cast<uint8_t*>(a.vqT) + ((size_t)bh * kD + 2 * p) * (a.n_pad / 2) + blk * 8;
        *reinterpret_cast<uint2*>(base) = make_uint2(w0[0], w0[1]);
        *reinterpret_cast<uint2*>(base + a.n_pad / 2) = make_uint2(w1[0], w1[1]);
      } else {
        int8_t* base = a.vqT + ((size_t)bh * kD + 2 * p) * a.n_pad + blk * 16;
        *reinterpret_cast<uint4*>(base) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
        *reinterpret_cast<uint4*>(base + a.n_pad) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
      }
    }
  }
}

}  // namespace had

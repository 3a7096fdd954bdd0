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
  double* sums;         // [2][BH][nchunks][64]
  float* amax;          // [BH][nchunks][64]
  unsigned* status;
};

template <typename T>
__global__ void __launch_bounds__(kPrepThreads) k_stats(const PrepArgs a) {
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

struct PackArgs {
  const void* X[3];
  int ntens, first_tensor;
  int B, H, n, nchunks, n_pad;
  const int32_t* seqlens;
  const double* sums;     // from k_stats (unused when mu_in != nullptr)
  const float* amax;
  const float* mu_in[2];  // optional caller means per tensor 0/1
  float* mu_out[2];       // optional mean outputs per tensor 0/1
  uint32_t* bits[2];      // [BH][n][kW] per tensor 0/1 (or null)
  int8_t* pm[2];          // [BH][n_pad][64] +-1 int8 rows per tensor 0/1 (or null); +1 past L
  int8_t* vqT;            // [BH][64][n_pad]
  float* vscale;          // [BH][64]
  unsigned* status;
};

template <typename T>
__global__ void __launch_bounds__(kPrepThreads) k_pack(const PackArgs a) {
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
  __shared__ float stat[kD];
  __shared__ __align__(16) int8_t vt[kD][kChunk];
  if (threadIdx.x < kD) {
    const int c = threadIdx.x;
    if (tz < 2) {
      float mu;
      if (a.mu_in[tz]) {
        mu = a.mu_in[tz][(size_t)bh * kD + c];
      } else {
        double s = 0.0;
        const int nch_valid = (L + kChunk - 1) / kChunk;
        for (int k = 0; k < nch_valid; ++k) s += a.sums[(((size_t)tz * gridDim.y + bh) * a.nchunks + k) * kD + c];
        mu = (L > 0) ? __double2float_rn(s / (double)L) : 0.0f;
      }
      stat[c] = mu;
      if (chunk == 0 && a.mu_out[tz]) a.mu_out[tz][(size_t)bh * kD + c] = mu;
    } else {
      float m = 0.0f;
      const int nch_valid = (L + kChunk - 1) / kChunk;
      for (int k = 0; k < nch_valid; ++k) m = fmaxf(m, a.amax[((size_t)bh * a.nchunks + k) * kD + c]);
      float s = (m > 0.0f) ? __fdiv_rn(m, 127.0f) : 1.0f;
      stat[c] = s;
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
        // +-1 int8 copy of the same signs: bit 1 -> 0xFF (-1), bit 0 -> 0x01 (+1)
        uint32_t w0 = expand_nibble_pm1(v & 15u);
        if (EPT == 8) {
          uint32_t w1 = expand_nibble_pm1((v >> 4) & 15u);
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
#pragma unroll
      for (int u = 0; u < EPT; ++u) {
        float r = rintf(__fdiv_rn(x[u], stat[cg * EPT + u]));
        r = fminf(fmaxf(r, -127.0f), 127.0f);
        vt[cg * EPT + u][t] = (int8_t)(int)r;
      }
    }
    __syncthreads();
    // write the 64 x 64 int8 block of V^T: row c, tokens [i0, i0+64) -- 16 bytes per thread
    int8_t* dst = a.vqT + (size_t)bh * kD * a.n_pad;
    const int c = threadIdx.x >> 2, seg = threadIdx.x & 3;
    if (i0 + seg * 16 < a.n_pad) {
      *reinterpret_cast<uint4*>(dst + (size_t)c * a.n_pad + i0 + seg * 16) =
          *reinterpret_cast<const uint4*>(&vt[c][seg * 16]);
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

constexpr int kHeadThreads = 256;
constexpr int kHeadMaxBytes = 128 * 1024;   // staged head: n * 64 * sizeof(T)

struct HeadArgs {
  const void* X[3];
  int first_tensor;
  int B, H, n, n_pad;
  const int32_t* seqlens;
  uint32_t* qbits;     // tensor 0 -> [BH][n][2]
  int8_t* kpm;         // tensor 1 -> [BH][n_pad][64]
  int8_t* vqT;         // tensor 2 -> [BH][64][n_pad]
  float* vscale;       // [BH][64]
  unsigned* status;
};

template <typename T>
__global__ void __launch_bounds__(kHeadThreads) k_prep_head(const HeadArgs a) {
  extern __shared__ __align__(16) uint8_t xs[];      // [L][64] of T
  __shared__ double part[4][kD];
  __shared__ float stat[kD];
  const int bh = blockIdx.x, tz = a.first_tensor + blockIdx.y, b = bh / a.H;
  const int L = valid_len(a.seqlens, b, a.n, a.status);
  const int tid = threadIdx.x;
  constexpr int kRow = kD * (int)sizeof(T);          // bytes per token
  const uint8_t* src = static_cast<const uint8_t*>(a.X[tz]) + (size_t)bh * a.n * kRow;
  for (int e = tid; e < L * (kRow / 16); e += kHeadThreads) {
    uint32_t d = (uint32_t)__cvta_generic_to_shared(xs + e * 16);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src + (size_t)e * 16));
  }
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
  __syncthreads();
  auto x_at = [&](int i, int ch) -> float {
    if (sizeof(T) == 2) return __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(xs)[i * kD + ch] << 16);
    return reinterpret_cast<const float*>(xs)[i * kD + ch];
  };
  // ---- channel statistic: thread (g, c) covers tokens i = g, g+4, ...
  {
    const int ch = tid & (kD - 1), g = tid >> 6;
    if (tz < 2) {
      double acc = 0.0;
      for (int i = g; i < L; i += 4) acc += (double)x_at(i, ch);
      part[g][ch] = acc;
    } else {
      float mx = 0.0f;
      for (int i = g; i < L; i += 4) mx = fmaxf(mx, fabsf(x_at(i, ch)));
      part[g][ch] = (double)mx;
    }
  }
  __syncthreads();
  if (tid < kD) {
    if (tz < 2) {
      const double s = ((part[0][tid] + part[1][tid]) + part[2][tid]) + part[3][tid];
      stat[tid] = (L > 0) ? __double2float_rn(s / (double)L) : 0.0f;
    } else {
      const float mx = fmaxf(fmaxf((float)part[0][tid], (float)part[1][tid]), fmaxf((float)part[2][tid], (float)part[3][tid]));
      const float sc = (mx > 0.0f) ? __fdiv_rn(mx, 127.0f) : 1.0f;
      stat[tid] = sc;
      a.vscale[(size_t)bh * kD + tid] = sc;
    }
  }
  __syncthreads();
  if (tz < 2) {
    // one thread per token: sign bits against the means
    for (int i = tid; i < (tz == 0 ? a.n : a.n_pad); i += kHeadThreads) {
      uint32_t w0 = 0, w1 = 0;
      if (i < L) {
#pragma unroll 8
        for (int ch = 0; ch < 32; ++ch) {
          w0 |= (x_at(i, ch) < stat[ch] ? 1u : 0u) << ch;
          w1 |= (x_at(i, ch + 32) < stat[ch + 32] ? 1u : 0u) << ch;
        }
      }
      if (tz == 0) {
        *reinterpret_cast<uint2*>(a.qbits + ((size_t)bh * a.n + i) * kW) = make_uint2(w0, w1);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(a.kpm + ((size_t)bh * a.n_pad + i) * kD);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t f = (q < 2 ? w0 : w1) >> ((q & 1) * 16);
          dst[q] = make_uint4(expand_nibble_pm1(f & 15u), expand_nibble_pm1((f >> 4) & 15u),
                              expand_nibble_pm1((f >> 8) & 15u), expand_nibble_pm1((f >> 12) & 15u));
        }
      }
    }
  } else {
    // thread (channel, block of 16 tokens): int8 V^T row segments of 16 bytes
    const int ch = tid & (kD - 1);
    const float sc = stat[ch];
    for (int blk = tid >> 6; blk * 16 < a.n_pad; blk += kHeadThreads / kD) {
      uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int i = blk * 16 + u;
        int q = 0;
        if (i < L) {
          float r = rintf(__fdiv_rn(x_at(i, ch), sc));
          r = fminf(fmaxf(r, -127.0f), 127.0f);
          q = (int)r;
        }
        w[u >> 2] |= ((uint32_t)q & 0xFFu) << (8 * (u & 3));
      }
      *reinterpret_cast<uint4*>(a.vqT + ((size_t)bh * kD + ch) * a.n_pad + blk * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

}  // namespace had

// dense_ref.cuh -- the library's dense comparison mode: standard attention on
// the unbinarized bf16 Q, K (BinaryAttention §2.3 equation without the sign
// step): l = (q . k) / sqrt(d) + b_ij with q . k on the bf16 tensor cores
// (mma.sync m16n8k16, fp32 accumulate), online fp32 softmax, bf16 P x bf16 V.
// Same CTA shape as the binarized kernel: 64 query rows, 64-key tiles, 4 warps.
#pragma once

#include "attn.cuh"

namespace had {

template <bool HAS_BIAS>
__global__ void __launch_bounds__(kAttnThreads) k_dense_ref(const __grid_constant__ AttnArgs a,
                                                            const __nv_bfloat16* __restrict__ Q,
                                                            const __nv_bfloat16* __restrict__ K) {
  __shared__ __align__(128) uint8_t kt[2][kKT * 128];
  __shared__ __align__(128) uint8_t vt[2][kKT * 128];
  __shared__ int koff[2][kKT];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int q0 = blockIdx.x * kQT;
  const int L = valid_len(a.seqlens, b, a.n, a.status);
  const int lr0 = warp * 16 + g;
  const int i0 = q0 + lr0, i1 = i0 + 8;
  const bool row_ok0 = i0 < L, row_ok1 = i1 < L;
  const float rsd = 0.125f;  // 1/sqrt(64)

  if (q0 >= L) {
    for (int e = tid; e < kQT * kD; e += kAttnThreads) {
      int r = q0 + e / kD, ch = e % kD;
      if (r < a.n) {
        size_t o = ((size_t)bh * a.n + r) * kD + ch;
        if (a.o_bf16) reinterpret_cast<__nv_bfloat16*>(a.O)[o] = __float2bfloat16(0.0f);
        else reinterpret_cast<float*>(a.O)[o] = 0.0f;
      }
    }
    return;
  }
  // Q A-fragments for the 4 k-steps of d = 64
  uint32_t qf[4][4];
  {
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(Q + (size_t)bh * a.n * kD);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      qf[kk][0] = row_ok0 ? q32[((size_t)i0 * kD + 16 * kk + 2 * q) / 2] : 0u;
      qf[kk][1] = row_ok1 ? q32[((size_t)i1 * kD + 16 * kk + 2 * q) / 2] : 0u;
      qf[kk][2] = row_ok0 ? q32[((size_t)i0 * kD + 16 * kk + 8 + 2 * q) / 2] : 0u;
      qf[kk][3] = row_ok1 ? q32[((size_t)i1 * kD + 16 * kk + 8 + 2 * q) / 2] : 0u;
    }
  }
  const float* tab = HAS_BIAS ? a.table + (size_t)h * a.th * a.tw : nullptr;
  int rb0 = -1, rb1 = -1;
  if (HAS_BIAS && a.bias_dense) {  // entry rb - koff = i n + j
    if (i0 < a.n) rb0 = i0 * a.n;
    if (i1 < a.n) rb1 = i1 * a.n;
  } else if (HAS_BIAS) {
    if (i0 >= a.prefix && i0 < a.n) { int t = i0 - a.prefix; rb0 = (t / a.gw + a.gh - 1) * a.tw + (t % a.gw + a.gw - 1); }
    if (i1 >= a.prefix && i1 < a.n) { int t = i1 - a.prefix; rb1 = (t / a.gw + a.gh - 1) * a.tw + (t % a.gw + a.gw - 1); }
  }
  const int ntiles = (L + kKT - 1) / kKT;
  const __nv_bfloat16* Kh = K + (size_t)bh * a.n * kD;
  const __nv_bfloat16* Vh = reinterpret_cast<const __nv_bfloat16*>(a.V) + (size_t)bh * a.n * kD;

  auto load_tile = [&](int buf, int t) {
    const int j0 = t * kKT;
    for (int e = tid; e < kKT * 8; e += kAttnThreads) {
      int r = e >> 3, seg = e & 7;
      const int off = r * 128 + ((seg ^ (r & 7)) * 16);
      if (j0 + r < L) {
        cp_async16(&kt[buf][off], Kh + (size_t)(j0 + r) * kD + seg * 8);
        cp_async16(&vt[buf][off], Vh + (size_t)(j0 + r) * kD + seg * 8);
      } else {
        *reinterpret_cast<uint4*>(&kt[buf][off]) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(&vt[buf][off]) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    if (HAS_BIAS && tid < kKT) {
      int j = j0 + tid, off = INT_MIN;
      if (a.bias_dense && j < a.n) off = -j;
      else if (!a.bias_dense && j >= a.prefix && j < a.n) { int tt = j - a.prefix; off = (tt / a.gw) * a.tw + tt % a.gw; }
      koff[buf][tid] = off;
    }
    cp_async_commit();
  };

  float of[8][4];
#pragma unroll
  for (int cb = 0; cb < 8; ++cb)
#pragma unroll
    for (int e = 0; e < 4; ++e) of[cb][e] = 0.0f;
  float run_m0 = -INFINITY, run_m1 = -INFINITY, lsum0 = 0.0f, lsum1 = 0.0f;
  const float kLog2e = 1.4426950408889634f;

  load_tile(0, 0);
  for (int t = 0; t < ntiles; ++t) {
    if (t + 1 < ntiles) { load_tile((t + 1) & 1, t + 1); cp_async_wait<1>(); }
    else cp_async_wait<0>();
    __syncthreads();
    const int buf = t & 1;
    const bool full = (t + 1) * kKT <= L;
    float lg[8][4];
    const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      float s[4] = {0.f, 0.f, 0.f, 0.f};
      // K B-fragments: key rows nb*8 + rr, channel chunks (mi) and (4 + mi)
      const int key = nb * 8 + rr;
      uint32_t kb0[4], kb1[4];
      ldmatrix_x4(kb0, &kt[buf][key * 128 + ((mi ^ (key & 7)) * 16)]);
      ldmatrix_x4(kb1, &kt[buf][key * 128 + (((4 + mi) ^ (key & 7)) * 16)]);
      mma_bf16_16x8x16(s, qf[0], kb0[0], kb0[1]);
      mma_bf16_16x8x16(s, qf[1], kb0[2], kb0[3]);
      mma_bf16_16x8x16(s, qf[2], kb1[0], kb1[1]);
      mma_bf16_16x8x16(s, qf[3], kb1[2], kb1[3]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int jl = nb * 8 + 2 * q + (e & 1);
        float bv = 0.0f;
        if (HAS_BIAS) {
          const int rb = (e < 2) ? rb0 : rb1, ko = koff[buf][jl];
          if (rb >= 0 && ko != INT_MIN) bv = __ldg(tab + (rb - ko));
        }
        const bool ok = (e < 2 ? row_ok0 : row_ok1) && (full || t * kKT + jl < L);
        lg[nb][e] = ok ? __fmaf_rn(s[e], rsd, bv) : -INFINITY;
      }
    }
    float tm0 = -INFINITY, tm1 = -INFINITY;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      tm0 = fmaxf(tm0, fmaxf(lg[nb][0], lg[nb][1]));
      tm1 = fmaxf(tm1, fmaxf(lg[nb][2], lg[nb][3]));
    }
    tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, 1));
    tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, 2));
    tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, 1));
    tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, 2));
    const float nm0 = fmaxf(run_m0, tm0), nm1 = fmaxf(run_m1, tm1);
    if (nm0 != run_m0) {
      const float al = (run_m0 == -INFINITY) ? 0.0f : fast_exp2((run_m0 - nm0) * kLog2e);
      lsum0 *= al;
#pragma unroll
      for (int cb = 0; cb < 8; ++cb) { of[cb][0] *= al; of[cb][1] *= al; }
    }
    if (nm1 != run_m1) {
      const float al = (run_m1 == -INFINITY) ? 0.0f : fast_exp2((run_m1 - nm1) * kLog2e);
      lsum1 *= al;
#pragma unroll
      for (int cb = 0; cb < 8; ++cb) { of[cb][2] *= al; of[cb][3] *= al; }
    }
    run_m0 = nm0; run_m1 = nm1;
    float pw[8][4];
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      pw[nb][0] = (lg[nb][0] == -INFINITY) ? 0.0f : fast_exp2((lg[nb][0] - nm0) * kLog2e);
      pw[nb][1] = (lg[nb][1] == -INFINITY) ? 0.0f : fast_exp2((lg[nb][1] - nm0) * kLog2e);
      pw[nb][2] = (lg[nb][2] == -INFINITY) ? 0.0f : fast_exp2((lg[nb][2] - nm1) * kLog2e);
      pw[nb][3] = (lg[nb][3] == -INFINITY) ? 0.0f : fast_exp2((lg[nb][3] - nm1) * kLog2e);
      lsum0 += pw[nb][0] + pw[nb][1];
      lsum1 += pw[nb][2] + pw[nb][3];
    }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t pa[4];
      pa[0] = pack_bf16x2(pw[2 * ks][0], pw[2 * ks][1]);
      pa[1] = pack_bf16x2(pw[2 * ks][2], pw[2 * ks][3]);
      pa[2] = pack_bf16x2(pw[2 * ks + 1][0], pw[2 * ks + 1][1]);
      pa[3] = pack_bf16x2(pw[2 * ks + 1][2], pw[2 * ks + 1][3]);
      const int key = ks * 16 + (mi & 1) * 8 + rr;
#pragma unroll
      for (int cbp = 0; cbp < 4; ++cbp) {
        const int chunk = 2 * cbp + (mi >> 1);
        uint32_t vb[4];
        ldmatrix_x4_trans(vb, &vt[buf][key * 128 + ((chunk ^ (key & 7)) * 16)]);
        mma_bf16_16x8x16(of[2 * cbp], pa, vb[0], vb[1]);
        mma_bf16_16x8x16(of[2 * cbp + 1], pa, vb[2], vb[3]);
      }
    }
    __syncthreads();
  }
  lsum0 += __shfl_xor_sync(0xffffffffu, lsum0, 1);
  lsum0 += __shfl_xor_sync(0xffffffffu, lsum0, 2);
  lsum1 += __shfl_xor_sync(0xffffffffu, lsum1, 1);
  lsum1 += __shfl_xor_sync(0xffffffffu, lsum1, 2);
  const float inv0 = row_ok0 ? 1.0f / lsum0 : 0.0f, inv1 = row_ok1 ? 1.0f / lsum1 : 0.0f;
#pragma unroll
  for (int rr2 = 0; rr2 < 2; ++rr2) {
    const int i = rr2 ? i1 : i0;
    if (i >= a.n) continue;
    const float inv = rr2 ? inv1 : inv0;
    const size_t o = ((size_t)bh * a.n + i) * kD;
#pragma unroll
    for (int cb = 0; cb < 8; ++cb) {
      const int ch = 8 * cb + 2 * q;
      const float x0 = of[cb][2 * rr2] * inv, x1 = of[cb][2 * rr2 + 1] * inv;
      if (a.o_bf16) *reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(a.O) + o + ch) = pack_bf16x2(x0, x1);
      else *reinterpret_cast<float2*>(reinterpret_cast<float*>(a.O) + o + ch) = make_float2(x0, x1);
    }
  }
}

}  // namespace had

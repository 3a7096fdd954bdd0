// common.cuh -- device helpers shared by the kernels of the binarized-QK top-N
// attention library (sm_100a).  Included once, by had_lib.cu.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace had {

constexpr int kD = 64;          // head dimension (the only one built)
constexpr int kW = kD / 32;     // packed 32-bit words per token
constexpr int kMaxN = 16384;    // longest sequence accepted
constexpr int kMaxHeads = 256;  // per-head logit scales travel in the kernel parameters

// Sticky device status bits (read and cleared by had_get_device_status()).
constexpr unsigned kDevErrSeqlen = 1u;
constexpr unsigned kDevErrTimeout = 2u;
constexpr unsigned kDevErrCapacity = 4u;

__device__ __forceinline__ void raise_status(unsigned* status, unsigned bits) {
  if (status) atomicOr(status, bits);
}

// Extended relative-position tables.  Entry rb(i) - koff(j) of the table is the
// bias of patch query i and patch key j, the (2gh-1) x (2gw-1) table being
// stored with a padded row stride S (the smallest S >= 2gw-1 with S = gw mod 32:
// the 32 consecutive query tokens of a warp then read 32 different shared-memory
// banks).  The extension appends regions that the same subtraction reaches for
// class-token queries (rb = rb_class), class-token keys (koff = k_class) and keys
// at or past the valid length (koff = k_invalid), so a kernel reads one table
// entry per (query, key) pair with no case analysis:
//   [0, T)              the table, T = (2gh-1) S (columns >= 2gw-1 unused)
//   [T, 2T + 2Kx)       class-token pairs (bias 0)
//   [2T + 2Kx, E)       keys past L (weight 0 / logit -inf), E = 3T + 3Kx rounded up to 4
// with Kx = (gh-1) S + gw the number of distinct patch key offsets y S + x.
struct RelposExt {
  int S, T, Kx, E, rb_class, k_class, k_invalid;
};
__host__ __device__ inline RelposExt relpos_ext(int gh, int gw) {
  RelposExt r;
  const int tw = 2 * gw - 1;
  r.S = tw + (((gw - tw) % 32) + 32) % 32;
  r.T = (2 * gh - 1) * r.S;
  r.Kx = (gh - 1) * r.S + gw;
  r.E = (3 * r.T + 3 * r.Kx + 3) / 4 * 4;  // padded to 16 bytes per head (bulk copies)
  r.rb_class = r.T - 1 + r.Kx;
  r.k_class = -(r.T + r.Kx);
  r.k_invalid = -(2 * r.T + 2 * r.Kx);
  return r;
}

// Extended tables of a dense bias matrix [n][n] (BinaryAttention §2.3, the
// "dense learnable matrix" option: one bias per query-key pair).  Row i sits at
// i * S with S >= n + 1 -- odd when the tables fit shared memory, so the 32
// query rows of a warp fall in distinct banks, else a multiple of 4 -- and
// column n of every row is the masked-key sentinel.  With
// rb(i) = i * S and koff(j) = -j (k_invalid = -n for keys past L), entry
// rb(i) - koff(j) is the pair (i, j), as with the relative-position tables.
// (S is odd only for tables small enough for shared memory; see below.)
// Tables that do not fit shared memory (more than kBiasSmemEntries entries) are
// read from global memory, and there a row stride that is a multiple of 4 lets a
// thread fetch 4 consecutive keys with one 16-byte load instead.
constexpr int kBiasSmemEntries = 6144;  // extended exp(bias) tables up to this many entries go to shared memory
struct DenseExt {
  int S, E, k_invalid;
};
__host__ __device__ inline DenseExt dense_ext(int n) {
  DenseExt r;
  r.S = (n + 1) | 1;
  if (n * r.S > kBiasSmemEntries) r.S = (n + 4) & ~3;
  r.E = (n * r.S + 3) / 4 * 4;  // padded to 16 bytes per head (bulk copies)
  r.k_invalid = -n;
  return r;
}
constexpr int kDenseBiasMaxN = 4096;  // a dense matrix grows as n^2: 2 tables of H * n * S floats

// Valid length of sequence b; an out-of-range entry raises the device status
// and returns 0, which makes every kernel treat that batch as empty (zero output).
__device__ __forceinline__ int valid_len(const int32_t* seqlens, int b, int n, unsigned* status) {
  if (!seqlens) return n;
  int L = seqlens[b];
  if (L < 1 || L > n) {
    raise_status(status, kDevErrSeqlen);
    return 0;
  }
  return L;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Expand 4 sign bits (bit 1 = -1) to four int8 lanes of +1 / -1 (0x01 / 0xFF).
__device__ __forceinline__ uint32_t expand_nibble_pm1(uint32_t nib) {
  uint32_t m = (nib * 0x00204081u) & 0x01010101u;  // one bit per byte, no carries
  return 0x01010101u | (m * 0xFEu);                // 0x01 -> +1, 0xFF -> -1
}
// The same four signs as e4m3 floats: +1.0 = 0x38, -1.0 = 0xB8 (the sign bit).
__device__ __forceinline__ uint32_t expand_nibble_pm1_e4m3(uint32_t nib) {
  uint32_t m = (nib * 0x00204081u) & 0x01010101u;
  return 0x38383838u | (m * 0x80u);
}
// Either encoding (bit 7 of a byte is its sign in both).
__device__ __forceinline__ uint32_t expand_nibble_pm(uint32_t nib, bool e4m3) {
  return e4m3 ? expand_nibble_pm1_e4m3(nib) : expand_nibble_pm1(nib);
}

// ---- legacy warp-level tensor-core MMAs (mma.sync), fp32 / s32 accumulators

__device__ __forceinline__ void mma_s8_16x8x32(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_u8s8_16x8x32(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16_16x8x16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void* smem_row_ptr) {
  uint32_t a = (uint32_t)__cvta_generic_to_shared(smem_row_ptr);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* smem_row_ptr) {
  uint32_t a = (uint32_t)__cvta_generic_to_shared(smem_row_ptr);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Order-preserving map of a float onto uint32 (x < y  <=>  key(x) < key(y)),
// with -0 folded onto +0 so that equal floats get equal keys.
__device__ __forceinline__ uint32_t float_order_key(float x) {
  uint32_t u = __float_as_uint(x + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// The float whose order key is k (the inverse of float_order_key on its range).
__device__ __forceinline__ float order_key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

}  // namespace had

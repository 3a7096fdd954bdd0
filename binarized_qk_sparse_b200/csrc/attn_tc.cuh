// attn_tc.cuh -- the fused binarized-QK top-N attention kernel on the sm_100a
// tensor cores (tcgen05 + TMA + tensor memory).
//
// One CTA = one (batch, head) and 128 query rows; query row r of the tile is
// tensor-memory lane r and softmax thread r, so every per-row step (histogram,
// threshold, tie rule, softmax, normalization) is thread-local.
//   warps 0-3  softmax/select: read a 64-key score tile from TMEM, build per-row
//              histograms, apply the top-N threshold, write P (or uint8 A) back
//              to TMEM, normalize and store O.
//   warp 4     MMA issuer (one thread) + TMEM allocation.
//   warp 5     TMA producer: +-1 int8 K tiles (64 keys x 64 B, 64-byte swizzle),
//              V tiles (bf16 [64 keys][64], 128-byte swizzle, MN-major B) or int8
//              V^T tiles ([64 channels][64 keys], 64-byte swizzle, K-major B).
// Tensor memory (256 columns): a ring of three score buffers S0..S2 [0,192), so
// the score MMAs of tiles t+1 and t+2 run while the softmax warps work on tile t,
// and O [192,256).  P of tile t is written over its own score buffer, each 32-key
// chunk inside that chunk's own 32 score columns (bf16 in [32c, 32c+16), the
// residual for fp32 V in [32c+16, 32c+32); uint8 codes in [32c, 32c+8)), so a
// thread never overwrites scores another thread has still to read.  The P.V MMA
// of tile t is issued before the score MMA that next writes that buffer, and
// MMAs from one thread run in issue order.
//
// Score (BinaryAttention §2.1/§2.2): S = Q~ K~^T with kind::i8 on +-1 operands,
// so S = d - 2*popcount(q XOR k) exactly.  A.V: kind::f16 (bf16 P from TMEM x
// bf16 V; fp32 V as bf16 head + residual, three products) or kind::i8 (uint8 A
// from TMEM x int8 V, BinaryAttention §2.4).
// Top-N (HAD: the N largest scores per query, ties to the lower key index):
//   LEVELS  histogram of the 65 score levels per row (thread-private counters);
//   no bias -> threshold level F and r_F ties to keep;
//   bias    -> band [fmaf(s_N,c,b_min), fmaf(s_max,c,b_max)]; RADIX passes over
//              the order-preserving uint32 key of l (128 bins) narrow it until the
//              threshold bin holds <= 64 keys; COLLECT ranks those exactly.
//   Keys with l > F are kept; keys with l == F are kept in key order while the
//   row's tie count is < r_F.
// Every mbarrier wait is bounded in SM clocks; on expiry the CTA records a
// device status bit, skips the rest of its work, and still frees its TMEM.
#pragma once

#include <climits>
#include <type_traits>

#include "common.cuh"
#include "sm100.cuh"

namespace had {
namespace tc {

using namespace had::sm100;

constexpr int kM = 128;            // query rows per CTA (TMEM lanes)
constexpr int kN = 64;             // keys per tile (score MMA N)
// Softmax threads per query row (SPLIT): dense attention always, and top-N without
// a bias on its P.V path for short ragged rows, split each 64-key tile between two threads
// (warps w and w + 4 share the TMEM lanes of quadrant w), which doubles the warps
// that hide latency; the two threads of a top-N row exchange their threshold-tie
// counts every tile so that ties are still kept in key order.  Long top-N rows,
// top-N with a bias and the top-N exports keep one thread per row.
__host__ __device__ constexpr int cta_threads(int split) { return 32 * (4 * split + 2); }
constexpr int kSplitMaxKeys = 256;  // top-N without a bias, ragged rows: two threads per row up to this n_pad
constexpr int kKStages = 4;
constexpr int kVStagesMax = 3;  // see v_stages()
// Score levels of a head dim: s = d - 2h takes d + 1 values.
__host__ __device__ constexpr int levels_of(int d) { return d + 1; }
constexpr int kRadixBins = 256;   // 16-bit counters, two per word (a row counts at most kMaxN keys)
constexpr int kCandCap = 128;    // power of two (the collect slot wraps)
constexpr int kSBufs = 3;
// Top-N with a bias on rows of at least kSampleMinTiles tiles: the first level pass
// reads one tile in kSampleStride (tile 8u + u % 8, which staggers the sample over
// every tile position), and each row brackets its threshold level from that sample
// with a margin of 5 binomial standard deviations.  The float-binned pass counts
// every key exactly and so verifies the bracket; if it failed for any row, the CTA
// runs the level pass again over every tile.
constexpr int kSampleStride = 8;   // power of two
constexpr int kSampleMinTiles = 64;
__host__ __device__ constexpr int tile_at(int u, int stride) { return stride == 1 ? u : u * stride + (u & (stride - 1)); }
// tiles u with tile_at(u, stride) < ntiles
__host__ __device__ constexpr int tiles_in_pass(int ntiles, int stride) {
  return stride == 1 ? ntiles : ntiles / stride + (((ntiles / stride) & (stride - 1)) < (ntiles & (stride - 1)) ? 1 : 0);
}
// TMEM: the score ring in columns [0, 192), O (d columns) from 192; 256 columns at
// d = 64 (two CTAs per SM), 512 at d = 128 (one CTA per SM).
constexpr uint32_t kColS = 0, kColO = 192;
__host__ __device__ constexpr uint32_t tmem_cols(int d) { return d <= 64 ? 256u : 512u; }
__host__ __device__ constexpr int ctas_per_sm(int d) { return d <= 64 ? 2 : 1; }
constexpr long long kWaitCycles = 2000000000LL;  // default bound of a pipeline wait: about one second
// First select pass of top-N with a bias (FBIN): u = sat(fmaf(l, sc, off)) in [0, 1]
// (one saturating FMA) and w = fmaf(u, 65535, kFbMg) are monotone functions of the
// logit l; w is an integer in [kFbMg, kFbMg + 65535] whose float bits carry w - kFbMg
// in their low 16 bits, and bits 9..15 are the bin (128 bins of 512 units): bin 0
// holds everything below the window, bins 1..126 the window, bin 127 the keys above
// it (and the top edge of the window).
constexpr float kFbMg = 12582912.0f;  // 1.5 * 2^23: unit spacing, bits 0x4B400000
constexpr float kFbSpan = 65535.0f;
constexpr int kFbGroup = 16;  // keys whose staged bias is read ahead of their histogram adds
__device__ __forceinline__ float fma_sat(float x, float y, float z) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(x), "f"(y), "f"(z));
  return r;
}
// How the softmax threads find the bias offset koff(j) = y_j * S + x_j of a key (S: table row stride):
constexpr int kKoffTable = 0;  // per-head table in shared memory (n_pad <= kKoffTableMax)
constexpr int kKoffWarp = 1;   // each softmax warp computes the tile's 64 offsets (double-buffered)
constexpr int kKoffTableMax = 1024;
// Bias variants of the kernel: none, extended tables read from global memory,
// (dense weights) the exp(bias) table staged in shared memory, or (dense
// weights) a dense bias matrix's exp(bias) rows read 4 keys per 16-byte load.
enum { BIAS_NONE = 0, BIAS_GLOBAL = 1, BIAS_SMEM = 2, BIAS_DGLOBAL = 3, BIAS_ROWS = 4 };
// BIAS_ROWS (a relative-position table with no class tokens on a grid whose rows
// hold a multiple of 64 patches): a warp's 32 query rows lie in one image row and
// a 64-key tile in another, so the bias of the pair (warp, tile) is 96 consecutive
// entries of one table row.  Each softmax warp copies that window into its own
// shared-memory slice (prefetched into registers one tile ahead), and a score's
// bias is then one shared load at a compile-time offset from a per-thread base.
constexpr int kRowWin = 96;  // entries of a warp's bias window (32 rows + 64 keys - 1, padded)
constexpr int kBiasSmemMax = kBiasSmemEntries;

// SEL_REF: the comparison mode -- standard dense attention on the unbinarized bf16
// Q and K (scores by a bf16 kind::f16 MMA, fp32 in TMEM), softmax(QK^T / sqrt(d) + B) V;
// it runs the dense softmax path with an online row maximum.
enum { SEL_DENSE = 0, SEL_TOPN_INT = 1, SEL_TOPN_FLOAT = 2, SEL_REF = 3 };
__host__ __device__ constexpr bool sel_dense(int sel) { return sel == SEL_DENSE || sel == SEL_REF; }
// V stages: three (the P.V tiles of dense and no-bias top-N kinds load further
// ahead), two for top-N with a bias and for fp32 V (their shared memory is fuller)
__host__ __device__ constexpr int v_stages(int sel, bool vf32) { return (sel == SEL_TOPN_FLOAT || vf32) ? 2 : 3; }
// MODE_Q4: uint8 A x 4-bit V (two keys per byte of V^T in HBM, expanded to the
// int8 MMA operand in shared memory by the TMA warp's lanes); otherwise as MODE_Q
enum { MODE_F = 0, MODE_Q = 1, MODE_Q4 = 2 };
enum { EXP_NONE = 0, EXP_IDX = 1, EXP_CODES = 2, EXP_SCORES = 3 };
enum { P_DONE = 0, P_NORM, P_LEVELS, P_FBIN, P_RADIX, P_COLLECT, P_KEPT_NORM, P_PV, P_IDX, P_CODES, P_SCORES };

struct TcArgs {
  CUtensorMap tm_k;   // +-1 int8 K [BH*n_pad][64], box {64, 64}, 64B swizzle
  CUtensorMap tm_v;   // V bf16 [BH*n][64], box {64, 64}, 128B swizzle          (float mode)
  CUtensorMap tm_vq;  // int8 V^T [BH*64][n_pad], box {64, 64}, 64B swizzle      (uint8 mode)
  CUtensorMap tm_vlo; // bf16 residual of fp32 V [BH*n][64], box {64, 64}         (fp32 V)
  CUtensorMap tm_q;   // comparison mode: raw bf16 Q [BH*n][D], box {64, 128}, 128B swizzle (tm_k: raw K, box {64, 64})
  const uint32_t* qbits;   // [BH][n][2]
  const int8_t* kpm;       // [BH][n_pad][64] +-1 codes of K (the score MMA's B operand)
  const void* v_raw;       // V as given, [BH][n][64] bf16 or fp32 (float mode)
  int v_f32;               // 1 if v_raw is fp32
  const float* vscale;     // [BH][64]
  const uint8_t* vq4;      // MODE_Q4: packed 4-bit V^T [BH][D][n_pad / 2], key 2k in the low nibble of byte k
  const float* table;      // [H][th][tw] or null
  int gh, gw, prefix, th, tw;
  const float* bminmax;    // [H][2] min/max of each head's table (0 included with class tokens)
  const float* expb;       // [H][E] extended exp(b - b_max(h)) table, or null
  const float* bext;       // [H][E] extended bias table, or null
  int ext_E, ext_S, rb_class, k_class, k_invalid;  // extended-table geometry (RelposExt or DenseExt)
  int bias_dense;          // 1: the bias is a dense [n][n] matrix per head (rb = i S, koff = -j)
  int int_levels;          // 1 if fp32(c*s) is strictly increasing in s for every head
  int koff_mode;           // kKoffTable / kKoffWarp
  const int32_t* seqlens;
  void* O;
  int o_bf16;
  int32_t* idx;
  uint8_t* codes;
  int row_begin, row_end;
  int B, H, n, n_pad, N;
  int32_t* scores;         // EXP_SCORES: [BH][n][n] int32
  unsigned* status;
  long long wait_cycles;   // bound of every pipeline wait, in SM clocks
  int force_expiry;        // test hook: one softmax thread first waits on a barrier nothing completes
  float c_head[kMaxHeads];
};

// Shared memory carve-up (offsets from a 1024-byte aligned base).
// d = 128 tiles are two 64-channel panels, each laid out as a d = 64 tile.
template <int D, int SEL, bool VF32, int BIAS>
struct Smem {
  static constexpr bool HAS_BIAS = BIAS != BIAS_NONE;
  static constexpr int kLev = levels_of(D);
  static constexpr int kVStage = (VF32 ? 2 : 1) * kN * D * 2;    // bf16 V tile (+ residual tile)
  static constexpr int kOpB = SEL == SEL_REF ? 2 : 1;            // bytes per Q, K element (bf16 or +-1 int8)
  static constexpr int kQ = 0;                                   // 128 x D elements
  static constexpr int kK = kQ + kM * D * kOpB;                  // 4 x 64 x D elements
  static constexpr int kVS = v_stages(SEL, VF32);
  static constexpr int kV = kK + kKStages * kN * D * kOpB;       // kVS V stages
  static constexpr int kKoff = kV + kVS * kVStage;               // bias key offsets (table, or 4 warps x 2 x 64)
  static constexpr int kBiasTab = kKoff + (HAS_BIAS ? kKoffTableMax * 4 : 0);  // exp(bias) table (dense)
  // row-pair exchange: dense 2 x 128 fp32 (partials); top-N 6 x 128 (threshold state) + 2 x 2 x 128 tie counts
  static constexpr int kXchg = kBiasTab + (BIAS == BIAS_SMEM ? kBiasSmemMax * 4 : 0);
  // top-N with a bias: a per-row candidate counter shared by the row's two threads, and a
  // second row of 128 for exchanging their radix counts
  static constexpr int kDq = kXchg + (sel_dense(SEL) ? 2 : SEL == SEL_TOPN_INT ? 10 : 2) * kM * 4;  // D dequant scales
  static constexpr int kBar = kDq + D * 4;
  static constexpr int kNumBars = 2 * kKStages + 2 * kVStagesMax + 2 * kSBufs + 5;
  static constexpr int kMisc = kBar + kNumBars * 8;              // [0] tmem base [1] abort
  static constexpr int kHist = (kMisc + 16 + 127) / 128 * 128;
  static constexpr int kHistBytes = sel_dense(SEL) ? kLev * 32 * 4
                                    : (SEL == SEL_TOPN_INT) ? kLev * kM * 4
                                    : (kCandCap > kLev ? kCandCap : kLev) * kM * 4;
  static constexpr int kTotal = kHist + kHistBytes + 1024;       // + alignment slack
  static_assert(kCandCap >= kRadixBins / 2, "the radix histogram fits the candidate area");
  static_assert(kMaxN < 65536, "a 16-bit radix counter holds every key of a row");
  static_assert((kCandCap & (kCandCap - 1)) == 0, "candidate slots wrap with a mask");
};

enum {
  B_KFULL = 0,
  B_KEMPTY = kKStages,
  B_VFULL = 2 * kKStages,
  B_VEMPTY = 2 * kKStages + kVStagesMax,
  B_SFULL = 2 * kKStages + 2 * kVStagesMax,  // one per score buffer
  B_TDONE = B_SFULL + kSBufs,             // one per score buffer
  B_OFULL = B_TDONE + kSBufs,
  B_FINAL,
  B_BIAS,  // staged exp(bias) table landed
  B_STALL,  // never completed: the force_expiry test hook waits on it
  B_QFULL   // comparison mode: the raw Q tile landed
};

// Bias offset of key j: koff = y_j * S + x_j for patch tokens, so that
// b_ij = ext[rb(i) - koff(j)]; class tokens and keys past L index the extension.
__device__ __forceinline__ int key_offset(const TcArgs& a, int j, int L) {
  if (j >= L) return a.k_invalid;
  if (a.bias_dense) return -j;
  if (j < a.prefix) return a.k_class;
  const int t = j - a.prefix;
  return (t / a.gw) * a.ext_S + t % a.gw;
}

// TMEM column (within a tile's P) of bf16 K-step k (16 keys): chunk k/2 sits in
// its own 32 columns, 8 columns per 16 keys.
__host__ __device__ constexpr uint32_t pcol(int k) { return 32u * (uint32_t)(k >> 1) + 8u * (uint32_t)(k & 1); }

// Of this chunk's threshold ties `eqm` (bit u = key jb + u, in key order), the
// ones the row keeps: ties are kept while fewer than r_F have been seen.
__device__ __forceinline__ uint32_t tie_keep(uint32_t eqm, int cut, int rF, int tie_seen) {
  uint32_t keep = eqm;
  if (cut && eqm != 0u) {
    const int allow = rF - tie_seen, cnt = __popc(eqm);
    if (allow <= 0) keep = 0u;
    else if (allow < cnt) keep = eqm & ((2u << __fns(eqm, 0u, allow)) - 1u);
  }
  return keep;
}

// Pairwise sum of 32 values (a depth-5 tree instead of a 32-long dependent chain).
__device__ __forceinline__ float sum32(const float (&e)[32]) {
  float t[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) t[u] = e[2 * u] + e[2 * u + 1];
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int u = 0; u < w; ++u) t[u] = t[2 * u] + t[2 * u + 1];
  return t[0];
}

template <int D, int SEL, int MODE, int BIAS, bool VF32, int EXPORT, int SPLIT>
__global__ void __launch_bounds__(cta_threads(SPLIT), ctas_per_sm(D)) k_attn_tc(const __grid_constant__ TcArgs a) {
  static_assert(D == 64 || D == 128, "head dims 64 and 128");
  constexpr int kLevels = levels_of(D);
  constexpr int kW = D / 32;        // packed words per token
  constexpr int kPan = D / 64;      // 64-channel panels of the Q~, K~ and V tiles
  constexpr uint32_t kTmemCols = tmem_cols(D);
  constexpr bool kRef = SEL == SEL_REF;        // the unbinarized comparison mode
  constexpr bool kQuant = MODE != MODE_F;       // uint8 A x int8 (or 4-bit) V
  // Top-N with a bias scores on the fp8 path: +-1 as e4m3 (kind::f8f6f4, fp32
  // accumulate), exact integers that the softmax threads read as floats; the other
  // kinds index level tables by the integer score and keep kind::i8.
  constexpr bool kF8 = SEL == SEL_TOPN_FLOAT;
  constexpr int kVStages = v_stages(SEL, VF32);
  constexpr bool kDense = sel_dense(SEL);
  static_assert(SPLIT == 1 || kDense || (SEL == SEL_TOPN_INT && EXPORT == EXP_NONE) ||
                    (SEL == SEL_TOPN_FLOAT && EXPORT == EXP_NONE && MODE == MODE_F),
                "two threads per row: dense, top-N without a bias on its P.V path, or top-N with a bias "
                "and float A.V");
  static_assert((BIAS != BIAS_SMEM && BIAS != BIAS_DGLOBAL) || kDense,
                "staged or vector-read exp(bias) tables serve the dense weights only");
  static_assert(BIAS != BIAS_ROWS || (SEL != SEL_TOPN_INT && 2 * (SPLIT == 2 ? 8 * 64 : 4 * kRowWin) <= kKoffTableMax),
                "the warps' bias-window slices fit the key-offset area");
  constexpr int kSplit = SPLIT;
  constexpr int kSoftWarps = 4 * kSplit;
  constexpr int kThreads = cta_threads(SPLIT);
  constexpr int kMmaWarp = kSoftWarps, kProdWarp = kSoftWarps + 1;
  constexpr int kChunks = 2 / kSplit;  // 32-key chunks of a tile per softmax thread
  constexpr bool HAS_BIAS = BIAS != BIAS_NONE;
  // top-N with a bias, float A.V: the final radix bin's keys are recorded (key
  // index) during the P.V pass and ranked, weighted and added to O afterwards,
  // instead of in a collect pass of their own; indices in slots [0, 64), their
  // logits in [64, 128) of the candidate area
  constexpr bool kMerge = SEL == SEL_TOPN_FLOAT && MODE == MODE_F && EXPORT == EXP_NONE;
  constexpr int kCap = kCandCap / 2;
  // top-N with a bias, two threads per row: both threads take every per-row decision
  // (from the shared histograms, so identically); candidates and recorded keys get
  // their slots from a per-row counter in shared memory
  constexpr bool kSplitF = kSplit == 2 && SEL == SEL_TOPN_FLOAT;
  using SM = Smem<D, SEL, VF32, BIAS>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sQ = sm + SM::kQ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + SM::kBar);
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + SM::kMisc);
  volatile uint32_t* abort_flag = misc + 1;
  int* koff_tab = reinterpret_cast<int*>(sm + SM::kKoff);
  float* dq = reinterpret_cast<float*>(sm + SM::kDq);
  uint32_t* hist = reinterpret_cast<uint32_t*>(sm + SM::kHist);
  float* xchg = reinterpret_cast<float*>(sm + SM::kXchg);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool is_soft = warp < kSoftWarps;
  const int srow = tid & (kM - 1);          // softmax thread: query row within the tile (TMEM lane)
  const int half = (warp >> 2) & 1;         // softmax thread: which 32-key chunk of a tile (split rows)
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int q0 = blockIdx.x * kM;
  const int L = valid_len(a.seqlens, b, a.n, a.status);
  const float c = a.c_head[h];
  const int keff = (a.N == 0 || a.N >= L) ? L : a.N;
  const int ntiles = (L + kN - 1) / kN;

  // ---------------------------------------------------------------- tile past L: zeros, no TMEM
  if (q0 >= L) {
    if (EXPORT == EXP_NONE) {
      for (int e = tid; e < kM * D; e += kThreads) {
        const int r = q0 + e / D, ch = e % D;
        if (r < a.n) {
          const size_t o = ((size_t)bh * a.n + r) * D + ch;
          if (a.o_bf16) reinterpret_cast<__nv_bfloat16*>(a.O)[o] = __float2bfloat16(0.0f);
          else reinterpret_cast<float*>(a.O)[o] = 0.0f;
        }
      }
    } else if (EXPORT == EXP_IDX) {
      for (int e = tid; e < kM * a.N; e += kThreads) {
        const int r = q0 + e / a.N;
        if (r < a.n) a.idx[((size_t)bh * a.n + r) * a.N + e % a.N] = -1;
      }
    } else if (EXPORT == EXP_SCORES) {
      for (int e = tid; e < kM * a.n; e += kThreads) {
        const int r = q0 + e / a.n;
        if (r < a.n) a.scores[((size_t)bh * a.n + r) * a.n + e % a.n] = 0;
      }
    } else {
      const int rows = a.row_end - a.row_begin;
      for (int e = tid; e < kM * a.n; e += kThreads) {
        const int r = q0 + e / a.n;
        if (r >= a.row_begin && r < a.row_end && r < a.n)
          a.codes[((size_t)bh * rows + (r - a.row_begin)) * a.n + e % a.n] = 0;
      }
    }
    return;
  }

  // ---------------------------------------------------------------- setup
  // K~ tile of key tile tt into K stage st: one 64-byte-wide box per 64-channel panel
  // (comparison mode: raw bf16 K rows, 128-byte panels of 64 channels)
  auto load_k = [&](uint32_t st, int tt) {
    mbar_arrive_expect_tx(&bars[B_KFULL + st], kN * D * SM::kOpB);
#pragma unroll
    for (int pn = 0; pn < kPan; ++pn) {
      if (kRef)
        tma_load_2d(sm + SM::kK + st * kN * D * 2 + pn * kN * 128, &a.tm_k, 64 * pn, bh * a.n + tt * kN,
                    &bars[B_KFULL + st]);
      else
        tma_load_2d(sm + SM::kK + st * kN * D + pn * kN * 64, &a.tm_k, 64 * pn, bh * a.n_pad + tt * kN,
                    &bars[B_KFULL + st]);
    }
  };
  int k_par[kKStages], v_par[kVStages];  // producer: parity of the last load per stage (-1 none)
#pragma unroll
  for (int s2 = 0; s2 < kKStages; ++s2) k_par[s2] = -1;
#pragma unroll
  for (int s2 = 0; s2 < kVStages; ++s2) v_par[s2] = -1;
  // the producer issues the first K tiles before the CTA-wide setup barrier, so
  // their load latency overlaps the staging of Q
  bool sample_levels = false;
  if (SEL == SEL_TOPN_FLOAT && ntiles >= kSampleMinTiles && keff < L) {
    // weights exp(l - m) with m from the sample stay inside fp32 while (2 d c + bias range) log2 e <= 100
    const float range = HAS_BIAS ? a.bminmax[2 * h + 1] - a.bminmax[2 * h] : 0.0f;
    sample_levels = c > 0.0f && (2.0f * D * c + range) * 1.4426950408889634f <= 100.0f;
  }
  const int s_first = sample_levels ? kSampleStride : 1;  // stride of the first pass's tiles
  const int n_sampled = tiles_in_pass(ntiles, kSampleStride);
  const int k_pre = min(tiles_in_pass(ntiles, s_first), kKStages);
  if (warp == kMmaWarp) {
    tmem_alloc(misc, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProdWarp && lane == 0) {
    for (int s = 0; s < kKStages; ++s) { mbar_init(&bars[B_KFULL + s], 1); mbar_init(&bars[B_KEMPTY + s], 1); }
    for (int s = 0; s < kVStages; ++s) { mbar_init(&bars[B_VFULL + s], 1); mbar_init(&bars[B_VEMPTY + s], 1); }
    for (int s = 0; s < kSBufs; ++s) { mbar_init(&bars[B_SFULL + s], 1); mbar_init(&bars[B_TDONE + s], 32 * kSoftWarps); }
    mbar_init(&bars[B_OFULL], 1);
    mbar_init(&bars[B_FINAL], 1);
    mbar_init(&bars[B_BIAS], 1);
    mbar_init(&bars[B_STALL], 1);
    mbar_init(&bars[B_QFULL], 1);
    misc[1] = 0;
    fence_barrier_init();
    if (BIAS == BIAS_SMEM) {
      // the head's exp(bias) table, one bulk copy that overlaps the rest of the setup
      mbar_arrive_expect_tx(&bars[B_BIAS], (uint32_t)a.ext_E * 4u);
      bulk_load(sm + SM::kBiasTab, a.expb + (size_t)h * a.ext_E, (uint32_t)a.ext_E * 4u, &bars[B_BIAS]);
    }
    prefetch_tensormap(&a.tm_k);
    if (EXPORT == EXP_NONE && MODE != MODE_Q4) prefetch_tensormap(MODE == MODE_Q ? &a.tm_vq : &a.tm_v);
    if (kRef) {  // the raw Q tile: rows past the tensor read as zeros, other heads' rows are never stored
      mbar_arrive_expect_tx(&bars[B_QFULL], kM * D * 2);
#pragma unroll
      for (int pn = 0; pn < kPan; ++pn)
        tma_load_2d(sQ + pn * kM * 128, &a.tm_q, 64 * pn, bh * a.n + q0, &bars[B_QFULL]);
    }
    for (int u = 0; u < k_pre; ++u) {  // stage u = the first pass's u-th tile, first use of every stage
      load_k((uint32_t)u, tile_at(u, s_first));
      k_par[u] = 0;
    }
  }
  const int row = q0 + srow;  // softmax threads
  const bool row_ok = is_soft && row < L;
  if (tid < kM) {
    // Q~ row into the 64-byte swizzled K-major A operand, one 128 x 64 B panel per
    // 64 channels (16-byte chunk c of a panel row -> c ^ ((row >> 1) & 3))
    uint32_t wq[kW];
#pragma unroll
    for (int k = 0; k < kW; ++k) wq[k] = 0u;
    if (row_ok && !kRef) {
      const uint2* qw = reinterpret_cast<const uint2*>(a.qbits + ((size_t)bh * a.n + row) * kW);
#pragma unroll
      for (int k = 0; k < kW / 2; ++k) {
        const uint2 w = __ldg(qw + k);
        wq[2 * k] = w.x;
        wq[2 * k + 1] = w.y;
      }
    }
#pragma unroll
    for (int c16 = 0; c16 < (kRef ? 0 : D / 16); ++c16) {  // 16 channels per chunk
      const uint32_t f = wq[c16 >> 1] >> ((c16 & 1) * 16);
      uint4 v;
      v.x = expand_nibble_pm(f & 15u, kF8);
      v.y = expand_nibble_pm((f >> 4) & 15u, kF8);
      v.z = expand_nibble_pm((f >> 8) & 15u, kF8);
      v.w = expand_nibble_pm((f >> 12) & 15u, kF8);
      const int pn = c16 >> 2, cch = c16 & 3;
      *reinterpret_cast<uint4*>(sQ + pn * kM * 64 + tid * 64 + ((cch ^ ((tid >> 1) & 3)) * 16)) = v;
    }
    if (!kDense)
      for (int lev = 0; lev < kLevels; ++lev) hist[lev * kM + srow] = 0u;
    if (kDense) {
      // per-lane copies of the level table exp(c * (s - d)), level k = (d - s) / 2, at [k][lane]
      // (lane l computes levels l, l + 32, ...; warp w writes levels w, w + 4, ... via shuffles)
      const float ck = -2.0f * a.c_head[h] * 1.4426950408889634f;
      float* lt = reinterpret_cast<float*>(hist);
      float lv[(kLevels + 31) / 32];
#pragma unroll
      for (int k = 0; k < (kLevels + 31) / 32; ++k) lv[k] = exp2f(ck * (float)(lane + 32 * k));
      for (int lev = warp; lev < kLevels; lev += 4) {
        float v = lv[0];
#pragma unroll
        for (int k = 1; k < (kLevels + 31) / 32; ++k) v = (lev >> 5) == k ? lv[k] : v;
        lt[lev * 32 + lane] = __shfl_sync(0xffffffffu, v, lev & 31);
      }
    }
    if (kQuant && EXPORT == EXP_NONE && tid < D) dq[tid] = __fdiv_rn(a.vscale[(size_t)bh * D + tid], 255.0f);
    if (HAS_BIAS && BIAS != BIAS_ROWS && a.koff_mode == kKoffTable)
      for (int j = tid; j < a.n_pad; j += kM) koff_tab[j] = 4 * key_offset(a, j, L);  // in bytes
    fence_proxy_async();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  // ---------------------------------------------------------------- per-row state (softmax threads)
  float F = -INFINITY, m = -INFINITY, scale = 1.0f, lsum = 0.0f;
  int rF = 0, cut = 0, tie_seen = 0, kept_seen = 0;
  uint32_t r_uhi = 0, r_span = 0;
  // r_state: 0 threshold known, 1 radix pass next, 2 collect pass next, 3 the
  // window's keys are recorded during the P.V pass (kMerge), 4 FBIN pass next,
  // 5 a bracket from the sampled level pass missed (the level pass runs again)
  int r_shift = 0, r_rank = 0, r_state = 0, r_cnt = 0;
  int r_above = 0;      // keys above the first radix window (counted in that pass)
  bool r_sampled = false;  // the FBIN bracket came from the sampled level pass
  float fb_sc = 0.0f, fb_off = 0.0f;  // r_state 4: the FBIN pass's map of logits onto bins
  // float window of the P.V pass: weight for l >= w_cut; keys in [w_lo, w_hi] are
  // the ties at F (w_lo = w_hi = w_cut = F), or, with the collect folded into
  // the P.V pass, the final radix bin (w_cut just above w_hi), ranked after it
  float w_lo = INFINITY, w_hi = INFINITY, w_cut = INFINITY;
  bool r_first = false;  // the next radix pass is the first of this row
  // row base of the extended bias tables: rb(i) - koff(j) indexes the pair (i, j);
  // class-token rows and rows past the tensor use the class-row base
  int rb = 0;
  if (HAS_BIAS) {
    rb = a.rb_class;
    if (a.bias_dense) {
      rb = min(row, a.n - 1) * a.ext_S;  // rows past the tensor are never stored
    } else if (row >= a.prefix && row < a.n) {
      const int t = row - a.prefix;
      rb = (t / a.gw + a.gh - 1) * a.ext_S + (t % a.gw + a.gw - 1);
    }
  }
  const float* tab = HAS_BIAS ? a.bext + (size_t)h * a.ext_E : nullptr;
  const float kLog2e = 1.4426950408889634f;
  // Dense weights as (level table) x exp(b - b_max): both factors <= 1, so no row
  // maximum is needed as long as the smallest product stays far from fp32 underflow.
  bool use_lut = false;
  if (kDense && !kRef) {
    const float range = HAS_BIAS ? a.bminmax[2 * h + 1] - a.bminmax[2 * h] : 0.0f;
    use_lut = c > 0.0f && (2.0f * D * c + range) * kLog2e <= 100.0f;
  }
  const bool sum_in_pv = (MODE == MODE_F) && (SEL == SEL_TOPN_FLOAT || (kDense && use_lut));
  int sF = 0;  // integer threshold score (top-N without bias)

  uint32_t g_k = 0, g_v = 0, g_s = 0;  // tiles issued so far (all passes), per role

  int pass = (kDense) ? (EXPORT == EXP_IDX ? P_IDX : EXPORT == EXP_SCORES ? P_SCORES : P_NORM) : P_LEVELS;
  if (kDense && EXPORT == EXP_NONE && MODE == MODE_F && use_lut) pass = P_PV;

  auto bounded_wait = [&](int bar, uint32_t parity) -> bool {
    if (mbar_test_wait(smem_u32(&bars[bar]), parity)) return true;  // phase already complete
    if (*abort_flag) return false;
    if (mbar_wait(&bars[bar], parity, a.wait_cycles)) return true;
    *abort_flag = 1u;
    raise_status(a.status, kDevErrTimeout);
    return false;
  };
  // test hook of the timeout path: one softmax thread first waits on a barrier
  // that nothing completes, so its bound expires and the CTA winds down
  if (a.force_expiry && tid == 0) bounded_wait(B_STALL, 0);

  // K tiles of a short key range stay in the K stages for every pass (loaded once)
  const bool k_res = ntiles <= kKStages;
  bool first_pass = true;
  int v_pref = 0;  // producer: V tiles of the P.V pass already issued
  int pv_xchg = 1;  // split P.V: some row of the CTA cuts its ties at F (the halves exchange tie counts)
  // producer, 4-bit V: the packed V^T rows (32 bytes = 64 keys per channel row, D / 32
  // rows per lane) of tile q4_tile, loaded ahead of their expansion
  uint4 q4_next[MODE == MODE_Q4 ? D / 32 : 1][2];
  int q4_tile = -1;
  auto q4_fetch = [&](int t) {
    if (MODE != MODE_Q4) return;
    const uint8_t* src = a.vq4 + (size_t)bh * D * (a.n_pad / 2) + (size_t)t * (kN / 2);
#pragma unroll
    for (int rr = 0; rr < (MODE == MODE_Q4 ? D / 32 : 1); ++rr) {
      const uint4* sp = reinterpret_cast<const uint4*>(src + (size_t)(lane + 32 * rr) * (a.n_pad / 2));
      q4_next[rr][0] = __ldg(sp);
      q4_next[rr][1] = __ldg(sp + 1);
    }
    q4_tile = t;
  };
  while (pass != P_DONE) {
    const bool pv = (pass == P_PV);
    // this pass's tiles: tile_at(u, p_stride) for u < npass (the sampled first level
    // pass, or every tile); the ring counters advance by npass
    const int p_stride = (pass == P_LEVELS && sample_levels) ? kSampleStride : 1;
    const int npass = p_stride == 1 ? ntiles : n_sampled;
    // ============================================================== producer warp
    if (warp == kProdWarp) {
      auto load_v = [&](int t) {
        const uint32_t vs = g_v % kVStages;
        if (MODE == MODE_Q4) {
          // 4-bit V: every lane expands D / 32 channel rows of the packed tile (32 bytes:
          // keys 64t ... 64t + 63) into the int8 V^T operand ([D][64], 64-byte swizzle:
          // 16-byte chunk q of row c at q ^ ((c >> 1) & 3)), then lane 0 marks it full.
          // The packed rows come from registers loaded one call earlier (the calls go
          // t = 0, 1, 2, ... in every P.V pass), so their latency overlaps a tile of work.
          if (q4_tile != t) q4_fetch(t);
          uint4 cur[D / 32][2];
#pragma unroll
          for (int rr = 0; rr < D / 32; ++rr) { cur[rr][0] = q4_next[rr][0]; cur[rr][1] = q4_next[rr][1]; }
          if (t + 1 < ntiles) q4_fetch(t + 1);
          const bool free_ok = __all_sync(0xffffffffu, g_v < (uint32_t)kVStages ||
                                                           bounded_wait(B_VEMPTY + vs, ((g_v / kVStages) - 1) & 1));
          if (free_ok && !*abort_flag) {
            uint8_t* dst = sm + SM::kV + vs * SM::kVStage;
#pragma unroll
            for (int rr = 0; rr < D / 32; ++rr) {
              const int c = lane + 32 * rr;
              const uint32_t pw[8] = {cur[rr][0].x, cur[rr][0].y, cur[rr][0].z, cur[rr][0].w,
                                      cur[rr][1].x, cur[rr][1].y, cur[rr][1].z, cur[rr][1].w};  // 8 keys per word
#pragma unroll
              for (int q = 0; q < 4; ++q) {  // 16 keys per 16-byte chunk: packed words 2q, 2q + 1
                uint32_t o[4];
#pragma unroll
                for (int hw = 0; hw < 2; ++hw) {
                  const uint32_t w = pw[2 * q + hw];
                  // nibbles to signed bytes: x | 0xF0 where bit 3 is set (8 * 0x1E = 0xF0, no
                  // carry between bytes); even keys in the low nibbles, odd keys in the high
                  uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
                  lo |= (lo & 0x08080808u) * 0x1Eu;
                  hi |= (hi & 0x08080808u) * 0x1Eu;
                  o[2 * hw] = __byte_perm(lo, hi, 0x5140);
                  o[2 * hw + 1] = __byte_perm(lo, hi, 0x7362);
                }
                *reinterpret_cast<uint4*>(dst + c * 64 + ((q ^ ((c >> 1) & 3)) * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
              }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_VFULL + vs]);
          }
          ++g_v;
          return;
        }
        if (lane == 0 && g_v >= (uint32_t)kVStages) bounded_wait(B_VEMPTY + vs, ((g_v / kVStages) - 1) & 1);
        if (lane == 0 && !*abort_flag) {
          uint8_t* dst = sm + SM::kV + vs * SM::kVStage;
          if (kQuant) {  // int8 V^T: D channels x 64 keys in one box
            mbar_arrive_expect_tx(&bars[B_VFULL + vs], D * kN);
            tma_load_2d(dst, &a.tm_vq, t * kN, bh * D, &bars[B_VFULL + vs]);
          } else {  // bf16 V: one [64 keys][64 channels] box per panel (+ the residual panels)
            mbar_arrive_expect_tx(&bars[B_VFULL + vs], SM::kVStage);
#pragma unroll
            for (int pn = 0; pn < kPan; ++pn) {
              tma_load_2d(dst + pn * kN * 128, &a.tm_v, 64 * pn, bh * a.n + t * kN, &bars[B_VFULL + vs]);
              if (VF32)
                tma_load_2d(dst + kN * D * 2 + pn * kN * 128, &a.tm_vlo, 64 * pn, bh * a.n + t * kN,
                            &bars[B_VFULL + vs]);
            }
          }
          v_par[vs] = (int)((g_v / kVStages) & 1);
        }
        ++g_v;
      };
      for (int u = 0; u < npass; ++u) {
        const int t = tile_at(u, p_stride);
        if (first_pass && u < k_pre) {
          ++g_k;  // issued during setup
        } else if (!k_res || first_pass) {
          const uint32_t st = k_res ? (uint32_t)t : g_k % kKStages;
          if (!k_res && lane == 0 && g_k >= (uint32_t)kKStages)
            bounded_wait(B_KEMPTY + st, ((g_k / kKStages) - 1) & 1);
          if (lane == 0 && !*abort_flag) {
            load_k(st, t);
            k_par[st] = k_res ? 0 : (int)((g_k / kKStages) & 1);
          }
          ++g_k;
        }
        if (pv && t >= v_pref) load_v(t);
      }
      // the P.V pass comes last: its first V tiles can load while this pass runs
      if (EXPORT == EXP_NONE && !pv && v_pref == 0)
        for (; v_pref < kVStages && v_pref < ntiles; ++v_pref) load_v(v_pref);
    }
    // ============================================================== MMA issuer warp (one thread)
    else if (warp == kMmaWarp) {
      if (lane == 0) {
        // scores: +-1 int8 (kind::i8), or bf16 Q x bf16 K (kind::f16) in the comparison mode
        const uint32_t id_s = kRef ? idesc_bf16(kM, kN, false) : kF8 ? idesc_e4m3(kM, kN) : idesc_i8(kM, kN, true, true, false);
        if (kRef && first_pass) bounded_wait(B_QFULL, 0);
        // P.V: uint8 codes x int8 V^T (N = D, one MMA per K-step), or bf16 P x bf16 V
        // (N = 64 per 64-channel panel)
        const uint32_t id_pv = (kQuant) ? idesc_i8(kM, D, false, true, false) : idesc_bf16(kM, 64, true);
        auto issue_scores = [&](int t) {
          const uint32_t gk = g_k + (uint32_t)t, buf = (g_s + (uint32_t)t) % kSBufs;
          const uint32_t st = k_res ? (uint32_t)t : gk % kKStages;
          if (!bounded_wait(B_KFULL + st, k_res ? 0u : (gk / kKStages) & 1)) return;
          tc_fence_after();
          const uint32_t kq = smem_u32(sQ), kk = smem_u32(sm + SM::kK + st * kN * D * SM::kOpB);
          if (kRef) {
#pragma unroll
            for (int pn = 0; pn < kPan; ++pn)  // four 16-channel K-steps per 64-channel bf16 panel
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_f16_ss(tmem + kColS + buf * kN, sdesc(kq + pn * kM * 128 + 32 * ks, 16, 1024, kSwizzle128B),
                           sdesc(kk + pn * kN * 128 + 32 * ks, 16, 1024, kSwizzle128B), id_s, (pn | ks) > 0 ? 1u : 0u);
          } else {
#pragma unroll
            for (int pn = 0; pn < kPan; ++pn)  // two 32-channel K-steps per 64-channel panel
#pragma unroll
              for (int ks = 0; ks < 2; ++ks)
                if (kF8)
                  mma_f8_ss(tmem + kColS + buf * kN, sdesc(kq + pn * kM * 64 + 32 * ks, 16, 512, kSwizzle64B),
                            sdesc(kk + pn * kN * 64 + 32 * ks, 16, 512, kSwizzle64B), id_s, (pn | ks) > 0 ? 1u : 0u);
                else
                  mma_i8_ss(tmem + kColS + buf * kN, sdesc(kq + pn * kM * 64 + 32 * ks, 16, 512, kSwizzle64B),
                            sdesc(kk + pn * kN * 64 + 32 * ks, 16, 512, kSwizzle64B), id_s, (pn | ks) > 0 ? 1u : 0u);
          }
          mma_commit(&bars[B_SFULL + buf]);
          if (!k_res) mma_commit(&bars[B_KEMPTY + st]);
        };
        for (int t = 0; t < kSBufs && t < npass; ++t) issue_scores(t);
        for (int t = 0; t < npass; ++t) {  // t counts this pass's tiles (all of them in the P.V pass)
          const uint32_t gs = g_s + (uint32_t)t, buf = gs % kSBufs;
          const uint32_t colP = kColS + buf * kN;  // P of this tile sits over its score buffer
          bounded_wait(B_TDONE + buf, (gs / kSBufs) & 1);
          tc_fence_after();
          if (pv && !*abort_flag) {
            const uint32_t gv = g_v + (uint32_t)t, vs = gv % kVStages;
            if (bounded_wait(B_VFULL + vs, (gv / kVStages) & 1)) {
              tc_fence_after();
              const uint32_t vbase = smem_u32(sm + SM::kV + vs * SM::kVStage);
              if (kQuant) {
#pragma unroll
                for (int k = 0; k < kN / 32; ++k)  // K-step k = key chunk k: codes at columns 32k
                  mma_i8_ts(tmem + kColO, tmem + colP + 32 * k, sdesc(vbase + 32 * k, 16, 512, kSwizzle64B), id_pv,
                            (t > 0 || k > 0) ? 1u : 0u);
              } else {
#pragma unroll
                for (int pn = 0; pn < kPan; ++pn) {  // O columns [64 pn, 64 pn + 64) from V panel pn
                  const uint32_t vp = vbase + pn * kN * 128, op = tmem + kColO + 64 * pn;
#pragma unroll
                  for (int k = 0; k < kN / 16; ++k)  // 16 keys per K-step: chunk k/2, columns 32(k/2) + 8(k%2)
                    mma_f16_ts(op, tmem + colP + pcol(k), sdesc(vp + 2048 * k, 0, 1024, kSwizzle128B), id_pv,
                               (t > 0 || k > 0) ? 1u : 0u);
                  if (VF32) {
                    // residual products: P_hi x V_lo and P_lo x V_hi
                    const uint32_t vlo = vbase + kN * D * 2 + pn * kN * 128;
#pragma unroll
                    for (int k = 0; k < kN / 16; ++k)
                      mma_f16_ts(op, tmem + colP + pcol(k), sdesc(vlo + 2048 * k, 0, 1024, kSwizzle128B), id_pv, 1u);
#pragma unroll
                    for (int k = 0; k < kN / 16; ++k)
                      mma_f16_ts(op, tmem + colP + pcol(k) + 16, sdesc(vp + 2048 * k, 0, 1024, kSwizzle128B), id_pv,
                                 1u);
                  }
                }
              }
              mma_commit(&bars[B_VEMPTY + vs]);
              if (t + 1 == ntiles) mma_commit(&bars[B_OFULL]);
            }
          }
          if (t + kSBufs < npass) issue_scores(t + kSBufs);
        }
      }
      g_k += npass;
      g_s += npass;
      if (pv) g_v += ntiles;
    }
    // ============================================================== softmax / select warps
    else {
      // a score from its TMEM word: an fp32 integer on the fp8 path, else an int32
      auto score_f = [&](uint32_t v) -> float { return kF8 ? __uint_as_float(v) : (float)(int)v; };
      const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
      const uint32_t hist_row = smem_u32(hist) + (uint32_t)srow * 4u;
      const float mo = -m * kLog2e;
      // P.V with two threads per row: the weighting cut, the float just above F for a row
      // whose ties at F are resolved by count (w_lo == w_cut), else w_cut itself
      const float pv_cut = (w_lo == w_cut && w_cut != INFINITY) ? order_key_float(float_order_key(w_cut) + 1u) : w_cut;
      const float* lut = reinterpret_cast<const float*>(hist);
      const float* lut_lane = lut + (D / 2) * 32 + lane;  // dense level table: entry for score s at lut_lane[-16 s]
      // this row's weight table (top-N without a bias): level (d - s) / 2 at
      // lut[(d/2 - s / 2) kM + srow], i.e. byte (d/2 kM + srow) * 4 - s * 2 kM (s is even)
      const char* wrow = reinterpret_cast<const char*>(lut + (D / 2) * kM + srow);
      // Passes compiled into this instantiation (the rest are pruned at compile time).
      constexpr bool kHasLevels = !kDense;
      constexpr bool kHasNorm = kDense;
      constexpr bool kHasRadix = SEL == SEL_TOPN_FLOAT;
      constexpr bool kHasKeptNorm = SEL == SEL_TOPN_FLOAT && (kQuant || EXPORT == EXP_CODES);
      constexpr bool kHasIdx = EXPORT == EXP_IDX;
      constexpr bool kHasCodes = EXPORT == EXP_CODES;
      constexpr bool kHasPv = EXPORT == EXP_NONE;
      // lut_e: dense weights from the level table x exp(bias - b_max) (no row max needed)
      // lut_w: top-N (no bias) weights from the row's level table, zero below the threshold
      const bool lut_e = (kDense) && use_lut && (pass == P_NORM || pass == P_PV || pass == P_CODES);
      const bool lut_w = (SEL == SEL_TOPN_INT) && a.int_levels && pass == P_PV;
      const bool wants_bias = HAS_BIAS && pass != P_LEVELS;
      // exp(b - b_max) of this row (dense): row base rb(i) into the staged or global table
      // (key offsets are kept in bytes: entry (i, j) sits at row base - koff_bytes(j))
      const char* eb_bytes = nullptr;
      if (BIAS == BIAS_SMEM) eb_bytes = reinterpret_cast<const char*>(reinterpret_cast<const float*>(sm + SM::kBiasTab) + rb);
      else if (HAS_BIAS && kDense) eb_bytes = reinterpret_cast<const char*>(a.expb + (size_t)h * a.ext_E + rb);
      const char* tab_bytes = HAS_BIAS ? reinterpret_cast<const char*>(tab + rb) : nullptr;
      // a warp whose 32 rows all lie past L only keeps the barrier phases going
      const bool warp_live = __any_sync(0xffffffffu, row < L);
      // per-warp offsets: patch (y, x) of keys j0 + lane and j0 + 32 + lane, advanced
      // by 64 keys per tile without a division
      int ya = 0, xa = 0, yb = 0, xb = 0;
      const int q64 = HAS_BIAS ? kN / a.gw : 0, r64 = HAS_BIAS ? kN % a.gw : 0;
      auto patch_of = [&](int j, int& y, int& x) {
        const int tt = max(j - a.prefix, 0);
        y = tt / a.gw;
        x = tt - y * a.gw;
      };
      auto advance = [&](int& y, int& x) {
        y += q64;
        x += r64;
        if (x >= a.gw) { x -= a.gw; ++y; }
      };
      auto offset_of = [&](int j, int y, int x) -> int {  // in bytes
        if (a.bias_dense) return 4 * (j >= L ? a.k_invalid : -j);
        return 4 * (j >= L ? a.k_invalid : (j < a.prefix ? a.k_class : y * a.ext_S + x));
      };
      // BIAS_ROWS: this warp's 32 rows (one image row) and its two window slices.
      // Entry e of the window of tile t is table[y_w - y_k + gh - 1][x_w - x_k + gw - 64 + e]
      // (x_k, y_k of the tile's first key): row (lane) and key u of the tile read entry
      // lane + 63 - u.  One thread per row reads entries 0..94; with two threads per row
      // each warp takes 32 keys and needs 63 entries starting at 32 (keys 0..31) or 0.
      constexpr int kRwEnt = kSplit == 2 ? 64 : kRowWin;  // entries per slice (32 per load)
      const int rw_first = kSplit == 2 ? 32 * (1 - half) : 0;
      float* rw_slice0 = nullptr;
      const float* rw_src = nullptr;
      int rw_yw = 0, rw_xw = 0;
      float rwb[kRwEnt / 32];
#pragma unroll
      for (int i = 0; i < kRwEnt / 32; ++i) rwb[i] = 0.0f;
      if (BIAS == BIAS_ROWS) {
        const int r0 = q0 + 32 * (warp & 3);
        rw_yw = r0 / a.gw;
        rw_xw = r0 - rw_yw * a.gw;
        rw_slice0 = reinterpret_cast<float*>(koff_tab) + warp * 2 * kRwEnt;
        // dense weights read exp(b - b_max) (the level-table path), the rest the bias itself
        rw_src = ((kDense && use_lut) ? a.expb : a.bext) + (size_t)h * a.ext_E + rw_first;
      }
      // the next tile's window into registers (coalesced loads); the tiles of a pass are
      // fetched in order, so the key tile's patch (rw_fy, rw_fx) advances by 64 columns
      // (grid rows hold a multiple of 64 patches)
      int rw_fy = 0, rw_fx = 0;
      auto rw_fetch = [&]() {
        const float* src = rw_src + (rw_yw - rw_fy + a.gh - 1) * a.ext_S + (rw_xw - rw_fx + a.gw - kN);
#pragma unroll
        for (int i = 0; i < kRwEnt / 32; ++i) rwb[i] = __ldg(src + 32 * i + lane);
        rw_fx += kN;
        if (rw_fx == a.gw) { rw_fx = 0; ++rw_fy; }
      };
      if (BIAS == BIAS_SMEM && first_pass) bounded_wait(B_BIAS, 0);
      for (int u = 0; u < npass; ++u) {
        const int t = tile_at(u, p_stride);
        const uint32_t gs = g_s + (uint32_t)u, buf = gs % kSBufs;
        const uint32_t colP = kColS + buf * kN;  // P of this tile is written over its score buffer
        const int j0 = t * kN;
        // bias offsets of this tile's keys: per-head table, or computed by this warp
        const int* ko = koff_tab + j0;
        if (BIAS != BIAS_ROWS && wants_bias && warp_live && a.koff_mode == kKoffWarp) {
          int* wk = koff_tab + (warp * 2 + (int)(gs & 1u)) * kN;  // alternates across passes too
          if (j0 < a.prefix + kN) {
            patch_of(j0 + lane, ya, xa);
            patch_of(j0 + 32 + lane, yb, xb);
          } else {
            advance(ya, xa);
            advance(yb, xb);
          }
          wk[lane] = offset_of(j0 + lane, ya, xa);
          wk[lane + 32] = offset_of(j0 + 32 + lane, yb, xb);
          __syncwarp();
          ko = wk;
        }
        // BIAS_ROWS: the bias (or exp(bias)) of this thread's row and key 32 cc + u of
        // its chunk cc is brow[-(32 cc + u)]
        const float* brow = nullptr;
        if (BIAS == BIAS_ROWS && wants_bias && warp_live) {
          float* sl = rw_slice0 + (t & 1) * kRwEnt;  // last read two tiles ago
          if (t == 0) { rw_fy = 0; rw_fx = 0; rw_fetch(); }
#pragma unroll
          for (int i = 0; i < kRwEnt / 32; ++i) sl[32 * i + lane] = rwb[i];
          __syncwarp();
          if (t + 1 < ntiles) rw_fetch();  // tile t + 1, lands while this tile is processed
          brow = sl + lane + (kN - 1) - rw_first - (kSplit == 2 ? 32 * half : 0);
        }
        const bool ok_wait = __all_sync(0xffffffffu, bounded_wait(B_SFULL + buf, (gs / kSBufs) & 1));
        tc_fence_after();
        if (!warp_live) {
          tc_fence_before();
          mbar_arrive(&bars[B_TDONE + buf]);
          continue;
        }
        uint32_t r[32 * kChunks];
        if (kSplit == 2) {
          tmem_ld32(tl + kColS + buf * kN + 32 * half, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        } else {
          tmem_ld32(tl + kColS + buf * kN, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          tmem_ld32(tl + kColS + buf * kN + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * (kChunks - 1)]));
        }
        tmem_wait_ld();
        const int nvalid = row_ok ? max(0, min(kN, L - j0)) : 0;
        // Dense with bias: keys past L carry the k_invalid offset (weight 0), and
        // rows past L are never stored, so every tile takes the unmasked path.
        constexpr bool kMaskInKoff = kDense && HAS_BIAS && BIAS != BIAS_ROWS;
        const bool full_tile = kMaskInKoff || __all_sync(0xffffffffu, nvalid == kN);

        // bias offsets of keys 32*ch+u .. +3 of this tile
        auto koff4 = [&](int idx) -> int4 { return *reinterpret_cast<const int4*>(ko + idx); };

        // ---- P (or uint8 A) of one 32-key chunk into TMEM, or codes to global (export)
        auto emit = [&](const float (&e)[32], int ch) {
          const int jb = j0 + 32 * ch;
          if (kHasCodes || kQuant) {
            // uint8 codes floor(255 p + 0.5): every kept weight is at most the row's
            // normalizer, so e * (255 / normalizer) + 0.5 < 256 and no clamp is needed
            uint32_t wq[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              uint32_t q[4];
#pragma unroll
              for (int v = 0; v < 4; ++v) q[v] = __float2uint_rd(__fmaf_rn(e[4 * u + v], scale, 0.5f));
              wq[u] = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
            }
            if (kHasCodes) {
              if (row >= a.row_begin && row < a.row_end && row < a.n) {
                const int rows = a.row_end - a.row_begin;
                uint8_t* dst = a.codes + ((size_t)bh * rows + (row - a.row_begin)) * a.n;
#pragma unroll
                for (int u = 0; u < 32; ++u)
                  if (jb + u < a.n) dst[jb + u] = (uint8_t)((wq[u >> 2] >> (8 * (u & 3))) & 0xFFu);
              }
            } else {
              tmem_st8(tl + colP + 32 * ch, wq);
            }
          } else {
            uint32_t wp[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) wp[u] = pack_bf16x2(e[2 * u], e[2 * u + 1]);
            if (sum_in_pv) lsum += sum32(e);
            tmem_st16(tl + colP + 32 * ch, wp);
            if (VF32) {
              uint32_t wl[16];
#pragma unroll
              for (int u = 0; u < 16; ++u) {
                const float h0 = __uint_as_float(wp[u] << 16), h1 = __uint_as_float(wp[u] & 0xFFFF0000u);
                wl[u] = pack_bf16x2(e[2 * u] - h0, e[2 * u + 1] - h1);
              }
              tmem_st16(tl + colP + 32 * ch + 16, wl);
            }
          }
        };

        auto tile_body = [&](auto full_tag) {
          constexpr bool FULL = decltype(full_tag)::value;
#pragma unroll
          for (int cc = 0; cc < kChunks; ++cc) {
            const int ch = (kSplit == 2) ? half : cc;  // chunk of the tile; registers r[32 cc ...]
            const int jb = j0 + 32 * ch;
            if (jb >= L && pass != P_CODES) {
              // every key of the chunk lies past L: nothing to count or sum; P is 0
              if (pv) {
                if (kQuant) {
                  const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                  tmem_st8(tl + colP + 32 * ch, z);
                } else {
                  const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                  tmem_st16(tl + colP + 32 * ch, z);
                  if (VF32) tmem_st16(tl + colP + 32 * ch + 16, z);
                }
              }
              continue;
            }
            if (kHasLevels && pass == P_LEVELS) {
              const uint32_t base = hist_row + (uint32_t)(D / 2) * kM * 4u;  // level (d - s)/2: + (d - s) * 256 B
#pragma unroll
              for (int u = 0; u < 32; ++u) {
                const int sc = kF8 ? (int)__uint_as_float(r[32 * cc + u]) : (int)r[32 * cc + u];
                const uint32_t ad = base - (uint32_t)(sc * (kM * 2));
                if (FULL) {
                  asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(ad) : "memory");
                } else {
                  asm volatile(
                      "{\n\t.reg .pred p;\n\tsetp.lt.s32 p, %1, %2;\n\t@p red.shared.add.u32 [%0], 1;\n\t}" ::"r"(ad),
                      "r"(32 * ch + u), "r"(nvalid)
                      : "memory");
                }
              }
            } else if (kDense && lut_e) {
              float e[32];
#pragma unroll
              for (int u = 0; u < 32; u += 4) {
                float bw[4] = {1.0f, 1.0f, 1.0f, 1.0f};
                if (BIAS == BIAS_DGLOBAL && jb + u + 3 < L) {
                  // a dense matrix row: keys jb+u .. +3 in one aligned 16-byte load
                  const float4 w4 = __ldg(reinterpret_cast<const float4*>(eb_bytes) + ((jb + u) >> 2));
                  bw[0] = w4.x; bw[1] = w4.y; bw[2] = w4.z; bw[3] = w4.w;
                } else if (BIAS == BIAS_ROWS) {
#pragma unroll
                  for (int v = 0; v < 4; ++v) bw[v] = brow[-(32 * cc + u + v)];
                } else if (HAS_BIAS) {
                  const int4 k4 = koff4(32 * ch + u);
                  const int kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                  for (int v = 0; v < 4; ++v)
                    bw[v] = (BIAS == BIAS_SMEM) ? *reinterpret_cast<const float*>(eb_bytes - kk[v])
                                                : __ldg(reinterpret_cast<const float*>(eb_bytes - kk[v]));
                }
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                  const int sc = (int)r[32 * cc + u + v];
                  float x = lut_lane[-16 * sc];  // level (64 - s) / 2 of this lane's table
                  if (HAS_BIAS) x *= bw[v];
                  e[u + v] = (FULL || 32 * ch + u + v < nvalid) ? x : 0.0f;
                }
              }
              if (pass == P_NORM) {
                lsum += sum32(e);
              } else {
                emit(e, ch);
              }
            } else if (SEL == SEL_TOPN_INT && lut_w) {
              float e[32];
#pragma unroll
              for (int u = 0; u < 32; ++u) {
                const int sc = (int)r[32 * cc + u];
                const float w = *reinterpret_cast<const float*>(wrow - sc * (2 * kM));
                const bool valid = FULL || 32 * ch + u < nvalid;
                const bool eq = valid && sc == sF;
                const bool drop_tie = eq && cut && tie_seen >= rF;
                tie_seen += eq ? 1 : 0;
                e[u] = (valid && !drop_tie) ? w : 0.0f;
              }
              emit(e, ch);
            } else if (kHasRadix && BIAS == BIAS_ROWS && !kRef && pass == P_FBIN) {
              // FBIN with the staged bias: per pair of keys the logits (a packed fp32x2 FMA,
              // each element rounded once as fmaf), the saturating bin map and two counts.
              // The bias is read first, so that the histogram adds wait on no load.
              if (r_state == 4) {
#pragma unroll
                for (int g = 0; g < 32; g += kFbGroup) {
                float bv[kFbGroup];
#pragma unroll
                for (int u = 0; u < kFbGroup; ++u) bv[u] = brow[-(32 * cc + g + u)];
#pragma unroll
                for (int u = g; u < g + kFbGroup; u += 2) {
                  const float2 sf2 = make_float2(score_f(r[32 * cc + u]), score_f(r[32 * cc + u + 1]));
                  const float2 l2 = __ffma2_rn(sf2, make_float2(c, c), make_float2(bv[u - g], bv[u - g + 1]));
                  const float la = (FULL || 32 * ch + u < nvalid) ? l2.x : -INFINITY;
                  const float lb = (FULL || 32 * ch + u + 1 < nvalid) ? l2.y : -INFINITY;
                  const float2 w2 = __ffma2_rn(make_float2(fma_sat(la, fb_sc, fb_off), fma_sat(lb, fb_sc, fb_off)),
                                               make_float2(kFbSpan, kFbSpan), make_float2(kFbMg, kFbMg));
                  asm volatile("red.shared.add.u32 [%0], 1;" ::"r"((__float_as_uint(w2.x) & 0xFE00u) + hist_row)
                               : "memory");
                  asm volatile("red.shared.add.u32 [%0], 1;" ::"r"((__float_as_uint(w2.y) & 0xFE00u) + hist_row)
                               : "memory");
                }
                }
              }
            } else {
              // generic path: exact logits (invalid keys -inf)
              float lg[32];
              uint32_t kinv = 0;  // keys past L (dense with bias: the sentinel, not the tile mask)
              if (BIAS == BIAS_ROWS && !kRef) {
                // staged bias: two logits per packed fp32x2 FMA (each element rounded once,
                // as fmaf)
#pragma unroll
                for (int u = 0; u < 32; u += 2) {
                  const float2 sf2 = make_float2(score_f(r[32 * cc + u]), score_f(r[32 * cc + u + 1]));
                  const float2 b2 = make_float2(brow[-(32 * cc + u)], brow[-(32 * cc + u + 1)]);
                  const float2 l2 = __ffma2_rn(sf2, make_float2(c, c), b2);
                  lg[u] = (FULL || 32 * ch + u < nvalid) ? l2.x : -INFINITY;
                  lg[u + 1] = (FULL || 32 * ch + u + 1 < nvalid) ? l2.y : -INFINITY;
                }
              } else {
#pragma unroll
              for (int u = 0; u < 32; u += 4) {
                int4 k4 = make_int4(0, 0, 0, 0);
                if (HAS_BIAS && BIAS != BIAS_ROWS) k4 = koff4(32 * ch + u);
                const int kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                  const int sc = (int)r[32 * cc + u + v];
                  // the score as a float: the integer count, or the comparison mode's fp32 dot product
                  const float sf = (kRef || kF8) ? __uint_as_float(r[32 * cc + u + v]) : (float)sc;
                  float l;
                  if (HAS_BIAS) {
                    if (kMaskInKoff) kinv |= (kk[v] == 4 * a.k_invalid ? 1u : 0u) << (u + v);
                    const float bv = (BIAS == BIAS_ROWS) ? brow[-(32 * cc + u + v)]
                                                         : __ldg(reinterpret_cast<const float*>(tab_bytes - kk[v]));
                    l = __fmaf_rn(sf, c, bv);
                  } else {
                    l = sf * c;
                  }
                  lg[u + v] = (FULL || 32 * ch + u + v < nvalid) ? l : -INFINITY;
                }
              }
              }
              if (kHasNorm && pass == P_NORM) {
                float tm = -INFINITY;
#pragma unroll
                for (int u = 0; u < 32; ++u) tm = fmaxf(tm, lg[u]);
                if (tm > m) {
                  lsum *= fast_exp2((m - tm) * kLog2e);
                  m = tm;
                }
                const float mo2 = -m * kLog2e;
                float ex[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) ex[u] = fast_exp2(__fmaf_rn(lg[u], kLog2e, mo2));
                lsum += sum32(ex);
              } else if (kHasRadix && pass == P_FBIN) {
                // bins of the row's logits: w = fmaf(sat(fmaf(l, sc, off)), 65535, kFbMg) is
                // monotone in l; bin b at word b of the row's column.  Every key is counted
                // (no branch): keys below the window land in bin 0, which is never read,
                // keys past L (l = -inf) too
                if (r_state == 4) {
#pragma unroll
                  for (int u = 0; u < 32; u += 2) {
                    const float2 w2 = __ffma2_rn(make_float2(fma_sat(lg[u], fb_sc, fb_off), fma_sat(lg[u + 1], fb_sc, fb_off)),
                                                 make_float2(kFbSpan, kFbSpan), make_float2(kFbMg, kFbMg));
                    asm volatile("red.shared.add.u32 [%0], 1;" ::"r"((__float_as_uint(w2.x) & 0xFE00u) + hist_row)
                                 : "memory");
                    asm volatile("red.shared.add.u32 [%0], 1;" ::"r"((__float_as_uint(w2.y) & 0xFE00u) + hist_row)
                                 : "memory");
                  }
                }
              } else if (kHasRadix && pass == P_RADIX) {
                // histogram of the keys inside the window [r_uhi - r_span, r_uhi] (order keys;
                // keys past L are -inf, below every window), and the count above it
                // (bin b: the low (b < 128) or high half of word b mod 128)
                if (r_state == 1) {
                  const uint32_t ulo = r_uhi - r_span;
#pragma unroll
                  for (int u = 0; u < 32; ++u) {
                    const uint32_t key = float_order_key(lg[u]);
                    const uint32_t t = key - ulo, bin = (r_span - t) >> r_shift;
                    r_above += key > r_uhi ? 1 : 0;
                    const uint32_t ad = hist_row + (bin & 127u) * (uint32_t)(kM * 4);
                    const uint32_t inc = 1u + (bin >> 7) * 0xFFFFu;
                    asm volatile(
                        "{\n\t.reg .pred p;\n\tsetp.le.u32 p, %1, %2;\n\t@p red.shared.add.u32 [%0], %3;\n\t}" ::"r"(ad),
                        "r"(t), "r"(r_span), "r"(inc)
                        : "memory");
                  }
                }
              } else if (kHasRadix && pass == P_COLLECT) {
                // the order keys inside the window, one column per row: [kCandCap][128 rows]
                // (the slot wraps, so a miscount stays in bounds and is reported after the pass)
                if (r_state == 2 && kSplitF) {
                  // two threads per row: slots from the row's shared counter
                  const uint32_t ulo = r_uhi - r_span;
#pragma unroll
                  for (int u = 0; u < 32; ++u) {
                    const uint32_t key = float_order_key(lg[u]);
                    if (key - ulo <= r_span) {
                      const int slot = atomicAdd(reinterpret_cast<int*>(xchg) + srow, 1);
                      hist[(slot & (kCandCap - 1)) * kM + srow] = key;
                    }
                  }
                } else if (r_state == 2) {
                  const uint32_t ulo = r_uhi - r_span;
#pragma unroll
                  for (int u = 0; u < 32; ++u) {
                    const uint32_t key = float_order_key(lg[u]);
                    const uint32_t t = key - ulo;
                    const uint32_t ad = hist_row + (uint32_t)(r_cnt & (kCandCap - 1)) * (uint32_t)(kM * 4);
                    asm volatile(
                        "{\n\t.reg .pred p;\n\tsetp.le.u32 p, %1, %2;\n\t@p st.shared.u32 [%0], %3;\n\t}" ::"r"(ad),
                        "r"(t), "r"(r_span), "r"(key)
                        : "memory");
                    r_cnt += t <= r_span ? 1 : 0;
                  }
                }
              } else if (SEL == SEL_TOPN_FLOAT && (pass == P_PV || pass == P_CODES)) {
                // weights of the keys at or above w_cut (keys past L are -inf, below it);
                // the keys in [w_lo, w_hi] are the ties at F, of which those past the
                // row's remaining allowance rF are dropped in key order, or (folded
                // collect) the final radix bin, whose key indices are recorded
                float e[32];
                uint32_t inm = 0u;
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                  const float x = fast_exp2(__fmaf_rn(lg[u], kLog2e, mo));
                  e[u] = lg[u] >= w_cut ? x : 0.0f;
                  inm |= (lg[u] >= w_lo && lg[u] <= w_hi ? 1u : 0u) << u;
                }
                if (kMerge && r_state == 3) {
                  while (inm) {
                    const int u = __ffs(inm) - 1;
                    inm &= inm - 1u;
                    hist[(r_cnt & (kCap - 1)) * kM + srow] = (uint32_t)(jb + u);
                    ++r_cnt;
                  }
                } else {
                  const uint32_t dropm = inm & ~tie_keep(inm, cut, rF, tie_seen);
                  tie_seen += __popc(inm);
                  if (dropm) {
#pragma unroll
                    for (int u = 0; u < 32; ++u) e[u] = ((dropm >> u) & 1u) ? 0.0f : e[u];
                  }
                }
                emit(e, ch);
              } else {
                // keep mask in key order; ties at F counted per row
                uint32_t keepm = 0;
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                  const bool valid = FULL || 32 * ch + u < nvalid;
                  bool k;
                  if (kDense) {
                    k = valid && !((kinv >> u) & 1u);
                  } else {
                    const bool gt = valid && lg[u] > F, eq = valid && lg[u] == F;
                    k = gt || (eq && (!cut || tie_seen < rF));
                    tie_seen += eq ? 1 : 0;
                  }
                  keepm |= (k ? 1u : 0u) << u;
                }
                if (kHasKeptNorm && pass == P_KEPT_NORM) {
                  float ex[32];
#pragma unroll
                  for (int u = 0; u < 32; ++u)
                    ex[u] = ((keepm >> u) & 1u) ? fast_exp2(__fmaf_rn(lg[u], kLog2e, mo)) : 0.0f;
                  lsum += sum32(ex);
                } else if (kHasIdx && pass == P_IDX) {
                  if (row_ok) {
                    int32_t* dst = a.idx + ((size_t)bh * a.n + row) * a.N;
                    if (kDense) {
                      // dense: every key below L is kept, so key j is the j-th kept index
#pragma unroll
                      for (int u = 0; u < 32; ++u)
                        if ((keepm >> u) & 1u) dst[jb + u] = jb + u;
                    } else {
#pragma unroll
                      for (int u = 0; u < 32; ++u)
                        if ((keepm >> u) & 1u) { if (kept_seen < a.N) dst[kept_seen] = jb + u; ++kept_seen; }
                    }
                  }
                } else if (kHasPv || kHasCodes) {
                  float e[32];
#pragma unroll
                  for (int u = 0; u < 32; ++u) {
                    const float x = fast_exp2(__fmaf_rn(lg[u], kLog2e, mo));
                    e[u] = ((keepm >> u) & 1u) ? x : 0.0f;
                  }
                  emit(e, ch);
                }
              }
            }
          }
        };
        if (EXPORT == EXP_SCORES) {
          // the integer scores of this tile as the score MMA left them in TMEM
          if (ok_wait && row < a.n) {
            int32_t* dst = a.scores + ((size_t)bh * a.n + row) * a.n;
#pragma unroll
            for (int u = 0; u < kN; ++u)
              if (j0 + u < a.n) dst[j0 + u] = (row_ok && j0 + u < L) ? (int32_t)r[u] : 0;
          }
        } else if (kSplitF && pv) {
          // top-N with a bias, P.V with two threads per row: this thread's 32 keys.  Keys at
          // or above w_cut are weighted; keys in [w_lo, w_hi] are the final bin (recorded
          // in shared slots, ranked after the pass) or, for a row resolved by a collect
          // pass, the ties at F, kept in key order: the two threads exchange their tie
          // counts every tile (both warps of the pair reach the barrier, whatever
          // happened to their waits)
          const int jb = j0 + 32 * half;
          const int nv = nvalid - 32 * half;  // valid keys of this chunk (<= 0: none)
          float e[32];
          uint32_t inm = 0u;
          // weights and final-bin mask of this thread's 32 keys (FULL: no key past L)
          auto pv_chunk = [&](auto full_tag) {
            constexpr bool FULL = decltype(full_tag)::value;
            const float mo_p = -m * kLog2e;
#pragma unroll
            for (int u = 0; u < 32; u += 2) {
              float2 b2;
              if (BIAS == BIAS_ROWS) {
                b2 = make_float2(brow[-u], brow[-(u + 1)]);
              } else {
                b2 = make_float2(__ldg(reinterpret_cast<const float*>(tab_bytes - ko[32 * half + u])),
                                 __ldg(reinterpret_cast<const float*>(tab_bytes - ko[32 * half + u + 1])));
              }
              // logits and exp arguments two at a time (packed fp32x2 FMAs, each rounded once)
              const float2 l2 = __ffma2_rn(make_float2(score_f(r[u]), score_f(r[u + 1])), make_float2(c, c), b2);
              const float la = (FULL || u < nv) ? l2.x : -INFINITY, lb = (FULL || u + 1 < nv) ? l2.y : -INFINITY;
              const float2 x2 = __ffma2_rn(make_float2(la, lb), make_float2(kLog2e, kLog2e), make_float2(mo_p, mo_p));
              const float xa = fast_exp2(x2.x), xb = fast_exp2(x2.y);
              e[u] = la >= w_cut ? xa : 0.0f;
              e[u + 1] = lb >= w_cut ? xb : 0.0f;
              inm |= (la >= w_lo && la <= w_hi ? 1u : 0u) << u;
              inm |= (lb >= w_lo && lb <= w_hi ? 1u : 0u) << (u + 1);
            }
          };
          // bf16 V: P goes straight into packed words with a running sum (no weight array
          // held across the tie exchange).  Keys at or above pv_cut are weighted, keys in
          // [w_lo, pv_cut) go to the mask: the final bin of a merge row, or a row's ties
          // at F (pv_cut just above F), which are weighted in a second computation of the
          // chunk if the tie rule keeps them (rare: the chunk that holds the threshold)
          uint32_t wp[16];
          float cs = 0.0f;
          auto pv_words = [&](auto full_tag, auto add_tag, uint32_t add) {
            constexpr bool FULL = decltype(full_tag)::value;
            constexpr bool ADD = decltype(add_tag)::value;  // also weight the keys of `add` (kept ties)
            const float mo_p = -m * kLog2e;
            cs = 0.0f;
            float cs1 = 0.0f;
#pragma unroll
            for (int u = 0; u < 32; u += 2) {
              float2 b2;
              if (BIAS == BIAS_ROWS) {
                b2 = make_float2(brow[-u], brow[-(u + 1)]);
              } else {
                b2 = make_float2(__ldg(reinterpret_cast<const float*>(tab_bytes - ko[32 * half + u])),
                                 __ldg(reinterpret_cast<const float*>(tab_bytes - ko[32 * half + u + 1])));
              }
              const float2 l2 = __ffma2_rn(make_float2(score_f(r[u]), score_f(r[u + 1])), make_float2(c, c), b2);
              const float la = (FULL || u < nv) ? l2.x : -INFINITY, lb = (FULL || u + 1 < nv) ? l2.y : -INFINITY;
              const float2 x2 = __ffma2_rn(make_float2(la, lb), make_float2(kLog2e, kLog2e), make_float2(mo_p, mo_p));
              const bool ga = la >= pv_cut, gb = lb >= pv_cut;
              const bool ka = ga || (ADD && ((add >> u) & 1u)), kb = gb || (ADD && ((add >> (u + 1)) & 1u));
              const float ea = ka ? fast_exp2(x2.x) : 0.0f, eb = kb ? fast_exp2(x2.y) : 0.0f;
              wp[u >> 1] = pack_bf16x2(ea, eb);
              cs += ea;
              cs1 += eb;
              if (!ADD) {
                inm |= (la >= w_lo && !ga ? 1u : 0u) << u;
                inm |= (lb >= w_lo && !gb ? 1u : 0u) << (u + 1);
              }
            }
            cs += cs1;
          };
          if (ok_wait && jb < L) {
            if (VF32) {
              if (full_tile) pv_chunk(std::true_type{});
              else pv_chunk(std::false_type{});
            } else {
              if (full_tile) pv_words(std::true_type{}, std::false_type{}, 0u);
              else pv_words(std::false_type{}, std::false_type{}, 0u);
            }
          } else if (VF32) {
#pragma unroll
            for (int u = 0; u < 32; ++u) e[u] = 0.0f;
          } else {
#pragma unroll
            for (int u = 0; u < 16; ++u) wp[u] = 0u;
          }
          uint32_t eqm = 0u;
          if (r_state == 3) {
            while (inm) {
              const int u = __ffs(inm) - 1;
              inm &= inm - 1u;
              const int slot = atomicAdd(reinterpret_cast<int*>(xchg) + srow, 1);
              hist[(slot & (kCap - 1)) * kM + srow] = (uint32_t)(jb + u);
            }
          } else {
            eqm = inm;
          }
          // the row's tie counts of this tile, from both threads (only when some row of
          // the CTA cuts its ties at F; the flag is the same for every thread)
          int c0 = 0, c1 = 0;
          if (pv_xchg) {
            int* tx = reinterpret_cast<int*>(hist) + (kCandCap - 8) * kM + (int)(gs & 1u) * 2 * kM;
            tx[half * kM + srow] = __popc(eqm);
            asm volatile("bar.sync %0, 64;" ::"r"(1 + (warp & 3)) : "memory");
            c0 = tx[srow];
            c1 = tx[kM + srow];
          }
          const uint32_t keep_t = tie_keep(eqm, cut, rF, tie_seen + (half ? c0 : 0));
          const uint32_t dropm = eqm & ~keep_t;
          if (!VF32 && (eqm & keep_t) && ok_wait && jb < L) {  // the chunk again, with its kept ties
            if (full_tile) pv_words(std::true_type{}, std::true_type{}, eqm & keep_t);
            else pv_words(std::false_type{}, std::true_type{}, eqm & keep_t);
          }
          if (VF32) {
#pragma unroll
            for (int u = 0; u < 32; ++u) e[u] = ((dropm >> u) & 1u) ? 0.0f : e[u];
          }
          tie_seen += c0 + c1;
          if (ok_wait) {
            if (jb >= L) {
              const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
              tmem_st16(tl + colP + 32 * half, z);
              if (VF32) tmem_st16(tl + colP + 32 * half + 16, z);
            } else if (VF32) {
              emit(e, half);
            } else {
              lsum += cs;
              tmem_st16(tl + colP + 32 * half, wp);
            }
          }
        } else if (kSplit == 2 && SEL == SEL_TOPN_INT && pv) {
          // top-N P.V with two threads per row: weights of this thread's chunk, then
          // the row's two threshold-tie counts of this tile are exchanged (every live
          // warp pair reaches the barrier, whatever happened to its waits)
          const int jb = j0 + 32 * half;
          const int nv = nvalid - 32 * half;  // valid keys of this chunk (<= 0: none)
          float e[32];
          uint32_t eqm = 0u;
          if (ok_wait && jb < L) {
            if (lut_w) {
#pragma unroll
              for (int u = 0; u < 32; ++u) {
                const int sc = (int)r[u];
                const bool valid = u < nv;
                e[u] = valid ? *reinterpret_cast<const float*>(wrow - sc * (2 * kM)) : 0.0f;
                eqm |= (valid && sc == sF) ? (1u << u) : 0u;
              }
            } else {
#pragma unroll
              for (int u = 0; u < 32; ++u) {
                const float l = (float)(int)r[u] * c;
                const bool valid = u < nv;
                e[u] = (valid && l >= F) ? fast_exp2(__fmaf_rn(l, kLog2e, mo)) : 0.0f;
                eqm |= (valid && l == F) ? (1u << u) : 0u;
              }
            }
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) e[u] = 0.0f;
          }
          int* tx = reinterpret_cast<int*>(xchg) + 6 * kM + (int)(gs & 1u) * 2 * kM;
          tx[half * kM + srow] = __popc(eqm);
          asm volatile("bar.sync %0, 64;" ::"r"(1 + (warp & 3)) : "memory");
          const int c0 = tx[srow], c1 = tx[kM + srow];
          const uint32_t dropm = eqm & ~tie_keep(eqm, cut, rF, tie_seen + (half ? c0 : 0));
          if (dropm) {
#pragma unroll
            for (int u = 0; u < 32; ++u) e[u] = ((dropm >> u) & 1u) ? 0.0f : e[u];
          }
          tie_seen += c0 + c1;
          if (ok_wait) {
            if (jb >= L) {
              if (kQuant) {
                const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                tmem_st8(tl + colP + 32 * half, z);
              } else {
                const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                tmem_st16(tl + colP + 32 * half, z);
                if (VF32) tmem_st16(tl + colP + 32 * half + 16, z);
              }
            } else {
              emit(e, half);
            }
          }
        } else if (ok_wait) {
          if (full_tile) tile_body(std::true_type{});
          else tile_body(std::false_type{});
        }
        if (pv) tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[B_TDONE + buf]);
      }
      g_k += npass;
      g_s += npass;
      if (pv) g_v += ntiles;
    }

    // ============================================================== per-row decisions after the pass
    // two threads per top-N row: both have finished adding to the row's level
    // histogram before the first reads it (and overwrites it with the weight table)
    if (kSplit == 2 && SEL == SEL_TOPN_INT && pass == P_LEVELS) __syncthreads();
    if (kSplitF && pass == P_RADIX) {
      // the row's two threads sum their counts of keys above the first radix window
      int* ra = reinterpret_cast<int*>(xchg) + kM;
      if (is_soft && half == 1) ra[srow] = r_above;
      __syncthreads();
      const int other = (is_soft && half == 0) ? ra[srow] : 0;
      __syncthreads();
      if (is_soft && half == 0) {
        r_above += other;
        ra[srow] = r_above;
      }
      __syncthreads();
      if (is_soft && half == 1) r_above = ra[srow];
    }
    // both threads of a row have finished adding to its histogram (or candidate list)
    if (kSplitF) __syncthreads();
    if (kSplit == 2 && pass == P_NORM) {
      // the row's two threads combine their partial normalizers (and running maxima)
      if (is_soft && half == 1) { xchg[srow] = lsum; xchg[kM + srow] = m; }
      __syncthreads();
      if (is_soft && half == 0) {
        const float l1 = xchg[srow], m1 = xchg[kM + srow];
        if (use_lut) {
          lsum += l1;
        } else {
          const float mm = fmaxf(m, m1);
          if (mm != -INFINITY)
            lsum = lsum * fast_exp2((m - mm) * kLog2e) + l1 * fast_exp2((m1 - mm) * kLog2e);
          m = mm;
        }
      }
    }
    if ((tid < kM || (kSplitF && is_soft)) && row_ok && !*abort_flag) {
      if (pass == P_LEVELS) {
        // the row's level counts, level (d - s) / 2: in registers at d = 64, read from
        // shared memory at d = 128 (129 of them)
        constexpr int kCached = kLevels <= 65 ? kLevels : 1;
        int cached[kCached];
#pragma unroll
        for (int lev = 0; lev < kCached; ++lev) cached[lev] = kCached == kLevels ? (int)hist[lev * kM + srow] : 0;
        auto cnt = [&](int lev) -> int { return kCached == kLevels ? cached[lev] : (int)hist[lev * kM + srow]; };
        int hmin = D, hN = D, cum = 0;
        bool found = false;
#pragma unroll
        for (int lev = kLevels - 1; lev >= 0; --lev) hmin = cnt(lev) > 0 ? lev : hmin;
#pragma unroll
        for (int lev = 0; lev < kLevels; ++lev) {
          cum += cnt(lev);
          if (!found && cum >= keff) { hN = lev; found = true; }
        }
        const int smax = D - 2 * hmin, sN = D - 2 * hN;
        if (SEL == SEL_TOPN_INT) {
          F = (float)sN * c;
          m = (float)smax * c;
          int gt = 0, eq = 0;
          float ls = 0.0f;
#pragma unroll
          for (int lev = 0; lev < kLevels; ++lev) {
            const float lv = (float)(D - 2 * lev) * c;
            const int k = cnt(lev);
            gt += (lv > F) ? k : 0;
            eq += (lv == F) ? k : 0;
            ls += (lv > F) ? (float)k * fast_exp2((lv - m) * kLog2e) : 0.0f;
          }
          rF = keff - gt;
          cut = rF < eq ? 1 : 0;
          ls += (float)rF * fast_exp2((F - m) * kLog2e);
          scale = (kQuant || EXPORT == EXP_CODES) ? 255.0f / ls : 1.0f / ls;
          sF = sN;
          // this row's weight per level: exp(l - m) above the threshold, the tie weight at it, 0 below
          float* wt = reinterpret_cast<float*>(hist);
#pragma unroll
          for (int lev = 0; lev < kLevels; ++lev) {
            const float lv = (float)(D - 2 * lev) * c;
            wt[lev * kM + srow] = (lv >= F) ? fast_exp2((lv - m) * kLog2e) : 0.0f;
          }
        } else {
          // the threshold lies in [sN c + b_min, sN c + b_max]: at least keff keys have a
          // score >= sN (so a logit >= the low end), fewer than keff a score > sN (only
          // those can exceed the high end); logits are monotone in (score, bias)
          const float bmin = a.bminmax[2 * h], bmax = a.bminmax[2 * h + 1];
          int s_lo = sN, s_hi = sN;
          if (p_stride != 1) {
            // a sample of ns keys: rank keff of the row maps to about rho in the sample.
            // s_hi: fewer than rho - del sampled keys score above it, so (likely) fewer
            // than keff keys do; s_lo: at least rho + del sampled keys reach it, so (likely)
            // keff keys do.  The FBIN pass checks both with exact counts.
            const int last = tile_at(n_sampled - 1, kSampleStride);
            const int ns = n_sampled * kN - (last == ntiles - 1 ? ntiles * kN - L : 0);
            const float rho = (float)keff * (float)ns / (float)L;
            const float del = 5.0f * sqrtf(rho * (1.0f - (float)keff / (float)L)) + 2.0f;
            const int k_hi = max(1, (int)floorf(rho - del)), k_lo = (int)ceilf(rho + del);
            int lhi = kLevels - 1, llo = kLevels - 1, cs = 0;
            bool fh = false, fl = false;
#pragma unroll
            for (int lev = 0; lev < kLevels; ++lev) {
              cs += cnt(lev);
              if (!fh && cs >= k_hi) { lhi = lev; fh = true; }
              if (!fl && cs >= k_lo) { llo = lev; fl = true; }
            }
            s_hi = D - 2 * lhi;
            s_lo = D - 2 * llo;  // the lowest level when the sample never reaches k_lo
          }
          const float lo = __fmaf_rn((float)s_lo, c, bmin);
          const float hw = __fmaf_rn((float)s_hi, c, bmax);
          r_rank = keff;
          r_sampled = p_stride != 1;
          // no logit exceeds m (with a sample: none by more than 2 d c, which the
          // sampling condition keeps inside fp32)
          m = __fmaf_rn((float)smax, c, bmax);
          // FBIN map: lo -> about u = 768 / 65535 (w in bin 1), hw -> about 64768 / 65535
          // (bin 126); the rounding of sc and off moves both by far less than a bin
          // (1 / 128 of u) while |lo * sc| < 2048, else the order-key radix takes the window
          const float sc_b = (125.0f * 512.0f / kFbSpan) / (hw - lo);
          const float lsc = lo * sc_b;
          if (hw > lo && isfinite(sc_b) && fabsf(lsc) < 2048.0f) {
            fb_sc = sc_b;
            fb_off = 768.0f / kFbSpan - lsc;
            r_state = 4;
          } else if (p_stride != 1) {
            r_state = 5;  // the radix window cannot check a sampled bracket: count every tile
          } else {
            r_uhi = float_order_key(hw);
            r_span = r_uhi - float_order_key(lo);
            r_shift = 0;
            while ((r_span >> r_shift) >= (uint32_t)kRadixBins) ++r_shift;
            r_first = true;
            r_state = 1;
          }
        }
      } else if (pass == P_FBIN && r_state == 4) {
        // the bin holding rank r_rank, counted from the top (bin 127: keys above the
        // window, fewer than r_rank of them; bin 0 is never reached: at least r_rank
        // keys reach the window's low end)
        int cum = 0, bsel = 0, kbin = 0;
        for (int b0 = 127; b0 >= 1 && bsel == 0; b0 -= 8) {  // eight counts in flight
          int kk[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) kk[j] = b0 - j >= 1 ? (int)hist[(b0 - j) * kM + srow] : 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (bsel != 0 || b0 - j < 1) continue;
            if (cum + kk[j] >= r_rank) { bsel = b0 - j; kbin = kk[j]; }
            else cum += kk[j];
          }
        }
        // a sampled bracket that missed: rank r_rank above the window (bin 127) or
        // below it (bin 0).  A bracket from every tile's levels cannot miss; should
        // rounding ever make it, the radix passes take the whole float range.
        if ((bsel == 0 || bsel == 127) && r_sampled) {
          r_state = 5;
        } else if (bsel == 0 || bsel == 127) {
          r_uhi = float_order_key(INFINITY);
          r_span = r_uhi - float_order_key(-INFINITY);
          r_shift = 0;
          while ((r_span >> r_shift) >= (uint32_t)kRadixBins) ++r_shift;
          r_first = true;
          r_state = 1;
        } else {
        // the bin's keys are the logits in [w_lo, w_cut): the least floats that map to
        // bins bsel and bsel + 1, found by bisection over the order keys of floats,
        // from 128 keys around the map's inverse when the map confirms that bracket
        auto fb_bin = [&](float x) -> int {
          const float w = __fmaf_rn(fma_sat(x, fb_sc, fb_off), kFbSpan, kFbMg);
          return (int)((__float_as_uint(w) & 0xFE00u) >> 9);
        };
        auto fb_least = [&](int bin) -> float {
          uint32_t klo = 0x007FFFFFu, khi = 0xFF800000u;  // -inf (bin 0), +inf (bin 127)
          const float est = ((512.0f * (float)bin - 0.5f) / kFbSpan - fb_off) / fb_sc;
          if (isfinite(est)) {
            const uint32_t ke = float_order_key(est);
            const uint32_t ka = ke - 64u, kb = ke + 64u;
            if (ka > klo && ka < ke && kb < khi && kb > ke && fb_bin(order_key_float(ka)) < bin &&
                fb_bin(order_key_float(kb)) >= bin) {
              klo = ka;
              khi = kb;
            }
          }
          while (khi - klo > 1u) {
            const uint32_t mid = klo + ((khi - klo) >> 1);
            if (fb_bin(order_key_float(mid)) >= bin) khi = mid;
            else klo = mid;
          }
          return order_key_float(khi);
        };
        w_lo = fb_least(bsel);
        w_cut = bsel >= 127 ? INFINITY : fb_least(bsel + 1);
        // the largest float below w_cut (no logit is -0, so below +0 means negative)
        w_hi = (w_cut == 0.0f) ? -1.4e-45f : order_key_float(float_order_key(w_cut) - 1u);
        r_rank -= cum;
        r_cnt = 0;
        if (kMerge && kbin <= kCap) {
          r_state = 3;
        } else {
          r_uhi = float_order_key(w_hi);
          r_span = r_uhi - float_order_key(w_lo);
          r_first = false;
          if (kbin <= kCandCap) {
            r_state = 2;
          } else {
            r_shift = 0;
            while ((r_span >> r_shift) >= (uint32_t)kRadixBins) ++r_shift;
            r_state = 1;
          }
        }
        }
      } else if (pass == P_RADIX && r_state == 1) {
        if (r_first) r_rank -= r_above;  // rank within the first window
        r_first = false;
        int cum = 0, bsel = kRadixBins - 1, kbin = 0;
        for (int bb = 0; bb < kRadixBins; ++bb) {
          const int k = (int)((hist[(bb & 127) * kM + srow] >> ((bb >> 7) * 16)) & 0xFFFFu);
          if (cum + k >= r_rank) { bsel = bb; kbin = k; break; }
          cum += k;
        }
        const int rank = r_rank - cum;
        const uint32_t uhi = r_uhi - ((uint32_t)bsel << r_shift);
        if (r_shift == 0) {
          F = order_key_float(uhi);
          rF = rank;
          cut = rank < kbin ? 1 : 0;
          r_state = 0;
          w_lo = w_hi = w_cut = F;
        } else {
          // the chosen bin becomes the window: collected if small, else binned again
          const uint32_t span_left = r_span - ((uint32_t)bsel << r_shift);
          r_uhi = uhi;
          r_span = min(((uint32_t)1 << r_shift) - 1u, span_left);
          r_rank = rank;
          r_cnt = 0;
          if (kMerge && kbin <= kCap) {
            r_state = 3;
            // no logit has the order key of -0 (keys are taken of l + 0): keep the
            // window's ends off it so that their float values compare as the keys do
            if (r_uhi == 0x7FFFFFFFu) { r_uhi -= 1u; r_span -= 1u; }
            if (r_uhi - r_span == 0x7FFFFFFFu) r_span -= 1u;
            w_hi = order_key_float(r_uhi);
            w_lo = order_key_float(r_uhi - r_span);
            w_cut = order_key_float(r_uhi + 1u);  // the next float above w_hi
          } else if (kbin <= kCandCap) {
            r_state = 2;
          } else {
            r_shift = r_shift > 8 ? r_shift - 8 : 0;
          }
        }
      } else if (pass == P_COLLECT && r_state == 2) {
        // the r_rank-th largest collected key: the one with fewer than r_rank keys
        // above it and at least r_rank at or above it
        const uint32_t* cand = hist;
        if (kSplitF) r_cnt = reinterpret_cast<const int*>(xchg)[srow];  // the row's shared counter
        const int nc = min(r_cnt, kCandCap);
        if (r_cnt > kCandCap) raise_status(a.status, kDevErrCapacity);
        uint32_t uF = 0u;
        int gt = 0, eq = 0;
        for (int x = 0; x < nc; ++x) {
          const uint32_t kx = cand[x * kM + srow];
          int g = 0, e = 0;
          for (int y = 0; y < nc; ++y) {
            const uint32_t ky = cand[y * kM + srow];
            g += ky > kx ? 1 : 0;
            e += ky == kx ? 1 : 0;
          }
          if (g < r_rank && r_rank <= g + e) {
            uF = kx;
            gt = g;
            eq = e;
            break;
          }
        }
        F = order_key_float(uF);
        rF = r_rank - gt;
        cut = rF < eq ? 1 : 0;
        r_state = 0;
        w_lo = w_hi = w_cut = F;
      } else if (pass == P_KEPT_NORM) {
        scale = 255.0f / lsum;
      } else if (pass == P_NORM) {
        scale = (kQuant || EXPORT == EXP_CODES) ? 255.0f / lsum : 1.0f / lsum;
      }
    }
    if (kSplit == 2 && SEL == SEL_TOPN_INT && pass == P_LEVELS) {
      // the row's threshold state (and its weight table, written above) to the second thread
      __syncthreads();
      if (is_soft && half == 0) {
        xchg[srow] = F; xchg[kM + srow] = m; xchg[2 * kM + srow] = scale;
        xchg[3 * kM + srow] = __int_as_float(sF); xchg[4 * kM + srow] = __int_as_float(rF);
        xchg[5 * kM + srow] = __int_as_float(cut);
      }
      __syncthreads();
      if (is_soft && half == 1) {
        F = xchg[srow]; m = xchg[kM + srow]; scale = xchg[2 * kM + srow];
        sF = __float_as_int(xchg[3 * kM + srow]); rF = __float_as_int(xchg[4 * kM + srow]);
        cut = __float_as_int(xchg[5 * kM + srow]);
      }
    }
    if (kSplit == 2 && pass == P_NORM) {
      __syncthreads();
      if (is_soft && half == 0) { xchg[srow] = scale; xchg[kM + srow] = m; }
      __syncthreads();
      if (is_soft && half == 1) { scale = xchg[srow]; m = xchg[kM + srow]; }
    }
    tie_seen = 0;
    // ---- the CTA chooses the next pass
    // Every thread takes the same next pass: the abort flag is voted on (a thread that
    // gave up a wait in this pass set it before reaching the vote), and the CTA-wide
    // votes on the row states run only where the select kind has the passes they
    // choose between.
    const int aborted = __syncthreads_or(*abort_flag != 0u);
    constexpr bool kVotes = SEL == SEL_TOPN_FLOAT;
    const int any_relevel = kVotes && __syncthreads_or(tid < kM && r_state == 5);
    if (kSplitF) pv_xchg = VF32 || __syncthreads_or(is_soft && row_ok && cut && w_lo == w_cut && w_cut != INFINITY);
    const int any_fbin = kVotes && __syncthreads_or(tid < kM && r_state == 4);
    const int any_refine = kVotes && __syncthreads_or(tid < kM && r_state == 1);
    const int any_collect = kVotes && __syncthreads_or(tid < kM && r_state == 2);
    int next;
    if (aborted) next = P_DONE;
    else if (pass == P_IDX || pass == P_CODES || pass == P_PV || pass == P_SCORES) next = P_DONE;
    else if (pass == P_NORM) next = (EXPORT == EXP_CODES) ? P_CODES : P_PV;
    else if (any_relevel) next = P_LEVELS;
    else if (any_fbin) next = P_FBIN;
    else if (any_refine) next = P_RADIX;
    else if (any_collect) next = P_COLLECT;
    else if (EXPORT == EXP_IDX) next = P_IDX;
    else if ((EXPORT == EXP_CODES || kQuant) && SEL == SEL_TOPN_FLOAT && pass != P_KEPT_NORM) next = P_KEPT_NORM;
    else if (EXPORT == EXP_CODES) next = P_CODES;
    else next = P_PV;
    if ((next == P_RADIX || next == P_FBIN) && tid < kM)
      for (int bb = 0; bb < kRadixBins / 2; ++bb) hist[bb * kM + srow] = 0u;
    if (next == P_LEVELS && tid < kM)
      for (int lev = 0; lev < kLevels; ++lev) hist[lev * kM + srow] = 0u;
    if (pass == P_LEVELS) sample_levels = false;  // a second level pass counts every tile
    if ((next == P_RADIX || next == P_FBIN) && is_soft) r_above = 0;
    if (kSplitF && (next == P_COLLECT || next == P_PV) && tid < kM) reinterpret_cast<int*>(xchg)[srow] = 0;
    if (next == P_KEPT_NORM && is_soft) lsum = 0.0f;
    __syncthreads();
    first_pass = false;
    pass = next;
  }

  // ---------------------------------------------------------------- epilogue
  // two threads per top-N row with a bias: the row's count of recorded keys, read
  // before the normalizer exchange below reuses its shared slot
  int rc_split = 0;
  if (kSplitF) {
    if (is_soft) rc_split = reinterpret_cast<const int*>(xchg)[srow];
    __syncthreads();
  }
  if (kSplit == 2 && sum_in_pv) {
    // the row's two threads add their partial normalizers
    if (is_soft) xchg[half * kM + srow] = lsum;
    __syncthreads();
    if (is_soft) lsum = xchg[srow] + xchg[kM + srow];
  }
  if (EXPORT == EXP_NONE) {
    if (is_soft) {
      constexpr int kOc = D / kSplit;                 // output channels per softmax thread
      const int c0 = (kSplit == 2) ? kOc * half : 0;  // first channel
      const bool ok = __all_sync(0xffffffffu, bounded_wait(B_OFULL, 0));
      tc_fence_after();
      const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
      // the final radix bin of this row (kMerge): logits of its recorded keys from the
      // same integer score (+-1 codes, exact) and bias entry as in the tiles, the
      // r_rank-th largest as threshold with its ties kept in key order; each kept key's
      // weight goes to the normalizer and replaces its logit in slot kCap + x (0 for a
      // dropped key), and its V row is added to O below, 32 channels at a time
      int n_merge = 0;
      const float* pw = reinterpret_cast<const float*>(hist) + kCap * kM + srow;  // weight x at pw[x * kM]
      const bool merge_row = kMerge && r_state == 3 && ok && row_ok && row < a.n;
      float merged = 0.0f;  // the kept recorded keys' weights
      // (two threads per row: the first takes the row's decisions, the second reads them)
      if (merge_row && (!kSplitF || half == 0)) {
        const int rc = kSplitF ? rc_split : r_cnt;
        n_merge = min(rc, kCap);
        if (rc > kCap) raise_status(a.status, kDevErrCapacity);
        // the recorded keys in key order (the two threads of a row fill the slots in whatever
        // order they reach them), so that the sums over the slots below are reproducible
        for (int x = 1; x < n_merge; ++x) {
          const uint32_t v = hist[x * kM + srow];
          int y = x - 1;
          for (; y >= 0 && hist[y * kM + srow] > v; --y) hist[(y + 1) * kM + srow] = hist[y * kM + srow];
          hist[(y + 1) * kM + srow] = v;
        }
        const int8_t* kb = a.kpm + (size_t)bh * a.n_pad * D;
        for (int x = 0; x < n_merge; ++x) {
          const int j = (int)hist[x * kM + srow];
          const uint4* kr = reinterpret_cast<const uint4*>(kb + (size_t)j * D);
          // s = d - 2 (channels whose signs differ): bit 7 of a +-1 byte is its sign in
          // both encodings (int8 and e4m3)
          int diff = 0;
#pragma unroll
          for (int c16 = 0; c16 < D / 16; ++c16) {
            const uint4 qv = *reinterpret_cast<const uint4*>(sQ + (c16 >> 2) * kM * 64 + srow * 64 +
                                                             (((c16 & 3) ^ ((srow >> 1) & 3)) * 16));
            const uint4 kv = __ldg(kr + c16);
            diff += __popc((qv.x ^ kv.x) & 0x80808080u) + __popc((qv.y ^ kv.y) & 0x80808080u) +
                    __popc((qv.z ^ kv.z) & 0x80808080u) + __popc((qv.w ^ kv.w) & 0x80808080u);
          }
          const int sc = D - 2 * diff;
          float l;
          if (HAS_BIAS) {
            int off;  // entry (i, j) of the extended table sits at rb - off
            if (a.bias_dense) {
              off = -j;
            } else if (j < a.prefix) {
              off = a.k_class;
            } else {
              const int t = j - a.prefix, y = t / a.gw;
              off = y * a.ext_S + (t - y * a.gw);
            }
            l = __fmaf_rn((float)sc, c, __ldg(tab + rb - off));
          } else {
            l = (float)sc * c;
          }
          hist[(kCap + x) * kM + srow] = __float_as_uint(l);
        }
        float* lc = reinterpret_cast<float*>(hist) + kCap * kM + srow;  // logit x at lc[x * kM]
        float vF = INFINITY;
        int gt = 0;
        for (int x = 0; x < n_merge; ++x) {
          const float vx = lc[x * kM];
          int g = 0, e = 0;
          for (int y = 0; y < n_merge; ++y) {
            const float vy = lc[y * kM];
            g += vy > vx ? 1 : 0;
            e += vy == vx ? 1 : 0;
          }
          if (g < r_rank && r_rank <= g + e) {
            vF = vx;
            gt = g;
            break;
          }
        }
        // keys above vF are kept; of the keys at vF, the r_rank - gt with the lowest
        // key indices (the slots need not be in key order)
        const int allow = r_rank - gt;
        uint64_t keep = 0;
        for (int x = 0; x < n_merge; ++x) {
          const float v = lc[x * kM];
          bool k = v > vF;
          if (v == vF) {
            const int jx = (int)hist[x * kM + srow];
            int before = 0;
            for (int y = 0; y < n_merge; ++y)
              before += (lc[y * kM] == vF && (int)hist[y * kM + srow] < jx) ? 1 : 0;
            k = before < allow;
          }
          keep |= (k ? 1ull : 0ull) << x;
        }
        const float mo_e = -m * kLog2e;
        for (int x = 0; x < n_merge; ++x) {
          float p = 0.0f;
          if ((keep >> x) & 1ull) {
            p = fast_exp2(__fmaf_rn(lc[x * kM], kLog2e, mo_e));
            merged += p;
          }
          lc[x * kM] = p;
        }
      }
      bool ok_out = ok;
      if (kSplitF) {
        // the second thread of the row takes the count and the merged weight sum
        float* mx = reinterpret_cast<float*>(koff_tab);  // the key-offset area is free after the passes
        if (half == 0) mx[srow] = merged;
        asm volatile("bar.sync %0, 64;" ::"r"(1 + (warp & 3)) : "memory");
        ok_out = ok && !*abort_flag;  // both warps of the pair see the same abort state here
        if (half == 1) {
          merged = mx[srow];
          n_merge = (merge_row && ok_out) ? min(rc_split, kCap) : 0;
        }
      }
      lsum += merged;
      const float inv = sum_in_pv ? 1.0f / lsum : scale;
#pragma unroll
      for (int cb = 0; cb < kOc; cb += 32) {
        uint32_t o[32];
        tmem_ld32(tl + kColO + c0 + cb, o);
        tmem_wait_ld();
        if (row < a.n) {
          float out[32];
          if (!ok_out || !row_ok) {
#pragma unroll
            for (int k = 0; k < 32; ++k) out[k] = 0.0f;
          } else if (kQuant) {
#pragma unroll
            for (int k = 0; k < 32; ++k) out[k] = (float)(int)o[k] * dq[c0 + cb + k];
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) out[k] = __uint_as_float(o[k]);
            for (int x = 0; x < n_merge; ++x) {  // kept keys of the final bin: p * V[j][channels]
              const float p = pw[x * kM];
              if (p == 0.0f) continue;
              const size_t vrow = (size_t)bh * a.n + (int)hist[x * kM + srow];
              if (a.v_f32) {
                const float4* vr = reinterpret_cast<const float4*>(a.v_raw) + (vrow * D + c0 + cb) / 4;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                  const float4 f = __ldg(vr + q);
                  out[4 * q] = __fmaf_rn(p, f.x, out[4 * q]);
                  out[4 * q + 1] = __fmaf_rn(p, f.y, out[4 * q + 1]);
                  out[4 * q + 2] = __fmaf_rn(p, f.z, out[4 * q + 2]);
                  out[4 * q + 3] = __fmaf_rn(p, f.w, out[4 * q + 3]);
                }
              } else {
                const uint4* vr = reinterpret_cast<const uint4*>(a.v_raw) + (vrow * D + c0 + cb) / 8;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const uint4 u4 = __ldg(vr + q);
                  const uint32_t wv[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
                  for (int t = 0; t < 4; ++t) {
                    out[8 * q + 2 * t] = __fmaf_rn(p, __uint_as_float(wv[t] << 16), out[8 * q + 2 * t]);
                    out[8 * q + 2 * t + 1] = __fmaf_rn(p, __uint_as_float(wv[t] & 0xFFFF0000u), out[8 * q + 2 * t + 1]);
                  }
                }
              }
            }
#pragma unroll
            for (int k = 0; k < 32; ++k) out[k] *= inv;
          }
          const size_t ob = ((size_t)bh * a.n + row) * D + c0 + cb;
          if (a.o_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.O) + ob);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              dst[k] = make_uint4(pack_bf16x2(out[8 * k], out[8 * k + 1]), pack_bf16x2(out[8 * k + 2], out[8 * k + 3]),
                                  pack_bf16x2(out[8 * k + 4], out[8 * k + 5]), pack_bf16x2(out[8 * k + 6], out[8 * k + 7]));
          } else {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.O) + ob);
#pragma unroll
            for (int k = 0; k < 8; ++k) dst[k] = make_float4(out[4 * k], out[4 * k + 1], out[4 * k + 2], out[4 * k + 3]);
          }
        }
      }
    }
  } else if (EXPORT == EXP_IDX) {
    if (tid < kM && row < a.n) {
      int32_t* dst = a.idx + ((size_t)bh * a.n + row) * a.N;
      for (int p = row_ok ? min(kDense ? L : kept_seen, a.N) : 0; p < a.N; ++p) dst[p] = -1;
    }
  } else if (EXPORT == EXP_SCORES) {
    if (tid < kM && row < a.n) {
      int32_t* dst = a.scores + ((size_t)bh * a.n + row) * a.n;
      for (int j = row_ok ? ntiles * kN : 0; j < a.n; ++j) dst[j] = 0;
    }
  } else {
    if (tid < kM && row >= a.row_begin && row < a.row_end && row < a.n) {
      const int rows = a.row_end - a.row_begin;
      uint8_t* dst = a.codes + ((size_t)bh * rows + (row - a.row_begin)) * a.n;
      for (int j = row_ok ? ntiles * kN : 0; j < a.n; ++j) dst[j] = 0;
    }
  }

  // ---------------------------------------------------------------- teardown
  if (warp == kProdWarp && lane == 0 && *abort_flag) {
    // let TMA loads still in flight land before the CTA's shared memory goes away
    for (int s2 = 0; s2 < kKStages; ++s2)
      if (k_par[s2] >= 0) mbar_wait(&bars[B_KFULL + s2], (uint32_t)k_par[s2], 200000000LL);
    for (int s2 = 0; s2 < kVStages; ++s2)
      if (v_par[s2] >= 0) mbar_wait(&bars[B_VFULL + s2], (uint32_t)v_par[s2], 200000000LL);
    if (BIAS == BIAS_SMEM) mbar_wait(&bars[B_BIAS], 0, 200000000LL);
    if (kRef) mbar_wait(&bars[B_QFULL], 0, 200000000LL);
  }
  if (warp == kMmaWarp && lane == 0) {
    // every tcgen05 operation this thread issued is complete before TMEM is freed
    mma_commit(&bars[B_FINAL]);
    mbar_wait(&bars[B_FINAL], 0, 200000000LL);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace tc
}  // namespace had

// had_lib.cu -- C ABI of the binarized-QK top-N attention library (include/had.h).
//
// Host side of every entry point: validate on the host (nothing is enqueued
// on an error), carve the caller's workspace, and enqueue the kernels on the
// caller's stream.  No allocation, no synchronization on the hot path.
//
// had_attention pipeline (method: "Hamming Attention Distillation" top-N over
// binarized keys/queries; "BinaryAttention" §2.2-§2.4):
//   k_stats       : fp64 channel partial sums of Q and K (+ fp32 absmax of V in uint8 modes)
//   k_stats_final : per-head means (and V absmax) from the partials
//   k_pack        : mu -> sign bits of Q (packed uint32) and K (+-1 int8 rows);
//                   V scale -> int8 or 4-bit V^T (uint8 modes)
//   k_bias_range + k_bias_fill (with a bias): per-head bias range, extended bias
//                   and exp(b - b_max) tables
//   k_attn_tc     : scores, logits, top-N select, softmax, A.V, output
//   (heads up to 128 KB: k_prep_head does the statistics, packing and tables in one launch)
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/had.h"
#include "common.cuh"
#include "prep.cuh"
#include "attn.cuh"
#include "attn_tc.cuh"
#include "launch.cuh"
#include "probe.cuh"
#include "qkv.cuh"

namespace had {

__device__ unsigned g_device_status;

namespace {
thread_local char t_last_error[256] = "";
}  // namespace

had_status cuda_fail(cudaError_t e, const char* what) {
  snprintf(t_last_error, sizeof(t_last_error), "%s: %s", what, cudaGetErrorString(e));
  return HAD_ERR_CUDA;
}

had_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? HAD_OK : cuda_fail(e, what);
}

// d = 64 is instantiated here, d = 128 in attn_d128.cu
HAD_DISPATCH_INST(, 64)
HAD_DISPATCH_INST(extern, 128)

namespace {

using tc::SEL_DENSE;
using tc::SEL_TOPN_INT;
using tc::SEL_TOPN_FLOAT;
using tc::EXP_NONE;
using tc::EXP_IDX;
using tc::EXP_CODES;

// bound of the fused kernel's pipeline waits and the timeout-path test hook
// (had_debug_bounded_wait); library-wide, read at each launch
std::atomic<long long> g_wait_cycles{tc::kWaitCycles};
std::atomic<int> g_force_expiry{0};

unsigned* status_ptr(int dev) {
  static std::mutex mu;
  static unsigned* ptrs[kMaxDevices] = {nullptr};
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<unsigned*>(p);
  }
  return ptrs[dev];
}


inline size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Dims {
  int B, H, n, d, BH, nchunks, n_pad;
};

constexpr int kQkvMaxDm = 16384;  // model width of the fused projection

Dims dims_of(const had_shape* s) {
  Dims d;
  d.B = s->B; d.H = s->H; d.n = s->n; d.d = s->d; d.BH = s->B * s->H;
  d.nchunks = (s->n + kChunk - 1) / kChunk;
  d.n_pad = d.nchunks * kChunk;
  return d;
}

// Head dims: 64 and 128 everywhere; 32 also in the pack and int8-V entry points.
had_status check_shape(const had_shape* s, bool allow_d32 = false) {
  if (!s) return HAD_ERR_INVALID;
  if (s->B <= 0 || s->H <= 0 || s->n <= 0 || s->d <= 0) return HAD_ERR_INVALID;
  if (s->in_dtype != HAD_F32 && s->in_dtype != HAD_BF16) return HAD_ERR_INVALID;
  const bool d_ok = s->d == 64 || s->d == 128 || (allow_d32 && s->d == 32);
  if (!d_ok || s->n > kMaxN || s->H > kMaxHeads || (long long)s->B * s->H > 65535) return HAD_ERR_UNSUPPORTED;
  if (s->seqlens && (reinterpret_cast<uintptr_t>(s->seqlens) & 3u)) return HAD_ERR_INVALID;
  return HAD_OK;
}

had_status check_bias(const had_shape* s, const had_relpos_bias* bias) {
  if (!bias || !bias->table) return HAD_OK;
  if (reinterpret_cast<uintptr_t>(bias->table) & 3u) return HAD_ERR_INVALID;
  if (bias->dense != 0) {
    if (bias->dense != 1) return HAD_ERR_INVALID;
    return s->n > kDenseBiasMaxN ? HAD_ERR_UNSUPPORTED : HAD_OK;
  }
  if (bias->gh <= 0 || bias->gw <= 0 || bias->prefix < 0) return HAD_ERR_INVALID;
  if ((long long)bias->gh * bias->gw + bias->prefix != s->n) return HAD_ERR_INVALID;
  if (reinterpret_cast<uintptr_t>(bias->table) & 3u) return HAD_ERR_INVALID;
  return HAD_OK;
}

struct Ws {
  size_t qbits, kpm, sums, amax, vqT, vscale, bminmax, bext, expb, vhi, vlo, total;
};

// Bits of the quantized V of a mode: 0 (float V), 8 (int8), 4 (packed 4-bit).
int vbits_of(had_mode mode) { return mode == HAD_MODE_U8I8 ? 8 : mode == HAD_MODE_U8I4 ? 4 : 0; }
bool mode_ok(had_mode mode) { return mode == HAD_MODE_FLOAT || mode == HAD_MODE_U8I8 || mode == HAD_MODE_U8I4; }

Ws ws_layout(const had_shape* s, int vbits, const had_relpos_bias* bias_desc) {
  const bool bias = bias_desc && bias_desc->table;
  const bool quant = vbits != 0;
  Dims d = dims_of(s);
  Ws w{};
  size_t off = 0;
  w.qbits = off; off += align_up((size_t)d.BH * d.n * (d.d / 32) * 4);
  w.kpm = off; off += align_up((size_t)d.BH * d.n_pad * d.d);
  w.sums = off; off += align_up((size_t)2 * d.BH * d.nchunks * d.d * 8);
  w.amax = w.vqT = w.vscale = w.bminmax = 0;
  if (quant) {
    w.amax = off; off += align_up((size_t)d.BH * d.nchunks * d.d * 4);
    w.vqT = off; off += align_up((size_t)d.BH * d.d * (vbits == 4 ? d.n_pad / 2 : d.n_pad));
    w.vscale = off; off += align_up((size_t)d.BH * d.d * 4);
  }
  w.bext = w.expb = 0;
  if (bias) {
    w.bminmax = off; off += align_up((size_t)s->H * 2 * 4);
    const size_t cells = bias_desc->dense ? (size_t)dense_ext(s->n).E : (size_t)relpos_ext(bias_desc->gh, bias_desc->gw).E;
    w.bext = off; off += align_up((size_t)s->H * cells * 4);
    w.expb = off; off += align_up((size_t)s->H * cells * 4);
  }
  w.vhi = w.vlo = 0;
  if (!quant && s->in_dtype == HAD_F32) {
    // fp32 V in float mode: bf16 head and residual copies for the tensor cores
    w.vhi = off; off += align_up((size_t)d.BH * d.n * d.d * 2);
    w.vlo = off; off += align_up((size_t)d.BH * d.n * d.d * 2);
  }
  w.total = off;
  return w;
}

__global__ void k_split_v(const float* __restrict__ V, size_t count, __nv_bfloat16* __restrict__ hi,
                          __nv_bfloat16* __restrict__ lo) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < count; e += (size_t)gridDim.x * blockDim.x) {
    const float v = V[e];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi[e] = h;
    lo[e] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

// ---------------------------------------------------------------------------- TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor [outer][inner] of `dt`, tile box {box_in, box_out}.
had_status encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                     uint64_t row_bytes, uint32_t box_in, uint32_t box_out, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cuda_fail(cudaErrorNotSupported, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_in, box_out};
  const cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(t_last_error, sizeof(t_last_error), "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return HAD_ERR_CUDA;
  }
  return HAD_OK;
}

// V^T codes back to [BH][n][d] int8 (a 4-bit code sign-extended from its nibble).
__global__ void k_untranspose_vq(const int8_t* vqT, int BH, int n, int d, int n_pad, int vbits, int8_t* Vq) {
  const size_t total = (size_t)BH * n * d;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const int c = (int)(e % d);
    const size_t ti = e / d;
    const int i = (int)(ti % n);
    const int bh = (int)(ti / n);
    if (vbits == 4) {
      const uint8_t byte = reinterpret_cast<const uint8_t*>(vqT)[((size_t)bh * d + c) * (n_pad / 2) + i / 2];
      const int nib = (i & 1) ? (byte >> 4) : (byte & 15);
      Vq[e] = (int8_t)(nib >= 8 ? nib - 16 : nib);
    } else {
      Vq[e] = vqT[((size_t)bh * d + c) * n_pad + i];
    }
  }
}

// ---------------------------------------------------------------------------- prep launches

had_status launch_prep(const had_shape* s, const void* X0, const void* X1, const void* X2, int first, int ntens,
                       double* sums, float* amax, const float* mu_in0, float* mu_out0, uint32_t* bits0,
                       int8_t* pm0, uint32_t* bits1, int8_t* pm1, int8_t* vqT, float* vscale, cudaStream_t st,
                       unsigned* status, int vbits = 8, bool pm_e4m3 = false,
                       const float* v_amax = nullptr) {
  Dims d = dims_of(s);
  PrepArgs pa{};
  pa.X[0] = X0; pa.X[1] = X1; pa.X[2] = X2;
  pa.ntens = ntens; pa.first_tensor = first;
  pa.B = d.B; pa.H = d.H; pa.n = d.n; pa.nchunks = d.nchunks;
  pa.seqlens = s->seqlens; pa.sums = sums; pa.amax = amax; pa.status = status;
  dim3 grid(d.nchunks, d.BH, ntens);
  // no statistics pass when the caller gives Q's mean (bits of Q alone) or V's absmax (V alone)
  const bool need_stats = !(mu_in0 && first == 0 && ntens == 1) && !(v_amax && first == 2 && ntens == 1);
  const bool bf = s->in_dtype == HAD_BF16;
  if (need_stats) {
    if (d.d == 32) bf ? k_stats<__nv_bfloat16, 32><<<grid, kPrepThreads, 0, st>>>(pa) : k_stats<float, 32><<<grid, kPrepThreads, 0, st>>>(pa);
    else if (d.d == 128) bf ? k_stats<__nv_bfloat16, 128><<<grid, kPrepThreads, 0, st>>>(pa) : k_stats<float, 128><<<grid, kPrepThreads, 0, st>>>(pa);
    else bf ? k_stats<__nv_bfloat16, 64><<<grid, kPrepThreads, 0, st>>>(pa) : k_stats<float, 64><<<grid, kPrepThreads, 0, st>>>(pa);
    had_status r = check_launch("k_stats");
    if (r != HAD_OK) return r;
    dim3 fgrid(d.BH, ntens);
    if (d.d == 32) k_stats_final<32><<<fgrid, 128, 0, st>>>(pa);
    else if (d.d == 128) k_stats_final<128><<<fgrid, 128, 0, st>>>(pa);
    else k_stats_final<64><<<fgrid, 128, 0, st>>>(pa);
    if ((r = check_launch("k_stats_final")) != HAD_OK) return r;
  }
  PackArgs ka{};
  ka.X[0] = X0; ka.X[1] = X1; ka.X[2] = X2;
  ka.ntens = ntens; ka.first_tensor = first;
  ka.B = d.B; ka.H = d.H; ka.n = d.n; ka.nchunks = d.nchunks; ka.n_pad = d.n_pad;
  ka.seqlens = s->seqlens; ka.sums = sums;
  ka.amax = need_stats ? amax : v_amax;
  ka.amax_ld = need_stats ? d.nchunks * d.d : d.d;
  ka.mu_in[0] = mu_in0; ka.mu_in[1] = nullptr;
  ka.mu_out[0] = mu_out0; ka.mu_out[1] = nullptr;
  ka.bits[0] = bits0; ka.bits[1] = bits1;
  ka.pm[0] = pm0; ka.pm[1] = pm1;
  ka.vqT = vqT; ka.vscale = vscale; ka.v_bits = vbits; ka.pm_e4m3 = pm_e4m3 ? 1 : 0; ka.status = status;
  if (d.d == 32) bf ? k_pack<__nv_bfloat16, 32><<<grid, kPrepThreads, 0, st>>>(ka) : k_pack<float, 32><<<grid, kPrepThreads, 0, st>>>(ka);
  else if (d.d == 128) bf ? k_pack<__nv_bfloat16, 128><<<grid, kPrepThreads, 0, st>>>(ka) : k_pack<float, 128><<<grid, kPrepThreads, 0, st>>>(ka);
  else bf ? k_pack<__nv_bfloat16, 64><<<grid, kPrepThreads, 0, st>>>(ka) : k_pack<float, 64><<<grid, kPrepThreads, 0, st>>>(ka);
  return check_launch("k_pack");
}

// ---------------------------------------------------------------------------- attention launches

// Host-side validation shared by the attention entry points.
template <int EXP>
had_status validate_attention(const void* Q, const void* K, const void* V, const had_shape* s,
                              const had_relpos_bias* bias, const float* alpha_q, const float* alpha_k, int N,
                              had_mode mode, const void* O, had_dtype o_dtype, const int32_t* idx,
                              const uint8_t* codes, int row_begin, int row_end, const void* workspace,
                              size_t ws_bytes, bool check_qk, bool check_o) {
  had_status r = check_shape(s);
  if (r != HAD_OK) return r;
  if ((r = check_bias(s, bias)) != HAD_OK) return r;
  if (N < 0 || !mode_ok(mode)) return HAD_ERR_INVALID;
  if (mode == HAD_MODE_U8I4 && EXP != EXP_NONE) return HAD_ERR_INVALID;
  if (check_qk && (!Q || !K || !aligned16(Q) || !aligned16(K))) return HAD_ERR_INVALID;
  if (EXP == EXP_NONE || EXP == EXP_CODES) {
    if (!V || !aligned16(V)) return HAD_ERR_INVALID;
  }
  if (EXP == EXP_NONE && check_o) {
    if (!O || !aligned16(O) || (o_dtype != HAD_F32 && o_dtype != HAD_BF16)) return HAD_ERR_INVALID;
  }
  if (EXP == EXP_IDX && (!idx || N < 1 || (reinterpret_cast<uintptr_t>(idx) & 3u))) return HAD_ERR_INVALID;
  if (EXP == tc::EXP_SCORES && (!idx || (reinterpret_cast<uintptr_t>(idx) & 3u))) return HAD_ERR_INVALID;
  if (EXP == EXP_CODES && (!codes || row_begin < 0 || row_end <= row_begin || row_end > s->n)) return HAD_ERR_INVALID;
  for (int h = 0; alpha_q && h < s->H; ++h)
    if (!(alpha_q[h] > 0.0f) || !std::isfinite(alpha_q[h])) return HAD_ERR_INVALID;
  for (int h = 0; alpha_k && h < s->H; ++h)
    if (!(alpha_k[h] > 0.0f) || !std::isfinite(alpha_k[h])) return HAD_ERR_INVALID;
  const Ws w = ws_layout(s, vbits_of(mode), bias);
  if (!workspace || ws_bytes < w.total || !aligned16(workspace)) return HAD_ERR_INVALID;
  return HAD_OK;
}

int select_kind(const had_shape* s, const had_relpos_bias* bias, int N) {
  if (N > 0 && N < s->n) return (bias && bias->table) ? SEL_TOPN_FLOAT : SEL_TOPN_INT;
  return SEL_DENSE;
}

// Opt-in dynamic shared memory of the short-head prep kernel, once per variant and device.
had_status set_prep_smem(int which, int small, int dev) {
  static std::mutex mu;
  static bool done[2][2][kMaxDevices] = {};
  std::lock_guard<std::mutex> lk(mu);
  if (dev < 0 || dev >= kMaxDevices || done[which][small][dev]) return HAD_OK;
  cudaError_t e;
  if (which == 0 && small) e = cudaFuncSetAttribute(k_prep_head<__nv_bfloat16, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kHeadMaxBytes);
  else if (which == 0) e = cudaFuncSetAttribute(k_prep_head<__nv_bfloat16, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize, kHeadMaxBytes);
  else if (small) e = cudaFuncSetAttribute(k_prep_head<float, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kHeadMaxBytes);
  else e = cudaFuncSetAttribute(k_prep_head<float, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize, kHeadMaxBytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(k_prep_head)");
  done[which][small][dev] = true;
  return HAD_OK;
}

// Stage 1: statistics, sign/pack of Q and K, int8 or 4-bit V (uint8 modes), bias range (top-N with bias).
had_status prepare_stage(const void* Q, const void* K, const void* V, const had_shape* s,
                         const had_relpos_bias* bias, int N, had_mode mode, bool need_v, void* workspace,
                         cudaStream_t st, unsigned* status) {
  const bool has_bias = bias && bias->table;
  const int vbits = vbits_of(mode);
  const bool quant = vbits != 0;
  const Ws w = ws_layout(s, vbits, bias);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* qbits = reinterpret_cast<uint32_t*>(ws + w.qbits);
  int8_t* kpm = reinterpret_cast<int8_t*>(ws + w.kpm);
  double* sums = reinterpret_cast<double*>(ws + w.sums);
  float* amax = quant ? reinterpret_cast<float*>(ws + w.amax) : nullptr;
  int8_t* vqT = quant ? reinterpret_cast<int8_t*>(ws + w.vqT) : nullptr;
  float* vscale = quant ? reinterpret_cast<float*>(ws + w.vscale) : nullptr;
  const bool do_v = quant && need_v;
  // top-N with a bias scores on the fp8 tensor path: K~ as e4m3 +-1
  const bool e4m3 = select_kind(s, bias, N) == SEL_TOPN_FLOAT;
  had_status r = HAD_OK;
  const size_t elem = (s->in_dtype == HAD_BF16) ? 2 : 4;
  const size_t head_bytes = (size_t)s->n * s->d * elem;
  BiasArgs ba{};
  if (has_bias) {
    ba.table = bias->table;
    ba.gh = bias->gh; ba.gw = bias->gw; ba.prefix = bias->prefix;
    ba.dense = bias->dense; ba.n = s->n;
    if (ba.dense) { ba.gh = ba.gw = 1; ba.prefix = 0; }
    ba.bminmax = reinterpret_cast<float*>(ws + w.bminmax);
    ba.bext = reinterpret_cast<float*>(ws + w.bext);
    ba.expb = reinterpret_cast<float*>(ws + w.expb);
  }
  if (has_bias && ba.dense) {
    // dense matrix: its range, then its tables over many CTAs per head
    k_dense_bias_range<<<s->H, kDenseRangeThreads, 0, st>>>(ba);
    if ((r = check_launch("k_dense_bias_range")) != HAD_OK) return r;
    dim3 tgrid((dense_ext(s->n).E + kDenseTabPerCta - 1) / kDenseTabPerCta, s->H);
    k_dense_bias_tables<<<tgrid, 256, 0, st>>>(ba);
    if ((r = check_launch("k_dense_bias_tables")) != HAD_OK) return r;
  }
  if (s->d == 64 && head_bytes <= (size_t)kHeadMaxBytes) {
    // short heads: one read of each head, statistics and packing from shared memory
    HeadArgs ha{};
    ha.X[0] = Q; ha.X[1] = K; ha.X[2] = V;
    ha.first_tensor = 0;
    ha.B = s->B; ha.H = s->H; ha.n = s->n; ha.n_pad = dims_of(s).n_pad;
    ha.seqlens = s->seqlens;
    ha.qbits = qbits; ha.kpm = kpm; ha.vqT = vqT; ha.vscale = vscale; ha.v_bits = vbits; ha.status = status;
    ha.kpm_e4m3 = e4m3 ? 1 : 0;
    ha.bias_slice = do_v ? 3 : 2;  // relative-position tables ride along as one more grid slice
    dim3 grid(dims_of(s).BH, ha.bias_slice + (has_bias && !ba.dense ? 1 : 0));
    const int smem = (int)head_bytes;
    int dev = 0;
    cudaGetDevice(&dev);
    const int which = (s->in_dtype == HAD_BF16) ? 0 : 1;
    const int small = head_bytes <= (size_t)kHeadSmallBytes ? 1 : 0;
    if ((r = set_prep_smem(which, small, dev)) != HAD_OK) return r;
    if (which == 0 && small) k_prep_head<__nv_bfloat16, 128><<<grid, 128, smem, st>>>(ha, ba);
    else if (which == 0) k_prep_head<__nv_bfloat16, 256><<<grid, 256, smem, st>>>(ha, ba);
    else if (small) k_prep_head<float, 128><<<grid, 128, smem, st>>>(ha, ba);
    else k_prep_head<float, 256><<<grid, 256, smem, st>>>(ha, ba);
    if ((r = check_launch("k_prep_head")) != HAD_OK) return r;
  } else {
    r = launch_prep(s, Q, K, V, 0, do_v ? 3 : 2, sums, amax, nullptr, nullptr, qbits, nullptr, nullptr, kpm, vqT,
                    vscale, st, status, vbits, e4m3);
    if (r != HAD_OK) return r;
    if (has_bias && !ba.dense) {
      k_bias_range<<<s->H, kBiasRangeThreads, 0, st>>>(ba);
      if ((r = check_launch("k_bias_range")) != HAD_OK) return r;
      dim3 fgrid((relpos_ext(ba.gh, ba.gw).E + kBiasFillPerCta - 1) / kBiasFillPerCta, s->H);
      k_bias_fill<<<fgrid, 256, 0, st>>>(ba);
      if ((r = check_launch("k_bias_fill")) != HAD_OK) return r;
    }
  }
  if (!quant && s->in_dtype == HAD_F32 && need_v) {
    const size_t count = (size_t)dims_of(s).BH * s->n * s->d;
    k_split_v<<<1024, 256, 0, st>>>(static_cast<const float*>(V), count,
                                     reinterpret_cast<__nv_bfloat16*>(ws + w.vhi),
                                     reinterpret_cast<__nv_bfloat16*>(ws + w.vlo));
    if ((r = check_launch("k_split_v")) != HAD_OK) return r;
  }
  return HAD_OK;
}

// Workspace of the comparison mode: the bias range and extended tables only.
struct RefWs {
  size_t bminmax, bext, expb, total;
};

RefWs ref_ws_layout(const had_shape* s, const had_relpos_bias* bias) {
  RefWs w{};
  if (!bias || !bias->table) return w;
  const size_t cells = bias->dense ? (size_t)dense_ext(s->n).E : (size_t)relpos_ext(bias->gh, bias->gw).E;
  size_t off = 0;
  w.bminmax = off; off += align_up((size_t)s->H * 2 * 4);
  w.bext = off; off += align_up((size_t)s->H * cells * 4);
  w.expb = off; off += align_up((size_t)s->H * cells * 4);
  w.total = off;
  return w;
}

// The bias range and extended tables of a relative-position table or a dense matrix.
had_status build_bias_tables(const had_shape* s, const had_relpos_bias* bias, uint8_t* bminmax, uint8_t* bext,
                             uint8_t* expb, cudaStream_t st) {
  BiasArgs ba{};
  ba.table = bias->table;
  ba.gh = bias->gh; ba.gw = bias->gw; ba.prefix = bias->prefix;
  ba.dense = bias->dense; ba.n = s->n;
  if (ba.dense) { ba.gh = ba.gw = 1; ba.prefix = 0; }
  ba.bminmax = reinterpret_cast<float*>(bminmax);
  ba.bext = reinterpret_cast<float*>(bext);
  ba.expb = reinterpret_cast<float*>(expb);
  had_status r;
  if (ba.dense) {
    k_dense_bias_range<<<s->H, kDenseRangeThreads, 0, st>>>(ba);
    if ((r = check_launch("k_dense_bias_range")) != HAD_OK) return r;
    dim3 tgrid((dense_ext(s->n).E + kDenseTabPerCta - 1) / kDenseTabPerCta, s->H);
    k_dense_bias_tables<<<tgrid, 256, 0, st>>>(ba);
    return check_launch("k_dense_bias_tables");
  }
  const int E = relpos_ext(ba.gh, ba.gw).E;
  if (E <= kBiasFillPerCta) {  // small tables: one CTA per head takes the range and fills the tables
    k_bias_tables<<<s->H, 256, 0, st>>>(ba);
    return check_launch("k_bias_tables");
  }
  k_bias_range<<<s->H, kBiasRangeThreads, 0, st>>>(ba);
  if ((r = check_launch("k_bias_range")) != HAD_OK) return r;
  dim3 fgrid((E + kBiasFillPerCta - 1) / kBiasFillPerCta, s->H);
  k_bias_fill<<<fgrid, 256, 0, st>>>(ba);
  return check_launch("k_bias_fill");
}

// The bias fields of the kernel arguments (extended-table geometry, table
// pointers) and the bias variant to launch: none, the exp(bias) table staged in
// shared memory (small tables), per-warp windows (relative-position tables with
// no class tokens on grid rows of a multiple of 64 patches: a warp's 32 rows and
// a tile's 64 keys each lie in one image row), 16-byte row loads (a dense matrix
// with a row stride of 4), or gathers from global memory.
int fill_bias_args(tc::TcArgs& a, const had_shape* s, const had_relpos_bias* bias, uint8_t* bminmax, uint8_t* bext,
                   uint8_t* expb, bool* rows) {
  const bool has_bias = bias && bias->table;
  *rows = false;
  if (!has_bias) return tc::BIAS_NONE;
  a.table = bias->table;
  a.bminmax = reinterpret_cast<float*>(bminmax);
  a.bext = reinterpret_cast<float*>(bext);
  a.expb = reinterpret_cast<float*>(expb);
  if (bias->dense) {
    const DenseExt x = dense_ext(s->n);
    a.bias_dense = 1;
    a.gh = 1; a.gw = 1; a.prefix = 0;
    a.th = s->n; a.tw = s->n;
    a.ext_E = x.E; a.ext_S = x.S; a.rb_class = 0; a.k_class = 0; a.k_invalid = x.k_invalid;
  } else {
    const RelposExt x = relpos_ext(bias->gh, bias->gw);
    a.gh = bias->gh; a.gw = bias->gw; a.prefix = bias->prefix;
    a.th = 2 * bias->gh - 1; a.tw = 2 * bias->gw - 1;
    a.ext_E = x.E; a.ext_S = x.S; a.rb_class = x.rb_class; a.k_class = x.k_class; a.k_invalid = x.k_invalid;
  }
  *rows = !bias->dense && bias->prefix == 0 && bias->gw % 64 == 0 && a.ext_S == 2 * bias->gw;
  return a.ext_E <= tc::kBiasSmemMax           ? tc::BIAS_SMEM
         : *rows                               ? tc::BIAS_ROWS
         : a.bias_dense && a.ext_S % 4 == 0    ? tc::BIAS_DGLOBAL
                                               : tc::BIAS_GLOBAL;
}

// Stage 2: the fused kernel over a prepared workspace.
template <int EXP>
had_status attend_stage(const void* V, const had_shape* s, const had_relpos_bias* bias, const float* alpha_q,
                        const float* alpha_k, int N, had_mode mode, void* O, had_dtype o_dtype, int32_t* idx,
                        uint8_t* codes, int row_begin, int row_end, void* workspace, cudaStream_t st,
                        unsigned* status) {
  const int vbits = vbits_of(mode);
  const bool quant = vbits != 0;
  const Ws w = ws_layout(s, vbits, bias);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  Dims d = dims_of(s);
  const bool vf32 = (s->in_dtype == HAD_F32) && !quant;
  tc::TcArgs a;
  memset(&a, 0, sizeof(a));
  // tiles are 64-channel panels: K~ boxes of 64 B x 64 keys, V boxes of 64 bf16 x 64 keys,
  // int8 V^T boxes of 64 keys x d channels
  had_status r = encode_2d(&a.tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, ws + w.kpm, d.d, (uint64_t)d.BH * d.n_pad, d.d, 64,
                           tc::kN, CU_TENSOR_MAP_SWIZZLE_64B);
  if (r != HAD_OK) return r;
  const bool needs_v = (EXP == EXP_NONE);
  if (needs_v && vbits == 4) {
    a.vq4 = ws + w.vqT;  // packed nibbles, expanded in shared memory by the producer warp
  } else if (needs_v && quant) {
    r = encode_2d(&a.tm_vq, CU_TENSOR_MAP_DATA_TYPE_UINT8, ws + w.vqT, d.n_pad, (uint64_t)d.BH * d.d, d.n_pad, tc::kN,
                  d.d, CU_TENSOR_MAP_SWIZZLE_64B);
    if (r != HAD_OK) return r;
  } else if (needs_v) {
    const void* vb = vf32 ? static_cast<const void*>(ws + w.vhi) : V;
    r = encode_2d(&a.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, vb, d.d, (uint64_t)d.BH * d.n, d.d * 2, 64, tc::kN,
                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (r != HAD_OK) return r;
    if (vf32) {
      r = encode_2d(&a.tm_vlo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ws + w.vlo, d.d, (uint64_t)d.BH * d.n, d.d * 2, 64,
                    tc::kN, CU_TENSOR_MAP_SWIZZLE_128B);
      if (r != HAD_OK) return r;
    }
  }
  a.qbits = reinterpret_cast<uint32_t*>(ws + w.qbits);
  a.kpm = reinterpret_cast<const int8_t*>(ws + w.kpm);
  a.v_raw = V;
  a.v_f32 = (s->in_dtype == HAD_F32) ? 1 : 0;
  a.vscale = quant ? reinterpret_cast<float*>(ws + w.vscale) : nullptr;
  bool rows = false;
  const int bias_kind = fill_bias_args(a, s, bias, ws + w.bminmax, ws + w.bext, ws + w.expb, &rows);
  a.seqlens = s->seqlens;
  a.O = O; a.o_bf16 = (o_dtype == HAD_BF16) ? 1 : 0;
  a.idx = idx; a.codes = codes; a.row_begin = row_begin; a.row_end = row_end;
  if (EXP == tc::EXP_SCORES) a.scores = idx;
  a.wait_cycles = g_wait_cycles.load();
  a.force_expiry = g_force_expiry.load();
  a.B = d.B; a.H = d.H; a.n = d.n; a.n_pad = d.n_pad; a.N = N;
  a.status = status;
  a.koff_mode = (d.n_pad <= tc::kKoffTableMax) ? tc::kKoffTable : tc::kKoffWarp;
  a.int_levels = 1;
  for (int h = 0; h < s->H; ++h) {
    const double aq = alpha_q ? (double)alpha_q[h] : 1.0, ak = alpha_k ? (double)alpha_k[h] : 1.0;
    const float c = (float)(aq * ak / std::sqrt((double)s->d));
    a.c_head[h] = c;
    // the d + 1 score levels must map to distinct fp32 logits for the integer tie test
    volatile float prev = -INFINITY;
    for (int sc = -s->d; sc <= s->d; sc += 2) {
      volatile float lv = (float)sc * c;
      if (!(lv > prev) || !std::isfinite(lv)) a.int_levels = 0;
      prev = lv;
    }
  }
  dim3 grid((s->n + tc::kM - 1) / tc::kM, d.BH);
  const int sel = EXP == tc::EXP_SCORES ? (int)tc::SEL_DENSE : select_kind(s, bias, N);
  const int md = vbits == 4 ? tc::MODE_Q4 : quant ? tc::MODE_Q : tc::MODE_F;
  if (s->d == 128) return launch::dispatch_tc<128, EXP>(sel, md, bias_kind, vf32, rows, a, grid, st);
  return launch::dispatch_tc<64, EXP>(sel, md, bias_kind, vf32, rows, a, grid, st);
}

// Workspace of the fused projection: the attention workspace (so that
// had_attention_prepared can run on it), then X's token partial sums, the
// partial means of Q and K, and V's column absmax per head.
struct QkvWs {
  size_t xpart, mu, vamax, total;
  int nch;
};

QkvWs qkv_ws_layout(const had_shape* s, int Dm, int vbits, const had_relpos_bias* bias) {
  QkvWs q{};
  size_t off = align_up(ws_layout(s, vbits, bias).total);
  q.nch = (s->n + qkv::kXsumChunk - 1) / qkv::kXsumChunk;
  q.xpart = off; off += align_up((size_t)s->B * q.nch * Dm * 8);
  q.mu = off; off += align_up((size_t)qkv::kMuSplit * 2 * s->B * s->H * 64 * 8);
  q.vamax = off; off += align_up((size_t)s->B * s->H * 64 * 4);
  q.total = off;
  return q;
}

had_status check_qkv_shape(const had_shape* s, int Dm) {
  had_status r = check_shape(s);
  if (r != HAD_OK) return r;
  if (s->d != 64 || s->in_dtype != HAD_BF16) return HAD_ERR_UNSUPPORTED;
  if (Dm <= 0 || Dm % 64 != 0) return HAD_ERR_INVALID;
  if (Dm > kQkvMaxDm || 3 * s->H > 65535) return HAD_ERR_UNSUPPORTED;
  return HAD_OK;
}

had_status device_status_ptr(unsigned** out) {
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
  *out = status_ptr(dev);
  if (!*out) return cuda_fail(cudaErrorInvalidSymbol, "status word");
  return HAD_OK;
}

// Shared body of had_attention and its exports.
template <int EXP>
had_status run_attention(const void* Q, const void* K, const void* V, const had_shape* s,
                         const had_relpos_bias* bias, const float* alpha_q, const float* alpha_k, int N,
                         had_mode mode, void* O, had_dtype o_dtype, int32_t* idx, uint8_t* codes, int row_begin,
                         int row_end, void* workspace, size_t ws_bytes, void* stream) {
  had_status r = validate_attention<EXP>(Q, K, V, s, bias, alpha_q, alpha_k, N, mode, O, o_dtype, idx, codes,
                                         row_begin, row_end, workspace, ws_bytes, true, true);
  if (r != HAD_OK) return r;
  unsigned* status = nullptr;
  if ((r = device_status_ptr(&status)) != HAD_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  r = prepare_stage(Q, K, V, s, bias, N, mode, EXP != EXP_IDX && EXP != tc::EXP_SCORES, workspace, st, status);
  if (r != HAD_OK) return r;
  return attend_stage<EXP>(V, s, bias, alpha_q, alpha_k, N, mode, O, o_dtype, idx, codes, row_begin, row_end,
                           workspace, st, status);
}

// ---------------------------------------------------------------------------- host buffers in and out

// Staging of had_attention_host in its device workspace: the seqlens and bias
// table copies, then `slots` chunk slots (Q, K, V, O and the kernels'
// workspace of one chunk of `cb` sequences) that consecutive chunks cycle through.
struct HostPlan {
  int cb = 0, hc = 0, hgroups = 0, chunks = 0, slots = 0;  // sequences per chunk, heads per chunk (when a
                                                            // sequence is split), head groups per sequence
  size_t in_b = 0, head_b = 0;                // bytes of one sequence, of one head, of Q (= K = V)
  size_t seq = 0, tab = 0, tab_bytes = 0, slot0 = 0, slot_bytes = 0, total = 0;
  size_t q = 0, k = 0, v = 0, o = 0, ws = 0;  // offsets inside a slot
  size_t ws_bytes = 0;
};

constexpr int kHostSlots = 4;    // two chunks computing, one copying in, one copying out
constexpr int kHostCompute = 2;  // compute streams: the caller's and one side stream, alternating chunks
constexpr size_t kHostChunkBytes = size_t(8) << 20;  // input bytes per chunk when the caller passes chunk_b = 0
constexpr size_t kHostSplitBytes = size_t(16) << 20;  // at most this per chunk when a sequence is split by heads

// Chunks: chunk_b > 0 takes chunk_b whole sequences per chunk.  chunk_b = 0 takes
// about kHostChunkBytes of inputs: whole sequences while one fits, else one
// sequence's heads in equal groups of at most kHostSplitBytes (so that long
// sequences also start computing after a short copy, and the copy of the last O
// is short).
had_status host_plan(const had_shape* s, had_mode mode, const had_relpos_bias* bias, int chunk_b, HostPlan* p) {
  if (!s) return HAD_ERR_INVALID;
  had_shape s0 = *s;
  s0.seqlens = nullptr;  // a host array here: checked by value in had_attention_host
  had_status r = check_shape(&s0);
  if (r != HAD_OK) return r;
  if ((r = check_bias(&s0, bias)) != HAD_OK) return r;
  if (chunk_b < 0) return HAD_ERR_INVALID;
  const bool has_bias = bias && bias->table;
  const size_t esz = s->in_dtype == HAD_BF16 ? 2 : 4;
  p->head_b = (size_t)s->n * s->d * esz;
  p->in_b = (size_t)s->H * p->head_b;
  const size_t head_ob = (size_t)s->n * s->d * 4;  // O as fp32 (the larger output type)
  p->hc = s->H;
  if (chunk_b > 0) {
    p->cb = std::min(chunk_b, s->B);
  } else if (3 * p->in_b <= kHostChunkBytes) {
    p->cb = (int)std::min<size_t>(kHostChunkBytes / (3 * p->in_b), (size_t)s->B);
  } else {
    // head groups of at most kHostSplitBytes of inputs, of equal size: enough rows per chunk that two
    // chunks in flight fill the GPU
    p->cb = 1;
    const int hmax = (int)std::max<size_t>(1, std::min<size_t>(kHostSplitBytes / (3 * p->head_b), (size_t)s->H));
    const int groups = (s->H + hmax - 1) / hmax;
    p->hc = (s->H + groups - 1) / groups;
  }
  p->hgroups = (s->H + p->hc - 1) / p->hc;
  p->chunks = ((s->B + p->cb - 1) / p->cb) * p->hgroups;
  p->slots = std::min(kHostSlots, p->chunks);
  had_shape sc = s0;
  sc.B = p->cb;
  sc.H = p->hc;
  p->ws_bytes = ws_layout(&sc, vbits_of(mode), has_bias ? bias : nullptr).total;
  size_t off = 0;
  p->seq = off;
  off += align_up((size_t)s->B * sizeof(int32_t));
  p->tab = off;
  p->tab_bytes = !has_bias ? 0
                 : bias->dense ? (size_t)s->H * s->n * s->n * sizeof(float)
                               : (size_t)s->H * (2 * bias->gh - 1) * (2 * bias->gw - 1) * sizeof(float);
  off += align_up(p->tab_bytes);
  p->slot0 = off;
  const size_t cin = (size_t)p->cb * p->hc * p->head_b, cout = (size_t)p->cb * p->hc * head_ob;
  size_t so = 0;
  p->q = so; so += align_up(cin);
  p->k = so; so += align_up(cin);
  p->v = so; so += align_up(cin);
  p->o = so; so += align_up(cout);
  p->ws = so; so += align_up(p->ws_bytes);
  p->slot_bytes = so;
  p->total = off + (size_t)p->slots * so;
  return HAD_OK;
}

// The side streams and events of one had_attention_host call.  Whatever has
// been enqueued when it goes out of scope (also after an error), the caller's
// stream is made to wait for it; the streams and events are then released
// (CUDA defers that until their pending work is done).
struct HostStreams {
  cudaStream_t main = nullptr, in = nullptr, out = nullptr, comp = nullptr;
  cudaEvent_t start = nullptr, join_in = nullptr, join_out = nullptr, join_comp = nullptr;
  cudaEvent_t in_done[kHostSlots] = {}, comp_done[kHostSlots] = {}, out_done[kHostSlots] = {};
  ~HostStreams() {
    if (in && join_in && cudaEventRecord(join_in, in) == cudaSuccess) cudaStreamWaitEvent(main, join_in, 0);
    if (out && join_out && cudaEventRecord(join_out, out) == cudaSuccess) cudaStreamWaitEvent(main, join_out, 0);
    if (comp && join_comp && cudaEventRecord(join_comp, comp) == cudaSuccess)
      cudaStreamWaitEvent(main, join_comp, 0);
    for (cudaEvent_t e : {start, join_in, join_out, join_comp})
      if (e) cudaEventDestroy(e);
    for (int i = 0; i < kHostSlots; ++i)
      for (cudaEvent_t e : {in_done[i], comp_done[i], out_done[i]})
        if (e) cudaEventDestroy(e);
    if (in) cudaStreamDestroy(in);
    if (out) cudaStreamDestroy(out);
    if (comp) cudaStreamDestroy(comp);
  }
};

// Chunk k: its Q, K, V are copied in on `in` (once the slot's previous chunk has
// been computed), computed on compute stream k % 2 (the caller's stream or the
// side compute stream; once its inputs are in and the slot's previous O has been
// copied out), and its O copied out on `out`.  Copy in, compute and copy out of
// consecutive chunks overlap, and so do the kernels of two consecutive chunks (the
// next chunk's CTAs fill the SMs that the last wave of the previous one leaves).
had_status host_attention(const void* Q, const void* K, const void* V, const had_shape* s,
                          const had_relpos_bias* bias, const float* alpha_q, const float* alpha_k, int N,
                          had_mode mode, void* O, had_dtype o_dtype, int chunk_b, void* workspace, size_t ws_bytes,
                          cudaStream_t st) {
  HostPlan p;
  had_status r = host_plan(s, mode, bias, chunk_b, &p);
  if (r != HAD_OK) return r;
  if (!Q || !K || !V || !O || (o_dtype != HAD_F32 && o_dtype != HAD_BF16)) return HAD_ERR_INVALID;
  if (N < 0 || !mode_ok(mode)) return HAD_ERR_INVALID;
  if (!workspace || ws_bytes < p.total || !aligned16(workspace)) return HAD_ERR_INVALID;
  for (int h = 0; alpha_q && h < s->H; ++h)
    if (!(alpha_q[h] > 0.0f) || !std::isfinite(alpha_q[h])) return HAD_ERR_INVALID;
  for (int h = 0; alpha_k && h < s->H; ++h)
    if (!(alpha_k[h] > 0.0f) || !std::isfinite(alpha_k[h])) return HAD_ERR_INVALID;
  for (int b = 0; s->seqlens && b < s->B; ++b)
    if (s->seqlens[b] < 1 || s->seqlens[b] > s->n) return HAD_ERR_INVALID;
  const bool has_bias = bias && bias->table;
  char* ws = static_cast<char*>(workspace);
  auto cu = [](cudaError_t e, const char* what) { return e == cudaSuccess ? HAD_OK : cuda_fail(e, what); };

  HostStreams hs;
  hs.main = st;
  const bool two = p.chunks > 1;  // a second compute stream only when there are chunks to overlap
  if ((r = cu(cudaStreamCreateWithFlags(&hs.in, cudaStreamNonBlocking), "cudaStreamCreateWithFlags")) != HAD_OK ||
      (r = cu(cudaStreamCreateWithFlags(&hs.out, cudaStreamNonBlocking), "cudaStreamCreateWithFlags")) != HAD_OK)
    return r;
  if (two && (r = cu(cudaStreamCreateWithFlags(&hs.comp, cudaStreamNonBlocking), "cudaStreamCreateWithFlags")) !=
                 HAD_OK)
    return r;
  for (cudaEvent_t* e : {&hs.start, &hs.join_in, &hs.join_out, &hs.join_comp})
    if ((r = cu(cudaEventCreateWithFlags(e, cudaEventDisableTiming), "cudaEventCreateWithFlags")) != HAD_OK) return r;
  for (int i = 0; i < p.slots; ++i)
    for (cudaEvent_t* e : {&hs.in_done[i], &hs.comp_done[i], &hs.out_done[i]})
      if ((r = cu(cudaEventCreateWithFlags(e, cudaEventDisableTiming), "cudaEventCreateWithFlags")) != HAD_OK)
        return r;
  // the side streams start behind the work already on the caller's stream
  if ((r = cu(cudaEventRecord(hs.start, st), "cudaEventRecord")) != HAD_OK ||
      (r = cu(cudaStreamWaitEvent(hs.in, hs.start, 0), "cudaStreamWaitEvent")) != HAD_OK ||
      (r = cu(cudaStreamWaitEvent(hs.out, hs.start, 0), "cudaStreamWaitEvent")) != HAD_OK)
    return r;
  if (two && (r = cu(cudaStreamWaitEvent(hs.comp, hs.start, 0), "cudaStreamWaitEvent")) != HAD_OK) return r;
  const cudaStream_t comp[kHostCompute] = {st, two ? hs.comp : st};
  const int32_t* dseq = nullptr;
  if (s->seqlens) {
    int32_t* d = reinterpret_cast<int32_t*>(ws + p.seq);
    if ((r = cu(cudaMemcpyAsync(d, s->seqlens, (size_t)s->B * sizeof(int32_t), cudaMemcpyHostToDevice, hs.in),
                "cudaMemcpyAsync(seqlens)")) != HAD_OK)
      return r;
    dseq = d;
  }
  had_relpos_bias bdev{};
  if (has_bias) {
    float* d = reinterpret_cast<float*>(ws + p.tab);
    if ((r = cu(cudaMemcpyAsync(d, bias->table, p.tab_bytes, cudaMemcpyHostToDevice, hs.in),
                "cudaMemcpyAsync(bias table)")) != HAD_OK)
      return r;
    bdev = *bias;
    bdev.table = d;
  }
  const char* hq = static_cast<const char*>(Q);
  const char* hk = static_cast<const char*>(K);
  const char* hv = static_cast<const char*>(V);
  char* ho = static_cast<char*>(O);
  const size_t head_ob = (size_t)s->n * s->d * (o_dtype == HAD_BF16 ? 2 : 4);
  const size_t tab_head = !has_bias ? 0
                          : bias->dense ? (size_t)s->n * s->n
                                        : (size_t)(2 * bias->gh - 1) * (2 * bias->gw - 1);
  for (int k = 0; k < p.chunks; ++k) {
    const int g = k % p.hgroups, b0 = (k / p.hgroups) * p.cb, nb = std::min(p.cb, s->B - b0);
    const int h0 = g * p.hc, nh = std::min(p.hc, s->H - h0), sl = k % p.slots;
    const cudaStream_t cs = comp[k % kHostCompute];
    char* slot = ws + p.slot0 + (size_t)sl * p.slot_bytes;
    // a chunk is whole sequences (h0 = 0, nh = H) or one sequence's heads h0 .. h0 + nh - 1: contiguous either way
    const size_t in_off = (size_t)b0 * p.in_b + (size_t)h0 * p.head_b, in_bytes = (size_t)nb * nh * p.head_b;
    const size_t o_off = ((size_t)b0 * s->H + h0) * head_ob, o_bytes = (size_t)nb * nh * head_ob;
    if (k >= p.slots && (r = cu(cudaStreamWaitEvent(hs.in, hs.comp_done[sl], 0), "cudaStreamWaitEvent")) != HAD_OK)
      return r;
    if ((r = cu(cudaMemcpyAsync(slot + p.q, hq + in_off, in_bytes, cudaMemcpyHostToDevice, hs.in), "cudaMemcpyAsync(Q)")) != HAD_OK ||
        (r = cu(cudaMemcpyAsync(slot + p.k, hk + in_off, in_bytes, cudaMemcpyHostToDevice, hs.in), "cudaMemcpyAsync(K)")) != HAD_OK ||
        (r = cu(cudaMemcpyAsync(slot + p.v, hv + in_off, in_bytes, cudaMemcpyHostToDevice, hs.in), "cudaMemcpyAsync(V)")) != HAD_OK ||
        (r = cu(cudaEventRecord(hs.in_done[sl], hs.in), "cudaEventRecord")) != HAD_OK ||
        (r = cu(cudaStreamWaitEvent(cs, hs.in_done[sl], 0), "cudaStreamWaitEvent")) != HAD_OK)
      return r;
    if (k >= p.slots && (r = cu(cudaStreamWaitEvent(cs, hs.out_done[sl], 0), "cudaStreamWaitEvent")) != HAD_OK)
      return r;
    had_shape csh = *s;
    csh.B = nb;
    csh.H = nh;
    csh.seqlens = dseq ? dseq + b0 : nullptr;
    had_relpos_bias cb = bdev;
    if (has_bias) cb.table = bdev.table + (size_t)h0 * tab_head;
    r = run_attention<EXP_NONE>(slot + p.q, slot + p.k, slot + p.v, &csh, has_bias ? &cb : nullptr,
                                alpha_q ? alpha_q + h0 : nullptr, alpha_k ? alpha_k + h0 : nullptr, N, mode,
                                slot + p.o, o_dtype, nullptr, nullptr, 0, 0, slot + p.ws, p.ws_bytes, cs);
    if (r != HAD_OK) return r;
    if ((r = cu(cudaEventRecord(hs.comp_done[sl], cs), "cudaEventRecord")) != HAD_OK ||
        (r = cu(cudaStreamWaitEvent(hs.out, hs.comp_done[sl], 0), "cudaStreamWaitEvent")) != HAD_OK ||
        (r = cu(cudaMemcpyAsync(ho + o_off, slot + p.o, o_bytes, cudaMemcpyDeviceToHost, hs.out), "cudaMemcpyAsync(O)")) != HAD_OK ||
        (r = cu(cudaEventRecord(hs.out_done[sl], hs.out), "cudaEventRecord")) != HAD_OK)
      return r;
  }
  return HAD_OK;
}

}  // namespace
}  // namespace had

using namespace had;

extern "C" {

size_t had_binarize_pack_workspace_size(const had_shape* s) {
  if (check_shape(s, true) != HAD_OK) return 0;
  Dims d = dims_of(s);
  return align_up((size_t)2 * d.BH * d.nchunks * d.d * 8);
}

had_status had_binarize_pack(const void* X, const had_shape* s, const float* mu_in, float* mu_out, uint32_t* bits,
                             void* workspace, size_t ws_bytes, void* stream) {
  had_status r = check_shape(s, true);
  if (r != HAD_OK) return r;
  if (!X || !bits || !aligned16(X) || (reinterpret_cast<uintptr_t>(bits) & 3u)) return HAD_ERR_INVALID;
  if ((mu_in && (reinterpret_cast<uintptr_t>(mu_in) & 3u)) || (mu_out && (reinterpret_cast<uintptr_t>(mu_out) & 3u)))
    return HAD_ERR_INVALID;
  if (!mu_in && (!workspace || ws_bytes < had_binarize_pack_workspace_size(s) || !aligned16(workspace)))
    return HAD_ERR_INVALID;
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
  unsigned* status = status_ptr(dev);
  if (!status) return cuda_fail(cudaErrorInvalidSymbol, "status word");
  return launch_prep(s, X, nullptr, nullptr, 0, 1, static_cast<double*>(workspace), nullptr, mu_in, mu_out, bits,
                     nullptr, nullptr, nullptr, nullptr, nullptr, static_cast<cudaStream_t>(stream), status);
}

size_t had_attention_workspace_size(const had_shape* s, int N, had_mode mode, const had_relpos_bias* bias) {
  (void)N;
  if (check_shape(s, true) != HAD_OK || check_bias(s, bias) != HAD_OK) return 0;
  return ws_layout(s, vbits_of(mode), bias).total;
}

had_status had_attention(const void* Q, const void* K, const void* V, const had_shape* s,
                         const had_relpos_bias* bias, const float* alpha_q, const float* alpha_k, int N,
                         had_mode mode, void* O, had_dtype o_dtype, void* workspace, size_t ws_bytes, void* stream) {
  return run_attention<EXP_NONE>(Q, K, V, s, bias, alpha_q, alpha_k, N, mode, O, o_dtype, nullptr, nullptr, 0, 0,
                                 workspace, ws_bytes, stream);
}

size_t had_attention_host_workspace_size(const had_shape* s, int N, had_mode mode, const had_relpos_bias* bias,
                                         int chunk_b) {
  (void)N;
  HostPlan p;
  return host_plan(s, mode, bias, chunk_b, &p) == HAD_OK ? p.total : 0;
}

had_status had_attention_host(const void* Q, const void* K, const void* V, const had_shape* s,
                              const had_relpos_bias* bias, const float* alpha_q, const float* alpha_k, int N,
                              had_mode mode, void* O, had_dtype o_dtype, int chunk_b, void* workspace,
                              size_t ws_bytes, void* stream) {
  return host_attention(Q, K, V, s, bias, alpha_q, alpha_k, N, mode, O, o_dtype, chunk_b, workspace, ws_bytes,
                        static_cast<cudaStream_t>(stream));
}

had_status had_attention_prepare(const void* Q, const void* K, const void* V, const had_shape* s,
                                 const had_relpos_bias* bias, int N, had_mode mode, void* workspace, size_t ws_bytes,
                                 void* stream) {
  had_status r = validate_attention<EXP_NONE>(Q, K, V, s, bias, nullptr, nullptr, N, mode, nullptr, HAD_F32, nullptr,
                                              nullptr, 0, 0, workspace, ws_bytes, true, false);
  if (r != HAD_OK) return r;
  unsigned* status = nullptr;
  if ((r = device_status_ptr(&status)) != HAD_OK) return r;
  return prepare_stage(Q, K, V, s, bias, N, mode, true, workspace, static_cast<cudaStream_t>(stream), status);
}

had_status had_attention_prepared(const void* V, const had_shape* s, const had_relpos_bias* bias,
                                  const float* alpha_q, const float* alpha_k, int N, had_mode mode, void* O,
                                  had_dtype o_dtype, void* workspace, size_t ws_bytes, void* stream) {
  had_status r = validate_attention<EXP_NONE>(nullptr, nullptr, V, s, bias, alpha_q, alpha_k, N, mode, O, o_dtype,
                                              nullptr, nullptr, 0, 0, workspace, ws_bytes, false, true);
  if (r != HAD_OK) return r;
  unsigned* status = nullptr;
  if ((r = device_status_ptr(&status)) != HAD_OK) return r;
  return attend_stage<EXP_NONE>(V, s, bias, alpha_q, alpha_k, N, mode, O, o_dtype, nullptr, nullptr, 0, 0, workspace,
                                static_cast<cudaStream_t>(stream), status);
}

size_t had_qkv_workspace_size(const had_shape* s, int Dm, int N, had_mode mode, const had_relpos_bias* bias) {
  (void)N;
  if (check_qkv_shape(s, Dm) != HAD_OK || check_bias(s, bias) != HAD_OK || !mode_ok(mode)) return 0;
  return qkv_ws_layout(s, Dm, vbits_of(mode), bias).total;
}

had_status had_qkv_prepare(const void* X, const void* Wqkv, const had_shape* s, int Dm, const had_relpos_bias* bias,
                           int N, had_mode mode, void* V_out, void* workspace, size_t ws_bytes, void* stream) {
  had_status r = check_qkv_shape(s, Dm);
  if (r != HAD_OK) return r;
  if ((r = check_bias(s, bias)) != HAD_OK) return r;
  if (N < 0 || !mode_ok(mode)) return HAD_ERR_INVALID;
  if (!X || !Wqkv || !V_out || !aligned16(X) || !aligned16(Wqkv) || !aligned16(V_out)) return HAD_ERR_INVALID;
  const int vbits = vbits_of(mode);
  const QkvWs q = qkv_ws_layout(s, Dm, vbits, bias);
  if (!workspace || ws_bytes < q.total || !aligned16(workspace)) return HAD_ERR_INVALID;
  unsigned* status = nullptr;
  if ((r = device_status_ptr(&status)) != HAD_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const Ws w = ws_layout(s, vbits, bias);
  Dims d = dims_of(s);
  const __nv_bfloat16* Xb = static_cast<const __nv_bfloat16*>(X);
  const __nv_bfloat16* Wb = static_cast<const __nv_bfloat16*>(Wqkv);
  {
    static std::mutex smu;
    static bool configured[kMaxDevices] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(smu);
    if (dev >= 0 && dev < kMaxDevices && !configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(qkv::k_qkv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           qkv::QkvSmem::kTotal);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(k_qkv_tc)");
      configured[dev] = true;
    }
  }
  double* xpart = reinterpret_cast<double*>(ws + q.xpart);
  double* mupart = reinterpret_cast<double*>(ws + q.mu);
  // the means of Q and K from X's token means
  uint32_t* vamax = reinterpret_cast<uint32_t*>(ws + q.vamax);
  qkv::k_xsum<<<dim3((Dm / 8 + qkv::kXsumThreads - 1) / qkv::kXsumThreads, q.nch, d.B),
                  qkv::kXsumThreads * qkv::kXsumGroups, 0, st>>>(Xb, d.n, Dm, d.H, s->seqlens, q.nch, xpart,
                                                                  vbits != 0 ? vamax : nullptr);
  if ((r = check_launch("k_xsum")) != HAD_OK) return r;
  qkv::k_mu<<<dim3((2 * d.H * 64 + qkv::kMuO - 1) / qkv::kMuO, (d.B + qkv::kMuB - 1) / qkv::kMuB, qkv::kMuSplit),
              qkv::kMuThreads, 0, st>>>(Wb, xpart, q.nch, d.n, s->seqlens, d.B, d.H, Dm, mupart);
  if ((r = check_launch("k_mu")) != HAD_OK) return r;
  // the projection, binarized in its epilogue, into the attention workspace
  qkv::QkvArgs qa;
  memset(&qa, 0, sizeof(qa));
  if ((r = encode_2d(&qa.tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, Dm, (uint64_t)d.B * d.n, (uint64_t)Dm * 2, 64,
                     qkv::kM, CU_TENSOR_MAP_SWIZZLE_128B)) != HAD_OK)
    return r;
  if ((r = encode_2d(&qa.tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Wqkv, Dm, (uint64_t)3 * d.H * 64, (uint64_t)Dm * 2,
                     64, qkv::kN, CU_TENSOR_MAP_SWIZZLE_128B)) != HAD_OK)
    return r;
  qa.B = d.B; qa.H = d.H; qa.n = d.n; qa.n_pad = d.n_pad; qa.Dm = Dm;
  qa.seqlens = s->seqlens;
  qa.mupart = mupart;
  qa.qbits = reinterpret_cast<uint32_t*>(ws + w.qbits);
  qa.kpm = reinterpret_cast<int8_t*>(ws + w.kpm);
  qa.k_e4m3 = select_kind(s, bias, N) == SEL_TOPN_FLOAT ? 1 : 0;  // the fp8 score path's +-1 encoding
  qa.V = static_cast<__nv_bfloat16*>(V_out);
  qa.vamax = vbits != 0 ? vamax : nullptr;
  qa.status = status;
  qkv::k_qkv_tc<<<dim3((d.n + qkv::kM - 1) / qkv::kM, d.B, (3 * d.H + qkv::kNB - 1) / qkv::kNB), qkv::kThreads,
                   qkv::QkvSmem::kTotal, st>>>(qa);
  if ((r = check_launch("k_qkv_tc")) != HAD_OK) return r;
  // the bias tables and, in the uint8 modes, the quantized V^T (scales from the epilogue's absmax), as the
  // attention's prepare stage makes them
  if (bias && bias->table &&
      (r = build_bias_tables(s, bias, ws + w.bminmax, ws + w.bext, ws + w.expb, st)) != HAD_OK)
    return r;
  if (vbits != 0) {
    qkv::k_vcodes<<<dim3(d.n_pad / 64, d.BH), qkv::kVcThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(V_out), vamax, d.H, d.n, d.n_pad, s->seqlens, vbits,
        reinterpret_cast<int8_t*>(ws + w.vqT), reinterpret_cast<float*>(ws + w.vscale));
    if ((r = check_launch("k_vcodes")) != HAD_OK) return r;
  }
  return HAD_OK;
}

had_status had_topn_indices(const void* Q, const void* K, const had_shape* s, const had_relpos_bias* bias,
                            const float* alpha_q, const float* alpha_k, int N, int32_t* idx, void* workspace,
                            size_t ws_bytes, void* stream) {
  return run_attention<EXP_IDX>(Q, K, nullptr, s, bias, alpha_q, alpha_k, N, HAD_MODE_FLOAT, nullptr, HAD_F32, idx,
                                nullptr, 0, 0, workspace, ws_bytes, stream);
}

had_status had_attention_scores(const void* Q, const void* K, const had_shape* s, int32_t* S, void* workspace,
                                size_t ws_bytes, void* stream) {
  return run_attention<tc::EXP_SCORES>(Q, K, nullptr, s, nullptr, nullptr, nullptr, 0, HAD_MODE_FLOAT, nullptr,
                                       HAD_F32, S, nullptr, 0, 0, workspace, ws_bytes, stream);
}

had_status had_debug_bounded_wait(long long max_cycles, int force_expiry) {
  if (max_cycles < 0 || (max_cycles > 0 && max_cycles < 10000)) return HAD_ERR_INVALID;
  g_wait_cycles.store(max_cycles == 0 ? tc::kWaitCycles : max_cycles);
  g_force_expiry.store(force_expiry ? 1 : 0);
  return HAD_OK;
}

had_status had_attention_codes_u8(const void* Q, const void* K, const void* V, const had_shape* s,
                                  const had_relpos_bias* bias, const float* alpha_q, const float* alpha_k, int N,
                                  int row_begin, int row_end, uint8_t* A, void* workspace, size_t ws_bytes,
                                  void* stream) {
  return run_attention<EXP_CODES>(Q, K, V, s, bias, alpha_q, alpha_k, N, HAD_MODE_U8I8, nullptr, HAD_F32, nullptr, A,
                                  row_begin, row_end, workspace, ws_bytes, stream);
}

namespace {

// Shared body of had_quantize_v (8-bit) and had_quantize_v4 (4-bit).
had_status quantize_v_bits(const void* V, const had_shape* s, int vbits, int8_t* Vq, float* vscale, void* workspace,
                           size_t ws_bytes, void* stream) {
  had_status r = check_shape(s, true);
  if (r != HAD_OK) return r;
  if (!V || !Vq || !vscale || !aligned16(V) || (reinterpret_cast<uintptr_t>(vscale) & 3u)) return HAD_ERR_INVALID;
  const Ws w = ws_layout(s, vbits, nullptr);
  if (!workspace || ws_bytes < w.total || !aligned16(workspace)) return HAD_ERR_INVALID;
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
  unsigned* status = status_ptr(dev);
  if (!status) return cuda_fail(cudaErrorInvalidSymbol, "status word");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Dims d = dims_of(s);
  int8_t* vqT = reinterpret_cast<int8_t*>(ws + w.vqT);
  r = launch_prep(s, nullptr, nullptr, V, 2, 1, reinterpret_cast<double*>(ws + w.sums),
                  reinterpret_cast<float*>(ws + w.amax), nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, vqT,
                  vscale, st, status, vbits);
  if (r != HAD_OK) return r;
  k_untranspose_vq<<<1024, 256, 0, st>>>(vqT, d.BH, d.n, d.d, d.n_pad, vbits, Vq);
  return check_launch("k_untranspose_vq");
}

}  // namespace

had_status had_quantize_v(const void* V, const had_shape* s, int8_t* Vq, float* vscale, void* workspace,
                          size_t ws_bytes, void* stream) {
  return quantize_v_bits(V, s, 8, Vq, vscale, workspace, ws_bytes, stream);
}

had_status had_quantize_v4(const void* V, const had_shape* s, int8_t* Vq, float* vscale, void* workspace,
                           size_t ws_bytes, void* stream) {
  return quantize_v_bits(V, s, 4, Vq, vscale, workspace, ws_bytes, stream);
}

size_t had_dense_reference_workspace_size(const had_shape* s, const had_relpos_bias* bias) {
  if (check_shape(s) != HAD_OK || check_bias(s, bias) != HAD_OK) return 0;
  return ref_ws_layout(s, bias).total;
}

had_status had_dense_reference_mode(const void* Q, const void* K, const void* V, const had_shape* s,
                                    const had_relpos_bias* bias, int N, void* O, had_dtype o_dtype,
                                    void* workspace, size_t ws_bytes, void* stream) {
  had_status r = check_shape(s);
  if (r != HAD_OK) return r;
  if ((r = check_bias(s, bias)) != HAD_OK) return r;
  if (s->in_dtype != HAD_BF16) return HAD_ERR_UNSUPPORTED;
  if (N < 0) return HAD_ERR_INVALID;
  if (N != 0 && N < s->n) return HAD_ERR_UNSUPPORTED;
  if (!Q || !K || !V || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return HAD_ERR_INVALID;
  if (o_dtype != HAD_F32 && o_dtype != HAD_BF16) return HAD_ERR_INVALID;
  const RefWs w = ref_ws_layout(s, bias);
  if (w.total > 0 && (!workspace || ws_bytes < w.total || !aligned16(workspace))) return HAD_ERR_INVALID;
  unsigned* status = nullptr;
  if ((r = device_status_ptr(&status)) != HAD_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const bool has_bias = bias && bias->table;
  if (has_bias && (r = build_bias_tables(s, bias, ws + w.bminmax, ws + w.bext, ws + w.expb, st)) != HAD_OK) return r;
  const Dims d = dims_of(s);
  tc::TcArgs a;
  memset(&a, 0, sizeof(a));
  // raw bf16 Q, K, V in 64-channel panels of 128 bytes (128-byte swizzle)
  if ((r = encode_2d(&a.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, d.d, (uint64_t)d.BH * d.n, d.d * 2, 64, tc::kM,
                     CU_TENSOR_MAP_SWIZZLE_128B)) != HAD_OK ||
      (r = encode_2d(&a.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, d.d, (uint64_t)d.BH * d.n, d.d * 2, 64, tc::kN,
                     CU_TENSOR_MAP_SWIZZLE_128B)) != HAD_OK ||
      (r = encode_2d(&a.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, V, d.d, (uint64_t)d.BH * d.n, d.d * 2, 64, tc::kN,
                     CU_TENSOR_MAP_SWIZZLE_128B)) != HAD_OK)
    return r;
  bool rows = false;
  const int bias_kind = fill_bias_args(a, s, bias, ws + w.bminmax, ws + w.bext, ws + w.expb, &rows);
  a.v_raw = V;
  a.seqlens = s->seqlens;
  a.O = O; a.o_bf16 = (o_dtype == HAD_BF16) ? 1 : 0;
  a.wait_cycles = g_wait_cycles.load();
  a.force_expiry = g_force_expiry.load();
  a.B = d.B; a.H = d.H; a.n = d.n; a.n_pad = d.n_pad; a.N = 0;
  a.status = status;
  a.koff_mode = (d.n_pad <= tc::kKoffTableMax) ? tc::kKoffTable : tc::kKoffWarp;
  const float c = (float)(1.0 / std::sqrt((double)s->d));  // standard attention: l = q.k / sqrt(d) + b
  for (int h = 0; h < s->H; ++h) a.c_head[h] = c;
  dim3 grid((s->n + tc::kM - 1) / tc::kM, d.BH);
  if (s->d == 128) return launch::dispatch_ref<128>(bias_kind, a, grid, st);
  return launch::dispatch_ref<64>(bias_kind, a, grid, st);
}

had_status had_scores_int(const uint32_t* qbits, const uint32_t* kbits, const had_shape* s, int32_t* S,
                          void* stream) {
  had_status r = check_shape(s);
  if (r != HAD_OK) return r;
  if (s->d != 64) return HAD_ERR_UNSUPPORTED;
  if (!qbits || !kbits || !S || (reinterpret_cast<uintptr_t>(qbits) & 7u) || (reinterpret_cast<uintptr_t>(kbits) & 7u) ||
      (reinterpret_cast<uintptr_t>(S) & 3u))
    return HAD_ERR_INVALID;
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
  unsigned* status = status_ptr(dev);
  if (!status) return cuda_fail(cudaErrorInvalidSymbol, "status word");
  Dims d = dims_of(s);
  dim3 grid((s->n + kQT - 1) / kQT, d.BH);
  k_scores_int<KMAP_U8><<<grid, kAttnThreads, 0, static_cast<cudaStream_t>(stream)>>>(qbits, kbits, s->H, s->n,
                                                                                      s->seqlens, S, status);
  return check_launch("k_scores_int");
}

}  // extern "C"

// ---------------------------------------------------------------------------- no-allocation variant
//
// Scratch for had_binarize_pack_noalloc: the fp64 per-chunk channel sums that
// had_binarize_pack keeps in the caller's workspace live here instead, in a
// fixed array that every GPU loading this library holds until the process
// exits.  In host code `g_pack_scratch` only names a host-side stand-in; the
// device address comes from cudaGetSymbolAddress, taken once per device.
namespace had {
namespace {

constexpr size_t kPackScratchBytes = (size_t)4 << 20;  // 4 MiB: B*H*ceil(n/64) <= 8192
__device__ __align__(256) unsigned char g_pack_scratch[kPackScratchBytes];

had_status pack_scratch_ptr(double** out) {
  static std::mutex mu;
  static double* ptrs[kMaxDevices] = {nullptr};
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    snprintf(t_last_error, sizeof(t_last_error), "had_binarize_pack_noalloc: device index %d is beyond the %d "
             "devices the library tracks", dev, kMaxDevices);
    return HAD_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    ce = cudaGetSymbolAddress(&p, g_pack_scratch);  // with `dev` current
    if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetSymbolAddress(g_pack_scratch)");
    ptrs[dev] = static_cast<double*>(p);
  }
  *out = ptrs[dev];
  return HAD_OK;
}

}  // namespace
}  // namespace had

extern "C" {

had_status had_binarize_pack_noalloc(const void* X, const had_shape* s, float* mu_out, uint32_t* bits,
                                     void* stream) {
  had_status r = check_shape(s, true);
  if (r != HAD_OK) return r;
  if (!X || !bits || !aligned16(X) || (reinterpret_cast<uintptr_t>(bits) & 3u)) return HAD_ERR_INVALID;
  if (mu_out && (reinterpret_cast<uintptr_t>(mu_out) & 3u)) return HAD_ERR_INVALID;
  const Dims d = dims_of(s);
  const size_t need = (size_t)d.BH * d.nchunks * d.d * sizeof(double);
  if (need > kPackScratchBytes) {
    snprintf(t_last_error, sizeof(t_last_error),
             "had_binarize_pack_noalloc: B*H*ceil(n/64)*d/64 = %lld exceeds the static scratch limit of %lld",
             (long long)d.BH * d.nchunks * d.d / 64, (long long)(kPackScratchBytes / (64 * sizeof(double))));
    return HAD_ERR_UNSUPPORTED;
  }
  double* scratch = nullptr;
  if ((r = pack_scratch_ptr(&scratch)) != HAD_OK) return r;
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
  unsigned* status = status_ptr(dev);
  if (!status) return cuda_fail(cudaErrorInvalidSymbol, "status word");
  // k_stats writes every partial sum k_pack reads, so no part of the scratch needs clearing.
  return launch_prep(s, X, nullptr, nullptr, 0, 1, scratch, nullptr, nullptr, mu_out, bits, nullptr, nullptr, nullptr,
                     nullptr, nullptr, static_cast<cudaStream_t>(stream), status);
}

had_status had_probe_mma_rate(int kind, int iters, double* tops, double* ms) {
  if ((kind != 0 && kind != 1) || iters < 2 || iters > (1 << 22) || !tops) return HAD_ERR_INVALID;
  int dev = 0, sms = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
  if ((ce = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return cuda_fail(ce, "cudaDeviceGetAttribute");
  unsigned* status = status_ptr(dev);
  if (!status) return cuda_fail(cudaErrorInvalidSymbol, "status word");
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if ((ce = cudaEventCreate(&e0)) != cudaSuccess || (ce = cudaEventCreate(&e1)) != cudaSuccess) {
    if (e0) cudaEventDestroy(e0);
    return cuda_fail(ce, "cudaEventCreate");
  }
  had_status r = HAD_OK;
  float t = 0.0f;
  // a short launch first (clocks up, code loaded), then the timed one
  probe::k_probe_mma<<<sms, probe::kThreads, probe::kSmemTotal, 0>>>(kind, iters / 8 + 2, status);
  cudaEventRecord(e0, 0);
  probe::k_probe_mma<<<sms, probe::kThreads, probe::kSmemTotal, 0>>>(kind, iters, status);
  cudaEventRecord(e1, 0);
  if ((r = check_launch("k_probe_mma")) == HAD_OK) {
    if ((ce = cudaEventSynchronize(e1)) != cudaSuccess || (ce = cudaEventElapsedTime(&t, e0, e1)) != cudaSuccess)
      r = cuda_fail(ce, "probe timing");
  }
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (r != HAD_OK) return r;
  const double k = kind == 0 ? 32.0 : 16.0;  // K elements per MMA
  const double ops = 2.0 * probe::kM * probe::kN * k * (double)iters * (double)sms;
  *tops = ops / ((double)t * 1e-3) / 1e12;
  if (ms) *ms = t;
  return HAD_OK;
}

had_status had_get_device_status(void) {
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
  if ((ce = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(ce, "cudaDeviceSynchronize");
  unsigned v = 0, zero = 0;
  if ((ce = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v))) != cudaSuccess) return cuda_fail(ce, "read status");
  if ((ce = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero))) != cudaSuccess) return cuda_fail(ce, "clear status");
  if (v & kDevErrTimeout) return HAD_ERR_TIMEOUT;
  if (v) return HAD_ERR_DEVICE;
  return HAD_OK;
}

const char* had_status_string(had_status st) {
  switch (st) {
    case HAD_OK: return "HAD_OK";
    case HAD_ERR_INVALID: return "HAD_ERR_INVALID: invalid argument";
    case HAD_ERR_UNSUPPORTED: return "HAD_ERR_UNSUPPORTED: shape, dtype or mode not supported";
    case HAD_ERR_CUDA: return "HAD_ERR_CUDA: CUDA call failed";
    case HAD_ERR_DEVICE: return "HAD_ERR_DEVICE: device-detected error (bad seqlens or candidate overflow)";
    case HAD_ERR_TIMEOUT: return "HAD_ERR_TIMEOUT: a bounded device wait expired";
  }
  return "unknown had_status";
}

const char* had_last_cuda_error(void) { return t_last_error; }

int had_version(void) { return 100; }

}  // extern "C"

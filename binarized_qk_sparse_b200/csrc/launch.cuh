// launch.cuh -- host-side launch of the fused kernel's instantiations, for one
// head dim D per translation unit (had_lib.cu builds D = 64, attn_d128.cu D = 128,
// so the two compile in parallel).  dispatch_tc<D, EXP> picks the instantiation
// from the select kind, mode (float, int8 or 4-bit V), bias layout and V dtype.
#pragma once

#include <mutex>

#include "../../include/had.h"
#include "attn_tc.cuh"

namespace had {

constexpr int kMaxDevices = 64;
// Both defined in had_lib.cu: record a CUDA error for had_last_cuda_error() and
// return HAD_ERR_CUDA; check the last launch.
had_status cuda_fail(cudaError_t e, const char* what);
had_status check_launch(const char* what);

namespace launch {

template <int D, int SEL, int MODE, int BIAS, bool VF32, int EXP, int SPLIT>
had_status launch_tc_t(const tc::TcArgs& a, dim3 grid, cudaStream_t st) {
  // head dim 128 allocates 512 TMEM columns: ask for enough shared memory that a
  // second CTA never shares the SM (its allocation would wait for the first)
  constexpr int kSmem = tc::Smem<D, SEL, VF32, BIAS>::kTotal;
  const int smem = (tc::ctas_per_sm(D) == 1 && kSmem < 120 * 1024) ? 120 * 1024 : kSmem;
  auto fn = tc::k_attn_tc<D, SEL, MODE, BIAS, VF32, EXP, SPLIT>;
  static std::mutex mu;
  static bool configured[kMaxDevices] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 0 && dev < kMaxDevices && !configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(k_attn_tc)");
      configured[dev] = true;
    }
  }
  fn<<<grid, tc::cta_threads(SPLIT), smem, st>>>(a);
  return check_launch("k_attn_tc");
}

// Dense: no bias, extended tables in global memory, the exp(bias) table staged in
// shared memory, or a dense bias matrix read 4 keys per load.
template <int D, int SEL, int MODE, bool VF32, int EXP>
had_status launch_tc_b(int bias, const tc::TcArgs& a, dim3 grid, cudaStream_t st) {
  using namespace tc;
  if (bias == BIAS_SMEM) return launch_tc_t<D, SEL, MODE, BIAS_SMEM, VF32, EXP, 2>(a, grid, st);
  if (bias == BIAS_ROWS) return launch_tc_t<D, SEL, MODE, BIAS_ROWS, VF32, EXP, 2>(a, grid, st);
  if (bias == BIAS_DGLOBAL) return launch_tc_t<D, SEL, MODE, BIAS_DGLOBAL, VF32, EXP, 2>(a, grid, st);
  if (bias == BIAS_GLOBAL) return launch_tc_t<D, SEL, MODE, BIAS_GLOBAL, VF32, EXP, 2>(a, grid, st);
  return launch_tc_t<D, SEL, MODE, BIAS_NONE, VF32, EXP, 2>(a, grid, st);
}

// Top-N without a bias: two threads per row on the P.V path of short ragged rows
// (per-sequence lengths, n <= 256), where a CTA's few tiles make it latency-bound;
// on full-length rows the per-tile tie exchange costs more than the extra warps gain.
template <int D, int SEL, int MODE, bool VF32, int EXP>
had_status launch_tc_n(const tc::TcArgs& a, dim3 grid, cudaStream_t st) {
  if (EXP == tc::EXP_NONE && a.n_pad <= tc::kSplitMaxKeys && a.seqlens != nullptr)
    return launch_tc_t<D, SEL, MODE, tc::BIAS_NONE, VF32, EXP, (EXP == tc::EXP_NONE ? 2 : 1)>(a, grid, st);
  return launch_tc_t<D, SEL, MODE, tc::BIAS_NONE, VF32, EXP, 1>(a, grid, st);
}

// Top-N with a bias: per-warp bias windows in shared memory (relative-position
// tables on grids with rows of a multiple of 64 patches and no class tokens), or
// gathers from the extended table in global memory.
template <int D, int MODE, bool VF32, int EXP>
had_status launch_tc_f(bool rows, const tc::TcArgs& a, dim3 grid, cudaStream_t st) {
  // float A.V: two threads per row (twice the softmax warps to hide latency)
  constexpr int SP = (MODE == tc::MODE_F && EXP == tc::EXP_NONE) ? 2 : 1;
  if (rows) return launch_tc_t<D, tc::SEL_TOPN_FLOAT, MODE, tc::BIAS_ROWS, VF32, EXP, SP>(a, grid, st);
  return launch_tc_t<D, tc::SEL_TOPN_FLOAT, MODE, tc::BIAS_GLOBAL, VF32, EXP, SP>(a, grid, st);
}

template <int D, int EXP>
had_status dispatch_tc(int sel, int mode, int bias, bool vf32, bool rows, const tc::TcArgs& a, dim3 grid,
                       cudaStream_t st) {
  using namespace tc;
  if (EXP == EXP_SCORES) return launch_tc_t<D, SEL_DENSE, MODE_F, BIAS_NONE, false, EXP_SCORES, 1>(a, grid, st);
  if constexpr (EXP == EXP_NONE) {  // 4-bit V: the output path only
    if (mode == MODE_Q4) {
      if (sel == SEL_DENSE) return launch_tc_b<D, SEL_DENSE, MODE_Q4, false, EXP>(bias, a, grid, st);
      if (sel == SEL_TOPN_INT) return launch_tc_n<D, SEL_TOPN_INT, MODE_Q4, false, EXP>(a, grid, st);
      return launch_tc_f<D, MODE_Q4, false, EXP>(rows, a, grid, st);
    }
  }
  if (EXP == EXP_CODES || (EXP == EXP_NONE && mode == MODE_Q)) {
    constexpr int E = EXP;
    if (sel == SEL_DENSE) return launch_tc_b<D, SEL_DENSE, MODE_Q, false, E>(bias, a, grid, st);
    if (sel == SEL_TOPN_INT) return launch_tc_n<D, SEL_TOPN_INT, MODE_Q, false, E>(a, grid, st);
    return launch_tc_f<D, MODE_Q, false, E>(rows, a, grid, st);
  }
  if (EXP == EXP_IDX) {
    if (sel == SEL_DENSE) return launch_tc_b<D, SEL_DENSE, MODE_F, false, EXP>(bias, a, grid, st);
    if (sel == SEL_TOPN_INT) return launch_tc_t<D, SEL_TOPN_INT, MODE_F, BIAS_NONE, false, EXP, 1>(a, grid, st);
    return launch_tc_f<D, MODE_F, false, EXP>(rows, a, grid, st);
  }
  if (vf32) {
    if (sel == SEL_DENSE) return launch_tc_b<D, SEL_DENSE, MODE_F, true, EXP>(bias, a, grid, st);
    if (sel == SEL_TOPN_INT) return launch_tc_n<D, SEL_TOPN_INT, MODE_F, true, EXP>(a, grid, st);
    return launch_tc_f<D, MODE_F, true, EXP>(rows, a, grid, st);
  }
  if (sel == SEL_DENSE) return launch_tc_b<D, SEL_DENSE, MODE_F, false, EXP>(bias, a, grid, st);
  if (sel == SEL_TOPN_INT) return launch_tc_n<D, SEL_TOPN_INT, MODE_F, false, EXP>(a, grid, st);
  return launch_tc_f<D, MODE_F, false, EXP>(rows, a, grid, st);
}

// The comparison mode (standard attention on the unbinarized inputs), dense only.
template <int D>
had_status dispatch_ref(int bias, const tc::TcArgs& a, dim3 grid, cudaStream_t st) {
  return launch_tc_b<D, tc::SEL_REF, tc::MODE_F, false, tc::EXP_NONE>(bias, a, grid, st);
}

}  // namespace launch

// The instantiations each translation unit provides.
#define HAD_DISPATCH_INST(KW, D)                                                                                   \
  KW template had_status launch::dispatch_tc<D, tc::EXP_NONE>(int, int, int, bool, bool, const tc::TcArgs&, dim3,  \
                                                              cudaStream_t);                                       \
  KW template had_status launch::dispatch_tc<D, tc::EXP_IDX>(int, int, int, bool, bool, const tc::TcArgs&, dim3,   \
                                                             cudaStream_t);                                        \
  KW template had_status launch::dispatch_tc<D, tc::EXP_CODES>(int, int, int, bool, bool, const tc::TcArgs&, dim3, \
                                                               cudaStream_t);                                      \
  KW template had_status launch::dispatch_tc<D, tc::EXP_SCORES>(int, int, int, bool, bool, const tc::TcArgs&, dim3, \
                                                                cudaStream_t);                                     \
  KW template had_status launch::dispatch_ref<D>(int, const tc::TcArgs&, dim3, cudaStream_t);

}  // namespace had

// prefill_sm100.h -- host-side interface of the prefill (multi-token, expanded form) kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace hra {

// Arguments of one prefill call (device pointers; layouts in hra.h and prefill_sm100.cu).
struct PrefillArgs {
  const __nv_bfloat16* q;      // [n, h, 192]
  const __nv_bfloat16* krope;  // rope rows, krope_stride elements apart
  long long krope_stride;
  __half* q16;                 // workspace: [n, h, 192] fp16 (alpha_q q_nope | rotated q_rope)
  __half* kr16;                // workspace: [l_pad, 64] fp16
  __half* k_exp;               // workspace: [n_branch, h, l_pad, 128] fp16
  __half* v_exp;               // workspace: [n_branch, h, l_pad, 128] fp16
  float* out_f32;              // [n, h, 128] or nullptr
  __nv_bfloat16* out_bf16;     // [n, h, 128] or nullptr
  int* status;                 // device status word
  int heads, n_branch, seq_len, n_query, l_pad;
  float alpha_q, alpha_kv, branch_scale, scale_log2, rope_theta;
  uint64_t wait_limit_ns;
};

// Tensor maps (fp16 ones over the workspace, bf16 ones over the inputs), 128-byte swizzle.
struct PrefillMaps {
  CUtensorMap ckv;   // bf16 [L, d_c], box {64, 128}
  CUtensorMap wuk;   // bf16 [h * 512, 128], box {64, 128}
  CUtensorMap wuv;   // bf16 [h * 512, 128], box {64, 128}
  CUtensorMap q16;   // fp16 [n, h * 192], box {64, 128}
  CUtensorMap k;     // fp16 [n_branch * h * l_pad, 128], box {64, 128}
  CUtensorMap v;     // fp16 [n_branch * h * l_pad, 128], box {64, 128}
  CUtensorMap kr16;  // fp16 [l_pad, 64], box {64, 128}
};

// prep -> expand -> attend on `stream`, chained with programmatic dependent launch.
cudaError_t launch_prefill(const PrefillMaps& m, const PrefillArgs& a, cudaStream_t stream);

}  // namespace hra

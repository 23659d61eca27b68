// absorb_combine.h -- host-side interface of the absorption and combine/up-projection kernels.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace hra {

struct AbsorbArgs {
  const __nv_bfloat16* q;     // [B, h, 192]
  const __nv_bfloat16* w_uk;  // [h, 512, 128]
  const int32_t* seq_lens;    // [B]
  __half* q_tilde;            // out: fp16 [B, h, 576], or (two_term) bf16 hi [B, h, 576] + bf16 lo [B, h, 576]
  int two_term;               // 1: store q~ as bf16 hi + bf16 lo (MLRA-4 kernel); 0: fp16
  int* status;                // cleared by this kernel (first kernel of a call)
  int batch, heads;
  float alpha_q, alpha_kv, rope_theta;
};

struct CombineArgs {
  const float* o_part;        // [slots, 4, 128, 128]
  const float2* ml_part;      // [slots, 4, 128]
  const int32_t* seq_lens;    // [B]
  const __nv_bfloat16* w_uv;  // [h, 512, 128]
  float* out_f32;             // [B, h, 128] or nullptr
  __nv_bfloat16* out_bf16;    // [B, h, 128] or nullptr
  int batch, heads, groups, tile_tokens;
  float alpha_kv, branch_scale;
};

cudaError_t launch_absorb_q(const AbsorbArgs& a, cudaStream_t stream);
cudaError_t launch_combine_upproj(const CombineArgs& a, cudaStream_t stream);

}  // namespace hra

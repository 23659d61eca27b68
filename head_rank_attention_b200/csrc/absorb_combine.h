// absorb_combine.h -- host-side interface of the absorption and combine/up-projection kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace hra {

struct AbsorbArgs {
  const __nv_bfloat16* q;     // [B, h, 192]
  const int32_t* seq_lens;    // [B]
  __half* q_tilde;            // out: fp16 [B, h, d_c + 64]: absorbed latent query | rotated rope part
  int* status;                // device status word (expired waits)
  int* tile_prefix;           // out: [B + 1] exclusive prefix of decode tiles per sequence
  int tile_tokens;            // decode tile size (tokens)
  int batch, heads;
  int d_c;                    // latent width: 512, or 256 / 128 (a shard of 128-wide branches)
  float alpha_q, alpha_kv, rope_theta;
  const int32_t* q_positions; // [B] query position per sequence, or nullptr: seq_lens[s] - 1
};

constexpr int kMaxOutPeers = 7;  // other ranks' out buffers the up-projection can add into

struct CombineArgs {
  const float* o_part;        // [slots, d_c / 128, 128, 128]
  const float2* ml_part;      // [slots, d_c / 128, 128]
  const int* tile_prefix;     // [B + 1], written by the absorb kernel
  __nv_bfloat16* o_lat;       // merged latent output, bf16 hi [h, B, d_c] then bf16 lo [h, B, d_c]
  const __nv_bfloat16* w_uv;  // [h, d_c, 128] (read directly by the small-batch combine)
  int* status;                // device status word (expired waits)
  float* out_f32;             // [B, h, 128] or nullptr
  __nv_bfloat16* out_bf16;    // [B, h, 128] or nullptr
  int accumulate;             // 1: add into out_f32 and every peers[k] (fp32 atomics) instead of storing
  int n_peers;
  float* peers[kMaxOutPeers]; // other ranks' out buffers (peer memory), [B, h, 128] fp32
  int batch, heads, groups;
  int d_c;                    // latent width (as in AbsorbArgs)
  int sms;                    // streaming multiprocessors of the device
  float alpha_kv, branch_scale;
  // partial mode: the merge writes fp32 [B, h, d_c] normalised latent rows and fp32
  // [B, h, d_c / 128] log2 softmax denominators here, and nothing runs after it
  float* part_o;
  float* part_lse;
  // hra_combine_partials: n_parts gathered states [n_parts, B, h, d_c] / [n_parts, B, h, d_c / 128]
  const float* parts_o;
  const float* parts_lse;
  int n_parts;
};

// Sequences per absorb CTA (the MMA's M); the q tensor map's box is {64, this} rows.
int absorb_seq_chunk(int batch);
// Rows of one o_lat box in the up-projection (its CTAs take 128 sequences in boxes of this many).
int upproj_seq_chunk();

// map_wuk: W_UK viewed as [h*d_c rows, 128] bf16, box {64, min(d_c, 256)}, SWIZZLE_128B.
// map_q:   q viewed as [B rows, h*192] bf16, box {64, absorb_seq_chunk(B)}, SWIZZLE_128B.
// pdl: launch with programmatic dependent launch (launch.h).
cudaError_t launch_absorb_q(const CUtensorMap& map_wuk, const CUtensorMap& map_q, const AbsorbArgs& a,
                            cudaStream_t stream, bool pdl);
// Batches of up to kSmallBatch sequences with few heads take one fused merge + up-projection
// kernel; the others the merge kernel and the tensor-core up-projection.
constexpr int kSmallBatch = 4;
// map_wuv:  W_UV viewed as [h*d_c rows, 128] bf16, box {64, 128}, SWIZZLE_128B.
// map_olat: a.o_lat viewed as [2*h*B rows, d_c] bf16, box {64, upproj_seq_chunk()}, SWIZZLE_128B.
cudaError_t launch_combine_upproj(const CUtensorMap& map_wuv, const CUtensorMap& map_olat, const CombineArgs& a,
                                  cudaStream_t stream, bool pdl);
// Merge a.n_parts gathered partial states (a.parts_o / a.parts_lse) into o_lat and run the
// up-projection (hra_combine_partials).
cudaError_t launch_combine_partials(const CUtensorMap& map_wuv, const CUtensorMap& map_olat, const CombineArgs& a,
                                    cudaStream_t stream, bool pdl);

}  // namespace hra

// decode_sm100.h -- host-side interface of the split-KV decode kernel.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace hra {

// Arguments of one decode launch (device pointers; see hra.h for layouts).
struct DecodeArgs {
  const __half* q_tilde;      // absorbed latent query (d_c) | rotated rope (64) per (sequence, head):
                              //   fp16 [B, h, d_c + 64], or for the 128-wide-branch kernel bf16 hi
                              //   [B, h, d_c + 64] followed by bf16 lo [B, h, d_c + 64]
  const int32_t* seq_lens;    // int32 [B]
  const int32_t* block_table; // int32 [B, max_pages] or nullptr (contiguous layout)
  int max_pages;
  int page_size;
  long long seq_stride;       // rows between sequences (contiguous layout)
  long long cache_rows;       // rows addressable through the tensor maps
  int batch;
  int heads;
  int d_c;                    // latent width held by this call: 512, or 256 / 128 for a branch shard
  float scale_log2;           // softmax scale * log2(e)
  float* o_part;              // fp32 [slots, d_c / 128, 128, 128]: un-normalised O per segment and slice
  float2* ml_part;            // fp32 [slots, d_c / 128, 128] pairs: (running max in log2 units, row sum)
  int* status;                // device status word
  uint64_t wait_limit_ns;     // global-time budget of one device-side wait
  int cache_int8;             // 1: the latent cache is int8 with per-(row, 128-column block) scales
  const float* ckv_scale;     // fp32 scales of row r at ckv_scale + r * scale_stride (int8 cache)
  long long scale_stride;
};

// Cache row of the 32-row chunk that starts at token `tok` of sequence s (length L):
// s * seq_stride + tok in the contiguous layout, or through the block table in the paged
// one (pages hold a multiple of 32 rows, so a chunk never straddles two pages).  A chunk
// that starts at or past the sequence end, or whose page is out of range, gets
// `cache_rows`: a row past the tensor map, which the TMA fills with zeros.  The block
// table is read before L is consulted so that both loads are in flight together.
__device__ __forceinline__ int cache_chunk_row(const DecodeArgs& a, int s, int tok) {
  long long row = a.cache_rows;
  const int L = a.seq_lens[s];
  if (a.block_table == nullptr) {
    row = static_cast<long long>(s) * a.seq_stride + tok;
  } else {
    const int pidx = tok / a.page_size;
    if (pidx < a.max_pages) {
      const int page = a.block_table[static_cast<long long>(s) * a.max_pages + pidx];
      row = static_cast<long long>(page) * a.page_size + tok % a.page_size;
    }
  }
  if (tok >= L || row < 0 || row >= a.cache_rows) row = a.cache_rows;
  return static_cast<int>(row);
}

// Tokens per cache tile for a branch width (decides the TMEM and shared-memory budget).
int decode_tile_tokens(int branch_width);
int decode_split_tile_tokens();
// Rows of one TMA box of the bf16 cache (the tensor maps' box height) for a branch width.
int decode_box_rows(int branch_width);

// 128-wide-branch kernel (MLRA-4, or a shard of its branches) with an fp16 query and the
// tile converted to fp16 in shared memory; grid (d_c / 128 branches, groups).
cudaError_t launch_decode_split_kernel(const CUtensorMap& map_ckv, const CUtensorMap& map_krope,
                                       const DecodeArgs& a, int groups, cudaStream_t stream, bool pdl);

// Launch the decode kernel on grid (d_c / 128 slices, `groups` KV splits); pdl:
// programmatic dependent launch (launch.h).  Branches 128 wide run the split kernel, 256
// and 512 wide the converting kernel.
cudaError_t launch_decode_kernel(int n_branch, const CUtensorMap& map_ckv, const CUtensorMap& map_krope,
                                 const DecodeArgs& a, int groups, cudaStream_t stream, bool pdl);

}  // namespace hra

// api.cu -- the C ABI of libhra.so (declared in include/hra.h): argument validation,
// workspace layout, TMA descriptor encoding and the launch sequence
//   absorb (tcgen05) -> split-KV decode (tcgen05) -> log-sum-exp merge -> up-projection (tcgen05)
// of one decode step, all on the caller's stream.  Nothing here allocates device memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "hra.h"
#include "absorb_combine.h"
#include "decode_sm100.h"
#include "prefill_sm100.h"
#include "schedule.cuh"
#include "sm100.cuh"

namespace {

thread_local std::string g_last_error;

hra_status fail(hra_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

hra_status cuda_fail(cudaError_t e, const char* what) {
  return fail(HRA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr uint64_t kDefaultWaitLimitUs = 1000000;  // 1 s per device-side wait
// Smallest limit a call may set: far above the time any one tile's copy, conversion or
// MMAs take, so that a wait only expires when the pipeline is really stuck.
constexpr uint64_t kMinWaitLimitUs = 10000;  // 10 ms

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

struct Plan {
  int groups = 0;
  long long slots = 0;
  size_t q_tilde = 0, o_part = 0, ml_part = 0, o_lat = 0, tile_prefix = 0, total = 0;
};

hra_status sm_count(int* n) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  e = cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  return HRA_OK;
}

hra_status validate(const hra_decode_params* p) {
  if (p == nullptr) return fail(HRA_ERR_INVALID_ARG, "params is NULL");
  if (p->d_rope != 64 || p->d_nope != 128 || p->d_v != 128)
    return fail(HRA_ERR_UNSUPPORTED, "widths (d_rope=%d, d_nope=%d, d_v=%d) must be 64/128/128", p->d_rope,
                p->d_nope, p->d_v);
  if (p->d_c == 512) {
    if (p->n_branch != 1 && p->n_branch != 2 && p->n_branch != 4)
      return fail(HRA_ERR_UNSUPPORTED, "n_branch=%d (supported with d_c=512: 1, 2, 4)", p->n_branch);
  } else if (!((p->d_c == 128 && p->n_branch == 1) || (p->d_c == 256 && (p->n_branch == 1 || p->n_branch == 2)))) {
    // a shard of the latent: 128-wide branches (d_c = 128 * branches held) or one 256-wide branch
    return fail(HRA_ERR_UNSUPPORTED,
                "d_c=%d with n_branch=%d (supported: d_c=512 with n_branch 1, 2, 4; d_c=256 with n_branch 1, 2; "
                "d_c=128 with n_branch 1)",
                p->d_c, p->n_branch);
  }
  if (p->batch < 1 || p->batch > hra::kMaxBatch)
    return fail(HRA_ERR_UNSUPPORTED, "batch=%d (supported: 1..%d)", p->batch, hra::kMaxBatch);
  if (p->num_heads < 1 || p->num_heads > 128)
    return fail(HRA_ERR_UNSUPPORTED, "num_heads=%d (supported: 1..128)", p->num_heads);
  // partial mode (a token range of a split sequence): the merged states go to part_o /
  // part_lse and out is not used
  const bool partial = p->part_o != nullptr || p->part_lse != nullptr;
  if (partial && (p->part_o == nullptr || p->part_lse == nullptr))
    return fail(HRA_ERR_INVALID_ARG, "part_o and part_lse must both be set (or both NULL)");
  const struct { const void* ptr; const char* name; } ptrs[] = {
      {p->q, "q"}, {p->ckv, "ckv"}, {p->krope, "krope"}, {p->seq_lens, "seq_lens"},
      {p->w_uk, "w_uk"}, {p->w_uv, "w_uv"}, {partial ? p->part_o : p->out, partial ? "part_o" : "out"},
      {partial ? p->part_lse : p->w_uv, "part_lse"}};
  for (const auto& x : ptrs) {
    if (x.ptr == nullptr) return fail(HRA_ERR_INVALID_ARG, "%s is NULL", x.name);
    if (!aligned16(x.ptr)) return fail(HRA_ERR_INVALID_ARG, "%s is not 16-byte aligned", x.name);
  }
  if (p->q_positions != nullptr && (reinterpret_cast<uintptr_t>(p->q_positions) & 3u) != 0)
    return fail(HRA_ERR_INVALID_ARG, "q_positions is not 4-byte aligned");
  if (p->ckv_stride < p->d_c || p->ckv_stride % 8 != 0)
    return fail(HRA_ERR_INVALID_ARG, "ckv_stride=%lld must be >= d_c=%d and a multiple of 8",
                (long long)p->ckv_stride, p->d_c);
  if (p->krope_stride < 64 || p->krope_stride % 8 != 0)
    return fail(HRA_ERR_INVALID_ARG, "krope_stride=%lld must be >= 64 and a multiple of 8",
                (long long)p->krope_stride);
  if (p->cache_rows < 1 || p->cache_rows > 0x7FFFFFFFLL)
    return fail(HRA_ERR_INVALID_ARG, "cache_rows=%lld out of range [1, 2^31-1]", (long long)p->cache_rows);
  if (p->block_table != nullptr) {
    if (p->max_pages < 1) return fail(HRA_ERR_INVALID_ARG, "max_pages=%d must be >= 1", p->max_pages);
    if (p->page_size < 32 || p->page_size % 32 != 0)
      return fail(HRA_ERR_UNSUPPORTED, "page_size=%d must be a positive multiple of 32", p->page_size);
  } else if (p->seq_stride < 0) {
    return fail(HRA_ERR_INVALID_ARG, "seq_stride=%lld must be >= 0", (long long)p->seq_stride);
  }
  if (p->out_dtype != HRA_BF16 && p->out_dtype != HRA_F32)
    return fail(HRA_ERR_INVALID_ARG, "out_dtype=%d", (int)p->out_dtype);
  if (p->num_splits < 0) return fail(HRA_ERR_INVALID_ARG, "num_splits=%d must be >= 0", p->num_splits);
  if (p->out_accumulate != 0 && p->out_accumulate != 1)
    return fail(HRA_ERR_INVALID_ARG, "out_accumulate=%d must be 0 or 1", p->out_accumulate);
  if (p->out_accumulate && p->out_dtype != HRA_F32)
    return fail(HRA_ERR_INVALID_ARG, "out_accumulate needs out_dtype = HRA_F32");
  if (p->n_out_peers < 0 || p->n_out_peers > hra::kMaxOutPeers)
    return fail(HRA_ERR_UNSUPPORTED, "n_out_peers=%d (supported: 0..%d)", p->n_out_peers, hra::kMaxOutPeers);
  if (p->n_out_peers > 0) {
    if (!p->out_accumulate) return fail(HRA_ERR_INVALID_ARG, "out_peers need out_accumulate = 1");
    if (p->out_peers == nullptr) return fail(HRA_ERR_INVALID_ARG, "out_peers is NULL");
    for (int k = 0; k < p->n_out_peers; ++k)
      if (p->out_peers[k] == nullptr || !aligned16(p->out_peers[k]))
        return fail(HRA_ERR_INVALID_ARG, "out_peers[%d] is NULL or not 16-byte aligned", k);
  }
  if (p->wait_limit < 0) return fail(HRA_ERR_INVALID_ARG, "wait_limit=%d must be >= 0", p->wait_limit);
  if (p->cache_dtype == HRA_INT8) {
    if (p->d_c / p->n_branch != 128)
      return fail(HRA_ERR_UNSUPPORTED, "an int8 cache is supported for 128-wide branches (d_c / n_branch = %d)",
                  p->d_c / p->n_branch);
    if (p->ckv_scale == nullptr || (reinterpret_cast<uintptr_t>(p->ckv_scale) & 3u) != 0)
      return fail(HRA_ERR_INVALID_ARG, "ckv_scale is NULL or not 4-byte aligned");
    if (p->ckv_scale_stride < p->d_c / 128)
      return fail(HRA_ERR_INVALID_ARG, "ckv_scale_stride=%lld must be >= d_c / 128", (long long)p->ckv_scale_stride);
    if (p->ckv_stride % 16 != 0)
      return fail(HRA_ERR_INVALID_ARG, "ckv_stride=%lld bytes must be a multiple of 16 for an int8 cache",
                  (long long)p->ckv_stride);
  } else if (p->cache_dtype != HRA_BF16) {
    return fail(HRA_ERR_INVALID_ARG, "cache_dtype=%d (HRA_BF16 or HRA_INT8)", (int)p->cache_dtype);
  }
  if (!std::isfinite(p->alpha_q) || !std::isfinite(p->alpha_kv) || !std::isfinite(p->branch_scale) ||
      !std::isfinite(p->softmax_scale) || !(p->rope_theta > 0.f) || !std::isfinite(p->rope_theta))
    return fail(HRA_ERR_INVALID_ARG, "scales must be finite and rope_theta > 0");
  return HRA_OK;
}

hra_status make_plan(const hra_decode_params* p, Plan* plan) {
  int sms = 0;
  if (p->num_splits > 0) {
    plan->groups = p->num_splits;
  } else {
    hra_status st = sm_count(&sms);
    if (st != HRA_OK) return st;
    plan->groups = sms / (p->d_c / 128) > 0 ? sms / (p->d_c / 128) : 1;  // one CTA per SM
  }
  if (plan->groups > 65535) return fail(HRA_ERR_INVALID_ARG, "num_splits=%d too large", plan->groups);
  plan->slots = static_cast<long long>(plan->groups) + p->batch;
  const size_t slices = static_cast<size_t>(p->d_c) / 128;
  size_t off = 256;  // device status word
  plan->q_tilde = off;  // fp16 [B, h, d_c + 64]
  off = round256(off + static_cast<size_t>(p->batch) * p->num_heads * (p->d_c + 64) * sizeof(__half));
  plan->o_part = off;
  off = round256(off + static_cast<size_t>(plan->slots) * slices * 128 * 128 * sizeof(float));
  plan->ml_part = off;
  off = round256(off + static_cast<size_t>(plan->slots) * slices * 128 * sizeof(float2));
  plan->o_lat = off;  // merged latent output as two bf16 terms
  off = round256(off + 2 * static_cast<size_t>(p->num_heads) * p->batch * p->d_c * sizeof(__nv_bfloat16));
  plan->tile_prefix = off;  // decode tiles per sequence, exclusive prefix [B + 1]
  off = round256(off + (static_cast<size_t>(p->batch) + 1) * sizeof(int));
  plan->total = off;
  return HRA_OK;
}

std::once_flag g_encode_once;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// 2-D view [rows, inner] with row stride `stride_elems`, boxes of box_inner x box_rows, 128-byte
// swizzle; bf16 elements, or bytes (int8 cache) with byte8 = true.
hra_status encode_map(CUtensorMap* map, const void* base, int64_t inner, int64_t rows, int64_t stride_elems,
                      int box_rows, bool byte8 = false, int box_inner = 64) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (g_encode == nullptr) return fail(HRA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(stride_elems) * (byte8 ? 1 : 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, byte8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HRA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return HRA_OK;
}

hra_status run_decode(const hra_decode_params* p, cudaStream_t stream) {
  hra_status st = validate(p);
  if (st != HRA_OK) return st;
  Plan plan;
  st = make_plan(p, &plan);
  if (st != HRA_OK) return st;
  if (p->workspace == nullptr) return fail(HRA_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(p->workspace) & 255u) != 0)
    return fail(HRA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (p->workspace_bytes < plan.total)
    return fail(HRA_ERR_WORKSPACE, "workspace_bytes=%zu < required %zu", p->workspace_bytes, plan.total);

  uint8_t* ws = static_cast<uint8_t*>(p->workspace);
  int* status = reinterpret_cast<int*>(ws);
  __half* q_tilde = reinterpret_cast<__half*>(ws + plan.q_tilde);
  float* o_part = reinterpret_cast<float*>(ws + plan.o_part);
  float2* ml_part = reinterpret_cast<float2*>(ws + plan.ml_part);
  __nv_bfloat16* o_lat = reinterpret_cast<__nv_bfloat16*>(ws + plan.o_lat);
  int* tile_prefix = reinterpret_cast<int*>(ws + plan.tile_prefix);

  // Every tensor map is encoded before the first launch so that no host work sits between
  // the kernels of one call.
  const int h = p->num_heads, B = p->batch, dc = p->d_c;
  CUtensorMap map_wuk, map_q, map_wuv, map_olat, map_ckv, map_krope;
  if ((st = encode_map(&map_wuk, p->w_uk, 128, static_cast<int64_t>(h) * dc, 128, dc < 256 ? dc : 256)) != HRA_OK)
    return st;
  if ((st = encode_map(&map_q, p->q, static_cast<int64_t>(h) * 192, B, static_cast<int64_t>(h) * 192,
                       hra::absorb_seq_chunk(B))) != HRA_OK)
    return st;
  if ((st = encode_map(&map_wuv, p->w_uv, 128, static_cast<int64_t>(h) * dc, 128, 128)) != HRA_OK) return st;
  if ((st = encode_map(&map_olat, o_lat, dc, 2 * static_cast<int64_t>(h) * B, dc, hra::upproj_seq_chunk())) !=
      HRA_OK)
    return st;
  const bool int8 = p->cache_dtype == HRA_INT8;
  // int8: one 128-byte box per 128-wide branch and 32 rows; bf16: 64-column boxes
  const int box_rows = int8 ? 32 : hra::decode_box_rows(dc / p->n_branch);
  if ((st = encode_map(&map_ckv, p->ckv, dc, p->cache_rows, p->ckv_stride, box_rows, int8, int8 ? 128 : 64)) !=
      HRA_OK)
    return st;
  if ((st = encode_map(&map_krope, p->krope, 64, p->cache_rows, p->krope_stride, box_rows)) != HRA_OK) return st;

  auto mark = [&](int k) -> cudaError_t {
    return p->stage_events ? cudaEventRecord(static_cast<cudaEvent_t>(p->stage_events[k]), stream) : cudaSuccess;
  };
  cudaError_t e = mark(0);
  if (e != cudaSuccess) return cuda_fail(e, "stage event");
  // The status word starts each call at zero.  It is cleared in stream order before any
  // kernel of the call runs, so that no block of any kernel can record an expired wait
  // before the clear lands (a memset allocates nothing).
  e = cudaMemsetAsync(status, 0, 4 * sizeof(int), stream);
  if (e != cudaSuccess) return cuda_fail(e, "status clear");

  hra::AbsorbArgs ab{};
  ab.q = static_cast<const __nv_bfloat16*>(p->q);
  ab.seq_lens = p->seq_lens;
  ab.q_tilde = q_tilde;
  ab.status = status;
  ab.batch = p->batch;
  ab.heads = p->num_heads;
  ab.alpha_q = p->alpha_q;
  ab.alpha_kv = p->alpha_kv;
  ab.rope_theta = p->rope_theta;
  ab.d_c = dc;
  ab.tile_prefix = tile_prefix;
  ab.tile_tokens = hra::decode_tile_tokens(dc / p->n_branch);
  ab.q_positions = p->q_positions;
  // Programmatic dependent launch lets each kernel start while the previous one drains;
  // the stage-timing mode launches plainly so that its events bracket whole kernels.
  const bool pdl = p->stage_events == nullptr;
  e = hra::launch_absorb_q(map_wuk, map_q, ab, stream, pdl);
  if (e != cudaSuccess) return cuda_fail(e, "absorb_q launch");

  const float tau = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(192.0f);
  hra::DecodeArgs da{};
  da.q_tilde = q_tilde;
  da.seq_lens = p->seq_lens;
  da.block_table = p->block_table;
  da.max_pages = p->max_pages;
  da.page_size = p->page_size;
  da.seq_stride = p->seq_stride;
  da.cache_rows = p->cache_rows;
  da.batch = p->batch;
  da.heads = p->num_heads;
  da.d_c = dc;
  da.scale_log2 = tau * 1.4426950408889634f;
  da.o_part = o_part;
  da.ml_part = ml_part;
  da.status = status;
  const uint64_t limit_us = p->wait_limit > 0 ? static_cast<uint64_t>(p->wait_limit) : kDefaultWaitLimitUs;
  da.wait_limit_ns = 1000ull * (limit_us < kMinWaitLimitUs ? kMinWaitLimitUs : limit_us);
  da.cache_int8 = int8 ? 1 : 0;
  da.ckv_scale = int8 ? p->ckv_scale : nullptr;
  da.scale_stride = int8 ? p->ckv_scale_stride : 0;
  if ((e = mark(1)) != cudaSuccess) return cuda_fail(e, "stage event");
  e = hra::launch_decode_kernel(p->n_branch, map_ckv, map_krope, da, plan.groups, stream, pdl);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  if ((e = mark(2)) != cudaSuccess) return cuda_fail(e, "stage event");

  hra::CombineArgs cb{};
  cb.o_part = o_part;
  cb.ml_part = ml_part;
  cb.tile_prefix = tile_prefix;
  cb.o_lat = o_lat;
  cb.w_uv = static_cast<const __nv_bfloat16*>(p->w_uv);
  cb.status = status;
  cb.out_f32 = p->out_dtype == HRA_F32 ? static_cast<float*>(p->out) : nullptr;
  cb.out_bf16 = p->out_dtype == HRA_BF16 ? static_cast<__nv_bfloat16*>(p->out) : nullptr;
  cb.accumulate = p->out_accumulate;
  cb.n_peers = p->n_out_peers;
  for (int k = 0; k < p->n_out_peers; ++k) cb.peers[k] = static_cast<float*>(p->out_peers[k]);
  cb.batch = p->batch;
  cb.heads = p->num_heads;
  cb.groups = plan.groups;
  cb.d_c = dc;
  if ((st = sm_count(&cb.sms)) != HRA_OK) return st;
  cb.part_o = p->part_o;
  cb.part_lse = p->part_lse;
  cb.alpha_kv = p->alpha_kv;
  cb.branch_scale = p->branch_scale;
  e = hra::launch_combine_upproj(map_wuv, map_olat, cb, stream, pdl);
  if (e != cudaSuccess) return cuda_fail(e, "combine_upproj launch");
  if ((e = mark(3)) != cudaSuccess) return cuda_fail(e, "stage event");
  g_last_error.clear();
  return HRA_OK;
}

// Merge the gathered states of a sequence split by token range, then the up-projection
// (hra_combine_partials).
constexpr int kMaxParts = 64;

hra_status run_combine_partials(const hra_decode_params* p, int n_parts, const float* parts_o, const float* parts_lse,
                                cudaStream_t stream) {
  if (p == nullptr) return fail(HRA_ERR_INVALID_ARG, "params is NULL");
  hra_decode_params q = *p;  // the decode's parameters, finishing into out
  q.part_o = nullptr;
  q.part_lse = nullptr;
  hra_status st = validate(&q);
  if (st != HRA_OK) return st;
  if (n_parts < 1 || n_parts > kMaxParts)
    return fail(HRA_ERR_INVALID_ARG, "n_parts=%d (supported: 1..%d)", n_parts, kMaxParts);
  if (parts_o == nullptr || parts_lse == nullptr || !aligned16(parts_o) || !aligned16(parts_lse))
    return fail(HRA_ERR_INVALID_ARG, "parts_o / parts_lse NULL or not 16-byte aligned");
  Plan plan;
  if ((st = make_plan(&q, &plan)) != HRA_OK) return st;
  if (q.workspace == nullptr) return fail(HRA_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(q.workspace) & 255u) != 0)
    return fail(HRA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (q.workspace_bytes < plan.total)
    return fail(HRA_ERR_WORKSPACE, "workspace_bytes=%zu < required %zu", q.workspace_bytes, plan.total);
  uint8_t* ws = static_cast<uint8_t*>(q.workspace);
  int* status = reinterpret_cast<int*>(ws);
  __nv_bfloat16* o_lat = reinterpret_cast<__nv_bfloat16*>(ws + plan.o_lat);
  const int h = q.num_heads, B = q.batch, dc = q.d_c;
  CUtensorMap map_wuv, map_olat;
  if ((st = encode_map(&map_wuv, q.w_uv, 128, static_cast<int64_t>(h) * dc, 128, 128)) != HRA_OK) return st;
  if ((st = encode_map(&map_olat, o_lat, dc, 2 * static_cast<int64_t>(h) * B, dc, hra::upproj_seq_chunk())) !=
      HRA_OK)
    return st;
  cudaError_t e = cudaMemsetAsync(status, 0, 4 * sizeof(int), stream);
  if (e != cudaSuccess) return cuda_fail(e, "status clear");
  hra::CombineArgs cb{};
  cb.o_lat = o_lat;
  cb.w_uv = static_cast<const __nv_bfloat16*>(q.w_uv);
  cb.status = status;
  cb.out_f32 = q.out_dtype == HRA_F32 ? static_cast<float*>(q.out) : nullptr;
  cb.out_bf16 = q.out_dtype == HRA_BF16 ? static_cast<__nv_bfloat16*>(q.out) : nullptr;
  cb.accumulate = q.out_accumulate;
  cb.n_peers = q.n_out_peers;
  for (int k = 0; k < q.n_out_peers; ++k) cb.peers[k] = static_cast<float*>(q.out_peers[k]);
  cb.batch = B;
  cb.heads = h;
  cb.groups = plan.groups;
  cb.d_c = dc;
  cb.alpha_kv = q.alpha_kv;
  cb.branch_scale = q.branch_scale;
  cb.parts_o = parts_o;
  cb.parts_lse = parts_lse;
  cb.n_parts = n_parts;
  e = hra::launch_combine_partials(map_wuv, map_olat, cb, stream, true);
  if (e != cudaSuccess) return cuda_fail(e, "combine_partials launch");
  g_last_error.clear();
  return HRA_OK;
}

// ---------------------------------------------------------------------------- prefill
constexpr long long kMaxPrefillLen = 1 << 20;

hra_status validate_prefill(const hra_prefill_params* p) {
  if (p == nullptr) return fail(HRA_ERR_INVALID_ARG, "params is NULL");
  if (p->d_c != 512 || p->d_rope != 64 || p->d_nope != 128 || p->d_v != 128)
    return fail(HRA_ERR_UNSUPPORTED, "widths (d_c=%d, d_rope=%d, d_nope=%d, d_v=%d) must be 512/64/128/128", p->d_c,
                p->d_rope, p->d_nope, p->d_v);
  if (p->n_branch != 1 && p->n_branch != 2 && p->n_branch != 4)
    return fail(HRA_ERR_UNSUPPORTED, "n_branch=%d (supported: 1, 2, 4)", p->n_branch);
  if (p->num_heads < 1 || p->num_heads > 128)
    return fail(HRA_ERR_UNSUPPORTED, "num_heads=%d (supported: 1..128)", p->num_heads);
  if (p->seq_len < 1 || p->seq_len > kMaxPrefillLen)
    return fail(HRA_ERR_UNSUPPORTED, "seq_len=%d (supported: 1..%lld)", p->seq_len, kMaxPrefillLen);
  if (p->n_query < 1 || p->n_query > p->seq_len)
    return fail(HRA_ERR_INVALID_ARG, "n_query=%d must be in [1, seq_len=%d]", p->n_query, p->seq_len);
  const struct { const void* ptr; const char* name; } ptrs[] = {
      {p->q, "q"}, {p->ckv, "ckv"}, {p->krope, "krope"}, {p->w_uk, "w_uk"}, {p->w_uv, "w_uv"}, {p->out, "out"}};
  for (const auto& x : ptrs) {
    if (x.ptr == nullptr) return fail(HRA_ERR_INVALID_ARG, "%s is NULL", x.name);
    if (!aligned16(x.ptr)) return fail(HRA_ERR_INVALID_ARG, "%s is not 16-byte aligned", x.name);
  }
  if (p->ckv_stride < 512 || p->ckv_stride % 8 != 0)
    return fail(HRA_ERR_INVALID_ARG, "ckv_stride=%lld must be >= 512 and a multiple of 8", (long long)p->ckv_stride);
  if (p->krope_stride < 64 || p->krope_stride % 8 != 0)
    return fail(HRA_ERR_INVALID_ARG, "krope_stride=%lld must be >= 64 and a multiple of 8",
                (long long)p->krope_stride);
  if (p->out_dtype != HRA_BF16 && p->out_dtype != HRA_F32)
    return fail(HRA_ERR_INVALID_ARG, "out_dtype=%d", (int)p->out_dtype);
  if (p->wait_limit < 0) return fail(HRA_ERR_INVALID_ARG, "wait_limit=%d must be >= 0", p->wait_limit);
  if (!std::isfinite(p->alpha_q) || !std::isfinite(p->alpha_kv) || !std::isfinite(p->branch_scale) ||
      !std::isfinite(p->softmax_scale) || !(p->rope_theta > 0.f) || !std::isfinite(p->rope_theta))
    return fail(HRA_ERR_INVALID_ARG, "scales must be finite and rope_theta > 0");
  return HRA_OK;
}

struct PrefillPlan {
  int l_pad = 0;
  size_t q16 = 0, kr16 = 0, k_exp = 0, v_exp = 0, total = 0;
};

PrefillPlan prefill_plan(const hra_prefill_params* p) {
  PrefillPlan pl;
  pl.l_pad = (p->seq_len + 127) / 128 * 128;
  const size_t h = static_cast<size_t>(p->num_heads);
  size_t off = 256;  // status word
  pl.q16 = off;
  off = round256(off + static_cast<size_t>(p->n_query) * h * 192 * 2);
  pl.kr16 = off;
  off = round256(off + static_cast<size_t>(pl.l_pad) * 64 * 2);
  pl.k_exp = off;
  off = round256(off + static_cast<size_t>(p->n_branch) * h * pl.l_pad * 128 * 2);
  pl.v_exp = off;
  off = round256(off + static_cast<size_t>(p->n_branch) * h * pl.l_pad * 128 * 2);
  pl.total = off;
  return pl;
}

hra_status run_prefill(const hra_prefill_params* p, cudaStream_t stream) {
  hra_status st = validate_prefill(p);
  if (st != HRA_OK) return st;
  const PrefillPlan pl = prefill_plan(p);
  if (p->workspace == nullptr) return fail(HRA_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(p->workspace) & 255u) != 0)
    return fail(HRA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (p->workspace_bytes < pl.total)
    return fail(HRA_ERR_WORKSPACE, "workspace_bytes=%zu < required %zu", p->workspace_bytes, pl.total);
  uint8_t* ws = static_cast<uint8_t*>(p->workspace);
  const int h = p->num_heads, nb = p->n_branch, L = p->seq_len, n = p->n_query;
  hra::PrefillArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(p->q);
  a.krope = static_cast<const __nv_bfloat16*>(p->krope);
  a.krope_stride = p->krope_stride;
  a.q16 = reinterpret_cast<__half*>(ws + pl.q16);
  a.kr16 = reinterpret_cast<__half*>(ws + pl.kr16);
  a.k_exp = reinterpret_cast<__half*>(ws + pl.k_exp);
  a.v_exp = reinterpret_cast<__half*>(ws + pl.v_exp);
  a.out_f32 = p->out_dtype == HRA_F32 ? static_cast<float*>(p->out) : nullptr;
  a.out_bf16 = p->out_dtype == HRA_BF16 ? static_cast<__nv_bfloat16*>(p->out) : nullptr;
  a.status = reinterpret_cast<int*>(ws);
  a.heads = h;
  a.n_branch = nb;
  a.seq_len = L;
  a.n_query = n;
  a.l_pad = pl.l_pad;
  a.alpha_q = p->alpha_q;
  a.alpha_kv = p->alpha_kv;
  a.branch_scale = p->branch_scale;
  const float tau = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(192.0f);
  a.scale_log2 = tau * 1.4426950408889634f;
  a.rope_theta = p->rope_theta;
  const uint64_t limit_us = p->wait_limit > 0 ? static_cast<uint64_t>(p->wait_limit) : kDefaultWaitLimitUs;
  a.wait_limit_ns = 1000ull * (limit_us < kMinWaitLimitUs ? kMinWaitLimitUs : limit_us);

  hra::PrefillMaps m;
  if ((st = encode_map(&m.ckv, p->ckv, 512, L, p->ckv_stride, 128)) != HRA_OK) return st;
  if ((st = encode_map(&m.wuk, p->w_uk, 128, static_cast<int64_t>(h) * 512, 128, 128)) != HRA_OK) return st;
  if ((st = encode_map(&m.wuv, p->w_uv, 128, static_cast<int64_t>(h) * 512, 128, 128)) != HRA_OK) return st;
  // fp16 workspace tensors: the copies move 16-bit elements, whatever their format
  if ((st = encode_map(&m.q16, a.q16, static_cast<int64_t>(h) * 192, n, static_cast<int64_t>(h) * 192, 128)) != HRA_OK)
    return st;
  const int64_t kv_rows = static_cast<int64_t>(nb) * h * pl.l_pad;
  if ((st = encode_map(&m.k, a.k_exp, 128, kv_rows, 128, 128)) != HRA_OK) return st;
  if ((st = encode_map(&m.v, a.v_exp, 128, kv_rows, 128, 128)) != HRA_OK) return st;
  if ((st = encode_map(&m.kr16, a.kr16, 64, pl.l_pad, 64, 128)) != HRA_OK) return st;

  cudaError_t e = cudaMemsetAsync(a.status, 0, 4 * sizeof(int), stream);
  if (e != cudaSuccess) return cuda_fail(e, "status clear");
  e = hra::launch_prefill(m, a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  g_last_error.clear();
  return HRA_OK;
}

hra_status read_status(void* workspace, cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int st[4] = {0, 0, 0, 0};
  e = cudaMemcpy(st, workspace, sizeof(st), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (st[0] != 0)
    return fail(HRA_ERR_DEVICE_TIMEOUT, "device wait expired (code %d, site %d, parity %d, block %d)", st[0], st[1],
                st[2], st[3]);
  g_last_error.clear();
  return HRA_OK;
}

__global__ void wait_timeout_selftest_kernel(int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    status[0] = status[1] = status[2] = status[3] = 0;
    hra::mbar_init(&bar, 1);
    abort_flag = 0;
    hra::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on `bar`: the wait must give up after limit_ns
    hra::mbar_wait(&bar, 0, limit_ns, &abort_flag, status, 99);
  }
  __syncthreads();
}

}  // namespace

namespace hra {
// Lets other entry points of this library report through hra_last_error().
void set_last_error(const char* msg) { g_last_error = msg; }
// Workspace bytes of a call, with the status of the validation or device query that failed.
hra_status workspace_bytes(const hra_decode_params* p, size_t* bytes) {
  *bytes = 0;
  hra_status st = validate(p);
  if (st != HRA_OK) return st;
  Plan plan;
  if ((st = make_plan(p, &plan)) != HRA_OK) return st;
  *bytes = plan.total;
  return HRA_OK;
}
}  // namespace hra

extern "C" {

size_t hra_workspace_size(const hra_decode_params* p) {
  if (validate(p) != HRA_OK) return 0;
  Plan plan;
  if (make_plan(p, &plan) != HRA_OK) return 0;
  return plan.total;
}

hra_status mlra_decode(const hra_decode_params* p, void* stream) {
  return run_decode(p, static_cast<cudaStream_t>(stream));
}

hra_status mla_decode(const hra_decode_params* p, void* stream) {
  if (p != nullptr && p->n_branch != 1)
    return fail(HRA_ERR_INVALID_ARG, "mla_decode requires n_branch == 1 (got %d)", p->n_branch);
  return run_decode(p, static_cast<cudaStream_t>(stream));
}

hra_status hra_combine_partials(const hra_decode_params* p, int n_parts, const float* parts_o, const float* parts_lse,
                                void* stream) {
  return run_combine_partials(p, n_parts, parts_o, parts_lse, static_cast<cudaStream_t>(stream));
}

hra_status hra_check_device_status(const hra_decode_params* p, void* stream) {
  if (p == nullptr || p->workspace == nullptr) return fail(HRA_ERR_INVALID_ARG, "params or workspace is NULL");
  return read_status(p->workspace, static_cast<cudaStream_t>(stream));
}

size_t hra_prefill_workspace_size(const hra_prefill_params* p) {
  if (validate_prefill(p) != HRA_OK) return 0;
  return prefill_plan(p).total;
}

hra_status mlra_prefill(const hra_prefill_params* p, void* stream) {
  return run_prefill(p, static_cast<cudaStream_t>(stream));
}

hra_status hra_check_prefill_status(const hra_prefill_params* p, void* stream) {
  if (p == nullptr || p->workspace == nullptr) return fail(HRA_ERR_INVALID_ARG, "params or workspace is NULL");
  return read_status(p->workspace, static_cast<cudaStream_t>(stream));
}

hra_status hra_selftest_wait_timeout(void* workspace, int limit_us, void* stream) {
  if (workspace == nullptr) return fail(HRA_ERR_INVALID_ARG, "workspace is NULL");
  if (limit_us < 1 || limit_us > 10000000) return fail(HRA_ERR_INVALID_ARG, "limit_us=%d out of [1, 1e7]", limit_us);
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<int*>(workspace), 1000ull * static_cast<uint64_t>(limit_us));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return HRA_OK;
}

const char* hra_last_error(void) { return g_last_error.c_str(); }

const char* hra_version(void) { return "hra 0.1.0 (sm_100a)"; }

}  // extern "C"

/*
 * hra.h -- C ABI of the B200 (sm_100a) latent-cache decode library (libhra.so).
 *
 * One call computes single-token decode attention for a batch of sequences over a
 * compressed latent KV cache, in the three steps of "Multi-Head Low-Rank Attention"
 * (section 方法步骤详情):
 *   1. query-side absorption: q~^(b),(i) = alpha_q * alpha_kv * W_UK^(b),(i) q_nope^(i),
 *      and RoPE on q_rope at position L-1;
 *   2. MQA-style decode over the shared key [C_KV | K_RoPE] with value C_KV, with one
 *      independent softmax per (head, branch); every branch reuses the shared K_RoPE;
 *   3. output up-projection and branch sum:
 *      out^(i) = branch_scale * alpha_kv * sum_b o_lat^(b),(i) W_UV^(b),(i).
 * n_branch = 1 is MLA ("ML Revisit: Attention", Multi-Head Latent Attention: the
 * absorbed QK^T = C_q W_q W_k^T C_kv^T with a decoupled RoPE key shared by all heads);
 * n_branch = 4 is MLRA-4 (核心方法: O = sum_b Softmax(Q K_b^T) V_b).
 * Branch shards (核心方法: under 4-way tensor parallelism each device holds one MLRA-4
 * branch's latent columns, a copy of K_RoPE and that branch's W_UK / W_UV rows): a call with
 * d_c = 128 * n_branch in {128, 256} computes the branches it holds, and its out is that
 * shard's part of the branch sum; summing out over the shards (an all-reduce across the
 * devices) gives the MLRA-4 output.  Pass the full model's branch_scale (1/2 for MLRA-4).
 * A call with d_c = 256 and n_branch = 1 attends over one 256-wide latent: a rank of MLRA-2
 * split by branch (branch_scale 1/sqrt(2), outs summed), or a rank of GLA-2 (研究动机: MLA's
 * latent split into two groups; the rank's heads only, branch_scale 1, outs concatenated
 * over heads).
 * The softmax scale of every branch is 1/sqrt(d_nope + d_rope) by default
 * ("vllbc02MLA", DeepseekV2Attention.__init__: scaling = qk_head_dim ** -0.5).
 *
 * Ownership: the caller owns every buffer.  The library allocates no device memory,
 * keeps no pointer after a call returns, and runs asynchronously on `stream`.
 * Errors: argument problems return a negative status before any launch, with a
 * message from hra_last_error() (thread-local).  Launch failures return HRA_ERR_CUDA.
 * Bounded device waits that expire write a status word in the workspace, read back
 * by hra_check_device_status().
 * Numerics: bf16 inputs, fp32 accumulation; softmax, combine and up-projection in fp32.
 * The decode kernels convert each cache tile to fp16 in shared memory (exact for bf16
 * values of fp16's range) and score it against the absorbed query in fp16; the softmax
 * weights P are fp16 in the P.V product.  |cache values| must stay below 65504.
 * Stream order: the kernels of a call are chained with programmatic dependent launch, so
 * a call may begin (set-up, loads of its inputs) while the previous call on the stream
 * drains; it touches the workspace only once that call has completed.
 */
#ifndef HRA_H
#define HRA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HRA_API __attribute__((visibility("default")))
#else
#define HRA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HRA_OK = 0,
  HRA_ERR_INVALID_ARG = -1,     /* null/misaligned pointer, bad size or stride           */
  HRA_ERR_UNSUPPORTED = -2,     /* shape outside the supported set (see below)           */
  HRA_ERR_WORKSPACE = -3,       /* workspace missing or smaller than hra_workspace_size  */
  HRA_ERR_CUDA = -4,            /* a CUDA runtime/driver call or a launch failed         */
  HRA_ERR_DEVICE_TIMEOUT = -5   /* a bounded device-side wait expired                    */
} hra_status;

typedef enum { HRA_BF16 = 0, HRA_F32 = 1, HRA_INT8 = 2 } hra_dtype;

/*
 * Parameters of one decode step.  All pointers are device pointers, 16-byte aligned.
 * Supported set: d_rope = 64, d_nope = 128, d_v = 128; d_c = 512 with n_branch in {1,2,4},
 * d_c = 256 with n_branch in {1,2}, d_c = 128 with n_branch = 1; 1 <= num_heads <= 128,
 * 1 <= batch <= 1024.
 */
typedef struct {
  int batch;            /* B, number of sequences (one query token each)               */
  int num_heads;        /* h, query heads sharing the latent cache                     */
  int n_branch;         /* 1 = MLA, 2 = two-branch MLRA, 4 = MLRA-4; for a branch shard,
                           the number of 128-wide branches this call holds               */
  int d_c, d_rope, d_nope, d_v;   /* 512 (128 or 256 for a shard), 64, 128, 128         */

  const void* q;        /* bf16 [B, h, d_nope + d_rope], dense: q_nope | q_rope; q_rope is
                           NOT rotated (the library rotates it at position seq_lens[b]-1) */
  const void* ckv;      /* bf16 latent rows: row r is C_KV at ckv + r * ckv_stride          */
  const void* krope;    /* bf16 RoPE-key rows, already rotated at their own positions:
                           row r at krope + r * krope_stride.  A fused [rows, 576] cache
                           is ckv = base, krope = base + 512, both strides 576 (a shard's
                           [rows, d_c + 64]: krope = base + d_c, strides d_c + 64)        */
  int64_t ckv_stride;   /* elements between consecutive rows; multiple of 8              */
  int64_t krope_stride; /* elements between consecutive rows; multiple of 8              */
  int64_t cache_rows;   /* rows addressable from ckv / krope (bounds every row access)   */

  const int32_t* seq_lens;   /* int32 [B]: cached tokens per sequence, including the
                                current one; 1 <= L.  L = 0 yields a zero output row    */
  const int32_t* block_table;/* NULL: contiguous, row(b,t) = b * seq_stride + t.
                                else int32 [B, max_pages]: row(b,t) =
                                block_table[b*max_pages + t/page_size]*page_size + t%page_size */
  int32_t max_pages;    /* columns of block_table                                       */
  int32_t page_size;    /* rows per page; a multiple of 32                               */
  int64_t seq_stride;   /* rows between sequences in the contiguous layout              */

  const void* w_uk;     /* bf16 [h, d_c, d_nope]: W_UK[i] maps the latent to K_nope      */
  const void* w_uv;     /* bf16 [h, d_c, d_v]:    W_UV[i] maps the latent to V            */
  float alpha_q;        /* variance-correction scale on q_nope                          */
  float alpha_kv;       /* variance-correction scale on the up-projected K_nope and V     */
  float branch_scale;   /* scale on the branch sum (1/sqrt(n_branch) in the workloads)   */
  float softmax_scale;  /* <= 0 selects 1/sqrt(d_nope + d_rope)                          */
  float rope_theta;     /* RoPE base; pairs (j, j + d_rope/2) turn by pos*theta^(-2j/d_rope) */

  void* out;            /* [B, h, d_v] in out_dtype                                      */
  hra_dtype out_dtype;

  void* workspace;      /* scratch of at least hra_workspace_size(p) bytes, 256-B aligned */
  size_t workspace_bytes;
  int num_splits;       /* KV splits = groups of d_c/128 CTAs streaming disjoint token
                           ranges; 0 = one group per d_c/128 SMs of the current device    */
  int wait_limit;       /* microseconds one device-side wait may last; 0 = 1 s.  Values
                           below 10000 (10 ms) are raised to 10 ms, far above the time any
                           one tile's copy, conversion or MMAs take                     */
  void* const* stage_events; /* optional, NULL = none: 4 caller-owned cudaEvent_t recorded on
                                `stream` before absorption, before the split-KV decode, before
                                the combine/up-projection and after it (per-stage timing)    */

  /* Tensor-parallel output, fused with the up-projection (optional; 0 = off).
     out_accumulate = 1: instead of storing out, the up-projection ADDS its result (fp32
     atomics; out_dtype must be HRA_F32) into out and into each out_peers[k].  With
     out_peers = the other ranks' out buffers mapped into this process (peer memory over
     NVLink: symmetric memory or IPC), every rank of a branch-sharded call writes its
     shard's part of the branch sum into every rank's out, so the sum over shards needs no
     separate all-reduce.  The caller zeroes the buffers and orders the ranks: every out is
     zeroed before any rank's call starts, and read only after every rank's call completed.
     The order of the additions varies, so the sum is not bitwise reproducible.          */
  int out_accumulate;   /* 0 or 1                                                        */
  int n_out_peers;      /* 0..7 entries in out_peers (requires out_accumulate = 1)        */
  void* const* out_peers; /* host array of device pointers to [B, h, d_v] fp32, 16-B aligned */

  /* Quantised latent cache (optional; 0 = the bf16 cache above).  The MLA tutorial's
     deployment notes ("从MHA到MLA", 部署注意事项) serve MLA in INT8, and "Multi-Head
     Low-Rank Attention" (未来方向) names KV-cache quantisation as the next step to combine
     with MLRA.  cache_dtype = HRA_INT8: ckv holds int8 latent rows (ckv_stride counted in
     bytes, a multiple of 16), each 128-column block b of row r standing for
     q[r, c] * ckv_scale[r * ckv_scale_stride + b] (symmetric, one fp32 scale per token and
     128-column block, i.e. per MLRA-4 branch; the caller writes both when it appends to the
     cache).  krope stays bf16.  Supported for 128-wide branches (MLRA-4 and its branch
     shards; others return HRA_ERR_UNSUPPORTED).  The decode kernel rescales each block
     to fp16 (|q * scale| < 65504).  The cache then holds d_c + 2 * d_rope + 4 * d_c / 128
     bytes per token instead of 2 * (d_c + d_rope).                                         */
  hra_dtype cache_dtype;        /* HRA_BF16 (default) or HRA_INT8                          */
  const float* ckv_scale;       /* fp32 scales, row r's at ckv_scale + r * ckv_scale_stride */
  int64_t ckv_scale_stride;     /* floats between consecutive rows' scales, >= d_c / 128   */

  /* One sequence split across devices by token range (optional; NULL = off).  A device
     holding tokens [a, b) of a sequence of L tokens passes its rows as the sequence
     (seq_lens[s] = b - a) and q_positions[s] = L - 1, the query's position; with part_o
     and part_lse set the call stops after the split-KV merge and writes, for every
     (sequence, head, 128-column slice of the latent), the slice's softmax-weighted latent
     row over its tokens (normalised) and the log2 of the slice's softmax denominator
     (log2 sum_t exp(score_t); -inf for an empty range, with a zero row).  out is then
     neither read nor written (it may be NULL).  The devices gather these states and one
     hra_combine_partials call merges them and finishes the decode.                      */
  const int32_t* q_positions;   /* [B] position of each sequence's query, or NULL: L - 1   */
  float* part_o;                /* fp32 [B, h, d_c], 16-B aligned, or NULL                 */
  float* part_lse;              /* fp32 [B, h, d_c / 128], 16-B aligned, or NULL           */
} hra_decode_params;

/* Bytes of workspace one call with these parameters needs (0 on invalid parameters).
 * Depends on batch, num_splits and the current device's SM count. */
HRA_API size_t hra_workspace_size(const hra_decode_params* p);

/* MLRA decode ("Multi-Head Low-Rank Attention", 方法步骤详情), n_branch in {1,2,4}, or a
 * branch shard (see above). */
HRA_API hra_status mlra_decode(const hra_decode_params* p, void* stream /* cudaStream_t */);

/* MLA decode: the same call restricted to n_branch == 1 ("ML Revisit: Attention",
 * Multi-Head Latent Attention; "vllbc02MLA", decode uses the absorbed MQA-like form). */
HRA_API hra_status mla_decode(const hra_decode_params* p, void* stream /* cudaStream_t */);

/* The same decode without a caller workspace, for callers that cannot allocate device
 * memory (code running inside another runtime's memory pool or an allocation-free
 * serving path, plain C callers without an allocator).  The paper has no counterpart:
 * this is a deployment variant of mlra_decode.  Scratch comes from one 32 MiB
 * file-scope device array that every GPU loading the library holds until exit;
 * p->workspace and p->workspace_bytes are ignored.  Calls whose hra_workspace_size
 * exceeds 32 MiB return HRA_ERR_WORKSPACE before any launch (the size depends on batch,
 * heads and the split count: with d_c = 512 and 37 splits, up to 35 sequences at h = 128
 * and 74 at h = 16; the size check itself queries the current device's SM count unless
 * num_splits > 0).  The first call on a device looks the array's device address up (make
 * it before any stream capture); the address is kept, so do not use the library across a
 * device reset.  All calls on a device share the array: calls that overlap on the GPU
 * race; the status word is cleared by every call, and expired device waits recorded there
 * are not reachable through hra_check_device_status.  Allocates nothing. */
HRA_API hra_status mlra_decode_static(const hra_decode_params* p, void* stream /* cudaStream_t */);

/* Finish a decode whose tokens were split into n_parts ranges (across devices, see
 * q_positions / part_o / part_lse above): parts_o fp32 [n_parts, B, h, d_c] and parts_lse
 * fp32 [n_parts, B, h, d_c / 128] hold the ranges' states in any order (device memory,
 * 16-B aligned; an all-gather of every device's part_o / part_lse produces them).  Per
 * (sequence, head, slice) the states are merged by their log-sum-exp (with m the largest
 * lse, each range's row is weighted by 2^(lse - m) and the weights' sum normalises), and
 * the merged latent rows go through the up-projection and branch sum of mlra_decode into
 * p->out (out_dtype, out_accumulate and out_peers as there).  p is the decode's parameter
 * block: shapes, w_uv, alpha_kv, branch_scale, out and a workspace of
 * hra_workspace_size(p) bytes; its part_o and part_lse are ignored.  1 <= n_parts <= 64. */
HRA_API hra_status hra_combine_partials(const hra_decode_params* p, int n_parts, const float* parts_o,
                                        const float* parts_lse, void* stream /* cudaStream_t */);

/*
 * Prefill: causal multi-token MLRA for one sequence, in the expanded form ("vllbc02MLA":
 * prefill is compute-bound and works with the per-head keys and values; generation is
 * memory-bound and uses the absorbed form).  The cache holds seq_len tokens; the queries
 * are the last n_query of them (query j at position seq_len - n_query + j sees the tokens
 * t <= its position), each attending per branch as in "Multi-Head Low-Rank Attention"
 * (核心方法), with the branch outputs summed and scaled as in mlra_decode.
 * The call forms K_nope^(b),(i) = alpha_kv C^(b) W_UK^(b),(i) and V^(b),(i) =
 * alpha_kv C^(b) W_UV^(b),(i) for every cached token in the workspace (fp16), then runs
 * a causal attention over them on the tensor cores (fp16 operands, fp32 accumulation,
 * fp32 softmax).  With n_query = 1 it computes the same output as mlra_decode of that
 * sequence.
 * Supported: d_c = 512, n_branch in {1, 2, 4}, d_rope = 64, d_nope = d_v = 128,
 * 1 <= num_heads <= 128, 1 <= n_query <= seq_len <= 2^20.  Pointers 16-byte aligned;
 * the caller owns every buffer; the library allocates nothing.
 */
typedef struct {
  int num_heads, n_branch;
  int d_c, d_rope, d_nope, d_v;   /* 512, 64, 128, 128                                    */
  int seq_len;          /* L, cached tokens including the queries                         */
  int n_query;          /* n, query tokens: the last n positions                          */
  const void* q;        /* bf16 [n, h, d_nope + d_rope], dense; q_rope NOT rotated        */
  const void* ckv;      /* bf16 latent rows 0..L-1 of the sequence, ckv_stride apart      */
  const void* krope;    /* bf16 rotated rope-key rows 0..L-1, krope_stride apart          */
  int64_t ckv_stride, krope_stride;  /* elements; multiples of 8                         */
  const void* w_uk;     /* bf16 [h, d_c, d_nope]                                          */
  const void* w_uv;     /* bf16 [h, d_c, d_v]                                             */
  float alpha_q, alpha_kv, branch_scale, softmax_scale, rope_theta;  /* as in mlra_decode */
  void* out;            /* [n, h, d_v] in out_dtype                                       */
  hra_dtype out_dtype;  /* HRA_BF16 or HRA_F32                                            */
  void* workspace;      /* at least hra_prefill_workspace_size(p) bytes, 256-byte aligned */
  size_t workspace_bytes;
  int wait_limit;       /* as in hra_decode_params                                        */
} hra_prefill_params;

/* Workspace bytes of one prefill call (0 on invalid parameters): the status word, the
 * fp16 queries, the fp16 rope keys and the expanded keys and values,
 * 2 * n_branch * h * ceil(L / 128) * 128 * 128 fp16 values. */
HRA_API size_t hra_prefill_workspace_size(const hra_prefill_params* p);

/* Prefill (see above); asynchronous on `stream`.  Device-side expired waits are read back
 * with hra_check_prefill_status. */
HRA_API hra_status mlra_prefill(const hra_prefill_params* p, void* stream /* cudaStream_t */);

/* Synchronize `stream` and read the device status word of p->workspace (as
 * hra_check_device_status does for a decode call). */
HRA_API hra_status hra_check_prefill_status(const hra_prefill_params* p, void* stream);

/* Synchronize `stream` and read the device status word of p->workspace.
 * HRA_OK, or HRA_ERR_DEVICE_TIMEOUT if a bounded wait expired during the last call. */
HRA_API hra_status hra_check_device_status(const hra_decode_params* p, void* stream);

/* Self-test of the bounded-wait machinery: one block waits on an mbarrier that nothing
 * arrives on, for at most `limit_us` microseconds (1..1e7), records the expiry in the
 * status word of `workspace` and returns.  No copy or MMA is in flight.  Host code then
 * reads the status with hra_check_device_status. */
HRA_API hra_status hra_selftest_wait_timeout(void* workspace, int limit_us, void* stream);

/* Message describing the last error on this thread ("" if none). */
HRA_API const char* hra_last_error(void);

/* Library version string. */
HRA_API const char* hra_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HRA_H */

// decode_split_sm100.cu -- split-KV decode for 128-wide latent branches (MLRA-4, or a
// shard of its branches) on tcgen05/TMEM, one CTA per branch.
//
// Step 2 of the decode in "Multi-Head Low-Rank Attention" (方法步骤详情): every head's
// absorbed query attends, MQA-style, over its branch's 128 latent columns of the shared
// cache plus the shared RoPE key, with one independent online softmax per (head, branch)
// (核心方法: O = sum_b Softmax(Q K_b^T) V_b), and V = the same 128 latent columns.
// Work decomposition (schedule.cuh): grid (d_c / 128 branches, G groups); group g streams
// a contiguous range of the batch's 128-token tiles laid end to end, and each CTA of the
// group handles one branch of those tiles, so a tile's latent columns are read from HBM
// once and its rope columns once per branch (the repeats hit L2).
//
// Precision: the absorbed query is fp16 (from the absorb kernel), the converter warps
// rewrite each arrived bf16 tile as fp16 in place (exact for |x| < 65504 down to fp16's
// normal range), and P is fp16, so QK^T and P.V are kind::f16 MMAs with fp32 accumulation.
//
// Per 128-token tile: 8 latent + 4 rope QK MMAs (M = 128 heads, N = 128 tokens, K = 16)
// and 8 P.V MMAs (N = 128 latent columns, K = 16 tokens).
//
// TMEM (512 columns): O [0,128) | S/P buffer 0 [128,256) | S/P buffer 1 [256,384) |
//                     q~ latent fp16 [384,448) | q~ rope fp16 [448,480).
// Tile j scores into buffer j % 2, so QK(j+1) runs while the softmax works on S(j).  The
// softmax writes P(j) (fp16 pairs) over the first half of the score columns it read:
// half h's 64 scores at [64h, 64h+64) become 32 P columns at [64h, 64h+32).  Buffer j % 2
// is scored again (tile j+2) once P.V(j) has completed.
//
// Warp roles (15 warps):
//   0-3   softmax half 0 (thread = head row = TMEM lane): score columns [0, 64), O [0, 64)
//   4-7   softmax half 1: score columns [64, 128), O [64, 128); the halves agree on each
//         row's tile maximum through shared memory
//   8-11  converters: bf16 -> fp16 in place, rows past the sequence end zeroed
//   12    TMA producer
//   13    TMEM allocator + QK issuer
//   14    P.V issuer
// Every wait is bounded (sm100.cuh).  A wait that expires raises the CTA's abort flag
// and records the site in the status word; each MMA issuer then waits for its own
// MMAs and the producer for its own copies (with a fixed bound independent of the
// caller's limit) before TMEM is released.
#include <cstdint>

#include "decode_sm100.h"
#include "launch.h"
#include "schedule.cuh"
#include "sm100.cuh"

namespace hra {

namespace {

constexpr uint32_t kAll = 0xffffffffu;

struct SplitCfg {
  static constexpr int NT = 128;                  // tokens per tile
  static constexpr int STAGES = 4;                // tile ring depth (48 KB per stage)
  static constexpr int W = 128;                   // branch width
  static constexpr int BOXES = 3;                 // 64-column boxes per tile: 2 latent + 1 rope
  static constexpr int BOX_BYTES = NT * 128;
  static constexpr int STAGE_BYTES = BOXES * BOX_BYTES;
  static constexpr int STAGE_BYTES_I8 = 2 * BOX_BYTES;  // int8 cache: 128 bytes of latent + the rope box per row
  static constexpr int CHUNKS = NT / 32;          // TMA row chunks per box
  static constexpr int TMEM_O = 0;
  static constexpr int TMEM_S = 128;              // two buffers of NT columns
  static constexpr int TMEM_Q = TMEM_S + 2 * NT;  // latent query, fp16 pairs (W / 2 columns)
  static constexpr int TMEM_QR = TMEM_Q + W / 2;  // rope query, fp16 pairs (32 columns)
  static constexpr int TMEM_COLS = 512;
  static constexpr int SOFTMAX_WARPS = 8;
  static constexpr int CONV_WARPS = 4;
  static constexpr int WARP_PRODUCER = SOFTMAX_WARPS + CONV_WARPS;  // 12
  static constexpr int WARP_QK = WARP_PRODUCER + 1;                 // 13
  static constexpr int WARP_PV = WARP_QK + 1;                       // 14
  static constexpr int THREADS = 32 * (WARP_PV + 1);                // 480
  static constexpr int BAR_BYTES = 512;
  static constexpr int RED_BYTES = (2 * 2 * 128 + 2 * 128) * 4;
  static constexpr int SCALE_BYTES = STAGES * NT * 4;  // int8 cache: each stage's 128 row scales
  static constexpr int MISC_BYTES = BAR_BYTES + RED_BYTES + SCALE_BYTES + 4 * (kMaxBatch + 1);
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + MISC_BYTES;
  static_assert(TMEM_QR + 32 <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit, volatile int* abort,
                                          int* status, int where) {
  const bool ok = mbar_wait(bar, parity, limit, abort, status, where);
  return __all_sync(kAll, ok);
}

// Walks this CTA's tiles in order, segment by segment (a segment = the CTA's tiles of
// one sequence).
struct TileCursor {
  const int* prefix;
  int B, t_end;
  int s, j, j0, j1, seg;
  bool valid;
  __device__ void init(const int* prefix_, int B_, int t_begin, int t_end_, int s_first) {
    prefix = prefix_;
    B = B_;
    t_end = t_end_;
    seg = -1;
    s = s_first;
    valid = false;
    for (; s < B && prefix[s] < t_end; ++s) {
      j0 = max(t_begin, prefix[s]);
      j1 = min(t_end, prefix[s + 1]);
      if (j0 < j1) { j = j0; seg = 0; valid = true; return; }
    }
  }
  __device__ void advance() {
    if (++j < j1) return;
    for (++s; s < B && prefix[s] < t_end; ++s) {
      j0 = prefix[s];
      j1 = min(t_end, prefix[s + 1]);
      if (j0 < j1) { j = j0; ++seg; return; }
    }
    valid = false;
  }
  __device__ bool first() const { return j == j0; }
};

// One MMA issuer's exit: wait (bounded by kDrainNs, whatever the abort flag says) until
// every tcgen05 operation it issued has completed, so that TMEM and the tile ring can be
// released.
__device__ __forceinline__ void drain_mmas(uint64_t* bar, volatile int* never, int* status, int where) {
  umma_commit(bar);
  mbar_wait(bar, 0, kDrainNs, never, status, where);
}

// INT8: the latent cache is int8 with per-(row, 128-column block) scales (a.cache_int8 = 1).
template <bool INT8>
__global__ void __launch_bounds__(SplitCfg::THREADS, 1)
decode_split_kernel(const __grid_constant__ CUtensorMap map_ckv, const __grid_constant__ CUtensorMap map_krope,
                    const DecodeArgs a) {
  using C = SplitCfg;
  constexpr int NT = C::NT, STAGES = C::STAGES, HALF = NT / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* misc = tiles + STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty = full + STAGES;
  uint64_t* conv = empty + STAGES;    // [STAGES] the stage holds fp16
  uint64_t* s_full = conv + STAGES;   // [2] per S/P buffer
  uint64_t* p_ready = s_full + 2;     // [2]
  uint64_t* pv_done = p_ready + 2;    // [2]
  uint64_t* q_ready = pv_done + 2;
  uint64_t* red_bar = q_ready + 1;    // [2] row-max exchange between the softmax halves
  uint64_t* lsum_bar = red_bar + 2;   // row-sum exchange, once per segment
  uint64_t* drain = lsum_bar + 1;     // [2] one per MMA issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* never_flag = abort_flag + 1;  // stays 0: exit-path waits ignore the abort flag
  float* red_max = reinterpret_cast<float*>(misc + C::BAR_BYTES);  // [2 buf][2 half][128]
  float* red_l = red_max + 2 * 2 * 128;                              // [2 half][128]
  float* row_scale = reinterpret_cast<float*>(misc + C::BAR_BYTES + C::RED_BYTES);  // [STAGES][NT]
  int* prefix = reinterpret_cast<int*>(misc + C::BAR_BYTES + C::RED_BYTES + C::SCALE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int slice = blockIdx.x;  // = branch
  const int G = gridDim.y;
  const int g = blockIdx.y;
  const int B = a.batch;
  const uint64_t limit = a.wait_limit_ns;
  int* status = a.status;

  if (warp == 0) tile_prefix_warp(a.seq_lens, B, NT, prefix);
  if (threadIdx.x == 0) grid_dep_launch();
  if (threadIdx.x == 32) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&conv[i], C::CONV_WARPS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_ready[b], C::SOFTMAX_WARPS);
      mbar_init(&pv_done[b], 1);
      mbar_init(&red_bar[b], C::SOFTMAX_WARPS);
      mbar_init(&drain[b], 1);
    }
    mbar_init(q_ready, C::SOFTMAX_WARPS);
    mbar_init(lsum_bar, C::SOFTMAX_WARPS);
    *abort_flag = 0;
    *never_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::WARP_QK) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::WARP_PRODUCER && lane == 0) {
    tma_prefetch_desc(&map_ckv);
    tma_prefetch_desc(&map_krope);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int T = prefix[B];
  const int t_begin = T > 0 ? group_tile_begin(g, G, T) : 0;
  const int t_end = T > 0 ? group_tile_begin(g + 1, G, T) : 0;
  const int s_first = (t_begin < t_end) ? seq_of_tile(prefix, B, t_begin) : B;

  if (warp == C::WARP_PRODUCER) {
    // ------------------------------------------------------------------ TMA producer
    // The CTA's tiles are the global tiles t_begin .. t_end-1 in order.  Each lane finds
    // the cache row of one 32-row chunk of a batch of 32 / CHUNKS tiles (block-table and
    // length loads in parallel), one batch ahead of the tiles lane 0 is issuing, so that
    // no dependent global load sits between two tiles' copies.
    constexpr int TPB = 32 / C::CHUNKS;
    const int ntiles = t_end - t_begin;
    const uint64_t policy = l2_policy_evict_first();
    auto chunk_row = [&](int it0) {
      const int t = t_begin + it0 + lane / C::CHUNKS;
      if (t >= t_end) return static_cast<int>(a.cache_rows);
      const int s = seq_of_tile(prefix, B, t);
      return cache_chunk_row(a, s, (t - prefix[s]) * NT + 32 * (lane % C::CHUNKS));
    };
    // int8 cache: the 32 block scales of this lane's chunk (0 for rows past the cache),
    // loaded one batch ahead like the rows themselves
    auto chunk_scales = [&](int crow, float* sc) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        sc[i] = crow + i < a.cache_rows ? a.ckv_scale[(static_cast<long long>(crow) + i) * a.scale_stride + slice]
                                        : 0.f;
    };
    int rows = chunk_row(0);
    float sc[INT8 ? 32 : 1];
    if constexpr (INT8) chunk_scales(rows, sc);
    int issued = 0;
    bool ok = true;
    for (int it0 = 0; ok && it0 < ntiles; it0 += TPB) {
      const int rows_next = chunk_row(it0 + TPB);
      float sc_next[INT8 ? 32 : 1];
      if constexpr (INT8) chunk_scales(rows_next, sc_next);
      for (int k = 0; k < TPB && it0 + k < ntiles; ++k) {
        const int it = it0 + k, stage = it % STAGES;
        if (it >= STAGES && !warp_wait(&empty[stage], ((it / STAGES) + 1) & 1, limit, abort_flag, status, 1)) {
          ok = false;
          break;
        }
        int y[C::CHUNKS];
#pragma unroll
        for (int r = 0; r < C::CHUNKS; ++r) y[r] = __shfl_sync(kAll, rows, k * C::CHUNKS + r);
        if (INT8 && lane / C::CHUNKS == k) {
          // the stage's row scales, written before the stage is armed (the arrive below
          // releases them to the converters' wait on full)
          float4* dst = reinterpret_cast<float4*>(row_scale + stage * NT + 32 * (lane % C::CHUNKS));
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_float4(sc[4 * i], sc[4 * i + 1], sc[4 * i + 2], sc[4 * i + 3]);
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[stage], INT8 ? C::STAGE_BYTES_I8 : C::STAGE_BYTES);
          uint8_t* dst = tiles + stage * C::STAGE_BYTES;
#pragma unroll
          for (int r = 0; r < C::CHUNKS; ++r) {
            if constexpr (INT8) {  // the branch's 128 int8 columns land where latent box 1 goes
              tma_load_2d(dst + C::BOX_BYTES + r * 4096, &map_ckv, &full[stage], slice * C::W, y[r], policy);
            } else {
#pragma unroll
              for (int d = 0; d < C::BOXES - 1; ++d)
                tma_load_2d(dst + d * C::BOX_BYTES + r * 4096, &map_ckv, &full[stage], slice * C::W + 64 * d, y[r],
                            policy);
            }
            tma_load_2d(dst + 2 * C::BOX_BYTES + r * 4096, &map_krope, &full[stage], 0, y[r], policy);
          }
        }
        __syncwarp();
        issued = it + 1;
      }
      rows = rows_next;
      if constexpr (INT8) {
#pragma unroll
        for (int i = 0; i < 32; ++i) sc[i] = sc_next[i];
      }
    }
    for (int k = max(0, issued - STAGES); k < issued; ++k) {  // every stage must come back
      if (ok && !warp_wait(&empty[k % STAGES], (k / STAGES) & 1, limit, abort_flag, status, 2)) ok = false;
      if (!ok) {  // aborted: wait (bounded, ignoring the abort flag) for the copy itself
        warp_wait(&full[k % STAGES], (k / STAGES) & 1, kDrainNs, never_flag, status, 3);
      }
    }
  } else if (warp == C::WARP_QK) {
    // ------------------------------------------------------------------ QK issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, NT, false);
      const uint32_t tiles_addr = smem_u32(tiles);
      TileCursor qc;
      qc.init(prefix, B, t_begin, t_end, s_first);
      for (int qi = 0; qc.valid; qc.advance(), ++qi) {
        const int b = qi & 1;
        // the tile is fp16 in shared memory, P.V of tile qi-2 (which read buffer b) has
        // completed, and (first tile of a segment) the segment's query is in TMEM
        if (!mbar_wait(&conv[qi % STAGES], (qi / STAGES) & 1, limit, abort_flag, status, 11) ||
            (qi >= 2 && !mbar_wait(&pv_done[b], ((qi - 2) >> 1) & 1, limit, abort_flag, status, 12)) ||
            (qc.first() && !mbar_wait(q_ready, qc.seg & 1, limit, abort_flag, status, 10)))
          break;
        tc_fence_after();
        const uint32_t k_base = tiles_addr + (qi % STAGES) * C::STAGE_BYTES;
        const uint32_t d_tmem = tmem + C::TMEM_S + b * NT;
#pragma unroll
        for (int k = 0; k < C::W / 16; ++k) {  // latent: boxes 0, 1
          const uint64_t bdesc = smem_desc_sw128(k_base + (k >> 2) * C::BOX_BYTES + (k & 3) * 32, 16, 1024);
          umma_f16_ts(d_tmem, tmem + C::TMEM_Q + k * 8, bdesc, idesc, k > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // rope: box 2
          const uint64_t bdesc = smem_desc_sw128(k_base + 2 * C::BOX_BYTES + k * 32, 16, 1024);
          umma_f16_ts(d_tmem, tmem + C::TMEM_QR + k * 8, bdesc, idesc, 1u);
        }
        umma_commit(&s_full[b]);
      }
      drain_mmas(&drain[0], never_flag, status, 14);
    }
    __syncwarp();
  } else if (warp == C::WARP_PV) {
    // ------------------------------------------------------------------ P.V issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, 128, true);
      const uint32_t tiles_addr = smem_u32(tiles);
      TileCursor pc;
      pc.init(prefix, B, t_begin, t_end, s_first);
      for (int pi = 0; pc.valid; pc.advance(), ++pi) {
        const int b = pi & 1;
        if (!mbar_wait(&p_ready[b], (pi >> 1) & 1, limit, abort_flag, status, 13)) break;
        tc_fence_after();
        const int stage = pi % STAGES;
        const uint32_t v_base = tiles_addr + stage * C::STAGE_BYTES;  // this branch's latent = boxes 0, 1
        const uint32_t p_base = tmem + C::TMEM_S + b * NT;
        const bool first = pc.first();
#pragma unroll
        for (int k = 0; k < NT / 16; ++k) {
          // tokens [16k, 16k+16): P columns of half k / 4 start at 64 (k / 4)
          const uint32_t a_tmem = p_base + 64 * (k >> 2) + 8 * (k & 3);
          const uint64_t bdesc = smem_desc_sw128(v_base + k * 16 * 128, C::BOX_BYTES, 1024);
          umma_f16_ts(tmem + C::TMEM_O, a_tmem, bdesc, idesc, (first && k == 0) ? 0u : 1u);
        }
        umma_commit(&pv_done[b]);
        // P.V(tile) completing implies QK(tile) completed (its S was read before P
        // existed), so the stage may be refilled.
        umma_commit(&empty[stage]);
      }
      drain_mmas(&drain[1], never_flag, status, 15);
    }
    __syncwarp();
  } else if (warp >= C::SOFTMAX_WARPS) {
    // ------------------------------------------------------------------ converters
    // Rewrites each arrived stage (3 boxes x 128 rows x 128 B, swizzled 16-byte chunks
    // within each row) as fp16 in place.  Rows at or past the sequence end hold whatever
    // the cache holds there; they are zeroed so that neither their scores (masked by the
    // softmax) nor 0 * Inf / NaN in P.V can reach O.  An int8 cache arrives as one 128-byte
    // row per token in latent box 1's place; thread ct then expands row ct: it reads the
    // row's 8 chunks, scales them by the row's block scale and writes 16 fp16 chunks over
    // boxes 0 and 1 (and converts the row's rope chunks).
    const int ct = threadIdx.x - 32 * C::SOFTMAX_WARPS;  // 0..127
    TileCursor cc;
    cc.init(prefix, B, t_begin, t_end, s_first);
    int L = cc.valid ? a.seq_lens[cc.s] : 0;
    int cur_s = cc.s;
    for (int it = 0; cc.valid; cc.advance(), ++it) {
      if (cc.s != cur_s) {
        cur_s = cc.s;
        L = a.seq_lens[cur_s];
      }
      const int stage = it % STAGES;
      const int n_valid = min(NT, L - (cc.j - prefix[cc.s]) * NT);
      uint8_t* st = tiles + stage * C::STAGE_BYTES;
      if constexpr (INT8) {
        const int r = ct;
        if (!warp_wait(&full[stage], (it / STAGES) & 1, limit, abort_flag, status, 20)) break;
        const float scale = row_scale[stage * NT + r];  // written by the producer with the stage
        const int sw = r & 7;
        const __half2 s2 = __float2half2_rn(scale);
        // Two halves of 4 chunks: the first half writes box 0 only; the second reads its
        // chunks (and the first half has read its own) before box 1 is overwritten.
#pragma unroll 1
        for (int c0 = 0; c0 < 8; c0 += 4) {
          uint4 raw[4];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            raw[c] = *reinterpret_cast<const uint4*>(st + C::BOX_BYTES + r * 128 + (((c0 + c) ^ sw) << 4));
#pragma unroll
          for (int c = 0; c < 4; ++c) {  // int8 columns [16 (c0+c), +16) -> fp16 chunks 2 (c0+c), 2 (c0+c) + 1
            const uint32_t wv[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
            uint32_t h[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint2 f = i8x4_to_f16x4(wv[q], s2);
              h[2 * q] = f.x;
              h[2 * q + 1] = f.y;
            }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const int j = 2 * (c0 + c) + k;
              const uint4 v = r < n_valid ? make_uint4(h[4 * k], h[4 * k + 1], h[4 * k + 2], h[4 * k + 3])
                                          : make_uint4(0u, 0u, 0u, 0u);
              *reinterpret_cast<uint4*>(st + (j >> 3) * C::BOX_BYTES + r * 128 + (((j & 7) ^ sw) << 4)) = v;
            }
          }
        }
        uint4* rope = reinterpret_cast<uint4*>(st + 2 * C::BOX_BYTES + r * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 v = rope[c];
          if (r < n_valid) {
            v.x = bf16x2_to_f16x2(v.x);
            v.y = bf16x2_to_f16x2(v.y);
            v.z = bf16x2_to_f16x2(v.z);
            v.w = bf16x2_to_f16x2(v.w);
          } else {
            v = make_uint4(0u, 0u, 0u, 0u);
          }
          rope[c] = v;
        }
      } else {
        if (!warp_wait(&full[stage], (it / STAGES) & 1, limit, abort_flag, status, 20)) break;
        uint4* r = reinterpret_cast<uint4*>(st);
#pragma unroll 4
        for (int e = ct; e < C::STAGE_BYTES / 16; e += 32 * C::CONV_WARPS) {
          const int row = (e >> 3) & (NT - 1);
          uint4 v = r[e];
          if (row < n_valid) {
            v.x = bf16x2_to_f16x2(v.x);
            v.y = bf16x2_to_f16x2(v.y);
            v.z = bf16x2_to_f16x2(v.z);
            v.w = bf16x2_to_f16x2(v.w);
          } else {
            v = make_uint4(0u, 0u, 0u, 0u);
          }
          r[e] = v;
        }
      }
      fence_proxy_async_smem();
      warp_arrive(&conv[stage]);
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    // The absorbed query comes from the previous kernel, and the split partials written
    // here are read by the previous call's merge: wait for those grids.  The producer, the
    // converters and the MMA issuers touch no memory another kernel writes.
    grid_dep_wait();
    const int half = warp >> 2;           // score columns [half*HALF, +HALF), O columns [64 half, +64)
    const int row = threadIdx.x & 127;    // head row == TMEM lane
    const uint32_t t_row = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float sl2 = a.scale_log2;
    const int q_stride = a.d_c + 64;  // query row: d_c latent columns then the rope part
    TileCursor cur;
    cur.init(prefix, B, t_begin, t_end, s_first);
    int it = 0, seg = 0;
    bool ok = true;
    while (ok && cur.valid) {
      const int s = cur.s;
      const int L = a.seq_lens[s];
      // this head's query for the branch: half 0 stores the latent columns [128 slice, +128),
      // half 1 the rope part [d_c, d_c + 64)
      {
        const long long base = (static_cast<long long>(s) * a.heads + min(row, a.heads - 1)) * q_stride;
        const bool live = row < a.heads;
        const uint4* src = reinterpret_cast<const uint4*>(a.q_tilde + base + (half == 0 ? slice * C::W : a.d_c));
#pragma unroll 1
        for (int c = 0; c < 2 - half; ++c) {
          uint32_t w[32];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint4 v = live ? __ldg(src + 8 * c + u) : make_uint4(0u, 0u, 0u, 0u);
            w[4 * u + 0] = v.x; w[4 * u + 1] = v.y; w[4 * u + 2] = v.z; w[4 * u + 3] = v.w;
          }
          tmem_st32(t_row + (half == 0 ? C::TMEM_Q + 32 * c : C::TMEM_QR), w);
        }
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(q_ready);
      }
      float m_ref = -INFINITY, l = 0.f;
      const int seg_j1 = cur.j1;
      for (; cur.valid && cur.s == s && cur.j < seg_j1; cur.advance(), ++it) {
        const int b = it & 1;
        if (!warp_wait(&s_full[b], (it >> 1) & 1, limit, abort_flag, status, 30)) { ok = false; break; }
        tc_fence_after();
        const bool first = cur.first();
        const int n_valid = min(NT, L - (cur.j - prefix[s]) * NT);
        const int n_mine = min(max(n_valid - half * HALF, 0), HALF);
        const uint32_t s_cols = t_row + C::TMEM_S + b * NT + half * HALF;
        uint32_t sr[HALF];
        tmem_load<HALF>(s_cols, sr);
        tmem_ld_wait();
        if (n_mine < HALF) {
#pragma unroll
          for (int k = 0; k < HALF; ++k)
            if (k >= n_mine) sr[k] = __float_as_uint(-INFINITY);
        }
        float mx[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) mx[q] = __uint_as_float(sr[q]);
#pragma unroll
        for (int k = 4; k + 8 <= HALF; k += 8)
#pragma unroll
          for (int q = 0; q < 4; ++q) mx[q] = fmax3(mx[q], __uint_as_float(sr[k + q]), __uint_as_float(sr[k + 4 + q]));
        const int rb = it & 1;
        float mt4 = fmaxf(mx[0], mx[1]);
#pragma unroll
        for (int q = 0; q < 4; ++q) mt4 = fmax3(mt4, mx[q], __uint_as_float(sr[HALF - 4 + q]));
        red_max[(rb * 2 + half) * 128 + row] = mt4;

        warp_arrive(&red_bar[rb]);
        if (!warp_wait(&red_bar[rb], (it >> 1) & 1, limit, abort_flag, status, 33)) { ok = false; break; }
        const float mt = fmaxf(red_max[(rb * 2) * 128 + row], red_max[(rb * 2 + 1) * 128 + row]) * sl2;
        float factor = 1.f;
        bool rescale = false;
        if (first) {
          m_ref = mt;
        } else if (mt > m_ref + 8.f) {  // lazy rescale: keep the reference unless it grew by 2^8
          factor = ex2_approx(m_ref - mt);
          m_ref = mt;
          rescale = true;
        }
        const float2 neg_m = make_float2(-m_ref, -m_ref);
        const float2 sl2v = make_float2(sl2, sl2);
        float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < HALF / 2; ++k) {
          const float2 x = fma2(make_float2(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1])), sl2v, neg_m);
          const float2 pk = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          if (k & 1) s1 = add2(s1, pk); else s0 = add2(s0, pk);
          sr[k] = pack_f16x2(pk.x, pk.y);
        }
        const float2 st = add2(s0, s1);
        const float tsum = st.x + st.y;
        l = first ? tsum : fmaf(l, factor, tsum);
        if (__any_sync(kAll, rescale)) {
          // every P.V so far must have completed before O is rescaled
          if (!warp_wait(&pv_done[b ^ 1], ((it - 1) >> 1) & 1, limit, abort_flag, status, 31)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int k = 0; k < 4; ++k) {  // 16 columns at a time: the packed P stays in registers
            uint32_t o[16];
            const uint32_t oaddr = t_row + C::TMEM_O + 64 * half + 16 * k;
            tmem_ld16(oaddr, o);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 16; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * factor);
            tmem_st16(oaddr, o);
          }
        }
        tmem_st32(s_cols, sr);  // P over the first 32 of this half's score columns
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(&p_ready[b]);
      }
      if (!ok) break;
      if (!warp_wait(&pv_done[(it - 1) & 1], ((it - 1) >> 1) & 1, limit, abort_flag, status, 32)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const long long slot = static_cast<long long>(g) + s;
      float4* dst =
          reinterpret_cast<float4*>(a.o_part + ((slot * gridDim.x + slice) * 128 + row) * 128 + 64 * half);
#pragma unroll 1
      for (int k = 0; k < 2; ++k) {
        uint32_t o[32];
        tmem_ld32(t_row + C::TMEM_O + 64 * half + 32 * k, o);
        tmem_ld_wait();
        if (row < a.heads) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            dst[k * 8 + u] = make_float4(__uint_as_float(o[4 * u]), __uint_as_float(o[4 * u + 1]),
                                         __uint_as_float(o[4 * u + 2]), __uint_as_float(o[4 * u + 3]));
        }
      }
      // the row sum is split across the halves: add them once per segment
      red_l[half * 128 + row] = l;
      warp_arrive(lsum_bar);
      if (!warp_wait(lsum_bar, seg & 1, limit, abort_flag, status, 34)) { ok = false; break; }
      ++seg;
      if (half == 0 && row < a.heads)
        a.ml_part[(slot * gridDim.x + slice) * 128 + row] = make_float2(m_ref, l + red_l[128 + row]);
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_QK) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace

int decode_split_tile_tokens() { return SplitCfg::NT; }

cudaError_t launch_decode_split_kernel(const CUtensorMap& map_ckv, const CUtensorMap& map_krope,
                                       const DecodeArgs& a, int groups, cudaStream_t stream, bool pdl) {
  using C = SplitCfg;
  auto kern = a.cache_int8 ? decode_split_kernel<true> : decode_split_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, dim3(a.d_c / 128, groups), dim3(C::THREADS), C::SMEM_BYTES, stream, pdl, map_ckv,
                       map_krope, a);
}

}  // namespace hra

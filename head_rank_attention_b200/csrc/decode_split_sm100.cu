// decode_split_sm100.cu -- split-KV MLRA-4 decode reading the bf16 cache straight into
// the tensor cores.
//
// Same computation and work decomposition as decode_sm100.cu (step 2 of "Multi-Head
// Low-Rank Attention", 方法步骤详情; one CTA per 128-wide latent slice = one MLRA-4
// branch, groups of d_c / 128 CTAs over contiguous tile ranges: 4 for MLRA-4, fewer when
// the call holds a shard of the branches), but the latent part of the
// cache tile is never rewritten: the absorbed query is carried as two bf16 terms
// q~ = q_hi + q_lo (q_lo = bf16(q~ - q_hi), together ~16 significant bits), and every
// latent score is the fp32 sum of two bf16 MMAs against the same bf16 tile.  The rope
// part is scored once in fp16: a converter warp rewrites the tile's 64-column rope box
// as fp16 in place and the rope query is fp16.  P is rounded to bf16 for P.V.
//
// TMEM (512 columns, NT = 128): O [0,128) | S [128,256) | P (bf16 pairs) [256,320) |
//                               q_hi [320,384) | q_lo [384,448) | q_rope fp16 [448,480).
// S and P are separate buffers: the QK of tile j+1 may start as soon as the softmax has
// copied S(j) into registers, and P(j+1) is written once P.V of tile j has completed.
//
// Warp roles (12 warps):
//   0-3  softmax half 0 (thread = head row = TMEM lane): score columns [0, NT/2), O [0, 64)
//   4-7  softmax half 1: score columns [NT/2, NT), O [64, 128); the halves agree on each
//        row's tile max through shared memory
//   8    TMA producer
//   9    TMEM allocator + QK issuer
//   10   P.V issuer
//   11   rope-box converter (bf16 -> fp16)
// The two MMA streams touch disjoint TMEM (S vs P and O), so a burst of QK instructions
// waiting for the tensor pipe never delays the P.V that a finished softmax released.
#include <cstdint>

#include "decode_sm100.h"
#include "launch.h"
#include "schedule.cuh"
#include "sm100.cuh"

namespace hra {

namespace {

constexpr uint32_t kAll = 0xffffffffu;
constexpr int kNT = 128;      // tokens per tile
constexpr int kStages = 4;    // tile ring depth (48 KB per stage)

template <int NT_, int STAGES_>
struct SplitCfg {
  static constexpr int NT = NT_;
  static constexpr int STAGES = STAGES_;
  static constexpr int W = 128;                   // MLRA-4 branch width
  static constexpr int QK_DIMS = W + 64;          // 192
  static constexpr int QK_BOXES = QK_DIMS / 64;   // 3 (2 latent + 1 rope)
  static constexpr int BOX_BYTES = NT * 128;
  static constexpr int STAGE_BYTES = QK_BOXES * BOX_BYTES;
  static constexpr int CHUNKS = NT / 32;
  static constexpr int TMEM_O = 0;
  static constexpr int TMEM_S = 128;
  static constexpr int TMEM_P = TMEM_S + NT;
  static constexpr int TMEM_QH = TMEM_P + NT / 2;  // latent query, bf16 hi term (W/2 columns)
  static constexpr int TMEM_QL = TMEM_QH + W / 2;  // latent query, bf16 lo term
  static constexpr int TMEM_QR = TMEM_QL + W / 2;  // rope query, fp16 (32 columns)
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 384;
  static constexpr int BAR_BYTES = 512;
  static constexpr int RED_BYTES = (2 * 2 * 128 + 2 * 128) * 4;
  static constexpr int MISC_BYTES = BAR_BYTES + RED_BYTES + 4 * (kMaxBatch + 1);
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + MISC_BYTES;
  static_assert(TMEM_QR + 32 <= TMEM_COLS, "TMEM budget");
  static_assert(NT % 32 == 0 && NT <= 128, "tile rows");
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

template <int NT_, int STAGES_>
__global__ void __launch_bounds__(384, 1)
decode_split_kernel(const __grid_constant__ CUtensorMap map_ckv, const __grid_constant__ CUtensorMap map_krope,
                    const DecodeArgs a) {
  using C = SplitCfg<NT_, STAGES_>;
  constexpr int NT = C::NT, STAGES = C::STAGES, HALF = NT / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* misc = tiles + STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty = full + STAGES;
  uint64_t* s_full = empty + STAGES;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_ready = s_free + 1;
  uint64_t* pv_done = p_ready + 1;
  uint64_t* q_ready = pv_done + 1;
  uint64_t* red_bar = q_ready + 1;   // [2] row-max exchange between the softmax halves
  uint64_t* lsum_bar = red_bar + 2;  // row-sum exchange, once per segment
  uint64_t* drain = lsum_bar + 1;    // [2] one per MMA issuer
  uint64_t* conv = drain + 2;        // [STAGES] the stage's rope box is fp16
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(conv + STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red_max = reinterpret_cast<float*>(misc + C::BAR_BYTES);  // [2 buf][2 half][128]
  float* red_l = red_max + 2 * 2 * 128;                              // [2 half][128]
  int* prefix = reinterpret_cast<int*>(misc + C::BAR_BYTES + C::RED_BYTES);

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
      mbar_init(&conv[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);
    mbar_init(p_ready, 8);
    mbar_init(pv_done, 1);
    mbar_init(q_ready, 8);
    mbar_init(&red_bar[0], 8);
    mbar_init(&red_bar[1], 8);
    mbar_init(lsum_bar, 8);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
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

  if (warp == 8) {
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
    int rows = chunk_row(0);
    int issued = 0;
    bool ok = true;
    for (int it0 = 0; ok && it0 < ntiles; it0 += TPB) {
      const int rows_next = chunk_row(it0 + TPB);
      for (int k = 0; k < TPB && it0 + k < ntiles; ++k) {
        const int it = it0 + k, stage = it % STAGES;
        if (it >= STAGES && !warp_wait(&empty[stage], ((it / STAGES) + 1) & 1, limit, abort_flag, status, 1)) {
          ok = false;
          break;
        }
        int y[C::CHUNKS];
#pragma unroll
        for (int r = 0; r < C::CHUNKS; ++r) y[r] = __shfl_sync(kAll, rows, k * C::CHUNKS + r);
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          uint8_t* dst = tiles + stage * C::STAGE_BYTES;
#pragma unroll
          for (int r = 0; r < C::CHUNKS; ++r) {
#pragma unroll
            for (int d = 0; d < C::QK_BOXES; ++d) {
              void* box = dst + d * C::BOX_BYTES + r * 4096;
              if (d < C::QK_BOXES - 1)
                tma_load_2d(box, &map_ckv, &full[stage], slice * C::W + 64 * d, y[r], policy);
              else
                tma_load_2d(box, &map_krope, &full[stage], 0, y[r], policy);
            }
          }
        }
        __syncwarp();
        issued = it + 1;
      }
      rows = rows_next;
    }
    for (int k = max(0, issued - STAGES); k < issued; ++k) {  // every stage must come back
      if (ok && !warp_wait(&empty[k % STAGES], (k / STAGES) & 1, limit, abort_flag, status, 2)) ok = false;
      if (!ok) {  // aborted: wait (bounded, ignoring the abort flag) for the copy itself
        volatile int never = 0;
        warp_wait(&full[k % STAGES], (k / STAGES) & 1, limit, &never, status, 3);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ QK issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, NT, false);
      constexpr uint32_t idesc_rope = idesc_f16_f32(128, NT, false);
      const uint32_t tiles_addr = smem_u32(tiles);
      TileCursor qc;
      qc.init(prefix, B, t_begin, t_end, s_first);
      bool ok = true;
      for (int qi = 0; qc.valid; qc.advance(), ++qi) {
        // the tile has landed, the softmax has copied the previous S out of TMEM, and (first
        // tile of a segment) the segment's query is in TMEM
        if (!mbar_wait(&full[qi % STAGES], (qi / STAGES) & 1, limit, abort_flag, status, 11) ||
            (qi >= 1 && !mbar_wait(s_free, (qi - 1) & 1, limit, abort_flag, status, 12)) ||
            (qc.first() && !mbar_wait(q_ready, qc.seg & 1, limit, abort_flag, status, 10))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_base = tiles_addr + (qi % STAGES) * C::STAGE_BYTES;
        const uint32_t d_tmem = tmem + C::TMEM_S;
#pragma unroll
        for (int k = 0; k < C::W / 16; ++k) {  // latent part: bf16 cache x two bf16 query terms
          const uint64_t bdesc = smem_desc_sw128(k_base + (k >> 2) * C::BOX_BYTES + (k & 3) * 32, 16, 1024);
          umma_f16_ts(d_tmem, tmem + C::TMEM_QH + k * 8, bdesc, idesc_qk, k > 0 ? 1u : 0u);
          umma_f16_ts(d_tmem, tmem + C::TMEM_QL + k * 8, bdesc, idesc_qk, 1u);
        }
        // rope part: the converter warp has rewritten the stage's rope box as fp16
        if (!mbar_wait(&conv[qi % STAGES], (qi / STAGES) & 1, limit, abort_flag, status, 16)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t bdesc = smem_desc_sw128(k_base + 2 * C::BOX_BYTES + k * 32, 16, 1024);
          umma_f16_ts(d_tmem, tmem + C::TMEM_QR + k * 8, bdesc, idesc_rope, 1u);
        }
        umma_commit(s_full);
      }
      if (!ok) {
        umma_commit(&drain[0]);
        volatile int never = 0;
        mbar_wait(&drain[0], 0, limit, &never, status, 14);
      }
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------------ P.V issuer
    if (lane == 0) {
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, true);
      const uint32_t tiles_addr = smem_u32(tiles);
      TileCursor pc;
      pc.init(prefix, B, t_begin, t_end, s_first);
      bool ok = true;
      for (int pi = 0; pc.valid; pc.advance(), ++pi) {
        if (!mbar_wait(p_ready, pi & 1, limit, abort_flag, status, 13)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int stage = pi % STAGES;
        const uint32_t v_base = tiles_addr + stage * C::STAGE_BYTES;  // this branch's latent = boxes 0,1
        const bool first = pc.first();
#pragma unroll
        for (int k = 0; k < NT / 16; ++k) {
          const uint64_t bdesc = smem_desc_sw128(v_base + k * 16 * 128, C::BOX_BYTES, 1024);
          umma_f16_ts(tmem + C::TMEM_O, tmem + C::TMEM_P + k * 8, bdesc, idesc_pv, (first && k == 0) ? 0u : 1u);
        }
        umma_commit(pv_done);
        // P.V(tile) completing implies QK(tile) completed (its S was read before P existed),
        // so this stage may be refilled.
        umma_commit(&empty[stage]);
      }
      if (!ok) {
        umma_commit(&drain[1]);
        volatile int never = 0;
        mbar_wait(&drain[1], 0, limit, &never, status, 15);
      }
    }
  } else if (warp == 11) {
    // ------------------------------------------------------------------ rope converter
    // Rewrites each stage's rope box (bf16 K_R, 128 rows x 64) as fp16 in place, for the
    // fp16 rope MMAs.  The conversion is exact for |values| < 65504.
    const int ntiles = t_end - t_begin;
    for (int it = 0; it < ntiles; ++it) {
      const int stage = it % STAGES;
      if (!warp_wait(&full[stage], (it / STAGES) & 1, limit, abort_flag, status, 20)) break;
      uint4* r = reinterpret_cast<uint4*>(tiles + stage * C::STAGE_BYTES + 2 * C::BOX_BYTES);
#pragma unroll 4
      for (int e = lane; e < C::BOX_BYTES / 16; e += 32) {
        uint4 v = r[e];
        v.x = bf16x2_to_f16x2(v.x);
        v.y = bf16x2_to_f16x2(v.y);
        v.z = bf16x2_to_f16x2(v.z);
        v.w = bf16x2_to_f16x2(v.w);
        r[e] = v;
      }
      fence_proxy_async_smem();
      warp_arrive(&conv[stage]);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax + epilogue
    // The absorbed query comes from the previous kernel, and the split partials written
    // here are read by the previous call's merge: wait for those grids.  The producer and
    // the MMA issuers touch no memory another kernel writes.
    grid_dep_wait();
    const int half = warp >> 2;           // score columns [half*HALF, +HALF), O columns [64 half, +64)
    const int row = threadIdx.x & 127;    // head row == TMEM lane
    const uint32_t t_row = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float sl2 = a.scale_log2;
    const __nv_bfloat16* q_hi = reinterpret_cast<const __nv_bfloat16*>(a.q_tilde);
    const int q_stride = a.d_c + 64;  // query row: d_c latent columns then the rope part
    const __nv_bfloat16* q_lo = q_hi + static_cast<long long>(a.batch) * a.heads * q_stride;
    TileCursor cur;
    cur.init(prefix, B, t_begin, t_end, s_first);
    int it = 0, seg = 0;
    bool ok = true;
    while (ok && cur.valid) {
      const int s = cur.s;
      const int L = a.seq_lens[s];
      // this head's query for the branch: latent columns [128 slice, +128) then rope [d_c, d_c + 64);
      // half 0 stores q_hi, half 1 stores q_lo
      {
        const long long base = (static_cast<long long>(s) * a.heads + min(row, a.heads - 1)) * q_stride;
        const bool live = row < a.heads;
        const uint4* src = reinterpret_cast<const uint4*>((half == 0 ? q_hi : q_lo) + base);
        const uint32_t col = half == 0 ? C::TMEM_QH : C::TMEM_QL;
#pragma unroll 1
        for (int c = 0; c < 2 + (half == 0); ++c) {  // latent chunks, then (half 0) the fp16 rope
          const int e0 = c < 2 ? slice * 128 + 64 * c : a.d_c;  // 16-bit element
          uint32_t w[32];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint4 v = live ? __ldg(src + (e0 >> 3) + u) : make_uint4(0u, 0u, 0u, 0u);
            w[4 * u + 0] = v.x; w[4 * u + 1] = v.y; w[4 * u + 2] = v.z; w[4 * u + 3] = v.w;
          }
          tmem_st32(t_row + (c < 2 ? col + 32 * c : C::TMEM_QR), w);
        }
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(q_ready);
      }
      float m_ref = -INFINITY, l = 0.f;
      const int seg_j1 = cur.j1;
      for (; cur.valid && cur.s == s && cur.j < seg_j1; cur.advance(), ++it) {
        if (!warp_wait(s_full, it & 1, limit, abort_flag, status, 30)) { ok = false; break; }
        tc_fence_after();
        const bool first = cur.first();
        const int n_valid = min(NT, L - (cur.j - prefix[s]) * NT);
        const int n_mine = min(max(n_valid - half * HALF, 0), HALF);
        uint32_t sr[HALF];
        tmem_load<HALF>(t_row + C::TMEM_S + half * HALF, sr);
        tmem_ld_wait();
        tc_fence_before();
        warp_arrive(s_free);  // the QK issuer may overwrite S once both halves got here
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (n_mine == HALF) {
#pragma unroll
          for (int k = 0; k < HALF; ++k) mx[k & 3] = fmaxf(mx[k & 3], __uint_as_float(sr[k]));
        } else {
#pragma unroll
          for (int k = 0; k < HALF; ++k) {
            if (k >= n_mine) sr[k] = __float_as_uint(-INFINITY);
            mx[k & 3] = fmaxf(mx[k & 3], __uint_as_float(sr[k]));
          }
        }
        const int rb = it & 1;
        red_max[(rb * 2 + half) * 128 + row] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
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
        const float neg_m = -m_ref;
        float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < HALF / 2; ++k) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(sr[2 * k]), sl2, neg_m));
          const float p1 = ex2_approx(fmaf(__uint_as_float(sr[2 * k + 1]), sl2, neg_m));
          sum[k & 3] += p0 + p1;
          sr[k] = pack_bf16x2(p0, p1);
        }
        const float tsum = (sum[0] + sum[1]) + (sum[2] + sum[3]);
        l = first ? tsum : fmaf(l, factor, tsum);
        if (!first) {
          // P.V of the previous tile must have completed: it reads the P buffer and O.
          if (!warp_wait(pv_done, (it - 1) & 1, limit, abort_flag, status, 31)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(kAll, rescale)) {
#pragma unroll 1
            for (int k = 0; k < 2; ++k) {
              uint32_t o[32];
              const uint32_t oaddr = t_row + C::TMEM_O + 64 * half + 32 * k;
              tmem_ld32(oaddr, o);
              tmem_ld_wait();
#pragma unroll
              for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * factor);
              tmem_st32(oaddr, o);
            }
          }
        }
        if (n_valid < NT) {
          // Rows at or past the sequence end hold whatever the cache holds there.  Their P
          // is zero, but 0 * Inf or NaN would still reach O: clear them in this stage's V.
          uint8_t* v = tiles + (it % STAGES) * C::STAGE_BYTES;
          for (int e = threadIdx.x; e < (NT - n_valid) * 16; e += 256) {
            const int r = n_valid + (e >> 4), box = (e >> 3) & 1;
            *reinterpret_cast<uint4*>(v + box * C::BOX_BYTES + r * 128 + (e & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();  // visible to the P.V MMAs that p_ready releases
        }
        tmem_store<HALF / 2>(t_row + C::TMEM_P + half * (HALF / 2), sr);
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(p_ready);
      }
      if (!ok) break;
      if (!warp_wait(pv_done, (it - 1) & 1, limit, abort_flag, status, 32)) { ok = false; break; }
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
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace

int decode_split_tile_tokens() { return kNT; }

cudaError_t launch_decode_split_kernel(const CUtensorMap& map_ckv, const CUtensorMap& map_krope,
                                       const DecodeArgs& a, int groups, cudaStream_t stream, bool pdl) {
  using C = SplitCfg<kNT, kStages>;
  auto kern = decode_split_kernel<kNT, kStages>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, dim3(a.d_c / 128, groups), dim3(C::THREADS), C::SMEM_BYTES, stream, pdl, map_ckv,
                       map_krope, a);
}

}  // namespace hra

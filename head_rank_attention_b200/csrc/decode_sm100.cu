// decode_sm100.cu -- split-KV latent-cache decode on tcgen05/TMEM with TMA tile streams.
//
// Step 2 of the decode in "Multi-Head Low-Rank Attention" (方法步骤详情): MQA-style
// attention of the absorbed per-head queries over the shared key [C_KV | K_RoPE] and
// value C_KV, one independent softmax per (head, branch) (核心方法:
// O = sum_b Softmax(Q K_b^T) V_b; MLA is the single-branch case).  This kernel serves
// branches 512 wide (NB = 1: MLA) and 256 wide (NB = 2: MLRA-2, or a call holding one
// 256-wide latent group: a rank of MLRA-2 split by branch, or of GLA-2); 128-wide branches
// run decode_split_sm100.cu.
//
// Work decomposition (one CTA per SM):
//   blockIdx.x = slice c in 0..d_c/128-1: the CTA owns output latent columns [128c, 128c+128),
//                which belong to branch b = c / (W/128) of width W = 512/NB;
//   blockIdx.y = group g: a contiguous range of cache tiles (see schedule.cuh).
// A CTA streams, for every tile of NT tokens (48 for MLA, 80 for 256-wide branches), the
// branch's W latent columns plus the 64 RoPE columns (TMA, 64-column boxes of 16 rows,
// 128-byte swizzle), converts them to fp16 in shared memory, computes
// S = Q~_b [C_b | K_R]^T for all 128 head rows with tcgen05 (A = Q~
// from TMEM, B = the tile, D = S in TMEM), runs the online softmax, writes P (fp16) back
// over S in TMEM and accumulates O += P V with V = its 128 latent columns of the same
// tile (A = P from TMEM, B = MN-major tile).  Each segment ends by writing the
// un-normalised O row, the running max m (log2 units) and the row sum l of every head.
//
// Warp roles (14 warps):
//   0-3   softmax half 0: TMEM lane = head row, score columns [0, NT/2), O columns [0, 64)
//   4-7   softmax half 1: same rows, score columns [NT/2, NT), O columns [64, 128)
//         (the two halves agree on every row's running max through shared memory)
//   8-11  bf16 -> fp16 conversion of each arrived tile (zeroing rows past the end)
//   12    TMA producer
//   13    TMEM allocator + MMA issuer (one elected thread)
// Every wait is bounded (see sm100.cuh); on expiry the CTA drains and exits with the
// failure recorded in the workspace status word.

#include <cstdint>

#include "decode_sm100.h"
#include "launch.h"
#include "schedule.cuh"
#include "sm100.cuh"

namespace hra {

template <int NB, int NT, int STAGES>
struct DecodeCfg {
  static constexpr int NT_ = NT;
  static constexpr int STAGES_ = STAGES;
  static constexpr int W = 512 / NB;                 // branch width
  static constexpr int QK_DIMS = W + 64;             // contraction length of one score
  static constexpr int QK_BOXES = QK_DIMS / 64;      // 64-wide boxes per tile (last = rope)
  static constexpr int SLICES_PER_BRANCH = W / 128;
  static constexpr int BOX_BYTES = NT * 128;         // one 64-column box over NT rows
  static constexpr int STAGE_BYTES = QK_BOXES * BOX_BYTES;
  static constexpr int CHUNK_ROWS = NT % 32 == 0 ? 32 : 16;  // rows of one TMA box
  static constexpr int CHUNKS = NT / CHUNK_ROWS;     // TMA row chunks per tile
  static constexpr int HALF = NT / 2;                // score columns per softmax thread
  static constexpr int TMEM_O = 0;                   // O: 128 fp32 columns
  static constexpr int TMEM_S = 128;                 // S/P double buffer: 2 x NT columns
  static constexpr int TMEM_Q = 128 + 2 * NT;        // Q~ (fp16 pairs): QK_DIMS/2 columns
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 448;
  // shared memory after the tile stages: barriers | row-max/row-sum exchange | tile prefix
  static constexpr int BAR_BYTES = 512;
  static constexpr int RED_BYTES = (2 * 2 * 128 + 2 * 128) * 4;
  static constexpr int MISC_BYTES = BAR_BYTES + RED_BYTES + 4 * (kMaxBatch + 1);
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + MISC_BYTES;
  static_assert(TMEM_Q + QK_DIMS / 2 <= TMEM_COLS, "TMEM budget");
  static_assert(NT % 16 == 0 && NT >= 32 && NT <= 256, "tile rows");
  static_assert(BOX_BYTES % 1024 == 0, "128-byte swizzle atoms");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

namespace {

constexpr uint32_t kFull = 0xffffffffu;

// All lanes of a warp poll; the result is made warp-uniform so that the .sync.aligned
// tcgen05 instructions and warp votes that follow see a converged warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit, volatile int* abort,
                                          int* status, int where) {
  const bool ok = mbar_wait(bar, parity, limit, abort, status, where);
  return __all_sync(kFull, ok);
}

// O += P V for cache tile number `tile_it` (CTA-local count): A = P (fp16) from the S/P
// buffer the tile used, B = this slice's 128 latent columns of the tile (MN-major).
template <class C>
__device__ __forceinline__ void issue_pv(uint32_t tiles_addr, uint32_t tmem, uint64_t* pv_done, uint64_t* empty,
                                         int tile_it, bool first, int pv_box) {
  constexpr int NT = C::NT_;
  constexpr uint32_t idesc_pv = idesc_f16_f32(128, 128, true);
  const int stage = tile_it % C::STAGES_;
  const uint32_t sb = tile_it & 1;
  const uint32_t v_base = tiles_addr + stage * C::STAGE_BYTES + pv_box * C::BOX_BYTES;
#pragma unroll
  for (int k = 0; k < NT / 16; ++k) {
    const uint64_t bdesc = smem_desc_sw128(v_base + k * 16 * 128, C::BOX_BYTES, 1024);
    umma_f16_ts(tmem + C::TMEM_O, tmem + C::TMEM_S + sb * NT + k * 8, bdesc, idesc_pv,
                (first && k == 0) ? 0u : 1u);
  }
  umma_commit(pv_done);
  umma_commit(&empty[stage]);
}

template <int NB, int NT, int STAGES>
__global__ void __launch_bounds__(448, 1)
decode_kernel(const __grid_constant__ CUtensorMap map_ckv, const __grid_constant__ CUtensorMap map_krope,
              const DecodeArgs a) {
  using C = DecodeCfg<NB, NT, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* misc = tiles + STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* conv = full + STAGES;
  uint64_t* empty = conv + STAGES;
  uint64_t* s_full = empty + STAGES;  // [2]
  uint64_t* p_ready = s_full + 2;     // [2]
  uint64_t* red_bar = p_ready + 2;    // [2] row-max exchange, alternating per tile
  uint64_t* lsum_bar = red_bar + 2;   // row-sum exchange, once per segment
  uint64_t* pv_done = lsum_bar + 1;
  uint64_t* q_ready = pv_done + 1;
  uint64_t* drain = q_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red_max = reinterpret_cast<float*>(misc + C::BAR_BYTES);  // [2 buf][2 half][128]
  float* red_l = red_max + 2 * 2 * 128;                              // [2 half][128]
  int* prefix = reinterpret_cast<int*>(misc + C::BAR_BYTES + C::RED_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int slice = blockIdx.x;
  const int branch = slice / C::SLICES_PER_BRANCH;
  const int pv_box = (slice % C::SLICES_PER_BRANCH) * 2;  // first of the 2 boxes holding V
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
      mbar_init(&conv[i], 128);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], 256);
      mbar_init(&red_bar[i], 256);
    }
    mbar_init(lsum_bar, 256);
    mbar_init(pv_done, 1);
    mbar_init(q_ready, 256);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 12 && lane == 0) {
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

  if (warp == 12) {
    // ------------------------------------------------------------------ TMA producer
    // The CTA's tiles are the global tiles t_begin .. t_end-1 in order.  Each lane finds
    // the cache row of one CHUNK_ROWS-row chunk of a batch of 32 / CHUNKS tiles (block-table and
    // length loads in parallel), one batch ahead of the tiles lane 0 is issuing, so that
    // no dependent global load sits between two tiles' copies.
    constexpr int TPB = 32 / C::CHUNKS;
    const int ntiles = t_end - t_begin;
    const uint64_t policy = l2_policy_evict_first();
    auto chunk_row = [&](int it0) {
      const int t = t_begin + it0 + lane / C::CHUNKS;
      if (t >= t_end) return static_cast<int>(a.cache_rows);
      const int s = seq_of_tile(prefix, B, t);
      return cache_chunk_row(a, s, (t - prefix[s]) * NT + C::CHUNK_ROWS * (lane % C::CHUNKS));
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
        for (int r = 0; r < C::CHUNKS; ++r) y[r] = __shfl_sync(kFull, rows, k * C::CHUNKS + r);
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          uint8_t* dst = tiles + stage * C::STAGE_BYTES;
#pragma unroll
          for (int r = 0; r < C::CHUNKS; ++r) {
#pragma unroll
            for (int d = 0; d < C::QK_BOXES; ++d) {
              void* box = dst + d * C::BOX_BYTES + r * C::CHUNK_ROWS * 128;
              if (d < C::QK_BOXES - 1)
                tma_load_2d(box, &map_ckv, &full[stage], branch * C::W + 64 * d, y[r], policy);
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
    // Tail: every stage handed out must come back before the CTA may exit, so that no
    // copy or MMA still targets this CTA's shared memory.
    for (int k = max(0, issued - STAGES); k < issued; ++k) {
      if (ok && !warp_wait(&empty[k % STAGES], (k / STAGES) & 1, limit, abort_flag, status, 2)) ok = false;
      if (!ok) {  // aborted: wait (bounded, ignoring the abort flag) for the copy itself
        volatile int never = 0;
        warp_wait(&full[k % STAGES], (k / STAGES) & 1, kDrainNs, &never, status, 3);
      }
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16_f32(128, NT, false);
      const uint32_t tiles_addr = smem_u32(tiles);
      int it = 0, seg = 0;
      bool ok = true;
      for (int s = s_first; ok && s < B && prefix[s] < t_end; ++s) {
        const int j0 = max(t_begin, prefix[s]), j1 = min(t_end, prefix[s + 1]);
        if (j0 >= j1) continue;
        if (!mbar_wait(q_ready, seg & 1, limit, abort_flag, status, 10)) { ok = false; break; }
        ++seg;
        tc_fence_after();
        for (int j = j0; j < j1; ++j, ++it) {
          const int stage = it % STAGES;
          if (!mbar_wait(&conv[stage], (it / STAGES) & 1, limit, abort_flag, status, 11)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sb = it & 1;
          const uint32_t k_base = tiles_addr + stage * C::STAGE_BYTES;
#pragma unroll
          for (int k = 0; k < C::QK_DIMS / 16; ++k) {
            const uint64_t bdesc = smem_desc_sw128(k_base + (k >> 2) * C::BOX_BYTES + (k & 3) * 32, 16, 1024);
            umma_f16_ts(tmem + C::TMEM_S + sb * NT, tmem + C::TMEM_Q + k * 8, bdesc, idesc_qk, k > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[sb]);
          if (j > j0) {
            if (!mbar_wait(&p_ready[(it - 1) & 1], ((it - 1) >> 1) & 1, limit, abort_flag, status, 12)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv<C>(tiles_addr, tmem, pv_done, empty, it - 1, j - 1 == j0, pv_box);
          }
        }
        if (!ok) break;
        if (!mbar_wait(&p_ready[(it - 1) & 1], ((it - 1) >> 1) & 1, limit, abort_flag, status, 13)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv<C>(tiles_addr, tmem, pv_done, empty, it - 1, j1 - 1 == j0, pv_box);
      }
      // drain: every MMA issued so far completes before TMEM is released (bounded by
      // kDrainNs, whatever the abort flag says)
      umma_commit(drain);
      volatile int never = 0;
      mbar_wait(drain, 0, kDrainNs, &never, status, 14);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------------ bf16 -> fp16
    const int ct = threadIdx.x - 256;
    constexpr int N16 = C::STAGE_BYTES / 16;
    static_assert(N16 % 128 == 0, "conversion split");
    int it = 0;
    bool ok = true;
    for (int s = s_first; ok && s < B && prefix[s] < t_end; ++s) {
      const int j0 = max(t_begin, prefix[s]), j1 = min(t_end, prefix[s + 1]);
      if (j0 >= j1) continue;
      const int L = a.seq_lens[s];
      for (int j = j0; j < j1; ++j, ++it) {
        const int stage = it % STAGES;
        if (!warp_wait(&full[stage], (it / STAGES) & 1, limit, abort_flag, status, 20)) { ok = false; break; }
        const int n_valid = min(NT, L - (j - prefix[s]) * NT);
        uint4* buf = reinterpret_cast<uint4*>(tiles + stage * C::STAGE_BYTES);
        if (n_valid == NT) {
#pragma unroll 2
          for (int c0 = ct; c0 < N16; c0 += 128 * 4) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (c0 + u * 128 < N16) v[u] = buf[c0 + u * 128];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (c0 + u * 128 < N16) {
                v[u].x = bf16x2_to_f16x2(v[u].x);
                v[u].y = bf16x2_to_f16x2(v[u].y);
                v[u].z = bf16x2_to_f16x2(v[u].z);
                v[u].w = bf16x2_to_f16x2(v[u].w);
                buf[c0 + u * 128] = v[u];
              }
            }
          }
        } else {
#pragma unroll 1
          for (int c = ct; c < N16; c += 128) {
            const int row = (c >> 3) % NT;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (row < n_valid) {
              v = buf[c];
              v.x = bf16x2_to_f16x2(v.x);
              v.y = bf16x2_to_f16x2(v.y);
              v.z = bf16x2_to_f16x2(v.z);
              v.w = bf16x2_to_f16x2(v.w);
            }
            buf[c] = v;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&conv[stage]);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    // The absorbed query comes from the previous kernel, and the split partials written
    // here are read by the previous call's merge: wait for those grids.
    grid_dep_wait();
    constexpr int HALF = C::HALF;
    const int half = warp >> 2;                        // which half of the score columns
    const int row = threadIdx.x & 127;                 // head row == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t t_row = tmem + lane_addr;
    const float sl2 = a.scale_log2;
    int it = 0, seg = 0;
    bool ok = true;
    for (int s = s_first; ok && s < B && prefix[s] < t_end; ++s) {
      const int j0 = max(t_begin, prefix[s]), j1 = min(t_end, prefix[s + 1]);
      if (j0 >= j1) continue;
      const int L = a.seq_lens[s];
      // Q~ row of this head for branch `branch`: W latent columns then the 64 rope columns;
      // the two halves store alternate 64-column chunks.
      {
        const uint4* qsrc = reinterpret_cast<const uint4*>(
            a.q_tilde + (static_cast<long long>(s) * a.heads + min(row, a.heads - 1)) * (a.d_c + 64));
        const bool live = row < a.heads;
        uint32_t w[32];
#pragma unroll 1
        for (int c = half; c < C::QK_DIMS / 64; c += 2) {
          const int col0 = (c < C::QK_DIMS / 64 - 1) ? branch * C::W + 64 * c : a.d_c;  // fp16 column
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint4 v = live ? __ldg(qsrc + (col0 >> 3) + u) : make_uint4(0u, 0u, 0u, 0u);
            w[4 * u + 0] = v.x; w[4 * u + 1] = v.y; w[4 * u + 2] = v.z; w[4 * u + 3] = v.w;
          }
          tmem_st32(t_row + C::TMEM_Q + 32 * c, w);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(q_ready);
      }
      float m_ref = -INFINITY, l = 0.f;
      for (int j = j0; j < j1; ++j, ++it) {
        const uint32_t sb = it & 1;
        if (!warp_wait(&s_full[sb], (it >> 1) & 1, limit, abort_flag, status, 30)) { ok = false; break; }
        tc_fence_after();
        const int n_valid = min(NT, L - (j - prefix[s]) * NT);
        const int col0 = half * HALF;
        const int n_mine = min(max(n_valid - col0, 0), HALF);  // valid columns in this half
        uint32_t sr[HALF];
        tmem_load<HALF>(t_row + C::TMEM_S + sb * NT + col0, sr);
        tmem_ld_wait();
        // tile max of the raw scores (4 independent chains), masked past the sequence end
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
        // both halves of the row agree on the tile max
        const int rb = it & 1;
        red_max[(rb * 2 + half) * 128 + row] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        mbar_arrive(&red_bar[rb]);
        if (!warp_wait(&red_bar[rb], (it >> 1) & 1, limit, abort_flag, status, 33)) { ok = false; break; }
        const float mt_raw = fmaxf(red_max[(rb * 2) * 128 + row], red_max[(rb * 2 + 1) * 128 + row]);
        const float mt = mt_raw * sl2;  // scale > 0 commutes with max
        const bool first = (j == j0);
        float factor = 1.f;
        bool rescale = false;
        if (first) {
          m_ref = mt;
        } else if (mt > m_ref + 8.f) {  // lazy rescale: keep the old reference unless it grew by 2^8
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
          sr[k] = pack_f16x2(p0, p1);  // overwrites score registers already consumed
        }
        tmem_store<HALF / 2>(t_row + C::TMEM_S + sb * NT + col0 / 2, sr);
        const float tsum = (sum[0] + sum[1]) + (sum[2] + sum[3]);
        l = first ? tsum : fmaf(l, factor, tsum);
        if (!first) {
          // O may only be touched once the previous tile's P*V has landed.
          if (!warp_wait(pv_done, (it - 1) & 1, limit, abort_flag, status, 31)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(kFull, rescale)) {
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
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_ready[sb]);
      }
      if (!ok) break;
      // epilogue: the segment's last P*V must land before O is read
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
      mbar_arrive(lsum_bar);
      if (!warp_wait(lsum_bar, seg & 1, limit, abort_flag, status, 34)) { ok = false; break; }
      ++seg;
      if (half == 0 && row < a.heads)
        a.ml_part[(slot * gridDim.x + slice) * 128 + row] = make_float2(m_ref, l + red_l[128 + row]);
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int NB, int NT, int STAGES>
cudaError_t launch_decode(const CUtensorMap& map_ckv, const CUtensorMap& map_krope, const DecodeArgs& a,
                          int groups, cudaStream_t stream, bool pdl) {
  using C = DecodeCfg<NB, NT, STAGES>;
  auto kern = decode_kernel<NB, NT, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, dim3(a.d_c / 128, groups), dim3(C::THREADS), C::SMEM_BYTES, stream, pdl, map_ckv,
                       map_krope, a);
}

}  // namespace

int decode_tile_tokens(int branch_width) {
  return branch_width == 128 ? decode_split_tile_tokens() : (branch_width == 256 ? 80 : 48);
}

int decode_box_rows(int branch_width) {
  return branch_width == 512 ? DecodeCfg<1, 48, 4>::CHUNK_ROWS
                             : (branch_width == 256 ? DecodeCfg<2, 80, 4>::CHUNK_ROWS : 32);
}

cudaError_t launch_decode_kernel(int n_branch, const CUtensorMap& map_ckv, const CUtensorMap& map_krope,
                                 const DecodeArgs& a, int groups, cudaStream_t stream, bool pdl) {
  if (n_branch < 1 || a.d_c % n_branch != 0 || a.d_c % 128 != 0 || a.d_c > 512) return cudaErrorInvalidValue;
  switch (a.d_c / n_branch) {  // branch width
    case 128: return launch_decode_split_kernel(map_ckv, map_krope, a, groups, stream, pdl);
    case 256: return launch_decode<2, 80, 4>(map_ckv, map_krope, a, groups, stream, pdl);
    case 512: return launch_decode<1, 48, 4>(map_ckv, map_krope, a, groups, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hra

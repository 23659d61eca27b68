// prefill_sm100.cu -- causal multi-token (prefill) MLRA in the expanded form, on tcgen05/TMEM.
//
// "vllbc02MLA" contrasts the two phases of MLA: prefill is compute-bound and works with the
// per-head keys and values (the expanded form), generation is memory-bound and uses the
// absorbed form.  Prefill of MLRA ("Multi-Head Low-Rank Attention", 核心方法: O = sum_b
// Softmax(Q K_b^T) V_b) for one sequence of L cached tokens whose last n are the queries
// (position p_j = L - n + j, query j sees the tokens t <= p_j):
//
//   prep     q16[j, i] = [alpha_q q_nope | RoPE(q_rope, p_j)] in fp16; K_R in fp16 (zero
//            rows past L);
//   expand   K^(b)[i, t] = alpha_kv C_t^(b) W_UK^(b),(i) and V^(b)[i, t] = alpha_kv C_t^(b)
//            W_UV^(b),(i), fp16 [n_branch, h, L_pad, 128] (rows past L zero): one tcgen05
//            GEMM per (128 tokens, head, branch), M = tokens, N = 128 + 128 (K and V side by
//            side in TMEM), K = the branch's w latent columns;
//   attend   per (128 queries, head): for each branch, an online softmax over the branch's
//            key tiles up to the tile holding the last query's position, S = q16 . [K | K_R]^T
//            (M = 128 queries, N = 128 keys, K = 192) and O_b += P V_b (N = 128, K = 128
//            keys); each branch's O_b / l_b is added into an fp32 sum in TMEM, and out =
//            branch_scale * the sum.
//
// The attention kernel follows the decode kernel's pipeline (decode_split_sm100.cu): a TMA
// producer, a QK issuer, a P.V issuer and 8 softmax warps in two halves of 64 key columns,
// two S/P buffers with P written over the scores it came from, lazy rescaling of the
// reference max.  Every wait is bounded; exit paths wait for in-flight copies and MMAs with
// a fixed bound (sm100.cuh) before TMEM is released.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "launch.h"
#include "prefill_sm100.h"
#include "sm100.cuh"

namespace hra {

namespace {

constexpr uint32_t kAll = 0xffffffffu;

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit, volatile int* abort,
                                          int* status, int where) {
  const bool ok = mbar_wait(bar, parity, limit, abort, status, where);
  return __all_sync(kAll, ok);
}

// ------------------------------------------------------------------------------- prep
// grid-stride over the query rows (n * h) and the rope rows (L_pad).
__global__ void prefill_prep_kernel(const PrefillArgs a) {
  __shared__ double turns[32];  // rotation pair d turns by theta^(-2d/64) / (2 pi) per position
  if (threadIdx.x < 32) turns[threadIdx.x] = pow(static_cast<double>(a.rope_theta), -2.0 * threadIdx.x / 64.0) *
                                             0.15915494309189535;
  if (threadIdx.x == 0) grid_dep_launch();
  __syncthreads();
  grid_dep_wait();  // q16 / kr16 are read by the previous call's attention
  const int nq = a.n_query * a.heads;
  const long long total = static_cast<long long>(nq) + a.l_pad;
  for (long long r = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; r < total;
       r += static_cast<long long>(gridDim.x) * blockDim.x) {
    if (r < nq) {
      const int j = static_cast<int>(r / a.heads);
      const __nv_bfloat16* q = a.q + r * 192;
      __half* dst = a.q16 + r * 192;
      for (int d = 0; d < 128; ++d) dst[d] = __float2half_rn(a.alpha_q * __bfloat162float(q[d]));
      // RoPE at p_j: pair (d, d + 32) turns by p * theta^(-2d/64); the angle in turns, fp64
      const double pos = static_cast<double>(a.seq_len - a.n_query + j);
      for (int d = 0; d < 32; ++d) {
        const double x = pos * turns[d];
        const float f = static_cast<float>(x - rint(x));
        float sn, cs;
        sincospif(2.f * f, &sn, &cs);
        const float x1 = __bfloat162float(q[128 + d]), x2 = __bfloat162float(q[160 + d]);
        dst[128 + d] = __float2half_rn(fmaf(x1, cs, -x2 * sn));
        dst[160 + d] = __float2half_rn(fmaf(x1, sn, x2 * cs));
      }
    } else {
      const long long t = r - nq;
      __half* dst = a.kr16 + t * 64;
      const __nv_bfloat16* src = a.krope + t * a.krope_stride;
      for (int d = 0; d < 64; ++d) dst[d] = t < a.seq_len ? __float2half_rn(__bfloat162float(src[d])) : __half(0.f);
    }
  }
}

// ------------------------------------------------------------------------------- expand
struct ExpandCfg {
  static constexpr int A_BYTES = 2 * 128 * 128;   // 128 tokens x 128 latent columns (2 boxes of 64)
  static constexpr int B_BYTES = 2 * 128 * 128;   // 128 latent rows x 128 output columns (2 boxes of 64)
  static constexpr int STAGE_BYTES = A_BYTES + 2 * B_BYTES;  // A, W_UK chunk, W_UV chunk
  static constexpr int STAGES = 2;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 128;
  static constexpr int TMEM_COLS = 256;           // D_K [0,128), D_V [128,256)
  static constexpr int THREADS = 256;
};

// grid (L_pad / 128, h, n_branch), 256 threads.  Warp 0 lane 0 streams the w / 128 K chunks
// through two stages and issues the MMAs; then warps 0-3 store K rows and warps 4-7 V rows
// (a thread owns one token row = TMEM lane).
__global__ void __launch_bounds__(ExpandCfg::THREADS, 1)
prefill_expand_kernel(const __grid_constant__ CUtensorMap map_ckv, const __grid_constant__ CUtensorMap map_wuk,
                      const __grid_constant__ CUtensorMap map_wuv, const PrefillArgs a) {
  using C = ExpandCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + C::STAGES * C::STAGE_BYTES);  // [2]
  uint64_t* empty = full + 2;                                                       // [2]
  uint64_t* done_bar = empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* never_flag = abort_flag + 1;
  const int t0 = blockIdx.x * 128, i = blockIdx.y, b = blockIdx.z;
  const int w = 512 / a.n_branch;      // branch width
  const int nchunks = w / 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    grid_dep_launch();
    for (int k = 0; k < 2; ++k) {
      mbar_init(&full[k], 1);
      mbar_init(&empty[k], 1);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    *never_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t keep = l2_policy_evict_last();
      auto load = [&](int c) {
        uint8_t* st = stages + (c % C::STAGES) * C::STAGE_BYTES;
        uint64_t* bar = &full[c % C::STAGES];
        mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
        const int col = b * w + 128 * c;  // latent column of the chunk
        for (int kb = 0; kb < 2; ++kb) tma_load_2d(st + kb * 16384, &map_ckv, bar, col + 64 * kb, t0, keep);
        for (int db = 0; db < 2; ++db) {
          tma_load_2d(st + C::A_BYTES + db * 16384, &map_wuk, bar, 64 * db, i * 512 + col, keep);
          tma_load_2d(st + C::A_BYTES + C::B_BYTES + db * 16384, &map_wuv, bar, 64 * db, i * 512 + col, keep);
        }
      };
      int issued = 0;
      for (int c = 0; c < nchunks && c < C::STAGES; ++c) load(c), ++issued;
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, true);  // B (W rows = latent) MN-major
      const uint32_t base = smem_u32(stages);
      bool ok = true;
      for (int c = 0; c < nchunks && ok; ++c) {
        const int st = c % C::STAGES;
        if (!mbar_wait(&full[st], (c / C::STAGES) & 1, a.wait_limit_ns, abort_flag, a.status, 60)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = base + st * C::STAGE_BYTES;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t adesc = smem_desc_sw128(sa + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
#pragma unroll
          for (int m = 0; m < 2; ++m) {  // K, then V
            const uint64_t bdesc = smem_desc_sw128(sa + C::A_BYTES + m * C::B_BYTES + ks * 2048, 16384, 1024);
            umma_f16_ss(tmem + 128 * m, adesc, bdesc, idesc, (c > 0 || ks > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[st]);
        if (c + C::STAGES < nchunks) {  // refill this stage once its MMAs have read it
          if (!mbar_wait(&empty[st], (c / C::STAGES) & 1, a.wait_limit_ns, abort_flag, a.status, 61)) {
            ok = false;
            break;
          }
          load(c + C::STAGES);
          ++issued;
        }
      }
      umma_commit(done_bar);
      // every copy issued has landed before the CTA may exit (bounded, whatever the abort flag)
      for (int c = max(0, issued - C::STAGES); c < issued; ++c)
        mbar_wait(&full[c % C::STAGES], (c / C::STAGES) & 1, kDrainNs, never_flag, a.status, 62);
    }
    __syncwarp();
  }
  grid_dep_wait();  // K / V are read by the previous call's attention
  const bool done = mbar_wait(done_bar, 0, kDrainNs, never_flag, a.status, 63);
  tc_fence_after();
  if (done && !*abort_flag) {
    const int m = warp >> 2;  // 0: K rows, 1: V rows
    const int r = 32 * (warp & 3) + lane;
    const int t = t0 + r;
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    __half* dst = (m == 0 ? a.k_exp : a.v_exp) + ((static_cast<long long>(b) * a.heads + i) * a.l_pad + t) * 128;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_base + 128 * m + 32 * c, v);
      tmem_ld_wait();
      if (t < a.l_pad) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          __align__(16) __half h8[8];
#pragma unroll
          for (int u = 0; u < 8; ++u)
            h8[u] = t < a.seq_len ? __float2half_rn(a.alpha_kv * __uint_as_float(v[8 * q + u])) : __half(0.f);
          *reinterpret_cast<uint4*>(dst + 32 * c + 8 * q) = *reinterpret_cast<const uint4*>(h8);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------- attend
struct AttendCfg {
  static constexpr int NT = 128;                   // keys per tile, queries per CTA
  static constexpr int STAGES = 2;
  static constexpr int BOX = 128 * 128;            // one 64-column box of 128 rows
  static constexpr int K_BYTES = 3 * BOX;          // K^(b) (2 boxes) | K_R (1 box)
  static constexpr int V_BYTES = 2 * BOX;
  static constexpr int STAGE_BYTES = K_BYTES + V_BYTES;
  static constexpr int Q_BYTES = 3 * BOX;          // q16: nope (2 boxes) | rope (1 box)
  static constexpr int TMEM_O = 0, TMEM_S = 128, TMEM_SUM = 384, TMEM_COLS = 512;
  static constexpr int WARP_PRODUCER = 8, WARP_QK = 9, WARP_PV = 10;
  static constexpr int THREADS = 32 * 11;
  static constexpr int BAR_BYTES = 256;
  static constexpr int RED_BYTES = (2 * 2 * 128 + 2 * 128) * 4;
  static constexpr int SMEM = 1024 + Q_BYTES + STAGES * STAGE_BYTES + BAR_BYTES + RED_BYTES;
  static_assert(SMEM <= 232448, "shared memory budget");
};

__global__ void __launch_bounds__(AttendCfg::THREADS, 1)
prefill_attend_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_kr,
                      const PrefillArgs a) {
  using C = AttendCfg;
  constexpr int NT = C::NT, STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* qbuf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = qbuf + C::Q_BYTES;
  uint8_t* misc = tiles + STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty = full + STAGES;
  uint64_t* s_full = empty + STAGES;   // [2]
  uint64_t* p_ready = s_full + 2;      // [2]
  uint64_t* pv_done = p_ready + 2;     // [2]
  uint64_t* q_full = pv_done + 2;
  uint64_t* red_bar = q_full + 1;      // [2]
  uint64_t* lsum_bar = red_bar + 2;
  uint64_t* drain = lsum_bar + 1;      // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* never_flag = abort_flag + 1;
  float* red_max = reinterpret_cast<float*>(misc + C::BAR_BYTES);  // [2 buf][2 half][128]
  float* red_l = red_max + 2 * 2 * 128;                              // [2 half][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = blockIdx.x * NT, i = blockIdx.y;
  const int nb = a.n_branch;
  const uint64_t limit = a.wait_limit_ns;
  int* status = a.status;
  // key tiles of one branch: up to the tile holding the last position this CTA's queries see
  const int p_last = min(a.seq_len - a.n_query + j0 + NT - 1, a.seq_len - 1);
  const int T = p_last / NT + 1;
  const int U = nb * T;  // tiles in all: u = b * T + t

  if (threadIdx.x == 32) {
    for (int k = 0; k < STAGES; ++k) {
      mbar_init(&full[k], 1);
      mbar_init(&empty[k], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&s_full[k], 1);
      mbar_init(&p_ready[k], 8);
      mbar_init(&pv_done[k], 1);
      mbar_init(&red_bar[k], 8);
      mbar_init(&drain[k], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(lsum_bar, 8);
    *abort_flag = 0;
    *never_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 0) grid_dep_launch();
  if (warp == C::WARP_QK) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::WARP_PRODUCER) {
    if (lane == 0) {
      // every input here (q16, K, V, K_R) is written by the previous kernels of this call
      grid_dep_wait();
      const uint64_t keep = l2_policy_evict_last();
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
      for (int c = 0; c < 3; ++c) tma_load_2d(qbuf + c * C::BOX, &map_q, q_full, i * 192 + 64 * c, j0, keep);
      bool ok = true;
      int issued = 0;
      for (int u = 0; u < U && ok; ++u) {
        const int st = u % STAGES, b = u / T, t = u % T;
        if (u >= STAGES && !mbar_wait(&empty[st], ((u / STAGES) + 1) & 1, limit, abort_flag, status, 70)) {
          ok = false;
          break;
        }
        uint8_t* dst = tiles + st * C::STAGE_BYTES;
        mbar_arrive_expect_tx(&full[st], C::STAGE_BYTES);
        const int krow = (b * a.heads + i) * a.l_pad + t * NT;
        for (int c = 0; c < 2; ++c) tma_load_2d(dst + c * C::BOX, &map_k, &full[st], 64 * c, krow, keep);
        tma_load_2d(dst + 2 * C::BOX, &map_kr, &full[st], 0, t * NT, keep);
        for (int c = 0; c < 2; ++c) tma_load_2d(dst + C::K_BYTES + c * C::BOX, &map_v, &full[st], 64 * c, krow, keep);
        issued = u + 1;
      }
      for (int u = max(0, issued - STAGES); u < issued; ++u) {  // every stage must come back
        if (ok && !mbar_wait(&empty[u % STAGES], (u / STAGES) & 1, limit, abort_flag, status, 71)) ok = false;
        if (!ok) mbar_wait(&full[u % STAGES], (u / STAGES) & 1, kDrainNs, never_flag, status, 72);
      }
      mbar_wait(q_full, 0, kDrainNs, never_flag, status, 73);
    }
    __syncwarp();
  } else if (warp == C::WARP_QK) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, NT, false);
      const uint32_t tiles_addr = smem_u32(tiles), q_addr = smem_u32(qbuf);
      for (int u = 0; u < U; ++u) {
        const int bsp = u & 1;
        if (!mbar_wait(&full[u % STAGES], (u / STAGES) & 1, limit, abort_flag, status, 74) ||
            (u == 0 && !mbar_wait(q_full, 0, limit, abort_flag, status, 75)) ||
            (u >= 2 && !mbar_wait(&pv_done[bsp], ((u - 2) >> 1) & 1, limit, abort_flag, status, 76)))
          break;
        tc_fence_after();
        const uint32_t k_base = tiles_addr + (u % STAGES) * C::STAGE_BYTES;
#pragma unroll
        for (int k = 0; k < 12; ++k) {  // nope (boxes 0, 1), rope (box 2); 4 K steps per box
          const uint32_t off = (k >> 2) * C::BOX + (k & 3) * 32;
          umma_f16_ss(tmem + C::TMEM_S + bsp * NT, smem_desc_sw128(q_addr + off, 16, 1024),
                      smem_desc_sw128(k_base + off, 16, 1024), idesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[bsp]);
      }
      umma_commit(&drain[0]);
      mbar_wait(&drain[0], 0, kDrainNs, never_flag, status, 77);
    }
    __syncwarp();
  } else if (warp == C::WARP_PV) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, 128, true);
      const uint32_t tiles_addr = smem_u32(tiles);
      for (int u = 0; u < U; ++u) {
        const int bsp = u & 1, st = u % STAGES;
        if (!mbar_wait(&p_ready[bsp], (u >> 1) & 1, limit, abort_flag, status, 78)) break;
        tc_fence_after();
        const uint32_t v_base = tiles_addr + st * C::STAGE_BYTES + C::K_BYTES;
        const uint32_t p_base = tmem + C::TMEM_S + bsp * NT;
        const bool first = (u % T) == 0;  // a branch's first tile starts its O
#pragma unroll
        for (int k = 0; k < NT / 16; ++k) {
          const uint32_t a_tmem = p_base + 64 * (k >> 2) + 8 * (k & 3);
          const uint64_t bdesc = smem_desc_sw128(v_base + k * 16 * 128, C::BOX, 1024);
          umma_f16_ts(tmem + C::TMEM_O, a_tmem, bdesc, idesc, (first && k == 0) ? 0u : 1u);
        }
        umma_commit(&pv_done[bsp]);
        umma_commit(&empty[st]);
      }
      umma_commit(&drain[1]);
      mbar_wait(&drain[1], 0, kDrainNs, never_flag, status, 79);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax + epilogues
    const int half = warp >> 2;
    const int row = threadIdx.x & 127;  // query j0 + row == TMEM lane
    const uint32_t t_row = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float sl2 = a.scale_log2;
    const int p_row = a.seq_len - a.n_query + j0 + row;  // this query's position (padding rows: past L)
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int u = 0; u < U && ok; ++u) {
      const int bsp = u & 1, b = u / T, t = u % T;
      const bool first = t == 0;
      if (!warp_wait(&s_full[bsp], (u >> 1) & 1, limit, abort_flag, status, 80)) { ok = false; break; }
      tc_fence_after();
      // causal: key t * NT + c is visible to this row iff t * NT + c <= p_row
      const int n_vis = min(max(p_row - t * NT + 1, 0), NT);
      const int n_mine = min(max(n_vis - half * 64, 0), 64);
      const uint32_t s_cols = t_row + C::TMEM_S + bsp * NT + half * 64;
      uint32_t sr[64];
      tmem_load<64>(s_cols, sr);
      tmem_ld_wait();
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int k = 0; k < 64; ++k) {
        if (k >= n_mine) sr[k] = __float_as_uint(-INFINITY);
        mx[k & 3] = fmaxf(mx[k & 3], __uint_as_float(sr[k]));
      }
      const int rb = u & 1;
      red_max[(rb * 2 + half) * 128 + row] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      warp_arrive(&red_bar[rb]);
      if (!warp_wait(&red_bar[rb], (u >> 1) & 1, limit, abort_flag, status, 81)) { ok = false; break; }
      const float mt = fmaxf(red_max[(rb * 2) * 128 + row], red_max[(rb * 2 + 1) * 128 + row]) * sl2;
      float factor = 1.f;
      bool rescale = false;
      if (first) {
        m_ref = mt;  // the first tile holds key 0, which every query sees
      } else if (mt > m_ref + 8.f) {
        factor = ex2_approx(m_ref - mt);
        m_ref = mt;
        rescale = true;
      }
      const float neg_m = -m_ref;
      float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(sr[2 * k]), sl2, neg_m));
        const float p1 = ex2_approx(fmaf(__uint_as_float(sr[2 * k + 1]), sl2, neg_m));
        sum[k & 3] += p0 + p1;
        sr[k] = pack_f16x2(p0, p1);
      }
      const float tsum = (sum[0] + sum[1]) + (sum[2] + sum[3]);
      l = first ? tsum : fmaf(l, factor, tsum);
      if (__any_sync(kAll, rescale)) {
        if (!warp_wait(&pv_done[bsp ^ 1], ((u - 1) >> 1) & 1, limit, abort_flag, status, 82)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
          uint32_t o[16];
          const uint32_t oaddr = t_row + C::TMEM_O + 64 * half + 16 * k;
          tmem_ld16(oaddr, o);
          tmem_ld_wait();
#pragma unroll
          for (int v = 0; v < 16; ++v) o[v] = __float_as_uint(__uint_as_float(o[v]) * factor);
          tmem_st16(oaddr, o);
        }
      }
      tmem_st32(s_cols, sr);
      tmem_st_wait();
      tc_fence_before();
      warp_arrive(&p_ready[bsp]);
      if (t == T - 1) {
        // end of branch b: O_b / l_b added into the branch sum
        if (!warp_wait(&pv_done[bsp], (u >> 1) & 1, limit, abort_flag, status, 83)) { ok = false; break; }
        tc_fence_after();
        red_l[half * 128 + row] = l;
        warp_arrive(lsum_bar);
        if (!warp_wait(lsum_bar, b & 1, limit, abort_flag, status, 84)) { ok = false; break; }
        const float lt = red_l[row] + red_l[128 + row];
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll 1
        for (int k = 0; k < 2; ++k) {
          uint32_t o[32], acc[32];
          tmem_ld32(t_row + C::TMEM_O + 64 * half + 32 * k, o);
          if (b > 0) tmem_ld32(t_row + C::TMEM_SUM + 64 * half + 32 * k, acc);
          tmem_ld_wait();
#pragma unroll
          for (int v = 0; v < 32; ++v)
            acc[v] = __float_as_uint((b > 0 ? __uint_as_float(acc[v]) : 0.f) + __uint_as_float(o[v]) * inv);
          tmem_st32(t_row + C::TMEM_SUM + 64 * half + 32 * k, acc);
        }
        tmem_st_wait();
        // the next branch's first P.V overwrites O: every thread has read it before the
        // exchange of the next branch's first row maxima
        tc_fence_before();
      }
    }
    if (ok) {
      const int j = j0 + row;
#pragma unroll 1
      for (int k = 0; k < 2; ++k) {
        uint32_t acc[32];
        tmem_ld32(t_row + C::TMEM_SUM + 64 * half + 32 * k, acc);
        tmem_ld_wait();
        if (j < a.n_query) {
          const long long o = (static_cast<long long>(j) * a.heads + i) * 128 + 64 * half + 32 * k;
          if (a.out_f32) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<float4*>(a.out_f32 + o + 4 * q) =
                  make_float4(a.branch_scale * __uint_as_float(acc[4 * q]), a.branch_scale * __uint_as_float(acc[4 * q + 1]),
                              a.branch_scale * __uint_as_float(acc[4 * q + 2]), a.branch_scale * __uint_as_float(acc[4 * q + 3]));
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              __align__(16) __nv_bfloat16 b8[8];
#pragma unroll
              for (int v = 0; v < 8; ++v) b8[v] = __float2bfloat16_rn(a.branch_scale * __uint_as_float(acc[8 * q + v]));
              *reinterpret_cast<uint4*>(a.out_bf16 + o + 8 * q) = *reinterpret_cast<const uint4*>(b8);
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_QK) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <class K>
cudaError_t set_smem(K kern, int bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

cudaError_t launch_prefill(const PrefillMaps& m, const PrefillArgs& a, cudaStream_t stream) {
  cudaError_t e = launch_kernel(prefill_prep_kernel, dim3(148 * 4), dim3(128), 0, stream, true, a);
  if (e != cudaSuccess) return e;
  if ((e = set_smem(prefill_expand_kernel, ExpandCfg::SMEM)) != cudaSuccess) return e;
  e = launch_kernel(prefill_expand_kernel, dim3(a.l_pad / 128, a.heads, a.n_branch), dim3(ExpandCfg::THREADS),
                    ExpandCfg::SMEM, stream, true, m.ckv, m.wuk, m.wuv, a);
  if (e != cudaSuccess) return e;
  if ((e = set_smem(prefill_attend_kernel, AttendCfg::SMEM)) != cudaSuccess) return e;
  return launch_kernel(prefill_attend_kernel, dim3((a.n_query + 127) / 128, a.heads), dim3(AttendCfg::THREADS),
                       AttendCfg::SMEM, stream, true, m.q16, m.k, m.v, m.kr16, a);
}

}  // namespace hra

// absorb_combine.cu -- the steps around the split-KV decode, on the tensor cores.
//
// absorb ("Multi-Head Low-Rank Attention", 方法步骤详情, step 1 -- query-side weight
// absorption), one CTA per (head i, chunk of 128 sequences, 256 columns of the latent):
//     q~[s,i,0:d_c] = alpha_q * alpha_kv * q_nope[s,i] . W_UK[i]^T        (W_UK[i]: d_c x 128)
// with d_c = 512, or 256 / 128 when the call holds a shard of 128-wide branches (tensor
// parallelism by branch, 核心方法: under 4-way TP each device holds one MLRA-4 branch).
// One tcgen05 pass with M = the chunk's sequences, N = min(d_c, 256) latent (the CTA's part),
// K = 128: A = the q_nope rows, B = W_UK[i] (its rows are latent indices, each with 128
// contiguous nope dims: K-major), D in 256 TMEM columns.  bf16 x bf16
// products are exact in the fp32 accumulator, so this equals the fp32 definition up to
// summation order.  A thread of the epilogue owns one sequence and 32 consecutive latent
// columns at a time, so q~ (fp16) is written with 16-byte stores.  The same threads rotate q_rope to position L-1.  The
// branch structure needs no special case: branch b's absorbed query is columns
// [b*w, (b+1)*w) of the same d_c-vector (W_UK^(b),(i) is the matching row block).
//
// merge (step 2b): the split-KV partial states of a (sequence, 128-wide latent slice,
// head) are combined by log-sum-exp, o = sum_g 2^(m_g - M) O_g / sum_g 2^(m_g - M) l_g,
// and o_lat is stored as bf16 hi + lo terms.
//
// upproj (step 3), one CTA per (head i, chunk of 128 sequences):
//     out[s,i,:] = branch_scale * alpha_kv * o_lat[s,i,:] . W_UV[i]        (W_UV[i]: d_c x 128)
// M = sequences, N = 128 output columns, K = d_c latent (both o_lat terms): A = o_lat
// rows (K-major), B = W_UV[i] read MN-major (its rows are latent indices with the 128
// output columns contiguous), streamed through two shared-memory stages in d_c / 128 K
// chunks.  The branches partition the latent, so summing the per-branch up-projections
// is this one contraction (and a branch shard's output is its part of that sum).
#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "absorb_combine.h"
#include "launch.h"
#include "schedule.cuh"
#include "sm100.cuh"

namespace hra {

namespace {

constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s bound on each wait

// ---------------------------------------------------------------------------- absorb
struct AbsorbCfg {
  static constexpr int Q_BYTES = 2 * 128 * 128;  // 2 K boxes of [128 sequences x 128 B]
  static constexpr int W_BYTES = 2 * 256 * 128;  // this CTA's latent half: 2 K boxes of [256 rows x 128 B]
  static constexpr int SMEM = 1024 + Q_BYTES + W_BYTES + 32 * 8 + 64;
  static constexpr int TMEM_COLS = 256;
  static constexpr int THREADS = 256;
};

// 32 consecutive fp32 values -> fp16 q~ at dst.
__device__ __forceinline__ void store_q32(const AbsorbArgs& a, long long dst, const float* x) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    __align__(16) __half h8[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) h8[u] = __float2half_rn(x[8 * v + u]);
    *reinterpret_cast<uint4*>(a.q_tilde + dst + 8 * v) = *reinterpret_cast<const uint4*>(h8);
  }
}

// grid (h, ceil(B / 128), max(d_c / 256, 1) latent parts), 256 threads, two CTAs per SM.
// Warp w owns the sequences of TMEM lane quadrant w % 4 and 128 of the CTA's
// min(d_c, 256) latent columns (w / 4; with 128 columns warps 4-7 only rotate q_rope).
__global__ void __launch_bounds__(AbsorbCfg::THREADS, 1)
absorb_tc_kernel(const __grid_constant__ CUtensorMap map_wuk, const __grid_constant__ CUtensorMap map_q,
                 const AbsorbArgs a) {
  using C = AbsorbCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* qbuf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wbuf = qbuf + C::Q_BYTES;
  double* turns = reinterpret_cast<double*>(wbuf + C::W_BYTES);  // [32] rope turns per position
  uint64_t* bars = reinterpret_cast<uint64_t*>(turns + 32);      // [0] loads landed, [1] MMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int i = blockIdx.x;
  const int s0 = blockIdx.y * 128;
  const int nh = blockIdx.z;  // latent part [256 nh, +nw)
  const int dc = a.d_c;
  const int nw = dc < 256 ? dc : 256;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    grid_dep_launch();
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 2) {  // rotation pair j turns by theta^(-2j/64) / (2 pi) per position, in fp64
    turns[lane] = pow(static_cast<double>(a.rope_theta), -2.0 * lane / 64.0) * 0.15915494309189535;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // warp 0 issues the loads and the MMAs from lane 0; its other lanes wait at the
    // __syncwarp so that no lane of this warp polls a barrier lane 0 has yet to release
    if (lane == 0) {
      const uint64_t stream_once = l2_policy_evict_first(), keep = l2_policy_evict_last();
      mbar_arrive_expect_tx(&bars[0], C::Q_BYTES + 2 * nw * 128);
      for (int kb = 0; kb < 2; ++kb)
        tma_load_2d(qbuf + kb * 16384, &map_q, &bars[0], i * 192 + 64 * kb, s0, stream_once);
      for (int kb = 0; kb < 2; ++kb)  // box {64, nw}
        tma_load_2d(wbuf + kb * 32768, &map_wuk, &bars[0], 64 * kb, i * dc + 256 * nh, keep);
      if (mbar_wait(&bars[0], 0, kWaitNs, abort_flag, a.status, 40)) {
        tc_fence_after();
        const uint32_t idesc = nw == 256 ? idesc_bf16_f32(128, 256, false) : idesc_bf16_f32(128, 128, false);
        const uint32_t qa = smem_u32(qbuf), wa = smem_u32(wbuf);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t adesc = smem_desc_sw128(qa + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(wa + (ks >> 2) * 32768 + (ks & 3) * 32, 16, 1024);
          umma_f16_ss(tmem, adesc, bdesc, idesc, ks > 0 ? 1u : 0u);
        }
      }
      umma_commit(&bars[1]);  // arrives once every MMA issued above (possibly none) completed
    }
    __syncwarp();
  }
  // Everything above reads only inputs of the call; what follows writes the workspace,
  // which the previous call's kernels read, so it waits for them.
  grid_dep_wait();
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && warp == 3)
    tile_prefix_warp(a.seq_lens, a.batch, a.tile_tokens, a.tile_prefix);
  const int r = 32 * (warp & 3) + lane;  // sequence within the chunk = TMEM lane
  const int s = s0 + r;
  const int part = warp >> 2;            // columns [256 nh + 128 part, +128); rope pairs [16 part, +16)
  const long long row = (static_cast<long long>(s) * a.heads + i) * (dc + 64);
  if (s < a.batch && nh == 0) {
    // RoPE of the query's rope part at position L-1 (or the caller's q_positions[s], for a
    // token range of a longer sequence), while the loads and MMAs run: pair (j, j + 32)
    // turns by pos * theta^(-2j/64) radians.  The angle is carried in turns (fp64: pos
    // reaches 2^21); its fractional part is exact and is then evaluated in fp32 by sincospif.
    const int L = a.seq_lens[s];
    const double pos = static_cast<double>(a.q_positions != nullptr ? max(a.q_positions[s], 0) : (L > 0 ? L - 1 : 0));
    const uint4* qr = reinterpret_cast<const uint4*>(a.q + (static_cast<long long>(s) * a.heads + i) * 192 + 128);
    __align__(16) __nv_bfloat16 x1[16], x2[16];
    *reinterpret_cast<uint4*>(x1) = qr[2 * part];
    *reinterpret_cast<uint4*>(x1 + 8) = qr[2 * part + 1];
    *reinterpret_cast<uint4*>(x2) = qr[4 + 2 * part];
    *reinterpret_cast<uint4*>(x2 + 8) = qr[4 + 2 * part + 1];
    float y1[16], y2[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const double x = pos * turns[16 * part + u];
      const float f = static_cast<float>(x - rint(x));  // in [-1/2, 1/2]
      float sn, cs;
      sincospif(2.f * f, &sn, &cs);
      const float a1 = __bfloat162float(x1[u]), a2 = __bfloat162float(x2[u]);
      y1[u] = fmaf(a1, cs, -a2 * sn);
      y2[u] = fmaf(a1, sn, a2 * cs);
    }
    // rotated pair halves: elements [16 part, +16) and [32 + 16 part, +16) of the rope part
    {
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const float* y = h2 == 0 ? y1 : y2;
        const long long dst = row + dc + 32 * h2 + 16 * part;
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          __align__(16) __half h8[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) h8[u] = __float2half_rn(y[8 * v + u]);
          *reinterpret_cast<uint4*>(a.q_tilde + dst + 8 * v) = *reinterpret_cast<const uint4*>(h8);
        }
      }
    }
  }
  const bool done = mbar_wait(&bars[1], 0, kWaitNs, abort_flag, a.status, 41);
  tc_fence_after();
  if (done && !*abort_flag && 128 * part < nw) {
    const float scale = a.alpha_q * a.alpha_kv;
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      const int col = 128 * part + 32 * c;  // TMEM column = latent column - 256 nh
      const int k0 = 256 * nh + col;
      uint32_t v[32];
      tmem_ld32(tmem + lane_base + col, v);
      tmem_ld_wait();
      if (s < a.batch) {
        float x[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) x[u] = scale * __uint_as_float(v[u]);
        store_q32(a, row + k0, x);
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

// Whether group g of G has a non-empty tile range over T tiles.  With T >= G every group
// has one; otherwise (T < G <= 65535) the products below stay under 2^32, so the test needs
// no 64-bit division.
__device__ __forceinline__ bool group_live(int g, int G, int T) {
  if (T >= G) return true;
  const uint32_t t0 = static_cast<uint32_t>(g) * static_cast<uint32_t>(T) / static_cast<uint32_t>(G);
  const uint32_t t1 = static_cast<uint32_t>(g + 1) * static_cast<uint32_t>(T) / static_cast<uint32_t>(G);
  return t0 != t1;
}

// ---------------------------------------------------------------------------- merge
// grid (ceil(h / (256 / TPH)), d_c / 128 slices, B), 256 * Z threads.  Thread = (head, CPT
// consecutive latent columns of the slice); the Z thread sets take alternate runs of GU
// groups and are merged through shared memory at the end.  Every load of a run of GU
// groups is issued before any of them is used.
template <int CPT, int Z, int GU, bool PARTIAL = false>
__global__ void __launch_bounds__(256 * Z) merge_kernel(const CombineArgs a) {
  constexpr int TPH = 128 / CPT;    // threads per head
  constexpr int HPB = 256 / TPH;    // heads per block
  constexpr int V = CPT / 4;        // float4 per thread per group
  __shared__ float xchg[Z > 1 ? 256 : 1][CPT + 2];
  if (threadIdx.x == 0) grid_dep_launch();
  grid_dep_wait();  // the split partials and the tile prefix come from the previous kernels
  const int t = threadIdx.x & 255, z = threadIdx.x >> 8;
  const int head = blockIdx.x * HPB + t / TPH;
  const int col = (t % TPH) * CPT;  // within the slice
  const int slice = blockIdx.y, seq = blockIdx.z;
  const int p0 = a.tile_prefix[seq], p1 = a.tile_prefix[seq + 1], T = a.tile_prefix[a.batch];
  const int G = a.groups;
  float acc[CPT];
#pragma unroll
  for (int u = 0; u < CPT; ++u) acc[u] = 0.f;
  float M = -INFINITY, den = 0.f;
  if (p1 > p0 && head < a.heads) {
    const int g_lo = group_of_tile(p0, G, T), g_hi = group_of_tile(p1 - 1, G, T);
    for (int gb = g_lo + GU * z; gb <= g_hi; gb += GU * Z) {
      float2 ml[GU];
      float4 o[GU][V];
#pragma unroll
      for (int u = 0; u < GU; ++u) {
        const int g = gb + u;
        // a group with an empty tile range (more groups than tiles) wrote nothing
        const bool live = g <= g_hi && group_live(g, G, T);
        const long long row = ((static_cast<long long>(g) + seq) * gridDim.y + slice) * 128 + head;
        ml[u] = live ? a.ml_part[row] : make_float2(-INFINITY, 0.f);
#pragma unroll
        for (int v = 0; v < V; ++v)
          o[u][v] = live ? *reinterpret_cast<const float4*>(a.o_part + row * 128 + col + 4 * v)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float mx = M;
#pragma unroll
      for (int u = 0; u < GU; ++u) mx = fmaxf(mx, ml[u].x);
      if (mx != -INFINITY) {
        const float r = exp2f(M - mx);
        den *= r;
#pragma unroll
        for (int u = 0; u < CPT; ++u) acc[u] *= r;
#pragma unroll
        for (int u = 0; u < GU; ++u) {
          const float w = exp2f(ml[u].x - mx);
          den = fmaf(w, ml[u].y, den);
#pragma unroll
          for (int v = 0; v < V; ++v) {
            acc[4 * v + 0] = fmaf(w, o[u][v].x, acc[4 * v + 0]);
            acc[4 * v + 1] = fmaf(w, o[u][v].y, acc[4 * v + 1]);
            acc[4 * v + 2] = fmaf(w, o[u][v].z, acc[4 * v + 2]);
            acc[4 * v + 3] = fmaf(w, o[u][v].w, acc[4 * v + 3]);
          }
        }
        M = mx;
      }
    }
  }
  if (Z > 1) {
    if (z == 1) {
      xchg[t][0] = M;
      xchg[t][1] = den;
#pragma unroll
      for (int u = 0; u < CPT; ++u) xchg[t][2 + u] = acc[u];
    }
    __syncthreads();
    if (z != 0) return;
    const float M1 = xchg[t][0];
    const float mx = fmaxf(M, M1);
    if (mx != -INFINITY) {
      const float r0 = exp2f(M - mx), r1 = exp2f(M1 - mx);
      den = den * r0 + xchg[t][1] * r1;
#pragma unroll
      for (int u = 0; u < CPT; ++u) acc[u] = acc[u] * r0 + xchg[t][2 + u] * r1;
    }
    M = mx;  // den and acc are now relative to the larger maximum
  }
  if (head >= a.heads) return;
  const float inv = den > 0.f ? 1.f / den : 0.f;  // an empty sequence gives zeros
  if constexpr (PARTIAL) {
    // the state of this token range: the normalised latent row and log2 of its softmax
    // denominator (sum_t 2^(score_t log2 e) = 2^M * den)
    const long long hs = static_cast<long long>(seq) * a.heads + head;
    float4* dst = reinterpret_cast<float4*>(a.part_o + hs * a.d_c + 128 * slice + col);
#pragma unroll
    for (int v = 0; v < CPT / 4; ++v)
      dst[v] = make_float4(acc[4 * v] * inv, acc[4 * v + 1] * inv, acc[4 * v + 2] * inv, acc[4 * v + 3] * inv);
    if (col == 0) a.part_lse[hs * gridDim.y + slice] = den > 0.f ? M + log2f(den) : -INFINITY;
    return;
  }
  // o_lat as hi / lo bf16 terms, [h][B][d_c] each
  const long long base = (static_cast<long long>(head) * a.batch + seq) * a.d_c + 128 * slice + col;
  __align__(16) __nv_bfloat16 hi[CPT], lo[CPT];
#pragma unroll
  for (int u = 0; u < CPT; ++u) {
    const float x = acc[u] * inv;
    hi[u] = __float2bfloat16_rn(x);
    lo[u] = __float2bfloat16_rn(x - __bfloat162float(hi[u]));
  }
  __nv_bfloat16* lo_base = a.o_lat + static_cast<long long>(a.heads) * a.batch * a.d_c;
  if constexpr (CPT >= 8) {
#pragma unroll
    for (int v = 0; v < CPT / 8; ++v) {
      *reinterpret_cast<uint4*>(a.o_lat + base + 8 * v) = reinterpret_cast<const uint4*>(hi)[v];
      *reinterpret_cast<uint4*>(lo_base + base + 8 * v) = reinterpret_cast<const uint4*>(lo)[v];
    }
  } else {
    static_assert(CPT == 4, "columns per thread");
    *reinterpret_cast<uint2*>(a.o_lat + base) = *reinterpret_cast<const uint2*>(hi);
    *reinterpret_cast<uint2*>(lo_base + base) = *reinterpret_cast<const uint2*>(lo);
  }
}

// ---------------------------------------------------------------------------- upproj
struct UpprojCfg {
  static constexpr int A_BYTES = 2 * 2 * 128 * 128;  // hi, lo x 2 latent boxes of [128 sequences x 128 B]
  static constexpr int B_BYTES = 2 * 128 * 128;      // 2 output-column boxes of [128 latent rows x 128 B]
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = 2;                   // K chunks of 128 latent: d_c / 128 of them
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 64;
  static constexpr int TMEM_COLS = 128;
  static constexpr int THREADS = 256;
};

// grid (h, ceil(B / 128)), 256 threads.  Warp w owns the sequences of TMEM lane quadrant
// w % 4 and output columns [64 (w / 4), +64).
__global__ void __launch_bounds__(UpprojCfg::THREADS, 1)
upproj_tc_kernel(const __grid_constant__ CUtensorMap map_wuv, const __grid_constant__ CUtensorMap map_olat,
                 const CombineArgs a) {
  using C = UpprojCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + C::STAGES * C::STAGE_BYTES);  // [2]
  uint64_t* empty = full + 2;                                                       // [2]
  uint64_t* done_bar = empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int i = blockIdx.x;
  const int s0 = blockIdx.y * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    grid_dep_launch();
    for (int k = 0; k < 2; ++k) {
      mbar_init(&full[k], 1);
      mbar_init(&empty[k], 1);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
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
    // lane 0 streams the four K chunks through two stages and issues the MMAs; the other
    // lanes wait at the __syncwarp
    if (lane == 0) {
      const uint64_t stream_once = l2_policy_evict_first(), keep = l2_policy_evict_last();
      const int row_hi = i * a.batch + s0;             // this head's o_lat rows
      const int row_lo = row_hi + a.heads * a.batch;   // the lo term, h*B rows later
      // only the 32-row boxes that hold this chunk's sequences are loaded; the other A
      // rows feed D rows that are never stored
      const int nbox = min(4, (a.batch - s0 + 31) / 32);
      const int nchunks = a.d_c / 128;
      auto load_w = [&](int c) {  // W_UV rows of chunk c (an input of the call) + the byte count
        uint8_t* st = stages + (c % C::STAGES) * C::STAGE_BYTES;
        uint64_t* bar = &full[c % C::STAGES];
        mbar_arrive_expect_tx(bar, 4 * nbox * 4096 + C::B_BYTES);
        for (int db = 0; db < 2; ++db)
          tma_load_2d(st + C::A_BYTES + db * 16384, &map_wuv, bar, 64 * db, i * a.d_c + 128 * c, keep);
      };
      auto load_o = [&](int c) {  // o_lat rows of chunk c, written by the merge kernel
        uint8_t* st = stages + (c % C::STAGES) * C::STAGE_BYTES;
        uint64_t* bar = &full[c % C::STAGES];
        for (int t = 0; t < 2; ++t)
          for (int kb = 0; kb < 2; ++kb)
            for (int rb = 0; rb < nbox; ++rb)
              tma_load_2d(st + (t * 2 + kb) * 16384 + rb * 4096, &map_olat, bar, 128 * c + 64 * kb,
                          (t ? row_lo : row_hi) + 32 * rb, stream_once);
      };
      auto load = [&](int c) {
        load_w(c);
        load_o(c);
      };
      const int first = min(C::STAGES, nchunks);  // chunks loaded before the first MMA
      for (int c = 0; c < first; ++c) load_w(c);
      grid_dep_wait();
      for (int c = 0; c < first; ++c) load_o(c);
      int issued = first;
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, true);  // B (W_UV) MN-major
      const uint32_t base = smem_u32(stages);
      bool ok = true;
      for (int c = 0; c < nchunks && ok; ++c) {
        const int st = c % C::STAGES;
        if (!mbar_wait(&full[st], (c / C::STAGES) & 1, kWaitNs, abort_flag, a.status, 42)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = base + st * C::STAGE_BYTES, sb = sa + C::A_BYTES;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {  // latent rows 128 c + 16 ks .. + 15
          const uint64_t bdesc = smem_desc_sw128(sb + ks * 2048, 16384, 1024);
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const uint64_t adesc = smem_desc_sw128(sa + (t * 2 + (ks >> 2)) * 16384 + (ks & 3) * 32, 16, 1024);
            umma_f16_ss(tmem, adesc, bdesc, idesc, (c > 0 || ks > 0 || t > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[st]);
        // refill the other stage once the previous chunk's MMAs (queued ahead of these)
        // have read it
        if (c >= 1 && c + 1 < nchunks) {
          const int prev = c - 1;
          if (!mbar_wait(&empty[prev % C::STAGES], (prev / C::STAGES) & 1, kWaitNs, abort_flag, a.status, 43)) {
            ok = false;
            break;
          }
          load(c + 1);
          ++issued;
        }
      }
      umma_commit(done_bar);  // every MMA issued above (possibly none) completed
      if (!ok) {  // copies still in flight land before the CTA may exit
        volatile int never = 0;
        for (int k = max(0, issued - C::STAGES); k < issued; ++k)
          mbar_wait(&full[k % C::STAGES], (k / C::STAGES) & 1, kWaitNs, &never, a.status, 44);
      }
    }
    __syncwarp();
  }
  grid_dep_wait();  // (a no-op after the first) before writing out and reading the status
  const bool done = mbar_wait(done_bar, 0, kWaitNs, abort_flag, a.status, 45);
  tc_fence_after();
  const int r = 32 * (warp & 3) + lane;  // sequence within the chunk = TMEM lane
  const int s = s0 + r;
  const int part = warp >> 2;
  if (done && !*abort_flag) {
    const float scale = a.branch_scale * a.alpha_kv;
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      const int d0 = 64 * part + 32 * c;
      uint32_t v[32];
      tmem_ld32(tmem + lane_base + d0, v);
      tmem_ld_wait();
      if (s < a.batch) {
        const long long o = (static_cast<long long>(s) * a.heads + i) * 128 + d0;
        if (a.out_f32 && a.accumulate) {
          // this call's part of a sum over calls (tensor-parallel ranks): add it into this
          // rank's out and into every peer's, over NVLink for peer memory
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 x =
                make_float4(scale * __uint_as_float(v[4 * q]), scale * __uint_as_float(v[4 * q + 1]),
                            scale * __uint_as_float(v[4 * q + 2]), scale * __uint_as_float(v[4 * q + 3]));
            atomicAdd(reinterpret_cast<float4*>(a.out_f32 + o + 4 * q), x);
            for (int k = 0; k < a.n_peers; ++k) atomicAdd(reinterpret_cast<float4*>(a.peers[k] + o + 4 * q), x);
          }
        } else if (a.out_f32) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(a.out_f32 + o + 4 * q) =
                make_float4(scale * __uint_as_float(v[4 * q]), scale * __uint_as_float(v[4 * q + 1]),
                            scale * __uint_as_float(v[4 * q + 2]), scale * __uint_as_float(v[4 * q + 3]));
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            __align__(16) __nv_bfloat16 b8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) b8[u] = __float2bfloat16_rn(scale * __uint_as_float(v[8 * q + u]));
            *reinterpret_cast<uint4*>(a.out_bf16 + o + 8 * q) = *reinterpret_cast<const uint4*>(b8);
          }
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

// ---------------------------------------------------------------------------- small batches
// Merge + up-projection in one kernel for B <= kSmallBatch, where the two kernels above are
// bound by their load latencies (the merge's dependent rounds over many groups, the
// up-projection's 128-row MMA tiles holding a few sequences).  Grid (d_c / 128 slices, h)
// in clusters of the slices of one head, 512 threads.  CTA (slice c, head i):
//   1. reads W_UV[i] rows [128 c, 128 c + 128) into registers (thread = 16 rows x 2
//      columns) before waiting for the decode, since no kernel of the call writes it;
//   2. merges the split partials of slice c for every sequence: the (sequence, group)
//      pairs are laid end to end and thread set z = t / 128 takes every fourth one, all of
//      its loads issued before any is used; the four sets are combined in shared memory;
//   3. multiplies the merged latent row by its W_UV rows (fp32 sums) and leaves the partial
//      output of each sequence in shared memory;
//   4. cluster rank 0 adds the slices' partials (distributed shared memory) and writes out.
// The only waits are the two cluster barriers, which every thread of every CTA reaches.
constexpr int kSmallThreads = 512;
constexpr int kSmallLoads = 10;  // (sequence, group) pairs a thread set loads per round

__global__ void __launch_bounds__(kSmallThreads, 2) combine_small_kernel(const CombineArgs a) {
  constexpr int SB = kSmallBatch;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ float x_acc[4][SB][128];
  __shared__ float2 x_md[4][SB][128];
  __shared__ float o_lat[SB][128];
  __shared__ float red[8][SB][128];
  __shared__ float part[SB][128];
  __shared__ int seg_pre[SB + 1], seg_gl[SB];
  const int t = threadIdx.x;
  const int c = blockIdx.x, slices = gridDim.x, i = blockIdx.y;
  if (t == 0) grid_dep_launch();

  // 1. W_UV rows 128 c + 16 rg + k (k < 16), columns 2 cp and 2 cp + 1
  const int rg = t >> 6, cp = t & 63;
  uint32_t w[16];
  {
    const uint32_t* src =
        reinterpret_cast<const uint32_t*>(a.w_uv + (static_cast<long long>(i) * a.d_c + 128 * c + 16 * rg) * 128) + cp;
#pragma unroll
    for (int k = 0; k < 16; ++k) w[k] = __ldg(src + 64 * k);
  }
  grid_dep_wait();  // the split partials and the tile prefix come from the previous kernels

  // 2. merge.  Lane s of warp 0 finds sequence s's group range [g_lo, g_lo + n); the ranges
  // are laid end to end (pair q of sequence s is group gl[s] + q).
  const int z = t >> 7, j = t & 127;
  const int B = a.batch, G = a.groups, T = a.tile_prefix[B];
  if (t < 32) {
    int g0 = 0, n = 0;
    if (t < B) {
      const int p0 = a.tile_prefix[t], p1 = a.tile_prefix[t + 1];
      if (p1 > p0) {
        g0 = group_of_tile(p0, G, T);
        n = group_of_tile(p1 - 1, G, T) - g0 + 1;
      }
    }
    int incl = n;  // inclusive prefix over the (at most SB) sequences
#pragma unroll
    for (int off = 1; off < SB; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (t >= off) incl += v;
    }
    if (t < SB) {
      seg_pre[t + 1] = incl;
      seg_gl[t] = g0 - (incl - n);
    }
    if (t == 0) seg_pre[0] = 0;
  }
  __syncthreads();
  int gl[SB], pre[SB + 1];
#pragma unroll
  for (int s = 0; s <= SB; ++s) pre[s] = seg_pre[s];
#pragma unroll
  for (int s = 0; s < SB; ++s) gl[s] = seg_gl[s];
  float acc[SB], M[SB], den[SB];
#pragma unroll
  for (int s = 0; s < SB; ++s) {
    acc[s] = 0.f;
    M[s] = -INFINITY;
    den[s] = 0.f;
  }
  for (int q0 = z; q0 < pre[SB]; q0 += 4 * kSmallLoads) {
    float2 ml[kSmallLoads];
    float o[kSmallLoads];
    int sq[kSmallLoads];
#pragma unroll
    for (int u = 0; u < kSmallLoads; ++u) {
      const int q = q0 + 4 * u;
      int s = 0;
#pragma unroll
      for (int k = 1; k < SB; ++k) s += q >= pre[k] ? 1 : 0;
      int g = q;
#pragma unroll
      for (int k = 0; k < SB; ++k) g += s == k ? gl[k] : 0;
      // a group with an empty tile range (more groups than tiles) wrote nothing
      const bool live = q < pre[SB] && group_live(g, G, T);
      const int row = ((g + s) * slices + c) * 128 + i;  // < (65535 + 1024) * 4 * 128
      sq[u] = s;
      ml[u] = live ? a.ml_part[row] : make_float2(-INFINITY, 0.f);
      o[u] = live ? a.o_part[static_cast<long long>(row) * 128 + j] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kSmallLoads; ++u) {
      if (ml[u].x == -INFINITY) continue;
#pragma unroll
      for (int s = 0; s < SB; ++s) {
        if (sq[u] != s) continue;
        const float mx = fmaxf(M[s], ml[u].x);
        const float r = ex2_approx(M[s] - mx), wt = ex2_approx(ml[u].x - mx);
        den[s] = fmaf(den[s], r, wt * ml[u].y);
        acc[s] = fmaf(acc[s], r, wt * o[u]);
        M[s] = mx;
      }
    }
  }
#pragma unroll
  for (int s = 0; s < SB; ++s) {
    x_acc[z][s][j] = acc[s];
    x_md[z][s][j] = make_float2(M[s], den[s]);
  }
  __syncthreads();
  if (z < SB) {  // thread (sequence z, column j) combines the four sets
    const int s = z;
    float mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < 4; ++k) mx = fmaxf(mx, x_md[k][s][j].x);
    float num = 0.f, d = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 md = x_md[k][s][j];
        const float wt = ex2_approx(md.x - mx);
        d = fmaf(wt, md.y, d);
        num = fmaf(wt, x_acc[k][s][j], num);
      }
    }
    o_lat[s][j] = d > 0.f ? num / d : 0.f;  // an empty sequence gives zeros
  }
  __syncthreads();

  // 3. partial up-projection over this slice's 128 latent rows
#pragma unroll
  for (int s = 0; s < SB; ++s) {
    if (s >= B) break;
    float2 y = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float x = o_lat[s][16 * rg + k];
      const float2 wf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
      y.x = fmaf(x, wf.x, y.x);
      y.y = fmaf(x, wf.y, y.y);
    }
    red[rg][s][2 * cp] = y.x;
    red[rg][s][2 * cp + 1] = y.y;
  }
  __syncthreads();
  if (z < SB && z < B) {
    float y = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) y += red[k][z][j];
    part[z][j] = y;
  }

  // 4. rank 0 of the head's cluster sums the slices and writes out
  cluster.sync();
  if (cluster.block_rank() == 0 && z < SB && z < B) {
    const int s = z;
    float y = part[s][j];
    for (int r = 1; r < slices; ++r) y += *cluster.map_shared_rank(&part[s][j], r);
    y *= a.branch_scale * a.alpha_kv;
    const long long o = (static_cast<long long>(s) * a.heads + i) * 128 + j;
    if (a.out_f32 && a.accumulate) {
      atomicAdd(a.out_f32 + o, y);
      for (int k = 0; k < a.n_peers; ++k) atomicAdd(a.peers[k] + o, y);
    } else if (a.out_f32) {
      a.out_f32[o] = y;
    } else {
      a.out_bf16[o] = __float2bfloat16_rn(y);
    }
  }
  cluster.sync();  // the other slices keep their shared memory until rank 0 has read it
}

// ---------------------------------------------------------------------------- partial states
// hra_combine_partials: grid (ceil(h / 32), d_c / 128 slices, B), 256 threads; thread =
// (head, 16 consecutive latent columns of the slice).  Merges the a.n_parts states of its
// (sequence, head, slice) by their log2 softmax denominators and writes the merged row as
// o_lat's hi / lo bf16 terms, which the up-projection then reads.
__global__ void __launch_bounds__(256) partial_combine_kernel(const CombineArgs a) {
  constexpr int CPT = 16;
  if (threadIdx.x == 0) grid_dep_launch();
  grid_dep_wait();  // o_lat is read by the previous call's up-projection
  const int head = blockIdx.x * 32 + threadIdx.x / 8;
  const int col = (threadIdx.x % 8) * CPT;
  const int slice = blockIdx.y, seq = blockIdx.z, slices = gridDim.y;
  if (head >= a.heads) return;
  const long long hs = static_cast<long long>(seq) * a.heads + head;
  const long long part_o = static_cast<long long>(a.batch) * a.heads * a.d_c;     // elements per part
  const long long part_l = static_cast<long long>(a.batch) * a.heads * slices;
  float m = -INFINITY;
  for (int r = 0; r < a.n_parts; ++r) m = fmaxf(m, a.parts_lse[r * part_l + hs * slices + slice]);
  float acc[CPT];
#pragma unroll
  for (int u = 0; u < CPT; ++u) acc[u] = 0.f;
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int r = 0; r < a.n_parts; ++r) {
      const float lse = a.parts_lse[r * part_l + hs * slices + slice];
      if (lse == -INFINITY) continue;
      const float wt = exp2f(lse - m);
      wsum += wt;
      const float4* src = reinterpret_cast<const float4*>(a.parts_o + r * part_o + hs * a.d_c + 128 * slice + col);
#pragma unroll
      for (int v = 0; v < CPT / 4; ++v) {
        const float4 x = src[v];
        acc[4 * v + 0] = fmaf(wt, x.x, acc[4 * v + 0]);
        acc[4 * v + 1] = fmaf(wt, x.y, acc[4 * v + 1]);
        acc[4 * v + 2] = fmaf(wt, x.z, acc[4 * v + 2]);
        acc[4 * v + 3] = fmaf(wt, x.w, acc[4 * v + 3]);
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;  // every range empty: zeros
  const long long base = (static_cast<long long>(head) * a.batch + seq) * a.d_c + 128 * slice + col;
  __align__(16) __nv_bfloat16 hi[CPT], lo[CPT];
#pragma unroll
  for (int u = 0; u < CPT; ++u) {
    const float x = acc[u] * inv;
    hi[u] = __float2bfloat16_rn(x);
    lo[u] = __float2bfloat16_rn(x - __bfloat162float(hi[u]));
  }
  __nv_bfloat16* lo_base = a.o_lat + static_cast<long long>(a.heads) * a.batch * a.d_c;
#pragma unroll
  for (int v = 0; v < CPT / 8; ++v) {
    *reinterpret_cast<uint4*>(a.o_lat + base + 8 * v) = reinterpret_cast<const uint4*>(hi)[v];
    *reinterpret_cast<uint4*>(lo_base + base + 8 * v) = reinterpret_cast<const uint4*>(lo)[v];
  }
}

template <class K>
cudaError_t set_smem(K kern, int bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

int absorb_seq_chunk(int) { return 128; }
int upproj_seq_chunk() { return 32; }

cudaError_t launch_absorb_q(const CUtensorMap& map_wuk, const CUtensorMap& map_q, const AbsorbArgs& a,
                            cudaStream_t stream, bool pdl) {
  cudaError_t e = set_smem(absorb_tc_kernel, AbsorbCfg::SMEM);
  if (e != cudaSuccess) return e;
  return launch_kernel(absorb_tc_kernel, dim3(a.heads, (a.batch + 127) / 128, a.d_c > 256 ? a.d_c / 256 : 1),
                       dim3(AbsorbCfg::THREADS),
                       AbsorbCfg::SMEM, stream, pdl, map_wuk, map_q, a);
}

cudaError_t launch_combine_upproj(const CUtensorMap& map_wuv, const CUtensorMap& map_olat, const CombineArgs& a,
                                  cudaStream_t stream, bool pdl) {
  // The fused kernel takes one CTA per (head, slice) and one or two load rounds per thread
  // set for up to 64 groups: used where that grid fits on the SMs at once.  With more heads
  // or groups the merge kernel and the tensor-core up-projection are faster (measured at
  // h = 128 with 37 and 148 groups).
  if (a.part_o != nullptr) {  // partial mode: the merged states are the call's output
    if (a.batch >= 16)
      return launch_kernel(merge_kernel<16, 1, 2, true>, dim3((a.heads + 31) / 32, a.d_c / 128, a.batch), dim3(256),
                           0, stream, pdl, a);
    return launch_kernel(merge_kernel<4, 2, 4, true>, dim3((a.heads + 7) / 8, a.d_c / 128, a.batch), dim3(512), 0,
                         stream, pdl, a);
  }
  if (a.batch <= kSmallBatch && (a.d_c / 128) * a.heads <= a.sms && a.groups <= 64)
    return launch_kernel_cluster(combine_small_kernel, dim3(a.d_c / 128, a.heads), dim3(kSmallThreads), 0, stream, pdl,
                                 a.d_c / 128, a);
  // Many sequences: 32 heads x 4 float4 per block.  Few sequences (each spread over many
  // groups): 8 heads x 1 float4 per block and two thread sets over alternate group runs.
  cudaError_t e;
  if (a.batch >= 16)
    e = launch_kernel(merge_kernel<16, 1, 2>, dim3((a.heads + 31) / 32, a.d_c / 128, a.batch), dim3(256), 0, stream,
                      pdl, a);
  else
    e = launch_kernel(merge_kernel<4, 2, 4>, dim3((a.heads + 7) / 8, a.d_c / 128, a.batch), dim3(512), 0, stream,
                      pdl, a);
  if (e != cudaSuccess) return e;
  if ((e = set_smem(upproj_tc_kernel, UpprojCfg::SMEM)) != cudaSuccess) return e;
  return launch_kernel(upproj_tc_kernel, dim3(a.heads, (a.batch + 127) / 128), dim3(UpprojCfg::THREADS),
                       UpprojCfg::SMEM, stream, pdl, map_wuv, map_olat, a);
}

cudaError_t launch_combine_partials(const CUtensorMap& map_wuv, const CUtensorMap& map_olat, const CombineArgs& a,
                                    cudaStream_t stream, bool pdl) {
  cudaError_t e = launch_kernel(partial_combine_kernel, dim3((a.heads + 31) / 32, a.d_c / 128, a.batch), dim3(256),
                                0, stream, pdl, a);
  if (e != cudaSuccess) return e;
  if ((e = set_smem(upproj_tc_kernel, UpprojCfg::SMEM)) != cudaSuccess) return e;
  return launch_kernel(upproj_tc_kernel, dim3(a.heads, (a.batch + 127) / 128), dim3(UpprojCfg::THREADS),
                       UpprojCfg::SMEM, stream, pdl, map_wuv, map_olat, a);
}

}  // namespace hra

// absorb_combine.cu -- the steps around the split-KV decode, on the tensor cores.
//
// absorb ("Multi-Head Low-Rank Attention", 方法步骤详情, step 1 -- query-side weight
// absorption), one CTA per (head i, chunk of BN sequences):
//     q~[s,i,0:512]^T = alpha_q * alpha_kv * W_UK[i] (512x128) . q_nope[s,i]^T
// as one tcgen05 pass: A = W_UK[i] (4 M-tiles of 128 latent rows, K = 128, K-major),
// B = the chunk's q_nope rows (N = BN, K-major), D in TMEM.  bf16 x bf16 products are
// exact in the fp32 accumulator, so this equals the fp32 definition up to summation
// order.  The epilogue stores q~ as fp16, or as the two-term bf16 split used by the MLRA-4
// kernel, and rotates q_rope at position L-1 (fp64 angles: positions reach 2^21).  The
// branch structure needs no special case: branch b's absorbed query is columns
// [b*w, (b+1)*w) of the same 512-vector (W_UK^(b),(i) is the matching row block).
//
// merge (step 2b): one warp per (sequence, 128-wide latent slice, head) combines the
// split-KV partial states by log-sum-exp: o = sum_g 2^(m_g - M) O_g / sum_g 2^(m_g - M) l_g,
// and stores o_lat as bf16 hi + lo terms.
//
// upproj (step 3), one CTA per (head i, chunk of BN sequences):
//     out[s,i,:]^T = branch_scale * alpha_kv * W_UV[i]^T (128x512) . o_lat[s,i,:]^T
// A = W_UV[i] read MN-major (its rows are latent indices, the 128 output columns are
// contiguous), B = o_lat hi and lo (two MMAs per K step), D in TMEM.  The branches
// partition the latent, so summing the per-branch up-projections is this one contraction.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "absorb_combine.h"
#include "schedule.cuh"
#include "sm100.cuh"

namespace hra {

namespace {

constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s bound on each wait

// ---------------------------------------------------------------------------- absorb
template <int BN>
struct AbsorbCfg {
  static constexpr int W_BYTES = 4 * 2 * 128 * 128;  // 4 M-tiles x 2 K-boxes of [128 rows x 128 B]
  static constexpr int Q_BYTES = 2 * BN * 128;       // 2 K-boxes of [BN rows x 128 B]
  static constexpr int SMEM = 1024 + W_BYTES + Q_BYTES + 64;
  static constexpr int TMEM_COLS = 4 * BN;
};

__device__ __forceinline__ void store_q(const AbsorbArgs& a, long long idx, float x) {
  if (a.two_term) {  // hi = bf16(x), lo = bf16(x - hi)
    __nv_bfloat16* hi = reinterpret_cast<__nv_bfloat16*>(a.q_tilde);
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi[idx] = h;
    hi[static_cast<long long>(a.batch) * a.heads * 576 + idx] = __float2bfloat16_rn(x - __bfloat162float(h));
  } else {
    a.q_tilde[idx] = __float2half_rn(x);
  }
}

// grid (h, ceil(B / BN)), 128 threads.
template <int BN>
__global__ void __launch_bounds__(128, 1)
absorb_tc_kernel(const __grid_constant__ CUtensorMap map_wuk, const __grid_constant__ CUtensorMap map_q,
                 const AbsorbArgs a) {
  using C = AbsorbCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* wbuf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qbuf = wbuf + C::W_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(qbuf + C::Q_BYTES);  // [0] loads landed, [1] MMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int i = blockIdx.x;
  const int s0 = blockIdx.y * BN;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < 4) a.status[threadIdx.x] = 0;  // fresh per call
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // warp 0 issues the loads and the MMAs from lane 0; its other lanes wait at the
    // __syncwarp so that no lane of this warp polls a barrier lane 0 has yet to release
    if (lane == 0) {
      const uint64_t stream_once = l2_policy_evict_first();
      mbar_arrive_expect_tx(&bars[0], C::W_BYTES + C::Q_BYTES);
      for (int m = 0; m < 4; ++m)
        for (int kb = 0; kb < 2; ++kb)
          tma_load_2d(wbuf + (m * 2 + kb) * 16384, &map_wuk, &bars[0], 64 * kb, i * 512 + 128 * m, stream_once);
      for (int kb = 0; kb < 2; ++kb)
        tma_load_2d(qbuf + kb * BN * 128, &map_q, &bars[0], i * 192 + 64 * kb, s0, stream_once);
      if (mbar_wait(&bars[0], 0, kWaitNs, abort_flag, a.status, 40)) {
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16_f32(128, BN, false);
        const uint32_t wa = smem_u32(wbuf), qa = smem_u32(qbuf);
        for (int m = 0; m < 4; ++m) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t adesc = smem_desc_sw128(wa + (m * 2 + (ks >> 2)) * 16384 + (ks & 3) * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(qa + (ks >> 2) * BN * 128 + (ks & 3) * 32, 16, 1024);
            umma_f16_ss(tmem + m * BN, adesc, bdesc, idesc, ks > 0 ? 1u : 0u);
          }
        }
      }
      umma_commit(&bars[1]);  // arrives once every MMA issued above (possibly none) completed
    }
    __syncwarp();
  } else {
    const int ns = min(BN, a.batch - s0);
    if (warp == 1 && blockIdx.x == 0 && blockIdx.y == 0) tile_prefix_warp(a.seq_lens, a.batch, a.tile_tokens, a.tile_prefix);
    // RoPE of the query's rope part at position L-1, while the loads and MMAs run: pair
    // (j, j + 32) turns by pos * theta^(-2j/64) radians.  The angle is carried in turns,
    // pos * theta^(-2j/64) / (2 pi), in fp64 (pos reaches 2^21); its fractional part is
    // exact and is then evaluated in fp32 by sincospif.  Lane = j for every thread here.
    const double turns = pow(static_cast<double>(a.rope_theta), -2.0 * lane / 64.0) * 0.15915494309189535;
    for (int e = threadIdx.x - 32; e < ns * 32; e += 96) {
      const int s = s0 + e / 32;
      const int L = a.seq_lens[s];
      const double x = static_cast<double>(L > 0 ? L - 1 : 0) * turns;
      const float f = static_cast<float>(x - rint(x));  // in [-1/2, 1/2]
      float sn, cs;
      sincospif(2.f * f, &sn, &cs);
      const __nv_bfloat16* qr = a.q + (static_cast<long long>(s) * a.heads + i) * 192 + 128;
      const float x1 = __bfloat162float(qr[lane]), x2 = __bfloat162float(qr[lane + 32]);
      const long long off = (static_cast<long long>(s) * a.heads + i) * 576 + 512;
      store_q(a, off + lane, fmaf(x1, cs, -x2 * sn));
      store_q(a, off + lane + 32, fmaf(x1, sn, x2 * cs));
    }
  }
  const bool done = mbar_wait(&bars[1], 0, kWaitNs, abort_flag, a.status, 41);
  tc_fence_after();
  if (done && !*abort_flag) {
    const float scale = a.alpha_q * a.alpha_kv;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int ns = min(BN, a.batch - s0);
#pragma unroll 1
    for (int m = 0; m < 4; ++m) {
      const int k = 128 * m + 32 * warp + lane;  // latent index = TMEM lane of tile m
#pragma unroll 1
      for (int c0 = 0; c0 < ns; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + m * BN + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 32; ++u)
          if (c0 + u < ns)
            store_q(a, (static_cast<long long>(s0 + c0 + u) * a.heads + i) * 576 + k, scale * __uint_as_float(v[u]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------- merge
// grid (ceil(h / (256 / TPH)), 4 slices, B), 256 * Z threads.  Thread = (head, CPT
// consecutive latent columns of the slice); the Z thread sets take alternate runs of GU
// groups and are merged through shared memory at the end.  Every load of a run of GU
// groups is issued before any of them is used.
template <int CPT, int Z, int GU>
__global__ void __launch_bounds__(256 * Z) merge_kernel(const CombineArgs a) {
  constexpr int TPH = 128 / CPT;    // threads per head
  constexpr int HPB = 256 / TPH;    // heads per block
  constexpr int V = CPT / 4;        // float4 per thread per group
  __shared__ float xchg[Z > 1 ? 256 : 1][CPT + 2];
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
        const bool live = g <= g_hi && group_tile_begin(g, G, T) != group_tile_begin(g + 1, G, T);
        const long long row = ((static_cast<long long>(g) + seq) * 4 + slice) * 128 + head;
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
  }
  if (head >= a.heads) return;
  const float inv = den > 0.f ? 1.f / den : 0.f;  // an empty sequence gives zeros
  // o_lat as hi / lo bf16 terms, [h][B][512] each
  const long long base = (static_cast<long long>(head) * a.batch + seq) * 512 + 128 * slice + col;
  __align__(16) __nv_bfloat16 hi[CPT], lo[CPT];
#pragma unroll
  for (int u = 0; u < CPT; ++u) {
    const float x = acc[u] * inv;
    hi[u] = __float2bfloat16_rn(x);
    lo[u] = __float2bfloat16_rn(x - __bfloat162float(hi[u]));
  }
  __nv_bfloat16* lo_base = a.o_lat + static_cast<long long>(a.heads) * a.batch * 512;
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
template <int BN>
struct UpprojCfg {
  static constexpr int W_BYTES = 4 * 2 * 128 * 128;  // 4 latent blocks x 2 output-column boxes
  static constexpr int O_BYTES = 2 * 8 * BN * 128;   // hi + lo, 8 latent boxes of [BN rows x 128 B]
  static constexpr int SMEM = 1024 + W_BYTES + O_BYTES + 64;
  static constexpr int TMEM_COLS = BN < 32 ? 32 : BN;
};

// grid (h, ceil(B / BN)), 128 threads.
template <int BN>
__global__ void __launch_bounds__(128, 1)
upproj_tc_kernel(const __grid_constant__ CUtensorMap map_wuv, const __grid_constant__ CUtensorMap map_olat,
                 const CombineArgs a) {
  using C = UpprojCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* wbuf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* obuf = wbuf + C::W_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(obuf + C::O_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int i = blockIdx.x;
  const int s0 = blockIdx.y * BN;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t stream_once = l2_policy_evict_first();
      mbar_arrive_expect_tx(&bars[0], C::W_BYTES + C::O_BYTES);
      for (int kb = 0; kb < 4; ++kb)
        for (int db = 0; db < 2; ++db)
          tma_load_2d(wbuf + (kb * 2 + db) * 16384, &map_wuv, &bars[0], 64 * db, i * 512 + 128 * kb, stream_once);
      const int row0 = i * a.batch + s0;  // this head's o_lat rows; the lo term sits h*B rows later
      for (int part = 0; part < 2; ++part)
        for (int kc = 0; kc < 8; ++kc)
          tma_load_2d(obuf + (part * 8 + kc) * BN * 128, &map_olat, &bars[0], 64 * kc, row0 + part * a.heads * a.batch,
                      stream_once);
      if (mbar_wait(&bars[0], 0, kWaitNs, abort_flag, a.status, 42)) {
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16_f32(128, BN, false) | (1u << 15);  // A MN-major
        const uint32_t wa = smem_u32(wbuf), oa = smem_u32(obuf);
#pragma unroll 1
        for (int ks = 0; ks < 32; ++ks) {  // latent rows k = 16 ks .. 16 ks + 15
          const uint64_t adesc = smem_desc_sw128(wa + (ks >> 3) * 2 * 16384 + (ks & 7) * 2048, 16384, 1024);
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const uint64_t bdesc = smem_desc_sw128(oa + (part * 8 + (ks >> 2)) * BN * 128 + (ks & 3) * 32, 16, 1024);
            umma_f16_ss(tmem, adesc, bdesc, idesc, (ks > 0 || part > 0) ? 1u : 0u);
          }
        }
      }
      umma_commit(&bars[1]);
    }
    __syncwarp();
  }
  const bool done = mbar_wait(&bars[1], 0, kWaitNs, abort_flag, a.status, 43);
  tc_fence_after();
  if (done && !*abort_flag) {
    const float scale = a.branch_scale * a.alpha_kv;
    const int d = 32 * warp + lane;  // output column = TMEM lane
    const int ns = min(BN, a.batch - s0);
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 16) {
      uint32_t v[16];
      tmem_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        if (c0 + u >= ns) continue;
        const long long o = (static_cast<long long>(s0 + c0 + u) * a.heads + i) * 128 + d;
        const float val = scale * __uint_as_float(v[u]);
        if (a.out_f32) a.out_f32[o] = val;
        else a.out_bf16[o] = __float2bfloat16_rn(val);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <class K>
cudaError_t set_smem(K kern, int bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

int absorb_seq_chunk(int batch) { return batch <= 32 ? 32 : 128; }
int upproj_seq_chunk() { return 32; }

cudaError_t launch_absorb_q(const CUtensorMap& map_wuk, const CUtensorMap& map_q, const AbsorbArgs& a,
                            cudaStream_t stream) {
  cudaError_t e;
  if (absorb_seq_chunk(a.batch) == 32) {
    if ((e = set_smem(absorb_tc_kernel<32>, AbsorbCfg<32>::SMEM)) != cudaSuccess) return e;
    absorb_tc_kernel<32><<<dim3(a.heads, (a.batch + 31) / 32), 128, AbsorbCfg<32>::SMEM, stream>>>(map_wuk, map_q, a);
  } else {
    if ((e = set_smem(absorb_tc_kernel<128>, AbsorbCfg<128>::SMEM)) != cudaSuccess) return e;
    absorb_tc_kernel<128><<<dim3(a.heads, (a.batch + 127) / 128), 128, AbsorbCfg<128>::SMEM, stream>>>(map_wuk,
                                                                                                         map_q, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_combine_upproj(const CUtensorMap& map_wuv, const CUtensorMap& map_olat, const CombineArgs& a,
                                  cudaStream_t stream) {
  // Many sequences: 32 heads x 4 float4 per block.  Few sequences (each spread over many
  // groups): 8 heads x 1 float4 per block and two thread sets over alternate group runs.
  if (a.batch >= 16)
    merge_kernel<16, 1, 2><<<dim3((a.heads + 31) / 32, 4, a.batch), 256, 0, stream>>>(a);
  else
    merge_kernel<4, 2, 4><<<dim3((a.heads + 7) / 8, 4, a.batch), 512, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  constexpr int BN = 32;
  if ((e = set_smem(upproj_tc_kernel<BN>, UpprojCfg<BN>::SMEM)) != cudaSuccess) return e;
  upproj_tc_kernel<BN><<<dim3(a.heads, (a.batch + BN - 1) / BN), 128, UpprojCfg<BN>::SMEM, stream>>>(map_wuv,
                                                                                                       map_olat, a);
  return cudaGetLastError();
}

}  // namespace hra

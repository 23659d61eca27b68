// absorb_combine.cu -- the two small steps around the split-KV decode.
//
// absorb_q ("Multi-Head Low-Rank Attention", 方法步骤详情, step 1 -- query-side weight
// absorption): for every sequence s and head i
//     q~[s,i,0:512]   = alpha_q * alpha_kv * W_UK[i] (512x128) . q_nope[s,i]
//     q~[s,i,512:576] = RoPE(q_rope[s,i], pos = L_s - 1)
// in fp32 (RoPE angles in fp64), stored as fp16 for the tensor-core decode.  The branch
// structure needs no special case here: branch b's absorbed query is columns
// [b*w, (b+1)*w) of the same 512-vector, because W_UK^(b),(i) is the matching row block.
//
// combine_upproj (steps 2b and 3): log-sum-exp merge of the split-KV partial states of
// every 128-wide latent slice into o_lat[s,i,0:512] = sum_t p_t C_t (per branch softmax),
// then the output up-projection and branch sum
//     out[s,i,:] = branch_scale * alpha_kv * o_lat[s,i,:] . W_UV[i]   (512x128)
// (the branches partition the latent, so summing the per-branch up-projections is one
// contraction over all 512 latent columns).
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "absorb_combine.h"
#include "schedule.cuh"

namespace hra {

namespace {

constexpr int kSeqPerBlock = 8;

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// One element of q~: fp16, or the two-term bf16 split hi = bf16(x), lo = bf16(x - hi).
__device__ __forceinline__ void store_q(const AbsorbArgs& a, long long idx, float x) {
  if (a.two_term) {
    __nv_bfloat16* hi = reinterpret_cast<__nv_bfloat16*>(a.q_tilde);
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi[idx] = h;
    hi[static_cast<long long>(a.batch) * a.heads * 576 + idx] = __float2bfloat16_rn(x - __bfloat162float(h));
  } else {
    a.q_tilde[idx] = __float2half_rn(x);
  }
}

// grid (h, ceil(B / 8)), 512 threads: thread t owns latent row t of W_UK[i] and issues all
// 16 vector loads of that row up front.
__global__ void __launch_bounds__(512) absorb_q_kernel(const AbsorbArgs a) {
  __shared__ __align__(16) float qn[128][kSeqPerBlock];  // [n][s]: 8 sequences per 2 vector loads
  const int i = blockIdx.x;
  const int s0 = blockIdx.y * kSeqPerBlock;
  const int ns = min(kSeqPerBlock, a.batch - s0);
  const int t = threadIdx.x;

  if (blockIdx.x == 0 && blockIdx.y == 0 && t < 4) a.status[t] = 0;  // fresh status per call

  uint4 w[16];
  const uint4* wrow = reinterpret_cast<const uint4*>(a.w_uk + (static_cast<long long>(i) * 512 + t) * 128);
#pragma unroll
  for (int c = 0; c < 16; ++c) w[c] = __ldg(wrow + c);

  for (int e = t; e < kSeqPerBlock * 128; e += 512) {
    const int s = e / 128, n = e % 128;
    qn[n][s] = s < ns ? __bfloat162float(a.q[(static_cast<long long>(s0 + s) * a.heads + i) * 192 + n]) : 0.f;
  }
  __syncthreads();

  float acc[kSeqPerBlock];
#pragma unroll
  for (int s = 0; s < kSeqPerBlock; ++s) acc[s] = 0.f;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint32_t wv[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float wf = (u & 1) ? bf_hi(wv[u >> 1]) : bf_lo(wv[u >> 1]);
      const float4 qa = *reinterpret_cast<const float4*>(&qn[c * 8 + u][0]);
      const float4 qb = *reinterpret_cast<const float4*>(&qn[c * 8 + u][4]);
      acc[0] = fmaf(wf, qa.x, acc[0]);
      acc[1] = fmaf(wf, qa.y, acc[1]);
      acc[2] = fmaf(wf, qa.z, acc[2]);
      acc[3] = fmaf(wf, qa.w, acc[3]);
      acc[4] = fmaf(wf, qb.x, acc[4]);
      acc[5] = fmaf(wf, qb.y, acc[5]);
      acc[6] = fmaf(wf, qb.z, acc[6]);
      acc[7] = fmaf(wf, qb.w, acc[7]);
    }
  }
  const float scale = a.alpha_q * a.alpha_kv;
  for (int s = 0; s < ns; ++s)
    store_q(a, (static_cast<long long>(s0 + s) * a.heads + i) * 576 + t, scale * acc[s]);

  // RoPE on the query's rope part at position L - 1: pair (j, j + 32) turns by
  // pos * theta^(-2j/64); angles in fp64 because positions reach 2^21.
  if (t < ns * 32) {
    const int s = t / 32, j = t % 32;
    const int L = a.seq_lens[s0 + s];
    const double pos = static_cast<double>(L > 0 ? L - 1 : 0);
    const double ang = pos * pow(static_cast<double>(a.rope_theta), -2.0 * j / 64.0);
    double sn, cs;
    sincos(ang, &sn, &cs);
    const __nv_bfloat16* qr = a.q + (static_cast<long long>(s0 + s) * a.heads + i) * 192 + 128;
    const double x1 = __bfloat162float(qr[j]), x2 = __bfloat162float(qr[j + 32]);
    const long long off = (static_cast<long long>(s0 + s) * a.heads + i) * 576 + 512;
    store_q(a, off + j, static_cast<float>(x1 * cs - x2 * sn));
    store_q(a, off + j + 32, static_cast<float>(x1 * sn + x2 * cs));
  }
}

// grid (h, ceil(B / 8)), 256 threads.
__global__ void __launch_bounds__(256) combine_upproj_kernel(const CombineArgs a) {
  __shared__ int prefix[kMaxBatch + 1];
  __shared__ __align__(16) float olat[512][kSeqPerBlock];  // [latent][s]
  __shared__ float part[4][kSeqPerBlock][128];
  const int i = blockIdx.x;
  const int s0 = blockIdx.y * kSeqPerBlock;
  const int ns = min(kSeqPerBlock, a.batch - s0);
  const int t = threadIdx.x;
  if (t < 32) tile_prefix_warp(a.seq_lens, a.batch, a.tile_tokens, prefix);
  __syncthreads();
  const int T = prefix[a.batch];
  const int G = a.groups;

  // 1) merge the partial softmax states: thread t owns latent columns 2t and 2t+1.  Every
  //    group between g_lo and g_hi that owns at least one tile streamed part of the
  //    sequence; groups with an empty range (more groups than tiles) wrote nothing.  The
  //    loads of several partials are independent and issued together.
  const int col = 2 * t, slice = col / 128, cin = col % 128;
  for (int s = 0; s < ns; ++s) {
    const int seq = s0 + s;
    float r0 = 0.f, r1 = 0.f;
    if (prefix[seq + 1] > prefix[seq]) {
      const int g_lo = group_of_tile(prefix[seq], G, T);
      const int g_hi = group_of_tile(prefix[seq + 1] - 1, G, T);
      float M = -INFINITY;
      for (int g0 = g_lo; g0 <= g_hi; g0 += 8) {
        float mv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int g = g0 + u;
          const bool live = g <= g_hi && group_tile_begin(g, G, T) != group_tile_begin(g + 1, G, T);
          mv[u] = live ? a.ml_part[((static_cast<long long>(g) + seq) * 4 + slice) * 128 + i].x : -INFINITY;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) M = fmaxf(M, mv[u]);
      }
      float den = 0.f;
      for (int g0 = g_lo; g0 <= g_hi; g0 += 4) {
        float2 mlv[4], ov[4];
        bool live[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int g = g0 + u;
          live[u] = g <= g_hi && group_tile_begin(g, G, T) != group_tile_begin(g + 1, G, T);
          const long long slot = static_cast<long long>(g) + seq;
          mlv[u] = live[u] ? a.ml_part[(slot * 4 + slice) * 128 + i] : make_float2(0.f, 0.f);
          ov[u] = live[u] ? *reinterpret_cast<const float2*>(a.o_part + ((slot * 4 + slice) * 128 + i) * 128 + cin)
                          : make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float wgt = live[u] ? exp2f(mlv[u].x - M) : 0.f;
          r0 = fmaf(wgt, ov[u].x, r0);
          r1 = fmaf(wgt, ov[u].y, r1);
          den = fmaf(wgt, mlv[u].y, den);
        }
      }
      r0 /= den;
      r1 /= den;
    }
    olat[col][s] = r0;
    olat[col + 1][s] = r1;
  }
  for (int s = ns; s < kSeqPerBlock; ++s) olat[col][s] = olat[col + 1][s] = 0.f;
  __syncthreads();

  // 2) out = branch_scale * alpha_kv * o_lat . W_UV[i]: thread t = (latent quarter kq,
  //    column pair d2), partial sums over 128 latent rows, reduced across quarters.  W is
  //    read 16 rows at a time so that 16 loads are in flight.
  const int d2 = t % 64, kq = t / 64;
  float acc0[kSeqPerBlock], acc1[kSeqPerBlock];
#pragma unroll
  for (int s = 0; s < kSeqPerBlock; ++s) acc0[s] = acc1[s] = 0.f;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(a.w_uv + static_cast<long long>(i) * 512 * 128) + d2;
#pragma unroll 1
  for (int k0 = kq * 128; k0 < kq * 128 + 128; k0 += 16) {
    uint32_t wv[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) wv[u] = __ldg(w + (k0 + u) * 64);
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const float w0 = bf_lo(wv[u]), w1 = bf_hi(wv[u]);
      const float4 oa = *reinterpret_cast<const float4*>(&olat[k0 + u][0]);
      const float4 ob = *reinterpret_cast<const float4*>(&olat[k0 + u][4]);
      const float ov[8] = {oa.x, oa.y, oa.z, oa.w, ob.x, ob.y, ob.z, ob.w};
#pragma unroll
      for (int s = 0; s < kSeqPerBlock; ++s) {
        acc0[s] = fmaf(ov[s], w0, acc0[s]);
        acc1[s] = fmaf(ov[s], w1, acc1[s]);
      }
    }
  }
  // reduce the 4 latent quarters
  for (int s = 0; s < kSeqPerBlock; ++s) {
    if (kq > 0) {
      part[kq][s][2 * d2] = acc0[s];
      part[kq][s][2 * d2 + 1] = acc1[s];
    }
  }
  __syncthreads();
  if (kq == 0) {
    const float scale = a.branch_scale * a.alpha_kv;
    for (int s = 0; s < ns; ++s) {
      const float v0 = scale * (acc0[s] + part[1][s][2 * d2] + part[2][s][2 * d2] + part[3][s][2 * d2]);
      const float v1 = scale * (acc1[s] + part[1][s][2 * d2 + 1] + part[2][s][2 * d2 + 1] + part[3][s][2 * d2 + 1]);
      const long long o = (static_cast<long long>(s0 + s) * a.heads + i) * 128 + 2 * d2;
      if (a.out_f32) {
        *reinterpret_cast<float2*>(a.out_f32 + o) = make_float2(v0, v1);
      } else {
        *reinterpret_cast<__nv_bfloat162*>(a.out_bf16 + o) = __floats2bfloat162_rn(v0, v1);
      }
    }
  }
}

}  // namespace

cudaError_t launch_absorb_q(const AbsorbArgs& a, cudaStream_t stream) {
  const dim3 grid(a.heads, (a.batch + kSeqPerBlock - 1) / kSeqPerBlock);
  absorb_q_kernel<<<grid, 512, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_combine_upproj(const CombineArgs& a, cudaStream_t stream) {
  const dim3 grid(a.heads, (a.batch + kSeqPerBlock - 1) / kSeqPerBlock);
  combine_upproj_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace hra

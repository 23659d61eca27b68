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

// grid (h, ceil(B / 8)), 256 threads: thread t owns latent rows t and t + 256 of W_UK[i].
__global__ void __launch_bounds__(256) absorb_q_kernel(const AbsorbArgs a) {
  __shared__ float qn[kSeqPerBlock][128];
  const int i = blockIdx.x;
  const int s0 = blockIdx.y * kSeqPerBlock;
  const int ns = min(kSeqPerBlock, a.batch - s0);
  const int t = threadIdx.x;

  if (blockIdx.x == 0 && blockIdx.y == 0 && t < 4) a.status[t] = 0;  // fresh status per call

  for (int e = t; e < ns * 128; e += 256) {
    const int s = e / 128, n = e % 128;
    qn[s][n] = __bfloat162float(a.q[(static_cast<long long>(s0 + s) * a.heads + i) * 192 + n]);
  }
  __syncthreads();

  const float scale = a.alpha_q * a.alpha_kv;
  const uint4* wrow0 = reinterpret_cast<const uint4*>(a.w_uk + (static_cast<long long>(i) * 512 + t) * 128);
  const uint4* wrow1 = reinterpret_cast<const uint4*>(a.w_uk + (static_cast<long long>(i) * 512 + t + 256) * 128);
  float acc0[kSeqPerBlock], acc1[kSeqPerBlock];
#pragma unroll
  for (int s = 0; s < kSeqPerBlock; ++s) acc0[s] = acc1[s] = 0.f;
#pragma unroll 2
  for (int c = 0; c < 16; ++c) {  // 8 bf16 of the row per step
    const uint4 w0 = __ldg(wrow0 + c), w1 = __ldg(wrow1 + c);
    const float a0[8] = {bf_lo(w0.x), bf_hi(w0.x), bf_lo(w0.y), bf_hi(w0.y),
                         bf_lo(w0.z), bf_hi(w0.z), bf_lo(w0.w), bf_hi(w0.w)};
    const float a1[8] = {bf_lo(w1.x), bf_hi(w1.x), bf_lo(w1.y), bf_hi(w1.y),
                         bf_lo(w1.z), bf_hi(w1.z), bf_lo(w1.w), bf_hi(w1.w)};
#pragma unroll
    for (int s = 0; s < kSeqPerBlock; ++s) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float qv = qn[s][c * 8 + u];
        acc0[s] = fmaf(a0[u], qv, acc0[s]);
        acc1[s] = fmaf(a1[u], qv, acc1[s]);
      }
    }
  }
  for (int s = 0; s < ns; ++s) {
    __half* dst = a.q_tilde + (static_cast<long long>(s0 + s) * a.heads + i) * 576;
    dst[t] = __float2half_rn(scale * acc0[s]);
    dst[t + 256] = __float2half_rn(scale * acc1[s]);
  }

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
    __half* dst = a.q_tilde + (static_cast<long long>(s0 + s) * a.heads + i) * 576 + 512;
    dst[j] = __float2half_rn(static_cast<float>(x1 * cs - x2 * sn));
    dst[j + 32] = __float2half_rn(static_cast<float>(x1 * sn + x2 * cs));
  }
}

// grid (h, ceil(B / 8)), 256 threads.
__global__ void __launch_bounds__(256) combine_upproj_kernel(const CombineArgs a) {
  __shared__ int prefix[kMaxBatch + 1];
  __shared__ float olat[kSeqPerBlock][512];
  __shared__ float part[4][kSeqPerBlock][128];
  const int i = blockIdx.x;
  const int s0 = blockIdx.y * kSeqPerBlock;
  const int ns = min(kSeqPerBlock, a.batch - s0);
  const int t = threadIdx.x;
  if (t < 32) tile_prefix_warp(a.seq_lens, a.batch, a.tile_tokens, prefix);
  __syncthreads();
  const int T = prefix[a.batch];
  const int G = a.groups;

  // 1) merge the partial softmax states: thread t owns latent columns 2t and 2t+1.
  const int col = 2 * t, slice = col / 128, cin = col % 128;
  for (int s = 0; s < ns; ++s) {
    const int seq = s0 + s;
    float r0 = 0.f, r1 = 0.f;
    if (prefix[seq + 1] > prefix[seq]) {
      const int g_lo = group_of_tile(prefix[seq], G, T);
      const int g_hi = group_of_tile(prefix[seq + 1] - 1, G, T);
      // Every group between g_lo and g_hi that owns at least one tile streamed part of this
      // sequence; groups with an empty range (more groups than tiles) wrote nothing.
      float M = -INFINITY;
      for (int g = g_lo; g <= g_hi; ++g) {
        if (group_tile_begin(g, G, T) == group_tile_begin(g + 1, G, T)) continue;
        M = fmaxf(M, a.ml_part[((static_cast<long long>(g) + seq) * 4 + slice) * 128 + i].x);
      }
      float den = 0.f;
      for (int g = g_lo; g <= g_hi; ++g) {
        if (group_tile_begin(g, G, T) == group_tile_begin(g + 1, G, T)) continue;
        const long long slot = static_cast<long long>(g) + seq;
        const float2 ml = a.ml_part[(slot * 4 + slice) * 128 + i];
        const float wgt = exp2f(ml.x - M);
        const float2 o = *reinterpret_cast<const float2*>(a.o_part + ((slot * 4 + slice) * 128 + i) * 128 + cin);
        r0 = fmaf(wgt, o.x, r0);
        r1 = fmaf(wgt, o.y, r1);
        den = fmaf(wgt, ml.y, den);
      }
      r0 /= den;
      r1 /= den;
    }
    olat[s][col] = r0;
    olat[s][col + 1] = r1;
  }
  __syncthreads();

  // 2) out = branch_scale * alpha_kv * o_lat . W_UV[i]: thread t = (latent quarter kq,
  //    column pair d2), partial sums over 128 latent rows, reduced across quarters.
  const int d2 = t % 64, kq = t / 64;
  float acc0[kSeqPerBlock], acc1[kSeqPerBlock];
#pragma unroll
  for (int s = 0; s < kSeqPerBlock; ++s) acc0[s] = acc1[s] = 0.f;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(a.w_uv + static_cast<long long>(i) * 512 * 128) + d2;
#pragma unroll 4
  for (int k = kq * 128; k < kq * 128 + 128; ++k) {
    const uint32_t wv = __ldg(w + k * 64);
    const float w0 = bf_lo(wv), w1 = bf_hi(wv);
#pragma unroll
    for (int s = 0; s < kSeqPerBlock; ++s) {
      const float o = olat[s][k];
      acc0[s] = fmaf(o, w0, acc0[s]);
      acc1[s] = fmaf(o, w1, acc1[s]);
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
  absorb_q_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_combine_upproj(const CombineArgs& a, cudaStream_t stream) {
  const dim3 grid(a.heads, (a.batch + kSeqPerBlock - 1) / kSeqPerBlock);
  combine_upproj_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace hra

// combine.cuh -- merge of key-range partial attentions through their softmax
// statistics, in fp32 (the per-rank statistics merge of "feat(ltx2): tile-parallel
// video VAE and the two-stage pipeline", commit "Onboard Lightricks LTX-2.5",
// applied here to key ranges of one GPU):
//     L = max_p lse_p,  w_p = 2^(lse_p - L),  O = sum_p w_p O_p / sum_p w_p
// where O_p is part p's normalised output and lse_p its base-2 log-sum-exp.
// One thread per 4 consecutive output elements; output bf16 BSHD.
#pragma once

#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace ltx {

constexpr int kCombineThreads = 256;

template <int D>
__global__ void __launch_bounds__(kCombineThreads)
    ltx_attn_combine(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                   __nv_bfloat16* __restrict__ out, int num_splits, int batch, int heads, int q_len,
                   int rows_pad) {
  constexpr int kVec = D / 4;
  const long long tid = (long long)blockIdx.x * kCombineThreads + threadIdx.x;
  const long long total = (long long)batch * q_len * heads * kVec;
  if (tid >= total) return;
  const int c = (int)(tid % kVec);
  const long long bsh = tid / kVec;  // (b*q_len + i)*heads + h
  const int h = (int)(bsh % heads);
  const long long bs = bsh / heads;
  const int i = (int)(bs % q_len);
  const int b = (int)(bs / q_len);

  const size_t split_stride = (size_t)batch * heads * rows_pad;
  const size_t row0 = ((size_t)b * heads + h) * rows_pad + i;
  float lmax = -INFINITY;
  for (int s = 0; s < num_splits; ++s) lmax = fmaxf(lmax, lse_part[s * split_stride + row0]);
  float wsum = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < num_splits; ++s) {
    const size_t r = s * split_stride + row0;
    const float w = ex2(lse_part[r] - lmax);
    const float4 o = reinterpret_cast<const float4*>(o_part + r * D)[c];
    wsum += w;
    acc.x = fmaf(w, o.x, acc.x);
    acc.y = fmaf(w, o.y, acc.y);
    acc.z = fmaf(w, o.z, acc.z);
    acc.w = fmaf(w, o.w, acc.w);
  }
  const float inv = 1.0f / wsum;
  uint2 packed;
  packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  reinterpret_cast<uint2*>(out + (size_t)bsh * D)[c] = packed;
}

}  // namespace ltx

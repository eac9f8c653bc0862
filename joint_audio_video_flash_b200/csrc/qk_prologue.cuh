// qk_prologue.cuh -- the queries' and keys' norm and rotary step ahead of attention, on
// sm_100a.  The LTX-2.5 DiT attends with "normed and rotated" queries and keys and keeps
// RoPE tables per latent grid ("feat(ltx2): tile-parallel video VAE and the two-stage
// pipeline", commit "Onboard Lightricks LTX-2.5"); the pages fix neither the norm nor the
// rotary layout, so this computes the plainest reading:
//
//   per token, over its whole inner dimension (heads * head_dim):
//     r = sqrt(mean x^2 + eps);  y = x / r * weight                       (RMSNorm)
//   within each head, for each pair of adjacent channels (2i, 2i+1):
//     out[2i] = y[2i] cos[l,i] - y[2i+1] sin[l,i];  out[2i+1] = y[2i] sin[l,i] + y[2i+1] cos[l,i]
//
// One warp per (tensor, token row): every lane keeps its 16-byte chunks of the row in
// registers, the warp reduces the sum of squares with shuffles, then each lane scales,
// rotates (fp32) and stores its chunks.  A row is read completely before any of it is
// written, so the output may be the input (in place).  Queries and keys run in one launch.
// The work streams HBM once: read q, k (bf16), write them (bf16); weights and tables are
// small and stay in cache.
#pragma once

#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace ltx {

constexpr int kPrologueWarps = 8;  // token rows per CTA

struct PrologueParams {
  const __nv_bfloat16* x[2];  // q, k: [rows][inner]
  __nv_bfloat16* out[2];      // q_out, k_out (may equal x)
  const __nv_bfloat16* w[2];  // weights [inner]
  const float* cos_t;         // [seq_len][head_dim / 2]
  const float* sin_t;
  long long rows;             // batch * seq_len
  int seq_len;
  int head_dim;
  float eps;
};

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// CHUNKS 16-byte (8 x bf16) chunks per lane: inner dimension = CHUNKS * 32 * 8.
template <int CHUNKS>
__global__ void __launch_bounds__(kPrologueWarps * 32)
    qk_norm_rope(const PrologueParams p) {
  constexpr int kInner = CHUNKS * 32 * 8;
  const int lane = threadIdx.x & 31;
  const long long gw = (long long)blockIdx.x * kPrologueWarps + (threadIdx.x >> 5);
  if (gw >= 2 * p.rows) return;
  const int t = gw >= p.rows ? 1 : 0;  // 0: queries, 1: keys
  const long long row = gw - (long long)t * p.rows;
  const int l = (int)(row % p.seq_len);
  // select by condition (a runtime index into the parameter arrays would copy them to
  // local memory)
  const __nv_bfloat16* x = t ? p.x[1] : p.x[0];
  __nv_bfloat16* out = t ? p.out[1] : p.out[0];
  const __nv_bfloat16* w = t ? p.w[1] : p.w[0];
  const uint4* src = reinterpret_cast<const uint4*>(x + row * kInner);

  uint4 v[CHUNKS];
  float ss = 0.0f;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    v[c] = src[c * 32 + lane];
    const uint32_t u[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = bf16_lo(u[j]), b = bf16_hi(u[j]);
      ss = fmaf(a, a, fmaf(b, b, ss));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float inv_r = rsqrtf(ss * (1.0f / kInner) + p.eps);

  const uint4* wv = reinterpret_cast<const uint4*>(w);
  uint4* dst = reinterpret_cast<uint4*>(out + row * kInner);
  const int half = p.head_dim >> 1;
  const float* cos_row = p.cos_t + (size_t)l * half;
  const float* sin_row = p.sin_t + (size_t)l * half;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int e0 = (c * 32 + lane) * 8;   // first element of the chunk in the row
    const int i0 = (e0 % p.head_dim) >> 1;  // first pair of the chunk within its head
    const uint4 w4 = __ldg(wv + c * 32 + lane);
    const float4 cs = __ldg(reinterpret_cast<const float4*>(cos_row + i0));
    const float4 sn = __ldg(reinterpret_cast<const float4*>(sin_row + i0));
    const uint32_t xu[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
    const uint32_t wu[4] = {w4.x, w4.y, w4.z, w4.w};
    const float cc[4] = {cs.x, cs.y, cs.z, cs.w};
    const float sc[4] = {sn.x, sn.y, sn.z, sn.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // pair j of the chunk: channels 2j, 2j+1
      const float y0 = bf16_lo(xu[j]) * inv_r * bf16_lo(wu[j]);
      const float y1 = bf16_hi(xu[j]) * inv_r * bf16_hi(wu[j]);
      o[j] = pack_bf16x2(fmaf(y0, cc[j], -y1 * sc[j]), fmaf(y0, sc[j], y1 * cc[j]));
    }
    dst[c * 32 + lane] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace ltx

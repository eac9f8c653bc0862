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
// The work streams HBM once (read q and k, write them, bf16); weights and tables are small
// and stay in cache.  So the kernel is built to keep loads in flight:
//  - a persistent grid (as many CTAs as fit on the SMs) walks groups of token rows; a CTA
//    of 8 warps takes 8 / WPR rows of a group, each row (of q or of k) held by WPR warps,
//    every lane keeping CHUNKS 16-byte chunks of it in registers;
//  - the next group's row is loaded before the current one is reduced and written, so a
//    warp always has a row in flight (two register sets, used alternately);
//  - the warps of a row reduce the sum of squares with shuffles and meet in shared memory
//    (two slots, alternating, so one barrier per group suffices);
//  - scaling and rotation run on packed fp32 pairs (two rotation pairs per instruction),
//    with 1/r folded into the cos and sin values.
// A row is read completely before any of it is written, and by the warps that write it,
// so the output may be the input (in place).  Queries and keys run in one launch.
#pragma once

#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace ltx {

constexpr int kPrologueWarps = 8;  // warps per CTA

struct PrologueParams {
  const __nv_bfloat16* x[2];  // q, k: [rows][inner]
  __nv_bfloat16* out[2];      // q_out, k_out (may equal x)
  const __nv_bfloat16* w[2];  // weights [inner]
  const float* cos_t;         // [seq_len][head_dim / 2]
  const float* sin_t;
  int rows;                   // batch * seq_len (< 2^30)
  int seq_len;
  int head_dim;
  float eps;
};

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Inner dimension = WPR warps * 32 lanes * CHUNKS chunks * 8 bf16.
template <int CHUNKS, int WPR>
struct PrologueRow {
  static constexpr int kInner = WPR * CHUNKS * 32 * 8;
  static constexpr int kRowsPerCta = kPrologueWarps / WPR;
};

template <int CHUNKS, int WPR>
__device__ __forceinline__ void prologue_load(const PrologueParams& p, int gr, int base,
                                              uint4 (&v)[CHUNKS]) {
  constexpr int kInner = PrologueRow<CHUNKS, WPR>::kInner;
  if (gr < 2 * p.rows) {
    const bool key = gr >= p.rows;
    const __nv_bfloat16* x = key ? p.x[1] : p.x[0];
    const uint4* src =
        reinterpret_cast<const uint4*>(x + (size_t)(gr - (key ? p.rows : 0)) * kInner) + base;
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) v[c] = __ldcs(src + c * 32);  // read once: evict first
  } else {
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) v[c] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Sum of squares, norm and rotation of the row group `g`'s rows held in v; `slot` picks the
// shared-memory reduction slots.
template <int CHUNKS, int WPR>
__device__ __forceinline__ void prologue_row(const PrologueParams& p, int gr, int base,
                                             const int (&pair0)[CHUNKS], const uint4 (&v)[CHUNKS],
                                             float* red) {
  constexpr int kInner = PrologueRow<CHUNKS, WPR>::kInner;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float2 ss2 = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const uint32_t u[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 ab = make_float2(bf16_lo(u[j]), bf16_hi(u[j]));
      ss2 = __ffma2_rn(ab, ab, ss2);
    }
  }
  float ss = ss2.x + ss2.y;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if constexpr (WPR > 1) {
    if (lane == 0) red[warp] = ss;
    // the whole CTA meets: a named barrier per row (so a CTA's two rows need not wait for
    // each other) measured 10 % slower at 4096 channels on B200
    __syncthreads();
    ss = 0.0f;
#pragma unroll
    for (int i = 0; i < WPR; ++i) ss += red[(warp / WPR) * WPR + i];
  }
  if (gr >= 2 * p.rows) return;
  const bool key = gr >= p.rows;
  const int row = gr - (key ? p.rows : 0);
  const int l = row % p.seq_len;
  const float inv_r = rsqrtf(ss * (1.0f / kInner) + p.eps);
  const float2 pr = make_float2(inv_r, inv_r), nr = make_float2(-inv_r, -inv_r);
  const uint4* wv = reinterpret_cast<const uint4*>(key ? p.w[1] : p.w[0]) + base;
  uint4* dst = reinterpret_cast<uint4*>((key ? p.out[1] : p.out[0]) + (size_t)row * kInner) + base;
  const int half = p.head_dim >> 1;
  const float* cos_row = p.cos_t + (size_t)l * half;
  const float* sin_row = p.sin_t + (size_t)l * half;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const uint4 w4 = __ldg(wv + c * 32);
    const float4 cs = __ldg(reinterpret_cast<const float4*>(cos_row + pair0[c]));
    const float4 sn = __ldg(reinterpret_cast<const float4*>(sin_row + pair0[c]));
    const uint32_t xu[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
    const uint32_t wu[4] = {w4.x, w4.y, w4.z, w4.w};
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // rotation pairs 2h and 2h+1 of the chunk, packed
      const int j = 2 * h;
      const float2 c2 = h ? make_float2(cs.z, cs.w) : make_float2(cs.x, cs.y);
      const float2 s2 = h ? make_float2(sn.z, sn.w) : make_float2(sn.x, sn.y);
      const float2 cr = __fmul2_rn(c2, pr), sr = __fmul2_rn(s2, pr), nsr = __fmul2_rn(s2, nr);
      // even and odd channels of the two pairs, times the weights
      const float2 ye = __fmul2_rn(make_float2(bf16_lo(xu[j]), bf16_lo(xu[j + 1])),
                                   make_float2(bf16_lo(wu[j]), bf16_lo(wu[j + 1])));
      const float2 yo = __fmul2_rn(make_float2(bf16_hi(xu[j]), bf16_hi(xu[j + 1])),
                                   make_float2(bf16_hi(wu[j]), bf16_hi(wu[j + 1])));
      const float2 oe = __ffma2_rn(ye, cr, __fmul2_rn(yo, nsr));  // y0 c - y1 s
      const float2 oo = __ffma2_rn(ye, sr, __fmul2_rn(yo, cr));   // y0 s + y1 c
      o[j] = pack_bf16x2(oe.x, oo.x);
      o[j + 1] = pack_bf16x2(oe.y, oo.y);
    }
    __stcs(dst + c * 32, make_uint4(o[0], o[1], o[2], o[3]));  // written once: evict first
  }
}

// MIN_CTAS: CTAs an SM must hold (the register cap; measured per row width, see the launch).
template <int CHUNKS, int WPR, int MIN_CTAS>
__global__ void __launch_bounds__(kPrologueWarps * 32, MIN_CTAS)
    ltx_qk_norm_rope(const PrologueParams p) {
  static_assert(kPrologueWarps % WPR == 0, "a CTA holds whole rows");
  constexpr int kRowsPerCta = PrologueRow<CHUNKS, WPR>::kRowsPerCta;
  __shared__ float red[2][kPrologueWarps];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int base = (warp % WPR) * CHUNKS * 32 + lane;  // this lane's first 16-byte chunk
  // pair index within its head of each chunk's first channel pair: chunk c starts at
  // element 8 * (base + 32 c), so the offset advances by 256 mod head_dim per chunk
  int pair0[CHUNKS];
  {
    int e = (base * 8) % p.head_dim;
    const int step = 256 % p.head_dim;
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      pair0[c] = e >> 1;
      e += step;
      if (e >= p.head_dim) e -= p.head_dim;
    }
  }
  const int n_groups = (2 * p.rows + kRowsPerCta - 1) / kRowsPerCta;
  const int slot = warp / WPR;
  uint4 va[CHUNKS], vb[CHUNKS];
  int g = blockIdx.x;
  prologue_load<CHUNKS, WPR>(p, g * kRowsPerCta + slot, base, va);
  while (g < n_groups) {  // g is the same for the whole CTA: the barriers inside are uniform
    const int g1 = g + gridDim.x;
    prologue_load<CHUNKS, WPR>(p, g1 * kRowsPerCta + slot, base, vb);
    prologue_row<CHUNKS, WPR>(p, g * kRowsPerCta + slot, base, pair0, va, red[0]);
    if (g1 >= n_groups) break;
    g = g1 + gridDim.x;
    prologue_load<CHUNKS, WPR>(p, g * kRowsPerCta + slot, base, va);
    prologue_row<CHUNKS, WPR>(p, g1 * kRowsPerCta + slot, base, pair0, vb, red[1]);
  }
}

}  // namespace ltx

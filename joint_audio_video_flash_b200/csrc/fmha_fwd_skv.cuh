// fmha_fwd_skv.cuh -- attention forward for a short key side (at most 256 keys) and
// head_dim 64 on sm_100a: a2v (video queries over the padded audio keys/values) and
// audio self-attention of an LTX-2 block ("LTX-2: replicate audio stream across
// Ulysses ranks by default", Description).  Same operation, layout and key mask as
// fmha_fwd.cuh.  With every key in one S tile the softmax max is exact, so there is
// no online rescale.  The work is bound by HBM (reading Q, writing O), so the design
// keeps loads and stores in flight instead of optimising the (small) MMAs:
//
//   - persistent: one CTA per SM walks a contiguous run of query tiles (flattened
//     over batch, head, tile); K and V of the current (batch, head) stay resident in
//     shared memory and are reloaded only when the run crosses into the next head;
//   - warp 0 streams Q tiles through a 4-stage TMA ring;
//   - warp 1 issues S = Q K^T (one M=128, N=128*n_kv MMA chain) for tile i+1 before
//     O = P V of tile i, so QK overlaps the softmax;
//   - two softmax warpgroups take alternate tiles, each with its own TMEM buffer
//     (S / P / O) and its own output staging buffer for the TMA store.
// TMEM (512 columns): buffer b at 256*b: S at [0, 128*n_kv), P packed over its first
// 64*n_kv columns, O at [128, 192) (for n_kv = 2 O reuses S columns the softmax has
// already read).
#pragma once

#include "fmha_fwd.cuh"

namespace ltx {

constexpr int kSkvThreads = 384;
constexpr int kSkvD = 64;
constexpr int kSkvMaxKvTiles = 2;

struct SkvSmem {
  static constexpr int kBoxBytes = kBlockM * 128;  // 128 rows x 64 bf16
  static constexpr int kQStages = 4;
  static constexpr int kK = 0;                                  // up to 2 key tiles
  static constexpr int kV = kK + kSkvMaxKvTiles * kBoxBytes;
  static constexpr int kQ = kV + kSkvMaxKvTiles * kBoxBytes;     // Q ring
  static constexpr int kStage = kQ + kQStages * kBoxBytes;       // 2 output staging
  static constexpr int kBar = kStage + 2 * kBoxBytes;
  static constexpr int bKVF = 0;
  static constexpr int bKVE = 1;
  static constexpr int bQF = 2;                 // kQStages
  static constexpr int bQE = bQF + kQStages;    // kQStages
  static constexpr int bSF = bQE + kQStages;    // 2
  static constexpr int bPF = bSF + 2;           // 2
  static constexpr int bOF = bPF + 2;           // 2
  static constexpr int bTF = bOF + 2;           // 2: TMEM buffer free
  static constexpr int bDrain = bTF + 2;
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kUsed = kAbort + 4;
  static constexpr int kAlloc = ((kUsed + 1024 + 1023) / 1024) * 1024 > kMinSmemFor1Cta
                                    ? ((kUsed + 1024 + 1023) / 1024) * 1024
                                    : kMinSmemFor1Cta;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 128;  // within a 256-column buffer
};

template <bool kUnused = false>
__global__ void __launch_bounds__(kSkvThreads, 1)
    fmha_fwd_skv_sm100(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using L = SkvSmem;
  constexpr int D = kSkvD;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_kv = p.n_kv_tiles;  // 1 or 2
  // contiguous run of flattened (batch, head, query tile) indices for this CTA
  const long long total = (long long)p.batch * p.heads * p.n_q_tiles;
  const long long t_begin = total * blockIdx.x / gridDim.x;
  const long long t_end = total * (blockIdx.x + 1) / gridDim.x;
  const int cnt = (int)(t_end - t_begin);
  auto tile_bh = [&](int i) -> int { return (int)((t_begin + i) / p.n_q_tiles); };
  auto tile_qt = [&](int i) -> int { return (int)((t_begin + i) % p.n_q_tiles); };

  if (threadIdx.x == 0) {
    mbar_init(bar(L::bKVF), 1);
    mbar_init(bar(L::bKVE), 1);
    for (int s = 0; s < L::kQStages; ++s) {
      mbar_init(bar(L::bQF + s), 1);
      mbar_init(bar(L::bQE + s), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar(L::bSF + g), 1);
      mbar_init(bar(L::bPF + g), kBlockM);
      mbar_init(bar(L::bOF + g), 1);
      mbar_init(bar(L::bTF + g), kBlockM);
    }
    mbar_init(bar(L::bDrain), 1);
    *abort_flag = (*reinterpret_cast<volatile int*>(p.status) != kDevOk) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + L::kTmemSlot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && !*abort_flag && cnt > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int cur_bh = -1, kv_loads = 0;
      int last_q[L::kQStages];
      for (int s = 0; s < L::kQStages; ++s) last_q[s] = -1;
      bool ok = true;
      for (int i = 0; i < cnt && ok; ++i) {
        const int bh = tile_bh(i);
        const int b = bh / p.heads, h = bh % p.heads;
        if (bh != cur_bh) {
          if (kv_loads > 0) ok = mbar_wait_lean(bar(L::bKVE), (uint32_t)(kv_loads - 1) & 1u, ctl);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(L::bKVF), 2 * n_kv * L::kBoxBytes);
          for (int t = 0; t < n_kv; ++t) {
            tma_load_4d(sbase + L::kK + t * L::kBoxBytes, &tm_k, bar(L::bKVF), 0, h,
                        t * kBlockN, b);
            tma_load_4d(sbase + L::kV + t * L::kBoxBytes, &tm_v, bar(L::bKVF), 0, h,
                        t * kBlockN, b);
          }
          cur_bh = bh;
          ++kv_loads;
        }
        const int qs = i % L::kQStages;
        ok = mbar_wait_lean(bar(L::bQE + qs), ((uint32_t)(i / L::kQStages) & 1u) ^ 1u, ctl);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(L::bQF + qs), L::kBoxBytes);
        tma_load_4d(sbase + L::kQ + qs * L::kBoxBytes, &tm_q, bar(L::bQF + qs), 0, h,
                    tile_qt(i) * kBlockM, b);
        last_q[qs] = i;
      }
      if (!ok) {
        for (int s = 0; s < L::kQStages; ++s)
          if (last_q[s] >= 0)
            mbar_wait_drain(bar(L::bQF + s), (uint32_t)(last_q[s] / L::kQStages) & 1u,
                            p.timeout_ns);
        if (kv_loads > 0)
          mbar_wait_drain(bar(L::bKVF), (uint32_t)(kv_loads - 1) & 1u, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && !*abort_flag && cnt > 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN * n_kv, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, D, true);
      bool issued = false;
      int kv_ver = -1, cur_bh = -1;
      // S_b = Q_i K^T into buffer b = i & 1 (waits for Q_i, the buffer and, on a head
      // change, the new K/V)
      auto qk = [&](int i) -> bool {
        const int bh = tile_bh(i);
        if (bh != cur_bh) {
          if (!mbar_wait_lean(bar(L::bKVF), (uint32_t)(kv_ver + 1) & 1u, ctl)) return false;
          ++kv_ver;
          cur_bh = bh;
        }
        const int bf = i & 1;
        const int qs = i % L::kQStages;
        if (!mbar_wait_lean(bar(L::bQF + qs), (uint32_t)(i / L::kQStages) & 1u, ctl) ||
            !mbar_wait_lean(bar(L::bTF + bf), ((uint32_t)(i >> 1) & 1u) ^ 1u, ctl))
          return false;
        tc_fence_after();
        const uint32_t q_base = sbase + L::kQ + qs * L::kBoxBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tmem + 256 * bf, smem_desc_sw128(q_base + kk * 32, 16, 1024),
                  smem_desc_sw128(sbase + L::kK + kk * 32, 16, 1024), idesc_qk,
                  kk > 0 ? 1u : 0u);
        issued = true;
        umma_commit(bar(L::bSF + bf));
        umma_commit(bar(L::bQE + qs));
        return true;
      };
      // O_b = P_b V (waits for P_i)
      auto pv = [&](int i) -> bool {
        const int bf = i & 1;
        if (!mbar_wait_lean(bar(L::bPF + bf), (uint32_t)(i >> 1) & 1u, ctl)) return false;
        tc_fence_after();
        for (int kk = 0; kk < (kBlockN / 16) * n_kv; ++kk)
          umma_ts(tmem + 256 * bf + L::kColO, tmem + 256 * bf + kk * 8,
                  smem_desc_sw128(sbase + L::kV + kk * 16 * 128, L::kBoxBytes, 1024), idesc_pv,
                  kk > 0 ? 1u : 0u);
        umma_commit(bar(L::bOF + bf));
        return true;
      };
      bool ok = qk(0);
      for (int i = 0; i < cnt && ok; ++i) {
        const bool next = i + 1 < cnt;
        const bool head_change = next && tile_bh(i + 1) != tile_bh(i);
        if (next && !head_change) ok = qk(i + 1);  // overlap QK(i+1) with softmax(i)
        if (ok) ok = pv(i);
        if (ok && head_change) {
          umma_commit(bar(L::bKVE));  // K/V of the finished head may be overwritten
          ok = qk(i + 1);
        }
      }
      if (!ok && issued) {
        umma_commit(bar(L::bDrain));
        mbar_wait_drain(bar(L::bDrain), 0, p.timeout_ns);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int g = (warp >> 2) - 1;  // tiles i with i & 1 == g, TMEM buffer g
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16) + 256 * g;
    const float sl2 = p.scale_log2;
    const int nkeys = kBlockN * n_kv;
    uint8_t* stage = smem + L::kStage + g * L::kBoxBytes;
    bool ok = !*abort_flag;
    for (int i = g; i < cnt && ok; i += 2) {
      const uint32_t ph = (uint32_t)(i >> 1) & 1u;
      // the group's four warps agree on every wait, so that all 128 threads leave the
      // loop together and the named barriers below never wait for a warp that left
      ok = named_bar_and(1 + g, kBlockM, mbar_wait(bar(L::bSF + g), ph, ctl));
      if (!ok) break;
      tc_fence_after();
      // pass 1: exact row max over every valid key
      float mx = -INFINITY;
      for (int c = 0; c < nkeys / 32; ++c) {
        float s[32];
        tmem_ld32(trow + c * 32, s);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (c * 32 + x < p.kv_valid) mx = fmaxf(mx, s[x]);
      }
      const float neg_m = -mx * sl2;
      // pass 2: exponentials, row sum, P packed over the first nkeys/2 columns (each
      // chunk's P lands on columns whose scores were already read)
      float l = 0.0f;
      for (int c = 0; c < nkeys / 32; ++c) {
        float s[32];
        tmem_ld32(trow + c * 32, s);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const int k0 = c * 32 + 2 * x;
          const float p0 = k0 < p.kv_valid ? ex2(fmaf(s[2 * x], sl2, neg_m)) : 0.0f;
          const float p1 = k0 + 1 < p.kv_valid ? ex2(fmaf(s[2 * x + 1], sl2, neg_m)) : 0.0f;
          l += p0 + p1;
          pk[x] = pack_bf16x2(p0, p1);
        }
        tmem_st16(trow + c * 16, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::bPF + g));
      // epilogue: wait for O, free the TMEM buffer, normalise, stage, TMA store
      ok = named_bar_and(1 + g, kBlockM, mbar_wait(bar(L::bOF + g), ph, ctl));
      if (!ok) break;
      tc_fence_after();
      float o[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c)
        tmem_ld32(trow + L::kColO + c * 32, *reinterpret_cast<float(*)[32]>(&o[c * 32]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar(L::bTF + g));  // S/P/O of buffer g may be overwritten now
      // the previous TMA store from this staging buffer must have read it
      if (wq == 0 && lane == 0) tma_store_wait_read0();
      named_bar_sync(1 + g, kBlockM);
      const float inv_l = 1.0f / l;
#pragma unroll
      for (int u = 0; u < 8; ++u) {  // 8 chunks of 16 bytes = 64 bf16
        const uint32_t w0 = pack_bf16x2(o[8 * u + 0] * inv_l, o[8 * u + 1] * inv_l);
        const uint32_t w1 = pack_bf16x2(o[8 * u + 2] * inv_l, o[8 * u + 3] * inv_l);
        const uint32_t w2 = pack_bf16x2(o[8 * u + 4] * inv_l, o[8 * u + 5] * inv_l);
        const uint32_t w3 = pack_bf16x2(o[8 * u + 6] * inv_l, o[8 * u + 7] * inv_l);
        *reinterpret_cast<uint4*>(stage + row * 128 + ((u ^ (row & 7)) << 4)) =
            make_uint4(w0, w1, w2, w3);
      }
      fence_proxy_async_smem();
      named_bar_sync(1 + g, kBlockM);
      if (wq == 0 && lane == 0) {
        const int bh = tile_bh(i);
        tma_store_4d(&tm_o, sbase + L::kStage + g * L::kBoxBytes, 0, bh % p.heads,
                     tile_qt(i) * kBlockM, bh / p.heads);
        tma_store_commit();
      }
    }
    if (wq == 0 && lane == 0) tma_store_wait_read0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace ltx

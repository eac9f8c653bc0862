// attn_fwd_pair.cuh -- attention forward for long query sides at head_dim 128 on sm_100a,
// with the tensor cores of two SMs working as one (a cluster of two CTAs, cta_group::2).
//
// Same operation, layout and mask as attn_fwd.cuh (video self-attention of an LTX-2 block;
// "LTX-2: replicate audio stream across Ulysses ranks by default", Description), direct
// bf16 output.  Each CTA of a pair owns two 128-row query tiles of one (batch, head), as in
// attn_fwd_pp.cuh; the pair's MMAs are M = 256 (the two CTAs' tiles of one slot stacked):
//   S_g = [Q_g(CTA 0); Q_g(CTA 1)] K_j^T      (A from each CTA's shared memory, B = K_j split
//                                              by keys: 64 keys in each CTA)
//   O_g += [P_g(CTA 0); P_g(CTA 1)] V_j       (A = P from each CTA's TMEM, B = V_j split by
//                                              columns: 64 of head_dim in each CTA)
// so each SM loads half of every K/V tile and serves half of every B operand: half the L2 ->
// SM traffic and half the shared-memory operand reads of the one-SM kernel per query row.
//
// Roles, per CTA (384 threads), as in attn_fwd_pp.cuh:
//   warp 0        TMA producer: this CTA's Q slots, then its halves of K_j and V_j; every load
//                 completes on the first CTA's barriers (each CTA arrives with its own bytes).
//   warp 1        MMA issuer, in the first CTA only: the same order as the one-SM kernel
//                 (PV_0(j-1), QK_0(j), PV_1(j-1), QK_1(j)); commits arrive on the barriers of
//                 both CTAs.  In both CTAs warp 1 allocates and frees the pair's TMEM.
//   warps 4-7     softmax of this CTA's rows of slot 0; warps 8-11 of slot 1.  P-ready
//                 arrivals go to the first CTA's barriers (8 warps of the pair each).
// TMEM columns (each CTA, its own 128 rows): S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512).
#pragma once

#include "attn_fwd_pp.cuh"

namespace ltx {

constexpr int kPairThreads = 384;

struct PairSmem {
  static constexpr int D = 128;
  static constexpr int kBoxBytes = kBlockM * 128;       // 128 rows x 64 bf16 (Q, V half)
  static constexpr int kQTileBytes = 2 * kBoxBytes;     // one query tile: 128 rows x 128
  static constexpr int kKHalfBox = 64 * 128;            // 64 keys x 64 dims
  static constexpr int kKHalfBytes = 2 * kKHalfBox;     // 64 keys x 128 dims
  static constexpr int kVHalfBytes = kBoxBytes;         // 128 keys x 64 dims
  static constexpr int kStages = 4;
  static constexpr int kQ = 0;                          // two query tiles
  static constexpr int kK = kQ + 2 * kQTileBytes;
  static constexpr int kV = kK + kStages * kKHalfBytes;
  static constexpr int kBar = kV + kStages * kVHalfBytes;
  // barriers (the *F and PF ones are used in the first CTA only; *E, SF, OF in both)
  static constexpr int bQF = 0;                // 2
  static constexpr int bKF = 2;                // kStages
  static constexpr int bKE = bKF + kStages;
  static constexpr int bVF = bKE + kStages;
  static constexpr int bVE = bVF + kStages;
  static constexpr int bSF = bVE + kStages;    // 2
  static constexpr int bPF = bSF + 2;          // 2 * kPPParts: [part * 2 + g]
  static constexpr int bOF = bPF + 2 * kPPParts;  // 2
  static constexpr int bDrain = bOF + 2;
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kUsed = kAbort + 4;
  static constexpr int kAlloc = ((kUsed + 1024 + 1023) / 1024) * 1024;
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColO = 256;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kAlloc <= 227 * 1024, "shared memory per CTA");
};

// Query tile of slot g of CTA r in pair qb: the pair's four tiles are 4 qb .. 4 qb + 3.
__device__ __forceinline__ int pair_q_tile(int qb, int g, int r) { return 4 * qb + 2 * g + r; }

// Abort path of a producer: its loads complete on the other CTA's barriers, which it cannot
// wait on, so it lets any copy still in flight land (1 ms of global time, far above a copy's
// latency) before the CTA may release its shared memory.
__device__ __forceinline__ void settle_inflight_copies() {
  const unsigned long long t0 = global_timer_ns();
  while (global_timer_ns() - t0 < 1000000ull) __nanosleep(20000);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    ltx_attn_fwd_pair(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using L = PairSmem;
  constexpr int D = L::D;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the pair's MMAs
  const int qb = blockIdx.x >> 1;           // pair index along the query side
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int n = p.n_kv_tiles;  // >= 1
  // the first CTA's copy of barrier i (loads and P-ready arrivals of both CTAs go there)
  auto bar0 = [&](int i) -> uint32_t { return mapa_shared(bar(i), 0); };

  if (threadIdx.x == 0) {
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar(L::bQF + g), 2);  // one arrive.expect_tx per CTA
      mbar_init(bar(L::bSF + g), 1);
      for (int part = 0; part < kPPParts; ++part)
        mbar_init(bar(L::bPF + part * 2 + g), 8);  // four softmax warps of each CTA
      mbar_init(bar(L::bOF + g), 1);
    }
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::bKF + s), 2);
      mbar_init(bar(L::bKE + s), 1);
      mbar_init(bar(L::bVF + s), 2);
      mbar_init(bar(L::bVE + s), 1);
    }
    mbar_init(bar(L::bDrain), 1);
    *abort_flag = (*reinterpret_cast<volatile int*>(p.status) != kDevOk) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(sbase + L::kTmemSlot, L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // both CTAs' barriers are initialised (and their TMEM allocated) before any remote use
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};

  if (warp < 4) {
    reg_dealloc_88();
    if (warp == 0 && lane == 0 && !*abort_flag) {
      // ---------------------------------------------------------- TMA producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      for (int g = 0; g < 2; ++g) {
        mbar_arrive_expect_tx_cluster(bar0(L::bQF + g), L::kQTileBytes);
        for (int bx = 0; bx < 2; ++bx)
          tma_load_4d_pair(sbase + L::kQ + g * L::kQTileBytes + bx * L::kBoxBytes, &tm_q,
                           bar0(L::bQF + g), bx * 64, h, pair_q_tile(qb, g, rank) * kBlockM, b);
      }
      bool ok = true;
      for (int j = 0; j < n && ok; ++j) {
        const int st = j % L::kStages;
        const uint32_t ph = (uint32_t)(j / L::kStages) & 1u;
        const int kv0 = j * kBlockN;
        // this CTA's 64 keys of K_j (all head_dim columns, two 64-column boxes)
        ok = mbar_wait_cluster_lean(bar(L::bKE + st), ph ^ 1u, ctl);
        if (!ok) break;
        mbar_arrive_expect_tx_cluster(bar0(L::bKF + st), L::kKHalfBytes);
        for (int bx = 0; bx < 2; ++bx)
          tma_load_4d_pair(sbase + L::kK + st * L::kKHalfBytes + bx * L::kKHalfBox, &tm_k,
                           bar0(L::bKF + st), bx * 64, h, kv0 + 64 * (int)rank, b);
        // this CTA's 64 head_dim columns of V_j (all 128 keys)
        ok = mbar_wait_cluster_lean(bar(L::bVE + st), ph ^ 1u, ctl);
        if (!ok) break;
        mbar_arrive_expect_tx_cluster(bar0(L::bVF + st), L::kVHalfBytes);
        tma_load_4d_pair(sbase + L::kV + st * L::kVHalfBytes, &tm_v, bar0(L::bVF + st),
                         64 * (int)rank, h, kv0, b);
      }
      if (!ok) settle_inflight_copies();
    } else if (warp == 1 && rank == 0 && !*abort_flag) {
      // ---------------------------------------------------------- MMA issuer (CTA 0)
      auto wt = [&](uint32_t bar_addr, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait_cluster_lean(bar_addr, parity, ctl));
      };
      auto elect = [&]() -> bool {
        uint32_t e;
        asm volatile(
            "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(e));
        return e != 0;
      };
      const bool leader = elect();
      constexpr uint32_t idesc_qk = idesc_bf16_f32(2 * kBlockM, kBlockN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(2 * kBlockM, D, true);
      bool issued = false;
      const SmemDesc dq = SmemDesc::sw128(sbase + L::kQ, 16, 1024);
      const SmemDesc dk = SmemDesc::sw128(sbase + L::kK, 16, 1024);
      const SmemDesc dv = SmemDesc::sw128(sbase + L::kV, L::kBoxBytes, 1024);
      auto qk = [&](int g, int st) {
        const uint32_t q_off = (uint32_t)g * L::kQTileBytes;
        const uint32_t k_off = (uint32_t)st * L::kKHalfBytes;
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ss_pair(tmem + L::kColS + 128 * g,
                         dq.at(q_off + (kk >> 2) * L::kBoxBytes + (kk & 3) * 32),
                         dk.at(k_off + (kk >> 2) * L::kKHalfBox + (kk & 3) * 32), idesc_qk,
                         kk > 0 ? 1u : 0u);
          umma_commit_pair(bar(L::bSF + g), 0x3);
        }
        __syncwarp();
      };
      // O_g (+)= P_g[:, keys kk0*16 .. kk1*16) V[keys, :]
      auto pv_part = [&](int g, int st, bool acc, int kk0, int kk1) {
        const uint32_t v_off = (uint32_t)st * L::kVHalfBytes;
        if (leader) {
#pragma unroll
          for (int kk = kk0; kk < kk1; ++kk)
            umma_ts_pair(tmem + L::kColO + D * g, tmem + L::kColS + 128 * g + kk * 8,
                         dv.at(v_off + kk * 16 * 128), idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
        __syncwarp();
      };
      auto pv = [&](int g, int st, bool acc, uint32_t pph) -> bool {
#pragma unroll
        for (int part = 0; part < kPPParts; ++part) {
          if (!wt(bar(L::bPF + part * 2 + g), pph)) return false;
          tc_fence_after();
          pv_part(g, st, acc, part * (kBlockN / 16 / kPPParts),
                  (part + 1) * (kBlockN / 16 / kPPParts));
        }
        return true;
      };
      auto commit_both = [&](int i) {
        if (leader) umma_commit_pair(bar(i), 0x3);
        __syncwarp();
      };
      bool ok = wt(bar(L::bKF + 0), 0) && wt(bar(L::bQF + 0), 0);
      if (ok) {
        tc_fence_after();
        qk(0, 0);
        issued = true;
        ok = wt(bar(L::bQF + 1), 0);
      }
      if (ok) {
        tc_fence_after();
        qk(1, 0);
        commit_both(L::bKE + 0);
      }
      for (int j = 1; j < n && ok; ++j) {
        const int sk = j % L::kStages;
        const int sv = (j - 1) % L::kStages;
        const uint32_t pph = (uint32_t)(j - 1) & 1u;
        ok = wt(bar(L::bKF + sk), (uint32_t)(j / L::kStages) & 1u) &&
             wt(bar(L::bVF + sv), (uint32_t)((j - 1) / L::kStages) & 1u) &&
             pv(0, sv, j > 1, pph);
        if (!ok) break;
        qk(0, sk);
        ok = pv(1, sv, j > 1, pph);
        if (!ok) break;
        commit_both(L::bVE + sv);
        qk(1, sk);
        commit_both(L::bKE + sk);
      }
      if (ok) {
        const int sv = (n - 1) % L::kStages;
        const uint32_t pph = (uint32_t)(n - 1) & 1u;
        ok = wt(bar(L::bVF + sv), (uint32_t)((n - 1) / L::kStages) & 1u) &&
             pv(0, sv, n > 1, pph);
        if (ok) {
          commit_both(L::bOF + 0);
          ok = pv(1, sv, n > 1, pph);
        }
        if (ok) commit_both(L::bOF + 1);
      }
      if (!ok && issued) {
        // every MMA issued must finish before either CTA releases its TMEM or shared memory
        if (leader) umma_commit_pair(bar(L::bDrain), 0x1);
        __syncwarp();
        mbar_wait_drain(bar(L::bDrain), 0, p.timeout_ns);
      }
    }
  } else {
    reg_alloc_208();
    // ------------------------------------------------------------ softmax g
    const int g = (warp >> 2) - 1;  // 0 for warps 4-7, 1 for warps 8-11
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t colS = L::kColS + 128 * g;
    const uint32_t colO = L::kColO + D * g;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.0f;
    bool ok = !*abort_flag;
    for (int j = 0; j < n && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(L::bSF + g), (uint32_t)j & 1u, ctl));
      if (!ok) break;
      tc_fence_after();
      float s[kBlockN];
#pragma unroll
      for (int c = 0; c < kBlockN / 32; ++c)
        tmem_ld32(trow + colS + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
      tmem_ld_wait();
      const int kv0 = j * kBlockN;
      if (kv0 + kBlockN > p.kv_valid) {  // last key tile only
        const int lim = p.kv_valid - kv0;
#pragma unroll
        for (int c = 0; c < kBlockN; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }
      float mx = row_max<kBlockN>(s) * sl2;
      if (j == 0) {
        m_run = mx;
      } else if (__any_sync(0xffffffffu, mx > m_run + kRescaleThreshold)) {
        // O_g holds PV_g(j-1) (committed with S_g(j)) and PV_g(j) waits for this P: quiescent
        mx = fmaxf(mx, m_run);
        const float f = ex2(m_run - mx);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(trow + colO + c * 32, o);
          tmem_ld_wait();
          uint32_t u[32];
#pragma unroll
          for (int x = 0; x < 32; ++x) u[x] = __float_as_uint(o[x] * f);
          tmem_st32(trow + colO + c * 32, u);
        }
        l_run *= f;
        m_run = mx;
      }
      const float2 nm2 = make_float2(-m_run, -m_run);
      const float2 sc2 = make_float2(sl2, sl2);
      float2 la = make_float2(0.0f, 0.0f), lb = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int part = 0; part < kPPParts; ++part) {
        constexpr int kChunks = kBlockN / 32 / kPPParts;
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          const int ch = part * kChunks + c;
          uint32_t pk[16];
          exp2_pack16(&s[ch * 32], sc2, nm2, la, lb, pk);
          tmem_st16(trow + colS + ch * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        // default (CTA-scope) release: the cluster-scope form cost each half of P several
        // hundred cycles and made this kernel slower than the one-SM kernel
        if (lane == 0) mbar_arrive_remote(bar0(L::bPF + part * 2 + g));
      }
      l_run += (la.x + la.y) + (lb.x + lb.y);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(L::bOF + g), 0, ctl));
    ok = named_bar_and(1 + g, kBlockM, ok && !*abort_flag);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      const int qt = pair_q_tile(qb, g, (int)rank);
      uint8_t* stage = smem + L::kQ + g * L::kQTileBytes;  // this slot's Q tile is done
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(trow + colO + c * 32, o);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) w[x] = pack_bf16x2(o[2 * x] * inv_l, o[2 * x + 1] * inv_l);
        const int bx = c >> 1;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int chunk = (c & 1) * 4 + u;
          uint4* dst = reinterpret_cast<uint4*>(stage + bx * L::kBoxBytes + row * 128 +
                                                ((chunk ^ (row & 7)) << 4));
          *dst = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1 + g, kBlockM);
      if (wq == 0 && lane == 0 && qt < p.n_q_tiles) {
        for (int bx = 0; bx < 2; ++bx)
          tma_store_4d(&tm_o, sbase + L::kQ + g * L::kQTileBytes + bx * L::kBoxBytes, bx * 64, h,
                       qt * kBlockM, b);
        tma_store_commit();
        tma_store_wait_read0();
      }
    }
  }

  // no CTA frees TMEM or leaves (its shared memory is read by the pair's MMAs) before every
  // role of both CTAs is done
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, L::kTmemCols);
  }
}

}  // namespace ltx

// attn_fwd_a2v.cuh -- attention forward for one short key tile (at most 128 keys) at
// head_dim 64 on sm_100a: a2v, video queries over the padded audio keys/values of an LTX-2
// block ("LTX-2: replicate audio stream across Ulysses ranks by default", Description).
// Same operation, layout and key mask as attn_fwd.cuh.
//
// The work per 128-row query tile is small (16 KB of Q in, 16 KB of O out, 16384 exp2 on the
// MUFU at 16 per clock per SM), so throughput comes from keeping many tiles in flight:
//   - persistent: CTA c takes units c, c + G, ... (G = the grid) of the order (batch, query
//     tile, head), head fastest, each unit bringing its own K and V (L2-resident) with its Q;
//   - warp 0 streams Q and K through one ring of stages (freed by QK) and V through another
//     (freed by PV); warp 1 issues QK up to kLookahead units ahead of PV;
//   - three warpgroups take every third unit each and do all of its row work: softmax (the row
//     in two 64-key halves, the first half's max as the stabiliser unless the second half's
//     exceeds it by more than 2^64), then, once PV has landed, the epilogue (O / l with l kept
//     in registers, bf16, this warpgroup's staging tile, TMA store).  While one warpgroup waits
//     for its PV the other two keep the MUFU busy.
// TMEM (512 columns): four buffers of 128 columns, unit i in buffer i % 4: S over all 128
// columns, P (bf16 pairs) over the first 64 once the scores it replaces were read, O (64 fp32)
// in the last 64 columns, over scores already read.
// Registers (setmaxnreg): issue warpgroup 56, each row warpgroup 152.
#pragma once

#include "attn_fwd_skv.cuh"

namespace ltx {

constexpr int kA2vThreads = 512;
constexpr int kA2vRegsIssue = 56;
constexpr int kA2vRegsWork = 152;
static_assert(128 * kA2vRegsIssue + 384 * kA2vRegsWork <= kA2vThreads * 128,
              "register split exceeds the launch allocation");

struct A2vSmem {
  static constexpr int D = 64;
  static constexpr int kTileBytes = kBlockM * 128;  // 128 rows x 64 bf16
  static constexpr int kQKStages = 3;               // Q and K of a unit
  static constexpr int kVStages = 3;
  static constexpr int kWG = 3;                     // row warpgroups
  static constexpr int kNB = 4;                     // TMEM buffers of 128 columns
  static constexpr int kLookahead = 2;              // QK ahead of PV, in units
  static constexpr uint32_t kColP = 0;
  static constexpr uint32_t kColO = 64;
  static constexpr int kQ = 0;                      // stage s: Q at kQ + 2 s tiles, K after it
  static constexpr int kK = kTileBytes;
  static constexpr int kV = kQKStages * 2 * kTileBytes;
  static constexpr int kStage = kV + kVStages * kTileBytes;  // one staging tile per warpgroup
  static constexpr int kBar = kStage + kWG * kTileBytes;
  static constexpr int bQF = 0;
  static constexpr int bQE = bQF + kQKStages;
  static constexpr int bVF = bQE + kQKStages;
  static constexpr int bVE = bVF + kVStages;
  static constexpr int bSF = bVE + kVStages;   // kNB
  static constexpr int bPF = bSF + kNB;        // kNB (4 warp arrivals)
  static constexpr int bOF = bPF + kNB;        // kNB
  static constexpr int bTF = bOF + kNB;        // kNB (4 warp arrivals): buffer free
  static constexpr int bDrain = bTF + kNB;
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kUsed = kAbort + 4;
  static constexpr int kAlloc = ((kUsed + 1024 + 1023) / 1024) * 1024;
  static_assert(kAlloc <= 227 * 1024, "shared memory per CTA");
  static_assert(kLookahead < kNB && kLookahead < kQKStages, "pipeline depth");
};

__global__ void __launch_bounds__(kA2vThreads, 1)
    ltx_attn_fwd_a2v(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using L = A2vSmem;
  constexpr int NB = L::kNB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long total = (long long)p.batch * p.heads * p.n_q_tiles;
  const int cnt = (int)((total - blockIdx.x + gridDim.x - 1) / gridDim.x);
  auto unit_of = [&](int i) -> long long { return (long long)blockIdx.x + (long long)i * gridDim.x; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kQKStages; ++s) {
      mbar_init(bar(L::bQF + s), 1);
      mbar_init(bar(L::bQE + s), 1);
    }
    for (int s = 0; s < L::kVStages; ++s) {
      mbar_init(bar(L::bVF + s), 1);
      mbar_init(bar(L::bVE + s), 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(bar(L::bSF + b), 1);
      mbar_init(bar(L::bPF + b), 4);
      mbar_init(bar(L::bOF + b), 1);
      mbar_init(bar(L::bTF + b), 4);
    }
    mbar_init(bar(L::bDrain), 1);
    *abort_flag = (*reinterpret_cast<volatile int*>(p.status) != kDevOk) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + L::kTmemSlot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    setmaxnreg_dec<kA2vRegsIssue>();
    if (lane == 0 && !*abort_flag && cnt > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int last_q[L::kQKStages], last_v[L::kVStages];
      for (int s = 0; s < L::kQKStages; ++s) last_q[s] = -1;
      for (int s = 0; s < L::kVStages; ++s) last_v[s] = -1;
      bool ok = true;
      for (int i = 0; i < cnt && ok; ++i) {
        SkvUnit u;
        u.init(unit_of(i), p);
        const int qs = i % L::kQKStages;
        ok = mbar_wait_lean(bar(L::bQE + qs), ((uint32_t)(i / L::kQKStages) & 1u) ^ 1u, ctl);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(L::bQF + qs), 2 * L::kTileBytes);
        tma_load_4d(sbase + L::kQ + qs * 2 * L::kTileBytes, &tm_q, bar(L::bQF + qs), 0, u.h,
                    u.qt * kBlockM, u.b);
        tma_load_4d(sbase + L::kK + qs * 2 * L::kTileBytes, &tm_k, bar(L::bQF + qs), 0, u.h, 0,
                    u.b);
        last_q[qs] = i;
        const int vs = i % L::kVStages;
        ok = mbar_wait_lean(bar(L::bVE + vs), ((uint32_t)(i / L::kVStages) & 1u) ^ 1u, ctl);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(L::bVF + vs), L::kTileBytes);
        tma_load_4d(sbase + L::kV + vs * L::kTileBytes, &tm_v, bar(L::bVF + vs), 0, u.h, 0, u.b);
        last_v[vs] = i;
      }
      if (!ok) {
        for (int s = 0; s < L::kQKStages; ++s)
          if (last_q[s] >= 0)
            mbar_wait_drain(bar(L::bQF + s), (uint32_t)(last_q[s] / L::kQKStages) & 1u,
                            p.timeout_ns);
        for (int s = 0; s < L::kVStages; ++s)
          if (last_v[s] >= 0)
            mbar_wait_drain(bar(L::bVF + s), (uint32_t)(last_v[s] / L::kVStages) & 1u,
                            p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    setmaxnreg_dec<kA2vRegsIssue>();
    if (!*abort_flag && cnt > 0) {
      auto wt = [&](uint32_t bar_addr, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait_lean(bar_addr, parity, ctl));
      };
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, L::D, true);
      const SmemDesc dq = SmemDesc::sw128(sbase + L::kQ, 16, 1024);
      const SmemDesc dk = SmemDesc::sw128(sbase + L::kK, 16, 1024);
      const SmemDesc dv = SmemDesc::sw128(sbase + L::kV, L::kTileBytes, 1024);
      bool issued = false;
      // S = Q_i K_i^T into buffer i % NB, once its previous unit's epilogue has read O
      auto qk = [&](int i) -> bool {
        const int bf = i % NB;
        const int qs = i % L::kQKStages;
        if (!wt(bar(L::bQF + qs), (uint32_t)(i / L::kQKStages) & 1u) ||
            !wt(bar(L::bTF + bf), ((uint32_t)(i / NB) & 1u) ^ 1u))
          return false;
        tc_fence_after();
        const uint32_t off = (uint32_t)qs * 2 * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < L::D / 16; ++kk)
          umma_ss_elect(tmem + 128 * bf, dq.at(off + kk * 32), dk.at(off + kk * 32), idesc_qk,
                        kk > 0 ? 1u : 0u);
        issued = true;
        umma_commit_elect(bar(L::bSF + bf));
        umma_commit_elect(bar(L::bQE + qs));
        return true;
      };
      // O = P_i V_i into buffer i % NB
      auto pv = [&](int i) -> bool {
        const int bf = i % NB;
        const int vs = i % L::kVStages;
        if (!wt(bar(L::bPF + bf), (uint32_t)(i / NB) & 1u) ||
            !wt(bar(L::bVF + vs), (uint32_t)(i / L::kVStages) & 1u))
          return false;
        tc_fence_after();
        const uint32_t buf = tmem + 128 * bf;
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk)
          umma_ts_elect(buf + L::kColO, buf + L::kColP + kk * 8,
                        dv.at((uint32_t)vs * L::kTileBytes + kk * 16 * 128), idesc_pv,
                        kk > 0 ? 1u : 0u);
        umma_commit_elect(bar(L::bOF + bf));
        umma_commit_elect(bar(L::bVE + vs));
        return true;
      };
      int nq = 0;
      bool ok = true;
      for (int i = 0; i < cnt && ok; ++i) {
        while (ok && nq < cnt && nq <= i + L::kLookahead) ok = qk(nq++);
        if (ok) ok = pv(i);
      }
      if (!ok && issued) {
        umma_commit_elect(bar(L::bDrain));
        mbar_wait_drain(bar(L::bDrain), 0, p.timeout_ns);
      }
    }
  } else if (warp < 4) {
    setmaxnreg_dec<kA2vRegsIssue>();  // warps 2-3: idle
  } else {
    // ------------------------------------------------------------ row warpgroups
    setmaxnreg_inc<kA2vRegsWork>();
    const int w = (warp >> 2) - 1;  // units i with i % 3 == w
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t tlane = tmem + ((uint32_t)(wq * 32) << 16);
    const float sl2 = p.scale_log2;
    const float2 sc2 = make_float2(sl2, sl2);
    const bool leader = wq == 0 && lane == 0;
    uint8_t* stage = smem + L::kStage + w * L::kTileBytes;
    const uint32_t stage_addr = sbase + L::kStage + w * L::kTileBytes;
    bool ok = !*abort_flag;
    for (int i = w; i < cnt && ok; i += L::kWG) {
      const int bf = i % NB;
      const uint32_t ph = (uint32_t)(i / NB) & 1u;
      const uint32_t trow = tlane + 128 * bf;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bSF + bf), ph, ctl));
      if (!ok) break;
      tc_fence_after();
      // ---- softmax, the row in two 64-key halves
      float s[64];
      float2 la = make_float2(0.0f, 0.0f), lb = make_float2(0.0f, 0.0f);
      tmem_ld32(trow, *reinterpret_cast<float(*)[32]>(&s[0]));
      tmem_ld32(trow + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
      tmem_ld_wait();
      mask_keys<2>(s, p.kv_valid);
      float m = row_max<64>(s);
      float2 nm2 = make_float2(-m * sl2, -m * sl2);
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // P of keys 0..63 over the scores of keys 0..31
        uint32_t pk[16];
        exp2_pack16(&s[c * 32], sc2, nm2, la, lb, pk);
        tmem_st16(trow + L::kColP + c * 16, pk);
      }
      tmem_ld32(trow + 64, *reinterpret_cast<float(*)[32]>(&s[0]));
      tmem_ld32(trow + 96, *reinterpret_cast<float(*)[32]>(&s[32]));
      tmem_ld_wait();
      mask_keys<2>(s, p.kv_valid - 64);
      const float mb = row_max<64>(s);
      if (__any_sync(0xffffffffu, (mb - m) * sl2 > 64.0f)) {
        // rare: the second half outgrows the first half's max by more than 2^64; raise the
        // stabiliser to the larger max and rescale the P already stored and its sums (lanes
        // whose max did not move scale by 1; tcgen05.ld/st are warp-collective)
        const float mn = fmaxf(m, mb);
        const float f = ex2((m - mn) * sl2);
        m = mn;
        nm2 = make_float2(-m * sl2, -m * sl2);
        la = make_float2(la.x * f, la.y * f);
        lb = make_float2(lb.x * f, lb.y * f);
        tmem_st_wait();
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t u[16];
          tmem_ld16(trow + L::kColP + c * 16, u);
          tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 16; ++x)
            u[x] = pack_bf16x2(__uint_as_float(u[x] << 16) * f,
                               __uint_as_float(u[x] & 0xffff0000u) * f);
          tmem_st16(trow + L::kColP + c * 16, u);
        }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // P of keys 64..127 over the scores of keys 32..63
        uint32_t pk[16];
        exp2_pack16(&s[c * 32], sc2, nm2, la, lb, pk);
        tmem_st16(trow + L::kColP + 32 + c * 16, pk);
      }
      const float l = (la.x + la.y) + (lb.x + lb.y);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::bPF + bf));
      // ---- epilogue, once PV has landed in this buffer
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bOF + bf), ph, ctl));
      ok = named_bar_and(1 + w, kBlockM, ok);  // the four warps leave together or not at all
      if (!ok) break;
      tc_fence_after();
      float o[64];
      tmem_ld32(trow + L::kColO, *reinterpret_cast<float(*)[32]>(&o[0]));
      tmem_ld32(trow + L::kColO + 32, *reinterpret_cast<float(*)[32]>(&o[32]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::bTF + bf));  // the buffer may take QK of unit i + 4
      // this warpgroup's previous store has read its staging tile
      if (leader) tma_store_wait_read<0>();
      named_bar_sync(1 + w, kBlockM);
      const float il = 1.0f / l;
      const float2 il2 = make_float2(il, il);
#pragma unroll
      for (int u = 0; u < 8; ++u) {  // 8 chunks of 16 bytes = 64 bf16
        uint32_t w4[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float2 v2 = __fmul2_rn(make_float2(o[8 * u + 2 * x], o[8 * u + 2 * x + 1]), il2);
          w4[x] = pack_bf16x2(v2.x, v2.y);
        }
        *reinterpret_cast<uint4*>(stage + row * 128 + ((u ^ (row & 7)) << 4)) =
            make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      fence_proxy_async_smem();
      named_bar_sync(1 + w, kBlockM);
      if (leader) {
        SkvUnit un;
        un.init(unit_of(i), p);
        tma_store_4d(&tm_o, stage_addr, 0, un.h, un.qt * kBlockM, un.b);
        tma_store_commit();
      }
    }
    if (leader) tma_store_wait_read<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace ltx

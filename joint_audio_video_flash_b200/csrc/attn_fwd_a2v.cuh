// attn_fwd_a2v.cuh -- attention forward for one short key tile (at most 128 keys) at
// head_dim 64 on sm_100a: a2v, video queries over the padded audio keys/values of an LTX-2
// block ("LTX-2: replicate audio stream across Ulysses ranks by default", Description).
// Same operation, layout and key mask as attn_fwd.cuh.
//
// The work per 128-row query tile is small (16 KB of Q in, 16 KB of O out, 16384 exp2 on the
// MUFU at 16 per clock per SM), so throughput comes from keeping many tiles in flight:
//   - persistent: CTA c takes units c, c + G, ... (G = the grid) of the order (batch, query
//     tile, head), head fastest: the G tiles loaded at once are every head of a few token
//     blocks, i.e. whole contiguous token rows of q and out, and each unit brings its own K
//     and V (a few KB, L2-resident) with its Q;
//   - warp 0 streams Q and K through one ring of stages (freed by QK) and V through another
//     (freed by PV); warp 1 issues QK up to kLookahead units ahead of PV;
//   - warps 4-11: two softmax warpgroups take alternate units (the whole 128-score row in
//     registers, so the max is exact and there is no rescale) and never wait for PV;
//   - warps 12-15: the epilogue warpgroup takes every unit in order: waits for O, divides by
//     l, rounds to bf16, stages the tile and issues its TMA store.
// TMEM (512 columns): four buffers of 128 columns, unit i in buffer i % 4: S over all 128
// columns, P (bf16 pairs) over the first 64 once the scores it replaces were read, O (64 fp32)
// in the last 64 columns, over scores already read.
// Registers (setmaxnreg): issue warpgroup 56, softmax 176, epilogue 104.
// One launch may take several such calls (A2vArgs): audio self-attention (one query tile per
// (batch, head)) then shares the launch of a2v.
#pragma once

#include <type_traits>

#include "attn_fwd_skv.cuh"

namespace ltx {

constexpr int kA2vThreads = 512;
constexpr int kA2vRegsIssue = 56;     // warps 0-3
constexpr int kA2vRegsSoftmax = 176;  // warps 4-11
constexpr int kA2vRegsEpi = 104;      // warps 12-15
static_assert(128 * kA2vRegsIssue + 256 * kA2vRegsSoftmax + 128 * kA2vRegsEpi <=
                  kA2vThreads * 128,
              "register split exceeds the launch allocation");

struct A2vSmem {
  static constexpr int D = 64;
  static constexpr int kTileBytes = kBlockM * 128;  // 128 rows x 64 bf16
  static constexpr int kQKStages = 4;               // Q and K of a unit
  static constexpr int kVStages = 4;
  static constexpr int kNB = 4;                     // TMEM buffers of 128 columns
  static constexpr int kLookahead = 2;              // QK ahead of PV, in units
  static constexpr uint32_t kColO = 64;             // O after P (64 columns of bf16 pairs)
  static constexpr int kQ = 0;                      // stage s: Q at kQ + 2 s tiles, K after it
  static constexpr int kK = kTileBytes;
  static constexpr int kV = kQKStages * 2 * kTileBytes;
  static constexpr int kStage = kV + kVStages * kTileBytes;  // output staging tile
  static constexpr int kRowSum = kStage + kTileBytes;        // l per buffer and row
  static constexpr int kBar = kRowSum + kNB * kBlockM * 4;
  static constexpr int bQF = 0;
  static constexpr int bQE = bQF + kQKStages;
  static constexpr int bVF = bQE + kQKStages;
  static constexpr int bVE = bVF + kVStages;
  static constexpr int bSF = bVE + kVStages;   // kNB
  static constexpr int bPF = bSF + kNB;        // kNB (4 softmax warp arrivals)
  static constexpr int bOF = bPF + kNB;        // kNB
  static constexpr int bTF = bOF + kNB;        // kNB (4 epilogue warp arrivals): buffer free
  static constexpr int bDrain = bTF + kNB;
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kUsed = kAbort + 4;
  static constexpr int kAlloc = ((kUsed + 1024 + 1023) / 1024) * 1024;
  static_assert(kAlloc <= 227 * 1024, "shared memory per CTA");
  static_assert(kLookahead < kNB && kLookahead < kQKStages, "pipeline depth");
};

// One attention call the kernel takes: head_dim 64, every valid key in one 128-key tile.
struct A2vProblem {
  int batch, heads, n_q_tiles;
  int kv_valid;
  float scale_log2;
  long long first_unit;  // units of the problems before this one
};
static_assert(sizeof(A2vProblem) == 32, "problem table entry (shared-memory layout)");

// Up to kA2vMaxProblems calls in one persistent launch (a group): their (batch, query tile,
// head) units are numbered one problem after another and walked as one sequence, so a small
// call (audio self-attention, 64 units) rides along with a large one (a2v) instead of paying
// a launch of its own.
constexpr int kA2vMaxProblems = 4;
struct A2vArgs {
  CUtensorMap q[kA2vMaxProblems], k[kA2vMaxProblems], v[kA2vMaxProblems], o[kA2vMaxProblems];
  A2vProblem prob[kA2vMaxProblems];
  int n_problems;
  long long total_units;
  int* status;
  unsigned long long timeout_ns;
};

// Calls f(std::integral_constant<int, P>) for every problem P < n in order: each role walks
// its units problem by problem with P known at compile time, so that every tensor map and
// every per-problem value is read at a constant offset of the parameter block (a runtime
// index into it made the kernel markedly slower).
template <class F>
__device__ __forceinline__ void a2v_for_each_problem(int n, F&& f) {
  static_assert(kA2vMaxProblems == 4, "one call per problem");
  f(std::integral_constant<int, 0>{});
  if (n > 1) f(std::integral_constant<int, 1>{});
  if (n > 2) f(std::integral_constant<int, 2>{});
  if (n > 3) f(std::integral_constant<int, 3>{});
}

// Number of this CTA's units (blockIdx.x + i * gridDim.x) below unit `u`.
__device__ __forceinline__ int a2v_units_below(long long u) {
  const long long d = u - (long long)blockIdx.x;
  return d > 0 ? (int)((d + gridDim.x - 1) / gridDim.x) : 0;
}

// Batch, head and query tile of unit u of problem pr (units ordered (batch, query tile, head),
// head fastest).
struct A2vUnit {
  int b, h, qt;
  __device__ __forceinline__ void init(long long u, const A2vProblem& pr) {
    u -= pr.first_unit;
    const long long t = u / pr.heads;
    h = (int)(u - t * pr.heads);
    b = (int)(t / pr.n_q_tiles);
    qt = (int)(t - (long long)b * pr.n_q_tiles);
  }
};

__global__ void __launch_bounds__(kA2vThreads, 1)
    ltx_attn_fwd_a2v(const __grid_constant__ A2vArgs a) {
  using L = A2vSmem;
  constexpr int NB = L::kNB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  float* row_sum = reinterpret_cast<float*>(smem + L::kRowSum);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_problems = a.n_problems;
  // this CTA's units: blockIdx.x + i * gridDim.x, i < cnt; those of problem P are
  // i in [first_i(P), first_i(P + 1))
  const int cnt = a2v_units_below(a.total_units);
  auto unit_of = [&](int i) -> long long { return (long long)blockIdx.x + (long long)i * gridDim.x; };
  auto first_i = [&](auto P) -> int { return a2v_units_below(a.prob[decltype(P)::value].first_unit); };
  auto end_i = [&](auto P) -> int {
    constexpr int p = decltype(P)::value;
    if constexpr (p + 1 < kA2vMaxProblems) {
      if (p + 1 < n_problems) return a2v_units_below(a.prob[p + 1].first_unit);
    }
    return cnt;
  };

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
    *abort_flag = (*reinterpret_cast<volatile int*>(a.status) != kDevOk) ? 1 : 0;
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
  const WaitCtl ctl{abort_flag, a.status, a.timeout_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    setmaxnreg_dec<kA2vRegsIssue>();
    if (lane == 0 && !*abort_flag && cnt > 0) {
      int last_q[L::kQKStages], last_v[L::kVStages];
      for (int s = 0; s < L::kQKStages; ++s) last_q[s] = -1;
      for (int s = 0; s < L::kVStages; ++s) last_v[s] = -1;
      bool ok = true;
      a2v_for_each_problem(n_problems, [&](auto P) {
        constexpr int p = decltype(P)::value;
        const A2vProblem& pr = a.prob[p];
        tma_prefetch_desc(&a.q[p]);
        tma_prefetch_desc(&a.k[p]);
        tma_prefetch_desc(&a.v[p]);
        const int i1 = end_i(P);
        for (int i = first_i(P); i < i1 && ok; ++i) {
          A2vUnit u;
          u.init(unit_of(i), pr);
          const int qs = i % L::kQKStages;
          ok = mbar_wait_lean(bar(L::bQE + qs), ((uint32_t)(i / L::kQKStages) & 1u) ^ 1u, ctl);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(L::bQF + qs), 2 * L::kTileBytes);
          tma_load_4d(sbase + L::kQ + qs * 2 * L::kTileBytes, &a.q[p], bar(L::bQF + qs), 0, u.h,
                      u.qt * kBlockM, u.b);
          tma_load_4d(sbase + L::kK + qs * 2 * L::kTileBytes, &a.k[p], bar(L::bQF + qs), 0, u.h,
                      0, u.b);
          last_q[qs] = i;
          const int vs = i % L::kVStages;
          ok = mbar_wait_lean(bar(L::bVE + vs), ((uint32_t)(i / L::kVStages) & 1u) ^ 1u, ctl);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(L::bVF + vs), L::kTileBytes);
          tma_load_4d(sbase + L::kV + vs * L::kTileBytes, &a.v[p], bar(L::bVF + vs), 0, u.h, 0,
                      u.b);
          last_v[vs] = i;
        }
      });
      if (!ok) {  // the copies already issued land before the CTA releases its memory
        for (int s = 0; s < L::kQKStages; ++s)
          if (last_q[s] >= 0)
            mbar_wait_drain(bar(L::bQF + s), (uint32_t)(last_q[s] / L::kQKStages) & 1u,
                            a.timeout_ns);
        for (int s = 0; s < L::kVStages; ++s)
          if (last_v[s] >= 0)
            mbar_wait_drain(bar(L::bVF + s), (uint32_t)(last_v[s] / L::kVStages) & 1u,
                            a.timeout_ns);
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
          umma_ts_elect(buf + L::kColO, buf + kk * 8,
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
        mbar_wait_drain(bar(L::bDrain), 0, a.timeout_ns);
      }
    }
  } else if (warp < 4) {
    setmaxnreg_dec<kA2vRegsIssue>();  // warps 2-3: idle
  } else if (warp < 12) {
    // ------------------------------------------------------------ softmax
    setmaxnreg_inc<kA2vRegsSoftmax>();
    const int g = (warp >> 2) - 1;  // units i with i & 1 == g
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t tlane = tmem + ((uint32_t)(wq * 32) << 16);
    bool ok = !*abort_flag;
    a2v_for_each_problem(n_problems, [&](auto P) {
      constexpr int p = decltype(P)::value;
      const int kv_valid = a.prob[p].kv_valid;
      const float sl2 = a.prob[p].scale_log2;
      const float2 sc2 = make_float2(sl2, sl2);
      const int i0 = first_i(P), i1 = end_i(P);
      for (int i = i0 + ((i0 & 1) != g ? 1 : 0); i < i1 && ok; i += 2) {
        const int bf = i % NB;
        const uint32_t trow = tlane + 128 * bf;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bSF + bf), (uint32_t)(i / NB) & 1u, ctl));
        if (!ok) break;
        tc_fence_after();
        // the whole 128-score row in registers: exact max, exponentials, P (bf16 pairs) over
        // the first 64 columns, the row sum in two packed fp32 accumulators
        float s[kBlockN];
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c)
          tmem_ld32(trow + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
        tmem_ld_wait();
        mask_keys<kBlockN / 32>(s, kv_valid);
        const float mx = row_max<kBlockN>(s);
        const float2 nm2 = make_float2(-mx * sl2, -mx * sl2);
        float2 la = make_float2(0.0f, 0.0f), lb = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) {
          uint32_t pk[16];
          exp2_pack16(&s[c * 32], sc2, nm2, la, lb, pk);
          tmem_st16(trow + c * 16, pk);
        }
        row_sum[bf * kBlockM + row] = (la.x + la.y) + (lb.x + lb.y);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::bPF + bf));  // P in TMEM and l in shared memory
      }
    });
  } else {
    // ------------------------------------------------------------ epilogue
    setmaxnreg_dec<kA2vRegsEpi>();
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t tlane = tmem + ((uint32_t)(wq * 32) << 16);
    const bool leader = wq == 0 && lane == 0;
    uint8_t* stage = smem + L::kStage;
    bool ok = !*abort_flag;
    a2v_for_each_problem(n_problems, [&](auto P) {
      constexpr int p = decltype(P)::value;
      const A2vProblem& pr = a.prob[p];
      const int i1 = end_i(P);
      for (int i = first_i(P); i < i1 && ok; ++i) {
        const int bf = i % NB;
        const uint32_t ph = (uint32_t)(i / NB) & 1u;
        // P_i (and with it l) published, then O_i = P_i V landed; the four warps agree so
        // that all 128 threads leave the loop together (named barriers follow)
        bool w = mbar_wait(bar(L::bPF + bf), ph, ctl);
        w = w && mbar_wait(bar(L::bOF + bf), ph, ctl);
        ok = named_bar_and(1, kBlockM, w);
        if (!ok) break;
        tc_fence_after();
        const uint32_t trow = tlane + 128 * bf;
        const float inv_l = 1.0f / row_sum[bf * kBlockM + row];
        float o[64];
        tmem_ld32(trow + L::kColO, *reinterpret_cast<float(*)[32]>(&o[0]));
        tmem_ld32(trow + L::kColO + 32, *reinterpret_cast<float(*)[32]>(&o[32]));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::bTF + bf));  // S/P/O and l of this buffer are free
        // the previous store has read the staging tile
        if (leader) tma_store_wait_read<0>();
        named_bar_sync(1, kBlockM);
        const float2 il2 = make_float2(inv_l, inv_l);
#pragma unroll
        for (int u = 0; u < 8; ++u) {  // 8 chunks of 16 bytes = 64 bf16
          uint32_t w4[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const float2 v2 =
                __fmul2_rn(make_float2(o[8 * u + 2 * x], o[8 * u + 2 * x + 1]), il2);
            w4[x] = pack_bf16x2(v2.x, v2.y);
          }
          *reinterpret_cast<uint4*>(stage + row * 128 + ((u ^ (row & 7)) << 4)) =
              make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async_smem();
        named_bar_sync(1, kBlockM);
        if (leader) {
          A2vUnit un;
          un.init(unit_of(i), pr);
          tma_store_4d(&a.o[p], sbase + L::kStage, 0, un.h, un.qt * kBlockM, un.b);
          tma_store_commit();
        }
      }
    });
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

// attn_fwd_pp.cuh -- attention forward for long query sides on sm_100a: one CTA owns
// TWO 128-row query tiles of the same (batch, head) that share every K/V tile, and
// two softmax warpgroups ping-pong so the tensor core always has one tile's MMAs to
// run while the other tile's softmax is computed.
//
// Same operation, layout, mask and split mode as attn_fwd.cuh (video self-attention,
// a2v and the long-key parts of v2a of an LTX-2 block; "LTX-2: replicate audio
// stream across Ulysses ranks by default", Description).
//
// Roles (384 threads):
//   warp 0        TMA producer: Q0, Q1 once, then K_j, V_j into stage rings.
//   warp 1        MMA issuer, per key tile j:  O0 += P0(j-1) V(j-1); S0 = Q0 K_j^T;
//                 O1 += P1(j-1) V(j-1); S1 = Q1 K_j^T.  Because tcgen05 MMAs from one
//                 thread run in issue order, the commit that publishes S_g(j) also
//                 guarantees PV_g(j-1) has landed in O_g, so softmax g may rescale O_g
//                 without any further wait.
//   warps 2-3     idle (complete the first warpgroup for the register split).
//   warps 4-7     softmax of query tile 0 (one row per thread, TMEM lane = row).
//   warps 8-11    softmax of query tile 1.
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
// Registers: the first warpgroup gives its registers back (setmaxnreg) so each
// softmax thread can hold a full 128-score row.
#pragma once

#include "attn_fwd.cuh"

namespace ltx {

constexpr int kPPThreads = 384;
constexpr int kPPRegsLaunch = 168;   // 65536 / 384, rounded down to a multiple of 8
constexpr int kPPRegsProducer = 88;  // warps 0-3 after setmaxnreg.dec
constexpr int kPPRegsSoftmax = 208;  // warps 4-11 after setmaxnreg.inc
static_assert(128 * kPPRegsProducer + 256 * kPPRegsSoftmax <= kPPThreads * kPPRegsLaunch,
              "register split exceeds the launch allocation");
// P of each tile is published to the MMA warp in this many key parts (2 or 4), so that
// the PV of the first parts overlaps the exponentials of the later ones
constexpr int kPPParts = 2;
static_assert(kPPParts == 2 || kPPParts == 4, "P parts");

template <int D>
struct PPSmem {
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = kBlockM * 128;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kStages = (D == 64) ? 4 : 2;
  static constexpr int kQ = 0;  // two query tiles
  static constexpr int kK = kQ + 2 * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBar = kV + kStages * kTileBytes;
  static constexpr int bQF = 0;  // 2
  static constexpr int bKF = 2;
  static constexpr int bKE = bKF + kStages;
  static constexpr int bVF = bKE + kStages;
  static constexpr int bVE = bVF + kStages;
  static constexpr int bSF = bVE + kStages;  // 2
  static constexpr int bPF = bSF + 2;        // 2 * kPPParts: [part * 2 + g]
  static constexpr int bOF = bPF + 2 * kPPParts;  // 2
  static constexpr int bDrain = bOF + 2;
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kUsed = kAbort + 4;
  static constexpr int kAlloc = ((kUsed + 1024 + 1023) / 1024) * 1024 > kMinSmemFor1Cta
                                    ? ((kUsed + 1024 + 1023) / 1024) * 1024
                                    : kMinSmemFor1Cta;
  static constexpr uint32_t kColS = 0;      // + 128 * g
  static constexpr uint32_t kColO = 256;    // + D * g
  static constexpr uint32_t kTmemCols = 512;
};

__device__ __forceinline__ void reg_dealloc_88() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 88;\n" ::: "memory");
}
__device__ __forceinline__ void reg_alloc_208() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 208;\n" ::: "memory");
}

template <int D, bool kSplit>
__global__ void __launch_bounds__(kPPThreads, 1)
    ltx_attn_fwd_pp(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using L = PPSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qb = blockIdx.x;  // 256-row query block: tiles 2*qb and 2*qb+1
  const int h = blockIdx.y;
  const int b = kSplit ? (int)blockIdx.z / p.num_splits : (int)blockIdx.z;
  const int split = kSplit ? (int)blockIdx.z % p.num_splits : 0;
  const int kv_begin = split * p.tiles_per_split;
  const int kv_end = min(kv_begin + p.tiles_per_split, p.n_kv_tiles);
  const int n = kv_end - kv_begin;  // >= 1

  if (threadIdx.x == 0) {
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar(L::bQF + g), 1);
      mbar_init(bar(L::bSF + g), 1);
      for (int part = 0; part < kPPParts; ++part)  // P keys of one part of tile g
        mbar_init(bar(L::bPF + part * 2 + g), 4);  // one arrival per softmax warp
      mbar_init(bar(L::bOF + g), 1);
    }
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::bKF + s), 1);
      mbar_init(bar(L::bKE + s), 1);
      mbar_init(bar(L::bVF + s), 1);
      mbar_init(bar(L::bVE + s), 1);
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

  if (warp < 4) {
    reg_dealloc_88();
    if (warp == 0 && lane == 0 && !*abort_flag) {
      // ---------------------------------------------------------- TMA producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      for (int g = 0; g < 2; ++g) {
        mbar_arrive_expect_tx(bar(L::bQF + g), L::kTileBytes);
        for (int bx = 0; bx < L::kBoxes; ++bx)
          tma_load_4d(sbase + L::kQ + g * L::kTileBytes + bx * L::kBoxBytes, &tm_q,
                      bar(L::bQF + g), bx * 64, h, (2 * qb + g) * kBlockM, b);
      }
      int last_k[L::kStages], last_v[L::kStages];
      for (int s = 0; s < L::kStages; ++s) last_k[s] = last_v[s] = -1;
      bool ok = true;
      for (int j = 0; j < n && ok; ++j) {
        const int st = j % L::kStages;
        const uint32_t ph = (uint32_t)(j / L::kStages) & 1u;
        const int kv0 = (kv_begin + j) * kBlockN;
        ok = mbar_wait_lean(bar(L::bKE + st), ph ^ 1u, ctl);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(L::bKF + st), L::kTileBytes);
        for (int bx = 0; bx < L::kBoxes; ++bx)
          tma_load_4d(sbase + L::kK + st * L::kTileBytes + bx * L::kBoxBytes, &tm_k,
                      bar(L::bKF + st), bx * 64, h, kv0, b);
        last_k[st] = j;
        ok = mbar_wait_lean(bar(L::bVE + st), ph ^ 1u, ctl);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(L::bVF + st), L::kTileBytes);
        for (int bx = 0; bx < L::kBoxes; ++bx)
          tma_load_4d(sbase + L::kV + st * L::kTileBytes + bx * L::kBoxBytes, &tm_v,
                      bar(L::bVF + st), bx * 64, h, kv0, b);
        last_v[st] = j;
      }
      if (!ok) {
        for (int s = 0; s < L::kStages; ++s) {
          if (last_k[s] >= 0)
            mbar_wait_drain(bar(L::bKF + s), (uint32_t)(last_k[s] / L::kStages) & 1u,
                            p.timeout_ns);
          if (last_v[s] >= 0)
            mbar_wait_drain(bar(L::bVF + s), (uint32_t)(last_v[s] / L::kStages) & 1u,
                            p.timeout_ns);
        }
        mbar_wait_drain(bar(L::bQF + 0), 0, p.timeout_ns);
        mbar_wait_drain(bar(L::bQF + 1), 0, p.timeout_ns);
      }
    } else if (warp == 1 && !*abort_flag) {
      // ---------------------------------------------------------- MMA issuer
      // The whole warp runs this loop (control values stay warp-uniform); one elected
      // lane issues each MMA and commit, and the lanes agree on every wait.
      auto wt = [&](uint32_t bar_addr, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait_lean(bar_addr, parity, ctl));
      };
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, D, true);
      bool issued = false;
      // shared-memory descriptors built once; each MMA moves them by an offset
      const SmemDesc dq = SmemDesc::sw128(sbase + L::kQ, 16, 1024);
      const SmemDesc dk = SmemDesc::sw128(sbase + L::kK, 16, 1024);
      const SmemDesc dv = SmemDesc::sw128(sbase + L::kV, L::kBoxBytes, 1024);
      auto qk = [&](int g, int st) {
        const uint32_t q_off = (uint32_t)g * L::kTileBytes;
        const uint32_t k_off = (uint32_t)st * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
          umma_ss_elect(tmem + L::kColS + 128 * g, dq.at(q_off + off), dk.at(k_off + off), idesc_qk,
                  kk > 0 ? 1u : 0u);
        }
        umma_commit_elect(bar(L::bSF + g));
      };
      // O_g (+)= P_g[:, keys kk0*16 .. kk1*16) V[keys, :]
      auto pv_part = [&](int g, int st, bool acc, int kk0, int kk1) {
        const uint32_t v_off = (uint32_t)st * L::kTileBytes;
#pragma unroll
        for (int kk = kk0; kk < kk1; ++kk)
          umma_ts_elect(tmem + L::kColO + D * g, tmem + L::kColS + 128 * g + kk * 8,
                  dv.at(v_off + kk * 16 * 128), idesc_pv, (acc || kk > 0) ? 1u : 0u);
      };
      // waits for P_g (both halves) and issues its PV; false on a failed wait
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
        umma_commit_elect(bar(L::bKE + 0));
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
        umma_commit_elect(bar(L::bVE + sv));
        qk(1, sk);
        umma_commit_elect(bar(L::bKE + sk));
      }
      if (ok) {
        const int sv = (n - 1) % L::kStages;
        const uint32_t pph = (uint32_t)(n - 1) & 1u;
        ok = wt(bar(L::bVF + sv), (uint32_t)((n - 1) / L::kStages) & 1u) &&
             pv(0, sv, n > 1, pph);
        if (ok) {
          umma_commit_elect(bar(L::bOF + 0));
          ok = pv(1, sv, n > 1, pph);
        }
        if (ok) umma_commit_elect(bar(L::bOF + 1));
      }
      if (!ok && issued) {
        umma_commit_elect(bar(L::bDrain));
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
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bSF + g), (uint32_t)j & 1u, ctl));
      if (!ok) break;
      tc_fence_after();
      float s[kBlockN];
#pragma unroll
      for (int c = 0; c < kBlockN / 32; ++c)
        tmem_ld32(trow + colS + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
      tmem_ld_wait();
      const int kv0 = (kv_begin + j) * kBlockN;
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
        // O_g already holds PV_g(j-1) (it was issued before S_g(j) and committed with it),
        // and PV_g(j) waits for this warpgroup's P, so O_g is quiescent here.
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
      // exponentials on the MUFU (argument and row sum in packed fp32 pairs); P is
      // published to the MMA warp in kPPParts key parts so the PV of the first parts
      // overlaps the exponentials of the later ones
      float2 la = make_float2(0.0f, 0.0f), lb = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int part = 0; part < kPPParts; ++part) {
        constexpr int kChunks = kBlockN / 32 / kPPParts;  // 32-key chunks per part
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
        if (lane == 0) mbar_arrive(bar(L::bPF + part * 2 + g));
      }
      l_run += (la.x + la.y) + (lb.x + lb.y);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bOF + g), 0, ctl));
    ok = named_bar_and(1 + g, kBlockM, ok && !*abort_flag);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      const int qt = 2 * qb + g;
      if constexpr (!kSplit) {
        uint8_t* stage = smem + L::kQ + g * L::kTileBytes;
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
          for (int bx = 0; bx < L::kBoxes; ++bx)
            tma_store_4d(&tm_o, sbase + L::kQ + g * L::kTileBytes + bx * L::kBoxBytes, bx * 64,
                         h, qt * kBlockM, b);
          tma_store_commit();
          tma_store_wait_read0();
        }
      } else {
        const int rows_pad = p.n_q_tiles * kBlockM;
        const int grow = qt * kBlockM + row;
        const bool live = grow < p.q_len;
        const size_t prow =
            (((size_t)split * p.batch + b) * p.heads + h) * (size_t)rows_pad + (size_t)grow;
        float4* dst = reinterpret_cast<float4*>(p.o_part + (live ? prow : 0) * D);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          __syncwarp();
          tmem_ld32(trow + colO + c * 32, o);
          tmem_ld_wait();
          if (live) {
#pragma unroll
            for (int x = 0; x < 8; ++x)
              dst[c * 8 + x] = make_float4(o[4 * x] * inv_l, o[4 * x + 1] * inv_l,
                                           o[4 * x + 2] * inv_l, o[4 * x + 3] * inv_l);
          }
        }
        if (live) p.lse_part[prow] = m_run + __log2f(l_run);
      }
    }
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

// attn_fwd_skv.cuh -- attention forward for a short key side (at most 256 keys) on
// sm_100a: the streams' queries over a padded text context at head_dim 64 or 128, and a2v
// (video queries over the padded audio keys/values of an LTX-2 block, "LTX-2: replicate
// audio stream across Ulysses ranks by default", Description) when the audio side has more
// than 128 valid keys.  (With at most 128 valid keys at head_dim 64, a2v runs on
// attn_fwd_a2v.cuh.)  Same operation, layout and key mask as attn_fwd.cuh.  With every key
// in one S tile the softmax max is exact, so there is no online rescale.  The work is bound
// by HBM (reading Q, writing O) and by the exponentials, so the design keeps both busy at
// once:
//
//   - persistent: one CTA per SM walks a contiguous run of query tiles (flattened
//     over batch, head, tile); K and V of the current (batch, head) stay resident in
//     shared memory and are reloaded only when the run crosses into the next head;
//   - warp 0 streams Q tiles through a deep TMA ring;
//   - warp 1 issues S = Q K^T two tiles ahead of O = P V, so a softmax warpgroup
//     finds its next scores computed when it finishes a tile;
//   - warps 4-11: two softmax warpgroups take alternate tiles (S -> P and the row
//     sum l); they never wait for the PV product;
//   - warps 12-15: the epilogue warpgroup takes every tile in order: waits for O,
//     divides by l, rounds to bf16, stages the tile and issues its TMA store.
// TMEM (512 columns) holds NB buffers (4 / NKV at head_dim 64, 2 at 128); tile i uses
// buffer i % NB.  In a buffer: S over the first 128*NKV columns, P packed as bf16 pairs
// over the first 64*NKV columns (written after the scores it replaces were read), O (D
// fp32 columns) right after P, over scores already read.  K and V are stored box-major
// ([64-column box][key tile]), so that QK over two key tiles (N = 256) and PV over 256
// keys see one contiguous row range per box.
// Registers (setmaxnreg): producer/MMA warpgroup 56, epilogue 104, softmax 176.
#pragma once

#include "attn_fwd.cuh"

namespace ltx {

constexpr int kSkvThreads = 512;
constexpr int kSkvMaxKvTiles = 2;
constexpr int kSkvRegsLaunch = 128;  // 65536 / 512
constexpr int kSkvRegsIssue = 56;    // warps 0-3
constexpr int kSkvRegsEpi = 104;     // warps 12-15
constexpr int kSkvRegsSoftmax = 176; // warps 4-11
static_assert(128 * kSkvRegsIssue + 128 * kSkvRegsEpi + 256 * kSkvRegsSoftmax <=
                  kSkvThreads * kSkvRegsLaunch,
              "register split exceeds the launch allocation");

// K/V of the current (batch, head) stay resident (reloaded when the CTA's contiguous run
// of units crosses into the next head); Q streams through a ring.
template <int D, int NKV>
struct SkvSmem {
  static_assert(NKV == 1 || NKV == 2, "one or two 128-key tiles");
  static_assert(D == 64 || D == 128, "head_dim");
  static constexpr int kBoxes = D / 64;            // 64-column (128-byte) boxes per row
  static constexpr int kBoxBytes = kBlockM * 128;  // 128 rows x 64 bf16
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kQStages = D == 64 ? (NKV == 1 ? 8 : 6) : (NKV == 1 ? 3 : 2);
  static constexpr int kStaging = D == 64 ? 2 : 1;     // output staging tiles
  static constexpr uint32_t kBufCols = D == 64 ? 128u * NKV : 256u;  // columns per buffer
  static constexpr int kNB = (int)(512u / kBufCols);    // TMEM buffers
  // QK runs this many tiles ahead of PV; QK(i + kLookahead) reuses the buffer of tile
  // i + kLookahead - kNB, whose epilogue needs PV(i + kLookahead - kNB) issued earlier
  static constexpr int kLookahead = kNB - 1 < 2 ? kNB - 1 : 2;
  static constexpr uint32_t kColO = 64u * NKV;          // O within a buffer (after P)
  static_assert(kColO + D <= kBufCols, "O fits its buffer");
  // K [box][key tile], V, then the Q ring
  static constexpr int kK = 0;
  static constexpr int kV = NKV * kTileBytes;
  static constexpr int kQ = 2 * NKV * kTileBytes;
  static constexpr int kStage = kQ + kQStages * kTileBytes;  // output staging
  static constexpr int kRowSum = kStage + kStaging * kTileBytes;  // l per buffer and row
  static constexpr int kBar = kRowSum + kNB * kBlockM * 4;
  static constexpr int bKVF = 0;
  static constexpr int bKVE = 1;
  static constexpr int bQF = 2;                 // kQStages
  static constexpr int bQE = bQF + kQStages;    // kQStages
  static constexpr int bSF = bQE + kQStages;    // kNB
  static constexpr int bPF = bSF + kNB;         // kNB
  static constexpr int bOF = bPF + kNB;         // kNB
  static constexpr int bTF = bOF + kNB;         // kNB: TMEM buffer free
  static constexpr int bDrain = bTF + kNB;
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kUsed = kAbort + 4;
  static constexpr int kAlloc = ((kUsed + 1024 + 1023) / 1024) * 1024 > kMinSmemFor1Cta
                                    ? ((kUsed + 1024 + 1023) / 1024) * 1024
                                    : kMinSmemFor1Cta;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kAlloc <= 227 * 1024, "shared memory per CTA");
  static_assert(kLookahead >= 1 && kLookahead <= kNB - 1 && kLookahead < kQStages,
                "pipeline depth");
};

// (batch, head, query tile) of consecutive flattened tile indices, advanced without
// division.
struct SkvCursor {
  int b, h, qt;
  __device__ __forceinline__ void init(long long t, const FwdParams& p) {
    const long long bh = t / p.n_q_tiles;
    qt = (int)(t - bh * p.n_q_tiles);
    b = (int)(bh / p.heads);
    h = (int)(bh - (long long)b * p.heads);
  }
  // true when the next tile starts another (batch, head)
  __device__ __forceinline__ bool advance(const FwdParams& p) {
    if (++qt < p.n_q_tiles) return false;
    qt = 0;
    if (++h == p.heads) {
      h = 0;
      ++b;
    }
    return true;
  }
};

template <int D, int NKV>
__global__ void __launch_bounds__(kSkvThreads, 1)
    ltx_attn_fwd_skv(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using L = SkvSmem<D, NKV>;
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
  // a contiguous run of flattened (batch, head, query tile) indices for this CTA
  const long long total = (long long)p.batch * p.heads * p.n_q_tiles;
  const long long t_begin = total * blockIdx.x / gridDim.x;
  const long long t_end = total * (blockIdx.x + 1) / gridDim.x;
  const int cnt = (int)(t_end - t_begin);

  if (threadIdx.x == 0) {
    mbar_init(bar(L::bKVF), 1);
    mbar_init(bar(L::bKVE), 1);
    for (int s = 0; s < L::kQStages; ++s) {
      mbar_init(bar(L::bQF + s), 1);
      mbar_init(bar(L::bQE + s), 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(bar(L::bSF + b), 1);
      mbar_init(bar(L::bPF + b), 4);  // one arrival per softmax warp
      mbar_init(bar(L::bOF + b), 1);
      mbar_init(bar(L::bTF + b), 4);  // one arrival per epilogue warp
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

  // The register split (setmaxnreg) sits inside each role's branch, so that ptxas
  // compiles every role under the limit it runs with.
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    setmaxnreg_dec<kSkvRegsIssue>();
    if (lane == 0 && !*abort_flag && cnt > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      SkvCursor cur;
      cur.init(t_begin, p);
      int kv_loads = 0;
      bool new_head = true;
      int last_q[L::kQStages];
      for (int s = 0; s < L::kQStages; ++s) last_q[s] = -1;
      bool ok = true;
      for (int i = 0; i < cnt && ok; ++i) {
        if (new_head) {
          if (kv_loads > 0) ok = mbar_wait_lean(bar(L::bKVE), (uint32_t)(kv_loads - 1) & 1u, ctl);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(L::bKVF), 2 * NKV * L::kTileBytes);
#pragma unroll
          for (int bx = 0; bx < L::kBoxes; ++bx)
#pragma unroll
            for (int t = 0; t < NKV; ++t) {
              const uint32_t off = (uint32_t)(bx * NKV + t) * L::kBoxBytes;
              tma_load_4d(sbase + L::kK + off, &tm_k, bar(L::bKVF), bx * 64, cur.h,
                          t * kBlockN, cur.b);
              tma_load_4d(sbase + L::kV + off, &tm_v, bar(L::bKVF), bx * 64, cur.h,
                          t * kBlockN, cur.b);
            }
          ++kv_loads;
        }
        const int qs = i % L::kQStages;
        ok = mbar_wait_lean(bar(L::bQE + qs), ((uint32_t)(i / L::kQStages) & 1u) ^ 1u, ctl);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(L::bQF + qs), L::kTileBytes);
#pragma unroll
        for (int bx = 0; bx < L::kBoxes; ++bx)
          tma_load_4d(sbase + L::kQ + qs * L::kTileBytes + bx * L::kBoxBytes, &tm_q,
                      bar(L::bQF + qs), bx * 64, cur.h, cur.qt * kBlockM, cur.b);
        last_q[qs] = i;
        new_head = cur.advance(p);
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
    setmaxnreg_dec<kSkvRegsIssue>();
    // The whole warp runs this loop (control values stay warp-uniform); one elected
    // lane issues each MMA and commit, and the lanes agree on every wait.
    if (!*abort_flag && cnt > 0) {
      auto wt = [&](uint32_t bar_addr, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait_lean(bar_addr, parity, ctl));
      };
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN * NKV, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, D, true);
      // shared-memory descriptors built once; each MMA moves them by a constant offset
      const SmemDesc dq = SmemDesc::sw128(sbase + L::kQ, 16, 1024);
      const SmemDesc dk = SmemDesc::sw128(sbase + L::kK, 16, 1024);
      // V is MN-major: its leading byte offset steps from one 64-column box to the next
      const SmemDesc dv = SmemDesc::sw128(sbase + L::kV, NKV * L::kBoxBytes, 1024);
      bool issued = false;
      int kv_ver = 0;       // K/V loads consumed so far
      // S = Q_i K^T into buffer i % NB (waits for Q_i and the buffer; `fresh_kv` also
      // waits for the K/V of a new (batch, head))
      auto qk = [&](int i, bool fresh_kv) -> bool {
        if (fresh_kv) {
          if (!wt(bar(L::bKVF), (uint32_t)kv_ver & 1u)) return false;
          ++kv_ver;
        }
        const int bf = i % NB;
        const int qs = i % L::kQStages;
        if (!wt(bar(L::bQF + qs), (uint32_t)(i / L::kQStages) & 1u) ||
            !wt(bar(L::bTF + bf), ((uint32_t)(i / NB) & 1u) ^ 1u))
          return false;
        tc_fence_after();
        const uint32_t q_off = (uint32_t)qs * L::kTileBytes;
        const uint32_t k_off = 0u;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // 16 head-dim columns: box kk / 4, 32-byte step kk % 4 within the box
          const uint32_t in_box = (kk & 3) * 32;
          umma_ss_elect(tmem + L::kBufCols * bf, dq.at(q_off + (kk >> 2) * L::kBoxBytes + in_box),
                        dk.at(k_off + (kk >> 2) * NKV * L::kBoxBytes + in_box), idesc_qk,
                        kk > 0 ? 1u : 0u);
        }
        issued = true;
        umma_commit_elect(bar(L::bSF + bf));
        umma_commit_elect(bar(L::bQE + qs));
        return true;
      };
      // O = P_i V into buffer i % NB (waits for P_i)
      auto pv = [&](int i) -> bool {
        const int bf = i % NB;
        if (!wt(bar(L::bPF + bf), (uint32_t)(i / NB) & 1u)) return false;
        tc_fence_after();
        const uint32_t buf = tmem + L::kBufCols * bf;
        const uint32_t v_off = 0u;
#pragma unroll
        for (int kk = 0; kk < (kBlockN / 16) * NKV; ++kk)
          umma_ts_elect(buf + L::kColO, buf + kk * 8, dv.at(v_off + kk * 16 * 128), idesc_pv,
                        kk > 0 ? 1u : 0u);
        umma_commit_elect(bar(L::bOF + bf));
        return true;
      };
      // QK runs up to kLookahead tiles ahead of PV but never into the next (batch, head)
      // before every PV of the current one is issued: the K/V buffers are shared.
      SkvCursor cq;  // tile nq
      cq.init(t_begin, p);
      int nq = 0;
      bool q_fresh = true;    // tile nq starts a (batch, head)
      bool ok = true;
      for (int i = 0; i < cnt && ok; ++i) {
        while (ok && nq < cnt && nq <= i + L::kLookahead && (!q_fresh || nq == i)) {
          if (q_fresh && nq > 0) umma_commit_elect(bar(L::bKVE));  // old K/V may be overwritten
          ok = qk(nq, q_fresh);
          ++nq;
          q_fresh = cq.advance(p);
        }
        if (ok) ok = pv(i);
      }
      if (!ok && issued) {
        umma_commit_elect(bar(L::bDrain));
        mbar_wait_drain(bar(L::bDrain), 0, p.timeout_ns);
      }
    }
  } else if (warp < 4) {
    setmaxnreg_dec<kSkvRegsIssue>();  // warps 2-3: idle
  } else if (warp < 12) {
    // ------------------------------------------------------------ softmax
    setmaxnreg_inc<kSkvRegsSoftmax>();
    const int g = (warp >> 2) - 1;  // tiles i with i & 1 == g
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t tlane = tmem + ((uint32_t)(wq * 32) << 16);
    const float sl2 = p.scale_log2;
    bool ok = !*abort_flag;
    for (int i = g; i < cnt && ok; i += 2) {
      const int bf = i % NB;
      const uint32_t trow = tlane + L::kBufCols * bf;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bSF + bf), (uint32_t)(i / NB) & 1u, ctl));
      if (!ok) break;
      tc_fence_after();
      // row sum in two packed accumulators (fp32 pairs)
      float2 la = make_float2(0.0f, 0.0f), lb = make_float2(0.0f, 0.0f);
      const float2 sc2 = make_float2(sl2, sl2);
      if constexpr (NKV == 1) {
        // the whole 128-score row in registers: exact max, exponentials, P over the
        // first 64 columns
        float s[kBlockN];
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c)
          tmem_ld32(trow + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
        tmem_ld_wait();
        mask_keys<kBlockN / 32>(s, p.kv_valid);
        const float mx = row_max<kBlockN>(s);
        const float2 nm2 = make_float2(-mx * sl2, -mx * sl2);
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) {
          uint32_t pk[16];
          exp2_pack16(&s[c * 32], sc2, nm2, la, lb, pk);
          tmem_st16(trow + c * 16, pk);
        }
      } else {
        // Two key tiles.  The softmax needs a stabiliser close to the row max, not the
        // max itself: the first tile's max m_a stabilises its exponentials at once; the
        // second tile reuses m_a unless its max exceeds m_a by more than 2^6 (then its
        // probabilities could overflow bf16's useful range), in which case this warp
        // redoes the row with the exact max over both tiles.
        float s[kBlockN];
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c)
          tmem_ld32(trow + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
        tmem_ld_wait();
        mask_keys<kBlockN / 32>(s, p.kv_valid);
        float m = row_max<kBlockN>(s);
        float2 nm2 = make_float2(-m * sl2, -m * sl2);
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) {
          uint32_t pk[16];
          exp2_pack16(&s[c * 32], sc2, nm2, la, lb, pk);
          tmem_st16(trow + c * 16, pk);
        }
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c)
          tmem_ld32(trow + kBlockN + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
        tmem_ld_wait();
        mask_keys<kBlockN / 32>(s, p.kv_valid - kBlockN);
        const float mb = row_max<kBlockN>(s);
        if (__any_sync(0xffffffffu, (mb - m) * sl2 > 64.0f)) {
          // rare (a row whose second tile outgrows the first by more than 2^64): raise
          // the stabiliser to the larger max; the first tile's P, already in TMEM, and its
          // partial sums scale by f = 2^((m - m_new) * scale_log2) <= 1 (f = 1 on the
          // lanes whose max did not move; tcgen05.ld/st are warp-collective)
          const float mn = fmaxf(m, mb);
          const float f = ex2((m - mn) * sl2);
          m = mn;
          nm2 = make_float2(-m * sl2, -m * sl2);
          la = make_float2(la.x * f, la.y * f);
          lb = make_float2(lb.x * f, lb.y * f);
          tmem_st_wait();
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {  // 64 columns of packed bf16 pairs, 16 at a time
            uint32_t u[16];
            tmem_ld16(trow + c * 16, u);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 16; ++x)
              u[x] = pack_bf16x2(__uint_as_float(u[x] << 16) * f,
                                 __uint_as_float(u[x] & 0xffff0000u) * f);
            tmem_st16(trow + c * 16, u);
          }
        }
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) {
          uint32_t pk[16];
          exp2_pack16(&s[c * 32], sc2, nm2, la, lb, pk);
          tmem_st16(trow + 64 + c * 16, pk);
        }
      }
      row_sum[bf * kBlockM + row] = (la.x + la.y) + (lb.x + lb.y);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::bPF + bf));  // P in TMEM and l in shared memory
    }
  } else {
    // ------------------------------------------------------------ epilogue
    setmaxnreg_dec<kSkvRegsEpi>();
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t tlane = tmem + ((uint32_t)(wq * 32) << 16);
    const bool leader = wq == 0 && lane == 0;
    SkvCursor cur;
    cur.init(t_begin, p);
    bool ok = !*abort_flag;
    for (int i = 0; i < cnt && ok; ++i) {
      const int bf = i % NB;
      const uint32_t ph = (uint32_t)(i / NB) & 1u;
      // P_i (and with it l) published, then O_i = P_i V landed; the four warps agree
      // so that all 128 threads leave the loop together (named barriers follow)
      bool w = mbar_wait(bar(L::bPF + bf), ph, ctl);
      w = w && mbar_wait(bar(L::bOF + bf), ph, ctl);
      ok = named_bar_and(1, kBlockM, w);
      if (!ok) break;
      tc_fence_after();
      const uint32_t trow = tlane + L::kBufCols * bf;
      const float inv_l = 1.0f / row_sum[bf * kBlockM + row];
      // the store issued kStaging tiles ago from this staging buffer must have read it
      const int sb = L::kStaging == 2 ? (i & 1) : 0;
      uint8_t* stage = smem + L::kStage + sb * L::kTileBytes;
      if (leader) tma_store_wait_read<L::kStaging - 1>();
      named_bar_sync(1, kBlockM);
      const float2 il2 = make_float2(inv_l, inv_l);
#pragma unroll
      for (int bx = 0; bx < L::kBoxes; ++bx) {  // 64 output columns per box
        float o[64];
        tmem_ld32(trow + L::kColO + bx * 64, *reinterpret_cast<float(*)[32]>(&o[0]));
        tmem_ld32(trow + L::kColO + bx * 64 + 32, *reinterpret_cast<float(*)[32]>(&o[32]));
        tmem_ld_wait();
        if (bx == L::kBoxes - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(L::bTF + bf));  // S/P/O and l of this buffer are free
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {  // 8 chunks of 16 bytes = 64 bf16
          uint32_t w[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const float2 v2 = __fmul2_rn(make_float2(o[8 * u + 2 * x], o[8 * u + 2 * x + 1]), il2);
            w[x] = pack_bf16x2(v2.x, v2.y);
          }
          *reinterpret_cast<uint4*>(stage + bx * L::kBoxBytes + row * 128 +
                                    ((u ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1, kBlockM);
      if (leader) {
#pragma unroll
        for (int bx = 0; bx < L::kBoxes; ++bx)
          tma_store_4d(&tm_o, sbase + L::kStage + sb * L::kTileBytes + bx * L::kBoxBytes,
                       bx * 64, cur.h, cur.qt * kBlockM, cur.b);
        tma_store_commit();
      }
      cur.advance(p);
    }
    if (leader) tma_store_wait_read<0>();
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

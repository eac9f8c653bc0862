// attn_fwd.cuh -- flash-style softmax attention forward for sm_100a.
//
// Computes O = softmax(scale * Q K^T + M) V per (batch, head) for the four
// attentions of an LTX-2 joint audio-video DiT block (video self, audio self,
// v2a = audio queries over video keys/values, a2v = video queries over audio
// keys/values; "LTX-2: replicate audio stream across Ulysses ranks by default",
// Description).  M is -inf on keys >= kv_valid (the zero-padded audio tail, same
// Description) and 0 elsewhere.  Tensors are bf16 BSHD: element (b, s, h, d) at
// ((b*len + s)*heads + h)*D + d.
//
// One CTA owns one 128-row query tile of one (batch, head) and streams 128-key
// tiles of K and V through shared memory:
//   warp 0      TMA producer: Q once, then K_j and V_j into 2-stage rings.
//   warp 1      MMA issuer: S_j = Q K_j^T (SS, bf16 -> fp32 in TMEM, S double
//               buffered) and O += P_j V_j (A = P read from TMEM, B = V from smem).
//   warps 2-5   softmax: one query row per thread (TMEM lane = row); row max with a
//               lazy rescale of O (only when the running max grows by > 2^8), exp2
//               on the MUFU, fp32 row sums, P written back over S as packed bf16;
//               then the epilogue.
// TMEM columns: S buffer 0 at [0,128), S buffer 1 at [128,256), O at [256,256+D).
//
// In split mode (short query side, long key side: v2a) the CTA covers one range
// of key tiles and writes its normalised fp32 partial output and its base-2
// log-sum-exp; combine.cuh merges the parts through those statistics (the merge of
// per-rank softmax statistics in "feat(ltx2): tile-parallel video VAE and the
// two-stage pipeline", commit "Onboard Lightricks LTX-2.5").
#pragma once

#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace ltx {

constexpr int kBlockM = 128;  // query rows per tile (= TMEM lanes)
constexpr int kBlockN = 128;  // keys per tile
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when max grows > 2^8
constexpr int kMinSmemFor1Cta = 120 * 1024;  // forces one CTA per SM (TMEM holds 512 columns)

struct FwdParams {
  int q_len;
  int kv_len;
  int kv_valid;
  int heads;
  int batch;
  int n_q_tiles;        // ceil(q_len / 128)
  int n_kv_tiles;       // ceil(kv_valid / 128)
  int num_splits;       // key-range parts (1 = direct bf16 output)
  int tiles_per_split;  // key tiles per part
  float scale_log2;     // scale * log2(e)
  float* o_part;        // split: [splits][batch][heads][n_q_tiles*128][D] fp32
  float* lse_part;      // split: [splits][batch][heads][n_q_tiles*128] base-2 LSE
  int* status;          // device status word
  unsigned long long timeout_ns;
};

// kSBuf = 2: S double buffered (QK of tile j+1 overlaps the softmax of tile j), 512
// TMEM columns, one CTA per SM, 192 threads (producer, MMA, four softmax warps).
// kSBuf = 1: one S buffer, 256 TMEM columns, 256 threads (producer, MMA and two idle
// warps in the first warpgroup, which hands registers to the softmax warpgroup), three K
// and two V stages, so that two CTAs share an SM and interleave their
// QK -> softmax -> PV chains (head_dim 64 only: shared memory and registers fit twice).
// P has its own 64 columns there (S [0,128), P [128,192), O [192,256)), so QK of the next
// key tile is issued as soon as the softmax has read S into registers and runs during the
// exponentials; the softmax computes P(j) in registers and stores it once PV(j-1) has read
// P(j-1).
template <int D, int kSBuf = 2>
struct FwdSmem {
  static_assert(kSBuf == 2 || (kSBuf == 1 && D == 64), "S buffers");
  static constexpr int kThreads = kSBuf == 1 ? 256 : 192;
  static constexpr int kSoftmaxWarp0 = kSBuf == 1 ? 4 : 2;  // first softmax warp
  // kSBuf == 1: 2 CTAs x 256 threads x 128 registers at launch; setmaxnreg moves the first
  // warpgroup to 56 and the softmax warpgroup to 200 (56 + 200 = 2 x 128)
  static constexpr int kBoxes = D / 64;             // 128-byte (64 x bf16) column boxes per row
  static constexpr int kBoxBytes = kBlockM * 128;   // one 128-row x 64-column box
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kKStages = kSBuf == 1 ? 3 : (D == 64) ? 3 : 2;
  static constexpr int kVStages = kSBuf == 1 ? 2 : (D == 64) ? 3 : 2;
  // the producer issues K this many tiles ahead of V (K is needed a softmax earlier)
  static constexpr int kKAhead = kKStages - kVStages;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kKStages * kTileBytes;
  static constexpr int kBar = kV + kVStages * kTileBytes;
  // barriers
  static constexpr int bQ = 0;
  static constexpr int bKF = 1;
  static constexpr int bKE = bKF + kKStages;
  static constexpr int bVF = bKE + kKStages;
  static constexpr int bVE = bVF + kVStages;
  static constexpr int bSF = bVE + kVStages;  // kSBuf
  static constexpr int bPF = bSF + 2;        // kSBuf
  static constexpr int bSE = bPF + 2;        // kSBuf == 1: S read into registers (4 warps)
  static constexpr int bOD = bSE + 1;        // O updated by a PV
  static constexpr int bOF = bOD + 1;        // final PV done
  static constexpr int bDrain = bOF + 1;     // abort-path drain
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kUsed = kAbort + 4;
  static constexpr int kRaw = ((kUsed + 1024 + 1023) / 1024) * 1024;
  static constexpr int kAlloc =
      kSBuf == 1 ? kRaw : (kRaw > kMinSmemFor1Cta ? kRaw : kMinSmemFor1Cta);
  static constexpr int kColP = 128;                    // kSBuf == 1: P's own columns
  static constexpr int kColO = kSBuf == 1 ? 192 : 256;
  static constexpr uint32_t kTmemCols = kSBuf == 1 ? 256 : 512;
  static_assert(kSBuf == 2 || 2 * kAlloc <= 227 * 1024, "two CTAs per SM");
};

// ---------------------------------------------------------------------------
// softmax row helpers (one query row per thread, scores in registers)
// ---------------------------------------------------------------------------
// Sets scores of keys >= `valid` to -inf in NC 32-column chunks (key 0 = s[0]).  Only
// the chunk holding the boundary pays per-element selects; the branches are uniform.
template <int NC>
__device__ __forceinline__ void mask_keys(float* s, int valid) {
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    if (valid <= c * 32) {
#pragma unroll
      for (int x = 0; x < 32; ++x) s[c * 32 + x] = -INFINITY;
    } else if (valid < c * 32 + 32) {
#pragma unroll
      for (int x = 0; x < 32; ++x)
        if (c * 32 + x >= valid) s[c * 32 + x] = -INFINITY;
    }
  }
}

// Maximum of N scores: four chains of three-input max.
template <int N>
__device__ __forceinline__ float row_max(const float* s) {
  static_assert(N % 8 == 0 && N >= 16, "row length");
  float m[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
  for (int c = 4; c + 8 <= N - 4; c += 8)
#pragma unroll
    for (int x = 0; x < 4; ++x) m[x] = fmax3(m[x], s[c + x], s[c + 4 + x]);
  // s[0 .. 4) seeded the chains and the loop consumed s[4 .. N-4); the last four remain
#pragma unroll
  for (int x = 0; x < 4; ++x) m[x] = fmaxf(m[x], s[N - 4 + x]);
  return fmax3(fmaxf(m[0], m[1]), m[2], m[3]);
}

// 32 scores -> p = 2^(s*scale_log2 - m) as 16 packed bf16 pairs; the fp32 p are added
// to the two packed row-sum accumulators.  Argument and sums use packed fp32 pairs.
__device__ __forceinline__ void exp2_pack16(const float* s, float2 sc2, float2 nm2, float2& la,
                                            float2& lb, uint32_t (&pk)[16]) {
#pragma unroll
  for (int x = 0; x < 16; ++x) {
    const float2 a = __ffma2_rn(make_float2(s[2 * x], s[2 * x + 1]), sc2, nm2);
    const float2 e = make_float2(ex2(a.x), ex2(a.y));
    if (x & 1)
      lb = __fadd2_rn(lb, e);
    else
      la = __fadd2_rn(la, e);
    pk[x] = pack_bf16x2(e.x, e.y);
  }
}

// Bounded wait that ignores the abort flag (used to drain copies / MMAs on the
// abort path before the CTA releases shared and tensor memory).
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity,
                                                unsigned long long timeout_ns) {
  const unsigned long long t0 = global_timer_ns();
  const unsigned long long max_polls = timeout_ns / 4 + 1024;
  unsigned long long polls = 0;
  while (!mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) {
    if (global_timer_ns() - t0 > timeout_ns || ++polls > max_polls) return false;
  }
  return true;
}

template <int D, bool kSplit, int kSBuf = 2>
__global__ void __launch_bounds__(FwdSmem<D, kSBuf>::kThreads, 3 - kSBuf)
    ltx_attn_fwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const FwdParams p) {
  using L = FwdSmem<D, kSBuf>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = blockIdx.x;
  const int h = blockIdx.y;
  const int b = kSplit ? (int)blockIdx.z / p.num_splits : (int)blockIdx.z;
  const int split = kSplit ? (int)blockIdx.z % p.num_splits : 0;
  const int kv_begin = split * p.tiles_per_split;
  const int kv_end = min(kv_begin + p.tiles_per_split, p.n_kv_tiles);
  const int n = kv_end - kv_begin;  // >= 1 by construction on the host

  if (threadIdx.x == 0) {
    mbar_init(bar(L::bQ), 1);
    for (int s = 0; s < L::kKStages; ++s) {
      mbar_init(bar(L::bKF + s), 1);
      mbar_init(bar(L::bKE + s), 1);
    }
    for (int s = 0; s < L::kVStages; ++s) {
      mbar_init(bar(L::bVF + s), 1);
      mbar_init(bar(L::bVE + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::bSF + s), 1);
      mbar_init(bar(L::bPF + s), 4);  // one arrival per softmax warp
    }
    mbar_init(bar(L::bSE), 4);
    mbar_init(bar(L::bOD), 1);
    mbar_init(bar(L::bOF), 1);
    mbar_init(bar(L::bDrain), 1);
    // a CTA that starts after another one failed does no work
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
    if constexpr (kSBuf == 1) setmaxnreg_dec<56>();
    if (lane == 0 && !*abort_flag) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bar(L::bQ), L::kTileBytes);
      for (int bx = 0; bx < L::kBoxes; ++bx)
        tma_load_4d(sbase + L::kQ + bx * L::kBoxBytes, &tm_q, bar(L::bQ), bx * 64, h,
                    qt * kBlockM, b);
      int last_k[L::kKStages], last_v[L::kVStages];
      for (int s = 0; s < L::kKStages; ++s) last_k[s] = -1;
      for (int s = 0; s < L::kVStages; ++s) last_v[s] = -1;
      bool ok = true;
      int nk = 0;  // next K tile to load (K runs kKAhead tiles ahead of V)
      for (int j = 0; j < n && ok; ++j) {
        for (; ok && nk < n && nk <= j + L::kKAhead; ++nk) {
          const int st = nk % L::kKStages;
          ok = mbar_wait(bar(L::bKE + st), ((uint32_t)(nk / L::kKStages) & 1u) ^ 1u, ctl);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(L::bKF + st), L::kTileBytes);
          for (int bx = 0; bx < L::kBoxes; ++bx)
            tma_load_4d(sbase + L::kK + st * L::kTileBytes + bx * L::kBoxBytes, &tm_k,
                        bar(L::bKF + st), bx * 64, h, (kv_begin + nk) * kBlockN, b);
          last_k[st] = nk;
        }
        if (!ok) break;
        const int sv = j % L::kVStages;
        ok = mbar_wait(bar(L::bVE + sv), ((uint32_t)(j / L::kVStages) & 1u) ^ 1u, ctl);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(L::bVF + sv), L::kTileBytes);
        for (int bx = 0; bx < L::kBoxes; ++bx)
          tma_load_4d(sbase + L::kV + sv * L::kTileBytes + bx * L::kBoxBytes, &tm_v,
                      bar(L::bVF + sv), bx * 64, h, (kv_begin + j) * kBlockN, b);
        last_v[sv] = j;
      }
      if (!ok) {
        // let every copy this thread started land before shared memory is released
        for (int s = 0; s < L::kKStages; ++s)
          if (last_k[s] >= 0)
            mbar_wait_drain(bar(L::bKF + s), (uint32_t)(last_k[s] / L::kKStages) & 1u,
                            p.timeout_ns);
        for (int s = 0; s < L::kVStages; ++s)
          if (last_v[s] >= 0)
            mbar_wait_drain(bar(L::bVF + s), (uint32_t)(last_v[s] / L::kVStages) & 1u,
                            p.timeout_ns);
        mbar_wait_drain(bar(L::bQ), 0, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if constexpr (kSBuf == 1) setmaxnreg_dec<56>();
    if (lane == 0 && !*abort_flag) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, D, true);
      bool ok = mbar_wait(bar(L::bQ), 0, ctl);
      bool issued = false;
      // shared-memory descriptors built once; each MMA moves them by an offset
      const SmemDesc dq = SmemDesc::sw128(sbase + L::kQ, 16, 1024);
      const SmemDesc dk = SmemDesc::sw128(sbase + L::kK, 16, 1024);
      const SmemDesc dv = SmemDesc::sw128(sbase + L::kV, L::kBoxBytes, 1024);
      auto pv = [&](int t) -> bool {
        const int sb = t % kSBuf;
        if (!mbar_wait(bar(L::bPF + sb), (uint32_t)(t / kSBuf) & 1u, ctl)) return false;
        const int st = t % L::kVStages;
        if (!mbar_wait(bar(L::bVF + st), (uint32_t)(t / L::kVStages) & 1u, ctl)) return false;
        tc_fence_after();
        const uint32_t v_off = (uint32_t)st * L::kTileBytes;
        // P: its own columns with one S buffer, else packed over the S buffer it came from
        const uint32_t p_col = kSBuf == 1 ? (uint32_t)L::kColP : (uint32_t)sb * 128;
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk) {
          // B = V tile, N = D (MN-major: d contiguous), K = 16 keys starting at kk*16
          umma_ts(tmem + L::kColO, tmem + p_col + kk * 8, dv.at(v_off + kk * 16 * 128),
                  idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(L::bVE + st));
        umma_commit(bar(L::bOD));
        return true;
      };
      // S(j) = Q K_j^T into S buffer j % kSBuf
      auto qk = [&](int j) -> bool {
        const int st = j % L::kKStages;
        if (!mbar_wait(bar(L::bKF + st), (uint32_t)(j / L::kKStages) & 1u, ctl)) return false;
        tc_fence_after();
        const int sb = j % kSBuf;
        const uint32_t k_off = (uint32_t)st * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
          umma_ss(tmem + sb * 128, dq.at(off), dk.at(k_off + off), idesc_qk, kk > 0 ? 1u : 0u);
        }
        issued = true;
        umma_commit(bar(L::bSF + sb));
        umma_commit(bar(L::bKE + st));
        return true;
      };
      if constexpr (kSBuf == 1) {
        // QK(j+1) needs only the softmax to have read S(j) (P has its own columns), so it
        // runs during the exponentials of tile j; PV(j) follows when P(j) is published
        ok = ok && qk(0);
        for (int j = 0; j < n && ok; ++j) {
          if (j + 1 < n) ok = mbar_wait(bar(L::bSE), (uint32_t)j & 1u, ctl) && qk(j + 1);
          ok = ok && pv(j);
        }
      } else {
        for (int j = 0; j < n && ok; ++j) {
          ok = qk(j);
          if (ok && j >= 1) ok = pv(j - 1);
        }
        if (ok) ok = pv(n - 1);
      }
      if (ok) {
        umma_commit(bar(L::bOF));
      } else if (issued) {
        // all MMAs this thread issued must finish before TMEM is released
        umma_commit(bar(L::bDrain));
        mbar_wait_drain(bar(L::bDrain), 0, p.timeout_ns);
      }
    }
  } else if (kSBuf == 1 && warp < L::kSoftmaxWarp0) {
    setmaxnreg_dec<56>();  // warps 2-3: idle members of the first warpgroup
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    if constexpr (kSBuf == 1) setmaxnreg_inc<200>();
    const int wq = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = wq * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.0f;
    bool ok = !*abort_flag;
    for (int j = 0; j < n && ok; ++j) {
      const int sb = j % kSBuf;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bSF + sb), (uint32_t)(j / kSBuf) & 1u, ctl));
      if (!ok) break;
      tc_fence_after();
      const uint32_t tS = trow + sb * 128;
      const int lim = p.kv_valid - (kv_begin + j) * kBlockN;  // valid keys in this tile
      // the whole 128-score row stays in registers
      float s[kBlockN];
#pragma unroll
      for (int c = 0; c < kBlockN / 32; ++c)
        tmem_ld32(tS + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
      tmem_ld_wait();
      if constexpr (kSBuf == 1) {
        // S(j) is in registers: QK(j+1) may overwrite it (one arrival per warp)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::bSE));
      }
      if (lim < kBlockN) {
#pragma unroll
        for (int c = 0; c < kBlockN; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }
      float mx = row_max<kBlockN>(s) * sl2;
      if (j == 0) {
        m_run = mx;
      } else if (__any_sync(0xffffffffu, mx > m_run + kRescaleThreshold)) {
        // Warp-uniform branch (tcgen05.ld/st are warp-collective): every lane of the
        // warp moves to its own new max; lanes whose max did not grow scale by 1.
        // O must hold the PV of tile j-1 before it is rescaled.
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bOD), (uint32_t)(j - 1) & 1u, ctl));
        if (!ok) break;
        tc_fence_after();
        mx = fmaxf(mx, m_run);
        const float f = ex2(m_run - mx);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(trow + L::kColO + c * 32, o);
          tmem_ld_wait();
          uint32_t u[32];
#pragma unroll
          for (int x = 0; x < 32; ++x) u[x] = __float_as_uint(o[x] * f);
          tmem_st32(trow + L::kColO + c * 32, u);
        }
        tmem_st_wait();
        l_run *= f;
        m_run = mx;
      }
      const float2 nm2 = make_float2(-m_run, -m_run);
      const float2 sc2 = make_float2(sl2, sl2);
      float2 la = make_float2(0.0f, 0.0f), lb = make_float2(0.0f, 0.0f);
      if constexpr (kSBuf == 1) {
        // P has its own columns, which PV(j-1) may still be reading: every exponential
        // first (P packed in registers), then the wait for that PV, then the stores, so the
        // exponentials overlap PV(j-1) instead of waiting behind it
        uint32_t pk[kBlockN / 32][16];
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) exp2_pack16(&s[c * 32], sc2, nm2, la, lb, pk[c]);
        if (j >= 1) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bOD), (uint32_t)(j - 1) & 1u, ctl));
          if (!ok) break;
          tc_fence_after();
        }
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) tmem_st16(trow + L::kColP + c * 16, pk[c]);
      } else {
        // P packed over the S buffer it came from
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) {
          uint32_t pk[16];
          exp2_pack16(&s[c * 32], sc2, nm2, la, lb, pk);
          tmem_st16(tS + c * 16, pk);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::bPF + sb));
      l_run += (la.x + la.y) + (lb.x + lb.y);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bOF), 0, ctl));
    // every softmax thread gets here (all waits are bounded); agree on one outcome so
    // that the epilogue's named barrier is reached by all 128 threads or by none
    ok = named_bar_and(1, kBlockM, ok && !*abort_flag);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      if constexpr (!kSplit) {
        // normalise, round to bf16, stage in the (now idle) Q tile with the
        // 128-byte swizzle the output tensor map expects, then one TMA store
        uint8_t* stage = smem + L::kQ;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(trow + L::kColO + c * 32, o);
          tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) w[x] = pack_bf16x2(o[2 * x] * inv_l, o[2 * x + 1] * inv_l);
          const int bx = c >> 1;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int chunk = (c & 1) * 4 + u;  // 16-byte chunk within the 128-byte row
            uint4* dst = reinterpret_cast<uint4*>(stage + bx * L::kBoxBytes + row * 128 +
                                                  ((chunk ^ (row & 7)) << 4));
            *dst = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, kBlockM);
        if (threadIdx.x == L::kSoftmaxWarp0 * 32) {
          for (int bx = 0; bx < L::kBoxes; ++bx)
            tma_store_4d(&tm_o, sbase + L::kQ + bx * L::kBoxBytes, bx * 64, h, qt * kBlockM, b);
          tma_store_commit();
          tma_store_wait_read0();
        }
      } else {
        const int rows_pad = p.n_q_tiles * kBlockM;
        const int grow = qt * kBlockM + row;
        const bool live = grow < p.q_len;  // padded tail rows of the last tile are not stored
        const size_t prow =
            (((size_t)split * p.batch + b) * p.heads + h) * (size_t)rows_pad + (size_t)grow;
        float4* dst = reinterpret_cast<float4*>(p.o_part + prow * D);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          __syncwarp();
          tmem_ld32(trow + L::kColO + c * 32, o);  // warp-collective: every lane loads
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

// na3d_fwd.cuh -- 3-D neighbourhood attention forward on sm_100a.
//
// The LTX-2.5 diffusion decoder's stages run 3-D neighbourhood attention (NATTEN's fused
// na3d, or a FlexAttention block mask that agrees with it to bf16 rounding; "LTX2.5",
// SGLang Diffusion cookbook, §4.6 Diffusion decoder).  Tokens sit on a T x Y x X grid in
// raster order (n = (t * Y + y) * X + x) in the same bf16 [batch, tokens, heads, head_dim]
// layout as the other kernels.  Along an axis of length N with odd window k <= N the query
// at i sees the k positions from s(i) = min(max(i - (k-1)/2, 0), N - k) (Neighborhood
// Attention's window: centred, shifted inward at the borders); a query attends to the box
// of its three windows:  O = softmax(scale * q K_nbhd^T) V_nbhd, per (batch, head).
//
// Blocking: a query tile is a brick of BT x BY x BX = 128 tokens (one 5-D TMA box, rows in
// raster order inside the brick).  The keys any of its queries can see form a box (the
// union of their windows); it is covered by key tiles that are KT x KY x KX bricks of 128
// keys starting at the box's corner (one 5-D TMA box each, zero fill past the grid), so a
// query brick meets nt * ny * nx key tiles.  The key tile's shape is chosen apart from the
// query brick's, to cover the box with as few tiles as possible (a 2 x 8 x 8 brick's box
// for a 3 x 7 x 7 window, 4 x 14 x 14, takes seven 4 x 2 x 16 tiles but eight 2 x 8 x 8).  The scores of every tile are masked per
// element against the query row's own window (a bias of 0 or -inf per key column and per
// (t, y) row of the tile, from three bit masks, one per axis), and a warp skips the
// exponentials of each 32-key chunk that lies outside all of its rows' windows.
// Softmax and epilogue warps arrive on their mbarriers once per warp, after __syncwarp.
//
// Persistent: one CTA per SM takes every gridDim.x-th (batch, head, brick) unit:
//   warp 0      TMA producer: Q bricks (2 stages, the next brick's Q issued with the
//               current brick's first K), K and V tiles through rings (K before V);
//   warp 1      MMA issuer (elected lane): S = Q K^T into one of two S buffers, then
//               O += P V of the previous tile (possibly the previous brick) into one of
//               two O buffers (brick i uses O buffer i % 2);
//   warps 4-7   softmax, one query row per thread: window mask, online softmax with the
//               lazy O rescale (only when a row's max grows by > 2^8; a row that has
//               seen no key yet takes its first max without touching O, which is still
//               zero), P written over S as bf16; at a brick's end its row sums l go to
//               shared memory;
//   warps 8-11  epilogue: waits for a brick's O and l, frees the O buffer, divides by l,
//               rounds to bf16, stages the brick and stores it with one 5-D TMA store
//               (clipped at the grid's edges), overlapping the next brick's MMAs.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256, 256+D), O1 [256+D, 256+2D).
// Registers (setmaxnreg): producer/MMA warpgroup 80, softmax 232, epilogue 128.
#pragma once

#include "attn_fwd.cuh"

namespace ltx {

struct Na3dParams {
  int batch;
  int heads;
  int grid_t, grid_y, grid_x;  // T, Y, X
  int win_t, win_y, win_x;     // odd window sizes, each <= its axis
  int nb_t, nb_y, nb_x;        // query bricks per axis
  int bricks;                  // nb_t * nb_y * nb_x (per batch element and head)
  float scale_log2;            // scale * log2(e)
  int* status;                 // device status word
  unsigned long long timeout_ns;
};

constexpr int kNaThreads = 384;
constexpr int kNaRegsLaunch = 168;  // what ptxas gives a 384-thread, 1-CTA kernel
constexpr int kNaRegsIssue = 80;    // warps 0-3
constexpr int kNaRegsSoftmax = 232; // warps 4-7
constexpr int kNaRegsEpi = 128;     // warps 8-11
static_assert(128 * (kNaRegsIssue + kNaRegsSoftmax + kNaRegsEpi) <= kNaThreads * kNaRegsLaunch,
              "register split exceeds the launch allocation");

template <int D>
struct NaSmem {
  static_assert(D == 64 || D == 128, "head_dim");
  static constexpr int kBoxes = D / 64;            // 64-column (128-byte) boxes per row
  static constexpr int kBoxBytes = kBlockM * 128;  // 128 rows x 64 bf16
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kQStages = 2;
  static constexpr int kKStages = D == 64 ? 4 : 2;
  static constexpr int kVStages = D == 64 ? 4 : 2;
  static constexpr int kStaging = D == 64 ? 2 : 1;  // output staging bricks
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQStages * kTileBytes;
  static constexpr int kV = kK + kKStages * kTileBytes;
  static constexpr int kStage = kV + kVStages * kTileBytes;
  static constexpr int kRowSum = kStage + kStaging * kTileBytes;  // l per O buffer and row
  static constexpr int kBar = kRowSum + 2 * kBlockM * 4;
  static constexpr int bQF = 0;
  static constexpr int bQE = bQF + kQStages;
  static constexpr int bKF = bQE + kQStages;
  static constexpr int bKE = bKF + kKStages;
  static constexpr int bVF = bKE + kKStages;
  static constexpr int bVE = bVF + kVStages;
  static constexpr int bSF = bVE + kVStages;  // 2: scores in S buffer
  static constexpr int bPF = bSF + 2;         // 2: P in S buffer (128 arrivals)
  static constexpr int bOF = bPF + 2;         // 2: a brick's last PV done in O buffer
  static constexpr int bOE = bOF + 2;         // 2: O buffer and its row sums read (128)
  static constexpr int bLF = bOE + 2;         // 2: row sums of a brick written (128)
  static constexpr int bOD = bLF + 2;         // every PV
  static constexpr int bDrain = bOD + 1;
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kUsed = kAbort + 4;
  static constexpr int kAlloc = ((kUsed + 1024 + 1023) / 1024) * 1024;
  static constexpr uint32_t kColO = 256;
  static_assert(kAlloc <= 227 * 1024, "shared memory per CTA");
};

// First position of the window of (odd) size k around i on an axis of n positions.
__host__ __device__ __forceinline__ int na_window_start(int i, int k, int n) {
  const int s = i - (k >> 1);
  return s < 0 ? 0 : (s > n - k ? n - k : s);
}

// Key box of the query positions [a0, min(a0 + bq, n)) on one axis: its first position and
// the number of bk-wide key tiles that cover it.
__host__ __device__ __forceinline__ void na_key_span(int a0, int bq, int bk, int k, int n,
                                                     int& r0, int& tiles) {
  const int a1 = a0 + bq < n ? a0 + bq : n;
  r0 = na_window_start(a0, k, n);
  const int r1 = na_window_start(a1 - 1, k, n) + k;
  tiles = (r1 - r0 + bk - 1) / bk;
}

// One query brick (BT x BY x BX) of one (batch, head) and the key tiles (KT x KY x KX
// bricks, 128 keys each) that cover its key box.
template <int BT, int BY, int BX, int KT, int KY, int KX>
struct NaBrick {
  int b, h;
  int t0, y0, x0;  // query brick origin
  int rt, ry, rx;  // key box origin
  int nt, ny, nx;  // key tiles per axis
  int n;           // key tiles
  __device__ __forceinline__ void init(long long u, const Na3dParams& p) {
    const long long bh = u / p.bricks;
    int br = (int)(u - bh * p.bricks);
    b = (int)(bh / p.heads);
    h = (int)(bh - (long long)b * p.heads);
    const int ix = br % p.nb_x;
    br /= p.nb_x;
    const int iy = br % p.nb_y;
    const int it = br / p.nb_y;
    t0 = it * BT;
    y0 = iy * BY;
    x0 = ix * BX;
    na_key_span(t0, BT, KT, p.win_t, p.grid_t, rt, nt);
    na_key_span(y0, BY, KY, p.win_y, p.grid_y, ry, ny);
    na_key_span(x0, BX, KX, p.win_x, p.grid_x, rx, nx);
    n = nt * ny * nx;
  }
  // origin of key tile j (x fastest)
  __device__ __forceinline__ void key_origin(int j, int& kt, int& ky, int& kx) const {
    const int jx = j % nx;
    const int r = j / nx;
    kt = rt + (r / ny) * KT;
    ky = ry + (r % ny) * KY;
    kx = rx + jx * KX;
  }
};

// Bits [max(lo, 0), min(hi, n)) of a 32-bit word (n <= 32).
__device__ __forceinline__ uint32_t na_bits(int lo, int hi, int n) {
  const int a = lo > 0 ? lo : 0;
  const int e = hi < n ? hi : n;
  return e > a ? ((0xffffffffu >> (32 - (e - a))) << a) : 0u;
}

template <int D, int BT, int BY, int BX, int KT, int KY, int KX>
__global__ void __launch_bounds__(kNaThreads, 1)
    ltx_na3d_fwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const Na3dParams p) {
  static_assert(BT * BY * BX == kBlockM && BX <= 32 && BY <= 32 && BT <= 32, "brick");
  static_assert(KT * KY * KX == kBlockN && KT * KY <= 32 && 32 % KX == 0 && KX % 2 == 0,
                "key tile: 128 keys, rows of KX keys filling whole 32-key chunks");
  using L = NaSmem<D>;
  using Brick = NaBrick<BT, BY, BX, KT, KY, KX>;
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
  // bricks blockIdx.x, blockIdx.x + gridDim.x, ...: at any moment the CTAs work on
  // neighbouring bricks of one (batch, head) and share their key tiles through L2 (a
  // contiguous run per CTA read 2.4 GB from DRAM for 0.8 GB of q, k, v; this order 0.95 GB)
  const long long total = (long long)p.batch * p.heads * p.bricks;
  const int cnt = (int)((total - blockIdx.x + gridDim.x - 1) / gridDim.x);
  auto unit = [&](int i) -> long long { return (long long)blockIdx.x + (long long)i * gridDim.x; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kQStages; ++s) {
      mbar_init(bar(L::bQF + s), 1);
      mbar_init(bar(L::bQE + s), 1);
    }
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
      mbar_init(bar(L::bPF + s), 4);
      mbar_init(bar(L::bOF + s), 1);
      mbar_init(bar(L::bOE + s), 4);
      mbar_init(bar(L::bLF + s), 4);
    }
    mbar_init(bar(L::bOD), 1);
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
    setmaxnreg_dec<kNaRegsIssue>();
    if (lane == 0 && !*abort_flag && cnt > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int last_q[L::kQStages], last_k[L::kKStages], last_v[L::kVStages];
      for (int s = 0; s < L::kQStages; ++s) last_q[s] = -1;
      for (int s = 0; s < L::kKStages; ++s) last_k[s] = -1;
      for (int s = 0; s < L::kVStages; ++s) last_v[s] = -1;
      auto load_q = [&](int i, const Brick& q) -> bool {
        const int qs = i % L::kQStages;
        if (!mbar_wait_lean(bar(L::bQE + qs), ((uint32_t)(i / L::kQStages) & 1u) ^ 1u, ctl))
          return false;
        mbar_arrive_expect_tx(bar(L::bQF + qs), L::kTileBytes);
#pragma unroll
        for (int bx = 0; bx < L::kBoxes; ++bx)
          tma_load_5d(sbase + L::kQ + qs * L::kTileBytes + bx * L::kBoxBytes, &tm_q,
                      bar(L::bQF + qs), q.h * D + bx * 64, q.x0, q.y0, q.t0, q.b);
        last_q[qs] = i;
        return true;
      };
      Brick cur, nxt;
      cur.init(unit(0), p);
      bool ok = load_q(0, cur);
      int g = 0;  // key tiles issued so far
      for (int i = 0; i < cnt && ok; ++i) {
        if (i + 1 < cnt) nxt.init(unit(i + 1), p);
        for (int j = 0; j < cur.n && ok; ++j, ++g) {
          int kt, ky, kx;
          cur.key_origin(j, kt, ky, kx);
          const int ks = g % L::kKStages;
          ok = mbar_wait_lean(bar(L::bKE + ks), ((uint32_t)(g / L::kKStages) & 1u) ^ 1u, ctl);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(L::bKF + ks), L::kTileBytes);
#pragma unroll
          for (int bx = 0; bx < L::kBoxes; ++bx)
            tma_load_5d(sbase + L::kK + ks * L::kTileBytes + bx * L::kBoxBytes, &tm_k,
                        bar(L::bKF + ks), cur.h * D + bx * 64, kx, ky, kt, cur.b);
          last_k[ks] = g;
          // the next brick's queries, once this brick's first keys are on their way
          if (j == 0 && i + 1 < cnt) {
            ok = load_q(i + 1, nxt);
            if (!ok) break;
          }
          const int vs = g % L::kVStages;
          ok = mbar_wait_lean(bar(L::bVE + vs), ((uint32_t)(g / L::kVStages) & 1u) ^ 1u, ctl);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(L::bVF + vs), L::kTileBytes);
#pragma unroll
          for (int bx = 0; bx < L::kBoxes; ++bx)
            tma_load_5d(sbase + L::kV + vs * L::kTileBytes + bx * L::kBoxBytes, &tm_v,
                        bar(L::bVF + vs), cur.h * D + bx * 64, kx, ky, kt, cur.b);
          last_v[vs] = g;
        }
        cur = nxt;
      }
      if (!ok) {
        // every copy this thread started lands before shared memory is released
        for (int s = 0; s < L::kQStages; ++s)
          if (last_q[s] >= 0)
            mbar_wait_drain(bar(L::bQF + s), (uint32_t)(last_q[s] / L::kQStages) & 1u,
                            p.timeout_ns);
        for (int s = 0; s < L::kKStages; ++s)
          if (last_k[s] >= 0)
            mbar_wait_drain(bar(L::bKF + s), (uint32_t)(last_k[s] / L::kKStages) & 1u,
                            p.timeout_ns);
        for (int s = 0; s < L::kVStages; ++s)
          if (last_v[s] >= 0)
            mbar_wait_drain(bar(L::bVF + s), (uint32_t)(last_v[s] / L::kVStages) & 1u,
                            p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    setmaxnreg_dec<kNaRegsIssue>();
    // the whole warp runs the loop; one elected lane issues, the lanes agree on waits
    if (!*abort_flag && cnt > 0) {
      auto wt = [&](uint32_t bar_addr, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait_lean(bar_addr, parity, ctl));
      };
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, D, true);
      const SmemDesc dq = SmemDesc::sw128(sbase + L::kQ, 16, 1024);
      const SmemDesc dk = SmemDesc::sw128(sbase + L::kK, 16, 1024);
      const SmemDesc dv = SmemDesc::sw128(sbase + L::kV, L::kBoxBytes, 1024);
      bool issued = false;
      // O += P_t V_t for key tile t (global count) = tile j of brick i, which has n tiles
      auto pv = [&](int t, int i, int j, int n) -> bool {
        const int sb = t & 1;
        const int vs = t % L::kVStages;
        const int ob = i & 1;
        if (!wt(bar(L::bPF + sb), (uint32_t)(t >> 1) & 1u) ||
            !wt(bar(L::bVF + vs), (uint32_t)(t / L::kVStages) & 1u))
          return false;
        // a brick's first PV overwrites its O buffer: the epilogue of brick i - 2 read it
        if (j == 0 && i >= 2 && !wt(bar(L::bOE + ob), (uint32_t)((i >> 1) - 1) & 1u))
          return false;
        tc_fence_after();
        const uint32_t v_off = (uint32_t)vs * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk)
          umma_ts_elect(tmem + L::kColO + ob * D, tmem + sb * 128 + kk * 8,
                        dv.at(v_off + kk * 16 * 128), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit_elect(bar(L::bVE + vs));
        umma_commit_elect(bar(L::bOD));
        if (j == n - 1) umma_commit_elect(bar(L::bOF + ob));
        return true;
      };
      bool ok = true;
      int g = 0;
      int pt = -1, pi = 0, pj = 0, pn = 0;  // the tile whose PV is still to issue
      Brick cur;
      for (int i = 0; i < cnt && ok; ++i) {
        cur.init(unit(i), p);
        const int qs = i % L::kQStages;
        ok = wt(bar(L::bQF + qs), (uint32_t)(i / L::kQStages) & 1u);
        for (int j = 0; j < cur.n && ok; ++j, ++g) {
          const int ks = g % L::kKStages;
          ok = wt(bar(L::bKF + ks), (uint32_t)(g / L::kKStages) & 1u);
          if (!ok) break;
          tc_fence_after();
          const int sb = g & 1;
          const uint32_t q_off = (uint32_t)qs * L::kTileBytes;
          const uint32_t k_off = (uint32_t)ks * L::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
            umma_ss_elect(tmem + sb * 128, dq.at(q_off + off), dk.at(k_off + off), idesc_qk,
                          kk > 0 ? 1u : 0u);
          }
          issued = true;
          umma_commit_elect(bar(L::bSF + sb));
          umma_commit_elect(bar(L::bKE + ks));
          if (j == cur.n - 1) umma_commit_elect(bar(L::bQE + qs));
          if (pt >= 0) ok = pv(pt, pi, pj, pn);
          pt = g;
          pi = i;
          pj = j;
          pn = cur.n;
        }
      }
      if (ok && pt >= 0) ok = pv(pt, pi, pj, pn);
      if (!ok && issued) {
        umma_commit_elect(bar(L::bDrain));
        mbar_wait_drain(bar(L::bDrain), 0, p.timeout_ns);
      }
    }
  } else if (warp < 4) {
    setmaxnreg_dec<kNaRegsIssue>();  // warps 2-3: idle
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax
    setmaxnreg_inc<kNaRegsSoftmax>();
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t tlane = tmem + ((uint32_t)(wq * 32) << 16);
    // this row's place in the brick
    const int lt = row / (BX * BY), ly = (row / BX) % BY, lx = row % BX;
    const float sl2 = p.scale_log2;
    const float2 sc2 = make_float2(sl2, sl2);
    bool ok = !*abort_flag;
    int g = 0;
    Brick cur;
    for (int i = 0; i < cnt && ok; ++i) {
      cur.init(unit(i), p);
      const int ob = i & 1;
      // window starts of this query (rows past the grid's edge take the last position's
      // window; their output is clipped by the store)
      const int wt0 = na_window_start(min(cur.t0 + lt, p.grid_t - 1), p.win_t, p.grid_t);
      const int wy0 = na_window_start(min(cur.y0 + ly, p.grid_y - 1), p.win_y, p.grid_y);
      const int wx0 = na_window_start(min(cur.x0 + lx, p.grid_x - 1), p.win_x, p.grid_x);
      float m_run = -INFINITY;  // log2 units; -inf until the row has seen a key
      float l_run = 0.0f;
      for (int j = 0; j < cur.n && ok; ++j, ++g) {
        const int sb = g & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bSF + sb), (uint32_t)(g >> 1) & 1u, ctl));
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tlane + sb * 128;
        float s[kBlockN];
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c)
          tmem_ld32(tS + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
        int kt, ky, kx;
        cur.key_origin(j, kt, ky, kx);
        const uint32_t mt = na_bits(wt0 - kt, wt0 - kt + p.win_t, KT);
        const uint32_t my = na_bits(wy0 - ky, wy0 - ky + p.win_y, KY);
        const uint32_t mx = na_bits(wx0 - kx, wx0 - kx + p.win_x, KX);
        // window mask as additive biases (0 inside, -inf outside): one per key column x
        // of the tile and one per (t, y) row of it, two packed adds per pair of scores
        float2 bx2[KX / 2];
#pragma unroll
        for (int c2 = 0; c2 < KX / 2; ++c2)
          bx2[c2] = make_float2((mx >> (2 * c2)) & 1u ? 0.0f : -INFINITY,
                                (mx >> (2 * c2 + 1)) & 1u ? 0.0f : -INFINITY);
        uint32_t rows_in = 0;  // (t, y) rows of the tile inside this query's window
        tmem_ld_wait();
#pragma unroll
        for (int r = 0; r < KT * KY; ++r) {
          const bool in = (mt >> (r / KY)) & (my >> (r % KY)) & 1u;
          rows_in |= (in ? 1u : 0u) << r;
          const float rb = in ? 0.0f : -INFINITY;
          const float2 rb2 = make_float2(rb, rb);
#pragma unroll
          for (int c2 = 0; c2 < KX / 2; ++c2) {
            float2 v = make_float2(s[r * KX + 2 * c2], s[r * KX + 2 * c2 + 1]);
            v = __fadd2_rn(__fadd2_rn(v, bx2[c2]), rb2);
            s[r * KX + 2 * c2] = v.x;
            s[r * KX + 2 * c2 + 1] = v.y;
          }
        }
        const float mx_t = row_max<kBlockN>(s) * sl2;
        const bool grow = m_run != -INFINITY && mx_t > m_run + kRescaleThreshold;
        if (__any_sync(0xffffffffu, grow)) {
          // O must hold the PV of the previous tile before it is rescaled (tcgen05.ld/st
          // are warp-collective: lanes whose max did not grow scale by 1)
          ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bOD), (uint32_t)(g - 1) & 1u, ctl));
          if (!ok) break;
          tc_fence_after();
          const float mn = grow ? mx_t : m_run;
          const float f = grow ? ex2(m_run - mn) : 1.0f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld32(tlane + L::kColO + ob * D + c * 32, o);
            tmem_ld_wait();
            uint32_t u[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) u[x] = __float_as_uint(o[x] * f);
            tmem_st32(tlane + L::kColO + ob * D + c * 32, u);
          }
          tmem_st_wait();
          l_run *= f;
          m_run = mn;
        }
        // a row's first keys: take their max (O and l of the row are still zero)
        if (m_run == -INFINITY) m_run = mx_t;
        const float m_use = m_run == -INFINITY ? 0.0f : m_run;
        const float2 nm2 = make_float2(-m_use, -m_use);
        float2 la = make_float2(0.0f, 0.0f), lb = make_float2(0.0f, 0.0f);
        if (mx == 0) rows_in = 0;
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) {
          // a 32-key chunk outside every window of this warp's rows: P = 0 without the
          // exponentials (the MUFU bounds this loop)
          constexpr int kRowsChunk = 32 / KX;
          const uint32_t chunk_rows = (rows_in >> (c * kRowsChunk)) & ((1u << kRowsChunk) - 1u);
          uint32_t pk[16];
          if (__any_sync(0xffffffffu, chunk_rows != 0)) {
            exp2_pack16(&s[c * 32], sc2, nm2, la, lb, pk);
          } else {
#pragma unroll
            for (int x = 0; x < 16; ++x) pk[x] = 0u;
          }
          tmem_st16(tS + c * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::bPF + sb));
        l_run += (la.x + la.y) + (lb.x + lb.y);
      }
      if (!ok) break;
      // the row sums of brick i - 2 in this slot were read by its epilogue
      if (i >= 2)
        ok = __all_sync(0xffffffffu,
                        mbar_wait(bar(L::bOE + ob), (uint32_t)((i >> 1) - 1) & 1u, ctl));
      if (!ok) break;
      row_sum[ob * kBlockM + row] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::bLF + ob));
    }
  } else {
    // ------------------------------------------------------------ epilogue
    setmaxnreg_dec<kNaRegsEpi>();
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t tlane = tmem + ((uint32_t)(wq * 32) << 16);
    const bool leader = wq == 0 && lane == 0;
    bool ok = !*abort_flag;
    Brick cur;
    for (int i = 0; i < cnt && ok; ++i) {
      cur.init(unit(i), p);
      const int ob = i & 1;
      const uint32_t ph = (uint32_t)(i >> 1) & 1u;
      bool w = mbar_wait(bar(L::bOF + ob), ph, ctl);
      w = w && mbar_wait(bar(L::bLF + ob), ph, ctl);
      ok = named_bar_and(1, kBlockM, w);  // the four warps leave together or not at all
      if (!ok) break;
      tc_fence_after();
      const float inv_l = 1.0f / row_sum[ob * kBlockM + row];
      const int sbuf = L::kStaging == 2 ? (i & 1) : 0;
      uint8_t* stage = smem + L::kStage + sbuf * L::kTileBytes;
      // the store issued kStaging bricks ago from this staging buffer must have read it
      if (leader) tma_store_wait_read<L::kStaging - 1>();
      named_bar_sync(1, kBlockM);
      const float2 il2 = make_float2(inv_l, inv_l);
#pragma unroll
      for (int bx = 0; bx < L::kBoxes; ++bx) {
        float o[64];
        tmem_ld32(tlane + L::kColO + ob * D + bx * 64, *reinterpret_cast<float(*)[32]>(&o[0]));
        tmem_ld32(tlane + L::kColO + ob * D + bx * 64 + 32,
                  *reinterpret_cast<float(*)[32]>(&o[32]));
        tmem_ld_wait();
        if (bx == L::kBoxes - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(L::bOE + ob));
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint32_t w4[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const float2 v2 =
                __fmul2_rn(make_float2(o[8 * u + 2 * x], o[8 * u + 2 * x + 1]), il2);
            w4[x] = pack_bf16x2(v2.x, v2.y);
          }
          *reinterpret_cast<uint4*>(stage + bx * L::kBoxBytes + row * 128 +
                                    ((u ^ (row & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1, kBlockM);
      if (leader) {
#pragma unroll
        for (int bx = 0; bx < L::kBoxes; ++bx)
          tma_store_5d(&tm_o, sbase + L::kStage + sbuf * L::kTileBytes + bx * L::kBoxBytes,
                       cur.h * D + bx * 64, cur.x0, cur.y0, cur.t0, cur.b);
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

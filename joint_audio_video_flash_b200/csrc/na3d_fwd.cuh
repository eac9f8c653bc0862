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
// union of their windows); it is covered by key tiles that are KT x KY x KX bricks of 112
// or 128 keys starting at the box's corner (one 5-D TMA box each, zero fill past the grid),
// so a query brick meets nt * ny * nx key tiles.  The key tile's shape is chosen apart from
// the query brick's, to cover the box with as few tiles and keys as possible (a 2 x 8 x 8
// brick's box for a 3 x 7 x 7 window, 4 x 14 x 14, is exactly seven 4 x 2 x 14 tiles; it
// takes seven 4 x 2 x 16 or eight 2 x 8 x 8 ones of 128 keys).
// The scores of every tile are masked per element against the query row's own window:
// a bias of 0 or -inf per key column x, and per (t, y) row of the tile a choice between the
// row's max offset and -inf in the exponent (three bit masks, one per axis); a warp skips
// the exponentials of each 32-key chunk that lies outside all of its rows' windows.
//
// Two softmax warpgroups split every key tile into halves of whole key rows: group g takes
// keys [n g, n g + n), n = 56 or 64, and writes their P as 64 keys (zero past its n) over
// columns [64 g, 64 g + 32) of S.  Each keeps its own running max, row sum and O accumulator
// (two PV products per tile, one per half), so the groups never wait for each other
// inside a brick and every SM sub-partition runs two softmax warps; the halves are merged
// once per brick (the group-0 statistics go to group 1 through shared memory, group 1
// writes both halves' weights, the epilogue sums the two O's with them).
// Softmax and epilogue warps arrive on their mbarriers once per warp, after __syncwarp.
//
// Persistent: one CTA per SM takes every gridDim.x-th (batch, head, brick) unit:
//   warp 0      TMA producer: Q bricks (2 stages, the next brick's Q issued with the
//               current brick's last K), K and V tiles through rings (K before V);
//   warp 1      MMA issuer (elected lane): S = Q K^T into one of two S buffers, then
//               O_g += P_g V_g of the previous tile (possibly the previous brick) for each
//               half g once its group has written P;
//   warps 4-11  softmax, two groups of four warps, one query row per thread and group:
//               window mask, online softmax with the lazy O rescale (only when a row's max
//               grows by > 2^8; a row that has seen no key yet takes its first max without
//               touching O, which is still zero), P written over its half of S as bf16;
//   warps 12-15 epilogue: waits for a brick's O's and weights, frees the O buffers, merges
//               the halves, rounds to bf16, stages the brick in its own Q stage and stores
//               it with one 5-D TMA store (clipped at the grid's edges), overlapping the
//               next brick's MMAs; the Q stage returns to the producer once the store has
//               read it.
// TMEM (512 columns): S0 [0,128), S1 [128,256) (a 112-key tile's QK writes the first 112
// columns; rows 112-127 of every V stage are zeroed once, since the second half's PV reads V
// rows up to 119 with P = 0 there); from 256 the O accumulators, one per group
// (head_dim 128), or one per group and brick parity (head_dim 64: 4 x 64 columns).
// Registers (setmaxnreg): producer/MMA warpgroup 88, softmax 168 (each group), epilogue 88.
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

constexpr int kNaThreads = 512;
constexpr int kNaRegsLaunch = 128;  // what ptxas gives a 512-thread, 1-CTA kernel
constexpr int kNaRegsIssue = 88;    // warps 0-3
constexpr int kNaRegsSoftmax = 168; // warps 4-11
constexpr int kNaRegsEpi = 88;      // warps 12-15
static_assert(128 * (kNaRegsIssue + 2 * kNaRegsSoftmax + kNaRegsEpi) <= kNaThreads * kNaRegsLaunch,
              "register split exceeds the launch allocation");
constexpr int kNaHalf = kBlockN / 2;  // keys of a tile per softmax group

template <int D>
struct NaSmem {
  static_assert(D == 64 || D == 128, "head_dim");
  static constexpr int kBoxes = D / 64;            // 64-column (128-byte) boxes per row
  static constexpr int kBoxBytes = kBlockM * 128;  // 128 rows x 64 bf16
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  // the epilogue stages a brick's output in the brick's own Q stage (its MMAs are done)
  static constexpr int kQStages = 2;
  static constexpr int kKStages = D == 64 ? 4 : 2;
  static constexpr int kVStages = D == 64 ? 4 : 3;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQStages * kTileBytes;
  static constexpr int kV = kK + kKStages * kTileBytes;
  // one slot of per-row brick statistics: group 0's (max, sum), which group 1 replaces by
  // the two halves' merge weights
  static constexpr int kStats = kV + kVStages * kTileBytes;
  static constexpr int kBar = kStats + kBlockM * 8;
  static constexpr int bQF = 0;
  static constexpr int bQE = bQF + kQStages;  // Q stage free: the brick's output store read it
  static constexpr int bKF = bQE + kQStages;
  static constexpr int bKE = bKF + kKStages;
  static constexpr int bVF = bKE + kKStages;
  static constexpr int bVE = bVF + kVStages;
  static constexpr int bSF = bVE + kVStages;  // 2: scores in S buffer
  static constexpr int bPF = bSF + 2;         // 2 x 2: P of group g in S buffer (4 warps)
  static constexpr int bOF = bPF + 4;         // 2: a brick's last PVs done (by brick parity)
  static constexpr int bOE = bOF + 2;         // 2: a brick's O's and weights read (4 warps)
  static constexpr int bSA = bOE + 2;         // group 0's statistics of a brick written
  static constexpr int bLF = bSA + 1;         // merge weights of a brick written
  static constexpr int bOD = bLF + 1;         // 2: every PV of group g
  static constexpr int bDrain = bOD + 2;
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kUsed = kAbort + 4;
  static constexpr int kAlloc = ((kUsed + 1024 + 1023) / 1024) * 1024;
  // O accumulators: one per group, and per brick parity where they fit (head_dim 64)
  static constexpr int kOBufs = D == 64 ? 2 : 1;
  static constexpr uint32_t kColO = 256;
  static_assert(kColO + 2 * kOBufs * D <= 512, "TMEM columns");
  __device__ __forceinline__ static uint32_t col_o(int g, int brick) {
    return kColO + (uint32_t)(((brick % kOBufs) * 2 + g) * D);
  }
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

// Eight 32-bit columns of this warp's TMEM lanes into registers.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

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
  // a key tile of kKeys keys: each softmax group takes kGrpKeys of them (whole rows of KX
  // keys) and writes their P over a 64-key span, zero past its keys
  constexpr int kKeys = KT * KY * KX;
  constexpr int kGrpKeys = kKeys / 2;
  static_assert(kKeys <= kBlockN && kGrpKeys % KX == 0 && kGrpKeys % 8 == 0 &&
                    kGrpKeys > kNaHalf - 16 && KT * KY <= 32 && KX % 2 == 0 && KX >= 4,
                "key tile: 112 to 128 keys, each half whole rows of an even number of keys");
  using L = NaSmem<D>;
  constexpr uint32_t kKVBytes = (uint32_t)kKeys * 128u * L::kBoxes;  // one K or V tile
  using Brick = NaBrick<BT, BY, BX, KT, KY, KX>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  float2* stats = reinterpret_cast<float2*>(smem + L::kStats);

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
      mbar_init(bar(L::bPF + 2 * s), 4);
      mbar_init(bar(L::bPF + 2 * s + 1), 4);
      mbar_init(bar(L::bOF + s), 1);
      mbar_init(bar(L::bOE + s), 4);
      mbar_init(bar(L::bOD + s), 1);
    }
    mbar_init(bar(L::bSA), 4);
    mbar_init(bar(L::bLF), 4);
    mbar_init(bar(L::bDrain), 1);
    *abort_flag = (*reinterpret_cast<volatile int*>(p.status) != kDevOk) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + L::kTmemSlot, 512);
    tmem_relinquish();
  }
  if constexpr (kKeys < kBlockN) {
    // rows [kKeys, 128) of the V stages are never loaded, and the second group's PV reads
    // rows up to kGrpKeys + 63 (with P = 0 past its keys): they must hold finite values
    constexpr int kPad16 = (kBlockN - kKeys) * 128 / 16;  // 16-byte units per box
    for (int i = threadIdx.x; i < L::kVStages * L::kBoxes * kPad16; i += blockDim.x)
      *reinterpret_cast<uint4*>(smem + L::kV + (i / kPad16) * L::kBoxBytes + kKeys * 128 +
                                (i % kPad16) * 16) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
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
          mbar_arrive_expect_tx(bar(L::bKF + ks), kKVBytes);
#pragma unroll
          for (int bx = 0; bx < L::kBoxes; ++bx)
            tma_load_5d(sbase + L::kK + ks * L::kTileBytes + bx * L::kBoxBytes, &tm_k,
                        bar(L::bKF + ks), cur.h * D + bx * 64, kx, ky, kt, cur.b);
          last_k[ks] = g;
          // the next brick's queries with this brick's last keys: their stage held the
          // output of brick i - 1, whose store must have read it
          if (j == cur.n - 1 && i + 1 < cnt) {
            ok = load_q(i + 1, nxt);
            if (!ok) break;
          }
          const int vs = g % L::kVStages;
          ok = mbar_wait_lean(bar(L::bVE + vs), ((uint32_t)(g / L::kVStages) & 1u) ^ 1u, ctl);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(L::bVF + vs), kKVBytes);
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
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kKeys, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, D, true);
      const SmemDesc dq = SmemDesc::sw128(sbase + L::kQ, 16, 1024);
      const SmemDesc dk = SmemDesc::sw128(sbase + L::kK, 16, 1024);
      const SmemDesc dv = SmemDesc::sw128(sbase + L::kV, L::kBoxBytes, 1024);
      bool issued = false;
      // O_g += P_g V_g over both halves g of key tile t (global count) = tile j of brick i,
      // which has n tiles; each half as soon as its group has written P
      auto pv = [&](int t, int i, int j, int n) -> bool {
        const int sb = t & 1;
        const int vs = t % L::kVStages;
        if (!wt(bar(L::bVF + vs), (uint32_t)(t / L::kVStages) & 1u)) return false;
        // a brick's first PVs overwrite their O buffers: the epilogue of brick i - kOBufs
        // read them
        const int ip = i - L::kOBufs;
        if (j == 0 && ip >= 0 && !wt(bar(L::bOE + (ip & 1)), (uint32_t)(ip >> 1) & 1u))
          return false;
        const uint32_t v_off = (uint32_t)vs * L::kTileBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (!wt(bar(L::bPF + 2 * sb + h), (uint32_t)(t >> 1) & 1u)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kNaHalf / 16; ++kk)
            umma_ts_elect(tmem + L::col_o(h, i), tmem + sb * 128 + h * kNaHalf + kk * 8,
                          dv.at(v_off + (h * kGrpKeys + kk * 16) * 128), idesc_pv,
                          (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit_elect(bar(L::bOD + h));
        }
        umma_commit_elect(bar(L::bVE + vs));
        if (j == n - 1) umma_commit_elect(bar(L::bOF + (i & 1)));
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
  } else if (warp < 12) {
    // ------------------------------------------------------------ softmax
    setmaxnreg_inc<kNaRegsSoftmax>();
    const int grp = (warp >> 2) - 1;  // 0: keys [0, 64) of every tile, 1: keys [64, 128)
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t tlane = tmem + ((uint32_t)(wq * 32) << 16);
    // this row's place in the brick
    const int lt = row / (BX * BY), ly = (row / BX) % BY, lx = row % BX;
    const float sl2 = p.scale_log2;
    const float2 sc2 = make_float2(sl2, sl2);
    constexpr int kRows = kGrpKeys / KX;  // (t, y) rows of a tile in this group's half
    const int r0 = grp * kRows;           // the half's first row in the tile
    bool ok = !*abort_flag;
    int g = 0;
    Brick cur;
    for (int i = 0; i < cnt && ok; ++i) {
      cur.init(unit(i), p);
      const uint32_t tO = tlane + L::col_o(grp, i);
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
        const uint32_t tS = tlane + sb * 128 + grp * kGrpKeys;  // this half's scores
        const uint32_t tP = tlane + sb * 128 + grp * kNaHalf;   // its P: 64 keys, 32 columns
        float s[kGrpKeys];
        if constexpr (kGrpKeys % 32 == 0) {
#pragma unroll
          for (int c = 0; c < kGrpKeys / 32; ++c)
            tmem_ld32(tS + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
        } else {
#pragma unroll
          for (int c = 0; c < kGrpKeys / 8; ++c)
            tmem_ld8(tS + c * 8, *reinterpret_cast<float(*)[8]>(&s[c * 8]));
        }
        int kt, ky, kx;
        cur.key_origin(j, kt, ky, kx);
        const uint32_t mt = na_bits(wt0 - kt, wt0 - kt + p.win_t, KT);
        const uint32_t my = na_bits(wy0 - ky, wy0 - ky + p.win_y, KY);
        const uint32_t mx = na_bits(wx0 - kx, wx0 - kx + p.win_x, KX);
        // the key columns x of the tile outside this query's window: a bias of -inf, one
        // packed add per pair of scores
        float2 bx2[KX / 2];
#pragma unroll
        for (int c2 = 0; c2 < KX / 2; ++c2)
          bx2[c2] = make_float2((mx >> (2 * c2)) & 1u ? 0.0f : -INFINITY,
                                (mx >> (2 * c2 + 1)) & 1u ? 0.0f : -INFINITY);
        uint32_t rows_in = 0;  // (t, y) rows of the half inside this query's window
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          const int rr = r0 + r;
          rows_in |= ((mt >> (rr / KY)) & (my >> (rr % KY)) & 1u) << r;
        }
        if (mx == 0) rows_in = 0;
        tmem_ld_wait();
        // the max over the keys inside the window: per row of the half over its
        // column-masked scores, rows outside the window left out
        float mrow = -INFINITY;
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          float* sr = &s[r * KX];
#pragma unroll
          for (int c2 = 0; c2 < KX / 2; ++c2) {
            const float2 v = __fadd2_rn(make_float2(sr[2 * c2], sr[2 * c2 + 1]), bx2[c2]);
            sr[2 * c2] = v.x;
            sr[2 * c2 + 1] = v.y;
          }
          float a = fmaxf(sr[0], sr[1]), b = fmaxf(sr[2], sr[3]);
#pragma unroll
          for (int c = 4; c + 4 <= KX; c += 4) {
            a = fmax3(a, sr[c], sr[c + 1]);
            b = fmax3(b, sr[c + 2], sr[c + 3]);
          }
          if constexpr (KX % 4 == 2) a = fmax3(a, sr[KX - 2], sr[KX - 1]);
          mrow = (rows_in >> r) & 1u ? fmax3(mrow, a, b) : mrow;
        }
        const float mx_t = mrow * sl2;
        const bool grow = m_run != -INFINITY && mx_t > m_run + kRescaleThreshold;
        if (__any_sync(0xffffffffu, grow)) {
          // O must hold this group's PV of the previous tile before it is rescaled
          // (tcgen05.ld/st are warp-collective: lanes whose max did not grow scale by 1)
          ok = __all_sync(0xffffffffu,
                          mbar_wait(bar(L::bOD + grp), (uint32_t)(g - 1) & 1u, ctl));
          if (!ok) break;
          tc_fence_after();
          const float mn = grow ? mx_t : m_run;
          const float f = grow ? ex2(m_run - mn) : 1.0f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_ld_wait();
            uint32_t u[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) u[x] = __float_as_uint(o[x] * f);
            tmem_st32(tO + c * 32, u);
          }
          tmem_st_wait();
          l_run *= f;
          m_run = mn;
        }
        // a row's first keys: take their max (O and l of the row are still zero)
        if (m_run == -INFINITY) m_run = mx_t;
        const float m_use = m_run == -INFINITY ? 0.0f : m_run;
        // rows outside the window get an exponent offset of -inf (p = 0)
        float2 nm2[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          const float nm = (rows_in >> r) & 1u ? -m_use : -INFINITY;
          nm2[r] = make_float2(nm, nm);
        }
        float2 la = make_float2(0.0f, 0.0f), lb = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int c = 0; c < kNaHalf / 32; ++c) {
          // a 32-key chunk outside every window of this warp's rows: P = 0 without the
          // exponentials; P past this half's keys is 0
          const int ra = c * 32 / KX;
          const int rb = (c * 32 + 31 < kGrpKeys ? c * 32 + 31 : kGrpKeys - 1) / KX;
          const uint32_t chunk_rows = rows_in & (((2u << rb) - 1u) & ~((1u << ra) - 1u));
          uint32_t pk[16];
          if (__any_sync(0xffffffffu, chunk_rows != 0)) {
#pragma unroll
            for (int x = 0; x < 16; ++x) {
              const int k = c * 32 + 2 * x;
              if (k >= kGrpKeys) {
                pk[x] = 0u;
                continue;
              }
              const float2 a = __ffma2_rn(make_float2(s[k], s[k + 1]), sc2, nm2[k / KX]);
              const float2 e = make_float2(ex2(a.x), ex2(a.y));
              if (x & 1)
                lb = __fadd2_rn(lb, e);
              else
                la = __fadd2_rn(la, e);
              pk[x] = pack_bf16x2(e.x, e.y);
            }
          } else {
#pragma unroll
            for (int x = 0; x < 16; ++x) pk[x] = 0u;
          }
          tmem_st16(tP + c * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::bPF + 2 * sb + grp));
        l_run += (la.x + la.y) + (lb.x + lb.y);
      }
      if (!ok) break;
      if (grp == 0) {
        // the slot's previous contents (brick i - 1's weights) were read by its epilogue
        if (i >= 1)
          ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bOE + ((i - 1) & 1)),
                                                 (uint32_t)((i - 1) >> 1) & 1u, ctl));
        if (!ok) break;
        stats[row] = make_float2(m_run, l_run);
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::bSA));
      } else {
        // merge weights of the two halves: O = w0 O_0 + w1 O_1 with w_g = 2^(m_g - m) / l,
        // m the larger max and l = l_0 2^(m_0 - m) + l_1 2^(m_1 - m)
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::bSA), (uint32_t)i & 1u, ctl));
        if (!ok) break;
        const float2 a = stats[row];
        const float m = fmaxf(a.x, m_run);
        const float f0 = a.x == -INFINITY ? 0.0f : ex2(a.x - m);
        const float f1 = m_run == -INFINITY ? 0.0f : ex2(m_run - m);
        const float l = a.y * f0 + l_run * f1;
        const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
        stats[row] = make_float2(f0 * inv_l, f1 * inv_l);
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::bLF));
      }
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
      bool w = mbar_wait(bar(L::bOF + (i & 1)), (uint32_t)(i >> 1) & 1u, ctl);
      w = w && mbar_wait(bar(L::bLF), (uint32_t)i & 1u, ctl);
      ok = named_bar_and(1, kBlockM, w);  // the four warps leave together or not at all
      if (!ok) break;
      tc_fence_after();
      const float2 wgt = stats[row];
      const float2 w0 = make_float2(wgt.x, wgt.x), w1 = make_float2(wgt.y, wgt.y);
      const uint32_t tO0 = tlane + L::col_o(0, i), tO1 = tlane + L::col_o(1, i);
      // the output is staged in the brick's Q stage: all of its MMAs are complete
      const int qs = i % L::kQStages;
      uint8_t* stage = smem + L::kQ + qs * L::kTileBytes;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o0[32], o1[32];
        tmem_ld32(tO0 + c * 32, o0);
        tmem_ld32(tO1 + c * 32, o1);
        tmem_ld_wait();
        if (c == D / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(L::bOE + (i & 1)));
        }
        // 32 columns: half of a 64-column box, four 16-byte units of the swizzled row
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t w4[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const int k = 8 * u + 2 * x;
            const float2 v2 = __ffma2_rn(make_float2(o0[k], o0[k + 1]), w0,
                                         __fmul2_rn(make_float2(o1[k], o1[k + 1]), w1));
            w4[x] = pack_bf16x2(v2.x, v2.y);
          }
          const int uu = (c & 1) * 4 + u;
          *reinterpret_cast<uint4*>(stage + (c >> 1) * L::kBoxBytes + row * 128 +
                                    ((uu ^ (row & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1, kBlockM);
      if (leader) {
#pragma unroll
        for (int bx = 0; bx < L::kBoxes; ++bx)
          tma_store_5d(&tm_o, sbase + L::kQ + qs * L::kTileBytes + bx * L::kBoxBytes,
                       cur.h * D + bx * 64, cur.x0, cur.y0, cur.t0, cur.b);
        tma_store_commit();
        // the stage goes back to the producer once the store has read it
        tma_store_wait_read<0>();
        mbar_arrive(bar(L::bQE + qs));
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

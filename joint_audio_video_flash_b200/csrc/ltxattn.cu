// ltxattn.cu -- host side of the C ABI declared in include/ltxattn.h: argument
// validation, per-device context, TMA tensor maps, key-range split planning,
// workspace and kernel launches.  No CPU compute path exists: every step of the
// attention runs in the kernels of attn_fwd.cuh, attn_fwd_pp.cuh, attn_fwd_skv.cuh and
// combine.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <map>
#include <mutex>
#include <utility>

#include "../../include/ltxattn.h"
#include "combine.cuh"
#include "debug_guard.cuh"
#include "attn_fwd.cuh"
#include "attn_fwd_a2v.cuh"
#include "attn_fwd_pair.cuh"
#include "attn_fwd_pp.cuh"
#include "attn_fwd_skv.cuh"
#include "na3d_fwd.cuh"
#include "qk_prologue.cuh"

namespace {

using ltx::FwdParams;
using ltx::FwdSmem;

constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait
// query sides of at most this many 128-row tiles (head_dim 64, long key side) run the
// two-CTAs-per-SM variant of the base kernel
constexpr int kDualMaxQTiles = 1;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};

struct Context {
  int device = -1;
  int num_sms = 0;
  int* d_status = nullptr;
  EncodeTiledFn encode = nullptr;
  std::map<cudaStream_t, Workspace> workspaces;
  // held from a split call's workspace lookup through its launches: a grow on one host
  // thread (stream-ordered free of the old buffer, then a new one) can neither free a
  // buffer another thread has looked up but not yet launched on, nor race its bookkeeping
  std::mutex launch_mu;
};

std::mutex g_mu;
std::map<int, Context*> g_ctx;

const char* const kEntryPoints[] = {
    "ltxattn_create",        "ltxattn_forward",          "ltxattn_forward_ex",
    "ltxattn_check",         "ltxattn_destroy",          "ltxattn_status_string",
    "ltxattn_selftest_wait_timeout", "ltxattn_num_entry_points", "ltxattn_entry_point_name",
    "ltxattn_forward_split_noalloc", "ltxattn_qk_norm_rope", "ltxattn_na3d_forward",
    "ltxattn_forward_partial", "ltxattn_combine", "ltxattn_forward_grouped",
    "ltxattn_na3d_plan", "ltxattn_forward_plan",
};

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// All checks that need no CUDA call, in the order the header documents.
// The size rules of an attention call (no pointers).
int validate_sizes(int q_len, int kv_len, int kv_valid_len, int batch, int heads, int head_dim,
                   float scale) {
  if (q_len < 1 || kv_len < 1 || batch < 1 || heads < 1) return LTXATTN_ERR_INVALID_ARG;
  if (kv_valid_len < 1 || kv_valid_len > kv_len) return LTXATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.0f)) return LTXATTN_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return LTXATTN_ERR_UNSUPPORTED;
  if (q_len > LTXATTN_MAX_LEN || kv_len > LTXATTN_MAX_LEN || heads > LTXATTN_MAX_HEADS ||
      batch > LTXATTN_MAX_BATCH)
    return LTXATTN_ERR_UNSUPPORTED;
  return LTXATTN_OK;
}

int validate(const void* q, const void* k, const void* v, void* out, int q_len, int kv_len,
             int kv_valid_len, int batch, int heads, int head_dim, float scale) {
  if (!q || !k || !v || !out) return LTXATTN_ERR_INVALID_ARG;
  const int st = validate_sizes(q_len, kv_len, kv_valid_len, batch, heads, head_dim, scale);
  if (st != LTXATTN_OK) return st;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out);
  if (mis & 15u) return LTXATTN_ERR_MISALIGNED;
  const size_t row = (size_t)heads * head_dim * 2;
  const size_t nq = (size_t)batch * q_len * row, nkv = (size_t)batch * kv_len * row;
  if (overlaps(out, nq, q, nq) || overlaps(out, nq, k, nkv) || overlaps(out, nq, v, nkv))
    return LTXATTN_ERR_INVALID_ARG;
  return LTXATTN_OK;
}

// BSHD bf16 tensor [batch, len, heads, head_dim] seen as a 4-D TMA tensor
// (d, h, s, b) with a 64-column x 128-row box and the 128-byte swizzle.
bool encode_bshd(const Context& c, CUtensorMap* map, const void* base, int len, int batch,
                 int heads, int head_dim, int box_rows = ltx::kBlockM) {
  const cuuint64_t dims[4] = {(cuuint64_t)head_dim, (cuuint64_t)heads, (cuuint64_t)len,
                              (cuuint64_t)batch};
  const cuuint64_t strides[3] = {(cuuint64_t)head_dim * 2, (cuuint64_t)heads * head_dim * 2,
                                 (cuuint64_t)len * heads * head_dim * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  // L2 fetch granule = one (token, head) row: a 256-byte promotion of a 128-byte row
  // would also fetch the next head's row, which a head-ordered walk reads much later
  const CUtensorMapL2promotion promo =
      head_dim * 2 >= 256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B;
  CUresult r = c.encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Key-range parts: enough (b, h, q-tile) x part CTAs to fill the SMs without
// over-splitting.  Cost model: waves x (tiles per part + fixed per-CTA overhead).
int plan_splits(int units, int n_kv_tiles, int num_sms) {
  if (n_kv_tiles < 4 || units >= num_sms) return 1;
  const int kOverheadTiles = 4;  // pipeline fill + partial write-out, in key tiles (measured)
  int best = 1;
  long long best_cost = -1;
  for (int s = 1; s <= std::min(n_kv_tiles, 64); ++s) {
    const long long waves = ((long long)units * s + num_sms - 1) / num_sms;
    const long long cost = waves * ((n_kv_tiles + s - 1) / s + kOverheadTiles);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

Context* current_context(int* err) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    *err = LTXATTN_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_ctx.find(dev);
  if (it == g_ctx.end()) {
    *err = LTXATTN_ERR_NOT_INITIALIZED;
    return nullptr;
  }
  *err = LTXATTN_OK;
  return it->second;
}

template <int D, bool kSplit, int kSBuf = 2>
cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const FwdParams& p, cudaStream_t stream) {
  dim3 grid(p.n_q_tiles, p.heads, p.batch * p.num_splits);
  ltx::ltx_attn_fwd<D, kSplit, kSBuf>
      <<<grid, FwdSmem<D, kSBuf>::kThreads, FwdSmem<D, kSBuf>::kAlloc, stream>>>(tq, tk, tv, to, p);
  return cudaGetLastError();
}

// Two query tiles per CTA (query sides of more than one 128-row tile).
template <int D, bool kSplit>
cudaError_t launch_fwd_pp(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& to, const FwdParams& p, cudaStream_t stream) {
  dim3 grid((p.n_q_tiles + 1) / 2, p.heads, p.batch * p.num_splits);
  ltx::ltx_attn_fwd_pp<D, kSplit><<<grid, ltx::kPPThreads, ltx::PPSmem<D>::kAlloc, stream>>>(
      tq, tk, tv, to, p);
  return cudaGetLastError();
}

template <int D, bool kSplit>
cudaError_t launch_attention(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, const FwdParams& p, cudaStream_t stream) {
  return p.n_q_tiles >= 2 ? launch_fwd_pp<D, kSplit>(tq, tk, tv, to, p, stream)
                          : launch_fwd<D, kSplit>(tq, tk, tv, to, p, stream);
}

// Short key side (every valid key in at most two 128-key tiles) with more query tiles
// than SMs: persistent CTAs, one per SM, each walking a contiguous run of query tiles.
// With at most one tile per SM (audio self-attention) the one-tile CTAs of the base
// kernels start faster.
bool use_short_kv(const FwdParams& p, int num_sms) {
  return p.num_splits == 1 && p.n_kv_tiles <= ltx::kSkvMaxKvTiles &&
         (long long)p.batch * p.heads * p.n_q_tiles > num_sms;
}

template <int D, int NKV>
cudaError_t launch_skv_n(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& to, const FwdParams& p, int grid,
                         cudaStream_t stream) {
  ltx::ltx_attn_fwd_skv<D, NKV>
      <<<grid, ltx::kSkvThreads, ltx::SkvSmem<D, NKV>::kAlloc, stream>>>(tq, tk, tv,
                                                                                 to, p);
  return cudaGetLastError();
}

// Appends a call (its maps and sizes) to a group of the a2v kernel.
void a2v_append(ltx::A2vArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                const CUtensorMap& tv, const CUtensorMap& to, const FwdParams& p) {
  const int j = a.n_problems++;
  a.q[j] = tq;
  a.k[j] = tk;
  a.v[j] = tv;
  a.o[j] = to;
  ltx::A2vProblem& pr = a.prob[j];
  pr.batch = p.batch;
  pr.heads = p.heads;
  pr.n_q_tiles = p.n_q_tiles;
  pr.kv_valid = p.kv_valid;
  pr.scale_log2 = p.scale_log2;
  pr.first_unit = a.total_units;
  a.total_units += (long long)p.batch * p.heads * p.n_q_tiles;
  a.status = p.status;
  a.timeout_ns = p.timeout_ns;
}

// One persistent CTA per SM (fewer with fewer units) over every unit of the group.
cudaError_t launch_a2v(const ltx::A2vArgs& a, int num_sms, cudaStream_t stream) {
  const int grid = (int)std::min<long long>(a.total_units, num_sms);
  ltx::ltx_attn_fwd_a2v<<<grid, ltx::kA2vThreads, ltx::A2vSmem::kAlloc, stream>>>(a);
  return cudaGetLastError();
}

// Calls the a2v kernel takes (alone or grouped): head_dim 64, every valid key in one tile,
// no key split.
bool a2v_eligible(const FwdParams& p, int head_dim) {
  return head_dim == 64 && p.n_kv_tiles == 1 && p.num_splits == 1;
}

cudaError_t launch_skv(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const FwdParams& p, int head_dim, int num_sms,
                       cudaStream_t stream) {
  const long long total = (long long)p.batch * p.heads * p.n_q_tiles;
  const int grid = (int)std::min<long long>(total, num_sms);
  // head_dim 64, one key tile (a2v): per-unit K/V and the strided (batch, query tile, head)
  // walk, two softmax warpgroups and an epilogue warpgroup
  if (a2v_eligible(p, head_dim)) {
    ltx::A2vArgs a{};
    a2v_append(a, tq, tk, tv, to, p);
    return launch_a2v(a, num_sms, stream);
  }
  if (head_dim == 64) return launch_skv_n<64, 2>(tq, tk, tv, to, p, grid, stream);
  return p.n_kv_tiles == 1 ? launch_skv_n<128, 1>(tq, tk, tv, to, p, grid, stream)
                           : launch_skv_n<128, 2>(tq, tk, tv, to, p, grid, stream);
}

template <int D>
cudaError_t launch_combine(const FwdParams& p, void* out, cudaStream_t stream) {
  const long long total = (long long)p.batch * p.q_len * p.heads * (D / 4);
  const long long blocks = (total + ltx::kCombineThreads - 1) / ltx::kCombineThreads;
  ltx::ltx_attn_combine<D><<<(unsigned)blocks, ltx::kCombineThreads, 0, stream>>>(
      p.o_part, p.lse_part, reinterpret_cast<__nv_bfloat16*>(out), p.num_splits, p.batch, p.heads,
      p.q_len, p.n_q_tiles * ltx::kBlockM);
  return cudaGetLastError();
}

cudaError_t set_smem_limits_dual() {
  cudaError_t e = cudaFuncSetAttribute(ltx::ltx_attn_fwd<64, true, 1>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       FwdSmem<64, 1>::kAlloc);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(ltx::ltx_attn_fwd<64, false, 1>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, FwdSmem<64, 1>::kAlloc);
}

template <int D>
cudaError_t set_smem_limits() {
  cudaError_t e = cudaFuncSetAttribute(ltx::ltx_attn_fwd<D, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       FwdSmem<D>::kAlloc);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(ltx::ltx_attn_fwd<D, true>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, FwdSmem<D>::kAlloc);
}

template <int D>
cudaError_t set_smem_limits_pp() {
  cudaError_t e = cudaFuncSetAttribute(ltx::ltx_attn_fwd_pp<D, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       ltx::PPSmem<D>::kAlloc);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(ltx::ltx_attn_fwd_pp<D, true>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              ltx::PPSmem<D>::kAlloc);
}

template <int D, int NKV>
cudaError_t set_smem_limit_skv() {
  return cudaFuncSetAttribute(ltx::ltx_attn_fwd_skv<D, NKV>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              ltx::SkvSmem<D, NKV>::kAlloc);
}

cudaError_t set_smem_limits_skv() {
  cudaError_t e = set_smem_limit_skv<64, 2>();
  if (e == cudaSuccess) e = set_smem_limit_skv<128, 1>();
  if (e == cudaSuccess) e = set_smem_limit_skv<128, 2>();
  return e;
}

__global__ void ltx_wait_probe(int* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ltx::mbar_init(ltx::smem_u32(&bar), 1);
    abort_flag = 0;
    ltx::fence_mbar_init();
  }
  __syncthreads();
  const ltx::WaitCtl ctl{&abort_flag, status, timeout_ns};
  // nothing ever arrives on the barrier, so phase 0 never completes
  if (threadIdx.x == 0) ltx::mbar_wait(ltx::smem_u32(&bar), 0, ctl);
  __syncthreads();
}

// Status word of the allocation-free path on device `dev` (defined with that path below):
// synchronises `stream`, reads the word and clears it; *ready is false (and nothing is
// read) when that path was never set up on the device.
int noalloc_take_status(int dev, cudaStream_t stream, bool* ready);

int read_and_clear_status(Context* c, cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) {
    cudaGetLastError();
    return LTXATTN_ERR_CUDA;
  }
  int h = 0;
  if (cudaMemcpy(&h, c->d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LTXATTN_ERR_CUDA;
  if (h != ltx::kDevOk) {
    if (cudaMemset(c->d_status, 0, sizeof(int)) != cudaSuccess) return LTXATTN_ERR_CUDA;
    return h == ltx::kDevGuard ? LTXATTN_ERR_WORKSPACE_GUARD : LTXATTN_ERR_DEVICE_TIMEOUT;
  }
  return LTXATTN_OK;
}

// Persistent grid of the prologue: as many CTAs as fit on the device at once (looked up
// once per device and kernel), fewer when there are fewer row groups.  MIN_CTAS caps the
// registers: 3 CTAs an SM (80 registers) streamed faster at 1024 and 8192 channels, 2 CTAs
// (128 registers) at 512, 2048 and 4096, on B200.
template <int CHUNKS, int WPR, int MIN_CTAS>
int launch_prologue(const ltx::PrologueParams& p, cudaStream_t stream) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static int resident[kMaxDevices];  // CTAs resident on the whole device; 0 = not looked up
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return LTXATTN_ERR_CUDA;
  }
  int ctas = 0;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (resident[dev] == 0) {
      int sms = 0, per_sm = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
          cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ltx::ltx_qk_norm_rope<CHUNKS, WPR, MIN_CTAS>,
                                                        ltx::kPrologueWarps * 32, 0) !=
              cudaSuccess ||
          sms < 1 || per_sm < 1) {
        cudaGetLastError();
        return LTXATTN_ERR_CUDA;
      }
      resident[dev] = sms * per_sm;
    }
    ctas = resident[dev];
  }
  constexpr int kRowsPerCta = ltx::PrologueRow<CHUNKS, WPR>::kRowsPerCta;
  const int groups = (2 * p.rows + kRowsPerCta - 1) / kRowsPerCta;
  const unsigned grid = (unsigned)std::min(groups, ctas);
  ltx::ltx_qk_norm_rope<CHUNKS, WPR, MIN_CTAS><<<grid, ltx::kPrologueWarps * 32, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? LTXATTN_OK : LTXATTN_ERR_CUDA;
}

// ---------------------------------------------------------------- neighbourhood attention
// Query brick (t x y x x = 128 tokens) and key tile (112 or 128 keys) shapes the kernel is
// built for; the host takes the pair whose bricks meet the fewest key tiles in total (a
// tile's MMAs do not depend on its width), of those the one with the fewest keys (K/V bytes
// and softmax work).  4 x 2 x 14 tiles cover the 4 x 14 x 14 key box of a 2 x 8 x 8 brick
// under a 3 x 7 x 7 window exactly: seven tiles of 112 keys instead of seven of 128.
struct NaShape {
  int bt, by, bx;  // query brick
  int kt, ky, kx;  // key tile
};
constexpr NaShape kNaShapes[] = {
    {2, 8, 8, 2, 8, 8}, {2, 8, 8, 4, 2, 16}, {1, 8, 16, 1, 8, 16},
    {1, 8, 16, 1, 16, 8}, {4, 4, 8, 4, 4, 8}, {4, 4, 8, 4, 2, 16},
    {2, 8, 8, 4, 2, 14},
};
constexpr int kNumNaShapes = (int)(sizeof(kNaShapes) / sizeof(kNaShapes[0]));

template <int D, int I>
cudaError_t na_set_smem() {
  constexpr NaShape s = kNaShapes[I];
  return cudaFuncSetAttribute(ltx::ltx_na3d_fwd<D, s.bt, s.by, s.bx, s.kt, s.ky, s.kx>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, ltx::NaSmem<D>::kAlloc);
}

template <int D, int... I>
cudaError_t na_set_smem_all(std::integer_sequence<int, I...>) {
  cudaError_t e = cudaSuccess;
  for (cudaError_t x : {na_set_smem<D, I>()...})
    if (x != cudaSuccess) e = x;
  return e;
}

cudaError_t set_smem_limits_na() {
  const cudaError_t a = na_set_smem_all<64>(std::make_integer_sequence<int, kNumNaShapes>{});
  const cudaError_t b = na_set_smem_all<128>(std::make_integer_sequence<int, kNumNaShapes>{});
  return a != cudaSuccess ? a : b;
}

// Key tiles met by all query bricks of one (batch, head): per axis the sum over bricks of
// the tiles covering their windows; the axes multiply.
long long na_tiles_total(const NaShape& b, int t, int y, int x, int kt, int ky, int kx) {
  auto axis = [](int n, int blk, int kblk, int k) {
    long long sum = 0;
    for (int a0 = 0; a0 < n; a0 += blk) {
      int r0, tiles;
      ltx::na_key_span(a0, blk, kblk, k, n, r0, tiles);
      sum += tiles;
    }
    return sum;
  };
  return axis(t, b.bt, b.kt, kt) * axis(y, b.by, b.ky, ky) * axis(x, b.bx, b.kx, kx);
}

// The shape pair (an index into kNaShapes) with the fewest key tiles over all bricks, then
// the fewest keys; its tile count per (batch, head) in *tiles when tiles is not null.
int na_pick(int t, int y, int x, int wt, int wy, int wx, long long* tiles) {
  int best = 0;
  long long best_keys = -1, best_tiles = -1;
  for (int i = 0; i < kNumNaShapes; ++i) {
    const NaShape& s = kNaShapes[i];
    const long long n = na_tiles_total(s, t, y, x, wt, wy, wx);
    const long long keys = n * (s.kt * s.ky * s.kx);
    if (best_tiles < 0 || n < best_tiles || (n == best_tiles && keys < best_keys)) {
      best_keys = keys;
      best_tiles = n;
      best = i;
    }
  }
  if (tiles) *tiles = best_tiles;
  return best;
}

// Grid and window rules of the neighbourhood entry points.
bool na_grid_ok(int grid_t, int grid_y, int grid_x, int window_t, int window_y, int window_x) {
  if (grid_t < 1 || grid_y < 1 || grid_x < 1) return false;
  const int grid_dims[3] = {grid_t, grid_y, grid_x}, win[3] = {window_t, window_y, window_x};
  for (int a = 0; a < 3; ++a)
    if (win[a] < 1 || win[a] % 2 == 0 || win[a] > grid_dims[a]) return false;
  return true;
}

// BSHD bf16 tensor over a T x Y x X grid, [batch, T*Y*X, heads, head_dim], seen as a 5-D
// TMA tensor (heads*head_dim, x, y, t, batch): a box is 64 columns of one head over a
// bt x by x bx brick of tokens, 128-byte swizzled.
bool encode_grid(const Context& c, CUtensorMap* map, const void* base, int batch, int t, int y,
                 int x, int heads, int head_dim, int bt, int by, int bx) {
  const cuuint64_t row = (cuuint64_t)heads * head_dim * 2;
  const cuuint64_t dims[5] = {(cuuint64_t)heads * head_dim, (cuuint64_t)x, (cuuint64_t)y,
                              (cuuint64_t)t, (cuuint64_t)batch};
  const cuuint64_t strides[4] = {row, row * x, row * x * y, row * x * y * t};
  const cuuint32_t box[5] = {64, (cuuint32_t)bx, (cuuint32_t)by, (cuuint32_t)bt, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUtensorMapL2promotion promo =
      head_dim * 2 >= 256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B;
  return c.encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int I>
cudaError_t launch_na_shape(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& to, const ltx::Na3dParams& p, int num_sms,
                            cudaStream_t stream) {
  constexpr NaShape s = kNaShapes[I];
  const long long total = (long long)p.batch * p.heads * p.bricks;
  const int grid = (int)std::min<long long>(total, num_sms);
  ltx::ltx_na3d_fwd<D, s.bt, s.by, s.bx, s.kt, s.ky, s.kx>
      <<<grid, ltx::kNaThreads, ltx::NaSmem<D>::kAlloc, stream>>>(tq, tk, tv, to, p);
  return cudaGetLastError();
}

// The instantiation for shape `shape` (an index into kNaShapes).
template <int D, int... I>
cudaError_t launch_na(int shape, const CUtensorMap& tq, const CUtensorMap& tk,
                      const CUtensorMap& tv, const CUtensorMap& to, const ltx::Na3dParams& p,
                      int num_sms, cudaStream_t stream, std::integer_sequence<int, I...>) {
  cudaError_t e = cudaErrorInvalidValue;
  ((shape == I ? (void)(e = launch_na_shape<D, I>(tq, tk, tv, to, p, num_sms, stream)) : (void)0),
   ...);
  return e;
}

// Rows of key-split partials: [splits][batch][heads][n_q_tiles * 128].
size_t partial_rows(const FwdParams& p) {
  return (size_t)p.num_splits * p.batch * p.heads * (size_t)p.n_q_tiles * ltx::kBlockM;
}

size_t partial_o_bytes(const FwdParams& p, int head_dim) {
  return partial_rows(p) * (size_t)head_dim * sizeof(float);
}

// Picks the kernel family and the key-range parts for a call whose sizes are already in
// `p`; fills p.num_splits and p.tiles_per_split.  num_splits = 0 plans (never above
// max_splits when that is > 0), >= 1 asks for that many parts (clamped to the key tiles).
// Returns true for the one-S-buffer, two-CTAs-per-SM variant (head_dim 64, one query tile,
// a key side longer than two tiles: v2a), whose CTA slots the planner counts twice.
bool plan_kernel(FwdParams& p, int head_dim, int num_splits, int num_sms, int max_splits) {
  const bool dual = head_dim == 64 && p.n_kv_tiles > ltx::kSkvMaxKvTiles &&
                    p.n_q_tiles <= kDualMaxQTiles;
  // CTAs per key-range part: the two-query-tile kernel takes query tiles in pairs
  const int q_ctas = (!dual && p.n_q_tiles >= 2) ? (p.n_q_tiles + 1) / 2 : p.n_q_tiles;
  const int units = q_ctas * p.heads * p.batch;
  int splits = num_splits > 0 ? std::min(num_splits, p.n_kv_tiles)
                              : plan_splits(units, p.n_kv_tiles, (dual ? 2 : 1) * num_sms);
  if (num_splits == 0 && max_splits > 0) splits = std::min(splits, max_splits);
  p.tiles_per_split = (p.n_kv_tiles + splits - 1) / splits;
  p.num_splits = (p.n_kv_tiles + p.tiles_per_split - 1) / p.tiles_per_split;  // no empty part
  return dual;
}

// Query sides of at least this many 128-row tiles at head_dim 128 (unsplit) run on CTA pairs.
constexpr int kPairMinQTiles = 8;

bool use_pair(const FwdParams& p, int head_dim, int num_sms) {
  return head_dim == 128 && p.num_splits == 1 && p.n_q_tiles >= kPairMinQTiles &&
         !use_short_kv(p, num_sms);
}

// Two CTAs per pair, four query tiles per pair; K is loaded in 64-key halves.
cudaError_t launch_pair(const CUtensorMap& tq, const CUtensorMap& tk_half, const CUtensorMap& tv,
                        const CUtensorMap& to, const FwdParams& p, cudaStream_t stream) {
  dim3 grid(2 * ((p.n_q_tiles + 3) / 4), p.heads, p.batch);
  ltx::ltx_attn_fwd_pair<<<grid, ltx::kPairThreads, ltx::PairSmem::kAlloc, stream>>>(
      tq, tk_half, tv, to, p);
  return cudaGetLastError();
}

// The attention kernel a planned call runs (the values of ltxattn_kernel).
int kernel_family(const FwdParams& p, int head_dim, bool dual, int num_sms) {
  if (use_pair(p, head_dim, num_sms)) return LTXATTN_KERNEL_PAIR;
  if (use_short_kv(p, num_sms))
    return a2v_eligible(p, head_dim) ? LTXATTN_KERNEL_A2V : LTXATTN_KERNEL_SHORT_KV;
  if (dual) return LTXATTN_KERNEL_ONE_TILE_DUAL;
  return p.n_q_tiles >= 2 ? LTXATTN_KERNEL_TWO_TILES : LTXATTN_KERNEL_ONE_TILE;
}

// Launches the planned kernel (and, with key-range parts, the merge into `out`).  `tk_half`
// is the key map with 64-row boxes, used by the pair kernel.
cudaError_t launch_planned(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& to, const FwdParams& p, int head_dim, bool dual,
                           int num_sms, void* out, cudaStream_t stream,
                           const CUtensorMap* tk_half = nullptr) {
  const bool split = p.num_splits > 1;
  const int family = kernel_family(p, head_dim, dual, num_sms);
  cudaError_t e;
  if (tk_half && family == LTXATTN_KERNEL_PAIR) {
    return launch_pair(tq, *tk_half, tv, to, p, stream);
  } else if (family == LTXATTN_KERNEL_A2V || family == LTXATTN_KERNEL_SHORT_KV) {
    return launch_skv(tq, tk, tv, to, p, head_dim, num_sms, stream);
  } else if (family == LTXATTN_KERNEL_ONE_TILE_DUAL) {
    e = split ? launch_fwd<64, true, 1>(tq, tk, tv, to, p, stream)
              : launch_fwd<64, false, 1>(tq, tk, tv, to, p, stream);
  } else if (head_dim == 64) {
    e = split ? launch_attention<64, true>(tq, tk, tv, to, p, stream)
              : launch_attention<64, false>(tq, tk, tv, to, p, stream);
  } else {
    e = split ? launch_attention<128, true>(tq, tk, tv, to, p, stream)
              : launch_attention<128, false>(tq, tk, tv, to, p, stream);
  }
  if (e == cudaSuccess && split)
    e = head_dim == 64 ? launch_combine<64>(p, out, stream) : launch_combine<128>(p, out, stream);
  return e;
}

#ifdef LTXATTN_DEBUG
// Checks the guard words and padded rows of the workspace of the split call just enqueued
// (p.o_part points just past the front guard).  LTXATTN_DEBUG_CORRUPT_GUARD=1 in the
// environment overwrites one byte of the back guard first, to exercise the detection.
cudaError_t debug_check_guards(const FwdParams& p, int head_dim, cudaStream_t stream) {
  const uint32_t* ws = reinterpret_cast<const uint32_t*>(
      reinterpret_cast<const char*>(p.o_part) - ltx::kGuardBytes);
  const char* corrupt = std::getenv("LTXATTN_DEBUG_CORRUPT_GUARD");
  if (corrupt && corrupt[0] == '1') {
    char* back = reinterpret_cast<char*>(p.lse_part) + partial_rows(p) * sizeof(float);
    cudaError_t e = cudaMemsetAsync(back + ltx::kGuardBytes - 1, 0x5A, 1, stream);
    if (e != cudaSuccess) return e;
  }
  ltx::ltx_debug_guard_check<<<256, 256, 0, stream>>>(ws, p.num_splits, p.batch, p.heads,
                                                      p.n_q_tiles * ltx::kBlockM, p.q_len,
                                                      head_dim, p.status);
  return cudaGetLastError();
}
#endif

// Shared-memory limits of every attention kernel on the current device.
cudaError_t set_smem_limits_all() {
  cudaError_t e = set_smem_limits<64>();
  if (e == cudaSuccess) e = set_smem_limits<128>();
  if (e == cudaSuccess) e = set_smem_limits_pp<64>();
  if (e == cudaSuccess) e = set_smem_limits_pp<128>();
  if (e == cudaSuccess) e = set_smem_limits_skv();
  if (e == cudaSuccess) e = set_smem_limits_dual();
  if (e == cudaSuccess) e = set_smem_limits_na();
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(ltx::ltx_attn_fwd_pair, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ltx::PairSmem::kAlloc);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(ltx::ltx_attn_fwd_a2v, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ltx::A2vSmem::kAlloc);
  return e;
}

// FwdParams of a validated call, before planning.
FwdParams call_params(const Context& c, int q_len, int kv_len, int kv_valid_len, int batch,
                      int heads, float scale) {
  FwdParams p{};
  p.q_len = q_len;
  p.kv_len = kv_len;
  p.kv_valid = kv_valid_len;
  p.heads = heads;
  p.batch = batch;
  p.n_q_tiles = (q_len + ltx::kBlockM - 1) / ltx::kBlockM;
  p.n_kv_tiles = (kv_valid_len + ltx::kBlockN - 1) / ltx::kBlockN;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = c.d_status;
  p.timeout_ns = kDefaultTimeoutNs;
  return p;
}

// One validated call on context `c`: plans it (num_splits as ltxattn_forward_ex takes it),
// takes the stream's workspace for key-range partials and enqueues the kernels.
int forward_one(Context* c, const void* q, const void* k, const void* v, void* out, int q_len,
                int kv_len, int kv_valid_len, int batch, int heads, int head_dim, float scale,
                int num_splits, int* splits_used, cudaStream_t stream) {
  FwdParams p = call_params(*c, q_len, kv_len, kv_valid_len, batch, heads, scale);
  const bool dual = plan_kernel(p, head_dim, num_splits, c->num_sms, 0);
  const int splits = p.num_splits;
  if ((long long)batch * splits > 65535) return LTXATTN_ERR_UNSUPPORTED;
  if (splits_used) *splits_used = splits;

  CUtensorMap tq, tk, tv, to, tk_half;
  if (!encode_bshd(*c, &tq, q, q_len, batch, heads, head_dim) ||
      !encode_bshd(*c, &tk, k, kv_len, batch, heads, head_dim) ||
      !encode_bshd(*c, &tv, v, kv_len, batch, heads, head_dim) ||
      !encode_bshd(*c, &to, out, q_len, batch, heads, head_dim) ||
      !encode_bshd(*c, &tk_half, k, kv_len, batch, heads, head_dim, ltx::kBlockN / 2))
    return LTXATTN_ERR_CUDA;

  std::unique_lock<std::mutex> launch_lock(c->launch_mu, std::defer_lock);
#ifdef LTXATTN_DEBUG
  const size_t guard = ltx::kGuardBytes;  // canary words before and after the partials
#else
  const size_t guard = 0;
#endif
  if (splits > 1) {
    const size_t o_bytes = partial_o_bytes(p, head_dim);
    const size_t need = o_bytes + partial_rows(p) * sizeof(float) + 2 * guard;
    launch_lock.lock();
    Workspace* ws;
    {
      std::lock_guard<std::mutex> lk(g_mu);
      ws = &c->workspaces[stream];
    }
    if (ws->bytes < need) {
      if (ws->ptr && cudaFreeAsync(ws->ptr, stream) != cudaSuccess) return LTXATTN_ERR_CUDA;
      ws->ptr = nullptr;
      ws->bytes = 0;
      if (cudaMallocAsync(&ws->ptr, need, stream) != cudaSuccess) {
        cudaGetLastError();
        return LTXATTN_ERR_CUDA;
      }
      ws->bytes = need;
    }
    p.o_part = reinterpret_cast<float*>(reinterpret_cast<char*>(ws->ptr) + guard);
    p.lse_part = reinterpret_cast<float*>(reinterpret_cast<char*>(ws->ptr) + guard + o_bytes);
#ifdef LTXATTN_DEBUG
    if (cudaMemsetAsync(ws->ptr, 0xA5, need, stream) != cudaSuccess) return LTXATTN_ERR_CUDA;
#endif
  }
  cudaError_t e =
      launch_planned(tq, tk, tv, to, p, head_dim, dual, c->num_sms, out, stream, &tk_half);
#ifdef LTXATTN_DEBUG
  if (e == cudaSuccess && splits > 1) e = debug_check_guards(p, head_dim, stream);
#endif
  return e == cudaSuccess ? LTXATTN_OK : LTXATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

int ltxattn_create(void) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LTXATTN_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_ctx.count(dev)) return LTXATTN_OK;
  Context* c = new Context();
  c->device = dev;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  bool ok = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, dev) ==
                cudaSuccess &&
            cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess && fn != nullptr;
  if (ok) {
    c->encode = reinterpret_cast<EncodeTiledFn>(fn);
    ok = cudaMalloc(&c->d_status, sizeof(int)) == cudaSuccess &&
         cudaMemset(c->d_status, 0, sizeof(int)) == cudaSuccess &&
         set_smem_limits_all() == cudaSuccess && cudaDeviceSynchronize() == cudaSuccess;
  }
  if (!ok) {
    cudaGetLastError();
    if (c->d_status) cudaFree(c->d_status);
    delete c;
    return LTXATTN_ERR_CUDA;
  }
  g_ctx[dev] = c;
  return LTXATTN_OK;
}

int ltxattn_forward_ex(const void* q, const void* k, const void* v, void* out, int q_len,
                       int kv_len, int kv_valid_len, int batch, int heads, int head_dim,
                       float scale, int num_splits, int* splits_used, ltxattn_stream_t stream_) {
  int st = validate(q, k, v, out, q_len, kv_len, kv_valid_len, batch, heads, head_dim, scale);
  if (st != LTXATTN_OK) return st;
  if (num_splits < 0) return LTXATTN_ERR_INVALID_ARG;
  Context* c = current_context(&st);
  if (!c) return st;
  return forward_one(c, q, k, v, out, q_len, kv_len, kv_valid_len, batch, heads, head_dim, scale,
                     num_splits, splits_used, reinterpret_cast<cudaStream_t>(stream_));
}

int ltxattn_forward_grouped(const ltxattn_call* calls, int n_calls, ltxattn_stream_t stream_) {
  if (!calls || n_calls < 1) return LTXATTN_ERR_INVALID_ARG;
  if (n_calls > LTXATTN_MAX_GROUP) return LTXATTN_ERR_UNSUPPORTED;
  for (int i = 0; i < n_calls; ++i) {
    const ltxattn_call& x = calls[i];
    const int st = validate(x.q, x.k, x.v, x.out, x.q_len, x.kv_len, x.kv_valid_len, x.batch,
                            x.heads, x.head_dim, x.scale);
    if (st != LTXATTN_OK) return st;
  }
  // no call's output may overlap another call's inputs or output
  for (int i = 0; i < n_calls; ++i) {
    const ltxattn_call& x = calls[i];
    const size_t nx = (size_t)x.batch * x.q_len * x.heads * x.head_dim * 2;
    for (int j = 0; j < n_calls; ++j) {
      if (j == i) continue;
      const ltxattn_call& y = calls[j];
      const size_t row = (size_t)y.heads * y.head_dim * 2;
      const size_t nq = (size_t)y.batch * y.q_len * row, nkv = (size_t)y.batch * y.kv_len * row;
      if (overlaps(x.out, nx, y.q, nq) || overlaps(x.out, nx, y.k, nkv) ||
          overlaps(x.out, nx, y.v, nkv) || overlaps(x.out, nx, y.out, nq))
        return LTXATTN_ERR_INVALID_ARG;
    }
  }
  int st;
  Context* c = current_context(&st);
  if (!c) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  // the calls the grouped kernel takes, launched after the others, largest first (measured
  // faster than small problems first: a2v ahead of audio self-attention)
  struct Grouped {
    long long units;
    int call;
  } grouped[LTXATTN_MAX_GROUP];
  int n_grouped = 0;
  for (int i = 0; i < n_calls; ++i) {
    const ltxattn_call& x = calls[i];
    FwdParams p = call_params(*c, x.q_len, x.kv_len, x.kv_valid_len, x.batch, x.heads, x.scale);
    plan_kernel(p, x.head_dim, 0, c->num_sms, 0);
    if (a2v_eligible(p, x.head_dim)) {
      grouped[n_grouped++] = {(long long)p.batch * p.heads * p.n_q_tiles, i};
      continue;
    }
    st = forward_one(c, x.q, x.k, x.v, x.out, x.q_len, x.kv_len, x.kv_valid_len, x.batch,
                     x.heads, x.head_dim, x.scale, 0, nullptr, stream);
    if (st != LTXATTN_OK) return st;
  }
  std::stable_sort(grouped, grouped + n_grouped,
                   [](const Grouped& x, const Grouped& y) { return x.units > y.units; });
  ltx::A2vArgs group{};
  for (int g = 0; g < n_grouped; ++g) {
    const ltxattn_call& x = calls[grouped[g].call];
    FwdParams p = call_params(*c, x.q_len, x.kv_len, x.kv_valid_len, x.batch, x.heads, x.scale);
    plan_kernel(p, x.head_dim, 0, c->num_sms, 0);
    CUtensorMap tq, tk, tv, to;
    if (!encode_bshd(*c, &tq, x.q, x.q_len, x.batch, x.heads, x.head_dim) ||
        !encode_bshd(*c, &tk, x.k, x.kv_len, x.batch, x.heads, x.head_dim) ||
        !encode_bshd(*c, &tv, x.v, x.kv_len, x.batch, x.heads, x.head_dim) ||
        !encode_bshd(*c, &to, x.out, x.q_len, x.batch, x.heads, x.head_dim))
      return LTXATTN_ERR_CUDA;
    a2v_append(group, tq, tk, tv, to, p);
    if (group.n_problems == ltx::kA2vMaxProblems) {
      if (launch_a2v(group, c->num_sms, stream) != cudaSuccess) return LTXATTN_ERR_CUDA;
      group = ltx::A2vArgs{};
    }
  }
  if (group.n_problems > 0 && launch_a2v(group, c->num_sms, stream) != cudaSuccess)
    return LTXATTN_ERR_CUDA;
  return LTXATTN_OK;
}

int ltxattn_forward(const void* q, const void* k, const void* v, void* out, int q_len, int kv_len,
                    int kv_valid_len, int batch, int heads, int head_dim, float scale,
                    ltxattn_stream_t stream) {
  return ltxattn_forward_ex(q, k, v, out, q_len, kv_len, kv_valid_len, batch, heads, head_dim,
                            scale, 0, nullptr, stream);
}

int ltxattn_check(ltxattn_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LTXATTN_ERR_CUDA;
  }
  int st;
  Context* c = current_context(&st);
  bool noalloc_ready = false;
  const int st_noalloc = noalloc_take_status(dev, stream, &noalloc_ready);
  if (!c && !noalloc_ready) return LTXATTN_ERR_NOT_INITIALIZED;
  const int st_ctx = c ? read_and_clear_status(c, stream) : LTXATTN_OK;
  for (int want : {(int)LTXATTN_ERR_CUDA, (int)LTXATTN_ERR_WORKSPACE_GUARD,
                   (int)LTXATTN_ERR_DEVICE_TIMEOUT})
    if (st_ctx == want || st_noalloc == want) return want;
  return LTXATTN_OK;
}

int ltxattn_destroy(void) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LTXATTN_ERR_CUDA;
  }
  Context* c = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_ctx.find(dev);
    if (it == g_ctx.end()) return LTXATTN_ERR_NOT_INITIALIZED;
    c = it->second;
    g_ctx.erase(it);
  }
  int st = LTXATTN_OK;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    st = LTXATTN_ERR_CUDA;
  } else {
    st = read_and_clear_status(c, nullptr);
  }
  for (auto& kv : c->workspaces)
    if (kv.second.ptr) cudaFree(kv.second.ptr);
  cudaFree(c->d_status);
  delete c;
  return st;
}

const char* ltxattn_status_string(int status) {
  switch (status) {
    case LTXATTN_OK: return "LTXATTN_OK";
    case LTXATTN_ERR_INVALID_ARG: return "LTXATTN_ERR_INVALID_ARG";
    case LTXATTN_ERR_UNSUPPORTED: return "LTXATTN_ERR_UNSUPPORTED";
    case LTXATTN_ERR_MISALIGNED: return "LTXATTN_ERR_MISALIGNED";
    case LTXATTN_ERR_CUDA: return "LTXATTN_ERR_CUDA";
    case LTXATTN_ERR_DEVICE_TIMEOUT: return "LTXATTN_ERR_DEVICE_TIMEOUT";
    case LTXATTN_ERR_NOT_INITIALIZED: return "LTXATTN_ERR_NOT_INITIALIZED";
    case LTXATTN_ERR_WORKSPACE_GUARD: return "LTXATTN_ERR_WORKSPACE_GUARD";
    default: return "LTXATTN_UNKNOWN_STATUS";
  }
}

int ltxattn_selftest_wait_timeout(unsigned long long timeout_ns, ltxattn_stream_t stream_) {
  if (timeout_ns < 1000ull || timeout_ns > 10000000000ull) return LTXATTN_ERR_INVALID_ARG;
  int st;
  Context* c = current_context(&st);
  if (!c) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  st = read_and_clear_status(c, stream);  // start from a clean word
  if (st == LTXATTN_ERR_CUDA) return st;
  ltx_wait_probe<<<1, 32, 0, stream>>>(c->d_status, timeout_ns);
  if (cudaGetLastError() != cudaSuccess) return LTXATTN_ERR_CUDA;
  return read_and_clear_status(c, stream);
}

int ltxattn_qk_norm_rope(const void* q, const void* k, void* q_out, void* k_out,
                         const void* q_weight, const void* k_weight, const float* cos_table,
                         const float* sin_table, int batch, int seq_len, int heads, int head_dim,
                         float eps, ltxattn_stream_t stream_) {
  const void* ptrs[8] = {q, k, q_out, k_out, q_weight, k_weight, cos_table, sin_table};
  for (const void* ptr : ptrs)
    if (!ptr) return LTXATTN_ERR_INVALID_ARG;
  if (batch < 1 || seq_len < 1 || heads < 1 || head_dim < 1) return LTXATTN_ERR_INVALID_ARG;
  if (!std::isfinite(eps) || eps < 0.0f) return LTXATTN_ERR_INVALID_ARG;
  if (seq_len > LTXATTN_MAX_LEN || batch > LTXATTN_MAX_BATCH || heads > LTXATTN_MAX_HEADS)
    return LTXATTN_ERR_UNSUPPORTED;
  const long long inner = (long long)heads * head_dim;
  if (head_dim % 8 != 0 ||
      (inner != 512 && inner != 1024 && inner != 2048 && inner != 4096 && inner != 8192))
    return LTXATTN_ERR_UNSUPPORTED;
  uintptr_t mis = 0;
  for (const void* ptr : ptrs) mis |= reinterpret_cast<uintptr_t>(ptr);
  if (mis & 15u) return LTXATTN_ERR_MISALIGNED;
  const size_t nbytes = (size_t)batch * seq_len * inner * 2;
  // each output may be its own input; no other overlap
  if ((q_out != q && overlaps(q_out, nbytes, q, nbytes)) || overlaps(q_out, nbytes, k, nbytes) ||
      (k_out != k && overlaps(k_out, nbytes, k, nbytes)) || overlaps(k_out, nbytes, q, nbytes) ||
      overlaps(q_out, nbytes, k_out, nbytes))
    return LTXATTN_ERR_INVALID_ARG;

  ltx::PrologueParams p{};
  p.x[0] = static_cast<const __nv_bfloat16*>(q);
  p.x[1] = static_cast<const __nv_bfloat16*>(k);
  p.out[0] = static_cast<__nv_bfloat16*>(q_out);
  p.out[1] = static_cast<__nv_bfloat16*>(k_out);
  p.w[0] = static_cast<const __nv_bfloat16*>(q_weight);
  p.w[1] = static_cast<const __nv_bfloat16*>(k_weight);
  p.cos_t = cos_table;
  p.sin_t = sin_table;
  if ((long long)batch * seq_len >= (1LL << 30)) return LTXATTN_ERR_UNSUPPORTED;
  p.rows = batch * seq_len;
  p.seq_len = seq_len;
  p.head_dim = head_dim;
  p.eps = eps;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  switch (inner) {
    case 512: return launch_prologue<2, 1, 2>(p, stream);
    case 1024: return launch_prologue<4, 1, 3>(p, stream);
    case 2048: return launch_prologue<4, 2, 2>(p, stream);
    case 4096: return launch_prologue<4, 4, 2>(p, stream);
    default: return launch_prologue<4, 8, 3>(p, stream);
  }
}

int ltxattn_na3d_forward(const void* q, const void* k, const void* v, void* out, int batch,
                         int grid_t, int grid_y, int grid_x, int heads, int head_dim,
                         int window_t, int window_y, int window_x, float scale,
                         ltxattn_stream_t stream_) {
  if (!q || !k || !v || !out) return LTXATTN_ERR_INVALID_ARG;
  if (batch < 1 || heads < 1 ||
      !na_grid_ok(grid_t, grid_y, grid_x, window_t, window_y, window_x))
    return LTXATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.0f)) return LTXATTN_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return LTXATTN_ERR_UNSUPPORTED;
  const long long tokens = (long long)grid_t * grid_y * grid_x;
  if (tokens > LTXATTN_MAX_LEN || heads > LTXATTN_MAX_HEADS || batch > LTXATTN_MAX_BATCH)
    return LTXATTN_ERR_UNSUPPORTED;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out);
  if (mis & 15u) return LTXATTN_ERR_MISALIGNED;
  const size_t bytes = (size_t)batch * tokens * heads * head_dim * 2;
  if (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes) ||
      overlaps(out, bytes, v, bytes))
    return LTXATTN_ERR_INVALID_ARG;
  int st;
  Context* c = current_context(&st);
  if (!c) return st;

  const int best = na_pick(grid_t, grid_y, grid_x, window_t, window_y, window_x, nullptr);
  const NaShape& sh = kNaShapes[best];
  ltx::Na3dParams p{};
  p.batch = batch;
  p.heads = heads;
  p.grid_t = grid_t;
  p.grid_y = grid_y;
  p.grid_x = grid_x;
  p.win_t = window_t;
  p.win_y = window_y;
  p.win_x = window_x;
  p.nb_t = (grid_t + sh.bt - 1) / sh.bt;
  p.nb_y = (grid_y + sh.by - 1) / sh.by;
  p.nb_x = (grid_x + sh.bx - 1) / sh.bx;
  p.bricks = p.nb_t * p.nb_y * p.nb_x;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = c->d_status;
  p.timeout_ns = kDefaultTimeoutNs;

  CUtensorMap tq, tk, tv, to;
  // queries and outputs move in query bricks, keys and values in key tiles
  const int gt = grid_t, gy = grid_y, gx = grid_x;
  if (!encode_grid(*c, &tq, q, batch, gt, gy, gx, heads, head_dim, sh.bt, sh.by, sh.bx) ||
      !encode_grid(*c, &tk, k, batch, gt, gy, gx, heads, head_dim, sh.kt, sh.ky, sh.kx) ||
      !encode_grid(*c, &tv, v, batch, gt, gy, gx, heads, head_dim, sh.kt, sh.ky, sh.kx) ||
      !encode_grid(*c, &to, out, batch, gt, gy, gx, heads, head_dim, sh.bt, sh.by, sh.bx))
    return LTXATTN_ERR_CUDA;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const auto shapes = std::make_integer_sequence<int, kNumNaShapes>{};
  const cudaError_t e =
      head_dim == 64 ? launch_na<64>(best, tq, tk, tv, to, p, c->num_sms, stream, shapes)
                     : launch_na<128>(best, tq, tk, tv, to, p, c->num_sms, stream, shapes);
  return e == cudaSuccess ? LTXATTN_OK : LTXATTN_ERR_CUDA;
}

int ltxattn_forward_plan(int q_len, int kv_len, int kv_valid_len, int batch, int heads,
                         int head_dim, int num_splits, int num_sms, int* kernel, int* parts) {
  if (!kernel || !parts || num_splits < 0 || num_sms < 1) return LTXATTN_ERR_INVALID_ARG;
  const int st = validate_sizes(q_len, kv_len, kv_valid_len, batch, heads, head_dim, 1.0f);
  if (st != LTXATTN_OK) return st;
  FwdParams p{};
  p.q_len = q_len;
  p.kv_len = kv_len;
  p.kv_valid = kv_valid_len;
  p.heads = heads;
  p.batch = batch;
  p.n_q_tiles = (q_len + ltx::kBlockM - 1) / ltx::kBlockM;
  p.n_kv_tiles = (kv_valid_len + ltx::kBlockN - 1) / ltx::kBlockN;
  const bool dual = plan_kernel(p, head_dim, num_splits, num_sms, 0);
  if ((long long)batch * p.num_splits > 65535) return LTXATTN_ERR_UNSUPPORTED;
  *kernel = kernel_family(p, head_dim, dual, num_sms);
  *parts = p.num_splits;
  return LTXATTN_OK;
}

int ltxattn_na3d_plan(int grid_t, int grid_y, int grid_x, int window_t, int window_y,
                      int window_x, int* shape, long long* tiles) {
  if (!shape || !tiles || !na_grid_ok(grid_t, grid_y, grid_x, window_t, window_y, window_x))
    return LTXATTN_ERR_INVALID_ARG;
  const NaShape& s = kNaShapes[na_pick(grid_t, grid_y, grid_x, window_t, window_y, window_x,
                                       tiles)];
  const int v[6] = {s.bt, s.by, s.bx, s.kt, s.ky, s.kx};
  for (int i = 0; i < 6; ++i) shape[i] = v[i];
  return LTXATTN_OK;
}

int ltxattn_forward_partial(const void* q, const void* k, const void* v, float* o_part,
                            float* lse, int q_len, int kv_len, int kv_valid_len, int batch,
                            int heads, int head_dim, float scale, ltxattn_stream_t stream_) {
  if (!o_part || !lse) return LTXATTN_ERR_INVALID_ARG;
  // q, k, v and a stand-in for the bf16 output: the same checks as ltxattn_forward
  int st = validate(q, k, v, o_part, q_len, kv_len, kv_valid_len, batch, heads, head_dim, scale);
  if (st != LTXATTN_OK) return st;
  if (reinterpret_cast<uintptr_t>(lse) & 15u) return LTXATTN_ERR_MISALIGNED;
  const size_t rows_pad = (size_t)((q_len + ltx::kBlockM - 1) / ltx::kBlockM) * ltx::kBlockM;
  const size_t n_rows = (size_t)batch * heads * rows_pad;
  const size_t o_bytes = n_rows * head_dim * 4, l_bytes = n_rows * 4;
  const size_t row = (size_t)heads * head_dim * 2;
  const size_t nq = (size_t)batch * q_len * row, nkv = (size_t)batch * kv_len * row;
  if (overlaps(o_part, o_bytes, q, nq) || overlaps(o_part, o_bytes, k, nkv) ||
      overlaps(o_part, o_bytes, v, nkv) || overlaps(lse, l_bytes, q, nq) ||
      overlaps(lse, l_bytes, k, nkv) || overlaps(lse, l_bytes, v, nkv) ||
      overlaps(lse, l_bytes, o_part, o_bytes))
    return LTXATTN_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  Context* c = current_context(&st);
  if (!c) return st;

  FwdParams p{};
  p.q_len = q_len;
  p.kv_len = kv_len;
  p.kv_valid = kv_valid_len;
  p.heads = heads;
  p.batch = batch;
  p.n_q_tiles = (q_len + ltx::kBlockM - 1) / ltx::kBlockM;
  p.n_kv_tiles = (kv_valid_len + ltx::kBlockN - 1) / ltx::kBlockN;
  p.num_splits = 1;
  p.tiles_per_split = p.n_kv_tiles;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = c->d_status;
  p.timeout_ns = kDefaultTimeoutNs;
  p.o_part = o_part;
  p.lse_part = lse;
  // the output map is never stored through in split mode; q's map stands in for it
  CUtensorMap tq, tk, tv;
  if (!encode_bshd(*c, &tq, q, q_len, batch, heads, head_dim) ||
      !encode_bshd(*c, &tk, k, kv_len, batch, heads, head_dim) ||
      !encode_bshd(*c, &tv, v, kv_len, batch, heads, head_dim))
    return LTXATTN_ERR_CUDA;
  const bool dual = head_dim == 64 && p.n_kv_tiles > ltx::kSkvMaxKvTiles &&
                    p.n_q_tiles <= kDualMaxQTiles;
  cudaError_t e;
  if (dual)
    e = launch_fwd<64, true, 1>(tq, tk, tv, tq, p, stream);
  else if (head_dim == 64)
    e = launch_attention<64, true>(tq, tk, tv, tq, p, stream);
  else
    e = launch_attention<128, true>(tq, tk, tv, tq, p, stream);
  return e == cudaSuccess ? LTXATTN_OK : LTXATTN_ERR_CUDA;
}

int ltxattn_combine(const float* o_parts, const float* lses, void* out, int parts, int q_len,
                    int batch, int heads, int head_dim, ltxattn_stream_t stream_) {
  if (!o_parts || !lses || !out) return LTXATTN_ERR_INVALID_ARG;
  if (parts < 1 || q_len < 1 || batch < 1 || heads < 1) return LTXATTN_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return LTXATTN_ERR_UNSUPPORTED;
  if (q_len > LTXATTN_MAX_LEN || heads > LTXATTN_MAX_HEADS || batch > LTXATTN_MAX_BATCH ||
      parts > 65536)
    return LTXATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(o_parts) | reinterpret_cast<uintptr_t>(lses) |
       reinterpret_cast<uintptr_t>(out)) & 15u)
    return LTXATTN_ERR_MISALIGNED;
  FwdParams p{};
  p.q_len = q_len;
  p.heads = heads;
  p.batch = batch;
  p.n_q_tiles = (q_len + ltx::kBlockM - 1) / ltx::kBlockM;
  p.num_splits = parts;
  const size_t n_rows = (size_t)parts * batch * heads * p.n_q_tiles * ltx::kBlockM;
  const size_t out_bytes = (size_t)batch * q_len * heads * head_dim * 2;
  if (overlaps(out, out_bytes, o_parts, n_rows * head_dim * 4) ||
      overlaps(out, out_bytes, lses, n_rows * 4))
    return LTXATTN_ERR_INVALID_ARG;
  const long long blocks =
      ((long long)batch * q_len * heads * (head_dim / 4) + ltx::kCombineThreads - 1) /
      ltx::kCombineThreads;
  if (blocks > 0x7fffffffLL) return LTXATTN_ERR_UNSUPPORTED;
  p.o_part = const_cast<float*>(o_parts);
  p.lse_part = const_cast<float*>(lses);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const cudaError_t e = head_dim == 64 ? launch_combine<64>(p, out, stream)
                                       : launch_combine<128>(p, out, stream);
  return e == cudaSuccess ? LTXATTN_OK : LTXATTN_ERR_CUDA;
}

int ltxattn_num_entry_points(void) {
  return (int)(sizeof(kEntryPoints) / sizeof(kEntryPoints[0]));
}

const char* ltxattn_entry_point_name(int i) {
  if (i < 0 || i >= ltxattn_num_entry_points()) return nullptr;
  return kEntryPoints[i];
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free key-split forward (ltxattn_forward_split_noalloc).
//
// For callers that may not allocate device memory (a plugin host that owns all
// of it, a serving loop with a fixed memory plan that must not stall on an
// allocation's device-wide synchronisation, a hard memory quota), the key-split
// partials live in this file-scope device array instead of a cudaMalloc'd
// workspace.  Host code cannot use the array's name as a device address, so the
// first call on each device looks the address up with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[LTXATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kNoallocMaxDevices = 64;
constexpr size_t kNoallocStatusBytes = 256;  // status word at offset 0, partials after it

struct NoallocDevice {
  bool ready = false;
  unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch on this device
  int num_sms = 0;
};

std::mutex g_noalloc_mu;
NoallocDevice g_noalloc_dev[kNoallocMaxDevices];
EncodeTiledFn g_noalloc_encode = nullptr;

// Once per device, with that device current: scratch address, SM count, kernel
// shared-memory limits and the tensor-map encoder.  Allocates nothing.
int noalloc_setup(int dev, NoallocDevice** out) {
  if (dev < 0 || dev >= kNoallocMaxDevices) return LTXATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoallocDevice& d = g_noalloc_dev[dev];
  if (!d.ready) {
    void* sym = nullptr;
    if (cudaGetSymbolAddress(&sym, g_noalloc_scratch) != cudaSuccess || sym == nullptr) {
      cudaGetLastError();
      return LTXATTN_ERR_CUDA;
    }
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        set_smem_limits_all() != cudaSuccess) {
      cudaGetLastError();
      return LTXATTN_ERR_CUDA;
    }
    if (!g_noalloc_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr) {
        cudaGetLastError();
        return LTXATTN_ERR_CUDA;
      }
      g_noalloc_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.scratch = static_cast<unsigned char*>(sym);
    d.ready = true;
  }
  *out = &d;
  return LTXATTN_OK;
}

size_t noalloc_bytes(int splits, int batch, int heads, int n_q_tiles, int head_dim) {
  const size_t rows = (size_t)splits * batch * heads * (size_t)n_q_tiles * ltx::kBlockM;
  return kNoallocStatusBytes + rows * (size_t)(head_dim + 1) * sizeof(float);
}

int noalloc_take_status(int dev, cudaStream_t stream, bool* ready) {
  *ready = false;
  if (dev < 0 || dev >= kNoallocMaxDevices) return LTXATTN_OK;
  unsigned char* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_dev[dev].ready) return LTXATTN_OK;
    scratch = g_noalloc_dev[dev].scratch;
  }
  *ready = true;
  if (cudaStreamSynchronize(stream) != cudaSuccess) {
    cudaGetLastError();
    return LTXATTN_ERR_CUDA;
  }
  int h = 0;
  if (cudaMemcpy(&h, scratch, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return LTXATTN_ERR_CUDA;
  }
  if (h == ltx::kDevOk) return LTXATTN_OK;
  if (cudaMemset(scratch, 0, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return LTXATTN_ERR_CUDA;
  }
  return LTXATTN_ERR_DEVICE_TIMEOUT;
}

}  // namespace

extern "C" int ltxattn_forward_split_noalloc(const void* q, const void* k, const void* v,
                                             void* out, int q_len, int kv_len, int kv_valid_len,
                                             int batch, int heads, int head_dim, float scale,
                                             int num_splits, ltxattn_stream_t stream_) {
  int st = validate(q, k, v, out, q_len, kv_len, kv_valid_len, batch, heads, head_dim, scale);
  if (st != LTXATTN_OK) return st;
  if (num_splits < 0) return LTXATTN_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LTXATTN_ERR_CUDA;
  }
  NoallocDevice* d = nullptr;
  st = noalloc_setup(dev, &d);
  if (st != LTXATTN_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);

  FwdParams p{};
  p.q_len = q_len;
  p.kv_len = kv_len;
  p.kv_valid = kv_valid_len;
  p.heads = heads;
  p.batch = batch;
  p.n_q_tiles = (q_len + ltx::kBlockM - 1) / ltx::kBlockM;
  p.n_kv_tiles = (kv_valid_len + ltx::kBlockN - 1) / ltx::kBlockN;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = kDefaultTimeoutNs;

  // the most key-range parts whose partials fit in the scratch after the status word; one
  // part needs no partials at all (the kernel writes the bf16 output itself)
  const size_t per_split =
      (size_t)batch * heads * (size_t)p.n_q_tiles * ltx::kBlockM * (size_t)(head_dim + 1) * 4;
  const size_t fit = (LTXATTN_NOALLOC_SCRATCH_BYTES - kNoallocStatusBytes) / per_split;
  const int max_splits = (int)std::max<size_t>(1, std::min<size_t>(fit, 1 << 20));
  const bool dual = plan_kernel(p, head_dim, num_splits, d->num_sms, max_splits);
  const int splits = p.num_splits;
  if ((long long)batch * splits > 65535) return LTXATTN_ERR_UNSUPPORTED;
  if (splits > 1 && noalloc_bytes(splits, batch, heads, p.n_q_tiles, head_dim) >
                        LTXATTN_NOALLOC_SCRATCH_BYTES)
    return LTXATTN_ERR_UNSUPPORTED;  // the asked-for partials would not fit in the scratch

  p.status = reinterpret_cast<int*>(d->scratch);
  if (splits > 1) {
    p.o_part = reinterpret_cast<float*>(d->scratch + kNoallocStatusBytes);
    p.lse_part = p.o_part + partial_rows(p) * (size_t)head_dim;
  }

  Context c;  // tensor-map encoder only; nothing in it is allocated
  c.encode = g_noalloc_encode;
  CUtensorMap tq, tk, tv, to, tk_half;
  if (!encode_bshd(c, &tq, q, q_len, batch, heads, head_dim) ||
      !encode_bshd(c, &tk, k, kv_len, batch, heads, head_dim) ||
      !encode_bshd(c, &tv, v, kv_len, batch, heads, head_dim) ||
      !encode_bshd(c, &to, out, q_len, batch, heads, head_dim) ||
      !encode_bshd(c, &tk_half, k, kv_len, batch, heads, head_dim, ltx::kBlockN / 2))
    return LTXATTN_ERR_CUDA;

  // the status word is the one thing that must start at zero
  if (cudaMemsetAsync(p.status, 0, sizeof(int), stream) != cudaSuccess) {
    cudaGetLastError();
    return LTXATTN_ERR_CUDA;
  }
  const cudaError_t e =
      launch_planned(tq, tk, tv, to, p, head_dim, dual, d->num_sms, out, stream, &tk_half);
  return e == cudaSuccess ? LTXATTN_OK : LTXATTN_ERR_CUDA;
}

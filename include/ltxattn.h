/*
 * ltxattn.h -- C ABI of the B200 (sm_100a) attention library for the LTX-2 joint
 * audio-video diffusion transformer block.
 *
 * What is computed.  For every batch element b, head h and query row i:
 *     s_j = scale * sum_d q[b,i,h,d] * k[b,j,h,d]          for keys j < kv_valid_len
 *     o[b,i,h,:] = sum_j exp(s_j - max s) v[b,j,h,:] / sum_j exp(s_j - max s)
 * which covers the four attentions of a block: video self-attention over the
 * video latent tokens, audio self-attention over the (padded) audio tokens, v2a
 * (audio queries over video keys/values) and a2v (video queries over audio
 * keys/values), as described in "LTX-2: replicate audio stream across Ulysses
 * ranks by default" (TensorRT-LLM pull request 16228), Description.  Keys at
 * index >= kv_valid_len are masked out: the audio stream is zero-padded before
 * attention (same Description), and the padded keys must not contribute.
 *
 * Layout.  All four tensors are bf16, contiguous, BSHD:
 *     q, out : [batch, q_len,  heads, head_dim]
 *     k, v   : [batch, kv_len, heads, head_dim]
 * element (b, s, h, d) at ((b*len + s)*heads + h)*head_dim + d.  Queries and
 * keys share `heads` and `head_dim`.
 *
 * Precision.  bf16 inputs, fp32 accumulation (tensor-core MMAs into tensor
 * memory), fp32 softmax statistics, probabilities rounded to bf16 before the
 * P*V product, output rounded to bf16 (round to nearest even).
 *
 * Ownership.  The caller owns q, k, v and out (device memory) and the stream;
 * the library never frees them.  The library owns a per-device context (device
 * status word, tensor-map encoder) and per-stream workspace for key-range
 * partials, allocated in stream order on first need and released by
 * ltxattn_destroy.
 *
 * Threading.  Calls on one device may come from any host thread.  Calls on the
 * same stream are ordered by the stream; calls on different streams use separate
 * workspaces.  A call that needs the key-split workspace holds a per-device lock from
 * the workspace lookup (and any grow) through its launches, so host threads sharing a
 * stream never launch on a buffer another thread is replacing.  ltxattn_destroy must
 * not run concurrently with other calls on the same device.
 *
 * Debug build.  Compiled with -DLTXATTN_DEBUG (libltxattn_debug.so), a key-split call puts
 * canary guard words before and after its fp32 partials, fills the padded rows of every
 * partial slab with the canary too, and checks all of them on the device after the merge;
 * an overwritten word is recorded in the device status word and reported by ltxattn_check
 * as LTXATTN_ERR_WORKSPACE_GUARD.  The release build has none of this.
 *
 * Errors.  Every entry point returns an ltxattn_status.  Argument checks run on
 * the host, before any CUDA call and before anything is enqueued, so a rejected
 * call has no effect.  Compute calls are asynchronous on `stream` and never
 * synchronise.  A kernel that finds its pipeline stalled past the library's
 * wait limit records LTXATTN_ERR_DEVICE_TIMEOUT in the device status word and
 * returns instead of hanging; ltxattn_check reads (and clears) that word.
 */
#ifndef LTXATTN_H_
#define LTXATTN_H_

#if defined(__GNUC__)
#define LTXATTN_API __attribute__((visibility("default")))
#else
#define LTXATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
struct CUstream_st;
typedef struct CUstream_st* ltxattn_stream_t;

typedef enum {
  LTXATTN_OK = 0,
  LTXATTN_ERR_INVALID_ARG = 1,     /* null pointer, bad size, kv_valid_len outside [1, kv_len],
                                      non-finite or non-positive scale, out aliasing an input */
  LTXATTN_ERR_UNSUPPORTED = 2,     /* head_dim not in {64, 128}, or a size beyond the limits */
  LTXATTN_ERR_MISALIGNED = 3,      /* a tensor base address not 16-byte aligned */
  LTXATTN_ERR_CUDA = 4,            /* a CUDA runtime or driver call failed */
  LTXATTN_ERR_DEVICE_TIMEOUT = 5,  /* a kernel hit its wait limit (see ltxattn_check) */
  LTXATTN_ERR_NOT_INITIALIZED = 6, /* no context on the current device: call ltxattn_create */
  LTXATTN_ERR_WORKSPACE_GUARD = 7  /* LTXATTN_DEBUG builds only: a key-split call wrote outside
                                      its partial rows (a guard word or a padded row of the
                                      workspace was overwritten; see ltxattn_check) */
} ltxattn_status;

/* Largest sizes accepted (larger values give LTXATTN_ERR_UNSUPPORTED). */
#define LTXATTN_MAX_LEN (1 << 24)   /* q_len, kv_len */
#define LTXATTN_MAX_HEADS 1024
#define LTXATTN_MAX_BATCH 1024

/*
 * Creates the context for the CUDA device current on the calling thread:
 * device properties, a zeroed device status word and the kernels' shared-memory
 * limits.  Idempotent: a second call on the same device returns LTXATTN_OK.
 * Errors: LTXATTN_ERR_CUDA (no device, allocation or attribute failure).
 */
LTXATTN_API int ltxattn_create(void);

/*
 * Attention forward on the current device, enqueued on `stream`.
 *   q, k, v     device pointers, bf16 BSHD as above, 16-byte aligned.
 *   out         device pointer, bf16 BSHD [batch, q_len, heads, head_dim],
 *               16-byte aligned, not overlapping q, k or v.
 *   q_len       query rows, 1 .. LTXATTN_MAX_LEN.  Query rows beyond the real
 *               tokens (padding) are computed like any other row.
 *   kv_len      key/value rows, 1 .. LTXATTN_MAX_LEN.
 *   kv_valid_len  keys [0, kv_valid_len) take part; 1 <= kv_valid_len <= kv_len.
 *               Keys are staged in whole 128-row tiles, so the value rows of
 *               the last, partially valid tile beyond kv_valid_len are read
 *               (with zero weight): they must be finite (zero padding is).
 *   batch, heads  1 .. LTXATTN_MAX_BATCH, 1 .. LTXATTN_MAX_HEADS.
 *   head_dim    64 or 128.
 *   scale       softmax scale, finite and > 0 (typically 1/sqrt(head_dim)).
 *   stream      CUDA stream (NULL = default stream).
 * Returns LTXATTN_OK once the work is enqueued, or the first failing check:
 * INVALID_ARG, UNSUPPORTED, MISALIGNED (all before any CUDA call),
 * NOT_INITIALIZED, CUDA (launch or workspace failure).
 */
LTXATTN_API int ltxattn_forward(const void* q, const void* k, const void* v, void* out, int q_len, int kv_len,
                    int kv_valid_len, int batch, int heads, int head_dim, float scale,
                    ltxattn_stream_t stream);

/*
 * ltxattn_forward with an explicit plan.  num_splits = 0 lets the library choose
 * (as ltxattn_forward does); num_splits >= 1 asks for that many key-range parts
 * merged through their softmax statistics (clamped to the number of 128-key
 * tiles; 1 = no split).  If splits_used is not NULL it receives the number of
 * parts actually launched.  Same errors as ltxattn_forward, plus INVALID_ARG for
 * num_splits < 0.
 */
LTXATTN_API int ltxattn_forward_ex(const void* q, const void* k, const void* v, void* out, int q_len,
                       int kv_len, int kv_valid_len, int batch, int heads, int head_dim,
                       float scale, int num_splits, int* splits_used, ltxattn_stream_t stream);

/* One call of ltxattn_forward_grouped: the arguments of ltxattn_forward of the same names. */
typedef struct ltxattn_call {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  int q_len;
  int kv_len;
  int kv_valid_len;
  int batch;
  int heads;
  int head_dim;
  float scale;
} ltxattn_call;

/* Most calls one ltxattn_forward_grouped takes (more give LTXATTN_ERR_UNSUPPORTED). */
#define LTXATTN_MAX_GROUP 64

/*
 * Several independent attention calls in as few launches as possible.  An LTX-2 block runs
 * four attentions per step ("LTX-2: replicate audio stream across Ulysses ranks by
 * default", Description): two of them, a2v (video queries over the audio keys) and audio
 * self-attention, have every valid key in one 128-key tile at head_dim 64, and audio
 * self-attention is so small (one query tile per head) that its own launch costs more than
 * its work.  Here such calls (head_dim 64, kv_valid_len <= 128) share one persistent launch,
 * up to four per launch, their (batch, query tile, head) units walked as one sequence by all
 * SMs, the calls with the most units first; every other call runs as ltxattn_forward runs it,
 * in the order given, ahead of the shared launches (the calls are independent, so the order
 * does not change any result).
 *
 *   calls    host array of n_calls descriptors (read during the call only; the pointers in
 *            it are device pointers, as for ltxattn_forward)
 *   n_calls  1 .. LTXATTN_MAX_GROUP
 * Each call computes what ltxattn_forward computes (same arithmetic and precision; a grouped
 * call may run on another kernel than the same call alone, so results agree to rounding,
 * not bit for bit).  Every call is checked as ltxattn_forward checks it, and no call's `out`
 * may overlap another call's q, k, v or out (INVALID_ARG); all checks run before anything
 * is enqueued.  Needs ltxattn_create.  Asynchronous on `stream`; LTXATTN_ERR_CUDA on a
 * failed launch (calls before it stay enqueued); a kernel wait that times out is reported by
 * ltxattn_check.
 */
LTXATTN_API int ltxattn_forward_grouped(const ltxattn_call* calls, int n_calls,
                                        ltxattn_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device (LTXATTN_ERR_WORKSPACE_GUARD for a guard error in the debug
 * build): the context's word (ltxattn_create) and, if
 * ltxattn_forward_split_noalloc was ever called on this device, that call's own
 * word in its scratch array (read with a plain device-to-host copy; nothing is
 * allocated).  Returns LTXATTN_ERR_DEVICE_TIMEOUT if a kernel recorded a stalled
 * wait since the last check, LTXATTN_ERR_CUDA if the synchronisation or a copy
 * failed, LTXATTN_ERR_NOT_INITIALIZED when neither word exists on this device,
 * else LTXATTN_OK.
 */
LTXATTN_API int ltxattn_check(ltxattn_stream_t stream);

/*
 * Synchronises the current device, checks the status word (as ltxattn_check)
 * and frees the context and all workspaces of the current device.  Returns the
 * status check's result; LTXATTN_ERR_NOT_INITIALIZED without a context.
 */
LTXATTN_API int ltxattn_destroy(void);

/* Human-readable name of a status code (static storage; never NULL). */
LTXATTN_API const char* ltxattn_status_string(int status);

/*
 * Self-test of the failure path: launches one CTA that waits on a barrier no
 * one arrives at, with a wait limit of `timeout_ns` nanoseconds (1e3 .. 1e10),
 * then synchronises `stream` and returns what ltxattn_check returns
 * (LTXATTN_ERR_DEVICE_TIMEOUT when the bounded wait works).  The status word is
 * cleared afterwards, so later calls are unaffected.
 */
LTXATTN_API int ltxattn_selftest_wait_timeout(unsigned long long timeout_ns, ltxattn_stream_t stream);

/*
 * Norm and rotary step of the queries and keys ahead of attention, both tensors in one
 * launch.  The LTX-2.5 DiT attends with "normed and rotated" queries and keys and keeps
 * RoPE tables per latent grid ("feat(ltx2): tile-parallel video VAE and the two-stage
 * pipeline", commit "Onboard Lightricks LTX-2.5"); the pages fix neither the norm nor the
 * rotary layout, and this call computes the following reading.  For each tensor x (q or k),
 * batch element b and token l, over the token's whole inner dimension heads * head_dim:
 *     r = sqrt(mean_{h,d} x[b,l,h,d]^2 + eps),   y[h,d] = x[b,l,h,d] / r * weight[h*head_dim + d]
 * then within every head, for each pair of adjacent channels (2i, 2i+1):
 *     out[2i]   = y[2i] * cos[l,i] - y[2i+1] * sin[l,i]
 *     out[2i+1] = y[2i] * sin[l,i] + y[2i+1] * cos[l,i]
 * The tables carry the positional scheme (1-D or per-grid 3-D angles), so the caller owns it.
 *
 *   q, k          bf16 [batch, seq_len, heads, head_dim] (device), read
 *   q_out, k_out  bf16, same shape (device), written; each may be its own input (in place),
 *                 but must not otherwise overlap q, k or each other
 *   q_weight, k_weight  bf16 [heads * head_dim] (device)
 *   cos_table, sin_table  fp32 [seq_len, head_dim / 2] (device)
 *   heads * head_dim  one of 512, 1024, 2048, 4096, 8192 (UNSUPPORTED otherwise); head_dim a
 *                 multiple of 8
 *   eps           finite, >= 0
 *   batch * seq_len  below 2^30 (UNSUPPORTED otherwise)
 * Arithmetic in fp32, output rounded to bf16 (nearest even).  Needs no ltxattn_create.
 * Pointers must be 16-byte aligned (MISALIGNED).  Checks run on the host before any
 * CUDA call (INVALID_ARG, UNSUPPORTED, MISALIGNED); LTXATTN_ERR_CUDA on a failed launch.
 * Asynchronous on `stream`.
 */
LTXATTN_API int ltxattn_qk_norm_rope(const void* q, const void* k, void* q_out, void* k_out,
                                     const void* q_weight, const void* k_weight,
                                     const float* cos_table, const float* sin_table, int batch,
                                     int seq_len, int heads, int head_dim, float eps,
                                     ltxattn_stream_t stream);

/*
 * 3-D neighbourhood attention forward.  The LTX-2.5 diffusion decoder's stages attend
 * over 3-D neighbourhoods (NATTEN's fused na3d; "LTX2.5", SGLang Diffusion cookbook, §4.6
 * Diffusion decoder); the page gives no grid or window, and this call computes
 * Neighborhood Attention's definition in three dimensions, without dilation and not
 * causal.  Tokens sit on a grid_t x grid_y x grid_x grid in raster order, token
 * n = (t * grid_y + y) * grid_x + x.  Along an axis of length N with window k, the query
 * at position i sees the k positions starting at s(i) = min(max(i - (k-1)/2, 0), N - k)
 * (centred, shifted inward at the borders); a query attends to the box of its three
 * windows:
 *     out[b,n,h,:] = sum_{m in box(n)} softmax_m(scale * q[b,n,h,:] . k[b,m,h,:]) v[b,m,h,:]
 *
 *   q, k, v, out  bf16 [batch, grid_t * grid_y * grid_x, heads, head_dim], contiguous
 *                 (device); out must not overlap q, k or v
 *   window_*      odd, 1 <= window <= its grid axis (INVALID_ARG otherwise)
 *   head_dim      64 or 128 (UNSUPPORTED otherwise)
 *   grid_t * grid_y * grid_x <= LTXATTN_MAX_LEN; heads, batch as for ltxattn_forward
 *   scale         finite, > 0
 * Precision as ltxattn_forward: bf16 products, fp32 scores and statistics, P rounded to
 * bf16 before the PV product, output rounded to bf16.  Needs ltxattn_create on the
 * current device.  Pointers 16-byte aligned (MISALIGNED).  Host checks run before any
 * CUDA call; LTXATTN_ERR_CUDA on a failed launch; a kernel wait that times out is
 * reported by ltxattn_check.  Asynchronous on `stream`.
 */
LTXATTN_API int ltxattn_na3d_forward(const void* q, const void* k, const void* v, void* out,
                                     int batch, int grid_t, int grid_y, int grid_x, int heads,
                                     int head_dim, int window_t, int window_y, int window_x,
                                     float scale, ltxattn_stream_t stream);

/*
 * The blocking ltxattn_na3d_forward uses for a grid and window, on the host only (no
 * device, no ltxattn_create): of the query brick / key tile shape pairs the kernel is built
 * for, the one whose bricks meet the fewest key tiles in all, then the fewest keys.
 *   shape   host int[6]: the query brick (t, y, x), then the key tile (t, y, x); the brick
 *           holds 128 tokens, the key tile 112 or 128 keys
 *   tiles   host: key tiles per (batch, head), i.e. the 128-query x (key tile) products
 *           the tensor cores multiply per (batch, head)
 * Same grid and window rules as ltxattn_na3d_forward (LTXATTN_ERR_INVALID_ARG otherwise,
 * and also for null pointers); LTXATTN_OK with both outputs written.
 */
LTXATTN_API int ltxattn_na3d_plan(int grid_t, int grid_y, int grid_x, int window_t, int window_y,
                                  int window_x, int* shape, long long* tiles);

/* The attention kernels ltxattn_forward chooses between (ltxattn_forward_plan). */
typedef enum ltxattn_kernel {
  LTXATTN_KERNEL_ONE_TILE = 0,       /* one 128-row query tile per CTA, S double-buffered */
  LTXATTN_KERNEL_TWO_TILES = 1,      /* two query tiles per CTA, softmax ping-pong */
  LTXATTN_KERNEL_ONE_TILE_DUAL = 2,  /* head_dim 64, one query tile: two CTAs per SM */
  LTXATTN_KERNEL_SHORT_KV = 3,       /* persistent, every valid key in one or two tiles */
  LTXATTN_KERNEL_A2V = 4,            /* persistent, head_dim 64, one key tile (groupable) */
  LTXATTN_KERNEL_PAIR = 5            /* head_dim 128, CTA pairs (cta_group::2) */
} ltxattn_kernel;

/*
 * Which kernel ltxattn_forward (and ltxattn_forward_ex with `num_splits`) runs for a call of
 * these sizes on a GPU with `num_sms` SMs, and into how many key-range parts it splits the
 * keys (1 = no split; more = fp32 partials and a merge kernel), on the host only: no device,
 * no ltxattn_create.  Sizes follow ltxattn_forward's rules (INVALID_ARG / UNSUPPORTED as
 * there); num_splits >= 0; num_sms >= 1; kernel and parts are host pointers, written on
 * LTXATTN_OK.
 */
LTXATTN_API int ltxattn_forward_plan(int q_len, int kv_len, int kv_valid_len, int batch,
                                     int heads, int head_dim, int num_splits, int num_sms,
                                     int* kernel, int* parts);

/*
 * Attention over one key range, left unnormalised across ranges: the building block of
 * context-parallel attention, where each rank holds a shard of the keys and values and the
 * ranks exchange per-range results in fp32 with their softmax statistics ("feat(ltx2):
 * tile-parallel video VAE and the two-stage pipeline", commit "Onboard Lightricks LTX-2.5":
 * CP over ranks with an fp32 statistics all-gather).  For every (b, h) and query row i:
 *     o_part[b][h][i][:] = softmax_j(scale * q_i . k_j) v_j   over keys j < kv_valid_len
 *     lse[b][h][i]       = log2 sum_{j < kv_valid_len} exp(scale * q_i . k_j)
 * (base-2 log-sum-exp).  q, k, v as for ltxattn_forward (bf16 BSHD, device).
 *
 *   o_part  fp32 [batch][heads][rows_pad][head_dim] (device), rows_pad = ceil(q_len/128)*128;
 *           rows i >= q_len are not written
 *   lse     fp32 [batch][heads][rows_pad] (device)
 * Same argument rules as ltxattn_forward (o_part takes out's place in the checks); neither
 * output may overlap q, k, v or the other; 16-byte aligned.  Needs ltxattn_create.
 * Asynchronous on `stream`; LTXATTN_ERR_CUDA on a failed launch.
 */
LTXATTN_API int ltxattn_forward_partial(const void* q, const void* k, const void* v, float* o_part,
                                        float* lse, int q_len, int kv_len, int kv_valid_len,
                                        int batch, int heads, int head_dim, float scale,
                                        ltxattn_stream_t stream);

/*
 * Merge of `parts` results of ltxattn_forward_partial for the same queries over disjoint key
 * ranges into the attention over their union (same statistics merge):
 *     L = max_p lse_p,  w_p = 2^(lse_p - L),  out = sum_p w_p o_p / sum_p w_p   (fp32, then bf16)
 *
 *   o_parts  fp32 [parts][batch][heads][rows_pad][head_dim] (device), rows_pad as above
 *   lses     fp32 [parts][batch][heads][rows_pad] (device)
 *   out      bf16 [batch][q_len][heads][head_dim] (device), must not overlap the inputs
 * head_dim 64 or 128; 1 <= parts <= 65536; 16-byte aligned pointers.  Needs no ltxattn_create.
 * Asynchronous on `stream`.
 */
LTXATTN_API int ltxattn_combine(const float* o_parts, const float* lses, void* out, int parts,
                                int q_len, int batch, int heads, int head_dim,
                                ltxattn_stream_t stream);

/* Size of the library's built-in scratch array used by ltxattn_forward_split_noalloc. */
#define LTXATTN_NOALLOC_SCRATCH_BYTES (16u << 20) /* 16 MiB per GPU */

/*
 * Key-split attention forward that allocates no memory at all.  (The pages this
 * library follows have no counterpart to this call; it exists for embedding.)
 *
 * Some callers cannot let a library call cudaMalloc: a host framework or plugin
 * host that owns every byte of device memory and hands out none, a serving loop
 * that has fixed its memory plan at start-up and must not stall other streams on
 * the device-wide synchronisation an allocation can cause, or a process running
 * under a hard device-memory quota.  ltxattn_forward may allocate its key-split
 * workspace (and ltxattn_create allocates the status word); this call never does.
 * It needs no ltxattn_create.
 *
 * It computes what ltxattn_forward computes, with the same kernels.  When the key
 * side is split into ranges (v2a-like shapes), the per-part fp32 partial outputs
 * and base-2 log-sum-exps live in one array of LTXATTN_NOALLOC_SCRATCH_BYTES in
 * the library's own device memory (a static device array: every GPU that loads
 * the library holds it until the process exits) and the merge kernel writes
 * `out`; with one part the attention kernel writes `out` directly and only the
 * status word of the array is used.  The caller passes inputs and outputs as for
 * ltxattn_forward.
 *
 *   num_splits  0 = the library's plan, capped at the most parts whose partials
 *               fit (one part always fits); >= 1 = that many key-range parts
 *               (clamped to the number of 128-key tiles).
 *   Scratch use with splits > 1: 256 + splits * batch * heads *
 *               ceil(q_len/128)*128 * (head_dim + 1) * 4 bytes must not exceed
 *               LTXATTN_NOALLOC_SCRATCH_BYTES, else LTXATTN_ERR_UNSUPPORTED is
 *               returned and nothing is enqueued.
 *
 * The first call on each device sets up that device (the scratch array's device
 * address via cudaGetSymbolAddress, the kernels' shared-memory limits, the
 * tensor-map encoder); make that first call before any stream capture.
 * Every call shares the one array and it keeps the last call's contents.  Nothing
 * in it has to start at zero except the status word in its first 256 bytes, which
 * each call clears on `stream` before its kernels run; every partial the merge
 * reads is written earlier in the same call.  Calls whose GPU work overlaps (on
 * different streams, or from different host threads without ordering) race on the
 * array and give wrong results: order them.  A kernel wait that runs out is
 * recorded in that status word, which each call clears when it starts:
 * ltxattn_check (which needs no context for this word) reports it, so check after
 * the call whose result matters and before the next one.
 * Returns LTXATTN_OK once enqueued, or INVALID_ARG / UNSUPPORTED / MISALIGNED (as
 * ltxattn_forward, before any CUDA call), UNSUPPORTED when the scratch is too
 * small, LTXATTN_ERR_CUDA on a failed set-up or launch.
 */
LTXATTN_API int ltxattn_forward_split_noalloc(const void* q, const void* k, const void* v,
                                              void* out, int q_len, int kv_len, int kv_valid_len,
                                              int batch, int heads, int head_dim, float scale,
                                              int num_splits, ltxattn_stream_t stream);

/*
 * Number of entry points above, and their names, for loaders that check the
 * exported symbols.
 */
LTXATTN_API int ltxattn_num_entry_points(void);
LTXATTN_API const char* ltxattn_entry_point_name(int i);

#ifdef __cplusplus
}
#endif

#endif /* LTXATTN_H_ */

// debug_guard.cuh -- guard words of the key-split workspace in the LTXATTN_DEBUG build.
//
// In that build the workspace of a key-split call is laid out as
//     [front guard][o_part: parts x batch x heads x rows_pad x D fp32][lse: ... x rows_pad][back guard]
// and filled with a canary word before the split kernel runs.  The split kernels write only the
// rows q < q_len of every (part, batch, head) slab, and the merge reads only those, so after the
// merge both guards and every padded row (q_len <= q < rows_pad) must still hold the canary.  A
// check kernel reads them and records kDevGuard in the device status word when one does not; it
// never asserts or traps, so the context stays usable and ltxattn_check reports the error.
#pragma once

#include <stdint.h>

#include "sm100_ptx.cuh"

namespace ltx {

constexpr uint32_t kGuardWord = 0xA5A5A5A5u;  // the canary: every byte 0xA5
constexpr size_t kGuardBytes = 4096;          // each guard

// One thread per checked word: the two guards, then the padded rows of o_part, then those of lse.
__global__ void ltx_debug_guard_check(const uint32_t* __restrict__ ws, int parts, int batch,
                                      int heads, int rows_pad, int q_len, int head_dim,
                                      int* status) {
  constexpr long long kGuardWords = kGuardBytes / 4;
  const long long slabs = (long long)parts * batch * heads;
  const long long pad = rows_pad - q_len;
  const long long o_words = slabs * rows_pad * head_dim;  // whole o_part, in words
  const long long n_o_pad = slabs * pad * head_dim;
  const long long n_l_pad = slabs * pad;
  const long long total = 2 * kGuardWords + n_o_pad + n_l_pad;
  const uint32_t* o_part = ws + kGuardWords;
  const uint32_t* lse = o_part + o_words;
  const uint32_t* back = lse + slabs * rows_pad;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    uint32_t w;
    if (i < kGuardWords) {
      w = ws[i];
    } else if (i < 2 * kGuardWords) {
      w = back[i - kGuardWords];
    } else if (i < 2 * kGuardWords + n_o_pad) {
      const long long j = i - 2 * kGuardWords;
      const long long slab = j / (pad * head_dim), r = (j / head_dim) % pad, c = j % head_dim;
      w = o_part[(slab * rows_pad + q_len + r) * head_dim + c];
    } else {
      const long long j = i - 2 * kGuardWords - n_o_pad;
      w = lse[(j / pad) * rows_pad + q_len + j % pad];
    }
    if (w != kGuardWord) atomicCAS(status, kDevOk, kDevGuard);
  }
}

}  // namespace ltx

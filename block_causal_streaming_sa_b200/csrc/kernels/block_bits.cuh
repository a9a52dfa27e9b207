// Block-sparse attention: the caller's block mask (one byte per 128 x 128 block,
// nonzero = attended) packed into bit rows before the attention launch, so that
// the attention kernel's roles find a query tile's next flagged key tile with one
// word load and a find-first-set instead of reading one flag byte per key tile.
#pragma once

#include <cstdint>

#include "../sa_internal.h"

namespace sa {

struct BlockBitsParams {
  const uint8_t* mask;       // [rows][n_k] bytes, rows = B * H * n_q_tiles
  unsigned long long* bits;  // [rows][n_words]: bit k % 64 of word k / 64 = flag k;
                             // bits past n_k are zero
  long long rows;
  int n_k, n_words;          // n_words = ceil(n_k / 64)
  unsigned* status;          // device status word (checked build: kDevErrBounds)
  unsigned long long mask_bytes, bits_words;  // buffer sizes (checked build)
};

// One warp per mask row: each round reads 64 consecutive flag bytes (two coalesced
// 32-byte loads) and lane 0 stores the word their two ballots make.
__global__ void __launch_bounds__(256) block_bits_kernel(const BlockBitsParams p) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.rows) return;
  const uint8_t* m = p.mask + row * p.n_k;
  unsigned long long* out = p.bits + row * p.n_words;
  [[maybe_unused]] const unsigned long long m0 = static_cast<unsigned long long>(row) * p.n_k;
  for (int wd = 0; wd < p.n_words; ++wd) {
    const int k = wd * 64 + lane;
    const unsigned lo = __ballot_sync(
        0xffffffffu, k < p.n_k && SA_IN_BOUNDS(p.status, m0 + k + 1, p.mask_bytes) && m[k] != 0);
    const unsigned hi =
        __ballot_sync(0xffffffffu, k + 32 < p.n_k &&
                                       SA_IN_BOUNDS(p.status, m0 + k + 33, p.mask_bytes) &&
                                       m[k + 32] != 0);
    if (lane == 0 &&
        SA_IN_BOUNDS(p.status, static_cast<unsigned long long>(row) * p.n_words + wd + 1,
                     p.bits_words))
      out[wd] = (static_cast<unsigned long long>(hi) << 32) | lo;
  }
}

}  // namespace sa

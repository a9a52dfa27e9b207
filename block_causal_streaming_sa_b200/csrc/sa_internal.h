// Internal types shared by the host side (sa_api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "../../include/sa.h"

namespace sa {

constexpr int kMaxGroups = SA_MAX_ATTENDED;
constexpr int kMaxSplitSlots = 128;  // tail tiles that may be split (grids of up to 256 CTAs)

// Attention kernel variants: every attended key (dense), caller-flagged 128 x 128
// blocks (sparse), or dense plus a last key group of source frames each query row
// sees only its own frame of (frame-aligned editing).
constexpr int kModeDense = 0;
constexpr int kModeSparse = 1;
constexpr int kModeAligned = 2;

// Device status word bits (written with atomicOr, read by sa_get_status):
// a bounded wait ran out; a Q or K pair had a norm above the fp16 maximum, so
// its rotated values were saturated for the score MMA.
constexpr unsigned kDevErrTimeout = 1u;
constexpr unsigned kDevWarnSaturated = 2u;
constexpr unsigned kDevErrBounds = 4u;

// Device-side bounds checks of the checked build (libsa_checked.so, compiled
// with SA_DEVICE_CHECKS): before a kernel reads or writes global memory
// directly, SA_IN_BOUNDS(status, end, size) compares the end of the access (one
// past its last element) with the buffer's size; an access past the end sets
// kDevErrBounds in the status word and is skipped. The release build compiles
// every check to `true`. (TMA loads need none: the tensor maps carry the
// extents and fill out-of-range boxes with zeros.)
#ifdef SA_DEVICE_CHECKS
__device__ __forceinline__ bool in_bounds(unsigned* status, unsigned long long end,
                                          unsigned long long size) {
  if (end <= size) return true;
  atomicOr(status, kDevErrBounds);
  return false;
}
#define SA_IN_BOUNDS(status, end, size) ::sa::in_bounds((status), (end), (size))
#else
#define SA_IN_BOUNDS(status, end, size) true
#endif

// fp32 (cos, sin) tables of the three RoPE bands (reading: bands [t | h | w] of
// D - 4*(D/6), 2*(D/6), 2*(D/6) dims, pair i of a band of size d turned by
// pos * theta^(-2i/d)). Row = position, column = pair index in the band.
struct RopeTables {
  const float2* t;  // [ref_frames + (S + W) * F][dt2]
  const float2* h;  // [tok_h][dh2]
  const float2* w;  // [dw2][tok_w] (pair-major: a warp's rows are consecutive columns)
  int dt2, dh2, dw2;
  int tok_h, tok_w, frame_tokens;  // frame_tokens = tok_h * tok_w
};

// Rotate-and-transpose of one chunk (or the reference image): in [B, L, H, D]
// -> out [B, H, L_out, D] (planes of L_out >= L rows; rows L.. untouched).
// K rows (bf16) are turned by their in-chunk (frame, row, column) position and
// written as fp16; V rows (blockIdx.y == 1) are copied as bf16, or, with
// second_is_key, turned and written as fp16 like K (two key tensors at once).
struct AppendParams {
  const __nv_bfloat16* k_in;
  const __nv_bfloat16* v_in;  // may be null (K only)
  __nv_bfloat16* k_out;
  __nv_bfloat16* v_out;
  int B, L, H, D;
  int L_out;  // rows per output plane
  int second_is_key;
  RopeTables rope;
  unsigned* status;  // device status word (kDevWarnSaturated, kDevErrBounds)
  unsigned long long in_elems, out_elems;  // sizes of each input and output tensor
};

// One attended key group: the reference image first (if set), then the
// attended chunks in ascending chunk-id order.
struct AttendGroup {
  int src;      // 0: cache slot of the selected tier, 1: the chunk being generated,
                // 2: the reference image, 3: the source frames of the chunk being
                // generated (frame-aligned editing; always the last group)
  int slot;     // cache slot (src == 0)
  int t_delta;  // temporal base of the current chunk minus this group's, >= 0
  int len;      // number of keys
};

struct AttendParams {
  const __nv_bfloat16* q;        // [B, L, H, D] unrotated
  __nv_bfloat16* o;              // [B, L, H, D]
  float* lse;                    // [B, H, L] or null
  const __nv_bfloat16* cache;    // selected tier: [slot][K|V][B][H][L_plane][D]; K planes
                                 // hold fp16 keys rotated in-chunk, V planes bf16
  const __nv_bfloat16* k_cur;    // current chunk K (fp16 bits), rotated in-chunk:
                                 // [B][H][L_plane][D]; for frame-aligned editing the
                                 // source keys follow as a second [B][H][L_plane][D]
  const __nv_bfloat16* v_cur;    // current chunk V as passed: [B][L][H][D]
  const __nv_bfloat16* ref;      // reference image [K|V][B][H][L_ref][D] (K fp16) or null
  int B, L, H, D;                // L: query rows of the current chunk
  int L_plane;                   // rows per cache / key-scratch plane (F * tok_h * tok_w)
  int L_ref;                     // rows per reference plane
  int n_groups;
  AttendGroup groups[kMaxGroups];
  float scale_log2;  // softmax scale * log2(e)
  RopeTables rope;
  unsigned* status;
  // Block-sparse mode: the caller's [B][H][n_q_tiles][n_k_tiles] mask as bit rows,
  // row (b * H + h) * n_q_tiles + q of ceil(n_k_tiles / 64) words, bit k % 64 of
  // word k / 64 set when key tile k (over every attended group, in order) is
  // attended by query tile q. Null in the other modes.
  const unsigned long long* block_bits;
  // Split tail: when the last round of work tiles would leave most CTAs idle,
  // its tiles are split into two key-range halves; each half writes a
  // normalised fp32 partial row and its lse, and per row the second finisher
  // (atomic counter) merges both. Regions sized for kMaxSplitSlots tiles.
  float* split_o;    // [slot][query tile 0/1][half][D / 4][128 rows][4]
  float* split_lse;  // [slot][query tile][half][128 rows]
  int* split_sem;    // [slot][query tile][128 rows]: entry 32 w counts warp w of the rows; zero between launches
  int split_ok;
  // Buffer sizes for the checked build's bounds checks (elements): Q and O, lse,
  // bit-row words, split-tail rows; for the SIMT kernel the key sources too.
  unsigned long long q_elems, lse_elems, bits_words, split_rows;
  unsigned long long cache_elems, kcur_elems, ref_elems;
  int debug_stall_producer;  // test hook: 1 = the TMA producer issues nothing, so the
                             // MMA warp's bounded wait runs out (timeout path)
  // Clock record: per CTA (blockIdx.x < kMaxClockCtas) the global timer (ns) and
  // the SM cycle counter at its start and at its end, or null.
  unsigned long long* clock_stamps;  // [CTA][4]
};

constexpr int kMaxClockCtas = 1024;

}  // namespace sa

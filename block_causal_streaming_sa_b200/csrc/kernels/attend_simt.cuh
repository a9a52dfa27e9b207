// Plain fp32 SIMT attention over the reference image (if set) and the sink +
// window chunks: one warp per query row, lanes split the head dimension, exact
// exp2f, online softmax over the key groups in order. Reads the same cache layout as the tensor-core kernel
// and applies the same query-side relocated rotation (rounded to fp16 like the
// MMA operand), so it is an independent check of the tensor-core machinery.
// Debug path only: sa_debug_attend_simt.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../sa_internal.h"
#include "rope.cuh"

namespace sa {

template <int D>
__global__ void __launch_bounds__(256) attend_simt_kernel(AttendParams p) {
  constexpr int DPL = D / 32;  // dims per lane (4 or 2), whole RoPE pairs
  const int lane = threadIdx.x & 31;
  const long long row_id = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row_id >= static_cast<long long>(p.B) * p.H * p.L) return;
  const int l = static_cast<int>(row_id % p.L);
  const int bh = static_cast<int>(row_id / p.L);
  const int h = bh % p.H, b = bh / p.H;
  const int f = l / p.rope.frame_tokens;
  const int y = (l / p.rope.tok_w) % p.rope.tok_h;
  const int x = l % p.rope.tok_w;

  const size_t row_off = ((static_cast<size_t>(b) * p.L + l) * p.H + h) * D;
  const __nv_bfloat16* qrow = p.q + row_off;
  // checked build: the row of Q and O lies inside the tensors
  if (!SA_IN_BOUNDS(p.status, row_off + D, p.q_elems)) return;
  float qraw[DPL];
#pragma unroll
  for (int d = 0; d < DPL; ++d) qraw[d] = __bfloat162float(qrow[lane * DPL + d]);
  bool saturated = false;  // a pair above the fp16 maximum in norm (see rope.cuh)
#pragma unroll
  for (int d = 0; d < DPL; d += 2)
    saturated |= fmaf(qraw[d], qraw[d], qraw[d + 1] * qraw[d + 1]) > kF16MaxSq;
  if (saturated) atomicOr(p.status, kDevWarnSaturated);

  float m = -INFINITY, lsum = 0.f, acc[DPL];
#pragma unroll
  for (int d = 0; d < DPL; ++d) acc[d] = 0.f;

  const size_t plane = static_cast<size_t>(p.L_plane) * D;
  const size_t ref_plane = static_cast<size_t>(p.L_ref) * D;
  for (int g = 0; g < p.n_groups; ++g) {
    const AttendGroup grp = p.groups[g];
    float q[DPL];
#pragma unroll
    for (int pp = 0; pp < DPL / 2; ++pp) {
      const float2 cs = rope_cs(p.rope, lane * (DPL / 2) + pp, grp.t_delta + f, y, x);
      const float a = qraw[2 * pp], bb = qraw[2 * pp + 1];
      q[2 * pp] = __half2float(__float2half_rn(fmaf(a, cs.x, -bb * cs.y)));
      q[2 * pp + 1] = __half2float(__float2half_rn(fmaf(a, cs.y, bb * cs.x)));
    }
    const __nv_bfloat16 *kb, *vb;
    size_t vstride;
#ifdef SA_DEVICE_CHECKS
    const __nv_bfloat16* k_lo;  // the buffer the group's keys and values lie in
    unsigned long long k_size, v_size;
    const __nv_bfloat16* v_lo;
#endif
    if (grp.src == 0) {
      kb = p.cache + ((static_cast<size_t>(grp.slot) * 2 * p.B + b) * p.H + h) * plane;
      vb = p.cache + (((static_cast<size_t>(grp.slot) * 2 + 1) * p.B + b) * p.H + h) * plane;
      vstride = D;
    } else if (grp.src == 2) {
      kb = p.ref + (static_cast<size_t>(b) * p.H + h) * ref_plane;
      vb = p.ref + ((static_cast<size_t>(p.B) + b) * p.H + h) * ref_plane;
      vstride = D;
    } else {
      kb = p.k_cur + (static_cast<size_t>(b) * p.H + h) * plane;
      vb = p.v_cur + static_cast<size_t>(b) * p.L * p.H * D + static_cast<size_t>(h) * D;
      vstride = static_cast<size_t>(p.H) * D;
    }
#ifdef SA_DEVICE_CHECKS
    if (grp.src == 0) {
      k_lo = v_lo = p.cache;
      k_size = v_size = p.cache_elems;
    } else if (grp.src == 2) {
      k_lo = v_lo = p.ref;
      k_size = v_size = p.ref_elems;
    } else {
      k_lo = p.k_cur;
      k_size = p.kcur_elems;
      v_lo = p.v_cur;
      v_size = p.q_elems;
    }
    const unsigned long long k_end = static_cast<unsigned long long>(kb - k_lo) +
                                     static_cast<unsigned long long>(grp.len - 1) * D + D;
    const unsigned long long v_end = static_cast<unsigned long long>(vb - v_lo) +
                                     static_cast<unsigned long long>(grp.len - 1) * vstride + D;
    if (!SA_IN_BOUNDS(p.status, k_end, k_size) || !SA_IN_BOUNDS(p.status, v_end, v_size)) continue;
#endif
    for (int n = 0; n < grp.len; ++n) {
      const __nv_bfloat16* kr = kb + static_cast<size_t>(n) * D + lane * DPL;
      const __nv_bfloat16* vr = vb + static_cast<size_t>(n) * vstride + lane * DPL;
      float s = 0.f;
#pragma unroll
      for (int d = 0; d < DPL; ++d)
        s = fmaf(q[d], __half2float(reinterpret_cast<const __half*>(kr)[d]), s);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      const float s2 = s * p.scale_log2;
      const float mnew = fmaxf(m, s2);
      const float corr = exp2f(m - mnew);
      const float pv = exp2f(s2 - mnew);
      lsum = lsum * corr + pv;
#pragma unroll
      for (int d = 0; d < DPL; ++d) acc[d] = fmaf(pv, __bfloat162float(vr[d]), acc[d] * corr);
      m = mnew;
    }
  }
  __nv_bfloat16* orow = p.o + ((static_cast<size_t>(b) * p.L + l) * p.H + h) * D;
  const float inv = 1.f / lsum;
#pragma unroll
  for (int d = 0; d < DPL; ++d) orow[lane * DPL + d] = __float2bfloat16_rn(acc[d] * inv);
  const size_t lse_idx = (static_cast<size_t>(b) * p.H + h) * p.L + l;
  if (p.lse != nullptr && lane == 0 && SA_IN_BOUNDS(p.status, lse_idx + 1, p.lse_elems))
    p.lse[lse_idx] = (m + log2f(lsum)) * 0.69314718055994531f;
}

}  // namespace sa

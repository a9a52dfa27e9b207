// 3D RoPE helpers and the chunk rotate/transpose kernel used by the cache append.
//
// RoPE (abbreviation table of "Vidu S2：实时可交互、可编辑、可立体的视频生成":
// each token's position in space and in time) is applied with the band
// reading [t | h | w], pair (2i, 2i+1) of a band turned by pos * theta^(-2i/d).
//
// Keys enter the cache rotated by their IN-CHUNK position and stored as fp16
// (frame f within the chunk, row y, column x). The relocated temporal base
// base(j) of a cached chunk ("RoPE relocation", section 选择三 of "Vidu S2 vs
// PixVerse R2") changes as the window slides, so it is not baked in: rotating
// every key of chunk j by base(j) is, inside q . k, the same as turning q back by
// base(j), so a query at base(c) + f is turned by base(c) - base(j) + f, once per
// attended chunk, on the query side (the reference image has base 0).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "../sa_internal.h"
#include "ptx.cuh"

namespace sa {

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// (cos, sin) of pair `pair` (0 .. D/2-1) of a head vector at position (pos_t, y, x).
__device__ __forceinline__ float2 rope_cs(const RopeTables& rt, int pair, int pos_t, int y,
                                          int x) {
  if (pair < rt.dt2) return __ldg(&rt.t[pos_t * rt.dt2 + pair]);
  pair -= rt.dt2;
  if (pair < rt.dh2) return __ldg(&rt.h[y * rt.dh2 + pair]);
  pair -= rt.dh2;
  return __ldg(&rt.w[x * rt.dw2 + pair]);
}

// Turn one bf16 pair by (cos, sin) in fp32; the result is rounded once to fp16,
// the operand type of the score MMA (11 significant bits instead of bf16's 8).
__device__ __forceinline__ uint32_t rope_pair(uint32_t ab, float2 cs) {
  const float a = bf16_lo(ab), b = bf16_hi(ab);
  return ptx::pack_f16x2(fmaf(a, cs.x, -b * cs.y), fmaf(a, cs.y, b * cs.x));
}

// 65504^2 (exact in fp32): the squared largest finite fp16 value.
constexpr float kF16MaxSq = 4290774016.0f;

// True when one of the 4 bf16 pairs of a 16-byte chunk has a norm above 65504.
// A rotation keeps each pair's norm, and at some angle one value of the pair
// equals it, so such a pair saturates when rounded to fp16 for some position;
// the test does not depend on the position, so relocation cannot change it.
__device__ __forceinline__ bool pair_norm_exceeds_f16(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = bf16_lo(w[i]), b = bf16_hi(w[i]);
    m = fmaxf(m, fmaf(a, a, b * b));
  }
  return m > kF16MaxSq;
}

// Rotate the 8 bf16 values (4 pairs) of 16-byte chunk `c` of a head vector into
// 8 fp16 values.
__device__ __forceinline__ uint4 rope_chunk(uint4 v, int c, const RopeTables& rt, int pos_t, int y,
                                            int x) {
  v.x = rope_pair(v.x, rope_cs(rt, 4 * c + 0, pos_t, y, x));
  v.y = rope_pair(v.y, rope_cs(rt, 4 * c + 1, pos_t, y, x));
  v.z = rope_pair(v.z, rope_cs(rt, 4 * c + 2, pos_t, y, x));
  v.w = rope_pair(v.w, rope_cs(rt, 4 * c + 3, pos_t, y, x));
  return v;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// Rotate-and-transpose of whole frame rows. Block x covers tokens x0 .. x0 + XT - 1
// (x0 = segment * XT, clipped to the row) of one frame row (b, f, y), so the
// frame, the row and their RoPE table entries are per-block constants and a
// token's column is x0 + k: the per-token index arithmetic is an add, and only
// the column band's (cos, sin) is read per token. Thread t moves 16-byte chunk
// t % (D/8) of head t / (D/8) of every token of the segment; it issues the loads
// of all XT tokens before the first store, so enough bytes are in flight to
// cover HBM latency. blockIdx.y: 0 = K (bf16 in, rotated, fp16 out), 1 = V
// (bf16, copied; rotated like K when second_is_key). Loads are coalesced (a
// token's H*D values are contiguous); each head's 2*D bytes are stored
// contiguously into its [B, H, L_out, D] plane.
// Tokens per segment (measured on B200 at 720p: 4 and 8 tie, 16 is slower, and a
// persistent grid with the next segment's loads in flight was no faster).
constexpr int kRopeSegment = 4;

template <int XT>
__global__ void __launch_bounds__(XT >= 16 ? 512 : 1024) rope_transpose_kernel(AppendParams p) {
  const int vec_per_head = p.D >> 3;
  const int t = threadIdx.x;
  if (t >= p.H * vec_per_head) return;
  const bool is_v = blockIdx.y == 1;
  const __nv_bfloat16* in = is_v ? p.v_in : p.k_in;
  __nv_bfloat16* out = is_v ? p.v_out : p.k_out;
  if (in == nullptr) return;
  const RopeTables& rt = p.rope;
  const int n_seg = (rt.tok_w + XT - 1) / XT;
  const int row = blockIdx.x / n_seg;  // frame row over [B][L / tok_w]
  const int x0 = (blockIdx.x - row * n_seg) * XT;
  const int nx = min(XT, rt.tok_w - x0);
  const int rows_per_b = p.L / rt.tok_w;
  const int b = row / rows_per_b, fy = row - b * rows_per_b;
  const int h = t / vec_per_head, c = t - h * vec_per_head;
  const int l0 = fy * rt.tok_w + x0;
  const size_t hd = static_cast<size_t>(p.H) * p.D;
  const size_t src_off = (static_cast<size_t>(b) * p.L + l0) * hd + static_cast<size_t>(h) * p.D + c * 8;
  const size_t dst_off = ((static_cast<size_t>(b) * p.H + h) * p.L_out + l0) * p.D + c * 8;
  const __nv_bfloat16* src = in + src_off;
  __nv_bfloat16* dst = out + dst_off;
  uint4 v[XT];
#pragma unroll
  for (int k = 0; k < XT; ++k)
    if (k < nx && SA_IN_BOUNDS(p.status, src_off + k * hd + 8, p.in_elems))
      v[k] = ld_nc_v4(src + k * hd);
  if (is_v && !p.second_is_key) {
#pragma unroll
    for (int k = 0; k < XT; ++k)
      if (k < nx && SA_IN_BOUNDS(p.status, dst_off + k * p.D + 8, p.out_elems))
        st_v4(dst + k * p.D, v[k]);
    return;
  }
  // The 4 pairs of this thread's chunk: a temporal or row-band pair's (cos, sin)
  // is fixed for the block; a column-band pair's is read per token (wcol >= 0).
  const int f = fy / rt.tok_h, y = fy - f * rt.tok_h;
  float2 cs[4];
  int wcol[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    int pr = 4 * c + j;
    wcol[j] = -1;
    if (pr < rt.dt2) {
      cs[j] = __ldg(&rt.t[f * rt.dt2 + pr]);
    } else if ((pr -= rt.dt2) < rt.dh2) {
      cs[j] = __ldg(&rt.h[y * rt.dh2 + pr]);
    } else {
      wcol[j] = pr - rt.dh2;
      cs[j] = make_float2(1.f, 0.f);
    }
  }
  bool saturated = false;
#pragma unroll
  for (int k = 0; k < XT; ++k) {
    if (k >= nx) break;
    const int xo = (x0 + k) * rt.dw2;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (wcol[j] >= 0) cs[j] = __ldg(&rt.w[xo + wcol[j]]);
    saturated |= pair_norm_exceeds_f16(v[k]);
    uint4 r;
    r.x = rope_pair(v[k].x, cs[0]);
    r.y = rope_pair(v[k].y, cs[1]);
    r.z = rope_pair(v[k].z, cs[2]);
    r.w = rope_pair(v[k].w, cs[3]);
    if (SA_IN_BOUNDS(p.status, dst_off + k * p.D + 8, p.out_elems)) st_v4(dst + k * p.D, r);
  }
  if (saturated) atomicOr(p.status, kDevWarnSaturated);
}

}  // namespace sa

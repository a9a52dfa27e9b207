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
  return __ldg(&rt.w[pair * rt.tok_w + x]);
}

// The same with the band sizes of head dim D fixed at compile time (temporal
// D - 4 (D/6) dims, row and column D/3 each, as the handle's tables are built):
// with `pair` a constant after unrolling, each call is one load from a known
// table, so a row's loads are all issued back to back.
template <int D>
__device__ __forceinline__ float2 rope_cs_d(const RopeTables& rt, int pair, int pos_t, int y,
                                            int x) {
  constexpr int dt2 = (D - 4 * (D / 6)) / 2, dh2 = D / 6;
  if (pair < dt2) return __ldg(&rt.t[pos_t * dt2 + pair]);
  if (pair < dt2 + dh2) return __ldg(&rt.h[y * dh2 + (pair - dt2)]);
  return __ldg(&rt.w[(pair - dt2 - dh2) * rt.tok_w + x]);
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

// Rotate-and-transpose of [B, L, H, D] bf16 tokens into [B, H, L_out, D] head
// planes. blockIdx.y: 0 = K (bf16 in, rotated, fp16 out), 1 = V (bf16, copied;
// rotated like K when second_is_key). Block x covers XT tokens x0 .. x0 + XT - 1
// of one frame row (b, f, y); thread (k, c) moves 16-byte chunk c of token
// x0 + k for every head, HG heads at a time (the HG loads before the first
// store). A chunk's 4 (cos, sin) pairs depend on (f, y, x) and the chunk only,
// so a thread reads them once for all H heads (the table reads per byte moved
// fall by a factor H). Per head, a warp loads and stores whole 2*D-byte token
// rows. Measured on B200 against a head-parallel block (a thread per (head,
// chunk), 4 tokens a block): equal at 12 heads, 1.5x faster at 40 heads, where
// that block has 640 threads.
template <int D>
constexpr int kRopeTokens = 2048 / D;  // XT: 256 threads a block
constexpr int kRopeHeadGroup = 6;      // HG

template <int XT, int HG>
__global__ void __launch_bounds__(256) rope_transpose_kernel(AppendParams p) {
  const int vec_per_head = p.D >> 3;
  const int k = threadIdx.x / vec_per_head, c = threadIdx.x - k * vec_per_head;
  const bool is_v = blockIdx.y == 1;
  const __nv_bfloat16* in = is_v ? p.v_in : p.k_in;
  __nv_bfloat16* out = is_v ? p.v_out : p.k_out;
  if (in == nullptr || k >= XT) return;
  const RopeTables& rt = p.rope;
  const int n_seg = (rt.tok_w + XT - 1) / XT;
  const int row = blockIdx.x / n_seg;  // frame row over [B][L / tok_w]
  const int x = (blockIdx.x - row * n_seg) * XT + k;
  if (x >= rt.tok_w) return;
  const int rows_per_b = p.L / rt.tok_w;
  const int b = row / rows_per_b, fy = row - b * rows_per_b;
  const int l = fy * rt.tok_w + x;
  const size_t src_off = (static_cast<size_t>(b) * p.L + l) * p.H * p.D + c * 8;
  const size_t dst_off = (static_cast<size_t>(b) * p.H * p.L_out + l) * p.D + c * 8;
  const size_t dst_head = static_cast<size_t>(p.L_out) * p.D;  // one head plane
  const bool rotate = !is_v || p.second_is_key;
  float2 cs[4];
  if (rotate) {
    const int f = fy / rt.tok_h, y = fy - f * rt.tok_h;
#pragma unroll
    for (int j = 0; j < 4; ++j) cs[j] = rope_cs(rt, 4 * c + j, f, y, x);
  }
  bool saturated = false;
  for (int h0 = 0; h0 < p.H; h0 += HG) {
    uint4 v[HG];
#pragma unroll
    for (int g = 0; g < HG; ++g)
      if (h0 + g < p.H && SA_IN_BOUNDS(p.status, src_off + (h0 + g) * p.D + 8, p.in_elems))
        v[g] = ld_nc_v4(in + src_off + (h0 + g) * p.D);
#pragma unroll
    for (int g = 0; g < HG; ++g) {
      if (h0 + g >= p.H) break;
      uint4 r = v[g];
      if (rotate) {
        saturated |= pair_norm_exceeds_f16(v[g]);
        r.x = rope_pair(v[g].x, cs[0]);
        r.y = rope_pair(v[g].y, cs[1]);
        r.z = rope_pair(v[g].z, cs[2]);
        r.w = rope_pair(v[g].w, cs[3]);
      }
      const size_t o = dst_off + (h0 + g) * dst_head;
      if (SA_IN_BOUNDS(p.status, o + 8, p.out_elems)) st_v4(out + o, r);
    }
  }
  if (saturated) atomicOr(p.status, kDevWarnSaturated);
}

}  // namespace sa

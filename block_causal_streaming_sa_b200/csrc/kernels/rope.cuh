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

// Tokens per block of rope_transpose_kernel: each thread issues the loads of all
// of them before the first store, so enough bytes are in flight to cover HBM
// latency (one token per thread leaves the copy latency-bound at about half the
// bandwidth).
constexpr int kRopeTokensPerBlock = 4;

// Block x covers tokens (b, l) = kRopeTokensPerBlock * x .. + kRopeTokensPerBlock - 1
// of the flattened [B * L] index; thread t moves 16-byte chunk t % (D/8) of head
// t / (D/8) of each. blockIdx.y: 0 = K (bf16 in, rotated, fp16 out), 1 = V (bf16,
// copied; rotated like K when second_is_key). Loads are fully coalesced (a
// token's H*D values are contiguous); each head's 2*D bytes are stored
// contiguously into its [B, H, L_out, D] plane.
__global__ void rope_transpose_kernel(AppendParams p) {
  const int vec_per_head = p.D >> 3;
  const int t = threadIdx.x;
  if (t >= p.H * vec_per_head) return;
  const bool is_v = blockIdx.y == 1;
  const __nv_bfloat16* in = is_v ? p.v_in : p.k_in;
  __nv_bfloat16* out = is_v ? p.v_out : p.k_out;
  if (in == nullptr) return;
  const int h = t / vec_per_head, c = t - h * vec_per_head;
  const int n_tok = p.B * p.L;
  const int tok0 = blockIdx.x * kRopeTokensPerBlock;
  bool saturated = false;
  uint4 v[kRopeTokensPerBlock];
#pragma unroll
  for (int k = 0; k < kRopeTokensPerBlock; ++k) {
    const int tok = tok0 + k;
    if (tok < n_tok) v[k] = ld_nc_v4(in + (static_cast<size_t>(tok) * p.H + h) * p.D + c * 8);
  }
#pragma unroll
  for (int k = 0; k < kRopeTokensPerBlock; ++k) {
    const int tok = tok0 + k;
    if (tok >= n_tok) break;
    const int b = tok / p.L, l = tok - b * p.L;
    if (!is_v || p.second_is_key) {
      const int f = l / p.rope.frame_tokens;
      const int y = (l / p.rope.tok_w) % p.rope.tok_h;
      const int x = l % p.rope.tok_w;
      saturated |= pair_norm_exceeds_f16(v[k]);
      v[k] = rope_chunk(v[k], c, p.rope, f, y, x);
    }
    st_v4(out + ((static_cast<size_t>(b) * p.H + h) * p.L_out + l) * p.D + c * 8, v[k]);
  }
  if (saturated) atomicOr(p.status, kDevWarnSaturated);
}

}  // namespace sa

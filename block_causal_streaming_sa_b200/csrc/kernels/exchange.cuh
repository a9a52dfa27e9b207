// Pack / unpack kernels of the Ulysses all-to-all exchange with a quantised
// payload ("Vidu S2：实时可交互、可编辑、可立体的视频生成", section 2.4: Ulysses-style
// context parallelism across GPUs, with the exchanged tensors quantised to cut
// communication).
//
// pack: x [B, T, C, D] bf16 -> G blocks, one per destination rank. split 1
// (heads): block g holds heads g*C/G .. of every token; split 0 (tokens): block
// g holds tokens g*T/G .. with every head. Inside a block the vectors are in
// [B][T'][C'] order. fp8 payload: codes [B][T'][C'][D] e4m3, then, 16-byte
// aligned, one fp32 scale per vector; bf16 payload: the values as they are.
// With dst[], pack writes block g straight to dst[g]: for a peer's receive buffer
// mapped into this process (CUDA IPC over NVLink) the quantisation and the
// transfer are one pass, with no staging copy and no separate collective.
// unpack: the G blocks received (block s from rank s, each laid out as the
// sender's pack made it) -> y: split 1: [B][G*T'][C'][D] (token shards in rank
// order); split 0: [B][T'][G*C'][D] (head groups in rank order).
//
// fp8 (e4m3) with one scale per (b, t, c) vector: scale = max|x| / 448 and
// inv = 448 / max|x| (one IEEE fp32 division each per vector), code =
// e4m3(x * inv), nearest even and saturated; on arrival code * scale in fp32,
// rounded to bf16. Every operation is a single IEEE fp32 one (div.rn, mul.rn),
// so the codes do not depend on how a quotient is approximated.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "../sa_internal.h"
#include "ptx.cuh"
#include "rope.cuh"

namespace sa {

constexpr int kMaxExchangeRanks = 64;

struct ExchangeParams {
  const __nv_bfloat16* x;  // pack input
  const uint8_t* in;       // unpack input (G blocks)
  uint8_t* out;            // pack output (G blocks), or null with dst[]
  uint8_t* dst[kMaxExchangeRanks];  // pack output: where block g goes (e.g. a peer's
                                    // receive buffer mapped into this process)
  __nv_bfloat16* y;        // unpack output
  int B, T, C, D, G;       // the sender's x shape and the rank count
  int split;               // 0: tokens, 1: heads
  int fp8;                 // payload: 1 fp8 + scales, 0 bf16
  long long block_bytes;   // bytes of one block
  long long scale_off;     // offset of the scales inside a block (fp8)
};

constexpr float kE4m3Max = 448.0f;

// Block g and the vector index inside it of sender vector (b, t, c).
__device__ __forceinline__ void exchange_place(const ExchangeParams& p, int b, int t, int c,
                                               int& g, long long& v) {
  const int Tb = p.split == 0 ? p.T / p.G : p.T;
  const int Cb = p.split == 1 ? p.C / p.G : p.C;
  int tl = t, cl = c;
  if (p.split == 0) {
    g = t / Tb;
    tl = t - g * Tb;
  } else {
    g = c / Cb;
    cl = c - g * Cb;
  }
  v = (static_cast<long long>(b) * Tb + tl) * Cb + cl;
}

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float2 e4m3x2_to_f32(uint16_t v) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
  float2 f;
  asm("{\n\t.reg .f16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
      : "=f"(f.x), "=f"(f.y)
      : "r"(h));
  return f;
}

// Lanes per (b, t, c) vector: each lane moves 8 elements (16 bytes of bf16), so
// a warp holds 32 / kLanes<D> vectors at a time; every lane issues the loads of
// kExchangeSteps such groups before its first store, so enough bytes are in
// flight to cover memory latency.
template <int D>
constexpr int kLanes = D / 8;
constexpr int kExchangeSteps = 4;
template <int D, int S = kExchangeSteps>
constexpr int kExchangeVecPerWarp = (32 / kLanes<D>) * S;

// Advance a (b, t, c) position over [B][T][C] by `step` vectors (step >= 1).
__device__ __forceinline__ void exchange_step(int step, int C, int T, int& b, int& t, int& c) {
  c += step;
  while (c >= C) {
    c -= C;
    if (++t == T) {
      t = 0;
      ++b;
    }
  }
}

// kLanes<D> lanes per vector of x: the amax of a vector is reduced over its lanes
// by shuffles; lane 0 of the vector writes its scale.
template <int D, int S = kExchangeSteps>
__global__ void __launch_bounds__(256) exchange_pack_kernel(ExchangeParams p) {
  constexpr int LPV = kLanes<D>, VPW = 32 / LPV;
  const int lane = threadIdx.x & 31, sub = lane / LPV, sl = lane - sub * LPV;
  const long long n_vec = static_cast<long long>(p.B) * p.T * p.C;
  const long long base =
      (static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * kExchangeVecPerWarp<D, S>;
  uint4 w[S];
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const long long vec = base + s * VPW + sub;
    w[s] = vec < n_vec ? ld_nc_v4(p.x + vec * D + sl * 8) : make_uint4(0u, 0u, 0u, 0u);
  }
  // (b, t, c) of this lane's first vector once (64-bit division is a long
  // routine), then stepped
  int c = 0, t = 0, b = 0;
  if (base + sub < n_vec) {
    const long long vec = base + sub;
    c = static_cast<int>(vec % p.C);
    const long long bt = vec / p.C;
    t = static_cast<int>(bt % p.T);
    b = static_cast<int>(bt / p.T);
  }
#pragma unroll
  for (int s = 0; s < S; ++s) {
    if (s > 0) exchange_step(VPW, p.C, p.T, b, t, c);
    const bool active = base + s * VPW + sub < n_vec;
    int g = 0;
    long long v = 0;
    if (active) exchange_place(p, b, t, c, g, v);
    uint8_t* blk = p.out != nullptr ? p.out + g * p.block_bytes : p.dst[g];
    if (!p.fp8) {
      if (active) st_v4(reinterpret_cast<__nv_bfloat16*>(blk) + v * D + sl * 8, w[s]);
      continue;
    }
    const uint32_t ww[4] = {w[s].x, w[s].y, w[s].z, w[s].w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(ww[i] << 16);
      f[2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u);
    }
    float amax = fmaxf(fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3]))),
                       fmaxf(fmaxf(fabsf(f[4]), fabsf(f[5])), fmaxf(fabsf(f[6]), fabsf(f[7]))));
    // every lane takes part (inactive ones with zeros): the shuffles need the full warp
#pragma unroll
    for (int off = LPV / 2; off > 0; off >>= 1)
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float scale = __fdiv_rn(amax, kE4m3Max);
    const float inv = amax > 0.f ? __fdiv_rn(kE4m3Max, amax) : 0.f;
    uint2 q = make_uint2(0u, 0u);
    if (scale > 0.f) {
      q.x = static_cast<uint32_t>(e4m3x2(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv))) |
            (static_cast<uint32_t>(e4m3x2(__fmul_rn(f[2], inv), __fmul_rn(f[3], inv))) << 16);
      q.y = static_cast<uint32_t>(e4m3x2(__fmul_rn(f[4], inv), __fmul_rn(f[5], inv))) |
            (static_cast<uint32_t>(e4m3x2(__fmul_rn(f[6], inv), __fmul_rn(f[7], inv))) << 16);
    }
    if (active) {
      *reinterpret_cast<uint2*>(blk + v * D + sl * 8) = q;
      if (sl == 0) reinterpret_cast<float*>(blk + p.scale_off)[v] = scale;
    }
  }
  if (p.out == nullptr) __threadfence_system();  // peer stores performed before the kernel ends
}

// kLanes<D> lanes per vector of y; all loads of a lane's kExchangeSteps vectors
// first, then the dequantise-and-store pass.
template <int D, int S = kExchangeSteps>
__global__ void __launch_bounds__(256) exchange_unpack_kernel(ExchangeParams p) {
  constexpr int LPV = kLanes<D>, VPW = 32 / LPV;
  const int Tb = p.split == 0 ? p.T / p.G : p.T;
  const int Cb = p.split == 1 ? p.C / p.G : p.C;
  // y is [B][Ty][Cy][D]
  const int Ty = p.split == 1 ? p.G * Tb : Tb;
  const int Cy = p.split == 0 ? p.G * Cb : Cb;
  const int lane = threadIdx.x & 31, sub = lane / LPV, sl = lane - sub * LPV;
  const long long n_vec = static_cast<long long>(p.B) * Ty * Cy;
  const long long base =
      (static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * kExchangeVecPerWarp<D, S>;
  int cy = 0, ty = 0, b = 0;  // of the lane's first vector once, then stepped
  if (base + sub < n_vec) {
    const long long vec = base + sub;
    cy = static_cast<int>(vec % Cy);
    const long long bt = vec / Cy;
    ty = static_cast<int>(bt % Ty);
    b = static_cast<int>(bt / Ty);
  }
  uint4 raw[S];  // 8 bf16 values, or the 8 code bytes in .x/.y (fp8)
  float scale[S];
#pragma unroll
  for (int s = 0; s < S; ++s) {
    if (s > 0) exchange_step(VPW, Cy, Ty, b, ty, cy);
    raw[s] = make_uint4(0u, 0u, 0u, 0u);
    scale[s] = 0.f;
    if (base + s * VPW + sub >= n_vec) continue;
    int src, tl = ty, cl = cy;  // sending rank, and the position in its block
    if (p.split == 1) {
      src = ty / Tb;
      tl = ty - src * Tb;
    } else {
      src = cy / Cb;
      cl = cy - src * Cb;
    }
    const long long v = (static_cast<long long>(b) * Tb + tl) * Cb + cl;
    const uint8_t* blk = p.in + src * p.block_bytes;
    if (!p.fp8) {
      raw[s] = ld_nc_v4(reinterpret_cast<const __nv_bfloat16*>(blk) + v * D + sl * 8);
    } else {
      scale[s] = __ldg(reinterpret_cast<const float*>(blk + p.scale_off) + v);
      const uint2 q = __ldg(reinterpret_cast<const uint2*>(blk + v * D + sl * 8));
      raw[s].x = q.x;
      raw[s].y = q.y;
    }
  }
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const long long vec = base + s * VPW + sub;
    if (vec >= n_vec) continue;
    uint4 o = raw[s];
    if (p.fp8) {
      const uint32_t q2[2] = {raw[s].x, raw[s].y};
      uint32_t r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 fv = e4m3x2_to_f32(static_cast<uint16_t>(q2[i / 2] >> (16 * (i & 1))));
        r[i] = ptx::pack_bf16x2(__fmul_rn(fv.x, scale[s]), __fmul_rn(fv.y, scale[s]));
      }
      o = make_uint4(r[0], r[1], r[2], r[3]);
    }
    st_v4(p.y + vec * D + sl * 8, o);
  }
}

}  // namespace sa

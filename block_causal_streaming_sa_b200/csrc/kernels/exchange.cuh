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

// Vectors per warp: each lane issues the loads of all of them before the first
// store, so enough bytes are in flight to cover memory latency.
constexpr int kExchangeVecPerWarp = 4;

// One warp per kExchangeVecPerWarp consecutive vectors of x; lane l holds
// elements l*E .. l*E + E - 1 of each (E = D / 32).
template <int D>
__global__ void __launch_bounds__(256) exchange_pack_kernel(ExchangeParams p) {
  constexpr int E = D / 32, V = kExchangeVecPerWarp;
  const long long vec0 = (static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * V;
  const int lane = threadIdx.x & 31;
  const long long n_vec = static_cast<long long>(p.B) * p.T * p.C;
  // E bf16 values of this lane as E / 2 packed 32-bit words, for each vector
  uint32_t w[V][E / 2];
#pragma unroll
  for (int k = 0; k < V; ++k) {
    if (vec0 + k >= n_vec) break;
    const __nv_bfloat16* src = p.x + (vec0 + k) * D + lane * E;
    if constexpr (E == 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(src);
      w[k][0] = u.x;
      w[k][1] = u.y;
    } else {
      w[k][0] = *reinterpret_cast<const uint32_t*>(src);
    }
  }
  // (b, t, c) of the first vector once (64-bit division is a long routine),
  // then stepped for the next ones
  int c = 0, t = 0, b = 0;
  if (vec0 < n_vec) {
    c = static_cast<int>(vec0 % p.C);
    const long long bt = vec0 / p.C;
    t = static_cast<int>(bt % p.T);
    b = static_cast<int>(bt / p.T);
  }
#pragma unroll
  for (int k = 0; k < V; ++k) {
    const long long vec = vec0 + k;
    if (vec >= n_vec) break;
    if (k > 0 && ++c == p.C) {
      c = 0;
      if (++t == p.T) {
        t = 0;
        ++b;
      }
    }
    int g;
    long long v;
    exchange_place(p, b, t, c, g, v);
    uint8_t* blk = p.out != nullptr ? p.out + g * p.block_bytes : p.dst[g];
    if (!p.fp8) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(blk) + v * D +
                                                  lane * E);
#pragma unroll
      for (int i = 0; i < E / 2; ++i) dst[i] = w[k][i];
      continue;
    }
    float f[E];
#pragma unroll
    for (int i = 0; i < E / 2; ++i) {
      f[2 * i] = __uint_as_float(w[k][i] << 16);
      f[2 * i + 1] = __uint_as_float(w[k][i] & 0xFFFF0000u);
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < E; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float scale = __fdiv_rn(amax, kE4m3Max);
    const float inv = amax > 0.f ? __fdiv_rn(kE4m3Max, amax) : 0.f;
    uint8_t* codes = blk + v * D + lane * E;
    uint16_t q[E / 2];
#pragma unroll
    for (int i = 0; i < E / 2; ++i)
      q[i] = scale > 0.f ? e4m3x2(__fmul_rn(f[2 * i], inv), __fmul_rn(f[2 * i + 1], inv))
                         : static_cast<uint16_t>(0);
    if constexpr (E == 4)
      *reinterpret_cast<uint32_t*>(codes) = static_cast<uint32_t>(q[0]) |
                                            (static_cast<uint32_t>(q[E / 2 - 1]) << 16);
    else
      *reinterpret_cast<uint16_t*>(codes) = q[0];
    if (lane == 0) reinterpret_cast<float*>(blk + p.scale_off)[v] = scale;
  }
  if (p.out == nullptr) __threadfence_system();  // peer stores performed before the kernel ends
}

// One warp per kExchangeVecPerWarp consecutive vectors of y.
template <int D>
__global__ void __launch_bounds__(256) exchange_unpack_kernel(ExchangeParams p) {
  constexpr int E = D / 32, V = kExchangeVecPerWarp;
  const int Tb = p.split == 0 ? p.T / p.G : p.T;
  const int Cb = p.split == 1 ? p.C / p.G : p.C;
  // y is [B][Ty][Cy][D]
  const int Ty = p.split == 1 ? p.G * Tb : Tb;
  const int Cy = p.split == 0 ? p.G * Cb : Cb;
  const long long vec0 = (static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * V;
  const int lane = threadIdx.x & 31;
  const long long n_vec = static_cast<long long>(p.B) * Ty * Cy;
  uint32_t raw[V][E / 2];  // bf16 words, or the E code bytes in raw[k][0] (fp8)
  float scale[V];
  int cy = 0, ty = 0, b = 0;  // of the first vector once, then stepped (as in pack)
  if (vec0 < n_vec) {
    cy = static_cast<int>(vec0 % Cy);
    const long long bt = vec0 / Cy;
    ty = static_cast<int>(bt % Ty);
    b = static_cast<int>(bt / Ty);
  }
#pragma unroll
  for (int k = 0; k < V; ++k) {
    const long long vec = vec0 + k;
    if (vec >= n_vec) break;
    if (k > 0 && ++cy == Cy) {
      cy = 0;
      if (++ty == Ty) {
        ty = 0;
        ++b;
      }
    }
    int s, tl = ty, cl = cy;
    if (p.split == 1) {
      s = ty / Tb;
      tl = ty - s * Tb;
    } else {
      s = cy / Cb;
      cl = cy - s * Cb;
    }
    const long long v = (static_cast<long long>(b) * Tb + tl) * Cb + cl;
    const uint8_t* blk = p.in + s * p.block_bytes;
    if (!p.fp8) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(
          reinterpret_cast<const __nv_bfloat16*>(blk) + v * D + lane * E);
#pragma unroll
      for (int i = 0; i < E / 2; ++i) raw[k][i] = src[i];
    } else {
      scale[k] = reinterpret_cast<const float*>(blk + p.scale_off)[v];
      const uint8_t* codes = blk + v * D + lane * E;
      if constexpr (E == 4)
        raw[k][0] = *reinterpret_cast<const uint32_t*>(codes);
      else
        raw[k][0] = *reinterpret_cast<const uint16_t*>(codes);
    }
  }
#pragma unroll
  for (int k = 0; k < V; ++k) {
    const long long vec = vec0 + k;
    if (vec >= n_vec) break;
    uint32_t* out = reinterpret_cast<uint32_t*>(p.y + vec * D + lane * E);
    if (!p.fp8) {
#pragma unroll
      for (int i = 0; i < E / 2; ++i) out[i] = raw[k][i];
      continue;
    }
#pragma unroll
    for (int i = 0; i < E / 2; ++i) {
      const float2 fv = e4m3x2_to_f32(static_cast<uint16_t>(raw[k][0] >> (16 * i)));
      out[i] = ptx::pack_bf16x2(__fmul_rn(fv.x, scale[k]), __fmul_rn(fv.y, scale[k]));
    }
  }
}

}  // namespace sa

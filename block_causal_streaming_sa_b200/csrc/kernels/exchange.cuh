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

// Position of a vector in the exchange: batch b, rank block g, and (tl, cl), its
// token and head inside the block (a block is [B][Tb][Cb] vectors). The pass
// walks its own tensor in order, head fastest, and the block index is either
// inside the token (g_inner: a head split of x, or a token split of y, where a
// token row holds all G blocks) or outside it (a token split of x, a head split
// of y). step(k) advances by k vectors with no division.
struct ExchangePos {
  int b, g, tl, cl;
  __device__ __forceinline__ void init(unsigned vec, bool g_inner, int G, int Tb, int Cb) {
    cl = static_cast<int>(vec % Cb);
    unsigned r = vec / Cb;
    if (g_inner) {
      g = static_cast<int>(r % G);
      r /= G;
      tl = static_cast<int>(r % Tb);
      b = static_cast<int>(r / Tb);
    } else {
      tl = static_cast<int>(r % Tb);
      r /= Tb;
      g = static_cast<int>(r % G);
      b = static_cast<int>(r / G);
    }
  }
  __device__ __forceinline__ void step(int k, bool g_inner, int G, int Tb, int Cb) {
    cl += k;
    while (cl >= Cb) {
      cl -= Cb;
      if (g_inner) {
        if (++g == G) {
          g = 0;
          if (++tl == Tb) {
            tl = 0;
            ++b;
          }
        }
      } else if (++tl == Tb) {
        tl = 0;
        if (++g == G) {
          g = 0;
          ++b;
        }
      }
    }
  }
  // vector index inside its block
  __device__ __forceinline__ long long in_block(int Tb, int Cb) const {
    return (static_cast<long long>(b) * Tb + tl) * Cb + cl;
  }
};

// Sixteen elements per lane: kLanes<D> = D / 16 lanes per vector, lane sl holding
// the vector's 16-byte chunks sl and sl + kLanes<D> (so each load and store
// instruction covers whole halves of the vectors), and a fixed number of vectors
// per warp in steps of VPW = 32 / kLanes<D>; all loads of a lane before its
// first store, so enough bytes are in flight to cover memory latency. Measured
// on B200 (720p, 12 heads): pack with 8 vectors per warp at 4 blocks of 256
// threads per SM (64 registers) beat 16 vectors per warp at 2 blocks (127
// registers) by 15 %; unpack (55 registers) runs 16.
template <int D>
constexpr int kLanes = D / 16;
constexpr int kPackVecPerWarp = 8;
constexpr int kUnpackVecPerWarp = 16;

// pack: the amax of a vector is reduced over its lanes by shuffles; lane 0 of the
// vector writes its scale. The warp's NV vectors need 2 NV divisions (scale and
// its reciprocal): lane l computes the one of vector l % NV, the scale for
// (l / NV) even and the reciprocal for odd, so the warp runs one division in
// all, and the results are shuffled back.
template <int D>
__global__ void __launch_bounds__(256, 4) exchange_pack_kernel(ExchangeParams p) {
  constexpr int LPV = kLanes<D>, VPW = 32 / LPV, NV = kPackVecPerWarp, S = NV / VPW;
  static_assert(VPW * S == NV && 2 * NV <= 32, "one division per lane");
  const int lane = threadIdx.x & 31, sub = lane / LPV, sl = lane - sub * LPV;
  const unsigned n_vec = static_cast<unsigned>(p.B) * p.T * p.C;
  const unsigned base = (blockIdx.x * 8u + (threadIdx.x >> 5)) * NV;
  uint4 w[S][2];
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const unsigned vec = base + s * VPW + sub;
    const __nv_bfloat16* src = p.x + static_cast<size_t>(vec) * D + sl * 8;
    w[s][0] = vec < n_vec ? ld_nc_v4(src) : make_uint4(0u, 0u, 0u, 0u);
    w[s][1] = vec < n_vec ? ld_nc_v4(src + LPV * 8) : make_uint4(0u, 0u, 0u, 0u);
  }
  const int Tb = p.split == 0 ? p.T / p.G : p.T;
  const int Cb = p.split == 1 ? p.C / p.G : p.C;
  const bool g_inner = p.split == 1;
  ExchangePos pos;
  pos.init(base + sub, g_inner, p.G, Tb, Cb);
  float amax[S];
#pragma unroll
  for (int s = 0; s < S; ++s) {
    float a = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t ww[4] = {w[s][h].x, w[s][h].y, w[s][h].z, w[s][h].w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        a = fmaxf(a, fmaxf(fabsf(__uint_as_float(ww[i] << 16)),
                           fabsf(__uint_as_float(ww[i] & 0xFFFF0000u))));
    }
    // every lane takes part (inactive ones with zeros): the shuffles need the full warp
#pragma unroll
    for (int off = LPV / 2; off > 0; off >>= 1)
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    amax[s] = a;
  }
  float quot = 0.f;  // this lane's division (fp8 only)
  if (p.fp8) {
    const int qv = lane % NV;  // vector s * VPW + sub of the warp
    float a = 0.f;
#pragma unroll
    for (int s = 0; s < S; ++s) {
      const float as = __shfl_sync(0xffffffffu, amax[s], (qv % VPW) * LPV);
      if (qv / VPW == s) a = as;
    }
    const bool recip = (lane / NV) & 1;
    quot = __fdiv_rn(recip ? kE4m3Max : a, recip ? a : kE4m3Max);
  }
#pragma unroll
  for (int s = 0; s < S; ++s) {
    if (s > 0) pos.step(VPW, g_inner, p.G, Tb, Cb);
    const bool active = base + s * VPW + sub < n_vec;
    const long long v = pos.in_block(Tb, Cb);
    const int g = active ? pos.g : 0;
    uint8_t* blk = p.out != nullptr ? p.out + g * p.block_bytes : p.dst[g];
    if (!p.fp8) {
      if (active) {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(blk) + v * D + sl * 8;
        st_v4(dst, w[s][0]);
        st_v4(dst + LPV * 8, w[s][1]);
      }
      continue;
    }
    const float scale = __shfl_sync(0xffffffffu, quot, s * VPW + sub);
    const float inv_q = __shfl_sync(0xffffffffu, quot, NV + s * VPW + sub);
    const float inv = amax[s] > 0.f ? inv_q : 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t ww[4] = {w[s][h].x, w[s][h].y, w[s][h].z, w[s][h].w};
      float f[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(ww[i] << 16);
        f[2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u);
      }
      uint2 q = make_uint2(0u, 0u);
      if (scale > 0.f) {
        q.x = static_cast<uint32_t>(e4m3x2(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv))) |
              (static_cast<uint32_t>(e4m3x2(__fmul_rn(f[2], inv), __fmul_rn(f[3], inv))) << 16);
        q.y = static_cast<uint32_t>(e4m3x2(__fmul_rn(f[4], inv), __fmul_rn(f[5], inv))) |
              (static_cast<uint32_t>(e4m3x2(__fmul_rn(f[6], inv), __fmul_rn(f[7], inv))) << 16);
      }
      if (active) *reinterpret_cast<uint2*>(blk + v * D + (sl + h * LPV) * 8) = q;
    }
    if (active && sl == 0) reinterpret_cast<float*>(blk + p.scale_off)[v] = scale;
  }
  if (p.out == nullptr) __threadfence_system();  // peer stores performed before the kernel ends
}

// unpack: kLanes<D> lanes per vector of y; all loads of a lane's vectors first,
// then the dequantise-and-store pass.
template <int D>
__global__ void __launch_bounds__(256) exchange_unpack_kernel(ExchangeParams p) {
  constexpr int LPV = kLanes<D>, VPW = 32 / LPV, NV = kUnpackVecPerWarp, S = NV / VPW;
  const int Tb = p.split == 0 ? p.T / p.G : p.T;
  const int Cb = p.split == 1 ? p.C / p.G : p.C;
  // y is [B][Ty][Cy][D]: split 1 [B][G * Tb][Cb], split 0 [B][Tb][G * Cb]
  const bool g_inner = p.split == 0;
  const int lane = threadIdx.x & 31, sub = lane / LPV, sl = lane - sub * LPV;
  const unsigned n_vec = static_cast<unsigned>(p.B) * p.T * p.C;
  const unsigned base = (blockIdx.x * 8u + (threadIdx.x >> 5)) * NV;
  ExchangePos pos;
  pos.init(base + sub, g_inner, p.G, Tb, Cb);
  uint4 raw[S][2];  // bf16 payload: the two chunks; fp8: their codes in .x/.y
  float scale[S];
#pragma unroll
  for (int s = 0; s < S; ++s) {
    if (s > 0) pos.step(VPW, g_inner, p.G, Tb, Cb);
    raw[s][0] = raw[s][1] = make_uint4(0u, 0u, 0u, 0u);
    scale[s] = 0.f;
    if (base + s * VPW + sub >= n_vec) continue;
    const long long v = pos.in_block(Tb, Cb);
    const uint8_t* blk = p.in + pos.g * p.block_bytes;  // block of sending rank g
    if (!p.fp8) {
      const __nv_bfloat16* in = reinterpret_cast<const __nv_bfloat16*>(blk) + v * D + sl * 8;
      raw[s][0] = ld_nc_v4(in);
      raw[s][1] = ld_nc_v4(in + LPV * 8);
    } else {
      scale[s] = __ldg(reinterpret_cast<const float*>(blk + p.scale_off) + v);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint2 q = __ldg(reinterpret_cast<const uint2*>(blk + v * D + (sl + h * LPV) * 8));
        raw[s][h].x = q.x;
        raw[s][h].y = q.y;
      }
    }
  }
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const unsigned vec = base + s * VPW + sub;
    if (vec >= n_vec) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint4 o = raw[s][h];
      if (p.fp8) {
        const uint32_t q2[2] = {raw[s][h].x, raw[s][h].y};
        uint32_t r[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 fv = e4m3x2_to_f32(static_cast<uint16_t>(q2[i / 2] >> (16 * (i & 1))));
          r[i] = ptx::pack_bf16x2(__fmul_rn(fv.x, scale[s]), __fmul_rn(fv.y, scale[s]));
        }
        o = make_uint4(r[0], r[1], r[2], r[3]);
      }
      st_v4(p.y + static_cast<size_t>(vec) * D + (sl + h * LPV) * 8, o);
    }
  }
}

}  // namespace sa

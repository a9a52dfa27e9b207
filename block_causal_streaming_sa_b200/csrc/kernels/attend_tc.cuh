// Tensor-core attention of one chunk over its sink + window chunks (sm_100a).
//
// What it computes ("Vidu S2 vs PixVerse R2：实时视频的两条技术路线", sections
// 「实时」改变了什么 and 选择三：有上限的记忆): for every query row of the chunk
// being generated, softmax attention over the keys of the reference image (if
// set: "Vidu S2：实时可交互、可编辑、可立体的视频生成", section 2.2), the cached sink and
// window chunks of one TwinCache tier and the chunk's own keys, with the
// temporal RoPE base of chunk j relocated to ref_frames + the frames of the
// attended chunks before it (rank(j) * F when all have F frames). Variants
// (template kMode): dense; sparse, where only the 128 x 128 blocks a caller flags
// are attended (section 选择四：速度从哪里来: block-sparse attention with most blocks
// skipped); aligned, frame-aligned editing ("Vidu S2：实时可交互、可编辑、可立体的视频生成",
// section 2.6): the dense key set plus the source frames of the generating
// chunk, each query row seeing only the source frame of its own moment.
//
// Design (B200):
//  * persistent CTAs, one per SM; a work tile is two 128-row query tiles of one
//    (batch, head), so every K/V tile brought in by TMA feeds two MMAs;
//  * warp 0 (one lane): TMA producer over a ring of NSTAGE 128x D tiles,
//    K_0 V_0 K_1 V_1 ..., 128-byte swizzle, straight from the cache slots, the
//    reference planes and the caller's V (no gather copy);
//  * warp 1 (one lane): tcgen05.mma issuer. S_i = Q_i K^T (SS form, fp16, both
//    operands K-major in shared memory) into TMEM, then O_i += P_i V (TS form,
//    bf16: P_i read from TMEM, written over the upper half of S_i, V MN-major
//    in shared memory); the two query tiles ping-pong so one tile's softmax
//    overlaps the other's MMAs. It also issues the TMA copy of each query tile
//    of the next work unit as soon as this unit's O of that tile is final, so
//    the copy runs under the epilogue;
//  * warps 4-7 / 8-11: one warpgroup per query tile, thread = query row =
//    TMEM lane. Each turns its row of the query tile in shared memory, runs the
//    online softmax on S rows read from TMEM in one round trip (no cross-thread
//    reduction: a thread owns a whole row; max as an 8-way tree of 3-input
//    maxima, scale-and-subtract and the row sum in packed fp32x2 instructions,
//    1 exponential in 8 on the FMA pipe by a fitted polynomial), writes P
//    back as bf16, rescales O in TMEM only when the running max grows by more
//    than 2^8, and calls the epilogue, which stores O through per-warp staging
//    in shared memory (64-byte row segments per store instruction);
//  * registers: launched at 168 per thread (384 threads), warpgroup 0 (warps
//    0-3: producer, MMA issuer, two idle) gives registers back with setmaxnreg
//    (104) and the softmax warpgroups take them (200), so a whole 128-score row
//    stays in registers without spills; the epilogue is a separate function so
//    its registers do not add to the score loop's;
//  * RoPE: keys are stored rotated by their in-chunk position; the relocated
//    temporal base of the attended chunk is applied by re-turning
//    the temporal band of the query tile when the key stream moves to the next
//    chunk, before the first QK^T MMA of that chunk;
//  * work units: rounds of gridDim.x work tiles; when the last round holds at
//    most half a grid of tiles, each of them is split by attended chunks into
//    two halves run by two CTAs, which write normalised fp32 partial rows and
//    their log-sum-exp; per warp of rows, the second half to finish merges both;
//  * block-sparse: the mask arrives as bit rows (one per query tile); step j of
//    a work tile loads and multiplies the j-th flagged key tile of each of its
//    two query tiles, so the ping-pong of the dense loop is kept (a key tile
//    both flag at the same step is loaded once).
// All mbarrier waits are bounded (see ptx.cuh); on a timeout every role drains
// its outstanding async work, TMEM is freed and the device status word is set.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "../sa_internal.h"
#include "ptx.cuh"
#include "rope.cuh"

namespace sa {

template <int D>
struct TcShape {
  static constexpr int BM = 128;                 // query rows per tile (= TMEM lanes)
  static constexpr int BN = 128;                 // keys per K/V tile
  static constexpr int KBLK = D / 64;            // 64-element (128-byte) swizzle atoms per row
  static constexpr int kTile = BM * D * 2;       // bytes of a Q, K or V tile (BM == BN)
  static constexpr int kBox = BN * 128;          // bytes of one 64-column TMA box
  static constexpr int NSTAGE = (D == 128) ? 4 : 8;
  static constexpr int kThreads = 384;
  // Register split (setmaxnreg): launched at kLaunchRegs per thread (the
  // __launch_bounds__(384, 1) budget); warpgroup 0 (producer, MMA) drops to
  // kRegsCtl, the two softmax warpgroups rise to kRegsSoftmax.
  // 128 * 104 + 256 * 200 = 64512 = 384 * 168 (the launch pool), and per SM
  // sub-partition 104 + 200 + 200 = 504 <= 512 registers per thread slot.
  static constexpr int kLaunchRegs = 168;
  static constexpr int kRegsCtl = 104;
  static constexpr int kRegsSoftmax = 200;
  static_assert(128 * kRegsCtl + 256 * kRegsSoftmax <= kThreads * kLaunchRegs, "register split");
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTile;
  static constexpr int kOffQRaw = kOffKV + NSTAGE * kTile;  // raw temporal chunks of both Q tiles
  static constexpr int kQRawRow = ((D - 4 * (D / 6) + 7) / 8) * 16;
  static constexpr int kOffBar = kOffQRaw + 2 * BM * kQRawRow;
  static constexpr int kOffGroups = kOffBar + 256;  // attended-chunk table, tile starts, schedule
  static constexpr int kSmemBytes = kOffGroups + 256 + 128 + 1024;  // + alignment slack
  static constexpr int kTmemCols = 512;
  static constexpr int kDt = D - 4 * (D / 6);             // temporal band width
  static constexpr int kTChunks = (kDt + 7) / 8;           // 16-byte chunks holding it
  static constexpr uint32_t kIdescQK = ptx::idesc_f32acc(BM, BN, 0, 0);  // fp16 Q~, K~
  static constexpr uint32_t kIdescPV = ptx::idesc_f32acc(BM, D, 1, 1);   // bf16 P, V
  __host__ __device__ static constexpr int col_s(int i) { return i * 128; }
  __host__ __device__ static constexpr int col_o(int i) { return 256 + i * D; }
  __host__ __device__ static constexpr int col_p(int i) { return i * 128 + 64; }  // bf16 P
  // barrier indices
  __host__ __device__ static constexpr int FULL(int s) { return s; }
  __host__ __device__ static constexpr int EMPTY(int s) { return NSTAGE + s; }
  __host__ __device__ static constexpr int QREADY(int i) { return 2 * NSTAGE + i; }
  __host__ __device__ static constexpr int SFULL(int i) { return 2 * NSTAGE + 2 + i; }
  __host__ __device__ static constexpr int PFULL(int i) { return 2 * NSTAGE + 4 + i; }
  __host__ __device__ static constexpr int OFINAL(int i) { return 2 * NSTAGE + 6 + i; }
  __host__ __device__ static constexpr int DRAIN() { return 2 * NSTAGE + 8; }
  __host__ __device__ static constexpr int QLOAD(int i) { return 2 * NSTAGE + 9 + i; }
  static constexpr int kNumBars = 2 * NSTAGE + 11;
  static_assert(kNumBars * 8 <= 224, "barrier area");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

// Offset of 16-byte chunk c of row r in a 128-byte-swizzled K-major tile of 128 rows.
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * (128 * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// Store columns [col0, col0 + 32) of a warp's 32 O rows (bf16): lane l passes its
// row's 16 packed words; they go through the warp's staging rows in shared
// memory (stride kQRawRow bytes, the warp's own raw-query rows, unused once its
// unit's last key tile is done) and come back so that each store instruction
// writes whole 64-byte (D = 64: 32-byte) segments of 8 (16) rows. Row k of the
// warp is stored when k < n_rows, at row_off0 + k * row_stride. (A thread
// storing its own row in 16-byte pieces, rows H * D * 2 bytes apart, made every
// store instruction touch 32 lines.)
template <int D>
__device__ __forceinline__ void warp_store_cols(const AttendParams& p, unsigned long long row_off0,
                                                unsigned long long row_stride, int n_rows,
                                                const uint32_t (&w)[16], uint32_t stage, int lane,
                                                int col0) {
  using T = TcShape<D>;
  constexpr int PW = T::kQRawRow >= 64 ? 64 : 32;  // staged bytes per row and pass
  constexpr int PP = PW / 16;                       // 16-byte pieces per row and pass
  constexpr int RPI = 32 / PP;                      // rows per store instruction
#pragma unroll
  for (int pass = 0; pass < 64 / PW; ++pass) {
    __syncwarp();  // the previous pass has read the staging rows
#pragma unroll
    for (int q = 0; q < PP; ++q) {
      const int wi = (pass * PP + q) * 4;
      st_shared_v4(stage + lane * T::kQRawRow + q * 16,
                   make_uint4(w[wi], w[wi + 1], w[wi + 2], w[wi + 3]));
    }
    __syncwarp();
#pragma unroll
    for (int k = 0; k < PP; ++k) {
      const int row = k * RPI + lane / PP, piece = lane % PP;
      const uint4 v = ld_shared_v4(stage + row * T::kQRawRow + piece * 16);
      const unsigned long long off =
          row_off0 + row * row_stride + col0 + pass * (PW / 2) + piece * 8;
      if (row < n_rows && SA_IN_BOUNDS(p.status, off + 8, p.q_elems))
        st_v4(p.o + off, v);
    }
  }
  __syncwarp();
}

// Epilogue of one query row of a work unit; a function of its own so that its
// registers do not count against the score loop's (it runs once per unit).
// O / l -> bf16 row of [B, L, H, D] and the natural-log LSE; a row that saw no
// key (every block unflagged) gets O = 0 and lse = -inf. For a chunk-range half
// of a split tile (half >= 0): write the normalised fp32 partial row and its
// lse; the second of the two halves to finish (per-row counter) merges the two
// in half order, so the result does not depend on timing.
template <int D>
__device__ __noinline__ void epilogue(const AttendParams& p, uint32_t tO, bool any_tile, float m,
                                      float lsum, int half, int slot, int i, int r,
                                      unsigned long long row_off, long long lse_idx, bool valid) {
  using T = TcShape<D>;
  const bool seen = lsum > 0.f;
  const float inv = seen ? 1.f / lsum : 0.f;
  const float lse_own = seen ? (m + __log2f(lsum)) * 0.69314718055994531f : -INFINITY;
  // checked build: the row of O and the lse entry lie inside their buffers
  valid = valid && SA_IN_BOUNDS(p.status, row_off + D, p.q_elems);
  const bool lse_ok = valid && p.lse != nullptr &&
                      SA_IN_BOUNDS(p.status, static_cast<unsigned long long>(lse_idx) + 1,
                                   p.lse_elems);
  // The warp's rows are consecutive tokens and its valid rows a prefix of its
  // lanes; O goes out through the warp's staging rows (its raw-query rows of this
  // tile; the dynamic shared memory base is re-derived here as the kernel aligns
  // it, rather than passed in).
  const int lane = r & 31;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  const uint32_t stage = raw_addr + ((1024u - (raw_addr & 1023u)) & 1023u) + T::kOffQRaw +
                         static_cast<uint32_t>((i * T::BM + (r & ~31)) * T::kQRawRow);
  const int n_rows = __popc(__ballot_sync(0xffffffffu, valid));
  const unsigned long long row_off0 = __shfl_sync(0xffffffffu, row_off, 0);
  const unsigned long long row_stride = static_cast<unsigned long long>(p.H) * D;
  if (half < 0) {
#pragma unroll 1
    for (int j = 0; j < D / 32; ++j) {
      uint32_t o[32];
      if (any_tile) {
        ptx::tmem_ld32(tO + j * 32, o);
        ptx::tmem_wait_ld();
      }
      uint32_t wv[16];
#pragma unroll
      for (int k = 0; k < 16; ++k)
        wv[k] = seen ? ptx::pack_bf16x2(__uint_as_float(o[2 * k]) * inv,
                                        __uint_as_float(o[2 * k + 1]) * inv)
                     : 0u;
      warp_store_cols<D>(p, row_off0, row_stride, n_rows, wv, stage, lane, j * 32);
    }
    if (valid && lse_ok) p.lse[lse_idx] = lse_own;
    return;
  }
  const size_t prow = ((static_cast<size_t>(slot) * 2 + i) * 2 + half) * T::BM + r;
  const size_t qrow = ((static_cast<size_t>(slot) * 2 + i) * 2 + (1 - half)) * T::BM + r;
  if (!__all_sync(0xffffffffu,
                  SA_IN_BOUNDS(p.status, (prow > qrow ? prow : qrow) + 1, p.split_rows)))
    return;
  // A half's partial rows are stored [D / 4][128 rows][4]: for one group of four
  // columns a warp's 16-byte accesses cover 512 contiguous bytes (row-major rows,
  // 512 bytes apart, made every warp access touch 32 lines; the merge's reads of
  // them took ~29 K clocks at the end of the kernel's last round).
  float4* pb = reinterpret_cast<float4*>(p.split_o + (prow - r) * D);
  const float4* qb = reinterpret_cast<const float4*>(p.split_o + (qrow - r) * D);
#pragma unroll 1
  for (int j = 0; j < D / 32; ++j) {
    uint32_t o[32];
    if (any_tile) {
      ptx::tmem_ld32(tO + j * 32, o);
      ptx::tmem_wait_ld();
    }
#pragma unroll
    for (int c = 0; c < 32; c += 4)
      pb[((j * 32 + c) / 4) * T::BM + r] =
          seen ? make_float4(__uint_as_float(o[c]) * inv, __uint_as_float(o[c + 1]) * inv,
                             __uint_as_float(o[c + 2]) * inv, __uint_as_float(o[c + 3]) * inv)
               : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  p.split_lse[prow] = lse_own;
  // One counter per warp of rows: the warp that finds the other half's warp done
  // merges all 32 rows, so the merge's stores can go through the staging rows as
  // well. Every lane's partial row is performed before its warp counts.
  __threadfence();
  __syncwarp();
  int* sem = p.split_sem + (static_cast<size_t>(slot) * 2 + i) * T::BM + (r & ~31);
  int prev = 0;
  if (lane == 0) prev = atomicAdd(sem, 1);
  if (__shfl_sync(0xffffffffu, prev, 0) != 1) return;  // the other half's warp merges
  __threadfence();
  const float lse_other = __ldcg(p.split_lse + qrow);
  const float l0 = half == 0 ? lse_own : lse_other;
  const float l1 = half == 0 ? lse_other : lse_own;
  const float4* o0 = half == 0 ? pb : qb;  // half 0's block, then half 1's
  const float4* o1 = half == 0 ? qb : pb;
  const float mx2 = fmaxf(l0, l1);
  float w0 = 0.f, w1 = 0.f, lse_tot = -INFINITY;
  if (mx2 != -INFINITY) {
    const float e0 = __expf(l0 - mx2), e1 = __expf(l1 - mx2);
    lse_tot = mx2 + __logf(e0 + e1);
    w0 = e0 / (e0 + e1);
    w1 = e1 / (e0 + e1);
  }
  // 32 columns of both partial rows requested at a time (this merge ends the
  // kernel's last round)
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 32) {
    float4 a[8], bv[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      a[k] = __ldcg(o0 + (c0 / 4 + k) * T::BM + r);
      bv[k] = __ldcg(o1 + (c0 / 4 + k) * T::BM + r);
    }
    uint32_t wv[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      wv[2 * k] = ptx::pack_bf16x2(fmaf(w1, bv[k].x, w0 * a[k].x), fmaf(w1, bv[k].y, w0 * a[k].y));
      wv[2 * k + 1] =
          ptx::pack_bf16x2(fmaf(w1, bv[k].z, w0 * a[k].z), fmaf(w1, bv[k].w, w0 * a[k].w));
    }
    warp_store_cols<D>(p, row_off0, row_stride, n_rows, wv, stage, lane, c0);
  }
  if (valid && lse_ok) p.lse[lse_idx] = lse_tot;
  __syncwarp();
  if (lane == 0) *sem = 0;  // ready for the next launch
}

template <int D, int kMode>
__global__ void __launch_bounds__(384, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tm_cache,
                     const __grid_constant__ CUtensorMap tm_kcur,
                     const __grid_constant__ CUtensorMap tm_vcur,
                     const __grid_constant__ CUtensorMap tm_ref,
                     const __grid_constant__ CUtensorMap tm_vsrc,
                     const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ AttendParams p) {
  using T = TcShape<D>;
  constexpr bool kSparse = kMode == kModeSparse;    // caller-flagged 128 x 128 blocks
  constexpr bool kAligned = kMode == kModeAligned;  // last group: same-frame source keys
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t bar0 = sbase + T::kOffBar;
  auto bar = [&](int idx) { return bar0 + 8u * static_cast<uint32_t>(idx); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::kOffBar + 224);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::kOffBar + 228);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // clock record: global timer and SM cycles at the CTA's start and end (the
  // condition re-read at the end rather than kept live through the kernel)
  if (threadIdx.x == 0 && p.clock_stamps != nullptr && blockIdx.x < kMaxClockCtas) {
    p.clock_stamps[4 * blockIdx.x] = ptx::globaltimer();
    p.clock_stamps[4 * blockIdx.x + 1] = static_cast<unsigned long long>(clock64());
  }
  const int n_qt = (p.L + T::BM - 1) / T::BM;
  const int n_pairs = (n_qt + 1) / 2;
  const int n_work = p.B * p.H * n_pairs;

  // Shared tables (dynamic indexing of a kernel parameter would copy it to local
  // memory): the attended chunks, the first key tile of each, and the schedule
  // sched = {rounds, tail, split, middle chunk} of the work units.
  AttendGroup* groups = reinterpret_cast<AttendGroup*>(smem + T::kOffGroups);
  int* gstart = reinterpret_cast<int*>(smem + T::kOffGroups + 256);
  volatile int* sched = reinterpret_cast<volatile int*>(smem + T::kOffGroups + 256 + 72);
  static_assert(sizeof(AttendGroup) * kMaxGroups <= 256, "group table");
  if (threadIdx.x == 0) {
    int acc = 0;
#pragma unroll
    for (int g = 0; g < kMaxGroups; ++g) {
      groups[g] = p.groups[g];
      gstart[g] = acc;
      if (g < p.n_groups) acc += (p.groups[g].len + T::BN - 1) / T::BN;
    }
    gstart[kMaxGroups] = acc;
    const int rounds = (n_work + gridDim.x - 1) / gridDim.x;
    const int tail = n_work - (rounds - 1) * gridDim.x;
    sched[0] = rounds;
    sched[1] = tail;
    sched[2] = p.split_ok && p.n_groups >= 2 && 2 * tail <= static_cast<int>(gridDim.x) &&
               tail <= kMaxSplitSlots;
    sched[3] = p.n_groups / 2;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::NSTAGE; ++s) {
      ptx::mbar_init(bar(T::FULL(s)), 1);
      ptx::mbar_init(bar(T::EMPTY(s)), 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(T::QREADY(i)), 128);
      ptx::mbar_init(bar(T::SFULL(i)), 1);
      ptx::mbar_init(bar(T::PFULL(i)), 128);
      ptx::mbar_init(bar(T::OFINAL(i)), 1);
      ptx::mbar_init(bar(T::QLOAD(i)), 1);
    }
    ptx::mbar_init(bar(T::DRAIN()), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_slot), T::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  const int n_kt_total = gstart[p.n_groups];

  // Work unit r of this CTA: work tile w over attended chunks [g_lo, g_hi).
  // half = -1 for a whole tile, 0 / 1 for the two halves of a split tail tile.
  auto unit = [&](int r, int& w, int& half) -> bool {
    const int rounds = sched[0];
    half = -1;
    if (!sched[2] || r < rounds - 1) {
      w = blockIdx.x + r * gridDim.x;
      return w < n_work;
    }
    if (r > rounds - 1 || static_cast<int>(blockIdx.x) >= 2 * sched[1]) return false;
    w = (rounds - 1) * gridDim.x + (blockIdx.x >> 1);
    half = blockIdx.x & 1;
    return true;
  };
  auto g_lo = [&](int half) { return half == 1 ? sched[3] : 0; };
  auto g_hi = [&](int half) { return half == 0 ? sched[3] : p.n_groups; };

  // Skipped key tiles, frame-aligned mode: of the last group (the source frames),
  // only the tiles [mo, mo1) holding the frames of the work tile's rows are
  // visited; every other group is visited whole.
  auto mask_rows = [&](int w, int& mo, int& mo1) {
    mo = mo1 = -1;
    if constexpr (kAligned) {
      const int pair = w % n_pairs;
      const int hw = p.rope.frame_tokens;
      const int q0 = 2 * pair * T::BM, q1 = min(q0 + 2 * T::BM, p.L) - 1;
      const int gs = p.n_groups - 1;
      mo = gstart[gs] + (q0 / hw) * hw / T::BN;
      mo1 = gstart[gs] + (min((q1 / hw + 1) * hw, groups[gs].len) + T::BN - 1) / T::BN;
    }
  };
  // First visited flat key tile in [from, hi), or a value >= hi if none.
  auto next_visited = [&](int mo, int mo1, int from, int hi) {
    if constexpr (kAligned) {
      if (from < gstart[p.n_groups - 1]) return from;
      const int u = from < mo ? mo : from;
      return u < mo1 && u < hi ? u : hi;
    } else {
      return from;
    }
  };

  // Block sparsity: the flagged key tiles of query tile i of work tile w as a bit
  // row (null when the pair has a single query tile), and the first flagged tile
  // of a row in [from, hi), or hi when there is none.
  const int n_words = (n_kt_total + 63) >> 6;
  auto bit_row = [&](int w, int i) -> const unsigned long long* {
    const int bh = w / n_pairs, q = 2 * (w - bh * n_pairs) + i;
    return q < n_qt ? p.block_bits + (static_cast<size_t>(bh) * n_qt + q) * n_words : nullptr;
  };
  auto next_set = [&](const unsigned long long* row, int from, int hi) -> int {
    if (row == nullptr || from >= hi) return hi;
    int wd = from >> 6;
#ifdef SA_DEVICE_CHECKS
    const unsigned long long row0 = static_cast<unsigned long long>(row - p.block_bits);
    if (!SA_IN_BOUNDS(p.status, row0 + n_words, p.bits_words)) return hi;
#endif
    unsigned long long bits = __ldg(row + wd) & (~0ull << (from & 63));
    while (bits == 0ull) {
      if (++wd << 6 >= hi) return hi;
      bits = __ldg(row + wd);
    }
    const int k = (wd << 6) + __ffsll(static_cast<long long>(bits)) - 1;
    return k < hi ? k : hi;
  };

  if (warp < 4) {
  ptx::setmaxnreg_dec<T::kRegsCtl>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && !p.debug_stall_producer) {
      ptx::tma_prefetch_desc(&tm_cache);
      ptx::tma_prefetch_desc(&tm_kcur);
      ptx::tma_prefetch_desc(&tm_vcur);
      if (groups[0].src == 2) ptx::tma_prefetch_desc(&tm_ref);
      if (kAligned) ptx::tma_prefetch_desc(&tm_vsrc);
      int stage = 0;
      uint32_t phase = 0, filled_mask = 0, filled_parity = 0;
      bool ok = true;
      // K (kv 0) or V (kv 1) of key tile t of group grp into the next stage.
      auto load_kv = [&](const AttendGroup grp, int b, int h, int t, int kv) -> bool {
        if (!ptx::mbar_wait(bar(T::EMPTY(stage)), phase ^ 1u, abort_flag, p.status))
          return false;
        const uint32_t full = bar(T::FULL(stage));
        ptx::mbar_arrive_expect_tx(full, T::kTile);
        const uint32_t dst = sbase + T::kOffKV + stage * T::kTile;
        for (int kb = 0; kb < T::KBLK; ++kb) {
          if (grp.src == 0) {
            const int plane = ((grp.slot * 2 + kv) * p.B + b) * p.H + h;
            ptx::tma_load_3d(dst + kb * T::kBox, &tm_cache, full, kb * 64, t * T::BN, plane);
          } else if (grp.src == 2) {
            ptx::tma_load_3d(dst + kb * T::kBox, &tm_ref, full, kb * 64, t * T::BN,
                             (kv * p.B + b) * p.H + h);
          } else if (grp.src == 3) {  // source frames: keys in scratch half 1
            if (kv == 0)
              ptx::tma_load_3d(dst + kb * T::kBox, &tm_kcur, full, kb * 64, t * T::BN,
                               (p.B + b) * p.H + h);
            else
              ptx::tma_load_4d(dst + kb * T::kBox, &tm_vsrc, full, kb * 64, h, t * T::BN, b);
          } else if (kv == 0) {
            ptx::tma_load_3d(dst + kb * T::kBox, &tm_kcur, full, kb * 64, t * T::BN,
                             b * p.H + h);
          } else {
            ptx::tma_load_4d(dst + kb * T::kBox, &tm_vcur, full, kb * 64, h, t * T::BN, b);
          }
        }
        filled_mask |= 1u << stage;
        filled_parity = (filled_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == T::NSTAGE) {
          stage = 0;
          phase ^= 1u;
        }
        return true;
      };
      for (int rr = 0; ok; ++rr) {
        int w, half;
        if (!unit(rr, w, half)) break;
        const int bh = w / n_pairs;
        const int b = bh / p.H, h = bh - b * p.H;
        if constexpr (kSparse) {
          // Step j of a unit: the K tiles, then the V tiles, of the j-th flagged key
          // tile of each query tile (one tile when the two coincide).
          const int lo = gstart[g_lo(half)], hi = gstart[g_hi(half)];
          const unsigned long long* r0 = bit_row(w, 0);
          const unsigned long long* r1 = bit_row(w, 1);
          int ta = next_set(r0, lo, hi), tb = next_set(r1, lo, hi);
          int ga = g_lo(half), gb = ga;
          while (ok && (ta < hi || tb < hi)) {
            while (ta < hi && ta >= gstart[ga + 1]) ++ga;
            while (tb < hi && tb >= gstart[gb + 1]) ++gb;
            for (int kv = 0; ok && kv < 2; ++kv) {
              if (ta < hi) ok = load_kv(groups[ga], b, h, ta - gstart[ga], kv);
              if (ok && tb < hi && tb != ta) ok = load_kv(groups[gb], b, h, tb - gstart[gb], kv);
            }
            ta = next_set(r0, ta + 1, hi);
            tb = next_set(r1, tb + 1, hi);
          }
        } else {
          int mo, mo1;
          mask_rows(w, mo, mo1);
          for (int g = g_lo(half); ok && g < g_hi(half); ++g) {
            const AttendGroup grp = groups[g];
            int t0 = 0, t1 = (grp.len + T::BN - 1) / T::BN;
            if (kAligned && g == p.n_groups - 1) {
              t0 = mo - gstart[g];
              t1 = mo1 - gstart[g];
            }
            for (int t = t0; ok && t < t1; ++t)
              for (int kv = 0; kv < 2; ++kv)
                if (!load_kv(grp, b, h, t, kv)) {
                  ok = false;
                  break;
                }
          }
        }
      }
      // Let every issued copy land before the CTA can exit.
      volatile int no_abort = 0;
      for (int s = 0; s < T::NSTAGE; ++s)
        if (filled_mask & (1u << s))
          ptx::mbar_wait(bar(T::FULL(s)), (filled_parity >> s) & 1u, &no_abort, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t pf_phase[2] = {0u, 0u};
      bool ok = true;
      auto take_stage = [&](int& s_out) -> bool {
        s_out = stage;
        const bool r = ptx::mbar_wait(bar(T::FULL(stage)), phase, abort_flag, p.status);
        if (++stage == T::NSTAGE) {
          stage = 0;
          phase ^= 1u;
        }
        return r;
      };
      auto issue_s = [&](int i, int sk) {
        const uint32_t qa = sbase + T::kOffQ + i * T::kTile;
        const uint32_t kb = sbase + T::kOffKV + sk * T::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * T::kBox + (kk & 3) * 32;
          ptx::umma_ss(tmem + T::col_s(i), ptx::smem_desc_sw128(qa + off, 16, 1024),
                       ptx::smem_desc_sw128(kb + off, 16, 1024), T::kIdescQK, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int i, int sv, bool accumulate) {
        const uint32_t vb = sbase + T::kOffKV + sv * T::kTile;
#pragma unroll
        for (int kk = 0; kk < T::BN / 16; ++kk) {
          ptx::umma_ts(tmem + T::col_o(i), tmem + T::col_p(i) + kk * 8,
                       ptx::smem_desc_sw128(vb + kk * 16 * 128, T::kBox, 1024), T::kIdescPV,
                       (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      // Query tile i of unit rr by TMA (rows past L read as zeros), issued here
      // once unit rr - 1's O is final: every MMA that read the previous tile is
      // then done, and the copy runs under that unit's epilogue. This thread has
      // nothing else to do until the new tile is ready.
      int q_issued[2] = {0, 0};  // units whose tile i was requested
      ptx::tma_prefetch_desc(&tm_q);
      for (int rr = 0; ok; ++rr) {
        int w, half;
        if (!unit(rr, w, half)) break;
        {
          const int bh = w / n_pairs, pair = w - bh * n_pairs;
          const int b = bh / p.H, h = bh - b * p.H;
          for (int i = 0; i < 2 && ok; ++i) {
            if (rr > 0) ok = ptx::mbar_wait(bar(T::OFINAL(i)), (rr - 1) & 1, abort_flag, p.status);
            if (!ok) break;
            const uint32_t qb = bar(T::QLOAD(i));
            ptx::mbar_arrive_expect_tx(qb, T::kTile);
#pragma unroll
            for (int kb = 0; kb < T::KBLK; ++kb)
              ptx::tma_load_4d(sbase + T::kOffQ + i * T::kTile + kb * T::kBox, &tm_q, qb, kb * 64,
                               h, (2 * pair + i) * T::BM, b);
            q_issued[i] = rr + 1;
          }
          if (!ok) break;
        }
        const int lo = gstart[g_lo(half)], hi = gstart[g_hi(half)];
        int mo, mo1;
        mask_rows(w, mo, mo1);
        int u = next_visited(mo, mo1, lo, hi);
        if (kAligned && u >= hi) {  // no key tile: nothing to multiply
          for (int i = 0; i < 2 && ok; ++i)
            ok = ptx::mbar_wait(bar(T::QREADY(i)), rr & 1, abort_flag, p.status);
          if (ok)
            for (int i = 0; i < 2; ++i) ptx::umma_commit(bar(T::OFINAL(i)));
          continue;
        }
        if constexpr (!kSparse) {
          int sk = 0, sv = 0;
          if (!take_stage(sk)) break;
          ptx::tc_fence_after();
          for (int i = 0; i < 2; ++i) {
            if (!ptx::mbar_wait(bar(T::QREADY(i)), rr & 1, abort_flag, p.status)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            issue_s(i, sk);
            ptx::umma_commit(bar(T::SFULL(i)));
          }
          if (!ok) break;
          ptx::umma_commit(bar(T::EMPTY(sk)));
          for (bool first = true; ok && u < hi; first = false) {
            const int nu = next_visited(mo, mo1, u + 1, hi);
            const bool has_next = nu < hi;
            if (!take_stage(sv) || (has_next && !take_stage(sk))) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            for (int i = 0; i < 2; ++i) {
              if (!ptx::mbar_wait(bar(T::PFULL(i)), pf_phase[i], abort_flag, p.status)) {
                ok = false;
                break;
              }
              pf_phase[i] ^= 1u;
              ptx::tc_fence_after();
              issue_pv(i, sv, !first);
              if (i == 1) ptx::umma_commit(bar(T::EMPTY(sv)));
              if (!has_next) ptx::umma_commit(bar(T::OFINAL(i)));
              if (has_next) {
                issue_s(i, sk);
                ptx::umma_commit(bar(T::SFULL(i)));
              }
            }
            if (ok && has_next) ptx::umma_commit(bar(T::EMPTY(sk)));
            u = nu;
          }
        } else {
          // Block-sparse, in the producer's order: step j multiplies the j-th flagged
          // key tile of each query tile, so the two softmax warpgroups alternate as
          // in the dense loop; a query tile with fewer blocks drops out early.
          const unsigned long long* r0 = bit_row(w, 0);
          const unsigned long long* r1 = bit_row(w, 1);
          int ta = next_set(r0, lo, hi), tb = next_set(r1, lo, hi);
          // Stages of the tiles a (query tile 0) and c (query tile 1) of one step,
          // -1 for none; one stage when a == c.
          auto take_pair = [&](int a, int c, int& s0, int& s1) -> bool {
            s0 = s1 = -1;
            if (a < hi && !take_stage(s0)) return false;
            if (c < hi) {
              if (c == a)
                s1 = s0;
              else if (!take_stage(s1))
                return false;
            }
            return true;
          };
          int sk0, sk1;
          if (!take_pair(ta, tb, sk0, sk1)) break;
          ptx::tc_fence_after();
          for (int i = 0; i < 2; ++i) {
            if (!ptx::mbar_wait(bar(T::QREADY(i)), rr & 1, abort_flag, p.status)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            const int sk = i == 0 ? sk0 : sk1;
            if (sk >= 0) {
              issue_s(i, sk);
              ptx::umma_commit(bar(T::SFULL(i)));
            }
          }
          if (!ok) break;
          if (sk0 >= 0) ptx::umma_commit(bar(T::EMPTY(sk0)));
          if (sk1 >= 0 && sk1 != sk0) ptx::umma_commit(bar(T::EMPTY(sk1)));
          bool issued[2] = {false, false};  // a P.V of tile i issued in this unit
          while (ok && (ta < hi || tb < hi)) {
            const int na = next_set(r0, ta + 1, hi), nb = next_set(r1, tb + 1, hi);
            int sv0, sv1, nk0 = -1;
            if (!take_pair(ta, tb, sv0, sv1)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            for (int i = 0; i < 2; ++i) {
              const int sv = i == 0 ? sv0 : sv1;
              if (sv >= 0) {
                if (!ptx::mbar_wait(bar(T::PFULL(i)), pf_phase[i], abort_flag, p.status)) {
                  ok = false;
                  break;
                }
                pf_phase[i] ^= 1u;
                ptx::tc_fence_after();
                issue_pv(i, sv, issued[i]);
                issued[i] = true;
                if (i == 1 || sv0 != sv1) ptx::umma_commit(bar(T::EMPTY(sv)));
              }
              // S of tile i's next flagged tile; its S region is free: the softmax
              // has published P of the current one, whose P.V is issued above. Its
              // K stage is taken only now: the ring holds one step, so the next
              // step's K tiles may still be loading while this step's P.V runs.
              const int nxt = i == 0 ? na : nb;
              if (nxt < hi) {
                int nk = nk0;
                if ((i == 0 || nb != na) && !take_stage(nk)) {
                  ok = false;
                  break;
                }
                if (i == 0) nk0 = nk;
                ptx::tc_fence_after();
                issue_s(i, nk);
                ptx::umma_commit(bar(T::SFULL(i)));
                if (i == 1 || nb != na) ptx::umma_commit(bar(T::EMPTY(nk)));
              }
            }
            ta = na;
            tb = nb;
          }
          // O of both query tiles, also of one without a block: its warpgroup waits
          // for this before it loads the next unit's query tile.
          if (ok)
            for (int i = 0; i < 2; ++i) ptx::umma_commit(bar(T::OFINAL(i)));
        }
      }
      // Every MMA issued so far must finish before TMEM is released, and the last
      // query copies must land before the CTA can exit (also after an abort).
      volatile int no_abort = 0;
      ptx::umma_commit(bar(T::DRAIN()));
      ptx::mbar_wait(bar(T::DRAIN()), 0, &no_abort, p.status);
      for (int i = 0; i < 2; ++i)
        if (q_issued[i] > 0)
          ptx::mbar_wait(bar(T::QLOAD(i)), (q_issued[i] - 1) & 1, &no_abort, p.status);
    }
  }
  } else {
    ptx::setmaxnreg_inc<T::kRegsSoftmax>();
    // ------------------------------------------------------------ softmax warpgroups
    const int i = (warp - 4) >> 2;  // query tile of this warpgroup
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;
    const uint32_t t_lane = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + t_lane + T::col_s(i);
    const uint32_t tO = tmem + t_lane + T::col_o(i);
    const uint32_t q_smem = sbase + T::kOffQ + i * T::kTile;
    uint32_t s_phase = 0;
    bool ok = true;
    for (int rr = 0; ok; ++rr) {
      int w, half;
      if (!unit(rr, w, half)) break;
      const int bh = w / n_pairs, pair = w - bh * n_pairs;
      const int b = bh / p.H, h = bh - b * p.H;
      const int q_row = (2 * pair + i) * T::BM + r;
      const bool valid = q_row < p.L;
      const int qr = valid ? q_row : 0;
      const int f = qr / p.rope.frame_tokens;
      const int y = (qr / p.rope.tok_w) % p.rope.tok_h;
      const int x = qr % p.rope.tok_w;
      const size_t row_off = ((static_cast<size_t>(b) * p.L + qr) * p.H + h) * D;
      const int glo = g_lo(half), ghi = g_hi(half);
      int mo = -1, mo1 = -1;
      if (kAligned) mask_rows(w, mo, mo1);
      // First chunk with a key tile of this query tile (it is rotated for it).
      // Sparse: the tiles flagged for this query tile only, cur being the next
      // one; frame-aligned units visit every group, the last one partly.
      // (The bit row and its end are re-derived where used: fewer live registers.)
      // any_tile stays true in sparse mode too: a query tile without a flagged
      // block runs no tile, keeps lsum = 0, and its epilogue writes O = 0 and
      // lse = -inf (the tensor memory it reads is not used). A run-time any_tile
      // made the sparse score loop spill.
      int g0 = glo, cur = 0;
      const bool any_tile = true;
      if (kSparse) {
        cur = next_set(bit_row(w, i), gstart[glo], gstart[ghi]);
        while (g0 + 1 < ghi && cur >= gstart[g0 + 1]) ++g0;
      }

      // Rotated query tile for that chunk; the raw temporal chunks are kept in
      // shared memory for the re-turns at chunk switches.
      const uint32_t q_raw = sbase + T::kOffQRaw + (i * T::BM + r) * T::kQRawRow;
      if (!ptx::mbar_wait(bar(T::QLOAD(i)), rr & 1, abort_flag, p.status)) break;
      {
        // Each thread turns its own row in place; the RoPE (cos, sin) of 8 chunks
        // are fetched at a time: two round trips to the tables per row.
        const int td0 = groups[g0].t_delta;
        bool saturated = false;
        uint4 qv[D / 8];
#pragma unroll
        for (int c = 0; c < D / 8; ++c) qv[c] = ld_shared_v4(q_smem + sw128_offset(r, c));
#pragma unroll
        for (int c8 = 0; c8 < D / 8; c8 += 8) {
          float2 cs[8][4];
#pragma unroll
          for (int cc = 0; cc < 8; ++cc)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              // block-sparse units are short, so their start weighs: the band of
              // each pair resolved at compile time there (in the dense and aligned
              // instantiations it moved the score loop's register allocation and
              // cost ~1 % per clock; sparse gained 2-2.5 %)
              if constexpr (kSparse)
                cs[cc][j] = rope_cs_d<D>(p.rope, 4 * (c8 + cc) + j, td0 + f, y, x);
              else
                cs[cc][j] = rope_cs(p.rope, 4 * (c8 + cc) + j, td0 + f, y, x);
            }
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const int c = c8 + cc;
            const uint4 v = qv[c];
            if (c < T::kTChunks) st_shared_v4(q_raw + c * 16, v);
            saturated |= pair_norm_exceeds_f16(v);
            uint4 rv;
            rv.x = rope_pair(v.x, cs[cc][0]);
            rv.y = rope_pair(v.y, cs[cc][1]);
            rv.z = rope_pair(v.z, cs[cc][2]);
            rv.w = rope_pair(v.w, cs[cc][3]);
            st_shared_v4(q_smem + sw128_offset(r, c), rv);
          }
        }
        if (saturated) atomicOr(p.status, kDevWarnSaturated);
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(bar(T::QREADY(i)));
      }

      float m = -INFINITY, lsum = 0.f;
      int kt = 0;  // key tiles processed in this unit
      for (int g = glo; ok && any_tile && g < ghi; ++g) {
        const int len = groups[g].len;
        int t0 = 0, t1 = (len + T::BN - 1) / T::BN;
        if (kAligned && g == p.n_groups - 1) {
          t0 = mo - gstart[g];
          t1 = mo1 - gstart[g];
        }
        for (int t = t0; t < t1; ++t) {
          int nxt = 0;  // sparse: the flagged tile after this one (gstart[ghi]: none)
          if constexpr (kSparse) {
            if (cur >= gstart[g] + t1) break;  // the next one lies in a later chunk
            t = cur - gstart[g];
            nxt = next_set(bit_row(w, i), cur + 1, gstart[ghi]);
          }
          if (!ptx::mbar_wait(bar(T::SFULL(i)), s_phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          s_phase ^= 1u;
          ptx::tc_fence_after();
          {
            // The whole score row (128 fp32) in one round trip; keys past the chunk end
            // masked, and in a source tile every key outside the row's own frame.
            int c_lo = 0, c_hi = min(T::BN, len - t * T::BN);
            if (kAligned && g == p.n_groups - 1) {
              const int k0 = t * T::BN - f * p.rope.frame_tokens;  // tile start - frame start
              c_lo = max(c_lo, -k0);
              c_hi = min(c_hi, p.rope.frame_tokens - k0);
            }
            uint32_t sr[4][32];
#pragma unroll
            for (int j = 0; j < 4; ++j) ptx::tmem_ld32(tS + j * 32, sr[j]);
            ptx::tmem_wait_ld();
            if (c_lo > 0 || c_hi < T::BN) {
#pragma unroll
              for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int c = 0; c < 32; ++c)
                  if (j * 32 + c < c_lo || j * 32 + c >= c_hi)
                    sr[j][c] = __float_as_uint(-INFINITY);
            }
            // Row max as a tree over 8 independent running maxima (3-input max).
            float mx8[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) mx8[a] = __uint_as_float(sr[0][a]);
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
              for (int c = 0; c < 32; c += 2)
                if (j > 0 || c >= 8)
                  mx8[(c >> 1) & 7] = ptx::fmax3(mx8[(c >> 1) & 7], __uint_as_float(sr[j][c]),
                                                 __uint_as_float(sr[j][c + 1]));
            const float mx =
                fmaxf(ptx::fmax3(mx8[0], mx8[1], mx8[2]),
                      fmaxf(ptx::fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            const float m_new = fmaxf(m, mx * p.scale_log2);
            const bool need = m_new > m + 8.0f;
            float alpha = 1.f;
            if (need) {
              alpha = ptx::ex2(m - m_new);
              m = m_new;
            }
            // P = 2^(s * scale * log2 e - m) as bf16 pairs in columns 64..127 of the S
            // region (P of key k in column 64 + k / 2). x = s * scale * log2(e) - m two
            // at a time; the row sum in 4 packed partial sums.
            float rs8[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) rs8[a] = 0.f;
            // A row of a frame-aligned unit can meet a source tile wholly outside its
            // frame before any visible key (m still -inf): subtract 0 there, not -inf.
            const float sl = p.scale_log2, nm = (kAligned && m == -INFINITY) ? 0.f : -m;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t pk[16];
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                float x0, x1;
                ptx::ffma2(x0, x1, __uint_as_float(sr[j][2 * c]),
                           __uint_as_float(sr[j][2 * c + 1]), sl, sl, nm, nm);
                // One pair in eight goes through the FMA-pipe polynomial, the rest
                // through the exp unit (measured best split on B200).
                const bool poly = (c & 7) == 7;
                const float p0 = poly ? ptx::exp2_poly(x0) : ptx::ex2(x0);
                const float p1 = poly ? ptx::exp2_poly(x1) : ptx::ex2(x1);
                const int a = (c & 3) * 2;
                ptx::fadd2(rs8[a], rs8[a + 1], rs8[a], rs8[a + 1], p0, p1);
                pk[c] = ptx::pack_bf16x2(p0, p1);
              }
              ptx::tmem_st16(tS + 64 + j * 16, pk);
            }
            const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) +
                             ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
            lsum = lsum * alpha + rs;
            // The first tile's P.V overwrote O; a later growth of the max rescales it.
            if (__any_sync(0xffffffffu, need && kt > 0)) {
#pragma unroll
              for (int j = 0; j < D / 32; ++j) {
                uint32_t o[32];
                ptx::tmem_ld32(tO + j * 32, o);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c)
                  o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                ptx::tmem_st32(tO + j * 32, o);
              }
            }
          }
          // Chunk switch: the next key tile lies in a later chunk; turn the query
          // tile's temporal band to that chunk's relocated offset first.
          int gn = g;
          if (kSparse) {
            if (nxt < gstart[ghi] && nxt >= gstart[g + 1])
              while (gn + 1 < ghi && nxt >= gstart[gn + 1]) ++gn;
            cur = nxt;
          } else if (t == t1 - 1 && g + 1 < ghi) {
            gn = g + 1;
          }
          if (gn != g) {
            const int td = groups[gn].t_delta;
#pragma unroll 2
            for (int c = 0; c < T::kTChunks; ++c)
              st_shared_v4(q_smem + sw128_offset(r, c),
                           rope_chunk(ld_shared_v4(q_raw + c * 16), c, p.rope, td + f, y, x));
            ptx::fence_proxy_async_smem();
          }
          ptx::tmem_wait_st();
          ptx::tc_fence_before();
          ptx::mbar_arrive(bar(T::PFULL(i)));
          ++kt;
        }
      }
      if (!ok) break;

      if (!ptx::mbar_wait(bar(T::OFINAL(i)), rr & 1, abort_flag, p.status)) break;
      ptx::tc_fence_after();
      epilogue<D>(p, tO, any_tile, m, lsum, half,
                  w - (sched[0] - 1) * static_cast<int>(gridDim.x), i, r, row_off,
                  (static_cast<long long>(b) * p.H + h) * p.L + q_row, valid);
      ptx::tc_fence_before();
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (threadIdx.x == 0 && p.clock_stamps != nullptr && blockIdx.x < kMaxClockCtas) {
    p.clock_stamps[4 * blockIdx.x + 2] = ptx::globaltimer();
    p.clock_stamps[4 * blockIdx.x + 3] = static_cast<unsigned long long>(clock64());
  }
  if (warp == 1) ptx::tmem_dealloc(tmem, T::kTmemCols);
}

}  // namespace sa

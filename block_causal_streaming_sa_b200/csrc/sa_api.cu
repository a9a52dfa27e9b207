// Host side of libsa.so: config validation, the per-tier ring cache manager,
// the attention plan (attended chunks, slots, relocated temporal bases), RoPE
// tables, TMA descriptors and kernel launches. See include/sa.h for the
// contract of each entry point.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "sa_internal.h"
#include "kernels/attend_simt.cuh"
#include "kernels/attend_tc.cuh"
#include "kernels/block_bits.cuh"
#include "kernels/exchange.cuh"
#include "kernels/rope.cuh"

using sa::AttendGroup;
using sa::AttendParams;
using sa::AppendParams;
using sa::RopeTables;

namespace {

thread_local std::string g_error;

// NVTX range over one entry point (visible in Nsight timelines; a no-op
// without a tool attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Derived {
  int B, H, D, F, th, tw, S, W, R, L;
  int RF, Lref;  // reference image: frames, keys
  int dt2, dh2, dw2;
  float scale, theta;
  size_t chunk_elems;  // B * H * L * D
  size_t ref_elems;    // B * H * Lref * D
  // byte offsets inside the device buffer
  size_t off_status, off_rope_t, off_rope_h, off_rope_w, off_tier[2], off_kcur, off_ref;
  size_t off_split_o, off_split_lse, off_split_sem, split_sem_bytes;
  size_t off_bits, bits_bytes;  // block-sparse mask as bit rows
  size_t total;
};

int validate(const sa_config* c, std::string* why) {
  auto fail = [&](int code, const char* msg) {
    if (why) *why = msg;
    return code;
  };
  if (c == nullptr) return fail(SA_ERR_INVALID_ARG, "config is NULL");
  if (c->batch < 1 || c->heads < 1) return fail(SA_ERR_INVALID_ARG, "batch and heads must be >= 1");
  if (c->head_dim != 64 && c->head_dim != 128)
    return fail(SA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (c->frames_per_chunk < 1 || c->tok_h < 1 || c->tok_w < 1)
    return fail(SA_ERR_INVALID_ARG, "frames_per_chunk, tok_h, tok_w must be >= 1");
  if (c->frames_per_chunk > 1023 || c->tok_h > 2047 || c->tok_w > 2047)
    return fail(SA_ERR_UNSUPPORTED, "frames_per_chunk must be < 1024 and tok_h, tok_w < 2048");
  if (c->sink_chunks < 0 || c->window_chunks < 1)
    return fail(SA_ERR_INVALID_ARG, "need sink_chunks >= 0 and window_chunks >= 1");
  if (c->ref_frames < 0 || c->ref_frames > 1023)
    return fail(SA_ERR_INVALID_ARG, "ref_frames must be in 0..1023");
  if (c->sink_chunks + c->window_chunks + (c->ref_frames > 0 ? 1 : 0) > SA_MAX_ATTENDED)
    return fail(SA_ERR_UNSUPPORTED,
                "sink_chunks + window_chunks (+ 1 with a reference) exceeds SA_MAX_ATTENDED");
  const long long L = 1LL * c->frames_per_chunk * c->tok_h * c->tok_w;
  if (L > SA_MAX_CHUNK_LEN) return fail(SA_ERR_UNSUPPORTED, "chunk longer than SA_MAX_CHUNK_LEN");
  const long long Lref = 1LL * c->ref_frames * c->tok_h * c->tok_w;
  if (Lref > SA_MAX_CHUNK_LEN)
    return fail(SA_ERR_UNSUPPORTED, "reference longer than SA_MAX_CHUNK_LEN");
  if (1LL * c->batch * Lref > (1LL << 31) - 1)
    return fail(SA_ERR_UNSUPPORTED, "batch * reference too big");
  if (1LL * c->heads * c->head_dim / 8 > 1024)
    return fail(SA_ERR_UNSUPPORTED, "heads * head_dim must be <= 8192");
  if (1LL * c->batch * L > (1LL << 31) - 1) return fail(SA_ERR_UNSUPPORTED, "batch * chunk too big");
  const long long planes = 2LL * (c->sink_chunks + c->window_chunks) * c->batch * c->heads;
  if (planes > (1LL << 31) - 1) return fail(SA_ERR_UNSUPPORTED, "too many cache planes");
  if (!std::isfinite(c->softmax_scale) || !std::isfinite(c->rope_theta))
    return fail(SA_ERR_INVALID_ARG, "softmax_scale and rope_theta must be finite");
  return SA_OK;
}

Derived derive(const sa_config& c) {
  Derived d{};
  d.B = c.batch;
  d.H = c.heads;
  d.D = c.head_dim;
  d.F = c.frames_per_chunk;
  d.th = c.tok_h;
  d.tw = c.tok_w;
  d.S = c.sink_chunks;
  d.W = c.window_chunks;
  d.R = d.W - 1;
  d.L = d.F * d.th * d.tw;
  d.RF = c.ref_frames;
  d.Lref = d.RF * d.th * d.tw;
  const int d_sp = 2 * (d.D / 6);
  d.dt2 = (d.D - 2 * d_sp) / 2;
  d.dh2 = d_sp / 2;
  d.dw2 = d_sp / 2;
  d.scale = c.softmax_scale > 0.f ? c.softmax_scale : 1.f / std::sqrt(static_cast<float>(d.D));
  d.theta = c.rope_theta > 0.f ? c.rope_theta : 10000.f;
  d.chunk_elems = static_cast<size_t>(d.B) * d.H * d.L * d.D;
  d.ref_elems = static_cast<size_t>(d.B) * d.H * d.Lref * d.D;
  const size_t slot_bytes = 2 * d.chunk_elems * sizeof(__nv_bfloat16);
  size_t off = 0;
  d.off_status = off;
  off += 1024;
  d.off_rope_t = off;
  off += align_up(static_cast<size_t>(d.RF + (d.S + d.W) * d.F) * d.dt2 * sizeof(float2), 1024);
  d.off_rope_h = off;
  off += align_up(static_cast<size_t>(d.th) * d.dh2 * sizeof(float2), 1024);
  d.off_rope_w = off;
  off += align_up(static_cast<size_t>(d.tw) * d.dw2 * sizeof(float2), 1024);
  for (int t = 0; t < 2; ++t) {
    d.off_tier[t] = off;
    off += align_up(static_cast<size_t>(d.S + d.R) * slot_bytes, 1024);
  }
  d.off_kcur = off;  // [target | source] rotated keys of the generating chunk
  off += align_up(2 * d.chunk_elems * sizeof(__nv_bfloat16), 1024);
  d.off_ref = off;
  off += align_up(2 * d.ref_elems * sizeof(__nv_bfloat16), 1024);
  // split-tail scratch: partial rows, their lse, per-row merge counters
  const size_t split_rows = static_cast<size_t>(sa::kMaxSplitSlots) * 2 * 2 * 128;
  d.off_split_o = off;
  off += align_up(split_rows * d.D * sizeof(float), 1024);
  d.off_split_lse = off;
  off += align_up(split_rows * sizeof(float), 1024);
  d.off_split_sem = off;
  d.split_sem_bytes = static_cast<size_t>(sa::kMaxSplitSlots) * 2 * 128 * sizeof(int);
  off += align_up(d.split_sem_bytes, 1024);
  // block-sparse bit rows: B * H * n_q_tiles rows of ceil(n_k_tiles / 64) words,
  // at most (S + W) chunks of ceil(L / 128) key tiles (no reference, no source)
  const size_t q_tiles = (static_cast<size_t>(d.L) + 127) / 128;
  const size_t words = (static_cast<size_t>(d.S + d.W) * q_tiles + 63) / 64;
  d.off_bits = off;
  d.bits_bytes = static_cast<size_t>(d.B) * d.H * q_tiles * words * sizeof(unsigned long long);
  off += align_up(d.bits_bytes, 1024);
  d.total = off;
  return d;
}

// Ring slot of chunk `id`: sinks in slots 0..S-1, later chunks in S + (id-S) mod R.
int slot_of(const Derived& d, int id) {
  if (id < 0) return -1;
  if (id < d.S) return id;
  if (d.R == 0) return -1;
  return d.S + (id - d.S) % d.R;
}

// Attended chunks of chunk c, ascending: sinks, the window's cached chunks, c.
int plan_ids(const Derived& d, int c, int* ids) {
  int n = 0;
  for (int j = 0; j < c && j < d.S; ++j) ids[n++] = j;
  const int lo = c - d.R > d.S ? c - d.R : d.S;
  for (int j = lo; j < c; ++j) ids[n++] = j;
  ids[n++] = c;
  return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 tensor whose rows of D elements are tiled by 64-column x `rows` boxes
// with 128-byte swizzle. dims[0] = D (contiguous); strides in bytes.
bool encode_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                const cuuint64_t* strides, const cuuint32_t* box) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
                  strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [planes][rows][D] with planes contiguous rows x D matrices.
bool encode_planes(CUtensorMap* map, const void* base, const Derived& d, int rows,
                   long long planes) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d.D), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d.D) * 2,
                           static_cast<cuuint64_t>(rows) * d.D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  return encode_map(map, base, 3, dims, strides, box);
}

// The caller's [B, L, H, D] tensor (L = rows) as (D, H, L, B).
bool encode_blhd(CUtensorMap* map, const void* base, const Derived& d, int rows) {
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d.D), static_cast<cuuint64_t>(d.H),
                        static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(d.B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d.D) * 2,
                           static_cast<cuuint64_t>(d.H) * d.D * 2,
                           static_cast<cuuint64_t>(rows) * d.H * d.D * 2};
  cuuint32_t box[4] = {64, 1, 128, 1};
  return encode_map(map, base, 4, dims, strides, box);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Memory type of a tensor pointer, queried on the host before anything is
// launched: device memory (of `device`, or of any device when device < 0) or
// managed memory passes; host memory (pageable or pinned) and unknown
// addresses are refused. NULL passes (presence is checked by the callers).
bool device_memory(const void* p, int device, const char* what, std::string* why) {
  if (p == nullptr) return true;
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error of the failed query
    *why = std::string(what) + " is not a CUDA pointer";
    return false;
  }
  if (a.type == cudaMemoryTypeManaged) return true;
  if (a.type != cudaMemoryTypeDevice) {
    *why = std::string(what) + " is host memory; it must be device memory";
    return false;
  }
  if (device >= 0 && a.device != device) {
    *why = std::string(what) + " is on another device than the handle";
    return false;
  }
  return true;
}

// Persistent grid: one CTA per SM at most; with the split tail allowed, a problem
// of fewer work tiles than SMs gets two CTAs per tile (key-range halves).
unsigned attend_grid(const Derived& d, int rows, int sm_count, bool split_ok) {
  const int n_qt = (rows + 127) / 128;
  const long long n_work = 1LL * d.B * d.H * ((n_qt + 1) / 2);
  long long g = n_work < sm_count ? n_work : sm_count;
  if (split_ok && n_work < sm_count) g = 2 * n_work < sm_count ? 2 * n_work : sm_count;
  return static_cast<unsigned>(g);
}

// The attention kernel instantiations: head dim 128 / 64, dense / block-sparse.
// Tensor maps of one launch: cache tier, key scratch, current V, reference,
// source V (frame-aligned editing), queries.
struct AttendMaps {
  const CUtensorMap* cache;
  const CUtensorMap* kcur;
  const CUtensorMap* vcur;
  const CUtensorMap* ref;
  const CUtensorMap* vsrc;
  const CUtensorMap* q;
};

template <int D, int kMode>
void launch_attend_tc_t(unsigned grid, cudaStream_t s, const AttendMaps& m,
                        const AttendParams& ap) {
  sa::attend_tc_kernel<D, kMode><<<grid, sa::TcShape<D>::kThreads, sa::TcShape<D>::kSmemBytes,
                                   s>>>(*m.cache, *m.kcur, *m.vcur, *m.ref, *m.vsrc, *m.q, ap);
}

template <int D>
void launch_attend_tc_d(int mode, unsigned grid, cudaStream_t s, const AttendMaps& m,
                        const AttendParams& ap) {
  if (mode == sa::kModeSparse)
    launch_attend_tc_t<D, sa::kModeSparse>(grid, s, m, ap);
  else if (mode == sa::kModeAligned)
    launch_attend_tc_t<D, sa::kModeAligned>(grid, s, m, ap);
  else
    launch_attend_tc_t<D, sa::kModeDense>(grid, s, m, ap);
}

void launch_attend_tc(int D, int mode, unsigned grid, cudaStream_t s, const AttendMaps& m,
                      const AttendParams& ap) {
  if (D == 128)
    launch_attend_tc_d<128>(mode, grid, s, m, ap);
  else
    launch_attend_tc_d<64>(mode, grid, s, m, ap);
}

// Every instantiation: the register count the setmaxnreg split assumes, and the
// dynamic shared memory it needs.
template <int D, int kMode>
bool prepare_attend_tc_t() {
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, sa::attend_tc_kernel<D, kMode>) != cudaSuccess ||
      fa.numRegs != sa::TcShape<D>::kLaunchRegs)
    return false;
  return cudaFuncSetAttribute(sa::attend_tc_kernel<D, kMode>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              sa::TcShape<D>::kSmemBytes) == cudaSuccess;
}

template <int D>
bool prepare_attend_tc_d() {
  return prepare_attend_tc_t<D, sa::kModeDense>() && prepare_attend_tc_t<D, sa::kModeSparse>() &&
         prepare_attend_tc_t<D, sa::kModeAligned>();
}

__global__ void exp2_probe_kernel(const float* x, float* y, int n, int poly) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = poly ? sa::ptx::exp2_poly(x[i]) : sa::ptx::ex2(x[i]);
}

}  // namespace

struct sa_handle {
  sa_config cfg;
  Derived d;
  int device;
  int sm_count;
  uint8_t* buf;
  int count[2];
  int frames[2][SA_MAX_ATTENDED];  // frames of the chunk each slot holds, per tier
  int staged_chunk;                // chunk whose keys sit in the scratch (-1: none)
  int staged_frames;               // its frames
  bool staged_source;              // source-frame keys staged beside them
  bool has_cache;
  bool has_ref;  // a reference image is set
  bool inject_cuda_error;  // test hook: the next launching call fails with SA_ERR_CUDA
  CUtensorMap tm_tier[2];
  CUtensorMap tm_kcur;
  CUtensorMap tm_ref;
  std::string err;

  int fail(int code, const std::string& msg) {
    err = msg;
    return code;
  }
  unsigned* status() { return reinterpret_cast<unsigned*>(buf + d.off_status); }
  __nv_bfloat16* tier_base(int t) { return reinterpret_cast<__nv_bfloat16*>(buf + d.off_tier[t]); }
  __nv_bfloat16* kcur() { return reinterpret_cast<__nv_bfloat16*>(buf + d.off_kcur); }
  __nv_bfloat16* ref() { return reinterpret_cast<__nv_bfloat16*>(buf + d.off_ref); }
  RopeTables rope() {
    RopeTables rt;
    rt.t = reinterpret_cast<const float2*>(buf + d.off_rope_t);
    rt.h = reinterpret_cast<const float2*>(buf + d.off_rope_h);
    rt.w = reinterpret_cast<const float2*>(buf + d.off_rope_w);
    rt.dt2 = d.dt2;
    rt.dh2 = d.dh2;
    rt.dw2 = d.dw2;
    rt.tok_h = d.th;
    rt.tok_w = d.tw;
    rt.frame_tokens = d.th * d.tw;
    return rt;
  }
};

namespace {

int check_device(sa_handle* h) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return h->fail(SA_ERR_CUDA, "cudaGetDevice failed");
  if (dev != h->device)
    return h->fail(SA_ERR_INVALID_ARG, "current device differs from the handle's device");
  if (h->inject_cuda_error) {  // test hook (sa_debug_inject_cuda_error)
    h->inject_cuda_error = false;
    return h->fail(SA_ERR_CUDA, "injected CUDA error (test hook)");
  }
  return SA_OK;
}

// Every non-NULL pointer must be device memory of the handle's device (or
// managed memory); checked before anything is launched.
int check_mem(sa_handle* h, std::initializer_list<std::pair<const void*, const char*>> ptrs) {
  std::string why;
  for (const auto& pr : ptrs)
    if (!device_memory(pr.first, h->device, pr.second, &why))
      return h->fail(SA_ERR_INVALID_ARG, why);
  return SA_OK;
}

// Rotate K (and copy V, if given; rotate it too with second_is_key) of `rows`
// tokens into [B, H, L_out, D] planes.
int launch_rope_transpose(sa_handle* h, const void* K, const void* V, __nv_bfloat16* k_out,
                          __nv_bfloat16* v_out, int rows, int L_out, cudaStream_t s,
                          bool second_is_key = false) {
  const Derived& d = h->d;
  AppendParams ap;
  ap.k_in = static_cast<const __nv_bfloat16*>(K);
  ap.v_in = static_cast<const __nv_bfloat16*>(V);
  ap.k_out = k_out;
  ap.v_out = v_out;
  ap.B = d.B;
  ap.L = rows;
  ap.H = d.H;
  ap.D = d.D;
  ap.L_out = L_out;
  ap.second_is_key = second_is_key ? 1 : 0;
  ap.rope = h->rope();
  ap.status = h->status();
  ap.in_elems = 1ULL * d.B * rows * d.H * d.D;
  ap.out_elems = 1ULL * d.B * d.H * L_out * d.D;
  // One block per segment of XT tokens of a frame row (rows = whole frames), a
  // thread per (token, 16-byte chunk).
  const int xt = d.D == 128 ? sa::kRopeTokens<128> : sa::kRopeTokens<64>;
  const long long frame_rows = 1LL * d.B * (rows / d.tw);
  const long long n_seg = (d.tw + xt - 1) / xt;
  dim3 grid(static_cast<unsigned>(frame_rows * n_seg), V != nullptr ? 2 : 1);
  if (d.D == 128)
    sa::rope_transpose_kernel<sa::kRopeTokens<128>, sa::kRopeHeadGroup><<<grid, 256, 0, s>>>(ap);
  else
    sa::rope_transpose_kernel<sa::kRopeTokens<64>, sa::kRopeHeadGroup><<<grid, 256, 0, s>>>(ap);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return h->fail(SA_ERR_CUDA, std::string("append launch: ") + cudaGetErrorString(e));
  return SA_OK;
}

int check_handle(sa_handle* h) {
  if (h == nullptr) {
    g_error = "handle is NULL";
    return SA_ERR_INVALID_ARG;
  }
  return SA_OK;
}

int check_frames(sa_handle* h, int n_frames) {
  if (n_frames < 1 || n_frames > h->d.F)
    return h->fail(SA_ERR_INVALID_ARG, "n_frames must be in 1..frames_per_chunk");
  return SA_OK;
}

// The attention plan of the generating chunk c (n_frames frames) on `tier`:
// attended chunk ids in ascending order, each with its cache slot (-1: the chunk
// itself), frames and relocated temporal base = ref_frames + the frames of the
// attended chunks before it.
struct Plan {
  int n;
  int ids[SA_MAX_ATTENDED], slot[SA_MAX_ATTENDED], frames[SA_MAX_ATTENDED],
      base[SA_MAX_ATTENDED];
};

Plan make_plan(const sa_handle* h, int tier, int n_frames) {
  const Derived& d = h->d;
  const int c = h->count[0];
  Plan pl;
  pl.n = plan_ids(d, c, pl.ids);
  int pos = d.RF;
  for (int g = 0; g < pl.n; ++g) {
    const int id = pl.ids[g];
    pl.slot[g] = id == c ? -1 : slot_of(d, id);
    pl.frames[g] = id == c ? n_frames : h->frames[tier][pl.slot[g]];
    pl.base[g] = pos;
    pos += pl.frames[g];
  }
  return pl;
}

// Key groups of the attention kernels: the reference image (if set), the plan's
// chunks, and for frame-aligned editing the source frames of the generating
// chunk (same positions as its own frames: t_delta 0). t_delta = base(current) -
// base(group) >= 0.
void fill_groups(const sa_handle* h, int tier, int n_frames, bool source, AttendParams* ap) {
  const Derived& d = h->d;
  const Plan pl = make_plan(h, tier, n_frames);
  const int base_c = pl.base[pl.n - 1];
  int n = 0;
  if (h->has_ref) {
    AttendGroup& grp = ap->groups[n++];
    grp.src = 2;
    grp.slot = 0;
    grp.t_delta = base_c;
    grp.len = d.Lref;
  }
  for (int g = 0; g < pl.n; ++g) {
    AttendGroup& grp = ap->groups[n++];
    grp.src = pl.slot[g] < 0 ? 1 : 0;
    grp.slot = pl.slot[g] < 0 ? 0 : pl.slot[g];
    grp.t_delta = base_c - pl.base[g];
    grp.len = pl.frames[g] * d.th * d.tw;
  }
  if (source) {
    AttendGroup& grp = ap->groups[n++];
    grp.src = 3;
    grp.slot = 0;
    grp.t_delta = 0;
    grp.len = n_frames * d.th * d.tw;
  }
  ap->n_groups = n;
}

// Most key groups an attention of this config can have (the kernel's table holds
// kMaxGroups): S + W chunks, the reference, the source frames.
int max_groups(const sa_handle* h, bool source) {
  return h->d.S + h->d.W + (h->d.RF > 0 ? 1 : 0) + (source ? 1 : 0);
}

unsigned long long* clock_record(const sa_handle* h);
void note_clock_grid(const sa_handle* h, unsigned grid);

// Everything of AttendParams but the key source of the current chunk.
void fill_common(sa_handle* h, int tier, int n_frames, bool source, const void* Q,
                 const void* Vc, void* O, float* lse, AttendParams* ap) {
  const Derived& d = h->d;
  std::memset(ap, 0, sizeof(*ap));
  ap->q = static_cast<const __nv_bfloat16*>(Q);
  ap->o = static_cast<__nv_bfloat16*>(O);
  ap->lse = lse;
  ap->cache = h->tier_base(tier);
  ap->v_cur = static_cast<const __nv_bfloat16*>(Vc);
  ap->ref = h->has_ref ? h->ref() : nullptr;
  ap->B = d.B;
  ap->L = n_frames * d.th * d.tw;
  ap->H = d.H;
  ap->D = d.D;
  ap->L_plane = d.L;
  ap->L_ref = d.Lref;
  fill_groups(h, tier, n_frames, source, ap);
  ap->scale_log2 = d.scale * 1.4426950408889634f;
  ap->rope = h->rope();
  ap->status = h->status();
  ap->q_elems = 1ULL * d.B * ap->L * d.H * d.D;
  ap->lse_elems = 1ULL * d.B * d.H * ap->L;
  ap->bits_words = d.bits_bytes / sizeof(unsigned long long);
  ap->split_rows = 1ULL * sa::kMaxSplitSlots * 2 * 2 * 128;
  ap->cache_elems = 2ULL * (d.S + d.R) * d.chunk_elems;
  ap->kcur_elems = 2ULL * d.chunk_elems;
  ap->ref_elems = 2ULL * d.ref_elems;
  ap->clock_stamps = clock_record(h);
}

int check_attend_ptrs(sa_handle* h, const void* Q, const void* Vc, const void* O,
                      const float* lse) {
  if (Q == nullptr || Vc == nullptr || O == nullptr)
    return h->fail(SA_ERR_INVALID_ARG, "Q, Vc and O must be non-NULL");
  if (!aligned16(Q) || !aligned16(Vc) || !aligned16(O))
    return h->fail(SA_ERR_INVALID_ARG, "Q, Vc and O must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
    return h->fail(SA_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  if (O == Q || O == Vc) return h->fail(SA_ERR_INVALID_ARG, "O must not alias an input");
  return check_mem(h, {{Q, "Q"}, {Vc, "Vc"}, {O, "O"}, {lse, "lse"}});
}

// Rotate the generating chunk's keys (and, for frame-aligned editing, its
// source keys Ks) into the key scratch.
int stage_keys(sa_handle* h, const void* Kc, int n_frames, sa_stream stream,
               const void* Ks = nullptr) {
  int rc = check_handle(h);
  if (rc != SA_OK) return rc;
  rc = check_frames(h, n_frames);
  if (rc != SA_OK) return rc;
  if (Kc == nullptr || !aligned16(Kc))
    return h->fail(SA_ERR_INVALID_ARG, "Kc must be a non-NULL 16-byte aligned pointer");
  if (Ks != nullptr && !aligned16(Ks))
    return h->fail(SA_ERR_INVALID_ARG, "Ks must be 16-byte aligned");
  rc = check_mem(h, {{Kc, "Kc"}, {Ks, "Ks"}});
  if (rc != SA_OK) return rc;
  if (h->count[0] != h->count[1])
    return h->fail(SA_ERR_STATE, "both tiers must hold the same chunks before attending");
  rc = check_device(h);
  if (rc != SA_OK) return rc;
  rc = launch_rope_transpose(h, Kc, Ks, h->kcur(), h->kcur() + h->d.chunk_elems,
                             n_frames * h->d.th * h->d.tw, h->d.L,
                             reinterpret_cast<cudaStream_t>(stream), Ks != nullptr);
  if (rc != SA_OK) return rc;
  h->staged_chunk = h->count[0];
  h->staged_frames = n_frames;
  h->staged_source = Ks != nullptr;
  return SA_OK;
}

// The attention launch over the staged keys. Vs non-null: frame-aligned editing
// (the source keys must have been staged with the chunk's keys).
int attend_staged(sa_handle* h, const void* Q, const void* Vc, int step_is_final, void* O,
                  float* lse, sa_stream stream, bool simt, bool debug_stall = false,
                  const uint8_t* block_mask = nullptr, const void* Vs = nullptr) {
  int rc = check_handle(h);
  if (rc != SA_OK) return rc;
  rc = check_attend_ptrs(h, Q, Vc, O, lse);
  if (rc != SA_OK) return rc;
  const bool aligned = Vs != nullptr;
  if (aligned && (!aligned16(Vs) || O == Vs))
    return h->fail(SA_ERR_INVALID_ARG, "Vs must be 16-byte aligned and not aliased by O");
  rc = check_mem(h, {{Vs, "Vs"}, {block_mask, "block_mask"}});
  if (rc != SA_OK) return rc;
  if (aligned && !h->staged_source)
    return h->fail(SA_ERR_STATE, "no source keys staged for frame-aligned attention");
  if (aligned && (simt || block_mask != nullptr))
    return h->fail(SA_ERR_UNSUPPORTED, "frame-aligned attention runs on the dense kernel only");
  if (h->count[0] != h->count[1])
    return h->fail(SA_ERR_STATE, "both tiers must hold the same chunks before attending");
  if (h->staged_chunk != h->count[0])
    return h->fail(SA_ERR_STATE, "no keys staged for the current chunk (call sa_stage_keys)");
  if (block_mask != nullptr && h->has_ref)
    return h->fail(SA_ERR_UNSUPPORTED, "block-sparse attention takes no reference image");
  if (max_groups(h, aligned) > sa::kMaxGroups)
    return h->fail(SA_ERR_UNSUPPORTED, "more than SA_MAX_ATTENDED key groups (chunks, "
                                       "reference and source frames)");
  rc = check_device(h);
  if (rc != SA_OK) return rc;
  const Derived& d = h->d;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int tier = step_is_final ? SA_TIER_CLEAN : SA_TIER_NOISY;

  AttendParams ap;
  fill_common(h, tier, h->staged_frames, aligned, Q, Vc, O, lse, &ap);
  ap.k_cur = h->kcur();
  ap.debug_stall_producer = debug_stall ? 1 : 0;
  ap.split_o = reinterpret_cast<float*>(h->buf + d.off_split_o);
  ap.split_lse = reinterpret_cast<float*>(h->buf + d.off_split_lse);
  ap.split_sem = reinterpret_cast<int*>(h->buf + d.off_split_sem);
  ap.split_ok = h->sm_count <= 2 * sa::kMaxSplitSlots ? 1 : 0;

  if (simt) {
    const long long rows = 1LL * d.B * d.H * ap.L;
    const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
    if (d.D == 128)
      sa::attend_simt_kernel<128><<<grid, 256, 0, s>>>(ap);
    else
      sa::attend_simt_kernel<64><<<grid, 256, 0, s>>>(ap);
  } else {
    CUtensorMap tm_v, tm_vs, tm_q;
    if (!encode_blhd(&tm_v, Vc, d, ap.L) || (aligned && !encode_blhd(&tm_vs, Vs, d, ap.L)) ||
        !encode_blhd(&tm_q, Q, d, ap.L))
      return h->fail(SA_ERR_CUDA, "TMA descriptor for Q / Vc / Vs failed");
    AttendMaps maps{h->has_cache ? &h->tm_tier[tier] : &h->tm_kcur, &h->tm_kcur, &tm_v,
                    d.RF > 0 ? &h->tm_ref : &h->tm_kcur, aligned ? &tm_vs : &tm_v, &tm_q};
    if (block_mask != nullptr) {
      // Pack the mask's rows for this launch's key groups into bit rows.
      sa::BlockBitsParams bp;
      bp.mask = block_mask;
      bp.bits = reinterpret_cast<unsigned long long*>(h->buf + d.off_bits);
      bp.n_k = 0;
      for (int g = 0; g < ap.n_groups; ++g) bp.n_k += (ap.groups[g].len + 127) / 128;
      bp.n_words = (bp.n_k + 63) / 64;
      bp.rows = 1LL * d.B * d.H * ((ap.L + 127) / 128);
      bp.status = h->status();
      bp.mask_bytes = static_cast<unsigned long long>(bp.rows) * bp.n_k;
      bp.bits_words = d.bits_bytes / sizeof(unsigned long long);
      if (static_cast<size_t>(bp.rows) * bp.n_words * sizeof(unsigned long long) > d.bits_bytes)
        return h->fail(SA_ERR_UNSUPPORTED, "block mask larger than the bit-row region");
      sa::block_bits_kernel<<<static_cast<unsigned>((bp.rows + 7) / 8), 256, 0, s>>>(bp);
      ap.block_bits = bp.bits;
    }
    const int mode = block_mask != nullptr ? sa::kModeSparse
                     : aligned             ? sa::kModeAligned
                                           : sa::kModeDense;
    const unsigned grid = attend_grid(d, ap.L, h->sm_count, ap.split_ok != 0);
    note_clock_grid(h, grid);
    launch_attend_tc(d.D, mode, grid, s, maps,
                     ap);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return h->fail(SA_ERR_CUDA, std::string("attend launch: ") + cudaGetErrorString(e));
  return SA_OK;
}

int attend_common(sa_handle* h, const void* Q, const void* Kc, const void* Vc, int n_frames,
                  int step_is_final, void* O, float* lse, sa_stream stream, bool simt,
                  const uint8_t* block_mask = nullptr) {
  int rc = check_handle(h);
  if (rc != SA_OK) return rc;
  if (Kc == nullptr) return h->fail(SA_ERR_INVALID_ARG, "Kc must be non-NULL");
  if (O == Kc) return h->fail(SA_ERR_INVALID_ARG, "O must not alias an input");
  // Validate the attention half before launching the staging half.
  rc = check_attend_ptrs(h, Q, Vc, O, lse);
  if (rc != SA_OK) return rc;
  if (block_mask != nullptr && h->has_ref)
    return h->fail(SA_ERR_UNSUPPORTED, "block-sparse attention takes no reference image");
  rc = check_mem(h, {{Kc, "Kc"}, {block_mask, "block_mask"}});
  if (rc != SA_OK) return rc;
  rc = stage_keys(h, Kc, n_frames, stream);
  if (rc != SA_OK) return rc;
  return attend_staged(h, Q, Vc, step_is_final, O, lse, stream, simt, false, block_mask);
}

int attend_aligned(sa_handle* h, const void* Q, const void* Kc, const void* Vc, const void* Ks,
                   const void* Vs, int n_frames, int step_is_final, void* O, float* lse,
                   sa_stream stream) {
  int rc = check_handle(h);
  if (rc != SA_OK) return rc;
  if (Kc == nullptr || Ks == nullptr || Vs == nullptr)
    return h->fail(SA_ERR_INVALID_ARG, "Kc, Ks and Vs must be non-NULL");
  if (!aligned16(Ks) || !aligned16(Vs))
    return h->fail(SA_ERR_INVALID_ARG, "Ks and Vs must be 16-byte aligned");
  if (O == Kc || O == Ks || O == Vs)
    return h->fail(SA_ERR_INVALID_ARG, "O must not alias an input");
  // Validate the attention half before launching the staging half.
  rc = check_attend_ptrs(h, Q, Vc, O, lse);
  if (rc != SA_OK) return rc;
  if (max_groups(h, true) > sa::kMaxGroups)
    return h->fail(SA_ERR_UNSUPPORTED, "more than SA_MAX_ATTENDED key groups (chunks, "
                                       "reference and source frames)");
  rc = check_mem(h, {{Kc, "Kc"}, {Ks, "Ks"}, {Vs, "Vs"}});
  if (rc != SA_OK) return rc;
  rc = stage_keys(h, Kc, n_frames, stream, Ks);
  if (rc != SA_OK) return rc;
  return attend_staged(h, Q, Vc, step_is_final, O, lse, stream, false, false, nullptr, Vs);
}

// ---------------------------------------------------------------- sa_attend_noalloc
// Key scratch of sa_attend_noalloc: a fixed device array instead of the
// handle's region. In host code `g_noalloc_keys` names a host-side stand-in,
// not a device address: the address is looked up once per device with
// cudaGetSymbolAddress while that device is current.
static __device__ __align__(256) uint8_t g_noalloc_keys[SA_NOALLOC_MAX_KEY_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
// Per device ordinal: the array's address and the CUDA context it was looked up
// in (a process-unique context id). A device reset or a new primary context
// reloads the module, which may move the array, so a different context id
// means the address is looked up again.
struct NoallocAddr {
  unsigned long long ctx_id;
  void* ptr;
};
NoallocAddr g_noalloc_addr[kMaxDevices] = {};

typedef CUresult (*PFN_ctx_get_current)(CUcontext*);
typedef CUresult (*PFN_ctx_get_id)(CUcontext, unsigned long long*);

// Id of the calling thread's current CUDA context (driver entry points found
// through the runtime, so the library needs no link to libcuda).
bool current_ctx_id(unsigned long long* id) {
  static PFN_ctx_get_current get_current = nullptr;
  static PFN_ctx_get_id get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_ctx_get_current>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_ctx_get_id>(p);
  });
  CUcontext ctx = nullptr;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS ||
      ctx == nullptr)
    return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of a static device array on `device` (current), from `table`
// or looked up and cached there; an empty string on success, else the reason.
std::string symbol_address(int device, const void* symbol, NoallocAddr* table, void** out) {
  unsigned long long ctx = 0;
  if (!current_ctx_id(&ctx)) return "no current CUDA context";
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoallocAddr& a = table[device];
  if (a.ptr == nullptr || a.ctx_id != ctx) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, symbol);
    if (e != cudaSuccess || ptr == nullptr)
      return std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e);
    a.ptr = ptr;
    a.ctx_id = ctx;
  }
  *out = a.ptr;
  return std::string();
}

int noalloc_scratch(sa_handle* h, void** out) {
  if (h->device < 0 || h->device >= kMaxDevices)
    return h->fail(SA_ERR_UNSUPPORTED, "device ordinal too large for sa_attend_noalloc");
  const std::string why = symbol_address(h->device, g_noalloc_keys, g_noalloc_addr, out);
  if (!why.empty()) return h->fail(SA_ERR_CUDA, "sa_attend_noalloc key scratch: " + why);
  return SA_OK;
}

// Clock record of the attention kernel (sa_debug_kernel_clock): per CTA the
// global timer and the SM cycle counter at its start and end, for the most recent
// attention launch on each device, and that launch's CTA count.
static __device__ unsigned long long g_clock_stamps[sa::kMaxClockCtas * 4];
NoallocAddr g_clock_addr[kMaxDevices] = {};
std::atomic<int> g_clock_grid[kMaxDevices];

// The record's device address, or null (the attention runs without it).
unsigned long long* clock_record(const sa_handle* h) {
  if (h->device < 0 || h->device >= kMaxDevices) return nullptr;
  void* p = nullptr;
  if (!symbol_address(h->device, g_clock_stamps, g_clock_addr, &p).empty()) return nullptr;
  return static_cast<unsigned long long*>(p);
}

void note_clock_grid(const sa_handle* h, unsigned grid) {
  if (h->device >= 0 && h->device < kMaxDevices)
    g_clock_grid[h->device].store(static_cast<int>(grid));
}

int attend_noalloc(sa_handle* h, const void* Q, const void* Kc, const void* Vc, int step_is_final,
                   void* O, float* lse, sa_stream stream) {
  int rc = check_handle(h);
  if (rc != SA_OK) return rc;
  if (Kc == nullptr || !aligned16(Kc) || O == Kc)
    return h->fail(SA_ERR_INVALID_ARG, "Kc must be non-NULL, 16-byte aligned, not aliased by O");
  rc = check_attend_ptrs(h, Q, Vc, O, lse);
  if (rc != SA_OK) return rc;
  rc = check_mem(h, {{Kc, "Kc"}});
  if (rc != SA_OK) return rc;
  if (h->count[0] != h->count[1])
    return h->fail(SA_ERR_STATE, "both tiers must hold the same chunks before attending");
  const Derived& d = h->d;
  if (d.chunk_elems * sizeof(__nv_bfloat16) > SA_NOALLOC_MAX_KEY_BYTES)
    return h->fail(SA_ERR_UNSUPPORTED,
                   "B*H*L*D*2 bytes exceed SA_NOALLOC_MAX_KEY_BYTES (64 MiB) of sa_attend_noalloc");
  rc = check_device(h);
  if (rc != SA_OK) return rc;
  void* scratch = nullptr;
  rc = noalloc_scratch(h, &scratch);
  if (rc != SA_OK) return rc;
  __nv_bfloat16* keys = static_cast<__nv_bfloat16*>(scratch);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int tier = step_is_final ? SA_TIER_CLEAN : SA_TIER_NOISY;

  CUtensorMap tm_keys, tm_v, tm_q;
  if (!encode_planes(&tm_keys, keys, d, d.L, 1LL * d.B * d.H) ||
      !encode_blhd(&tm_v, Vc, d, d.L) || !encode_blhd(&tm_q, Q, d, d.L))
    return h->fail(SA_ERR_CUDA, "TMA descriptors for sa_attend_noalloc failed");

  AttendParams ap;
  fill_common(h, tier, d.F, false, Q, Vc, O, lse, &ap);
  ap.k_cur = keys;
  ap.kcur_elems = SA_NOALLOC_MAX_KEY_BYTES / sizeof(__nv_bfloat16);
  ap.split_ok = 0;  // no scratch but the fixed key array: no split tail

  // Every element of the scratch that the attention reads is written first by
  // this launch, or lies past the chunk's keys and is masked.
  rc = launch_rope_transpose(h, Kc, nullptr, keys, nullptr, d.L, d.L, s);
  if (rc != SA_OK) return rc;
  AttendMaps maps{h->has_cache ? &h->tm_tier[tier] : &tm_keys, &tm_keys, &tm_v,
                  d.RF > 0 ? &h->tm_ref : &tm_keys, &tm_v, &tm_q};
  const unsigned grid = attend_grid(d, d.L, h->sm_count, false);
  note_clock_grid(h, grid);
  launch_attend_tc(d.D, sa::kModeDense, grid, s, maps, ap);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return h->fail(SA_ERR_CUDA, std::string("attend launch: ") + cudaGetErrorString(e));
  return SA_OK;
}

int append_chunk(sa_handle* h, int tier, const void* K, const void* V, int n_frames,
                 sa_stream stream) {
  int rc = check_handle(h);
  if (rc != SA_OK) return rc;
  if (tier != SA_TIER_NOISY && tier != SA_TIER_CLEAN)
    return h->fail(SA_ERR_INVALID_ARG, "tier must be SA_TIER_NOISY or SA_TIER_CLEAN");
  rc = check_frames(h, n_frames);
  if (rc != SA_OK) return rc;
  if (K == nullptr || V == nullptr) return h->fail(SA_ERR_INVALID_ARG, "K and V must be non-NULL");
  if (!aligned16(K) || !aligned16(V))
    return h->fail(SA_ERR_INVALID_ARG, "K and V must be 16-byte aligned");
  if (h->count[tier] > h->count[1 - tier])
    return h->fail(SA_ERR_STATE, "this tier is already one chunk ahead of the other");
  rc = check_mem(h, {{K, "K"}, {V, "V"}});
  if (rc != SA_OK) return rc;
  rc = check_device(h);
  if (rc != SA_OK) return rc;
  const Derived& d = h->d;
  const int id = h->count[tier];
  const int slot = slot_of(d, id);
  if (slot >= 0) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    __nv_bfloat16* base = h->tier_base(tier) + static_cast<size_t>(slot) * 2 * d.chunk_elems;
    const int rows = n_frames * d.th * d.tw;
    rc = launch_rope_transpose(h, K, V, base, base + d.chunk_elems, rows, d.L, s);
    if (rc != SA_OK) return rc;
    // A short chunk's last key tile reads V rows past its end: P is 0 there, so
    // they only need to be finite. Zero them up to the tile boundary (the slot
    // may never have been written).
    const int hi = std::min(d.L, (rows + 127) / 128 * 128);
    if (hi > rows) {
      const size_t row_bytes = static_cast<size_t>(d.D) * sizeof(__nv_bfloat16);
      if (cudaMemset2DAsync(base + d.chunk_elems + static_cast<size_t>(rows) * d.D,
                            static_cast<size_t>(d.L) * row_bytes, 0,
                            static_cast<size_t>(hi - rows) * row_bytes,
                            static_cast<size_t>(d.B) * d.H, s) != cudaSuccess)
        return h->fail(SA_ERR_CUDA, std::string("clearing a short chunk's tail: ") +
                                        cudaGetErrorString(cudaGetLastError()));
    }
    h->frames[tier][slot] = n_frames;
  }
  h->count[tier] = id + 1;
  return SA_OK;
}

// ---------------------------------------------------------------- Ulysses exchange
// Checks the sender's shape and fills the layout fields; false (and g_error) on a
// bad argument.
bool exchange_layout(int B, int T, int C, int D, int G, int split, int payload,
                     sa::ExchangeParams* ep) {
  if (B < 1 || T < 1 || C < 1 || G < 1 || (D != 64 && D != 128) || (split != 0 && split != 1) ||
      (payload != SA_PAYLOAD_FP8 && payload != SA_PAYLOAD_BF16)) {
    g_error = "exchange: need B, T, C, G >= 1, D in {64, 128}, split 0/1, a known payload";
    return false;
  }
  if ((split == 0 ? T : C) % G != 0) {
    g_error = "exchange: the split dimension must be a multiple of the rank count";
    return false;
  }
  const long long n_vec = 1LL * B * T * C;
  if (n_vec >= (1LL << 31)) {  // the kernels index vectors in 32 bits
    g_error = "exchange: tensor too large (B*T*C must stay below 2^31 vectors)";
    return false;
  }
  const long long per_block = n_vec / G;
  std::memset(ep, 0, sizeof(*ep));
  ep->B = B;
  ep->T = T;
  ep->C = C;
  ep->D = D;
  ep->G = G;
  ep->split = split;
  ep->fp8 = payload == SA_PAYLOAD_FP8 ? 1 : 0;
  if (ep->fp8) {
    ep->scale_off = static_cast<long long>(align_up(static_cast<size_t>(per_block) * D, 16));
    ep->block_bytes =
        ep->scale_off + static_cast<long long>(align_up(static_cast<size_t>(per_block) * 4, 16));
  } else {
    ep->block_bytes = per_block * D * 2;
  }
  return true;
}

int launch_exchange(bool pack, sa::ExchangeParams& ep, sa_stream stream) {
  const long long n_vec = 1LL * ep.B * ep.T * ep.C;  // vectors of x (pack) and of y (unpack)
  const long long per_block = 8LL * (pack ? sa::kPackVecPerWarp : sa::kUnpackVecPerWarp);  // 8 warps
  const unsigned grid = static_cast<unsigned>((n_vec + per_block - 1) / per_block);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (pack)
    ep.D == 128 ? sa::exchange_pack_kernel<128><<<grid, 256, 0, s>>>(ep)
                : sa::exchange_pack_kernel<64><<<grid, 256, 0, s>>>(ep);
  else
    ep.D == 128 ? sa::exchange_unpack_kernel<128><<<grid, 256, 0, s>>>(ep)
                : sa::exchange_unpack_kernel<64><<<grid, 256, 0, s>>>(ep);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    g_error = std::string("exchange launch: ") + cudaGetErrorString(e);
    return SA_ERR_CUDA;
  }
  return SA_OK;
}

}  // namespace

extern "C" {

SA_API size_t sa_exchange_block_bytes(int B, int T, int C, int D, int G, int split_dim,
                                      int payload) {
  sa::ExchangeParams ep;
  if (!exchange_layout(B, T, C, D, G, split_dim, payload, &ep)) return 0;
  return static_cast<size_t>(ep.block_bytes);
}

SA_API int sa_exchange_pack(const void* x, int B, int T, int C, int D, int G, int split_dim,
                            int payload, void* buf, sa_stream stream) {
  NvtxRange range_("sa_exchange_pack");
  sa::ExchangeParams ep;
  if (!exchange_layout(B, T, C, D, G, split_dim, payload, &ep)) return SA_ERR_INVALID_ARG;
  if (x == nullptr || buf == nullptr || !aligned16(x) || !aligned16(buf)) {
    g_error = "exchange: x and buf must be non-NULL and 16-byte aligned";
    return SA_ERR_INVALID_ARG;
  }
  if (!device_memory(x, -1, "exchange: x", &g_error) ||
      !device_memory(buf, -1, "exchange: buf", &g_error))
    return SA_ERR_INVALID_ARG;
  ep.x = static_cast<const __nv_bfloat16*>(x);
  ep.out = static_cast<uint8_t*>(buf);
  return launch_exchange(true, ep, stream);
}

SA_API int sa_exchange_pack_to(const void* x, int B, int T, int C, int D, int G, int split_dim,
                               int payload, void* const* dst_blocks, sa_stream stream) {
  NvtxRange range_("sa_exchange_pack_to");
  sa::ExchangeParams ep;
  if (!exchange_layout(B, T, C, D, G, split_dim, payload, &ep)) return SA_ERR_INVALID_ARG;
  if (G > sa::kMaxExchangeRanks) {
    g_error = "exchange: more ranks than sa_exchange_pack_to supports (64)";
    return SA_ERR_UNSUPPORTED;
  }
  if (x == nullptr || dst_blocks == nullptr || !aligned16(x)) {
    g_error = "exchange: x and dst_blocks must be non-NULL, x 16-byte aligned";
    return SA_ERR_INVALID_ARG;
  }
  if (!device_memory(x, -1, "exchange: x", &g_error)) return SA_ERR_INVALID_ARG;
  for (int g = 0; g < G; ++g) {
    if (dst_blocks[g] == nullptr || !aligned16(dst_blocks[g])) {
      g_error = "exchange: every destination block must be non-NULL and 16-byte aligned";
      return SA_ERR_INVALID_ARG;
    }
    if (!device_memory(dst_blocks[g], -1, "exchange: a destination block", &g_error))
      return SA_ERR_INVALID_ARG;
    ep.dst[g] = static_cast<uint8_t*>(dst_blocks[g]);
  }
  ep.x = static_cast<const __nv_bfloat16*>(x);
  ep.out = nullptr;
  return launch_exchange(true, ep, stream);
}

SA_API int sa_ipc_alloc(size_t bytes, void** dev_ptr_out) {
  if (dev_ptr_out == nullptr || bytes == 0) {
    g_error = "ipc: NULL output or zero size";
    return SA_ERR_INVALID_ARG;
  }
  *dev_ptr_out = nullptr;
  cudaError_t e = cudaMalloc(dev_ptr_out, bytes);
  if (e != cudaSuccess) {
    g_error = std::string("cudaMalloc of an IPC buffer: ") + cudaGetErrorString(e);
    return SA_ERR_CUDA;
  }
  return SA_OK;
}

SA_API int sa_ipc_free(void* dev_ptr) {
  if (dev_ptr == nullptr) return SA_OK;
  cudaError_t e = cudaFree(dev_ptr);
  if (e != cudaSuccess) {
    g_error = std::string("cudaFree of an IPC buffer: ") + cudaGetErrorString(e);
    return SA_ERR_CUDA;
  }
  return SA_OK;
}

SA_API int sa_ipc_handle(const void* dev_ptr, void* handle_out) {
  if (dev_ptr == nullptr || handle_out == nullptr) {
    g_error = "ipc: NULL argument";
    return SA_ERR_INVALID_ARG;
  }
  cudaIpcMemHandle_t hdl;
  cudaError_t e = cudaIpcGetMemHandle(&hdl, const_cast<void*>(dev_ptr));
  if (e != cudaSuccess) {
    g_error = std::string("cudaIpcGetMemHandle: ") + cudaGetErrorString(e);
    return SA_ERR_CUDA;
  }
  static_assert(sizeof(hdl) == SA_IPC_HANDLE_BYTES, "IPC handle size");
  std::memcpy(handle_out, &hdl, sizeof(hdl));
  return SA_OK;
}

SA_API int sa_ipc_open(const void* handle, void** dev_ptr_out) {
  if (handle == nullptr || dev_ptr_out == nullptr) {
    g_error = "ipc: NULL argument";
    return SA_ERR_INVALID_ARG;
  }
  cudaIpcMemHandle_t hdl;
  std::memcpy(&hdl, handle, sizeof(hdl));
  *dev_ptr_out = nullptr;
  cudaError_t e = cudaIpcOpenMemHandle(dev_ptr_out, hdl, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) {
    g_error = std::string("cudaIpcOpenMemHandle: ") + cudaGetErrorString(e);
    return SA_ERR_CUDA;
  }
  return SA_OK;
}

SA_API int sa_ipc_close(void* dev_ptr) {
  if (dev_ptr == nullptr) return SA_OK;
  cudaError_t e = cudaIpcCloseMemHandle(dev_ptr);
  if (e != cudaSuccess) {
    g_error = std::string("cudaIpcCloseMemHandle: ") + cudaGetErrorString(e);
    return SA_ERR_CUDA;
  }
  return SA_OK;
}

SA_API int sa_exchange_unpack(const void* buf, int B, int T, int C, int D, int G, int split_dim,
                              int payload, void* y, sa_stream stream) {
  NvtxRange range_("sa_exchange_unpack");
  sa::ExchangeParams ep;
  if (!exchange_layout(B, T, C, D, G, split_dim, payload, &ep)) return SA_ERR_INVALID_ARG;
  if (y == nullptr || buf == nullptr || !aligned16(y) || !aligned16(buf) || y == buf) {
    g_error = "exchange: buf and y must be non-NULL, 16-byte aligned and distinct";
    return SA_ERR_INVALID_ARG;
  }
  if (!device_memory(buf, -1, "exchange: buf", &g_error) ||
      !device_memory(y, -1, "exchange: y", &g_error))
    return SA_ERR_INVALID_ARG;
  ep.in = static_cast<const uint8_t*>(buf);
  ep.y = static_cast<__nv_bfloat16*>(y);
  return launch_exchange(false, ep, stream);
}

SA_API int sa_validate_config(const sa_config* cfg) {
  std::string why;
  int rc = validate(cfg, &why);
  if (rc != SA_OK) g_error = why;
  return rc;
}

SA_API size_t sa_required_bytes(const sa_config* cfg) {
  if (sa_validate_config(cfg) != SA_OK) return 0;
  return derive(*cfg).total;
}

SA_API int sa_create(const sa_config* cfg, void* dev_buf, size_t bytes, sa_handle** out) {
  if (out == nullptr) {
    g_error = "out is NULL";
    return SA_ERR_INVALID_ARG;
  }
  *out = nullptr;
  std::string why;
  int rc = validate(cfg, &why);
  if (rc != SA_OK) {
    g_error = why;
    return rc;
  }
  const Derived d = derive(*cfg);
  if (dev_buf == nullptr || (reinterpret_cast<uintptr_t>(dev_buf) & 255u) != 0) {
    g_error = "dev_buf must be a non-NULL, 256-byte aligned device pointer";
    return SA_ERR_INVALID_ARG;
  }
  if (bytes < d.total) {
    g_error = "dev_buf smaller than sa_required_bytes(cfg)";
    return SA_ERR_INVALID_ARG;
  }
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, dev_buf) != cudaSuccess || attr.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    g_error = "dev_buf is not device memory";
    return SA_ERR_INVALID_ARG;
  }
  int dev = -1, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || attr.device != dev) {
    g_error = "dev_buf is not on the current device";
    return SA_ERR_INVALID_ARG;
  }
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10 || minor != 0) {
    g_error = "this library is built for sm_100a (B200) only";
    return SA_ERR_UNSUPPORTED;
  }

  sa_handle* h = new sa_handle();
  h->cfg = *cfg;
  h->d = d;
  h->device = dev;
  h->sm_count = sms;
  h->buf = static_cast<uint8_t*>(dev_buf);
  h->count[0] = h->count[1] = 0;
  for (int t = 0; t < 2; ++t)
    for (int s = 0; s < SA_MAX_ATTENDED; ++s) h->frames[t][s] = d.F;
  h->staged_chunk = -1;
  h->staged_frames = d.F;
  h->staged_source = false;
  h->has_ref = false;
  h->inject_cuda_error = false;

  // RoPE tables: angle pos * theta^(-2i/d) in double, cos/sin cast to float.
  // Temporal positions run over the reference frames and S + W chunks.
  const int n_tpos = d.RF + (d.S + d.W) * d.F;
  std::vector<float2> t(static_cast<size_t>(n_tpos) * d.dt2);
  std::vector<float2> th(static_cast<size_t>(d.th) * d.dh2), tw(static_cast<size_t>(d.tw) * d.dw2);
  // t and h position-major ([pos][pair]); w pair-major ([pair][x]), so that the
  // 32 rows of a warp, which lie at consecutive columns, read one pair's entries
  // from consecutive addresses.
  auto fill = [&](std::vector<float2>& tab, int npos, int npair, bool pair_major) {
    const double band = 2.0 * npair;
    for (int pos = 0; pos < npos; ++pos)
      for (int i = 0; i < npair; ++i) {
        const double a = pos * std::pow(static_cast<double>(d.theta), -2.0 * i / band);
        const size_t at = pair_major ? static_cast<size_t>(i) * npos + pos
                                     : static_cast<size_t>(pos) * npair + i;
        tab[at] = make_float2(static_cast<float>(std::cos(a)), static_cast<float>(std::sin(a)));
      }
  };
  fill(t, n_tpos, d.dt2, false);
  fill(th, d.th, d.dh2, false);
  fill(tw, d.tw, d.dw2, true);
  bool ok = cudaMemset(h->buf + d.off_status, 0, 1024) == cudaSuccess &&
            cudaMemset(h->buf + d.off_split_sem, 0, d.split_sem_bytes) == cudaSuccess;
  ok = ok && cudaMemcpy(h->buf + d.off_rope_t, t.data(), t.size() * sizeof(float2),
                        cudaMemcpyHostToDevice) == cudaSuccess;
  ok = ok && cudaMemcpy(h->buf + d.off_rope_h, th.data(), th.size() * sizeof(float2),
                        cudaMemcpyHostToDevice) == cudaSuccess;
  ok = ok && cudaMemcpy(h->buf + d.off_rope_w, tw.data(), tw.size() * sizeof(float2),
                        cudaMemcpyHostToDevice) == cudaSuccess;
  if (!ok) {
    g_error = std::string("uploading RoPE tables failed: ") + cudaGetErrorString(cudaGetLastError());
    delete h;
    return SA_ERR_CUDA;
  }
  h->has_cache = d.S + d.R > 0;
  if (h->has_cache) {
    for (int tier = 0; tier < 2; ++tier)
      if (!encode_planes(&h->tm_tier[tier], h->tier_base(tier), d, d.L,
                         2LL * (d.S + d.R) * d.B * d.H)) {
        g_error = "TMA descriptor for the cache failed";
        delete h;
        return SA_ERR_CUDA;
      }
  }
  if (!encode_planes(&h->tm_kcur, h->kcur(), d, d.L, 2LL * d.B * d.H)) {
    g_error = "TMA descriptor for the key scratch failed";
    delete h;
    return SA_ERR_CUDA;
  }
  if (d.RF > 0 && !encode_planes(&h->tm_ref, h->ref(), d, d.Lref, 2LL * d.B * d.H)) {
    g_error = "TMA descriptor for the reference image failed";
    delete h;
    return SA_ERR_CUDA;
  }
  // The kernel's register split assumes it is launched with exactly
  // TcShape::kLaunchRegs registers per thread; refuse to run otherwise.
  if (!prepare_attend_tc_d<128>() || !prepare_attend_tc_d<64>()) {
    g_error = "attention kernel: unexpected register count or shared memory attribute failed";
    delete h;
    return SA_ERR_UNSUPPORTED;
  }
  *out = h;
  return SA_OK;
}

SA_API int sa_destroy(sa_handle* h) {
  delete h;
  return SA_OK;
}

SA_API int sa_reset(sa_handle* h) {
  if (h == nullptr) {
    g_error = "handle is NULL";
    return SA_ERR_INVALID_ARG;
  }
  int rc = check_device(h);
  if (rc != SA_OK) return rc;
  h->count[0] = h->count[1] = 0;
  for (int t = 0; t < 2; ++t)
    for (int s = 0; s < SA_MAX_ATTENDED; ++s) h->frames[t][s] = h->d.F;
  h->staged_chunk = -1;
  h->has_ref = false;
  if (cudaMemset(h->buf + h->d.off_status, 0, 1024) != cudaSuccess ||
      cudaMemset(h->buf + h->d.off_split_sem, 0, h->d.split_sem_bytes) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess)
    return h->fail(SA_ERR_CUDA, "clearing the status word failed");
  return SA_OK;
}

SA_API int sa_append_chunk(sa_handle* h, int tier, const void* K, const void* V,
                           sa_stream stream) {
  NvtxRange range_("sa_append_chunk");
  if (h == nullptr) return check_handle(h);
  return append_chunk(h, tier, K, V, h->d.F, stream);
}

SA_API int sa_append_chunk_frames(sa_handle* h, int tier, const void* K, const void* V,
                                  int n_frames, sa_stream stream) {
  NvtxRange range_("sa_append_chunk_frames");
  return append_chunk(h, tier, K, V, n_frames, stream);
}

SA_API int sa_set_reference(sa_handle* h, const void* K, const void* V, sa_stream stream) {
  NvtxRange range_("sa_set_reference");
  int rc = check_handle(h);
  if (rc != SA_OK) return rc;
  if (K == nullptr && V == nullptr) {
    h->has_ref = false;
    return SA_OK;
  }
  if (h->d.RF == 0)
    return h->fail(SA_ERR_STATE, "the config has ref_frames == 0: no room for a reference image");
  if (K == nullptr || V == nullptr || !aligned16(K) || !aligned16(V))
    return h->fail(SA_ERR_INVALID_ARG, "K and V must both be non-NULL and 16-byte aligned");
  rc = check_mem(h, {{K, "K"}, {V, "V"}});
  if (rc != SA_OK) return rc;
  rc = check_device(h);
  if (rc != SA_OK) return rc;
  rc = launch_rope_transpose(h, K, V, h->ref(), h->ref() + h->d.ref_elems, h->d.Lref, h->d.Lref,
                             reinterpret_cast<cudaStream_t>(stream));
  if (rc != SA_OK) return rc;
  h->has_ref = true;
  return SA_OK;
}

SA_API int sa_attend(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                     int step_is_final, void* O, float* lse, sa_stream stream) {
  NvtxRange range_("sa_attend");
  if (h == nullptr) return check_handle(h);
  return attend_common(h, Q, Kc, Vc, h->d.F, step_is_final, O, lse, stream, false);
}

SA_API int sa_attend_frames(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                            int n_frames, int step_is_final, void* O, float* lse,
                            sa_stream stream) {
  NvtxRange range_("sa_attend_frames");
  return attend_common(h, Q, Kc, Vc, n_frames, step_is_final, O, lse, stream, false);
}

SA_API int sa_attend_aligned(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                             const void* Ks, const void* Vs, int n_frames, int step_is_final,
                             void* O, float* lse, sa_stream stream) {
  NvtxRange range_("sa_attend_aligned");
  return attend_aligned(h, Q, Kc, Vc, Ks, Vs, n_frames, step_is_final, O, lse, stream);
}

SA_API int sa_stage_keys(sa_handle* h, const void* Kc, sa_stream stream) {
  NvtxRange range_("sa_stage_keys");
  if (h == nullptr) return check_handle(h);
  return stage_keys(h, Kc, h->d.F, stream);
}

SA_API int sa_stage_keys_frames(sa_handle* h, const void* Kc, int n_frames, sa_stream stream) {
  NvtxRange range_("sa_stage_keys_frames");
  return stage_keys(h, Kc, n_frames, stream);
}

SA_API int sa_attend_staged(sa_handle* h, const void* Q, const void* Vc, int step_is_final,
                            void* O, float* lse, sa_stream stream) {
  NvtxRange range_("sa_attend_staged");
  return attend_staged(h, Q, Vc, step_is_final, O, lse, stream, false);
}

SA_API int sa_debug_attend_simt(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                                int step_is_final, void* O, float* lse, sa_stream stream) {
  if (h == nullptr) return check_handle(h);
  return attend_common(h, Q, Kc, Vc, h->d.F, step_is_final, O, lse, stream, true);
}

SA_API int sa_attend_noalloc(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                             int step_is_final, void* O, float* lse, sa_stream stream) {
  NvtxRange range_("sa_attend_noalloc");
  return attend_noalloc(h, Q, Kc, Vc, step_is_final, O, lse, stream);
}

SA_API int sa_attend_sparse(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                            int step_is_final, const uint8_t* block_mask, void* O, float* lse,
                            sa_stream stream) {
  NvtxRange range_("sa_attend_sparse");
  int rc = check_handle(h);
  if (rc != SA_OK) return rc;
  if (block_mask == nullptr) return h->fail(SA_ERR_INVALID_ARG, "block_mask must be non-NULL");
  return attend_common(h, Q, Kc, Vc, h->d.F, step_is_final, O, lse, stream, false, block_mask);
}

SA_API int sa_block_grid(const sa_config* cfg, int32_t chunk, int32_t* n_q_tiles,
                         int32_t* n_k_tiles) {
  std::string why;
  if (validate(cfg, &why) != SA_OK || chunk < 0 || n_q_tiles == nullptr || n_k_tiles == nullptr) {
    g_error = why.empty() ? "bad chunk or NULL output" : why;
    return SA_ERR_INVALID_ARG;
  }
  const Derived d = derive(*cfg);
  int ids[SA_MAX_ATTENDED];
  const int n = plan_ids(d, chunk, ids);
  *n_q_tiles = (d.L + 127) / 128;
  *n_k_tiles = n * ((d.L + 127) / 128);
  return SA_OK;
}

SA_API int sa_debug_attend_stalled(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                                   int step_is_final, void* O, sa_stream stream) {
  if (h == nullptr) return check_handle(h);
  int rc = stage_keys(h, Kc, h->d.F, stream);
  if (rc != SA_OK) return rc;
  return attend_staged(h, Q, Vc, step_is_final, O, nullptr, stream, false, true);
}

SA_API int sa_debug_exp2(int use_polynomial, const float* x, float* y, int n, sa_stream stream) {
  if (x == nullptr || y == nullptr || n < 0) {
    g_error = "x and y must be non-NULL and n >= 0";
    return SA_ERR_INVALID_ARG;
  }
  if (n == 0) return SA_OK;
  exp2_probe_kernel<<<(n + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      x, y, n, use_polynomial ? 1 : 0);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    g_error = std::string("exp2 probe launch: ") + cudaGetErrorString(e);
    return SA_ERR_CUDA;
  }
  return SA_OK;
}

SA_API int sa_debug_kernel_clock(double* sm_mhz, double* span_us) {
  if (sm_mhz == nullptr || span_us == nullptr) {
    g_error = "sa_debug_kernel_clock: NULL output";
    return SA_ERR_INVALID_ARG;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    g_error = "sa_debug_kernel_clock: no usable current device";
    return SA_ERR_CUDA;
  }
  const int n = g_clock_grid[dev].load();
  if (n <= 0) {
    g_error = "sa_debug_kernel_clock: no attention has run on this device";
    return SA_ERR_STATE;
  }
  const int ctas = n < sa::kMaxClockCtas ? n : sa::kMaxClockCtas;
  std::vector<unsigned long long> st(4 * static_cast<size_t>(ctas));
  if (cudaDeviceSynchronize() != cudaSuccess ||
      cudaMemcpyFromSymbol(st.data(), g_clock_stamps, st.size() * sizeof(st[0])) != cudaSuccess) {
    g_error = std::string("sa_debug_kernel_clock: ") + cudaGetErrorString(cudaGetLastError());
    return SA_ERR_CUDA;
  }
  std::vector<double> mhz;
  unsigned long long t0 = ~0ull, t1 = 0;
  for (int c = 0; c < ctas; ++c) {
    const unsigned long long* r = &st[4 * static_cast<size_t>(c)];
    if (r[2] <= r[0] || r[3] <= r[1]) continue;  // not stamped by this launch
    mhz.push_back(1e3 * static_cast<double>(r[3] - r[1]) / static_cast<double>(r[2] - r[0]));
    t0 = std::min(t0, r[0]);
    t1 = std::max(t1, r[2]);
  }
  if (mhz.empty()) {
    g_error = "sa_debug_kernel_clock: the last launch left no stamps";
    return SA_ERR_STATE;
  }
  std::sort(mhz.begin(), mhz.end());
  const size_t k = mhz.size();
  *sm_mhz = k % 2 ? mhz[k / 2] : 0.5 * (mhz[k / 2 - 1] + mhz[k / 2]);
  *span_us = 1e-3 * static_cast<double>(t1 - t0);
  return SA_OK;
}

SA_API int sa_debug_inject_cuda_error(sa_handle* h) {
  int rc = check_handle(h);
  if (rc != SA_OK) return rc;
  h->inject_cuda_error = true;
  return SA_OK;
}

SA_API int sa_chunk_count(const sa_handle* h, int tier) {
  if (h == nullptr || (tier != SA_TIER_NOISY && tier != SA_TIER_CLEAN)) return -SA_ERR_INVALID_ARG;
  return h->count[tier];
}

SA_API int sa_debug_layout(const sa_handle* h, int tier, int32_t* slot_chunk_ids,
                           int32_t* slot_ranks, int n) {
  if (h == nullptr || slot_chunk_ids == nullptr || (tier != SA_TIER_NOISY && tier != SA_TIER_CLEAN))
    return -SA_ERR_INVALID_ARG;
  const Derived& d = h->d;
  const int slots = d.S + d.R;
  const int m = n < slots ? n : slots;
  int held[SA_MAX_ATTENDED];
  for (int s = 0; s < slots; ++s) held[s] = -1;
  const int cnt = h->count[tier];
  for (int j = 0; j < cnt; ++j) {  // the latest chunk written to a slot holds it
    const int s = slot_of(d, j);
    if (s >= 0) held[s] = j;
  }
  for (int s = 0; s < m; ++s) {
    slot_chunk_ids[s] = held[s];
    if (slot_ranks == nullptr) continue;
    // rank = number of held chunks older than this one (ascending id order)
    int rank = 0;
    for (int u = 0; u < slots; ++u) rank += held[u] >= 0 && held[u] < held[s];
    slot_ranks[s] = held[s] < 0 ? -1 : rank;
  }
  return m;
}

SA_API int sa_plan(const sa_config* cfg, int32_t chunk, int32_t* ids, int32_t* slots,
                   int32_t* t_base, int cap) {
  std::string why;
  if (validate(cfg, &why) != SA_OK || chunk < 0) {
    g_error = chunk < 0 ? "chunk must be >= 0" : why;
    return -SA_ERR_INVALID_ARG;
  }
  const Derived d = derive(*cfg);
  int tmp[SA_MAX_ATTENDED];
  const int n = plan_ids(d, chunk, tmp);
  if (cap < n) {
    g_error = "cap too small";
    return -SA_ERR_INVALID_ARG;
  }
  for (int g = 0; g < n; ++g) {
    if (ids) ids[g] = tmp[g];
    if (slots) slots[g] = tmp[g] == chunk ? -1 : slot_of(d, tmp[g]);
    if (t_base) t_base[g] = d.RF + g * d.F;
  }
  return n;
}

SA_API int sa_stream_plan(const sa_handle* h, int step_is_final, int n_frames, int32_t* ids,
                          int32_t* t_base, int32_t* lens, int cap) {
  if (h == nullptr) {
    g_error = "handle is NULL";
    return -SA_ERR_INVALID_ARG;
  }
  sa_handle* hm = const_cast<sa_handle*>(h);  // for the error text only
  if (n_frames < 1 || n_frames > h->d.F) {
    hm->err = "n_frames must be in 1..frames_per_chunk";
    return -SA_ERR_INVALID_ARG;
  }
  if (h->count[0] != h->count[1]) {
    hm->err = "both tiers must hold the same chunks before attending";
    return -SA_ERR_STATE;
  }
  const Plan pl = make_plan(h, step_is_final ? SA_TIER_CLEAN : SA_TIER_NOISY, n_frames);
  if (cap < pl.n) {
    hm->err = "cap too small";
    return -SA_ERR_INVALID_ARG;
  }
  for (int g = 0; g < pl.n; ++g) {
    if (ids) ids[g] = pl.ids[g];
    if (t_base) t_base[g] = pl.base[g];
    if (lens) lens[g] = pl.frames[g] * h->d.th * h->d.tw;
  }
  return pl.n;
}

SA_API int sa_slot_of(const sa_config* cfg, int32_t chunk) {
  if (validate(cfg, nullptr) != SA_OK) return -1;
  return slot_of(derive(*cfg), chunk);
}

SA_API int sa_get_status(sa_handle* h, sa_stream stream) {
  if (h == nullptr) {
    g_error = "handle is NULL";
    return SA_ERR_INVALID_ARG;
  }
  unsigned word = 0;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess ||
      cudaMemcpy(&word, h->status(), sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return h->fail(SA_ERR_CUDA, std::string("reading the status word: ") +
                                    cudaGetErrorString(cudaGetLastError()));
  if (word & sa::kDevErrTimeout) return h->fail(SA_ERR_TIMEOUT, "a kernel gave up a bounded wait");
  if (word & sa::kDevErrBounds)
    return h->fail(SA_ERR_BOUNDS, "a kernel of the checked build skipped an access past the end "
                                  "of a buffer");
  if (word & sa::kDevWarnSaturated)
    return h->fail(SA_ERR_RANGE,
                   "a Q or K pair had a norm above 65504 and was saturated to fp16 for the "
                   "score MMA");
  return SA_OK;
}

SA_API const char* sa_last_error(const sa_handle* h) {
  return h != nullptr ? h->err.c_str() : g_error.c_str();
}

SA_API int sa_build_info(void) {
#ifdef SA_DEVICE_CHECKS
  return SA_BUILD_DEVICE_CHECKS;
#else
  return 0;
#endif
}

SA_API const char* sa_status_string(int status) {
  switch (status) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG";
    case SA_ERR_STATE: return "SA_ERR_STATE";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED";
    case SA_ERR_CUDA: return "SA_ERR_CUDA";
    case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT";
    case SA_ERR_RANGE: return "SA_ERR_RANGE";
    case SA_ERR_BOUNDS: return "SA_ERR_BOUNDS";
    default: return "SA_ERR_UNKNOWN";
  }
}

}  // extern "C"

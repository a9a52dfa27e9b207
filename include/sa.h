/*
 * sa.h - C ABI of the block-causal streaming attention library (libsa.so).
 *
 * One chunk's attention over a bounded two-tier KV cache of sink chunks plus a
 * rolling window of recent chunks, with relocated temporal RoPE, on NVIDIA B200
 * (sm_100a).
 *
 * Where the operation is defined (web pages, cited by title and section):
 *  - "Vidu S2 vs PixVerse R2：实时视频的两条技术路线" (orkas.ai blog):
 *      section 「实时」改变了什么 - video is generated chunk by chunk in order; a
 *      chunk sees what came before it, never what comes after (block causal).
 *      section 选择三：有上限的记忆 - the first chunks are kept for good as anchors
 *      (sink), a sliding window of the most recent chunks is kept and older ones
 *      are dropped; temporal positions are relocated into the trained range
 *      ("RoPE relocation"); TwinCache caches every history chunk twice, noisy and
 *      clean: intermediate denoising steps read the noisy copy, the final step
 *      reads the clean copy.
 *  - "Vidu S2：实时可交互、可编辑、可立体的视频生成" (paper read of Vidu S2):
 *      abbreviation table - the KV cache stores history keys and values so they
 *      are not recomputed; RoPE encodes each token's position in space and time.
 *      section 2.2 - block-wise causal mask, anchor chunks, sliding-window
 *      context, noisy KV cache, a reference image shared by every segment.
 *      section 2.4 - multi-GPU Ulysses context parallelism with quantised
 *      inter-GPU tensors; section 2.6 - the editing model's frame-aligned
 *      attention.
 *  The extensions cite their sections at each call: reference image and chunk
 *  length (sa_set_reference, sa_append_chunk_frames), block sparsity
 *  (sa_attend_sparse), frame-aligned editing (sa_attend_aligned), Ulysses
 *  exchange (sa_exchange_*).
 *
 * Conventions shared by every call
 *  - Tensors are bfloat16, row-major [B, L, H, D] (batch, token of the chunk,
 *    head, head dim), contiguous, 16-byte aligned, in device memory of the
 *    device the handle was created on. Token l of a chunk is frame
 *    l / (tok_h * tok_w), row (l / tok_w) % tok_h, column l % tok_w.
 *  - K and V passed in are UNROTATED; the library applies the 3D RoPE.
 *  - All device work is asynchronous on the caller's stream (a cudaStream_t
 *    passed as sa_stream; NULL is the legacy default stream). After sa_create,
 *    the append, reference, staging and attention calls allocate no memory and
 *    never synchronise the host (sa_reset and sa_get_status do synchronise).
 *  - Before anything is launched, every tensor pointer is checked on the host
 *    (cudaPointerGetAttributes): it must be device memory of the handle's
 *    device or managed memory, else SA_ERR_INVALID_ARG. A host pointer
 *    (pageable or pinned) is refused, not read by a kernel.
 *  - The device calls can be captured into a CUDA graph. A captured attention
 *    keeps the plan of the chunk it was captured for (attended chunks, slots
 *    and relocated positions are launch arguments): replay it for that chunk's
 *    steps of the same tier, with new contents in the same input buffers.
 *  - Every call returns an sa_status. On error nothing is launched and the
 *    handle's counters are unchanged; sa_last_error() explains the failure.
 *  - A handle is not thread-safe: one host thread drives one handle.
 */
#ifndef BLOCK_CAUSAL_STREAMING_SA_H
#define BLOCK_CAUSAL_STREAMING_SA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SA_API __attribute__((visibility("default")))

typedef struct sa_handle sa_handle;
typedef void* sa_stream; /* a cudaStream_t */

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or config field */
  SA_ERR_STATE = 2,        /* call not allowed in the handle's current state */
  SA_ERR_UNSUPPORTED = 3,  /* valid request the library does not serve (e.g. D) */
  SA_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed */
  SA_ERR_TIMEOUT = 5,      /* a kernel gave up a bounded wait (device status) */
  SA_ERR_RANGE = 6,        /* an operand left the fp16 range of the score MMA and
                              was saturated (device status; outputs degraded) */
  SA_ERR_BOUNDS = 7        /* checked build only: a kernel skipped an access past
                              the end of a buffer (a library bug; device status) */
} sa_status;

typedef enum { SA_TIER_NOISY = 0, SA_TIER_CLEAN = 1 } sa_tier;

/* Shape of one attention layer's stream. */
typedef struct {
  int32_t batch;            /* B >= 1 */
  int32_t heads;            /* H >= 1 */
  int32_t head_dim;         /* D: 64 or 128 */
  int32_t frames_per_chunk; /* F >= 1 latent frames per chunk */
  int32_t tok_h, tok_w;     /* tokens per frame: rows x columns */
  int32_t sink_chunks;      /* S >= 0 chunks kept for good */
  int32_t window_chunks;    /* W >= 1 most recent chunks attended, counting the
                               chunk being generated; W - 1 are cached */
  float softmax_scale;      /* <= 0 selects 1/sqrt(D) */
  float rope_theta;         /* <= 0 selects 10000 */
  int32_t ref_frames;       /* frames of the reference image, 0..1023 (0: none).
                               Every chunk's temporal positions start after them,
                               whether or not a reference is set. */
} sa_config;

/* Upper bounds of the library (checked by sa_validate_config). */
#define SA_MAX_ATTENDED 16 /* S + W, and S + W + 1 when ref_frames > 0 */
#define SA_MAX_CHUNK_LEN (1 << 22)

/* Validate a config; SA_OK or SA_ERR_INVALID_ARG / SA_ERR_UNSUPPORTED. Host only. */
SA_API int sa_validate_config(const sa_config* cfg);

/* Bytes of device memory sa_create needs for cfg (0 if cfg is invalid):
 * a status word, fp32 RoPE tables, both cache tiers ((S + W - 1) slots of K and
 * V each, layout [slot][K|V][B][H][L][D], K fp16, V bf16), two rotated-key chunks of
 * scratch for the chunk being generated (its keys and, for sa_attend_aligned,
 * its source keys), when ref_frames > 0 the reference image
 * ([K|V][B][H][ref_frames * tok_h * tok_w][D]), the split-tail scratch and
 * the bit rows sa_attend_sparse packs its mask into (B * H * ceil(L / 128)
 * rows of ceil((S + W) * ceil(L / 128) / 64) 64-bit words). Host only. */
SA_API size_t sa_required_bytes(const sa_config* cfg);

/* Create a handle over a caller-owned device buffer of at least
 * sa_required_bytes(cfg) bytes, 256-byte aligned, on the current device.
 * Writes the RoPE tables into it (synchronously) and encodes the TMA
 * descriptors of the cache. The buffer stays owned by the caller and must
 * outlive the handle. Returns SA_OK and *out, or an error and *out = NULL. */
SA_API int sa_create(const sa_config* cfg, void* dev_buf, size_t bytes, sa_handle** out);

/* Release the handle (host memory only; the caller frees dev_buf). NULL is OK. */
SA_API int sa_destroy(sa_handle* h);

/* Forget every cached chunk and the reference image, and clear the device
 * status word (start a new stream). Enqueues one small memset on the default
 * stream of the device and waits for it; not for use inside graph capture. */
SA_API int sa_reset(sa_handle* h);

/* Append the next chunk's K/V ([B, L, H, D], unrotated) to one tier.
 * Chunk ids count from 0 per tier. Chunk id n goes to slot n if n < S, else to
 * window slot S + (n - S) mod (W - 1), overwriting (evicting) the oldest
 * non-sink chunk once the window is full; with W == 1 a non-sink chunk is not
 * stored. K is rotated by its in-chunk (frame, row, column) position on the way
 * in and kept as fp16 (the score MMA's operand type). A pair (2i, 2i+1) whose
 * norm exceeds 65504, the fp16 maximum, is out of range: at some rotation
 * angles its values leave fp16 and are saturated to +-65504. The device status
 * word records every such pair whatever its angle (sa_get_status then returns
 * SA_ERR_RANGE until sa_reset); the same check covers Q and the keys of every
 * other call. V is kept as bf16. The relocated
 * temporal offset is applied at attend time.
 * A tier may run at most one chunk ahead of the other: appending to the tier
 * that is already ahead is SA_ERR_STATE. K and V may be freed once the launch
 * on `stream` has run. */
SA_API int sa_append_chunk(sa_handle* h, int tier, const void* K, const void* V,
                           sa_stream stream);

/* sa_append_chunk for a chunk of n_frames <= F frames (K, V: [B, n_frames *
 * tok_h * tok_w, H, D]). "Vidu S2 vs PixVerse R2", section 选择五: a chunk's
 * length follows the control signal up to a cap; here the cap is F and the
 * chunk keeps a whole slot. Later chunks' temporal positions follow from the
 * frames actually stored (see sa_attend). n_frames outside [1, F] is
 * SA_ERR_INVALID_ARG. sa_append_chunk is this call with n_frames = F. */
SA_API int sa_append_chunk_frames(sa_handle* h, int tier, const void* K, const void* V,
                                  int n_frames, sa_stream stream);

/* Set, replace or (K = V = NULL) clear the reference image: K, V [B, ref_frames
 * * tok_h * tok_w, H, D] bf16, unrotated. "Vidu S2：实时可交互、可编辑、可立体的视频生成",
 * section 2.2: every chunk also sees a shared reference image; "Vidu S2 vs
 * PixVerse R2" (Vidu S2's side): one shared reference keeps the subject's
 * identity. The reference sits at temporal positions 0 .. ref_frames - 1 (keys
 * rotated once here by their (frame, row, column)), ahead of every chunk; it
 * has a single copy read at every denoising step and is attended by every
 * chunk until replaced, cleared or sa_reset. Requires ref_frames > 0 in the
 * config (else SA_ERR_STATE). Asynchronous on `stream`: attention calls on
 * other streams must be ordered after it by the caller. */
SA_API int sa_set_reference(sa_handle* h, const void* K, const void* V, sa_stream stream);

/* Attention of the chunk being generated (chunk id c = number of chunks in
 * both tiers) at one denoising step:
 *   O = softmax(rope(Q) rope(K)^T * scale) V
 * over the keys of every cached sink and window chunk of the selected tier
 * (clean if step_is_final != 0, else noisy) followed by the chunk's own Kc/Vc,
 * all bidirectional inside the chunk, preceded by the reference image when
 * one is set (sa_set_reference). Frame f of attended chunk j sits at temporal
 * position ref_frames + (frames of the attended chunks before j) + f; with
 * every chunk of F frames that is ref_frames + rank(j) * F + f, rank = index of
 * j among the attended chunks in ascending id order, so positions stay below
 * ref_frames + (S + W) * F.
 * Q, Kc, Vc: [B, L, H, D] bf16 (unrotated), read only. Rotated Q and K enter
 * the score MMA as fp16, P and V the output MMA as bf16; accumulation is fp32.
 * O: [B, L, H, D] bf16, fully overwritten (must not alias the inputs).
 * lse: optional [B, H, L] fp32 natural-log sum of exp of the scaled scores
 *      (NULL to skip), for merging partial attentions.
 * Requires both tiers to hold the same number of chunks (else SA_ERR_STATE).
 * Uses the handle's rotated-key scratch: calls on one handle must be ordered
 * on the GPU (same stream, or events). */
SA_API int sa_attend(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                     int step_is_final, void* O, float* lse, sa_stream stream);

/* sa_attend for a generating chunk of n_frames <= F frames: Q, Kc, Vc, O are
 * [B, Lc, H, D] and lse [B, H, Lc] with Lc = n_frames * tok_h * tok_w.
 * sa_attend is this call with n_frames = F. */
SA_API int sa_attend_frames(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                            int n_frames, int step_is_final, void* O, float* lse,
                            sa_stream stream);

/* Frame-aligned editing attention. "Vidu S2：实时可交互、可编辑、可立体的视频生成",
 * section 2.6 (the editing model S2-Editing): the source video is encoded as
 * condition tokens next to the noisy target tokens; every generated frame
 * exchanges information only with the source frame of the same moment; the
 * reference image is seen by every frame; each source frame is consumed with
 * its target frame and never cached ("Vidu S2：实时数字人、实时视频编辑都做到了，空间视频还只是
 * 探索", section on S2-Editing, says the same).
 * Computes sa_attend_frames over the usual keys (reference if set, cached sink
 * and window chunks of the selected tier, the chunk's own Kc/Vc) plus the
 * source tokens Ks/Vs ([B, Lc, H, D] bf16, unrotated, the same frames and
 * token grid as Q), where a query token of frame f sees only the source tokens
 * of frame f. Source frame f takes the temporal and spatial coordinates of
 * target frame f. Nothing of Ks/Vs is kept after the call. The key scratch
 * holds Kc and Ks rotated; one staging launch and one attention launch.
 * Needs S + W (+ 1 with a reference) + 1 <= SA_MAX_ATTENDED key groups, else
 * SA_ERR_UNSUPPORTED. O, lse, n_frames and the error rules as sa_attend_frames. */
SA_API int sa_attend_aligned(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                             const void* Ks, const void* Vs, int n_frames, int step_is_final,
                             void* O, float* lse, sa_stream stream);

/* Block-sparse attention ("Vidu S2 vs PixVerse R2：实时视频的两条技术路线", section
 * 选择四：速度从哪里来: PixVerse R2 learns block-sparse attention and skips more than
 * 90 % of the blocks). Same as sa_attend, but only the blocks flagged in
 * block_mask are attended: a block is 128 query rows (tile qt: rows 128*qt ..)
 * x 128 keys of the attended key sequence (the attended chunks in ascending id
 * order, each cut into 128-key tiles from its first token, the last tile of a
 * chunk possibly short). block_mask: device uint8 [B][H][n_q_tiles][n_k_tiles]
 * (nonzero = attended); read only. n_k_tiles is the sum over the attended chunks
 * of ceil(keys / 128): sa_block_grid gives it when every chunk has F frames,
 * sa_stream_plan's lens in general. Three launches on the stream: the key
 * staging of sa_stage_keys, the mask packed into bit rows in the handle's
 * buffer (so block_mask may be rewritten once the call's work has run), and
 * the attention. Only flagged blocks are loaded and multiplied (a key tile that
 * both query tiles of a 256-row pair flag at the same step is loaded once).
 * A row that sees no key gets O = 0
 * and lse = -inf. The reference image is not part of the block grid: with a
 * reference set this call returns SA_ERR_UNSUPPORTED. */
SA_API int sa_attend_sparse(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                            int step_is_final, const uint8_t* block_mask, void* O, float* lse,
                            sa_stream stream);

/* Block grid of chunk `chunk`'s attention for config cfg: *n_q_tiles =
 * ceil(L / 128), *n_k_tiles = (attended chunks) * ceil(L / 128). Host only. */
SA_API int sa_block_grid(const sa_config* cfg, int32_t chunk, int32_t* n_q_tiles,
                         int32_t* n_k_tiles);

/* The two halves of sa_attend, for callers that time or schedule them apart.
 * sa_stage_keys rotates the generating chunk's Kc ([B, L, H, D] bf16) by its
 * in-chunk positions into the handle's key scratch (one HBM-bound kernel).
 * sa_attend_staged then runs the attention kernel over the cache and the staged
 * keys, with Vc read in place (Q, Vc, O, lse of the staged chunk's frames). sa_attend_staged requires a preceding
 * sa_stage_keys for the same chunk (else SA_ERR_STATE); the staged keys stay
 * valid until the next sa_stage_keys / sa_attend on this handle. */
SA_API int sa_stage_keys(sa_handle* h, const void* Kc, sa_stream stream);
/* sa_stage_keys for a generating chunk of n_frames <= F frames; the following
 * sa_attend_staged then takes Q, Vc, O, lse of n_frames frames. */
SA_API int sa_stage_keys_frames(sa_handle* h, const void* Kc, int n_frames, sa_stream stream);
SA_API int sa_attend_staged(sa_handle* h, const void* Q, const void* Vc, int step_is_final,
                            void* O, float* lse, sa_stream stream);

/* sa_attend for callers that cannot allocate device memory. (The pages have no
 * counterpart to this call; it exists for integration.)
 * Some callers may not call cudaMalloc at all: code running inside another
 * framework's allocator-free region, a real-time loop that must not allocate
 * after start-up, or a plugin that is handed only the tensors it works on.
 * This call computes exactly what sa_attend computes, with the same arguments,
 * but it allocates nothing and does not use the handle's key scratch: the
 * generating chunk's rotated keys go to a fixed array of
 * SA_NOALLOC_MAX_KEY_BYTES (64 MiB) compiled into the library. Every device
 * that loads the library holds that array until the process exits.
 * Limits and rules:
 *  - B * H * L * D * 2 bytes must fit in SA_NOALLOC_MAX_KEY_BYTES, else
 *    SA_ERR_UNSUPPORTED and nothing is launched;
 *  - the array is shared by every call in the process on that device and keeps
 *    the last call's keys: calls that overlap on the GPU (two streams, two
 *    handles) race; order them (one stream, or events);
 *  - the first call on a device looks up the array's device address (a
 *    runtime symbol query); make that first call before any stream capture.
 *    The address is kept per device together with the CUDA context it was
 *    found in: after a device reset (cudaDeviceReset) or in a new context the
 *    first call looks it up again, so make that call, too, outside capture.
 * Returns the same statuses as sa_attend. */
#define SA_NOALLOC_MAX_KEY_BYTES (64u << 20)
SA_API int sa_attend_noalloc(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                             int step_is_final, void* O, float* lse, sa_stream stream);

/* Same contract as sa_attend, computed by a plain fp32 SIMT kernel (one warp
 * per query row, no tensor cores). A debugging cross-check of the tensor-core
 * kernel, an order of magnitude slower; not used by sa_attend. */
SA_API int sa_debug_attend_simt(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                                int step_is_final, void* O, float* lse, sa_stream stream);

/* Test hook for the failure path: runs sa_attend with the kernel's TMA producer
 * switched off, so the MMA warp's wait for the first key tile runs out (about
 * one second). The kernel then drains, frees its tensor memory and sets the
 * device status word: sa_get_status returns SA_ERR_TIMEOUT until sa_reset. O is
 * left unspecified. The CUDA context stays usable. */
SA_API int sa_debug_attend_stalled(sa_handle* h, const void* Q, const void* Kc, const void* Vc,
                                   int step_is_final, void* O, sa_stream stream);

/* Evaluate the attention kernel's device exponentials on n fp32 values (device
 * pointers x, y): use_polynomial = 0 -> the exp unit (ex2.approx), 1 -> the
 * FMA-pipe polynomial 2^x used for part of the softmax (degree-3 minimax fit,
 * relative error <= 7.5e-5 for x >= -125; x below -125 gives 2^-125). A test
 * hook for the kernel's arithmetic; asynchronous on `stream`. */
SA_API int sa_debug_exp2(int use_polynomial, const float* x, float* y, int n, sa_stream stream);

/* Clock record of the most recent attention kernel (tensor-core path) that ran
 * on the calling thread's current device, from any handle: every CTA stamps
 * the global timer and its SM cycle counter when it starts and when it ends.
 * *sm_mhz = the median over the CTAs of (SM cycles / timer ns) * 1000, the
 * clock the kernel's SMs actually ran at (the clock a management library
 * reports can stay at its maximum while the SMs run slower under power
 * management); *span_us = first CTA start to last CTA end. Synchronizes the
 * device first. SA_ERR_STATE when no attention has run on this device in this
 * process; SA_ERR_CUDA without a usable device. Launches on several streams
 * overwrite one record. */
SA_API int sa_debug_kernel_clock(double* sm_mhz, double* span_us);

/* Test hook for the host error path: the next call of this handle that would
 * launch device work fails with SA_ERR_CUDA before launching anything (as a
 * failed CUDA call would), leaving the handle's state unchanged; later calls
 * work again. No device work, no fault. */
SA_API int sa_debug_inject_cuda_error(sa_handle* h);

/* Chunks appended so far to `tier`, or a negative sa_status. */
SA_API int sa_chunk_count(const sa_handle* h, int tier);

/* Cache layout of `tier`, for bit-exact checks of the ring and the relocation
 * ("Vidu S2 vs PixVerse R2", section 选择三：有上限的记忆: sinks kept, the window
 * slides, positions relocated). For each of the first min(n, S + W - 1) slots:
 * slot_chunk_ids[s] = the chunk id the slot holds (-1 = empty), and, if
 * slot_ranks is not NULL, slot_ranks[s] = the rank of that chunk among the
 * chunks the next attention of this tier reads (the held chunks in ascending
 * id order, then the generating chunk; -1 = empty slot). The chunk's temporal
 * base is ref_frames + rank * F when every chunk has F frames (sa_stream_plan
 * gives the bases for chunks of any length). Returns the number of slots
 * written, or a negative sa_status. Host only. */
SA_API int sa_debug_layout(const sa_handle* h, int tier, int32_t* slot_chunk_ids,
                           int32_t* slot_ranks, int n);

/* The attention plan of chunk `chunk` of a stream with config cfg whose chunks
 * all have F frames, computed on the host with no handle and no device: writes,
 * for each attended chunk in ascending id order, its id, its cache slot (-1 for
 * the chunk itself) and its relocated temporal base ref_frames + rank * F.
 * Returns the count (<= S + W) or a negative sa_status if cap is too small. */
SA_API int sa_plan(const sa_config* cfg, int32_t chunk, int32_t* ids, int32_t* slots,
                   int32_t* t_base, int cap);

/* The attention plan the handle would run now for a generating chunk of
 * n_frames frames at the given step (host only, no device work): for each
 * attended chunk in ascending id order its id, its relocated temporal base
 * (ref_frames + the frames of the attended chunks before it, from the frames
 * the selected tier actually stored) and its number of keys. The reference
 * image is not listed (it always sits at 0). Returns the count or a negative
 * sa_status (tiers out of step, bad n_frames, cap too small). */
SA_API int sa_stream_plan(const sa_handle* h, int step_is_final, int n_frames, int32_t* ids,
                          int32_t* t_base, int32_t* lens, int cap);

/* ---- Ulysses head sharding across GPUs ("Vidu S2：实时可交互、可编辑、可立体的视频生成",
 * section 2.4; "Vidu S2 vs PixVerse R2", section 选择四：速度从哪里来: multi-GPU runs
 * split load and activations with Ulysses context parallelism and quantise the
 * tensors the GPUs exchange). G ranks each hold a contiguous 1/G of a chunk's
 * tokens with all heads; an all-to-all gives each rank all tokens of H/G heads
 * before attention, and a second one returns the output to token shards.
 * These two calls are the local halves of such an exchange; the all-to-all of
 * the G equal blocks between them is the caller's (NCCL over NVLink in the
 * Python layer).
 *
 * x: [B, T, C, D] bf16 on the device (T tokens, C heads), 16-byte aligned.
 * split_dim 1 (heads, before attention): block g holds heads g*C/G .. of every
 * token; split_dim 0 (tokens, after attention): block g holds tokens g*T/G ..
 * with every head. The split dimension must be a multiple of G.
 * Payload SA_PAYLOAD_FP8: each (b, t, c) vector of D values is sent as fp8
 * e4m3 codes (scale = max|x| / 448, inv = 448 / max|x|, code = e4m3(x * inv),
 * nearest even, saturating; each an IEEE fp32 operation) followed by its fp32
 * scale, D + 4 bytes
 * instead of 2 D; on arrival code * scale (fp32) rounded to bf16. An all-zero
 * vector has scale 0. SA_PAYLOAD_BF16 sends the values unchanged. Inputs must
 * be finite.
 * buf: G blocks of sa_exchange_block_bytes(...) bytes each, block g for rank g.
 * sa_exchange_unpack takes the G blocks received (block s from rank s; every
 * sender used the same B, T, C, D, G, split_dim, payload, which the call
 * repeats) and writes y: split_dim 1 -> [B, G*T, C/G, D] (token shards in rank
 * order); split_dim 0 -> [B, T/G, G*C, D] (head groups in rank order).
 * Asynchronous on `stream`; SA_ERR_INVALID_ARG on a bad shape or pointer. */
#define SA_PAYLOAD_FP8 0
#define SA_PAYLOAD_BF16 1
SA_API size_t sa_exchange_block_bytes(int B, int T, int C, int D, int G, int split_dim,
                                      int payload); /* 0 if invalid; host only */
SA_API int sa_exchange_pack(const void* x, int B, int T, int C, int D, int G, int split_dim,
                            int payload, void* buf, sa_stream stream);
SA_API int sa_exchange_unpack(const void* buf, int B, int T, int C, int D, int G, int split_dim,
                              int payload, void* y, sa_stream stream);

/* sa_exchange_pack that writes block g straight to dst_blocks[g] (a host array
 * of G device pointers, each 16-byte aligned, e.g. this rank's slot in rank g's
 * receive buffer mapped with sa_ipc_open): quantisation and transfer in one
 * pass over peer memory, no staging copy, no separate collective. The caller
 * orders the receivers' sa_exchange_unpack after every sender's launch (a
 * barrier) and keeps a receiver from reusing a buffer that a sender may still
 * be writing (two receive buffers used in turn). G <= 64. */
SA_API int sa_exchange_pack_to(const void* x, int B, int T, int C, int D, int G, int split_dim,
                               int payload, void* const* dst_blocks, sa_stream stream);

/* CUDA IPC of device buffers between processes (the peer mappings of
 * sa_exchange_pack_to): sa_ipc_alloc / sa_ipc_free make and release a whole
 * cudaMalloc allocation on the current device (a receive buffer; the only
 * allocations this library makes itself); sa_ipc_handle writes the
 * SA_IPC_HANDLE_BYTES-byte handle of such an allocation (dev_ptr = its start);
 * sa_ipc_open maps another process's handle into this one (peer access enabled
 * on first use); sa_ipc_close unmaps it. A handle cannot be opened in the
 * process that made it. */
#define SA_IPC_HANDLE_BYTES 64
SA_API int sa_ipc_alloc(size_t bytes, void** dev_ptr_out);
SA_API int sa_ipc_free(void* dev_ptr);
SA_API int sa_ipc_handle(const void* dev_ptr, void* handle_out);
SA_API int sa_ipc_open(const void* handle, void** dev_ptr_out);
SA_API int sa_ipc_close(void* dev_ptr);

/* Slot of chunk id `chunk` in a tier (-1 if it is never stored). Host only. */
SA_API int sa_slot_of(const sa_config* cfg, int32_t chunk);

/* Wait for `stream`, then read and return the device status word: SA_OK;
 * SA_ERR_TIMEOUT if a kernel gave up a bounded wait since the last reset;
 * else SA_ERR_BOUNDS (checked build only, see sa_build_info) if a kernel
 * skipped an out-of-range access; else SA_ERR_RANGE if a rotated Q or K pair
 * of some call since the last reset had a norm above 65504 and was saturated
 * to fp16 (the outputs were computed with the saturated values). */
SA_API int sa_get_status(sa_handle* h, sa_stream stream);

/* Text of the handle's last error (never NULL); with h == NULL, of the last
 * error of a call that had no handle yet (sa_create). */
SA_API const char* sa_last_error(const sa_handle* h);

/* Build flags of the loaded library: SA_BUILD_DEVICE_CHECKS is set in the
 * checked build (libsa_checked.so, the same sources compiled with
 * SA_DEVICE_CHECKS): there every kernel of the attention path (key staging,
 * appends, the reference image, mask packing, the tensor-core and SIMT
 * attention) compares the end of each direct global load or store with the
 * size of its buffer before making it; an access past the end is skipped and
 * recorded in the device status word (sa_get_status -> SA_ERR_BOUNDS). A
 * debugging aid in place of a memory checker; the release build (libsa.so)
 * has no checks. Host only. */
#define SA_BUILD_DEVICE_CHECKS 1
SA_API int sa_build_info(void);

/* Name of an sa_status value. */
SA_API const char* sa_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* BLOCK_CAUSAL_STREAMING_SA_H */

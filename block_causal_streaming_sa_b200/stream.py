"""Torch-facing wrapper around one libsa handle (argument checks and marshalling).

PyTorch provides the device buffer and the current stream; the work itself is
done by the library's kernels through the C ABI.
"""

import torch

from . import _binding as B


class StreamingAttention:
    """One attention layer's sink + window TwinCache on the current CUDA device.

    ``cfg`` is a dict with the sa_config fields (batch, heads, head_dim,
    frames_per_chunk, tok_h, tok_w, sink_chunks, window_chunks and optionally
    softmax_scale, rope_theta, ref_frames). Tensors are bf16 [B, L, H, D],
    contiguous, on the device the object was created on; a chunk may have fewer
    frames than frames_per_chunk (L = frames * tok_h * tok_w).
    """

    def __init__(self, cfg, device=None):
        self.cfg_dict = dict(cfg)
        self.cfg = B.make_config(**self.cfg_dict)
        nbytes = B.sa_required_bytes(self.cfg)
        if nbytes == 0:
            raise B.SaError(B.sa_validate_config(self.cfg), B.last_error())
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        with torch.cuda.device(self.device):
            self.buffer = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            self.handle = B.sa_create(self.cfg, self.buffer.data_ptr(), nbytes)
        c = self.cfg_dict
        self.frame_tokens = c["tok_h"] * c["tok_w"]
        self.frames = c["frames_per_chunk"]
        self.shape = self._shape(self.frames)

    # -- helpers
    def _shape(self, frames):
        c = self.cfg_dict
        return (c["batch"], frames * self.frame_tokens, c["heads"], c["head_dim"])

    def _frames_of(self, t, name):
        n = t.shape[1] // self.frame_tokens if t.dim() == 4 else 0
        if not 1 <= n <= self.frames:
            raise ValueError(f"{name} must hold 1..{self.frames} frames of {self.frame_tokens} "
                             f"tokens")
        return n

    def _ptr(self, t, name, frames=None):
        shape = self._shape(self.frames if frames is None else frames)
        if t.dtype != torch.bfloat16 or tuple(t.shape) != shape or not t.is_contiguous() \
                or t.device != self.device:
            raise ValueError(f"{name} must be a contiguous bf16 tensor of shape {shape} "
                             f"on {self.device}")
        return t.data_ptr()

    def _stream(self, stream):
        s = torch.cuda.current_stream(self.device) if stream is None else stream
        return s.cuda_stream

    # -- the calls
    def append(self, tier, K, V, stream=None):
        """Append a chunk (any 1..F frames) to one tier."""
        n = self._frames_of(K, "K")
        k, v = self._ptr(K, "K", n), self._ptr(V, "V", n)
        if n == self.frames:
            B.sa_append_chunk(self.handle, tier, k, v, self._stream(stream))
        else:
            B.sa_append_chunk_frames(self.handle, tier, k, v, n, self._stream(stream))

    def set_reference(self, K, V, stream=None):
        """Set or replace the reference image (ref_frames frames); None clears it."""
        if K is None and V is None:
            B.sa_set_reference(self.handle, 0, 0, self._stream(stream))
            return
        n = self.cfg_dict.get("ref_frames", 0)
        shape = self._shape(n)
        for t, name in ((K, "K"), (V, "V")):
            if t is None or t.dtype != torch.bfloat16 or tuple(t.shape) != shape \
                    or not t.is_contiguous() or t.device != self.device:
                raise ValueError(f"reference {name} must be contiguous bf16 {shape}")
        B.sa_set_reference(self.handle, K.data_ptr(), V.data_ptr(), self._stream(stream))

    def attend(self, Q, Kc, Vc, step_is_final, out=None, lse=None, stream=None, simt=False):
        """Attention of the generating chunk (any 1..F frames, from Q's shape)."""
        n = self._frames_of(Q, "Q")
        shape = self._shape(n)
        if out is None:
            out = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        lse_ptr = 0
        if lse is not None:
            b, l, h, _ = shape
            if lse.dtype != torch.float32 or tuple(lse.shape) != (b, h, l) \
                    or not lse.is_contiguous():
                raise ValueError(f"lse must be contiguous fp32 of shape {(b, h, l)}")
            lse_ptr = lse.data_ptr()
        ptrs = (self._ptr(Q, "Q", n), self._ptr(Kc, "Kc", n), self._ptr(Vc, "Vc", n))
        if simt:
            if n != self.frames:
                raise ValueError("the SIMT debug path takes whole chunks only")
            B.sa_debug_attend_simt(self.handle, *ptrs, step_is_final, self._ptr(out, "O"),
                                   lse_ptr, self._stream(stream))
        elif n == self.frames:
            B.sa_attend(self.handle, *ptrs, step_is_final, self._ptr(out, "O"), lse_ptr,
                        self._stream(stream))
        else:
            B.sa_attend_frames(self.handle, *ptrs, n, step_is_final, self._ptr(out, "O", n),
                               lse_ptr, self._stream(stream))
        return out

    def attend_aligned(self, Q, Kc, Vc, Ks, Vs, step_is_final, out=None, lse=None, stream=None):
        """Frame-aligned editing attention: the usual keys plus, for each query
        token, the source tokens Ks/Vs of its own frame (same shape as Q)."""
        n = self._frames_of(Q, "Q")
        shape = self._shape(n)
        if out is None:
            out = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        lse_ptr = 0
        if lse is not None:
            b, l, h, _ = shape
            if lse.dtype != torch.float32 or tuple(lse.shape) != (b, h, l) \
                    or not lse.is_contiguous():
                raise ValueError(f"lse must be contiguous fp32 of shape {(b, h, l)}")
            lse_ptr = lse.data_ptr()
        ptrs = [self._ptr(t, name, n) for t, name in
                ((Q, "Q"), (Kc, "Kc"), (Vc, "Vc"), (Ks, "Ks"), (Vs, "Vs"))]
        B.sa_attend_aligned(self.handle, *ptrs, n, step_is_final, self._ptr(out, "O", n), lse_ptr,
                            self._stream(stream))
        return out

    def plan(self, step_is_final, n_frames=None):
        """(ids, t_base, lens) the next attention would use."""
        return B.sa_stream_plan(self.handle, step_is_final,
                                self.frames if n_frames is None else n_frames)

    def attend_sparse(self, Q, Kc, Vc, step_is_final, block_mask, out=None, lse=None,
                      stream=None):
        """Block-sparse attention; block_mask: uint8 [B, H, n_q_tiles, n_k_tiles] on the device."""
        b, l, h, _ = self.shape
        nq, nk = self.block_grid(step_is_final)
        if block_mask.dtype != torch.uint8 or tuple(block_mask.shape) != (b, h, nq, nk) \
                or not block_mask.is_contiguous() or block_mask.device != self.device:
            raise ValueError(f"block_mask must be contiguous uint8 {(b, h, nq, nk)} on {self.device}")
        if out is None:
            out = torch.empty(self.shape, dtype=torch.bfloat16, device=self.device)
        lse_ptr = 0 if lse is None else lse.data_ptr()
        B.sa_attend_sparse(self.handle, self._ptr(Q, "Q"), self._ptr(Kc, "Kc"), self._ptr(Vc, "Vc"),
                           step_is_final, block_mask.data_ptr(), self._ptr(out, "O"), lse_ptr,
                           self._stream(stream))
        return out

    def block_grid(self, step_is_final):
        """(n_q_tiles, n_k_tiles) of the block mask of the next whole-chunk
        attention: 128-key tiles of each attended chunk, from the frames stored."""
        _, _, lens = self.plan(step_is_final)
        return -(-self.shape[1] // 128), sum(-(-n // 128) for n in lens)

    def reset(self):
        B.sa_reset(self.handle)

    def status(self, stream=None):
        return B.sa_get_status(self.handle, self._stream(stream))

    def chunk_count(self, tier):
        return B.sa_chunk_count(self.handle, tier)

    def layout(self, tier):
        """Chunk id held by each slot of the tier (-1: empty)."""
        return self.layout_ranks(tier)[0]

    def layout_ranks(self, tier):
        """(chunk id per slot, rank of that chunk in the next attention's list)."""
        c = self.cfg_dict
        return B.sa_debug_layout(self.handle, tier, c["sink_chunks"] + c["window_chunks"] - 1)

    def close(self):
        if getattr(self, "handle", None) is not None:
            B.sa_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

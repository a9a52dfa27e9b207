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
    softmax_scale, rope_theta). Tensors are bf16 [B, L, H, D], contiguous, on
    the device the object was created on.
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
        self.shape = (c["batch"], c["frames_per_chunk"] * c["tok_h"] * c["tok_w"], c["heads"],
                      c["head_dim"])

    # -- helpers
    def _ptr(self, t, name):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != self.shape or not t.is_contiguous() \
                or t.device != self.device:
            raise ValueError(f"{name} must be a contiguous bf16 tensor of shape {self.shape} "
                             f"on {self.device}")
        return t.data_ptr()

    def _stream(self, stream):
        s = torch.cuda.current_stream(self.device) if stream is None else stream
        return s.cuda_stream

    # -- the four calls
    def append(self, tier, K, V, stream=None):
        B.sa_append_chunk(self.handle, tier, self._ptr(K, "K"), self._ptr(V, "V"),
                          self._stream(stream))

    def attend(self, Q, Kc, Vc, step_is_final, out=None, lse=None, stream=None, simt=False):
        if out is None:
            out = torch.empty(self.shape, dtype=torch.bfloat16, device=self.device)
        lse_ptr = 0
        if lse is not None:
            b, l, h, _ = self.shape
            if lse.dtype != torch.float32 or tuple(lse.shape) != (b, h, l) \
                    or not lse.is_contiguous():
                raise ValueError(f"lse must be contiguous fp32 of shape {(b, h, l)}")
            lse_ptr = lse.data_ptr()
        fn = B.sa_debug_attend_simt if simt else B.sa_attend
        fn(self.handle, self._ptr(Q, "Q"), self._ptr(Kc, "Kc"), self._ptr(Vc, "Vc"),
           step_is_final, self._ptr(out, "O"), lse_ptr, self._stream(stream))
        return out

    def attend_sparse(self, Q, Kc, Vc, step_is_final, block_mask, out=None, lse=None,
                      stream=None):
        """Block-sparse attention; block_mask: uint8 [B, H, n_q_tiles, n_k_tiles] on the device."""
        b, l, h, _ = self.shape
        nq, nk = B.sa_block_grid(self.cfg, self.chunk_count(B.SA_TIER_NOISY))
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

    def reset(self):
        B.sa_reset(self.handle)

    def status(self, stream=None):
        return B.sa_get_status(self.handle, self._stream(stream))

    def chunk_count(self, tier):
        return B.sa_chunk_count(self.handle, tier)

    def layout(self, tier):
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

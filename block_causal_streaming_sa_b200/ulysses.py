"""Ulysses head sharding of the streaming attention across the ranks of a
process group, with a quantised all-to-all payload.

"Vidu S2：实时可交互、可编辑、可立体的视频生成", section 2.4, and "Vidu S2 vs PixVerse R2",
section 选择四：速度从哪里来: several GPUs split the load and the activation memory
with Ulysses context parallelism and quantise the tensors they exchange.

Each rank holds a contiguous 1/G of every chunk's tokens with all H heads (the
layout of the surrounding model). Before attention one all-to-all per tensor
(Q, Kc, Vc, appended K/V, reference, source frames) gives each rank all tokens
of its H/G heads; the rank runs the single-GPU streaming attention on them
with its own two-tier cache; one all-to-all brings O back to token shards. The
local halves of every exchange are the library's pack / unpack kernels
(fp8 e4m3 payload with a per-vector scale, or bf16); the exchange itself is
one NCCL all-to-all of G equal byte blocks per tensor over NVLink.
"""

import torch
import torch.distributed as dist

from . import _binding as B
from .stream import StreamingAttention


def all_to_all_blocks(buf, group=None):
    """Exchange G equal blocks: block g of this rank goes to rank g; block s of the
    result came from rank s. One process (G = 1) returns buf itself."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world == 1:
        return buf
    out = torch.empty_like(buf)
    dist.all_to_all_single(out, buf, group=group)
    return out


class UlyssesAttention:
    """One attention layer's stream, head-sharded over the ranks of ``group``.

    ``cfg``: the sa_config fields of the whole layer (``heads`` = all heads H,
    a multiple of the rank count G). Tensors passed in are this rank's token
    shard, bf16 [B, L_c / G, H, D] (L_c = frames * tok_h * tok_w, a multiple of
    G); attention outputs come back the same way. ``payload``: "fp8" (quantised
    exchange) or "bf16" (exact).
    """

    def __init__(self, cfg, group=None, payload="fp8", device=None):
        self.group = group
        self.G = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.H, self.D = cfg["heads"], cfg["head_dim"]
        if self.H % self.G:
            raise ValueError(f"heads ({self.H}) must be a multiple of the rank count ({self.G})")
        self.payload = {"fp8": B.SA_PAYLOAD_FP8, "bf16": B.SA_PAYLOAD_BF16}[payload]
        self.local = StreamingAttention(dict(cfg, heads=self.H // self.G), device)
        self.device = self.local.device

    def _stream(self):
        return torch.cuda.current_stream(self.device).cuda_stream

    def _exchange(self, x, split_dim):
        """pack -> all-to-all -> unpack of one bf16 tensor [B, T, C, D]."""
        if x.dtype != torch.bfloat16 or not x.is_contiguous() or x.device != self.device:
            raise ValueError("tensors must be contiguous bf16 on the layer's device")
        b, t, c, d = x.shape
        G = self.G
        nbytes = B.sa_exchange_block_bytes(b, t, c, d, G, split_dim, self.payload)
        if nbytes == 0:
            raise B.SaError(B.SA_ERR_INVALID_ARG, B.last_error())
        send = torch.empty(G * nbytes, dtype=torch.uint8, device=self.device)
        B.sa_exchange_pack(x.data_ptr(), b, t, c, d, G, split_dim, self.payload, send.data_ptr(),
                           self._stream())
        recv = all_to_all_blocks(send, self.group)
        shape = (b, G * t, c // G, d) if split_dim == 1 else (b, t // G, G * c, d)
        y = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        B.sa_exchange_unpack(recv.data_ptr(), b, t, c, d, G, split_dim, self.payload, y.data_ptr(),
                             self._stream())
        return y

    def to_heads(self, x):
        """Token shard [B, T, H, D] -> all tokens of this rank's heads [B, G*T, H/G, D]."""
        return self._exchange(x, 1)

    def to_tokens(self, o):
        """This rank's heads [B, L, H/G, D] -> its token shard [B, L/G, H, D]."""
        return self._exchange(o, 0)

    def append(self, tier, K, V):
        self.local.append(tier, self.to_heads(K), self.to_heads(V))

    def set_reference(self, K, V):
        if K is None and V is None:
            self.local.set_reference(None, None)
        else:
            self.local.set_reference(self.to_heads(K), self.to_heads(V))

    def attend(self, Q, Kc, Vc, step_is_final):
        o = self.local.attend(self.to_heads(Q), self.to_heads(Kc), self.to_heads(Vc),
                              step_is_final)
        return self.to_tokens(o)

    def attend_aligned(self, Q, Kc, Vc, Ks, Vs, step_is_final):
        o = self.local.attend_aligned(*(self.to_heads(t) for t in (Q, Kc, Vc, Ks, Vs)),
                                      step_is_final)
        return self.to_tokens(o)

    def status(self, stream=None):
        return self.local.status(stream)

    def close(self):
        self.local.close()

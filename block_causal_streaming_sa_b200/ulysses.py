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


def _world(group):
    return dist.get_world_size(group) if dist.is_initialized() else 1


def all_to_all_blocks(buf, group=None):
    """Exchange G equal blocks: block g of this rank goes to rank g; block s of the
    result came from rank s. One process (G = 1) returns buf itself."""
    if _world(group) == 1:
        return buf
    out = torch.empty_like(buf)
    dist.all_to_all_single(out, buf, group=group)
    return out


class PeerExchange:
    """Transport that writes each block straight into the receiving rank's
    buffer: every rank owns two receive buffers (used in turn) made with
    sa_ipc_alloc, maps every peer's pair with CUDA IPC once, and per exchange
    runs sa_exchange_pack_to (quantise and store over NVLink in one kernel), a
    barrier, and sa_exchange_unpack from its own buffer. The barrier is an
    all-reduce of one integer on the current stream for NCCL groups, or a stream
    synchronise plus a host barrier for other backends. Two buffers used in turn
    keep a fast sender from overwriting a buffer a slow receiver still reads: a
    sender reaches exchange k + 2 only after the barrier of exchange k + 1, which
    every receiver passes only after unpacking exchange k."""

    def __init__(self, nbytes, group, device):
        self.group, self.device = group, device
        self.G, self.rank = _world(group), (dist.get_rank(group) if dist.is_initialized() else 0)
        self.nbytes = nbytes  # capacity of one receive buffer (G blocks)
        self.own = [B.sa_ipc_alloc(nbytes) for _ in range(2)]
        self.peer = [list(self.own) for _ in range(self.G)]
        if self.G > 1:
            handles = [B.sa_ipc_handle(p) for p in self.own]
            every = [None] * self.G
            dist.all_gather_object(every, handles, group=group)
            for g in range(self.G):
                if g != self.rank:
                    self.peer[g] = [B.sa_ipc_open(h) for h in every[g]]
        self.turn = 0
        self.nccl = self.G > 1 and dist.get_backend(group) == "nccl"
        self.flag = torch.zeros(1, dtype=torch.int32, device=device)

    def barrier(self):
        if self.G == 1:
            return
        if self.nccl:
            dist.all_reduce(self.flag, group=self.group)
        else:
            torch.cuda.current_stream(self.device).synchronize()
            dist.barrier(group=self.group)

    def exchange(self, x, split_dim, payload, stream):
        b, t, c, d = x.shape
        G = self.G
        n = B.sa_exchange_block_bytes(b, t, c, d, G, split_dim, payload)
        if n == 0:
            raise B.SaError(B.SA_ERR_INVALID_ARG, B.last_error())
        if G * n > self.nbytes:
            raise ValueError(f"exchange of {G * n} bytes exceeds the receive buffers ({self.nbytes})")
        k, self.turn = self.turn, self.turn ^ 1
        dst = [self.peer[g][k] + self.rank * n for g in range(G)]
        B.sa_exchange_pack_to(x.data_ptr(), b, t, c, d, G, split_dim, payload, dst, stream)
        self.barrier()
        shape = (b, G * t, c // G, d) if split_dim == 1 else (b, t // G, G * c, d)
        y = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        B.sa_exchange_unpack(self.own[k], b, t, c, d, G, split_dim, payload, y.data_ptr(), stream)
        return y

    def close(self):
        if self.own is None:
            return
        torch.cuda.synchronize(self.device)
        self.barrier()  # no peer still writes into our buffers
        for g in range(self.G):
            if g != self.rank:
                for p in self.peer[g]:
                    B.sa_ipc_close(p)
        for p in self.own:
            B.sa_ipc_free(p)
        self.own = None


class UlyssesAttention:
    """One attention layer's stream, head-sharded over the ranks of ``group``.

    ``cfg``: the sa_config fields of the whole layer (``heads`` = all heads H,
    a multiple of the rank count G). Tensors passed in are this rank's token
    shard, bf16 [B, L_c / G, H, D] (L_c = frames * tok_h * tok_w, a multiple of
    G); attention outputs come back the same way. ``payload``: "fp8" (quantised
    exchange) or "bf16" (exact). ``transport``: "nccl" (pack, one all-to-all,
    unpack) or "p2p" (pack straight into the peers' receive buffers, see
    PeerExchange).
    """

    def __init__(self, cfg, group=None, payload="fp8", device=None, transport="nccl"):
        self.group = group
        self.G = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.H, self.D = cfg["heads"], cfg["head_dim"]
        if self.H % self.G:
            raise ValueError(f"heads ({self.H}) must be a multiple of the rank count ({self.G})")
        self.payload = {"fp8": B.SA_PAYLOAD_FP8, "bf16": B.SA_PAYLOAD_BF16}[payload]
        self.local = StreamingAttention(dict(cfg, heads=self.H // self.G), device)
        self.device = self.local.device
        self.peer = None
        if transport == "p2p":
            # receive buffers sized for the largest exchange of this layer: a whole
            # chunk (or the reference image) of all heads, either direction
            L = max(cfg["frames_per_chunk"], cfg.get("ref_frames", 0)) * cfg["tok_h"] * cfg["tok_w"]
            cap = max(B.sa_exchange_block_bytes(cfg["batch"], L // self.G, self.H, self.D, self.G,
                                                1, self.payload),
                      B.sa_exchange_block_bytes(cfg["batch"], L, self.H // self.G, self.D,
                                                self.G, 0, self.payload))
            if cap == 0:
                raise ValueError("chunk and reference tokens must be multiples of the rank count")
            self.peer = PeerExchange(self.G * cap, group, self.device)
        elif transport != "nccl":
            raise ValueError(f"unknown transport {transport!r}")

    def _stream(self):
        return torch.cuda.current_stream(self.device).cuda_stream

    def _exchange(self, x, split_dim):
        """pack -> all-to-all -> unpack of one bf16 tensor [B, T, C, D]."""
        if x.dtype != torch.bfloat16 or not x.is_contiguous() or x.device != self.device:
            raise ValueError("tensors must be contiguous bf16 on the layer's device")
        if self.peer is not None:
            return self.peer.exchange(x, split_dim, self.payload, self._stream())
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
        if self.peer is not None:
            self.peer.close()
            self.peer = None
        self.local.close()

"""One chunk's attention over the sink + window TwinCache, float64.
(Oracle: test infrastructure only.)

What is computed for the chunk c being generated, at one denoising step:

1. Tier ([orkas] section 选择三, TwinCache): the final denoising step reads
   the clean copy of every cached chunk, every earlier step the noisy copy
   (reading R6: sinks too).
2. Attended chunks ([orkas] sections 「实时」改变了什么 and 选择三; [s2read]
   section 2.2): the cached sink and window chunks, all earlier than c, plus c
   itself (R2: all of c's own tokens). Listed ascending by chunk id.
3. Positions ([orkas] section 选择三, RoPE relocation): chunk j gets the rank
   r(j) = its index in that list; frame f of chunk j sits at temporal position
   r(j) * F + f, so positions stay below (S + W) * F however long the stream
   runs (R3). Rows and columns keep their in-frame coordinates.
4. Every key and every query is rotated at its position ([s2read]
   abbreviation table; reading R4), then plain softmax attention with scale
   1/sqrt(D) (R5) runs over the materialised key list.

``masked_full_attention`` computes the same thing a second way, as full
attention over every chunk of the stream so far under a block mask, for the
"sink + window equals masked full attention" check.
"""

from dataclasses import dataclass

import numpy as np

from .attention import softmax_attention
from .cache import RingCacheModel
from .rope import rotate, token_positions

NOISY, CLEAN = 0, 1


@dataclass(frozen=True)
class OracleConfig:
    batch: int
    heads: int
    head_dim: int
    frames: int
    tok_h: int
    tok_w: int
    sink: int
    window: int
    scale: float = 0.0  # <= 0 means 1/sqrt(head_dim)
    theta: float = 10000.0

    @property
    def chunk_len(self):
        return self.frames * self.tok_h * self.tok_w

    @property
    def softmax_scale(self):
        return self.scale if self.scale > 0 else 1.0 / np.sqrt(self.head_dim)


def _f64(x):
    return np.asarray(x, dtype=np.float64)


class StreamOracle:
    """Holds the appended K/V of both tiers and answers attention queries.

    Tensors are [B, L, H, D] arrays (any float dtype; kept as float64).
    With ``keep_history`` every appended chunk is also kept after eviction,
    for the masked full-stream check and causality tests.
    """

    def __init__(self, cfg, keep_history=False):
        self.cfg = cfg
        self.model = {t: RingCacheModel(cfg.sink, cfg.window) for t in (NOISY, CLEAN)}
        self.store = {NOISY: {}, CLEAN: {}}
        self.keep_history = keep_history
        self.history = {NOISY: {}, CLEAN: {}}

    def append(self, tier, K, V):
        """Append the next chunk's K/V to ``tier``; return (slot, evicted id)."""
        cid = self.model[tier].count
        slot, evicted = self.model[tier].append()
        kv = (_f64(K), _f64(V))
        if slot is not None:
            self.store[tier][cid] = kv
        if evicted is not None and evicted != cid:
            del self.store[tier][evicted]
        if self.keep_history:
            self.history[tier][cid] = kv
        return slot, evicted

    def current_chunk(self):
        n_noisy, n_clean = self.model[NOISY].count, self.model[CLEAN].count
        if n_noisy != n_clean:
            raise RuntimeError("both tiers must hold the same chunks before attending")
        return n_noisy

    def attended(self, final):
        """(ascending attended chunk ids, rank map) of the current chunk."""
        self.current_chunk()
        model = self.model[CLEAN if final else NOISY]
        return model.attended(), model.ranks()

    def attend(self, Q, Kc, Vc, final, rows=None, heads=None, batches=None):
        """Attention output of the current chunk.

        Q, Kc, Vc: [B, L, H, D] of the current chunk (unrotated).
        ``rows``/``heads``/``batches`` restrict which outputs are computed.
        Returns (O [nb, nrows, nh, D], lse [nb, nh, nrows]) in float64.
        """
        cfg = self.cfg
        c = self.current_chunk()
        tier = CLEAN if final else NOISY
        ids, rank = self.attended(final)
        L, F = cfg.chunk_len, cfg.frames
        rows = np.arange(L) if rows is None else np.asarray(rows)
        heads = range(cfg.heads) if heads is None else heads
        batches = range(cfg.batch) if batches is None else batches
        f, y, x = token_positions(L, cfg.tok_h, cfg.tok_w)
        Q, Kc, Vc = _f64(Q), _f64(Kc), _f64(Vc)

        O = np.zeros((len(batches), len(rows), len(heads), cfg.head_dim))
        lse = np.zeros((len(batches), len(heads), len(rows)))
        for bi, b in enumerate(batches):
            for hi, h in enumerate(heads):
                keys, vals = [], []
                for j in ids:
                    Kj, Vj = (Kc, Vc) if j == c else self.store[tier][j]
                    keys.append(rotate(Kj[b, :, h, :], rank[j] * F + f, y, x, cfg.theta))
                    vals.append(Vj[b, :, h, :])
                q = rotate(Q[b, rows, h, :], rank[c] * F + f[rows], y[rows], x[rows], cfg.theta)
                o, l = softmax_attention(q, np.concatenate(keys), np.concatenate(vals),
                                         cfg.softmax_scale)
                O[bi, :, hi, :] = o
                lse[bi, hi, :] = l
        return O, lse


def masked_full_attention(cfg, history, c, Q, Kc, Vc, final, rows=None):
    """The current chunk's attention as full attention over chunks 0..c.

    ``history[tier][j]`` holds (K, V) of every earlier chunk j < c, evicted
    ones included. A key of chunk j is visible to chunk c iff j <= c (block
    causal) and j is a sink chunk (j < S) or one of the W most recent chunks
    (c - j < W). A visible chunk's temporal base is F times the number of
    visible chunks before it. Returns (O [B, nrows, H, D], lse [B, H, nrows]).
    """
    tier = CLEAN if final else NOISY
    L, F, S, W = cfg.chunk_len, cfg.frames, cfg.sink, cfg.window
    rows = np.arange(L) if rows is None else np.asarray(rows)
    f, y, x = token_positions(L, cfg.tok_h, cfg.tok_w)
    visible = [j <= c and (j < S or c - j < W) for j in range(c + 1)]
    base = [F * sum(visible[:j]) for j in range(c + 1)]
    Q, Kc, Vc = _f64(Q), _f64(Kc), _f64(Vc)
    O = np.zeros((cfg.batch, len(rows), cfg.heads, cfg.head_dim))
    lse = np.zeros((cfg.batch, cfg.heads, len(rows)))
    for b in range(cfg.batch):
        for h in range(cfg.heads):
            keys, vals, seen = [], [], []
            for j in range(c + 1):
                Kj, Vj = (Kc, Vc) if j == c else history[tier][j]
                keys.append(rotate(_f64(Kj)[b, :, h, :], base[j] + f, y, x, cfg.theta))
                vals.append(_f64(Vj)[b, :, h, :])
                seen.append(np.full(L, visible[j]))
            q = rotate(Q[b, rows, h, :], base[c] + f[rows], y[rows], x[rows], cfg.theta)
            mask = np.broadcast_to(np.concatenate(seen)[None, :], (len(rows), (c + 1) * L))
            o, l = softmax_attention(q, np.concatenate(keys), np.concatenate(vals),
                                     cfg.softmax_scale, mask=mask)
            O[b, :, h, :] = o
            lse[b, h, :] = l
    return O, lse

"""One chunk's attention over the sink + window TwinCache, float64.
(Oracle: test infrastructure only.)

What is computed for the chunk c being generated, at one denoising step:

1. Tier ([orkas] section 选择三, TwinCache): the final denoising step reads
   the clean copy of every cached chunk, every earlier step the noisy copy
   (reading R6: sinks too).
2. Attended chunks ([orkas] sections 「实时」改变了什么 and 选择三; [s2read]
   section 2.2): the cached sink and window chunks, all earlier than c, plus c
   itself (R2: all of c's own tokens). Listed ascending by chunk id.
3. Positions ([orkas] section 选择三, RoPE relocation): the attended chunks get
   consecutive temporal positions in list order: chunk j starts at the number
   of frames of the attended chunks before it, so frame f of chunk j sits at
   r(j) * F + f when every chunk has F frames, and positions stay below
   (S + W) * F however long the stream runs (R3). Rows and columns keep their
   in-frame coordinates.
3a. Reference image ([s2read] section 2.2: every segment sees a shared reference
   image; [bloom] "Vidu S2 到底是什么": one shared reference keeps the identity;
   it can be replaced during the stream): reading R13, ``ref_frames`` frames of
   reference tokens on the same spatial grid sit at temporal positions
   0 .. ref_frames - 1, ahead of every chunk (whose positions shift by
   ref_frames), one clean copy, visible to every chunk at every step.
3b. Variable chunk length ([orkas] section 选择五: a chunk's length follows the
   control signal, up to a cap): reading R14, chunk j has F_j <= F frames
   (its tensors have F_j * tok_h * tok_w rows); positions as in 3.
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
    ref_frames: int = 0  # frames of the reference image (0: none)

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
        self.reference = None  # (K, V) of the reference image, [B, ref_frames*h*w, H, D]

    def set_reference(self, K, V):
        """Set (or replace; None clears) the reference image's K/V."""
        if K is None:
            self.reference = None
            return
        K, V = _f64(K), _f64(V)
        if K.shape[1] != self.cfg.ref_frames * self.cfg.tok_h * self.cfg.tok_w:
            raise ValueError("reference must have ref_frames * tok_h * tok_w tokens")
        self.reference = (K, V)

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

    def frames(self, tensor):
        return tensor.shape[1] // (self.cfg.tok_h * self.cfg.tok_w)

    def positions(self, final, current_frames):
        """Temporal base of every attended chunk: ref_frames + the frames of the
        attended chunks before it (list order)."""
        c = self.current_chunk()
        ids, _ = self.attended(final)
        tier = CLEAN if final else NOISY
        base, pos = {}, self.cfg.ref_frames
        for j in ids:
            base[j] = pos
            pos += current_frames if j == c else self.frames(self.store[tier][j][0])
        return ids, base

    def attend(self, Q, Kc, Vc, final, rows=None, heads=None, batches=None):
        """Attention output of the current chunk.

        Q, Kc, Vc: [B, L_c, H, D] of the current chunk (unrotated; L_c = F_c *
        tok_h * tok_w, F_c <= F). ``rows``/``heads``/``batches`` restrict which
        outputs are computed. Returns (O [nb, nrows, nh, D], lse [nb, nh, nrows]).
        """
        cfg = self.cfg
        c = self.current_chunk()
        tier = CLEAN if final else NOISY
        Q, Kc, Vc = _f64(Q), _f64(Kc), _f64(Vc)
        Lc = Q.shape[1]
        ids, base = self.positions(final, self.frames(Q))
        rows = np.arange(Lc) if rows is None else np.asarray(rows)
        heads = range(cfg.heads) if heads is None else heads
        batches = range(cfg.batch) if batches is None else batches
        fq, yq, xq = token_positions(Lc, cfg.tok_h, cfg.tok_w)

        O = np.zeros((len(batches), len(rows), len(heads), cfg.head_dim))
        lse = np.zeros((len(batches), len(heads), len(rows)))
        for bi, b in enumerate(batches):
            for hi, h in enumerate(heads):
                keys, vals = [], []
                if self.reference is not None:
                    Kr, Vr = self.reference
                    f, y, x = token_positions(Kr.shape[1], cfg.tok_h, cfg.tok_w)
                    keys.append(rotate(Kr[b, :, h, :], f, y, x, cfg.theta))
                    vals.append(Vr[b, :, h, :])
                for j in ids:
                    Kj, Vj = (Kc, Vc) if j == c else self.store[tier][j]
                    f, y, x = token_positions(Kj.shape[1], cfg.tok_h, cfg.tok_w)
                    keys.append(rotate(Kj[b, :, h, :], base[j] + f, y, x, cfg.theta))
                    vals.append(Vj[b, :, h, :])
                q = rotate(Q[b, rows, h, :], base[c] + fq[rows], yq[rows], xq[rows], cfg.theta)
                o, l = softmax_attention(q, np.concatenate(keys), np.concatenate(vals),
                                         cfg.softmax_scale)
                O[bi, :, hi, :] = o
                lse[bi, hi, :] = l
        return O, lse


def masked_full_attention(cfg, history, c, Q, Kc, Vc, final, rows=None, reference=None):
    """The current chunk's attention as full attention over chunks 0..c.

    ``history[tier][j]`` holds (K, V) of every earlier chunk j < c, evicted
    ones included (any number of frames each). A key of chunk j is visible to
    chunk c iff j <= c (block causal) and j is a sink chunk (j < S) or one of
    the W most recent chunks (c - j < W); the reference image, if given, is
    visible to every chunk. A visible chunk's temporal base is ref_frames plus
    the frames of the visible chunks before it. Returns (O [B, nrows, H, D],
    lse [B, H, nrows]).
    """
    tier = CLEAN if final else NOISY
    S, W, hw = cfg.sink, cfg.window, cfg.tok_h * cfg.tok_w
    Q, Kc, Vc = _f64(Q), _f64(Kc), _f64(Vc)
    Lc = Q.shape[1]
    rows = np.arange(Lc) if rows is None else np.asarray(rows)
    chunks = [history[tier][j] if j < c else (Kc, Vc) for j in range(c + 1)]
    chunks = [(_f64(K), _f64(V)) for K, V in chunks]
    visible = [j <= c and (j < S or c - j < W) for j in range(c + 1)]
    frames = [K.shape[1] // hw for K, _ in chunks]
    base = [cfg.ref_frames + sum(frames[i] for i in range(j) if visible[i]) for j in range(c + 1)]
    fq, yq, xq = token_positions(Lc, cfg.tok_h, cfg.tok_w)
    O = np.zeros((cfg.batch, len(rows), cfg.heads, cfg.head_dim))
    lse = np.zeros((cfg.batch, cfg.heads, len(rows)))
    for b in range(cfg.batch):
        for h in range(cfg.heads):
            keys, vals, seen = [], [], []
            if reference is not None:
                Kr, Vr = (_f64(t) for t in reference)
                f, y, x = token_positions(Kr.shape[1], cfg.tok_h, cfg.tok_w)
                keys.append(rotate(Kr[b, :, h, :], f, y, x, cfg.theta))
                vals.append(Vr[b, :, h, :])
                seen.append(np.full(Kr.shape[1], True))
            for j, (Kj, Vj) in enumerate(chunks):
                f, y, x = token_positions(Kj.shape[1], cfg.tok_h, cfg.tok_w)
                keys.append(rotate(Kj[b, :, h, :], base[j] + f, y, x, cfg.theta))
                vals.append(Vj[b, :, h, :])
                seen.append(np.full(Kj.shape[1], visible[j]))
            q = rotate(Q[b, rows, h, :], base[c] + fq[rows], yq[rows], xq[rows], cfg.theta)
            seen = np.concatenate(seen)
            mask = np.broadcast_to(seen[None, :], (len(rows), seen.size))
            o, l = softmax_attention(q, np.concatenate(keys), np.concatenate(vals),
                                     cfg.softmax_scale, mask=mask)
            O[b, :, h, :] = o
            lse[b, h, :] = l
    return O, lse

"""Block-sparse attention over the sink + window keys, float64.
(Oracle: test infrastructure only.)

[orkas] section 选择四：速度从哪里来: PixVerse R2 learns block-sparse attention in
training, with more than 90 % of the blocks skipped. The pages give neither the
block size nor the mask; reading R11: blocks are 128 query rows x 128 keys of
the attended key sequence (the keys of the attended chunks in ascending chunk
order, each chunk split into 128-key tiles from its first token, the last tile
of a chunk possibly short), and the mask is given by the caller, one flag per
(batch, head, query tile, key tile). A query row sees exactly the keys of the
blocks flagged for its tile; a row that sees no key has O = 0 and lse = -inf.
"""

import numpy as np

from .attention import softmax_attention
from .rope import rotate, token_positions
from .stream import CLEAN, NOISY

# (The reference image, when set, is not part of the block grid: reading R11
# covers the chunks' keys only; block_sparse_attend requires no reference.)

TILE = 128


def key_tiles(lengths, tile=TILE):
    """(chunk index, first key, last key + 1) of each key tile, in order."""
    out = []
    for g, n in enumerate(lengths):
        for s in range(0, n, tile):
            out.append((g, s, min(s + tile, n)))
    return out


def block_sparse_attend(orc, Q, Kc, Vc, final, block_mask, rows=None, heads=None, batches=None):
    """Attention of the current chunk of StreamOracle ``orc`` restricted to the
    flagged blocks. ``block_mask``: [B, H, n_q_tiles, n_key_tiles] (nonzero =
    visible). Returns (O [nb, nrows, nh, D], lse [nb, nh, nrows])."""
    cfg = orc.cfg
    c = orc.current_chunk()
    tier = CLEAN if final else NOISY
    if orc.reference is not None:
        raise ValueError("block-sparse attention takes no reference image")
    Q, Kc, Vc = (np.asarray(t, dtype=np.float64) for t in (Q, Kc, Vc))
    ids, base = orc.positions(final, orc.frames(Q))
    L = Q.shape[1]
    rows = np.arange(L) if rows is None else np.asarray(rows)
    heads = range(cfg.heads) if heads is None else heads
    batches = range(cfg.batch) if batches is None else batches
    f, y, x = token_positions(L, cfg.tok_h, cfg.tok_w)
    lengths = [L if j == c else orc.store[tier][j][0].shape[1] for j in ids]
    starts = np.concatenate([[0], np.cumsum(lengths)])
    tiles = key_tiles(lengths)

    O = np.zeros((len(batches), len(rows), len(heads), cfg.head_dim))
    lse = np.full((len(batches), len(heads), len(rows)), -np.inf)
    for bi, b in enumerate(batches):
        for hi, h in enumerate(heads):
            keys, vals = [], []
            for j in ids:
                Kj, Vj = (Kc, Vc) if j == c else orc.store[tier][j]
                fj, yj, xj = token_positions(Kj.shape[1], cfg.tok_h, cfg.tok_w)
                keys.append(rotate(Kj[b, :, h, :], base[j] + fj, yj, xj, cfg.theta))
                vals.append(Vj[b, :, h, :])
            keys, vals = np.concatenate(keys), np.concatenate(vals)
            q = rotate(Q[b, rows, h, :], base[c] + f[rows], y[rows], x[rows], cfg.theta)
            # visible keys of each query row: the keys of the flagged blocks of its tile
            mask = np.zeros((len(rows), len(keys)), dtype=bool)
            for ri, r in enumerate(rows):
                for kt, (g, s, e) in enumerate(tiles):
                    if block_mask[b, h, r // TILE, kt]:
                        mask[ri, starts[g] + s:starts[g] + e] = True
            seen = mask.any(axis=1)
            if seen.any():
                o, l = softmax_attention(q[seen], keys, vals, cfg.softmax_scale, mask=mask[seen])
                O[bi, seen, hi, :] = o
                lse[bi, hi, seen] = l
    return O, lse

"""Frame-aligned editing attention, float64.  (Oracle: test infrastructure only.)

Where the operation is described:
  [s2read] "Vidu S2：实时可交互、可编辑、可立体的视频生成", section 2.6 (the editing
          model S2-Editing): the source video and the reference image are encoded
          as condition tokens and put next to the noisy target tokens, each stream
          with its own rotary positions; every generated frame exchanges
          information only with the source frame of the same moment, never across
          moments; the reference is visible to every frame; streaming training is
          the same as for the avatar model (causal mask over the history); at
          inference each source frame is consumed together with its target frame
          and is not cached.
  [bloom] "Vidu S2：实时数字人、实时视频编辑都做到了，空间视频还只是探索", section
          "S2-Editing：把编辑搬进正在播放的视频流": each generated frame reads only
          the source frame of the same time step; reference tokens take part from
          the first frame to the last; source frames are dropped after use.
  [orkas] "Vidu S2 vs PixVerse R2：实时视频的两条技术路线", section 选择五：人怎么操控它:
          in editing mode each output frame reads only the original video's frame
          of the same moment.

Reading R15 (the pages give no formula):
  * the query rows are the target tokens of the chunk being generated;
  * a target token of frame f sees everything the generation path gives it (the
    reference image, the cached sink and window chunks of the selected tier, the
    chunk's own target tokens) plus the source tokens of frame f of the same
    chunk, and no other source token;
  * source frame f sits at the same temporal and spatial coordinates as target
    frame f (base(c) + f, row, column); the pages name a condition-specific
    rotary encoding but give none of it, so nothing is added;
  * source tokens never enter the cache.
"""

import numpy as np

from .attention import softmax_attention
from .rope import rotate, token_positions
from .stream import CLEAN, NOISY


def source_positions(f, base_c):
    """Temporal position of source frame f of the chunk whose base is base_c."""
    return base_c + f


def aligned_mask(f_rows, f_keys):
    """[rows, keys] visibility of source keys: the same frame only."""
    return f_rows[:, None] == f_keys[None, :]


def frame_aligned_attend(orc, Q, Kc, Vc, Ks, Vs, final, rows=None, heads=None, batches=None):
    """Editing attention of the current chunk of StreamOracle ``orc``.

    Q, Kc, Vc: [B, L_c, H, D] target tokens of the generating chunk (unrotated);
    Ks, Vs: [B, L_c, H, D] source tokens of the same frames (unrotated).
    Returns (O [nb, nrows, nh, D], lse [nb, nh, nrows]).
    """
    cfg = orc.cfg
    c = orc.current_chunk()
    tier = CLEAN if final else NOISY
    Q, Kc, Vc, Ks, Vs = (np.asarray(t, dtype=np.float64) for t in (Q, Kc, Vc, Ks, Vs))
    if Ks.shape != Q.shape or Vs.shape != Q.shape:
        raise ValueError("source tokens must have the shape of the target chunk")
    Lc = Q.shape[1]
    ids, base = orc.positions(final, orc.frames(Q))
    rows = np.arange(Lc) if rows is None else np.asarray(rows)
    heads = range(cfg.heads) if heads is None else heads
    batches = range(cfg.batch) if batches is None else batches
    fq, yq, xq = token_positions(Lc, cfg.tok_h, cfg.tok_w)

    O = np.zeros((len(batches), len(rows), len(heads), cfg.head_dim))
    lse = np.zeros((len(batches), len(heads), len(rows)))
    for bi, b in enumerate(batches):
        for hi, h in enumerate(heads):
            keys, vals = [], []
            if orc.reference is not None:
                Kr, Vr = orc.reference
                f, y, x = token_positions(Kr.shape[1], cfg.tok_h, cfg.tok_w)
                keys.append(rotate(Kr[b, :, h, :], f, y, x, cfg.theta))
                vals.append(Vr[b, :, h, :])
            for j in ids:
                Kj, Vj = (Kc, Vc) if j == c else orc.store[tier][j]
                f, y, x = token_positions(Kj.shape[1], cfg.tok_h, cfg.tok_w)
                keys.append(rotate(Kj[b, :, h, :], base[j] + f, y, x, cfg.theta))
                vals.append(Vj[b, :, h, :])
            n_shared = sum(k.shape[0] for k in keys)
            keys.append(rotate(Ks[b, :, h, :], source_positions(fq, base[c]), yq, xq, cfg.theta))
            vals.append(Vs[b, :, h, :])
            q = rotate(Q[b, rows, h, :], base[c] + fq[rows], yq[rows], xq[rows], cfg.theta)
            mask = np.ones((len(rows), n_shared + Lc), dtype=bool)
            mask[:, n_shared:] = aligned_mask(fq[rows], fq)
            o, l = softmax_attention(q, np.concatenate(keys), np.concatenate(vals),
                                     cfg.softmax_scale, mask=mask)
            O[bi, :, hi, :] = o
            lse[bi, hi, :] = l
    return O, lse

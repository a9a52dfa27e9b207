"""Pins of the block-sparse oracle (CPU only)."""

import math

import numpy as np
import torch

from oracle import sparse as osparse
from oracle.rope import rotate, token_positions
from oracle.stream import CLEAN, NOISY, OracleConfig, StreamOracle
from sa_inputs import normal_bf16, seed_of

RNG = np.random.default_rng(99)


def _cfg():
    # L = 2 * 10 * 14 = 280 tokens: tiles of 128, 128, 24 per chunk (ragged tail)
    return OracleConfig(1, 2, 64, 2, 10, 14, 1, 3)


def _t(cfg, tag):
    return normal_bf16(seed_of("sparse-pin", tag),
                       (cfg.batch, cfg.chunk_len, cfg.heads, cfg.head_dim)).double().numpy()


def _stream(cfg, n):
    orc = StreamOracle(cfg)
    for c in range(n):
        for tier in (NOISY, CLEAN):
            orc.append(tier, _t(cfg, ("K", c, tier)), _t(cfg, ("V", c, tier)))
    return orc


def _grid(cfg, orc):
    n_q = math.ceil(cfg.chunk_len / 128)
    ids, _ = orc.attended(True)
    n_k = len(osparse.key_tiles([cfg.chunk_len] * len(ids)))
    return n_q, n_k


def test_all_blocks_equals_dense_attention():
    cfg = _cfg()
    orc = _stream(cfg, 4)
    Q, Kc, Vc = (_t(cfg, n) for n in "QKV")
    n_q, n_k = _grid(cfg, orc)
    ones = np.ones((cfg.batch, cfg.heads, n_q, n_k), dtype=np.uint8)
    for final in (False, True):
        o1, l1 = osparse.block_sparse_attend(orc, Q, Kc, Vc, final, ones)
        o2, l2 = orc.attend(Q, Kc, Vc, final)
        np.testing.assert_allclose(o1, o2, atol=1e-12)
        np.testing.assert_allclose(l1, l2, atol=1e-12)


def test_random_masks_match_per_row_gather():
    """Each row: gather exactly its visible keys and run a plain softmax."""
    cfg = _cfg()
    orc = _stream(cfg, 4)
    Q, Kc, Vc = (_t(cfg, n) for n in "QKV")
    n_q, n_k = _grid(cfg, orc)
    mask = (RNG.random((cfg.batch, cfg.heads, n_q, n_k)) < 0.3).astype(np.uint8)
    mask[0, 1, 1, :] = 0  # one query tile of head 1 sees nothing
    o, l = osparse.block_sparse_attend(orc, Q, Kc, Vc, True, mask)

    ids, rank = orc.attended(True)
    c = orc.current_chunk()
    L, F = cfg.chunk_len, cfg.frames
    f, y, x = token_positions(L, cfg.tok_h, cfg.tok_w)
    for h in range(cfg.heads):
        keys, vals, tile_of = [], [], []
        for gi, j in enumerate(ids):
            Kj, Vj = (Kc, Vc) if j == c else orc.store[CLEAN][j]
            keys.append(rotate(Kj[0, :, h], rank[j] * F + f, y, x))
            vals.append(Vj[0, :, h])
            tile_of.append(gi * math.ceil(L / 128) + np.arange(L) // 128)
        keys, vals, tile_of = np.concatenate(keys), np.concatenate(vals), np.concatenate(tile_of)
        for r in range(0, L, 7):
            q = rotate(Q[0, r:r + 1, h], np.array([rank[c] * F + f[r]]), y[r:r + 1], x[r:r + 1])[0]
            vis = np.flatnonzero(mask[0, h, r // 128][tile_of])
            if vis.size == 0:
                assert np.all(o[0, r, h] == 0) and l[0, h, r] == -np.inf
                continue
            s = keys[vis] @ q / math.sqrt(cfg.head_dim)
            p = np.exp(s - s.max())
            np.testing.assert_allclose(o[0, r, h], p @ vals[vis] / p.sum(), atol=1e-12)
            np.testing.assert_allclose(l[0, h, r], s.max() + np.log(p.sum()), atol=1e-12)


def test_one_chunk_mask_is_attention_over_that_chunk_only():
    cfg = _cfg()
    orc = _stream(cfg, 2)  # attends chunks 0, 1 and the current chunk 2
    Q, Kc, Vc = (_t(cfg, n) for n in "QKV")
    n_q, n_k = _grid(cfg, orc)
    per_chunk = math.ceil(cfg.chunk_len / 128)
    mask = np.zeros((cfg.batch, cfg.heads, n_q, n_k), dtype=np.uint8)
    mask[..., per_chunk:2 * per_chunk] = 1  # chunk 1 only
    o, _ = osparse.block_sparse_attend(orc, Q, Kc, Vc, False, mask)
    ids, rank = orc.attended(False)
    L, F = cfg.chunk_len, cfg.frames
    f, y, x = token_positions(L, cfg.tok_h, cfg.tok_w)
    K1, V1 = orc.store[NOISY][1]
    for h in range(cfg.heads):
        k = rotate(K1[0, :, h], rank[1] * F + f, y, x)
        q = rotate(Q[0, :, h], rank[2] * F + f, y, x)
        ref = torch.nn.functional.scaled_dot_product_attention(
            *(torch.from_numpy(np.ascontiguousarray(a))[None, None] for a in (q, k, V1[0, :, h])),
            scale=1 / math.sqrt(cfg.head_dim))[0, 0].numpy()
        np.testing.assert_allclose(o[0, :, h], ref, atol=1e-12)


def test_planted_tile_shift_breaks_the_gather_pin(monkeypatch):
    cfg = _cfg()
    orc = _stream(cfg, 3)
    Q, Kc, Vc = (_t(cfg, n) for n in "QKV")
    n_q, n_k = _grid(cfg, orc)
    mask = (RNG.random((cfg.batch, cfg.heads, n_q, n_k)) < 0.5).astype(np.uint8)
    good, _ = osparse.block_sparse_attend(orc, Q, Kc, Vc, True, mask)
    real = osparse.key_tiles
    monkeypatch.setattr(osparse, "key_tiles",
                        lambda lengths, tile=128: [(g, min(s + 1, e - 1), e) for g, s, e in real(lengths)])
    bad, _ = osparse.block_sparse_attend(orc, Q, Kc, Vc, True, mask)
    assert np.abs(bad - good).max() > 1e-3

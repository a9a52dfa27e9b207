"""Pins of the frame-aligned editing attention oracle (CPU)."""

import math

import numpy as np
import pytest
import torch

import oracle.editing as editing
from oracle import rope as orope
from oracle.editing import frame_aligned_attend
from oracle.stream import CLEAN, NOISY, OracleConfig, StreamOracle
from sa_inputs import normal_bf16, seed_of

RNG = np.random.default_rng(11)


def _cfg(ref_frames=1, sink=1, window=3, frames=3, heads=2):
    return OracleConfig(1, heads, 64, frames, 4, 5, sink, window, ref_frames=ref_frames)


def _t(cfg, tag, frames):
    return normal_bf16(seed_of("editing-pin", tag),
                       (cfg.batch, frames * cfg.tok_h * cfg.tok_w, cfg.heads,
                        cfg.head_dim)).double().numpy()


def _stream(cfg, frame_seq, ref=True):
    orc = StreamOracle(cfg)
    if ref and cfg.ref_frames:
        orc.set_reference(_t(cfg, "Kref", cfg.ref_frames), _t(cfg, "Vref", cfg.ref_frames))
    for c, fr in enumerate(frame_seq):
        for tier in (NOISY, CLEAN):
            orc.append(tier, _t(cfg, ("K", c, tier), fr), _t(cfg, ("V", c, tier), fr))
    return orc


def _rope_complex(x, pt, ph, pw, theta=10000.0):
    """Rotation written with complex numbers, independent of oracle.rope.rotate."""
    out = np.empty_like(x)
    start = 0
    for d, pos in zip(orope.band_sizes(x.shape[-1]), (pt, ph, pw)):
        z = x[:, start:start + d:2] + 1j * x[:, start + 1:start + d:2]
        z = z * np.exp(1j * np.outer(pos, [theta ** (-(2.0 * i) / d) for i in range(d // 2)]))
        out[:, start:start + d:2], out[:, start + 1:start + d:2] = z.real, z.imag
        start += d
    return out


def _source_only(cfg, Q, Ks, Vs, base_c, b, h):
    """Each target row against the source tokens of its own frame only, by an
    explicit per-frame loop (complex RoPE, numpy softmax): (O [L, D], lse [L])."""
    hw = cfg.tok_h * cfg.tok_w
    L = Q.shape[1]
    l = np.arange(L)
    f, y, x = l // hw, (l // cfg.tok_w) % cfg.tok_h, l % cfg.tok_w
    q = _rope_complex(Q[b, :, h], base_c + f, y, x)
    k = _rope_complex(Ks[b, :, h], base_c + f, y, x)
    O, lse = np.zeros((L, cfg.head_dim)), np.zeros(L)
    for fr in range(L // hw):
        sl = slice(fr * hw, (fr + 1) * hw)
        s = q[sl] @ k[sl].T / math.sqrt(cfg.head_dim)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        O[sl] = e @ Vs[b, sl, h] / e.sum(axis=1, keepdims=True)
        lse[sl] = (m + np.log(e.sum(axis=1, keepdims=True)))[:, 0]
    return O, lse


@pytest.mark.parametrize("ref_frames,sink,window", [(1, 1, 3), (0, 2, 2), (2, 0, 1)])
def test_equals_lse_merge_of_generation_attention_and_aligned_source(ref_frames, sink, window):
    """Softmax over a union of key sets = the log-sum-exp merge of the softmax
    over each part: generation-path attention (pinned elsewhere) merged with a
    per-frame source attention written here independently."""
    cfg = _cfg(ref_frames, sink, window)
    orc = _stream(cfg, list(RNG.integers(1, cfg.frames + 1, size=5)))
    for final in (False, True):
        fq = int(RNG.integers(1, cfg.frames + 1))
        Q, Kc, Vc, Ks, Vs = (_t(cfg, (n, final), fq) for n in ("Q", "Kc", "Vc", "Ks", "Vs"))
        o, l = frame_aligned_attend(orc, Q, Kc, Vc, Ks, Vs, final)
        ob, lb = orc.attend(Q, Kc, Vc, final)
        _, base = orc.positions(final, fq)
        base_c = base[orc.current_chunk()]
        for h in range(cfg.heads):
            os_, ls = _source_only(cfg, Q, Ks, Vs, base_c, 0, h)
            lt = np.logaddexp(lb[0, h], ls)
            merged = (np.exp(lb[0, h] - lt)[:, None] * ob[0, :, h]
                      + np.exp(ls - lt)[:, None] * os_)
            np.testing.assert_allclose(o[0, :, h], merged, atol=1e-12)
            np.testing.assert_allclose(l[0, h], lt, atol=1e-12)


def test_single_frame_current_only_is_sdpa_over_target_and_source():
    """F = 1, no sink, W = 1, no reference: the chunk's target tokens and its one
    source frame, all at temporal position 0 — torch SDPA over the two lists."""
    cfg = _cfg(ref_frames=0, sink=0, window=1, frames=1)
    orc = _stream(cfg, [1, 1], ref=False)
    Q, Kc, Vc, Ks, Vs = (_t(cfg, ("sdpa", n), 1) for n in ("Q", "Kc", "Vc", "Ks", "Vs"))
    o, _ = frame_aligned_attend(orc, Q, Kc, Vc, Ks, Vs, True)
    hw = cfg.tok_h * cfg.tok_w
    y, x = np.arange(hw) // cfg.tok_w, np.arange(hw) % cfg.tok_w
    z = np.zeros(hw)
    for h in range(cfg.heads):
        k = np.concatenate([_rope_complex(Kc[0, :, h], z, y, x), _rope_complex(Ks[0, :, h], z, y, x)])
        v = np.concatenate([Vc[0, :, h], Vs[0, :, h]])
        q = _rope_complex(Q[0, :, h], z, y, x)
        ref = torch.nn.functional.scaled_dot_product_attention(
            *(torch.from_numpy(np.ascontiguousarray(a))[None, None] for a in (q, k, v)),
            scale=1 / math.sqrt(cfg.head_dim))[0, 0].numpy()
        np.testing.assert_allclose(o[0, :, h], ref, atol=1e-12)


def test_no_mixing_across_times():
    """Changing source frame f changes exactly the rows of target frame f."""
    cfg = _cfg()
    orc = _stream(cfg, [3, 3, 2])
    Q, Kc, Vc, Ks, Vs = (_t(cfg, ("mix", n), 3) for n in ("Q", "Kc", "Vc", "Ks", "Vs"))
    o0, _ = frame_aligned_attend(orc, Q, Kc, Vc, Ks, Vs, False)
    hw = cfg.tok_h * cfg.tok_w
    for f in range(3):
        Ks2, Vs2 = Ks.copy(), Vs.copy()
        Ks2[:, f * hw:(f + 1) * hw] += 1.5
        Vs2[:, f * hw:(f + 1) * hw] -= 2.0
        o1, _ = frame_aligned_attend(orc, Q, Kc, Vc, Ks2, Vs2, False)
        inside = np.zeros(o0.shape[1], dtype=bool)
        inside[f * hw:(f + 1) * hw] = True
        np.testing.assert_array_equal(o1[:, ~inside], o0[:, ~inside])
        assert (np.abs(o1[:, inside] - o0[:, inside]).max(axis=-1) > 0).all()
        assert np.abs(o1[:, inside] - o0[:, inside]).max() > 1e-2


def test_source_is_not_cached_and_history_is():
    """The next chunk's attention does not depend on an earlier source, while it
    does depend on the earlier chunks' cached target tokens."""
    cfg = _cfg()
    orc = _stream(cfg, [3, 3])
    Q, Kc, Vc = (_t(cfg, ("cache", n), 3) for n in ("Q", "Kc", "Vc"))
    a = [_t(cfg, ("srcA", n), 3) for n in ("Ks", "Vs")]
    frame_aligned_attend(orc, Q, Kc, Vc, *a, True)  # uses source A, appends nothing
    for tier in (NOISY, CLEAN):
        orc.append(tier, _t(cfg, ("K", 2, tier), 3), _t(cfg, ("V", 2, tier), 3))
    b = [_t(cfg, ("srcB", n), 3) for n in ("Ks", "Vs")]
    o_after, _ = frame_aligned_attend(orc, Q, Kc, Vc, *b, True)
    fresh = _stream(cfg, [3, 3])
    for tier in (NOISY, CLEAN):
        fresh.append(tier, _t(cfg, ("K", 2, tier), 3), _t(cfg, ("V", 2, tier), 3))
    o_fresh, _ = frame_aligned_attend(fresh, Q, Kc, Vc, *b, True)
    np.testing.assert_array_equal(o_after, o_fresh)
    other = _stream(cfg, [3, 2])  # a different cached target chunk 1
    for tier in (NOISY, CLEAN):
        other.append(tier, _t(cfg, ("K", 2, tier), 3), _t(cfg, ("V", 2, tier), 3))
    o_other, _ = frame_aligned_attend(other, Q, Kc, Vc, *b, True)
    assert np.abs(o_other - o_fresh).max() > 1e-3


@pytest.mark.parametrize("mistake", ["next_frame", "no_base_shift"])
def test_planted_mistakes_break_a_pin(mistake, monkeypatch):
    if mistake == "next_frame":
        monkeypatch.setattr(editing, "aligned_mask",
                            lambda fr, fk: (fr[:, None] + 1) % 3 == fk[None, :])
        with pytest.raises(AssertionError):
            test_no_mixing_across_times()
    else:
        monkeypatch.setattr(editing, "source_positions", lambda f, base_c: f)
        with pytest.raises(AssertionError):
            test_equals_lse_merge_of_generation_attention_and_aligned_source(1, 1, 3)

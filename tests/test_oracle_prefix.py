"""Pins of the oracle's reference-image prefix and variable chunk length (CPU)."""

import math

import numpy as np
import pytest
import torch

from oracle import rope as orope
from oracle.stream import CLEAN, NOISY, OracleConfig, StreamOracle, masked_full_attention
from sa_inputs import normal_bf16, seed_of

RNG = np.random.default_rng(7)


def _cfg(ref_frames=1, sink=1, window=3, frames=3):
    return OracleConfig(1, 2, 64, frames, 4, 5, sink, window, ref_frames=ref_frames)


def _t(cfg, tag, frames):
    return normal_bf16(seed_of("prefix-pin", tag),
                       (cfg.batch, frames * cfg.tok_h * cfg.tok_w, cfg.heads,
                        cfg.head_dim)).double().numpy()


def _stream(cfg, frame_seq, ref=True, keep_history=True):
    orc = StreamOracle(cfg, keep_history=keep_history)
    if ref and cfg.ref_frames:
        orc.set_reference(_t(cfg, "Kref", cfg.ref_frames), _t(cfg, "Vref", cfg.ref_frames))
    for c, fr in enumerate(frame_seq):
        for tier in (NOISY, CLEAN):
            orc.append(tier, _t(cfg, ("K", c, tier), fr), _t(cfg, ("V", c, tier), fr))
    return orc


def _rope_complex(x, pt, ph, pw, theta=10000.0):
    out = np.empty_like(x)
    start = 0
    for d, pos in zip(orope.band_sizes(x.shape[-1]), (pt, ph, pw)):
        z = x[:, start:start + d:2] + 1j * x[:, start + 1:start + d:2]
        z = z * np.exp(1j * np.outer(pos, [theta ** (-(2.0 * i) / d) for i in range(d // 2)]))
        out[:, start:start + d:2], out[:, start + 1:start + d:2] = z.real, z.imag
        start += d
    return out


@pytest.mark.parametrize("ref_frames,sink,window", [(1, 1, 3), (2, 0, 2), (0, 2, 2), (1, 2, 1)])
def test_gathered_equals_masked_full_stream_with_reference_and_variable_frames(ref_frames, sink,
                                                                               window):
    cfg = _cfg(ref_frames, sink, window)
    seq = list(RNG.integers(1, cfg.frames + 1, size=6))
    orc = _stream(cfg, [])
    for c, fr in enumerate(seq):
        for k in range(2):
            fq = int(RNG.integers(1, cfg.frames + 1))
            Q, Kc, Vc = (_t(cfg, (n, c, k), fq) for n in "QKV")
            o1, l1 = orc.attend(Q, Kc, Vc, k == 1)
            o2, l2 = masked_full_attention(cfg, orc.history, c, Q, Kc, Vc, k == 1,
                                           reference=orc.reference)
            np.testing.assert_allclose(o1, o2, atol=1e-12)
            np.testing.assert_allclose(l1, l2, atol=1e-12)
        for tier in (NOISY, CLEAN):
            orc.append(tier, _t(cfg, ("K", c, tier), fr), _t(cfg, ("V", c, tier), fr))


def test_hand_written_positions_complex_rope_and_sdpa():
    """Reference at t = 0, then chunks of 2, 1 and 3 frames, the current one of 2
    frames: every position written out by hand."""
    cfg = _cfg(ref_frames=1, sink=1, window=4)
    orc = _stream(cfg, [2, 1, 3])  # no eviction yet: all three cached
    Q, Kc, Vc = (_t(cfg, ("hand", n), 2) for n in "QKV")
    o, _ = orc.attend(Q, Kc, Vc, True)
    hw = cfg.tok_h * cfg.tok_w
    # temporal base: reference 0 (1 frame), chunk0 1 (2 frames), chunk1 3 (1), chunk2 4 (3), current 7
    bases = [1, 3, 4, 7]
    Kr, Vr = orc.reference
    for h in range(cfg.heads):
        keys, vals = [], []
        y, x = (np.arange(hw) // cfg.tok_w), (np.arange(hw) % cfg.tok_w)
        keys.append(_rope_complex(Kr[0, :, h], np.zeros(hw), y, x))
        vals.append(Vr[0, :, h])
        for j, base in zip(range(3), bases[:3]):
            K, V = orc.store[CLEAN][j]
            n = K.shape[1]
            keys.append(_rope_complex(K[0, :, h], base + np.arange(n) // hw,
                                      (np.arange(n) // cfg.tok_w) % cfg.tok_h, np.arange(n) % cfg.tok_w))
            vals.append(V[0, :, h])
        n = Kc.shape[1]
        pos = (bases[3] + np.arange(n) // hw, (np.arange(n) // cfg.tok_w) % cfg.tok_h,
               np.arange(n) % cfg.tok_w)
        keys.append(_rope_complex(Kc[0, :, h], *pos))
        vals.append(Vc[0, :, h])
        q = _rope_complex(Q[0, :, h], *pos)
        ref = torch.nn.functional.scaled_dot_product_attention(
            *(torch.from_numpy(np.ascontiguousarray(a))[None, None]
              for a in (q, np.concatenate(keys), np.concatenate(vals))),
            scale=1 / math.sqrt(cfg.head_dim))[0, 0].numpy()
        np.testing.assert_allclose(o[0, :, h], ref, atol=1e-12)


def test_positions_stay_bounded_for_long_variable_streams():
    cfg = _cfg(ref_frames=2, sink=2, window=4, frames=3)
    orc = StreamOracle(cfg)
    top_allowed = cfg.ref_frames + (cfg.sink + cfg.window) * cfg.frames - 1
    dummy = np.zeros((1, cfg.tok_h * cfg.tok_w, 1, 1))
    for c in range(200):
        fr = int(RNG.integers(1, cfg.frames + 1))
        ids, base = orc.positions(True, fr)
        frames = {j: (fr if j == c else orc.frames(orc.store[CLEAN][j][0])) for j in ids}
        assert max(base[j] + frames[j] - 1 for j in ids) <= top_allowed
        for tier in (NOISY, CLEAN):
            orc.append(tier, np.repeat(dummy, fr, axis=1), np.repeat(dummy, fr, axis=1))


def test_reference_is_seen_by_every_chunk_and_can_be_replaced():
    cfg = _cfg(ref_frames=1)
    orc = _stream(cfg, [3, 3, 3, 3])
    Q, Kc, Vc = (_t(cfg, ("rep", n), 3) for n in "QKV")
    o1, _ = orc.attend(Q, Kc, Vc, True)
    saved = orc.reference
    orc.set_reference(_t(cfg, "Kref2", 1), _t(cfg, "Vref2", 1))
    o2, _ = orc.attend(Q, Kc, Vc, True)
    assert np.abs(o2 - o1).max() > 1e-3
    orc.set_reference(*saved)
    np.testing.assert_array_equal(orc.attend(Q, Kc, Vc, True)[0], o1)


def test_ref_frames_without_a_reference_is_a_pure_shift():
    """With no reference set, ref_frames only shifts every temporal position."""
    a, b = _cfg(ref_frames=0), _cfg(ref_frames=4)
    oa, ob = _stream(a, [3, 2, 3, 1], ref=False), _stream(b, [3, 2, 3, 1], ref=False)
    Q, Kc, Vc = (_t(a, ("shift", n), 2) for n in "QKV")
    np.testing.assert_allclose(oa.attend(Q, Kc, Vc, False)[0], ob.attend(Q, Kc, Vc, False)[0],
                               atol=1e-10)

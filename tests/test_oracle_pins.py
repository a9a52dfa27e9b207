"""Pins of the oracle to things other than itself (CPU only).

Each test ties one oracle function to the pages (hand-worked golden fixtures),
to closed forms, to invariants, or to an independent library routine, so that a
dropped term, a wrong sign or index, or a transposed operand fails somewhere.
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import rope as orope
from oracle import stream as ostream
from oracle.cache import RingCacheModel
from oracle.stream import CLEAN, NOISY, OracleConfig, StreamOracle, masked_full_attention
from sa_inputs import WORKLOADS, normal_bf16, seed_of

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _f64(t):
    return t.to(torch.float64).numpy()


# --------------------------------------------------------------------------- cache


def _read_ring_golden(name):
    events = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#")[0].strip()
        if not line:
            continue
        kind, rest = line.split(None, 1)
        if kind == "append":
            cid, slot, ev = rest.split()
            events.append(("append", int(cid), None if slot == "-" else int(slot),
                           None if ev == "-" else int(ev)))
        else:
            ids, bases = rest.split("|")
            ids = [int(v) for v in ids.split()]
            events.append(("attend", ids[0], ids[1:], [int(v) for v in bases.split()]))
    return events


@pytest.mark.parametrize("fname,sink,window", [
    ("ring_s1_w3_f3.txt", 1, 3), ("ring_s2_w4_f3.txt", 2, 4),
    ("ring_s0_w2_f3.txt", 0, 2), ("ring_s2_w1_f3.txt", 2, 1)])
def test_cache_model_matches_hand_worked_golden(fname, sink, window):
    model = RingCacheModel(sink, window)
    F = 3
    for ev in _read_ring_golden(fname):
        if ev[0] == "append":
            assert model.count == ev[1]
            assert model.append() == (ev[2], ev[3]), ev
        else:
            assert model.count == ev[1]
            ids = model.attended()
            assert ids == ev[2], ev
            ranks = model.ranks()
            assert [ranks[j] * F for j in ids] == ev[3]


@pytest.mark.parametrize("sink,window", [(0, 1), (0, 2), (1, 1), (1, 2), (1, 3), (2, 4),
                                         (3, 2), (0, 5), (4, 7)])
def test_cache_model_against_closed_form_ring(sink, window):
    """Search-based slot model == modular ring formula, over 200 chunks."""
    ring = window - 1
    model = RingCacheModel(sink, window)
    for cid in range(200):
        held = set(range(min(cid, sink))) | set(range(max(sink, cid - ring), cid))
        assert set(model.held()) == held
        assert model.attended() == sorted(held) + [cid]
        # closed form of the ring slot and of the evicted chunk
        if cid < sink:
            want = (cid, None)
        elif ring == 0:
            want = (None, cid)
        else:
            want = (sink + (cid - sink) % ring, cid - ring if cid - ring >= sink else None)
        assert model.append() == want
        # never more than sink + window - 1 chunks cached
        assert len(model.held()) <= sink + ring


def test_relocated_positions_stay_bounded_for_long_streams():
    """200-chunk stress stream: every temporal position < (S + W) * F, and
    window-to-current distances equal the absolute chunk distances."""
    w = WORKLOADS["long_stream_stress"]
    model = RingCacheModel(w.sink, w.window)
    for c in range(w.stream):
        ids, ranks = model.attended(), model.ranks()
        top = max(ranks[j] * w.frames + w.frames - 1 for j in ids)
        assert top <= (w.sink + w.window) * w.frames - 1
        for j in ids:
            if j >= w.sink:  # window chunks and the current chunk
                assert ranks[c] - ranks[j] == c - j
        model.append()


# --------------------------------------------------------------------------- rope


def test_band_sizes_reading():
    assert orope.band_sizes(128) == (44, 42, 42)
    assert orope.band_sizes(64) == (24, 20, 20)
    assert orope.band_sizes(6) == (2, 2, 2)


def _read_rope_golden():
    cases = []
    env = {"cos": math.cos, "sin": math.sin}
    for line in open(os.path.join(GOLDEN, "rope_small.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        head, vin, vout = line.split("|")
        D, pt, ph, pw = (int(v) for v in head.split())
        x = [float(v) for v in vin.split()]
        y = [float(eval(tok, {"__builtins__": {}}, env)) for tok in vout.split()]
        cases.append((D, pt, ph, pw, x, y))
    return cases


@pytest.mark.parametrize("case", _read_rope_golden())
def test_rope_hand_worked_values(case):
    D, pt, ph, pw, x, y = case
    out = orope.rotate(np.array([x]), np.array([pt]), np.array([ph]), np.array([pw]))
    np.testing.assert_allclose(out[0], y, atol=1e-15)


def test_rope_zero_position_is_identity_and_norm_is_kept():
    x = RNG.standard_normal((50, 128))
    zero = np.zeros(50, dtype=int)
    np.testing.assert_array_equal(orope.rotate(x, zero, zero, zero), x)
    pos = RNG.integers(0, 200, size=(3, 50))
    y = orope.rotate(x, *pos)
    # every pair keeps its length
    np.testing.assert_allclose(np.hypot(y[:, 0::2], y[:, 1::2]),
                               np.hypot(x[:, 0::2], x[:, 1::2]), rtol=1e-13)


def _rope_complex(x, pt, ph, pw, theta=10000.0):
    """Independent formulation: each pair as a complex number times e^{i a}."""
    D = x.shape[-1]
    out = np.empty_like(x)
    start = 0
    for d, pos in zip(orope.band_sizes(D), (pt, ph, pw)):
        z = x[:, start:start + d:2] + 1j * x[:, start + 1:start + d:2]
        freq = np.array([theta ** (-(2.0 * i) / d) for i in range(d // 2)])
        z = z * np.exp(1j * np.outer(pos, freq))
        out[:, start:start + d:2], out[:, start + 1:start + d:2] = z.real, z.imag
        start += d
    return out


@pytest.mark.parametrize("D", [64, 128])
def test_rope_matches_complex_formulation(D):
    x = RNG.standard_normal((40, D))
    pos = RNG.integers(0, 300, size=(3, 40))
    np.testing.assert_allclose(orope.rotate(x, *pos), _rope_complex(x, *pos), atol=1e-12)


@pytest.mark.parametrize("axis", [0, 1, 2])
def test_rope_dot_depends_only_on_position_difference(axis):
    q, k = RNG.standard_normal((2, 30, 128))
    pq = RNG.integers(0, 50, size=(3, 30))
    pk = RNG.integers(0, 50, size=(3, 30))
    shift = np.zeros((3, 1), dtype=int)
    shift[axis] = 37
    a = np.sum(orope.rotate(q, *pq) * orope.rotate(k, *pk), axis=1)
    b = np.sum(orope.rotate(q, *(pq + shift)) * orope.rotate(k, *(pk + shift)), axis=1)
    np.testing.assert_allclose(a, b, atol=1e-10)


def test_token_positions_frame_row_column_order():
    f, y, x = orope.token_positions(3 * 2 * 4, 2, 4)
    assert list(f[:9]) == [0] * 8 + [1]
    assert list(y[:9]) == [0, 0, 0, 0, 1, 1, 1, 1, 0]
    assert list(x[:9]) == [0, 1, 2, 3, 0, 1, 2, 3, 0]


# --------------------------------------------------------------------------- attention


def test_attention_special_cases():
    q = RNG.standard_normal((7, 64))
    k = RNG.standard_normal((33, 64))
    ones = np.ones((33, 64))
    o, _ = oracle.softmax_attention(q, k, ones, 0.125)
    np.testing.assert_allclose(o, 1.0, rtol=1e-14)
    v = RNG.standard_normal((33, 64))
    o, lse = oracle.softmax_attention(q, k[:1], v[:1], 0.125)
    np.testing.assert_allclose(o, np.broadcast_to(v[:1], o.shape), rtol=1e-14)
    np.testing.assert_allclose(lse, (q @ k[0]) * 0.125, rtol=1e-13)
    o, _ = oracle.softmax_attention(np.zeros((3, 64)), k, v, 0.125)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=0), o.shape), atol=1e-14)


def test_attention_matches_torch_sdpa_and_logsumexp():
    q = RNG.standard_normal((50, 128)) * 2
    k = RNG.standard_normal((300, 128)) * 2
    v = RNG.standard_normal((300, 128))
    scale = 1 / math.sqrt(128)
    o, lse = oracle.softmax_attention(q, k, v, scale)
    tq, tk, tv = (torch.from_numpy(a)[None, None] for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)[0, 0]
    np.testing.assert_allclose(o, ref.numpy(), atol=1e-12)
    ref_lse = torch.logsumexp(torch.from_numpy(q @ k.T * scale), dim=1).numpy()
    np.testing.assert_allclose(lse, ref_lse, atol=1e-12)


def test_attention_mask_hides_keys():
    q = RNG.standard_normal((5, 64))
    k = RNG.standard_normal((20, 64))
    v = RNG.standard_normal((20, 64))
    mask = np.zeros((5, 20), dtype=bool)
    mask[:, :12] = True
    k2, v2 = k.copy(), v.copy()
    k2[12:] *= 1e3
    v2[12:] = 1e6
    a, _ = oracle.softmax_attention(q, k, v, 0.1, mask)
    b, _ = oracle.softmax_attention(q, k2, v2, 0.1, mask)
    c, _ = oracle.softmax_attention(q, k[:12], v[:12], 0.1)
    np.testing.assert_allclose(a, b, rtol=1e-14)
    np.testing.assert_allclose(a, c, rtol=1e-13)


# --------------------------------------------------------------------------- stream


def _tiny_cfg(sink=1, window=2, heads=2, D=64, frames=3, th=4, tw=4, batch=1):
    return OracleConfig(batch, heads, D, frames, th, tw, sink, window)


def _rand(cfg, tag, scale=1.0):
    shape = (cfg.batch, cfg.chunk_len, cfg.heads, cfg.head_dim)
    return _f64(normal_bf16(seed_of("pin", tag), shape, scale=scale))


def _run_stream(cfg, n_chunks, steps=2, check=None):
    """Drive an oracle stream; call check(oracle, c, k, Q, Kc, Vc, final)."""
    orc = StreamOracle(cfg, keep_history=True)
    for c in range(n_chunks):
        for k in range(steps):
            Q, Kc, Vc = (_rand(cfg, (n, c, k)) for n in ("Q", "Kc", "Vc"))
            if check is not None:
                check(orc, c, k, Q, Kc, Vc, k == steps - 1)
        for tier in (NOISY, CLEAN):
            orc.append(tier, _rand(cfg, ("K", c, tier)), _rand(cfg, ("V", c, tier)))
    return orc


@pytest.mark.parametrize("sink,window", [(1, 2), (1, 3), (2, 2), (0, 2), (2, 1)])
def test_gathered_attention_equals_masked_full_stream(sink, window):
    """Sink + window gather == full attention under the block-causal mask
    restricted to sink and window chunks, on the materialised whole stream."""
    cfg = _tiny_cfg(sink, window)

    def check(orc, c, k, Q, Kc, Vc, final):
        o1, l1 = orc.attend(Q, Kc, Vc, final)
        o2, l2 = masked_full_attention(cfg, orc.history, c, Q, Kc, Vc, final)
        np.testing.assert_allclose(o1, o2, atol=1e-12)
        np.testing.assert_allclose(l1, l2, atol=1e-12)

    _run_stream(cfg, 6, check=check)


def _textbook_block_causal(cfg, history, c, Q, Kc, Vc, final):
    """Absolute positions, every earlier chunk visible, torch SDPA, complex RoPE."""
    tier = CLEAN if final else NOISY
    L, F = cfg.chunk_len, cfg.frames
    f, y, x = orope.token_positions(L, cfg.tok_h, cfg.tok_w)
    O = np.zeros((cfg.batch, L, cfg.heads, cfg.head_dim))
    for b in range(cfg.batch):
        for h in range(cfg.heads):
            ks, vs = [], []
            for j in range(c + 1):
                Kj, Vj = (Kc, Vc) if j == c else history[tier][j]
                ks.append(_rope_complex(Kj[b, :, h], j * F + f, y, x))
                vs.append(Vj[b, :, h])
            q = _rope_complex(Q[b, :, h], c * F + f, y, x)
            o = torch.nn.functional.scaled_dot_product_attention(
                *(torch.from_numpy(np.ascontiguousarray(a))[None, None]
                  for a in (q, np.concatenate(ks), np.concatenate(vs))),
                scale=1 / math.sqrt(cfg.head_dim))
            O[b, :, h] = o[0, 0].numpy()
    return O


def test_no_eviction_is_textbook_block_causal_attention():
    """Before any eviction, ranks are chunk ids: plain block-causal attention
    with absolute positions (torch SDPA + complex-number RoPE)."""
    cfg = _tiny_cfg(1, 3)  # holds chunks 0..2, first eviction when chunk 3 is appended

    def check(orc, c, k, Q, Kc, Vc, final):
        if c > cfg.sink + cfg.window - 1:
            return
        o1, _ = orc.attend(Q, Kc, Vc, final)
        o2 = _textbook_block_causal(cfg, orc.history, c, Q, Kc, Vc, final)
        np.testing.assert_allclose(o1, o2, atol=1e-12)

    _run_stream(cfg, 4, check=check)


def test_relocation_is_invariant_to_a_constant_temporal_shift():
    """Adding a constant to every temporal position changes no output."""
    cfg = _tiny_cfg(1, 2)
    orc = _run_stream(cfg, 4)
    Q, Kc, Vc = (_rand(cfg, ("shift", n)) for n in "QKV")
    base, _ = orc.attend(Q, Kc, Vc, True)
    real_rotate = ostream.rotate
    try:
        ostream.rotate = lambda x, pt, ph, pw, theta: real_rotate(x, pt + 1000, ph, pw, theta)
        shifted, _ = orc.attend(Q, Kc, Vc, True)
    finally:
        ostream.rotate = real_rotate
    np.testing.assert_allclose(base, shifted, atol=1e-9)


def test_twincache_tier_selection():
    """Final step reads only the clean tier, earlier steps only the noisy one."""
    cfg = _tiny_cfg(1, 3)
    orc = _run_stream(cfg, 5)
    Q, Kc, Vc = (_rand(cfg, ("tier", n)) for n in "QKV")
    final0, _ = orc.attend(Q, Kc, Vc, True)
    mid0, _ = orc.attend(Q, Kc, Vc, False)
    for cid in list(orc.store[NOISY]):
        K, V = orc.store[NOISY][cid]
        orc.store[NOISY][cid] = (K + 3.0, V - 2.0)
    final1, _ = orc.attend(Q, Kc, Vc, True)
    mid1, _ = orc.attend(Q, Kc, Vc, False)
    np.testing.assert_array_equal(final0, final1)
    assert np.abs(mid1 - mid0).max() > 0.1
    for cid in list(orc.store[CLEAN]):
        K, V = orc.store[CLEAN][cid]
        orc.store[CLEAN][cid] = (K * 0.5, V + 1.0)
    final2, _ = orc.attend(Q, Kc, Vc, True)
    mid2, _ = orc.attend(Q, Kc, Vc, False)
    np.testing.assert_array_equal(mid1, mid2)
    assert np.abs(final2 - final1).max() > 0.1


def test_causality_future_chunks_are_never_read():
    """A chunk's output does not change when later chunks (filled with 1e4)
    exist in the history, and the attended list never holds a later id."""
    cfg = _tiny_cfg(1, 2)
    orc = _run_stream(cfg, 3)
    c = orc.current_chunk()
    Q, Kc, Vc = (_rand(cfg, ("causal", n)) for n in "QKV")
    o1, _ = masked_full_attention(cfg, orc.history, c, Q, Kc, Vc, True)
    big = np.full_like(Q, 1e4)
    for tier in (NOISY, CLEAN):
        for j in range(c + 1, c + 4):
            orc.history[tier][j] = (big, big)
    o2, _ = masked_full_attention(cfg, orc.history, c, Q, Kc, Vc, True)
    np.testing.assert_array_equal(o1, o2)
    ids, _ = orc.attended(True)
    assert max(ids) == c and all(j <= c for j in ids)


def test_attend_requires_tiers_in_step():
    cfg = _tiny_cfg()
    orc = StreamOracle(cfg)
    orc.append(NOISY, _rand(cfg, "k"), _rand(cfg, "v"))
    with pytest.raises(RuntimeError):
        orc.current_chunk()


def test_row_subset_matches_full_output():
    cfg = _tiny_cfg(1, 2, heads=3, batch=2)
    orc = _run_stream(cfg, 3)
    Q, Kc, Vc = (_rand(cfg, ("rows", n)) for n in "QKV")
    full, lse = orc.attend(Q, Kc, Vc, False)
    rows = np.array([0, 5, 17, cfg.chunk_len - 1])
    part, lpart = orc.attend(Q, Kc, Vc, False, rows=rows, heads=[2, 0], batches=[1])
    # same arithmetic on a row subset; only the matmul blocking may differ
    np.testing.assert_allclose(part[0, :, 0], full[1, rows, 2], atol=1e-14)
    np.testing.assert_allclose(part[0, :, 1], full[1, rows, 0], atol=1e-14)
    np.testing.assert_allclose(lpart[0, 1], lse[1, 0, rows], atol=1e-13)


# --------------------------------------------------------------------------- planted mistakes


def test_pins_catch_planted_mistakes(monkeypatch):
    """Mistakes planted in the oracle (on the CPU) must break a pin."""
    x = RNG.standard_normal((10, 64))
    pos = RNG.integers(0, 40, size=(3, 10))
    good = _rope_complex(x, *pos)

    # 1. wrong rotation sign
    real = orope.band_angles
    monkeypatch.setattr(orope, "band_angles", lambda p, d, t: -real(p, d, t))
    assert not np.allclose(orope.rotate(x, *pos), good, atol=1e-6)
    monkeypatch.setattr(orope, "band_angles", real)
    np.testing.assert_allclose(orope.rotate(x, *pos), good, atol=1e-12)

    # 2. band sizes swapped (temporal band too small)
    monkeypatch.setattr(orope, "band_sizes", lambda D: (2 * (D // 6), D - 4 * (D // 6), 2 * (D // 6)))
    assert not np.allclose(orope.rotate(x, *pos), good, atol=1e-6)
    monkeypatch.undo()

    # 3. final step reading the noisy tier: the TwinCache pin must notice
    cfg = _tiny_cfg(1, 3)
    orc = _run_stream(cfg, 4)
    Q, Kc, Vc = (_rand(cfg, ("plant", n)) for n in "QKV")
    good_final, _ = orc.attend(Q, Kc, Vc, True)
    monkeypatch.setattr(ostream, "CLEAN", NOISY)
    bad_final, _ = orc.attend(Q, Kc, Vc, True)
    monkeypatch.undo()
    assert np.abs(bad_final - good_final).max() > 0.05

    # 4. an off-by-one rank (current chunk one frame-block further away) breaks
    #    the masked full-stream pin
    c = orc.current_chunk()
    ref, _ = masked_full_attention(cfg, orc.history, c, Q, Kc, Vc, True)
    real_positions = StreamOracle.positions

    def shifted_positions(self, final, current_frames):
        ids, base = real_positions(self, final, current_frames)
        base = dict(base)
        base[ids[-1]] += cfg.frames  # current chunk one chunk further away
        return ids, base
    monkeypatch.setattr(StreamOracle, "positions", shifted_positions)
    bad, _ = orc.attend(Q, Kc, Vc, True)
    monkeypatch.undo()
    assert np.abs(bad - ref).max() > 1e-3

    # 5. a window that forgets the most recent chunk breaks the ring pin
    real_attended_model = RingCacheModel.attended
    monkeypatch.setattr(RingCacheModel, "attended",
                        lambda self: [j for j in real_attended_model(self) if j != self.count - 1])
    m = RingCacheModel(1, 3)
    for _ in range(5):
        m.append()
    assert m.attended() != [0, 3, 4, 5]

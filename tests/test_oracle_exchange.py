"""Pins of the quantised Ulysses exchange oracle (CPU)."""

import numpy as np
import pytest
import torch

from oracle import exchange as ex
from sa_inputs import normal_bf16, seed_of

RNG = np.random.default_rng(5)


def test_e4m3_codes_decode_to_the_format_values():
    """Hand-worked codes of the e4m3 format (bias 7, 3 mantissa bits)."""
    table = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
             0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0, 0x80: -0.0, 0xB8: -1.0,
             0xFE: -448.0}
    for code, value in table.items():
        assert ex.e4m3_decode(np.array([code]))[0] == value, hex(code)
    assert np.isnan(ex.e4m3_decode(np.array([0x7F, 0xFF]))).all()


def test_e4m3_encode_matches_torch_float8_cast():
    """Rounding (nearest, ties to even, saturation, sign of zero) agrees with
    torch's float8_e4m3fn conversion on a dense sweep, the grid, its midpoints
    and values past the largest finite one."""
    vals, _ = ex._grid()
    mids = (vals[1:] + vals[:-1]) / 2
    sweep = np.concatenate([RNG.normal(size=20000) * 10.0 ** RNG.uniform(-4, 3, 20000),
                            vals, -vals, mids, -mids, [0.0, -0.0, 447.9, 464.0, 479.9, 1e4, -1e4]])
    sweep = sweep.astype(np.float32)
    mine = ex.e4m3_encode(sweep)
    t = torch.from_numpy(np.clip(sweep, -448, 448)).to(torch.float8_e4m3fn)
    theirs = t.view(torch.uint8).numpy()
    bad = mine != theirs
    assert not bad.any(), (sweep[bad][:5], mine[bad][:5], theirs[bad][:5])


def test_quantize_bounds_and_scale():
    x = normal_bf16(seed_of("exchange-pin", "x"), (2, 7, 3, 128), outlier_frac=0.02).float().numpy()
    x[0, 0, 0] = 0.0  # an all-zero vector
    codes, scale = ex.quantize(x)
    assert scale[0, 0, 0] == 0 and (codes[0, 0, 0] == 0).all()
    y = ex.e4m3_decode(codes) * scale[..., None]
    amax = np.abs(x).max(axis=-1)
    # the largest element of each vector lands on +-448 * scale (within fp32 rounding)
    i = np.abs(x).argmax(axis=-1)
    top = np.take_along_axis(np.abs(y), i[..., None], axis=-1)[..., 0]
    np.testing.assert_allclose(top, amax, rtol=1e-6)
    # round-trip error: half a unit in the last place of a 3-bit mantissa
    err = np.abs(y - x)
    normal = np.abs(x) >= 2.0 ** -6 * scale[..., None]
    assert (err[normal] <= 2.0 ** -4 * np.abs(x[normal]) * (1 + 1e-6)).all()
    assert (err[~normal] <= 2.0 ** -10 * np.broadcast_to(scale[..., None], x.shape)[~normal]
            * (1 + 1e-6)).all()


def test_bf16_round_matches_torch():
    v = (RNG.normal(size=50000) * 10.0 ** RNG.uniform(-6, 6, 50000)).astype(np.float32)
    mine = ex.bf16_round(v)
    theirs = torch.from_numpy(v).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(mine, theirs)


@pytest.mark.parametrize("G", [1, 2, 4])
def test_unquantised_exchange_is_the_ulysses_permutation(G):
    """Without quantisation, rank r holds heads r*H/G.. of every token after the
    first exchange, and the second exchange gives back the token shards."""
    B, L, H, D = 2, 24, 8, 16
    x = RNG.normal(size=(B, L, H, D))
    shards = [x[:, s * L // G:(s + 1) * L // G] for s in range(G)]
    heads = ex.tokens_to_heads(shards, quantised=False)
    for r in range(G):
        np.testing.assert_array_equal(heads[r], x[:, :, r * H // G:(r + 1) * H // G])
    back = ex.heads_to_tokens(heads, quantised=False)
    for s in range(G):
        np.testing.assert_array_equal(back[s], shards[s])


def test_quantised_exchange_rounds_each_vector_once():
    B, L, H, D = 1, 16, 4, 64
    x = normal_bf16(seed_of("exchange-pin", "ulysses"), (B, L, H, D)).double().numpy()
    shards = [x[:, :8], x[:, 8:]]
    heads = ex.tokens_to_heads(shards)
    full = ex.dequantize(*ex.quantize(x))  # per-vector quantisation does not depend on G
    np.testing.assert_array_equal(heads[0], full[:, :, :2])
    np.testing.assert_array_equal(heads[1], full[:, :, 2:])
    rel = np.abs(full - x).max() / np.abs(x).max()
    assert 0 < rel <= 2.0 ** -4 + 2.0 ** -8


def test_planted_rounding_mistake_breaks_a_pin(monkeypatch):
    """Ties rounded away from zero instead of to even: the torch comparison fails."""
    vals, codes = ex._grid()

    def bad_encode(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.minimum(np.abs(x), ex.E4M3_MAX)
        hi = np.minimum(np.searchsorted(vals, a, side="left"), len(vals) - 1)
        lo = np.maximum(hi - 1, 0)
        pick_hi = (vals[hi] - a) <= (a - vals[lo])
        code = codes[np.where(a == vals[hi], hi, np.where(pick_hi, hi, lo))]
        return np.where(np.signbit(x), code | 0x80, code).astype(np.uint8)

    monkeypatch.setattr(ex, "e4m3_encode", bad_encode)
    with pytest.raises(AssertionError):
        test_e4m3_encode_matches_torch_float8_cast()

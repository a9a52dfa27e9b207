"""CUDA path vs the float64 oracle, element by element, through the C ABI."""

import numpy as np
import pytest
import torch

import block_causal_streaming_sa_b200 as sa
from harness import TOL, Pair, check_output, sample_rows
from oracle.stream import CLEAN, NOISY
from sa_inputs import WORKLOADS, Workload

pytestmark = pytest.mark.gpu


def _assert_close(o_gpu, o_ref, l_gpu, l_ref, what, allow_output_rounding=False):
    err, _ = check_output(o_gpu, o_ref, what, allow_output_rounding)
    lerr = np.abs(l_gpu - l_ref).max()
    assert lerr <= 1e-2, f"{what}: max |lse - oracle| = {lerr:.3e}"
    return err


@pytest.mark.parametrize("simt", [False, True], ids=["tcgen05", "simt"])
def test_tiny_stream_every_chunk_and_step(simt):
    """Every output of every step of the 6-chunk tiny stream, plus the cache
    layout after every append, bit-exact."""
    w = WORKLOADS["tiny"]
    pair = Pair(w)
    for c in range(w.stream):
        for k in range(w.steps):
            _assert_close(*pair.attend(k, k == w.steps - 1, simt=simt), f"chunk {c} step {k}")
        pair.append()
        pair.check_layout()
    assert pair.gpu.status() == sa.SA_OK


EDGE = [
    # name, B, H, D, F, th, tw, S, W  -- ragged tails, single partial tiles, degenerate windows
    ("one_partial_tile", 2, 3, 64, 2, 5, 7, 1, 2),
    ("ragged_d128", 1, 2, 128, 3, 9, 11, 2, 3),
    ("no_sink", 1, 2, 128, 2, 10, 10, 0, 2),
    ("sinks_only", 1, 2, 64, 2, 8, 8, 2, 1),
    ("current_only", 2, 1, 128, 1, 13, 13, 0, 1),
    ("single_frame_wide_window", 1, 3, 64, 1, 16, 20, 1, 5),
    ("exact_tiles", 1, 1, 128, 4, 8, 8, 1, 3),
]


@pytest.mark.parametrize("case", EDGE, ids=[e[0] for e in EDGE])
def test_edge_shapes_and_windows(case):
    name, B, H, D, F, th, tw, S, W = case
    w = Workload("edge_" + name, B, H, D, F, th, tw, sink=S, window=W, steps=2, stream=S + W + 2)
    pair = Pair(w)
    for c in range(w.stream):
        for k in range(w.steps):
            _assert_close(*pair.attend(k, k == 1), f"{name} chunk {c} step {k}")
        pair.append()
        pair.check_layout()
    assert pair.gpu.status() == sa.SA_OK


def test_tensor_core_and_simt_kernels_agree():
    w = Workload("agree", 2, 4, 128, 3, 12, 20, sink=1, window=3, steps=2, stream=5)
    pair = Pair(w)
    for _ in range(w.stream):
        pair.append()
    Q, Kc, Vc = (t.cuda() for t in pair.tensors(("Q", "Kc", "Vc")))
    a = pair.gpu.attend(Q, Kc, Vc, False)
    b = pair.gpu.attend(Q, Kc, Vc, False, simt=True)
    torch.cuda.synchronize()
    assert (a.double() - b.double()).abs().max().item() <= TOL


def test_twincache_tier_selection_on_gpu():
    """Changing the noisy tier leaves the final step bit-identical and vice versa."""
    w = Workload("tiers", 1, 2, 128, 3, 8, 8, sink=1, window=3, steps=2, stream=5)
    outs = {}
    for variant in ("base", "noisy_changed", "clean_changed"):
        h = sa.StreamingAttention(w.config_dict())
        for c in range(w.stream):
            Kn, Vn, Kcl, Vcl = (w.tensor(n, c).cuda() for n in ("Kn", "Vn", "Kcl", "Vcl"))
            if variant == "noisy_changed":
                Kn, Vn = Kn * 2 + 1, -Vn
            if variant == "clean_changed":
                Kcl, Vcl = Kcl * 0.5 - 1, Vcl + 3
            h.append(NOISY, Kn.contiguous(), Vn.contiguous())
            h.append(CLEAN, Kcl.contiguous(), Vcl.contiguous())
        Q, Kc, Vc = (w.tensor(n, w.stream).cuda() for n in ("Q", "Kc", "Vc"))
        outs[variant] = (h.attend(Q, Kc, Vc, False).cpu(), h.attend(Q, Kc, Vc, True).cpu())
    assert torch.equal(outs["base"][1], outs["noisy_changed"][1])
    assert not torch.equal(outs["base"][0], outs["noisy_changed"][0])
    assert torch.equal(outs["base"][0], outs["clean_changed"][0])
    assert not torch.equal(outs["base"][1], outs["clean_changed"][1])


def test_evicted_and_future_chunks_are_never_read():
    """Two streams that differ only in an evicted chunk give bit-identical
    outputs; appended chunks never exceed the current id in the plan."""
    w = Workload("causal", 1, 2, 128, 3, 8, 8, sink=1, window=2, steps=1, stream=4)
    outs = []
    for poison in (False, True):
        h = sa.StreamingAttention(w.config_dict())
        for c in range(w.stream):
            K, V = (w.tensor(n, c).cuda() for n in ("Kcl", "Vcl"))
            if poison and c == 1:  # chunk 1 is evicted when chunk 2 is appended
                K, V = torch.full_like(K, 1e4), torch.full_like(V, 1e4)
            h.append(NOISY, K, V)
            h.append(CLEAN, K, V)
        Q, Kc, Vc = (w.tensor(n, w.stream).cuda() for n in ("Q", "Kc", "Vc"))
        outs.append(h.attend(Q, Kc, Vc, True).cpu())
        ids, _, _ = sa.sa_plan(h.cfg, w.stream)
        assert 1 not in ids and max(ids) == w.stream
    assert torch.equal(outs[0], outs[1])


def test_state_errors():
    w = WORKLOADS["tiny"]
    h = sa.StreamingAttention(w.config_dict())
    K, V = (w.tensor(n, 0).cuda() for n in ("Kn", "Vn"))
    h.append(NOISY, K, V)
    with pytest.raises(sa.SaError) as e:
        h.append(NOISY, K, V)  # noisy already one ahead
    assert e.value.status == sa.SA_ERR_STATE
    Q = w.tensor("Q", 1).cuda()
    with pytest.raises(sa.SaError) as e:
        h.attend(Q, K, V, False)  # tiers out of step
    assert e.value.status == sa.SA_ERR_STATE
    h.append(CLEAN, K, V)
    h.attend(Q, K, V, False)
    with pytest.raises(sa.SaError) as e:
        sa.sa_attend(h.handle, Q.data_ptr() + 2, K.data_ptr(), V.data_ptr(), 0,
                     torch.empty_like(Q).data_ptr())
    assert e.value.status == sa.SA_ERR_INVALID_ARG
    h.reset()
    assert h.chunk_count(NOISY) == 0 and h.status() == sa.SA_OK


FULL = [
    # workload, heads the oracle checks, batches, rows per (b, h)
    ("s1_540p", None, None, 256),
    ("refiner_720p", None, None, 256),
    ("backbone_540p_large", [0, 13, 27, 39], None, 256),
    ("long_stream_stress", [0, 11, 23], [0, 3], 256),
]


@pytest.mark.parametrize("case", FULL, ids=[c[0] for c in FULL])
def test_full_size_sampled_rows(case):
    """The full-size workloads in the bench's launch configuration: the first
    chunk (no cache) and, after eviction has begun, one noisy and one clean
    step, on >= 256 sampled query rows per checked (b, h)."""
    name, heads, batches, nrows = case
    w = WORKLOADS[name]
    big = w.outlier_frac > 0  # +-8 outliers in V: |O| reaches 4..8
    pair = Pair(w, batches=batches, heads=heads)
    rows = sample_rows(w.chunk_len, nrows, seed=7)
    _assert_close(*pair.attend(0, w.steps == 1, rows=rows), f"{name} chunk 0", big)
    first_evicting = w.sink + w.window  # this chunk's plan no longer holds chunk S
    while pair.chunk < first_evicting:
        pair.append()
    pair.check_layout()
    if w.steps > 1:
        _assert_close(*pair.attend(0, False, rows=rows), f"{name} noisy step", big)
    _assert_close(*pair.attend(w.steps - 1, True, rows=rows), f"{name} clean step", big)
    assert pair.gpu.status() == sa.SA_OK

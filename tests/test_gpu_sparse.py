"""Block-sparse attention on the GPU vs the block-sparse float64 oracle."""

import numpy as np
import pytest
import torch

import block_causal_streaming_sa_b200 as sa
from harness import Pair, check_output, sample_rows
from sa_inputs import WORKLOADS, Workload

pytestmark = pytest.mark.gpu


def _grid(pair):
    return sa.sa_block_grid(pair.gpu.cfg, pair.chunk)


def _check(o_gpu, o_ref, l_gpu, l_ref, what):
    check_output(o_gpu, o_ref, what)
    seen = np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(l_gpu), seen), f"{what}: rows without keys differ"
    assert np.all(o_gpu[~np.broadcast_to(seen.transpose(0, 2, 1)[..., None], o_gpu.shape)] == 0)
    if seen.any():
        assert np.abs(l_gpu[seen] - l_ref[seen]).max() <= 1e-2, what


@pytest.mark.parametrize("density", [0.05, 0.3, 0.7])
def test_random_masks_every_chunk(density):
    w = Workload("sparse_rand", 2, 3, 128, 3, 10, 14, sink=1, window=3, steps=2, stream=5)
    pair = Pair(w)
    rng = np.random.default_rng(int(density * 100))
    for c in range(w.stream):
        nq, nk = _grid(pair)
        mask = (rng.random((w.batch, w.heads, nq, nk)) < density).astype(np.uint8)
        mask[0, 0, 0, :] = 0            # a query tile that sees nothing
        mask[1, 2, :, :] = 0            # a whole (b, h) with nothing: empty work tiles
        for k in range(w.steps):
            _check(*pair.attend_sparse(k, k == 1, mask), f"chunk {c} step {k} density {density}")
        pair.append()
    assert pair.gpu.status() == sa.SA_OK


def test_structured_masks_skip_chunks_and_partner_tiles():
    """Whole attended chunks skipped (the query rotation must jump chunks), and
    blocks flagged for only one query tile of a 256-row pair."""
    w = Workload("sparse_struct", 1, 2, 64, 2, 12, 16, sink=2, window=3, steps=1, stream=6)
    pair = Pair(w)
    for _ in range(w.stream):
        pair.append()
    nq, nk = _grid(pair)
    per_chunk = -(-w.chunk_len // 128)
    n_chunks = nk // per_chunk
    masks = []
    m = np.zeros((w.batch, w.heads, nq, nk), dtype=np.uint8)
    m[..., 0:per_chunk] = 1                       # first sink only
    m[..., (n_chunks - 1) * per_chunk:] = 1       # and the chunk itself
    masks.append(m)
    m = np.zeros_like(masks[0])
    m[:, :, 0::2, :] = 1                          # even query tiles only: partners unflagged
    masks.append(m)
    m = np.zeros_like(masks[0])
    m[:, :, :, 2 * per_chunk:3 * per_chunk] = 1   # one middle chunk only
    masks.append(m)
    m = np.zeros_like(masks[0])
    m[:, :, 1::2, :] = 1                          # odd query tiles only: the first
    masks.append(m)                               # tile of every pair sees nothing
    rng = np.random.default_rng(3)
    m = (rng.random(masks[0].shape) < 0.4).astype(np.uint8)
    m[:, :, 1::2, :] = m[:, :, 0:nq - 1:2, :]     # both tiles of a pair alike: every
    masks.append(m)                               # key tile is shared by the pair
    for i, m in enumerate(masks):
        _check(*pair.attend_sparse(0, True, m), f"structured mask {i}")


@pytest.mark.parametrize("density", [0.02, 0.5])
def test_rows_of_more_than_64_key_tiles(density):
    """72 key tiles a query tile: the mask's bit rows span two words."""
    w = Workload("sparse_wide", 1, 2, 128, 3, 16, 32, sink=1, window=5, steps=1, stream=6)
    pair = Pair(w)
    for _ in range(5):
        pair.append()
    nq, nk = _grid(pair)
    assert nk > 64
    rng = np.random.default_rng(int(density * 1000))
    mask = (rng.random((w.batch, w.heads, nq, nk)) < density).astype(np.uint8)
    mask[0, 0, 1, 60:70] = 1                      # a run across the word boundary
    mask[0, 1, 2, :] = 0
    mask[0, 1, 2, 64] = 1                         # a single block just past it
    _check(*pair.attend_sparse(0, True, mask), f"wide rows density {density}")
    assert pair.gpu.status() == sa.SA_OK


def test_all_ones_mask_is_the_dense_kernel_bit_for_bit():
    w = WORKLOADS["tiny"]
    pair = Pair(w)
    for _ in range(3):
        pair.append()
    Q, Kc, Vc = (t.cuda() for t in pair.tensors(("Q", "Kc", "Vc")))
    nq, nk = _grid(pair)
    ones = torch.ones((w.batch, w.heads, nq, nk), dtype=torch.uint8, device="cuda")
    a = pair.gpu.attend(Q, Kc, Vc, True)
    b = pair.gpu.attend_sparse(Q, Kc, Vc, True, ones)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_full_size_720p_at_90_percent_sparsity():
    w = WORKLOADS["refiner_720p"]
    pair = Pair(w, heads=[0, 5, 11])
    while pair.chunk < w.sink + w.window:
        pair.append()
    nq, nk = _grid(pair)
    rng = np.random.default_rng(90)
    mask = (rng.random((w.batch, w.heads, nq, nk)) < 0.1).astype(np.uint8)
    rows = sample_rows(w.chunk_len, 256, seed=9)
    _check(*pair.attend_sparse(0, True, mask, rows=rows), "720p 90% sparse")
    assert pair.gpu.status() == sa.SA_OK

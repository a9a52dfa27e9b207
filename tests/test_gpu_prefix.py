"""Reference-image prefix and variable chunk length on the GPU vs the float64 oracle.

The library is driven through the C ABI (sa_set_reference, sa_append_chunk_frames,
sa_attend_frames, sa_stream_plan and the whole-chunk calls); the oracle is fed
the same seeded tensors.
"""

import numpy as np
import pytest
import torch

import block_causal_streaming_sa_b200 as sa
from harness import TOL, check_output, f64, sample_rows
from oracle.sparse import block_sparse_attend, key_tiles
from oracle.stream import CLEAN, NOISY, OracleConfig, StreamOracle
from sa_inputs import normal_bf16, seed_of

pytestmark = pytest.mark.gpu


class PrefixPair:
    """A library handle and an oracle stream with a reference image and chunks
    of any 1..F frames. ``heads`` restricts what the oracle computes."""

    def __init__(self, name, B, H, D, F, th, tw, S, W, ref_frames, heads=None):
        self.name, self.hw, self.F = name, th * tw, F
        self.B, self.H, self.D = B, H, D
        self.cfg = dict(batch=B, heads=H, head_dim=D, frames_per_chunk=F, tok_h=th, tok_w=tw,
                        sink_chunks=S, window_chunks=W, ref_frames=ref_frames)
        self.gpu = sa.StreamingAttention(self.cfg)
        self.hsel = list(range(H)) if heads is None else list(heads)
        self.ocfg = OracleConfig(B, len(self.hsel), D, F, th, tw, S, W, ref_frames=ref_frames)
        self.oracle = StreamOracle(self.ocfg)
        self.chunk = 0

    def t(self, tag, frames):
        return normal_bf16(seed_of(self.name, tag), (self.B, frames * self.hw, self.H, self.D))

    def _o(self, t):
        return f64(t)[:, :, self.hsel]

    def set_reference(self, tag):
        n = self.cfg["ref_frames"]
        K, V = self.t(("Kref", tag), n), self.t(("Vref", tag), n)
        self.gpu.set_reference(K.cuda(), V.cuda())
        self.oracle.set_reference(self._o(K), self._o(V))

    def clear_reference(self):
        self.gpu.set_reference(None, None)
        self.oracle.set_reference(None, None)

    def append(self, frames):
        for tier in (NOISY, CLEAN):
            K, V = self.t(("K", self.chunk, tier), frames), self.t(("V", self.chunk, tier), frames)
            self.gpu.append(tier, K.cuda(), V.cuda())
            self.oracle.append(tier, self._o(K), self._o(V))
        self.chunk += 1

    def inputs(self, step, frames):
        return [self.t((n, self.chunk, step), frames) for n in ("Q", "Kc", "Vc")]

    def attend(self, step, final, frames, rows=None, noalloc=False):
        Q, Kc, Vc = self.inputs(step, frames)
        L = Q.shape[1]
        lse = torch.empty((self.B, self.H, L), dtype=torch.float32, device="cuda")
        if noalloc:
            out = torch.empty_like(Q, device="cuda")
            Qd, Kd, Vd = Q.cuda(), Kc.cuda(), Vc.cuda()  # held until the kernel has run
            sa.sa_attend_noalloc(self.gpu.handle, Qd.data_ptr(), Kd.data_ptr(), Vd.data_ptr(),
                                 final, out.data_ptr(), lse.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream)
        else:
            out = self.gpu.attend(Q.cuda(), Kc.cuda(), Vc.cuda(), final, lse=lse)
        torch.cuda.synchronize()
        rows = np.arange(L) if rows is None else np.asarray(rows)
        o_gpu = f64(out.cpu())[:, rows][:, :, self.hsel]
        l_gpu = lse.cpu().double().numpy()[:, self.hsel][:, :, rows]
        o_ref, l_ref = self.oracle.attend(self._o(Q), self._o(Kc), self._o(Vc), final, rows=rows)
        return o_gpu, o_ref, l_gpu, l_ref

    def check_plan(self, final, frames):
        ids, base = self.oracle.positions(final, frames)
        tier = CLEAN if final else NOISY
        lens = [frames * self.hw if j == self.chunk else self.oracle.store[tier][j][0].shape[1]
                for j in ids]
        assert self.gpu.plan(final, frames) == (ids, [base[j] for j in ids], lens)


def _close(o_gpu, o_ref, l_gpu, l_ref, what):
    check_output(o_gpu, o_ref, what)
    lerr = np.abs(l_gpu - l_ref).max()
    assert lerr <= 1e-2, f"{what}: max |lse - oracle| = {lerr:.3e}"


CASES = [
    # name, B, H, D, F, th, tw, S, W, ref_frames
    ("d128_s1w3_r1", 1, 2, 128, 3, 9, 11, 1, 3, 1),
    ("d64_s2w2_r2", 2, 2, 64, 3, 8, 10, 2, 2, 2),
    ("d128_s0w4_r1", 1, 3, 128, 4, 6, 7, 0, 4, 1),
    ("d64_s1w1_r3", 1, 2, 64, 2, 10, 13, 1, 1, 3),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_variable_frames_with_reference_every_step(case):
    """Random chunk lengths (cached and generating), a reference image, both
    tiers, every output, past several evictions; the plan bit-exact."""
    name, B, H, D, F, th, tw, S, W, RF = case
    pair = PrefixPair(name, B, H, D, F, th, tw, S, W, RF)
    pair.set_reference(0)
    rng = np.random.default_rng(sum(map(ord, name)))
    for c in range(S + W + 3):
        for k, final in enumerate((False, True)):
            fq = int(rng.integers(1, F + 1))
            pair.check_plan(final, fq)
            _close(*pair.attend(k, final, fq), f"{name} chunk {c} step {k} ({fq} frames)")
        pair.append(int(rng.integers(1, F + 1)))
    assert pair.gpu.status() == sa.SA_OK


def test_variable_frames_without_reference_positions_shift():
    """ref_frames set but no reference given: positions still start after it."""
    pair = PrefixPair("noref", 1, 2, 128, 3, 8, 9, 1, 3, ref_frames=2)
    for fr in (3, 1, 2, 3, 2):
        pair.append(fr)
    for fq in (1, 3):
        pair.check_plan(True, fq)
        _close(*pair.attend(0, True, fq), f"no reference, {fq} frames")


def test_reference_replace_and_clear():
    pair = PrefixPair("replace", 1, 2, 128, 3, 8, 8, 1, 3, ref_frames=1)
    pair.set_reference("a")
    for fr in (3, 3, 2, 3):
        pair.append(fr)
    first, *_ = pair.attend(0, True, 3)
    _close(*pair.attend(0, True, 3), "reference a")
    pair.set_reference("b")
    o_b, o_ref_b, l_b, l_ref_b = pair.attend(0, True, 3)
    _close(o_b, o_ref_b, l_b, l_ref_b, "reference b")
    assert np.abs(o_b - first).max() > 10 * TOL  # the new reference is used
    pair.clear_reference()
    _close(*pair.attend(1, False, 2), "reference cleared")
    pair.set_reference("a")
    o_a, *_ = pair.attend(0, True, 3)
    assert np.array_equal(o_a, first)  # same inputs, same bits


def test_reference_with_current_chunk_only():
    """S = 0, W = 1: the chunk sees the reference and itself only."""
    pair = PrefixPair("refonly", 2, 2, 64, 2, 9, 9, 0, 1, ref_frames=2)
    pair.set_reference(0)
    for c in range(3):
        for fq in (2, 1):
            pair.check_plan(True, fq)
            _close(*pair.attend(c, True, fq), f"chunk {c}, {fq} frames")
        pair.append(2)


def test_full_size_720p_with_reference_sampled_rows():
    """720p chunk (3 x 45 x 80 tokens, 12 heads), one reference frame, short
    cached chunks; sampled rows of two heads against the oracle."""
    pair = PrefixPair("ref720", 1, 12, 128, 3, 45, 80, 1, 3, ref_frames=1, heads=[0, 7])
    pair.set_reference(0)
    for fr in (3, 2, 3, 1):
        pair.append(fr)
    for fq, final in ((3, True), (2, False)):
        L = fq * 45 * 80
        rows = sample_rows(L, 48, seed=fq)
        pair.check_plan(final, fq)
        _close(*pair.attend(0, final, fq, rows=rows), f"720p {fq} frames final={final}")


def test_noalloc_and_simt_with_reference():
    pair = PrefixPair("ref_paths", 1, 3, 128, 3, 10, 12, 1, 3, ref_frames=1)
    pair.set_reference(0)
    for fr in (3, 2, 3, 3):
        pair.append(fr)
    _close(*pair.attend(0, True, 3, noalloc=True), "noalloc with reference")
    Q, Kc, Vc = (t.cuda() for t in pair.inputs(0, 3))
    a = pair.gpu.attend(Q, Kc, Vc, True)
    b = pair.gpu.attend(Q, Kc, Vc, True, simt=True)
    torch.cuda.synchronize()
    assert (a.double() - b.double()).abs().max().item() <= TOL


def test_sparse_variable_frames_and_reference_refusal():
    pair = PrefixPair("sparse_frames", 1, 2, 128, 3, 10, 14, 1, 3, ref_frames=1)
    for fr in (2, 3, 1, 3):
        pair.append(fr)
    Q, Kc, Vc = pair.inputs(0, 3)
    nq, nk = pair.gpu.block_grid(True)
    _, _, lens = pair.gpu.plan(True)
    assert nk == len(key_tiles(lens))
    rng = np.random.default_rng(5)
    mask = (rng.random((1, 2, nq, nk)) < 0.4).astype(np.uint8)
    lse = torch.empty((1, 2, Q.shape[1]), dtype=torch.float32, device="cuda")
    out = pair.gpu.attend_sparse(Q.cuda(), Kc.cuda(), Vc.cuda(), True,
                                 torch.from_numpy(mask).cuda(), lse=lse)
    torch.cuda.synchronize()
    o_ref, l_ref = block_sparse_attend(pair.oracle, f64(Q), f64(Kc), f64(Vc), True, mask)
    check_output(f64(out.cpu()), o_ref, "sparse, variable frames")
    seen = np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(lse.cpu().numpy()), seen)
    # with a reference set the block grid does not cover its keys: refused
    pair.set_reference(0)
    with pytest.raises(sa.SaError) as e:
        pair.gpu.attend_sparse(Q.cuda(), Kc.cuda(), Vc.cuda(), True, torch.from_numpy(mask).cuda())
    assert e.value.status == sa.SA_ERR_UNSUPPORTED


def test_bad_frames_and_reference_arguments():
    h = sa.StreamingAttention(dict(batch=1, heads=1, head_dim=64, frames_per_chunk=2, tok_h=8,
                                   tok_w=8, sink_chunks=1, window_chunks=2))
    K = torch.zeros((1, 128, 1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sa.SaError) as e:
        sa.sa_set_reference(h.handle, K.data_ptr(), K.data_ptr())
    assert e.value.status == sa.SA_ERR_STATE
    for n in (0, 3):
        with pytest.raises(sa.SaError) as e:
            sa.sa_append_chunk_frames(h.handle, NOISY, K.data_ptr(), K.data_ptr(), n)
        assert e.value.status == sa.SA_ERR_INVALID_ARG
        with pytest.raises(sa.SaError) as e:
            sa.sa_attend_frames(h.handle, K.data_ptr(), K.data_ptr(), K.data_ptr(), n, 0,
                                torch.empty_like(K).data_ptr())
        assert e.value.status == sa.SA_ERR_INVALID_ARG
    assert h.chunk_count(NOISY) == 0

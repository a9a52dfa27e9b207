"""Frame-aligned editing attention on the GPU vs the float64 oracle (sa_attend_aligned)."""

import numpy as np
import pytest
import torch

import block_causal_streaming_sa_b200 as sa
from harness import check_output, f64, sample_rows
from oracle.editing import frame_aligned_attend
from oracle.stream import CLEAN, NOISY, OracleConfig, StreamOracle
from sa_inputs import normal_bf16, seed_of

pytestmark = pytest.mark.gpu


class EditPair:
    """A library handle and an oracle stream driven with the same target chunks,
    source frames and reference image. ``heads`` restricts the oracle."""

    def __init__(self, name, B, H, D, F, th, tw, S, W, ref_frames=0, heads=None):
        self.name, self.hw = name, th * tw
        self.B, self.H, self.D = B, H, D
        self.cfg = dict(batch=B, heads=H, head_dim=D, frames_per_chunk=F, tok_h=th, tok_w=tw,
                        sink_chunks=S, window_chunks=W, ref_frames=ref_frames)
        self.gpu = sa.StreamingAttention(self.cfg)
        self.hsel = list(range(H)) if heads is None else list(heads)
        self.oracle = StreamOracle(OracleConfig(B, len(self.hsel), D, F, th, tw, S, W,
                                                ref_frames=ref_frames))
        self.chunk = 0
        if ref_frames:
            K, V = (self.t(("ref", n), ref_frames) for n in "KV")
            self.gpu.set_reference(K.cuda(), V.cuda())
            self.oracle.set_reference(self._o(K), self._o(V))

    def t(self, tag, frames):
        return normal_bf16(seed_of(self.name, tag), (self.B, frames * self.hw, self.H, self.D))

    def _o(self, t):
        return f64(t)[:, :, self.hsel]

    def append(self, frames):
        for tier in (NOISY, CLEAN):
            K, V = (self.t((n, self.chunk, tier), frames) for n in "KV")
            self.gpu.append(tier, K.cuda(), V.cuda())
            self.oracle.append(tier, self._o(K), self._o(V))
        self.chunk += 1

    def inputs(self, step, frames):
        return [self.t((n, self.chunk, step), frames) for n in ("Q", "Kc", "Vc", "Ks", "Vs")]

    def attend(self, step, final, frames, rows=None, inputs=None):
        Q, Kc, Vc, Ks, Vs = inputs if inputs is not None else self.inputs(step, frames)
        L = Q.shape[1]
        lse = torch.empty((self.B, self.H, L), dtype=torch.float32, device="cuda")
        dev = [t.cuda() for t in (Q, Kc, Vc, Ks, Vs)]
        out = self.gpu.attend_aligned(*dev, final, lse=lse)
        torch.cuda.synchronize()
        rows = np.arange(L) if rows is None else np.asarray(rows)
        o_gpu = f64(out.cpu())[:, rows][:, :, self.hsel]
        l_gpu = lse.cpu().double().numpy()[:, self.hsel][:, :, rows]
        o_ref, l_ref = frame_aligned_attend(self.oracle, *(self._o(t) for t in (Q, Kc, Vc, Ks, Vs)),
                                            final, rows=rows)
        return o_gpu, o_ref, l_gpu, l_ref


def _close(o_gpu, o_ref, l_gpu, l_ref, what):
    check_output(o_gpu, o_ref, what)
    lerr = np.abs(l_gpu - l_ref).max()
    assert lerr <= 1e-2, f"{what}: max |lse - oracle| = {lerr:.3e}"


CASES = [
    # name, B, H, D, F, th, tw, S, W, ref_frames
    ("d128_s1w3_ref", 1, 2, 128, 3, 9, 11, 1, 3, 1),   # 99 tokens a frame: tiles hold 2 frames
    ("d64_s2w2", 2, 2, 64, 3, 12, 15, 2, 2, 0),         # 180 tokens a frame: tiles straddle
    ("d128_tiny_frames", 1, 2, 128, 8, 4, 5, 1, 2, 0),  # 20 tokens a frame: 6+ frames a tile
    ("d64_current_only", 1, 3, 64, 2, 10, 10, 0, 1, 2),  # source group alone in a split half
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_every_chunk_and_step_with_variable_frames(case):
    name, B, H, D, F, th, tw, S, W, RF = case
    pair = EditPair(name, B, H, D, F, th, tw, S, W, RF)
    rng = np.random.default_rng(sum(map(ord, name)))
    for c in range(S + W + 2):
        for k, final in enumerate((False, True)):
            fq = int(rng.integers(1, F + 1))
            _close(*pair.attend(k, final, fq), f"{name} chunk {c} step {k} ({fq} frames)")
        pair.append(int(rng.integers(1, F + 1)))
    assert pair.gpu.status() == sa.SA_OK


def test_full_size_720p_sampled_rows():
    """720p chunk (3 x 45 x 80 tokens): 128-row tiles straddle frame edges."""
    pair = EditPair("edit720", 1, 12, 128, 3, 45, 80, 1, 3, ref_frames=1, heads=[0, 11])
    for fr in (3, 3, 3):
        pair.append(fr)
    L = 3 * 3600
    rows = np.unique(np.concatenate([sample_rows(L, 40, seed=3),
                                     [3599, 3600, 3601, 7199, 7200, 3583, 3584, 7167, 7168]]))
    _close(*pair.attend(0, True, 3, rows=rows), "720p editing, final step")
    _close(*pair.attend(1, False, 2, rows=rows[rows < 7200]), "720p editing, 2 frames")


def test_no_mixing_across_times_on_gpu():
    """Perturbing source frame f changes only target rows of frame f (bit-exact elsewhere)."""
    pair = EditPair("mixing", 1, 2, 128, 4, 6, 7, 1, 2)
    for _ in range(3):
        pair.append(4)
    Q, Kc, Vc, Ks, Vs = (t.cuda() for t in pair.inputs(0, 4))
    base = pair.gpu.attend_aligned(Q, Kc, Vc, Ks, Vs, True).clone()
    hw = pair.hw
    for f in range(4):
        Ks2, Vs2 = Ks.clone(), Vs.clone()
        Ks2[:, f * hw:(f + 1) * hw] += 1.0
        Vs2[:, f * hw:(f + 1) * hw] -= 1.0
        out = pair.gpu.attend_aligned(Q, Kc, Vc, Ks2, Vs2, True)
        torch.cuda.synchronize()
        inside = torch.zeros(out.shape[1], dtype=torch.bool, device="cuda")
        inside[f * hw:(f + 1) * hw] = True
        assert torch.equal(out[:, ~inside], base[:, ~inside]), f"frame {f} leaked"
        assert (out[:, inside] != base[:, inside]).any()


def test_plain_attention_after_editing_uses_no_source():
    """sa_attend after sa_attend_aligned on the same chunk sees no source keys."""
    pair = EditPair("after", 1, 2, 64, 2, 8, 8, 1, 2)
    pair.append(2)
    Q, Kc, Vc, Ks, Vs = (t.cuda() for t in pair.inputs(0, 2))
    pair.gpu.attend_aligned(Q, Kc, Vc, Ks, Vs, False)
    out = pair.gpu.attend(Q, Kc, Vc, False)
    torch.cuda.synchronize()
    o_ref, _ = pair.oracle.attend(*(pair._o(t.cpu()) for t in (Q, Kc, Vc)), False)
    check_output(f64(out.cpu()), o_ref, "plain attention after editing")


def test_too_many_key_groups_is_refused():
    h = sa.StreamingAttention(dict(batch=1, heads=1, head_dim=64, frames_per_chunk=1, tok_h=8,
                                   tok_w=8, sink_chunks=6, window_chunks=10))
    x = torch.zeros((1, 64, 1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sa.SaError) as e:
        h.attend_aligned(x, x, x, x, x, True)
    assert e.value.status == sa.SA_ERR_UNSUPPORTED

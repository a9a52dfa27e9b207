"""Seeded random configurations against the oracle: head dim, batch, heads, frame
grid (ragged tiles), sink / window sizes, reference frames, chunk lengths, and
which entry point serves each step (plain, frame-aligned editing, SIMT)."""

import numpy as np
import pytest
import torch

import block_causal_streaming_sa_b200 as sa
from harness import check_output, f64
from oracle.editing import frame_aligned_attend
from oracle.stream import CLEAN, NOISY, OracleConfig, StreamOracle
from sa_inputs import normal_bf16, seed_of

pytestmark = pytest.mark.gpu


def _config(rng):
    D = int(rng.choice([64, 128]))
    S = int(rng.integers(0, 3))
    W = int(rng.integers(1, 4))
    return dict(batch=int(rng.integers(1, 3)), heads=int(rng.integers(1, 4)), head_dim=D,
                frames_per_chunk=int(rng.integers(1, 4)), tok_h=int(rng.integers(3, 13)),
                tok_w=int(rng.integers(3, 17)), sink_chunks=S, window_chunks=W,
                ref_frames=int(rng.choice([0, 0, 1, 2])))


@pytest.mark.parametrize("seed", range(40))
def test_random_configuration_stream(seed):
    rng = np.random.default_rng(1000 + seed)
    cfg = _config(rng)
    B, H, D, F = cfg["batch"], cfg["heads"], cfg["head_dim"], cfg["frames_per_chunk"]
    hw = cfg["tok_h"] * cfg["tok_w"]
    gpu = sa.StreamingAttention(cfg)
    orc = StreamOracle(OracleConfig(B, H, D, F, cfg["tok_h"], cfg["tok_w"], cfg["sink_chunks"],
                                    cfg["window_chunks"], ref_frames=cfg["ref_frames"]))
    t = lambda tag, fr: normal_bf16(seed_of("fuzz", seed, tag), (B, fr * hw, H, D))  # noqa: E731
    if cfg["ref_frames"] and rng.random() < 0.8:
        Kr, Vr = t("Kr", cfg["ref_frames"]), t("Vr", cfg["ref_frames"])
        gpu.set_reference(Kr.cuda(), Vr.cuda())
        orc.set_reference(f64(Kr), f64(Vr))
    for c in range(cfg["sink_chunks"] + cfg["window_chunks"] + 2):
        for k, final in enumerate((False, True)):
            fq = int(rng.integers(1, F + 1))
            Q, Kc, Vc = (t((n, c, k), fq) for n in ("Q", "Kc", "Vc"))
            mode = rng.choice(["plain", "aligned", "simt"] if fq == F else ["plain", "aligned"])
            if mode == "aligned":
                Ks, Vs = t(("Ks", c, k), fq), t(("Vs", c, k), fq)
                out = gpu.attend_aligned(*(x.cuda() for x in (Q, Kc, Vc, Ks, Vs)), final)
                ref, _ = frame_aligned_attend(orc, *(f64(x) for x in (Q, Kc, Vc, Ks, Vs)), final)
            else:
                out = gpu.attend(Q.cuda(), Kc.cuda(), Vc.cuda(), final, simt=(mode == "simt"))
                ref, _ = orc.attend(f64(Q), f64(Kc), f64(Vc), final)
            torch.cuda.synchronize()
            check_output(f64(out.cpu()), ref, f"seed {seed} {cfg} chunk {c} step {k} {mode}")
        fr = int(rng.integers(1, F + 1))
        for tier in (NOISY, CLEAN):
            K, V = t(("K", c, tier), fr), t(("V", c, tier), fr)
            gpu.append(tier, K.cuda(), V.cuda())
            orc.append(tier, f64(K), f64(V))
    assert gpu.status() == sa.SA_OK

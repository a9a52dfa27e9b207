"""Tensors past 2^31 elements: one chunk of 266 240 tokens x 64 heads x 128 dims
(2.18e9 elements, 4.4 GB per tensor), so row offsets, the key staging and the
TMA descriptors of the caller's V (strides of several GB) need 64-bit
arithmetic. Sampled rows of two heads against the oracle."""

import numpy as np
import pytest
import torch

import block_causal_streaming_sa_b200 as sa
from harness import check_output, f64, sample_rows
from oracle.stream import OracleConfig, StreamOracle
from sa_inputs import device_normal_bf16, seed_of

pytestmark = pytest.mark.gpu


def test_chunk_past_two_to_the_31_elements():
    B, H, D, F, th, tw = 1, 64, 128, 1, 520, 512
    L = F * th * tw
    assert B * L * H * D > 2 ** 31
    cfg = dict(batch=B, heads=H, head_dim=D, frames_per_chunk=F, tok_h=th, tok_w=tw,
               sink_chunks=0, window_chunks=1)
    attn = sa.StreamingAttention(cfg)
    Q, Kc, Vc = (device_normal_bf16(seed_of("large", n), (B, L, H, D), "cuda")
                 for n in ("Q", "Kc", "Vc"))
    lse = torch.empty((B, H, L), dtype=torch.float32, device="cuda")
    O = attn.attend(Q, Kc, Vc, True, lse=lse)
    torch.cuda.synchronize()
    assert attn.status() == sa.SA_OK
    heads = [0, H - 1]
    rows = np.unique(np.concatenate([sample_rows(L, 24, seed=11), [L - 1, L // 2]]))
    # the oracle sees the checked heads only (it works per (b, h))
    orc = StreamOracle(OracleConfig(B, len(heads), D, F, th, tw, 0, 1))
    sel = lambda t: f64(t[:, :, heads].cpu())  # noqa: E731
    o_ref, l_ref = orc.attend(sel(Q), sel(Kc), sel(Vc), True,
                              rows=rows)
    o_gpu = f64(O[:, rows][:, :, heads].cpu())
    check_output(o_gpu, o_ref, "2^31+ elements")
    l_gpu = lse[:, heads][:, :, rows].double().cpu().numpy()
    assert np.abs(l_gpu - l_ref).max() <= 1e-2

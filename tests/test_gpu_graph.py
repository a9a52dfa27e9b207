"""CUDA graph capture of the attention call.

The calls enqueue work on the caller's stream and neither allocate nor
synchronise, so they can be captured. A captured attention keeps the plan of
the chunk it was captured for (attended chunks, slots, relocated positions are
launch arguments), so it is replayed for that chunk's steps of the same tier
with new contents in the same input buffers.
"""

import pytest
import torch

import block_causal_streaming_sa_b200 as sa
from oracle.stream import CLEAN, NOISY
from sa_inputs import Workload

pytestmark = pytest.mark.gpu


def test_graph_replays_noisy_steps_bit_identical_to_direct_calls():
    w = Workload("graph", 1, 4, 128, 3, 10, 12, sink=1, window=3, steps=4, stream=4)
    attn = sa.StreamingAttention(w.config_dict())
    for c in range(w.stream):
        for tier, names in ((NOISY, ("Kn", "Vn")), (CLEAN, ("Kcl", "Vcl"))):
            K, V = (w.tensor(n, c).cuda() for n in names)
            attn.append(tier, K, V)
    c = w.stream
    Qb, Kb, Vb = (torch.empty(w.shape(), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    Ob = torch.empty_like(Qb)
    for t, n in zip((Qb, Kb, Vb), ("Q", "Kc", "Vc")):
        t.copy_(w.tensor(n, c, 0))
    attn.attend(Qb, Kb, Vb, False, out=Ob)  # warm-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        attn.attend(Qb, Kb, Vb, False, out=Ob)
    for step in range(w.steps - 1):
        Q, Kc, Vc = (w.tensor(n, c, step).cuda() for n in ("Q", "Kc", "Vc"))
        Qb.copy_(Q)
        Kb.copy_(Kc)
        Vb.copy_(Vc)
        g.replay()
        torch.cuda.synchronize()
        direct = attn.attend(Q, Kc, Vc, False)
        torch.cuda.synchronize()
        assert torch.equal(Ob, direct), step
    assert attn.status() == sa.SA_OK

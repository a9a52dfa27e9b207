"""sa_attend_noalloc, the attention call that allocates nothing.

Some callers may not call cudaMalloc at all: code inside another framework's
allocator-free region, a real-time loop that must not allocate after start-up,
or a plugin that is handed only the tensors it works on. For them the library
has sa_attend_noalloc: the same attention as sa_attend, with the one piece of
per-call scratch (the generating chunk's rotated keys) kept in a fixed array
inside the library instead of in caller-provided memory.

These tests call it through the C ABI and check it against sa_attend on two
calls in a row, and that a chunk too large for the fixed array is refused.
This file is collected last, so a failure here leaves every other test run.
"""

import pytest
import torch

import block_causal_streaming_sa_b200 as sa
from harness import TOL
from oracle.stream import CLEAN, NOISY
from sa_inputs import Workload

pytestmark = pytest.mark.gpu


def _stream(w):
    h = sa.StreamingAttention(w.config_dict())
    for c in range(w.stream):
        Kn, Vn, Kcl, Vcl = (w.tensor(n, c).cuda() for n in ("Kn", "Vn", "Kcl", "Vcl"))
        h.append(NOISY, Kn, Vn)
        h.append(CLEAN, Kcl, Vcl)
    return h


def _call(fn, h, Q, Kc, Vc, final):
    b, l, heads, _ = Q.shape
    out = torch.empty_like(Q)
    lse = torch.empty((b, heads, l), dtype=torch.float32, device=Q.device)
    fn(h.handle, Q.data_ptr(), Kc.data_ptr(), Vc.data_ptr(), final, out.data_ptr(),
       lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return out, lse


@pytest.mark.parametrize("D", [128, 64])
def test_noalloc_matches_sa_attend_on_two_calls_in_a_row(D):
    w = Workload(f"noalloc_d{D}", 2, 3, D, 3, 12, 20, sink=1, window=3, steps=2, stream=5)
    h = _stream(w)
    inputs = [tuple(w.tensor(n, w.stream, step).cuda() for n in ("Q", "Kc", "Vc"))
              for step in range(2)]
    finals = (False, True)
    refs = [_call(sa.sa_attend, h, *x, f) for x, f in zip(inputs, finals)]
    # two calls in a row on the shared fixed array, then the first again
    for k in (0, 1, 0):
        out, lse = _call(sa.sa_attend_noalloc, h, *inputs[k], finals[k])
        torch.cuda.synchronize()
        err = (out.double() - refs[k][0].double()).abs().max().item()
        lerr = (lse - refs[k][1]).abs().max().item()
        assert err <= TOL and lerr <= TOL, (k, err, lerr)
    assert h.status() == sa.SA_OK


def test_noalloc_refuses_chunks_beyond_its_fixed_array():
    # B*H*L*D*2 = 2*40*6120*128*2 bytes = 125 MB > 64 MiB
    w = Workload("noalloc_big", 2, 40, 128, 3, 34, 60, sink=0, window=1, steps=1, stream=0)
    h = sa.StreamingAttention(w.config_dict())
    Q = torch.zeros(w.shape(), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sa.SaError) as e:
        _call(sa.sa_attend_noalloc, h, Q, Q.clone(), Q.clone(), True)
    assert e.value.status == sa.SA_ERR_UNSUPPORTED

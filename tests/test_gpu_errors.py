"""Host-side error paths with a live handle: every refused call launches nothing,
leaves the handle's counters as they were, and the handle keeps working. No
device fault is involved (the CUDA-error case is a host-side test hook)."""

import ctypes

import numpy as np
import pytest
import torch

import block_causal_streaming_sa_b200 as sa
from harness import check_output, f64
from oracle.stream import CLEAN, NOISY, OracleConfig, StreamOracle
from sa_inputs import Workload

pytestmark = pytest.mark.gpu

W = Workload("errors", 1, 2, 64, 2, 8, 8, sink=1, window=2, steps=2, stream=3)


def _tensors(c, step=0):
    return [W.tensor(n, c, step).cuda() for n in ("Q", "Kc", "Vc")]


def _ptrs(*ts):
    return [t.data_ptr() for t in ts]


def test_tiers_out_of_step_and_double_append_are_state_errors():
    h = sa.StreamingAttention(W.config_dict())
    K, V = W.tensor("Kn", 0).cuda(), W.tensor("Vn", 0).cuda()
    h.append(NOISY, K, V)
    with pytest.raises(sa.SaError) as e:  # clean tier one behind: no attention
        h.attend(*_tensors(1), False)
    assert e.value.status == sa.SA_ERR_STATE
    with pytest.raises(sa.SaError) as e:  # noisy tier already ahead
        h.append(NOISY, K, V)
    assert e.value.status == sa.SA_ERR_STATE
    assert (h.chunk_count(NOISY), h.chunk_count(CLEAN)) == (1, 0)
    h.append(CLEAN, W.tensor("Kcl", 0).cuda(), W.tensor("Vcl", 0).cuda())
    # the refused attention staged no keys either: its attention half alone is refused
    Q, _, Vc = _tensors(1)
    O = torch.empty_like(Q)
    with pytest.raises(sa.SaError) as e:
        sa.sa_attend_staged(h.handle, Q.data_ptr(), Vc.data_ptr(), False, O.data_ptr())
    assert e.value.status == sa.SA_ERR_STATE
    h.attend(*_tensors(1), False)
    torch.cuda.synchronize()
    assert h.status() == sa.SA_OK


def test_staged_attention_needs_staged_keys():
    h = sa.StreamingAttention(W.config_dict())
    Q, _, Vc = _tensors(0)
    O = torch.empty_like(Q)
    with pytest.raises(sa.SaError) as e:
        sa.sa_attend_staged(h.handle, Q.data_ptr(), Vc.data_ptr(), False, O.data_ptr())
    assert e.value.status == sa.SA_ERR_STATE


def test_undersized_or_host_buffer_is_refused():
    cfg = sa.make_config(**W.config_dict())
    need = sa.sa_required_bytes(cfg)
    buf = torch.empty(need, dtype=torch.uint8, device="cuda")
    with pytest.raises(sa.SaError) as e:
        sa.sa_create(cfg, buf.data_ptr(), need - 1)
    assert e.value.status == sa.SA_ERR_INVALID_ARG
    host = torch.empty(need + 256, dtype=torch.uint8).pin_memory()
    base = (host.data_ptr() + 255) // 256 * 256
    with pytest.raises(sa.SaError) as e:
        sa.sa_create(cfg, base, need)
    assert e.value.status == sa.SA_ERR_INVALID_ARG
    handle = sa.sa_create(cfg, buf.data_ptr(), need)  # the right buffer works
    sa.sa_destroy(handle)


def test_misaligned_and_aliased_pointers_are_refused():
    h = sa.StreamingAttention(W.config_dict())
    Q, Kc, Vc = _tensors(0)
    O = torch.empty_like(Q)
    stream = torch.cuda.current_stream().cuda_stream
    lib = sa.lib()
    bad = Q.data_ptr() + 2
    for args in ((bad, Kc.data_ptr(), Vc.data_ptr(), O.data_ptr()),
                 (Q.data_ptr(), Kc.data_ptr(), Vc.data_ptr(), Q.data_ptr())):
        rc = lib.sa_attend(h.handle, ctypes.c_void_p(args[0]), ctypes.c_void_p(args[1]),
                           ctypes.c_void_p(args[2]), 0, ctypes.c_void_p(args[3]), None,
                           ctypes.c_void_p(stream))
        assert rc == sa.SA_ERR_INVALID_ARG, sa.last_error(h.handle)
    assert h.status() == sa.SA_OK


def test_injected_cuda_error_launches_nothing_and_the_handle_recovers():
    h = sa.StreamingAttention(W.config_dict())
    orc = StreamOracle(OracleConfig(W.batch, W.heads, W.head_dim, W.frames, W.tok_h, W.tok_w,
                                    W.sink, W.window))
    for c in range(2):
        for tier, names in ((NOISY, ("Kn", "Vn")), (CLEAN, ("Kcl", "Vcl"))):
            K, V = (W.tensor(n, c) for n in names)
            sa.sa_debug_inject_cuda_error(h.handle)
            with pytest.raises(sa.SaError) as e:
                h.append(tier, K.cuda(), V.cuda())
            assert e.value.status == sa.SA_ERR_CUDA
            h.append(tier, K.cuda(), V.cuda())
            orc.append(tier, f64(K), f64(V))
    assert (h.chunk_count(NOISY), h.chunk_count(CLEAN)) == (2, 2)
    Q, Kc, Vc = _tensors(2)
    sa.sa_debug_inject_cuda_error(h.handle)
    with pytest.raises(sa.SaError) as e:
        h.attend(Q, Kc, Vc, True)
    assert e.value.status == sa.SA_ERR_CUDA
    out = h.attend(Q, Kc, Vc, True)
    torch.cuda.synchronize()
    ref, _ = orc.attend(*(f64(t.cpu()) for t in (Q, Kc, Vc)), True)
    check_output(f64(out.cpu()), ref, "after an injected error")
    assert h.status() == sa.SA_OK
    assert np.isfinite(f64(out.cpu())).all()

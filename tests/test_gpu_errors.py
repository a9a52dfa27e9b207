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


def test_host_pointers_are_refused_before_any_launch():
    """Pageable or pinned host memory passed as a tensor is refused on the host
    (SA_ERR_INVALID_ARG): nothing is launched, no key is staged, the counters
    stay, and the handle keeps working."""
    h = sa.StreamingAttention(W.config_dict())
    lib = sa.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = ctypes.c_void_p
    K, V = W.tensor("Kn", 0).cuda(), W.tensor("Vn", 0).cuda()
    pageable = W.tensor("Kn", 0)  # CPU tensor
    pinned = W.tensor("Vn", 0).pin_memory()
    for host in (pageable, pinned):
        hp = host.data_ptr()
        assert lib.sa_append_chunk(h.handle, NOISY, p(hp), p(V.data_ptr()), stream) \
            == sa.SA_ERR_INVALID_ARG
        assert "host memory" in sa.last_error(h.handle)
        assert lib.sa_append_chunk(h.handle, NOISY, p(K.data_ptr()), p(hp), stream) \
            == sa.SA_ERR_INVALID_ARG
    assert (h.chunk_count(NOISY), h.chunk_count(CLEAN)) == (0, 0)
    h.append(NOISY, K, V)
    h.append(CLEAN, K, V)
    Q, Kc, Vc = _tensors(1)
    O = torch.empty_like(Q)
    lse = torch.empty((W.batch, W.heads, W.chunk_len), dtype=torch.float32, device="cuda")
    lse_host = torch.empty_like(lse, device="cpu").pin_memory()
    hq = pinned.data_ptr()
    dev = dict(Q=Q.data_ptr(), Kc=Kc.data_ptr(), Vc=Vc.data_ptr(), O=O.data_ptr())
    for which in ("Q", "Kc", "Vc", "O"):
        args = dict(dev, **{which: hq})
        rc = lib.sa_attend(h.handle, p(args["Q"]), p(args["Kc"]), p(args["Vc"]), 0, p(args["O"]),
                           None, stream)
        assert rc == sa.SA_ERR_INVALID_ARG, which
        assert which in sa.last_error(h.handle)
    rc = lib.sa_attend(h.handle, p(dev["Q"]), p(dev["Kc"]), p(dev["Vc"]), 0, p(dev["O"]),
                       p(lse_host.data_ptr()), stream)
    assert rc == sa.SA_ERR_INVALID_ARG
    # no refused call staged keys: the attention half alone still finds none
    rc = lib.sa_attend_staged(h.handle, p(dev["Q"]), p(dev["Vc"]), 0, p(dev["O"]), None, stream)
    assert rc == sa.SA_ERR_STATE
    nq, nk = h.block_grid(False)
    mask_host = torch.ones((W.batch, W.heads, nq, nk), dtype=torch.uint8).pin_memory()
    rc = lib.sa_attend_sparse(h.handle, p(dev["Q"]), p(dev["Kc"]), p(dev["Vc"]), 0,
                              p(mask_host.data_ptr()), p(dev["O"]), None, stream)
    assert rc == sa.SA_ERR_INVALID_ARG and "block_mask" in sa.last_error(h.handle)
    rc = lib.sa_attend_noalloc(h.handle, p(dev["Q"]), p(hq), p(dev["Vc"]), 0, p(dev["O"]), None,
                               stream)
    assert rc == sa.SA_ERR_INVALID_ARG
    # exchange calls (no handle)
    x = torch.zeros((1, 8, 4, 64), dtype=torch.bfloat16)
    nbytes = sa.sa_exchange_block_bytes(1, 8, 4, 64, 2, 1, sa.SA_PAYLOAD_FP8)
    buf = torch.empty(2 * nbytes, dtype=torch.uint8, device="cuda")
    with pytest.raises(sa.SaError) as e:
        sa.sa_exchange_pack(x.data_ptr(), 1, 8, 4, 64, 2, 1, sa.SA_PAYLOAD_FP8, buf.data_ptr())
    assert e.value.status == sa.SA_ERR_INVALID_ARG
    # the handle still computes the right thing
    orc = StreamOracle(OracleConfig(W.batch, W.heads, W.head_dim, W.frames, W.tok_h, W.tok_w,
                                    W.sink, W.window))
    orc.append(NOISY, f64(K.cpu()), f64(V.cpu()))
    orc.append(CLEAN, f64(K.cpu()), f64(V.cpu()))
    out = h.attend(Q, Kc, Vc, True)
    torch.cuda.synchronize()
    ref, _ = orc.attend(*(f64(t.cpu()) for t in (Q, Kc, Vc)), True)
    check_output(f64(out.cpu()), ref, "after refused host pointers")
    assert h.status() == sa.SA_OK


def test_fp16_range_of_rotated_pairs_is_flagged():
    """A Q or K pair with a norm above 65504 cannot enter the fp16 score MMA at
    every angle: the device status word records it (SA_ERR_RANGE) whatever the
    pair's position, until sa_reset; pairs just inside the range are not
    flagged."""
    h = sa.StreamingAttention(W.config_dict())
    Kn, Vn = W.tensor("Kn", 0).cuda(), W.tensor("Vn", 0).cuda()

    def with_pair(t, a, b, token=37, head=1, pair=5):
        t = t.clone()
        t[0, token, head, 2 * pair] = a
        t[0, token, head, 2 * pair + 1] = b
        return t

    # norm 60000.x: inside the range
    h.append(NOISY, with_pair(Kn, 60000.0, 1.0), Vn)
    h.append(CLEAN, Kn, Vn)
    Q, Kc, Vc = _tensors(1)
    h.attend(with_pair(Q, -60000.0, 0.5), Kc, Vc, False)
    assert h.status() == sa.SA_OK
    # each value inside fp16, the pair's norm (70711) outside: flagged
    h.append(NOISY, with_pair(Kn, 50000.0, 50000.0), Vn)
    assert h.status() == sa.SA_ERR_RANGE
    assert "65504" in sa.last_error(h.handle)
    h.reset()
    assert h.status() == sa.SA_OK
    # one value above the fp16 maximum, in the current chunk's keys, then in Q
    h.append(NOISY, Kn, Vn)
    h.append(CLEAN, Kn, Vn)
    h.attend(Q, with_pair(Kc, 1.0e5, 0.0, token=0, head=0, pair=0), Vc, True)
    assert h.status() == sa.SA_ERR_RANGE
    h.reset()
    h.append(NOISY, Kn, Vn)
    h.append(CLEAN, Kn, Vn)
    h.attend(with_pair(Q, 0.0, -7.0e4, token=W.chunk_len - 1), Kc, Vc, True)
    assert h.status() == sa.SA_ERR_RANGE
    h.reset()
    h.append(NOISY, Kn, Vn)
    h.append(CLEAN, Kn, Vn)
    h.attend(Q, Kc, Vc, True)
    assert h.status() == sa.SA_OK


def test_kernel_clock_record_of_the_last_attention():
    """sa_debug_kernel_clock reads the per-CTA stamps of the most recent attention
    launch: a clock between 300 MHz and the part's 2.1 GHz ceiling, and a span
    no longer than the launch as CUDA events time it."""
    h = sa.StreamingAttention(W.config_dict())
    Kn, Vn = W.tensor("Kn", 0).cuda(), W.tensor("Vn", 0).cuda()
    h.append(NOISY, Kn, Vn)
    h.append(CLEAN, Kn, Vn)
    Q, Kc, Vc = _tensors(1)
    h.attend(Q, Kc, Vc, False)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    h.attend(Q, Kc, Vc, True)
    e1.record()
    mhz, span_us = sa.sa_debug_kernel_clock()
    assert 300.0 < mhz < 2100.0, mhz
    assert 0.0 < span_us <= 1e3 * e0.elapsed_time(e1) + 5.0, (span_us, e0.elapsed_time(e1))
    assert h.status() == sa.SA_OK

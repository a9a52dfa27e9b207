"""The C ABI on the CPU: the library loads, exports what include/sa.h declares,
validates configs, and its host-side cache plan matches the oracle bit for bit."""

import ctypes

import pytest
import torch

import block_causal_streaming_sa_b200 as sa
from oracle.cache import RingCacheModel
from sa_inputs import WORKLOADS


def _cfg(**kw):
    base = dict(batch=1, heads=2, head_dim=64, frames_per_chunk=3, tok_h=8, tok_w=8,
                sink_chunks=1, window_chunks=2)
    base.update(kw)
    return sa.make_config(**base)


def test_library_exports_every_declared_symbol():
    syms = sa.header_symbols()
    assert {"sa_create", "sa_append_chunk", "sa_attend", "sa_destroy"} <= set(syms)
    handle = ctypes.CDLL(sa._binding.LIB_PATH)
    for name in syms:
        assert hasattr(handle, name), name
    sa.lib()  # argtypes for every declared symbol bind
    assert set(syms) <= set(sa._binding._SIGNATURES)


def test_validate_config_and_required_bytes():
    assert sa.sa_validate_config(_cfg()) == sa.SA_OK
    assert sa.sa_validate_config(_cfg(head_dim=96)) == sa.SA_ERR_UNSUPPORTED
    assert sa.sa_validate_config(_cfg(batch=0)) == sa.SA_ERR_INVALID_ARG
    assert sa.sa_validate_config(_cfg(window_chunks=0)) == sa.SA_ERR_INVALID_ARG
    assert sa.sa_validate_config(_cfg(sink_chunks=-1)) == sa.SA_ERR_INVALID_ARG
    assert sa.sa_validate_config(_cfg(sink_chunks=8, window_chunks=9)) == sa.SA_ERR_UNSUPPORTED
    assert sa.sa_validate_config(_cfg(softmax_scale=float("nan"))) == sa.SA_ERR_INVALID_ARG
    assert sa.sa_required_bytes(_cfg(head_dim=96)) == 0
    small = sa.sa_required_bytes(_cfg())
    big = sa.sa_required_bytes(_cfg(window_chunks=5))
    # two tiers x (S + W - 1) slots x (K + V) x B*H*L*D bf16 at least
    L = 3 * 8 * 8
    assert small >= 2 * 2 * 2 * (1 * 2 * L * 64) * 2
    assert big - small >= 2 * 3 * 2 * (2 * L * 64) * 2


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_plan_matches_oracle_cache_model(name):
    """ids, slots and relocated temporal bases of every chunk of the stream."""
    w = WORKLOADS[name]
    cfg = sa.make_config(**w.config_dict())
    model = RingCacheModel(w.sink, w.window)
    slot_of_id = {}
    for c in range(max(w.stream, 40)):
        ids, slots, tbase = sa.sa_plan(cfg, c)
        assert ids == model.attended()
        ranks = model.ranks()
        assert tbase == [ranks[j] * w.frames for j in ids]
        assert slots == [slot_of_id[j] if j != c else -1 for j in ids]
        slot, _ = model.append()
        assert sa.sa_slot_of(cfg, c) == (-1 if slot is None else slot)
        slot_of_id[c] = slot


@pytest.mark.parametrize("sink,window", [(0, 1), (0, 2), (2, 1), (3, 5), (7, 9), (0, 16)])
def test_plan_degenerate_and_extreme_windows(sink, window):
    cfg = _cfg(sink_chunks=sink, window_chunks=window)
    model = RingCacheModel(sink, window)
    for c in range(60):
        ids, slots, tbase = sa.sa_plan(cfg, c)
        assert ids == model.attended()
        assert max(tbase) + 2 <= (sink + window) * 3 - 1
        slot, _ = model.append()
        assert sa.sa_slot_of(cfg, c) == (-1 if slot is None else slot)


def test_plan_rejects_bad_arguments():
    with pytest.raises(sa.SaError):
        sa.sa_plan(_cfg(), -1)
    with pytest.raises(sa.SaError):
        sa.sa_plan(_cfg(head_dim=96), 0)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_create_without_gpu_fails_cleanly():
    with pytest.raises(sa.SaError) as e:
        sa.sa_create(_cfg(), 0x100000, 1 << 30)
    assert e.value.status in (sa.SA_ERR_INVALID_ARG, sa.SA_ERR_CUDA)
    with pytest.raises(sa.SaError):
        sa.sa_create(_cfg(), 0, 1 << 30)
    with pytest.raises(sa.SaError):
        sa.sa_create(_cfg(), 0x100000, 16)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_kernel_clock_without_gpu_fails_cleanly():
    mhz, span = ctypes.c_double(), ctypes.c_double()
    rc = sa.lib().sa_debug_kernel_clock(ctypes.byref(mhz), ctypes.byref(span))
    assert rc in (sa.SA_ERR_CUDA, sa.SA_ERR_STATE)
    assert sa.lib().sa_debug_kernel_clock(None, None) == sa.SA_ERR_INVALID_ARG


def test_null_handle_calls_fail_cleanly():
    lib = sa.lib()
    assert lib.sa_attend(None, None, None, None, 0, None, None, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_append_chunk(None, 0, None, None, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_reset(None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_chunk_count(None, 0) < 0
    assert lib.sa_destroy(None) == sa.SA_OK
    assert sa.last_error() != ""


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_block_grid_matches_oracle_tiling(name):
    from oracle.sparse import key_tiles

    w = WORKLOADS[name]
    cfg = sa.make_config(**w.config_dict())
    model = RingCacheModel(w.sink, w.window)
    for c in range(12):
        nq, nk = sa.sa_block_grid(cfg, c)
        assert nq == -(-w.chunk_len // 128)
        assert nk == len(key_tiles([w.chunk_len] * len(model.attended())))
        model.append()


def test_reference_config_validation_and_bytes():
    assert sa.sa_validate_config(_cfg(ref_frames=1)) == sa.SA_OK
    assert sa.sa_validate_config(_cfg(ref_frames=-1)) == sa.SA_ERR_INVALID_ARG
    assert sa.sa_validate_config(_cfg(ref_frames=1024)) == sa.SA_ERR_INVALID_ARG
    # the reference takes one of the SA_MAX_ATTENDED key groups
    assert sa.sa_validate_config(_cfg(sink_chunks=6, window_chunks=10)) == sa.SA_OK
    assert sa.sa_validate_config(_cfg(sink_chunks=6, window_chunks=10, ref_frames=1)) \
        == sa.SA_ERR_UNSUPPORTED
    assert sa.sa_validate_config(_cfg(sink_chunks=5, window_chunks=10, ref_frames=2)) == sa.SA_OK
    base = sa.sa_required_bytes(_cfg())
    with_ref = sa.sa_required_bytes(_cfg(ref_frames=2))
    # K and V planes of 2 frames x 64 tokens x 2 heads x 64 dims, bf16
    assert with_ref - base >= 2 * (2 * 64) * 2 * 64 * 2


@pytest.mark.parametrize("ref_frames", [1, 4])
def test_plan_bases_shift_by_reference_frames(ref_frames):
    """sa_plan's bases equal the oracle's positions for whole-chunk streams."""
    import numpy as np

    from oracle.stream import CLEAN, NOISY, OracleConfig, StreamOracle

    cfg = _cfg(sink_chunks=1, window_chunks=3, ref_frames=ref_frames)
    ocfg = OracleConfig(1, 1, 64, 3, 8, 8, 1, 3, ref_frames=ref_frames)
    orc = StreamOracle(ocfg)
    blank = np.zeros((1, 3 * 64, 1, 1))
    for c in range(10):
        ids, _, tbase = sa.sa_plan(cfg, c)
        o_ids, o_base = orc.positions(True, 3)
        assert ids == o_ids
        assert tbase == [o_base[j] for j in ids]
        for tier in (NOISY, CLEAN):
            orc.append(tier, blank, blank)


def test_null_handle_new_calls_fail_cleanly():
    lib = sa.lib()
    assert lib.sa_append_chunk_frames(None, 0, None, None, 1, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_set_reference(None, None, None, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_attend_frames(None, None, None, None, 1, 0, None, None, None) \
        == sa.SA_ERR_INVALID_ARG
    assert lib.sa_stage_keys_frames(None, None, 1, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_stream_plan(None, 0, 1, None, None, None, 16) < 0


def test_exchange_block_bytes_and_shape_checks():
    P8, P16 = sa.SA_PAYLOAD_FP8, sa.SA_PAYLOAD_BF16
    # fp8: D code bytes per vector, then one fp32 scale per vector, each part 16-byte aligned
    n = 1 * 2700 * 3  # vectors per block: B * T * H/G
    assert sa.sa_exchange_block_bytes(1, 2700, 12, 128, 4, 1, P8) == n * 128 + n * 4
    assert sa.sa_exchange_block_bytes(1, 10800, 3, 128, 4, 0, P16) == 2700 * 3 * 128 * 2
    assert sa.sa_exchange_block_bytes(1, 3, 1, 64, 1, 0, P8) == 192 + 16  # 12 B of scales -> 16
    for bad in [(1, 7, 3, 128, 2, 0, P8), (1, 8, 3, 128, 2, 1, P8), (1, 8, 4, 96, 2, 1, P8),
                (0, 8, 4, 64, 2, 1, P8), (1, 8, 4, 64, 0, 1, P8), (1, 8, 4, 64, 2, 2, P8),
                (1, 8, 4, 64, 2, 1, 7)]:
        assert sa.sa_exchange_block_bytes(*bad) == 0, bad
    with pytest.raises(sa.SaError):
        sa.sa_exchange_pack(0, 1, 8, 4, 64, 2, 1, P8, 0)


def test_status_codes_match_the_header():
    """The binding's status constants are the header's enum values, and every
    one has a name."""
    import re

    text = open(sa._binding.HEADER).read()
    enum = text[text.index("typedef enum {"):text.index("} sa_status;")]
    codes = {m.group(1): int(m.group(2)) for m in re.finditer(r"(SA_\w+)\s*=\s*(\d+)", enum)}
    assert codes == {n: getattr(sa._binding, n) for n in codes}
    assert set(codes) >= {"SA_OK", "SA_ERR_TIMEOUT", "SA_ERR_RANGE"}
    for name, value in codes.items():
        assert sa._binding.status_name(value) == name


def test_debug_layout_and_host_pointers_without_a_gpu():
    lib = sa.lib()
    ids = (ctypes.c_int32 * 4)()
    assert lib.sa_debug_layout(None, 0, ids, None, 4) < 0
    # exchange: a host pointer is not device memory (no GPU here: not a CUDA pointer)
    x = torch.zeros((1, 8, 4, 64), dtype=torch.bfloat16)
    buf = torch.zeros(1 << 14, dtype=torch.uint8)
    with pytest.raises(sa.SaError) as e:
        sa.sa_exchange_pack(x.data_ptr(), 1, 8, 4, 64, 2, 1, sa.SA_PAYLOAD_FP8, buf.data_ptr())
    assert e.value.status == sa.SA_ERR_INVALID_ARG
    assert "exchange: x" in sa.last_error()


def test_checked_build_exports_the_same_calls_and_says_so():
    """libsa_checked.so (device-side bounds checks) exports every declared call,
    and sa_build_info tells the two builds apart."""
    import os

    from block_causal_streaming_sa_b200 import build

    assert os.path.exists(build.LIB_CHECKED), "build() makes both libraries"
    checked = ctypes.CDLL(build.LIB_CHECKED)
    for name in sa.header_symbols():
        assert hasattr(checked, name), name
    assert checked.sa_build_info() == sa.SA_BUILD_DEVICE_CHECKS
    assert sa.lib().sa_build_info() == 0

"""The attention kernel's device exponentials against CUDA's exp2f and float64.

The softmax computes most of its 2^x on the exp unit (ex2.approx) and one in
eight with a polynomial on the FMA pipe (ptx::exp2_poly, coefficients from
csrc/kernels/fit_exp2_poly.py). Both are checked here through sa_debug_exp2.
"""

import numpy as np
import pytest
import torch

import block_causal_streaming_sa_b200 as sa

pytestmark = pytest.mark.gpu


def _run(poly, x):
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    sa.sa_debug_exp2(poly, xd.data_ptr(), yd.data_ptr(), xd.numel(),
                     torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return yd.cpu().numpy().astype(np.float64)


def test_polynomial_exp2_error_bound():
    # the softmax range: x = s*scale*log2e - m <= 8 (running max kept within 2^8)
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001),
                        np.arange(-125, 9).astype(np.float64) + 0.5,
                        np.arange(-125, 9).astype(np.float64)]).astype(np.float32)
    y = _run(True, x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() <= 1e-4, rel.max()
    # CUDA's exp2f (torch.exp2 on the device) agrees to the same bound
    cuda = torch.exp2(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    assert (np.abs(y - cuda) / cuda).max() <= 1.1e-4


def test_polynomial_exp2_clamps_below_range():
    x = np.array([-126.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    y = _run(True, x)
    assert np.all(y > 0) and np.all(y <= 2.0 ** -124.5)


def test_exp_unit_matches_exp2f():
    x = np.linspace(-100.0, 8.0, 1_000_001).astype(np.float32)
    y = _run(False, x)
    cuda = torch.exp2(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    assert (np.abs(y - cuda) / cuda).max() <= 1e-6
    assert _run(False, np.array([-np.inf], dtype=np.float32))[0] == 0.0

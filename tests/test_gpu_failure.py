"""Failure detection on the GPU without a GPU fault.

A test hook switches off the attention kernel's TMA producer, so a bounded
mbarrier wait of the MMA warp runs out (nothing ever arrives). The kernel must
finish by itself, report SA_ERR_TIMEOUT through the device status word, and
leave the context usable: the next normal call on the same handle is correct.
"""

import time

import pytest
import torch

import block_causal_streaming_sa_b200 as sa
from harness import Pair, check_output
from sa_inputs import WORKLOADS

pytestmark = pytest.mark.gpu


def test_stalled_wait_times_out_and_context_recovers():
    w = WORKLOADS["tiny"]
    pair = Pair(w)
    for _ in range(3):
        pair.append()
    Q, Kc, Vc = (t.cuda() for t in pair.tensors(("Q", "Kc", "Vc")))
    out = torch.empty_like(Q)
    t0 = time.time()
    sa.sa_debug_attend_stalled(pair.gpu.handle, Q.data_ptr(), Kc.data_ptr(), Vc.data_ptr(), True,
                               out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    status = pair.gpu.status()
    elapsed = time.time() - t0
    assert status == sa.SA_ERR_TIMEOUT
    assert elapsed < 30.0, elapsed
    # the status word stays set until reset; nothing else is broken
    assert pair.gpu.status() == sa.SA_ERR_TIMEOUT
    torch.cuda.synchronize()
    # a normal call on the same handle (and stream) is still correct
    o_gpu, o_ref, _, _ = pair.attend(0, True)
    check_output(o_gpu, o_ref, "after timeout")


def test_reset_clears_the_status_word_and_the_stream():
    w = WORKLOADS["tiny"]
    h = sa.StreamingAttention(w.config_dict())
    Q, Kc, Vc = (w.tensor(n, 0).cuda() for n in ("Q", "Kc", "Vc"))
    sa.sa_debug_attend_stalled(h.handle, Q.data_ptr(), Kc.data_ptr(), Vc.data_ptr(), False,
                               torch.empty_like(Q).data_ptr(),
                               torch.cuda.current_stream().cuda_stream)
    assert h.status() == sa.SA_ERR_TIMEOUT
    h.reset()
    assert h.status() == sa.SA_OK and h.chunk_count(sa.SA_TIER_NOISY) == 0
    h.attend(Q, Kc, Vc, False)
    assert h.status() == sa.SA_OK

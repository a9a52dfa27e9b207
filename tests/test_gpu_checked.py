"""The checked build (libsa_checked.so: the same sources compiled with device-side
bounds checks on every direct global load and store of the attention path's
kernels) runs a cross-section of the GPU parity tests in a process of its own:
every test still matches the oracle and ends with a clean status word, i.e. no
kernel reached past the end of a buffer (a reach would have been skipped and
reported as SA_ERR_BOUNDS)."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SUBSET = [
    "tests/test_gpu_parity.py::test_tiny_stream_every_chunk_and_step",
    "tests/test_gpu_parity.py::test_edge_shapes_and_windows",
    "tests/test_gpu_parity.py::test_state_errors",
    "tests/test_gpu_sparse.py::test_random_masks_every_chunk",
    "tests/test_gpu_sparse.py::test_structured_masks_skip_chunks_and_partner_tiles",
    "tests/test_gpu_sparse.py::test_rows_of_more_than_64_key_tiles",
    "tests/test_gpu_editing.py::test_every_chunk_and_step_with_variable_frames",
    "tests/test_gpu_prefix.py::test_variable_frames_with_reference_every_step",
    "tests/test_gpu_prefix.py::test_noalloc_and_simt_with_reference",
    "tests/test_gpu_fuzz.py",
]


def _env():
    return dict(os.environ, SA_LIBRARY="checked")


def test_checked_library_is_the_one_loaded():
    code = ("import block_causal_streaming_sa_b200 as sa; "
            "assert sa.sa_build_info() & sa.SA_BUILD_DEVICE_CHECKS; "
            "assert sa._binding.LIB_PATH.endswith('libsa_checked.so')")
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=_env(),
                         capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]


def test_parity_cross_section_on_the_checked_build():
    res = subprocess.run([sys.executable, "-m", "pytest", *SUBSET, "-m", "gpu", "-q", "-x",
                          "-p", "no:cacheprovider"],
                         cwd=ROOT, env=_env(), capture_output=True, text=True, timeout=1800)
    assert res.returncode == 0, res.stdout[-4000:] + res.stderr[-2000:]
    assert " passed" in res.stdout

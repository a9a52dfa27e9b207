"""The seeded input generator: deterministic, standard normal, shaped as asked."""

import numpy as np
import torch

from sa_inputs import WORKLOADS, normal_bf16, normals, seed_of, uniforms


def test_splitmix64_reference_values():
    # splitmix64 seeded with 0: published first outputs of the generator
    # (Steele, Lea, Flood 2014; also the seeding routine of xoshiro256).
    z = uniforms(0, 0, 3) * (1 << 53)
    first = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    assert [int(v) for v in z] == [f >> 11 for f in first]


def test_normals_moments_and_determinism():
    a = normals(7, 200000)
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1.0) < 0.01
    np.testing.assert_array_equal(a[:1000], normals(7, 1000))
    assert not np.array_equal(a[:1000], normals(8, 1000))


def test_normal_bf16_outliers_and_scale():
    t = normal_bf16(seed_of("x"), (64, 1000), scale=0.5, outlier_frac=0.01, outlier_mag=8.0)
    assert t.dtype == torch.bfloat16 and t.shape == (64, 1000)
    v = t.float().numpy()
    share = np.mean(np.abs(v) == 8.0)
    assert 0.007 < share < 0.013
    inl = v[np.abs(v) != 8.0]
    assert abs(inl.std() - 0.5) < 0.02


def test_workload_shapes():
    w = WORKLOADS["refiner_720p"]
    assert w.chunk_len == 10800 and w.kv_len == 43200
    assert WORKLOADS["s1_540p"].kv_len == 24480
    assert WORKLOADS["long_stream_stress"].kv_len == 64800
    assert WORKLOADS["tiny"].chunk_len == 192 and WORKLOADS["tiny"].kv_len == 576
    t = WORKLOADS["tiny"].tensor("Q", chunk=0)
    assert tuple(t.shape) == (1, 192, 2, 64)
    assert torch.equal(t, WORKLOADS["tiny"].tensor("Q", chunk=0))


def test_tensor_slices_equal_the_whole_tensor():
    """tensor_at draws exactly the (batch, head) slices of the full tensor,
    outliers and the K scale included (the generator is counter-based)."""
    from sa_inputs import Workload

    w = Workload("slices", 3, 5, 64, 2, 6, 7, sink=1, window=2, steps=1, stream=2,
                 k_scale=0.5, outlier_frac=0.02)
    for name in ("Q", "Kn"):
        full = w.tensor(name, 4, 1, 2)
        part = w.tensor_at(name, 4, 1, 2, batches=[0, 2], heads=[1, 4])
        assert torch.equal(part, full[[0, 2]][:, :, [1, 4]])
    assert torch.equal(w.tensor_at("Vc", 0), w.tensor("Vc", 0))

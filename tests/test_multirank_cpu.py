"""The multi-rank host path of bench.py on CPU: two gloo ranks.

bench.py under torchrun runs one independent stream per rank (weak scaling);
its only collectives are a barrier around the timed region and a max over
ranks of each reported time. These tests drive that exact code (bench.Ranks,
bench.whole_job_tflops) with world size 2 on the gloo backend, and check that
the reference arm does its work on rank 0 only.
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench

    ranks = bench.Ranks("gloo", "cpu", timeout_s=60)
    ranks.barrier()
    local_ms = 10.0 * (rank + 1)          # rank 1 is the slow one
    ms_max = ranks.max(local_ms)
    value = bench.whole_job_tflops(2e12, ms_max, ranks.world)
    ranks.barrier()
    ranks.close()
    out.put((rank, ms_max, value))


def test_two_rank_barrier_max_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # both ranks see the slowest rank's time; value = work of both ranks / that time
    assert [r[1] for r in res] == [20.0, 20.0]
    assert res[0][2] == pytest.approx(2 * 2e12 / 20e-3 / 1e12)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_on_rank_zero():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "1"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


@pytest.mark.parametrize("flags, key, mode", [
    (["--sparsity", "0.5"], "block_sparsity", "block-sparse"),
    (["--editing"], "frame_aligned_editing", "frame-aligned editing"),
    (["--ref-frames", "1"], "ref_frames", "1-frame reference"),
])
def test_reference_arm_times_the_oracle_of_the_named_mode(flags, key, mode):
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "0", *flags], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["config"][key] and mode in line["cpu_baseline"]["sample"] and line["value"] > 0


def test_oracle_sample_flops_follow_the_mode():
    """FLOPs of a sampled call: 4 D x (keys each sampled row sees), as the GPU arm counts."""
    import numpy as np

    import bench
    from sa_inputs import WORKLOADS

    w = WORKLOADS["tiny"]
    hw = w.tok_h * w.tok_w
    assert bench.OracleSample(w).run(8) == 4.0 * 8 * w.kv_len * w.head_dim
    assert bench.OracleSample(w, ref_frames=2).run(8) == 4.0 * 8 * (w.kv_len + 2 * hw) * w.head_dim
    assert bench.OracleSample(w, editing=True).run(8) == 4.0 * 8 * (w.kv_len + hw) * w.head_dim
    o = bench.OracleSample(w, sparsity=0.5)
    o.rng = np.random.default_rng(0)
    sel = np.random.default_rng(0).choice(w.chunk_len, size=8, replace=False)
    nq = -(-w.chunk_len // 128)
    tile = np.array([128, w.chunk_len - 128] * (w.sink + w.window))
    keys = sum(int((o.mask[0, 0, q // 128] * tile).sum()) for q in sel)
    assert o.run(8) == 4.0 * w.head_dim * keys and nq == 2


@pytest.mark.parametrize("flags, why", [
    (["--sparsity", "0.9", "--ulysses"], "different workloads"),
    (["--editing", "--sparsity", "0.5"], "different workloads"),
    (["--sparsity", "0.9", "--ref-frames", "1"], "no reference image"),
    (["--sparsity", "1.0"], "must be in [0, 1)"),
])
def test_bench_refuses_mixed_workload_flags(flags, why):
    """A mode flag the timed loop would ignore must not reach the FLOP count."""
    r = subprocess.run([sys.executable, "bench.py", *flags], cwd=ROOT, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 2 and why in r.stderr, r.stderr


def _a2a_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    from block_causal_streaming_sa_b200.ulysses import all_to_all_blocks

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    nbytes = 24
    # block g of rank r holds the byte pattern (r, g, i)
    send = torch.tensor([(rank * 16 + g) * 3 + i % 3 for g in range(world) for i in range(nbytes)],
                        dtype=torch.int64).to(torch.uint8)
    recv = all_to_all_blocks(send)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, recv.tolist()))


@pytest.mark.parametrize("world", [2, 3])
def test_ulysses_block_all_to_all_on_gloo(world):
    """The exchange primitive of the Ulysses layer: block s of rank r's result is
    block r of rank s's send buffer (the layout sa_exchange_unpack expects)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_a2a_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    nbytes = 24
    for r in range(world):
        want = [((s * 16 + r) * 3 + i % 3) % 256 for s in range(world) for i in range(nbytes)]
        assert res[r] == want, r

"""The peer-memory transport of the Ulysses layer (sa_exchange_pack_to + CUDA IPC).

Two processes share one GPU: each maps the other's receive buffers with CUDA
IPC and quantises its token shard straight into them. They synchronise on the
host (stream synchronise + a gloo barrier), so no kernel waits for the other
process. Each rank checks what it received against the oracle, bit-exact, and
its attention against the oracle on those inputs.
"""

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

CFG = dict(batch=1, heads=4, head_dim=128, frames_per_chunk=2, tok_h=8, tok_w=12,
           sink_chunks=1, window_chunks=2, ref_frames=1)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _full(tag, tokens):
    from sa_inputs import normal_bf16, seed_of

    return normal_bf16(seed_of("p2p", tag), (CFG["batch"], tokens, CFG["heads"], CFG["head_dim"]))


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    try:
        import torch.distributed as dist

        import block_causal_streaming_sa_b200 as sa
        from block_causal_streaming_sa_b200.ulysses import UlyssesAttention
        from harness import check_output, f64
        from oracle import exchange as ex
        from oracle.stream import CLEAN, NOISY, OracleConfig, StreamOracle

        torch.cuda.set_device(0)
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world, timeout=datetime.timedelta(seconds=120))
        uly = UlyssesAttention(CFG, transport="p2p")
        G, L, hw = world, CFG["frames_per_chunk"] * 96, 96
        hl = CFG["heads"] // G
        orc = StreamOracle(OracleConfig(1, hl, 128, 2, 8, 12, 1, 2, ref_frames=1))

        def shard(x, n):
            return x[:, rank * n // G:(rank + 1) * n // G].contiguous()

        def received(x, n):  # what rank `rank` holds after the exchange, by the oracle
            parts = [f64(x[:, s * n // G:(s + 1) * n // G]) for s in range(G)]
            return ex.tokens_to_heads(parts)[rank]

        Kr, Vr = _full("Kref", hw), _full("Vref", hw)
        uly.set_reference(shard(Kr, hw).cuda(), shard(Vr, hw).cuda())
        orc.set_reference(received(Kr, hw), received(Vr, hw))
        checks = 0
        for c in range(3):
            Q, Kc, Vc = (_full((n, c), L) for n in ("Q", "Kc", "Vc"))
            got = uly.to_heads(shard(Q, L).cuda())
            torch.cuda.synchronize()
            np.testing.assert_array_equal(f64(got.cpu()), received(Q, L))
            o = uly.local.attend(got, uly.to_heads(shard(Kc, L).cuda()),
                                 uly.to_heads(shard(Vc, L).cuda()), True)
            back = uly.to_tokens(o)
            torch.cuda.synchronize()
            o_ref, _ = orc.attend(received(Q, L), received(Kc, L), received(Vc, L), True)
            check_output(f64(o.cpu()), o_ref, f"rank {rank} chunk {c}")
            every = [None] * G
            dist.all_gather_object(every, f64(o.cpu()))
            np.testing.assert_array_equal(f64(back.cpu()), ex.heads_to_tokens(every)[rank])
            for tier in (NOISY, CLEAN):
                K, V = _full(("K", c, tier), L), _full(("V", c, tier), L)
                uly.append(tier, shard(K, L).cuda(), shard(V, L).cuda())
                orc.append(tier, received(K, L), received(V, L))
            checks += 1
        assert uly.status() == sa.SA_OK
        uly.close()
        dist.barrier()
        dist.destroy_process_group()
        out.put((rank, "ok", checks))
    except Exception as e:  # report instead of hanging the parent
        import traceback

        out.put((rank, "error", traceback.format_exc()[-3000:]))


def test_two_processes_one_gpu_peer_exchange():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=600) for _ in procs]
    for p in procs:
        p.join(timeout=120)
    for rank, status, info in res:
        assert status == "ok", f"rank {rank}:\n{info}"
        assert info == 3
    assert all(p.exitcode == 0 for p in procs)


def test_single_rank_peer_transport_equals_nccl_transport():
    sys.path.insert(0, ROOT)
    from block_causal_streaming_sa_b200.ulysses import UlyssesAttention

    a = UlyssesAttention(CFG, transport="p2p")
    b = UlyssesAttention(CFG, transport="nccl")
    L = 2 * 96
    for c in range(2):
        Q, Kc, Vc = (_full(("one", n, c), L).cuda() for n in ("Q", "Kc", "Vc"))
        assert torch.equal(a.attend(Q, Kc, Vc, False), b.attend(Q, Kc, Vc, False))
        for tier in (0, 1):
            K, V = (_full(("oneKV", n, c, tier), L).cuda() for n in "KV")
            a.append(tier, K, V)
            b.append(tier, K, V)
    a.close()
    b.close()

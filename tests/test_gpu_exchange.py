"""Ulysses exchange kernels (sa_exchange_pack / sa_exchange_unpack) and the head-
sharded attention on one GPU, against the oracle.

G ranks are emulated on one device: each virtual rank packs its shard with the
library, the all-to-all is a plain reassembly of the byte blocks (block r of
sender s becomes block s of receiver r), and each rank unpacks with the
library. No kernel waits for another rank.
"""

import numpy as np
import pytest
import torch

import block_causal_streaming_sa_b200 as sa
from block_causal_streaming_sa_b200.ulysses import UlyssesAttention
from harness import TOL, check_output, f64
from oracle import exchange as ex
from oracle.stream import CLEAN, NOISY, OracleConfig, StreamOracle
from sa_inputs import normal_bf16, seed_of

pytestmark = pytest.mark.gpu
P8, P16 = sa.SA_PAYLOAD_FP8, sa.SA_PAYLOAD_BF16


def _pack(x, G, split, payload):
    b, t, c, d = x.shape
    n = sa.sa_exchange_block_bytes(b, t, c, d, G, split, payload)
    buf = torch.empty(G * n, dtype=torch.uint8, device="cuda")
    sa.sa_exchange_pack(x.data_ptr(), b, t, c, d, G, split, payload, buf.data_ptr())
    return buf.view(G, n)


def _unpack(blocks, shape, G, split, payload):
    b, t, c, d = shape
    recv = blocks.contiguous()
    out_shape = (b, G * t, c // G, d) if split == 1 else (b, t // G, G * c, d)
    y = torch.empty(out_shape, dtype=torch.bfloat16, device="cuda")
    sa.sa_exchange_unpack(recv.data_ptr(), b, t, c, d, G, split, payload, y.data_ptr())
    return y


def _exchange(shards, G, split, payload):
    """Emulated all-to-all over G virtual ranks: returns each rank's unpacked tensor."""
    sent = [_pack(x, G, split, payload) for x in shards]
    return [_unpack(torch.stack([sent[s][r] for s in range(G)]), shards[0].shape, G, split,
                    payload) for r in range(G)]


def _input(tag, shape, outliers=0.0):
    x = normal_bf16(seed_of("exchange-gpu", tag), shape, outlier_frac=outliers)
    return x


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("split", [0, 1])
@pytest.mark.parametrize("G", [1, 2, 3, 4])
def test_pack_codes_and_scales_bit_exact(D, split, G):
    shape = (2, 12, 12, D) if split == 1 else (2, 12 * G, 5, D)
    x = _input(("pack", D, split, G), shape, outliers=0.02)
    x[0, 0, 0] = 0.0                      # all-zero vector: scale 0, codes 0
    x[1, 2, 3, :5] = -0.0                 # signed zeros keep their sign
    buf = _pack(x.cuda(), G, split, P8).cpu().numpy()
    xs = x.float().numpy()
    b, t, c, d = shape
    for g in range(G):
        part = xs[:, :, g * c // G:(g + 1) * c // G] if split == 1 else \
            xs[:, g * t // G:(g + 1) * t // G]
        codes, scales = ex.quantize(part)
        n_vec = codes.size // D
        blk = buf[g]
        np.testing.assert_array_equal(blk[:n_vec * D], codes.reshape(-1), err_msg=f"codes {g}")
        off = -(-n_vec * D // 16) * 16
        got = blk[off:off + 4 * n_vec].view(np.float32)
        np.testing.assert_array_equal(got, scales.reshape(-1), err_msg=f"scales {g}")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("payload", [P8, P16])
def test_both_exchanges_match_the_oracle_bit_exact(D, G, payload):
    B, L, H = 2, 8 * G, 4 * G
    full = _input(("round", D, G, payload), (B, L, H, D), outliers=0.01)
    shards = [full[:, s * L // G:(s + 1) * L // G].contiguous() for s in range(G)]
    quant = payload == P8
    heads = _exchange([s.cuda() for s in shards], G, 1, payload)
    want = ex.tokens_to_heads([f64(s) for s in shards], quantised=quant)
    for r in range(G):
        np.testing.assert_array_equal(f64(heads[r].cpu()), want[r])
    back = _exchange(heads, G, 0, payload)
    want_back = ex.heads_to_tokens([f64(h.cpu()) for h in heads], quantised=quant)
    for s in range(G):
        np.testing.assert_array_equal(f64(back[s].cpu()), want_back[s])


@pytest.mark.parametrize("G", [2, 4])
@pytest.mark.parametrize("payload", [P8, P16])
def test_head_sharded_attention_over_a_stream(G, payload):
    """G virtual ranks, each with its own H/G-head cache, over a 5-chunk stream:
    every rank's attention matches the oracle on the tensors it received, and the
    output exchange matches the oracle's quantisation of those outputs."""
    B, H, D, F, th, tw, S, W = 1, 4 * G // 2 * 2, 128, 2, 8, 12, 1, 3
    L = F * th * tw
    cfg = dict(batch=B, heads=H // G, head_dim=D, frames_per_chunk=F, tok_h=th, tok_w=tw,
               sink_chunks=S, window_chunks=W)
    ranks = [sa.StreamingAttention(cfg) for _ in range(G)]
    oracles = [StreamOracle(OracleConfig(B, H // G, D, F, th, tw, S, W)) for _ in range(G)]
    quant = payload == P8

    def scatter(tag):
        full = _input(tag, (B, L, H, D))
        shards = [full[:, s * L // G:(s + 1) * L // G].contiguous() for s in range(G)]
        got = _exchange([x.cuda() for x in shards], G, 1, payload)
        return got, ex.tokens_to_heads([f64(x) for x in shards], quantised=quant)

    for c in range(5):
        for k, final in enumerate((False, True)):
            (q, q_o), (kc, kc_o), (vc, vc_o) = (scatter((n, c, k)) for n in ("Q", "Kc", "Vc"))
            outs = []
            for r in range(G):
                o = ranks[r].attend(q[r], kc[r], vc[r], final)
                torch.cuda.synchronize()
                o_ref, _ = oracles[r].attend(q_o[r], kc_o[r], vc_o[r], final)
                check_output(f64(o.cpu()), o_ref, f"rank {r} chunk {c} step {k}")
                outs.append(o)
            back = _exchange(outs, G, 0, payload)
            want = ex.heads_to_tokens([f64(o.cpu()) for o in outs], quantised=quant)
            for s in range(G):
                np.testing.assert_array_equal(f64(back[s].cpu()), want[s])
        for tier in (NOISY, CLEAN):
            (kk, kk_o), (vv, vv_o) = scatter(("K", c, tier)), scatter(("V", c, tier))
            for r in range(G):
                ranks[r].append(tier, kk[r], vv[r])
                oracles[r].append(tier, kk_o[r], vv_o[r])
    for r in ranks:
        assert r.status() == sa.SA_OK


def test_ulysses_layer_single_rank_equals_local_attention_on_exchanged_inputs():
    """The Python layer with one rank: quantise-dequantise in, attention, and
    quantise-dequantise out, bit-identical to the same kernels called by hand."""
    cfg = dict(batch=1, heads=4, head_dim=128, frames_per_chunk=2, tok_h=8, tok_w=8,
               sink_chunks=1, window_chunks=2, ref_frames=1)
    uly = UlyssesAttention(cfg, payload="fp8")
    ref = sa.StreamingAttention(cfg)
    L = 2 * 64
    rt = lambda x: _exchange([x], 1, 1, P8)[0]  # noqa: E731  (one-rank round trip)
    Kr, Vr = (_input(("ref", n), (1, 64, 4, 128)).cuda() for n in "KV")
    uly.set_reference(Kr, Vr)
    ref.set_reference(rt(Kr), rt(Vr))
    for c in range(3):
        Q, Kc, Vc = (_input((n, c), (1, L, 4, 128)).cuda() for n in ("Q", "Kc", "Vc"))
        a = uly.attend(Q, Kc, Vc, True)
        b = _exchange([ref.attend(rt(Q), rt(Kc), rt(Vc), True)], 1, 0, P8)[0]
        torch.cuda.synchronize()
        assert torch.equal(a, b), c
        for tier in (NOISY, CLEAN):
            K, V = (_input((n, c, tier), (1, L, 4, 128)).cuda() for n in "KV")
            uly.append(tier, K, V)
            ref.append(tier, rt(K), rt(V))
    assert uly.status() == sa.SA_OK


def test_quantised_exchange_error_against_unquantised_attention():
    """The fp8 payload costs accuracy (3 mantissa bits on Q, K, V and O); report
    it against attention on the exact inputs and keep it bounded."""
    G, B, H, D, F, th, tw = 2, 1, 4, 128, 2, 8, 12
    L = F * th * tw
    cfg = dict(batch=B, heads=H // G, head_dim=D, frames_per_chunk=F, tok_h=th, tok_w=tw,
               sink_chunks=0, window_chunks=1)
    ranks = [sa.StreamingAttention(cfg) for _ in range(G)]
    full = {n: _input(("err", n), (B, L, H, D)) for n in ("Q", "Kc", "Vc")}
    moved = {n: _exchange([t[:, s * L // G:(s + 1) * L // G].contiguous().cuda()
                           for s in range(G)], G, 1, P8) for n, t in full.items()}
    outs = [ranks[r].attend(moved["Q"][r], moved["Kc"][r], moved["Vc"][r], True) for r in range(G)]
    back = torch.cat(_exchange(outs, G, 0, P8), dim=1)
    orc = StreamOracle(OracleConfig(B, H, D, F, th, tw, 0, 1))
    exact, _ = orc.attend(*(f64(full[n]) for n in ("Q", "Kc", "Vc")), True)
    err = np.abs(f64(back.cpu()) - exact).max()
    assert err < 0.1, err           # fp8 e4m3 quantisation, not a kernel tolerance
    assert err > TOL / 10           # the payload is really quantised

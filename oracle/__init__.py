"""Plain CPU oracle for block-causal sink + window TwinCache attention.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it. It shares no code with the
CUDA library under ``block_causal_streaming_sa_b200/``.

Everything is computed in float64 with numpy, with no blocking, fusion or
reordering beyond the plain definitions, so that each step can be checked
against the pages by eye.

Sources (web pages, cited by title and section):
  [orkas] "Vidu S2 vs PixVerse R2：实时视频的两条技术路线" (orkas.ai blog)
          - section 「实时」改变了什么: video is cut into chunks generated in order;
            a chunk sees what came before it and never what comes after.
          - section 选择三：有上限的记忆: the first chunks are kept forever as
            anchors (sink), a sliding window of the most recent chunks is kept,
            the rest is discarded; temporal positions are relocated so they
            stay inside the trained range; TwinCache keeps a noisy and a clean
            copy of every history chunk, intermediate denoising steps read the
            noisy one and the final step reads the clean one.
  [s2read] "Vidu S2：实时可交互、可编辑、可立体的视频生成" (paper read of Vidu S2)
          - abbreviation table: KV cache = stored keys/values of history tokens;
            RoPE encodes each token's position in space and in time.
          - section 2.2: block-wise causal mask; anchor chunks, sliding-window
            context and a noisy KV cache.
  [bloom] "Vidu S2：实时数字人、实时视频编辑都做到了，空间视频还只是探索"
          - section "Vidu S2 到底是什么": temporal attention becomes a block-wise
            causal mask; sliding-window context plus a rolling KV cache keep
            memory bounded.

Readings where the pages are silent (the prefix, variable-length, editing and
exchange readings R13-R16 are stated in stream.py, editing.py and exchange.py):
  R1  the window W counts the current chunk: keys = (S + W) * L.
  R2  inside a chunk attention is bidirectional.
  R3  relocated temporal position of frame f of chunk j is rank(j) * F + f,
      rank = index of j in the ascending attended list.
  R4  3D RoPE bands [t | h | w] of sizes D - 4*(D//6), 2*(D//6), 2*(D//6);
      interleaved pairs (2i, 2i+1); angle pos * theta**(-2i / d_band);
      theta = 10000.
  R5  softmax scale 1/sqrt(D); token order in a chunk is frame, row, column.
  R6  sink chunks have both tiers; the tier selector applies to every cached
      chunk; the current chunk's K/V are passed with the query.
"""

from .rope import band_sizes, rotate, token_positions
from .cache import RingCacheModel
from .attention import softmax_attention
from .stream import StreamOracle, OracleConfig, masked_full_attention

__all__ = [
    "band_sizes",
    "rotate",
    "token_positions",
    "RingCacheModel",
    "softmax_attention",
    "StreamOracle",
    "OracleConfig",
    "masked_full_attention",
]

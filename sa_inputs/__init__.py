"""Seeded synthetic inputs and workload shapes, shared by tests and the bench.

This module holds no arithmetic of the attention method: it only draws random
numbers and names the workload shapes. Both the CUDA path and the oracle are
fed from it; neither imports the other.

Generator: counter-based splitmix64 (Steele, Lea, Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014): draw i of a stream with seed s is
mix(s + (i + 1) * 0x9E3779B97F4A7C15). Two 53-bit uniforms per element feed
the Box-Muller transform, n = sqrt(-2 ln(1 - u1)) * cos(2 pi u2). Values are
drawn in float64, rounded to float32, then to bfloat16 (round to nearest even).
Element order is the C order of the requested shape, so a tensor is a pure
function of (seed, shape) and can be re-drawn anywhere.
"""

import hashlib
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
import torch

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_BLOCK = 1 << 22


def _mix(z):
    z = z ^ (z >> np.uint64(30))
    z = z * _M1
    z = z ^ (z >> np.uint64(27))
    z = z * _M2
    return z ^ (z >> np.uint64(31))


def uniforms(seed, start, count):
    """Draws start..start+count-1 of stream ``seed`` as float64 in [0, 1)."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = _mix(np.uint64(seed) + idx * _GAMMA)
    return (z >> np.uint64(11)).astype(np.float64) * (1.0 / (1 << 53))


_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1))
    return _POOL


def _blocks(count, fn):
    """Run fn(start, n) over blocks of the index range (threads; numpy drops the GIL)."""
    starts = range(0, count, _BLOCK)
    if count <= _BLOCK:
        for s in starts:
            fn(s, min(_BLOCK, count - s))
        return
    list(_pool().map(lambda s: fn(s, min(_BLOCK, count - s)), starts))


def normals(seed, count):
    """``count`` standard normal float64 values of stream ``seed``."""
    out = np.empty(count, dtype=np.float64)

    def fill(s, n):
        u = uniforms(seed, 2 * s, 2 * n)
        out[s:s + n] = np.sqrt(-2.0 * np.log1p(-u[0::2])) * np.cos(2.0 * np.pi * u[1::2])

    _blocks(count, fill)
    return out


def _uniform_at(seed, pos):
    """Draw ``pos`` (int64 array of stream positions) of stream ``seed``, as
    ``uniforms`` would give it."""
    with np.errstate(over="ignore"):
        z = _mix(np.uint64(seed) + (pos.astype(np.uint64) + np.uint64(1)) * _GAMMA)
    return (z >> np.uint64(11)).astype(np.float64) * (1.0 / (1 << 53))


def seed_of(*fields):
    """Stable 64-bit seed of a tuple of names and numbers."""
    key = "|".join(str(f) for f in fields).encode()
    return int.from_bytes(hashlib.blake2b(key, digest_size=8).digest(), "little")


def normal_bf16(seed, shape, scale=1.0, outlier_frac=0.0, outlier_mag=8.0):
    """bf16 CPU tensor of N(0, scale^2) values; optionally a Bernoulli
    ``outlier_frac`` share of elements replaced by +-``outlier_mag``."""
    count = int(np.prod(shape))
    vals = normals(seed, count)
    out = np.empty(count, dtype=np.float32)
    s_pick, s_sign = seed_of(seed, "outlier"), seed_of(seed, "sign")

    def fill(s, n):
        v = vals[s:s + n] * scale
        if outlier_frac > 0.0:
            pick = uniforms(s_pick, s, n) < outlier_frac
            sign = np.where(uniforms(s_sign, s, n) < 0.5, -1.0, 1.0)
            v = np.where(pick, sign * outlier_mag, v)
        out[s:s + n] = v

    _blocks(count, fill)
    return torch.from_numpy(out.reshape(shape)).to(torch.bfloat16)


def normal_bf16_at(seed, index, scale=1.0, outlier_frac=0.0, outlier_mag=8.0):
    """The elements at flat C-order positions ``index`` (int64 array, any shape)
    of ``normal_bf16(seed, shape, ...)``, as a bf16 CPU tensor of index's shape:
    the generator is counter-based, so element i depends only on (seed, i) and a
    slice of a large tensor can be drawn without drawing the rest."""
    i = np.asarray(index, dtype=np.int64).reshape(-1)
    u1, u2 = _uniform_at(seed, 2 * i), _uniform_at(seed, 2 * i + 1)
    v = np.sqrt(-2.0 * np.log1p(-u1)) * np.cos(2.0 * np.pi * u2) * scale
    if outlier_frac > 0.0:
        pick = _uniform_at(seed_of(seed, "outlier"), i) < outlier_frac
        sign = np.where(_uniform_at(seed_of(seed, "sign"), i) < 0.5, -1.0, 1.0)
        v = np.where(pick, sign * outlier_mag, v)
    out = v.astype(np.float32).reshape(np.shape(index))
    return torch.from_numpy(out).to(torch.bfloat16)


def device_normal_bf16(seed, shape, device):
    """N(0, 1) bf16 tensor made on `device` by torch's seeded generator of that
    device, for inputs too large to draw on the host (tens of GB). Deterministic
    for a given seed, shape and device type; slices of it are copied to the host
    where a check needs them."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


@dataclass(frozen=True)
class Workload:
    """Shape of one synthetic workload (all tensors [B, L, H, D] bf16)."""

    name: str
    batch: int
    heads: int
    head_dim: int
    frames: int
    tok_h: int
    tok_w: int
    sink: int
    window: int          # counts the chunk being generated
    steps: int           # denoising steps per chunk; the last reads the clean tier
    stream: int          # chunks in the stream used for parity / eviction runs
    layers: int = 1
    k_scale: float = 1.0
    outlier_frac: float = 0.0
    outlier_mag: float = 8.0
    notes: str = field(default="", compare=False)

    @property
    def chunk_len(self):
        return self.frames * self.tok_h * self.tok_w

    @property
    def kv_len(self):
        return (self.sink + self.window) * self.chunk_len

    def shape(self):
        return (self.batch, self.chunk_len, self.heads, self.head_dim)

    def tensor(self, name, chunk, step=0, layer=0):
        """Seeded tensor ``name`` of one chunk / step / layer.

        Names: Q, Kc, Vc (current chunk at a denoising step), Kn, Vn (noisy
        tier copy appended after the chunk), Kcl, Vcl (clean tier copy).
        """
        scale = self.k_scale if name.startswith("K") else 1.0
        return normal_bf16(seed_of(self.name, layer, chunk, step, name), self.shape(),
                           scale=scale, outlier_frac=self.outlier_frac,
                           outlier_mag=self.outlier_mag)

    def tensor_at(self, name, chunk, step=0, layer=0, batches=None, heads=None):
        """The (batch, head) slices ``tensor(...)[batches][:, :, heads]`` of a
        seeded tensor, [nb, L, nh, D], drawn without drawing the whole tensor."""
        b = np.arange(self.batch) if batches is None else np.asarray(batches)
        h = np.arange(self.heads) if heads is None else np.asarray(heads)
        L, H, D = self.chunk_len, self.heads, self.head_dim
        idx = (((b[:, None, None, None] * L + np.arange(L)[None, :, None, None]) * H
                + h[None, None, :, None]) * D + np.arange(D)[None, None, None, :])
        scale = self.k_scale if name.startswith("K") else 1.0
        return normal_bf16_at(seed_of(self.name, layer, chunk, step, name), idx, scale=scale,
                              outlier_frac=self.outlier_frac, outlier_mag=self.outlier_mag)

    def config_dict(self):
        return dict(batch=self.batch, heads=self.heads, head_dim=self.head_dim,
                    frames_per_chunk=self.frames, tok_h=self.tok_h, tok_w=self.tok_w,
                    sink_chunks=self.sink, window_chunks=self.window)


WORKLOADS = {
    w.name: w
    for w in (
        Workload("tiny", 1, 2, 64, 3, 8, 8, sink=1, window=2, steps=2, stream=6,
                 notes="oracle-sized case"),
        Workload("s1_540p", 1, 12, 128, 3, 34, 60, sink=1, window=3, steps=4, stream=6,
                 notes="540p latent chunk, 6120 tokens"),
        Workload("refiner_720p", 1, 12, 128, 3, 45, 80, sink=1, window=3, steps=1, stream=6,
                 notes="720p refiner, single clean-tier step"),
        Workload("backbone_540p_large", 1, 40, 128, 3, 34, 60, sink=1, window=3, steps=4,
                 stream=32, layers=40, k_scale=0.5, notes="40 layers per step"),
        Workload("long_stream_stress", 4, 24, 128, 3, 45, 80, sink=2, window=4, steps=4,
                 stream=200, outlier_frac=0.01, outlier_mag=8.0,
                 notes="3 noisy steps + 1 clean step per chunk, 1% outliers of +-8"),
    )
}

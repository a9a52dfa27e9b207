"""3D rotary position embedding, float64.  (Oracle: test infrastructure only.)

[s2read] abbreviation table: RoPE tells attention where each token sits in space
and in time, so every token carries a (t, h, w) position. The pages give no
formula; the reading used here (R4, R5 in the package docstring):

* the head vector is split into three consecutive bands [t | h | w] with sizes
  d_t = D - 4*(D//6), d_h = d_w = 2*(D//6)   (D=128: 44/42/42, D=64: 24/20/20);
* inside a band of size d, pair (2i, 2i+1) is turned by the angle
  pos * theta**(-2i/d), where pos is the token's coordinate on that band's axis:
      x'_{2i}   = x_{2i} cos(a) - x_{2i+1} sin(a)
      x'_{2i+1} = x_{2i} sin(a) + x_{2i+1} cos(a)
* a token with in-chunk index l has frame f = l // (H*W), row y = (l // W) % H,
  column x = l % W (frame-major, then row, then column).
"""

import numpy as np


def band_sizes(head_dim):
    """(d_t, d_h, d_w) for a head of size ``head_dim`` (reading R4)."""
    d_sp = 2 * (head_dim // 6)
    return head_dim - 2 * d_sp, d_sp, d_sp


def band_angles(pos, d_band, theta):
    """Angles pos * theta**(-2i/d_band) for i < d_band/2, shape [n, d_band/2]."""
    i = np.arange(d_band // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / d_band)
    return np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]


def token_positions(n_tokens, tok_h, tok_w):
    """(frame, row, column) of in-chunk token indices 0..n_tokens-1."""
    l = np.arange(n_tokens)
    return l // (tok_h * tok_w), (l // tok_w) % tok_h, l % tok_w


def rotate(x, pos_t, pos_h, pos_w, theta=10000.0):
    """Rotate the rows of ``x`` ([..., n, D], float64) by their 3D positions.

    ``pos_t``, ``pos_h``, ``pos_w`` are integer arrays of length n: the
    temporal, row and column coordinate of each row of ``x``.
    """
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    start = 0
    for d_band, pos in zip(band_sizes(x.shape[-1]), (pos_t, pos_h, pos_w)):
        ang = band_angles(pos, d_band, theta)
        c, s = np.cos(ang), np.sin(ang)
        even = x[..., start:start + d_band:2]
        odd = x[..., start + 1:start + d_band:2]
        out[..., start:start + d_band:2] = even * c - odd * s
        out[..., start + 1:start + d_band:2] = even * s + odd * c
        start += d_band
    return out

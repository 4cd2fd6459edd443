"""Rotary position embedding at striped position ids (oracle; test
infrastructure only).

The Striped review ("Striped Attention: Faster Ring Attention for Causal
Transformers", 位置编码处理) states that a position encoding such as RoPE has
to see the same stripe permutation as the tokens, and that the training
targets are permuted the same way.  The pages name RoPE but do not define
it.  Reading taken: the rotary embedding of RoFormer (Su et al., 2021) in its
usual parameterisation, applied to q and k at their ORIGINAL token positions:

    theta_i = base ** (-2 i / d),   i = 0 .. d/2 - 1
    (u, w)  ->  (u cos(pos theta_i) - w sin(pos theta_i),
                 u sin(pos theta_i) + w cos(pos theta_i))

where the pair (u, w) of rotation i is either the adjacent dimensions
(2i, 2i+1) ("interleaved", the RoFormer paper's layout) or the dimensions
(i, i + d/2) ("half", the split-halves layout many models use).

Applying it at original positions and then permuting into layout order is
the same as permuting the position ids with the stripe and applying it in
layout order; ``rope_partition`` states the former.
"""

import numpy as np

from . import partition as _partition

INTERLEAVED = "interleaved"
HALF = "half"


def frequencies(d, base):
    """theta_i = base^(-2i/d) for i = 0 .. d/2 - 1 (float64)."""
    if d % 2:
        raise ValueError("d must be even")
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d)


def pair_index(d, pairing):
    """(first, second) dimension index arrays of the d/2 rotation pairs."""
    i = np.arange(d // 2)
    if pairing == INTERLEAVED:
        return 2 * i, 2 * i + 1
    if pairing == HALF:
        return i, i + d // 2
    raise ValueError(pairing)


def rope(x, pos, base=10000.0, pairing=INTERLEAVED):
    """Rotate the rows of x ([..., n, d]) by their positions pos ([n])."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    pos = np.asarray(pos, dtype=np.float64)
    ang = pos[:, None] * frequencies(d, base)[None, :]        # [n, d/2]
    cos, sin = np.cos(ang), np.sin(ang)
    a, b = pair_index(d, pairing)
    u, w = x[..., a], x[..., b]
    out = np.empty_like(x)
    out[..., a] = u * cos - w * sin
    out[..., b] = u * sin + w * cos
    return out


def rope_partition(x, P, layout, base=10000.0, pairing=INTERLEAVED):
    """RoPE at original token positions 0..N-1, then the layout permutation
    (axis -2 is the token axis)."""
    N = x.shape[-2]
    return _partition.partition(rope(x, np.arange(N), base, pairing), P, layout)

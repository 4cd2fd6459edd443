"""Merging two partial attention results (oracle; test infrastructure only).

Source: 1cademy page "Computing Attention Weights in Sequence Parallelism":
the softmax denominator of query i is a sum of per-node partial sums,
sum_{all t} exp(b_it) = sum_u sum_{t in K^[u]} exp(b_it).

With each partial result given as (O_u, lse_u), where lse_u = ln of node u's
partial denominator and O_u its locally normalised output, the denominator
of the union is exp(lse_a) + exp(lse_b), and the union's output is the
partial outputs weighted by their share of that denominator:

    lse = ln(exp(lse_a) + exp(lse_b))
    O   = exp(lse_a - lse) O_a + exp(lse_b - lse) O_b

Reading for a side with no keys at all (lse = -inf): it contributes nothing;
if both sides are empty the result is O = 0, lse = -inf.
"""

import numpy as np


def lse_merge(o_a, lse_a, o_b, lse_b):
    o_a = np.asarray(o_a, dtype=np.float64)
    o_b = np.asarray(o_b, dtype=np.float64)
    lse_a = np.asarray(lse_a, dtype=np.float64)
    lse_b = np.asarray(lse_b, dtype=np.float64)
    with np.errstate(divide="ignore"):
        lse = np.logaddexp(lse_a, lse_b)
    both_empty = np.isneginf(lse)
    safe = np.where(both_empty, 0.0, lse)
    wa = np.where(both_empty, 0.0, np.exp(lse_a - safe))
    wb = np.where(both_empty, 0.0, np.exp(lse_b - safe))
    o = wa[..., None] * o_a + wb[..., None] * o_b
    return o, lse

"""The merged segment-list top-k the fused kernel uses (for topk <= 32) is
exact: under the strict order "larger score first, then lower chunk index"
(NaN ranking as -inf), the k best chunks of a pair are the first k of the
merge of every scoring segment's 32 best.  Checked here on the definition
itself, on random splits of random and heavily tied score arrays."""
import math

import numpy as np
import pytest

LIST = 32


def order_key(scores, i):
    """Sort key of chunk i: larger score first, ties (and NaN = -inf) to the
    lower index (the selection rule of sec. 3.3 "top-k chunks")."""
    s = scores[i]
    if math.isnan(s):
        s = -math.inf
    return (-s, i)


def topk_definition(scores, k):
    idx = sorted(range(len(scores)), key=lambda i: order_key(scores, i))
    return sorted(idx[:k])


def topk_merged(scores, k, cuts):
    """Each segment [cuts[t], cuts[t+1]) keeps its 32 best; the merge of the
    lists is ranked by the same key and cut to k."""
    kept = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        seg = sorted(range(a, b), key=lambda i: order_key(scores, i))
        kept.extend(seg[:LIST])
    kept.sort(key=lambda i: order_key(scores, i))
    return sorted(kept[:k])


def random_cuts(rng, n):
    m = int(rng.integers(1, 12))
    inner = sorted(set(int(x) for x in rng.integers(1, max(n, 2), size=m) if 0 < x < n))
    return [0] + inner + [n]


@pytest.mark.parametrize("levels", [0, 3, 1])
def test_merged_lists_equal_definition(levels):
    rng = np.random.default_rng(1234 + levels)
    for _ in range(300):
        n = int(rng.integers(1, 400))
        if levels:
            scores = rng.integers(0, levels, size=n).astype(np.float64)  # many ties
        else:
            scores = rng.standard_normal(n)
        if rng.random() < 0.2:
            scores[rng.integers(0, n)] = np.nan
        k = int(rng.integers(0, LIST + 1))
        cuts = random_cuts(rng, n)
        assert topk_merged(scores, k, cuts) == topk_definition(scores, k)


def test_list_length_bound_is_needed():
    """With lists shorter than k the merge can miss a chunk: one segment
    holding all k best chunks must publish at least k of them."""
    scores = np.array([9.0, 8.0, 7.0, 1.0, 0.0])
    k = 3

    def merged_with(length):
        kept = []
        for a, b in ((0, 3), (3, 5)):
            seg = sorted(range(a, b), key=lambda i: order_key(scores, i))
            kept.extend(seg[:length])
        kept.sort(key=lambda i: order_key(scores, i))
        return sorted(kept[:k])

    assert merged_with(3) == topk_definition(scores, k)
    assert merged_with(2) != topk_definition(scores, k)

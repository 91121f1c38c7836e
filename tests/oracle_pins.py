"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes an ``oracle.ssa_oracle.Oracle`` and raises
``AssertionError`` when the oracle disagrees with
  * the independent numpy brute force (dense matmul scoring, k-subset
    enumeration for top-k, explicit token list + one dense softmax),
  * textbook attention from ``torch.nn.functional.scaled_dot_product_attention``
    in fp64 (the k = M and k = 0 invariants of the method),
  * closed forms (one visible token, all keys equal, a query parallel to one
    gist key, the context-size identity),
  * the hand-worked example in ``tests/golden/hand_example.json``.
The same pins run against every planted mutant of the oracle; each mutant must
fail at least one of them.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

from oracle import bruteforce

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, lens, J=0, gm=0):
    M_max = n_max // C
    case = {
        "q": rng.standard_normal((B, Hq, d)).astype(np.float32),
        "k_raw": rng.standard_normal((B, Hkv, n_max, d)).astype(np.float32),
        "v_raw": rng.standard_normal((B, Hkv, n_max, d)).astype(np.float32),
        "k_gist": rng.standard_normal((B, Hkv, M_max, g, d)).astype(np.float32),
        "v_gist": rng.standard_normal((B, Hkv, M_max, g, d)).astype(np.float32),
        "seq_lens": np.asarray(lens, np.int32),
    }
    if J:
        S_max = M_max // J
        case["k_meta"] = rng.standard_normal((B, Hkv, S_max, gm, d)).astype(np.float32)
        case["v_meta"] = rng.standard_normal((B, Hkv, S_max, gm, d)).astype(np.float32)
    return case


def _args(c):
    return (c["q"], c["k_raw"], c["v_raw"], c["k_gist"], c["v_gist"], c["seq_lens"])


def _close(a, b, tol=1e-10, what=""):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    fin = np.isfinite(b)
    assert np.array_equal(np.isfinite(a), fin), f"{what}: finiteness differs"
    assert np.array_equal(a[~fin], b[~fin]), f"{what}: infinities differ"
    err = np.abs(a[fin] - b[fin]).max() if fin.any() else 0.0
    assert err <= tol, f"{what}: max abs err {err:g} > {tol:g}"


# single-level shapes: (B, Hq, Hkv, d, C, g, n_max, seq_lens, topk)
SINGLE_CASES = [
    (1, 1, 1, 8, 4, 2, 32, [27], 3),
    (2, 4, 2, 8, 4, 2, 40, [40, 33], 4),
    (2, 8, 2, 16, 8, 2, 64, [61, 9], 2),
    (1, 6, 3, 8, 5, 3, 50, [49], 5),
    (2, 4, 1, 8, 4, 1, 24, [23, 3], 0),
    (1, 2, 2, 8, 3, 2, 30, [30], 20),   # topk > M: select all
    (2, 4, 2, 8, 4, 2, 16, [2, 16], 2), # M = 0 for one sequence
]


def pin_bruteforce_single(orc):
    rng = np.random.default_rng(1234)
    for (B, Hq, Hkv, d, C, g, n_max, lens, topk) in SINGLE_CASES:
        c = _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, lens)
        o = orc.decode(*_args(c), C=C, g=g, topk=topk)
        r = bruteforce.decode(*_args(c), C=C, g=g, topk=topk)
        _close(o["scores"], r["scores"], 1e-12, "scores")
        assert np.array_equal(o["sel_idx"], r["sel_idx"]), ("sel", o["sel_idx"], r["sel_idx"])
        assert np.array_equal(o["ctx"], r["ctx"]), ("ctx", o["ctx"], r["ctx"])
        _close(o["out"], r["out"], 1e-12, "out")
        _close(o["lse"], r["lse"], 1e-12, "lse")


def pin_given_selection(orc):
    """Attention on a given (non top-k) selection equals the brute force's."""
    rng = np.random.default_rng(99)
    B, Hq, Hkv, d, C, g, n_max, topk = 2, 4, 2, 8, 4, 2, 40, 3
    c = _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, [38, 21])
    sel = np.full((B, Hkv, topk), -1, np.int32)
    sel[0, 0, :3] = [0, 4, 8]
    sel[0, 1, :1] = [7]
    sel[1, 0, :2] = [1, 2]
    o = orc.decode(*_args(c), C=C, g=g, topk=topk, sel=sel)
    r = bruteforce.decode(*_args(c), C=C, g=g, topk=topk, sel=sel)
    assert np.array_equal(o["sel_idx"], sel)
    _close(o["out"], r["out"], 1e-12, "out")
    assert np.array_equal(o["ctx"], r["ctx"])


def pin_ties(orc):
    """Equal scores go to the lower chunk index."""
    rng = np.random.default_rng(7)
    B, Hq, Hkv, d, C, g, n_max = 1, 2, 1, 8, 4, 2, 32
    c = _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, [32])
    # chunk 5 is a copy of chunk 2 and both beat every other chunk
    q = c["q"][0]
    boost = (q.sum(0) / np.linalg.norm(q.sum(0))).astype(np.float32) * 6.0
    c["k_gist"][0, 0, 2, 0] = boost
    c["k_gist"][0, 0, 5] = c["k_gist"][0, 0, 2]
    o = orc.decode(*_args(c), C=C, g=g, topk=1)
    assert o["scores"][0, 0, 2] == o["scores"][0, 0, 5]
    assert list(o["sel_idx"][0, 0]) == [2], o["sel_idx"]
    o3 = orc.decode(*_args(c), C=C, g=g, topk=2)
    assert list(o3["sel_idx"][0, 0]) == [2, 5], o3["sel_idx"]
    # all gist keys equal -> all scores equal -> chunks 0..k-1
    c["k_gist"][:] = c["k_gist"][0, 0, 0, 0]
    o = orc.decode(*_args(c), C=C, g=g, topk=3)
    assert list(o["sel_idx"][0, 0]) == [0, 1, 2], o["sel_idx"]
    r = bruteforce.decode(*_args(c), C=C, g=g, topk=3)
    assert np.array_equal(o["sel_idx"], r["sel_idx"])


def _sdpa(qh, K, V):
    """Textbook softmax attention of one query from torch (fp64)."""
    qt = torch.from_numpy(np.asarray(qh, np.float64))[None, None, None, :]
    Kt = torch.from_numpy(np.asarray(K, np.float64))[None, None]
    Vt = torch.from_numpy(np.asarray(V, np.float64))[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt)
    logits = (Kt[0, 0] @ qt[0, 0, 0]) / math.sqrt(qh.shape[-1])
    return out[0, 0, 0].numpy(), torch.logsumexp(logits, 0).item()


def pin_dense_when_all_selected(orc):
    """k >= M  =>  dense causal attention over all n raw tokens."""
    rng = np.random.default_rng(5)
    B, Hq, Hkv, d, C, g, n_max = 2, 4, 2, 16, 4, 2, 48
    lens = [45, 17]
    c = _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, lens)
    o = orc.decode(*_args(c), C=C, g=g, topk=n_max // C)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            j = h // G
            ref, l = _sdpa(c["q"][b, h], c["k_raw"][b, j, :lens[b]], c["v_raw"][b, j, :lens[b]])
            _close(o["out"][b, h], ref, 1e-12, "dense out")
            _close(o["lse"][b, h], l, 1e-12, "dense lse")


def pin_gists_when_none_selected(orc):
    """k = 0  =>  attention over all gists of complete chunks plus the tail."""
    rng = np.random.default_rng(6)
    B, Hq, Hkv, d, C, g, n_max = 2, 4, 2, 16, 4, 3, 48
    lens = [47, 12]
    c = _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, lens)
    o = orc.decode(*_args(c), C=C, g=g, topk=0)
    G = Hq // Hkv
    for b in range(B):
        M = lens[b] // C
        for h in range(Hq):
            j = h // G
            K = np.concatenate([c["k_gist"][b, j, :M].reshape(M * g, d),
                                c["k_raw"][b, j, M * C:lens[b]]])
            V = np.concatenate([c["v_gist"][b, j, :M].reshape(M * g, d),
                                c["v_raw"][b, j, M * C:lens[b]]])
            ref, l = _sdpa(c["q"][b, h], K, V)
            _close(o["out"][b, h], ref, 1e-12, "gist-only out")
            _close(o["lse"][b, h], l, 1e-12, "gist-only lse")


def pin_single_token(orc):
    """n = 1: the context is the one raw token, so out = its value exactly."""
    rng = np.random.default_rng(8)
    c = _rand_case(rng, 1, 2, 1, 8, 4, 2, 8, [1])
    o = orc.decode(*_args(c), C=4, g=2, topk=2)
    for h in range(2):
        assert np.array_equal(o["out"][0, h], c["v_raw"][0, 0, 0].astype(np.float64))
    assert list(o["sel_idx"][0, 0]) == [-1, -1]
    assert o["ctx"][0, 0] == 1


def pin_equal_keys_mean(orc):
    """All keys equal => uniform softmax => out = mean of the context's values."""
    rng = np.random.default_rng(9)
    B, Hq, Hkv, d, C, g, n_max, n = 1, 2, 1, 8, 4, 2, 28, 26
    c = _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, [n])
    key = rng.standard_normal(d).astype(np.float32)
    c["k_raw"][:] = key
    c["k_gist"][:] = key
    sel = np.array([[[1, 4]]], np.int32)
    o = orc.decode(*_args(c), C=C, g=g, topk=2, sel=sel)
    M = n // C
    vals = [c["v_gist"][0, 0, m] for m in range(M) if m not in (1, 4)]
    vals += [c["v_raw"][0, 0, 4:8], c["v_raw"][0, 0, 16:20], c["v_raw"][0, 0, M * C:n]]
    mean = np.concatenate(vals).astype(np.float64).mean(0)
    for h in range(Hq):
        _close(o["out"][0, h], mean, 1e-12, "equal-keys mean")


def pin_context_size(orc):
    """|X| = (M - k) g + k C + T for every (sequence, KV head)."""
    rng = np.random.default_rng(10)
    for (B, Hq, Hkv, d, C, g, n_max, lens, topk) in SINGLE_CASES:
        c = _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, lens)
        o = orc.decode(*_args(c), C=C, g=g, topk=topk)
        for b in range(B):
            M = lens[b] // C
            k = min(topk, M)
            T = lens[b] - M * C
            assert (o["ctx"][b] == (M - k) * g + k * C + T).all(), (b, o["ctx"][b])


def pin_parallel_query(orc):
    """q = a*e for one head, one nonzero gist key e: that chunk scores a|e|^2/sqrt(d)."""
    B, Hq, Hkv, d, C, g, n_max = 1, 4, 1, 16, 4, 2, 32
    z = lambda *s: np.zeros(s, np.float32)
    c = {"q": z(B, Hq, d), "k_raw": z(B, Hkv, n_max, d), "v_raw": z(B, Hkv, n_max, d),
         "k_gist": z(B, Hkv, n_max // C, g, d), "v_gist": z(B, Hkv, n_max // C, g, d),
         "seq_lens": np.array([32], np.int32)}
    e = np.zeros(d, np.float32)
    e[3], e[7] = 1.5, -2.0
    c["k_gist"][0, 0, 6, 1] = e
    c["q"][0, 2] = 3.0 * e
    o = orc.decode(*_args(c), C=C, g=g, topk=1)
    want = 3.0 * float(e @ e) / math.sqrt(d)
    assert abs(o["scores"][0, 0, 6] - want) <= 1e-12, (o["scores"][0, 0, 6], want)
    others = np.delete(o["scores"][0, 0], 6)
    assert (others == 0.0).all()
    assert list(o["sel_idx"][0, 0]) == [6]


def pin_hand_example(orc):
    """The hand-worked example in tests/golden/hand_example.json."""
    with open(os.path.join(GOLDEN, "hand_example.json")) as f:
        ex = json.load(f)
    s = ex["shape"]
    arr = lambda k: np.asarray(ex[k], np.float32)
    o = orc.decode(arr("q"), arr("k_raw"), arr("v_raw"), arr("k_gist"), arr("v_gist"),
                   np.asarray(ex["seq_lens"], np.int32), C=s["C"], g=s["g"], topk=s["topk"])
    e = ex["expected"]
    want_scores = [float(x) for x in e["scores"]]
    _close(o["scores"][0, 0], want_scores, 1e-15, "hand scores")
    assert list(o["sel_idx"][0, 0]) == e["sel_idx"]
    assert int(o["ctx"][0, 0]) == e["ctx"]
    w = np.exp(np.asarray(e["context_logits"], np.float64))
    vals = np.asarray(e["context_values"], np.float64)
    want = (w[:, None] * vals).sum(0) / w.sum()
    _close(o["out"][0, 0], want, 1e-15, "hand out")
    _close(o["lse"][0, 0], math.log(w.sum()), 1e-15, "hand lse")


H2_CASES = [
    # (B, Hq, Hkv, d, C, g, n_max, lens, J, gm, topk_super, topk_chunk)
    (1, 2, 1, 8, 4, 2, 96, [93], 4, 2, 2, 3),      # S=5, R=3 remainder chunks, tail 1
    (2, 4, 2, 8, 2, 1, 64, [64, 37], 3, 2, 1, 2),  # remainder + tails
    (1, 4, 1, 8, 4, 2, 64, [64], 4, 3, 0, 2),      # no superchunk kept: remainder only
]


def pin_bruteforce_h2(orc):
    rng = np.random.default_rng(4321)
    for (B, Hq, Hkv, d, C, g, n_max, lens, J, gm, ts, tc) in H2_CASES:
        c = _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, lens, J=J, gm=gm)
        args = _args(c)[:5] + (c["k_meta"], c["v_meta"], c["seq_lens"])
        o = orc.decode_h2(*args, C=C, g=g, J=J, gm=gm, topk_super=ts, topk_chunk=tc)
        r = bruteforce.decode_h2(*args, C=C, g=g, J=J, gm=gm, topk_super=ts, topk_chunk=tc)
        _close(o["super_scores"], r["super_scores"], 1e-12, "h2 super scores")
        _close(o["scores"], r["scores"], 1e-12, "h2 chunk scores")
        assert np.array_equal(o["sel_super"], r["sel_super"]), (o["sel_super"], r["sel_super"])
        assert np.array_equal(o["sel_idx"], r["sel_idx"]), (o["sel_idx"], r["sel_idx"])
        assert np.array_equal(o["ctx"], r["ctx"])
        _close(o["out"], r["out"], 1e-12, "h2 out")
        _close(o["lse"], r["lse"], 1e-12, "h2 lse")


def pin_h2_reduces_to_single(orc):
    """Keeping every superchunk makes the two-level step the single-level one."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, d, C, g, n_max, J, gm = 2, 4, 2, 8, 4, 2, 96, 3, 2
    lens = [95, 50]
    c = _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, lens, J=J, gm=gm)
    args = _args(c)[:5] + (c["k_meta"], c["v_meta"], c["seq_lens"])
    o2 = orc.decode_h2(*args, C=C, g=g, J=J, gm=gm, topk_super=100, topk_chunk=4)
    o1 = orc.decode(*_args(c), C=C, g=g, topk=4)
    assert np.array_equal(o2["sel_idx"], o1["sel_idx"])
    _close(o2["out"], o1["out"], 1e-12, "h2->single out")
    # and with every chunk kept too: dense attention
    o3 = orc.decode_h2(*args, C=C, g=g, J=J, gm=gm, topk_super=100, topk_chunk=100)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            ref, _ = _sdpa(c["q"][b, h], c["k_raw"][b, h // G, :lens[b]],
                           c["v_raw"][b, h // G, :lens[b]])
            _close(o3["out"][b, h], ref, 1e-12, "h2 dense")


def pin_bad_length(orc):
    """A length outside [1, n_max] is reported and zeroes that sequence."""
    rng = np.random.default_rng(12)
    c = _rand_case(rng, 2, 2, 1, 8, 4, 2, 16, [16, 17])
    o = orc.decode(*_args(c), C=4, g=2, topk=2)
    assert o["bad_seq"] == 2
    assert (o["out"][1] == 0).all() and (o["sel_idx"][1] == -1).all()
    assert np.isfinite(o["out"][0]).all() and (o["sel_idx"][0] >= 0).all()


def pin_nan_gist_key(orc):
    """A NaN logit never wins a chunk's score maximum, and a chunk whose every
    logit is NaN scores -inf, ranks last and is selected only when k reaches
    it (ties to the lower index among the -inf chunks)."""
    rng = np.random.default_rng(21)
    B, Hq, Hkv, d, C, g, n_max = 1, 2, 1, 8, 4, 2, 32
    c = _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, [31])   # M = 7, tail of 3
    q = c["q"][0]
    boost = (q.sum(0) / np.linalg.norm(q.sum(0))).astype(np.float32) * 6.0
    # chunk 2: one gist row NaN, the other the clear winner -> still selected
    c["k_gist"][0, 0, 2, 0] = boost
    c["k_gist"][0, 0, 2, 1, 3] = np.nan
    # chunk 5: every gist key NaN -> score -inf
    c["k_gist"][0, 0, 5] = np.nan
    o = orc.decode(*_args(c), C=C, g=g, topk=2)
    r = bruteforce.decode(*_args(c), C=C, g=g, topk=2)
    s = o["scores"][0, 0]
    assert np.isfinite(s[2]) and s[2] == s.max()
    assert s[5] == -np.inf
    assert 2 in o["sel_idx"][0, 0] and 5 not in o["sel_idx"][0, 0]
    assert np.array_equal(o["sel_idx"], r["sel_idx"]), (o["sel_idx"], r["sel_idx"])
    # chunk 5's NaN gist keys are in the context (unselected): the output is NaN
    assert np.isnan(o["out"]).all() and np.isnan(r["out"]).all()
    # k = 6 of 7: chunk 5 is the one left out; k = 7: all chunks, a finite output
    o6 = orc.decode(*_args(c), C=C, g=g, topk=6)
    assert list(o6["sel_idx"][0, 0]) == [0, 1, 2, 3, 4, 6]
    r6 = bruteforce.decode(*_args(c), C=C, g=g, topk=6)
    assert np.array_equal(o6["sel_idx"], r6["sel_idx"])
    o7 = orc.decode(*_args(c), C=C, g=g, topk=7)
    r7 = bruteforce.decode(*_args(c), C=C, g=g, topk=7)
    assert list(o7["sel_idx"][0, 0]) == list(range(7))
    _close(o7["out"], r7["out"], 1e-12, "all selected around NaN gists")
    # two all-NaN chunks tie at -inf: the lower index goes first
    c["k_gist"][0, 0, 1] = np.nan
    o6 = orc.decode(*_args(c), C=C, g=g, topk=6)
    assert list(o6["sel_idx"][0, 0]) == [0, 1, 2, 3, 4, 6]
    r6 = bruteforce.decode(*_args(c), C=C, g=g, topk=6)
    assert np.array_equal(o6["sel_idx"], r6["sel_idx"])


VARIANT_CASES = [
    # (B, Hq, Hkv, d, C, g, n_max, seq_lens, topk)
    (1, 4, 1, 8, 4, 2, 32, [30], 2),
    (2, 4, 2, 8, 4, 2, 40, [40, 27], 3),
    (1, 6, 2, 8, 5, 3, 45, [44], 2),
    (2, 2, 2, 8, 3, 2, 30, [30, 7], 20),   # topk > M: every chunk
    (1, 4, 2, 8, 4, 2, 16, [3], 2),        # M = 0: tail only
    (2, 8, 2, 8, 4, 2, 24, [23, 24], 0),   # topk = 0
]


def pin_variants_bruteforce(orc):
    """Both context readings and both selection readings against the brute
    force (dense scoring, subset-enumeration top-k, explicit token list)."""
    rng = np.random.default_rng(4321)
    for (B, Hq, Hkv, d, C, g, n_max, lens, topk) in VARIANT_CASES:
        c = _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, lens)
        for context in (0, 1):
            for select in (0, 1):
                o = orc.decode(*_args(c), C=C, g=g, topk=topk, context=context, select=select)
                r = bruteforce.decode(*_args(c), C=C, g=g, topk=topk, context=context,
                                      select=select)
                what = f"context={context} select={select} case={(B, Hq, Hkv, C, g, lens, topk)}"
                _close(o["scores"], r["scores"], 1e-12, "scores " + what)
                assert np.array_equal(o["sel_idx"], r["sel_idx"]), ("sel " + what, o["sel_idx"],
                                                                   r["sel_idx"])
                assert np.array_equal(o["ctx"], r["ctx"]), ("ctx " + what, o["ctx"], r["ctx"])
                _close(o["out"], r["out"], 1e-12, "out " + what)
                _close(o["lse"], r["lse"], 1e-12, "lse " + what)


def pin_selected_only_closed_forms(orc):
    """Context "selected only": |X| = k (C + g) + T; with k = M it is textbook
    attention over every raw token and every gist token; with k = 0 it is
    attention over the tail alone (an empty context gives 0 and lse -inf)."""
    rng = np.random.default_rng(77)
    B, Hq, Hkv, d, C, g, n_max = 2, 4, 2, 8, 4, 2, 40
    c = _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, [38, 32])
    G = Hq // Hkv
    for topk in (0, 2, 5, 10):
        o = orc.decode(*_args(c), C=C, g=g, topk=topk, context=1)
        for b, n in enumerate(c["seq_lens"]):
            M, T = int(n) // C, int(n) % C
            k = min(topk, M)
            assert (o["ctx"][b] == k * (C + g) + T).all(), (topk, b, o["ctx"][b])
    o = orc.decode(*_args(c), C=C, g=g, topk=10, context=1)
    for b, n in enumerate(c["seq_lens"]):
        n = int(n)
        M = n // C
        for h in range(Hq):
            j = h // G
            K = np.concatenate([c["k_raw"][b, j, :n], c["k_gist"][b, j, :M].reshape(-1, d)])
            V = np.concatenate([c["v_raw"][b, j, :n], c["v_gist"][b, j, :M].reshape(-1, d)])
            ref, lse = _sdpa(c["q"][b, h], K, V)
            _close(o["out"][b, h], ref, 1e-12, "selected-only, k = M")
            _close(o["lse"][b, h], lse, 1e-12, "selected-only lse, k = M")
    o0 = orc.decode(*_args(c), C=C, g=g, topk=0, context=1)
    for b, n in enumerate(c["seq_lens"]):
        n = int(n)
        M = n // C
        for h in range(Hq):
            j = h // G
            if n == M * C:
                assert (o0["out"][b, h] == 0).all() and o0["lse"][b, h] == -np.inf
            else:
                ref, _ = _sdpa(c["q"][b, h], c["k_raw"][b, j, M * C:n], c["v_raw"][b, j, M * C:n])
                _close(o0["out"][b, h], ref, 1e-12, "selected-only, k = 0")


def pin_union_reductions(orc):
    """Per-head selection + union: with one query head per KV head it is the
    shared selection; with equal queries in a group every head picks the
    shared top-k, so the union is it; in general the union holds every head's
    own top-k of its own scores and has between k and min(G k, M) chunks."""
    rng = np.random.default_rng(5)
    # G = 1
    c = _rand_case(rng, 2, 3, 3, 8, 4, 2, 40, [40, 29])
    for context in (0, 1):
        a = orc.decode(*_args(c), C=4, g=2, topk=3, context=context, select=0)
        u = orc.decode(*_args(c), C=4, g=2, topk=3, context=context, select=1)
        assert np.array_equal(a["sel_idx"], u["sel_idx"])
        _close(u["out"], a["out"], 1e-12, "union with G = 1")
        _close(u["scores"], a["scores"], 1e-12, "per-head scores with G = 1")
    # equal queries in each group
    c = _rand_case(rng, 1, 8, 2, 8, 4, 2, 48, [46])
    c["q"][0, 1:4] = c["q"][0, 0]
    c["q"][0, 5:8] = c["q"][0, 4]
    a = orc.decode(*_args(c), C=4, g=2, topk=4, select=0)
    u = orc.decode(*_args(c), C=4, g=2, topk=4, select=1)
    assert np.array_equal(u["sel_idx"][..., :4], a["sel_idx"]) and (u["sel_idx"][..., 4:] == -1).all()
    _close(u["out"], a["out"], 1e-12, "union of equal heads")
    # general: containment and size
    c = _rand_case(rng, 2, 8, 2, 8, 4, 2, 64, [64, 50])
    topk = 3
    u = orc.decode(*_args(c), C=4, g=2, topk=topk, select=1)
    G = 4
    for b, n in enumerate(c["seq_lens"]):
        M = int(n) // 4
        for j in range(2):
            chosen = [int(x) for x in u["sel_idx"][b, j] if x >= 0]
            assert chosen == sorted(set(chosen))
            assert min(topk, M) <= len(chosen) <= min(G * topk, M)
            for r in range(G):
                own = bruteforce.topk_subsets(u["scores"][b, j * G + r], range(M), topk)
                assert set(own) <= set(chosen), (b, j, r, own, chosen)


def _hier_case(rng, B, Hq, Hkv, d, C, g, n_max, lens, J, gs):
    """Random inputs with one summary tensor per level >= 2 (gs[l-2] tokens)."""
    c = _rand_case(rng, B, Hq, Hkv, d, C, g, n_max, lens)
    umax = n_max // C
    c["k_sum"], c["v_sum"] = [], []
    for gl in gs:
        umax //= J
        c["k_sum"].append(rng.standard_normal((B, Hkv, umax, gl, d)).astype(np.float32))
        c["v_sum"].append(rng.standard_normal((B, Hkv, umax, gl, d)).astype(np.float32))
    return c


HIER_CASES = [
    # (B, Hq, Hkv, d, C, g, n_max, seq_lens, J, gs (levels 2..t), topks (levels 1..t))
    (1, 4, 2, 8, 2, 2, 32, [31], 2, [2, 3], [2, 1, 1]),       # 15 chunks: remainders at 2 levels
    (2, 2, 1, 8, 2, 1, 36, [36, 25], 3, [2], [3, 1]),
    (1, 4, 1, 8, 2, 2, 34, [34], 2, [1, 2, 2], [3, 2, 1, 1]),  # four levels
    (2, 4, 2, 8, 3, 2, 42, [41, 13], 2, [2, 2], [0, 2, 1]),   # topk 0 at the chunk level
    (1, 2, 1, 8, 2, 2, 28, [27], 3, [2], [20, 9]),           # every unit kept
]


def pin_hier_bruteforce(orc):
    """t-level selection against the recursive brute force (subset top-k per
    level, explicit context list), for t = 2, 3, 4 with remainder units."""
    rng = np.random.default_rng(2468)
    for (B, Hq, Hkv, d, C, g, n_max, lens, J, gs, topks) in HIER_CASES:
        c = _hier_case(rng, B, Hq, Hkv, d, C, g, n_max, lens, J, gs)
        o = orc.decode_hier(*_args(c)[:5], c["k_sum"], c["v_sum"], c["seq_lens"], C=C, g=g, J=J,
                            topks=topks)
        r = bruteforce.decode_hier(*_args(c)[:5], c["k_sum"], c["v_sum"], c["seq_lens"], C, g, J,
                                   topks)
        for l in range(len(topks)):
            assert np.array_equal(o["sels"][l], r["sels"][l]), (l, o["sels"][l], r["sels"][l])
        assert np.array_equal(o["ctx"], r["ctx"]), (o["ctx"], r["ctx"])
        _close(o["out"], r["out"], 1e-12, f"hier out J={J} topks={topks}")


def pin_hier_reductions(orc):
    """One level is the single-level step; two levels are the two-level step;
    t levels whose top level keeps every unit are the t-1 levels below it."""
    rng = np.random.default_rng(1357)
    B, Hq, Hkv, d, C, g, n_max, J = 2, 4, 2, 8, 2, 2, 64, 2
    c = _hier_case(rng, B, Hq, Hkv, d, C, g, n_max, [64, 45], J, [2, 3, 2])
    a = _args(c)
    one = orc.decode_hier(*a[:5], [], [], c["seq_lens"], C=C, g=g, J=J, topks=[5])
    ref = orc.decode(*a, C=C, g=g, topk=5)
    assert np.array_equal(one["sels"][0], ref["sel_idx"])
    _close(one["out"], ref["out"], 1e-12, "one level")
    two = orc.decode_hier(*a[:5], c["k_sum"][:1], c["v_sum"][:1], c["seq_lens"], C=C, g=g, J=J,
                          topks=[4, 3])
    ref2 = orc.decode_h2(*a[:5], c["k_sum"][0], c["v_sum"][0], c["seq_lens"], C=C, g=g, J=J,
                         gm=2, topk_super=3, topk_chunk=4)
    assert np.array_equal(two["sels"][0], ref2["sel_idx"])
    assert np.array_equal(two["sels"][1], ref2["sel_super"])
    _close(two["out"], ref2["out"], 1e-12, "two levels")
    for t in (3, 4):
        lower = orc.decode_hier(*a[:5], c["k_sum"][:t - 2], c["v_sum"][:t - 2], c["seq_lens"],
                                C=C, g=g, J=J, topks=[4, 3, 2][:t - 1])
        upper = orc.decode_hier(*a[:5], c["k_sum"][:t - 1], c["v_sum"][:t - 1], c["seq_lens"],
                                C=C, g=g, J=J, topks=[4, 3, 2][:t - 1] + [1000])
        for l in range(t - 1):
            assert np.array_equal(upper["sels"][l], lower["sels"][l]), (t, l)
        _close(upper["out"], lower["out"], 1e-12, f"{t} levels, top kept")
        # the context counts: candidates' summaries or raw tokens, plus the tail
        for b, n in enumerate(c["seq_lens"]):
            M = int(n) // C
            U = [M]
            for _ in range(1, t):
                U.append(U[-1] // J)
            for j in range(Hkv):
                size = int(n) - M * C
                kept = []
                gl = [g, 2, 3, 2]
                for lv in range(t, 0, -1):
                    cand = (list(range(U[lv - 1])) if lv == t else
                            [x * J + i for x in kept for i in range(J)] + list(range(U[lv] * J, U[lv - 1])))
                    keep = [int(x) for x in upper["sels"][lv - 1][b, j] if x >= 0]
                    assert set(keep) <= set(cand)
                    size += sum(C if (lv == 1 and x in keep) else (0 if x in keep else gl[lv - 1])
                                for x in cand)
                    kept = keep
                assert upper["ctx"][b, j] == size, (t, b, j, upper["ctx"][b, j], size)


# ------------------------------------------------- adaptive top-k (App. A) ---

def pin_adaptive_topk_properties(orc):
    """The properties App. A states for the budget (its formula is not
    printed, so the exact value stays unpinned): a chunk is always chosen; the
    group's union of raw tokens, G k L, tracks n_kv / L_eff (effective
    compression L for SSA, L J for H-SSA); dividing by G keeps that union from
    growing with the group size; more cache never lowers the budget."""
    for L in (16, 64, 128):
        for G in (1, 4, 8):
            for J in (1, 4, 16):
                l_eff = L * J
                assert orc.adaptive_topk(0, L, G, J) == 1
                assert orc.adaptive_topk(1, L, G, J) == 1
                prev = 0
                for e in range(8, 27, 2):
                    n_kv = (1 << e) + 12345
                    k = orc.adaptive_topk(n_kv, L, G, J)
                    assert k >= 1 and k >= prev, (n_kv, L, G, J, k, prev)
                    prev = k
                    union = G * k * L
                    target = n_kv / l_eff
                    assert target < union <= target + G * L, (n_kv, L, G, J, k)
    # the union budget is (nearly) independent of G at a fixed cache size
    for G in (1, 2, 4, 8, 16):
        k = orc.adaptive_topk(1 << 24, 64, G, 1)
        assert abs(G * k - (1 << 24) // (64 * 64)) <= G, (G, k)


# --------------------------------------- prefill under the gist mask (3.1) ---

def _prefill_case(rng, B, Hq, Hkv, d, C, g, n_max, lens):
    M_max = n_max // C
    f = lambda *shape: rng.standard_normal(shape).astype(np.float32)
    return {"q_raw": f(B, Hq, n_max, d), "q_gist": f(B, Hq, M_max, g, d),
            "k_raw": f(B, Hkv, n_max, d), "k_gist": f(B, Hkv, M_max, g, d),
            "v_raw": f(B, Hkv, n_max, d), "v_gist": f(B, Hkv, M_max, g, d),
            "seq_lens": np.asarray(lens, np.int32)}


def _prefill(orc, c, C, g):
    return orc.prefill(c["q_raw"], c["q_gist"], c["k_raw"], c["k_gist"], c["v_raw"],
                       c["v_gist"], c["seq_lens"], C, g)


def pin_prefill_one_chunk_is_causal(orc):
    """With at most one chunk the gist mask is plain causal attention over
    the interleaved order (the chunk's raw tokens, then its gists): textbook
    causal softmax from torch, fp64."""
    B, Hq, Hkv, d, C, g = 3, 4, 2, 16, 16, 3
    c = _prefill_case(np.random.default_rng(71), B, Hq, Hkv, d, C, g, C, [16, 11, 1])
    res = _prefill(orc, c, C, g)
    G = Hq // Hkv
    for b, n in enumerate(c["seq_lens"]):
        n = int(n)
        ng = g if n == C else 0
        for h in range(Hq):
            j = h // G
            q = np.concatenate([c["q_raw"][b, h, :n], c["q_gist"][b, h, 0, :ng]])
            k = np.concatenate([c["k_raw"][b, j, :n], c["k_gist"][b, j, 0, :ng]])
            v = np.concatenate([c["v_raw"][b, j, :n], c["v_gist"][b, j, 0, :ng]])
            t = lambda x: torch.from_numpy(x.astype(np.float64))[None, None]
            want = torch.nn.functional.scaled_dot_product_attention(
                t(q), t(k), t(v), is_causal=True)[0, 0].numpy()
            _close(res["o_raw"][b, h, :n], want[:n], 1e-12, f"raw rows b={b} h={h}")
            if ng:
                _close(res["o_gist"][b, h, 0, :ng], want[n:], 1e-12, f"gist rows b={b} h={h}")


def _visible_sets(n, C, g):
    """Interleaved positions each row sees, listed from the sentence of sec.
    3.1 (its own chunk up to itself, every gist of the earlier chunks)."""
    M = n // C
    pos_raw = lambda i: (i // C) * (C + g) + i % C if i < M * C else M * (C + g) + i - M * C
    pos_gist = lambda m, t: m * (C + g) + C + t
    earlier_gists = lambda m: [pos_gist(mm, t) for mm in range(m) for t in range(g)]
    raw_rows, gist_rows = [], []
    for i in range(n):
        m = i // C
        own = [pos_raw(x) for x in range(m * C, i + 1)]
        raw_rows.append((own, earlier_gists(m)))
    for m in range(M):
        for t in range(g):
            own = [pos_raw(x) for x in range(m * C, m * C + C)] + [pos_gist(m, u) for u in range(t + 1)]
            gist_rows.append((own, earlier_gists(m)))
    return raw_rows, gist_rows, pos_raw, pos_gist


def pin_prefill_visible_sets(orc):
    """Zero keys make every visible key equally weighted, so each output row is
    the mean of the value features over the row's visible set: the share of
    gist keys, and the mean and mean square of their interleaved positions,
    checked against the sets listed from the sentence of sec. 3.1."""
    B, Hq, Hkv, d, C, g, n_max = 2, 2, 1, 8, 5, 2, 30
    lens = [28, 13]
    c = _prefill_case(np.random.default_rng(5), B, Hq, Hkv, d, C, g, n_max, lens)
    c["k_raw"][:] = 0
    c["k_gist"][:] = 0
    c["v_raw"][:] = 0
    c["v_gist"][:] = 0
    for b, n in enumerate(lens):
        raw_rows, gist_rows, pos_raw, pos_gist = _visible_sets(n, C, g)
        scale = 1.0 / 64
        for i in range(n):
            c["v_raw"][b, 0, i, :3] = (0.0, pos_raw(i) * scale, (pos_raw(i) * scale) ** 2)
        for m in range(n // C):
            for t in range(g):
                p = pos_gist(m, t) * scale
                c["v_gist"][b, 0, m, t, :3] = (1.0, p, p * p)
    res = _prefill(orc, c, C, g)
    for b, n in enumerate(lens):
        raw_rows, gist_rows, pos_raw, pos_gist = _visible_sets(n, C, g)
        for kind, rows in (("raw", raw_rows), ("gist", gist_rows)):
            for r, (own, gists) in enumerate(rows):
                allp = np.asarray(own + gists, np.float64) / 64
                n_gist = len(gists) + (sum(1 for x in own if x % (C + g) >= C
                                           and x < (n // C) * (C + g)))
                want = np.array([n_gist / len(allp), allp.mean(), (allp ** 2).mean()])
                got = (res["o_raw"][b, :, r, :3] if kind == "raw"
                       else res["o_gist"][b, :, r // g, r % g, :3])
                for h in range(Hq):
                    _close(got[h], want, 1e-12, f"{kind} row {r} b={b} h={h}")


def pin_prefill_last_token_is_decode(orc):
    """The last raw token of a sequence with a non-empty tail sees every gist
    and the tail up to itself: the decode step's context with nothing
    unfolded (k = 0), from the decode oracle."""
    B, Hq, Hkv, d, C, g, n_max = 2, 4, 2, 16, 6, 2, 48
    lens = [45, 20]
    c = _prefill_case(np.random.default_rng(9), B, Hq, Hkv, d, C, g, n_max, lens)
    res = _prefill(orc, c, C, g)
    q_last = np.stack([c["q_raw"][b, :, n - 1] for b, n in enumerate(lens)])
    dec = orc.decode(q_last, c["k_raw"], c["v_raw"], c["k_gist"], c["v_gist"], c["seq_lens"],
                     C=C, g=g, topk=0)
    for b, n in enumerate(lens):
        _close(res["o_raw"][b, :, n - 1], dec["out"][b], 1e-12, f"b={b}")


# ------------------------------------------- prefill block mask (sec. 3.6) ---

def _entry(block, part, full):
    return (block << 2) | (part << 1) | int(full)


def pin_prefill_blocks_causal(orc):
    """No complete chunk: the mask is causal over the raw tokens, so tile
    [r0, r1) lists raw blocks 0 .. (r1 - 1) // BN, full when the block ends at
    or before row r0's own column."""
    for (n, C, BM, BN) in ((1, 8, 4, 4), (13, 16, 4, 4), (30, 64, 8, 4), (31, 32, 4, 8)):
        plan = orc.prefill_blocks(n, C, 2, BM, BN)
        want = []
        for r0 in range(0, n, BM):
            r1 = min(n, r0 + BM)
            ents = [_entry(b, 1, b * BN + BN <= r0 + 1 and b * BN + BN <= n)
                    for b in range(0, (r1 - 1) // BN + 1)]
            want.append(((0, r0, r1 - r0), ents))
        assert plan == want, (n, C, BM, BN, plan, want)


def pin_prefill_blocks_counts(orc):
    """Chunks of C >= BM rows: a raw tile of chunk m lists the gist blocks
    covering [0, m g) (full when inside it) and the raw blocks of its own
    chunk up to its last row; a gist tile lists the gist blocks up to its last
    row (causal) and the raw blocks of the chunks its rows summarise (full
    only when all its rows belong to one chunk)."""
    for (n, C, g, BM, BN) in ((300, 128, 8, 64, 64), (1000, 64, 8, 16, 32), (517, 32, 3, 16, 16)):
        M = n // C
        ng = M * g
        plan = orc.prefill_blocks(n, C, g, BM, BN)
        want = []
        for r0 in range(0, n, BM):
            r1 = min(n, r0 + BM)
            m = r0 // C
            ents = [_entry(b, 0, b * BN + BN <= m * g) for b in range(-(-(m * g) // BN))]
            ents += [_entry(b, 1, b * BN + BN <= r0 + 1)
                     for b in range(m * C // BN, (r1 - 1) // BN + 1)]
            want.append(((0, r0, r1 - r0), ents))
        for r0 in range(0, ng, BM):
            r1 = min(ng, r0 + BM)
            m0, m1 = r0 // g, (r1 - 1) // g
            ents = [_entry(b, 0, b * BN + BN <= min(r0 + 1, ng)) for b in range((r1 - 1) // BN + 1)]
            ents += [_entry(b, 1, m0 == m1 and C % BN == 0)
                     for b in range(m0 * C // BN, ((m1 + 1) * C - 1) // BN + 1)]
            want.append(((1, r0, r1 - r0), ents))
        assert plan == want, (n, C, g, BM, BN)


def pin_prefill_block_sparse_matches_dense(orc):
    """Attention evaluated only over the listed blocks, with the element mask
    applied inside partial blocks and not inside full ones, gives the dense
    masked result (the block mask keeps the defined attention)."""
    B, Hq, Hkv, d, C, g, n_max = 2, 2, 1, 8, 12, 3, 96
    lens = [95, 40]
    BM, BN = 8, 8
    c = _prefill_case(np.random.default_rng(13), B, Hq, Hkv, d, C, g, n_max, lens)
    dense = _prefill(orc, c, C, g)
    for b, n in enumerate(lens):
        M = n // C
        raw_rows, gist_rows, pos_raw, pos_gist = _visible_sets(n, C, g)
        count = (M * g, n)  # columns of part 0 (gists) and part 1 (raw)
        col_pos = (lambda r: pos_gist(r // g, r % g), pos_raw)
        plan = orc.prefill_blocks(n, C, g, BM, BN)
        for (kind, r0, rows), ents in plan:
            for r in range(r0, r0 + rows):
                own, gists = (raw_rows if kind == 0 else gist_rows)[r]
                seen = set(own) | set(gists)
                for h in range(Hq):
                    q = (c["q_raw"][b, h, r] if kind == 0 else c["q_gist"][b, h, r // g, r % g])
                    ks, vs = [], []
                    for e in ents:
                        blk, part, full = e >> 2, (e >> 1) & 1, e & 1
                        for col in range(blk * BN, blk * BN + BN):
                            exists = col < count[part]
                            if not full and not (exists and col_pos[part](col) in seen):
                                continue
                            if part == 0:
                                kv = ((c["k_gist"][b, 0, col // g, col % g],
                                       c["v_gist"][b, 0, col // g, col % g]) if exists
                                      else (np.zeros(d), np.full(d, 1e3)))
                            else:
                                kv = ((c["k_raw"][b, 0, col], c["v_raw"][b, 0, col]) if exists
                                      else (np.zeros(d), np.full(d, 1e3)))
                            ks.append(kv[0])
                            vs.append(kv[1])
                    K = np.asarray(ks, np.float64)
                    V = np.asarray(vs, np.float64)
                    lg = K @ np.asarray(q, np.float64) / math.sqrt(d)
                    w = np.exp(lg - lg.max())
                    out = (w[:, None] * V).sum(0) / w.sum()
                    want = (dense["o_raw"][b, h, r] if kind == 0
                            else dense["o_gist"][b, h, r // g, r % g])
                    _close(out, want, 1e-10, f"b={b} kind={kind} row={r} h={h}")


ALL_PINS = [
    pin_bruteforce_single, pin_given_selection, pin_ties, pin_dense_when_all_selected,
    pin_gists_when_none_selected, pin_single_token, pin_equal_keys_mean, pin_context_size,
    pin_parallel_query, pin_hand_example, pin_bruteforce_h2, pin_h2_reduces_to_single,
    pin_bad_length, pin_nan_gist_key, pin_variants_bruteforce, pin_selected_only_closed_forms,
    pin_union_reductions, pin_hier_bruteforce, pin_hier_reductions,
    pin_adaptive_topk_properties, pin_prefill_one_chunk_is_causal, pin_prefill_visible_sets,
    pin_prefill_last_token_is_decode, pin_prefill_blocks_causal, pin_prefill_blocks_counts,
    pin_prefill_block_sparse_matches_dense,
]

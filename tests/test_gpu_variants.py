"""The context and selection readings of ssa_decode_variant against the fp64
oracle, through the C ABI: the sec. 3.3 "selected chunks only" context and
the App. A per-head selection with a union over the GQA group, on oracle-sized
variants of the workloads (several tiles, ragged tails, odd C and g, k = 0,
k > M) and on the 128K workload at full size (every sequence)."""
import numpy as np
import pytest
import torch

from gist_token_chunk_b200.inputs import WORKLOADS, Workload, make_inputs
from parity import check_variant, host

pytestmark = pytest.mark.gpu

READINGS = [(0, 0), (1, 0), (0, 1), (1, 1)]
RIDS = ["gists_groupmax", "selected_groupmax", "gists_union", "selected_union"]


@pytest.fixture(scope="module")
def ssa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gist_token_chunk_b200 import ssa as mod

    mod.ssa_set_debug_flags(0)
    mod.ssa_set_wait_limit(0)
    return mod


def W(name, **kw):
    base = dict(name=name, B=2, Hq=32, Hkv=8, d=64, n_max=4096, C=64, g=8, topk=16)
    base.update(kw)
    return Workload(**base)


CASES = [
    W("128k_like", n_max=8192, C=128, g=8, topk=32, seq_lens=(8192, 5000), planted=16),
    W("32k_like", n_max=4096, C=64, g=8, topk=16, seq_lens=(4096, 3001), planted=16),
    W("d128", B=2, Hq=8, Hkv=2, d=128, n_max=2048, C=64, g=8, topk=8, seq_lens=(2048, 1500)),
    W("odd_C_g", B=2, Hq=8, Hkv=2, n_max=4800, C=48, g=3, topk=7, seq_lens=(4799, 100)),
    W("topk0", B=2, Hq=8, Hkv=2, n_max=2048, C=64, g=8, topk=0, seq_lens=(2048, 1111)),
    W("dense", B=2, Hq=8, Hkv=2, n_max=2048, C=64, g=8, topk=40, seq_lens=(2048, 1111)),
    W("short", B=4, Hq=8, Hkv=2, n_max=256, C=64, g=8, topk=2, seq_lens=(1, 5, 63, 64)),
    W("fp32_d32", B=2, Hq=4, Hkv=2, d=32, n_max=512, C=16, g=2, topk=5, dtype="fp32",
      seq_lens=(512, 77)),
]


@pytest.mark.parametrize("reading", READINGS, ids=RIDS)
@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_variant_matches_oracle(ssa, orc, w, reading):
    context, select = reading
    inp = make_inputs(w, seed=3000 + len(w.name))
    g = {k: v.cuda() for k, v in inp.items() if k != "planted_idx"}
    out, sel = ssa.ssa_decode_variant(g["q"], g["k_raw"], g["v_raw"], g["k_gist"], g["v_gist"],
                                      g["seq_lens"], w.C, w.g, w.topk, context, select)
    assert ssa.ssa_get_device_status() == 0
    stats = check_variant(orc, inp, w.C, w.g, w.topk, context, select, out, sel)
    print(w.name, reading, stats)


def test_default_reading_equals_ssa_decode(ssa):
    w = CASES[0]
    g = make_inputs(w, seed=9, device="cuda")
    args = (g["q"], g["k_raw"], g["v_raw"], g["k_gist"], g["v_gist"], g["seq_lens"], w.C, w.g,
            w.topk)
    o1, s1 = ssa.ssa_decode(*args)
    o2, s2 = ssa.ssa_decode_variant(*args, 0, 0)
    assert torch.equal(s1, s2)
    assert (o1 - o2).abs().max().item() <= 1e-5


def test_union_contains_group_max_selection_size(ssa):
    """Under the head union every KV head selects between k and G k chunks."""
    w = CASES[1]
    g = make_inputs(w, seed=10, device="cuda")
    _, sel = ssa.ssa_decode_variant(g["q"], g["k_raw"], g["v_raw"], g["k_gist"], g["v_gist"],
                                    g["seq_lens"], w.C, w.g, w.topk, 0, 1)
    s = host(sel)
    G = w.Hq // w.Hkv
    lens = host(g["seq_lens"])
    for b in range(w.B):
        M = int(lens[b]) // w.C
        for j in range(w.Hkv):
            n = int((s[b, j] >= 0).sum())
            assert min(w.topk, M) <= n <= min(G * w.topk, M)
            assert (np.diff(s[b, j][:n]) > 0).all() and (s[b, j][n:] == -1).all()


@pytest.mark.parametrize("reading", READINGS[1:], ids=RIDS[1:])
def test_variant_full_size_128k(ssa, orc, reading):
    context, select = reading
    w = WORKLOADS["llama1b_128k_var"]
    inp = make_inputs(w, seed=1003, device="cuda")
    out, sel = ssa.ssa_decode_variant(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"],
                                      inp["v_gist"], inp["seq_lens"], w.C, w.g, w.topk, context,
                                      select)
    assert ssa.ssa_get_device_status() == 0
    for b in range(w.B):
        one = {k: v[b:b + 1].cpu() for k, v in inp.items() if k != "planted_idx"}
        stats = check_variant(orc, one, w.C, w.g, w.topk, context, select, out[b:b + 1],
                              sel[b:b + 1])
        print("128k", reading, b, stats)

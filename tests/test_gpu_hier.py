"""Coarse-to-fine selection over t levels (ssa_decode_hier) against the fp64
oracle through the C ABI: t = 1, 2 equal the single- and two-level steps;
t = 3, 4 with remainder units, k = 0 at a level, every unit kept at the top,
fp32; and a 1M-token sequence with three levels (every sequence checked)."""
import pytest
import torch

from gist_token_chunk_b200.inputs import Workload, make_inputs, make_level_summaries
from parity import check_hier

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gist_token_chunk_b200 import ssa as mod

    mod.ssa_set_debug_flags(0)
    mod.ssa_set_wait_limit(0)
    return mod


def W(name, **kw):
    base = dict(name=name, B=2, Hq=8, Hkv=2, d=64, n_max=4096, C=16, g=4, topk=8)
    base.update(kw)
    return Workload(**base)


# (workload, J, g_sum of levels 2..t, topk of levels 1..t)
CASES = [
    (W("t3", seq_lens=(4096, 3000), planted=8), 4, [4, 4], [8, 4, 2]),
    (W("t3_odd_J", n_max=4800, C=16, seq_lens=(4799, 1234)), 3, [2, 3], [6, 3, 2]),
    (W("t4", B=1, n_max=8192, C=8, g=2, seq_lens=(8000,)), 4, [2, 2, 2], [8, 4, 2, 2]),
    (W("t3_k0", seq_lens=(4096, 77)), 4, [4, 4], [0, 3, 2]),
    (W("t3_topall", seq_lens=(4096, 2222)), 4, [4, 4], [8, 4, 1000]),
    (W("t3_fp32", B=2, Hq=4, Hkv=2, d=32, n_max=1024, C=8, g=2, dtype="fp32",
       seq_lens=(1024, 600)), 2, [2, 2], [5, 3, 2]),
    (W("t3_d128", B=1, Hq=8, Hkv=2, d=128, n_max=2048, C=16, g=4, seq_lens=(2047,)), 4, [4, 4],
     [6, 3, 2]),
]


def run(ssa, w, J, g_sum, topks, seed):
    """Inputs drawn on the GPU (the oracle reads host copies of them)."""
    g = make_inputs(w, seed=seed, device="cuda")
    g.pop("planted_idx")
    ks, vs = make_level_summaries(w, J, g_sum, seed=seed + 1, device="cuda")
    out, sels = ssa.ssa_decode_hier(g["q"], g["k_raw"], g["v_raw"], g["k_gist"], g["v_gist"],
                                    g["seq_lens"], w.C, w.g, J, ks, vs, topks)
    return g, ks, vs, g, out, sels


@pytest.mark.parametrize("case", CASES, ids=[c[0].name for c in CASES])
def test_hier_matches_oracle(ssa, orc, case):
    w, J, g_sum, topks = case
    inp, ks, vs, _, out, sels = run(ssa, w, J, g_sum, topks, seed=4000 + len(w.name))
    assert ssa.ssa_get_device_status() == 0
    stats = check_hier(orc, inp, ks, vs, w.C, w.g, J, topks, out, sels)
    print(w.name, stats)


def test_one_and_two_levels_equal_the_fixed_steps(ssa):
    w = W("t2", seq_lens=(4096, 3001), planted=8)
    inp = make_inputs(w, seed=11, device="cuda")
    ks, vs = make_level_summaries(w, 4, [4], seed=12, device="cuda")
    a = (inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"], inp["v_gist"], inp["seq_lens"])
    o1, s1 = ssa.ssa_decode_hier(*a, w.C, w.g, 4, [], [], [8])
    r1, rs1 = ssa.ssa_decode(*a, w.C, w.g, 8)
    assert torch.equal(s1[0], rs1)
    assert (o1 - r1).abs().max().item() <= 1e-5
    o2, s2 = ssa.ssa_decode_hier(*a, w.C, w.g, 4, ks, vs, [8, 3])
    r2, rsup, rsel = ssa.ssa_decode_h2(*a[:5], ks[0], vs[0], inp["seq_lens"], w.C, w.g, 4, 4, 3, 8)
    assert torch.equal(s2[0], rsel) and torch.equal(s2[1], rsup)
    assert (o2 - r2).abs().max().item() <= 1e-5


def test_hier_1m_tokens_three_levels(ssa, orc):
    """One 1M-token sequence per batch entry (C=64, g=8: 16384 chunks), J=16:
    1024 level-2 and 64 level-3 units."""
    w = Workload("hier_1m", B=1, Hq=32, Hkv=8, d=64, n_max=1 << 20, C=64, g=8, topk=16,
                 seq_lens=(1 << 20,), planted=16)
    J, g_sum, topks = 16, [8, 8], [16, 8, 4]
    inp, ks, vs, _, out, sels = run(ssa, w, J, g_sum, topks, seed=77)
    assert ssa.ssa_get_device_status() == 0
    stats = check_hier(orc, inp, ks, vs, w.C, w.g, J, topks, out, sels)
    print("1M", stats)

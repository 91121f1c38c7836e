"""Seeded random shapes through every decode entry point, against the fp64
oracle: dtype, head dim, GQA group, C, g, topk (0 to beyond M), lengths from
1 token to the capacity, and each call's reading -- the default step, the two
context readings, the two selection readings, two and three levels.  Every
case is drawn from a fixed seed, so a failure names a reproducible shape."""
import random

import pytest
import torch

from gist_token_chunk_b200.inputs import Workload, make_inputs, make_level_summaries
from parity import check_h2, check_hier, check_single, check_variant

pytestmark = pytest.mark.gpu

N_CASES = 64


def draw(i):
    rnd = random.Random(7000 + i)
    dtype = "bf16" if rnd.random() < 0.75 else "fp32"
    d = rnd.choice([64, 64, 128]) if dtype == "bf16" else rnd.choice([32, 64, 96])
    Hkv = rnd.choice([1, 2, 4])
    G = rnd.choice([1, 2, 4, 8])
    C = rnd.choice([8, 16, 32, 64])
    g = rnd.choice([1, 2, 3, 4, 8])
    M_max = rnd.randint(4, 48)
    n_max = C * M_max
    B = rnd.randint(1, 3)
    lens = tuple(rnd.choice([1, rnd.randint(1, n_max), n_max, n_max - rnd.randint(0, C - 1)])
                 for _ in range(B))
    topk = rnd.choice([0, 1, rnd.randint(1, 12), rnd.randint(10, 60)])
    kind = rnd.choice(["decode", "decode", "variant", "h2", "hier3"])
    reading = (rnd.randint(0, 1), rnd.randint(0, 1))
    w = Workload(f"fuzz{i}", B=B, Hq=Hkv * G, Hkv=Hkv, d=d, n_max=n_max, C=C, g=g, topk=topk,
                 dtype=dtype, seq_lens=lens)
    return w, kind, reading, rnd


CASES = [draw(i) for i in range(N_CASES)]


@pytest.fixture(scope="module")
def ssa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gist_token_chunk_b200 import ssa as mod

    mod.ssa_set_debug_flags(0)
    mod.ssa_set_wait_limit(0)
    return mod


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0].name}-{c[1]}" for c in CASES])
def test_fuzz_against_oracle(ssa, orc, case):
    w, kind, reading, rnd = case
    seed = 9000 + int(w.name[4:])
    inp = make_inputs(w, seed=seed)
    g = {k: v.cuda() for k, v in inp.items() if k != "planted_idx"}
    a = (g["q"], g["k_raw"], g["v_raw"], g["k_gist"], g["v_gist"], g["seq_lens"])
    if kind == "decode":
        out, sel = ssa.ssa_decode(*a, w.C, w.g, w.topk)
        assert ssa.ssa_get_device_status() == 0
        check_single(orc, inp, w.C, w.g, w.topk, out, sel)
    elif kind == "variant":
        out, sel = ssa.ssa_decode_variant(*a, w.C, w.g, w.topk, *reading)
        assert ssa.ssa_get_device_status() == 0
        check_variant(orc, inp, w.C, w.g, w.topk, reading[0], reading[1], out, sel)
    elif kind == "h2":
        J = rnd.choice([2, 3, 4])
        gm = rnd.choice([1, 2, 4])
        ks = rnd.choice([0, 1, 3, 50])
        k_sum, v_sum = make_level_summaries(w, J, [gm], seed=seed + 1)
        out, sup, sel = ssa.ssa_decode_h2(*a[:5], k_sum[0].cuda(), v_sum[0].cuda(),
                                          g["seq_lens"], w.C, w.g, J, gm, ks, w.topk)
        assert ssa.ssa_get_device_status() == 0
        one = dict(inp, k_meta=k_sum[0], v_meta=v_sum[0])
        check_h2(orc, one, w.C, w.g, J, gm, ks, w.topk, out, sup, sel)
    else:
        J = rnd.choice([2, 3])
        g_sum = [rnd.choice([1, 2, 3]), rnd.choice([1, 2])]
        topks = [w.topk, rnd.choice([0, 1, 4]), rnd.choice([1, 2, 30])]
        k_sum, v_sum = make_level_summaries(w, J, g_sum, seed=seed + 2)
        out, sels = ssa.ssa_decode_hier(*a, w.C, w.g, J, [x.cuda() for x in k_sum],
                                        [x.cuda() for x in v_sum], topks)
        assert ssa.ssa_get_device_status() == 0
        check_hier(orc, inp, k_sum, v_sum, w.C, w.g, J, topks, out, sels)

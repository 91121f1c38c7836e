"""CUDA path (through the C ABI) against the fp64 oracle, element by element.

Bars (the accuracy criteria of this path, applied in tests/parity.py): selections bit-exact
unless the oracle's k-th/(k+1)-th score gap is <= 1e-4 (then the GPU's choice
must be a valid top-k and the oracle is re-run on it); outputs within max-abs
1e-2 and mean-abs 1e-3 of the oracle.

* oracle-sized variants of the five workloads (several tiles per sequence,
  ragged tails) and edge cases, checked on every output;
* the five workloads at full size, in the launch configuration the bench
  times, checked on every sequence (the oracle recomputes them one by one);
* the two single-level bf16 paths (two-kernel pipeline, one-kernel fused
  kernel) against each other at full size.
"""
import numpy as np
import pytest
import torch

from gist_token_chunk_b200.inputs import WORKLOADS, Workload, make_inputs
from parity import check_h2, check_single, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gist_token_chunk_b200 import ssa as mod

    mod.ssa_set_tuning(0, 0)
    mod.ssa_set_debug_flags(0)
    mod.ssa_set_wait_limit(0)
    return mod


def to_dev(inp, dev="cuda"):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) and k != "planted_idx" else v)
            for k, v in inp.items()}


def W(name, **kw):
    base = dict(name=name, B=2, Hq=32, Hkv=8, d=64, n_max=4096, C=64, g=8, topk=16)
    base.update(kw)
    return Workload(**base)


SINGLE = [
    WORKLOADS["tiny_fp32"],
    W("32k_like", n_max=4096, C=64, g=8, topk=16, seq_lens=(4096, 3001), planted=16),
    W("128k_like", n_max=8192, C=128, g=8, topk=32, seq_lens=(8192, 5000), planted=16),
    W("512k_like", B=1, n_max=32768, C=256, g=8, topk=64, seq_lens=(32768,), planted_frac=0.05),
    W("gqa1", B=1, Hq=4, Hkv=4, n_max=2048, C=64, g=8, topk=8, seq_lens=(2000,)),
    W("gqa8", B=1, Hq=16, Hkv=2, n_max=2048, C=32, g=4, topk=10, seq_lens=(2047,)),
    W("gqa16", B=1, Hq=16, Hkv=1, n_max=1024, C=64, g=8, topk=4, seq_lens=(1024,)),
    W("d128", B=2, Hq=8, Hkv=2, d=128, n_max=2048, C=64, g=8, topk=8, seq_lens=(2048, 1500)),
    W("odd_C_g", B=2, Hq=8, Hkv=2, n_max=4800, C=48, g=3, topk=7, seq_lens=(4799, 100)),
    W("g1_C16", B=1, Hq=8, Hkv=2, n_max=2048, C=16, g=1, topk=20, seq_lens=(2040,)),
    W("big_g", B=1, Hq=8, Hkv=2, n_max=8192, C=256, g=64, topk=4, seq_lens=(8000,)),
    W("topk0", B=2, Hq=8, Hkv=2, n_max=2048, C=64, g=8, topk=0, seq_lens=(2048, 1111)),
    W("dense", B=2, Hq=8, Hkv=2, n_max=2048, C=64, g=8, topk=32, seq_lens=(2048, 1111)),
    W("short", B=4, Hq=8, Hkv=2, n_max=256, C=64, g=8, topk=2, seq_lens=(1, 5, 63, 64)),
    W("fp32_d32", B=2, Hq=4, Hkv=2, d=32, n_max=512, C=16, g=2, topk=5, dtype="fp32",
      seq_lens=(512, 77)),
    W("fp32_d64", B=1, Hq=8, Hkv=2, d=64, n_max=1024, C=32, g=4, topk=6, dtype="fp32",
      seq_lens=(1000,)),
]


@pytest.mark.parametrize("w", SINGLE, ids=[w.name for w in SINGLE])
def test_decode_matches_oracle(ssa, orc, w):
    inp = make_inputs(w, seed=1000 + len(w.name))
    g = to_dev(inp)
    out, sel = ssa.ssa_decode(g["q"], g["k_raw"], g["v_raw"], g["k_gist"], g["v_gist"],
                              g["seq_lens"], w.C, w.g, w.topk)
    assert ssa.ssa_get_device_status() == 0
    stats = check_single(orc, inp, w.C, w.g, w.topk, out, sel)
    print(w.name, stats)


@pytest.mark.parametrize("w", SINGLE[:4] + SINGLE[7:9] + SINGLE[-2:],
                         ids=[w.name for w in SINGLE[:4] + SINGLE[7:9] + SINGLE[-2:]])
def test_components_match_oracle(ssa, orc, w):
    """ssa_score_gists -> ssa_topk_chunks -> ssa_sparse_decode, each vs the oracle."""
    inp = make_inputs(w, seed=77)
    g = to_dev(inp)
    ref = orc.decode(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"], inp["v_gist"],
                     inp["seq_lens"], C=w.C, g=w.g, topk=w.topk)
    scores = ssa.ssa_score_gists(g["q"], g["k_gist"], g["seq_lens"], w.C, w.g, w.n_max)
    s = host(scores).astype(np.float64)
    fin = np.isfinite(ref["scores"])
    assert np.array_equal(np.isfinite(s), fin)
    assert (s[~fin] == -np.inf).all()
    assert np.abs(s[fin] - ref["scores"][fin]).max() <= 1e-4 * max(1.0, np.abs(ref["scores"][fin]).max())
    sel = ssa.ssa_topk_chunks(scores, g["seq_lens"], w.C, w.topk, w.n_max)
    # the GPU's top-k on the GPU's scores must be exactly the top-k definition on them
    gsel = host(sel)
    lens = host(inp["seq_lens"])
    for b in range(w.B):
        M = int(lens[b]) // w.C
        k = min(w.topk, M)
        for j in range(w.Hkv):
            order = sorted(range(M), key=lambda m: (-s[b, j, m], m))[:k]
            want = sorted(order) + [-1] * (w.topk - k)
            assert list(gsel[b, j]) == want, (b, j)
    out = ssa.ssa_sparse_decode(g["q"], g["k_raw"], g["v_raw"], g["k_gist"], g["v_gist"],
                                g["seq_lens"], w.C, w.g, w.topk, sel)
    assert ssa.ssa_get_device_status() == 0
    ref2 = orc.decode(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"], inp["v_gist"],
                      inp["seq_lens"], C=w.C, g=w.g, topk=w.topk, sel=gsel)
    err = np.abs(host(out) - ref2["out"])
    assert err.max() <= 1e-2 and err.mean() <= 1e-3, (err.max(), err.mean())


H2 = [
    W("hssa_like", B=2, n_max=16384, C=64, g=8, J=16, gm=8, topk_super=8, topk=16,
      seq_lens=(16384, 16384), planted=16),
    W("hssa_rem_tail", B=2, n_max=16384, C=64, g=8, J=16, gm=8, topk_super=4, topk=16,
      seq_lens=(16384, 13000), planted=8),
    W("hssa_small_J", B=1, Hq=8, Hkv=2, n_max=4096, C=32, g=4, J=5, gm=3, topk_super=3,
      topk=7, seq_lens=(4000,)),
    W("hssa_all_super", B=1, Hq=8, Hkv=2, n_max=4096, C=64, g=8, J=4, gm=2, topk_super=64,
      topk=6, seq_lens=(4000,)),
    W("hssa_fp32", B=1, Hq=4, Hkv=2, d=32, n_max=1024, C=16, g=2, J=4, gm=2, topk_super=3,
      topk=5, dtype="fp32", seq_lens=(1000,)),
]


@pytest.mark.parametrize("w", H2, ids=[w.name for w in H2])
def test_decode_h2_matches_oracle(ssa, orc, w):
    inp = make_inputs(w, seed=2000 + len(w.name))
    g = to_dev(inp)
    out, sup, sel = ssa.ssa_decode_h2(g["q"], g["k_raw"], g["v_raw"], g["k_gist"], g["v_gist"],
                                      g["k_meta"], g["v_meta"], g["seq_lens"], w.C, w.g, w.J,
                                      w.gm, w.topk_super, w.topk)
    assert ssa.ssa_get_device_status() == 0
    stats = check_h2(orc, inp, w.C, w.g, w.J, w.gm, w.topk_super, w.topk, out, sup, sel)
    print(w.name, stats)


def test_h2_with_all_superchunks_equals_single_level(ssa):
    w = H2[3]
    inp = to_dev(make_inputs(w, seed=5))
    out2, _, sel2 = ssa.ssa_decode_h2(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"],
                                      inp["v_gist"], inp["k_meta"], inp["v_meta"],
                                      inp["seq_lens"], w.C, w.g, w.J, w.gm, 1000, w.topk)
    out1, sel1 = ssa.ssa_decode(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"],
                                inp["v_gist"], inp["seq_lens"], w.C, w.g, w.topk)
    assert torch.equal(sel1, sel2)
    assert (out1 - out2).abs().max().item() <= 1e-5


# ---------------------------------------------------------------- full size

def sample_seq(inp, b):
    """Host copy of sequence b's inputs (the oracle checks one sequence at a time)."""
    out = {}
    for k, v in inp.items():
        if k == "planted_idx":
            continue
        out[k] = v[b:b + 1].cpu()
    return out


@pytest.mark.parametrize("name", ["llama1b_32k", "llama1b_128k_var", "llama1b_512k"])
def test_full_size_sampled(ssa, orc, name):
    w = WORKLOADS[name]
    inp = make_inputs(w, seed=1000 + list(WORKLOADS).index(name) + 1, device="cuda")
    out, sel = ssa.ssa_decode(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"],
                              inp["v_gist"], inp["seq_lens"], w.C, w.g, w.topk)
    assert ssa.ssa_get_device_status() == 0
    for b in range(w.B):  # every sequence, one at a time through the oracle
        one = sample_seq(inp, b)
        stats = check_single(orc, one, w.C, w.g, w.topk, out[b:b + 1], sel[b:b + 1])
        print(name, b, stats)


def test_full_size_h2_sampled(ssa, orc):
    w = WORKLOADS["hssa_128k"]
    inp = make_inputs(w, seed=1005, device="cuda")
    out, sup, sel = ssa.ssa_decode_h2(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"],
                                      inp["v_gist"], inp["k_meta"], inp["v_meta"],
                                      inp["seq_lens"], w.C, w.g, w.J, w.gm, w.topk_super, w.topk)
    assert ssa.ssa_get_device_status() == 0
    for b in range(w.B):
        one = sample_seq(inp, b)
        stats = check_h2(orc, one, w.C, w.g, w.J, w.gm, w.topk_super, w.topk, out[b:b + 1],
                         sup[b:b + 1], sel[b:b + 1])
        print("hssa_128k", b, stats)


@pytest.mark.parametrize("M,topk,levels", [
    (1024, 32, 0),      # continuous scores: filtered path
    (2048, 64, 4),      # 4 distinct values: many ties at the boundary
    (2048, 200, 0),     # k > 128: radix path
    (2048, 64, 1),      # all equal: more candidates than the filter keeps
    (777, 100, 9),      # ragged length, ties
    (4096, 1, 0),
])
def test_topk_ties_and_paths(ssa, M, topk, levels):
    """ssa_topk_chunks on given scores equals the top-k definition on those
    same fp32 values: largest first, ties to the lower index, ascending."""
    B, Hkv, C = 2, 3, 16
    g = torch.Generator().manual_seed(M + topk)
    sc = torch.randn(B, Hkv, M, generator=g)
    if levels:
        sc = torch.randint(0, levels, (B, Hkv, M), generator=g).float()
    sc[:, 1, 5] = float("nan")          # NaN ranks as -inf
    sc[:, 2, 7] = -0.0                  # -0 and +0 compare equal
    lens = torch.tensor([M * C, (M - 3) * C + 5], dtype=torch.int32)
    sel = ssa.ssa_topk_chunks(sc.cuda(), lens.cuda(), C, topk, M * C)
    got = sel.cpu().numpy()
    for b in range(B):
        Mb = int(lens[b]) // C
        k = min(topk, Mb)
        for j in range(Hkv):
            v = sc[b, j, :Mb].double().numpy()
            v = np.where(np.isnan(v), -np.inf, v)
            order = sorted(range(Mb), key=lambda m: (-v[m], m))[:k]
            want = sorted(order) + [-1] * (topk - k)
            assert list(got[b, j]) == want, (b, j)


@pytest.mark.parametrize("name", ["llama1b_32k", "llama1b_128k_var", "llama1b_512k"])
def test_pipeline_and_fused_path_agree(ssa, name):
    """The two single-level bf16 paths compute the same selection, and the
    same output up to fp32 summation order, on the full-size workloads."""
    w = WORKLOADS[name]
    inp = make_inputs(w, seed=31, device="cuda")
    args = (inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"], inp["v_gist"], inp["seq_lens"],
            w.C, w.g, w.topk)
    out_p, sel_p = ssa.ssa_decode(*args)
    ssa.ssa_set_debug_flags(ssa.SSA_DEBUG_FUSED_PATH)
    try:
        out_f, sel_f = ssa.ssa_decode(*args)
    finally:
        ssa.ssa_set_debug_flags(0)
    assert ssa.ssa_get_device_status() == 0
    assert torch.equal(sel_p, sel_f)
    assert (out_p - out_f).abs().max().item() <= 1e-5


@pytest.mark.parametrize("flags", [0, 2], ids=["pipeline", "fused"])
def test_nan_gist_keys(ssa, orc, flags):
    """NaN gist keys: a NaN logit never wins a chunk's score maximum, a chunk
    of NaN keys scores -inf and is left out, and a NaN key left in the
    context makes that KV head's outputs NaN -- as in the oracle."""
    w = W("nan", B=1, Hq=8, Hkv=2, n_max=2048, C=64, g=8, topk=4, seq_lens=(2000,))
    inp = make_inputs(w, seed=8)
    kg = inp["k_gist"]
    q = inp["q"].float()
    boost = q[0, :4].sum(0)
    kg[0, 0, 2, 0] = (boost / boost.norm() * 6.0).to(kg.dtype)   # chunk 2 wins for KV head 0
    kg[0, 0, 2, 1, 3] = float("nan")                              # ... despite one NaN key
    kg[0, 0, 5] = float("nan")                                    # chunk 5 of head 0: all NaN
    ref = orc.decode(inp["q"], inp["k_raw"], inp["v_raw"], kg, inp["v_gist"], inp["seq_lens"],
                     C=w.C, g=w.g, topk=w.topk)
    g = to_dev(inp)
    ssa.ssa_set_debug_flags(flags)
    try:
        out, sel = ssa.ssa_decode(g["q"], g["k_raw"], g["v_raw"], g["k_gist"], g["v_gist"],
                                  g["seq_lens"], w.C, w.g, w.topk)
    finally:
        ssa.ssa_set_debug_flags(0)
    assert ssa.ssa_get_device_status() == 0
    s = host(sel)
    assert 2 in s[0, 0] and 5 not in s[0, 0]
    assert np.array_equal(s, ref["sel_idx"])
    o = host(out)
    nan_ref = np.isnan(ref["out"])
    assert nan_ref[0, :4].all()          # KV head 0 keeps chunk 5's NaN gist keys
    assert not nan_ref[0, 4:].any()      # KV head 1 has none
    assert np.array_equal(np.isnan(o), nan_ref)
    err = np.abs(o[~nan_ref] - ref["out"][~nan_ref])
    assert err.max() <= 1e-2 and err.mean() <= 1e-3


def test_pipeline_at_its_chunk_limit(ssa, orc):
    """8192 chunks per sequence (512K tokens, C = 64), the most the two-kernel
    pipeline takes: its top-k falls back from the 128-candidate path to the
    radix path, and the score rows are longest."""
    w = Workload("chunk_limit", B=1, Hq=32, Hkv=8, d=64, n_max=524288, C=64, g=8, topk=64,
                 seq_lens=(524288 - 37,), planted=64)
    sh = ssa.make_shape(w.B, w.Hq, w.Hkv, w.d, w.n_max, ssa.SSA_BF16)
    assert ssa.ssa_decode_path(sh, w.C, w.g, w.topk) == ssa.SSA_PATH_PIPELINE
    inp = make_inputs(w, seed=8192, device="cuda")
    out, sel = ssa.ssa_decode(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"],
                              inp["v_gist"], inp["seq_lens"], w.C, w.g, w.topk)
    assert ssa.ssa_get_device_status() == 0
    stats = check_single(orc, sample_seq(inp, 0), w.C, w.g, w.topk, out, sel)
    print("chunk_limit", stats)

"""The prefill kernel against the fp64 oracle (GPU).

Every case runs the library's block plan and ssa_prefill on cuda:0 and
compares each valid output row with the oracle's dense masked attention
(sec. 3.1) on the same bf16 inputs.  Small cases compare every row; the
32K-token workload the bench times (Llama-3.2-1B attention: 32/8 heads,
d = 64, C = 128, g = 8) compares a spread of sampled rows.  Tolerance: the
decode path's (max 1e-2, mean 1e-3 absolute); the kernel's own error is fp32
summation order plus the residue of P after its bf16 pair (about 2^-17
relative), far below it.
"""
import numpy as np
import pytest
import torch

from parity import MAX_ABS, MEAN_ABS

pytestmark = pytest.mark.gpu


def _inputs(B, Hq, Hkv, d, C, g, n_max, seed, q_scale=1.0):
    gen = torch.Generator().manual_seed(seed)
    M_max = n_max // C
    f = lambda *s: torch.randn(*s, generator=gen).to(torch.bfloat16)
    x = {"q_raw": f(B, Hq, n_max, d), "q_gist": f(B, Hq, M_max, g, d),
         "k_raw": f(B, Hkv, n_max, d), "k_gist": f(B, Hkv, M_max, g, d),
         "v_raw": f(B, Hkv, n_max, d), "v_gist": f(B, Hkv, M_max, g, d)}
    if q_scale != 1.0:
        x["q_raw"] = (x["q_raw"].float() * q_scale).to(torch.bfloat16)
        x["q_gist"] = (x["q_gist"].float() * q_scale).to(torch.bfloat16)
    return x


def _run(x, lens, C, g):
    from gist_token_chunk_b200 import ssa

    n_max = x["q_raw"].shape[2]
    tiles, entries = ssa.ssa_prefill_plan(lens, n_max, C, g)
    dev = {k: v.cuda() for k, v in x.items()}
    o_raw = torch.full(tuple(x["q_raw"].shape), float("nan"), device="cuda")
    o_gist = torch.full(tuple(x["q_gist"].shape), float("nan"), device="cuda")
    ssa.ssa_prefill(dev["q_raw"], dev["q_gist"], dev["k_raw"], dev["k_gist"], dev["v_raw"],
                    dev["v_gist"], C, g, tiles.cuda(), entries.cuda(), o_raw, o_gist)
    torch.cuda.synchronize()
    assert ssa.ssa_prefill_get_status() == 0
    return o_raw.cpu().numpy(), o_gist.cpu().numpy()


def _compare(got, want, what):
    got = np.asarray(got, np.float64)
    assert got.shape == np.shape(want), (what, got.shape, np.shape(want))
    if got.size == 0:  # an empty sequence has no rows
        return
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - want)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, \
        f"{what}: max {err.max():.3g} mean {err.mean():.3g}"


# (B, Hq, Hkv, d, C, g, n_max, seq_lens, q_scale): chunks of two tiles with a
# tail; chunks shorter than a tile and an empty sequence; d = 128, C not a
# multiple of the block, no grouping; more gists than a tile; no complete
# chunk; a sharp softmax (queries x 4)
CASES = [
    (2, 4, 2, 64, 128, 8, 1024, [1024, 777], 1.0),
    (3, 8, 2, 64, 16, 2, 768, [768, 700, 0], 1.0),
    (2, 4, 4, 128, 100, 7, 1000, [1000, 450], 1.0),
    (1, 16, 1, 64, 64, 80, 256, [256], 1.0),
    (2, 2, 1, 64, 128, 8, 512, [100, 5], 1.0),
    (1, 4, 2, 64, 128, 8, 4096, [4096], 4.0),
    (2, 8, 2, 128, 32, 3, 2048, [2047, 1600], 1.0),
]


@pytest.mark.parametrize("B, Hq, Hkv, d, C, g, n_max, lens, q_scale", CASES)
def test_prefill_matches_oracle(orc, B, Hq, Hkv, d, C, g, n_max, lens, q_scale):
    x = _inputs(B, Hq, Hkv, d, C, g, n_max, seed=B * 1000 + n_max + C, q_scale=q_scale)
    o_raw, o_gist = _run(x, lens, C, g)
    ref = orc.prefill(x["q_raw"], x["q_gist"], x["k_raw"], x["k_gist"], x["v_raw"], x["v_gist"],
                      np.asarray(lens, np.int32), C, g)
    for b, n in enumerate(lens):
        ng = (n // C) * g
        _compare(o_raw[b, :, :n], ref["o_raw"][b, :, :n], f"raw rows b={b}")
        if ng:
            got = o_gist[b].reshape(Hq, -1, d)[:, :ng]
            want = ref["o_gist"][b].reshape(Hq, -1, d)[:, :ng]
            _compare(got, want, f"gist rows b={b}")
        # rows past the sequence are not written
        assert np.isnan(o_raw[b, :, n:]).all()
        assert np.isnan(o_gist[b].reshape(Hq, -1, d)[:, ng:]).all()


def _sample_rows(rng, B, Hq, lens, C, g, per_seq):
    rows = []
    for b, n in enumerate(lens):
        ng = (n // C) * g
        picks = [(0, 0), (0, n - 1), (0, min(n - 1, 63)), (0, min(n - 1, 64))]
        if ng:
            picks += [(1, 0), (1, ng - 1), (1, ng // 2)]
        picks += [(0, int(r)) for r in rng.integers(0, n, per_seq)]
        if ng:
            picks += [(1, int(r)) for r in rng.integers(0, ng, per_seq // 4 + 1)]
        for part, r in picks:
            rows.append((b, int(rng.integers(0, Hq)), part, r))
    return rows


@pytest.mark.parametrize("B, Hq, Hkv, d, C, g, n_max, lens", [
    (1, 32, 8, 64, 128, 8, 32768, [32768]),
    (2, 8, 2, 128, 64, 4, 8192, [8191, 3000]),
])
def test_prefill_large_sampled_rows(orc, B, Hq, Hkv, d, C, g, n_max, lens):
    x = _inputs(B, Hq, Hkv, d, C, g, n_max, seed=7 + n_max)
    o_raw, o_gist = _run(x, lens, C, g)
    rows = _sample_rows(np.random.default_rng(3), B, Hq, lens, C, g, per_seq=40)
    want = orc.prefill_rows(x["q_raw"], x["q_gist"], x["k_raw"], x["k_gist"], x["v_raw"],
                            x["v_gist"], np.asarray(lens, np.int32), C, g, rows)
    got = np.stack([o_raw[b, h, r] if part == 0 else o_gist[b, h, r // g, r % g]
                    for b, h, part, r in rows])
    _compare(got, want, "sampled rows")


def test_prefill_bad_plan_is_reported_not_followed():
    """A plan that does not fit the arrays: the kernel skips what is out of
    range, writes nothing for a skipped tile and records the device status."""
    from gist_token_chunk_b200 import ssa

    B, Hq, Hkv, d, C, g, n_max = 1, 4, 2, 64, 64, 4, 512
    lens = [512]
    x = _inputs(B, Hq, Hkv, d, C, g, n_max, seed=11)
    tiles, entries = ssa.ssa_prefill_plan(lens, n_max, C, g)
    bad_t = tiles.clone()
    bad_t[0, 0] = 5          # sequence out of range
    bad_e = entries.clone()
    last = int(bad_t[-1, 5])
    bad_e[last] = (1 << 20) << 2 | 2  # a raw block far past the end
    dev = {k: v.cuda() for k, v in x.items()}
    o_raw = torch.full((B, Hq, n_max, d), float("nan"), device="cuda")
    o_gist = torch.full((B, Hq, n_max // C, g, d), float("nan"), device="cuda")
    ssa.ssa_prefill_get_status()
    ssa.ssa_prefill(dev["q_raw"], dev["q_gist"], dev["k_raw"], dev["k_gist"], dev["v_raw"],
                    dev["v_gist"], C, g, bad_t.cuda(), bad_e.cuda(), o_raw, o_gist)
    torch.cuda.synchronize()
    assert ssa.ssa_prefill_get_status() == ssa.SSA_ERR_DEVICE_STATUS
    kind, r0, rows = (int(v) for v in tiles[0, 1:4])
    skipped = (o_raw[0, :, r0:r0 + rows] if kind == 0
               else o_gist[0].reshape(Hq, -1, d)[:, r0:r0 + rows])
    assert torch.isnan(skipped).all()
    assert ssa.ssa_prefill_get_status() == 0

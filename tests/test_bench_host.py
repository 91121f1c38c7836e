"""bench.py's reference arm (the fp64 oracle timed on the host cores) runs
without a GPU and prints one JSON line with the keys the bench contract
asks for."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_line():
    r = subprocess.run(
        [sys.executable, "bench.py", "--impl", "reference", "--config", "tiny_fp32", "--steps", "2",
         "--warmup", "3"],
        cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, lines
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 3
    assert d["config"]["workload"] == "tiny_fp32"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"]


# ------------------------------------------------ the bench's bytes models

def _bench():
    import importlib.util

    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _fixed(w, sel_entries):
    """q, out, selection and lengths: the bytes every model adds per step."""
    e = 2 if w.dtype == "bf16" else 4
    return w.B * w.Hq * w.d * e + w.B * w.Hq * w.d * 4 + sel_entries * 4 + w.B * 4


def test_bytes_models_match_the_oracles_context_sizes(orc):
    """Every context row is read as a key and a value. The models add the
    summary keys that are scored but not attended: the selected chunks' gists
    (unselected-gist context), the unselected chunks' gists (selected-only
    context), the kept units' summaries at every level (t levels). So
    model = e d (2 |X| + those rows) + the fixed bytes, with |X| the oracle's
    own context count."""
    import numpy as np

    sys.path.insert(0, ROOT)
    from gist_token_chunk_b200.inputs import Workload, make_inputs, make_level_summaries

    bench = _bench()
    w = Workload("bytes", B=3, Hq=8, Hkv=2, d=16, n_max=640, C=16, g=4, topk=5,
                 seq_lens=(640, 333, 40), dtype="fp32")
    x = make_inputs(w, seed=3)
    a = (x["q"], x["k_raw"], x["v_raw"], x["k_gist"], x["v_gist"], x["seq_lens"])
    lens = [int(v) for v in x["seq_lens"]]
    e = 4
    for context in (0, 1):
        for select in (0, 1):
            r = orc.decode(*a, C=w.C, g=w.g, topk=w.topk, context=context, select=select)
            sel = r["sel_idx"]
            extra = 0
            for b, n in enumerate(lens):
                M = n // w.C
                for j in range(w.Hkv):
                    k = int((sel[b, j] >= 0).sum())
                    extra += (k if context == 0 else M - k) * w.g
            want = e * w.d * (2 * int(r["ctx"].sum()) + extra) + _fixed(w, sel.size)
            if context == 0 and select == 0:
                got = bench.algorithmic_bytes(w, lens)
                assert got == want, (got, want)
            got = bench.variant_bytes(w, lens, sel, context)
            assert got == want, (context, select, got, want)
    # t levels
    J, g_sum, topks = 3, [2, 3], [4, 2, 1]
    ks, vs = make_level_summaries(w, J, g_sum, seed=4)
    r = orc.decode_hier(*a[:5], ks, vs, x["seq_lens"], C=w.C, g=w.g, J=J, topks=topks)
    gl = [w.g] + g_sum
    extra = sum(int((r["sels"][l] >= 0).sum()) * gl[l] for l in range(len(topks)))
    want = e * w.d * (2 * int(r["ctx"].sum()) + extra) + _fixed(w, sum(s.size for s in r["sels"]))
    got = bench.hier_bytes(w, lens, [np.asarray(s) for s in r["sels"]], J, g_sum, topks)
    assert got == want, (got, want)


def test_prefill_pair_count_matches_the_mask():
    """The bench's count of kept (query, key) pairs against a pair-by-pair
    walk of the interleaved sequence under the sec. 3.1 mask."""
    import bench

    for n, C, g in ((300, 128, 8), (517, 32, 3), (64, 64, 2), (1, 8, 2), (129, 16, 5)):
        M = n // C
        pos = {}
        for i in range(n):
            m = i // C
            pos[("r", i)] = (m * (C + g) + i % C if m < M else M * (C + g) + i - M * C, m, False)
        for m in range(M):
            for t in range(g):
                pos[("g", m * g + t)] = (m * (C + g) + C + t, m, True)
        want = sum(1 for pq, mq, _ in pos.values() for pk, mk, gk in pos.values()
                   if pk <= pq and (mk == mq or (gk and mk < mq)))
        assert bench.prefill_visible_pairs(n, C, g) == want, (n, C, g)
